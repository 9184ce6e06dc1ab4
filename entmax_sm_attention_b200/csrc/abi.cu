// abi.cu -- the C ABI of libentmax_attn.so (declared and documented in
// include/entmax_attn.h): argument checks, workspace layout, TMA descriptors, launches.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <cmath>
#include <cstdint>
#include <cstring>

#include "../../include/entmax_attn.h"
#include "common.cuh"
#include "kernels.h"

using namespace entmax;

namespace {

constexpr int kDefaultSweeps = 12;
constexpr int kMaxSweeps = 64;
constexpr float kMaxAlpha = 16.f;   // largest alpha accepted (u^{1/(alpha-1)} keeps fp32 sense)

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Workspace layout. Everything the forward writes comes first (up to fwd_total); the
// backward-only parts follow.
struct Layout {
  int BH, Tr, Tc, Wc, Wr, W64c, W64r;
  size_t off_status, off_M, off_MT, off_M64T, off_M64, off_sumg, off_Ot, off_stats, off_v16, fwd_total;
  size_t off_delta, off_bstats, off_do16, total;
  size_t bytes_M, bytes_MT, bytes_M64T, bytes_M64, bytes_stats, bytes_bstats;
};

bool layout_of(const entmax_attn_desc* d, Layout* l) {
  l->BH = d->B * d->H;
  l->Tr = (d->L + kTile - 1) / kTile;
  l->Tc = l->Tr;
  l->Wc = (l->Tc + 31) / 32;
  l->Wr = (l->Tr + 31) / 32;
  l->W64c = (2 * l->Tc + 31) / 32;
  l->W64r = (2 * l->Tr + 31) / 32;
  const size_t rows = (size_t)l->BH * d->L;
  size_t off = 0;
  l->off_status = off;
  off += 256;
  l->off_M = off;
  l->bytes_M = (size_t)l->BH * l->Tr * l->Wc * 4;
  off += align256(l->bytes_M);
  l->off_MT = off;
  l->bytes_MT = (size_t)l->BH * l->Tc * l->Wr * 4;
  off += align256(l->bytes_MT);
  l->off_sumg = off;
  off += align256(rows * 4);
  l->off_Ot = off;
  off += align256(rows * kD * 4);
  l->off_stats = off;
  l->bytes_stats = (size_t)l->BH * l->Tr * kFwdStats * 4;
  off += align256(l->bytes_stats);
  l->off_v16 = off;
  off += align256(rows * kD * 2);
  l->off_M64T = off;
  l->bytes_M64T = (size_t)l->BH * 2 * l->Tc * l->W64r * 4;
  off += align256(l->bytes_M64T);
  l->off_M64 = off;
  l->bytes_M64 = (size_t)l->BH * 2 * l->Tr * l->W64c * 4;
  off += align256(l->bytes_M64);
  l->fwd_total = off;
  l->off_delta = off;
  off += align256(rows * 4);
  l->off_bstats = off;
  l->bytes_bstats = (size_t)l->BH * l->Tc * kBwdStats * 4;
  off += align256(l->bytes_bstats);
  l->off_do16 = off;
  off += align256(rows * kD * 2);
  l->total = off;
  return true;
}

entmax_status check_desc(const entmax_attn_desc* d) {
  if (!d) return ENTMAX_EINVAL;
  if (d->B < 1 || d->H < 1 || d->L < 1 || d->d < 1) return ENTMAX_EINVAL;
  if ((long long)d->B * d->H * d->L > (1ll << 31)) return ENTMAX_EINVAL;
  if (!(d->scale > 0.f) || !std::isfinite(d->scale)) return ENTMAX_EINVAL;
  if (d->causal != 0 && d->causal != 1) return ENTMAX_EINVAL;
  if (d->max_sweeps < 0 || d->max_sweeps > kMaxSweeps) return ENTMAX_EINVAL;
  if (d->dtype != ENTMAX_BF16 && d->dtype != ENTMAX_FP32) return ENTMAX_EINVAL;
  if (d->wait_limit_us < 0) return ENTMAX_EINVAL;
  if (d->selftest != 0 && d->selftest != ENTMAX_SELFTEST_STALL) return ENTMAX_EINVAL;
  if (d->mask64 != 0 && d->mask64 != 1) return ENTMAX_EINVAL;
  if (d->d != kD) return ENTMAX_EUNSUPPORTED;
  if (d->L > ENTMAX_MAX_L) return ENTMAX_EUNSUPPORTED;
  if (!(d->alpha > 1.0f) || !std::isfinite(d->alpha)) return ENTMAX_EINVAL;
  if (d->alpha > kMaxAlpha) return ENTMAX_EUNSUPPORTED;
  // fp32 inputs: the CUDA-core forward has closed-form powers for alpha in {1.5, 2} only.
  if (d->dtype == ENTMAX_FP32 && d->alpha != 1.5f && d->alpha != 2.0f) return ENTMAX_EUNSUPPORTED;
  if (d->dtype == ENTMAX_FP32 && d->alibi_slopes) return ENTMAX_EUNSUPPORTED;   // bf16 path only
  return ENTMAX_OK;
}

// The kernels' alpha variant: closed-form powers for 1.5 and 2, the run-time one otherwise.
int alpha_kind(float alpha) { return alpha == 1.5f ? kAlpha15 : (alpha == 2.0f ? kAlpha2 : kAlphaGen); }

bool aligned(const void* p, size_t a) { return p && (reinterpret_cast<uintptr_t>(p) % a) == 0; }

unsigned long long wait_limit_ns(const entmax_attn_desc* d) {
  return d->wait_limit_us == 0 ? kWaitLimitNs : (unsigned long long)d->wait_limit_us * 1000ull;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// [BH][L][64] 16-bit tensor viewed as 3-D; box = one 128 x 64 tile, 128-byte swizzle.
// Rows past L read as zeros.
bool make_map(CUtensorMap* m, const void* base, int L, int BH, bool f16 = false) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)kD, (cuuint64_t)L, (cuuint64_t)BH};
  cuuint64_t strides[2] = {(cuuint64_t)kD * 2, (cuuint64_t)L * kD * 2};
  cuuint32_t box[3] = {(cuuint32_t)kD, (cuuint32_t)kTile, 1}, es[3] = {1, 1, 1};
  return fn(m, f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base),
            dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// fp32 [BH][L][64] as 3-D with a 32 x 128 box (128-byte rows, 128-byte swizzle): the
// target of the backward's dQ reduce-adds.
bool make_map_f32_half(CUtensorMap* m, void* base, int L, int BH) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)kD, (cuuint64_t)L, (cuuint64_t)BH};
  cuuint64_t strides[2] = {(cuuint64_t)kD * 4, (cuuint64_t)L * kD * 4};
  cuuint32_t box[3] = {32, (cuuint32_t)kTile, 1}, es[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, base, dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

extern "C" size_t entmax_attn_workspace_bytes(const entmax_attn_desc* d) {
  if (check_desc(d) != ENTMAX_OK) return 0;
  Layout l;
  layout_of(d, &l);
  return l.total;
}

namespace entmax {
size_t fwd_workspace_bytes(const entmax_attn_desc* d) {
  if (check_desc(d) != ENTMAX_OK) return 0;
  Layout l;
  layout_of(d, &l);
  return l.fwd_total;
}
}  // namespace entmax

extern "C" entmax_status entmax_attn_fwd(const entmax_attn_desc* d, const void* Q, const void* K, const void* V,
                                         float* O, float* tau, void* ws, void* stream) {
  entmax_status st = check_desc(d);
  if (st != ENTMAX_OK) return st;
  if (!aligned(Q, 16) || !aligned(K, 16) || !aligned(V, 16) || !aligned(O, 16) || !aligned(tau, 4) ||
      !aligned(ws, 256))
    return ENTMAX_EINVAL;
  Layout l;
  layout_of(d, &l);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* w = static_cast<uint8_t*>(ws);
  if (cudaMemsetAsync(w + l.off_status, 0, 256, s) != cudaSuccess) return ENTMAX_ECUDA;
  if (cudaMemsetAsync(w + l.off_MT, 0, l.bytes_MT, s) != cudaSuccess) return ENTMAX_ECUDA;
  if (d->mask64 && cudaMemsetAsync(w + l.off_M64T, 0, l.bytes_M64T, s) != cudaSuccess) return ENTMAX_ECUDA;
  if (d->dtype == ENTMAX_FP32) {
    FwdF32Params q;
    std::memset(&q, 0, sizeof(q));
    q.Q = static_cast<const float*>(Q);
    q.K = static_cast<const float*>(K);
    q.V = static_cast<const float*>(V);
    q.O = O;
    q.tau = tau;
    q.M = reinterpret_cast<uint32_t*>(w + l.off_M);
    q.MT = reinterpret_cast<uint32_t*>(w + l.off_MT);
    q.M64 = d->mask64 ? reinterpret_cast<uint32_t*>(w + l.off_M64) : nullptr;
    q.M64T = d->mask64 ? reinterpret_cast<uint32_t*>(w + l.off_M64T) : nullptr;
    q.W64c = l.W64c;
    q.W64r = l.W64r;
    q.stats = reinterpret_cast<int*>(w + l.off_stats);
    q.status = reinterpret_cast<int*>(w + l.off_status);
    q.kv_len = d->kv_len;
    q.H = d->H;
    q.L = d->L;
    q.Tr = l.Tr;
    q.Tc = l.Tc;
    q.Wc = l.Wc;
    q.Wr = l.Wr;
    q.BH = l.BH;
    q.cz = (d->alpha - 1.0f) * d->scale;
    q.causal = d->causal || d->window >= 0;
    q.window = d->window < 0 ? -1 : d->window;
    q.max_sweeps = d->max_sweeps == 0 ? kDefaultSweeps : d->max_sweeps;
    return launch_fwd_f32(d->alpha == 1.5f, q, l.BH * l.Tr, s) == cudaSuccess ? ENTMAX_OK : ENTMAX_ECUDA;
  }
  FwdParams p;
  std::memset(&p, 0, sizeof(p));
  void* v16 = w + l.off_v16;
  if (!make_map(&p.tQ, Q, d->L, l.BH) || !make_map(&p.tK, K, d->L, l.BH) || !make_map(&p.tV, v16, d->L, l.BH, true))
    return ENTMAX_ECUDA;
  if (launch_bf16_to_f16(V, v16, (long)l.BH * d->L * kD, reinterpret_cast<int*>(w + l.off_status), s) != cudaSuccess)
    return ENTMAX_ECUDA;
  p.O = O;
  p.tau = tau;
  p.sumg = reinterpret_cast<float*>(w + l.off_sumg);
  p.Ot = reinterpret_cast<float*>(w + l.off_Ot);
  p.Vb = static_cast<const uint16_t*>(V);
  p.M = reinterpret_cast<uint32_t*>(w + l.off_M);
  p.MT = reinterpret_cast<uint32_t*>(w + l.off_MT);
  p.M64 = d->mask64 ? reinterpret_cast<uint32_t*>(w + l.off_M64) : nullptr;   // the 64 x 64 variant
  p.M64T = d->mask64 ? reinterpret_cast<uint32_t*>(w + l.off_M64T) : nullptr;
  p.W64c = l.W64c;
  p.W64r = l.W64r;
  p.stats = reinterpret_cast<int*>(w + l.off_stats);
  p.status = reinterpret_cast<int*>(w + l.off_status);
  p.kv_len = d->kv_len;
  p.H = d->H;
  p.L = d->L;
  p.Tr = l.Tr;
  p.Tc = l.Tc;
  p.Wc = l.Wc;
  p.Wr = l.Wr;
  p.BH = l.BH;
  p.cz = (d->alpha - 1.0f) * d->scale;
  p.causal = d->causal || d->window >= 0;
  p.window = d->window < 0 ? -1 : d->window;
  p.max_sweeps = d->max_sweeps == 0 ? kDefaultSweeps : d->max_sweeps;
  p.ae = 1.0f / (d->alpha - 1.0f);
  p.am1 = d->alpha - 1.0f;
  p.alibi = d->alibi_slopes;
  p.inv_scale = 1.0f / d->scale;
  p.wait_limit_ns = wait_limit_ns(d);
  p.selftest = d->selftest;
  return launch_fwd(alpha_kind(d->alpha), p, l.BH * l.Tr, s) == cudaSuccess ? ENTMAX_OK : ENTMAX_ECUDA;
}

extern "C" entmax_status entmax_attn_bwd(const entmax_attn_desc* d, const void* Q, const void* K, const void* V,
                                         const void* dO, const float* tau, void* ws, float* dQ, float* dK,
                                         float* dV, void* stream) {
  entmax_status st = check_desc(d);
  if (st != ENTMAX_OK) return st;
  if (d->dtype != ENTMAX_BF16) return ENTMAX_EUNSUPPORTED;   // the fp32 path is forward-only
  if (!aligned(Q, 16) || !aligned(K, 16) || !aligned(V, 16) || !aligned(dO, 16) || !aligned(tau, 4) ||
      !aligned(ws, 256) || !aligned(dQ, 16) || !aligned(dK, 16) || !aligned(dV, 16))
    return ENTMAX_EINVAL;
  Layout l;
  layout_of(d, &l);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* w = static_cast<uint8_t*>(ws);
  BwdParams p;
  std::memset(&p, 0, sizeof(p));
  // V's fp16 copy was made by the forward (same workspace); dO gets one here.
  void* do16 = w + l.off_do16;
  if (!make_map(&p.tQ, Q, d->L, l.BH) || !make_map(&p.tK, K, d->L, l.BH) ||
      !make_map(&p.tV, w + l.off_v16, d->L, l.BH, true) || !make_map(&p.tdO, do16, d->L, l.BH, true) ||
      !make_map_f32_half(&p.tdQ, dQ, d->L, l.BH))
    return ENTMAX_ECUDA;
  float* delta = reinterpret_cast<float*>(w + l.off_delta);
  p.tau = tau;
  p.delta = delta;
  p.MT = reinterpret_cast<const uint32_t*>(w + l.off_MT);
  p.M64T = d->mask64 ? reinterpret_cast<const uint32_t*>(w + l.off_M64T) : nullptr;
  p.W64r = l.W64r;
  p.dQ = dQ;
  p.dK = dK;
  p.dV = dV;
  p.status = reinterpret_cast<int*>(w + l.off_status);
  p.stats = reinterpret_cast<int*>(w + l.off_bstats);
  p.kv_len = d->kv_len;
  p.H = d->H;
  p.L = d->L;
  p.Tr = l.Tr;
  p.Tc = l.Tc;
  p.Wr = l.Wr;
  p.BH = l.BH;
  p.cz = (d->alpha - 1.0f) * d->scale;
  p.scale = d->scale;
  p.ae = 1.0f / (d->alpha - 1.0f);
  p.alibi = d->alibi_slopes;
  p.causal = d->causal || d->window >= 0;
  p.window = d->window < 0 ? -1 : d->window;
  p.wait_limit_ns = wait_limit_ns(d);
  p.selftest = d->selftest;
  const long rows = (long)l.BH * d->L;
  DeltaParams dp;
  std::memset(&dp, 0, sizeof(dp));
  dp.Q = static_cast<const uint16_t*>(Q);
  dp.K = static_cast<const uint16_t*>(K);
  dp.V = static_cast<const uint16_t*>(V);
  dp.dO = static_cast<const uint16_t*>(dO);
  dp.tau = tau;
  dp.V16 = reinterpret_cast<const uint16_t*>(w + l.off_v16);
  dp.Ot = reinterpret_cast<const float*>(w + l.off_Ot);
  dp.sumg = reinterpret_cast<const float*>(w + l.off_sumg);
  dp.M = reinterpret_cast<const uint32_t*>(w + l.off_M);
  dp.delta = delta;
  dp.kv_len = d->kv_len;
  dp.H = d->H;
  dp.L = d->L;
  dp.Tr = l.Tr;
  dp.Wc = l.Wc;
  dp.BH = l.BH;
  dp.cz = (d->alpha - 1.0f) * d->scale;
  dp.ae = 1.0f / (d->alpha - 1.0f);
  dp.alibi = d->alibi_slopes;
  dp.scale = d->scale;
  dp.causal = d->causal || d->window >= 0;
  dp.window = d->window < 0 ? -1 : d->window;
  if (launch_delta(alpha_kind(d->alpha), dp, s) != cudaSuccess) return ENTMAX_ECUDA;
  if (cudaMemsetAsync(dQ, 0, (size_t)rows * kD * 4, s) != cudaSuccess) return ENTMAX_ECUDA;
  if (launch_bf16_to_f16(dO, do16, rows * kD, reinterpret_cast<int*>(w + l.off_status), s) != cudaSuccess)
    return ENTMAX_ECUDA;
  return launch_bwd(alpha_kind(d->alpha), p, l.BH * l.Tc, s) == cudaSuccess ? ENTMAX_OK : ENTMAX_ECUDA;
}

extern "C" entmax_status entmax_rows(const float* S, int rows, int n, int ld, float alpha, float* P, float* tau,
                                     int* status, void* stream) {
  if (rows < 0 || n < 1 || ld < n || (ld % 4) != 0) return ENTMAX_EINVAL;
  if (alpha != 1.5f && alpha != 2.0f) return ENTMAX_EUNSUPPORTED;
  if (rows == 0) return ENTMAX_OK;
  if (!aligned(S, 16) || !aligned(P, 16) || !aligned(tau, 4)) return ENTMAX_EINVAL;
  if (status && !aligned(status, 4)) return ENTMAX_EINVAL;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return launch_rows(alpha == 1.5f, S, rows, n, ld, P, tau, status, s) == cudaSuccess ? ENTMAX_OK : ENTMAX_ECUDA;
}

extern "C" entmax_status entmax_last_device_status(const entmax_attn_desc* d, const void* ws, int* status_out,
                                                   void* stream) {
  if (check_desc(d) != ENTMAX_OK || !status_out) return ENTMAX_EINVAL;
  if (!ws) {
    ws = noalloc_scratch();   // the no-allocation forward's scratch on the current device
    if (!ws) return ENTMAX_ECUDA;
  }
  if (!aligned(ws, 256)) return ENTMAX_EINVAL;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return ENTMAX_ECUDA;
  int word = 0;
  if (cudaMemcpy(&word, ws, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return ENTMAX_ECUDA;
  *status_out = word;
  if (word & kStatusTimeout) return ENTMAX_ETIMEOUT;
  if (word & kStatusRange) return ENTMAX_ERANGE;
  if (word & kStatusNoConverge) return ENTMAX_ENOCONVERGE;
  return ENTMAX_OK;
}

extern "C" entmax_status entmax_attn_block_mask64(const entmax_attn_desc* d, const void* ws, uint32_t* M64,
                                                  void* stream) {
  if (check_desc(d) != ENTMAX_OK || !aligned(ws, 256) || !M64 || !d->mask64) return ENTMAX_EINVAL;
  Layout l;
  layout_of(d, &l);
  const uint8_t* w = static_cast<const uint8_t*>(ws);
  if (cudaMemcpyAsync(M64, w + l.off_M64, l.bytes_M64, cudaMemcpyDeviceToDevice, static_cast<cudaStream_t>(stream)) !=
      cudaSuccess)
    return ENTMAX_ECUDA;
  return ENTMAX_OK;
}

extern "C" entmax_status entmax_attn_block_mask(const entmax_attn_desc* d, const void* ws, uint32_t* M,
                                                int* stats, int* bwd_stats, void* stream) {
  if (check_desc(d) != ENTMAX_OK || !aligned(ws, 256)) return ENTMAX_EINVAL;
  Layout l;
  layout_of(d, &l);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const uint8_t* w = static_cast<const uint8_t*>(ws);
  if (M && cudaMemcpyAsync(M, w + l.off_M, l.bytes_M, cudaMemcpyDeviceToDevice, s) != cudaSuccess)
    return ENTMAX_ECUDA;
  if (stats && cudaMemcpyAsync(stats, w + l.off_stats, l.bytes_stats, cudaMemcpyDeviceToDevice, s) != cudaSuccess)
    return ENTMAX_ECUDA;
  if (bwd_stats &&
      cudaMemcpyAsync(bwd_stats, w + l.off_bstats, l.bytes_bstats, cudaMemcpyDeviceToDevice, s) != cudaSuccess)
    return ENTMAX_ECUDA;
  return ENTMAX_OK;
}
