// fwd_f32.cu -- alpha-entmax attention forward for fp32 Q, K, V (CUDA cores, fp32 FMA).
//
// Same method and phases as the bf16 kernel ("AdaSplash-2: Faster Differentiable
// Sparse Attention", §3.3), for inputs that must keep fp32 precision in the scores:
//   1. a max pass over the active key tiles, with per-(row, key tile) maxima;
//   2. tau on those maxima, a lower bound of tau* (§2.4 bracket);
//   3. a pass that copies every score above that bound (the only support
//      candidates) to shared memory, then an exact on-chip solve (safeguarded Newton
//      ending with the exact root of the current support's piece). If the copies
//      overflow, the row takes bracketed Newton passes instead;
//   4. the block mask from the tile maxima at the final tau (Appendix C.4 packing);
//   5. an output pass over the flagged tiles: O = sum_j A_ij V_j, in fp32.
// One CTA per (batch*head, 128-row query tile); thread r owns query row r; K and V
// tiles are staged in shared memory and read as broadcasts. This path is forward-only
// (the workspace's sum g and Ot are not written), and meant for small fp32 problems.
#include "common.cuh"
#include "kernels.h"

namespace entmax {

namespace {

constexpr int kThreads32 = 128;
constexpr int kCand32 = 64;

__device__ __forceinline__ void acc32(float u, float& S1, float& S2, float& C, float& umin) {
  if (u > 0.f) {
    S1 += u;
    S2 = fmaf(u, u, S2);
    C += 1.f;
    umin = fminf(umin, u);
  }
}

// Exact threshold of one row over `n` scores vals[k*stride] that contain its support.
template <int AK>
__device__ bool solve32(const float* vals, int n, int stride, float cz, float t, float lo, float hi, float& out) {
  for (int it = 0; it < 64; ++it) {
    float S1 = 0.f, S2 = 0.f, C = 0.f, umin = INFINITY;
    for (int k = 0; k < n; ++k) acc32(fmaf(vals[k * stride], cz, -t), S1, S2, C, umin);
    const float f = (AK == kAlpha15) ? S2 - 1.f : S1 - 1.f;
    const float fp = (AK == kAlpha15) ? 2.f * S1 : C;
    if (C > 0.f) {
      float d = -1.f;
      if (AK == kAlpha15) {
        const float disc = S1 * S1 - C * (S2 - 1.f);
        if (disc >= 0.f) d = (S2 - 1.f) / (S1 + sqrtf(disc));
      } else {
        d = (S1 - 1.f) / C;
      }
      if (d >= 0.f && d < umin) {
        out = t + d;
        return true;
      }
    }
    if (fabsf(f) <= 1e-7f && fp > 0.f) {
      out = t + f / fp;
      return true;
    }
    if (f > 0.f) lo = t; else hi = t;
    float tn = t + f / fp;
    if (!(tn > lo && tn <= hi && tn != t)) tn = 0.5f * (lo + hi);   // the root may sit at hi (uniform scores); a stalled step bisects
    t = tn;
  }
  out = t;
  return false;
}

// Cooperative copy of one [128][64] fp32 tile (rows past L read as zeros).
__device__ __forceinline__ void stage_tile(float* dst, const float* src, int row0, int L) {
  const int r = threadIdx.x;
  float4* d = reinterpret_cast<float4*>(dst + r * kD);
  if (row0 + r < L) {
    const float4* s = reinterpret_cast<const float4*>(src + (size_t)(row0 + r) * kD);
#pragma unroll
    for (int c = 0; c < kD / 4; ++c) d[c] = s[c];
  } else {
#pragma unroll
    for (int c = 0; c < kD / 4; ++c) d[c] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
}

__device__ __forceinline__ float dot64(const float (&q)[kD], const float* k) {
  const float4* k4 = reinterpret_cast<const float4*>(k);
  float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
  for (int c = 0; c < kD / 4; ++c) {
    const float4 v = k4[c];
    a0 = fmaf(q[4 * c], v.x, a0);
    a1 = fmaf(q[4 * c + 1], v.y, a1);
    a2 = fmaf(q[4 * c + 2], v.z, a2);
    a3 = fmaf(q[4 * c + 3], v.w, a3);
  }
  return (a0 + a1) + (a2 + a3);
}

}  // namespace

template <int AK>
__global__ void __launch_bounds__(kThreads32) fwd_f32_kernel(const FwdF32Params p) {
  extern __shared__ __align__(16) float sm[];
  float* sK = sm;                          // [128][64]
  float* sV = sK + kTile * kD;             // [128][64]
  float* tmax = sV + kTile * kD;           // [Tc][128]
  float* cand = tmax + p.Tc * kTile;       // [64][128]
  __shared__ uint32_t act[kMaskWords], flag[kMaskWords];
  __shared__ uint32_t m64[2][2 * kMaskWords];   // the mask at 64 x 64 blocks: [row half][key block bits]
  __shared__ int any_need;

  const int r = threadIdx.x;
  const int bh = blockIdx.x % p.BH;
  const int qt = p.Tr - 1 - blockIdx.x / p.BH;
  const int b = bh / p.H;
  const Pattern pat{p.L, p.kv_len ? min(max(p.kv_len[b], 1), p.L) : p.L, p.causal, p.window};
  const int i0 = qt * kTile, i1 = min(p.L, i0 + kTile);
  const int i = i0 + r;
  const bool valid = i < p.L;
  const size_t head = (size_t)bh * p.L * kD;
  const float cz = p.cz;

  if (r < kMaskWords) act[r] = flag[r] = 0;
  if (r < 4 * kMaskWords) (&m64[0][0])[r] = 0;
  __syncthreads();
  for (int jt = r; jt < p.Tc; jt += kThreads32)
    if (pat.block_active(i0, i1, jt * kTile, min(p.L, jt * kTile + kTile))) atomicOr(&act[jt >> 5], 1u << (jt & 31));
  __syncthreads();
  uint32_t a[kMaskWords];
#pragma unroll
  for (int w = 0; w < kMaskWords; ++w) a[w] = act[w];

  float q[kD];
#pragma unroll
  for (int c = 0; c < kD; ++c) q[c] = valid ? p.Q[head + (size_t)i * kD + c] : 0.f;

  // 1. Max pass and per-tile maxima.
  float m = -INFINITY;
  for_each_bit(a, kMaskWords, [&](int jt) {
    __syncthreads();
    stage_tile(sK, p.K + head, jt * kTile, p.L);
    __syncthreads();
    float tm = -INFINITY;
    for (int c = 0; c < kTile; ++c)
      if (pat.active(i, jt * kTile + c)) tm = fmaxf(tm, dot64(q, sK + c * kD));
    tmax[jt * kTile + r] = tm;
    m = fmaxf(m, tm);
  });

  // 2. Bracket and the tile-maxima lower bound.
  const int n_act = valid ? pat.count(i) : 1;
  float lo = m * cz - 1.f;
  float hi = m * cz - ((AK == kAlpha15) ? rsqrtf((float)n_act) : 1.f / (float)n_act);
  float tau = INFINITY;
  bool done = !valid;
  if (valid) {
    int nl = 0;
    for_each_bit(a, kMaskWords, [&](int jt) {
      const float v = tmax[jt * kTile + r];
      if (nl < kCand32 && fmaf(v, cz, -lo) > 0.f) cand[nl++ * kTile + r] = v;
    });
    float t = lo;
    solve32<AK>(cand + r, nl, kTile, cz, lo, lo, hi, t);
    tau = fminf(fmaxf(t, lo), hi);
  }

  // 3. Candidate pass (then bracketed Newton passes for rows whose candidates overflow).
  int sweeps = 0;
  for (;;) {
    if (r == 0) any_need = 0;
    __syncthreads();
    if (!done && sweeps < p.max_sweeps) any_need = 1;
    __syncthreads();
    if (!any_need) break;
    const bool collect = (sweeps == 0);
    float S1 = 0.f, S2 = 0.f, C = 0.f, umin = INFINITY;
    int nc = 0;
    for_each_bit(a, kMaskWords, [&](int jt) {
      __syncthreads();
      stage_tile(sK, p.K + head, jt * kTile, p.L);
      __syncthreads();
      if (done) return;
      for (int c = 0; c < kTile; ++c) {
        if (!pat.active(i, jt * kTile + c)) continue;
        const float s = dot64(q, sK + c * kD);
        const float u = fmaf(s, cz, -tau);
        acc32(u, S1, S2, C, umin);
        if (collect && u > 0.f) {
          if (nc < kCand32) cand[nc * kTile + r] = s;
          ++nc;
        }
      }
    });
    ++sweeps;
    if (!done) {
      const float f = (AK == kAlpha15) ? S2 - 1.f : S1 - 1.f;
      const float fp = (AK == kAlpha15) ? 2.f * S1 : C;
      if (f > 0.f) lo = fmaxf(lo, tau); else hi = fminf(hi, tau);
      float t;
      if (collect && nc <= kCand32 && solve32<AK>(cand + r, nc, kTile, cz, tau, lo, hi, t)) {
        tau = t;
        done = true;
      } else if (fabsf(f) <= 3e-5f && fp > 0.f) {
        tau += f / fp;
        done = true;
      } else {
        float tn = tau + f / fp;
        if (!(tn > lo && tn <= hi && tn != tau)) tn = 0.5f * (lo + hi);   // the root may sit at hi (uniform scores); a stalled step bisects
        tau = tn;
      }
    }
  }
  if (valid && !done) atomicOr(p.status, kStatusNoConverge);

  // 4. Block mask from the tile maxima at the final tau.
  for_each_bit(a, kMaskWords, [&](int jt) {
    if (valid && fmaf(tmax[jt * kTile + r], cz, -tau) > 0.f) atomicOr(&flag[jt >> 5], 1u << (jt & 31));
  });
  __syncthreads();
  uint32_t f[kMaskWords];
#pragma unroll
  for (int w = 0; w < kMaskWords; ++w) f[w] = flag[w];
  if (r < p.Wc) p.M[((size_t)bh * p.Tr + qt) * p.Wc + r] = f[r];
  if (r == 0)
    for_each_bit(f, kMaskWords, [&](int jt) {
      atomicOr(&p.MT[((size_t)bh * p.Tc + jt) * p.Wr + (qt >> 5)], 1u << (qt & 31));
    });

  // 5. Output over the flagged tiles.
  float o[kD];
#pragma unroll
  for (int c = 0; c < kD; ++c) o[c] = 0.f;
  int n_out = 0;
  for_each_bit(f, kMaskWords, [&](int jt) {
    __syncthreads();
    stage_tile(sK, p.K + head, jt * kTile, p.L);
    stage_tile(sV, p.V + head, jt * kTile, p.L);
    __syncthreads();
    ++n_out;
    bool nz[2] = {false, false};   // a nonzero weight in key half 0 / 1 of the tile
    for (int c = 0; c < kTile; ++c) {
      if (!pat.active(i, jt * kTile + c)) continue;
      const float u = fmaf(dot64(q, sK + c * kD), cz, -tau);
      if (!(u > 0.f)) continue;
      nz[c >> 6] = true;
      const float w = (AK == kAlpha15) ? u * u : u;
      const float4* v4 = reinterpret_cast<const float4*>(sV + c * kD);
#pragma unroll
      for (int cc = 0; cc < kD / 4; ++cc) {
        const float4 v = v4[cc];
        o[4 * cc] = fmaf(w, v.x, o[4 * cc]);
        o[4 * cc + 1] = fmaf(w, v.y, o[4 * cc + 1]);
        o[4 * cc + 2] = fmaf(w, v.z, o[4 * cc + 2]);
        o[4 * cc + 3] = fmaf(w, v.w, o[4 * cc + 3]);
      }
    }
#pragma unroll
    for (int h = 0; h < 2; ++h)
      if (nz[h]) atomicOr(&m64[r >> 6][(2 * jt + h) >> 5], 1u << ((2 * jt + h) & 31));
  });
  __syncthreads();
  if (p.M64 && r < 2 * p.W64c) {   // rows 2 qt and 2 qt + 1 of the 64 x 64 mask, and its transpose
    const int h = r / p.W64c, w = r % p.W64c;
    const uint32_t bits = m64[h][w];
    const int qb = 2 * qt + h;
    p.M64[((size_t)bh * 2 * p.Tr + qb) * p.W64c + w] = bits;
    for (uint32_t b = bits; b; b &= b - 1) {
      const int kb = w * 32 + __ffs(b) - 1;
      atomicOr(&p.M64T[((size_t)bh * 2 * p.Tc + kb) * p.W64r + (qb >> 5)], 1u << (qb & 31));
    }
  }
  if (valid) {
    float4* dst = reinterpret_cast<float4*>(p.O + head + (size_t)i * kD);
#pragma unroll
    for (int cc = 0; cc < kD / 4; ++cc) dst[cc] = make_float4(o[4 * cc], o[4 * cc + 1], o[4 * cc + 2], o[4 * cc + 3]);
    p.tau[(size_t)bh * p.L + i] = tau;
  }
  if (r == 0) {
    int na = 0, nflag = 0;
    for (int w = 0; w < kMaskWords; ++w) {
      na += __popc(a[w]);
      nflag += __popc(f[w]);
    }
    int4* st = reinterpret_cast<int4*>(p.stats + ((size_t)bh * p.Tr + qt) * kFwdStats);
    st[0] = make_int4(sweeps, 0, nflag, na);
    st[1] = make_int4(0, 0, 0, 0);   // no phase timing on this path
  }
}

int fwd_f32_smem_bytes(int Tc) { return (2 * kTile * kD + Tc * kTile + kCand32 * kTile) * 4; }

cudaError_t launch_fwd_f32(bool alpha15, const FwdF32Params& p, int grid, cudaStream_t s) {
  const int smem = fwd_f32_smem_bytes(p.Tc);
  auto kern = alpha15 ? fwd_f32_kernel<kAlpha15> : fwd_f32_kernel<kAlpha2>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  kern<<<grid, kThreads32, smem, s>>>(p);
  return cudaGetLastError();
}

}  // namespace entmax
