// rows.cu -- row-wise alpha-entmax of explicit fp32 score rows (no matrix product, so
// no tensor cores: one CTA per row, block reductions).
//
// "AdaSplash-2: Faster Differentiable Sparse Attention":
//   - §2.3 Eq. 3 gives p = [(alpha-1) s - tau]_+^{1/(alpha-1)}.
//   - §2.4 Eq. 4 gives f(tau), with the bracket [m - 1, m - n^{1-alpha}].
//   - §3.2 describes the safeguarded hybrid solver.
// Each iteration reduces count C, S1 = sum u, S2 = sum u^2 and the smallest positive
// u over the row, where u = [z - tau]_+ and z = (alpha-1) s. Two steps are then
// possible:
//   - the exact root of Eq. 4 restricted to the current support. For alpha = 1.5 it is
//     the smaller root of C d^2 - 2 S1 d + S2 - 1 = 0; for alpha = 2 it is
//     d = (S1 - 1)/C. When the root stays below the smallest positive u, no element
//     leaves the support, so it is tau* and the solve ends.
//   - otherwise a Newton step on Eq. 4, clamped to the bracket, with bisection as the
//     fallback.
// Rows of up to kRowsSmem scores are staged once in shared memory, so the iterations
// read them there; longer rows are re-read from global memory (L2) on each iteration.
// A row that reaches the iteration cap keeps tau inside the bracket and sets bit 0 of the
// optional status word.
#include "common.cuh"
#include "kernels.h"

namespace entmax {

namespace {
constexpr int kRowThreads = 256;
constexpr int kRowsSmem = 16384;   // longest row staged in shared memory (64 KB)
constexpr int kRowIters = 100;

struct Red {
  float s1, s2, c, umin;
};

__device__ __forceinline__ Red red_combine(Red a, Red b) {
  return {a.s1 + b.s1, a.s2 + b.s2, a.c + b.c, fminf(a.umin, b.umin)};
}

__device__ Red block_reduce(Red v, Red* buf) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    Red w{__shfl_xor_sync(0xffffffffu, v.s1, o), __shfl_xor_sync(0xffffffffu, v.s2, o),
          __shfl_xor_sync(0xffffffffu, v.c, o), __shfl_xor_sync(0xffffffffu, v.umin, o)};
    v = red_combine(v, w);
  }
  __syncthreads();   // buf reuse across calls
  if (lane == 0) buf[warp] = v;
  __syncthreads();
  Red r = buf[0];
  for (int w = 1; w < kRowThreads / 32; ++w) r = red_combine(r, buf[w]);
  return r;
}
}  // namespace

template <int AK>
__global__ void __launch_bounds__(kRowThreads) rows_kernel(const float* __restrict__ S, int n, long ld,
                                                            float* __restrict__ P, float* __restrict__ tau_out,
                                                            int* status) {
  __shared__ Red buf[kRowThreads / 32];
  extern __shared__ float srow[];
  const float* x = S + (long)blockIdx.x * ld;
  if (n <= kRowsSmem) {
    for (int j = threadIdx.x; j < n; j += kRowThreads) srow[j] = x[j];
    __syncthreads();
    x = srow;
  }
  const float c = (AK == kAlpha15) ? 0.5f : 1.0f;   // alpha - 1

  // Row max (-inf entries are inactive) and active count.
  Red acc{-INFINITY, 0.f, 0.f, INFINITY};
  for (int j = threadIdx.x; j < n; j += kRowThreads) {
    const float v = x[j];
    if (v != -INFINITY) {
      acc.s1 = fmaxf(acc.s1, v);
      acc.c += 1.f;
    }
  }
  {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int o = 16; o > 0; o >>= 1) {
      acc.s1 = fmaxf(acc.s1, __shfl_xor_sync(0xffffffffu, acc.s1, o));
      acc.c += __shfl_xor_sync(0xffffffffu, acc.c, o);
    }
    if (lane == 0) buf[warp] = acc;
    __syncthreads();
    Red r = buf[0];
    for (int w = 1; w < kRowThreads / 32; ++w) {
      r.s1 = fmaxf(r.s1, buf[w].s1);
      r.c += buf[w].c;
    }
    acc = r;
  }
  const float mz = c * acc.s1;
  const float n_act = fmaxf(acc.c, 1.f);
  float lo = mz - 1.f;
  float hi = mz - ((AK == kAlpha15) ? rsqrtf(n_act) : 1.f / n_act);
  float t = lo;
  bool settled = false;
  for (int it = 0; it < kRowIters; ++it) {
    Red v{0.f, 0.f, 0.f, INFINITY};
    for (int j = threadIdx.x; j < n; j += kRowThreads) {
      const float u = fmaf(x[j], c, -t);
      if (u > 0.f) {
        v.s1 += u;
        v.s2 = fmaf(u, u, v.s2);
        v.c += 1.f;
        v.umin = fminf(v.umin, u);
      }
    }
    const Red r = block_reduce(v, buf);
    const float f = (AK == kAlpha15) ? r.s2 - 1.f : r.s1 - 1.f;
    const float fp = (AK == kAlpha15) ? 2.f * r.s1 : r.c;   // |f'(t)|
    if (r.c > 0.f) {
      float d = -1.f;
      if (AK == kAlpha15) {
        const float disc = r.s1 * r.s1 - r.c * (r.s2 - 1.f);
        if (disc >= 0.f) d = (r.s2 - 1.f) / (r.s1 + sqrtf(disc));   // = (S1 - sqrt(disc)) / C
      } else {
        d = (r.s1 - 1.f) / r.c;
      }
      if (d >= 0.f && d < r.umin) {   // support unchanged at t + d: exact root
        t += d;
        settled = true;
        break;
      }
    }
    if (fabsf(f) <= 1e-7f && fp > 0.f) {
      t += f / fp;
      settled = true;
      break;
    }
    if (f > 0.f) lo = t; else hi = t;
    float tn = t + f / fp;
    if (!(tn > lo && tn <= hi && tn != t)) tn = 0.5f * (lo + hi);   // the root may sit at hi (uniform scores); a stalled step bisects
    t = tn;
  }
  if (threadIdx.x == 0) {
    tau_out[blockIdx.x] = t;
    if (!settled && status) atomicOr(status, kStatusNoConverge);
  }
  float* out = P + (long)blockIdx.x * ld;
  for (int j = threadIdx.x; j < n; j += kRowThreads) {
    const float u = fmaxf(fmaf(x[j], c, -t), 0.f);
    out[j] = (AK == kAlpha15) ? u * u : u;
  }
}

cudaError_t launch_rows(bool alpha15, const float* S, int rows, int n, long ld, float* P, float* tau, int* status,
                        cudaStream_t s) {
  const int smem = n <= kRowsSmem ? n * 4 : 0;
  auto kern = alpha15 ? rows_kernel<kAlpha15> : rows_kernel<kAlpha2>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kRowsSmem * 4);
  if (e != cudaSuccess) return e;
  kern<<<rows, kRowThreads, smem, s>>>(S, n, ld, P, tau, status);
  return cudaGetLastError();
}

}  // namespace entmax
