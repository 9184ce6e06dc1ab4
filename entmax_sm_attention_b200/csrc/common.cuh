// common.cuh -- shared definitions of the fused alpha-entmax attention kernels.
#pragma once
#include <cuda.h>
#include <cstdint>
#include "sm100.cuh"

namespace entmax {

constexpr int kTile = 128;      // query / key tile edge (also the block-mask granularity)
constexpr int kD = 64;          // head dimension (one 128-byte bf16 row)
constexpr int kTileBytes = kTile * kD * 2;   // one bf16 [128][64] tile = 16 KB
constexpr int kMaxTc = 128;     // longest sequence = 128 key tiles = 16384 tokens
constexpr int kMaskWords = kMaxTc / 32;

// Alpha variants: A = u^{1/(alpha-1)}, g = u^{(2-alpha)/(alpha-1)} for u = z - tau > 0.
//   kAlpha15: A = u^2, g = u          kAlpha2: A = u, g = [u > 0]
//   kAlphaGen: any alpha > 1 at run time, with e = 1/(alpha-1): A = u^e, g = u^{e-1},
//     through exp2(e log2 u) (the hardware's approximate base-2 exponential and
//     logarithm: relative error near 2^-22 each).
enum AlphaKind { kAlpha15 = 0, kAlpha2 = 1, kAlphaGen = 2 };

// ALiBi ("AdaSplash-2" §4.3, NAPE heads; Press et al.): the score of key j for query i
// is lowered by m_h |i - j|. The kernels work on raw scores s = q . k (z = cz s), so they
// subtract cb |i - j| with cb = m_h / scale from the raw scores of keys j0 + c.
template <int N>
__device__ __forceinline__ void alibi_apply(float (&s)[N], float cb, int i, int j0) {
  const float base = (float)(i - j0);
#pragma unroll
  for (int c = 0; c < N; ++c) s[c] = fmaf(-cb, fabsf(base - (float)c), s[c]);
}

// u^x for u > 0 (exp2 of x log2 u); callers pass only positive u.
__device__ __forceinline__ float pow_pos(float u, float x) { return exp2f(x * __log2f(u)); }

// Structural attention pattern of one (batch, head).
struct Pattern {
  int L, kv, causal, window;
  // Active key set of query row i (model card "Causal Splash Masking with Sink
  // Preservation"; key padding keeps j < kv).
  __device__ __forceinline__ bool active(int i, int j) const {
    if (j >= kv) return false;
    if (window >= 0) return j <= i && (j == 0 || i - j <= window);
    if (causal) return j <= i;
    return true;
  }
  // Number of active keys of row i (n in the §2.4 bracket).
  __device__ __forceinline__ int count(int i) const {
    if (window >= 0) {
      int hi = min(i, kv - 1), lo = max(1, i - window);
      return 1 + max(0, hi - lo + 1);
    }
    if (causal) return min(i + 1, kv);
    return kv;
  }
  // Does the rows [i0, i1) x keys [j0, j1) block hold any active pair?
  __device__ __forceinline__ bool block_active(int i0, int i1, int j0, int j1) const {
    if (j0 >= kv) return false;
    if (window >= 0) {
      if (j0 == 0) return true;
      int jl = j0, jh = min(j1, kv) - 1;
      return jl <= i1 - 1 && jh >= i0 - window;
    }
    if (causal) return j0 <= i1 - 1;
    return true;
  }
  // Is every pair of the block active (no per-element masking needed)?
  __device__ __forceinline__ bool block_full(int i0, int i1, int j0, int j1) const {
    if (j1 > kv) return false;
    if (window >= 0) return false;
    if (causal) return j1 - 1 <= i0;
    return true;
  }
};

// Iterate the set bits of a packed tile mask in increasing order (AdaSplash-2 Appendix
// C.4 traversal with popc / find-next-set; here __ffs on each 32-bit word).
template <class F>
__device__ __forceinline__ void for_each_bit(const uint32_t* words, int nwords, F&& f) {
  for (int w = 0; w < nwords; ++w) {
    uint32_t bits = words[w];
    while (bits) {
      int b = __ffs(bits) - 1;
      bits &= bits - 1;
      f(w * 32 + b);
    }
  }
}

// Vote among the `nthreads` row-owner threads (warps 0..nthreads/32-1, named barrier 2):
// true if any passes `pred`. votes[r] must be zero before decision r; each decision
// uses its own slot.
__device__ __forceinline__ bool rows_any(bool pred, int* votes, int r, int lane, int nthreads) {
  const unsigned bal = __ballot_sync(0xffffffffu, pred);
  if (lane == 0 && bal) atomicAdd(&votes[r], 1);
  named_bar(2, nthreads);
  return *reinterpret_cast<volatile int*>(&votes[r]) > 0;
}

}  // namespace entmax
