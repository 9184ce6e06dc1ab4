// fwd.cu -- fused alpha-entmax attention forward for sm_100a.
//
// One CTA per (batch*head, 128-row query tile) computes the phases of "AdaSplash-2:
// Faster Differentiable Sparse Attention", §3.3:
//   Phase 1 (maximum): stream the structurally active key tiles; S = Q K^T on the
//     tensor cores (tcgen05, accumulator in TMEM). Each row keeps its max in every key
//     tile, in shared memory.
//   Initial threshold: each thread keeps the four largest of its part-tile maxima (the
//     maxima over its 32 columns of each key tile) in registers; the row's tau
//     restricted to those 16 scores (four threads per row) is a lower bound
//     tau_T <= tau* (entmax on a subset of the scores has fewer nonnegative terms in
//     Eq. 4). It plays the role the paper gives its on-chip histogram (Phase 2), without
//     an extra pass over K.
//   Phase 3 and 4 fused (alpha 1.5 and 2): one output pass at tau_T over the key tiles
//     where some row has a score above tau_T. Per tile the row owners copy every score
//     with u_T = z - tau_T > 0 (score and key index) into shared memory (32 per row and
//     column part, 128 per row), and write A_T = u_T^{1/(alpha-1)} in fp16 (2^-11
//     rounding; bf16 would give 2^-8) into TMEM over the S columns they have read; the
//     tensor cores accumulate O_T = sum A_T V with the A operand read from TMEM and B an
//     fp16 copy of V. Since tau_T <= tau*, the copies hold the whole support, so a row
//     whose copies fit is solved exactly on chip (four lanes of one warp per row):
//     safeguarded Newton on Eq. 4 (§3.2), finished by the exact root of the current
//     support's piece (alpha = 2: (S1-1)/C; alpha = 1.5: the smaller root of
//     C d^2 - 2 S1 d + S2 - 1 = 0) once no candidate leaves the support. Every key with
//     u_T > 0 lies in a visited tile, so the epilogue turns O_T into O at the final tau by
//     adding sum_j (A*_j - fp16(A_T,j)) V_j over the copies in fp32 (A* = 0 outside the
//     support): the result is the support sum with A* in fp32.
//   Fallback: a row whose copies overflow sweeps again (S only), accumulating S1 = sum u,
//     S2 = sum u^2 and the count for a Newton step bracketed by §2.4. Eq. 4's f is convex
//     and decreasing in tau, so a Newton step from tau <= tau* stays <= tau*, and the
//     next sweep's copies (fewer, above a higher tau) again qualify. The query tile then
//     takes an output pass at the final tau over its flagged tiles, which recomputes O.
//     The run-time alpha variant always takes a collecting sweep and then this output
//     pass.
//   Block mask: bit (query tile, key tile) = some row has a key-tile max above its
//     final tau. Packed 32 key tiles per uint32 (Appendix C.4), plus the transpose for
//     the backward; with the 64 x 64 variant also the mask at 64 x 64 blocks.
//   Epilogue: the backward's delta = sum_j g_ij dO_i . V_j / sum_j g_ij needs sum g V and
//     sum g over each row's support; a row solved on its copies has its support listed,
//     and the epilogue sums over it in fp32, gathering the bf16 V rows.
//
// Roles (640 threads): warps 0-15 are row owners. Warp w reads TMEM lanes 32(w%4)..+31
// (one query row per lane) and columns [32(w/4), 32(w/4)+32) of every S tile, so four
// threads share a row and combine partial sums in shared memory; four warps per SM
// sub-partition hide the latency of the per-score work. Warp 16 issues TMA loads into a
// 4-slot ring of 16 KB K/V tiles. Warps 17 and 18 issue the S = Q K^T MMAs of the max pass
// and the sweeps, alternating tiles (one thread blocks while its MMAs enter the tensor
// pipe, so two issuers keep the pipe fed while each probes barriers and commits); warp 17
// owns TMEM and issues the S tiles of the output-type passes (fused or final), and warp
// 19 the O = A V chain.
// TMEM (512 columns): during the max pass and the sweeps, four S buffers at
// 0/128/256/384, so the issuers run up to three tiles ahead. During an output-type pass
// (OutLayout):
//   - three S buffers at 0, 128 and 384, tile k in buffer k % 3. The row owner of keys
//     [32q, 32q+32) writes their A (fp16 pairs) into columns [32q, 32q+16): only over S
//     columns it has read itself;
//   - O at [256,320).
#include <type_traits>

#include "common.cuh"
#include "kernels.h"

namespace entmax {

namespace {

constexpr int kMathWarps = 16;                // row owners: kParts per TMEM lane quadrant
constexpr int kParts = kMathWarps / 4;        // threads per query row
constexpr int kCols = kTile / kParts;         // key columns per thread
constexpr int kOCols = kD / kParts;           // output columns per thread in the epilogue
constexpr int kThreads = (kMathWarps + 4) * 32;
constexpr int kMathThreads = kMathWarps * 32;
constexpr int kProducerWarp = kMathWarps;
constexpr int kMmaWarp = kMathWarps + 1;      // S issuer 0 (even tiles of the max pass and sweeps; the output pass)
constexpr int kSWarp2 = kMathWarps + 2;       // S issuer 1 (odd tiles of the max pass and sweeps)
constexpr int kOWarp = kMathWarps + 3;        // the O = A V chain of the output pass
constexpr int kOBufsMax = 3;    // S/A buffers in the output pass (at most; see OutLayout)
constexpr int kSlots = 4;
constexpr int kSBufs = 4;
constexpr int kCandPerThread = kTile / kParts;   // candidates per (row, column part) for L <= 8192
constexpr int kCandLong = 24;                     // the same above 64 key tiles (shared memory)
constexpr float kTolF = 3e-5f;         // |f(tau)| = |sum p - 1| small enough to stop sweeping
constexpr int kMaxVotes = 72;

// Diagnostic builds (-DENTMAX_DIAG, never the shipped library) also record, per query tile,
// the cycles each role spends waiting: [8] row owner 0 on S in the max pass, [9] on S in
// the sweeps, [10] on S in the output pass, [11] the first sweep loop in total, [12] the S
// issuer on its barriers in the max pass and sweeps, [13] in the output pass, [14] the O
// issuer on its barriers, [15] the TMA producer on free ring slots; then row owner 0's
// steps per phase ([16..18] max pass: TMEM load, release, compute; [19..21] sweeps;
// [22..24] output: TMEM load, compute, store + release) and the issuers' issue and commit
// cycles ([25, 26] S issuer in the max pass and sweeps, [27, 28] O issuer).
#ifdef ENTMAX_DIAG
#define DIAG(...) __VA_ARGS__
#else
#define DIAG(...)
#endif

// What the decision step publishes to the TMA and MMA warps: a refinement sweep (K tiles,
// S only), an output pass (K and V tiles, S and O), the fused first pass (an output pass at
// tau_T whose row owners also collect the candidates; more decisions follow), or nothing
// more (the fused pass's O is final).
constexpr int kKindSweep = 0;
constexpr int kKindOutput = 1;
constexpr int kKindFused = 2;
constexpr int kKindDone = 3;
__device__ __forceinline__ bool last_kind(int kind) { return kind == kKindOutput || kind == kKindDone; }

struct Shared {
  uint64_t full[kSlots], empty[kSlots];
  uint64_t bar_q;
  uint64_t s_full[kSBufs], s_free[kSBufs];     // sweeps: MMA -> rows, rows -> MMA
  uint64_t o_full[kOBufsMax], o_ready[kOBufsMax], pv_done[kOBufsMax];  // output pass, buffer c = k % obufs
  uint64_t mma_drain;                          // end of kernel: every issuer's MMAs complete
  uint64_t never;                              // self-test: a barrier nothing completes
  uint32_t tmem_base;
  int abort_flag;
  int ctl_kind, ctl_buf;
  uint32_t act[kMaskWords];          // structurally active key tiles
  uint32_t lists[2][kMaskWords];     // key tiles of the next sweep / the final mask
  uint32_t m64[2][2 * kMaskWords];   // the mask at 64 x 64 blocks: [row half][key block bits]
  int votes[kMaxVotes];
};

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// Order-preserving float <-> int map (shared-memory atomicMax on floats).
__device__ __forceinline__ int f2ord(float f) {
  const int i = __float_as_int(f);
  return i >= 0 ? i : i ^ 0x7fffffff;
}
__device__ __forceinline__ float ord2f(int i) { return __int_as_float(i >= 0 ? i : i ^ 0x7fffffff); }

// Load kCols consecutive fp32 TMEM columns of this thread's lane.
template <int N>
__device__ __forceinline__ void ldc(uint32_t taddr, float (&s)[N]);

// Load 64 consecutive fp32 TMEM columns of this thread's lane.
[[maybe_unused]] __device__ __forceinline__ void ld64(uint32_t taddr, float (&s)[64]) {
  uint32_t a[32], b[32];
  tmem_ld32(taddr, a);
  tmem_ld32(taddr + 32, b);
  tmem_wait_ld();
#pragma unroll
  for (int c = 0; c < 32; ++c) {
    s[c] = __uint_as_float(a[c]);
    s[32 + c] = __uint_as_float(b[c]);
  }
}

template <int N>
__device__ __forceinline__ void ldc(uint32_t taddr, float (&s)[N]) {
  if constexpr (N == 64) {
    ld64(taddr, s);
  } else {
    static_assert(N == 32, "32 or 64 columns per thread");
    uint32_t a[32];
    tmem_ld32(taddr, a);
    tmem_wait_ld();
#pragma unroll
    for (int c = 0; c < 32; ++c) s[c] = __uint_as_float(a[c]);
  }
}

// Loads kOCols fp32 TMEM columns (16 or 32) as raw words.
template <int N>
__device__ __forceinline__ void ldw(uint32_t taddr, uint32_t (&o)[N]) {
  if constexpr (N == 32) {
    tmem_ld32(taddr, o);
  } else {
    static_assert(N == 16, "16 or 32 columns per thread");
    tmem_ld16(taddr, o);
  }
  tmem_wait_ld();
}

// Output-pass TMEM layout per alpha. alpha = 2: g is 0 or 1, exact in fp16, so three S/A
// buffers at columns 0, 128, 384. alpha = 1.5: g = u is split into fp16 g_hi + g_lo (the
// rounding of g alone would move delta = dO . Ot / sum g by 2^-12 relative, which dK
// multiplies by |Q|); two S/A buffers at 0 and 128, and their g_lo blocks (64 columns of
// fp16 pairs each) at 384 and 448. O and Ot sit at 256 and 320 in both layouts.
template <int AK>
struct OutLayout {
  static constexpr int kBufs = 3;
  __device__ static __forceinline__ uint32_t sbuf(int c) { return c == 0 ? 0u : (c == 1 ? 128u : 384u); }
};

// Shared-memory layout of the forward (offsets from the 1024-aligned base): Q tile, K/V
// ring, the tile maxima [Tc][128], the candidate scores [4][cap][128] (fp32) and key
// indices [4][cap][128] (uint16), the partials. cap = 32 candidates per row and column part
// up to 64 key tiles, 24 beyond (so that L = 16384 fits in 227 KB).
__host__ __device__ constexpr int fwd_cand_cap(int Tc) { return Tc > 64 ? kCandLong : kCandPerThread; }
__host__ __device__ constexpr int fwd_off_region() { return kTileBytes * (1 + 4); }
__host__ __device__ constexpr int fwd_region_bytes(int Tc) {
  return Tc * kTile * 4 + 4 * fwd_cand_cap(Tc) * kTile * (4 + 2);
}

// Appends the scores of an 8-key group that pass tau (u = s cz - tau > 0) to this thread's
// candidate copies, without branches: every element is written to slot min(nc, cap-1) and
// nc advances only on a pass. A failing element lands in the next free slot, which the next
// passing one overwrites; once the list is full (nc >= cap) the copies are not used.
__device__ __forceinline__ void collect8(const float* s, int j, float cz, float tau, int cap, float* mycand,
                                         uint16_t* myidx, int& nc) {
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const bool pass = fmaf(s[e], cz, -tau) > 0.f;
    const int slot = min(nc, cap - 1);
    mycand[slot * kTile] = s[e];
    myidx[slot * kTile] = (uint16_t)(j + e);
    nc += pass ? 1 : 0;
  }
}

// The same append for four scores against a threshold in score units (s > thr).
__device__ __forceinline__ void collect4(const float* s, int j, float thr, int cap, float* mycand, uint16_t* myidx,
                                         int& nc) {
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const bool pass = s[e] > thr;
    const int slot = min(nc, cap - 1);
    mycand[slot * kTile] = s[e];
    myidx[slot * kTile] = (uint16_t)(j + e);
    nc += pass ? 1 : 0;
  }
}

// A score threshold below tau / cz (cz > 0): every s with fmaf(s, cz, -tau) > 0, that is
// s cz > tau exactly, has s > thr. The few extra scores at the boundary (u <= 0) are
// harmless candidates: every use of the copies tests u > 0.
__device__ __forceinline__ float cand_threshold(float tau, float cz) {
  const float q = tau / cz;
  return q - (fabsf(q) * 0x1p-20f + 1e-30f);
}

// Adds one candidate at u = z - t to the sums of the current support (u > 0), without
// a branch: the lanes of a warp follow one path whatever their candidates. S1 and S2 are
// sum u and sum u^2 (alpha = 1.5, 2); for the run-time variant they are sum g = sum u^{e-1}
// and sum p = sum u^e. In every case f = sum p - 1 and |f'| = e sum g (see root_terms).
template <int AK>
__device__ __forceinline__ void accumulate(float u, float e, float& S1, float& S2, float& C, float& umin) {
  const bool in = u > 0.f;
  if constexpr (AK == kAlphaGen) {
    const float l = __log2f(in ? u : 1.f);
    S1 += in ? exp2f((e - 1.f) * l) : 0.f;
    S2 += in ? exp2f(e * l) : 0.f;
  } else {
    const float v = in ? u : 0.f;
    S1 += v;
    S2 = fmaf(v, v, S2);
  }
  C += in ? 1.f : 0.f;
  umin = fminf(umin, in ? u : INFINITY);
}

// f(t) = sum_j p_j - 1 (Eq. 4) and |f'(t)| = e sum_j g_j from the sums of accumulate.
template <int AK>
__device__ __forceinline__ void root_terms(float S1, float S2, float C, float e, float& f, float& fp) {
  if constexpr (AK == kAlpha15) {
    f = S2 - 1.f;
    fp = 2.f * S1;
  } else if constexpr (AK == kAlpha2) {
    f = S1 - 1.f;
    fp = C;
  } else {
    f = S2 - 1.f;
    fp = e * S1;
  }
}

// Exact root of Eq. 4 restricted to the current support (alpha = 1.5: the smaller root of
// C d^2 - 2 S1 d + S2 - 1 = 0; alpha = 2: (S1-1)/C), as the step d from t; -1 when there is
// no closed form (run-time alpha) or no real root.
template <int AK>
__device__ __forceinline__ float piece_root(float S1, float S2, float C) {
  if constexpr (AK == kAlpha15) {
    const float disc = S1 * S1 - C * (S2 - 1.f);
    return disc >= 0.f ? (S2 - 1.f) / (S1 + sqrtf(disc)) : -1.f;   // = (S1 - sqrt(disc)) / C
  } else if constexpr (AK == kAlpha2) {
    return (S1 - 1.f) / C;
  } else {
    return -1.f;
  }
}

// Support sums of list[k*stride], k < n, at t: four independent partial sums, so the
// adds do not form one serial chain.
template <int AK>
__device__ __forceinline__ void sum_list(const float* list, int n, int stride, float cz, float t, float e, float& S1,
                                         float& S2, float& C, float& umin) {
  float a1[4] = {0.f, 0.f, 0.f, 0.f}, a2[4] = {0.f, 0.f, 0.f, 0.f}, ac[4] = {0.f, 0.f, 0.f, 0.f};
  float am[4] = {INFINITY, INFINITY, INFINITY, INFINITY};
  int k = 0;
  for (; k + 4 <= n; k += 4) {
#pragma unroll
    for (int q = 0; q < 4; ++q)
      accumulate<AK>(fmaf(list[(k + q) * stride], cz, -t), e, a1[q], a2[q], ac[q], am[q]);
  }
  for (; k < n; ++k) accumulate<AK>(fmaf(list[k * stride], cz, -t), e, a1[0], a2[0], ac[0], am[0]);
  S1 += (a1[0] + a1[1]) + (a1[2] + a1[3]);
  S2 += (a2[0] + a2[1]) + (a2[2] + a2[3]);
  C += (ac[0] + ac[1]) + (ac[2] + ac[3]);
  umin = fminf(umin, fminf(fminf(am[0], am[1]), fminf(am[2], am[3])));
}

// Safeguarded solve of Eq. 4 for one row over raw scores vals[q*list_stride + k*stride]
// (q < kParts, k < n[q]), which must hold every score that can be in the support.
// u = fma(s, cz, -t). Starts at t (a lower bound) inside [lo, hi]; on success returns
// true with the exact root up to fp32 rounding.
template <int AK>
__device__ bool solve_list(const float* vals, const int (&n)[kParts], int list_stride, int stride, float cz,
                           float e, float t, float lo, float hi, float& t_out) {
  // The run-time alpha variant has no closed form; for alpha > 2, f is concave with an
  // unbounded slope where a candidate enters the support, so Newton can crawl: every
  // fourth step bisects, which halves the bracket at least that often.
  constexpr int kIters = AK == kAlphaGen ? 96 : 48;
  for (int it = 0; it < kIters; ++it) {
    float S1 = 0.f, S2 = 0.f, C = 0.f, umin = INFINITY;
#pragma unroll
    for (int q = 0; q < kParts; ++q) sum_list<AK>(vals + q * list_stride, n[q], stride, cz, t, e, S1, S2, C, umin);
    float f, fp;   // f(t) and |f'(t)|
    root_terms<AK>(S1, S2, C, e, f, fp);
    if (C > 0.f) {
      const float d = piece_root<AK>(S1, S2, C);
      if (d >= 0.f && d < umin) {   // no candidate leaves the support at t + d: exact
        t_out = t + d;
        return true;
      }
    }
    // Without a closed form, Newton stops once f is at the rounding level of its sum (the
    // powers come from approximate exp2 / log2, relative error near 2^-21 per term).
    const float tol = AK == kAlphaGen ? fmaxf(4e-6f, C * 0x1p-19f) : 1e-7f;
    if (fabsf(f) <= tol && fp > 0.f) {
      t_out = t + f / fp;
      return true;
    }
    if (f > 0.f) lo = t; else hi = t;
    // Where f is nearly vertical (alpha > 2, a key just inside the support) |f| may never
    // reach its tolerance: the bracket reaching fp32 resolution ends the solve instead.
    if (AK == kAlphaGen && hi - lo <= fmaxf(fabsf(lo), 1.f) * 0x1p-22f) {
      t_out = 0.5f * (lo + hi);
      return true;
    }
    float tn = t + f / fp;
    if (!(tn > lo && tn <= hi && tn != t)) tn = 0.5f * (lo + hi);   // the root may sit at hi; a stalled step bisects
    if (AK == kAlphaGen && (it & 3) == 3) tn = 0.5f * (lo + hi);
    t = tn;
  }
  t_out = t;
  return false;
}

// The same solve with one row's work spread over the four lanes of a quad (lanes 4r..4r+3
// of a warp): each lane sums its own list (list[k*stride], k < n) and two butterfly
// shuffles combine the sums, so all four lanes take the same steps. Every lane of the warp
// runs the loop until all of its rows have finished; a lane whose row needs no solve passes
// active = false. Returns true (and the root in t_out) for a row solved exactly.
template <int AK>
__device__ bool solve_quad(const float* list, int n, int stride, bool active, float cz, float e, float t, float lo,
                           float hi, float& t_out) {
  constexpr int kIters = AK == kAlphaGen ? 96 : 48;
  bool fin = !active, ok = false;
  t_out = t;
  for (int it = 0; it < kIters && !__all_sync(0xffffffffu, fin); ++it) {
    float S1 = 0.f, S2 = 0.f, C = 0.f, umin = INFINITY;
    sum_list<AK>(list, n, stride, cz, t, e, S1, S2, C, umin);
#pragma unroll
    for (int m = 1; m <= 2; m <<= 1) {
      S1 += __shfl_xor_sync(0xffffffffu, S1, m);
      S2 += __shfl_xor_sync(0xffffffffu, S2, m);
      C += __shfl_xor_sync(0xffffffffu, C, m);
      umin = fminf(umin, __shfl_xor_sync(0xffffffffu, umin, m));
    }
    if (fin) continue;
    float f, fp;   // f(t) and |f'(t)|
    root_terms<AK>(S1, S2, C, e, f, fp);
    if (C > 0.f) {
      const float d = piece_root<AK>(S1, S2, C);
      if (d >= 0.f && d < umin) {   // no candidate leaves the support at t + d: exact
        t_out = t + d;
        ok = fin = true;
        continue;
      }
    }
    const float tol = AK == kAlphaGen ? fmaxf(4e-6f, C * 0x1p-19f) : 1e-7f;
    if (fabsf(f) <= tol && fp > 0.f) {
      t_out = t + f / fp;
      ok = fin = true;
      continue;
    }
    if (f > 0.f) lo = t; else hi = t;
    if (AK == kAlphaGen && hi - lo <= fmaxf(fabsf(lo), 1.f) * 0x1p-22f) {
      t_out = 0.5f * (lo + hi);
      ok = fin = true;
      continue;
    }
    float tn = t + f / fp;
    if (!(tn > lo && tn <= hi && tn != t)) tn = 0.5f * (lo + hi);
    if (AK == kAlphaGen && (it & 3) == 3) tn = 0.5f * (lo + hi);
    t = tn;
  }
  return ok;
}

// Threshold of Eq. 4 restricted to N raw scores v (some may be -inf), in registers:
// safeguarded Newton from lo inside [lo, hi], finished by the exact root of the current
// support's piece once no value leaves the support. A subset of the row's scores has a
// threshold at or below the row's tau*, so the result is a lower bound on tau*.
template <int AK, int N>
__device__ __forceinline__ float solveN(const float (&v)[N], float cz, float e, float lo, float hi) {
  float t = lo;
  for (int it = 0; it < 24; ++it) {
    float S1 = 0.f, S2 = 0.f, C = 0.f, umin = INFINITY;
#pragma unroll
    for (int q = 0; q < N; ++q) accumulate<AK>(fmaf(v[q], cz, -t), e, S1, S2, C, umin);
    float f, fp;
    root_terms<AK>(S1, S2, C, e, f, fp);
    if (C > 0.f) {
      const float d = piece_root<AK>(S1, S2, C);
      if (d >= 0.f && d < umin) return t + d;
    }
    if (fabsf(f) <= (AK == kAlphaGen ? 1e-6f : 1e-7f) && fp > 0.f) return t + f / fp;
    if (f > 0.f) lo = t; else hi = t;
    float tn = t + f / fp;
    if (!(tn > lo && tn <= hi && tn != t)) tn = 0.5f * (lo + hi);
    t = tn;
  }
  return lo;   // not settled: lo is still a lower bound
}

}  // namespace

// The 64 x 64 mask from the support lists (row owners, once per CTA; kept out of line so
// that it does not change the register allocation of the kernel's loops). A thread's keys
// lie in its column part qp of each tile, so a support key of tile jt is in 64-key block
// 2 jt + qp/2: the thread marks tiles, the warp (32 rows of one row half, one part) ORs the
// marks, and lane 0 spreads them to blocks and adds them to the shared mask m64 [2][8].
__device__ __noinline__ void m64_mark(uint32_t* m64, const float* mycand, const uint16_t* myidx, int nc, bool use,
                                      float cz, float tau, int quad, int qp, int lane) {
  uint32_t tm[kMaskWords];
#pragma unroll
  for (int w = 0; w < kMaskWords; ++w) tm[w] = 0u;
  if (use)
    for (int k = 0; k < nc; ++k)
      if (fmaf(mycand[k * kTile], cz, -tau) > 0.f) {
        const int jt = myidx[k * kTile] >> 7;
#pragma unroll
        for (int w = 0; w < kMaskWords; ++w) tm[w] |= (jt >> 5) == w ? 1u << (jt & 31) : 0u;
      }
#pragma unroll
  for (int w = 0; w < kMaskWords; ++w) {
    const uint32_t x = __reduce_or_sync(0xffffffffu, tm[w]);
    if (lane == 0 && x != 0u) {
      // tile bit b of word w -> block bit 2 b + qp/2, in words 2w and 2w + 1
#pragma unroll
      for (int hw = 0; hw < 2; ++hw) {
        uint32_t v = (x >> (16 * hw)) & 0xffffu;   // spread 16 bits to the even positions
        v = (v | (v << 8)) & 0x00ff00ffu;
        v = (v | (v << 4)) & 0x0f0f0f0fu;
        v = (v | (v << 2)) & 0x33333333u;
        v = (v | (v << 1)) & 0x55555555u;
        if (v) atomicOr(&m64[(quad >> 1) * 2 * kMaskWords + 2 * w + hw], v << (qp >> 1));
      }
    }
  }
}

// Rows 2 qt and 2 qt + 1 of the 64 x 64 mask and their bits of the transpose (threads
// tid < 2 W64c, after every mark is in m64).
__device__ __noinline__ void m64_write(const uint32_t* m64, const FwdParams& p, int tid, int bh, int qt) {
  const int h = tid / p.W64c, w = tid % p.W64c;
  const uint32_t bits = m64[h * 2 * kMaskWords + w];
  const int qb = 2 * qt + h;
  p.M64[((size_t)bh * 2 * p.Tr + qb) * p.W64c + w] = bits;
  for (uint32_t b = bits; b; b &= b - 1) {
    const int kb = w * 32 + __ffs(b) - 1;
    atomicOr(&p.M64T[((size_t)bh * 2 * p.Tc + kb) * p.W64r + (qb >> 5)], 1u << (qb & 31));
  }
}

template <int AK, bool kAlibi, bool kM64>
__global__ void __launch_bounds__(kThreads, 1) fwd_kernel(const __grid_constant__ FwdParams p) {
  using OL = OutLayout<AK>;
  constexpr int kOBufs = OL::kBufs;
  extern __shared__ uint8_t dsm_raw[];
  __shared__ Shared sh;
  uint8_t* dsm = align1024(dsm_raw);
  static_assert(kSlots == 4 && kParts == 4, "fwd_region_bytes assumes these");
  uint8_t* sQ = dsm;
  uint8_t* ring = dsm + kTileBytes;
  int* tmax = reinterpret_cast<int*>(dsm + fwd_off_region());    // [Tc][128], f2ord
  const int cap = fwd_cand_cap(p.Tc);
  float* cand = reinterpret_cast<float*>(tmax + p.Tc * kTile);   // [kParts][cap][128] scores
  uint16_t* cidx = reinterpret_cast<uint16_t*>(cand + kParts * cap * kTile);   // [kParts][cap][128] key indices
  float* part = reinterpret_cast<float*>(dsm + fwd_off_region() + fwd_region_bytes(p.Tc));   // [kParts][4][128]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bh = blockIdx.x % p.BH;
  const int qt = p.Tr - 1 - blockIdx.x / p.BH;     // longest (causal) tiles first
  const int b = bh / p.H;
  const Pattern pat{p.L, p.kv_len ? min(max(p.kv_len[b], 1), p.L) : p.L, p.causal, p.window};
  const int i0 = qt * kTile, i1 = min(p.L, i0 + kTile);
  int* status = p.status;
  const WaitCtx wc{status, &sh.abort_flag, p.wait_limit_ns};

  if (tid == 0) {
    for (int s = 0; s < kSlots; ++s) {
      mbar_init(&sh.full[s], 1);
      mbar_init(&sh.empty[s], 1);   // one commit by the MMA issuer that reads the slot
    }
    mbar_init(&sh.bar_q, 1);
    for (int s = 0; s < kSBufs; ++s) {
      mbar_init(&sh.s_full[s], 1);
      mbar_init(&sh.s_free[s], kMathWarps);
    }
    for (int s = 0; s < kOBufsMax; ++s) {
      mbar_init(&sh.o_full[s], 1);
      mbar_init(&sh.o_ready[s], kMathWarps);
      mbar_init(&sh.pv_done[s], 1);   // the O chain
    }
    mbar_init(&sh.mma_drain, 3);   // one commit per MMA issuer
    mbar_init(&sh.never, 1);
    sh.abort_flag = 0;
    fence_mbar_init();
  }
  if (tid < kMaskWords) {
    sh.act[tid] = 0;
    sh.lists[0][tid] = 0;
    sh.lists[1][tid] = 0;
  }
  for (int v = tid; v < kMaxVotes; v += kThreads) sh.votes[v] = 0;
  if (tid < 4 * kMaskWords) (&sh.m64[0][0])[tid] = 0;
  for (int e = tid; e < p.Tc * kTile; e += kThreads) tmax[e] = f2ord(-INFINITY);
  if (warp == kMmaWarp) {
    tmem_alloc(&sh.tmem_base, 512);
    tmem_relinquish();
  }
  __syncthreads();
  for (int jt = tid; jt < p.Tc; jt += kThreads)
    if (pat.block_active(i0, i1, jt * kTile, min(p.L, jt * kTile + kTile)))
      atomicOr(&sh.act[jt >> 5], 1u << (jt & 31));
  __syncthreads();
  tc_fence_after();
  const long long clk0 = clock64();
  const uint32_t T = sh.tmem_base;
  uint32_t act[kMaskWords];
#pragma unroll
  for (int w = 0; w < kMaskWords; ++w) act[w] = sh.act[w];

  if (warp == kProducerWarp) {
    // ------------------------------------------------------------------ TMA producer
    // Ring positions are taken in program order: every tile of phase 1 and of each
    // sweep is one K load; the output pass loads K_k, V_k, K_{k+1}, V_{k+1}, ...
    // After a failed wait (abort) no further copy is issued, so at most kSlots copies,
    // one per slot, are ever in flight, and the drain below sees each slot's last one.
    uint32_t seq = 0;
    bool live = true;
    DIAG(long long dg_wait = 0);
    auto load = [&](const CUtensorMap* map, int jt) {
      if (!live) return;
      const int slot = seq % kSlots;
      DIAG(const long long d0 = clock64());
      if (!mbar_wait(&sh.empty[slot], ((seq / kSlots) & 1) ^ 1, wc)) {
        live = false;
        return;
      }
      DIAG(dg_wait += clock64() - d0);
      mbar_expect_tx(&sh.full[slot], kTileBytes);
      tma_load_3d(ring + slot * kTileBytes, map, &sh.full[slot], 0, jt * kTile, bh);
      ++seq;
    };
    if (lane == 0) {
      tma_prefetch_desc(&p.tQ);
      tma_prefetch_desc(&p.tK);
      tma_prefetch_desc(&p.tV);
      mbar_expect_tx(&sh.bar_q, kTileBytes);
      tma_load_3d(sQ, &p.tQ, &sh.bar_q, 0, i0, bh);
      for_each_bit(act, kMaskWords, [&](int jt) { load(&p.tK, jt); });
    }
    __syncwarp();
    while (true) {
      named_bar(1, kThreads);
      const int kind = sh.ctl_kind;
      uint32_t list[kMaskWords];
#pragma unroll
      for (int w = 0; w < kMaskWords; ++w) list[w] = sh.lists[sh.ctl_buf][w];
      if (lane == 0) {
        if (kind == kKindSweep) {
          for_each_bit(list, kMaskWords, [&](int jt) { load(&p.tK, jt); });
        } else if (kind != kKindDone) {
          for_each_bit(list, kMaskWords, [&](int jt) {
            load(&p.tK, jt);
            load(&p.tV, jt);
          });
        }
      }
      __syncwarp();
      if (last_kind(kind)) break;
    }
    DIAG(if (lane == 0) p.stats[((size_t)bh * p.Tr + qt) * kFwdStats + 15] = (int)dg_wait);
    // Make sure no copy is still in flight when the CTA retires.
    if (lane == 0) {
      mbar_drain(&sh.bar_q, 0, status);
      for (uint32_t k = (seq > kSlots ? seq - kSlots : 0); k < seq; ++k)
        mbar_drain(&sh.full[k % kSlots], (k / kSlots) & 1, status);
    }
    __syncwarp();
  } else if (warp == kMmaWarp || warp == kSWarp2) {
    // ------------------------------------------------------------------- MMA issuer
    uint32_t seq = 0;            // next ring position (sweeps consume in order)
    uint32_t sfree_par = 0;      // per sweep S buffer: parity of its uses so far (bit b)
    uint32_t sbuf = 0;           // next sweep S buffer
    uint32_t obase = 0;          // output tiles of earlier output-type passes (buffer phases)
    bool live = true;            // false after a failed wait: no further MMA is issued
    // Two S issuers share the max pass and the sweeps: issuer me takes the tiles whose
    // buffer (tile index % 4) has parity me, so each one's barrier probes and commits
    // overlap the other's MMAs. Both walk every tile to keep the positions and parities.
    const uint32_t me = warp == kMmaWarp ? 0u : 1u;
    DIAG(long long dg_sw = 0; long long dg_out = 0; long long dg_iss = 0);
    const uint32_t idS = idesc_bf16(128, 128, 0, 0);
    const uint64_t qd0 = sdesc_sw128(smem_u32(sQ), 16, 1024);      // Q tile, K-major
    const uint64_t kd0 = sdesc_sw128(smem_u32(ring), 16, 1024);    // ring slot 0, K-major
    // S = Q K^T from ring position `pos` (already landed) into TMEM columns [dcol, dcol+128).
    auto mma_s = [&](uint32_t pos, uint32_t dcol) {
      const int slot = pos % kSlots;
      tc_fence_after();
      const uint64_t kd = sdesc_add(kd0, slot * kTileBytes);
#pragma unroll
      for (int k = 0; k < 4; ++k) mma_ss(T + dcol, sdesc_add(qd0, k * 32), sdesc_add(kd, k * 32), idS, k > 0);
      mma_commit(&sh.empty[slot]);   // a K slot is read by this issuer only
    };
    auto sweep_tile = [&]() {
      const uint32_t bf = sbuf;
      const uint32_t pos = seq++;
      if ((bf & 1u) == me) {
        // S buffer consumed by the row owners, and K tile landed.
        DIAG(const long long d0 = clock64());
        live = live && mbar_wait2(&sh.s_free[bf], ((sfree_par >> bf) & 1) ^ 1, &sh.full[pos % kSlots],
                                  (pos / kSlots) & 1, wc);
        DIAG(dg_sw += clock64() - d0);
        if (live) {
          mma_s(pos, bf * 128);
          mma_commit(&sh.s_full[bf]);
        }
        DIAG(dg_iss += clock64() - d0);
      }
      sfree_par ^= 1u << bf;
      sbuf = (sbuf + 1) & (kSBufs - 1);
    };
    if (lane == 0) {
      if ((p.selftest & kSelftestStall) && me == 0) live = mbar_wait(&sh.never, 0, wc);   // expires: nothing completes it
      live = live && mbar_wait(&sh.bar_q, 0, wc);
      for_each_bit(act, kMaskWords, [&](int) { sweep_tile(); });
    }
    __syncwarp();
    while (true) {
      named_bar(1, kThreads);
      const int kind = sh.ctl_kind;
      uint32_t list[kMaskWords];
#pragma unroll
      for (int w = 0; w < kMaskWords; ++w) list[w] = sh.lists[sh.ctl_buf][w];
      if (lane == 0) {
        if (kind == kKindSweep) {
          sbuf = 0;
          for_each_bit(list, kMaskWords, [&](int) { sweep_tile(); });
        } else if (kind != kKindDone) {
          int n = 0;
#pragma unroll
          for (int w = 0; w < kMaskWords; ++w) n += __popc(list[w]);
          if (me == 0) {
            // Output-type pass: this warp issues only the S tiles. Tile k of the pass is
            // output tile ko = obase + k overall and uses buffer c = ko % 3 (TMEM column 0,
            // 128 or 384), free once O of output tile ko - 3 is done. K_k is at ring
            // position seq + 2k, V_k at seq + 2k + 1.
            for (int k = 0; k < n; ++k) {
              const uint32_t ko = obase + k;
              const int c = ko % kOBufs;
              const uint32_t pos = seq + 2 * k;
              DIAG(const long long d0 = clock64());
              if (ko >= kOBufs)
                live = live && mbar_wait2(&sh.pv_done[c], ((ko - kOBufs) / kOBufs) & 1, &sh.full[pos % kSlots],
                                          (pos / kSlots) & 1, wc);
              else
                live = live && mbar_wait(&sh.full[pos % kSlots], (pos / kSlots) & 1, wc);
              DIAG(dg_out += clock64() - d0);
              if (!live) break;
              mma_s(pos, OL::sbuf(c));
              mma_commit(&sh.o_full[c]);
            }
            DIAG(p.stats[((size_t)bh * p.Tr + qt) * kFwdStats + 12] = (int)dg_sw);
            DIAG(p.stats[((size_t)bh * p.Tr + qt) * kFwdStats + 13] = (int)dg_out);
            DIAG(p.stats[((size_t)bh * p.Tr + qt) * kFwdStats + 25] = (int)(dg_iss - dg_sw));
          }
          seq += 2 * n;
          obase += n;
        }
      }
      __syncwarp();
      if (last_kind(kind)) break;
    }
  } else if (warp == kOWarp) {
    // ------------------------------------------------------ O issuer (output passes)
    const uint32_t idO = idesc_f16(128, 64, 0, 1);
    const uint64_t vd0 = sdesc_sw128(smem_u32(ring), 8192, 1024);   // ring slot 0, MN-major
    uint32_t seq = 0;     // ring positions, tracked exactly like the producer's
    uint32_t obase = 0;   // output tiles of earlier output-type passes
    for_each_bit(act, kMaskWords, [&](int) { ++seq; });
    while (true) {
      named_bar(1, kThreads);
      const int kind = sh.ctl_kind;
      uint32_t list[kMaskWords];
#pragma unroll
      for (int w = 0; w < kMaskWords; ++w) list[w] = sh.lists[sh.ctl_buf][w];
      int n = 0;
#pragma unroll
      for (int w = 0; w < kMaskWords; ++w) n += __popc(list[w]);
      if (kind == kKindSweep) {
        seq += n;
      } else if (kind != kKindDone) {
        if (lane == 0) {
          DIAG(long long dg_o = 0);
          for (int k = 0; k < n; ++k) {
            const uint32_t ko = obase + k;
            const int c = ko % kOBufs;
            const uint32_t pa = OL::sbuf(c);
            const uint32_t vpos = seq + 2 * k + 1;
            const int vslot = vpos % kSlots;
            DIAG(const long long d0 = clock64());
            if (!mbar_wait2(&sh.full[vslot], (vpos / kSlots) & 1, &sh.o_ready[c], (ko / kOBufs) & 1, wc)) break;
            DIAG(dg_o += clock64() - d0);
            tc_fence_after();
            const uint64_t vd = sdesc_add(vd0, vslot * kTileBytes);
#pragma unroll
            for (int t = 0; t < 8; ++t) {
              // keys 16t..16t+15: part 16t / kCols, pair columns ((16t) % kCols) / 2 of its A block
              const uint32_t col = pa + (16 * t / kCols) * kCols + ((16 * t) % kCols) / 2;   // A block
              mma_ts(T + 256, T + col, sdesc_add(vd, t * 2048), idO, (k > 0 || t > 0) ? 1u : 0u);
            }
            mma_commit(&sh.empty[vslot]);   // V_k is read by this issuer only
            mma_commit(&sh.pv_done[c]);
          }
          DIAG(p.stats[((size_t)bh * p.Tr + qt) * kFwdStats + 14] = (int)dg_o);
        }
        seq += 2 * n;
        obase += n;
      }
      __syncwarp();
      if (last_kind(kind)) break;
    }
  } else {
    // ---------------------------------------------------------------- row owners
    const int quad = warp & 3, qp = warp >> 2;   // TMEM lane quadrant, column part
    const int row = quad * 32 + lane;
    const int i = i0 + row;
    const bool valid = i < p.L;
    const uint32_t tl = T + ((uint32_t)(quad * 32) << 16);
    const float cz = p.cz;
    const float cb = kAlibi ? p.alibi[bh % p.H] * p.inv_scale : 0.f;   // ALiBi, raw score units
    uint32_t sfull_par = 0, sbuf = 0;
    float m = -INFINITY;
    float top[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
    DIAG(long long dg_s1 = 0; long long dg_s2 = 0; long long dg_s3 = 0; long long dg_sw1 = 0);
    DIAG(long long dgr[9] = {0, 0, 0, 0, 0, 0, 0, 0, 0}; long long dtk = 0);
    DIAG(long long dgx[6] = {0, 0, 0, 0, 0, 0});   // [26] tau_T solve, [27] decisions, [28] post-sweep solves, [29] epilogue
    DIAG(long long dg_solve = 0);                  // [11] the exact solves alone

    // Phase 1: per-key-tile row maxima over this thread's column part (combined in smem).
    for_each_bit(act, kMaskWords, [&](int jt) {
      const uint32_t bf = sbuf;
      DIAG(const long long d0 = clock64());
      warp_wait(&sh.s_full[bf], (sfull_par >> bf) & 1, wc);
      DIAG(const long long d1 = clock64(); dg_s1 += d1 - d0);
      sfull_par ^= 1u << bf;
      tc_fence_after();
      const int j0 = jt * kTile + qp * kCols;
      float s[kCols];
      ldc(tl + bf * 128 + qp * kCols, s);
      DIAG(const long long d2 = clock64(); dgr[0] += d2 - d1);
      tc_fence_before();
      warp_arrive(&sh.s_free[bf]);
      DIAG(dtk = clock64(); dgr[1] += dtk - d2);
      if constexpr (kAlibi) alibi_apply(s, cb, i, j0);
      if (!pat.block_full(i0, i1, jt * kTile, jt * kTile + kTile)) {
#pragma unroll
        for (int c = 0; c < kCols; ++c)
          if (!pat.active(i, j0 + c)) s[c] = -INFINITY;
      }
      float t8[8];   // eight independent max chains
#pragma unroll
      for (int c = 0; c < 8; ++c) t8[c] = s[c];
#pragma unroll
      for (int c = 8; c < kCols; ++c) t8[c & 7] = fmaxf(t8[c & 7], s[c]);
      const float tm = fmaxf(fmaxf(fmaxf(t8[0], t8[1]), fmaxf(t8[2], t8[3])),
                             fmaxf(fmaxf(t8[4], t8[5]), fmaxf(t8[6], t8[7])));
      atomicMax(&tmax[jt * kTile + row], f2ord(tm));
      // Keep the four largest part-tile maxima, sorted (compare-exchange, no branch).
      float x = tm;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float big = fmaxf(top[k], x);
        x = fminf(top[k], x);
        top[k] = big;
      }
      sbuf = (sbuf + 1) & (kSBufs - 1);
      DIAG(dgr[2] += clock64() - dtk);
    });
    // All column parts' four largest part-tile maxima: the row max and the values of the
    // initial threshold.
#pragma unroll
    for (int k = 0; k < 4; ++k) part[(qp * 4 + k) * kTile + row] = top[k];
    named_bar(3, kMathThreads);
    float vt[4 * kParts];
#pragma unroll
    for (int k = 0; k < 4 * kParts; ++k) vt[k] = part[k * kTile + row];
    named_bar(3, kMathThreads);   // read before anyone rewrites the partials
    const long long clk1 = clock64();
    long long clk2 = clk1;
#pragma unroll
    for (int q = 0; q < kParts; ++q) m = fmaxf(m, vt[4 * q]);

    // Bracket (§2.4) and the tile-maxima lower bound (identical in all threads of a row).
    const int n_act = valid ? pat.count(i) : 1;
    const float mz = m * cz;
    float lo = mz - 1.f;
    float hi = mz - ((AK == kAlpha15)  ? rsqrtf((float)n_act)
                     : (AK == kAlpha2) ? 1.f / (float)n_act
                                       : pow_pos((float)n_act, -p.am1));   // n^{1-alpha}
    float tau = INFINITY;
    bool done = !valid;
    bool listed = false;   // solved on candidate copies that hold the whole support
    bool near_once = false;   // a Newton correction within tolerance was taken while the copies overflowed
    int nc = 0;            // this thread's candidate count in the sweep that solved its row
    if (valid) {
      // The row's largest part-tile maxima are a subset of its scores, so the threshold
      // of entmax on them is a lower bound tau_T <= tau*.
      DIAG(const long long ds0 = clock64());
      const float t = solveN<AK, 4 * kParts>(vt, cz, p.ae, lo, hi);
      tau = fminf(fmaxf(t, lo), hi);
      DIAG(dgx[0] += clock64() - ds0);
    }
    int sweeps = 0;
    int fused_passes = 0;   // the fused first pass counts as a sweep for max_sweeps, not in the counters
    uint32_t n_s = 0;       // S tiles computed (phase 1, sweeps, output) for the counters
    uint32_t obase = 0;     // output tiles of earlier output-type passes (barrier phases)
    float tau_T = tau;      // the threshold at which the fused pass formed A
    for_each_bit(act, kMaskWords, [&](int) { ++n_s; });
    float* mycand = cand + qp * cap * kTile + row;
    uint16_t* myidx = cidx + qp * cap * kTile + row;

    // Candidate collection on one tile's scores: the maxima of the eight 4-key groups
    // (independent pairs), then an append of only the groups whose maximum passes the
    // threshold thr (cand_threshold). A group is appended when any lane of the warp has a
    // candidate in it (a warp-uniform branch; 32 rows share the vote, so smaller groups
    // are scanned less often); each lane then runs the same branch-free append.
    auto collect_tile = [&](const float (&sv)[kCols], int j0, bool collect, float thr) {
      float gm[kCols / 4];
#pragma unroll
      for (int g = 0; g < kCols / 4; ++g) gm[g] = fmaxf(fmaxf(sv[4 * g], sv[4 * g + 1]), fmaxf(sv[4 * g + 2], sv[4 * g + 3]));
#pragma unroll
      for (int g = 0; g < kCols / 4; ++g)
        if (__any_sync(0xffffffffu, collect && gm[g] > thr))
          if (collect) collect4(sv + 4 * g, j0 + 4 * g, thr, cap, mycand, myidx, nc);
    };
    // One tile of an output-type pass (output tile ko overall, buffer ko % 3): recompute
    // S, optionally collect this thread's candidates at tau, and write A = u^{1/(alpha-1)}
    // at tau in fp16 over the S columns this thread has read (the part's keys qp*kCols..
    // go into its own columns [qp*kCols, +kCols/2), so the row's other parts never see an
    // overwritten S value).
    auto out_tile = [&](int jt, uint32_t ko, float thr, auto collect_tag, auto mark_tag) {
      constexpr bool collect = decltype(collect_tag)::value, mark = decltype(mark_tag)::value;
      const int c = ko % kOBufs;
      const uint32_t pa = OL::sbuf(c);
      DIAG(const long long d0 = clock64());
      warp_wait(&sh.o_full[c], (ko / kOBufs) & 1, wc);
      DIAG(const long long d1 = clock64(); dg_s3 += d1 - d0);
      tc_fence_after();
      const int j0 = jt * kTile + qp * kCols;
      float s[kCols];
      ldc(tl + pa + qp * kCols, s);
      DIAG(const long long d2 = clock64(); dgr[6] += d2 - d1);
      if constexpr (kAlibi) alibi_apply(s, cb, i, j0);
      if (!pat.block_full(i0, i1, jt * kTile, jt * kTile + kTile)) {
#pragma unroll
        for (int cc = 0; cc < kCols; ++cc)
          if (!pat.active(i, j0 + cc)) s[cc] = -INFINITY;
      }
      if constexpr (collect) collect_tile(s, j0, !done, thr);
      if constexpr (mark) {   // the 64 x 64 mask at the final tau: a score of this part above tau
        float mx = s[0];
#pragma unroll
        for (int cc = 1; cc < kCols; ++cc) mx = fmaxf(mx, s[cc]);
        const int kb = 2 * jt + (qp >> 1);
        if (__any_sync(0xffffffffu, fmaf(mx, cz, -tau) > 0.f) && lane == 0)
          atomicOr(&sh.m64[quad >> 1][kb >> 5], 1u << (kb & 31));
      }
      uint32_t aw[kCols / 2];
#pragma unroll
      for (int cc = 0; cc < kCols / 2; ++cc) {
        const float2 u = __ffma2_rn(make_float2(s[2 * cc], s[2 * cc + 1]), make_float2(cz, cz),
                                    make_float2(-tau, -tau));
        const float v0 = fmaxf(u.x, 0.f), v1 = fmaxf(u.y, 0.f);
        if constexpr (AK == kAlpha15) {
          const float2 a = __fmul2_rn(make_float2(v0, v1), make_float2(v0, v1));
          aw[cc] = pack_f16(a.x, a.y);
        } else if constexpr (AK == kAlpha2) {
          aw[cc] = pack_f16(v0, v1);
        } else {
          aw[cc] = pack_f16(v0 > 0.f ? pow_pos(v0, p.ae) : 0.f, v1 > 0.f ? pow_pos(v1, p.ae) : 0.f);
        }
      }
      const uint32_t col = pa + qp * kCols;
      DIAG(const long long d3 = clock64(); dgr[7] += d3 - d2);
#pragma unroll
      for (int h = 0; h < kCols / 32; ++h) tmem_st16(tl + col + 16 * h, *reinterpret_cast<uint32_t(*)[16]>(&aw[16 * h]));
      tmem_wait_st();
      tc_fence_before();
      warp_arrive(&sh.o_ready[c]);
      DIAG(dgr[8] += clock64() - d3);
      ++n_s;
    };

    // Decision points: publish one more refinement sweep, the fused first pass, the final
    // mask with an output pass, or the final mask alone.
    //
    // For alpha in {1.5, 2} the first pass after the max pass is fused: an output pass at
    // tau_T over the tiles where some row has a score above tau_T, whose row owners also
    // collect the candidates (u_T > 0). A row whose copies fit is then solved exactly on
    // them, and its O = sum_j A*_j V_j follows from the pass's O_T = sum_j fp16(A_T,j) V_j
    // (every j with u_T,j > 0 lies in a visited tile) and its copies: the epilogue adds
    // sum_j (A*_j - fp16(A_T,j)) V_j over the copies in fp32, with A* at the final tau
    // (zero outside the support). When every row of the tile is solved that way no second
    // pass over K and V is needed. Otherwise the remaining rows sweep as below, and an
    // output pass at the final tau recomputes O for the whole tile.
    for (int r = 0;; ++r) {
      DIAG(const long long dd0 = clock64());
      const int buf = r & 1;
      const bool need = !done && sweeps < p.max_sweeps;
      const bool final_mask = !rows_any(need, sh.votes, r, lane, kMathThreads);
      const bool fuse = AK != kAlphaGen && r == 0 && !final_mask;
      // The fused pass's O is final when every row was solved on that pass's copies.
      const bool o_final = AK != kAlphaGen && r == 1 && final_mask &&
                           !rows_any(valid && !listed, sh.votes, kMaxVotes - 1, lane, kMathThreads);
      {
        // Tiles that some row still needs (refinement) or that hold a nonzero (mask): the
        // warps of column part qp take the groups of eight tiles 8 g with g % 4 == qp (the
        // four warps of a part cover all 128 rows); each builds its bits from eight
        // independent loads and votes per group and ORs them into the list once per word.
        const bool take = final_mask ? valid : !done;
        for (int w = 0; w < kMaskWords; ++w) {
          if (act[w] == 0) continue;
          uint32_t word = 0;
          for (int b0 = 8 * qp; b0 < 32 && w * 32 + b0 < p.Tc; b0 += 8 * kParts) {
            const int jb = w * 32 + b0;
            float v[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) v[q] = jb + q < p.Tc ? ord2f(tmax[(jb + q) * kTile + row]) : -INFINITY;
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              const uint32_t bal = __ballot_sync(0xffffffffu, take && fmaf(v[q], cz, -tau) > 0.f);
              word |= (bal != 0u ? 1u : 0u) << (b0 + q);
            }
          }
          if (lane == 0 && word) atomicOr(&sh.lists[buf][w], word & act[w]);
        }
      }
      named_bar(2, kMathThreads);
      if (tid == 0) {
        sh.ctl_kind = final_mask ? (o_final ? kKindDone : kKindOutput) : (fuse ? kKindFused : kKindSweep);
        sh.ctl_buf = buf;
        for (int w = 0; w < kMaskWords; ++w) sh.lists[buf ^ 1][w] = 0;   // for the next decision
      }
      uint32_t list[kMaskWords];
#pragma unroll
      for (int w = 0; w < kMaskWords; ++w) list[w] = sh.lists[buf][w];
      named_bar(1, kThreads);
      DIAG(dgx[1] += clock64() - dd0);

      if (final_mask) {
        if (!o_final) clk2 = clock64();
        if (!done && qp == 0) atomicOr(status, kStatusNoConverge);   // cap reached; tau stays bracketed
        // Block mask row of this query tile and the transposed bits (Appendix C.4).
        if (tid < p.Wc) p.M[((size_t)bh * p.Tr + qt) * p.Wc + tid] = list[tid];
        if (tid == 0) {
          for_each_bit(list, kMaskWords, [&](int jt) {
            atomicOr(&p.MT[((size_t)bh * p.Tc + jt) * p.Wr + (qt >> 5)], 1u << (qt & 31));
          });
        }
        int n_out = 0;
#pragma unroll
        for (int w = 0; w < kMaskWords; ++w) n_out += __popc(list[w]);
        DIAG(const long long de0 = clock64());
        if (!o_final) {
          // Phase 4: output pass at the final tau over the flagged tiles.
          int k = 0;
          for_each_bit(list, kMaskWords,
                       [&](int jt) { out_tile(jt, obase + k++, 0.f, std::false_type{}, std::integral_constant<bool, kM64>{}); });
          if (k > 0) warp_wait(&sh.pv_done[(obase + k - 1) % kOBufs], ((obase + k - 1) / kOBufs) & 1, wc);
          obase += k;
        }
        DIAG(const long long de1 = clock64(); dgx[4] += de1 - de0);
        // Epilogue: O from TMEM (each thread of a row writes kOCols of the 64 columns).
        tc_fence_after();
        uint32_t o[kOCols];
        ldw(tl + 256 + qp * kOCols, o);
        if (valid) {
          float4* dst = reinterpret_cast<float4*>(p.O + ((size_t)bh * p.L + i) * kD + qp * kOCols);
#pragma unroll
          for (int cc = 0; cc < kOCols / 4; ++cc)
            dst[cc] = make_float4(__uint_as_float(o[4 * cc]), __uint_as_float(o[4 * cc + 1]),
                                  __uint_as_float(o[4 * cc + 2]), __uint_as_float(o[4 * cc + 3]));
        }
        // The backward's delta needs Ot_i = sum_j g_ij V_j and sum_j g_ij over row i's support.
        // A row solved on its candidate copies has them all in shared memory (scores and key
        // indices from the sweep that solved it). The gather of the bf16 V rows (exact;
        // widened with shifts) is laid out for the memory system rather than for TMEM: eight
        // lanes per row, each lane 8 of the 64 columns, so one load instruction reads four
        // whole 128-byte V rows, and the warps take 64 rows per round. A row without complete
        // copies (refinement cap, or a Newton finish) gets sum g = -1, and the backward
        // recomputes its support.
        DIAG(const long long de2 = clock64(); dgx[5] += de2 - de1);
        if constexpr (kM64)
          if (o_final)   // the 64 x 64 mask from the support lists
            m64_mark(&sh.m64[0][0], mycand, myidx, nc, valid && listed, cz, tau, quad, qp, lane);
        if (qp == 0) {
          part[3 * kTile + row] = tau;
          part[7 * kTile + row] = (valid && listed) ? 1.f : 0.f;
          part[11 * kTile + row] = tau_T;
          if (valid) p.tau[(size_t)bh * p.L + i] = tau;
        }
        named_bar(3, kMathThreads);
        if constexpr (kM64)
          if (tid < 2 * p.W64c) m64_write(&sh.m64[0][0], p, tid, bh, qt);
        {
          const int sub = lane & 7;                      // columns 8 sub .. 8 sub + 7
          const uint4* vbase = reinterpret_cast<const uint4*>(p.Vb + (size_t)bh * p.L * kD) + sub;
          for (int rr = 0; rr < kTile; rr += 4 * kMathWarps) {
            const int r = rr + warp * 4 + (lane >> 3);     // the row this lane serves
            const int ir = i0 + r;
            if (ir < p.L) {
              const size_t rix = (size_t)bh * p.L + ir;
              if (part[7 * kTile + r] != 0.f) {
                const float tr = part[3 * kTile + r];
                const float tT = part[11 * kTile + r];
                float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
                float aco[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};   // O correction (o_final)
                float sgv = 0.f;
                int pe[kParts + 1];
                pe[0] = 0;
#pragma unroll
                for (int q = 0; q < kParts; ++q) pe[q + 1] = pe[q] + (int)part[(q * 4 + 2) * kTile + r];
                const int ntot = pe[kParts];
                for (int k0 = 0; k0 < ntot; k0 += 4) {   // four V rows in flight
                  float gk[4], ck[4];
                  uint4 vw[4];
#pragma unroll
                  for (int t = 0; t < 4; ++t) {
                    const int f = min(k0 + t, ntot - 1);
                    const int q = (f >= pe[1]) + (f >= pe[2]) + (f >= pe[3]);
                    const int e = (q * cap + (f - pe[q])) * kTile + r;
                    const float u = fmaf(cand[e], cz, -tr);
                    const float gu = AK == kAlpha15 ? u : (AK == kAlpha2 ? 1.f : pow_pos(fmaxf(u, 1e-30f), p.ae - 1.f));
                    gk[t] = (k0 + t < ntot && u > 0.f) ? gu : 0.f;
                    if constexpr (AK != kAlphaGen) {
                      // A* at the final tau minus the fp16 A_T the fused pass multiplied.
                      const float uT = fmaf(cand[e], cz, -tT);
                      const float aT = uT > 0.f ? round_f16(AK == kAlpha15 ? uT * uT : uT) : 0.f;
                      const float as = u > 0.f ? (AK == kAlpha15 ? u * u : u) : 0.f;
                      ck[t] = (o_final && k0 + t < ntot) ? as - aT : 0.f;
                    } else {
                      ck[t] = 0.f;
                    }
                    vw[t] = vbase[(size_t)cidx[e] * (kD / 8)];
                  }
#pragma unroll
                  for (int t = 0; t < 4; ++t) {
                    sgv += gk[t];
                    const uint32_t w4[4] = {vw[t].x, vw[t].y, vw[t].z, vw[t].w};
#pragma unroll
                    for (int c2 = 0; c2 < 4; ++c2) {   // bf16 pair -> two floats: shifts, exact
                      const float va = __uint_as_float(w4[c2] << 16), vb = __uint_as_float(w4[c2] & 0xffff0000u);
                      acc[2 * c2] = fmaf(gk[t], va, acc[2 * c2]);
                      acc[2 * c2 + 1] = fmaf(gk[t], vb, acc[2 * c2 + 1]);
                      aco[2 * c2] = fmaf(ck[t], va, aco[2 * c2]);
                      aco[2 * c2 + 1] = fmaf(ck[t], vb, aco[2 * c2 + 1]);
                    }
                  }
                }
                float4* dst = reinterpret_cast<float4*>(p.Ot + rix * kD + 8 * sub);
                dst[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
                dst[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
                if (sub == 0) p.sumg[rix] = sgv;
                if (o_final) {   // O = O_T + the correction (this row's O_T was written above)
                  float4* po = reinterpret_cast<float4*>(p.O + rix * kD + 8 * sub);
                  float4 x0 = po[0], x1 = po[1];
                  x0.x += aco[0]; x0.y += aco[1]; x0.z += aco[2]; x0.w += aco[3];
                  x1.x += aco[4]; x1.y += aco[5]; x1.z += aco[6]; x1.w += aco[7];
                  po[0] = x0;
                  po[1] = x1;
                }
              } else if (sub == 0) {
                p.sumg[rix] = -1.f;
              }
            }
          }
        }
        DIAG(dgx[3] += clock64() - de0);
        if (tid == 0) {
          int na = 0;
          for (int w = 0; w < kMaskWords; ++w) na += __popc(act[w]);
          const long long clk3 = clock64();
          int4* st = reinterpret_cast<int4*>(p.stats + ((size_t)bh * p.Tr + qt) * kFwdStats);
          st[0] = make_int4(sweeps - fused_passes, (int)n_s, n_out, na);
          st[1] = make_int4((int)(clk1 - clk0), (int)(clk2 - clk1), (int)(clk3 - clk2), (int)(clk3 - clk0));
          DIAG(st[2] = make_int4((int)dg_s1, (int)dg_s2, (int)dg_s3, (int)dg_solve));
          DIAG(st[4] = make_int4((int)dgr[0], (int)dgr[1], (int)dgr[2], (int)dgr[3]));
          DIAG(st[5] = make_int4((int)dgr[4], (int)dgr[5], (int)dgr[6], (int)dgr[7]));
          DIAG(st[6].x = (int)dgr[8]);
          DIAG(st[6].z = (int)dgx[0]; st[6].w = (int)dgx[1]; st[7].x = (int)dgx[2]; st[7].y = (int)dgx[3]; st[7].z = (int)dgx[4]; st[7].w = (int)dgx[5]);
        }
        break;
      }

      // Phase 3: one refinement sweep at the current tau. Every sweep collects this
      // thread's candidates u > 0: when tau <= tau* (f >= 0) they hold the whole support.
      // The first sweep runs at the tile-maxima bound tau_T <= tau*, so its candidates
      // hold the support by construction and it only collects them: one max over the
      // thread's 32 scores and a test against tau, with an element scan only when that
      // max passes (rare). Later sweeps (rows whose candidates overflowed, or Newton
      // steps) also accumulate S1, S2 and the count for f(tau) and f'(tau).
      // A row already solved keeps the copies (and count) of the sweep that solved it.
      const bool cand_only = sweeps == 0;
      const bool collect = !done;
      float S1 = 0.f, S2 = 0.f;
      if (collect) nc = 0;
      sbuf = 0;
      const float cthr = cand_threshold(tau, cz);   // the candidate-only sweep's threshold
      DIAG(const long long dsw0 = clock64());
      if (fuse) {
        // The fused first pass: output pass at tau_T with candidate collection.
        clk2 = clock64();
        tau_T = tau;
        int k = 0;
        const float thr = cand_threshold(tau, cz);
        for_each_bit(list, kMaskWords, [&](int jt) { out_tile(jt, obase + k++, thr, std::true_type{}, std::false_type{}); });
        // O of the last tile done: the epilogue reads O, and a later sweep reuses its columns.
        if (k > 0) warp_wait(&sh.pv_done[(obase + k - 1) % kOBufs], ((obase + k - 1) / kOBufs) & 1, wc);
        obase += k;
        ++fused_passes;
      } else for_each_bit(list, kMaskWords, [&](int jt) {
        const uint32_t bf = sbuf;
        DIAG(const long long d0 = clock64());
        warp_wait(&sh.s_full[bf], (sfull_par >> bf) & 1, wc);
        DIAG(const long long d1 = clock64(); dg_s2 += d1 - d0);
        sfull_par ^= 1u << bf;
        tc_fence_after();
        const int j0 = jt * kTile + qp * kCols;
        float s[kCols];
        ldc(tl + bf * 128 + qp * kCols, s);
        DIAG(const long long d2 = clock64(); dgr[3] += d2 - d1);
        tc_fence_before();
        warp_arrive(&sh.s_free[bf]);
        DIAG(dtk = clock64(); dgr[4] += dtk - d2);
        if constexpr (kAlibi) alibi_apply(s, cb, i, j0);
        if (!pat.block_full(i0, i1, jt * kTile, jt * kTile + kTile)) {
#pragma unroll
          for (int cc = 0; cc < kCols; ++cc)
            if (!pat.active(i, j0 + cc)) s[cc] = -INFINITY;
        }
        if (cand_only) {
          collect_tile(s, j0, collect, cthr);
          ++n_s;
          sbuf = (sbuf + 1) & (kSBufs - 1);
          DIAG(dgr[5] += clock64() - dtk);
          return;
        }
        float2 s1[4], s2[4];
#pragma unroll
        for (int a = 0; a < 4; ++a) {
          s1[a] = make_float2(0.f, 0.f);
          s2[a] = make_float2(0.f, 0.f);
        }
        // Groups of 8 scores: u+ summed per group (feeds S1), straight-line for all groups;
        // then only the groups with a positive sum (rare: a support candidate) are scanned
        // element by element. The run-time alpha variant sums g = u^{e-1} into S1 and
        // p = u^e into S2 instead.
        uint32_t gmask = 0;
#pragma unroll
        for (int g = 0; g < kCols / 8; ++g) {
          float2 v[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 u = __ffma2_rn(make_float2(s[8 * g + 2 * e], s[8 * g + 2 * e + 1]), make_float2(cz, cz),
                                        make_float2(-tau, -tau));
            v[e] = make_float2(fmaxf(u.x, 0.f), fmaxf(u.y, 0.f));
            if constexpr (AK == kAlphaGen) {
              float dummy_c = 0.f, dummy_m = INFINITY;
              accumulate<AK>(u.x, p.ae, s1[e].x, s2[e].x, dummy_c, dummy_m);
              accumulate<AK>(u.y, p.ae, s1[e].y, s2[e].y, dummy_c, dummy_m);
            } else {
              s2[e] = __ffma2_rn(v[e], v[e], s2[e]);
            }
          }
          const float2 gs = __fadd2_rn(__fadd2_rn(v[0], v[1]), __fadd2_rn(v[2], v[3]));
          if constexpr (AK != kAlphaGen) s1[g & 3] = __fadd2_rn(s1[g & 3], gs);
          gmask |= (gs.x + gs.y > 0.f ? 1u : 0u) << g;
        }
#pragma unroll
        for (int g = 0; g < kCols / 8; ++g)
          if (__any_sync(0xffffffffu, collect && ((gmask >> g) & 1u)))
            if (collect) collect8(s + 8 * g, j0 + 8 * g, cz, tau, cap, mycand, myidx, nc);
        const float2 s1t = __fadd2_rn(__fadd2_rn(s1[0], s1[1]), __fadd2_rn(s1[2], s1[3]));
        const float2 s2t = __fadd2_rn(__fadd2_rn(s2[0], s2[1]), __fadd2_rn(s2[2], s2[3]));
        S1 += s1t.x + s1t.y;
        S2 += s2t.x + s2t.y;
        ++n_s;
        sbuf = (sbuf + 1) & (kSBufs - 1);
      });
      DIAG(if (cand_only) dg_sw1 = clock64() - dsw0);
      DIAG(const long long dp0 = clock64());
      // Combine the column parts of each row.
      float* mp = part + qp * 4 * kTile + row;
      mp[0] = S1;
      mp[kTile] = S2;
      mp[2 * kTile] = (float)nc;
      named_bar(3, kMathThreads);
      S1 = 0.f;
      S2 = 0.f;
      int ncs[kParts];
      int ntot = 0;
      bool fits = true;
#pragma unroll
      for (int q = 0; q < kParts; ++q) {
        const float* pq = part + q * 4 * kTile + row;
        S1 += pq[0];
        S2 += pq[kTile];
        ncs[q] = (int)pq[2 * kTile];
        ntot += ncs[q];
        fits = fits && ncs[q] < cap;   // collect8 keeps the last slot free
      }
      const float C = (float)ntot;   // support size at tau (alpha = 2: |f'(tau)|)
      named_bar(3, kMathThreads);   // partials consumed before anyone rewrites them
      ++sweeps;
      DIAG(const long long dsv0 = clock64());
      if (cand_only) {
        // tau = tau_T <= tau*: if the copies fit they hold the support; solve on them.
        // Otherwise tau stays and the next sweep measures f(tau) and f'(tau). The solve
        // runs with four lanes of one warp per row (solve_quad), eight rows per warp:
        // the row's tau and bracket go through shared memory and the result comes back.
        if (qp == 0) {
          part[3 * kTile + row] = tau;
          part[7 * kTile + row] = lo;
          part[11 * kTile + row] = hi;
          part[15 * kTile + row] = (!done && fits) ? 1.f : 0.f;
        }
        named_bar(3, kMathThreads);
        {
          const int rq = warp * 8 + (lane >> 2), sub = lane & 3;
          const bool go = part[15 * kTile + rq] != 0.f;
          const int nq = (int)part[(sub * 4 + 2) * kTile + rq];
          float t;
          const bool ok = solve_quad<AK>(cand + sub * cap * kTile + rq, go ? nq : 0, kTile, go, cz, p.ae,
                                         part[3 * kTile + rq], part[7 * kTile + rq], part[11 * kTile + rq], t);
          named_bar(3, kMathThreads);   // every quad has read its row's inputs
          if (sub == 0) {
            part[3 * kTile + rq] = t;
            part[15 * kTile + rq] = ok ? 1.f : 0.f;
          }
        }
        named_bar(3, kMathThreads);
        if (!done && fits && part[15 * kTile + row] != 0.f) {
          tau = part[3 * kTile + row];
          done = true;
          listed = true;
        }
        DIAG(dg_solve += clock64() - dsv0);
      } else if (!done) {
        float f, fp;   // f(tau) and |f'(tau)|
        root_terms<AK>(S1, S2, C, p.ae, f, fp);
        if (f > 0.f) lo = fmaxf(lo, tau); else hi = fminf(hi, tau);
        if (f >= 0.f && fits) {
          // tau <= tau*, so every score of the support is in the candidate lists: the
          // exact solve on chip ends the refinement.
          float t;
          if (solve_list<AK>(cand + row, ncs, cap * kTile, kTile, cz, p.ae, tau, lo, hi, t)) {
            tau = t;
            done = true;
            listed = true;
          }
        }
        if (!done) {
          // f is a sum of C positive terms in fp32; its rounding error grows with C (and,
          // for the run-time alpha variant, with the approximate powers).
          const float tolf = AK == kAlphaGen ? fmaxf(4.f * kTolF, C * 0x1p-19f) : fmaxf(kTolF, C * 0x1p-22f);
          const bool narrow = AK == kAlphaGen && hi - lo <= fmaxf(fabsf(lo), 1.f) * 0x1p-22f;
          if (narrow) {   // bracket at fp32 resolution (see solve_list)
            tau = 0.5f * (lo + hi);
            done = true;
            listed = fits && f >= 0.f;
          } else if (fabsf(f) <= tolf && fp > 0.f && (fits || near_once)) {
            // Final Newton correction, no further sweep needed. The copies of this sweep
            // hold the support when they fit (tau moves by at most the tolerance over the
            // slope). When they do not, the row first sweeps once more at the corrected
            // tau, where fewer scores qualify; only a row whose support exceeds the copies
            // then ends without them.
            tau += f / fp;
            done = true;
            listed = fits;
          } else if (fabsf(f) <= tolf && fp > 0.f) {
            tau += f / fp;
            near_once = true;
          } else {
            float t = tau + f / fp;
            if (!(t > lo && t <= hi && t != tau)) t = 0.5f * (lo + hi);   // safeguard; the root may sit at hi
            tau = t;
          }
        }
      }
      DIAG(dgx[2] += clock64() - dp0);
    }
  }

  // No MMA may still write tensor memory when it is freed: each issuer commits once more
  // and waits for all three commits (a drain, bounded and independent of the abort flag).
  if ((warp == kMmaWarp || warp == kSWarp2 || warp == kOWarp) && lane == 0) {
    mma_commit(&sh.mma_drain);
    mbar_drain(&sh.mma_drain, 0, status);
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) tmem_dealloc(T, 512);
}

int fwd_smem_bytes(int Tc) { return 1024 + fwd_off_region() + fwd_region_bytes(Tc) + kParts * 4 * kTile * 4; }

cudaError_t launch_fwd(int alpha_kind, const FwdParams& p, int grid, cudaStream_t s) {
  const int smem = fwd_smem_bytes(p.Tc);
  // ALiBi and the 64 x 64 mask are compile-time variants, so calls without them carry none of
  // their code.
  const bool ab = p.alibi != nullptr, m64 = p.M64 != nullptr;
  using K = void (*)(FwdParams);
  auto pick = [&](K a00, K a01, K a10, K a11) { return ab ? (m64 ? a11 : a10) : (m64 ? a01 : a00); };
  const K kern = alpha_kind == kAlpha15 ? pick(fwd_kernel<kAlpha15, false, false>, fwd_kernel<kAlpha15, false, true>,
                                               fwd_kernel<kAlpha15, true, false>, fwd_kernel<kAlpha15, true, true>)
                 : alpha_kind == kAlpha2 ? pick(fwd_kernel<kAlpha2, false, false>, fwd_kernel<kAlpha2, false, true>,
                                                fwd_kernel<kAlpha2, true, false>, fwd_kernel<kAlpha2, true, true>)
                                         : pick(fwd_kernel<kAlphaGen, false, false>, fwd_kernel<kAlphaGen, false, true>,
                                                fwd_kernel<kAlphaGen, true, false>, fwd_kernel<kAlphaGen, true, true>);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  kern<<<grid, kThreads, smem, s>>>(p);
  return cudaGetLastError();
}

}  // namespace entmax
