// fwd.cu -- fused alpha-entmax attention forward for sm_100a.
//
// One CTA per (batch*head, 128-row query tile) computes the four phases of
// "AdaSplash-2: Faster Differentiable Sparse Attention", §3.3:
//   Phase 1 (maximum): stream the structurally active key tiles; S = Q K^T on the
//     tensor cores (tcgen05, accumulator in TMEM). Each row keeps its running max and
//     its max in every key tile (kept in shared memory).
//   Initial threshold: the row's tau restricted to its key-tile maxima. Entmax on a
//     subset of the scores has a smaller threshold than on all of them (fewer
//     nonnegative terms in Eq. 4), so this is a lower bound on tau*. It plays the role
//     the paper gives its on-chip histogram (Phase 2): it costs no extra pass over K,
//     because the tile maxima come out of Phase 1.
//   Phase 3 (refinement): full sweeps over the key tiles that can still hold support
//     (tile max above the row's current tau). Per row they accumulate count, S1 =
//     sum u, S2 = sum u^2 with u = [z - tau]_+, then take a Newton step on Eq. 4,
//     safeguarded by the bracket of §2.4 with bisection when the step leaves it (§3.2
//     "safeguarded hybrid solver"). Eq. 4 is convex and decreasing for alpha <= 2, so
//     Newton from the left never overshoots. A row stops when |f(tau)| <= kTolF; then
//     one last Newton correction is applied without another sweep.
//   Block mask: bit (query tile, key tile) = some row has a key-tile max above its
//     final tau. Packed 32 key tiles per uint32 (Appendix C.4), plus the transpose
//     for the backward.
//   Phase 4 (output): only the flagged key tiles. Recompute S and form
//     A = u^{1/(alpha-1)} and g = u^{(2-alpha)/(alpha-1)}. Each is written to TMEM as a
//     two-term bf16 split (hi + lo); A goes over the S columns it replaces. Then the
//     tensor cores compute O += A V and Ot += g V, reading the A operand from TMEM.
//     The split keeps the products at about fp32 accuracy: a single bf16 term (2^-8
//     relative) would cost more than the gradient tolerance once it reaches dK through
//     delta. sum_j g_ij is kept per row for the backward.
//
// Roles: warps 0-3 own one query row per thread (TMEM lane = row); warp 4 issues the
// TMA loads (a 3-slot ring of 16 KB K/V tiles); warp 5 owns TMEM and issues the MMAs.
// TMEM (512 columns): [0,128) S tile, overwritten by A hi/lo; [128,256) g hi/lo;
// [256,320) O; [320,384) Ot. Per 32-key quarter q: hi at +32q, lo at +32q+16.
#include "common.cuh"
#include "kernels.h"

namespace entmax {

namespace {

constexpr int kThreads = 192;
constexpr int kSlots = 3;
constexpr float kTolF = 3e-5f;   // stop when |f(tau)| = |sum p - 1| <= kTolF
constexpr int kMaxVotes = 72;

constexpr int kKindSweep = 0;
constexpr int kKindOutput = 1;

struct Shared {
  uint64_t full[kSlots], empty[kSlots];
  uint64_t bar_q, s_full, s_free, pv_done;
  uint32_t tmem_base;
  int abort_flag;
  int ctl_kind, ctl_buf;
  uint32_t act[kMaskWords];          // structurally active key tiles
  uint32_t lists[2][kMaskWords];     // key tiles of the next sweep / the final mask
  int votes[kMaxVotes];
};

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// Load 64 consecutive fp32 TMEM columns of this thread's lane.
__device__ __forceinline__ void ld64(uint32_t taddr, float (&s)[64]) {
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

// tau on the key-tile maxima of one row (a lower bound of the row's tau*, see above):
// Newton on Eq. 4 from the bracket's left end, where f >= 0.
template <int AK>
__device__ float tau_on_tile_maxima(const float* tmax, const uint32_t (&act)[kMaskWords], int row, float cz,
                                    float lo) {
  float t = lo;
  for (int it = 0; it < 40; ++it) {
    float S1 = 0.f, S2 = 0.f, C = 0.f;
    for (int w = 0; w < kMaskWords; ++w) {
      uint32_t bits = act[w];
      while (bits) {
        int jt = w * 32 + __ffs(bits) - 1;
        bits &= bits - 1;
        float u = fmaf(tmax[jt * kTile + row], cz, -t);
        if (u > 0.f) {
          S1 += u;
          S2 = fmaf(u, u, S2);
          C += 1.f;
        }
      }
    }
    float f = (AK == kAlpha15) ? S2 - 1.f : S1 - 1.f;
    float fp = (AK == kAlpha15) ? 2.f * S1 : C;
    if (!(fp > 0.f)) break;
    float step = f / fp;
    t += step;
    if (fabsf(f) <= 1e-6f) break;
  }
  return t;
}

}  // namespace

template <int AK>
__global__ void __launch_bounds__(kThreads, 1) fwd_kernel(const __grid_constant__ FwdParams p) {
  extern __shared__ uint8_t dsm_raw[];
  __shared__ Shared sh;
  uint8_t* dsm = align1024(dsm_raw);
  uint8_t* sQ = dsm;
  uint8_t* ring = dsm + kTileBytes;
  float* tmax = reinterpret_cast<float*>(dsm + kTileBytes * (1 + kSlots));  // [Tc][128]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bh = blockIdx.x % p.BH;
  const int qt = p.Tr - 1 - blockIdx.x / p.BH;     // longest (causal) tiles first
  const int b = bh / p.H;
  const Pattern pat{p.L, p.kv_len ? min(max(p.kv_len[b], 1), p.L) : p.L, p.causal, p.window};
  const int i0 = qt * kTile, i1 = min(p.L, i0 + kTile);
  int* status = p.status;
  volatile int* abrt = &sh.abort_flag;

  if (tid == 0) {
    for (int s = 0; s < kSlots; ++s) {
      mbar_init(&sh.full[s], 1);
      mbar_init(&sh.empty[s], 1);
    }
    mbar_init(&sh.bar_q, 1);
    mbar_init(&sh.s_full, 1);
    mbar_init(&sh.s_free, 4);
    mbar_init(&sh.pv_done, 1);
    sh.abort_flag = 0;
    fence_mbar_init();
  }
  if (tid < kMaskWords) {
    sh.act[tid] = 0;
    sh.lists[0][tid] = 0;
    sh.lists[1][tid] = 0;
  }
  for (int v = tid; v < kMaxVotes; v += kThreads) sh.votes[v] = 0;
  if (warp == 5) {
    tmem_alloc(&sh.tmem_base, 512);
    tmem_relinquish();
  }
  __syncthreads();
  for (int jt = tid; jt < p.Tc; jt += kThreads)
    if (pat.block_active(i0, i1, jt * kTile, min(p.L, jt * kTile + kTile)))
      atomicOr(&sh.act[jt >> 5], 1u << (jt & 31));
  __syncthreads();
  tc_fence_after();
  const uint32_t T = sh.tmem_base;
  uint32_t act[kMaskWords];
#pragma unroll
  for (int w = 0; w < kMaskWords; ++w) act[w] = sh.act[w];

  if (warp == 4) {
    // ------------------------------------------------------------------ TMA producer
    uint32_t seq = 0;
    auto load = [&](const CUtensorMap* map, int jt) {
      const int slot = seq % kSlots;
      mbar_wait(&sh.empty[slot], ((seq / kSlots) & 1) ^ 1, status, abrt);
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
        } else {
          for_each_bit(list, kMaskWords, [&](int jt) {
            load(&p.tK, jt);
            load(&p.tV, jt);
          });
        }
      }
      __syncwarp();
      if (kind != kKindSweep) break;
    }
    // Make sure no copy is still in flight when the CTA retires.
    if (lane == 0) {
      for (uint32_t k = (seq > kSlots ? seq - kSlots : 0); k < seq; ++k) {
        volatile int no_abort = 0;
        mbar_wait(&sh.full[k % kSlots], (k / kSlots) & 1, status, &no_abort);
      }
    }
    __syncwarp();
  } else if (warp == 5) {
    // ------------------------------------------------------------------- MMA issuer
    uint32_t seq = 0, n_s = 0, n_pv = 0;
    const uint32_t idS = idesc_bf16(128, 128, 0, 0);
    const uint32_t idO = idesc_bf16(128, 64, 0, 1);
    const uint32_t sQa = smem_u32(sQ);
    auto issue_s = [&]() {
      const int slot = seq % kSlots;
      mbar_wait(&sh.full[slot], (seq / kSlots) & 1, status, abrt);
      if (n_s > 0) mbar_wait(&sh.s_free, (n_s - 1) & 1, status, abrt);
      if (n_pv > 0) mbar_wait(&sh.pv_done, (n_pv - 1) & 1, status, abrt);
      tc_fence_after();
      const uint32_t kb = smem_u32(ring + slot * kTileBytes);
#pragma unroll
      for (int k = 0; k < 4; ++k)
        mma_ss(T, sdesc_sw128(sQa + k * 32, 16, 1024), sdesc_sw128(kb + k * 32, 16, 1024), idS, k > 0);
      mma_commit(&sh.empty[slot]);
      mma_commit(&sh.s_full);
      ++n_s;
      ++seq;
    };
    if (lane == 0) {
      mbar_wait(&sh.bar_q, 0, status, abrt);
      for_each_bit(act, kMaskWords, [&](int) { issue_s(); });
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
          for_each_bit(list, kMaskWords, [&](int) { issue_s(); });
        } else {
          for_each_bit(list, kMaskWords, [&](int) {
            issue_s();
            const int slot = seq % kSlots;
            mbar_wait(&sh.full[slot], (seq / kSlots) & 1, status, abrt);
            mbar_wait(&sh.s_free, (n_s - 1) & 1, status, abrt);   // A and g written
            tc_fence_after();
            const uint32_t vb = smem_u32(ring + slot * kTileBytes);
#pragma unroll
            for (int t = 0; t < 8; ++t) {
              // key step t = quarter t/2, half t%2; hi at +0, lo at +16 within the quarter
              const uint32_t col = (t >> 1) * 32 + (t & 1) * 8;
              const uint64_t bd = sdesc_sw128(vb + t * 2048, 8192, 1024);
              const uint32_t acc = (n_pv > 0 || t > 0) ? 1u : 0u;
              mma_ts(T + 256, T + col, bd, idO, acc);
              mma_ts(T + 256, T + col + 16, bd, idO, 1u);
              mma_ts(T + 320, T + 128 + col, bd, idO, acc);
              if (AK == kAlpha15) mma_ts(T + 320, T + 128 + col + 16, bd, idO, 1u);
            }
            mma_commit(&sh.empty[slot]);
            mma_commit(&sh.pv_done);
            ++n_pv;
            ++seq;
          });
        }
      }
      __syncwarp();
      if (kind != kKindSweep) break;
    }
  } else {
    // ---------------------------------------------------------------- row owners
    const int row = tid;
    const int i = i0 + row;
    const bool valid = i < p.L;
    const uint32_t tl = T + ((uint32_t)(warp * 32) << 16);
    const float cz = p.cz;
    uint32_t n_s = 0;
    float m = -INFINITY;

    // Phase 1: row max and per-key-tile maxima.
    for_each_bit(act, kMaskWords, [&](int jt) {
      warp_wait(&sh.s_full, n_s & 1, status, abrt);
      tc_fence_after();
      const int j0 = jt * kTile;
      const bool full = pat.block_full(i0, i1, j0, j0 + kTile);
      float tm = -INFINITY;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        float s[64];
        ld64(tl + h * 64, s);
        if (full) {
#pragma unroll
          for (int c = 0; c < 64; ++c) tm = fmaxf(tm, s[c]);
        } else {
#pragma unroll
          for (int c = 0; c < 64; ++c)
            if (pat.active(i, j0 + h * 64 + c)) tm = fmaxf(tm, s[c]);
        }
      }
      tc_fence_before();
      warp_arrive(&sh.s_free);
      tmax[jt * kTile + row] = tm;
      m = fmaxf(m, tm);
      ++n_s;
    });

    // Bracket (§2.4) and the tile-maxima lower bound.
    const int n_act = valid ? pat.count(i) : 1;
    const float mz = m * cz;
    float lo = mz - 1.f;
    float hi = mz - ((AK == kAlpha15) ? rsqrtf((float)n_act) : 1.f / (float)n_act);
    float tau = valid ? tau_on_tile_maxima<AK>(tmax, act, row, cz, lo) : INFINITY;
    tau = fminf(fmaxf(tau, lo), hi);
    if (!valid) tau = INFINITY;
    bool done = !valid;
    float sg = 0.f;
    int sweeps = 0;

    // Decision points: publish either one more refinement sweep or the final mask.
    for (int r = 0;; ++r) {
      const int buf = r & 1;
      const bool need = !done && sweeps < p.max_sweeps;
      const bool final_mask = !rows_any(need, sh.votes, r, lane);
      // Tiles that some row still needs (refinement) or that hold a nonzero (mask).
      for_each_bit(act, kMaskWords, [&](int jt) {
        const bool take = final_mask ? valid : !done;
        const bool hit = take && fmaf(tmax[jt * kTile + row], cz, -tau) > 0.f;
        const uint32_t bal = __ballot_sync(0xffffffffu, hit);
        if (lane == 0 && bal) atomicOr(&sh.lists[buf][jt >> 5], 1u << (jt & 31));
      });
      named_bar(2, 128);
      if (tid == 0) {
        sh.ctl_kind = final_mask ? kKindOutput : kKindSweep;
        sh.ctl_buf = buf;
        // clear the other buffer for the next decision (nobody reads it any more)
        for (int w = 0; w < kMaskWords; ++w) sh.lists[buf ^ 1][w] = 0;
      }
      uint32_t list[kMaskWords];
#pragma unroll
      for (int w = 0; w < kMaskWords; ++w) list[w] = sh.lists[buf][w];
      named_bar(1, kThreads);

      if (final_mask) {
        if (!done) atomicOr(status, kStatusNoConverge);   // cap reached; tau stays bracketed
        // Block mask row of this query tile and the transposed bits (Appendix C.4).
        if (tid < p.Wc) p.M[((size_t)bh * p.Tr + qt) * p.Wc + tid] = list[tid];
        if (tid == 0) {
          for_each_bit(list, kMaskWords, [&](int jt) {
            atomicOr(&p.MT[((size_t)bh * p.Tc + jt) * p.Wr + (qt >> 5)], 1u << (qt & 31));
          });
        }
        // Phase 4: output sweep over the flagged tiles.
        int n_out = 0;
        for_each_bit(list, kMaskWords, [&](int jt) {
          warp_wait(&sh.s_full, n_s & 1, status, abrt);
          tc_fence_after();
          const int j0 = jt * kTile;
          const bool full = pat.block_full(i0, i1, j0, j0 + kTile);
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            float s[64];
            ld64(tl + h * 64, s);
            if (!full) {
#pragma unroll
              for (int c = 0; c < 64; ++c)
                if (!pat.active(i, j0 + h * 64 + c)) s[c] = -INFINITY;
            }
#pragma unroll
            for (int q = 0; q < 2; ++q) {
              uint32_t ah[16], al[16], gh[16], gl[16];
#pragma unroll
              for (int c = 0; c < 16; ++c) {
                const float u0 = fmaf(s[q * 32 + 2 * c], cz, -tau);
                const float u1 = fmaf(s[q * 32 + 2 * c + 1], cz, -tau);
                const float v0 = fmaxf(u0, 0.f), v1 = fmaxf(u1, 0.f);
                if (AK == kAlpha15) {
                  split_bf16x2(v0 * v0, v1 * v1, ah[c], al[c]);
                  split_bf16x2(v0, v1, gh[c], gl[c]);
                  sg += v0 + v1;
                } else {
                  const float g0 = u0 > 0.f ? 1.f : 0.f, g1 = u1 > 0.f ? 1.f : 0.f;
                  split_bf16x2(v0, v1, ah[c], al[c]);
                  gh[c] = pack_bf16(g0, g1);   // 0 and 1 are exact in bf16
                  sg += g0 + g1;
                }
              }
              const uint32_t col = h * 64 + q * 32;   // key quarter (2h + q)
              tmem_st16(tl + col, ah);
              tmem_st16(tl + col + 16, al);
              tmem_st16(tl + 128 + col, gh);
              if (AK == kAlpha15) tmem_st16(tl + 128 + col + 16, gl);
            }
          }
          tmem_wait_st();
          tc_fence_before();
          warp_arrive(&sh.s_free);
          ++n_s;
          ++n_out;
        });
        // Epilogue: O and Ot from TMEM.
        warp_wait(&sh.pv_done, (n_out - 1) & 1, status, abrt);
        tc_fence_after();
        float o[64];
        ld64(tl + 256, o);
        if (valid) {
          float4* dst = reinterpret_cast<float4*>(p.O + ((size_t)bh * p.L + i) * kD);
#pragma unroll
          for (int c = 0; c < 16; ++c) dst[c] = make_float4(o[4 * c], o[4 * c + 1], o[4 * c + 2], o[4 * c + 3]);
        }
        __syncwarp();
        ld64(tl + 320, o);
        if (valid) {
          float4* dst = reinterpret_cast<float4*>(p.Ot + ((size_t)bh * p.L + i) * kD);
#pragma unroll
          for (int c = 0; c < 16; ++c) dst[c] = make_float4(o[4 * c], o[4 * c + 1], o[4 * c + 2], o[4 * c + 3]);
          p.tau[(size_t)bh * p.L + i] = tau;
          p.sumg[(size_t)bh * p.L + i] = sg;
        }
        if (tid == 0) {
          int n_act = 0;
          for (int w = 0; w < kMaskWords; ++w) n_act += __popc(act[w]);
          int4* st = reinterpret_cast<int4*>(p.stats) + (size_t)bh * p.Tr + qt;
          *st = make_int4(sweeps, (int)n_s, n_out, n_act);
        }
        break;
      }

      // Phase 3: one refinement sweep.
      float S1 = 0.f, S2 = 0.f, C = 0.f;
      for_each_bit(list, kMaskWords, [&](int jt) {
        warp_wait(&sh.s_full, n_s & 1, status, abrt);
        tc_fence_after();
        const int j0 = jt * kTile;
        const bool full = pat.block_full(i0, i1, j0, j0 + kTile);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          float s[64];
          ld64(tl + h * 64, s);
          if (!full) {
#pragma unroll
            for (int c = 0; c < 64; ++c)
              if (!pat.active(i, j0 + h * 64 + c)) s[c] = -INFINITY;
          }
#pragma unroll
          for (int c = 0; c < 64; ++c) {
            const float u = fmaf(s[c], cz, -tau);
            const float v = fmaxf(u, 0.f);
            S1 += v;
            S2 = fmaf(v, v, S2);
            C += u > 0.f ? 1.f : 0.f;
          }
        }
        tc_fence_before();
        warp_arrive(&sh.s_free);
        ++n_s;
      });
      ++sweeps;
      if (!done) {
        const float f = (AK == kAlpha15) ? S2 - 1.f : S1 - 1.f;
        const float fp = (AK == kAlpha15) ? 2.f * S1 : C;   // |f'(tau)|
        if (fabsf(f) <= kTolF && fp > 0.f) {
          tau += f / fp;     // final Newton correction, no further sweep needed
          done = true;
        } else {
          if (f > 0.f) lo = tau; else hi = tau;
          float t = tau + f / fp;
          if (!(t > lo && t < hi)) t = 0.5f * (lo + hi);   // bisection safeguard
          tau = t;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) tmem_dealloc(T, 512);
}

// At least 120 KB, so that one CTA holds an SM: it allocates all 512 TMEM columns.
int fwd_smem_bytes(int Tc) {
  const int need = 1024 + kTileBytes * (1 + kSlots) + Tc * kTile * 4;
  return need > 120 * 1024 ? need : 120 * 1024;
}

cudaError_t launch_fwd(bool alpha15, const FwdParams& p, int grid, cudaStream_t s) {
  const int smem = fwd_smem_bytes(p.Tc);
  auto kern = alpha15 ? fwd_kernel<kAlpha15> : fwd_kernel<kAlpha2>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  kern<<<grid, kThreads, smem, s>>>(p);
  return cudaGetLastError();
}

}  // namespace entmax
