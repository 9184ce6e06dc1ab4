// bwd.cu -- fused alpha-entmax attention backward for sm_100a.
//
// "AdaSplash-2: Faster Differentiable Sparse Attention", §3.3 "Backward pass" and
// Appendix C.6: gradients are nonzero only on the entmax support, so the backward
// visits only the (query tile, key tile) blocks the forward flagged, through the
// transposed block mask. The Jacobian is not printed on the pages. From Eq. 3,
// implicit differentiation of sum_j p_j = 1 gives dp_j/ds_k = g_j delta_jk - g_j g_k /
// sum g, with g = p^{2-alpha}. Per element that yields
//   dS_ij = g_ij (dA_ij - delta_i),  dA_ij = dO_i . V_j,  delta_i = dO_i . Ot_i / sum_j g_ij
// and dQ = scale dS K, dK = scale dS^T Q, dV = A^T dO.
//
// One CTA per (batch*head, 128-key tile). K_j and V_j stay in shared memory; the
// flagged query tiles stream through a 2-stage ring of (Q_i, dO_i). Per query tile the
// tensor cores compute S = Q_i K_j^T and dA = dO_i V_j^T into TMEM (M = queries).
// Warps 0-15 are row owners: warp w reads TMEM lanes 32(w%4)..+31 (one query row per
// lane) and the columns of keys [32(w/4), 32(w/4)+32), so four threads share a row and
// four warps share each SM sub-partition, which hides the latency of forming A and dS.
// A warp reads its S and dA in two halves of 16 columns (fewer live registers) and
// releases them after the second, so the MMA warp computes S and dA of the next query
// tile while the row owners finish forming A and dS. Both go to swizzled shared-memory
// buffers: A in fp16 (with the fp16 copy of dO; 2^-11 rounding), dS as a two-term
// bf16 split (hi + lo, about fp32 accuracy in its products). A single 16-bit dS costs
// too much in dK at large query variance. Those buffers then feed dV += A^T dO_i and
// dK += dS^T Q_i as MN-major operands (M = keys, accumulated in TMEM), and
// dQ_i = dS K_j as a K-major operand (double-buffered in TMEM). dA = dO_i V_j^T uses the
// fp16 copies of dO and V (exact conversions of the bf16 inputs). The row owners copy
// dQ_i from TMEM into a swizzled fp32 staging tile in shared memory, and one thread adds
// it to global dQ with a TMA reduce-add (cp.reduce.async.bulk.tensor .add), one query
// tile behind the MMAs. Warp 16 issues the TMA loads. Warp 17 issues S, dA and the dQ chain,
// warp 18 the dV and dK chains: one thread issues an N=64 MMA only every ~54 cycles, so
// the 40 MMAs of a tile's gradient products are split between two issuers.
// TMEM: [0,128) S, [128,256) dA, [256,320) dV, [320,384) dK, [384,512) dQ x2.
// With the 64 x 64 mask (kM64) the MMA warps leave out the dQ steps of a 64-key half and
// the dV/dK steps of a 64-query half that hold no nonzero weight.
#include "common.cuh"
#include "kernels.h"

namespace entmax {

namespace {

constexpr int kMathWarps = 16;   // row owners: 4 per TMEM lane quadrant, 32 keys each
constexpr int kThreads = (kMathWarps + 3) * 32;
constexpr int kProducerWarp = kMathWarps;
constexpr int kMmaWarp = kMathWarps + 1;    // S, dA and the dQ chain
constexpr int kMma2Warp = kMathWarps + 2;   // the dV and dK chains
constexpr int kStages = 2;
constexpr int kPairBytes = 2 * kTileBytes;   // Q_i and dO_i

struct Shared {
  uint64_t full[kStages], empty[kStages];
  uint64_t bar_kv, s_full, sda_free, p_ready, mma2_done;
  uint64_t mma_drain;   // end of kernel: both issuers' MMAs complete
  uint64_t never;       // self-test: a barrier nothing completes
  uint32_t tmem_base;
  int abort_flag;
  uint32_t qlist[kMaskWords];
  uint32_t k64[2][2 * kMaskWords];   // rows 2 kt and 2 kt + 1 of the transposed 64 x 64 mask
  uint8_t quarters[32 * kMaskWords];   // per visited query tile: bit 2 qh + kh = quarter (qh, kh) nonzero
};

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}


}  // namespace

// dQ_s = dS K_j over key steps T0..T0+NT-1 (16 keys each; panel t/4): straight-line issue.
template <int T0, int NT>
__device__ __forceinline__ void dq_steps(uint32_t dq, uint64_t dHd, uint64_t dLd, uint64_t kM, uint32_t idQ) {
#pragma unroll
  for (int t = 0; t < NT; ++t) {
    constexpr int kTb = kTileBytes;
    const int tk = T0 + t;
    const uint32_t koff = (tk >> 2) * kTb + (tk & 3) * 32;
    const uint64_t bK = sdesc_add(kM, tk * 2048);
    mma_ss(dq, sdesc_add(dHd, koff), bK, idQ, t > 0 ? 1u : 0u);
    mma_ss(dq, sdesc_add(dLd, koff), bK, idQ, 1u);
  }
}

// dV += A^T dO_s and dK += dS^T Q_s over query steps T0..T0+NT-1 (16 queries each).
template <int T0, int NT>
__device__ __forceinline__ void dvk_steps(uint32_t T, uint64_t aM, uint64_t dHM, uint64_t dLM, uint64_t oM,
                                          uint64_t qM, uint32_t idV, uint32_t idK, bool started) {
#pragma unroll
  for (int tq = 0; tq < NT; ++tq) {
    const int t = T0 + tq;
    const uint32_t acc = (started || tq > 0) ? 1u : 0u;
    const uint64_t bO = sdesc_add(oM, t * 2048), bQ = sdesc_add(qM, t * 2048);
    mma_ss(T + 256, sdesc_add(aM, t * 2048), bO, idV, acc);
    mma_ss(T + 320, sdesc_add(dHM, t * 2048), bQ, idK, acc);
    mma_ss(T + 320, sdesc_add(dLM, t * 2048), bQ, idK, 1u);
  }
}

int bwd_smem_bytes() { return 1024 + 2 * kTileBytes + kStages * kPairBytes + 6 * kTileBytes + 2 * kTileBytes; }

template <int AK, bool kAlibi, bool kM64>
__global__ void __launch_bounds__(kThreads, 1) bwd_kernel(const __grid_constant__ BwdParams p) {
  extern __shared__ uint8_t dsm_raw[];
  __shared__ Shared sh;
  uint8_t* dsm = align1024(dsm_raw);
  uint8_t* sK = dsm;
  uint8_t* sV = dsm + kTileBytes;
  uint8_t* ring = dsm + 2 * kTileBytes;                       // stage s: Q at +0, dO at +16 KB
  // [128 q][128 k] 16-bit matrices, each as 2 swizzled panels of 64 keys: A (fp16),
  // dS hi, dS lo (bf16)
  uint8_t* sA = ring + kStages * kPairBytes;
  uint8_t* sdS = sA + 2 * kTileBytes;
  uint8_t* sdSl = sdS + 2 * kTileBytes;
  uint8_t* sStage = sdSl + 2 * kTileBytes;   // dQ tile: two [128][32] fp32 boxes, 128-byte swizzle

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bh = blockIdx.x % p.BH;
  const int kt = blockIdx.x / p.BH;          // key tile (low key tiles have the most query tiles)
  constexpr int kMathThreads = kMathWarps * 32;
  const int b = bh / p.H;
  const Pattern pat{p.L, p.kv_len ? min(max(p.kv_len[b], 1), p.L) : p.L, p.causal, p.window};
  const int j0 = kt * kTile;
  int* status = p.status;
  const WaitCtx wc{status, &sh.abort_flag, p.wait_limit_ns};

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sh.full[s], 1);
      mbar_init(&sh.empty[s], 2);   // one commit per MMA warp reading the stage
    }
    mbar_init(&sh.bar_kv, 1);
    mbar_init(&sh.s_full, 1);
    mbar_init(&sh.sda_free, kMathWarps);
    mbar_init(&sh.p_ready, kMathWarps);
    mbar_init(&sh.mma2_done, 2);  // dQ chain and dV/dK chains
    mbar_init(&sh.mma_drain, 2);
    mbar_init(&sh.never, 1);
    sh.abort_flag = 0;
    fence_mbar_init();
  }
  if (tid < kMaskWords) sh.qlist[tid] = (tid < p.Wr) ? p.MT[((size_t)bh * p.Tc + kt) * p.Wr + tid] : 0u;
  if (kM64 && tid >= 32 && tid < 32 + 4 * kMaskWords) {
    const int h = (tid - 32) / (2 * kMaskWords), w = (tid - 32) % (2 * kMaskWords);
    sh.k64[h][w] = w < p.W64r ? p.M64T[((size_t)bh * 2 * p.Tc + 2 * kt + h) * p.W64r + w] : 0u;
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&sh.tmem_base, 512);
    tmem_relinquish();
  }
  __syncthreads();
  // The 64 x 64 quarters of each visited query tile (query half qh, key half kh): the
  // thread of query tile it writes entry rank(it) = number of visited tiles before it.
  for (int it = tid; kM64 && it < p.Tr; it += kThreads) {
    const uint32_t wbits = sh.qlist[it >> 5];
    if ((wbits >> (it & 31)) & 1u) {
      int rank = __popc(wbits & ((1u << (it & 31)) - 1u));
      for (int w = 0; w < (it >> 5); ++w) rank += __popc(sh.qlist[w]);
      uint32_t q = 0;
#pragma unroll
      for (int qh = 0; qh < 2; ++qh)
#pragma unroll
        for (int kh = 0; kh < 2; ++kh) {
          const int qb = 2 * it + qh;
          q |= ((sh.k64[kh][qb >> 5] >> (qb & 31)) & 1u) << (2 * qh + kh);
        }
      sh.quarters[rank] = (uint8_t)q;
    }
  }
  __syncthreads();
  tc_fence_after();
  const long long clk0 = clock64();
  const uint32_t T = sh.tmem_base;
  uint32_t qlist[kMaskWords];
#pragma unroll
  for (int w = 0; w < kMaskWords; ++w) qlist[w] = sh.qlist[w];
  int nq = 0;
#pragma unroll
  for (int w = 0; w < kMaskWords; ++w) nq += __popc(qlist[w]);

  if (warp == kProducerWarp) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0 && nq > 0) {
      tma_prefetch_desc(&p.tQ);
      tma_prefetch_desc(&p.tdO);
      mbar_expect_tx(&sh.bar_kv, 2 * kTileBytes);
      tma_load_3d(sK, &p.tK, &sh.bar_kv, 0, j0, bh);
      tma_load_3d(sV, &p.tV, &sh.bar_kv, 0, j0, bh);
      // After a failed wait (abort) no further copy is issued: at most kStages copies,
      // one per stage, are in flight, and the drain below sees each stage's last one.
      uint32_t seq = 0;
      bool live = true;
      for_each_bit(qlist, kMaskWords, [&](int it) {
        const int st = seq % kStages;
        live = live && mbar_wait(&sh.empty[st], ((seq / kStages) & 1) ^ 1, wc);
        if (!live) return;
        mbar_expect_tx(&sh.full[st], kPairBytes);
        tma_load_3d(ring + st * kPairBytes, &p.tQ, &sh.full[st], 0, it * kTile, bh);
        tma_load_3d(ring + st * kPairBytes + kTileBytes, &p.tdO, &sh.full[st], 0, it * kTile, bh);
        ++seq;
      });
      mbar_drain(&sh.bar_kv, 0, status);
      for (uint32_t k = (seq > kStages ? seq - kStages : 0); k < seq; ++k)
        mbar_drain(&sh.full[k % kStages], (k / kStages) & 1, status);
    }
    __syncwarp();
  } else if (warp == kMmaWarp) {
    // -------------------------------------------- MMA issuer: S, dA and the dQ chain
    if (lane == 0 && nq > 0) {
      const uint32_t idS = idesc_bf16(128, 128, 0, 0);    // S = Q K^T
      const uint32_t idA = idesc_f16(128, 128, 0, 0);     // dA = dO V^T (fp16 copies)
      const uint32_t idQ = idesc_bf16(128, 64, 0, 1);     // dQ = dS K: A K-major (sdS), B MN-major (K_j)
      const uint64_t kK = sdesc_sw128(smem_u32(sK), 16, 1024), vK = sdesc_sw128(smem_u32(sV), 16, 1024);
      const uint64_t kM = sdesc_sw128(smem_u32(sK), 8192, 1024);    // K_j as MN-major B (dQ)
      const uint64_t rK = sdesc_sw128(smem_u32(ring), 16, 1024);    // ring stage 0, K-major
      const uint64_t dHd = sdesc_sw128(smem_u32(sdS), 16, 1024), dLd = sdesc_sw128(smem_u32(sdSl), 16, 1024);
      bool live = true;   // false after a failed wait: no further MMA is issued
      if (p.selftest & kSelftestStall) live = mbar_wait(&sh.never, 0, wc);   // expires: nothing completes it
      live = live && mbar_wait(&sh.bar_kv, 0, wc);
      // S = Q_s K^T and dA = dO_s V^T into TMEM [0,256).
      auto issue_sda = [&](int s) {
        const int st = s % kStages;
        const uint64_t qd = sdesc_add(rK, st * kPairBytes), od = sdesc_add(qd, kTileBytes);
        live = live && mbar_wait(&sh.full[st], (s / kStages) & 1, wc);
        if (s > 0) live = live && mbar_wait(&sh.sda_free, (s - 1) & 1, wc);   // S, dA of s-1 are in registers
        if (!live) return;
        tc_fence_after();
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          mma_ss(T, sdesc_add(qd, k * 32), sdesc_add(kK, k * 32), idS, k > 0);
          mma_ss(T + 128, sdesc_add(od, k * 32), sdesc_add(vK, k * 32), idA, k > 0);
        }
        mma_commit(&sh.s_full);
      };
      issue_sda(0);
      for (int s = 0; s < nq; ++s) {
        if (s + 1 < nq) issue_sda(s + 1);   // overlaps the row owners' work on tile s
        live = live && mbar_wait(&sh.p_ready, s & 1, wc);   // A and dS of tile s in shared memory
        if (!live) break;
        tc_fence_after();
        const uint32_t dq = T + 384 + (s & 1) * 64;
        // dQ_s = dS K_j: K = keys, M = queries. A key half with no nonzero weight in either
        // query half (64 x 64 mask) contributes nothing, so its four steps are left out; the
        // choice is made once per tile between straight-line sequences (a branch around each
        // MMA would slow the issue).
        const uint32_t qu = kM64 ? sh.quarters[s] : 15u;
        const uint32_t kl = (qu | (qu >> 2)) & 3u;   // bit kh: key half kh has a nonzero weight
        if (!kM64 || kl == 3u) dq_steps<0, 8>(dq, dHd, dLd, kM, idQ);
        else if (kl == 1u) dq_steps<0, 4>(dq, dHd, dLd, kM, idQ);
        else dq_steps<4, 4>(dq, dHd, dLd, kM, idQ);
        mma_commit(&sh.empty[s % kStages]);   // S and dA of tile s were this warp's last reads
        mma_commit(&sh.mma2_done);
      }
    }
    __syncwarp();
  } else if (warp == kMma2Warp) {
    // --------------------------------------------- second MMA issuer: dV and dK chains
    if (lane == 0 && nq > 0) {
      const uint32_t idV = idesc_f16(128, 64, 1, 1);      // dV += A^T dO: A MN-major (sA), B MN-major
      const uint32_t idK = idesc_bf16(128, 64, 1, 1);     // dK += dS^T Q: A MN-major (sdS), B MN-major
      const uint64_t aM = sdesc_sw128(smem_u32(sA), 16384, 1024);      // A, MN-major (dV)
      const uint64_t dHM = sdesc_sw128(smem_u32(sdS), 16384, 1024), dLM = sdesc_sw128(smem_u32(sdSl), 16384, 1024);
      const uint64_t rM = sdesc_sw128(smem_u32(ring), 8192, 1024);     // ring stage 0, MN-major
      bool started = false;   // the dV and dK accumulators hold a first product
      for (int s = 0; s < nq; ++s) {
        const int st = s % kStages;
        const uint64_t qM = sdesc_add(rM, st * kPairBytes), oM = sdesc_add(qM, kTileBytes);
        if (!mbar_wait(&sh.full[st], (s / kStages) & 1, wc)) break;   // Q_s and dO_s landed
        if (!mbar_wait(&sh.p_ready, s & 1, wc)) break;                // A and dS of tile s written
        tc_fence_after();
        // dV += A^T dO_s and dK += dS^T Q_s: K = queries, M = keys. A query half with no
        // nonzero weight in either key half contributes nothing (chosen once per tile).
        const uint32_t qu = kM64 ? sh.quarters[s] : 15u;
        const uint32_t ql = ((qu & 3u) ? 1u : 0u) | ((qu & 12u) ? 2u : 0u);   // bit qh: query half qh live
        if (!kM64 || ql == 3u) dvk_steps<0, 8>(T, aM, dHM, dLM, oM, qM, idV, idK, started);
        else if (ql == 1u) dvk_steps<0, 4>(T, aM, dHM, dLM, oM, qM, idV, idK, started);
        else dvk_steps<4, 4>(T, aM, dHM, dLM, oM, qM, idV, idK, started);
        started = true;
        mma_commit(&sh.empty[st]);
        mma_commit(&sh.mma2_done);
      }
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- row owners
    const int quad = warp & 3, qc = warp >> 2;   // TMEM lane quadrant, key quarter
    const int row = quad * 32 + lane;
    const uint32_t tl = T + ((uint32_t)(quad * 32) << 16);
    const float cz = p.cz;
    const float cb = kAlibi ? p.alibi[bh % p.H] / p.scale : 0.f;   // ALiBi, raw score units
    uint32_t seq = 0;
    int prev_it = -1;
    long long cyc_s = 0, cyc_mma = 0, cyc_form = 0, cyc_flush = 0, cyc_ld = 0;   // first row-owner warp's breakdown
    // Adds dQ of the query tile `it` handled at step `s` (TMEM buffer s % 2) to global
    // memory. The caller has already waited for that step's MMAs. Each thread stages its
    // 16 columns (scaled) in the swizzled box that holds them (one box per 32 of dQ's 64
    // columns); then thread 0 issues
    // one TMA reduce-add per box. The staging buffer is reused only after the previous
    // reduce-adds have read it.
    auto flush_dq = [&](uint32_t s, int it) {
      if (tid == 0) bulk_wait_read_all();
      named_bar(1, kMathThreads);
      tc_fence_after();
      uint32_t a[16];
      tmem_ld16(tl + 384 + (s & 1) * 64 + qc * 16, a);
      tmem_wait_ld();
      uint8_t* box = sStage + (qc >> 1) * kTileBytes + row * 128;
      const float sc = p.scale;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int ch = (qc & 1) * 4 + c;
        *reinterpret_cast<float4*>(box + ((ch ^ (row & 7)) << 4)) =
            make_float4(sc * __uint_as_float(a[4 * c]), sc * __uint_as_float(a[4 * c + 1]),
                        sc * __uint_as_float(a[4 * c + 2]), sc * __uint_as_float(a[4 * c + 3]));
      }
      fence_proxy_async_smem();
      named_bar(1, kMathThreads);
      if (tid == 0) {
        tma_reduce_add_3d(&p.tdQ, sStage, 0, it * kTile, bh);
        tma_reduce_add_3d(&p.tdQ, sStage + kTileBytes, 32, it * kTile, bh);
        bulk_commit();
      }
    };
    for_each_bit(qlist, kMaskWords, [&](int it) {
      const int i = it * kTile + row;
      const bool valid = i < p.L;
      const float tau = valid ? p.tau[(size_t)bh * p.L + i] : INFINITY;
      const float dl = valid ? p.delta[(size_t)bh * p.L + i] : 0.f;
      const bool full = pat.block_full(it * kTile, min(p.L, it * kTile + kTile), j0, j0 + kTile);
      const long long c0 = clock64();
      warp_wait(&sh.s_full, seq & 1, wc);
      const long long c1 = clock64();
      tc_fence_after();
      // Keys [32 qc, 32 qc + 32) of row `row`: panel qc/2, 16-byte chunks 4(qc%2)..+3.
      const int pan = (qc >> 1) * kTileBytes;
      // S and dA are read in two halves of 16 columns, so only 32 of them are live at a
      // time; the second half's read releases the TMEM columns (sda_free) for the next tile.
      uint32_t sr[16], ar[16];
      auto form_half = [&](int hf) {
#pragma unroll
        for (int ch = 0; ch < 2; ++ch) {
          const int cc = 2 * hf + ch;
          uint32_t ah[4], dh[4], dl2[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int c = ch * 8 + 2 * e;         // column within the half
            const int cq = hf * 16 + c;           // column within the thread's 32 keys
            float s0 = __uint_as_float(sr[c]), s1 = __uint_as_float(sr[c + 1]);
            if constexpr (kAlibi) {   // ALiBi: -cb |i - j| on the raw scores
              const float dj = (float)(i - (j0 + qc * 32 + cq));
              s0 = fmaf(-cb, fabsf(dj), s0);
              s1 = fmaf(-cb, fabsf(dj - 1.f), s1);
            }
            if (!full) {
              const int jj = j0 + qc * 32 + cq;
              if (!pat.active(i, jj)) s0 = -INFINITY;
              if (!pat.active(i, jj + 1)) s1 = -INFINITY;
            }
            const float2 u = __ffma2_rn(make_float2(s0, s1), make_float2(cz, cz), make_float2(-tau, -tau));
            const float v0 = fmaxf(u.x, 0.f), v1 = fmaxf(u.y, 0.f);
            const float2 d = __fadd2_rn(make_float2(__uint_as_float(ar[c]), __uint_as_float(ar[c + 1])),
                                        make_float2(-dl, -dl));
            if constexpr (AK == kAlpha15) {
              const float2 a = __fmul2_rn(make_float2(v0, v1), make_float2(v0, v1));
              const float2 ds = __fmul2_rn(make_float2(v0, v1), d);
              ah[e] = pack_f16(a.x, a.y);
              split_bf16x2(ds.x, ds.y, dh[e], dl2[e]);
            } else if constexpr (AK == kAlpha2) {
              ah[e] = pack_f16(v0, v1);
              split_bf16x2(u.x > 0.f ? d.x : 0.f, u.y > 0.f ? d.y : 0.f, dh[e], dl2[e]);
            } else {
              // g = u^{e-1} from one logarithm and one power, and A = u^e = g u (two
              // special-function operations per score instead of three).
              const float l0 = __log2f(u.x > 0.f ? u.x : 1.f), l1 = __log2f(u.y > 0.f ? u.y : 1.f);
              const float g0 = u.x > 0.f ? exp2f((p.ae - 1.f) * l0) : 0.f;
              const float g1 = u.y > 0.f ? exp2f((p.ae - 1.f) * l1) : 0.f;
              const float a0 = g0 * v0, a1 = g1 * v1;
              ah[e] = pack_f16(a0, a1);
              split_bf16x2(g0 * d.x, g1 * d.y, dh[e], dl2[e]);
            }
          }
          const uint32_t off = pan + sw128_offset(row, ((qc & 1) * 4 + cc) * 8);
          *reinterpret_cast<uint4*>(sA + off) = make_uint4(ah[0], ah[1], ah[2], ah[3]);
          *reinterpret_cast<uint4*>(sdS + off) = make_uint4(dh[0], dh[1], dh[2], dh[3]);
          *reinterpret_cast<uint4*>(sdSl + off) = make_uint4(dl2[0], dl2[1], dl2[2], dl2[3]);
        }
      };
      tmem_ld16(tl + qc * 32, sr);
      tmem_ld16(tl + 128 + qc * 32, ar);
      tmem_wait_ld();
      const long long c1b = clock64();
      // The previous tile's dV/dK/dQ MMAs must be done reading sA / sdS.
      const long long c2 = clock64();
      if (seq > 0) warp_wait(&sh.mma2_done, (seq - 1) & 1, wc);
      const long long c3 = clock64();
      // In a 64 x 64 quarter without a nonzero weight every u <= 0, so A and dS come out
      // zero there; the MMA issuers leave out the steps of empty halves.
      form_half(0);
      tmem_ld16(tl + qc * 32 + 16, sr);
      tmem_ld16(tl + 128 + qc * 32 + 16, ar);
      tmem_wait_ld();
      tc_fence_before();
      warp_arrive(&sh.sda_free);
      form_half(1);
      fence_proxy_async_smem();
      warp_arrive(&sh.p_ready);
      const long long c4 = clock64();
      if (seq > 0) flush_dq(seq - 1, prev_it);   // its MMAs were waited for above
      const long long c5 = clock64();
      cyc_s += c1 - c0;
      cyc_mma += c3 - c2;
      cyc_form += (c2 - c1) + (c4 - c3);
      cyc_ld += c1b - c1;
      cyc_flush += c5 - c4;
      prev_it = it;
      ++seq;
    });
    if (seq > 0) {
      const long long c0 = clock64();
      warp_wait(&sh.mma2_done, (seq - 1) & 1, wc);
      const long long c1 = clock64();
      flush_dq(seq - 1, prev_it);
      cyc_mma += c1 - c0;
      cyc_flush += clock64() - c1;
    }
    if (tid == 0) bulk_wait_all();   // the last reduce-adds complete before the CTA retires
    // dK and dV of this key tile (TMEM lane = key); each thread writes 16 of the 64
    // columns of each. Every lane executes the TMEM loads (.sync.aligned); only the global
    // stores depend on the key being inside L.
    const int j = j0 + row;
    const bool jvalid = j < p.L;
    float* dk = p.dK + ((size_t)bh * p.L + (jvalid ? j : 0)) * kD + qc * 16;
    float* dv = p.dV + ((size_t)bh * p.L + (jvalid ? j : 0)) * kD + qc * 16;
    const float sc = p.scale;
    uint32_t a[16], c[16];
    if (seq > 0) {
      tc_fence_after();
      tmem_ld16(tl + 256 + qc * 16, a);
      tmem_ld16(tl + 320 + qc * 16, c);
      tmem_wait_ld();
    } else {
#pragma unroll
      for (int k = 0; k < 16; ++k) a[k] = c[k] = 0u;
    }
    if (jvalid) {
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        reinterpret_cast<float4*>(dv)[k] = make_float4(__uint_as_float(a[4 * k]), __uint_as_float(a[4 * k + 1]),
                                                       __uint_as_float(a[4 * k + 2]), __uint_as_float(a[4 * k + 3]));
        reinterpret_cast<float4*>(dk)[k] =
            make_float4(sc * __uint_as_float(c[4 * k]), sc * __uint_as_float(c[4 * k + 1]),
                        sc * __uint_as_float(c[4 * k + 2]), sc * __uint_as_float(c[4 * k + 3]));
      }
    }
    if (tid == 0) {
      int4* st = reinterpret_cast<int4*>(p.stats + ((size_t)bh * p.Tc + kt) * kBwdStats);
      st[0] = make_int4(nq, (int)(clock64() - clk0), (int)cyc_s, (int)cyc_mma);
      st[1] = make_int4((int)cyc_form, (int)cyc_flush, (int)cyc_ld, 0);
    }
    __syncwarp();
  }

  // No MMA may still write tensor memory when it is freed: both issuers commit once more
  // and wait for both commits (a drain, bounded and independent of the abort flag).
  if ((warp == kMmaWarp || warp == kMma2Warp) && lane == 0) {
    mma_commit(&sh.mma_drain);
    mbar_drain(&sh.mma_drain, 0, status);
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) tmem_dealloc(T, 512);
}

cudaError_t launch_bwd(int alpha_kind, const BwdParams& p, int grid, cudaStream_t s) {
  const int smem = bwd_smem_bytes();
  // ALiBi and the 64 x 64 skipping are compile-time variants, as in the forward.
  const bool ab = p.alibi != nullptr, m64 = p.M64T != nullptr;
  using K = void (*)(BwdParams);
  auto pick = [&](K a00, K a01, K a10, K a11) { return ab ? (m64 ? a11 : a10) : (m64 ? a01 : a00); };
  const K kern = alpha_kind == kAlpha15 ? pick(bwd_kernel<kAlpha15, false, false>, bwd_kernel<kAlpha15, false, true>,
                                               bwd_kernel<kAlpha15, true, false>, bwd_kernel<kAlpha15, true, true>)
                 : alpha_kind == kAlpha2 ? pick(bwd_kernel<kAlpha2, false, false>, bwd_kernel<kAlpha2, false, true>,
                                                bwd_kernel<kAlpha2, true, false>, bwd_kernel<kAlpha2, true, true>)
                                         : pick(bwd_kernel<kAlphaGen, false, false>, bwd_kernel<kAlphaGen, false, true>,
                                                bwd_kernel<kAlphaGen, true, false>, bwd_kernel<kAlphaGen, true, true>);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  kern<<<grid, kThreads, smem, s>>>(p);
  return cudaGetLastError();
}

// delta_i = sum_j g_ij dA_ij / sum_j g_ij = dO_i . Ot_i / sum_j g_ij, with dA_ij = dO_i . V_j,
// g = u^{(2-alpha)/(alpha-1)} and u = (alpha-1) scale q_i . k_j - tau_i > 0 (the support).
// The forward sums Ot_i = sum_j g_ij V_j and sum_j g_ij exactly (fp32) over each row's
// support; one lane per row forms the dot here. A row whose support the forward could not
// list (sum g = -1: the refinement cap, or a Newton finish on near-uniform rows) is served
// by its whole warp afterwards: the lanes take the keys of the row's flagged key tiles,
// recompute u from q_i . k_j in fp32 (exact bf16 products) and sum g dO_i . V_j.
namespace {
constexpr int kDeltaWarps = 4;

__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }
__device__ __forceinline__ float2 f16x2(uint32_t w) {
  float lo, hi;
  asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %2;\n\tcvt.f32.f16 %0, l;\n\tcvt.f32.f16 %1, h;\n\t}"
      : "=f"(lo), "=f"(hi)
      : "r"(w));
  return make_float2(lo, hi);
}

// dot of a bf16 (is_f16 = false) or fp16 row with 64 floats in shared memory (broadcast
// reads: every lane reads the same x).
__device__ __forceinline__ float dot_s(const uint4* __restrict__ row, const float* x, bool is_f16) {
  float a0 = 0.f, a1 = 0.f;
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const uint4 w = row[k];
    const uint32_t w4[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = is_f16 ? f16x2(w4[e]) : make_float2(bf16lo(w4[e]), bf16hi(w4[e]));
      a0 = fmaf(f.x, x[8 * k + 2 * e], a0);
      a1 = fmaf(f.y, x[8 * k + 2 * e + 1], a1);
    }
  }
  return a0 + a1;
}
}  // namespace

template <int AK>
__global__ void __launch_bounds__(32 * kDeltaWarps, 4) bwd_delta_kernel(const __grid_constant__ DeltaParams p) {
  __shared__ float xs[kDeltaWarps][2][kD];   // brute-force path: q_i and dO_i of the row served
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long rows = (long)p.BH * p.L;
  const long r0 = ((long)blockIdx.x * kDeltaWarps + warp) * 32;
  if (r0 >= rows) return;
  const long r = r0 + lane;
  const bool valid = r < rows;
  const long rc = valid ? r : r0;
  const float sgf = p.sumg[rc];
  const bool listed = sgf >= 0.f;
  float delta = 0.f;
  if (valid && listed) {
    const uint4* dr = reinterpret_cast<const uint4*>(p.dO + rc * kD);
    const float4* orow = reinterpret_cast<const float4*>(p.Ot + rc * kD);
    float a0 = 0.f, a1 = 0.f;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const uint4 w = dr[k];
      const float4 o0 = orow[2 * k], o1 = orow[2 * k + 1];
      a0 = fmaf(bf16lo(w.x), o0.x, a0);
      a1 = fmaf(bf16hi(w.x), o0.y, a1);
      a0 = fmaf(bf16lo(w.y), o0.z, a0);
      a1 = fmaf(bf16hi(w.y), o0.w, a1);
      a0 = fmaf(bf16lo(w.z), o1.x, a0);
      a1 = fmaf(bf16hi(w.z), o1.y, a1);
      a0 = fmaf(bf16lo(w.w), o1.z, a0);
      a1 = fmaf(bf16hi(w.w), o1.w, a1);
    }
    delta = (a0 + a1) / sgf;
  }
  uint32_t ovf = __ballot_sync(0xffffffffu, valid && !listed);
  while (ovf) {
    const int ol = __ffs(ovf) - 1;
    ovf &= ovf - 1;
    const long ro = r0 + ol;
    const int i = (int)(ro % p.L), bho = (int)(ro / p.L);   // the warp's rows may span two heads
    __syncwarp();
    {
      const uint32_t qw = reinterpret_cast<const uint32_t*>(p.Q + ro * kD)[lane];
      const uint32_t dw = reinterpret_cast<const uint32_t*>(p.dO + ro * kD)[lane];
      xs[warp][0][2 * lane] = bf16lo(qw);
      xs[warp][0][2 * lane + 1] = bf16hi(qw);
      xs[warp][1][2 * lane] = bf16lo(dw);
      xs[warp][1][2 * lane + 1] = bf16hi(dw);
    }
    __syncwarp();
    const float to = p.tau[ro];
    const float cbo = p.alibi ? p.alibi[bho % p.H] / p.scale : 0.f;   // ALiBi of the row's head
    const uint4* Ko = reinterpret_cast<const uint4*>(p.K + (size_t)bho * p.L * kD);
    const uint4* Vo = reinterpret_cast<const uint4*>(p.V16 + (size_t)bho * p.L * kD);
    const int b = bho / p.H;
    const Pattern pat{p.L, p.kv_len ? min(max(p.kv_len[b], 1), p.L) : p.L, p.causal, p.window};
    const uint32_t* words = p.M + ((size_t)bho * p.Tr + i / kTile) * p.Wc;
    float og = 0.f, ogd = 0.f;
    for (int w = 0; w < p.Wc; ++w) {
      uint32_t bits = words[w];
      while (bits) {
        const int jt = w * 32 + __ffs(bits) - 1;
        bits &= bits - 1;
#pragma unroll
        for (int jj = lane; jj < kTile; jj += 32) {   // four keys per lane, loads in flight together
          const int jk = jt * kTile + jj;
          if (jk < p.L && pat.active(i, jk)) {
            const float sraw = dot_s(Ko + (size_t)jk * 8, xs[warp][0], false) - cbo * fabsf((float)(i - jk));
            const float uu = fmaf(sraw, p.cz, -to);
            if (uu > 0.f) {
              const float g = (AK == kAlpha15) ? uu : (AK == kAlpha2 ? 1.f : pow_pos(uu, p.ae - 1.f));
              og += g;
              ogd = fmaf(g, dot_s(Vo + (size_t)jk * 8, xs[warp][1], true), ogd);
            }
          }
        }
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      og += __shfl_xor_sync(0xffffffffu, og, o);
      ogd += __shfl_xor_sync(0xffffffffu, ogd, o);
    }
    if (lane == ol) delta = ogd / og;
  }
  if (valid) p.delta[r] = delta;
}

cudaError_t launch_delta(int alpha_kind, const DeltaParams& p, cudaStream_t s) {
  const long rows = (long)p.BH * p.L;
  const long per_block = (long)kDeltaWarps * 32;
  const unsigned grid = (unsigned)((rows + per_block - 1) / per_block);
  if (alpha_kind == kAlpha15)
    bwd_delta_kernel<kAlpha15><<<grid, 32 * kDeltaWarps, 0, s>>>(p);
  else if (alpha_kind == kAlpha2)
    bwd_delta_kernel<kAlpha2><<<grid, 32 * kDeltaWarps, 0, s>>>(p);
  else
    bwd_delta_kernel<kAlphaGen><<<grid, 32 * kDeltaWarps, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace entmax
