/*
 * entmax_attn.h -- C ABI of the fused alpha-entmax attention library for NVIDIA B200
 * (sm_100a). The library is libentmax_attn.so.
 *
 * Operation (definitions from "AdaSplash-2: Faster Differentiable Sparse Attention"):
 *   - §2.2: scores s_ij = scale * q_i . k_j and output O = pi(S) V.
 *   - §2.3 Eq. 3: pi = alpha-entmax, p_ij = [(alpha-1) s_ij - tau_i]_+^{1/(alpha-1)}.
 *   - §2.4 Eq. 4: tau_i is the root of
 *     f(tau) = -1 + sum_j [(alpha-1) s_ij - tau]_+^{1/(alpha-1)}, inside the bracket
 *     m - 1 <= tau <= m - n^{1-alpha}, with m = (alpha-1) max_j s_ij.
 *   - §3.3 Phases 1-4: the forward takes a max pass, threshold refinement, a bit-packed
 *     block mask, and an output pass over the flagged blocks only. The same section's
 *     "Backward pass" reuses that mask.
 *   - Appendix C.4: mask packing, 32 key tiles per uint32.
 *   - "gpt2-adasplash-attention" model card, "Causal Splash Masking with Sink
 *     Preservation": window mask {0} U [max(1, i-W), i].
 *   - §4.3, NAPE heads: an optional ALiBi distance penalty per head (see alibi_slopes).
 * At alpha = 1.5 this equals the model cards' score-unit form
 * A_ij = max(0, (s_ij - tau'_i)/2)^2 with tau' = tau / (alpha-1).
 *
 * Backward: the Jacobian of Eq. 3 is dp_j/ds_k = g_j delta_jk - g_j g_k / sum_l g_l, with
 * g = p^{2-alpha}. The pages state only that gradients live on the support (§3.3); this
 * formula comes from implicit differentiation of sum_j p_j = 1. Hence
 *   dS_ij = g_ij (dO_i . V_j - delta_i),   delta_i = dO_i . Ot_i / sum_j g_ij,
 *   Ot_i  = sum_j g_ij V_j                (summed by the forward in fp32 over the support
 *                                          of each row, and kept in the workspace),
 *   dQ = scale dS K,  dK = scale dS^T Q,  dV = P^T dO.
 *
 * Conventions for every entry point:
 *   - Layout: Q, K, V, dO, O, dQ, dK, dV are contiguous row-major [B, H, L, d] (one
 *     64-element row per token); tau is [B, H, L]. All are device pointers.
 *   - Ownership: the caller allocates and frees all memory, the workspace included.
 *     The library never allocates or frees device memory. It keeps one piece of device
 *     memory and global state: the ENTMAX_NOALLOC_SCRATCH_BYTES scratch array of
 *     entmax_attn_fwd_noalloc, present on every GPU that loads the library until the
 *     process exits (with its device address, cached per device), plus a cached driver
 *     entry point.
 *   - Streams: `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream). All device work is enqueued on it. No call synchronises except
 *     entmax_last_device_status.
 *   - Errors: argument errors are found on the host before anything is launched, and
 *     are returned as ENTMAX_EINVAL or ENTMAX_EUNSUPPORTED. A failed launch returns
 *     ENTMAX_ECUDA. Conditions found on the device (solver cap reached, a bounded wait
 *     that expired) are recorded in the workspace status word and read back with
 *     entmax_last_device_status. Nothing throws across the ABI.
 *   - Bounded waits: every wait inside a kernel (pipeline barriers between the copy,
 *     tensor-core and row roles) gives up after desc->wait_limit_us (default 2 s). The
 *     CTA then issues no further copy or MMA, finishes its control flow, frees its
 *     tensor memory and records ENTMAX_ETIMEOUT; the results of that call are undefined,
 *     and the CUDA context stays usable.
 *   - Non-finite inputs give undefined results. The probability-side products (O = A V,
 *     Ot = g V, dV = A^T dO, dA = dO V^T) run in fp16, so bf16 V and dO must lie within
 *     the fp16 range (|x| <= 65504); a value outside it sets ENTMAX_ERANGE.
 */
#ifndef ENTMAX_ATTN_H
#define ENTMAX_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    ENTMAX_OK = 0,
    ENTMAX_EINVAL = 1,        /* bad pointer, size, stride or option                     */
    ENTMAX_EUNSUPPORTED = 2,  /* valid request that this build does not implement         */
    ENTMAX_ECUDA = 3,         /* a CUDA call or kernel launch failed                      */
    ENTMAX_ENOCONVERGE = 4,   /* device: a row hit the refinement cap (tau kept bracketed) */
    ENTMAX_ETIMEOUT = 5,      /* device: a bounded wait inside a kernel expired            */
    ENTMAX_ERANGE = 6         /* device: a bf16 V or dO value beyond fp16 range (|x|>65504) */
} entmax_status;

typedef enum { ENTMAX_BF16 = 0, ENTMAX_FP32 = 1 } entmax_dtype;

typedef struct {
    int B, H, L, d;       /* batch, heads, sequence length, head dim. d must be 64;
                             1 <= L <= ENTMAX_MAX_L.                                     */
    float alpha;          /* 1 < alpha <= 16 (alpha <= 1 or NaN -> ENTMAX_EINVAL, above 16
                             -> ENTMAX_EUNSUPPORTED). 1.5 and 2 use closed-form powers and
                             an exact on-chip solve; other alpha take u^{1/(alpha-1)} through
                             exp2/log2 and a safeguarded Newton solve (§3.2). With fp32 inputs
                             only 1.5 and 2 are supported. For alpha > 2 the backward's
                             g = p^{2-alpha} is unbounded as p -> 0 (a property of the
                             Jacobian), so gradients of keys at the support's edge are
                             ill-conditioned.                                             */
    float scale;          /* score scale, usually 1/sqrt(d); must be > 0                 */
    int causal;           /* 0: every key j < kv_len is active; 1: only keys j <= i      */
    int window;           /* < 0: no window. >= 0: active = {0} U [max(1, i-window), i];
                             this implies causal                                          */
    const int *kv_len;    /* device int32[B]: valid keys per sequence (1 <= kv_len <= L),
                             or NULL for all L. Every query row is computed, including
                             rows at or past kv_len.                                      */
    entmax_dtype dtype;   /* dtype of Q, K, V (and dO). ENTMAX_FP32 is forward-only.      */
    int max_sweeps;       /* cap on threshold-refinement passes; 0 = library default (12) */
    int wait_limit_us;    /* bound on each in-kernel wait in microseconds; 0 = 2 s.
                             Must be >= 0.                                                 */
    const float *alibi_slopes; /* device float[H] or NULL. ALiBi ("AdaSplash-2" §4.3: NAPE
                             heads; Press et al.): the score of key j for query i becomes
                             scale q_i . k_j - alibi_slopes[h] |i - j| (0 for a head without
                             it). bf16 inputs only (fp32 -> ENTMAX_EUNSUPPORTED).          */
    int selftest;         /* 0 for normal use. ENTMAX_SELFTEST_STALL makes one thread of
                             every CTA of the fwd/bwd kernels wait on a barrier that
                             nothing completes, so that the wait expires after
                             wait_limit_us and the call reports ENTMAX_ETIMEOUT: a test of
                             the failure path that faults and hangs nothing.              */
    int mask64;           /* 0 (default) or 1. With 1 the forward also builds the block mask at
                             64 x 64 blocks (entmax_attn_block_mask64) and the backward
                             leaves out the MMA steps of 64-row and 64-key halves of a
                             flagged tile that hold no nonzero weight. Both passes of a call
                             pair must use the same value. Separate kernel builds, so the
                             default path carries none of it.                              */
} entmax_attn_desc;

#define ENTMAX_SELFTEST_STALL 1

#define ENTMAX_MAX_L 16384   /* longest supported sequence (the per-row tile maxima live
                                in shared memory, 4 bytes per key tile per row)           */
#define ENTMAX_TILE 128      /* query and key tile edge; the block mask uses this size    */

/* Bytes of device workspace needed by entmax_attn_fwd / entmax_attn_bwd for *desc.
 * The workspace holds the status word, the block mask M and its transpose M^T, the
 * per-row sum_j g_ij and Ot_i = sum_j g_ij V_j, delta_i, per-tile counters of both
 * passes and fp16 copies of V and dO. Returns 0 for an invalid descriptor. The base
 * address must be 256-byte aligned; the fwd -> bwd pair must use the same workspace,
 * and the caller keeps it alive in between. */
size_t entmax_attn_workspace_bytes(const entmax_attn_desc *desc);

/* Forward (AdaSplash-2 §3.3 Phases 1-4).
 * In:  Q, K, V [B,H,L,d] in desc->dtype.
 * Out: O [B,H,L,d] fp32; tau [B,H,L] fp32 in Eq. 3 units; the workspace (block mask,
 *      its transpose, sum g, Ot, refinement counts, status).
 * The status word is cleared at the start of each forward. */
entmax_status entmax_attn_fwd(const entmax_attn_desc *desc, const void *Q, const void *K,
                              const void *V, float *O, float *tau, void *workspace, void *stream);

/* Backward over the blocks the forward flagged (§3.3 "Backward pass").
 * In:  Q, K, V, dO [B,H,L,d] (bf16); tau from the forward; the forward's workspace.
 * Out: dQ, dK, dV [B,H,L,d] fp32. The call overwrites them; dQ is zeroed on the stream
 *      and then accumulated.
 * The forward output O is not an input: delta needs Ot = sum g V, not O (see above). */
entmax_status entmax_attn_bwd(const entmax_attn_desc *desc, const void *Q, const void *K,
                              const void *V, const void *dO, const float *tau,
                              void *workspace, float *dQ, float *dK, float *dV, void *stream);

/* Row-wise alpha-entmax of explicit fp32 scores (AdaSplash-2 §2.3-2.4; the §4.1 solver
 * study works on such score vectors). Row r holds S[r*ld + j], j < n. Scores of -inf
 * are inactive; every row needs at least one finite score.
 * Out: P[r*ld + j] = [(alpha-1) S - tau_r]_+^{1/(alpha-1)} and tau[r] (Eq. 3 units).
 * status: a device int32 or NULL. When a row reaches the solver's iteration cap (its tau
 * then stays inside the §2.4 bracket) the kernel ORs 1 into it; the caller zeroes it
 * beforehand and reads it after the stream has finished.
 * Constraints: rows >= 0, 1 <= n <= ld, 16-byte-aligned S and P, ld % 4 == 0,
 * alpha in {1.5, 2}. rows == 0 is a no-op. */
entmax_status entmax_rows(const float *S, int rows, int n, int ld, float alpha, float *P,
                          float *tau, int *status, void *stream);

/* Synchronises `stream`, then reads the workspace status word left by the last
 * fwd/bwd: ENTMAX_OK, ENTMAX_ENOCONVERGE, ENTMAX_ETIMEOUT or ENTMAX_ERANGE. *status_out receives the
 * raw word: bit 0 = no convergence, bit 1 = wait timeout, bit 2 = a V or dO value outside
 * the fp16 range (ENTMAX_ERANGE; the results of that call are then undefined).
 * workspace == NULL reads the status word of entmax_attn_fwd_noalloc's scratch on the
 * current device instead (the last no-allocation forward on that device). */
entmax_status entmax_last_device_status(const entmax_attn_desc *desc, const void *workspace,
                                        int *status_out, void *stream);

/* Copies the forward's packed block mask and the per-tile counters of both passes out of
 * the workspace, device to device, on `stream`.
 *   - M is uint32 [B, H, Tr, ceil(Tc/32)], with Tr = Tc = ceil(L/128). Bit (jt % 32)
 *     of word jt/32 is set when some row of query tile it has a nonzero weight in key
 *     tile jt (Appendix C.4).
 *   - stats is int32 [B, H, Tr, 8]. Per query tile of the last forward: the refinement
 *     passes used, the S = Q K^T tiles computed (all passes), the flagged key tiles
 *     (the output pass), the structurally active key tiles; then SM clock cycles of the
 *     CTA in the max pass, in threshold refinement and the mask decision, in the output
 *     pass with its epilogue, and in total. (The fp32 forward leaves the cycles at 0.)
 *   - bwd_stats is int32 [B, H, Tc, 8]. Per key tile of the last backward: the flagged
 *     query tiles visited, the CTA's cycles in total, then the first row-owner warp's
 *     cycles waiting for S and dA, waiting for the previous tile's gradient MMAs,
 *     forming A and dS, staging dQ for its reduce-add, and the part of forming spent
 *     loading S and dA from tensor memory; one zero word.
 * Any output may be NULL. */
entmax_status entmax_attn_block_mask(const entmax_attn_desc *desc, const void *workspace,
                                     uint32_t *M, int *stats, int *bwd_stats, void *stream);

/* Copies the forward's block mask at 64 x 64 blocks ("AdaSplash-2", §4.2 and Fig. 7 measure
 * block sparsity at this unit) out of the workspace, device to device, on `stream`.
 * M64 is uint32 [B, H, 2*Tr, ceil(2*Tc/32)] (Tr = Tc = ceil(L/128)): bit (kb % 32) of word
 * kb/32 of row qb is set when some query row in [64 qb, 64 qb + 64) has a nonzero weight on
 * a key in [64 kb, 64 kb + 64). Blocks past L are 0. Like the 128 x 128 mask it is exact for
 * the fp32 scores at the final tau. Only a forward run with desc->mask64 = 1 builds it
 * (otherwise ENTMAX_EINVAL). The backward of such a call pair reads its transpose from the
 * workspace and leaves out the empty halves of flagged 128 x 128 tiles. */
entmax_status entmax_attn_block_mask64(const entmax_attn_desc *desc, const void *workspace, uint32_t *M64,
                                       void *stream);

/* Forward for callers that cannot allocate device memory. Some callers are handed
 * only their input and output buffers: a plugin inside a host framework that owns
 * every device allocation and gives the plugin no allocator, or a latency-critical
 * loop that must not call cudaMalloc after start-up (cudaMalloc can synchronise the
 * device). This call runs the same forward as entmax_attn_fwd, with the same arguments
 * minus the workspace. Its scratch is a fixed array of ENTMAX_NOALLOC_SCRATCH_BYTES
 * that the library keeps on every GPU that loads it, until the process exits.
 * The paper has no counterpart to this entry point; it exists for deployment only.
 *   - Limit: the forward's part of the workspace (status word, block masks, per-tile
 *     counters, and per row sum g, Ot and the fp16 copy of V: about 388 bytes per row)
 *     must fit in ENTMAX_NOALLOC_SCRATCH_BYTES (16 MiB, roughly B*H*L <= 43000 rows).
 *     A larger problem returns ENTMAX_EUNSUPPORTED before anything is launched.
 *   - Allocates nothing: no cudaMalloc, no cudaFree, no allocating library routine.
 *   - The first call on a device looks up the device address of the scratch array
 *     while that device is current. Make that first call before any stream capture.
 *   - All calls on a device share the one scratch array, and it keeps the last
 *     call's contents. Each call clears the parts that must start at zero. Calls whose
 *     GPU work overlaps (different streams, or host threads without ordering) race on
 *     the array and give undefined results, so serialise them.
 *   - Forward only: no workspace remains to pass to entmax_attn_bwd. The status word of
 *     the last call on a device (no convergence, wait timeout, fp16 range) is read with
 *     entmax_last_device_status(desc, NULL, &word, stream). */
#define ENTMAX_NOALLOC_SCRATCH_BYTES (16u << 20)
entmax_status entmax_attn_fwd_noalloc(const entmax_attn_desc *desc, const void *Q, const void *K,
                                      const void *V, float *O, float *tau, void *stream);

#ifdef __cplusplus
}
#endif
#endif /* ENTMAX_ATTN_H */
