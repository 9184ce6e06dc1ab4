// kernels.h -- kernel parameter blocks and launch helpers shared by the C ABI layer.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <cstdint>

namespace entmax {

// Per-query-tile counters written by the forward kernels (int32 each):
//   0 refinement sweeps, 1 S = Q K^T tiles computed (all passes), 2 flagged key tiles
//   (output pass), 3 structurally active key tiles, then SM clock cycles (clock64
//   differences) of 4 the max pass, 5 threshold refinement and mask decision, 6 the output
//   pass and epilogue, 7 the whole CTA.
#ifdef ENTMAX_DIAG
// Diagnostic builds append wait and step counters per query tile (see fwd.cu).
constexpr int kFwdStats = 32;
#else
constexpr int kFwdStats = 8;
#endif
// Per-key-tile counters of the backward kernel: 0 flagged query tiles visited, then cycles
// of 1 the whole CTA, and, for the first row-owner warp, 2 waiting for S and dA, 3 waiting
// for the previous tile's gradient MMAs, 4 forming A and dS, 5 staging dQ (reduce-add),
// 6 the part of 4 spent loading S and dA from tensor memory.
constexpr int kBwdStats = 8;
// Self-test switch: every CTA makes one bounded wait on an mbarrier that nothing
// completes, so the wait expires and the abort path runs.
constexpr int kSelftestStall = 1;

struct FwdParams {
  CUtensorMap tQ, tK, tV;   // [B*H][L][64], box 64 x 128 x 1, 128-byte swizzle (Q, K bf16; V fp16)
  float* O;                 // [B*H][L][64]
  float* tau;               // [B*H][L]
  float* sumg;              // [B*H][L]      sum_j g_ij over the support (-1: not listed, see fwd.cu)
  float* Ot;                // [B*H][L][64]  sum_j g_ij V_j
  const uint16_t* Vb;       // [B*H][L][64]  V as given (bf16)
  uint32_t* M;              // [B*H][Tr][Wc]
  uint32_t* MT;             // [B*H][Tc][Wr] (zeroed before the launch)
  uint32_t* M64;            // [B*H][2 Tr][W64c]: the mask at 64 x 64 blocks, or nullptr (not built)
  uint32_t* M64T;           // [B*H][2 Tc][W64r] (zeroed before the launch), or nullptr
  int* stats;               // [B*H][Tr][kFwdStats] (layout above)
  int* status;
  const int* kv_len;        // [B] or nullptr
  int H, L, Tr, Tc, Wc, Wr, BH;
  int W64c, W64r;           // words per row of M64 and of M64T
  float cz;                 // (alpha - 1) * scale
  float ae, am1;            // 1 / (alpha - 1) and alpha - 1 (the run-time alpha variant)
  const float* alibi;       // [H] ALiBi slopes (score units per position), or nullptr
  float inv_scale;          // 1 / scale (ALiBi slopes in raw score units)
  int causal, window, max_sweeps;
  unsigned long long wait_limit_ns;   // bound on every in-kernel wait
  int selftest;             // kSelftestStall: one wait per CTA on a barrier nothing completes
};

struct BwdParams {
  CUtensorMap tQ, tK, tV, tdO;   // [B*H][L][64]: Q, K bf16; V, dO fp16
  CUtensorMap tdQ;               // fp32 [B*H][L][64], box 32 x 128 x 1, 128-byte swizzle (reduce-add)
  const float* tau;              // [B*H][L]
  const float* delta;            // [B*H][L]
  const uint32_t* MT;            // [B*H][Tc][Wr]
  const uint32_t* M64T;          // [B*H][2 Tc][W64r]: the transposed mask at 64 x 64 blocks, or nullptr
  float* dQ;                     // [B*H][L][64] (zeroed, accumulated with atomics)
  float* dK;
  float* dV;
  int* status;
  int* stats;                    // [B*H][Tc][kBwdStats] (layout above)
  const int* kv_len;
  int H, L, Tr, Tc, Wr, BH;
  int W64r;
  float cz;                      // (alpha - 1) * scale
  float scale;
  float ae;                      // 1 / (alpha - 1)
  const float* alibi;            // [H] ALiBi slopes, or nullptr
  int causal, window;
  unsigned long long wait_limit_ns;
  int selftest;
};

// Inputs of the backward's delta kernel (bwd.cu).
struct DeltaParams {
  const uint16_t* Q;            // bf16 [B*H][L][64]
  const uint16_t* K;
  const uint16_t* V;
  const uint16_t* V16;          // fp16 copy of V (made by the forward)
  const uint16_t* dO;
  const float* tau;             // [B*H][L]
  const float* Ot;              // [B*H][L][64]
  const float* sumg;            // [B*H][L] (-1: the forward did not list the row's support)
  const uint32_t* M;            // [B*H][Tr][Wc]
  float* delta;                 // [B*H][L]
  const int* kv_len;
  int H, L, Tr, Wc, BH;
  float cz;
  float ae;                     // 1 / (alpha - 1)
  const float* alibi;           // [H] ALiBi slopes, or nullptr
  float scale;
  int causal, window;
};

struct FwdF32Params {
  const float* Q;           // fp32 [B*H][L][64]
  const float* K;
  const float* V;
  float* O;
  float* tau;
  uint32_t* M;
  uint32_t* MT;
  uint32_t* M64;            // as in FwdParams
  uint32_t* M64T;
  int* stats;               // [B*H][Tr][kFwdStats]
  int* status;
  const int* kv_len;
  int H, L, Tr, Tc, Wc, Wr, BH;
  int W64c, W64r;
  float cz;
  int causal, window, max_sweeps;
};

// Host-side launchers (each defined next to its kernel). They set the kernel's
// dynamic shared-memory limit and launch on `s`; they return the launch error.
int fwd_smem_bytes(int Tc);
int bwd_smem_bytes();
cudaError_t launch_fwd(int alpha_kind, const FwdParams& p, int grid, cudaStream_t s);
cudaError_t launch_fwd_f32(bool alpha15, const FwdF32Params& p, int grid, cudaStream_t s);
cudaError_t launch_bwd(int alpha_kind, const BwdParams& p, int grid, cudaStream_t s);
cudaError_t launch_bf16_to_f16(const void* src, void* dst, long elems, int* status, cudaStream_t s);
cudaError_t launch_delta(int alpha_kind, const DeltaParams& p, cudaStream_t s);
cudaError_t launch_rows(bool alpha15, const float* S, int rows, int n, long ld, float* P, float* tau, int* status,
                        cudaStream_t s);

// Device address of the no-allocation forward's static scratch on the current device
// (looked up on first use per device), or nullptr on failure.
void* noalloc_scratch();

}  // namespace entmax
