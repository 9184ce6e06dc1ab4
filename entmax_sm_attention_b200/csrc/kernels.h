// kernels.h -- kernel parameter blocks and launch helpers shared by the C ABI layer.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <cstdint>

namespace entmax {

struct FwdParams {
  CUtensorMap tQ, tK, tV;   // [B*H][L][64], box 64 x 128 x 1, 128-byte swizzle (Q, K bf16; V fp16)
  float* O;                 // [B*H][L][64]
  float* tau;               // [B*H][L]
  float* sumg;              // [B*H][L]      sum_j g_ij
  float* Ot;                // [B*H][L][64]  sum_j g_ij V_j
  uint32_t* M;              // [B*H][Tr][Wc]
  uint32_t* MT;             // [B*H][Tc][Wr] (zeroed before the launch)
  int* stats;               // [B*H][Tr][4]: sweeps, S tiles computed, flagged tiles, active tiles
  int* status;
  const int* kv_len;        // [B] or nullptr
  int H, L, Tr, Tc, Wc, Wr, BH;
  float cz;                 // (alpha - 1) * scale
  int causal, window, max_sweeps;
};

struct BwdParams {
  CUtensorMap tQ, tK, tV, tdO;   // [B*H][L][64]: Q, K bf16; V, dO fp16
  CUtensorMap tdQ;               // fp32 [B*H][L][64], box 32 x 128 x 1, 128-byte swizzle (reduce-add)
  const float* tau;              // [B*H][L]
  const float* delta;            // [B*H][L]
  const uint32_t* MT;            // [B*H][Tc][Wr]
  float* dQ;                     // [B*H][L][64] (zeroed, accumulated with atomics)
  float* dK;
  float* dV;
  int* status;
  const int* kv_len;
  int H, L, Tr, Tc, Wr, BH;
  float cz;                      // (alpha - 1) * scale
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
  int* stats;
  int* status;
  const int* kv_len;
  int H, L, Tr, Tc, Wc, Wr, BH;
  float cz;
  int causal, window, max_sweeps;
};

// Host-side launchers (each defined next to its kernel). They set the kernel's
// dynamic shared-memory limit and launch on `s`; they return the launch error.
int fwd_smem_bytes(int Tc);
int bwd_smem_bytes();
cudaError_t launch_fwd(bool alpha15, const FwdParams& p, int grid, cudaStream_t s);
cudaError_t launch_fwd_f32(bool alpha15, const FwdF32Params& p, int grid, cudaStream_t s);
cudaError_t launch_bwd(bool alpha15, const BwdParams& p, int grid, cudaStream_t s);
cudaError_t launch_bf16_to_f16(const void* src, void* dst, long elems, int* status, cudaStream_t s);
cudaError_t launch_delta(const uint16_t* dO, const float* Ot, const float* sumg, float* delta, long rows,
                         cudaStream_t s);
cudaError_t launch_rows(bool alpha15, const float* S, int rows, int n, long ld, float* P, float* tau,
                        cudaStream_t s);

}  // namespace entmax
