// convert.cu -- fp16 copies of bf16 operands for the probability-side products.
//
// A = p and g are formed in fp16 (2^-11 relative rounding; bf16 would give 2^-8, which
// shows up in O and, through delta, in dK at the size of the gradient tolerance). The
// tensor cores need both factors in the same type, so V (for O = A V, Ot = g V) and dO
// (for dV = A^T dO, dA = dO V^T) get fp16 copies. A bf16 value converts to fp16
// exactly when 2^-14 <= |x| <= 65504 (or x = 0). Only the overflow side is flagged:
// |x| > 65504 sets the status bit kStatusRange. Below 2^-14 the value lands on fp16's
// subnormal grid (spacing 2^-24) and below 2^-25 it rounds to zero; either way the
// absolute error is at most 2^-25, far inside the output and gradient tolerances, so it
// is not reported.
#include "common.cuh"
#include "kernels.h"

namespace entmax {

__global__ void bf16_to_f16_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst, long n8, int* status) {
  bool bad = false;
  for (long k = (long)blockIdx.x * blockDim.x + threadIdx.x; k < n8; k += (long)gridDim.x * blockDim.x) {
    const uint4 w = src[k];
    const uint32_t in[4] = {w.x, w.y, w.z, w.w};
    uint32_t out[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float lo = __uint_as_float(in[e] << 16), hi = __uint_as_float(in[e] & 0xffff0000u);
      bad |= fabsf(lo) > 65504.f || fabsf(hi) > 65504.f;
      out[e] = pack_f16(lo, hi);
    }
    dst[k] = make_uint4(out[0], out[1], out[2], out[3]);
  }
  if (__any_sync(0xffffffffu, bad) && (threadIdx.x & 31) == 0) atomicOr(status, kStatusRange);
}

cudaError_t launch_bf16_to_f16(const void* src, void* dst, long elems, int* status, cudaStream_t s) {
  const long n8 = elems / 8;   // rows of 64 elements: always a multiple of 8
  long blocks = (n8 + 255) / 256;
  if (blocks > 148 * 16) blocks = 148 * 16;
  if (blocks < 1) blocks = 1;
  bf16_to_f16_kernel<<<(unsigned)blocks, 256, 0, s>>>(static_cast<const uint4*>(src), static_cast<uint4*>(dst), n8,
                                                    status);
  return cudaGetLastError();
}

}  // namespace entmax
