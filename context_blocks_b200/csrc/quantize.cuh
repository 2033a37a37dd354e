// Per-tensor e4m3 quantisation of a bf16 tensor on the device, for the fp8
// forward (the storage format the diffusers "ParaAttention" guide quantises
// activations to, its fp8 section):
//     amax  = max |x|
//     scale = amax / 448 in fp32 (1 when amax = 0)          (dequantisation)
//     inv   = 448 / amax in fp32 (1 when amax = 0)          (quantisation)
//     q     = e4m3 nearest to x * inv (one fp32 multiply), ties to even,
//             saturated to +-448
// Three stream-ordered launches share the caller's 4-byte `scale` word:
//   1. amax_kernel: |x| as bf16 bits (non-negative, so integer order is value
//      order) reduced per warp and combined with atomicMax into the word;
//   2. quantize_kernel: every block reads amax from the word, converts;
//   3. scale_kernel: one thread replaces the word by the float scale (and
//      reports a non-finite amax in the device status word).
// Both passes stream x with 16-byte loads (8 bf16); the second pass usually
// hits L2 for inputs up to its size.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "fwd_common.cuh"
#include "ptx.cuh"

namespace pa {
namespace quant {

constexpr int kThreads = 256;

__device__ __forceinline__ uint32_t abs_bits2(uint32_t two_bf16) {
  return max(two_bf16 & 0x7FFFu, (two_bf16 >> 16) & 0x7FFFu);
}

__global__ void __launch_bounds__(kThreads) amax_kernel(const __nv_bfloat16* __restrict__ x, long long n,
                                                        unsigned* __restrict__ word) {
  const long long n8 = n / 8;
  const uint4* x8 = reinterpret_cast<const uint4*>(x);
  uint32_t m = 0;
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < n8; i += stride) {
    const uint4 v = __ldg(x8 + i);  // cached: a tensor that fits in L2 is read from there by the second pass
    m = max(m, max(max(abs_bits2(v.x), abs_bits2(v.y)), max(abs_bits2(v.z), abs_bits2(v.w))));
  }
  if (blockIdx.x == 0 && threadIdx.x < n - n8 * 8) {
    const uint16_t b = reinterpret_cast<const uint16_t*>(x)[n8 * 8 + threadIdx.x];
    m = max(m, static_cast<uint32_t>(b & 0x7FFFu));
  }
  m = __reduce_max_sync(0xffffffffu, m);
  if ((threadIdx.x & 31) == 0 && m != 0) atomicMax(word, m);
}

__device__ __forceinline__ float scale_from_word(unsigned w) {
  if (w == 0) return 1.f;
  const float amax = __uint_as_float(w << 16);  // bf16 bits -> fp32
  return amax / 448.f;
}
__device__ __forceinline__ float inv_from_word(unsigned w) {
  if (w == 0) return 1.f;
  return 448.f / __uint_as_float(w << 16);
}

__device__ __forceinline__ uint32_t quant4(uint32_t a, uint32_t b, float inv) {
  // two bf16 pairs -> four e4m3 bytes (lowest element in the low byte)
  const float x0 = __uint_as_float(a << 16), x1 = __uint_as_float(a & 0xFFFF0000u);
  const float x2 = __uint_as_float(b << 16), x3 = __uint_as_float(b & 0xFFFF0000u);
  return pack_e4m3x2(__fmul_rn(x0, inv), __fmul_rn(x1, inv)) |
         (pack_e4m3x2(__fmul_rn(x2, inv), __fmul_rn(x3, inv)) << 16);
}

__global__ void __launch_bounds__(kThreads) quantize_kernel(const __nv_bfloat16* __restrict__ x, long long n,
                                                            const unsigned* __restrict__ word,
                                                            uint8_t* __restrict__ q) {
  const float inv = inv_from_word(*word);
  const long long n8 = n / 8;
  const uint4* x8 = reinterpret_cast<const uint4*>(x);
  uint2* q8 = reinterpret_cast<uint2*>(q);
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < n8; i += stride) {
    const uint4 v = __ldcs(x8 + i);
    q8[i] = make_uint2(quant4(v.x, v.y, inv), quant4(v.z, v.w, inv));
  }
  if (blockIdx.x == 0 && threadIdx.x < n - n8 * 8) {
    const long long e = n8 * 8 + threadIdx.x;
    const float xv = __uint_as_float(static_cast<uint32_t>(reinterpret_cast<const uint16_t*>(x)[e]) << 16);
    q[e] = static_cast<uint8_t>(pack_e4m3x2(__fmul_rn(xv, inv), 0.f) & 0xFFu);
  }
}

// A non-finite amax (an Inf or NaN element: bf16 magnitude bits >= 0x7F80)
// leaves no usable scale; it is recorded in the device status word.
__global__ void scale_kernel(unsigned* word, int* status) {
  const unsigned w = *word;
  if (w >= 0x7F80u) atomicCAS(status, 0, kStatusBadInput);
  *reinterpret_cast<float*>(word) = scale_from_word(w);
}

}  // namespace quant
}  // namespace pa
