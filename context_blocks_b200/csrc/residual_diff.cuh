// First Block Cache's residual difference (diffusers "ParaAttention" guide,
// section "First Block Cache": the change of the first transformer block's
// residual output between two denoising steps stands in for the change of
// the model's output, and cached residuals are reused while it is small):
//     diff = sum_i |cur_i - prev_i| / sum_i |prev_i|
// over n bf16 elements, accumulated in fp32.
//
// HBM-bound: 4 bytes read per element.  Deterministic two-pass reduction: a
// fixed grid of blocks sums its grid-stride share of 16-byte vectors (8
// elements, streaming loads) per thread, then through a fixed shuffle tree,
// and leaves one (diff, prev) pair per block in a small static array; one
// block adds the pairs in block order and writes the ratio (0 when both sums
// are 0, +inf when only the denominator is).  Calls that overlap on the GPU
// race on that array; calls ordered on a stream do not.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "lse_merge.cuh"  // unpack_bf16x8

namespace pa {

constexpr int kRdThreads = 256;
constexpr int kRdMaxBlocks = 1024;

static __device__ float2 g_rd_partial[kRdMaxBlocks];

// Sum of a float2 over the block, in a fixed order; valid in thread 0.
__device__ __forceinline__ float2 rd_block_sum(float2 v) {
  __shared__ float2 warp_sums[kRdThreads / 32];
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    v.x += __shfl_xor_sync(0xffffffffu, v.x, off);
    v.y += __shfl_xor_sync(0xffffffffu, v.y, off);
  }
  if ((threadIdx.x & 31) == 0) warp_sums[threadIdx.x >> 5] = v;
  __syncthreads();
  float2 s = make_float2(0.f, 0.f);
  if (threadIdx.x == 0)
    for (int w = 0; w < kRdThreads / 32; ++w) {
      s.x += warp_sums[w].x;
      s.y += warp_sums[w].y;
    }
  return s;
}

__global__ void __launch_bounds__(kRdThreads)
    residual_diff_partial_kernel(const __nv_bfloat16* __restrict__ cur, const __nv_bfloat16* __restrict__ prev,
                                 long long n) {
  const long long nv = n / 8;  // whole 16-byte vectors
  const uint4* c4 = reinterpret_cast<const uint4*>(cur);
  const uint4* p4 = reinterpret_cast<const uint4*>(prev);
  float sd = 0.f, sp = 0.f;
  const long long stride = static_cast<long long>(gridDim.x) * kRdThreads;
  for (long long i = static_cast<long long>(blockIdx.x) * kRdThreads + threadIdx.x; i < nv; i += stride) {
    float a[8], b[8];
    unpack_bf16x8(__ldcs(c4 + i), a);
    unpack_bf16x8(__ldcs(p4 + i), b);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      sd += fabsf(a[e] - b[e]);
      sp += fabsf(b[e]);
    }
  }
  if (blockIdx.x == 0)  // the last n mod 8 elements
    for (long long i = nv * 8 + threadIdx.x; i < n; i += kRdThreads) {
      const float a = __bfloat162float(cur[i]), b = __bfloat162float(prev[i]);
      sd += fabsf(a - b);
      sp += fabsf(b);
    }
  const float2 s = rd_block_sum(make_float2(sd, sp));
  if (threadIdx.x == 0) g_rd_partial[blockIdx.x] = s;
}

__global__ void __launch_bounds__(kRdThreads) residual_diff_final_kernel(int nblocks, float* __restrict__ out) {
  float2 v = make_float2(0.f, 0.f);
  for (int b = threadIdx.x; b < nblocks; b += kRdThreads) {
    v.x += g_rd_partial[b].x;
    v.y += g_rd_partial[b].y;
  }
  const float2 s = rd_block_sum(v);
  if (threadIdx.x == 0) out[0] = (s.y == 0.f) ? (s.x == 0.f ? 0.f : INFINITY) : s.x / s.y;
}

}  // namespace pa
