// Merge of per-chunk partial attention results into the full result.
//
// For every row r (of B*H*N rows) and n partial results (O_p, LSE_p) computed
// over disjoint key chunks:
//     M = max_p LSE_p,   w_p = exp(LSE_p - M),   L = sum_p w_p
//     O = sum_p w_p O_p / L,   LSE = M + ln L
// This is how the per-block results of Ring Attention become the exact
// full-sequence attention once every block has been seen (diffusers
// "Context parallelism" guide, section "Ring Attention").  A part whose LSE is
// -inf (an empty chunk) carries no weight and its O_p is not read; a row whose
// parts are all -inf gets O = 0 and LSE = -inf.
//
// HBM-bound: each row is d bf16 per part; D/8 threads own one row and each
// moves 16 bytes per part with streaming (evict-first) loads.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

namespace pa {

constexpr int kMergeThreads = 256;

__device__ __forceinline__ void unpack_bf16x8(const uint4& raw, float (&f)[8]) {
  const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    f[2 * e] = __uint_as_float(w[e] << 16);
    f[2 * e + 1] = __uint_as_float(w[e] & 0xffff0000u);
  }
}

template <int D>
__global__ void __launch_bounds__(kMergeThreads)
    lse_merge_kernel(const __nv_bfloat16* __restrict__ o_parts, const float* __restrict__ lse_parts,
                     int n_parts, __nv_bfloat16* __restrict__ o, float* __restrict__ lse, long long rows) {
  constexpr int kTpr = D / 8;                 // threads per row
  constexpr int kRpb = kMergeThreads / kTpr;  // rows per block per sweep
  const int sub = threadIdx.x % kTpr;
  const long long stride = static_cast<long long>(gridDim.x) * kRpb;
  for (long long row = static_cast<long long>(blockIdx.x) * kRpb + threadIdx.x / kTpr; row < rows;
       row += stride) {
    float big_m = -INFINITY;
    for (int q = 0; q < n_parts; ++q) big_m = fmaxf(big_m, __ldg(lse_parts + q * rows + row));
    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.f;
    float out_lse = -INFINITY;
    if (big_m != -INFINITY) {
      float big_l = 0.f;
#pragma unroll 4
      for (int q = 0; q < n_parts; ++q) {
        const float lq = __ldg(lse_parts + q * rows + row);
        if (lq == -INFINITY) continue;
        const float w = __expf(lq - big_m);
        big_l += w;
        const uint4 raw = __ldcs(reinterpret_cast<const uint4*>(
            o_parts + (static_cast<long long>(q) * rows + row) * D + sub * 8));
        float f[8];
        unpack_bf16x8(raw, f);
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] = fmaf(w, f[e], acc[e]);
      }
      const float inv = 1.f / big_l;
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[e] *= inv;
      out_lse = big_m + __logf(big_l);
    }
    uint4 packed;
    {
      __nv_bfloat162 h0 = __floats2bfloat162_rn(acc[0], acc[1]);
      __nv_bfloat162 h1 = __floats2bfloat162_rn(acc[2], acc[3]);
      __nv_bfloat162 h2 = __floats2bfloat162_rn(acc[4], acc[5]);
      __nv_bfloat162 h3 = __floats2bfloat162_rn(acc[6], acc[7]);
      packed.x = *reinterpret_cast<uint32_t*>(&h0);
      packed.y = *reinterpret_cast<uint32_t*>(&h1);
      packed.z = *reinterpret_cast<uint32_t*>(&h2);
      packed.w = *reinterpret_cast<uint32_t*>(&h3);
    }
    __stcs(reinterpret_cast<uint4*>(o + row * D + sub * 8), packed);
    if (sub == 0) lse[row] = out_lse;
  }
}

}  // namespace pa
