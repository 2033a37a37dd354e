// Definitions shared by the forward kernels (attn_fwd.cuh, attn_fwd_pair.cuh):
// tile sizes, launch parameters and the small arithmetic helpers of the
// online softmax.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "ptx.cuh"

namespace pa {

constexpr int kBM = 128;           // query rows per tile (= TMEM lanes)
constexpr int kBN = 128;           // keys per K/V tile
constexpr int kQTiles = 2;         // query tiles per CTA
constexpr uint32_t kTmemCols = 512;
// Lazy rescaling: the reference maximum of a row moves only when a tile's
// maximum exceeds it by more than 2^kRescaleLog2 (in base-2 logits).
constexpr float kRescaleLog2 = 8.0f;

// Device status codes written by kernels (mirror PA_ERR_* in pa_attn.h).
constexpr int kStatusTimeout = -5;

struct FwdParams {
  __nv_bfloat16* o;     // [B*H, Nq, D]
  float* lse;           // [B*H, Nq]
  int Nq;
  int Nk;               // keys in all chunks of the launch
  int n_kv_tiles;       // key tiles in all chunks of the launch
  float scale_log2;     // scale * log2(e)
  int* status;          // device status word
  unsigned long long timeout_ns;
  float qk_scale;       // logits are also multiplied by this (q_scale * k_scale; 1 for bf16)
  float o_scale;        // O is multiplied by this (the V dequantisation scale; 1 for bf16)
  // Device-side dequantisation scales (e4m3 inputs), used instead of
  // qk_scale / o_scale when dscale_q is not null.
  const float* dscale_q;
  const float* dscale_k;
  const float* dscale_v;
};

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float lg2_approx(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);  // .x (low half) = lo
  return *reinterpret_cast<uint32_t*>(&h);
}

// ---- packed fp32 pairs (Blackwell f32x2 ALU forms) -------------------------
__device__ __forceinline__ uint64_t f2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2_split(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ float max3f(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// 2^x on the FMA pipe for both halves of a pair, to take load off the MUFU
// unit.  Range reduction x = n + f with n = round-to-nearest(x) (adding and
// subtracting 1.5 * 2^23) and f in [-1/2, 1/2]; 2^f by a degree-3 polynomial
// (coefficients from gen_exp2_poly.py: minimax in relative error, 7.6e-5 on
// the reduced range); 2^n by adding n to the exponent field.  x is clamped to
// >= -126 so that the exponent add cannot underflow into the sign bit; the
// result for smaller x is ~2^-126, i.e. zero at the precision P is kept in.
constexpr float kExp2C0 = 9.999275804e-01f;
constexpr float kExp2C1 = 6.932516098e-01f;
constexpr float kExp2C2 = 2.426152676e-01f;
constexpr float kExp2C3 = 5.522262305e-02f;
constexpr float kRoundMagic = 12582912.0f;  // 1.5 * 2^23

__device__ __forceinline__ uint64_t exp2_poly_x2(uint64_t x) {
  float a, b;
  f2_split(x, a, b);
  const uint64_t xc = f2(fmaxf(a, -126.f), fmaxf(b, -126.f));
  const uint64_t t = f2_add(xc, f2(kRoundMagic, kRoundMagic));        // magic + n
  const uint64_t n = f2_add(t, f2(-kRoundMagic, -kRoundMagic));       // n (exact)
  const uint64_t fr = f2_fma(n, f2(-1.f, -1.f), xc);                  // f = x - n (exact)
  uint64_t p = f2_fma(f2(kExp2C3, kExp2C3), fr, f2(kExp2C2, kExp2C2));
  p = f2_fma(p, fr, f2(kExp2C1, kExp2C1));
  p = f2_fma(p, fr, f2(kExp2C0, kExp2C0));
  float p0, p1, t0, t1;
  f2_split(p, p0, p1);
  f2_split(t, t0, t1);
  // low bits of t hold n; shifting by 23 moves n into the exponent field
  const float r0 = __uint_as_float(__float_as_uint(p0) + (__float_as_uint(t0) << 23));
  const float r1 = __uint_as_float(__float_as_uint(p1) + (__float_as_uint(t1) << 23));
  return f2(r0, r1);
}

}  // namespace pa
