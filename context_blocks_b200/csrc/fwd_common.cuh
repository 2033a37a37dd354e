// Definitions shared by the forward kernels: tile sizes, launch parameters
// and the small arithmetic helpers of the online softmax.
#pragma once

#include <cuda_bf16.h>
#include <cfloat>
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
constexpr int kStatusBadInput = -6;

// Accumulate-mode flags (FwdParams::acc_flags; PA_ACCUM_* in pa_attn.h).
constexpr int kAccFirst = 1;   // no incoming state: start from an empty one
constexpr int kAccFinal = 2;   // write the bf16 output instead of the fp32 state

struct FwdParams {
  __nv_bfloat16* o;     // [B*H, Nq, D]
  float* lse;           // [B*H, Nq]
  int items;            // work items: B*H * blocks_per_bh
  int blocks_per_bh;    // query blocks of kQTiles * kBM rows per (b, h)
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
  // Accumulate mode (acc_o != null): acc_o [B*H, Nq, D] fp32 and acc_lse
  // [B*H, Nq] hold the running (normalised O, LSE) that the launch folds its
  // keys into; `lse` is unused and `o` is written only with kAccFinal.
  float* acc_o;
  float* acc_lse;
  int acc_flags;
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
// unit: degree 2 in the e4m3 path (whose P is rounded to e4m3 right after),
// degree 3 in the bf16 path (P rounded to bf16, half step 2^-9).  Cody-Waite
// range reduction x = n + f, n = round-to-nearest(x) by adding and subtracting
// 1.5 * 2^23, f in [-1/2, 1/2]; 2^f by a degree-2 polynomial minimax in
// relative error (1.73e-3; coefficients from gen_exp2_poly.py); 2^n by adding
// n to the exponent field.  x is clamped to >= -126 so that the exponent add
// cannot reach the sign bit (masked keys, x = -inf, give ~2^-126, which
// rounds to 0 in e4m3).
constexpr float kExp2P2C0 = 1.000443101e+00f;
constexpr float kExp2P2C1 = 7.034479976e-01f;
constexpr float kExp2P2C2 = 2.384289354e-01f;
constexpr float kRoundMagic = 12582912.0f;  // 1.5 * 2^23

__device__ __forceinline__ uint64_t exp2_poly2_x2(uint64_t x) {
  float a, b;
  f2_split(x, a, b);
  const uint64_t xc = f2(fmaxf(a, -126.f), fmaxf(b, -126.f));
  const uint64_t t = f2_add(xc, f2(kRoundMagic, kRoundMagic));   // magic + n
  const uint64_t n = f2_add(t, f2(-kRoundMagic, -kRoundMagic));  // n (exact)
  const uint64_t fr = f2_fma(n, f2(-1.f, -1.f), xc);             // f = x - n (exact)
  uint64_t p = f2_fma(f2(kExp2P2C2, kExp2P2C2), fr, f2(kExp2P2C1, kExp2P2C1));
  p = f2_fma(p, fr, f2(kExp2P2C0, kExp2P2C0));
  float p0, p1, t0, t1;
  f2_split(p, p0, p1);
  f2_split(t, t0, t1);
  // the low bits of t hold n; shifted by 23 they land in the exponent field
  return f2(__uint_as_float(__float_as_uint(p0) + (__float_as_uint(t0) << 23)),
            __uint_as_float(__float_as_uint(p1) + (__float_as_uint(t1) << 23)));
}

// The same with a degree-3 polynomial (relative error 7.5e-5 on the reduced
// range, 1.4e-4 with the float32 steps; coefficients from gen_exp2_poly.py).
constexpr float kExp2P3C0 = 9.999280572e-01f;
constexpr float kExp2P3C1 = 6.932609677e-01f;
constexpr float kExp2P3C2 = 2.426111251e-01f;
constexpr float kExp2P3C3 = 5.517166853e-02f;

__device__ __forceinline__ uint64_t exp2_poly3_x2(uint64_t x) {
  float a, b;
  f2_split(x, a, b);
  const uint64_t xc = f2(fmaxf(a, -126.f), fmaxf(b, -126.f));
  const uint64_t t = f2_add(xc, f2(kRoundMagic, kRoundMagic));   // magic + n
  const uint64_t n = f2_add(t, f2(-kRoundMagic, -kRoundMagic));  // n (exact)
  const uint64_t fr = f2_fma(n, f2(-1.f, -1.f), xc);             // f = x - n (exact)
  uint64_t p = f2_fma(f2(kExp2P3C3, kExp2P3C3), fr, f2(kExp2P3C2, kExp2P3C2));
  p = f2_fma(p, fr, f2(kExp2P3C1, kExp2P3C1));
  p = f2_fma(p, fr, f2(kExp2P3C0, kExp2P3C0));
  float p0, p1, t0, t1;
  f2_split(p, p0, p1);
  f2_split(t, t0, t1);
  return f2(__uint_as_float(__float_as_uint(p0) + (__float_as_uint(t0) << 23)),
            __uint_as_float(__float_as_uint(p1) + (__float_as_uint(t1) << 23)));
}

}  // namespace pa
