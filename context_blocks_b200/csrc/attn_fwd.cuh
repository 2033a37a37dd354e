// Blockwise attention forward for one K/V chunk on sm_100a.
//
// Computes, for every (b, h) and query row i of this call,
//     O_i   = sum_j softmax_j(scale * q_i . k_j) v_j        (normalised)
//     LSE_i = ln sum_j exp(scale * q_i . k_j)               (natural log)
// over the keys j of the chunk given to the call.  This is the per-block
// step of Ring Attention as the diffusers "Context parallelism" guide
// describes it (section "Ring Attention": each device attends with the K/V
// block it holds); the (O, LSE) pair is what the merge kernel needs to
// combine blocks into the exact full-sequence result.  Keys past the chunk's
// real length never enter the softmax (section "Ring Anything Attention":
// blocks are trimmed back to their real length before attention).
//
// Kernel structure (one CTA per 256 query rows of one (b, h)):
//   warps 0-3  softmax warpgroup for query tile 0 (rows   0..127 of the block)
//   warps 4-7  softmax warpgroup for query tile 1 (rows 128..255 of the block)
//   warp  8    TMEM allocation + tcgen05.mma issue for query tile 0
//   warp  9    single-thread TMA producer (Q once, then K_j / V_j ring)
//   warp 10    tcgen05.mma issue for query tile 1
//   warp 11    idle (completes warpgroup 2 for register re-allocation)
// Each query tile has its own issuing thread, on its own SMSP: a thread that
// has just issued a burst of MMAs only gets to its next barrier wait once the
// tensor cores have taken them, so one thread serving both tiles would keep
// the tensor cores waiting on the slower tile's P.
// Tensor memory (512 columns x 128 lanes, fp32):
//   [0,128)        S_0 = Q_0 K_j^T   (P_0 is written back over it as bf16)
//   [128,256)      S_1 = Q_1 K_j^T   (P_1 likewise)
//   [256,256+D)    O_0 accumulator
//   [256+D,256+2D) O_1 accumulator
// Thread t of softmax warpgroup i owns TMEM lane t = query row t of tile i,
// so row max, row sum and rescaling need no cross-thread reduction.
//
// Online softmax in base 2: x = s * scale * log2(e).  m_ref is the reference
// maximum the exponentials of this row use; it moves only when a new tile's
// maximum exceeds it by more than kRescaleLog2 (lazy rescaling), in which case
// the running sum l and the O accumulator are multiplied by
// 2^(m_ref_old - m_ref_new).  Unnormalised P = 2^(x - m_ref) <= 2^kRescaleLog2.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "ptx.cuh"

namespace pa {

constexpr int kBM = 128;           // query rows per tile (= TMEM lanes)
constexpr int kBN = 128;           // keys per K/V tile
constexpr int kQTiles = 2;         // query tiles per CTA
constexpr int kStages = 4;         // K/V ring slots (each holds one K or one V tile)
constexpr int kFwdThreads = 384;   // 12 warps = 3 warpgroups
constexpr int kMmaWarp = 8;        // MMA issue for query tile 0 (tile 1: warp kMmaWarp + 2)
constexpr int kTmaWarp = 9;        // warp 11 only completes warpgroup 2
// Registers: the kernel is launched with kLaunchRegs per thread (what ptxas
// assigns under __launch_bounds__(384, 1); the host refuses to launch if it
// differs).  Warpgroup 2 (MMA issue, TMA, idle) then gives registers back and
// the two softmax warpgroups take them:
//   128 * kOtherRegs + 256 * kSoftmaxRegs == 384 * kLaunchRegs  (= 64512),
// and per SMSP (one warp of each warpgroup) 224 + 224 + 56 <= 512.
constexpr int kLaunchRegs = 168;
constexpr int kSoftmaxRegs = 224;
constexpr int kOtherRegs = 56;
static_assert(128 * kOtherRegs + 256 * kSoftmaxRegs == kFwdThreads * kLaunchRegs,
              "register split must use exactly the launch allocation");
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleLog2 = 8.0f;

// Exponential phase of the two softmax warpgroups runs in turns (warpgroup 0
// on tile j, then warpgroup 1 on tile j, then warpgroup 0 on tile j+1, ...):
// each then has the SM's MUFU units alone, and the tensor cores work on the
// other warpgroup's P.V and next S meanwhile.
#ifndef PA_SEQ_EXP
#define PA_SEQ_EXP 1
#endif
constexpr bool kSeqExp = PA_SEQ_EXP != 0;

// Threads issuing tcgen05.mma: 2 = one per query tile (warps 8 and 10),
// 1 = warp 8 serves both tiles.
#ifndef PA_MMA_THREADS
#define PA_MMA_THREADS 2
#endif
constexpr int kMmaThreads = PA_MMA_THREADS;
static_assert(kMmaThreads == 1 || kMmaThreads == 2, "one or two MMA-issuing threads");

// Device status codes written by kernels (mirror PA_ERR_* in pa_attn.h).
constexpr int kStatusTimeout = -5;

template <int D>
struct FwdLayout {
  static_assert(D == 64 || D == 128, "head dim must be 64 or 128");
  static constexpr int kBoxBytes = 128 * 128;        // 128 rows x 64 bf16, 128B-swizzled
  static constexpr int kBoxes = D / 64;
  static constexpr int kTileBytes = kBoxes * kBoxBytes;  // one 128-row tile of Q, K or V
  static constexpr int kQOff = 0;
  static constexpr int kRingOff = kQOff + kQTiles * kTileBytes;
  static constexpr int kBarOff = kRingOff + kStages * kTileBytes;
  // q_full[2], kv_full[S], kv_empty[S] (one arrival per issuing thread), s_full[2],
  // p_full[2][2], o_full[2], drain (one arrival per issuing thread), turn[2]
  static constexpr int kNumBars = 2 + 2 * kStages + 2 + 4 + 2 + 1 + 2;
  static constexpr int kTmemSlotOff = kBarOff + kNumBars * 8;
  static constexpr int kAbortOff = kTmemSlotOff + 4;
  static constexpr int kBytes = kAbortOff + 4;
  // Slack to align the base to 1024 B.  The request is also padded so that a
  // second CTA never fits on the SM: each CTA takes all 512 TMEM columns, and
  // a co-resident CTA would only sit blocked in tcgen05.alloc.
  static constexpr int kMinOneCtaPerSm = 120 * 1024;
  static constexpr int kAllocBytes =
      (kBytes + 1024 > kMinOneCtaPerSm) ? (kBytes + 1024) : kMinOneCtaPerSm;
};

struct FwdParams {
  __nv_bfloat16* o;     // [B*H, Nq, D]
  float* lse;           // [B*H, Nq]
  int Nq;
  int Nk;
  int n_kv_tiles;       // ceil(Nk / kBN)
  float scale_log2;     // scale * log2(e)
  int* status;          // device status word
  unsigned long long timeout_ns;
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

// Share of exponentials computed on the FMA pipe (see exp2_poly_x2): one pair
// in kEmuEvery; 0 = all on MUFU.
#ifndef PA_EMU_EVERY
#define PA_EMU_EVERY 0
#endif
constexpr int kEmuEvery = PA_EMU_EVERY;  // 0: every exponential on MUFU


template <int D>
__global__ void __launch_bounds__(kFwdThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
  using L = FwdLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);

  const uint32_t sQ = base + L::kQOff;
  const uint32_t sRing = base + L::kRingOff;
  const uint32_t bars = base + L::kBarOff;
  const uint32_t bar_q_full0 = bars;
  const uint32_t bar_kv_full0 = bars + 8 * 2;
  const uint32_t bar_kv_empty0 = bars + 8 * (2 + kStages);
  const uint32_t bar_s_full0 = bars + 8 * (2 + 2 * kStages);
  const uint32_t bar_p_full0 = bars + 8 * (4 + 2 * kStages);   // [tile i][half h] at 8 * (2i + h)
  const uint32_t bar_o_full0 = bars + 8 * (8 + 2 * kStages);
  const uint32_t bar_drain = bars + 8 * (10 + 2 * kStages);
  const uint32_t bar_turn0 = bars + 8 * (11 + 2 * kStages);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + L::kTmemSlotOff);
  volatile int* abort_word = reinterpret_cast<volatile int*>(gbase + L::kAbortOff);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const int q0 = blockIdx.x * (kQTiles * kBM);
  const int bh = blockIdx.y;
  const int n = p.n_kv_tiles;
  const uint64_t lim = p.timeout_ns;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) mbar_init(bar_q_full0 + 8 * i, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar_kv_full0 + 8 * s, 1);
      mbar_init(bar_kv_empty0 + 8 * s, kMmaThreads);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar_s_full0 + 8 * i, 1);
      mbar_init(bar_p_full0 + 8 * (2 * i), 4);      // one arrival per softmax warp
      mbar_init(bar_p_full0 + 8 * (2 * i + 1), 4);
      mbar_init(bar_o_full0 + 8 * i, 1);
    }
    mbar_init(bar_drain, kMmaThreads);
    for (int i = 0; i < 2; ++i) mbar_init(bar_turn0 + 8 * i, 4);  // one arrival per softmax warp
    *abort_word = 0;
    fence_barrier_init();
  }
  if (warp == kTmaWarp && lane == 0) {
    prefetch_tensormap(&tm_q);
    prefetch_tensormap(&tm_k);
    prefetch_tensormap(&tm_v);
  }
  if (warp == kMmaWarp) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // Warpgroup 2 hands registers back before the softmax warpgroups take
  // them (each call is made by every warp of its warpgroup).
  if (warp >= 8) setmaxnreg_dec<kOtherRegs>();
  if (warp == kTmaWarp) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      for (int i = 0; i < kQTiles; ++i) {
        mbar_arrive_expect_tx(bar_q_full0 + 8 * i, L::kTileBytes);
#pragma unroll
        for (int b = 0; b < L::kBoxes; ++b)
          tma_load_3d(sQ + i * L::kTileBytes + b * L::kBoxBytes, &tm_q, bar_q_full0 + 8 * i, b * 64,
                      q0 + i * kBM, bh);
      }
      bool ok = true;
      int idx = 0;  // ring loads issued so far
      for (int j = 0; j < n && ok; ++j) {
        for (int t = 0; t < 2; ++t) {  // t = 0: K_j, t = 1: V_j
          const int s = idx % kStages;
          const uint32_t u = idx / kStages;
          if (!mbar_wait(bar_kv_empty0 + 8 * s, (u & 1) ^ 1, abort_word, p.status, kStatusTimeout, lim)) {
            ok = false;
            break;
          }
          const uint32_t full = bar_kv_full0 + 8 * s;
          mbar_arrive_expect_tx(full, L::kTileBytes);
          const CUtensorMap* map = t ? &tm_v : &tm_k;
#pragma unroll
          for (int b = 0; b < L::kBoxes; ++b)
            tma_load_3d(sRing + s * L::kTileBytes + b * L::kBoxBytes, map, full, b * 64, j * kBN, bh);
          ++idx;
        }
      }
      if (!ok) {
        // Aborted: let every copy already in flight land before the CTA exits.
        // Slot s received ceil((idx - s) / kStages) loads; wait for the last.
        for (int i = 0; i < kQTiles; ++i)
          mbar_wait(bar_q_full0 + 8 * i, 0, nullptr, p.status, kStatusTimeout, lim);
        for (int s = 0; s < kStages && s < idx; ++s) {
          const int cnt = (idx - s + kStages - 1) / kStages;
          mbar_wait(bar_kv_full0 + 8 * s, (cnt - 1) & 1, nullptr, p.status, kStatusTimeout, lim);
        }
      }
    }
    __syncwarp();
  } else if (warp == kMmaWarp || (kMmaThreads == 2 && warp == kMmaWarp + 2)) {
    // ------------------------------------------------------------ MMA issue
    // This thread serves query tiles [i_lo, i_hi): S_i = Q_i K_j^T and
    // O_i += P_i V_j for each of them.
    if (lane == 0) {
      const int i_lo = (kMmaThreads == 2) ? (warp - kMmaWarp) / 2 : 0;
      const int i_hi = (kMmaThreads == 2) ? i_lo + 1 : 2;
      constexpr uint32_t kIdS = idesc_bf16(128, kBN, false, false);
      constexpr uint32_t kIdPV = idesc_bf16(128, D, false, true);

      // S_i = Q_i K^T : K-major Q and K, 16 bf16 of depth per instruction.
      auto issue_qk = [&](int i, uint32_t sK) {
        const uint32_t sQi = sQ + i * L::kTileBytes;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk / 4) * L::kBoxBytes + (kk % 4) * 32;
          umma_ss(tmem + i * kBN, sdesc_k_sw128(sQi + off), sdesc_k_sw128(sK + off), kIdS, kk > 0);
        }
      };
      // O_i (+)= P_i V, half h = keys [64h, 64h + 64): P from TMEM (bf16
      // pairs, 8 columns per 16 keys), V MN-major (16 keys = 2048 bytes).
      auto issue_pv_half = [&](int i, uint32_t sV, int h, bool acc) {
#pragma unroll
        for (int q = 0; q < kBN / 32; ++q) {
          const int kk = h * (kBN / 32) + q;
          umma_ts(tmem + 2 * kBN + i * D, tmem + i * kBN + kk * 8,
                  sdesc_mn_sw128(sV + kk * 2048, L::kBoxBytes), kIdPV, (acc || kk > 0) ? 1u : 0u);
        }
      };

      bool ok = mbar_wait(bar_kv_full0, 0, abort_word, p.status, kStatusTimeout, lim);
      for (int i = i_lo; i < i_hi && ok; ++i) {
        ok = mbar_wait(bar_q_full0 + 8 * i, 0, abort_word, p.status, kStatusTimeout, lim);
        if (ok) {
          tc_fence_after();
          issue_qk(i, sRing);
          umma_commit(bar_s_full0 + 8 * i);
        }
      }
      if (ok) umma_commit(bar_kv_empty0);
      int idx = 1;  // ring position of the next tile to consume (K0 was 0)
      for (int j = 0; j < n && ok; ++j) {
        const int sv = idx % kStages;
        const uint32_t uv = idx / kStages;
        ++idx;
        int sk = 0;
        uint32_t uk = 0;
        const bool more = (j + 1 < n);
        if (more) {
          sk = idx % kStages;
          uk = idx / kStages;
          ++idx;
        }
        if (!mbar_wait(bar_kv_full0 + 8 * sv, uv & 1, abort_word, p.status, kStatusTimeout, lim)) {
          ok = false;
          break;
        }
        for (int i = i_lo; i < i_hi && ok; ++i) {
          // O_i += P_i V_j in two halves: the first half of P is ready while
          // the softmax warpgroup still computes the second.
          for (int h = 0; h < 2 && ok; ++h) {
            ok = mbar_wait(bar_p_full0 + 8 * (2 * i + h), j & 1, abort_word, p.status, kStatusTimeout, lim);
            if (ok) {
              tc_fence_after();
              issue_pv_half(i, sRing + sv * L::kTileBytes, h, j > 0);
            }
          }
          if (!ok) break;
          if (i == i_hi - 1) umma_commit(bar_kv_empty0 + 8 * sv);
          if (more) {
            if (i == i_lo) {
              if (!mbar_wait(bar_kv_full0 + 8 * sk, uk & 1, abort_word, p.status, kStatusTimeout, lim)) {
                ok = false;
                break;
              }
              tc_fence_after();
            }
            // S_i(j+1) overwrites the columns P_i(j) occupies: issued after
            // the P.V that reads them, and MMAs of one thread run in order.
            issue_qk(i, sRing + sk * L::kTileBytes);
            umma_commit(bar_s_full0 + 8 * i);
            if (i == i_hi - 1) umma_commit(bar_kv_empty0 + 8 * sk);
          } else {
            umma_commit(bar_o_full0 + 8 * i);
          }
        }
      }
      // Every MMA this thread issued completes before tensor memory is freed.
      umma_commit(bar_drain);
      mbar_wait(bar_drain, 0, nullptr, p.status, kStatusTimeout, lim);
    }
    __syncwarp();
  } else if (warp < 8) {
    // ------------------------------------------------------------ softmax
    setmaxnreg_inc<kSoftmaxRegs>();
    const int i = warp / 4;                    // query tile of this warpgroup
    const int t = threadIdx.x % 128;           // row within the tile = TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>((warp % 4) * 32) << 16;
    const uint32_t tS = tmem + i * kBN + lane_off;
    const uint32_t tO = tmem + 2 * kBN + i * D + lane_off;
    const int row = q0 + i * kBM + t;
    const float c = p.scale_log2;
    float m_ref = -INFINITY;
    float l = 0.f;
    bool ok = true;

    for (int j = 0; j < n; ++j) {
      const bool got = mbar_wait(bar_s_full0 + 8 * i, j & 1, abort_word, p.status, kStatusTimeout, lim);
      if (__any_sync(0xffffffffu, !got)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t sr[kBN];
      tmem_ld_x128(tS, sr);
      float s[kBN];
#pragma unroll
      for (int e = 0; e < kBN; ++e) s[e] = __uint_as_float(sr[e]);
      const int valid = p.Nk - j * kBN;  // keys of this tile inside the chunk
      const bool full_tile = valid >= kBN;
      if (!full_tile) {
#pragma unroll
        for (int e = 0; e < kBN; ++e)
          if (e >= valid) s[e] = -INFINITY;
      }
      // Row max: 8 independent chains of 3-input max (depth ~10, not 127).
      float m8[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) m8[k] = fmaxf(s[k], s[k + 8]);
#pragma unroll
      for (int e = 16; e < kBN; e += 16)
#pragma unroll
        for (int k = 0; k < 8; ++k) m8[k] = max3f(m8[k], s[e + k], s[e + 8 + k]);
      float mx = fmaxf(max3f(m8[0], m8[1], m8[2]), max3f(m8[3], m8[4], max3f(m8[5], m8[6], m8[7])));
      mx *= c;
      float alpha = 1.f;
      bool rescale = false;
      if (mx > m_ref + kRescaleLog2) {
        alpha = ex2_approx(m_ref - mx);  // 0 on the first tile (m_ref = -inf)
        l *= alpha;
        m_ref = mx;
        rescale = (j > 0);
      }
      if (__any_sync(0xffffffffu, rescale)) {
        // PV of tile j-1 has completed: S_i(j) was issued after it and the
        // tcgen05 ops of the issuing thread complete in order.
#pragma unroll
        for (int ch = 0; ch < D / 32; ++ch) {
          uint32_t orr[32];
          tmem_ld_x32(tO + ch * 32, orr);
#pragma unroll
          for (int e = 0; e < 32; ++e) orr[e] = __float_as_uint(__uint_as_float(orr[e]) * alpha);
          tmem_st_x32(tO + ch * 32, orr);
        }
      }
      if (kSeqExp) {
        // turn[i] completes when the other warpgroup has finished its
        // exponentials of the previous tile (warpgroup 0's first turn is free).
        const bool got = mbar_wait(bar_turn0 + 8 * i, (j & 1) ^ (i == 0 ? 1u : 0u), abort_word, p.status,
                                   kStatusTimeout, lim);
        if (__any_sync(0xffffffffu, !got)) {
          ok = false;
          break;
        }
      }
      // x = s * scale * log2(e) - m_ref, in place, two per instruction.
      {
        const uint64_t c2 = f2(c, c), nm2 = f2(-m_ref, -m_ref);
#pragma unroll
        for (int e = 0; e < kBN / 2; ++e) {
          const uint64_t x = f2_fma(f2(s[2 * e], s[2 * e + 1]), c2, nm2);
          f2_split(x, s[2 * e], s[2 * e + 1]);
        }
      }
      // P = 2^x (in place, fp32 kept for the row sum) and its bf16 pairs, in
      // two halves of 64 keys; each half goes to tensor memory and to the MMA
      // thread as soon as it is done.
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t pk[kBN / 4];
        if (full_tile) {
#pragma unroll
          for (int e = 0; e < kBN / 4; ++e) {
            const int k0 = h * (kBN / 2) + 2 * e;
            if (kEmuEvery > 0 && (e % (kEmuEvery > 0 ? kEmuEvery : 1)) == kEmuEvery - 1) {
              f2_split(exp2_poly_x2(f2(s[k0], s[k0 + 1])), s[k0], s[k0 + 1]);
            } else {
              s[k0] = ex2_approx(s[k0]);
              s[k0 + 1] = ex2_approx(s[k0 + 1]);
            }
            pk[e] = pack_bf16x2(s[k0], s[k0 + 1]);
          }
        } else {
          // Tail tile: MUFU only, so masked keys give exactly 2^-inf = 0.
#pragma unroll
          for (int e = 0; e < kBN / 4; ++e) {
            const int k0 = h * (kBN / 2) + 2 * e;
            s[k0] = ex2_approx(s[k0]);
            s[k0 + 1] = ex2_approx(s[k0 + 1]);
            pk[e] = pack_bf16x2(s[k0], s[k0 + 1]);
          }
        }
        if (kSeqExp && h == 1) {
          __syncwarp();
          if (lane == 0) mbar_arrive(bar_turn0 + 8 * (1 - i));
        }
        tmem_st_x32(tS + h * (kBN / 4), pk);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_p_full0 + 8 * (2 * i + h));
      }
      // Row sum, off the path to the MMA thread.
      {
        uint64_t acc[4] = {f2(0.f, 0.f), f2(0.f, 0.f), f2(0.f, 0.f), f2(0.f, 0.f)};
#pragma unroll
        for (int e = 0; e < kBN / 2; ++e) acc[e & 3] = f2_add(acc[e & 3], f2(s[2 * e], s[2 * e + 1]));
        acc[0] = f2_add(f2_add(acc[0], acc[1]), f2_add(acc[2], acc[3]));
        float a0, a1;
        f2_split(acc[0], a0, a1);
        l += a0 + a1;
      }
    }

    if (ok) {
      const bool got = mbar_wait(bar_o_full0 + 8 * i, 0, abort_word, p.status, kStatusTimeout, lim);
      ok = !__any_sync(0xffffffffu, !got);
    }
    if (ok) {
      tc_fence_after();
      const float inv_l = 1.f / l;
      const bool in_range = row < p.Nq;
      __nv_bfloat16* orow = p.o + (static_cast<size_t>(bh) * p.Nq + row) * D;
#pragma unroll
      for (int ch = 0; ch < D / 32; ++ch) {
        uint32_t orr[32];
        tmem_ld_x32(tO + ch * 32, orr);
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          pk[e] = pack_bf16x2(__uint_as_float(orr[2 * e]) * inv_l, __uint_as_float(orr[2 * e + 1]) * inv_l);
        if (in_range) {
          uint4* dst = reinterpret_cast<uint4*>(orow + ch * 32);
#pragma unroll
          for (int v = 0; v < 4; ++v)
            dst[v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
        }
      }
      if (in_range)
        p.lse[static_cast<size_t>(bh) * p.Nq + row] = (m_ref + lg2_approx(l)) * 0.69314718055994531f;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace pa
