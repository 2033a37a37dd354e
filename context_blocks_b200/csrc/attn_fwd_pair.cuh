// Blockwise attention forward on a pair of CTAs (thread-block cluster of 2)
// using the CTA-pair tensor-core MMA (tcgen05 cta_group::2), head dim 128.
//
// Same computation, warp roles, tensor-memory layout and online softmax as
// attn_fwd_kernel (attn_fwd.cuh); what changes is how the two query tiles of
// the two CTAs share the tensor cores.  The pair covers 512 query rows: each
// CTA holds 2 x 128 rows, and the leader CTA (cluster rank 0) issues, for
// query tile i, one M = 256 MMA over its own Q_i rows and the peer's.  The B
// operand of a pair MMA is split along N between the CTAs, so each CTA loads
// only half of every K tile (64 keys) and half of every V tile (64 head-dim
// columns): half the shared-memory operand traffic and half the K/V loads
// per query row of the single-CTA kernel, where an M = 128, N = 128 MMA
// reading both operands from shared memory needs the SM's full shared-memory
// bandwidth.
//
// Synchronisation across the pair:
//   * each CTA's TMA loads count their bytes on the leader's full barriers,
//     whose expected byte count (set by the leader) covers both halves;
//   * the leader's tcgen05.commit arrives, by multicast, on the barrier at
//     the same offset in both CTAs (S ready, O ready, slot free);
//   * both CTAs' softmax warps arrive on the leader's P-ready barriers;
//   * waits on phases another CTA completes go through mbar_wait_cluster
//     (default scope unless PA_PAIR_CLUSTER_SCOPE asks for explicit cluster
//     scope), and a cluster barrier brackets set-up and teardown.
// The producer and MMA roles run as warp-uniform loops with one elected lane
// issuing, as in attn_fwd.cuh.
// The loads are plain per-CTA loads: nothing in this kernel multicasts data.
#pragma once

#include "fwd_common.cuh"

namespace pa {
namespace pairk {

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


// Share of exponentials computed on the FMA pipe (see exp2_poly_x2): one pair
// in kEmuEvery; 0 = all on MUFU.
#ifndef PA_EMU_EVERY
#define PA_EMU_EVERY 0
#endif
constexpr int kEmuEvery = PA_EMU_EVERY;  // 0: every exponential on MUFU


constexpr int kPairStages = 8;  // K/V ring slots of 16 KB (one K half or one V half)

struct PairLayout {
  static constexpr int kQBoxBytes = kBM * 128;          // 128 rows x 64 bf16, 128B-swizzled
  static constexpr int kQTileBytes = 2 * kQBoxBytes;    // one 128 x 128 query tile
  static constexpr int kKBoxBytes = (kBN / 2) * 128;    // 64 keys x 64 bf16
  static constexpr int kSlotBytes = kBN * 128;          // K half (2 boxes of 64 keys) or V half (128 keys x 64)
  static constexpr int kQOff = 0;
  static constexpr int kRingOff = kQOff + kQTiles * kQTileBytes;
  static constexpr int kBarOff = kRingOff + kPairStages * kSlotBytes;
  // q_full[2], kv_full[S], kv_empty[S], s_full[2], p_full[2][2], o_full[2], drain, turn[2]
  static constexpr int kNumBars = 2 + 2 * kPairStages + 2 + 4 + 2 + 1 + 2;
  static constexpr int kTmemSlotOff = kBarOff + kNumBars * 8;
  static constexpr int kAbortOff = kTmemSlotOff + 4;
  static constexpr int kBytes = kAbortOff + 4;
  static constexpr int kAllocBytes = kBytes + 1024;     // slack to align the base to 1024 B
  static_assert(kAllocBytes <= 227 * 1024, "shared memory");
};

template <int D>
__global__ void __launch_bounds__(kFwdThreads, 1)
    attn_fwd_pair_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
  static_assert(D == 128, "the CTA-pair kernel is written for d = 128");
  using L = PairLayout;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);

  const uint32_t sQ = base + L::kQOff;
  const uint32_t sRing = base + L::kRingOff;
  const uint32_t bars = base + L::kBarOff;
  const uint32_t bar_q_full0 = bars;
  const uint32_t bar_kv_full0 = bars + 8 * 2;
  const uint32_t bar_kv_empty0 = bars + 8 * (2 + kPairStages);
  const uint32_t bar_s_full0 = bars + 8 * (2 + 2 * kPairStages);
  const uint32_t bar_p_full0 = bars + 8 * (4 + 2 * kPairStages);   // [tile i][half h] at 8 * (2i + h)
  const uint32_t bar_o_full0 = bars + 8 * (8 + 2 * kPairStages);
  const uint32_t bar_drain = bars + 8 * (10 + 2 * kPairStages);
  const uint32_t bar_turn0 = bars + 8 * (11 + 2 * kPairStages);
  // This CTA's place in the pair: rank 0 (the leader) issues every MMA of the
  // pair; both CTAs load their own operand halves and run their own softmax.
  const uint32_t rank = cluster_ctarank();
  const bool leader = (rank == 0);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + L::kTmemSlotOff);
  volatile int* abort_word = reinterpret_cast<volatile int*>(gbase + L::kAbortOff);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const int q0 = (blockIdx.x / 2) * (2 * kQTiles * kBM) + static_cast<int>(rank) * (kQTiles * kBM);
  const int bh = blockIdx.y;
  const int n = p.n_kv_tiles;
  const uint64_t lim = p.timeout_ns;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) mbar_init(bar_q_full0 + 8 * i, 1);
    for (int s = 0; s < kPairStages; ++s) {
      mbar_init(bar_kv_full0 + 8 * s, 1);
      mbar_init(bar_kv_empty0 + 8 * s, kMmaThreads);  // one commit per leader issuing thread
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar_s_full0 + 8 * i, 1);
      mbar_init(bar_p_full0 + 8 * (2 * i), 8);      // one arrival per softmax warp of both CTAs
      mbar_init(bar_p_full0 + 8 * (2 * i + 1), 8);
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
    // Same warp in both CTAs: the pair gets the same columns in each TMEM.
    tmem_alloc_pair(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // barriers of both CTAs initialised before any remote use
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // Warpgroup 2 hands registers back before the softmax warpgroups take
  // them (each call is made by every warp of its warpgroup).
  if (warp >= 8) setmaxnreg_dec<kOtherRegs>();
  if (warp == kTmaWarp) {
    // ------------------------------------------------------------ producer
    // Each CTA loads its own Q tiles and its halves of every K and V tile into
    // its own shared memory; the bytes are counted on the leader's barriers,
    // whose expected byte counts (set by the leader) cover both CTAs.
    // Ring order: K_0, V_0, K_1, V_1, ...; load idx goes to slot idx % kPairStages.
    // The whole warp runs the loop in step; the elected lane issues.
    const bool el = elect_one();
    if (el) {
      for (int i = 0; i < kQTiles; ++i) {
        const uint32_t full = bar_q_full0 + 8 * i;
        if (leader) mbar_arrive_expect_tx(full, 2 * L::kQTileBytes);
        const uint32_t full_l = mapa_shared(full, 0);
#pragma unroll
        for (int bx = 0; bx < 2; ++bx)
          tma_load_3d_pair(sQ + i * L::kQTileBytes + bx * L::kQBoxBytes, &tm_q, full_l, bx * 64, q0 + i * kBM, bh);
      }
    }
    __syncwarp();
    bool ok = true;
    int idx = 0;  // ring loads issued so far
    for (int j = 0; j < n && ok; ++j) {
      for (int t = 0; t < 2; ++t) {  // t = 0: K_j half, t = 1: V_j half
        const int s = idx % kPairStages;
        const uint32_t u = idx / kPairStages;
        const bool got =
            mbar_wait_cluster(bar_kv_empty0 + 8 * s, (u & 1) ^ 1, abort_word, p.status, kStatusTimeout, lim);
        if (!__all_sync(0xffffffffu, got)) {
          ok = false;
          break;
        }
        if (el) {
          const uint32_t full = bar_kv_full0 + 8 * s;
          if (leader) mbar_arrive_expect_tx(full, 2 * L::kSlotBytes);
          const uint32_t full_l = mapa_shared(full, 0);
          const uint32_t dst = sRing + s * L::kSlotBytes;
          if (t == 0) {
            // keys [128 j + 64 rank, +64) x all 128 head-dim columns (two boxes)
#pragma unroll
            for (int bx = 0; bx < 2; ++bx)
              tma_load_3d_pair(dst + bx * L::kKBoxBytes, &tm_k, full_l, bx * 64,
                               j * kBN + static_cast<int>(rank) * (kBN / 2), bh);
          } else {
            // all 128 keys x head-dim columns [64 rank, +64) (one box)
            tma_load_3d_pair(dst, &tm_v, full_l, static_cast<int>(rank) * 64, j * kBN, bh);
          }
        }
        __syncwarp();
        ++idx;
      }
    }
    if (!ok) {
      // Aborted.  The leader's barriers count both CTAs' bytes: the leader
      // waits (bounded) for the last phase of each slot it armed; then both
      // CTAs give straggling copies a further 200 us before leaving.
      if (leader) {
        for (int i = 0; i < kQTiles; ++i)
          mbar_wait_cluster(bar_q_full0 + 8 * i, 0, nullptr, p.status, kStatusTimeout, lim);
        for (int s = 0; s < kPairStages && s < idx; ++s) {
          const int cnt = (idx - s + kPairStages - 1) / kPairStages;
          mbar_wait_cluster(bar_kv_full0 + 8 * s, (cnt - 1) & 1, nullptr, p.status, kStatusTimeout, lim);
        }
      }
      const uint64_t t0 = globaltimer_ns();
      while (globaltimer_ns() - t0 < 200000ull) {
      }
    }
    __syncwarp();
  } else if (leader && (warp == kMmaWarp || (kMmaThreads == 2 && warp == kMmaWarp + 2))) {
    // ------------------------------------------------------------ MMA issue
    // Leader CTA only.  This warp serves query tiles [i_lo, i_hi): the pair
    // MMAs S_i = Q_i K_j^T and O_i += P_i V_j cover the Q_i rows of both CTAs
    // (M = 256), each CTA's TMEM receiving its own 128 rows.  The whole warp
    // runs the loop in step; the elected lane issues.  Shared-memory
    // descriptors are built once and advanced by constant offsets.
    const bool el = elect_one();
    const int i_lo = (kMmaThreads == 2) ? (warp - kMmaWarp) / 2 : 0;
    const int i_hi = (kMmaThreads == 2) ? i_lo + 1 : 2;
    constexpr uint32_t kIdS = idesc_bf16(2 * kBM, kBN, false, false);
    constexpr uint32_t kIdPV = idesc_bf16(2 * kBM, D, false, true);
    const uint64_t dQ = sdesc_k_sw128(sQ);
    const uint64_t dK = sdesc_k_sw128(sRing);
    const uint64_t dV = sdesc_mn_sw128(sRing, L::kSlotBytes);

    // S_i = Q_i K^T : A = this CTA's Q_i (K-major, 16 KB per 64-column box),
    // B = each CTA's 64 keys of K_j (K-major, 8 KB per 64-column box).
    auto issue_qk = [&](int i, int slot) {
      const uint64_t dq = dQ + static_cast<uint64_t>(i * (L::kQTileBytes >> 4));
      const uint64_t dk = dK + static_cast<uint64_t>(slot * (L::kSlotBytes >> 4));
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint64_t oa = static_cast<uint64_t>(((kk / 4) * L::kQBoxBytes + (kk % 4) * 32) >> 4);
        const uint64_t ob = static_cast<uint64_t>(((kk / 4) * L::kKBoxBytes + (kk % 4) * 32) >> 4);
        umma_ss_pair(tmem + i * kBN, dq + oa, dk + ob, kIdS, kk > 0);
      }
    };
    // O_i (+)= P_i V, half h = keys [64h, 64h + 64): A = P_i in each CTA's
    // TMEM (bf16 pairs, 8 columns per 16 keys); B = each CTA's 64 head-dim
    // columns of V_j (MN-major, 16 keys = 2048 bytes).
    auto issue_pv_half = [&](int i, int slot, int h, bool acc) {
      const uint64_t dv = dV + static_cast<uint64_t>(slot * (L::kSlotBytes >> 4));
#pragma unroll
      for (int q = 0; q < kBN / 32; ++q) {
        const int kk = h * (kBN / 32) + q;
        umma_ts_pair(tmem + 2 * kBN + i * D, tmem + i * kBN + kk * 8, dv + static_cast<uint64_t>(kk * (2048 >> 4)),
                     kIdPV, (acc || kk > 0) ? 1u : 0u);
      }
    };
    auto wait_all = [&](uint32_t bar, uint32_t parity) {
      const bool got = mbar_wait_cluster(bar, parity, abort_word, p.status, kStatusTimeout, lim);
      return __all_sync(0xffffffffu, got);
    };

    bool ok = wait_all(bar_kv_full0, 0);
    for (int i = i_lo; i < i_hi && ok; ++i) {
      ok = wait_all(bar_q_full0 + 8 * i, 0);
      if (ok) {
        tc_fence_after();
        if (el) {
          issue_qk(i, 0);
          umma_commit_pair_both(bar_s_full0 + 8 * i);
        }
        __syncwarp();
      }
    }
    if (ok && el) umma_commit_pair_both(bar_kv_empty0);
    __syncwarp();
    int idx = 1;  // ring position of the next tile to consume (K0 was 0)
    for (int j = 0; j < n && ok; ++j) {
      const int sv = idx % kPairStages;
      const uint32_t uv = idx / kPairStages;
      ++idx;
      int sk = 0;
      uint32_t uk = 0;
      const bool more = (j + 1 < n);
      if (more) {
        sk = idx % kPairStages;
        uk = idx / kPairStages;
        ++idx;
      }
      if (!wait_all(bar_kv_full0 + 8 * sv, uv & 1)) {
        ok = false;
        break;
      }
      for (int i = i_lo; i < i_hi && ok; ++i) {
        // O_i += P_i V_j in two halves: the first half of P is ready while
        // the softmax warpgroups still compute the second.
        for (int h = 0; h < 2 && ok; ++h) {
          ok = wait_all(bar_p_full0 + 8 * (2 * i + h), j & 1);
          if (ok) {
            tc_fence_after();
            if (el) issue_pv_half(i, sv, h, j > 0);
            __syncwarp();
          }
        }
        if (!ok) break;
        if (el && i == i_hi - 1) umma_commit_pair_both(bar_kv_empty0 + 8 * sv);
        __syncwarp();
        if (more) {
          if (i == i_lo) {
            if (!wait_all(bar_kv_full0 + 8 * sk, uk & 1)) {
              ok = false;
              break;
            }
            tc_fence_after();
          }
          // S_i(j+1) overwrites the columns P_i(j) occupies: issued after
          // the P.V that reads them, and MMAs of one thread run in order.
          if (el) {
            issue_qk(i, sk);
            umma_commit_pair_both(bar_s_full0 + 8 * i);
            if (i == i_hi - 1) umma_commit_pair_both(bar_kv_empty0 + 8 * sk);
          }
        } else if (el) {
          umma_commit_pair_both(bar_o_full0 + 8 * i);
        }
        __syncwarp();
      }
    }
    // Every MMA this warp issued completes before tensor memory is freed.
    if (el) umma_commit_pair_both(bar_drain);
    __syncwarp();
    mbar_wait_cluster(bar_drain, 0, nullptr, p.status, kStatusTimeout, lim);
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
      const bool got = mbar_wait_cluster(bar_s_full0 + 8 * i, j & 1, abort_word, p.status, kStatusTimeout, lim);
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
        if (lane == 0) mbar_arrive_cluster(mapa_shared(bar_p_full0 + 8 * (2 * i + h), 0));
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
      const bool got = mbar_wait_cluster(bar_o_full0 + 8 * i, 0, abort_word, p.status, kStatusTimeout, lim);
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
  // Neither CTA leaves while the other may still read its shared memory (pair
  // MMAs), count bytes on its barriers or arrive on them.
  cluster_sync_all();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, kTmemCols);
  }
}

}  // namespace pairk
}  // namespace pa
