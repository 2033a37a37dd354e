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
// Kernel structure (persistent: each CTA walks work items, an item being 256
// query rows of one (b, h); the next item's Q load and first Q K^T overlap the
// current item's last tiles and epilogue):
//   warps 0-3  softmax warpgroup for query tile 0 (rows   0..127 of the block)
//   warps 4-7  softmax warpgroup for query tile 1 (rows 128..255 of the block)
//   warp  8    TMEM allocation + tcgen05.mma issue (the whole warp runs the
//              loop in step, one elected lane issues)
//   warp  9    TMA producer (Q once, then the K_j / V_j ring; same scheme)
//   warps 10-11 idle, completing warpgroup 2 for a register split
//              that gives the softmax warps 208 registers
// Tensor memory (512 columns x 128 lanes, fp32):
//   [0,128)        S_0 = Q_0 K_j^T   (P_0 is written back over it: bf16
//                  pairs, or four e4m3 per column with e4m3 inputs)
//   [128,256)      S_1 = Q_1 K_j^T   (P_1 likewise)
//   [256,256+D)    O_0 accumulator
//   [256+D,256+2D) O_1 accumulator
// Thread t of softmax warpgroup i owns TMEM lane t = query row t of tile i,
// so row max, row sum and rescaling need no cross-thread reduction.  Each
// warpgroup hands P to the MMA warp in two halves, so P.V on the first 64
// keys starts while the second half is still being computed.
//
// Accumulate mode (kAcc; FwdParams::acc_o and acc_lse set): the launch folds
// its chunk into a caller-owned running state, a normalised fp32 O and its
// LSE.  That state is
// exactly (O_unnormalised = O, l = 1, m = LSE * log2(e)) in the online softmax
// below, so the softmax threads load it into the O accumulator before the
// first tile and carry on; the epilogue writes the updated state back (or,
// on the final fold, the bf16 output).
//
// With kFp8 the same kernel takes e4m3 Q, K, V (per-tensor scales folded into
// the logit scale and the epilogue) and issues kind::f8f6f4 MMAs.  A share of
// the exponentials (1 in 4 in both paths) runs on the FMA pipe.
//
// Shared memory: Q (two tiles), a 4-slot K/V ring, a 4 KB output staging area
// per softmax warp, then the barriers (230.6 KB with bf16 d = 128).
//
// Online softmax in base 2: x = s * scale * log2(e).  m_ref is the reference
// maximum the exponentials of this row use; it moves only when a new tile's
// maximum exceeds it by more than kRescaleLog2 (lazy rescaling), in which case
// the running sum l and the O accumulator are multiplied by
// 2^(m_ref_old - m_ref_new).  Unnormalised P = 2^(x - m_ref) <= 2^kRescaleLog2.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "fwd_common.cuh"

namespace pa {
namespace single {

// Waits of the softmax warps and of the MMA-issuing warp pass this
// suspend-time hint to mbarrier.try_wait: a waiting thread sleeps until the
// phase completes instead of probing the barrier again and again.
constexpr uint32_t kSuspendHintNs = 1000000;  // 1 ms; the wait itself stays bounded by the time limit

constexpr int kPParts = 2;         // P is handed to the MMA warp in this many parts
constexpr int kStages = 4;         // K/V ring slots (each holds one K or one V tile)
constexpr int kMaxChunks = 8;      // K/V chunks one launch can consume
// Pairs e of each 32-key chunk whose bit is set here take 2^x on the FMA pipe
// instead of MUFU.  With the softmax warps at 208 registers, 1 in 4 pairs was
// measured fastest in both paths: e4m3 (exp2_poly2_x2; the tensor pipe needs
// half the time of the exponentials there) against 3/16, 5/16 and 1/2, bf16
// (exp2_poly3_x2) against 1/8, 3/16, 5/16 and 3/8.  The FMA pipe draws more
// power, so under the power cap the gain is smaller than per clock.
constexpr uint32_t kPolyPairsFp8 = 0x8888u;
constexpr uint32_t kPolyPairsBf16 = 0x8888u;

// The K/V chunks of one launch: keys are the concatenation of the chunks, in
// order; each chunk has its own tensor maps and its own (possibly ragged)
// length, so a chunk's last tile is masked at that chunk's length.  Passed as a
// __grid_constant__ kernel parameter (the TMA unit reads the maps in place).
struct KvChunks {
  CUtensorMap k[kMaxChunks];
  CUtensorMap v[kMaxChunks];
  int nk[kMaxChunks];          // keys in chunk c
  int tiles[kMaxChunks];       // ceil(nk[c] / kBN)
  int tile_start[kMaxChunks];  // key tiles before chunk c (unused entries: INT_MAX)
  int n_chunks;
};
constexpr int kMmaWarp = 8;
constexpr int kTmaWarp = 9;
// 12 warps, warps 10 and 11 idle so that warps 8-11 form a warpgroup for the
// register split below (both paths; the e4m3 path gains 2% from it).
// The split: each sub-partition holds three warps of 168 registers at launch
// (3 x 32 x 168 = 16128 of its 16384); warpgroup 2 (MMA, TMA, 2 idle) drops
// to 88 and the two softmax warpgroups rise to 208 (32 x (88 + 2 x 208) =
// 16128, the launch's own allocation).  The host checks that the kernel was
// built with exactly kLaunchRegs registers before it launches one.
constexpr int kFwdThreads = 384;
constexpr int kLaunchRegs = 168;
constexpr int kSoftmaxRegs = 208;
constexpr int kControlRegs = 88;
static_assert(kControlRegs + 2 * kSoftmaxRegs == 3 * kLaunchRegs, "register split must sum to the launch allocation");

// kFp8: Q, K, V are e4m3 (one byte per element) instead of bf16.
template <int D, bool kFp8 = false>
struct FwdLayout {
  static_assert(D == 64 || D == 128, "head dim must be 64 or 128");
  static_assert(!kFp8 || D == 128, "the e4m3 path is written for d = 128 (one 128-byte row per key)");
  static constexpr int kElemBytes = kFp8 ? 1 : 2;
  static constexpr int kBoxCols = 128 / kElemBytes;  // elements in one 128-byte swizzled row
  static constexpr int kBoxBytes = 128 * 128;        // 128 rows x 128 bytes, 128B-swizzled
  static constexpr int kBoxes = D / kBoxCols;
  // Contraction depth of one MMA: 32 bytes = 16 bf16 or 32 e4m3 elements.
  static constexpr int kKPerMma = kFp8 ? 32 : 16;
  static constexpr int kTileBytes = kBoxes * kBoxBytes;  // one 128-row tile of Q, K or V
  static constexpr int kQOff = 0;
  static constexpr int kRingOff = kQOff + kQTiles * kTileBytes;
  // One 4 KB staging area per softmax warp: 32 rows x 128 bytes of O (or of
  // the fp32 running state) on their way between TMEM and global memory.
  static constexpr int kStageOff = kRingOff + kStages * kTileBytes;
  static constexpr int kStageWarpBytes = 32 * 128;
  static constexpr int kBarOff = kStageOff + 8 * kStageWarpBytes;
  // q_full[2], kv_full[S], kv_empty[S], s_full[2], p_full[2], o_full[2], drain,
  // p_part[2][3] (parts of P before the last, which arrives on p_full), q_empty
  static constexpr int kNumBars = 2 + 2 * kStages + 2 + 2 + 2 + 1 + 6 + 1;
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

// O rows move between TMEM and global memory through a 4 KB staging area per
// warp, 128 bytes of each of the warp's 32 rows at a time.  A thread holds one
// row (its TMEM lane); it writes or reads its row's piece in the staging area
// with 16-byte chunk c of row r at chunk position c ^ (r % 8), so that 8
// consecutive rows fall in distinct banks, while global memory sees 4 rows x
// 128 contiguous bytes per warp instruction instead of 32 separate rows.
// Both helpers stay out of line: they run once per work item, and inlined
// into the kernel they cost the key loop registers.
//
// Global rows: row r of the warp is at dst0 + r * D elements; rows
// r >= rows_left are neither read nor written.

// Scale this thread's O row (TMEM columns [tO, tO + D)) by inv_l and store it:
// bf16 to `o_bf16`, or, when o_bf16 is null, fp32 to `o_f32`.
template <int D>
__device__ __noinline__ void store_o_rows(uint32_t tO, uint32_t stg, __nv_bfloat16* o_bf16, float* o_f32,
                                          int rows_left, float inv_l) {
  const int lane = threadIdx.x % 32;
  const int r0 = lane >> 3, c = lane & 7;
  auto stage4 = [&](int c0, const uint32_t (&w)[16]) {
#pragma unroll
    for (int u = 0; u < 4; ++u)
      st_shared_v4(stg + lane * 128 + (((c0 + u) ^ (lane & 7)) << 4), w[4 * u], w[4 * u + 1], w[4 * u + 2],
                   w[4 * u + 3]);
  };
  auto drain = [&](uint8_t* dst, int row_bytes) {
    dst += r0 * row_bytes + c * 16;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int r = 4 * k + r0;
      const uint4 x = ld_shared_v4(stg + r * 128 + ((c ^ (r & 7)) << 4));
      if (r < rows_left) *reinterpret_cast<uint4*>(dst + k * 4 * row_bytes) = x;
    }
  };
  if (o_bf16 != nullptr) {
#pragma unroll 1
    for (int h = 0; h < D / 64; ++h) {  // 64 bf16 columns = 128 bytes a piece
      __syncwarp();                      // the previous piece has left the staging area
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        uint32_t orr[32], pk[16];
        tmem_ld_x32(tO + h * 64 + hh * 32, orr);
#pragma unroll
        for (int e = 0; e < 16; ++e)
          pk[e] = pack_bf16x2(__uint_as_float(orr[2 * e]) * inv_l, __uint_as_float(orr[2 * e + 1]) * inv_l);
        stage4(4 * hh, pk);
      }
      __syncwarp();
      drain(reinterpret_cast<uint8_t*>(o_bf16 + h * 64), D * 2);
    }
  } else {
#pragma unroll 1
    for (int ch = 0; ch < D / 32; ++ch) {  // 32 fp32 columns = 128 bytes a piece
      uint32_t orr[32];
      tmem_ld_x32(tO + ch * 32, orr);
      __syncwarp();
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        uint32_t w[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) w[e] = __float_as_uint(__uint_as_float(orr[16 * hh + e]) * inv_l);
        stage4(4 * hh, w);
      }
      __syncwarp();
      drain(reinterpret_cast<uint8_t*>(o_f32 + ch * 32), D * 4);
    }
  }
}

// Load this thread's row of a running state: its LSE (returned; -inf for
// rows r >= rows_left) and its fp32 O into TMEM columns [tO, tO + D) (zeros
// where the LSE is -inf); waits for the TMEM stores.  All of the warp's
// global loads are issued before any is used (one round trip).
template <int D>
__device__ __noinline__ float load_state_rows(uint32_t tO, uint32_t stg, const float* src0, const float* lse_row,
                                              int rows_left) {
  const int lane = threadIdx.x % 32;
  const int r0 = lane >> 3, c = lane & 7;
  const float lse0 = (lane < rows_left) ? *lse_row : -INFINITY;
  uint4 buf[D / 32][8];
#pragma unroll
  for (int ch = 0; ch < D / 32; ++ch) {
    const uint4* src = reinterpret_cast<const uint4*>(src0 + r0 * D + ch * 32) + c;
#pragma unroll
    for (int k = 0; k < 8; ++k)
      buf[ch][k] = (4 * k + r0 < rows_left) ? __ldg(src + k * 4 * (D / 4)) : make_uint4(0u, 0u, 0u, 0u);
  }
  const bool have = lse0 > -INFINITY;
#pragma unroll
  for (int ch = 0; ch < D / 32; ++ch) {
    __syncwarp();  // the previous piece has left the staging area
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int r = 4 * k + r0;
      st_shared_v4(stg + r * 128 + ((c ^ (r & 7)) << 4), buf[ch][k].x, buf[ch][k].y, buf[ch][k].z, buf[ch][k].w);
    }
    __syncwarp();
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      uint32_t w[16];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const uint4 x = ld_shared_v4(stg + lane * 128 + (((4 * hh + u) ^ (lane & 7)) << 4));
        w[4 * u] = have ? x.x : 0u;
        w[4 * u + 1] = have ? x.y : 0u;
        w[4 * u + 2] = have ? x.z : 0u;
        w[4 * u + 3] = have ? x.w : 0u;
      }
      tmem_st_x16(tO + ch * 32 + hh * 16, w);
    }
  }
  tmem_st_wait();
  return lse0;
}

template <int D, bool kFp8 = false, bool kAcc = false>
__global__ void __launch_bounds__(kFwdThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ KvChunks kv,
                    const FwdParams p) {
  using L = FwdLayout<D, kFp8>;
  // Contraction depth of one MMA: 16 bf16 or 32 e4m3 elements (32 bytes).
  constexpr int kKPerMma = kFp8 ? 32 : 16;
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
  const uint32_t bar_p_full0 = bars + 8 * (4 + 2 * kStages);
  const uint32_t bar_o_full0 = bars + 8 * (6 + 2 * kStages);
  const uint32_t bar_drain = bars + 8 * (8 + 2 * kStages);
  const uint32_t bar_p_part0 = bars + 8 * (9 + 2 * kStages);  // + 8 * (3 * i + part)
  const uint32_t bar_q_empty = bars + 8 * (15 + 2 * kStages);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + L::kTmemSlotOff);
  volatile int* abort_word = reinterpret_cast<volatile int*>(gbase + L::kAbortOff);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const int n = p.n_kv_tiles;
  const uint64_t lim = p.timeout_ns;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) mbar_init(bar_q_full0 + 8 * i, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar_kv_full0 + 8 * s, 1);
      mbar_init(bar_kv_empty0 + 8 * s, 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar_s_full0 + 8 * i, 1);
      mbar_init(bar_p_full0 + 8 * i, 4);  // one arrival per softmax warp
      for (int q = 0; q < 3; ++q) mbar_init(bar_p_part0 + 8 * (3 * i + q), 4);
      mbar_init(bar_o_full0 + 8 * i, 1);
    }
    mbar_init(bar_drain, 1);
    mbar_init(bar_q_empty, 1);
    *abort_word = 0;
    fence_barrier_init();
  }
  if (warp == kTmaWarp && lane == 0) {
    prefetch_tensormap(&tm_q);
    for (int c = 0; c < kv.n_chunks; ++c) {
      prefetch_tensormap(&kv.k[c]);
      prefetch_tensormap(&kv.v[c]);
    }
  }
  if (warp == kMmaWarp) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp >= 10) {
    setmaxnreg_dec<kControlRegs>();  // idle: completes warpgroup 2
  } else if (warp == kTmaWarp) {
    setmaxnreg_dec<kControlRegs>();
    // ------------------------------------------------------------ producer
    // The whole warp runs the loop in step; the elected lane issues the loads.
    const bool leader = elect_one();
    bool ok = true;
    int idx = 0;      // ring loads issued so far (over all items)
    int q_loads = 0;  // items whose Q was issued
    for (int item = blockIdx.x; item < p.items && ok; item += gridDim.x) {
      const int bh = item / p.blocks_per_bh;
      const int q0 = (item % p.blocks_per_bh) * (kQTiles * kBM);
      // Q of this item once every Q K^T of the previous one has completed.
      if (!__all_sync(0xffffffffu, mbar_wait(bar_q_empty, (q_loads & 1) ^ 1, abort_word, p.status, kStatusTimeout,
                                             lim))) {
        ok = false;
        break;
      }
      if (leader) {
        for (int i = 0; i < kQTiles; ++i) {
          mbar_arrive_expect_tx(bar_q_full0 + 8 * i, L::kTileBytes);
#pragma unroll
          for (int b = 0; b < L::kBoxes; ++b)
            tma_load_3d(sQ + i * L::kTileBytes + b * L::kBoxBytes, &tm_q, bar_q_full0 + 8 * i, b * L::kBoxCols,
                        q0 + i * kBM, bh);
        }
      }
      __syncwarp();
      ++q_loads;
      for (int jt = 0; jt < n && ok; ++jt) {
        // Chunk of key tile jt and the tile's row offset inside that chunk.
        int c = 0;
#pragma unroll
        for (int cc = 1; cc < kMaxChunks; ++cc) c += (jt >= kv.tile_start[cc]) ? 1 : 0;
        const int row0 = (jt - kv.tile_start[c]) * kBN;
        for (int t = 0; t < 2; ++t) {  // t = 0: K tile, t = 1: V tile
          const int s = idx % kStages;
          const uint32_t u = idx / kStages;
          const bool got = mbar_wait(bar_kv_empty0 + 8 * s, (u & 1) ^ 1, abort_word, p.status, kStatusTimeout, lim);
          if (!__all_sync(0xffffffffu, got)) {
            ok = false;
            break;
          }
          if (leader) {
            const uint32_t full = bar_kv_full0 + 8 * s;
            mbar_arrive_expect_tx(full, L::kTileBytes);
            const CUtensorMap* map = t ? &kv.v[c] : &kv.k[c];
#pragma unroll
            for (int b = 0; b < L::kBoxes; ++b)
              tma_load_3d(sRing + s * L::kTileBytes + b * L::kBoxBytes, map, full, b * L::kBoxCols, row0, bh);
          }
          __syncwarp();
          ++idx;
        }
      }
    }
    if (!ok) {
      // Aborted: let every copy already in flight land before the CTA exits.
      // Slot s received ceil((idx - s) / kStages) loads; wait for the last.
      if (q_loads > 0)
        for (int i = 0; i < kQTiles; ++i)
          mbar_wait(bar_q_full0 + 8 * i, (q_loads - 1) & 1, nullptr, p.status, kStatusTimeout, lim);
      for (int s = 0; s < kStages && s < idx; ++s) {
        const int cnt = (idx - s + kStages - 1) / kStages;
        mbar_wait(bar_kv_full0 + 8 * s, (cnt - 1) & 1, nullptr, p.status, kStatusTimeout, lim);
      }
    }
    __syncwarp();
  } else if (warp == kMmaWarp) {
    setmaxnreg_dec<kControlRegs>();
    // ------------------------------------------------------------ MMA issue
    // The whole warp runs the loop in step and waits on the barriers; the
    // elected lane issues every tcgen05.mma and tcgen05.commit.  Shared-memory
    // descriptors are built once and advanced by constant offsets.
    const bool leader = elect_one();
    constexpr uint32_t kIdS = kFp8 ? idesc_e4m3(128, kBN, false) : idesc_bf16(128, kBN, false, false);
    constexpr uint32_t kIdPV = kFp8 ? idesc_e4m3(128, D, true) : idesc_bf16(128, D, false, true);
    constexpr uint64_t kTileDesc = L::kTileBytes >> 4;  // one tile in descriptor address units
    const uint32_t tO0 = tmem + 2 * kBN;
    const uint64_t dQ = sdesc_k_sw128(sQ);
    const uint64_t dK = sdesc_k_sw128(sRing);
    const uint64_t dV = sdesc_mn_sw128(sRing, L::kBoxBytes);

    // S_i = Q_i K^T : K-major Q and K, 32 bytes of depth per instruction (16
    // bf16 or 32 e4m3) inside a 128-byte row; the next row's worth of head
    // dimension is the next box.
    auto issue_qk = [&](int i, int slot) {
      const uint64_t dq = dQ + i * kTileDesc, dk = dK + slot * kTileDesc;
#pragma unroll
      for (int kk = 0; kk < D / kKPerMma; ++kk) {
        constexpr int kBox = L::kBoxBytes;
        const uint64_t off = static_cast<uint64_t>(((kk / 4) * kBox + (kk % 4) * 32) >> 4);
        if constexpr (kFp8)
          umma_ss_f8(tmem + i * kBN, dq + off, dk + off, kIdS, kk > 0);
        else
          umma_ss(tmem + i * kBN, dq + off, dk + off, kIdS, kk > 0);
      }
    };
    // O_i (+)= P_i V : P from TMEM (bf16 pairs, 8 columns per 16 keys),
    // V MN-major (rows of 64 head-dim elements, 16 keys = 2048 bytes).
    // P occupies 8 TMEM columns per MMA (16 bf16 or 32 e4m3 keys); V is
    // MN-major, one MMA's keys = kKPerMma rows of 128 bytes.
    auto issue_pv = [&](int i, int slot, bool acc, int kk0 = 0, int kk1 = kBN / L::kKPerMma) {
      const uint64_t dv = dV + slot * kTileDesc;
#pragma unroll
      for (int kk = kk0; kk < kk1; ++kk) {
        const uint64_t voff = static_cast<uint64_t>(kk * ((kKPerMma * 128) >> 4));
        if constexpr (kFp8)
          umma_ts_f8(tO0 + i * D, tmem + i * kBN + kk * 8, dv + voff, kIdPV, (acc || kk > 0) ? 1u : 0u);
        else
          umma_ts(tO0 + i * D, tmem + i * kBN + kk * 8, dv + voff, kIdPV, (acc || kk > 0) ? 1u : 0u);
      }
    };
    auto wait_all = [&](uint32_t bar, uint32_t parity) {
      const bool got = mbar_wait_hint(bar, parity, abort_word, p.status, kStatusTimeout, lim, kSuspendHintNs);
      return __all_sync(0xffffffffu, got);
    };
    // With a running state loaded into O (accumulate mode) even the first
    // P.V accumulates.
    const bool o_loaded = kAcc && !(p.acc_flags & kAccFirst);

    bool ok = true;
    int idx = 0;  // ring position (over all items)
    int g = 0;    // key tiles over all items: phases of the S and P barriers
    int t = 0;    // items of this CTA
    for (int item = blockIdx.x; item < p.items && ok; item += gridDim.x, ++t) {
      if (!wait_all(bar_q_full0, t & 1) || !wait_all(bar_q_full0 + 8, t & 1) ||
          !wait_all(bar_kv_full0 + 8 * (idx % kStages), (idx / kStages) & 1)) {
        ok = false;
        break;
      }
      tc_fence_after();
      if (leader) {
        issue_qk(0, idx % kStages);
        umma_commit(bar_s_full0);
        issue_qk(1, idx % kStages);
        umma_commit(bar_s_full0 + 8);
        umma_commit(bar_kv_empty0 + 8 * (idx % kStages));
        if (n == 1) umma_commit(bar_q_empty);
      }
      __syncwarp();
      ++idx;
      for (int j = 0; j < n && ok; ++j, ++g) {
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
        if (!wait_all(bar_kv_full0 + 8 * sv, uv & 1)) {
          ok = false;
          break;
        }
        for (int i = 0; i < 2; ++i) {
          // P.V part by part: part q covers keys [q, q + 1) * kBN / kPParts.
          constexpr int kKkPerPart = (kBN / kKPerMma) / kPParts;
          for (int q = 0; q < kPParts - 1 && ok; ++q) {
            if (!wait_all(bar_p_part0 + 8 * (3 * i + q), g & 1)) {
              ok = false;
              break;
            }
            tc_fence_after();
            if (leader) issue_pv(i, sv, o_loaded || j > 0 || q > 0, q * kKkPerPart, (q + 1) * kKkPerPart);
            __syncwarp();
          }
          if (!ok || !wait_all(bar_p_full0 + 8 * i, g & 1)) {
            ok = false;
            break;
          }
          tc_fence_after();
          // The last part accumulates unless it is also the first of the item.
          if (leader)
            issue_pv(i, sv, kPParts > 1 || o_loaded || j > 0, (kPParts - 1) * kKkPerPart, kBN / kKPerMma);
          if (leader && i == 1) umma_commit(bar_kv_empty0 + 8 * sv);
          __syncwarp();
          if (more) {
            if (i == 0) {
              if (!wait_all(bar_kv_full0 + 8 * sk, uk & 1)) {
                ok = false;
                break;
              }
              tc_fence_after();
            }
            if (leader) {
              issue_qk(i, sk);
              umma_commit(bar_s_full0 + 8 * i);
              if (i == 1) {
                umma_commit(bar_kv_empty0 + 8 * sk);
                if (j + 2 == n) umma_commit(bar_q_empty);  // the item's last Q K^T
              }
            }
          } else if (leader) {
            umma_commit(bar_o_full0 + 8 * i);
          }
          __syncwarp();
        }
      }
    }
    // Every MMA issued completes before tensor memory is freed.
    if (leader) umma_commit(bar_drain);
    __syncwarp();
    mbar_wait(bar_drain, 0, nullptr, p.status, kStatusTimeout, lim);
    __syncwarp();
  } else {
    setmaxnreg_inc<kSoftmaxRegs>();
    // ------------------------------------------------------------ softmax
    const int i = warp / 4;                    // query tile of this warpgroup
    const int t = threadIdx.x % 128;           // row within the tile = TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>((warp % 4) * 32) << 16;
    const uint32_t tS = tmem + i * kBN + lane_off;
    const uint32_t tO = tmem + 2 * kBN + i * D + lane_off;
    // Logit scale in log2 units; e4m3 inputs may carry their dequantisation
    // scales in device memory, which are checked here: a scale that is not
    // finite and positive is reported in the status word (the outputs are then
    // meaningless, as the header says).
    float c = p.scale_log2;
    float o_mul = 1.f;
    if constexpr (kFp8) {
      if (p.dscale_q != nullptr) {
        const float sq = __ldg(p.dscale_q), sk = __ldg(p.dscale_k), sv = __ldg(p.dscale_v);
        const bool good = (sq > 0.f && sq <= FLT_MAX) && (sk > 0.f && sk <= FLT_MAX) && (sv > 0.f && sv <= FLT_MAX);
        if (!good && threadIdx.x == 0) atomicCAS(p.status, 0, kStatusBadInput);
        c *= sq * sk;
        o_mul = sv;
      } else {
        c *= p.qk_scale;
        o_mul = p.o_scale;
      }
    }
    const bool o_loaded = kAcc && !(p.acc_flags & kAccFirst);
    bool ok = true;
    int g = 0;   // key tiles over all items: phases of the S barrier
    int it = 0;  // items of this CTA: phase of the O barrier
    // This thread's query row of an item, and its index in [B*H, Nq]
    // (recomputed where needed rather than kept live through the key loop).
    auto row_of = [&](int item) { return (item % p.blocks_per_bh) * (kQTiles * kBM) + i * kBM + t; };
    auto index_of = [&](int item) {
      return static_cast<size_t>(item / p.blocks_per_bh) * p.Nq + row_of(item);
    };
    for (int item = blockIdx.x; item < p.items && ok; item += gridDim.x, ++it) {
      float m_ref = -INFINITY;
      float l = 0.f;
      // Accumulate mode: start from the caller's running (O, LSE) instead of
      // an empty state.  Rows past Nq and rows whose running LSE is -inf (no
      // key seen yet) start empty, with O = 0.  (This warpgroup's epilogue of
      // the previous item has read O out; its P V are complete.)
      if (o_loaded) {
        const int row0 = row_of(item) - lane;  // first row of this warp's 32
        const size_t idx0 = index_of(item) - lane;
        const float lse0 = load_state_rows<D>(tO, base + L::kStageOff + warp * L::kStageWarpBytes,
                                              p.acc_o + idx0 * D, p.acc_lse + idx0 + lane, p.Nq - row0);
        if (lse0 > -INFINITY) {
          m_ref = lse0 * 1.4426950408889634f;
          l = 1.f;
        }
      }

      for (int j = 0; j < n; ++j, ++g) {
        // Chunk of key tile j, from the prefix tile counts (no state carried).
        int chunk = 0;
#pragma unroll
        for (int cc = 1; cc < kMaxChunks; ++cc) chunk += (j >= kv.tile_start[cc]) ? 1 : 0;
        const int valid = kv.nk[chunk] - (j - kv.tile_start[chunk]) * kBN;  // keys of this tile in its chunk
        const bool got =
            mbar_wait_hint(bar_s_full0 + 8 * i, g & 1, abort_word, p.status, kStatusTimeout, lim, kSuspendHintNs);
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
        if (valid < kBN) {
#pragma unroll
          for (int e = 0; e < kBN; ++e)
            if (e >= valid) s[e] = -INFINITY;
        }
        // Row max: 8 independent chains of 3-input max.
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
          alpha = ex2_approx(m_ref - mx);  // 0 when the row was empty (m_ref = -inf)
          l *= alpha;
          m_ref = mx;
          rescale = (j > 0) || o_loaded;
        }
        if (__any_sync(0xffffffffu, rescale)) {
          // PV of tile j-1 has completed: S_i(j) was issued after it and the
          // tcgen05 ops of the issuing thread complete in order.  (On tile 0 of
          // a fold, O holds the loaded state this thread stored.)
#pragma unroll
          for (int ch = 0; ch < D / 32; ++ch) {
            uint32_t orr[32];
            tmem_ld_x32(tO + ch * 32, orr);
#pragma unroll
            for (int e = 0; e < 32; ++e) orr[e] = __float_as_uint(__uint_as_float(orr[e]) * alpha);
            tmem_st_x32(tO + ch * 32, orr);
          }
        }
        // x = s * c - m_ref on packed pairs, P = 2^x on MUFU (a share of the
        // pairs on the FMA pipe instead, see kPolyPairs*), the row sum in four
        // packed partial sums.
        const float neg_m = -m_ref;
        const uint64_t c2 = f2(c, c), nm2 = f2(neg_m, neg_m);
        uint64_t l4[4] = {f2(0.f, 0.f), f2(0.f, 0.f), f2(0.f, 0.f), f2(0.f, 0.f)};
#pragma unroll
        for (int ch = 0; ch < kBN / 32; ++ch) {
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const uint64_t x2 = f2_fma(f2(s[ch * 32 + 2 * e], s[ch * 32 + 2 * e + 1]), c2, nm2);
            float p0, p1;
            if (kFp8 && ((kPolyPairsFp8 >> e) & 1)) {
              f2_split(exp2_poly2_x2(x2), p0, p1);
            } else if (!kFp8 && ((kPolyPairsBf16 >> e) & 1)) {
              f2_split(exp2_poly3_x2(x2), p0, p1);
            } else {
              float x0, x1;
              f2_split(x2, x0, x1);
              p0 = ex2_approx(x0);
              p1 = ex2_approx(x1);
            }
            l4[e & 3] = f2_add(l4[e & 3], f2(p0, p1));
            if constexpr (kFp8) {
              // four e4m3 keys per 32-bit column, lowest key in the low byte
              const uint32_t h = pack_e4m3x2(p0, p1);
              if (e & 1)
                pk[e >> 1] |= h << 16;
              else
                pk[e >> 1] = h;
            } else {
              pk[e] = pack_bf16x2(p0, p1);
            }
          }
          if constexpr (kFp8) {
            const uint32_t(&pk8)[8] = *reinterpret_cast<const uint32_t(*)[8]>(pk);
            tmem_st_x8(tS + ch * 8, pk8);
          } else {
            tmem_st_x16(tS + ch * 16, pk);
          }
          constexpr int kChPerPart = (kBN / 32) / kPParts;  // 32-key chunks per part
          if ((ch + 1) % kChPerPart == 0 && ch + 1 < kBN / 32) {
            // Part (ch + 1) / kChPerPart - 1 of P is in TMEM: hand it over.
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_p_part0 + 8 * (3 * i + (ch + 1) / kChPerPart - 1));
          }
        }
        {
          const uint64_t sum = f2_add(f2_add(l4[0], l4[1]), f2_add(l4[2], l4[3]));
          float a, b;
          f2_split(sum, a, b);
          l += a + b;
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_p_full0 + 8 * i);
      }

      if (!ok) break;
      {
        const bool got = mbar_wait(bar_o_full0 + 8 * i, it & 1, abort_word, p.status, kStatusTimeout, lim);
        ok = !__any_sync(0xffffffffu, !got);
      }
      if (ok) {
        tc_fence_after();
        const int row0 = row_of(item) - lane;  // first row of this warp's 32
        const size_t idx0 = index_of(item) - lane;
        const float lse_out = (m_ref + lg2_approx(l)) * 0.69314718055994531f;
        // bf16 output, or (accumulate mode, before the final fold) the
        // running state: normalised fp32 O.
        const bool state_out = kAcc && !(p.acc_flags & kAccFinal);
        store_o_rows<D>(tO, base + L::kStageOff + warp * L::kStageWarpBytes, state_out ? nullptr : p.o + idx0 * D,
                        kAcc ? p.acc_o + idx0 * D : nullptr, p.Nq - row0, o_mul / l);
        if (row0 + lane < p.Nq) (kAcc ? p.acc_lse : p.lse)[idx0 + lane] = lse_out;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace single
}  // namespace pa
