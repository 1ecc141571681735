// attn_fwd.cu -- causal forward (prefill) attention for sm_100a, BF16 and
// FP8 e4m3, head dims (128,128) and MLA (192,128).
//
// Sources (ZYFA announcement as re-reported by three web pages):
//   [P1] "Zyphra ZYFA : FlashAttention en FP8 pour l'AMD MI355X, jusqu'a 1,76
//        fois plus rapide" (lefilia.fr), paragraph 3: FP8 doubles matrix
//        throughput but not the softmax; Lean P (an e4m3 pattern read as an
//        integer grows by 8 per doubling, so a multiply-add replaces exp);
//        each 64-key block scaled by a power of 2 and division by the sum of
//        the rounded probabilities.
//   [P2] "Zyphra rilascia ZYFA ..." (aicronaca.it), "Perche l'FP8 non basta da
//        solo": the block scale is absorbed by a scaled matrix instruction and
//        the rounded row sum comes from one more matrix instruction.
//   [P3] "Zyphra ZYFA ... FP8 FlashAttention for AMD MI355X" (ai4bro.com),
//        TL;DR (causal prefill, FP8 e4m3 and BF16, d 128 and MLA 192/128) and
//        "How ZYFA works" (scaling by powers of 2 before rounding).
//
// A unit is one 128-row query tile of one (batch, head).  With more than 64
// query tiles per head every CTA runs one unit (grid = units); shorter
// sequences run persistent CTAs (grid = min(units, SMs)) that take units in
// a zigzag order and carry their barrier phases from unit to unit.  Warp
// roles:
//   warps 0-7  softmax + epilogue.  TMEM lane quarter q (query rows
//              32q..32q+31) belongs to warps q and q+4, 16 rows each; inside
//              a warp, threads t and t+16 share a row, thread t taking keys
//              0-63 of every tile and thread t+16 keys 64-127 (one 64-key
//              scale block each; 16x32bx2 TMEM accesses)
//   warp 8     TMA producer: Q per unit, then K and V tiles through an
//              NS-stage ring (K and V of a stage land together), or, with
//              2 stages (BF16 MLA), through separate K and V rings that
//              refill independently
//   warp 9     TMEM allocator and tcgen05 issuer (the whole warp runs the
//              loop, one elected lane issues)
// Tensor memory (512 columns x 128 lanes, fp32 words):
//   S0 [0,128) S1 [128,256)   score tiles; P (bf16x2 or 4 x e4m3 per word) of
//                             keys 64h..64h+63 is written over the first
//                             columns of S half h (column 64h onwards)
//   O  [256,256+DV)           output accumulator
//   RS [384,400)              FP8: rounded row sum (P times the ones block)
//   SFA [400,408)             FP8: UE8M0 scales of P, one 4-column set per S
//                             buffer (replicated layout, see sf_smem below)
//   SFB [408,416)             FP8: scales of V and of the ones block, all 2^0
// FP8's rounded row sum is the PV MMA run with N = d_v + 16 against V and a
// block of ones, so it lands in TMEM columns 384..399 right after O.
// MMA issue order: QK_0, QK_1, PV_0, QK_2, PV_1, ... so the softmax of tile
// j+1 overlaps PV_j and QK_{j+2}.
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <cuda.h>

#include <atomic>
#include <cstdint>

#include "attn_math.cuh"
#include "schedule.h"
#include "sm100_ptx.cuh"
#include "zq_internal.h"

namespace zq {

constexpr int kSoftmaxThreads = 256;
constexpr int kThreads = kSoftmaxThreads + 64;
constexpr int kWarpProducer = 8, kWarpMma = 9;
constexpr uint32_t kColS0 = 0, kColO = 256, kColRS = 384, kColSFA = 400, kColSFB = 408;
constexpr uint32_t kTmemCols = 512;

template <int DT, int DQK, int DV>
struct Geo {
  static constexpr int ES = DT == 0 ? 2 : 1;
  static constexpr int QROW = DQK * ES;                    // bytes per Q/K row
  static constexpr int NCH = (QROW + 127) / 128;           // 128-byte chunks (last may be 64)
  static constexpr int LASTW = QROW - (NCH - 1) * 128;     // 128 or 64
  static constexpr int QBYTES = kTile * QROW;
  static constexpr int KBYTES = QBYTES;
  static constexpr int VBYTES = kTile * DV * ES;
  static constexpr int VCH = DV * ES / 128;                // 128-byte N chunks of V
  static constexpr int QK_STEPS = QROW / 32;               // 32 bytes of K per MMA
  static constexpr int PV_STEPS = DT == 0 ? 8 : 4;         // 16 (bf16) / 32 (fp8) keys per MMA
  // K/V ring stages: as many as fit in 227 KB of shared memory
  static constexpr int NS = DT == 1 ? 4 : (DQK == 128 ? 3 : 2);
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + QBYTES;
  static constexpr int OFF_V = OFF_K + NS * KBYTES;
  // FP8: one 128-key x 128-byte block of e4m3 ones after the V stages.  The
  // PV MMA runs with N = d_v + 16 and reaches it as the second 128-column
  // atom of V (leading byte offset = ONES - V stage), so the rounded row sum
  // lands in O's columns d_v .. d_v + 15.
  static constexpr int ONES_BYTES = DT == 1 ? 16384 : 0;
  static constexpr int OFF_ONES = OFF_V + NS * VBYTES;
  static constexpr int OFF_SF = OFF_ONES + ONES_BYTES;     // FP8: [2 buf] 512 B scale tiles
  static constexpr int SF_BYTES = DT == 1 ? 1024 : 0;
  static constexpr int OFF_BAR = OFF_SF + SF_BYTES;
  static constexpr int NBAR = 1 + 4 * NS + 2 + 2 + 1 + 2 + 1;
  static constexpr int SMEM = OFF_BAR + NBAR * 8 + 16 + 1024;  // + alignment slack
  static_assert(SMEM <= 232448, "227 KB of shared memory per CTA");
  static_assert(DV == 128, "the two halves of a row split d_v = 128 in 64 + 64");
  static_assert(QBYTES % 1024 == 0 && VBYTES % 1024 == 0, "1 KB aligned tiles");
};

// Debug trace (clock64 of the traced CTA), per key tile j, 16 slots:
//   [0] row 0 saw S_j  [1] row 0 loaded S_j  [2] row 0 computed P_j
//   [3] warp 0 released P_j  [4] warp 3 released P_j
//   [11] warp 1 released P_j  [12] warp 5 released P_j (warps 1 and 5 share
//        their SM sub-partition with the MMA warp)
//   MMA warp: [5] K_j landed, QK_j issue starts  [13] two QK_j MMAs issued
//   [6] QK_j issued + committed  [7] P_j seen  [8] block scales copied
//   [14] two PV_j MMAs issued  [9] PV_j MMAs issued  [10] PV_j committed
//   [15] unused
// Lives after the S/P/SF dump in the debug buffer.
constexpr int kTraceOffsetWords = 128 * 128 + 128 * 64 + 256;
constexpr int kTraceTiles = 512;
constexpr int kTraceSlots = 16;


// PERSIST = 0: one unit per CTA (the grid has one CTA per unit).
template <int DT, int DQK, int DV, int MODE, int BS, int DBG, int PERSIST>
__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmQ2,
                    const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmK2,
                    const __grid_constant__ CUtensorMap tmV, const AttnParams p) {
  using G = Geo<DT, DQK, DV>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + G::OFF_BAR);
  uint64_t* bar_q = bars;
  // With two stages (BF16 at d_qk = 192) K and V have separate rings: K_j is
  // consumed by QK_j, about two tiles before PV_j needs V_j, so a K stage
  // frees and refills much earlier, which a two-stage ring needs to hide the
  // load latency.  With more stages K_j and V_j share a stage: both land on
  // bar_kfull, and PV_j's commit on bar_vfree frees both (one commit and one
  // wait fewer per tile for the MMA warp, which measured faster there).
  constexpr bool kSplit = G::NS == 2;
  uint64_t* bar_kfull = bars + 1;             // [NS] K_j (and V_j unless split) landed
  uint64_t* bar_kfree = bar_kfull + G::NS;    // [NS] QK_j done: K stage reusable
  uint64_t* bar_vfull = bar_kfree + G::NS;    // [NS] V_j landed
  // bar_vfree[s] completes when PV_j (j = s mod NS) is done: it frees the V
  // stage and tells the softmax that O holds tiles <= j.  Softmax j
  // (j >= 1) waits for PV_{j-1}: of that stage's phases only the awaited
  // one or the one before can be complete, since PV_{j-1+NS} needs
  // P_{j-1+NS}; so the parity test is unambiguous.
  uint64_t* bar_vfree = bar_vfull + G::NS;    // [NS]
  uint64_t* bar_sfull = bar_vfree + G::NS;    // [2]
  uint64_t* bar_pfull = bar_sfull + 2;        // [2]
  uint64_t* bar_ofinal = bar_pfull + 2;       // [1] last PV of a unit landed
  // A CTA runs units one after another (persistent); the barrier phases run
  // on across units, every role counting the same sequence of key tiles
  // (jt) and of units with work (nq).
  uint64_t* bar_qfree = bar_ofinal + 1;       // [1] last QK of a unit done: Q reusable
  uint64_t* bar_ofree = bar_qfree + 1;        // [1] softmax read O (and RS) of a unit
  uint64_t* bar_drain = bar_ofree + 1;        // [1] after an abort: the MMA issuer's work landed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + G::NBAR);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  // FP8 scale factors staged for tcgen05.cp: per S buffer a 32-row x
  // 16-byte tile; query row r puts its word at byte 16*(r%32) + 4*(r/32),
  // and the copy lands it in TMEM column r/32 of the buffer's 4-column set at
  // lanes r%32 + 32q of every lane quarter q -- the replicated layout the
  // block-scaled MMA reads.  Byte k of the word scales keys 32k..32k+31.
  uint32_t* sf_smem = reinterpret_cast<uint32_t*>(smem + G::OFF_SF);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  const int n_units = p.n_qtiles * p.B * p.Hq;
  // the k-th unit of this CTA (zigzag rounds; schedule.h)
  auto unit_at = [&](int k) -> int { return zq::unit_at(k, (int)gridDim.x, (int)blockIdx.x); };
  const int shift = p.Sk - p.Sq;
  // debug dumps and the trace exist only in the DBG instantiation
  auto traced_unit = [&](const Unit& w) { return DBG && p.dbg != nullptr && w.t == p.dbg_t && w.bh == p.dbg_bh; };
  uint64_t* const trace_buf =
      DBG && p.dbg ? reinterpret_cast<uint64_t*>(static_cast<uint32_t*>(p.dbg) + kTraceOffsetWords) : nullptr;

  if (threadIdx.x == 0) {
    mbar_init(bar_q, 1);
    for (int s = 0; s < G::NS; ++s) {
      mbar_init(bar_kfull + s, 1);
      mbar_init(bar_kfree + s, 1);
      mbar_init(bar_vfull + s, 1);
      mbar_init(bar_vfree + s, 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar_sfull + s, 1);
      mbar_init(bar_pfull + s, kSoftmaxThreads);
    }
    mbar_init(bar_ofinal, 1);
    mbar_init(bar_qfree, 1);
    mbar_init(bar_ofree, kSoftmaxThreads);
    mbar_init(bar_drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (DT == 1) {  // ones operand for the rounded row sum: e4m3 1.0 = 0x38
    uint32_t* ones = reinterpret_cast<uint32_t*>(smem + G::OFF_ONES);
    for (int i = threadIdx.x; i < G::ONES_BYTES / 4; i += kThreads) ones[i] = 0x38383838u;
    fence_proxy_async_smem();
  }
  if (warp == kWarpMma) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  if (warp == kWarpProducer && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    if (G::LASTW == 64) {
      tma_prefetch_desc(&tmQ2);
      tma_prefetch_desc(&tmK2);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;
  const uint64_t lim = p.timeout_ns;

  // producer: the last load armed on each barrier, for the drain after an
  // abort -- Q loads issued, and the CTA-wide tile index of the last K/V (or
  // K and V) stage armed
  int q_loads = 0, x_last = -1, xk_last = -1, xv_last = -1;

  auto fail = [&]() {
    *abort_flag = 1;
    if (p.status) atomicExch(p.status, -7 /* ZQ_ERR_TIMEOUT */);
  };

  if (warp == kWarpProducer) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int jt = 0, nq = 0;
      bool ok = true;
      for (int k = 0, u = unit_at(0); ok && u < n_units; u = PERSIST ? unit_at(++k) : n_units) {
        const Unit w = unit_of(p, u);
        if (w.n_kv == 0) continue;
        // Q of the previous unit is read until its last QK completes
        if (nq > 0 && !mbar_wait(bar_qfree, (nq - 1) & 1, lim, abort_flag)) { ok = false; break; }
        uint8_t* sq = smem + G::OFF_Q;
        mbar_arrive_expect_tx(bar_q, G::QBYTES);
        ++q_loads;
#pragma unroll
        for (int c = 0; c < G::NCH; ++c) {
          const bool narrow = (c == G::NCH - 1) && G::LASTW == 64;
          tma_load_4d(sq + c * 16384, narrow ? (const void*)&tmQ2 : (const void*)&tmQ, bar_q,
                      c * 128 / G::ES, w.h, w.q0, w.b);
        }
        if constexpr (!kSplit) {
          for (int j = 0; j < w.n_kv; ++j) {
            const int x = jt + j, s = x % G::NS;
            // the stage is free once PV of its previous tile is done (first pass: free)
            if (!mbar_wait(bar_vfree + s, ((x / G::NS) & 1) ^ 1, lim, abort_flag)) { ok = false; break; }
            uint8_t* sk = smem + G::OFF_K + s * G::KBYTES;
            uint8_t* sv = smem + G::OFF_V + s * G::VBYTES;
            mbar_arrive_expect_tx(bar_kfull + s, G::KBYTES + G::VBYTES);
            x_last = x;
#pragma unroll
            for (int c = 0; c < G::NCH; ++c) {
              const bool narrow = (c == G::NCH - 1) && G::LASTW == 64;
              tma_load_4d(sk + c * 16384, narrow ? (const void*)&tmK2 : (const void*)&tmK,
                          bar_kfull + s, c * 128 / G::ES, w.g, j * kTile, w.b);
            }
#pragma unroll
            for (int c = 0; c < G::VCH; ++c)
              tma_load_4d(sv + c * 16384, &tmV, bar_kfull + s, c * 128 / G::ES, w.g, j * kTile, w.b);
          }
        } else {
          // K runs ahead of V inside the unit; each ring refills as its stages free
          int jk = 0, jv = 0;
          uint64_t t0 = 0;
          uint32_t idle = 0;
          while (jv < w.n_kv) {
            bool progressed = false;
            if (jk < w.n_kv) {
              const int x = jt + jk, s = x % G::NS;
              if (mbar_test_wait(smem_u32(bar_kfree + s), ((x / G::NS) & 1) ^ 1)) {  // first pass: free
                uint8_t* sk = smem + G::OFF_K + s * G::KBYTES;
                mbar_arrive_expect_tx(bar_kfull + s, G::KBYTES);
                xk_last = x;
#pragma unroll
                for (int c = 0; c < G::NCH; ++c) {
                  const bool narrow = (c == G::NCH - 1) && G::LASTW == 64;
                  tma_load_4d(sk + c * 16384, narrow ? (const void*)&tmK2 : (const void*)&tmK,
                              bar_kfull + s, c * 128 / G::ES, w.g, jk * kTile, w.b);
                }
                ++jk;
                progressed = true;
              }
            }
            if (jv < jk) {
              const int x = jt + jv, s = x % G::NS;
              if (mbar_test_wait(smem_u32(bar_vfree + s), ((x / G::NS) & 1) ^ 1)) {
                uint8_t* sv = smem + G::OFF_V + s * G::VBYTES;
                mbar_arrive_expect_tx(bar_vfull + s, G::VBYTES);
                xv_last = x;
#pragma unroll
                for (int c = 0; c < G::VCH; ++c)
                  tma_load_4d(sv + c * 16384, &tmV, bar_vfull + s, c * 128 / G::ES, w.g, jv * kTile, w.b);
                ++jv;
                progressed = true;
              }
            }
            if (progressed) {
              idle = 0;
            } else {
              // nothing to load yet: back off; give up after the time limit
              if (idle == 0) t0 = globaltimer_ns();
              ++idle;
              __nanosleep(32);
              if ((idle & 63u) == 0 && (*abort_flag || globaltimer_ns() - t0 > lim)) {
                ok = false;
                break;
              }
            }
          }
        }
        if (!ok) break;
        jt += w.n_kv;
        ++nq;
      }
      if (!ok) fail();
    }
  } else if (warp == kWarpMma) {
    // ------------------------------------------------------------ MMA issuer
    // tcgen05.mma issue runs nearly in step with execution, so this loop is
    // on the critical path.  The whole warp runs it, so that descriptors and
    // control stay warp-uniform; one elected lane issues every tcgen05 op
    // (the same lane each time: elect.sync picks the lowest active lane).
    if (!(DBG && (p.dbg_flags & 1))) {  // flag 1: withhold all work (test hook)
      const uint32_t sbase = smem_u32(smem);
      constexpr uint32_t idesc_qk = idesc_dense(DT == 0 ? 1u : 0u, 0u, 128, 128);
      constexpr uint32_t idesc_pv_bf16 = idesc_dense(1u, 1u, 128, DV);
      // descriptors of stage 0; stage s adds its byte offset >> 4 to the
      // 14-bit start-address field (all addresses stay below 256 KB)
      uint64_t dq[G::QK_STEPS], dk[G::QK_STEPS], dvv[G::PV_STEPS];
#pragma unroll
      for (int kk = 0; kk < G::QK_STEPS; ++kk) {
        const int pos = kk * 32;
        const int c = pos / 128;
        const bool narrow = (c == G::NCH - 1) && G::LASTW == 64;
        const uint32_t off = c * 16384 + (pos % 128);
        dq[kk] = smem_desc(sbase + G::OFF_Q + off, 16, narrow ? 512 : 1024, narrow ? SW_64B : SW_128B);
        dk[kk] = smem_desc(sbase + G::OFF_K + off, 16, narrow ? 512 : 1024, narrow ? SW_64B : SW_128B);
      }
#pragma unroll
      for (int kk = 0; kk < G::PV_STEPS; ++kk)  // 16 (bf16) or 32 (fp8) keys of V per step
        dvv[kk] = smem_desc(sbase + G::OFF_V + kk * (DT == 0 ? 16 : 32) * 128, 16384, 1024, SW_128B);
      auto wait_all = [&](uint64_t* bar, uint32_t parity) -> bool {
        return __all_sync(0xffffffffu, mbar_wait(bar, parity, lim, abort_flag));
      };
      // FP8: the second N atom (the ones block) sits at ONES - V_s, so the
      // descriptor's leading-offset field differs per stage (see voff below)
      // jg: the tile's place in the CTA's sequence (stage, buffer, parity);
      // j: its index inside the unit (accumulate flag, trace slot)
      uint64_t* trace = nullptr;
      auto issue_qk = [&](int jg, int j) -> bool {
        const int s = jg % G::NS;
        if (!wait_all(bar_kfull + s, (jg / G::NS) & 1)) return false;
        tc_fence_after();
        if (trace && lane == 0 && j < kTraceTiles) trace[j * kTraceSlots + 5] = clk64();
        const uint32_t dS = tbase + kColS0 + (jg & 1) * 128;
        const uint64_t koff = (uint64_t)((s * G::KBYTES) >> 4);
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < G::QK_STEPS; ++kk) {
            if (DT == 0)
              mma_f16_ss(dS, dq[kk], dk[kk] + koff, idesc_qk, kk > 0);
            else
              mma_f8_ss(dS, dq[kk], dk[kk] + koff, idesc_qk, kk > 0);
            if (trace && kk == 1 && j < kTraceTiles) trace[j * kTraceSlots + 13] = clk64();
          }
          if (kSplit) tc_commit(bar_kfree + s);
          tc_commit(bar_sfull + (jg & 1));
        }
        __syncwarp();
        if (trace && lane == 0 && j < kTraceTiles) trace[j * kTraceSlots + 6] = clk64();
        return true;
      };
      auto issue_pv = [&](int jg, int j) -> bool {
        const int s = jg % G::NS;
        if (!wait_all(bar_pfull + (jg & 1), (jg >> 1) & 1)) return false;
        if (kSplit && !wait_all(bar_vfull + s, (jg / G::NS) & 1)) return false;
        tc_fence_after();
        if (trace && lane == 0 && j < kTraceTiles) trace[j * kTraceSlots + 7] = clk64();
        uint64_t voff = (uint64_t)((s * G::VBYTES) >> 4);
        if (DT == 1) {  // replace LBO 16384 by ONES - V_s (both fit the 14-bit field)
          const uint32_t lbo = (uint32_t)(G::OFF_ONES - (G::OFF_V + s * G::VBYTES));
          voff += ((uint64_t)(lbo >> 4) << 16) - ((uint64_t)(16384u >> 4) << 16);
        }
        // P of keys [64h, 64h + 64) sits at the start of S half h
        const uint32_t aP = tbase + kColS0 + (jg & 1) * 128;
        if (elect_one()) {
          if (DT == 1 && BS)
            tmem_cp_32x128b_x4(tbase + kColSFA + (jg & 1) * 4,
                               smem_desc(sbase + G::OFF_SF + (jg & 1) * 512, 16, 128, SW_NONE));
          if (trace && j < kTraceTiles) trace[j * kTraceSlots + 8] = clk64();
#pragma unroll
          for (int kk = 0; kk < G::PV_STEPS; ++kk) {
            const uint32_t acc = (j > 0 || kk > 0) ? 1u : 0u;
            if (DT == 0) {
              // 16 keys per step = 8 packed bf16x2 columns of P
              mma_f16_ts(tbase + kColO, aP + (kk >> 2) * 64 + (kk & 3) * 8, dvv[kk] + voff, idesc_pv_bf16, acc);
            } else {
              // 32 keys per step = 8 columns of 4 x e4m3; scale byte kk
              // N = d_v + 16: V and the ones block in one instruction
              const uint32_t sfa = (tbase + kColSFA + (jg & 1) * 4) | ((uint32_t)kk << 30);
              const uint32_t sfb = (tbase + kColSFB) | ((uint32_t)kk << 30);
              mma_mxf8_ts(tbase + kColO, aP + (kk >> 1) * 64 + (kk & 1) * 8, dvv[kk] + voff,
                          idesc_mx(1u, 128, DV + 16, kk, kk), sfa, sfb, acc);
            }
            if (trace && kk == 1 && j < kTraceTiles) trace[j * kTraceSlots + 14] = clk64();
          }
          if (trace && j < kTraceTiles) trace[j * kTraceSlots + 9] = clk64();
          tc_commit(bar_vfree + s);
        }
        __syncwarp();
        if (trace && lane == 0 && j < kTraceTiles) trace[j * kTraceSlots + 10] = clk64();
        return true;
      };
      int jt = 0, nq = 0;
      bool ok = true;
      for (int k = 0, u = unit_at(0); ok && u < n_units; u = PERSIST ? unit_at(++k) : n_units) {
        const Unit w = unit_of(p, u);
        if (w.n_kv == 0) continue;
        trace = traced_unit(w) ? trace_buf : nullptr;
        if (!wait_all(bar_q, nq & 1)) { ok = false; break; }
        for (int j = 0; j < w.n_kv; ++j) {
          if (!issue_qk(jt + j, j)) { ok = false; break; }
          if (j == w.n_kv - 1) {
            // the unit's last QK: Q may be replaced once it completes
            if (elect_one()) tc_commit(bar_qfree);
            __syncwarp();
          }
          if (j == 1 && nq > 0) {
            // PV_0 overwrites O: the softmax must have read the last unit's
            if (!wait_all(bar_ofree, (nq - 1) & 1)) { ok = false; break; }
          }
          if (j > 0 && !issue_pv(jt + j - 1, j - 1)) { ok = false; break; }
        }
        if (!ok) break;
        if (w.n_kv == 1 && nq > 0 && !wait_all(bar_ofree, (nq - 1) & 1)) { ok = false; break; }
        if (!issue_pv(jt + w.n_kv - 1, w.n_kv - 1)) { ok = false; break; }
        if (elect_one()) tc_commit(bar_ofinal);
        __syncwarp();
        jt += w.n_kv;
        ++nq;
      }
      if (!ok && lane == 0) fail();
    }
  } else {
    // ------------------------------------------------------ softmax (rows)
    // Warps q and q + 4 share TMEM lane quarter q: warp q owns lanes
    // 32q..32q+15 and warp q + 4 lanes 32q+16..32q+31 (16x32bx2 accesses).
    // Inside a warp, threads t and t + 16 own the same query row: thread t
    // takes keys [0, 64) of every tile, thread t + 16 keys [64, 128) -- one
    // 64-key scale block each -- and the two agree on the row's reference
    // with one shuffle.  P of keys [64h, 64h + 64) goes over the first
    // columns of S half h, which only this thread pair reads.
    const int qd = warp & 3, sub = warp >> 2;
    const int half = lane >> 4;
    const int row = qd * 32 + sub * 16 + (lane & 15);  // query row == TMEM lane
    const uint32_t col_h = (uint32_t)half * 64;
    const uint32_t lane_off = (uint32_t)(qd * 32 + sub * 16) << 16;  // 16-lane group
    constexpr unsigned kFull = 0xffffffffu;
    float c = p.softmax_scale * 1.4426950408889634f;  // log2(e); FP8: set per unit
    float vscale = 1.0f;
    if (DT == 1) {
      if (sub == 0) {
        // SFB (scales of V and of the ones matrix): all 2^0 = 0x7F; warp q
        // writes all 32 lanes of its quarter
        const uint32_t q_off = (uint32_t)(qd * 32) << 16;
        tmem_st4(tbase + q_off + kColSFB, 0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu);
        tmem_st4(tbase + q_off + kColSFB + 4, 0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu);
        if (!BS) {  // running mode: every block scale is 2^0 as well
          tmem_st4(tbase + q_off + kColSFA, 0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu);
          tmem_st4(tbase + q_off + kColSFA + 4, 0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu);
        }
        tmem_st_wait();
      }
    }
    const int T = p.headroom_T;
    float yref = -INFINITY;   // BF16 / FP8 running mode: log2-domain reference
    int eref = kInvalidExp;   // FP8: reference exponent E (invalid until a key is seen)
    float l = 0.0f;           // BF16: this thread's half of the row sum (fp32, unrounded p)
    bool ok = true;
    int jt = 0, nq = 0;       // key tiles and units with work so far (as the MMA warp counts)

    // O holds tiles < j at the old reference: rescale this thread's 64 O
    // columns by f once PV_{j-1} has landed (rare: the reference is lazy)
    auto rescale_o = [&](int jg, float f) -> bool {
      const bool w2 = mbar_wait(bar_vfree + (jg - 1) % G::NS, ((jg - 1) / G::NS) & 1, lim, abort_flag);
      if (!__all_sync(kFull, w2)) return false;
      tc_fence_after();
#pragma unroll 1
      for (int ch = 0; ch < 2; ++ch) {
        uint32_t o[32];
        const uint32_t to = tbase + lane_off + kColO + ch * 32;
        tmem_ld16x2_32<64>(to, o);
        tmem_ld_wait();
#pragma unroll
        for (int q = 0; q < 32; ++q) o[q] = __float_as_uint(__uint_as_float(o[q]) * f);
        tmem_st16x2_32<64>(to, o);
      }
      if (DT == 1) {
        // all 16 row-sum columns hold the same sum: half 0 keeps column RS,
        // half 1 column RS + 1
        uint32_t rs;
        tmem_ld16x2_1<1>(tbase + lane_off + kColRS, rs);
        tmem_ld_wait();
        tmem_st16x2_1<1>(tbase + lane_off + kColRS, __float_as_uint(__uint_as_float(rs) * f));
      }
      return true;
    };

    for (int k = 0, u = unit_at(0); ok && u < n_units; u = PERSIST ? unit_at(++k) : n_units) {
    const Unit wu = unit_of(p, u);
    const int n_kv = wu.n_kv, min_lim = wu.min_lim, b = wu.b, h = wu.h;
    const bool traced = traced_unit(wu);
    uint64_t* const trace = traced ? trace_buf : nullptr;
    const int i = wu.q0 + row;
    const int row_lim = p.causal ? min(i + shift, p.Sk - 1) : p.Sk - 1;
    yref = -INFINITY;
    eref = kInvalidExp;
    l = 0.0f;
    if (DT == 1) {
      // dequantisation scales of this unit's (batch, kv head), or the
      // per-tensor ones; the score scale folds q and k descales and log2(e)
      const int di = p.descale_per_kv ? b * p.Hkv + wu.g : 0;
      const float qds = p.q_descale ? p.q_descale[di] : 1.0f;
      const float kds = p.k_descale ? p.k_descale[di] : 1.0f;
      vscale = p.v_descale ? p.v_descale[di] : 1.0f;
      c = ((p.softmax_scale * qds) * kds) * 1.4426950408889634f;
    }
    for (int j = 0; ok && j < n_kv; ++j) {
      const int jg = jt + j;
      const int buf = jg & 1;
      const bool w = mbar_wait(bar_sfull + buf, (jg >> 1) & 1, lim, abort_flag);
      if (!__all_sync(kFull, w)) { ok = false; break; }
      tc_fence_after();
      if (trace && warp == 0 && lane == 0 && j < kTraceTiles) trace[j * kTraceSlots + 0] = clk64();
      float s[64];  // explicit bit casts: no type punning through pointers
      {
        uint32_t a0[32], a1[32];
        const uint32_t ts = tbase + lane_off + kColS0 + buf * 128;
        tmem_ld16x2_32<64>(ts, a0);
        tmem_ld16x2_32<64>(ts + 32, a1);
        tmem_ld_wait_regs(a0, a1);
#pragma unroll
        for (int cc = 0; cc < 32; ++cc) {
          s[cc] = __uint_as_float(a0[cc]);
          s[32 + cc] = __uint_as_float(a1[cc]);
        }
      }
      if (trace && warp == 0 && lane == 0 && j < kTraceTiles) trace[j * kTraceSlots + 1] = clk64();
      const bool dump = traced && j == 0;
      if (dump) {
        float* ds = static_cast<float*>(p.dbg) + row * 128 + col_h;
#pragma unroll
        for (int cc = 0; cc < 64; ++cc) ds[cc] = s[cc];
      }
      const int kbase = j * kTile + (int)col_h;
      if (kbase + 63 > min_lim) {
#pragma unroll
        for (int cc = 0; cc < 64; ++cc)
          if (kbase + cc > row_lim) s[cc] = -INFINITY;
      }
      const float m = max64(s);  // raw block maximum
      const uint32_t tP = tbase + lane_off + kColS0 + buf * 128;

      if constexpr (DT == 0) {
        // ------------------------------------------------ BF16, exact exp2
        const float ym = m * c;
        const float ymax = fmaxf(ym, __shfl_xor_sync(kFull, ym, 16));  // the row's maximum
        if (__builtin_expect(__any_sync(kFull, ymax > yref + 8.0f), 0)) {
          const float nref = fmaxf(yref, ymax);
          const float f = (nref == -INFINITY || yref == nref) ? 1.0f : ex2_approx(yref - nref);
          yref = nref;
          l *= f;
          if (j > 0 && !rescale_o(jg, f)) { ok = false; break; }
        }
        const float nb = yref == -INFINITY ? 0.0f : -yref;
        uint32_t pk[32];
        float lp0 = 0.0f, lp1 = 0.0f;
#pragma unroll
        for (int cc = 0; cc < 64; cc += 2) {
          float z0, z1, p0, p1;
          ffma2(z0, z1, s[cc], s[cc + 1], c, nb);
          if ((cc & 6) == 0) {  // a quarter of the pairs on the FMA pipe
            exp2_poly_x2<3>(p0, p1, z0, z1);
          } else {
            p0 = ex2_approx(z0);
            p1 = ex2_approx(z1);
          }
          lp0 += p0;
          lp1 += p1;
          pk[cc / 2] = pack_bf16x2(p0, p1);
        }
        l += lp0 + lp1;
        if (trace && warp == 0 && lane == 0 && j < kTraceTiles) trace[j * kTraceSlots + 2] = clk64();
        tmem_st16x2_32<64>(tP, pk);
        if (dump) {
          uint32_t* dp = static_cast<uint32_t*>(p.dbg) + 128 * 128;
#pragma unroll
          for (int q = 0; q < 32; ++q) dp[row * 64 + half * 32 + q] = pk[q];
        }
      } else {
        // ------------------------------------------------ FP8 P path
        // e: this thread's block exponent; the row's reference E (eref)
        // moves only when a block exceeds it by more than 32 (block scale),
        // or follows the running maximum (running mode: one exponent per row)
        int e, nref;
        if (BS) {
          e = m != -INFINITY ? (int)ceilf(m * c) - T : kInvalidExp;
          nref = next_ref(eref, max(e, __shfl_xor_sync(kFull, e, 16)), 32);
        } else {
          const float ym = m * c;
          yref = fmaxf(yref, fmaxf(ym, __shfl_xor_sync(kFull, ym, 16)));
          nref = yref != -INFINITY ? (int)ceilf(yref) - T : kInvalidExp;
          e = nref;  // the row's exponent for both blocks
        }
        const bool grow = eref > kInvalidExp && nref != eref;
        if (__builtin_expect(j > 0 && __any_sync(kFull, grow), 0)) {
          // O and the row sum hold tiles < j at scale 2^(-eref): move them
          // to 2^(-nref) exactly
          if (!rescale_o(jg, grow ? pow2i(max(eref - nref, -126)) : 1.0f)) { ok = false; break; }
        }
        eref = nref;
        const bool v = e > kInvalidExp;
        uint32_t pk[16];
        if (MODE == 0) {
          // exact: e4m3_rne(exp2(y - e))
          const float ne = v ? -(float)e : 0.0f;
#pragma unroll
          for (int cc = 0; cc < 64; cc += 4) {
            float z0, z1, z2, z3, p0, p1;
            ffma2(z0, z1, s[cc], s[cc + 1], c, ne);
            ffma2(z2, z3, s[cc + 2], s[cc + 3], c, ne);
            if ((cc & 4) == 0) {
              exp2_poly_x2<4>(p0, p1, z0, z1);  // a quarter of the values on the FMA pipe
            } else {
              p0 = ex2_approx(z0);
              p1 = ex2_approx(z1);
            }
            pk[cc / 4] = pack_e4m3x4(p0, p1, ex2_approx(z2), ex2_approx(z3));
          }
        } else {
          // Lean P: u = sat((8(y - e) + 56) / 128) clamps the code at 0; the
          // magic add 1.5*2^23 rounds 128u half-to-even into the low byte.
          const float a = c * 0.0625f;  // 8c / 128
          const float magic = 12582912.0f;
          const float k0 = v ? (float)(56 - 8 * e) * 0.0078125f : 0.0f;
#pragma unroll
          for (int cc = 0; cc < 64; cc += 4) {
            const float u0 = fma_sat(s[cc], a, k0);
            const float u1 = fma_sat(s[cc + 1], a, k0);
            const float u2 = fma_sat(s[cc + 2], a, k0);
            const float u3 = fma_sat(s[cc + 3], a, k0);
            float x0, x1, x2, x3;
            ffma2(x0, x1, u0, u1, 128.0f, magic);
            ffma2(x2, x3, u2, u3, 128.0f, magic);
            pk[cc / 4] = prmt(prmt(__float_as_uint(x0), __float_as_uint(x1), 0x0040u),
                              prmt(__float_as_uint(x2), __float_as_uint(x3), 0x0040u), 0x5410u);
          }
        }
        if (trace && warp == 0 && lane == 0 && j < kTraceTiles) trace[j * kTraceSlots + 2] = clk64();
        tmem_st16x2_16<64>(tP, pk);
        const int sf = v ? min(max(e - eref + 127, 0), 254) : 0;
        if (BS) {
          // bytes 2h, 2h+1 of the row's word: K32 chunks 2h and 2h+1
          reinterpret_cast<uint16_t*>(sf_smem + buf * 128 + (row & 31) * 4 + (row >> 5))[half] =
              (uint16_t)(sf * 0x0101u);
          fence_proxy_async_smem();
        }
        if (dump) {
          uint32_t* dp = static_cast<uint32_t*>(p.dbg) + 128 * 128;
#pragma unroll
          for (int q = 0; q < 16; ++q) dp[row * 64 + half * 16 + q] = pk[q];
          dp[128 * 64 + half * 128 + row] = (uint32_t)sf * 0x01010101u;
        }
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar_pfull + buf);
      if (trace && j < kTraceTiles && lane == 0) {
        if (warp == 0) trace[j * kTraceSlots + 3] = clk64();
        if (warp == 3) trace[j * kTraceSlots + 4] = clk64();
        if (warp == 1) trace[j * kTraceSlots + 11] = clk64();
        if (warp == 5) trace[j * kTraceSlots + 12] = clk64();
      }
    }
    if (!ok) break;
    {
      // ------------------------------------------------------------ epilogue
      bool wok = true;
      if (n_kv > 0) wok = __all_sync(kFull, mbar_wait(bar_ofinal, nq & 1, lim, abort_flag));
      if (!wok) {
        ok = false;
        break;
      }
      tc_fence_after();
      // O and the row sum into registers, then hand O back to the MMA warp
      // (the next unit's first PV overwrites it) before the stores
      uint32_t o[64];
      float L = 0.0f, lse_v = -INFINITY;
      if (n_kv > 0) {
        tmem_ld16x2_32<64>(tbase + lane_off + kColO, *reinterpret_cast<uint32_t(*)[32]>(o));
        tmem_ld16x2_32<64>(tbase + lane_off + kColO + 32, *reinterpret_cast<uint32_t(*)[32]>(o + 32));
        uint32_t rs = 0u;
        if (DT == 1) tmem_ld16x2_1<1>(tbase + lane_off + kColRS, rs);  // columns RS / RS + 1: equal
        tmem_ld_wait_regs(*reinterpret_cast<uint32_t(*)[32]>(o), *reinterpret_cast<uint32_t(*)[32]>(o + 32));
        asm volatile("" : "+r"(rs)::"memory");  // rs, too, is read only after the wait
        if (DT == 1) L = __uint_as_float(rs);
        tc_fence_before();
        mbar_arrive(bar_ofree);
      } else {
#pragma unroll
        for (int q = 0; q < 64; ++q) o[q] = 0u;
      }
      if (DT == 0) L = l + __shfl_xor_sync(kFull, l, 16);  // same value in both halves
      // no visible key: L == 0 (FP8), or the reference never left -inf (BF16;
      // the software exp2 maps masked scores to ~2^-126 instead of 0)
      const bool empty = !(L > 0.0f) || (DT == 0 && yref == -INFINITY);
      const float inv = empty ? 0.0f : vscale / L;
      if (!empty) {
        const float ref = DT == 0 ? yref : (float)eref;
        lse_v = (ref + __log2f(L)) * 0.6931471805599453f;
      }
      if (i < p.Sq) {
        uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) +
                                              (((int64_t)b * p.Sq + i) * p.Hq + h) * DV + col_h);
#pragma unroll
        for (int q = 0; q < 8; ++q)
          dst[q] = make_uint4(pack_bf16x2(__uint_as_float(o[8 * q]) * inv, __uint_as_float(o[8 * q + 1]) * inv),
                              pack_bf16x2(__uint_as_float(o[8 * q + 2]) * inv, __uint_as_float(o[8 * q + 3]) * inv),
                              pack_bf16x2(__uint_as_float(o[8 * q + 4]) * inv, __uint_as_float(o[8 * q + 5]) * inv),
                              pack_bf16x2(__uint_as_float(o[8 * q + 6]) * inv, __uint_as_float(o[8 * q + 7]) * inv));
        if (half == 0 && p.lse) p.lse[((int64_t)b * p.Hq + h) * p.Sq + i] = lse_v;
      }
    }
    jt += n_kv;
    if (n_kv > 0) ++nq;
    }  // units
    if (!ok && lane == 0) fail();
    // no tensor-memory access of this thread is still in flight
    tmem_ld_wait();
    tmem_st_wait();
  }

  tc_fence_before();
  __syncthreads();
  if (*abort_flag) {
    // Some role gave up (a wait ran out): asynchronous work already issued
    // lands before the CTA frees its tensor memory and exits.  Each waits
    // again at most the time limit.
    if (warp == kWarpProducer && lane == 0) {
      // every TMA load into shared memory: a barrier's last armed phase
      // completes only once all its bytes arrived (earlier phases of the
      // same barrier were consumed before it was re-armed)
      if (q_loads > 0) mbar_wait_bounded(bar_q, (q_loads - 1) & 1, lim);
      for (int x = max(x_last - G::NS + 1, 0); x <= x_last; ++x)
        mbar_wait_bounded(bar_kfull + x % G::NS, (x / G::NS) & 1, lim);
      for (int x = max(xk_last - G::NS + 1, 0); x <= xk_last; ++x)
        mbar_wait_bounded(bar_kfull + x % G::NS, (x / G::NS) & 1, lim);
      for (int x = max(xv_last - G::NS + 1, 0); x <= xv_last; ++x)
        mbar_wait_bounded(bar_vfull + x % G::NS, (x / G::NS) & 1, lim);
    }
    if (warp == kWarpMma) {
      // every MMA and scale copy the issuing lane started
      if (elect_one()) tc_commit(bar_drain);
      __syncwarp();
      mbar_wait_bounded(bar_drain, 0, lim);
    }
    __syncthreads();
  }
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc(tbase, kTmemCols);
  }
}

// Evaluates the software exp2 (degree 3 or 4), CUDA's exp2f (degree 0) or
// the MUFU ex2.approx (degree -1) elementwise, for the test of the polynomial.
__global__ void exp2_check_kernel(const float* __restrict__ x, float* __restrict__ y, int64_t n,
                                  int degree) {
  const int64_t i0 = 2 * ((int64_t)blockIdx.x * blockDim.x + threadIdx.x);
  if (i0 >= n) return;
  const float a = x[i0], b = i0 + 1 < n ? x[i0 + 1] : 0.0f;
  float r0, r1;
  if (degree == 3) {
    exp2_poly_x2<3>(r0, r1, a, b);
  } else if (degree == 4) {
    exp2_poly_x2<4>(r0, r1, a, b);
  } else if (degree == 0) {
    r0 = exp2f(a);
    r1 = exp2f(b);
  } else {
    r0 = ex2_approx(a);
    r1 = ex2_approx(b);
  }
  y[i0] = r0;
  if (i0 + 1 < n) y[i0 + 1] = r1;
}

cudaError_t launch_exp2_check(const float* x, float* y, int64_t n, int degree, cudaStream_t st) {
  const int64_t pairs = (n + 1) / 2;
  const unsigned blocks = (unsigned)((pairs + 255) / 256);
  if (blocks == 0) return cudaSuccess;
  exp2_check_kernel<<<blocks, 256, 0, st>>>(x, y, n, degree);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ host side

template <int DT, int DQK, int DV, int MODE, int BS>
static cudaError_t launch_variant(const AttnLaunch& a, cudaStream_t st) {
  using G = Geo<DT, DQK, DV>;
  CUtensorMap mQ, mQ2, mK, mK2, mV;
  const int es = G::ES;
  const auto& p = a.p;
  if (!make_map(&mQ, a.q, es, p.B, p.Sq, p.Hq, DQK, 128 / es, CU_TENSOR_MAP_SWIZZLE_128B, kTile) ||
      !make_map(&mK, a.k, es, p.B, p.Sk, p.Hkv, DQK, 128 / es, CU_TENSOR_MAP_SWIZZLE_128B, kTile) ||
      !make_map(&mV, a.v, es, p.B, p.Sk, p.Hkv, DV, 128 / es, CU_TENSOR_MAP_SWIZZLE_128B, kTile))
    return cudaErrorInvalidValue;
  if (G::LASTW == 64) {
    if (!make_map(&mQ2, a.q, es, p.B, p.Sq, p.Hq, DQK, 64 / es, CU_TENSOR_MAP_SWIZZLE_64B, kTile) ||
        !make_map(&mK2, a.k, es, p.B, p.Sk, p.Hkv, DQK, 64 / es, CU_TENSOR_MAP_SWIZZLE_64B, kTile))
      return cudaErrorInvalidValue;
  } else {
    mQ2 = mQ;
    mK2 = mK;
  }
  const long long n_units = (long long)p.n_qtiles * p.B * p.Hq;
  if (n_units <= 0) return cudaSuccess;
  if (n_units > 0x7fffffffLL) return cudaErrorInvalidValue;
  // persistent CTAs (one per SM) for short sequences, else one CTA per
  // unit from the one-unit instantiation (schedule.h)
  const bool persist = use_persistent(p.n_qtiles);
  int sms = 0;
  if (persist) {
    int dev = 0;
    cudaError_t e0 = cudaGetDevice(&dev);
    if (e0 == cudaSuccess) e0 = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e0 != cudaSuccess) return e0;
  }
  const long long nblocks = grid_size(p.n_qtiles, n_units, sms);
  auto kern = p.dbg ? (persist ? attn_fwd_kernel<DT, DQK, DV, MODE, BS, 1, 1> : attn_fwd_kernel<DT, DQK, DV, MODE, BS, 1, 0>)
                    : (persist ? attn_fwd_kernel<DT, DQK, DV, MODE, BS, 0, 1> : attn_fwd_kernel<DT, DQK, DV, MODE, BS, 0, 0>);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, G::SMEM);
  if (e != cudaSuccess) return e;
  kern<<<(unsigned)nblocks, kThreads, G::SMEM, st>>>(mQ, mQ2, mK, mK2, mV, p);
  return cudaGetLastError();
}

int attn_smem_bytes(int dtype, int dqk) {
  if (dtype == 0) return dqk == 128 ? Geo<0, 128, 128>::SMEM : Geo<0, 192, 128>::SMEM;
  return dqk == 128 ? Geo<1, 128, 128>::SMEM : Geo<1, 192, 128>::SMEM;
}

int attn_threads() { return kThreads; }

cudaError_t launch_attention(const AttnLaunch& a, cudaStream_t st) {
  if (use_pair_kernel(a.dtype, a.dqk, a.p.n_qtiles)) return launch_attention_pp(a, st);
  if (a.dtype == 0) {
    if (a.dqk == 128) return launch_variant<0, 128, 128, 0, 0>(a, st);
    return launch_variant<0, 192, 128, 0, 0>(a, st);
  }
  if (a.dqk == 128) {
    if (a.mode == 1) return a.block_scale ? launch_variant<1, 128, 128, 1, 1>(a, st)
                                          : launch_variant<1, 128, 128, 1, 0>(a, st);
    return a.block_scale ? launch_variant<1, 128, 128, 0, 1>(a, st)
                         : launch_variant<1, 128, 128, 0, 0>(a, st);
  }
  if (a.mode == 1) return a.block_scale ? launch_variant<1, 192, 128, 1, 1>(a, st)
                                        : launch_variant<1, 192, 128, 1, 0>(a, st);
  return a.block_scale ? launch_variant<1, 192, 128, 0, 1>(a, st)
                       : launch_variant<1, 192, 128, 0, 0>(a, st);
}

}  // namespace zq
