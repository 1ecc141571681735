// attn_pp.cu -- BF16 causal forward (prefill) attention for sm_100a, head
// dims (128, 128), with two 128-row query tiles per CTA.
//
// Same method as the BF16 path of attn_fwd.cu ([P3] "Zyphra ZYFA ... FP8
// FlashAttention for AMD MI355X" (ai4bro.com), TL;DR: causal prefill in
// BF16 and FP8, d 128): softmax(Q K^T * scale) V with an exact exp2 and a
// lazily moved row reference, the row sum in fp32 over the unrounded
// probabilities.  What differs is the schedule on the SM (measured faster
// for BF16 at d = 128 with more than 64 query tiles, where every CTA runs one
// unit; slower for FP8, whose softmax is shorter than its MMA issue chain,
// for d_qk = 192 and for short sequences, which attn_fwd.cu keeps):
//
//   * A unit is a pair of consecutive query tiles (PairUnit, schedule.h);
//     the grid has one CTA per unit.
//     Each tile has its own softmax team of four warps, one thread per query
//     row, and its own MMA issuer warp, so that one team's softmax runs while
//     the tensor core works on the other team's tiles.  The two teams share
//     every K/V tile.
//   * Keys come in tiles of 64, so a thread holds 64 scores of its row per
//     tile and the row's reference needs no exchange between threads.
//   * P has TMEM buffers of its own (two per team), so the score buffer is
//     free for the next QK as soon as the team has loaded it.
//
// Warps:
//   0-3   team 0 (query rows 2tp*128 + 32q + lane, TMEM lane quarter q = warp)
//   4-7   team 1 (rows (2tp+1)*128 + ..., quarter q = warp - 4)
//   8     TMA producer: Q of each team per unit, then (K_j, V_j) stages
//   9, 10 tcgen05 issuers of teams 0 and 1 (warp 9 also owns the TMEM
//         allocation); each issues in order QK_0, QK_1, PV_0, QK_2, PV_1, ...
// Tensor memory (512 columns), per team t:
//   S_t   [64t, 64t + 64)          scores of the current key tile (fp32)
//   O_t   [128 + 128t, +128)       output accumulator (fp32)
//   P_t,b [384 + 32(2t+b), +32)    P of the key tiles with parity b (bf16x2)
#include "attn_math.cuh"
#include "schedule.h"
#include "sm100_ptx.cuh"
#include "zq_internal.h"

namespace zq {

constexpr int kPPSoftmaxThreads = 256;
constexpr int kPPThreads = kPPSoftmaxThreads + 96;
constexpr int kPPWarpProducer = 8, kPPWarpIssuer0 = 9;
constexpr int kPPTeamThreads = 128;
constexpr uint32_t kPPTmemCols = 512;

struct GeoPP {
  static constexpr int D = 128;                          // d_qk = d_v
  static constexpr int KT = kPairKeyTile;                // keys per key tile
  static constexpr int ROW = D * 2;                      // bytes per bf16 row
  static constexpr int NCH = ROW / 128;                  // 128-byte chunks per row
  static constexpr int QBYTES = kTile * ROW;             // one Q tile; chunk c at c * 16 KB
  static constexpr int KBYTES = KT * ROW;                // one K tile; chunk c at c * 8 KB
  static constexpr int VBYTES = KT * ROW;                // one V tile; chunk c at c * 8 KB
  static constexpr int STAGE = KBYTES + VBYTES;          // K_j then V_j
  static constexpr int QK_STEPS = ROW / 32;              // 16 channels of K per MMA
  static constexpr int PV_STEPS = KT / 16;               // 16 keys per MMA
  static constexpr int NS = 5;                           // K/V stages
  static constexpr int OFF_Q = 0;                        // team t at t * QBYTES
  static constexpr int OFF_KV = 2 * QBYTES;
  static constexpr int OFF_BAR = OFF_KV + NS * STAGE;
  static constexpr int NBAR = 2 + 2 + 2 * NS + 2 + 2 + 4 + 2 + 2 + 2 + 1;
  static constexpr int SMEM = OFF_BAR + NBAR * 8 + 16 + 1024;  // + alignment slack
  __host__ __device__ static constexpr uint32_t col_s(int t) { return 64u * t; }
  __host__ __device__ static constexpr uint32_t col_o(int t) { return 128u + 128u * t; }
  __host__ __device__ static constexpr uint32_t col_p(int t, int b) { return 384u + 32u * (2 * t + b); }
  static_assert(384 + 4 * 32 <= kPPTmemCols, "tensor memory has 512 columns");
  static_assert(SMEM <= 232448, "227 KB of shared memory per CTA");
  static_assert(QBYTES % 1024 == 0 && STAGE % 1024 == 0 && KBYTES % 1024 == 0, "1 KB aligned tiles");
};

// Debug trace of the traced tile (clock64), per key tile j, 8 slots at
// (j * 2 + team) * 8: [0] S_j seen (warp 0 of the team, lane 0) [1] S_j
// loaded [2] P_j computed [3] P_j released; issuer: [4] QK_j issue starts
// [5] QK_j committed [6] P_j seen [7] PV_j committed.  After the S/P dump.
constexpr int kPPTraceOffsetWords = 128 * 128 + 128 * 64 + 256;
constexpr int kPPTraceTiles = 512;  // 512 tiles x 2 teams x 8 slots = the 512 x 16 trace area

template <int DBG>
__global__ void __launch_bounds__(kPPThreads, 1)
    attn_pp_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const AttnParams p) {
  using G = GeoPP;
  constexpr int NS = G::NS;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + G::OFF_BAR);
  uint64_t* bar_q = bars;                    // [2] Q_t landed
  uint64_t* bar_qfree = bars + 2;            // [2] the unit's last QK_t done: Q_t reusable
  uint64_t* bar_kvfull = bars + 4;           // [NS] K_j and V_j landed
  uint64_t* bar_kvfree = bar_kvfull + NS;    // [NS] both teams done with the stage (2 arrivals)
  uint64_t* bar_sfull = bar_kvfree + NS;     // [2] QK_t(j) done
  uint64_t* bar_sfree = bar_sfull + 2;       // [2] team t loaded S_t(j) (128 arrivals)
  uint64_t* bar_pfull = bar_sfree + 2;       // [2][2] team t wrote P_t(j) into buffer j & 1
  uint64_t* bar_pvdone = bar_pfull + 4;      // [2] PV_t(j) done
  uint64_t* bar_ofinal = bar_pvdone + 2;     // [2] the unit's last PV_t done
  uint64_t* bar_ofree = bar_ofinal + 2;      // [2] team t read O_t of a unit (128 arrivals)
  uint64_t* bar_drain = bar_ofree + 2;       // [1] after an abort: both issuers' work landed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + G::NBAR);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n_units = n_pairs_of(p.n_qtiles) * p.B * p.Hq;
  // one unit per CTA; the role loops below run over it once, and their
  // barrier phase counters would carry over unchanged to further units
  const int u0 = (int)blockIdx.x;
  const int shift = p.Sk - p.Sq;
  // the traced 128-row tile (dbg_bh, dbg_t) is team dbg_t & 1 of pair dbg_t / 2
  auto traced_team = [&](const PairUnit& w) -> int {
    if (!(DBG && p.dbg != nullptr) || w.bh != p.dbg_bh || w.tp != (p.dbg_t >> 1)) return -1;
    return p.dbg_t & 1;
  };
  uint64_t* const trace_buf =
      DBG && p.dbg ? reinterpret_cast<uint64_t*>(static_cast<uint32_t*>(p.dbg) + kPPTraceOffsetWords) : nullptr;

  if (threadIdx.x == 0) {
    for (int t = 0; t < 2; ++t) {
      mbar_init(bar_q + t, 1);
      mbar_init(bar_qfree + t, 1);
      mbar_init(bar_sfull + t, 1);
      mbar_init(bar_sfree + t, kPPTeamThreads);
      mbar_init(bar_pfull + 2 * t, kPPTeamThreads);
      mbar_init(bar_pfull + 2 * t + 1, kPPTeamThreads);
      mbar_init(bar_pvdone + t, 1);
      mbar_init(bar_ofinal + t, 1);
      mbar_init(bar_ofree + t, kPPTeamThreads);
    }
    for (int s = 0; s < NS; ++s) {
      mbar_init(bar_kvfull + s, 1);
      mbar_init(bar_kvfree + s, 2);
    }
    mbar_init(bar_drain, 2);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kPPWarpIssuer0) {
    tmem_alloc(tmem_slot, kPPTmemCols);
    tmem_relinquish();
  }
  if (warp == kPPWarpProducer && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;
  const uint64_t lim = p.timeout_ns;

  // producer: the last load armed on each barrier, for the drain after an abort
  int q_loads0 = 0, q_loads1 = 0, x_last = -1;

  auto fail = [&]() {
    *abort_flag = 1;
    if (p.status) atomicExch(p.status, -7 /* ZQ_ERR_TIMEOUT */);
  };

  if (warp == kPPWarpProducer) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int jkv = 0, nq0 = 0, nq1 = 0;
      bool ok = true;
      for (int u = u0; ok && u < n_units; u = n_units) {
        const PairUnit w = pair_of(p, u);
        if (w.n_kv_max == 0) continue;
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          if (!ok || w.n_kv[t] == 0) continue;
          const int nq = t ? nq1 : nq0;
          // Q_t of the previous unit is read until its last QK_t completes
          if (nq > 0 && !mbar_wait(bar_qfree + t, (nq - 1) & 1, lim, abort_flag)) { ok = false; break; }
          uint8_t* sq = smem + G::OFF_Q + t * G::QBYTES;
          mbar_arrive_expect_tx(bar_q + t, G::QBYTES);
#pragma unroll
          for (int c = 0; c < G::NCH; ++c) tma_load_4d(sq + c * 16384, &tmQ, bar_q + t, c * 64, w.h, w.q0[t], w.b);
          if (t) {
            ++nq1;
            ++q_loads1;
          } else {
            ++nq0;
            ++q_loads0;
          }
        }
        if (!ok) break;
        for (int j = 0; j < w.n_kv_max; ++j) {
          const int x = jkv + j, s = x % NS;
          // the stage is free once both teams are done with its last tile (first pass: free)
          if (!mbar_wait(bar_kvfree + s, ((x / NS) & 1) ^ 1, lim, abort_flag)) { ok = false; break; }
          uint8_t* sk = smem + G::OFF_KV + s * G::STAGE;
          uint8_t* sv = sk + G::KBYTES;
          mbar_arrive_expect_tx(bar_kvfull + s, G::STAGE);
          x_last = x;
#pragma unroll
          for (int c = 0; c < G::NCH; ++c) {
            tma_load_4d(sk + c * 8192, &tmK, bar_kvfull + s, c * 64, w.g, j * G::KT, w.b);
            tma_load_4d(sv + c * 8192, &tmV, bar_kvfull + s, c * 64, w.g, j * G::KT, w.b);
          }
        }
        jkv += w.n_kv_max;
      }
      if (!ok) fail();
    }
  } else if (warp > kPPWarpProducer) {
    // ------------------------------------------------------------ issuers
    // The whole warp runs the loop (descriptors and control stay
    // warp-uniform); one elected lane issues every tcgen05 op.
    const int t = warp - kPPWarpIssuer0;
    if (!(DBG && (p.dbg_flags & 1))) {  // flag 1: withhold all work (test hook)
      const uint32_t sbase = smem_u32(smem);
      constexpr uint32_t idesc_qk = idesc_dense(1u, 0u, 128, G::KT);
      constexpr uint32_t idesc_pv = idesc_dense(1u, 1u, 128, G::D);
      // descriptors of stage 0; stage s adds its byte offset >> 4 to the
      // 14-bit start-address field (all addresses stay below 256 KB)
      uint64_t dq[G::QK_STEPS], dk[G::QK_STEPS], dvv[G::PV_STEPS];
#pragma unroll
      for (int kk = 0; kk < G::QK_STEPS; ++kk) {
        const int pos = kk * 32, c = pos / 128;
        dq[kk] = smem_desc(sbase + G::OFF_Q + t * G::QBYTES + c * 16384 + pos % 128, 16, 1024, SW_128B);
        dk[kk] = smem_desc(sbase + G::OFF_KV + c * 8192 + pos % 128, 16, 1024, SW_128B);
      }
#pragma unroll
      for (int kk = 0; kk < G::PV_STEPS; ++kk)  // 16 keys of V per step; the two 64-column chunks 8 KB apart
        dvv[kk] = smem_desc(sbase + G::OFF_KV + G::KBYTES + kk * 16 * 128, 8192, 1024, SW_128B);
      auto wait_all = [&](uint64_t* bar, uint32_t parity) -> bool {
        return __all_sync(0xffffffffu, mbar_wait(bar, parity, lim, abort_flag));
      };
      const uint32_t dS = tbase + G::col_s(t);
      const uint32_t dO = tbase + G::col_o(t);
      uint64_t* trace = nullptr;
      // g: the team's tile count in this CTA (buffers, parities); x: the
      // CTA's K/V tile count (stage); j: index inside the unit
      auto issue_qk = [&](int g, int x, int j) -> bool {
        const int s = x % NS;
        if (!wait_all(bar_kvfull + s, (x / NS) & 1)) return false;
        if (g > 0 && !wait_all(bar_sfree + t, (g - 1) & 1)) return false;
        tc_fence_after();
        if (trace && lane == 0 && j < kPPTraceTiles) trace[(j * 2 + t) * 8 + 4] = clk64();
        const uint64_t koff = (uint64_t)((s * G::STAGE) >> 4);
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < G::QK_STEPS; ++kk) mma_f16_ss(dS, dq[kk], dk[kk] + koff, idesc_qk, kk > 0);
          tc_commit(bar_sfull + t);
        }
        __syncwarp();
        if (trace && lane == 0 && j < kPPTraceTiles) trace[(j * 2 + t) * 8 + 5] = clk64();
        return true;
      };
      auto issue_pv = [&](int g, int x, int j) -> bool {
        const int s = x % NS, b = g & 1;
        if (!wait_all(bar_pfull + 2 * t + b, (g >> 1) & 1)) return false;
        tc_fence_after();
        if (trace && lane == 0 && j < kPPTraceTiles) trace[(j * 2 + t) * 8 + 6] = clk64();
        const uint64_t voff = (uint64_t)((s * G::STAGE) >> 4);
        const uint32_t aP = tbase + G::col_p(t, b);
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < G::PV_STEPS; ++kk)  // 16 keys per step = 8 packed bf16x2 columns of P
            mma_f16_ts(dO, aP + kk * 8, dvv[kk] + voff, idesc_pv, (j > 0 || kk > 0) ? 1u : 0u);
          tc_commit(bar_pvdone + t);
          tc_commit(bar_kvfree + s);
        }
        __syncwarp();
        if (trace && lane == 0 && j < kPPTraceTiles) trace[(j * 2 + t) * 8 + 7] = clk64();
        return true;
      };
      int jt = 0, jkv = 0, nq = 0;
      bool ok = true;
      for (int u = u0; ok && u < n_units; u = n_units) {
        const PairUnit w = pair_of(p, u);
        if (w.n_kv_max == 0) continue;
        trace = traced_team(w) == t ? trace_buf : nullptr;
        const int n = t ? w.n_kv[1] : w.n_kv[0];  // (no dynamic index: keeps w in registers)
        if (n > 0) {
          if (!wait_all(bar_q + t, nq & 1)) { ok = false; break; }
          if (!issue_qk(jt, jkv, 0)) { ok = false; break; }
          if (n == 1) {
            if (elect_one()) tc_commit(bar_qfree + t);  // the unit's last QK_t
            __syncwarp();
          }
          for (int j = 0; j < n; ++j) {
            if (j + 1 < n) {
              if (!issue_qk(jt + j + 1, jkv + j + 1, j + 1)) { ok = false; break; }
              if (j + 2 == n) {
                if (elect_one()) tc_commit(bar_qfree + t);
                __syncwarp();
              }
            }
            // PV_t(0) overwrites O_t: the team must have read the last unit's
            if (j == 0 && nq > 0 && !wait_all(bar_ofree + t, (nq - 1) & 1)) { ok = false; break; }
            if (!issue_pv(jt + j, jkv + j, j)) { ok = false; break; }
          }
          if (!ok) break;
          if (elect_one()) tc_commit(bar_ofinal + t);
          __syncwarp();
          jt += n;
          ++nq;
        }
        // key tiles this team skips: release its share of their stages once loaded
        for (int j = n; j < w.n_kv_max; ++j) {
          const int x = jkv + j;
          if (!wait_all(bar_kvfull + x % NS, (x / NS) & 1)) { ok = false; break; }
          if (lane == 0) mbar_arrive(bar_kvfree + x % NS);
          __syncwarp();
        }
        if (!ok) break;
        jkv += w.n_kv_max;
      }
      if (!ok && lane == 0) fail();
    }
  } else {
    // ------------------------------------------------------ softmax teams
    const int t = warp >> 2, qd = warp & 3;
    const int row = qd * 32 + lane;  // query row in the team's tile == TMEM lane
    const uint32_t lane_off = (uint32_t)(qd * 32) << 16;
    const uint32_t tS = tbase + lane_off + G::col_s(t);
    const uint32_t tO = tbase + lane_off + G::col_o(t);
    constexpr unsigned kFull = 0xffffffffu;
    const float c = p.softmax_scale * 1.4426950408889634f;  // log2(e)
    float yref = -INFINITY;  // log2-domain reference of the row
    float l = 0.0f;          // the row sum (fp32, unrounded p)
    bool ok = true;
    int jt = 0, nq = 0;      // team tiles and units with work so far (as the issuer counts)

    // O_t holds tiles < j at the old reference: rescale this row by f once
    // PV_t(j - 1) has landed (rare: the reference is lazy).  bar_pvdone is in
    // phase j - 1 or j here: PV_t(j - 2) was issued before QK_t(j), whose
    // completion the caller saw, and PV_t(j) needs P_t(j), not yet written.
    auto rescale_o = [&](int g, float f) -> bool {
      const bool w2 = mbar_wait(bar_pvdone + t, (g - 1) & 1, lim, abort_flag);
      if (!__all_sync(kFull, w2)) return false;
      tc_fence_after();
#pragma unroll 1
      for (int ch = 0; ch < G::D / 32; ++ch) {
        uint32_t o[32];
        tmem_ld32_x32(tO + ch * 32, o);
        tmem_ld_wait_on(o);
#pragma unroll
        for (int q = 0; q < 32; ++q) o[q] = __float_as_uint(__uint_as_float(o[q]) * f);
        tmem_st32_x32(tO + ch * 32, o);
      }
      return true;
    };

    for (int u = u0; ok && u < n_units; u = n_units) {
      const PairUnit wu = pair_of(p, u);
      const int n = t ? wu.n_kv[1] : wu.n_kv[0], b = wu.b, h = wu.h;
      const int min_lim = t ? wu.min_lim[1] : wu.min_lim[0];
      const bool traced = traced_team(wu) == t;
      uint64_t* const trace = traced ? trace_buf : nullptr;
      const int i = (t ? wu.q0[1] : wu.q0[0]) + row;
      const int row_lim = p.causal ? min(i + shift, p.Sk - 1) : p.Sk - 1;
      yref = -INFINITY;
      l = 0.0f;
      for (int j = 0; ok && j < n; ++j) {
        const int g = jt + j;
        const int buf = g & 1;
        const bool w = mbar_wait(bar_sfull + t, g & 1, lim, abort_flag);
        if (!__all_sync(kFull, w)) { ok = false; break; }
        tc_fence_after();
        if (trace && qd == 0 && lane == 0 && j < kPPTraceTiles) trace[(j * 2 + t) * 8 + 0] = clk64();
        float s[64];
        {
          uint32_t a[64];
          tmem_ld32_x64(tS, a);
          tmem_ld_wait_on(a);
#pragma unroll
          for (int cc = 0; cc < 64; ++cc) s[cc] = __uint_as_float(a[cc]);
        }
        // S_t is free for QK_t(j + 1)
        tc_fence_before();
        mbar_arrive(bar_sfree + t);
        if (trace && qd == 0 && lane == 0 && j < kPPTraceTiles) trace[(j * 2 + t) * 8 + 1] = clk64();
        const bool dump = traced && j < 2;
        if (dump) {
          float* ds = static_cast<float*>(p.dbg) + row * 128 + j * 64;
#pragma unroll
          for (int cc = 0; cc < 64; ++cc) ds[cc] = s[cc];
        }
        const int kbase = j * G::KT;
        if (kbase + G::KT - 1 > min_lim) {
#pragma unroll
          for (int cc = 0; cc < 64; ++cc)
            if (kbase + cc > row_lim) s[cc] = -INFINITY;
        }
        const float ym = max64(s) * c;  // the block's maximum, log2 domain
        if (__builtin_expect(__any_sync(kFull, ym > yref + 8.0f), 0)) {
          const float nref = fmaxf(yref, ym);
          const float f = (nref == -INFINITY || yref == nref) ? 1.0f : ex2_approx(yref - nref);
          yref = nref;
          l *= f;
          if (j > 0 && !rescale_o(g, f)) { ok = false; break; }
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
        if (trace && qd == 0 && lane == 0 && j < kPPTraceTiles) trace[(j * 2 + t) * 8 + 2] = clk64();
        tmem_st32_x32(tbase + lane_off + G::col_p(t, buf), pk);
        if (dump) {
          uint32_t* dp = static_cast<uint32_t*>(p.dbg) + 128 * 128;
#pragma unroll
          for (int q = 0; q < 32; ++q) dp[row * 64 + j * 32 + q] = pk[q];
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(bar_pfull + 2 * t + buf);
        if (trace && qd == 0 && lane == 0 && j < kPPTraceTiles) trace[(j * 2 + t) * 8 + 3] = clk64();
      }
      if (!ok) break;
      {
        // ---------------------------------------------------------- epilogue
        float inv = 0.0f, lse_v = -INFINITY;
        if (n > 0) {
          // the unit's last PV_t (one phase of bar_ofinal per unit with work)
          const bool wok = mbar_wait(bar_ofinal + t, nq & 1, lim, abort_flag);
          if (!__all_sync(kFull, wok)) {
            ok = false;
            break;
          }
          tc_fence_after();
          // no visible key: the reference never left -inf (the software exp2
          // maps masked scores to ~2^-126, not 0)
          const bool empty = !(l > 0.0f) || yref == -INFINITY;
          inv = empty ? 0.0f : 1.0f / l;
          if (!empty) lse_v = (yref + __log2f(l)) * 0.6931471805599453f;
        }
        __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(p.out) + (((int64_t)b * p.Sq + i) * p.Hq + h) * G::D;
#pragma unroll 1
        for (int ch = 0; ch < 2; ++ch) {
          uint32_t o[64];
          if (n > 0) {
            tmem_ld32_x64(tO + ch * 64, o);
            tmem_ld_wait_on(o);
          } else {
#pragma unroll
            for (int q = 0; q < 64; ++q) o[q] = 0u;
          }
          if (ch == 1 && n > 0) {
            // O_t read: hand it back to the issuer (the next unit's PV_t(0))
            tc_fence_before();
            mbar_arrive(bar_ofree + t);
          }
          if (i < p.Sq) {
            uint4* dst = reinterpret_cast<uint4*>(orow + ch * 64);
#pragma unroll
            for (int q = 0; q < 8; ++q)
              dst[q] = make_uint4(pack_bf16x2(__uint_as_float(o[8 * q]) * inv, __uint_as_float(o[8 * q + 1]) * inv),
                                  pack_bf16x2(__uint_as_float(o[8 * q + 2]) * inv, __uint_as_float(o[8 * q + 3]) * inv),
                                  pack_bf16x2(__uint_as_float(o[8 * q + 4]) * inv, __uint_as_float(o[8 * q + 5]) * inv),
                                  pack_bf16x2(__uint_as_float(o[8 * q + 6]) * inv, __uint_as_float(o[8 * q + 7]) * inv));
          }
        }
        if (i < p.Sq && p.lse) p.lse[((int64_t)b * p.Hq + h) * p.Sq + i] = lse_v;
      }
      jt += n;
      if (n > 0) ++nq;
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
    if (warp == kPPWarpProducer && lane == 0) {
      if (q_loads0 > 0) mbar_wait_bounded(bar_q, (q_loads0 - 1) & 1, lim);
      if (q_loads1 > 0) mbar_wait_bounded(bar_q + 1, (q_loads1 - 1) & 1, lim);
      for (int x = max(x_last - NS + 1, 0); x <= x_last; ++x)
        mbar_wait_bounded(bar_kvfull + x % NS, (x / NS) & 1, lim);
    }
    if (warp > kPPWarpProducer) {
      // every MMA the issuing lanes started
      if (elect_one()) tc_commit(bar_drain);
      __syncwarp();
      mbar_wait_bounded(bar_drain, 0, lim);
    }
    __syncthreads();
  }
  if (warp == kPPWarpIssuer0) {
    tc_fence_after();
    tmem_dealloc(tbase, kPPTmemCols);
  }
}

bool use_pair_kernel(int dtype, int dqk, int n_qtiles) {
  return dtype == 0 && dqk == GeoPP::D && !use_persistent(n_qtiles);
}

int attn_pp_smem_bytes() { return GeoPP::SMEM; }

int attn_pp_threads() { return kPPThreads; }

cudaError_t launch_attention_pp(const AttnLaunch& a, cudaStream_t st) {
  using G = GeoPP;
  if (!use_pair_kernel(a.dtype, a.dqk, a.p.n_qtiles) || a.dv != G::D) return cudaErrorInvalidValue;
  const auto& p = a.p;
  CUtensorMap mQ, mK, mV;
  if (!make_map(&mQ, a.q, 2, p.B, p.Sq, p.Hq, G::D, 64, CU_TENSOR_MAP_SWIZZLE_128B, kTile) ||
      !make_map(&mK, a.k, 2, p.B, p.Sk, p.Hkv, G::D, 64, CU_TENSOR_MAP_SWIZZLE_128B, G::KT) ||
      !make_map(&mV, a.v, 2, p.B, p.Sk, p.Hkv, G::D, 64, CU_TENSOR_MAP_SWIZZLE_128B, G::KT))
    return cudaErrorInvalidValue;
  const long long n_units = (long long)n_pairs_of(p.n_qtiles) * p.B * p.Hq;
  if (n_units <= 0) return cudaSuccess;
  if (n_units > 0x7fffffffLL) return cudaErrorInvalidValue;
  const long long nblocks = grid_size(p.n_qtiles, n_units, 0);  // one CTA per unit
  auto kern = p.dbg ? attn_pp_kernel<1> : attn_pp_kernel<0>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, G::SMEM);
  if (e != cudaSuccess) return e;
  kern<<<(unsigned)nblocks, kPPThreads, G::SMEM, st>>>(mQ, mK, mV, p);
  return cudaGetLastError();
}

}  // namespace zq
