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
// One CTA computes one 128-row query tile of one (batch, head).  Warp roles:
//   warps 0-3  softmax + epilogue; thread t owns query row t (TMEM lane t)
//   warp 4     TMA producer (Q once, then K/V tiles through an NS-stage ring)
//   warp 5     TMEM allocator and single-thread tcgen05.mma issuer
// Tensor memory (512 columns x 128 lanes, fp32 words):
//   S0 [0,128) S1 [128,256)   score tiles; P (bf16x2 or 4 x e4m3 per word)
//                             is written over the first columns of its S
//   O  [256,256+DV)           output accumulator
//   RS [384,400)              FP8: rounded row sum (P times a ones matrix)
//   SFA0/SFA1 [400,404),[404,408)  FP8: per-(row, 32-key chunk) UE8M0 scales
//   SFB [408,412)             FP8: scales of V / ones, all 2^0
// MMA issue order: QK_0, QK_1, PV_0, QK_2, PV_1, ... so the softmax of tile
// j+1 overlaps PV_j and QK_{j+2}.
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <cuda.h>

#include <cstdint>

#include "sm100_ptx.cuh"
#include "zq_internal.h"

namespace zq {

constexpr int kTile = 128;
constexpr int kThreads = 192;
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
  static constexpr int NS = DT == 0 ? 2 : 4;               // K and V ring stages
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + QBYTES;
  static constexpr int OFF_V = OFF_K + NS * KBYTES;
  static constexpr int OFF_ONES = OFF_V + NS * VBYTES;     // 16 x 128 keys e4m3, K-major
  static constexpr int OFF_SF = OFF_ONES + 2048;           // 2 x 128 uint32
  static constexpr int OFF_BAR = OFF_SF + 1024;
  static constexpr int NBAR = 1 + 4 * NS + 2 + 2 + 1 + 2 + 1;
  static constexpr int SMEM = OFF_BAR + NBAR * 8 + 16 + 1024;  // + alignment slack
  static_assert(QBYTES % 1024 == 0 && VBYTES % 1024 == 0, "1 KB aligned tiles");
};

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float max3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ float pow2i(int e) {  // exact 2^e for -126 <= e <= 127
  return __int_as_float((e + 127) << 23);
}
// max over n consecutive floats with 3-input max
template <int N>
__device__ __forceinline__ float rowmax(const float* s) {
  float m0 = s[0], m1 = s[1];
#pragma unroll
  for (int c = 2; c + 3 < N; c += 4) {
    m0 = max3(m0, s[c], s[c + 1]);
    m1 = max3(m1, s[c + 2], s[c + 3]);
  }
  m0 = max3(m0, s[N - 2], s[N - 1]);
  return fmaxf(m0, m1);
}

template <int DT, int DQK, int DV, int MODE, int BS>
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
  uint64_t* bar_kfull = bars + 1;
  uint64_t* bar_kempty = bar_kfull + G::NS;
  uint64_t* bar_vfull = bar_kempty + G::NS;
  uint64_t* bar_vempty = bar_vfull + G::NS;
  uint64_t* bar_sfull = bar_vempty + G::NS;  // [2]
  uint64_t* bar_pfull = bar_sfull + 2;       // [2]
  // bar_pvdone completes once per PV_j.  When softmax j (j >= 1) needs O it
  // waits for phase j-1: PV_0..PV_{j-2} are complete (S_j's commit came
  // after them) and PV_j cannot start before P_j, so exactly phases j-1 and
  // j are possible and the parity test is unambiguous.
  uint64_t* bar_pvdone = bar_pfull + 2;      // [1]
  uint64_t* bar_sf = bar_pvdone + 1;         // [2]
  uint64_t* bar_ofinal = bar_sf + 2;         // [1] last PV landed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + G::NBAR);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  uint32_t* sf_smem = reinterpret_cast<uint32_t*>(smem + G::OFF_SF);  // [2][128]

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---- work unit: longest causal rows first
  const int BH = p.B * p.Hq;
  const int t = p.n_qtiles - 1 - (int)(blockIdx.x / BH);
  const int bh = (int)(blockIdx.x % BH);
  const int b = bh / p.Hq, h = bh % p.Hq;
  const int g = h / (p.Hq / p.Hkv);
  const int q0 = t * kTile;
  const int q1 = min(q0 + kTile - 1, p.Sq - 1);
  const int shift = p.Sk - p.Sq;
  int max_key = p.causal ? min(q1 + shift, p.Sk - 1) : p.Sk - 1;
  const int n_kv = max_key < 0 ? 0 : max_key / kTile + 1;
  const int min_lim = p.causal ? min(q0 + shift, p.Sk - 1) : p.Sk - 1;

  if (threadIdx.x == 0) {
    mbar_init(bar_q, 1);
    for (int s = 0; s < G::NS; ++s) {
      mbar_init(bar_kfull + s, 1);
      mbar_init(bar_kempty + s, 1);
      mbar_init(bar_vfull + s, 1);
      mbar_init(bar_vempty + s, 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar_sfull + s, 1);
      mbar_init(bar_pfull + s, 128);
      mbar_init(bar_sf + s, 128);
    }
    mbar_init(bar_pvdone, 1);
    mbar_init(bar_ofinal, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (DT == 1) {  // ones operand for the rounded row sum: e4m3 1.0 = 0x38
    uint32_t* ones = reinterpret_cast<uint32_t*>(smem + G::OFF_ONES);
    for (int i = threadIdx.x; i < 512; i += kThreads) ones[i] = 0x38383838u;
    fence_proxy_async_smem();
  }
  if (warp == 5) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  if (warp == 4 && lane == 0) {
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

  auto fail = [&]() {
    *abort_flag = 1;
    if (p.status) atomicExch(p.status, -7 /* ZQ_ERR_TIMEOUT */);
  };

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && n_kv > 0) {
      uint8_t* sq = smem + G::OFF_Q;
      mbar_arrive_expect_tx(bar_q, G::QBYTES);
#pragma unroll
      for (int c = 0; c < G::NCH; ++c) {
        const bool narrow = (c == G::NCH - 1) && G::LASTW == 64;
        tma_load_4d(sq + c * 16384, narrow ? (const void*)&tmQ2 : (const void*)&tmQ, bar_q,
                    c * 128 / G::ES, h, q0, b);
      }
      for (int j = 0; j < n_kv; ++j) {
        const int s = j % G::NS;
        const uint32_t ph = ((j / G::NS) & 1) ^ 1;
        if (!mbar_wait(bar_kempty + s, ph, lim, abort_flag)) { fail(); break; }
        uint8_t* sk = smem + G::OFF_K + s * G::KBYTES;
        mbar_arrive_expect_tx(bar_kfull + s, G::KBYTES);
#pragma unroll
        for (int c = 0; c < G::NCH; ++c) {
          const bool narrow = (c == G::NCH - 1) && G::LASTW == 64;
          tma_load_4d(sk + c * 16384, narrow ? (const void*)&tmK2 : (const void*)&tmK,
                      bar_kfull + s, c * 128 / G::ES, g, j * kTile, b);
        }
        if (!mbar_wait(bar_vempty + s, ph, lim, abort_flag)) { fail(); break; }
        uint8_t* sv = smem + G::OFF_V + s * G::VBYTES;
        mbar_arrive_expect_tx(bar_vfull + s, G::VBYTES);
#pragma unroll
        for (int c = 0; c < G::VCH; ++c)
          tma_load_4d(sv + c * 16384, &tmV, bar_vfull + s, c * 128 / G::ES, g, j * kTile, b);
      }
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && n_kv > 0) {
      const uint32_t sbase = smem_u32(smem);
      constexpr uint32_t idesc_qk = idesc_dense(DT == 0 ? 1u : 0u, 0u, 128, 128);
      constexpr uint32_t idesc_pv_bf16 = idesc_dense(1u, 1u, 128, DV);
      auto qk_desc = [&](uint32_t base, int kk) -> uint64_t {
        const int pos = kk * 32;
        const int c = pos / 128;
        const bool narrow = (c == G::NCH - 1) && G::LASTW == 64;
        return smem_desc(base + c * 16384 + (pos % 128), 16, narrow ? 512 : 1024,
                         narrow ? SW_64B : SW_128B);
      };
      auto issue_qk = [&](int j) -> bool {
        const int s = j % G::NS;
        if (!mbar_wait(bar_kfull + s, (j / G::NS) & 1, lim, abort_flag)) return false;
        tc_fence_after();
        const uint32_t dS = tbase + kColS0 + (j & 1) * 128;
        const uint32_t kb = sbase + G::OFF_K + s * G::KBYTES;
        const uint32_t qb = sbase + G::OFF_Q;
#pragma unroll
        for (int kk = 0; kk < G::QK_STEPS; ++kk) {
          if (DT == 0)
            mma_f16_ss(dS, qk_desc(qb, kk), qk_desc(kb, kk), idesc_qk, kk > 0);
          else
            mma_f8_ss(dS, qk_desc(qb, kk), qk_desc(kb, kk), idesc_qk, kk > 0);
        }
        tc_commit(bar_kempty + s);
        tc_commit(bar_sfull + (j & 1));
        return true;
      };
      auto issue_pv = [&](int j) -> bool {
        const int s = j % G::NS;
        if (!mbar_wait(bar_pfull + (j & 1), (j >> 1) & 1, lim, abort_flag)) return false;
        if (!mbar_wait(bar_vfull + s, (j / G::NS) & 1, lim, abort_flag)) return false;
        tc_fence_after();
        const uint32_t vb = sbase + G::OFF_V + s * G::VBYTES;
        const uint32_t aP = tbase + kColS0 + (j & 1) * 128;
#pragma unroll
        for (int kk = 0; kk < G::PV_STEPS; ++kk) {
          const uint32_t acc = (j > 0 || kk > 0) ? 1u : 0u;
          if (DT == 0) {
            // 16 keys per step = 8 packed bf16x2 columns of P; V rows 16*kk..
            const uint64_t dv = smem_desc(vb + kk * 16 * 128, 16384, 1024, SW_128B);
            mma_f16_ts(tbase + kColO, aP + kk * 8, dv, idesc_pv_bf16, acc);
          } else {
            // 32 keys per step = 8 columns of 4 x e4m3; scale byte kk
            const uint64_t dv = smem_desc(vb + kk * 32 * 128, 16384, 1024, SW_128B);
            const uint32_t sfa =
                (tbase + kColSFA + (j & 1) * 4) | ((uint32_t)kk << 30);
            const uint32_t sfb = (tbase + kColSFB) | ((uint32_t)kk << 30);
            mma_mxf8_ts(tbase + kColO, aP + kk * 8, dv, idesc_mx(1u, 128, DV, kk, kk), sfa, sfb,
                        acc);
            const uint64_t d1 =
                smem_desc(sbase + G::OFF_ONES + kk * 32, 16, 1024, SW_128B);
            mma_mxf8_ts(tbase + kColRS, aP + kk * 8, d1, idesc_mx(0u, 128, 16, kk, kk), sfa,
                        sfb, acc);
          }
        }
        tc_commit(bar_vempty + s);
        tc_commit(bar_pvdone);
        return true;
      };
      bool ok = true;
      if (!mbar_wait(bar_q, 0, lim, abort_flag)) ok = false;
      for (int j = 0; ok && j < n_kv; ++j) {
        if (!issue_qk(j)) { ok = false; break; }
        if (j > 0 && !issue_pv(j - 1)) { ok = false; break; }
      }
      if (ok && !issue_pv(n_kv - 1)) ok = false;
      if (ok) tc_commit(bar_ofinal);
      if (!ok) fail();
    }
  } else {
    // ------------------------------------------------------ softmax (rows)
    const int row = threadIdx.x;  // 0..127 == TMEM lane
    const int i = q0 + row;
    const int row_lim = p.causal ? min(i + shift, p.Sk - 1) : p.Sk - 1;
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    float c = p.softmax_scale * 1.4426950408889634f;  // log2(e)
    float vscale = 1.0f;
    if (DT == 1) {
      const float qd = p.q_descale ? *p.q_descale : 1.0f;
      const float kd = p.k_descale ? *p.k_descale : 1.0f;
      vscale = p.v_descale ? *p.v_descale : 1.0f;
      c = ((p.softmax_scale * qd) * kd) * 1.4426950408889634f;
      // SFB (scales of V and of the ones matrix): all 2^0 = 0x7F
      tmem_st4(tbase + lane_off + kColSFB, 0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu);
      tmem_st_wait();
    }
    const int T = p.headroom_T;
    float yref = -INFINITY;  // BF16: log2-domain reference max
    int eref = 0;            // FP8: reference exponent E
    bool have_ref = false;
    float l = 0.0f;          // BF16 row sum (fp32, unrounded p)
    bool ok = true;

    for (int j = 0; ok && j < n_kv; ++j) {
      const int buf = j & 1;
      bool w = mbar_wait(bar_sfull + buf, (j >> 1) & 1, lim, abort_flag);
      if (!__all_sync(0xffffffffu, w)) { ok = false; break; }
      tc_fence_after();
      uint32_t sr[128];
      {
        uint32_t(&a0)[32] = *reinterpret_cast<uint32_t(*)[32]>(sr);
        uint32_t(&a1)[32] = *reinterpret_cast<uint32_t(*)[32]>(sr + 32);
        uint32_t(&a2)[32] = *reinterpret_cast<uint32_t(*)[32]>(sr + 64);
        uint32_t(&a3)[32] = *reinterpret_cast<uint32_t(*)[32]>(sr + 96);
        const uint32_t ts = tbase + lane_off + kColS0 + buf * 128;
        tmem_ld32(ts, a0);
        tmem_ld32(ts + 32, a1);
        tmem_ld32(ts + 64, a2);
        tmem_ld32(ts + 96, a3);
        tmem_ld_wait();
      }
      float* s = reinterpret_cast<float*>(sr);
      const bool dump = p.dbg != nullptr && j == 0 && t == 0 && bh == 0;
      if (dump) {
        float* ds = static_cast<float*>(p.dbg) + row * 128;
#pragma unroll
        for (int cc = 0; cc < 128; ++cc) ds[cc] = s[cc];
      }
      const int kbase = j * kTile;
      if (kbase + kTile - 1 > min_lim) {
#pragma unroll
        for (int cc = 0; cc < 128; ++cc)
          if (kbase + cc > row_lim) s[cc] = -INFINITY;
      }
      const uint32_t tP = tbase + lane_off + kColS0 + buf * 128;

      if constexpr (DT == 0) {
        // ------------------------------------------------ BF16, exact exp2
        const float ymax = rowmax<128>(s) * c;
        const bool need = ymax > yref + 8.0f;
        if (__any_sync(0xffffffffu, need)) {
          const float nref = fmaxf(yref, ymax);
          const float f = (nref == -INFINITY || yref == nref) ? 1.0f : ex2_approx(yref - nref);
          yref = nref;
          l *= f;
          if (j > 0) {
            // O holds tiles < j; PV_{j-1} must have landed before rescaling
            w = mbar_wait(bar_pvdone, (j - 1) & 1, lim, abort_flag);
            if (!__all_sync(0xffffffffu, w)) { ok = false; break; }
            tc_fence_after();
#pragma unroll 1
            for (int ch = 0; ch < DV / 32; ++ch) {
              uint32_t o[32];
              const uint32_t to = tbase + lane_off + kColO + ch * 32;
              tmem_ld32(to, o);
              tmem_ld_wait();
#pragma unroll
              for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * f);
              tmem_st32(to, o);
            }
          }
        }
        const float nb = yref == -INFINITY ? 0.0f : -yref;
        uint32_t pk[64];
#pragma unroll
        for (int cc = 0; cc < 128; cc += 2) {
          const float p0 = ex2_approx(fmaf(s[cc], c, nb));
          const float p1 = ex2_approx(fmaf(s[cc + 1], c, nb));
          l += p0 + p1;
          pk[cc / 2] = pack_bf16x2(p0, p1);
        }
        tmem_st32(tP, *reinterpret_cast<uint32_t(*)[32]>(pk));
        tmem_st32(tP + 32, *reinterpret_cast<uint32_t(*)[32]>(pk + 32));
        if (dump) {
          uint32_t* dp = reinterpret_cast<uint32_t*>(static_cast<float*>(p.dbg) + 128 * 128);
#pragma unroll
          for (int e = 0; e < 64; ++e) dp[row * 64 + e] = pk[e];
        }
      } else {
        // ------------------------------------------------ FP8 P path
        const float m0 = rowmax<64>(s), m1 = rowmax<64>(s + 64);
        int e0, e1, emax;
        bool v0, v1;
        if (BS) {
          v0 = m0 != -INFINITY;
          v1 = m1 != -INFINITY;
          e0 = v0 ? (int)ceilf(m0 * c) - T : -100000;
          e1 = v1 ? (int)ceilf(m1 * c) - T : -100000;
          emax = max(e0, e1);
        } else {
          // running mode: one exponent from the running max, shared by both blocks
          const float mm = fmaxf(m0, m1);
          const float ymx = fmaxf(mm * c, yref);
          yref = ymx;
          v0 = v1 = ymx != -INFINITY;
          e0 = e1 = emax = v0 ? (int)ceilf(ymx) - T : -100000;
        }
        const bool valid = v0 || v1;
        // reference exponent: first valid tile; raised lazily (block mode,
        // when a block exceeds E by 32) or whenever it grows (running mode)
        const bool need = valid && (!have_ref || emax > eref + (BS ? 32 : 0));
        if (__any_sync(0xffffffffu, need)) {
          const int nref = need ? emax : eref;
          const float f = (have_ref && need) ? pow2i(max(eref - nref, -126)) : 1.0f;
          const bool had = have_ref;
          if (need) { eref = nref; have_ref = true; }
          if (j > 0 && __any_sync(0xffffffffu, had && need)) {
            w = mbar_wait(bar_pvdone, (j - 1) & 1, lim, abort_flag);
            if (!__all_sync(0xffffffffu, w)) { ok = false; break; }
            tc_fence_after();
#pragma unroll 1
            for (int ch = 0; ch < DV / 32; ++ch) {
              uint32_t o[32];
              const uint32_t to = tbase + lane_off + kColO + ch * 32;
              tmem_ld32(to, o);
              tmem_ld_wait();
#pragma unroll
              for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * f);
              tmem_st32(to, o);
            }
            uint32_t rs;
            tmem_ld1(tbase + lane_off + kColRS, rs);
            tmem_ld_wait();
            tmem_st1(tbase + lane_off + kColRS, __float_as_uint(__uint_as_float(rs) * f));
          }
        }
        // UE8M0 scale bytes 2^(e_k - E): chunks 0,1 -> block 0; 2,3 -> block 1
        const int sf0 = v0 ? min(max(e0 - eref + 127, 0), 254) : 0;
        const int sf1 = v1 ? min(max(e1 - eref + 127, 0), 254) : 0;
        const uint32_t sfw = (uint32_t)sf0 * 0x0101u | ((uint32_t)sf1 * 0x0101u) << 16;
        uint32_t pk[32];
        if (MODE == 0) {
          // exact: e4m3_rne(exp2(y - e))
#pragma unroll
          for (int blk = 0; blk < 2; ++blk) {
            const float ne = -(float)(blk == 0 ? (v0 ? e0 : 0) : (v1 ? e1 : 0));
#pragma unroll
            for (int cc = blk * 64; cc < blk * 64 + 64; cc += 4) {
              const float p0 = ex2_approx(fmaf(s[cc], c, ne));
              const float p1 = ex2_approx(fmaf(s[cc + 1], c, ne));
              const float p2 = ex2_approx(fmaf(s[cc + 2], c, ne));
              const float p3 = ex2_approx(fmaf(s[cc + 3], c, ne));
              const uint32_t lo = __nv_cvt_float2_to_fp8x2(make_float2(p0, p1), __NV_SATFINITE, __NV_E4M3);
              const uint32_t hi = __nv_cvt_float2_to_fp8x2(make_float2(p2, p3), __NV_SATFINITE, __NV_E4M3);
              pk[cc / 4] = lo | (hi << 16);
            }
          }
        } else {
          // Lean P: bits of fma(s, 8c, 56 - 8e + 1.5*2^23) hold rne(8(y-e))+56
          // in their low byte; clamp at code 0 by an integer max.
          const float c8 = c * 8.0f;
          const int magic = 0x4B400000;  // bits of 1.5 * 2^23
#pragma unroll
          for (int blk = 0; blk < 2; ++blk) {
            const int e = blk == 0 ? (v0 ? e0 : 0) : (v1 ? e1 : 0);
            const float kadd = 12582912.0f + (float)(56 - 8 * e);
#pragma unroll
            for (int cc = blk * 64; cc < blk * 64 + 64; cc += 4) {
              const int b0 = max(__float_as_int(fmaf(s[cc], c8, kadd)), magic);
              const int b1 = max(__float_as_int(fmaf(s[cc + 1], c8, kadd)), magic);
              const int b2 = max(__float_as_int(fmaf(s[cc + 2], c8, kadd)), magic);
              const int b3 = max(__float_as_int(fmaf(s[cc + 3], c8, kadd)), magic);
              pk[cc / 4] = prmt(prmt(b0, b1, 0x0040u), prmt(b2, b3, 0x0040u), 0x5410u);
            }
          }
        }
        tmem_st32(tP, pk);
        if (dump) {
          uint32_t* dp = reinterpret_cast<uint32_t*>(static_cast<float*>(p.dbg) + 128 * 128);
#pragma unroll
          for (int e = 0; e < 32; ++e) dp[row * 64 + e] = pk[e];
          dp[128 * 64 + row] = sfw;
        }
        // scale factors: the row of query r goes to column r/32 of the SFA
        // block, replicated in all four lane quarters (lane r%32 + 32q)
        sf_smem[buf * 128 + row] = sfw;
        mbar_arrive(bar_sf + buf);
        w = mbar_wait(bar_sf + buf, (j >> 1) & 1, lim, abort_flag);
        if (!__all_sync(0xffffffffu, w)) { ok = false; break; }
        tmem_st4(tbase + lane_off + kColSFA + buf * 4, sf_smem[buf * 128 + lane],
                 sf_smem[buf * 128 + 32 + lane], sf_smem[buf * 128 + 64 + lane],
                 sf_smem[buf * 128 + 96 + lane]);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar_pfull + buf);
    }
    if (!ok) {
      fail();
    } else {
      // ------------------------------------------------------------ epilogue
      float L = l, lse_v = -INFINITY;
      bool wok = true;
      if (n_kv > 0) {
        wok = mbar_wait(bar_ofinal, 0, lim, abort_flag);
        wok = __all_sync(0xffffffffu, wok);
      }
      if (!wok) {
        fail();
      } else {
        tc_fence_after();
        if (DT == 1 && n_kv > 0) {
          uint32_t rs;
          tmem_ld1(tbase + lane_off + kColRS, rs);
          tmem_ld_wait();
          L = __uint_as_float(rs);
        }
        const bool empty = !(L > 0.0f);
        const float inv = empty ? 0.0f : vscale / L;
        if (!empty) {
          const float ref = DT == 0 ? yref : (float)eref;
          lse_v = (ref + __log2f(L)) * 0.6931471805599453f;
        }
        __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(p.out) + (((int64_t)b * p.Sq + i) * p.Hq + h) * DV;
#pragma unroll 1
        for (int ch = 0; ch < DV / 32; ++ch) {
          uint32_t o[32];
          if (n_kv > 0) {
            tmem_ld32(tbase + lane_off + kColO + ch * 32, o);
            tmem_ld_wait();
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = 0u;
          }
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e)
            pk[e] = pack_bf16x2(__uint_as_float(o[2 * e]) * inv, __uint_as_float(o[2 * e + 1]) * inv);
          if (i < p.Sq) {
            uint4* dst = reinterpret_cast<uint4*>(orow + ch * 32);
#pragma unroll
            for (int e = 0; e < 4; ++e)
              dst[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
          }
        }
        if (p.lse && i < p.Sq) p.lse[((int64_t)b * p.Hq + h) * p.Sq + i] = lse_v;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tbase, kTmemCols);
  }
}

// ------------------------------------------------------------------ host side
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

// Tensor (B, S, H, d) of `es`-byte elements; box = `box_elems` channels x 1
// head x 128 rows x 1 batch.
static bool make_map(CUtensorMap* m, const void* base, int es, int B, int S, int H, int d,
                     int box_elems, CUtensorMapSwizzle sw) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)S, (cuuint64_t)B};
  cuuint64_t strides[3] = {(cuuint64_t)d * es, (cuuint64_t)H * d * es, (cuuint64_t)S * H * d * es};
  cuuint32_t box[4] = {(cuuint32_t)box_elems, 1, (cuuint32_t)kTile, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = enc(m, es == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8, 4,
                   const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int DT, int DQK, int DV, int MODE, int BS>
static cudaError_t launch_variant(const AttnLaunch& a, cudaStream_t st) {
  using G = Geo<DT, DQK, DV>;
  CUtensorMap mQ, mQ2, mK, mK2, mV;
  const int es = G::ES;
  const auto& p = a.p;
  if (!make_map(&mQ, a.q, es, p.B, p.Sq, p.Hq, DQK, 128 / es, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map(&mK, a.k, es, p.B, p.Sk, p.Hkv, DQK, 128 / es, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map(&mV, a.v, es, p.B, p.Sk, p.Hkv, DV, 128 / es, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  if (G::LASTW == 64) {
    if (!make_map(&mQ2, a.q, es, p.B, p.Sq, p.Hq, DQK, 64 / es, CU_TENSOR_MAP_SWIZZLE_64B) ||
        !make_map(&mK2, a.k, es, p.B, p.Sk, p.Hkv, DQK, 64 / es, CU_TENSOR_MAP_SWIZZLE_64B))
      return cudaErrorInvalidValue;
  } else {
    mQ2 = mQ;
    mK2 = mK;
  }
  auto kern = attn_fwd_kernel<DT, DQK, DV, MODE, BS>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, G::SMEM);
  if (e != cudaSuccess) return e;
  const long long nblocks = (long long)p.n_qtiles * p.B * p.Hq;
  if (nblocks <= 0) return cudaSuccess;
  kern<<<(unsigned)nblocks, kThreads, G::SMEM, st>>>(mQ, mQ2, mK, mK2, mV, p);
  return cudaGetLastError();
}

cudaError_t launch_attention(const AttnLaunch& a, cudaStream_t st) {
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
