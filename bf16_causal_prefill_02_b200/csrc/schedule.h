// schedule.h -- the attention kernel's work units, their order and the
// launch shape.  Shared by the kernel (device) and the C-ABI layer (host),
// so that zq_attn_plan_launch reports exactly what a launch does.
//
// [P3] "Zyphra ZYFA ... FP8 FlashAttention for AMD MI355X" (ai4bro.com),
// TL;DR: causal prefill.  A query tile visits only the key tiles that hold
// at least one key visible to one of its rows (causal skipping); query head
// h reads kv head h / (Hq / Hkv) (GQA).
#pragma once
#include <cstdint>

#include "zq_internal.h"

namespace zq {

constexpr int kTile = 128;  // query rows per unit and keys per key tile

// One work unit: the 128-row query tile t of flat head bh = batch * Hq + head.
// Units are numbered in groups of head_group consecutive flat heads; inside a
// group, longest causal rows first (t descending), interleaved across the
// group's heads.
struct Unit {
  int t, bh, b, h, g, q0, n_kv, min_lim;
};
__host__ __device__ __forceinline__ Unit unit_of(const AttnParams& p, int u) {
  Unit w;
  const int GH = p.head_group;
  const int gi = u / (GH * p.n_qtiles), gr = u % (GH * p.n_qtiles);
  w.t = p.n_qtiles - 1 - gr / GH;
  w.bh = gi * GH + gr % GH;
  w.b = w.bh / p.Hq;
  w.h = w.bh % p.Hq;
  w.g = w.h / (p.Hq / p.Hkv);
  w.q0 = w.t * kTile;
  // bottom-right causal alignment: key c is visible to query i iff
  // c <= i + Sk - Sq.  n_kv = key tiles up to the last visible key of the
  // tile's last row; min_lim = last key visible to its first row (tiles
  // whose keys all lie at or below it need no mask).
  const int q1 = min(w.q0 + kTile - 1, p.Sq - 1);
  const int shift = p.Sk - p.Sq;
  const int max_key = p.causal ? min(q1 + shift, p.Sk - 1) : p.Sk - 1;
  w.n_kv = max_key < 0 ? 0 : max_key / kTile + 1;
  w.min_lim = p.causal ? min(w.q0 + shift, p.Sk - 1) : p.Sk - 1;
  return w;
}

// The paired kernel's unit: two consecutive 128-row query tiles 2tp and
// 2tp + 1 of one flat head, one per softmax team, sharing every K/V tile.
// Keys come in tiles of 64 (kPairKeyTile).  Numbering as for Unit (groups
// of head_group flat heads, longest rows first), over (n_qtiles + 1) / 2
// pairs per head.  Team t visits key tiles 0 .. n_kv[t] - 1; the second
// tile's rows are later, so n_kv[1] >= n_kv[0] whenever the second tile
// has rows (a tile past Sq has none: n_kv = 0).
constexpr int kPairKeyTile = 64;
struct PairUnit {
  int tp, bh, b, h, g;
  int q0[2], n_kv[2], min_lim[2];
  int n_kv_max;
};
__host__ __device__ __forceinline__ int n_pairs_of(int n_qtiles) { return (n_qtiles + 1) / 2; }
__host__ __device__ __forceinline__ PairUnit pair_of(const AttnParams& p, int u) {
  PairUnit w;
  const int GH = p.head_group;
  const int np = n_pairs_of(p.n_qtiles);
  const int gi = u / (GH * np), gr = u % (GH * np);
  w.tp = np - 1 - gr / GH;
  w.bh = gi * GH + gr % GH;
  w.b = w.bh / p.Hq;
  w.h = w.bh % p.Hq;
  w.g = w.h / (p.Hq / p.Hkv);
  const int shift = p.Sk - p.Sq;
  w.n_kv_max = 0;
  for (int t = 0; t < 2; ++t) {
    const int q0 = (2 * w.tp + t) * kTile;
    w.q0[t] = q0;
    if (q0 >= p.Sq) {
      w.n_kv[t] = 0;
      w.min_lim[t] = -1;
      continue;
    }
    const int q1 = min(q0 + kTile - 1, p.Sq - 1);
    const int max_key = p.causal ? min(q1 + shift, p.Sk - 1) : p.Sk - 1;
    w.n_kv[t] = max_key < 0 ? 0 : max_key / kPairKeyTile + 1;
    w.min_lim[t] = p.causal ? min(q0 + shift, p.Sk - 1) : p.Sk - 1;
    w.n_kv_max = max(w.n_kv_max, w.n_kv[t]);
  }
  return w;
}

// The k-th unit of CTA `cta` among `grid` persistent CTAs: rounds of `grid`
// units, walked forwards in even rounds and backwards in odd ones, so that
// under longest-rows-first numbering every CTA pairs long units with short
// ones (a plain stride would hand CTA 0 about twice the work of the last
// CTA).  Strictly increasing in k.  With one unit per CTA (grid = units),
// unit_at(0, grid, cta) = cta.
__host__ __device__ __forceinline__ int unit_at(int k, int grid, int cta) {
  return k * grid + ((k & 1) ? grid - 1 - cta : cta);
}

// Heads per group.  Launches with one CTA per unit (more than 64 query
// tiles): the query heads of one kv head (Hq / Hkv; one head without GQA),
// so that the ~148 blocks that run together all stream the same K/V tiles,
// which stay in L2 (measured against groups of 4 and of all heads: FP8 16K
// +11%, MLA 16K +13% FP8 / +8% BF16, BF16 16K +13%, 32K equal or better).
// Persistent launches: 4 heads (one K/V head under 4:1 GQA) when the K/V of
// all heads is well past what the 126 MB L2 keeps around (96 MB), else every
// head in one group (plain longest-rows-first, which balances the tail best).
inline bool use_persistent(int n_qtiles);
inline int choose_head_group(int B, int Hq, int Hkv, int Sq, int Sk, int d_qk, int d_v, int elem_bytes) {
  const int bh = B * Hq;
  const int n_qtiles = (Sq + kTile - 1) / kTile;
  if (!use_persistent(n_qtiles)) return Hq / Hkv;
  const double kv_bytes = (double)B * Hkv * Sk * (d_qk + d_v) * elem_bytes;
  if (kv_bytes > 96.0 * 1024 * 1024) return bh % 4 == 0 ? 4 : (bh % 2 == 0 ? 2 : 1);
  return bh;
}

// Short sequences (at most 64 query tiles) run persistent: one CTA per SM,
// each walking its share of the units, so that a unit's loads and first QK
// overlap the previous unit's tail.  Longer ones launch a CTA per unit: the
// hardware scheduler then balances units of very different lengths better
// than the static share, and the per-unit setup is a small part of a long
// unit.
inline bool use_persistent(int n_qtiles) { return n_qtiles <= 64; }
inline long long grid_size(int n_qtiles, long long n_units, int num_sms) {
  if (use_persistent(n_qtiles) && num_sms > 0 && num_sms < n_units) return num_sms;
  return n_units;
}

}  // namespace zq
