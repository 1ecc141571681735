"""The attention kernel's schedule, checked on the host through the C ABI
(zq_attn_plan_launch computes it with the same code the kernel runs; no GPU
is touched).  Causal skipping is checked against brute force over keys, the
unit order against its definition, and the persistent CTAs' share of work
against a plain stride."""
import numpy as np
import pytest

import bf16_causal_prefill_02_b200 as zq

CASES = [
    # B, Sq, Sk, Hq, Hkv, causal
    (2, 600, 600, 80, 16, True),
    (1, 300, 100, 4, 2, True),     # Sq > Sk: the first tiles see no key
    (1, 100, 300, 4, 4, True),     # Sq < Sk: chunked prefill
    (1, 257, 129, 3, 3, True),
    (2, 200, 520, 6, 2, False),
    (1, 4096, 4096, 32, 8, True),
    (1, 32768, 32768, 32, 32, True),
    (1, 1, 1, 1, 1, True),
]


def _brute_n_kv(t, Sq, Sk, causal):
    """Key tiles holding at least one key visible to some row of query tile t."""
    rows = np.arange(128 * t, min(128 * t + 128, Sq))
    vis = []
    for j in range((Sk + 127) // 128):
        keys = np.arange(128 * j, min(128 * j + 128, Sk))
        if not causal:
            vis.append(True)
        else:
            vis.append(bool(np.any(keys[None, :] <= rows[:, None] + (Sk - Sq))))
    vis = np.array(vis, dtype=bool)
    n = int(vis.sum())
    assert np.all(vis[:n]), "visible key tiles must form a prefix"
    return n


@pytest.mark.parametrize("B,Sq,Sk,Hq,Hkv,causal", CASES)
def test_units_cover_every_tile_once(B, Sq, Sk, Hq, Hkv, causal):
    plan, u = zq.attn_plan(B, Sq, Sk, Hq, Hkv, causal=causal)
    nq = (Sq + 127) // 128
    assert plan.n_units == nq * B * Hq
    pairs = set(zip(u["tile"].tolist(), u["bh"].tolist()))
    assert len(pairs) == plan.n_units
    assert pairs == {(t, bh) for t in range(nq) for bh in range(B * Hq)}


@pytest.mark.parametrize("B,Sq,Sk,Hq,Hkv,causal", CASES[:5])
def test_causal_skip_matches_brute_force(B, Sq, Sk, Hq, Hkv, causal):
    _, u = zq.attn_plan(B, Sq, Sk, Hq, Hkv, causal=causal)
    want = {t: _brute_n_kv(t, Sq, Sk, causal) for t in range((Sq + 127) // 128)}
    for t, n in zip(u["tile"].tolist(), u["n_kv"].tolist()):
        assert n == want[t], (t, n, want[t])


def test_causal_skip_counts_at_32k():
    # S = 32768: tile t visits t + 1 key tiles, 256 * 257 / 2 pairs per head
    _, u = zq.attn_plan(1, 32768, 32768, 32, 32)
    assert np.array_equal(u["n_kv"], u["tile"] + 1)
    assert int(u["n_kv"].sum()) == 32 * 256 * 257 // 2


@pytest.mark.parametrize("B,Sq,Sk,Hq,Hkv,causal", CASES)
def test_longest_rows_first_inside_head_groups(B, Sq, Sk, Hq, Hkv, causal):
    plan, u = zq.attn_plan(B, Sq, Sk, Hq, Hkv, causal=causal)
    GH, nq = plan.head_group, (Sq + 127) // 128
    assert (B * Hq) % GH == 0
    for gi in range(B * Hq // GH):
        sl = slice(gi * GH * nq, (gi + 1) * GH * nq)
        tiles, heads = u["tile"][sl], u["bh"][sl]
        # tiles descend, the group's heads interleave within each tile
        assert np.array_equal(tiles, np.repeat(np.arange(nq - 1, -1, -1), GH))
        assert np.array_equal(heads, np.tile(np.arange(gi * GH, (gi + 1) * GH), nq))


@pytest.mark.parametrize("B,S,Hq,Hkv,dqk,dtype,want", [
    # one CTA per unit (more than 64 query tiles): the query heads of one kv head
    (1, 32768, 32, 32, 128, zq.ZQ_DTYPE_FP8_E4M3, 1),
    (1, 16384, 32, 8, 128, zq.ZQ_DTYPE_FP8_E4M3, 4),     # 4:1 GQA
    (1, 16384, 16, 16, 192, zq.ZQ_DTYPE_BF16, 1),
    (2, 9000, 12, 3, 128, zq.ZQ_DTYPE_BF16, 4),
    # persistent (at most 64 query tiles): by the size of K/V
    (1, 4096, 32, 8, 128, zq.ZQ_DTYPE_FP8_E4M3, 32),     # 8 MB: all heads
    (1, 8192, 32, 32, 128, zq.ZQ_DTYPE_BF16, 4),         # 134 MB > 96 MB
    (1, 8192, 32, 32, 128, zq.ZQ_DTYPE_FP8_E4M3, 32),    # 67 MB
    (1, 8192, 6, 6, 128, zq.ZQ_DTYPE_BF16, 6),           # 25 MB
    (8, 8192, 6, 6, 128, zq.ZQ_DTYPE_BF16, 4),           # 201 MB, 48 heads: groups of 4
    (4, 8192, 6, 6, 128, zq.ZQ_DTYPE_BF16, 24),          # exactly 96 MiB: not above
    (1, 8192, 50, 50, 192, zq.ZQ_DTYPE_BF16, 2),         # 262 MB, 50 heads: groups of 2
])
def test_head_group_choice(B, S, Hq, Hkv, dqk, dtype, want):
    plan, _ = zq.attn_plan(B, S, S, Hq, Hkv, d_qk=dqk, dtype=dtype)
    assert plan.head_group == want


@pytest.mark.parametrize("B,Sq,Sk,Hq,Hkv,causal", [c for c in CASES if (c[1] + 127) // 128 <= 64])
def test_persistent_ctas_partition_the_units(B, Sq, Sk, Hq, Hkv, causal):
    plan, u = zq.attn_plan(B, Sq, Sk, Hq, Hkv, causal=causal, num_sms=148)
    assert plan.persistent == 1 and plan.grid == min(148, plan.n_units)
    assert np.all(u["cta"] >= 0) and np.all(u["cta"] < plan.grid) and np.all(u["round"] >= 0)
    for c in range(plan.grid):
        mine = np.flatnonzero(u["cta"] == c)
        # round k of CTA c is unit k*G + c (k even) or k*G + G-1-c (k odd)
        k = u["round"][mine]
        assert np.array_equal(np.sort(k), np.arange(len(mine)))
        G = plan.grid
        assert np.array_equal(mine, np.where(k % 2 == 0, k * G + c, k * G + G - 1 - c))


@pytest.mark.parametrize("cfg", [(2, 600, 600, 80, 16), (1, 4096, 4096, 32, 8), (1, 8192, 8192, 32, 32),
                                 (4, 2048, 2048, 16, 16), (1, 1000, 1000, 64, 8)])
def test_zigzag_balances_work_better_than_a_stride(cfg):
    plan, u = zq.attn_plan(*cfg, num_sms=148)
    assert plan.persistent == 1
    work = np.bincount(u["cta"], weights=u["n_kv"], minlength=plan.grid)
    stride = np.bincount(np.arange(plan.n_units) % plan.grid, weights=u["n_kv"], minlength=plan.grid)
    assert work.sum() == stride.sum() == u["n_kv"].sum()
    assert work.max() <= stride.max()
    assert work.max() / work.mean() <= 1.12


def test_long_sequences_launch_one_cta_per_unit():
    plan, u = zq.attn_plan(1, 32768, 32768, 32, 32, num_sms=148)
    assert plan.persistent == 0 and plan.grid == plan.n_units == 8192
    assert np.array_equal(u["cta"], np.arange(8192)) and not u["round"].any()
    assert plan.threads == 320 and 0 < plan.smem_bytes <= 227 * 1024


def test_plan_argument_errors():
    a = zq.zq_attn_args()
    a.q = a.k = a.v = a.out = 1 << 20
    a.B, a.Sq, a.Sk, a.Hq, a.Hkv, a.d_qk, a.d_v = 1, 128, 128, 3, 2, 128, 128
    a.dtype = zq.ZQ_DTYPE_BF16
    assert zq.zq_attn_plan_launch(a, 148, zq.zq_attn_plan()) == zq.ZQ_ERR_SHAPE
    a.Hq = 2
    assert zq._lib.zq_attn_plan_launch(a, 148, None, None, None, None, None, None) == zq.ZQ_ERR_NULL
    a.d_qk = 64
    assert zq.zq_attn_plan_launch(a, 148, zq.zq_attn_plan()) == zq.ZQ_ERR_UNSUPPORTED


# ------------------------------------------------- paired units (BF16, d = 128)
LONG = [
    # B, Sq, Sk, Hq, Hkv, causal: more than 64 query tiles (one CTA per unit)
    (1, 8320, 8320, 2, 1, True),      # 65 tiles: the last pair has one tile
    (1, 9000, 12000, 3, 3, True),     # Sq < Sk
    (1, 12000, 9000, 2, 2, True),     # Sq > Sk: the first rows see no key
    (2, 8500, 8700, 2, 1, False),
    (1, 32768, 32768, 32, 32, True),
]


def _brute_n_kv_rows(r0, r1, Sq, Sk, causal, kt):
    """Key tiles of kt keys holding a key visible to some query row in [r0, r1)."""
    rows = np.arange(r0, min(r1, Sq))
    if rows.size == 0:
        return 0
    if not causal:
        return (Sk + kt - 1) // kt
    last = min(int(rows.max()) + Sk - Sq, Sk - 1)  # visible keys of the last row form a prefix
    return 0 if last < 0 else last // kt + 1


@pytest.mark.parametrize("B,Sq,Sk,Hq,Hkv,causal", LONG)
def test_long_bf16_d128_units_are_tile_pairs(B, Sq, Sk, Hq, Hkv, causal):
    # BF16 at d = 128 with more than 64 query tiles runs the paired kernel:
    # a unit is two consecutive 128-row tiles (256 rows) with 64-key tiles,
    # one CTA per unit; every pair once, longest rows first in head groups
    plan, u = zq.attn_plan(B, Sq, Sk, Hq, Hkv, dtype=zq.ZQ_DTYPE_BF16, causal=causal, num_sms=148)
    npairs = ((Sq + 127) // 128 + 1) // 2
    assert plan.rows_per_unit == 256 and plan.keys_per_tile == 64
    assert plan.n_units == npairs * B * Hq and plan.persistent == 0 and plan.grid == plan.n_units
    assert plan.threads == 352 and 0 < plan.smem_bytes <= 227 * 1024
    assert set(zip(u["tile"].tolist(), u["bh"].tolist())) == {(t, bh) for t in range(npairs) for bh in range(B * Hq)}
    GH = plan.head_group
    for gi in range(B * Hq // GH):
        sl = slice(gi * GH * npairs, (gi + 1) * GH * npairs)
        assert np.array_equal(u["tile"][sl], np.repeat(np.arange(npairs - 1, -1, -1), GH))
    assert np.array_equal(u["cta"], np.arange(plan.n_units)) and not u["round"].any()


@pytest.mark.parametrize("B,Sq,Sk,Hq,Hkv,causal", LONG[:4])
def test_pair_causal_skip_matches_brute_force(B, Sq, Sk, Hq, Hkv, causal):
    # a pair visits the 64-key tiles its later tile needs; the earlier tile
    # stops at its own diagonal (the kernel's parity tests check the rows)
    _, u = zq.attn_plan(B, Sq, Sk, Hq, Hkv, dtype=zq.ZQ_DTYPE_BF16, causal=causal)
    for t, n in zip(u["tile"].tolist(), u["n_kv"].tolist()):
        assert n == _brute_n_kv_rows(256 * t, 256 * t + 256, Sq, Sk, causal, 64), (t, n)


def test_pair_counts_at_32k():
    # S = 32768: pair t visits 4t + 4 key tiles of 64 keys
    _, u = zq.attn_plan(1, 32768, 32768, 32, 32, dtype=zq.ZQ_DTYPE_BF16)
    assert np.array_equal(u["n_kv"], 4 * u["tile"] + 4)
    assert int(u["n_kv"].sum()) == 32 * 4 * 128 * 129 // 2


@pytest.mark.parametrize("B,S,dtype,dqk", [
    (1, 8192, zq.ZQ_DTYPE_BF16, 128),       # 64 tiles: persistent, single-tile kernel
    (2, 1000, zq.ZQ_DTYPE_BF16, 128),
    (1, 16384, zq.ZQ_DTYPE_BF16, 192),      # MLA
    (1, 16384, zq.ZQ_DTYPE_FP8_E4M3, 128),  # FP8
    (1, 16384, zq.ZQ_DTYPE_FP8_E4M3, 192),
])
def test_other_shapes_keep_single_tile_units(B, S, dtype, dqk):
    plan, u = zq.attn_plan(B, S, S, 4, 2, d_qk=dqk, dtype=dtype)
    assert plan.rows_per_unit == 128 and plan.keys_per_tile == 128 and plan.threads == 320
    assert plan.n_units == (S + 127) // 128 * B * 4
