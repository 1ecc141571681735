"""GPU parity of the paired BF16 kernel (two 128-row query tiles per CTA,
64-key tiles), which BF16 at d = 128 runs when Sq has more than 64 query
tiles: sampled rows against the fp64 oracle at sizes that cross every edge
of its schedule -- a last pair with one tile, Sq < Sk, Sq > Sk (rows without
keys), non-causal, GQA, a reference that moves many times -- plus bitwise
determinism, the debug dump of a tile of either team and the timeout path."""
import numpy as np
import pytest
import torch

import workloads
from attn_cases import Case, check_against_oracle

pytestmark = pytest.mark.gpu


def _rows(B, Hq, Sq, every=97):
    """Flat rows (b*Hq + h)*Sq + i: a stride through every head, plus the
    first, second and last rows of every 128-row tile of the last four pairs
    and of the first pair (both teams, the diagonal tiles, the ragged end)."""
    nq = (Sq + 127) // 128
    tiles = sorted(set(range(max(0, nq - 8), nq)) | {0, 1})
    edge = sorted({i for t in tiles for i in (128 * t, 128 * t + 1, 128 * t + 127) if i < Sq})
    rows = []
    for bh in range(B * Hq):
        idx = sorted(set(range(bh % 7, Sq, every)) | set(edge) | {Sq - 1})
        rows.extend(bh * Sq + i for i in idx)
    return np.asarray(rows, dtype=np.int64)


def _uses_pair_kernel(case):
    import bf16_causal_prefill_02_b200 as zq

    plan, _ = zq.attn_plan(case.B, case.Sq, case.Sk, case.Hq, case.Hkv, d_qk=case.dqk, d_v=case.dv,
                           dtype=zq.ZQ_DTYPE_BF16, causal=case.causal)
    return plan.rows_per_unit == 256


@pytest.mark.parametrize("B,Sq,Sk,Hq,Hkv,causal", [
    (1, 8320, 8320, 2, 1, True),      # 65 tiles: the last pair has one tile
    (1, 9000, 12000, 2, 2, True),     # Sq < Sk (chunked prefill)
    (1, 12000, 9000, 2, 2, True),     # Sq > Sk: the first 3000 rows see no key
    (2, 8500, 8700, 2, 1, False),     # non-causal, GQA, a ragged last key tile
    (1, 8448, 8448, 4, 1, True),      # 4:1 GQA, 66 tiles
    (1, 8193, 8193, 1, 1, True),      # the last tile holds one row
    (1, 9000, 1, 2, 2, True),         # one key: only the last row sees it
    (1, 9000, 70, 1, 1, False),       # fewer keys than one key tile, non-causal
])
def test_pair_kernel_sampled_rows(B, Sq, Sk, Hq, Hkv, causal):
    c = Case(B, Sq, Sk, Hq, Hkv, 128, 128, dtype="bf16", causal=causal, seed=Sq % 97 + Sk % 89)
    assert _uses_pair_kernel(c)
    res = check_against_oracle(c, rows=_rows(B, Hq, Sq))
    print(B, Sq, Sk, Hq, Hkv, causal, res)


def test_pair_kernel_lazy_rescale():
    # scores growing along the sequence move the row reference many times
    q, k, v = workloads.make_custom(1, 8400, 8400, 2, 2, 128, 128, seed=23)
    ramp = torch.linspace(0.2, 6.0, 8400)[None, :, None, None]
    c = Case(1, 8400, 8400, 2, 2, 128, 128, dtype="bf16", inputs=(q * 3.0, k * ramp, v))
    assert _uses_pair_kernel(c)
    check_against_oracle(c, rows=_rows(1, 2, 8400))


def test_pair_kernel_bitwise_deterministic():
    c = Case(1, 9000, 9000, 4, 2, 128, 128, dtype="bf16", seed=8)
    assert _uses_pair_kernel(c)
    run = c.runner()
    o0, l0 = run()
    o, l = torch.empty_like(o0), torch.empty_like(l0)
    for _ in range(10):
        run(out=o, lse=l)
        assert torch.equal(o.view(torch.int16), o0.view(torch.int16))
        assert torch.equal(l.view(torch.int32), l0.view(torch.int32))


@pytest.mark.parametrize("tile", [63, 64])
def test_pair_kernel_debug_dump_is_qk_and_p(tile):
    # tile 63 is team 1 of pair 31, tile 64 team 0 of the one-tile pair 32:
    # the dump holds that tile's raw scores for keys 0..127 and the bf16 P
    # words written for them
    import bf16_causal_prefill_02_b200 as zq

    Sq = 8320
    c = Case(1, Sq, Sq, 1, 1, 128, 128, dtype="bf16", seed=31)
    assert _uses_pair_kernel(c)
    dbg = torch.zeros(zq.ZQ_DEBUG_BYTES // 4, dtype=torch.float32, device="cuda")
    c.run_gpu(debug=dbg, debug_at=(0, tile))
    torch.cuda.synchronize()
    d = dbg.cpu()
    S = d[: 128 * 128].numpy().reshape(128, 128).astype(np.float64)
    P = d[128 * 128: 128 * 128 + 128 * 64].view(torch.int32).numpy().view(np.uint32).reshape(128, 64)
    rows = c.qd[0, 128 * tile: 128 * tile + 128, 0]
    ref = rows @ c.kd[0, :128, 0].T
    assert np.abs(S - ref).max() / np.abs(ref).max() < 1e-5
    # P: bf16 of exp2(y - yref).  Every key of these rows is visible (their
    # diagonal is far away), so P > 0; the first key tile sets the reference
    # to its row maximum (P <= 1 there), and the lazy reference lets a later
    # tile's maximum exceed it by at most 8 in log2 (P <= 2^8)
    p = (P.astype(np.uint64)[:, :, None] >> np.array([0, 16], dtype=np.uint64)) & 0xFFFF
    pf = (p.astype(np.uint32) << 16).view(np.float32).reshape(128, 128).astype(np.float64)
    assert np.all(pf > 0) and np.all(pf[:, :64] <= 1.0) and np.all(pf <= 256.0)
    assert np.all(pf[:, :64].max(axis=1) > 0.99)  # the row maximum of tile 0 maps to 1
    # inside one key tile (one reference) the ratio of two keys' P is exp of
    # their score difference, up to two bf16 roundings (8 significant bits:
    # relative 2^-8 each) and the exp2 error (< 1e-4 each)
    y = S * c.scale
    ratio = pf[:, 0::2] / pf[:, 1::2]
    want = np.exp(y[:, 0::2] - y[:, 1::2])
    assert np.all(np.abs(np.log(ratio / want)) < 2.0 ** -7 + 2e-4)


def test_pair_kernel_timeout_path_reports_status_and_context_survives():
    # flag 1: the issuers withhold all work, every other role's bounded wait
    # runs out, the kernel writes ZQ_ERR_TIMEOUT and returns
    import bf16_causal_prefill_02_b200 as zq

    c = Case(1, 8320, 8320, 1, 1, 128, 128, dtype="bf16", seed=4)
    assert _uses_pair_kernel(c)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    dbg = torch.zeros(zq.ZQ_DEBUG_BYTES // 4, dtype=torch.int32, device="cuda")
    c.run_gpu(debug=dbg, status=st, debug_flags=1)
    torch.cuda.synchronize()
    assert int(st.item()) == zq.ZQ_ERR_TIMEOUT
    check_against_oracle(c, rows=_rows(1, 1, 8320, every=331))
