"""GPU parity of the FP8 quantiser against the oracle's quantiser: bitwise
identical codes and descale, with and without the fused Hadamard rotation."""
import numpy as np
import pytest
import torch

import oracle
import workloads

pytestmark = pytest.mark.gpu


def _run(x32: torch.Tensor, src: str, hadamard: bool):
    import bf16_causal_prefill_02_b200 as zq

    if src == "bf16":
        xb = x32.to(torch.bfloat16)
        ref_in = xb.view(torch.int16).numpy().view(np.uint16)
        xg = xb.cuda()
    else:
        ref_in = x32.numpy()
        xg = x32.cuda()
    codes, ds = zq.quantize_fp8(xg, hadamard=hadamard)
    torch.cuda.synchronize()
    rc, rds = oracle.quantize_fp8(ref_in, hadamard=hadamard)
    return codes.view(torch.uint8).cpu().numpy(), float(ds.cpu()[0]), rc, float(rds)


@pytest.mark.parametrize("hadamard", [False, True])
@pytest.mark.parametrize("src", ["f32", "bf16"])
@pytest.mark.parametrize("n_vec,d", [(1000, 128), (1, 128), (4097, 256)])
def test_quantize_bitwise(n_vec, d, src, hadamard):
    x = torch.randn((n_vec, d), generator=torch.Generator().manual_seed(n_vec + d)) * 3.0
    g, gds, r, rds = _run(x, src, hadamard)
    assert gds == rds
    assert np.array_equal(g, r), "%d of %d codes differ" % (int((g != r).sum()), g.size)


@pytest.mark.parametrize("n_vec,d", [(333, 192), (5, 8), (7, 24)])
def test_quantize_bitwise_other_widths(n_vec, d):
    x = torch.randn((n_vec, d), generator=torch.Generator().manual_seed(d))
    g, gds, r, rds = _run(x, "f32", False)
    assert gds == rds and np.array_equal(g, r)


@pytest.mark.parametrize("src", ["f32", "bf16"])
@pytest.mark.parametrize("n_vec", [1, 333, 20000])
def test_quantize_d192_rotation_bitwise(n_vec, src):
    # MLA queries/keys: H128 on channels 0..127, sqrt2 * H64 on 128..191;
    # one warp per vector, more vectors than the grid covers at 20000
    x = torch.randn((n_vec, 192), generator=torch.Generator().manual_seed(n_vec)) * 2.0
    x[0, 150] = 40.0  # an outlier in the 64-channel slice
    g, gds, r, rds = _run(x, src, True)
    assert gds == rds
    assert np.array_equal(g, r), "%d of %d codes differ" % (int((g != r).sum()), g.size)


def test_quantize_empty_and_zero():
    import bf16_causal_prefill_02_b200 as zq

    codes, ds = zq.quantize_fp8(torch.zeros((0, 128), device="cuda"))
    torch.cuda.synchronize()
    assert float(ds.cpu()[0]) == 0.0
    codes, ds = zq.quantize_fp8(torch.zeros((64, 128), device="cuda"))
    assert float(ds.cpu()[0]) == 0.0 and not codes.view(torch.uint8).any()


def test_quantize_outliers_saturate_nothing():
    x = torch.randn((512, 128), generator=torch.Generator().manual_seed(3))
    x[7, 5] = 1e4
    x[100, 64] = -3e4
    g, gds, r, rds = _run(x, "f32", False)
    assert gds == rds and np.array_equal(g, r)
    assert g.reshape(-1)[100 * 128 + 64] == 0xFE


@pytest.mark.parametrize("hadamard", [False, True])
def test_quantize_full_size_q_at_32k(hadamard):
    """The Gaussian 32K workload's Q (32768 x 32 heads x 128): the size the
    benchmark quantises every step."""
    w = workloads.get("gauss")
    g = torch.Generator().manual_seed(w.seed)
    x = torch.randn((w.B * w.S * w.Hq, w.dqk), generator=g)
    gc, gds, rc, rds = _run(x, "f32", hadamard)
    assert gds == rds
    assert np.array_equal(gc, rc)


def test_quantize_repeatable():
    import bf16_causal_prefill_02_b200 as zq

    x = torch.randn((2048, 128), generator=torch.Generator().manual_seed(9)).cuda()
    outs = [zq.quantize_fp8(x, hadamard=True) for _ in range(5)]
    torch.cuda.synchronize()
    c0 = outs[0][0].view(torch.uint8)
    for c, d in outs[1:]:
        assert torch.equal(c.view(torch.uint8), c0) and torch.equal(d, outs[0][1])


@pytest.mark.parametrize("B,S,H,d,g,src,hadamard", [
    (2, 300, 8, 128, 4, "f32", False),    # queries of 8:2 GQA
    (2, 300, 8, 128, 1, "bf16", True),    # keys, rotated
    (1, 257, 4, 192, 2, "f32", True),     # MLA width, d = 192 rotation
    (2, 50, 16, 192, 4, "bf16", True),
    (2, 100, 6, 192, 3, "bf16", False),   # rows not a whole number of 128-slices
    (3, 1, 2, 64, 1, "f32", False),
    (1, 1000, 32, 128, 8, "f32", True),   # more items than the grid covers
    (4, 17, 3, 8, 3, "f32", False),
])
def test_quantize_grouped_bitwise(B, S, H, d, g, src, hadamard):
    # one scale per (batch, group of g heads): codes and descales bit-identical
    # to the oracle, which quantises each slot as a tensor of its own
    import bf16_causal_prefill_02_b200 as zq

    gen = torch.Generator().manual_seed(B * 1000 + S + H + d + g)
    x = torch.randn((B, S, H, d), generator=gen)
    # heads far apart in magnitude, so that every slot has its own scale
    x *= torch.pow(2.0, torch.randint(-6, 7, (B, 1, H, 1), generator=gen).float())
    if src == "bf16":
        xb = x.to(torch.bfloat16)
        ref_in = xb.view(torch.int16).numpy().view(np.uint16)
        xg = xb.cuda()
    else:
        ref_in = x.numpy()
        xg = x.cuda()
    codes, ds = zq.quantize_fp8_grouped(xg, heads_per_scale=g, hadamard=hadamard)
    torch.cuda.synchronize()
    rc, rds = oracle.quantize_fp8_grouped(ref_in, heads_per_scale=g, hadamard=hadamard)
    assert tuple(ds.shape) == (B, H // g)
    assert np.array_equal(ds.cpu().numpy(), rds)
    got = codes.view(torch.uint8).cpu().numpy()
    assert np.array_equal(got, rc), "%d of %d codes differ" % (int((got != rc).sum()), rc.size)


def test_quantize_grouped_empty_sequence():
    import bf16_causal_prefill_02_b200 as zq

    codes, ds = zq.quantize_fp8_grouped(torch.zeros((2, 0, 4, 128), device="cuda"), heads_per_scale=2)
    torch.cuda.synchronize()
    assert codes.numel() == 0 and ds.shape == (2, 2) and not ds.cpu().any()


@pytest.mark.parametrize("case", [
    # (shape, src, hadamard) per tensor: Q, K, V of an attention call
    [((2, 300, 4, 128), "f32", True), ((2, 300, 2, 128), "f32", True), ((2, 300, 2, 128), "f32", False)],
    [((1, 257, 2, 192), "bf16", True), ((1, 257, 2, 192), "f32", True), ((1, 257, 2, 128), "bf16", False)],
    [((4096, 32, 128), "f32", False)],
    [((0, 128), "f32", False), ((5, 8), "f32", False), ((33, 256), "bf16", True), ((1, 192), "f32", True)],
])
def test_quantize_multi_bitwise_equals_oracle_per_tensor(case):
    # one call for several tensors: every tensor's codes and descale are the
    # oracle's quantiser applied to that tensor alone (mixed dtypes, the
    # rotation on some, d = 192, an empty tensor)
    import bf16_causal_prefill_02_b200 as zq

    xs, refs, flags = [], [], []
    for k, (shape, src, had) in enumerate(case):
        x = torch.randn(shape, generator=torch.Generator().manual_seed(11 + k)) * (1.0 + 3 * k)
        if src == "bf16":
            xb = x.to(torch.bfloat16)
            refs.append(oracle.quantize_fp8(xb.view(torch.int16).numpy().view(np.uint16), hadamard=had))
            xs.append(xb.cuda())
        else:
            refs.append(oracle.quantize_fp8(x.numpy(), hadamard=had))
            xs.append(x.cuda())
        flags.append(had)
    for _ in range(2):  # the workspace keeps the last call's words: twice in a row
        codes, ds = zq.quantize_fp8_multi(xs, hadamard=flags)
        torch.cuda.synchronize()
        for c, d, (rc, rds) in zip(codes, ds, refs):
            assert float(d.cpu()[0]) == float(rds)
            assert np.array_equal(c.view(torch.uint8).cpu().numpy().reshape(rc.shape), rc)


def test_quantize_multi_equals_three_single_calls_full_size():
    # the 32K Gaussian workload's Q, K, V: one multi call against three
    # per-tensor calls, byte for byte
    import bf16_causal_prefill_02_b200 as zq

    w = workloads.get("gauss")
    q, k, v = (t.cuda() for t in workloads.make_inputs(w))
    codes, ds = zq.quantize_fp8_multi([q, k, v], hadamard=[True, True, False])
    for x, had, c, d in zip((q, k, v), (True, True, False), codes, ds):
        c1, d1 = zq.quantize_fp8(x, hadamard=had)
        torch.cuda.synchronize()
        assert torch.equal(c.view(torch.uint8), c1.view(torch.uint8))
        assert torch.equal(d, d1)
