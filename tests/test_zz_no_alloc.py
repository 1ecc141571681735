"""The allocation-free quantiser entry point, zq_quantize_fp8_noalloc.

It exists for callers that cannot hand the library device scratch memory
(their device memory belongs to another allocator without a scratch API, or
they must not call cudaMalloc in a latency-critical loop); its scratch is a
fixed device array inside the library.  Its results must match the regular
entry point's bit for bit (the tolerance every quantiser test uses), call
after call, because the shared array keeps the previous call's contents.

This file is named to be collected last, so a failure here cannot hide
another test's result in a run that stops at the first failure.
"""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


def _regular(zq, x, xd, hadamard):
    d = x.shape[-1]
    out = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    ds = torch.empty(1, dtype=torch.float32, device=x.device)
    ws = torch.empty(zq.zq_quantize_workspace_bytes(), dtype=torch.uint8, device=x.device)
    rc = zq.zq_quantize_fp8(x.data_ptr(), xd, x.numel() // d, d, int(hadamard), out.data_ptr(),
                            ds.data_ptr(), ws.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert rc == zq.ZQ_OK, zq.zq_status_string(rc)
    return out, ds


def _noalloc(zq, x, xd, hadamard):
    d = x.shape[-1]
    out = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    ds = torch.empty(1, dtype=torch.float32, device=x.device)
    rc = zq.zq_quantize_fp8_noalloc(x.data_ptr(), xd, x.numel() // d, d, int(hadamard), out.data_ptr(),
                                    ds.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert rc == zq.ZQ_OK, zq.zq_status_string(rc)
    return out, ds


@pytest.mark.parametrize("hadamard", [False, True])
def test_noalloc_matches_regular_entry_two_calls_in_a_row(hadamard):
    import bf16_causal_prefill_02_b200 as zq

    assert zq.zq_quantize_noalloc_scratch_bytes() >= zq.zq_quantize_workspace_bytes()
    g = torch.Generator().manual_seed(123)
    # first input has a much larger maximum than the second: a scratch word
    # left over from call 1 would corrupt call 2
    x1 = (torch.randn((4096, 128), generator=g) * 50.0).cuda()
    x2 = (torch.randn((3000, 128), generator=g) * 0.5).to(torch.bfloat16).cuda()
    for x, xd in ((x1, zq.ZQ_X_F32), (x2, zq.ZQ_X_BF16)):
        ref_codes, ref_ds = _regular(zq, x, xd, hadamard)
        codes, ds = _noalloc(zq, x, xd, hadamard)
        torch.cuda.synchronize()
        assert torch.equal(ds, ref_ds)
        assert torch.equal(codes, ref_codes), "%d codes differ" % int((codes != ref_codes).sum())


def test_noalloc_rejects_bad_arguments_like_the_regular_entry():
    import bf16_causal_prefill_02_b200 as zq

    ds = torch.empty(1, dtype=torch.float32, device="cuda")
    x = torch.zeros((4, 128), device="cuda")
    out = torch.empty((4, 128), dtype=torch.uint8, device="cuda")
    s = torch.cuda.current_stream().cuda_stream
    assert zq.zq_quantize_fp8_noalloc(x.data_ptr(), 0, 4, 128, 0, out.data_ptr(), None, s) == zq.ZQ_ERR_NULL
    assert zq.zq_quantize_fp8_noalloc(x.data_ptr(), 0, 4, 320, 1, out.data_ptr(), ds.data_ptr(), s) == zq.ZQ_ERR_UNSUPPORTED
    assert zq.zq_quantize_fp8_noalloc(x.data_ptr() + 4, 0, 4, 128, 0, out.data_ptr(), ds.data_ptr(), s) == zq.ZQ_ERR_ALIGN
    # empty input: only the descale (0) is written
    assert zq.zq_quantize_fp8_noalloc(None, 0, 0, 128, 0, None, ds.data_ptr(), s) == zq.ZQ_OK
    torch.cuda.synchronize()
    assert float(ds.item()) == 0.0
