"""The kernels' software exp2 (Cody-Waite reduction + Remez minimax
polynomial) against CUDA's exp2f on the device, within the error bound the
fit reports (bf16_causal_prefill_02_b200/csrc/exp2_poly_fit.py)."""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

BOUND = {3: 7.6e-5 + 2e-7, 4: 2.8e-6 + 2e-7}


def _run(x: torch.Tensor, degree: int) -> np.ndarray:
    import bf16_causal_prefill_02_b200 as zq

    y = torch.empty_like(x)
    rc = zq.zq_debug_exp2(x.data_ptr(), y.data_ptr(), x.numel(), degree, torch.cuda.current_stream().cuda_stream)
    assert rc == zq.ZQ_OK
    torch.cuda.synchronize()
    return y.cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("degree", [3, 4])
def test_poly_exp2_within_remez_bound_of_cuda_exp2f(degree):
    g = torch.Generator().manual_seed(degree)
    x = torch.rand(1_000_003, generator=g) * 134.0 - 126.0  # [-126, 8]
    edges = torch.tensor([0.0, -0.5, 0.5, 1.5, -1.5, 8.0, -125.9, 7.999, -0.4999, 0.4999], dtype=torch.float32)
    x = torch.cat([x, edges]).cuda()
    ref = _run(x, 0)
    got = _run(x, degree)
    assert np.all(np.isfinite(got))
    rel = np.abs(got / ref - 1.0)
    assert rel.max() <= BOUND[degree], rel.max()


def test_poly_exp2_of_masked_scores_is_negligible():
    x = torch.tensor([-float("inf"), -1e30, -200.0, -127.0], device="cuda")
    for degree in (3, 4):
        got = _run(x, degree)
        assert np.all(got >= 0) and np.all(got <= 2.0 ** -125)
