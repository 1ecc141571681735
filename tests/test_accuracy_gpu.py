"""End-to-end accuracy of the FP8 path against fp64 attention on the
unquantised fp32 inputs, with and without the Hadamard rotation of Q and K.

This is the pages' accuracy notion (error of the FP8 kernel against an fp64
reference: [P1] lefilia.fr paragraph 2; [P2] aicronaca.it "I numeri
dichiarati"), and the place where the rotation ([P2] "Perche l'FP8 non basta
da solo": it roughly halves the input quantisation error) can show.  The
inputs go through the product path: the GPU quantiser, then the attention
kernel; the error is measured on sampled rows of the full-size workloads.
The parity gates (against the oracle on the kernel's own inputs) live in
test_attn_gpu.py; here the GPU's end-to-end error must also match the
oracle emulation's end-to-end error on the same rows, since both see the
same quantised bytes."""
import numpy as np
import pytest
import torch

import oracle
import workloads

pytestmark = pytest.mark.gpu

_cache = {}


def _workload(name):
    if name not in _cache:
        w = workloads.get(name)
        q, k, v = workloads.make_inputs(w)
        rows = workloads.sample_rows(w.B, w.Hq, w.S, every=max(64, w.S // 32)).numpy()
        ref, _ = oracle.attn_ref(*(t.numpy().astype(np.float64) for t in (q, k, v)), rows=rows)
        _cache.clear()
        _cache[name] = (w, (q, k, v), rows, ref)
    return _cache[name]


def _errors(name, dtype, hadamard):
    import bf16_causal_prefill_02_b200 as zq

    w, (q, k, v), rows, ref = _workload(name)
    qg, kg, vg = q.cuda(), k.cuda(), v.cuda()
    (qc, kc, vc), (dq, dk, dv) = zq.quantize_fp8_multi([qg, kg, vg], hadamard=[hadamard, hadamard, False])
    mode = zq.ZQ_SOFTMAX_EXACT if dtype == "exact" else zq.ZQ_SOFTMAX_LEANP
    o, _ = zq.attn_fwd(qc, kc, vc, q_descale=dq, k_descale=dk, v_descale=dv, softmax_mode=mode)
    torch.cuda.synchronize()
    b, rem = rows // (w.Hq * w.S), rows % (w.Hq * w.S)
    h, i = rem // w.S, rem % w.S
    og = o.float().cpu().numpy().astype(np.float64)[b, i, h]
    # the oracle on the same quantised bytes (GPU quantiser == oracle R3)
    deq = [oracle.dequant_e4m3(c.view(torch.uint8).cpu().numpy(), float(d.cpu()[0]))
           for c, d in ((qc, dq), (kc, dk), (vc, dv))]
    r2, _ = oracle.attn_fp8_emul(*deq, rows=rows,
                                 mode=oracle.MODE_EXACT if dtype == "exact" else oracle.MODE_LEANP)
    return oracle.rel_rmse(og, ref), oracle.rel_rmse(r2, ref)


@pytest.mark.parametrize("dtype", ["exact", "leanp"])
@pytest.mark.parametrize("name", ["long_shared", "long", "gqa"])
def test_error_vs_unquantised_inputs(name, dtype):
    e0, r0 = _errors(name, dtype, False)
    e1, r1 = _errors(name, dtype, True)
    print("%s %s vs fp64 on the fp32 inputs: plain %.4f (oracle %.4f), rotated %.4f (oracle %.4f)"
          % (name, dtype, e0, r0, e1, r1))
    # the kernel's end-to-end error is the method's own (its deviation from
    # the emulation is far below the quantisation error)
    assert abs(e0 - r0) <= 0.02 * r0 + 1e-3 and abs(e1 - r1) <= 0.02 * r1 + 1e-3
    if name == "long_shared":
        # outlier channels shared by Q and K: the rotation spreads them over
        # all channels, and the error falls well below half
        assert e1 < 0.5 * e0, (e0, e1)
