"""Shared helpers for the GPU parity tests: build the kernel inputs on the CPU
(through the oracle's quantiser for FP8), run the CUDA path through the C ABI,
and evaluate the oracle on exactly the same inputs."""
from __future__ import annotations

import numpy as np
import torch

import oracle
import workloads

# Tolerances.  Against the exact fp64 reference R1 on the kernel inputs, the
# bounds are the ones the target states (rel-RMSE; BF16 also max-abs).
# Against the FP8 emulation R2 of the same mode the only differences left are
# fp32 accumulation order, ex2.approx vs exp2, and the final bf16 rounding of
# the output (half an ulp = 2^-9 relative, RMS ~1.1e-3 of each value).
TOL_R1 = {"bf16": 5e-3, "exact": 4e-2, "leanp": 6e-2}
TOL_R1_MAXABS_BF16 = 2e-2
TOL_R2 = 3e-3
TOL_LSE_BF16 = 2e-3   # vs R1 (fp32 row sum of unrounded p)
TOL_LSE_FP8 = 5e-3    # vs R2 of the same mode, for all but a few rows:
# a row's lse moves by one code step of its dominant p~ when the GPU's fp32
# score of that key lands on the other side of an e4m3 rounding boundary
# than the fp64 emulation: ln 2^(1/8) for Lean P (a code is 1/8 of a
# doubling), ln(1 + 1/8) for the exact mode (one mantissa step at the bottom
# of a binade).  Scores agree to ~1e-6, so such rows are rare: at most
# LSE_FLIP_FRAC of them may exceed TOL_LSE_FP8, none the mode's bound.
LSE_FLIP_BOUND = {"leanp": float(np.log(2.0) / 8.0), "exact": float(np.log(1.0 + 1.0 / 8.0))}
LSE_FLIP_FRAC = 1e-3
# Element bound vs R2: the GPU output is R2 rounded to bf16 (half an ulp)
# plus fp32 accumulation-order differences in O and the row sum;
# ulp(x) = 2^(floor(log2|x|) - 7) for bf16.  Measured on the tiny, S = 1000,
# S = 700 (std 1.5) and GQA 4K cases: at most 0.41 of (1 ulp + 1e-3 max|r2|).
# A code flip of a key that carries a few percent of its row's weight moves
# the row's output past that bound while its lse stays within TOL_LSE_FP8;
# such rows count with the lse flips against LSE_FLIP_FRAC, and no row may
# move by more than one code step of its whole weight:
# |o - r2| <= step * 2 max|v| (step 2^(1/8) - 1 for Lean P, 1/8 exact).
ELEM_ULPS = 2.0
ELEM_ABS = 1e-3
CODE_STEP = {"leanp": 2.0 ** 0.125 - 1.0, "exact": 0.125}


def bf16_ulp(x):
    a = np.abs(np.asarray(x, dtype=np.float64))
    return np.exp2(np.floor(np.log2(np.maximum(a, 1e-30))) - 7.0)


class Case:
    def __init__(self, B, Sq, Sk, Hq, Hkv, dqk, dv, dtype="bf16", causal=True, block_scale=True,
                 T=8, hadamard=False, seed=0, std=1.0, inputs=None, per_kv_descale=False):
        self.B, self.Sq, self.Sk, self.Hq, self.Hkv, self.dqk, self.dv = B, Sq, Sk, Hq, Hkv, dqk, dv
        self.dtype, self.causal, self.block_scale, self.T = dtype, causal, block_scale, T
        self.hadamard, self.seed, self.std = hadamard, seed, std
        self.per_kv_descale = per_kv_descale
        if inputs is None:
            inputs = workloads.make_custom(B, Sq, Sk, Hq, Hkv, dqk, dv, seed=seed, std=std)
        self.q32, self.k32, self.v32 = (t.contiguous() for t in inputs)
        self.scale = 1.0 / np.sqrt(dqk)
        self._prepare()

    @property
    def fp8(self):
        return self.dtype in ("exact", "leanp")

    def _prepare(self):
        if not self.fp8:
            self.qb, self.kb, self.vb = (t.to(torch.bfloat16) for t in (self.q32, self.k32, self.v32))
            self.qd, self.kd, self.vd = (t.to(torch.float64).numpy() for t in (self.qb, self.kb, self.vb))
            return
        if self.per_kv_descale:
            # one scale per (batch, kv head): the query heads of a kv head
            # share theirs
            enc = []
            for t, g, rot in ((self.q32, self.Hq // self.Hkv, self.hadamard), (self.k32, 1, self.hadamard),
                              (self.v32, 1, False)):
                enc.append(oracle.quantize_fp8_grouped(t.numpy(), heads_per_scale=g, hadamard=rot))
            (self.cq, self.dsq), (self.ck, self.dsk), (self.cv, self.dsv) = enc
            self.qd = oracle.dequant_grouped(self.cq, self.dsq)
            self.kd = oracle.dequant_grouped(self.ck, self.dsk)
            self.vd = oracle.dequant_grouped(self.cv, self.dsv)
            return
        enc = []
        for t, rot in ((self.q32, self.hadamard), (self.k32, self.hadamard), (self.v32, False)):
            codes, ds = oracle.quantize_fp8(t.numpy(), hadamard=rot)
            enc.append((codes, ds))
        (self.cq, self.dsq), (self.ck, self.dsk), (self.cv, self.dsv) = enc
        self.qd = oracle.dequant_e4m3(self.cq, float(self.dsq))
        self.kd = oracle.dequant_e4m3(self.ck, float(self.dsk))
        self.vd = oracle.dequant_e4m3(self.cv, float(self.dsv))

    # ------------------------------------------------------------ CUDA path
    def runner(self):
        """A function that launches the CUDA path on inputs uploaded once."""
        import bf16_causal_prefill_02_b200 as zq

        dev = "cuda"
        if not self.fp8:
            q, k, v = (t.to(dev) for t in (self.qb, self.kb, self.vb))

            def run(debug=None, status=None, out=None, lse=None, debug_at=(0, 0), debug_flags=0):
                return zq.attn_fwd(q, k, v, causal=self.causal, debug=debug, debug_at=debug_at, status=status,
                                   out=out, lse=lse, debug_flags=debug_flags)
            return run
        q, k, v = (torch.from_numpy(c).to(dev).view(torch.float8_e4m3fn) for c in (self.cq, self.ck, self.cv))
        dq, dk, dv = (torch.tensor(np.asarray(d, dtype=np.float32).reshape(-1), device=dev)
                      for d in (self.dsq, self.dsk, self.dsv))
        mode = zq.ZQ_SOFTMAX_EXACT if self.dtype == "exact" else zq.ZQ_SOFTMAX_LEANP

        def run(debug=None, status=None, out=None, lse=None, debug_at=(0, 0), debug_flags=0):
            return zq.attn_fwd(q, k, v, causal=self.causal, q_descale=dq, k_descale=dk, v_descale=dv,
                               softmax_mode=mode, block_scale=self.block_scale, headroom_T=self.T,
                               debug=debug, debug_at=debug_at, status=status, out=out, lse=lse,
                               debug_flags=debug_flags)
        return run

    def run_gpu(self, debug=None, status=None, out=None, lse=None, debug_at=(0, 0), debug_flags=0):
        return self.runner()(debug=debug, status=status, out=out, lse=lse, debug_at=debug_at,
                             debug_flags=debug_flags)

    # --------------------------------------------------------------- oracle
    def r1(self, rows=None):
        return oracle.attn_ref(self.qd, self.kd, self.vd, scale=self.scale, causal=self.causal, rows=rows)

    def r2(self, rows=None):
        mode = oracle.MODE_EXACT if self.dtype == "exact" else oracle.MODE_LEANP
        return oracle.attn_fp8_emul(self.qd, self.kd, self.vd, scale=self.scale, causal=self.causal,
                                    mode=mode, block_scale=self.block_scale, T=self.T, rows=rows)

    def gather(self, o, lse, rows):
        """Pick flat rows (b*Hq+h)*Sq+i out of GPU outputs."""
        rows = np.asarray(rows)
        b, rem = rows // (self.Hq * self.Sq), rows % (self.Hq * self.Sq)
        h, i = rem // self.Sq, rem % self.Sq
        o = o.float().cpu().numpy().astype(np.float64)
        lse = lse.cpu().numpy().astype(np.float64)
        return o[b, i, h], lse[b, h, i]


def check_against_oracle(case: Case, rows=None, o_gpu=None, lse_gpu=None, gate_r1=True):
    """Run the CUDA path (unless outputs are given) and assert the tolerances.
    gate_r1=False keeps only the emulation gate (R2) for FP8: options away
    from the default headroom change the method's own error, which R2
    reproduces.  Returns a dict of measured errors."""
    if o_gpu is None:
        o_gpu, lse_gpu = case.run_gpu()
        torch.cuda.synchronize()
    if rows is None:
        o = o_gpu.float().cpu().numpy().astype(np.float64)
        l = lse_gpu.cpu().numpy().astype(np.float64)
        r1o, r1l = case.r1()
    else:
        o, l = case.gather(o_gpu, lse_gpu, rows)
        r1o, r1l = case.r1(rows)
    assert np.all(np.isfinite(o)), "non-finite output"
    res = {"r1": oracle.rel_rmse(o, r1o)}
    empty = np.isneginf(r1l)
    assert np.array_equal(np.isneginf(l), empty), "empty-row lse mismatch"
    emp_o = empty.transpose(0, 2, 1) if rows is None else empty
    assert np.all(o[emp_o] == 0), "rows without visible keys must be zero"
    fin = ~empty
    if not case.fp8:
        res["maxabs"] = float(np.max(np.abs(o - r1o))) if o.size else 0.0
        res["lse"] = float(np.max(np.abs(l[fin] - r1l[fin]))) if fin.any() else 0.0
        assert res["r1"] <= TOL_R1["bf16"], res
        assert res["maxabs"] <= TOL_R1_MAXABS_BF16, res
        assert res["lse"] <= TOL_LSE_BF16, res
    else:
        r2o, r2l = case.r2(rows)
        res["r2"] = oracle.rel_rmse(o, r2o)
        dl = np.abs(l[fin] - r2l[fin])
        res["lse"] = float(dl.max()) if fin.any() else 0.0
        res["lse_frac_over"] = float(np.mean(dl > TOL_LSE_FP8)) if fin.any() else 0.0
        # element by element, rows in (b, h, i) order as the lse
        if rows is None:
            og = o.transpose(0, 2, 1, 3).reshape(-1, o.shape[-1])
            rg = r2o.transpose(0, 2, 1, 3).reshape(-1, r2o.shape[-1])
        else:
            og, rg = o, r2o
        flip = np.zeros(l.size, dtype=bool)
        flip[fin.reshape(-1)] = dl.reshape(-1) > TOL_LSE_FP8
        if rg.size:
            bound = ELEM_ULPS * bf16_ulp(rg) + ELEM_ABS * np.abs(rg).max()
            over = (np.abs(og - rg) / bound).max(axis=1) > 1.0
            hard = CODE_STEP[case.dtype] * 2.0 * float(np.abs(case.vd).max())
            res["elem_max"] = float(np.abs(og - rg).max())
        else:
            over, hard = np.zeros(0, dtype=bool), 0.0
            res["elem_max"] = 0.0
        res["flip_rows"] = float(np.mean(flip | over)) if l.size else 0.0
        if gate_r1:
            assert res["r1"] <= TOL_R1[case.dtype], res
        assert res["r2"] <= TOL_R2, res
        assert res["lse"] <= LSE_FLIP_BOUND[case.dtype], res
        assert res["flip_rows"] <= LSE_FLIP_FRAC, res
        assert res["elem_max"] <= hard, res
    return res
