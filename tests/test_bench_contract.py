"""The bench.py contract on the host: the reference arm (the oracle on host
cores) prints one JSON line with the keys the driver reads, and exits 0 on a
machine without a GPU; under a multi-rank launch only rank 0 prints."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(args, env_extra=None):
    env = dict(os.environ)
    env.update(env_extra or {})
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py")] + args, cwd=ROOT, env=env,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    return [json.loads(l) for l in r.stdout.splitlines() if l.startswith("{")]


def test_reference_arm_line():
    lines = _run(["--impl", "reference", "--workload", "tiny", "--steps", "3", "--warmup", "1"])
    assert len(lines) == 1
    r = lines[0]
    assert r["impl"] == "reference"
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in r, key
    assert r["unit"] == "TFLOP/s" and r["higher_is_better"] is True
    assert r["steps"] == 3 and r["warmup"] == 1
    assert r["value"] > 0 and r["cpu_baseline"]["value"] == r["value"]
    assert r["cpu_baseline"]["kind"] == "oracle" and r["cpu_baseline"]["cores"] >= 1
    assert r["e2e"] == {"value": r["value"], "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}
    assert r["config"]["workload"] == "tiny_leanp"


def test_reference_arm_other_ranks_are_silent():
    lines = _run(["--impl", "reference", "--workload", "tiny", "--steps", "2", "--warmup", "1"],
                 {"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"})
    assert lines == []


def test_reference_arm_per_kv_head_scales():
    lines = _run(["--impl", "reference", "--workload", "tiny", "--steps", "2", "--warmup", "1",
                  "--descale", "kv", "--hadamard"])
    assert len(lines) == 1
    r = lines[0]
    assert r["config"]["workload"] == "tiny_leanp_hadamard_kvscale"
    assert r["value"] > 0 and r["cpu_baseline"]["kind"] == "oracle"


def test_traffic_is_reported_only_for_the_kernel_it_was_taken_on():
    sys.path.insert(0, ROOT)
    import bench

    files = {"attn_fwd.cu": b"kernel", "sm100_ptx.cuh": b"ptx", "zq_internal.h": b"params"}

    def read(n):
        return list(files) if n is None else files[n]
    d0 = bench.kernel_sources_digest(read)
    assert d0 == bench.kernel_sources_digest(read)
    files["attn_fwd.cu"] = b"kernel, changed"
    assert bench.kernel_sources_digest(read) != d0
    # the recorded figures carry the digest of the sources they were taken on
    val, stale = bench.load_traffic("gauss_leanp_S32768")
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
        rec = json.load(f)
    if rec["_kernel_sources_sha256"] == bench.kernel_sources_digest():
        assert val == rec["gauss_leanp_S32768"] and stale is None
    else:
        assert val is None and stale == rec["gauss_leanp_S32768"]
    assert bench.load_traffic("no_such_workload") == (None, None)


def test_reference_arm_config_matches_ours():
    # both arms describe the workload with the same function, so the driver
    # sees identical config dicts for the same command line
    sys.path.insert(0, ROOT)
    import argparse

    import bench
    import workloads

    lines = _run(["--impl", "reference", "--workload", "tiny", "--steps", "2", "--warmup", "1"])
    args = argparse.Namespace(dtype="leanp", hadamard=False, descale="tensor", T=8)
    ours = bench.config_dict(workloads.get("tiny"), args, 1)
    assert lines[0]["config"] == ours
    for key in ("block_scale", "headroom_T", "step", "l2", "parallelism"):
        assert key in ours
    assert lines[0]["cpu_baseline"]["cpu_model"]


def test_attention_kernel_name_follows_the_library_dispatch():
    # the bench names the kernel the library runs: the paired kernel for
    # BF16 at d = 128 beyond 64 query tiles, the single-tile one otherwise
    # (zq_attn_plan_launch reports the same choice as rows_per_unit)
    import bench
    import bf16_causal_prefill_02_b200 as zq

    for kind, dqk, S in (("bf16", 128, 32768), ("bf16", 128, 8192), ("bf16", 128, 8193), ("bf16", 192, 16384),
                         ("fp8", 128, 32768), ("fp8", 192, 16384)):
        plan, _ = zq.attn_plan(1, S, S, 2, 2, d_qk=dqk,
                               dtype=zq.ZQ_DTYPE_BF16 if kind == "bf16" else zq.ZQ_DTYPE_FP8_E4M3)
        want = "attn_pp_kernel" if plan.rows_per_unit == 256 else "attn_fwd_kernel"
        assert bench.attention_kernel_name(kind, dqk, S) == want, (kind, dqk, S)
