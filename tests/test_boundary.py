"""C-ABI boundary checks that need no GPU: the library loads, exports every
function include/zattn.h declares, and rejects bad arguments with the
documented status before touching the device.

No test here passes a fake pointer together with otherwise valid arguments,
so nothing can reach a kernel launch on a machine that has a GPU.
"""
import ctypes
import os

import pytest

import bf16_causal_prefill_02_b200 as zq


def test_library_exports_every_header_function():
    names = zq.header_functions()
    assert set(names) >= {"zq_attn_fwd", "zq_attn_fwd_ex", "zq_quantize_fp8",
                          "zq_quantize_workspace_bytes", "zq_status_string", "zq_version"}
    lib = ctypes.CDLL(zq.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n


def test_status_strings_and_version():
    for s in range(0, -8, -1):
        assert zq.zq_status_string(s) and zq.zq_status_string(s) != "unknown status"
    assert zq.zq_status_string(-99) == "unknown status"
    assert zq.zq_version() >= 100
    assert zq.zq_quantize_workspace_bytes() >= 4


A = 1 << 20  # a 16-byte aligned address that is never dereferenced


def _args(**kw):
    a = zq.zq_attn_args()
    d = dict(q=A, k=A, v=A, out=A, lse=None, B=1, Sq=128, Sk=128, Hq=2, Hkv=1, d_qk=128, d_v=128,
             softmax_scale=0.0, causal=1, dtype=zq.ZQ_DTYPE_BF16, q_descale=None, k_descale=None,
             v_descale=None, softmax_mode=zq.ZQ_SOFTMAX_LEANP, block_scale=1, headroom_T=8, status=None,
             descale_layout=0)
    d.update(kw)
    for k, v in d.items():
        setattr(a, k, v)
    return a


@pytest.mark.parametrize("kw,code", [
    (dict(q=None), zq.ZQ_ERR_NULL),
    (dict(k=None), zq.ZQ_ERR_NULL),
    (dict(v=None), zq.ZQ_ERR_NULL),
    (dict(out=None), zq.ZQ_ERR_NULL),
    (dict(B=0), zq.ZQ_ERR_SHAPE),
    (dict(Sq=-1), zq.ZQ_ERR_SHAPE),
    (dict(Sk=0), zq.ZQ_ERR_SHAPE),
    (dict(Hq=3, Hkv=2), zq.ZQ_ERR_SHAPE),
    (dict(Hkv=0), zq.ZQ_ERR_SHAPE),
    (dict(d_qk=64, d_v=64), zq.ZQ_ERR_UNSUPPORTED),
    (dict(d_qk=128, d_v=192), zq.ZQ_ERR_UNSUPPORTED),
    (dict(d_qk=256, d_v=128), zq.ZQ_ERR_UNSUPPORTED),
    (dict(dtype=2), zq.ZQ_ERR_UNSUPPORTED),
    (dict(dtype=1, softmax_mode=2), zq.ZQ_ERR_UNSUPPORTED),
    (dict(dtype=1, block_scale=2), zq.ZQ_ERR_UNSUPPORTED),
    (dict(dtype=1, headroom_T=9), zq.ZQ_ERR_UNSUPPORTED),
    (dict(dtype=1, headroom_T=-1), zq.ZQ_ERR_UNSUPPORTED),
    (dict(dtype=1, descale_layout=2), zq.ZQ_ERR_UNSUPPORTED),
    (dict(dtype=1, descale_layout=-1), zq.ZQ_ERR_UNSUPPORTED),
    (dict(q=A + 8), zq.ZQ_ERR_ALIGN),
    (dict(out=A + 2), zq.ZQ_ERR_ALIGN),
    (dict(lse=A + 4), zq.ZQ_ERR_ALIGN),
    (dict(softmax_scale=float("nan")), zq.ZQ_ERR_SHAPE),
    (dict(B=65536, Sq=1 << 20, Hq=64, Hkv=64), zq.ZQ_ERR_SHAPE),
])
def test_attn_argument_errors(kw, code):
    assert zq.zq_attn_fwd_ex(_args(**kw), None) == code


def test_attn_plain_entry_validates_too():
    rc = zq.zq_attn_fwd(A, A, A, None, None, 1, 128, 128, 2, 1, 128, 128, 0.0, 1, 0, None, None, None, None)
    assert rc == zq.ZQ_ERR_NULL
    rc = zq.zq_attn_fwd(A, A, A, A, None, 1, 128, 128, 3, 2, 128, 128, 0.0, 1, 0, None, None, None, None)
    assert rc == zq.ZQ_ERR_SHAPE


@pytest.mark.parametrize("args,code", [
    ((None, 0, 4, 128, 0, A, A, A), zq.ZQ_ERR_NULL),
    ((A, 0, 4, 128, 0, None, A, A), zq.ZQ_ERR_NULL),
    ((None, 0, 0, 128, 0, None, None, A), zq.ZQ_ERR_NULL),
    ((A, 0, 4, 128, 0, A, None, A), zq.ZQ_ERR_NULL),
    ((A, 0, 4, 128, 0, A, A, None), zq.ZQ_ERR_NULL),
    ((A, 0, -1, 128, 0, A, A, A), zq.ZQ_ERR_SHAPE),
    ((A, 0, 4, 0, 0, A, A, A), zq.ZQ_ERR_SHAPE),
    ((A, 2, 4, 128, 0, A, A, A), zq.ZQ_ERR_UNSUPPORTED),
    ((A, 0, 4, 12, 0, A, A, A), zq.ZQ_ERR_UNSUPPORTED),
    ((A, 0, 4, 320, 1, A, A, A), zq.ZQ_ERR_UNSUPPORTED),  # rotation: d % 128 == 0 or d == 192
    ((A + 4, 0, 4, 128, 0, A, A, A), zq.ZQ_ERR_ALIGN),
    ((A, 0, 4, 128, 0, A + 1, A, A), zq.ZQ_ERR_ALIGN),
    ((A, 0, 4, 128, 0, A, A, A + 8), zq.ZQ_ERR_ALIGN),
])
def test_quantize_argument_errors(args, code):
    x, xd, n, d, had, out, ds, ws = args
    assert zq.zq_quantize_fp8(x, xd, n, d, had, out, ds, ws, None) == code


@pytest.mark.parametrize("args,code", [
    # x, x_dtype, B, S, H, d, heads_per_scale, hadamard, x_fp8, descale, workspace
    ((A, 0, 2, 10, 8, 128, 2, 0, A, None, A), zq.ZQ_ERR_NULL),
    ((A, 0, 2, 10, 8, 128, 2, 0, A, A, None), zq.ZQ_ERR_NULL),
    ((None, 0, 2, 10, 8, 128, 2, 0, A, A, A), zq.ZQ_ERR_NULL),
    ((A, 0, 2, 10, 8, 128, 2, 0, None, A, A), zq.ZQ_ERR_NULL),
    ((A, 0, 0, 10, 8, 128, 2, 0, A, A, A), zq.ZQ_ERR_SHAPE),
    ((A, 0, 2, -1, 8, 128, 2, 0, A, A, A), zq.ZQ_ERR_SHAPE),
    ((A, 0, 2, 10, 0, 128, 1, 0, A, A, A), zq.ZQ_ERR_SHAPE),
    ((A, 0, 2, 10, 8, 0, 2, 0, A, A, A), zq.ZQ_ERR_SHAPE),
    ((A, 0, 2, 10, 8, 128, 0, 0, A, A, A), zq.ZQ_ERR_SHAPE),
    ((A, 0, 2, 10, 8, 128, 3, 0, A, A, A), zq.ZQ_ERR_SHAPE),      # H % g != 0
    ((A, 0, 70000, 10, 1, 128, 1, 0, A, A, A), zq.ZQ_ERR_SHAPE),  # > 65535 slots
    ((A, 2, 2, 10, 8, 128, 2, 0, A, A, A), zq.ZQ_ERR_UNSUPPORTED),
    ((A, 0, 2, 10, 8, 12, 2, 0, A, A, A), zq.ZQ_ERR_UNSUPPORTED),
    ((A, 0, 2, 10, 8, 320, 2, 1, A, A, A), zq.ZQ_ERR_UNSUPPORTED),
    ((A + 4, 0, 2, 10, 8, 128, 2, 0, A, A, A), zq.ZQ_ERR_ALIGN),
    ((A, 0, 2, 10, 8, 128, 2, 0, A + 1, A, A), zq.ZQ_ERR_ALIGN),
    ((A, 0, 2, 10, 8, 128, 2, 0, A, A, A + 8), zq.ZQ_ERR_ALIGN),
])
def test_quantize_grouped_argument_errors(args, code):
    assert zq.zq_quantize_fp8_grouped(*args, None) == code


def test_quantize_grouped_workspace_bytes():
    assert zq.zq_quantize_grouped_workspace_bytes(2, 8, 4) == 16     # 4 slots
    assert zq.zq_quantize_grouped_workspace_bytes(3, 8, 1) == 96     # 24 slots
    assert zq.zq_quantize_grouped_workspace_bytes(1, 5, 1) == 32     # 5 slots, rounded up
    assert zq.zq_quantize_grouped_workspace_bytes(2, 8, 3) == 0      # g does not divide H
    assert zq.zq_quantize_grouped_workspace_bytes(0, 8, 1) == 0
    assert zq.zq_quantize_grouped_workspace_bytes(70000, 1, 1) == 0  # too many slots


def test_descale_layout_from_tensor_sizes():
    import torch

    one, per = torch.ones(1), torch.ones(2 * 4)
    assert zq._descale_layout(2, 4, None, None, None) == zq.ZQ_DESCALE_PER_TENSOR
    assert zq._descale_layout(2, 4, one, one, None) == zq.ZQ_DESCALE_PER_TENSOR
    assert zq._descale_layout(2, 4, per, per, per) == zq.ZQ_DESCALE_PER_KV_HEAD
    assert zq._descale_layout(2, 4, per, None, per) == zq.ZQ_DESCALE_PER_KV_HEAD
    with pytest.raises(ValueError):
        zq._descale_layout(2, 4, one, per, per)
    with pytest.raises(ValueError):
        zq._descale_layout(2, 4, torch.ones(3), None, None)


def test_no_cpu_fallback_without_library(tmp_path, monkeypatch):
    # The binding must fail loudly when the shared library is missing.
    import importlib.util
    import shutil

    pkg = tmp_path / "zpkg"
    pkg.mkdir()
    shutil.copy(zq.__file__, pkg / "__init__.py")
    spec = importlib.util.spec_from_file_location("zpkg", pkg / "__init__.py")
    mod = importlib.util.module_from_spec(spec)
    with pytest.raises(ImportError):
        spec.loader.exec_module(mod)


def test_torch_helpers_reject_host_tensors():
    # the helpers never fall back to the CPU: host tensors are refused
    import torch

    x = torch.zeros((1, 4, 2, 128))
    with pytest.raises(ValueError):
        zq.quantize_fp8(x)
    with pytest.raises(ValueError):
        zq.quantize_fp8_grouped(x, heads_per_scale=1)
    with pytest.raises(ValueError):
        zq.attn_fwd(x.bfloat16(), x.bfloat16(), x.bfloat16())


def _bf(*shape):
    import torch

    return torch.zeros(shape, dtype=torch.bfloat16)


@pytest.mark.parametrize("q,k,v,msg", [
    ((1, 8, 2, 128), (2, 8, 1, 128), (1, 8, 1, 128), "same batch"),
    ((1, 8, 2, 128), (1, 8, 1, 128), (2, 8, 1, 128), "same batch"),
    ((1, 8, 2, 192), (1, 8, 1, 128), (1, 8, 1, 128), "head dim"),
    ((1, 8, 2, 128), (1, 8, 1, 128), (1, 9, 1, 128), "sequence length"),
    ((1, 8, 2, 128), (1, 8, 1, 128), (1, 8, 2, 128), "head count"),
    ((8, 2, 128), (1, 8, 1, 128), (1, 8, 1, 128), "4-D"),
])
def test_attn_helper_rejects_mismatched_qkv_before_launch(q, k, v, msg):
    # checked on the host before any device access (host tensors here)
    with pytest.raises(ValueError, match=msg):
        zq.attn_fwd(_bf(*q), _bf(*k), _bf(*v))


@pytest.mark.parametrize("kw,msg", [
    (dict(out=_bf(1, 8, 2, 64)), "out must have shape"),
    (dict(out=_bf(1, 8, 2, 128).float()), "out must be"),
    (dict(out=_bf(1, 8, 128, 2).transpose(2, 3)), "out must be contiguous"),
    (dict(lse=_bf(1, 2, 8).float()[:, :1]), "lse must have shape"),
    (dict(lse=_bf(1, 2, 8)), "lse must be"),
    (dict(status=_bf(1)), "status must be an int32"),
    (dict(debug=_bf(16)), "debug must hold"),
])
def test_attn_helper_rejects_bad_output_buffers(kw, msg):
    with pytest.raises(ValueError, match=msg):
        zq.attn_fwd(_bf(1, 8, 2, 128), _bf(1, 8, 1, 128), _bf(1, 8, 1, 128), **kw)


def test_attn_helper_rejects_bad_descales():
    import torch

    q = torch.zeros((1, 8, 2, 128), dtype=torch.uint8)
    k = torch.zeros((1, 8, 1, 128), dtype=torch.uint8)
    with pytest.raises(ValueError, match="k_descale must be a contiguous float32"):
        zq.attn_fwd(q, k, k, k_descale=torch.ones(1, dtype=torch.float64))
    with pytest.raises(ValueError, match="q_descale must be a CUDA tensor|must be a CUDA tensor"):
        zq.attn_fwd(q, k, k, q_descale=torch.ones(1))


def test_quantize_helpers_reject_bad_buffers():
    import torch

    x = torch.zeros((1, 4, 2, 128))
    # host x is refused first; a CUDA-less host cannot build a CUDA x, so the
    # buffer checks are exercised through the order of the checks instead:
    # a wrong `out` shape is reported by _check_buffer before any device test
    with pytest.raises(ValueError, match="out must have shape"):
        zq._check_buffer("out", torch.zeros((1, 4, 2, 64), dtype=torch.uint8), x.shape, torch.uint8)
    with pytest.raises(ValueError, match="descale must be"):
        zq._check_buffer("descale", torch.zeros(1, dtype=torch.float64), (1,), torch.float32)
    with pytest.raises(ValueError, match="must be a CUDA tensor"):
        zq._check_same_cuda_device(torch.device("cuda", 0), [("workspace", torch.zeros(4))])


def test_binding_has_no_library_override():
    # the binding loads exactly the in-tree library; no environment variable
    # can redirect it
    import inspect

    src = inspect.getsource(zq)
    assert "os.environ" not in src
    assert zq.LIB_PATH == os.path.join(os.path.dirname(zq.__file__), "libzattn.so")


def _qt(**kw):
    t = zq.zq_quant_tensor()
    d = dict(x=A, x_dtype=0, n_vec=4, d=128, hadamard=0, x_fp8=A, descale=A)
    d.update(kw)
    for k, v in d.items():
        setattr(t, k, v)
    return t


@pytest.mark.parametrize("items,count,ws,code", [
    ([{}], 0, A, zq.ZQ_ERR_SHAPE),
    ([{}] * 5, 5, A, zq.ZQ_ERR_SHAPE),
    ([{}], 1, None, zq.ZQ_ERR_NULL),
    ([{}, dict(descale=None)], 2, A, zq.ZQ_ERR_NULL),
    ([{}, dict(x=None)], 2, A, zq.ZQ_ERR_NULL),
    ([dict(n_vec=-1)], 1, A, zq.ZQ_ERR_SHAPE),
    ([{}, {}, dict(d=0)], 3, A, zq.ZQ_ERR_SHAPE),
    ([dict(x_dtype=2)], 1, A, zq.ZQ_ERR_UNSUPPORTED),
    ([{}, dict(d=12)], 2, A, zq.ZQ_ERR_UNSUPPORTED),
    ([dict(d=320, hadamard=1)], 1, A, zq.ZQ_ERR_UNSUPPORTED),
    ([{}, dict(x=A + 4)], 2, A, zq.ZQ_ERR_ALIGN),
    ([dict(x_fp8=A + 1)], 1, A, zq.ZQ_ERR_ALIGN),
    ([{}], 1, A + 8, zq.ZQ_ERR_ALIGN),
])
def test_quantize_multi_argument_errors(items, count, ws, code):
    arr = (zq.zq_quant_tensor * len(items))(*[_qt(**kw) for kw in items])
    assert zq.zq_quantize_fp8_multi(arr, count, ws, None) == code


def test_quantize_multi_workspace_bytes():
    assert zq.zq_quantize_multi_workspace_bytes() >= 16
