"""B200 (sm_100a) causal prefill attention in FP8 e4m3 and BF16.

A thin ctypes binding over ``libzattn.so`` (the C ABI in ``include/zattn.h``).
Every step of the computation runs in this package's CUDA kernels; PyTorch is
only used for device memory and streams.  There is no CPU fallback: if the
shared library is missing, importing this package raises.

Low-level names mirror the C ABI (``zq_attn_fwd``, ``zq_attn_fwd_ex``,
``zq_quantize_fp8``, ``zq_quantize_fp8_multi``, ``zq_quantize_fp8_grouped``,
``zq_attn_plan_launch``, ...) and take raw integers (device addresses, sizes,
a stream handle).  The torch-level helpers ``attn_fwd``, ``quantize_fp8``,
``quantize_fp8_multi``, ``quantize_fp8_grouped`` and ``flash_attn_func``
marshal tensors into those calls; ``attn_plan``
returns the schedule of a call (host only).
"""
from __future__ import annotations

import ctypes
import math
import os
import re

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libzattn.so")
HEADER_PATH = os.path.join(os.path.dirname(HERE), "include", "zattn.h")

ZQ_DTYPE_BF16, ZQ_DTYPE_FP8_E4M3 = 0, 1
ZQ_X_F32, ZQ_X_BF16 = 0, 1
ZQ_SOFTMAX_EXACT, ZQ_SOFTMAX_LEANP = 0, 1
ZQ_DESCALE_PER_TENSOR, ZQ_DESCALE_PER_KV_HEAD = 0, 1
ZQ_OK, ZQ_ERR_NULL, ZQ_ERR_SHAPE, ZQ_ERR_UNSUPPORTED = 0, -1, -2, -3
ZQ_ERR_ALIGN, ZQ_ERR_ARCH, ZQ_ERR_CUDA, ZQ_ERR_TIMEOUT = -4, -5, -6, -7


class ZQError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__("%s failed: %s (%d)" % (where, zq_status_string(status), status))
        self.status = status


class zq_attn_args(ctypes.Structure):
    _fields_ = [
        ("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
        ("out", ctypes.c_void_p), ("lse", ctypes.c_void_p),
        ("B", ctypes.c_int), ("Sq", ctypes.c_int), ("Sk", ctypes.c_int), ("Hq", ctypes.c_int),
        ("Hkv", ctypes.c_int), ("d_qk", ctypes.c_int), ("d_v", ctypes.c_int),
        ("softmax_scale", ctypes.c_float), ("causal", ctypes.c_int), ("dtype", ctypes.c_int),
        ("q_descale", ctypes.c_void_p), ("k_descale", ctypes.c_void_p), ("v_descale", ctypes.c_void_p),
        ("softmax_mode", ctypes.c_int), ("block_scale", ctypes.c_int), ("headroom_T", ctypes.c_int),
        ("status", ctypes.c_void_p), ("descale_layout", ctypes.c_int),
    ]


class zq_quant_tensor(ctypes.Structure):
    _fields_ = [
        ("x", ctypes.c_void_p), ("x_dtype", ctypes.c_int), ("n_vec", ctypes.c_int64), ("d", ctypes.c_int),
        ("hadamard", ctypes.c_int), ("x_fp8", ctypes.c_void_p), ("descale", ctypes.c_void_p),
    ]


class zq_attn_plan(ctypes.Structure):
    _fields_ = [
        ("n_units", ctypes.c_int64), ("grid", ctypes.c_int64), ("persistent", ctypes.c_int),
        ("head_group", ctypes.c_int), ("smem_bytes", ctypes.c_int), ("threads", ctypes.c_int),
        ("rows_per_unit", ctypes.c_int), ("keys_per_tile", ctypes.c_int),
    ]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            "libzattn.so not found at %s; build it with `python bf16_causal_prefill_02_b200/build.py`"
            % LIB_PATH
        )
    lib = ctypes.CDLL(LIB_PATH)
    P, i32, i64, f32 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float
    lib.zq_attn_fwd.argtypes = [P, P, P, P, P, i32, i32, i32, i32, i32, i32, i32, f32, i32, i32,
                                P, P, P, P]
    lib.zq_attn_fwd.restype = i32
    lib.zq_attn_fwd_ex.argtypes = [ctypes.POINTER(zq_attn_args), P]
    lib.zq_attn_fwd_ex.restype = i32
    lib.zq_attn_plan_launch.argtypes = [ctypes.POINTER(zq_attn_args), i32, ctypes.POINTER(zq_attn_plan),
                                        P, P, P, P, P]
    lib.zq_attn_plan_launch.restype = i32
    lib.zq_attn_fwd_debug.argtypes = [ctypes.POINTER(zq_attn_args), P, i32, i32, i32, P]
    lib.zq_attn_fwd_debug.restype = i32
    lib.zq_quantize_fp8.argtypes = [P, i32, i64, i32, i32, P, P, P, P]
    lib.zq_quantize_fp8.restype = i32
    lib.zq_quantize_fp8_multi.argtypes = [ctypes.POINTER(zq_quant_tensor), i32, P, P]
    lib.zq_quantize_fp8_multi.restype = i32
    lib.zq_quantize_multi_workspace_bytes.argtypes = []
    lib.zq_quantize_multi_workspace_bytes.restype = ctypes.c_size_t
    lib.zq_quantize_fp8_noalloc.argtypes = [P, i32, i64, i32, i32, P, P, P]
    lib.zq_quantize_fp8_noalloc.restype = i32
    lib.zq_quantize_fp8_grouped.argtypes = [P, i32, i32, i64, i32, i32, i32, i32, P, P, P, P]
    lib.zq_quantize_fp8_grouped.restype = i32
    lib.zq_quantize_grouped_workspace_bytes.argtypes = [i32, i32, i32]
    lib.zq_quantize_grouped_workspace_bytes.restype = ctypes.c_size_t
    lib.zq_quantize_noalloc_scratch_bytes.argtypes = []
    lib.zq_quantize_noalloc_scratch_bytes.restype = ctypes.c_size_t
    lib.zq_debug_exp2.argtypes = [P, P, i64, i32, P]
    lib.zq_debug_exp2.restype = i32
    lib.zq_quantize_workspace_bytes.argtypes = []
    lib.zq_quantize_workspace_bytes.restype = ctypes.c_size_t
    lib.zq_status_string.argtypes = [i32]
    lib.zq_status_string.restype = ctypes.c_char_p
    lib.zq_version.argtypes = []
    lib.zq_version.restype = i32
    return lib


_lib = _load()


def header_functions() -> list[str]:
    """Names of the functions include/zattn.h declares."""
    txt = open(HEADER_PATH).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(zq_[a-z0-9_]+)\s*\(", txt)))


# ------------------------------------------------------------------ C ABI names
def zq_attn_fwd(q, k, v, out, lse, B, Sq, Sk, Hq, Hkv, d_qk, d_v, softmax_scale, causal, dtype,
                q_descale, k_descale, v_descale, stream) -> int:
    return _lib.zq_attn_fwd(q, k, v, out, lse, B, Sq, Sk, Hq, Hkv, d_qk, d_v, softmax_scale,
                            causal, dtype, q_descale, k_descale, v_descale, stream)


def zq_attn_fwd_ex(args: zq_attn_args, stream) -> int:
    return _lib.zq_attn_fwd_ex(ctypes.byref(args), stream)


def zq_attn_plan_launch(args: zq_attn_args, num_sms, plan: zq_attn_plan, unit_tile=None, unit_bh=None,
                        unit_nkv=None, unit_cta=None, unit_round=None) -> int:
    """Host-only: the launch shape and per-unit schedule zq_attn_fwd_ex would
    use.  The unit_* arguments are host addresses of int32 arrays (or None)."""
    return _lib.zq_attn_plan_launch(ctypes.byref(args), num_sms, ctypes.byref(plan), unit_tile, unit_bh,
                                    unit_nkv, unit_cta, unit_round)


def attn_plan(B, Sq, Sk, Hq, Hkv, d_qk=128, d_v=128, dtype=ZQ_DTYPE_FP8_E4M3, causal=True, num_sms=148):
    """Schedule of an attention call on the host: (plan, units) with units a
    dict of numpy int32 arrays tile, bh, n_kv, cta, round indexed by unit."""
    import numpy as np

    a = zq_attn_args()
    fake = 1 << 20  # 16-byte aligned; the planner never dereferences it
    a.q = a.k = a.v = a.out = fake
    a.B, a.Sq, a.Sk, a.Hq, a.Hkv, a.d_qk, a.d_v = B, Sq, Sk, Hq, Hkv, d_qk, d_v
    a.causal, a.dtype = int(bool(causal)), dtype
    a.softmax_mode, a.block_scale, a.headroom_T = ZQ_SOFTMAX_LEANP, 1, 8
    plan = zq_attn_plan()
    _check(zq_attn_plan_launch(a, num_sms, plan), "zq_attn_plan_launch")
    n = int(plan.n_units)
    arrs = {k: np.full(n, -1, dtype=np.int32) for k in ("tile", "bh", "n_kv", "cta", "round")}
    _check(zq_attn_plan_launch(a, num_sms, plan, *(arrs[k].ctypes.data for k in ("tile", "bh", "n_kv", "cta", "round"))),
           "zq_attn_plan_launch")
    return plan, arrs


def zq_attn_fwd_debug(args: zq_attn_args, dbg, dbg_bh, dbg_qtile, flags, stream) -> int:
    return _lib.zq_attn_fwd_debug(ctypes.byref(args), dbg, dbg_bh, dbg_qtile, flags, stream)


ZQ_DEBUG_BYTES = 128 * 128 * 4 + 128 * 64 * 4 + 256 * 4 + 512 * 16 * 8


def zq_quantize_fp8(x, x_dtype, n_vec, d, hadamard, x_fp8, descale, workspace, stream) -> int:
    return _lib.zq_quantize_fp8(x, x_dtype, n_vec, d, hadamard, x_fp8, descale, workspace, stream)


def zq_quantize_fp8_multi(tensors, count, workspace, stream) -> int:
    """`tensors`: a ctypes array (or pointer) of zq_quant_tensor."""
    return _lib.zq_quantize_fp8_multi(tensors, count, workspace, stream)


def zq_quantize_multi_workspace_bytes() -> int:
    return int(_lib.zq_quantize_multi_workspace_bytes())


def zq_quantize_fp8_noalloc(x, x_dtype, n_vec, d, hadamard, x_fp8, descale, stream) -> int:
    """zq_quantize_fp8 without a workspace: for callers that cannot supply
    device scratch (their device memory belongs to another allocator, or
    they must not call cudaMalloc in a latency-critical loop).  Uses one
    fixed scratch array inside the library; calls that overlap on the GPU
    race.  The first call on a device sets up the array's address."""
    return _lib.zq_quantize_fp8_noalloc(x, x_dtype, n_vec, d, hadamard, x_fp8, descale, stream)


def zq_quantize_fp8_grouped(x, x_dtype, B, S, H, d, heads_per_scale, hadamard, x_fp8, descale,
                            workspace, stream) -> int:
    return _lib.zq_quantize_fp8_grouped(x, x_dtype, B, S, H, d, heads_per_scale, hadamard, x_fp8,
                                        descale, workspace, stream)


def zq_quantize_grouped_workspace_bytes(B, H, heads_per_scale) -> int:
    return int(_lib.zq_quantize_grouped_workspace_bytes(B, H, heads_per_scale))


def zq_quantize_noalloc_scratch_bytes() -> int:
    return int(_lib.zq_quantize_noalloc_scratch_bytes())


def zq_debug_exp2(x, y, n, degree, stream) -> int:
    return _lib.zq_debug_exp2(x, y, n, degree, stream)


def zq_quantize_workspace_bytes() -> int:
    return int(_lib.zq_quantize_workspace_bytes())


def zq_status_string(status: int) -> str:
    return _lib.zq_status_string(status).decode()


def zq_version() -> int:
    return int(_lib.zq_version())


# ------------------------------------------------------------- torch helpers
def _torch():
    import torch

    return torch


def _ptr(t):
    return None if t is None else t.data_ptr()


def _stream(stream):
    torch = _torch()
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _check(rc: int, where: str):
    if rc != ZQ_OK:
        raise ZQError(rc, where)


def _is_fp8(t) -> bool:
    torch = _torch()
    return t.dtype in (torch.float8_e4m3fn, torch.uint8)


def _check_buffer(name, t, shape, dtype):
    """A caller-supplied output or side buffer: contiguous, exact shape and dtype."""
    if tuple(t.shape) != tuple(shape):
        raise ValueError("%s must have shape %s, got %s" % (name, tuple(shape), tuple(t.shape)))
    if t.dtype != dtype:
        raise ValueError("%s must be %s, got %s" % (name, dtype, t.dtype))
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)


def _check_same_cuda_device(dev, named):
    """Every given tensor lives on CUDA device `dev` (no host pointers reach
    the library, and no tensor of another GPU)."""
    for name, t in named:
        if t is None:
            continue
        if not t.is_cuda:
            raise ValueError("%s must be a CUDA tensor" % name)
        if t.device != dev:
            raise ValueError("%s is on %s, expected %s" % (name, t.device, dev))


def quantize_fp8(x, hadamard: bool = False, out=None, descale=None, workspace=None, stream=None):
    """Per-tensor e4m3 quantisation of a CUDA tensor (fp32 or bf16, last dim d).

    Returns (codes as torch.float8_e4m3fn, descale fp32 tensor of shape (1,))."""
    torch = _torch()
    if not x.is_cuda or not x.is_contiguous():
        raise ValueError("x must be a contiguous CUDA tensor")
    if x.dtype == torch.float32:
        xd = ZQ_X_F32
    elif x.dtype == torch.bfloat16:
        xd = ZQ_X_BF16
    else:
        raise TypeError("quantize_fp8 takes float32 or bfloat16")
    if x.dim() == 0:
        raise ValueError("x needs a last (channel) dimension")
    d = x.shape[-1]
    if out is None:
        out = torch.empty(x.shape, dtype=torch.float8_e4m3fn, device=x.device)
    elif out.dtype not in (torch.float8_e4m3fn, torch.uint8):
        raise ValueError("out must be float8_e4m3fn or uint8")
    else:
        _check_buffer("out", out, x.shape, out.dtype)
    if descale is None:
        descale = torch.empty(1, dtype=torch.float32, device=x.device)
    else:
        _check_buffer("descale", descale, (1,), torch.float32)
    if workspace is None:
        workspace = torch.empty(zq_quantize_workspace_bytes(), dtype=torch.uint8, device=x.device)
    elif workspace.numel() * workspace.element_size() < zq_quantize_workspace_bytes() or not workspace.is_contiguous():
        raise ValueError("workspace must be contiguous and hold zq_quantize_workspace_bytes() bytes")
    _check_same_cuda_device(x.device, [("out", out), ("descale", descale), ("workspace", workspace)])
    _check(zq_quantize_fp8(x.data_ptr(), xd, x.numel() // d, d, int(bool(hadamard)), out.data_ptr(),
                           descale.data_ptr(), workspace.data_ptr(), _stream(stream)), "zq_quantize_fp8")
    return out, descale


def quantize_fp8_multi(xs, hadamard=None, outs=None, descales=None, workspace=None, stream=None):
    """Per-tensor e4m3 quantisation of up to four CUDA tensors in one call
    (three stream operations in all), e.g. q, k, v with the rotation on q and k.

    hadamard: one flag per tensor (default all False).  Returns (codes list,
    descales list), each as quantize_fp8 returns them for the tensor alone."""
    torch = _torch()
    xs = list(xs)
    n = len(xs)
    if not 1 <= n <= 4:
        raise ValueError("quantize_fp8_multi takes 1 to 4 tensors")
    hadamard = [False] * n if hadamard is None else [bool(h) for h in hadamard]
    if len(hadamard) != n:
        raise ValueError("one hadamard flag per tensor")
    outs = [None] * n if outs is None else list(outs)
    descales = [None] * n if descales is None else list(descales)
    arr = (zq_quant_tensor * n)()
    for i, x in enumerate(xs):
        if not x.is_cuda or not x.is_contiguous() or x.dim() == 0:
            raise ValueError("every tensor must be a contiguous CUDA tensor")
        if x.dtype == torch.float32:
            xd = ZQ_X_F32
        elif x.dtype == torch.bfloat16:
            xd = ZQ_X_BF16
        else:
            raise TypeError("quantize_fp8_multi takes float32 or bfloat16")
        if x.device != xs[0].device:
            raise ValueError("all tensors must be on one device")
        if outs[i] is None:
            outs[i] = torch.empty(x.shape, dtype=torch.float8_e4m3fn, device=x.device)
        elif outs[i].dtype not in (torch.float8_e4m3fn, torch.uint8):
            raise ValueError("out must be float8_e4m3fn or uint8")
        else:
            _check_buffer("out", outs[i], x.shape, outs[i].dtype)
        if descales[i] is None:
            descales[i] = torch.empty(1, dtype=torch.float32, device=x.device)
        else:
            _check_buffer("descale", descales[i], (1,), torch.float32)
        _check_same_cuda_device(x.device, [("out", outs[i]), ("descale", descales[i])])
        d = x.shape[-1]
        arr[i].x, arr[i].x_dtype, arr[i].n_vec, arr[i].d = x.data_ptr(), xd, x.numel() // d, d
        arr[i].hadamard, arr[i].x_fp8, arr[i].descale = int(hadamard[i]), outs[i].data_ptr(), descales[i].data_ptr()
    nbytes = zq_quantize_multi_workspace_bytes()
    if workspace is None:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=xs[0].device)
    elif workspace.numel() * workspace.element_size() < nbytes or not workspace.is_contiguous():
        raise ValueError("workspace must be contiguous and hold zq_quantize_multi_workspace_bytes() bytes")
    _check_same_cuda_device(xs[0].device, [("workspace", workspace)])
    _check(zq_quantize_fp8_multi(arr, n, workspace.data_ptr(), _stream(stream)), "zq_quantize_fp8_multi")
    return outs, descales


def quantize_fp8_grouped(x, heads_per_scale=1, hadamard: bool = False, out=None, descale=None,
                         workspace=None, stream=None):
    """e4m3 quantisation of a (B, S, H, d) CUDA tensor with one scale per
    (batch, group of heads_per_scale heads).

    Queries take heads_per_scale = Hq / Hkv, keys and values 1: the result
    feeds attn_fwd with per-(batch, kv head) descales.  Returns (codes as
    torch.float8_e4m3fn, descale fp32 tensor of shape (B, H / heads_per_scale))."""
    torch = _torch()
    if not x.is_cuda or not x.is_contiguous() or x.dim() != 4:
        raise ValueError("x must be a contiguous (B, S, H, d) CUDA tensor")
    if x.dtype == torch.float32:
        xd = ZQ_X_F32
    elif x.dtype == torch.bfloat16:
        xd = ZQ_X_BF16
    else:
        raise TypeError("quantize_fp8_grouped takes float32 or bfloat16")
    B, S, H, d = x.shape
    g = int(heads_per_scale)
    if g <= 0 or H % g != 0:
        raise ValueError("heads_per_scale must divide the head count")
    if out is None:
        out = torch.empty(x.shape, dtype=torch.float8_e4m3fn, device=x.device)
    elif out.dtype not in (torch.float8_e4m3fn, torch.uint8):
        raise ValueError("out must be float8_e4m3fn or uint8")
    else:
        _check_buffer("out", out, x.shape, out.dtype)
    if descale is None:
        descale = torch.empty((B, H // g), dtype=torch.float32, device=x.device)
    elif descale.numel() != B * (H // g) or descale.dtype != torch.float32 or not descale.is_contiguous():
        raise ValueError("descale must be a contiguous float32 tensor of B * H / heads_per_scale values")
    nbytes = zq_quantize_grouped_workspace_bytes(B, H, g)
    if workspace is None:
        workspace = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=x.device)
    elif workspace.numel() * workspace.element_size() < nbytes or not workspace.is_contiguous():
        raise ValueError("workspace must be contiguous and hold zq_quantize_grouped_workspace_bytes() bytes")
    _check_same_cuda_device(x.device, [("out", out), ("descale", descale), ("workspace", workspace)])
    _check(zq_quantize_fp8_grouped(x.data_ptr(), xd, B, S, H, d, g, int(bool(hadamard)), out.data_ptr(),
                                   descale.data_ptr(), workspace.data_ptr(), _stream(stream)),
           "zq_quantize_fp8_grouped")
    return out, descale


def _descale_layout(B, Hkv, *descales) -> int:
    """Per-tensor when every given descale holds one value, per-(batch, kv
    head) when they hold B * Hkv values."""
    sizes = {t.numel() for t in descales if t is not None}
    if not sizes or sizes == {1}:
        return ZQ_DESCALE_PER_TENSOR
    if sizes == {B * Hkv}:
        return ZQ_DESCALE_PER_KV_HEAD
    raise ValueError("descales must all hold 1 or all hold B * Hkv values, got %s" % sorted(sizes))


def attn_fwd(q, k, v, out=None, lse=None, softmax_scale=None, causal=True, q_descale=None,
             k_descale=None, v_descale=None, softmax_mode=ZQ_SOFTMAX_LEANP, block_scale=True,
             headroom_T=8, status=None, return_lse=True, stream=None, debug=None, debug_at=(0, 0),
             debug_flags=0):
    """Causal prefill attention on CUDA tensors.

    q (B,Sq,Hq,d_qk), k (B,Sk,Hkv,d_qk), v (B,Sk,Hkv,d_v): bfloat16, or FP8
    e4m3 (float8_e4m3fn / uint8) with fp32 descale tensors: one value each
    (per tensor) or B * Hkv values each (per batch and kv head, as
    quantize_fp8_grouped returns them).
    Returns (out bf16 (B,Sq,Hq,d_v), lse fp32 (B,Hq,Sq) or None)."""
    torch = _torch()
    for name, t in (("q", q), ("k", k), ("v", v)):
        if t.dim() != 4:
            raise ValueError("%s must be 4-D (batch, seq, heads, dim), got %d-D" % (name, t.dim()))
        if not t.is_contiguous():
            raise ValueError("%s must be contiguous" % name)
    if _is_fp8(q) and _is_fp8(k) and _is_fp8(v):
        dtype = ZQ_DTYPE_FP8_E4M3
    elif q.dtype == k.dtype == v.dtype == torch.bfloat16:
        dtype = ZQ_DTYPE_BF16
    else:
        raise TypeError("q, k, v must all be bfloat16 or all FP8 e4m3")
    B, Sq, Hq, dqk = q.shape
    Sk, Hkv, dv = k.shape[1], k.shape[2], v.shape[3]
    # the kernel addresses k and v with q's batch and k's sequence, heads and
    # width: every pair must agree, or it would read past an allocation
    if k.shape[0] != B or v.shape[0] != B:
        raise ValueError("q, k, v must have the same batch size, got %d, %d, %d" % (B, k.shape[0], v.shape[0]))
    if k.shape[3] != dqk:
        raise ValueError("k must have q's head dim %d, got %d" % (dqk, k.shape[3]))
    if v.shape[1] != Sk or v.shape[2] != Hkv:
        raise ValueError("v must have k's sequence length and head count (%d, %d), got (%d, %d)"
                         % (Sk, Hkv, v.shape[1], v.shape[2]))
    if out is None:
        out = torch.empty((B, Sq, Hq, dv), dtype=torch.bfloat16, device=q.device)
    else:
        _check_buffer("out", out, (B, Sq, Hq, dv), torch.bfloat16)
    if lse is None and return_lse:
        lse = torch.empty((B, Hq, Sq), dtype=torch.float32, device=q.device)
    elif lse is not None:
        _check_buffer("lse", lse, (B, Hq, Sq), torch.float32)
    descales = (("q_descale", q_descale), ("k_descale", k_descale), ("v_descale", v_descale))
    if dtype == ZQ_DTYPE_FP8_E4M3:
        for name, t in descales:
            if t is not None and (t.dtype != torch.float32 or not t.is_contiguous()):
                raise ValueError("%s must be a contiguous float32 tensor" % name)
    if status is not None and (status.dtype != torch.int32 or status.numel() < 1):
        raise ValueError("status must be an int32 tensor with at least one element")
    if debug is not None and debug.numel() * debug.element_size() < ZQ_DEBUG_BYTES:
        raise ValueError("debug must hold ZQ_DEBUG_BYTES bytes")
    _check_same_cuda_device(q.device, [("q", q), ("k", k), ("v", v), ("out", out), ("lse", lse), ("status", status),
                                       ("debug", debug)] + (list(descales) if dtype == ZQ_DTYPE_FP8_E4M3 else []))
    a = zq_attn_args()
    a.q, a.k, a.v, a.out, a.lse = q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), _ptr(lse)
    a.B, a.Sq, a.Sk, a.Hq, a.Hkv, a.d_qk, a.d_v = B, Sq, Sk, Hq, Hkv, dqk, dv
    a.softmax_scale = float(softmax_scale) if softmax_scale else 0.0
    a.causal = int(bool(causal))
    a.dtype = dtype
    a.q_descale, a.k_descale, a.v_descale = _ptr(q_descale), _ptr(k_descale), _ptr(v_descale)
    a.softmax_mode = int(softmax_mode)
    a.block_scale = int(bool(block_scale))
    a.headroom_T = int(headroom_T)
    a.status = _ptr(status)
    a.descale_layout = _descale_layout(B, Hkv, q_descale, k_descale, v_descale) if dtype == ZQ_DTYPE_FP8_E4M3 else 0
    if debug is not None:
        _check(zq_attn_fwd_debug(a, debug.data_ptr(), int(debug_at[0]), int(debug_at[1]), int(debug_flags),
                                 _stream(stream)), "zq_attn_fwd_debug")
    else:
        _check(zq_attn_fwd_ex(a, _stream(stream)), "zq_attn_fwd_ex")
    return out, lse


def flash_attn_func(q, k, v, softmax_scale=None, causal=True, return_attn_probs=False, **fp8_kwargs):
    """flash_attn_func-style entry: (B,S,H,d) tensors in, (B,S,H,d_v) bf16 out.

    With return_attn_probs=True returns (out, lse, None) like flash-attn."""
    out, lse = attn_fwd(q, k, v, softmax_scale=softmax_scale, causal=causal,
                        return_lse=return_attn_probs, **fp8_kwargs)
    return (out, lse, None) if return_attn_probs else out


def causal_flops(B, Sq, Hq, dqk, dv, Sk=None) -> float:
    """2*B*Hq*S^2*(d_qk+d_v)/2 for the causal Sq == Sk case."""
    S = Sq if Sk is None else math.sqrt(Sq * Sk)
    return 2.0 * B * Hq * S * S * (dqk + dv) / 2.0
