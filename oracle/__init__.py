"""CPU oracle for causal prefill attention (FP8 e4m3 / BF16) -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference
legs of ``bench.py`` may import this package.  It shares no code with the CUDA
path (``bf16_causal_prefill_02_b200``) and never imports it.

Sources (web pages re-reporting the ZYFA announcement):
  [P1] "Zyphra ZYFA : FlashAttention en FP8 pour l'AMD MI355X, jusqu'a 1,76
       fois plus rapide" (lefilia.fr), paragraphs 1-3.
  [P2] "Zyphra rilascia ZYFA, kernel di attenzione FP8 ottimizzati per le GPU
       AMD" (aicronaca.it), section "Perche l'FP8 non basta da solo".
  [P3] "Zyphra ZYFA ... FP8 FlashAttention for AMD MI355X" (ai4bro.com),
       sections TL;DR and "How ZYFA works".

Functions (all fp64 unless stated):
  attn_ref          R1  exact softmax(QK^T*scale + causal mask) V
  attn_fp8_emul     R2  FP8 P path: per-(row, 64-key block) power-of-2 scale,
                        exact-exp2 or Lean P rounding, rounded-row-sum division
  quantize_fp8      R3  per-tensor amax quantiser, optional 128-point FWHT
  quantize_fp8_grouped  R3 applied per (batch, group of heads): one scale
                        per (batch, kv head), the flash_attn_func FP8 layout
  dequant_grouped       codes times the per-(batch, head group) descale
  e4m3_decode/encode    OCP e4m3fn codec
  leanp_code            the Lean P byte of a log2-domain value (R2's rounding)
  brute_attn            dense numpy softmax for tiny inputs (a cross-check)

Every function here is pinned by ``tests/test_oracle.py`` against something
other than itself (library special cases, closed forms, invariants).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "zq_oracle.c")
_LIB_PATH = os.path.join(_HERE, "_zq_oracle.so")
_lib = None

MODE_EXACT, MODE_LEANP, MODE_NOROUND = 0, 1, 2


def build(force: bool = False) -> str:
    """Compile the C oracle into ``oracle/_zq_oracle.so`` (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + ".tmp%d" % os.getpid()
        subprocess.check_call(
            ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-Wall", "-o", tmp, _SRC, "-lm"]
        )
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _L():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        P = ctypes.c_void_p
        i32, i64, f64 = ctypes.c_int, ctypes.c_int64, ctypes.c_double
        lib.zo_num_threads.restype = i32
        lib.zo_set_num_threads.argtypes = [i32]
        lib.zo_set_num_threads.restype = i32
        lib.zo_leanp_code.argtypes = [f64]
        lib.zo_leanp_code.restype = i32
        lib.zo_e4m3_decode.argtypes = [ctypes.c_uint8]
        lib.zo_e4m3_decode.restype = f64
        lib.zo_e4m3_encode_rne_sat.argtypes = [f64]
        lib.zo_e4m3_encode_rne_sat.restype = ctypes.c_uint8
        lib.zo_fwht128_f32.argtypes = [P]
        lib.zo_fwht64_f32.argtypes = [P]
        lib.zo_quantize_fp8.argtypes = [P, i32, i64, i32, i32, P, P]
        lib.zo_quantize_fp8.restype = i32
        lib.zo_attn_ref.argtypes = [P, P, P, i32, i32, i32, i32, i32, i32, i32, f64, i32, P, i64, P, P]
        lib.zo_attn_ref.restype = i32
        lib.zo_attn_fp8_emul.argtypes = [P, P, P, i32, i32, i32, i32, i32, i32, i32, f64, i32,
                                         i32, i32, i32, P, i64, P, P, P]
        lib.zo_attn_fp8_emul.restype = i32
        lib.zo_dequant_e4m3.argtypes = [P, i64, f64, P]
        _lib = lib
    return _lib


def _ptr(a):
    return a.ctypes.data_as(ctypes.c_void_p) if a is not None else None


def num_threads() -> int:
    return int(_L().zo_num_threads())


def set_num_threads(n: int) -> int:
    """Thread count of the oracle's parallel loops (timing only; results do
    not depend on it).  Returns the count in effect."""
    return int(_L().zo_set_num_threads(int(n)))


def leanp_code(z) -> np.ndarray:
    """Lean P byte of each log2-domain value z = y - e: 8z rounded half to
    even, plus 56, clamped to [0, 126] (the function R2 uses)."""
    z = np.asarray(z, dtype=np.float64)
    f = _L().zo_leanp_code
    return np.array([f(float(t)) for t in z.ravel()], dtype=np.int64).reshape(z.shape)


# ----------------------------------------------------------------- codec
def e4m3_decode(codes) -> np.ndarray:
    """Exact fp64 value of each e4m3fn byte (NaN for 0x7F / 0xFF)."""
    c = np.ascontiguousarray(codes, dtype=np.uint8)
    out = np.empty(c.shape, dtype=np.float64)
    _L().zo_dequant_e4m3(_ptr(c), c.size, 1.0, _ptr(out))
    return out


def e4m3_encode(x) -> np.ndarray:
    """Round each value to e4m3fn, ties to even, saturating to +-448."""
    x = np.asarray(x, dtype=np.float64)
    f = _L().zo_e4m3_encode_rne_sat
    return np.array([f(float(t)) for t in x.ravel()], dtype=np.uint8).reshape(x.shape)


def dequant_e4m3(codes: np.ndarray, descale: float) -> np.ndarray:
    """codes * descale, exactly, in fp64."""
    c = np.ascontiguousarray(codes, dtype=np.uint8)
    out = np.empty(c.shape, dtype=np.float64)
    _L().zo_dequant_e4m3(_ptr(c), c.size, float(descale), _ptr(out))
    return out


# ------------------------------------------------------------- quantiser
def fwht128(x: np.ndarray) -> np.ndarray:
    """Unnormalised 128-point FWHT of each 128-slice, fp32 butterflies."""
    x = np.array(x, dtype=np.float32, copy=True, order="C")
    assert x.shape[-1] % 128 == 0
    flat = x.reshape(-1, 128)
    lib = _L()
    for r in range(flat.shape[0]):
        row = np.ascontiguousarray(flat[r])
        lib.zo_fwht128_f32(_ptr(row))
        flat[r] = row
    return flat.reshape(x.shape)


def fwht64(x: np.ndarray) -> np.ndarray:
    """Unnormalised 64-point FWHT of each 64-slice, fp32 butterflies."""
    x = np.array(x, dtype=np.float32, copy=True, order="C")
    assert x.shape[-1] % 64 == 0
    flat = x.reshape(-1, 64)
    lib = _L()
    for r in range(flat.shape[0]):
        row = np.ascontiguousarray(flat[r])
        lib.zo_fwht64_f32(_ptr(row))
        flat[r] = row
    return flat.reshape(x.shape)


def quantize_fp8(x: np.ndarray, hadamard: bool = False):
    """R3.  x: float32 array, or uint16 array holding bf16 bits, last dim d.

    Returns (codes uint8 of x.shape, descale float32)."""
    x = np.ascontiguousarray(x)
    if x.dtype == np.float32:
        xd = 0
    elif x.dtype == np.uint16:
        xd = 1
    else:
        raise TypeError("quantize_fp8 takes float32 or bf16 bits (uint16)")
    d = x.shape[-1]
    n_vec = x.size // d
    out = np.empty(x.shape, dtype=np.uint8)
    ds = np.zeros(1, dtype=np.float32)
    rc = _L().zo_quantize_fp8(_ptr(x), xd, n_vec, d, int(bool(hadamard)), _ptr(out), _ptr(ds))
    if rc != 0:
        raise ValueError("zo_quantize_fp8 rejected the arguments")
    return out, np.float32(ds[0])


def quantize_fp8_grouped(x: np.ndarray, heads_per_scale: int = 1, hadamard: bool = False):
    """R3 with one scale per (batch, group of heads).

    x: (B, S, H, d) float32, or uint16 holding bf16 bits.  The heads
    [gi*heads_per_scale, (gi+1)*heads_per_scale) of batch b form slot
    (b, gi); each slot, x[b, :, heads of gi, :], is quantised on its own
    exactly as quantize_fp8 quantises a whole tensor (own amax, own descale).
    With heads_per_scale = Hq / Hkv for queries and 1 for keys and values
    this gives the (batch, kv head) descales of flash_attn_func's FP8
    interface, which the pages name as the interface the kernel replaces
    ([P2] "Che cosa ha annunciato Zyphra").

    Returns (codes uint8 (B, S, H, d), descale float32 (B, H/heads_per_scale))."""
    x = np.ascontiguousarray(x)
    if x.ndim != 4:
        raise ValueError("quantize_fp8_grouped takes x of shape (B, S, H, d)")
    B, S, H, d = x.shape
    g = int(heads_per_scale)
    if g <= 0 or H % g != 0:
        raise ValueError("heads_per_scale must divide H")
    codes = np.zeros(x.shape, dtype=np.uint8)
    ds = np.zeros((B, H // g), dtype=np.float32)
    for b in range(B):
        for gi in range(H // g):
            sl = np.ascontiguousarray(x[b, :, gi * g:(gi + 1) * g, :])
            c, dsc = quantize_fp8(sl, hadamard=hadamard)
            codes[b, :, gi * g:(gi + 1) * g, :] = c
            ds[b, gi] = dsc
    return codes, ds


def dequant_grouped(codes: np.ndarray, descale: np.ndarray) -> np.ndarray:
    """codes (B, S, H, d) times descale (B, G) of head group h // (H / G),
    exactly, in fp64."""
    B, S, H, d = codes.shape
    G = descale.shape[1]
    val = e4m3_decode(codes)
    per_head = np.repeat(np.asarray(descale, dtype=np.float64), H // G, axis=1)  # (B, H)
    return val * per_head[:, None, :, None]


# ------------------------------------------------------------- attention
def _shapes(q, k, v):
    B, Sq, Hq, dqk = q.shape
    B2, Sk, Hkv, dqk2 = k.shape
    assert B == B2 and dqk == dqk2 and v.shape[:3] == (B, Sk, Hkv)
    return B, Sq, Sk, Hq, Hkv, dqk, v.shape[3]


def _rows_arg(rows):
    if rows is None:
        return None, 0
    r = np.ascontiguousarray(rows, dtype=np.int64)
    return r, r.size


def attn_ref(q, k, v, scale=None, causal=True, rows=None):
    """R1, fp64.  q (B,Sq,Hq,dqk), k (B,Sk,Hkv,dqk), v (B,Sk,Hkv,dv).

    rows: optional flat row ids (b*Hq + h)*Sq + i.  Returns (o, lse) with
    o (B,Sq,Hq,dv) and lse (B,Hq,Sq) when rows is None, else o (n,dv), lse (n)."""
    q, k, v = (np.ascontiguousarray(t, dtype=np.float64) for t in (q, k, v))
    B, Sq, Sk, Hq, Hkv, dqk, dv = _shapes(q, k, v)
    if scale is None:
        scale = 1.0 / np.sqrt(dqk)
    r, n = _rows_arg(rows)
    nr = n if r is not None else B * Hq * Sq
    o = np.empty((nr, dv))
    lse = np.empty(nr)
    rc = _L().zo_attn_ref(_ptr(q), _ptr(k), _ptr(v), B, Sq, Sk, Hq, Hkv, dqk, dv, float(scale),
                          int(bool(causal)), _ptr(r), n, _ptr(o), _ptr(lse))
    if rc != 0:
        raise ValueError("zo_attn_ref rejected the arguments")
    if r is None:
        return o.reshape(B, Hq, Sq, dv).transpose(0, 2, 1, 3).copy(), lse.reshape(B, Hq, Sq)
    return o, lse


def attn_fp8_emul(q, k, v, scale=None, causal=True, mode=MODE_LEANP, block_scale=True, T=8,
                  rows=None, want_p=False):
    """R2 (see zq_oracle.c).  Same layout conventions as attn_ref.

    want_p: also return the rounded p~ of the first evaluated row (Sk values)."""
    q, k, v = (np.ascontiguousarray(t, dtype=np.float64) for t in (q, k, v))
    B, Sq, Sk, Hq, Hkv, dqk, dv = _shapes(q, k, v)
    if scale is None:
        scale = 1.0 / np.sqrt(dqk)
    r, n = _rows_arg(rows)
    nr = n if r is not None else B * Hq * Sq
    o = np.empty((nr, dv))
    lse = np.empty(nr)
    pd = np.zeros(Sk) if want_p else None
    rc = _L().zo_attn_fp8_emul(_ptr(q), _ptr(k), _ptr(v), B, Sq, Sk, Hq, Hkv, dqk, dv,
                               float(scale), int(bool(causal)), int(mode), int(bool(block_scale)),
                               int(T), _ptr(r), n, _ptr(o), _ptr(lse), _ptr(pd))
    if rc != 0:
        raise ValueError("zo_attn_fp8_emul rejected the arguments")
    if r is None:
        o = o.reshape(B, Hq, Sq, dv).transpose(0, 2, 1, 3).copy()
        lse = lse.reshape(B, Hq, Sq)
    return (o, lse, pd) if want_p else (o, lse)


def brute_attn(q, k, v, scale=None, causal=True):
    """Dense softmax attention in numpy fp64 for tiny inputs (cross-check)."""
    q, k, v = (np.asarray(t, dtype=np.float64) for t in (q, k, v))
    B, Sq, Hq, dqk = q.shape
    Sk, Hkv = k.shape[1], k.shape[2]
    if scale is None:
        scale = 1.0 / np.sqrt(dqk)
    rep = Hq // Hkv
    kk = np.repeat(k, rep, axis=2)
    vv = np.repeat(v, rep, axis=2)
    s = np.einsum("bihd,bjhd->bhij", q, kk) * scale
    if causal:
        i = np.arange(Sq)[:, None]
        j = np.arange(Sk)[None, :]
        s = np.where(j <= i + (Sk - Sq), s, -np.inf)
    m = s.max(axis=-1, keepdims=True)
    with np.errstate(invalid="ignore"):
        p = np.exp(s - m)
        l = p.sum(axis=-1, keepdims=True)
        o = np.einsum("bhij,bjhd->bihd", p / l, vv)
        lse = (m + np.log(l))[..., 0]
    empty = ~np.isfinite(m[..., 0])  # rows with no visible key
    o = np.where(empty.transpose(0, 2, 1)[..., None], 0.0, o)
    lse = np.where(empty, -np.inf, lse)
    return o, lse


def rel_rmse(x, ref) -> float:
    """sqrt(sum (x-ref)^2 / sum ref^2) over all elements."""
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = float(np.sum(ref * ref))
    return float(np.sqrt(np.sum((x - ref) ** 2) / den)) if den > 0 else float(np.sqrt(np.sum(x * x)))
