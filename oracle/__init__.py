"""CPU oracle for the SVDQuant W4A4 and AWQ W4A16 linear layers.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg may import this package; the product path never
does. The arithmetic lives in ``svdq_oracle.c`` (plain C, float64
accumulation, one rounding per fp32 step); this module compiles it with gcc
on first use and wraps it with ctypes/numpy.

Parity pins (what fixes this oracle other than itself) are in
``tests/test_oracle_pins.py``.
"""

from __future__ import annotations

import ctypes as C
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "svdq_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_CFLAGS = ["-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
           "-fno-fast-math", "-Wall", "-Wno-unknown-pragmas"]
_lock = threading.Lock()
_lib = None

NVFP4, INT4 = 0, 1


def build(force: bool = False) -> str:
    """Compile the oracle's shared library (in-tree). Returns its path."""
    with _lock:
        stale = (not os.path.exists(_LIB_PATH)
                 or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC))
        if force or stale:
            tmp = _LIB_PATH + f".{os.getpid()}.tmp"
            subprocess.check_call(["gcc", *_CFLAGS, "-o", tmp, _SRC, "-lm"])
            os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def lib():
    global _lib
    if _lib is None:
        build()
        L = C.CDLL(_LIB_PATH)
        P = C.c_void_p
        i32, i64, u64, f32 = C.c_int, C.c_int64, C.c_uint64, C.c_float
        sig = {
            "orc_set_threads": (None, [i32]),
            "orc_get_threads": (i32, []),
            "orc_bf16_rn": (C.c_uint16, [f32]),
            "orc_bf16_rn_f64": (C.c_uint16, [C.c_double]),
            "orc_bf16_to_f32": (f32, [C.c_uint16]),
            "orc_e4m3_rn_sat": (C.c_uint8, [f32]),
            "orc_e4m3_to_f32": (f32, [C.c_uint8]),
            "orc_e2m1_rn_sat": (C.c_uint8, [f32]),
            "orc_e2m1_to_f32": (f32, [C.c_uint8]),
            "orc_check_cvt_range": (None, [u64, u64, P, P, P, P, P]),
            "orc_nvfp4_group": (None, [P, f32, P, P]),
            "orc_int4_group": (None, [P, P, P]),
            "orc_svdq_pack_weight": (i32, [i32, i32, i32, i32, P, P, P, P, P, P, P, P, P]),
            "orc_svdq_quantize_act": (i32, [i32, i32, i32, i32, P, P, f32, P, P, P, P]),
            "orc_svdq_linear": (i32, [i32, i32, i32, i32, i32, P, P, f32, P, P, P, f32, P, P,
                                      i32, P, P]),
            "orc_int4_group_sums": (i32, [i32, i32, i32, P, P, P]),
            "orc_awq_pack_weight": (i32, [i32, i32, P, P, P, P]),
            "orc_awq_linear": (i32, [i32, i32, i32, P, P, P, P, P, P]),
            "orc_qkv_norm_rope": (i32, [i32, i32, i32, P, P, P, C.c_double, P, P, P]),
            "orc_gelu_bf16": (None, [P, i64, P]),
            "orc_bf16_rn_f64_array": (None, [P, i64, P]),
            "orc_e4m3_rn_array": (None, [P, i64, P]),
            "orc_e2m1_rn_array": (None, [P, i64, P]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(C.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def set_threads(n: int) -> None:
    lib().orc_set_threads(int(n))


def threads() -> int:
    return int(lib().orc_get_threads())


# ---------------------------------------------------------------- formats
def bf16_rn(v) -> np.ndarray:
    """Round float64 (or float32) values to bfloat16 bit patterns (uint16)."""
    v = _c(v, np.float64)
    out = np.empty(v.shape, np.uint16)
    lib().orc_bf16_rn_f64_array(_p(v), v.size, _p(out))
    return out


def bf16_to_f32(b) -> np.ndarray:
    return (np.asarray(b, np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def e4m3_rn(v) -> np.ndarray:
    v = _c(v, np.float32)
    out = np.empty(v.shape, np.uint8)
    lib().orc_e4m3_rn_array(_p(v), v.size, _p(out))
    return out


def e2m1_rn(v) -> np.ndarray:
    v = _c(v, np.float32)
    out = np.empty(v.shape, np.uint8)
    lib().orc_e2m1_rn_array(_p(v), v.size, _p(out))
    return out


def e4m3_to_f32(c) -> np.ndarray:
    L = lib()
    table = np.array([L.orc_e4m3_to_f32(i) for i in range(256)], np.float32)
    return table[np.asarray(c, np.uint8)]


def e2m1_to_f32(c) -> np.ndarray:
    L = lib()
    table = np.array([L.orc_e2m1_to_f32(i) for i in range(16)], np.float32)
    return table[np.asarray(c, np.uint8) & 0xF]


def check_cvt_range(start: int, count: int, e2m1=None, e4m3=None, bf16=None):
    """Compare device conversions of fp32 bit patterns [start, start+count)."""
    bad = np.zeros(3, np.int64)
    first = np.zeros(3, np.uint32)
    lib().orc_check_cvt_range(start, count, _p(e2m1), _p(e4m3), _p(bf16), _p(bad), _p(first))
    return bad, first


def nvfp4_group(v, t: float):
    v = _c(v, np.float32)
    assert v.size == 16
    codes = np.empty(16, np.uint8)
    sf = np.empty(1, np.uint8)
    lib().orc_nvfp4_group(_p(v), float(t), _p(codes), _p(sf))
    return codes, int(sf[0])


def int4_group(v):
    v = _c(v, np.float32)
    assert v.size == 64
    q = np.empty(64, np.int8)
    s = np.empty(1, np.uint16)
    lib().orc_int4_group(_p(v), _p(q), _p(s))
    return q, int(s[0])


def unpack_nibbles(codes: np.ndarray) -> np.ndarray:
    """[rows, K/2] packed bytes -> [rows, K] nibbles (element 2j = low nibble)."""
    codes = np.asarray(codes, np.uint8)
    out = np.empty(codes.shape[:-1] + (codes.shape[-1] * 2,), np.uint8)
    out[..., 0::2] = codes & 0xF
    out[..., 1::2] = codes >> 4
    return out


# ---------------------------------------------------------------- svdq_w4a4
def _prec(p):
    return {"nvfp4": NVFP4, "int4": INT4, NVFP4: NVFP4, INT4: INT4}[p]


def pack_weight(prec, W, lam, L1, L2, want_R=False):
    prec = _prec(prec)
    W = _c(W, np.float32)
    K, N = W.shape
    L1 = _c(L1, np.uint16).reshape(K, -1)
    r = L1.shape[1]
    L2 = _c(L2, np.uint16).reshape(r, N)
    lam = _c(lam, np.float32)
    codes = np.zeros((N, K // 2), np.uint8)
    scales = np.zeros((N, K // 16), np.uint8) if prec == NVFP4 else np.zeros((N, K // 64), np.uint16)
    s_tw = np.zeros(1, np.float32)
    inv_lam = np.zeros(K, np.float32)
    R = np.zeros((K, N), np.float32) if want_R else None
    rc = lib().orc_svdq_pack_weight(prec, K, N, r, _p(W), _p(lam), _p(L1), _p(L2), _p(codes),
                                    _p(scales), _p(s_tw), _p(inv_lam), _p(R))
    if rc:
        raise ValueError(f"orc_svdq_pack_weight: {rc}")
    out = dict(codes=codes, scales=scales, s_tw=float(s_tw[0]), inv_lam=inv_lam)
    if want_R:
        out["R"] = R
    return out


def quantize_act(prec, x, inv_lam, s_tx, L1):
    prec = _prec(prec)
    x = _c(x, np.uint16)
    M, K = x.shape
    L1 = _c(L1, np.uint16).reshape(K, -1)
    r = L1.shape[1]
    codes = np.zeros((M, K // 2), np.uint8)
    scales = np.zeros((M, K // 16), np.uint8) if prec == NVFP4 else np.zeros((M, K // 64), np.uint16)
    P = np.zeros((M, r), np.uint16)
    rc = lib().orc_svdq_quantize_act(prec, M, K, r, _p(x), _p(_c(inv_lam, np.float32)),
                                     float(s_tx), _p(L1), _p(codes), _p(scales), _p(P))
    if rc:
        raise ValueError(f"orc_svdq_quantize_act: {rc}")
    return dict(codes=codes, scales=scales, P=P)


def linear(prec, xq, wq, s_tx, L2, bias=None, rows=None):
    """Unrounded layer output (float64) for all rows, or for ``rows``."""
    prec = _prec(prec)
    M, K2 = xq["codes"].shape
    K = 2 * K2
    N = wq["codes"].shape[0]
    P = _c(xq["P"], np.uint16)
    r = P.shape[1]
    L2 = _c(L2, np.uint16).reshape(r, N)
    sel = None if rows is None else _c(rows, np.int32)
    n_rows = M if sel is None else sel.size
    y = np.zeros((n_rows, N), np.float64)
    b = None if bias is None else _c(bias, np.uint16)
    rc = lib().orc_svdq_linear(prec, M, K, N, r, _p(_c(xq["codes"], np.uint8)),
                               _p(np.ascontiguousarray(xq["scales"])), float(s_tx), _p(P),
                               _p(_c(wq["codes"], np.uint8)), _p(np.ascontiguousarray(wq["scales"])),
                               float(wq.get("s_tw", 1.0)), _p(L2), _p(b), n_rows, _p(sel), _p(y))
    if rc:
        raise ValueError(f"orc_svdq_linear: {rc}")
    return y


def int4_group_sums(x_codes, w_codes):
    x_codes = _c(x_codes, np.uint8)
    w_codes = _c(w_codes, np.uint8)
    M, K2 = x_codes.shape
    N = w_codes.shape[0]
    K = 2 * K2
    out = np.zeros((M, N, K // 64), np.int32)
    rc = lib().orc_int4_group_sums(M, K, N, _p(x_codes), _p(w_codes), _p(out))
    if rc:
        raise ValueError(f"orc_int4_group_sums: {rc}")
    return out


def qkv_norm_rope(y, heads: int, head_dim: int, wq, wk, eps: float, cos, sin):
    """Fused QKV epilogue on the unrounded layer output y [M, 3*heads*head_dim]
    (Q, K, V in that order): per-head RMSNorm of Q and K with bf16 weights wq,
    wk [head_dim], then the rotary embedding of adjacent pairs with cos, sin
    [M, head_dim/2]; V passes through. Returns float64, unrounded."""
    y = _c(y, np.float64)
    M = y.shape[0]
    assert y.shape[1] == 3 * heads * head_dim
    cos = _c(cos, np.float32).reshape(M, head_dim // 2)
    sin = _c(sin, np.float32).reshape(M, head_dim // 2)
    out = np.zeros_like(y)
    rc = lib().orc_qkv_norm_rope(M, heads, head_dim, _p(y), _p(_c(wq, np.uint16)), _p(_c(wk, np.uint16)),
                                 float(eps), _p(cos), _p(sin), _p(out))
    if rc:
        raise ValueError(f"orc_qkv_norm_rope: {rc}")
    return out


def gelu_bf16(y) -> np.ndarray:
    """bf16 bits of GELU (erf form) of the unrounded values y, one rounding."""
    y = _c(y, np.float64)
    h = np.zeros(y.shape, np.uint16)
    lib().orc_gelu_bf16(_p(y), y.size, _p(h))
    return h


def mlp_gelu_down_act(prec, y_up, inv_lam_down, s_tx, L1_down):
    """Fused GELU-MLP epilogue: the down-projection's activation-pass outputs
    (codes, scales, P) from the up-projection's unrounded output."""
    return quantize_act(prec, gelu_bf16(y_up), inv_lam_down, s_tx, L1_down)


# ---------------------------------------------------------------- awq_w4a16
def awq_pack_weight(W):
    W = _c(W, np.float32)
    K, N = W.shape
    q = np.zeros((N, K // 2), np.uint8)
    s = np.zeros((N, K // 64), np.uint16)
    z = np.zeros((N, K // 64), np.uint16)
    rc = lib().orc_awq_pack_weight(K, N, _p(W), _p(q), _p(s), _p(z))
    if rc:
        raise ValueError(f"orc_awq_pack_weight: {rc}")
    return dict(q=q, s=s, z=z)


def awq_linear(x, pk, bias=None):
    x = _c(x, np.uint16)
    M, K = x.shape
    N = pk["q"].shape[0]
    y = np.zeros((M, N), np.float64)
    b = None if bias is None else _c(bias, np.uint16)
    rc = lib().orc_awq_linear(M, K, N, _p(x), _p(_c(pk["q"], np.uint8)), _p(_c(pk["s"], np.uint16)),
                              _p(_c(pk["z"], np.uint16)), _p(b), _p(y))
    if rc:
        raise ValueError(f"orc_awq_linear: {rc}")
    return y
