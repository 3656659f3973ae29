"""B200 (sm_100a) SVDQuant W4A4 and AWQ W4A16 linear layers.

A thin ctypes binding over ``libsvdq.so`` (C ABI in ``include/svdq.h``).
Every function here only marshals arguments: torch tensors provide device
memory and the current CUDA stream, and every step of the layer runs in the
library's kernels. There is no CPU fallback: importing works without a GPU,
but calling an entry point without the built library raises.

The layer (blog "Introducing Nunchaku 4-bit inference in Diffusers", section
"Background: SVDQuant and Nunchaku"):
    y = Q4(x_hat) . Q4(R) + (x_hat L1) L2 + b,  x_hat = bf16(x / lambda),
    R = diag(lambda) W - L1 L2,
with svdq_w4a4 NVFP4 (group 16) or INT4 (group 64) and awq_w4a16 INT4
(group 64) (Diffusers "Nunchaku Lite" page, table "Supported quantization
types").
"""

from __future__ import annotations

import ctypes as C
import enum
import os
from dataclasses import dataclass
from typing import Optional

import torch

__all__ = [
    "NVFP4", "INT4", "Status", "SvdqError", "PackedWeight", "QuantAct", "AwqWeight",
    "library_path", "load", "scale_bytes", "pack_weight", "quantize_act", "w4a4_linear",
    "w4a4_linear_qkv", "qkv_norm_rope", "RopeTable", "pack_rope", "svdq_linear", "awq_pack_weight", "awq_w4a16_linear", "device_error", "set_wait_limit_ns",
    "probe_convert", "probe_wait_timeout", "probe_mma_peak", "debug_force_arch",
]

NVFP4, INT4 = 0, 1
_OUT = {"bf16": 0, "f32": 1, "i32_groups": 2, "bf16_gelu": 3}
_HERE = os.path.dirname(os.path.abspath(__file__))


class Status(enum.IntEnum):
    OK = 0
    INVALID_ARG = 1
    SHAPE = 2
    ALIGN = 3
    UNSUPPORTED_ARCH = 4
    CUDA = 5
    TIMEOUT = 6


class SvdqError(RuntimeError):
    def __init__(self, fn: str, status: int, msg: str):
        super().__init__(f"{fn}: {msg} (status {status})")
        self.status = Status(status)


_lib = None


def library_path() -> str:
    return os.path.join(_HERE, "libsvdq.so")


# name -> (restype, argtypes)
_P, _I, _F, _U64, _I64 = C.c_void_p, C.c_int, C.c_float, C.c_ulonglong, C.c_longlong
SIGNATURES = {
    "svdq_status_str": (C.c_char_p, [_I]),
    "svdq_scale_bytes": (C.c_size_t, [_I, _I, _I]),
    "svdq_lr_up_elems": (C.c_size_t, [_I, _I, _I]),
    "svdq_pack_weight": (_I, [_I, _I, _I, _I, _P, _P, _P, _P, _F, _P, _P, _P, _P, _P, _P]),
    "svdq_quantize_act": (_I, [_I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P, _P]),
    "svdq_w4a4_linear": (_I, [_I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _P]),
    "svdq_rope_packed_bytes": (C.c_size_t, [_I]),
    "svdq_rope_pack": (_I, [_I, _P, _P, _P, _P]),
    "svdq_w4a4_linear_qkv": (_I, [_I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _F, _P, _P, _P]),
    "svdq_qkv_norm_rope": (_I, [_I, _I, _P, _P, _F, _P, _P, _P, _P]),
    "awq_pack_weight": (_I, [_I, _I, _P, _P, _P, _P, _P]),
    "awq_w4a16_linear": (_I, [_I, _I, _I, _P, _P, _P, _P, _P, _P, _P]),
    "svdq_device_error": (_I, [_P]),
    "svdq_set_wait_limit_ns": (None, [_U64]),
    "svdq_probe_convert": (_I, [_P, _I64, _P, _P, _P, _P]),
    "svdq_probe_wait_timeout": (_I, [_U64, _P]),
    "svdq_debug_force_arch": (None, [_I, _I]),
    "svdq_probe_mma_peak": (_I, [_I, _I, _P]),
}


def load():
    """Load ``libsvdq.so`` (raises if it has not been built)."""
    global _lib
    if _lib is None:
        path = library_path()
        if not os.path.exists(path):
            raise RuntimeError(
                f"{path} is missing: build it with `python -m bit_w4a4_quantized_nvfp4_b200.build` "
                "(nvcc, sm_100a); this package has no fallback implementation")
        L = C.CDLL(path)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _check(fn: str, status: int) -> None:
    if status != 0:
        raise SvdqError(fn, status, load().svdq_status_str(status).decode())


def _ptr(t: Optional[torch.Tensor], dev: Optional[int] = None):
    """Device address of a contiguous CUDA tensor on the current device
    (``dev``, when the caller has already read it)."""
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    cur = torch.cuda.current_device() if dev is None else dev
    if t.get_device() != cur:
        raise ValueError(f"tensor on {t.device}, but the current device is cuda:{cur}")
    return t.data_ptr()


def _ptrs(*ts):
    """_ptr of several tensors, reading the current device once."""
    dev = None
    out = []
    for t in ts:
        if t is not None and dev is None:
            if not t.is_cuda:
                raise ValueError("expected a CUDA tensor")
            dev = torch.cuda.current_device()
        out.append(_ptr(t, dev))
    return out


def _need(cond: bool, what, *args) -> None:
    """Argument check of the binding: the C ABI receives bare pointers and
    cannot see sizes, so every shape and dtype is checked here, before any
    pointer reaches the library (a wrong size would otherwise become a read
    or write past an allocation). The message is formatted only on failure."""
    if not cond:
        raise ValueError(what.format(*args) if args else what)


def _is(t: Optional[torch.Tensor], dtype, shape, name: str) -> None:
    if t is None:
        raise ValueError(f"{name}: missing")
    if t.dtype is not dtype:
        raise ValueError(f"{name}: dtype {t.dtype}, expected {dtype}")
    if t.shape != shape:
        raise ValueError(f"{name}: shape {tuple(t.shape)}, expected {tuple(shape)}")


def _at_least(t: torch.Tensor, dtype, nbytes: int, name: str) -> None:
    if t.dtype is not dtype:
        raise ValueError(f"{name}: dtype {t.dtype}, expected {dtype}")
    if t.numel() * t.element_size() < nbytes:
        raise ValueError(f"{name}: {t.numel() * t.element_size()} bytes, need {nbytes}")


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _prec(p) -> int:
    if isinstance(p, str):
        return {"nvfp4": NVFP4, "int4": INT4}[p]
    return int(p)


def scale_bytes(prec, rows: int, K: int) -> int:
    return int(load().svdq_scale_bytes(_prec(prec), rows, K))


@dataclass
class PackedWeight:
    prec: int
    K: int
    N: int
    r: int
    codes: torch.Tensor          # uint8 [N, K/2]
    scales: torch.Tensor         # uint8 (tiled e4m3 bytes or bf16 pairs)
    tensor_scale: torch.Tensor   # float32 [2] = {s_tw, s_tx}
    inv_lambda: torch.Tensor     # float32 [K]
    lr_up: Optional[torch.Tensor]  # bf16 [N, 2r] (NVFP4) or [N, r] (INT4)
    act_tensor_scale: float


@dataclass
class QuantAct:
    prec: int
    M: int
    K: int
    r: int
    codes: torch.Tensor    # uint8 [M, K/2]
    scales: torch.Tensor   # uint8 bytes
    P: Optional[torch.Tensor]  # bf16 [M, r]


def _check_packed(pw: PackedWeight) -> None:
    """The buffers of a packed weight have the sizes its (prec, K, N, r) imply."""
    _need(pw.prec in (NVFP4, INT4), "precision {!r}", pw.prec)
    _is(pw.codes, torch.uint8, (pw.N, pw.K // 2), "pw.codes")
    _at_least(pw.scales, torch.uint8, scale_bytes(pw.prec, pw.N, pw.K), "pw.scales")
    _is(pw.tensor_scale, torch.float32, (2,), "pw.tensor_scale")
    _is(pw.inv_lambda, torch.float32, (pw.K,), "pw.inv_lambda")
    if pw.r:
        _is(pw.lr_up, torch.bfloat16, (pw.N, 2 * pw.r if pw.prec == NVFP4 else pw.r), "pw.lr_up")


def pack_weight(prec, W: torch.Tensor, lam: torch.Tensor, L1: Optional[torch.Tensor],
                L2: Optional[torch.Tensor], act_tensor_scale: float = 1.0, stream=None) -> PackedWeight:
    """svdq_pack_weight: W fp32 [K, N], lam fp32 [K], L1 bf16 [K, r], L2 bf16 [r, N]."""
    p = _prec(prec)
    _need(p in (NVFP4, INT4), "precision {!r}", prec)
    _need(W.dim() == 2 and W.dtype == torch.float32, "W: expected float32 [K, N]")
    K, N = W.shape
    r = 0 if L1 is None else L1.shape[1]
    _is(lam, torch.float32, (K,), "lambda")
    if r:
        _is(L1, torch.bfloat16, (K, r), "L1")
        _is(L2, torch.bfloat16, (r, N), "L2")
    else:
        _need(L2 is None or L2.numel() == 0, "L2 given without L1")
    dev = W.device
    codes = torch.empty((N, K // 2), dtype=torch.uint8, device=dev)
    scales = torch.empty(max(scale_bytes(p, N, K), 16), dtype=torch.uint8, device=dev)
    ts = torch.empty(4, dtype=torch.float32, device=dev)[:2]
    inv = torch.empty(K, dtype=torch.float32, device=dev)
    rr = (2 * r if p == NVFP4 else r)
    lr_up = torch.empty((N, rr), dtype=torch.bfloat16, device=dev) if r else None
    _check("svdq_pack_weight", load().svdq_pack_weight(
        p, K, N, r, _ptr(W), _ptr(lam), _ptr(L1), _ptr(L2), float(act_tensor_scale), _ptr(codes),
        _ptr(scales), _ptr(ts), _ptr(inv), _ptr(lr_up), _stream(stream)))
    return PackedWeight(p, K, N, r, codes, scales, ts, inv, lr_up, float(act_tensor_scale))


def quantize_act(x: torch.Tensor, pw: PackedWeight, L1: Optional[torch.Tensor], stream=None,
                 out: Optional[QuantAct] = None) -> QuantAct:
    """svdq_quantize_act: x bf16 [M, K] -> codes, scales, P. The activation
    tensor scale is the one packed into ``pw.tensor_scale`` (read on the device)."""
    _need(x.dim() == 2 and x.dtype == torch.bfloat16, "x: expected bfloat16 [M, K]")
    M, K = x.shape
    _check_packed(pw)
    p, r = pw.prec, pw.r
    _need(K == pw.K, "x has K = {}, the packed weight K = {}", K, pw.K)
    if r:
        _is(L1, torch.bfloat16, (K, r), "L1")
    dev = x.device
    if out is None:
        out = QuantAct(p, M, K, r, torch.empty((M, K // 2), dtype=torch.uint8, device=dev),
                       torch.empty(max(scale_bytes(p, M, K), 16), dtype=torch.uint8, device=dev),
                       torch.empty((M, r), dtype=torch.bfloat16, device=dev) if r else None)
    else:
        _need(out.prec == p and out.M == M and out.K == K and out.r == r,
              "out: QuantAct of another shape or precision")
        _is(out.codes, torch.uint8, (M, K // 2), "out.codes")
        _at_least(out.scales, torch.uint8, scale_bytes(p, M, K), "out.scales")
        if r:
            _is(out.P, torch.bfloat16, (M, r), "out.P")
    px, pil, pts, pl1, pc, psc, pp = _ptrs(x, pw.inv_lambda, pw.tensor_scale, L1, out.codes, out.scales, out.P)
    _check("svdq_quantize_act", load().svdq_quantize_act(p, M, K, r, px, pil, pts, pl1, pc, psc, pp, _stream(stream)))
    return out


def w4a4_linear(qa: QuantAct, pw: PackedWeight, bias: Optional[torch.Tensor] = None,
                out_dtype: str = "bf16", stream=None, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """svdq_w4a4_linear: the 4-bit GEMM with the low-rank up-projection and bias fused."""
    M, K, N = qa.M, qa.K, pw.N
    _check_packed(pw)
    _need(qa.prec == pw.prec and qa.K == pw.K and qa.r == pw.r,
          "activations (prec {}, K {}, r {}) do not match the weight (prec {}, K {}, r {})",
          qa.prec, qa.K, qa.r, pw.prec, pw.K, pw.r)
    _is(qa.codes, torch.uint8, (M, K // 2), "qa.codes")
    _at_least(qa.scales, torch.uint8, scale_bytes(qa.prec, M, K), "qa.scales")
    if qa.r:
        _is(qa.P, torch.bfloat16, (M, qa.r), "qa.P")
    if bias is not None:
        _is(bias, torch.bfloat16, (N,), "bias")
    _need(out_dtype in _OUT, "out_dtype {!r}", out_dtype)
    want = {"bf16": (torch.bfloat16, (M, N)), "f32": (torch.float32, (M, N)),
            "i32_groups": (torch.int32, (M, N, K // 64)), "bf16_gelu": (torch.bfloat16, (M, N))}[out_dtype]
    if out is not None:
        _is(out, want[0], want[1], "out")
    if out is None:
        if out_dtype in ("bf16", "bf16_gelu"):
            out = torch.empty((M, N), dtype=torch.bfloat16, device=qa.codes.device)
        elif out_dtype == "f32":
            out = torch.empty((M, N), dtype=torch.float32, device=qa.codes.device)
        else:
            out = torch.empty((M, N, K // 64), dtype=torch.int32, device=qa.codes.device)
    ptrs = _ptrs(qa.codes, qa.scales, qa.P, pw.codes, pw.scales, pw.tensor_scale, pw.lr_up, bias, out)
    _check("svdq_w4a4_linear", load().svdq_w4a4_linear(pw.prec, M, K, N, pw.r, *ptrs, _OUT[out_dtype],
                                                       _stream(stream)))
    return out


@dataclass
class RopeTable:
    """The rotary cos/sin tables of M rows in svdq_rope_pack's layout (fp32,
    svdq_rope_packed_bytes(M) bytes)."""
    M: int
    data: torch.Tensor


def pack_rope(cos: torch.Tensor, sin: torch.Tensor, stream=None) -> RopeTable:
    """svdq_rope_pack: cos, sin fp32 [M, 64] -> the packed table the fused QKV
    epilogue reads (once per set of positions; every layer can share it)."""
    _need(cos.dim() == 2, "cos: expected [M, 64]")
    M = cos.shape[0]
    _is(cos, torch.float32, (M, 64), "cos")
    _is(sin, torch.float32, (M, 64), "sin")
    data = torch.empty(load().svdq_rope_packed_bytes(M) // 4, dtype=torch.float32, device=cos.device)
    pc, ps, pr = _ptrs(cos, sin, data)
    _check("svdq_rope_pack", load().svdq_rope_pack(M, pc, ps, pr, _stream(stream)))
    return RopeTable(M, data)


def w4a4_linear_qkv(qa: QuantAct, pw: PackedWeight, heads: int, norm_q: torch.Tensor, norm_k: torch.Tensor,
                    eps: float, rope: RopeTable, bias: Optional[torch.Tensor] = None,
                    stream=None, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """svdq_w4a4_linear_qkv: the NVFP4 layer as a grouped Q/K/V projection (N =
    3 * heads * 128) with per-head RMSNorm of Q and K and the rotary embedding
    in the GEMM's epilogue. rope: pack_rope of the M rows' cos/sin [M, 64]."""
    M, K, N = qa.M, qa.K, pw.N
    _check_packed(pw)
    _need(pw.prec == NVFP4 and qa.prec == NVFP4, "the fused QKV epilogue is NVFP4 only")
    _need(qa.K == pw.K and qa.r == pw.r, "activations (K {}, r {}) do not match the weight (K {}, r {})",
          qa.K, qa.r, pw.K, pw.r)
    _need(heads > 0 and N == 3 * heads * 128, "N = {} is not 3 * heads * 128 with heads = {}", N, heads)
    _is(qa.codes, torch.uint8, (M, K // 2), "qa.codes")
    _at_least(qa.scales, torch.uint8, scale_bytes(qa.prec, M, K), "qa.scales")
    if qa.r:
        _is(qa.P, torch.bfloat16, (M, qa.r), "qa.P")
    _is(norm_q, torch.bfloat16, (128,), "norm_q")
    _is(norm_k, torch.bfloat16, (128,), "norm_k")
    _need(isinstance(rope, RopeTable) and rope.M == M, "rope: expected pack_rope of the layer's {} rows", M)
    _is(rope.data, torch.float32, (load().svdq_rope_packed_bytes(M) // 4,), "rope.data")
    if bias is not None:
        _is(bias, torch.bfloat16, (N,), "bias")
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=qa.codes.device)
    else:
        _is(out, torch.bfloat16, (M, N), "out")
    ptrs = _ptrs(qa.codes, qa.scales, qa.P, pw.codes, pw.scales, pw.tensor_scale, pw.lr_up, bias, norm_q, norm_k)
    pr, po = _ptrs(rope.data, out)
    _check("svdq_w4a4_linear_qkv", load().svdq_w4a4_linear_qkv(M, K, heads, pw.r, *ptrs, float(eps), pr, po,
                                                               _stream(stream)))
    return out


def qkv_norm_rope(y: torch.Tensor, heads: int, norm_q: torch.Tensor, norm_k: torch.Tensor, eps: float,
                  cos: torch.Tensor, sin: torch.Tensor, stream=None) -> torch.Tensor:
    """svdq_qkv_norm_rope: per-head RMSNorm + rotary embedding of the Q and K
    sections of a bf16 grouped-QKV output y [M, 3 * heads * 128], in place."""
    _need(y.dim() == 2 and y.dtype == torch.bfloat16, "y: expected bfloat16 [M, N]")
    M, N = y.shape
    _need(heads > 0 and N == 3 * heads * 128, "N = {} is not 3 * heads * 128 with heads = {}", N, heads)
    _is(norm_q, torch.bfloat16, (128,), "norm_q")
    _is(norm_k, torch.bfloat16, (128,), "norm_k")
    _is(cos, torch.float32, (M, 64), "cos")
    _is(sin, torch.float32, (M, 64), "sin")
    pq, pk, pc, ps, py = _ptrs(norm_q, norm_k, cos, sin, y)
    _check("svdq_qkv_norm_rope", load().svdq_qkv_norm_rope(M, heads, pq, pk, float(eps), pc, ps, py,
                                                           _stream(stream)))
    return y


def svdq_linear(x: torch.Tensor, pw: PackedWeight, L1: Optional[torch.Tensor],
                bias: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """The whole layer: quantize_act then w4a4_linear (two launches)."""
    return w4a4_linear(quantize_act(x, pw, L1, stream), pw, bias, stream=stream)


@dataclass
class AwqWeight:
    K: int
    N: int
    q: torch.Tensor       # uint8 [N, K/2]
    scales: torch.Tensor  # bf16 [N, K/64]
    zeros: torch.Tensor   # bf16 [N, K/64]


def awq_pack_weight(W: torch.Tensor, stream=None, out: Optional[AwqWeight] = None) -> AwqWeight:
    """awq_pack_weight: W fp32 [K, N] -> q, scales, zeros (into ``out``'s
    buffers when given)."""
    _need(W.dim() == 2 and W.dtype == torch.float32, "W: expected float32 [K, N]")
    K, N = W.shape
    dev = W.device
    if out is None:
        out = AwqWeight(K, N, torch.empty((N, K // 2), dtype=torch.uint8, device=dev),
                        torch.empty((N, K // 64), dtype=torch.bfloat16, device=dev),
                        torch.empty((N, K // 64), dtype=torch.bfloat16, device=dev))
    else:
        _need(out.K == K and out.N == N, "out: AwqWeight of K {}, N {}", out.K, out.N)
        _is(out.q, torch.uint8, (N, K // 2), "out.q")
        _is(out.scales, torch.bfloat16, (N, K // 64), "out.scales")
        _is(out.zeros, torch.bfloat16, (N, K // 64), "out.zeros")
    _check("awq_pack_weight", load().awq_pack_weight(K, N, _ptr(W), _ptr(out.q), _ptr(out.scales),
                                                     _ptr(out.zeros), _stream(stream)))
    return out


def awq_w4a16_linear(x: torch.Tensor, w: AwqWeight, bias: Optional[torch.Tensor] = None, stream=None,
                     out: Optional[torch.Tensor] = None) -> torch.Tensor:
    _need(x.dim() == 2 and x.dtype == torch.bfloat16, "x: expected bfloat16 [M, K]")
    M, K = x.shape
    _need(K == w.K, "x has K = {}, the packed weight K = {}", K, w.K)
    _is(w.q, torch.uint8, (w.N, w.K // 2), "w.q")
    _is(w.scales, torch.bfloat16, (w.N, w.K // 64), "w.scales")
    _is(w.zeros, torch.bfloat16, (w.N, w.K // 64), "w.zeros")
    if bias is not None:
        _is(bias, torch.bfloat16, (w.N,), "bias")
    if out is not None:
        _is(out, torch.bfloat16, (M, w.N), "out")
    if out is None:
        out = torch.empty((M, w.N), dtype=torch.bfloat16, device=x.device)
    _check("awq_w4a16_linear", load().awq_w4a16_linear(
        M, K, w.N, _ptr(x), _ptr(w.q), _ptr(w.scales), _ptr(w.zeros), _ptr(bias), _ptr(out),
        _stream(stream)))
    return out


def device_error() -> int:
    """Reads and clears the device error word; raises SvdqError if it was set."""
    bits = C.c_uint(0)
    st = load().svdq_device_error(C.byref(bits))
    if st not in (0, int(Status.TIMEOUT), int(Status.CUDA)):
        _check("svdq_device_error", st)
    if st:
        raise SvdqError("svdq_device_error", st, f"device error word = {bits.value:#x}")
    return bits.value


def set_wait_limit_ns(ns: int) -> None:
    load().svdq_set_wait_limit_ns(int(ns))


def probe_convert(x: torch.Tensor, e2m1: bool = True, e4m3: bool = True, bf16: bool = True, stream=None):
    n = x.numel()
    o1 = torch.empty(n, dtype=torch.uint8, device=x.device) if e2m1 else None
    o2 = torch.empty(n, dtype=torch.uint8, device=x.device) if e4m3 else None
    o3 = torch.empty(n, dtype=torch.int16, device=x.device) if bf16 else None
    _check("svdq_probe_convert", load().svdq_probe_convert(_ptr(x), n, _ptr(o1), _ptr(o2), _ptr(o3),
                                                           _stream(stream)))
    return o1, o2, o3


def probe_wait_timeout(limit_ns: int, stream=None) -> None:
    _check("svdq_probe_wait_timeout", load().svdq_probe_wait_timeout(int(limit_ns), _stream(stream)))


def probe_mma_peak(iters: int, mode: int = 0, stream=None) -> float:
    """Launches the tensor-core rate probe; returns the FLOPs it performs (the
    caller times it on its stream)."""
    _check("svdq_probe_mma_peak", load().svdq_probe_mma_peak(int(iters), int(mode), _stream(stream)))
    sms = torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count
    return float(sms // 2) * iters * 4 * 2.0 * 256 * 256 * 64


def debug_force_arch(major: int, minor: int = 0) -> None:
    load().svdq_debug_force_arch(int(major), int(minor))
