"""Test helpers: layout conversions for comparison, tolerance rules, and
moving synthetic inputs onto the GPU. Nothing here computes the layer."""

from __future__ import annotations

import numpy as np


def untile_nvfp4_scales(tiled: np.ndarray, rows: int, K: int) -> np.ndarray:
    """Tiled NVFP4 scale bytes (the layout documented for svdq_scale_bytes) ->
    plain [rows, K/16]."""
    tiled = np.asarray(tiled, np.uint8).reshape(-1)
    m = np.arange(rows)[:, None]
    b = np.arange(K // 16)[None, :]
    idx = ((m // 128) * (K // 64) + b // 4) * 512 + 16 * (m % 32) + 4 * ((m % 128) // 32) + b % 4
    return tiled[idx]


def int4_act_scale_pitch(K: int) -> int:
    """Row pitch (in scales) of INT4 activation scales: K/64 rounded up to a
    multiple of 8, so that every row starts on a 16-byte boundary."""
    return ((K // 64 + 7) // 8) * 8


def unpad_int4_act_scales(raw: np.ndarray, rows: int, K: int) -> np.ndarray:
    """INT4 activation scale bytes (row pitch int4_act_scale_pitch) -> plain
    bf16 bits [rows, K/64]."""
    pitch = int4_act_scale_pitch(K)
    return np.asarray(raw, np.uint8).reshape(-1)[: rows * pitch * 2].view(np.uint16).reshape(rows, pitch)[:, : K // 64]


def bf16_ulp(v: np.ndarray) -> np.ndarray:
    a = np.abs(np.asarray(v, np.float64))
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -126)))
    return np.exp2(e - 7)


def check_bf16_output(y_gpu_bf16_as_f32: np.ndarray, y_ref_exact: np.ndarray, y_ref_bf16_as_f32: np.ndarray,
                      frob_tol: float = 2e-3, abs_rms: float = 1e-2):
    """bf16 outputs: relative Frobenius error <= frob_tol against the oracle's
    bf16-rounded output, and per element |d| <= abs_rms * rms(y) + 1 bf16 ulp
    of the reference (one ulp absorbs a flip of the final rounding)."""
    g = np.asarray(y_gpu_bf16_as_f32, np.float64)
    r = np.asarray(y_ref_bf16_as_f32, np.float64)
    rms = np.sqrt(np.mean(np.asarray(y_ref_exact, np.float64) ** 2))
    d = np.abs(g - r)
    frob = np.linalg.norm(g - r) / max(np.linalg.norm(r), 1e-300)
    bound = abs_rms * rms + bf16_ulp(r)
    worst = float(np.max(d - bound)) if d.size else 0.0
    stats = dict(frob=float(frob), max_abs=float(d.max()) if d.size else 0.0, rms=float(rms),
                 n_over=int((d > bound).sum()), worst_excess=worst)
    assert frob <= frob_tol, stats
    assert (d <= bound).all(), stats
    return stats


def check_f32_output(y_gpu: np.ndarray, y_ref_exact: np.ndarray, frob_tol: float = 2e-3, abs_rms: float = 1e-2):
    """fp32 (unrounded) outputs: strict max|d| <= abs_rms * rms(y) and relative
    Frobenius <= frob_tol against the oracle's exact (float64) output."""
    g = np.asarray(y_gpu, np.float64)
    r = np.asarray(y_ref_exact, np.float64)
    rms = np.sqrt(np.mean(r ** 2))
    d = np.abs(g - r)
    frob = np.linalg.norm(g - r) / max(np.linalg.norm(r), 1e-300)
    stats = dict(frob=float(frob), max_abs=float(d.max()) if d.size else 0.0, rms=float(rms))
    assert frob <= frob_tol, stats
    assert d.max() <= abs_rms * rms, stats
    return stats
