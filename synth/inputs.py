"""Seeded, diffusion-transformer-shaped synthetic inputs.

The pages describe SVDQuant checkpoints of diffusion transformers (ERNIE-Image,
Flux) run at 1024x1024 for 8 steps (Diffusers "Nunchaku Lite" page, section
"Load a quantized pipeline"; blog "Introducing Nunchaku 4-bit inference in
Diffusers", section "Background: SVDQuant and Nunchaku"). Their weights and
prompts are not available here, so these tensors stand in for them with the
shapes of one DiT block: hidden size 3072, 4096 image + 512 text tokens.

Random numbers
--------------
Every tensor draws from its own sub-stream ``key = splitmix64(seed*1000 +
tensor_id)``. Element ``i`` of a stream is ``splitmix64_mix(key + (i+1) *
0x9E3779B97F4A7C15)`` (Steele, Lea, Flood, "Fast splittable pseudorandom number
generators", OOPSLA 2014), mapped to a double in [0, 1) by its top 53 bits.
Normals use the Box-Muller transform on the even/odd counter pairs.

Layer-parameter recipe (stand-in for a calibrated checkpoint)
--------------------------------------------------------------
SVDQuant migrates activation outliers into the weights with a per-channel
smoothing vector and keeps a 16-bit low-rank branch (blog, "Background:
SVDQuant and Nunchaku"). A deployed layer reads lambda, L1 and L2 from its
checkpoint; calibration itself is offline tooling and out of scope. Here they
are produced from the synthetic x and W with the recipe the workload
description states: lambda_k = sqrt(max_m |x_mk| / max_n |W_kn|) (1 where either
maximum is 0), and L1 = bf16(U_r S_r), L2 = bf16(V_r^T) from a rank-r SVD of
diag(lambda) W, computed in float64 by randomized subspace iteration (Halko,
Martinsson, Tropp 2011) with a seeded Gaussian test matrix. Both the CUDA path
and the oracle take lambda, L1 and L2 as inputs, so the SVD's own accuracy does
not enter parity.
"""

from __future__ import annotations

import numpy as np
import torch

_GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)

# tensor ids inside one seed
_T_X, _T_W, _T_B, _T_XOUT, _T_WOUT, _T_OMEGA = 1, 2, 3, 4, 5, 6
_T_WQ, _T_WK = 7, 8  # RMSNorm weights of the fused QKV epilogue


def _mix(z: np.ndarray) -> np.ndarray:
    with np.errstate(over="ignore"):
        z = (z ^ (z >> np.uint64(30))) * _M1
        z = (z ^ (z >> np.uint64(27))) * _M2
        return z ^ (z >> np.uint64(31))


def _key(seed: int, tensor_id: int) -> np.uint64:
    base = np.array([(seed * 1000 + tensor_id) & 0xFFFFFFFFFFFFFFFF], dtype=np.uint64)
    with np.errstate(over="ignore"):
        return _mix(base + _GOLDEN)[0]


def _bits(key: np.uint64, start: int, n: int) -> np.ndarray:
    ctr = np.arange(start + 1, start + n + 1, dtype=np.uint64)
    with np.errstate(over="ignore"):
        return _mix(key + ctr * _GOLDEN)


def uniform(seed: int, tensor_id: int, n: int) -> np.ndarray:
    """n doubles in [0, 1) from sub-stream (seed, tensor_id)."""
    z = _bits(_key(seed, tensor_id), 0, n)
    return (z >> np.uint64(11)).astype(np.float64) * (1.0 / 9007199254740992.0)


def normal(seed: int, tensor_id: int, n: int, chunk: int = 1 << 22) -> np.ndarray:
    """n standard normals (float64) from sub-stream (seed, tensor_id)."""
    key = _key(seed, tensor_id)
    out = np.empty(n, dtype=np.float64)
    for s in range(0, n, chunk):
        m = min(chunk, n - s)
        z = _bits(key, 2 * s, 2 * m)
        u = (z >> np.uint64(11)).astype(np.float64) * (1.0 / 9007199254740992.0)
        u1 = 1.0 - u[0::2]  # (0, 1]
        u2 = u[1::2]
        out[s:s + m] = np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * np.pi * u2)
    return out


def _pick(seed: int, tensor_id: int, count: int, total: int) -> np.ndarray:
    """``count`` distinct indices of ``range(total)``, seeded."""
    if count <= 0:
        return np.zeros(0, dtype=np.int64)
    order = np.argsort(uniform(seed, tensor_id, total), kind="stable")
    return np.sort(order[:count])


def bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float values to bfloat16 (round-to-nearest-even, via torch) and
    return the 16-bit patterns as uint16."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32)


def _gelu_erf(z: np.ndarray) -> np.ndarray:
    from scipy.special import erf

    return 0.5 * z * (1.0 + erf(z / np.sqrt(2.0)))


def _activations(seed, tid_off, M, K, out_frac, out_scale, kind):
    z = normal(seed, _T_X + tid_off, M * K).reshape(M, K)
    ch = _pick(seed, _T_XOUT + tid_off, int(round(out_frac * K)), K)
    if len(ch):
        z[:, ch] *= out_scale
    if kind == "gelu":
        z = _gelu_erf(z)
    return bf16_bits(z), ch


def _low_rank(seed, tid_off, What: np.ndarray, r: int, oversample=16, iters=3):
    K, N = What.shape
    if r == 0:
        return np.zeros((K, 0)), np.zeros((0, N))
    ell = min(r + oversample, min(K, N))
    omega = normal(seed, _T_OMEGA + tid_off, N * ell).reshape(N, ell)
    Q, _ = np.linalg.qr(What @ omega)
    for _ in range(iters):
        Q, _ = np.linalg.qr(What.T @ Q)
        Q, _ = np.linalg.qr(What @ Q)
    B = Q.T @ What
    Ub, S, Vt = np.linalg.svd(B, full_matrices=False)
    U = Q @ Ub
    re = min(r, S.size)  # a rank above min(K, N) is padded with zero factors
    L1 = np.zeros((K, r))
    L2 = np.zeros((r, N))
    L1[:, :re] = U[:, :re] * S[:re]
    L2[:re] = Vt[:re]
    return L1, L2


def svdq_layer(seed: int, M: int, K: int, N: int, r: int, *, x_out_frac=0.01,
               x_out_scale=20.0, w_out_rows=0, w_out_scale=1.0, w_std=0.02,
               b_std=0.01, bias=True, x_kind="normal", tid_off=0,
               lam_one=False):
    """One svdq_w4a4 layer's inputs.

    Returns a dict of numpy arrays: x (bf16 bits [M,K]), W (fp32 [K,N]),
    b (bf16 bits [N] or None), lam (fp32 [K]), L1 (bf16 bits [K,r]),
    L2 (bf16 bits [r,N]), plus the outlier channel list ``x_outliers``.

    ``lam_one`` forces lambda = 1 (used by the invariant tests).
    """
    x, ch = _activations(seed, tid_off, M, K, x_out_frac, x_out_scale, x_kind)
    W = normal(seed, _T_W + tid_off, K * N).reshape(K, N) * w_std
    rows = _pick(seed, _T_WOUT + tid_off, w_out_rows, K)
    if len(rows):
        W[rows, :] *= w_out_scale
    W = W.astype(np.float32)
    b = bf16_bits(normal(seed, _T_B + tid_off, N) * b_std) if bias else None

    xf = np.abs(bf16_bits_to_f32(x).astype(np.float64)).max(axis=0) if M else np.zeros(K)
    wf = np.abs(W.astype(np.float64)).max(axis=1)
    lam = np.ones(K)
    ok = (xf > 0) & (wf > 0)
    lam[ok] = np.sqrt(xf[ok] / wf[ok])
    if lam_one:
        lam[:] = 1.0
    lam = lam.astype(np.float32)

    What = lam.astype(np.float64)[:, None] * W.astype(np.float64)
    U, V = _low_rank(seed, tid_off, What, r)
    L1 = bf16_bits(U).reshape(K, r)
    L2 = bf16_bits(V).reshape(r, N)
    return dict(x=x, W=W, b=b, lam=lam, L1=L1, L2=L2, x_outliers=ch,
                M=M, K=K, N=N, r=r)


def awq_inputs(seed: int, M: int, K: int, N: int, w_std=0.02):
    """awq_w4a16 inputs: x bf16 bits [M,K] ~ N(0,1), W fp32 [K,N] ~ N(0, w_std)."""
    x = bf16_bits(normal(seed, _T_X, M * K).reshape(M, K))
    W = (normal(seed, _T_W, K * N).reshape(K, N) * w_std).astype(np.float32)
    return dict(x=x, W=W, M=M, K=K, N=N)


def qkv_epilogue_inputs(seed: int, M: int, head_dim: int, heads: int, rope_base: float = 10000.0):
    """Inputs of the fused QKV epilogue on a grouped Q/K/V projection of `heads`
    heads of `head_dim` columns per section: RMSNorm weights wq, wk (bf16 bits
    [head_dim], ~ U(0.5, 1.5), standing in for trained ones) and rotary tables
    cos, sin (fp32 [M, head_dim/2]) for token positions 0..M-1 with the usual
    frequencies base^(-2i/head_dim). eps = 1e-6."""
    wq = bf16_bits(0.5 + uniform(seed, _T_WQ, head_dim))
    wk = bf16_bits(0.5 + uniform(seed, _T_WK, head_dim))
    pos = np.arange(M, dtype=np.float64)[:, None]
    freq = rope_base ** (-2.0 * np.arange(head_dim // 2, dtype=np.float64) / head_dim)[None, :]
    ang = pos * freq
    return dict(wq=wq, wk=wk, cos=np.cos(ang).astype(np.float32), sin=np.sin(ang).astype(np.float32),
                eps=1e-6, heads=heads, head_dim=head_dim)


# The five workloads. Sizes, distributions and outlier structure follow the
# workload description; seeds are the workload index minus one.
CONFIGS = {
    "c1_smoke_nvfp4": dict(kind="svdq", prec="nvfp4", seed=0, M=256, K=1024, N=1024, r=32,
                           x_out_frac=0.01, x_out_scale=20.0, w_out_rows=8, w_out_scale=10.0),
    "c2_awq_gemv": dict(kind="awq", seed=1, Ms=(1, 2, 4, 16), K=3072, N=18432),
    "c3_qkv_nvfp4": dict(kind="svdq", prec="nvfp4", seed=2, M=4608, K=3072, N=9216, r=32,
                         x_out_frac=0.005, x_out_scale=30.0),
    "c4_mlp_up_nvfp4": dict(kind="svdq", prec="nvfp4", seed=3, M=4608, K=3072, N=12288, r=32,
                            x_out_frac=0.005, x_out_scale=30.0),
    "c4_mlp_down_nvfp4": dict(kind="svdq", prec="nvfp4", seed=3, M=4608, K=12288, N=3072, r=32,
                              x_out_frac=0.005, x_out_scale=30.0, x_kind="gelu", tid_off=10),
    "c5_qkv_int4": dict(kind="svdq", prec="int4", seed=4, M=4608, K=3072, N=9216, r=32,
                        x_out_frac=0.005, x_out_scale=30.0),
}


def config_layer(name: str, M: int | None = None):
    """Inputs of a named svdq workload (optionally with fewer rows M)."""
    c = dict(CONFIGS[name])
    assert c.pop("kind") == "svdq"
    c.pop("prec")
    if M is not None:
        c["M"] = M
    return svdq_layer(**c)
