"""GPU parity of the fused GELU-MLP epilogue (Diffusers "Nunchaku Lite" page,
section on fused kernels: the MLP's GELU runs inside the up-projection
kernel): svdq_w4a4_linear with the bf16_gelu output computes GELU (erf form)
of the unrounded layer output and rounds once to bf16; that output is the
down-projection's activation-pass input as it stands.

Tolerance for h = GELU(y): GELU is Lipschitz with constant
max |GELU'| = 1.1289 (at y = sqrt 2), so the layer's own bf16 rule for y
(relative Frobenius <= 2e-3, |d| <= 1e-2 rms(y) + 1 ulp) carries over with
that factor, measured against rms and norm of y, not of h.
"""

import numpy as np
import pytest
import torch

import oracle
import synth
import bit_w4a4_quantized_nvfp4_b200 as svdq
from tests._util import bf16_ulp, untile_nvfp4_scales

pytestmark = pytest.mark.gpu

GELU_LIP = 1.1289


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from bit_w4a4_quantized_nvfp4_b200 import build

    build.build()
    svdq.load()


def bf16_dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def bf16_np(t):
    return t.cpu().view(torch.int16).numpy().view(np.uint16)


def pack(d):
    L1 = bf16_dev(d["L1"]) if d["r"] else None
    L2 = bf16_dev(d["L2"]) if d["r"] else None
    pw = svdq.pack_weight("nvfp4", torch.from_numpy(d["W"]).cuda(), torch.from_numpy(d["lam"]).cuda(), L1, L2)
    return pw, L1


def check_gelu_output(h_gpu_bits, y_exact, h_ref_bits):
    """h_gpu against the oracle's bf16 GELU of the exact layer output."""
    g = oracle.bf16_to_f32(h_gpu_bits).astype(np.float64)
    r = oracle.bf16_to_f32(h_ref_bits).astype(np.float64)
    y = np.asarray(y_exact, np.float64)
    rms_y = np.sqrt(np.mean(y ** 2))
    d = np.abs(g - r)
    bound = GELU_LIP * 1e-2 * rms_y + bf16_ulp(r)
    frob = np.linalg.norm(g - r) / max(np.linalg.norm(y), 1e-300)
    stats = dict(frob=float(frob), max_abs=float(d.max()), rms_y=float(rms_y), n_over=int((d > bound).sum()))
    assert frob <= GELU_LIP * 2e-3, stats
    assert (d <= bound).all(), stats
    return stats


def gelu64(y):
    from scipy.special import erf

    return 0.5 * y * (1.0 + erf(y / np.sqrt(2.0)))


CASES = [
    # M, K, N, r
    (256, 1024, 2048, 32),
    (200, 320, 392, 16),
    (129, 256, 136, 32),
    (5, 64, 8, 0),
    (1, 512, 264, 16),
]


@pytest.mark.parametrize("M,K,N,r", CASES)
def test_gelu_epilogue_matches_oracle(M, K, N, r):
    d = synth.svdq_layer(31, M, K, N, r)
    pw, L1 = pack(d)
    qa = svdq.quantize_act(bf16_dev(d["x"]), pw, L1)
    b = bf16_dev(d["b"])
    h = svdq.w4a4_linear(qa, pw, b, out_dtype="bf16_gelu")
    y32 = svdq.w4a4_linear(qa, pw, b, out_dtype="f32")
    torch.cuda.synchronize()
    assert svdq.device_error() == 0
    assert h.dtype == torch.bfloat16 and tuple(h.shape) == (M, N)
    w = oracle.pack_weight("nvfp4", d["W"], d["lam"], d["L1"], d["L2"])
    a = oracle.quantize_act("nvfp4", d["x"], w["inv_lam"], 1.0, d["L1"])
    yo = oracle.linear("nvfp4", a, w, 1.0, d["L2"], d["b"])
    hg = bf16_np(h)
    check_gelu_output(hg, yo, oracle.gelu_bf16(yo))
    # the epilogue's own arithmetic: GELU of this kernel's unrounded output,
    # in float64, rounded once. fp32 erf and products leave at most the
    # rounding flip of one bf16 ulp plus a few fp32 ulps of y.
    y = y32.cpu().numpy().astype(np.float64)
    hr = oracle.bf16_to_f32(oracle.bf16_rn(gelu64(y))).astype(np.float64)
    dd = np.abs(oracle.bf16_to_f32(hg).astype(np.float64) - hr)
    assert (dd <= bf16_ulp(hr) + 2.0 ** -20 * np.abs(y) + 1e-30).all(), float(dd.max())
    assert (dd == 0).mean() > 0.99


def test_gelu_epilogue_full_size_mlp_up_sampled_rows():
    """The MLP pair's up-projection at full size (M4608 K3072 N12288) in the
    benchmark's launch configuration, GELU output on 512 seeded rows."""
    c = dict(synth.CONFIGS["c4_mlp_up_nvfp4"])
    d = synth.config_layer("c4_mlp_up_nvfp4")
    pw, L1 = pack(d)
    qa = svdq.quantize_act(bf16_dev(d["x"]), pw, L1)
    h = svdq.w4a4_linear(qa, pw, bf16_dev(d["b"]), out_dtype="bf16_gelu")
    torch.cuda.synchronize()
    assert svdq.device_error() == 0
    rows = np.sort(np.random.default_rng(5).choice(c["M"], 512, replace=False)).astype(np.int32)
    w = oracle.pack_weight("nvfp4", d["W"], d["lam"], d["L1"], d["L2"])
    a = oracle.quantize_act("nvfp4", d["x"], w["inv_lam"], 1.0, d["L1"])
    yo = oracle.linear("nvfp4", a, w, 1.0, d["L2"], d["b"], rows=rows)
    check_gelu_output(bf16_np(h)[rows], yo, oracle.gelu_bf16(yo))


def test_mlp_chain_feeds_the_down_projection():
    """Up-projection with the GELU output, then the down-projection's
    activation pass on that output, against the oracle's chain
    (oracle.mlp_gelu_down_act on the oracle's exact up output). Every
    16-element group whose GELU values agree bit for bit must give the same
    codes and scale; the groups that differ are the ones holding a GELU value
    one rounding apart."""
    M, K, F, r = 256, 1024, 2048, 32
    up = synth.svdq_layer(32, M, K, F, r)
    down = synth.svdq_layer(33, M, F, 512, r, x_kind="gelu", tid_off=10)
    pw_u, L1u = pack(up)
    pw_d, L1d = pack(down)
    qa = svdq.quantize_act(bf16_dev(up["x"]), pw_u, L1u)
    h = svdq.w4a4_linear(qa, pw_u, bf16_dev(up["b"]), out_dtype="bf16_gelu")
    qd = svdq.quantize_act(h, pw_d, L1d)
    torch.cuda.synchronize()
    assert svdq.device_error() == 0

    wu = oracle.pack_weight("nvfp4", up["W"], up["lam"], up["L1"], up["L2"])
    au = oracle.quantize_act("nvfp4", up["x"], wu["inv_lam"], 1.0, up["L1"])
    yo = oracle.linear("nvfp4", au, wu, 1.0, up["L2"], up["b"])
    wd = oracle.pack_weight("nvfp4", down["W"], down["lam"], down["L1"], down["L2"])
    ad = oracle.mlp_gelu_down_act("nvfp4", yo, wd["inv_lam"], 1.0, down["L1"])

    hg = bf16_np(h)
    ho = oracle.gelu_bf16(yo)
    check_gelu_output(hg, yo, ho)
    same = (hg == ho).reshape(M, F // 16, 16).all(axis=2)
    assert same.mean() > 0.5, float(same.mean())
    codes_g = qd.codes.cpu().numpy().reshape(M, F // 16, 8)
    codes_o = ad["codes"].reshape(M, F // 16, 8)
    sc_g = untile_nvfp4_scales(qd.scales.cpu().numpy(), M, F)
    assert np.array_equal(codes_g[same], codes_o[same])
    assert np.array_equal(sc_g[same], ad["scales"][same])
    # P of the down-projection: continuous in h, within the GELU rule on |P|
    Pg = oracle.bf16_to_f32(bf16_np(qd.P)).astype(np.float64)
    Po = oracle.bf16_to_f32(ad["P"]).astype(np.float64)
    rel = np.linalg.norm(Pg - Po) / np.linalg.norm(Po)
    assert rel <= 1e-2, float(rel)


def test_gelu_output_mode_is_nvfp4_only():
    d = synth.svdq_layer(34, 16, 128, 64, 0)
    W, lam = torch.from_numpy(d["W"]).cuda(), torch.from_numpy(d["lam"]).cuda()
    pw = svdq.pack_weight("int4", W, lam, None, None)
    qa = svdq.quantize_act(bf16_dev(d["x"]), pw, None)
    with pytest.raises(svdq.SvdqError) as e:
        svdq.w4a4_linear(qa, pw, None, out_dtype="bf16_gelu")
    assert e.value.status == svdq.Status.INVALID_ARG
    torch.cuda.synchronize()
