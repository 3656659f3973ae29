"""GPU parity of the fused QKV epilogue (svdq_w4a4_linear_qkv): the NVFP4
layer as a grouped Q/K/V projection with per-head RMSNorm of Q and K and the
rotary embedding in the GEMM's epilogue, against the oracle's qkv_norm_rope
applied to the oracle's unrounded layer output (Diffusers "Nunchaku Lite"
page, section on fused kernels). bf16 output, the bf16 tolerance rule of
tests/_util.py. The V section must equal the plain layer's output bit for
bit (it takes the same epilogue)."""

import numpy as np
import pytest
import torch

import oracle
import synth
import bit_w4a4_quantized_nvfp4_b200 as svdq
from tests._util import check_bf16_output

pytestmark = pytest.mark.gpu


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


def run_case(d, e, heads, rows=None, bias=True):
    M, N = d["M"], d["N"]
    L1 = bf16_dev(d["L1"]) if d["r"] else None
    L2 = bf16_dev(d["L2"]) if d["r"] else None
    pw = svdq.pack_weight("nvfp4", torch.from_numpy(d["W"]).cuda(), torch.from_numpy(d["lam"]).cuda(), L1, L2)
    qa = svdq.quantize_act(bf16_dev(d["x"]), pw, L1)
    b = bf16_dev(d["b"]) if bias else None
    cos, sin = torch.from_numpy(e["cos"]).cuda(), torch.from_numpy(e["sin"]).cuda()
    rope = svdq.pack_rope(cos, sin)
    y = svdq.w4a4_linear_qkv(qa, pw, heads, bf16_dev(e["wq"]), bf16_dev(e["wk"]), e["eps"], rope, b)
    y_plain = svdq.w4a4_linear(qa, pw, b)
    torch.cuda.synchronize()
    assert svdq.device_error() == 0
    yg, yp = bf16_np(y), bf16_np(y_plain)
    # V heads: the plain epilogue, bit for bit
    assert np.array_equal(yg[:, 2 * heads * 128:], yp[:, 2 * heads * 128:])
    w = oracle.pack_weight("nvfp4", d["W"], d["lam"], d["L1"], d["L2"])
    a = oracle.quantize_act("nvfp4", d["x"], w["inv_lam"], 1.0, d["L1"])
    sel = np.arange(M, dtype=np.int32) if rows is None else rows
    yl = oracle.linear("nvfp4", a, w, 1.0, d["L2"], d["b"] if bias else None, rows=sel)
    yo = oracle.qkv_norm_rope(yl, heads, 128, e["wq"], e["wk"], e["eps"], e["cos"][sel], e["sin"][sel])
    return check_bf16_output(oracle.bf16_to_f32(yg[sel]), yo, oracle.bf16_to_f32(oracle.bf16_rn(yo)))


@pytest.mark.parametrize("M,K,heads,r,bias", [(200, 512, 3, 16, True), (33, 256, 1, 32, False),
                                              (129, 1024, 2, 32, True)])
def test_qkv_epilogue_matches_oracle(M, K, heads, r, bias):
    """Ragged rows, an odd head count (tiles that start in one section and
    end in the next), one head per section, no bias."""
    N = 3 * heads * 128
    d = synth.svdq_layer(41, M, K, N, r, x_out_frac=0.01, x_out_scale=20.0, bias=bias)
    e = synth.qkv_epilogue_inputs(41, M, 128, heads)
    run_case(d, e, heads, bias=bias)


def test_qkv_epilogue_c3_full_size():
    """The fused-QKV projection of the benchmark workload (M4608 K3072, 24
    heads of 128 per section, N 9216, r 32) with the C3 rotary tables: 512
    seeded rows against the oracle, the V section against the plain layer."""
    c = synth.CONFIGS["c3_qkv_nvfp4"]
    d = synth.config_layer("c3_qkv_nvfp4")
    e = synth.qkv_epilogue_inputs(c["seed"], c["M"], 128, c["N"] // 384)
    rows = np.sort(np.random.default_rng(11).choice(c["M"], 512, replace=False)).astype(np.int32)
    run_case(d, e, c["N"] // 384, rows=rows)


@pytest.mark.parametrize("M,heads", [(77, 3), (256, 2)])
def test_separate_norm_rope_pass_matches_oracle(M, heads):
    """svdq_qkv_norm_rope on a bf16 grouped-QKV tensor against the oracle's
    qkv_norm_rope of the same bf16 values; the V section is untouched."""
    N = 3 * heads * 128
    rng = np.random.default_rng(M + heads)
    yb = synth.bf16_bits(rng.normal(0, 2.0, (M, N)))
    e = synth.qkv_epilogue_inputs(43, M, 128, heads)
    y = bf16_dev(yb)
    svdq.qkv_norm_rope(y, heads, bf16_dev(e["wq"]), bf16_dev(e["wk"]), e["eps"],
                       torch.from_numpy(e["cos"]).cuda(), torch.from_numpy(e["sin"]).cuda())
    torch.cuda.synchronize()
    yg = bf16_np(y)
    assert np.array_equal(yg[:, 2 * heads * 128:], yb[:, 2 * heads * 128:])
    yo = oracle.qkv_norm_rope(oracle.bf16_to_f32(yb).astype(np.float64), heads, 128, e["wq"], e["wk"], e["eps"],
                              e["cos"], e["sin"])
    check_bf16_output(oracle.bf16_to_f32(yg), yo, oracle.bf16_to_f32(oracle.bf16_rn(yo)))


@pytest.mark.parametrize("M", [77, 64, 1])
def test_rope_pack_layout(M):
    """svdq_rope_pack moves every cos/sin value, unchanged, to the offset the
    header states; the rows that pad the last 32-row block are zero."""
    e = synth.qkv_epilogue_inputs(44, M, 128, 1)
    rope = svdq.pack_rope(torch.from_numpy(e["cos"]).cuda(), torch.from_numpy(e["sin"]).cuda())
    torch.cuda.synchronize()
    got = rope.data.cpu().numpy().view(np.uint32)
    nb = (M + 31) // 32
    assert got.size == nb * 4096
    want = np.zeros(nb * 4096, np.uint32)
    for tab, part in ((e["cos"], 0), (e["sin"], 1)):
        bits = np.ascontiguousarray(tab, np.float32).view(np.uint32)
        for m in range(M):
            for i in range(64):
                want[((m // 32 * 16 + i // 4) * 2 + part) * 128 + (m % 32) * 4 + i % 4] = bits[m, i]
    assert np.array_equal(got, want)


def test_qkv_epilogue_writes_nothing_past_y():
    """The fused epilogue's output lives in a larger buffer filled with a
    sentinel: after the call the bytes past y still hold it (ragged M, an odd
    head count so the last column tile is half past N), and y matches the
    oracle."""
    M, K, heads, r = 77, 256, 3, 16
    N = 3 * heads * 128
    d = synth.svdq_layer(45, M, K, N, r)
    e = synth.qkv_epilogue_inputs(45, M, 128, heads)
    L1, L2 = bf16_dev(d["L1"]), bf16_dev(d["L2"])
    pw = svdq.pack_weight("nvfp4", torch.from_numpy(d["W"]).cuda(), torch.from_numpy(d["lam"]).cuda(), L1, L2)
    qa = svdq.quantize_act(bf16_dev(d["x"]), pw, L1)
    rope = svdq.pack_rope(torch.from_numpy(e["cos"]).cuda(), torch.from_numpy(e["sin"]).cuda())
    pad = 8192
    buf = torch.full((M * N + pad,), -555.0, dtype=torch.bfloat16, device="cuda")
    y = buf[: M * N].view(M, N)
    svdq.w4a4_linear_qkv(qa, pw, heads, bf16_dev(e["wq"]), bf16_dev(e["wk"]), e["eps"], rope, bf16_dev(d["b"]), out=y)
    torch.cuda.synchronize()
    assert svdq.device_error() == 0
    assert (buf[M * N:] == -555.0).all(), "write past the end of y"
    w = oracle.pack_weight("nvfp4", d["W"], d["lam"], d["L1"], d["L2"])
    a = oracle.quantize_act("nvfp4", d["x"], w["inv_lam"], 1.0, d["L1"])
    yl = oracle.linear("nvfp4", a, w, 1.0, d["L2"], d["b"])
    yo = oracle.qkv_norm_rope(yl, heads, 128, e["wq"], e["wk"], e["eps"], e["cos"], e["sin"])
    check_bf16_output(oracle.bf16_to_f32(bf16_np(y)), yo, oracle.bf16_to_f32(oracle.bf16_rn(yo)))
