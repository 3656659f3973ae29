"""GPU parity of the svdq_w4a4 path against the CPU oracle.

Packed codes and scales must match bit for bit; P and y within the float
tolerance rule (tests/_util.py): bf16 y against the oracle's bf16-rounded
output with relative Frobenius <= 2e-3 and |d| <= 1e-2 rms(y) + 1 bf16 ulp;
fp32 y (before the final rounding) against the oracle's exact output with
max |d| <= 1e-2 rms(y) and relative Frobenius <= 2e-3.
"""

import numpy as np
import pytest
import torch

import oracle
import synth
import bit_w4a4_quantized_nvfp4_b200 as svdq
from tests._util import (bf16_ulp, check_bf16_output, check_f32_output, int4_act_scale_pitch,
                         unpad_int4_act_scales, untile_nvfp4_scales)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from bit_w4a4_quantized_nvfp4_b200 import build

    build.build()
    svdq.load()


def bf16_dev(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def bf16_np(t: torch.Tensor) -> np.ndarray:
    return t.cpu().view(torch.int16).numpy().view(np.uint16)


def as_f32(bits: np.ndarray) -> np.ndarray:
    return oracle.bf16_to_f32(bits)


CASES = [
    # name, M, K, N, r, extra synth kwargs
    ("c1_smoke", 256, 1024, 1024, 32, dict(x_out_frac=0.01, x_out_scale=20.0, w_out_rows=8, w_out_scale=10.0)),
    ("ragged_k_tail", 200, 320, 392, 16, dict()),
    ("single_row_block", 129, 256, 128, 32, dict()),
    ("second_rb_partial", 130, 512, 136, 32, dict()),
    ("tiny_m", 5, 64, 8, 0, dict()),
    ("r0_lambda1", 64, 256, 128, 0, dict(lam_one=True)),
    ("m1", 1, 512, 264, 16, dict()),
]


def run_layer(prec, d, s_tx=1.0, out_dtype="bf16"):
    W = torch.from_numpy(d["W"]).cuda()
    lam = torch.from_numpy(d["lam"]).cuda()
    L1 = bf16_dev(d["L1"]) if d["r"] else None
    L2 = bf16_dev(d["L2"]) if d["r"] else None
    x = bf16_dev(d["x"])
    b = bf16_dev(d["b"]) if d["b"] is not None else None
    pw = svdq.pack_weight(prec, W, lam, L1, L2, act_tensor_scale=s_tx)
    qa = svdq.quantize_act(x, pw, L1)
    y = svdq.w4a4_linear(qa, pw, b, out_dtype=out_dtype)
    torch.cuda.synchronize()
    assert svdq.device_error() == 0
    return pw, qa, y


def oracle_layer(prec, d, s_tx=1.0, rows=None):
    w = oracle.pack_weight(prec, d["W"], d["lam"], d["L1"], d["L2"])
    a = oracle.quantize_act(prec, d["x"], w["inv_lam"], s_tx, d["L1"])
    y = oracle.linear(prec, a, w, s_tx, d["L2"], d["b"], rows=rows)
    return w, a, y


def compare_pack_and_act(prec, d, pw, qa, w, a):
    M, K, N, r = d["M"], d["K"], d["N"], d["r"]
    assert np.array_equal(pw.codes.cpu().numpy(), w["codes"])
    assert np.array_equal(pw.inv_lambda.cpu().numpy(), w["inv_lam"])
    ts = pw.tensor_scale.cpu().numpy()
    assert ts[0] == np.float32(w["s_tw"])
    if prec == "nvfp4":
        assert np.array_equal(untile_nvfp4_scales(pw.scales.cpu().numpy(), N, K), w["scales"])
        assert np.array_equal(untile_nvfp4_scales(qa.scales.cpu().numpy(), M, K), a["scales"])
    else:
        assert np.array_equal(unpad_int4_act_scales(qa.scales.cpu().numpy(), M, K), a["scales"])
    assert np.array_equal(qa.codes.cpu().numpy(), a["codes"])
    if r:
        # P = bf16(x_hat L1): the kernel accumulates in fp32 on tensor cores, the
        # oracle in float64. Bound: one bf16 ulp of the final rounding plus
        # 2^-13 * sum_k |x_hat L1| for K/4 + 3 fp32 accumulation steps (a single
        # wrong or dropped term, ~sum/K in size, exceeds it).
        Pg = as_f32(bf16_np(qa.P)).astype(np.float64)
        Po = as_f32(a["P"]).astype(np.float64)
        xf = as_f32(d["x"]).astype(np.float32)
        xh = as_f32(oracle.bf16_rn((xf * w["inv_lam"][None, :]).astype(np.float64))).astype(np.float64)
        mag = np.abs(xh) @ np.abs(as_f32(d["L1"]).astype(np.float64))
        bound = bf16_ulp(Po) + mag * 2.0 ** -13
        assert (np.abs(Pg - Po) <= bound).all(), float(np.max(np.abs(Pg - Po) / bound))
        assert (Pg != Po).mean() < 0.05
        if prec == "nvfp4":
            # prepared up-projection: hi + lo = L2 / (s_tw s_tx) to ~2^-16
            lr = bf16_np(pw.lr_up).reshape(N, 2 * r)
            hl = as_f32(lr[:, :r]).astype(np.float64) + as_f32(lr[:, r:]).astype(np.float64)
            want = as_f32(d["L2"]).astype(np.float64).T / (np.float64(ts[0]) * np.float64(ts[1]))
            assert np.allclose(hl, want, rtol=2.0 ** -15, atol=0)


@pytest.mark.parametrize("name,M,K,N,r,kw", CASES, ids=[c[0] for c in CASES])
def test_nvfp4_layer_matches_oracle(name, M, K, N, r, kw):
    d = synth.svdq_layer(21, M, K, N, r, **kw)
    pw, qa, y = run_layer("nvfp4", d)
    w, a, yo = oracle_layer("nvfp4", d)
    compare_pack_and_act("nvfp4", d, pw, qa, w, a)
    check_bf16_output(as_f32(bf16_np(y)), yo, as_f32(oracle.bf16_rn(yo)))
    # fp32 output before the final rounding, strict bound
    _, _, y32 = run_layer("nvfp4", d, out_dtype="f32")
    check_f32_output(y32.cpu().numpy(), yo)


def test_nvfp4_activation_tensor_scale():
    d = synth.svdq_layer(22, 128, 512, 256, 32)
    pw, qa, y = run_layer("nvfp4", d, s_tx=0.25)
    w, a, yo = oracle_layer("nvfp4", d, s_tx=0.25)
    compare_pack_and_act("nvfp4", d, pw, qa, w, a)
    check_bf16_output(as_f32(bf16_np(y)), yo, as_f32(oracle.bf16_rn(yo)))


def test_nvfp4_no_bias_and_canaries():
    d = synth.svdq_layer(23, 100, 256, 264, 16, bias=False)
    W = torch.from_numpy(d["W"]).cuda()
    lam = torch.from_numpy(d["lam"]).cuda()
    L1, L2, x = bf16_dev(d["L1"]), bf16_dev(d["L2"]), bf16_dev(d["x"])
    pw = svdq.pack_weight("nvfp4", W, lam, L1, L2)
    qa = svdq.quantize_act(x, pw, L1)
    M, N = 100, 264
    big = torch.full((M * N + 4096,), -12345.0, dtype=torch.bfloat16, device="cuda")
    y = big[: M * N].view(M, N)
    svdq.w4a4_linear(qa, pw, None, out=y)
    torch.cuda.synchronize()
    assert (big[M * N:] == -12345.0).all(), "write past the end of y"
    w, a, yo = oracle_layer("nvfp4", d)
    check_bf16_output(as_f32(bf16_np(y)), yo, as_f32(oracle.bf16_rn(yo)))


def test_zero_residual_gpu():
    """W = L1 L2 exactly: every weight code and scale is zero and y is the
    low-rank branch plus bias."""
    rng = np.random.default_rng(9)
    M, K, N, r = 64, 256, 128, 16
    L1f = rng.integers(-3, 4, (K, r)) * 0.25
    L2f = rng.integers(-3, 4, (r, N)) * 0.125
    d = dict(x=synth.bf16_bits(rng.normal(0, 1, (M, K))), W=(L1f @ L2f).astype(np.float32),
             b=synth.bf16_bits(rng.normal(0, 0.01, N)), lam=np.ones(K, np.float32),
             L1=synth.bf16_bits(L1f), L2=synth.bf16_bits(L2f), M=M, K=K, N=N, r=r)
    pw, qa, y = run_layer("nvfp4", d)
    assert not pw.codes.any() and not pw.scales.any()
    assert pw.tensor_scale.cpu()[0].item() == 1.0
    w, a, yo = oracle_layer("nvfp4", d)
    compare_pack_and_act("nvfp4", d, pw, qa, w, a)
    check_bf16_output(as_f32(bf16_np(y)), yo, as_f32(oracle.bf16_rn(yo)))


@pytest.mark.parametrize("name", ["c3_qkv_nvfp4", "c4_mlp_up_nvfp4", "c4_mlp_down_nvfp4"])
def test_full_size_workload_sampled_rows(name):
    """The full-size NVFP4 workloads in the benchmark's launch configuration:
    the fused-QKV projection (M4608 K3072 N9216, the benchmark's workload) and
    both projections of the MLP pair (4608x3072 -> 12288 and, on GELU inputs,
    4608x12288 -> 3072; the K = 12288 activation pass walks 48 chunks, four
    times the QKV's). Weight and activation codes and scales and P are compared
    in full, y on 512 seeded rows (the oracle computes those one by one)."""
    c = dict(synth.CONFIGS[name])
    d = synth.config_layer(name)
    pw, qa, y = run_layer("nvfp4", d)
    rows = np.sort(np.random.default_rng(3).choice(c["M"], 512, replace=False)).astype(np.int32)
    w, a, yo = oracle_layer("nvfp4", d, rows=rows)
    compare_pack_and_act("nvfp4", d, pw, qa, w, a)
    check_bf16_output(as_f32(bf16_np(y))[rows], yo, as_f32(oracle.bf16_rn(yo)))


@pytest.mark.parametrize("prec,M,K,r", [("nvfp4", 100, 320, 16), ("nvfp4", 33, 1024, 32), ("int4", 70, 192, 32)])
def test_activation_pass_writes_nothing_past_its_outputs(prec, M, K, r):
    """Every output of the activation pass (codes, scales, P) lives in a larger
    buffer filled with a sentinel; after the pass the bytes past each output's
    end still hold it, and the outputs match the oracle (ragged M and K)."""
    d = synth.svdq_layer(27, M, K, 64, r)
    W = torch.from_numpy(d["W"]).cuda()
    lam = torch.from_numpy(d["lam"]).cuda()
    L1, L2 = bf16_dev(d["L1"]), bf16_dev(d["L2"])
    pw = svdq.pack_weight(prec, W, lam, L1, L2)
    pad = 4096
    nc, ns = M * K // 2, svdq.scale_bytes(prec, M, K)
    codes = torch.full((nc + pad,), 0xA5, dtype=torch.uint8, device="cuda")
    scales = torch.full((ns + pad,), 0x5A, dtype=torch.uint8, device="cuda")
    P = torch.full((M * r + pad,), -777.0, dtype=torch.bfloat16, device="cuda")
    out = svdq.QuantAct(pw.prec, M, K, r, codes[:nc].view(M, K // 2), scales[:ns], P[: M * r].view(M, r))
    svdq.quantize_act(bf16_dev(d["x"]), pw, L1, out=out)
    torch.cuda.synchronize()
    assert svdq.device_error() == 0
    assert (codes[nc:] == 0xA5).all(), "write past the end of the codes"
    assert (scales[ns:] == 0x5A).all(), "write past the end of the scales"
    assert (P[M * r:] == -777.0).all(), "write past the end of P"
    w = oracle.pack_weight(prec, d["W"], d["lam"], d["L1"], d["L2"])
    a = oracle.quantize_act(prec, d["x"], w["inv_lam"], 1.0, d["L1"])
    compare_pack_and_act(prec, d, pw, out, w, a)


# ------------------------------------------------------------------ INT4 (activation and pack side)
@pytest.mark.parametrize("M,K,N,r", [(256, 1024, 512, 32), (37, 192, 72, 16), (3, 64, 8, 0)])
def test_int4_pack_and_quantize_match_oracle(M, K, N, r):
    d = synth.svdq_layer(24, M, K, N, r, x_out_frac=0.02, x_out_scale=30.0)
    W = torch.from_numpy(d["W"]).cuda()
    lam = torch.from_numpy(d["lam"]).cuda()
    L1 = bf16_dev(d["L1"]) if r else None
    L2 = bf16_dev(d["L2"]) if r else None
    pw = svdq.pack_weight("int4", W, lam, L1, L2)
    qa = svdq.quantize_act(bf16_dev(d["x"]), pw, L1)
    torch.cuda.synchronize()
    w = oracle.pack_weight("int4", d["W"], d["lam"], d["L1"], d["L2"])
    a = oracle.quantize_act("int4", d["x"], w["inv_lam"], 1.0, d["L1"])
    compare_pack_and_act("int4", d, pw, qa, w, a)
    assert np.array_equal(unpad_int4_act_scales(qa.scales.cpu().numpy(), M, K), a["scales"])
    # weight scales are stored group-major [K/64, N]
    assert np.array_equal(pw.scales.cpu().numpy()[: N * (K // 64) * 2].view(np.uint16).reshape(K // 64, N).T,
                          w["scales"])
    if r:
        assert np.array_equal(bf16_np(pw.lr_up).reshape(N, r), d["L2"].T)


# ------------------------------------------------------------------ error paths
def test_unsupported_arch_is_refused():
    d = synth.svdq_layer(25, 8, 64, 8, 0)
    W = torch.from_numpy(d["W"]).cuda()
    lam = torch.from_numpy(d["lam"]).cuda()
    svdq.debug_force_arch(9, 0)
    try:
        with pytest.raises(svdq.SvdqError) as e:
            svdq.pack_weight("nvfp4", W, lam, None, None)
        assert e.value.status == svdq.Status.UNSUPPORTED_ARCH
    finally:
        svdq.debug_force_arch(0, 0)
    svdq.pack_weight("nvfp4", W, lam, None, None)
    torch.cuda.synchronize()


def test_bounded_wait_reports_timeout_and_context_survives():
    svdq.device_error()  # clear
    svdq.probe_wait_timeout(2_000_000)  # 2 ms: nothing ever arrives
    torch.cuda.synchronize()
    with pytest.raises(svdq.SvdqError) as e:
        svdq.device_error()
    assert e.value.status == svdq.Status.TIMEOUT
    assert svdq.device_error() == 0  # cleared
    # the context is still usable
    test_nvfp4_layer_matches_oracle(*CASES[4])


# ------------------------------------------------------------------ INT4 GEMM
@pytest.mark.parametrize("M,K,N,r", [(256, 1024, 512, 32), (37, 192, 72, 16), (130, 256, 264, 64), (3, 64, 8, 0)])
def test_int4_linear_matches_oracle(M, K, N, r):
    d = synth.svdq_layer(26, M, K, N, r, x_out_frac=0.02, x_out_scale=30.0)
    pw, qa, y = run_layer("int4", d)
    w, a, yo = oracle_layer("int4", d)
    compare_pack_and_act("int4", d, pw, qa, w, a)
    check_bf16_output(as_f32(bf16_np(y)), yo, as_f32(oracle.bf16_rn(yo)))
    _, _, y32 = run_layer("int4", d, out_dtype="f32")
    check_f32_output(y32.cpu().numpy(), yo)
    # the int32 group dot products are exact
    gs = svdq.w4a4_linear(qa, pw, None, out_dtype="i32_groups")
    torch.cuda.synchronize()
    assert np.array_equal(gs.cpu().numpy(), oracle.int4_group_sums(a["codes"], w["codes"]))


def test_c5_int4_full_size():
    """INT4 workload (M4608 K3072 N9216 r32, g64): codes and scales in full, y
    on 512 seeded rows, exact int32 group sums on the first 48 rows."""
    c = synth.CONFIGS["c5_qkv_int4"]
    d = synth.config_layer("c5_qkv_int4")
    pw, qa, y = run_layer("int4", d)
    rows = np.sort(np.random.default_rng(5).choice(c["M"], 512, replace=False)).astype(np.int32)
    w, a, yo = oracle_layer("int4", d, rows=rows)
    compare_pack_and_act("int4", d, pw, qa, w, a)
    check_bf16_output(as_f32(bf16_np(y))[rows], yo, as_f32(oracle.bf16_rn(yo)))
    sub = svdq.QuantAct(qa.prec, 48, qa.K, qa.r, qa.codes[:48].contiguous(),
                        qa.scales[: 48 * int4_act_scale_pitch(qa.K) * 2].contiguous(),
                        qa.P[:48].contiguous() if qa.P is not None else None)
    gs = svdq.w4a4_linear(sub, pw, None, out_dtype="i32_groups")
    torch.cuda.synchronize()
    assert np.array_equal(gs.cpu().numpy(), oracle.int4_group_sums(a["codes"][:48], w["codes"]))
