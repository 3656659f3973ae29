"""GPU parity of the awq_w4a16 path (pack bit-exact, output within the float
tolerance rule) against the CPU oracle."""

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


@pytest.fixture(scope="module")
def full_weight():
    c = synth.CONFIGS["c2_awq_gemv"]
    d = synth.awq_inputs(c["seed"], 16, c["K"], c["N"])
    pk = oracle.awq_pack_weight(d["W"])
    w = svdq.awq_pack_weight(torch.from_numpy(d["W"]).cuda())
    torch.cuda.synchronize()
    return d, pk, w


def test_awq_pack_full_size_bit_exact(full_weight):
    d, pk, w = full_weight
    assert np.array_equal(w.q.cpu().numpy(), pk["q"])
    assert np.array_equal(bf16_np(w.scales), pk["s"])
    assert np.array_equal(bf16_np(w.zeros), pk["z"])


@pytest.mark.parametrize("M", [1, 2, 4, 16])
def test_awq_gemv_full_size(full_weight, M):
    d, pk, w = full_weight
    x = d["x"][:M]
    y = svdq.awq_w4a16_linear(bf16_dev(x), w)
    torch.cuda.synchronize()
    yo = oracle.awq_linear(x, pk)
    check_bf16_output(oracle.bf16_to_f32(bf16_np(y)), yo, oracle.bf16_to_f32(oracle.bf16_rn(yo)))


@pytest.mark.parametrize("M,K,N", [(3, 128, 72), (17, 192, 136), (40, 64, 8), (1, 4096, 24),
                                   # one to four rows (the GEMV kernel): K not a whole number of
                                   # 512-wide stages, an odd group count, N not a whole 64-row tile;
                                   # three rows (the fourth MMA row zero); four rows at K = 16384
                                   # (shared memory too small for the GEMV: the batched kernel)
                                   (1, 320, 72), (2, 576, 200), (2, 64, 8), (1, 1088, 136), (2, 16384, 64),
                                   (3, 320, 72), (4, 576, 200), (4, 64, 8), (3, 1088, 136), (4, 16384, 64)])
def test_awq_ragged_shapes_with_bias(M, K, N):
    d = synth.awq_inputs(31, M, K, N)
    b = synth.bf16_bits(np.linspace(-0.05, 0.05, N))
    pk = oracle.awq_pack_weight(d["W"])
    w = svdq.awq_pack_weight(torch.from_numpy(d["W"]).cuda())
    big = torch.full((M * N + 1024,), 777.0, dtype=torch.bfloat16, device="cuda")
    y = big[: M * N].view(M, N)
    svdq.awq_w4a16_linear(bf16_dev(d["x"]), w, bf16_dev(b), out=y)
    torch.cuda.synchronize()
    assert (big[M * N:] == 777.0).all()
    assert np.array_equal(w.q.cpu().numpy(), pk["q"])
    yo = oracle.awq_linear(d["x"], pk, b)
    check_bf16_output(oracle.bf16_to_f32(bf16_np(y)), yo, oracle.bf16_to_f32(oracle.bf16_rn(yo)))


def test_awq_chained_launches_read_the_previous_output():
    """Three back-to-back launches on one stream, each reading the previous
    one's output as its activations (no host synchronisation between them).
    The launches may start before the previous one finishes, so this checks
    that every launch waits for its input: each output must match the oracle
    applied to the GPU's own previous output. The intermediate buffers start
    as NaN, so a launch that read them early would not pass."""
    M, K = 4, 512
    ws, pks = [], []
    for i in range(3):
        d = synth.awq_inputs(40 + i, M, K, K, w_std=0.05)
        ws.append(svdq.awq_pack_weight(torch.from_numpy(d["W"]).cuda()))
        pks.append(oracle.awq_pack_weight(d["W"]))
    x0 = synth.awq_inputs(39, M, K, K)["x"]
    ys = [torch.full((M, K), float("nan"), dtype=torch.bfloat16, device="cuda") for _ in range(3)]
    torch.cuda.synchronize()
    inp = bf16_dev(x0)
    for i in range(3):
        svdq.awq_w4a16_linear(inp, ws[i], out=ys[i])
        inp = ys[i]
    torch.cuda.synchronize()
    assert svdq.device_error() == 0
    prev = x0
    for i in range(3):
        got = bf16_np(ys[i])
        yo = oracle.awq_linear(prev, pks[i])
        check_bf16_output(oracle.bf16_to_f32(got), yo, oracle.bf16_to_f32(oracle.bf16_rn(yo)))
        prev = got


def test_awq_reads_weights_written_just_before():
    """The GEMV may be scheduled before the previous kernel in the stream
    finishes (dependent launch), so it must read none of its inputs early.
    Two cases, each with no host synchronisation between the writer and the
    GEMV: awq_pack_weight of a new weight into the buffers of an old one, and
    a device copy of pre-packed tensors into those buffers (as a checkpoint
    load would do). Each output must match the new weight."""
    c = synth.CONFIGS["c2_awq_gemv"]
    K, N = c["K"], c["N"]
    old = synth.awq_inputs(50, 2, K, N)
    new = synth.awq_inputs(51, 2, K, N, w_std=0.05)
    pk_new = oracle.awq_pack_weight(new["W"])
    yo = oracle.awq_linear(new["x"], pk_new)
    x = bf16_dev(new["x"])
    Wn = torch.from_numpy(new["W"]).cuda()

    w = svdq.awq_pack_weight(torch.from_numpy(old["W"]).cuda())
    torch.cuda.synchronize()
    svdq.awq_pack_weight(Wn, out=w)
    y = svdq.awq_w4a16_linear(x, w)
    torch.cuda.synchronize()
    assert svdq.device_error() == 0
    check_bf16_output(oracle.bf16_to_f32(bf16_np(y)), yo, oracle.bf16_to_f32(oracle.bf16_rn(yo)))

    src = svdq.awq_pack_weight(Wn)
    svdq.awq_pack_weight(torch.from_numpy(old["W"]).cuda(), out=w)
    torch.cuda.synchronize()
    w.q.copy_(src.q)
    w.scales.copy_(src.scales)
    w.zeros.copy_(src.zeros)
    y2 = svdq.awq_w4a16_linear(x, w)
    torch.cuda.synchronize()
    check_bf16_output(oracle.bf16_to_f32(bf16_np(y2)), yo, oracle.bf16_to_f32(oracle.bf16_rn(yo)))


@pytest.mark.parametrize("M", [1, 2, 3, 4])
def test_awq_gemv_outlier_activations(M):
    """Activations with 1% of channels scaled x30 (as in the svdq workloads):
    the GEMV kernel (up to four rows) applies the zero point through
    activation group sums, so large group sums must not cost accuracy."""
    K, N = 3072, 512
    d = synth.awq_inputs(52, M, K, N)
    x = oracle.bf16_to_f32(d["x"]).astype(np.float64)
    ch = np.random.default_rng(7).choice(K, K // 100, replace=False)
    x[:, ch] *= 30.0
    xb = synth.bf16_bits(x)
    pk = oracle.awq_pack_weight(d["W"])
    w = svdq.awq_pack_weight(torch.from_numpy(d["W"]).cuda())
    y = svdq.awq_w4a16_linear(bf16_dev(xb), w)
    torch.cuda.synchronize()
    assert svdq.device_error() == 0
    yo = oracle.awq_linear(xb, pk)
    check_bf16_output(oracle.bf16_to_f32(bf16_np(y)), yo, oracle.bf16_to_f32(oracle.bf16_rn(yo)))
