"""The C-ABI library builds, loads and exports every symbol include/svdq.h
declares; host-side validation rejects bad arguments before touching a device.
No kernel is launched here (these tests run without a GPU)."""

import ctypes as C
import os
import re

import pytest

import bit_w4a4_quantized_nvfp4_b200 as svdq
from bit_w4a4_quantized_nvfp4_b200 import build as svdq_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "svdq.h")


@pytest.fixture(scope="module")
def lib():
    svdq_build.build()
    return svdq.load()


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(svdq_\w+|awq_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = _declared()
    for need in ("svdq_pack_weight", "svdq_quantize_act", "svdq_w4a4_linear", "awq_pack_weight",
                 "awq_w4a16_linear", "svdq_status_str"):
        assert need in names


def test_every_declared_symbol_is_exported(lib):
    for name in _declared():
        assert hasattr(lib, name), name
    assert set(_declared()) == set(svdq.SIGNATURES), "binding signatures match the header"


def test_status_strings(lib):
    for s in svdq.Status:
        assert lib.svdq_status_str(int(s))
    assert lib.svdq_status_str(99) == b"unknown status"


def test_scale_sizes(lib):
    assert lib.svdq_scale_bytes(0, 256, 1024) == 256 * 64
    assert lib.svdq_scale_bytes(0, 200, 1024) == 256 * 64   # rows padded to 128
    assert lib.svdq_scale_bytes(0, 300, 1024) == 384 * 64
    assert lib.svdq_scale_bytes(1, 200, 1024) == 200 * 16 * 2
    assert lib.svdq_scale_bytes(1, 200, 192) == 200 * 8 * 2  # INT4 row pitch: 3 groups padded to 8
    assert lib.svdq_scale_bytes(1, 7, 3072) == 7 * 48 * 2
    assert lib.svdq_scale_bytes(0, 8, 100) == 0             # K % 64 != 0
    assert lib.svdq_lr_up_elems(0, 9216, 32) == 9216 * 64
    assert lib.svdq_lr_up_elems(1, 9216, 32) == 9216 * 32


FAKE = 1 << 20  # never dereferenced: every call below fails validation first


def test_validation_rejects_before_any_device_access(lib):
    S = svdq.Status
    # bad precision / shapes / rank
    assert lib.svdq_pack_weight(7, 64, 8, 0, FAKE, FAKE, None, None, 1.0, FAKE, FAKE, FAKE, FAKE, None, None) == S.INVALID_ARG
    assert lib.svdq_pack_weight(0, 100, 8, 0, FAKE, FAKE, None, None, 1.0, FAKE, FAKE, FAKE, FAKE, None, None) == S.SHAPE
    assert lib.svdq_pack_weight(0, 64, 12, 0, FAKE, FAKE, None, None, 1.0, FAKE, FAKE, FAKE, FAKE, None, None) == S.SHAPE
    assert lib.svdq_pack_weight(0, 64, 8, 48, FAKE, FAKE, FAKE, FAKE, 1.0, FAKE, FAKE, FAKE, FAKE, FAKE, None) == S.SHAPE
    assert lib.svdq_pack_weight(0, 64, 8, 8, FAKE, FAKE, FAKE, FAKE, 1.0, FAKE, FAKE, FAKE, FAKE, FAKE, None) == S.SHAPE
    assert lib.svdq_pack_weight(0, 64, 8, 16, FAKE, FAKE, None, FAKE, 1.0, FAKE, FAKE, FAKE, FAKE, FAKE, None) == S.INVALID_ARG
    assert lib.svdq_pack_weight(0, 64, 8, 0, FAKE, FAKE, None, None, 0.0, FAKE, FAKE, FAKE, FAKE, None, None) == S.INVALID_ARG
    assert lib.svdq_pack_weight(0, 64, 8, 0, FAKE + 4, FAKE, None, None, 1.0, FAKE, FAKE, FAKE, FAKE, None, None) == S.ALIGN
    # quantize (the 7th argument is the packed weight's tensor scales {s_tw, s_tx})
    assert lib.svdq_quantize_act(0, -1, 64, 0, FAKE, FAKE, FAKE, None, FAKE, FAKE, None, None) == S.INVALID_ARG
    assert lib.svdq_quantize_act(0, 0, 64, 0, None, None, None, None, None, None, None, None) == S.OK  # M = 0 no-op
    assert lib.svdq_quantize_act(1, 4, 96, 0, FAKE, FAKE, None, None, FAKE, FAKE, None, None) == S.SHAPE
    assert lib.svdq_quantize_act(0, 4, 64, 16, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE + 8, None) == S.ALIGN
    # NVFP4 needs the tensor scales (s_tx is read from them); INT4 does not
    assert lib.svdq_quantize_act(0, 4, 64, 0, FAKE, FAKE, None, None, FAKE, FAKE, None, None) == S.INVALID_ARG
    assert lib.svdq_quantize_act(0, 4, 64, 0, FAKE, FAKE, FAKE + 4, None, FAKE, FAKE, None, None) == S.ALIGN
    # linear
    assert lib.svdq_w4a4_linear(0, 4, 64, 8, 0, FAKE, FAKE, None, FAKE, FAKE, FAKE, None, None, FAKE, 2, None) == S.INVALID_ARG
    assert lib.svdq_w4a4_linear(0, 4, 64, 8, 0, FAKE, FAKE, None, FAKE, FAKE, FAKE, None, None, FAKE, 9, None) == S.INVALID_ARG
    # the GELU output (fused GELU-MLP up-projection) is NVFP4 only
    assert lib.svdq_w4a4_linear(1, 4, 64, 8, 0, FAKE, FAKE, None, FAKE, FAKE, FAKE, None, None, FAKE, 3, None) == S.INVALID_ARG
    assert lib.svdq_w4a4_linear(0, 4, 64, 8, 0, FAKE, FAKE, None, FAKE, FAKE, FAKE, None, None, None, 0, None) == S.INVALID_ARG
    assert lib.svdq_w4a4_linear(0, 0, 64, 8, 0, None, None, None, None, None, None, None, None, None, 0, None) == S.OK
    assert lib.svdq_w4a4_linear(0, 4, 64, 8, 16, FAKE, FAKE, None, FAKE, FAKE, FAKE, FAKE, None, FAKE, 0, None) == S.INVALID_ARG
    assert lib.svdq_w4a4_linear(0, 4, 64, 8, 0, FAKE, FAKE, None, FAKE, FAKE, FAKE, None, FAKE + 1, FAKE, 0, None) == S.ALIGN
    # awq
    assert lib.awq_pack_weight(96, 8, FAKE, FAKE, FAKE, FAKE, None) == S.SHAPE
    assert lib.awq_pack_weight(64, 8, None, FAKE, FAKE, FAKE, None) == S.INVALID_ARG
    assert lib.awq_w4a16_linear(1, 64, 12, FAKE, FAKE, FAKE, FAKE, None, FAKE, None) == S.SHAPE
    assert lib.awq_w4a16_linear(0, 64, 8, None, None, None, None, None, None, None) == S.OK
    assert lib.awq_w4a16_linear(1, 64, 8, FAKE + 2, FAKE, FAKE, FAKE, None, FAKE, None) == S.ALIGN
    assert lib.svdq_probe_convert(None, 5, None, None, None, None) == S.INVALID_ARG


def test_awq_rejects_k_beyond_the_shared_memory_bound(lib):
    # the activations of a block of rows are held in shared memory: K <= 16384
    assert lib.awq_w4a16_linear(1, 16384 + 64, 8, FAKE, FAKE, FAKE, FAKE, None, FAKE, None) == svdq.Status.SHAPE


def test_binding_refuses_host_and_strided_tensors():
    # the binding passes device pointers only; a host or non-contiguous tensor
    # is refused before anything reaches the library
    import torch
    with pytest.raises(ValueError, match="CUDA"):
        svdq._ptr(torch.zeros(4))
    if torch.cuda.is_available():
        with pytest.raises(ValueError, match="contiguous"):
            svdq._ptr(torch.zeros(4, 4, device="cuda").t())


# ------------------------------------------------------------------ binding argument checks
# The C ABI sees bare pointers, so the binding checks every shape, dtype and
# device before a pointer reaches the library. These run on CPU tensors: a
# mismatch must raise ValueError naming the argument; a well-formed call gets
# as far as the device check ("expected a CUDA tensor") and no further.
import torch  # noqa: E402


def _bf16(*shape):
    return torch.zeros(shape, dtype=torch.bfloat16)


def _packed(prec=svdq.NVFP4, K=128, N=16, r=16):
    scales = torch.zeros(max(svdq.scale_bytes(prec, N, K), 16), dtype=torch.uint8)
    lr = _bf16(N, 2 * r if prec == svdq.NVFP4 else r) if r else None
    return svdq.PackedWeight(prec, K, N, r, torch.zeros((N, K // 2), dtype=torch.uint8), scales,
                             torch.ones(2), torch.ones(K), lr, 1.0)


def _act(prec=svdq.NVFP4, M=8, K=128, r=16):
    return svdq.QuantAct(prec, M, K, r, torch.zeros((M, K // 2), dtype=torch.uint8),
                         torch.zeros(max(svdq.scale_bytes(prec, M, K), 16), dtype=torch.uint8),
                         _bf16(M, r) if r else None)


def _raises(match, fn, *a, **kw):
    with pytest.raises(ValueError, match=match):
        fn(*a, **kw)


def test_binding_checks_quantize_act(lib):
    pw = _packed()
    L1 = _bf16(128, 16)
    _raises("CUDA", svdq.quantize_act, _bf16(8, 128), pw, L1)            # well formed
    _raises("x: expected", svdq.quantize_act, torch.zeros(8, 128), pw, L1)
    _raises("K = 64", svdq.quantize_act, _bf16(8, 64), pw, L1)
    _raises("L1: shape", svdq.quantize_act, _bf16(8, 128), pw, _bf16(128, 32))
    _raises("L1: dtype", svdq.quantize_act, _bf16(8, 128), pw, torch.zeros(128, 16))
    bad = _packed()
    bad.inv_lambda = torch.ones(64)
    _raises("pw.inv_lambda", svdq.quantize_act, _bf16(8, 128), bad, L1)
    bad = _packed()
    bad.tensor_scale = torch.ones(1)
    _raises("pw.tensor_scale", svdq.quantize_act, _bf16(8, 128), bad, L1)
    out = _act(M=8)
    out.codes = torch.zeros((8, 32), dtype=torch.uint8)
    _raises("out.codes", svdq.quantize_act, _bf16(8, 128), pw, L1, out=out)
    out = _act(M=8)
    out.scales = torch.zeros(16, dtype=torch.uint8)
    _raises("out.scales", svdq.quantize_act, _bf16(8, 128), pw, L1, out=out)
    _raises("another shape", svdq.quantize_act, _bf16(8, 128), pw, L1, out=_act(M=4))


def test_binding_checks_w4a4_linear(lib):
    pw, qa = _packed(), _act()
    _raises("CUDA", svdq.w4a4_linear, qa, pw)                            # well formed
    _raises("do not match", svdq.w4a4_linear, _act(K=256), pw)
    _raises("do not match", svdq.w4a4_linear, _act(prec=svdq.INT4), pw)
    _raises("do not match", svdq.w4a4_linear, _act(r=0), pw)
    _raises("bias: shape", svdq.w4a4_linear, qa, pw, _bf16(8))
    _raises("bias: dtype", svdq.w4a4_linear, qa, pw, torch.zeros(16))
    _raises("out: shape", svdq.w4a4_linear, qa, pw, out=_bf16(8, 8))
    _raises("out: dtype", svdq.w4a4_linear, qa, pw, out=torch.zeros(8, 16))
    _raises("out: shape", svdq.w4a4_linear, qa, pw, out_dtype="f32", out=torch.zeros(8, 8))
    bad = _packed()
    bad.codes = torch.zeros((16, 32), dtype=torch.uint8)
    _raises("pw.codes", svdq.w4a4_linear, qa, bad)
    bad = _packed()
    bad.lr_up = _bf16(16, 16)
    _raises("pw.lr_up", svdq.w4a4_linear, qa, bad)
    bad = _act()
    bad.P = _bf16(8, 8)
    _raises("qa.P", svdq.w4a4_linear, bad, pw)
    _raises("out_dtype", svdq.w4a4_linear, qa, pw, out_dtype="f16")


def test_binding_checks_pack_and_awq(lib):
    W = torch.zeros(128, 16)
    _raises("CUDA", svdq.pack_weight, "nvfp4", W, torch.ones(128), _bf16(128, 16), _bf16(16, 16))
    _raises("W: expected", svdq.pack_weight, "nvfp4", W.double(), torch.ones(128), None, None)
    _raises("lambda: shape", svdq.pack_weight, "nvfp4", W, torch.ones(64), None, None)
    _raises("L2: shape", svdq.pack_weight, "nvfp4", W, torch.ones(128), _bf16(128, 16), _bf16(16, 8))
    _raises("precision", svdq.pack_weight, 5, W, torch.ones(128), None, None)
    aw = svdq.AwqWeight(128, 16, torch.zeros((16, 64), dtype=torch.uint8), _bf16(16, 2), _bf16(16, 2))
    _raises("CUDA", svdq.awq_w4a16_linear, _bf16(1, 128), aw)            # well formed
    _raises("K = 64", svdq.awq_w4a16_linear, _bf16(1, 64), aw)
    _raises("x: expected", svdq.awq_w4a16_linear, torch.zeros(1, 128), aw)
    _raises("bias: shape", svdq.awq_w4a16_linear, _bf16(1, 128), aw, _bf16(8))
    _raises("out: shape", svdq.awq_w4a16_linear, _bf16(2, 128), aw, out=_bf16(1, 16))
    bad = svdq.AwqWeight(128, 16, torch.zeros((16, 64), dtype=torch.uint8), _bf16(16, 1), _bf16(16, 2))
    _raises("w.scales", svdq.awq_w4a16_linear, _bf16(1, 128), bad)
    _raises("W: expected", svdq.awq_pack_weight, torch.zeros(128, 16, dtype=torch.float64))


def test_qkv_entry_validation(lib):
    S = svdq.Status
    f = lib.svdq_w4a4_linear_qkv
    # (M, K, heads, r, x_codes, x_scales, P, w_codes, w_scales, ts, lr_up, bias, nq, nk, eps, rope, y, stream)
    ok = [4, 64, 1, 0, FAKE, FAKE, None, FAKE, FAKE, FAKE, None, None, FAKE, FAKE, 1e-6, FAKE, FAKE, None]

    def call(**kw):
        args = list(ok)
        names = ["M", "K", "heads", "r", "xc", "xs", "P", "wc", "ws", "ts", "lr", "b", "nq", "nk", "eps", "rope",
                 "y", "s"]
        for k, v in kw.items():
            args[names.index(k)] = v
        return f(*args)

    assert call(heads=0) == S.INVALID_ARG
    assert call(K=96) == S.SHAPE
    assert call(eps=-1.0) == S.INVALID_ARG
    assert call(nq=None) == S.INVALID_ARG
    assert call(rope=None) == S.INVALID_ARG
    assert call(r=16) == S.INVALID_ARG            # r > 0 needs P and lr_up
    assert call(rope=FAKE + 4) == S.ALIGN
    assert call(M=0, xc=None, xs=None, wc=None, ws=None, ts=None, nq=None, nk=None, rope=None, y=None) == S.OK


def test_rope_pack_entry_validation(lib):
    S = svdq.Status
    f = lib.svdq_rope_pack
    assert lib.svdq_rope_packed_bytes(0) == 0
    assert lib.svdq_rope_packed_bytes(1) == 16384
    assert lib.svdq_rope_packed_bytes(64) == 2 * 16384
    assert lib.svdq_rope_packed_bytes(65) == 3 * 16384
    assert lib.svdq_rope_packed_bytes(-1) == 0
    far = FAKE + (1 << 24)
    assert f(-1, FAKE, FAKE + 65536, far, None) == S.INVALID_ARG
    assert f(0, None, None, None, None) == S.OK
    assert f(4, None, FAKE + 65536, far, None) == S.INVALID_ARG
    assert f(4, FAKE + 8, FAKE + 65536, far, None) == S.ALIGN
    assert f(4, FAKE, FAKE + 65536, FAKE + 512, None) == S.INVALID_ARG   # rope overlaps cos


def test_binding_checks_qkv(lib):
    pw, qa = _packed(N=384), _act()
    nq, nk = _bf16(128), _bf16(128)
    rope = svdq.RopeTable(8, torch.zeros(4096))
    _raises("CUDA", svdq.w4a4_linear_qkv, qa, pw, 1, nq, nk, 1e-6, rope)   # well formed
    _raises("3 \\* heads", svdq.w4a4_linear_qkv, qa, pw, 2, nq, nk, 1e-6, rope)
    _raises("norm_q: shape", svdq.w4a4_linear_qkv, qa, pw, 1, _bf16(64), nk, 1e-6, rope)
    _raises("rope: expected", svdq.w4a4_linear_qkv, qa, pw, 1, nq, nk, 1e-6, svdq.RopeTable(9, torch.zeros(4096)))
    _raises("rope.data: shape", svdq.w4a4_linear_qkv, qa, pw, 1, nq, nk, 1e-6, svdq.RopeTable(8, torch.zeros(64)))
    _raises("NVFP4 only", svdq.w4a4_linear_qkv, _act(prec=svdq.INT4), _packed(prec=svdq.INT4, N=384), 1, nq, nk,
            1e-6, rope)
    _raises("cos: shape", svdq.pack_rope, torch.zeros(8, 32), torch.zeros(8, 64))
    _raises("sin: dtype", svdq.pack_rope, torch.zeros(8, 64), torch.zeros(8, 64, dtype=torch.float64))
