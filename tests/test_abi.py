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
    # quantize
    assert lib.svdq_quantize_act(0, -1, 64, 0, FAKE, FAKE, 1.0, None, FAKE, FAKE, None, None) == S.INVALID_ARG
    assert lib.svdq_quantize_act(0, 0, 64, 0, None, None, 1.0, None, None, None, None, None) == S.OK  # M = 0 no-op
    assert lib.svdq_quantize_act(1, 4, 96, 0, FAKE, FAKE, 1.0, None, FAKE, FAKE, None, None) == S.SHAPE
    assert lib.svdq_quantize_act(0, 4, 64, 16, FAKE, FAKE, 1.0, FAKE, FAKE, FAKE, FAKE + 8, None) == S.ALIGN
    # linear
    assert lib.svdq_w4a4_linear(0, 4, 64, 8, 0, FAKE, FAKE, None, FAKE, FAKE, FAKE, None, None, FAKE, 2, None) == S.INVALID_ARG
    assert lib.svdq_w4a4_linear(0, 4, 64, 8, 0, FAKE, FAKE, None, FAKE, FAKE, FAKE, None, None, FAKE, 9, None) == S.INVALID_ARG
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
