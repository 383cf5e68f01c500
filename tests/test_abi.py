"""The C-ABI library loads, exports every entry point the header declares, and
rejects bad arguments on the host (these paths make no CUDA call, so they run
without a GPU)."""
import ctypes
import os
import re

import pytest

from conftest import ROOT, build_library

HEADER = os.path.join(ROOT, "include", "qlora_nf4.h")


def declared_functions():
    src = open(HEADER).read()
    return re.findall(r"QLORA_API\s+[\w\s\*]+?\b(\w+)\s*\(", src)


@pytest.fixture(scope="module")
def q():
    build_library()
    import bit_nf4_quantized_05_b200 as mod
    return mod


def test_header_declares_the_layer_entry_points():
    names = declared_functions()
    for n in ["nf4_quantize", "nf4_dequantize", "qlora_linear_fwd", "qlora_linear_bwd",
              "qlora_fwd_workspace_bytes", "qlora_bwd_workspace_bytes", "nf4_device_status",
              "nf4_status_string"]:
        assert n in names


def test_library_exports_every_declared_symbol(q):
    lib = ctypes.CDLL(q.LIB_PATH)
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_status_strings(q):
    for code in range(8):
        s = q.status_string(code)
        assert s and s != "unknown status"
    assert q.status_string(99) == "unknown status"


def test_workspace_queries(q):
    a = q.fwd_workspace_bytes(16, 1024, 1024, 8)
    b = q.fwd_workspace_bytes(2048, 1024, 1024, 8)
    assert 256 <= a <= b and b >= 2048 * 8 * 2 and b % 256 == 0
    c = q.bwd_workspace_bytes(16, 1024, 1024, 8)
    d = q.bwd_workspace_bytes(2048, 5120, 5120, 16)
    # the backward keeps bf16 (alpha/r) u and (alpha/r) v, [M, r] each
    assert 256 <= c <= d and d >= 2 * 2048 * 16 * 2 and d % 256 == 0


FAKE = 0x10000  # aligned, never dereferenced: validation fails or M == 0 returns first


def weight(q, n=64, k=64, block=64, dq=0, codes=FAKE, absmax=FAKE, q8=FAKE, cg=FAKE):
    return q.NF4WeightStruct(n, k, block, dq, codes, absmax, q8, cg)


def call_fwd(q, w, M=4, r=8, alpha=16.0, x=FAKE, A=FAKE, B=FAKE, h=FAKE, u=None, ws=FAKE,
             wsb=1 << 30):
    return q.lib.qlora_linear_fwd(ctypes.byref(w), x, M, A, B, r, alpha, h, u, ws, wsb, None)


def test_quantize_argument_checks(q):
    L = q.lib
    assert L.nf4_quantize(FAKE, None, None) == q.NF4_ERR_INVALID_ARG
    assert L.nf4_quantize(FAKE, ctypes.byref(weight(q, block=32)), None) == q.NF4_ERR_INVALID_ARG
    assert L.nf4_quantize(FAKE, ctypes.byref(weight(q, dq=2)), None) == q.NF4_ERR_INVALID_ARG
    assert L.nf4_quantize(FAKE, ctypes.byref(weight(q, n=60)), None) == q.NF4_ERR_UNSUPPORTED_SHAPE
    assert L.nf4_quantize(FAKE, ctypes.byref(weight(q, k=96)), None) == q.NF4_ERR_UNSUPPORTED_SHAPE
    assert L.nf4_quantize(None, ctypes.byref(weight(q)), None) == q.NF4_ERR_INVALID_ARG
    assert L.nf4_quantize(FAKE + 4, ctypes.byref(weight(q)), None) == q.NF4_ERR_ALIGNMENT
    assert L.nf4_quantize(FAKE, ctypes.byref(weight(q, codes=FAKE + 8)), None) == q.NF4_ERR_ALIGNMENT
    assert L.nf4_quantize(FAKE, ctypes.byref(weight(q, dq=1, q8=None)), None) == q.NF4_ERR_INVALID_ARG
    assert L.nf4_dequantize(ctypes.byref(weight(q)), FAKE, 2, None) == q.NF4_ERR_INVALID_ARG
    assert L.nf4_dequantize(ctypes.byref(weight(q)), FAKE + 2, 1, None) == q.NF4_ERR_ALIGNMENT


def test_layer_argument_checks(q):
    w = weight(q)
    assert call_fwd(q, w, r=7) == q.NF4_ERR_UNSUPPORTED_SHAPE
    assert call_fwd(q, w, r=0) == q.NF4_ERR_UNSUPPORTED_SHAPE
    assert call_fwd(q, w, r=136) == q.NF4_ERR_UNSUPPORTED_SHAPE
    assert call_fwd(q, w, alpha=float("nan")) == q.NF4_ERR_INVALID_ARG
    assert call_fwd(q, w, alpha=float("inf")) == q.NF4_ERR_INVALID_ARG
    assert call_fwd(q, w, M=-1) == q.NF4_ERR_UNSUPPORTED_SHAPE
    assert call_fwd(q, w, A=None) == q.NF4_ERR_INVALID_ARG
    assert call_fwd(q, w, x=FAKE + 2) == q.NF4_ERR_ALIGNMENT
    assert call_fwd(q, w, h=None) == q.NF4_ERR_INVALID_ARG
    assert call_fwd(q, w, ws=None) == q.NF4_ERR_WORKSPACE
    assert call_fwd(q, w, wsb=16) == q.NF4_ERR_WORKSPACE
    assert call_fwd(q, w, ws=FAKE + 16) == q.NF4_ERR_ALIGNMENT
    assert call_fwd(q, w, M=0) == q.NF4_OK              # empty batch: nothing to launch
    bw = q.lib.qlora_linear_bwd
    args = lambda **kw: [ctypes.byref(kw.get("w", w)), FAKE, kw.get("M", 4), FAKE, FAKE,
                         kw.get("r", 8), 16.0, kw.get("dY", FAKE), None, None,
                         kw.get("dA", FAKE), kw.get("dB", FAKE), kw.get("ws", FAKE),
                         kw.get("wsb", 16), None]
    assert bw(*args(r=12)) == q.NF4_ERR_UNSUPPORTED_SHAPE
    assert bw(*args(dA=None)) == q.NF4_ERR_INVALID_ARG
    assert bw(*args(dY=None)) == q.NF4_ERR_INVALID_ARG
    assert bw(*args(dB=FAKE + 4)) == q.NF4_ERR_ALIGNMENT
    assert bw(*args(wsb=16)) == q.NF4_ERR_WORKSPACE


def test_python_binding_refuses_cpu_tensors(q):
    import torch
    W = torch.zeros(64, 64)
    with pytest.raises(ValueError):
        q.nf4_quantize(W)


def test_typed_quantize_and_merge_argument_checks(q):
    L = q.lib
    w = weight(q)
    assert L.nf4_quantize_typed(FAKE, 3, ctypes.byref(w), None) == q.NF4_ERR_INVALID_ARG
    assert L.nf4_quantize_typed(FAKE, -1, ctypes.byref(w), None) == q.NF4_ERR_INVALID_ARG
    assert L.nf4_quantize_typed(FAKE + 2, 1, ctypes.byref(w), None) == q.NF4_ERR_ALIGNMENT
    assert L.nf4_quantize_typed(None, 2, ctypes.byref(w), None) == q.NF4_ERR_INVALID_ARG
    merge = lambda **kw: L.qlora_merge(ctypes.byref(kw.get("w", w)), kw.get("A", FAKE), kw.get("B", FAKE),
                                       kw.get("r", 8), kw.get("alpha", 16.0), kw.get("out", FAKE),
                                       kw.get("bf16", 1), None)
    assert merge(r=12) == q.NF4_ERR_UNSUPPORTED_SHAPE
    assert merge(r=136) == q.NF4_ERR_UNSUPPORTED_SHAPE
    assert merge(alpha=float("nan")) == q.NF4_ERR_INVALID_ARG
    assert merge(bf16=2) == q.NF4_ERR_INVALID_ARG
    assert merge(out=None) == q.NF4_ERR_INVALID_ARG
    assert merge(A=FAKE + 8) == q.NF4_ERR_ALIGNMENT
    assert merge(w=weight(q, block=96)) == q.NF4_ERR_INVALID_ARG
    # 128-element blocks need K to be a multiple of 128
    assert merge(w=weight(q, block=128)) == q.NF4_ERR_UNSUPPORTED_SHAPE
    assert L.nf4_quantize(FAKE, ctypes.byref(weight(q, k=192, block=128)), None) == q.NF4_ERR_UNSUPPORTED_SHAPE


def test_multi_adapter_and_dropout_argument_checks(q):
    L = q.lib
    w = weight(q)
    al = (ctypes.c_float * 16)(*([16.0] * 16))

    def multi(**kw):
        return L.qlora_multi_lora_fwd(ctypes.byref(w), FAKE, kw.get("M", 4), FAKE, FAKE, kw.get("r", 8),
                                      kw.get("n", 2), kw.get("al", al), kw.get("idx", FAKE),
                                      kw.get("h", FAKE), kw.get("ws", FAKE), kw.get("wsb", 1 << 30), None)
    assert multi(n=0) == q.NF4_ERR_INVALID_ARG
    assert multi(n=17) == q.NF4_ERR_INVALID_ARG
    assert multi(al=None) == q.NF4_ERR_INVALID_ARG
    assert multi(r=4) == q.NF4_ERR_UNSUPPORTED_SHAPE           # r % 8
    assert multi(r=16, n=9) == q.NF4_ERR_UNSUPPORTED_SHAPE     # 144 stacked ranks > 128
    bad = (ctypes.c_float * 2)(16.0, float("inf"))
    assert multi(al=bad) == q.NF4_ERR_INVALID_ARG
    assert multi(idx=None) == q.NF4_ERR_INVALID_ARG
    assert multi(idx=FAKE + 4) == q.NF4_ERR_ALIGNMENT
    assert multi(M=0) == q.NF4_OK
    assert multi(wsb=16) == q.NF4_ERR_WORKSPACE

    def fwd_do(**kw):
        return L.qlora_linear_fwd_dropout(ctypes.byref(w), FAKE, kw.get("M", 4), FAKE, FAKE, 8, 16.0,
                                          kw.get("p", 0.05), kw.get("keep", FAKE), FAKE, None,
                                          FAKE, kw.get("wsb", 1 << 30), None)
    assert fwd_do(keep=None) == q.NF4_ERR_INVALID_ARG
    assert fwd_do(p=1.0) == q.NF4_ERR_INVALID_ARG
    assert fwd_do(p=-0.1) == q.NF4_ERR_INVALID_ARG
    assert fwd_do(p=float("nan")) == q.NF4_ERR_INVALID_ARG
    assert fwd_do(keep=FAKE + 1) == q.NF4_ERR_ALIGNMENT
    assert fwd_do(M=0, keep=None) == q.NF4_OK                 # an empty batch has an empty mask
    assert fwd_do(M=0, keep=None, p=1.0) == q.NF4_ERR_INVALID_ARG
    assert fwd_do(wsb=16) == q.NF4_ERR_WORKSPACE

    def bwd_do(**kw):
        return L.qlora_linear_bwd_dropout(ctypes.byref(w), FAKE, 4, FAKE, FAKE, 8, 16.0,
                                          kw.get("p", 0.05), kw.get("keep", FAKE), FAKE, None, None,
                                          FAKE, FAKE, FAKE, kw.get("wsb", 16), None)
    assert bwd_do(keep=None) == q.NF4_ERR_INVALID_ARG
    assert bwd_do(p=1.5) == q.NF4_ERR_INVALID_ARG
    # the dropout backward needs M * k * 4 more workspace bytes than the plain one
    plain = q.bwd_workspace_bytes(4, 64, 64, 8)
    assert bwd_do(wsb=plain) == q.NF4_ERR_WORKSPACE
    assert L.qlora_bwd_dropout_workspace_bytes(4, 64, 64, 8) >= plain + 4 * 64 * 4


def test_drawn_mask_dropout_argument_checks(q):
    L = q.lib
    w = weight(q)

    def fwd(**kw):
        return L.qlora_linear_fwd_dropout_philox(ctypes.byref(w), FAKE, kw.get("M", 4), FAKE, FAKE, 8,
                                                 16.0, kw.get("p", 0.05), 1, 2, FAKE, None, FAKE,
                                                 kw.get("wsb", 1 << 30), None)
    assert fwd(p=1.0) == q.NF4_ERR_INVALID_ARG
    assert fwd(p=-0.1) == q.NF4_ERR_INVALID_ARG
    assert fwd(p=float("nan")) == q.NF4_ERR_INVALID_ARG
    assert fwd(M=0) == q.NF4_OK
    assert fwd(wsb=16) == q.NF4_ERR_WORKSPACE

    def bwd(**kw):
        return L.qlora_linear_bwd_dropout_philox(ctypes.byref(w), FAKE, 4, FAKE, FAKE, 8, 16.0,
                                                 kw.get("p", 0.05), 1, 2, FAKE, None, None, FAKE, FAKE,
                                                 FAKE, kw.get("wsb", 16), None)
    assert bwd(p=1.5) == q.NF4_ERR_INVALID_ARG
    plain = q.bwd_workspace_bytes(4, 64, 64, 8)
    assert bwd(wsb=plain) == q.NF4_ERR_WORKSPACE

    # the fp32-gradient backward takes the plain backward's workspace
    def bwd32(**kw):
        return L.qlora_linear_bwd_f32grad(ctypes.byref(w), FAKE, 4, FAKE, FAKE, kw.get("r", 8), 16.0,
                                          FAKE, None, None, kw.get("dA", FAKE), FAKE, FAKE,
                                          kw.get("wsb", 16), None)
    assert bwd32(r=4) == q.NF4_ERR_UNSUPPORTED_SHAPE
    assert bwd32(dA=None) == q.NF4_ERR_INVALID_ARG
    assert bwd32(dA=FAKE + 4) == q.NF4_ERR_ALIGNMENT
    assert bwd32(wsb=16) == q.NF4_ERR_WORKSPACE


def test_debug_flag_wait_hook_argument_checks(q):
    L = q.lib
    assert L.nf4_debug_flag_wait(2, 0) == q.NF4_ERR_INVALID_ARG
    assert L.nf4_debug_flag_wait(0, -1) == q.NF4_ERR_INVALID_ARG


def test_last_cuda_error_is_a_string(q):
    s = q.lib.nf4_last_cuda_error()
    assert isinstance(s, bytes)
