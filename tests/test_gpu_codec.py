"""GPU parity of nf4_quantize / nf4_dequantize against the CPU oracle:
bit-exact codes, fp32 absmax, 8-bit double-quant codes and group constants,
and bit-exact dequantised values (fp32 and the bf16 matmul operand)."""
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def q():
    import bit_nf4_quantized_05_b200 as mod
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    return mod


def quant_both(q, W: np.ndarray, dq: bool, block: int = 64):
    ref = oracle.quantize(W.reshape(-1), block=block, dq=dq)
    qw = q.nf4_quantize(torch.from_numpy(np.ascontiguousarray(W)).cuda(), double_quant=dq, block_size=block)
    torch.cuda.synchronize()
    assert q.device_status() == q.NF4_OK
    return ref, qw


def assert_quant_equal(ref, qw):
    assert np.array_equal(qw.codes.cpu().numpy(), ref.codes), "NF4 codes differ"
    assert np.array_equal(qw.absmax.cpu().numpy().view(np.uint32), ref.absmax.view(np.uint32)), \
        "absmax differs"
    if ref.dq:
        nb = ref.absmax.size
        assert np.array_equal(qw.absmax_q8.cpu().numpy()[:nb], ref.q8), "q8 differs"
        assert np.array_equal(qw.absmax_c.cpu().numpy()[:ref.cg.size].view(np.uint32),
                              ref.cg.view(np.uint32)), "group constants differ"


def assert_dequant_equal(q, ref, qw):
    wt = oracle.dequantize(ref)
    g32 = q.nf4_dequantize(qw, bf16=False).cpu().numpy().reshape(-1)
    assert np.array_equal(g32.view(np.uint32), wt.view(np.uint32)), "fp32 dequant differs"
    g16 = q.nf4_dequantize(qw, bf16=True).cpu().view(torch.int16).numpy().view(np.uint16).reshape(-1)
    assert np.array_equal(g16, oracle.f32_to_bf16(wt)), "bf16 dequant differs"


@pytest.mark.parametrize("shape,dq", [((64, 64), False), ((8, 128), True), ((24, 832), True),
                                      ((200, 640), False), ((136, 1024), True)])
def test_quantize_random_shapes(q, shape, dq):
    rng = np.random.default_rng(shape[0] * 7 + shape[1])
    W = rng.normal(0, 0.02, size=shape).astype(np.float32)
    W *= rng.uniform(0.2, 5.0, size=(shape[0], 1)).astype(np.float32)
    ref, qw = quant_both(q, W, dq)
    assert_quant_equal(ref, qw)
    assert_dequant_equal(q, ref, qw)


def test_quantize_midpoints_and_special_blocks(q):
    lv = oracle.levels()
    mids = [(Fraction(float(lv[i])) + Fraction(float(lv[i + 1]))) / 2 for i in range(15)]
    vals = []
    for m in mids:
        v = np.float32(float(m))
        vals += [v, np.nextafter(v, np.float32(2)), np.nextafter(v, np.float32(-2))]
    vals = np.array(vals, dtype=np.float32)
    blocks = []
    for i in range(0, vals.size, 63):             # unit absmax: w' == w exactly
        b = np.zeros(64, dtype=np.float32)
        b[0] = 1.0
        chunk = vals[i:i + 63]
        b[1:1 + chunk.size] = chunk
        blocks.append(b)
    blocks.append(np.zeros(64, dtype=np.float32))          # all-zero block
    b = np.zeros(64, dtype=np.float32); b[7] = -3.5; blocks.append(b)   # single negative max
    b = np.full(64, 1e-38, dtype=np.float32); blocks.append(b)          # tiny values
    b = (np.float32(0.123) * lv[np.arange(64) % 16]).astype(np.float32); blocks.append(b)
    while len(blocks) % 8:
        blocks.append(np.random.default_rng(len(blocks)).normal(size=64).astype(np.float32))
    W = np.concatenate(blocks).reshape(8, -1)
    for dq in (False, True):
        ref, qw = quant_both(q, W, dq)
        assert_quant_equal(ref, qw)
        assert_dequant_equal(q, ref, qw)


def test_quantize_dense_fp32_sweep(q):
    """Every 97th fp32 bit pattern in [0, 1] and its negative, against a unit
    absmax (so w' == w). Together with the midpoint test (every step of the
    monotone code function and its fp32 neighbours) this leaves no room for a
    different mapping."""
    one = np.float32(1.0).view(np.uint32)
    pos = np.arange(0, int(one), 97, dtype=np.uint32).view(np.float32)
    vals = np.concatenate([pos, -pos])
    pad = (-vals.size) % 63
    vals = np.concatenate([vals, np.zeros(pad, dtype=np.float32)]).reshape(-1, 63)
    W = np.concatenate([np.ones((vals.shape[0], 1), dtype=np.float32), vals], axis=1)
    blocks = W.shape[0]
    W = W[: blocks - blocks % 64].reshape(-1, 64 * 8)   # 8 blocks per row, rows % 8 == 0
    ref, qw = quant_both(q, W, False)
    assert np.array_equal(qw.codes.cpu().numpy(), ref.codes)


def test_quantize_outlier_workload_full_size(q):
    w = workloads.WORKLOADS["decode_mlp_up_13824x5120"]
    W = workloads.make_weight(w).numpy()
    ref, qw = quant_both(q, W, True)
    assert_quant_equal(ref, qw)


@pytest.mark.slow
def test_quantize_70b_mlp_full_size(q):
    w = workloads.WORKLOADS["llama2_70b_mlp_28672x8192"]
    W = workloads.make_weight(w).numpy()
    ref, qw = quant_both(q, W, True)
    assert_quant_equal(ref, qw)


def test_nonfinite_weight_sets_status(q):
    W = torch.randn(64, 128, device="cuda")
    W[3, 17] = float("nan")
    q.nf4_quantize(W, double_quant=True)
    assert q.device_status() == q.NF4_ERR_NONFINITE
    assert q.device_status() == q.NF4_OK          # the status word is cleared once read
    W[3, 17] = float("inf")
    q.nf4_quantize(W, double_quant=False)
    assert q.device_status() == q.NF4_ERR_NONFINITE


# ------------------------------------------------------------ 16-bit input --
def quant_16(q, W16: torch.Tensor, dq: bool, block: int = 64):
    """GPU quantisation of a 16-bit weight and the oracle's of its exact fp32 image."""
    ref = oracle.quantize(W16.float().numpy().reshape(-1), block=block, dq=dq)
    qw = q.nf4_quantize(W16.contiguous().cuda(), double_quant=dq, block_size=block)
    torch.cuda.synchronize()
    assert q.device_status() == q.NF4_OK
    return ref, qw


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("shape,dq", [((64, 64), False), ((24, 832), True), ((136, 1280), True),
                                      ((1000, 640), False)])
def test_quantize_16bit_input(q, dtype, shape, dq):
    rng = np.random.default_rng(shape[0] * 7 + shape[1])
    W = rng.normal(0, 0.02, size=shape).astype(np.float32)
    W *= rng.uniform(0.2, 5.0, size=(shape[0], 1)).astype(np.float32)
    ref, qw = quant_16(q, torch.from_numpy(W).to(dtype), dq)
    assert_quant_equal(ref, qw)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
def test_quantize_16bit_special_blocks(q, dtype):
    """Zero blocks, subnormals and the largest finite values of the type."""
    info = torch.finfo(dtype)
    rows = []
    rows.append(torch.zeros(64))
    rows.append(torch.full((64,), float(info.tiny)))                     # smallest normal
    rows.append(torch.full((64,), float(info.tiny) / 4))                 # subnormal
    # the largest finite value and smaller multiples of it (every one finite in the type)
    rows.append(torch.tensor([(-1.0) ** j * float(info.max) * (1.0 - j / 64.0) for j in range(64)]))
    rows.append(torch.tensor([(-1.0) ** i * 0.5 ** (i % 20) for i in range(64)]))
    while len(rows) % 8:
        rows.append(torch.from_numpy(np.random.default_rng(len(rows)).normal(size=64).astype(np.float32)))
    W = torch.stack(rows).reshape(8, -1).to(dtype)
    for dq in (False, True):
        ref, qw = quant_16(q, W, dq)
        assert_quant_equal(ref, qw)


def test_quantize_bf16_outlier_workload_full_size(q):
    w = workloads.WORKLOADS["decode_mlp_up_13824x5120"]
    W = workloads.make_weight(w).to(torch.bfloat16)
    ref, qw = quant_16(q, W, True)
    assert_quant_equal(ref, qw)
