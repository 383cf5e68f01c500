"""GPU parity of the quantiser's reciprocal fast path at block scales other
than 1 ("QLoRA Finetuner -- Juan Martos", section 2: each weight is divided by
its block's absmax and mapped to the nearest NF4 quantile).

The kernel codes an element from p = fl32(w * rcp(s)) (hardware reciprocal)
and falls back to the exact quotient fl32(w / s) only when p lies within 2^-21
of the decision threshold of its bucket, or when s is outside [2^-125, 2^125].
With s = 1 the reciprocal is exact and that guard decides nothing, so these
blocks use awkward, tiny and huge scales, and elements built so that
fl32(w / s) lands on each of the 15 thresholds and its fp32 neighbours
(inside the guard band), or a few ulps either side of the band's edge (where
the fast path decides alone). Codes, absmax, 8-bit scale codes and group
constants must equal the oracle's bit for bit, for fp32, bf16 and fp16
weights at blocks of 64 and 128.
"""
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu

GUARD = 2.0 ** -21


@pytest.fixture(scope="module")
def q():
    import bit_nf4_quantized_05_b200 as mod
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    return mod


def thresholds() -> np.ndarray:
    """The 15 exact level midpoints rounded toward -inf in fp32 (a value on a
    midpoint goes to the lower level). Input construction only."""
    lv = oracle.levels()
    out = []
    for i in range(15):
        m = (Fraction(float(lv[i])) + Fraction(float(lv[i + 1]))) / 2
        v = np.float32(float(m))
        if Fraction(float(v)) > m:
            v = np.nextafter(v, np.float32(-2))
        out.append(v)
    return np.array(out, dtype=np.float32)


T = thresholds()


def f32_step(v: np.float32, k: int) -> np.float32:
    """v moved by k fp32 ulps (no zero crossing for these values)."""
    b = np.array(v, dtype=np.float32).view(np.int32)
    b = b + (k if v > 0 else -k)
    return np.array(b, dtype=np.int32).view(np.float32)[()]


def targets_inside():
    return [f32_step(t, k) for t in T for k in range(-4, 5)]


def targets_edge():
    out = []
    for t in T:
        ulp = abs(float(f32_step(t, 1)) - float(t))
        g = int(np.ceil(GUARD / ulp))
        for k in (g - 2, g - 1, g, g + 1, g + 2, g + 4):
            out += [f32_step(t, k), f32_step(t, -k)]
    return out


def solve_fp32(v: np.float32, s: np.float32) -> np.float32:
    """An fp32 w with fl32(w / s) == v if one is within 8 ulps of fl32(v s),
    else the closest found; |w| <= s."""
    w0 = np.float32(v * s)
    best, bestd = w0, None
    for k in range(-8, 9):
        w = f32_step(w0, k) if w0 != 0 else w0
        if abs(w) > s:
            continue
        with np.errstate(all="ignore"):
            qv = np.float32(w) / s
        d = abs(float(qv) - float(v))
        if bestd is None or d < bestd:
            best, bestd = w, d
        if d == 0:
            break
    return np.float32(best)


def blocks_from(values, s, block, rng):
    """Blocks of `block` elements: +-s (the absmax) at a random position, the
    values in order, zero padding."""
    out = []
    per = block - 1
    for i in range(0, len(values), per):
        chunk = np.array(values[i:i + per], dtype=np.float32)
        b = np.zeros(block, dtype=np.float32)
        pos = int(rng.integers(0, block))
        rest = [j for j in range(block) if j != pos]
        b[rest[:chunk.size]] = chunk
        b[pos] = s if rng.random() < 0.5 else -s
        out.append(b)
    return out


def pad_to_matrix(blocks, block, rng, dtype=None):
    """Rows of 8 blocks, a multiple of 8 rows (the GPU path's shape rules); the
    padding blocks are random values of the weight's type."""
    blocks = list(blocks)
    while len(blocks) % 64:
        pad = torch.from_numpy(rng.normal(0, 0.02, block).astype(np.float32))
        if dtype is not None:
            pad = pad.to(dtype).float()
        blocks.append(pad.numpy())
    return np.concatenate(blocks).reshape(-1, 8 * block)


def fp32_scales(rng):
    special = [0.987654321, 1.2345678, 0.70710678, 1.0000001, 0.99999994, 3.3333333e-3,
               1.7e-3, 1234.5679, 987.6543, 3e-38, 1e-37, 2.3e-38, 1.17e-38, 4e37, 5e37, 3.4e38,
               1e-39, 6.02e23, 1.6e-19]
    rand = np.exp(rng.uniform(np.log(1e-3), np.log(1e3), 48))
    return [np.float32(v) for v in special] + [np.float32(v) for v in rand]


def quant_both(q, W, dq, block, dtype=None):
    Wt = torch.from_numpy(np.ascontiguousarray(W))
    if dtype is not None:
        Wt = Wt.to(dtype)
        ref = oracle.quantize(Wt.float().numpy().reshape(-1), block=block, dq=dq)
    else:
        ref = oracle.quantize(W.reshape(-1), block=block, dq=dq)
    qw = q.nf4_quantize(Wt.cuda(), double_quant=dq, block_size=block)
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


def guard_count(W, block):
    """Elements whose exact quotient fl32(w / s) lies within 2^-21 of a threshold."""
    B = W.reshape(-1, block).astype(np.float32)
    s = np.max(np.abs(B), axis=1, keepdims=True)
    with np.errstate(all="ignore"):
        p = np.where(s > 0, B / s, 0).astype(np.float32)
    d = np.min(np.abs(p.reshape(-1, 1).astype(np.float64) - T.astype(np.float64)), axis=1)
    return int(np.count_nonzero(d <= GUARD))


@pytest.mark.parametrize("block", [64, 128])
def test_fastpath_fp32_non_unit_scales(q, block):
    rng = np.random.default_rng(100 + block)
    inside, edge = targets_inside(), targets_edge()
    blocks = []
    for s in fp32_scales(rng):
        blocks += blocks_from([solve_fp32(v, s) for v in inside], s, block, rng)
        blocks += blocks_from([solve_fp32(v, s) for v in edge], s, block, rng)
    W = pad_to_matrix(blocks, block, rng)
    n_guard = guard_count(W, block)
    assert n_guard >= 3000, n_guard
    for dq in (True, False):
        ref, qw = quant_both(q, W, dq, block)
        assert_quant_equal(ref, qw)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("block", [64, 128])
def test_fastpath_16bit_non_unit_scales(q, dtype, block):
    """16-bit weights: s is a value of the type, the elements are the values of
    the type nearest to t_i s and their neighbours (a 16-bit grid reaches each
    threshold only to about 2^-9 relative, so a few land inside the guard band
    and the rest near it)."""
    rng = np.random.default_rng(200 + block + (0 if dtype == torch.bfloat16 else 7))
    lo, hi = (1e-30, 1e30) if dtype == torch.bfloat16 else (1e-3, 3e4)
    scales = torch.tensor(np.exp(rng.uniform(np.log(lo), np.log(hi), 160)), dtype=torch.float32).to(dtype)
    finfo = torch.finfo(dtype)
    blocks = []
    for s16 in scales:
        s = float(s16)
        vals = []
        for t in T:
            w = torch.tensor(float(t) * s, dtype=torch.float32).to(dtype)
            b = w.view(torch.int16).item()
            for k in range(-4, 5):
                c = torch.tensor(b + (k if float(w) > 0 else -k), dtype=torch.int16).view(dtype)
                if abs(float(c)) <= s and abs(float(c)) <= float(finfo.max):
                    vals.append(np.float32(float(c)))
        blocks += blocks_from(vals, np.float32(s), block, rng)
    W = pad_to_matrix(blocks, block, rng, dtype)
    W16 = torch.from_numpy(W).to(dtype)
    assert torch.equal(W16.float(), torch.from_numpy(W)), "inputs must be exact in the 16-bit type"
    assert guard_count(W, block) >= 1
    for dq in (True, False):
        ref, qw = quant_both(q, W, dq, block, dtype=dtype)
        assert_quant_equal(ref, qw)
