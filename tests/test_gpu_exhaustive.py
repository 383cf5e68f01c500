"""Every fp32 value in [-1, 1] through the GPU quantiser against the oracle's
nearest-level rule ("QLoRA Finetuner -- Juan Martos", section 2: nearest of
the 16 NF4 quantiles after normalisation by the block absmax).

Each 64-element block holds 1.0 and 63 consecutive fp32 values, so its absmax
is 1 and every value is its own normalised value. The GPU codes of all
2.13e9 values, in value order, must be a monotone step function; at each step
the values on both sides, and the two ends of the range, are checked against
the oracle, whose own nearest-level function is monotone (pinned on the CPU).
Between two GPU steps the oracle then starts and ends on the GPU's code and,
being monotone, keeps it, so the two agree on every value of the range
without running the oracle 2e9 times."""
import numpy as np
import pytest
import torch

import oracle

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

SLAB_BLOCKS = 1 << 22              # 64-element blocks per quantiser call (1 GiB of fp32)
ROW = 8192                         # the weight is viewed as [blocks * 64 / ROW, ROW]


@pytest.fixture(scope="module")
def q():
    import bit_nf4_quantized_05_b200 as mod
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    return mod


def codes_of_range(q, lo_bits: int, hi_bits: int):
    """GPU codes of the fp32 values whose int32 bit patterns are lo_bits..hi_bits
    (inclusive), in bit-pattern order; yields (first bit pattern, codes uint8)."""
    per = 63 * SLAB_BLOCKS
    start = lo_bits
    while start <= hi_bits:
        count = min(per, hi_bits - start + 1)
        bits = torch.arange(start, start + count, dtype=torch.int32, device="cuda")
        body = torch.zeros(SLAB_BLOCKS * 63, dtype=torch.float32, device="cuda")
        body[:count] = bits.view(torch.float32)
        W = torch.empty(SLAB_BLOCKS, 64, dtype=torch.float32, device="cuda")
        W[:, 0] = 1.0
        W[:, 1:] = body.view(SLAB_BLOCKS, 63)
        qw = q.nf4_quantize(W.view(-1, ROW), double_quant=False)
        torch.cuda.synchronize()
        assert q.device_status() == q.NF4_OK
        assert bool((qw.absmax == 1.0).all())
        b = qw.codes.view(SLAB_BLOCKS, 32)
        c = torch.stack((b >> 4, b & 15), dim=2).view(SLAB_BLOCKS, 64)
        assert bool((c[:, 0] == 15).all())                 # the unit maximum
        yield start, c[:, 1:].reshape(-1)[:count].clone()
        del bits, W, body, qw, b, c
        start += count


def steps(q, lo_bits, hi_bits, increasing: bool):
    """(bit pattern before, bit pattern after, code before, code after) at every
    change of code over the range, checking monotonicity on the way."""
    out = []
    prev_code = prev_bits = None
    for start, c in codes_of_range(q, lo_bits, hi_bits):
        ci = c.to(torch.int16)
        if prev_code is not None and int(ci[0]) != prev_code:
            out.append((prev_bits, start, prev_code, int(ci[0])))
        d = ci[1:] - ci[:-1]
        assert bool((d >= 0).all() if increasing else (d <= 0).all()), "codes are not monotone"
        idx = torch.nonzero(d).view(-1)
        lo, hi = ci[idx].tolist(), ci[idx + 1].tolist()
        for i, cb, ca in zip(idx.tolist(), lo, hi):
            out.append((start + i, start + i + 1, cb, ca))
        prev_code, prev_bits = int(ci[-1]), start + c.numel() - 1
    return out


def f32(bits: int) -> np.float32:
    return np.array([bits], dtype=np.int64).astype(np.int32).view(np.float32)[0]


def test_every_fp32_in_unit_interval(q):
    pos = steps(q, 0, 0x3F800000, increasing=True)                       # +0 .. 1
    neg = steps(q, -0x80000000, -0x80000000 + 0x3F800000, increasing=False)  # -0 .. -1
    # 8 steps from code 7 up to 15, 7 from 7 down to 0, one level at a time
    assert len(pos) == 8 and len(neg) == 7
    for before, after, cb, ca in pos + neg:
        assert abs(ca - cb) == 1
        assert oracle.nearest_level(f32(before)) == cb
        assert oracle.nearest_level(f32(after)) == ca
    # the ends of both ranges
    assert oracle.nearest_level(np.float32(0.0)) == 7 and oracle.nearest_level(np.float32(-0.0)) == 7
    assert oracle.nearest_level(np.float32(1.0)) == 15 and oracle.nearest_level(np.float32(-1.0)) == 0
    assert sorted(c for _, _, c, _ in pos) == list(range(7, 15))
    assert sorted(c for _, _, c, _ in neg) == list(range(1, 8))
