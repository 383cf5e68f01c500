"""Failure detection on the GPU without a fault: a bounded wait that runs out.

The fused GEMM splits some output tiles between two CTA pairs (stream-K): the
pair that owns a tile's first half waits, bounded, for the flag with which
the next pair publishes the partial sum of the second half. A test hook
(nf4_debug_flag_wait) keeps those flags from being raised -- a flag that
nothing sets -- and shortens that one wait to microseconds. The call must
then report NF4_ERR_TIMEOUT through the device status, leave the context
usable, and a following normal call must give the clean result bit for bit.
"""
import pytest
import torch

import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def q():
    import bit_nf4_quantized_05_b200 as mod
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    return mod


def layer(N, K, M=1024, r=16):
    w = workloads.LayerWorkload("t", N, K, M, r, 32.0, 0.02, True, 8080)
    return w, workloads.make_inputs(w)


@pytest.mark.parametrize("direction", ["forward", "backward"])
def test_split_tile_wait_runs_out_and_next_call_is_clean(q, direction):
    # 4 x 20 = 80 output tiles of 256 x 256 in the GEMM under test (h [1024, 5120] in the
    # forward, dX [1024, 5120] in the backward) over 74 resident pairs: the last tiles are split
    w, inp = layer(5120, 1024) if direction == "forward" else layer(1024, 5120)
    qw = q.nf4_quantize(inp["W0"].cuda(), double_quant=True)
    x, A, B, dY = (inp[k].cuda() for k in ("x", "A", "B", "dY"))

    def call():
        h, u = q.qlora_linear_fwd(qw, x, A, B, w.alpha)
        if direction == "forward":
            return h
        dX, _, _ = q.qlora_linear_bwd(qw, x, A, B, w.alpha, dY, u=u)
        return dX

    clean = call()
    torch.cuda.synchronize()
    assert q.device_status() == q.NF4_OK
    try:
        assert q.lib.nf4_debug_flag_wait(1, 20000) == q.NF4_OK
        bad = call()
        torch.cuda.synchronize()
        st = q.device_status()
    finally:
        assert q.lib.nf4_debug_flag_wait(0, 0) == q.NF4_OK
    assert st == q.NF4_ERR_TIMEOUT, q.status_string(st)
    assert q.device_status() == q.NF4_OK              # read once, then cleared
    # the tiles that gave up on their second halves' partial sums differ
    assert not torch.equal(bad, clean)
    again = call()
    torch.cuda.synchronize()
    assert q.device_status() == q.NF4_OK
    assert torch.equal(again, clean)
