"""Every output and workspace of the layer's entry points is handed over with
guard bands of a known byte pattern on both sides; after the calls the bands
must be untouched (no write outside the caller's buffers) and the results must
equal those of the same calls on freshly allocated buffers, bit for bit (the
kernels are deterministic: every sum has a fixed order)."""
import numpy as np
import pytest
import torch

import workloads

pytestmark = pytest.mark.gpu

GUARD = 256          # bytes on each side; keeps the 256-byte alignment of the workspace
PATTERN = 0xA5


@pytest.fixture(scope="module")
def q():
    import bit_nf4_quantized_05_b200 as mod
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    return mod


class Guarded:
    """A tensor of the given shape and dtype inside a byte buffer whose GUARD
    bytes before and after it hold PATTERN."""

    def __init__(self, shape, dtype, device="cuda"):
        numel = int(np.prod(shape)) if len(shape) else 1
        self.nbytes = numel * torch.empty((), dtype=dtype).element_size()
        self.buf = torch.full((self.nbytes + 2 * GUARD,), PATTERN, dtype=torch.uint8, device=device)
        self.t = self.buf[GUARD:GUARD + self.nbytes].view(dtype).view(shape)

    def intact(self) -> bool:
        return bool((self.buf[:GUARD] == PATTERN).all()) and \
            bool((self.buf[GUARD + self.nbytes:] == PATTERN).all())


def guarded_weight(q, n, k, dq, block):
    nb = n * k // block
    parts = {"codes": Guarded((n * k // 2,), torch.uint8), "absmax": Guarded((nb,), torch.float32),
             "q8": Guarded((nb,), torch.uint8), "cg": Guarded(((nb + 255) // 256,), torch.float32)}
    qw = q.QuantizedWeight(n, k, dq, parts["codes"].t, parts["absmax"].t,
                           parts["q8"].t if dq else None, parts["cg"].t if dq else None, block)
    return qw, parts


def all_intact(parts):
    bad = [name for name, g in parts.items() if not g.intact()]
    assert not bad, f"writes outside the buffers of {bad}"


CASES = [
    # (N, K, M, r, dq, block)  GEMM path with ragged tiles; decode path (M <= 16)
    (264, 640, 77, 16, True, 64),
    (264, 640, 5, 16, True, 64),
    (520, 1152, 300, 64, False, 128),
    (136, 1152, 16, 8, True, 128),
]


@pytest.mark.parametrize("N,K,M,r,dq,block", CASES)
def test_layer_writes_stay_in_their_buffers(q, N, K, M, r, dq, block):
    w = workloads.LayerWorkload("t", N, K, M, r, 16.0, 0.02, dq, 2024 + N + M)
    inp = workloads.make_inputs(w)
    W0, x, A, B, dY = (inp[k].cuda() for k in ("W0", "x", "A", "B", "dY"))
    qw, wparts = guarded_weight(q, N, K, dq, block)
    q.nf4_quantize(W0, double_quant=dq, out=qw)
    g = {"h": Guarded((M, N), torch.bfloat16), "u": Guarded((M, r), torch.float32),
         "ws_f": Guarded((q.fwd_workspace_bytes(M, N, K, r),), torch.uint8),
         "dX": Guarded((M, K), torch.bfloat16), "dA": Guarded((r, K), torch.bfloat16),
         "dB": Guarded((N, r), torch.bfloat16),
         "ws_b": Guarded((q.bwd_workspace_bytes(M, N, K, r),), torch.uint8)}
    q.qlora_linear_fwd(qw, x, A, B, 16.0, h=g["h"].t, u=g["u"].t, workspace=g["ws_f"].t)
    q.qlora_linear_bwd(qw, x, A, B, 16.0, dY, u=g["u"].t, workspace=g["ws_b"].t,
                       outs=(g["dX"].t, g["dA"].t, g["dB"].t))
    torch.cuda.synchronize()
    assert q.device_status() == q.NF4_OK
    all_intact(wparts)
    all_intact(g)
    # the same calls on fresh buffers
    ref = q.nf4_quantize(W0, double_quant=dq, block_size=block)
    assert torch.equal(ref.codes, qw.codes) and torch.equal(ref.absmax, qw.absmax)
    h, u = q.qlora_linear_fwd(ref, x, A, B, 16.0)
    dX, dA, dB = q.qlora_linear_bwd(ref, x, A, B, 16.0, dY, u=u)
    torch.cuda.synchronize()
    for name, t in (("h", h), ("u", u), ("dX", dX), ("dA", dA), ("dB", dB)):
        assert torch.equal(t, g[name].t), name


@pytest.mark.parametrize("M", [200, 9])
def test_dropout_multi_and_merge_writes_stay_in_their_buffers(q, M):
    N, K, r, p = 264, 640, 16, 0.1
    w = workloads.LayerWorkload("t", N, K, M, r, 32.0, 0.02, True, 77 + M)
    inp = workloads.make_inputs(w)
    W0, x, A, B, dY = (inp[k].cuda() for k in ("W0", "x", "A", "B", "dY"))
    qw = q.nf4_quantize(W0, double_quant=True)
    keep = q.pack_keep(torch.from_numpy(np.random.default_rng(M).random((M, K)) >= p).cuda())
    nbw = int(q.lib.qlora_bwd_dropout_workspace_bytes(M, N, K, r))
    g = {"h": Guarded((M, N), torch.bfloat16),
         "ws_f": Guarded((q.fwd_workspace_bytes(M, N, K, r),), torch.uint8),
         "dX": Guarded((M, K), torch.bfloat16), "dA": Guarded((r, K), torch.bfloat16),
         "dB": Guarded((N, r), torch.bfloat16), "ws_b": Guarded((nbw,), torch.uint8),
         "hm": Guarded((M, N), torch.bfloat16),
         "ws_m": Guarded((q.fwd_workspace_bytes(M, N, K, 2 * r),), torch.uint8),
         "merged": Guarded((N, K), torch.bfloat16)}
    _, u = q.qlora_linear_fwd_dropout(qw, x, A, B, 32.0, p, keep, h=g["h"].t, workspace=g["ws_f"].t)
    q.qlora_linear_bwd_dropout(qw, x, A, B, 32.0, p, keep, dY, u=u, workspace=g["ws_b"].t,
                               outs=(g["dX"].t, g["dA"].t, g["dB"].t))
    A2, B2 = torch.cat([A, A.flip(0)]), torch.cat([B, B.flip(1)], dim=1)
    idx = torch.from_numpy(np.random.default_rng(M + 1).integers(-1, 2, size=M).astype(np.int32)).cuda()
    q.qlora_multi_lora_fwd(qw, x, A2, B2, r, [32.0, 16.0], idx, h=g["hm"].t, workspace=g["ws_m"].t)
    q.qlora_merge(qw, A, B, 32.0, bf16=True, out=g["merged"].t)
    torch.cuda.synchronize()
    assert q.device_status() == q.NF4_OK
    all_intact(g)
    h, u2 = q.qlora_linear_fwd_dropout(qw, x, A, B, 32.0, p, keep)
    dX, dA, dB = q.qlora_linear_bwd_dropout(qw, x, A, B, 32.0, p, keep, dY, u=u2)
    hm = q.qlora_multi_lora_fwd(qw, x, A2, B2, r, [32.0, 16.0], idx)
    merged = q.qlora_merge(qw, A, B, 32.0, bf16=True)
    torch.cuda.synchronize()
    for name, t in (("h", h), ("dX", dX), ("dA", dA), ("dB", dB), ("hm", hm), ("merged", merged)):
        assert torch.equal(t, g[name].t), name
