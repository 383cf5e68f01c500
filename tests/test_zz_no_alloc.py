"""The allocation-free forward (qlora_linear_fwd_noalloc) against the regular one.

Some callers cannot allocate device memory while they run: a process that
reserved its whole memory budget at start-up and forbids later allocations,
or code running inside a memory allocator's own callback, where calling
cudaMalloc would re-enter it. For them the library offers a forward that
takes no workspace and uses a fixed 4 MiB scratch array inside the library
instead. These tests call it through the C ABI, twice in a row on the same
inputs (the second call finds the first call's leftovers in the shared
scratch), and compare both results with the workspace forward, within the
tolerance the other layer tests use. The workspace forward may split a
tile's reduction between two CTA pairs (stream-K), so the two forwards add
the same fp32 terms in a different grouping and each rounds its own sum to
bf16: h may differ by one bf16 unit in the last place (at most 2^-7 of the
value) on top of that tolerance. This file is named so that pytest collects
it last."""
import numpy as np
import pytest
import torch

import workloads

pytestmark = pytest.mark.gpu
TOL = 2e-2


@pytest.fixture(scope="module")
def q():
    import bit_nf4_quantized_05_b200 as mod
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    return mod


def rel_err(got: torch.Tensor, ref: torch.Tensor, bf16_ulp: bool = False) -> float:
    """max |got - ref| / rms(ref); with bf16_ulp, one bf16 ulp of ref (2^-7 |ref|)
    is allowed per element first."""
    g = got.double().cpu().numpy()
    r = ref.double().cpu().numpy()
    d = np.abs(g - r)
    if bf16_ulp:
        d = d - 2.0 ** -7 * np.abs(r)
    return float(np.max(d) / max(np.sqrt(np.mean(r ** 2)), 1e-300))


@pytest.mark.parametrize("name", ["single_1024", "llama13b_attn_5120"])
def test_noalloc_forward_matches_workspace_forward(q, name):
    w = workloads.WORKLOADS[name]
    inp = workloads.make_inputs(w, with_dy=False)
    dev = torch.device("cuda")
    qw = q.nf4_quantize(inp["W0"].to(dev), double_quant=w.double_quant)
    x, A, B = (inp[k].to(dev) for k in ("x", "A", "B"))
    h_ref, u_ref = q.qlora_linear_fwd(qw, x, A, B, w.alpha)
    # outputs preallocated, so the calls below allocate nothing at all
    h = torch.empty_like(h_ref)
    u = torch.empty_like(u_ref)
    for call in range(2):
        h.fill_(float("nan"))
        u.fill_(float("nan"))
        q.qlora_linear_fwd_noalloc(qw, x, A, B, w.alpha, h=h, u=u)
        torch.cuda.synchronize()
        assert q.device_status() == q.NF4_OK
        assert torch.isfinite(h).all() and torch.isfinite(u).all()
        eh, eu = rel_err(h, h_ref, bf16_ulp=True), rel_err(u, u_ref)
        assert eh <= TOL and eu <= TOL, f"call {call}: h {eh:.3g}, u {eu:.3g} x rms"


def test_noalloc_rejects_batches_beyond_its_scratch(q):
    # r = 64 needs M * 2 * 64 bytes <= 4 MiB, i.e. at most 32768 tokens
    N, K, r, M = 64, 64, 64, 32769
    dev = torch.device("cuda")
    qw = q.nf4_quantize(torch.randn(N, K, device=dev) * 0.02, double_quant=False)
    x = torch.randn(M, K, device=dev).to(torch.bfloat16)
    A = torch.randn(r, K, device=dev).to(torch.bfloat16)
    B = torch.randn(N, r, device=dev).to(torch.bfloat16)
    with pytest.raises(q.NF4Error) as e:
        q.qlora_linear_fwd_noalloc(qw, x, A, B, 16.0)
    assert e.value.code == q.NF4_ERR_UNSUPPORTED_SHAPE
    # one token fewer fits
    h, _ = q.qlora_linear_fwd_noalloc(qw, x[: M - 1], A, B, 16.0)
    torch.cuda.synchronize()
    assert q.device_status() == q.NF4_OK and torch.isfinite(h).all()
