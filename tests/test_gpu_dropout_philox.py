"""GPU parity of LoRA dropout with the mask drawn inside the kernels
("QLoRA Finetuner -- Juan Martos", section 1: h = W0 x + (alpha/r) B(A(dropout
x)); "QLoRA explained", the recipe's lora_dropout = 0.05).

The kernels draw each element's keep bit from Philox4x32-10 at (seed, offset)
and regenerate it in the backward. The oracle draws the same mask on the CPU
(oracle.dropout_keep_mask, pinned to the generator's published known-answer
vectors). Two checks per case:
  * the drawn-mask entry points equal, bit for bit, the keep-mask entry points
    given the oracle's mask: the kernels' mask is exactly the oracle's;
  * the results are within the layer's bar of the oracle's fp64 layer with
    that mask.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads

pytestmark = pytest.mark.gpu
TOL = 2e-2


@pytest.fixture(scope="module")
def q():
    import bit_nf4_quantized_05_b200 as mod
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    return mod


def bits(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def to_f64(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def rel_err(got, ref, ulp_allowance=False):
    rms = max(np.sqrt(np.mean(ref ** 2)), 1e-300)
    if not ulp_allowance:
        return float(np.max(np.abs(got - ref)) / rms)
    return float(np.max(np.abs(got - ref) - 2.0 ** -8 * np.abs(ref)) / rms)


def oracle_weight(qw):
    nb = qw.n * qw.k // qw.block_size
    return oracle.Quantized(qw.codes.cpu().numpy(), qw.absmax.cpu().numpy()[:nb],
                            qw.absmax_q8.cpu().numpy()[:nb] if qw.double_quant else None,
                            qw.absmax_c.cpu().numpy()[: (nb + 255) // 256] if qw.double_quant else None,
                            qw.block_size, qw.double_quant, 256, qw.n * qw.k)


def both_paths(q, qw, inp, alpha, p, seed, offset):
    """(drawn-mask results, keep-mask results with the oracle's mask, that mask)."""
    M, K = inp["x"].shape
    x, A, B, dY = (inp[k].cuda() for k in ("x", "A", "B", "dY"))
    h1, u1 = q.qlora_linear_fwd_dropout_philox(qw, x, A, B, alpha, p, seed, offset)
    g1 = q.qlora_linear_bwd_dropout_philox(qw, x, A, B, alpha, p, seed, offset, dY, u=u1)
    kb = oracle.dropout_keep_mask(M, K, p, seed, offset)
    keep = torch.from_numpy(kb).cuda()
    h2, u2 = q.qlora_linear_fwd_dropout(qw, x, A, B, alpha, p, keep)
    g2 = q.qlora_linear_bwd_dropout(qw, x, A, B, alpha, p, keep, dY, u=u2)
    torch.cuda.synchronize()
    assert q.device_status() == q.NF4_OK
    return (h1, u1) + tuple(g1), (h2, u2) + tuple(g2), kb


SHAPES = [
    # (N, K, M, r, p, dq, seed, offset)  GEMM path with ragged tiles, and the decode path (M <= 16)
    (384, 512, 300, 16, 0.05, True, 1, 0),
    (520, 640, 77, 64, 0.3, False, 0xDEADBEEFCAFEF00D, 12345678901),
    (264, 512, 12, 16, 0.1, True, 7, 2 ** 40 + 3),
    (256, 1088, 16, 8, 0.5, True, 99, 1),
]


@pytest.mark.parametrize("N,K,M,r,p,dq,seed,offset", SHAPES)
def test_drawn_mask_equals_oracle_mask_and_layer(q, N, K, M, r, p, dq, seed, offset):
    w = workloads.LayerWorkload("t", N, K, M, r, 32.0, 0.02, dq, 555 + N + M)
    inp = workloads.make_inputs(w)
    qw = q.nf4_quantize(inp["W0"].cuda(), double_quant=dq)
    drawn, given, kb = both_paths(q, qw, inp, w.alpha, p, seed, offset)
    for name, a, b in zip(("h", "u", "dX", "dA", "dB"), drawn, given):
        assert torch.equal(a, b), f"{name}: the drawn mask differs from the oracle's"
    ow = oracle_weight(qw)
    xb, Ab, Bb = bits(inp["x"]), bits(inp["A"]), bits(inp["B"])
    h_ref, u_ref = oracle.qlora_fwd_rows_dropout(ow, N, K, xb, Ab, Bb, r, w.alpha, p, kb)
    g_ref = oracle.qlora_bwd_dropout(ow, N, K, xb, Ab, Bb, r, w.alpha, p, kb, bits(inp["dY"]))
    errs = {}
    for name, g, rf in zip(("h", "u", "dX", "dA", "dB"), drawn, (h_ref, u_ref) + tuple(g_ref)):
        errs[name] = rel_err(to_f64(g), np.asarray(rf), M < 16)
    assert all(v <= TOL for v in errs.values()), errs


def test_new_offset_draws_a_new_mask(q):
    N, K, M, r, p = 256, 512, 64, 16, 0.3
    w = workloads.LayerWorkload("t", N, K, M, r, 16.0, 0.02, True, 4444)
    inp = workloads.make_inputs(w)
    qw = q.nf4_quantize(inp["W0"].cuda(), double_quant=True)
    x, A, B = (inp[k].cuda() for k in ("x", "A", "B"))
    _, u0 = q.qlora_linear_fwd_dropout_philox(qw, x, A, B, w.alpha, p, 5, 0)
    _, u0b = q.qlora_linear_fwd_dropout_philox(qw, x, A, B, w.alpha, p, 5, 0)
    _, u1 = q.qlora_linear_fwd_dropout_philox(qw, x, A, B, w.alpha, p, 5, 1)
    _, u2 = q.qlora_linear_fwd_dropout_philox(qw, x, A, B, w.alpha, p, 6, 0)
    torch.cuda.synchronize()
    assert torch.equal(u0, u0b)                      # same (seed, offset): same mask
    assert not torch.equal(u0, u1) and not torch.equal(u0, u2)


def test_p_zero_keeps_everything(q):
    N, K, M, r = 384, 512, 200, 16
    w = workloads.LayerWorkload("t", N, K, M, r, 32.0, 0.02, True, 999)
    inp = workloads.make_inputs(w)
    qw = q.nf4_quantize(inp["W0"].cuda(), double_quant=True)
    x, A, B = (inp[k].cuda() for k in ("x", "A", "B"))
    h1, u1 = q.qlora_linear_fwd_dropout_philox(qw, x, A, B, w.alpha, 0.0, 123, 0)
    h2, u2 = q.qlora_linear_fwd(qw, x, A, B, w.alpha)
    torch.cuda.synchronize()
    assert torch.equal(h1, h2) and torch.equal(u1, u2)


def test_drawn_mask_full_size_attention_projection(q):
    """The LLaMA-13B-like projection at p = 0.05: bit for bit the keep-mask entry
    points with the oracle's drawn mask, and sampled rows of h and dX and all of
    dA and dB against the oracle."""
    wl = workloads.WORKLOADS["llama13b_attn_5120"]
    N, K, M, r, p = wl.N, wl.K, wl.M, wl.r, 0.05
    inp = workloads.make_inputs(wl)
    qw = q.nf4_quantize(inp["W0"].cuda(), double_quant=True)
    drawn, given, kb = both_paths(q, qw, inp, wl.alpha, p, 2024, 17)
    for name, a, b in zip(("h", "u", "dX", "dA", "dB"), drawn, given):
        assert torch.equal(a, b), name
    rng = np.random.default_rng(12)
    rows = np.sort(rng.choice(M, size=24, replace=False))
    ow = oracle_weight(qw)
    xb, Ab, Bb = bits(inp["x"]), bits(inp["A"]), bits(inp["B"])
    h_ref, _ = oracle.qlora_fwd_rows_dropout(ow, N, K, xb, Ab, Bb, r, wl.alpha, p, kb, rows=rows)
    dX_ref, dA_ref, dB_ref = oracle.qlora_bwd_dropout(ow, N, K, xb, Ab, Bb, r, wl.alpha, p, kb,
                                                      bits(inp["dY"]), dx_rows=rows)
    h, _, dX, dA, dB = drawn
    errs = {"h": rel_err(to_f64(h)[rows], h_ref), "dX": rel_err(to_f64(dX)[rows], dX_ref),
            "dA": rel_err(to_f64(dA), dA_ref), "dB": rel_err(to_f64(dB), dB_ref)}
    assert all(v <= TOL for v in errs.values()), errs
    # the fraction kept is the Bernoulli(1 - p) mean within 6 sigma
    kept = int(np.unpackbits(kb, bitorder="little").sum())
    assert abs(kept - M * K * (1 - p)) < 6 * np.sqrt(M * K * p * (1 - p))
