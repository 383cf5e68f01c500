"""GPU parity of the fused QLoRA forward and backward against the CPU oracle.

Bar (per output tensor): max|gpu - oracle| <= 2e-2 * rms(oracle), with the
oracle in fp64 from the same bf16 inputs and the same NF4 weight (the GPU's
own quantisation, already checked bit-exact against the oracle's). The LoRA
branch is also checked alone (W0 = 0) against its own rms, because at large
shapes it is only a few percent of h.

The outputs are bf16, so rounding the exact result alone costs up to 2^-9 of
each value. For the edge shapes below (one token, an outer-product dA/dB)
max|y| / rms(y) exceeds 10 and that rounding by itself reaches the bar, so
those cases add an element-wise allowance of 2^-8 * |oracle| (one bf16 ulp)
to it. The named workloads use the bar as stated."""
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


def bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def rel_err(got: np.ndarray, ref: np.ndarray, ulp_allowance: bool = False) -> float:
    """max over elements of |got - ref| / (TOL-scaled bar); <= TOL passes."""
    rms = max(np.sqrt(np.mean(ref ** 2)), 1e-300)
    if not ulp_allowance:
        return float(np.max(np.abs(got - ref)) / rms)
    # |got - ref| <= TOL*rms + 2^-8 |ref|  <=>  excess/rms <= TOL
    return float(np.max(np.abs(got - ref) - 2.0 ** -8 * np.abs(ref)) / rms)


def oracle_weight(qw):
    """The GPU's quantised weight as an oracle Quantized record."""
    nb = qw.n * qw.k // qw.block_size
    return oracle.Quantized(qw.codes.cpu().numpy(), qw.absmax.cpu().numpy()[:nb],
                            qw.absmax_q8.cpu().numpy()[:nb] if qw.double_quant else None,
                            qw.absmax_c.cpu().numpy()[: (nb + 255) // 256] if qw.double_quant else None,
                            qw.block_size, qw.double_quant, 256, qw.n * qw.k)


def run_layer(q, W0, A, B, x, dY, alpha, dq, rows=None, need_bwd=True, block=64):
    dev = "cuda"
    qw = q.nf4_quantize(W0.to(dev), double_quant=dq, block_size=block)
    xd, Ad, Bd = x.to(dev), A.to(dev), B.to(dev)
    h, u = q.qlora_linear_fwd(qw, xd, Ad, Bd, alpha)
    out = {"qw": qw, "h": h, "u": u}
    if need_bwd:
        dX, dA, dB = q.qlora_linear_bwd(qw, xd, Ad, Bd, alpha, dY.to(dev), u=u)
        out.update(dX=dX, dA=dA, dB=dB)
    torch.cuda.synchronize()
    assert q.device_status() == q.NF4_OK
    return out


def check_against_oracle(q, res, A, B, x, dY, alpha, rows=None, need_bwd=True, tag="",
                         edge=False):
    qw = res["qw"]
    N, K, r, M = qw.n, qw.k, A.shape[0], x.shape[0]
    ow = oracle_weight(qw)
    xb, Ab, Bb = bits(x), bits(A), bits(B)
    rows = np.arange(M) if rows is None else np.asarray(rows)
    h_ref, u_ref = oracle.qlora_fwd_rows(ow, N, K, xb, Ab, Bb, r, alpha, rows=rows)
    errs = {"h": rel_err(to_f64(res["h"])[rows], h_ref, edge),
            "u": rel_err(res["u"].cpu().numpy().astype(np.float64)[rows], u_ref)}
    if need_bwd:
        dX_ref, dA_ref, dB_ref = oracle.qlora_bwd(ow, N, K, xb, Ab, Bb, r, alpha, bits(dY),
                                                  dx_rows=rows)
        errs.update(dX=rel_err(to_f64(res["dX"])[rows], dX_ref, edge),
                    dA=rel_err(to_f64(res["dA"]), dA_ref, edge),
                    dB=rel_err(to_f64(res["dB"]), dB_ref, edge))
    bad = {k: v for k, v in errs.items() if not v <= TOL}
    assert not bad, f"{tag} relative errors over {TOL}: {errs}"
    return errs


SMALL = [
    # (N, K, M, r, alpha, dq)   several tiles in every dimension, ragged tails
    (384, 512, 300, 16, 32.0, True),
    (256, 256, 128, 8, 16.0, False),
    (520, 640, 77, 64, 16.0, True),
    (264, 192, 1, 128, 32.0, True),
    (128, 1088, 513, 32, 8.0, False),
]


@pytest.mark.parametrize("N,K,M,r,alpha,dq", SMALL)
def test_layer_small_shapes(q, N, K, M, r, alpha, dq):
    w = workloads.LayerWorkload("t", N, K, M, r, alpha, 0.02, dq, 12345 + N + K + M + r)
    inp = workloads.make_inputs(w)
    res = run_layer(q, inp["W0"], inp["A"], inp["B"], inp["x"], inp["dY"], alpha, dq)
    check_against_oracle(q, res, inp["A"], inp["B"], inp["x"], inp["dY"], alpha,
                         tag=f"{N}x{K} M={M} r={r}", edge=M < 16)


# More 256 x 256 output tiles than resident CTA pairs (74 on a B200): round-
# robin waves, then the last tiles split between pairs (stream-K); ragged
# token and feature tails, one and two LoRA stages, blocks of 64 and 128.
STREAM_K_SHAPES = [
    # (N, K, M, r, alpha, dq, block)
    (8000, 576, 600, 16, 32.0, True, 64),
    (8000, 512, 520, 128, 16.0, False, 64),
    (7944, 1152, 700, 64, 16.0, True, 128),
]


@pytest.mark.parametrize("N,K,M,r,alpha,dq,block", STREAM_K_SHAPES)
def test_layer_stream_k_ragged(q, N, K, M, r, alpha, dq, block):
    w = workloads.LayerWorkload("t", N, K, M, r, alpha, 0.02, dq, 3131 + N + K + M + r)
    inp = workloads.make_inputs(w)
    res = run_layer(q, inp["W0"], inp["A"], inp["B"], inp["x"], inp["dY"], alpha, dq, block=block)
    check_against_oracle(q, res, inp["A"], inp["B"], inp["x"], inp["dY"], alpha,
                         rows=sampled_rows(M, 40, 7), tag=f"{N}x{K} M={M} r={r} b{block}")


def test_stream_k_lora_branch_alone(q):
    """W0 = 0 on a stream-K forward: h is the up-projection stage alone, also in
    the tiles split between two CTA pairs."""
    N, K, M, r, alpha = 8000, 512, 520, 64, 16.0
    w = workloads.LayerWorkload("t", N, K, M, r, alpha, 0.02, True, 6262)
    inp = workloads.make_inputs(w)
    res = run_layer(q, torch.zeros(N, K), inp["A"], inp["B"], inp["x"], inp["dY"], alpha, True,
                    need_bwd=False)
    check_against_oracle(q, res, inp["A"], inp["B"], inp["x"], None, alpha, need_bwd=False,
                         rows=sampled_rows(M, 40, 9), tag="stream-K lora-only")
    assert float(res["h"].float().abs().max()) > 0


@pytest.mark.parametrize("r", [8, 64])
def test_lora_branch_alone(q, r):
    """W0 = 0: every code is the zero level, h and dX are the LoRA terms only."""
    N, K, M, alpha = 320, 384, 200, 16.0
    w = workloads.LayerWorkload("t", N, K, M, r, alpha, 0.02, True, 777 + r)
    inp = workloads.make_inputs(w)
    W0 = torch.zeros(N, K)
    res = run_layer(q, W0, inp["A"], inp["B"], inp["x"], inp["dY"], alpha, True)
    assert torch.all(res["qw"].codes == 0x77)
    errs = check_against_oracle(q, res, inp["A"], inp["B"], inp["x"], inp["dY"], alpha,
                                tag="lora-only")
    assert float(res["h"].float().abs().max()) > 0


def test_b_zero_is_base_only(q):
    N, K, M, r, alpha = 256, 320, 130, 16, 32.0
    w = workloads.LayerWorkload("t", N, K, M, r, alpha, 0.02, True, 4242)
    inp = workloads.make_inputs(w)
    B0 = torch.zeros_like(inp["B"])
    res = run_layer(q, inp["W0"], inp["A"], B0, inp["x"], inp["dY"], alpha, True)
    check_against_oracle(q, res, inp["A"], B0, inp["x"], inp["dY"], alpha, tag="B=0")
    assert float(res["dA"].float().abs().max()) == 0.0   # v = dY B = 0


@pytest.mark.parametrize("N,K,M,r,alpha,dq", [SMALL[0], SMALL[2], SMALL[4],
                                              (5120, 5120, 2048, 16, 32.0, True)])
def test_fp32_adapter_gradients(q, N, K, M, r, alpha, dq):
    """qlora_linear_bwd_f32grad: dA and dB in fp32 against the oracle at the
    bar, and their bf16 rounding is the bf16 entry point's result bit for bit
    (both round the same fp32 sums; dX is the same launch sequence)."""
    w = workloads.LayerWorkload("t", N, K, M, r, alpha, 0.02, dq, 999 + N + K + M + r)
    inp = workloads.make_inputs(w)
    dev = "cuda"
    qw = q.nf4_quantize(inp["W0"].to(dev), double_quant=dq)
    x, A, B, dY = (inp[k].to(dev) for k in ("x", "A", "B", "dY"))
    h, u = q.qlora_linear_fwd(qw, x, A, B, alpha)
    dX16, dA16, dB16 = q.qlora_linear_bwd(qw, x, A, B, alpha, dY, u=u)
    dX32, dA32, dB32 = q.qlora_linear_bwd(qw, x, A, B, alpha, dY, u=u, grad_dtype=torch.float32)
    torch.cuda.synchronize()
    assert q.device_status() == q.NF4_OK
    assert dA32.dtype == torch.float32 and dB32.dtype == torch.float32
    assert torch.equal(dA32.to(torch.bfloat16), dA16) and torch.equal(dB32.to(torch.bfloat16), dB16)
    assert torch.equal(dX32, dX16)
    ow = oracle_weight(qw)
    _, dA_ref, dB_ref = oracle.qlora_bwd(ow, N, K, bits(inp["x"]), bits(inp["A"]), bits(inp["B"]), r,
                                         alpha, bits(inp["dY"]), dx_rows=[])
    assert rel_err(to_f64(dA32), dA_ref) <= TOL and rel_err(to_f64(dB32), dB_ref) <= TOL


def test_single_1024_workload(q):
    w = workloads.WORKLOADS["single_1024"]
    inp = workloads.make_inputs(w)
    res = run_layer(q, inp["W0"], inp["A"], inp["B"], inp["x"], inp["dY"], w.alpha, w.double_quant)
    check_against_oracle(q, res, inp["A"], inp["B"], inp["x"], inp["dY"], w.alpha, tag=w.name)


def sampled_rows(M, count, seed):
    rng = np.random.default_rng(seed)
    rows = rng.choice(M, size=min(count, M), replace=False)
    rows[:2] = [0, M - 1]
    return np.sort(rows)


def test_llama13b_attention_full_size(q):
    w = workloads.WORKLOADS["llama13b_attn_5120"]
    inp = workloads.make_inputs(w)
    res = run_layer(q, inp["W0"], inp["A"], inp["B"], inp["x"], inp["dY"], w.alpha, w.double_quant)
    check_against_oracle(q, res, inp["A"], inp["B"], inp["x"], inp["dY"], w.alpha,
                         rows=sampled_rows(w.M, 48, 1), tag=w.name)


@pytest.mark.parametrize("layer,proj", [(0, 0), (17, 2), (39, 3)])
def test_llama13b_stack_projection_full_size(q, layer, proj):
    """Projections of the 40-layer x {Q,K,V,O} adapter stack, each with its own seed, at the
    stack's 4096 tokens: every row of dA and dB, sampled rows of h and dX."""
    w = workloads.WORKLOADS["llama13b_stack_40x4"]
    inp = workloads.make_inputs(w, seed=workloads.stack_seed(layer, proj))
    res = run_layer(q, inp["W0"], inp["A"], inp["B"], inp["x"], inp["dY"], w.alpha, w.double_quant)
    check_against_oracle(q, res, inp["A"], inp["B"], inp["x"], inp["dY"], w.alpha,
                         rows=sampled_rows(w.M, 32, 100 + layer), tag=f"{w.name} {layer}/{proj}")


@pytest.mark.parametrize("M", [1, 4, 16])
def test_decode_workload_full_size(q, M):
    w = workloads.WORKLOADS["decode_mlp_up_13824x5120"]
    inp = workloads.make_inputs(w, M=M)
    res = run_layer(q, inp["W0"], inp["A"], inp["B"], inp["x"], None, w.alpha, w.double_quant,
                    need_bwd=False)
    check_against_oracle(q, res, inp["A"], inp["B"], inp["x"], None, w.alpha, need_bwd=False,
                         tag=f"{w.name} M={M}")


@pytest.mark.slow
def test_llama2_70b_mlp_full_size(q):
    w = workloads.WORKLOADS["llama2_70b_mlp_28672x8192"]
    inp = workloads.make_inputs(w)
    res = run_layer(q, inp["W0"], inp["A"], inp["B"], inp["x"], inp["dY"], w.alpha, w.double_quant)
    check_against_oracle(q, res, inp["A"], inp["B"], inp["x"], inp["dY"], w.alpha,
                         rows=sampled_rows(w.M, 12, 2), tag=w.name)


# ------------------------------------------------------------------ merge --
def merge_bound(qw, A, B, r, alpha, oracle_out, out_bf16):
    """Element-wise bar for the merge: the fp32 rank-r sum (r + 2 roundings of
    relative size 2^-24 on the sum of |terms|) plus, for bf16 output, the final
    rounding (2^-8 of the value, one bf16 unit in the last place)."""
    K = qw.k
    absBA = np.abs(oracle.bf16_to_f64(B)) @ np.abs(oracle.bf16_to_f64(A))
    w32 = np.abs(oracle.dequantize(oracle_weight(qw)).astype(np.float64).reshape(qw.n, K))
    acc = (r + 2) * 2.0 ** -24 * (w32 + (alpha / r) * absBA)
    return acc + (2.0 ** -8 * np.abs(oracle_out) if out_bf16 else 0.0)


MERGE_SHAPES = [
    # (N, K, r, alpha, dq)   ragged tiles in both dimensions; every supported rank class
    (200, 320, 16, 32.0, True),
    (64, 128, 8, 16.0, False),
    (136, 576, 64, 16.0, True),
    (72, 192, 128, 32.0, False),
    # 64 column stripes leave ~9 CTAs per stripe for 16 row tiles (the last one 40 rows): CTAs walk
    # several tiles with the next tile's operands in flight, and end on a ragged tile
    (1000, 8192, 16, 32.0, True),
    (1000, 8192, 64, 16.0, False),
]


@pytest.mark.parametrize("N,K,r,alpha,dq", MERGE_SHAPES)
@pytest.mark.parametrize("out_bf16", [True, False])
def test_merge_matches_oracle(q, N, K, r, alpha, dq, out_bf16):
    w = workloads.LayerWorkload("t", N, K, 1, r, alpha, 0.02, dq, 777 + N + r)
    inp = workloads.make_inputs(w)
    qw = q.nf4_quantize(inp["W0"].to("cuda"), double_quant=dq)
    out = q.qlora_merge(qw, inp["A"].cuda(), inp["B"].cuda(), alpha, bf16=out_bf16)
    torch.cuda.synchronize()
    assert q.device_status() == q.NF4_OK
    ref = oracle.qlora_merge(oracle_weight(qw), N, K, bits(inp["A"]), bits(inp["B"]), r, alpha)
    got = to_f64(out)
    bound = merge_bound(qw, bits(inp["A"]), bits(inp["B"]), r, alpha, ref, out_bf16)
    assert np.all(np.abs(got - ref) <= bound), float(np.max(np.abs(got - ref) - bound))
    assert np.max(np.abs(got - ref)) <= TOL * np.sqrt(np.mean(ref ** 2))


def test_merge_b_zero_is_dequantize(q):
    w = workloads.LayerWorkload("t", 128, 256, 1, 16, 32.0, 0.02, True, 4321)
    inp = workloads.make_inputs(w)
    qw = q.nf4_quantize(inp["W0"].to("cuda"), double_quant=True)
    B0 = torch.zeros_like(inp["B"]).cuda()
    for bf16 in (True, False):
        out = q.qlora_merge(qw, inp["A"].cuda(), B0, 32.0, bf16=bf16)
        assert torch.equal(out, q.nf4_dequantize(qw, bf16=bf16))


def test_merge_full_size_attention_projection(q):
    """The LLaMA-13B-like attention projection: every element against the oracle."""
    w = workloads.WORKLOADS["llama13b_attn_5120"]
    inp = workloads.make_inputs(w, M=0, with_dy=False)
    qw = q.nf4_quantize(inp["W0"].to("cuda"), double_quant=True)
    out = q.qlora_merge(qw, inp["A"].cuda(), inp["B"].cuda(), w.alpha, bf16=True)
    torch.cuda.synchronize()
    ref = oracle.qlora_merge(oracle_weight(qw), w.N, w.K, bits(inp["A"]), bits(inp["B"]), w.r, w.alpha)
    bound = merge_bound(qw, bits(inp["A"]), bits(inp["B"]), w.r, w.alpha, ref, True)
    assert np.all(np.abs(to_f64(out) - ref) <= bound)


# ---------------------------------------------------------- multi-adapter --
MULTI_SHAPES = [
    # (N, K, M, r, n_adapters)  decode path (n_adapters * r <= 64, M <= 16) and the GEMM path
    (264, 512, 12, 8, 4),
    (520, 640, 16, 16, 4),
    (384, 576, 300, 16, 8),
    (256, 320, 77, 8, 16),
]


def multi_inputs(N, K, M, r, n_ad, seed, zero_w=False):
    w = workloads.LayerWorkload("t", N, K, M, r * n_ad, 16.0, 0.02, True, seed)
    inp = workloads.make_inputs(w, with_dy=False)
    W0 = torch.zeros(N, K) if zero_w else inp["W0"]
    rng = np.random.default_rng(seed)
    adapter = rng.integers(-1, n_ad, size=M).astype(np.int32)
    alphas = [float(v) for v in rng.choice([8.0, 16.0, 32.0], size=n_ad)]
    return W0, inp["x"], inp["A"], inp["B"], adapter, alphas


@pytest.mark.parametrize("N,K,M,r,n_ad", MULTI_SHAPES)
@pytest.mark.parametrize("zero_w", [False, True])
def test_multi_adapter_forward(q, N, K, M, r, n_ad, zero_w):
    """Per-token adapters against the oracle; with W0 = 0 the output is the
    adapter terms alone, checked against their own rms."""
    W0, x, A_all, B_all, adapter, alphas = multi_inputs(N, K, M, r, n_ad, 900 + N + M, zero_w)
    qw = q.nf4_quantize(W0.cuda(), double_quant=True)
    h = q.qlora_multi_lora_fwd(qw, x.cuda(), A_all.cuda(), B_all.cuda(), r, alphas,
                               torch.from_numpy(adapter).cuda())
    torch.cuda.synchronize()
    assert q.device_status() == q.NF4_OK
    ref = oracle.qlora_multi_fwd_rows(oracle_weight(qw), N, K, bits(x), bits(A_all), bits(B_all),
                                      r, alphas, adapter)
    # W0 = 0 leaves the adapter terms alone, with zero rows for tokens without an
    # adapter: max/rms reaches ~7 and rounding the exact result to bf16 alone costs
    # ~0.016 of the bar, so these checks take the one-ulp allowance of the edge cases
    err = rel_err(to_f64(h), ref, M < 16 or zero_w)
    assert err <= TOL, err
    if zero_w:
        assert np.all(to_f64(h)[adapter < 0] == 0.0)     # no adapter, zero base: exactly zero


def test_multi_adapter_single_adapter_equals_layer_forward(q):
    """One adapter applied to every token is the ordinary forward, bit for bit."""
    N, K, M, r = 384, 512, 200, 16
    W0, x, A, B, _, _ = multi_inputs(N, K, M, r, 1, 4242)
    qw = q.nf4_quantize(W0.cuda(), double_quant=True)
    idx = torch.zeros(M, dtype=torch.int32, device="cuda")
    h1 = q.qlora_multi_lora_fwd(qw, x.cuda(), A.cuda(), B.cuda(), r, [16.0], idx)
    h2, _ = q.qlora_linear_fwd(qw, x.cuda(), A.cuda(), B.cuda(), 16.0)
    assert torch.equal(h1, h2)


# ---------------------------------------------------------------- dropout --
DROPOUT_SHAPES = [
    # (N, K, M, r, p, dq)   GEMM path with ragged tiles, and the decode path (M <= 16)
    (384, 512, 300, 16, 0.05, True),
    (520, 640, 77, 64, 0.3, False),
    (264, 512, 12, 16, 0.1, True),
]


def dropout_run(q, N, K, M, r, p, dq, seed, zero_w=False):
    w = workloads.LayerWorkload("t", N, K, M, r, 32.0, 0.02, dq, seed)
    inp = workloads.make_inputs(w)
    W0 = torch.zeros(N, K) if zero_w else inp["W0"]
    keep_bool = torch.from_numpy(np.random.default_rng(seed).random((M, K)) >= p)
    keep = q.pack_keep(keep_bool.cuda())
    qw = q.nf4_quantize(W0.cuda(), double_quant=dq)
    x, A, B, dY = (inp[k].cuda() for k in ("x", "A", "B", "dY"))
    h, u = q.qlora_linear_fwd_dropout(qw, x, A, B, w.alpha, p, keep)
    dX, dA, dB = q.qlora_linear_bwd_dropout(qw, x, A, B, w.alpha, p, keep, dY, u=u)
    torch.cuda.synchronize()
    assert q.device_status() == q.NF4_OK
    ow = oracle_weight(qw)
    kb = oracle.pack_keep(keep_bool.numpy())
    h_ref, u_ref = oracle.qlora_fwd_rows_dropout(ow, N, K, bits(inp["x"]), bits(inp["A"]), bits(inp["B"]),
                                                 r, w.alpha, p, kb)
    g_ref = oracle.qlora_bwd_dropout(ow, N, K, bits(inp["x"]), bits(inp["A"]), bits(inp["B"]), r,
                                     w.alpha, p, kb, bits(inp["dY"]))
    return (h, u, dX, dA, dB), (h_ref, u_ref) + tuple(g_ref)


@pytest.mark.parametrize("N,K,M,r,p,dq", DROPOUT_SHAPES)
@pytest.mark.parametrize("zero_w", [False, True])
def test_dropout_forward_backward(q, N, K, M, r, p, dq, zero_w):
    """With W0 = 0 the outputs are the masked adapter terms alone (h, dX), against their own rms."""
    got, ref = dropout_run(q, N, K, M, r, p, dq, 321 + N + M, zero_w)
    names = ("h", "u", "dX", "dA", "dB")
    errs = {}
    for name, g, rf in zip(names, got, ref):
        gv = g.detach().float().cpu().numpy().astype(np.float64)
        errs[name] = rel_err(gv, np.asarray(rf), M < 16 or zero_w)
    bad = {k: v for k, v in errs.items() if not v <= TOL}
    assert not bad, errs


def test_dropout_keep_all_forward_is_the_plain_forward(q):
    N, K, M, r = 384, 512, 200, 16
    w = workloads.LayerWorkload("t", N, K, M, r, 32.0, 0.02, True, 999)
    inp = workloads.make_inputs(w)
    qw = q.nf4_quantize(inp["W0"].cuda(), double_quant=True)
    x, A, B = (inp[k].cuda() for k in ("x", "A", "B"))
    keep = q.pack_keep(torch.ones(M, K, dtype=torch.bool, device="cuda"))
    h1, u1 = q.qlora_linear_fwd_dropout(qw, x, A, B, w.alpha, 0.0, keep)
    h2, u2 = q.qlora_linear_fwd(qw, x, A, B, w.alpha)
    assert torch.equal(h1, h2) and torch.equal(u1, u2)


def test_dropout_full_size_attention_projection(q):
    """The LLaMA-13B-like projection with p = 0.05 (the pages' recipe): sampled rows
    of h and dX, all of dA and dB."""
    wl = workloads.WORKLOADS["llama13b_attn_5120"]
    N, K, M, r, p = wl.N, wl.K, wl.M, wl.r, 0.05
    inp = workloads.make_inputs(wl)
    keep_bool = torch.from_numpy(np.random.default_rng(5).random((M, K)) >= p)
    keep = q.pack_keep(keep_bool.cuda())
    qw = q.nf4_quantize(inp["W0"].cuda(), double_quant=True)
    x, A, B, dY = (inp[k].cuda() for k in ("x", "A", "B", "dY"))
    h, u = q.qlora_linear_fwd_dropout(qw, x, A, B, wl.alpha, p, keep)
    dX, dA, dB = q.qlora_linear_bwd_dropout(qw, x, A, B, wl.alpha, p, keep, dY, u=u)
    torch.cuda.synchronize()
    rows = sampled_rows(M, 32, 11)
    ow = oracle_weight(qw)
    kb = oracle.pack_keep(keep_bool.numpy())
    h_ref, _ = oracle.qlora_fwd_rows_dropout(ow, N, K, bits(inp["x"]), bits(inp["A"]), bits(inp["B"]),
                                             r, wl.alpha, p, kb, rows=rows)
    dX_ref, dA_ref, dB_ref = oracle.qlora_bwd_dropout(ow, N, K, bits(inp["x"]), bits(inp["A"]),
                                                      bits(inp["B"]), r, wl.alpha, p, kb,
                                                      bits(inp["dY"]), dx_rows=rows)
    errs = {"h": rel_err(to_f64(h)[rows], h_ref), "dX": rel_err(to_f64(dX)[rows], dX_ref),
            "dA": rel_err(to_f64(dA), dA_ref), "dB": rel_err(to_f64(dB), dB_ref)}
    assert all(v <= TOL for v in errs.values()), errs


def test_empty_batch(q):
    """M = 0: the forwards write nothing; the backwards write zero dA and dB (the
    gradient of an empty batch), with or without dropout."""
    N, K, r = 136, 640, 16
    w = workloads.LayerWorkload("t", N, K, 1, r, 16.0, 0.02, True, 31)
    inp = workloads.make_inputs(w)
    qw = q.nf4_quantize(inp["W0"].cuda(), double_quant=True)
    A, B = inp["A"].cuda(), inp["B"].cuda()
    x = torch.empty(0, K, dtype=torch.bfloat16, device="cuda")
    dY = torch.empty(0, N, dtype=torch.bfloat16, device="cuda")
    keep = q.pack_keep(torch.ones(0, K, dtype=torch.bool, device="cuda"))

    def nan_outs():
        return (torch.empty(0, K, dtype=torch.bfloat16, device="cuda"),
                torch.full((r, K), float("nan"), dtype=torch.bfloat16, device="cuda"),
                torch.full((N, r), float("nan"), dtype=torch.bfloat16, device="cuda"))

    h, u = q.qlora_linear_fwd(qw, x, A, B, 16.0)
    outs = nan_outs()
    q.qlora_linear_bwd(qw, x, A, B, 16.0, dY, u=u, outs=outs)
    hd, ud = q.qlora_linear_fwd_dropout(qw, x, A, B, 16.0, 0.1, keep)
    outs_d = nan_outs()
    q.qlora_linear_bwd_dropout(qw, x, A, B, 16.0, 0.1, keep, dY, u=ud, outs=outs_d)
    torch.cuda.synchronize()
    assert q.device_status() == q.NF4_OK
    assert h.shape == (0, N) and u.shape == (0, r) and hd.shape == (0, N)
    for t in outs[1:] + outs_d[1:]:
        assert int(torch.count_nonzero(t)) == 0
