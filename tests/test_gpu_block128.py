"""GPU parity with 128-element NF4 blocks ("QLoRA Finetuner -- Juan Martos",
section 2: blocks of 64 or 128 weights, one absmax each). Codes, scales and
double-quant codes bit for bit; the layer's forward, backward, decode path,
merge, multi-adapter and dropout forms within the floating-point bar."""
import numpy as np
import pytest
import torch

import oracle
import test_gpu_codec as C
import test_gpu_layer as L
import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def q():
    import bit_nf4_quantized_05_b200 as mod
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    return mod


# ------------------------------------------------------------------ codec --
@pytest.mark.parametrize("shape,dq", [((8, 128), True), ((24, 896), True), ((200, 640), False),
                                      ((136, 1280), True), ((64, 4096), False)])
def test_quantize_block128_random_shapes(q, shape, dq):
    """Ragged stages (32 blocks) and groups (256 blocks) in every shape but the last."""
    rng = np.random.default_rng(shape[0] * 5 + shape[1])
    W = rng.normal(0, 0.02, size=shape).astype(np.float32)
    W *= rng.uniform(0.2, 5.0, size=(shape[0], 1)).astype(np.float32)
    ref, qw = C.quant_both(q, W, dq, block=128)
    C.assert_quant_equal(ref, qw)
    C.assert_dequant_equal(q, ref, qw)


def test_quantize_block128_midpoints_and_special_blocks(q):
    """Level midpoints and their fp32 neighbours against a unit absmax, the
    maximum in either half of a block, all-zero and tiny blocks."""
    lv = oracle.levels()
    mids = [np.float32((float(lv[i]) + float(lv[i + 1])) / 2) for i in range(15)]
    vals = []
    for v in mids:
        vals += [v, np.nextafter(v, np.float32(2)), np.nextafter(v, np.float32(-2))]
    vals = np.array(vals, dtype=np.float32)
    blocks = []
    for i, pos in enumerate([0, 127, 64, 63]):          # where the unit maximum sits
        b = np.zeros(128, dtype=np.float32)
        b[pos] = -1.0 if i % 2 else 1.0
        rest = [j for j in range(128) if j != pos]
        b[rest[: vals.size]] = vals
        blocks.append(b)
    blocks.append(np.zeros(128, dtype=np.float32))
    b = np.full(128, 1e-38, dtype=np.float32); blocks.append(b)
    b = (np.float32(0.37) * lv[np.arange(128) % 16]).astype(np.float32); blocks.append(b)
    while len(blocks) % 8:
        blocks.append(np.random.default_rng(len(blocks)).normal(size=128).astype(np.float32))
    W = np.concatenate(blocks).reshape(8, -1)
    for dq in (False, True):
        ref, qw = C.quant_both(q, W, dq, block=128)
        C.assert_quant_equal(ref, qw)
        C.assert_dequant_equal(q, ref, qw)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("shape,dq", [((24, 896), True), ((1000, 640), False)])
def test_quantize_block128_16bit_input(q, dtype, shape, dq):
    rng = np.random.default_rng(shape[0] + shape[1])
    W = rng.normal(0, 0.02, size=shape).astype(np.float32)
    ref, qw = C.quant_16(q, torch.from_numpy(W).to(dtype), dq, block=128)
    C.assert_quant_equal(ref, qw)


def test_quantize_block128_outlier_workload_full_size(q):
    w = workloads.WORKLOADS["decode_mlp_up_13824x5120"]
    ref, qw = C.quant_both(q, workloads.make_weight(w).numpy(), True, block=128)
    C.assert_quant_equal(ref, qw)


# ------------------------------------------------------------------ layer --
SMALL_128 = [
    # (N, K, M, r, alpha, dq)   GEMM path with ragged tiles; decode path (M <= 16) with
    # K / 128 = 9 blocks per row, so double-quant groups start inside rows and chunks
    (384, 512, 300, 16, 32.0, True),
    (520, 640, 77, 64, 16.0, True),
    (256, 1152, 129, 8, 16.0, False),
    (264, 1152, 1, 128, 32.0, True),
    (512, 1152, 16, 16, 16.0, True),
    (136, 640, 5, 32, 8.0, False),
]


@pytest.mark.parametrize("N,K,M,r,alpha,dq", SMALL_128)
def test_layer_block128_small_shapes(q, N, K, M, r, alpha, dq):
    w = workloads.LayerWorkload("t", N, K, M, r, alpha, 0.02, dq, 5150 + N + K + M + r)
    inp = workloads.make_inputs(w)
    res = L.run_layer(q, inp["W0"], inp["A"], inp["B"], inp["x"], inp["dY"], alpha, dq, block=128)
    assert res["qw"].block_size == 128
    L.check_against_oracle(q, res, inp["A"], inp["B"], inp["x"], inp["dY"], alpha,
                           tag=f"b128 {N}x{K} M={M} r={r}", edge=M < 16)


def test_layer_block128_attention_full_size(q):
    w = workloads.WORKLOADS["llama13b_attn_5120"]
    inp = workloads.make_inputs(w)
    res = L.run_layer(q, inp["W0"], inp["A"], inp["B"], inp["x"], inp["dY"], w.alpha, w.double_quant,
                      block=128)
    L.check_against_oracle(q, res, inp["A"], inp["B"], inp["x"], inp["dY"], w.alpha,
                           rows=L.sampled_rows(w.M, 32, 7), tag=f"b128 {w.name}")


@pytest.mark.parametrize("M", [1, 16])
def test_decode_block128_full_size(q, M):
    w = workloads.WORKLOADS["decode_mlp_up_13824x5120"]
    inp = workloads.make_inputs(w, M=M)
    res = L.run_layer(q, inp["W0"], inp["A"], inp["B"], inp["x"], None, w.alpha, w.double_quant,
                      need_bwd=False, block=128)
    L.check_against_oracle(q, res, inp["A"], inp["B"], inp["x"], None, w.alpha, need_bwd=False,
                           tag=f"b128 {w.name} M={M}")


@pytest.mark.parametrize("dq", [False, True])
@pytest.mark.parametrize("out_bf16", [True, False])
def test_merge_block128(q, dq, out_bf16):
    N, K, r, alpha = 200, 640, 16, 32.0
    w = workloads.LayerWorkload("t", N, K, 1, r, alpha, 0.02, dq, 8128)
    inp = workloads.make_inputs(w)
    qw = q.nf4_quantize(inp["W0"].cuda(), double_quant=dq, block_size=128)
    out = q.qlora_merge(qw, inp["A"].cuda(), inp["B"].cuda(), alpha, bf16=out_bf16)
    torch.cuda.synchronize()
    assert q.device_status() == q.NF4_OK
    Ab, Bb = L.bits(inp["A"]), L.bits(inp["B"])
    ref = oracle.qlora_merge(L.oracle_weight(qw), N, K, Ab, Bb, r, alpha)
    bound = L.merge_bound(qw, Ab, Bb, r, alpha, ref, out_bf16)
    assert np.all(np.abs(L.to_f64(out) - ref) <= bound)


@pytest.mark.parametrize("N,K,M", [(264, 512, 12), (384, 640, 300)])
def test_multi_adapter_block128(q, N, K, M):
    r, n_ad = 8, 4
    W0, x, A_all, B_all, adapter, alphas = L.multi_inputs(N, K, M, r, n_ad, 1280 + M)
    qw = q.nf4_quantize(W0.cuda(), double_quant=True, block_size=128)
    h = q.qlora_multi_lora_fwd(qw, x.cuda(), A_all.cuda(), B_all.cuda(), r, alphas,
                               torch.from_numpy(adapter).cuda())
    torch.cuda.synchronize()
    assert q.device_status() == q.NF4_OK
    ref = oracle.qlora_multi_fwd_rows(L.oracle_weight(qw), N, K, L.bits(x), L.bits(A_all),
                                      L.bits(B_all), r, alphas, adapter)
    err = L.rel_err(L.to_f64(h), ref, M < 16)
    assert err <= L.TOL, err


@pytest.mark.parametrize("N,K,M", [(384, 512, 300), (264, 640, 12)])
def test_dropout_block128(q, N, K, M):
    r, p, alpha, seed = 16, 0.1, 32.0, 6128 + M
    w = workloads.LayerWorkload("t", N, K, M, r, alpha, 0.02, True, seed)
    inp = workloads.make_inputs(w)
    keep_bool = torch.from_numpy(np.random.default_rng(seed).random((M, K)) >= p)
    keep = q.pack_keep(keep_bool.cuda())
    qw = q.nf4_quantize(inp["W0"].cuda(), double_quant=True, block_size=128)
    x, A, B, dY = (inp[k].cuda() for k in ("x", "A", "B", "dY"))
    h, u = q.qlora_linear_fwd_dropout(qw, x, A, B, alpha, p, keep)
    dX, dA, dB = q.qlora_linear_bwd_dropout(qw, x, A, B, alpha, p, keep, dY, u=u)
    torch.cuda.synchronize()
    assert q.device_status() == q.NF4_OK
    ow = L.oracle_weight(qw)
    kb = oracle.pack_keep(keep_bool.numpy())
    xb, Ab, Bb = L.bits(inp["x"]), L.bits(inp["A"]), L.bits(inp["B"])
    h_ref, u_ref = oracle.qlora_fwd_rows_dropout(ow, N, K, xb, Ab, Bb, r, alpha, p, kb)
    dX_ref, dA_ref, dB_ref = oracle.qlora_bwd_dropout(ow, N, K, xb, Ab, Bb, r, alpha, p, kb, L.bits(inp["dY"]))
    edge = M < 16
    errs = {"h": L.rel_err(L.to_f64(h), h_ref, edge),
            "u": L.rel_err(u.cpu().numpy().astype(np.float64), u_ref),
            "dX": L.rel_err(L.to_f64(dX), dX_ref, edge),
            "dA": L.rel_err(L.to_f64(dA), dA_ref, edge),
            "dB": L.rel_err(L.to_f64(dB), dB_ref, edge)}
    assert all(v <= L.TOL for v in errs.values()), errs
