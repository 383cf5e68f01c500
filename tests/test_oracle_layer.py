"""Pins for the oracle's QLoRA forward and backward: the merged-weight
identity, B = 0 and W0 = 0 special cases, exact central differences on
dyadic inputs, an independent fp64 autograd opinion, and the pages'
parameter-count arithmetic."""
import numpy as np
import pytest
import torch

import oracle
from conftest import read_golden_kv


def dyadic_bf16(rng, shape, scale_pow=2):
    """Small integers times 2^-scale_pow: exact in bf16 and in fp64 sums."""
    vals = rng.integers(-2, 3, size=shape).astype(np.float32) * np.float32(2.0 ** -scale_pow)
    return oracle.f32_to_bf16(vals)


def random_layer(rng, N, K, M, r, dq, sigma=0.02, block=64):
    W = rng.normal(0, sigma, size=(N, K)).astype(np.float32)
    qw = oracle.quantize(W.reshape(-1), block=block, dq=dq)
    x = oracle.f32_to_bf16(rng.normal(size=(M, K)).astype(np.float32))
    A = oracle.f32_to_bf16(rng.uniform(-K ** -0.5, K ** -0.5, size=(r, K)).astype(np.float32))
    B = oracle.f32_to_bf16(rng.normal(0, 0.01, size=(N, r)).astype(np.float32))
    dY = oracle.f32_to_bf16(rng.normal(size=(M, N)).astype(np.float32))
    return qw, x, A, B, dY


def operand(qw, N, K):
    """The bf16 matmul operand RNE(w~) as fp64, via the oracle's codec."""
    return oracle.bf16_to_f64(oracle.f32_to_bf16(oracle.dequantize(qw))).reshape(N, K)


def f64(a):
    return oracle.bf16_to_f64(a)


@pytest.mark.parametrize("block", [64, 128])
@pytest.mark.parametrize("dq", [False, True])
def test_forward_equals_merged_weight(dq, block):
    rng = np.random.default_rng(21)
    N, K, M, r, alpha = 96, 256, 7, 8, 16.0
    qw, x, A, B, _ = random_layer(rng, N, K, M, r, dq, block=block)
    h, u = oracle.qlora_fwd_rows(qw, N, K, x, A, B, r, alpha)
    s = alpha / r
    merged = operand(qw, N, K) + s * f64(B) @ f64(A)        # W~ + (alpha/r) B A
    ref = f64(x) @ merged.T
    assert np.max(np.abs(h - ref)) <= 1e-12 * np.sqrt(np.mean(ref ** 2))
    assert np.allclose(u, f64(x) @ f64(A).T, rtol=0, atol=1e-13)
    # a subset of rows is the same as those rows of the full result
    h2, _ = oracle.qlora_fwd_rows(qw, N, K, x, A, B, r, alpha, rows=[6, 0, 3])
    assert np.array_equal(h2, h[[6, 0, 3]])


def test_b_zero_gives_base_output():
    rng = np.random.default_rng(22)
    N, K, M, r = 64, 128, 5, 16
    qw, x, A, B, _ = random_layer(rng, N, K, M, r, True)
    B0 = np.zeros_like(B)
    h, _ = oracle.qlora_fwd_rows(qw, N, K, x, A, B0, r, 32.0)
    assert np.array_equal(h, np.asarray(f64(x) @ operand(qw, N, K).T)) or \
        np.max(np.abs(h - f64(x) @ operand(qw, N, K).T)) < 1e-13


def test_w0_zero_gives_lora_only():
    rng = np.random.default_rng(23)
    N, K, M, r, alpha = 64, 128, 5, 8, 16.0
    qw = oracle.quantize(np.zeros(N * K, dtype=np.float32), dq=True)
    assert np.all(qw.codes == 0x77) and np.all(qw.absmax == 0)
    _, x, A, B, _ = random_layer(rng, N, K, M, r, True)
    h, _ = oracle.qlora_fwd_rows(qw, N, K, x, A, B, r, alpha)
    ref = (alpha / r) * (f64(x) @ f64(A).T) @ f64(B).T
    assert np.max(np.abs(h - ref)) <= 1e-13 * np.max(np.abs(ref))
    assert np.max(np.abs(ref)) > 0


def loss(qw, N, K, x, A, B, r, alpha, dY):
    h, _ = oracle.qlora_fwd_rows(qw, N, K, x, A, B, r, alpha)
    return float(np.sum(f64(dY) * h))


def test_backward_equals_exact_central_differences():
    """L = sum(dY * h) is linear in each of x, A, B; with dyadic inputs and a
    dyadic step the central difference is the exact partial derivative."""
    rng = np.random.default_rng(24)
    N, K, M, r, alpha = 16, 64, 3, 4, 8.0
    W = rng.normal(0, 0.02, size=(N, K)).astype(np.float32)
    qw = oracle.quantize(W.reshape(-1), dq=True)
    x, A, B, dY = (dyadic_bf16(rng, s) for s in [(M, K), (r, K), (N, r), (M, N)])
    dX, dA, dB = oracle.qlora_bwd(qw, N, K, x, A, B, r, alpha, dY)
    delta = np.float32(0.25)

    def fd(which, idx):
        arrs = {"x": x, "A": A, "B": B}
        base = f64(arrs[which]).astype(np.float32)
        plus, minus = base.copy(), base.copy()
        plus[idx] += delta
        minus[idx] -= delta
        lp = dict(arrs); lp[which] = oracle.f32_to_bf16(plus)
        lm = dict(arrs); lm[which] = oracle.f32_to_bf16(minus)
        assert np.array_equal(f64(lp[which]).astype(np.float32), plus)
        Lp = loss(qw, N, K, lp["x"], lp["A"], lp["B"], r, alpha, dY)
        Lm = loss(qw, N, K, lm["x"], lm["A"], lm["B"], r, alpha, dY)
        return (Lp - Lm) / (2 * float(delta))

    for idx in [(0, 0), (1, 17), (2, 63), (0, 31)]:
        assert fd("x", idx) == pytest.approx(dX[idx], rel=1e-12, abs=1e-12)
    for idx in [(0, 0), (3, 63), (1, 5), (2, 40)]:
        assert fd("A", idx) == pytest.approx(dA[idx], rel=1e-12, abs=1e-12)
    for idx in [(0, 0), (15, 3), (7, 1), (9, 2)]:
        assert fd("B", idx) == pytest.approx(dB[idx], rel=1e-12, abs=1e-12)
    # the gradients are not trivially zero
    assert np.abs(dX).max() > 0 and np.abs(dA).max() > 0 and np.abs(dB).max() > 0


@pytest.mark.parametrize("block", [64, 128])
@pytest.mark.parametrize("dq", [False, True])
def test_backward_matches_fp64_autograd(dq, block):
    rng = np.random.default_rng(25)
    N, K, M, r, alpha = 48, 128, 9, 8, 16.0
    qw, x, A, B, dY = random_layer(rng, N, K, M, r, dq, block=block)
    dX, dA, dB = oracle.qlora_bwd(qw, N, K, x, A, B, r, alpha, dY)
    Wt = torch.from_numpy(operand(qw, N, K))
    xt = torch.from_numpy(f64(x)).requires_grad_(True)
    At = torch.from_numpy(f64(A)).requires_grad_(True)
    Bt = torch.from_numpy(f64(B)).requires_grad_(True)
    h = xt @ Wt.T + (alpha / r) * (xt @ At.T) @ Bt.T
    (torch.from_numpy(f64(dY)) * h).sum().backward()
    for got, ref in [(dX, xt.grad), (dA, At.grad), (dB, Bt.grad)]:
        ref = ref.numpy()
        assert np.max(np.abs(got - ref)) <= 1e-12 * max(1e-30, np.sqrt(np.mean(ref ** 2)))
    # dX rows subset
    dX2, _, _ = oracle.qlora_bwd(qw, N, K, x, A, B, r, alpha, dY, dx_rows=[8, 2],
                                 want_dA=False, want_dB=False)
    assert np.array_equal(dX2, dX[[8, 2]])


def test_adapter_gradient_sizes_match_parameter_count():
    g = read_golden_kv("lora_param_count.txt")
    d, k, r = int(g["d"]), int(g["k"]), int(g["r"])
    rng = np.random.default_rng(26)
    qw = oracle.quantize(np.zeros(k * d, dtype=np.float32), dq=True)
    x = oracle.f32_to_bf16(rng.normal(size=(1, d)).astype(np.float32))
    A = np.zeros((r, d), dtype=np.uint16)
    B = np.zeros((k, r), dtype=np.uint16)
    dY = np.zeros((1, k), dtype=np.uint16)
    _, dA, dB = oracle.qlora_bwd(qw, k, d, x, A, B, r, 32.0, dY, dx_rows=[])
    assert dA.size + dB.size == int(g["per_matrix"])
    assert 4 * (dA.size + dB.size) == int(g["per_layer"])
    assert round(int(g["layers"]) * 4 * (dA.size + dB.size) / 1e6, 1) == float(g["total_millions"])


# ------------------------------------------------------------------ merge --
def test_merge_with_b_zero_is_the_dequantised_weight():
    rng = np.random.default_rng(31)
    N, K, r = 24, 192, 8
    qw, _, A, B, _ = random_layer(rng, N, K, 1, r, dq=True)
    out = oracle.qlora_merge(qw, N, K, A, np.zeros_like(B), r, 16.0)
    assert np.array_equal(out, oracle.dequantize(qw).astype(np.float64).reshape(N, K))


def test_merge_of_zero_weight_is_the_scaled_adapter_product():
    """W0 = 0 quantises to the zero level everywhere, so the merge is (alpha/r) B A alone,
    here checked against a library matrix product of the widened adapters."""
    rng = np.random.default_rng(32)
    N, K, r, alpha = 40, 128, 16, 32.0
    qw = oracle.quantize(np.zeros(N * K, dtype=np.float32), dq=False)
    A = oracle.f32_to_bf16(rng.uniform(-0.1, 0.1, size=(r, K)).astype(np.float32))
    B = oracle.f32_to_bf16(rng.normal(0, 0.01, size=(N, r)).astype(np.float32))
    out = oracle.qlora_merge(qw, N, K, A, B, r, alpha)
    ref = (alpha / r) * (f64(B) @ f64(A))
    assert np.allclose(out, ref, rtol=1e-13, atol=1e-16)
    # orientation: a transposed or unscaled product is far off
    assert not np.allclose(out, f64(B) @ f64(A), rtol=1e-3)


@pytest.mark.parametrize("dq", [False, True])
def test_merged_weight_reproduces_the_layer_forward(dq):
    """x W_merged^T equals the layer's forward up to the bf16 rounding of the base
    operand (the forward multiplies RNE_bf16(w~); the merge keeps w~ in fp32)."""
    rng = np.random.default_rng(33 + dq)
    N, K, M, r, alpha = 48, 256, 6, 16, 32.0
    qw, x, A, B, _ = random_layer(rng, N, K, M, r, dq)
    merged = oracle.qlora_merge(qw, N, K, A, B, r, alpha)
    h, _ = oracle.qlora_fwd_rows(qw, N, K, x, A, B, r, alpha)
    w32 = oracle.dequantize(qw).astype(np.float64).reshape(N, K)
    bound = np.abs(f64(x)) @ np.abs(operand(qw, N, K) - w32).T + 1e-12
    assert np.all(np.abs(f64(x) @ merged.T - h) <= bound)
    # without the adapter term the gap is far larger than the bound
    assert np.max(np.abs(f64(x) @ w32.T - h) - bound) > 0


# ---------------------------------------------------------- multi-adapter --
def test_multi_adapter_rows_equal_single_adapter_forwards():
    """Each token's row is the single-adapter forward with its own adapter (a
    separately pinned oracle); tokens without an adapter get the base output."""
    rng = np.random.default_rng(41)
    N, K, M, r, n_ad = 40, 192, 9, 8, 3
    alphas = [16.0, 8.0, 32.0]
    qw, x, _, _, _ = random_layer(rng, N, K, M, r, dq=True)
    As = [oracle.f32_to_bf16(rng.uniform(-0.1, 0.1, size=(r, K)).astype(np.float32)) for _ in range(n_ad)]
    Bs = [oracle.f32_to_bf16(rng.normal(0, 0.05, size=(N, r)).astype(np.float32)) for _ in range(n_ad)]
    A_all = np.concatenate(As, axis=0)
    B_all = np.concatenate(Bs, axis=1)
    adapter = np.array([0, 1, 2, -1, 2, 1, 0, -1, 1], dtype=np.int32)
    h = oracle.qlora_multi_fwd_rows(qw, N, K, x, A_all, B_all, r, alphas, adapter)
    for m in range(M):
        a = adapter[m]
        A1 = As[a] if a >= 0 else As[0]
        B1 = Bs[a] if a >= 0 else np.zeros_like(Bs[0])
        ref, _ = oracle.qlora_fwd_rows(qw, N, K, x, A1, B1, r, alphas[a] if a >= 0 else 1.0, rows=[m])
        assert np.array_equal(h[m], ref[0])
    # a wrong adapter for any token changes its row
    h_wrong = oracle.qlora_multi_fwd_rows(qw, N, K, x, A_all, B_all, r, alphas, (adapter + 1) % n_ad)
    assert not np.allclose(h_wrong, h, rtol=1e-3)


# ---------------------------------------------------------------- dropout --
def dropout_case(seed, N=32, K=192, M=7, r=8, p=0.25):
    rng = np.random.default_rng(seed)
    qw, x, A, B, dY = random_layer(rng, N, K, M, r, dq=True)
    keep_bool = rng.random((M, K)) >= p
    return qw, x, A, B, dY, keep_bool, oracle.pack_keep(keep_bool)


def test_dropout_with_nothing_dropped_is_the_plain_layer():
    qw, x, A, B, dY, _, _ = dropout_case(51)
    N, K, M, r = 32, 192, 7, 8
    allkeep = oracle.pack_keep(np.ones((M, K), dtype=bool))
    h, u = oracle.qlora_fwd_rows_dropout(qw, N, K, x, A, B, r, 16.0, 0.0, allkeep)
    h0, u0 = oracle.qlora_fwd_rows(qw, N, K, x, A, B, r, 16.0)
    assert np.array_equal(h, h0) and np.array_equal(u, u0)
    g = oracle.qlora_bwd_dropout(qw, N, K, x, A, B, r, 16.0, 0.0, allkeep, dY)
    g0 = oracle.qlora_bwd(qw, N, K, x, A, B, r, 16.0, dY)
    for a, b in zip(g, g0):
        assert np.array_equal(a, b)


def test_dropout_is_the_masked_input_with_rescaled_alpha():
    """Inverted dropout on the LoRA input equals the plain layer's adapter branch fed
    the masked tokens with alpha / (1 - p), plus the base of the unmasked tokens;
    the gradients follow the same composition, with the mask applied to the
    adapter part of dX."""
    N, K, M, r, alpha, p = 32, 192, 7, 8, 16.0, 0.25
    qw, x, A, B, dY, keep_bool, keep = dropout_case(52, N, K, M, r, p)
    xm = np.where(keep_bool, x, 0).astype(np.uint16)       # masked tokens (exact in bf16)
    a2 = alpha / (1.0 - p)
    zB = np.zeros_like(B)
    h, u = oracle.qlora_fwd_rows_dropout(qw, N, K, x, A, B, r, alpha, p, keep)
    base, _ = oracle.qlora_fwd_rows(qw, N, K, x, A, zB, r, alpha)
    hm, um = oracle.qlora_fwd_rows(qw, N, K, xm, A, B, r, a2)
    hm0, _ = oracle.qlora_fwd_rows(qw, N, K, xm, A, zB, r, a2)
    assert np.allclose(h, base + (hm - hm0), rtol=1e-12, atol=1e-14)
    assert np.array_equal(u, um)
    dX, dA, dB = oracle.qlora_bwd_dropout(qw, N, K, x, A, B, r, alpha, p, keep, dY)
    dXm, dAm, dBm = oracle.qlora_bwd(qw, N, K, xm, A, B, r, a2, dY)
    dX0, _, _ = oracle.qlora_bwd(qw, N, K, xm, A, zB, r, a2, dY)
    assert np.allclose(dA, dAm, rtol=1e-12, atol=1e-14)
    assert np.allclose(dB, dBm, rtol=1e-12, atol=1e-14)
    assert np.allclose(dX, dX0 + np.where(keep_bool, dXm - dX0, 0.0), rtol=1e-12, atol=1e-14)
    # the mask matters: without it every output moves
    assert not np.allclose(dA, oracle.qlora_bwd(qw, N, K, x, A, B, r, a2, dY)[1], rtol=1e-3)


def test_block128_with_equal_half_maxima_is_the_64_block_layer():
    """A 128-element block whose two halves have the same absmax quantises to
    the codes of two 64-element blocks with that scale; every layer result is
    then that of the 64-block weight, bit for bit."""
    rng = np.random.default_rng(41)
    N, K, M, r, alpha = 40, 384, 6, 8, 16.0
    W = np.clip(rng.normal(0, 0.02, size=(N, K)), -0.05, 0.05).astype(np.float32)
    W[:, 0::128] = 0.08
    W[:, 64::128] = -0.08
    q128 = oracle.quantize(W.reshape(-1), block=128)
    q64 = oracle.quantize(W.reshape(-1), block=64)
    assert np.array_equal(q128.codes, q64.codes)
    assert np.array_equal(np.repeat(q128.absmax, 2), q64.absmax)
    _, x, A, B, dY = random_layer(rng, N, K, M, r, False)
    h128, u128 = oracle.qlora_fwd_rows(q128, N, K, x, A, B, r, alpha)
    h64, u64 = oracle.qlora_fwd_rows(q64, N, K, x, A, B, r, alpha)
    assert np.array_equal(h128, h64) and np.array_equal(u128, u64)
    for g128, g64 in zip(oracle.qlora_bwd(q128, N, K, x, A, B, r, alpha, dY),
                         oracle.qlora_bwd(q64, N, K, x, A, B, r, alpha, dY)):
        assert np.array_equal(g128, g64)
    assert np.array_equal(oracle.qlora_merge(q128, N, K, A, B, r, alpha),
                          oracle.qlora_merge(q64, N, K, A, B, r, alpha))


def test_keep_mask_bit_convention():
    """Element e = m * k + kk of the mask is bit (e & 7) of byte e >> 3 (1 = kept),
    for the oracle's packer and the binding's (run here on CPU tensors)."""
    import bit_nf4_quantized_05_b200 as q
    M, K = 3, 64
    for e in (0, 1, 7, 8, 63, 64, 100, M * K - 1):
        keep = np.zeros((M, K), dtype=bool)
        keep.reshape(-1)[e] = True
        expect = np.zeros(M * K // 8, dtype=np.uint8)
        expect[e >> 3] = 1 << (e & 7)
        assert np.array_equal(oracle.pack_keep(keep), expect)
        assert np.array_equal(q.pack_keep(torch.from_numpy(keep)).numpy(), expect)


@pytest.mark.parametrize("block", [64, 128])
def test_operand_given_layer_functions_equal_the_plain_ones(block):
    """The forward and backward run on a dequantised operand formed once equal
    the functions that form it themselves, bit for bit; the operand is the
    bf16 image of the codec's dequantised weight."""
    rng = np.random.default_rng(41)
    N, K, M, r, alpha = 72, 256, 6, 16, 32.0
    qw, x, A, B, dY = random_layer(rng, N, K, M, r, True, block=block)
    Wt = oracle.dequant_operand(qw, N, K)
    assert np.array_equal(Wt.astype(np.float64), operand(qw, N, K))
    h, u = oracle.qlora_fwd_rows(qw, N, K, x, A, B, r, alpha)
    h2, u2 = oracle.qlora_fwd_rows_op(Wt, x, A, B, r, alpha)
    assert np.array_equal(h, h2) and np.array_equal(u, u2)
    g = oracle.qlora_bwd(qw, N, K, x, A, B, r, alpha, dY, dx_rows=[5, 1])
    g2 = oracle.qlora_bwd_op(Wt, x, A, B, r, alpha, dY, dx_rows=[5, 1])
    for a, b in zip(g, g2):
        assert np.array_equal(a, b)
