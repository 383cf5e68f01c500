"""Pins for the oracle's NF4 codec: codebook, nearest level, packing, double
quantisation and dequantisation. Every check here is fixed by the pages
(golden fixtures), by closed forms, or by exact-rational brute force -- not
by re-typing the oracle's own formulas."""
from fractions import Fraction

import numpy as np
import pytest

import oracle
from conftest import read_golden_kv, read_golden_lines

LEVELS = oracle.levels()


# ---------------------------------------------------------------- codebook --
def test_levels_match_printed_16_digits():
    printed = np.array([float(v) for v in read_golden_lines("nf4_levels_16digit.txt")])
    assert printed.size == 16
    # every printed value is exactly an fp32 number
    assert np.all(printed.astype(np.float32).astype(np.float64) == printed)
    assert np.array_equal(LEVELS, printed.astype(np.float32))


def test_levels_match_4_digit_table():
    rows = [l.split() for l in read_golden_lines("nf4_levels_4digit.txt")]
    assert len(rows) == 16
    for idx, (i, binary, val) in enumerate(rows):
        assert int(i) == idx and int(binary, 2) == idx
        assert abs(float(LEVELS[idx]) - float(val)) <= 0.5e-4 + 1e-9


def test_levels_invariants():
    assert np.all(np.diff(LEVELS.astype(np.float64)) > 0)          # strictly increasing
    assert LEVELS[0] == -1.0 and LEVELS[15] == 1.0                  # normalised to [-1, 1]
    assert np.count_nonzero(LEVELS == 0.0) == 1 and LEVELS[7] == 0.0  # one exact zero
    assert np.count_nonzero(LEVELS < 0) == 7 and np.count_nonzero(LEVELS > 0) == 8


def test_levels_derived_from_normal_quantiles():
    derived = oracle.derive_levels()
    assert derived[0] == -1.0 and derived[15] == 1.0 and derived[7] == 0.0
    assert np.max(np.abs(derived - LEVELS.astype(np.float64))) < 1e-6
    # a different endpoint gives a visibly different table: the pin has teeth
    other = oracle.derive_levels(0.99)
    assert np.max(np.abs(other - LEVELS.astype(np.float64))) > 1e-3


# ------------------------------------------------------------ nearest level --
def exact_nearest(wn: np.float32) -> int:
    """argmin_j |w' - c_j| in exact rationals, ties to the lower index."""
    w = Fraction(float(wn))
    best, best_d = 0, None
    for j, c in enumerate(LEVELS):
        d = abs(w - Fraction(float(c)))
        if best_d is None or d < best_d:
            best, best_d = j, d
    return best


def midpoints():
    return [(Fraction(float(LEVELS[i])) + Fraction(float(LEVELS[i + 1]))) / 2 for i in range(15)]


def f32_neighbours(x: float, k: int = 3):
    v = np.float32(x)
    out = [v]
    lo = hi = v
    for _ in range(k):
        lo = np.nextafter(lo, np.float32(-np.inf), dtype=np.float32)
        hi = np.nextafter(hi, np.float32(np.inf), dtype=np.float32)
        out += [lo, hi]
    return out


def test_nearest_level_brute_force_at_midpoints():
    checked = 0
    for m in midpoints():
        for v in f32_neighbours(float(m), 4):
            assert oracle.nearest_level(v) == exact_nearest(v), (float(m), float(v))
            checked += 1
    assert checked == 15 * 9


def test_exact_ties_go_to_lower_index():
    exact = [i for i, m in enumerate(midpoints()) if Fraction(float(np.float32(float(m)))) == m]
    assert len(exact) >= 1
    for i in exact:
        m = np.float32(float(midpoints()[i]))
        assert oracle.nearest_level(m) == i            # lower of the two levels
        assert oracle.nearest_level(np.nextafter(m, np.float32(2))) == i + 1


def test_nearest_level_random_and_monotone():
    rng = np.random.default_rng(7)
    vals = np.sort(np.concatenate([rng.uniform(-1, 1, 3000), rng.normal(0, 0.05, 1000).clip(-1, 1)])
                   ).astype(np.float32)
    codes = [oracle.nearest_level(v) for v in vals]
    assert all(a <= b for a, b in zip(codes, codes[1:]))
    for v, c in zip(vals[::7], codes[::7]):
        assert c == exact_nearest(v)
    assert oracle.nearest_level(np.float32(1.0)) == 15
    assert oracle.nearest_level(np.float32(-1.0)) == 0
    assert oracle.nearest_level(np.float32(0.0)) == 7
    assert oracle.nearest_level(np.float32(-0.0)) == 7
    assert oracle.nearest_level(np.float32(1e-30)) == 7


# -------------------------------------------------------- worked example --
def test_worked_example_from_page():
    g = read_golden_kv("worked_example.txt")
    W = np.array([float(v) for v in g["input"].split()], dtype=np.float32).reshape(2, 3)
    q = oracle.quantize(W, block=6)
    assert q.absmax[0] == np.float32(float(g["absmax"]))
    norm = W.reshape(-1) / q.absmax[0]
    assert np.allclose(np.round(norm.astype(np.float64), 4),
                       [float(v) for v in g["normalized_4dp"].split()], atol=1e-12)
    codes = []
    for b in q.codes:
        codes += [int(b) >> 4, int(b) & 15]
    assert codes == [int(v) for v in g["codes"].split()]
    assert [int(b) for b in q.codes] == [int(v) for v in g["packed_bytes"].split()]
    assert np.allclose(np.round(LEVELS[codes].astype(np.float64), 4),
                       [float(v) for v in g["nearest_value_4dp"].split()])
    stored = q.codes.nbytes + q.absmax.nbytes
    assert W.nbytes == int(g["original_bytes"]) and stored == int(g["stored_bytes"])
    assert round(100 * (1 - stored / W.nbytes), 1) == float(g["reduction_percent"])


# ------------------------------------------------------------- quantize --
def brute_quantize(W: np.ndarray, block: int):
    """Independent quantiser: fp32 absmax and division, exact-rational argmin,
    high nibble first."""
    W = W.astype(np.float32).reshape(-1)
    codes, scales = [], []
    for b in range(W.size // block):
        blk = W[b * block:(b + 1) * block]
        s = np.float32(np.max(np.abs(blk)))
        scales.append(s)
        for w in blk:
            codes.append(7 if s == 0 else exact_nearest(np.float32(w) / s))
    packed = [(codes[2 * i] << 4) | codes[2 * i + 1] for i in range(len(codes) // 2)]
    return np.array(packed, dtype=np.uint8), np.array(scales, dtype=np.float32)


@pytest.mark.parametrize("block", [2, 4, 6, 64, 128])
def test_quantize_brute_force_tiny(block):
    rng = np.random.default_rng(block)
    W = rng.normal(0, 0.02, size=block * 12).astype(np.float32)
    # plant exact midpoints (and their neighbours) against a unit absmax
    if block >= 4:
        mids = [np.float32(float(m)) for m in midpoints()]
        W[:block] = 0
        W[0] = 1.0
        W[1:block] = (mids * block)[: block - 1]
    q = oracle.quantize(W, block=block)
    bc, bs = brute_quantize(W, block)
    assert np.array_equal(q.codes, bc)
    assert np.array_equal(q.absmax, bs)


def test_all_zero_block_and_negative_zero():
    W = np.zeros(128, dtype=np.float32)
    W[64:] = np.random.default_rng(1).normal(size=64)
    W[1] = -0.0
    q = oracle.quantize(W)
    assert q.absmax[0] == 0 and np.all(q.codes[:32] == 0x77)
    assert np.all(oracle.dequantize(q)[:64] == 0)


def test_rejects_nonfinite_and_bad_blocks():
    W = np.zeros(64, dtype=np.float32)
    W[5] = np.nan
    with pytest.raises(oracle.OracleError):
        oracle.quantize(W)
    W[5] = np.inf
    with pytest.raises(oracle.OracleError):
        oracle.quantize(W)
    with pytest.raises(oracle.OracleError):
        oracle.quantize(np.zeros(60, dtype=np.float32), block=64)
    with pytest.raises(oracle.OracleError):
        oracle.quantize(np.zeros(63, dtype=np.float32), block=63)


@pytest.mark.parametrize("block", [64, 128])
def test_dequant_of_quant_is_exact_on_codebook_multiples(block):
    rng = np.random.default_rng(3)
    for _ in range(50):
        c = np.float32(rng.uniform(1e-3, 10.0))
        js = rng.integers(0, 16, size=block)
        js[rng.integers(0, block)] = 15                 # absmax = c * 1 = c
        W = (c * LEVELS[js]).astype(np.float32)         # fl32(c * c_j)
        q = oracle.quantize(W, block=block)
        assert q.absmax[0] == c
        got = []
        for b in q.codes:
            got += [int(b) >> 4, int(b) & 15]
        assert got == list(js)
        assert np.array_equal(oracle.dequantize(q), W)


@pytest.mark.parametrize("block", [64, 128])
def test_roundtrip_error_bound(block):
    rng = np.random.default_rng(11)
    W = rng.normal(0, 0.02, size=128 * 250).astype(np.float32)
    q = oracle.quantize(W, block=block)
    wt = oracle.dequantize(q).astype(np.float64)
    half_gap = np.max(np.diff(LEVELS.astype(np.float64))) / 2     # 0.1519...
    s = np.repeat(q.absmax.astype(np.float64), block)
    err = np.abs(W.astype(np.float64) - wt)
    assert np.all(err <= s * half_gap * (1 + 1e-6))
    # NF4 error is far below the half-gap bound on average for normal data
    assert err.mean() < 0.05 * s.mean()


# ------------------------------------------------------- double quant --
def test_double_quant_storage_bits_match_page():
    g = read_golden_kv("double_quant_overhead.txt")
    N = K = 5120
    W = np.zeros(N * K, dtype=np.float32)
    q = oracle.quantize(W, dq=True)
    bits_dq = (q.q8.nbytes * 8 + q.cg.nbytes * 8) / (N * K)
    bits_fp32 = q.absmax.nbytes * 8 / (N * K)
    assert bits_fp32 == float(g["bits_per_param_fp32_scales"])
    assert round(bits_dq, 3) == float(g["bits_per_param_double_quant"])
    assert round(bits_fp32 - bits_dq, 3) == float(g["saving_bits_per_param"])
    assert q.q8.size == N * K // 64 and q.cg.size == N * K // 64 // 256


def test_double_quant_integer_closed_form():
    # group max 127 and block maxima j = 0..127: s/c*127 lands on j, so q8 = j
    # and the dequantised scale is exactly j.
    blocks = []
    for j in list(range(128)) + [127] * 128:
        b = np.zeros(64, dtype=np.float32)
        b[3] = np.float32(j)
        b[10] = -np.float32(j) / 2
        blocks.append(b)
    W = np.concatenate(blocks)
    q = oracle.quantize(W, dq=True)
    assert q.cg[0] == 127.0
    assert list(q.q8[:128]) == list(range(128))
    assert np.array_equal(oracle.block_scales(q)[:128], np.arange(128, dtype=np.float32))
    # codes are taken against the unquantised scales: same codes with and without DQ
    assert np.array_equal(q.codes, oracle.quantize(W, dq=False).codes)


def test_double_quant_properties_random():
    rng = np.random.default_rng(5)
    nb = 256 * 3 + 40                                   # partial last group
    W = (rng.normal(0, 0.02, size=(nb, 64)) * rng.uniform(0.1, 3, size=(nb, 1))).astype(np.float32)
    W[300] = 0.0                                        # a zero block
    q = oracle.quantize(W.reshape(-1), dq=True)
    ng = (nb + 255) // 256
    assert q.cg.size == ng
    for g in range(ng):
        sl = slice(g * 256, min(nb, (g + 1) * 256))
        assert q.cg[g] == q.absmax[sl].max()
        imax = g * 256 + int(np.argmax(q.absmax[sl]))
        assert q.q8[imax] == 127
        assert np.all(q.q8[sl] <= 127)
        # monotone in s within a group
        order = np.argsort(q.absmax[sl], kind="stable")
        assert np.all(np.diff(q.q8[sl][order].astype(int)) >= 0)
    assert q.q8[300] == 0
    s_hat = oracle.block_scales(q).astype(np.float64)
    bound = np.repeat(q.cg.astype(np.float64), 256)[:nb] / 254 * (1 + 1e-5)
    assert np.all(np.abs(s_hat - q.absmax.astype(np.float64)) <= bound)
    # power-of-two rescaling of one group rescales c_g and leaves q8 unchanged
    W2 = W.copy()
    W2[256:512] *= 4
    q2 = oracle.quantize(W2.reshape(-1), dq=True)
    assert q2.cg[1] == 4 * q.cg[1] and np.array_equal(q2.q8, q.q8)


def test_zero_group():
    W = np.zeros(64 * 300, dtype=np.float32)
    W[64 * 280] = 0.5
    q = oracle.quantize(W, dq=True)
    assert q.cg[0] == 0 and np.all(q.q8[:256] == 0)
    assert np.all(oracle.block_scales(q)[:256] == 0)
    assert q.cg[1] == 0.5 and q.q8[280] == 127


def test_llama13b_storage_matches_page():
    """Bytes per parameter of the stored format (codes, 8-bit scale codes and
    group constants), measured on an oracle-quantised tensor, scaled to 13e9
    parameters: the page's ~7 GB at 4-bit against 26 GB in 16 bits."""
    g = read_golden_kv("llama13b_storage.txt")
    n = float(g["params"])
    W = np.random.default_rng(13).normal(0, 0.02, size=64 * 256 * 8).astype(np.float32)
    q = oracle.quantize(W, dq=True)
    per_param = (q.codes.nbytes + q.q8.nbytes + q.cg.nbytes) / W.size
    assert per_param == 0.5 + 1 / 64 + 4 / (64 * 256)
    assert round(n * 2 / 1e9) == int(g["bf16_gb"])
    assert round(n * per_param / 1e9) == int(g["nf4_gb_approx"])       # 6.70 GB


def test_quantize_brute_force_random_blocks_and_magnitudes():
    """Random even block sizes and block magnitudes from 2^-120 to 2^120 (the
    normalisation w / s is exact-rounded at every scale) against the brute-force
    quantiser, including blocks that straddle zero with tiny elements."""
    from hypothesis import given, settings, strategies as st

    @settings(max_examples=60, deadline=None, derandomize=True)
    @given(st.integers(1, 64).map(lambda h: 2 * h), st.integers(1, 4), st.integers(-120, 120),
           st.integers(0, 2 ** 32 - 1))
    def check(block, nblocks, exp, seed):
        rng = np.random.default_rng(seed)
        W = (rng.standard_normal(block * nblocks) * 2.0 ** exp).astype(np.float32)
        W[rng.random(W.size) < 0.1] = 0.0
        q = oracle.quantize(W, block=block)
        bc, bs = brute_quantize(W, block)
        assert np.array_equal(q.codes, bc)
        assert np.array_equal(q.absmax, bs)

    check()
