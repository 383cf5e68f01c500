"""Pins for the oracle's LoRA-dropout draw ("QLoRA Finetuner -- Juan Martos",
section 1: dropout on the adapter input; "QLoRA explained", the recipe's
lora_dropout = 0.05). The pages fix no generator; the reading is the
counter-based Philox4x32-10 (Salmon et al., SC'11), one 32-bit word per
element of x, so that the backward regenerates the forward's mask from
(seed, offset). Pinned here: the generator against its published
known-answer vectors, the drop threshold against exact arithmetic, the
element -> (counter, word) mapping against the generator called element by
element, and the statistics of the mask (binomial bounds)."""
from fractions import Fraction

import numpy as np
import pytest

import oracle
from conftest import read_golden_lines


def test_philox_known_answer_vectors():
    rows = read_golden_lines("philox4x32_10_kat.txt")
    assert len(rows) == 3
    for row in rows:
        ctr, key, out = (list(int(v, 16) for v in part.split()) for part in row.split("|"))
        got = oracle.philox4x32_10(ctr, key)
        assert [int(v) for v in got] == out, row


def test_threshold_is_floor_of_p_times_2_32():
    for p in (0.0, 0.05, 0.1, 0.3, 0.5, 0.999, 1e-9, np.nextafter(np.float32(1), np.float32(0))):
        p32 = np.float32(p)
        want = int(Fraction(float(p32)) * 2 ** 32)          # floor of the exact product
        assert oracle.dropout_threshold(p32) == want, p
    assert oracle.dropout_threshold(0.5) == 2 ** 31


def test_mask_mapping_element_by_element():
    rng = np.random.default_rng(5)
    M, K, p = 3, 192, np.float32(0.3)
    seed, offset = 0x0123456789ABCDEF, 0xFEDCBA9876543210
    mask = oracle.dropout_keep_mask(M, K, p, seed, offset)
    t = oracle.dropout_threshold(p)
    key = [seed & 0xFFFFFFFF, seed >> 32]
    for e in rng.choice(M * K, size=80, replace=False):
        g = int(e) // 4
        w = oracle.philox4x32_10([g & 0xFFFFFFFF, g >> 32, offset & 0xFFFFFFFF, offset >> 32], key)
        kept = int(w[int(e) % 4]) >= t
        assert ((int(mask[e >> 3]) >> (int(e) & 7)) & 1) == int(kept), int(e)


def test_mask_statistics_and_special_cases():
    M, K = 256, 5120
    assert np.all(oracle.dropout_keep_mask(M, K, 0.0, 1, 0) == 0xFF)        # p = 0 keeps all
    for p in (0.05, 0.3):
        bits = np.unpackbits(oracle.dropout_keep_mask(M, K, p, 1234, 0), bitorder="little")
        n = M * K
        kept = int(bits.sum())
        mean, sd = n * (1 - p), np.sqrt(n * p * (1 - p))
        assert abs(kept - mean) < 6 * sd, (p, kept, mean)
        # rows and columns are not biased: per-column keep rate within bounds
        cols = bits.reshape(M, K).mean(axis=0)
        assert abs(cols.mean() - (1 - p)) < 6 * np.sqrt(p * (1 - p) / n)
    # a new offset gives a different mask (about 2 p (1 - p) of the bits differ)
    a = np.unpackbits(oracle.dropout_keep_mask(M, K, 0.3, 1234, 0), bitorder="little")
    b = np.unpackbits(oracle.dropout_keep_mask(M, K, 0.3, 1234, 1), bitorder="little")
    c = np.unpackbits(oracle.dropout_keep_mask(M, K, 0.3, 1235, 0), bitorder="little")
    for other in (b, c):
        frac = float(np.mean(a != other))
        assert abs(frac - 2 * 0.3 * 0.7) < 0.01
    # the same (seed, offset) gives the same mask, and a shorter x is a prefix
    assert np.array_equal(oracle.dropout_keep_mask(M, K, 0.3, 1234, 0),
                          np.packbits(a, bitorder="little"))
    assert np.array_equal(oracle.dropout_keep_mask(10, K, 0.3, 1234, 0),
                          oracle.dropout_keep_mask(M, K, 0.3, 1234, 0)[: 10 * K // 8])
