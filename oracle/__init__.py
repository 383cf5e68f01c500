"""CPU oracle for the QLoRA linear layer: NF4 codec, double quantisation,
forward and backward.

TEST INFRASTRUCTURE ONLY. Only the test suite, the package entry point's smoke
check and the benchmark's CPU-baseline leg may import this package. It shares
no code with the CUDA library under ``bit_nf4_quantized_05_b200`` and imports
nothing from it.

The arithmetic lives in ``nf4_oracle.c`` (plain loops, fp32 where the pages
fix fp32, fp64 accumulation for the matmuls); this module only marshals numpy
arrays through ctypes. bf16 tensors travel as ``uint16`` arrays holding the
bf16 bit patterns.

The codebook derivation below follows the pages' description of NF4 in
"Parameter-Efficient Fine-Tuning: From LoRA to QLoRA", Pillar 1 (quantile
quantisation: each bin receives an equal expected share of a standard normal)
and "QLoRA Finetuner", section 2 (16 theoretical quantiles, normalised to
[-1, 1]); "QLoRA explained", "Common misconceptions" prints the resulting
table, which is the canonical one used everywhere else.
"""
from __future__ import annotations

import ctypes
import os
import statistics
from dataclasses import dataclass
from typing import Optional, Sequence

import numpy as np

from . import build as _build

_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        i64, i32, f64 = ctypes.c_int64, ctypes.c_int32, ctypes.c_double
        vp = ctypes.c_void_p
        L.oracle_nf4_levels.argtypes = [vp]
        L.oracle_nf4_levels.restype = None
        L.oracle_nearest_level.argtypes = [ctypes.c_float]
        L.oracle_nearest_level.restype = ctypes.c_int
        L.oracle_nf4_quantize.argtypes = [vp, i64, i32, i32, i32, vp, vp, vp, vp]
        L.oracle_nf4_quantize.restype = ctypes.c_int
        L.oracle_nf4_dequantize.argtypes = [vp, vp, vp, vp, i64, i32, i32, i32, vp]
        L.oracle_nf4_dequantize.restype = None
        L.oracle_block_scales.argtypes = [i64, vp, vp, vp, i32, i32, vp]
        L.oracle_block_scales.restype = None
        L.oracle_f32_to_bf16_array.argtypes = [vp, i64, vp]
        L.oracle_f32_to_bf16_array.restype = None
        L.oracle_qlora_fwd_rows.argtypes = [vp, vp, vp, vp, i32, i64, i64, vp, i64, vp, vp,
                                            i32, f64, vp, i64, vp, vp]
        L.oracle_qlora_fwd_rows.restype = ctypes.c_int
        L.oracle_qlora_bwd.argtypes = [vp, vp, vp, vp, i32, i64, i64, vp, i64, vp, vp, i32,
                                       f64, vp, vp, i64, vp, vp, vp]
        L.oracle_qlora_bwd.restype = ctypes.c_int
        L.oracle_philox4x32_10.argtypes = [vp, vp, vp]
        L.oracle_philox4x32_10.restype = None
        L.oracle_dropout_threshold.argtypes = [ctypes.c_float]
        L.oracle_dropout_threshold.restype = ctypes.c_uint32
        L.oracle_dropout_keep_mask.argtypes = [i64, i64, ctypes.c_float, ctypes.c_uint64,
                                               ctypes.c_uint64, vp]
        L.oracle_dropout_keep_mask.restype = None
        L.oracle_dequant_operand.argtypes = [vp, vp, vp, vp, i64, i64, i32, vp]
        L.oracle_dequant_operand.restype = None
        L.oracle_qlora_fwd_rows_op.argtypes = [vp, i64, i64, vp, i64, vp, vp, i32, f64, vp, i64,
                                               vp, vp]
        L.oracle_qlora_fwd_rows_op.restype = ctypes.c_int
        L.oracle_qlora_bwd_op.argtypes = [vp, i64, i64, vp, i64, vp, vp, i32, f64, vp, vp, i64,
                                          vp, vp, vp]
        L.oracle_qlora_bwd_op.restype = ctypes.c_int
        L.oracle_qlora_merge.argtypes = [vp, vp, vp, vp, i32, i64, i64, vp, vp, i32, f64, vp]
        L.oracle_qlora_merge.restype = ctypes.c_int
        L.oracle_qlora_multi_fwd_rows.argtypes = [vp, vp, vp, vp, i32, i64, i64, vp, i64, vp, vp,
                                                  i32, i32, vp, vp, vp, i64, vp]
        L.oracle_qlora_multi_fwd_rows.restype = ctypes.c_int
        L.oracle_qlora_fwd_rows_dropout.argtypes = [vp, vp, vp, vp, i32, i64, i64, vp, i64, vp, vp,
                                                    i32, f64, f64, vp, vp, i64, vp, vp]
        L.oracle_qlora_fwd_rows_dropout.restype = ctypes.c_int
        L.oracle_qlora_bwd_dropout.argtypes = [vp, vp, vp, vp, i32, i64, i64, vp, i64, vp, vp, i32,
                                               f64, f64, vp, vp, vp, i64, vp, vp, vp]
        L.oracle_qlora_bwd_dropout.restype = ctypes.c_int
        _lib = L
    return _lib


class OracleError(ValueError):
    pass


def _ptr(a: Optional[np.ndarray]):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


# --------------------------------------------------------------------------
# codebook
# --------------------------------------------------------------------------
def levels() -> np.ndarray:
    """The 16 canonical NF4 levels (fp32), index 0 = -1 ... index 15 = +1."""
    out = np.zeros(16, dtype=np.float32)
    lib().oracle_nf4_levels(_ptr(out))
    return out


# Endpoint probability of the quantile construction. The pages say only that
# the levels are standard-normal quantiles with equal expected mass per bin,
# normalised so the extremes are +-1, with an exact zero and more positive
# than negative levels; they never print the endpoint. This value (the mean
# of 1 - 1/(2*15) and 1 - 1/(2*16), the two half-bin offsets for 15 and 16
# levels) reproduces the printed table to fp32 rounding.
QUANTILE_ENDPOINT = 1.0 - 0.5 * (1.0 / 30.0 + 1.0 / 32.0)


def derive_levels(p: float = QUANTILE_ENDPOINT) -> np.ndarray:
    """Derive the 16 NF4 levels from standard-normal quantiles (fp64).

    8 positive levels: Phi^-1 at 8 evenly spaced probabilities from p toward
    1/2 (1/2 itself excluded); 7 negative levels: the negatives of Phi^-1 at 7
    evenly spaced probabilities from p toward 1/2; plus an exact 0. All are
    divided by Phi^-1(p) so that the extremes are exactly -1 and +1.
    """
    nd = statistics.NormalDist()

    def spaced(count: int) -> list:
        # count points from p (inclusive) toward 0.5 (exclusive)
        step = (0.5 - p) / count
        return [p + i * step for i in range(count)]

    pos = [nd.inv_cdf(q) for q in spaced(8)]
    neg = [-nd.inv_cdf(q) for q in spaced(7)]
    top = nd.inv_cdf(p)
    vals = sorted([v / top for v in pos] + [0.0] + [v / top for v in neg])
    return np.array(vals, dtype=np.float64)


def nearest_level(wn: float) -> int:
    """Index of the nearest level to one normalised fp32 value (ties -> lower)."""
    return int(lib().oracle_nearest_level(ctypes.c_float(float(np.float32(wn)))))


# --------------------------------------------------------------------------
# codec
# --------------------------------------------------------------------------
@dataclass
class Quantized:
    codes: np.ndarray            # uint8, numel/2 (element 2j -> high nibble of byte j)
    absmax: np.ndarray           # float32, numel/block
    q8: Optional[np.ndarray]     # uint8, numel/block (double quant only)
    cg: Optional[np.ndarray]     # float32, ceil(nblocks/dq_group) (double quant only)
    block: int
    dq: bool
    dq_group: int
    numel: int


def quantize(W: np.ndarray, block: int = 64, dq: bool = False, dq_group: int = 256) -> Quantized:
    """Blockwise NF4 quantisation of a float32 array (flattened row-major)."""
    W = np.ascontiguousarray(W, dtype=np.float32).reshape(-1)
    numel = W.size
    if block <= 0 or block % 2 or numel % block:
        raise OracleError(f"numel {numel} must be a multiple of an even block size {block}")
    nb = numel // block
    codes = np.zeros(numel // 2, dtype=np.uint8)
    absmax = np.zeros(nb, dtype=np.float32)
    ng = (nb + dq_group - 1) // dq_group if dq else 0
    q8 = np.zeros(nb, dtype=np.uint8) if dq else None
    cg = np.zeros(max(ng, 1), dtype=np.float32) if dq else None
    rc = lib().oracle_nf4_quantize(_ptr(W), numel, block, int(dq), dq_group, _ptr(codes),
                                   _ptr(absmax), _ptr(q8), _ptr(cg))
    if rc == 4:
        raise OracleError("non-finite value in the weight")
    if rc != 0:
        raise OracleError(f"oracle_nf4_quantize failed ({rc})")
    if dq:
        cg = cg[:ng]
    return Quantized(codes, absmax, q8, cg, block, bool(dq), dq_group, numel)


def block_scales(qw: Quantized) -> np.ndarray:
    """Scale used by dequantisation per block (s_i, or its double-quant image)."""
    nb = qw.numel // qw.block
    out = np.zeros(nb, dtype=np.float32)
    lib().oracle_block_scales(nb, _ptr(qw.absmax), _ptr(qw.q8), _ptr(qw.cg), int(qw.dq),
                              qw.dq_group, _ptr(out))
    return out


def dequantize(qw: Quantized) -> np.ndarray:
    """fp32 w~ = fl32(scale * NF4[q]) for every element (flattened)."""
    out = np.zeros(qw.numel, dtype=np.float32)
    lib().oracle_nf4_dequantize(_ptr(qw.codes), _ptr(qw.absmax), _ptr(qw.q8), _ptr(qw.cg),
                                qw.numel, qw.block, int(qw.dq), qw.dq_group, _ptr(out))
    return out


def f32_to_bf16(a: np.ndarray) -> np.ndarray:
    """Round-to-nearest-even fp32 -> bf16 bit patterns (uint16)."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    out = np.zeros(a.shape, dtype=np.uint16)
    lib().oracle_f32_to_bf16_array(_ptr(a), a.size, _ptr(out))
    return out


def bf16_to_f64(a: np.ndarray) -> np.ndarray:
    a = np.ascontiguousarray(a, dtype=np.uint16)
    return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


# --------------------------------------------------------------------------
# layer
# --------------------------------------------------------------------------
def _check_layer(qw: Quantized, N: int, K: int) -> Quantized:
    """The weight as the layer functions read it: 64-element blocks.

    The C layer functions dequantise in 64-element blocks. A 128-element block
    is handed to them as its two 64-element halves, each carrying the block's
    dequantisation scale (s, or its double-quant image) as a plain fp32
    absmax: every element then dequantises to the same fl32(scale * NF4[q])."""
    if qw.block not in (64, 128) or qw.dq_group != 256 or qw.numel != N * K or K % qw.block:
        raise OracleError("layer oracle expects blocks of 64 or 128, groups of 256 and K % block == 0")
    if qw.block == 64:
        return qw
    halves = np.repeat(block_scales(qw), qw.block // 64).astype(np.float32)
    return Quantized(qw.codes, halves, None, None, 64, False, 256, qw.numel)


def qlora_fwd_rows(qw: Quantized, N: int, K: int, x: np.ndarray, A: np.ndarray, B: np.ndarray,
                   r: int, alpha: float, rows: Optional[Sequence[int]] = None):
    """h rows (fp64) and u rows (fp64) of h = x W~^T + (alpha/r)(x A^T) B^T.

    x: uint16 [M, K] bf16 bits; A: uint16 [r, K]; B: uint16 [N, r].
    rows: token indices to compute (default: all)."""
    qw = _check_layer(qw, N, K)
    x = np.ascontiguousarray(x, dtype=np.uint16)
    A = np.ascontiguousarray(A, dtype=np.uint16)
    B = np.ascontiguousarray(B, dtype=np.uint16)
    M = x.shape[0]
    assert x.shape == (M, K) and A.shape == (r, K) and B.shape == (N, r)
    rows = np.arange(M, dtype=np.int64) if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    h = np.zeros((rows.size, N), dtype=np.float64)
    u = np.zeros((rows.size, r), dtype=np.float64)
    rc = lib().oracle_qlora_fwd_rows(_ptr(qw.codes), _ptr(qw.absmax), _ptr(qw.q8), _ptr(qw.cg),
                                     int(qw.dq), N, K, _ptr(x), M, _ptr(A), _ptr(B), r,
                                     float(alpha), _ptr(rows), rows.size, _ptr(h), _ptr(u))
    if rc != 0:
        raise OracleError(f"oracle_qlora_fwd_rows failed ({rc})")
    return h, u


def qlora_bwd(qw: Quantized, N: int, K: int, x: np.ndarray, A: np.ndarray, B: np.ndarray,
              r: int, alpha: float, dY: np.ndarray, dx_rows: Optional[Sequence[int]] = None,
              want_dA: bool = True, want_dB: bool = True):
    """(dX rows, dA, dB) in fp64 for the layer's backward; W0 gets no gradient.

    dY: uint16 [M, N] bf16 bits. dx_rows: token rows of dX to compute
    (default: all; an empty list skips dX)."""
    qw = _check_layer(qw, N, K)
    x = np.ascontiguousarray(x, dtype=np.uint16)
    A = np.ascontiguousarray(A, dtype=np.uint16)
    B = np.ascontiguousarray(B, dtype=np.uint16)
    dY = np.ascontiguousarray(dY, dtype=np.uint16)
    M = x.shape[0]
    assert dY.shape == (M, N)
    rows = np.arange(M, dtype=np.int64) if dx_rows is None else np.ascontiguousarray(dx_rows, dtype=np.int64)
    dX = np.zeros((rows.size, K), dtype=np.float64)
    dA = np.zeros((r, K), dtype=np.float64) if want_dA else None
    dB = np.zeros((N, r), dtype=np.float64) if want_dB else None
    rc = lib().oracle_qlora_bwd(_ptr(qw.codes), _ptr(qw.absmax), _ptr(qw.q8), _ptr(qw.cg),
                                int(qw.dq), N, K, _ptr(x), M, _ptr(A), _ptr(B), r, float(alpha),
                                _ptr(dY), _ptr(rows), rows.size, _ptr(dX) if rows.size else None,
                                _ptr(dA), _ptr(dB))
    if rc != 0:
        raise OracleError(f"oracle_qlora_bwd failed ({rc})")
    return dX, dA, dB


def dequant_operand(qw: Quantized, N: int, K: int) -> np.ndarray:
    """The bf16 matmul operand RNE_bf16(fl32(scale * NF4[q])) of the whole
    weight, as fp32 [N, K] (reading R6). The layer functions form it on every
    call; forming it once lets a caller run many batches through one frozen
    weight (the *_op functions below)."""
    qw = _check_layer(qw, N, K)
    out = np.zeros((N, K), dtype=np.float32)
    lib().oracle_dequant_operand(_ptr(qw.codes), _ptr(qw.absmax), _ptr(qw.q8), _ptr(qw.cg),
                                 N, K, int(qw.dq), _ptr(out))
    return out


def qlora_fwd_rows_op(Wt: np.ndarray, x: np.ndarray, A: np.ndarray, B: np.ndarray, r: int,
                      alpha: float, rows: Optional[Sequence[int]] = None):
    """qlora_fwd_rows with the dequantised operand Wt [N, K] given."""
    Wt = np.ascontiguousarray(Wt, dtype=np.float32)
    N, K = Wt.shape
    x = np.ascontiguousarray(x, dtype=np.uint16)
    A = np.ascontiguousarray(A, dtype=np.uint16)
    B = np.ascontiguousarray(B, dtype=np.uint16)
    M = x.shape[0]
    assert x.shape == (M, K) and A.shape == (r, K) and B.shape == (N, r)
    rows = np.arange(M, dtype=np.int64) if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    h = np.zeros((rows.size, N), dtype=np.float64)
    u = np.zeros((rows.size, r), dtype=np.float64)
    rc = lib().oracle_qlora_fwd_rows_op(_ptr(Wt), N, K, _ptr(x), M, _ptr(A), _ptr(B), r,
                                        float(alpha), _ptr(rows), rows.size, _ptr(h), _ptr(u))
    if rc != 0:
        raise OracleError(f"oracle_qlora_fwd_rows_op failed ({rc})")
    return h, u


def qlora_bwd_op(Wt: np.ndarray, x: np.ndarray, A: np.ndarray, B: np.ndarray, r: int,
                 alpha: float, dY: np.ndarray, dx_rows: Optional[Sequence[int]] = None):
    """qlora_bwd with the dequantised operand Wt [N, K] given."""
    Wt = np.ascontiguousarray(Wt, dtype=np.float32)
    N, K = Wt.shape
    x = np.ascontiguousarray(x, dtype=np.uint16)
    A = np.ascontiguousarray(A, dtype=np.uint16)
    B = np.ascontiguousarray(B, dtype=np.uint16)
    dY = np.ascontiguousarray(dY, dtype=np.uint16)
    M = x.shape[0]
    assert dY.shape == (M, N)
    rows = np.arange(M, dtype=np.int64) if dx_rows is None else np.ascontiguousarray(dx_rows, dtype=np.int64)
    dX = np.zeros((rows.size, K), dtype=np.float64)
    dA = np.zeros((r, K), dtype=np.float64)
    dB = np.zeros((N, r), dtype=np.float64)
    rc = lib().oracle_qlora_bwd_op(_ptr(Wt), N, K, _ptr(x), M, _ptr(A), _ptr(B), r, float(alpha),
                                   _ptr(dY), _ptr(rows), rows.size, _ptr(dX) if rows.size else None,
                                   _ptr(dA), _ptr(dB))
    if rc != 0:
        raise OracleError(f"oracle_qlora_bwd_op failed ({rc})")
    return dX, dA, dB


def qlora_merge(qw: Quantized, N: int, K: int, A: np.ndarray, B: np.ndarray, r: int,
                alpha: float) -> np.ndarray:
    """W~ + (alpha/r) B A in fp64, [N, K]: the adapters folded into the dequantised
    (fp32) base weight, as for inference without adapters.

    A: uint16 [r, K] bf16 bits; B: uint16 [N, r]."""
    qw = _check_layer(qw, N, K)
    A = np.ascontiguousarray(A, dtype=np.uint16)
    B = np.ascontiguousarray(B, dtype=np.uint16)
    assert A.shape == (r, K) and B.shape == (N, r)
    out = np.zeros((N, K), dtype=np.float64)
    rc = lib().oracle_qlora_merge(_ptr(qw.codes), _ptr(qw.absmax), _ptr(qw.q8), _ptr(qw.cg),
                                  int(qw.dq), N, K, _ptr(A), _ptr(B), r, float(alpha), _ptr(out))
    if rc != 0:
        raise OracleError(f"oracle_qlora_merge failed ({rc})")
    return out


def qlora_multi_fwd_rows(qw: Quantized, N: int, K: int, x: np.ndarray, A_all: np.ndarray,
                         B_all: np.ndarray, r: int, alphas: Sequence[float], adapter: np.ndarray,
                         rows: Optional[Sequence[int]] = None) -> np.ndarray:
    """h rows (fp64) of one NF4 base with per-token adapters:
    h[m] = x[m] W~^T + (alpha_a / r)(x[m] A_a^T) B_a^T for a = adapter[m] (none when < 0).

    A_all: uint16 [n_ad * r, K] (stacked A_a); B_all: uint16 [N, n_ad * r] (stacked B_a);
    adapter: int32 [M]."""
    qw = _check_layer(qw, N, K)
    x = np.ascontiguousarray(x, dtype=np.uint16)
    A_all = np.ascontiguousarray(A_all, dtype=np.uint16)
    B_all = np.ascontiguousarray(B_all, dtype=np.uint16)
    n_ad = len(alphas)
    M = x.shape[0]
    assert A_all.shape == (n_ad * r, K) and B_all.shape == (N, n_ad * r)
    adapter = np.ascontiguousarray(adapter, dtype=np.int32)
    assert adapter.shape == (M,)
    al = np.ascontiguousarray(alphas, dtype=np.float64)
    rows = np.arange(M, dtype=np.int64) if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    h = np.zeros((rows.size, N), dtype=np.float64)
    rc = lib().oracle_qlora_multi_fwd_rows(_ptr(qw.codes), _ptr(qw.absmax), _ptr(qw.q8),
                                           _ptr(qw.cg), int(qw.dq), N, K, _ptr(x), M, _ptr(A_all),
                                           _ptr(B_all), r, n_ad, _ptr(al), _ptr(adapter),
                                           _ptr(rows), rows.size, _ptr(h))
    if rc != 0:
        raise OracleError(f"oracle_qlora_multi_fwd_rows failed ({rc})")
    return h


def qlora_fwd_rows_dropout(qw: Quantized, N: int, K: int, x: np.ndarray, A: np.ndarray,
                           B: np.ndarray, r: int, alpha: float, p: float, keep: np.ndarray,
                           rows: Optional[Sequence[int]] = None):
    """(h rows, u rows) in fp64 with dropout on the LoRA input:
    u = (keep . x) A^T, h = x W~^T + (alpha/r)/(1-p) u B^T.

    keep: uint8 bit mask over x, bit (e & 7) of byte e >> 3 for e = m K + k (1 = kept)."""
    qw = _check_layer(qw, N, K)
    x = np.ascontiguousarray(x, dtype=np.uint16)
    A = np.ascontiguousarray(A, dtype=np.uint16)
    B = np.ascontiguousarray(B, dtype=np.uint16)
    keep = np.ascontiguousarray(keep, dtype=np.uint8)
    M = x.shape[0]
    assert keep.size == M * K // 8
    rows = np.arange(M, dtype=np.int64) if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    h = np.zeros((rows.size, N), dtype=np.float64)
    u = np.zeros((rows.size, r), dtype=np.float64)
    rc = lib().oracle_qlora_fwd_rows_dropout(_ptr(qw.codes), _ptr(qw.absmax), _ptr(qw.q8),
                                             _ptr(qw.cg), int(qw.dq), N, K, _ptr(x), M, _ptr(A),
                                             _ptr(B), r, float(alpha), float(p), _ptr(keep),
                                             _ptr(rows), rows.size, _ptr(h), _ptr(u))
    if rc != 0:
        raise OracleError(f"oracle_qlora_fwd_rows_dropout failed ({rc})")
    return h, u


def qlora_bwd_dropout(qw: Quantized, N: int, K: int, x: np.ndarray, A: np.ndarray, B: np.ndarray,
                      r: int, alpha: float, p: float, keep: np.ndarray, dY: np.ndarray,
                      dx_rows: Optional[Sequence[int]] = None):
    """(dX rows, dA, dB) in fp64 with dropout on the LoRA input (same mask convention)."""
    qw = _check_layer(qw, N, K)
    x = np.ascontiguousarray(x, dtype=np.uint16)
    A = np.ascontiguousarray(A, dtype=np.uint16)
    B = np.ascontiguousarray(B, dtype=np.uint16)
    dY = np.ascontiguousarray(dY, dtype=np.uint16)
    keep = np.ascontiguousarray(keep, dtype=np.uint8)
    M = x.shape[0]
    assert keep.size == M * K // 8 and dY.shape == (M, N)
    rows = np.arange(M, dtype=np.int64) if dx_rows is None else np.ascontiguousarray(dx_rows, dtype=np.int64)
    dX = np.zeros((rows.size, K), dtype=np.float64)
    dA = np.zeros((r, K), dtype=np.float64)
    dB = np.zeros((N, r), dtype=np.float64)
    rc = lib().oracle_qlora_bwd_dropout(_ptr(qw.codes), _ptr(qw.absmax), _ptr(qw.q8), _ptr(qw.cg),
                                        int(qw.dq), N, K, _ptr(x), M, _ptr(A), _ptr(B), r,
                                        float(alpha), float(p), _ptr(keep), _ptr(dY), _ptr(rows),
                                        rows.size, _ptr(dX) if rows.size else None, _ptr(dA), _ptr(dB))
    if rc != 0:
        raise OracleError(f"oracle_qlora_bwd_dropout failed ({rc})")
    return dX, dA, dB


def pack_keep(keep_bool: np.ndarray) -> np.ndarray:
    """Bit mask (uint8, bit e & 7 of byte e >> 3) of a boolean keep array, row-major."""
    return np.packbits(np.ascontiguousarray(keep_bool, dtype=bool).reshape(-1), bitorder="little")


# --------------------------------------------------------------------------
# dropout mask drawn from Philox4x32-10 (counter-based; regenerated, not stored)
# --------------------------------------------------------------------------
def philox4x32_10(counter: Sequence[int], key: Sequence[int]) -> np.ndarray:
    """The four 32-bit outputs of Philox4x32-10 for one counter and key."""
    c = np.ascontiguousarray(counter, dtype=np.uint32)
    k = np.ascontiguousarray(key, dtype=np.uint32)
    assert c.size == 4 and k.size == 2
    out = np.zeros(4, dtype=np.uint32)
    lib().oracle_philox4x32_10(_ptr(c), _ptr(k), _ptr(out))
    return out


def dropout_threshold(p: float) -> int:
    """floor(p * 2^32) for an fp32 p: elements whose draw is below it are dropped."""
    return int(lib().oracle_dropout_threshold(ctypes.c_float(float(np.float32(p)))))


def dropout_keep_mask(M: int, K: int, p: float, seed: int, offset: int) -> np.ndarray:
    """Keep bit mask (pack_keep's convention) of x [M, K] drawn for (seed, offset):
    element e = m K + k is kept when word e mod 4 of Philox4x32-10 at counter
    (e div 4 as two 32-bit halves, offset as two halves), key (seed halves) is at
    least dropout_threshold(p)."""
    out = np.zeros((M * K + 7) // 8, dtype=np.uint8)
    lib().oracle_dropout_keep_mask(M, K, ctypes.c_float(float(np.float32(p))), int(seed) & (2 ** 64 - 1),
                                   int(offset) & (2 ** 64 - 1), _ptr(out))
    return out
