"""The Python binding checks every tensor against the shape, dtype, layout and
device its call implies before a pointer reaches the C library (which cannot
see a tensor's extent). Runs on the CPU: arguments of the right shape get as
far as the CUDA-device check, wrong ones are refused by name."""
import pytest
import torch

from conftest import build_library

N, K, M, R = 64, 128, 5, 8


@pytest.fixture(scope="module")
def q():
    build_library()
    import bit_nf4_quantized_05_b200 as mod
    return mod


def bf16(*shape):
    return torch.zeros(*shape, dtype=torch.bfloat16)


@pytest.fixture
def args(q):
    qw = q.QuantizedWeight.empty(N, K, True, "cpu")
    return dict(qw=qw, x=bf16(M, K), A=bf16(R, K), B=bf16(N, R), dY=bf16(M, N),
                keep=torch.zeros(M * K // 8, dtype=torch.uint8))


def cuda_refusal(fn, *a, **kw):
    with pytest.raises(ValueError, match="CUDA tensors"):
        fn(*a, **kw)


def shape_refusal(match, fn, *a, **kw):
    with pytest.raises(ValueError, match=match):
        fn(*a, **kw)


def test_well_formed_arguments_reach_the_device_check(q, args):
    a = args
    qw, x, A, B, dY, keep = a["qw"], a["x"], a["A"], a["B"], a["dY"], a["keep"]
    ws = torch.zeros(1024, dtype=torch.uint8)
    cuda_refusal(q.qlora_linear_fwd, qw, x, A, B, 16.0, h=bf16(M, N),
                 u=torch.zeros(M, R), workspace=ws)
    cuda_refusal(q.qlora_linear_fwd_noalloc, qw, x, A, B, 16.0)
    cuda_refusal(q.qlora_linear_bwd, qw, x, A, B, 16.0, dY, u=torch.zeros(M, R), workspace=ws,
                 outs=(bf16(M, K), bf16(R, K), bf16(N, R)))
    cuda_refusal(q.qlora_linear_bwd, qw, x, A, B, 16.0, dY, outs=(None, bf16(R, K), bf16(N, R)))
    cuda_refusal(q.qlora_linear_fwd_dropout, qw, x, A, B, 16.0, 0.1, keep, h=bf16(M, N))
    cuda_refusal(q.qlora_linear_bwd_dropout, qw, x, A, B, 16.0, 0.1, keep, dY,
                 outs=(bf16(M, K), bf16(R, K), bf16(N, R)))
    A2, B2 = bf16(2 * R, K), bf16(N, 2 * R)
    cuda_refusal(q.qlora_multi_lora_fwd, qw, x, A2, B2, R, [16.0, 8.0],
                 torch.zeros(M, dtype=torch.int32), h=bf16(M, N))
    cuda_refusal(q.qlora_merge, qw, A, B, 16.0, bf16=True, out=bf16(N, K))
    cuda_refusal(q.qlora_merge, qw, A, B, 16.0, bf16=False, out=torch.zeros(N, K))


def test_wrong_shapes_dtypes_and_layouts_are_refused(q, args):
    a = args
    qw, x, A, B, dY, keep = a["qw"], a["x"], a["A"], a["B"], a["dY"], a["keep"]
    fwd, bwd = q.qlora_linear_fwd, q.qlora_linear_bwd
    shape_refusal("x: expected shape", fwd, qw, bf16(M, K + 64), A, B, 16.0)
    shape_refusal("x: expected", fwd, qw, torch.zeros(M, K), A, B, 16.0)          # fp32 tokens
    shape_refusal("x and A must be 2-D", fwd, qw, bf16(M * K), A, B, 16.0)
    shape_refusal("A: expected shape", fwd, qw, x, bf16(R, K - 64), B, 16.0)
    shape_refusal("B: expected shape", fwd, qw, x, A, bf16(N, R + 8), 16.0)
    shape_refusal("B: expected shape", fwd, qw, x, A, bf16(R, N), 16.0)           # transposed B
    shape_refusal("B must be contiguous", fwd, qw, x, A, bf16(R, N).t(), 16.0)
    shape_refusal("h: expected shape", fwd, qw, x, A, B, 16.0, h=bf16(M, N - 8))
    shape_refusal("u: expected", fwd, qw, x, A, B, 16.0, u=bf16(M, R))            # u is fp32
    shape_refusal("workspace", fwd, qw, x, A, B, 16.0, workspace=torch.zeros(64))
    shape_refusal("dY: expected shape", bwd, qw, x, A, B, 16.0, bf16(M, N + 8))
    shape_refusal("dA: expected shape", bwd, qw, x, A, B, 16.0, dY,
                  outs=(bf16(M, K), bf16(R, K - 64), bf16(N, R)))
    shape_refusal("dX: expected shape", bwd, qw, x, A, B, 16.0, dY,
                  outs=(bf16(M + 1, K), bf16(R, K), bf16(N, R)))
    shape_refusal("keep: expected shape", q.qlora_linear_fwd_dropout, qw, x, A, B, 16.0, 0.1,
                  keep[:-1])
    shape_refusal("keep: expected", q.qlora_linear_bwd_dropout, qw, x, A, B, 16.0, 0.1,
                  keep.to(torch.int32), dY)
    shape_refusal("A_all must stack", q.qlora_multi_lora_fwd, qw, x, bf16(3 * R, K),
                  bf16(N, 2 * R), R, [16.0, 8.0], torch.zeros(M, dtype=torch.int32))
    shape_refusal("B: expected shape", q.qlora_multi_lora_fwd, qw, x, bf16(2 * R, K),
                  bf16(N, R), R, [16.0, 8.0], torch.zeros(M, dtype=torch.int32))
    shape_refusal("adapter_of_token", q.qlora_multi_lora_fwd, qw, x, bf16(2 * R, K),
                  bf16(N, 2 * R), R, [16.0, 8.0], torch.zeros(M, dtype=torch.int64))
    shape_refusal("out: expected", q.qlora_merge, qw, A, B, 16.0, bf16=True, out=torch.zeros(N, K))
    shape_refusal("A: expected shape", q.qlora_merge, qw, bf16(R, K + 64), B, 16.0)


def test_weight_arrays_are_checked(q):
    qw = q.QuantizedWeight.empty(N, K, True, "cpu")
    qw.struct()
    short = q.QuantizedWeight(N, K, True, qw.codes[:-1], qw.absmax, qw.absmax_q8, qw.absmax_c)
    shape_refusal("codes", short.struct)
    no_c = q.QuantizedWeight(N, K, True, qw.codes, qw.absmax, qw.absmax_q8, None)
    shape_refusal("absmax_c is required", no_c.struct)
    wrong = q.QuantizedWeight(N, K, False, qw.codes, qw.absmax.to(torch.float64), None, None)
    shape_refusal("absmax", wrong.struct)
    b128 = q.QuantizedWeight(N, K, False, qw.codes, qw.absmax[: N * K // 128], None, None, 128)
    b128.struct()                                       # 128-element blocks need half the scales
    shape_refusal("block_size", q.QuantizedWeight(N, K, False, qw.codes, qw.absmax, None, None, 96).struct)
    with pytest.raises(ValueError):
        q.QuantizedWeight.empty(N, K, True, "cpu", block_size=32)


def test_empty_batch_arguments_reach_the_device_check(q, args):
    qw, A, B = args["qw"], args["A"], args["B"]
    x, dY = bf16(0, K), bf16(0, N)
    keep = torch.zeros(0, dtype=torch.uint8)
    cuda_refusal(q.qlora_linear_fwd, qw, x, A, B, 16.0)
    cuda_refusal(q.qlora_linear_bwd, qw, x, A, B, 16.0, dY, u=torch.zeros(0, R),
                 outs=(bf16(0, K), bf16(R, K), bf16(N, R)))
    cuda_refusal(q.qlora_linear_fwd_dropout, qw, x, A, B, 16.0, 0.1, keep)
    cuda_refusal(q.qlora_linear_bwd_dropout, qw, x, A, B, 16.0, 0.1, keep, dY)
