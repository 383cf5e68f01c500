"""Data-parallel host logic on CPU with two gloo ranks.

Each rank takes its share of the tokens (dp.shard_rows), computes the adapter
gradients of its tokens (here with the CPU oracle, standing in for the GPU
kernels), and the flat dA+dB buffer -- fp32, the dtype the benchmark reduces --
is all-reduced (dp.allreduce_adapter_grads). The sum over ranks must equal the
gradient of the whole batch, because dA and dB are sums over tokens."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from bit_nf4_quantized_05_b200 import dp


def test_shard_rows_partition():
    for M in (0, 1, 7, 2048, 2049):
        for world in (1, 2, 3, 8):
            spans = [dp.shard_rows(M, r, world) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == M
            assert all(a[1] == b[0] for a, b in zip(spans, spans[1:]))
            sizes = [b - a for a, b in spans]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        dp.shard_rows(10, 2, 2)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, inputs, out_path):
    import oracle
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    qw, N, K, x, A, B, r, alpha, dY = inputs
    a, b = dp.shard_rows(x.shape[0], rank, world)
    _, dA, dB = oracle.qlora_bwd(qw, N, K, x[a:b], A, B, r, alpha, dY[a:b], dx_rows=[])
    # the buffer the benchmark reduces (dp.grad_buffer's default dtype), filled
    # with this rank's gradients as the backward writes them
    flat, gA, gB = dp.grad_buffer(r, K, N)
    gA.copy_(torch.from_numpy(dA))
    gB.copy_(torch.from_numpy(dB))
    dp.allreduce_adapter_grads(flat, world, average=False)
    if rank == 0:
        np.save(out_path, flat.double().numpy())
    dist.barrier()
    dist.destroy_process_group()


def test_two_rank_gradient_allreduce_equals_full_batch(tmp_path):
    import oracle
    rng = np.random.default_rng(31)
    N, K, M, r, alpha = 48, 128, 13, 8, 16.0
    W = rng.normal(0, 0.02, size=(N, K)).astype(np.float32)
    qw = oracle.quantize(W.reshape(-1), dq=True)
    bf = lambda a: oracle.f32_to_bf16(a.astype(np.float32))
    x, A = bf(rng.normal(size=(M, K))), bf(rng.uniform(-0.1, 0.1, size=(r, K)))
    B, dY = bf(rng.normal(0, 0.01, size=(N, r))), bf(rng.normal(size=(M, N)))
    out = str(tmp_path / "grads.npy")
    ctx = mp.get_context("spawn")
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(rk, 2, port, (qw, N, K, x, A, B, r, alpha, dY), out))
             for rk in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = np.load(out)
    _, dA, dB = oracle.qlora_bwd(qw, N, K, x, A, B, r, alpha, dY, dx_rows=[])
    assert dp.grad_buffer(1, 1, 1)[0].dtype == torch.float32
    # dA and dB are sums over tokens: the fp32 sum of the ranks' fp32 gradients
    # is the full batch's gradient to fp32 rounding, far inside the layer's bar
    for g, ref in ((got[: r * K], dA.reshape(-1)), (got[r * K:], dB.reshape(-1))):
        rms = np.sqrt(np.mean(ref ** 2))
        assert np.max(np.abs(g - ref)) <= 2e-2 * rms
        assert np.max(np.abs(g - ref)) <= 4 * 2.0 ** -24 * np.max(np.abs(ref)) + 1e-30


def test_grad_buffer_views_share_storage():
    flat, dA, dB = dp.grad_buffer(4, 64, 16, dtype=torch.float32)
    dA.fill_(1.0)
    dB.fill_(2.0)
    assert flat[: 4 * 64].eq(1).all() and flat[4 * 64:].eq(2).all()
    assert dp.allreduce_adapter_grads(flat, 1) is flat      # single rank: no-op
