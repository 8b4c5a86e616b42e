"""Data-parallel decomposition of the QLoRA linear layer on CPU (gloo, world size 2).

Each rank holds the same frozen quantized weight and adapters and a disjoint
shard of the token rows.  The LoRA gradients are sums over tokens, so the
all-reduce (sum) of the per-shard gradients must equal the full-batch
gradient; dX needs no exchange (it is per token).  This is the exchange that
bench.py performs with NCCL for --gpus N > 1.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import synthetic_inputs as si
from oracle import nf4_oracle as o

WORLD = 2
M, N, K, R, ALPHA = 24, 64, 128, 4, 8.0


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _problem():
    W, X, A, B, dY = si.custom_linear(N, K, M, R, seed=41)
    qw = o.quantize_nf4_dq(si.bf16_bits(W))
    Wh = o.dequantize(qw["codes"], qw["c1_codes"], qw["c2"], qw["mu"], N, K)
    return Wh, si.bf16_bits(X), si.bf16_bits(A), si.bf16_bits(B), si.bf16_bits(dY)


def _worker(rank, port, out_path):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=WORLD)
    Wh, X, A, B, dY = _problem()
    rows = np.array_split(np.arange(M), WORLD)[rank]
    g = o.linear_backward(X[rows], dY[rows], Wh, A, B, ALPHA, R)
    flat = torch.from_numpy(np.concatenate([g["dA"].ravel(), g["dB"].ravel()]))
    dist.all_reduce(flat)
    if rank == 0:
        np.save(out_path, flat.numpy())
    dist.barrier()
    dist.destroy_process_group()


def test_sharded_lora_gradients_all_reduce_to_full_batch(tmp_path):
    out = str(tmp_path / "reduced.npy")
    mp.spawn(_worker, args=(_free_port(), out), nprocs=WORLD, join=True)
    reduced = np.load(out)
    Wh, X, A, B, dY = _problem()
    g = o.linear_backward(X, dY, Wh, A, B, ALPHA, R)
    full = np.concatenate([g["dA"].ravel(), g["dB"].ravel()])
    assert np.allclose(reduced, full, rtol=1e-12, atol=1e-12)


# A multi-linear workload shaped like the decoder block (square, wide and tall linears; gate and
# up share their input), small enough for the oracle: the flat gradient buffer of bench.py.
BLOCK = si.Workload("dp_block", ((64, 64), (64, 64), (192, 64), (192, 64), (64, 192)), 24, 4, 8.0,
                    dist="t5_outliers")


def _block_problem():
    lins = []
    for i, (n, k) in enumerate(BLOCK.linears):
        qw = o.quantize_nf4_dq(si.bf16_bits(si.weight(BLOCK, i)))
        Wh = o.dequantize(qw["codes"], qw["c1_codes"], qw["c2"], qw["mu"], n, k)
        A, B = (si.bf16_bits(t) for t in si.lora(BLOCK, i))
        X = si.bf16_bits(si.activations(BLOCK, k, BLOCK.M))
        dY = si.bf16_bits(si.grad_output(BLOCK, i, BLOCK.M))
        lins.append((Wh, X, A, B, dY))
    return lins


def _block_worker(rank, port, out_path):
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=WORLD)
    rows = np.array_split(np.arange(BLOCK.M), WORLD)[rank]
    grads = torch.full((bench.grad_buffer_numel(BLOCK),), float("nan"), dtype=torch.float64)
    for (Wh, X, A, B, dY), (dA, dB) in zip(_block_problem(), bench.grad_views(BLOCK, grads)):
        g = o.linear_backward(X[rows], dY[rows], Wh, A, B, BLOCK.alpha, BLOCK.r)
        dA.copy_(torch.from_numpy(g["dA"]))
        dB.copy_(torch.from_numpy(g["dB"]))
    dist.all_reduce(grads)                      # the one collective of a data-parallel step
    if rank == 0:
        np.save(out_path, grads.numpy())
    dist.barrier()
    dist.destroy_process_group()


def test_bench_gradient_buffer_all_reduces_to_every_linears_full_batch_gradients(tmp_path):
    import bench
    out = str(tmp_path / "grads.npy")
    mp.spawn(_block_worker, args=(_free_port(), out), nprocs=WORLD, join=True)
    reduced = torch.from_numpy(np.load(out))
    assert torch.isfinite(reduced).all()           # every element of the buffer belongs to a view
    views = bench.grad_views(BLOCK, reduced)
    assert len(views) == len(BLOCK.linears)
    for (Wh, X, A, B, dY), (dA, dB) in zip(_block_problem(), views):
        g = o.linear_backward(X, dY, Wh, A, B, BLOCK.alpha, BLOCK.r)
        assert dA.shape == g["dA"].shape and dB.shape == g["dB"].shape
        assert np.allclose(dA.numpy(), g["dA"], rtol=1e-12, atol=1e-12)
        assert np.allclose(dB.numpy(), g["dB"], rtol=1e-12, atol=1e-12)


def test_weak_scaling_accounting():
    import bench
    wl = si.WORKLOADS["block65b"]
    per_rank = bench.step_flops(wl, wl.M)
    # fwd 2MNK + 2Mr(N+K) and bwd 2MNK + 4Mr(N+K) per linear
    expect = sum(4 * wl.M * n * k + 6 * wl.M * wl.r * (n + k) for n, k in wl.linears)
    assert per_rank == expect
