"""Data-parallel exchange on CPU: two gloo ranks each compute the adapter
gradients of their token shard with the oracle, sum them with the same
all-reduce the benchmark uses, and must reproduce the full-batch gradients;
after one Adam step on the summed gradients the replicas stay identical.
Also checks the max-over-ranks timing reduction and the shard split."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out_dir):
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import torch.distributed as dist

    import oracle
    import synth
    from qlora_bit_frozen_b200 import dp

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        wl = synth.workload("fp32_single_256", R=37)
        W = synth.weight(wl, 0)
        A, B = synth.adapters(wl, 0)
        X, _, dY, _ = synth.activations(wl, 0)
        w = oracle.quantize_nf4(W)
        lo, hi = dp.shard_rows(wl.R, world, rank)
        _, dA, dB = oracle.linear_bwd(w, X[lo:hi], dY[lo:hi], A, B, wl.r, wl.alpha, want_dx=False)
        gA = torch.from_numpy(dA.copy())
        gB = torch.from_numpy(dB.copy())
        dp.allreduce_adapter_grads([gA, gB])
        # the benchmark's form: every gradient in one flat arena, one collective
        flat = torch.from_numpy(np.concatenate([dA.ravel(), dB.ravel()]))
        dp.allreduce_flat(flat)
        np.save(os.path.join(out_dir, f"flat{rank}.npy"), flat.numpy())
        # every replica then takes the same Adam step on the summed gradients
        params = np.concatenate([A.ravel(), B.ravel()]).astype(np.float32)
        grads = np.concatenate([gA.numpy().ravel(), gB.numpy().ravel()]).astype(np.float32)
        zero = np.zeros_like(params)
        p1, _, _ = oracle.adam_step(params, grads, zero, zero, 1, 1e-3)
        np.save(os.path.join(out_dir, f"p{rank}.npy"), p1)
        t = dp.max_over_ranks(float(rank + 1))
        np.save(os.path.join(out_dir, f"dA{rank}.npy"), gA.numpy())
        np.save(os.path.join(out_dir, f"dB{rank}.npy"), gB.numpy())
        np.save(os.path.join(out_dir, f"t{rank}.npy"), np.array([t]))
    finally:
        dist.destroy_process_group()


def test_shard_rows_cover_everything():
    from qlora_bit_frozen_b200 import dp
    for R in (0, 1, 7, 37, 4096):
        for world in (1, 2, 3, 8):
            spans = [dp.shard_rows(R, world, k) for k in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == R
            assert all(a[1] == b[0] for a, b in zip(spans, spans[1:]))


def test_two_rank_gradient_sum_equals_full_batch(tmp_path):
    import oracle
    import synth
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    procs = [ctx.Process(target=_worker, args=(r, world, port, str(tmp_path))) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    wl = synth.workload("fp32_single_256", R=37)
    W = synth.weight(wl, 0)
    A, B = synth.adapters(wl, 0)
    X, _, dY, _ = synth.activations(wl, 0)
    _, dA, dB = oracle.linear_bwd(oracle.quantize_nf4(W), X, dY, A, B, wl.r, wl.alpha, want_dx=False)
    for r in range(world):
        gA = np.load(tmp_path / f"dA{r}.npy")
        gB = np.load(tmp_path / f"dB{r}.npy")
        assert np.allclose(gA, dA, rtol=1e-12, atol=1e-14)
        assert np.allclose(gB, dB, rtol=1e-12, atol=1e-14)
        assert float(np.load(tmp_path / f"t{r}.npy")[0]) == 2.0
        flat = np.load(tmp_path / f"flat{r}.npy")
        assert np.array_equal(flat, np.concatenate([gA.ravel(), gB.ravel()]))
    # replicas stay identical after the optimizer step, and follow the
    # full-batch step
    p0, p1 = np.load(tmp_path / "p0.npy"), np.load(tmp_path / "p1.npy")
    assert np.array_equal(p0, p1)
    params = np.concatenate([A.ravel(), B.ravel()]).astype(np.float32)
    grads = np.concatenate([dA.ravel(), dB.ravel()]).astype(np.float32)
    zero = np.zeros_like(params)
    full, _, _ = oracle.adam_step(params, grads, zero, zero, 1, 1e-3)
    assert np.allclose(p0, full, rtol=1e-9, atol=1e-9)
