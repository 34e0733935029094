"""The sharded scoring path on CPU: world size 2 over gloo (no GPU).

Each rank scores the layers LPT assigns it (with the oracle standing in for the GPU
kernels), the scores are all-gathered with ScoreGather, and every rank selects from the
full vector: the selection must equal the single-process one on every rank.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from quantized_lora_setup_b200.shard import ScoreGather, lpt_partition


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _scores(wl):
    import oracle
    from quantized_lora_setup_b200 import synth
    out = []
    for i, spec in enumerate(wl.layers):
        w = synth.layer_host(spec, wl.seed, i)
        out.append(oracle.layer_error(synth.bits_u16(w), oracle.F16)[2])
    return np.array(out, np.float32)


def _worker(rank, world, port, result_dir):
    import oracle
    from quantized_lora_setup_b200 import synth
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    try:
        wl = synth.tiny(0)
        parts = lpt_partition([s.numel for s in wl.layers], world)
        mine = parts[rank]
        local = []
        for i in mine:
            w = synth.layer_host(wl.layers[i], wl.seed, i)
            local.append(oracle.layer_error(synth.bits_u16(w), oracle.F16)[2])
        gather = ScoreGather(parts, rank, len(wl.layers), torch.device("cpu"))
        full = gather(torch.tensor(local, dtype=torch.float32)).numpy()
        cost = [oracle.cost_bytes(s.numel) for s in wl.layers]
        sel = oracle.select_topk(full, cost, wl.budgets[0], wl.k_cap)
        np.save(os.path.join(result_dir, f"rank{rank}.npy"),
                np.concatenate([full, np.array(sel, np.float32)]))
    finally:
        dist.destroy_process_group()


def test_lpt_partition_properties():
    sizes = [5, 3, 8, 8, 1, 7, 2, 2, 9]
    for world in (1, 2, 3, 4, 12):
        parts = lpt_partition(sizes, world)
        flat = sorted(i for p in parts for i in p)
        assert flat == list(range(len(sizes)))
        loads = [sum(sizes[i] for i in p) for p in parts]
        assert max(loads) - min(loads) <= max(sizes)
        assert parts == lpt_partition(sizes, world)  # deterministic
    with pytest.raises(ValueError):
        lpt_partition(sizes, 0)


def test_lpt_balances_a_7b_shaped_model():
    from quantized_lora_setup_b200 import synth
    wl = synth.model_7b(0)
    sizes = [s.numel for s in wl.layers]
    for world in (2, 4, 8):
        loads = [sum(sizes[i] for i in p) for p in lpt_partition(sizes, world)]
        assert max(loads) / min(loads) < 1.02


def test_two_ranks_select_like_one(tmp_path):
    from quantized_lora_setup_b200 import synth
    import oracle
    wl = synth.tiny(0)
    ref_scores = _scores(wl)
    cost = [oracle.cost_bytes(s.numel) for s in wl.layers]
    ref_sel = oracle.select_topk(ref_scores, cost, wl.budgets[0], wl.k_cap)
    port = _free_port()
    mp.start_processes(_worker, args=(2, port, str(tmp_path)), nprocs=2, join=True,
                       start_method="spawn")
    L = len(wl.layers)
    for rank in range(2):
        got = np.load(tmp_path / f"rank{rank}.npy")
        assert np.array_equal(got[:L], ref_scores)
        assert got[L:].astype(int).tolist() == ref_sel


def _duration_worker(rank, world, port, result_dir):
    """bench.py's fixed-duration loop with a per-rank chunk time (rank 1 is slower and
    uneven): the max-over-ranks collective must make both ranks take the same chunks."""
    import importlib.util
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(root, "bench.py"))
    bench = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(bench)
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    try:
        times = iter([100.0] * 50) if rank == 0 else iter([50.0, 500.0] * 25)

        def max_over_ranks(ms):
            t = torch.tensor([ms], dtype=torch.float64)
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            return float(t.item())

        chunks, total = bench.fixed_duration_chunks(lambda: next(times), max_over_ranks, 2000.0)
        np.save(os.path.join(result_dir, f"dur{rank}.npy"), np.array([chunks, total]))
    finally:
        dist.destroy_process_group()


def test_fixed_duration_loop_agrees_across_ranks(tmp_path):
    port = _free_port()
    mp.start_processes(_duration_worker, args=(2, port, str(tmp_path)), nprocs=2, join=True,
                       start_method="spawn")
    got = [np.load(tmp_path / f"dur{r}.npy").tolist() for r in range(2)]
    # per chunk max(100, 50 or 500) = 100, 500, 100, 500, ...; the running sum first
    # reaches 2000 ms at 2400 after 8 chunks
    assert got[0] == got[1] == [8.0, 2400.0]
