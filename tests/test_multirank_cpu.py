"""Host logic of the multi-GPU benchmark on CPU (gloo, world size 2): every
rank owns a different seeded sequence and the timed region is reported as
the maximum over ranks."""
import os
import socket

import numpy as np
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    import sys
    sys.path.insert(0, ROOT)
    import bench
    from workload import CONFIGS, make_hidden_states
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        got = bench.max_over_ranks(1.5 + rank, "cpu")
        X, planted = make_hidden_states(CONFIGS["tiny"], b=rank)
        out[rank] = (got, int(X[0][:4, :4].astype(np.int64).sum()), planted[1][:8].tolist())
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_ranks_report_the_max_and_own_different_sequences():
    world = 2
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.start_processes(_worker, args=(world, port, out), nprocs=world, join=True, start_method="spawn")
        res = dict(out)
    assert res[0][0] == res[1][0] == 2.5
    assert res[0][1] != res[1][1] and res[0][2] != res[1][2]


def test_single_process_max_is_identity():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.25) == 3.25


def test_reference_arm_prints_the_contract_line():
    """`bench.py --impl reference` (the oracle on the host cores) prints one
    JSON line with the arm's keys: the same metric and unit as the CUDA arm,
    impl "reference", a cpu_baseline describing the run and an e2e block with
    no host-device bytes."""
    import json
    import subprocess
    import sys
    import time
    t0 = time.time()
    out = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--config", "tiny", "--steps", "3",
                          "--warmup", "1"], capture_output=True, text=True, timeout=300,
                         cwd=os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    wall = time.time() - t0
    assert out.returncode == 0, out.stderr[-2000:]
    line = json.loads(out.stdout.strip().splitlines()[-1])
    # the steps it reports are the steps it timed: they fit in the run's wall time
    assert line["steps"] * line["ms_per_step"] / 1e3 <= wall
    assert line["requested"] == {"steps": 3, "warmup": 1}
    # the same config keys as the CUDA arm's line, with the oracle's own sets
    assert set(line["config"]) == {"workload", "l2", "parallelism", "active_tokens", "attention_pairs"}
    assert line["config"]["active_tokens"] == {"loop2": 192, "loop3": 102, "loop4": 51}
    assert line["impl"] == "reference" and line["unit"] == "tokens/s" and line["value"] > 0
    assert line["higher_is_better"] is True and line["n_gpus"] == 1 and line["steps"] == 1
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == line["value"] and cb["sample"]
    e2e = line["e2e"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0 and e2e["value"] == line["value"]


def _head_split_worker(rank, world, port, out):
    """One rank of the head-sharded partition: the gate on the replicated
    hidden states, projections, caches and attention for its own heads, and
    its partial output projection O[:, own heads] W_o[:, own heads]^T,
    summed over ranks by an all-reduce."""
    import sys
    sys.path.insert(0, ROOT)
    import torch

    import oracle as O
    from workload import CONFIGS, bf16_bits_to_f32, f32_to_bf16_bits, make_hidden_states, make_weights
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        cfg = CONFIGS["tiny"]
        W = make_weights(cfg)
        X, _ = make_hidden_states(cfg)
        per = cfg.n_heads // world
        heads = list(range(rank * per, (rank + 1) * per))
        run = O.OracleSequence(cfg, W, X, heads=heads).run()
        dh = cfg.head_dim
        cols = np.concatenate([np.arange(h * dh, (h + 1) * dh) for h in heads])
        wo = bf16_bits_to_f32(W["wo"]).astype(np.float64)[:, cols]     # this rank's input columns of W_o
        res = {}
        for r in range(1, cfg.n_loops + 1):
            act = run.active[r]
            o = bf16_bits_to_f32(run.O_hist[r][act]).astype(np.float64)  # this rank's heads only
            part = torch.from_numpy(o @ wo.T)
            dist.all_reduce(part, op=dist.ReduceOp.SUM)
            res[r] = (act.tolist(), f32_to_bf16_bits(part.numpy().astype(np.float32)).tolist())
        out[rank] = res
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_head_split_partial_outputs_sum_to_single_rank_output():
    """The head-sharded partition (SURVEY-style split: hidden states
    replicated, each rank owning half of the heads' projections, caches,
    selections and attention state, W_o split along its input columns): both
    ranks gate identically, and the all-reduced partial projections equal the
    single-rank output Y of every loop, for every active row."""
    import sys
    sys.path.insert(0, ROOT)
    import oracle as O
    from workload import CONFIGS, bf16_bits_to_f32, make_hidden_states, make_weights
    world = 2
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.start_processes(_head_split_worker, args=(world, port, out), nprocs=world, join=True,
                           start_method="spawn")
        res = dict(out)
    cfg = CONFIGS["tiny"]
    W = make_weights(cfg)
    X, _ = make_hidden_states(cfg)
    full = O.OracleSequence(cfg, W, X).run()
    for r in range(1, cfg.n_loops + 1):
        act = full.active[r]
        assert res[0][r][0] == res[1][r][0] == act.tolist()           # identical gates on both ranks
        want = bf16_bits_to_f32(full.Y_hist[r][act]).astype(np.float64)
        for rank in range(world):
            got = bf16_bits_to_f32(np.asarray(res[rank][r][1], dtype=np.uint16)).astype(np.float64)
            # the two sums differ only in the order of float64 additions: at most one bf16 step
            assert np.all(np.abs(got - want) <= 2.0 ** -7 * np.abs(want) + 1e-30), (r, rank)
            assert np.mean(got == want) > 0.99, (r, rank)
