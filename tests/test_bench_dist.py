"""Multi-process plumbing of bench.py on CPU: gloo, world size 2.

Each rank runs its own replica batch (weak scaling, no collective on the data
path); the ranks only meet at the barrier and in the max / sum of timings.
"""

import os
import socket

import pytest
import torch.multiprocessing as mp

import bench
from support import block_allocator


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    r, w = bench.init_dist("gloo", timeout_s=60)
    bench.barrier()
    # a per-rank "step time" and byte count, as the bench aggregates them
    t = bench.max_over_ranks(1.0 + r)
    b = bench.sum_over_ranks(100.0 * (r + 1))
    seed = bench.replica_seed(395, r)
    from paged_kv_cache_394_b200 import workloads as W
    wl = W.make("tiny", seed=seed)
    out.put((r, w, t, b, seed, int(wl.q.view("int16").astype("int64").sum())))
    import torch.distributed as dist
    dist.destroy_process_group()


def test_two_rank_plumbing():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = free_port()
    procs = [ctx.Process(target=worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r for r, *_ in res] == [0, 1]
    assert all(w == 2 for _, w, *_ in res)
    assert all(t == 2.0 for _, _, t, *_ in res)        # max over ranks
    assert all(x[3] == 300.0 for x in res)            # sum over ranks
    seeds = {x[4] for x in res}
    assert len(seeds) == 2                              # independent replicas
    assert res[0][5] != res[1][5]


def test_single_process_is_identity():
    assert bench.max_over_ranks(3.5) == 3.5
    assert bench.sum_over_ranks(2.0) == 2.0


def test_step_bytes_counts_kv_q_out_and_writes():
    from paged_kv_cache_394_b200 import workloads as W
    w = W.make("tiny")
    kv = 2 * int(w.context_lens.sum()) * w.num_kv_heads * w.head_dim * 2
    qo = 2 * w.num_seqs * w.num_heads * w.head_dim * 2
    assert bench.decode_bytes(w) == kv + qo
    assert bench.write_bytes(w) == 4 * len(w.slot_mapping) * w.num_kv_heads * w.head_dim * 2 \
        + 8 * len(w.slot_mapping)
    assert bench.step_bytes(w) == bench.decode_bytes(w) + bench.write_bytes(w)


def test_reference_arm_non_zero_rank_does_nothing(monkeypatch, capsys):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    bench.run_reference(bench.parse_args(["--impl", "reference", "--steps", "1"]))
    assert capsys.readouterr().out == ""


@pytest.mark.parametrize("name,unit", [("tiny", "GB/s"), ("tiny_fp8", "GB/s"),
                                       ("tiny_cascade", "GB/s"), ("gqa_prefill", "TFLOP/s"),
                                       ("gqa_prefill_fp8", "TFLOP/s")])
def test_reference_arm_prints_one_line(monkeypatch, capsys, name, unit):
    """The reference arm follows each workload's metric and unit (decode
    GB/s, prefill TFLOP/s; E4M3 over quantised codes) in a bounded sample."""
    import json
    monkeypatch.delenv("RANK", raising=False)
    monkeypatch.delenv("WORLD_SIZE", raising=False)
    bench.run_reference(bench.parse_args(["--impl", "reference", "--workload", name,
                                          "--steps", "2", "--warmup", "3",
                                          "--cpu-seconds", "0.3"]))
    lines = capsys.readouterr().out.strip().splitlines()
    assert len(lines) == 1
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["unit"] == unit and rec["value"] > 0
    assert rec["config"]["workload"] == name
    assert rec["e2e"]["h2d_bytes_per_step"] == 0 and rec["cpu_baseline"]["kind"] == "oracle"
    assert rec["ms_per_step"] < 30000


def test_reference_arm_prints_one_contract_line():
    """bench.py --impl reference (the oracle on the host cores) prints one
    JSON line with the contract's keys, on the small workload."""
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    res = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference",
                          "--workload", "tiny", "--steps", "2", "--warmup", "1",
                          "--cpu-seconds", "0.2"], capture_output=True, text=True, timeout=300)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [l for l in res.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    for k in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
              "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
              "cpu_baseline", "e2e"):
        assert k in line, k
    assert line["impl"] == "reference" and line["value"] > 0 and line["steps"] == 2
    assert line["warmup"] >= 3                      # warm-up is clamped to at least 3
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"


def _slots_read(w):
    """Every (physical block, slot) the decode reads, by brute force."""
    seen = set()
    for i, c in enumerate(w.context_lens):
        for t in range(int(c)):
            seen.add((int(w.block_tables[i, t // w.block_size]), t % w.block_size))
    return seen


@pytest.mark.parametrize("kv_elem", [2, 1])
def test_unique_bytes_count_each_shared_slot_once(kv_elem):
    from paged_kv_cache_394_b200 import workloads as W
    w = W.build_prefix_share_workload(3, 4, 37, 5, 40, 8, 2, 64, 16, "fp16", seed=5,
                                      allocator=block_allocator)
    per_slot = 2 * w.num_kv_heads * w.head_dim * kv_elem
    qo = 2 * w.num_seqs * w.num_heads * w.head_dim * 2
    assert bench.unique_decode_bytes(w, kv_elem) == len(_slots_read(w)) * per_slot + qo
    assert bench.unique_decode_bytes(w, kv_elem) < bench.decode_bytes(w, kv_elem)


def test_unique_bytes_equal_logical_without_sharing():
    from paged_kv_cache_394_b200 import workloads as W
    w = W.make("tiny")
    assert bench.unique_decode_bytes(w) == bench.decode_bytes(w)


@pytest.mark.parametrize("prompt_len,bs", [(37, 16), (64, 16), (100, 32)])
def test_cascade_groups_share_exactly_their_whole_prompt_blocks(prompt_len, bs):
    """Every member of a group has the same first shared_blocks[g] table
    entries (the prompt's whole blocks), those blocks are shared by no other
    group, and the next entry, if any, differs between members (a partial
    prompt block is copied on write; divergent tokens get fresh blocks)."""
    import numpy as np
    from paged_kv_cache_394_b200 import workloads as W
    w = W.build_prefix_share_workload(3, 4, prompt_len, 5, 40, 8, 2, 64, bs, "fp16", seed=7,
                                      allocator=block_allocator)
    gs, shared = W.cascade_groups(w)
    assert gs[0] == 0 and gs[-1] == w.num_seqs and (np.diff(gs) > 0).all()
    seen = set()
    for g in range(len(shared)):
        rows = w.block_tables[gs[g]:gs[g + 1]]
        n = int(shared[g])
        assert n == prompt_len // bs
        assert (rows[:, :n] == rows[0, :n]).all()
        assert not seen & set(rows[0, :n].tolist())
        seen |= set(rows[0, :n].tolist())
        if rows.shape[1] > n and len(rows) > 1:
            assert len(set(rows[:, n].tolist())) == len(rows)
        assert (w.context_lens[gs[g]:gs[g + 1]] >= n * bs).all()


@pytest.mark.parametrize("name", ["tiny_cascade", "no_such_workload", "llama7b_cascade"])
def test_our_arm_rejects_workloads_it_cannot_run(name):
    """Refused on the host, before any device work."""
    with pytest.raises(ValueError):
        bench.run_ours(bench.parse_args(["--workload", name]))
