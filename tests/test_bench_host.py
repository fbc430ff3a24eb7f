"""Host-side logic of bench.py (CPU only): the work model, the max-over-ranks
reduction on two gloo ranks, and the reference (CPU oracle) arm."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.multiprocessing as mp

import bench
import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_selected_pairs_follow_the_topk_rule():
    x = synth.make_inputs(0)
    # min(k, s+1) distinct keys in [0, s] per row (the padding sits above s).
    assert bench.selected_pairs(x) == sum(min(32, s + 1) for s in range(128))
    x.topk_idx = torch.cat([x.topk_idx, x.topk_idx, torch.full_like(x.topk_idx, -3)], dim=-1)
    assert bench.selected_pairs(x) == sum(min(32, s + 1) for s in range(128))
    x.topk_idx = None
    assert bench.selected_pairs(x) == 128 * 129 // 2


def test_work_model_of_the_headline_workload():
    x = synth.make_inputs(0, T=4096, H=1, topk=2048)  # H=1 keeps it cheap; FLOPs scale with H
    wm = bench.work_model(x)
    assert wm["pairs"] == 6_292_480
    assert wm["flops_kvb"] == 2 * 4096 * 512 * 256
    assert wm["flops_wo"] == 2 * 4096 * 128 * 7168
    # At H=128 the three steps are 137.4 / 515.5 / 962.1 GFLOP.
    assert abs(wm["flops_kvb"] * 128 / 1e9 - 137.4) < 0.1
    assert abs(wm["flops_attn"] * 128 / 1e9 - 515.5) < 0.1
    assert abs(wm["flops_wo"] * 128 / 1e9 - 962.1) < 0.1


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench.barrier(world)
        q.put((rank, bench.max_over_ranks(1.5 + rank, world)))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_on_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs)
    got = dict(q.get(timeout=5) for _ in range(2))
    assert got == {0: 2.5, 1: 2.5}


def test_reference_arm_prints_one_line_on_rank_zero_only():
    env = dict(os.environ, RANK="0", WORLD_SIZE="1")
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--config", "0", "--steps", "3",
                        "--warmup", "1"], cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "TFLOP/s" and d["value"] > 0
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["nproc"] >= cb["cores"] and cb["cpu_model"]
    assert cb["extrapolated_full_step_s"] > 0 and "extrapolated" in cb["extrapolation"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0
    env["RANK"], env["WORLD_SIZE"] = "1", "2"
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--config", "0", "--steps", "3"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_cpu_baseline_sample_is_bounded():
    x = synth.make_inputs(0)
    d = bench.cpu_baseline(x, 0.5, 2.2e9)
    assert d["kind"] == "oracle" and d["cores"] >= 1 and d["value"] > 0
    assert d["seconds"] < 5
    assert d["nproc"] >= 1 and d["extrapolated_full_step_s"] > 0


def test_oracle_sample_credits_the_work_model():
    # Two rows of one sequence: every key either selects is up-projected once
    # per head, every selected pair costs H * 640 FLOP, every row's W_o
    # 2 * H * 128 * 7168 FLOP (the GPU line's work model).
    x = synth.make_inputs(0, B=1, T=64, H=2, topk=8, seed=9)
    rows = [10, 63]
    sets = bench.selected_sets(x, rows)
    keys = len(set(sets[0].tolist()) | set(sets[1].tolist()))
    pairs = len(sets[0]) + len(sets[1])
    assert len(sets[0]) == 8 and len(sets[1]) == 8  # s always selected, plus 7 distinct earlier keys
    dt, fl = bench.oracle_sample(x, rows, threads=2)
    assert dt > 0
    assert fl == keys * 2 * 2 * 512 * 256 + pairs * 2 * 640 + 2 * 2 * 2 * 128 * 7168


def test_step_defaults_per_mode():
    # The decode step is ~0.2 ms, so its default timed region (2000 graph
    # replays) still spans many clock samples; the other modes keep 200.
    assert bench.parse_args([]).steps == 200
    assert bench.parse_args(["--mode", "decode"]).steps == 2000
    assert bench.parse_args(["--mode", "decode", "--impl", "reference"]).steps == 200
    assert bench.parse_args(["--mode", "decode", "--steps", "7"]).steps == 7


def test_decode_selection_sets():
    # Set 0 of the decode bench's rotation is the inputs' own selection; the
    # others follow the same rule (s = T-1 plus distinct earlier positions).
    d = synth.make_decode_inputs(3, 50, 2, 16, seed=11)
    assert torch.equal(synth.decode_topk(3, 50, 16, 11), d.topk_idx)
    other = synth.decode_topk(3, 50, 16, 12)
    assert not torch.equal(other, d.topk_idx)
    for row in other:
        vals = sorted(row.tolist())
        assert len(set(vals)) == 16 and vals[-1] == 49 and vals[0] >= 0


def test_decode_reference_unit_is_the_oracle_row_per_head():
    # The decode reference arm times the oracle on (sequence, head) units laid
    # out as a compact causal problem over the selected positions; its output
    # must be the oracle's own row s = T-1 for that head, and the heads'
    # shares of W_o must add up to the row's output.
    import numpy as np
    import oracle
    x = synth.make_inputs(0, B=1, T=64, H=2, topk=16, seed=5)
    s = x.T - 1
    tk = x.topk_idx[0, s]
    sel = torch.unique(tk[(tk >= 0) & (tk <= s)])
    attn_full, out_full = oracle.prefill_rows(x, [s])
    out_sum = np.zeros_like(out_full)
    for h in range(x.H):
        y = bench.decode_unit_problem(x.q[0, s, h], x.kv_latent[0], x.k_pe[0], x.W_kvb, x.W_o, sel, h, x.scale)
        attn_y, out_y = oracle.prefill_rows(y, [y.T - 1])
        assert np.array_equal(attn_y[0, 0], attn_full[0, h])
        out_sum += out_y
    assert np.allclose(out_sum, out_full, rtol=1e-12, atol=1e-12)


def test_decode_reference_arm_prints_the_decode_metric():
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--mode", "decode", "--B", "2",
                        "--T", "200", "--H", "2", "--topk", "24", "--steps", "2", "--warmup", "0"],
                       cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "tokens/s" and d["value"] > 0
    assert d["metric"] == bench.DECODE_METRIC and d["config"]["workload"] == "decode_B2_T200"


def test_reference_arm_follows_the_activation_mode():
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--config", "4", "--act", "e4m3",
                        "--B", "1", "--T", "256", "--H", "2", "--steps", "2", "--warmup", "0"],
                       cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr
    d = json.loads(r.stdout.strip().splitlines()[-1])
    assert d["config"]["activations"] == "e4m3 dynamic 1x128" and d["config"]["weights"] == "e4m3 block-128"
    assert "e4m3 activations" in d["cpu_baseline"]["sample"] and d["value"] > 0
