"""The benchmark's host logic (CPU only): the pair counts behind its FLOP numbers, and the
multi-rank path -- barrier, max-over-ranks timing and whole-job throughput -- on two gloo ranks."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import bench


@pytest.mark.parametrize("N,causal,window", [(1, 0, 0), (7, 0, 0), (128, 1, 0), (300, 1, 7), (300, 1, 1),
                                             (300, 1, 299), (300, 1, 300), (300, 1, 5000)])
def test_visible_pairs_closed_form(N, causal, window):
    i = np.arange(N)[:, None]
    j = np.arange(N)[None, :]
    vis = np.ones((N, N), bool)
    if causal:
        vis &= j <= i
    if window > 0:
        vis &= j >= i - window + 1
    assert bench.visible_pairs(N, causal, window) == int(vis.sum())


def test_headline_flops():
    # 4 * D * N(N+1)/2 * B * Hq for the causal GQA N=8192 workload
    assert bench.prefill_flops() == 4 * 128 * (8192 * 8193 // 2) * 2 * 32


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    r, w, local = bench.dist_env()
    bench.init_dist(w, "gloo")
    bench.barrier(w)
    elapsed = 10.0 + 5.0 * r          # rank 1 is the slow one
    mx = bench.reduce_max(elapsed, w)
    value = bench.job_throughput(units_per_rank=1000.0, world=w, seconds=mx)
    out[r] = (r, w, local, mx, value)
    torch.distributed.destroy_process_group()


def test_two_gloo_ranks_take_the_max_and_sum_the_work():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    for r in range(world):
        rr, w, local, mx, value = out[r]
        assert (rr, w, local) == (r, world, r)
        assert mx == 15.0                      # slowest rank
        assert value == 1000.0 * world / 15.0  # all ranks' units over the slowest time


def test_peak_choice_follows_the_timed_region():
    """A leg timed for under a second is compared with the burst GEMM rate, a longer one with the
    sustained rate (the clocks settle under the power cap only after a while)."""
    peaks = {"bf16_tflops": 1615.5, "bf16_tflops_sustained": 1379.5, "hbm_gbs": 6559.4}
    p, kind = bench.tensor_peak_for(peaks, "measured", 0.03)
    assert p == 1615.5 and "burst" in kind
    p, kind = bench.tensor_peak_for(peaks, "measured", 2.5)
    assert p == 1379.5 and "sustained" in kind
    p, kind = bench.tensor_peak_for({"bf16_tflops": 1590.0, "hbm_gbs": 6650.0}, "fallback", 5.0)
    assert p == 1590.0


def test_reference_arm_line(capsys):
    """`--impl reference` (the fp64 oracle on the host cores) prints one JSON line with the
    contract's keys, its e2e and cpu_baseline equal to its own value, and no host<->device bytes."""
    import json
    bench.main(["--impl", "reference", "--steps", "1", "--warmup", "3"])
    lines = [ln for ln in capsys.readouterr().out.splitlines() if ln.strip()]
    assert len(lines) == 1
    line = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
                "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["n_gpus"] == 1 and line["steps"] == 1 and line["warmup"] == 3
    assert line["value"] > 0 and line["higher_is_better"] is True and line["unit"] == "TFLOP/s"
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["cpu_baseline"]["cores"] >= 1 and line["cpu_baseline"]["sample"]
    assert line["e2e"] == {"value": line["value"], "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_reference_arm_other_ranks_do_no_work():
    """Under torchrun only rank 0 runs the oracle and prints; the other ranks return at once."""
    args = bench.parse_args(["--impl", "reference", "--steps", "1", "--warmup", "3"])
    assert bench.run_reference(args, rank=1, world=2) is None
