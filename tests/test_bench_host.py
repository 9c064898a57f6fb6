"""Host-side logic of bench.py (no GPU): the max-over-ranks timing and the
whole-job aggregation on two gloo ranks, the clock-sample parser, and the
reference arm (the fp64 oracle on the host cores) on a small sequence."""

import json
import os
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _rank_main(rank, world, port, out):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    local_ms = 100.0 + 50.0 * rank  # rank 1 is the slow one
    m = bench.max_over_ranks(local_ms, world)
    out[rank] = (m, bench.aggregate(1e12, 10, world, m))
    dist.destroy_process_group()


def test_max_over_ranks_and_aggregate_two_gloo_ranks():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    port = 29500 + os.getpid() % 1000
    mp.start_processes(_rank_main, args=(world, port, out), nprocs=world, start_method="spawn", join=True)
    for r in range(world):
        m, v = out[r]
        assert m == 150.0
        # 2 ranks x 10 steps x 1 TFLOP in 150 ms
        assert v == pytest.approx(2 * 10 * 1e12 / 0.150 / 1e12)


def test_single_rank_is_identity():
    assert bench.max_over_ranks(12.5, 1) == 12.5
    assert bench.aggregate(2e12, 5, 1, 1000.0) == pytest.approx(10.0)


def test_clock_sample_parser():
    c = bench.ClockSampler(0)
    c.lines = ["0, 1800, 1965, 900.1, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
               "0, 1700, 1965, 950.0, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
               "0, 1900, 1965, 500.0, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active"]
    s = c.summary()
    assert s["sm_mhz"] == 1800 and s["sm_max_mhz"] == 1965 and s["reasons"] == ["sw_power_cap"]


def test_sample_flops_counts_visible_keys():
    from exact_attention_150_b200 import workloads
    w = workloads.LONG_CTX
    # causal: row r sees r+1 keys; 4 d flops per key forward, 3.5x with backward
    assert bench.sample_flops(w, [0, 9]) == 4.0 * w.d * (1 + 10) * 3.5


def test_reference_arm_prints_one_line():
    env = dict(os.environ, RANK="0", WORLD_SIZE="1")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--seq", "1024",
                          "--steps", "2", "--warmup", "1"], capture_output=True, text=True, env=env, timeout=600)
    assert out.returncode == 0, out.stderr
    lines = [l for l in out.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC and d["unit"] == "TFLOP/s"
    assert d["value"] > 0 and d["cpu_baseline"]["kind"] == "oracle"
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["higher_is_better"] is True


def test_reference_arm_other_ranks_exit_quietly():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--seq", "256",
                          "--steps", "1", "--warmup", "0"], capture_output=True, text=True, env=env, timeout=300)
    assert out.returncode == 0 and out.stdout.strip() == ""


def test_varlen_mix_is_seeded_and_bounded():
    import torch
    from exact_attention_150_b200 import workloads
    m = workloads.VARLEN_MIX
    a = workloads.varlen_lengths(m["seed"], m["total"], m["lo"], m["hi"])
    b = workloads.varlen_lengths(m["seed"], m["total"], m["lo"], m["hi"])
    assert a == b and sum(a) == m["total"]
    assert all(1 <= n <= m["hi"] for n in a) and all(n >= m["lo"] for n in a[:-1])
    q, k, v, do, cu = workloads.make_varlen_inputs([3, 5], 2, 8, torch.bfloat16, 7)
    assert q.shape == (2, 8, 8) and cu.tolist() == [0, 3, 8] and cu.dtype == torch.int32
    q2 = workloads.make_varlen_inputs([3, 5], 2, 8, torch.bfloat16, 7)[0]
    assert torch.equal(q, q2)


def test_add_spread_median_and_min():
    import bench

    class Ev:
        def __init__(self, t):
            self.t = t

        def elapsed_time(self, other):
            return other.t - self.t

    # three steps, events at cumulative times; kernel spans (0,1) and (1,2)
    evs = [[Ev(0.0), Ev(2.0), Ev(7.0)], [Ev(0.0), Ev(1.0), Ev(5.0)], [Ev(0.0), Ev(4.0), Ev(6.0)]]
    kernels = {"a": {"ms": 0.0}, "b": {"ms": 0.0}}
    bench.add_spread(kernels, evs, {"a": (0, 1), "b": (1, 2), "missing": (0, 2)})
    assert kernels["a"]["ms_median"] == 2.0 and kernels["a"]["ms_min"] == 1.0
    assert kernels["b"]["ms_median"] == 4.0 and kernels["b"]["ms_min"] == 2.0
    assert "missing" not in kernels
    bench.add_spread(kernels, [], {"a": (0, 1)})  # no steps: nothing added, no error


def test_sample_parity_against_the_oracle_rows():
    # The oracle's sampled rows checked against outputs made by the oracle on
    # the whole problem: zero error; a perturbed O or dQ is reported.
    import numpy as np
    import torch

    import bench
    import oracle
    from exact_attention_150_b200 import workloads
    w = workloads.Workload("t", 1, 2, 300, 64, "bf16", True, True, 77)
    q, k, v, do = workloads.make_inputs(w, with_grad=True)
    dt, fl, desc, ref = bench.oracle_sample_run(w, q, k, v, do, 100)
    f64 = lambda t: t.to(torch.float64).numpy()
    o, lse, _ = oracle.forward(f64(q), f64(k), f64(v), w.scale, True)
    dq, _, _ = oracle.backward(f64(q), f64(k), f64(v), f64(do), w.scale, True)
    o_t, lse_t, dq_t = (torch.from_numpy(np.ascontiguousarray(x)) for x in (o, lse, dq))
    good = bench.sample_parity(w, ref, o_t, lse_t, dq_t)
    assert good["within_tol"] and good["o_max_abs_err"] < 1e-9 and good["dq_rel_fro_err"] < 1e-9
    assert good["rows"] == "query rows [200,300) of head (0,0)"
    o_t[0, 0, 250, 3] += 0.5
    bad = bench.sample_parity(w, ref, o_t, lse_t, None)
    assert not bad["within_tol"] and abs(bad["o_max_abs_err"] - 0.5) < 1e-9 and "dq_rel_fro_err" not in bad
    import json
    json.dumps(bad, allow_nan=False)


def test_sample_parity_non_finite_output_stays_strict_json():
    import json

    import torch

    import bench
    from exact_attention_150_b200 import workloads
    w = workloads.Workload("t", 1, 1, 130, 64, "fp16", False, False, 78)
    q, k, v, do = workloads.make_inputs(w, with_grad=True)
    _, _, _, ref = bench.oracle_sample_run(w, q, k, v, do, 10)
    o = torch.full((1, 1, 130, 64), float("nan"))
    lse = torch.zeros(1, 1, 130)
    out = bench.sample_parity(w, ref, o, lse, None)
    assert out["o_max_abs_err"] == "non-finite" and out["within_tol"] is False
    json.dumps(out, allow_nan=False)


def test_l2_flush_rule_follows_the_input_size():
    """Workloads whose inputs fit the 126 MB L2 are timed with a flush before
    every step and say so; larger ones are not, and say that instead."""
    from exact_attention_150_b200 import workloads
    small = [workloads.TINY, workloads.SWEEP[512], workloads.SWEEP[1024], workloads.TRAIN_D64]
    large = [workloads.LONG_CTX, workloads.LAYER_7B, workloads.CAUSAL_SWEEP[4096], workloads.LONG_CTX_D256]
    for w in small:
        assert bench.needs_flush(w), w.name
        assert bench.config_of(w, 1)["l2"].startswith("flush:"), w.name
    for w in large:
        assert not bench.needs_flush(w), w.name
        assert bench.config_of(w, 1)["l2"].startswith("no flush:"), w.name
    # The rule counts the inputs one step reads: Q, K, V, and dO with a backward.
    assert bench.step_input_bytes(workloads.TRAIN_D64) == 4 * 2 * 16 * 4096 * 64 * 2
    assert bench.step_input_bytes(workloads.LAYER_7B) == 3 * 4 * 32 * 2048 * 128 * 2
