"""Host-side logic of bench.py, on CPU: max-over-ranks timing with 2 gloo ranks, whole-job
aggregation, clock-sample parsing, algorithmic work counts, and the CLI guard rails."""
import os
import socket
import subprocess
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    r, w, lr = bench.dist_env()
    t = bench.reduce_max(0.25 + rank, w)          # rank 1 is the slow one
    agg = bench.aggregate(16, w, t, 10)
    q.put((r, w, lr, t, agg["value"]))
    dist.barrier()
    dist.destroy_process_group()


def test_two_rank_max_over_ranks_and_aggregate():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[0] for r in res] == [0, 1] and all(r[1] == 2 for r in res)
    assert all(r[3] == pytest.approx(1.25) for r in res)          # both see the slowest rank
    assert all(r[4] == pytest.approx(16 * 2 * 10 / 1.25) for r in res)


def test_aggregate_single_rank():
    a = bench.aggregate(16, 1, 0.5, 100)
    assert a["value"] == pytest.approx(3200.0) and a["ms_per_step"] == pytest.approx(5.0)


def test_parse_clocks():
    csv = ("index, clocks.sm [MHz], clocks.max.sm [MHz], power.draw [W], clocks_event_reasons.active,"
           " hw_slowdown, hw_thermal_slowdown, sw_thermal_slowdown, sw_power_cap\n"
           "0, 1965 MHz, 1965 MHz, 850.1 W, 0x0, Not Active, Not Active, Not Active, Not Active\n"
           "0, 1890 MHz, 1965 MHz, 998.0 W, 0x4, Not Active, Not Active, Not Active, Active\n"
           "0, 345 MHz, 1965 MHz, 120.0 W, 0x0, Not Active, Not Active, Not Active, Not Active\n")
    c = bench.parse_clocks(csv)
    assert c["sm_mhz"] == pytest.approx((1965 + 1890) / 2)
    assert c["sm_max_mhz"] == 1965 and c["reasons"] == ["sw_power_cap"]
    assert c["samples"] == 3 and c["samples_under_load"] == 2


def test_algorithmic_work_counts_only_touched_experts():
    a = bench.algorithmic(T=16, H=2880, E=32, k=4, I=2880, counts=[2] * 24 + [0] * 8)
    assert a["touched"] == 24
    assert a["gate_up_bytes"] == 24 * 2880 * 5760 * 2 + 16 * 2880 * 2 + 64 * 2880 * 2
    assert a["gate_up_flops"] == 2 * 64 * 2880 * 5760
    assert a["down_flops"] == 2 * 64 * 2880 * 2880


def test_cli_refuses_too_few_warmup_steps():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--warmup", "2"],
                       capture_output=True, text=True, timeout=120)
    assert r.returncode != 0 and "warmup" in r.stderr


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU refusal")
def test_bench_refuses_to_run_without_gpu():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--steps", "1", "--warmup", "3"],
                       capture_output=True, text=True, timeout=300)
    assert r.returncode != 0 and "CUDA" in (r.stderr + r.stdout)


def test_algorithmic_bytes_of_mxfp4_weights():
    """MXFP4 streams half a byte per weight plus one scale byte per 32 weights."""
    b = bench.algorithmic(16, 2880, 32, 4, 2880, [1] * 27, "mxfp4")
    f = bench.algorithmic(16, 2880, 32, 4, 2880, [1] * 27)
    per_expert_gu = 2880 * 5760 // 2 + 2880 // 32 * 5760
    assert b["gate_up_bytes"] - f["gate_up_bytes"] == 27 * (per_expert_gu - 2880 * 5760 * 2)
    assert b["flops"] == f["flops"]


def test_default_steps_make_the_timed_region_last_a_second():
    assert bench.steps_for(0.0204) * 0.0204 >= bench.MIN_TIMED_S          # 131K layer, ~20 ms
    assert bench.steps_for(0.0002) * 0.0002 >= bench.MIN_TIMED_S          # decode, ~0.2 ms
    assert bench.steps_for(5.0) == 10                                       # never fewer than 10
    assert bench.steps_for(1e-9) == 200000                                  # bounded


def test_cpu_baseline_runs_on_the_workloads_seeded_sample():
    import moe_inputs as mi
    w = mi.WORKLOADS["131k_skewed"]
    toks = bench.baseline_tokens(w, w.T)
    assert toks.size == w.oracle_sample == 4096
    assert np.array_equal(toks, mi.sample_tokens(w.T, 4096, w.seed))
    assert np.all(np.diff(toks) > 0) and toks[-1] < w.T
    d = mi.WORKLOADS["20b_decode"]
    assert np.array_equal(bench.baseline_tokens(d, d.T), np.arange(d.T))


def test_default_workload_is_the_largest_single_gpu_config():
    import moe_inputs as mi
    ap_default = bench.main.__code__.co_consts
    w = mi.WORKLOADS["131k_skewed"]
    assert "131k_skewed" in ap_default
    assert w.T == max(x.T for x in mi.WORKLOADS.values())


def test_peak_labels_for_measured_and_fallback_peaks():
    assert bench.peak_label("measured", "hbm_gbs") == "measured hbm_gbs (MEASURED_PEAKS.json)"
    assert bench.peak_label("fallback", "bf16_tflops (burst)").startswith("fallback bf16_tflops")
    hbm, bf16, sus, src = bench.measured_peaks()
    assert src in ("measured", "fallback") and hbm > 0 and bf16 > sus > 0


def test_family_split_follows_the_dispatch_rule():
    # a call allowed to stream: each expert by its own count, skew keeps three families when the
    # dispatch is per expert; by default the non-streamed experts take one tcgen05 family by
    # their mean count (1385 rows / 5 experts >= 128: row tiles)
    counts = [0, 3, 4, 5, 16, 17, 40, 128, 300, 900]
    f = bench.split_families(counts, "auto", 1024, 1024, 16, 128, per_expert=True)
    assert f == {"stream": [3, 4, 5, 16], "tile": [17, 40, 128], "gemm": [300, 900]}
    f = bench.split_families(counts, "auto", 1024, 1024, 16, 128)
    assert f == {"stream": [3, 4, 5, 16], "tile": [], "gemm": [17, 40, 128, 300, 900]}
    f = bench.split_families([0, 20, 30, 40, 200], "auto", 1024, 3, 16, 128)
    assert f == {"stream": [], "tile": [20, 30, 40, 200], "gemm": []}
    # larger calls do not stream; uniform counts around the boundary snap to one family
    f = bench.split_families([100, 110, 120, 130, 140], "auto", 1024, 3, 16, 128)
    assert f == {"stream": [], "tile": [100, 110, 120, 130, 140], "gemm": []}
    f = bench.split_families([120, 130, 140, 150, 160], "auto", 1024, 3, 16, 128)
    assert f == {"stream": [], "tile": [], "gemm": [120, 130, 140, 150, 160]}
    # skew across the boundary keeps the per-expert choice when asked for
    f = bench.split_families([20, 30, 40, 500, 600], "auto", 1024, 3, 16, 128, per_expert=True)
    assert f == {"stream": [], "tile": [20, 30, 40], "gemm": [500, 600]}
    f = bench.split_families([20, 30, 40, 500, 600], "auto", 1024, 3, 16, 128)
    assert f == {"stream": [], "tile": [], "gemm": [20, 30, 40, 500, 600]}
    assert bench.split_families([5, 40], "gemm", 8, 3, 16, 128) == {"stream": [], "tile": [], "gemm": [5, 40]}
    assert bench.split_families([5, 40], "auto", 16, 3, 16, 128, "mxfp4")["stream"] == [5, 40]
    assert bench.split_families([5, 40], "auto", 300, 3, 16, 128, "mxfp4")["tile"] == [5, 40]


def test_family_work_and_dominant_roofline():
    w = bench.family_work([64, 64], 2880, 2880)
    assert w["experts"] == 2 and w["rows"] == 128
    assert w["gate_up_bytes"] == 2 * 2880 * 5760 * 2 + 128 * 2880 * 2 + 128 * 2880 * 2
    assert w["gate_up_flops"] == 2 * 128 * 2880 * 5760
    work = {"stream": bench.family_work([2] * 24, 2880, 2880), "tile": w,
            "gemm": bench.family_work([4096] * 32, 2880, 2880)}
    # the tile kernel dominates and is bandwidth-bound at 64 rows per expert
    r = bench.dominant_roofline(work, {"stream": 0.05, "tile": 0.02, "gemm": 0.0}, 6548.8,
                                1661.1, 1383.9, "measured")
    assert r["family"] == "stream" and r["bound"] == "hbm"
    r = bench.dominant_roofline(work, {"stream": 0.0, "tile": 0.02, "gemm": 0.0}, 6548.8,
                                1661.1, 1383.9, "fallback")
    assert r["bound"] == "hbm" and r["achieved"] == pytest.approx(w["gate_up_bytes"] / 2e-5 / 1e9)
    assert r["kernel"] == "expert_tile_kernel<0>" and r["frac"] == pytest.approx(r["achieved"] / 6548.8)
    r = bench.dominant_roofline(work, {"stream": 0.01, "tile": 0.02, "gemm": 12.0}, 6548.8,
                                1661.1, 1383.9, "measured")
    assert r["family"] == "gemm" and r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert r["achieved"] == pytest.approx(2 * 4096 * 32 * 2880 * 5760 / 12e-3 / 1e12)


def test_traffic_lookup_matches_workload_T_and_sources():
    import json
    entries = json.load(open(bench.TRAFFIC_FILE))
    for kernel, caps in entries.items():
        for c in caps:
            for p in c["sources"]:
                assert os.path.exists(os.path.join(ROOT, p)), p
            assert os.path.exists(os.path.join(ROOT, c["capture"])), c["capture"]
            got = bench.ncu_traffic(kernel, c["workload"], c["T"])
            # a committed capture stays valid only while its kernel's sources are unchanged
            fresh = c["sources_sha"] == bench.source_digest(c["sources"])
            assert (got == c["dram_bytes_per_launch"]) if fresh else got is None
            assert bench.ncu_traffic(kernel, c["workload"], c["T"] + 1) is None
    assert bench.ncu_traffic("no_such_kernel", "tiny", 64) is None


def test_small_steps_rotate_their_input_batches():
    # field-wise means of the per-batch work, and the size below which steps rotate batches
    assert bench.mean_dicts([{"a": 1, "b": 2}, {"a": 3, "b": 6}]) == {"a": 2.0, "b": 4.0}
    l2 = 126 << 20
    one_token_120b = bench.algorithmic(1, 2880, 128, 4, 2880, [1, 1, 1, 1] + [0] * 124)
    decode_20b = bench.algorithmic(16, 2880, 32, 4, 2880, [3] * 21 + [1] * 1 + [0] * 10)
    assert one_token_120b["layer_bytes"] < bench.ROTATE_L2_FACTOR * l2 <= decode_20b["layer_bytes"]
