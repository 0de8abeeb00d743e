"""Host-side logic of bench.py, on CPU: the reference arm's JSON line, the
silent non-zero ranks, and the max-over-ranks / whole-job aggregation of the
multi-GPU replicas exercised over a world-size-2 gloo group, and the rule that
roofline.traffic is reported only for the sources it was captured on."""
import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _bench(args, env_extra=None):
    env = dict(os.environ)
    env.update(env_extra or {})
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], capture_output=True, text=True,
                          env=env, timeout=300)


def test_reference_arm_prints_the_contract_line():
    r = _bench(["--impl", "reference", "--workload", "t2b_f32_b1c4_16x16", "--steps", "2", "--warmup", "1",
                "--cpu-seconds", "0.5"])
    assert r.returncode == 0, r.stderr
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
              "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert k in d, k
    assert d["impl"] == "reference" and d["steps"] == 2 and d["warmup"] == 1
    assert d["config"]["workload"] == "t2b_f32_b1c4_16x16"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"] > 0
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_block_reference_arm_prints_the_contract_line():
    r = _bench(["--impl", "reference", "--workload", "block_cp2_bf16_b32c1152_64x64", "--batch", "1", "--steps",
                "1", "--warmup", "0", "--cpu-seconds", "0.2"])
    assert r.returncode == 0, r.stderr
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["config"]["C_proxy"] == 2 and d["value"] > 0
    assert d["cpu_baseline"]["value"] == d["value"]


def test_block_bytes_count_x_y_and_the_proxy_inputs():
    import bench
    import synth
    w = synth.BlockWorkload("b", 2, 16, 8, 8, 4, 1, 0)
    n = 2 * 16 * 64
    want = 2 * n * 2 + 4 * 2 * 4 * 64 * 2 + 4 * 2 * 3 * 64 * 2 + 2 * 16 * 4 * 2 + 5 * 4 * 4
    assert bench.block_bytes(w) == want


def test_reference_arm_other_ranks_exit_without_work():
    r = _bench(["--impl", "reference", "--workload", "t2b_f32_b1c4_16x16", "--steps", "1"],
               {"RANK": "1", "WORLD_SIZE": "2"})
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_job_value_counts_every_rank_over_the_slowest_time():
    import bench
    assert bench.job_gbs(2_000_000_000, 1, 1000.0) == pytest.approx(2.0)
    assert bench.job_gbs(2_000_000_000, 4, 2000.0) == pytest.approx(4.0)
    assert bench.max_over_ranks(None, 3.5, "cpu") == 3.5


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    import datetime

    import torch.distributed as dist

    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        local_ms = [7.0, 11.0][rank]
        ms = bench.max_over_ranks(dist, local_ms, "cpu")
        q.put((rank, ms, bench.job_gbs(1_000_000_000, world, ms)))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_max_over_ranks_with_two_gloo_ranks():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    ps = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in ps:
        p.start()
    for p in ps:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in ps)
    res = sorted(q.get(timeout=5) for _ in range(2))
    for rank, ms, gbs in res:
        assert ms == 11.0                       # every rank sees the slowest rank's time
        assert gbs == pytest.approx(2 * 1_000_000_000 / 11e-3 / 1e9)  # both ranks' bytes


def test_roofline_traffic_only_for_the_sources_it_was_captured_on(monkeypatch):
    """roofline.traffic comes from the committed ncu capture only while the
    dominant kernel's sources hash to the value stored with it; any source
    change turns it into null until a new capture is committed."""
    import bench
    import synth
    w = synth.WORKLOADS["compact_4dir_bf16_b32c1152_64x64"]
    with open(os.path.join(ROOT, "profiles", "ncu_traffic.json")) as f:
        stored = json.load(f)[w.name]
    for kernel_pass in ("fwd", "bwd"):
        ent = stored[kernel_pass]
        assert ent["dram_bytes_per_launch"] > 0
        monkeypatch.setattr(bench, "csrc_hash", lambda p, h=ent["csrc_hash"]: h)
        assert bench.ncu_traffic(kernel_pass, w) == ent["dram_bytes_per_launch"]
        monkeypatch.setattr(bench, "csrc_hash", lambda p: "0" * 16)
        assert bench.ncu_traffic(kernel_pass, w) is None
    # a workload without a capture has no traffic either
    assert bench.ncu_traffic("bwd", synth.WORKLOADS["t2b_f32_b1c4_16x16"]) is None


def test_l2_flush_only_where_a_pass_fits_in_l2():
    """The timing rule: inputs larger than L2, or L2 flushed between timed
    passes.  Passes of at least the L2's 126 MB are timed back to back; a
    smaller pass (the 16x16 problem, the generic 130x70 forward) gets a flush."""
    import bench
    import synth
    fits = {}
    for name, w in list(synth.WORKLOADS.items()) + list(synth.EXTRA_WORKLOADS.items()):
        fb, bb = bench.pass_bytes(w)
        fits[name] = fb < bench.L2_BYTES or bb < bench.L2_BYTES
    assert fits == {
        "t2b_f32_b1c4_16x16": True,
        "4dir_f32_b8c96_56x56": False,
        "4dir_local4_bf16_b32c192_28x28": False,
        "compact_4dir_bf16_b32c1152_64x64": False,
        "compact_4dir_bf16_b2c1152_128x128_fwdbwd": False,
        "generic_4dir_f32_b2c64_130x70": True,
        "large_compact_4dir_bf16_b2c1152_256x256": False,
    }
    assert bench.L2_BYTES == 126 * 2**20


def test_config_names_the_launch_form_and_the_l2_rule():
    import bench
    import synth
    w = synth.WORKLOADS["compact_4dir_bf16_b32c1152_64x64"]
    c = bench.config_of(w, 1)
    assert c["workload"] == w.name and c["launch"] == "direct" and c["l2"].startswith("inputs larger than L2")
    c = bench.config_of(w, 1, graph=True, flushed=True)
    assert c["launch"] == "cuda_graph" and c["l2"].startswith("flushed")
    assert "model" not in c
