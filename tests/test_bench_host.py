"""Host-side logic of bench.py (CPU only): the max-over-ranks reduction and
per-rank seeding on a 2-rank gloo group, clock-sample parsing, the recorded
traffic guard, and the reference arm end to end."""
import json
import os
import subprocess
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _worker(rank, world, port, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    w, r, _ = bench.dist_env()
    d = bench.init_dist(w, "gloo")
    dev = torch.device("cpu")
    bench.barrier(d, dev)
    m = bench.max_over_ranks(10.0 + 5 * r, d, dev)
    q.put((r, m, bench.rank_seed(50, r)))
    d.destroy_process_group()


def test_max_over_ranks_and_seeds_on_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + os.getpid() % 1000
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    out.sort()
    assert [m for _, m, _ in out] == [15.0, 15.0]
    assert out[0][2] != out[1][2]


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(3.5, None, torch.device("cpu")) == 3.5


def test_clock_parse():
    text = ("1965, 1965, 812.5, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active\n"
            "1850, 1965, 998.1, 0x0000000000000004, Not Active, Not Active, Not Active, Active\n"
            "1900, 1965, [N/A], 0x0000000000000000, Not Active, Not Active, Not Active, Not Active\n")
    c = bench.ClockSampler.parse(text)
    assert c["sm_mhz"] == 1900 and c["sm_max_mhz"] == 1965
    assert c["reasons"] == ["sw_power_cap"] and c["power_w_max"] == 998.1 and c["samples"] == 3
    assert bench.ClockSampler.parse("") is None


def test_traffic_record_needs_matching_sources(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    (tmp_path / "profiles").mkdir()
    rec = {"ln_bf16_65536x16384": {"traffic_bytes_per_launch": 123, "source_digest": "stale"}}
    (tmp_path / "profiles" / "ncu_traffic.json").write_text(json.dumps(rec))
    assert bench.recorded_traffic("ln_bf16_65536x16384") is None
    rec["ln_bf16_65536x16384"]["source_digest"] = bench.source_digest()
    (tmp_path / "profiles" / "ncu_traffic.json").write_text(json.dumps(rec))
    assert bench.recorded_traffic("ln_bf16_65536x16384") == 123
    assert bench.recorded_traffic("absent") is None


def test_reference_arm_prints_one_line():
    res = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--steps", "2", "--warmup", "3"], capture_output=True, text=True,
                         timeout=300, cwd=ROOT)
    assert res.returncode == 0, res.stderr
    lines = [l for l in res.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "rows/s" and d["value"] > 0
    assert d["metric"] == bench.METRIC and d["higher_is_better"] is True
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0


def test_warmup_minimum_enforced():
    res = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--warmup", "1"],
                         capture_output=True, text=True, timeout=120, cwd=ROOT)
    assert res.returncode != 0


def test_cpu_baseline_times_all_cores_and_one_thread():
    """cpu_baseline over a step's items (host tensors here): every row on all
    cores, and a proportional sample on one thread."""
    from transformer_row_normalization_b200 import workloads as wl

    class FakeStep:
        items = [(wl.WORKLOADS[n], wl.make_inputs(wl.WORKLOADS[n]), None)
                 for n in ("dual_bf16_decode", "rms_f32_4x128x1024", "ln_f32_1x1024x768")]

    b = bench.cpu_baseline(FakeStep(), chunk_rows=256, single_share=4)
    assert b["kind"] == "oracle" and b["cores"] >= 1 and b["value"] > 0
    assert "(1576 rows" in b["sample"]  # 32 + 8 query/key head rows, 512, 1024
    st = b["single_thread"]
    assert st["cores"] == 1 and st["value"] > 0
    # a quarter of each part's rows: 32/4 + 8/4 + 512/4 + 1024/4
    assert "(394 rows)" in st["sample"]


@pytest.mark.parametrize("chunks", [1, 3, 8])
def test_e2e_chunks_cover_every_row_once(chunks):
    """The end-to-end pipeline's row chunks (host tensors here) tile each
    workload exactly: every row in one chunk, outputs beside their inputs,
    the dual workload cut by whole tokens."""
    from transformer_row_normalization_b200 import workloads as wl
    for name in ("dual_bf16_decode", "rms_f32_4x128x1024", "ln_f32_1x1024x768"):
        w = wl.WORKLOADS[name]
        a = wl.make_inputs(w)
        out = ((torch.empty_like(a["q"]), torch.empty_like(a["k"])) if w.op == "dual"
               else (torch.empty_like(a["x"]),))
        parts = bench.chunk_views(w, a, out, chunks)
        assert 1 <= len(parts) <= chunks
        for ins, outs in parts:
            assert len(ins) == len(outs)
            for i, o in zip(ins, outs):
                assert i.shape == o.shape
        if w.op == "dual":
            assert sum(p[0][0].shape[0] for p in parts) == a["q"].shape[0]
            assert torch.equal(torch.cat([p[0][1] for p in parts]), a["k"])
        else:
            got = torch.cat([p[0][0] for p in parts])
            assert torch.equal(got, a["x"].reshape(-1, w.dim))
            ptrs = [p[1][0].data_ptr() for p in parts]
            assert ptrs == sorted(ptrs) and ptrs[0] == out[0].data_ptr()
