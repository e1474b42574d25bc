"""Host logic of bench.py on the CPU: bandwidth arithmetic, buffer rotation,
clock parsing, and the multi-rank timing reduction on 2 gloo ranks."""

import json
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def test_busbw_and_bytes():
    # 1 MiB per rank at P=8 in 10 us: algbw 104.8576 GB/s, busbw x 2*7/8
    assert bench.busbw_gbs(8, 524288, 2, 10e-6) == pytest.approx(1048576 / 10e-6 * 1.75 / 1e9)
    assert bench.busbw_gbs(1, 100, 4, 1.0) == pytest.approx(400 / 1e9)
    assert bench.b_min_bytes(8, 524288, 2) == 16 * 1024 * 1024


def test_algorithmic_bytes_per_algorithm():
    """B_alg counted access by access for small cases, against the closed forms."""
    s = 2
    # write mode moves exactly the minimum: P inputs read, P outputs written
    assert bench.b_alg_bytes("twostage_write", 8, 1, s) == bench.b_min_bytes(8, 1, s) == 32
    # one-shot: every one of P ranks reads P inputs and writes its output
    assert bench.b_alg_bytes("oneshot", 8, 1, s) == (8 * 8 + 8) * s
    # pull two-stage: P n s of inputs read, n s of reduced chunks written, then every rank reads
    # and writes the (P - 1) chunks it lacks: P + 1 + 2 (P - 1) = 3P - 1 times n s
    assert bench.b_alg_bytes("twostage", 8, 1, s) == (3 * 8 - 1) * s
    # recursive doubling, 8 ranks: inputs + outputs, and per step each rank writes and reads
    # 8 bytes of payload per 4 data bytes
    steps, per_step = 3, 2 * (8 * 1 * s * 2)
    assert bench.b_alg_bytes("rd", 8, 1, s) == 2 * 8 * 1 * s + steps * per_step
    assert bench.b_alg_bytes("rd", 8, 1, s, fp32_wire=True) == 2 * 8 * 1 * s + steps * 2 * per_step
    assert bench.b_alg_bytes("rd", 8, 1, 4, fp32_wire=True) == bench.b_alg_bytes("rd", 8, 1, 4)
    # hierarchical 4 x 8: 2 P n s plus 2 steps of payload on n / 8 per rank: 3 P n s
    assert bench.b_alg_bytes("hier", 32, 8, s, L=8) == 3 * 32 * 8 * s
    with pytest.raises(ValueError):
        bench.b_alg_bytes("auto", 8, 1, s)


def test_rotation_exceeds_l2():
    for set_bytes in (2 << 20, 16 << 20, 128 << 20, 3758096384):
        R = bench.rotation_sets(set_bytes)
        assert R >= 1
        assert R * set_bytes >= min(3 * bench.L2_BYTES, set_bytes * 64) or set_bytes > 3 * bench.L2_BYTES


def test_parse_clocks():
    text = "\n".join([
        "0, 1965 MHz, 1965 MHz, 650.10 W, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
        "0, 1800 MHz, 1965 MHz, 990.00 W, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "0, 345 MHz, 1965 MHz, 120.00 W, 0x0000000000000001, Not Active, Not Active, Not Active, Not Active",
    ])
    c = bench.parse_clocks_csv(text)
    assert c["sm_mhz"] == pytest.approx(1882.5)
    assert c["sm_max_mhz"] == 1965
    assert c["reasons"] == ["sw_power_cap"]
    assert c["samples"] == 3 and c["samples_under_load"] == 2


def test_peaks_fallback(tmp_path):
    assert bench.load_peaks(str(tmp_path / "missing.json")) == (bench.FALLBACK_HBM_GBS, "fallback")
    p = tmp_path / "p.json"
    p.write_text('{"hbm_gbs": 6451.5}')
    assert bench.load_peaks(str(p)) == (6451.5, "measured")
    nested = tmp_path / "nested.json"
    nested.write_text(json.dumps({"gpu": "B200", "peaks": {"hbm_gbs": 6400.0, "bf16_tflops": 1590.0}}))
    assert bench.load_peaks(str(nested)) == (6400.0, "measured")
    junk = tmp_path / "junk.json"
    junk.write_text(json.dumps({"hbm_gbs": "fast"}))
    assert bench.load_peaks(str(junk)) == (bench.FALLBACK_HBM_GBS, "fallback")


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench.barrier(world)
        m = bench.max_over_ranks(1.5 + rank, world)
        q.put((rank, m))
        bench.barrier(world)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_world2():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert got == {0: 2.5, 1: 2.5}


def test_reference_arm_other_ranks_exit_without_work(monkeypatch):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    assert bench.run_reference(bench.argparse.Namespace(steps=3, warmup=3)) is None


def test_reference_arm_line_on_cpu(monkeypatch, capsys):
    monkeypatch.setenv("RANK", "0")
    monkeypatch.setenv("WORLD_SIZE", "1")
    bench.main(["--impl", "reference", "--steps", "3", "--warmup", "3"])
    line = bench.json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "GB/s" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"
    assert line["metric"] == bench.METRIC


def test_row_flags():
    assert bench.with_flags("twostage_write") == ("twostage_write", False, False)
    assert bench.with_flags("oneshot+edge") == ("oneshot", True, False)
    assert bench.with_flags("twostage_write+fp8") == ("twostage_write", False, True)
    assert bench.with_flags("twostage+edge+fp8") == ("twostage", True, True)


def test_cpu_baseline_host_facts_and_pinning():
    import os
    h = bench.host_description()
    assert h["nproc"] == os.cpu_count() and h["nproc"] >= 1
    before = os.sched_getaffinity(0)
    with bench.one_core() as pin:
        inside = os.sched_getaffinity(0)
        assert len(inside) == 1 and inside <= before
        assert pin.describe() == f"os.sched_setaffinity to core {min(before)}"
    assert os.sched_getaffinity(0) == before, "the affinity must be restored"


def test_reference_arm_prints_one_line_on_the_cpu(capsys):
    """The reference arm times the CPU oracle on slices of the step's workload
    and needs no GPU."""
    import json
    bench.main(["--impl", "reference", "--steps", "2", "--warmup", "3"])
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["metric"] == bench.METRIC and line["value"] > 0
    assert line["config"]["workload"] == bench.WORKLOAD["name"] and line["config"]["n"] == 16384 * 7168
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] == 1 and cb["threads"] == 1 and "nproc" in cb
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
