"""Host-side pieces of bench.py (no GPU): the algorithmic flop and byte
counts behind the roofline fields, the workload parser, the oracle
CPU-baseline sampler, and the reference arm's JSON line."""
import json
import os
import subprocess
import sys

import pytest

import bench
from gram_newton_schulz_b200 import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_alg_flops_closed_form():
    # 3 m^2 n + 17 m^3 per matrix, orientation-free
    assert bench.alg_flops([(2, 4)]) == 3 * 4 * 4 + 17 * 8
    assert bench.alg_flops([(4, 2)]) == bench.alg_flops([(2, 4)])
    w = synth.workload("qwen2.5-7b-layer-set-x28")
    assert bench.alg_flops(w.shapes) == pytest.approx(1.789e14, rel=2e-3)


def test_momentum_bytes():
    assert bench.momentum_bytes([(10, 10)]) == 100 * 12
    assert bench.momentum_bytes([(10, 10)], grad_bytes=4) == 100 * 14
    assert bench.momentum_bytes([(10, 10)], image16=True) == 100 * 16


def test_custom_workload_parser():
    w = bench.custom_workload("3584x3584*2,512x3584")
    assert w.shapes == ((3584, 3584), (3584, 3584), (512, 3584))
    assert w.dtype == "bf16" and w.dist == "spiked"


def test_oracle_sample_is_bounded_and_scaled():
    shapes = [(64, 256)] * 3 + [(128, 512)] * 2
    total, threads, sample, spent, extrapolated = bench.oracle_sample_seconds(shapes, budget_s=5.0)
    assert total > 0 and threads >= 1
    # two matrices of each bucket are timed, then each bucket scaled to its count
    assert "2 x 64x256" in sample and "2 x 128x512" in sample and "5 matrices" in sample
    assert extrapolated  # 4 of the 5 matrices were timed
    assert spent < 30
    total1, _, _, _, extrap1 = bench.oracle_sample_seconds([(64, 256)] * 2, budget_s=5.0)
    assert not extrap1 and total1 > 0


def test_reference_arm_prints_one_json_line():
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1", "--warmup", "0",
           "--shapes", "64x256*2", "--ref-budget", "2"]
    out = subprocess.run(cmd, capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert out.returncode == 0, out.stderr
    lines = [l for l in out.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "ms" and d["higher_is_better"] is False
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"


def test_gemm_alg_bytes_closed_form():
    # one 2x4 matrix, K = 5: SYRK 2*8 + 4*2, products 17*12*2, final 4*2 + 6*8
    assert bench.gemm_alg_bytes([(2, 4)]) == (16 + 8) + 17 * 24 + (8 + 48)
    # m >= 1024: the final reads P as one fp16 operand (2 bytes per stored element)
    m, n = 1024, 2048
    half = m * m / 2
    assert bench.gemm_alg_bytes([(m, n)]) == (2 * m * n + 4 * half) + 17 * 12 * half + (2 * half + 6 * m * n)
    assert bench.gemm_alg_bytes([(4, 2)]) == bench.gemm_alg_bytes([(2, 4)])


def test_captured_traffic_applies_only_to_its_sources(monkeypatch):
    cap = dict(bench.TRAFFIC_CAPTURE)
    assert bench.captured_traffic("uniform-64x512x2048") is None
    monkeypatch.setattr(bench, "TRAFFIC_CAPTURE", dict(cap, sha256="0" * 64))
    assert bench.captured_traffic(cap["workload"]) is None
    import hashlib
    h = hashlib.sha256()
    for rel in cap["sources"]:
        with open(os.path.join(ROOT, rel), "rb") as fh:
            h.update(fh.read())
    monkeypatch.setattr(bench, "TRAFFIC_CAPTURE", dict(cap, sha256=h.hexdigest()))
    assert bench.captured_traffic(cap["workload"]) == cap["dram_bytes_per_step"]


def test_schedule_summary_has_gram_syrk_and_final_entries():
    sch = {"gram": {3584: "cta_pair", 512: "single_cta_n128"},
           "syrk": {(3584, 18944): "cta_pair_n512", (512, 3584): "cta_pair_k2"},
           "final": {(3584, 18944): "single_cta"}}
    out = bench.schedule_summary(sch)
    assert out == {"gram": {"m3584": "cta_pair", "m512": "single_cta_n128"},
                   "syrk": {"3584x18944": "cta_pair_n512", "512x3584": "cta_pair_k2"},
                   "final": {"3584x18944": "single_cta"}}


def test_captured_traffic_names_its_schedules():
    # the capture records the schedule choices it ran under, in the bench
    # line's own form, so a run can say whether its choices were the same
    assert set(bench.TRAFFIC_CAPTURE["schedule"]) == {"gram", "syrk", "final"}


def test_executed_flops_counts_issued_mma_work():
    # one 256 x 512 matrix: one 256 x 256 upper tile, SPLIT3 (3 MMAs) below m = 1024
    up = 256 * 256
    assert bench.executed_flops([(256, 512)]) == 2 * up * 512 + 17 * 3 * 2 * up * 256 + 4 * 256 * 256 * 512
    # m = 1024: 4 x 4 blocks, 10 upper tiles, one F16 MMA per K slice, final one term
    up = 10 * 256 * 256
    assert bench.executed_flops([(1024, 4096)]) == 2 * up * 4096 + 17 * 1 * 2 * up * 1024 + 2 * 1024 * 1024 * 4096
    w = synth.workload("qwen2.5-7b-layer-set-x28")
    assert 1.0 < bench.executed_flops(w.shapes) / bench.alg_flops(w.shapes) < 1.15


def _agree_worker(rank, world, port, q):
    import datetime
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        all_true = bench.all_ranks_ok(True, "cpu", world)
        one_false = bench.all_ranks_ok(rank != 1, "cpu", world)
        q.put((rank, all_true, one_false))
    finally:
        dist.destroy_process_group()


def test_all_ranks_ok_is_a_min_over_ranks():
    """bench.py decides the graph-timed and e2e legs collectively: one rank's
    failure turns the leg off everywhere, so no rank waits alone in a
    collective.  Three gloo ranks on 127.0.0.1."""
    import socket
    import torch.multiprocessing as mp
    sock = socket.socket()
    sock.bind(("127.0.0.1", 0))
    port = sock.getsockname()[1]
    sock.close()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_agree_worker, args=(r, 3, port, q)) for r in range(3)]
    for p in procs:
        p.start()
    try:
        res = [q.get(timeout=120) for _ in range(3)]
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert all(a is True and b is False for _, a, b in res)
    assert bench.all_ranks_ok(False, "cpu", 1) is False and bench.all_ranks_ok(True, "cpu", 1) is True


def test_pin_copies_reports_failure_instead_of_raising(monkeypatch):
    import torch

    class Bad:
        def to(self, *_):
            raise RuntimeError("cannot pin")

    out, why = bench.pin_copies([Bad()])
    assert out is None and "cannot pin" in why
    ok, why = bench.pin_copies([torch.zeros(3)]) if torch.cuda.is_available() else ([None], None)
    assert why is None


def test_reference_arm_under_two_ranks():
    """Rank 0 alone runs the oracle for the whole job -- one layer set split
    over the ranks in the default owner mode, two layer sets in replica
    mode; the other rank exits 0 without work or output."""
    base = [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1", "--warmup", "0",
            "--shapes", "64x256*2", "--ref-budget", "2"]
    env0 = dict(os.environ, WORLD_SIZE="2", RANK="0", LOCAL_RANK="0")
    out = subprocess.run(base, capture_output=True, text=True, timeout=300, cwd=ROOT, env=env0)
    assert out.returncode == 0, out.stderr
    d = json.loads([l for l in out.stdout.splitlines() if l.strip()][0])
    assert d["n_gpus"] == 2 and d["config"]["matrices_total"] == 2 and d["scaling"] == "strong"
    out = subprocess.run(base + ["--shard", "replica"], capture_output=True, text=True, timeout=300, cwd=ROOT,
                         env=env0)
    assert out.returncode == 0, out.stderr
    d = json.loads([l for l in out.stdout.splitlines() if l.strip()][0])
    assert d["config"]["matrices_total"] == 4 and "2 replica ranks" in d["cpu_baseline"]["sample"]
    env1 = dict(os.environ, WORLD_SIZE="2", RANK="1", LOCAL_RANK="1")
    out1 = subprocess.run(base, capture_output=True, text=True, timeout=300, cwd=ROOT, env=env1)
    assert out1.returncode == 0 and out1.stdout.strip() == ""
