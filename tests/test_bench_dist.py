"""The multi-rank plumbing of bench.py on CPU: two gloo ranks (no GPU).

Every (sequence, head) of the pass is independent, so N ranks run N replicas of the
workload (weak scaling) with no collective on the data path; the only collectives are
the barrier around the timed region and the max over ranks of the elapsed time.
"""

import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(world),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench
    d = bench.Dist(backend="gloo")
    try:
        d.barrier()
        # rank r "took" 1 + r seconds: the job time is the slowest rank's
        t = d.max(1.0 + rank)
        s = d.sum(10.0)
        v = bench.weak_scaling_value(1000.0, t, d.world)
        args = type("A", (), {"workload": "tiny", "reference_tokens": 16, "warmup": 0,
                              "steps": 1})()
        ref = bench.run_reference(args, d) if rank != 0 else "rank0"
        out.put((rank, t, s, v, ref))
    finally:
        d.close()


def test_two_gloo_ranks_max_sum_and_weak_scaling():
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
    for rank, t, s, v, ref in res:
        assert t == pytest.approx(2.0)          # max over ranks
        assert s == pytest.approx(20.0)
        assert v == pytest.approx(1000.0 * 2 / 2.0)  # both ranks' units over the max time
    assert res[1][4] is None                     # the reference arm runs on rank 0 only


def test_single_process_defaults():
    sys.path.insert(0, ROOT)
    import bench
    d = bench.Dist()
    assert d.world == int(os.environ.get("WORLD_SIZE", "1"))
    assert d.max(3.5) == 3.5
    assert bench.weak_scaling_value(10.0, 2.0, 1) == 5.0


def test_measured_traffic_scales_and_expires(tmp_path, monkeypatch):
    """The roofline's `traffic` comes from the committed capture, scaled to a launch; once
    the kernel's source no longer has the recorded hash it is reported as null."""
    import hashlib
    import json
    sys.path.insert(0, ROOT)
    import bench
    src = tmp_path / "kernel.cuh"
    src.write_text("// kernel source\n")
    sha = hashlib.sha256(src.read_bytes()).hexdigest()[:16]
    (tmp_path / "profiles").mkdir()
    rec = {"k": {"dram_bytes_per_unit": 100, "source": "kernel.cuh", "source_sha256_16": sha}}
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.measured_traffic("k", 512, "dram_bytes_per_unit") == 51200
    assert bench.measured_traffic("other", 512, "dram_bytes_per_unit") is None
    src.write_text("// kernel source, changed\n")
    assert bench.measured_traffic("k", 512, "dram_bytes_per_unit") is None


def test_committed_traffic_records_are_well_formed():
    """profiles/traffic.json names, per kernel, its capture summary, the kernel source and
    the source hash the capture was taken with (a changed source reports null traffic)."""
    import json
    rec = json.load(open(os.path.join(ROOT, "profiles", "traffic.json")))
    assert {"slot_chunk_kernel", "decode_kernel"} <= set(rec)
    for name, r in rec.items():
        assert os.path.exists(os.path.join(ROOT, "profiles", r["capture"])), name
        assert os.path.exists(os.path.join(ROOT, r["source"])), name
        assert len(r["source_sha256_16"]) == 16, name
        assert [k for k in r if k.startswith("dram_bytes_per_")], name
