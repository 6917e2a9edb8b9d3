"""Host-side logic of bench.py's multi-rank path, on CPU with gloo
(world size 2): max / sum over ranks, rank-0-only reference arm, and the
command-line contract."""
import os
import socket

import pytest
import torch.multiprocessing as mp

import bench


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    r, w = bench.init_dist("gloo")
    bench.barrier()
    mx = bench.max_over_ranks(1.5 + rank)
    sm = bench.sum_over_ranks(10.0 * (rank + 1))
    ref = bench.run_reference(type("A", (), {"warmup": 0, "steps": 0, "bwd_mode": "eden"})()) if rank else None
    q.put((rank, r, w, mx, sm, ref))
    import torch.distributed as dist
    dist.destroy_process_group()


def test_two_ranks_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(i, 2, port, q)) for i in range(2)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, r, w, mx, sm, ref in out:
        assert (r, w) == (rank, 2)
        assert mx == 2.5          # max over ranks of 1.5 + rank
        assert sm == 30.0         # 10 + 20
        if rank == 1:
            assert ref is None    # the reference arm runs on rank 0 only


def test_single_rank_reductions_are_identity():
    assert bench.max_over_ranks(3.25) == 3.25
    assert bench.sum_over_ranks(2.0) == 2.0


def test_cli_rejects_short_warmup():
    with pytest.raises(SystemExit):
        bench.main(["--warmup", "2"])


def test_step_accounting():
    flops = bench.gemm_flops()
    assert flops == 3 * 2 * 8192 * 14336 * 4096
    calls = bench.quant_calls()
    assert [n for _, n, _ in calls] == [8192 * 4096, 14336 * 4096, 8192 * 14336, 14336 * 4096, 8192 * 4096]


@pytest.mark.parametrize("mode", sorted(bench.BWD_MODES))
def test_reference_arm_sample_runs_in_every_backward_mode(mode):
    """The CPU reference arm times the oracle on a bounded sample in each
    backward mode the bench offers, and names that mode in its workload."""
    dt, desc, threads = bench.oracle_sample(budget_rows=1, gemm_rows=2, gemm_cols=2, bwd_mode=mode)
    assert dt > 0 and threads >= 1
    assert "dY rows+cols: 16x14336" in desc
    assert bench.BWD_NAMES[mode] in bench.workload(mode)


def test_quantize_bytes_per_element():
    # bf16 read once + 0.5 B of codes and 1/16 B of scale per element and
    # orientation (1D); 2D blocks carry one scale per 256 elements
    assert bench.quant_bytes_per_elem(bench.ROW) == 2.5625
    assert bench.quant_bytes_per_elem(bench.COL) == 2.5625
    assert bench.quant_bytes_per_elem(bench.ROW | bench.COL) == 3.125
    assert bench.quant_bytes_per_elem(bench.ROW | bench.B2D) == 2 + 0.5 + 1 / 256
    assert bench.quant_bytes_per_elem(bench.ROW | bench.COL | bench.B2D) == 3 + 2 / 256


def test_quantize_roofline_takes_the_larger_floor_per_kernel():
    # kernel 1: 592e6 warp instructions at 1000 MHz on 148 SMs = 1000 us of
    # issue against 1 us of HBM; kernel 2: 665e6 bytes at 6650 GB/s = 100 us
    # of HBM against ~0 us of issue
    rec = {"kernels": [{"warp_instructions": 592_000_000, "algorithmic_bytes": 6_650_000},
                       {"warp_instructions": 1, "algorithmic_bytes": 665_000_000}]}
    r = bench.quantize_roofline(rec, quant_ms=2.2, sm_mhz=1000.0, n_sm=148, hbm_gbs=6650.0)
    assert r["floor_us"] == pytest.approx(1100.0, abs=0.2)
    assert r["issue_floor_us"] == pytest.approx(1000.0, abs=0.2)
    assert r["hbm_floor_us"] == pytest.approx(101.0, abs=0.2)
    assert r["frac"] == pytest.approx(0.5, rel=1e-3)


def test_quantizer_issue_record_checks_the_sources(tmp_path, monkeypatch):
    import json
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "quantizer_issue.json").write_text(json.dumps({"source_sha256_16": "0" * 16, "kernels": []}))
    csrc = tmp_path / "nvfp4_block_quantization_amax_b200" / "csrc"
    csrc.mkdir(parents=True)
    for f in bench.QUANT_SOURCES:
        (csrc / f).write_text(f)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.quantizer_issue_record() is None   # taken on other sources
    import hashlib
    h = hashlib.sha256(b"".join(f.encode() for f in bench.QUANT_SOURCES)).hexdigest()[:16]
    (prof / "quantizer_issue.json").write_text(json.dumps({"source_sha256_16": h, "kernels": []}))
    assert bench.quantizer_issue_record() == {"source_sha256_16": h, "kernels": []}


def test_carve_lays_shapes_end_to_end():
    # the e2e buffers: X, W, dY (and Y, dX, dW) as consecutive row-major views
    # of one buffer, so each direction is a single copy of all of them
    import torch
    shapes = [(3, 4), (5, 4), (3, 5)]
    buf = torch.arange(sum(r * c for r, c in shapes), dtype=torch.float32)
    views = bench.carve(buf, shapes)
    assert [tuple(v.shape) for v in views] == shapes
    assert all(v.is_contiguous() for v in views)
    assert torch.equal(torch.cat([v.reshape(-1) for v in views]), buf)
    views[1][0, 0] = -1.0   # views, not copies
    assert buf[12].item() == -1.0
