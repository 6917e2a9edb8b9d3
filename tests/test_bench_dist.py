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
