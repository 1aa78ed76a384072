"""The N > 1 path of bench.py on CPU: two gloo ranks run the aggregation the
benchmark uses (max-over-ranks time, whole-job throughput of independent
replicas) and its barriers, and the reference arm leaves ranks > 0 idle;
plus the host-side kernel count the batched workload reports."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    import datetime

    import torch.distributed as dist

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench

    bench.barrier(world)
    local_ms = 100.0 + 50.0 * rank                      # rank 1 is the slow one
    max_ms, value = bench.aggregate(local_ms, steps=10, bytes_per_step=2_000_000_000, world=world)
    bench.barrier(world)
    ref_rc = bench.run_reference(bench.parse_args(["--impl", "reference", "--steps", "1", "--warmup", "0"])) \
        if rank == 1 else 0
    q.put((rank, max_ms, value, ref_rc))
    dist.destroy_process_group()


def test_two_gloo_ranks_aggregate_max_and_whole_job_throughput():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs)
    res = sorted(q.get(timeout=5) for _ in range(2))
    for rank, max_ms, value, ref_rc in res:
        assert max_ms == pytest.approx(150.0)
        # 2 replicas x 10 steps x 2 GB in 150 ms
        assert value == pytest.approx(2 * 10 * 2.0 / 0.150)
        assert ref_rc == 0


def test_batched_step_launch_count(monkeypatch):
    """The batched step's kernel count that bench.py reports: 6 launches per
    layer on the multi-row GEMV path, 8 (two bf16 casts) once Wo and W2 run
    on the tcgen05 GEMM from 4 sequences on, the embedding rows, the LM head
    and the position advance around them; 211 at 8 sequences matches the
    launch list taken under ncu."""
    import synth
    from bit_quantized_transformer_b200 import workloads as WL

    def model(n_seq, **kw):
        bm = WL.BatchDecoderModel.__new__(WL.BatchDecoderModel)
        bm.shape = synth.DecoderShape(**kw)
        bm.n_seq, bm.L = n_seq, bm.shape.n_layers
        return bm

    monkeypatch.delenv("VOX_BATCH_GEMM", raising=False)
    assert model(8).launches() == 211
    assert model(4).launches() == 211
    assert model(3).launches() == 159
    assert model(1).launches() == 159
    assert model(8, n_layers=2).launches() == 19
    assert model(8, ffn=9216 + 32).launches() == 159      # W2's K not a multiple of 64: GEMV
    monkeypatch.setenv("VOX_BATCH_GEMM", "0")
    assert model(8).launches() == 159
