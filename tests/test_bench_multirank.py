"""The multi-process benchmark plumbing on CPU: two gloo ranks, barrier, max-over-ranks of the device time
and the whole-job throughput (weak scaling, replicas, no data-path collective)."""
import os
import socket

import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _rank_main(rank, world, port, q):
    import sys

    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world), RANK=str(rank),
                      LOCAL_RANK=str(rank))
    import bench

    ctx = bench.DistCtx("gloo")
    ctx.barrier()
    t_local = 10.0 * (rank + 1)          # the slower rank decides the job time
    t_max = ctx.max(t_local)
    v = bench.job_throughput(100.0, 5, ctx.world, t_max)
    q.put((rank, ctx.world, t_max, v))
    ctx.close()


def test_two_gloo_ranks_max_time_and_job_throughput():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, w, t_max, v in res:
        assert w == 2 and t_max == 20.0
        assert abs(v - 100.0 * 5 * 2 / 0.020) < 1e-6


def test_single_process_defaults():
    import sys

    sys.path.insert(0, ROOT)
    import bench

    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK"):
        os.environ.pop(k, None)
    ctx = bench.DistCtx("gloo")
    assert not ctx.on and ctx.max(3.5) == 3.5
    assert bench.attn_flops(1, 32, 4096, 64, False) == 2 * bench.attn_flops(1, 32, 4096, 64, True)
    assert bench.attn_flops(1, 32, 4096, 64, False) == 4 * 32 * 4096 ** 2 * 64


def test_kernel_source_hash_ignores_comments(tmp_path, monkeypatch):
    """Recorded profiler counters stay keyed to the kernel code: a comment-only edit keeps the hash, a code
    edit changes it."""
    import shutil
    import sys

    sys.path.insert(0, ROOT)
    import bench

    csrc = tmp_path / "exact_tiled_attention_43_b200" / "csrc"
    csrc.mkdir(parents=True)
    for f in ("ptx.cuh", "prefill.cuh", "decode.cuh"):
        shutil.copy(os.path.join(ROOT, "exact_tiled_attention_43_b200", "csrc", f), csrc / f)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h0 = bench.kernel_source_hash()
    assert h0 == bench.__dict__["kernel_source_hash"]()
    p = csrc / "prefill.cuh"
    src = p.read_text()
    p.write_text("// a new comment line\n" + src.replace("#pragma once", "#pragma once  // trailing note /* x */", 1))
    assert bench.kernel_source_hash() == h0
    p.write_text(src + "\nstatic const int eta_extra_constant = 1;\n")
    assert bench.kernel_source_hash() != h0
