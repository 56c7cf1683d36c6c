"""The N > 1 path of bench.py on CPU: two gloo ranks.

Rows are sharded across ranks with no collective on the data path (the
transitions of independent sequences batch freely: jiphyeonjeon review
"Recurrent Looped Transformer" §5); the only cross-rank step is the
max-over-ranks reduction of the timing.  These tests run bench's own helpers
in two spawned processes.
"""
import json
import os
import socket
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, out_dir: str):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    import datetime

    import torch.distributed as dist

    import bench
    import rlt_inputs as ri

    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        cfg = ri.CONFIGS["parity_bf16"]
        B, T = 5, 9
        toks = bench.shard_tokens(cfg, rank, B, T)
        # rank-dependent "time": the job's time is the slowest rank's
        ms = 10.0 + 7.5 * rank
        job_ms = bench.max_over_ranks(ms, world, "cpu")
        value = bench.job_tokens_per_s(B, T, world, job_ms)
        # the reference arm does its work on rank 0 only
        import contextlib
        import io
        buf = io.StringIO()

        class A:
            steps, warmup = 1, 0
        if rank != 0:
            with contextlib.redirect_stdout(buf):
                bench.run_reference(A, cfg)
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump({"toks": toks.tolist(), "job_ms": job_ms, "value": value,
                       "ref_out": buf.getvalue()}, f)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks(tmp_path):
    mp = pytest.importorskip("torch.multiprocessing")
    port = _free_port()
    ctx = mp.get_context("spawn")
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, str(tmp_path))) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        if p.is_alive():
            p.kill()
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(2)]

    sys.path.insert(0, ROOT)
    import rlt_inputs as ri
    cfg = ri.CONFIGS["parity_bf16"]
    # shards are disjoint consecutive row ranges of one global stream
    full = ri.make_tokens(cfg, 10, 9)
    np.testing.assert_array_equal(np.array(res[0]["toks"]), full[:5])
    np.testing.assert_array_equal(np.array(res[1]["toks"]), full[5:])
    assert not np.array_equal(full[:5], full[5:])
    # both ranks agree on the slowest rank's time and on the job's value
    for r in res:
        assert r["job_ms"] == pytest.approx(17.5)
        assert r["value"] == pytest.approx(2 * 5 * 9 / 17.5e-3)
    # the reference arm's rank 1 ran nothing and printed nothing
    assert res[1]["ref_out"] == ""
