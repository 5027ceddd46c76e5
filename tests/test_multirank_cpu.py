"""The N > 1 path on CPU: two gloo ranks run the benchmark's distributed
plumbing (process group, barrier, max over ranks, per-rank workloads,
whole-job throughput). Sequences shard across GPUs with no data-path
collective, so this is all the multi-rank logic there is."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port() -> int:
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world), RANK=str(rank),
                      LOCAL_RANK=str(rank))
    try:
        from paged_kv_cache_340_b200 import dist as pdist
        from paged_kv_cache_340_b200.workloads import SPECS
        w, r, _ = pdist.init("gloo", timeout_s=60)
        spec = pdist.rank_spec(SPECS["llama7b_mha_fp16"], r)
        pdist.barrier(w)
        t_max = pdist.max_over_ranks(10.0 + 3.0 * r, w)   # each rank's "time"
        thr = pdist.job_throughput(1_000_000_000, t_max, w)
        pdist.barrier(w)
        pdist.finalize(w)
        q.put((r, w, spec.seed, (spec.num_seqs, spec.num_heads, spec.head_dim), t_max, thr))
    except Exception as e:  # pragma: no cover - reported through the queue
        q.put((rank, "error", repr(e)))


def test_two_gloo_ranks_time_is_max_and_batches_are_per_rank():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = [q.get(timeout=180) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert all(res[1] != "error" for res in results), results
    results.sort()
    (r0, w0, seed0, shape0, t0, thr0), (r1, w1, seed1, shape1, t1, thr1) = results
    assert (r0, r1, w0, w1) == (0, 1, 2, 2)
    assert seed0 != seed1 and shape0 == shape1          # own data, same shapes (weak scaling)
    assert t0 == t1 == 13.0                             # the slowest rank's time on every rank
    assert thr0 == thr1 == pytest.approx(2 * 1e9 / 13e-3 / 1e9)


def test_single_rank_needs_no_process_group():
    from paged_kv_cache_340_b200 import dist as pdist
    assert pdist.max_over_ranks(4.5, 1) == 4.5
    pdist.barrier(1)
    assert pdist.job_throughput(2_000_000_000, 2.0, 1) == pytest.approx(1000.0)
