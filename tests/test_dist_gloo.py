"""Multi-rank host path of the data-parallel bench, as world-size-2 gloo ranks
on the CPU (spawned processes, rendezvous on 127.0.0.1).

Checked: the job time is the max over ranks and the job throughput the
weak-scaling aggregate; every rank draws its own reproducible sequences; a
rank that dies before the barrier makes the survivor fail within the
process-group timeout instead of waiting for ever."""
import hashlib
import multiprocessing as mp
import os
import socket

import pytest

WORLD = 2


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _env(rank, port):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(WORLD), LOCAL_RANK=str(rank))


def _digest(t):
    return hashlib.sha256(t.contiguous().view(-1).view(dtype=__import__("torch").uint8)
                          .numpy().tobytes()).hexdigest()[:16]


def _tiny_inputs(rank):
    import lte_inputs as LI
    from learnable_kv_token_b200 import dist as DI
    wl = LI.WORKLOADS["tiny"]
    inp = LI.lte_inputs(wl.with_(seed=DI.shard_seed(wl.seed, rank)), T=wl.T)
    extra = inp["mask"] if "mask" in inp else inp["cnn"][0]
    return _digest(inp["q"]) + _digest(inp["k"]) + _digest(extra)


def _rank_main(rank, port, q):
    try:
        _env(rank, port)
        import torch.distributed as tdist
        from learnable_kv_token_b200 import dist as DI
        r, w, _ = DI.env_ranks()
        DI.init(w, "gloo", timeout_s=30)
        t_ms = 10.0 + 5.0 * r                      # the slower rank defines the job time
        job_ms = DI.max_over_ranks(t_ms, w)
        DI.barrier(w)
        thr = DI.job_throughput(1000.0, w, job_ms / 1e3)
        digests = [None] * w
        tdist.all_gather_object(digests, _tiny_inputs(r))
        DI.shutdown(w)
        q.put((rank, "ok", job_ms, thr, digests))
    except Exception as e:  # reported to the parent
        q.put((rank, "error", repr(e), None, None))


def _cnn_grads(rank):
    """The oracle's CNN weight gradients of rank `rank`'s shard (two sequences,
    one KV head, small sizes), as float64 tensors."""
    import numpy as np
    import torch
    from learnable_kv_token_b200 import dist as DI
    from oracle import lte_oracle as O
    rng = np.random.default_rng(DI.shard_seed(5, rank))
    n, D, c1 = 24, 3, 4
    # the same weights on every rank (a shared model), each rank its own sequences
    w = O.CNN(np.random.default_rng(5).standard_normal((c1, 2 * D, 5)) * 0.5,
              np.zeros(c1), np.random.default_rng(6).standard_normal((c1, 3)) * 0.5, 0.1, 2, 1)
    acc = None
    for _ in range(2):
        k, v, dr = rng.standard_normal((n, D)), rng.standard_normal((n, D)), rng.standard_normal(n)
        _, _, dw1, db1, dw2, db2 = O.cnn_backward(k, v, w, dr, n - w.future)
        g = [dw1, db1, dw2, np.array([db2])]
        acc = g if acc is None else [a + b for a, b in zip(acc, g)]
    return [torch.tensor(x) for x in acc]


def _grad_rank_main(rank, port, q):
    try:
        _env(rank, port)
        from learnable_kv_token_b200 import dist as DI
        r, w, _ = DI.env_ranks()
        DI.init(w, "gloo", timeout_s=30)
        grads = _cnn_grads(r)
        DI.all_reduce_sum_(grads, w)
        DI.shutdown(w)
        q.put((rank, "ok", [g.numpy() for g in grads]))
    except Exception as e:  # reported to the parent
        q.put((rank, "error", repr(e)))


def _dying_rank_main(rank, port, q):
    try:
        _env(rank, port)
        from learnable_kv_token_b200 import dist as DI
        DI.init(WORLD, "gloo", timeout_s=5)
        if rank == 1:
            q.put((rank, "exited", None))
            q.close()
            q.join_thread()                        # the message is out before the hard exit
            os._exit(0)                            # leaves without joining the barrier
        try:
            DI.barrier(WORLD)
            q.put((rank, "no-error", None))
        except Exception as e:
            q.put((rank, "error", type(e).__name__))
    except Exception as e:
        q.put((rank, "setup-error", repr(e)))


def _run(target, timeout):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=target, args=(r, port, q)) for r in range(WORLD)]
    for p in procs:
        p.start()
    out = []
    try:
        for _ in range(WORLD):
            out.append(q.get(timeout=timeout))
    finally:
        for p in procs:
            p.join(timeout=10)
            if p.is_alive():
                p.kill()                           # our own child, by its handle
                p.join()
    return sorted(out, key=lambda t: t[0])


def test_job_time_throughput_and_shards():
    res = _run(_rank_main, timeout=120)
    for rank, status, *rest in res:
        assert status == "ok", (rank, rest)
    (_, _, job0, thr0, dig0), (_, _, job1, thr1, dig1) = res
    assert job0 == job1 == 15.0                    # max over ranks, seen alike by both
    assert thr0 == thr1 == pytest.approx(1000.0 * WORLD / 0.015)
    assert dig0 == dig1 and dig0[0] != dig0[1]     # each rank its own sequences
    assert dig0 == [_tiny_inputs(0), _tiny_inputs(1)]   # reproducible from the rank alone


def test_dead_rank_fails_the_barrier_instead_of_hanging():
    res = _run(_dying_rank_main, timeout=90)
    status = {r: s for r, s, _ in res}
    assert status[1] == "exited"
    assert status[0] == "error", res


def test_cnn_weight_gradients_sum_over_ranks():
    """Data-parallel training: the CNN weight gradients each rank computes on
    its own sequences are summed over ranks by one coalesced all-reduce; every
    rank ends with the sum of both shards' gradients."""
    import numpy as np
    res = _run(_grad_rank_main, timeout=120)
    for rank, status, payload in res:
        assert status == "ok", (rank, payload)
    want = [a.numpy() + b.numpy() for a, b in zip(_cnn_grads(0), _cnn_grads(1))]
    for _, _, got in res:
        for g, w_ in zip(got, want):
            np.testing.assert_allclose(g, w_, rtol=0, atol=1e-12)
