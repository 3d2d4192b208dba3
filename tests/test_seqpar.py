"""Sequence-parallel prefill (positive_quadratic_b200.seqpar): the rank logic checked against
the oracle over the whole sequence -- as two gloo ranks on the CPU with the oracle as the
local backend, and on one GPU with the library as the backend (ranks run in one process)."""
import os
import socket

import numpy as np
import pytest
import torch

import oracle
from positive_quadratic_b200 import inputs as I
from positive_quadratic_b200 import seqpar


class OracleBackend:
    """Local steps in fp64 on the CPU: the oracle's recurrence with explicit states."""

    def segment_state(self, k, v, group_id, L, G, eps):
        B, Hkv, T, d = k.shape
        Hq = group_id.shape[0]
        q = np.zeros((B, Hq, T, d))
        _, st = oracle.recurrent(q, k.numpy(), v.numpy(), group_id, L, G, eps,
                                 return_state=True)
        return {"st": st, "tokens": 0}

    def body(self, state, B, Hkv):
        st = state["st"]
        flat = np.concatenate([st.H0.ravel(), st.H1.ravel(), st.H2.ravel()])
        t = torch.from_numpy(flat)
        state["_flat"] = t
        return t

    def set_tokens(self, state, tokens):
        state["tokens"] = tokens

    def combine(self, parts, n_parts, body):
        body.copy_(parts[:n_parts].sum(dim=0))

    def continue_from(self, q, k, v, group_id, L, G, eps, state):
        st, flat = state["st"], state["_flat"].numpy()
        n0, n1 = st.H0.size, st.H1.size
        st.H0[...] = flat[:n0].reshape(st.H0.shape)
        st.H1[...] = flat[n0:n0 + n1].reshape(st.H1.shape)
        st.H2[...] = flat[n0 + n1:].reshape(st.H2.shape)
        y, st2 = oracle.recurrent(q.numpy(), k.numpy(), v.numpy(), group_id, L, G, eps,
                                  state=st, return_state=True)
        state["st"] = st2
        return torch.from_numpy(y)


def _problem():
    return I.small_layer(4242, B=1, T=74, Hq=4, Hkv=2, dtype="f32")


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import torch.distributed as dist
    from datetime import timedelta
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        p = _problem()
        T = p.q.shape[2]
        seg = T // world
        s = p.slice_tokens(rank * seg, (rank + 1) * seg)
        y, state = seqpar.sequence_parallel_prefill(
            torch.from_numpy(s.q), torch.from_numpy(s.k), torch.from_numpy(s.v), p.group_id,
            p.L, p.G, p.eps, rank=rank, world=world, tokens_before=rank * seg,
            backend=OracleBackend())
        out[rank] = (y.numpy(), state["st"].H2.copy())
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_gloo_ranks_match_whole_sequence(world):
    import torch.multiprocessing as mp
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
        for pr in procs:
            pr.start()
        for pr in procs:
            pr.join(180)
        assert all(pr.exitcode == 0 for pr in procs), [pr.exitcode for pr in procs]
        res = dict(out)
    p = _problem()
    seg = p.q.shape[2] // world
    n = world * seg  # tokens the ranks cover (the ragged remainder is left out)
    ref, st = oracle.recurrent(p.q[:, :, :n], p.k[:, :, :n], p.v[:, :, :n], p.group_id, p.L,
                               p.G, p.eps, return_state=True)
    y = np.concatenate([res[r][0] for r in range(world)], axis=2)
    np.testing.assert_allclose(y, ref, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(res[world - 1][1], st.H2, rtol=1e-10, atol=1e-12)


def _rank_main_uneven(rank, world, port, bounds, out):
    import torch.distributed as dist
    from datetime import timedelta
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        p = _problem()
        t0, t1 = bounds[rank], bounds[rank + 1]
        s = p.slice_tokens(t0, t1)
        y, state = seqpar.sequence_parallel_prefill(
            torch.from_numpy(s.q), torch.from_numpy(s.k), torch.from_numpy(s.v), p.group_id,
            p.L, p.G, p.eps, rank=rank, world=world, tokens_before=t0,
            backend=OracleBackend())
        out[rank] = (y.numpy(), state["st"].H2.copy(), state["tokens"])
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_gloo_ranks_uneven_segments_cover_the_sequence():
    """Four ranks hold segments of 9, 0, 40 and 25 tokens (one empty) of a 74-token sequence:
    together they give every token's output and, on the last rank, the whole state."""
    import torch.multiprocessing as mp
    world, bounds = 4, [0, 9, 9, 49, 74]
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        procs = [ctx.Process(target=_rank_main_uneven, args=(r, world, port, bounds, out))
                 for r in range(world)]
        for pr in procs:
            pr.start()
        for pr in procs:
            pr.join(180)
        assert all(pr.exitcode == 0 for pr in procs), [pr.exitcode for pr in procs]
        res = dict(out)
    p = _problem()
    ref, st = oracle.recurrent(p.q, p.k, p.v, p.group_id, p.L, p.G, p.eps, return_state=True)
    y = np.concatenate([res[r][0] for r in range(world)], axis=2)
    assert y.shape == ref.shape
    np.testing.assert_allclose(y, ref, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(res[world - 1][1], st.H2, rtol=1e-10, atol=1e-12)
    assert [res[r][2] for r in range(world)] == bounds[:-1]


@pytest.mark.gpu
def test_segments_on_one_gpu_match_whole_sequence(cuda):
    """Three ranks run in this process on the library: each rank's output equals the
    corresponding rows of one prefill over the whole sequence."""
    from positive_quadratic_b200 import oal
    from tests._metrics import TOL_BF16, row_rel_err
    p = I.small_layer(4343, B=2, T=3 * 300, Hq=14, Hkv=2, dtype="bf16")
    ref = oracle.recurrent(p.q, p.k, p.v, p.group_id, p.L, p.G, p.eps)
    world, seg = 3, 300
    t = lambda a, d=None: torch.from_numpy(np.ascontiguousarray(a)).to(cuda, d)
    g, L, G = t(p.group_id), t(p.L), t(p.G)
    segs = [p.slice_tokens(r * seg, (r + 1) * seg) for r in range(world)]
    dev = [(t(s.q, torch.bfloat16), t(s.k, torch.bfloat16), t(s.v, torch.bfloat16))
           for s in segs]
    backend = seqpar.LibraryBackend(14)
    # the all-gather of the segment states, done in-process: every rank's segment state
    bodies = [oal.state_body(oal.prefill_state(k, v, g, L, G, p.eps, 14), 2, 14, 2).clone()
              for (_, k, v) in dev]
    for r, (q, k, v) in enumerate(dev):
        y, _ = seqpar.sequence_parallel_prefill(
            q, k, v, g, L, G, p.eps, rank=r, world=world, tokens_before=r * seg,
            backend=backend, allgather=lambda body: bodies)
        torch.cuda.synchronize()
        assert oal.device_error() == 0
        assert row_rel_err(y.cpu().numpy(), ref[:, :, r * seg:(r + 1) * seg]) <= TOL_BF16


@pytest.mark.gpu
@pytest.mark.parametrize("n_parts", [0, 1, 3])
def test_state_prefix_sum(cuda, n_parts):
    """oal_state_prefix_sum adds the parts in order: equal, bit for bit, to fp32 additions in
    the same order."""
    from positive_quadratic_b200 import oal
    n = 2 * 2176 * 65
    g = torch.Generator().manual_seed(n_parts)
    parts = torch.randn(4, n, generator=g).to(cuda)
    out = torch.full((n,), float("nan"), device=cuda)
    oal.state_prefix_sum(parts, n_parts, out)
    ref = torch.zeros(n, device=cuda)
    for r in range(n_parts):
        ref = ref + parts[r]
    torch.cuda.synchronize()
    assert torch.equal(out, ref)


def _rank_main_failing(rank, world, port, out):
    import torch.distributed as dist
    from datetime import timedelta
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=10))
    if rank == 1:  # this rank fails before its exchange step and leaves
        raise SystemExit(3)
    p = _problem()
    s = p.slice_tokens(0, 37)
    try:
        seqpar.sequence_parallel_prefill(
            torch.from_numpy(s.q), torch.from_numpy(s.k), torch.from_numpy(s.v), p.group_id,
            p.L, p.G, p.eps, rank=rank, world=world, tokens_before=0, backend=OracleBackend())
        out[rank] = "returned"
    except Exception as exc:  # the collective reports the lost peer
        out[rank] = "error: " + type(exc).__name__


def test_a_failed_rank_ends_the_others_exchange_with_an_error():
    """A rank that leaves before the exchange step makes the other ranks' all-gather end with
    an error (the peer's closed connection or the process group's short timeout), not a hang."""
    import time
    import torch.multiprocessing as mp
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    t0 = time.monotonic()
    with ctx.Manager() as mgr:
        out = mgr.dict()
        procs = [ctx.Process(target=_rank_main_failing, args=(r, world, port, out))
                 for r in range(world)]
        for pr in procs:
            pr.start()
        for pr in procs:
            pr.join(120)
        alive = [pr.is_alive() for pr in procs]
        for pr in procs:
            if pr.is_alive():
                pr.kill()
        res = dict(out)
    assert not any(alive), "a rank hung"
    assert procs[1].exitcode == 3
    assert res.get(0, "").startswith("error"), res
    assert time.monotonic() - t0 < 120
