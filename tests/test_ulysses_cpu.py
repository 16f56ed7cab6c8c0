"""Ulysses context parallelism (sequence-sharded Q, K, V and tangents, all-to-all
to head shards and back) on CPU ranks over gloo.  The local attention is the
fp64 oracle, so the sharded result must equal the oracle on the unsharded
tensors exactly: this checks the layout logic of the two exchanges."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _inputs(B, H, Lq, Lk, d, seed):
    g = torch.Generator().manual_seed(seed)
    shp_q, shp_k = (B, H, Lq, d), (B, H, Lk, d)
    return {n: torch.randn(shp_q if n in ("q", "tq") else shp_k, generator=g, dtype=torch.float64)
            for n in ("q", "k", "v", "tq", "tk", "tv")}


def _oracle_fn(q, k, v, tq, tk, tv, scale):
    import oracle
    return tuple(torch.from_numpy(x) for x in oracle.attn_jvp(q, k, v, tq, tk, tv, scale))


def _worker(rank, world, port, shape, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from attention_forward_mode_b200.ulysses import ulysses_attn_jvp
        B, H, Lq, Lk, d = shape
        full = _inputs(B, H, Lq, Lk, d, seed=7)
        sq, sk = Lq // world, Lk // world
        shard = {n: (t[:, :, rank * sq:(rank + 1) * sq] if n in ("q", "tq") else t[:, :, rank * sk:(rank + 1) * sk])
                 .contiguous() for n, t in full.items()}
        o, to, lse = ulysses_attn_jvp(shard["q"], shard["k"], shard["v"], shard["tq"], shard["tk"], shard["tv"],
                                      scale=0.3, local_fn=_oracle_fn)
        ro, rto, rlse = _oracle_fn(*(full[n] for n in ("q", "k", "v", "tq", "tk", "tv")), 0.3)
        sl = slice(rank * sq, (rank + 1) * sq)
        out[rank] = (bool(torch.equal(o, ro[:, :, sl])), bool(torch.equal(to, rto[:, :, sl])),
                     bool(torch.equal(lse, rlse[:, :, sl])), tuple(o.shape), tuple(lse.shape))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(240)
@pytest.mark.parametrize("world,shape", [(2, (1, 4, 24, 24, 8)),     # self-attention
                                         (2, (2, 2, 16, 40, 4)),     # cross-attention, Lq != Lk
                                         (4, (1, 8, 32, 20, 8))])    # four ranks
def test_ulysses_matches_unsharded(world, shape):
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        procs = [ctx.Process(target=_worker, args=(r, world, port, shape, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(200)
        assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
        res = dict(out)
    B, H, Lq, Lk, d = shape
    for r in range(world):
        eq_o, eq_to, eq_lse, oshape, lshape = res[r]
        assert oshape == (B, H, Lq // world, d) and lshape == (B, H, Lq // world)
        assert eq_o and eq_to and eq_lse, res[r]


def test_single_rank_is_the_local_call():
    from attention_forward_mode_b200.ulysses import ulysses_attn_jvp
    t = _inputs(1, 2, 8, 8, 4, seed=1)
    a = ulysses_attn_jvp(t["q"], t["k"], t["v"], t["tq"], t["tk"], t["tv"], scale=0.5, local_fn=_oracle_fn)
    b = _oracle_fn(t["q"], t["k"], t["v"], t["tq"], t["tk"], t["tv"], 0.5)
    for x, y in zip(a, b):
        assert np.array_equal(x.numpy(), y.numpy())


def test_heads_must_divide():
    from attention_forward_mode_b200 import ulysses
    t = _inputs(1, 3, 8, 8, 4, seed=1)
    orig = ulysses.dist.is_initialized, ulysses.dist.get_world_size
    ulysses.dist.is_initialized = lambda: True
    ulysses.dist.get_world_size = lambda group=None: 2
    try:
        with pytest.raises(ValueError):
            ulysses.ulysses_attn_jvp(t["q"], t["k"], t["v"], t["tq"], t["tk"], t["tv"], local_fn=_oracle_fn)
    finally:
        ulysses.dist.is_initialized, ulysses.dist.get_world_size = orig


def _oracle_fwd_train(q, k, v, tq, tk, tv, scale):
    o, to, lse = _oracle_fn(q, k, v, tq, tk, tv, scale)
    return o, to, lse, torch.zeros_like(lse)  # the oracle backward recomputes everything it needs


def _oracle_bwd(q, k, v, tq, tk, tv, o, to, lse, mu, dout, dtout, scale):
    import oracle
    g = oracle.attn_jvp_bwd(q, k, v, tq, tk, tv, dout, dtout, scale)
    return {n: torch.from_numpy(x) for n, x in g.items()}


def _bwd_worker(rank, world, port, shape, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from attention_forward_mode_b200.ulysses import ulysses_attn_jvp_bwd, ulysses_attn_jvp_train
        B, H, Lq, Lk, d = shape
        full = _inputs(B, H, Lq, Lk, d, seed=11)
        g = torch.Generator().manual_seed(12)
        cot = {n: torch.randn((B, H, Lq, d), generator=g, dtype=torch.float64) for n in ("dout", "dtout")}
        sq, sk = Lq // world, Lk // world
        qsl, ksl = slice(rank * sq, (rank + 1) * sq), slice(rank * sk, (rank + 1) * sk)
        shard = {n: (t[:, :, qsl] if n in ("q", "tq") else t[:, :, ksl]).contiguous() for n, t in full.items()}
        o, to, lse, ctx = ulysses_attn_jvp_train(*(shard[n] for n in ("q", "k", "v", "tq", "tk", "tv")), scale=0.3,
                                                 local_fwd=_oracle_fwd_train)
        grads = ulysses_attn_jvp_bwd(ctx, cot["dout"][:, :, qsl].contiguous(), cot["dtout"][:, :, qsl].contiguous(),
                                     local_bwd=_oracle_bwd)
        ref = _oracle_bwd(*(full[n] for n in ("q", "k", "v", "tq", "tk", "tv")), None, None, None, None,
                          cot["dout"], cot["dtout"], 0.3)
        eq = {n: bool(torch.equal(grads[n], ref[n][:, :, qsl if n in ("dq", "dtq") else ksl])) for n in ref}
        out[rank] = (eq, {n: tuple(t.shape) for n, t in grads.items()})
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(300)
@pytest.mark.parametrize("world,shape", [(2, (1, 4, 16, 24, 8)),   # cross-attention shapes
                                         (4, (1, 8, 32, 32, 4))])  # four ranks
def test_ulysses_backward_matches_unsharded(world, shape):
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        procs = [ctx.Process(target=_bwd_worker, args=(r, world, port, shape, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(240)
        assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
        res = dict(out)
    B, H, Lq, Lk, d = shape
    for r in range(world):
        eq, shapes = res[r]
        assert all(eq.values()), (r, eq)
        assert shapes["dq"] == (B, H, Lq // world, d) and shapes["dk"] == (B, H, Lk // world, d)


def test_single_rank_backward_is_the_local_call():
    from attention_forward_mode_b200.ulysses import ulysses_attn_jvp_bwd, ulysses_attn_jvp_train
    t = _inputs(1, 2, 8, 6, 4, seed=3)
    names = ("q", "k", "v", "tq", "tk", "tv")
    _, _, _, ctx = ulysses_attn_jvp_train(*(t[n] for n in names), scale=0.5, local_fwd=_oracle_fwd_train)
    dout, dtout = torch.ones(1, 2, 8, 4, dtype=torch.float64), torch.full((1, 2, 8, 4), 0.5, dtype=torch.float64)
    a = ulysses_attn_jvp_bwd(ctx, dout, dtout, local_bwd=_oracle_bwd)
    b = _oracle_bwd(*(t[n] for n in names), None, None, None, None, dout, dtout, 0.5)
    for n in b:
        assert torch.equal(a[n], b[n])


def _causal_fwd_train(q, k, v, tq, tk, tv, scale):
    import oracle
    o, to, lse = (torch.from_numpy(x) for x in oracle.attn_jvp_causal(q, k, v, tq, tk, tv, scale))
    return o, to, lse, torch.zeros_like(lse)  # the oracle backward recomputes everything it needs


def _causal_bwd(q, k, v, tq, tk, tv, o, to, lse, mu, dout, dtout, scale):
    import oracle
    g = oracle.attn_jvp_bwd_causal(q, k, v, tq, tk, tv, dout, dtout, scale)
    return {n: torch.from_numpy(x) for n, x in g.items()}


def _causal_worker(rank, world, port, shape, out):
    # the causal mask needs every row's global position: after the exchange a rank
    # holds whole sequences in order, so the sharded result equals the unsharded one
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from attention_forward_mode_b200.ulysses import ulysses_attn_jvp_bwd, ulysses_attn_jvp_train
        B, H, Lq, Lk, d = shape
        names = ("q", "k", "v", "tq", "tk", "tv")
        full = _inputs(B, H, Lq, Lk, d, seed=13)
        g = torch.Generator().manual_seed(14)
        cot = {n: torch.randn((B, H, Lq, d), generator=g, dtype=torch.float64) for n in ("dout", "dtout")}
        sq, sk = Lq // world, Lk // world
        qsl, ksl = slice(rank * sq, (rank + 1) * sq), slice(rank * sk, (rank + 1) * sk)
        shard = {n: (t[:, :, qsl] if n in ("q", "tq") else t[:, :, ksl]).contiguous() for n, t in full.items()}
        o, to, lse, ctx = ulysses_attn_jvp_train(*(shard[n] for n in names), scale=0.3, local_fwd=_causal_fwd_train,
                                                 causal=True)
        grads = ulysses_attn_jvp_bwd(ctx, cot["dout"][:, :, qsl].contiguous(), cot["dtout"][:, :, qsl].contiguous(),
                                     local_bwd=_causal_bwd)
        ro, rto, rlse, _ = _causal_fwd_train(*(full[n] for n in names), 0.3)
        ref = _causal_bwd(*(full[n] for n in names), None, None, None, None, cot["dout"], cot["dtout"], 0.3)
        eq = {n: bool(torch.equal(grads[n], ref[n][:, :, qsl if n in ("dq", "dtq") else ksl])) for n in ref}
        eq["o"] = bool(torch.equal(o, ro[:, :, qsl]))
        eq["to"] = bool(torch.equal(to, rto[:, :, qsl]))
        eq["lse"] = bool(torch.equal(lse, rlse[:, :, qsl]))
        out[rank] = eq
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(300)
@pytest.mark.parametrize("world,shape", [(2, (1, 4, 16, 24, 8)), (4, (1, 4, 32, 16, 4))])
def test_ulysses_causal_matches_unsharded(world, shape):
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        procs = [ctx.Process(target=_causal_worker, args=(r, world, port, shape, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(240)
        assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
        res = dict(out)
    for r in range(world):
        assert all(res[r].values()), (r, res[r])


def _dropout_worker(rank, world, port, out):
    # rank 1 leaves before the exchange; rank 0's all-to-all must end with an error
    # (the peer's connection closes, or the short process-group timeout expires),
    # not wait for good
    import datetime
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=5))
    if rank == 1:
        out[rank] = "left"
        os._exit(0)  # no collective, no clean shutdown: the rank is simply gone
    try:
        from attention_forward_mode_b200.ulysses import ulysses_attn_jvp
        t = _inputs(1, 2, 8, 8, 4, seed=1)
        shard = {n: x[:, :, :4].contiguous() for n, x in t.items()}
        ulysses_attn_jvp(shard["q"], shard["k"], shard["v"], shard["tq"], shard["tk"], shard["tv"], scale=0.5,
                         local_fn=_oracle_fn)
        out[rank] = "completed"
    except Exception as e:  # the expected outcome
        out[rank] = f"raised {type(e).__name__}"


@pytest.mark.timeout(120)
def test_ulysses_peer_loss_raises_instead_of_hanging():
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        procs = [ctx.Process(target=_dropout_worker, args=(r, 2, port, out)) for r in range(2)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(90)
        alive = [p.is_alive() for p in procs]
        for p in procs:
            if p.is_alive():
                p.kill()
        res = dict(out)
    assert not any(alive), (alive, res)
    assert res.get(1) == "left" and str(res.get(0, "")).startswith("raised"), res
