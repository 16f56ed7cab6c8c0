"""The Ulysses wrapper on the GPU, checked against the fp64 oracle.

1. One-rank NCCL group: the all-to-all exchanges run for real (as identity
   exchanges) around the CUDA kernels.  The result must equal the direct
   calls bit for bit AND the oracle within the bf16 bounds (O 1e-2, tO 2e-2,
   lse 1e-3; each gradient 2e-2), for the forward, the training forward and
   backward, and the causal training path; self-attention (ragged tails) and
   cross-attention (Lq != Lk).
2. Two and four ranks emulated in threads of one process: the exchange is a
   host-side all_to_all_single (ranks meet at a barrier and copy each
   other's chunks), so the head / sequence permutation of a real multi-rank
   run happens, with the CUDA kernels as the local steps; the gathered
   sequence shards must equal the unsharded oracle.  No kernel waits on
   another rank: the ranks only meet on the host between launches.
"""
import datetime
import socket
import threading

import numpy as np
import pytest
import torch
import torch.distributed as dist

import attention_forward_mode_b200 as ajvp
import attention_forward_mode_b200.ulysses as uly
import oracle
from attention_forward_mode_b200.workloads import custom, make_cotangents, make_inputs
from gpu_common import TOL, max_rel

pytestmark = pytest.mark.gpu

NAMES = ("q", "k", "v", "tq", "tk", "tv")
GTOL = 2e-2  # per gradient, as for the direct backward entry points


def _fwd_err(out, ref):
    o, to, lse = (t.float().cpu().numpy() for t in out)
    return {"o": max_rel(o, ref[0]), "to": max_rel(to, ref[1]), "lse": max_rel(lse, ref[2])}


def _check_fwd(out, ref, what):
    err = _fwd_err(out, ref)
    print(what, err)
    for key in ("o", "to", "lse"):
        assert err[key] <= TOL["bf16"][key], (what, key, err)


def _check_grads(g, ref, what):
    err = {n: max_rel(g[n].float().cpu().numpy(), ref[n]) for n in ajvp.GRAD_NAMES}
    print(what, err)
    for n, e in err.items():
        assert e <= GTOL, (what, n, err)


@pytest.fixture(scope="module")
def nccl_one_rank():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    store = dist.TCPStore("127.0.0.1", port, 1, True, timeout=datetime.timedelta(seconds=60))
    dist.init_process_group("nccl", store=store, rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60), device_id=torch.device("cuda", 0))
    try:
        yield
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("shape", [(1, 4, 384, 640), (2, 2, 520, 520)])
def test_one_rank_nccl_forward(nccl_one_rank, shape):
    w = custom(*shape, 128)
    inp = make_inputs(w, seed=3, device="cuda")
    a = uly.ulysses_attn_jvp(*(inp[n] for n in NAMES), scale=w.scale)
    b = ajvp.attn_jvp_fwd(*(inp[n] for n in NAMES), w.scale)
    torch.cuda.synchronize()
    for x, y in zip(a, b):
        assert torch.equal(x, y)
    ref = oracle.attn_jvp(*(inp[n].cpu() for n in NAMES), w.scale)
    _check_fwd(a, ref, f"ulysses nccl forward {shape}")


@pytest.mark.parametrize("shape", [(1, 4, 384, 640), (2, 2, 520, 520)])
def test_one_rank_nccl_training(nccl_one_rank, shape):
    w = custom(*shape, 128)
    inp = make_inputs(w, seed=3, device="cuda")
    cot = make_cotangents(w, seed=4, device="cuda")
    o, to, lse, ctx = uly.ulysses_attn_jvp_train(*(inp[n] for n in NAMES), scale=w.scale)
    g = uly.ulysses_attn_jvp_bwd(ctx, cot["dout"], cot["dtout"])
    ro, rto, rlse, rmu = ajvp.attn_jvp_fwd_stats(*(inp[n] for n in NAMES), w.scale)
    rg = ajvp.attn_jvp_bwd(*(inp[n] for n in NAMES), ro, rto, rlse, rmu, cot["dout"], cot["dtout"], w.scale)
    torch.cuda.synchronize()
    assert torch.equal(o, ro) and torch.equal(to, rto) and torch.equal(lse, rlse)
    for n in ajvp.GRAD_NAMES:
        assert torch.equal(g[n], rg[n]), n
    cpu = {n: t.cpu() for n, t in inp.items()}
    _check_fwd((o, to, lse), oracle.attn_jvp(*(cpu[n] for n in NAMES), w.scale), f"ulysses train fwd {shape}")
    ref = oracle.attn_jvp_bwd(*(cpu[n] for n in NAMES), cot["dout"].cpu(), cot["dtout"].cpu(), w.scale)
    _check_grads(g, ref, f"ulysses train bwd {shape}")


def test_one_rank_nccl_causal_training(nccl_one_rank):
    # Lq < Lk: every row sees at least Lk - Lq + 1 keys (bottom-right aligned mask)
    w = custom(1, 4, 384, 640, 128)
    inp = make_inputs(w, seed=5, device="cuda")
    cot = make_cotangents(w, seed=6, device="cuda")
    o, to, lse, ctx = uly.ulysses_attn_jvp_train(*(inp[n] for n in NAMES), scale=w.scale, causal=True)
    g = uly.ulysses_attn_jvp_bwd(ctx, cot["dout"], cot["dtout"])
    ro, rto, rlse, rmu = ajvp.attn_jvp_fwd_causal_stats(*(inp[n] for n in NAMES), w.scale)
    rg = ajvp.attn_jvp_bwd_causal(*(inp[n] for n in NAMES), ro, rto, rlse, rmu, cot["dout"], cot["dtout"], w.scale)
    torch.cuda.synchronize()
    assert torch.equal(o, ro) and torch.equal(to, rto) and torch.equal(lse, rlse)
    for n in ajvp.GRAD_NAMES:
        assert torch.equal(g[n], rg[n]), n
    cpu = {n: t.cpu() for n, t in inp.items()}
    _check_fwd((o, to, lse), oracle.attn_jvp_causal(*(cpu[n] for n in NAMES), w.scale), "ulysses causal fwd")
    ref = oracle.attn_jvp_bwd_causal(*(cpu[n] for n in NAMES), cot["dout"].cpu(), cot["dtout"].cpu(), w.scale)
    _check_grads(g, ref, "ulysses causal bwd")


# ---------------------------------------------------------------- emulated ranks
class _Exchange:
    """World-wide state of the emulated ranks: one slot per rank and a barrier."""

    def __init__(self, world):
        self.world = world
        self.slots = [None] * world
        self.barrier = threading.Barrier(world, timeout=120)


class _Group:
    def __init__(self, ex, rank):
        self.ex, self.rank = ex, rank


class _HostDist:
    """The three torch.distributed calls the wrapper makes, for ranks that are
    threads of one process.  all_to_all_single with equal splits: chunk p of
    rank r's send buffer becomes chunk r of rank p's receive buffer."""

    @staticmethod
    def is_initialized():
        return True

    @staticmethod
    def get_world_size(group=None):
        return group.ex.world

    @staticmethod
    def all_to_all_single(recv, send, group=None):
        ex, r = group.ex, group.rank
        ex.barrier.wait()  # every rank has finished reading the previous exchange
        ex.slots[r] = send
        ex.barrier.wait()  # every rank's send buffer is posted
        for p in range(ex.world):
            recv[p].copy_(ex.slots[p][r])
        torch.cuda.synchronize()


def _run_ranks(world, fn):
    """fn(rank, group) on `world` threads; returns the per-rank results."""
    ex = _Exchange(world)
    res, errs = [None] * world, []

    def body(r):
        try:
            res[r] = fn(r, _Group(ex, r))
        except BaseException as e:  # noqa: BLE001 -- re-raised below
            errs.append(e)
            ex.barrier.abort()

    ts = [threading.Thread(target=body, args=(r,)) for r in range(world)]
    for t in ts:
        t.start()
    for t in ts:
        t.join()
    if errs:
        raise errs[0]
    return res


def _shard(x, r, world):
    L = x.shape[2]
    return x[:, :, r * L // world:(r + 1) * L // world].contiguous()


@pytest.mark.parametrize("world,shape", [(2, (1, 4, 512, 768)), (4, (2, 4, 640, 640))])
def test_emulated_ranks_forward_and_training(monkeypatch, world, shape):
    monkeypatch.setattr(uly, "dist", _HostDist)
    w = custom(*shape, 128)
    inp = make_inputs(w, seed=7, device="cuda")
    cot = make_cotangents(w, seed=8, device="cuda")

    def rank_fn(r, grp):
        sh = {n: _shard(t, r, world) for n, t in inp.items()}
        fwd = uly.ulysses_attn_jvp(*(sh[n] for n in NAMES), scale=w.scale, group=grp)
        o, to, lse, ctx = uly.ulysses_attn_jvp_train(*(sh[n] for n in NAMES), scale=w.scale, group=grp)
        g = uly.ulysses_attn_jvp_bwd(ctx, _shard(cot["dout"], r, world), _shard(cot["dtout"], r, world), group=grp)
        torch.cuda.synchronize()
        return fwd, (o, to, lse), g

    res = _run_ranks(world, rank_fn)
    cat = lambda xs: torch.cat(xs, dim=2)  # noqa: E731 -- sequence shards back in order
    fwd = tuple(cat([res[r][0][i] for r in range(world)]) for i in range(3))
    trn = tuple(cat([res[r][1][i] for r in range(world)]) for i in range(3))
    g = {n: cat([res[r][2][n] for r in range(world)]) for n in ajvp.GRAD_NAMES}
    # heads are independent, so the sharded run equals the unsharded kernel bit for bit
    direct = ajvp.attn_jvp_fwd(*(inp[n] for n in NAMES), w.scale)
    torch.cuda.synchronize()
    for x, y in zip(fwd, direct):
        assert torch.equal(x, y)
    for x, y in zip(trn, direct):
        assert torch.equal(x, y)
    cpu = {n: t.cpu() for n, t in inp.items()}
    ref = oracle.attn_jvp(*(cpu[n] for n in NAMES), w.scale)
    _check_fwd(fwd, ref, f"emulated {world} ranks forward")
    _check_fwd(trn, ref, f"emulated {world} ranks training forward")
    gref = oracle.attn_jvp_bwd(*(cpu[n] for n in NAMES), cot["dout"].cpu(), cot["dtout"].cpu(), w.scale)
    _check_grads(g, gref, f"emulated {world} ranks backward")


def test_emulated_ranks_causal(monkeypatch):
    monkeypatch.setattr(uly, "dist", _HostDist)
    world = 2
    w = custom(1, 2, 512, 512, 128)
    inp = make_inputs(w, seed=9, device="cuda")
    cot = make_cotangents(w, seed=10, device="cuda")

    def rank_fn(r, grp):
        sh = {n: _shard(t, r, world) for n, t in inp.items()}
        o, to, lse, ctx = uly.ulysses_attn_jvp_train(*(sh[n] for n in NAMES), scale=w.scale, group=grp,
                                                     causal=True)
        g = uly.ulysses_attn_jvp_bwd(ctx, _shard(cot["dout"], r, world), _shard(cot["dtout"], r, world), group=grp)
        torch.cuda.synchronize()
        return (o, to, lse), g

    res = _run_ranks(world, rank_fn)
    out = tuple(torch.cat([res[r][0][i] for r in range(world)], dim=2) for i in range(3))
    g = {n: torch.cat([res[r][1][n] for r in range(world)], dim=2) for n in ajvp.GRAD_NAMES}
    cpu = {n: t.cpu() for n, t in inp.items()}
    _check_fwd(out, oracle.attn_jvp_causal(*(cpu[n] for n in NAMES), w.scale), "emulated causal forward")
    gref = oracle.attn_jvp_bwd_causal(*(cpu[n] for n in NAMES), cot["dout"].cpu(), cot["dtout"].cpu(), w.scale)
    # row 0 sees one key: its exact dq, dtq vanish and the kernel's are bounded by the
    # bf16 row statistics' leak (the causal backward tests hold that row to its own
    # bound); over the whole tensor of this short problem the relative bound holds
    _check_grads(g, gref, "emulated causal backward")
    assert np.isfinite(g["dq"].float().cpu().numpy()).all()
