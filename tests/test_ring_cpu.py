"""Ring (context-parallel) forward on the CPU: the schedule, the single-device emulation
and the point-to-point ring over gloo (world sizes 2 and 4), with the fp64 oracle put in
place of the GPU kernels.  Each result must equal the oracle's attention over the whole
sequence: this checks which chunk pairs are computed, with which mask, and that every K/V
chunk reaches every rank."""
import datetime
import os
import socket
import sys

import numpy as np
import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402

import oracle  # noqa: E402
from long_context_attention_fwd_b200 import inputs as I  # noqa: E402
from long_context_attention_fwd_b200 import ring  # noqa: E402

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def oracle_attend(q, k, v, causal, scale):
    B, C, Hq, D = q.shape
    tok = lambda t: t.numpy().reshape(B * C, t.shape[2], D)
    o, lse = oracle.fwd(tok(q), tok(k), tok(v), causal, scale, B=B, S=C)
    return torch.from_numpy(np.ascontiguousarray(o)).reshape(q.shape), torch.from_numpy(lse)


def oracle_merge(o_parts, lse_parts):
    B, C, H, D = o_parts[0].shape
    po = [p.numpy().reshape(-1, D) for p in o_parts]                      # rows (b, i, h)
    pl = [l.numpy().transpose(0, 2, 1).reshape(-1) for l in lse_parts]    # same row order
    o, lse = oracle.merge_partials(po, pl)
    return (torch.from_numpy(o).reshape(B, C, H, D),
            torch.from_numpy(np.ascontiguousarray(lse.reshape(B, C, H).transpose(0, 2, 1))))


def full_problem(B, S, Hq, Hkv, D, seed):
    def t(h, sub):
        return torch.from_numpy(I.normal(I.stream_key(seed, sub), B * S * h * D)
                                .reshape(B, S, h, D) * 0.8)
    return t(Hq, 1), t(Hkv, 2), t(Hkv, 3)


@pytest.mark.parametrize("world", [1, 2, 3, 4, 8])
@pytest.mark.parametrize("causal", [True, False])
def test_schedule_covers_each_visible_chunk_once(world, causal):
    for r in range(world):
        sched = ring.ring_schedule(r, world, causal)
        chunks = [j for _, j, _ in sched]
        want = list(range(r + 1)) if causal else list(range(world))
        assert sorted(chunks) == want
        for s, j, c in sched:
            assert j == (r - s) % world          # what the ring has delivered by step s
            assert c == (causal and j == r)      # only the diagonal chunk is masked
        assert [s for s, _, _ in sched] == sorted(s for s, _, _ in sched)


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("world", [2, 4])
def test_single_device_emulation_equals_full_attention(causal, world):
    B, S, Hq, Hkv, D = 2, 48, 4, 2, 8
    q, k, v = full_problem(B, S, Hq, Hkv, D, 5)
    o, lse = ring.ring_attn_fwd_single_device(q, k, v, world, causal, 0.3,
                                              attend=oracle_attend, merge=oracle_merge)
    of, lf = oracle.fwd(q.numpy().reshape(B * S, Hq, D), k.numpy().reshape(B * S, Hkv, D),
                        v.numpy().reshape(B * S, Hkv, D), causal, 0.3, B=B, S=S)
    np.testing.assert_allclose(o.numpy().reshape(of.shape), of, atol=1e-12)
    np.testing.assert_allclose(lse.numpy(), lf, atol=1e-12)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, causal, q_out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        B, S, Hq, Hkv, D = 1, 16 * world, 4, 2, 8
        q, k, v = full_problem(B, S, Hq, Hkv, D, 9)
        C = S // world
        sl = slice(rank * C, (rank + 1) * C)
        o, lse = ring.ring_attn_fwd(q[:, sl].contiguous(), k[:, sl].contiguous(),
                                    v[:, sl].contiguous(), causal, 0.35,
                                    attend=oracle_attend, merge=oracle_merge)
        of, lf = oracle.fwd(q.numpy()[0], k.numpy()[0], v.numpy()[0], causal, 0.35, B=B, S=S)
        err_o = float(np.abs(o.numpy().reshape(C, Hq, D) - of[sl]).max())
        err_l = float(np.abs(lse.numpy()[0] - lf[0][:, sl]).max())
        q_out.put((rank, err_o, err_l))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,causal", [(2, True), (4, True), (4, False)])
def test_gloo_ring_equals_full_attention(world, causal):
    ctx = mp.get_context("spawn")
    q_out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, causal, q_out))
             for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q_out.get(timeout=180) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r for r, _, _ in res] == list(range(world))
    for r, err_o, err_l in res:
        assert err_o < 1e-12, (r, err_o)
        assert err_l < 1e-12, (r, err_l)


# ---------------------------------------------------------------- backward
def oracle_bwd_pair(q, k, v, o, lse, do, causal, scale):
    B, C = q.shape[:2]
    g = oracle.bwd_given(q.numpy().reshape(B * C, q.shape[2], -1), k.numpy().reshape(B * C, k.shape[2], -1),
                         v.numpy().reshape(B * C, v.shape[2], -1), o.numpy().reshape(B * C, o.shape[2], -1),
                         lse.numpy(), do.numpy().reshape(B * C, do.shape[2], -1), causal, scale, B=B, S=C)
    return tuple(torch.from_numpy(np.ascontiguousarray(x)).reshape(t.shape) for x, t in zip(g, (q, k, v)))


def _acc(a, x, init):
    if init:
        a.copy_(x)
    else:
        a.add_(x)
    return a


RING_HOOKS = ring.RingHooks(fwd=oracle_attend, merge=oracle_merge, bwd=oracle_bwd_pair, acc=_acc,
                            cast=lambda a: a.clone(), acc_dtype=torch.float64)


def _full_grads(q, k, v, do, causal, scale):
    B, S, Hq, D = q.shape
    tok = lambda t: t.numpy().reshape(B * S, t.shape[2], D)
    g = oracle.bwd(tok(q), tok(k), tok(v), tok(do), causal, scale, B=B, S=S)
    return [x.reshape(t.shape) for x, t in zip(g, (q, k, v))]


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("world", [2, 3])
def test_single_device_backward_equals_full_gradients(causal, world):
    B, S, Hq, Hkv, D = 2, 12 * world, 4, 2, 4
    q, k, v = full_problem(B, S, Hq, Hkv, D, 21)
    do = torch.from_numpy(I.normal(I.stream_key(21, 9), B * S * Hq * D).reshape(B, S, Hq, D))
    o, lse = ring.ring_attn_fwd_single_device(q, k, v, world, causal, 0.3, attend=oracle_attend,
                                              merge=oracle_merge)
    dq, dk, dv = ring.ring_attn_bwd_single_device(q, k, v, o, lse, do, world, causal, 0.3,
                                                  hooks=RING_HOOKS)
    for got, want in zip((dq, dk, dv), _full_grads(q, k, v, do, causal, 0.3)):
        np.testing.assert_allclose(got.numpy(), want, atol=1e-11)


def _bwd_worker(rank, world, port, causal, q_out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        B, S, Hq, Hkv, D = 1, 8 * world, 4, 2, 4
        q, k, v = full_problem(B, S, Hq, Hkv, D, 23)
        do = torch.from_numpy(I.normal(I.stream_key(23, 9), B * S * Hq * D).reshape(B, S, Hq, D))
        C = S // world
        sl = slice(rank * C, (rank + 1) * C)
        ql, kl, vl = (t[:, sl].contiguous().requires_grad_(True) for t in (q, k, v))
        o = ring.ring_attention(ql, kl, vl, causal, 0.35, hooks=RING_HOOKS)
        o.backward(do[:, sl].contiguous())
        want = _full_grads(q, k, v, do, causal, 0.35)
        errs = [float(np.abs(g.detach().numpy() - w_[:, sl]).max())
                for g, w_ in zip((ql.grad, kl.grad, vl.grad), want)]
        q_out.put((rank, errs))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,causal", [(2, True), (4, True), (3, False)])
def test_gloo_ring_backward_equals_full_gradients(world, causal):
    ctx = mp.get_context("spawn")
    q_out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_bwd_worker, args=(r, world, port, causal, q_out))
             for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q_out.get(timeout=180) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r, errs in res:
        assert max(errs) < 1e-11, (r, errs)


def test_wrappers_refuse_packed_layouts():
    from long_context_attention_fwd_b200 import ulysses
    packed = torch.zeros(64, 4, 8, dtype=torch.float64)
    with pytest.raises(ValueError):
        ring.ring_attn_fwd_single_device(packed, packed, packed, 2)
    with pytest.raises(ValueError):
        ring.ring_attn_bwd_single_device(packed, packed, packed, packed, None, packed, 2)
    with pytest.raises(ValueError):
        ulysses.ulysses_attention_single_device(packed, packed, packed, 2)
