"""Ulysses sequence parallelism on the CPU: the layout steps, the single-device emulation
and the real all-to-all exchanges over gloo (world sizes 2 and 4), forward and backward,
with the fp64 oracle in place of the GPU kernels and a plain tensor transpose in place of
the relayout kernel.  Every result must equal the oracle's attention (and gradients) over
the whole sequence."""
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
from long_context_attention_fwd_b200 import ulysses as U  # noqa: E402

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def cpu_transpose(x, n_outer, n_inner):
    return x.reshape(n_outer, n_inner, -1).transpose(0, 1).contiguous()


def _tok(t):
    B, S, H, D = t.shape
    return t.detach().numpy().reshape(B * S, H, D)


def oracle_fwd(q, k, v, causal, scale, cu=None):
    if cu is not None:   # packed: [T][H][D] with the batch's offsets
        o, lse = oracle.fwd(*(t.detach().numpy() for t in (q, k, v)), causal, scale,
                            cu_seqlens=np.asarray(cu, dtype=np.int32))
        return torch.from_numpy(np.ascontiguousarray(o)), torch.from_numpy(lse)
    B, S, Hq, D = q.shape
    o, lse = oracle.fwd(_tok(q), _tok(k), _tok(v), causal, scale, B=B, S=S)
    return torch.from_numpy(np.ascontiguousarray(o)).reshape(q.shape), torch.from_numpy(lse)


def oracle_bwd(q, k, v, o, lse, do, causal, scale, cu=None):
    if cu is not None:
        g = oracle.bwd(*(t.detach().numpy() for t in (q, k, v, do)), causal, scale,
                       cu_seqlens=np.asarray(cu, dtype=np.int32))
        return tuple(torch.from_numpy(np.ascontiguousarray(x)) for x in g)
    B, S = q.shape[:2]
    g = oracle.bwd(_tok(q), _tok(k), _tok(v), _tok(do), causal, scale, B=B, S=S)
    return tuple(torch.from_numpy(np.ascontiguousarray(x)).reshape(t.shape)
                 for x, t in zip(g, (q, k, v)))


HOOKS = U.Hooks(fwd=oracle_fwd, bwd=oracle_bwd, transpose=cpu_transpose)


def problem(B, S, Hq, Hkv, D, seed):
    def t(h, sub):
        return torch.from_numpy(I.normal(I.stream_key(seed, sub), B * S * h * D)
                                .reshape(B, S, h, D) * 0.7)
    return t(Hq, 1), t(Hkv, 2), t(Hkv, 3), t(Hq, 4)


def reference(q, k, v, do, causal, scale):
    B, S = q.shape[:2]
    o, _ = oracle.fwd(_tok(q), _tok(k), _tok(v), causal, scale, B=B, S=S)
    g = oracle.bwd(_tok(q), _tok(k), _tok(v), _tok(do), causal, scale, B=B, S=S)
    return [x.reshape(t.shape) for x, t in zip((o,) + tuple(g), (q, q, k, v))]


@pytest.mark.parametrize("B", [1, 3])
def test_layout_steps_round_trip(B):
    N, C, H, D = 4, 5, 8, 2
    x = torch.arange(B * C * H * D, dtype=torch.float64).reshape(B, C, H, D)
    s = U.seq_to_send(x, N, cpu_transpose)
    for p in range(N):                      # chunk p = the heads of rank p
        assert torch.equal(s[p], x[:, :, p * (H // N):(p + 1) * (H // N)])
    assert torch.equal(U.recv_to_seq(s, cpu_transpose), x)
    full = torch.arange(B * N * C * 2 * D, dtype=torch.float64).reshape(B, N * C, 2, D)
    snd = U.full_to_send(full, N, cpu_transpose)
    for p in range(N):                      # chunk p = the tokens of rank p
        assert torch.equal(snd[p], full[:, p * C:(p + 1) * C])
    assert torch.equal(U.recv_to_full(snd, cpu_transpose), full)


def test_split_must_divide_heads():
    with pytest.raises(ValueError):
        U.check_split(28, 4, 8)
    U.check_split(28, 4, 4)


@pytest.mark.parametrize("world,causal,B", [(2, True, 1), (4, True, 2), (4, False, 1)])
def test_single_device_emulation(world, causal, B):
    q, k, v, do = problem(B, 24, 8, 4, 4, 3)
    got = U.ulysses_attention_single_device(q, k, v, world, causal, 0.4, do=do, hooks=HOOKS)
    for g, r in zip(got, reference(q, k, v, do, causal, 0.4)):
        np.testing.assert_allclose(g.numpy(), r, atol=1e-12)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, causal, B, q_out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        S = 8 * world
        q, k, v, do = problem(B, S, 2 * world, world, 4, 11)
        C = S // world
        sl = slice(rank * C, (rank + 1) * C)
        ql, kl, vl = (t[:, sl].contiguous().requires_grad_(True) for t in (q, k, v))
        o = U.ulysses_attention(ql, kl, vl, causal, 0.3, hooks=HOOKS)
        o.backward(do[:, sl].contiguous())
        ref = reference(q, k, v, do, causal, 0.3)
        errs = [float(np.abs(x.detach().numpy() - r[:, sl]).max())
                for x, r in zip((o, ql.grad, kl.grad, vl.grad), ref)]
        q_out.put((rank, errs))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,causal,B", [(2, True, 1), (4, True, 2), (4, False, 1)])
def test_gloo_all_to_all_forward_and_backward(world, causal, B):
    ctx = mp.get_context("spawn")
    q_out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, causal, B, q_out))
             for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q_out.get(timeout=180) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r for r, _ in res] == list(range(world))
    for r, errs in res:
        assert max(errs) < 1e-12, (r, errs)


# ---------------------------------------------------------------- packed batches
LENS = [5, 11, 1, 7, 0, 8]          # T = 32; the rank slices cut sequences mid-way


def packed_problem(Hq, Hkv, D, seed):
    T = sum(LENS)
    def t(h, sub):
        return torch.from_numpy(I.normal(I.stream_key(seed, sub), T * h * D).reshape(T, h, D) * 0.7)
    return t(Hq, 1), t(Hkv, 2), t(Hkv, 3), t(Hq, 4), I.cu_seqlens_from(LENS)


def packed_reference(q, k, v, do, cu, causal, scale):
    o, _ = oracle.fwd(q.numpy(), k.numpy(), v.numpy(), causal, scale, cu_seqlens=cu)
    g = oracle.bwd(q.numpy(), k.numpy(), v.numpy(), do.numpy(), causal, scale, cu_seqlens=cu)
    return (o,) + tuple(g)


@pytest.mark.parametrize("world,causal", [(2, True), (4, True), (4, False)])
def test_single_device_emulation_packed(world, causal):
    q, k, v, do, cu = packed_problem(8, 4, 4, 21)
    got = U.ulysses_attention_single_device(q, k, v, world, causal, 0.4, do=do, hooks=HOOKS,
                                            cu_seqlens=torch.from_numpy(cu))
    for g, r in zip(got, packed_reference(q, k, v, do, cu, causal, 0.4)):
        assert g.shape == r.shape
        np.testing.assert_allclose(g.numpy(), r, atol=1e-12)


def _worker_packed(rank, world, port, causal, q_out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        q, k, v, do, cu = packed_problem(2 * world, world, 4, 23)
        C = q.shape[0] // world
        sl = slice(rank * C, (rank + 1) * C)
        ql, kl, vl = (t[sl].contiguous().requires_grad_(True) for t in (q, k, v))
        o = U.ulysses_attention(ql, kl, vl, causal, 0.3, hooks=HOOKS,
                                cu_seqlens=torch.from_numpy(cu))
        o.backward(do[sl].contiguous())
        ref = packed_reference(q, k, v, do, cu, causal, 0.3)
        errs = [float(np.abs(x.detach().numpy() - r[sl]).max())
                for x, r in zip((o, ql.grad, kl.grad, vl.grad), ref)]
        q_out.put((rank, errs))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,causal", [(2, True), (4, False)])
def test_gloo_all_to_all_packed(world, causal):
    ctx = mp.get_context("spawn")
    q_out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker_packed, args=(r, world, port, causal, q_out))
             for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q_out.get(timeout=180) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r for r, _ in res] == list(range(world))
    for r, errs in res:
        assert max(errs) < 1e-12, (r, errs)
