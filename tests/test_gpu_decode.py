"""Decode attention over a key/value cache (attn_decode) on the GPU against the fp64
oracle, element by element: every output row of every workload.

The caches hold bf16 NaN past each sequence's length, so a read of any entry past the
length would show up as NaN in the output.  Cases cover lengths on and around the
128-key tile edges (0, 1, 127, 128, 129, ...), grouped-query ratios 1, 7 and 64 (the
last needs two warps of rows per stream), both head dimensions, the split plans of a
single 32K sequence (64 splits) and of 16 sequences of 16K-32K keys, and determinism.
"""
import numpy as np
import pytest

import oracle
from helpers import TOL_LSE, bits_of, f64, o_error_report, torch_bf16
from long_context_attention_fwd_b200 import inputs as I

torch = pytest.importorskip("torch")


def _run(w):
    from long_context_attention_fwd_b200 import ops
    x = I.make_decode_inputs(w, poison_tail=True)
    q = torch_bf16(x["q"]).view(w.B, w.Hq, w.D)
    k = torch_bf16(x["k"]).view(w.B, w.Lmax, w.Hkv, w.D)
    v = torch_bf16(x["v"]).view(w.B, w.Lmax, w.Hkv, w.D)
    cl = torch.from_numpy(x["cache_len"]).cuda()
    o = torch.empty_like(q)
    o.view(torch.int16).fill_(0x7FC0)
    lse = torch.full((w.B, w.Hq), float("nan"), device="cuda")
    o, lse = ops.attn_decode(q, k, v, cl, scale=w.softmax_scale, out=o, lse=lse)
    torch.cuda.synchronize()
    from long_context_attention_fwd_b200 import capi
    st, site = capi.attn_device_status(None)   # no wait or drain may have run out
    assert st == capi.ATTN_OK, (capi.strerror(st), hex(site))
    return x, o, lse


def _check(w, x, o, lse):
    # oracle on the same bits, with the poisoned tail replaced by zeros (never read)
    kf, vf = f64(x["k"]).copy(), f64(x["v"]).copy()
    for b, L in enumerate(w.lens):
        kf[b, L:] = 0.0
        vf[b, L:] = 0.0
    qf = f64(x["q"])
    o_r, l_r = oracle.decode(qf, kf, vf, x["cache_len"], w.softmax_scale)
    oa_r, _ = oracle.decode(qf, kf, np.abs(vf), x["cache_len"], w.softmax_scale)
    og = f64(bits_of(o)).reshape(w.B, w.Hq, w.D)
    lg = lse.double().cpu().numpy()
    empty = np.array(w.lens) == 0
    assert not np.isnan(og).any() and not np.isnan(lg).any()
    assert (og[empty] == 0).all() and np.isneginf(lg[empty]).all()
    full = ~empty
    rep = o_error_report(og[full], o_r[full], oa_r[full])
    assert rep["n_over_model"] == 0 and rep["max_abs"] <= 1e-2, rep
    assert np.abs(lg[full] - l_r[full]).max() <= TOL_LSE
    return rep


CASES = [
    I.decode_workload(0),
    I.DecodeWorkload("decode_gqa7_D128", B=3, Hq=28, Hkv=4, Lmax=1000, D=128,
                     lens=[1000, 385, 129], seed=41),
    I.DecodeWorkload("decode_mqa64_D128", B=2, Hq=64, Hkv=1, Lmax=520, D=128, lens=[520, 1],
                     seed=42),
    I.DecodeWorkload("decode_mha_D64", B=2, Hq=8, Hkv=8, Lmax=300, D=64, lens=[300, 0], seed=43),
    I.DecodeWorkload("decode_one_tile_D128", B=4, Hq=28, Hkv=4, Lmax=128, D=128,
                     lens=[128, 64, 1, 127], seed=44),
]


@pytest.mark.gpu
@pytest.mark.parametrize("w", CASES, ids=[c.name for c in CASES])
def test_decode_small_matches_oracle(w):
    x, o, lse = _run(w)
    _check(w, x, o, lse)


@pytest.mark.gpu
@pytest.mark.parametrize("idx", [1, 2], ids=["B1_L32K", "B16_L16K-32K"])
def test_decode_full_size_matches_oracle(idx):
    w = I.decode_workload(idx)
    x, o, lse = _run(w)
    _check(w, x, o, lse)


@pytest.mark.gpu
def test_decode_deterministic():
    w = CASES[1]
    _, o1, l1 = _run(w)
    _, o2, l2 = _run(w)
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16)) and torch.equal(l1, l2)


@pytest.mark.gpu
def test_decode_workspace_needs_no_initialisation():
    """The splits of a (sequence, kv head) mark themselves done in the workspace, and one
    that sees them all done merges.  Whatever the workspace holds when a call starts (all
    ones, random bytes, the previous call's leftovers) the result must be the same, bit for
    bit, and a call leaves its done flags cleared.  Replaying one captured launch (same call tag)
    must also give the same result every time."""
    from long_context_attention_fwd_b200 import ops
    w = I.DecodeWorkload("decode_ws_reuse", B=3, Hq=28, Hkv=4, Lmax=2000, D=128,
                         lens=[2000, 1, 777], seed=45)
    x = I.make_decode_inputs(w, poison_tail=True)
    q = torch_bf16(x["q"]).view(w.B, w.Hq, w.D)
    k = torch_bf16(x["k"]).view(w.B, w.Lmax, w.Hkv, w.D)
    v = torch_bf16(x["v"]).view(w.B, w.Lmax, w.Hkv, w.D)
    cl = torch.from_numpy(x["cache_len"]).cuda()
    nbytes = ops.attn_decode_workspace_size(q, k)
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    # the workspace is nsplit bf16 partials, their fp32 lse rows, then one 8-byte done flag
    # per (sequence, kv head, split), each part rounded up to 256 bytes; find nsplit
    up = lambda x: -(-x // 256) * 256
    rows = w.B * w.Hq
    nsplit = next(n for n in range(1, 129)
                  if up(n * rows * w.D * 2) + up(n * rows * 4) + up(w.B * w.Hkv * n * 8) == nbytes)
    flag_at, flag_bytes = nbytes - up(w.B * w.Hkv * nsplit * 8), w.B * w.Hkv * nsplit * 8
    outs = []
    gen = torch.Generator(device="cuda").manual_seed(3)
    for fill in ("ones", "random", "leftover", "leftover"):
        if fill == "ones":
            ws.fill_(0xFF)
        elif fill == "random":
            ws.copy_(torch.randint(0, 256, (nbytes,), generator=gen, device="cuda",
                                   dtype=torch.int32).to(torch.uint8))
        o = torch.full_like(q, float("nan"))
        lse = torch.full((w.B, w.Hq), float("nan"), device="cuda")
        ops.attn_decode(q, k, v, cl, scale=w.softmax_scale, out=o, lse=lse, workspace=ws)
        torch.cuda.synchronize()
        assert (ws[flag_at:flag_at + flag_bytes] == 0).all(), fill
        outs.append((o.clone(), lse.clone()))
    _check(w, x, *outs[0])
    for o, lse in outs[1:]:
        assert torch.equal(o.view(torch.int16), outs[0][0].view(torch.int16))
        assert torch.equal(lse, outs[0][1])
    # one captured launch replayed: the call tag repeats, the cleared words make it work
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.Hq), device="cuda")
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        ops.attn_decode(q, k, v, cl, scale=w.softmax_scale, out=o, lse=lse, workspace=ws)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, capture_error_mode="relaxed"):
        ops.attn_decode(q, k, v, cl, scale=w.softmax_scale, out=o, lse=lse, workspace=ws)
    for _ in range(3):
        o.fill_(float("nan"))
        graph.replay()
        torch.cuda.synchronize()
        assert torch.equal(o.view(torch.int16), outs[0][0].view(torch.int16))
        assert torch.equal(lse, outs[0][1])
    del graph
    from long_context_attention_fwd_b200 import capi
    st, site = capi.attn_device_status(None)
    assert st == capi.ATTN_OK, (capi.strerror(st), hex(site))
