"""attn_bwd_noalloc: the backward for callers that cannot allocate device memory --
integrations with no device allocator where they call the backward, or runtimes
that reserve all device memory up front.  It works in a fixed scratch array inside
the library, so it must give the gradients attn_bwd gives with a caller-owned
workspace, on every call (the array keeps the previous call's contents), and it
must refuse problems whose workspace does not fit the array.

This file is collected last on purpose, so that a run stopping at its first
failure has already run every other test."""
import numpy as np
import pytest

from helpers import TOL_GRAD, make_case, rel_l2, torch_bf16
from long_context_attention_fwd_b200 import capi
from long_context_attention_fwd_b200 import inputs as I

torch = pytest.importorskip("torch")

CASES = [
    ("dense_gqa4x2_S1000_D128_causal", make_case(1, 4, 2, 1000, 128, True, seed=31)),
    ("packed_mha2_D64_full", make_case(0, 2, 2, 0, 64, False, seed=32, lens=[300, 0, 1, 513, 129])),
]


def _tensors(w):
    x = I.make_inputs(w)
    dense = w.varlen is None
    T = w.tokens
    shp_q = (w.B, w.S, w.Hq, w.D) if dense else (T, w.Hq, w.D)
    shp_k = (w.B, w.S, w.Hkv, w.D) if dense else (T, w.Hkv, w.D)
    q = torch_bf16(x["q"]).view(shp_q)
    k = torch_bf16(x["k"]).view(shp_k)
    v = torch_bf16(x["v"]).view(shp_k)
    do = torch_bf16(x["do"]).view(shp_q)
    cu = None if dense else torch.from_numpy(x["cu_seqlens"]).cuda()
    B = w.B if dense else len(w.varlen)
    S = w.S if dense else T
    return q, k, v, do, cu, B, S


@pytest.mark.gpu
@pytest.mark.parametrize("name,w", CASES, ids=[c[0] for c in CASES])
def test_noalloc_matches_workspace_backward_on_consecutive_calls(name, w):
    from long_context_attention_fwd_b200 import ops
    q, k, v, do, cu, B, S = _tensors(w)
    scale = w.softmax_scale
    o, lse = ops.attn_fwd(q, k, v, causal=w.causal, scale=scale, cu_seqlens=cu)
    ref = ops.attn_bwd(q, k, v, o, lse, do, causal=w.causal, scale=scale, cu_seqlens=cu)
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream().cuda_stream
    for call in range(2):
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        for t in (dq, dk, dv):
            t.view(torch.int16).fill_(0x7FC0)  # NaN poison: every element must be written
        st = capi.attn_bwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                   lse.data_ptr(), do.data_ptr(), dq.data_ptr(), dk.data_ptr(),
                                   dv.data_ptr(), B, w.Hq, w.Hkv, S, w.D, w.causal, scale,
                                   cu.data_ptr() if cu is not None else None, stream)
        capi.check(st, "attn_bwd_noalloc")
        torch.cuda.synchronize()
        st, site = capi.attn_device_status(None)
        assert st == capi.ATTN_OK, (st, hex(site))
        for got, want, label in ((dq, ref[0], "dq"), (dk, ref[1], "dk"), (dv, ref[2], "dv")):
            g = got.float().cpu().numpy()
            assert np.isfinite(g).all(), (call, label)
            e = rel_l2(g, want.float().cpu().numpy())
            assert e <= TOL_GRAD, (call, label, e)


@pytest.mark.gpu
def test_noalloc_refuses_problems_larger_than_its_scratch():
    q = torch.zeros(1, 128, 2, 128, device="cuda", dtype=torch.bfloat16)
    lse = torch.zeros(1, 2, 128, device="cuda")
    # S = 65536 with 28 heads needs ~0.9 GB of workspace: far above the scratch size.
    st = capi.attn_bwd_noalloc(*([q.data_ptr()] * 4), lse.data_ptr(), *([q.data_ptr()] * 4),
                               1, 28, 4, 65536, 128, 1, 0.1, None, None)
    assert st == capi.ATTN_ERR_INVALID_ARG
    assert "exceeds the static scratch" in capi.attn_last_error()
