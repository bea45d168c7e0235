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

from helpers import bf16_ulp, make_case, record, rel_l2, torch_bf16
from long_context_attention_fwd_b200 import capi
from long_context_attention_fwd_b200 import inputs as I

torch = pytest.importorskip("torch")

# Sizes on either side of the scratch limit at D = 128: the workspace is
# Hq * ntile * 128 * (4 D + 8) bytes with ntile = (T >> 7) + B, i.e. 66560 bytes per
# (head, 128-row tile); 64 MiB holds 1008.25 of them.  16 heads x 63 tiles (B = 1,
# S = 8000) is the largest problem that fits; 1 head x 1009 tiles is refused.
JUST_BELOW = dict(B=1, Hq=16, Hkv=2, S=8000, D=128)
JUST_ABOVE = dict(B=1, Hq=1, Hkv=1, S=129024, D=128)

CASES = [
    ("dense_gqa4x2_S1000_D128_causal", make_case(1, 4, 2, 1000, 128, True, seed=31)),
    ("packed_mha2_D64_full", make_case(0, 2, 2, 0, 64, False, seed=32, lens=[300, 0, 1, 513, 129])),
    ("limit_gqa16x2_S8000_D128_causal", make_case(1, 16, 2, 8000, 128, True, seed=33)),
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


def _ws_size(B, Hq, S, D, **_):
    return int(capi.lib().attn_bwd_workspace_size(B, Hq, S, D, None))


def test_limit_cases_straddle_the_scratch_size():
    import re
    hdr = open(capi.HEADER).read()
    m = re.search(r"#define ATTN_BWD_NOALLOC_MAX_BYTES \((\d+)u << (\d+)\)", hdr)
    assert m and int(m.group(1)) << int(m.group(2)) == capi.ATTN_BWD_NOALLOC_MAX_BYTES
    assert _ws_size(**JUST_BELOW) <= capi.ATTN_BWD_NOALLOC_MAX_BYTES
    assert _ws_size(**JUST_ABOVE) > capi.ATTN_BWD_NOALLOC_MAX_BYTES
    w = CASES[-1][1]
    assert (w.B, w.Hq, w.Hkv, w.S, w.D) == tuple(JUST_BELOW[n] for n in ("B", "Hq", "Hkv", "S", "D"))


def test_noalloc_refuses_problems_larger_than_its_scratch():
    """Refused before anything touches the GPU: the size check comes first, so the
    pointers (never dereferenced) can be dummies and no device is needed."""
    fake = 1 << 20
    for dims in (JUST_ABOVE, dict(B=1, Hq=28, Hkv=4, S=65536, D=128)):
        st = capi.attn_bwd_noalloc(*([fake] * 5), *([fake] * 4), dims["B"], dims["Hq"],
                                   dims["Hkv"], dims["S"], dims["D"], 1, 0.1, None, None)
        assert st == capi.ATTN_ERR_INVALID_ARG
        assert "exceeds the static scratch" in capi.attn_last_error()
    st = capi.attn_bwd_noalloc(*([fake] * 9), 1, 2, 2, 0, 64, 1, 0.1, None, None)
    assert st == capi.ATTN_ERR_INVALID_ARG and "invalid sizes" in capi.attn_last_error()
    st = capi.attn_bwd_noalloc(None, *([fake] * 8), 1, 2, 2, 128, 64, 1, 0.1, None, None)
    assert st == capi.ATTN_ERR_INVALID_ARG and "null pointer" in capi.attn_last_error()


@pytest.mark.gpu
@pytest.mark.parametrize("name,w", CASES, ids=[c[0] for c in CASES])
def test_noalloc_matches_workspace_backward_on_consecutive_calls(name, w):
    """dk and dv must equal the workspace backward's bit for bit (both are deterministic,
    and both read the LSE and Delta rows the backward keeps in its scratch).  dq is summed
    from per-key-tile partials with fp32 atomics in either run, so it may differ by the
    summation order: the fp32 sums differ by a few fp32 roundings of the partials'
    magnitudes (below 2^-14 of the tensor's largest element at these sizes), and the bf16
    rounding of dq can turn that into one bf16 ulp.  A stale scratch (an accumulator not
    cleared, rows of another call) would show up as errors of the order of dq itself."""
    from long_context_attention_fwd_b200 import ops
    q, k, v, do, cu, B, S = _tensors(w)
    scale = w.softmax_scale
    o, lse = ops.attn_fwd(q, k, v, causal=w.causal, scale=scale, cu_seqlens=cu)
    ref = ops.attn_bwd(q, k, v, o, lse, do, causal=w.causal, scale=scale, cu_seqlens=cu)
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream().cuda_stream
    dq_ref = ref[0].float().cpu().numpy().astype(np.float64)
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
        assert torch.equal(dk, ref[1]), (call, "dk")
        assert torch.equal(dv, ref[2]), (call, "dv")
        g = dq.float().cpu().numpy().astype(np.float64)
        assert np.isfinite(g).all(), call
        diff = np.abs(g - dq_ref)
        bound = bf16_ulp(np.maximum(np.abs(g), np.abs(dq_ref))) + 2.0 ** -14 * np.abs(dq_ref).max()
        e = rel_l2(g, dq_ref)
        record(f"noalloc/{name}/call{call}", dq_max_abs_diff=float(diff.max()),
               dq_n_differ=int((diff > 0).sum()), dq_rel_l2=e,
               dq_worst_diff_over_bound=float((diff / bound).max()))
        assert (diff <= bound).all(), (call, "dq")
        assert e <= 1e-3, (call, e)
