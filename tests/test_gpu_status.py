"""Failure detection on the GPU without a fault: a kernel waits on a barrier that
nothing ever completes, its bounded wait gives up after the limit, the event is
recorded in the status word, and the context stays usable afterwards."""
import pytest

from long_context_attention_fwd_b200 import capi

torch = pytest.importorskip("torch")


@pytest.mark.gpu
def test_bounded_wait_reports_timeout_and_context_survives():
    st, _ = capi.attn_device_status(None)  # clear anything left over
    assert st in (capi.ATTN_OK, capi.ATTN_ERR_TIMEOUT)
    capi.check(capi.attn_selftest_wait_timeout(2_000_000, None), "selftest")  # 2 ms limit
    st, site = capi.attn_device_status(None)
    assert st == capi.ATTN_ERR_TIMEOUT
    assert site == 0x400
    st, _ = capi.attn_device_status(None)
    assert st == capi.ATTN_OK  # the record was cleared
    # the context is still healthy: a real launch works and reports no error
    from long_context_attention_fwd_b200 import ops
    q = torch.randn(1, 128, 2, 64, device="cuda").bfloat16()
    o, lse = ops.attn_fwd(q, q, q, causal=True)
    torch.cuda.synchronize()
    assert torch.isfinite(o.float()).all()
    st, _ = capi.attn_device_status(None)
    assert st == capi.ATTN_OK


@pytest.mark.gpu
def test_invalid_arguments_launch_nothing():
    q = torch.zeros(1, 128, 3, 64, device="cuda", dtype=torch.bfloat16)
    k = torch.zeros(1, 128, 2, 64, device="cuda", dtype=torch.bfloat16)
    lse = torch.zeros(1, 3, 128, device="cuda")
    st = capi.attn_fwd(q.data_ptr(), k.data_ptr(), k.data_ptr(), q.data_ptr(), lse.data_ptr(),
                       1, 3, 2, 128, 64, 1, 0.125, None, None)
    assert st == capi.ATTN_ERR_INVALID_ARG
    st = capi.attn_fwd(q.data_ptr() + 2, k.data_ptr(), k.data_ptr(), q.data_ptr(), lse.data_ptr(),
                       1, 2, 2, 128, 64, 1, 0.125, None, None)
    assert st == capi.ATTN_ERR_MISALIGNED


@pytest.mark.gpu
def test_calls_from_another_host_thread():
    """The library is usable from any host thread (autograd runs backward on its own)."""
    import threading
    from long_context_attention_fwd_b200 import ops
    q = torch.randn(1, 256, 2, 64, device="cuda").bfloat16()
    do = torch.randn_like(q)
    o, lse = ops.attn_fwd(q, q, q, causal=True)
    ref = ops.attn_bwd(q, q, q, o, lse, do, causal=True)
    torch.cuda.synchronize()
    box = {}

    def work():
        try:
            torch.cuda.set_device(q.device)
            box["r"] = ops.attn_bwd(q, q, q, o, lse, do, causal=True)
            torch.cuda.synchronize()
        except Exception as e:  # surfaced below with the library's error text
            box["e"] = e

    t = threading.Thread(target=work)
    t.start()
    t.join()
    assert "e" not in box, box.get("e")
    assert torch.equal(box["r"][1], ref[1]) and torch.equal(box["r"][2], ref[2])


@pytest.mark.gpu
def test_calls_leave_the_callers_current_device_alone():
    """Each entry point makes the tensors' device current for its own launches and gives
    the calling thread its current device back on return."""
    if torch.cuda.device_count() < 2:
        pytest.skip("needs two GPUs")
    from long_context_attention_fwd_b200 import ops
    torch.cuda.set_device(0)
    torch.zeros(1, device="cuda:0")  # device 0's context is active
    q = torch.randn(1, 256, 2, 64, device="cuda:1").bfloat16()
    o, lse = ops.attn_fwd(q, q, q, causal=True)
    assert torch.cuda.current_device() == 0
    dq, dk, dv = ops.attn_bwd(q, q, q, o, lse, torch.ones_like(q))
    assert torch.cuda.current_device() == 0
    torch.cuda.synchronize(1)
    with torch.cuda.device(1):
        o1, _ = ops.attn_fwd(q, q, q, causal=True)
    torch.cuda.synchronize(1)
    assert torch.equal(o, o1)


@pytest.mark.gpu
def test_wrapper_rejects_mismatched_tensors_before_launching():
    """Outputs supplied by the caller, and inputs whose size the kernel takes from q or k,
    must match exactly: a smaller one would be written or read past its end."""
    from long_context_attention_fwd_b200 import ops
    q = torch.randn(1, 256, 4, 64, device="cuda").bfloat16()
    k = torch.randn(1, 256, 2, 64, device="cuda").bfloat16()
    o, lse = ops.attn_fwd(q, k, k, causal=True)
    bad = [
        lambda: ops.attn_fwd(q, k, k, out=torch.empty(1, 255, 4, 64, device="cuda", dtype=torch.bfloat16)),
        lambda: ops.attn_fwd(q, k, k, lse=torch.empty(1, 4, 255, device="cuda")),
        lambda: ops.attn_fwd(q, k, k, lse=torch.empty(1, 4, 256, device="cuda", dtype=torch.float64)),
        lambda: ops.attn_fwd(q, k, k[:, :, :1].contiguous()),                    # v is not k's shape
        lambda: ops.attn_bwd(q, k, k, o, lse, q[:, :128].contiguous()),           # dout too short
        lambda: ops.attn_bwd(q, k, k, o[:, :128].contiguous(), lse, q),           # o too short
        lambda: ops.attn_bwd(q, k, k, o, lse[:, :2].contiguous(), q),             # lse too small
        lambda: ops.attn_bwd(q, k, k, o, lse, q, dk=torch.empty_like(q)),         # dk is q's shape
        lambda: ops.attn_bwd(q, k, k, o, lse, q, workspace=torch.empty(16, device="cpu")),
        lambda: ops.attn_merge([o, o], [lse, lse], lse=torch.empty(1, 4, 100, device="cuda")),
        lambda: ops.convert_f32_bf16(torch.zeros(10, device="cuda"),
                                     out=torch.empty(9, device="cuda", dtype=torch.bfloat16)),
    ]
    for i, call in enumerate(bad):
        with pytest.raises(ValueError):
            call()
    # a workspace of another dtype is measured in bytes, not elements
    need = ops.attn_bwd_workspace_size(q)
    ws = torch.empty((need + 3) // 4, dtype=torch.float32, device="cuda")
    dq, dk, dv = ops.attn_bwd(q, k, k, o, lse, q, workspace=ws)
    dq2, dk2, dv2 = ops.attn_bwd(q, k, k, o, lse, q)
    torch.cuda.synchronize()
    assert torch.equal(dk, dk2) and torch.equal(dv, dv2)
