"""The kernel trace brackets each library launch with its own event pair and
names the kernel, so per-kernel times can be read on the launching stream."""
import pytest
import torch

pytestmark = pytest.mark.gpu


def test_trace_names_and_times():
    import structured_sparse_attention_block_b200 as m
    from structured_sparse_attention_block_b200.inputs import training_inputs
    q, k, v, dout = training_inputs(B=1, Lq=512, Lk=512, Hq=4, Hkv=2, d=64, seed=3, device="cuda")
    quad = m.cowa_default_quad(512, 2, 16, 64)
    o, lse = m.cowa_fwd(q, k, v, quad)  # warm (module set-up outside the trace)
    torch.cuda.synchronize()
    n0 = m.cowa_launch_count()
    m.cowa_trace_start(16)
    o, lse = m.cowa_fwd(q, k, v, quad)
    m.cowa_bwd(q, k, v, o, lse, dout, quad)
    m.cowa_trace_stop()
    torch.cuda.synchronize()
    entries, dropped = m.cowa_trace_entries()
    names = [n for n, _ in entries]
    assert dropped == 0
    assert len(entries) == m.cowa_launch_count() - n0
    assert "fwd_sm100" in names and "dkdv_sm100" in names and "dq_sm100" in names
    assert "bwd_prep" in names and "schedule" not in names  # the tcgen05 kernels form their own tile ranges
    assert all(t > 0 for _, t in entries)
    # capacity 1: the rest of the backward's launches are counted as dropped
    m.cowa_trace_start(1)
    m.cowa_bwd(q, k, v, o, lse, dout, quad)
    m.cowa_trace_stop()
    entries, dropped = m.cowa_trace_entries()
    assert len(entries) == 1 and dropped == 2
    # a filter records only the named kernel
    m.cowa_trace_start(8, only="dkdv_sm100")
    m.cowa_bwd(q, k, v, o, lse, dout, quad)
    m.cowa_trace_stop()
    entries, dropped = m.cowa_trace_entries()
    assert [n for n, _ in entries] == ["dkdv_sm100"] and dropped == 0
    m.cowa_trace_start(0)
    assert m.cowa_trace_entries() == ([], 0)
