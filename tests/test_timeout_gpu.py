"""The timeout path of the kernels' bounded waits, without a GPU fault: the
self-test kernel waits on a barrier that nothing completes, its wait runs out
after the 2 s limit and records COWA_ERR_TIMEOUT, the host reads it through
cowa_get_device_error, and the context keeps working afterwards."""
import time

import pytest
import torch

import structured_sparse_attention_block_b200 as cowa
from structured_sparse_attention_block_b200.inputs import training_inputs

pytestmark = pytest.mark.gpu


def test_bounded_wait_runs_out_and_reports_timeout():
    cowa.cowa_get_device_error()  # nothing pending
    t0 = time.monotonic()
    cowa.cowa_selftest_wait_timeout()
    with pytest.raises(cowa.CowaError) as err:
        cowa.cowa_get_device_error()
    elapsed = time.monotonic() - t0
    assert err.value.status == 6  # COWA_ERR_TIMEOUT
    assert 1.5 < elapsed < 60.0
    cowa.cowa_get_device_error()  # read and cleared
    # the context is usable: a forward runs and reports no error
    q, k, v, _ = training_inputs(1, 256, 256, 4, 2, 64, device="cuda", seed=3, with_dout=False)
    o, lse = cowa.cowa_fwd(q, k, v, (4, 32, 0, 112))
    cowa.cowa_get_device_error()
    assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()
