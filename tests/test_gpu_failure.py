"""Device-side failure detection, exercised without a GPU fault: a bounded wait on
a barrier that nothing completes must give up after its limit, record a timeout
in the device error word and return, and the context must stay usable."""
import time

import numpy as np
import pytest
import torch

from oracle import sparse_attn_oracle as orc
from tests.helpers import assert_output_close, to_np

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import free_block_sparse_mean_b200 as sa
    from free_block_sparse_mean_b200 import workloads as wl


def test_bounded_wait_times_out_and_context_survives():
    dev = torch.device("cuda:0")
    torch.cuda.synchronize()
    assert sa.sparse_attn_device_error() == 0          # clean start
    t0 = time.perf_counter()
    sa.sparse_attn_selftest_wait_timeout(200_000)      # 0.2 s limit
    torch.cuda.synchronize()
    waited = time.perf_counter() - t0
    code = sa.sparse_attn_device_error()
    assert code & 1, f"no timeout recorded (error word {code})"
    assert 0.15 < waited < 5.0, f"the wait took {waited:.3f} s"
    assert sa.sparse_attn_device_error() == 0          # reading cleared it

    # the context still works: a plan and forward on the tiny workload match the oracle
    w = wl.WORKLOADS["tiny"]
    q, k, v = wl.generate(w, seed=0, device=dev)
    plan = sa.sparse_attn_plan(q, k, 0.95)
    o = sa.sparse_attn_fwd(q, k, v, plan, -12.0)
    torch.cuda.synchronize()
    assert sa.sparse_attn_device_error() == 0
    mask = to_np(plan.mask)
    ref = orc.fwd(q.cpu(), k.cpu(), v.cpu(), mask, -12.0)
    assert_output_close(to_np(o), ref, "tiny workload after the timeout diagnostic")


def test_public_host_call_raises_on_a_device_error():
    """sparse_attention reads the device error word after its work: a fired check
    (here the timeout diagnostic's, left in the word before the call) raises
    SparseAttnError with SA_ERR_DEVICE_CHECK instead of returning a silent
    result; the word is cleared by that read, and the next call succeeds."""
    dev = torch.device("cuda:0")
    w = wl.WORKLOADS["tiny"]
    q, k, v = wl.generate(w, seed=0, device=dev)
    qh, kh, vh = (x.cpu().pin_memory() for x in (q, k, v))
    torch.cuda.synchronize()
    assert sa.sparse_attn_device_error() == 0
    sa.sparse_attn_selftest_wait_timeout(50_000)       # records a timeout, returns normally
    with pytest.raises(sa.SparseAttnError) as ei:
        sa.sparse_attention(qh, kh, vh, 0.95, -12.0)
    assert ei.value.status == 5                        # SA_ERR_DEVICE_CHECK
    o = sa.sparse_attention(qh, kh, vh, 0.95, -12.0)
    ref = sa.sparse_attn_fwd(q, k, v, sa.sparse_attn_plan(q, k, 0.95), -12.0)
    torch.cuda.synchronize()
    assert torch.equal(o, ref.cpu())
