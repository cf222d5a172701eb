"""The failure path of the library's kernels, exercised without a fault: every
wait on an internal barrier is bounded, and when one runs out the kernel
records it in a device error word and returns.  A probe kernel makes such a
wait run out on purpose (a barrier that nothing arrives on); sage_check must
report SAGE_ERR_TIMEOUT with the site bit, clear the word, and leave the
context usable."""
import pytest
import torch

import quantized_attention_qk_b200 as sage
from quantized_attention_qk_b200.inputs import WORKLOADS, make_qkv

pytestmark = [pytest.mark.gpu, pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


def test_a_bounded_wait_that_runs_out_is_reported_and_the_context_survives():
    w = WORKLOADS["tiny"]
    q, k, v, _ = make_qkv(w, device="cuda")
    before = sage.sage_attn_fwd(q, k, v, sm_scale=w.sm_scale)
    torch.cuda.synchronize()
    sage.sage_check()                       # clean to start with
    sage.sage_debug_wait_timeout(20000)     # gives up after ~20 ms of SM clocks
    torch.cuda.synchronize()
    with pytest.raises(sage.SageError) as e:
        sage.sage_check()
    assert e.value.status == 5              # SAGE_ERR_TIMEOUT
    assert "0x101" in str(e.value)          # bit 0 and bit 8 + site 0
    sage.sage_check()                       # the word was cleared
    after = sage.sage_attn_fwd(q, k, v, sm_scale=w.sm_scale)
    torch.cuda.synchronize()
    sage.sage_check()
    assert torch.equal(after, before)
