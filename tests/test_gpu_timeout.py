"""The bounded-wait failure path of the single-CTA decode kernel (up to 64 query rows per
request over a bf16 cache), exercised without faulting or hanging the GPU: mla_fault_injection_arm makes the next call's copy producer skip one slot fill and
shortens every pipeline wait to a few milliseconds.  The slot's consumer then waits in vain,
the bound runs out, the kernel sets MLA_STATUS_WAIT_TIMEOUT in the workspace status word, every
role of the CTA unwinds (copies in flight drained, tensor memory freed) and the call returns.
A normal call that follows on the same stream must be correct and report no error."""
import numpy as np
import pytest
import torch

import mla_inputs as mi
import oracle
from tests._helpers import compare, to_device

pytestmark = pytest.mark.gpu

WAIT_LIMIT = 1 << 22   # SM clock cycles: about 2 ms at B200 clocks


@pytest.mark.parametrize("withhold", [0, 3, 12, 40])
def test_withheld_fill_times_out_and_next_call_is_correct(cuda_ok, withhold):
    import attention_mla_get_b200 as mla
    # one part: the whole batch runs on one CTA, so fill indices up to 9 per 128-token step exist
    case = mi.make_case(2, 1, 64, [1000, 300], seed=61)
    q, kv, bt, sl = to_device(case)
    md, ns = mla.mla_get_metadata(sl, case.rows, 1, num_sm_parts=1)
    ws = torch.zeros(mla.mla_workspace_size(case.batch, 1, case.rows, 1), dtype=torch.uint8, device="cuda")
    mla.mla_fault_injection_arm(WAIT_LIMIT, withhold)
    mla.mla_decode_kvcache(q, kv, bt, sl, 512, md, ns, softmax_scale=case.softmax_scale, workspace=ws)
    torch.cuda.synchronize()  # the call returned: no hang, no fault
    assert mla.mla_read_status(ws, reset=True) & 1
    assert mla.mla_read_status(ws) == 0

    o_ref, l_ref = oracle.mla_decode_reference(case)
    for parts in (1, None):
        md2, ns2 = mla.mla_get_metadata(sl, case.rows, 1, num_sm_parts=parts)
        ws2 = ws if parts == 1 else torch.zeros(mla.mla_workspace_size(case.batch, md2.shape[0], case.rows, 1),
                                                dtype=torch.uint8, device="cuda")
        out, lse = mla.mla_decode_kvcache(q, kv, bt, sl, 512, md2, ns2, softmax_scale=case.softmax_scale,
                                          workspace=ws2)
        torch.cuda.synchronize()
        assert mla.mla_read_status(ws2) == 0
        compare(case, out.float().cpu().numpy(), lse.cpu().numpy(), o_ref, l_ref)


def test_arm_is_taken_by_one_call_only(cuda_ok):
    """An armed setting applies to exactly one call: the call after it runs with the normal bound."""
    import attention_mla_get_b200 as mla
    case = mi.make_case(1, 1, 64, [700], seed=62)
    q, kv, bt, sl = to_device(case)
    md, ns = mla.mla_get_metadata(sl, case.rows, 1, num_sm_parts=1)
    ws = torch.zeros(mla.mla_workspace_size(case.batch, 1, case.rows, 1), dtype=torch.uint8, device="cuda")
    mla.mla_fault_injection_arm(WAIT_LIMIT, 5)
    mla.mla_decode_kvcache(q, kv, bt, sl, 512, md, ns, softmax_scale=case.softmax_scale, workspace=ws)
    torch.cuda.synchronize()
    assert mla.mla_read_status(ws, reset=True) & 1
    out, lse = mla.mla_decode_kvcache(q, kv, bt, sl, 512, md, ns, softmax_scale=case.softmax_scale, workspace=ws)
    torch.cuda.synchronize()
    assert mla.mla_read_status(ws) == 0
    o_ref, l_ref = oracle.mla_decode_reference(case)
    compare(case, out.float().cpu().numpy(), lse.cpu().numpy(), o_ref, l_ref)


@pytest.mark.parametrize("withhold", [0, 5, 17])
def test_16_row_tile_withheld_fill_times_out(cuda_ok, withhold):
    """The same with the 16-row tile (the memory-bound shape): a skipped fill times out, the
    status bit is set, and the next call on the same workspace is correct."""
    import attention_mla_get_b200 as mla
    case = mi.make_case(2, 1, 16, [1000, 300], seed=63)   # one part: 11 steps, 99 slot fills
    q, kv, bt, sl = to_device(case)
    md, ns = mla.mla_get_metadata(sl, case.rows, 1, num_sm_parts=1)
    ws = torch.zeros(mla.mla_workspace_size(case.batch, 1, case.rows, 1), dtype=torch.uint8, device="cuda")
    mla.mla_fault_injection_arm(WAIT_LIMIT, withhold)
    mla.mla_decode_kvcache(q, kv, bt, sl, 512, md, ns, softmax_scale=case.softmax_scale, workspace=ws)
    torch.cuda.synchronize()
    assert mla.mla_read_status(ws, reset=True) & 1
    out, lse = mla.mla_decode_kvcache(q, kv, bt, sl, 512, md, ns, softmax_scale=case.softmax_scale, workspace=ws)
    torch.cuda.synchronize()
    assert mla.mla_read_status(ws) == 0
    o_ref, l_ref = oracle.mla_decode_reference(case)
    compare(case, out.float().cpu().numpy(), lse.cpu().numpy(), o_ref, l_ref)
