"""The serving session (mla_session_* in include/mla.h): several pipelined steps with host
inputs and outputs give, step by step, the bit-identical results of the direct device calls on
the same inputs (same kernels, same scheduler parts).  Each step has its own query, lengths and
(token-sparse) index lists, so a step that read another step's staging buffers would differ."""
import numpy as np
import pytest
import torch

import mla_inputs as mi
from tests._helpers import to_device

pytestmark = pytest.mark.gpu

KINDS = [
    # (name, batch, s_q, h_q, seqlens, kv_format, topk, causal)
    ("bf16_r16", 3, 1, 16, [300, 1000, 64], "bf16", 0, False),
    ("bf16_pair_causal", 2, 2, 96, [700, 130], "bf16", 0, True),
    ("fp8_r128", 2, 1, 128, [500, 1200], "fp8", 0, False),
    ("sparse_r16", 3, 1, 16, [400, 900, 70], "bf16", 128, False),
    ("sparse_pair", 2, 1, 128, [1000, 2500], "bf16", 300, False),
]
STEPS = 5


@pytest.mark.parametrize("name,batch,s_q,h_q,seqlens,kv_format,topk,causal", KINDS, ids=[k[0] for k in KINDS])
def test_session_matches_direct_calls(name, batch, s_q, h_q, seqlens, kv_format, topk, causal):
    import attention_mla_get_b200 as mla
    case = mi.make_case(batch, s_q, h_q, seqlens, causal=causal, kv_format=kv_format, seed=11, spare_blocks=2)
    _, kv, bt, _ = to_device(case)
    max_blocks = case.block_table.shape[1]
    sess = mla.MLASession(batch, s_q, h_q, max_blocks, topk=topk,
                          kv_dtype=mla.KV_FP8 if kv_format == "fp8" else mla.KV_BF16)
    g = torch.Generator().manual_seed(5)
    base = np.asarray(seqlens, dtype=np.int32)
    steps = []
    for k in range(STEPS):
        q_h = torch.randn((batch, s_q, h_q, mi.D_QK), generator=g).to(torch.bfloat16).pin_memory()
        sl_h = torch.from_numpy(np.maximum(base - 37 * k, 1).astype(np.int32)).pin_memory()
        idx_h = None
        if topk:
            idx_h = torch.from_numpy(np.ascontiguousarray(
                mi.make_sparse_indices(sl_h.numpy(), s_q, topk, seed=k, invalid_frac=0.1))).pin_memory()
        out_h = torch.empty((batch, s_q, h_q, 512), dtype=torch.bfloat16).pin_memory()
        lse_h = torch.empty((batch, h_q, s_q), dtype=torch.float32).pin_memory()
        steps.append((q_h, sl_h, idx_h, out_h, lse_h))
    bt_h = torch.from_numpy(case.block_table).pin_memory()
    for q_h, sl_h, idx_h, out_h, lse_h in steps:
        sess.decode(q_h, kv, bt_h, sl_h, out_h, lse_h, indices_host=idx_h, softmax_scale=case.softmax_scale,
                    causal=causal)
    sess.join()
    torch.cuda.synchronize()
    assert sess.status() == 0
    for k, (q_h, sl_h, idx_h, out_h, lse_h) in enumerate(steps):
        q, sl = q_h.cuda(), sl_h.cuda()
        if topk:
            md, ns = mla.mla_get_metadata_sparse(batch, s_q, topk, h_q, 1, num_sm_parts=sess.num_sm_parts)
            out, lse = mla.mla_decode_kvcache_sparse(q, kv, bt, sl, idx_h.cuda(), 512, md, ns,
                                                     softmax_scale=case.softmax_scale)
        else:
            md, ns = mla.mla_get_metadata(sl, s_q * h_q, 1, num_sm_parts=sess.num_sm_parts)
            out, lse = mla.mla_decode_kvcache(q, kv, bt, sl, 512, md, ns, softmax_scale=case.softmax_scale,
                                              causal=causal)
        torch.cuda.synchronize()
        assert torch.equal(out.cpu().view(torch.int16), out_h.view(torch.int16)), f"step {k}: out"
        assert torch.equal(lse.cpu(), lse_h), f"step {k}: lse"
    sess.close()


def test_session_rejects_device_host_buffers():
    import attention_mla_get_b200 as mla
    case = mi.make_case(2, 1, 16, [100, 200], seed=3)
    q, kv, bt, sl = to_device(case)
    sess = mla.MLASession(2, 1, 16, case.block_table.shape[1])
    out_h = torch.empty((2, 1, 16, 512), dtype=torch.bfloat16)
    lse_h = torch.empty((2, 16, 1), dtype=torch.float32)
    with pytest.raises(ValueError):
        sess.decode(q, kv, bt.cpu(), sl.cpu(), out_h, lse_h)  # q on the device
    with pytest.raises(ValueError):
        sess.decode(q.cpu(), kv.cpu(), bt.cpu(), sl.cpu(), out_h, lse_h)  # the cache on the host
    sess.close()
