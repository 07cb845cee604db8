"""Helpers shared by the GPU tests: move a seeded case to the device, run the library,
and compare with the oracle under the stated tolerances."""
from __future__ import annotations

import numpy as np
import torch

import mla_inputs as mi

# tolerances for the bf16 cache: |dO| <= 5e-3 + 1e-2 |O_ref|, |dLSE| <= 1e-3
BF16_O_ABS, BF16_O_REL, BF16_LSE = 5e-3, 1e-2, 1e-3
# FP8 cache: |dO| <= 2e-2 + 2e-2 |O_ref|; LSE keeps its own bound below
FP8_O_ABS, FP8_O_REL, FP8_LSE = 2e-2, 2e-2, 2e-2


def to_device(case: mi.DecodeCase, device="cuda"):
    q = torch.from_numpy(case.q_bits.view(np.int16)).view(torch.bfloat16).to(device)
    if case.kv_format == "bf16":
        kv = torch.from_numpy(case.kv.view(np.int16)).view(torch.bfloat16).reshape(
            case.num_blocks, mi.PAGE, 1, mi.D_QK).to(device)
    else:
        kv = torch.from_numpy(case.kv).to(device)
    bt = torch.from_numpy(case.block_table).to(device)
    sl = torch.from_numpy(case.cache_seqlens).to(device)
    return q, kv, bt, sl


def run_gpu(case: mi.DecodeCase, num_sm_parts=None, tensors=None):
    import attention_mla_get_b200 as mla
    q, kv, bt, sl = tensors if tensors is not None else to_device(case)
    md, ns = mla.mla_get_metadata(sl, case.rows, 1, num_sm_parts=num_sm_parts)
    ws = torch.zeros(mla.mla_workspace_size(case.batch, md.shape[0], case.rows, 1), dtype=torch.uint8,
                     device=q.device)
    out, lse = mla.mla_decode_kvcache(q, kv, bt, sl, 512, md, ns, softmax_scale=case.softmax_scale,
                                      causal=case.causal, workspace=ws)
    torch.cuda.synchronize()
    status = mla.mla_read_status(ws)
    return out.float().cpu().numpy(), lse.cpu().numpy(), status, (md, ns)


def compare(case, out, lse, O_ref, L_ref, requests=None, fp8=None):
    """Element-wise check; returns a dict of worst errors (raises AssertionError on failure)."""
    fp8 = case.kv_format == "fp8" if fp8 is None else fp8
    o_abs, o_rel, l_tol = (FP8_O_ABS, FP8_O_REL, FP8_LSE) if fp8 else (BF16_O_ABS, BF16_O_REL, BF16_LSE)
    reqs = list(range(case.batch)) if requests is None else list(requests)
    o, r = out[reqs].astype(np.float64), O_ref[reqs]
    l, lr = lse[reqs].astype(np.float64), L_ref[reqs]
    assert np.isfinite(o).all(), "non-finite output"
    bound = o_abs + o_rel * np.abs(r)
    excess = np.abs(o - r) - bound
    worst_o = float(np.max(np.abs(o - r)))
    assert excess.max() <= 0, f"O out of tolerance: max |dO| = {worst_o:.3e}, worst excess {excess.max():.3e}"
    inf_ref = np.isneginf(lr)
    assert np.array_equal(np.isneginf(l), inf_ref), "LSE -inf pattern differs"
    dl = np.abs(l[~inf_ref] - lr[~inf_ref])
    worst_l = float(dl.max()) if dl.size else 0.0
    assert worst_l <= l_tol, f"LSE out of tolerance: max |dLSE| = {worst_l:.3e}"
    return {"max_dO": worst_o, "max_dLSE": worst_l}


def run_gpu_sparse(case: mi.DecodeCase, indices, num_sm_parts=None, tensors=None):
    """Token-sparse decode of `case` over `indices` (int32 [b, s_q, topk]) through the library."""
    import attention_mla_get_b200 as mla
    q, kv, bt, sl = tensors if tensors is not None else to_device(case)
    idx = torch.from_numpy(np.ascontiguousarray(indices, dtype=np.int32)).to(q.device)
    topk = idx.shape[-1]
    md, ns = mla.mla_get_metadata_sparse(case.batch, case.s_q, topk, case.h_q, 1, num_sm_parts=num_sm_parts,
                                         device=q.device)
    ws = torch.zeros(mla.mla_workspace_size(case.batch * case.s_q, md.shape[0], case.h_q, 1), dtype=torch.uint8,
                     device=q.device)
    out, lse = mla.mla_decode_kvcache_sparse(q, kv, bt, sl, idx, 512, md, ns, softmax_scale=case.softmax_scale,
                                             workspace=ws)
    torch.cuda.synchronize()
    status = mla.mla_read_status(ws)
    return out.float().cpu().numpy(), lse.cpu().numpy(), status, (md, ns)
