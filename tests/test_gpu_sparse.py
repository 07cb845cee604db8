"""GPU parity of token-sparse decode (mla_decode_kvcache_sparse, through the C-ABI) against
the fp64 oracle (mla_sparse_decode_reference).  bf16 cache tolerances:
|dO| <= 5e-3 + 1e-2 |O_ref| element-wise, |dLSE| <= 1e-3.  The metadata for batch * s_q
query positions of topk tokens must be bit-exact to the oracle's scheduler rule."""
import zlib

import numpy as np
import pytest
import torch

import mla_inputs as mi
import oracle
from tests._helpers import compare, run_gpu, run_gpu_sparse, to_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu(cuda_ok):
    import attention_mla_get_b200  # noqa: F401  (fails loudly if libmla.so is missing)
    yield


CASES = [
    # (name, batch, s_q, h_q, seqlens, topk, invalid_frac, duplicate_frac)
    ("sp_r16", 3, 1, 16, [300, 1000, 64], 128, 0.0, 0.0),
    ("sp_r16_gaps_dups", 3, 1, 16, [300, 1000, 5], 200, 0.2, 0.1),
    ("sp_sq2_r16", 2, 2, 16, [500, 2000], 256, 0.1, 0.0),
    ("sp_r32_ragged_topk", 2, 1, 32, [129, 3000], 333, 0.0, 0.0),
    ("sp_r64", 2, 1, 64, [700, 1500], 300, 0.0, 0.05),
    ("sp_r128_two_groups", 2, 1, 128, [1000, 4000], 512, 0.05, 0.05),
    # CTA pairs with a part-filled row group: rows past h_q are clipped by the output map
    ("sp_r96_pair_pad_rows", 3, 1, 96, [700, 2000, 90], 384, 0.1, 0.0),
    ("sp_r192_two_pairs", 2, 1, 192, [600, 1500], 300, 0.05, 0.05),
    ("sp_sq2_r48_pad_rows", 2, 2, 48, [400, 90], 160, 0.1, 0.0),
    ("sp_topk_over_L", 2, 1, 16, [40, 70], 256, 0.0, 0.0),
]


@pytest.mark.parametrize("name,batch,s_q,h_q,seqlens,topk,inv,dup", CASES, ids=[c[0] for c in CASES])
@pytest.mark.parametrize("parts", [None, 1, 7])
def test_sparse_parity(name, batch, s_q, h_q, seqlens, topk, inv, dup, parts):
    seed = zlib.crc32(name.encode()) % 1000
    case = mi.make_case(batch, s_q, h_q, seqlens, seed=seed, spare_blocks=2)
    idx = mi.make_sparse_indices(case.cache_seqlens, s_q, topk, seed, invalid_frac=inv, duplicate_frac=dup)
    O_ref, L_ref = oracle.mla_sparse_decode_reference(case, idx)
    out, lse, status, (md, ns) = run_gpu_sparse(case, idx, num_sm_parts=parts)
    assert status == 0
    compare(case, out, lse, O_ref, L_ref)
    md_ref, ns_ref = oracle.schedule(np.full(batch * s_q, topk, dtype=np.int32), md.shape[0])
    assert np.array_equal(md.cpu().numpy(), md_ref) and np.array_equal(ns.cpu().numpy(), ns_ref)


def test_sparse_empty_list_gives_zero_and_neg_inf():
    case = mi.make_case(2, 2, 16, [300, 500], seed=41)
    idx = mi.make_sparse_indices(case.cache_seqlens, 2, 64, 41)
    idx[0, 1, :] = -1                       # query (0, 1) lists nothing
    idx[1, 0, :] = 500 + np.arange(64)      # every entry past L_1
    O_ref, L_ref = oracle.mla_sparse_decode_reference(case, idx)
    out, lse, status, _ = run_gpu_sparse(case, idx)
    assert status == 0
    assert np.all(out[0, 1] == 0) and np.all(np.isneginf(lse[0, :, 1]))
    assert np.all(out[1, 0] == 0) and np.all(np.isneginf(lse[1, :, 0]))
    compare(case, out, lse, O_ref, L_ref)


def test_sparse_listing_every_position_matches_dense():
    case = mi.make_case(2, 1, 16, [700, 1300], seed=42)
    rng = np.random.default_rng(5)
    idx = np.full((2, 1, 1300), -1, dtype=np.int32)
    for b, L in enumerate([700, 1300]):
        idx[b, 0, :L] = rng.permutation(L)
    o_s, l_s, st_s, _ = run_gpu_sparse(case, idx)
    o_d, l_d, st_d, _ = run_gpu(case)
    assert st_s == 0 and st_d == 0
    O_ref, L_ref = oracle.mla_decode_reference(case)
    compare(case, o_s, l_s, O_ref, L_ref)
    compare(case, o_d, l_d, O_ref, L_ref)


def test_sparse_nan_in_unread_slots_does_not_leak():
    clean = mi.make_case(2, 1, 16, [70, 129], seed=43, poison=False, spare_blocks=3)
    dirty = mi.make_case(2, 1, 16, [70, 129], seed=43, poison=True, spare_blocks=3)
    idx = mi.make_sparse_indices(clean.cache_seqlens, 1, 96, 43, invalid_frac=0.3)
    o1, l1, _, _ = run_gpu_sparse(clean, idx)
    o2, l2, _, _ = run_gpu_sparse(dirty, idx)
    assert np.isfinite(o2).all()
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def test_sparse_index_order_only_rounds():
    case = mi.make_case(2, 1, 64, [900, 2000], seed=44)
    idx = mi.make_sparse_indices(case.cache_seqlens, 1, 400, 44)
    perm = idx[..., np.random.default_rng(1).permutation(400)]
    o1, l1, _, _ = run_gpu_sparse(case, idx)
    o2, l2, _, _ = run_gpu_sparse(case, perm)
    O_ref, L_ref = oracle.mla_sparse_decode_reference(case, idx)
    compare(case, o1, l1, O_ref, L_ref)
    compare(case, o2, l2, O_ref, L_ref)


@pytest.mark.slow
def test_full_sparse_workload_sampled():
    case = mi.make_workload("sparse_b128_h128_L8192_topk2048")
    out, lse, status, (md, ns) = run_gpu_sparse(case, case.indices)
    assert status == 0
    assert np.isfinite(out).all()
    sample = [0, 57, case.batch - 1]
    O_ref, L_ref = oracle.mla_sparse_decode_reference(case, case.indices, requests=sample)
    compare(case, out, lse, O_ref, L_ref, requests=sample)


# ---------------------------------------------------------------- sparse prefill
PREFILL_CASES = [
    # (name, s_q, h_q, s_kv, topk, invalid_frac)
    ("pf_r16", 37, 16, 1000, 128, 0.1),
    ("pf_r64_ragged_kv", 64, 64, 777, 256, 0.0),
    ("pf_r128", 16, 128, 4096, 512, 0.05),
    ("pf_r96_pair_pad_rows", 24, 96, 1500, 300, 0.1),
    ("pf_r32_many_tokens", 200, 32, 300, 64, 0.2),
]


def run_prefill(case, num_sm_parts=None):
    import attention_mla_get_b200 as mla
    s_kv = int(case.cache_seqlens[0])
    q = torch.from_numpy(case.q_bits[0].view(np.int16)).view(torch.bfloat16).cuda()
    kv = torch.from_numpy(np.ascontiguousarray(case.kv.reshape(-1, mi.D_QK)[:s_kv]).view(np.int16)).view(
        torch.bfloat16).reshape(s_kv, 1, mi.D_QK).cuda()
    idx = torch.from_numpy(np.ascontiguousarray(case.indices[0])).cuda()
    md, ns = mla.mla_get_metadata_sparse(1, case.s_q, idx.shape[-1], case.h_q, 1, num_sm_parts=num_sm_parts)
    ws = torch.zeros(mla.mla_workspace_size(case.s_q, md.shape[0], case.h_q, 1), dtype=torch.uint8, device="cuda")
    out, lse = mla.mla_sparse_prefill(q, kv, idx, case.softmax_scale, tile_md=md, num_splits=ns, workspace=ws)
    torch.cuda.synchronize()
    return out.float().cpu().numpy(), lse.cpu().numpy(), mla.mla_read_status(ws)


@pytest.mark.parametrize("name,s_q,h_q,s_kv,topk,inv", PREFILL_CASES, ids=[c[0] for c in PREFILL_CASES])
@pytest.mark.parametrize("parts", [None, 5])
def test_sparse_prefill_parity(name, s_q, h_q, s_kv, topk, inv, parts):
    case = mi.make_prefill_case(s_q, h_q, s_kv, topk, seed=zlib.crc32(name.encode()) % 1000, invalid_frac=inv)
    s_kv_rows = case.kv.reshape(-1, mi.D_QK)[:s_kv]
    O_ref, L_ref = oracle.mla_sparse_prefill_reference(case.q_bits[0], s_kv_rows, case.indices[0],
                                                       case.softmax_scale)
    out, lse, status = run_prefill(case, num_sm_parts=parts)
    assert status == 0
    compare(case, out[None], lse[None], O_ref[None], L_ref[None])


def test_flash_mla_sparse_fwd_spelling():
    import attention_mla_get_b200 as mla
    case = mi.make_prefill_case(8, 16, 500, 64, seed=77)
    q = torch.from_numpy(case.q_bits[0].view(np.int16)).view(torch.bfloat16).cuda()
    kv = torch.from_numpy(np.ascontiguousarray(case.kv.reshape(-1, mi.D_QK)[:500]).view(np.int16)).view(
        torch.bfloat16).reshape(500, 1, mi.D_QK).cuda()
    idx = torch.from_numpy(np.ascontiguousarray(case.indices[0])).reshape(8, 1, 64).cuda()
    out, lse = mla.flash_mla_sparse_fwd(q, kv, idx, case.softmax_scale, d_v=512)
    torch.cuda.synchronize()
    O_ref, L_ref = oracle.mla_sparse_prefill_reference(case.q_bits[0], case.kv.reshape(-1, mi.D_QK)[:500],
                                                       case.indices[0], case.softmax_scale)
    compare(case, out.float().cpu().numpy()[None], lse.cpu().numpy()[None], O_ref[None], L_ref[None])
