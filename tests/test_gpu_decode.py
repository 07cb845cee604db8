"""GPU parity of the CUDA path (through the C-ABI) against the fp64 oracle.

Tolerances: bf16 cache |dO| <= 5e-3 + 1e-2 |O_ref| element-wise, |dLSE| <= 1e-3;
FP8 cache |dO| <= 2e-2 + 2e-2 |O_ref|.  The scheduler metadata must be bit-exact to the
oracle's scheduler rule.  Sizes span several 128-token steps and ragged page tails; the
full-size workloads are checked on sampled requests that the oracle computes one by one.
"""
import zlib

import numpy as np
import pytest
import torch

import mla_inputs as mi
import oracle
from tests._helpers import compare, run_gpu, to_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu(cuda_ok):
    import attention_mla_get_b200  # noqa: F401  (fails loudly if libmla.so is missing)
    yield


# ----------------------------------------------------------------------------- scheduler
@pytest.mark.parametrize("seed", range(7))
def test_scheduler_bit_exact(seed):
    import attention_mla_get_b200 as mla
    rng = np.random.default_rng(100 + seed)
    B = int(rng.integers(1, 300)) if seed < 6 else 2500  # the last: several 1024-request tiles
    sl = rng.integers(0, 20000, size=B).astype(np.int32)
    sl[rng.random(B) < 0.1] = 0
    for parts in (1, 7, 37, 74, 148, 400):
        md, ns = mla.mla_get_metadata(torch.from_numpy(sl).cuda(), 16, 1, num_sm_parts=parts)
        md_ref, ns_ref = oracle.schedule(sl, parts)
        assert np.array_equal(md.cpu().numpy(), md_ref), parts
        assert np.array_equal(ns.cpu().numpy(), ns_ref), parts


def test_scheduler_bit_exact_large_batch():
    """More than 8192 requests: the scheduler keeps its prefix array in global memory instead of
    shared memory and overwrites num_splits between its passes."""
    import attention_mla_get_b200 as mla
    rng = np.random.default_rng(7)
    B = 9000
    sl = rng.integers(0, 3000, size=B).astype(np.int32)
    sl[rng.random(B) < 0.05] = 0
    for parts in (1, 148, 1000):
        md, ns = mla.mla_get_metadata(torch.from_numpy(sl).cuda(), 16, 1, num_sm_parts=parts)
        md_ref, ns_ref = oracle.schedule(sl, parts)
        assert np.array_equal(md.cpu().numpy(), md_ref), parts
        assert np.array_equal(ns.cpu().numpy(), ns_ref), parts


def test_scheduler_cost_overflow_is_flagged():
    """A batch whose total cost (sum of ceil(L/128) + 2) reaches 2^31 does not fit the scheduler's
    32-bit prefix sums: the metadata comes back empty and flagged, and a decode call given it
    raises MLA_STATUS_BAD_METADATA and writes O = 0, LSE = -inf instead of reading the cache."""
    import attention_mla_get_b200 as mla
    B = 160
    sl = np.full(B, 2**31 - 1, dtype=np.int32)      # 2^24 blocks each: total cost about 2.7e9
    sl_d = torch.from_numpy(sl).cuda()
    md, ns = mla.mla_get_metadata(sl_d, 16, 1, num_sm_parts=148)
    md, ns = md.cpu().numpy(), ns.cpu().numpy()
    assert (md[:, 5] == 1).all() and (md[:, 0] == B).all() and (md[:, 2] == B).all()
    assert (ns == 0).all()
    # a decode call with that metadata: a one-page cache that no part ever reads
    q = torch.randn(B, 1, 16, 576, device="cuda").to(torch.bfloat16)
    kv = torch.zeros(1, 64, 1, 576, dtype=torch.bfloat16, device="cuda")
    bt = torch.zeros(B, 1, dtype=torch.int32, device="cuda")
    md_d, ns_d = torch.from_numpy(md).cuda(), torch.from_numpy(ns).cuda()
    ws = torch.zeros(mla.mla_workspace_size(B, 148, 16, 1), dtype=torch.uint8, device="cuda")
    out, lse = mla.mla_decode_kvcache(q, kv, bt, sl_d, 512, md_d, ns_d, workspace=ws)
    torch.cuda.synchronize()
    assert mla.mla_read_status(ws) == 2
    assert (out.float() == 0).all() and torch.isneginf(lse).all()


def test_num_sm_parts_matches_rule():
    import attention_mla_get_b200 as mla
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    for rows in (1, 16, 32, 64, 65, 128, 256, 300):
        assert mla.mla_num_sm_parts(rows, 1) == oracle.num_sm_parts_for(rows, 1, sms)


# ----------------------------------------------------------------------------- parity
CASES = [
    # (name, batch, s_q, h_q, seqlens, causal)
    ("r16_ragged", 4, 1, 16, [1, 200, 1000, 4097], False),
    ("r16_short", 3, 1, 16, [63, 64, 65], False),
    ("r8_pad_rows", 2, 1, 8, [300, 77], False),
    ("r32", 3, 1, 32, [129, 640, 2049], False),
    ("r32_causal_sq2", 3, 2, 16, [2, 130, 1000], True),
    ("r64", 2, 1, 64, [500, 1537], False),
    ("r128", 3, 1, 128, [64, 333, 2000], False),
    ("r256_causal", 3, 2, 128, [2, 129, 1500], True),
    ("r48_pad_groups", 2, 1, 48, [257, 1], False),
    ("r96_two_groups", 2, 1, 96, [700, 128], False),
    # CTA-pair path (more than 64 rows): odd block counts per chunk, a half-empty second pair
    ("r128_odd_blocks", 4, 1, 128, [129, 385, 640, 1], False),
    ("r192_two_pairs_causal", 2, 2, 96, [1000, 300], True),
]


@pytest.mark.parametrize("name,batch,s_q,h_q,seqlens,causal", CASES, ids=[c[0] for c in CASES])
@pytest.mark.parametrize("parts", [None, 1, 7])
def test_parity_small(name, batch, s_q, h_q, seqlens, causal, parts):
    case = mi.make_case(batch, s_q, h_q, seqlens, causal=causal, seed=zlib.crc32(name.encode()) % 1000, spare_blocks=2)
    O_ref, L_ref = oracle.mla_decode_reference(case)
    out, lse, status, _ = run_gpu(case, num_sm_parts=parts)
    assert status == 0
    compare(case, out, lse, O_ref, L_ref)


def test_tiny_workload_exact_config():
    case = mi.make_workload("tiny_b2_h16")
    O_ref, L_ref = oracle.mla_decode_reference(case)
    out, lse, status, _ = run_gpu(case)
    assert status == 0
    compare(case, out, lse, O_ref, L_ref)


def test_zero_length_and_fully_masked_rows():
    # request 1 has no cached token; request 0 (causal, L=1, s_q=3) has rows that see nothing
    case = mi.make_case(3, 3, 16, [1, 0, 200], causal=True, seed=21)
    O_ref, L_ref = oracle.mla_decode_reference(case)
    out, lse, status, _ = run_gpu(case)
    assert status == 0
    compare(case, out, lse, O_ref, L_ref)


def test_block_table_permutation_is_bit_invariant():
    case = mi.make_case(3, 1, 16, [300, 1000, 77], seed=22)
    out1, lse1, _, _ = run_gpu(case)
    rng = np.random.default_rng(5)
    perm = rng.permutation(case.num_blocks)
    kv2 = np.empty_like(case.kv)
    kv2[perm] = case.kv
    bt2 = case.block_table.copy()
    bt2[bt2 >= 0] = perm[bt2[bt2 >= 0]]
    case2 = mi.DecodeCase(**{**case.__dict__, "kv": kv2, "block_table": bt2})
    out2, lse2, _, _ = run_gpu(case2)
    assert np.array_equal(out1, out2) and np.array_equal(lse1, lse2)


def test_nan_in_unreadable_slots_does_not_leak():
    clean = mi.make_case(3, 2, 16, [70, 130, 1], causal=True, seed=23, poison=False, spare_blocks=4)
    dirty = mi.make_case(3, 2, 16, [70, 130, 1], causal=True, seed=23, poison=True, spare_blocks=4)
    o1, l1, _, _ = run_gpu(clean)
    o2, l2, _, _ = run_gpu(dirty)
    assert np.isfinite(o2).all()
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def test_pair_fully_masked_rows_and_nan_tails():
    # more than 64 rows (CTA pairs): causal rows that see nothing, an empty request, and NaN
    # in every cache slot no request position covers
    clean = mi.make_case(3, 3, 64, [1, 0, 200], causal=True, seed=26, poison=False, spare_blocks=4)
    dirty = mi.make_case(3, 3, 64, [1, 0, 200], causal=True, seed=26, poison=True, spare_blocks=4)
    O_ref, L_ref = oracle.mla_decode_reference(clean)
    o1, l1, s1, _ = run_gpu(clean)
    o2, l2, s2, _ = run_gpu(dirty)
    assert s1 == 0 and s2 == 0
    compare(clean, o1, l1, O_ref, L_ref)
    assert np.isfinite(o2).all()
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def test_pair_block_table_permutation_is_bit_invariant():
    case = mi.make_case(2, 1, 128, [700, 77], seed=27)
    out1, lse1, _, _ = run_gpu(case)
    rng = np.random.default_rng(6)
    perm = rng.permutation(case.num_blocks)
    kv2 = np.empty_like(case.kv)
    kv2[perm] = case.kv
    bt2 = case.block_table.copy()
    bt2[bt2 >= 0] = perm[bt2[bt2 >= 0]]
    case2 = mi.DecodeCase(**{**case.__dict__, "kv": kv2, "block_table": bt2})
    out2, lse2, _, _ = run_gpu(case2)
    assert np.array_equal(out1, out2) and np.array_equal(lse1, lse2)


def test_split_count_invariance():
    case = mi.make_case(2, 1, 128, [5000, 3000], seed=24)
    O_ref, L_ref = oracle.mla_decode_reference(case)
    results = []
    for parts in (1, 3, 74):
        out, lse, status, _ = run_gpu(case, num_sm_parts=parts)
        assert status == 0
        compare(case, out, lse, O_ref, L_ref)
        results.append((out, lse))
    for out, lse in results[1:]:
        assert np.abs(out - results[0][0]).max() <= 1e-2
        assert np.abs(lse - results[0][1]).max() <= 1e-4


def test_flashmla_style_aliases():
    import attention_mla_get_b200 as mla
    case = mi.make_case(2, 1, 16, [100, 500], seed=25)
    q, kv, bt, sl = to_device(case)
    md, ns = mla.get_mla_metadata(sl, case.s_q * case.h_q // 1, 1)
    out, lse = mla.flash_mla_with_kvcache(q, kv, bt, sl, 512, md, ns, causal=False)
    O_ref, L_ref = oracle.mla_decode_reference(case)
    compare(case, out.float().cpu().numpy(), lse.cpu().numpy(), O_ref, L_ref)


# ------------------------------------------------------------------ full-size workloads
FULL = ["mem_b128_h16_L8192", "varlen_b128_h128", "causal_b64_sq2_h128"]


@pytest.mark.slow
@pytest.mark.parametrize("name", FULL)
def test_full_workload_sampled(name):
    case = mi.make_workload(name)
    out, lse, status, (md, ns) = run_gpu(case)
    assert status == 0
    assert np.isfinite(out).all()
    ns_h = ns.cpu().numpy()
    md_ref, ns_ref = oracle.schedule(case.cache_seqlens, md.shape[0])
    assert np.array_equal(md.cpu().numpy(), md_ref) and np.array_equal(ns_h, ns_ref)
    # sample: the first and last request, the longest, and requests split over several parts
    splits = np.diff(ns_h)
    multi = [int(i) for i in np.nonzero(splits > 1)[0][:2]]
    sample = sorted({0, case.batch - 1, int(np.argmax(case.cache_seqlens)), *multi})
    O_ref, L_ref = oracle.mla_decode_reference(case, requests=sample)
    compare(case, out, lse, O_ref, L_ref, requests=sample)


# ------------------------------------------------------------------------ FP8 cache
FP8_CASES = [
    ("fp8_r16", 3, 1, 16, [1, 300, 2049], False),
    ("fp8_r32", 2, 1, 32, [64, 777], False),
    ("fp8_r64", 2, 1, 64, [129, 1000], False),
    ("fp8_r128", 2, 1, 128, [130, 1000], False),
    ("fp8_r96_pair_pad_rows", 2, 1, 96, [300, 64], False),
    ("fp8_r256_causal", 2, 2, 128, [3, 700], True),
]


@pytest.mark.parametrize("name,batch,s_q,h_q,seqlens,causal", FP8_CASES, ids=[c[0] for c in FP8_CASES])
@pytest.mark.parametrize("parts", [None, 3])
def test_parity_fp8_small(name, batch, s_q, h_q, seqlens, causal, parts):
    case = mi.make_case(batch, s_q, h_q, seqlens, causal=causal, kv_format="fp8",
                        seed=zlib.crc32(name.encode()) % 1000, spare_blocks=2)
    O_ref, L_ref = oracle.mla_decode_reference(case)
    out, lse, status, _ = run_gpu(case, num_sm_parts=parts)
    assert status == 0
    compare(case, out, lse, O_ref, L_ref)


@pytest.mark.parametrize("h_q", [16, 128])
def test_fp8_small_scales(h_q):
    """Scales below 2^-14 (the f16 normal range) take the fp32 product in the dequant of the
    CTA-pair path.  The case is the unit case with every scale and RoPE value times 2^-10 and
    the softmax scale times 2^10: the same softmax, O times 2^-10 (compared at unit scale)."""
    case = mi.make_case(2, 1, h_q, [300, 1000], kv_format="fp8", seed=57, spare_blocks=2)
    kv = case.kv.reshape(-1, mi.FP8_TOKEN_BYTES)
    scales = kv[:, 512:528].copy().view(np.float32) * np.float32(2.0 ** -10)
    kv[:, 512:528] = scales.view(np.uint8)
    rope = kv[:, 528:656].copy().view(np.uint16).astype(np.uint32) << 16
    rope = (rope.view(np.float32) * np.float32(2.0 ** -10)).view(np.uint32) >> 16
    kv[:, 528:656] = rope.astype(np.uint16).view(np.uint8)
    assert float(np.nanmax(scales)) < 2.0 ** -14
    case.softmax_scale = case.softmax_scale * 2.0 ** 10
    O_ref, L_ref = oracle.mla_decode_reference(case)
    out, lse, status, _ = run_gpu(case)
    assert status == 0
    compare(case, out.astype(np.float64) * 2.0 ** 10, lse, O_ref * 2.0 ** 10, L_ref)


def _bf16_bits(x):
    return np.float32(x).view(np.uint32) >> 16


@pytest.mark.parametrize("what", ["scale", "q", "rope", "none"])
def test_fp8_pair_reports_f16_range(what):
    """The CTA-pair FP8 path multiplies f16 operands; a value that leaves the f16 range raises
    MLA_STATUS_F16_RANGE (4) instead of passing silently.  A group scale above 65504 / 448, a
    q value of 70000, or a RoPE dim of 70000 in a token that exists each trigger it; NaN page
    tails (never read into a result) and in-range data do not."""
    case = mi.make_case(2, 1, 128, [300, 1000], kv_format="fp8", seed=58, poison=True, spare_blocks=2)
    kv = case.kv.reshape(-1, 64, mi.FP8_TOKEN_BYTES)
    blk = int(case.block_table[1, 3])          # request 1, tokens 192..255: all exist
    if what == "scale":
        sc = kv[blk, 5, 512:528].copy().view(np.float32)
        sc[2] = np.float32(200.0)
        kv[blk, 5, 512:528] = sc.view(np.uint8)
    elif what == "rope":
        r = kv[blk, 7, 528:656].copy().view(np.uint16)
        r[11] = _bf16_bits(70000.0)
        kv[blk, 7, 528:656] = r.view(np.uint8)
    elif what == "q":
        case.q_bits[0, 0, 77, 300] = _bf16_bits(70000.0)
    out, lse, status, _ = run_gpu(case)
    assert status == (0 if what == "none" else 4)


def test_fp8_nan_in_unreadable_slots_does_not_leak():
    clean = mi.make_case(2, 1, 128, [70, 129], kv_format="fp8", seed=31, poison=False, spare_blocks=3)
    dirty = mi.make_case(2, 1, 128, [70, 129], kv_format="fp8", seed=31, poison=True, spare_blocks=3)
    o1, l1, _, _ = run_gpu(clean)
    o2, l2, _, _ = run_gpu(dirty)
    assert np.isfinite(o2).all()
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


@pytest.mark.slow
def test_full_fp8_workload_sampled():
    case = mi.make_workload("fp8_b128_h128_L16384")
    out, lse, status, (md, ns) = run_gpu(case)
    assert status == 0
    assert np.isfinite(out).all()
    ns_h = ns.cpu().numpy()
    multi = [int(i) for i in np.nonzero(np.diff(ns_h) > 1)[0][:2]]
    sample = sorted({0, case.batch - 1, *multi})
    O_ref, L_ref = oracle.mla_decode_reference(case, requests=sample)
    compare(case, out, lse, O_ref, L_ref, requests=sample)
