"""GPU parity of decode with up to 32 query rows over a bf16 cache (the single-CTA kernel's 16-
and 32-row tiles; the memory-bound shape) against the fp64 oracle: row counts that leave part of
the tile empty, requests that end inside a page or a step or have no second page, requests with
no tokens, causal rows that see nothing, NaN in unreadable cache slots, scheduler part counts
from one to more than there are steps (empty parts), split-count invariance and the block
table's permutation invariance.  Tolerances as in test_gpu_decode.py."""
import numpy as np
import pytest

import mla_inputs as mi
import oracle
from tests._helpers import compare, run_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu(cuda_ok):
    import attention_mla_get_b200  # noqa: F401  (fails loudly if libmla.so is missing)
    yield


@pytest.mark.parametrize("h_q,s_q,causal", [(1, 1, False), (7, 1, False), (16, 1, False), (12, 2, True),
                                            (16, 2, True), (32, 1, False), (5, 3, True)])
def test_row_counts(h_q, s_q, causal):
    # lengths: inside the first page, exactly one page, one page and a token, a step minus one,
    # several steps with a ragged tail
    case = mi.make_case(6, s_q, h_q, [5, 64, 65, 127, 128, 1500], causal=causal, seed=80 + h_q + s_q)
    O_ref, L_ref = oracle.mla_decode_reference(case)
    out, lse, status, _ = run_gpu(case)
    assert status == 0
    compare(case, out, lse, O_ref, L_ref)


@pytest.mark.parametrize("parts", [1, 2, 3, 7, 148, 149])
def test_part_counts(parts):
    # more parts than steps leave parts empty
    case = mi.make_case(3, 1, 16, [4000, 300, 2100], seed=90)
    O_ref, L_ref = oracle.mla_decode_reference(case)
    out, lse, status, (md, ns) = run_gpu(case, num_sm_parts=parts)
    assert status == 0
    md_ref, ns_ref = oracle.schedule(case.cache_seqlens, parts)
    assert np.array_equal(md.cpu().numpy(), md_ref) and np.array_equal(ns.cpu().numpy(), ns_ref)
    compare(case, out, lse, O_ref, L_ref)


def test_empty_requests_masked_rows_and_nan_tails():
    # request 1 has no token; request 0 (causal, L = 1, s_q = 2) has a row that sees nothing;
    # every cache slot no request position covers holds NaN in the dirty copy
    clean = mi.make_case(3, 2, 16, [1, 0, 200], causal=True, seed=91, poison=False, spare_blocks=4)
    dirty = mi.make_case(3, 2, 16, [1, 0, 200], causal=True, seed=91, poison=True, spare_blocks=4)
    O_ref, L_ref = oracle.mla_decode_reference(clean)
    o1, l1, s1, _ = run_gpu(clean)
    o2, l2, s2, _ = run_gpu(dirty)
    assert s1 == 0 and s2 == 0
    compare(clean, o1, l1, O_ref, L_ref)
    assert np.isfinite(o2).all()
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def test_split_count_invariance():
    case = mi.make_case(2, 1, 16, [9000, 3000], seed=92)
    O_ref, L_ref = oracle.mla_decode_reference(case)
    results = []
    for parts in (1, 5, 148):
        out, lse, status, _ = run_gpu(case, num_sm_parts=parts)
        assert status == 0
        compare(case, out, lse, O_ref, L_ref)
        results.append((out, lse))
    for out, lse in results[1:]:
        assert np.abs(out - results[0][0]).max() <= 1e-2
        assert np.abs(lse - results[0][1]).max() <= 1e-4


def test_block_table_permutation_is_bit_invariant():
    case = mi.make_case(3, 1, 16, [700, 77, 1300], seed=93)
    out1, lse1, _, _ = run_gpu(case)
    rng = np.random.default_rng(8)
    perm = rng.permutation(case.num_blocks)
    kv2 = np.empty_like(case.kv)
    kv2[perm] = case.kv
    bt2 = case.block_table.copy()
    bt2[bt2 >= 0] = perm[bt2[bt2 >= 0]]
    case2 = mi.DecodeCase(**{**case.__dict__, "kv": kv2, "block_table": bt2})
    out2, lse2, _, _ = run_gpu(case2)
    assert np.array_equal(out1, out2) and np.array_equal(lse1, lse2)
