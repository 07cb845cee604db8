"""Pins of the token-sparse decode oracle (mla_sparse_decode_reference) against things other
than itself.

* brute force: scalar loops over an index list, with a gather written independently here
* the dense definition: listing every cache position once (in any order) is dense,
  non-causal decode
* closed forms: every position listed twice gives the same O and LSE + ln 2; one valid
  entry gives O = V_j and LSE = s_j; an empty list gives O = 0 and LSE = -inf
* invariants: permuting a list; entries outside [0, L) (including NaN-poisoned unused
  slots) contribute nothing
* planted mistakes: each check above is shown to fail when a plausible bug is planted in
  the oracle (monkeypatched, on the CPU)
"""
import math
import struct

import numpy as np
import pytest

import mla_inputs as mi
import oracle
from oracle import mla_decode_ref as ref


def _bf16(bits: int) -> float:
    return struct.unpack(">f", struct.pack(">I", (int(bits) & 0xFFFF) << 16))[0]


def _err(*diffs):
    m = max(float(np.max(np.abs(d))) if np.size(d) else 0.0 for d in diffs)
    return math.inf if math.isnan(m) else m


def brute_force_sparse(case, idx):
    B, s_q, h_q = case.batch, case.s_q, case.h_q
    O = np.zeros((B, s_q, h_q, 512))
    LSE = np.zeros((B, h_q, s_q))
    for b in range(B):
        L = int(case.cache_seqlens[b])
        for i in range(s_q):
            keys = []
            for j in idx[b][i]:
                j = int(j)
                if 0 <= j < L:
                    page = int(case.block_table[b][j // 64])
                    keys.append([_bf16(x) for x in case.kv[page][j % 64]])
            for h in range(h_q):
                q = [_bf16(x) for x in case.q_bits[b][i][h]]
                s = [case.softmax_scale * sum(q[d] * k[d] for d in range(576)) for k in keys]
                if not s:
                    LSE[b, h, i] = -math.inf
                    continue
                m = max(s)
                lse = m + math.log(sum(math.exp(x - m) for x in s))
                LSE[b, h, i] = lse
                for d in range(512):
                    O[b, i, h, d] = sum(math.exp(s[k] - lse) * keys[k][d] for k in range(len(keys)))
    return O, LSE


def _case(seqlens=(70, 130), s_q=2, h_q=2, seed=21, **kw):
    return mi.make_case(len(seqlens), s_q, h_q, list(seqlens), seed=seed, **kw)


def check_brute_force():
    case = _case()
    idx = mi.make_sparse_indices(case.cache_seqlens, case.s_q, 24, 5, invalid_frac=0.2, duplicate_frac=0.2)
    O, L = oracle.mla_sparse_decode_reference(case, idx)
    Ob, Lb = brute_force_sparse(case, idx)
    return _err(O - Ob, L - Lb)


def test_brute_force():
    assert check_brute_force() < 1e-11


def check_all_positions_is_dense():
    case = _case(seqlens=(70, 200, 1), s_q=2, h_q=3, seed=22, causal=False)
    rng = np.random.default_rng(3)
    topk = int(case.cache_seqlens.max()) + 5
    idx = np.full((case.batch, case.s_q, topk), -1, dtype=np.int32)
    for b in range(case.batch):
        for i in range(case.s_q):
            L = int(case.cache_seqlens[b])
            idx[b, i, :L] = rng.permutation(L)
            rng.shuffle(idx[b, i])
    O, L = oracle.mla_sparse_decode_reference(case, idx)
    Od, Ld = oracle.mla_decode_reference(case)
    return _err(O - Od, L - Ld)


def test_all_positions_is_dense():
    assert check_all_positions_is_dense() < 1e-12


def check_duplicates_double_the_weight():
    case = _case(seed=23)
    idx = mi.make_sparse_indices(case.cache_seqlens, case.s_q, 16, 6)
    twice = np.concatenate([idx, idx], axis=-1)
    O1, L1 = oracle.mla_sparse_decode_reference(case, idx)
    O2, L2 = oracle.mla_sparse_decode_reference(case, twice)
    return _err(O2 - O1, L2 - (L1 + math.log(2.0)))


def test_duplicates_double_the_weight():
    assert check_duplicates_double_the_weight() < 1e-12


def check_single_entry():
    case = _case(seed=24, s_q=1, h_q=2)
    idx = np.full((case.batch, 1, 8), -1, dtype=np.int32)
    idx[:, 0, 5] = [17, 99]                                # one valid position per request
    O, L = oracle.mla_sparse_decode_reference(case, idx)
    err = 0.0
    for b, j in enumerate([17, 99]):
        # key j read straight from its page (not through the oracle's gather)
        kj = np.array([_bf16(x) for x in case.kv[int(case.block_table[b][j // 64])][j % 64]])
        q = np.array([[_bf16(x) for x in row] for row in case.q_bits[b, 0]])
        s = case.softmax_scale * (q @ kj)
        err = max(err, _err(O[b, 0] - kj[None, :512], L[b, :, 0] - s))
    return err


def test_single_entry():
    assert check_single_entry() < 1e-12


def test_empty_lists():
    case = _case(seed=25)
    idx = np.full((case.batch, case.s_q, 4), -1, dtype=np.int32)
    idx[0, 0, :] = [70, 71, 5000, -7]                      # all outside [0, L_0 = 70)
    O, L = oracle.mla_sparse_decode_reference(case, idx)
    assert np.all(O == 0.0) and np.all(np.isneginf(L))


def check_permutation_invariant():
    case = _case(seed=26)
    idx = mi.make_sparse_indices(case.cache_seqlens, case.s_q, 32, 8, invalid_frac=0.2)
    perm = idx[..., np.random.default_rng(9).permutation(idx.shape[-1])]
    O1, L1 = oracle.mla_sparse_decode_reference(case, idx)
    O2, L2 = oracle.mla_sparse_decode_reference(case, perm)
    return _err(O2 - O1, L2 - L1)


def test_permutation_invariant():
    assert check_permutation_invariant() < 1e-12


def test_unused_slots_never_read():
    # positions past L (their page slots hold NaN in the poisoned case) contribute nothing
    clean = _case(seed=27, poison=False, spare_blocks=2)
    dirty = _case(seed=27, poison=True, spare_blocks=2)
    idx = mi.make_sparse_indices(clean.cache_seqlens, clean.s_q, 40, 10, invalid_frac=0.3)
    O1, L1 = oracle.mla_sparse_decode_reference(clean, idx)
    O2, L2 = oracle.mla_sparse_decode_reference(dirty, idx)
    assert np.isfinite(O2).all()
    assert np.array_equal(O1, O2) and np.array_equal(L1, L2)


# --------------------------------------------------------------- planted mistakes
def _plant_ignore_validity(monkeypatch):
    real = ref.attend_rows

    def bad(qrows, K, n_visible, scale):
        return real(qrows, K, np.maximum(n_visible - 1, 0), scale)   # drops the last listed key
    monkeypatch.setattr(ref, "attend_rows", bad)


def test_planted_dropped_entry(monkeypatch):
    _plant_ignore_validity(monkeypatch)
    assert check_brute_force() > 1e-6
    assert check_all_positions_is_dense() > 1e-6


def test_planted_value_offset(monkeypatch):
    real = ref.gather_request_keys

    def bad(case, b):
        K = real(case, b).copy()
        if K.shape[0] > 1:
            K[:, :512] = np.roll(K[:, :512], 1, axis=0)            # V of the wrong token
        return K
    monkeypatch.setattr(ref, "gather_request_keys", bad)
    assert check_brute_force() > 1e-6
    assert check_single_entry() > 1e-6


# --------------------------------------------------------------- sparse prefill
def _prefill_kv(case):
    s_kv = int(case.cache_seqlens[0])
    return case.kv.reshape(-1, case.kv.shape[-1])[:s_kv]


def check_prefill_brute_force():
    case = mi.make_prefill_case(3, 2, 150, 20, seed=31, invalid_frac=0.2)
    O, L = oracle.mla_sparse_prefill_reference(case.q_bits[0], _prefill_kv(case), case.indices[0], case.softmax_scale)
    Ob, Lb = brute_force_sparse(case, case.indices)          # one request, identity block table
    return _err(O - Ob[0], L - Lb[0])


def test_prefill_brute_force():
    assert check_prefill_brute_force() < 1e-11


def test_prefill_is_one_request_of_sparse_decode():
    case = mi.make_prefill_case(5, 3, 333, 64, seed=32, invalid_frac=0.1)
    O, L = oracle.mla_sparse_prefill_reference(case.q_bits[0], _prefill_kv(case), case.indices[0], case.softmax_scale)
    Od, Ld = oracle.mla_sparse_decode_reference(case, case.indices)
    assert _err(O - Od[0], L - Ld[0]) < 1e-12


def test_planted_prefill_row_offset(monkeypatch):
    real = ref.attend_rows

    def bad(qrows, K, n_visible, scale):
        K2 = K.copy()
        K2[:, :512] = np.roll(K[:, :512], 1, axis=0)                  # values of the wrong rows
        return real(qrows, K2, n_visible, scale)
    monkeypatch.setattr(ref, "attend_rows", bad)
    assert check_prefill_brute_force() > 1e-6
