"""Pins of the fp64 oracle against things other than itself.

* brute force: scalar Python loops over a gather written independently here
* closed forms: equal scores give LSE = log n + s and O = mean of V; a single key
  gives O = V_0 and LSE = s_0
* invariants: block-table permutation, NaN in unreadable slots, causal with s_q = 1,
  causal row 0 of s_q = 2 equals non-causal over L - 1 keys, a constant added to
  every score of a row, a scale applied to V, a dominant key, split-and-merge by LSE
* planted mistakes: each check above is shown to fail when a plausible bug is
  planted in the oracle (monkeypatched, on the CPU)
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


def brute_force(case):
    """Dense attention written as scalar loops straight from the definition."""
    B, s_q, h_q = case.batch, case.s_q, case.h_q
    O = np.zeros((B, s_q, h_q, 512))
    LSE = np.zeros((B, h_q, s_q))
    for b in range(B):
        L = int(case.cache_seqlens[b])
        keys = []
        for j in range(L):
            page = int(case.block_table[b][j // 64])
            keys.append([_bf16(x) for x in case.kv[page][j % 64]])
        for i in range(s_q):
            limit = L if not case.causal else min(L, L - s_q + i + 1)
            for h in range(h_q):
                q = [_bf16(x) for x in case.q_bits[b][i][h]]
                s = []
                for j in range(limit):
                    acc = 0.0
                    k = keys[j]
                    for d in range(576):
                        acc += q[d] * k[d]
                    s.append(case.softmax_scale * acc)
                if not s:
                    LSE[b, h, i] = -math.inf
                    continue
                m = max(s)
                lse = m + math.log(sum(math.exp(x - m) for x in s))
                LSE[b, h, i] = lse
                for d in range(512):
                    O[b, i, h, d] = sum(math.exp(s[j] - lse) * keys[j][d] for j in range(limit))
    return O, LSE


def _err(*diffs):
    """Largest absolute difference; NaN anywhere counts as an infinite error."""
    m = max(float(np.max(np.abs(d))) if np.size(d) else 0.0 for d in diffs)
    return math.inf if math.isnan(m) else m


def _tiny(causal, s_q=2, h_q=2, seqlens=(70, 130), seed=11, **kw):
    return mi.make_case(len(seqlens), s_q, h_q, list(seqlens), causal=causal, seed=seed, **kw)


def check_brute_force(causal):
    case = _tiny(causal)
    O, L = oracle.mla_decode_reference(case)
    Ob, Lb = brute_force(case)
    return _err(O - Ob, L - Lb)


@pytest.mark.parametrize("causal", [False, True])
def test_brute_force(causal):
    assert check_brute_force(causal) < 1e-11


def check_closed_form_equal_scores():
    # q = 0: every score is 0, so LSE = log n and O is the plain mean of V
    case = _tiny(False, s_q=1, h_q=3, seqlens=(1, 64, 65, 300))
    case.q_bits[:] = 0
    O, L = oracle.mla_decode_reference(case)
    err = 0.0
    for b in range(case.batch):
        n = int(case.cache_seqlens[b])
        V = np.array([[_bf16(x) for x in case.kv[case.block_table[b][j // 64]][j % 64][:512]] for j in range(n)])
        err = max(err, np.abs(L[b] - math.log(n)).max(), np.abs(O[b, 0] - V.mean(0)).max())
    return err


def test_closed_form_equal_scores():
    assert check_closed_form_equal_scores() < 1e-12


def check_identical_keys():
    # every key is the same vector k: s = scale * q.k for all n keys, LSE = log n + s, O = k[:512]
    case = _tiny(False, s_q=1, h_q=4, seqlens=(129,), seed=5)
    k = case.kv[int(case.block_table[0][0])][0].copy()
    case.kv[:] = k
    O, L = oracle.mla_decode_reference(case)
    kf = np.array([_bf16(x) for x in k])
    err = 0.0
    for h in range(4):
        q = np.array([_bf16(x) for x in case.q_bits[0][0][h]])
        s = case.softmax_scale * float(np.dot(q, kf))
        err = max(err, abs(L[0, h, 0] - (math.log(129) + s)), np.abs(O[0, 0, h] - kf[:512]).max())
    return err


def test_identical_keys():
    assert check_identical_keys() < 1e-11


def check_single_key():
    case = _tiny(False, s_q=1, h_q=2, seqlens=(1, 1), seed=6)
    O, L = oracle.mla_decode_reference(case)
    err = 0.0
    for b in range(2):
        k = np.array([_bf16(x) for x in case.kv[case.block_table[b][0]][0]])
        for h in range(2):
            q = np.array([_bf16(x) for x in case.q_bits[b][0][h]])
            err = max(err, abs(L[b, h, 0] - case.softmax_scale * float(np.dot(q, k))),
                      np.abs(O[b, 0, h] - k[:512]).max())
    return err


def test_single_key():
    assert check_single_key() < 1e-12


def test_block_table_permutation_invariant():
    case = _tiny(True, s_q=2, h_q=3, seqlens=(200, 77, 129), seed=7)
    O, L = oracle.mla_decode_reference(case)
    rng = np.random.default_rng(123)
    perm = rng.permutation(case.num_blocks)          # new physical position of each page
    kv2 = np.empty_like(case.kv)
    kv2[perm] = case.kv
    bt2 = case.block_table.copy()
    used = bt2 >= 0
    bt2[used] = perm[bt2[used]]
    case2 = mi.DecodeCase(**{**case.__dict__, "kv": kv2, "block_table": bt2})
    O2, L2 = oracle.mla_decode_reference(case2)
    assert np.array_equal(O, O2) and np.array_equal(L, L2)


def test_nan_poison_unreadable_slots():
    clean = _tiny(False, s_q=1, h_q=2, seqlens=(70, 130, 1), seed=8, poison=False, spare_blocks=3)
    dirty = _tiny(False, s_q=1, h_q=2, seqlens=(70, 130, 1), seed=8, poison=True, spare_blocks=3)
    assert np.isnan(mi.bf16_bits_to_f32(dirty.kv)).any()
    O1, L1 = oracle.mla_decode_reference(clean)
    O2, L2 = oracle.mla_decode_reference(dirty)
    assert np.isfinite(O2).all() and np.isfinite(L2).all()
    assert np.array_equal(O1, O2) and np.array_equal(L1, L2)


def test_causal_single_query_equals_noncausal():
    a = _tiny(True, s_q=1, h_q=4, seqlens=(5, 64, 200), seed=9)
    b = mi.DecodeCase(**{**a.__dict__, "causal": False})
    Oa, La = oracle.mla_decode_reference(a)
    Ob, Lb = oracle.mla_decode_reference(b)
    assert np.array_equal(Oa, Ob) and np.array_equal(La, Lb)


def check_causal_first_row():
    a = _tiny(True, s_q=2, h_q=3, seqlens=(65, 130, 2), seed=10, poison=False)
    short = mi.DecodeCase(**{**a.__dict__, "causal": False, "s_q": 1,
                             "cache_seqlens": a.cache_seqlens - 1,
                             "q_bits": a.q_bits[:, :1].copy()})
    Oa, La = oracle.mla_decode_reference(a)
    Os, Ls = oracle.mla_decode_reference(short)
    return max(np.abs(Oa[:, 0] - Os[:, 0]).max(), np.abs(La[:, :, 0] - Ls[:, :, 0]).max())


def test_causal_first_row():
    assert check_causal_first_row() == 0.0


def test_constant_score_shift():
    case = _tiny(False, s_q=1, h_q=2, seqlens=(100, 33), seed=12)
    one = np.uint16(0x3F80)                           # bf16 1.0 in the last RoPE dim of every key
    case.kv[:, :, 575] = one
    shifted = mi.DecodeCase(**{**case.__dict__, "q_bits": case.q_bits.copy()})
    case.q_bits[..., 575] = np.uint16(0x4000)         # q[575] = 2.0
    shifted.q_bits[..., 575] = np.uint16(0x4080)      # q[575] = 4.0: every score moves by 2 * scale
    O, L = oracle.mla_decode_reference(case)
    O2, L2 = oracle.mla_decode_reference(shifted)
    assert np.abs(L2 - L - 2.0 * case.softmax_scale).max() < 1e-12
    assert np.abs(O2 - O).max() < 1e-12


def test_value_scaling():
    case = _tiny(False, s_q=1, h_q=2, seqlens=(90,), seed=13)
    case.q_bits[..., :512] = 0                        # scores use the RoPE dims only
    O, L = oracle.mla_decode_reference(case)
    k = mi.bf16_bits_to_f32(case.kv[..., :512]) * np.float32(2.0)   # exact in bf16
    scaled = mi.DecodeCase(**{**case.__dict__, "kv": case.kv.copy()})
    scaled.kv[..., :512] = mi.f32_to_bf16_bits(k)
    O2, L2 = oracle.mla_decode_reference(scaled)
    assert np.abs(L2 - L).max() == 0.0
    assert np.abs(O2 - 2.0 * O).max() < 1e-12


def test_dominant_key():
    case = _tiny(False, s_q=1, h_q=1, seqlens=(150,), seed=14)
    j = 77
    page = int(case.block_table[0][j // 64])
    k = case.kv[page][j % 64]
    case.q_bits[0, 0, 0] = mi.f32_to_bf16_bits(mi.bf16_bits_to_f32(k) * np.float32(4.0))
    O, L = oracle.mla_decode_reference(case)
    kf = mi.bf16_bits_to_f32(k).astype(np.float64)
    assert np.abs(O[0, 0, 0] - kf[:512]).max() < 1e-9


def test_split_and_merge_by_lse():
    """Attending over key ranges separately and merging with weights exp(lse_s - LSE)
    gives the full result (the algebra the split-KV combine relies on)."""
    case = _tiny(False, s_q=1, h_q=4, seqlens=(1000,), seed=15)
    K = oracle.gather_request_keys(case, 0)
    q = oracle.bf16_to_f64(case.q_bits[0]).reshape(4, 576)
    full_o, full_l = oracle.attend_rows(q, K, np.full(4, 1000), case.softmax_scale)
    cuts = [0, 128, 129, 640, 1000]
    parts = [oracle.attend_rows(q, K[a:b], np.full(4, b - a), case.softmax_scale) for a, b in zip(cuts, cuts[1:])]
    lses = np.stack([p[1] for p in parts])            # [splits, rows]
    m = lses.max(0)
    lse = m + np.log(np.exp(lses - m).sum(0))
    o = sum(np.exp(l - lse)[:, None] * p for p, l in zip([p[0] for p in parts], lses))
    assert np.abs(lse - full_l).max() < 1e-12
    assert np.abs(o - full_o).max() < 1e-12


def test_zero_visible_keys():
    case = _tiny(True, s_q=3, h_q=2, seqlens=(1, 0), seed=16)
    O, L = oracle.mla_decode_reference(case)
    # request 0: L = 1, s_q = 3 -> positions 0, 1 see nothing, position 2 sees key 0
    assert np.isneginf(L[0, :, 0]).all() and np.isneginf(L[0, :, 1]).all() and np.isfinite(L[0, :, 2]).all()
    assert (O[0, :2] == 0).all()
    assert np.isneginf(L[1]).all() and (O[1] == 0).all()


# ---------------------------------------------------------------------------
# planted mistakes: every pin above must catch at least one plausible bug
# ---------------------------------------------------------------------------

def _planted(monkeypatch, name, fn):
    monkeypatch.setattr(ref, name, fn)


def test_planted_causal_off_by_one(monkeypatch):
    orig = ref.visible_keys
    _planted(monkeypatch, "visible_keys", lambda L, s_q, i, causal: orig(L, s_q, i, causal) - (1 if causal else 0))
    assert check_brute_force(True) > 1e-3


def test_planted_dropped_rope_dims(monkeypatch):
    orig = ref.gather_request_keys

    def bad(case, b):
        K = orig(case, b).copy()
        K[:, 512:] = 0
        return K
    _planted(monkeypatch, "gather_request_keys", bad)
    assert check_brute_force(False) > 1e-3


def test_planted_value_offset(monkeypatch):
    orig = ref.attend_rows

    def bad(qrows, K, n_visible, scale):
        K2 = np.concatenate([K[:, 64:], K[:, :64]], axis=1)   # V taken from dims 64..575
        o, _ = orig(qrows, K2, n_visible, scale)
        _, l = orig(qrows, K, n_visible, scale)
        return o, l
    _planted(monkeypatch, "attend_rows", bad)
    assert check_single_key() > 1e-3


def test_planted_page_index_swap(monkeypatch):
    def bad(case, b):
        L = int(case.cache_seqlens[b])
        n = (L + 63) // 64
        pages = case.block_table[b, :n][::-1].astype(np.int64)     # pages in the wrong order
        raw = case.kv[pages].reshape(n * 64, -1)[:L]
        return ref.bf16_to_f64(raw)
    _planted(monkeypatch, "gather_request_keys", bad)
    assert check_brute_force(False) > 1e-3


def test_planted_missing_scale(monkeypatch):
    orig = ref.attend_rows
    _planted(monkeypatch, "attend_rows", lambda q, K, n, s: orig(q, K, n, 1.0))
    assert check_identical_keys() > 1e-3


def test_planted_log2(monkeypatch):
    orig = ref.attend_rows

    def bad(q, K, n, s):
        o, l = orig(q, K, n, s)
        return o, l / math.log(2.0)
    _planted(monkeypatch, "attend_rows", bad)
    assert check_closed_form_equal_scores() > 1e-3


def test_planted_row_order(monkeypatch):
    orig = ref.mla_decode_reference

    def bad(case, requests=None):
        O, L = orig(case, requests)
        # row fold r = h*s_q + i instead of i*h_q + h
        Ob = O.transpose(0, 2, 1, 3).reshape(O.shape[0], -1, 512).reshape(O.shape)
        return Ob, L
    import oracle as orc
    monkeypatch.setattr(orc, "mla_decode_reference", bad)
    assert check_brute_force(True) > 1e-3
