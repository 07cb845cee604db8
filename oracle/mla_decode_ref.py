"""Oracle (test infrastructure): MLA decode over a paged KV cache, fp64, by definition.

What is computed (FlashMLA pages: "flash_api.cpp" excerpt on the mmssai.com page --
q is batch x seqlen_q x num_heads x head_size, kcache is num_blocks x
page_block_size x num_heads_k x head_size, head_size_v is the value width,
seqlens_k and block_table address the pages, softmax_scale and is_causal; the
query fold q.view(b, s_q, h_kv, ngroups, d).transpose(2, 3) on the
deepseekonline.chat page; 576 = 512 latent + 64 RoPE dims and the 64-token page on
the wmrh.cn and kdjingpai.com pages):

  for request b, query position i in [0, s_q) and head h:
    K_b[j]  = kvcache[block_table[b][j // 64]][j % 64][0][0:576]     for j < L_b
    visible = { j < L_b }, and if causal also j <= L_b - s_q + i
              (the query block sits at the end of the cache)
    s_j     = softmax_scale * sum_d q[b, i, h, d] * K_b[j][d]        over all 576 dims
    LSE     = m + log sum_j exp(s_j - m),  m = max_j s_j              (natural log)
    O[d]    = sum_j exp(s_j - LSE) * K_b[j][d]                        for d < 512

O is [b, s_q, h_q, 512], LSE is [b, h_q, s_q].  With h_kv = 1 every head of a
request reads the same cached vectors.  A row with no visible key has O = 0 and
LSE = -inf.  Everything is fp64; bf16 inputs are widened exactly.  The only
library primitives used are numpy's matrix product and exp/log.
"""
from __future__ import annotations

import numpy as np

from .fp8_format import decode_fp8_tokens

D_QK, D_V, PAGE = 576, 512, 64


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact value of bf16 bit patterns (the high half of a float32)."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def gather_request_keys(case, b: int) -> np.ndarray:
    """K_b [L_b, 576] fp64: logical token j lives in page block_table[b][j // 64], slot j % 64."""
    L = int(case.cache_seqlens[b])
    if L <= 0:
        return np.zeros((0, D_QK), dtype=np.float64)
    n_pages = (L + PAGE - 1) // PAGE
    pages = case.block_table[b, :n_pages].astype(np.int64)
    raw = case.kv[pages]                                   # [n_pages, 64, ...]
    raw = raw.reshape(n_pages * PAGE, raw.shape[-1])[:L]
    if case.kv_format == "bf16":
        return bf16_to_f64(raw)
    if case.kv_format == "fp8":
        return decode_fp8_tokens(raw)
    raise ValueError(case.kv_format)


def visible_keys(L: int, s_q: int, i: int, causal: bool) -> int:
    """Number of keys query position i may see: the first n of the request's L keys."""
    n = L if not causal else min(L, L - s_q + i + 1)
    return max(0, n)


def attend_rows(qrows: np.ndarray, K: np.ndarray, n_visible: np.ndarray, scale: float):
    """Softmax attention of fp64 query rows [n, 576] over the first n_visible[r] rows of K.

    Returns (O [n, 512], LSE [n]).  Rows with no visible key give O = 0, LSE = -inf.
    """
    n = qrows.shape[0]
    O = np.zeros((n, D_V), dtype=np.float64)
    lse = np.full(n, -np.inf, dtype=np.float64)
    if K.shape[0] == 0:
        return O, lse
    S = scale * (qrows @ K.T)                              # [n, L] scaled scores
    for r in range(n):
        v = int(n_visible[r])
        if v <= 0:
            continue
        s = S[r, :v]
        m = s.max()
        lse[r] = m + np.log(np.exp(s - m).sum())
        p = np.exp(s - lse[r])
        O[r] = p @ K[:v, :D_V]
    return O, lse


def mla_decode_reference(case, requests=None):
    """Decode every request (or the listed ones).

    Returns (O fp64 [b, s_q, h_q, 512], LSE fp64 [b, h_q, s_q]); entries of requests
    not listed are NaN.
    """
    assert case.h_kv == 1, "the oracle follows the h_kv = 1 reading of the pages"
    B, s_q, h_q = case.batch, case.s_q, case.h_q
    O = np.full((B, s_q, h_q, D_V), np.nan, dtype=np.float64)
    LSE = np.full((B, h_q, s_q), np.nan, dtype=np.float64)
    todo = range(B) if requests is None else requests
    for b in todo:
        L = int(case.cache_seqlens[b])
        K = gather_request_keys(case, b)
        q = bf16_to_f64(case.q_bits[b]).reshape(s_q * h_q, D_QK)     # row r = i*h_q + h
        nvis = np.array([visible_keys(L, s_q, r // h_q, case.causal) for r in range(s_q * h_q)])
        o, l = attend_rows(q, K, nvis, case.softmax_scale)
        O[b] = o.reshape(s_q, h_q, D_V)
        LSE[b] = l.reshape(s_q, h_q).T
    return O, LSE


def mla_sparse_decode_reference(case, indices, requests=None):
    """Token-sparse decode (the `indices` argument of flash_mla_with_kvcache and `topk` of
    get_mla_metadata on the gitcode FlashMLA page, "解码阶段使用示例" / "稀疏解码场景"),
    by definition, in fp64.

    Reading (the page gives the call, not the shape): indices is int32 [b, s_q, topk];
    query position i of request b attends to the tokens at the logical cache positions
    indices[b, i, :] (addressed through block_table like every other key); an entry outside
    [0, L_b) is an empty slot and contributes nothing; a position listed twice counts twice.
    No causal mask applies (the index list already says what a query sees).

      s_k  = softmax_scale * q[b, i, h] . K_b[indices[b, i, k]]       for valid k
      LSE  = log sum_k exp(s_k),  O = sum_k exp(s_k - LSE) * K_b[indices[b, i, k]][:512]

    Returns (O fp64 [b, s_q, h_q, 512], LSE fp64 [b, h_q, s_q]); a query with no valid
    entry has O = 0 and LSE = -inf; requests not listed are NaN.
    """
    assert case.h_kv == 1, "the oracle follows the h_kv = 1 reading of the pages"
    idx = np.asarray(indices)
    B, s_q, h_q = case.batch, case.s_q, case.h_q
    assert idx.ndim == 3 and idx.shape[:2] == (B, s_q), idx.shape
    O = np.full((B, s_q, h_q, D_V), np.nan, dtype=np.float64)
    LSE = np.full((B, h_q, s_q), np.nan, dtype=np.float64)
    todo = range(B) if requests is None else requests
    for b in todo:
        L = int(case.cache_seqlens[b])
        K = gather_request_keys(case, b)                             # [L, 576]
        q = bf16_to_f64(case.q_bits[b])                              # [s_q, h_q, 576]
        for i in range(s_q):
            sel = [int(j) for j in idx[b, i] if 0 <= int(j) < L]
            Ki = K[sel] if sel else np.zeros((0, D_QK), dtype=np.float64)
            o, l = attend_rows(q[i], Ki, np.full(h_q, len(sel)), case.softmax_scale)
            O[b, i] = o
            LSE[b, :, i] = l
    return O, LSE


def mla_sparse_prefill_reference(q_bits, kv_bits, indices, softmax_scale: float):
    """Sparse prefill (flash_mla_sparse_fwd(q, kv, indices, sm_scale, d_v = 512) on the gitcode
    FlashMLA page, "稀疏预填充使用"), by definition, in fp64: query token i, head h attends to
    the rows kv[indices[i, k]] with 0 <= indices[i, k] < s_kv (other entries are empty slots):

      s_k = softmax_scale * q[i, h] . kv[indices[i, k]],  LSE = log sum_k exp(s_k),
      O   = sum_k exp(s_k - LSE) * kv[indices[i, k]][:512]

    q_bits bf16 bits [s_q, h_q, 576], kv_bits bf16 bits [s_kv, 576], indices [s_q, topk].
    Returns (O fp64 [s_q, h_q, 512], LSE fp64 [h_q, s_q]); no valid entry: O = 0, LSE = -inf.
    """
    q = bf16_to_f64(q_bits)
    kv = bf16_to_f64(kv_bits)
    s_kv = kv.shape[0]
    s_q, h_q = q.shape[0], q.shape[1]
    O = np.zeros((s_q, h_q, D_V), dtype=np.float64)
    LSE = np.full((h_q, s_q), -np.inf, dtype=np.float64)
    for i in range(s_q):
        sel = [int(j) for j in np.asarray(indices[i]).reshape(-1) if 0 <= int(j) < s_kv]
        if not sel:
            continue
        o, l = attend_rows(q[i], kv[sel], np.full(h_q, len(sel)), softmax_scale)
        O[i] = o
        LSE[:, i] = l
    return O, LSE
