"""Seeded synthetic inputs for MLA decode over a paged KV cache.

This module only builds inputs: random query rows, a paged latent KV cache, a
block table and per-request cache lengths, in the shapes of the workloads the
FlashMLA pages describe (q [b, s_q, h_q, 576], kvcache [num_blocks, 64, h_kv=1,
576], block_table [b, max_blocks], cache_seqlens [b]; "flash_api.cpp" excerpt on
the mmssai.com page, and the usage snippets on the kdjingpai.com / aiboss88.com
pages).  It holds none of the attention arithmetic: both the fp64 oracle and the
CUDA path consume what it returns.

All arrays are numpy.  bf16 values are carried as their uint16 bit patterns.
Random streams are counter-keyed numpy ``SeedSequence`` children, one per
(stream, chunk), so the result depends only on the seed and never on the number
of host threads used to fill it.

FP8 cache layout (wmrh.cn page, "FP8 KV缓存内存效率" table): every token is 656
bytes -- 512 float8_e4m3 codes of the latent (NoPE) dims, then 4 float32 scales
(one per 128 latent dims), then 64 bfloat16 RoPE dims.  The quantiser that
produces those bytes from bf16 N(0,1) values is input construction (it is what a
cache writer does), not part of decode: scale = max|x| / 448 per 128-dim group,
code = e4m3(x / scale) rounded to nearest-even with saturation to +-448, and a
group of zeros stores scale 0 and zero codes.
"""
from __future__ import annotations

import math
import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field, replace
from typing import Optional, Sequence

import numpy as np

D_QK = 576          # 512 latent (NoPE) dims + 64 RoPE dims
D_V = 512           # V is the first 512 dims of the cached vector
D_ROPE = 64
PAGE = 64           # tokens per KV page
FP8_TOKEN_BYTES = 656
FP8_GROUP = 128     # latent dims per fp32 scale
E4M3_MAX = 448.0

BF16_NAN = np.uint16(0x7FC0)
E4M3_NAN = np.uint8(0x7F)

_CHUNK_ELEMS = 1 << 22   # elements per random chunk (fixed: keeps results thread-count independent)

# random stream ids
_S_SEQLENS, _S_PERM, _S_Q, _S_KV, _S_IDX = 0, 1, 2, 3, 4


@dataclass
class DecodeCase:
    """One batch of decode inputs (host arrays)."""
    q_bits: np.ndarray            # uint16 [b, s_q, h_q, 576]  bf16 bits
    kv: np.ndarray                # uint16 [num_blocks, 64, 576] (bf16 bits) | uint8 [num_blocks, 64, 656]
    block_table: np.ndarray       # int32 [b, max_blocks], unused entries = -1
    cache_seqlens: np.ndarray     # int32 [b]
    s_q: int
    h_q: int
    causal: bool
    softmax_scale: float
    kv_format: str = "bf16"       # "bf16" | "fp8"
    h_kv: int = 1
    name: str = ""
    meta: dict = field(default_factory=dict)
    indices: Optional[np.ndarray] = None   # token-sparse decode: int32 [b, s_q, topk], else None

    @property
    def topk(self) -> int:
        return 0 if self.indices is None else int(self.indices.shape[-1])

    @property
    def batch(self) -> int:
        return int(self.cache_seqlens.shape[0])

    @property
    def rows(self) -> int:
        """Query rows per kv head: s_q * h_q / h_kv."""
        return self.s_q * self.h_q // self.h_kv

    @property
    def num_blocks(self) -> int:
        return int(self.kv.shape[0])

    def kv_bytes_per_token(self) -> int:
        return FP8_TOKEN_BYTES if self.kv_format == "fp8" else 2 * D_QK


# ----------------------------------------------------------------------------
# workload presets (the five decode workloads, by what they are)
# ----------------------------------------------------------------------------

@dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    s_q: int
    h_q: int
    seqlens: str                  # "fixed:<L>", "list:<a,b,..>", "uniform:<lo>:<hi>", "normal:<mu>:<sigma>:<lo>:<hi>"
    causal: bool
    kv_format: str
    seed: int
    description: str
    topk: int = 0                 # > 0: token-sparse decode over topk cache positions per query
    prefill: bool = False         # sparse prefill: batch 1, s_q query tokens, one contiguous cache


WORKLOADS = {
    "tiny_b2_h16": Workload(
        "tiny_b2_h16", 2, 1, 16, "list:200,77", False, "bf16", 1,
        "tiny MLA decode: batch 2, s_q 1, h_q 16, cache_seqlens {200, 77}, non-causal"),
    "mem_b128_h16_L8192": Workload(
        "mem_b128_h16_L8192", 128, 1, 16, "fixed:8192", False, "bf16", 2,
        "memory-bound decode: batch 128, s_q 1, h_q 16, every cache_seqlen 8192"),
    "varlen_b128_h128": Workload(
        "varlen_b128_h128", 128, 1, 128, "uniform:1:16384", False, "bf16", 3,
        "variable-length decode: batch 128, s_q 1, h_q 128, cache_seqlens ~ U[1, 16384]"),
    "causal_b64_sq2_h128": Workload(
        "causal_b64_sq2_h128", 64, 2, 128, "normal:4096:1024:2:8192", True, "bf16", 4,
        "multi-token causal decode: batch 64, s_q 2, h_q 128, cache_seqlens ~ round(N(4096, 1024)) in [2, 8192]"),
    "fp8_b128_h128_L16384": Workload(
        "fp8_b128_h128_L16384", 128, 1, 128, "fixed:16384", False, "fp8", 5,
        "FP8 KV decode: batch 128, s_q 1, h_q 128, every cache_seqlen 16384, 656-byte tokens"),
    "sparse_b128_h128_L8192_topk2048": Workload(
        "sparse_b128_h128_L8192_topk2048", 128, 1, 128, "fixed:8192", False, "bf16", 6,
        "token-sparse decode: batch 128, s_q 1, h_q 128, every cache_seqlen 8192, 2048 distinct "
        "cache positions per query in random order", topk=2048),
    "sparse_prefill_s4096_h128_kv8192_topk2048": Workload(
        "sparse_prefill_s4096_h128_kv8192_topk2048", 1, 4096, 128, "fixed:8192", False, "bf16", 7,
        "sparse prefill: 4096 query tokens of 128 heads over one contiguous 8192-token cache, 2048 "
        "distinct listed positions per query token in random order", topk=2048, prefill=True),
}


def _seq(seed: int, stream: int, chunk: int = 0) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence(entropy=seed, spawn_key=(stream, chunk))))


def _threads() -> int:
    return max(1, min(32, os.cpu_count() or 1))


def _normal_f32(seed: int, stream: int, n: int) -> np.ndarray:
    """n standard normals (float32), chunked so every chunk has its own generator."""
    out = np.empty(n, dtype=np.float32)
    nchunks = (n + _CHUNK_ELEMS - 1) // _CHUNK_ELEMS

    def fill(i: int) -> None:
        lo = i * _CHUNK_ELEMS
        hi = min(n, lo + _CHUNK_ELEMS)
        _seq(seed, stream, i).standard_normal(hi - lo, dtype=np.float32, out=out[lo:hi])

    if nchunks <= 1:
        for i in range(nchunks):
            fill(i)
    else:
        with ThreadPoolExecutor(_threads()) as ex:
            list(ex.map(fill, range(nchunks)))
    return out


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16 (round-to-nearest-even) and return the bits."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float32 (a bit shift; no rounding)."""
    return (bits.astype(np.uint32) << 16).view(np.float32)


def draw_seqlens(spec: str, batch: int, seed: int) -> np.ndarray:
    kind, _, rest = spec.partition(":")
    if kind == "fixed":
        return np.full(batch, int(rest), dtype=np.int32)
    if kind == "list":
        vals = [int(v) for v in rest.split(",")]
        assert len(vals) == batch, (vals, batch)
        return np.asarray(vals, dtype=np.int32)
    g = _seq(seed, _S_SEQLENS)
    if kind == "uniform":
        lo, hi = (int(v) for v in rest.split(":"))
        return g.integers(lo, hi + 1, size=batch, dtype=np.int64).astype(np.int32)
    if kind == "normal":
        mu, sigma, lo, hi = (float(v) for v in rest.split(":"))
        x = np.rint(g.normal(mu, sigma, size=batch))
        return np.clip(x, lo, hi).astype(np.int32)
    raise ValueError(spec)


def make_block_table(cache_seqlens: np.ndarray, seed: int, spare_blocks: int = 0):
    """Deal a seeded random permutation of the physical pages out to the requests.

    Returns (block_table int32 [b, max_blocks] with -1 in unused entries, num_blocks).
    ``spare_blocks`` extra physical pages are allocated that no request references.
    """
    n_pages = [(int(L) + PAGE - 1) // PAGE for L in cache_seqlens]
    used = int(sum(n_pages))
    num_blocks = used + int(spare_blocks)
    perm = _seq(seed, _S_PERM).permutation(num_blocks).astype(np.int32)
    max_blocks = max(1, max(n_pages) if n_pages else 1)
    bt = np.full((len(n_pages), max_blocks), -1, dtype=np.int32)
    pos = 0
    for b, n in enumerate(n_pages):
        bt[b, :n] = perm[pos:pos + n]
        pos += n
    return bt, num_blocks


def _quantize_fp8_tokens(x_bits: np.ndarray) -> np.ndarray:
    """bf16 tokens [..., 576] -> 656-byte FP8 tokens [..., 656] (input construction only)."""
    import torch
    lead = x_bits.shape[:-1]
    xb = x_bits.reshape(-1, D_QK)
    ntok = xb.shape[0]
    out = np.empty((ntok, FP8_TOKEN_BYTES), dtype=np.uint8)
    latent = bf16_bits_to_f32(xb[:, :D_V]).reshape(ntok, D_V // FP8_GROUP, FP8_GROUP)
    amax = np.abs(latent).max(axis=2)                                   # f32 [ntok, 4]
    scale = (amax / np.float32(E4M3_MAX)).astype(np.float32)            # f32 division
    safe = np.where(scale > 0, scale, np.float32(1.0)).astype(np.float32)
    y = (latent / safe[:, :, None]).astype(np.float32)
    y = np.clip(y, -E4M3_MAX, E4M3_MAX)
    y = np.where(scale[:, :, None] > 0, y, np.float32(0.0)).astype(np.float32)
    codes = torch.from_numpy(np.ascontiguousarray(y)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    out[:, :D_V] = codes.reshape(ntok, D_V)
    out[:, D_V:D_V + 16] = np.ascontiguousarray(scale.astype("<f4")).view(np.uint8).reshape(ntok, 16)
    out[:, D_V + 16:] = np.ascontiguousarray(xb[:, D_V:].astype("<u2")).view(np.uint8).reshape(ntok, 2 * D_ROPE)
    return out.reshape(*lead, FP8_TOKEN_BYTES)


def _gen_kv(seed: int, num_blocks: int, kv_format: str) -> np.ndarray:
    n = num_blocks * PAGE * D_QK
    if kv_format == "bf16":
        vals = _normal_f32(seed, _S_KV, n)
        return f32_to_bf16_bits(vals).reshape(num_blocks, PAGE, D_QK)
    if kv_format == "fp8":
        out = np.empty((num_blocks, PAGE, FP8_TOKEN_BYTES), dtype=np.uint8)
        pages_per = 256
        nparts = (num_blocks + pages_per - 1) // pages_per
        # draw the same bf16 values the bf16 layout would hold, then quantise part by part
        vals = _normal_f32(seed, _S_KV, n).reshape(num_blocks, PAGE, D_QK)

        def work(i: int) -> None:
            lo, hi = i * pages_per, min(num_blocks, (i + 1) * pages_per)
            out[lo:hi] = _quantize_fp8_tokens(f32_to_bf16_bits(vals[lo:hi]))

        if nparts > 1:
            with ThreadPoolExecutor(_threads()) as ex:
                list(ex.map(work, range(nparts)))
        else:
            work(0)
        return out
    raise ValueError(kv_format)


def poison_unused(case: DecodeCase) -> None:
    """NaN-fill every cache slot no request may read: page tails past cache_seqlens
    and physical pages that the block table does not reference (in place)."""
    referenced = np.zeros(case.num_blocks, dtype=bool)
    for b in range(case.batch):
        L = int(case.cache_seqlens[b])
        n = (L + PAGE - 1) // PAGE
        pages = case.block_table[b, :n]
        referenced[pages] = True
        if n > 0 and L % PAGE:
            last = int(pages[n - 1])
            _poison_slots(case, last, L % PAGE, PAGE)
    for blk in np.nonzero(~referenced)[0]:
        _poison_slots(case, int(blk), 0, PAGE)


def _poison_slots(case: DecodeCase, blk: int, lo: int, hi: int) -> None:
    if case.kv_format == "bf16":
        case.kv[blk, lo:hi, :] = BF16_NAN
    else:
        case.kv[blk, lo:hi, :D_V] = E4M3_NAN
        nan_f32 = np.array([np.nan] * 4, dtype="<f4").view(np.uint8)
        case.kv[blk, lo:hi, D_V:D_V + 16] = nan_f32
        case.kv[blk, lo:hi, D_V + 16:] = np.frombuffer(np.array([0x7FC0] * D_ROPE, dtype="<u2").tobytes(), np.uint8)


def make_case(batch: int, s_q: int, h_q: int, cache_seqlens: Sequence[int] | np.ndarray, *,
              causal: bool = False, kv_format: str = "bf16", seed: int = 0,
              softmax_scale: Optional[float] = None, spare_blocks: int = 0,
              poison: bool = True, name: str = "") -> DecodeCase:
    """Build one seeded decode batch: q, kv ~ N(0,1) rounded to bf16 (then FP8-encoded
    for kv_format="fp8"), pages scattered by a seeded random block table."""
    seqlens = np.asarray(cache_seqlens, dtype=np.int32).reshape(batch)
    bt, num_blocks = make_block_table(seqlens, seed, spare_blocks)
    q = f32_to_bf16_bits(_normal_f32(seed, _S_Q, batch * s_q * h_q * D_QK)).reshape(batch, s_q, h_q, D_QK)
    kv = _gen_kv(seed, num_blocks, kv_format)
    case = DecodeCase(q_bits=q, kv=kv, block_table=bt, cache_seqlens=seqlens, s_q=s_q, h_q=h_q,
                      causal=causal, softmax_scale=float(softmax_scale if softmax_scale is not None else D_QK ** -0.5),
                      kv_format=kv_format, name=name)
    if poison:
        poison_unused(case)
    return case


def make_sparse_indices(cache_seqlens, s_q: int, topk: int, seed: int, *, invalid_frac: float = 0.0,
                        duplicate_frac: float = 0.0) -> np.ndarray:
    """Seeded index lists int32 [b, s_q, topk] for token-sparse decode.

    Each (request b, query i) lists min(topk, L_b) distinct cache positions of [0, L_b) in
    random order, then -1 for the remaining slots.  Optionally a fraction of the entries is
    replaced by an empty-slot value (-1, or a position >= L_b) and a fraction by a copy of
    another entry of the same list (a position counted twice)."""
    L = np.asarray(cache_seqlens, dtype=np.int64).reshape(-1)
    B = L.shape[0]
    g = _seq(seed, _S_IDX)
    out = np.full((B, s_q, topk), -1, dtype=np.int32)
    for b in range(B):
        for i in range(s_q):
            n = int(min(topk, max(L[b], 0)))
            if n > 0:
                out[b, i, :n] = g.permutation(int(L[b]))[:n]
            if invalid_frac > 0:
                m = g.random(topk) < invalid_frac
                bad = np.where(g.random(topk) < 0.5, -1, L[b] + g.integers(0, 1000, size=topk))
                out[b, i, m] = bad[m].astype(np.int32)
            if duplicate_frac > 0 and topk > 1:
                m = g.random(topk) < duplicate_frac
                src = g.integers(0, topk, size=topk)
                out[b, i, m] = out[b, i, src[m]]
    return out


def make_prefill_case(s_q: int, h_q: int, s_kv: int, topk: int, seed: int, *, invalid_frac: float = 0.0,
                      softmax_scale: Optional[float] = None, name: str = "") -> DecodeCase:
    """Sparse prefill inputs as a one-request case: s_q query tokens of h_q heads, one
    contiguous cache of s_kv tokens (pages in order: block_table = 0, 1, 2, ...; the prefill
    call reads kv = the first s_kv rows of case.kv), indices int32 [1, s_q, topk]."""
    n_pages = (int(s_kv) + PAGE - 1) // PAGE
    q = f32_to_bf16_bits(_normal_f32(seed, _S_Q, s_q * h_q * D_QK)).reshape(1, s_q, h_q, D_QK)
    kv = _gen_kv(seed, n_pages, "bf16")
    bt = np.arange(n_pages, dtype=np.int32).reshape(1, n_pages)
    sl = np.asarray([s_kv], dtype=np.int32)
    case = DecodeCase(q_bits=q, kv=kv, block_table=bt, cache_seqlens=sl, s_q=s_q, h_q=h_q, causal=False,
                      softmax_scale=float(softmax_scale if softmax_scale is not None else D_QK ** -0.5),
                      kv_format="bf16", name=name)
    case.indices = make_sparse_indices(sl, s_q, topk, seed, invalid_frac=invalid_frac)
    return case


def make_workload(name: str, *, batch: Optional[int] = None, poison: bool = True,
                  spare_blocks: int = 0) -> DecodeCase:
    """One of the named decode workloads at its full size (or with ``batch`` requests:
    the first ``batch`` of the full draw of cache lengths)."""
    w = WORKLOADS[name]
    if w.prefill:
        s_kv = int(w.seqlens.partition(":")[2])
        case = make_prefill_case(w.s_q, w.h_q, s_kv, w.topk, w.seed, name=name)
        case.meta["workload"] = w.description
        case.meta["prefill"] = True
        return case
    seqlens = draw_seqlens(w.seqlens, w.batch, w.seed)
    b = w.batch if batch is None else int(batch)
    if b != w.batch:
        seqlens = np.resize(seqlens, b).astype(np.int32)
    case = make_case(b, w.s_q, w.h_q, seqlens, causal=w.causal, kv_format=w.kv_format, seed=w.seed,
                     spare_blocks=spare_blocks, poison=poison, name=name)
    case.meta["workload"] = w.description
    if w.topk > 0:
        case.indices = make_sparse_indices(case.cache_seqlens, w.s_q, w.topk, w.seed)
    return case


def workload_units(case: DecodeCase) -> dict:
    """Algorithmic work of one decode pass: KV bytes at exact token counts (plus
    page-rounded), q/out/lse bytes and the FLOPs of the visible (row, key) pairs."""
    L = case.cache_seqlens.astype(np.int64)
    R = case.rows
    if case.indices is not None:
        # token-sparse: each query position attends to its valid listed positions; the cache
        # bytes are those of the distinct positions each request lists (read once at best)
        valid = (case.indices >= 0) & (case.indices < L[:, None, None])
        n_sel = int(valid.sum())
        distinct = sum(int(np.unique(case.indices[b][valid[b]]).size) for b in range(case.batch))
        kv_bytes = distinct * case.kv_bytes_per_token()
        qob = case.batch * R * (D_QK * 2 + D_V * 2 + 4) + case.indices.size * 4
        pairs = n_sel * case.h_q
        return {"kv_bytes": kv_bytes, "kv_bytes_paged": kv_bytes, "bytes": kv_bytes + qob,
                "qol_bytes": qob, "flops": 2 * (D_QK + D_V) * pairs, "pairs": pairs, "tokens": n_sel}
    kv_tok = int(L.sum())
    kv_bytes = kv_tok * case.kv_bytes_per_token()
    kv_bytes_paged = int(((L + PAGE - 1) // PAGE).sum()) * PAGE * case.kv_bytes_per_token()
    qob = case.batch * R * (D_QK * 2 + D_V * 2 + 4)
    if case.causal:
        pairs = 0
        for i in range(case.s_q):
            vis = np.clip(np.minimum(L, L - case.s_q + i + 1), 0, None)
            pairs += int(vis.sum()) * (case.h_q // case.h_kv)
        pairs *= case.h_kv
    else:
        pairs = kv_tok * R * case.h_kv
    flops = 2 * (D_QK + D_V) * pairs
    return {"kv_bytes": kv_bytes, "kv_bytes_paged": kv_bytes_paged, "bytes": kv_bytes + qob,
            "qol_bytes": qob, "flops": flops, "pairs": pairs, "tokens": kv_tok}


__all__ = [
    "D_QK", "D_V", "D_ROPE", "PAGE", "FP8_TOKEN_BYTES", "FP8_GROUP", "E4M3_MAX",
    "DecodeCase", "Workload", "WORKLOADS", "make_case", "make_workload", "make_block_table",
    "draw_seqlens", "poison_unused", "f32_to_bf16_bits", "bf16_bits_to_f32", "workload_units",
    "make_sparse_indices", "make_prefill_case",
]
