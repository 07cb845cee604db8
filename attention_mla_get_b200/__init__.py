"""MLA decode over a paged KV cache on NVIDIA B200 (sm_100a).

A thin ctypes binding of libmla (include/mla.h).  It only checks tensors, allocates
outputs / workspace through PyTorch and passes raw device pointers and the current CUDA
stream; every step of the computation runs in the library's CUDA kernels.  Importing the
package fails loudly when libmla.so has not been built: there is no fallback.

Calls (same names as the C-ABI):
    mla_num_sm_parts(rows_per_kv_head, h_kv=1, device=None)
    mla_get_metadata(cache_seqlens, rows_per_kv_head, h_kv=1, num_sm_parts=None)
        -> (tile_md int32 [num_sm_parts, 8], num_splits int32 [batch + 1])
    mla_workspace_size(batch, num_sm_parts, rows_per_kv_head, h_kv=1)
    mla_decode_kvcache(q, kvcache, block_table, cache_seqlens, d_v, tile_md, num_splits,
                       softmax_scale=None, causal=False, ...) -> (out bf16, lse fp32)
    mla_get_metadata_sparse(batch, s_q, topk, h_q, h_kv=1, num_sm_parts=None)
        -> (tile_md, num_splits int32 [batch * s_q + 1])        (token-sparse decode)
    mla_decode_kvcache_sparse(q, kvcache, block_table, cache_seqlens, indices, d_v, tile_md,
                              num_splits, softmax_scale=None) -> (out bf16, lse fp32)
    mla_read_status(workspace, reset=False)
    MLASession(batch, s_q, h_q, max_blocks, topk=0, kv_dtype=KV_BF16)     (mla_session_*)
        .decode(q_host, kvcache, block_table_host, cache_seqlens_host, out_host, lse_host,
                indices_host=None, softmax_scale=None, causal=False)    host buffers, pipelined
        .join(), .status(reset=False), .close()

The FlashMLA-style spellings of the usage examples on the pages are provided too:
get_mla_metadata(cache_seqlens, s_q * h_q // h_kv, h_kv) and
flash_mla_with_kvcache(q, kvcache, block_table, cache_seqlens, dv, tile_scheduler_metadata,
num_splits, causal=..., softmax_scale=...).
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmla.so")

D_QK = 576
D_V = 512
PAGE = 64
FP8_TOKEN_BYTES = 656
KV_BF16 = 0
KV_FP8 = 1

MLA_ERRORS = {
    -1: "MLA_ERR_NULL_POINTER", -2: "MLA_ERR_MISALIGNED", -3: "MLA_ERR_BAD_DIM", -4: "MLA_ERR_BAD_HEADS",
    -5: "MLA_ERR_BAD_KV_DTYPE", -6: "MLA_ERR_WORKSPACE", -7: "MLA_ERR_BAD_SHAPE", -8: "MLA_ERR_BAD_PARTS",
    -9: "MLA_ERR_NO_DEVICE", -10: "MLA_ERR_SCRATCH_LIMIT", -100: "MLA_ERR_CUDA",
}


class MLAError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {MLA_ERRORS.get(code, code)} ({mla_strerror(code)})")
        self.code = code


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is not built; run `python attention_mla_get_b200/build.py` "
                          "(there is no non-CUDA fallback)")
    lib = ctypes.CDLL(LIB_PATH)
    i32, i64, vp, sz = ctypes.c_int, ctypes.c_int64, ctypes.c_void_p, ctypes.c_size_t
    lib.mla_num_sm_parts.argtypes = [i32, i32, i32]
    lib.mla_num_sm_parts.restype = i32
    lib.mla_get_metadata.argtypes = [vp, i32, i32, i32, vp, i32, vp, vp]
    lib.mla_get_metadata.restype = i32
    lib.mla_workspace_size.argtypes = [i32, i32, i32, i32]
    lib.mla_workspace_size.restype = sz
    lib.mla_decode_kvcache.argtypes = [vp, vp, i64, vp, i32, vp, i32, i32, i32, i32, i32, vp, i32, vp,
                                       ctypes.c_float, i32, i32, vp, vp, vp, sz, vp]
    lib.mla_decode_kvcache.restype = i32
    lib.mla_get_metadata_sparse.argtypes = [i32, i32, i32, i32, i32, vp, i32, vp, vp]
    lib.mla_get_metadata_sparse.restype = i32
    lib.mla_decode_kvcache_sparse.argtypes = [vp, vp, i64, vp, i32, vp, i32, i32, i32, i32, i32, vp, i32, vp, i32,
                                              vp, ctypes.c_float, i32, vp, vp, vp, sz, vp]
    lib.mla_decode_kvcache_sparse.restype = i32
    lib.mla_sparse_prefill.argtypes = [vp, vp, i32, vp, i32, i32, i32, i32, i32, vp, i32, vp, ctypes.c_float, vp, vp,
                                       vp, sz, vp]
    lib.mla_sparse_prefill.restype = i32
    lib.mla_fault_injection_arm.argtypes = [ctypes.c_longlong, i32]
    lib.mla_fault_injection_arm.restype = i32
    lib.mla_read_status.argtypes = [vp, i32, ctypes.POINTER(i32), vp]
    lib.mla_read_status.restype = i32
    lib.mla_session_create.argtypes = [i32, i32, i32, i32, i32, i32, i32, i32, i32, ctypes.POINTER(vp)]
    lib.mla_session_create.restype = i32
    lib.mla_session_decode.argtypes = [vp, vp, vp, i64, vp, vp, vp, ctypes.c_float, i32, vp, vp, vp]
    lib.mla_session_decode.restype = i32
    lib.mla_session_join.argtypes = [vp, vp]
    lib.mla_session_join.restype = i32
    lib.mla_session_status.argtypes = [vp, i32, ctypes.POINTER(i32)]
    lib.mla_session_status.restype = i32
    lib.mla_session_destroy.argtypes = [vp]
    lib.mla_session_destroy.restype = i32
    lib.mla_strerror.argtypes = [i32]
    lib.mla_strerror.restype = ctypes.c_char_p
    lib.mla_version.argtypes = []
    lib.mla_version.restype = ctypes.c_char_p
    return lib


_lib = _load()

EXPORTED = ("mla_num_sm_parts", "mla_get_metadata", "mla_workspace_size", "mla_decode_kvcache",
            "mla_decode_kvcache_noalloc", "mla_noalloc_read_status", "mla_get_metadata_sparse", "mla_decode_kvcache_sparse", "mla_sparse_prefill",
            "mla_session_create", "mla_session_decode", "mla_session_join", "mla_session_status",
            "mla_session_destroy", "mla_read_status", "mla_fault_injection_arm", "mla_strerror", "mla_version")


def mla_strerror(code: int) -> str:
    return _lib.mla_strerror(int(code)).decode()


def mla_version() -> str:
    return _lib.mla_version().decode()


def _check(code: int, what: str) -> None:
    if code != 0:
        raise MLAError(code, what)


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _require(t, name: str, dtype, ndim: Optional[int] = None, shape=None) -> None:
    """dtype / rank / shape check of one tensor argument (before any device check, so that a
    wrong dtype is reported as such whatever the device)."""
    if not isinstance(t, torch.Tensor):
        raise ValueError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dimensions, got shape {tuple(t.shape)}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def _on_device(device, **tensors) -> None:
    """Every tensor argument is CUDA-resident on `device` and contiguous (the library reads
    raw row-major device memory)."""
    if device.type != "cuda":
        raise ValueError(f"{next(iter(tensors))} must be a CUDA tensor, got {device}")
    for name, t in tensors.items():
        if t is None:
            continue
        if not t.is_cuda or t.device != device:
            raise ValueError(f"{name} must be a CUDA tensor on {device}, got {t.device}")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")


def mla_num_sm_parts(rows_per_kv_head: int, h_kv: int = 1, device=None) -> int:
    dev = torch.cuda.current_device() if device is None else torch.device(device).index or 0
    n = _lib.mla_num_sm_parts(int(rows_per_kv_head), int(h_kv), int(dev))
    if n < 1:
        raise MLAError(n, "mla_num_sm_parts")
    return n


def mla_workspace_size(batch: int, num_sm_parts: int, rows_per_kv_head: int, h_kv: int = 1) -> int:
    return int(_lib.mla_workspace_size(int(batch), int(num_sm_parts), int(rows_per_kv_head), int(h_kv)))


def mla_get_metadata(cache_seqlens: torch.Tensor, rows_per_kv_head: int, h_kv: int = 1,
                     num_sm_parts: Optional[int] = None, stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Tile-scheduler metadata for one decode step (reusable by every layer)."""
    if cache_seqlens.dtype != torch.int32 or not cache_seqlens.is_cuda or cache_seqlens.dim() != 1:
        raise ValueError("cache_seqlens must be a 1-D int32 CUDA tensor")
    cache_seqlens = cache_seqlens.contiguous()
    batch = cache_seqlens.shape[0]
    if num_sm_parts is None:
        num_sm_parts = mla_num_sm_parts(rows_per_kv_head, h_kv, cache_seqlens.device)
    tile_md = torch.empty((num_sm_parts, 8), dtype=torch.int32, device=cache_seqlens.device)
    num_splits = torch.empty((batch + 1,), dtype=torch.int32, device=cache_seqlens.device)
    _check(_lib.mla_get_metadata(_ptr(cache_seqlens), batch, int(rows_per_kv_head), int(h_kv), _ptr(tile_md),
                                 int(num_sm_parts), _ptr(num_splits), _stream(stream)), "mla_get_metadata")
    return tile_md, num_splits


def mla_decode_kvcache(q: torch.Tensor, kvcache: torch.Tensor, block_table: torch.Tensor,
                       cache_seqlens: torch.Tensor, d_v: int, tile_md: torch.Tensor, num_splits: torch.Tensor,
                       softmax_scale: Optional[float] = None, causal: bool = False,
                       kv_dtype: Optional[int] = None, out: Optional[torch.Tensor] = None,
                       lse: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                       stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """MLA decode: returns (out bf16 [b, s_q, h_q, 512], lse fp32 [b, h_q, s_q])."""
    _require(q, "q", torch.bfloat16, 4)
    if q.shape[-1] != D_QK:
        raise ValueError("q must be bf16 [batch, s_q, h_q, 576]")
    b, s_q, h_q, _ = q.shape
    if kv_dtype is None:
        kv_dtype = KV_FP8 if kvcache.dtype == torch.uint8 else KV_BF16
    if kv_dtype == KV_BF16:
        if kvcache.dtype != torch.bfloat16 or kvcache.dim() not in (3, 4) or kvcache.shape[1] != PAGE or \
                kvcache.shape[-1] != D_QK:
            raise ValueError("bf16 kvcache must be [num_blocks, 64, (1,) 576]")
    elif kv_dtype == KV_FP8:
        if kvcache.dtype != torch.uint8 or kvcache.dim() not in (3, 4) or kvcache.shape[1] != PAGE or \
                kvcache.shape[-1] != FP8_TOKEN_BYTES:
            raise ValueError("fp8 kvcache must be uint8 [num_blocks, 64, (1,) 656]")
    else:
        raise ValueError("kv_dtype must be KV_BF16 or KV_FP8")
    h_kv = kvcache.shape[2] if kvcache.dim() == 4 else 1
    _require(block_table, "block_table", torch.int32, 2)
    if block_table.shape[0] != b:
        raise ValueError("block_table must be int32 [batch, max_blocks]")
    _require(cache_seqlens, "cache_seqlens", torch.int32, shape=(b,))
    _require(tile_md, "tile_md", torch.int32, 2)
    if tile_md.shape[1] != 8 or tile_md.shape[0] < 1:
        raise ValueError("tile_md must be int32 [num_sm_parts, 8] from mla_get_metadata")
    _require(num_splits, "num_splits", torch.int32, shape=(b + 1,))
    if out is not None:
        _require(out, "out", torch.bfloat16, shape=(b, s_q, h_q, D_V))
    if lse is not None:
        _require(lse, "lse", torch.float32, shape=(b, h_q, s_q))
    if workspace is not None:
        _require(workspace, "workspace", torch.uint8)
    q = q.contiguous() if q.is_cuda else q
    block_table = block_table.contiguous() if block_table.is_cuda else block_table
    _on_device(q.device, q=q, kvcache=kvcache, block_table=block_table, cache_seqlens=cache_seqlens,
               tile_md=tile_md, num_splits=num_splits, out=out, lse=lse, workspace=workspace)
    if softmax_scale is None:
        softmax_scale = D_QK ** -0.5
    rows = s_q * h_q // max(1, h_kv)
    num_sm_parts = tile_md.shape[0]
    if out is None:
        out = torch.empty((b, s_q, h_q, D_V), dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty((b, h_q, s_q), dtype=torch.float32, device=q.device)
    need = mla_workspace_size(b, num_sm_parts, rows, h_kv)
    if workspace is None:
        workspace = torch.zeros((max(need, 256),), dtype=torch.uint8, device=q.device)
    _check(_lib.mla_decode_kvcache(
        _ptr(q), _ptr(kvcache), kvcache.shape[0], _ptr(block_table), block_table.shape[1], _ptr(cache_seqlens),
        b, s_q, h_q, h_kv, int(d_v), _ptr(tile_md), num_sm_parts, _ptr(num_splits), float(softmax_scale),
        1 if causal else 0, int(kv_dtype), _ptr(out), _ptr(lse), _ptr(workspace), workspace.numel(),
        _stream(stream)), "mla_decode_kvcache")
    return out, lse


def mla_get_metadata_sparse(batch: int, s_q: int, topk: int, h_q: int, h_kv: int = 1,
                            num_sm_parts: Optional[int] = None, device=None,
                            stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Tile-scheduler metadata for token-sparse decode: batch * s_q query positions of topk
    listed tokens each -> (tile_md int32 [num_sm_parts, 8], num_splits int32 [batch * s_q + 1])."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    if num_sm_parts is None:
        num_sm_parts = mla_num_sm_parts(h_q, h_kv, dev)
    tile_md = torch.empty((num_sm_parts, 8), dtype=torch.int32, device=dev)
    num_splits = torch.empty((batch * s_q + 1,), dtype=torch.int32, device=dev)
    _check(_lib.mla_get_metadata_sparse(int(batch), int(s_q), int(topk), int(h_q), int(h_kv), _ptr(tile_md),
                                        int(num_sm_parts), _ptr(num_splits), _stream(stream)),
           "mla_get_metadata_sparse")
    return tile_md, num_splits


def mla_decode_kvcache_sparse(q: torch.Tensor, kvcache: torch.Tensor, block_table: torch.Tensor,
                              cache_seqlens: torch.Tensor, indices: torch.Tensor, d_v: int, tile_md: torch.Tensor,
                              num_splits: torch.Tensor, softmax_scale: Optional[float] = None,
                              out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                              workspace: Optional[torch.Tensor] = None,
                              stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Token-sparse MLA decode over indices int32 [b, s_q, topk] (bf16 cache):
    returns (out bf16 [b, s_q, h_q, 512], lse fp32 [b, h_q, s_q])."""
    _require(q, "q", torch.bfloat16, 4)
    if q.shape[-1] != D_QK:
        raise ValueError("q must be bf16 [batch, s_q, h_q, 576]")
    b, s_q, h_q, _ = q.shape
    if kvcache.dtype != torch.bfloat16 or kvcache.dim() not in (3, 4) or kvcache.shape[1] != PAGE or \
            kvcache.shape[-1] != D_QK:
        raise ValueError("kvcache must be bf16 [num_blocks, 64, (1,) 576] (token-sparse decode reads bf16 caches)")
    h_kv = kvcache.shape[2] if kvcache.dim() == 4 else 1
    _require(indices, "indices", torch.int32, 3)
    if tuple(indices.shape[:2]) != (b, s_q):
        raise ValueError("indices must be int32 [batch, s_q, topk]")
    _require(block_table, "block_table", torch.int32, 2)
    if block_table.shape[0] != b:
        raise ValueError("block_table must be int32 [batch, max_blocks]")
    _require(cache_seqlens, "cache_seqlens", torch.int32, shape=(b,))
    _require(tile_md, "tile_md", torch.int32, 2)
    if tile_md.shape[1] != 8 or tile_md.shape[0] < 1:
        raise ValueError("tile_md must be int32 [num_sm_parts, 8] from mla_get_metadata_sparse")
    _require(num_splits, "num_splits", torch.int32, shape=(b * s_q + 1,))
    if out is not None:
        _require(out, "out", torch.bfloat16, shape=(b, s_q, h_q, D_V))
    if lse is not None:
        _require(lse, "lse", torch.float32, shape=(b, h_q, s_q))
    if workspace is not None:
        _require(workspace, "workspace", torch.uint8)
    if q.is_cuda:
        q, indices, block_table = q.contiguous(), indices.contiguous(), block_table.contiguous()
    _on_device(q.device, q=q, kvcache=kvcache, block_table=block_table, cache_seqlens=cache_seqlens,
               indices=indices, tile_md=tile_md, num_splits=num_splits, out=out, lse=lse, workspace=workspace)
    topk = indices.shape[2]
    if softmax_scale is None:
        softmax_scale = D_QK ** -0.5
    num_sm_parts = tile_md.shape[0]
    if out is None:
        out = torch.empty((b, s_q, h_q, D_V), dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty((b, h_q, s_q), dtype=torch.float32, device=q.device)
    need = mla_workspace_size(b * s_q, num_sm_parts, h_q, h_kv)
    if workspace is None:
        workspace = torch.zeros((max(need, 256),), dtype=torch.uint8, device=q.device)
    _check(_lib.mla_decode_kvcache_sparse(
        _ptr(q), _ptr(kvcache), kvcache.shape[0], _ptr(block_table), block_table.shape[1], _ptr(cache_seqlens),
        b, s_q, h_q, h_kv, int(d_v), _ptr(indices), int(topk), _ptr(tile_md), num_sm_parts, _ptr(num_splits),
        float(softmax_scale), KV_BF16, _ptr(out), _ptr(lse), _ptr(workspace), workspace.numel(),
        _stream(stream)), "mla_decode_kvcache_sparse")
    return out, lse


def mla_sparse_prefill(q: torch.Tensor, kv: torch.Tensor, indices: torch.Tensor, softmax_scale: float,
                       d_v: int = D_V, tile_md: Optional[torch.Tensor] = None, num_splits: Optional[torch.Tensor] = None,
                       out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                       workspace: Optional[torch.Tensor] = None, stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Sparse prefill: q bf16 [s_q, h_q, 576], kv bf16 [s_kv, (1,) 576], indices int32 [s_q, (1,) topk]
    -> (out bf16 [s_q, h_q, 512], lse fp32 [h_q, s_q]).  Metadata is computed when not given."""
    _require(q, "q", torch.bfloat16, 3)
    if q.shape[-1] != D_QK:
        raise ValueError("q must be bf16 [s_q, h_q, 576]")
    s_q, h_q, _ = q.shape
    if kv.dtype != torch.bfloat16 or kv.shape[-1] != D_QK or not kv.is_contiguous():
        raise ValueError("kv must be contiguous bf16 [s_kv, (1,) 576]")
    s_kv = kv.shape[0]
    idx = indices.reshape(s_q, -1) if indices.dim() == 3 else indices
    _require(idx, "indices", torch.int32, 2)
    if idx.shape[0] != s_q:
        raise ValueError("indices must be int32 [s_q, (1,) topk]")
    topk = idx.shape[1]
    if (tile_md is None) != (num_splits is None):
        raise ValueError("pass tile_md and num_splits together (or neither)")
    if tile_md is not None:
        _require(tile_md, "tile_md", torch.int32, 2)
        if tile_md.shape[1] != 8 or tile_md.shape[0] < 1:
            raise ValueError("tile_md must be int32 [num_sm_parts, 8] from mla_get_metadata_sparse")
        _require(num_splits, "num_splits", torch.int32, shape=(s_q + 1,))
    if out is not None:
        _require(out, "out", torch.bfloat16, shape=(s_q, h_q, D_V))
    if lse is not None:
        _require(lse, "lse", torch.float32, shape=(h_q, s_q))
    if workspace is not None:
        _require(workspace, "workspace", torch.uint8)
    if q.is_cuda:
        q, idx = q.contiguous(), idx.contiguous()
    _on_device(q.device, q=q, kv=kv, indices=idx, tile_md=tile_md, num_splits=num_splits, out=out, lse=lse,
               workspace=workspace)
    if tile_md is None:
        tile_md, num_splits = mla_get_metadata_sparse(1, s_q, topk, h_q, 1, device=q.device, stream=stream)
    num_sm_parts = tile_md.shape[0]
    if out is None:
        out = torch.empty((s_q, h_q, D_V), dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty((h_q, s_q), dtype=torch.float32, device=q.device)
    need = mla_workspace_size(s_q, num_sm_parts, h_q, 1)
    if workspace is None:
        workspace = torch.zeros((max(need, 256),), dtype=torch.uint8, device=q.device)
    _check(_lib.mla_sparse_prefill(_ptr(q), _ptr(kv), int(s_kv), _ptr(idx), int(s_q), int(h_q), 1, int(d_v),
                                   int(topk), _ptr(tile_md), num_sm_parts, _ptr(num_splits), float(softmax_scale),
                                   _ptr(out), _ptr(lse), _ptr(workspace), workspace.numel(), _stream(stream)),
           "mla_sparse_prefill")
    return out, lse


def flash_mla_sparse_fwd(q, kv, indices, sm_scale, d_v=D_V):
    """The spelling of the sparse prefill call on the pages."""
    return mla_sparse_prefill(q, kv, indices, sm_scale, d_v=d_v)


def mla_fault_injection_arm(wait_limit_cycles: int, withhold_fill: int = -1) -> None:
    """Tests only: arm the next mla_decode_kvcache call with a shorter wait bound and a slot fill
    that its producer skips (see include/mla.h)."""
    _check(_lib.mla_fault_injection_arm(int(wait_limit_cycles), int(withhold_fill)), "mla_fault_injection_arm")


def mla_read_status(workspace: torch.Tensor, reset: bool = False, stream=None) -> int:
    v = ctypes.c_int(0)
    _check(_lib.mla_read_status(_ptr(workspace), 1 if reset else 0, ctypes.byref(v), _stream(stream)),
           "mla_read_status")
    return v.value


# FlashMLA-style spellings from the pages' usage examples
def get_mla_metadata(cache_seqlens: torch.Tensor, num_heads_per_head_k: int, num_heads_k: int):
    return mla_get_metadata(cache_seqlens, num_heads_per_head_k, num_heads_k)


def flash_mla_with_kvcache(q, k_cache, block_table, cache_seqlens, head_dim_v, tile_scheduler_metadata,
                           num_splits, softmax_scale=None, causal=False, is_fp8_kvcache=False):
    return mla_decode_kvcache(q, k_cache, block_table, cache_seqlens, head_dim_v, tile_scheduler_metadata,
                              num_splits, softmax_scale=softmax_scale, causal=causal,
                              kv_dtype=KV_FP8 if is_fp8_kvcache else None)


__all__ = [
    "mla_num_sm_parts", "mla_get_metadata", "mla_workspace_size", "mla_decode_kvcache", "mla_read_status",
    "mla_get_metadata_sparse", "mla_decode_kvcache_sparse", "mla_sparse_prefill", "flash_mla_sparse_fwd",
    "mla_strerror", "mla_version", "get_mla_metadata", "flash_mla_with_kvcache", "MLAError", "LIB_PATH",
    "KV_BF16", "KV_FP8",
]


class MLASession:
    """Decode steps with host (CPU, preferably pinned) inputs and outputs through the library's
    serving session (mla_session_* in include/mla.h): the copies of step k + 1's inputs and of
    step k - 1's outputs overlap step k on the GPU.  `decode` returns at once; call `join()`
    and synchronise the stream before reading the host outputs."""

    def __init__(self, batch: int, s_q: int, h_q: int, max_blocks: int, topk: int = 0, kv_dtype: int = KV_BF16,
                 h_kv: int = 1, num_sm_parts: Optional[int] = None, device=None):
        dev = torch.cuda.current_device() if device is None else torch.device(device).index
        if num_sm_parts is None:
            num_sm_parts = mla_num_sm_parts(h_q if topk > 0 else s_q * h_q, h_kv, dev)
        handle = ctypes.c_void_p()
        _check(_lib.mla_session_create(int(dev), int(batch), int(s_q), int(h_q), int(h_kv), int(max_blocks), int(topk),
                                       int(kv_dtype), int(num_sm_parts), ctypes.byref(handle)), "mla_session_create")
        self._h = handle
        self.batch, self.s_q, self.h_q, self.max_blocks, self.topk = batch, s_q, h_q, max_blocks, topk
        self.num_sm_parts = num_sm_parts

    @staticmethod
    def _host(t: torch.Tensor, dtype, numel: int, name: str) -> int:
        if t.is_cuda or t.dtype != dtype or not t.is_contiguous() or t.numel() != numel:
            raise ValueError(f"{name}: a contiguous host {dtype} tensor of {numel} elements is required")
        return t.data_ptr()

    def decode(self, q_host: torch.Tensor, kvcache: torch.Tensor, block_table_host: torch.Tensor,
               cache_seqlens_host: torch.Tensor, out_host: torch.Tensor, lse_host: torch.Tensor,
               indices_host: Optional[torch.Tensor] = None, softmax_scale: Optional[float] = None,
               causal: bool = False, stream=None) -> None:
        if self._h is None:
            raise RuntimeError("session closed")
        if not kvcache.is_cuda:
            raise ValueError("kvcache must be a device tensor")
        b, s_q, h_q = self.batch, self.s_q, self.h_q
        positions = b * s_q
        if softmax_scale is None:
            softmax_scale = D_QK ** -0.5
        num_blocks = kvcache.shape[0]
        qp = self._host(q_host, torch.bfloat16, positions * h_q * D_QK, "q_host")
        btp = self._host(block_table_host, torch.int32, b * self.max_blocks, "block_table_host")
        slp = self._host(cache_seqlens_host, torch.int32, b, "cache_seqlens_host")
        op = self._host(out_host, torch.bfloat16, positions * h_q * D_V, "out_host")
        lp = self._host(lse_host, torch.float32, positions * h_q, "lse_host")
        ip = None
        if self.topk > 0:
            if indices_host is None:
                raise ValueError("indices_host is required in a token-sparse session")
            ip = self._host(indices_host, torch.int32, positions * self.topk, "indices_host")
        _check(_lib.mla_session_decode(self._h, qp, _ptr(kvcache), int(num_blocks), btp, slp, ip, float(softmax_scale),
                                       1 if causal else 0, op, lp, _stream(stream)), "mla_session_decode")

    def join(self, stream=None) -> None:
        _check(_lib.mla_session_join(self._h, _stream(stream)), "mla_session_join")

    def status(self, reset: bool = False) -> int:
        v = ctypes.c_int(0)
        _check(_lib.mla_session_status(self._h, 1 if reset else 0, ctypes.byref(v)), "mla_session_status")
        return v.value

    def close(self) -> None:
        if self._h is not None:
            h, self._h = self._h, None
            _check(_lib.mla_session_destroy(h), "mla_session_destroy")

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
