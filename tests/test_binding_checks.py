"""The Python binding rejects malformed tensor arguments before anything reaches the library:
a wrong dtype, rank or length of cache_seqlens, tile_md and num_splits (an int64 cache_seqlens
would otherwise be read as the wrong lengths), and host tensors where device memory is needed.
These checks run on the host, without a GPU."""
import pytest
import torch

import attention_mla_get_b200 as mla

B, S_Q, H_Q, NB, MB, P = 3, 1, 16, 8, 4, 5


def _args(**over):
    a = dict(q=torch.zeros((B, S_Q, H_Q, 576), dtype=torch.bfloat16),
             kvcache=torch.zeros((NB, 64, 1, 576), dtype=torch.bfloat16),
             block_table=torch.zeros((B, MB), dtype=torch.int32),
             cache_seqlens=torch.ones((B,), dtype=torch.int32),
             d_v=512,
             tile_md=torch.zeros((P, 8), dtype=torch.int32),
             num_splits=torch.zeros((B + 1,), dtype=torch.int32))
    a.update(over)
    return a


@pytest.mark.parametrize("name,bad,msg", [
    ("cache_seqlens", torch.ones((B,), dtype=torch.int64), "cache_seqlens must be torch.int32"),
    ("cache_seqlens", torch.ones((B + 1,), dtype=torch.int32), "cache_seqlens must have shape"),
    ("tile_md", torch.zeros((P, 8), dtype=torch.int64), "tile_md must be torch.int32"),
    ("tile_md", torch.zeros((P, 4), dtype=torch.int32), "tile_md must be int32 [num_sm_parts, 8]"),
    ("tile_md", torch.zeros((P * 8,), dtype=torch.int32), "tile_md must have 2 dimensions"),
    ("num_splits", torch.zeros((B + 1,), dtype=torch.int64), "num_splits must be torch.int32"),
    ("num_splits", torch.zeros((B,), dtype=torch.int32), "num_splits must have shape"),
    ("block_table", torch.zeros((B, MB), dtype=torch.int64), "block_table must be torch.int32"),
    ("q", torch.zeros((B, S_Q, H_Q, 576), dtype=torch.float16), "q must be torch.bfloat16"),
])
def test_dense_decode_rejects_bad_tensors(name, bad, msg):
    with pytest.raises(ValueError) as e:
        mla.mla_decode_kvcache(**_args(**{name: bad}))
    assert msg in str(e.value)


def test_dense_decode_rejects_bad_outputs():
    with pytest.raises(ValueError, match="out must have shape"):
        mla.mla_decode_kvcache(**_args(), out=torch.zeros((B, S_Q, H_Q, 256), dtype=torch.bfloat16))
    with pytest.raises(ValueError, match="lse must be torch.float32"):
        mla.mla_decode_kvcache(**_args(), lse=torch.zeros((B, H_Q, S_Q), dtype=torch.float64))


def test_dense_decode_rejects_host_tensors():
    # every dtype and shape right, but nothing is in device memory
    with pytest.raises(ValueError, match="must be a CUDA tensor"):
        mla.mla_decode_kvcache(**_args())


@pytest.mark.parametrize("name,bad,msg", [
    ("cache_seqlens", torch.ones((B,), dtype=torch.int64), "cache_seqlens must be torch.int32"),
    ("tile_md", torch.zeros((P, 8), dtype=torch.int64), "tile_md must be torch.int32"),
    ("num_splits", torch.zeros((B + 1,), dtype=torch.int32), "num_splits must have shape"),  # needs b*s_q + 1
    ("indices", torch.zeros((B, 2, 64), dtype=torch.int64), "indices must be torch.int32"),
])
def test_sparse_decode_rejects_bad_tensors(name, bad, msg):
    a = _args(q=torch.zeros((B, 2, H_Q, 576), dtype=torch.bfloat16),
              num_splits=torch.zeros((B * 2 + 1,), dtype=torch.int32),
              indices=torch.zeros((B, 2, 64), dtype=torch.int32))
    a[name] = bad
    with pytest.raises(ValueError) as e:
        mla.mla_decode_kvcache_sparse(a["q"], a["kvcache"], a["block_table"], a["cache_seqlens"], a["indices"], 512,
                                      a["tile_md"], a["num_splits"])
    assert msg in str(e.value)


def test_sparse_prefill_rejects_bad_tensors():
    q = torch.zeros((8, H_Q, 576), dtype=torch.bfloat16)
    kv = torch.zeros((100, 1, 576), dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="indices must be torch.int32"):
        mla.mla_sparse_prefill(q, kv, torch.zeros((8, 32), dtype=torch.int64), 0.04)
    with pytest.raises(ValueError, match="num_splits must have shape"):
        mla.mla_sparse_prefill(q, kv, torch.zeros((8, 32), dtype=torch.int32), 0.04,
                               tile_md=torch.zeros((P, 8), dtype=torch.int32),
                               num_splits=torch.zeros((3,), dtype=torch.int32))
    with pytest.raises(ValueError, match="must be a CUDA tensor"):
        mla.mla_sparse_prefill(q, kv, torch.zeros((8, 32), dtype=torch.int32), 0.04)
