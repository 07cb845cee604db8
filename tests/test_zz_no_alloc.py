"""mla_decode_kvcache_noalloc through the C-ABI: the decode call for callers that cannot
allocate device memory (its workspace is a 16 MiB array inside libmla).  Its output must
match the regular entry point's, within the tolerances of the other GPU tests, on two calls
in a row (the second call reuses the array the first one left behind), and the fp64 oracle
within the same tolerances; its device status word, read back with mla_noalloc_read_status,
must be clear after each call; a problem whose workspace exceeds the array is rejected
before anything runs.

This file is collected last on purpose: it runs after every other test, and it also runs
alone in a fresh process."""
import ctypes
import os

import numpy as np
import pytest
import torch

import mla_inputs as mi
import oracle

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SO = os.path.join(ROOT, "attention_mla_get_b200", "libmla.so")
MLA_ERR_SCRATCH_LIMIT = -10


def _lib():
    L = ctypes.CDLL(SO)
    vp, i32, i64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64
    L.mla_decode_kvcache_noalloc.argtypes = [vp, vp, i64, vp, i32, vp, i32, i32, i32, i32, i32, vp, i32, vp,
                                             ctypes.c_float, i32, i32, vp, vp, vp]
    L.mla_decode_kvcache_noalloc.restype = i32
    L.mla_noalloc_read_status.argtypes = [i32, ctypes.POINTER(i32), vp]
    L.mla_noalloc_read_status.restype = i32
    return L


def _status(L):
    v = ctypes.c_int(-1)
    assert L.mla_noalloc_read_status(0, ctypes.byref(v), torch.cuda.current_stream().cuda_stream) == 0
    return v.value


def _noalloc(L, case, q, kv, bt, sl, md, ns, out, lse):
    stream = torch.cuda.current_stream().cuda_stream
    return L.mla_decode_kvcache_noalloc(q.data_ptr(), kv.data_ptr(), kv.shape[0], bt.data_ptr(), bt.shape[1],
                                        sl.data_ptr(), case.batch, case.s_q, case.h_q, 1, 512, md.data_ptr(),
                                        md.shape[0], ns.data_ptr(), case.softmax_scale, int(case.causal), 0,
                                        out.data_ptr(), lse.data_ptr(), stream)


def _device(case):
    q = torch.from_numpy(case.q_bits.view(np.int16)).view(torch.bfloat16).cuda()
    kv = torch.from_numpy(case.kv.view(np.int16)).view(torch.bfloat16).reshape(case.num_blocks, 64, 1, 576).cuda()
    return q, kv, torch.from_numpy(case.block_table).cuda(), torch.from_numpy(case.cache_seqlens).cuda()


def test_noalloc_matches_regular_entry_point_twice(cuda_ok):
    import attention_mla_get_b200 as mla
    L = _lib()
    # lengths chosen so that requests are split over several SM parts (partials in the scratch)
    for seed, seqlens in ((41, [1000, 5000, 77, 3000]), (42, [6000, 129, 4097, 2])):
        case = mi.make_case(len(seqlens), 1, 16, seqlens, seed=seed)
        q, kv, bt, sl = _device(case)
        md, ns = mla.mla_get_metadata(sl, case.rows, 1)
        assert int((ns[1:] - ns[:-1]).max()) > 1
        ref_out, ref_lse = mla.mla_decode_kvcache(q, kv, bt, sl, 512, md, ns, softmax_scale=case.softmax_scale)
        ref_o = ref_out.float().cpu().numpy()
        ref_l = ref_lse.cpu().numpy()
        o64, l64 = oracle.mla_decode_reference(case)
        for _ in range(2):
            out = torch.full_like(ref_out, float("nan"))
            lse = torch.full_like(ref_lse, float("nan"))
            assert _noalloc(L, case, q, kv, bt, sl, md, ns, out, lse) == 0
            torch.cuda.synchronize()
            assert _status(L) == 0
            o, l = out.float().cpu().numpy(), lse.cpu().numpy()
            assert np.isfinite(o).all() and np.isfinite(l).all()
            assert np.all(np.abs(o - ref_o) <= 5e-3 + 1e-2 * np.abs(ref_o))
            assert np.abs(l - ref_l).max() <= 1e-3
            # and directly against the fp64 oracle
            assert np.all(np.abs(o - o64) <= 5e-3 + 1e-2 * np.abs(o64))
            assert np.abs(l - l64).max() <= 1e-3


def test_noalloc_rejects_problems_larger_than_its_scratch(cuda_ok):
    import attention_mla_get_b200 as mla
    L = _lib()
    case = mi.make_case(128, 1, 128, [64] * 128, seed=43)      # workspace > 16 MiB
    assert mla.mla_workspace_size(case.batch, 74, case.rows, 1) > 16 << 20
    q, kv, bt, sl = _device(case)
    md, ns = mla.mla_get_metadata(sl, case.rows, 1)
    out = torch.empty((case.batch, 1, 128, 512), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((case.batch, 128, 1), dtype=torch.float32, device="cuda")
    assert _noalloc(L, case, q, kv, bt, sl, md, ns, out, lse) == MLA_ERR_SCRATCH_LIMIT
