"""Pins of the oracle's FP8 token decode: a hand-worked token (tests/golden) and the
library's own float8_e4m3fn conversion for all 256 codes."""
import os
import struct

import numpy as np
import torch

import mla_inputs as mi
import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "fp8_token_example.txt")


def _load_golden():
    tok = np.zeros(656, dtype=np.uint8)
    expect = {}
    for line in open(GOLDEN):
        line = line.split("#")[0].strip()
        if not line:
            continue
        kind, a, b = line.split()
        if kind == "code":
            tok[int(a)] = int(b, 16)
        elif kind == "scale":
            tok[512 + 4 * int(a): 516 + 4 * int(a)] = np.frombuffer(struct.pack("<f", float(b)), np.uint8)
        elif kind == "rope":
            d = int(a) - 512
            tok[528 + 2 * d: 530 + 2 * d] = np.frombuffer(struct.pack("<H", int(b, 16)), np.uint8)
        elif kind == "expect":
            expect[int(a)] = float(b)
    return tok, expect


def test_hand_worked_token():
    tok, expect = _load_golden()
    vals = oracle.decode_fp8_tokens(tok[None])[0]
    for d, v in expect.items():
        assert vals[d] == v, (d, vals[d], v)


def test_e4m3_table_matches_library_conversion():
    table = oracle.e4m3_table()
    lib = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    nan_t, nan_l = np.isnan(table), np.isnan(lib)
    assert np.array_equal(nan_t, nan_l)
    assert np.array_equal(table[~nan_t], lib[~nan_l])
    assert nan_t.sum() == 2                         # 0x7f and 0xff


def test_generated_fp8_roundtrip_error_bound():
    """Quantised tokens decode to within half an e4m3 ulp (2^-4 relative) of the bf16
    values they were made from, and the group maximum maps to exactly +-448 * scale."""
    case_b = mi.make_case(1, 1, 1, [64], seed=3, poison=False)
    case_f = mi.make_case(1, 1, 1, [64], seed=3, poison=False, kv_format="fp8")
    x = mi.bf16_bits_to_f32(case_b.kv[0]).astype(np.float64)         # [64, 576]
    y = oracle.decode_fp8_tokens(case_f.kv[0])                        # [64, 576]
    assert np.array_equal(x[:, 512:], y[:, 512:])                    # RoPE stays bf16
    scales = np.ascontiguousarray(case_f.kv[0][:, 512:528]).view("<f4").astype(np.float64)
    for g in range(4):
        xs, ys = x[:, 128 * g:128 * (g + 1)], y[:, 128 * g:128 * (g + 1)]
        s = scales[:, g:g + 1]
        assert np.all(np.abs(xs - ys) <= 2.0 ** -4 * np.abs(xs) + s * 2.0 ** -10 + 1e-12)
