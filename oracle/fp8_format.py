"""Oracle (test infrastructure): decode of the FP8 KV token layout, in fp64.

Layout (wmrh.cn page, "FP8 KV缓存内存效率" table: NoPE part 512 bytes float8_e4m3,
scale factors 16 bytes float32, RoPE part 128 bytes bfloat16): one token is 656
bytes, in that order.  Scale g (little-endian float32 at byte 512 + 4g) multiplies
latent dims 128g .. 128g+127.  The RoPE dims are stored as bf16 and used as they are.

float8_e4m3 ("fn" flavour, as used for KV caches): bit 7 sign, bits 6..3 exponent
with bias 7, bits 2..0 mantissa.  Exponent field 0 is subnormal (m/8 * 2^-6); the
single pattern with exponent 15 and mantissa 7 is NaN; there is no infinity.
Every finite code is exactly representable in fp64, and the oracle multiplies
code * scale in fp64, so it reads the stored bytes exactly.
"""
from __future__ import annotations

import math

import numpy as np

D_QK, D_V, FP8_TOKEN_BYTES, GROUP = 576, 512, 656, 128


def e4m3_table() -> np.ndarray:
    """float64 value of every e4m3 byte 0..255, from the bit-field definition."""
    out = np.empty(256, dtype=np.float64)
    for code in range(256):
        sign = -1.0 if code & 0x80 else 1.0
        exp = (code >> 3) & 0xF
        man = code & 0x7
        if exp == 0xF and man == 0x7:
            out[code] = math.nan
        elif exp == 0:
            out[code] = sign * (man / 8.0) * 2.0 ** (1 - 7)
        else:
            out[code] = sign * (1.0 + man / 8.0) * 2.0 ** (exp - 7)
    return out


_TABLE = None


def decode_fp8_tokens(tok: np.ndarray) -> np.ndarray:
    """uint8 [..., 656] tokens -> float64 [..., 576] (latent * scale, then RoPE)."""
    global _TABLE
    if _TABLE is None:
        _TABLE = e4m3_table()
    tok = np.asarray(tok, dtype=np.uint8)
    lead = tok.shape[:-1]
    t = tok.reshape(-1, FP8_TOKEN_BYTES)
    codes = _TABLE[t[:, :D_V]]                                              # [n, 512]
    scales = np.ascontiguousarray(t[:, D_V:D_V + 16]).view("<f4").astype(np.float64)  # [n, 4]
    latent = codes.reshape(-1, D_V // GROUP, GROUP) * scales[:, :, None]
    rope_bits = np.ascontiguousarray(t[:, D_V + 16:]).view("<u2")
    rope = (rope_bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    out = np.concatenate([latent.reshape(-1, D_V), rope], axis=1)
    return out.reshape(*lead, D_QK)
