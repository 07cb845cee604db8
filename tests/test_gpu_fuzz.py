"""Seeded random sweep of decode shapes against the fp64 oracle: query rows from 1 to 256 (every
tile size of the single-CTA kernel and one or two CTA-pair row groups), one to four query
positions with and without the causal mask, bf16 and FP8 caches, lengths that start, end and
straddle pages and 128-token steps (and empty requests), and scheduler part counts from one to
more than there are blocks.  Each case is small enough for the oracle to finish in a second or
two; the draw is fixed by the case number, so a failure names a reproducible shape."""
import numpy as np
import pytest

import mla_inputs as mi
import oracle
from tests._helpers import compare, run_gpu

pytestmark = pytest.mark.gpu

HEADS = [1, 3, 8, 16, 20, 32, 48, 64, 65, 96, 128]
PARTS = [None, 1, 2, 5, 13, 148]
EDGES = [0, 1, 63, 64, 65, 127, 128, 129, 255, 256, 257]


def draw(i: int):
    rng = np.random.default_rng(1000 + i)
    h_q = int(rng.choice(HEADS))
    s_q = int(rng.integers(1, 5)) if h_q <= 64 else int(rng.integers(1, 3))
    batch = int(rng.integers(1, 5))
    causal = bool(rng.integers(0, 2))
    fp8 = bool(rng.integers(0, 3) == 0)
    lens = []
    for _ in range(batch):
        if rng.integers(0, 3) == 0:
            lens.append(int(rng.choice(EDGES)) + 128 * int(rng.integers(0, 6)))
        else:
            lens.append(int(rng.integers(1, 1800)))
    parts = PARTS[int(rng.integers(0, len(PARTS)))]
    return batch, s_q, h_q, lens, causal, fp8, parts


@pytest.mark.parametrize("i", range(32))
def test_random_shape(cuda_ok, i):
    batch, s_q, h_q, lens, causal, fp8, parts = draw(i)
    case = mi.make_case(batch, s_q, h_q, lens, causal=causal, kv_format="fp8" if fp8 else "bf16",
                        seed=500 + i, spare_blocks=1)
    O_ref, L_ref = oracle.mla_decode_reference(case)
    out, lse, status, _ = run_gpu(case, num_sm_parts=parts)
    assert status == 0
    compare(case, out, lse, O_ref, L_ref)
