"""End to end on the long-context workload (batch 4 x 131072 tokens, 128 heads, d_model 7168,
one layer): cache append and absorbed query in one call, split-KV attention, W_UV projection,
against the oracle's non-absorbed decode step on a seeded subset of heads.

At inputs x4 the logits spread ~16, and the bf16 rounding of the absorbed query alone would
move o_heads by up to ~1.5e-2 (relative L2); the query's remainder (q_lo) is carried from the
projection into the attention there.  At inputs x1 both forms are checked."""
import numpy as np
import pytest
import torch

from tests.gpu_common import Workload, assert_close, to_np

pytestmark = pytest.mark.gpu

N = 131072
HEADS_PER_SEQ = 4


def _heads(seed, b):
    rng = np.random.default_rng(seed * 100 + b)
    return sorted(rng.choice(128, HEADS_PER_SEQ, replace=False).tolist())


@pytest.mark.parametrize("scale,remainder", [(4.0, True), (1.0, True), (1.0, False)])
def test_long_context_end_to_end(scale, remainder):
    seed = 3
    wl = Workload(seed, 4, 128, 7168, [N - 1] * 4, scale=scale, with_w_o=False)
    got = wl.run_gpu(want_out=False, fused=True, query_remainder=remainder)
    assert got["status"] == 0
    for b in range(4):
        heads = _heads(seed, b)
        ref = wl.oracle(b, heads=heads, with_out=False)
        assert_close(to_np(got["o_heads"][b][heads]), ref["o_heads"], torch.bfloat16,
                     f"o_heads b={b} heads={heads} scale={scale}")
