"""Workload shapes, the rank rule and the byte accounting (CPU only)."""
import json
import os

import pytest

from binary_rank_linear_lb_b200.configs import (LLAMA2_13B, LLAMA2_70B, LLAMA2_7B, linear_bytes,
                                                 rank_for, stored_model_bytes)

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")

# Ranks worked out by hand from r = floor(bpw*in*out / (2*(in+out)) / 64) * 64.
RANKS = {
    (4096, 4096): (1024, 512, 256, 64),
    (4096, 11008): (1472, 768, 384, 128),
    (5120, 5120): (1280, 704, 384, 128),
    (5120, 13824): (1856, 1024, 512, 128),
    (8192, 8192): (2048, 1088, 576, 192),
    (8192, 1024): (448, 192, 128, 0),
    (8192, 28672): (3136, 1728, 896, 256),
}


@pytest.mark.parametrize("shape", sorted(RANKS))
def test_rank_rule(shape):
    for bpw, r in zip((1.0, 0.55, 0.3, 0.1), RANKS[shape]):
        assert rank_for(bpw, *shape) == r
        assert rank_for(bpw, shape[1], shape[0]) == r


def test_bytes_per_token():
    mb = lambda m, b: m.bytes_per_token(b) / 1e6
    assert mb(LLAMA2_13B, 0.55) == pytest.approx(886.9, rel=2e-3)
    assert mb(LLAMA2_13B, 0.1) == pytest.approx(141.0, rel=2e-3)
    assert mb(LLAMA2_70B, 1.0) == pytest.approx(8500, rel=2e-3)
    assert mb(LLAMA2_70B, 0.55) == pytest.approx(4660, rel=2e-3)
    assert linear_bytes(512, 256, 32) == 2 * 32 * 768 // 8 + 2 * 2 * (512 + 256 + 32)


def fp16_params(m, vocab=32000):
    per_layer = sum(i * o for i, o in m.shapes())
    return m.n_layers * per_layer + 2 * vocab * m.hidden


def test_format_sizes_close_to_pages_table3():
    """Loose check only: our ranks round down to 64, so sizes come out 5-7% low."""
    t3 = json.load(open(os.path.join(GOLDEN, "table3_sizes.json")))
    assert 2 * fp16_params(LLAMA2_13B) / 1e9 == pytest.approx(t3["llama2-13b"]["fp16"], rel=0.01)
    assert 2 * fp16_params(LLAMA2_7B) / 1e9 == pytest.approx(t3["llama2-7b"]["fp16"], rel=0.01)
    for m, key, bpw in ((LLAMA2_13B, "llama2-13b", 0.1), (LLAMA2_7B, "llama2-7b", 0.3),
                        (LLAMA2_7B, "llama2-7b", 0.1)):
        ours = stored_model_bytes(m, bpw) / 1e9
        page = t3[key][str(bpw)]
        assert 0.90 * page < ours <= page, (key, bpw, ours, page)
