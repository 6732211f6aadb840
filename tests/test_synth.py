"""Host-side checks of the seeded input generators (CPU only)."""
import numpy as np
import torch

from cascade_token_head_b200 import synth


def test_bf16_rounding_matches_torch():
    g = np.random.default_rng(0)
    x = np.concatenate([g.standard_normal(10000) * 10.0 ** g.uniform(-30, 30, 10000),
                        [0.0, -0.0, 1.0, 1.00390625, 1.01171875, 65504.0, 3.0e38]])
    want = torch.tensor(x, dtype=torch.float64).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(synth.to_bf16_f64(x), want)


def test_draws_are_deterministic_and_shaped():
    w = synth.scaled_prefill(synth.bert_base_prefill(), B=2, T=64, L=2, token_keep=[64, 58],
                             head_keep=[12, 12])
    a, b = synth.draw_prefill(w), synth.draw_prefill(w)
    assert a["X"].shape == (2, 64, 768) and a["w_qkv"][1].shape == (768, 3 * 768)
    np.testing.assert_array_equal(a["X"], b["X"])
    np.testing.assert_array_equal(a["key_gain"], b["key_gain"])
    assert (a["key_gain"] == 4.0).sum(axis=1).tolist() == [26, 26]


def test_span_boost_is_contiguous_and_disjoint():
    w = synth.scaled_prefill(synth.long_prefill(), D=64, L=1, token_keep=[16384], head_keep=[32])
    g = synth.draw_prefill(w)["key_gain"][0]
    assert (g == 4.0).sum() == 8 * 41
    edges = np.flatnonzero(np.diff(np.concatenate([[0], (g == 4.0).astype(int), [0]])))
    assert len(edges) == 16 and np.all(edges[1::2] - edges[0::2] == 41)


def test_topk_rows_have_exact_duplicates():
    x = synth.draw_topk_row_block(4, 4096, "lognormal", 0.01, seed=3)
    assert x.dtype == np.float32
    for r in range(4):
        assert len(np.unique(x[r])) <= 4096 - 30
