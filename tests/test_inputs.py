"""The seeded input generator: determinism, bf16 rounding, sink/positional structure."""
import numpy as np
import torch

from block_sparse_cross_sparvar_b200 import inputs


def test_bf16_rounding_matches_torch():
    x = np.random.default_rng(0).standard_normal(100000).astype(np.float32) * 7
    x[:4] = [0.0, -0.0, 1.00390625, 1.01171875]  # includes exact ties
    bits, vals = inputs.bf16_round(x)
    ref = torch.from_numpy(x).to(torch.bfloat16)
    assert np.array_equal(bits, ref.view(torch.int16).numpy().view(np.uint16))
    assert np.array_equal(vals, ref.float().numpy())


def test_seeded_and_shaped():
    a = inputs.make_qkv(3, 1, 2, inputs.TINY_SIDES, 64, 2, pe=False)
    b = inputs.make_qkv(3, 1, 2, inputs.TINY_SIDES, 64, 2, pe=False)
    assert a["q"].shape == (1, 2, 341, 64)
    assert np.array_equal(a["k"], b["k"])
    c = inputs.make_qkv(4, 1, 2, inputs.TINY_SIDES, 64, 2, pe=False)
    assert not np.array_equal(a["k"], c["k"])


def test_sink_tokens_share_a_vector():
    d = inputs.make_qkv(0, 2, 2, inputs.TINY_SIDES, 64, 2, pe=False, sink_amp=30.0)
    # the first 5 tokens (scales 1x1 and 2x2) share a large common component per head
    k = d["kf"]
    sink_mean = k[:, :, :5].mean(axis=2)
    rest_mean = k[:, :, 5:].mean(axis=2)
    assert np.abs(sink_mean).mean() > 10 * np.abs(rest_mean).mean()
    assert np.allclose(sink_mean[0], sink_mean[1], atol=3.0)


def test_positional_component_makes_neighbours_closer():
    t = inputs.positional_table(inputs.INFINITY_SIDES, 128)
    off = inputs.token_offsets(inputs.INFINITY_SIDES)
    last = t[off[-2]:off[-1]]
    g = last @ last.T
    # a token's own position scores highest, a distant one lower
    assert g[0, 0] > g[0, 1] > g[0, 63 * 64 + 63]
