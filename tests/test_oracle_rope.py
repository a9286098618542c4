"""Pins for the oracle's RoPE front end and anchor position IDs.

The rotary map is checked against two independent formulations of the same
rotation (complex multiplication, and the rotate-half form applied to a
permuted vector), against its invariants (norm, group law, relative
positions), and phase 1 with anchor position IDs is checked against brute
force: the augmented block [anchor | block i] built token by token as the
pages describe it, with its position IDs, encoded by torch's causal SDPA.
"""

import numpy as np
import pytest
import torch

from oracle import star_oracle as so


def rope_complex(x, pos, base=so.ROPE_BASE):
    """The rotation as complex multiplication: (x_2k + i x_2k+1) * e^(i pos w_k)."""
    x = np.asarray(x, np.float64)
    D = x.shape[-1]
    w = float(base) ** (-np.arange(0, D, 2, dtype=np.float64) / D)
    z = (x[..., 0::2] + 1j * x[..., 1::2]) * np.exp(1j * np.outer(pos, w))
    out = np.empty_like(x)
    out[..., 0::2] = z.real
    out[..., 1::2] = z.imag
    return out


def rope_rotate_half(x, pos, base=so.ROPE_BASE):
    """The rotate-half form on the de-interleaved vector [x_0, x_2, .. | x_1, x_3, ..]."""
    x = np.asarray(x, np.float64)
    D = x.shape[-1]
    perm = np.concatenate([np.arange(0, D, 2), np.arange(1, D, 2)])
    xp = x[..., perm]
    w = float(base) ** (-np.arange(0, D, 2, dtype=np.float64) / D)
    ang = np.concatenate([np.outer(pos, w)] * 2, axis=-1)
    half = np.concatenate([-xp[..., D // 2:], xp[..., :D // 2]], axis=-1)
    yp = xp * np.cos(ang) + half * np.sin(ang)
    y = np.empty_like(x)
    y[..., perm] = yp
    return y


@pytest.mark.parametrize("D,base", [(2, 10000.0), (8, 500000.0), (128, 500000.0)])
def test_rope_matches_two_other_formulations(rng, D, base):
    x = rng.standard_normal((3, 17, D))
    pos = rng.integers(0, 1 << 20, size=17)
    y = so.rope(x, pos, base)
    np.testing.assert_allclose(y, rope_complex(x, pos, base), rtol=0, atol=1e-12)
    np.testing.assert_allclose(y, rope_rotate_half(x, pos, base), rtol=0, atol=1e-12)


def test_rope_invariants(rng):
    D = 64
    q = rng.standard_normal((5, D))
    k = rng.standard_normal((5, D))
    p = rng.integers(0, 100000, size=5)
    s = rng.integers(0, 100000, size=5)
    # norm preserved; position 0 is the identity; R(a) R(b) = R(a + b)
    np.testing.assert_allclose(np.linalg.norm(so.rope(q, p), axis=-1), np.linalg.norm(q, axis=-1), rtol=1e-12)
    np.testing.assert_allclose(so.rope(q, np.zeros(5, np.int64)), q, atol=0)
    np.testing.assert_allclose(so.rope(so.rope(q, p), s), so.rope(q, p + s), atol=1e-9)
    # scores depend on positions only through their difference
    d1 = (so.rope(q, p) * so.rope(k, s)).sum(-1)
    d2 = (so.rope(q, p + 777) * so.rope(k, s + 777)).sum(-1)
    np.testing.assert_allclose(d1, d2, atol=1e-9)


def test_rope_first_pair_turns_one_radian_per_position():
    # w_0 = base^0 = 1: the first pair of e_0 at position p is (cos p, sin p)
    x = np.zeros((1, 4))
    x[0, 0] = 1.0
    y = so.rope(x, np.array([3]))
    assert abs(y[0, 0] - np.cos(3.0)) < 1e-15 and abs(y[0, 1] - np.sin(3.0)) < 1e-15
    assert y[0, 2] == 0.0 and y[0, 3] == 0.0


def test_anchor_positions_follow_the_three_variants():
    ap = so.anchor_positions("first", 4, 8, 8)
    assert (ap == np.arange(8)).all() and ap.shape == (3, 8)
    ap = so.anchor_positions("previous", 4, 8, 8)      # b_a = b: the previous block's positions
    assert (ap[0] == np.arange(0, 8)).all() and (ap[2] == np.arange(16, 24)).all()
    ap = so.anchor_positions("previous", 3, 8, 3)      # b_a < b: the 3 positions before the block
    assert (ap[0] == [5, 6, 7]).all() and (ap[1] == [13, 14, 15]).all()


def brute_force_block(Q, K, V, b, b_a, scale, anchor_pos, i, base=so.ROPE_BASE):
    """Outputs of block i's own rows from the explicit augmented sequence:
    tokens [c_1[:b_a] | c_i] with position IDs [anchor_pos | own], rotated by
    the complex formulation, encoded by causal SDPA (float64)."""
    L = Q.shape[2]
    s, e = i * b, min((i + 1) * b, L)
    own = np.arange(s, e)
    if i == 0:
        idx, pos = own, own
    else:
        idx = np.concatenate([np.arange(b_a), own])
        pos = np.concatenate([np.asarray(anchor_pos[i - 1]), own])
    G = Q.shape[1] // K.shape[1]
    outs = []
    for h in range(Q.shape[1]):
        q = torch.tensor(rope_complex(Q[0, h][idx], pos, base))[None, None]
        k = torch.tensor(rope_complex(K[0, h // G][idx], pos, base))[None, None]
        v = torch.tensor(V[0, h // G][idx])[None, None]
        o = torch.nn.functional.scaled_dot_product_attention(q, k, v, is_causal=True, scale=scale)
        outs.append(o[0, 0, len(idx) - len(own):].numpy())
    return np.stack(outs)


@pytest.mark.parametrize("mode,L,b,b_a", [("first", 12, 4, 4), ("previous", 12, 4, 4),
                                          ("previous", 13, 5, 3), ("given", 12, 4, 4)])
def test_ctx_encode_rope_matches_the_augmented_sequence(rng, mode, L, b, b_a):
    D, Hq, Hkv, scale = 8, 4, 2, 0.37
    Q = rng.standard_normal((1, Hq, L, D))
    K = rng.standard_normal((1, Hkv, L, D))
    V = rng.standard_normal((1, Hkv, L, D))
    n = len(so.block_table(L, b))
    given = None
    if mode == "given":   # random IDs from [0, i*b), as in the position-ID ablation
        given = np.stack([np.sort(rng.choice(i * b, size=b_a, replace=False)) for i in range(1, n)])
    ap = so.anchor_positions(mode, n, b, b_a, given)
    O, _ = so.ctx_encode_rope(Q, K, V, b, b_a, scale, ap, base=10000.0)
    for i, (s, m) in enumerate(so.block_table(L, b)):
        ref = brute_force_block(Q, K, V, b, b_a, scale, ap, i, base=10000.0)
        np.testing.assert_allclose(O[0, :, s:s + m], ref, atol=1e-10)


def test_first_variant_is_star_phase1_on_rotated_inputs(rng):
    L, b, b_a, D = 20, 8, 5, 16
    Q = rng.standard_normal((2, 4, L, D))
    K = rng.standard_normal((2, 2, L, D))
    V = rng.standard_normal((2, 2, L, D))
    ap = so.anchor_positions("first", 3, b, b_a)
    O, S = so.ctx_encode_rope(Q, K, V, b, b_a, 0.25, ap)
    O2, S2 = so.ctx_encode(so.rope(Q, np.arange(L)), so.rope(K, np.arange(L)), V, b, b_a, 0.25)
    np.testing.assert_allclose(O, O2, atol=1e-12)
    np.testing.assert_allclose(S, S2, atol=1e-12)


def test_planted_position_mistake_is_caught(rng, monkeypatch):
    """An oracle that rotated the anchor at its own indices whatever the
    variant must fail the brute-force pin of the 'previous' variant."""
    good = so.ctx_encode_rope

    def ignores_anchor_ids(Q, K, V, b, b_a, scale, anchor_pos, base=so.ROPE_BASE, rows=None):
        first = np.broadcast_to(np.arange(b_a), np.asarray(anchor_pos).shape)
        return good(Q, K, V, b, b_a, scale, first, base, rows)

    monkeypatch.setattr(so, "ctx_encode_rope", ignores_anchor_ids)
    with pytest.raises(AssertionError):
        test_ctx_encode_rope_matches_the_augmented_sequence(rng, "previous", 12, 4, 4)


def test_round_bf16_is_round_to_nearest_even():
    x = np.array([1 + 2 ** -8, 1 + 2 ** -8 + 2 ** -20, 1 + 3 * 2 ** -8, -(2 + 2 ** -7), 3.0])
    np.testing.assert_array_equal(so.round_bf16(x), [1.0, 1 + 2 ** -7, 1 + 2 ** -6, -2.0, 3.0])
