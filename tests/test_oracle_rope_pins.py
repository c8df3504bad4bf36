"""Pins for the oracle's KV-append-with-RoPE rows (CPU).

Fixed by properties and closed forms, not by re-typing the formula: no
rotation at position 0 or without a base; unit vectors that fix the NeoX
pairing (dimension i rotates with i + d/2) and the direction of rotation; a
hand-computed frequency value; per-pair norm preservation; positions compose
additively; and the defining property of rotary embeddings: the dot product of
a rotated query and key depends only on their position difference.
"""
import math

import numpy as np
import pytest
import torch

from oracle import rope_append


def _rand(shape, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(shape, generator=g, dtype=torch.float64)


def test_values_are_copied_and_no_base_means_no_rotation():
    k, v = _rand((2, 3, 5, 8), 1), _rand((2, 3, 5, 8), 2)
    ko, vo = rope_append(k, v, start_pos=7, base=0.0)
    np.testing.assert_array_equal(ko, k.numpy())
    np.testing.assert_array_equal(vo, v.numpy())
    _, vo = rope_append(k, v, start_pos=7, base=10000.0)
    np.testing.assert_array_equal(vo, v.numpy())


def test_position_zero_is_the_identity():
    k = _rand((1, 2, 1, 16), 3)
    ko, _ = rope_append(k, k, start_pos=0, base=10000.0)
    np.testing.assert_allclose(ko, k.numpy(), rtol=0, atol=1e-15)


@pytest.mark.parametrize("p", [1, 3, 100])
def test_first_pair_rotates_with_the_middle_dimension(p):
    """Pair 0 has frequency 1 for every base: e_0 -> cos(p) e_0 + sin(p) e_{d/2}
    and e_{d/2} -> -sin(p) e_0 + cos(p) e_{d/2} (NeoX pairing, positive
    rotation); every other dimension stays zero."""
    d = 8
    k = torch.zeros((1, 1, 2, d), dtype=torch.float64)
    k[0, 0, 0, 0] = 1.0
    k[0, 0, 1, d // 2] = 1.0
    ko, _ = rope_append(k, k, start_pos=p, base=10000.0)
    e0 = np.zeros(d); e0[0], e0[d // 2] = math.cos(p), math.sin(p)
    eh = np.zeros(d); eh[0], eh[d // 2] = -math.sin(p + 1), math.cos(p + 1)
    np.testing.assert_allclose(ko[0, 0, 0], e0, rtol=0, atol=1e-14)
    np.testing.assert_allclose(ko[0, 0, 1], eh, rtol=0, atol=1e-14)


def test_second_pair_frequency_hand_computed():
    """base 16, d = 4: pair 1 has frequency 16^(-2/4) = 1/4, so position 4
    turns it by exactly one radian: cos 1 = 0.5403023058681398,
    sin 1 = 0.8414709848078965."""
    k = torch.zeros((1, 1, 1, 4), dtype=torch.float64)
    k[0, 0, 0, 1] = 1.0
    ko, _ = rope_append(k, k, start_pos=4, base=16.0)
    np.testing.assert_allclose(ko[0, 0, 0], [0.0, 0.5403023058681398, 0.0, 0.8414709848078965],
                               rtol=0, atol=1e-15)


def test_rotation_preserves_each_pair_norm():
    k = _rand((2, 2, 6, 16), 4)
    ko, _ = rope_append(k, k, start_pos=123, base=500.0)
    h = 8
    a = k.numpy()
    np.testing.assert_allclose(ko[..., :h] ** 2 + ko[..., h:] ** 2, a[..., :h] ** 2 + a[..., h:] ** 2,
                               rtol=1e-12)


def test_positions_compose():
    """Rotating by p1 and then by p2 equals rotating by p1 + p2."""
    k = _rand((1, 1, 1, 12), 5)
    once, _ = rope_append(k, k, start_pos=37, base=1000.0)
    twice, _ = rope_append(torch.from_numpy(once), k, start_pos=30, base=1000.0)
    direct, _ = rope_append(k, k, start_pos=67, base=1000.0)
    np.testing.assert_allclose(twice, direct, rtol=1e-12, atol=1e-12)


def test_scores_depend_only_on_the_position_difference():
    q, k = _rand((1, 1, 1, 16), 6), _rand((1, 1, 1, 16), 7)
    def score(pq, pk):
        rq, _ = rope_append(q, q, start_pos=pq, base=10000.0)
        rk, _ = rope_append(k, k, start_pos=pk, base=10000.0)
        return float(np.dot(rq.ravel(), rk.ravel()))
    assert score(50, 20) == pytest.approx(score(530, 500), rel=1e-10, abs=1e-12)
    assert score(3, 3) == pytest.approx(float(np.dot(q.numpy().ravel(), k.numpy().ravel())), rel=1e-12)


def test_each_new_token_uses_its_own_position():
    """Token t of a batch append sits at start_pos + t."""
    k = _rand((1, 1, 4, 8), 8)
    batch, _ = rope_append(k, k, start_pos=10, base=10000.0)
    for t in range(4):
        single, _ = rope_append(k[:, :, t:t + 1].contiguous(), k[:, :, t:t + 1].contiguous(),
                                start_pos=10 + t, base=10000.0)
        np.testing.assert_array_equal(batch[:, :, t], single[:, :, 0])


def test_odd_head_size_is_rejected():
    k = _rand((1, 1, 1, 5), 9)
    with pytest.raises(ValueError):
        rope_append(k, k, start_pos=0, base=10000.0)
