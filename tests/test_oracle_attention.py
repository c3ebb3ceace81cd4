"""Pins of oracle.attention: a library routine (torch SDPA in fp64), closed forms, invariants."""
import math

import numpy as np
import pytest
import torch

from oracle.attention import attend, bf16_to_f64, softmax_weights
from oracle.sets import full_set, local_set


def _rand(rng, *shape):
    return rng.standard_normal(shape)


def _sdpa(q, K, V, S):
    """torch scaled_dot_product_attention over rows S, GQA by repeating KV heads."""
    Hq, d = q.shape
    t, Hkv, _ = K.shape
    g = Hq // Hkv
    mask = torch.zeros(1, 1, 1, t, dtype=torch.bool)
    mask[..., [p - 1 for p in S]] = True
    qt = torch.from_numpy(q)[None, :, None, :]
    Kt = torch.from_numpy(K).permute(1, 0, 2).repeat_interleave(g, dim=0)[None]
    Vt = torch.from_numpy(V).permute(1, 0, 2).repeat_interleave(g, dim=0)[None]
    o = torch.nn.functional.scaled_dot_product_attention(qt, Kt, Vt, attn_mask=mask)
    return o[0, :, 0, :].numpy()


@pytest.mark.parametrize("t,s,w,Hq,Hkv", [(37, 2, 8, 4, 2), (64, 4, 16, 8, 2), (5, 4, 2048, 4, 4),
                                          (300, 4, 128, 8, 8), (1, 4, 2048, 2, 1)])
def test_matches_torch_sdpa(t, s, w, Hq, Hkv):
    rng = np.random.default_rng(t * 7 + Hq)
    d = 16
    q, K, V = _rand(rng, Hq, d), _rand(rng, t, Hkv, d), _rand(rng, t, Hkv, d)
    for S in (local_set(t, s, w), full_set(t)):
        o = attend(q, K, V, S)
        ref = _sdpa(q, K, V, S)
        assert np.max(np.abs(o - ref)) < 1e-12


def test_zero_query_gives_mean_of_values():
    rng = np.random.default_rng(1)
    t, Hkv, d = 50, 2, 8
    K, V = _rand(rng, t, Hkv, d), _rand(rng, t, Hkv, d)
    S = local_set(t, 3, 10)
    o = attend(np.zeros((4, d)), K, V, S)
    rows = [p - 1 for p in sorted(S)]
    for h in range(4):
        assert np.allclose(o[h], V[rows, h // 2].mean(axis=0), atol=1e-14)


def test_single_position_returns_its_value():
    rng = np.random.default_rng(2)
    K, V = _rand(rng, 9, 1, 8), _rand(rng, 9, 1, 8)
    o = attend(_rand(rng, 2, 8), K, V, {4})
    assert np.array_equal(o[0], V[3, 0]) and np.array_equal(o[1], V[3, 0])


def test_dominant_key_selects_its_value():
    rng = np.random.default_rng(3)
    t, d = 20, 8
    K, V = _rand(rng, t, 1, d), _rand(rng, t, 1, d)
    K[7, 0] = 0.0
    K[7, 0, 0] = 1.0
    q = np.zeros((1, d))
    q[0, 0] = 1e4 * math.sqrt(d)
    K[:, 0, 0][np.arange(t) != 7] = -1.0
    o = attend(q, K, V, full_set(t))
    assert np.allclose(o[0], V[7, 0], atol=1e-12)


def test_weights_sum_to_one_and_scale():
    rng = np.random.default_rng(4)
    s = rng.standard_normal(1000) * 30
    w = softmax_weights(s)
    assert abs(w.sum() - 1.0) < 1e-12 and (w >= 0).all()
    # scores are divided by sqrt(d_k): doubling d (with q, k scaled so q.k is fixed) changes o
    q = np.ones((1, 4))
    K = np.zeros((2, 1, 4))
    K[0, 0, 0] = 2.0
    V = np.array([[[1.0, 0, 0, 0]], [[0.0, 0, 0, 0]]])
    o = attend(q, K, V, {1, 2})
    p = 1.0 / (1.0 + math.exp(-2.0 / 2.0))  # q.k / sqrt(4) = 1
    assert abs(o[0, 0] - p) < 1e-15


def test_position_permutation_invariance():
    rng = np.random.default_rng(5)
    t, Hkv, d = 30, 2, 8
    q, K, V = _rand(rng, 4, d), _rand(rng, t, Hkv, d), _rand(rng, t, Hkv, d)
    perm = rng.permutation(t)
    inv = np.argsort(perm)
    S = {1, 3, 5, 8, 13, 21, 30}
    o1 = attend(q, K, V, S)
    o2 = attend(q, K[perm], V[perm], {int(inv[p - 1]) + 1 for p in S})
    assert np.allclose(o1, o2, atol=1e-14)


def test_bf16_decode_exact():
    bits = np.array([0x3F80, 0xC000, 0x0001, 0x7F80, 0x0000, 0x8000, 0x3FC0], dtype=np.uint16)
    v = bf16_to_f64(bits)
    assert v[0] == 1.0 and v[1] == -2.0 and v[2] == 2.0 ** -133 and math.isinf(v[3])
    assert v[4] == 0.0 and v[5] == 0.0 and math.copysign(1, v[5]) < 0 and v[6] == 1.5
    x = torch.tensor([0.1, -3.3, 1e-20, 65504.0], dtype=torch.float32).to(torch.bfloat16)
    assert np.array_equal(bf16_to_f64(x.view(torch.int16).numpy().view(np.uint16)),
                          x.to(torch.float64).numpy())
