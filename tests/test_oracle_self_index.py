"""Pins of the oracle's Self-Indexing form (sign-pattern VQ index, LUT
scores, top-k selection, sparse attention over sinks + selected tokens),
independent of any CUDA code.

- Sign patterns against a hand-worked example.
- Centroids: each non-empty centroid's signs equal its pattern, and the
  count-weighted centroids of a group sum to the centred keys' sum (zero).
- LUT scores equal the dot products with the VQ reconstruction (a numpy
  matmul), so the table is exactly the compressed-domain score.
- Centring does not change attention (softmax invariance), checked against
  torch's scaled_dot_product_attention.
- Selecting every post-sink token reduces the sparse attention to full
  attention (SDPA); selection ties go to the lower position.
- Selection equals the first k of a brute-force sort of (-score, position)
  tuples; sparse attention equals SDPA with a boolean mask over sinks +
  picked.
"""
import math

import numpy as np
import torch

from oracle import self_index as S


def _sdpa(q, k, v, scale):
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a, np.float64))
    return torch.nn.functional.scaled_dot_product_attention(
        t(q)[None, None], t(k)[None, None], t(v)[None, None], scale=scale)[0, 0].numpy()


def test_sign_patterns_hand_worked():
    # two tokens, d = 8; mean (0.5, -0.5, ...) subtracted first
    K = np.array([[1.0, -2.0, 3.0, 0.5, 0.0, 1.0, -1.0, 2.0],
                  [0.0, 1.0, -3.0, 0.5, 2.0, -1.0, 1.0, -2.0]])
    mu, codes, cent = S.build_index(K)
    assert np.allclose(mu, K.mean(0))
    # centred: token 0 = (0.5, -1.5, 3, 0 | -1, 1, -1, 2); token 1 = negatives
    # token 0 group 0: bits (1, 0, 1, 0) -> 1 + 4 = 5; group 1: (0, 1, 0, 1) -> 10
    # token 1 group 0: (0, 1, 0, 0) -> 2; group 1: (1, 0, 1, 0) -> 5
    assert codes.tolist() == [[5, 10], [2, 5]]
    assert np.allclose(cent[0, 5], [0.5, -1.5, 3.0, 0.0])
    assert not cent[0, 0].any()  # an index no token has


def test_centroid_signs_and_balance():
    rng = np.random.default_rng(0)
    T, d = 500, 32
    K = rng.standard_normal((T, d)) * rng.uniform(0.5, 3, d) + rng.standard_normal(d)
    mu, codes, cent = S.build_index(K)
    for g in range(d // 4):
        counts = np.bincount(codes[:, g], minlength=16)
        total = (counts[:, None] * cent[g]).sum(axis=0)
        assert np.abs(total).max() < 1e-9 * T  # centred keys sum to zero
        for p in range(16):
            if counts[p]:
                signs = (cent[g, p] > 0).astype(int)
                assert (signs * (1 << np.arange(4))).sum() == p


def test_lut_scores_equal_reconstruction_dot():
    rng = np.random.default_rng(1)
    T, d = 300, 64
    K = rng.standard_normal((T, d))
    q = rng.standard_normal(d)
    mu, codes, cent = S.build_index(K)
    recon = cent[np.arange(d // 4)[None, :], codes.astype(int)].reshape(T, d)
    assert np.abs(S.lut_scores(q, codes, cent) - recon @ q).max() < 1e-12


def test_centring_does_not_change_attention():
    rng = np.random.default_rng(2)
    T, d = 200, 32
    K, V = rng.standard_normal((T, d)) + 3.0, rng.standard_normal((T, d))
    q = rng.standard_normal(d)
    sc = 1.0 / math.sqrt(d)
    a = _sdpa(q[None], K, V, sc)[0]
    b = _sdpa(q[None], K - K.mean(0), V, sc)[0]
    assert np.abs(a - b).max() < 1e-12


def test_full_selection_is_full_attention_and_ties():
    rng = np.random.default_rng(3)
    T, d = 150, 16
    K, V = rng.standard_normal((T, d)), rng.standard_normal((T, d))
    q = rng.standard_normal(d)
    out, picked = S.decode(q, K, V, k=T)
    assert np.array_equal(picked, np.arange(S.N_SINK, T))
    assert np.abs(out - _sdpa(q[None], K, V, 1.0 / math.sqrt(d))[0]).max() < 1e-12
    # ties: equal scores keep the lower positions
    sc = np.zeros(T)
    sc[100] = sc[120] = sc[70] = 5.0
    assert S.select(sc, 2).tolist() == [70, 100]
    # only sinks when nothing else is picked
    out0 = S.sparse_attention(q, K, V, [])
    ref0 = _sdpa(q[None], K[:S.N_SINK], V[:S.N_SINK], 1.0 / math.sqrt(d))[0]
    assert np.abs(out0 - ref0).max() < 1e-12


def test_select_against_brute_force_order():
    # the k best of (-score, position) tuples by Python's sort, on integer
    # scores so that ties are common
    rng = np.random.default_rng(4)
    for trial in range(40):
        T = int(rng.integers(0, 300))
        n_sink = int(rng.choice([0, 5, 64]))
        k = int(rng.integers(1, 320))
        sc = rng.integers(-4, 5, T).astype(np.float64)
        ranked = sorted(range(n_sink, T), key=lambda t: (-sc[t], t))
        assert S.select(sc, k, n_sink).tolist() == sorted(ranked[:k])


def test_sparse_attention_equals_masked_sdpa():
    rng = np.random.default_rng(5)
    T, d = 400, 32
    K, V = rng.standard_normal((T, d)), rng.standard_normal((T, d))
    q = rng.standard_normal(d)
    picked = np.sort(rng.choice(np.arange(S.N_SINK, T), 37, replace=False))
    keep = np.zeros(T, bool)
    keep[:S.N_SINK] = True
    keep[picked] = True
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a, np.float64))
    ref = torch.nn.functional.scaled_dot_product_attention(
        t(q)[None, None, None], t(K)[None, None], t(V)[None, None],
        attn_mask=torch.from_numpy(keep)[None, None, None], scale=0.3)[0, 0, 0].numpy()
    assert np.abs(S.sparse_attention(q, K, V, picked, scale=0.3) - ref).max() < 1e-12
