"""Pins of the oracle's Tensor Cache (ring L1, outer-product L2 fed by
evictions, gated fusion), independent of the CUDA path.

- Per-token writes A <- lambda A + eta k (x) v over a chunk equal the
  weighted-sum form lambda^C A + eta sum_i lambda^(C-1-i) k_i (x) v_i (the
  page's parallel scan is defined as equal to the sequential writes).
- The read satisfies the linear-attention identity: q A =
  sum_i eta lambda^(age_i) <q, k_i> v_i over the evicted tokens.
- The ring keeps exactly the last W tokens; every token is in exactly one
  level; a gate of -inf (sigmoid 0) leaves torch's softmax attention over the
  last W tokens.
"""
import math

import numpy as np
import pytest
import torch

from oracle.tensor_cache import TensorCache


def _sdpa(q, k, v, scale):
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a, np.float64))
    return torch.nn.functional.scaled_dot_product_attention(
        t(q)[None, None], t(k)[None, None], t(v)[None, None], scale=scale)[0, 0].numpy()


def _run(O, d, B, Hkv, G, W, steps, seed, gate):
    P = O.Params(d, seed=0)
    rng = np.random.default_rng(seed)
    lam = rng.uniform(0.8, 0.99, Hkv)
    eta = rng.uniform(0.05, 0.5, Hkv)
    tc = TensorCache(P, B, Hkv, W, lam, eta, gate)
    K, V, res = [], [], []
    for s in range(steps):
        k = rng.standard_normal((B, Hkv, d))
        v = rng.standard_normal((B, Hkv, d))
        q = rng.standard_normal((B, G * Hkv, d))
        y, yl, m = tc.step(q, k, v, 1.0 / math.sqrt(d))
        K.append(np.float16(k).astype(np.float64))
        V.append(np.float16(v).astype(np.float64))
        res.append((q, y, yl, m))
    return P, tc, np.stack(K, 2), np.stack(V, 2), res, lam, eta


def test_chunk_weighted_sum_equals_sequential_writes(O):
    d, C = 16, 37
    P = O.Params(d, seed=0)
    rng = np.random.default_rng(1)
    A0 = rng.standard_normal((d, d))
    k, v = rng.standard_normal((C, d)), rng.standard_normal((C, d))
    lam, eta = 0.93, 0.2
    tc = TensorCache(P, 1, 1, 4, [lam], [eta], [0.0], A=A0[None, None])
    for i in range(C):
        tc.write(0, 0, k[i], v[i])
    closed = lam ** C * A0 + eta * sum(lam ** (C - 1 - i) * np.outer(k[i], v[i]) for i in range(C))
    assert np.abs(tc.A[0, 0] - closed).max() <= 1e-12 * np.abs(closed).max()


@pytest.mark.parametrize("G", [1, 4])
def test_ring_partition_and_linear_attention_identity(O, G):
    d, B, Hkv, W, steps = 32, 2, 2, 7, 20
    P, tc, K, V, res, lam, eta = _run(O, d, B, Hkv, G, W, steps, 5 + G, [0.3] * (G * Hkv))
    for s, (q, y, yl, m) in enumerate(res):
        total = s + 1
        n_ev = max(0, total - W)  # tokens in L2 during this step's read
        for b in range(B):
            for hq in range(G * Hkv):
                h = hq // G
                # q A = sum over evicted tokens of eta lambda^(age) <q, k_i> v_i
                ref = sum(eta[h] * lam[h] ** (n_ev - 1 - i) * (q[b, hq] @ K[b, h, i]) * V[b, h, i]
                          for i in range(n_ev)) if n_ev else np.zeros(d)
                assert np.abs(m[b, hq] - ref).max() <= 1e-10 * max(1.0, np.abs(ref).max())
                loc = _sdpa(q[b, hq][None], K[b, h, n_ev:total], V[b, h, n_ev:total],
                            1.0 / math.sqrt(d))[0]
                assert np.abs(yl[b, hq] - loc).max() <= 1e-10 * max(1.0, np.abs(loc).max())
                g = 1.0 / (1.0 + math.exp(-0.3))
                assert np.abs(y[b, hq] - (loc + g * ref)).max() <= 1e-9 * max(1.0, np.abs(loc).max())
    for b in range(B):
        for h in range(Hkv):
            ring = np.stack([kv[0] for kv in tc.ring[b][h]])
            assert np.array_equal(ring, K[b, h, steps - W:])


def test_shut_gate_is_local_attention(O):
    d, B, Hkv, G, W, steps = 16, 1, 1, 2, 5, 12
    P, tc, K, V, res, lam, eta = _run(O, d, B, Hkv, G, W, steps, 9, [-1e9] * G)
    for (q, y, yl, m) in res:
        assert np.array_equal(y, yl)
