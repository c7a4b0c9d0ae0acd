"""Tensor Cache's two-level decode state, step by step, on top of the CPU
oracle.

TEST INFRASTRUCTURE ONLY (see the package docstring): imported by ``tests/``,
never by the product path.  Plain numpy in fp64 plus the oracle's attention.

What it follows ("Tensor Cache: Eviction-conditioned Associative Memory for
Transformers", gist.science, section "Methodik: Tensor Cache (TC)"):
  - L1 is a ring buffer holding the last W tokens, read with exact softmax
    attention;
  - L2 is a fixed-size outer-product matrix A written only by evictions: when
    the ring overwrites an entry, the evicted pair enters as
    A <- lambda A + eta (k (x) v), lambda and eta per head;
  - a query reads r = q A, and the outputs are fused as
    y = y_local + sigmoid(g) r with a per-head gate g.

Readings where the page leaves a step open:
  - Heads: A, lambda and eta belong to the kv head whose keys and values are
    evicted; the query heads sharing that kv head read the same A; g is per
    query head.
  - Order within a step: the step's token enters the ring, which evicts the
    oldest token into A when the ring is full; then the query attends to the
    ring (the new token included) and reads A (the just-evicted token
    included), so every token is in exactly one of the two levels.
  - The evicted k, v are the ring's fp16 values; the read uses q unscaled
    (q A as written); y_local is the oracle's softmax attention over the ring
    with the usual 1/sqrt(d) scale.

Parity status: pinned by ``tests/test_oracle_tensor_cache.py`` (the chunked
weighted-sum form equals per-token writes; the linear-attention identity
q (k (x) v) = <q, k> v; a shut gate reduces to softmax attention over the
last W tokens).
"""
import math

import numpy as np

from . import attention


def sigmoid(x):
    if x >= 0:
        return 1.0 / (1.0 + math.exp(-x))
    e = math.exp(x)  # no overflow for large negative x
    return e / (1.0 + e)


class TensorCache:
    def __init__(self, params, B, Hkv, W, lam, eta, gate, A=None):
        self.P = params
        self.B, self.Hkv, self.d, self.W = B, Hkv, params.d, int(W)
        self.lam = np.asarray(lam, np.float64)
        self.eta = np.asarray(eta, np.float64)
        self.gate = np.asarray(gate, np.float64)
        self.A = (np.zeros((B, Hkv, self.d, self.d)) if A is None
                  else np.array(A, np.float64, copy=True))
        self.ring = [[[] for _ in range(Hkv)] for _ in range(B)]  # (k, v) oldest first

    def write(self, b, h, k, v):
        """One eviction: A <- lambda A + eta k (x) v."""
        self.A[b, h] = self.lam[h] * self.A[b, h] + self.eta[h] * np.outer(k, v)

    def append(self, k_new, v_new):
        f16 = lambda a: np.float16(a).astype(np.float64)
        for b in range(self.B):
            for h in range(self.Hkv):
                r = self.ring[b][h]
                if len(r) == self.W:
                    k_old, v_old = r.pop(0)
                    self.write(b, h, k_old, v_old)
                r.append((f16(k_new[b, h]), f16(v_new[b, h])))

    def read(self, q):
        """r = q A for every query head ([B, Hq, d])."""
        G = q.shape[1] // self.Hkv
        r = np.empty(q.shape)
        for b in range(self.B):
            for hq in range(q.shape[1]):
                r[b, hq] = q[b, hq] @ self.A[b, hq // G]
        return r

    def local(self, q, scale):
        n = np.array([len(self.ring[b][0]) for b in range(self.B)], np.int32)
        Wd = max(1, int(n.max()))
        k = np.zeros((self.B, self.Hkv, Wd, self.d))
        v = np.zeros((self.B, self.Hkv, Wd, self.d))
        for b in range(self.B):
            for h in range(self.Hkv):
                for t, (kr, vr) in enumerate(self.ring[b][h]):
                    k[b, h, t], v[b, h, t] = kr, vr
        out, _ = attention(self.P, q, self.Hkv, scale, k, v, n, None, 16,
                           np.zeros((self.B, self.Hkv, 1), np.int32), np.zeros(self.B, np.int32))
        return out.reshape(q.shape)

    def step(self, q, k_new, v_new, scale):
        self.append(k_new, v_new)
        y_local = self.local(q, scale)
        m = self.read(q)
        g = np.array([sigmoid(x) for x in self.gate])
        return y_local + g[None, :, None] * m, y_local, m
