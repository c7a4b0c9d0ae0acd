"""Self-Indexing KV cache (sign-pattern vector quantisation as a token index,
LUT top-k selection, sparse attention over the selected tokens and the sink
tokens), on the CPU in fp64.

TEST INFRASTRUCTURE ONLY (see the package docstring): imported by ``tests/``,
never by the product path.  Plain numpy.

What it follows ("Self-Indexing KVCache", page 2 of the pages, section
"Methodologie: Self-Indexing KVCache", items 1-4):
  1. keys are cut into 4-dimensional subvectors; the signs of a subvector form
     a 4-bit index (0-15); a codebook of 16 centroids per group is built in
     one pass;
  2. before the signs are taken the channel mean is subtracted (softmax is
     invariant to it, since <q, mu> is the same for every token);
  3. top-k retrieval in the compressed domain: a table of the query against
     the 16 centroids of every group, token scores by table lookup and sum;
  4. token-wise codes; the first 64 tokens ("sinks") are kept at full
     precision and always attended.

Readings where the page leaves a step open:
  - Sign bit i of a group's index is 1 where coordinate 4g + i of k - mu is
    positive (zero counts as not positive).
  - The centroid of (group g, index p) is the mean of the centred subvectors
    of the tokens whose group g has index p; an index no token has gets the
    zero vector.
  - Selection is per query head, over the tokens after the sinks, by the LUT
    score (the score of the centred key's reconstruction); ties go to the
    lower position.
  - The sparse attention is exact softmax attention of the query over the
    sinks and the selected tokens with the stored (full-precision) keys and
    values, scale 1/sqrt(d) by default.
"""
import math

import numpy as np

N_SINK = 64


def build_index(K):
    """K [T, d] keys of one (batch, kv head).  Returns (mu [d], codes [T, d/4]
    uint8 sign patterns, centroids [d/4, 16, 4])."""
    K = np.asarray(K, np.float64)
    T, d = K.shape
    assert d % 4 == 0
    mu = K.mean(axis=0) if T else np.zeros(d)
    Kc = (K - mu).reshape(T, d // 4, 4)
    bits = (Kc > 0).astype(np.int64)
    codes = (bits * (1 << np.arange(4))).sum(axis=2).astype(np.uint8)  # [T, d/4]
    cent = np.zeros((d // 4, 16, 4))
    for g in range(d // 4):
        for p in range(16):
            sel = codes[:, g] == p
            if sel.any():
                cent[g, p] = Kc[sel, g].mean(axis=0)
    return mu, codes, cent


def lut_scores(q, codes, cent):
    """Score of every token: sum over groups of the table <q_g, c_{g, p}>."""
    q = np.asarray(q, np.float64)
    G4 = cent.shape[0]
    lut = np.einsum("gpi,gi->gp", cent, q.reshape(G4, 4))  # [d/4, 16]
    return lut[np.arange(G4)[None, :], codes.astype(np.int64)].sum(axis=1)


def select(scores, k, n_sink=N_SINK):
    """Positions of the k best scores after the sinks (ties to the lower
    position), in increasing position order."""
    T = len(scores)
    cand = np.arange(n_sink, T)
    if k >= len(cand):
        return cand
    order = np.lexsort((cand, -scores[cand]))  # score descending, position ascending
    return np.sort(cand[order[:k]])


def sparse_attention(q, K, V, picked, n_sink=N_SINK, scale=None):
    """Softmax attention of q over the sinks and the picked positions."""
    K = np.asarray(K, np.float64)
    V = np.asarray(V, np.float64)
    d = K.shape[1]
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    idx = np.concatenate([np.arange(min(n_sink, len(K))), np.asarray(picked, np.int64)])
    if len(idx) == 0:
        return np.zeros(d)
    s = (K[idx] @ np.asarray(q, np.float64)) * scale
    p = np.exp(s - s.max())
    return (p / p.sum()) @ V[idx]


def decode(q, K, V, k, n_sink=N_SINK, scale=None):
    """One query head: index, LUT scores, selection, sparse attention."""
    mu, codes, cent = build_index(K)
    sc = lut_scores(q, codes, cent)
    picked = select(sc, k, n_sink)
    return sparse_attention(q, K, V, picked, n_sink, scale), picked
