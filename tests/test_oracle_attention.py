"""Pins of the oracle's decode attention and top-k search.

Zero-residual reduction: records written directly with gamma = 0 describe
keys K_t = n Pi^T c_hat_t and values V_t = n_v Pi^T c_hat_v,t exactly, so the
compressed attention must equal textbook softmax attention over those K, V
(torch's scaled_dot_product_attention in fp64 on the CPU) and the compressed
search must return the exact inner-product top-k."""
import math

import numpy as np
import pytest
import torch


def _direct_records(rng, N, d, m, gamma_zero=True):
    f16 = lambda a: np.float16(a).astype(np.float64)
    return dict(sign=rng.integers(0, 2, (N, d)).astype(np.int32),
                mag=rng.integers(0, 2, (N, d)).astype(np.int32),
                qbits=rng.integers(0, 2, (N, m)).astype(np.int32),
                n=f16(rng.uniform(2.0, 14.0, N)),
                gamma=np.zeros(N) if gamma_zero else f16(rng.uniform(0.0, 0.4, N)),
                vcode=rng.integers(0, 16, (N, d)).astype(np.int32),
                vn=f16(rng.uniform(2.0, 14.0, N)))


def _reconstruct(P, rec):
    kh = np.where(rec["sign"] == 1, -1.0, 1.0) * P.kc[rec["mag"]]
    vh = np.where(rec["vcode"] >> 3, -1.0, 1.0) * P.vc[rec["vcode"] & 7]
    return rec["n"][:, None] * (kh @ P.pi32), rec["vn"][:, None] * (vh @ P.pi32)


def _sdpa(q, k, v, scale):
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a, np.float64))
    return torch.nn.functional.scaled_dot_product_attention(
        t(q)[None, None], t(k)[None, None], t(v)[None, None], scale=scale)[0, 0].numpy()


@pytest.mark.parametrize("d,G,cold,hot", [(64, 1, 256, 0), (64, 8, 300, 50), (128, 4, 517, 33),
                                          (128, 4, 0, 40), (64, 2, 129, 0)])
def test_zero_residual_equals_exact_attention(O, d, G, cold, hot):
    m = d
    P = O.Params(d, seed=12)
    rng = np.random.default_rng(d + G + cold)
    B, Hkv = 2, 2
    Hq = G * Hkv
    max_pages = max(1, math.ceil(cold / 128)) + 1
    nbytes, _ = O.page_layout(d, m, True)
    n_pages = B * Hkv * max_pages
    pool = rng.integers(0, 256, size=n_pages * nbytes, dtype=np.uint8)  # garbage in unused slots
    table = rng.permutation(n_pages).astype(np.int32).reshape(B, Hkv, max_pages)
    W = max(hot, 1)
    k_hot = np.float16(rng.standard_normal((B, Hkv, W, d))).astype(np.float64)
    v_hot = np.float16(rng.standard_normal((B, Hkv, W, d))).astype(np.float64)
    q = rng.standard_normal((B, Hq, d))
    cold_len = np.array([cold, max(cold - 77, 0)], np.int32)
    hot_len = np.array([hot, max(hot - 9, 0)], np.int32)
    recs = {}
    for b in range(B):
        for h in range(Hkv):
            n = int(cold_len[b])
            rec = _direct_records(rng, n, d, m)
            t = np.arange(n)
            O.pack(pool, nbytes, d, m, True, table[b, h, t // 128], t % 128, rec)
            recs[b, h] = rec
    scale = 1.0 / math.sqrt(d)
    out, groups = O.attention(P, q, Hkv, scale, k_hot, v_hot, hot_len, pool, nbytes, table, cold_len)
    for gi, (b, h) in enumerate(groups):
        K, V = _reconstruct(P, recs[b, h])
        K = np.concatenate([K, k_hot[b, h, :hot_len[b]]])
        V = np.concatenate([V, v_hot[b, h, :hot_len[b]]])
        for g in range(G):
            qh = q[b, h * G + g][None]
            if len(K) == 0:
                ref = np.zeros(d)
            else:
                ref = _sdpa(qh, K, V, scale)[0]
            assert np.abs(out[gi, g] - ref).max() <= 1e-10 * max(1.0, np.abs(ref).max())


def test_gqa_grouping_uses_own_kv_head(O):
    """q heads h*G..h*G+G-1 read kv head h: permuting kv heads permutes outputs."""
    d = m = 64
    P = O.Params(d, seed=1)
    rng = np.random.default_rng(0)
    B, Hkv, G = 1, 3, 2
    nbytes, _ = O.page_layout(d, m, True)
    pool = np.zeros(Hkv * nbytes, np.uint8)
    table = np.arange(Hkv, dtype=np.int32).reshape(1, Hkv, 1)
    for h in range(Hkv):
        rec = _direct_records(rng, 100, d, m, gamma_zero=False)
        O.pack(pool, nbytes, d, m, True, np.full(100, h), np.arange(100), rec)
    q = np.repeat(rng.standard_normal((1, 1, d)), Hkv * G, axis=1)
    out, _ = O.attention(P, q, Hkv, 0.125, None, None, None, pool, nbytes, table, np.array([100]))
    table2 = table[:, ::-1].copy()
    out2, _ = O.attention(P, q, Hkv, 0.125, None, None, None, pool, nbytes, table2, np.array([100]))
    assert np.allclose(out2, out[::-1]) and not np.allclose(out[0], out[1])


def test_qjl_term_reduces_score_error(O):
    """With the stored residual sketch, estimated scores are closer on average
    to the exact <q, k> than the quantised key alone (1-bit correction)."""
    d = 128
    P = O.Params(d, seed=3)
    rng = np.random.default_rng(4)
    x = rng.standard_normal((4000, d))
    q = rng.standard_normal(d)
    rec = O.encode(P, x, True)
    chat = np.where(rec["sign"] == 1, -1.0, 1.0) * P.kc[rec["mag"]]
    qrot = P.pi32 @ q
    base = rec["n"] * (chat @ qrot)
    sq = P.S @ qrot
    corr = rec["n"] * P.alpha * rec["gamma"] * ((1 - 2 * rec["qbits"]) @ sq)
    exact = x @ q
    err0 = base - exact
    err1 = base + corr - exact
    # the correction is unbiased: its mean error is no larger than 3 standard errors
    assert abs(err1.mean()) < 3 * err1.std() / math.sqrt(len(err1))
    # and it removes the part of the error correlated with the residual direction
    assert np.corrcoef(corr, -err0)[0, 1] > 0.5


def test_topk_zero_residual_is_exact_inner_product_topk(O):
    d = m = 64
    P = O.Params(d, seed=21)
    rng = np.random.default_rng(22)
    N, k = 1000, 10
    nbytes, _ = O.page_layout(d, m, False)
    pool = np.zeros(math.ceil(N / 128) * nbytes, np.uint8)
    rec = _direct_records(rng, N, d, m)
    ids = np.arange(N)
    O.pack(pool, nbytes, d, m, False, ids // 128, ids % 128,
           {key: rec[key] for key in ("sign", "mag", "qbits", "n", "gamma")})
    K, _ = _reconstruct(P, rec)
    Q = rng.standard_normal((7, d))
    got_ids, got_sc = O.topk(P, Q, pool, nbytes, N, k)
    exact = Q @ K.T
    for i in range(len(Q)):
        order = np.lexsort((np.arange(N), -exact[i]))[:k]
        assert np.array_equal(got_ids[i], order)
        assert np.allclose(got_sc[i], exact[i, order], rtol=1e-12, atol=1e-12)


def test_topk_ties_go_to_lower_id(O):
    d = m = 64
    P = O.Params(d, seed=5)
    rng = np.random.default_rng(6)
    nbytes, _ = O.page_layout(d, m, False)
    base = _direct_records(rng, 1, d, m, gamma_zero=False)
    N = 40
    rec = {key: np.repeat(base[key], N, axis=0) for key in ("sign", "mag", "qbits", "n", "gamma")}
    pool = np.zeros(nbytes, np.uint8)
    O.pack(pool, nbytes, d, m, False, np.zeros(N), np.arange(N), rec)
    ids, sc = O.topk(P, rng.standard_normal((2, d)), pool, nbytes, N, 5)
    assert np.array_equal(ids, np.tile(np.arange(5), (2, 1)))
    assert np.all(sc == sc[:, :1])


@pytest.mark.parametrize("d,G", [(64, 8), (128, 4)])
def test_threshold_gate_selects_hot_only_or_hot_and_cold(O, d, G):
    """Monarch's gate ("Vereinfachte Decode-Schleife"): a head reads its cold
    tokens only when max_t <q, k_hot_t> is below the threshold.  With exact
    (zero-residual) records the gated result must be textbook attention over
    either hot or hot + cold, per head, decided by a numpy matmul of q with
    the hot keys; the threshold sits between the raw maxima so that both
    outcomes occur and a scaled-score gate would give a different split."""
    m = d
    P = O.Params(d, seed=5)
    rng = np.random.default_rng(100 + d + G)
    B, Hkv = 3, 2
    Hq = G * Hkv
    max_pages = 3
    nbytes, _ = O.page_layout(d, m, True)
    n_pages = B * Hkv * max_pages
    pool = np.zeros(n_pages * nbytes, np.uint8)
    table = rng.permutation(n_pages).astype(np.int32).reshape(B, Hkv, max_pages)
    W = 70
    k_hot = np.float16(rng.standard_normal((B, Hkv, W, d))).astype(np.float64)
    v_hot = np.float16(rng.standard_normal((B, Hkv, W, d))).astype(np.float64)
    q = rng.standard_normal((B, Hq, d))
    cold_len = np.array([300, 129, 0], np.int32)
    hot_len = np.array([70, 0, 33], np.int32)
    recs = {}
    for b in range(B):
        for h in range(Hkv):
            n = int(cold_len[b])
            rec = _direct_records(rng, n, d, m)
            t = np.arange(n)
            O.pack(pool, nbytes, d, m, True, table[b, h, t // 128], t % 128, rec)
            recs[b, h] = rec
    scale = 1.0 / math.sqrt(d)
    hmax = np.full((B, Hq), -np.inf)
    for b in range(B):
        for hq in range(Hq):
            if hot_len[b]:
                hmax[b, hq] = (k_hot[b, hq // G, :hot_len[b]] @ q[b, hq]).max()
    finite = np.sort(hmax[np.isfinite(hmax)])
    thr = 0.5 * (finite[len(finite) // 2 - 1] + finite[len(finite) // 2])
    out, groups, opened = O.attention(P, q, Hkv, scale, k_hot, v_hot, hot_len, pool, nbytes,
                                      table, cold_len, threshold=thr)
    want_open = hmax < thr
    assert want_open.any() and (~want_open[np.isfinite(hmax)]).any()
    assert (hmax * scale < thr).sum() != want_open.sum()  # the scale matters for this threshold
    for gi, (b, h) in enumerate(groups):
        Kc, Vc = _reconstruct(P, recs[b, h])
        Kh, Vh = k_hot[b, h, :hot_len[b]], v_hot[b, h, :hot_len[b]]
        for g in range(G):
            hq = h * G + g
            assert opened[gi, g] == int(want_open[b, hq])
            K = np.concatenate([Kc, Kh]) if want_open[b, hq] else Kh
            V = np.concatenate([Vc, Vh]) if want_open[b, hq] else Vh
            ref = np.zeros(d) if len(K) == 0 else _sdpa(q[b, hq][None], K, V, scale)[0]
            assert np.abs(out[gi, g] - ref).max() <= 1e-10 * max(1.0, np.abs(ref).max())
    # +inf opens every head: the ungated result; -inf shuts every head: hot
    # tokens alone, zeros where there are none
    ung, _ = O.attention(P, q, Hkv, scale, k_hot, v_hot, hot_len, pool, nbytes, table, cold_len)
    out_inf, _, op_inf = O.attention(P, q, Hkv, scale, k_hot, v_hot, hot_len, pool, nbytes,
                                     table, cold_len, threshold=np.inf)
    assert op_inf.all() and np.array_equal(out_inf, ung)
    out_ninf, _, op_ninf = O.attention(P, q, Hkv, scale, k_hot, v_hot, hot_len, pool, nbytes,
                                       table, cold_len, threshold=-np.inf)
    assert not op_ninf.any()
    for gi, (b, h) in enumerate(groups):
        for g in range(G):
            if hot_len[b] == 0:
                assert not out_ninf[gi, g].any()
            else:
                ref = _sdpa(q[b, h * G + g][None], k_hot[b, h, :hot_len[b]],
                            v_hot[b, h, :hot_len[b]], scale)[0]
                assert np.abs(out_ninf[gi, g] - ref).max() <= 1e-10 * max(1.0, np.abs(ref).max())
