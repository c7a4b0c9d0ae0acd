"""Pins of the QJL correction inside the oracle's scores (residual norm > 0).

Source: "TurboQuant" summary, de.news.hada.io topic 27867, section "QJL: Eine
1-Bit-Methode ohne Overhead" (the sign bits of a Gaussian projection of the
residual, paired with the full-precision query, give an inner-product
estimate), and "Die KV-Cache-Optimierung von Google erklaert", section "Stufe
2" (the estimate is unbiased).

For a key x with stored norm n, rotated value x_rot and residual
r = x_rot / n - c_hat, the estimated score is
    s = n (<q_rot, c_hat> + sqrt(pi/2)/m * gamma * <S q_rot, 1 - 2 b>),
b_i = [(S r)_i < 0], gamma = |r| (fp16).  Over Gaussian S it is unbiased for
the exact score t = <q_rot, x_rot>, with variance
    n^2 [ (pi/2) |q_rot|^2 gamma^2 - gamma^2 <q_rot, r>^2 / |r|^2 ] / m
(E[(g.q)^2] = |q|^2 and E[sign(g.r) g.q] = sqrt(2/pi) <q, r>/|r| for a
Gaussian row g).  The keys are symmetric in distribution (x -> -x flips r and
every bit), so the error has mean zero for every key and errors of different
keys are uncorrelated even under a shared S; averaging over keys and several
seeds (several S) estimates the S-averaged variance.

The tests read the estimate from the oracle's top-k search (scores of every
key) and from its decode attention (the logit difference against a reference
token whose residual is zero), and compare both with the exact inner products
computed here with numpy -- never with the oracle's own scorer.  A mistake in
the estimator (the sketch of q instead of q_rot, a wrong constant, a flipped
sign) moves the variance or the slope of the error against <q_rot, r>."""
import math

import numpy as np
import pytest

D_SEEDS = [(64, [3, 4, 5, 6, 7, 8, 9, 10]), (128, [11, 12, 13, 14])]
NQ, NK = 64, 128  # queries and keys per seed: every query scores every key
NATT = 1024       # (query, key) pairs per seed read back through the attention


def _keys_only_pages(O, d, rec):
    nb, _ = O.page_layout(d, d, False)
    N = len(rec["n"])
    pool = np.zeros(nb * ((N + 127) // 128), np.uint8)
    idx = np.arange(N)
    O.pack(pool, nb, d, d, False, idx // 128, idx % 128,
           {k: rec[k] for k in ("sign", "mag", "qbits", "n", "gamma")})
    return pool, nb


def _chat(P, sign, mag):
    return np.where(sign == 1, -1.0, 1.0) * P.kc[mag]


def _estimates(O, d, seed):
    """One seed (one S): NQ random unit queries against NK keys.  Returns, per
    (query, key) pair, the search estimate, the exact score, n <q_rot, r> and
    the closed-form variance, and for the pairs (i mod NQ, i) the estimate
    recovered from the decode attention for NATT random pairs."""
    P = O.Params(d, seed=seed)
    rng = np.random.default_rng(1000 + seed)
    x = np.float32(rng.standard_normal((NK, d))).astype(np.float64)
    q = rng.standard_normal((NQ, d))
    q /= np.linalg.norm(q, axis=1, keepdims=True)
    rec = O.encode(P, x, True)
    assert np.all(rec["gamma"] > 0)
    qrot = q @ P.pi32.T                                # [NQ, d]
    exact = qrot @ rec["xrot"].T                       # <q_rot, x_rot>
    chat = _chat(P, rec["sign"], rec["mag"])
    r = rec["xrot"] / rec["n"][:, None] - chat         # residual, rotated unit domain
    n, g = rec["n"], rec["gamma"]
    qr = qrot @ r.T                                    # [NQ, NK]
    var = (n ** 2 * g ** 2)[None] * ((math.pi / 2) * np.sum(qrot ** 2, 1)[:, None]
                                     - qr ** 2 / np.sum(r * r, 1)[None]) / d

    # 1. search: every key's estimate for every query (k = NK)
    pool, nb = _keys_only_pages(O, d, rec)
    ids, sc = O.topk(P, q, pool, nb, NK, NK)
    s_topk = np.empty((NQ, NK))
    np.put_along_axis(s_topk, ids.astype(np.int64), sc, axis=1)

    # 2. attention: sequence i (query qi[i]) holds a reference record
    # (gamma = 0, so its estimate is exactly n_ref <q_rot, c_hat_ref>) in
    # slot 0 and key ki[i] in slot 1; both carry the same value code, the key with
    # twice the value norm, so out = v_hat_ref (1 + p_i) and the logit
    # difference log(p_i / (1 - p_i)) is s_i - s_ref (scale 1).
    N = NATT
    nbv, _ = O.page_layout(d, d, True)
    ref_sign = rng.integers(0, 2, d).astype(np.int32)
    ref_mag = rng.integers(0, 2, d).astype(np.int32)
    ref_n = float(np.float16(3.0))
    vcode = rng.integers(0, 16, d).astype(np.int32)
    vn_ref = float(np.float16(1.5))
    qi = rng.integers(0, NQ, N)
    ki = rng.integers(0, NK, N)
    s_ref = ref_n * (qrot[qi] @ _chat(P, ref_sign, ref_mag))
    recs = dict(sign=np.concatenate([np.tile(ref_sign, (N, 1)), rec["sign"][ki]]),
                mag=np.concatenate([np.tile(ref_mag, (N, 1)), rec["mag"][ki]]),
                qbits=np.concatenate([np.zeros((N, d), np.int32), rec["qbits"][ki]]),
                n=np.concatenate([np.full(N, ref_n), n[ki]]),
                gamma=np.concatenate([np.zeros(N), g[ki]]),
                vcode=np.tile(vcode, (2 * N, 1)),
                vn=np.concatenate([np.full(N, vn_ref), np.full(N, 2 * vn_ref)]))
    vpool = np.zeros(N * nbv, np.uint8)
    seq = np.arange(N)
    O.pack(vpool, nbv, d, d, True, np.concatenate([seq, seq]),
           np.concatenate([np.zeros(N, int), np.ones(N, int)]), recs)
    table = seq.astype(np.int32).reshape(N, 1, 1)
    out, _ = O.attention(P, q[qi][:, None, :], 1, 1.0, None, None, None, vpool, nbv, table,
                         np.full(N, 2, np.int32))
    vc = np.where(vcode >> 3, -1.0, 1.0) * P.vc[vcode & 7]
    vhat = vn_ref * (vc @ P.pi32)
    p = out[:, 0, :] @ vhat / (vhat @ vhat) - 1.0
    s_attn = s_ref + np.log(p / (1.0 - p))
    return dict(topk=s_topk.ravel(), exact=exact.ravel(), nqr=(n[None] * qr).ravel(),
                var=var.ravel(), attn=s_attn, attn_exact=exact[qi, ki],
                attn_nqr=n[ki] * qr[qi, ki], attn_var=var[qi, ki], attn_topk=s_topk[qi, ki])


@pytest.fixture(scope="module")
def samples(O):
    res = {}
    for d, seeds in D_SEEDS:
        parts = [_estimates(O, d, s) for s in seeds]
        res[d] = {k: np.concatenate([p[k] for p in parts]) for k in parts[0]}
    return res


def _check_unbiased(e, nqr, var):
    N = len(e)
    se = e.std(ddof=1) / math.sqrt(N)
    assert abs(e.mean()) <= 3 * se, (e.mean(), se)
    # sample variance against the S-averaged closed form
    assert abs(e.var(ddof=1) / var.mean() - 1.0) < 0.10, (e.var(ddof=1), var.mean())
    # unbiased for every key: no trend of the error against n <q_rot, r>
    slope = np.cov(e, nqr)[0, 1] / nqr.var(ddof=1)
    resid = e - slope * (nqr - nqr.mean())
    se_slope = resid.std(ddof=2) / (nqr.std(ddof=1) * math.sqrt(N))
    assert abs(slope) <= 4 * se_slope, (slope, se_slope)


@pytest.mark.parametrize("d", [64, 128])
def test_search_estimate_unbiased_with_closed_form_variance(samples, d):
    s = samples[d]
    _check_unbiased(s["topk"] - s["exact"], s["nqr"], s["var"])


@pytest.mark.parametrize("d", [64, 128])
def test_attention_estimate_unbiased_with_closed_form_variance(samples, d):
    s = samples[d]
    _check_unbiased(s["attn"] - s["attn_exact"], s["attn_nqr"], s["attn_var"])


@pytest.mark.parametrize("d", [64, 128])
def test_attention_logit_difference_equals_search_score(samples, d):
    """The decode attention scores a cold key exactly as the search does (the
    logit difference recovered from the attention output equals the search
    estimate of the same query and key)."""
    s = samples[d]
    assert np.max(np.abs(s["attn"] - s["attn_topk"])) < 1e-10
