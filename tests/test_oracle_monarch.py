"""Pins of the oracle's Monarch cache (hot window, eviction to cold, gated
attention), independent of the CUDA path.

- Window invariant: after every step the hot window holds min(total, window)
  tokens for E = 1 (the loop as written) and between window and
  window + E - 1 once warm for larger E.
- Placement: the hot tokens are the last ones appended, in order; the cold
  pages hold the encoding of every earlier token at its position.
- Attention with the gate shut equals textbook attention over exactly the
  last hot_len appended tokens (torch's scaled_dot_product_attention, fp64).
"""
import math

import numpy as np
import pytest
import torch

from oracle.monarch import MonarchCache


def _sdpa(q, k, v, scale):
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a, np.float64))
    return torch.nn.functional.scaled_dot_product_attention(
        t(q)[None, None], t(k)[None, None], t(v)[None, None], scale=scale)[0, 0].numpy()


def _run(O, d, B, Hkv, G, window, E, steps, seed, threshold):
    P = O.Params(d, seed=3)
    rng = np.random.default_rng(seed)
    max_pages = (steps + 127) // 128 + 1
    table = rng.permutation(B * Hkv * max_pages).astype(np.int32).reshape(B, Hkv, max_pages)
    cache = MonarchCache(P, B, Hkv, window, E, table)
    toks_k, toks_v, outs = [], [], []
    for s in range(steps):
        k = rng.standard_normal((B, Hkv, d))
        v = rng.standard_normal((B, Hkv, d))
        q = rng.standard_normal((B, G * Hkv, d))
        out, opened = cache.step(q, k, v, 1.0 / math.sqrt(d), threshold)
        toks_k.append(np.float16(k).astype(np.float64))
        toks_v.append(np.float16(v).astype(np.float64))
        outs.append((q, out, opened, cache.hot_len(0), int(cache.cold_len[0])))
    return P, cache, np.stack(toks_k, 2), np.stack(toks_v, 2), outs


@pytest.mark.parametrize("E", [1, 8])
def test_window_invariant_and_placement(O, E):
    d, B, Hkv, G, window, steps = 64, 2, 2, 2, 12, 45
    P, cache, K, V, outs = _run(O, d, B, Hkv, G, window, E, steps, 7 + E, None)
    for s, (_, _, _, hl, cl) in enumerate(outs):
        total = s + 1
        if E == 1:
            assert hl == min(total, window)
        else:
            assert hl < window + E and (total < window or hl >= window)
        assert hl + cl == total
    hl, cl = cache.hot_len(0), int(cache.cold_len[0])
    for b in range(B):
        for h in range(Hkv):
            hot = np.stack([kv[0] for kv in cache.hot[b][h]])
            assert np.array_equal(hot, K[b, h, cl:])
            t = np.arange(cl)
            got = O.unpack(cache.pool, cache.page_bytes, d, d, True, cache.table[b, h, t // 128],
                           t % 128)
            want = O.encode(P, K[b, h, :cl], True)
            assert np.array_equal(got["sign"], want["sign"]) and np.array_equal(got["mag"], want["mag"])
            assert np.array_equal(got["qbits"], want["qbits"])
            wv = O.encode(P, V[b, h, :cl], False)
            assert np.array_equal(got["vcode"], wv["vcode"])


def test_shut_gate_attends_to_the_last_hot_tokens(O):
    d, B, Hkv, G, window, E, steps = 64, 2, 2, 4, 10, 4, 30
    P, cache, K, V, outs = _run(O, d, B, Hkv, G, window, E, steps, 21, -np.inf)
    prev = 0
    for s, (q, out, opened, hl, cl) in enumerate(outs):
        total = s + 1
        n_att = prev + 1  # the step's token joins the window before attention
        prev = hl
        assert not opened.any()
        for b in range(B):
            for hq in range(Hkv * G):
                h = hq // G
                Kh, Vh = K[b, h, total - n_att:total], V[b, h, total - n_att:total]
                ref = _sdpa(q[b, hq][None], Kh, Vh, 1.0 / math.sqrt(d))[0]
                assert np.abs(out[b, hq] - ref).max() <= 1e-10 * max(1.0, np.abs(ref).max())


# --------------------------------------------------------------------------
# attention-weighted promotion with stickiness
# --------------------------------------------------------------------------
def _promo_cache(O, d=64, Hkv=2, G=2, n_cold=300, n_hot=8, attractors=(), c_attr=10.0, seed=5,
                 promotion=None, window=64, E=16, W_max=96):
    """One sequence: n_cold cold tokens (random keys, N(0,1)) of which the
    positions in `attractors` hold keys c_attr * u (u a unit direction), a few
    hot tokens, and queries 8 u (+ small noise) or -8 u: at scale 1/sqrt(d) an
    attractor's logit is about +-c_attr, a random key's about N(0, 1)."""
    P = O.Params(d, seed=9)
    rng = np.random.default_rng(seed)
    u = rng.standard_normal(d)
    u /= np.linalg.norm(u)
    max_pages = (n_cold + 200) // 128 + 2
    table = np.arange(Hkv * max_pages, dtype=np.int32).reshape(1, Hkv, max_pages)
    nb, _ = O.page_layout(d, d, True)
    pool = np.zeros(Hkv * max_pages * nb, np.uint8)
    K = rng.standard_normal((Hkv, n_cold + n_hot, d))
    V = rng.standard_normal((Hkv, n_cold + n_hot, d))
    for a in attractors:
        K[:, a] = c_attr * u
    t = np.arange(n_cold)
    for h in range(Hkv):
        kr, vr = O.encode(P, K[h, :n_cold], True), O.encode(P, V[h, :n_cold], False)
        O.pack(pool, nb, d, d, True, table[0, h, t // 128], t % 128,
               dict(sign=kr["sign"], mag=kr["mag"], qbits=kr["qbits"], n=kr["n"], gamma=kr["gamma"],
                    vcode=vr["vcode"], vn=vr["vn"]))
    f16 = lambda a: np.float16(a).astype(np.float64)
    hot_k = [[list(f16(K[h, n_cold:])) for h in range(Hkv)]]
    hot_v = [[list(f16(V[h, n_cold:])) for h in range(Hkv)]]
    cache = MonarchCache(P, 1, Hkv, window, E, table, cold_len=[n_cold], pool=pool, hot_k=hot_k,
                         hot_v=hot_v, promotion=promotion, W_max=W_max)
    return P, cache, u, rng


def _promo_step(cache, u, rng, sign=1.0, threshold=None, G=2):
    d, Hkv = cache.d, cache.Hkv
    q = sign * 8.0 * u + 0.05 * rng.standard_normal((1, G * Hkv, d))
    k = rng.standard_normal((1, Hkv, d))
    v = rng.standard_normal((1, Hkv, d))
    return cache.step(q, k, v, 1.0 / math.sqrt(d), threshold)


@pytest.mark.parametrize("threshold", [None, 1.0e9, "split"])
def test_promotion_path_attention_equals_c_attention(O, threshold):
    """With a promotion threshold no weight reaches, the promotion path's
    step-by-step attention equals the oracle's C attention (pinned against
    SDPA) at every step, gated or not."""
    promo = dict(threshold=2.0, sticky=3, max_per_step=4)
    _, a, u, ra = _promo_cache(O, attractors=(10, 200), promotion=promo)
    _, b, _, rb = _promo_cache(O, attractors=(10, 200), promotion=None)
    for s in range(12):
        thr = threshold
        if threshold == "split":  # between the largest raw hot scores of the two kv heads' heads
            thr = 8.0 * (1.5 if s % 2 else 0.5)
        oa, ga = _promo_step(a, u, ra, threshold=thr)
        ob, gb = _promo_step(b, u, rb, threshold=thr)
        assert np.max(np.abs(oa - ob)) < 1e-10
        if thr is not None:
            assert np.array_equal(ga, gb)
    assert not a.cold_mask.any() and not a.counts.any()


def test_attractor_moves_back_after_sticky_steps(O):
    """A cold key aligned with the queries (weight well above 0.15) counts one
    step per step and moves back at the third: its slot is masked, its count
    reset, its decompressed key and value (n Pi^T c_hat, fp16) are the newest
    hot tokens of every kv head; random keys (weights far below) never move."""
    promo = dict(threshold=0.15, sticky=3, max_per_step=4)
    P, cache, u, rng = _promo_cache(O, attractors=(123,), promotion=promo)
    for s in range(1, 6):
        _promo_step(cache, u, rng)
        if s < 3:
            assert cache.counts[0, 123] == s and not cache.cold_mask[0, 123]
        assert np.count_nonzero(cache.counts[0, :300]) <= 1
    assert cache.cold_mask[0, 123] and cache.cold_mask[0].sum() == 1
    assert cache.counts[0, 123] == 0
    rec = O.unpack(cache.pool, cache.page_bytes, 64, 64, True, cache.table[0, :, 123 // 128],
                   np.full(2, 123 % 128))
    for h in range(2):
        ck = np.where(rec["sign"][h] == 1, -1.0, 1.0) * P.kc[rec["mag"][h]]
        cv = np.where(rec["vcode"][h] >> 3, -1.0, 1.0) * P.vc[rec["vcode"][h] & 7]
        kd = np.float16(rec["n"][h] * (ck @ P.pi32)).astype(np.float64)
        vd = np.float16(rec["vn"][h] * (cv @ P.pi32)).astype(np.float64)
        # moved back after step 3's attention; steps 4 and 5 appended two tokens after it
        k3, v3 = cache.hot[0][h][-3]
        assert np.array_equal(k3, kd) and np.array_equal(v3, vd)


def test_masked_position_is_skipped(O):
    """After the move, attention skips the masked cold slot: the step's output
    equals the C attention over a cache whose cold pages hold every other
    record and whose hot window is the same."""
    promo = dict(threshold=0.15, sticky=1, max_per_step=4)
    P, cache, u, rng = _promo_cache(O, attractors=(77,), promotion=promo)
    _promo_step(cache, u, rng)  # moves 77 back
    assert cache.cold_mask[0, 77]
    state = (rng.bit_generator.state, )
    out, _ = _promo_step(cache, u, rng, sign=-1.0)
    rng.bit_generator.state = state[0]
    q = -8.0 * u + 0.05 * rng.standard_normal((1, 4, 64))
    cl = int(cache.cold_len[0])
    keep = np.array([t for t in range(cl) if not cache.cold_mask[0, t]])
    nb = cache.page_bytes
    table = np.arange(2 * 4, dtype=np.int32).reshape(1, 2, 4)
    pool = np.zeros(8 * nb, np.uint8)
    for h in range(2):
        rec = O.unpack(cache.pool, nb, 64, 64, True, cache.table[0, h, keep // 128], keep % 128)
        t = np.arange(len(keep))
        O.pack(pool, nb, 64, 64, True, table[0, h, t // 128], t % 128, rec)
    # the hot window before the step's token was appended and before eviction
    hl = cache.hot_len(0)
    kh = np.zeros((1, 2, hl, 64))
    vh = np.zeros((1, 2, hl, 64))
    for h in range(2):
        for i, (kr, vr) in enumerate(cache.hot[0][h]):
            kh[0, h, i], vh[0, h, i] = kr, vr
    ref, _ = O.attention(P, q, 2, 1.0 / 8.0, kh, vh, np.array([hl], np.int32), pool, nb, table,
                         np.array([len(keep)], np.int32))
    assert np.max(np.abs(out.reshape(-1, 64) - ref.reshape(-1, 64))) < 1e-10


def test_alternating_weight_never_counts_to_sticky(O):
    """The count is of consecutive steps: an attractor whose weight alternates
    high and low never reaches a sticky threshold of 2; with 1 it moves at its
    first high step."""
    for sticky, moved_at in ((2, None), (1, 1)):
        promo = dict(threshold=0.15, sticky=sticky, max_per_step=4)
        _, cache, u, rng = _promo_cache(O, attractors=(50,), promotion=promo)
        first = None
        for s in range(1, 9):
            _promo_step(cache, u, rng, sign=1.0 if s % 2 else -1.0)
            if cache.cold_mask[0, 50] and first is None:
                first = s
            assert cache.counts[0, 50] <= 1
        assert first == moved_at


def test_per_step_and_ring_limits(O):
    """Three attractors qualify together: at most max_per_step move in a step,
    in increasing position order, and never more than leave one free ring
    slot for the next step's token."""
    promo = dict(threshold=0.15, sticky=1, max_per_step=2)
    _, cache, u, rng = _promo_cache(O, attractors=(30, 90, 250), promotion=promo)
    _promo_step(cache, u, rng)
    assert list(np.nonzero(cache.cold_mask[0])[0]) == [30, 90]
    _promo_step(cache, u, rng)
    assert list(np.nonzero(cache.cold_mask[0])[0]) == [30, 90, 250]
    # ring room: 8 hot + 1 appended = 9 of W_max 11, one slot kept free -> one move
    promo = dict(threshold=0.15, sticky=1, max_per_step=4)
    _, cache, u, rng = _promo_cache(O, attractors=(30, 90, 250), promotion=promo, window=9, E=2,
                                    W_max=11)
    _promo_step(cache, u, rng)
    assert list(np.nonzero(cache.cold_mask[0])[0]) == [30]
    assert cache.hot_len(0) == 10  # 9 + the moved token; below window + E = 11, nothing evicted
