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
