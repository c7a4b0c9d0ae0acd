"""Parity of Monarch's attention-weighted promotion with stickiness
(tq_monarch_step_promote, through the C ABI) with the oracle's Monarch cache,
step by step.

Both sides start from the same state: cold pages written by the oracle's
packer, in which a few positions hold "attractor" keys aligned with the
sequence's queries (weight far above the 0.15 threshold), the others random
keys (weights far below it), and the same hot tokens; both take the same
seeded tokens and queries (8 u + noise on most steps, -8 u on some, so that
counts also reset).  Per step: ring start and lengths exact; the moved-back
mask and the per-position counts exact; attention within 2e-3 + 1e-2 |ref|.
The moved-back rows are n Pi^T c_hat rounded to fp16 on both sides (fp32 on
the GPU, fp64 in the oracle): equal within one fp16 unit in the last place
plus the fp32 sum's rounding error (moved_row_tol).
Without eviction every hot row is compared; with eviction the evicted rows
are compressed by each side, so outputs are compared only before the first
eviction that takes a moved-back row."""
import math

import numpy as np
import pytest

import compressed_kv_decode_b200 as tq
from oracle.monarch import MonarchCache

from decode_cases import assert_close

pytestmark = pytest.mark.gpu


def f16(a):
    return np.float16(a).astype(np.float64)


def moved_row_tol(row):
    """Tolerance of a moved-back row, n Pi^T c_hat rounded to fp16, GPU
    (fp32 sums of d products) against the oracle (fp64): one fp16 unit in the
    last place, plus the fp32 accumulation's error, at most d * 2^-24 times
    the sum of the products' magnitudes, which is taken as 2^-17 (d <= 128)
    times the row's largest element (the products are of the order of the
    row's entries; an entry that cancels to near zero keeps this absolute
    error)."""
    row = np.asarray(row, np.float64)
    return np.abs(np.spacing(np.float16(row)).astype(np.float64)) + 2.0 ** -17 * np.abs(row).max()


def run(O, d, G, steps, window, E, W_max, attractors, promo, mode="open", seed=3, n_cold=300,
        n_hot=8, signs=None):
    """mode "open": every head reads the cold tier; "mid": threshold 40 on
    the raw hot scores, and every new key of kv head 1 is 6 u, so that its
    heads keep off the cold tier (raw score 48) while kv head 0's read it
    (raw hot scores of random keys about N(0, 64)) until a moved-back
    attractor (raw score about 80) enters its hot window."""
    import torch
    P = O.Params(d, seed=0)
    ctx = tq.Context(d, 0)
    B, Hkv = 2, 2
    Hq = G * Hkv
    rng = np.random.default_rng(seed)
    u = rng.standard_normal((B, d))
    u /= np.linalg.norm(u, axis=1, keepdims=True)
    max_pages = (n_cold + steps + 127) // 128 + 1
    table = rng.permutation(B * Hkv * max_pages).astype(np.int32).reshape(B, Hkv, max_pages)
    nb, _ = O.page_layout(d, d, True)
    pool = np.zeros(B * Hkv * max_pages * nb, np.uint8)
    hot_k = [[None] * Hkv for _ in range(B)]
    hot_v = [[None] * Hkv for _ in range(B)]
    cold0 = [n_cold, n_cold - 37]
    for b in range(B):
        for h in range(Hkv):
            n = cold0[b] + n_hot
            K, V = rng.standard_normal((n, d)), rng.standard_normal((n, d))
            for a in attractors:
                if a < cold0[b]:
                    K[a] = 10.0 * u[b]
            t = np.arange(cold0[b])
            kr, vr = O.encode(P, K[:cold0[b]], True), O.encode(P, V[:cold0[b]], False)
            O.pack(pool, nb, d, d, True, table[b, h, t // 128], t % 128,
                   dict(sign=kr["sign"], mag=kr["mag"], qbits=kr["qbits"], n=kr["n"],
                        gamma=kr["gamma"], vcode=vr["vcode"], vn=vr["vn"]))
            hot_k[b][h] = list(f16(K[cold0[b]:]))
            hot_v[b][h] = list(f16(V[cold0[b]:]))
    cache = MonarchCache(P, B, Hkv, window, E, table, cold_len=cold0, pool=pool, hot_k=hot_k,
                         hot_v=hot_v, promotion=promo, W_max=W_max)
    starts = [W_max - 3, 5]
    kr_ = np.full((B, Hkv, W_max, d), np.nan)
    vr_ = np.full((B, Hkv, W_max, d), np.nan)
    for b in range(B):
        for h in range(Hkv):
            for i in range(n_hot):
                kr_[b, h, (starts[b] + i) % W_max] = hot_k[b][h][i]
                vr_[b, h, (starts[b] + i) % W_max] = hot_v[b][h][i]
    dev = "cuda"
    k_hot = torch.from_numpy(kr_).half().to(dev)
    v_hot = torch.from_numpy(vr_).half().to(dev)
    hs = torch.tensor(starts, dtype=torch.int32, device=dev)
    hl = torch.tensor([n_hot] * B, dtype=torch.int32, device=dev)
    cl = torch.tensor(cold0, dtype=torch.int32, device=dev)
    gpool = torch.from_numpy(pool.reshape(-1, nb).copy()).to(dev)
    tbl = torch.from_numpy(table).to(dev)
    out = torch.empty((B, Hq, d), dtype=torch.float32, device=dev)
    used = torch.empty((B, Hq), dtype=torch.int32, device=dev)
    ws = torch.empty(tq.tq_monarch_workspace_bytes(ctx.handle, B, Hq, Hkv, max_pages, W_max, E),
                     dtype=torch.uint8, device=dev)
    cap = max_pages * 128
    gpromo = dict(promo, cold_mask=torch.zeros((B, cap // 32), dtype=torch.int32, device=dev),
                  counts=torch.zeros((B, cap), dtype=torch.uint8, device=dev),
                  logits=torch.empty((B, Hq, cap), dtype=torch.float32, device=dev))
    scale = 1.0 / math.sqrt(d)
    exp_start = list(starts)
    moved_rows = [set() for _ in range(B)]  # logical ring indices of moved-back rows
    compare = True
    n_moves = 0
    n_prev = [0] * B
    for s in range(steps):
        sg = 1.0 if signs is None else signs[s % len(signs)]
        q = sg * 8.0 * np.repeat(u, Hq, axis=0).reshape(B, Hq, d) + 0.05 * rng.standard_normal((B, Hq, d))
        k_new, v_new = f16(rng.standard_normal((B, Hkv, d))), f16(rng.standard_normal((B, Hkv, d)))
        thr = np.inf
        if mode == "mid":
            k_new[:, 1] = f16(6.0 * u)
            thr = 40.0
        hot_before = [cache.hot_len(b) for b in range(B)]
        ref, opened = cache.step(q, k_new, v_new, scale, thr)
        tq.tq_monarch_step_promote(ctx.handle, torch.from_numpy(q).float().to(dev),
                                   torch.from_numpy(k_new).half().to(dev),
                                   torch.from_numpy(v_new).half().to(dev), k_hot, v_hot, hs, hl,
                                   gpool, tbl, cl, thr, window, E, gpromo, out, ws, Hkv,
                                   cold_used=used)
        torch.cuda.synchronize()
        assert tq.tq_get_error(ctx.handle) == tq.TQ_OK
        got = out.cpu().numpy().astype(np.float64)
        gm = gpromo["cold_mask"].cpu().numpy().view(np.uint32)
        gc = gpromo["counts"].cpu().numpy()
        assert np.array_equal(gu := used.cpu().numpy(), opened), "gate decisions"
        for b in range(B):
            bits = np.unpackbits(gm[b].view(np.uint8), bitorder="little").astype(bool)
            assert np.array_equal(bits, cache.cold_mask[b]), "moved-back mask, step %d" % s
            assert np.array_equal(gc[b].astype(np.int32), cache.counts[b]), "counts, step %d" % s
        # ring bookkeeping: eviction advances the start
        for b in range(B):
            moved_now = int(cache.cold_mask[b].sum()) - n_prev[b]
            n_prev[b] += moved_now
            for i in range(moved_now):  # the step's moves follow its appended token
                moved_rows[b].add(hot_before[b] + 1 + i)
            n_moves += moved_now
            ev = hot_before[b] + 1 + moved_now - cache.hot_len(b)
            if ev:
                if any(i < ev for i in moved_rows[b]):
                    compare = False  # a moved-back row went back to cold
                moved_rows[b] = {i - ev for i in moved_rows[b] if i >= ev}
                exp_start[b] = (exp_start[b] + ev) % W_max
                # each side compresses the evicted rows; a bit may differ at a
                # rounding boundary (see test_gpu_monarch), and then outputs
                # are compared no further
                t = np.arange(int(cache.cold_len[b]) - ev, int(cache.cold_len[b]))
                gp_now = gpool.cpu().numpy().reshape(-1)
                for h in range(Hkv):
                    a = O.unpack(gp_now, nb, d, d, True, table[b, h, t // 128], t % 128)
                    o = O.unpack(cache.pool, nb, d, d, True, table[b, h, t // 128], t % 128)
                    if any(not np.array_equal(a[key], o[key]) for key in o):
                        compare = False
        assert np.array_equal(hl.cpu().numpy(), [cache.hot_len(b) for b in range(B)])
        assert np.array_equal(cl.cpu().numpy(), cache.cold_len)
        assert np.array_equal(hs.cpu().numpy(), exp_start)
        if compare:
            for b in range(B):
                for hq in range(Hq):
                    assert_close(got[b, hq], ref[b, hq], what="step %d head %s" % (s, (b, hq)))
            kg = k_hot.float().cpu().numpy()
            vg = v_hot.float().cpu().numpy()
            for b in range(B):
                for h in range(Hkv):
                    for i in range(cache.hot_len(b)):
                        slot = (exp_start[b] + i) % W_max
                        kk, vv = cache.hot[b][h][i]
                        if i in moved_rows[b]:
                            for g_, w_ in ((kg[b, h, slot], kk), (vg[b, h, slot], vv)):
                                assert np.all(np.abs(g_ - w_) <= moved_row_tol(w_)), "moved-back row"
                        else:
                            assert np.array_equal(kg[b, h, slot], kk)
                            assert np.array_equal(vg[b, h, slot], vv)
    return cache, n_moves


@pytest.mark.parametrize("d,G", [(64, 2), (128, 4), (64, 8)])
def test_attractors_move_back_like_the_oracle(O, d, G):
    promo = dict(threshold=0.15, sticky=3, max_per_step=2)
    cache, n = run(O, d, G, steps=14, window=64, E=16, W_max=96, attractors=(5, 140, 141, 299),
                   promo=promo, signs=[1, 1, 1, 1, -1, 1, 1, 1, 1, 1])
    assert n >= 6  # every attractor of both sequences moved (one of sequence 1 lies past its cold end)


def test_counts_reset_on_low_steps(O):
    """Alternating queries: an attractor's weight is high every other step, so
    with a sticky count of 2 nothing moves on either side."""
    promo = dict(threshold=0.15, sticky=2, max_per_step=4)
    cache, n = run(O, 64, 4, steps=9, window=64, E=16, W_max=96, attractors=(40, 200),
                   promo=promo, signs=[1, -1])
    assert n == 0 and cache.counts.max() == 1


def test_gate_split_and_ring_limit(O):
    """The heads of kv head 1 keep off the cold tier: weights come from kv
    head 0's heads alone; a ring of 13 slots leaves room for 3 of the 5
    candidates of the first step."""
    promo = dict(threshold=0.15, sticky=1, max_per_step=8)
    cache, n = run(O, 64, 2, steps=8, window=9, E=3, W_max=13, attractors=(1, 2, 3, 100, 101),
                   promo=promo, mode="mid")
    assert n >= 6


def test_moves_then_eviction(O):
    """A small window: moved-back rows are evicted again into new cold
    positions; masks, counts and lengths stay exact throughout."""
    promo = dict(threshold=0.15, sticky=2, max_per_step=3)
    cache, n = run(O, 128, 4, steps=24, window=12, E=4, W_max=20, attractors=(7, 8, 250),
                   promo=promo)
    assert n >= 8  # the attractors moved back again after their eviction


def test_promotion_arguments_rejected(O):
    import torch
    ctx = tq.Context(64, 0)
    dev = "cuda"
    B, Hkv, Hq, d, W_max, max_pages = 1, 1, 2, 64, 8, 2
    z = lambda *s, dt=torch.float32: torch.zeros(s, dtype=dt, device=dev)
    args = dict(q=z(B, Hq, d), k_new=z(B, Hkv, d, dt=torch.float16),
                v_new=z(B, Hkv, d, dt=torch.float16), k_hot=z(B, Hkv, W_max, d, dt=torch.float16),
                v_hot=z(B, Hkv, W_max, d, dt=torch.float16), hot_start=z(B, dt=torch.int32),
                hot_len=z(B, dt=torch.int32), page_pool=z(2, ctx.page_bytes(True), dt=torch.uint8),
                page_table=z(B, Hkv, max_pages, dt=torch.int32), cold_len=z(B, dt=torch.int32))
    ws = z(tq.tq_monarch_workspace_bytes(ctx.handle, B, Hq, Hkv, max_pages, W_max, 2), dt=torch.uint8)
    good = dict(threshold=0.15, sticky=3, max_per_step=2, cold_mask=z(B, 8, dt=torch.int32),
                counts=z(B, 256, dt=torch.uint8), logits=z(B, Hq, 256))
    for bad in (dict(threshold=0.0), dict(threshold=float("nan")), dict(sticky=0),
                dict(max_per_step=0), dict(max_per_step=tq.TQ_PROMOTE_MAX_PER_STEP + 1)):
        with pytest.raises(tq.TQError) as e:
            tq.tq_monarch_step_promote(ctx.handle, args["q"], args["k_new"], args["v_new"],
                                       args["k_hot"], args["v_hot"], args["hot_start"],
                                       args["hot_len"], args["page_pool"], args["page_table"],
                                       args["cold_len"], float("inf"), 4, 2, dict(good, **bad),
                                       z(B, Hq, d), ws, Hkv)
        assert e.value.status == tq.TQ_ERR_INVALID_ARG
    ctx.close()


def test_tinyllama_shape_promotion(O):
    """The promotion step at the TinyLlama decode shape the benchmark times
    (B = 1, 32 q / 4 kv heads, d = 64, 1024 cold tokens written by the
    oracle's packer, 384 hot tokens in a 512-slot ring, E = 128; K, V with
    4 outlier channels x10): the same query every step, the threshold placed
    in the widest gap of the oracle's first-step weights among the largest
    ones (so no decision lies near it), sticky 2, up to 8 moves per step.
    Masks, counts, lengths and ring start exact after every step; outputs
    within the decode tolerance; moved-back rows within moved_row_tol."""
    import copy
    import torch
    from compressed_kv_decode_b200 import workloads as W
    cfg = W.DECODE["tinyllama"]
    B, Hq, Hkv, d = cfg["B"], cfg["Hq"], cfg["Hkv"], cfg["d"]
    G = Hq // Hkv
    n_cold, n_hot, W_max, E = 1024, 384, 512, 128
    window = W_max - E
    steps = 6
    P = O.Params(d, seed=0)
    ctx = tq.Context(d, 0)
    sk, sv, sq, so = cfg["seeds"]
    chans = W.outlier_channels(so, Hkv, d, cfg["n_out"])
    T = n_cold + n_hot + steps
    max_pages = (n_cold + steps + 127) // 128 + 1
    table, n_pages = W.random_page_table(5, B, Hkv, max_pages)
    nb, _ = O.page_layout(d, d, True)
    pool = np.zeros(n_pages * nb, np.uint8)
    seqs = []
    hot_k = [[None] * Hkv]
    hot_v = [[None] * Hkv]
    for h in range(Hkv):
        K, V = W.kv_sequence(sk, sv, 0, h, T, d, chans[h], cfg["factor"])
        K, V = f16(K), f16(V)
        seqs.append((K, V))
        t = np.arange(n_cold)
        kr, vr = O.encode(P, K[:n_cold], True), O.encode(P, V[:n_cold], False)
        O.pack(pool, nb, d, d, True, table[0, h, t // 128], t % 128,
               dict(sign=kr["sign"], mag=kr["mag"], qbits=kr["qbits"], n=kr["n"],
                    gamma=kr["gamma"], vcode=vr["vcode"], vn=vr["vn"]))
        hot_k[0][h] = list(K[n_cold:n_cold + n_hot])
        hot_v[0][h] = list(V[n_cold:n_cold + n_hot])
    q = W.queries(sq, B, Hq, d, cfg["q_dtype"])
    scale = 1.0 / math.sqrt(d)
    new_k = [np.stack([seqs[h][0][n_cold + n_hot + s] for h in range(Hkv)])[None] for s in range(steps)]
    new_v = [np.stack([seqs[h][1][n_cold + n_hot + s] for h in range(Hkv)])[None] for s in range(steps)]
    base = MonarchCache(P, B, Hkv, window, E, table, cold_len=[n_cold], pool=pool, hot_k=hot_k,
                        hot_v=hot_v, promotion=dict(threshold=1.0, sticky=2, max_per_step=8),
                        W_max=W_max)
    probe = copy.deepcopy(base)
    probe.append(new_k[0], new_v[0])
    _, _, wmax = probe.attend_weights(q, scale)
    w = np.sort(wmax[0])[::-1][:40]
    gaps = w[:-1] / np.maximum(w[1:], 1e-30)
    i = int(np.argmax(gaps[4:])) + 4  # at least five positions above the threshold
    assert gaps[i] > 1.3, gaps
    thr = float(np.sqrt(w[i] * w[i + 1]))
    promo = dict(threshold=thr, sticky=2, max_per_step=8)
    cache = copy.deepcopy(base)
    cache.promo = promo
    dev = "cuda"
    kr_ = np.full((B, Hkv, W_max, d), np.nan)
    vr_ = np.full((B, Hkv, W_max, d), np.nan)
    for h in range(Hkv):
        kr_[0, h, :n_hot] = np.stack(hot_k[0][h])
        vr_[0, h, :n_hot] = np.stack(hot_v[0][h])
    k_hot = torch.from_numpy(kr_).half().to(dev)
    v_hot = torch.from_numpy(vr_).half().to(dev)
    hs = torch.zeros(B, dtype=torch.int32, device=dev)
    hl = torch.full((B,), n_hot, dtype=torch.int32, device=dev)
    cl = torch.full((B,), n_cold, dtype=torch.int32, device=dev)
    gpool = torch.from_numpy(pool.reshape(n_pages, nb).copy()).to(dev)
    tbl = torch.from_numpy(table).to(dev)
    out = torch.empty((B, Hq, d), dtype=torch.float32, device=dev)
    used = torch.empty((B, Hq), dtype=torch.int32, device=dev)
    ws = torch.empty(tq.tq_monarch_workspace_bytes(ctx.handle, B, Hq, Hkv, max_pages, W_max, E),
                     dtype=torch.uint8, device=dev)
    cap = max_pages * 128
    gpromo = dict(promo, cold_mask=torch.zeros((B, cap // 32), dtype=torch.int32, device=dev),
                  counts=torch.zeros((B, cap), dtype=torch.uint8, device=dev),
                  logits=torch.empty((B, Hq, cap), dtype=torch.float32, device=dev))
    qd = torch.from_numpy(q).to(torch.float16).to(dev)
    n_moved = 0
    for s in range(steps):
        hot_before = cache.hot_len(0)
        ref, opened = cache.step(q, new_k[s], new_v[s], scale, np.inf)
        tq.tq_monarch_step_promote(ctx.handle, qd, torch.from_numpy(new_k[s]).half().to(dev),
                                   torch.from_numpy(new_v[s]).half().to(dev), k_hot, v_hot, hs, hl,
                                   gpool, tbl, cl, float("inf"), window, E, gpromo, out, ws, Hkv,
                                   cold_used=used)
        torch.cuda.synchronize()
        assert tq.tq_get_error(ctx.handle) == tq.TQ_OK
        gm = gpromo["cold_mask"].cpu().numpy().view(np.uint32)
        bits = np.unpackbits(gm[0].view(np.uint8), bitorder="little").astype(bool)
        assert np.array_equal(bits, cache.cold_mask[0]), "moved-back mask, step %d" % s
        assert np.array_equal(gpromo["counts"].cpu().numpy()[0].astype(np.int32), cache.counts[0])
        assert hl.item() == cache.hot_len(0) and cl.item() == cache.cold_len[0] and hs.item() == 0
        got = out.cpu().numpy().astype(np.float64)
        for hq in range(Hq):
            assert_close(got[0, hq], ref[0, hq], what="step %d head %d" % (s, hq))
        moved = cache.hot_len(0) - hot_before - 1
        kg = k_hot.float().cpu().numpy()
        for h in range(Hkv):
            for i in range(hot_before + 1, cache.hot_len(0)):
                kk, vv = cache.hot[0][h][i]
                for g_, w_ in ((kg[0, h, i], kk), (v_hot.float().cpu().numpy()[0, h, i], vv)):
                    assert np.all(np.abs(g_ - w_) <= moved_row_tol(w_)), "moved-back row, step %d" % s
        n_moved += moved
    assert n_moved >= 5
