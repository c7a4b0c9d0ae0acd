"""Parity of tq_monarch_step (append to the hot ring, gated attention,
eviction of the oldest hot tokens into cold pages) with the oracle's Monarch
cache, step by step, through the C ABI.

Both sides start from the same state (cold pages written by the oracle's
packer, the same hot tokens) and take the same seeded tokens and queries.
Per step: ring indices and lengths exact; gate decisions equal except for
heads whose raw hot maximum lies within GAP of the threshold (then the GPU's
decision is checked against the oracle's result for that decision);
attention within 2e-3 + 1e-2 |ref|.  Each side compresses the evicted tokens
itself, and a code or sketch bit may legitimately differ where the rotated
coordinate (or S r) lies within the fp16 rotation's error bound of a decision
boundary; one such bit of a heavily weighted cold token moves the output by
more than the attention tolerance.  So a head that read its cold tokens is
compared only while every record its group evicted so far is identical on
both sides (heads with the gate shut are always compared), and at the end
every evicted record must match the oracle's encoding up to those boundary
cases.  The hot ring must hold exactly the oracle's hot tokens."""
import math

import numpy as np
import pytest

import compressed_kv_decode_b200 as tq
from compressed_kv_decode_b200 import workloads as W
from oracle.monarch import MonarchCache

from decode_cases import assert_close
from test_gpu_compress import compare_records

pytestmark = pytest.mark.gpu

GAP = 2e-3
_ctx = {}


def ctx_for(d):
    if d not in _ctx:
        _ctx[d] = tq.Context(d, 0)
    return _ctx[d]


def f16(a):
    return np.float16(a).astype(np.float64)


def run_case(O, d, G, window, E, steps, mode, seed, cold0=(150, 0), hot0=None, starts=None):
    import torch
    P = O.Params(d, seed=0)
    ctx = ctx_for(d)
    B, Hkv = 2, 2
    Hq = G * Hkv
    W_max = window + E
    hot0 = hot0 if hot0 is not None else [window + E - 4, 5]
    starts = starts if starts is not None else [W_max - 3, 0]
    rng = np.random.default_rng(seed)
    max_pages = (max(cold0) + steps + 127) // 128 + 1
    table, n_pages = W.random_page_table(seed + 1, B, Hkv, max_pages, spare=2)
    nbytes, offs = O.page_layout(d, d, True)
    pool = np.zeros(n_pages * nbytes, np.uint8)
    hot_k = [[[] for _ in range(Hkv)] for _ in range(B)]
    hot_v = [[[] for _ in range(Hkv)] for _ in range(B)]
    seq = [[None for _ in range(Hkv)] for _ in range(B)]  # every token of (b, h), in order
    for b in range(B):
        for h in range(Hkv):
            n = cold0[b] + hot0[b]
            K, V = f16(rng.standard_normal((n, d))), f16(rng.standard_normal((n, d)))
            if cold0[b]:
                kr, vr = O.encode(P, K[:cold0[b]], True), O.encode(P, V[:cold0[b]], False)
                rec = dict(sign=kr["sign"], mag=kr["mag"], qbits=kr["qbits"], n=kr["n"],
                           gamma=kr["gamma"], vcode=vr["vcode"], vn=vr["vn"])
                t = np.arange(cold0[b])
                O.pack(pool, nbytes, d, d, True, table[b, h, t // 128], t % 128, rec)
            hot_k[b][h] = list(K[cold0[b]:])
            hot_v[b][h] = list(V[cold0[b]:])
            seq[b][h] = [list(K), list(V)]
    cache = MonarchCache(P, B, Hkv, window, E, table, cold_len=cold0, pool=pool, hot_k=hot_k,
                         hot_v=hot_v)
    # the GPU ring: logical hot token i of sequence b at slot (start + i) mod W_max
    kr_ = np.full((B, Hkv, W_max, d), np.nan)
    vr_ = np.full((B, Hkv, W_max, d), np.nan)
    for b in range(B):
        for h in range(Hkv):
            for i in range(hot0[b]):
                kr_[b, h, (starts[b] + i) % W_max] = hot_k[b][h][i]
                vr_[b, h, (starts[b] + i) % W_max] = hot_v[b][h][i]
    dev = "cuda"
    k_hot = torch.from_numpy(kr_).half().to(dev)
    v_hot = torch.from_numpy(vr_).half().to(dev)
    hs = torch.tensor(starts, dtype=torch.int32, device=dev)
    hl = torch.tensor(hot0, dtype=torch.int32, device=dev)
    cl = torch.tensor(cold0, dtype=torch.int32, device=dev)
    gpool = torch.from_numpy(pool.reshape(n_pages, nbytes).copy()).to(dev)
    tbl = torch.from_numpy(table).to(dev)
    out = torch.empty((B, Hq, d), dtype=torch.float32, device=dev)
    used = torch.empty((B, Hq), dtype=torch.int32, device=dev)
    ws = torch.empty(tq.tq_monarch_workspace_bytes(ctx.handle, B, Hq, Hkv, max_pages, W_max, E),
                     dtype=torch.uint8, device=dev)
    scale = 1.0 / math.sqrt(d)
    exp_start = list(starts)
    thr = None
    n_near = 0
    diverged = set()  # (b, h) groups whose evicted records differ somewhere
    n_cmp = n_skip = 0
    for s in range(steps):
        k_new, v_new = f16(rng.standard_normal((B, Hkv, d))), f16(rng.standard_normal((B, Hkv, d)))
        q = rng.standard_normal((B, Hq, d))
        cache.append(k_new, v_new)
        for b in range(B):
            for h in range(Hkv):
                seq[b][h][0].append(k_new[b, h])
                seq[b][h][1].append(v_new[b, h])
        kh, _ = cache._hot_arrays()
        hmax = np.array([[(kh[b, hq // G, :cache.hot_len(b)] @ q[b, hq]).max()
                          for hq in range(Hq)] for b in range(B)])
        if thr is None:
            thr = {"open": np.inf, "shut": -np.inf, "mid": float(np.median(hmax))}[mode]
        ref, opened = cache.attend(q, scale, thr)
        alt_open, _ = cache.attend(q, scale, np.inf)
        alt_shut, _ = cache.attend(q, scale, -np.inf)
        moved = cache.evict()
        tq.tq_monarch_step(ctx.handle, torch.from_numpy(q).float().to(dev),
                           torch.from_numpy(k_new).half().to(dev),
                           torch.from_numpy(v_new).half().to(dev), k_hot, v_hot, hs, hl, gpool,
                           tbl, cl, thr, window, E, out, ws, Hkv, cold_used=used)
        torch.cuda.synchronize()
        assert tq.tq_get_error(ctx.handle) == tq.TQ_OK
        got, gu = out.cpu().numpy().astype(np.float64), used.cpu().numpy()
        for b in range(B):
            exp_start[b] = (exp_start[b] + int(moved[b])) % W_max
        assert np.array_equal(hl.cpu().numpy(), [cache.hot_len(b) for b in range(B)])
        assert np.array_equal(cl.cpu().numpy(), cache.cold_len)
        assert np.array_equal(hs.cpu().numpy(), exp_start)
        for b in range(B):
            for hq in range(Hq):
                if gu[b, hq] == opened[b, hq]:
                    r = ref[b, hq]
                else:
                    assert abs(hmax[b, hq] - thr) < GAP, "gate differs away from the threshold"
                    n_near += 1
                    r = alt_open[b, hq] if gu[b, hq] else alt_shut[b, hq]
                if gu[b, hq] and (b, hq // G) in diverged:
                    n_skip += 1
                    continue
                n_cmp += 1
                assert_close(got[b, hq], r, what="step %d head %s" % (s, (b, hq)))
        # records this step evicted: identical on both sides, or the group is
        # compared no further where it reads cold tokens
        if moved.any():
            gp_now = gpool.cpu().numpy().reshape(-1)
            for b in range(B):
                if not moved[b]:
                    continue
                t = np.arange(int(cache.cold_len[b]) - int(moved[b]), int(cache.cold_len[b]))
                for h in range(Hkv):
                    a = O.unpack(gp_now, nbytes, d, d, True, table[b, h, t // 128], t % 128)
                    o = O.unpack(cache.pool, nbytes, d, d, True, table[b, h, t // 128], t % 128)
                    if any(not np.array_equal(a[key], o[key]) for key in o):
                        diverged.add((b, h))
    # the ring holds the oracle's hot tokens; evicted records match the oracle's encoding
    kg = k_hot.float().cpu().numpy()
    for b in range(B):
        for h in range(Hkv):
            for i in range(cache.hot_len(b)):
                assert np.array_equal(kg[b, h, (exp_start[b] + i) % W_max], cache.hot[b][h][i][0])
    gp = gpool.cpu().numpy().reshape(-1)
    eps = 2.0 ** -11  # fp16 input: unit roundoff of the lo part of Pi
    for b in range(B):
        c1 = int(cache.cold_len[b])
        if c1 == cold0[b]:
            continue
        t = np.arange(cold0[b], c1)
        for h in range(Hkv):
            got = O.unpack(gp, nbytes, d, d, True, table[b, h, t // 128], t % 128)
            for isk, x in ((True, np.stack(seq[b][h][0][cold0[b]:c1])),
                           (False, np.stack(seq[b][h][1][cold0[b]:c1]))):
                rec = O.encode(P, x, isk)
                err = (np.abs(x) @ np.abs(P.pi32).T) * (eps * eps * 2 + 64 * 2.0 ** -24)
                compare_records(O, P, x, rec, got, isk, err)
    assert n_cmp >= 2 * n_skip, "too few strict comparisons (%d of %d)" % (n_cmp, n_cmp + n_skip)
    return cache, n_near


@pytest.mark.parametrize("d,G,window,E,mode", [(64, 8, 20, 8, "open"), (128, 4, 24, 1, "mid"),
                                               (64, 2, 16, 16, "shut"), (128, 4, 30, 128, "mid")])
def test_monarch_steps_match_oracle(O, d, G, window, E, mode):
    steps = 40 if E < 128 else 140
    run_case(O, d, G, window, E, steps, mode, seed=d + G + E)


def test_full_ring_is_reported_and_token_dropped(O):
    """A ring already holding W_max tokens cannot take the step's token: the
    append reports TQ_ERR_CAPACITY and leaves the ring and lengths as they
    were; the rest of the step still runs on the stored state."""
    import torch
    d, G, window, E = 64, 2, 6, 2
    ctx = ctx_for(d)
    B, Hkv = 1, 1
    Hq, W_max = G * Hkv, window + E
    dev = "cuda"
    k_hot = torch.randn((B, Hkv, W_max, d), device=dev).half()
    v_hot = torch.randn((B, Hkv, W_max, d), device=dev).half()
    k0 = k_hot.clone()
    hs = torch.tensor([3], dtype=torch.int32, device=dev)
    hl = torch.tensor([W_max], dtype=torch.int32, device=dev)
    cl = torch.zeros(1, dtype=torch.int32, device=dev)
    nbytes = ctx.page_bytes(True)
    pool = torch.zeros((4, nbytes), dtype=torch.uint8, device=dev)
    tbl = torch.arange(2, dtype=torch.int32, device=dev).view(1, 1, 2)
    out = torch.empty((B, Hq, d), device=dev)
    ws = torch.empty(tq.tq_monarch_workspace_bytes(ctx.handle, B, Hq, Hkv, 2, W_max, E),
                     dtype=torch.uint8, device=dev)
    q = torch.randn((B, Hq, d), device=dev)
    kn = torch.randn((B, Hkv, d), device=dev).half()
    tq.tq_monarch_step(ctx.handle, q, kn, kn, k_hot, v_hot, hs, hl, pool, tbl, cl, float("inf"),
                       window, E, out, ws, Hkv)
    torch.cuda.synchronize()
    assert tq.tq_get_error(ctx.handle) == tq.TQ_ERR_CAPACITY
    # the stored window was full: the step then evicted its E oldest tokens
    assert int(hl.item()) == W_max - E and int(cl.item()) == E
    assert int(hs.item()) == (3 + E) % W_max
    assert torch.equal(k_hot, k0)  # the dropped token was not written
    assert torch.isfinite(out).all()


def test_invalid_window_arguments_rejected():
    import torch
    ctx = ctx_for(64)
    dev = "cuda"
    B, Hkv, d = 1, 1, 64
    k_hot = torch.zeros((B, Hkv, 8, d), device=dev).half()
    z = torch.zeros(1, dtype=torch.int32, device=dev)
    pool = torch.zeros((2, ctx.page_bytes(True)), dtype=torch.uint8, device=dev)
    tbl = torch.zeros((1, 1, 2), dtype=torch.int32, device=dev)
    out = torch.empty((B, 1, d), device=dev)
    ws = torch.empty(1 << 20, dtype=torch.uint8, device=dev)
    q = torch.zeros((B, 1, d), device=dev)
    with pytest.raises(tq.TQError):  # window + E > W_max
        tq.tq_monarch_step(ctx.handle, q, None, None, k_hot, k_hot, z, z, pool, tbl, z,
                           float("inf"), 7, 2, out, ws, Hkv)
    with pytest.raises(tq.TQError):  # E = 0
        tq.tq_monarch_step(ctx.handle, q, None, None, k_hot, k_hot, z, z, pool, tbl, z,
                           float("inf"), 4, 0, out, ws, Hkv)
