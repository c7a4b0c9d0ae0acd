"""Parity of the Self-Indexing index build and LUT scores (CUDA, through the
C ABI) with the oracle's Self-Indexing form.

- Build: the channel mean within 1e-4; the sign-pattern codes equal wherever
  every centred coordinate of the group is farther than 1e-3 from zero (the
  GPU's fp32 mean may put a near-zero coordinate on the other side); the
  centroids within 1e-4 for every (group, index) whose token count agrees.
- Scores: given the oracle's index, every token score within 1e-4 +
  1e-5 |score| of the oracle's table lookup.
- Selection: bit-exact with the oracle's top-k on the same fp32 scores
  (heavy ties, -0.0 beside +0.0, top_k above the candidates, T at or below
  the sinks).
- Sparse attention: given the oracle's picked positions, within 2e-4 +
  1e-3 |out| of the oracle's exact softmax over sinks + picked tokens.
- The whole chain on the GPU (build, scores, select, attend) at 7.5 % of
  T = 8192: the picked set is a valid top-k of the GPU's own scores (all
  distinct, sorted, after the sinks, none scored below an unpicked one) and
  the attention over it matches the oracle's."""
import numpy as np
import pytest

import compressed_kv_decode_b200 as tq
from oracle import self_index as S

pytestmark = pytest.mark.gpu

_ctx = {}


def ctx_for(d):
    if d not in _ctx:
        _ctx[d] = tq.Context(d, 0)
    return _ctx[d]


def keys(d, B, Hkv, T, seed):
    rng = np.random.default_rng(seed)
    scale = rng.uniform(0.5, 3.0, (Hkv, d))
    off = rng.standard_normal((Hkv, d))
    K = rng.standard_normal((B, Hkv, T, d)) * scale[None, :, None] + off[None, :, None]
    return np.float16(K).astype(np.float64)


@pytest.mark.parametrize("d,T", [(128, 1000), (64, 777), (128, 20000), (64, 5)])
def test_build_matches_oracle(d, T):
    import torch
    ctx = ctx_for(d)
    B, Hkv = 2, 3
    K = keys(d, B, Hkv, T, d + T)
    kt = torch.from_numpy(K).half().cuda()
    mu = torch.empty((B, Hkv, d), device="cuda")
    codes = torch.empty((B, Hkv, T, d // 4), dtype=torch.uint8, device="cuda")
    cent = torch.empty((B, Hkv, d // 4, 16, 4), device="cuda")
    tq.tq_self_index_build(ctx.handle, kt, mu, codes, cent)
    torch.cuda.synchronize()
    assert tq.tq_get_error(ctx.handle) == tq.TQ_OK
    gm, gc, gz = mu.cpu().numpy(), codes.cpu().numpy(), cent.cpu().numpy()
    for b in range(B):
        for h in range(Hkv):
            om, oc, oz = S.build_index(K[b, h])
            assert np.abs(gm[b, h] - om).max() <= 1e-4
            centred = np.abs((K[b, h] - om).reshape(T, d // 4, 4)).min(axis=2)
            clear = centred > 1e-3
            assert np.array_equal(gc[b, h][clear], oc[clear])
            for g in range(d // 4):
                n_gpu = np.bincount(gc[b, h, :, g], minlength=16)
                n_or = np.bincount(oc[:, g], minlength=16)
                same = n_gpu == n_or
                assert np.abs(gz[b, h, g][same] - oz[g][same]).max() <= 1e-4


@pytest.mark.parametrize("d,G,qdt", [(128, 4, "bfloat16"), (64, 8, "float32")])
def test_scores_match_oracle(d, G, qdt):
    import torch
    ctx = ctx_for(d)
    B, Hkv, T = 2, 2, 1234
    Hq = G * Hkv
    K = keys(d, B, Hkv, T, 7 * d + G)
    codes = np.empty((B, Hkv, T, d // 4), np.uint8)
    cent = np.empty((B, Hkv, d // 4, 16, 4), np.float32)
    for b in range(B):
        for h in range(Hkv):
            _, codes[b, h], c = S.build_index(K[b, h])
            cent[b, h] = c.astype(np.float32)
    q = torch.randn((B, Hq, d), generator=torch.Generator().manual_seed(5)).to(getattr(torch, qdt))
    scores = torch.empty((B, Hq, T), device="cuda")
    tq.tq_self_index_scores(ctx.handle, q.cuda(), torch.from_numpy(codes).cuda(),
                            torch.from_numpy(cent).cuda(), scores, Hkv)
    torch.cuda.synchronize()
    got = scores.cpu().numpy().astype(np.float64)
    qv = q.double().numpy()
    for b in range(B):
        for hq in range(Hq):
            ref = S.lut_scores(qv[b, hq], codes[b, hq // G], cent[b, hq // G].astype(np.float64))
            assert np.all(np.abs(got[b, hq] - ref) <= 1e-4 + 1e-5 * np.abs(ref))


def _scores_rows(kind, rows, T, seed):
    rng = np.random.default_rng(seed)
    if kind == "normal":
        return rng.standard_normal((rows, T)).astype(np.float32)
    if kind == "ties":
        return rng.integers(-3, 4, (rows, T)).astype(np.float32)
    if kind == "nan":  # NaN scores rank below -inf, ties among them to the lower position
        s = rng.standard_normal((rows, T)).astype(np.float32)
        s[rng.random((rows, T)) < 0.6] = np.nan
        s[rng.random((rows, T)) < 0.05] = -np.inf
        return s
    # zeros of both signs among a few positive and negative values
    s = rng.integers(-1, 2, (rows, T)).astype(np.float32)
    neg0 = (s == 0) & (rng.random((rows, T)) < 0.5)
    s[neg0] = np.float32(-0.0)
    return s


@pytest.mark.parametrize("kind,T,n_sink,top_k", [
    ("normal", 5000, 64, 300), ("ties", 3000, 64, 1000), ("zeros", 2000, 0, 777),
    ("normal", 200, 64, 500), ("normal", 50, 64, 10), ("ties", 40000, 64, 3000),
    ("nan", 3000, 64, 1500), ("ties", 60000, 64, 5000), ("normal", 70000, 0, 4000)])
def test_select_matches_oracle(kind, T, n_sink, top_k):
    """Rows of up to 50176 candidates are staged in shared memory, longer
    ones re-read from global memory (T = 60000, 70000); rows longer than
    32768 candidates take more than one ordered pass."""
    import torch
    ctx = ctx_for(128)
    B, Hq = 2, 4
    sc = _scores_rows(kind, B * Hq, T, T + top_k)
    picked = torch.full((B, Hq, top_k), 7, dtype=torch.int32, device="cuda")
    tq.tq_self_index_select(ctx.handle, torch.from_numpy(sc).reshape(B, Hq, T).cuda(), picked,
                            n_sink=n_sink)
    torch.cuda.synchronize()
    got = picked.cpu().numpy().reshape(B * Hq, top_k)
    for r in range(B * Hq):
        ref = S.select(sc[r].astype(np.float64), top_k, n_sink)
        assert np.array_equal(got[r, :len(ref)], ref)
        assert (got[r, len(ref):] == -1).all()


def test_select_more_rows_than_sms():
    """The selection CTAs are persistent over the rows (one per SM): 320 rows."""
    import torch
    ctx = ctx_for(64)
    B, Hq, T, n_sink, top_k = 10, 32, 3000, 64, 225
    sc = _scores_rows("ties", B * Hq, T, 99)
    picked = torch.empty((B, Hq, top_k), dtype=torch.int32, device="cuda")
    tq.tq_self_index_select(ctx.handle, torch.from_numpy(sc).reshape(B, Hq, T).cuda(), picked,
                            n_sink=n_sink)
    torch.cuda.synchronize()
    got = picked.cpu().numpy().reshape(B * Hq, top_k)
    for r in range(B * Hq):
        assert np.array_equal(got[r], S.select(sc[r].astype(np.float64), top_k, n_sink))


@pytest.mark.parametrize("d,G,qdt,T,top_k", [
    (128, 4, "bfloat16", 1500, 200), (64, 8, "float32", 1000, 150),
    (128, 4, "float16", 100, 50), (128, 2, "float32", 40, 16)])
def test_attend_matches_oracle(d, G, qdt, T, top_k):
    import torch
    ctx = ctx_for(d)
    B, Hkv = 2, 2
    Hq = G * Hkv
    K = keys(d, B, Hkv, T, 3 * T + d)
    V = np.float16(np.random.default_rng(T).standard_normal((B, Hkv, T, d))).astype(np.float64)
    q = torch.randn((B, Hq, d), generator=torch.Generator().manual_seed(T)).to(getattr(torch, qdt))
    qv = q.double().numpy()
    picked = np.full((B, Hq, top_k), -1, np.int32)
    for b in range(B):
        for hq in range(Hq):
            _, codes, cent = S.build_index(K[b, hq // G])
            sel = S.select(S.lut_scores(qv[b, hq], codes, cent), top_k)
            picked[b, hq, :len(sel)] = sel
    out = torch.empty((B, Hq, d), device="cuda")
    tq.tq_self_index_attend(ctx.handle, q.cuda(), torch.from_numpy(K).half().cuda(),
                            torch.from_numpy(V).half().cuda(), torch.from_numpy(picked).cuda(),
                            out)
    torch.cuda.synchronize()
    assert tq.tq_get_error(ctx.handle) == tq.TQ_OK
    got = out.cpu().numpy().astype(np.float64)
    for b in range(B):
        for hq in range(Hq):
            sel = picked[b, hq][picked[b, hq] >= 0]
            ref = S.sparse_attention(qv[b, hq], K[b, hq // G], V[b, hq // G], sel)
            assert np.all(np.abs(got[b, hq] - ref) <= 2e-4 + 1e-3 * np.abs(ref))


def test_chain_on_the_gpu_is_a_valid_top_k():
    import torch
    d, B, Hkv, G, T = 128, 1, 2, 4, 8192
    Hq, top_k = G * Hkv, round(0.075 * T)
    ctx = ctx_for(d)
    K = keys(d, B, Hkv, T, 99)
    V = np.float16(np.random.default_rng(98).standard_normal((B, Hkv, T, d))).astype(np.float64)
    q = torch.randn((B, Hq, d), generator=torch.Generator().manual_seed(97))
    kt, vt = torch.from_numpy(K).half().cuda(), torch.from_numpy(V).half().cuda()
    mu = torch.empty((B, Hkv, d), device="cuda")
    codes = torch.empty((B, Hkv, T, d // 4), dtype=torch.uint8, device="cuda")
    cent = torch.empty((B, Hkv, d // 4, 16, 4), device="cuda")
    scores = torch.empty((B, Hq, T), device="cuda")
    picked = torch.empty((B, Hq, top_k), dtype=torch.int32, device="cuda")
    out = torch.empty((B, Hq, d), device="cuda")
    qd = q.cuda()
    tq.tq_self_index_build(ctx.handle, kt, mu, codes, cent)
    tq.tq_self_index_scores(ctx.handle, qd, codes, cent, scores, Hkv)
    tq.tq_self_index_select(ctx.handle, scores, picked)
    tq.tq_self_index_attend(ctx.handle, qd, kt, vt, picked, out)
    torch.cuda.synchronize()
    assert tq.tq_get_error(ctx.handle) == tq.TQ_OK
    sc, pk, got = scores.cpu().numpy(), picked.cpu().numpy(), out.cpu().numpy()
    qv = q.double().numpy()
    for hq in range(Hq):
        p = pk[0, hq]
        assert len(np.unique(p)) == top_k and (np.diff(p) > 0).all()
        assert p[0] >= S.N_SINK and p[-1] < T
        rest = np.setdiff1d(np.arange(S.N_SINK, T), p)
        assert sc[0, hq, p].min() >= sc[0, hq, rest].max()
        ref = S.sparse_attention(qv[0, hq], K[0, hq // G], V[0, hq // G], p)
        assert np.all(np.abs(got[0, hq] - ref) <= 2e-4 + 1e-3 * np.abs(ref))
