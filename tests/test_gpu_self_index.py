"""Parity of the Self-Indexing index build and LUT scores (CUDA, through the
C ABI) with the oracle's Self-Indexing form.

- Build: the channel mean within 1e-4; the sign-pattern codes equal wherever
  every centred coordinate of the group is farther than 1e-3 from zero (the
  GPU's fp32 mean may put a near-zero coordinate on the other side); the
  centroids within 1e-4 for every (group, index) whose token count agrees.
- Scores: given the oracle's index, every token score within 1e-4 +
  1e-5 |score| of the oracle's table lookup."""
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


@pytest.mark.parametrize("d,T", [(128, 1000), (64, 777)])
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
