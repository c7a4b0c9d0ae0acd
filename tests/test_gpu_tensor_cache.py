"""Parity of tq_tensor_cache_step (fp16 ring L1 with exact attention, fp32
outer-product L2 fed by the ring's evictions, gated fusion) with the
oracle's Tensor Cache, step by step, through the C ABI.

Per step: ring start and length exact, outputs within 2e-3 + 1e-2 |ref|
(the decode tolerance; the read q A is fp32 against fp64).  At the end the
ring holds exactly the oracle's tokens and A agrees to 1e-5 of its largest
entry."""
import math

import numpy as np
import pytest

import compressed_kv_decode_b200 as tq
from oracle.tensor_cache import TensorCache

from decode_cases import assert_close

pytestmark = pytest.mark.gpu

_ctx = {}


def ctx_for(d):
    if d not in _ctx:
        _ctx[d] = tq.Context(d, 0)
    return _ctx[d]


def f16(a):
    return np.float16(a).astype(np.float64)


@pytest.mark.parametrize("d,G,W,qdt", [(128, 4, 16, "bfloat16"), (64, 8, 9, "float16"),
                                       (128, 1, 33, "float32")])
def test_tensor_cache_steps_match_oracle(O, d, G, W, qdt):
    import torch
    P = O.Params(d, seed=0)
    ctx = ctx_for(d)
    B, Hkv, steps = 2, 2, 45
    Hq = G * Hkv
    rng = np.random.default_rng(d + G + W)
    lam = rng.uniform(0.85, 0.99, Hkv)
    eta = rng.uniform(0.05, 0.3, Hkv)
    gate = rng.uniform(-2.0, 2.0, Hq)
    gate[0] = -30.0  # a nearly shut gate
    A0 = rng.standard_normal((B, Hkv, d, d)) * 0.1
    A0 = A0.astype(np.float32).astype(np.float64)
    tc = TensorCache(P, B, Hkv, W, lam.astype(np.float32), eta.astype(np.float32),
                     gate.astype(np.float32), A=A0)
    # sequence 1 starts with a full ring at start 5, sequence 0 empty
    ring_k = np.full((B, Hkv, W, d), np.nan)
    ring_v = np.full((B, Hkv, W, d), np.nan)
    start, length = [0, 5], [0, W]
    for h in range(Hkv):
        for i in range(W):
            k, v = f16(rng.standard_normal(d)), f16(rng.standard_normal(d))
            ring_k[1, h, (5 + i) % W], ring_v[1, h, (5 + i) % W] = k, v
            tc.ring[1][h].append((k, v))
    dev = "cuda"
    kr = torch.from_numpy(ring_k).half().to(dev)
    vr = torch.from_numpy(ring_v).half().to(dev)
    rs = torch.tensor(start, dtype=torch.int32, device=dev)
    rl = torch.tensor(length, dtype=torch.int32, device=dev)
    A = torch.from_numpy(A0).float().to(dev)
    lam_t = torch.from_numpy(lam).float().to(dev)
    eta_t = torch.from_numpy(eta).float().to(dev)
    gate_t = torch.from_numpy(gate).float().to(dev)
    out = torch.empty((B, Hq, d), dtype=torch.float32, device=dev)
    ws = torch.empty(tq.tq_tensor_cache_workspace_bytes(ctx.handle, B, Hq, Hkv, W),
                     dtype=torch.uint8, device=dev)
    exp_start = list(start)
    for s in range(steps):
        k_new, v_new = f16(rng.standard_normal((B, Hkv, d))), f16(rng.standard_normal((B, Hkv, d)))
        q = rng.standard_normal((B, Hq, d))
        qt = torch.from_numpy(q).to(getattr(torch, qdt))
        qv = qt.double().numpy()
        full = [len(tc.ring[b][0]) == W for b in range(B)]
        y, _, _ = tc.step(qv, k_new, v_new, 1.0 / math.sqrt(d))
        tq.tq_tensor_cache_step(ctx.handle, qt.to(dev), torch.from_numpy(k_new).half().to(dev),
                                torch.from_numpy(v_new).half().to(dev), kr, vr, rs, rl, A,
                                lam_t, eta_t, gate_t, out, ws, Hkv)
        torch.cuda.synchronize()
        assert tq.tq_get_error(ctx.handle) == tq.TQ_OK
        for b in range(B):
            if full[b]:
                exp_start[b] = (exp_start[b] + 1) % W
        assert np.array_equal(rs.cpu().numpy(), exp_start)
        assert np.array_equal(rl.cpu().numpy(), [len(tc.ring[b][0]) for b in range(B)])
        got = out.cpu().numpy().astype(np.float64)
        for b in range(B):
            assert_close(got[b], y[b], what="step %d sequence %d" % (s, b))
    kg = kr.float().cpu().numpy()
    for b in range(B):
        for h in range(Hkv):
            for i, (k, _) in enumerate(tc.ring[b][h]):
                assert np.array_equal(kg[b, h, (exp_start[b] + i) % W], k)
    Ag = A.cpu().numpy().astype(np.float64)
    assert np.abs(Ag - tc.A).max() <= 1e-5 * np.abs(tc.A).max()


def test_invalid_ring_state_is_reported_and_reset(O):
    import torch
    d, Hkv, G, W = 64, 1, 2, 4
    ctx = ctx_for(d)
    dev = "cuda"
    B = 2
    kr = torch.zeros((B, Hkv, W, d), device=dev).half()
    rs = torch.tensor([0, 0], dtype=torch.int32, device=dev)
    rl = torch.tensor([W + 3, 1], dtype=torch.int32, device=dev)  # sequence 0 is corrupt
    A = torch.zeros((B, Hkv, d, d), device=dev)
    lam = torch.ones(Hkv, device=dev)
    eta = torch.ones(Hkv, device=dev)
    gate = torch.zeros(Hkv * G, device=dev)
    out = torch.empty((B, Hkv * G, d), device=dev)
    ws = torch.empty(tq.tq_tensor_cache_workspace_bytes(ctx.handle, B, Hkv * G, Hkv, W),
                     dtype=torch.uint8, device=dev)
    q = torch.randn((B, Hkv * G, d), device=dev)
    kn = torch.randn((B, Hkv, d), device=dev).half()
    tq.tq_tensor_cache_step(ctx.handle, q, kn, kn, kr, kr.clone(), rs, rl, A, lam, eta, gate, out,
                            ws, Hkv)
    torch.cuda.synchronize()
    assert tq.tq_get_error(ctx.handle) == tq.TQ_ERR_CAPACITY
    assert rl.cpu().tolist() == [0, 2] and rs.cpu().tolist() == [0, 0]
    assert torch.isfinite(out).all() and not out[0].any()
