"""Parity of the stage-1 variants (tq_stage1_encode / tq_stage1_decode,
CUDA through the C ABI) with the oracle on the same fp32 rotated inputs.

- PolarQuant: every decision is an fp32 comparison formed identically on
  both sides, so codes and the fp16 radius bits are bit-exact; the GPU
  reconstruction (fp32 products of tabulated cosines) is within 1e-5 |x| of
  the oracle's fp64 one.
- MSE-only b bits: codes bit-exact wherever the stored fp16 norms agree (the
  GPU's fp32 norm may round to the other fp16 neighbour at a rounding
  midpoint); reconstruction within 1e-6 |x|.
- Distortion (relative MSE, inner-product error against random unit
  queries) of GPU encode -> decode equals the oracle's within 1e-3 relative.
"""
import numpy as np
import pytest

import compressed_kv_decode_b200 as tq

from test_gpu_compress import fp16_midpoint_close

pytestmark = pytest.mark.gpu

_ctx = {}


def ctx_for(d):
    if d not in _ctx:
        _ctx[d] = tq.Context(d, 0)
    return _ctx[d]


def inputs(d, N, seed):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((N, d)).astype(np.float32)
    x[0] = 0.0                      # zero vector
    x[1, :6] = 0.0                  # zero pairs
    x[2, 0], x[2, 1] = 0.0, 1.25    # pairs on the axes
    x[2, 2], x[2, 3] = -3.0, 0.0
    x[2, 4], x[2, 5] = 0.0, -0.5
    x[3] *= 1e-3                    # small and large scales
    x[4] *= 300.0
    return x


def gpu_roundtrip(ctx, kind, b1, b2, x):
    import torch
    N, d = x.shape
    cb = tq.tq_stage1_code_bytes(ctx.handle, kind, b1, b2)
    xt = torch.from_numpy(x).cuda()
    codes = torch.zeros((N, cb), dtype=torch.uint8, device="cuda")
    norms = torch.zeros(N, dtype=torch.int16, device="cuda")
    xh = torch.empty((N, d), dtype=torch.float32, device="cuda")
    tq.tq_stage1_encode(ctx.handle, kind, b1, b2, xt, codes, norms)
    tq.tq_stage1_decode(ctx.handle, kind, b1, b2, codes, norms, xh)
    torch.cuda.synchronize()
    return (codes.cpu().numpy(), norms.cpu().numpy().view(np.uint16),
            xh.cpu().numpy().astype(np.float64))


def distortion(x, xh, seed=9):
    x = x.astype(np.float64)
    rel = np.sum((xh - x) ** 2, axis=1) / np.maximum(np.sum(x * x, axis=1), 1e-300)
    q = np.random.default_rng(seed).standard_normal((64, x.shape[1]))
    q /= np.linalg.norm(q, axis=1, keepdims=True)
    ip = (xh - x) @ q.T
    return float(np.mean(rel[np.sum(x * x, axis=1) > 0])), float(np.sqrt(np.mean(ip ** 2)))


@pytest.mark.parametrize("d,b1,b2", [(128, 4, 2), (64, 4, 2), (128, 3, 3), (128, 5, 1),
                                     (64, 2, 2), (128, 2, 1), (128, 5, 3), (64, 5, 3),
                                     (64, 3, 1)])
def test_polar_bit_exact(O, d, b1, b2):
    ctx = ctx_for(d)
    x = inputs(d, 2000, d + 10 * b1 + b2)
    codes, rad, xh = gpu_roundtrip(ctx, tq.TQ_STAGE1_POLAR, b1, b2, x)
    oc, orad = O.polar_encode(x, b1, b2)
    assert np.array_equal(codes, oc)
    assert np.array_equal(rad, orad)
    ref = O.polar_decode(oc, orad, d, b1, b2)
    scale = np.maximum(np.linalg.norm(ref, axis=1, keepdims=True), 1e-30)
    assert np.all(np.abs(xh - ref) <= 1e-5 * scale)
    assert not xh[0].any()
    g, o = distortion(x, xh), distortion(x, ref)
    assert abs(g[0] - o[0]) <= 1e-3 * o[0] and abs(g[1] - o[1]) <= 1e-3 * o[1]


@pytest.mark.parametrize("d,bits", [(128, 2), (128, 3), (128, 4), (64, 2), (64, 3), (64, 4)])
def test_mse_codes_and_reconstruction(O, d, bits):
    ctx = ctx_for(d)
    P = O.Params(d, seed=0)
    x = inputs(d, 2000, 100 + d + bits)
    codes, norms, xh = gpu_roundtrip(ctx, tq.TQ_STAGE1_MSE, bits, 0, x)
    oc, on, cpos = O.mse_encode(P, x.astype(np.float64), bits)
    gn = np.array([O.f16_value(int(v)) for v in norms])
    same_n = gn == on
    assert np.all(same_n | fp16_midpoint_close(np.linalg.norm(x.astype(np.float64), axis=1)))
    assert np.array_equal(codes[same_n], oc[same_n])
    ref = O.mse_decode(oc, on, cpos, d, bits)
    scale = np.maximum(np.linalg.norm(ref, axis=1, keepdims=True), 1e-30)
    assert np.all(np.abs(xh - ref)[same_n] <= 1e-6 * scale[same_n])
    assert not xh[0].any()
    g, o = distortion(x, xh), distortion(x, ref)
    assert abs(g[0] - o[0]) <= 1e-3 * o[0] and abs(g[1] - o[1]) <= 1e-3 * o[1]


def test_unsupported_bits_rejected():
    ctx = ctx_for(128)
    assert tq.tq_stage1_code_bytes(ctx.handle, tq.TQ_STAGE1_POLAR, 6, 2) == 0
    assert tq.tq_stage1_code_bytes(ctx.handle, tq.TQ_STAGE1_MSE, 5, 0) == 0
    assert tq.tq_stage1_code_bytes(ctx.handle, tq.TQ_STAGE1_POLAR, 4, 2) == 48
    assert tq.tq_stage1_code_bytes(ctx.handle, tq.TQ_STAGE1_MSE, 3, 0) == 48


def test_empty_batch_and_unsupported_calls():
    import torch
    ctx = ctx_for(128)
    x = torch.zeros((0, 128), device="cuda")
    codes = torch.zeros((0, 48), dtype=torch.uint8, device="cuda")
    norms = torch.zeros(0, dtype=torch.int16, device="cuda")
    tq.tq_stage1_encode(ctx.handle, tq.TQ_STAGE1_POLAR, 4, 2, x, codes, norms)  # N = 0: no-op
    x1 = torch.zeros((1, 128), device="cuda")
    c1 = torch.zeros((1, 64), dtype=torch.uint8, device="cuda")
    n1 = torch.zeros(1, dtype=torch.int16, device="cuda")
    with pytest.raises(tq.TQError):
        tq.tq_stage1_encode(ctx.handle, tq.TQ_STAGE1_POLAR, 6, 2, x1, c1, n1)
    with pytest.raises(tq.TQError):
        tq.tq_stage1_encode(ctx.handle, tq.TQ_STAGE1_MSE, 1, 0, x1, c1, n1)
    torch.cuda.synchronize()
    assert tq.tq_get_error(ctx.handle) == tq.TQ_OK
