"""Parity of tq_compress_append (CUDA, through the C ABI) with the oracle's
encoder and packer.

Given identical fp32 rotated inputs (TQ_INPUT_ROTATED), codes are bit-exact
wherever the stored norm agrees; the norm itself (fp32 sum on the GPU, fp64
in the oracle) may differ only where |x| is within rounding of an fp16
rounding midpoint.  Sign bits of the QJL sketch (GPU: r rounded to fp16,
fp32 accumulation) may differ only where |S r| is within that error bound.
From raw bf16/fp16 inputs (rotation on the tensor cores, Pi split hi + lo)
a code may differ only where x_rot lies within the rotation's error bound of
a decision threshold."""
import math

import numpy as np
import pytest

import compressed_kv_decode_b200 as tq
from compressed_kv_decode_b200 import workloads as W

pytestmark = pytest.mark.gpu

_ctx = {}
_par = {}


def ctx_for(d):
    if d not in _ctx:
        _ctx[d] = tq.Context(d, 0)
    return _ctx[d]


def params_for(O, d):
    if d not in _par:
        _par[d] = O.Params(d, seed=0)
    return _par[d]


def gpu_append(ctx, chunks, B, Hkv, d, max_pages, with_values=True, dtype="float32",
               rotated=True, start=None):
    """Append the chunks ([(k, v)] of [B, Hkv, n, d] fp64 arrays) in order;
    returns pool (numpy), table, cold_len after."""
    import torch
    page_bytes = ctx.page_bytes(with_values)
    table, n_pages = W.random_page_table(77, B, Hkv, max_pages, spare=2)
    pool = torch.zeros((n_pages, page_bytes), dtype=torch.uint8, device="cuda")
    tbl = torch.from_numpy(table).cuda()
    cl = torch.zeros(B, dtype=torch.int32, device="cuda") if start is None else \
        torch.tensor(start, dtype=torch.int32, device="cuda")
    td = getattr(torch, dtype)
    for k, v in chunks:
        kt = torch.from_numpy(np.ascontiguousarray(k)).to(td).cuda()
        vt = torch.from_numpy(np.ascontiguousarray(v)).to(td).cuda() if (with_values and v is not None) else None
        tq.tq_compress_append(ctx.handle, kt, vt, pool, tbl, cl, rotated=rotated)
    torch.cuda.synchronize()
    return pool.cpu().numpy(), table, cl.cpu().numpy()


def unpack_seq(O, pool, table, b, h, n, d, with_values, page_bytes):
    t = np.arange(n)
    return O.unpack(pool.reshape(-1), page_bytes, d, d, with_values, table[b, h, t // 128], t % 128)


def fp16_midpoint_close(x, rel=3e-7):
    """True where x is within `rel` (relative) of a rounding midpoint of fp16."""
    x = np.abs(np.asarray(x, np.float64))
    h = x.astype(np.float16).astype(np.float64)
    up = np.nextafter(x.astype(np.float16), np.float16(np.inf)).astype(np.float64)
    dn = np.nextafter(x.astype(np.float16), np.float16(0)).astype(np.float64)
    mids = np.stack([(h + up) / 2, (h + dn) / 2])
    return np.min(np.abs(mids - x), axis=0) <= rel * np.maximum(x, 1e-30)


def compare_records(O, P, x, rec, got, is_key, xrot_err):
    """got: unpacked GPU records; rec: oracle records for the same inputs.
    xrot_err: per-element bound on |x_rot(GPU) - x_rot(oracle)| (0 for
    identical rotated inputs).  Returns counts of tolerated mismatches."""
    n_ok = got["n"] == rec["n"] if is_key else got["vn"] == rec["n"]
    norms = np.linalg.norm(rec["xrot"], axis=1) if xrot_err is None else np.linalg.norm(x, axis=1)
    assert np.all(n_ok | fp16_midpoint_close(norms)), "norm mismatch away from rounding midpoints"
    n = rec["n"][:, None]
    tpos = P.kt if is_key else P.vt
    # element decision margins: |x_rot| against the fp32 thresholds n*t, and 0
    thr = (n[..., None] * tpos[None, None, :]).astype(np.float32).astype(np.float64)
    margin = np.min(np.abs(np.abs(rec["xrot"])[..., None] - thr), axis=-1)
    margin = np.minimum(margin, np.abs(rec["xrot"]))
    near = margin <= (0 if xrot_err is None else xrot_err)
    if is_key:
        same = (got["sign"] == rec["sign"]) & (got["mag"] == rec["mag"])
    else:
        same = got["vcode"] == rec["vcode"]
    rows = n_ok[:, None]
    bad = rows & ~same & ~near
    assert not bad.any(), "%d code mismatches away from decision boundaries" % bad.sum()
    return int((rows & ~same).sum())


@pytest.mark.parametrize("d", [64, 128])
def test_bit_exact_given_rotated_inputs(O, d):
    P = params_for(O, d)
    ctx = ctx_for(d)
    B, Hkv, n = 2, 3, 300
    rng = np.random.default_rng(d)
    scales = rng.lognormal(0, 1, (Hkv, d))
    k = (rng.standard_normal((B, Hkv, n, d)) * scales[None, :, None, :]).astype(np.float32).astype(np.float64)
    v = (rng.standard_normal((B, Hkv, n, d)) * scales[None, :, None, :]).astype(np.float32).astype(np.float64)
    k[0, 0, 5] = 0.0  # a zero vector
    pool, table, cl = gpu_append(ctx, [(k, v)], B, Hkv, d, 3)
    assert np.array_equal(cl, [n, n])
    nb = ctx.page_bytes(True)
    total_sign_flips = 0
    for b in range(B):
        for h in range(Hkv):
            got = unpack_seq(O, pool, table, b, h, n, d, True, nb)
            rk = O.encode(P, k[b, h], True, rotated=True)
            rv = O.encode(P, v[b, h], False, rotated=True)
            assert compare_records(O, P, k[b, h], rk, got, True, None) == 0
            assert compare_records(O, P, v[b, h], rv, got, False, None) == 0
            rows = got["n"] == rk["n"]
            g_ok = (got["gamma"] == rk["gamma"])
            chat = np.where(rk["sign"] == 1, -1.0, 1.0) * P.kc[rk["mag"]]
            nz = rk["n"][:, None]
            r = np.where(nz > 0, rk["xrot"] / np.where(nz > 0, nz, 1) - chat, 0.0)
            assert np.all(g_ok | ~rows | fp16_midpoint_close(np.linalg.norm(r, axis=1), 2e-6))
            # sketch sign bits: allowed to differ only within the fp16(r) error bound
            pexact = r @ P.S.T
            bound = (np.abs(r) * 2.0 ** -11) @ np.abs(P.S).T + d * 2.0 ** -23 * (np.abs(r) @ np.abs(P.S).T)
            flips = (got["qbits"] != rk["qbits"]) & rows[:, None]
            assert np.all(~flips | (np.abs(pexact) <= bound)), "sign flip away from zero"
            total_sign_flips += int(flips.sum())
    assert total_sign_flips <= 0.01 * B * Hkv * n * d


@pytest.mark.parametrize("dtype", ["bfloat16", "float16"])
def test_raw_inputs_within_rotation_error(O, dtype):
    d = 128
    P = params_for(O, d)
    ctx = ctx_for(d)
    B, Hkv, n = 1, 2, 256
    scales = W.compress_scales(21, Hkv, d)
    x = np.stack([W.compress_data(22, scales, n)])  # [1, Hkv, n, d], bf16 values
    x = W.round_to(x, dtype)
    pool, table, cl = gpu_append(ctx, [(x, x)], B, Hkv, d, 2, dtype=dtype, rotated=False)
    nb = ctx.page_bytes(True)
    eps = 2.0 ** -8 if dtype == "bfloat16" else 2.0 ** -11  # unit roundoff of the lo part
    flips = 0
    for h in range(Hkv):
        got = unpack_seq(O, pool, table, 0, h, n, d, True, nb)
        rk = O.encode(P, x[0, h], True)
        rv = O.encode(P, x[0, h], False)
        # |Pi - (hi + lo)| <= eps^2 |Pi| per entry, plus fp32 accumulation
        err = (np.abs(x[0, h]) @ np.abs(P.pi32).T) * (eps * eps * 2 + 64 * 2.0 ** -24)
        flips += compare_records(O, P, x[0, h], rk, got, True, err)
        flips += compare_records(O, P, x[0, h], rv, got, False, err)
    print("code differences at decision boundaries: %d of %d" % (flips, 2 * Hkv * n * d))


def test_ragged_appends_match_one_shot(O):
    """Appends of odd lengths (pages and token pairs split across calls)
    produce the same records as the oracle's encoding of the whole sequence."""
    d = 64
    P = params_for(O, d)
    ctx = ctx_for(d)
    B, Hkv = 2, 2
    sizes = [1, 7, 128, 33, 2, 130, 1]
    n = sum(sizes)
    rng = np.random.default_rng(3)
    k = rng.standard_normal((B, Hkv, n, d)).astype(np.float32).astype(np.float64)
    v = rng.standard_normal((B, Hkv, n, d)).astype(np.float32).astype(np.float64)
    chunks, t = [], 0
    for s in sizes:
        chunks.append((k[:, :, t:t + s], v[:, :, t:t + s]))
        t += s
    pool, table, cl = gpu_append(ctx, chunks, B, Hkv, d, math.ceil(n / 128))
    assert np.array_equal(cl, [n, n])
    nb = ctx.page_bytes(True)
    for b in range(B):
        for h in range(Hkv):
            got = unpack_seq(O, pool, table, b, h, n, d, True, nb)
            rk = O.encode(P, k[b, h], True, rotated=True)
            rv = O.encode(P, v[b, h], False, rotated=True)
            assert compare_records(O, P, k[b, h], rk, got, True, None) == 0
            assert compare_records(O, P, v[b, h], rv, got, False, None) == 0


def test_keys_only_pages(O):
    d = 128
    P = params_for(O, d)
    ctx = ctx_for(d)
    rng = np.random.default_rng(4)
    k = rng.standard_normal((1, 1, 200, d)).astype(np.float32).astype(np.float64)
    pool, table, cl = gpu_append(ctx, [(k, None)], 1, 1, d, 2, with_values=False)
    got = unpack_seq(O, pool, table, 0, 0, 200, d, False, ctx.page_bytes(False))
    rk = O.encode(P, k[0, 0], True, rotated=True)
    assert compare_records(O, P, k[0, 0], rk, got, True, None) == 0


def check_sketch_raw(P, rk, got, err):
    """Residual norm and sketch sign bits of raw-input records against the
    oracle's, on rows whose norm and codes match: the GPU residual differs
    from the oracle's by the rotation error err/n plus fp16 rounding, so
    gamma may differ by that much and a sign bit may flip only where
    |S r| is within the error that carries through S."""
    d = P.d
    nz = rk["n"][:, None]
    rows = (got["n"] == rk["n"]) & np.all((got["sign"] == rk["sign"]) & (got["mag"] == rk["mag"]), axis=1)
    rows &= rk["n"] > 0
    chat = np.where(rk["sign"] == 1, -1.0, 1.0) * P.kc[rk["mag"]]
    r = np.where(nz > 0, rk["xrot"] / np.where(nz > 0, nz, 1) - chat, 0.0)
    dr = err / np.where(nz > 0, nz, 1)  # per-element bound on the residual's rotation error
    gam = np.linalg.norm(r, axis=1)
    gbound = gam * 2.0 ** -10 + np.linalg.norm(dr, axis=1) + 1e-12
    assert np.all(~rows | (np.abs(got["gamma"] - rk["gamma"]) <= gbound)), "residual norm"
    pexact = r @ P.S.T
    bound = ((dr + np.abs(r) * 2.0 ** -11) @ np.abs(P.S).T) + d * 2.0 ** -23 * (np.abs(r) @ np.abs(P.S).T)
    flips = (got["qbits"] != rk["qbits"]) & rows[:, None]
    assert np.all(~flips | (np.abs(pexact) <= bound)), "sketch sign flip away from zero"
    return int(flips.sum())


@pytest.mark.parametrize("dtype", ["bfloat16", "float16"])
def test_raw_keys_only_many_tiles(O, dtype):
    """Keys-only appends of raw 16-bit inputs (the software-pipelined tensor-
    core path): 4 x 8 sequences of 2050 tokens, several page tiles per CTA, a
    partial last page; records match the oracle within the rotation error."""
    d = 128
    P = params_for(O, d)
    ctx = ctx_for(d)
    B, Hkv, n = 4, 8, 2050
    scales = W.compress_scales(21, Hkv, d)
    x = np.stack([W.compress_data(22 + b, scales, n) for b in range(B)])  # [B, Hkv, n, d]
    x = W.round_to(x, dtype)
    x[0, 0, 5] = 0.0    # zero vectors: all codes, norms and signs 0
    x[3, 7, 2049] = 0.0
    pool, table, cl = gpu_append(ctx, [(x, None)], B, Hkv, d, math.ceil(n / 128), with_values=False,
                                 dtype=dtype, rotated=False)
    assert np.array_equal(cl, [n] * B)
    nb = ctx.page_bytes(False)
    eps = 2.0 ** -8 if dtype == "bfloat16" else 2.0 ** -11
    flips = sflips = 0
    for b in range(B):
        for h in range(Hkv):
            got = unpack_seq(O, pool, table, b, h, n, d, False, nb)
            rk = O.encode(P, x[b, h], True)
            err = (np.abs(x[b, h]) @ np.abs(P.pi32).T) * (eps * eps * 2 + 64 * 2.0 ** -24)
            flips += compare_records(O, P, x[b, h], rk, got, True, err)
            sflips += check_sketch_raw(P, rk, got, err)
    for b, h, t in ((0, 0, 5), (3, 7, 2049)):
        got = unpack_seq(O, pool, table, b, h, n, d, False, nb)
        for f in ("sign", "mag", "qbits", "n", "gamma"):
            assert not np.any(got[f][t]), f
    assert sflips <= 0.01 * B * Hkv * n * d
    print("code differences at decision boundaries: %d, sketch sign flips near zero: %d, of %d"
          % (flips, sflips, B * Hkv * n * d))


def test_raw_keys_only_ragged_appends(O):
    """Keys-only raw appends of odd lengths split pages across calls; every
    record matches the oracle's encoding of the whole sequence within the
    rotation error."""
    d = 64
    P = params_for(O, d)
    ctx = ctx_for(d)
    B, Hkv = 2, 3
    sizes = [5, 128, 77, 300, 1, 250]
    n = sum(sizes)
    scales = W.compress_scales(23, Hkv, d)
    x = W.round_to(np.stack([W.compress_data(24 + b, scales, n) for b in range(B)]), "bfloat16")
    chunks, t = [], 0
    for sz in sizes:
        chunks.append((x[:, :, t:t + sz], None))
        t += sz
    pool, table, cl = gpu_append(ctx, chunks, B, Hkv, d, math.ceil(n / 128), with_values=False,
                                 dtype="bfloat16", rotated=False)
    assert np.array_equal(cl, [n] * B)
    nb = ctx.page_bytes(False)
    eps = 2.0 ** -8
    for b in range(B):
        for h in range(Hkv):
            got = unpack_seq(O, pool, table, b, h, n, d, False, nb)
            rk = O.encode(P, x[b, h], True)
            err = (np.abs(x[b, h]) @ np.abs(P.pi32).T) * (eps * eps * 2 + 64 * 2.0 ** -24)
            compare_records(O, P, x[b, h], rk, got, True, err)
            check_sketch_raw(P, rk, got, err)


def test_capacity_error(O):
    ctx = ctx_for(64)
    k = np.random.default_rng(5).standard_normal((1, 1, 300, 64))
    tq.tq_get_error(ctx.handle)
    gpu_append(ctx, [(k, k)], 1, 1, 64, 2)  # 256 slots for 300 tokens
    assert tq.tq_get_error(ctx.handle) == tq.TQ_ERR_CAPACITY


def test_compress_then_decode_end_to_end(O):
    """GPU compress -> GPU decode against oracle compress -> oracle decode on
    the same raw inputs (no GPU-written page reaches the oracle)."""
    import torch
    d, B, Hkv, G, n_cold, n_hot = 128, 2, 2, 4, 400, 24
    P = params_for(O, d)
    ctx = ctx_for(d)
    rng = np.random.default_rng(9)
    k = W.round_to(rng.standard_normal((B, Hkv, n_cold + n_hot, d)), "bfloat16")
    v = W.round_to(rng.standard_normal((B, Hkv, n_cold + n_hot, d)), "bfloat16")
    pool, table, cl = gpu_append(ctx, [(k[:, :, :n_cold], v[:, :, :n_cold])], B, Hkv, d, 4,
                                 dtype="bfloat16", rotated=False)
    q = W.round_to(rng.standard_normal((B, Hkv * G, d)), "bfloat16")
    k_hot = W.round_to(k[:, :, n_cold:], "float16")
    v_hot = W.round_to(v[:, :, n_cold:], "float16")
    dev = "cuda"
    out = torch.empty((B, Hkv * G, d), dtype=torch.float32, device=dev)
    ws = ctx.workspace(B, Hkv * G, Hkv, 4, n_hot)
    tq.tq_decode_attention(ctx.handle, torch.from_numpy(q).to(torch.bfloat16).to(dev),
                           torch.from_numpy(k_hot).half().to(dev), torch.from_numpy(v_hot).half().to(dev),
                           torch.full((B,), n_hot, dtype=torch.int32, device=dev),
                           torch.from_numpy(pool).to(dev), torch.from_numpy(table).to(dev),
                           torch.from_numpy(cl).to(dev), out, ws, Hkv)
    got = out.cpu().numpy()
    # the oracle's own pages from the same raw inputs
    nb, _ = O.page_layout(d, d, True)
    opool = np.zeros(pool.size, np.uint8)
    for b in range(B):
        for h in range(Hkv):
            rk = O.encode(P, k[b, h, :n_cold], True)
            rv = O.encode(P, v[b, h, :n_cold], False)
            t = np.arange(n_cold)
            O.pack(opool, nb, d, d, True, table[b, h, t // 128], t % 128,
                   dict(sign=rk["sign"], mag=rk["mag"], qbits=rk["qbits"], n=rk["n"],
                        gamma=rk["gamma"], vcode=rv["vcode"], vn=rv["vn"]))
    ref, groups = O.attention(P, q, Hkv, 1 / math.sqrt(d), k_hot, v_hot, np.full(B, n_hot),
                              opool, nb, table, cl)
    # the two pipelines store different bits only where a decision lies within
    # rounding of its threshold (sketch signs of near-zero projections, codes at
    # boundaries); such a flip moves one logit by a bounded step, so the two
    # outputs must agree far more closely than either agrees with exact attention
    diff, qerr = [], []
    for gi, (b, h) in enumerate(groups):
        K = k[b, h]
        V = v[b, h]
        for gq in range(G):
            s = (K @ q[b, h * G + gq]) / math.sqrt(d)
            p_ = np.exp(s - s.max())
            exact = (p_ / p_.sum()) @ V
            diff.append(np.abs(got[b, h * G + gq] - ref[gi, gq]))
            qerr.append(np.abs(ref[gi, gq] - exact))
    diff, qerr = np.concatenate(diff), np.concatenate(qerr)
    assert diff.max() < 2e-2
    assert diff.mean() < 0.1 * qerr.mean(), (diff.mean(), qerr.mean())


def test_compress_4m_sampled_records(O):
    """The full compress workload in the benchmark's launch configuration
    (8 kv heads x 524288 bf16 vectors, d = 128, x = N(0,1) sigma[h, j], sigma
    LogNormal(0,1), one call, keys-only pages): 8192 records sampled over all
    heads and page tiles (first and last page of every head included) match
    the oracle's encoding of the same input rows within the rotation error."""
    import torch
    d, H, T = 128, 8, 524288
    P = params_for(O, d)
    ctx = ctx_for(d)
    dev = torch.device("cuda")
    gen = torch.Generator(device=dev)
    gen.manual_seed(21)
    sigma = torch.exp(torch.randn((H, d), generator=gen, device=dev))
    x = (torch.randn((1, H, T, d), generator=gen, device=dev) * sigma[None, :, None, :]).to(torch.bfloat16)
    pages = H * T // 128
    pool = torch.zeros((pages, ctx.page_bytes(False)), dtype=torch.uint8, device=dev)
    table = torch.arange(pages, dtype=torch.int32, device=dev).view(1, H, T // 128)
    cold = torch.zeros(1, dtype=torch.int32, device=dev)
    tq.tq_compress_append(ctx.handle, x, None, pool, table, cold)
    torch.cuda.synchronize()
    assert tq.tq_get_error(ctx.handle) == tq.TQ_OK
    assert int(cold.item()) == T
    rng = np.random.default_rng(41)
    nb = ctx.page_bytes(False)
    eps = 2.0 ** -8
    flips = sflips = total = 0
    for h in range(H):
        t = np.concatenate([rng.choice(T, 1030, replace=False), [0, 127, T - 128, T - 1]])
        t = np.unique(t)
        rows = x[0, h, torch.from_numpy(t).to(dev)].double().cpu().numpy()
        pg = (h * (T // 128) + t // 128).astype(np.int64)
        uniq, inv = np.unique(pg, return_inverse=True)
        sub = pool[torch.from_numpy(uniq).to(dev)].cpu().numpy().reshape(-1)
        got = O.unpack(sub, nb, d, d, False, inv.astype(np.int32), (t % 128).astype(np.int32))
        rk = O.encode(P, rows, True)
        err = (np.abs(rows) @ np.abs(P.pi32).T) * (eps * eps * 2 + 64 * 2.0 ** -24)
        flips += compare_records(O, P, rows, rk, got, True, err)
        sflips += check_sketch_raw(P, rk, got, err)
        total += len(t) * d
    assert total >= 8192 * d
    assert sflips <= 0.01 * total
    print("4M compress, %d sampled records: code differences at decision boundaries %d, "
          "sketch sign flips near zero %d" % (total // d, flips, sflips))
