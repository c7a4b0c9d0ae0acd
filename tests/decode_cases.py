"""Shared builders for decode-attention parity tests: seeded K, V, q from
the workload generators, cold pages written by the oracle's encoder and
packer (never by the CUDA path), hot windows in fp16."""
import math

import numpy as np

from compressed_kv_decode_b200 import workloads as W


class DecodeCase:
    pass


def build(O, P, B, Hq, Hkv, d, cold_len, hot_len, W_max, max_pages, q_dtype="float32",
          seeds=(101, 102, 103, 104), n_out=0, factor=1.0, real_groups=None, nan_hot_tail=True,
          seed=0):
    """real_groups: (b, h) pairs whose cold pages hold oracle-encoded K, V;
    None means all groups.  Pages of the other groups hold random records."""
    c = DecodeCase()
    c.B, c.Hq, c.Hkv, c.d, c.G = B, Hq, Hkv, d, Hq // Hkv
    c.cold_len = np.asarray(cold_len, np.int32)
    c.hot_len = np.asarray(hot_len, np.int32)
    c.W_max, c.max_pages = W_max, max_pages
    nbytes, _ = O.page_layout(d, d, True)
    c.page_bytes = nbytes
    c.table, n_pages = W.random_page_table(seed + 1, B, Hkv, max_pages, spare=3)
    c.pool = W.random_page_bytes(seed + 2, n_pages, nbytes, O.norm_slots(d, d, True))
    chans = W.outlier_channels(seeds[3], Hkv, d, n_out)
    c.k_hot = np.zeros((B, Hkv, max(W_max, 1), d))
    c.v_hot = np.zeros((B, Hkv, max(W_max, 1), d))
    if nan_hot_tail:  # slots past hot_len must never be read
        c.k_hot[:] = np.nan
        c.v_hot[:] = np.nan
    groups = real_groups if real_groups is not None else [(b, h) for b in range(B) for h in range(Hkv)]
    c.groups = groups
    flat = c.pool.reshape(-1)
    for (b, h) in groups:
        nc, nh = int(c.cold_len[b]), int(c.hot_len[b])
        K, V = W.kv_sequence(seeds[0], seeds[1], b, h, nc + nh, d, chans[h], factor)
        if nh:
            c.k_hot[b, h, :nh] = W.round_to(K[nc:], "float16")
            c.v_hot[b, h, :nh] = W.round_to(V[nc:], "float16")
        if nc:
            kr = O.encode(P, K[:nc], True)
            vr = O.encode(P, V[:nc], False)
            rec = dict(sign=kr["sign"], mag=kr["mag"], qbits=kr["qbits"], n=kr["n"],
                       gamma=kr["gamma"], vcode=vr["vcode"], vn=vr["vn"])
            t = np.arange(nc)
            O.pack(flat, nbytes, d, d, True, c.table[b, h, t // 128], t % 128, rec)
    c.q = W.queries(seeds[2], B, Hq, d, q_dtype)
    c.q_dtype = q_dtype
    c.W_max = W_max
    return c


def oracle_out(O, P, c, scale=None):
    """Oracle output for the case's real groups: {(b, h): [G, d]}."""
    scale = 1.0 / math.sqrt(c.d) if scale is None else scale
    res = {}
    for (b, h) in c.groups:
        q = c.q[b:b + 1, h * c.G:(h + 1) * c.G]
        kh = c.k_hot[b:b + 1, h:h + 1, :max(int(c.hot_len[b]), 1)]
        vh = c.v_hot[b:b + 1, h:h + 1, :max(int(c.hot_len[b]), 1)]
        out, _ = O.attention(P, q, 1, scale, np.nan_to_num(kh), np.nan_to_num(vh),
                             c.hot_len[b:b + 1], c.pool.reshape(-1), c.page_bytes,
                             c.table[b:b + 1, h:h + 1], c.cold_len[b:b + 1])
        res[(b, h)] = out[0]
    return res


def gpu_out(tq, ctx, c, scale=0.0, pool_pages=None, table=None):
    import torch
    dev = "cuda"
    qd = getattr(torch, c.q_dtype)
    q = torch.from_numpy(c.q).to(qd).to(dev)
    k_hot = torch.from_numpy(c.k_hot).to(torch.float16).to(dev) if c.W_max else None
    v_hot = torch.from_numpy(c.v_hot).to(torch.float16).to(dev) if c.W_max else None
    hot_len = torch.from_numpy(c.hot_len).to(dev)
    cold_len = torch.from_numpy(c.cold_len).to(dev)
    pool = torch.from_numpy(c.pool).to(dev)
    tbl = torch.from_numpy(c.table if table is None else table).to(dev)
    out = torch.full((c.B, c.Hq, c.d), float("nan"), dtype=torch.float32, device=dev)
    ws = torch.empty(tq.tq_workspace_bytes(ctx.handle, c.B, c.Hq, c.Hkv, c.max_pages, c.W_max),
                     dtype=torch.uint8, device=dev)
    if pool_pages is not None:
        pool = pool[:pool_pages]
    tq.tq_decode_attention(ctx.handle, q, k_hot, v_hot, hot_len, pool, tbl, cold_len, out, ws,
                           c.Hkv, scale)
    torch.cuda.synchronize()
    return out.cpu().numpy().astype(np.float64)


def assert_close(gpu, ref, atol=2e-3, rtol=1e-2, what=""):
    err = np.abs(gpu - ref)
    bound = atol + rtol * np.abs(ref)
    bad = ~(err <= bound)
    assert not bad.any(), "%s: %d of %d outside tolerance; worst err %.3g at ref %.3g" % (
        what, bad.sum(), bad.size, err.max(), ref.reshape(-1)[np.argmax(err)])
