"""Seeded synthetic inputs shaped like the workloads on the pages.

Random draws only: nothing here encodes, quantises or attends.  The tests
feed the same arrays to the CUDA library and to the CPU oracle; the
benchmark uses the same shapes and distributions.

Workloads (names used by tests and bench):
  tiny          1 head, d=64, 256 cold tokens, K, V, q iid N(0,1) fp32 from
                one generator seeded 0, drawn in the order K, V, q.
  tinyllama     B=1, 32 q heads / 4 kv heads, d=64, 512 hot fp16 + 1024 cold;
                K, V ~ N(0,1) with 4 outlier channels per kv head scaled x10;
                q fp16 N(0,1).  Seeds: K 1, V 2, q 3, outlier channels 4.
  llama3_8b_32k B=16, 32 q / 8 kv heads, d=128, 32768 tokens: last 1024 hot
                fp16, 31744 cold; 8 outlier channels x8; q bf16.  Seeds: K 11,
                V 12, q 13, outliers 14.
  compress_4m   8 kv heads x 524288 tokens of bf16 d=128 vectors,
                x = N(0,1) * sigma[h, j], sigma ~ LogNormal(0, 1).  Seeds:
                scales 21, data 22.
  search_1m     10^6 database and 4096 query unit vectors (Gaussian,
                normalised), d=128.  Seeds: database 31, queries 32.
"""
import numpy as np

DECODE = {
    "tiny": dict(B=1, Hq=1, Hkv=1, d=64, cold=256, hot=0, q_dtype="float32", n_out=0, factor=1.0,
                 seeds=(0, 0, 0, 0)),
    "tinyllama": dict(B=1, Hq=32, Hkv=4, d=64, cold=1024, hot=512, q_dtype="float16", n_out=4,
                      factor=10.0, seeds=(1, 2, 3, 4)),
    "llama3_8b_32k": dict(B=16, Hq=32, Hkv=8, d=128, cold=31744, hot=1024, q_dtype="bfloat16",
                          n_out=8, factor=8.0, seeds=(11, 12, 13, 14)),
}


def outlier_channels(seed, Hkv, d, n_out):
    rng = np.random.default_rng(seed)
    return [np.sort(rng.choice(d, n_out, replace=False)) if n_out else np.zeros(0, np.int64)
            for _ in range(Hkv)]


def kv_sequence(seed_k, seed_v, b, h, T, d, channels, factor):
    """K, V [T, d] fp64 for one (batch, kv head): N(0,1) with the outlier
    channels scaled.  Each (b, h) has its own generator, so any subset of
    groups can be drawn without the others."""
    K = np.random.default_rng([seed_k, b, h]).standard_normal((T, d))
    V = np.random.default_rng([seed_v, b, h]).standard_normal((T, d))
    if len(channels):
        K[:, channels] *= factor
        V[:, channels] *= factor
    return K, V


def round_to(x, dtype):
    """Round fp64 values to a storage dtype and widen back to fp64."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x, np.float64)).to(getattr(torch, dtype))
    return t.to(torch.float64).numpy()


def queries(seed, B, Hq, d, dtype):
    q = np.random.default_rng(seed).standard_normal((B, Hq, d))
    return round_to(q, dtype)


def tiny_case():
    """The tiny workload: one generator, draw order K, V, q."""
    rng = np.random.default_rng(0)
    K = rng.standard_normal((256, 64)).astype(np.float32).astype(np.float64)
    V = rng.standard_normal((256, 64)).astype(np.float32).astype(np.float64)
    q = rng.standard_normal((1, 1, 64)).astype(np.float32).astype(np.float64)
    return K, V, q


def compress_scales(seed, H, d):
    return np.random.default_rng(seed).lognormal(0.0, 1.0, (H, d))


def compress_data(seed, scales, T, rows=None):
    """bf16-rounded x = N(0,1) * scale for heads x tokens; rows=(h, t0, t1)
    draws a slice (generator per head)."""
    H, d = scales.shape
    out = []
    heads = range(H) if rows is None else [rows[0]]
    for h in heads:
        g = np.random.default_rng([seed, h])
        x = g.standard_normal((T, d))
        if rows is not None:
            x = x[rows[1]:rows[2]]
        out.append(round_to(x * scales[h], "bfloat16"))
    return np.stack(out)


def unit_vectors(seed, n, d):
    x = np.random.default_rng(seed).standard_normal((n, d))
    return x / np.linalg.norm(x, axis=1, keepdims=True)


def random_page_table(seed, B, Hkv, max_pages, spare=0):
    """A random permutation of pool pages (plus `spare` unused pages)."""
    n = B * Hkv * max_pages
    perm = np.random.default_rng(seed).permutation(n + spare)[:n]
    return perm.astype(np.int32).reshape(B, Hkv, max_pages), n + spare


def random_page_bytes(seed, n_pages, page_bytes, norm_slots):
    """Random bytes for pages whose content does not matter, with every fp16
    norm field set to a finite value in [2, 14) (gamma in [0, 0.5)).
    norm_slots: field name (kn, kg, vn) -> byte offsets of the 128 token
    slots' fp16 fields inside a page."""
    rng = np.random.default_rng(seed)
    pool = rng.integers(0, 256, size=(n_pages, page_bytes), dtype=np.uint8)
    for name, lo, hi in (("kn", 2.0, 14.0), ("kg", 0.0, 0.5), ("vn", 2.0, 14.0)):
        offs = norm_slots.get(name)
        if offs is None:
            continue
        offs = np.asarray(offs, np.int64)
        vals = rng.uniform(lo, hi, size=(n_pages, len(offs))).astype(np.float16).view(np.uint8)
        pool[:, offs] = vals[:, 0::2]
        pool[:, offs + 1] = vals[:, 1::2]
    return pool
