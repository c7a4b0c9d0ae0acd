"""CPU oracle for TurboQuant-style KV compression, compressed-cache decode
attention and compressed top-k search.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, by the package smoke check
and by the CPU-baseline leg of ``bench.py``; never by the product path.  It
shares no code with the CUDA library (its arithmetic lives in
``oracle/tq_oracle.c``, compiled with gcc; this module only marshals numpy
arrays).  See the C file's header for the passages each function follows and
the readings taken where the pages are silent.

Parity status: every function here is pinned by ``tests/test_oracle_*.py``
against closed forms, library routines, published values or brute force.
"""
import ctypes as C
import math
import os

import numpy as np

from . import build as _build

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = C.CDLL(path)
        dp = C.POINTER(C.c_double)
        ip = C.POINTER(C.c_int32)
        u8 = C.POINTER(C.c_uint8)
        sz = C.c_size_t
        L.or_normals.argtypes = [C.c_uint64, C.c_int64, dp]
        L.or_uniforms.argtypes = [C.c_uint64, C.c_int64, dp]
        L.or_round_f16.argtypes = [C.c_double]
        L.or_round_f16.restype = C.c_double
        L.or_f16_bits.argtypes = [C.c_double]
        L.or_f16_bits.restype = C.c_uint16
        L.or_f16_value.argtypes = [C.c_uint16]
        L.or_f16_value.restype = C.c_double
        L.or_rotation.argtypes = [C.c_int, C.c_uint64, dp]
        L.or_rotation.restype = C.c_int
        L.or_qjl_matrix.argtypes = [C.c_int, C.c_int, C.c_uint64, dp]
        L.or_sphere_mass.argtypes = [C.c_int, C.c_double, C.c_double]
        L.or_sphere_mass.restype = C.c_double
        L.or_sphere_first_moment.argtypes = [C.c_int, C.c_double, C.c_double]
        L.or_sphere_first_moment.restype = C.c_double
        L.or_lloyd_max.argtypes = [C.c_int, C.c_int, C.c_int, dp, dp, dp]
        L.or_lloyd_max.restype = C.c_int
        L.or_page_layout.argtypes = [C.c_int, C.c_int, C.c_int, C.POINTER(C.c_size_t)]
        L.or_page_layout.restype = sz
        L.or_pack_batch.argtypes = [u8, sz, C.c_int, C.c_int, C.c_int, C.c_int64, ip, ip, ip,
                                    ip, ip, dp, dp, ip, dp]
        L.or_unpack_batch.argtypes = [u8, sz, C.c_int, C.c_int, C.c_int, C.c_int64, ip, ip, ip,
                                      ip, ip, dp, dp, ip, dp]
        L.or_encode.argtypes = [C.c_int, C.c_int, dp, dp, dp, dp, C.c_int, dp, C.c_int64,
                                C.c_int, C.c_int, ip, ip, ip, dp, dp, dp, C.c_int]
        L.or_qjl_estimate.argtypes = [C.c_int, dp, ip, C.c_double]
        L.or_qjl_estimate.restype = C.c_double
        L.or_qjl_montecarlo.argtypes = [C.c_int, C.c_int, dp, dp, C.c_int64, C.c_uint64, dp, dp]
        L.or_attention.argtypes = [C.c_int, C.c_int, dp, dp, dp, dp, C.c_int, C.c_int, C.c_int,
                                   dp, C.c_double, dp, dp, C.c_int, ip, u8, sz, ip, C.c_int, ip,
                                   ip, C.c_int, dp, C.c_int]
        L.or_attention.restype = C.c_int
        L.or_attention_gated.argtypes = [C.c_int, C.c_int, dp, dp, dp, dp, C.c_int, C.c_int,
                                         C.c_int, dp, C.c_double, dp, dp, C.c_int, ip, u8, sz, ip,
                                         C.c_int, ip, ip, C.c_int, C.c_int, C.c_double, ip, dp,
                                         C.c_int]
        L.or_attention_gated.restype = C.c_int
        L.or_cold_logits.argtypes = [C.c_int, C.c_int, dp, dp, dp, C.c_int, dp, C.c_double, u8,
                                     sz, ip, C.c_int, dp]
        L.or_cold_logits.restype = None
        L.or_topk.argtypes = [C.c_int, C.c_int, dp, dp, dp, dp, C.c_int, u8, sz, C.c_int64,
                              C.c_int, ip, dp, C.c_int]
        L.or_max_threads.restype = C.c_int
        L.or_angle_lloyd_max.argtypes = [C.c_int, C.c_int, C.c_int, dp, dp]
        L.or_angle_lloyd_max.restype = C.c_int
        L.or_polar_code_bytes.argtypes = [C.c_int, C.c_int, C.c_int]
        L.or_polar_code_bytes.restype = sz
        L.or_polar_encode.argtypes = [C.c_int, C.POINTER(C.c_float), C.c_int64, C.c_int, C.c_int,
                                      u8, C.POINTER(C.c_uint16)]
        L.or_polar_decode.argtypes = [C.c_int, u8, C.POINTER(C.c_uint16), C.c_int64, C.c_int,
                                      C.c_int, dp]
        L.or_polar_transform.argtypes = [C.c_int, dp, dp, dp]
        L.or_polar_inverse.argtypes = [C.c_int, C.c_double, dp, dp]
        _lib = L
    return _lib


def _d(a):
    a = np.ascontiguousarray(a, dtype=np.float64)
    return a, a.ctypes.data_as(C.POINTER(C.c_double))


def _i(a):
    a = np.ascontiguousarray(a, dtype=np.int32)
    return a, a.ctypes.data_as(C.POINTER(C.c_int32))


def _u8(a):
    assert a.dtype == np.uint8 and a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(C.POINTER(C.c_uint8))


def _nullable(a, conv):
    if a is None:
        return None, None
    return conv(a)


# --------------------------------------------------------------------------
# random streams and rounding
# --------------------------------------------------------------------------
def normals(seed, count):
    out = np.empty(count, np.float64)
    lib().or_normals(seed, count, out.ctypes.data_as(C.POINTER(C.c_double)))
    return out


def uniforms(seed, count):
    out = np.empty(count, np.float64)
    lib().or_uniforms(seed, count, out.ctypes.data_as(C.POINTER(C.c_double)))
    return out


def round_f16(x):
    return lib().or_round_f16(float(x))


def f16_bits(x):
    return lib().or_f16_bits(float(x))


def f16_value(bits):
    return lib().or_f16_value(int(bits))


# --------------------------------------------------------------------------
# parameters
# --------------------------------------------------------------------------
def rotation(d, seed):
    """Haar rotation in fp64 (QR of the Gaussian matrix, diag(R) > 0)."""
    pi = np.empty((d, d), np.float64)
    rc = lib().or_rotation(d, seed, pi.ctypes.data_as(C.POINTER(C.c_double)))
    assert rc == 0
    return pi


def qjl_matrix(m, d, seed):
    s = np.empty((m, d), np.float64)
    lib().or_qjl_matrix(m, d, seed, s.ctypes.data_as(C.POINTER(C.c_double)))
    return s


def sphere_mass(d, a, b):
    return lib().or_sphere_mass(d, a, b)


def sphere_first_moment(d, a, b):
    return lib().or_sphere_first_moment(d, a, b)


def lloyd_max(d, bits, max_iter=100000):
    """Positive centroids c (2^(bits-1)), positive boundaries t, MSE, iterations."""
    L = 1 << (bits - 1)
    c = np.empty(L, np.float64)
    t = np.empty(max(L - 1, 1), np.float64)
    mse = C.c_double()
    it = lib().or_lloyd_max(d, bits, max_iter, c.ctypes.data_as(C.POINTER(C.c_double)),
                            t.ctypes.data_as(C.POINTER(C.c_double)), C.byref(mse))
    return c, t[: L - 1], mse.value, it


class Params:
    """All tables of one configuration, as both sides store them:
    pi32 = fp32(Pi), S = fp16-valued Gaussian, codebooks fp32."""

    def __init__(self, d, m=None, key_bits=2, value_bits=4, seed=0):
        self.d, self.m = d, (m if m is not None else d)
        self.key_bits, self.value_bits, self.seed = key_bits, value_bits, seed
        self.pi64 = rotation(d, seed)
        self.pi32 = self.pi64.astype(np.float32).astype(np.float64)
        self.S = qjl_matrix(self.m, d, seed)
        kc, kt, self.key_mse, _ = lloyd_max(d, key_bits)
        vc, vt, self.value_mse, _ = lloyd_max(d, value_bits)
        self.kc64, self.kt64, self.vc64, self.vt64 = kc, kt, vc, vt
        f32 = lambda a: a.astype(np.float32).astype(np.float64)
        self.kc, self.kt, self.vc, self.vt = f32(kc), f32(kt), f32(vc), f32(vt)

    @property
    def alpha(self):
        return math.sqrt(math.pi / 2.0) / self.m


# --------------------------------------------------------------------------
# page format
# --------------------------------------------------------------------------
PAGE_TOKENS = 128


def page_layout(d, m, with_values=True):
    """(page bytes, offsets).  Keys-only pages (record layout): section offsets
    kc, qs, kn, kg and block = 0.  Pages with values (block layout): offsets
    inside a 16-token block -- kc (key plane H), kl (plane L), qs, vc, kn and
    kg (the norm pair of the block's token 0), vn -- and the block size."""
    offs = (C.c_size_t * 8)()
    nbytes = lib().or_page_layout(d, m, 1 if with_values else 0, offs)
    return int(nbytes), dict(zip(["kc", "qs", "vc", "kn", "kg", "vn", "block", "kl"],
                                 [int(o) for o in offs]))


def norm_slots(d, m, with_values=True):
    """Byte offsets inside a page of the fp16 norm fields of the 128 token
    slots: dict kn, kg (and vn for pages with values) -> int array [128]."""
    _, L = page_layout(d, m, with_values)
    s = np.arange(PAGE_TOKENS)
    if L["block"]:
        base = (s // 16) * L["block"]
        t = s % 16
        return dict(kn=base + L["kn"] + 4 * t, kg=base + L["kg"] + 4 * t, vn=base + L["vn"] + 2 * t)
    return dict(kn=L["kn"] + 2 * s, kg=L["kg"] + 2 * s)


def pack(pool, page_bytes, d, m, with_values, page_id, slot, rec):
    """Write records into pages.  rec: dict with sign, mag [N,d], qbits [N,m],
    n, gamma [N] and (values) vcode [N,d], vn [N]."""
    N = len(page_id)
    pid, pidp = _i(page_id)
    sl, slp = _i(slot)
    sg, sgp = _i(rec["sign"])
    mg, mgp = _i(rec["mag"])
    qb, qbp = _i(rec["qbits"])
    n, np_ = _d(rec["n"])
    g, gp = _d(rec["gamma"])
    vc, vcp = _nullable(rec.get("vcode"), _i)
    vn, vnp = _nullable(rec.get("vn"), _d)
    lib().or_pack_batch(_u8(pool), page_bytes, d, m, 1 if with_values else 0, N, pidp, slp, sgp,
                        mgp, qbp, np_, gp, vcp, vnp)


def unpack(pool, page_bytes, d, m, with_values, page_id, slot):
    N = len(page_id)
    pid, pidp = _i(page_id)
    sl, slp = _i(slot)
    rec = dict(sign=np.empty((N, d), np.int32), mag=np.empty((N, d), np.int32),
               qbits=np.empty((N, m), np.int32), n=np.empty(N), gamma=np.empty(N))
    if with_values:
        rec["vcode"] = np.empty((N, d), np.int32)
        rec["vn"] = np.empty(N)
    P = lambda k, t: rec[k].ctypes.data_as(C.POINTER(t)) if k in rec else None
    lib().or_unpack_batch(_u8(pool), page_bytes, d, m, 1 if with_values else 0, N, pidp, slp,
                          P("sign", C.c_int32), P("mag", C.c_int32), P("qbits", C.c_int32),
                          P("n", C.c_double), P("gamma", C.c_double), P("vcode", C.c_int32),
                          P("vn", C.c_double))
    return rec


# --------------------------------------------------------------------------
# encoding
# --------------------------------------------------------------------------
def encode(params, x, is_key, rotated=False, threads=0):
    """Encode rows of x [N, d] (values exactly as stored, widened to fp64).
    Returns dict(sign, mag, qbits, n, gamma, xrot); for values, vcode too."""
    p = params
    x, xp = _d(np.asarray(x).reshape(-1, p.d))
    N = x.shape[0]
    sign = np.empty((N, p.d), np.int32)
    mag = np.empty((N, p.d), np.int32)
    qbits = np.zeros((N, p.m), np.int32)
    n = np.empty(N)
    gamma = np.zeros(N)
    xrot = np.empty((N, p.d))
    pi, pip = _d(p.pi32)
    S, Sp = _d(p.S)
    cpos, cposp = _d(p.kc if is_key else p.vc)
    tpos, tposp = _d(p.kt if is_key else p.vt)
    L = 1 << ((p.key_bits if is_key else p.value_bits) - 1)
    ptr = lambda a, t: a.ctypes.data_as(C.POINTER(t))
    lib().or_encode(p.d, p.m, pip, Sp, cposp, tposp, L, xp, N, 1 if rotated else 0,
                    1 if is_key else 0, ptr(sign, C.c_int32), ptr(mag, C.c_int32),
                    ptr(qbits, C.c_int32), ptr(n, C.c_double), ptr(gamma, C.c_double),
                    ptr(xrot, C.c_double), threads)
    rec = dict(sign=sign, mag=mag, qbits=qbits, n=n, gamma=gamma, xrot=xrot)
    if not is_key:
        rec["vcode"] = (sign << 3) | mag
        rec["vn"] = n
    return rec


def qjl_estimate(sq, qbits, gamma):
    sq, sqp = _d(sq)
    qb, qbp = _i(qbits)
    return lib().or_qjl_estimate(len(sq), sqp, qbp, gamma)


def qjl_montecarlo(q, r, trials, seed0):
    q, qp = _d(q)
    r, rp = _d(r)
    mean, var = C.c_double(), C.c_double()
    lib().or_qjl_montecarlo(len(q), len(q), qp, rp, trials, seed0, C.byref(mean), C.byref(var))
    return mean.value, var.value


# --------------------------------------------------------------------------
# attention and search
# --------------------------------------------------------------------------
def attention(params, q, Hkv, scale, k_hot, v_hot, hot_len, pool, page_bytes, page_table,
              cold_len, groups=None, threads=0, threshold=None):
    """q [B, Hq, d]; k_hot/v_hot [B, Hkv, W, d] or None; hot_len, cold_len [B];
    page_table [B, Hkv, max_pages].  groups: list of (b, kv_head) or None=all.
    Returns out [len(groups), G, d] (fp64) and the group list.  With a
    threshold, a head reads its cold tokens only when its largest raw hot
    score is below it, and the result is (out, groups, open [len(groups), G])."""
    p = params
    q, qp = _d(q)
    B, Hq, d = q.shape
    G = Hq // Hkv
    if groups is None:
        groups = [(b, h) for b in range(B) for h in range(Hkv)]
    sel, selp = _i(np.asarray(groups, np.int32).reshape(-1))
    if k_hot is not None:
        kh, khp = _d(k_hot)
        vh, vhp = _d(v_hot)
        W = kh.shape[2]
    else:
        kh = vh = khp = vhp = None
        W = 0
    hl, hlp = _nullable(None if hot_len is None else np.asarray(hot_len), _i)
    cl, clp = _nullable(None if cold_len is None else np.asarray(cold_len), _i)
    pt, ptp = _i(page_table)
    max_pages = pt.shape[-1]
    pi, pip = _d(p.pi32)
    S, Sp = _d(p.S)
    kc, kcp = _d(p.kc)
    vc, vcp = _d(p.vc)
    out = np.empty((len(groups), G, d))
    if pool is None:
        pool = np.zeros(16, np.uint8)
    if threshold is None:
        rc = lib().or_attention(d, p.m, pip, Sp, kcp, vcp, B, Hq, Hkv, qp, scale, khp, vhp, W,
                                hlp, _u8(pool), page_bytes, ptp, max_pages, clp, selp,
                                len(groups), out.ctypes.data_as(C.POINTER(C.c_double)), threads)
        assert rc == 0
        return out, groups
    opened = np.empty((len(groups), G), np.int32)
    rc = lib().or_attention_gated(d, p.m, pip, Sp, kcp, vcp, B, Hq, Hkv, qp, scale, khp, vhp, W,
                                  hlp, _u8(pool), page_bytes, ptp, max_pages, clp, selp,
                                  len(groups), 1, float(threshold),
                                  opened.ctypes.data_as(C.POINTER(C.c_int32)),
                                  out.ctypes.data_as(C.POINTER(C.c_double)), threads)
    assert rc == 0
    return out, groups, opened


def cold_logits(params, q, scale, pool, page_bytes, pages, cold_len):
    """Estimated cold scores of one (batch, kv head) group as the decode
    attention forms them: q [G, d]; pages: the group's page-table row.
    Returns [G, cold_len]."""
    p = params
    q, qp = _d(np.asarray(q).reshape(-1, p.d))
    G = q.shape[0]
    pg, pgp = _i(pages)
    pi, pip = _d(p.pi32)
    S, Sp = _d(p.S)
    kc, kcp = _d(p.kc)
    out = np.empty((G, int(cold_len)))
    lib().or_cold_logits(p.d, p.m, pip, Sp, kcp, G, qp, scale, _u8(pool), page_bytes, pgp,
                         int(cold_len), out.ctypes.data_as(C.POINTER(C.c_double)))
    return out


def topk(params, queries, db_pool, page_bytes, N, k, threads=0):
    p = params
    qs, qsp = _d(queries)
    Q = qs.shape[0]
    ids = np.empty((Q, k), np.int32)
    scores = np.empty((Q, k))
    pi, pip = _d(p.pi32)
    S, Sp = _d(p.S)
    kc, kcp = _d(p.kc)
    lib().or_topk(p.d, p.m, pip, Sp, kcp, qsp, Q, _u8(db_pool), page_bytes, N, k,
                  ids.ctypes.data_as(C.POINTER(C.c_int32)),
                  scores.ctypes.data_as(C.POINTER(C.c_double)), threads)
    return ids, scores


def max_threads():
    return lib().or_max_threads()


# --------------------------------------------------------------------------
# stage-1 variants: PolarQuant and MSE-only b-bit codes
# --------------------------------------------------------------------------
def angle_lloyd_max(k, bits, max_iter=100000):
    """Lloyd-Max levels and boundaries of the angle between two blocks of k
    coordinates (density proportional to sin^(k-1)(2 phi) on [0, pi/2])."""
    c = np.empty(1 << bits)
    t = np.empty((1 << bits) - 1)
    it = lib().or_angle_lloyd_max(k, bits, max_iter, c.ctypes.data_as(C.POINTER(C.c_double)),
                                  t.ctypes.data_as(C.POINTER(C.c_double)))
    return c, t, it


def polar_code_bytes(d, b1, b2):
    return int(lib().or_polar_code_bytes(d, b1, b2))


def polar_encode(x, b1, b2):
    """x [N, d] rotated vectors (rounded to fp32).  Returns codes uint8
    [N, polar_code_bytes] and the fp16 bits of the final radii [N]."""
    x = np.ascontiguousarray(np.asarray(x, np.float32))
    N, d = x.shape
    cb = polar_code_bytes(d, b1, b2)
    codes = np.zeros((N, cb), np.uint8)
    rad = np.zeros(N, np.uint16)
    lib().or_polar_encode(d, x.ctypes.data_as(C.POINTER(C.c_float)), N, b1, b2, _u8(codes),
                          rad.ctypes.data_as(C.POINTER(C.c_uint16)))
    return codes, rad


def polar_decode(codes, rad, d, b1, b2):
    codes = np.ascontiguousarray(codes, np.uint8)
    rad = np.ascontiguousarray(rad, np.uint16)
    N = codes.shape[0]
    out = np.empty((N, d))
    lib().or_polar_decode(d, _u8(codes), rad.ctypes.data_as(C.POINTER(C.c_uint16)), N, b1, b2,
                          out.ctypes.data_as(C.POINTER(C.c_double)))
    return out


def polar_transform(x):
    """Exact (fp64) transform of one vector: final radius, angles (level 1
    first, then levels 2, 3, ...)."""
    x, xp = _d(x)
    d = x.shape[0]
    r = C.c_double()
    ang = np.empty(d - 1)
    lib().or_polar_transform(d, xp, C.byref(r), ang.ctypes.data_as(C.POINTER(C.c_double)))
    return r.value, ang


def polar_inverse(radius, angles):
    angles, ap = _d(angles)
    d = angles.shape[0] + 1
    out = np.empty(d)
    lib().or_polar_inverse(d, float(radius), ap, out.ctypes.data_as(C.POINTER(C.c_double)))
    return out


def mse_pack(sign, mag, bits):
    """MSE-only b-bit codes, one vector per row: code_j = sign << (b-1) | mag
    in bits [b j, b j + b) of a little-endian bit stream."""
    sign = np.asarray(sign, np.int64)
    mag = np.asarray(mag, np.int64)
    N, d = sign.shape
    code = (sign << (bits - 1)) | mag
    out = np.zeros((N, (bits * d + 7) // 8), np.uint8)
    for j in range(d):
        for i in range(bits):
            pos = bits * j + i
            out[:, pos >> 3] |= (((code[:, j] >> i) & 1) << (pos & 7)).astype(np.uint8)
    return out


def mse_unpack(packed, d, bits):
    packed = np.asarray(packed, np.uint8)
    N = packed.shape[0]
    code = np.zeros((N, d), np.int64)
    for j in range(d):
        for i in range(bits):
            pos = bits * j + i
            code[:, j] |= ((packed[:, pos >> 3] >> (pos & 7)) & 1).astype(np.int64) << i
    return code >> (bits - 1), code & ((1 << (bits - 1)) - 1)


def mse_encode(params, x_rot, bits):
    """MSE-only b-bit stage 1 on rotated vectors: the oracle's quantiser with
    a 2^(b-1)-level Lloyd-Max codebook (no QJL).  Returns packed codes, the
    fp16 norms and the codebook."""
    p = params
    x = np.asarray(x_rot, np.float64).reshape(-1, p.d)
    c, t, _, _ = lloyd_max(p.d, bits)
    f32 = lambda a: a.astype(np.float32).astype(np.float64)
    cpos, tpos = f32(c), f32(t)
    N = x.shape[0]
    sign = np.empty((N, p.d), np.int32)
    mag = np.empty((N, p.d), np.int32)
    qbits = np.zeros((N, p.m), np.int32)
    n = np.empty(N)
    gamma = np.zeros(N)
    xr = np.empty((N, p.d))
    x, xp = _d(x)
    pi, pip = _d(p.pi32)
    S, Sp = _d(p.S)
    cp_, cpp = _d(cpos)
    tp_, tpp = _d(tpos)
    ptr = lambda a, ty: a.ctypes.data_as(C.POINTER(ty))
    lib().or_encode(p.d, p.m, pip, Sp, cpp, tpp, len(cpos), xp, N, 1, 0, ptr(sign, C.c_int32),
                    ptr(mag, C.c_int32), ptr(qbits, C.c_int32), ptr(n, C.c_double),
                    ptr(gamma, C.c_double), ptr(xr, C.c_double), 0)
    return mse_pack(sign, mag, bits), n, cpos


def mse_decode(packed, n, cpos, d, bits):
    sign, mag = mse_unpack(packed, d, bits)
    return np.asarray(n)[:, None] * np.where(sign == 1, -1.0, 1.0) * cpos[mag]
