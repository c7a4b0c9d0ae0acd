"""Pins of the oracle's encoder and page packer: hand-worked format examples,
inverse-map derivation of every bit position, round trips, exhaustive
nearest-centroid search, Monte-Carlo unbiasedness and variance of the QJL
estimator, and the value quantiser's distortion against the codebook MSE."""
import math
import os

import numpy as np
import pytest

D_M = [(64, 64), (128, 128)]


def _golden():
    path = os.path.join(os.path.dirname(__file__), "golden", "page_format_examples.txt")
    rows = {}
    for line in open(path):
        if line.strip() and not line.startswith("#"):
            kind, *fields = line.split()
            rows[kind] = dict(f.split("=") for f in fields)
    return rows


@pytest.mark.parametrize("d,m,wv,expect", [(128, 128, 1, 15104), (128, 128, 0, 6656),
                                           (64, 64, 1, 7936), (64, 64, 0, 3584)])
def test_page_bytes(O, d, m, wv, expect):
    nbytes, offs = O.page_layout(d, m, bool(wv))
    assert nbytes == expect
    assert all(v % 16 == 0 for v in offs.values())
    # key codes 2 bits, QJL 1 bit, value codes 4 bits, three fp16 per token
    assert offs["qs"] - offs["kc"] == 128 * d * 2 // 8
    assert (offs["vc"] - offs["qs"] if wv else offs["kn"] - offs["qs"]) == 128 * m // 8


def _empty_records(N, d, m):
    z = lambda *s: np.zeros(s, np.int32)
    return dict(sign=z(N, d), mag=z(N, d), qbits=z(N, m), n=np.ones(N), gamma=np.zeros(N),
                vcode=z(N, d), vn=np.ones(N))


def test_golden_format_examples(O):
    g = _golden()
    d = m = 64
    nbytes, offs = O.page_layout(d, m, True)
    pool = np.zeros(nbytes, np.uint8)
    rec = _empty_records(6, d, m)
    for j in map(int, g["key"]["sign"].split(",")):
        rec["sign"][0, j] = 1
    for j in map(int, g["key"]["mag"].split(",")):
        rec["mag"][0, j] = 1
    for i in map(int, g["qjl"]["bits"].split(",")):
        rec["qbits"][0, i] = 1
    cj = int(g["value"]["coord"])
    rec["vcode"][2, cj] = int(g["value"]["slot2"], 16)
    rec["vcode"][3, cj] = int(g["value"]["slot3"], 16)
    cj2 = int(g["value2"]["coord"])
    rec["vcode"][4, cj2] = int(g["value2"]["slot26"], 16)
    rec["vcode"][5, cj2] = int(g["value2"]["slot27"], 16)
    O.pack(pool, nbytes, d, m, True, [0] * 6, [0, 1, 2, 3, 26, 27], rec)
    word = lambda off: int.from_bytes(pool[off:off + 4].tobytes(), "little")
    assert word(offs["kc"]) == int(g["key"]["word0"], 16)
    assert word(offs["qs"]) == int(g["qjl"]["word0"], 16)
    assert pool[offs["vc"] + int(g["value"]["offset"])] == int(g["value"]["byte"], 16)
    assert pool[offs["vc"] + int(g["value2"]["offset"])] == int(g["value2"]["byte"], 16)
    assert np.count_nonzero(pool[offs["vc"]:offs["kn"]]) == 2


@pytest.mark.parametrize("d,m", D_M)
def test_value_byte_positions(O, d, m):
    """Every (token pair, coordinate) lands on its own byte of the value
    section (a bijection onto its 64 d bytes), and all bytes of a 16-token
    block stay inside that block's 8 d bytes."""
    nbytes, offs = O.page_layout(d, m, True)
    seen = set()
    for p in range(64):
        for j in range(d):
            pool = np.zeros(nbytes, np.uint8)
            rec = _empty_records(1, d, m)
            rec["vcode"][0, j] = 0x9
            O.pack(pool, nbytes, d, m, True, [0], [2 * p + 1], rec)
            sec = pool[offs["vc"]: offs["vc"] + 64 * d]
            (pos,) = np.nonzero(sec)
            assert len(pos) == 1 and sec[pos[0]] == 0x90
            assert pos[0] // (8 * d) == p // 8
            seen.add(int(pos[0]))
    assert len(seen) == 64 * d


@pytest.mark.parametrize("d,m", D_M)
def test_pack_unpack_round_trip(O, d, m):
    rng = np.random.default_rng(1)
    N = 300
    nbytes, _ = O.page_layout(d, m, True)
    pool = rng.integers(0, 256, size=3 * nbytes, dtype=np.uint8)  # garbage elsewhere
    rec = dict(sign=rng.integers(0, 2, (N, d)), mag=rng.integers(0, 2, (N, d)),
               qbits=rng.integers(0, 2, (N, m)),
               n=np.float16(rng.uniform(0.1, 30, N)).astype(np.float64),
               gamma=np.float16(rng.uniform(0, 1, N)).astype(np.float64),
               vcode=rng.integers(0, 16, (N, d)),
               vn=np.float16(rng.uniform(0.1, 30, N)).astype(np.float64))
    perm = rng.permutation(3 * 128)[:N]
    pid, slot = perm // 128, perm % 128
    O.pack(pool, nbytes, d, m, True, pid, slot, rec)
    back = O.unpack(pool, nbytes, d, m, True, pid, slot)
    for k in rec:
        assert np.array_equal(np.asarray(back[k], rec[k].dtype), rec[k]), k
    # keys-only pages keep the key fields
    nb2, _ = O.page_layout(d, m, False)
    pool2 = np.zeros(3 * nb2, np.uint8)
    O.pack(pool2, nb2, d, m, False, pid, slot, {k: rec[k] for k in ("sign", "mag", "qbits", "n", "gamma")})
    back2 = O.unpack(pool2, nb2, d, m, False, pid, slot)
    for k in ("sign", "mag", "qbits", "n", "gamma"):
        assert np.array_equal(np.asarray(back2[k], rec[k].dtype), rec[k]), k


@pytest.mark.parametrize("d", [64, 128])
def test_quantiser_is_nearest_centroid(O, d):
    """Codes equal the exhaustive nearest of all 2^b signed levels to x_rot/n,
    except within rounding of a decision boundary."""
    P = O.Params(d, seed=2)
    rng = np.random.default_rng(3)
    x = rng.standard_normal((400, d)) * rng.lognormal(0, 1, d)
    for is_key, cpos, tpos in ((True, P.kc, P.kt), (False, P.vc, P.vt)):
        rec = O.encode(P, x, is_key)
        n = rec["n"][:, None]
        u = rec["xrot"] / n
        levels = np.concatenate([-cpos[::-1], cpos])
        nearest = levels[np.argmin(np.abs(u[..., None] - levels), axis=-1)]
        got = np.where(rec["sign"] == 1, -1.0, 1.0) * cpos[rec["mag"]]
        near_edge = np.min(np.abs(np.abs(u)[..., None] - tpos), axis=-1) < 1e-5 * np.abs(u) + 1e-9
        assert np.all((got == nearest) | near_edge)
        assert near_edge.mean() < 1e-3
        # the stored norm is fp16(|x|)
        assert np.array_equal(n[:, 0], np.float16(np.linalg.norm(x, axis=1)).astype(np.float64))


def test_zero_vector(O):
    P = O.Params(64)
    rec = O.encode(P, np.zeros((2, 64)), True)
    for k in ("sign", "mag", "qbits", "n", "gamma"):
        assert not np.any(rec[k])


def test_residual_norm_and_sketch_signs(O):
    P = O.Params(64, seed=4)
    x = np.random.default_rng(5).standard_normal((50, 64))
    rec = O.encode(P, x, True)
    chat = np.where(rec["sign"] == 1, -1.0, 1.0) * P.kc[rec["mag"]]
    r = rec["xrot"] / rec["n"][:, None] - chat
    assert np.array_equal(rec["gamma"], np.float16(np.linalg.norm(r, axis=1)).astype(np.float64))
    p = r @ P.S.T
    assert np.array_equal(rec["qbits"], (p < 0).astype(np.int32))


def test_qjl_estimator_unbiased_monte_carlo(O):
    """Mean of the estimate of <q, r> over 1e5 independent S is within three
    standard errors; its variance is within 5% of
    [(pi/2)|q|^2|r|^2 - <q,r>^2]/m (from E[(g.q)^2] = |q|^2, g Gaussian)."""
    d = 64
    rng = np.random.default_rng(6)
    q, r = rng.standard_normal(d), 0.2 * rng.standard_normal(d)
    trials = 100_000
    mean, var = O.qjl_montecarlo(q, r, trials, 1000)
    exact = q @ r
    assert abs(mean - exact) <= 3 * math.sqrt(var / trials)
    closed = ((math.pi / 2) * (q @ q) * (r @ r) - exact ** 2) / d
    assert abs(var / closed - 1.0) < 0.05


def test_qjl_estimate_matches_exact_for_large_m(O):
    d, m = 32, 16384
    rng = np.random.default_rng(7)
    q, r = rng.standard_normal(d), rng.standard_normal(d)
    S = O.qjl_matrix(m, d, 77)
    bits = (S @ r < 0).astype(np.int32)
    est = O.qjl_estimate(S @ q, bits, float(np.linalg.norm(r)))
    sd = math.sqrt(((math.pi / 2) * (q @ q) * (r @ r) - (q @ r) ** 2) / m)
    assert abs(est - q @ r) < 4 * sd


def test_value_distortion_matches_codebook(O):
    """Relative error of n * Pi^T c_hat equals d times the 4-bit codebook MSE."""
    d = 128
    P = O.Params(d, seed=8)
    x = np.random.default_rng(9).standard_normal((3000, d))
    rec = O.encode(P, x, False)
    chat = np.where(rec["sign"] == 1, -1.0, 1.0) * P.vc[rec["mag"]]
    xhat = rec["n"][:, None] * (chat @ P.pi32)
    rel = np.sum((x - xhat) ** 2, axis=1) / np.sum(x ** 2, axis=1)
    assert abs(rel.mean() / (d * P.value_mse) - 1.0) < 0.03
