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
    rows = []
    for line in open(path):
        if line.strip() and not line.startswith("#"):
            kind, *fields = line.split()
            rows.append((kind, dict(f.split("=") for f in fields)))
    return rows


def _one(rows, kind):
    (row,) = [r for k, r in rows if k == kind]
    return row


# The format as the header states it (include/tq.h, tq_page_bytes), typed
# here from that text: the bit of plane index j for token t of a block, and
# the value byte of coordinate j for token t of a block.
def _plane_pos(j, t):
    return 16 * (4 * (j // 32) + (j // 4) % 4) + 4 * (2 * ((j // 16) % 2) + t // 8) + j % 4, t % 8


def _value_pos(j, t):
    q = t // 2
    c, th = q % 4, q // 4
    i, g, jh = j // 16, j % 8, (j % 16) // 8
    return (i // 4) * 512 + (4 * g + c) * 16 + (i % 4) * 4 + jh + 2 * th


@pytest.mark.parametrize("d,m,wv,expect", [(128, 128, 1, 15104), (128, 128, 0, 6656),
                                           (64, 64, 1, 7936), (64, 64, 0, 3584)])
def test_page_bytes(O, d, m, wv, expect):
    nbytes, offs = O.page_layout(d, m, bool(wv))
    assert nbytes == expect
    if wv:  # 8 blocks of 16 slots; 118 (d=128) or 62 (d=64) bytes per token
        assert offs["block"] * 8 == nbytes and offs["block"] == 16 * (12 * d + 2 * m + 96) // 16
        assert [offs[k] for k in ("kc", "kl", "qs", "vc", "kn", "vn")] == \
            [0, 2 * d, 4 * d, 4 * d + 2 * m, 12 * d + 2 * m, 12 * d + 2 * m + 64]
        assert offs["kg"] == offs["kn"] + 2
        assert all(offs[k] % 16 == 0 for k in ("kc", "kl", "qs", "vc", "kn", "vn", "block"))
    else:  # record layout: key codes 2 bits, QJL 1 bit, two fp16 per token
        assert offs["block"] == 0
        assert all(v % 16 == 0 for v in offs.values())
        assert offs["qs"] - offs["kc"] == 128 * d * 2 // 8
        assert offs["kn"] - offs["qs"] == 128 * m // 8


def _empty_records(N, d, m):
    z = lambda *s: np.zeros(s, np.int32)
    return dict(sign=z(N, d), mag=z(N, d), qbits=z(N, m), n=np.ones(N), gamma=np.zeros(N),
                vcode=z(N, d), vn=np.ones(N))


def test_golden_record_layout_examples(O):
    """Keys-only pages: hand-worked key and QJL words."""
    g = _golden()
    d = m = 64
    nbytes, offs = O.page_layout(d, m, False)
    pool = np.zeros(nbytes, np.uint8)
    rec = _empty_records(1, d, m)
    key, qjl = _one(g, "key"), _one(g, "qjl")
    for j in map(int, key["sign"].split(",")):
        rec["sign"][0, j] = 1
    for j in map(int, key["mag"].split(",")):
        rec["mag"][0, j] = 1
    for i in map(int, qjl["bits"].split(",")):
        rec["qbits"][0, i] = 1
    O.pack(pool, nbytes, d, m, False, [0], [0], {k: rec[k] for k in ("sign", "mag", "qbits", "n", "gamma")})
    word = lambda off: int.from_bytes(pool[off:off + 4].tobytes(), "little")
    assert word(offs["kc"]) == int(key["word0"], 16)
    assert word(offs["qs"]) == int(qjl["word0"], 16)


def test_golden_block_layout_examples(O):
    """Pages with values: hand-worked plane words, norms and value bytes."""
    g = _golden()
    d = m = 64
    nbytes, offs = O.page_layout(d, m, True)
    pool = np.zeros(nbytes, np.uint8)
    b1, b2 = _one(g, "block"), _one(g, "block2")
    v1, v2 = _one(g, "value"), _one(g, "value2")
    rec = _empty_records(2, d, m)
    vrec = _empty_records(4, d, m)
    ints = lambda s: [int(x) for x in s.split(",")]
    for j in ints(b1["sign"]):
        rec["sign"][0, j] = 1
    for j in ints(b1["mag"]):
        rec["mag"][0, j] = 1
    for i in ints(b1["qjl"]):
        rec["qbits"][0, i] = 1
    rec["n"][0], rec["gamma"][0], rec["vn"][0] = float(b1["n"]), float(b1["gamma"]), float(b1["vn"])
    for j in ints(b2["sign"]):
        rec["sign"][1, j] = 1
    cj, cj2 = int(v1["coord"]), int(v2["coord"])
    vrec["vcode"][0, cj] = int(v1["slot2"], 16)
    vrec["vcode"][1, cj] = int(v1["slot3"], 16)
    vrec["vcode"][2, cj2] = int(v2["slot26"], 16)
    vrec["vcode"][3, cj2] = int(v2["slot27"], 16)
    O.pack(pool, nbytes, d, m, True, [0] * 2, [int(b1["slot"]), int(b2["slot"])], rec)
    vpool = np.zeros(nbytes, np.uint8)  # the value examples on a page of their own
    O.pack(vpool, nbytes, d, m, True, [0] * 4, [2, 3, 26, 27], vrec)
    sec = {"kh": offs["kc"], "kl": offs["kl"], "qs": offs["qs"], "nk": offs["kn"], "vn": offs["vn"]}
    word = lambda off: int.from_bytes(pool[off:off + 4].tobytes(), "little")
    assert int(b1["base"]) == offs["block"] == int(b2["base"])
    for kind, r in g:
        if kind in ("block_word", "block_word2"):
            assert word(offs["block"] + sec[r["section"]] + int(r["off"])) == int(r["word"], 16), r
        if kind == "block_half":
            off = offs["block"] + sec[r["section"]] + int(r["off"])
            assert int.from_bytes(pool[off:off + 2].tobytes(), "little") == int(r["half"], 16)
    for v in (v1, v2):
        assert vpool[int(v["block"]) * offs["block"] + offs["vc"] + int(v["offset"])] == int(v["byte"], 16)
    assert sum(np.count_nonzero(vpool[b * offs["block"] + offs["vc"]:b * offs["block"] + offs["kn"]])
               for b in range(8)) == 2


@pytest.mark.parametrize("d,m", D_M)
def test_block_plane_positions(O, d, m):
    """Every (token, index) bit of the H, L and QJL planes lands on the byte
    and bit the format states, inside its block's plane (each plane a
    bijection of the block's 16 tokens x d indices onto its 2d bytes)."""
    nbytes, offs = O.page_layout(d, m, True)
    blk = offs["block"]
    for plane, size in (("kc", d), ("kl", d), ("qs", m)):
        seen = set()
        for slot in list(range(16, 32)) + [0, 77, 127]:
            for j in range(size):
                pool = np.zeros(nbytes, np.uint8)
                rec = _empty_records(1, d, m)
                if plane == "kc":    # H = 1 - sign: every sign set except coordinate j
                    rec["sign"][0] = 1
                    rec["sign"][0, j] = 0
                    rec["mag"][0] = 1     # L = 0 everywhere
                    rec["mag"][0, j] = 0
                elif plane == "kl":  # L = sign XOR mag: one magnitude bit, no signs
                    rec["mag"][0, j] = 1
                else:
                    rec["qbits"][0, j] = 1
                O.pack(pool, nbytes, d, m, True, [0], [slot], rec)
                base = (slot // 16) * blk + offs[plane]
                sec = pool[base:base + 2 * size]
                (pos,) = np.nonzero(sec)
                byte, bit = _plane_pos(j, slot % 16)
                assert list(pos) == [byte] and sec[byte] == 1 << bit, (plane, slot, j)
                if 16 <= slot < 32:
                    seen.add((byte, bit))
        assert len(seen) == 16 * size


@pytest.mark.parametrize("d,m", D_M)
def test_value_byte_positions(O, d, m):
    """Every (token, coordinate) lands on the byte the format states, in the
    nibble of its token's parity, inside its block's value section (a
    bijection onto the block's 8 d bytes)."""
    nbytes, offs = O.page_layout(d, m, True)
    blk = offs["block"]
    seen = set()
    for slot in range(32, 48):
        for j in range(d):
            pool = np.zeros(nbytes, np.uint8)
            rec = _empty_records(1, d, m)
            rec["vcode"][0, j] = 0x9
            O.pack(pool, nbytes, d, m, True, [0], [slot], rec)
            base = (slot // 16) * blk + offs["vc"]
            sec = pool[base: base + 8 * d]
            (pos,) = np.nonzero(sec)
            assert list(pos) == [_value_pos(j, slot % 16)]
            assert sec[pos[0]] == (0x90 if slot & 1 else 0x09)
            seen.add(int(pos[0]) * 2 + (slot & 1))
    assert len(seen) == 16 * d


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
