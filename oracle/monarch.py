"""Monarch's hot/cold decode cache, step by step, on top of the CPU oracle.

TEST INFRASTRUCTURE ONLY (see the package docstring): imported by ``tests/``
and ``bench.py``'s reference leg, never by the product path.  Plain Python
over the oracle's encoder, packer and attention; no CUDA code is shared.

What it follows ("Monarch v3: NES-inspiriertes KV-Paging", openclawradar.com):
  - section "Wie es funktioniert": the last N tokens stay hot at full
    precision, older tokens are compressed into the cold region;
  - section "Vereinfachte Decode-Schleife": per step the query scores the hot
    tokens, reads the cold pages only if max(scores_hot) < threshold, takes
    one softmax, then evicts the oldest hot tokens to cold when the hot
    window is longer than window_size.

Readings where the pages leave a step open:
  - Eviction block E: when a step leaves at least window + E hot tokens, the
    oldest E of them are compressed and appended to the cold pages.  E = 1 is
    the loop as written (evict whenever len(kv_hot) > window_size); larger E
    compresses a block at a time and keeps between window and window + E - 1
    tokens hot.
  - All kv heads of a sequence share one hot length (a token enters and leaves
    the hot window for every head at once).
  - The new token of a step is appended before attention, so it attends to
    itself (as in standard decoding).
  - The gate is the oracle attention's: per query head, on the raw hot scores.
  - Attention-weighted promotion with stickiness (section "Wie es
    funktioniert": tokens with high attention move back to the hot region,
    with a sticking mechanism against thrashing; section "Vereinfachte
    Decode-Schleife": cold tokens read in a step are moved to the hot region
    for the next step; section "Wie man es ausprobiert": promotion threshold
    0.15, sticky threshold 3).  A cold position's weight in a step is its
    largest softmax probability over the query heads of the sequence that
    read the cold tier (a position, not a kv head, moves: all kv heads of a
    sequence share one hot window).  A weight at or above the threshold
    counts the step, a weight below it resets the count (consecutive
    steps); a position whose count reaches the sticky threshold moves back
    after the step's attention: its decompressed key and value (n Pi^T c_hat,
    the residual's sketch being no vector, and n_v Pi^T c_hat_v, rounded to
    fp16) join the hot window of every kv head as its newest tokens, its
    cold slot is masked (attention skips it from then on) and its count
    returns to 0.  At most max_per_step positions move per step, in
    increasing position order, and never more than leave one free ring slot
    for the next step's token; the others keep their counts.  Eviction runs
    after promotion.

Parity status: pinned by ``tests/test_oracle_monarch.py`` (window
invariant, token placement against the appended sequence, attention with a
shut gate against torch's scaled_dot_product_attention; the promotion path:
its attention against the oracle's C attention and against SDPA without the
masked tokens, counting, moving, masking and the per-step and ring limits).
"""
import numpy as np

from . import attention, cold_logits, encode, pack, page_layout, unpack


def _f16(a):
    """Round to the nearest fp16 value (ties to even), widened to fp64."""
    return np.asarray(a, np.float64).astype(np.float16).astype(np.float64)


class MonarchCache:
    """State for B sequences x Hkv kv heads: hot tokens in age order (fp16
    values widened to fp64) and cold records in the oracle's page pool."""

    def __init__(self, params, B, Hkv, window, evict_block, page_table, cold_len=None,
                 pool=None, hot_k=None, hot_v=None, promotion=None, W_max=None):
        """promotion: None, or dict(threshold, sticky, max_per_step); W_max:
        the ring size (needed with promotion)."""
        self.P = params
        self.B, self.Hkv, self.d = B, Hkv, params.d
        self.window, self.E = int(window), int(evict_block)
        self.table = np.ascontiguousarray(page_table, np.int32)
        self.page_bytes, _ = page_layout(self.d, params.m, True)
        n_pages = int(self.table.max()) + 1 if self.table.size else 1
        self.pool = (np.zeros(n_pages * self.page_bytes, np.uint8) if pool is None
                     else np.ascontiguousarray(pool, np.uint8).reshape(-1).copy())
        self.cold_len = (np.zeros(B, np.int32) if cold_len is None
                         else np.asarray(cold_len, np.int32).copy())
        # hot[b][h]: list of (k, v) rows, oldest first
        self.hot = [[[] for _ in range(Hkv)] for _ in range(B)]
        self.promo = promotion
        self.W_max = W_max
        cap = self.table.shape[-1] * 128
        self.cold_mask = np.zeros((B, cap), bool)  # moved back: skipped by attention
        self.counts = np.zeros((B, cap), np.int32)   # consecutive counted steps
        if hot_k is not None:
            for b in range(B):
                for h in range(Hkv):
                    for t in range(len(hot_k[b][h])):
                        self.hot[b][h].append((np.asarray(hot_k[b][h][t], np.float64),
                                               np.asarray(hot_v[b][h][t], np.float64)))

    def hot_len(self, b):
        return len(self.hot[b][0])

    def _hot_arrays(self):
        W = max(1, max(self.hot_len(b) for b in range(self.B)))
        k = np.zeros((self.B, self.Hkv, W, self.d))
        v = np.zeros((self.B, self.Hkv, W, self.d))
        for b in range(self.B):
            for h in range(self.Hkv):
                for t, (kr, vr) in enumerate(self.hot[b][h]):
                    k[b, h, t] = kr
                    v[b, h, t] = vr
        return k, v

    def append(self, k_new, v_new):
        """k_new, v_new [B, Hkv, d]: rounded to fp16 (the hot window's type)."""
        f16 = lambda a: np.float16(a).astype(np.float64)
        for b in range(self.B):
            for h in range(self.Hkv):
                self.hot[b][h].append((f16(k_new[b, h]), f16(v_new[b, h])))

    def attend(self, q, scale, threshold=None):
        """Attention of q [B, Hq, d] over hot and (gated) cold tokens.
        Returns out [B, Hq, d] and, with a threshold, the gate decisions."""
        k, v = self._hot_arrays()
        hl = np.array([self.hot_len(b) for b in range(self.B)], np.int32)
        res = attention(self.P, q, self.Hkv, scale, k, v, hl, self.pool, self.page_bytes,
                        self.table, self.cold_len, threshold=threshold)
        G = q.shape[1] // self.Hkv
        out = res[0].reshape(self.B, self.Hkv * G, self.d)
        opened = None if threshold is None else res[2].reshape(self.B, self.Hkv * G)
        return out, opened

    def _cold_values(self, b, h, cl):
        """Reconstructed cold values n_v Pi^T c_hat_v [cl, d] of group (b, h)."""
        t = np.arange(cl)
        rec = unpack(self.pool, self.page_bytes, self.d, self.P.m, True, self.table[b, h, t // 128],
                     t % 128)
        chat = np.where(rec["vcode"] >> 3, -1.0, 1.0) * self.P.vc[rec["vcode"] & 7]
        return rec["vn"][:, None] * (chat @ self.P.pi32)

    def attend_weights(self, q, scale, threshold=None):
        """The attention of attend() computed step by step in fp64 (cold scores
        from the oracle's scorer, values n_v Pi^T c_hat_v, one softmax per query
        head over its hot tokens and, where its gate opens, the cold tokens not
        moved back), also returning per sequence the largest weight of every
        cold position over the query heads that read the cold tier."""
        B, Hq, d = q.shape
        G = Hq // self.Hkv
        out = np.zeros((B, Hq, d))
        opened = np.zeros((B, Hq), np.int32)
        wmax = []
        for b in range(B):
            cl, hl = int(self.cold_len[b]), self.hot_len(b)
            live = ~self.cold_mask[b, :cl]
            w = np.zeros(cl)
            for h in range(self.Hkv):
                qg = np.asarray(q[b, h * G:(h + 1) * G], np.float64)
                kh = np.array([kv[0] for kv in self.hot[b][h]]).reshape(hl, d)
                vh = np.array([kv[1] for kv in self.hot[b][h]]).reshape(hl, d)
                raw = qg @ kh.T
                cs = cold_logits(self.P, qg, scale, self.pool, self.page_bytes, self.table[b, h], cl) \
                    if cl else np.zeros((G, 0))
                cv = self._cold_values(b, h, cl) if cl else np.zeros((0, d))
                for g in range(G):
                    gmax = raw[g].max() if hl else -np.inf
                    op = threshold is None or gmax < threshold
                    opened[b, h * G + g] = op
                    lc = cs[g][live] if op else np.zeros(0)
                    logits = np.concatenate([lc, raw[g] * scale])
                    if len(logits) == 0:
                        continue
                    e = np.exp(logits - logits.max())
                    p = e / e.sum()
                    out[b, h * G + g] = p @ np.concatenate([cv[live] if op else np.zeros((0, d)), vh])
                    if op:
                        wc = np.zeros(cl)
                        wc[live] = p[:len(lc)]
                        w = np.maximum(w, wc)
            wmax.append(w)
        return out, opened, wmax

    def promote(self, wmax):
        """Count, then move back the positions whose count reached the sticky
        threshold (see the module docstring); returns the moved positions per
        sequence."""
        pr = self.promo
        moved = []
        for b in range(self.B):
            cl = int(self.cold_len[b])
            live = ~self.cold_mask[b, :cl]
            hit = live & (wmax[b] >= pr["threshold"])
            self.counts[b, :cl] = np.where(hit, np.minimum(self.counts[b, :cl] + 1, 255), 0)
            cand = np.nonzero(live & (self.counts[b, :cl] >= pr["sticky"]))[0]
            room = max(0, self.W_max - 1 - self.hot_len(b))
            chosen = cand[:min(int(pr["max_per_step"]), room)]
            for h in range(self.Hkv):
                if len(chosen) == 0:
                    break
                rec = unpack(self.pool, self.page_bytes, self.d, self.P.m, True,
                             self.table[b, h, chosen // 128], chosen % 128)
                ck = np.where(rec["sign"] == 1, -1.0, 1.0) * self.P.kc[rec["mag"]]
                cv = np.where(rec["vcode"] >> 3, -1.0, 1.0) * self.P.vc[rec["vcode"] & 7]
                kd = _f16(rec["n"][:, None] * (ck @ self.P.pi32))
                vd = _f16(rec["vn"][:, None] * (cv @ self.P.pi32))
                for i in range(len(chosen)):
                    self.hot[b][h].append((kd[i], vd[i]))
            self.cold_mask[b, chosen] = True
            self.counts[b, chosen] = 0
            moved.append(chosen)
        return moved

    def evict(self):
        """Move the oldest E hot tokens of every sequence holding at least
        window + E of them to the cold pages; returns how many per sequence."""
        moved = np.zeros(self.B, np.int32)
        for b in range(self.B):
            if self.hot_len(b) < self.window + self.E:
                continue
            c0 = int(self.cold_len[b])
            pos = c0 + np.arange(self.E)
            for h in range(self.Hkv):
                old = self.hot[b][h][:self.E]
                K = np.stack([kv[0] for kv in old])
                V = np.stack([kv[1] for kv in old])
                kr, vr = encode(self.P, K, True), encode(self.P, V, False)
                rec = dict(sign=kr["sign"], mag=kr["mag"], qbits=kr["qbits"], n=kr["n"],
                           gamma=kr["gamma"], vcode=vr["vcode"], vn=vr["vn"])
                pack(self.pool, self.page_bytes, self.d, self.P.m, True,
                     self.table[b, h, pos // 128], pos % 128, rec)
                del self.hot[b][h][:self.E]
            self.cold_len[b] += self.E
            moved[b] = self.E
        return moved

    def step(self, q, k_new, v_new, scale, threshold=None):
        """One decode step: append, attend, (promote,) evict."""
        self.append(k_new, v_new)
        if self.promo is None:
            out, opened = self.attend(q, scale, threshold)
        else:
            out, opened, wmax = self.attend_weights(q, scale, threshold)
            self.promote(wmax)
        self.evict()
        return out, opened
