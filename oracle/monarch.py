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

Parity status: pinned by ``tests/test_oracle_monarch.py`` (window
invariant, token placement against the appended sequence, attention with a
shut gate against torch's scaled_dot_product_attention).
"""
import numpy as np

from . import attention, encode, pack, page_layout


class MonarchCache:
    """State for B sequences x Hkv kv heads: hot tokens in age order (fp16
    values widened to fp64) and cold records in the oracle's page pool."""

    def __init__(self, params, B, Hkv, window, evict_block, page_table, cold_len=None,
                 pool=None, hot_k=None, hot_v=None):
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
        """One decode step: append, attend, evict."""
        self.append(k_new, v_new)
        out, opened = self.attend(q, scale, threshold)
        self.evict()
        return out, opened
