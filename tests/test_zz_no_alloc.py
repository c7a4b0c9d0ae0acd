"""tq_decode_attention_noalloc -- the decode call for callers that may not
allocate device memory (a plugin whose host runtime owns the device-memory
budget, a serving loop that must not block on the allocator) and so cannot
pass a workspace -- against tq_decode_attention with a caller workspace, on
the same inputs, through the C ABI.  Two calls in a row with different
problem sizes show that the shared scratch keeps nothing the next call
depends on.  This file is collected last so that a run stopping at the first
failure has already run every other test; it also passes alone."""
import ctypes as C

import numpy as np
import pytest

import compressed_kv_decode_b200 as tq
from compressed_kv_decode_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _case(torch, ctx, seed, B, Hkv, G, d, hot, max_pages, qdtype):
    """Random but valid decode inputs on the device (pages of random records)."""
    dev = "cuda"
    nb = ctx.page_bytes(True)
    table, n_pages = W.random_page_table(seed, B, Hkv, max_pages, spare=1)
    # fp16 norm fields of a values page: 8 blocks of 16 slots, each block
    # 14 d + 96 bytes ending in 16 (n, gamma) pairs and 16 value norms
    blk, s = 14 * d + 96, np.arange(128)
    kn = (s // 16) * blk + 12 * d + 2 * d + 4 * (s % 16)
    pool = W.random_page_bytes(seed + 1, n_pages, nb, {"kn": kn, "kg": kn + 2,
                                                       "vn": (s // 16) * blk + 14 * d + 64 + 2 * (s % 16)})
    rng = np.random.default_rng(seed + 2)
    k_hot = rng.standard_normal((B, Hkv, hot, d)).astype(np.float16)
    v_hot = rng.standard_normal((B, Hkv, hot, d)).astype(np.float16)
    q = rng.standard_normal((B, Hkv * G, d))
    cold_len = rng.integers(0, max_pages * 128 + 1, B).astype(np.int32)
    hot_len = rng.integers(0, hot + 1, B).astype(np.int32)
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev)
    return dict(q=t(q).to(getattr(torch, qdtype)), k_hot=t(k_hot), v_hot=t(v_hot),
                hot_len=t(hot_len), pool=t(pool), table=t(table), cold_len=t(cold_len),
                B=B, Hq=Hkv * G, Hkv=Hkv, d=d, max_pages=max_pages, hot=hot)


def _with_workspace(torch, ctx, c):
    out = torch.empty((c["B"], c["Hq"], c["d"]), dtype=torch.float32, device="cuda")
    ws = ctx.workspace(c["B"], c["Hq"], c["Hkv"], c["max_pages"], c["hot"])
    tq.tq_decode_attention(ctx.handle, c["q"], c["k_hot"], c["v_hot"], c["hot_len"], c["pool"],
                           c["table"], c["cold_len"], out, ws, c["Hkv"])
    torch.cuda.synchronize()
    return out.cpu().numpy()


def _without_workspace(torch, ctx, c):
    out = torch.full((c["B"], c["Hq"], c["d"]), float("nan"), dtype=torch.float32, device="cuda")
    tq.tq_decode_attention_noalloc(ctx.handle, c["q"], c["k_hot"], c["v_hot"], c["hot_len"],
                                   c["pool"], c["table"], c["cold_len"], out, c["Hkv"])
    torch.cuda.synchronize()
    return out.cpu().numpy()


def test_noalloc_matches_workspace_call_twice_in_a_row():
    import torch
    ctx = tq.Context(128, seed=0)
    big = _case(torch, ctx, 11, B=4, Hkv=8, G=4, d=128, hot=64, max_pages=40, qdtype="bfloat16")
    small = _case(torch, ctx, 21, B=3, Hkv=2, G=8, d=128, hot=16, max_pages=3, qdtype="float16")
    for c in (big, small):
        ref = _with_workspace(torch, ctx, c)
        got = _without_workspace(torch, ctx, c)
        assert tq.tq_get_error(ctx.handle) == tq.TQ_OK
        # the same deterministic kernels on the same inputs: equal bit for bit,
        # so anything left in the shared scratch by the previous call would show
        assert np.array_equal(got, ref)
    ctx.close()


def test_noalloc_rejects_workspace_beyond_its_scratch():
    import torch
    ctx = tq.Context(128, seed=0)
    need = tq.tq_workspace_bytes(ctx.handle, 1024, 32, 8, 4, 16)
    assert need > tq.TQ_NOALLOC_SCRATCH_BYTES
    q = torch.zeros((1024, 32, 128), dtype=torch.bfloat16, device="cuda")
    out = torch.zeros((1024, 32, 128), dtype=torch.float32, device="cuda")
    hot = torch.zeros((1024, 8, 16, 128), dtype=torch.float16, device="cuda")
    lens = torch.zeros(1024, dtype=torch.int32, device="cuda")
    table = torch.zeros((1024, 8, 4), dtype=torch.int32, device="cuda")
    pool = torch.zeros((1, ctx.page_bytes(True)), dtype=torch.uint8, device="cuda")
    with pytest.raises(tq.TQError) as e:
        tq.tq_decode_attention_noalloc(ctx.handle, q, hot, hot, lens, pool, table, lens, out, 8)
    assert e.value.status == tq.TQ_ERR_CAPACITY
    ctx.close()
