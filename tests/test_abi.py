"""Host-side checks of the C-ABI library (no GPU needed): it loads, exports
every entry point include/tq.h declares, validates arguments, and its own
host-side table generation (written independently of the oracle) agrees
with the oracle's tables."""
import ctypes as C
import os
import re

import numpy as np
import pytest

import compressed_kv_decode_b200 as tq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "tq.h")).read()
    return sorted(set(re.findall(r"TQ_API[^;(]*?\b(tq_\w+)\s*\(", src)))


def test_exports_every_declared_symbol():
    names = _declared()
    assert len(names) >= 12
    L = tq.lib()
    for n in names:
        assert hasattr(L, n), n


def test_range_checked_build_exports_every_declared_symbol():
    """libtq_debug.so (the same sources compiled with TQ_DEBUG) is built
    in-tree beside libtq.so and exports the same entry points."""
    from compressed_kv_decode_b200 import build
    path = build.build(debug=True)
    assert path.endswith("libtq_debug.so") and os.path.exists(path)
    L = C.CDLL(path)
    for n in _declared():
        assert hasattr(L, n), n


def test_status_strings():
    for s in range(8):
        assert tq.status_string(s) and "unknown" not in tq.status_string(s)
    assert "unknown" in tq.status_string(99)


@pytest.mark.parametrize("d,seed", [(64, 0), (128, 7)])
def test_host_tables_match_oracle(O, d, seed):
    lib_t = tq.tq_generate_params(tq.make_config(d, seed))
    P = O.Params(d, seed=seed)
    # QJL matrix: same published generator, rounded to fp16 -> identical
    assert np.array_equal(lib_t["qjl"].astype(np.float64), P.S)
    # rotation: Gram-Schmidt (library) vs Householder (oracle), both fp64, then fp32
    assert np.abs(lib_t["rot"].astype(np.float64) - P.pi64).max() <= 1e-6
    assert np.mean(lib_t["rot"].astype(np.float64) == P.pi32) > 0.999
    for a, b in (("key_c", P.kc64), ("key_t", P.kt64), ("val_c", P.vc64), ("val_t", P.vt64)):
        got = lib_t[a].astype(np.float64)
        assert np.abs(got - b).max() <= 4e-8 * max(1.0, np.abs(b).max()), a
        assert np.array_equal(lib_t[a], b.astype(np.float32)), a


def test_generate_params_rejects_bad_config():
    bad = tq.make_config(100, 0)  # not a multiple of 16
    with pytest.raises(tq.TQError) as e:
        tq.tq_generate_params(bad)
    assert e.value.status == tq.TQ_ERR_INVALID_ARG


def test_null_context_and_arguments():
    L = tq.lib()
    assert L.tq_page_bytes(None, 1) == 0
    assert L.tq_workspace_bytes(None, 1, 1, 1, 1, 1) == 0
    assert L.tq_get_error(None) == tq.TQ_ERR_INVALID_ARG
    # ctx, q, q_dtype, B, Hq, Hkv, scale, k_hot, v_hot, W_max, hot_len, pool, pool_pages,
    # page_table, max_pages, cold_len, out, workspace, ws_bytes, stream
    args = [None, None, 0, 1, 1, 1, 0.0, None, None, 0, None, None, 0, None, 0, None, None, None, 0, None]
    assert L.tq_decode_attention(*args) == tq.TQ_ERR_INVALID_ARG
    assert L.tq_score_topk(None, None, 1, None, 1, 1, None, None, None, 0, None) == tq.TQ_ERR_INVALID_ARG
    assert L.tq_compress_append(None, None, None, 0, 0, 1, 1, 1, None, 1, None, 1, None, None) == tq.TQ_ERR_INVALID_ARG
    L.tq_destroy(None)


def test_init_without_device_fails_cleanly():
    import torch
    if torch.cuda.is_available():
        pytest.skip("a device is present")
    h = C.c_void_p()
    cfg = tq.make_config(128, 0)
    st = tq.lib().tq_init_codebook(C.byref(cfg), C.byref(h))
    assert st == tq.TQ_ERR_CUDA and not h.value


def test_null_context_on_the_next_row_entries():
    """The gated decode, Monarch and Tensor Cache steps, the stage-1 variants
    and the Self-Indexing calls reject a null context (and report no sizes)
    on the host, before any device call."""
    L = tq.lib()
    INV = tq.TQ_ERR_INVALID_ARG
    assert L.tq_monarch_workspace_bytes(None, 1, 1, 1, 1, 8, 1) == 0
    assert L.tq_tensor_cache_workspace_bytes(None, 1, 1, 1, 8) == 0
    assert L.tq_stage1_code_bytes(None, tq.TQ_STAGE1_POLAR, 4, 2) == 0
    # ctx, q, q_dtype, B, Hq, Hkv, scale, k_hot, v_hot, W_max, hot_start, hot_len, pool,
    # pool_pages, page_table, max_pages, cold_len, threshold, cold_used, out, workspace,
    # ws_bytes, stream
    gated = [None, None, 0, 1, 1, 1, 0.0, None, None, 0, None, None, None, 0, None, 0, None,
             0.0, None, None, None, 0, None]
    assert L.tq_decode_attention_gated(*gated) == INV
    # ctx, q, q_dtype, B, Hq, Hkv, scale, k_new, v_new, k_hot, v_hot, W_max, hot_start,
    # hot_len, pool, pool_pages, page_table, max_pages, cold_len, threshold, window, E,
    # cold_used, out, workspace, ws_bytes, stream
    mon = [None, None, 0, 1, 1, 1, 0.0, None, None, None, None, 8, None, None, None, 1, None, 1,
           None, 0.0, 4, 2, None, None, None, 0, None]
    assert L.tq_monarch_step(*mon) == INV
    # ctx, q, q_dtype, B, Hq, Hkv, scale, k_new, v_new, k_ring, v_ring, W, ring_start,
    # ring_len, A, lambda, eta, gate, out, workspace, ws_bytes, stream
    tcs = [None, None, 0, 1, 1, 1, 0.0, None, None, None, None, 8, None, None, None, None, None,
           None, None, None, 0, None]
    assert L.tq_tensor_cache_step(*tcs) == INV
    assert L.tq_stage1_encode(None, 1, 4, 2, None, 1, None, None, None) == INV
    assert L.tq_stage1_decode(None, 1, 4, 2, None, None, 1, None, None) == INV
    assert L.tq_self_index_build(None, None, 1, 1, 1, None, None, None, None) == INV
    assert L.tq_self_index_scores(None, None, 0, 1, 1, 1, 1, None, None, None, None) == INV
    assert L.tq_self_index_select(None, None, 1, 1, 64, 1, None, None) == INV
    assert L.tq_self_index_attend(None, None, 0, 1, 1, 1, 1, None, None, None, 64, 1, 0.0, None,
                                  None) == INV
