"""Python binding of libtq (TurboQuant-style compressed KV cache and decode
attention for B200).  Argument marshalling only: every step of the hot path
runs in the CUDA kernels behind the C ABI declared in ``include/tq.h``.

The functions keep the C names.  Device buffers are torch CUDA tensors
(passed by data pointer); the stream is torch's current CUDA stream unless
one is given.  There is no CPU fallback: if ``libtq.so`` is missing or the
device is absent the calls raise.
"""
import ctypes as C
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
# TQ_LIB=debug selects the range-checked build (libtq_debug.so, compiled with
# TQ_DEBUG: every checked index outside its array records TQ_ERR_RANGE and the
# access is skipped)
LIB_PATH = os.path.join(_HERE, "libtq_debug.so" if os.environ.get("TQ_LIB") == "debug" else "libtq.so")

TQ_OK, TQ_ERR_INVALID_ARG, TQ_ERR_UNSUPPORTED, TQ_ERR_CUDA = 0, 1, 2, 3
TQ_ERR_OOM, TQ_ERR_CAPACITY, TQ_ERR_TIMEOUT, TQ_ERR_RANGE = 4, 5, 6, 7
TQ_F32, TQ_F16, TQ_BF16 = 0, 1, 2
TQ_INPUT_ROTATED = 1
TQ_PAGE_TOKENS = 128
TQ_NOALLOC_SCRATCH_BYTES = 8 << 20
TQ_PROMOTE_MAX_PER_STEP = 64


class TQError(RuntimeError):
    def __init__(self, status, what=""):
        self.status = status
        super().__init__("%s: %s (status %d)" % (what, status_string(status), status))


class tq_promotion(C.Structure):
    _fields_ = [("threshold", C.c_float), ("sticky", C.c_int), ("max_per_step", C.c_int),
                ("cold_mask", C.c_void_p), ("counts", C.c_void_p), ("logits", C.c_void_p)]


class tq_config(C.Structure):
    _fields_ = [("head_dim", C.c_int), ("key_bits", C.c_int), ("qjl_dim", C.c_int),
                ("value_bits", C.c_int), ("page_tokens", C.c_int), ("seed", C.c_uint64)]


_lib = None


def lib():
    """Load libtq.so (building it first when the sources are newer)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH) or os.environ.get("TQ_REBUILD"):
            from . import build as _build
            _build.build(debug=LIB_PATH.endswith("_debug.so"))
        L = C.CDLL(LIB_PATH)
        vp, i32p, f32p, u8p = C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p
        L.tq_generate_params.argtypes = [C.POINTER(tq_config)] + [C.c_void_p] * 6
        L.tq_generate_params.restype = C.c_int
        L.tq_init_codebook.argtypes = [C.POINTER(tq_config), C.POINTER(C.c_void_p)]
        L.tq_init_codebook.restype = C.c_int
        L.tq_get_params.argtypes = [vp] + [C.c_void_p] * 6
        L.tq_get_params.restype = C.c_int
        L.tq_page_bytes.argtypes = [vp, C.c_int]
        L.tq_page_bytes.restype = C.c_size_t
        L.tq_compress_append.argtypes = [vp, vp, vp, C.c_int, C.c_int, C.c_int, C.c_int, C.c_int,
                                          u8p, C.c_int64, i32p, C.c_int, i32p, vp]
        L.tq_compress_append.restype = C.c_int
        L.tq_workspace_bytes.argtypes = [vp, C.c_int, C.c_int, C.c_int, C.c_int, C.c_int]
        L.tq_workspace_bytes.restype = C.c_size_t
        L.tq_decode_attention.argtypes = [vp, vp, C.c_int, C.c_int, C.c_int, C.c_int, C.c_float,
                                          vp, vp, C.c_int, i32p, u8p, C.c_int64, i32p, C.c_int,
                                          i32p, f32p, vp, C.c_size_t, vp]
        L.tq_decode_attention.restype = C.c_int
        L.tq_decode_attention_gated.argtypes = [vp, vp, C.c_int, C.c_int, C.c_int, C.c_int,
                                                C.c_float, vp, vp, C.c_int, i32p, i32p, u8p,
                                                C.c_int64, i32p, C.c_int, i32p, C.c_float, i32p,
                                                f32p, vp, C.c_size_t, vp]
        L.tq_decode_attention_gated.restype = C.c_int
        L.tq_monarch_workspace_bytes.argtypes = [vp, C.c_int, C.c_int, C.c_int, C.c_int, C.c_int,
                                                 C.c_int]
        L.tq_monarch_workspace_bytes.restype = C.c_size_t
        L.tq_monarch_step.argtypes = [vp, vp, C.c_int, C.c_int, C.c_int, C.c_int, C.c_float, vp,
                                      vp, vp, vp, C.c_int, i32p, i32p, u8p, C.c_int64, i32p,
                                      C.c_int, i32p, C.c_float, C.c_int, C.c_int, i32p, f32p, vp,
                                      C.c_size_t, vp]
        L.tq_monarch_step.restype = C.c_int
        L.tq_monarch_step_promote.argtypes = [vp, vp, C.c_int, C.c_int, C.c_int, C.c_int,
                                              C.c_float, vp, vp, vp, vp, C.c_int, i32p, i32p,
                                              u8p, C.c_int64, i32p, C.c_int, i32p, C.c_float,
                                              C.c_int, C.c_int, C.POINTER(tq_promotion), i32p,
                                              f32p, vp, C.c_size_t, vp]
        L.tq_monarch_step_promote.restype = C.c_int
        L.tq_stage1_code_bytes.argtypes = [vp, C.c_int, C.c_int, C.c_int]
        L.tq_stage1_code_bytes.restype = C.c_size_t
        L.tq_stage1_encode.argtypes = [vp, C.c_int, C.c_int, C.c_int, f32p, C.c_int64, u8p, vp,
                                       vp]
        L.tq_stage1_encode.restype = C.c_int
        L.tq_stage1_decode.argtypes = [vp, C.c_int, C.c_int, C.c_int, u8p, vp, C.c_int64, f32p,
                                       vp]
        L.tq_stage1_decode.restype = C.c_int
        L.tq_tensor_cache_workspace_bytes.argtypes = [vp, C.c_int, C.c_int, C.c_int, C.c_int]
        L.tq_tensor_cache_workspace_bytes.restype = C.c_size_t
        L.tq_tensor_cache_step.argtypes = [vp, vp, C.c_int, C.c_int, C.c_int, C.c_int, C.c_float,
                                           vp, vp, vp, vp, C.c_int, i32p, i32p, f32p, f32p, f32p,
                                           f32p, f32p, vp, C.c_size_t, vp]
        L.tq_tensor_cache_step.restype = C.c_int
        L.tq_self_index_build.argtypes = [vp, vp, C.c_int, C.c_int, C.c_int, f32p, u8p, f32p, vp]
        L.tq_self_index_build.restype = C.c_int
        L.tq_self_index_scores.argtypes = [vp, vp, C.c_int, C.c_int, C.c_int, C.c_int, C.c_int, u8p,
                                           f32p, f32p, vp]
        L.tq_self_index_scores.restype = C.c_int
        L.tq_self_index_select.argtypes = [vp, f32p, C.c_int, C.c_int, C.c_int, C.c_int, i32p, vp]
        L.tq_self_index_select.restype = C.c_int
        L.tq_self_index_attend.argtypes = [vp, vp, C.c_int, C.c_int, C.c_int, C.c_int, C.c_int, vp,
                                           vp, i32p, C.c_int, C.c_int, C.c_float, f32p, vp]
        L.tq_self_index_attend.restype = C.c_int
        L.tq_decode_attention_noalloc.argtypes = [vp, vp, C.c_int, C.c_int, C.c_int, C.c_int,
                                                  C.c_float, vp, vp, C.c_int, i32p, u8p, C.c_int64,
                                                  i32p, C.c_int, i32p, f32p, vp]
        L.tq_decode_attention_noalloc.restype = C.c_int
        L.tq_topk_workspace_bytes.argtypes = [vp, C.c_int, C.c_int64, C.c_int]
        L.tq_topk_workspace_bytes.restype = C.c_size_t
        L.tq_score_topk.argtypes = [vp, f32p, C.c_int, u8p, C.c_int64, C.c_int, i32p, f32p, vp,
                                    C.c_size_t, vp]
        L.tq_score_topk.restype = C.c_int
        L.tq_set_profile_events.argtypes = [vp, vp, vp]
        L.tq_set_profile_events.restype = C.c_int
        L.tq_set_wait_test.argtypes = [vp, C.c_int, C.c_uint64]
        L.tq_set_wait_test.restype = C.c_int
        L.tq_get_error.argtypes = [vp]
        L.tq_get_error.restype = C.c_int
        L.tq_status_string.argtypes = [C.c_int]
        L.tq_status_string.restype = C.c_char_p
        L.tq_destroy.argtypes = [vp]
        L.tq_destroy.restype = None
        _lib = L
    return _lib


def status_string(s):
    return lib().tq_status_string(int(s)).decode()


def _check(status, what):
    if status != TQ_OK:
        raise TQError(status, what)


def make_config(head_dim=128, seed=0, key_bits=2, value_bits=4, qjl_dim=None):
    return tq_config(head_dim, key_bits, head_dim if qjl_dim is None else qjl_dim, value_bits,
                     TQ_PAGE_TOKENS, seed)


def _ptr(t):
    """Device (or host) address of a torch tensor / numpy array; None -> NULL."""
    if t is None:
        return None
    if isinstance(t, np.ndarray):
        return t.ctypes.data
    return t.data_ptr()


def _dtype_code(t):
    import torch
    return {torch.float32: TQ_F32, torch.float16: TQ_F16, torch.bfloat16: TQ_BF16}[t.dtype]


def _stream(stream):
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return C.c_void_p(s.cuda_stream)


def _require_cuda(*tensors):
    for t in tensors:
        if t is not None and not t.is_cuda:
            raise ValueError("device tensor expected")
        if t is not None and not t.is_contiguous():
            raise ValueError("contiguous tensor expected")


# ---------------------------------------------------------------------------
# C entry points, same names
# ---------------------------------------------------------------------------
def tq_generate_params(cfg):
    """Host-only table generation (no device needed).  Returns numpy arrays."""
    d, m = cfg.head_dim, cfg.qjl_dim
    out = dict(rot=np.empty((d, d), np.float32), qjl=np.empty((m, d), np.float32),
               key_c=np.empty(1 << (cfg.key_bits - 1), np.float32),
               key_t=np.empty(max((1 << (cfg.key_bits - 1)) - 1, 1), np.float32),
               val_c=np.empty(1 << (cfg.value_bits - 1), np.float32),
               val_t=np.empty(max((1 << (cfg.value_bits - 1)) - 1, 1), np.float32))
    _check(lib().tq_generate_params(C.byref(cfg), *[_ptr(out[k]) for k in
                                                    ("rot", "qjl", "key_c", "key_t", "val_c", "val_t")]),
           "tq_generate_params")
    out["key_t"] = out["key_t"][: (1 << (cfg.key_bits - 1)) - 1]
    out["val_t"] = out["val_t"][: (1 << (cfg.value_bits - 1)) - 1]
    return out


def tq_init_codebook(cfg):
    h = C.c_void_p()
    _check(lib().tq_init_codebook(C.byref(cfg), C.byref(h)), "tq_init_codebook")
    return h


def tq_get_params(ctx, cfg):
    d, m = cfg.head_dim, cfg.qjl_dim
    out = dict(rot=np.empty((d, d), np.float32), qjl=np.empty((m, d), np.float32),
               key_c=np.empty(2, np.float32), key_t=np.empty(1, np.float32),
               val_c=np.empty(8, np.float32), val_t=np.empty(7, np.float32))
    _check(lib().tq_get_params(ctx, *[_ptr(out[k]) for k in
                                      ("rot", "qjl", "key_c", "key_t", "val_c", "val_t")]),
           "tq_get_params")
    return out


def tq_page_bytes(ctx, with_values=True):
    return int(lib().tq_page_bytes(ctx, 1 if with_values else 0))


def tq_compress_append(ctx, k, v, page_pool, page_table, cold_len, rotated=False, stream=None):
    """k, v: [B, Hkv, n_new, d] CUDA tensors (fp16/bf16, or fp32 when rotated);
    v may be None (keys-only pages).  page_pool: uint8 [pool_pages, page_bytes];
    page_table: int32 [B, Hkv, max_pages]; cold_len: int32 [B] (advanced)."""
    _require_cuda(k, v, page_pool, page_table, cold_len)
    B, Hkv, n_new, _ = k.shape
    _check(lib().tq_compress_append(
        ctx, _ptr(k), _ptr(v), _dtype_code(k), TQ_INPUT_ROTATED if rotated else 0, B, Hkv, n_new,
        _ptr(page_pool), page_pool.shape[0], _ptr(page_table), page_table.shape[-1],
        _ptr(cold_len), _stream(stream)), "tq_compress_append")


def tq_workspace_bytes(ctx, B, Hq, Hkv, max_pages, W_max):
    return int(lib().tq_workspace_bytes(ctx, B, Hq, Hkv, max_pages, W_max))


def tq_decode_attention(ctx, q, k_hot, v_hot, hot_len, page_pool, page_table, cold_len, out,
                        workspace, Hkv, scale=0.0, stream=None):
    """q: [B, Hq, d]; k_hot, v_hot: fp16 [B, Hkv, W_max, d] or None; hot_len,
    cold_len: int32 [B]; page_pool uint8 [pool_pages, page_bytes]; page_table
    int32 [B, Hkv, max_pages]; out fp32 [B, Hq, d]; workspace uint8 CUDA tensor."""
    _require_cuda(q, k_hot, v_hot, hot_len, page_pool, page_table, cold_len, out, workspace)
    B, Hq, _ = q.shape
    W_max = 0 if k_hot is None else k_hot.shape[2]
    max_pages = 0 if page_table is None else page_table.shape[-1]
    pool_pages = 0 if page_pool is None else page_pool.shape[0]
    _check(lib().tq_decode_attention(
        ctx, _ptr(q), _dtype_code(q), B, Hq, Hkv, float(scale), _ptr(k_hot), _ptr(v_hot), W_max,
        _ptr(hot_len), _ptr(page_pool), pool_pages, _ptr(page_table), max_pages, _ptr(cold_len),
        _ptr(out), _ptr(workspace), workspace.numel() * workspace.element_size(),
        _stream(stream)), "tq_decode_attention")


def tq_decode_attention_gated(ctx, q, k_hot, v_hot, hot_len, page_pool, page_table, cold_len,
                              threshold, out, workspace, Hkv, scale=0.0, hot_start=None,
                              cold_used=None, stream=None):
    """tq_decode_attention with Monarch's threshold gate: a q head reads its
    cold tokens only when max_t <q, k_hot_t> (raw, fp32) < threshold.
    hot_start: int32 [B] ring slot of the oldest hot token, or None;
    cold_used: int32 [B, Hq] out (1 = the head read its cold tokens), or None."""
    _require_cuda(q, k_hot, v_hot, hot_len, page_pool, page_table, cold_len, out, workspace,
                  hot_start, cold_used)
    B, Hq, _ = q.shape
    W_max = 0 if k_hot is None else k_hot.shape[2]
    max_pages = 0 if page_table is None else page_table.shape[-1]
    pool_pages = 0 if page_pool is None else page_pool.shape[0]
    _check(lib().tq_decode_attention_gated(
        ctx, _ptr(q), _dtype_code(q), B, Hq, Hkv, float(scale), _ptr(k_hot), _ptr(v_hot), W_max,
        _ptr(hot_start), _ptr(hot_len), _ptr(page_pool), pool_pages, _ptr(page_table), max_pages,
        _ptr(cold_len), float(threshold), _ptr(cold_used), _ptr(out), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream)),
        "tq_decode_attention_gated")


def tq_monarch_workspace_bytes(ctx, B, Hq, Hkv, max_pages, W_max, evict_block):
    return int(lib().tq_monarch_workspace_bytes(ctx, B, Hq, Hkv, max_pages, W_max, evict_block))


def tq_monarch_step(ctx, q, k_new, v_new, k_hot, v_hot, hot_start, hot_len, page_pool,
                    page_table, cold_len, threshold, window, evict_block, out, workspace, Hkv,
                    scale=0.0, cold_used=None, stream=None):
    """One Monarch decode step: append (k_new, v_new fp16 [B, Hkv, d], or
    None), gated attention over the hot ring and cold pages, eviction of the
    oldest evict_block hot tokens of every sequence holding window +
    evict_block of them.  k_hot, v_hot fp16 [B, Hkv, W_max, d]; hot_start,
    hot_len, cold_len int32 [B] (all updated on the device)."""
    _require_cuda(q, k_new, v_new, k_hot, v_hot, hot_start, hot_len, page_pool, page_table,
                  cold_len, out, workspace, cold_used)
    B, Hq, _ = q.shape
    W_max = k_hot.shape[2]
    _check(lib().tq_monarch_step(
        ctx, _ptr(q), _dtype_code(q), B, Hq, Hkv, float(scale), _ptr(k_new), _ptr(v_new),
        _ptr(k_hot), _ptr(v_hot), W_max, _ptr(hot_start), _ptr(hot_len), _ptr(page_pool),
        page_pool.shape[0], _ptr(page_table), page_table.shape[-1], _ptr(cold_len),
        float(threshold), int(window), int(evict_block), _ptr(cold_used), _ptr(out),
        _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream)),
        "tq_monarch_step")


def tq_monarch_step_promote(ctx, q, k_new, v_new, k_hot, v_hot, hot_start, hot_len, page_pool,
                            page_table, cold_len, threshold, window, evict_block, promo, out,
                            workspace, Hkv, scale=0.0, cold_used=None, stream=None):
    """tq_monarch_step with Monarch's promotion.  promo: dict(threshold,
    sticky, max_per_step, cold_mask (int32 [B, max_pages * 4]), counts (uint8
    [B, max_pages * 128]), logits (fp32 [B, Hq, max_pages * 128])), device
    tensors updated in place; None runs tq_monarch_step."""
    _require_cuda(q, k_new, v_new, k_hot, v_hot, hot_start, hot_len, page_pool, page_table,
                  cold_len, out, workspace, cold_used)
    B, Hq, _ = q.shape
    W_max = k_hot.shape[2]
    pr = None
    if promo is not None:
        _require_cuda(promo["cold_mask"], promo["counts"], promo["logits"])
        pr = C.byref(tq_promotion(float(promo["threshold"]), int(promo["sticky"]),
                                  int(promo["max_per_step"]), _ptr(promo["cold_mask"]),
                                  _ptr(promo["counts"]), _ptr(promo["logits"])))
    _check(lib().tq_monarch_step_promote(
        ctx, _ptr(q), _dtype_code(q), B, Hq, Hkv, float(scale), _ptr(k_new), _ptr(v_new),
        _ptr(k_hot), _ptr(v_hot), W_max, _ptr(hot_start), _ptr(hot_len), _ptr(page_pool),
        page_pool.shape[0], _ptr(page_table), page_table.shape[-1], _ptr(cold_len),
        float(threshold), int(window), int(evict_block), pr, _ptr(cold_used), _ptr(out),
        _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream)),
        "tq_monarch_step_promote")


def tq_tensor_cache_workspace_bytes(ctx, B, Hq, Hkv, W):
    return int(lib().tq_tensor_cache_workspace_bytes(ctx, B, Hq, Hkv, W))


def tq_tensor_cache_step(ctx, q, k_new, v_new, k_ring, v_ring, ring_start, ring_len, A, lam, eta,
                         gate, out, workspace, Hkv, scale=0.0, stream=None):
    """One Tensor Cache step: the token enters the fp16 ring (evicting the
    oldest into A when full), then y = softmax attention over the ring +
    sigmoid(gate) * (q A).  k_ring, v_ring [B, Hkv, W, d]; A fp32 [B, Hkv, d, d];
    lam, eta fp32 [Hkv]; gate fp32 [Hq]."""
    _require_cuda(q, k_new, v_new, k_ring, v_ring, ring_start, ring_len, A, lam, eta, gate, out,
                  workspace)
    B, Hq, _ = q.shape
    _check(lib().tq_tensor_cache_step(
        ctx, _ptr(q), _dtype_code(q), B, Hq, Hkv, float(scale), _ptr(k_new), _ptr(v_new),
        _ptr(k_ring), _ptr(v_ring), k_ring.shape[2], _ptr(ring_start), _ptr(ring_len), _ptr(A),
        _ptr(lam), _ptr(eta), _ptr(gate), _ptr(out), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream)), "tq_tensor_cache_step")


def tq_self_index_build(ctx, k, mu, codes, centroids, stream=None):
    """k fp16 [B, Hkv, T, d] -> mu fp32 [B, Hkv, d], codes uint8 [B, Hkv, T, d/4],
    centroids fp32 [B, Hkv, d/4, 16, 4] (sign-pattern index of the centred keys)."""
    _require_cuda(k, mu, codes, centroids)
    B, Hkv, T, _ = k.shape
    _check(lib().tq_self_index_build(ctx, _ptr(k), B, Hkv, T, _ptr(mu), _ptr(codes),
                                     _ptr(centroids), _stream(stream)), "tq_self_index_build")


def tq_self_index_scores(ctx, q, codes, centroids, scores, Hkv, stream=None):
    """q [B, Hq, d]; codes, centroids from tq_self_index_build; scores fp32
    [B, Hq, T] out: sum over groups of <q_g, centroid[g][code]>."""
    _require_cuda(q, codes, centroids, scores)
    B, Hq, _ = q.shape
    T = codes.shape[2]
    _check(lib().tq_self_index_scores(ctx, _ptr(q), _dtype_code(q), B, Hq, Hkv, T, _ptr(codes),
                                      _ptr(centroids), _ptr(scores), _stream(stream)),
           "tq_self_index_scores")


def tq_self_index_select(ctx, scores, picked, n_sink=64, stream=None):
    """scores fp32 [B, Hq, T] -> picked int32 [B, Hq, top_k]: the best
    positions after the n_sink sinks in increasing order (ties to the lower
    position), -1 past the available count."""
    _require_cuda(scores, picked)
    T = scores.shape[-1]
    rows = int(np.prod(scores.shape[:-1]))
    if tuple(picked.shape[:-1]) != tuple(scores.shape[:-1]):
        raise ValueError("picked must be [..., top_k] over the rows of scores")
    _check(lib().tq_self_index_select(ctx, _ptr(scores), rows, T, n_sink, picked.shape[-1],
                                      _ptr(picked), _stream(stream)), "tq_self_index_select")


def tq_self_index_attend(ctx, q, keys, values, picked, out, n_sink=64, scale=0.0, stream=None):
    """q [B, Hq, d]; keys, values fp16 [B, Hkv, T, d]; picked int32
    [B, Hq, top_k] -> out fp32 [B, Hq, d]: softmax attention over the sinks
    and the picked positions."""
    _require_cuda(q, keys, values, picked, out)
    B, Hq, _ = q.shape
    Hkv, T = keys.shape[1], keys.shape[2]
    _check(lib().tq_self_index_attend(ctx, _ptr(q), _dtype_code(q), B, Hq, Hkv, T, _ptr(keys),
                                      _ptr(values), _ptr(picked), n_sink, picked.shape[-1],
                                      float(scale), _ptr(out), _stream(stream)),
           "tq_self_index_attend")


TQ_STAGE1_MSE, TQ_STAGE1_POLAR = 0, 1


def tq_stage1_code_bytes(ctx, kind, bits1, bits2=0):
    return int(lib().tq_stage1_code_bytes(ctx, kind, bits1, bits2))


def tq_stage1_encode(ctx, kind, bits1, bits2, x_rot, codes, norms, stream=None):
    """x_rot fp32 [N, d] -> codes uint8 [N, code_bytes], norms fp16-bits
    (int16 / uint16 tensor) [N]."""
    _require_cuda(x_rot, codes, norms)
    _check(lib().tq_stage1_encode(ctx, int(kind), int(bits1), int(bits2), _ptr(x_rot),
                                  x_rot.shape[0], _ptr(codes), _ptr(norms), _stream(stream)),
           "tq_stage1_encode")


def tq_stage1_decode(ctx, kind, bits1, bits2, codes, norms, x_hat, stream=None):
    _require_cuda(codes, norms, x_hat)
    _check(lib().tq_stage1_decode(ctx, int(kind), int(bits1), int(bits2), _ptr(codes),
                                  _ptr(norms), codes.shape[0], _ptr(x_hat), _stream(stream)),
           "tq_stage1_decode")


def tq_decode_attention_noalloc(ctx, q, k_hot, v_hot, hot_len, page_pool, page_table, cold_len,
                                out, Hkv, scale=0.0, stream=None):
    """tq_decode_attention for callers that may not allocate device memory:
    no workspace argument; the library's fixed scratch array (at most
    TQ_NOALLOC_SCRATCH_BYTES of workspace) is used instead.  Make the first
    call on a device before any stream capture; calls that overlap on the GPU
    race on the shared scratch."""
    _require_cuda(q, k_hot, v_hot, hot_len, page_pool, page_table, cold_len, out)
    B, Hq, _ = q.shape
    W_max = 0 if k_hot is None else k_hot.shape[2]
    max_pages = 0 if page_table is None else page_table.shape[-1]
    pool_pages = 0 if page_pool is None else page_pool.shape[0]
    _check(lib().tq_decode_attention_noalloc(
        ctx, _ptr(q), _dtype_code(q), B, Hq, Hkv, float(scale), _ptr(k_hot), _ptr(v_hot), W_max,
        _ptr(hot_len), _ptr(page_pool), pool_pages, _ptr(page_table), max_pages, _ptr(cold_len),
        _ptr(out), _stream(stream)), "tq_decode_attention_noalloc")


def tq_topk_workspace_bytes(ctx, Q, N, k):
    return int(lib().tq_topk_workspace_bytes(ctx, Q, N, k))


def tq_score_topk(ctx, queries, db_pages, N, k, out_ids, out_scores, workspace, stream=None):
    _require_cuda(queries, db_pages, out_ids, out_scores, workspace)
    _check(lib().tq_score_topk(
        ctx, _ptr(queries), queries.shape[0], _ptr(db_pages), int(N), int(k), _ptr(out_ids),
        _ptr(out_scores), _ptr(workspace), workspace.numel() * workspace.element_size(),
        _stream(stream)), "tq_score_topk")


def tq_set_profile_events(ctx, ev_start, ev_stop):
    """ev_start/ev_stop: torch.cuda.Event(enable_timing=True) or None."""
    a = None if ev_start is None else C.c_void_p(ev_start.cuda_event)
    b = None if ev_stop is None else C.c_void_p(ev_stop.cuda_event)
    _check(lib().tq_set_profile_events(ctx, a, b), "tq_set_profile_events")


def tq_set_wait_test(ctx, skip_unit, limit_ns=0):
    """Testing aid for the bounded waits: skip the copy of cold unit skip_unit
    (-1: none) and bound every attention wait by limit_ns (0: default)."""
    _check(lib().tq_set_wait_test(ctx, int(skip_unit), int(limit_ns)), "tq_set_wait_test")


def tq_get_error(ctx):
    return int(lib().tq_get_error(ctx))


def tq_destroy(ctx):
    lib().tq_destroy(ctx)


# ---------------------------------------------------------------------------
# convenience wrapper owning a context
# ---------------------------------------------------------------------------
class Context:
    def __init__(self, head_dim=128, seed=0):
        self.cfg = make_config(head_dim, seed)
        self.handle = tq_init_codebook(self.cfg)
        self.d = head_dim

    def params(self):
        return tq_get_params(self.handle, self.cfg)

    def page_bytes(self, with_values=True):
        return tq_page_bytes(self.handle, with_values)

    def workspace(self, B, Hq, Hkv, max_pages, W_max, device="cuda"):
        import torch
        n = tq_workspace_bytes(self.handle, B, Hq, Hkv, max_pages, W_max)
        return torch.empty(n, dtype=torch.uint8, device=device)

    def check(self):
        s = tq_get_error(self.handle)
        if s != TQ_OK:
            raise TQError(s, "device")

    def close(self):
        if self.handle is not None:
            tq_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
