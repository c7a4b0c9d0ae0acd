// C ABI entry points of libtq: argument validation, context lifetime, table
// upload, and dispatch to the kernel launchers.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <nvtx3/nvToolsExt.h>

#include <cmath>
#include <cstring>
#include <new>

#include "tq_internal.h"

namespace tq {

PageLayout page_layout(int d, int m, bool with_values) {
  auto up16 = [](size_t x) { return (x + 15) & ~static_cast<size_t>(15); };
  const size_t P = TQ_PAGE_TOKENS;
  PageLayout L{};
  if (with_values) {
    const size_t D = static_cast<size_t>(d), M = static_cast<size_t>(m);
    L.kc = 0;
    L.kl = 2 * D;
    L.qs = 4 * D;
    L.vc = 4 * D + 2 * M;
    L.kn = 12 * D + 2 * M;
    L.kg = L.kn + 2;
    L.vn = L.kn + 64;
    L.block = L.kn + 96;
    L.bytes = (P / 16) * L.block;
    return L;
  }
  size_t off = 0;
  L.kc = off;
  off = up16(off + P * d / 4);
  L.qs = off;
  off = up16(off + P * m / 8);
  L.kn = off;
  off = up16(off + 2 * P);
  L.kg = off;
  off = up16(off + 2 * P);
  L.bytes = off;
  return L;
}

namespace {

// NVTX range over one host call (visible in Nsight timelines; the NVTX
// library is loaded only when a tool injects it, otherwise each push / pop is a
// no-op check)
struct Range {
  explicit Range(const char* name) { nvtxRangePushA(name); }
  ~Range() { nvtxRangePop(); }
};

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

uint16_t bf16_bits(float x) { return __bfloat16_as_ushort(__float2bfloat16_rn(x)); }
float bf16_value(uint16_t b) { return __bfloat162float(__ushort_as_bfloat16(b)); }
uint16_t f16_bits(float x) { return __half_as_ushort(__float2half_rn(x)); }
float f16_value(uint16_t b) { return __half2float(__ushort_as_half(b)); }

}  // namespace
}  // namespace tq

extern "C" {

const char* tq_status_string(tq_status s) {
  switch (s) {
    case TQ_OK: return "ok";
    case TQ_ERR_INVALID_ARG: return "invalid argument";
    case TQ_ERR_UNSUPPORTED: return "unsupported configuration";
    case TQ_ERR_CUDA: return "CUDA error";
    case TQ_ERR_OOM: return "out of device memory";
    case TQ_ERR_CAPACITY: return "capacity exceeded (page table, pool or window)";
    case TQ_ERR_TIMEOUT: return "bounded wait timed out";
    case TQ_ERR_RANGE: return "index out of range (range-checked build)";
  }
  return "unknown status";
}

tq_status tq_generate_params(const tq_config* cfg, float* rot, float* qjl, float* key_c,
                             float* key_t, float* val_c, float* val_t) {
  if (!cfg || !tq::config_valid(*cfg)) return TQ_ERR_INVALID_ARG;
  tq::HostTables t;
  if (!tq::generate_tables(*cfg, t)) return TQ_ERR_INVALID_ARG;
  auto put = [](float* dst, const std::vector<float>& src) {
    if (dst && !src.empty()) std::memcpy(dst, src.data(), src.size() * sizeof(float));
  };
  put(rot, t.rot);
  put(qjl, t.qjl);
  put(key_c, t.key_c);
  put(key_t, t.key_t);
  put(val_c, t.val_c);
  put(val_t, t.val_t);
  return TQ_OK;
}

tq_status tq_init_codebook(const tq_config* cfg, tq_ctx** out) {
  tq::Range range("tq_init_codebook");
  if (!cfg || !out) return TQ_ERR_INVALID_ARG;
  *out = nullptr;
  if (!tq::config_valid(*cfg)) return TQ_ERR_INVALID_ARG;
  if (!tq::config_supported(*cfg)) return TQ_ERR_UNSUPPORTED;
  tq_ctx* ctx = new (std::nothrow) tq_ctx();
  if (!ctx) return TQ_ERR_OOM;
  ctx->cfg = *cfg;
  ctx->wait_skip_unit = -1;
  if (!tq::generate_tables(*cfg, ctx->host)) {
    delete ctx;
    return TQ_ERR_INVALID_ARG;
  }
  if (cudaGetDevice(&ctx->device) != cudaSuccess ||
      cudaDeviceGetAttribute(&ctx->num_sms, cudaDevAttrMultiProcessorCount, ctx->device) !=
          cudaSuccess) {
    delete ctx;
    return TQ_ERR_CUDA;
  }
  const int d = cfg->head_dim, m = cfg->qjl_dim;
  const tq::HostTables& h = ctx->host;
  std::memset(&ctx->cb, 0, sizeof(ctx->cb));
  for (size_t i = 0; i < h.key_c.size() && i < 2; ++i) ctx->cb.key_c[i] = h.key_c[i];
  for (size_t i = 0; i < h.key_t.size() && i < 1; ++i) ctx->cb.key_t[i] = h.key_t[i];
  for (size_t i = 0; i < h.val_c.size() && i < 8; ++i) ctx->cb.val_c[i] = h.val_c[i];
  for (size_t i = 0; i < h.val_t.size() && i < 7; ++i) ctx->cb.val_t[i] = h.val_t[i];

  // one device block: rot f32 | qjl f32 | qjl f16 | rot bf16 hi, lo | rot f16 hi, lo | S Pi f32 | err
  const size_t dd = static_cast<size_t>(d) * d, md = static_cast<size_t>(m) * d;
  auto a256 = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
  size_t off_rot = 0, off_qjl = a256(off_rot + dd * 4), off_qjlh = a256(off_qjl + md * 4);
  size_t off_bh = a256(off_qjlh + md * 2), off_bl = a256(off_bh + dd * 2);
  size_t off_hh = a256(off_bl + dd * 2), off_hl = a256(off_hh + dd * 2);
  size_t off_sp = a256(off_hl + dd * 2);  // S Pi, fp32 [m][d]
  size_t off_err = a256(off_sp + md * 4), total = a256(off_err + 256);
  std::vector<uint8_t> img(total, 0);
  std::memcpy(img.data() + off_rot, h.rot.data(), dd * 4);
  std::memcpy(img.data() + off_qjl, h.qjl.data(), md * 4);
  uint16_t* qh = reinterpret_cast<uint16_t*>(img.data() + off_qjlh);
  for (size_t i = 0; i < md; ++i) qh[i] = tq::f16_bits(h.qjl[i]);
  uint16_t* bh = reinterpret_cast<uint16_t*>(img.data() + off_bh);
  uint16_t* bl = reinterpret_cast<uint16_t*>(img.data() + off_bl);
  uint16_t* hh = reinterpret_cast<uint16_t*>(img.data() + off_hh);
  uint16_t* hl = reinterpret_cast<uint16_t*>(img.data() + off_hl);
  for (size_t i = 0; i < dd; ++i) {
    const float x = h.rot[i];
    bh[i] = tq::bf16_bits(x);
    bl[i] = tq::bf16_bits(x - tq::bf16_value(bh[i]));
    hh[i] = tq::f16_bits(x);
    hl[i] = tq::f16_bits(x - tq::f16_value(hh[i]));
  }
  {
    // S Pi (fp64 sums, fp32 store): the decode prep forms q_s = S (Pi q) as
    // (S Pi) q, in the same pass as Pi q
    float* sp = reinterpret_cast<float*>(img.data() + off_sp);
    for (int r = 0; r < m; ++r)
      for (int c = 0; c < d; ++c) {
        double acc = 0.0;
        for (int k = 0; k < d; ++k)
          acc += static_cast<double>(h.qjl[static_cast<size_t>(r) * d + k]) *
                 static_cast<double>(h.rot[static_cast<size_t>(k) * d + c]);
        sp[static_cast<size_t>(r) * d + c] = static_cast<float>(acc);
      }
  }
  void* blk = nullptr;
  if (cudaMalloc(&blk, total) != cudaSuccess) {
    delete ctx;
    return TQ_ERR_OOM;
  }
  if (cudaMemcpy(blk, img.data(), total, cudaMemcpyHostToDevice) != cudaSuccess) {
    cudaFree(blk);
    delete ctx;
    return TQ_ERR_CUDA;
  }
  uint8_t* b = static_cast<uint8_t*>(blk);
  ctx->dev_block = blk;
  ctx->dev.rot = reinterpret_cast<const float*>(b + off_rot);
  ctx->dev.qjl = reinterpret_cast<const float*>(b + off_qjl);
  ctx->dev.qjl_h = reinterpret_cast<const uint16_t*>(b + off_qjlh);
  ctx->dev.rot_bf_hi = reinterpret_cast<const uint16_t*>(b + off_bh);
  ctx->dev.rot_bf_lo = reinterpret_cast<const uint16_t*>(b + off_bl);
  ctx->dev.rot_h_hi = reinterpret_cast<const uint16_t*>(b + off_hh);
  ctx->dev.rot_h_lo = reinterpret_cast<const uint16_t*>(b + off_hl);
  ctx->dev.sp = reinterpret_cast<const float*>(b + off_sp);
  ctx->dev.err = reinterpret_cast<int*>(b + off_err);
  *out = ctx;
  return TQ_OK;
}

tq_status tq_get_params(const tq_ctx* ctx, float* rot, float* qjl, float* key_c, float* key_t,
                        float* val_c, float* val_t) {
  if (!ctx) return TQ_ERR_INVALID_ARG;
  auto put = [](float* dst, const std::vector<float>& src) {
    if (dst && !src.empty()) std::memcpy(dst, src.data(), src.size() * sizeof(float));
  };
  put(rot, ctx->host.rot);
  put(qjl, ctx->host.qjl);
  put(key_c, ctx->host.key_c);
  put(key_t, ctx->host.key_t);
  put(val_c, ctx->host.val_c);
  put(val_t, ctx->host.val_t);
  return TQ_OK;
}

size_t tq_page_bytes(const tq_ctx* ctx, int with_values) {
  if (!ctx) return 0;
  return tq::page_layout(ctx->cfg.head_dim, ctx->cfg.qjl_dim, with_values != 0).bytes;
}

tq_status tq_compress_append(const tq_ctx* ctx, const void* k, const void* v, tq_dtype dtype,
                             int flags, int B, int Hkv, int n_new, uint8_t* page_pool,
                             int64_t pool_pages, const int32_t* page_table, int max_pages,
                             int32_t* cold_len, void* stream) {
  tq::Range range("tq_compress_append");
  if (!ctx || !k || !page_pool || !page_table || !cold_len) return TQ_ERR_INVALID_ARG;
  if (B <= 0 || Hkv <= 0 || n_new < 0 || max_pages <= 0 || pool_pages <= 0)
    return TQ_ERR_INVALID_ARG;
  if (dtype != TQ_F32 && dtype != TQ_F16 && dtype != TQ_BF16) return TQ_ERR_INVALID_ARG;
  if ((flags & ~TQ_INPUT_ROTATED) != 0) return TQ_ERR_INVALID_ARG;
  const bool rotated = (flags & TQ_INPUT_ROTATED) != 0;
  if (rotated != (dtype == TQ_F32)) return TQ_ERR_UNSUPPORTED;
  if (!tq::aligned(page_pool, 16) || !tq::aligned(k, 16) || (v && !tq::aligned(v, 16)))
    return TQ_ERR_INVALID_ARG;
  if (n_new == 0) return TQ_OK;
  return static_cast<tq_status>(tq::launch_compress(ctx, k, v, dtype, flags, B, Hkv, n_new,
                                                    page_pool, pool_pages, page_table, max_pages,
                                                    cold_len, stream));
}

size_t tq_workspace_bytes(const tq_ctx* ctx, int B, int Hq, int Hkv, int max_pages, int W_max) {
  if (!ctx) return 0;
  return tq::decode_workspace_bytes(ctx, B, Hq, Hkv, max_pages, W_max);
}

namespace {

tq_status decode_common(const tq_ctx* ctx, const void* q, tq_dtype q_dtype, int B, int Hq,
                        int Hkv, float scale, const void* k_hot, const void* v_hot, int W_max,
                        const int32_t* hot_start, const int32_t* hot_len,
                        const uint8_t* page_pool, int64_t pool_pages, const int32_t* page_table,
                        int max_pages, const int32_t* cold_len, const tq::DecodeGate* gate,
                        float* out, void* workspace, size_t ws_bytes, void* stream) {
  if (!ctx || !q || !out || !workspace) return TQ_ERR_INVALID_ARG;
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || W_max < 0 || max_pages < 0)
    return TQ_ERR_INVALID_ARG;
  if (q_dtype != TQ_F32 && q_dtype != TQ_F16 && q_dtype != TQ_BF16) return TQ_ERR_INVALID_ARG;
  if (!(scale >= 0.0f) || !std::isfinite(scale)) return TQ_ERR_INVALID_ARG;
  const int G = Hq / Hkv;
  if (G != 1 && G != 2 && G != 4 && G != 8) return TQ_ERR_UNSUPPORTED;
  if (W_max > 0 && (!k_hot || !v_hot || !hot_len)) return TQ_ERR_INVALID_ARG;
  if (W_max > 0 && (!tq::aligned(k_hot, 16) || !tq::aligned(v_hot, 16))) return TQ_ERR_INVALID_ARG;
  if (max_pages > 0 && (!page_pool || !page_table || !cold_len || pool_pages <= 0))
    return TQ_ERR_INVALID_ARG;
  if (page_pool && !tq::aligned(page_pool, 16)) return TQ_ERR_INVALID_ARG;
  if (!tq::aligned(workspace, 256)) return TQ_ERR_INVALID_ARG;
  if (gate && std::isnan(gate->threshold)) return TQ_ERR_INVALID_ARG;
  const size_t need = tq::decode_workspace_bytes(ctx, B, Hq, Hkv, max_pages, W_max);
  if (need == 0 || ws_bytes < need) return TQ_ERR_INVALID_ARG;
  return static_cast<tq_status>(tq::launch_decode(
      ctx, q, q_dtype, B, Hq, Hkv, scale, W_max > 0 ? k_hot : nullptr,
      W_max > 0 ? v_hot : nullptr, W_max, W_max > 0 ? hot_start : nullptr,
      W_max > 0 ? hot_len : nullptr, max_pages > 0 ? page_pool : nullptr, pool_pages,
      max_pages > 0 ? page_table : nullptr, max_pages, max_pages > 0 ? cold_len : nullptr, gate,
      out, workspace, ws_bytes, stream));
}

}  // namespace

tq_status tq_decode_attention(const tq_ctx* ctx, const void* q, tq_dtype q_dtype, int B, int Hq,
                              int Hkv, float scale, const void* k_hot, const void* v_hot,
                              int W_max, const int32_t* hot_len, const uint8_t* page_pool,
                              int64_t pool_pages, const int32_t* page_table, int max_pages,
                              const int32_t* cold_len, float* out, void* workspace,
                              size_t ws_bytes, void* stream) {
  tq::Range range("tq_decode_attention");
  return decode_common(ctx, q, q_dtype, B, Hq, Hkv, scale, k_hot, v_hot, W_max, nullptr, hot_len,
                       page_pool, pool_pages, page_table, max_pages, cold_len, nullptr, out,
                       workspace, ws_bytes, stream);
}

tq_status tq_decode_attention_gated(const tq_ctx* ctx, const void* q, tq_dtype q_dtype, int B,
                                    int Hq, int Hkv, float scale, const void* k_hot,
                                    const void* v_hot, int W_max, const int32_t* hot_start,
                                    const int32_t* hot_len, const uint8_t* page_pool,
                                    int64_t pool_pages, const int32_t* page_table, int max_pages,
                                    const int32_t* cold_len, float threshold, int32_t* cold_used,
                                    float* out, void* workspace, size_t ws_bytes, void* stream) {
  const tq::DecodeGate gate{threshold, cold_used};
  return decode_common(ctx, q, q_dtype, B, Hq, Hkv, scale, k_hot, v_hot, W_max, hot_start,
                       hot_len, page_pool, pool_pages, page_table, max_pages, cold_len, &gate,
                       out, workspace, ws_bytes, stream);
}

size_t tq_monarch_workspace_bytes(const tq_ctx* ctx, int B, int Hq, int Hkv, int max_pages,
                                  int W_max, int evict_block) {
  if (!ctx) return 0;
  return tq::monarch_workspace_bytes(ctx, B, Hq, Hkv, max_pages, W_max, evict_block);
}

tq_status tq_monarch_step(const tq_ctx* ctx, const void* q, tq_dtype q_dtype, int B, int Hq,
                          int Hkv, float scale, const void* k_new, const void* v_new, void* k_hot,
                          void* v_hot, int W_max, int32_t* hot_start, int32_t* hot_len,
                          uint8_t* page_pool, int64_t pool_pages, const int32_t* page_table,
                          int max_pages, int32_t* cold_len, float threshold, int window,
                          int evict_block, int32_t* cold_used, float* out, void* workspace,
                          size_t ws_bytes, void* stream) {
  return tq_monarch_step_promote(ctx, q, q_dtype, B, Hq, Hkv, scale, k_new, v_new, k_hot, v_hot,
                                 W_max, hot_start, hot_len, page_pool, pool_pages, page_table,
                                 max_pages, cold_len, threshold, window, evict_block, nullptr,
                                 cold_used, out, workspace, ws_bytes, stream);
}

tq_status tq_monarch_step_promote(const tq_ctx* ctx, const void* q, tq_dtype q_dtype, int B,
                                  int Hq, int Hkv, float scale, const void* k_new,
                                  const void* v_new, void* k_hot, void* v_hot, int W_max,
                                  int32_t* hot_start, int32_t* hot_len, uint8_t* page_pool,
                                  int64_t pool_pages, const int32_t* page_table, int max_pages,
                                  int32_t* cold_len, float threshold, int window,
                                  int evict_block, const tq_promotion* promo,
                                  int32_t* cold_used, float* out, void* workspace,
                                  size_t ws_bytes, void* stream) {
  tq::Range range("tq_monarch_step");
  if (promo) {
    if (!(promo->threshold > 0.0f) || !std::isfinite(promo->threshold) || promo->sticky < 1 ||
        promo->max_per_step < 1 || promo->max_per_step > TQ_PROMOTE_MAX_PER_STEP ||
        !promo->cold_mask || !promo->counts || !promo->logits ||
        !tq::aligned(promo->cold_mask, 4) || !tq::aligned(promo->logits, 4))
      return TQ_ERR_INVALID_ARG;
  }
  if (!ctx || !q || !out || !workspace || !k_hot || !v_hot || !hot_start || !hot_len)
    return TQ_ERR_INVALID_ARG;
  if (!page_pool || !page_table || !cold_len || pool_pages <= 0 || max_pages <= 0)
    return TQ_ERR_INVALID_ARG;
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0) return TQ_ERR_INVALID_ARG;
  if (q_dtype != TQ_F32 && q_dtype != TQ_F16 && q_dtype != TQ_BF16) return TQ_ERR_INVALID_ARG;
  if (!(scale >= 0.0f) || !std::isfinite(scale) || std::isnan(threshold)) return TQ_ERR_INVALID_ARG;
  if (window < 0 || evict_block < 1 || W_max < 1 ||
      static_cast<long long>(window) + evict_block > W_max)
    return TQ_ERR_INVALID_ARG;
  if ((k_new == nullptr) != (v_new == nullptr)) return TQ_ERR_INVALID_ARG;
  const int G = Hq / Hkv;
  if (G != 1 && G != 2 && G != 4 && G != 8) return TQ_ERR_UNSUPPORTED;
  if (!tq::aligned(k_hot, 16) || !tq::aligned(v_hot, 16) || !tq::aligned(page_pool, 16) ||
      !tq::aligned(workspace, 256))
    return TQ_ERR_INVALID_ARG;
  if (k_new && (!tq::aligned(k_new, 16) || !tq::aligned(v_new, 16))) return TQ_ERR_INVALID_ARG;
  const size_t need = tq::monarch_workspace_bytes(ctx, B, Hq, Hkv, max_pages, W_max, evict_block);
  if (need == 0 || ws_bytes < need) return TQ_ERR_INVALID_ARG;
  return static_cast<tq_status>(tq::launch_monarch_step(
      ctx, q, q_dtype, B, Hq, Hkv, scale, k_new, v_new, k_hot, v_hot, W_max, hot_start, hot_len,
      page_pool, pool_pages, page_table, max_pages, cold_len, threshold, window, evict_block,
      promo, cold_used, out, workspace, ws_bytes, stream));
}

size_t tq_tensor_cache_workspace_bytes(const tq_ctx* ctx, int B, int Hq, int Hkv, int W) {
  if (!ctx || B <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || W <= 0) return 0;
  return tq::tensor_cache_workspace_bytes(ctx, B, Hq, Hkv, W);
}

tq_status tq_tensor_cache_step(const tq_ctx* ctx, const void* q, tq_dtype q_dtype, int B, int Hq,
                               int Hkv, float scale, const void* k_new, const void* v_new,
                               void* k_ring, void* v_ring, int W, int32_t* ring_start,
                               int32_t* ring_len, float* A, const float* lambda,
                               const float* eta, const float* gate, float* out,
                               void* workspace, size_t ws_bytes, void* stream) {
  if (!ctx || !q || !k_new || !v_new || !k_ring || !v_ring || !ring_start || !ring_len || !A ||
      !lambda || !eta || !gate || !out || !workspace)
    return TQ_ERR_INVALID_ARG;
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || W <= 0) return TQ_ERR_INVALID_ARG;
  if (q_dtype != TQ_F32 && q_dtype != TQ_F16 && q_dtype != TQ_BF16) return TQ_ERR_INVALID_ARG;
  if (!(scale >= 0.0f) || !std::isfinite(scale)) return TQ_ERR_INVALID_ARG;
  const int G = Hq / Hkv;
  if (G != 1 && G != 2 && G != 4 && G != 8) return TQ_ERR_UNSUPPORTED;
  if (!tq::aligned(k_ring, 16) || !tq::aligned(v_ring, 16) || !tq::aligned(workspace, 256))
    return TQ_ERR_INVALID_ARG;
  const size_t need = tq::tensor_cache_workspace_bytes(ctx, B, Hq, Hkv, W);
  if (need == 0 || ws_bytes < need) return TQ_ERR_INVALID_ARG;
  return static_cast<tq_status>(tq::launch_tensor_cache_step(
      ctx, q, q_dtype, B, Hq, Hkv, scale, k_new, v_new, k_ring, v_ring, W, ring_start, ring_len,
      A, lambda, eta, gate, out, workspace, ws_bytes, stream));
}

tq_status tq_self_index_build(const tq_ctx* ctx, const void* k, int B, int Hkv, int T, float* mu,
                              uint8_t* codes, float* centroids, void* stream) {
  if (!ctx || !k || !mu || !codes || !centroids || B <= 0 || Hkv <= 0 || T <= 0)
    return TQ_ERR_INVALID_ARG;
  if (!tq::aligned(k, 16) || !tq::aligned(codes, 16) || !tq::aligned(centroids, 16))
    return TQ_ERR_INVALID_ARG;
  return static_cast<tq_status>(
      tq::launch_self_index_build(ctx, k, B, Hkv, T, mu, codes, centroids, stream));
}

tq_status tq_self_index_scores(const tq_ctx* ctx, const void* q, tq_dtype q_dtype, int B, int Hq,
                               int Hkv, int T, const uint8_t* codes, const float* centroids,
                               float* scores, void* stream) {
  if (!ctx || !q || !codes || !centroids || !scores || B <= 0 || Hq <= 0 || Hkv <= 0 || T <= 0 ||
      Hq % Hkv != 0)
    return TQ_ERR_INVALID_ARG;
  if (q_dtype != TQ_F32 && q_dtype != TQ_F16 && q_dtype != TQ_BF16) return TQ_ERR_INVALID_ARG;
  if (!tq::aligned(codes, 16) || !tq::aligned(centroids, 16)) return TQ_ERR_INVALID_ARG;
  return static_cast<tq_status>(tq::launch_self_index_scores(ctx, q, q_dtype, B, Hq, Hkv, T, codes,
                                                             centroids, scores, stream));
}

// Tokens the selection returns per row: top_k, or every position after the
// sinks when there are fewer.
static int self_index_k_eff(int T, int n_sink, int top_k) {
  const int cand = T > n_sink ? T - n_sink : 0;
  return top_k < cand ? top_k : cand;
}

tq_status tq_self_index_select(const tq_ctx* ctx, const float* scores, int rows, int T,
                               int n_sink, int top_k, int32_t* picked, void* stream) {
  if (!ctx || !scores || !picked || rows <= 0 || T < 0 || n_sink < 0 || top_k <= 0)
    return TQ_ERR_INVALID_ARG;
  const int lo = n_sink < T ? n_sink : T;
  return static_cast<tq_status>(tq::launch_self_index_select(
      ctx, scores, rows, T, lo, self_index_k_eff(T, n_sink, top_k), top_k, picked, stream));
}

tq_status tq_self_index_attend(const tq_ctx* ctx, const void* q, tq_dtype q_dtype, int B, int Hq,
                               int Hkv, int T, const void* keys, const void* values,
                               const int32_t* picked, int n_sink, int top_k, float scale,
                               float* out, void* stream) {
  if (!ctx || !q || !keys || !values || !picked || !out || B <= 0 || Hq <= 0 || Hkv <= 0 ||
      Hq % Hkv != 0 || T < 0 || n_sink < 0 || top_k <= 0)
    return TQ_ERR_INVALID_ARG;
  if (q_dtype != TQ_F32 && q_dtype != TQ_F16 && q_dtype != TQ_BF16) return TQ_ERR_INVALID_ARG;
  if (!tq::aligned(keys, 16) || !tq::aligned(values, 16)) return TQ_ERR_INVALID_ARG;
  if (!(scale >= 0.0f) || !std::isfinite(scale)) return TQ_ERR_INVALID_ARG;
  if (scale == 0.0f) scale = 1.0f / std::sqrt(static_cast<float>(ctx->cfg.head_dim));
  const int n_s = n_sink < T ? n_sink : T;
  return static_cast<tq_status>(tq::launch_self_index_attend(
      ctx, q, q_dtype, B, Hq, Hkv, T, keys, values, picked, top_k,
      self_index_k_eff(T, n_sink, top_k), n_s, scale, out, stream));
}

size_t tq_stage1_code_bytes(const tq_ctx* ctx, int kind, int bits1, int bits2) {
  if (!ctx) return 0;
  return tq::stage1_code_bytes(ctx->cfg.head_dim, kind, bits1, bits2);
}

tq_status tq_stage1_encode(const tq_ctx* ctx, int kind, int bits1, int bits2, const float* x_rot,
                           int64_t N, uint8_t* codes, uint16_t* norms, void* stream) {
  if (!ctx || N < 0 || (N > 0 && (!x_rot || !codes || !norms))) return TQ_ERR_INVALID_ARG;
  if (N > 0 && (!tq::aligned(x_rot, 16) || !tq::aligned(codes, 4))) return TQ_ERR_INVALID_ARG;
  if (tq::stage1_code_bytes(ctx->cfg.head_dim, kind, bits1, bits2) == 0) return TQ_ERR_UNSUPPORTED;
  return static_cast<tq_status>(tq::launch_stage1(ctx, kind, bits1, bits2, true, x_rot, nullptr,
                                                  codes, nullptr, norms, nullptr, N, stream));
}

tq_status tq_stage1_decode(const tq_ctx* ctx, int kind, int bits1, int bits2, const uint8_t* codes,
                           const uint16_t* norms, int64_t N, float* x_hat, void* stream) {
  if (!ctx || N < 0 || (N > 0 && (!x_hat || !codes || !norms))) return TQ_ERR_INVALID_ARG;
  if (N > 0 && (!tq::aligned(x_hat, 16) || !tq::aligned(codes, 4))) return TQ_ERR_INVALID_ARG;
  if (tq::stage1_code_bytes(ctx->cfg.head_dim, kind, bits1, bits2) == 0) return TQ_ERR_UNSUPPORTED;
  return static_cast<tq_status>(tq::launch_stage1(ctx, kind, bits1, bits2, false, nullptr, codes,
                                                  nullptr, norms, nullptr, x_hat, N, stream));
}

size_t tq_topk_workspace_bytes(const tq_ctx* ctx, int Q, int64_t N, int k) {
  if (!ctx || Q <= 0 || N <= 0 || k <= 0) return 0;
  return tq::topk_workspace_bytes(ctx, Q, N, k);
}

tq_status tq_score_topk(const tq_ctx* ctx, const float* queries, int Q, const uint8_t* db_pages,
                        int64_t N, int k, int32_t* out_ids, float* out_scores, void* workspace,
                        size_t ws_bytes, void* stream) {
  tq::Range range("tq_score_topk");
  if (!ctx || !queries || !db_pages || !out_ids || !out_scores || !workspace)
    return TQ_ERR_INVALID_ARG;
  if (Q <= 0 || N <= 0 || k <= 0) return TQ_ERR_INVALID_ARG;
  if (k > 32) return TQ_ERR_UNSUPPORTED;
  if (!tq::aligned(db_pages, 16) || !tq::aligned(queries, 16) || !tq::aligned(workspace, 256))
    return TQ_ERR_INVALID_ARG;
  const size_t need = tq::topk_workspace_bytes(ctx, Q, N, k);
  if (need == 0 || ws_bytes < need) return TQ_ERR_INVALID_ARG;
  return static_cast<tq_status>(tq::launch_topk(ctx, queries, Q, db_pages, N, k, out_ids,
                                                out_scores, workspace, ws_bytes, stream));
}

tq_status tq_set_profile_events(tq_ctx* ctx, void* ev_start, void* ev_stop) {
  if (!ctx || ((ev_start == nullptr) != (ev_stop == nullptr))) return TQ_ERR_INVALID_ARG;
  ctx->prof_start = ev_start;
  ctx->prof_stop = ev_stop;
  return TQ_OK;
}

tq_status tq_set_wait_test(tq_ctx* ctx, int skip_unit, uint64_t limit_ns) {
  if (!ctx || skip_unit < -1) return TQ_ERR_INVALID_ARG;
  ctx->wait_skip_unit = skip_unit;
  ctx->wait_ns = limit_ns;
  return TQ_OK;
}

tq_status tq_get_error(const tq_ctx* ctx) {
  if (!ctx) return TQ_ERR_INVALID_ARG;
  int v = 0;
  if (cudaMemcpy(&v, ctx->dev.err, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
    return TQ_ERR_CUDA;
  if (v != 0) {
    const int zero = 0;
    if (cudaMemcpy(ctx->dev.err, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess)
      return TQ_ERR_CUDA;
  }
  return static_cast<tq_status>(v);
}

void tq_destroy(tq_ctx* ctx) {
  if (!ctx) return;
  if (ctx->dev_block) cudaFree(ctx->dev_block);
  delete ctx;
}

}  // extern "C"
