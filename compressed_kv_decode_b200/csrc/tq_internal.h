// Internal declarations shared by the host-side files of libtq.
#pragma once

#include <cuda_runtime.h>

#include <atomic>
#include <cstddef>
#include <cstdint>
#include <vector>

#include "../../include/tq.h"

namespace tq {

// The dynamic shared-memory limit already raised for one kernel, per device
// (zero-initialised as a static; safe to share between threads).
struct SmemAttr {
  std::atomic<int> bytes[64];
};

// Raise `kernel`'s dynamic shared-memory limit to at least `bytes` on the
// current device, once per device and size.
template <typename K>
inline bool raise_smem_limit(K kernel, int bytes, SmemAttr& st) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  std::atomic<int>* slot = (dev >= 0 && dev < 64) ? &st.bytes[dev] : nullptr;
  if (slot && slot->load(std::memory_order_acquire) >= bytes) return true;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess)
    return false;
  if (slot) {
    int cur = slot->load(std::memory_order_relaxed);
    while (cur < bytes && !slot->compare_exchange_weak(cur, bytes, std::memory_order_release)) {
    }
  }
  return true;
}

struct HostTables {
  std::vector<float> rot;    // [d*d] row-major, x_rot = rot x
  std::vector<float> qjl;    // [m*d] row-major, fp16-valued
  std::vector<float> key_c;  // positive levels
  std::vector<float> key_t;  // positive boundaries
  std::vector<float> val_c;
  std::vector<float> val_t;
};

bool config_valid(const tq_config& c);
bool config_supported(const tq_config& c);
bool generate_tables(const tq_config& cfg, HostTables& out);
// Lloyd-Max codebooks used by the stage-1 variants (fp64 results):
// positive levels / boundaries of one sphere coordinate at `bits` bits, and
// the levels / boundaries of the block-pair angle (density sin^(k-1)(2 phi)).
void sphere_lloyd_max(int d, int bits, std::vector<double>& c, std::vector<double>& t);
void angle_lloyd_max(int k, int bits, std::vector<double>& c, std::vector<double>& t);

// Small per-context constants passed to kernels by value.
struct Codebook {
  float key_c[2];
  float key_t[1];
  float val_c[8];
  float val_t[7];
};

// Device tables owned by a context.
struct DeviceTables {
  const float* rot;          // [d*d] fp32
  const float* qjl;          // [m*d] fp32 (fp16 values)
  const uint16_t* qjl_h;     // [m*d] fp16 bits
  const uint16_t* rot_bf_hi; // [d*d] bf16 bits of rot
  const uint16_t* rot_bf_lo; // [d*d] bf16 bits of rot - bf16(rot)
  const uint16_t* rot_h_hi;  // [d*d] fp16 bits of rot
  const uint16_t* rot_h_lo;  // [d*d] fp16 bits of rot - fp16(rot)
  const float* sp;           // [m*d] S Pi (fp32)
  int* err;                  // device error word (first error wins)
};

}  // namespace tq

struct tq_ctx {
  tq_config cfg;
  int device;
  int num_sms;
  tq::HostTables host;
  tq::Codebook cb;
  tq::DeviceTables dev;
  void* dev_block;  // single allocation holding every device table
  void* prof_start; // optional cudaEvent_t pair around the main kernel
  void* prof_stop;
  int wait_skip_unit;         // testing aid: cold unit whose copy is not issued (-1: none)
  unsigned long long wait_ns; // testing aid: bound of the attention's waits (0: default)
};

namespace tq {

// Page layout (bytes) for head dim d, sketch dim m.  Keys-only pages (record
// layout): section offsets kc, qs, kn, kg; block = 0.  Pages with values
// (block layout, 8 blocks of 16 token slots): offsets inside a block -- kc (key
// plane H), kl (key plane L), qs, vc, kn (the (n, gamma) pair of token 0), vn
// (value norm of token 0) -- and the block size.
struct PageLayout {
  size_t kc, kl, qs, vc, kn, kg, vn, block, bytes;
};
PageLayout page_layout(int d, int m, bool with_values);

// Threshold gate of the gated decode: a q head reads its cold tokens only
// when its largest raw hot score is below threshold; cold_used [B, Hq] (may
// be null) receives 1 / 0 per head.
struct DecodeGate {
  float threshold;
  int32_t* cold_used;
};

// Optional parts of a decode call that steps a ring (Tensor Cache): the prep
// launch writes the step's token (fp16 rows of [B, Hkv, D]) into ring slot
// (hot_start + hot_len - 1) mod W_max of its (batch, kv head) before the
// attention reads the ring; the combine's epilogue adds sigmoid(gate[h]) r
// (the memory read) and copies the ring start and length of the step back to
// the caller's arrays.
struct DecodeFuse {
  const float* r;         // [B, Hq, D]
  const float* gate;      // [Hq]
  const int32_t* src_start;
  const int32_t* src_len;  // [B]
  int32_t* dst_start;
  int32_t* dst_len;  // [B]
  const void* k_new;
  const void* v_new;  // fp16 [B, Hkv, D], or null: no token to write
  void* k_ring;
  void* v_ring;  // fp16 [B, Hkv, W_max, D]
};

// Launchers (defined in the .cu files).  Return a tq_status.
// Inputs and outputs of Monarch's promotion for the decode (all device):
// cold positions moved back are skipped; the attention writes every cold
// logit (log2 domain, scale folded in) and the combine the log-sum-exp of each
// query head over the tokens it attended (+inf where its gate kept it off the
// cold tier, or where it attended nothing).
struct DecodePromo {
  const uint32_t* cold_mask;  // [B][max_pages * 4] bit p % 32 of word p / 32: position p skipped
  float* logits;              // [B][Hq][max_pages * 128]
  float* lse;                 // [B][Hq]
};

int launch_decode(const tq_ctx* ctx, const void* q, tq_dtype q_dtype, int B, int Hq, int Hkv,
                  float scale, const void* k_hot, const void* v_hot, int W_max,
                  const int32_t* hot_start, const int32_t* hot_len, const uint8_t* pool,
                  int64_t pool_pages, const int32_t* page_table, int max_pages,
                  const int32_t* cold_len, const DecodeGate* gate, float* out, void* ws,
                  size_t ws_bytes, void* stream, const DecodeFuse* fuse = nullptr,
                  const DecodePromo* promo = nullptr);
size_t decode_workspace_bytes(const tq_ctx* ctx, int B, int Hq, int Hkv, int max_pages, int W_max);

int launch_compress(const tq_ctx* ctx, const void* k, const void* v, tq_dtype dtype, int flags,
                    int B, int Hkv, int n_new, uint8_t* pool, int64_t pool_pages,
                    const int32_t* page_table, int max_pages, int32_t* cold_len, void* stream);

// n_new_b (device [B], may be null): tokens appended per sequence, at most
// n_new each (the input still holds n_new rows per (batch, kv head)); with it
// cold_len is left for the caller to advance.
int launch_compress_tc(const tq_ctx* ctx, const void* k, const void* v, bool bf16, int B, int Hkv,
                       int n_new, uint8_t* pool, int64_t pool_pages, const int32_t* page_table,
                       int max_pages, int32_t* cold_len, void* stream,
                       const int32_t* n_new_b = nullptr);

// One Monarch decode step (append, gated attention, eviction); see tq.h.
int launch_monarch_step(const tq_ctx* ctx, const void* q, tq_dtype q_dtype, int B, int Hq, int Hkv,
                        float scale, const void* k_new, const void* v_new, void* k_hot,
                        void* v_hot, int W_max, int32_t* hot_start, int32_t* hot_len,
                        uint8_t* pool, int64_t pool_pages, const int32_t* page_table,
                        int max_pages, int32_t* cold_len, float threshold, int window,
                        int evict_block, const tq_promotion* promo, int32_t* cold_used,
                        float* out, void* ws, size_t ws_bytes, void* stream);
size_t tensor_cache_workspace_bytes(const tq_ctx* ctx, int B, int Hq, int Hkv, int W);
int launch_tensor_cache_step(const tq_ctx* ctx, const void* q, tq_dtype q_dtype, int B, int Hq,
                             int Hkv, float scale, const void* k_new, const void* v_new,
                             void* k_ring, void* v_ring, int W, int32_t* ring_start,
                             int32_t* ring_len, float* A, const float* lambda, const float* eta,
                             const float* gate, float* out, void* ws, size_t ws_bytes,
                             void* stream);
int launch_self_index_build(const tq_ctx* ctx, const void* k, int B, int Hkv, int T, float* mu,
                            uint8_t* codes, float* cent, void* stream);
int launch_self_index_scores(const tq_ctx* ctx, const void* q, tq_dtype q_dtype, int B, int Hq,
                             int Hkv, int T, const uint8_t* codes, const float* cent,
                             float* scores, void* stream);
int launch_self_index_select(const tq_ctx* ctx, const float* scores, int rows, int T, int lo,
                             int k_eff, int k_cap, int32_t* picked, void* stream);
int launch_self_index_attend(const tq_ctx* ctx, const void* q, tq_dtype q_dtype, int B, int Hq,
                             int Hkv, int T, const void* keys, const void* values,
                             const int32_t* picked, int k_cap, int k_eff, int n_s, float scale,
                             float* out, void* stream);
size_t stage1_code_bytes(int d, int kind, int b1, int b2);
int launch_stage1(const tq_ctx* ctx, int kind, int b1, int b2, bool encode, const float* x,
                  const uint8_t* codes_in, uint8_t* codes_out, const uint16_t* norms_in,
                  uint16_t* norms_out, float* xhat, long long N, void* stream);
size_t monarch_workspace_bytes(const tq_ctx* ctx, int B, int Hq, int Hkv, int max_pages,
                               int W_max, int evict_block);

int launch_topk(const tq_ctx* ctx, const float* queries, int Q, const uint8_t* db, int64_t N,
                int k, int32_t* out_ids, float* out_scores, void* ws, size_t ws_bytes,
                void* stream);
size_t topk_workspace_bytes(const tq_ctx* ctx, int Q, int64_t N, int k);

}  // namespace tq
