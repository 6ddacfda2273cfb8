// C ABI of libcsa2: argument validation, workspace sizing and kernel launches.
// The declarations, argument meanings, layouts and error behaviour are documented in
// include/csa2.h; this file only checks host-visible arguments and enqueues kernels.
#include <cmath>
#include <cstdint>

#include "csa2_device.cuh"

namespace csa2 {
cudaError_t launch_pack_kv(const void* kv, const void* ik, int64_t T, int ratio,
                           const int64_t* dst, int64_t pool_entries, uint8_t* kv_pool,
                           uint8_t* ik_pool, uint32_t* status, cudaStream_t stream, int num_sms);
cudaError_t launch_pack_kv_normed(const void* kv, const void* ik, int64_t T, int ratio, const int64_t* pos,
                                  const float* rope_cos, const float* rope_sin, int64_t n_pos, const float* gamma,
                                  float eps, const int64_t* dst, int64_t pool_entries, uint8_t* kv_pool,
                                  uint8_t* ik_pool, uint32_t* status, cudaStream_t stream, int num_sms);
cudaError_t launch_index(int mode, const float* q, const float* w, const uint8_t* ik_pool,
                         int64_t pool_entries, const int64_t* seq_base, const int32_t* n_vis,
                         const int32_t* blocks, int B, int Q, int HI, int n_blocks, int block,
                         int K, int64_t max_n_vis, int32_t* out_idx, float* out_score,
                         uint32_t* keys, int64_t key_stride, uint32_t* status,
                         cudaStream_t stream, int withheld_tile = -1, uint32_t* gmax = nullptr,
                         int64_t gstride = 0);
size_t attn_workspace_bytes(int B, int Q, int H, int K, int window);
cudaError_t launch_sparse_attn(const float* q, const uint8_t* kv_pool, int64_t pool_entries,
                               const int64_t* seq_base, const int32_t* topk, int K,
                               const uint8_t* swa, int S_w, const int64_t* swa_start,
                               const int64_t* q_pos, int window, int B, int Q, int H,
                               float sm_scale, float* out, float* lse, void* ws,
                               uint32_t* status, cudaStream_t stream);
cudaError_t launch_shard_vis(const int32_t* n_vis, const int64_t* lo, const int64_t* len, int B, int Q,
                             int32_t* out, uint32_t* status, cudaStream_t stream);
cudaError_t launch_topk_merge(const int32_t* cand, const float* score, int64_t part, const int64_t* shard_off,
                              int C, int B, int Q, int Kc, int K, int32_t* topk, float* topk_score, uint32_t* keys,
                              int32_t* labels, int64_t stride, uint32_t* status, cudaStream_t stream);
cudaError_t launch_topk_localize(const int32_t* topk, int B, int Q, int K, const int64_t* off, const int64_t* len,
                                 int32_t* out, uint32_t* status, cudaStream_t stream);
cudaError_t launch_attn_combine(const float* out_parts, int64_t part_o, const float* lse_parts, int64_t part_l,
                                int C, int64_t N, float* out, float* lse, cudaStream_t stream);
}  // namespace csa2

namespace {

constexpr int64_t kMaxQueries = 65535;  // grid.y limit of the per-query kernels
constexpr int64_t kMaxNVis = (int64_t)1 << 23;  // largest accepted visible count: a selection CTA then
                                                // counts at most 2^23 keys in 32-bit counters

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

size_t round256(size_t x) { return (x + 255) & ~(size_t)255; }

// Keys per query row in the workspace, rounded up so every row starts 16-byte aligned.
int64_t key_row(int64_t n) { return (n + 3) & ~(int64_t)3; }

csa2_status launched(cudaError_t e) { return e == cudaSuccess ? CSA2_OK : CSA2_ERR_CUDA; }

bool valid_block(int block) {
  return block == 1 || block == 2 || block == 4 || block == 8 || block == 16 || block == 32;
}

int current_sm_count() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

// Checks shared by the three indexer calls.
csa2_status check_index_common(const float* q, const float* w, const uint8_t* ik_pool,
                               int64_t pool_entries, const int64_t* seq_base,
                               const int32_t* n_vis, int B, int Q, int HI, int64_t max_n_vis) {
  if (B < 0 || Q < 0 || pool_entries < 0 || max_n_vis < 0) return CSA2_ERR_INVALID_ARG;
  if ((int64_t)B * Q == 0) return CSA2_OK;
  if (!q || !w || !ik_pool || !seq_base || !n_vis) return CSA2_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(w, 4) || !aligned(ik_pool, 16) || !aligned(seq_base, 8) ||
      !aligned(n_vis, 4))
    return CSA2_ERR_INVALID_ARG;
  if (HI < 1 || HI > CSA2_MAX_HI) return CSA2_ERR_UNSUPPORTED;
  if ((int64_t)B * Q > kMaxQueries || max_n_vis > kMaxNVis) return CSA2_ERR_UNSUPPORTED;
  return CSA2_OK;
}

csa2_status check_ws(const void* ws, size_t ws_bytes, size_t need) {
  if (need == 0) return CSA2_OK;
  if (!ws || ws_bytes < need || !aligned(ws, 256)) return CSA2_ERR_INVALID_ARG;
  return CSA2_OK;
}

}  // namespace

extern "C" {

const char* csa2_status_string(csa2_status s) {
  switch (s) {
    case CSA2_OK: return "CSA2_OK";
    case CSA2_ERR_INVALID_ARG: return "CSA2_ERR_INVALID_ARG: null/misaligned pointer or bad size";
    case CSA2_ERR_UNSUPPORTED: return "CSA2_ERR_UNSUPPORTED: shape outside the supported range";
    case CSA2_ERR_CUDA: return "CSA2_ERR_CUDA: kernel launch failed";
    case CSA2_ERR_TIMEOUT: return "CSA2_ERR_TIMEOUT: a device-side wait hit its cap";
    case CSA2_ERR_DEVICE_INPUT: return "CSA2_ERR_DEVICE_INPUT: out-of-range device-side value";
  }
  return "unknown csa2_status";
}

csa2_status csa2_status_from_device_word(uint32_t word) {
  if (word & CSA2_DEV_TIMEOUT) return CSA2_ERR_TIMEOUT;
  if (word & (CSA2_DEV_BAD_INDEX | CSA2_DEV_BAD_COUNT)) return CSA2_ERR_DEVICE_INPUT;
  return CSA2_OK;
}

int csa2_version(void) { return 100; }

csa2_status csa2_pack_kv(const void* kv, const void* ik, int64_t T, int ratio,
                         const int64_t* dst_entry, int64_t pool_entries, uint8_t* kv_pool,
                         uint8_t* ik_pool, uint32_t* dev_status, cudaStream_t stream) {
  if (ratio != 1 && ratio != 2) return CSA2_ERR_UNSUPPORTED;
  if (T < 0 || pool_entries < 0 || T % ratio != 0) return CSA2_ERR_INVALID_ARG;
  if (T == 0) return CSA2_OK;
  if (!kv || !ik || !kv_pool || !ik_pool) return CSA2_ERR_INVALID_ARG;
  if (!aligned(kv, 16) || !aligned(ik, 16) || !aligned(kv_pool, 16) || !aligned(ik_pool, 16))
    return CSA2_ERR_INVALID_ARG;
  if (dst_entry && !aligned(dst_entry, 8)) return CSA2_ERR_INVALID_ARG;
  if (!dst_entry && T / ratio > pool_entries) return CSA2_ERR_INVALID_ARG;
  if (dev_status && !aligned(dev_status, 4)) return CSA2_ERR_INVALID_ARG;
  return launched(csa2::launch_pack_kv(kv, ik, T, ratio, dst_entry, pool_entries, kv_pool,
                                       ik_pool, dev_status, stream, current_sm_count()));
}

csa2_status csa2_pack_kv_normed(const void* kv, const void* ik, int64_t T, int ratio, const int64_t* pos,
                                const float* rope_cos, const float* rope_sin, int64_t n_pos, const float* gamma,
                                float eps, const int64_t* dst_entry, int64_t pool_entries, uint8_t* kv_pool,
                                uint8_t* ik_pool, uint32_t* dev_status, cudaStream_t stream) {
  if (ratio != 1 && ratio != 2) return CSA2_ERR_UNSUPPORTED;
  if (T < 0 || pool_entries < 0 || n_pos < 0 || T % ratio != 0) return CSA2_ERR_INVALID_ARG;
  if (!(eps >= 0.0f) || !std::isfinite(eps)) return CSA2_ERR_INVALID_ARG;
  if (T == 0) return CSA2_OK;
  if (!kv || !ik || !pos || !rope_cos || !rope_sin || !kv_pool || !ik_pool) return CSA2_ERR_INVALID_ARG;
  if (!aligned(kv, 16) || !aligned(ik, 16) || !aligned(kv_pool, 16) || !aligned(ik_pool, 16) ||
      !aligned(pos, 8) || !aligned(rope_cos, 16) || !aligned(rope_sin, 16) || (gamma && !aligned(gamma, 16)))
    return CSA2_ERR_INVALID_ARG;
  if (dst_entry && !aligned(dst_entry, 8)) return CSA2_ERR_INVALID_ARG;
  if (!dst_entry && T / ratio > pool_entries) return CSA2_ERR_INVALID_ARG;
  if (dev_status && !aligned(dev_status, 4)) return CSA2_ERR_INVALID_ARG;
  return launched(csa2::launch_pack_kv_normed(kv, ik, T, ratio, pos, rope_cos, rope_sin, n_pos, gamma, eps,
                                              dst_entry, pool_entries, kv_pool, ik_pool, dev_status, stream,
                                              current_sm_count()));
}

// The flat index workspace: the keys [B*Q][key_row(max_n_vis)], then the largest key of every
// 32 [B*Q][key_row(ceil(max_n_vis / 32))].
size_t full_keys_bytes(int B, int Q, int64_t max_n_vis) {
  return round256((size_t)B * Q * (size_t)key_row(max_n_vis) * sizeof(uint32_t));
}
int64_t full_gmax_row(int64_t max_n_vis) { return key_row((max_n_vis + 31) / 32); }

size_t csa2_index_full_workspace_size(int B, int Q, int HI, int K, int64_t max_n_vis) {
  (void)HI;
  (void)K;
  if (B <= 0 || Q <= 0 || max_n_vis <= 0) return 0;
  return full_keys_bytes(B, Q, max_n_vis) +
         round256((size_t)B * Q * (size_t)full_gmax_row(max_n_vis) * sizeof(uint32_t));
}

csa2_status csa2_index_full(const float* q, const float* w, const uint8_t* ik_pool,
                            int64_t pool_entries, const int64_t* seq_base, const int32_t* n_vis,
                            int B, int Q, int HI, int K, int64_t max_n_vis, int32_t* topk,
                            float* topk_score, void* ws, size_t ws_bytes, uint32_t* dev_status,
                            cudaStream_t stream) {
  csa2_status st = check_index_common(q, w, ik_pool, pool_entries, seq_base, n_vis, B, Q, HI,
                                      max_n_vis);
  if (st != CSA2_OK) return st;
  if (K < 1 || K > CSA2_MAX_K) return CSA2_ERR_UNSUPPORTED;
  if ((int64_t)B * Q == 0) return CSA2_OK;
  if (!topk || !aligned(topk, 4) || (topk_score && !aligned(topk_score, 4))) return CSA2_ERR_INVALID_ARG;
  const size_t need = csa2_index_full_workspace_size(B, Q, HI, K, max_n_vis);
  if ((st = check_ws(ws, ws_bytes, need)) != CSA2_OK) return st;
  uint32_t* gmax = reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(ws) + full_keys_bytes(B, Q, max_n_vis));
  return launched(csa2::launch_index(0, q, w, ik_pool, pool_entries, seq_base, n_vis, nullptr, B,
                                     Q, HI, 0, 1, K, max_n_vis, topk, topk_score,
                                     static_cast<uint32_t*>(ws), key_row(max_n_vis), dev_status, stream, -1,
                                     gmax, full_gmax_row(max_n_vis)));
}

csa2_status csa2_test_index_full_withheld_copy(const float* q, const float* w, const uint8_t* ik_pool,
                                               int64_t pool_entries, const int64_t* seq_base,
                                               const int32_t* n_vis, int B, int Q, int HI, int K,
                                               int64_t max_n_vis, int32_t* topk, float* topk_score, void* ws,
                                               size_t ws_bytes, uint32_t* dev_status, cudaStream_t stream,
                                               int withheld_tile) {
  csa2_status st = check_index_common(q, w, ik_pool, pool_entries, seq_base, n_vis, B, Q, HI,
                                      max_n_vis);
  if (st != CSA2_OK) return st;
  if (K < 1 || K > CSA2_MAX_K) return CSA2_ERR_UNSUPPORTED;
  if (withheld_tile < 0) return CSA2_ERR_INVALID_ARG;
  if ((int64_t)B * Q == 0) return CSA2_OK;
  if (!topk || !aligned(topk, 4) || (topk_score && !aligned(topk_score, 4))) return CSA2_ERR_INVALID_ARG;
  const size_t need = csa2_index_full_workspace_size(B, Q, HI, K, max_n_vis);
  if ((st = check_ws(ws, ws_bytes, need)) != CSA2_OK) return st;
  return launched(csa2::launch_index(0, q, w, ik_pool, pool_entries, seq_base, n_vis, nullptr, B,
                                     Q, HI, 0, 1, K, max_n_vis, topk, topk_score,
                                     static_cast<uint32_t*>(ws), key_row(max_n_vis), dev_status, stream,
                                     withheld_tile));
}

size_t csa2_index_hier_workspace_size(int B, int Q, int HI, int n_blocks, int block,
                                      int64_t max_n_vis) {
  (void)HI;
  (void)n_blocks;
  if (B <= 0 || Q <= 0 || max_n_vis <= 0 || block <= 0) return 0;
  const int64_t nb = (max_n_vis + block - 1) / block;
  return round256((size_t)B * Q * (size_t)key_row(nb) * sizeof(uint32_t));
}

csa2_status csa2_index_hier(const float* q, const float* w, const uint8_t* ik_pool,
                            int64_t pool_entries, const int64_t* seq_base, const int32_t* n_vis,
                            int B, int Q, int HI, int n_blocks, int block, int64_t max_n_vis,
                            int32_t* blocks, float* block_score, void* ws, size_t ws_bytes,
                            uint32_t* dev_status, cudaStream_t stream) {
  csa2_status st = check_index_common(q, w, ik_pool, pool_entries, seq_base, n_vis, B, Q, HI,
                                      max_n_vis);
  if (st != CSA2_OK) return st;
  if (n_blocks < 1 || n_blocks > CSA2_MAX_K || !valid_block(block)) return CSA2_ERR_UNSUPPORTED;
  if ((int64_t)B * Q == 0) return CSA2_OK;
  if (!blocks || !aligned(blocks, 4) || (block_score && !aligned(block_score, 4)))
    return CSA2_ERR_INVALID_ARG;
  const size_t need = csa2_index_hier_workspace_size(B, Q, HI, n_blocks, block, max_n_vis);
  if ((st = check_ws(ws, ws_bytes, need)) != CSA2_OK) return st;
  const int64_t stride = key_row((max_n_vis + block - 1) / block);
  return launched(csa2::launch_index(1, q, w, ik_pool, pool_entries, seq_base, n_vis, nullptr, B,
                                     Q, HI, n_blocks, block, n_blocks, max_n_vis, blocks,
                                     block_score, static_cast<uint32_t*>(ws), stride, dev_status,
                                     stream));
}

size_t csa2_reindex_workspace_size(int B, int Q, int HI, int n_blocks, int block, int K) {
  (void)HI;
  (void)K;
  if (B <= 0 || Q <= 0 || n_blocks <= 0 || block <= 0) return 0;
  return round256((size_t)B * Q * (size_t)key_row((int64_t)n_blocks * block) * sizeof(uint32_t));
}

csa2_status csa2_reindex(const float* q, const float* w, const uint8_t* ik_pool,
                         int64_t pool_entries, const int64_t* seq_base, const int32_t* n_vis,
                         const int32_t* blocks, int n_blocks, int block, int B, int Q, int HI,
                         int K, int32_t* topk, float* topk_score, void* ws, size_t ws_bytes,
                         uint32_t* dev_status, cudaStream_t stream) {
  csa2_status st = check_index_common(q, w, ik_pool, pool_entries, seq_base, n_vis, B, Q, HI,
                                      kMaxNVis);
  if (st != CSA2_OK) return st;
  if (n_blocks < 1 || n_blocks > CSA2_MAX_K || !valid_block(block)) return CSA2_ERR_UNSUPPORTED;
  if (K < 1 || K > CSA2_MAX_K) return CSA2_ERR_UNSUPPORTED;
  if ((int64_t)B * Q == 0) return CSA2_OK;
  if (!blocks || !aligned(blocks, 4) || !topk || !aligned(topk, 4) ||
      (topk_score && !aligned(topk_score, 4)))
    return CSA2_ERR_INVALID_ARG;
  const size_t need = csa2_reindex_workspace_size(B, Q, HI, n_blocks, block, K);
  if ((st = check_ws(ws, ws_bytes, need)) != CSA2_OK) return st;
  return launched(csa2::launch_index(2, q, w, ik_pool, pool_entries, seq_base, n_vis, blocks, B, Q,
                                     HI, n_blocks, block, K, kMaxNVis, topk, topk_score,
                                     static_cast<uint32_t*>(ws), key_row((int64_t)n_blocks * block),
                                     dev_status, stream));
}

size_t csa2_sparse_attn_workspace_size(int B, int Q, int H, int K, int window) {
  if (B <= 0 || Q <= 0 || H <= 0 || K < 0 || window < 0) return 0;
  return round256(csa2::attn_workspace_bytes(B, Q, H, K, window));
}

csa2_status csa2_sparse_attn(const float* q, const uint8_t* kv_pool, int64_t pool_entries,
                             const int64_t* seq_base, const int32_t* topk, int K,
                             const uint8_t* swa, int S_w, const int64_t* swa_start,
                             const int64_t* q_pos, int window, int B, int Q, int H,
                             float sm_scale, float* out, float* lse, void* ws, size_t ws_bytes,
                             uint32_t* dev_status, cudaStream_t stream) {
  if (B < 0 || Q < 0 || K < 0 || S_w < 0 || window < 0 || pool_entries < 0)
    return CSA2_ERR_INVALID_ARG;
  if (!std::isfinite(sm_scale)) return CSA2_ERR_INVALID_ARG;
  if (H != 16 && H != 32 && H != 48 && H != 64) return CSA2_ERR_UNSUPPORTED;
  if (K > CSA2_MAX_K || window > CSA2_MAX_WINDOW) return CSA2_ERR_UNSUPPORTED;
  if ((int64_t)B * Q > kMaxQueries) return CSA2_ERR_UNSUPPORTED;
  if ((int64_t)B * Q == 0) return CSA2_OK;
  if (!q || !seq_base || !q_pos || !out || !lse) return CSA2_ERR_INVALID_ARG;
  if (K > 0 && (!topk || !kv_pool)) return CSA2_ERR_INVALID_ARG;
  if (S_w > 0 && (!swa || !swa_start)) return CSA2_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(seq_base, 8) || !aligned(q_pos, 8) || !aligned(out, 16) ||
      !aligned(lse, 4) || (topk && !aligned(topk, 4)) || (kv_pool && !aligned(kv_pool, 16)) ||
      (swa && !aligned(swa, 16)) || (swa_start && !aligned(swa_start, 8)))
    return CSA2_ERR_INVALID_ARG;
  const int win = S_w > 0 ? window : 0;
  const size_t need = csa2_sparse_attn_workspace_size(B, Q, H, K, win);
  csa2_status st = check_ws(ws, ws_bytes, need);
  if (st != CSA2_OK) return st;
  return launched(csa2::launch_sparse_attn(q, kv_pool, pool_entries, seq_base, topk, K, swa, S_w,
                                           swa_start, q_pos, window, B, Q, H, sm_scale, out, lse,
                                           ws, dev_status, stream));
}

// ---- context-parallel decode -----------------------------------------------------------

csa2_status csa2_cp_shard_vis(const int32_t* n_vis, const int64_t* shard_lo, const int64_t* shard_len, int B,
                              int Q, int32_t* n_vis_local, uint32_t* dev_status, cudaStream_t stream) {
  if (B < 0 || Q < 0) return CSA2_ERR_INVALID_ARG;
  if ((int64_t)B * Q == 0) return CSA2_OK;
  if (!n_vis || !shard_lo || !shard_len || !n_vis_local) return CSA2_ERR_INVALID_ARG;
  if (!aligned(n_vis, 4) || !aligned(shard_lo, 8) || !aligned(shard_len, 8) || !aligned(n_vis_local, 4))
    return CSA2_ERR_INVALID_ARG;
  return launched(csa2::launch_shard_vis(n_vis, shard_lo, shard_len, B, Q, n_vis_local, dev_status, stream));
}

size_t csa2_topk_merge_workspace_size(int C, int B, int Q, int Kc) {
  if (C <= 0 || B <= 0 || Q <= 0 || Kc <= 0) return 0;
  const size_t row = (size_t)key_row((int64_t)C * Kc);
  return 2 * round256((size_t)B * Q * row * sizeof(uint32_t));
}

csa2_status csa2_topk_merge(const int32_t* cand, const float* cand_score, int64_t part_stride,
                            const int64_t* shard_off, int C, int B, int Q, int Kc, int K, int32_t* topk,
                            float* topk_score, void* ws, size_t ws_bytes, uint32_t* dev_status,
                            cudaStream_t stream) {
  if (B < 0 || Q < 0 || part_stride < 0) return CSA2_ERR_INVALID_ARG;
  if (C < 1 || C > CSA2_MAX_SHARDS || Kc < 1 || Kc > CSA2_MAX_K || K < 1 || K > CSA2_MAX_K)
    return CSA2_ERR_UNSUPPORTED;
  if ((int64_t)B * Q > kMaxQueries) return CSA2_ERR_UNSUPPORTED;
  if ((int64_t)B * Q == 0) return CSA2_OK;
  if (!cand || !cand_score || !shard_off || !topk) return CSA2_ERR_INVALID_ARG;
  if (!aligned(cand, 4) || !aligned(cand_score, 4) || !aligned(shard_off, 8) || !aligned(topk, 4) ||
      (topk_score && !aligned(topk_score, 4)))
    return CSA2_ERR_INVALID_ARG;
  const size_t need = csa2_topk_merge_workspace_size(C, B, Q, Kc);
  csa2_status st = check_ws(ws, ws_bytes, need);
  if (st != CSA2_OK) return st;
  const int64_t part = part_stride > 0 ? part_stride : (int64_t)B * Q * Kc;
  if (part < (int64_t)B * Q * Kc) return CSA2_ERR_INVALID_ARG;
  const int64_t stride = key_row((int64_t)C * Kc);
  uint32_t* keys = static_cast<uint32_t*>(ws);
  int32_t* labels = reinterpret_cast<int32_t*>(static_cast<uint8_t*>(ws) + need / 2);
  return launched(csa2::launch_topk_merge(cand, cand_score, part, shard_off, C, B, Q, Kc, K, topk, topk_score, keys,
                                          labels, stride, dev_status, stream));
}

csa2_status csa2_topk_localize(const int32_t* topk, int B, int Q, int K, const int64_t* shard_off,
                               const int64_t* shard_len, int32_t* topk_local, uint32_t* dev_status,
                               cudaStream_t stream) {
  if (B < 0 || Q < 0 || K < 0) return CSA2_ERR_INVALID_ARG;
  if ((int64_t)B * Q == 0 || K == 0) return CSA2_OK;
  if (!topk || !shard_off || !shard_len || !topk_local) return CSA2_ERR_INVALID_ARG;
  if (!aligned(topk, 4) || !aligned(shard_off, 8) || !aligned(shard_len, 8) || !aligned(topk_local, 4))
    return CSA2_ERR_INVALID_ARG;
  if (topk == topk_local) return CSA2_ERR_INVALID_ARG;
  return launched(csa2::launch_topk_localize(topk, B, Q, K, shard_off, shard_len, topk_local, dev_status, stream));
}

csa2_status csa2_attn_combine(const float* out_parts, int64_t out_part_stride, const float* lse_parts,
                              int64_t lse_part_stride, int C, int B, int Q, int H, float* out, float* lse,
                              cudaStream_t stream) {
  if (B < 0 || Q < 0 || H < 0 || out_part_stride < 0 || lse_part_stride < 0) return CSA2_ERR_INVALID_ARG;
  if (C < 1 || C > CSA2_MAX_SHARDS) return CSA2_ERR_UNSUPPORTED;
  const int64_t N = (int64_t)B * Q * H;
  if (N == 0) return CSA2_OK;
  if (N > ((int64_t)1 << 31)) return CSA2_ERR_UNSUPPORTED;
  if (!out_parts || !lse_parts || !out || !lse) return CSA2_ERR_INVALID_ARG;
  const int64_t part_o = out_part_stride > 0 ? out_part_stride : N * CSA2_D;
  const int64_t part_l = lse_part_stride > 0 ? lse_part_stride : N;
  if (part_o < N * CSA2_D || part_o % 4 != 0 || part_l < N) return CSA2_ERR_INVALID_ARG;
  if (!aligned(out_parts, 16) || !aligned(lse_parts, 4) || !aligned(out, 16) || !aligned(lse, 4))
    return CSA2_ERR_INVALID_ARG;
  return launched(csa2::launch_attn_combine(out_parts, part_o, lse_parts, part_l, C, N, out, lse, stream));
}

}  // extern "C"
