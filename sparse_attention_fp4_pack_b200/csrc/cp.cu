// Context-parallel decode: one sequence's cached entries split over several GPUs.
//
// The pages describe a single device (P1 = onedev.kr "KV 캐시를 토큰당 890바이트로 압축한
// 552B 멀티모달 MoE, DeepSeek-V4.1-Flash", §무엇과 다른가: a Full layer takes the Top-K of
// everything its query sees; P3 = genexis.ai "100만 토큰을 0.9GB에…", §전역 어텐션과 지역
// 어텐션: one softmax over the selected entries and the window).  Split over shards of
// contiguous entries, both results decompose exactly:
//   - the Top-K of the whole is the Top-K of the union of every shard's own Top-K;
//   - attention over the union of disjoint key sets follows from each set's normalised
//     output and log-sum-exp.
// Each rank scans and attends over its own shard with the ordinary calls; the kernels here
// are the glue around the two exchanges (which the caller performs, e.g. an NCCL
// all-gather): the visible count inside a shard, the merge of the gathered candidate
// lists (a selection over caller-built keys, run by the indexer's select kernel), the
// rank's own part of the merged list, and the log-sum-exp combine.
#include <cmath>
#include <cstdint>

#include "csa2_device.cuh"

namespace csa2 {

cudaError_t launch_select_labeled(const uint32_t* keys, const int32_t* labels, int64_t key_stride,
                                  int64_t n_items, int BQ, int K, int32_t* out_idx, float* out_score,
                                  cudaStream_t stream);

// n_vis_local[b][i] = clamp(n_vis[b][i] - lo[b], 0, len[b]).
__global__ void shard_vis_kernel(const int32_t* n_vis, const int64_t* lo, const int64_t* len, int Q,
                                 int64_t BQ, int32_t* out, uint32_t* status) {
  chain_enter();
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= BQ) return;
  const int64_t b = i / Q;
  const int64_t l = lo[b], n = len[b], v = n_vis[i];
  if (l < 0 || n < 0) {
    flag(status, CSA2_DEV_BAD_INDEX);
    out[i] = 0;
    return;
  }
  if (v < 0) flag(status, CSA2_DEV_BAD_COUNT);
  int64_t r = v - l;
  r = r < 0 ? 0 : (r > n ? n : r);
  out[i] = (int32_t)r;
}

// Selection keys and labels of the gathered candidates: row bq holds item c*Kc + j =
// candidate j of shard c (at c*part + bq*Kc + j of cand and score), key = order-preserving
// image of its score (0 = no candidate), label = shard_off[c][b] + cand.  Rows are `stride`
// items long; the pad past C*Kc gets key 0.
__global__ void merge_prep_kernel(const int32_t* cand, const float* score, int64_t part, const int64_t* shard_off,
                                  int C, int B, int Q, int Kc, int64_t stride, uint32_t* keys, int32_t* labels,
                                  uint32_t* status) {
  chain_enter();
  const int bq = blockIdx.y, b = bq / Q;
  const int64_t n = (int64_t)C * Kc;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < stride; i += (int64_t)gridDim.x * blockDim.x) {
    uint32_t key = 0u;
    int32_t lab = -1;
    if (i < n) {
      const int64_t c = i / Kc, j = i - c * Kc;
      const int64_t src = c * part + (int64_t)bq * Kc + j;
      const int32_t x = cand[src];
      if (x >= 0) {
        const int64_t off = shard_off[c * B + b];
        const int64_t g = off + x;
        if (off < 0 || g > INT32_MAX) {
          flag(status, CSA2_DEV_BAD_INDEX);
        } else {
          key = score_key(score[src]);
          lab = (int32_t)g;
        }
      } else if (x != -1) {
        flag(status, CSA2_DEV_BAD_INDEX);
      }
    }
    keys[bq * stride + i] = key;
    labels[bq * stride + i] = lab;
  }
}

// One warp per query row: the labels of `topk` inside [off[b], off[b] + len[b]), minus
// off[b], compacted to the front in slot order; -1 after them.
__global__ void localize_kernel(const int32_t* topk, int Q, int64_t BQ, int K, const int64_t* off,
                                const int64_t* len, int32_t* out, uint32_t* status) {
  chain_enter();
  const int64_t row = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (row >= BQ) return;
  const int64_t b = row / Q;
  const int64_t o = off[b], n = len[b];
  const bool ok = o >= 0 && n >= 0;
  if (!ok && lane == 0) flag(status, CSA2_DEV_BAD_INDEX);
  const int32_t* in = topk + row * K;
  int32_t* dst = out + row * K;
  int w = 0;
  for (int s0 = 0; s0 < K; s0 += 32) {
    const int s = s0 + lane;
    const int32_t x = s < K ? in[s] : -1;
    const int64_t rel = (int64_t)x - o;
    const bool keep = ok && x >= 0 && rel >= 0 && rel < n;
    const uint32_t m = __ballot_sync(0xffffffffu, keep);
    if (keep) dst[w + __popc(m & ((1u << lane) - 1u))] = (int32_t)rel;
    w += __popc(m);
  }
  for (int s = w + lane; s < K; s += 32) dst[s] = -1;
}

// One warp per output row r of N: with M = max_c lse_c, weights w_c = exp(lse_c - M),
// out = sum_c w_c out_c / sum_c w_c, lse = M + log(sum_c w_c).  Part c's row r is at
// out_parts + c*part_o + 512 r, its lse at lse_parts[c*part_l + r].  Lane l holds channels
// 4(l + 32k) .. +3, k < 4 (16-byte loads, consecutive lanes on consecutive addresses).
__global__ void combine_kernel(const float* out_parts, int64_t part_o, const float* lse_parts, int64_t part_l,
                               int C, int64_t N, float* out, float* lse) {
  chain_enter();
  const int64_t r = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (r >= N) return;
  float m = -INFINITY;
  for (int c = 0; c < C; ++c) m = fmaxf(m, lse_parts[(int64_t)c * part_l + r]);
  float4 acc[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) acc[k] = make_float4(0.f, 0.f, 0.f, 0.f);
  float4* o = reinterpret_cast<float4*>(out + r * kD);
  if (m == -INFINITY) {  // no part has a key
#pragma unroll
    for (int k = 0; k < 4; ++k) o[lane + 32 * k] = acc[k];
    if (lane == 0) lse[r] = -INFINITY;
    return;
  }
  float l = 0.f;
  for (int c = 0; c < C; ++c) {
    const float lc = lse_parts[(int64_t)c * part_l + r];
    if (lc == -INFINITY) continue;
    const float wc = expf(lc - m);
    l += wc;
    const float4* p = reinterpret_cast<const float4*>(out_parts + (int64_t)c * part_o + r * kD);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float4 v = p[lane + 32 * k];
      acc[k].x += wc * v.x;
      acc[k].y += wc * v.y;
      acc[k].z += wc * v.z;
      acc[k].w += wc * v.w;
    }
  }
  const float inv = 1.0f / l;
#pragma unroll
  for (int k = 0; k < 4; ++k)
    o[lane + 32 * k] = make_float4(acc[k].x * inv, acc[k].y * inv, acc[k].z * inv, acc[k].w * inv);
  if (lane == 0) lse[r] = m + logf(l);
}

// ---- host launchers ---------------------------------------------------------------------

cudaError_t launch_shard_vis(const int32_t* n_vis, const int64_t* lo, const int64_t* len, int B, int Q,
                             int32_t* out, uint32_t* status, cudaStream_t stream) {
  const int64_t BQ = (int64_t)B * Q;
  if (BQ == 0) return cudaSuccess;
  const unsigned blocks = (unsigned)((BQ + 255) / 256);
  cudaError_t e = launch_chained(shard_vis_kernel, dim3(blocks), dim3(256), 0, stream, 0, n_vis, lo, len, Q, BQ,
                                 out, status);
  return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t launch_topk_merge(const int32_t* cand, const float* score, int64_t part, const int64_t* shard_off,
                              int C, int B, int Q, int Kc, int K, int32_t* topk, float* topk_score, uint32_t* keys,
                              int32_t* labels, int64_t stride, uint32_t* status, cudaStream_t stream) {
  const int BQ = B * Q;
  if (BQ == 0) return cudaSuccess;
  const unsigned gx = (unsigned)((stride + 255) / 256 < 64 ? (stride + 255) / 256 : 64);
  cudaError_t e = launch_chained(merge_prep_kernel, dim3(gx, (unsigned)BQ), dim3(256), 0, stream, 0, cand, score,
                                 part, shard_off, C, B, Q, Kc, stride, keys, labels, status);
  if (e != cudaSuccess) return e;
  return launch_select_labeled(keys, labels, stride, (int64_t)C * Kc, BQ, K, topk, topk_score, stream);
}

cudaError_t launch_topk_localize(const int32_t* topk, int B, int Q, int K, const int64_t* off, const int64_t* len,
                                 int32_t* out, uint32_t* status, cudaStream_t stream) {
  const int64_t BQ = (int64_t)B * Q;
  if (BQ == 0) return cudaSuccess;
  const unsigned blocks = (unsigned)((BQ + 3) / 4);  // 4 warps (rows) per CTA
  cudaError_t e = launch_chained(localize_kernel, dim3(blocks), dim3(128), 0, stream, 0, topk, Q, BQ, K, off, len,
                                 out, status);
  return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t launch_attn_combine(const float* out_parts, int64_t part_o, const float* lse_parts, int64_t part_l,
                                int C, int64_t N, float* out, float* lse, cudaStream_t stream) {
  if (N == 0) return cudaSuccess;
  const unsigned blocks = (unsigned)((N + 7) / 8);  // 8 warps (rows) per CTA
  cudaError_t e = launch_chained(combine_kernel, dim3(blocks), dim3(256), 0, stream, 0, out_parts, part_o, lse_parts,
                                 part_l, C, N, out, lse);
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace csa2
