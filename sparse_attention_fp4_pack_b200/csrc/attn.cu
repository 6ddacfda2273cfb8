// a6/a7: sparse MQA attention over Top-K FP4 entries plus the FP8 sliding window, on
// the sm_100a tensor cores (tcgen05.mma, accumulators in tensor memory).
//
// P1 (onedev.kr "KV 캐시를 토큰당 890바이트로…") §어떻게 동작하나 — every CSA2 layer has a
//   global branch and sliding-window attention; §무엇과 다른가 — Reuse layers inherit the
//   Top-K list and only attend.
// P3 (genexis.ai "100만 토큰을 0.9GB에…") §전역 어텐션과 지역 어텐션 — a 128-token window;
//   §4비트로 적어도 되는 이유 — the window is kept in 8 bits.
//
// Split-KV.  A query's key slots are [0, K) for its Top-K entries, then [K, K+window)
// for window tokens t-window+1 .. t.  One CTA (256 threads) owns 128 consecutive slots:
//   1. gathers the selected 288 B entries (16 B loads) and dequantises them into a
//      128 x 512 f16 tile in shared memory (E2M1 -> f16 by cvt, times the E4M3 block
//      scale; every product is exact in f16), window tokens by E4M3 -> f16 cvt;
//      empty slots become zero rows;
//   2. S^T[128 keys x 64 heads] = Kt . Qs^T with tcgen05.mma (M=128, N=64, K=512),
//      queries pre-scaled by sm_scale*log2(e) so the softmax works in base 2;
//   3. per-head max / exp2 / sum across the 128 TMEM lanes (warp transpose-reductions),
//      P^T written to shared memory as f16;
//   4. O^T[512 dims x 64 heads] = Kt^T . P^T: the same key tile read MN-major as the A
//      operand (4 MMAs of M=128 per K step) — the latent is both key and value;
//   5. unnormalised O^T and (m, l) per head go to the workspace; a combine kernel merges
//      the splits by their log-sum-exp.
// Heads are padded to 64 (zero query rows) so every MMA has N = 64.
#include <cuda_fp16.h>

#include "csa2_device.cuh"
#include "tc.cuh"

namespace csa2 {

constexpr int kTile = 128;        // key slots per CTA = UMMA M
constexpr int kHeadsPad = 64;     // UMMA N
constexpr int kAttnThreads = 256;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0, kColO = 256;
constexpr uint32_t kOffK = 0;           // 8 dim-blocks x [128 rows x 128 B]
constexpr uint32_t kOffQ = 131072;      // 8 dim-blocks x [64 rows x 128 B]
constexpr uint32_t kOffP = 196608;      // [128 keys x 64 heads] f16
constexpr uint32_t kOffMisc = 212992;
constexpr uint32_t kSmemBytes = kOffMisc + 4096 + 1024;  // + alignment slack
constexpr uint32_t kMaxPolls = 1u << 22;

struct AttnArgs {
  const float* q;
  const uint8_t* kv_pool;
  int64_t pool_entries;
  const int64_t* seq_base;
  const int32_t* topk;
  int K;
  const uint8_t* swa;
  int S_w;
  const int64_t* swa_start;
  const int64_t* q_pos;
  int window;
  int Q, H;
  float sm_scale;
  int n_splits;
  float* part_o;   // [BQ][n_splits][H][512] unnormalised
  float* part_ml;  // [BQ][n_splits][H][2]  (max in base-2 logit units, sum)
  float* out;
  float* lse;
  uint32_t* status;
};

__device__ __forceinline__ uint32_t half2_bits(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// 8 E2M1 codes (one 32-bit word, code i in bits 4i..4i+3) times an f16x2 scale -> 8 f16.
__device__ __forceinline__ uint4 e2m1x8_to_f16(uint32_t w, uint32_t scale2) {
  uint32_t h0, h1, h2, h3;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
      "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
      "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
      : "=r"(h0), "=r"(h1), "=r"(h2), "=r"(h3)
      : "r"(w));
  uint4 o;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(o.x) : "r"(h0), "r"(scale2));
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(o.y) : "r"(h1), "r"(scale2));
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(o.z) : "r"(h2), "r"(scale2));
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(o.w) : "r"(h3), "r"(scale2));
  return o;
}

// 4 E4M3 bytes (one word) -> 4 f16 (two f16x2 words).
__device__ __forceinline__ uint2 e4m3x4_to_f16(uint32_t w) {
  uint2 o;
  asm("{\n\t.reg .b16 lo, hi;\n\t"
      "mov.b32 {lo, hi}, %2;\n\t"
      "cvt.rn.f16x2.e4m3x2 %0, lo;\n\t"
      "cvt.rn.f16x2.e4m3x2 %1, hi;\n\t}"
      : "=r"(o.x), "=r"(o.y)
      : "r"(w));
  return o;
}

// E4M3 scale byte -> f16x2 with the value in both halves.
__device__ __forceinline__ uint32_t e4m3_scale_f16x2(uint32_t byte) {
  uint32_t h;
  const uint16_t pair = (uint16_t)(byte | (byte << 8));
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"(pair));
  return h;
}

// Reduce 32 values per lane across the warp so that lane i ends with the reduction of
// value i over all 32 lanes (5 halving exchange steps, 31 shuffles).
template <bool kMax>
__device__ __forceinline__ float xpose_reduce(float (&v)[32], int lane) {
#pragma unroll
  for (int n = 16; n >= 1; n >>= 1) {
    const bool upper = (lane & n) != 0;
#pragma unroll
    for (int j = 0; j < n; ++j) {
      const float send = upper ? v[j] : v[j + n];
      const float keep = upper ? v[j + n] : v[j];
      const float recv = __shfl_xor_sync(0xffffffffu, send, n);
      v[j] = kMax ? fmaxf(keep, recv) : keep + recv;
    }
  }
  return v[0];
}

__global__ void __launch_bounds__(kAttnThreads, 1) attn_tc_kernel(AttnArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* Ks = sm + kOffK;
  uint8_t* Qs = sm + kOffQ;
  uint8_t* Ps = sm + kOffP;
  float* red_max = reinterpret_cast<float*>(sm + kOffMisc);  // [4][64]
  float* red_sum = red_max + 256;                           // [4][64]
  float* m_s = red_sum + 256;                               // [64]
  float* l_s = m_s + 64;                                    // [64]
  int* valid_s = reinterpret_cast<int*>(l_s + 64);          // [128]
  uint64_t* mbar = reinterpret_cast<uint64_t*>(valid_s + 128);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mbar + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bq = blockIdx.y, split = blockIdx.x;
  const int b = bq / a.Q;
  const int H = a.H;
  const int64_t base = a.seq_base[b];
  const int64_t t = a.q_pos[bq];
  const uint32_t mbar_a = tc::smem_u32(mbar);

  if (warp == 0) tc::tmem_alloc(tc::smem_u32(tmem_slot), kTmemCols);
  if (tid == 32) tc::mbar_init(mbar_a, 1);

  // Issue the key gather first so its latency overlaps the query loads.
  const int r = tid >> 1, hf = tid & 1;
  const int slot = split * kTile + r;
  int kind = 0;  // 0 empty, 1 cached entry, 2 window token
  uint4 kraw[16];
  uint4 ksc = make_uint4(0u, 0u, 0u, 0u);
  if (slot < a.K) {
    const int32_t j = a.topk[(int64_t)bq * a.K + slot];
    if (j >= 0) {
      if (base >= 0 && base + j < a.pool_entries) {
        const uint4* e = reinterpret_cast<const uint4*>(a.kv_pool + (base + j) * kKvBytes);
#pragma unroll
        for (int i = 0; i < 8; ++i) kraw[i] = e[hf * 8 + i];
        ksc = e[16 + hf];
        kind = 1;
      } else if (hf == 0) {
        flag(a.status, CSA2_DEV_BAD_INDEX);
      }
    }
  } else if (slot < a.K + a.window && a.S_w > 0) {
    const int64_t u = t - a.window + 1 + (slot - a.K);
    const int64_t row = u - a.swa_start[b];
    if (u >= 0 && row >= 0 && row < a.S_w) {
      const uint4* src = reinterpret_cast<const uint4*>(a.swa + ((int64_t)b * a.S_w + row) * kD + hf * 256);
#pragma unroll
      for (int i = 0; i < 16; ++i) kraw[i] = src[i];
      kind = 2;
    }
  }

  // ---- queries: f16(q * sm_scale * log2 e), rows >= H are zero ---------------------------
  // thread -> (head row tid/4, quarter tid%4 = 128 channels), two batches of 16 x 16 B
  const float qscale = a.sm_scale * 1.4426950408889634f;
  {
    const int h = tid >> 2, qq = tid & 3;
    const float4* src = reinterpret_cast<const float4*>(a.q + ((int64_t)bq * H + h) * kD + qq * 128);
#pragma unroll
    for (int bt = 0; bt < 2; ++bt) {
      float4 x[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) x[i] = h < H ? src[bt * 16 + i] : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int i = 0; i < 8; ++i) {  // 8 chunks of 8 channels
        const float4 x0 = x[2 * i], x1 = x[2 * i + 1];
        uint4 v;
        v.x = half2_bits(x0.x * qscale, x0.y * qscale);
        v.y = half2_bits(x0.z * qscale, x0.w * qscale);
        v.z = half2_bits(x1.x * qscale, x1.y * qscale);
        v.w = half2_bits(x1.z * qscale, x1.w * qscale);
        const int ch = qq * 16 + bt * 8 + i, db = ch >> 3, c = ch & 7;
        *reinterpret_cast<uint4*>(Qs + db * 8192 + tc::sw128(h, c * 16)) = v;
      }
    }
  }

  // ---- keys: two threads per slot, each dequantises 256 of the 512 channels -------------
  const bool ok = kind != 0;
  if (kind == 1) {
    const uint32_t scw[4] = {ksc.x, ksc.y, ksc.z, ksc.w};
#pragma unroll
    for (int dl = 0; dl < 4; ++dl) {
      uint8_t* blk = Ks + (4 * hf + dl) * 16384;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const uint4 q4 = kraw[2 * dl + (c >> 2)];
        const uint32_t wcode = (c & 3) == 0 ? q4.x : (c & 3) == 1 ? q4.y : (c & 3) == 2 ? q4.z : q4.w;
        const int sidx = dl * 4 + (c >> 1);  // block scale index within this half (0..15)
        const uint32_t sbyte = (scw[sidx >> 2] >> (8 * (sidx & 3))) & 0xFFu;
        *reinterpret_cast<uint4*>(blk + tc::sw128(r, c * 16)) = e2m1x8_to_f16(wcode, e4m3_scale_f16x2(sbyte));
      }
    }
  } else if (kind == 2) {
#pragma unroll
    for (int i = 0; i < 16; ++i) {  // 16 channels per load: chunks 2i, 2i+1 of this half
      const int ch = 2 * i;         // chunk of 8 channels within this half's 32 chunks
      uint8_t* blk = Ks + (4 * hf + (ch >> 3)) * 16384;
      const uint2 a0 = e4m3x4_to_f16(kraw[i].x), a1 = e4m3x4_to_f16(kraw[i].y);
      const uint2 a2 = e4m3x4_to_f16(kraw[i].z), a3 = e4m3x4_to_f16(kraw[i].w);
      *reinterpret_cast<uint4*>(blk + tc::sw128(r, (ch & 7) * 16)) = make_uint4(a0.x, a0.y, a1.x, a1.y);
      *reinterpret_cast<uint4*>(blk + tc::sw128(r, ((ch + 1) & 7) * 16)) = make_uint4(a2.x, a2.y, a3.x, a3.y);
    }
  }
  if (!ok) {
#pragma unroll
    for (int dl = 0; dl < 4; ++dl)
#pragma unroll
      for (int c = 0; c < 8; ++c)
        *reinterpret_cast<uint4*>(Ks + (4 * hf + dl) * 16384 + tc::sw128(r, c * 16)) = make_uint4(0u, 0u, 0u, 0u);
  }
  if (hf == 0) valid_s[r] = ok ? 1 : 0;

  tc::fence_async_smem();
  tc::fence_before_sync();
  const int any_valid = __syncthreads_or(ok ? 1 : 0);
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  const int64_t pbase = ((int64_t)bq * a.n_splits + split) * H;

  bool timed_out = false;
  if (any_valid) {
    // ---- S^T = Kt . Qs^T ----------------------------------------------------------------
    if (tid == 0) {
      constexpr uint32_t idesc = tc::idesc_f16(kTile, kHeadsPad, false, false);
#pragma unroll 1
      for (int ks = 0; ks < kD / 16; ++ks) {
        const int db = ks >> 2, kk = ks & 3;
        const uint64_t ad = tc::smem_desc_sw128(tc::smem_u32(Ks + db * 16384 + kk * 32), 16, 1024);
        const uint64_t bd = tc::smem_desc_sw128(tc::smem_u32(Qs + db * 8192 + kk * 32), 16, 1024);
        tc::mma_f16(tmem + kColS, ad, bd, idesc, ks > 0 ? 1u : 0u);
      }
      tc::commit(mbar_a);
    }
    timed_out = __syncthreads_or(tc::mbar_wait(mbar_a, 0, kMaxPolls) ? 0 : 1) != 0;
    tc::fence_after_sync();
  }
  if (any_valid && !timed_out) {
    const int q4 = warp & 3, half = warp >> 2;
    const int key = q4 * 32 + lane;
    uint32_t raw[32];
    tc::tmem_ld32(tmem + ((uint32_t)(q4 * 32) << 16) + kColS + half * 32, raw);
    const bool kv = valid_s[key] != 0;
    float s[32], v[32];
#pragma unroll
    for (int jj = 0; jj < 32; ++jj) {
      s[jj] = kv ? __uint_as_float(raw[jj]) : -INFINITY;
      v[jj] = s[jj];
    }
    red_max[q4 * 64 + half * 32 + lane] = xpose_reduce<true>(v, lane);
    __syncthreads();
    if (tid < kHeadsPad)
      m_s[tid] = fmaxf(fmaxf(red_max[tid], red_max[64 + tid]), fmaxf(red_max[128 + tid], red_max[192 + tid]));
    __syncthreads();
    uint32_t ph[16];
#pragma unroll
    for (int jj = 0; jj < 32; jj += 2) {
      const float m0 = m_s[half * 32 + jj], m1 = m_s[half * 32 + jj + 1];
      const float p0 = m0 == -INFINITY ? 0.0f : exp2f(s[jj] - m0);
      const float p1 = m1 == -INFINITY ? 0.0f : exp2f(s[jj + 1] - m1);
      __half2 hp = __floats2half2_rn(p0, p1);
      ph[jj >> 1] = *reinterpret_cast<uint32_t*>(&hp);
      const float2 back = __half22float2(hp);
      v[jj] = back.x;  // the sum uses exactly the f16 values the PV product sees
      v[jj + 1] = back.y;
    }
#pragma unroll
    for (int c = 0; c < 4; ++c)
      *reinterpret_cast<uint4*>(Ps + tc::sw128(key, half * 64 + c * 16)) =
          make_uint4(ph[4 * c], ph[4 * c + 1], ph[4 * c + 2], ph[4 * c + 3]);
    red_sum[q4 * 64 + half * 32 + lane] = xpose_reduce<false>(v, lane);
    tc::fence_async_smem();
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    // ---- O^T = Kt^T . P^T (key tile read MN-major) ---------------------------------------
    if (tid == 0) {
      constexpr uint32_t idesc = tc::idesc_f16(kTile, kHeadsPad, true, true);
#pragma unroll 1
      for (int mt = 0; mt < 4; ++mt)
#pragma unroll 1
        for (int ks = 0; ks < kTile / 16; ++ks) {
          const uint64_t ad = tc::smem_desc_sw128(tc::smem_u32(Ks + (2 * mt) * 16384 + ks * 2048), 16384, 1024);
          const uint64_t bd = tc::smem_desc_sw128(tc::smem_u32(Ps + ks * 2048), 8192, 1024);
          tc::mma_f16(tmem + kColO + mt * 64, ad, bd, idesc, ks > 0 ? 1u : 0u);
        }
      tc::commit(mbar_a);
    }
    if (tid < kHeadsPad)
      l_s[tid] = (red_sum[tid] + red_sum[64 + tid]) + (red_sum[128 + tid] + red_sum[192 + tid]);
    timed_out = __syncthreads_or(tc::mbar_wait(mbar_a, 1, kMaxPolls) ? 0 : 1) != 0;
    tc::fence_after_sync();
    if (!timed_out) {
#pragma unroll 1
      for (int mt = 0; mt < 4; ++mt) {
        tc::tmem_ld32(tmem + ((uint32_t)(q4 * 32) << 16) + kColO + mt * 64 + half * 32, raw);
        const int d = mt * 128 + q4 * 32 + lane;
#pragma unroll
        for (int jj = 0; jj < 32; ++jj) {
          const int h = half * 32 + jj;
          if (h < H) a.part_o[(pbase + h) * kD + d] = __uint_as_float(raw[jj]);
        }
      }
      if (tid < H) {
        a.part_ml[(pbase + tid) * 2] = m_s[tid];
        a.part_ml[(pbase + tid) * 2 + 1] = l_s[tid];
      }
    }
  }
  if (!any_valid && tid < H) {
    a.part_ml[(pbase + tid) * 2] = -INFINITY;
    a.part_ml[(pbase + tid) * 2 + 1] = 0.0f;
  }
  if (timed_out) {
    if (tid == 0) flag(a.status, CSA2_DEV_TIMEOUT);
    if (tid < H) a.part_ml[(pbase + tid) * 2 + 1] = 0.0f;
    tc::mbar_wait(mbar_a, 1, kMaxPolls);  // let any MMA still in flight drain (bounded)
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, kTmemCols);
  }
}

// Merge the split partials of one query: grid (H, BQ), one thread per channel.
__global__ void __launch_bounds__(kD) attn_combine_kernel(AttnArgs a) {
  const int h = blockIdx.x, bq = blockIdx.y, c = threadIdx.x;
  const int H = a.H;
  float M = -INFINITY;
  for (int s = 0; s < a.n_splits; ++s) {
    const int64_t p = ((int64_t)bq * a.n_splits + s) * H + h;
    if (a.part_ml[p * 2 + 1] > 0.0f) M = fmaxf(M, a.part_ml[p * 2]);
  }
  float L = 0.0f, o = 0.0f;
  if (M != -INFINITY) {
    for (int s = 0; s < a.n_splits; ++s) {
      const int64_t p = ((int64_t)bq * a.n_splits + s) * H + h;
      const float l = a.part_ml[p * 2 + 1];
      if (l > 0.0f) {
        const float f = exp2f(a.part_ml[p * 2] - M);
        L = fmaf(l, f, L);
        o = fmaf(a.part_o[p * kD + c], f, o);
      }
    }
  }
  const int64_t oi = ((int64_t)bq * H + h);
  a.out[oi * kD + c] = L > 0.0f ? o / L : 0.0f;
  if (c == 0) a.lse[oi] = L > 0.0f ? (M + log2f(L)) * 0.69314718055994531f : -INFINITY;
}

size_t attn_workspace_bytes(int B, int Q, int H, int K, int window) {
  const int64_t n_splits = (K + window + kTile - 1) / kTile;
  const int64_t BQ = (int64_t)B * Q;
  return (size_t)(BQ * n_splits * H * (kD + 2) * sizeof(float));
}

cudaError_t launch_sparse_attn(const float* q, const uint8_t* kv_pool, int64_t pool_entries,
                               const int64_t* seq_base, const int32_t* topk, int K,
                               const uint8_t* swa, int S_w, const int64_t* swa_start,
                               const int64_t* q_pos, int window, int B, int Q, int H,
                               float sm_scale, float* out, float* lse, void* ws,
                               uint32_t* status, cudaStream_t stream) {
  AttnArgs a;
  a.q = q;
  a.kv_pool = kv_pool;
  a.pool_entries = pool_entries;
  a.seq_base = seq_base;
  a.topk = topk;
  a.K = K;
  a.swa = swa;
  a.S_w = S_w;
  a.swa_start = swa_start;
  a.q_pos = q_pos;
  a.window = S_w > 0 ? window : 0;
  a.Q = Q;
  a.H = H;
  a.sm_scale = sm_scale;
  a.n_splits = (K + a.window + kTile - 1) / kTile;
  const int64_t BQ = (int64_t)B * Q;
  a.part_o = static_cast<float*>(ws);
  a.part_ml = a.part_o + BQ * a.n_splits * H * kD;
  a.out = out;
  a.lse = lse;
  a.status = status;
  if (BQ == 0) return cudaSuccess;
  if (a.n_splits > 0) {
    cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kSmemBytes);
    if (e != cudaSuccess) return e;
    attn_tc_kernel<<<dim3(a.n_splits, (unsigned)BQ), kAttnThreads, kSmemBytes, stream>>>(a);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  attn_combine_kernel<<<dim3(H, (unsigned)BQ), kD, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace csa2
