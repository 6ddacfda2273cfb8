// a6/a7: sparse MQA attention over Top-K FP4 entries plus the FP8 sliding window, on
// the sm_100a tensor cores (tcgen05.mma, accumulators in tensor memory).
//
// P1 (onedev.kr "KV 캐시를 토큰당 890바이트로…") §어떻게 동작하나 — every CSA2 layer has a
//   global branch and sliding-window attention; §무엇과 다른가 — Reuse layers inherit the
//   Top-K list and only attend.
// P3 (genexis.ai "100만 토큰을 0.9GB에…") §전역 어텐션과 지역 어텐션 — a 128-token window;
//   §4비트로 적어도 되는 이유 — the window is kept in 8 bits.
//
// A query's key slots are [0, K) for its Top-K entries, then [K, K+window) for window
// tokens t-window+1 .. t, cut into tiles of 128 slots.  One thread-block cluster of
// C = min(tiles, 8) CTAs (256 threads each) handles one query; CTA r takes tiles
// r, r+C, ...:
//   1. the fp32 queries arrive by one bulk copy into shared memory and become f16
//      (times sm_scale*log2 e, so the softmax works in base 2), heads padded with zero
//      rows up to the products' N; meanwhile each thread gathers its half of a selected
//      288 B entry;
//   2. the entries are dequantised into a 128 x 512 f16 tile in 128-byte-swizzled
//      shared memory (E2M1 -> f16 by cvt times the E4M3 block scale, exact in f16);
//      window tokens by E4M3 -> f16 cvt; empty slots become zero rows;
//   3. S^T[128 keys x N heads] = Kt . Qs^T by tcgen05.mma (M=128, K=512) into
//      tensor memory;
//   4. per-head max / exp2 / sum across the 128 TMEM lanes by warp transpose
//      reductions; a running max rescales the accumulated output when a CTA takes more
//      than one tile; P^T goes to shared memory as f16;
//   5. O^T[512 dims x heads] += Kt^T . P^T with the same key tile read MN-major as
//      the A operand (the latent is both key and value); both products take N = the
//      cluster's heads rounded up to 16, 32 or 64, P^T in rows of that width;
//   6. every CTA exports its O^T and (max, sum) per head in shared memory; after a
//      cluster barrier CTA r merges heads [r*H/C, (r+1)*H/C) of all CTAs through
//      distributed shared memory and writes the normalised output and log-sum-exp.
#include <cooperative_groups.h>
#include <cuda_fp16.h>

#include "csa2_device.cuh"
#include "tc.cuh"

namespace csa2 {

namespace cg = cooperative_groups;

constexpr int kTile = 128;        // key slots per tile = UMMA M
constexpr int kHeadsPad = 64;     // most heads per cluster (largest UMMA N used)
constexpr int kAttnThreads = 256;
constexpr int kMaxCluster = 8;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0, kColO = 256;
constexpr uint32_t kOffK = 0;           // keys: 8 dim-blocks x [128 rows x 128 B] f16; also the
                                        // fp32 query staging and the fp32 O export [64][512]
constexpr uint32_t kOffQ = 131072;      // queries: 8 dim-blocks x [64 rows x 128 B] f16
constexpr uint32_t kOffP = 196608;      // P^T: [128 keys x 64 heads] f16
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
  int n_tiles, csize;
  int hgroups, hg_size;  // a query's heads in hgroups groups of hg_size, one cluster each
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

// The same for 16 values: 4 exchange steps within each half-warp leave lane i with value
// i mod 16 reduced over its 16 lanes; one more exchange adds the other half-warp.
template <bool kMax>
__device__ __forceinline__ float xpose_reduce16(float (&v)[16], int lane) {
#pragma unroll
  for (int n = 8; n >= 1; n >>= 1) {
    const bool upper = (lane & n) != 0;
#pragma unroll
    for (int j = 0; j < n; ++j) {
      const float send = upper ? v[j] : v[j + n];
      const float keep = upper ? v[j + n] : v[j];
      const float recv = __shfl_xor_sync(0xffffffffu, send, n);
      v[j] = kMax ? fmaxf(keep, recv) : keep + recv;
    }
  }
  const float other = __shfl_xor_sync(0xffffffffu, v[0], 16);
  return kMax ? fmaxf(v[0], other) : v[0] + other;
}

// One key slot's raw data for this thread's half of the 512 channels.
struct SlotRaw {
  uint4 v[16];
  uint4 sc;
  int kind;  // 0 empty, 1 cached entry, 2 window token
};

// Entry index of Top-K slot `slot` (-1 for an empty slot or a window slot).
__device__ __forceinline__ int32_t slot_entry(const AttnArgs& a, int bq, int slot) {
  return slot < a.K ? a.topk[(int64_t)bq * a.K + slot] : -1;
}

// Issue the loads of this thread's half of key slot `slot`: j = slot_entry(...) and
// sws = swa_start[b] are passed in, so a caller can load them early.
__device__ __forceinline__ void gather_slot(const AttnArgs& a, int b, int64_t base, int64_t t, int slot, int hf,
                                            int32_t j, int64_t sws, SlotRaw& s) {
  s.kind = 0;
  if (slot < a.K) {
    if (j >= 0) {
      if (base >= 0 && base + j < a.pool_entries) {
        const uint4* e = reinterpret_cast<const uint4*>(a.kv_pool + (base + j) * kKvBytes);
#pragma unroll
        for (int i = 0; i < 8; ++i) s.v[i] = e[hf * 8 + i];
        s.sc = e[16 + hf];
        s.kind = 1;
      } else if (hf == 0) {
        flag(a.status, CSA2_DEV_BAD_INDEX);
      }
    }
  } else if (slot < a.K + a.window && a.S_w > 0) {
    const int64_t u = t - a.window + 1 + (slot - a.K);
    const int64_t row = u - sws;
    if (u >= 0 && row >= 0 && row < a.S_w) {
      const uint4* src = reinterpret_cast<const uint4*>(a.swa + ((int64_t)b * a.S_w + row) * kD + hf * 256);
#pragma unroll
      for (int i = 0; i < 16; ++i) s.v[i] = src[i];
      s.kind = 2;
    }
  }
}

// Dequantise this thread's half row (256 channels) of tile row r into the key tile.
__device__ __forceinline__ void store_slot(uint8_t* Ks, int r, int hf, const SlotRaw& s) {
  if (s.kind == 1) {
    const uint32_t scw[4] = {s.sc.x, s.sc.y, s.sc.z, s.sc.w};
#pragma unroll
    for (int dl = 0; dl < 4; ++dl) {
      uint8_t* blk = Ks + (4 * hf + dl) * 16384;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const uint4 q4 = s.v[2 * dl + (c >> 2)];
        const uint32_t wcode = (c & 3) == 0 ? q4.x : (c & 3) == 1 ? q4.y : (c & 3) == 2 ? q4.z : q4.w;
        const int sidx = dl * 4 + (c >> 1);  // block scale index within this half (0..15)
        const uint32_t sbyte = (scw[sidx >> 2] >> (8 * (sidx & 3))) & 0xFFu;
        *reinterpret_cast<uint4*>(blk + tc::sw128(r, c * 16)) = e2m1x8_to_f16(wcode, e4m3_scale_f16x2(sbyte));
      }
    }
  } else if (s.kind == 2) {
#pragma unroll
    for (int i = 0; i < 16; ++i) {  // 16 channels per load: chunks 2i, 2i+1 of this half
      const int ch = 2 * i;
      uint8_t* blk = Ks + (4 * hf + (ch >> 3)) * 16384;
      const uint2 a0 = e4m3x4_to_f16(s.v[i].x), a1 = e4m3x4_to_f16(s.v[i].y);
      const uint2 a2 = e4m3x4_to_f16(s.v[i].z), a3 = e4m3x4_to_f16(s.v[i].w);
      *reinterpret_cast<uint4*>(blk + tc::sw128(r, (ch & 7) * 16)) = make_uint4(a0.x, a0.y, a1.x, a1.y);
      *reinterpret_cast<uint4*>(blk + tc::sw128(r, ((ch + 1) & 7) * 16)) = make_uint4(a2.x, a2.y, a3.x, a3.y);
    }
  } else {
#pragma unroll
    for (int dl = 0; dl < 4; ++dl)
#pragma unroll
      for (int c = 0; c < 8; ++c)
        *reinterpret_cast<uint4*>(Ks + (4 * hf + dl) * 16384 + tc::sw128(r, c * 16)) = make_uint4(0u, 0u, 0u, 0u);
  }
}

__global__ void __launch_bounds__(kAttnThreads, 1) attn_tc_kernel(AttnArgs a) {
  chain_enter();
  // phase: started
  cg::cluster_group cluster = cg::this_cluster();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = tc::align_smem_1024(smem_raw);
  uint8_t* Ks = sm + kOffK;
  uint8_t* Qs = sm + kOffQ;
  uint8_t* Ps = sm + kOffP;
  float* red_max = reinterpret_cast<float*>(sm + kOffMisc);  // [4][64]
  float* red_sum = red_max + 256;                           // [4][64]
  float* m_run = red_sum + 256;                             // [64] running max (base-2 logits)
  float* l_run = m_run + 64;                                // [64] running sum
  float* alpha = l_run + 64;                                // [64] rescale of this tile
  int* valid_s = reinterpret_cast<int*>(alpha + 64);        // [128]
  uint64_t* mbar = reinterpret_cast<uint64_t*>(valid_s + 128);  // [0] MMA completion, [1] query copy
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mbar + 2);
  float* Of = reinterpret_cast<float*>(Ks);                 // export [64][512] fp32

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int rank = (int)cluster.block_rank();
  const int C = a.csize;
  const int bq = blockIdx.y / a.hgroups;
  const int b = bq / a.Q;
  const int H = a.H;                                 // heads of the query (output layout)
  const int h_base = (blockIdx.y % a.hgroups) * a.hg_size;
  const int NH = min(a.hg_size, H - h_base);         // heads of this cluster, rows 0..NH-1
  const int r = tid >> 1, hf = tid & 1;
  const int my_tiles = rank < a.n_tiles ? (a.n_tiles - 1 - rank) / C + 1 : 0;
  // every load the first gather depends on, issued together
  const int64_t base = a.seq_base[b];
  const int64_t t = a.q_pos[bq];
  const int32_t j0 = my_tiles > 0 ? slot_entry(a, bq, rank * kTile + r) : -1;
  const int64_t sws = a.S_w > 0 ? a.swa_start[b] : 0;
  const uint32_t mbar_mma = tc::smem_u32(&mbar[0]), mbar_q = tc::smem_u32(&mbar[1]);

  // Start every global read before any set-up barrier: thread 0 initialises the query
  // barrier and issues the bulk copy of the fp32 queries into the key area, every thread
  // gathers its half of its first key slot, then warp 0 allocates tensor memory.
  if (tid == 0) {
    tc::mbar_init(mbar_mma, 1);
    tc::mbar_init(mbar_q, 1);
    const uint32_t bytes = (uint32_t)NH * kD * 4;
    tc::mbar_arrive_expect_tx(mbar_q, bytes);
    const uint8_t* src = reinterpret_cast<const uint8_t*>(a.q + ((int64_t)bq * H + h_base) * kD);
    for (uint32_t off = 0; off < bytes; off += 32768)
      tc::bulk_g2s(tc::smem_u32(Ks) + off, src + off, bytes - off < 32768 ? bytes - off : 32768, mbar_q);
  }
  SlotRaw sr;
  sr.kind = 0;
  if (my_tiles > 0) gather_slot(a, b, base, t, rank * kTile + r, hf, j0, sws, sr);
  // phase: gather issued
  if (warp == 0) tc::tmem_alloc(tc::smem_u32(tmem_slot), kTmemCols);
  if (tid < kHeadsPad) {
    m_run[tid] = -INFINITY;
    l_run[tid] = 0.0f;
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  // phase: setup
  bool timed_out = __syncthreads_or(tc::mbar_wait(mbar_q, 0, kMaxPolls) ? 0 : 1) != 0;
  // phase: queries landed
  // The S product's N: this cluster's heads rounded up to 16, 32 or 64.  Query rows past NH
  // up to NQ are zero; rows past NQ are never read.
  const int NQ = NH <= 16 ? 16 : (NH <= 32 ? 32 : kHeadsPad);
  {  // fp32 staging -> f16 query tile (scaled), 8 channels per 16 B chunk
    const float qscale = a.sm_scale * 1.4426950408889634f;
#pragma unroll 4
    for (int i = tid; i < NQ * 64; i += kAttnThreads) {
      const int h = i >> 6, ch = i & 63, db = ch >> 3, c = ch & 7;
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (h < NH && !timed_out) {
        const float4 x0 = *reinterpret_cast<const float4*>(Of + h * kD + ch * 8);
        const float4 x1 = *reinterpret_cast<const float4*>(Of + h * kD + ch * 8 + 4);
        v.x = half2_bits(x0.x * qscale, x0.y * qscale);
        v.y = half2_bits(x0.z * qscale, x0.w * qscale);
        v.z = half2_bits(x1.x * qscale, x1.y * qscale);
        v.w = half2_bits(x1.z * qscale, x1.w * qscale);
      }
      *reinterpret_cast<uint4*>(Qs + db * 8192 + tc::sw128(h, c * 16)) = v;
    }
  }
  __syncthreads();  // staging consumed: the key area is free
  // phase: queries converted

  const int q4 = warp & 3, half = warp >> 2;
  const int key = q4 * 32 + lane;
  const uint32_t lane_base = tmem + ((uint32_t)(q4 * 32) << 16);
  uint32_t commits = 0;
  int processed = 0;
  for (int it = 0; it < my_tiles && !timed_out; ++it) {
    if (it > 0) {
      const int slot = (rank + it * C) * kTile + r;
      gather_slot(a, b, base, t, slot, hf, slot_entry(a, bq, slot), sws, sr);
    }
    store_slot(Ks, r, hf, sr);
    if (hf == 0) valid_s[r] = sr.kind != 0;
    tc::fence_async_smem();
    tc::fence_before_sync();
    const int any_valid = __syncthreads_or(sr.kind != 0);
    tc::fence_after_sync();
  // phase: keys stored
    if (!any_valid) continue;
    // ---- S^T = Kt . Qs^T --------------------------------------------------------------------
    if (tid == 0) {
      // N covers this cluster's heads only (rows past NH of the query tile are zero and the
      // softmax masks those columns)
      const uint32_t idesc = tc::idesc_f16(kTile, NQ, false, false);
#pragma unroll 4
      for (int ks = 0; ks < kD / 16; ++ks) {
        const int db = ks >> 2, kk = ks & 3;
        const uint64_t ad = tc::smem_desc_sw128(tc::smem_u32(Ks + db * 16384 + kk * 32), 16, 1024);
        const uint64_t bd = tc::smem_desc_sw128(tc::smem_u32(Qs + db * 8192 + kk * 32), 16, 1024);
        tc::mma_f16(tmem + kColS, ad, bd, idesc, ks > 0 ? 1u : 0u);
      }
      tc::commit(mbar_mma);
    }
    timed_out = __syncthreads_or(tc::mbar_wait(mbar_mma, commits & 1, kMaxPolls) ? 0 : 1) != 0;
    ++commits;
    tc::fence_after_sync();
    if (timed_out) break;
  // phase: qk done
    const bool kv = valid_s[key] != 0;
    float s[32], v[32];
    if (NQ == 16) {  // heads 0..15 only: warps 0-3 take them, warps 4-7 have no columns
      if (half == 0) {
        uint32_t raw[16];
        tc::tmem_ld16(lane_base + kColS, raw);
        float v16[16];
#pragma unroll
        for (int jj = 0; jj < 16; ++jj) {
          s[jj] = (kv && jj < NH) ? __uint_as_float(raw[jj]) : -INFINITY;
          v16[jj] = s[jj];
        }
        const float m16 = xpose_reduce16<true>(v16, lane);
        if (lane < 16) red_max[q4 * 64 + lane] = m16;
      }
    } else {
      uint32_t raw[32];
      tc::tmem_ld32(lane_base + kColS + half * 32, raw);
#pragma unroll
      for (int jj = 0; jj < 32; ++jj) {
        s[jj] = (kv && half * 32 + jj < NH) ? __uint_as_float(raw[jj]) : -INFINITY;  // pad heads: no keys
        v[jj] = s[jj];
      }
      red_max[q4 * 64 + half * 32 + lane] = xpose_reduce<true>(v, lane);
    }
    __syncthreads();
    if (tid < NQ) {
      const float mt = fmaxf(fmaxf(red_max[tid], red_max[64 + tid]), fmaxf(red_max[128 + tid], red_max[192 + tid]));
      const float mo = m_run[tid];
      const float mn = fmaxf(mo, mt);
      alpha[tid] = mo == -INFINITY ? 0.0f : exp2f(mo - mn);
      m_run[tid] = mn;
    }
    __syncthreads();
    if (processed > 0 && half * 32 < NQ) {  // rescale the output accumulated from earlier tiles
#pragma unroll 1
      for (int mt = 0; mt < 4; ++mt) {
        uint32_t o[32];
        const uint32_t ta = lane_base + kColO + mt * 64 + half * 32;
        tc::tmem_ld32(ta, o);
#pragma unroll
        for (int jj = 0; jj < 32; ++jj) o[jj] = __float_as_uint(__uint_as_float(o[jj]) * alpha[half * 32 + jj]);
        tc::tmem_st32(ta, o);
      }
    }
    if (NQ == 16) {
      if (half == 0) {
        uint32_t ph[8];
        float v16[16];
#pragma unroll
        for (int jj = 0; jj < 16; jj += 2) {
          const float m0 = m_run[jj], m1 = m_run[jj + 1];
          const float p0 = m0 == -INFINITY ? 0.0f : exp2f(s[jj] - m0);
          const float p1 = m1 == -INFINITY ? 0.0f : exp2f(s[jj + 1] - m1);
          __half2 hp = __floats2half2_rn(p0, p1);
          ph[jj >> 1] = *reinterpret_cast<uint32_t*>(&hp);
          const float2 back = __half22float2(hp);
          v16[jj] = back.x;  // the sum uses exactly the f16 values the PV product sees
          v16[jj + 1] = back.y;
        }
        // P^T rows of 16 heads (32 B, 32-byte swizzle)
        *reinterpret_cast<uint4*>(Ps + tc::swz(key, 0, 32)) = make_uint4(ph[0], ph[1], ph[2], ph[3]);
        *reinterpret_cast<uint4*>(Ps + tc::swz(key, 16, 32)) = make_uint4(ph[4], ph[5], ph[6], ph[7]);
        const float s16 = xpose_reduce16<false>(v16, lane);
        if (lane < 16) red_sum[q4 * 64 + lane] = s16;
      }
    } else {
      uint32_t ph[16];
#pragma unroll
      for (int jj = 0; jj < 32; jj += 2) {
        const float m0 = m_run[half * 32 + jj], m1 = m_run[half * 32 + jj + 1];
        const float p0 = m0 == -INFINITY ? 0.0f : exp2f(s[jj] - m0);
        const float p1 = m1 == -INFINITY ? 0.0f : exp2f(s[jj + 1] - m1);
        __half2 hp = __floats2half2_rn(p0, p1);
        ph[jj >> 1] = *reinterpret_cast<uint32_t*>(&hp);
        const float2 back = __half22float2(hp);
        v[jj] = back.x;  // the sum uses exactly the f16 values the PV product sees
        v[jj + 1] = back.y;
      }
      // P^T rows of NQ heads (NQ * 2 bytes, swizzle of that width); with NQ = 32 the upper
      // warps hold no heads of the product
      if (NQ == kHeadsPad) {
#pragma unroll
        for (int c = 0; c < 4; ++c)
          *reinterpret_cast<uint4*>(Ps + tc::swz(key, half * 64 + c * 16, 128)) =
              make_uint4(ph[4 * c], ph[4 * c + 1], ph[4 * c + 2], ph[4 * c + 3]);
      } else if (half == 0) {
#pragma unroll
        for (int c = 0; c < 4; ++c)
          *reinterpret_cast<uint4*>(Ps + tc::swz(key, c * 16, 64)) =
              make_uint4(ph[4 * c], ph[4 * c + 1], ph[4 * c + 2], ph[4 * c + 3]);
      }
      red_sum[q4 * 64 + half * 32 + lane] = xpose_reduce<false>(v, lane);
    }
  // phase: softmax done
    tc::fence_async_smem();
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    // ---- O^T += Kt^T . P^T (key tile read MN-major) --------------------------------------
    if (tid == 0) {
      // B = P^T [128 keys x NQ heads], MN-major, rows of rb = 2 NQ bytes: 8-row groups at
      // 8 rb, 16 keys (one K step) at 16 rb
      const uint32_t idesc = tc::idesc_f16(kTile, NQ, true, true);
      const uint32_t rb = 2u * (uint32_t)NQ, pcode = tc::swizzle_code(rb);
#pragma unroll 1
      for (int mt = 0; mt < 4; ++mt)
#pragma unroll 4
        for (int ks = 0; ks < kTile / 16; ++ks) {
          const uint64_t ad = tc::smem_desc_sw128(tc::smem_u32(Ks + (2 * mt) * 16384 + ks * 2048), 16384, 1024);
          const uint64_t bd = tc::smem_desc(tc::smem_u32(Ps + ks * 16 * rb), 64u * rb, 8u * rb, pcode);
          tc::mma_f16(tmem + kColO + mt * 64, ad, bd, idesc, (ks > 0 || processed > 0) ? 1u : 0u);
        }
      tc::commit(mbar_mma);
    }
    if (tid < NQ)
      l_run[tid] = l_run[tid] * alpha[tid] + ((red_sum[tid] + red_sum[64 + tid]) + (red_sum[128 + tid] + red_sum[192 + tid]));
    timed_out = __syncthreads_or(tc::mbar_wait(mbar_mma, commits & 1, kMaxPolls) ? 0 : 1) != 0;
    ++commits;
    tc::fence_after_sync();
    ++processed;
  // phase: pv done
  }
  if (timed_out) {
    if (tid == 0) flag(a.status, CSA2_DEV_TIMEOUT);
    if (tid < kHeadsPad) l_run[tid] = 0.0f;  // contribute nothing
  }

  // ---- export O^T (fp32 [head][channel]) into the key area --------------------------------
  // Items (dim block mt, column group g of cw heads) are shared by the two warp halves.
  if (processed > 0 && !timed_out) {
    const int cw = NQ == 16 ? 16 : 32;
    const int ngroups = (NH + cw - 1) / cw;
#pragma unroll 1
    for (int item = half; item < 4 * ngroups; item += 2) {
      const int mt = item / ngroups, g = item - mt * ngroups;
      const uint32_t ta = lane_base + kColO + mt * 64 + g * cw;
      const int d = mt * 128 + q4 * 32 + lane;
      if (cw == 16) {
        uint32_t o[16];
        tc::tmem_ld16(ta, o);
#pragma unroll
        for (int jj = 0; jj < 16; ++jj)
          if (jj < NH) Of[jj * kD + d] = __uint_as_float(o[jj]);
      } else {
        uint32_t o[32];
        tc::tmem_ld32(ta, o);
#pragma unroll
        for (int jj = 0; jj < 32; ++jj)
          if (g * 32 + jj < NH) Of[(g * 32 + jj) * kD + d] = __uint_as_float(o[jj]);
      }
    }
  }
  tc::fence_before_sync();
  cluster.sync();

  // phase: exported
  // ---- merge heads [h0, h1) across the cluster through distributed shared memory ----------
  // Remote loads are issued together (unrolled over the largest cluster), since each one
  // pays the cluster interconnect latency.
  const int hpc = (NH + C - 1) / C;
  const int h0 = rank * hpc, h1 = h0 + hpc < NH ? h0 + hpc : NH;  // this cluster's head rows
  // the P^T tile is free once the last PV product has completed
  float* fac = reinterpret_cast<float*>(Ps);  // [kMaxCluster][64] merge factor of each CTA's partial
  float* linv = fac + kMaxCluster * 64;       // [64] 1 / merged sum
  if (tid < h1 - h0) {
    const int hh = h0 + tid;
    float mr[kMaxCluster], lr[kMaxCluster];
#pragma unroll
    for (int c = 0; c < kMaxCluster; ++c) {
      mr[c] = c < C ? __uint_as_float(tc::ld_cluster_u32(tc::mapa(tc::smem_u32(m_run + hh), (uint32_t)c))) : -INFINITY;
      lr[c] = c < C ? __uint_as_float(tc::ld_cluster_u32(tc::mapa(tc::smem_u32(l_run + hh), (uint32_t)c))) : 0.0f;
    }
    float M = -INFINITY;
#pragma unroll
    for (int c = 0; c < kMaxCluster; ++c)
      if (lr[c] > 0.0f) M = fmaxf(M, mr[c]);
    float L = 0.0f;
#pragma unroll
    for (int c = 0; c < kMaxCluster; ++c) {
      const float f = (lr[c] > 0.0f) ? exp2f(mr[c] - M) : 0.0f;
      fac[c * 64 + tid] = f;
      L = fmaf(lr[c], f, L);
    }
    linv[tid] = L > 0.0f ? 1.0f / L : 0.0f;
    a.lse[(int64_t)bq * H + h_base + hh] = L > 0.0f ? (M + log2f(L)) * 0.69314718055994531f : -INFINITY;
  }
  __syncthreads();
  // thread -> (float4 column d4, heads hb, hb+2, hb+4, hb+6 per pass): every remote float4
  // of a pass is loaded before any is used, so a pass costs one interconnect round trip
  const int d4 = tid & 127;
  const int nh = h1 - h0;
  const uint32_t of_a = tc::smem_u32(Of);
  for (int hb = tid >> 7; hb < nh; hb += 8) {
    float4 o[4][kMaxCluster];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int hl = hb + 2 * u;
#pragma unroll
      for (int c = 0; c < kMaxCluster; ++c)
        o[u][c] = (hl < nh && c < C && fac[c * 64 + hl] > 0.0f)
                      ? tc::ld_cluster_f32x4(tc::mapa(of_a + (uint32_t)(((h0 + hl) * kD + 4 * d4) * 4), (uint32_t)c))
                      : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int hl = hb + 2 * u;
      if (hl < nh) {
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int c = 0; c < kMaxCluster; ++c) {
          const float f = c < C ? fac[c * 64 + hl] : 0.0f;
          acc.x = fmaf(o[u][c].x, f, acc.x);
          acc.y = fmaf(o[u][c].y, f, acc.y);
          acc.z = fmaf(o[u][c].z, f, acc.z);
          acc.w = fmaf(o[u][c].w, f, acc.w);
        }
        const float inv = linv[hl];
        reinterpret_cast<float4*>(a.out + ((int64_t)bq * H + h_base + h0 + hl) * kD)[d4] =
            make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
      }
    }
  }
  cluster.sync();  // remote reads finished before any CTA releases its shared memory
  // phase: merged
  if (warp == 0) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, kTmemCols);
  }
}

size_t attn_workspace_bytes(int B, int Q, int H, int K, int window) {
  (void)B;
  (void)Q;
  (void)H;
  (void)K;
  (void)window;
  return 0;  // partial results stay in distributed shared memory
}

cudaError_t launch_sparse_attn(const float* q, const uint8_t* kv_pool, int64_t pool_entries,
                               const int64_t* seq_base, const int32_t* topk, int K,
                               const uint8_t* swa, int S_w, const int64_t* swa_start,
                               const int64_t* q_pos, int window, int B, int Q, int H,
                               float sm_scale, float* out, float* lse, void* ws,
                               uint32_t* status, cudaStream_t stream) {
  (void)ws;
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
  a.n_tiles = (K + a.window + kTile - 1) / kTile;
  a.out = out;
  a.lse = lse;
  a.status = status;
  const int64_t BQ = (int64_t)B * Q;
  if (BQ == 0) return cudaSuccess;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // Key split: the C CTAs of a query's cluster take its tiles round-robin.  Few queries want
  // a wide split (more SMs at work), many queries want none (no merge, fewer waves).  C
  // minimises waves x (set-up + tiles per CTA x per-tile time + merge when split), with one
  // CTA per SM and costs in microseconds measured on the kernel's phases.
  {
    constexpr double kSetup = 5.0, kPerTile = 7.0, kMerge = 5.0;
    const int cmax = a.n_tiles < 1 ? 1 : (a.n_tiles > kMaxCluster ? kMaxCluster : a.n_tiles);
    double best = 0.0;
    a.csize = 1;
    for (int c = 1; c <= cmax; ++c) {
      const double waves = (double)((BQ * c + sms - 1) / sms);
      const double per_cta = kSetup + (double)((a.n_tiles + c - 1) / c) * kPerTile + (c > 1 ? kMerge : 0.0);
      if (c == 1 || waves * per_cta < best) {
        best = waves * per_cta;
        a.csize = c;
      }
    }
  }
  // When the clusters do not fill the GPU, split each query's heads into groups of 16 or 32,
  // one cluster per group: a CTA then converts, exports and merges only its group's heads.
  a.hgroups = 1;
  for (int g = 4; g >= 2; g >>= 1)
    if (H % (16 * g) == 0 && BQ * a.csize * g <= sms) {
      a.hgroups = g;
      break;
    }
  a.hg_size = H / a.hgroups;
  cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
  if (e != cudaSuccess) return e;
  e = launch_chained(attn_tc_kernel, dim3((unsigned)a.csize, (unsigned)(BQ * a.hgroups)), dim3(kAttnThreads), kSmemBytes, stream,
                     (unsigned)a.csize, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace csa2
