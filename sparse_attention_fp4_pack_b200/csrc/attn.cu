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
// tokens t-window+1 .. t, cut into tiles of 128 slots.  A thread-block cluster of C CTAs
// takes one query and a group of its heads (all heads share the key set: MQA); CTA r of
// the cluster walks tiles r, r+C, ... .  Its 8 warps gather, dequantise and run the
// softmax; thread 0 also issues the tensor-core products, each once every thread has
// arrived on the mbarrier that guards its operands:
//   * the fp32 queries arrive by bulk copy and become f16 (times sm_scale*log2 e, so the
//     softmax works in base 2), heads padded with zero rows up to the products' N;
//   * each worker owns half a tile row: it gathers the row's entry (or window token)
//     into registers (prefetched into L2 one tile ahead, gathered while the previous
//     tile's PV product runs) and dequantises it into the 128 x 512 f16 key tile
//     (128-byte swizzle, 8 blocks of 64 dims; E2M1 x E4M3 block scale and E4M3 window
//     values are exact in f16) in two halves of 256 dims;
//   * S^T[128 keys x N heads] = Kt . Qs^T is accumulated in four partial sums (dim-block
//     d into sum d mod 4), so four independent chains of products run interleaved, and
//     it starts on the first half of the dims while the second is still being written;
//   * the softmax reads the four partial sums from tensor memory (lanes = keys), reduces
//     per head across lanes, writes P^T (f16) to shared memory and keeps a per-head
//     running max and sum;
//   * O^T[512 dims x N heads] += Kt^T . P^T reads the same key tile MN-major (the latent
//     is both key and value) as four 128-dim M-tiles issued interleaved; the next tile's
//     dequantisation starts as soon as they have completed;
//   * the running max is raised only when a tile's max exceeds it by more than 8 (base
//     2): probabilities stay below 2^8, exact enough in f16, and the accumulated output
//     is rescaled in tensor memory only on those tiles;
//   * a CTA alone (C = 1) divides its rows of O^T by the heads' sums and writes them out
//     (consecutive lanes = consecutive channels).  In a cluster, once every CTA has
//     finished its products, each one writes its partial O^T, max and sum for the heads
//     of CTA o into CTA o's shared memory (distributed shared memory stores); after a
//     second cluster barrier CTA o merges its heads from local shared memory.
#include <cuda_fp16.h>

#include "csa2_device.cuh"
#include "tc.cuh"

namespace csa2 {

constexpr int kTile = 128;        // key slots per tile = UMMA M
constexpr int kHeadsPad = 64;     // most heads per CTA (largest UMMA N used)
constexpr int kWorkers = 256;     // two threads per tile row
constexpr int kAttnThreads = kWorkers;
constexpr uint32_t kTmemCols = 512;
constexpr int kMaxCluster = 8;
constexpr int kWorkerBar = 1;     // named barrier of all 256 threads (0 is __syncthreads)
constexpr uint32_t kColS = 0;     // S^T partial sum i at kColS + 64 i, NQ columns each
constexpr uint32_t kColO = 256;   // O^T M-tile mt at kColO + 64 mt, NQ columns each
constexpr uint32_t kOffK = 0;           // keys: 8 dim-blocks x [128 rows x 128 B] f16; also the
                                        // fp32 query staging [NH][512] at the start
constexpr uint32_t kOffQ = 131072;      // queries: 8 dim-blocks x [64 rows x 128 B] f16
constexpr uint32_t kOffP = 196608;      // P^T: [128 keys x NQ heads] f16
constexpr uint32_t kOffMisc = 212992;   // reductions, running stats, flags, barriers
constexpr uint32_t kOffIdx = kOffMisc + 4096;            // Top-K entry index per slot
constexpr uint32_t kOffRecv = 0;        // merge: partial O^T received from the cluster,
                                        // [C][512][hpc] fp32 over the key and query tiles
constexpr uint32_t kSmemBytes = kOffIdx + CSA2_MAX_K * 4 + 1024;  // + alignment slack
constexpr uint32_t kMaxPolls = 1u << 22;
constexpr float kStaleMax = 8.0f;       // raise the running max only beyond this margin

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
  int n_tiles, csize;    // key tiles per query; CTAs per cluster (key split)
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
  const uint4 h = e2m1x8_f16(w);
  uint4 o;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(o.x) : "r"(h.x), "r"(scale2));
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(o.y) : "r"(h.y), "r"(scale2));
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(o.z) : "r"(h.z), "r"(scale2));
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(o.w) : "r"(h.w), "r"(scale2));
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

// The same for 8 values per lane: 3 exchange steps within each group of 8 lanes leave lane i
// with value i mod 8 reduced over its 8 lanes; two more exchanges add the other groups.
template <bool kMax>
__device__ __forceinline__ float xpose_reduce8(float (&v)[8], int lane) {
#pragma unroll
  for (int n = 4; n >= 1; n >>= 1) {
    const bool upper = (lane & n) != 0;
#pragma unroll
    for (int j = 0; j < n; ++j) {
      const float send = upper ? v[j] : v[j + n];
      const float keep = upper ? v[j + n] : v[j];
      const float recv = __shfl_xor_sync(0xffffffffu, send, n);
      v[j] = kMax ? fmaxf(keep, recv) : keep + recv;
    }
  }
  float x = v[0];
#pragma unroll
  for (int o = 8; o <= 16; o <<= 1) {
    const float other = __shfl_xor_sync(0xffffffffu, x, o);
    x = kMax ? fmaxf(x, other) : x + other;
  }
  return x;
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

// One key slot's raw data for this thread's half of the 512 channels: dim-blocks
// d_i = 2i + hf (i = 0..3) of 64 channels.  Entry: codes of block d_i in v[2i], v[2i+1]
// and its four E4M3 scales in sc[i]; window token: block d_i's 64 bytes in v[4i..4i+3].
struct SlotRaw {
  uint4 v[16];
  uint32_t sc[4];
  int kind;  // 0 empty, 1 cached entry, 2 window token
};

// Issue the loads of this thread's half of key slot `slot` (j = its Top-K entry index,
// read by the caller; sws = swa_start[b]).
__device__ __forceinline__ void gather_slot(const AttnArgs& a, int b, int64_t base, int64_t t, int slot, int hf,
                                            int32_t j, int64_t sws, SlotRaw& s) {
  s.kind = 0;
  if (slot < a.K) {
    if (j >= 0) {
      if (base >= 0 && base + j < a.pool_entries) {
        const uint8_t* e = a.kv_pool + (base + j) * kKvBytes;
        const uint4* e4 = reinterpret_cast<const uint4*>(e);
        const uint32_t* es = reinterpret_cast<const uint32_t*>(e + 256);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int d = 2 * i + hf;
          s.v[2 * i] = e4[2 * d];
          s.v[2 * i + 1] = e4[2 * d + 1];
          s.sc[i] = es[d];
        }
        s.kind = 1;
      } else if (hf == 0) {
        flag(a.status, CSA2_DEV_BAD_INDEX);
      }
    }
  } else if (slot < a.K + a.window && a.S_w > 0) {
    const int64_t u = t - a.window + 1 + (slot - a.K);
    const int64_t row = u - sws;
    if (u >= 0 && row >= 0 && row < a.S_w) {
      const uint4* src = reinterpret_cast<const uint4*>(a.swa + ((int64_t)b * a.S_w + row) * kD);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int d = 2 * i + hf;
#pragma unroll
        for (int k = 0; k < 4; ++k) s.v[4 * i + k] = src[4 * d + k];
      }
      s.kind = 2;
    }
  }
}

// Prefetch key slot `slot` (its whole 288 B entry or 512 B window token) into L2.
__device__ __forceinline__ void prefetch_slot(const AttnArgs& a, int b, int64_t base, int64_t t, int slot,
                                              const int32_t* idx_s, int64_t sws) {
  const void* src = nullptr;
  uint32_t bytes = 0;
  if (slot < a.K) {
    const int32_t j = idx_s[slot];
    if (j >= 0 && base >= 0 && base + j < a.pool_entries) {
      src = a.kv_pool + (base + j) * kKvBytes;
      bytes = kKvBytes;
    }
  } else if (slot < a.K + a.window && a.S_w > 0) {
    const int64_t u = t - a.window + 1 + (slot - a.K);
    const int64_t row = u - sws;
    if (u >= 0 && row >= 0 && row < a.S_w) {
      src = a.swa + ((int64_t)b * a.S_w + row) * kD;
      bytes = kD;
    }
  }
  if (bytes) asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

// Dequantise blocks i0, i0+1 of this thread's half row (dim-blocks 2i + hf) of tile row r
// into the key tile.
__device__ __forceinline__ void store_half(uint8_t* Ks, int r, int hf, int i0, const SlotRaw& s) {
#pragma unroll
  for (int ii = 0; ii < 2; ++ii) {
    const int i = i0 + ii;
    uint8_t* blk = Ks + (2 * i + hf) * 16384;
    if (s.kind == 1) {
#pragma unroll
      for (int c = 0; c < 8; ++c) {  // 8 channels per 16 B chunk; scale of channels 16(c/2)..
        const uint4 q4 = s.v[2 * i + (c >> 2)];
        const uint32_t wcode = (c & 3) == 0 ? q4.x : (c & 3) == 1 ? q4.y : (c & 3) == 2 ? q4.z : q4.w;
        const uint32_t sbyte = (s.sc[i] >> (8 * (c >> 1))) & 0xFFu;
        *reinterpret_cast<uint4*>(blk + tc::sw128(r, c * 16)) = e2m1x8_to_f16(wcode, e4m3_scale_f16x2(sbyte));
      }
    } else if (s.kind == 2) {
#pragma unroll
      for (int k = 0; k < 4; ++k) {  // 16 channels per 16 B load: chunks 2k, 2k+1
        const uint4 w = s.v[4 * i + k];
        const uint2 a0 = e4m3x4_to_f16(w.x), a1 = e4m3x4_to_f16(w.y);
        const uint2 a2 = e4m3x4_to_f16(w.z), a3 = e4m3x4_to_f16(w.w);
        *reinterpret_cast<uint4*>(blk + tc::sw128(r, (2 * k) * 16)) = make_uint4(a0.x, a0.y, a1.x, a1.y);
        *reinterpret_cast<uint4*>(blk + tc::sw128(r, (2 * k + 1) * 16)) = make_uint4(a2.x, a2.y, a3.x, a3.y);
      }
    } else {
#pragma unroll
      for (int c = 0; c < 8; ++c) *reinterpret_cast<uint4*>(blk + tc::sw128(r, c * 16)) = make_uint4(0u, 0u, 0u, 0u);
    }
  }
}

// NQ columns of this thread's TMEM lane starting at column `col`, times per-column factors
// (NQ = 16, 32 or 64), written back.
__device__ __forceinline__ void tmem_scale_cols(uint32_t taddr, int NQ, const float* f) {
  if (NQ == 16) {
    uint32_t o[16];
    tc::tmem_ld16(taddr, o);
    uint32_t w[32];
#pragma unroll
    for (int j = 0; j < 16; ++j) w[j] = __float_as_uint(__uint_as_float(o[j]) * f[j]);
    asm volatile("tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
                 "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};\n\t"
                 "tcgen05.wait::st.sync.aligned;" ::"r"(taddr),
                 "r"(w[0]), "r"(w[1]), "r"(w[2]), "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7]),
                 "r"(w[8]), "r"(w[9]), "r"(w[10]), "r"(w[11]), "r"(w[12]), "r"(w[13]), "r"(w[14]), "r"(w[15])
                 : "memory");
  } else {
#pragma unroll 1
    for (int c0 = 0; c0 < NQ; c0 += 32) {
      uint32_t o[32];
      tc::tmem_ld32(taddr + c0, o);
#pragma unroll
      for (int j = 0; j < 32; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * f[c0 + j]);
      tc::tmem_st32(taddr + c0, o);
    }
  }
}

// Barrier over every thread of every CTA of the cluster; orders shared::cluster stores
// before it with loads after it.
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ void st_cluster_f32(uint32_t caddr, float v) {
  asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(caddr), "f"(v) : "memory");
}
__device__ __forceinline__ void st_cluster_v4(uint32_t caddr, uint32_t x, uint32_t y, uint32_t z, uint32_t w) {
  asm volatile("st.shared::cluster.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(caddr), "r"(x), "r"(y), "r"(z), "r"(w)
               : "memory");
}

// NQ: the products' N (the CTA's heads rounded up to 16, 32 or 64), a template parameter
// so each launch runs one compact code path.
template <int NQ>
__global__ void __launch_bounds__(kAttnThreads, 1) attn_kernel(AttnArgs a) {
  chain_launch_dependents();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = tc::align_smem_1024(smem_raw);
  uint8_t* Ks = sm + kOffK;
  uint8_t* Qs = sm + kOffQ;
  uint8_t* Ps = sm + kOffP;
  float* red_max = reinterpret_cast<float*>(sm + kOffMisc);  // [4][64]; merge: received max [C][hpc]
  float* red_sum = red_max + 256;                           // [4][64]; merge: received sum [C][hpc]
  float* m_run = red_sum + 256;                             // [64] running max (base-2 logits)
  float* l_run = m_run + 64;                                // [64] running sum
  float* alpha = l_run + 64;                                // [64] rescale of this tile
  int* valid_s = reinterpret_cast<int*>(alpha + 64);        // [128]
  uint64_t* mbar = reinterpret_cast<uint64_t*>(valid_s + 128);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mbar + 8);
  int32_t* idx_s = reinterpret_cast<int32_t*>(sm + kOffIdx);  // [K] Top-K entry index per slot
  // barriers (mbar[0] unused): key-tile halves written (A: dims 0-255, B: 256-511); S^T
  // ready; P^T ready; PV done
  const uint32_t bar_ka = tc::smem_u32(&mbar[1]), bar_kb = tc::smem_u32(&mbar[2]);
  const uint32_t bar_s = tc::smem_u32(&mbar[3]), bar_p = tc::smem_u32(&mbar[4]), bar_pv = tc::smem_u32(&mbar[5]);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int C = a.csize;
  const int rank = C > 1 ? (int)tc::cluster_ctarank() : 0;
  const int bq = blockIdx.y / a.hgroups;
  const int b = bq / a.Q;
  const int H = a.H;                                 // heads of the query (output layout)
  const int h_base = (blockIdx.y % a.hgroups) * a.hg_size;
  const int NH = min(a.hg_size, H - h_base);         // heads of this cluster, rows 0..NH-1
  const int T = rank < a.n_tiles ? (a.n_tiles - 1 - rank) / C + 1 : 0;  // tiles rank + k C
  const int r = tid >> 1, hf = tid & 1;              // worker: tile row and half

  // set-up that touches no global memory runs while the predecessor finishes
  if (tid == 0) {
    tc::mbar_init(bar_ka, kWorkers);
    tc::mbar_init(bar_kb, kWorkers);
    tc::mbar_init(bar_s, 1);
    tc::mbar_init(bar_p, kWorkers);
    tc::mbar_init(bar_pv, 1);
  }
  if (tid < kHeadsPad) {
    m_run[tid] = -INFINITY;
    l_run[tid] = 0.0f;
  }
  if (warp == 0) tc::tmem_alloc(tc::smem_u32(tmem_slot), kTmemCols);
  // The queries are a caller input that no library call writes, so they are staged while the
  // predecessor finishes: fp32 -> f16 tile scaled by sm_scale * log2(e), rows past NH zero, 8
  // channels per chunk.  (A library kernel starts early only behind another library kernel,
  // and whatever produced the queries before that one has completed by then.)
  if (T > 0) {
    const float qscale = a.sm_scale * 1.4426950408889634f;
    const float* qg = a.q + ((int64_t)bq * H + h_base) * kD;
#pragma unroll 4
    for (int i = tid; i < NQ * 64; i += kWorkers) {
      const int h = i >> 6, ch = i & 63, db = ch >> 3, c = ch & 7;
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (h < NH) {
        const float4 x0 = __ldg(reinterpret_cast<const float4*>(qg + h * kD + ch * 8));
        const float4 x1 = __ldg(reinterpret_cast<const float4*>(qg + h * kD + ch * 8 + 4));
        v.x = half2_bits(x0.x * qscale, x0.y * qscale);
        v.y = half2_bits(x0.z * qscale, x0.w * qscale);
        v.z = half2_bits(x1.x * qscale, x1.y * qscale);
        v.w = half2_bits(x1.z * qscale, x1.w * qscale);
      }
      *reinterpret_cast<uint4*>(Qs + db * 8192 + tc::sw128(h, c * 16)) = v;
    }
    tc::fence_async_smem();
  }
  chain_wait();
  const int64_t base = a.seq_base[b];
  const int64_t tq = a.q_pos[bq];
  const int64_t sws = a.S_w > 0 ? a.swa_start[b] : 0;

  // the first tile's gather depends on one index load only; the indices of the later
  // tiles are staged by asynchronous copies
  SlotRaw sr;
  sr.kind = 0;
  if (T > 0) {
    const int slot0 = rank * kTile + r;
    const int32_t j0 = slot0 < a.K ? a.topk[(int64_t)bq * a.K + slot0] : -1;
    gather_slot(a, b, base, tq, slot0, hf, j0, sws, sr);
    const int32_t* trow = a.topk + (int64_t)bq * a.K;
    for (int i = tid; i < (T - 1) * kTile; i += kWorkers) {
      const int slot = (rank + (1 + i / kTile) * C) * kTile + (i % kTile);
      if (slot < a.K) tc::cp_async4(tc::smem_u32(idx_s + slot), trow + slot);
    }
    tc::cp_async_commit();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  bool timed_out = false;

  // ---- tensor-core products, issued by thread 0 ---------------------------------------------------
  const uint32_t idesc_s = tc::idesc_f16(kTile, NQ, false, false);
  const uint32_t idesc_o = tc::idesc_f16(kTile, NQ, true, true);
  const uint32_t rb = 2u * (uint32_t)NQ, pcode = tc::swizzle_code(rb);
  const uint32_t ks_a = tc::smem_u32(Ks), qs_a = tc::smem_u32(Qs), ps_a = tc::smem_u32(Ps);
  uint32_t last_bar = 0, last_par = 0;  // thread 0: the last commit
  // descriptors of the operands' first bytes; each MMA advances them by a constant
  const uint64_t kd0 = tc::smem_desc_sw128(ks_a, 16, 1024), qd0 = tc::smem_desc_sw128(qs_a, 16, 1024);
  const uint64_t kmn0 = tc::smem_desc_sw128(ks_a, 16384, 1024);
  const uint64_t pd0 = tc::smem_desc(ps_a, 64u * rb, 8u * rb, pcode);
  // S^T = Kt . Qs^T over dims 256 hb .. 256 hb + 255: dim-block db adds to partial sum db mod 4
  auto issue_qk = [&](int hb) {
#pragma unroll
    for (int kk = 0; kk < 4; ++kk)
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int db = hb * 4 + i;
        tc::mma_f16(tmem + kColS + 64 * i, tc::desc_add(kd0, db * 16384 + kk * 32), tc::desc_add(qd0, db * 8192 + kk * 32),
                    idesc_s, (hb > 0 || kk > 0) ? 1u : 0u);
      }
  };
  // O^T += Kt^T . P^T: B = P^T [128 keys x NQ heads], MN-major, rows of rb = 2 NQ bytes
  // (8-row groups at 8 rb, one 16-key K step at 16 rb); the four M-tiles are independent
  // accumulators, issued interleaved
  auto issue_pv = [&](int k) {
#pragma unroll
    for (int ks = 0; ks < kTile / 16; ++ks)
#pragma unroll
      for (int mt = 0; mt < 4; ++mt)
        tc::mma_f16(tmem + kColO + 64 * mt, tc::desc_add(kmn0, (2 * mt) * 16384 + ks * 2048),
                    tc::desc_add(pd0, ks * 16 * rb), idesc_o, (ks > 0 || k > 0) ? 1u : 0u);
  };

  {
    // ---- workers --------------------------------------------------------------------------------
    bool fail = false;

    const int q4 = warp & 3, half = warp >> 2;
    const int key = q4 * 32 + lane;                   // this thread's TMEM lane (tile row)
    const uint32_t lane_base = tmem + ((uint32_t)(q4 * 32) << 16);
    // S^T columns of this warp: with 16 heads, 8 in each half of the warps; else 32 per warp
    // of the halves that hold any
    const bool s_cols = NQ == 16 || half * 32 < NQ;
    const int ncols = NQ == 16 ? 8 : 32;
    const int col0 = NQ == 16 ? half * 8 : half * 32;
    for (int k = 0; k < T && !timed_out; ++k) {
      const uint32_t par = (uint32_t)k & 1u;
      const int tile = rank + k * C;
      // ---- dequantise tile k once PV(k-1) has read the key tile -----------------------------
      if (k > 0) fail |= !tc::mbar_wait(bar_pv, par ^ 1u, kMaxPolls);
      tc::fence_after_sync();
      store_half(Ks, r, hf, 0, sr);
      if (hf == 0) valid_s[r] = sr.kind != 0;
      tc::fence_async_smem();
      tc::mbar_arrive(bar_ka);
      if (tid == 0) {  // every row's first half is written
        fail |= !tc::mbar_wait(bar_ka, par, kMaxPolls);
        tc::fence_after_sync();
        issue_qk(0);
      }
      store_half(Ks, r, hf, 2, sr);
      tc::fence_async_smem();
      tc::mbar_arrive(bar_kb);
      if (tid == 0) {
        fail |= !tc::mbar_wait(bar_kb, par, kMaxPolls);
        tc::fence_after_sync();
        issue_qk(1);
        tc::commit(bar_s);
        last_bar = bar_s;
        last_par = par;
      }
      // ---- bring the next tile's rows into L2 (no registers held across the softmax) ------------
      if (k + 1 < T) {
        if (k == 0) {  // the staged indices are visible to every worker
          tc::cp_async_wait<0>();
          tc::named_sync_or(kWorkerBar, kWorkers, false);
        }
        if (hf == 0) prefetch_slot(a, b, base, tq, (tile + C) * kTile + r, idx_s, sws);
      }
      // ---- softmax of tile k -------------------------------------------------------------------
      fail |= !tc::mbar_wait(bar_s, par, kMaxPolls);
      tc::fence_after_sync();
      if (tc::named_sync_or(kWorkerBar, kWorkers, fail)) {  // valid_s complete; agree on giving up
        timed_out = true;
        break;
      }
      const bool kv = valid_s[key] != 0;
      float s[32], v[32];
      if (s_cols) {
#pragma unroll
        for (int jj = 0; jj < 32; ++jj) s[jj] = 0.0f;
#pragma unroll
        for (int i = 0; i < 4; ++i) {  // the four partial sums of S^T
          uint32_t raw[32];
          if (NQ == 16) tc::tmem_ld8(lane_base + kColS + 64 * i + col0, raw);
          else tc::tmem_ld32(lane_base + kColS + 64 * i + col0, raw);
#pragma unroll
          for (int jj = 0; jj < 32; ++jj) s[jj] += jj < ncols ? __uint_as_float(raw[jj]) : 0.0f;
        }
#pragma unroll
        for (int jj = 0; jj < 32; ++jj) {
          s[jj] = (jj < ncols && kv && col0 + jj < NH) ? s[jj] : -INFINITY;
          v[jj] = s[jj];
        }
        if (NQ == 16) {
          float v8[8];
#pragma unroll
          for (int jj = 0; jj < 8; ++jj) v8[jj] = v[jj];
          const float m8 = xpose_reduce8<true>(v8, lane);
          if (lane < 8) red_max[q4 * 64 + col0 + lane] = m8;
        } else {
          red_max[q4 * 64 + half * 32 + lane] = xpose_reduce<true>(v, lane);
        }
      }
      tc::named_sync_or(kWorkerBar, kWorkers, false);
      bool raise = false;
      if (tid < NQ) {  // per head: the tile's max, and whether the running max must move
        const float mt = fmaxf(fmaxf(red_max[tid], red_max[64 + tid]), fmaxf(red_max[128 + tid], red_max[192 + tid]));
        const float mo = m_run[tid];
        float f = 1.0f;
        if (tid < NH && mt != -INFINITY) {
          if (mo == -INFINITY) {
            m_run[tid] = mt;  // nothing accumulated yet: no rescale
          } else if (mt > mo + kStaleMax) {
            m_run[tid] = mt;
            f = exp2f(mo - mt);
            raise = true;
          }
        }
        alpha[tid] = f;
      }
      const bool rescale = tc::named_sync_or(kWorkerBar, kWorkers, raise) && k > 0;
      if (s_cols) {
        uint32_t ph[16];
#pragma unroll
        for (int jj = 0; jj < 32; jj += 2) {
          const int c0 = col0 + jj;
          const float m0 = jj < ncols ? m_run[c0] : -INFINITY, m1 = jj < ncols ? m_run[c0 + 1] : -INFINITY;
          const float p0 = m0 == -INFINITY ? 0.0f : exp2f(s[jj] - m0);
          const float p1 = m1 == -INFINITY ? 0.0f : exp2f(s[jj + 1] - m1);
          __half2 hp = __floats2half2_rn(p0, p1);
          ph[jj >> 1] = *reinterpret_cast<uint32_t*>(&hp);
          const float2 back = __half22float2(hp);
          v[jj] = back.x;  // the sum uses exactly the f16 values the PV product sees
          v[jj + 1] = back.y;
        }
        // P^T rows of NQ heads (2 NQ bytes, the swizzle of that width)
        if (NQ == 16) {
          *reinterpret_cast<uint4*>(Ps + tc::swz(key, half * 16, 32)) = make_uint4(ph[0], ph[1], ph[2], ph[3]);
          float v8[8];
#pragma unroll
          for (int jj = 0; jj < 8; ++jj) v8[jj] = v[jj];
          const float s8 = xpose_reduce8<false>(v8, lane);
          if (lane < 8) red_sum[q4 * 64 + col0 + lane] = s8;
        } else {
          const uint32_t rbw = 2u * (uint32_t)NQ;
#pragma unroll
          for (int c = 0; c < 4; ++c)
            *reinterpret_cast<uint4*>(Ps + tc::swz(key, half * 64 + c * 16, rbw)) =
                make_uint4(ph[4 * c], ph[4 * c + 1], ph[4 * c + 2], ph[4 * c + 3]);
          red_sum[q4 * 64 + half * 32 + lane] = xpose_reduce<false>(v, lane);
        }
      }
      if (rescale) {  // PV(k-1) has completed (waited above): scale the accumulated output
#pragma unroll 1
        for (int mt = half; mt < 4; mt += 2) tmem_scale_cols(lane_base + kColO + 64 * mt, NQ, alpha);
      }
      tc::fence_async_smem();
      tc::fence_before_sync();
      tc::named_sync_or(kWorkerBar, kWorkers, false);
      if (tid < NQ)
        l_run[tid] = l_run[tid] * alpha[tid] +
                     ((red_sum[tid] + red_sum[64 + tid]) + (red_sum[128 + tid] + red_sum[192 + tid]));
      tc::mbar_arrive(bar_p);
      if (tid == 0) {  // every P^T row is written and the output rescaled
        fail |= !tc::mbar_wait(bar_p, par, kMaxPolls);
        tc::fence_after_sync();
        issue_pv(k);
        tc::commit(bar_pv);
        last_bar = bar_pv;
        last_par = par;
      }
      // ---- gather the next tile (L2 hits by now; lands while PV(k) runs) -----------------------
      if (k + 1 < T) {
        const int slot = (tile + C) * kTile + r;
        gather_slot(a, b, base, tq, slot, hf, slot < a.K ? idx_s[slot] : -1, sws, sr);
      }
    }
    if (!timed_out && T > 0) timed_out = !tc::mbar_wait(bar_pv, (uint32_t)(T - 1) & 1u, kMaxPolls);
    timed_out = tc::named_sync_or(kWorkerBar, kWorkers, timed_out);  // l_run final; agree on the outcome
    tc::fence_after_sync();
    if (timed_out) {
      if (tid == 0) flag(a.status, CSA2_DEV_TIMEOUT);
      if (tid < kHeadsPad) l_run[tid] = 0.0f;  // contribute nothing
    }
    if (C == 1 && !timed_out) {
      // ---- output: O^T rows (lanes = channels) / l, log-sum-exp ------------------------------------
      const int cw = NQ == 16 ? 16 : 32;
#pragma unroll 1
      for (int mt = half; mt < 4; mt += 2) {
        const int d = mt * 128 + q4 * 32 + lane;
#pragma unroll 1
        for (int c0 = 0; c0 < NQ; c0 += cw) {
          uint32_t o[32];
          if (T > 0) {
            if (cw == 16) tc::tmem_ld16(lane_base + kColO + 64 * mt + c0, o);
            else tc::tmem_ld32(lane_base + kColO + 64 * mt + c0, o);
          }
#pragma unroll
          for (int jj = 0; jj < 32; ++jj) {
            const int h = c0 + jj;
            if (jj < cw && h < NH) {
              const float l = l_run[h];
              a.out[((int64_t)bq * H + h_base + h) * kD + d] = l > 0.0f ? __uint_as_float(o[jj]) / l : 0.0f;
            }
          }
        }
      }
      if (tid < NH) {
        const float l = l_run[tid];
        a.lse[(int64_t)bq * H + h_base + tid] = l > 0.0f ? (m_run[tid] + log2f(l)) * 0.69314718055994531f : -INFINITY;
      }
    }
  }

  if (C > 1) {
    // ---- merge across the cluster: head h belongs to CTA h / hpc, hpc a multiple of 4 -------------
    // Partials travel as 16-byte distributed-shared-memory stores of 4 heads of one channel:
    // CTA o receives recv[c][d][0..hpc) from every CTA c (its heads' partial O^T rows).
    const int hpc = (((NH + C - 1) / C) + 3) & ~3;
    const int h0 = rank * hpc, n_own = max(0, min(hpc, NH - h0));
    float* fac = reinterpret_cast<float*>(Ps);                // [C][64] merge factors
    float* linv = fac + kMaxCluster * kHeadsPad;              // [hpc]
    // With 16 heads, a CTA's query tile uses 16 of the 64 rows of each 8 KB dim-block and its
    // P tile 4 KB of 16: the received partials go to that spare space (rows 16-63 of the dim-
    // blocks, then the P area past the tile, in 6 KB pieces), and the per-head max and sum to
    // the tail of the misc area.  Nothing else reads or writes those bytes, so a CTA may push
    // as soon as its own products are done: no cluster barrier first.  Otherwise the partials
    // go over the key and query tiles, once every CTA of the cluster is done with them.
    const bool spare = NQ == 16 && C * kD * hpc * 4 <= 10 * 6144;
    auto recv_off = [&](uint32_t byte) -> uint32_t {  // shared-memory offset of a received byte
      if (!spare) return kOffRecv + byte;
      const uint32_t g = byte / 6144u, r = byte - g * 6144u;
      return g < 8u ? kOffQ + g * 8192u + 2048u + r : kOffP + 4096u + (g - 8u) * 6144u + r;
    };
    float* rml = reinterpret_cast<float*>(sm + kOffMisc + 3584);  // spare: max [C][hpc], sum [C][hpc]
    float* rmax = spare ? rml : red_max;
    float* rsum = spare ? rml + C * hpc : red_sum;
    tc::fence_before_sync();
    if (!spare) cluster_sync_all();  // every CTA has finished its products: key and query tiles are free
    {
      const int q4 = warp & 3, half = warp >> 2;
      const uint32_t lane_base = tmem + ((uint32_t)(q4 * 32) << 16);
      const uint32_t sm_a = tc::smem_u32(sm);
      tc::fence_after_sync();
      const int cw = NQ == 16 ? 16 : 32;
      const bool have = T > 0 && !timed_out;
#pragma unroll 1
      for (int mt = half; mt < 4; mt += 2) {
        const int d = mt * 128 + q4 * 32 + lane;
#pragma unroll 1
        for (int c0 = 0; c0 < NQ; c0 += cw) {
          uint32_t o[32];
          if (have) {
            if (cw == 16) tc::tmem_ld16(lane_base + kColO + 64 * mt + c0, o);
            else tc::tmem_ld32(lane_base + kColO + 64 * mt + c0, o);
          }
#pragma unroll
          for (int j4 = 0; j4 < 8; ++j4) {
            const int h = c0 + 4 * j4;  // heads h..h+3 share an owner (hpc is a multiple of 4)
            if (4 * j4 < cw && h < NH) {
              const int o_rank = h / hpc, hl = h - o_rank * hpc;
              const uint32_t dst = sm_a + recv_off((uint32_t)(((rank * kD + d) * hpc + hl) * 4));
              if (have)
                st_cluster_v4(tc::mapa(dst, (uint32_t)o_rank), o[4 * j4], o[4 * j4 + 1], o[4 * j4 + 2], o[4 * j4 + 3]);
              else
                st_cluster_v4(tc::mapa(dst, (uint32_t)o_rank), 0u, 0u, 0u, 0u);
            }
          }
        }
      }
      if (tid < NH) {  // this CTA's max and sum of head tid, to its owner
        const int o_rank = tid / hpc, hl = tid - o_rank * hpc;
        const float l = l_run[tid];
        st_cluster_f32(tc::mapa(tc::smem_u32(rmax + rank * hpc + hl), (uint32_t)o_rank),
                       l > 0.0f ? m_run[tid] : -INFINITY);
        st_cluster_f32(tc::mapa(tc::smem_u32(rsum + rank * hpc + hl), (uint32_t)o_rank), l);
      }
    }
    cluster_sync_all();  // every partial has arrived
    {
      if (tid < n_own) {
        float M = -INFINITY;
        for (int c = 0; c < C; ++c)
          if (rsum[c * hpc + tid] > 0.0f) M = fmaxf(M, rmax[c * hpc + tid]);
        float L = 0.0f;
        for (int c = 0; c < C; ++c) {
          const float lc = rsum[c * hpc + tid];
          const float f = lc > 0.0f ? exp2f(rmax[c * hpc + tid] - M) : 0.0f;
          fac[c * kHeadsPad + tid] = f;
          L = fmaf(lc, f, L);
        }
        linv[tid] = L > 0.0f ? 1.0f / L : 0.0f;
        a.lse[(int64_t)bq * H + h_base + h0 + tid] = L > 0.0f ? (M + log2f(L)) * 0.69314718055994531f : -INFINITY;
      }
      tc::named_sync_or(kWorkerBar, kWorkers, false);
      // thread -> (channel d, 4 heads); the sums for each head go to consecutive channels
      for (int i = tid; i < n_own * (kD / 4); i += kWorkers) {
        const int g4 = i / kD, d = i % kD;  // heads 4 g4 .. 4 g4 + 3 of this CTA
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int c = 0; c < C; ++c) {
          const float4 x =
              *reinterpret_cast<const float4*>(sm + recv_off((uint32_t)(((c * kD + d) * hpc + 4 * g4) * 4)));
          acc.x = fmaf(x.x, fac[c * kHeadsPad + 4 * g4 + 0], acc.x);
          acc.y = fmaf(x.y, fac[c * kHeadsPad + 4 * g4 + 1], acc.y);
          acc.z = fmaf(x.z, fac[c * kHeadsPad + 4 * g4 + 2], acc.z);
          acc.w = fmaf(x.w, fac[c * kHeadsPad + 4 * g4 + 3], acc.w);
        }
        const float v4[4] = {acc.x, acc.y, acc.z, acc.w};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int hl = 4 * g4 + u;
          if (hl < n_own) a.out[((int64_t)bq * H + h_base + h0 + hl) * kD + d] = v4[u] * linv[hl];
        }
      }
    }
  }
  // every issued product completes before the accumulators are released (this matters
  // only when a wait gave up)
  if (tid == 0 && last_bar) tc::mbar_wait(last_bar, last_par, kMaxPolls);
  tc::fence_before_sync();
  __syncthreads();
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
  return 0;  // every partial result stays on chip
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
  // Split: C CTAs per cluster take a query's tiles round-robin (few queries want a wide
  // split: more SMs at work on each), and a query's heads may go to G clusters of H/G heads
  // (each gathers and dequantises the same keys, but its softmax and merge are smaller).
  // (C, G) minimises waves x per-CTA time, with one CTA per SM and per-phase costs in
  // microseconds measured on the kernel: set-up, a tile, the cluster merge, the last two
  // growing with the CTA's heads.
  {
    double best = 1e30;
    a.csize = 1;
    a.hgroups = 1;
    const int cmax = a.n_tiles < 1 ? 1 : (a.n_tiles > kMaxCluster ? kMaxCluster : a.n_tiles);
    for (int g = 1; g <= 4; ++g) {
      if (H % g != 0 || (H / g) % 16 != 0 || H / g > kHeadsPad) continue;
      const double hfrac = (double)(H / g) / 64.0;
      for (int c = 1; c <= cmax; ++c) {
        const double waves = (double)((BQ * g * c + sms - 1) / sms);
        const double per_cta = (2.5 + 0.5 * hfrac) + (double)((a.n_tiles + c - 1) / c) * (1.8 + 0.7 * hfrac) +
                               (c > 1 ? 0.8 + 1.5 * hfrac : 0.0);
        if (waves * per_cta < best - 1e-9) {
          best = waves * per_cta;
          a.csize = c;
          a.hgroups = g;
        }
      }
    }
  }
  a.hg_size = H / a.hgroups;
  const int nq = a.hg_size <= 16 ? 16 : (a.hg_size <= 32 ? 32 : kHeadsPad);
  auto* fn = nq == 16 ? attn_kernel<16> : (nq == 32 ? attn_kernel<32> : attn_kernel<kHeadsPad>);
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
  if (e != cudaSuccess) return e;
  e = launch_chained(fn, dim3((unsigned)a.csize, (unsigned)(BQ * a.hgroups)), dim3(kAttnThreads), kSmemBytes,
                     stream, a.csize > 1 ? (unsigned)a.csize : 0u, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace csa2
