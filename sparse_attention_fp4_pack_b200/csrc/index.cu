// a2..a5: indexer scan (flat, hierarchical, Reindex) on the sm_100a tensor cores, and
// Top-K selection.
//
// P1 (onedev.kr "KV 캐시를 토큰당 890바이트로 압축한 552B 멀티모달 MoE, DeepSeek-V4.1-Flash")
//   §무엇과 다른가 — a Full layer scores every causally visible entry with its own indexer
//   Q and picks Top-K; Reindex rescoring with the layer's own indexer Q; the
//   hierarchical indexer's first Full layer builds a candidate pool of blocks of 8
//   positions, 2,048 of them giving 16,384 candidates.
// P3 (genexis.ai "100만 토큰을 0.9GB에…") §레이어 40개 가운데 4개만 전역 캐시를 만듭니다 —
//   Reindex layers pick 512 inside that pool.
//
// Score of entry j for one query:  score_j = s_j * sum_h w_h * max(0, q_h . c_j)
// (c_j the key's E2M1 values, s_j >= 0 its fp32 scale, so the ReLU commutes with s_j).
//
// scan_tc_kernel computes the dot products exactly on the tensor cores (tcgen05.mma
// kind::i8, int32 accumulation):
//   * A (128 entries x 128 dims, u8): u = 2c + 12 in [0, 24] — the E2M1 value doubled and
//     offset to be non-negative; two byte-permutes per 4 codes build it (sign-replicate
//     selects the positive or negative table).
//   * B (N rows x 128 dims, s8): each query head h is scaled by S_h = 127 / max|q_h| and
//     split into four int8 limbs, x = q*S_h = L0 + L1/128 + L2/128^2 + L3/128^3 with an
//     error below 0.5/128^3 (about 2e-9 of max|q_h|).
//   * D (128 x N, s32): acc_p = sum_d u_d L_p,d, so sum_d c_d L_p,d = (acc_p - 12 T_p)/2
//     with T_p = sum_d L_p,d; the epilogue combines the limbs in fp32:
//     q_h . c_j = (sum_p 128^-p (acc_p - 12 T_p)) / (2 S_h).
// The raw 68 B keys reach shared memory through cp.async (16 B copies, ragged ends with
// 4 B copies, one tile ahead); Reindex tiles are 16 gathered blocks of 8 entries.  Each
// of the 128 threads owns one tile row (entry) end to end: it builds the row's A operand,
// and after the MMA reads the same TMEM lane and writes the entry's order-preserving
// uint32 key (hierarchical mode: the max over `block` neighbouring lanes).  A CTA takes
// a group of up to G queries of one sequence (multi-query verify), so the A operand is
// built once for the group.
#include "csa2_device.cuh"
#include "tc.cuh"

namespace csa2 {

enum ScanMode : int { kFlat = 0, kHier = 1, kReindex = 2 };

constexpr int kRows = 128;               // entries per tile = UMMA M
constexpr int kScanThreads = 128;
constexpr int kRawBytes = 12288;         // raw staging per buffer (covers every gather block size)
constexpr uint32_t kScanPolls = 1u << 22;

struct ScanArgs {
  const float* q;
  const float* w;
  const uint8_t* ik_pool;
  int64_t pool_entries;
  const int64_t* seq_base;
  const int32_t* n_vis;
  const int32_t* blocks;  // reindex only
  int Q, HI, hipad, G, n_groups, n_blocks, block;
  int N;                  // MMA N = G * hipad * 4
  int tmem_cols;
  int tiles_per_cta;
  int64_t max_n_vis;
  int64_t key_stride;
  uint32_t* keys;
  uint32_t* status;
};

__device__ __forceinline__ int64_t valid_count(const ScanArgs& a, int b, int bq, bool report) {
  const int64_t base = a.seq_base[b];
  const int64_t n = a.n_vis[bq];
  if (n < 0 || n > a.max_n_vis || base < 0 || base + n > a.pool_entries) {
    if (report) flag(a.status, CSA2_DEV_BAD_COUNT);
    return 0;
  }
  return n;
}

// Copy bytes [src, src+nbytes) (4-byte granular) to shared memory at dst, where
// dst and src agree modulo 16: 4 B copies up to the first 16 B boundary, then 16 B
// copies, then 4 B copies.  Work is split over `nthr` threads numbered `sub`.
__device__ __forceinline__ void stage_async(uint32_t dst, const uint8_t* src, int nbytes, int sub, int nthr) {
  const int mis = (int)(reinterpret_cast<uintptr_t>(src) & 15u);
  const int head = mis ? min(nbytes, 16 - mis) : 0;
  const int body = (nbytes - head) & ~15;
  const int tail = nbytes - head - body;
  for (int i = sub; i < head / 4; i += nthr) tc::cp_async4(dst + 4 * i, src + 4 * i);
  for (int i = sub; i < body / 16; i += nthr) tc::cp_async16(dst + head + 16 * i, src + head + 16 * i);
  for (int i = sub; i < tail / 4; i += nthr)
    tc::cp_async4(dst + head + body + 4 * i, src + head + body + 4 * i);
}

// 8 E2M1 codes (one word) -> 8 bytes u = 2c + 12.
__device__ __forceinline__ uint2 codes_to_u8(uint32_t w) {
  // tables indexed by the 3-bit magnitude m: 12 + 2|c| and 12 - 2|c|
  constexpr uint32_t kPosLo = 0x0F0E0D0Cu, kPosHi = 0x18141210u;
  constexpr uint32_t kNegLo = 0x090A0B0Cu, kNegHi = 0x00040608u;
  const uint32_t wn = w ^ 0x88888888u;
  uint32_t p0, p1, n0, n1;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(p0) : "r"(kPosLo), "r"(kPosHi), "r"(w));
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(p1) : "r"(kPosLo), "r"(kPosHi), "r"(w >> 16));
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(n0) : "r"(kNegLo), "r"(kNegHi), "r"(wn));
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(n1) : "r"(kNegLo), "r"(kNegHi), "r"(wn >> 16));
  return make_uint2(p0 | n0, p1 | n1);
}

template <int MODE, int HIPAD>
__global__ void __launch_bounds__(kScanThreads) scan_tc_kernel(ScanArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* As = sm;                                   // [128 rows x 128 B], 128 B swizzle
  uint8_t* Bs = As + kRows * 128;                     // [N rows x 128 B]
  uint8_t* raw = Bs + a.N * 128;                      // 2 x kRawBytes
  int32_t* corr = reinterpret_cast<int32_t*>(raw + 2 * kRawBytes);  // [N]
  float* wq = reinterpret_cast<float*>(corr + a.N);                 // [G * HIPAD]
  int64_t* nq = reinterpret_cast<int64_t*>(wq + a.G * HIPAD);       // [G] visible count per query
  int32_t* segc = reinterpret_cast<int32_t*>(nq + a.G);             // [2][128] gathered block ids
  uint64_t* mbar = reinterpret_cast<uint64_t*>(segc + 256);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mbar + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int b = blockIdx.y / a.n_groups;
  const int gidx = blockIdx.y % a.n_groups;
  const int q0 = gidx * a.G;
  const int G = min(a.G, a.Q - q0);
  const int64_t base = a.seq_base[b];

  // items of this CTA's query group: entries (flat/hier) or candidate slots (reindex)
  int64_t limit = 0;
  for (int g = 0; g < G; ++g) {
    const int64_t n = valid_count(a, b, b * a.Q + q0 + g, false);
    limit = n > limit ? n : limit;
  }
  if (MODE == kReindex) limit = (int64_t)a.n_blocks * a.block;
  const int64_t item0 = (int64_t)blockIdx.x * a.tiles_per_cta * kRows;
  if (item0 >= limit) return;
  const int64_t left_tiles = (limit - item0 + kRows - 1) / kRows;
  const int ntiles = (int)(left_tiles < a.tiles_per_cta ? left_tiles : a.tiles_per_cta);

  if (warp == 0) tc::tmem_alloc(tc::smem_u32(tmem_slot), a.tmem_cols);
  if (tid == 32) tc::mbar_init(tc::smem_u32(mbar), 1);
  if (tid < G) nq[tid] = valid_count(a, b, b * a.Q + q0 + tid, blockIdx.x == 0);

  const uint8_t* seq = a.ik_pool + base * kIkBytes;
  const int mis = (int)((reinterpret_cast<uintptr_t>(seq)) & 15u);  // same for every tile
  const uint32_t raw_a = tc::smem_u32(raw);
  // reindex tiles: 128 / block gathered blocks, each staged at seg_stride (16 B multiple)
  const int seg_stride = ((a.block * kIkBytes + 16) + 15) & ~15;

  // raw tile loader: tile index ti into buffer ti & 1
  auto load_tile = [&](int ti) {
    const int64_t i0 = item0 + (int64_t)ti * kRows;
    const uint32_t dst = raw_a + (ti & 1) * kRawBytes;
    if (MODE != kReindex) {
      const int cnt = (int)(limit - i0 < kRows ? limit - i0 : kRows);
      stage_async(dst + mis, seq + i0 * kIkBytes, cnt * kIkBytes, tid, kScanThreads);
    } else {
      const int s = tid / a.block, sub = tid % a.block;  // 128/block blocks, `block` threads each
      const int64_t slot_blk = i0 / a.block + s;
      int32_t c = -1;
      if (slot_blk < a.n_blocks) c = a.blocks[(int64_t)(b * a.Q + q0) * a.n_blocks + slot_blk];
      if (sub == 0) {
        segc[(ti & 1) * 128 + s] = c;
        if (c < -1) flag(a.status, CSA2_DEV_BAD_INDEX);
      }
      int cnt = 0;
      if (c >= 0) {
        const int64_t rem = nq[0] - (int64_t)c * a.block;
        cnt = rem <= 0 ? 0 : (int)(rem < a.block ? rem : a.block);
      }
      if (cnt > 0) {
        // a block starts at its own address residue mod 16 unless block*68 is a 16 B multiple
        const uint8_t* src = seq + (int64_t)c * a.block * kIkBytes;
        const int smis = (int)(reinterpret_cast<uintptr_t>(src) & 15u);
        stage_async(dst + s * seg_stride + smis, src, cnt * kIkBytes, sub, a.block);
      }
    }
    tc::cp_async_commit();
  };

  // ---- B operand: four int8 limbs of every (query, head), plus epilogue constants ---------
  for (int gh = warp; gh < a.G * HIPAD; gh += kScanThreads / 32) {
    const int g = gh / HIPAD, h = gh % HIPAD;
    const bool live = g < G && h < a.HI;
    float x[4] = {0.f, 0.f, 0.f, 0.f};
    float wv = 0.f;
    if (live) {
      const int64_t bq = (int64_t)b * a.Q + q0 + g;
      const float4 v = reinterpret_cast<const float4*>(a.q + (bq * a.HI + h) * kDI)[lane];
      x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w;
      wv = a.w[bq * a.HI + h];
    }
    float m = fmaxf(fmaxf(fabsf(x[0]), fabsf(x[1])), fmaxf(fabsf(x[2]), fabsf(x[3])));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    // power-of-two scale S = 2^(5 - exponent(m)): x = q*S is exact and |x| < 64, so the
    // first limb never leaves int8 and the limbs represent x to 2^-21 (heads whose max is
    // below 1e-30 count as zero)
    float S = 0.f;
    if (m > 1e-30f) {
      const int E = (int)((__float_as_uint(m) >> 23) & 0xFFu) - 127;
      S = __uint_as_float((uint32_t)(127 + 5 - E) << 23);
    }
    uint32_t limb[4] = {0u, 0u, 0u, 0u};
    int lsum[4] = {0, 0, 0, 0};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      float r = x[e] * S;
#pragma unroll
      for (int p = 0; p < 4; ++p) {
        const float L = rintf(r);
        const int li = (int)L;
        limb[p] |= ((uint32_t)(li & 0xFF)) << (8 * e);
        lsum[p] += li;
        r = (r - L) * 128.0f;
      }
    }
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      const int n = gh * 4 + p;
      *reinterpret_cast<uint32_t*>(Bs + tc::sw128(n, lane * 4)) = limb[p];
      int t = lsum[p];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
      if (lane == 0) corr[n] = 0x4B400000 - 12 * t;
    }
    if (lane == 0) wq[gh] = S > 0.f ? wv / (2.0f * S) : 0.f;
  }

  __syncthreads();  // nq visible to every thread before the first gather
  load_tile(0);
  tc::fence_async_smem();
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  const uint32_t idesc = tc::idesc_i8(kRows, a.N, false, true);
  const uint32_t lane_addr = tmem + ((uint32_t)(warp * 32) << 16);
  bool timed_out = false;

  for (int ti = 0; ti < ntiles; ++ti) {
    if (ti + 1 < ntiles) load_tile(ti + 1);
    else tc::cp_async_commit();  // keep the group count uniform
    tc::cp_async_wait<1>();
    __syncthreads();
    const int64_t i0 = item0 + (int64_t)ti * kRows;
    // ---- this thread's row: locate the entry, build the A row --------------------------
    const uint8_t* rbuf = raw + (ti & 1) * kRawBytes;
    const uint8_t* ent;
    bool valid;
    int64_t j;  // entry index within the sequence
    if (MODE != kReindex) {
      j = i0 + tid;
      valid = j < limit;
      ent = rbuf + mis + tid * kIkBytes;
    } else {
      const int s = tid / a.block, r = tid % a.block;
      const int32_t c = segc[(ti & 1) * 128 + s];
      j = (int64_t)c * a.block + r;
      valid = c >= 0 && j < nq[0];
      const int smis = c >= 0 ? (int)(reinterpret_cast<uintptr_t>(seq + (int64_t)c * a.block * kIkBytes) & 15u) : 0;
      ent = rbuf + s * seg_stride + smis + r * kIkBytes;
    }
    float sj = 0.f;
    if (valid) {
      const uint32_t* ew = reinterpret_cast<const uint32_t*>(ent);
      uint32_t cw[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) cw[i] = ew[i];
      sj = __uint_as_float(ew[16]);
#pragma unroll
      for (int c16 = 0; c16 < 8; ++c16) {  // 16 codes -> one 16 B chunk of the A row
        const uint2 lo = codes_to_u8(cw[2 * c16]);
        const uint2 hi = codes_to_u8(cw[2 * c16 + 1]);
        *reinterpret_cast<uint4*>(As + tc::sw128(tid, c16 * 16)) = make_uint4(lo.x, lo.y, hi.x, hi.y);
      }
    }
    tc::fence_async_smem();
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (tid == 0) {
#pragma unroll
      for (int ks = 0; ks < 4; ++ks) {  // K = 128 dims in steps of 32
        const uint64_t ad = tc::smem_desc_sw128(tc::smem_u32(As + ks * 32), 16, 1024);
        const uint64_t bd = tc::smem_desc_sw128(tc::smem_u32(Bs + ks * 32), 16, 1024);
        tc::mma_i8(tmem, ad, bd, idesc, ks > 0 ? 1u : 0u);
      }
      tc::commit(tc::smem_u32(mbar));
    }
    timed_out = __syncthreads_or(tc::mbar_wait(tc::smem_u32(mbar), ti & 1, kScanPolls) ? 0 : 1) != 0;
    tc::fence_after_sync();
    if (timed_out) break;
    // ---- epilogue: limbs -> fp32 dot products -> ReLU-weighted score -> key --------------
    for (int g = 0; g < G; ++g) {
      uint32_t r[HIPAD * 4];
      if (HIPAD == 4) {
        tc::tmem_ld16(lane_addr + g * 16, r);
      } else {
#pragma unroll
        for (int c = 0; c < HIPAD / 8; ++c) tc::tmem_ld32(lane_addr + g * HIPAD * 4 + c * 32,
                                                         *reinterpret_cast<uint32_t(*)[32]>(r + 32 * c));
      }
      float tot = 0.f;
#pragma unroll
      for (int h = 0; h < HIPAD; ++h) {
        const int nb = (g * HIPAD + h) * 4;
        float f[4];
#pragma unroll
        for (int p = 0; p < 4; ++p) f[p] = __int_as_float((int)r[h * 4 + p] + corr[nb + p]) - 12582912.0f;
        const float z = fmaf(fmaf(fmaf(f[3], 0.0078125f, f[2]), 0.0078125f, f[1]), 0.0078125f, f[0]);
        tot = fmaf(wq[g * HIPAD + h], fmaxf(z, 0.f), tot);
      }
      const bool vis = valid && j < nq[g];
      uint32_t key = vis ? score_key(sj * tot) : 0u;
      uint32_t* krow = a.keys + ((int64_t)b * a.Q + q0 + g) * a.key_stride;
      if (MODE == kHier) {
        for (int o = 1; o < a.block; o <<= 1) key = max(key, __shfl_xor_sync(0xffffffffu, key, o));
        if ((tid & (a.block - 1)) == 0 && i0 + tid < nq[g]) krow[(i0 + tid) / a.block] = key;
      } else if (i0 + tid < limit) {
        krow[i0 + tid] = key;
      }
    }
    tc::fence_before_sync();
  }
  if (timed_out && tid == 0) flag(a.status, CSA2_DEV_TIMEOUT);
  tc::cp_async_wait<0>();
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, a.tmem_cols);
  }
}

// ------------------------------------------------------------------------------------
// Top-K selection over one query's keys (one CTA of 1024 threads per query).
//
// Most-significant-digit radix select with digits of 11, 11 and 10 bits:
//   1. histogram the current digit of every key that matches the prefix chosen so far
//      (the first pass sees all keys) and find the bin T holding the need-th largest;
//      keys in bins above T are selected, need shrinks by their number;
//   2. as soon as bin T holds at most kCap keys, one ordered pass over the keys writes
//      the selected ones to the output in index order and copies bin T's keys (with their
//      indices, in index order) into shared memory, where the remaining digits are
//      resolved without touching global memory again;
//   3. keys equal to the K-th key are taken lowest index first.
// Every output position comes from a block-wide prefix sum, so the result (contents and
// order) is deterministic.
// ------------------------------------------------------------------------------------
constexpr int kSelThreads = 1024;
constexpr int kBins = 2048;
constexpr int kCap = 8192;          // shared-memory candidates
constexpr int kPer = 16;            // keys per thread per tile (4 x 16 B loads in flight)
constexpr int kSelSmem = kBins * 4 + kCap * 8 + 34 * 4 + 64;
static_assert(kSelThreads * kPer <= 65535, "packed 16-bit tile counts");

struct SelectArgs {
  const uint32_t* keys;
  int64_t key_stride;
  int mode;
  int Q, block, n_blocks, K;
  const int64_t* seq_base;
  const int32_t* n_vis;
  int64_t max_n_vis, pool_entries;
  const int32_t* blocks;
  int32_t* out_idx;
  float* out_score;
};

__device__ __forceinline__ int64_t item_label(const SelectArgs& a, int bq, int64_t i) {
  if (a.mode == kReindex) {
    const int32_t c = a.blocks[(int64_t)bq * a.n_blocks + i / a.block];
    return (int64_t)c * a.block + i % a.block;
  }
  return i;
}

// Block-wide exclusive prefix sum of one uint32 per thread (1024 threads); *total gets
// the sum.  ws must hold 33 words.
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, uint32_t* ws, uint32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) ws[warp] = x;
  __syncthreads();
  if (warp == 0) {
    const uint32_t w = ws[lane];
    uint32_t z = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, z, o);
      if (lane >= o) z += y;
    }
    ws[lane] = z - w;
    if (lane == 31) ws[32] = z;
  }
  __syncthreads();
  const uint32_t r = ws[warp] + x - v;
  *total = ws[32];
  __syncthreads();
  return r;
}

// Load keys [i0, i0+kPer) (zero past n); rows are 16-byte aligned and i0 % 4 == 0.
__device__ __forceinline__ void load_keys(const uint32_t* keys, int64_t i0, int64_t n, uint32_t (&k)[kPer]) {
  if (i0 + kPer <= n) {
#pragma unroll
    for (int v = 0; v < kPer / 4; ++v) {
      const uint4 a4 = *reinterpret_cast<const uint4*>(keys + i0 + 4 * v);
      k[4 * v] = a4.x;
      k[4 * v + 1] = a4.y;
      k[4 * v + 2] = a4.z;
      k[4 * v + 3] = a4.w;
    }
  } else {
#pragma unroll
    for (int e = 0; e < kPer; ++e) k[e] = (i0 + e < n) ? keys[i0 + e] : 0u;
  }
}

// Find the bin T of hist[0, nb) holding the need-th largest counted key.  Executed by
// warp 0; results in *T_out / *above_out (keys in bins above T).  Also returns the total.
__device__ __forceinline__ void find_bin(const uint32_t* hist, int nb, uint32_t need, uint32_t* T_out,
                                         uint32_t* above_out, uint32_t* total_out) {
  const int lane = threadIdx.x & 31;
  const int per = nb / 32;
  uint32_t run = 0;
  for (int i = 0; i < per; ++i) run += hist[lane * per + i];
  uint32_t suf = run;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_down_sync(0xffffffffu, suf, o);
    if (lane + o < 32) suf += y;
  }
  const uint32_t above_lane = suf - run;
  if (lane == 0) *total_out = suf;
  if (above_lane < need && suf >= need) {
    uint32_t acc = above_lane;
    for (int i = per - 1; i >= 0; --i) {
      const uint32_t h = hist[lane * per + i];
      if (acc + h >= need) {
        *T_out = lane * per + i;
        *above_out = acc;
        break;
      }
      acc += h;
    }
  }
}

__global__ void __launch_bounds__(kSelThreads) select_kernel(SelectArgs a) {
  extern __shared__ __align__(16) uint32_t sel_smem[];
  uint32_t* hist = sel_smem;                  // [kBins]
  uint32_t* cand_key = hist + kBins;          // [kCap]
  uint32_t* cand_idx = cand_key + kCap;       // [kCap]
  uint32_t* scan_ws = cand_idx + kCap;        // [33]
  uint32_t* s_misc = scan_ws + 34;            // T, above, total

  const int tid = threadIdx.x;
  const int bq = blockIdx.x;
  const int b = bq / a.Q;
  const int K = a.K;
  int32_t* out = a.out_idx + (int64_t)bq * K;
  float* out_s = a.out_score ? a.out_score + (int64_t)bq * K : nullptr;

  int64_t n;
  {
    const int64_t base = a.seq_base[b];
    int64_t nv = a.n_vis[bq];
    if (nv < 0 || nv > a.max_n_vis || base < 0 || base + nv > a.pool_entries) nv = 0;
    if (a.mode == kFlat)
      n = nv;
    else if (a.mode == kHier)
      n = (nv + a.block - 1) / a.block;
    else
      n = (int64_t)a.n_blocks * a.block;
  }
  const uint32_t* keys = a.keys + (int64_t)bq * a.key_stride;

  auto emit = [&](int pos, int64_t i, uint32_t k) {
    out[pos] = (int32_t)item_label(a, bq, i);
    if (out_s) out_s[pos] = key_score(k);
  };

  // ---- radix levels over global memory until the threshold bin fits in shared memory ----
  uint32_t prefix = 0, mask = 0, need = (uint32_t)K, inbin = 0;
  int level = 0;
  const int shifts[3] = {21, 10, 0};
  const int widths[3] = {11, 11, 10};
  for (;; ++level) {
    const int sh = shifts[level];
    const uint32_t nb = 1u << widths[level];
    for (int i = tid; i < kBins; i += kSelThreads) hist[i] = 0;
    __syncthreads();
    for (int64_t i0 = (int64_t)tid * kPer; i0 < n; i0 += (int64_t)kSelThreads * kPer) {
      uint32_t k[kPer];
      load_keys(keys, i0, n, k);
#pragma unroll
      for (int e = 0; e < kPer; ++e)
        if (k[e] != 0 && (k[e] & mask) == prefix) atomicAdd(&hist[(k[e] >> sh) & (nb - 1)], 1u);
    }
    __syncthreads();
    if (tid < 32) find_bin(hist, nb, need, &s_misc[0], &s_misc[1], &s_misc[2]);
    __syncthreads();
    if (level == 0 && s_misc[2] <= (uint32_t)K) break;  // everything valid is selected
    const uint32_t T = s_misc[0];
    need -= s_misc[1];
    prefix |= T << sh;
    mask |= (nb - 1) << sh;
    inbin = hist[T];
    __syncthreads();
    if (inbin <= (uint32_t)kCap || level == 2) break;
  }
  const bool all_valid = (mask == 0);

  // ---- one ordered pass: selected keys to the output, threshold-bin keys to smem --------
  // (all_valid: every non-zero key is selected; level 2 with a full-key tie: the first
  //  `need` equal keys are taken directly)
  const bool direct_ties = !all_valid && inbin > (uint32_t)kCap;
  uint32_t n_gt = 0, n_eq = 0;
  for (int64_t t0 = 0; t0 < n; t0 += (int64_t)kSelThreads * kPer) {
    const int64_t i0 = t0 + (int64_t)tid * kPer;
    uint32_t k[kPer];
    load_keys(keys, i0, n, k);
    uint32_t cg = 0, ce = 0;
#pragma unroll
    for (int e = 0; e < kPer; ++e) {
      const uint32_t kp = k[e] & mask;
      const bool valid = k[e] != 0;
      cg += (valid && (all_valid || kp > prefix)) ? 1u : 0u;
      ce += (valid && !all_valid && kp == prefix) ? 1u : 0u;
    }
    uint32_t tot;
    const uint32_t pos = block_excl_scan(cg | (ce << 16), scan_ws, &tot);
    uint32_t pg = n_gt + (pos & 0xFFFFu), pe = n_eq + (pos >> 16);
#pragma unroll
    for (int e = 0; e < kPer; ++e) {
      const uint32_t kp = k[e] & mask;
      const bool valid = k[e] != 0;
      if (valid && (all_valid || kp > prefix)) {
        emit((int)pg, i0 + e, k[e]);
        ++pg;
      } else if (valid && kp == prefix) {
        if (direct_ties) {
          if (pe < need) emit((int)(K - need + pe), i0 + e, k[e]);
        } else {
          cand_key[pe] = k[e];
          cand_idx[pe] = (uint32_t)(i0 + e);
        }
        ++pe;
      }
    }
    n_gt += tot & 0xFFFFu;
    n_eq += tot >> 16;
  }
  if (all_valid) {
    for (int i = (int)n_gt + tid; i < K; i += kSelThreads) {
      out[i] = -1;
      if (out_s) out_s[i] = -INFINITY;
    }
    return;
  }
  if (direct_ties) return;

  // ---- resolve the remaining digits among the shared-memory candidates -------------------
  const int cnt = (int)n_eq;
  __syncthreads();
  for (int lv = level + 1; lv < 3 && (uint32_t)cnt > need; ++lv) {
    const int sh = shifts[lv];
    const uint32_t nb = 1u << widths[lv];
    for (int i = tid; i < kBins; i += kSelThreads) hist[i] = 0;
    __syncthreads();
    for (int i = tid; i < cnt; i += kSelThreads) {
      const uint32_t k = cand_key[i];
      if ((k & mask) == prefix) atomicAdd(&hist[(k >> sh) & (nb - 1)], 1u);
    }
    __syncthreads();
    if (tid < 32) find_bin(hist, nb, need, &s_misc[0], &s_misc[1], &s_misc[2]);
    __syncthreads();
    const uint32_t T = s_misc[0];
    need -= s_misc[1];
    prefix |= T << sh;
    mask |= (nb - 1) << sh;
    const uint32_t in2 = hist[T];
    __syncthreads();
    if (in2 == need) break;
  }
  // candidates above the threshold prefix, then equal ones lowest index first (cand is
  // in index order)
  const uint32_t base_out = (uint32_t)K - need;  // first tie slot
  uint32_t g2 = n_gt, e2 = 0;
  for (int c0 = 0; c0 < cnt; c0 += kSelThreads * kPer) {
    const int i0 = c0 + tid * kPer;
    uint32_t cg = 0, ce = 0;
#pragma unroll
    for (int e = 0; e < kPer; ++e) {
      if (i0 + e < cnt) {
        const uint32_t kp = cand_key[i0 + e] & mask;
        cg += kp > prefix ? 1u : 0u;
        ce += kp == prefix ? 1u : 0u;
      }
    }
    uint32_t tot;
    const uint32_t pos = block_excl_scan(cg | (ce << 16), scan_ws, &tot);
    uint32_t pg = g2 + (pos & 0xFFFFu), pe = e2 + (pos >> 16);
#pragma unroll
    for (int e = 0; e < kPer; ++e) {
      if (i0 + e < cnt) {
        const uint32_t k = cand_key[i0 + e];
        const uint32_t kp = k & mask;
        if (kp > prefix) {
          emit((int)pg, cand_idx[i0 + e], k);
          ++pg;
        } else if (kp == prefix) {
          if (pe < need) emit((int)(base_out + pe), cand_idx[i0 + e], k);
          ++pe;
        }
      }
    }
    g2 += tot & 0xFFFFu;
    e2 += tot >> 16;
  }
}

// ------------------------------------------------------------------------------------
// host launchers
// ------------------------------------------------------------------------------------
static int pow2_at_least(int x) {
  int p = 32;
  while (p < x) p <<= 1;
  return p;
}

template <int MODE>
static cudaError_t launch_scan(ScanArgs a, int64_t items, int B, cudaStream_t st) {
  a.hipad = a.HI <= 4 ? 4 : (a.HI <= 8 ? 8 : 16);
  a.G = MODE == kReindex ? 1 : max(1, min(a.Q, 256 / (a.hipad * 4)));
  a.n_groups = (a.Q + a.G - 1) / a.G;
  a.N = a.G * a.hipad * 4;
  a.tmem_cols = pow2_at_least(a.N);
  a.tiles_per_cta = MODE == kReindex ? 2 : 8;
  const int64_t per_cta = (int64_t)a.tiles_per_cta * kRows;
  const dim3 grid((unsigned)((items + per_cta - 1) / per_cta), (unsigned)(B * a.n_groups));
  if (grid.x == 0 || grid.y == 0) return cudaSuccess;
  const size_t smem = 1024 + (size_t)kRows * 128 + (size_t)a.N * 128 + 2 * kRawBytes + (size_t)a.N * 4 +
                      (size_t)a.G * a.hipad * 4 + (size_t)a.G * 8 + 256 * 4 + 16;
  cudaError_t e;
#define CSA2_SCAN_LAUNCH(HP)                                                                        \
  e = cudaFuncSetAttribute(scan_tc_kernel<MODE, HP>, cudaFuncAttributeMaxDynamicSharedMemorySize, \
                           (int)smem);                                                              \
  if (e != cudaSuccess) return e;                                                                   \
  scan_tc_kernel<MODE, HP><<<grid, kScanThreads, smem, st>>>(a);
  if (a.hipad == 4) {
    CSA2_SCAN_LAUNCH(4)
  } else if (a.hipad == 8) {
    CSA2_SCAN_LAUNCH(8)
  } else {
    CSA2_SCAN_LAUNCH(16)
  }
#undef CSA2_SCAN_LAUNCH
  return cudaGetLastError();
}

cudaError_t launch_index(int mode, const float* q, const float* w, const uint8_t* ik_pool,
                         int64_t pool_entries, const int64_t* seq_base, const int32_t* n_vis,
                         const int32_t* blocks, int B, int Q, int HI, int n_blocks, int block,
                         int K, int64_t max_n_vis, int32_t* out_idx, float* out_score,
                         uint32_t* keys, int64_t key_stride, uint32_t* status,
                         cudaStream_t stream) {
  ScanArgs a;
  a.q = q;
  a.w = w;
  a.ik_pool = ik_pool;
  a.pool_entries = pool_entries;
  a.seq_base = seq_base;
  a.n_vis = n_vis;
  a.blocks = blocks;
  a.Q = Q;
  a.HI = HI;
  a.n_blocks = n_blocks;
  a.block = block;
  a.max_n_vis = max_n_vis;
  a.key_stride = key_stride;
  a.keys = keys;
  a.status = status;
  const int BQ = B * Q;
  if (BQ == 0) return cudaSuccess;
  cudaError_t e;
  if (mode == kFlat)
    e = launch_scan<kFlat>(a, max_n_vis, B, stream);
  else if (mode == kHier)
    e = launch_scan<kHier>(a, max_n_vis, B, stream);
  else
    e = launch_scan<kReindex>(a, (int64_t)n_blocks * block, B * Q, stream);
  if (e != cudaSuccess) return e;

  SelectArgs s;
  s.keys = keys;
  s.key_stride = key_stride;
  s.mode = mode;
  s.Q = Q;
  s.block = block;
  s.n_blocks = n_blocks;
  s.K = K;
  s.seq_base = seq_base;
  s.n_vis = n_vis;
  s.max_n_vis = max_n_vis;
  s.pool_entries = pool_entries;
  s.blocks = blocks;
  s.out_idx = out_idx;
  s.out_score = out_score;
  e = cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSelSmem);
  if (e != cudaSuccess) return e;
  select_kernel<<<BQ, kSelThreads, kSelSmem, stream>>>(s);
  return cudaGetLastError();
}

}  // namespace csa2
