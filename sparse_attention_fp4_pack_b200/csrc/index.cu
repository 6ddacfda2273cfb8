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
// The streaming scan (stream_scan_kernel: flat and hierarchical) computes the dot products
// on the tensor cores as tcgen05.mma kind::f16 (f16 operands, fp32 accumulation):
//   * A (128 entries x 128 dims, f16, in tensor memory): the key's E2M1 values themselves,
//     which f16 holds exactly (the hardware's e2m1x2 -> f16x2 conversion, 8 codes per four
//     instructions); each thread stores its entry's row into its own lane.
//   * B (N rows x 128 dims, f16, twice): each query head h is scaled by the power of two
//     S_h = 2^(14 - exponent(max|q_h|)), so x = q*S_h is exact with |x| < 2^15, and split
//     into hi = f16(x) and lo = f16(x - hi), which represent x to 2^-22 of each element.
//   * D (128 x N, fp32): the MMAs of hi and lo accumulate into the same columns, so D holds
//     sum_d c_d (hi_d + lo_d) = S_h (q_h . c_j) with every product exact (2 x 11 significant
//     bits) and fp32 sums; the epilogue applies the ReLU, the weights w_h / S_h and the key's
//     scale.
// The Reindex scan (reindex_scan_kernel: one tile per CTA, so its MMA chain is on the
// critical path) uses tcgen05.mma kind::i8, whose K = 32 per instruction halves that chain:
//   * A (128 entries x 128 dims, u8, shared memory): u = 2c + 12 in [0, 24] — the E2M1 value
//     doubled and offset to be non-negative; two byte-permutes per 4 codes build it
//     (sign-replicate selects the positive or negative table).
//   * B (N rows x 128 dims, s8): each query head h is scaled by the power of two
//     S_h = 2^(5 - exponent(max|q_h|)), so x = q*S_h is exact with |x| < 64, and split into
//     four int8 limbs x = L0 + L1/128 + L2/128^2 + L3/128^3 (error below 2^-22).
//   * D (128 x N, s32): acc_p = sum_d u_d L_p,d, so sum_d c_d L_p,d = (acc_p - 12 T_p)/2
//     with T_p = sum_d L_p,d; the epilogue removes the offset exactly in integers and
//     combines the limbs in fp32: q_h . c_j = (sum_p 128^-p (acc_p - 12 T_p)) / (2 S_h).
// One thread owns one tile row (entry) end to end: it builds the row's A operand, and
// after the MMA reads the same TMEM lane and writes the entry's order-preserving uint32
// key (hierarchical mode: the max over `block` neighbouring lanes).  The streaming scan
// takes a group of queries of one sequence per CTA (multi-query verify and prefill: 4 of
// 8 heads), so the A operand is built once for the group.
#include <algorithm>
#include <cooperative_groups.h>
#include <cuda_fp16.h>

#include "csa2_device.cuh"
#include "tc.cuh"

namespace csa2 {

// kMerge: selection only, over caller-built keys and labels (the merge of several lists)
enum ScanMode : int { kFlat = 0, kHier = 1, kReindex = 2, kMerge = 3 };

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
  int block_shift;        // log2(block)
  int N;                  // MMA N = G * hipad rounded up to 16
  int tmem_cols;
  int tiles_per_cta;
  int64_t max_n_vis;
  int64_t key_stride;
  uint32_t* keys;
  uint32_t* gmax;         // flat, may be null: the largest key of every 32 keys, per query row
  int64_t gstride;        // gmax words per query row
  uint32_t* status;
  int withheld_tile;      // test hook: the first CTA never copies this tile (-1: off)
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

constexpr int kATmemCols = 64;       // an A tile in tensor memory: 128 f16 per lane, two per column

// The B rows of one query head, from the head's 128 fp32 elements (lane l holds elements
// 4l..4l+3; zeros for a padding row).  x = q*S with S = 2^(14 - exponent(max|q|)), so
// |x| < 2^15 and the scaling is exact; hi = f16(x) and lo = f16(x - hi) (x - hi is exact in
// fp32) represent x to 2^-22 of each element.  hi goes to row n of the operand at Bs and lo to
// row n_lo of the operand at Blo (the same operand when the two are stacked along N); an
// operand is two 128-byte-swizzled K-halves of npad rows (elements 0..63 and 64..127).
// Returns 1/S (0 for a head whose largest element is below 1e-30).
__device__ __forceinline__ float build_b_head(uint8_t* Bs, uint8_t* Blo, int npad, int n, int n_lo, float4 v) {
  const int lane = threadIdx.x & 31;
  float m = fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w)));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  float S = 0.f, inv = 0.f;
  if (m > 1e-30f) {
    const int E = (int)((__float_as_uint(m) >> 23) & 0xFFu) - 127;
    S = __uint_as_float((uint32_t)(127 + 14 - E) << 23);
    inv = __uint_as_float((uint32_t)(127 - 14 + E) << 23);
  }
  const float x[4] = {v.x * S, v.y * S, v.z * S, v.w * S};
  uint32_t hw[2], lw[2];
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    const __half2 h = __floats2half2_rn(x[2 * e], x[2 * e + 1]);
    const float2 hf = __half22float2(h);
    const __half2 l = __floats2half2_rn(x[2 * e] - hf.x, x[2 * e + 1] - hf.y);
    hw[e] = *reinterpret_cast<const uint32_t*>(&h);
    lw[e] = *reinterpret_cast<const uint32_t*>(&l);
  }
  const uint32_t kh = (uint32_t)(lane >> 4) * (uint32_t)npad * 128u, byte = (uint32_t)(lane & 15) * 8u;
  *reinterpret_cast<uint2*>(Bs + kh + tc::sw128((uint32_t)n, byte)) = make_uint2(hw[0], hw[1]);
  *reinterpret_cast<uint2*>(Blo + kh + tc::sw128((uint32_t)n_lo, byte)) = make_uint2(lw[0], lw[1]);
  return inv;
}

// The MMAs of one tile: A (its 128 x 128 f16 in tensor memory, 64 columns from a_tmem) times
// `parts` B operands at b_addr (each two swizzled K-halves of npad rows: hi and then lo, or one
// operand holding both), all accumulating into the npad columns at d; 8 MMAs per operand.
__device__ __forceinline__ void issue_tile_mma(uint32_t d, uint32_t a_tmem, uint32_t b_addr, int npad, int parts,
                                               uint32_t idesc) {
  const uint32_t bh = (uint32_t)npad * 128u;  // one K-half of one B operand
  const uint64_t b0 = tc::smem_desc_sw128(b_addr, 16, 1024);
  for (int p = 0; p < parts; ++p)
#pragma unroll
    for (int kh = 0; kh < 2; ++kh)
#pragma unroll
      for (int ks = 0; ks < 4; ++ks)  // 16 elements per MMA: 8 columns of A, 32 B of a B row
        tc::mma_f16_ts(d, a_tmem + (uint32_t)(kh * 32 + ks * 8),
                       tc::desc_add(b0, (uint32_t)(2 * p + kh) * bh + (uint32_t)ks * 32u), idesc,
                       (p | kh | ks) ? 1u : 0u);
}

// One entry's A row: its 128 E2M1 codes (16 words at ea in shared memory; zeros when !valid)
// as f16 pairs into 64 columns of this thread's tensor-memory lane from taddr, then the wait
// for the stores.  Warp-wide: every lane of the warp calls it.
__device__ __forceinline__ void build_a_row(uint32_t taddr, uint32_t ea, bool valid) {
  uint32_t cw[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) cw[i] = valid ? tc::ld_shared_u32(ea + 4u * (uint32_t)i) : 0u;
  uint32_t o0[32], o1[32];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint4 h0 = e2m1x8_f16(cw[i]), h1 = e2m1x8_f16(cw[8 + i]);
    o0[4 * i] = h0.x;
    o0[4 * i + 1] = h0.y;
    o0[4 * i + 2] = h0.z;
    o0[4 * i + 3] = h0.w;
    o1[4 * i] = h1.x;
    o1[4 * i + 1] = h1.y;
    o1[4 * i + 2] = h1.z;
    o1[4 * i + 3] = h1.w;
  }
  tc::tmem_st32_nowait(taddr, o0);
  tc::tmem_st32_nowait(taddr + 32u, o1);
  tc::tmem_wait_st();
}

// Reindex scan: one CTA row per (sequence, query), each CTA scoring kRows-candidate tiles
// gathered from the query's block list (128 / block blocks of `block` consecutive keys per
// tile, staged by cp.async one tile ahead).
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

template <int HIPAD>
__global__ void __launch_bounds__(kScanThreads) reindex_scan_kernel(ScanArgs a) {
  chain_launch_dependents();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = tc::align_smem_1024(smem_raw);
  uint8_t* As = sm;                                   // [128 rows x 128 B], 128 B swizzle
  uint8_t* Bs = As + kRows * 128;                     // [N rows x 128 B]
  uint8_t* raw = Bs + a.N * 128;                      // 2 x kRawBytes
  int32_t* corr = reinterpret_cast<int32_t*>(raw + 2 * kRawBytes);  // [N]
  float* wq = reinterpret_cast<float*>(corr + a.N);                 // [HIPAD]
  int32_t* segc = reinterpret_cast<int32_t*>(wq + HIPAD);           // [2][128] gathered block ids
  uint64_t* mbar = reinterpret_cast<uint64_t*>(segc + 256);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mbar + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bq = blockIdx.y;  // (sequence, query) of this CTA row
  const int b = bq / a.Q;
  const int64_t limit = (int64_t)a.n_blocks * a.block;  // candidate slots
  const int64_t item0 = (int64_t)blockIdx.x * a.tiles_per_cta * kRows;
  if (item0 >= limit) return;
  const int64_t left_tiles = (limit - item0 + kRows - 1) / kRows;
  const int ntiles = (int)(left_tiles < a.tiles_per_cta ? left_tiles : a.tiles_per_cta);
  // set-up that touches no global memory runs while the predecessor finishes
  if (warp == 0) tc::tmem_alloc(tc::smem_u32(tmem_slot), a.tmem_cols);
  if (tid == 32) tc::mbar_init(tc::smem_u32(mbar), 1);
  // The B operand (the indexer queries and head weights: caller inputs that no library call
  // writes) is built while the predecessor finishes; a warp takes HIPAD / 4 heads.
  constexpr int kHeadsPerWarp = HIPAD / (kScanThreads / 32);
  float4 qpre[kHeadsPerWarp];
  float wpre[kHeadsPerWarp];
#pragma unroll
  for (int k = 0; k < kHeadsPerWarp; ++k) {
    const int h = warp + k * (kScanThreads / 32);
    qpre[k] = make_float4(0.f, 0.f, 0.f, 0.f);
    wpre[k] = 0.f;
    if (h < a.HI) {
      qpre[k] = reinterpret_cast<const float4*>(a.q + ((int64_t)bq * a.HI + h) * kDI)[lane];
      wpre[k] = a.w[(int64_t)bq * a.HI + h];
    }
  }
  // ---- B operand: four int8 limbs of every head, plus epilogue constants ----------------
#pragma unroll
  for (int k = 0; k < kHeadsPerWarp; ++k) {
    const int h = warp + k * (kScanThreads / 32);
    const float x[4] = {qpre[k].x, qpre[k].y, qpre[k].z, qpre[k].w};
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
      const int n = h * 4 + p;
      *reinterpret_cast<uint32_t*>(Bs + tc::sw128(n, lane * 4)) = limb[p];
      int t = lsum[p];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
      if (lane == 0) corr[n] = 0x4B400000 - 12 * t;
    }
    if (lane == 0) wq[h] = S > 0.f ? wpre[k] / (2.0f * S) : 0.f;
  }
  tc::fence_async_smem();
  chain_wait();
  const int64_t nvis = valid_count(a, b, bq, blockIdx.x == 0);  // 0 if the count is bad

  const uint8_t* seq = a.ik_pool + a.seq_base[b] * kIkBytes;
  const uint32_t raw_a = tc::smem_u32(raw);
  // a tile's 128 / block gathered blocks, each staged at seg_stride (a 16 B multiple)
  const int seg_stride = ((a.block * kIkBytes + 16) + 15) & ~15;

  // gathered tile loader: tile ti into buffer ti & 1; `block` threads copy each block
  auto load_tile = [&](int ti) {
    const int64_t i0 = item0 + (int64_t)ti * kRows;
    const uint32_t dst = raw_a + (ti & 1) * kRawBytes;
    const int s = tid >> a.block_shift, sub = tid & (a.block - 1);
    const int64_t slot_blk = (i0 >> a.block_shift) + s;
    int32_t c = -1;
    if (slot_blk < a.n_blocks) c = a.blocks[(int64_t)bq * a.n_blocks + slot_blk];
    if (sub == 0) {
      segc[(ti & 1) * 128 + s] = c;
      if (c < -1) flag(a.status, CSA2_DEV_BAD_INDEX);
    }
    int cnt = 0;
    if (c >= 0) {
      const int64_t rem = nvis - (int64_t)c * a.block;
      cnt = rem <= 0 ? 0 : (int)(rem < a.block ? rem : a.block);
    }
    if (cnt > 0) {
      // a block starts at its own address residue mod 16 unless block*68 is a 16 B multiple
      const uint8_t* src = seq + (int64_t)c * a.block * kIkBytes;
      const int smis = (int)(reinterpret_cast<uintptr_t>(src) & 15u);
      stage_async(dst + s * seg_stride + smis, src, cnt * kIkBytes, sub, a.block);
    }
    tc::cp_async_commit();
  };

  load_tile(0);

  tc::fence_async_smem();
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  const uint32_t idesc = tc::idesc_i8(kRows, a.N, false, true);
  const uint32_t lane_addr = tmem + ((uint32_t)(warp * 32) << 16);
  uint32_t* krow = a.keys + (int64_t)bq * a.key_stride;
  bool timed_out = false;

  for (int ti = 0; ti < ntiles; ++ti) {
    if (ti + 1 < ntiles) load_tile(ti + 1);
    else tc::cp_async_commit();  // keep the group count uniform
    tc::cp_async_wait<1>();
    __syncthreads();
    const int64_t i0 = item0 + (int64_t)ti * kRows;
    // ---- this thread's row: locate the candidate, build the A row ------------------------
    const int s = tid >> a.block_shift, r = tid & (a.block - 1);
    const int32_t c = segc[(ti & 1) * 128 + s];
    const int64_t j = (int64_t)c * a.block + r;  // entry index within the sequence
    const bool valid = c >= 0 && j < nvis;
    float sj = 0.f;
    if (valid) {
      const int smis = (int)(reinterpret_cast<uintptr_t>(seq + (int64_t)c * a.block * kIkBytes) & 15u);
      const uint32_t* ew =
          reinterpret_cast<const uint32_t*>(raw + (ti & 1) * kRawBytes + s * seg_stride + smis + r * kIkBytes);
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
    uint32_t acc[HIPAD * 4];
    if (HIPAD == 4) {
      tc::tmem_ld16(lane_addr, acc);
    } else {
#pragma unroll
      for (int c32 = 0; c32 < HIPAD / 8; ++c32)
        tc::tmem_ld32(lane_addr + c32 * 32, *reinterpret_cast<uint32_t(*)[32]>(acc + 32 * c32));
    }
    float tot = 0.f;
#pragma unroll
    for (int h = 0; h < HIPAD; ++h) {
      float f[4];
#pragma unroll
      for (int p = 0; p < 4; ++p) f[p] = __int_as_float((int)acc[h * 4 + p] + corr[h * 4 + p]) - 12582912.0f;
      const float z = fmaf(fmaf(fmaf(f[3], 0.0078125f, f[2]), 0.0078125f, f[1]), 0.0078125f, f[0]);
      tot = fmaf(wq[h], fmaxf(z, 0.f), tot);
    }
    if (i0 + tid < limit) krow[i0 + tid] = valid ? score_key(sj * tot) : 0u;
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
// Streaming scan for the flat and hierarchical modes.  A CTA walks a contiguous run of
// tiles of one sequence:
//   * the copy warp (warp 4) moves each tile (128 consecutive 68 B keys) with one bulk
//     copy into a ring of kStages raw buffers, up to kStages tiles ahead of the math; the
//     copy starts at the 16 B boundary at or below the tile's first key (that lead,
//     0..12 bytes, is the same for every tile of a sequence) and is rounded up to 16 B,
//     falling back to word copies when the rounded copy would run past the pool.  It also
//     issues each tile's MMAs once the workers report the tile's A rows built;
//   * the four worker warps own one tile row each.  The accumulator is doubled: once tile
//     t's MMAs have completed (they free the A tile in tensor memory), the workers build
//     tile t+1's rows and report them, then run tile t's epilogue while tile t+1's MMAs run.
//     No worker issues MMAs, so none lags the others at the per-tile vote.
// Four CTAs share an SM (tensor memory: the A tile and the accumulator pair, at most 128
// columns).  Every wait is bounded; the workers agree on giving up through a reducing
// barrier and tell the copy warp, and the copy warp waits for its outstanding copies and
// MMAs before the CTA exits.
// ------------------------------------------------------------------------------------
constexpr int kStreamWorkers = 128;                       // one tile row per thread
constexpr int kStreamThreads = kStreamWorkers + 32;       // plus the copy warp
constexpr int kStages = 4;                                // raw tiles in flight per CTA
constexpr int kRawTile = kRows * kIkBytes + 16;           // one tile plus its lead, 16 B multiple
constexpr int kWorkerBar = 1;                             // named barrier of the workers
constexpr int kStreamN = 32;                              // largest MMA N: G * HIPAD, rounded up to 16

template <int MODE, int HIPAD>
__global__ void __launch_bounds__(kStreamThreads, 4) stream_scan_kernel(ScanArgs a) {
  chain_enter();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = tc::align_smem_1024(smem_raw);
  uint8_t* Bs = sm;                                   // hi, lo x 2 K-halves x [N rows x 128 B]
  uint8_t* raw = Bs + 4 * a.N * 128;                  // kStages x kRawTile
  float* wq = reinterpret_cast<float*>(raw + kStages * kRawTile);        // [N] head weight / S
  int64_t* nq = reinterpret_cast<int64_t*>(wq + a.N);                    // [G] visible count per query
  uint64_t* full = reinterpret_cast<uint64_t*>(nq + a.G);                // [kStages] raw tile landed
  uint64_t* empty = full + kStages;                                      // [kStages] raw tile consumed
  uint64_t* dfull = empty + kStages;                                     // [2] accumulator ready
  uint64_t* built = dfull + 2;                                           // the A tile is built
  uint32_t* misc = reinterpret_cast<uint32_t*>(built + 1);  // tmem base, tiles consumed, copied, stop, issued

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int b = blockIdx.y / a.n_groups;
  const int gidx = blockIdx.y % a.n_groups;
  const int q0 = gidx * a.G;
  const int G = min(a.G, a.Q - q0);

  if (blockIdx.x == 0 && tid < G) valid_count(a, b, b * a.Q + q0 + tid, true);  // report bad counts once
  int64_t limit = 0;
  for (int g = 0; g < G; ++g) {
    const int64_t n = valid_count(a, b, b * a.Q + q0 + g, false);
    limit = n > limit ? n : limit;
  }
  const int64_t item0 = (int64_t)blockIdx.x * a.tiles_per_cta * kRows;
  if (item0 >= limit) return;
  const int64_t left_tiles = (limit - item0 + kRows - 1) / kRows;
  const int ntiles = (int)(left_tiles < a.tiles_per_cta ? left_tiles : a.tiles_per_cta);
  if (tid < G) nq[tid] = valid_count(a, b, b * a.Q + q0 + tid, false);

  const uint8_t* seq = a.ik_pool + a.seq_base[b] * kIkBytes;
  const uint32_t lead = (uint32_t)(reinterpret_cast<uintptr_t>(seq) & 15u);
  const uint32_t raw_a = tc::smem_u32(raw);
  const uint32_t full_a = tc::smem_u32(full), empty_a = tc::smem_u32(empty), dfull_a = tc::smem_u32(dfull);

  if (warp == 0) tc::tmem_alloc(tc::smem_u32(misc), a.tmem_cols);
  if (tid == 32) {
    for (int s = 0; s < kStages; ++s) {
      tc::mbar_init(full_a + 8 * s, 1);
      tc::mbar_init(empty_a + 8 * s, kStreamWorkers);
    }
    tc::mbar_init(dfull_a, 1);
    tc::mbar_init(dfull_a + 8, 1);
    tc::mbar_init(tc::smem_u32(built), 1);
  }

  // ---- B operands: hi and lo f16 rows of every (query, head), zero padding rows ----------
  // One query (G = 1): hi in rows [0, HIPAD) and lo in rows [HIPAD, 2 HIPAD) of one operand,
  // filling N's padding, so a tile takes 8 MMAs; else the hi and lo operands, 16 MMAs.
  const bool stacked = a.G == 1;
  const int nb = stacked ? HIPAD : a.N;  // B rows built from heads
  for (int gh = warp; gh < nb; gh += kStreamThreads / 32) {
    const int g = gh / HIPAD, h = gh % HIPAD;
    const bool live = g < G && h < a.HI;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    float wv = 0.f;
    if (live) {
      const int64_t bq = (int64_t)b * a.Q + q0 + g;
      v = reinterpret_cast<const float4*>(a.q + (bq * a.HI + h) * kDI)[lane];
      wv = a.w[bq * a.HI + h];
    }
    const float inv = stacked ? build_b_head(Bs, Bs, a.N, gh, HIPAD + gh, v)
                              : build_b_head(Bs, Bs + 2 * a.N * 128, a.N, gh, gh, v);
    if (lane == 0) wq[gh] = 0.5f * wv * inv;  // halved: the epilogue weighs z + |z| = 2 max(z, 0)
  }
  if (stacked)  // rows [2 HIPAD, N) of both K-halves are zero
    for (int i = tid; i < 2 * (a.N - 2 * HIPAD) * 32; i += kStreamThreads) {
      const int kh = i / ((a.N - 2 * HIPAD) * 32), rest = i % ((a.N - 2 * HIPAD) * 32);
      *reinterpret_cast<uint32_t*>(Bs + kh * a.N * 128 + (2 * HIPAD + rest / 32) * 128 + (rest % 32) * 4) = 0u;
    }
  tc::fence_async_smem();
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = misc[0];

  const uint32_t built_a = tc::smem_u32(built);
  const uint32_t idesc = tc::idesc_f16(kRows, a.N, false, false);
  if (warp == kStreamWorkers / 32) {
    // ---- copy and MMA warp ------------------------------------------------------------------
    // Tile t's MMAs go out once the workers report its A tile built; that report also frees
    // its raw buffer, so tile t + kStages is copied right after.
    const uint8_t* pool_end = a.ik_pool + a.pool_entries * kIkBytes;
    int copied = 0, mma_issued = 0;
    bool ok = true, withheld = false;
    auto copy_tile = [&](int t) -> bool {
      // test hook: stop copying, so the workers' wait for this tile runs out
      if (t == a.withheld_tile && blockIdx.x == 0 && blockIdx.y == 0) withheld = true;
      if (withheld) return true;
      const int s = t % kStages;
      bool cok = true;
      if (t >= kStages) cok = tc::mbar_wait(empty_a + 8 * s, (uint32_t)((t / kStages) - 1) & 1u, kScanPolls);
      if (!__all_sync(0xffffffffu, cok)) return false;
      const int64_t i0 = item0 + (int64_t)t * kRows;
      const int cnt = (int)(limit - i0 < kRows ? limit - i0 : kRows);
      const uint8_t* src = seq + i0 * kIkBytes;
      const uint32_t nbytes = (lead + (uint32_t)cnt * kIkBytes + 15u) & ~15u;
      if (src - lead + nbytes <= pool_end) {
        if (lane == 0) {
          tc::mbar_arrive_expect_tx(full_a + 8 * s, nbytes);
          tc::bulk_g2s(raw_a + s * kRawTile, src - lead, nbytes, full_a + 8 * s);
        }
      } else {  // the tile ends within 16 B of the pool's end
        const uint32_t* sw = reinterpret_cast<const uint32_t*>(src);
        uint32_t* dw = reinterpret_cast<uint32_t*>(raw + s * kRawTile + lead);
        for (int k = lane; k < cnt * (kIkBytes / 4); k += 32) dw[k] = sw[k];
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(full_a + 8 * s);
      }
      copied = t + 1;
      return true;
    };
    for (int t = 0; t < ntiles && t < kStages && ok; ++t) ok = copy_tile(t);
    for (int t = 0; t < ntiles && ok; ++t) {
      ok = __all_sync(0xffffffffu, tc::mbar_wait(built_a, (uint32_t)t & 1u, kScanPolls));
      if (!ok || misc[3] != 0u) break;  // no report, or the workers gave up
      if (lane == 0) {
        tc::fence_after_sync();
        issue_tile_mma(tmem + (uint32_t)(kATmemCols + (t & 1) * a.N), tmem, tc::smem_u32(Bs), a.N,
                       a.G == 1 ? 1 : 2, idesc);
        tc::commit(dfull_a + 8u * (uint32_t)(t & 1));
      }
      mma_issued = t + 1;
      __syncwarp();
      if (t + kStages < ntiles) ok = copy_tile(t + kStages);
    }
    if (lane == 0) {
      if (!ok) flag(a.status, CSA2_DEV_TIMEOUT);
      misc[2] = (uint32_t)copied;
      misc[4] = (uint32_t)mma_issued;
    }
  } else {
    // ---- workers ----------------------------------------------------------------------------
    const int row = tid;
    // tensor memory: the A tile in columns [0, 64), accumulator u in [64 + u*N, 64 + (u+1)*N)
    const uint32_t lane_addr = tmem + ((uint32_t)(warp * 32) << 16);
    const uint32_t wq_a = tc::smem_u32(wq), nq_a = tc::smem_u32(nq);

    // build tile t's A row from its raw buffer (the previous tile's MMAs have completed);
    // false if the copy never landed
    auto build = [&](int t, float& sj, bool& valid) -> bool {
      const int s = t % kStages;
      const bool ok = tc::mbar_wait(full_a + 8 * s, (uint32_t)(t / kStages) & 1u, kScanPolls);
      const int64_t j = item0 + (int64_t)t * kRows + row;
      valid = ok && j < limit;
      const uint32_t ea = raw_a + s * kRawTile + lead + row * kIkBytes;
      build_a_row(lane_addr, ea, valid);
      sj = valid ? __uint_as_float(tc::ld_shared_u32(ea + 64)) : 0.f;
      if (ok) tc::mbar_arrive(empty_a + 8 * s);
      tc::fence_before_sync();
      return ok;
    };
    // report tile t's A tile built (after the workers' vote, which orders their tensor-memory
    // stores before it), or that the workers gave up
    auto report = [&](bool give_up) {
      if (tid == 0) {
        misc[3] = give_up ? 1u : 0u;
        tc::mbar_arrive(built_a);
      }
    };
    // dot products -> ReLU-weighted score -> order-preserving keys of tile t
    auto epilogue = [&](int t, float sj, bool valid) -> bool {
      const bool ok = tc::mbar_wait(dfull_a + 8u * (uint32_t)(t & 1), (uint32_t)(t >> 1) & 1u, kScanPolls);
      tc::fence_after_sync();
      const int64_t j = item0 + (int64_t)t * kRows + row;
      const uint32_t acc = lane_addr + (uint32_t)(kATmemCols + (t & 1) * a.N);
      uint32_t r[kStreamN];
      if (a.N == 16)
        tc::tmem_ld16(acc, r);
      else
        tc::tmem_ld32(acc, r);
      constexpr int kGmax = kStreamN / HIPAD;
#pragma unroll
      for (int g = 0; g < kGmax; ++g) {
        if (g >= G) break;
        // w * max(z, 0) as (w / 2) * (z + |z|): z + |z| is 2z or 0 exactly and w / 2 exact, so
        // the products are the same, on the FMA pipe instead of a max on the ALU pipe (the
        // weights in shared memory are already halved)
        float tot = 0.f;
        if (stacked) {  // one query: head h's hi sum in column h, its lo sum in column HIPAD + h
#pragma unroll
          for (int h4 = 0; h4 < HIPAD / 4; ++h4) {
            const uint4 w4 = tc::ld_shared_v4(wq_a + (uint32_t)(h4 * 4) * 4u);
            const int c = h4 * 4;
            const float z0 = __uint_as_float(r[c + 0]) + __uint_as_float(r[HIPAD + c + 0]);
            const float z1 = __uint_as_float(r[c + 1]) + __uint_as_float(r[HIPAD + c + 1]);
            const float z2 = __uint_as_float(r[c + 2]) + __uint_as_float(r[HIPAD + c + 2]);
            const float z3 = __uint_as_float(r[c + 3]) + __uint_as_float(r[HIPAD + c + 3]);
            tot = fmaf(__uint_as_float(w4.x), z0 + fabsf(z0), tot);
            tot = fmaf(__uint_as_float(w4.y), z1 + fabsf(z1), tot);
            tot = fmaf(__uint_as_float(w4.z), z2 + fabsf(z2), tot);
            tot = fmaf(__uint_as_float(w4.w), z3 + fabsf(z3), tot);
          }
        } else {
#pragma unroll
          for (int h4 = 0; h4 < HIPAD / 4; ++h4) {
            const uint4 w4 = tc::ld_shared_v4(wq_a + (uint32_t)(g * HIPAD + h4 * 4) * 4u);
            const int c = g * HIPAD + h4 * 4;
            const float z0 = __uint_as_float(r[c + 0]), z1 = __uint_as_float(r[c + 1]);
            const float z2 = __uint_as_float(r[c + 2]), z3 = __uint_as_float(r[c + 3]);
            tot = fmaf(__uint_as_float(w4.x), z0 + fabsf(z0), tot);
            tot = fmaf(__uint_as_float(w4.y), z1 + fabsf(z1), tot);
            tot = fmaf(__uint_as_float(w4.z), z2 + fabsf(z2), tot);
            tot = fmaf(__uint_as_float(w4.w), z3 + fabsf(z3), tot);
          }
        }
        const int64_t nqg = (int64_t)tc::ld_shared_u64(nq_a + 8u * (uint32_t)g);
        const bool vis = valid && j < nqg;
        uint32_t key = vis ? score_key(sj * tot) : 0u;
        uint32_t* krow = a.keys + ((int64_t)b * a.Q + q0 + g) * a.key_stride;
        if (MODE == kHier) {
          for (int o = 1; o < a.block; o <<= 1) key = max(key, __shfl_xor_sync(0xffffffffu, key, o));
          if ((row & (a.block - 1)) == 0 && j < nqg) krow[j >> a.block_shift] = key;
        } else {
          if (j < limit) krow[j] = key;
          if (a.gmax != nullptr) {  // the largest key of this warp's 32 rows
            const uint32_t m = __reduce_max_sync(0xffffffffu, key);
            if ((row & 31) == 0 && j < limit) a.gmax[((int64_t)b * a.Q + q0 + g) * a.gstride + (j >> 5)] = m;
          }
        }
      }
      tc::fence_before_sync();
      return ok;
    };

    // step t: once tile t's MMAs have completed (they free the A tile), build tile t+1 and
    // report it to the MMA warp, then run the epilogue of tile t while tile t+1's MMAs run
    float sj = 0.f, sj_nxt = 0.f;
    bool v = false, v_nxt = false;
    int consumed = 0;  // tiles whose raw buffers every worker has read
    bool bad = tc::named_sync_or(kWorkerBar, kStreamWorkers, !build(0, sj, v));
    report(bad);
    if (!bad) consumed = 1;
    bool pend = false;  // a failed accumulator wait, voted on at the next barrier
    for (int t = 0; t < ntiles && !bad; ++t) {
      if (t + 1 < ntiles) {
        const bool mok = tc::mbar_wait(dfull_a + 8u * (uint32_t)(t & 1), (uint32_t)(t >> 1) & 1u, kScanPolls);
        tc::fence_after_sync();
        const bool bok = build(t + 1, sj_nxt, v_nxt);  // warp-wide: every worker builds
        bad = tc::named_sync_or(kWorkerBar, kStreamWorkers, !mok || !bok || pend);
        report(bad);
        if (bad) break;
        consumed = t + 2;
      }
      pend |= !epilogue(t, sj, v);
      sj = sj_nxt;
      v = v_nxt;
    }
    // every worker reaches this vote: either all completed the loop or all left it together
    bad = tc::named_sync_or(kWorkerBar, kStreamWorkers, bad || pend);
    if (tid == 0) {
      if (bad) flag(a.status, CSA2_DEV_TIMEOUT);
      misc[1] = (uint32_t)(bad ? consumed : ntiles);
    }
  }
  __syncthreads();
  if (tid == kStreamWorkers) {
    // the last issued MMAs finish before the accumulators go (they complete in order; no later
    // commit on that barrier, so its phase is still the one to wait for)
    const int last = (int)misc[4] - 1;
    if (last >= 0) tc::mbar_wait(dfull_a + 8u * (uint32_t)(last & 1), (uint32_t)(last >> 1) & 1u, kScanPolls);
    for (int t = (int)misc[1]; t < (int)misc[2]; ++t)  // copies that landed in no consumed tile
      tc::mbar_wait(full_a + 8 * (t % kStages), (uint32_t)(t / kStages) & 1u, kScanPolls);
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, a.tmem_cols);
  }
}

// ------------------------------------------------------------------------------------
// Top-K selection over one query's keys: a thread-block cluster of C CTAs (C <= 8) per
// query, each holding a contiguous slice of the keys in shared memory (1024 threads x
// 2^PS keys, index order = thread order).
//
// Most-significant-digit radix select with adaptive digit windows:
//   0. the cluster reduces min / max / count of the valid (non-zero) keys; bits above the
//      highest bit where min and max differ are common to every key, so the first
//      10-bit digit starts right below them (keys spread over the histogram instead of
//      piling into a few bins);
//   1. per level: each CTA histograms the digit of the keys matching the prefix chosen
//      so far, the histograms are summed across the cluster through distributed shared
//      memory, and the bin holding the need-th largest key is fixed (the same in every
//      CTA); keys in higher bins are selected;
//   2. one ordered pass writes the selected keys in index order — positions come from
//      block-wide prefix sums plus a prefix over the cluster's CTAs — and the keys equal
//      to the K-th (all bits resolved) lowest index first.
// The result (contents and order) is deterministic.  PS = 4 (16 keys per thread) serves
// long key lists; PS = 2 (4 keys per thread) a list of at most 4,096 keys, which then
// takes a quarter of the per-key work.
// ------------------------------------------------------------------------------------
constexpr int kSelThreads = 1024;
constexpr int kDigitBits = 10;                   // radix digit: 1024 bins
constexpr int kBins = 1 << kDigitBits;
constexpr int kMaxCluster = 8;
// Shared memory, in 32-bit words:
//   sub   [kBins] one 32-bit counter per bin, counted by shared-memory atomics (lanes of a
//         warp that hit the same bin are serialised by the hardware; that measured cheaper
//         than lane-private counters, whose per-bin sums cost more than the collisions);
//         once the levels are done, the selected items are staged here
//   ks    [kSelThreads][kKeyRow]: the chunk of keys, thread t's kPer keys in row t (the pad
//         word puts key e of consecutive threads in consecutive banks)
//   hist  [kBins] this CTA's histogram;  hsum [kBins] the cluster's
//   scan scratch (32 x u64), cluster exchange words (16) and misc (8), padded to 64 words
//   blk   [CSA2_MAX_K] the query's Reindex block ids
// A CTA counts at most 2^23 keys (the host caps max_n_vis at 2^23), so no 32-bit counter
// can overflow.
constexpr int kSubWords = kBins > 2 * CSA2_MAX_K ? kBins : 2 * CSA2_MAX_K;
constexpr int kCand = 4096;  // keys of the cut bin a multi-chunk CTA keeps in shared memory
template <int PS>
struct SelShape {
  static constexpr int kPer = 1 << PS;                  // keys per thread per chunk
  static constexpr int kChunk = kSelThreads * kPer;     // keys per CTA per chunk
  static constexpr int kKeyRow = kPer + 1;              // a thread's keys in shared memory, padded
  static constexpr int kKeyWords = kSelThreads * kKeyRow;
  static constexpr int kSmem = (kSubWords + kKeyWords + 2 * kBins + 128 + 64 + CSA2_MAX_K + (PS >= 4 ? 2 * kCand : 0)) * 4;
};
static_assert(2 * CSA2_MAX_K <= kSubWords, "selected items are staged in the counter area");

struct SelectArgs {
  const uint32_t* keys;
  int64_t key_stride;
  int mode;
  int Q, block, n_blocks, K;
  int block_shift;           // log2(block)
  int csize;                 // CTAs per query (cluster size)
  const int64_t* seq_base;
  const int32_t* n_vis;
  int64_t max_n_vis, pool_entries;
  const int32_t* blocks;
  const int32_t* labels;     // kMerge: label of item i at labels[bq * key_stride + i]
  const uint32_t* gmax;      // kFlat, may be null: the largest key of every 32, per query row
  int64_t gstride;
  int64_t n_items;           // kMerge: items per query
  int32_t* out_idx;
  float* out_score;
};

// Entry index of item i (Reindex: slot i of the candidate pool; blk = the query's block
// ids, staged in shared memory).
__device__ __forceinline__ int64_t item_label(const SelectArgs& a, const int32_t* blk, int64_t i) {
  if (a.mode == kReindex) {
    const int32_t c = blk[i >> a.block_shift];
    return ((int64_t)c << a.block_shift) + (i & (a.block - 1));
  }
  if (a.mode == kMerge) return a.labels[(int64_t)blockIdx.y * a.key_stride + i];
  return i;
}

// Block-wide exclusive prefix sum of one value per thread (kSelThreads threads) of a
// 64-bit packed pair; ws holds kSelThreads/32 + 1 entries.
template <int NT = kSelThreads>
__device__ __forceinline__ uint64_t block_excl_scan64(uint64_t v, uint64_t* ws, uint64_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  constexpr int nw = NT / 32;
  uint64_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint64_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) ws[warp] = x;
  __syncthreads();
  if (warp == 0) {
    const uint64_t w = lane < nw ? ws[lane] : 0ull;
    uint64_t z = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint64_t y = __shfl_up_sync(0xffffffffu, z, o);
      if (lane >= o) z += y;
    }
    if (lane < nw) ws[lane] = z - w;
    if (lane == nw - 1) ws[nw] = z;
  }
  __syncthreads();
  const uint64_t r = ws[warp] + x - v;
  *total = ws[nw];
  __syncthreads();
  return r;
}

// Bin of hist[0, nb) (nb <= kBins) holding the need-th largest counted key, by one warp:
// lane l sums the R = max(nb/32, 1) bins nb-1-lR down to nb-R-lR; an inclusive scan over
// the lanes (top bins first) finds the lane whose run reaches need; then the whole warp
// scans that run (lane i takes its i-th bin from the top) and a ballot finds the bin.  The
// caller guarantees 1 <= need <= the total count.
__device__ __forceinline__ void find_bin_warp(const uint32_t* hist, int nb, uint32_t need, uint32_t* T_out,
                                              uint32_t* above_out) {
  const int lane = threadIdx.x & 31;
  const int R = nb >= 32 ? nb >> 5 : 1;
  const int top = nb - 1 - lane * R;
  uint32_t run = 0u;
#pragma unroll 8
  for (int i = 0; i < R; ++i) {  // rotated by the lane so the lanes' reads fall in different banks
    const int ii = (i + lane) & (R - 1);
    run += top - ii >= 0 ? hist[top - ii] : 0u;
  }
  uint32_t inc = run;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += y;
  }
  const uint32_t above = inc - run;
  // the lane whose run reaches need, and the count above its run
  const uint32_t hit = __ballot_sync(0xffffffffu, above < need && inc >= need);
  const int wl = __ffs(hit) - 1;
  const uint32_t w_above = __shfl_sync(0xffffffffu, above, wl);
  const int w_top = nb - 1 - wl * R;
  // lane i: i-th bin of that run from the top (R <= 32)
  const int b = w_top - lane;
  const uint32_t h = (lane < R && b >= 0) ? hist[b] : 0u;
  uint32_t hinc = h;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, hinc, o);
    if (lane >= o) hinc += y;
  }
  const uint32_t reach = __ballot_sync(0xffffffffu, lane < R && w_above + hinc >= need);
  const int fl = __ffs(reach) - 1;
  if (lane == fl) {
    *T_out = (uint32_t)b;
    *above_out = w_above + hinc - h;
  }
}

template <int PS>
__global__ void __launch_bounds__(kSelThreads, 1) select_kernel(SelectArgs a) {
  constexpr int kPerShift = PS;
  constexpr int kPer = SelShape<PS>::kPer;
  constexpr int kSelChunk = SelShape<PS>::kChunk;
  constexpr int kKeyRow = SelShape<PS>::kKeyRow;
  constexpr int kKeyWords = SelShape<PS>::kKeyWords;
  chain_launch_dependents();
  // phase: started
  namespace cg = cooperative_groups;
  cg::cluster_group cluster = cg::this_cluster();
  extern __shared__ __align__(16) uint32_t sel_smem[];
  uint32_t* sub = sel_smem;                  // [kBins/2][32] per-lane counters; then staging
  uint32_t* ks = sub + kSubWords;            // [kSelThreads][kKeyRow] keys of the chunk
  uint32_t* hist = ks + kKeyWords;           // [kBins] this CTA's histogram
  uint32_t* hsum = hist + kBins;             // [kBins] cluster-summed histogram
  uint64_t* scan_ws = reinterpret_cast<uint64_t*>(hsum + kBins);  // [kSelThreads/32 + 1]
  uint32_t* xch = reinterpret_cast<uint32_t*>(scan_ws + 64);       // [16] values exported to the cluster
  uint32_t* misc = xch + 16;                                        // [8]
  int32_t* blk = reinterpret_cast<int32_t*>(misc + 8);              // [n_blocks] Reindex block ids

  const int tid = threadIdx.x, lane = tid & 31;
  const int rank = (int)cluster.block_rank();
  const int C = a.csize;
  const int bq = blockIdx.y;
  const int b = bq / a.Q;
  const int K = a.K;
  for (int i = tid; i < kSubWords / 4; i += kSelThreads)  // counters start at zero
    reinterpret_cast<uint4*>(sub)[i] = make_uint4(0u, 0u, 0u, 0u);
  __syncthreads();  // every counter is cleared before any thread counts into it
  chain_wait();
  int32_t* out = a.out_idx + (int64_t)bq * K;
  float* out_s = a.out_score ? a.out_score + (int64_t)bq * K : nullptr;
  // shared::cluster address of `src` in CTA r
  auto remote = [&](const uint32_t* src, int r) { return tc::mapa(tc::smem_u32(src), (uint32_t)r); };

  int64_t n;
  if (a.mode == kMerge) {
    n = a.n_items;
  } else {
    const int64_t base = a.seq_base[b];
    int64_t nv = a.n_vis[bq];
    if (nv < 0 || nv > a.max_n_vis || base < 0 || base + nv > a.pool_entries) nv = 0;
    if (a.mode == kFlat)
      n = nv;
    else if (a.mode == kHier)
      n = (nv + a.block - 1) >> a.block_shift;
    else
      n = (int64_t)a.n_blocks * a.block;
  }
  const uint32_t* keys = a.keys + (int64_t)bq * a.key_stride;
  // this CTA's slice [lo, hi), a multiple of 4 keys so rows stay 16-byte aligned
  const int64_t slice = (((n + C - 1) / C) + 3) & ~int64_t(3);
  const int64_t lo = (int64_t)rank * slice;
  const int64_t hi = lo + slice < n ? lo + slice : n;
  const int nchunks = hi > lo ? (int)((hi - lo + kSelChunk - 1) / kSelChunk) : 0;

  if (a.mode == kReindex)  // read back with the labels of the selected items (barriers follow)
    for (int i = tid; i < a.n_blocks; i += kSelThreads) blk[i] = a.blocks[(int64_t)bq * a.n_blocks + i];

  // chunk ch of the slice -> ks (item lo + ch*kSelChunk + kPer*t + e is key e of thread t; 0 past hi)
  const uint32_t* mk = ks + tid * kKeyRow;
  uint32_t kmin = 0xFFFFFFFFu, kmax = 0u, cnt = 0u;  // over the valid (non-zero) keys
  constexpr int kLoads = kSelChunk / 4 / kSelThreads;  // 16 B loads per thread, all in flight
  // issue chunk ch's loads into registers (no wait)
  auto fetch_chunk = [&](int ch, uint4 (&v)[kLoads]) {
    const int64_t c0 = lo + (int64_t)ch * kSelChunk;
    const int64_t cn = hi - c0 < kSelChunk ? hi - c0 : kSelChunk;
#pragma unroll
    for (int u = 0; u < kLoads; ++u) {
      const int i = 4 * (tid + u * kSelThreads);
      v[u] = make_uint4(0u, 0u, 0u, 0u);
      if (i + 4 <= cn) {
        v[u] = *reinterpret_cast<const uint4*>(keys + c0 + i);
      } else if (i < cn) {
        v[u].x = keys[c0 + i];
        v[u].y = i + 1 < cn ? keys[c0 + i + 1] : 0u;
        v[u].z = i + 2 < cn ? keys[c0 + i + 2] : 0u;
      }
    }
  };
  // fetched keys -> ks, between barriers (earlier readers of ks are done; the rows are complete)
  auto stash_chunk = [&](const uint4 (&v)[kLoads], bool range) {
    __syncthreads();
#pragma unroll
    for (int u = 0; u < kLoads; ++u) {
      const int i = 4 * (tid + u * kSelThreads);
      if (range) {
        const uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          if (w[e] != 0u) {
            kmin = min(kmin, w[e]);
            kmax = max(kmax, w[e]);
            ++cnt;
          }
        }
      }
      uint32_t* d = ks + (i >> kPerShift) * kKeyRow + (i & (kPer - 1));
      d[0] = v[u].x;
      d[1] = v[u].y;
      d[2] = v[u].z;
      d[3] = v[u].w;
    }
    __syncthreads();
  };
  auto load_chunk = [&](int ch, bool range) {
    uint4 v[kLoads];
    fetch_chunk(ch, v);
    stash_chunk(v, range);
  };
  // ---- one CTA walking several chunks: two passes over the keys ------------------------------
  // Each pass fetches the next chunk into registers while the current one is processed.
  // Pass 1 counts the top 10 bits (sign, exponent, one mantissa bit) of every valid key; the
  // bin holding the K-th largest is the cut.  Pass 2 writes every key above that bin straight
  // to its slot (index order, per-chunk block prefixes) and copies the bin's keys, with their
  // item indices and in index order, into shared memory; the remaining radix levels and the
  // tied keys are resolved on that list.  The bin's keys must fit the list (kCand); when they
  // do not, the counters are cleared and the general path below runs instead.  Against the
  // general path (a range pass, one pass per level, a counting pass and an output pass, each
  // reloading every chunk) this reads the keys twice instead of about six times.
  // Shared by the one-CTA paths below: the listed keys (candk/candi, nc of them, in index
  // order; every one shares the bits of `mask` with `prefix`, the highest undecided bit being
  // p) resolved into the slots from `base`: the remaining radix levels in two alternating
  // histograms, then the taken keys in index order and the first `need` keys tied at the cut.
  uint32_t* candk = reinterpret_cast<uint32_t*>(blk + CSA2_MAX_K);  // [kCand] listed keys
  int32_t* candi = reinterpret_cast<int32_t*>(candk + kCand);        // [kCand] their item indices
  auto finish_list = [&](int nc, uint32_t base, uint32_t need, uint32_t prefix, uint32_t mask, int p,
                         int32_t* out, float* out_s) {

    for (int i = tid; i < kBins; i += kSelThreads) {
      hist[i] = 0u;
      hsum[i] = 0u;
    }
    __syncthreads();  // the list and the cleared counters are visible
    int cur = 0;
    while (p >= 0) {
      const int sh = p >= kDigitBits - 1 ? p - (kDigitBits - 1) : 0;
      const uint32_t nb = 1u << (p - sh + 1);
      uint32_t* h = cur ? hsum : hist;
      uint32_t* hn = cur ? hist : hsum;
      for (int i = tid; i < nc; i += kSelThreads) {
        const uint32_t key = candk[i];
        if ((key & mask) == prefix) atomicAdd(&h[(key >> sh) & (nb - 1u)], 1u);
      }
      for (int i = tid; i < kBins; i += kSelThreads) hn[i] = 0u;  // last read on the level before
      __syncthreads();
      if (tid < 32) {
        find_bin_warp(h, (int)nb, need, &misc[0], &misc[1]);
        __syncwarp();
        if (tid == 0) misc[2] = h[misc[0]];
      }
      __syncthreads();
      const uint32_t T = misc[0], inbin = misc[2];
      need -= misc[1];
      prefix |= T << sh;
      mask |= (nb - 1u) << sh;
      if (inbin == need || sh == 0) break;
      p = sh - 1;
      cur ^= 1;
    }
    // the list's taken keys after the first pass's, then its first `need` tied keys; a
    // thread takes a contiguous run of the list, so both stay in index order
    const int per = (nc + kSelThreads - 1) / kSelThreads;
    const int c0 = tid * per, c1 = min(nc, c0 + per);
    uint32_t g2 = 0u, e2 = 0u;
    for (int i = c0; i < c1; ++i) {
      const uint32_t kp = candk[i] & mask;
      if (kp > prefix) ++g2;
      else if (kp == prefix) ++e2;
    }
    uint64_t t2;
    const uint64_t m2 = block_excl_scan64((uint64_t)g2 | ((uint64_t)e2 << 32), scan_ws, &t2);
    uint32_t lg = base + (uint32_t)m2, le = (uint32_t)(m2 >> 32);
    const uint32_t tie0 = (uint32_t)K - need;
    for (int i = c0; i < c1; ++i) {
      const uint32_t key = candk[i], kp = key & mask;
      if (kp > prefix) {
        out[lg] = (int32_t)item_label(a, blk, candi[i]);
        if (out_s) out_s[lg] = key_score(key);
        ++lg;
      } else if (kp == prefix) {
        if (le < need) {
          out[tie0 + le] = (int32_t)item_label(a, blk, candi[i]);
          if (out_s) out_s[tie0 + le] = key_score(key);
        }
        ++le;
      }
    }
  };

  // ---- one CTA, with the scan's group maxima: a threshold, then only the groups above it ----
  // The flat scan also leaves the largest key of every 32 (gm).  At least K groups have a
  // maximum at or above x, the K-th largest maximum cut to its top 22 bits, so at least K keys
  // are >= x and the K best are among them.  Only the groups whose maximum reaches x are read
  // (a thread per group): their keys >= x go, with their item indices and in index order, to the
  // shared-memory list that the remaining radix levels resolve.  With fewer than K valid
  // groups x = 1, every valid key.  When the groups above x (kGroupList) or their keys
  // (kCand) do not fit, the counters are cleared and the two-pass path below runs instead.
  if constexpr (PS >= 4) {
    if (C == 1 && nchunks > 1 && a.gmax != nullptr) {
      constexpr int kGroupList = 8192;
      static_assert(2 * kGroupList <= kKeyWords, "the group list is kept where the chunks would be");
      const uint32_t* gm = a.gmax + (int64_t)bq * a.gstride;
      const int ng = (int)((n + 31) >> 5);
      uint32_t gc = 0u;
      for (int g = tid; g < ng; g += kSelThreads) {
        const uint32_t m = gm[g];
        if (m != 0u) {
          atomicAdd(&sub[m >> 20], 1u);
          ++gc;
        }
      }
      uint64_t gtot;
      block_excl_scan64((uint64_t)gc, scan_ws, &gtot);  // also orders the counts before the search
      uint32_t x = 1u;
      if (gtot >= (uint64_t)K) {
        // the 12-bit bin of the K-th largest maximum: its group of 4 among 1024, then the bin
        for (int g = tid; g < kBins; g += kSelThreads) {
          hist[g] = sub[4 * g] + sub[4 * g + 1] + sub[4 * g + 2] + sub[4 * g + 3];
          hsum[g] = 0u;
        }
        __syncthreads();
        if (tid < 32) {
          find_bin_warp(hist, kBins, (uint32_t)K, &misc[0], &misc[1]);
          __syncwarp();
          if (tid == 0) {
            uint32_t above = misc[1], need1 = (uint32_t)K - above, t = 4 * misc[0] + 3;
            for (int jj = 3; jj > 0; --jj, --t) {  // bins of the group from the top
              const uint32_t c = sub[t];
              if (need1 <= c) break;
              need1 -= c;
              above += c;
            }
            misc[2] = t;
            misc[3] = above;
          }
        }
        __syncthreads();
        const uint32_t T1 = misc[2], above1 = misc[3];
        // the next 10 bits, among the maxima in that bin
        for (int g = tid; g < ng; g += kSelThreads) {
          const uint32_t m = gm[g];
          if ((m >> 20) == T1) atomicAdd(&hsum[(m >> 10) & (kBins - 1)], 1u);
        }
        __syncthreads();
        if (tid < 32) find_bin_warp(hsum, kBins, (uint32_t)K - above1, &misc[4], &misc[5]);
        __syncthreads();
        x = max((T1 << 20) | (misc[4] << 10), 1u);
      }
      // the groups whose maximum reaches x, in index order (a thread takes a contiguous run)
      uint32_t* gl = ks;                // [kGroupList] their group numbers
      uint32_t* goff = ks + kGroupList;  // [kGroupList] their keys >= x, then their first list slots
      const int per = (ng + kSelThreads - 1) / kSelThreads;
      const int g0 = tid * per, g1 = min(ng, g0 + per);
      uint32_t sc = 0u;
      for (int g = g0; g < g1; ++g) sc += gm[g] >= x ? 1u : 0u;
      uint64_t stot;
      uint32_t so = (uint32_t)block_excl_scan64((uint64_t)sc, scan_ws, &stot);
      const int S = (int)stot;
      if (S <= kGroupList) {
        for (int g = g0; g < g1; ++g)
          if (gm[g] >= x) gl[so++] = (uint32_t)g;
        __syncthreads();
        // a thread takes whole groups: its 32 keys in eight 16-byte loads, all in flight at
        // once (keys past n read as 0)
        auto group_keys = [&](int sidx, uint32_t (&kk)[32]) {
          const int64_t i0 = (int64_t)gl[sidx] * 32;
          const uint4* src = reinterpret_cast<const uint4*>(keys + i0);
#pragma unroll
          for (int v = 0; v < 8; ++v) {
            const uint4 q = i0 + 4 * v + 3 < n ? src[v] : make_uint4(0u, 0u, 0u, 0u);
            kk[4 * v] = q.x;
            kk[4 * v + 1] = q.y;
            kk[4 * v + 2] = q.z;
            kk[4 * v + 3] = q.w;
          }
          if (i0 + 32 > n)  // the tail group: word loads of its keys below n
#pragma unroll
            for (int e = 0; e < 32; ++e) kk[e] = i0 + e < n ? keys[i0 + e] : 0u;
        };
        for (int sidx = tid; sidx < S; sidx += kSelThreads) {
          uint32_t kk[32];
          group_keys(sidx, kk);
          uint32_t c = 0u;
#pragma unroll
          for (int e = 0; e < 32; ++e) c += kk[e] >= x ? 1u : 0u;
          goff[sidx] = c;
        }
        __syncthreads();
        const int per2 = (S + kSelThreads - 1) / kSelThreads;
        const int s0 = tid * per2, s1 = min(S, s0 + per2);
        uint32_t cc = 0u;
        for (int si = s0; si < s1; ++si) cc += goff[si];
        uint64_t ctot;
        uint32_t co = (uint32_t)block_excl_scan64((uint64_t)cc, scan_ws, &ctot);
        const int nc = (int)ctot;
        if (nc <= kCand) {
          for (int si = s0; si < s1; ++si) {
            const uint32_t c = goff[si];
            goff[si] = co;
            co += c;
          }
          __syncthreads();
          for (int sidx = tid; sidx < S; sidx += kSelThreads) {
            uint32_t kk[32];
            group_keys(sidx, kk);
            uint32_t pos = goff[sidx];
            const int32_t gi = (int32_t)gl[sidx] * 32;
#pragma unroll
            for (int e = 0; e < 32; ++e)
              if (kk[e] >= x) {
                candk[pos] = kk[e];
                candi[pos] = gi + e;
                ++pos;
              }
          }
          if (nc <= K) {  // every valid key (fewer than K groups), in index order, then -1
            __syncthreads();
            for (int i = tid; i < K; i += kSelThreads) {
              if (i < nc) {
                out[i] = (int32_t)item_label(a, blk, candi[i]);
                if (out_s) out_s[i] = key_score(candk[i]);
              } else {
                out[i] = -1;
                if (out_s) out_s[i] = -INFINITY;
              }
            }
            return;
          }
          finish_list(nc, 0u, (uint32_t)K, 0u, 0u, 31, out, out_s);
          return;
        }
      }
      __syncthreads();  // every thread has left the counters and the list
      for (int i = tid; i < kSubWords / 4; i += kSelThreads)
        reinterpret_cast<uint4*>(sub)[i] = make_uint4(0u, 0u, 0u, 0u);
      __syncthreads();
    }
  }

  if (C == 1 && nchunks > 1) {
    uint32_t cnt = 0u;
    uint4 nxt[kLoads];  // the next chunk's keys, in flight while this one is counted
    fetch_chunk(0, nxt);
    for (int ch = 0; ch < nchunks; ++ch) {
      stash_chunk(nxt, false);
      if (ch + 1 < nchunks) fetch_chunk(ch + 1, nxt);
#pragma unroll 4
      for (int e = 0; e < kPer; ++e) {
        const uint32_t key = mk[e];
        if (key != 0u) {
          atomicAdd(&sub[key >> 20], 1u);
          ++cnt;
        }
      }
    }
    uint64_t tot;
    block_excl_scan64((uint64_t)cnt, scan_ws, &tot);  // also orders the counts before the search
    const bool all_valid = tot <= (uint64_t)K;
    uint32_t T1 = 0u, above1 = 0u, inbin1 = 0u;
    if (!all_valid) {  // the cut bin of 4096: its group of 4 among 1024 groups, then the bin
      for (int g = tid; g < kBins; g += kSelThreads)
        hist[g] = sub[4 * g] + sub[4 * g + 1] + sub[4 * g + 2] + sub[4 * g + 3];
      __syncthreads();
      if (tid < 32) {
        find_bin_warp(hist, kBins, (uint32_t)K, &misc[0], &misc[1]);
        __syncwarp();
        if (tid == 0) {
          uint32_t above = misc[1], need1 = (uint32_t)K - above, t = 4 * misc[0] + 3;
          for (int jj = 3; jj > 0; --jj, --t) {  // bins of the group from the top
            const uint32_t c = sub[t];
            if (need1 <= c) break;
            need1 -= c;
            above += c;
          }
          misc[2] = t;
          misc[3] = above;
          misc[4] = sub[t];
        }
      }
      __syncthreads();
      T1 = misc[2];
      above1 = misc[3];
      inbin1 = misc[4];
    }
    if (all_valid || inbin1 <= (uint32_t)kCand) {
      int32_t* out = a.out_idx + (int64_t)bq * K;
      float* out_s = a.out_score ? a.out_score + (int64_t)bq * K : nullptr;
      uint32_t base_g = 0u, base_c = 0u;
      fetch_chunk(0, nxt);
      for (int ch = 0; ch < nchunks; ++ch) {
        stash_chunk(nxt, false);
        if (ch + 1 < nchunks) fetch_chunk(ch + 1, nxt);
        uint32_t cg = 0u, cc = 0u;
#pragma unroll 4
        for (int e = 0; e < kPer; ++e) {
          const uint32_t key = mk[e];
          if (key != 0u) {
            const uint32_t d = key >> 20;
            if (all_valid || d > T1) ++cg;
            else if (d == T1) ++cc;
          }
        }
        uint64_t ctot;
        const uint64_t cm = block_excl_scan64((uint64_t)cg | ((uint64_t)cc << 32), scan_ws, &ctot);
        uint32_t lg = base_g + (uint32_t)cm, lc = base_c + (uint32_t)(cm >> 32);
        const int64_t i0 = lo + (int64_t)ch * kSelChunk + (int64_t)tid * kPer;
#pragma unroll 2
        for (int e = 0; e < kPer; ++e) {
          const uint32_t key = mk[e];
          if (key == 0u) continue;
          const uint32_t d = key >> 20;
          if (all_valid || d > T1) {
            out[lg] = (int32_t)item_label(a, blk, i0 + e);
            if (out_s) out_s[lg] = key_score(key);
            ++lg;
          } else if (d == T1) {
            candk[lc] = key;
            candi[lc] = (int32_t)(i0 + e);
            ++lc;
          }
        }
        base_g += (uint32_t)ctot;
        base_c += (uint32_t)(ctot >> 32);
      }
      if (all_valid) {
        for (int i = (int)base_g + tid; i < K; i += kSelThreads) {
          out[i] = -1;
          if (out_s) out_s[i] = -INFINITY;
        }
        return;
      }
      finish_list((int)base_c, above1, (uint32_t)K - above1, T1 << 20, 0xFFF00000u, 19, out, out_s);
      return;
    }
    __syncthreads();  // every thread has read the search's result before the counters clear
    for (int i = tid; i < kSubWords / 4; i += kSelThreads)
      reinterpret_cast<uint4*>(sub)[i] = make_uint4(0u, 0u, 0u, 0u);
    __syncthreads();
  }

  // ---- 0. cluster-wide min / max / count of valid keys, taken while loading -------------
  for (int ch = 0; ch < nchunks; ++ch) load_chunk(ch, true);  // a single chunk stays loaded
  // phase: keys loaded
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    kmin = min(kmin, __shfl_xor_sync(0xffffffffu, kmin, o));
    kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, o));
    cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
  }
  if (tid < 16) xch[tid] = (tid == 0) ? 0xFFFFFFFFu : 0u;
  __syncthreads();
  if (lane == 0) {
    atomicMin(&xch[0], kmin);
    atomicMax(&xch[1], kmax);
    atomicAdd(&xch[2], cnt);
  }
  if (C == 1) __syncthreads();
  else cluster.sync();
  uint32_t gmin = 0xFFFFFFFFu, gmax = 0u, gcnt = 0u;
  // phase: range reduced
  if (C == 1) {
    gmin = xch[0];
    gmax = xch[1];
    gcnt = xch[2];
  } else {
    uint32_t v[kMaxCluster][3];
#pragma unroll
    for (int r = 0; r < kMaxCluster; ++r) {
      const uint32_t ra = remote(xch, r < C ? r : 0);
      v[r][0] = tc::ld_cluster_u32(ra);
      v[r][1] = tc::ld_cluster_u32(ra + 4);
      v[r][2] = r < C ? tc::ld_cluster_u32(ra + 8) : 0u;
    }
#pragma unroll
    for (int r = 0; r < kMaxCluster; ++r) {
      gmin = min(gmin, v[r][0]);
      gmax = max(gmax, v[r][1]);
      gcnt += v[r][2];
    }
  }

  // ---- 1. radix levels ------------------------------------------------------------------
  uint32_t prefix = 0u, mask = 0u, need = (uint32_t)K;
  const bool all_valid = gcnt <= (uint32_t)K;
  if (!all_valid) {
    if (gmin == gmax) {
      prefix = gmin;  // every valid key is equal: ties only
      mask = 0xFFFFFFFFu;
    } else {
      int p = 31 - __clz(gmin ^ gmax);  // highest bit where keys differ
      mask = p == 31 ? 0u : ~((2u << p) - 1u);
      prefix = gmin & mask;
      for (;;) {
        const int sh = p >= kDigitBits - 1 ? p - (kDigitBits - 1) : 0;
        const int width = p - sh + 1;
        const uint32_t nb = 1u << width;
        for (int ch = 0; ch < nchunks; ++ch) {
          if (nchunks > 1) load_chunk(ch, false);
#pragma unroll 4
          for (int e = 0; e < kPer; ++e) {
            const uint32_t key = mk[e];
            if (key != 0u && (key & mask) == prefix) {
              const uint32_t bin = (key >> sh) & (nb - 1u);
              atomicAdd(&sub[bin], 1u);
            }
          }
        }
        __syncthreads();
        // bin totals to hist; the counters are zeroed for the next level
        for (int c = tid; c < (int)nb; c += kSelThreads) {
          hist[c] = sub[c];
          sub[c] = 0u;
        }
  // phase: level counted
        const uint32_t* hs = hist;
        if (C > 1) {  // sum every CTA's histogram
          cluster.sync();
          for (int i = tid; i < (int)nb; i += kSelThreads) {
            uint32_t v[kMaxCluster];
#pragma unroll
            for (int r = 0; r < kMaxCluster; ++r) v[r] = r < C ? tc::ld_cluster_u32(remote(hist, r) + 4u * i) : 0u;
            uint32_t sum = 0u;
#pragma unroll
            for (int r = 0; r < kMaxCluster; ++r) sum += v[r];
            hsum[i] = sum;
          }
          hs = hsum;
        }
        __syncthreads();
        if (tid < 32) find_bin_warp(hs, (int)nb, need, &misc[0], &misc[1]);
        __syncthreads();
  // phase: level found
        const uint32_t T = misc[0];
        need -= misc[1];
        prefix |= T << sh;
        mask |= (nb - 1u) << sh;
        const uint32_t inbin = hs[T];
        if (C > 1) cluster.sync();  // remote reads of `hist` done before it is rewritten
        if (inbin == need) break;   // every key of the bin is selected
        if (sh == 0) break;
        p = sh - 1;
      }
    }
  }

  // ---- 2. ordered output -----------------------------------------------------------------
  // phase: levels done
  // per-CTA counts of selected keys (gt) and of keys equal to the threshold prefix (eq)
  auto classify = [&](uint32_t key, bool& gt, bool& eq) {
    const uint32_t kp = key & mask;
    gt = key != 0u && (all_valid || kp > prefix);
    eq = key != 0u && !all_valid && kp == prefix;
  };
  uint32_t my_gt = 0u, my_eq = 0u;
  for (int ch = 0; ch < nchunks; ++ch) {
    if (nchunks > 1) load_chunk(ch, false);
#pragma unroll 4
    for (int e = 0; e < kPer; ++e) {
      bool gt, eq;
      classify(mk[e], gt, eq);
      my_gt += gt;
      my_eq += eq;
    }
  }
  uint64_t tot;
  const uint64_t mine = block_excl_scan64((uint64_t)my_gt | ((uint64_t)my_eq << 32), scan_ws, &tot);
  if (tid == 0) {
    xch[4] = (uint32_t)tot;
    xch[5] = (uint32_t)(tot >> 32);
  }
  if (C == 1) __syncthreads();
  else cluster.sync();
  uint32_t cta_gt = 0u, cta_eq = 0u, all_gt = (uint32_t)tot;
  if (C > 1) {
    uint32_t g[kMaxCluster], q[kMaxCluster];
#pragma unroll
    for (int r = 0; r < kMaxCluster; ++r) {
      const uint32_t ra = remote(xch, r < C ? r : 0);
      g[r] = r < C ? tc::ld_cluster_u32(ra + 16) : 0u;
      q[r] = r < C ? tc::ld_cluster_u32(ra + 20) : 0u;
    }
    all_gt = 0u;
#pragma unroll
    for (int r = 0; r < kMaxCluster; ++r) {
      if (r < rank) {
        cta_gt += g[r];
        cta_eq += q[r];
      }
      all_gt += g[r];
    }
  }
  // phase: positions known
  // This CTA's selected keys go to out[cta_gt, cta_gt + G) in index order, and its first
  // e_take keys equal to the threshold to out[tie0 + cta_eq, ...): staged in shared memory
  // in that order, then copied out with consecutive threads on consecutive slots.
  const uint32_t G = (uint32_t)tot, E = (uint32_t)(tot >> 32);
  const uint32_t tie0 = (uint32_t)K - need;  // first slot of the equal keys
  const uint32_t e_take = need > cta_eq ? min(E, need - cta_eq) : 0u;
  int32_t* s_idx = reinterpret_cast<int32_t*>(sub);  // [G + e_take <= K]
  float* s_sc = reinterpret_cast<float*>(sub + CSA2_MAX_K);
  // With one chunk, thread order is index order and the counting pass's prefix places
  // every item.  With several, a thread's items are not contiguous in index order across
  // chunks, so each chunk gets its own block-wide prefix on top of the counts of the
  // chunks before it: the staged order is then index order throughout.
  uint32_t base_g = 0u, base_e = 0u;
  for (int ch = 0; ch < nchunks; ++ch) {
    uint32_t lg = (uint32_t)mine, le = (uint32_t)(mine >> 32);
    if (nchunks > 1) {
      load_chunk(ch, false);
      uint32_t cg = 0u, ce = 0u;
#pragma unroll 4
      for (int e = 0; e < kPer; ++e) {
        bool gt, eq;
        classify(mk[e], gt, eq);
        cg += gt;
        ce += eq;
      }
      uint64_t ctot;
      const uint64_t cm = block_excl_scan64((uint64_t)cg | ((uint64_t)ce << 32), scan_ws, &ctot);
      lg = base_g + (uint32_t)cm;
      le = base_e + (uint32_t)(cm >> 32);
      base_g += (uint32_t)ctot;
      base_e += (uint32_t)(ctot >> 32);
    }
    const int64_t i0 = lo + (int64_t)ch * kSelChunk + (int64_t)tid * kPer;
#pragma unroll 2
    for (int e = 0; e < kPer; ++e) {
      const uint32_t key = mk[e];
      bool gt, eq;
      classify(key, gt, eq);
      if (gt) {
        s_idx[lg] = (int32_t)item_label(a, blk, i0 + e);
        s_sc[lg] = key_score(key);
        ++lg;
      } else if (eq) {
        if (le < e_take) {
          s_idx[G + le] = (int32_t)item_label(a, blk, i0 + e);
          s_sc[G + le] = key_score(key);
        }
        ++le;
      }
    }
  }
  __syncthreads();
  for (uint32_t i = tid; i < G + e_take; i += kSelThreads) {
    const uint32_t slot = i < G ? cta_gt + i : tie0 + cta_eq + (i - G);
    out[slot] = s_idx[i];
    if (out_s) out_s[slot] = s_sc[i];
  }
  // phase: written
  if (all_valid && rank == 0) {
    for (int i = (int)all_gt + tid; i < K; i += kSelThreads) {
      out[i] = -1;
      if (out_s) out_s[i] = -INFINITY;
    }
  }
  if (C > 1) cluster.sync();  // keep every CTA's shared memory alive until remote reads are done
}

// Flat selection with the scan's group maxima, one small CTA per query (many queries: verify,
// prefill).  The same threshold and list method as select_kernel's one-CTA group path, in 256
// threads and 48 KB of shared memory, so four CTAs share an SM and a verify step's 512
// queries take one wave.  The 12-bit histogram of the maxima and the key list share one area
// (the list is written after the histogram is read), as do the radix histograms and the
// group list.  When the groups at or above x or their keys do not fit, the CTA selects
// exactly over all n keys from global memory instead (radix levels, one pass per level).
constexpr int kGsThreads = 256;
constexpr int kGsList = 2048;   // groups at or above the threshold
constexpr int kGsCand = 4096;   // keys at or above the threshold
constexpr int kGsSmemBytes = (kGsCand * 2 + 2 * kGsList + 64 + 16) * 4;

__global__ void __launch_bounds__(kGsThreads) group_select_kernel(SelectArgs a) {
  chain_launch_dependents();
  extern __shared__ __align__(16) uint32_t gs_smem[];
  uint32_t* sub = gs_smem;                                        // [4096] maxima histogram
  uint32_t* candk = gs_smem;                                      // [kGsCand] listed keys (after sub)
  int32_t* candi = reinterpret_cast<int32_t*>(gs_smem + kGsCand);  // [kGsCand] their indices
  uint32_t* hist = gs_smem + 2 * kGsCand;                         // [kBins]
  uint32_t* hsum = hist + kBins;                                  // [kBins]
  uint32_t* gl = hist;                                            // [kGsList] groups (after hist/hsum)
  uint32_t* goff = gl + kGsList;                                  // [kGsList]
  uint64_t* scan_ws = reinterpret_cast<uint64_t*>(gl + 2 * kGsList);  // [kGsThreads/32 + 1]
  uint32_t* misc = reinterpret_cast<uint32_t*>(scan_ws + 32);         // [8]
  static_assert(2 * kBins <= 2 * kGsList, "the radix histograms fit the group list area");
  static_assert(4096 <= kGsCand, "the maxima histogram fits the key list area");
  const int tid = threadIdx.x;
  const int bq = blockIdx.x;
  const int b = bq / a.Q;
  const int K = a.K;
  for (int i = tid; i < 4096 / 4; i += kGsThreads) reinterpret_cast<uint4*>(sub)[i] = make_uint4(0u, 0u, 0u, 0u);
  __syncthreads();  // every counter is cleared before any thread counts into it
  chain_wait();
  int32_t* out = a.out_idx + (int64_t)bq * K;
  float* out_s = a.out_score ? a.out_score + (int64_t)bq * K : nullptr;
  const int64_t base = a.seq_base[b];
  int64_t n = a.n_vis[bq];
  if (n < 0 || n > a.max_n_vis || base < 0 || base + n > a.pool_entries) n = 0;
  const uint32_t* keys = a.keys + (int64_t)bq * a.key_stride;
  const uint32_t* gm = a.gmax + (int64_t)bq * a.gstride;
  const int ng = (int)((n + 31) >> 5);

  // the listed keys (nc, index order, sharing `mask` bits with `prefix`, bit p the highest
  // undecided) resolved into the slots from `base0`: radix levels, then the taken keys and the
  // first `need` tied keys in index order
  auto finish_list = [&](int nc, uint32_t base0, uint32_t need, uint32_t prefix, uint32_t mask, int p) {
    for (int i = tid; i < kBins; i += kGsThreads) {
      hist[i] = 0u;
      hsum[i] = 0u;
    }
    __syncthreads();
    int cur = 0;
    while (p >= 0) {
      const int sh = p >= kDigitBits - 1 ? p - (kDigitBits - 1) : 0;
      const uint32_t nb = 1u << (p - sh + 1);
      uint32_t* h = cur ? hsum : hist;
      uint32_t* hn = cur ? hist : hsum;
      for (int i = tid; i < nc; i += kGsThreads) {
        const uint32_t key = candk[i];
        if ((key & mask) == prefix) atomicAdd(&h[(key >> sh) & (nb - 1u)], 1u);
      }
      for (int i = tid; i < kBins; i += kGsThreads) hn[i] = 0u;
      __syncthreads();
      if (tid < 32) {
        find_bin_warp(h, (int)nb, need, &misc[0], &misc[1]);
        __syncwarp();
        if (tid == 0) misc[2] = h[misc[0]];
      }
      __syncthreads();
      const uint32_t T = misc[0], inbin = misc[2];
      need -= misc[1];
      prefix |= T << sh;
      mask |= (nb - 1u) << sh;
      if (inbin == need || sh == 0) break;
      p = sh - 1;
      cur ^= 1;
    }
    const int per = (nc + kGsThreads - 1) / kGsThreads;
    const int c0 = tid * per, c1 = min(nc, c0 + per);
    uint32_t g2 = 0u, e2 = 0u;
    for (int i = c0; i < c1; ++i) {
      const uint32_t kp = candk[i] & mask;
      if (kp > prefix) ++g2;
      else if (kp == prefix) ++e2;
    }
    uint64_t t2;
    const uint64_t m2 = block_excl_scan64<kGsThreads>((uint64_t)g2 | ((uint64_t)e2 << 32), scan_ws, &t2);
    uint32_t lg = base0 + (uint32_t)m2, le = (uint32_t)(m2 >> 32);
    const uint32_t tie0 = (uint32_t)K - need;
    for (int i = c0; i < c1; ++i) {
      const uint32_t key = candk[i], kp = key & mask;
      if (kp > prefix) {
        out[lg] = candi[i];
        if (out_s) out_s[lg] = key_score(key);
        ++lg;
      } else if (kp == prefix) {
        if (le < need) {
          out[tie0 + le] = candi[i];
          if (out_s) out_s[tie0 + le] = key_score(key);
        }
        ++le;
      }
    }
  };

  // ---- the threshold x from the group maxima ------------------------------------------------
  uint32_t gc = 0u;
  for (int g = tid; g < ng; g += kGsThreads) {
    const uint32_t m = gm[g];
    if (m != 0u) {
      atomicAdd(&sub[m >> 20], 1u);
      ++gc;
    }
  }
  uint64_t gtot;
  block_excl_scan64<kGsThreads>((uint64_t)gc, scan_ws, &gtot);
  uint32_t x = 1u;
  if (gtot >= (uint64_t)K) {
    for (int g = tid; g < kBins; g += kGsThreads) {
      hist[g] = sub[4 * g] + sub[4 * g + 1] + sub[4 * g + 2] + sub[4 * g + 3];
      hsum[g] = 0u;
    }
    __syncthreads();
    if (tid < 32) {
      find_bin_warp(hist, kBins, (uint32_t)K, &misc[0], &misc[1]);
      __syncwarp();
      if (tid == 0) {
        uint32_t above = misc[1], need1 = (uint32_t)K - above, t = 4 * misc[0] + 3;
        for (int jj = 3; jj > 0; --jj, --t) {
          const uint32_t c = sub[t];
          if (need1 <= c) break;
          need1 -= c;
          above += c;
        }
        misc[2] = t;
        misc[3] = above;
      }
    }
    __syncthreads();
    const uint32_t T1 = misc[2], above1 = misc[3];
    for (int g = tid; g < ng; g += kGsThreads) {
      const uint32_t m = gm[g];
      if ((m >> 20) == T1) atomicAdd(&hsum[(m >> 10) & (kBins - 1)], 1u);
    }
    __syncthreads();
    if (tid < 32) find_bin_warp(hsum, kBins, (uint32_t)K - above1, &misc[4], &misc[5]);
    __syncthreads();
    x = max((T1 << 20) | (misc[4] << 10), 1u);
  }
  // ---- the groups at or above x, in index order --------------------------------------------
  const int per = (ng + kGsThreads - 1) / kGsThreads;
  const int g0 = tid * per, g1 = min(ng, g0 + per);
  uint32_t sc = 0u;
  for (int g = g0; g < g1; ++g) sc += gm[g] >= x ? 1u : 0u;
  uint64_t stot;
  uint32_t so = (uint32_t)block_excl_scan64<kGsThreads>((uint64_t)sc, scan_ws, &stot);  // ends in a barrier
  const int S = (int)stot;
  if (S <= kGsList) {
    for (int g = g0; g < g1; ++g)
      if (gm[g] >= x) gl[so++] = (uint32_t)g;
    __syncthreads();
    // a thread takes whole groups: its 32 keys in eight 16-byte loads, all in flight at once
    // (keys past n read as 0)
    auto group_keys = [&](int sidx, uint32_t (&kk)[32]) {
      const int64_t i0 = (int64_t)gl[sidx] * 32;
      const uint4* src = reinterpret_cast<const uint4*>(keys + i0);
#pragma unroll
      for (int v = 0; v < 8; ++v) {
        const uint4 q = i0 + 4 * v + 3 < n ? src[v] : make_uint4(0u, 0u, 0u, 0u);
        kk[4 * v] = q.x;
        kk[4 * v + 1] = q.y;
        kk[4 * v + 2] = q.z;
        kk[4 * v + 3] = q.w;
      }
      if (i0 + 32 > n)  // the tail group: word loads of its keys below n
#pragma unroll
        for (int e = 0; e < 32; ++e) kk[e] = i0 + e < n ? keys[i0 + e] : 0u;
    };
    for (int sidx = tid; sidx < S; sidx += kGsThreads) {
      uint32_t kk[32];
      group_keys(sidx, kk);
      uint32_t c = 0u;
#pragma unroll
      for (int e = 0; e < 32; ++e) c += kk[e] >= x ? 1u : 0u;
      goff[sidx] = c;
    }
    __syncthreads();
    const int per2 = (S + kGsThreads - 1) / kGsThreads;
    const int s0 = tid * per2, s1 = min(S, s0 + per2);
    uint32_t cc = 0u;
    for (int si = s0; si < s1; ++si) cc += goff[si];
    uint64_t ctot;
    uint32_t co = (uint32_t)block_excl_scan64<kGsThreads>((uint64_t)cc, scan_ws, &ctot);
    const int nc = (int)ctot;
    if (nc <= kGsCand) {
      for (int si = s0; si < s1; ++si) {
        const uint32_t c = goff[si];
        goff[si] = co;
        co += c;
      }
      __syncthreads();
      for (int sidx = tid; sidx < S; sidx += kGsThreads) {
        uint32_t kk[32];
        group_keys(sidx, kk);
        uint32_t pos = goff[sidx];
        const int32_t gi = (int32_t)gl[sidx] * 32;
#pragma unroll
        for (int e = 0; e < 32; ++e)
          if (kk[e] >= x) {
            candk[pos] = kk[e];
            candi[pos] = gi + e;
            ++pos;
          }
      }
      __syncthreads();  // the list is complete; the group list is no longer read
      if (nc <= K) {  // every valid key (fewer than K groups), in index order, then -1
        for (int i = tid; i < K; i += kGsThreads) {
          if (i < nc) {
            out[i] = candi[i];
            if (out_s) out_s[i] = key_score(candk[i]);
          } else {
            out[i] = -1;
            if (out_s) out_s[i] = -INFINITY;
          }
        }
        return;
      }
      finish_list(nc, 0u, (uint32_t)K, 0u, 0u, 31);
      return;
    }
  }
  __syncthreads();  // every thread has left the lists
  // ---- heavy ties: exact select over all n keys from global memory -------------------------
  // counting passes stride over the keys (coalesced); the output passes give thread t the keys
  // [t * chunk, (t + 1) * chunk), so block prefixes keep index order
  const int64_t chunk = (n + kGsThreads - 1) / kGsThreads;
  const int64_t k0 = (int64_t)tid * chunk, k1 = k0 + chunk < n ? k0 + chunk : n;
  uint32_t vc = 0u;
  for (int64_t i = k0; i < k1; ++i) vc += keys[i] != 0u ? 1u : 0u;
  uint64_t vtot;
  uint64_t vo = block_excl_scan64<kGsThreads>((uint64_t)vc, scan_ws, &vtot);
  if (vtot <= (uint64_t)K) {  // every valid key, in index order, then -1
    for (int64_t i = k0; i < k1; ++i)
      if (keys[i] != 0u) {
        out[vo] = (int32_t)i;
        if (out_s) out_s[vo] = key_score(keys[i]);
        ++vo;
      }
    for (int i = (int)vtot + tid; i < K; i += kGsThreads) {
      out[i] = -1;
      if (out_s) out_s[i] = -INFINITY;
    }
    return;
  }
  uint32_t need = (uint32_t)K, prefix = 0u, mask = 0u;
  int p = 31;
  while (p >= 0) {
    const int sh = p >= kDigitBits - 1 ? p - (kDigitBits - 1) : 0;
    const uint32_t nb = 1u << (p - sh + 1);
    for (int i = tid; i < kBins; i += kGsThreads) hist[i] = 0u;
    __syncthreads();
    for (int64_t i = tid; i < n; i += kGsThreads) {
      const uint32_t key = keys[i];
      if (key != 0u && (key & mask) == prefix) atomicAdd(&hist[(key >> sh) & (nb - 1u)], 1u);
    }
    __syncthreads();
    if (tid < 32) {
      find_bin_warp(hist, (int)nb, need, &misc[0], &misc[1]);
      __syncwarp();
      if (tid == 0) misc[2] = hist[misc[0]];
    }
    __syncthreads();
    const uint32_t T = misc[0], inbin = misc[2];
    need -= misc[1];
    prefix |= T << sh;
    mask |= (nb - 1u) << sh;
    if (inbin == need || sh == 0) break;
    p = sh - 1;
  }
  uint32_t g2 = 0u, e2 = 0u;
  for (int64_t i = k0; i < k1; ++i) {
    const uint32_t key = keys[i];
    if (key == 0u) continue;
    const uint32_t kp = key & mask;
    if (kp > prefix) ++g2;
    else if (kp == prefix) ++e2;
  }
  uint64_t t2;
  const uint64_t m2 = block_excl_scan64<kGsThreads>((uint64_t)g2 | ((uint64_t)e2 << 32), scan_ws, &t2);
  uint32_t lg = (uint32_t)m2, le = (uint32_t)(m2 >> 32);
  const uint32_t tie0 = (uint32_t)K - need;
  for (int64_t i = k0; i < k1; ++i) {
    const uint32_t key = keys[i];
    if (key == 0u) continue;
    const uint32_t kp = key & mask;
    if (kp > prefix) {
      out[lg] = (int32_t)i;
      if (out_s) out_s[lg] = key_score(key);
      ++lg;
    } else if (kp == prefix) {
      if (le < need) {
        out[tie0 + le] = (int32_t)i;
        if (out_s) out_s[tie0 + le] = key_score(key);
      }
      ++le;
    }
  }
}

// Selection of lists held in registers: a query's keys are split over a cluster of C CTAs
// (C = 1 .. 8, the cluster's x dimension), CTA r holding keys [r * 1024 * KPT, (r + 1) * 1024 *
// KPT), thread t of it KPT consecutive keys, so (rank, thread, slot) order is index order.
// Same radix levels, tie rule and output order as select_kernel.  Per level: every CTA counts
// its keys into one of two histograms, one cluster barrier, then each thread sums its bin over
// the cluster (distributed shared memory) and clears the other histogram (the one the
// cluster read on the level before, which every CTA has finished reading by this barrier),
// and one warp finds the bin.  The output positions take one more cluster exchange.
template <int KPT>
__global__ void __launch_bounds__(1024, 1) select_cl_kernel(SelectArgs a) {
  static_assert(KPT % 4 == 0, "keys are loaded 16 bytes at a time");
  constexpr int NT = 1024;
  chain_launch_dependents();
  __shared__ uint32_t hist[2][kBins];   // this CTA's counts, alternating per level
  __shared__ uint32_t hsum[kBins];      // the cluster's counts of the current level
  __shared__ uint32_t wred[3][32];      // per-warp min, max, count of valid keys (one CTA)
  __shared__ uint32_t wsum[2][32];      // per-warp totals of taken / tied keys
  __shared__ uint32_t xch[8];           // exported to the cluster: [4] taken and [5] tied keys
  __shared__ uint32_t lvl[4];           // bin found, keys above it, keys in it
  __shared__ uint32_t wtop[32];         // per-warp counts of a level's bins (bin search)
  __shared__ int32_t blk[CSA2_MAX_K];   // Reindex block ids of the query
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int C = a.csize;
  const int rank = C > 1 ? (int)tc::cluster_ctarank() : 0;
  const int bq = blockIdx.y;
  const int b = bq / a.Q;
  const int K = a.K;
  hist[0][tid] = 0u;
  __syncthreads();  // every counter is cleared before any thread counts into it
  chain_wait();
  auto cluster_sync = [&]() {
    if (C > 1) {
      asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
    } else {
      __syncthreads();
    }
  };
  // word w of `arr` in CTA r of the cluster
  auto remote = [&](const uint32_t* arr, int w, int r) {
    return tc::ld_cluster_u32(tc::mapa(tc::smem_u32(arr + w), (uint32_t)r));
  };

  int n;  // keys of this query (at most C * 1024 * KPT, checked by the host)
  if (a.mode == kMerge) {
    n = (int)a.n_items;
  } else {
    const int64_t base = a.seq_base[b];
    int64_t nv = a.n_vis[bq];
    if (nv < 0 || nv > a.max_n_vis || base < 0 || base + nv > a.pool_entries) nv = 0;
    if (a.mode == kFlat)
      n = (int)nv;
    else if (a.mode == kHier)
      n = (int)((nv + a.block - 1) >> a.block_shift);
    else
      n = a.n_blocks * a.block;
  }
  if (a.mode == kReindex)
    for (int i = tid; i < a.n_blocks; i += NT) blk[i] = a.blocks[(int64_t)bq * a.n_blocks + i];

  // ---- keys into registers; the range of the valid (non-zero) keys ---------------------------
  const uint32_t* keys = a.keys + (int64_t)bq * a.key_stride;
  const int i0 = rank * NT * KPT + tid * KPT;
  uint32_t k[KPT];
#pragma unroll
  for (int u = 0; u < KPT / 4; ++u) {
    const int i = i0 + 4 * u;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (i + 4 <= n) {
      v = *reinterpret_cast<const uint4*>(keys + i);
    } else if (i < n) {
      v.x = keys[i];
      v.y = i + 1 < n ? keys[i + 1] : 0u;
      v.z = i + 2 < n ? keys[i + 2] : 0u;
    }
    k[4 * u] = v.x;
    k[4 * u + 1] = v.y;
    k[4 * u + 2] = v.z;
    k[4 * u + 3] = v.w;
  }
  // One CTA: the range of the valid keys aims the first digit at the highest bit where they
  // differ.  A cluster skips that exchange (about 1-2 us): its first digit is the top 10 bits,
  // and the count of valid keys comes from that level's summed histogram.
  uint32_t gmin = 0xFFFFFFFFu, gmax = 0u, gcnt = 0u;
  if (C == 1) {
    uint32_t cnt = 0u;
#pragma unroll
    for (int e = 0; e < KPT; ++e) {
      if (k[e] != 0u) {
        gmin = min(gmin, k[e]);
        gmax = max(gmax, k[e]);
        ++cnt;
      }
    }
    gcnt = cnt;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      gmin = min(gmin, __shfl_xor_sync(0xffffffffu, gmin, o));
      gmax = max(gmax, __shfl_xor_sync(0xffffffffu, gmax, o));
      gcnt += __shfl_xor_sync(0xffffffffu, gcnt, o);
    }
    if (lane == 0) {
      wred[0][warp] = gmin;
      wred[1][warp] = gmax;
      wred[2][warp] = gcnt;
    }
    __syncthreads();
    // every warp reduces the warps' partials, lane w taking warp w's
    gmin = wred[0][lane];
    gmax = wred[1][lane];
    gcnt = wred[2][lane];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      gmin = min(gmin, __shfl_xor_sync(0xffffffffu, gmin, o));
      gmax = max(gmax, __shfl_xor_sync(0xffffffffu, gmax, o));
      gcnt += __shfl_xor_sync(0xffffffffu, gcnt, o);
    }
  }

  // ---- radix levels --------------------------------------------------------------------------
  uint32_t prefix = 0u, mask = 0u, need = (uint32_t)K;
  bool all_valid = C == 1 && gcnt <= (uint32_t)K;
  int p = 31;  // highest bit of the first digit; -1: no level
  if (C == 1 && !all_valid) {
    if (gmin == gmax) {
      prefix = gmin;  // every valid key is equal: ties only
      mask = 0xFFFFFFFFu;
      p = -1;
    } else {
      p = 31 - __clz(gmin ^ gmax);  // highest bit where keys differ
      mask = p == 31 ? 0u : ~((2u << p) - 1u);
      prefix = gmin & mask;
    }
  }
  if (!all_valid && p >= 0) {
    int cur = 0;
    for (int level = 0;; ++level) {
      const int sh = p >= kDigitBits - 1 ? p - (kDigitBits - 1) : 0;
      const uint32_t nb = 1u << (p - sh + 1);
      uint32_t* h = hist[cur];
#pragma unroll
      for (int e = 0; e < KPT; ++e) {
        const uint32_t key = k[e];
        if (key != 0u && (key & mask) == prefix) atomicAdd(&h[(key >> sh) & (nb - 1u)], 1u);
      }
      const uint32_t* hs = h;
      if (C > 1) {
        cluster_sync();  // every CTA's counts are in; the other histogram is read by no one
        uint32_t sum = 0u;
        if (tid < (int)nb) {
          uint32_t v[kMaxCluster];
#pragma unroll
          for (int r = 0; r < kMaxCluster; ++r) v[r] = r < C ? remote(h, tid, r) : 0u;
#pragma unroll
          for (int r = 0; r < kMaxCluster; ++r) sum += v[r];
        }
        hsum[tid] = sum;
        hs = hsum;
      }
      hist[cur ^ 1][tid] = 0u;  // the next level's counters
      __syncthreads();
      // The bin holding the need-th largest key, by every thread at once: thread t holds bin
      // t's count, a suffix scan (from the top bin down) over the block gives the keys above
      // each bin, and the one thread whose bin reaches `need` reports it.
      const uint32_t cb = tid < (int)nb ? hs[tid] : 0u;
      uint32_t sfx = cb;  // this warp's bins from this one up
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_down_sync(0xffffffffu, sfx, o);
        if (lane + o < 32) sfx += y;
      }
      if (lane == 0) wtop[warp] = sfx;
      __syncthreads();
      uint32_t wt = wtop[lane], wsfx = wt;  // the warps' totals, suffix-summed over warps
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_down_sync(0xffffffffu, wsfx, o);
        if (lane + o < 32) wsfx += y;
      }
      const uint32_t total = __shfl_sync(0xffffffffu, wsfx, 0);
      const uint32_t above_warp = __shfl_sync(0xffffffffu, wsfx - wt, warp);  // warps above this one
      const uint32_t incl = sfx + above_warp, excl = incl - cb;
      if (C > 1 && level == 0 && total <= need) {  // at most K valid keys: every one is taken
        all_valid = true;
        break;
      }
      if (cb != 0u && excl < need && incl >= need) {
        lvl[0] = (uint32_t)tid;
        lvl[1] = excl;
        lvl[2] = cb;
      }
      __syncthreads();
      const uint32_t T = lvl[0], inbin = lvl[2];
      need -= lvl[1];
      prefix |= T << sh;
      mask |= (nb - 1u) << sh;
      if (inbin == need || sh == 0) break;  // every key of the bin is taken, or keys are equal
      p = sh - 1;
      cur ^= 1;
    }
  }

  // ---- output: taken keys in index order, then the first `need` keys tied at the cut --------
  // a valid key is taken when key & mask > prefix (every valid key when all_valid) and tied
  // at the cut when key & mask == prefix
  uint32_t my_gt = 0u, my_eq = 0u;
#pragma unroll
  for (int e = 0; e < KPT; ++e) {
    const uint32_t kp = k[e] & mask;
    if (k[e] != 0u && (all_valid || kp >= prefix)) {
      if (all_valid || kp > prefix) ++my_gt;
      else ++my_eq;
    }
  }
  // block scan: warp-inclusive sums, then a scan over the warps' totals (lane w: warp w)
  uint32_t ig = my_gt, ie = my_eq;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t yg = __shfl_up_sync(0xffffffffu, ig, o);
    const uint32_t ye = __shfl_up_sync(0xffffffffu, ie, o);
    if (lane >= o) {
      ig += yg;
      ie += ye;
    }
  }
  if (lane == 31) {
    wsum[0][warp] = ig;
    wsum[1][warp] = ie;
  }
  __syncthreads();
  uint32_t sg = wsum[0][lane], se = wsum[1][lane];
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t yg = __shfl_up_sync(0xffffffffu, sg, o);
    const uint32_t ye = __shfl_up_sync(0xffffffffu, se, o);
    if (lane >= o) {
      sg += yg;
      se += ye;
    }
  }
  const uint32_t cta_g = __shfl_sync(0xffffffffu, sg, 31), cta_e = __shfl_sync(0xffffffffu, se, 31);
  uint32_t lg = (warp > 0 ? __shfl_sync(0xffffffffu, sg, (warp - 1) & 31) : 0u) + ig - my_gt;
  uint32_t le = (warp > 0 ? __shfl_sync(0xffffffffu, se, (warp - 1) & 31) : 0u) + ie - my_eq;
  uint32_t G = cta_g;  // taken keys of the whole query
  if (C > 1) {  // this CTA's items follow those of the lower ranks
    if (tid == 0) {
      xch[4] = cta_g;
      xch[5] = cta_e;
    }
    cluster_sync();
    uint32_t rg = lane < C ? remote(xch, 4, lane) : 0u, re = lane < C ? remote(xch, 5, lane) : 0u;
    const uint32_t below_g = lane < rank ? rg : 0u, below_e = lane < rank ? re : 0u;
    uint32_t bg = below_g, be = below_e;
    // the last remote reads of this CTA are done: arrive now, wait just before exiting (the
    // other CTAs may still be reading this one's exchange words until they arrive)
    asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      bg += __shfl_xor_sync(0xffffffffu, bg, o);
      be += __shfl_xor_sync(0xffffffffu, be, o);
      rg += __shfl_xor_sync(0xffffffffu, rg, o);
    }
    lg += bg;
    le += be;
    G = rg;
  }
  const uint32_t tie0 = (uint32_t)K - need;  // first slot of the tied keys
  int32_t* out = a.out_idx + (int64_t)bq * K;
  float* out_s = a.out_score ? a.out_score + (int64_t)bq * K : nullptr;
#pragma unroll
  for (int e = 0; e < KPT; ++e) {
    const uint32_t key = k[e];
    const uint32_t kp = key & mask;
    if (key != 0u && (all_valid || kp >= prefix)) {  // taken, or tied at the cut
      const bool gt = all_valid || kp > prefix;
      if (gt || le < need) {
        const uint32_t slot = gt ? lg : tie0 + le;
        out[slot] = (int32_t)item_label(a, blk, i0 + e);
        if (out_s) out_s[slot] = key_score(key);
      }
      if (gt) ++lg;
      else ++le;
    }
  }
  if (all_valid && rank == 0) {
    for (int i = (int)G + tid; i < K; i += NT) {
      out[i] = -1;
      if (out_s) out_s[i] = -INFINITY;
    }
  }
  if (C > 1) asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");  // see the arrive above
}

// ------------------------------------------------------------------------------------
// host launchers
// ------------------------------------------------------------------------------------
static int pow2_at_least(int x) {
  int p = 32;
  while (p < x) p <<= 1;
  return p;
}

// Reindex scan: one CTA row per (sequence, query), one 128-candidate tile per CTA (512 CTAs
// for 4 queries of 16,384 candidates fit one wave; two tiles per CTA measured 4% slower on the
// whole hier1m step, each CTA's chain then holding two build -> MMA -> epilogue rounds).
static cudaError_t launch_reindex_scan(ScanArgs a, int64_t items, int BQ, cudaStream_t st) {
  a.hipad = a.HI <= 4 ? 4 : (a.HI <= 8 ? 8 : 16);
  a.G = 1;
  a.n_groups = a.Q;
  a.N = a.hipad * 4;
  a.tmem_cols = pow2_at_least(a.N);
  a.tiles_per_cta = 1;
  const int64_t per_cta = (int64_t)a.tiles_per_cta * kRows;
  const dim3 grid((unsigned)((items + per_cta - 1) / per_cta), (unsigned)BQ);
  if (grid.x == 0 || grid.y == 0) return cudaSuccess;
  const size_t smem = 1024 + (size_t)kRows * 128 + (size_t)a.N * 128 + 2 * (size_t)kRawBytes + (size_t)a.N * 4 +
                      (size_t)a.hipad * 4 + 256 * 4 + 16;
  cudaError_t e;
#define CSA2_REINDEX_LAUNCH(HP)                                                                     \
  e = cudaFuncSetAttribute(reindex_scan_kernel<HP>, cudaFuncAttributeMaxDynamicSharedMemorySize,    \
                           (int)smem);                                                              \
  if (e != cudaSuccess) return e;                                                                   \
  e = launch_chained(reindex_scan_kernel<HP>, grid, dim3(kScanThreads), smem, st, 0, a);            \
  if (e != cudaSuccess) return e;
  if (a.hipad == 4) {
    CSA2_REINDEX_LAUNCH(4)
  } else if (a.hipad == 8) {
    CSA2_REINDEX_LAUNCH(8)
  } else {
    CSA2_REINDEX_LAUNCH(16)
  }
#undef CSA2_REINDEX_LAUNCH
  return cudaGetLastError();
}

// CTAs of `fn` that fit on one SM at once, from its register count, its shared memory and
// the device's per-SM limits (registers are allocated per warp in units of 256).
template <typename F>
static cudaError_t resident_ctas(F fn, int dev, int threads, size_t dyn_smem, int* out) {
  cudaFuncAttributes fa;
  cudaError_t e = cudaFuncGetAttributes(&fa, fn);
  if (e != cudaSuccess) return e;
  int regs_sm = 0, smem_sm = 0, reserved = 0, thr_sm = 0, blk_sm = 0;
  if ((e = cudaDeviceGetAttribute(&regs_sm, cudaDevAttrMaxRegistersPerMultiprocessor, dev)) != cudaSuccess ||
      (e = cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev)) != cudaSuccess ||
      (e = cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev)) != cudaSuccess ||
      (e = cudaDeviceGetAttribute(&thr_sm, cudaDevAttrMaxThreadsPerMultiProcessor, dev)) != cudaSuccess ||
      (e = cudaDeviceGetAttribute(&blk_sm, cudaDevAttrMaxBlocksPerMultiprocessor, dev)) != cudaSuccess)
    return e;
  const int warps = (threads + 31) / 32;
  const int regs_cta = warps * (((fa.numRegs * 32) + 255) / 256) * 256;
  int n = blk_sm;
  n = std::min(n, thr_sm / (warps * 32));
  if (regs_cta > 0) n = std::min(n, regs_sm / regs_cta);
  n = std::min(n, (int)((size_t)smem_sm / (dyn_smem + fa.sharedSizeBytes + (size_t)reserved)));
  *out = std::max(n, 1);
  return cudaSuccess;
}

// Flat / hierarchical scan: a few waves of stream_scan_kernel CTAs, each taking a contiguous
// run of at least 8 tiles.
template <int MODE>
static cudaError_t launch_stream(ScanArgs a, int64_t items, int B, cudaStream_t st) {
  a.hipad = a.HI <= 4 ? 4 : (a.HI <= 8 ? 8 : 16);
  // G queries of hipad heads per CTA, N = G * hipad <= 32 columns rounded up to 16 (the
  // smallest N of an M = 128 MMA); the A tile and the accumulator pair take 64 + 2N <= 128
  // columns, so four CTAs' tensor memory fits an SM
  a.G = max(1, min(a.Q, kStreamN / a.hipad));
  a.n_groups = (a.Q + a.G - 1) / a.G;
  // one query stacks its hi and lo rows in one operand of 2 * hipad rows
  a.N = ((a.G == 1 ? 2 : a.G) * a.hipad + 15) / 16 * 16;
  a.tmem_cols = pow2_at_least(kATmemCols + 2 * a.N);
  const int64_t tiles = (items + kRows - 1) / kRows;
  const int64_t rows = (int64_t)B * a.n_groups;
  if (tiles == 0 || rows == 0) return cudaSuccess;
  const size_t smem = 1024 + 4 * (size_t)a.N * 128 + (size_t)kStages * kRawTile +
                      (size_t)a.N * 4 + (size_t)a.G * 8 + (2 * kStages + 3) * 8 + 32;
  // Runs of tiles sized for about `waves` waves of CTAs: 2 when few query rows share the
  // sequence walk, 8 when many do (multi-query verify and prefill, 128 and 256 rows of 4
  // queries), whose longer runs per CTA otherwise leave a tail (8 waves measured 5-7% faster
  // there and no better for 4 or 32 rows).
  const int64_t waves = rows >= 64 ? 8 : 2;
  int dev = 0, sms = 148, occ = 1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
#define CSA2_STREAM_LAUNCH(HP)                                                                          \
  {                                                                                                     \
    auto* fn = stream_scan_kernel<MODE, HP>;                                                            \
    e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);               \
    if (e != cudaSuccess) return e;                                                                     \
    e = cudaFuncSetAttribute(fn, cudaFuncAttributePreferredSharedMemoryCarveout,                        \
                             (int)cudaSharedmemCarveoutMaxShared);                                      \
    if (e != cudaSuccess) return e;                                                                     \
    e = resident_ctas(fn, dev, kStreamThreads, smem, &occ);                                             \
    if (e != cudaSuccess) return e;                                                                     \
    const int64_t slots = (int64_t)sms * (occ > 0 ? occ : 1);                                           \
    int64_t tpc = (tiles * rows + waves * slots - 1) / (waves * slots);                                 \
    tpc = tpc < 8 ? 8 : tpc;                                                                            \
    tpc = tpc > tiles ? tiles : tpc;                                                                    \
    a.tiles_per_cta = (int)tpc;                                                                         \
    const dim3 grid((unsigned)((tiles + tpc - 1) / tpc), (unsigned)rows);                               \
    e = launch_chained(fn, grid, dim3(kStreamThreads), smem, st, 0, a);                                 \
    if (e != cudaSuccess) return e;                                                                     \
  }
  if (a.hipad == 4) {
    CSA2_STREAM_LAUNCH(4)
  } else if (a.hipad == 8) {
    CSA2_STREAM_LAUNCH(8)
  } else {
    CSA2_STREAM_LAUNCH(16)
  }
#undef CSA2_STREAM_LAUNCH
  return cudaGetLastError();
}

// Selection of the K best of `items` keys per query row (blockIdx.y = row).
static cudaError_t launch_select(SelectArgs s, int64_t items, int BQ, cudaStream_t stream) {
  cudaError_t e;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // flat lists with the scan's group maxima, at least one query per SM: one 256-thread CTA per
  // query, four to an SM (verify: 0.974 -> 0.956 ms per step, prefill 1.780 -> 1.755 against
  // select_kernel's one-CTA path; with fewer queries select_kernel's 1024 threads per query
  // finish sooner: full128k's 32 queries took 0.178 ms per step here against 0.172)
  if (s.gmax != nullptr && items > SelShape<2>::kChunk && BQ >= sms) {
    s.csize = 1;
    e = cudaFuncSetAttribute(group_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kGsSmemBytes);
    if (e != cudaSuccess) return e;
    e = launch_chained(group_select_kernel, dim3((unsigned)BQ), dim3(kGsThreads), (size_t)kGsSmemBytes, stream, 0u, s);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
  }
  // Lists whose keys fit the registers of a cluster of at most 8 CTAs, when the clusters of all
  // queries fit two waves: the fewest keys per thread (the most CTAs) that do.  Flat lists with
  // the scan's group maxima and more than 16,384 keys stay with select_kernel's one-CTA group
  // path (full128k: 0.179 ms per step there against 0.205 in 16-key register clusters); the
  // hierarchical block select (131,072 block keys) takes a cluster of 8 16-key CTAs (hier1m
  // 0.521 -> 0.516 ms per step against select_kernel's cluster of 8).
  {
    for (int kpt = 4; kpt <= 16; kpt *= 2) {
      const int64_t c = (items + 1024 * kpt - 1) / (1024 * kpt);
      if (c > kMaxCluster || (c > 1 && (int64_t)BQ * c > 2 * (int64_t)sms) ||
          (kpt == 16 && c > 1 && s.gmax != nullptr))
        continue;
      s.csize = (int)(c < 1 ? 1 : c);
      const dim3 grid((unsigned)s.csize, (unsigned)BQ);
      const unsigned cl = s.csize > 1 ? (unsigned)s.csize : 0u;
      if (kpt == 4)
        e = launch_chained(select_cl_kernel<4>, grid, dim3(1024), 0, stream, cl, s);
      else if (kpt == 8)
        e = launch_chained(select_cl_kernel<8>, grid, dim3(1024), 0, stream, cl, s);
      else
        e = launch_chained(select_cl_kernel<16>, grid, dim3(1024), 0, stream, cl, s);
      if (e != cudaSuccess) return e;
      return cudaGetLastError();
    }
  }
  // Otherwise select_kernel, which stages chunks of keys in shared memory: one CTA for at most
  // 4,096 keys, else one CTA per 16,384 keys, up to 8.
  if (items <= SelShape<2>::kChunk) {
    s.csize = 1;
    e = cudaFuncSetAttribute(select_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, SelShape<2>::kSmem);
    if (e != cudaSuccess) return e;
    e = launch_chained(select_kernel<2>, dim3((unsigned)s.csize, (unsigned)BQ), dim3(kSelThreads),
                       SelShape<2>::kSmem, stream, (unsigned)s.csize, s);
  } else {
    // one CTA per 16,384 keys, up to a cluster of 8; when the queries' clusters would not fit
    // one wave (one CTA per SM), fewer CTAs per query, each walking several chunks: a second
    // wave costs more than the longer walk (full128k, 32 queries of 131,072 keys: 4 CTAs per
    // query measured 7% faster on the whole step than 8)
    int64_t c = (items + SelShape<4>::kChunk - 1) / SelShape<4>::kChunk;
    c = c < 1 ? 1 : (c > kMaxCluster ? kMaxCluster : c);
    // with the scan's group maxima one CTA reads little more than the groups above the
    // threshold (full128k, 32 queries of up to 131,072 keys: 10% faster on the whole step than
    // 4 CTAs walking the keys)
    if (s.gmax != nullptr) c = 1;
    const int64_t fit = (int64_t)sms / (BQ > 0 ? BQ : 1);  // CTAs per query in one wave
    if (c > fit) c = fit < 1 ? 1 : (fit >= 8 ? 8 : (fit >= 4 ? 4 : (fit >= 2 ? 2 : 1)));
    s.csize = (int)c;
    e = cudaFuncSetAttribute(select_kernel<4>, cudaFuncAttributeMaxDynamicSharedMemorySize, SelShape<4>::kSmem);
    if (e != cudaSuccess) return e;
    e = launch_chained(select_kernel<4>, dim3((unsigned)s.csize, (unsigned)BQ), dim3(kSelThreads),
                       SelShape<4>::kSmem, stream, (unsigned)s.csize, s);
  }
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

// Merge: the K best of n_items caller-built keys (0 = no candidate) per query row, each
// item named by its label; keys and labels are rows of key_stride (a multiple of 4).
cudaError_t launch_select_labeled(const uint32_t* keys, const int32_t* labels, int64_t key_stride,
                                  int64_t n_items, int BQ, int K, int32_t* out_idx, float* out_score,
                                  cudaStream_t stream) {
  SelectArgs s = {};
  s.keys = keys;
  s.key_stride = key_stride;
  s.mode = kMerge;
  s.Q = 1;
  s.block = 1;
  s.block_shift = 0;
  s.K = K;
  s.labels = labels;
  s.n_items = n_items;
  s.out_idx = out_idx;
  s.out_score = out_score;
  if (BQ == 0) return cudaSuccess;
  return launch_select(s, n_items, BQ, stream);
}

cudaError_t launch_index(int mode, const float* q, const float* w, const uint8_t* ik_pool,
                         int64_t pool_entries, const int64_t* seq_base, const int32_t* n_vis,
                         const int32_t* blocks, int B, int Q, int HI, int n_blocks, int block,
                         int K, int64_t max_n_vis, int32_t* out_idx, float* out_score,
                         uint32_t* keys, int64_t key_stride, uint32_t* status,
                         cudaStream_t stream, int withheld_tile, uint32_t* gmax, int64_t gstride) {
  ScanArgs a;
  a.withheld_tile = withheld_tile;
  a.gmax = mode == kFlat ? gmax : nullptr;
  a.gstride = gstride;
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
  a.block_shift = __builtin_ctz((unsigned)block);
  a.max_n_vis = max_n_vis;
  a.key_stride = key_stride;
  a.keys = keys;
  a.status = status;
  const int BQ = B * Q;
  if (BQ == 0) return cudaSuccess;
  cudaError_t e;
  if (mode == kFlat)
    e = launch_stream<kFlat>(a, max_n_vis, B, stream);
  else if (mode == kHier)
    e = launch_stream<kHier>(a, max_n_vis, B, stream);
  else
    e = launch_reindex_scan(a, (int64_t)n_blocks * block, BQ, stream);
  if (e != cudaSuccess) return e;

  SelectArgs s;
  s.keys = keys;
  s.key_stride = key_stride;
  s.mode = mode;
  s.Q = Q;
  s.block = block;
  s.block_shift = __builtin_ctz((unsigned)block);
  s.n_blocks = n_blocks;
  s.K = K;
  s.seq_base = seq_base;
  s.n_vis = n_vis;
  s.max_n_vis = max_n_vis;
  s.pool_entries = pool_entries;
  s.blocks = blocks;
  s.labels = nullptr;
  s.n_items = 0;
  s.gmax = mode == kFlat ? gmax : nullptr;
  s.gstride = gstride;
  s.out_idx = out_idx;
  s.out_score = out_score;
  const int64_t items = mode == kFlat ? max_n_vis
                        : mode == kHier ? (max_n_vis + block - 1) / block
                                        : (int64_t)n_blocks * block;
  return launch_select(s, items, BQ, stream);
}

}  // namespace csa2
