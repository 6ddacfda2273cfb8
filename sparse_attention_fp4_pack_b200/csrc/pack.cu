// a1: pack new global-KV entries into the FP4 layout.
//
// P3 (genexis.ai "100만 토큰을 0.9GB에, 딥시크 V4.1 논문이 KV 캐시를 줄인 방법"):
//   §레이어 40개 가운데 4개만 전역 캐시를 만듭니다 — 288 B FP4 main KV (256 B values +
//   32 B scales) + 68 B indexer key per entry; encoder entries cover 2 tokens.
//   §4비트로 적어도 되는 이유 — NVFP4 without the second-level global scale: one 8-bit
//   scale per 16 channels.
//
// One warp packs one entry: lane l owns main-KV block l (channels 16l..16l+15, 32 B of
// bf16 per token, so a warp reads 1 KB contiguous) and indexer dims 4l..4l+3.  The
// kernel is HBM-bound (1280 B read + 356 B written per 1:1 entry), so the per-element
// work is kept to a few instructions:
//   * the main-KV quotient x/scale is formed from |x| with a correctly rounded
//     reciprocal r = 1/scale and one FMA correction (Markstein's refinement,
//     q = y0 + r*(|x| - scale*y0), y0 = |x|*r).  For every finite x whose block scale is
//     scale, the E2M1 code of q equals the code of the IEEE quotient: scales have at
//     most 4 significant bits, so the exact quotient is never within half an ulp of an
//     E2M1 rounding midpoint unless it equals it; the parity tests check this over every
//     bf16 value against every scale.  The sign bit is taken from x itself.
//   * the indexer-key quotient uses IEEE division (its scale is a full fp32 value).
#include <cuda_bf16.h>

#include "csa2_device.cuh"

namespace csa2 {

__device__ __forceinline__ float refined_quot(float a, float sd, float r) {
  float y0 = a * r;
  float e = fmaf(-y0, sd, a);
  return fmaf(e, r, y0);
}

// Main-KV block `lane` of an entry (x: its 16 channels, already pair-averaged at ratio 2)
// and indexer dims 4 lane .. 4 lane + 3 (ia, ib: the bf16 of the entry's one or two
// tokens), encoded into the entry at ek / ei.
__device__ __forceinline__ void encode_entry(int lane, const float (&x)[16], uint2 ia, uint2 ib, int ratio,
                                             uint8_t* ek, uint8_t* ei) {
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(x[i]));
  const uint32_t s = e4m3_rn_sat(__fdiv_rn(amax, 6.0f));
  const float sd = e4m3_value(s);
  uint32_t c0 = 0, c1 = 0;
  if (sd != 0.0f) {
    const float r = __frcp_rn(sd);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      float q0 = refined_quot(fabsf(x[2 * i]), sd, r);
      float q1 = refined_quot(fabsf(x[2 * i + 1]), sd, r);
      uint32_t byte = e2m1x2_rn_sat(q0, q1);
      byte |= ((__float_as_uint(x[2 * i]) >> 31) << 3) | ((__float_as_uint(x[2 * i + 1]) >> 31) << 7);
      if (i < 4)
        c0 |= byte << (8 * i);
      else
        c1 |= byte << (8 * (i - 4));
    }
  }
  __stcs(reinterpret_cast<uint2*>(ek) + lane, make_uint2(c0, c1));
  ek[256 + lane] = (uint8_t)s;

  // ---- indexer key dims 4*lane .. 4*lane+3 ------------------------------------------
  float y[4];
  {
    const uint2 a = ia;
    if (ratio == 1) {
      y[0] = bf16_lo(a.x); y[1] = bf16_hi(a.x); y[2] = bf16_lo(a.y); y[3] = bf16_hi(a.y);
    } else {
      const uint2 b = ib;
      y[0] = (bf16_lo(a.x) + bf16_lo(b.x)) * 0.5f;
      y[1] = (bf16_hi(a.x) + bf16_hi(b.x)) * 0.5f;
      y[2] = (bf16_lo(a.y) + bf16_lo(b.y)) * 0.5f;
      y[3] = (bf16_hi(a.y) + bf16_hi(b.y)) * 0.5f;
    }
  }
  float im = fmaxf(fmaxf(fabsf(y[0]), fabsf(y[1])), fmaxf(fabsf(y[2]), fabsf(y[3])));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) im = fmaxf(im, __shfl_xor_sync(0xffffffffu, im, o));
  const float is = __fdiv_rn(im, 6.0f);
  uint32_t ic = 0;
  if (is != 0.0f) {
    uint32_t b0 = e2m1x2_rn_sat(__fdiv_rn(fabsf(y[0]), is), __fdiv_rn(fabsf(y[1]), is));
    uint32_t b1 = e2m1x2_rn_sat(__fdiv_rn(fabsf(y[2]), is), __fdiv_rn(fabsf(y[3]), is));
    b0 |= ((__float_as_uint(y[0]) >> 31) << 3) | ((__float_as_uint(y[1]) >> 31) << 7);
    b1 |= ((__float_as_uint(y[2]) >> 31) << 3) | ((__float_as_uint(y[3]) >> 31) << 7);
    ic = b0 | (b1 << 8);
  }
  reinterpret_cast<uint16_t*>(ei)[lane] = (uint16_t)ic;
  if (lane == 0) *reinterpret_cast<float*>(ei + 64) = is;
}

__global__ void __launch_bounds__(256) pack_kv_kernel(const uint16_t* __restrict__ kv,
                                                      const uint16_t* __restrict__ ik, int64_t E,
                                                      int ratio, const int64_t* __restrict__ dst,
                                                      int64_t pool_entries,
                                                      uint8_t* __restrict__ kv_pool,
                                                      uint8_t* __restrict__ ik_pool,
                                                      uint32_t* status) {
  chain_enter();
  const int lane = threadIdx.x & 31;
  const int64_t warp0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  for (int64_t j = warp0; j < E; j += nwarps) {
    const int64_t d = dst ? dst[j] : j;
    if (d < 0 || d >= pool_entries) {
      if (lane == 0) flag(status, CSA2_DEV_BAD_INDEX);
      continue;
    }
    // every load of the entry is issued before any arithmetic: one memory round trip
    const uint2* pi = reinterpret_cast<const uint2*>(ik + (j * ratio) * kDI) + lane;
    const uint2 ia = __ldcs(pi);
    const uint2 ib = ratio == 1 ? make_uint2(0u, 0u) : __ldcs(pi + kDI / 4);
    // ---- main KV block `lane` -------------------------------------------------------
    float x[16];
    {
      const uint4* p0 = reinterpret_cast<const uint4*>(kv + (j * ratio) * kD) + lane * 2;
      uint4 a0 = __ldcs(p0), a1 = __ldcs(p0 + 1);
      uint32_t w[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      if (ratio == 1) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          x[2 * i] = bf16_lo(w[i]);
          x[2 * i + 1] = bf16_hi(w[i]);
        }
      } else {
        const uint4* p1 = p0 + kD / 8;  // next token
        uint4 b0 = __ldcs(p1), b1 = __ldcs(p1 + 1);
        uint32_t v[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          x[2 * i] = (bf16_lo(w[i]) + bf16_lo(v[i])) * 0.5f;
          x[2 * i + 1] = (bf16_hi(w[i]) + bf16_hi(v[i])) * 0.5f;
        }
      }
    }
    encode_entry(lane, x, ia, ib, ratio, kv_pool + d * kKvBytes, ik_pool + d * kIkBytes);
  }
}

cudaError_t launch_pack_kv(const void* kv, const void* ik, int64_t T, int ratio,
                           const int64_t* dst, int64_t pool_entries, uint8_t* kv_pool,
                           uint8_t* ik_pool, uint32_t* status, cudaStream_t stream, int num_sms) {
  const int64_t E = T / ratio;
  if (E == 0) return cudaSuccess;
  const int threads = 256;
  int64_t blocks = (E + 7) / 8;
  const int64_t cap = (int64_t)num_sms * 16;  // 16 resident 256-thread blocks per SM
  if (blocks > cap) blocks = cap;
  cudaError_t e = launch_chained(pack_kv_kernel, dim3((unsigned)blocks), dim3(threads), 0, stream, 0,
                                 static_cast<const uint16_t*>(kv), static_cast<const uint16_t*>(ik), E, ratio,
                                 dst, pool_entries, kv_pool, ik_pool, status);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

// ------------------------------------------------------------------------------------
// Producer: RMSNorm + rotation of the raw main-KV tokens, then the same encoding (P3
// §4비트로 적어도 되는 이유: cached values are normalised and rotated before caching, which
// bounds them by sqrt(512)).  Per token, with every operation one fp32 rounding (no
// contraction):
//   S = sum of x_c^2: halving within each 16-channel block, then over the 32 block sums
//       (lane l holds block l: in-lane halving, then an xor butterfly 16, 8, 4, 2, 1);
//   r = 1 / sqrt(S / 512 + eps) (add, square root, reciprocal: each correctly rounded);
//   n_c = x_c r (times gamma_c when a gain is given);
//   pairs (2i, 2i+1) rotated by cos/sin[pos][i]: (n_2i c - n_2i+1 s, n_2i s + n_2i+1 c);
//   the result rounded to bf16, then packed like csa2_pack_kv packs bf16 tokens.
// ------------------------------------------------------------------------------------
struct NormArgs {
  const uint16_t* kv;
  const uint16_t* ik;
  int64_t E;
  int ratio;
  const int64_t* pos;
  const float* rope_cos;
  const float* rope_sin;
  int64_t n_pos;
  const float* gamma;
  float eps;
  const int64_t* dst;
  int64_t pool_entries;
  uint8_t* kv_pool;
  uint8_t* ik_pool;
  uint32_t* status;
};

// Block `lane` of one raw token (its bf16 in w), normalised and rotated at table row p,
// rounded to bf16, as fp32 values.
__device__ __forceinline__ void norm_rope_block(const NormArgs& a, int lane, const uint32_t (&w)[8], int64_t p,
                                                float (&out)[16]) {
  float x[16], q[16];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    x[2 * i] = bf16_lo(w[i]);
    x[2 * i + 1] = bf16_hi(w[i]);
  }
#pragma unroll
  for (int i = 0; i < 16; ++i) q[i] = __fmul_rn(x[i], x[i]);
#pragma unroll
  for (int h = 8; h >= 1; h >>= 1)
#pragma unroll
    for (int i = 0; i < h; ++i) q[i] = __fadd_rn(q[i], q[i + h]);
  float S = q[0];
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) S = __fadd_rn(S, __shfl_xor_sync(0xffffffffu, S, o));
  const float r = __frcp_rn(__fsqrt_rn(__fadd_rn(__fmul_rn(S, 0.001953125f), a.eps)));  // S / 512 is exact
  float n[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) n[i] = __fmul_rn(x[i], r);
  if (a.gamma) {
    const float4* g4 = reinterpret_cast<const float4*>(a.gamma) + lane * 4;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float4 g = __ldg(g4 + k);
      n[4 * k] = __fmul_rn(n[4 * k], g.x);
      n[4 * k + 1] = __fmul_rn(n[4 * k + 1], g.y);
      n[4 * k + 2] = __fmul_rn(n[4 * k + 2], g.z);
      n[4 * k + 3] = __fmul_rn(n[4 * k + 3], g.w);
    }
  }
  const float4* c4 = reinterpret_cast<const float4*>(a.rope_cos + p * (kD / 2)) + lane * 2;
  const float4* s4 = reinterpret_cast<const float4*>(a.rope_sin + p * (kD / 2)) + lane * 2;
  const float4 ca = __ldg(c4), cb = __ldg(c4 + 1), sa = __ldg(s4), sb = __ldg(s4 + 1);
  const float c[8] = {ca.x, ca.y, ca.z, ca.w, cb.x, cb.y, cb.z, cb.w};
  const float s[8] = {sa.x, sa.y, sa.z, sa.w, sb.x, sb.y, sb.z, sb.w};
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const float y0 = __fsub_rn(__fmul_rn(n[2 * k], c[k]), __fmul_rn(n[2 * k + 1], s[k]));
    const float y1 = __fadd_rn(__fmul_rn(n[2 * k], s[k]), __fmul_rn(n[2 * k + 1], c[k]));
    out[2 * k] = __bfloat162float(__float2bfloat16_rn(y0));
    out[2 * k + 1] = __bfloat162float(__float2bfloat16_rn(y1));
  }
}

__global__ void __launch_bounds__(256) pack_kv_normed_kernel(NormArgs a) {
  chain_enter();
  const int lane = threadIdx.x & 31;
  const int64_t warp0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  for (int64_t j = warp0; j < a.E; j += nwarps) {
    const int64_t d = a.dst ? a.dst[j] : j;
    const int64_t p0 = a.pos[j * a.ratio];
    const int64_t p1 = a.ratio == 2 ? a.pos[j * a.ratio + 1] : p0;
    if (d < 0 || d >= a.pool_entries || p0 < 0 || p0 >= a.n_pos || p1 < 0 || p1 >= a.n_pos) {
      if (lane == 0) flag(a.status, CSA2_DEV_BAD_INDEX);
      continue;
    }
    const uint2* pi = reinterpret_cast<const uint2*>(a.ik + (j * a.ratio) * kDI) + lane;
    const uint2 ia = __ldcs(pi);
    const uint2 ib = a.ratio == 1 ? make_uint2(0u, 0u) : __ldcs(pi + kDI / 4);
    const uint4* pk = reinterpret_cast<const uint4*>(a.kv + (j * a.ratio) * kD) + lane * 2;
    float x[16];
    {
      const uint4 a0 = __ldcs(pk), a1 = __ldcs(pk + 1);
      const uint32_t w[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      norm_rope_block(a, lane, w, p0, x);
    }
    if (a.ratio == 2) {  // the second token at its own position, then the pair mean
      const uint4 b0 = __ldcs(pk + kD / 8), b1 = __ldcs(pk + kD / 8 + 1);
      const uint32_t v[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
      float y[16];
      norm_rope_block(a, lane, v, p1, y);
#pragma unroll
      for (int i = 0; i < 16; ++i) x[i] = (x[i] + y[i]) * 0.5f;
    }
    encode_entry(lane, x, ia, ib, a.ratio, a.kv_pool + d * kKvBytes, a.ik_pool + d * kIkBytes);
  }
}

cudaError_t launch_pack_kv_normed(const void* kv, const void* ik, int64_t T, int ratio, const int64_t* pos,
                                  const float* rope_cos, const float* rope_sin, int64_t n_pos, const float* gamma,
                                  float eps, const int64_t* dst, int64_t pool_entries, uint8_t* kv_pool,
                                  uint8_t* ik_pool, uint32_t* status, cudaStream_t stream, int num_sms) {
  NormArgs a;
  a.kv = static_cast<const uint16_t*>(kv);
  a.ik = static_cast<const uint16_t*>(ik);
  a.E = T / ratio;
  a.ratio = ratio;
  a.pos = pos;
  a.rope_cos = rope_cos;
  a.rope_sin = rope_sin;
  a.n_pos = n_pos;
  a.gamma = gamma;
  a.eps = eps;
  a.dst = dst;
  a.pool_entries = pool_entries;
  a.kv_pool = kv_pool;
  a.ik_pool = ik_pool;
  a.status = status;
  if (a.E == 0) return cudaSuccess;
  int64_t blocks = (a.E + 7) / 8;
  const int64_t cap = (int64_t)num_sms * 16;
  if (blocks > cap) blocks = cap;
  cudaError_t e = launch_chained(pack_kv_normed_kernel, dim3((unsigned)blocks), dim3(256), 0, stream, 0, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace csa2
