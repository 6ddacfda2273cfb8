// Device-side helpers shared by the libcsa2 kernels (sm_100a).
//
// Format facts (P3 = genexis.ai "100만 토큰을 0.9GB에, 딥시크 V4.1 논문이 KV 캐시를 줄인
// 방법", §4비트로 적어도 되는 이유 and §레이어 40개 가운데 4개만 전역 캐시를 만듭니다):
// E2M1 values with one E4M3 scale per 16 channels (288 B per 512-channel entry) and a
// 68 B indexer key (64 B E2M1 codes + fp32 scale).
#pragma once

#include <cstdint>
#include <utility>
#include <cuda_runtime.h>

#include "csa2.h"

namespace csa2 {

constexpr int kD = CSA2_D;
constexpr int kDI = CSA2_DI;
constexpr int kKvBytes = CSA2_KV_ENTRY_BYTES;
constexpr int kIkBytes = CSA2_IK_ENTRY_BYTES;

// Programmatic dependent launch.  Every libcsa2 kernel is launched with programmatic
// stream serialization, so its CTAs may be scheduled while the previous kernel in the
// stream is still running.  Each kernel starts with chain_enter: it lets its own successor
// begin launching, then waits until its predecessor has completed and that kernel's
// writes are visible, before it touches global memory that a library kernel writes.  What
// overlaps is the launch, CTA scheduling and on-chip set-up, plus (attention) the staging
// of the queries: a caller input that no library kernel writes, whose producer has always
// completed by then (a kernel starts early only behind a library kernel).
__device__ __forceinline__ void chain_enter() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
// The two halves of chain_enter, for kernels that first do set-up touching no global
// memory (barrier initialisation, tensor-memory allocation) while the predecessor runs.
__device__ __forceinline__ void chain_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void chain_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Host side: launch `kernel` with programmatic stream serialization, plus a cluster of
// cluster_x CTAs along x when cluster_x > 0.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_chained(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                                  cudaStream_t stream, unsigned cluster_x, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  unsigned n = 0;
  attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[n].val.programmaticStreamSerializationAllowed = 1;
  ++n;
  if (cluster_x > 0) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = cluster_x;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

__device__ __forceinline__ void flag(uint32_t* status, uint32_t bit) {
  if (status) atomicOr(status, bit);
}

// bf16 pair (element 2i in the low half) -> two fp32 values.
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Two non-negative fp32 values -> one byte of two E2M1 codes (lo in bits 3..0), round to
// nearest even, saturating at 6.
__device__ __forceinline__ uint32_t e2m1x2_rn_sat(float lo, float hi) {
  uint16_t r;
  asm("{\n\t.reg .b8 t;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\t"
      "cvt.u16.u8 %0, t;\n\t}"
      : "=h"(r)
      : "f"(hi), "f"(lo));
  return r & 0xFFu;
}

// 8 E2M1 codes (one 32-bit word, code i in bits 4i..4i+3) -> 8 f16, exact (E2M1 values are
// f16 values); code i lands in half i of the result, so the words keep the codes' order.
__device__ __forceinline__ uint4 e2m1x8_f16(uint32_t w) {
  uint4 o;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
      "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
      "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
      : "=r"(o.x), "=r"(o.y), "=r"(o.z), "=r"(o.w)
      : "r"(w));
  return o;
}

// Non-negative fp32 -> E4M3 byte, round to nearest even, saturating at 448.
__device__ __forceinline__ uint32_t e4m3_rn_sat(float x) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(x));
  return r & 0xFFu;
}

// E4M3 byte (sign clear) -> fp32, exact.
__device__ __forceinline__ float e4m3_value(uint32_t s) {
  uint32_t e = (s >> 3) & 15u, m = s & 7u;
  if (e == 0) return __uint2float_rn(m) * 0.001953125f;  // m * 2^-9
  return __uint_as_float(((e + 120u) << 23) | (m << 20));
}

// Order-preserving map of an fp32 score onto uint32 (larger score -> larger key).
// Key 0 is reserved for "no candidate" (it is the image of a negative NaN only).
__device__ __forceinline__ uint32_t score_key(float s) {
  uint32_t b = __float_as_uint(s);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float key_score(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

}  // namespace csa2
