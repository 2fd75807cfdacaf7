// Device helpers shared by the NVFP4 kernels (sm_100a only).
//
// Number formats (ARCQuant blog post, section 1; Replay the Curvature abstract):
//   E2M1 code  = sign (bit 3) | magnitude index (bits 0-2) onto {0,.5,1,1.5,2,3,4,6}
//   E4M3 scale = bias-7 float with 3 mantissa bits, max 448, subnormal step 2^-9.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "nvfp4.h"

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "this library targets sm_100a only"
#endif

namespace nvfp4 {

// ---------------------------------------------------------------- workspace
// The caller-owned workspace starts with this header; the RMSNorm variant
// stores one fp32 rinv per row after it.  Every kernel that uses a counter or
// a running maximum leaves it at zero when it finishes.
struct WsHeader {
  unsigned int amax_bits[2];   // running max of |x| (resp. |r|) as fp32 bit patterns
  unsigned int arrive[2];      // CTA arrival counters (last-CTA-finishes pattern)
  unsigned int reserved[60];
};
static_assert(sizeof(WsHeader) == 256, "workspace header is 256 bytes");
constexpr size_t kWsHeaderBytes = 256;

// Tensor scales below this are treated as an all-zero tensor (every d = 0).
#define NVFP4_MIN_TENSOR_SCALE 0x1p-110f

__device__ __forceinline__ void report_status(int* st, int code) {
  if (st != nullptr) atomicCAS(st, 0, code);
}

// ------------------------------------------------------------ conversions

// fp32 -> E4M3 byte, round-to-nearest-even, saturating to +-448.
__device__ __forceinline__ uint32_t f32_to_e4m3(float x) {
  uint16_t pair;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %1;" : "=h"(pair) : "f"(x));
  return pair & 0xFFu;
}

// Eight fp32 -> eight E2M1 nibbles (RNE, saturating to +-6); v0 in bits 0-3,
// v1 in bits 4-7, ..., v7 in bits 28-31.  The PTX conversion stores its first
// source operand in the high nibble of each byte.
__device__ __forceinline__ uint32_t f32x8_to_e2m1(float v0, float v1, float v2, float v3,
                                                  float v4, float v5, float v6, float v7) {
  uint32_t packed;
  asm("{\n\t.reg .b8 q0, q1, q2, q3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 q0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 q1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 q2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 q3, %8, %7;\n\t"
      "mov.b32 %0, {q0, q1, q2, q3};\n\t}"
      : "=r"(packed)
      : "f"(v0), "f"(v1), "f"(v2), "f"(v3), "f"(v4), "f"(v5), "f"(v6), "f"(v7));
  return packed;
}

// E2M1 nibble -> fp32 value, by construction from the bit fields.
__device__ __forceinline__ float e2m1_value(uint32_t c) {
  const uint32_t m = c & 7u;
  const float mag = (m < 2u) ? 0.5f * (float)m
                             : __uint_as_float((((m >> 1) + 126u) << 23) | ((m & 1u) << 22));
  return (c & 8u) ? -mag : mag;
}

// E4M3 byte (non-negative, finite) -> fp32 value.
__device__ __forceinline__ float e4m3_value(uint32_t b) {
  const uint32_t e = (b >> 3) & 15u, m = b & 7u;
  return (e == 0u) ? (float)m * 0x1p-9f : __uint_as_float(((e + 120u) << 23) | (m << 20));
}

// |x| as an order-preserving unsigned key; NaN/Inf map to >= 0x7F800000.
__device__ __forceinline__ uint32_t abs_key(float x) { return __float_as_uint(x) & 0x7FFFFFFFu; }

// ---------------------------------------------------------------- loads

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t h) { return __uint_as_float(h << 16); }

// Load 8 consecutive elements as fp32 (16-byte aligned source).
__device__ __forceinline__ void load8(const __nv_bfloat16* p, float v[8]) {
  const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
  v[0] = __uint_as_float(u.x << 16); v[1] = __uint_as_float(u.x & 0xFFFF0000u);
  v[2] = __uint_as_float(u.y << 16); v[3] = __uint_as_float(u.y & 0xFFFF0000u);
  v[4] = __uint_as_float(u.z << 16); v[5] = __uint_as_float(u.z & 0xFFFF0000u);
  v[6] = __uint_as_float(u.w << 16); v[7] = __uint_as_float(u.w & 0xFFFF0000u);
}
__device__ __forceinline__ void load8(const float* p, float v[8]) {
  const float4 a = __ldg(reinterpret_cast<const float4*>(p));
  const float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

__device__ __forceinline__ float load1(const __nv_bfloat16* p) {
  return bf16_bits_to_f32(*reinterpret_cast<const uint16_t*>(p));
}
__device__ __forceinline__ float load1(const float* p) { return *p; }

// Two fp32 -> packed bf16x2 (round to nearest even); `lo` in the low half.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

// ------------------------------------------------------------ scale layout

// Byte offset of block scale (row r, block b) of a matrix with nblk = cols/16 blocks.
__device__ __forceinline__ int64_t scale_offset(int64_t r, int64_t b, int64_t nblk, bool tiled) {
  if (!tiled) return r * nblk + b;
  const int64_t katoms = (nblk + 3) >> 2;
  return ((r >> 7) * katoms + (b >> 2)) * 512 + (r & 31) * 16 + ((r >> 5) & 3) * 4 + (b & 3);
}

// ------------------------------------------------- division by an invariant
// n / d for any 32-bit n and 1 <= d < 2^32 by one multiply-high, one
// subtract, one add and two shifts (Granlund and Montgomery, "Division by
// invariant integers using multiplication", PLDI 1994, section 4).
struct DivMagic {
  uint32_t m, s1, s2;
};
inline DivMagic make_div_magic(uint32_t d) {
  uint32_t l = 0;
  while (l < 32 && (uint64_t(1) << l) < d) ++l;                  // ceil(log2 d)
  const uint64_t m = (((uint64_t(1) << 32) * ((uint64_t(1) << l) - d)) / d) + 1;
  return DivMagic{(uint32_t)m, l < 1 ? l : 1u, l > 1 ? l - 1 : 0u};
}
__device__ __forceinline__ uint32_t div_invariant(uint32_t n, const DivMagic& dm) {
  const uint32_t t1 = __umulhi(dm.m, n);
  return (t1 + ((n - t1) >> dm.s1)) >> dm.s2;
}

// ------------------------------------------------------------ reductions

__device__ __forceinline__ uint32_t warp_max_u32(uint32_t v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = max(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
  return v;
}

__device__ __forceinline__ double warp_sum_f64(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  return v;
}

// Block-wide max of an unsigned key; result valid in every thread.
// `red` must hold blockDim.x / 32 words.
__device__ __forceinline__ uint32_t block_max_u32(uint32_t v, uint32_t* red) {
  v = warp_max_u32(v);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31, nw = blockDim.x >> 5;
  __syncthreads();
  if (l == 0) red[w] = v;
  __syncthreads();
  uint32_t r = (l < nw) ? red[l] : 0u;
  return warp_max_u32(r);
}

// Block-wide sum of doubles holding exact integers (< 2^53 in total).
__device__ __forceinline__ double block_sum_f64(double v, double* red) {
  v = warp_sum_f64(v);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31, nw = blockDim.x >> 5;
  __syncthreads();
  if (l == 0) red[w] = v;
  __syncthreads();
  double r = (l < nw) ? red[l] : 0.0;
  return warp_sum_f64(r);
}

}  // namespace nvfp4
