// Per-block NVFP4 encoding shared by the quantizer kernels and the fused
// decode kernel, so that every path produces identical codes and scales.
//
// Every rounding step uses an explicit _rn intrinsic, so no multiply-add is
// contracted.  Thread mapping: one thread owns 8 consecutive elements (a
// "unit"); the two threads of an even/odd lane pair own one 16-element block
// and exchange their half-block maxima with one shuffle.
#pragma once

#include "common.cuh"
#include "kernels.h"
#include "tcgen05.cuh"

namespace nvfp4 {

// Quantize the 8 values this thread owns (half of a 16-block; the partner lane
// lane^1 owns the other half).  All 32 lanes must call it together.
// Returns 8 packed E2M1 nibbles; d_byte receives the block's E4M3 scale; when
// deq != nullptr it receives fl32(fl32(v(c) * d) * s) per element.
__device__ __forceinline__ uint32_t quant_half_block(const float v[8], float s, uint32_t& d_byte,
                                                     float* deq) {
  float a = 0.0f;
#pragma unroll
  for (int i = 0; i < 8; ++i) a = fmaxf(a, fabsf(v[i]));
  a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, 1));
  uint32_t db = 0;
  if (s >= NVFP4_MIN_TENSOR_SCALE) db = f32_to_e4m3(__fdiv_rn(a, __fmul_rn(6.0f, s)));
  const float d = e4m3_value(db);
  const float inv = (d != 0.0f) ? __frcp_rn(__fmul_rn(d, s)) : 0.0f;
  const uint32_t codes =
      f32x8_to_e2m1(__fmul_rn(v[0], inv), __fmul_rn(v[1], inv), __fmul_rn(v[2], inv),
                    __fmul_rn(v[3], inv), __fmul_rn(v[4], inv), __fmul_rn(v[5], inv),
                    __fmul_rn(v[6], inv), __fmul_rn(v[7], inv));
  if (deq != nullptr) {
#pragma unroll
    for (int i = 0; i < 8; ++i) deq[i] = __fmul_rn(__fmul_rn(e2m1_value(codes >> (4 * i)), d), s);
  }
  d_byte = db;
  return codes;
}

// Quantize one whole 16-element block held by one thread: the arithmetic of
// quant_half_block (same block maximum, scale, reciprocal and per-element
// rounding), without the pair exchange and with the per-block work done once.
// Returns the 16 packed E2M1 nibbles, element i in bits 4i..4i+3.
__device__ __forceinline__ uint64_t quant_block16(const float v[16], float s, uint32_t& d_byte, float* deq) {
  float a = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; ++i) a = fmaxf(a, fabsf(v[i]));
  uint32_t db = 0;
  if (s >= NVFP4_MIN_TENSOR_SCALE) db = f32_to_e4m3(__fdiv_rn(a, __fmul_rn(6.0f, s)));
  const float d = e4m3_value(db);
  const float inv = (d != 0.0f) ? __frcp_rn(__fmul_rn(d, s)) : 0.0f;
  const uint32_t lo =
      f32x8_to_e2m1(__fmul_rn(v[0], inv), __fmul_rn(v[1], inv), __fmul_rn(v[2], inv), __fmul_rn(v[3], inv),
                    __fmul_rn(v[4], inv), __fmul_rn(v[5], inv), __fmul_rn(v[6], inv), __fmul_rn(v[7], inv));
  const uint32_t hi =
      f32x8_to_e2m1(__fmul_rn(v[8], inv), __fmul_rn(v[9], inv), __fmul_rn(v[10], inv), __fmul_rn(v[11], inv),
                    __fmul_rn(v[12], inv), __fmul_rn(v[13], inv), __fmul_rn(v[14], inv), __fmul_rn(v[15], inv));
  if (deq != nullptr) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      deq[i] = __fmul_rn(__fmul_rn(e2m1_value(lo >> (4 * i)), d), s);
      deq[8 + i] = __fmul_rn(__fmul_rn(e2m1_value(hi >> (4 * i)), d), s);
    }
  }
  d_byte = db;
  return (uint64_t)lo | ((uint64_t)hi << 32);
}

// quant_block16 for the streaming quantizer: the block maximum arrives as an
// abs key (max of abs_key over the 16 values, so fl32 of it is max |v|), and
// the E4M3 value d and the reciprocal fl32(1 / fl32(d * s)) of each of the 256
// scale codes come from tables filled by make_scale_tables for this s.  Same
// arithmetic as quant_block16, so the same codes and scales.
__device__ __forceinline__ uint64_t quant_block16_tab(const float v[16], uint32_t amax_key, float s,
                                                      const float* d_tab, const float* inv_tab, uint32_t& d_byte,
                                                      float* deq) {
  uint32_t db = 0;
  if (s >= NVFP4_MIN_TENSOR_SCALE) db = f32_to_e4m3(__fdiv_rn(__uint_as_float(amax_key), __fmul_rn(6.0f, s)));
  const float d = d_tab[db], inv = inv_tab[db];
  const uint32_t lo =
      f32x8_to_e2m1(__fmul_rn(v[0], inv), __fmul_rn(v[1], inv), __fmul_rn(v[2], inv), __fmul_rn(v[3], inv),
                    __fmul_rn(v[4], inv), __fmul_rn(v[5], inv), __fmul_rn(v[6], inv), __fmul_rn(v[7], inv));
  const uint32_t hi =
      f32x8_to_e2m1(__fmul_rn(v[8], inv), __fmul_rn(v[9], inv), __fmul_rn(v[10], inv), __fmul_rn(v[11], inv),
                    __fmul_rn(v[12], inv), __fmul_rn(v[13], inv), __fmul_rn(v[14], inv), __fmul_rn(v[15], inv));
  if (deq != nullptr) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      deq[i] = __fmul_rn(__fmul_rn(e2m1_value(lo >> (4 * i)), d), s);
      deq[8 + i] = __fmul_rn(__fmul_rn(e2m1_value(hi >> (4 * i)), d), s);
    }
  }
  d_byte = db;
  return (uint64_t)lo | ((uint64_t)hi << 32);
}
// Fill the 256-entry tables of quant_block16_tab for tensor scale s (all
// threads of the block; the caller synchronises before use).
__device__ __forceinline__ void make_scale_tables(float s, float* d_tab, float* inv_tab) {
  for (int b = threadIdx.x; b < 256; b += blockDim.x) {
    const float d = e4m3_value((uint32_t)b);
    d_tab[b] = d;
    inv_tab[b] = (d != 0.0f) ? __frcp_rn(__fmul_rn(d, s)) : 0.0f;
  }
}
// Max abs key of 16 values given as 8 words of packed bf16 pairs: the key of
// a bf16 value is its 15 magnitude bits in the high half of the word.
__device__ __forceinline__ uint32_t bf16x16_amax_key(const uint4& a, const uint4& b) {
  uint32_t m = __vmaxu2(a.x & 0x7FFF7FFFu, a.y & 0x7FFF7FFFu);
  m = __vmaxu2(m, a.z & 0x7FFF7FFFu);
  m = __vmaxu2(m, a.w & 0x7FFF7FFFu);
  m = __vmaxu2(m, b.x & 0x7FFF7FFFu);
  m = __vmaxu2(m, b.y & 0x7FFF7FFFu);
  m = __vmaxu2(m, b.z & 0x7FFF7FFFu);
  m = __vmaxu2(m, b.w & 0x7FFF7FFFu);
  return max(m & 0xFFFF0000u, m << 16);
}

// Load 16 consecutive elements (32-byte aligned for bf16, 64-byte for fp32) as fp32.
__device__ __forceinline__ void load16(const __nv_bfloat16* p, float v[16]) {
  load8(p, v);
  load8(p + 8, v + 8);
}
__device__ __forceinline__ void load16(const float* p, float v[16]) {
  load8(p, v);
  load8(p + 8, v + 8);
}

// Store the codes (8 bytes) and scale of block b of `row` (block-per-thread kernels).
__device__ __forceinline__ void store_block16(const QOut& q, int64_t row, int b, uint64_t codes, uint32_t d_byte) {
  *reinterpret_cast<uint64_t*>(q.codes + row * (q.cols >> 1) + (int64_t)b * 8) = codes;
  q.scales[scale_offset(row, b, q.cols >> 4, q.tiled)] = (uint8_t)d_byte;
}

__device__ __forceinline__ void store_half_block(const QOut& q, int64_t row, int64_t col8,
                                                 uint32_t codes, uint32_t d_byte) {
  *reinterpret_cast<uint32_t*>(q.codes + row * (q.cols >> 1) + col8 * 4) = codes;
  if ((col8 & 1) == 0) q.scales[scale_offset(row, col8 >> 1, q.cols >> 4, q.tiled)] = (uint8_t)d_byte;
}

template <typename T>
struct Raw8;
template <>
struct Raw8<__nv_bfloat16> {
  uint4 u;
  __device__ __forceinline__ void load(const __nv_bfloat16* p) { u = __ldg(reinterpret_cast<const uint4*>(p)); }
  __device__ __forceinline__ void store_smem(__nv_bfloat16* p) const { *reinterpret_cast<uint4*>(p) = u; }
  __device__ __forceinline__ void zero() { u = make_uint4(0u, 0u, 0u, 0u); }
  __device__ __forceinline__ void get(float v[8]) const {
    v[0] = __uint_as_float(u.x << 16); v[1] = __uint_as_float(u.x & 0xFFFF0000u);
    v[2] = __uint_as_float(u.y << 16); v[3] = __uint_as_float(u.y & 0xFFFF0000u);
    v[4] = __uint_as_float(u.z << 16); v[5] = __uint_as_float(u.z & 0xFFFF0000u);
    v[6] = __uint_as_float(u.w << 16); v[7] = __uint_as_float(u.w & 0xFFFF0000u);
  }
  // max over the 8 elements of abs_key (the fp32 bit pattern of |x|), on the
  // packed halves: |bf16| bit patterns order like the values, NaN/Inf included
  __device__ __forceinline__ uint32_t abs_key_max() const {
    uint32_t m;
    asm("max.u16x2 %0, %1, %2;" : "=r"(m) : "r"(u.x & 0x7FFF7FFFu), "r"(u.y & 0x7FFF7FFFu));
    asm("max.u16x2 %0, %0, %1;" : "+r"(m) : "r"(u.z & 0x7FFF7FFFu));
    asm("max.u16x2 %0, %0, %1;" : "+r"(m) : "r"(u.w & 0x7FFF7FFFu));
    return max(m << 16, m & 0xFFFF0000u);
  }
};
template <>
struct Raw8<float> {
  float4 a, b;
  __device__ __forceinline__ void load(const float* p) {
    a = __ldg(reinterpret_cast<const float4*>(p));
    b = __ldg(reinterpret_cast<const float4*>(p) + 1);
  }
  __device__ __forceinline__ void store_smem(float* p) const {
    reinterpret_cast<float4*>(p)[0] = a;
    reinterpret_cast<float4*>(p)[1] = b;
  }
  __device__ __forceinline__ void zero() { a = b = make_float4(0.0f, 0.0f, 0.0f, 0.0f); }
  __device__ __forceinline__ void get(float v[8]) const {
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  }
  __device__ __forceinline__ uint32_t abs_key_max() const {
    return max(max(max(abs_key(a.x), abs_key(a.y)), max(abs_key(a.z), abs_key(a.w))),
               max(max(abs_key(b.x), abs_key(b.y)), max(abs_key(b.z), abs_key(b.w))));
  }
};

// Cluster-wide maximum of `key` (every thread of the cluster, at most 32 CTAs,
// calls it with the same `slot`, a word this CTA publishes to its peers).
// Result in every thread.
__device__ __forceinline__ uint32_t cluster_max_u32(uint32_t key, uint32_t* red, uint32_t* slot) {
  const uint32_t m = block_max_u32(key, red);
  if (threadIdx.x == 0) *slot = m;
  tc::cluster_sync();  // release/acquire: every CTA's slot is visible cluster-wide
  const uint32_t lane = threadIdx.x & 31, n = tc::cluster_nctarank();
  uint32_t a = 0u;
  if (lane < n) a = __float_as_uint(tc::ld_cluster_f32(tc::mapa_shared(tc::saddr(slot), lane)));
  return warp_max_u32(a);
}

// Tensor scale from a |.| maximum key: fl32(amax / 2688), or 0 with
// NVFP4_ERR_NONFINITE for an Inf/NaN maximum (reported once per cluster).
__device__ __forceinline__ float scale_from_key(uint32_t a, bool reporter, int* st) {
  if (a >= 0x7F800000u) {
    if (reporter) report_status(st, NVFP4_ERR_NONFINITE);
    return 0.0f;
  }
  return __fdiv_rn(__uint_as_float(a), 2688.0f);
}

}  // namespace nvfp4
