// MXFP4 activation quantizer (a NEXT row of the hot path), sm_100a.
//
// MX format: 32-element blocks of E2M1 values sharing one E8M0 scale, a power
// of two 2^(b - 127); no tensor scale (ARCQuant blog sections 2.2 and 4.2: MX
// formats use E8M0 scales, step 2^1, and 32-element blocks).  Scale rule
// (shared exponent; the pages give none): b = floor(log2 amax_b) - 2 + 127,
// clamped at 0, and 0 for an all-zero block.  With an fp32 block maximum of
// biased exponent E (E = 0 for zero and subnormals) that is max(E - 2, 0).
// Elements: E2M1_RNE_satfinite(x * 2^-(b - 127)); the multiply by a power of
// two is exact for every element the rounding does not send to zero.  The
// residue (ResServe abstract: FP4 base plus FP4 residue) is
// R = fl32(x - v(code) 2^(b-127)), quantized the same way with its own scales.
//
// One pass over X (no tensor scale to wait for): one thread per 32-element
// block, loads of the next block in flight while the current one is encoded.
#include "common.cuh"
#include "kernels.h"
#include "quant_common.cuh"

namespace nvfp4 {
namespace {

// E8M0 byte of a block from the abs key of its largest element (order-
// preserving fp32 bits); keys of NaN/Inf give 253 (reported separately).
__device__ __forceinline__ uint32_t mx_scale_byte(uint32_t amax_key) {
  const int e = (int)(amax_key >> 23);
  return (uint32_t)max(e - 2, 0);
}

// 2^-(b - 127) as fp32 (b <= 253: the exponent 127 - (b - 127) stays in range).
__device__ __forceinline__ float mx_inv_scale(uint32_t b) {
  const int t = 254 - (int)b;                  // biased exponent of 2^(127 - b)
  return t >= 1 ? __uint_as_float((uint32_t)t << 23) : 0x1p-127f;
}

__device__ __forceinline__ float mx_scale(uint32_t b) {
  return b >= 1 ? __uint_as_float(b << 23) : 0x1p-127f;   // 2^(b - 127)
}

// Encode 32 values; returns the scale byte and writes 16 bytes of codes.
__device__ __forceinline__ uint32_t mx_block(const float v[32], uint4& packed, float* deq) {
  uint32_t key = 0;
#pragma unroll
  for (int i = 0; i < 32; ++i) key = max(key, abs_key(v[i]));
  const uint32_t b = mx_scale_byte(key);
  const float inv = mx_inv_scale(b);
  uint32_t w[4];
#pragma unroll
  for (int g = 0; g < 4; ++g)
    w[g] = f32x8_to_e2m1(__fmul_rn(v[8 * g], inv), __fmul_rn(v[8 * g + 1], inv), __fmul_rn(v[8 * g + 2], inv),
                         __fmul_rn(v[8 * g + 3], inv), __fmul_rn(v[8 * g + 4], inv), __fmul_rn(v[8 * g + 5], inv),
                         __fmul_rn(v[8 * g + 6], inv), __fmul_rn(v[8 * g + 7], inv));
  packed = make_uint4(w[0], w[1], w[2], w[3]);
  if (deq != nullptr) {
    const float sc = mx_scale(b);
#pragma unroll
    for (int i = 0; i < 32; ++i) deq[i] = __fmul_rn(e2m1_value(w[i >> 3] >> (4 * (i & 7))), sc);
  }
  return b;
}

template <typename T, bool RES>
__global__ void __launch_bounds__(256) k_mx_quant(const T* __restrict__ x, int64_t M, int64_t K, int64_t ldx,
                                                  uint8_t* codes, uint8_t* scales, uint8_t* r_codes,
                                                  uint8_t* r_scales, bool tiled, int* st) {
  const int64_t nb = K / 32, nblk = M * nb;
  uint32_t bad = 0;
  for (int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; j < nblk; j += (int64_t)gridDim.x * blockDim.x) {
    const int64_t row = j / nb, b = j - row * nb;
    const T* p = x + row * ldx + b * 32;
    float v[32];
#pragma unroll
    for (int g = 0; g < 4; ++g) load8(p + 8 * g, v + 8 * g);
    float deq[32];
    uint4 packed;
    const uint32_t sb = mx_block(v, packed, RES ? deq : nullptr);
    bad = max(bad, sb);
    *reinterpret_cast<uint4*>(codes + row * (K / 2) + b * 16) = packed;
    const int64_t so = scale_offset(row, b, nb, tiled);   // an atom holds 4 blocks, as for NVFP4
    scales[so] = (uint8_t)sb;
    if (RES) {
      float r[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) r[i] = __fsub_rn(v[i], deq[i]);
      uint4 rp;
      const uint32_t rb = mx_block(r, rp, nullptr);
      *reinterpret_cast<uint4*>(r_codes + row * (K / 2) + b * 16) = rp;
      r_scales[so] = (uint8_t)rb;
    }
  }
  if (bad >= 253u) report_status(st, NVFP4_ERR_NONFINITE);   // a NaN/Inf block maximum
}

template <typename T>
cudaError_t launch_mx_t(const void* x, int64_t M, int64_t K, int64_t ldx, uint8_t* codes, uint8_t* scales,
                        uint8_t* r_codes, uint8_t* r_scales, bool tiled, int* st, int num_sms,
                        cudaStream_t stream) {
  const int64_t nblk = M * (K / 32);
  const unsigned g = (unsigned)std::max<int64_t>(1, std::min<int64_t>((nblk + 255) / 256, (int64_t)num_sms * 8));
  if (r_codes != nullptr)
    k_mx_quant<T, true><<<g, 256, 0, stream>>>(static_cast<const T*>(x), M, K, ldx, codes, scales, r_codes,
                                                r_scales, tiled, st);
  else
    k_mx_quant<T, false><<<g, 256, 0, stream>>>(static_cast<const T*>(x), M, K, ldx, codes, scales, nullptr,
                                                 nullptr, tiled, st);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_mx_quant(const void* x, nvfp4_dtype dt, int64_t M, int64_t K, int64_t ldx, uint8_t* codes,
                            uint8_t* scales, uint8_t* r_codes, uint8_t* r_scales, bool tiled, int* st,
                            int num_sms, cudaStream_t stream) {
  return dt == NVFP4_BF16
             ? launch_mx_t<__nv_bfloat16>(x, M, K, ldx, codes, scales, r_codes, r_scales, tiled, st, num_sms, stream)
             : launch_mx_t<float>(x, M, K, ldx, codes, scales, r_codes, r_scales, tiled, st, num_sms, stream);
}

}  // namespace nvfp4
