// Offline weight preparation for the augmented W4A4 linear, sm_100a.
//
// ARCQuant blog post, sections 3.1 and 6.3: the weight takes the activations'
// channel order, and the weight columns of the S outlier channels are appended
// so that one GEMM over K + S columns also multiplies the activation residue.
// OSFP4 page, abstract: a per-channel smoothing vector sigma is absorbed at
// inference time, as X diag(sigma)^-1 on the activation side (folded into the
// RMSNorm gain) and W diag(sigma) on the weight side, which this step applies.
//
//   W'[:, j]  = fl32(W[:, perm[j]] * sigma[perm[j]])    (no sigma: W[:, perm[j]])
//   W_aug     = [W' | W'[:, 0..S)]
//   s_w       = scale_in ? *scale_in : fl32(amax|W'| / 2688)
//   w_aug     = Q(W_aug) under s_w
//
// The last S columns hold the same values as the first S under the same
// tensor scale, so their codes and block scales are the first S columns'
// codes and scales, written twice.  Two launches: the tensor maximum, then one
// thread per reordered 16-element block (a gather through the permutation:
// this runs once per weight, offline, and is not tuned).
#include "kernels.h"
#include "quant_common.cuh"

namespace nvfp4 {
namespace {

template <typename T>
__device__ __forceinline__ float load_elem(const T* p);
template <>
__device__ __forceinline__ float load_elem<float>(const float* p) { return __ldg(p); }
template <>
__device__ __forceinline__ float load_elem<__nv_bfloat16>(const __nv_bfloat16* p) {
  return __bfloat162float(*p);
}

// Last-CTA-finishes reduction of the running maximum into s_out.
__device__ void finish_weight_scale(uint32_t key, WsHeader* ws, float* s_out, int* st) {
  __shared__ uint32_t red[32];
  __shared__ bool last;
  const uint32_t m = block_max_u32(key, red);
  if (threadIdx.x == 0) {
    if (m != 0u) atomicMax(&ws->amax_bits[0], m);
    __threadfence();
    last = (atomicAdd(&ws->arrive[0], 1u) == gridDim.x * gridDim.y - 1u);
  }
  __syncthreads();
  if (last && threadIdx.x == 0) {
    __threadfence();
    const uint32_t a = atomicAdd(&ws->amax_bits[0], 0u);
    float s = 0.0f;
    if (a >= 0x7F800000u) report_status(st, NVFP4_ERR_NONFINITE);
    else s = __fdiv_rn(__uint_as_float(a), 2688.0f);
    *s_out = s;
    ws->amax_bits[0] = 0u;   // the workspace is left zeroed for the next call
    ws->arrive[0] = 0u;
    __threadfence();
  }
}

// max |fl32(w * sigma)| over the whole matrix (the permutation does not change it).
template <typename T>
__global__ void __launch_bounds__(256) k_weight_amax(const T* __restrict__ w, int64_t N, int64_t K, int64_t ldw,
                                                     const float* __restrict__ sigma, WsHeader* ws, float* s_out,
                                                     int* st) {
  uint32_t key = 0u;
  for (int64_t r = blockIdx.y; r < N; r += gridDim.y)
    for (int64_t c = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; c < K; c += (int64_t)gridDim.x * blockDim.x) {
      float v = load_elem(w + r * ldw + c);
      if (sigma != nullptr) v = __fmul_rn(v, __ldg(sigma + c));
      key = max(key, abs_key(v));
    }
  finish_weight_scale(key, ws, s_out, st);
}

// One thread per reordered 16-element block (row r, block b): gather, scale,
// quantize, store at block b and, for b < S/16, again at block K/16 + b.
template <typename T>
__global__ void __launch_bounds__(256) k_weight_quant(const T* __restrict__ w, int64_t N, int64_t K, int64_t ldw,
                                                      const float* __restrict__ sigma,
                                                      const int32_t* __restrict__ perm, int64_t S,
                                                      const float* s_ptr, QOut q, int* st) {
  const int64_t nb = K >> 4, nbr = S >> 4;
  const float s = *s_ptr;
  if (blockIdx.x == 0 && threadIdx.x == 0 && q.s != s_ptr) *q.s = s;   // a given scale is the output's too
  uint32_t bad = 0u;
  bool bad_perm = false;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < N * nb; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = i / nb, b = i - r * nb;
    float v[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      const int64_t j = b * 16 + e;
      int64_t c = perm != nullptr ? (int64_t)__ldg(perm + j) : j;
      if (c < 0 || c >= K) {   // not a permutation of 0..K-1: report, never index out of range
        bad_perm = true;
        c = 0;
      }
      float x = load_elem(w + r * ldw + c);
      if (sigma != nullptr) x = __fmul_rn(x, __ldg(sigma + c));
      bad = max(bad, abs_key(x));
      v[e] = x;
    }
    uint32_t db;
    const uint64_t codes = quant_block16(v, s, db, nullptr);
    store_block16(q, r, (int)b, codes, db);
    if (b < nbr) store_block16(q, r, (int)(nb + b), codes, db);
  }
  if (bad >= 0x7F800000u) report_status(st, NVFP4_ERR_NONFINITE);
  if (bad_perm) report_status(st, NVFP4_ERR_INVALID_ARG);
}

template <typename T>
cudaError_t launch_t(const void* w, int64_t N, int64_t K, int64_t ldw, const float* sigma, const int32_t* perm,
                     int64_t S, const float* s_in, const QOut& q, WsHeader* ws, int* st, int num_sms,
                     cudaStream_t stream) {
  const T* wt = static_cast<const T*>(w);
  if (s_in == nullptr) {
    const unsigned gx = (unsigned)std::min<int64_t>((K + 255) / 256, 8);
    const unsigned gy = (unsigned)std::max<int64_t>(1, std::min<int64_t>(N, (int64_t)num_sms * 8 / gx + 1));
    k_weight_amax<T><<<dim3(gx, gy), 256, 0, stream>>>(wt, N, K, ldw, sigma, ws, q.s, st);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  const int64_t blocks = N * (K >> 4);
  const unsigned g = (unsigned)std::max<int64_t>(1, std::min<int64_t>((blocks + 255) / 256, (int64_t)num_sms * 8));
  k_weight_quant<T><<<g, 256, 0, stream>>>(wt, N, K, ldw, sigma, perm, S, s_in ? s_in : q.s, q, st);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_weight_quant(const void* w, nvfp4_dtype dt, int64_t N, int64_t K, int64_t ldw,
                                const float* sigma, const int32_t* perm, int64_t S, const float* s_in,
                                const QOut& q, WsHeader* ws, int* st, int num_sms, cudaStream_t stream) {
  return dt == NVFP4_BF16 ? launch_t<__nv_bfloat16>(w, N, K, ldw, sigma, perm, S, s_in, q, ws, st, num_sms, stream)
                          : launch_t<float>(w, N, K, ldw, sigma, perm, S, s_in, q, ws, st, num_sms, stream);
}

}  // namespace nvfp4
