// NVFP4 activation quantizers for sm_100a.
//
//  k_amax          per-tensor |x| maximum -> s = fl32(amax / 2688)      (tensor scale)
//  k_quant         block amax, E4M3 block scale, E2M1 codes; optional
//                  ResServe residue R = X - deq(Q(X)) with its own scale
//  k_rms_stats     ARCQuant fused path, pass 1: exact per-row mean square,
//                  rinv, and the tensor amax of the normalised rows
//  k_reorder_quant ARCQuant fused path, pass 2: normalise, gather by the
//                  channel permutation, quantize, append the outlier residue
//
// Sources: ARCQuant blog post (zizhi168.cn) sections 1 and 3.1-3.2 (format,
// two-stage quantization, fused reorder/RMSNorm/quantize kernel, reorder
// indices cached in shared memory); ResServe abstract (FP4 residue).
//
// Every rounding step uses an explicit _rn intrinsic so that no multiply-add
// is contracted: the codes and scales are bit-identical to the definition in
// include/nvfp4.h.  Thread mapping: one thread owns one 16-element block (two
// 16-byte bf16 vectors), so the per-block scale, division and reciprocal are
// computed once per block.
#include "common.cuh"
#include "kernels.h"
#include "quant_common.cuh"
#include "tcgen05.cuh"

namespace nvfp4 {

// Last-CTA-finishes reduction of a running |.| maximum into a tensor scale.
// Every thread of every CTA calls it; `key` is the thread's local maximum.
__device__ void finish_tensor_scale(uint32_t key, unsigned int* amax_cell, unsigned int* arrive,
                                    float* s_out, int* st) {
  __shared__ uint32_t red[32];
  __shared__ bool last;
  const uint32_t m = block_max_u32(key, red);
  if (threadIdx.x == 0) {
    if (m != 0u) atomicMax(amax_cell, m);
    __threadfence();
    const unsigned int total = gridDim.x * gridDim.y;
    last = (atomicAdd(arrive, 1u) == total - 1u);
  }
  __syncthreads();
  if (last && threadIdx.x == 0) {
    __threadfence();
    const uint32_t a = atomicAdd(amax_cell, 0u);
    float s = 0.0f;
    if (a >= 0x7F800000u) {
      report_status(st, NVFP4_ERR_NONFINITE);
    } else {
      s = __fdiv_rn(__uint_as_float(a), 2688.0f);
    }
    *s_out = s;
    *amax_cell = 0u;  // leave the workspace zeroed for the next call
    *arrive = 0u;
    __threadfence();
  }
}

// Streaming passes: every thread issues kUnroll independent loads before it
// consumes any, so that each SM keeps tens of KB in flight (what HBM needs);
// a CTA covers kUnroll x 256 consecutive units per iteration.
constexpr int kUnroll = 4;

// |x| maximum.  Contiguous rows (ldx == K) are one flat array of 8-element
// units; otherwise rows are grid-strided over blockIdx.y.
template <typename T>
__global__ void __launch_bounds__(256) k_amax(const T* __restrict__ x, int64_t M, int64_t K,
                                              int64_t ldx, WsHeader* ws, int slot, float* s_out,
                                              int* st) {
  tc::griddep_launch_dependents();   // the quantizer may launch; it waits for this grid's result
  const int64_t upr = K >> 3;
  uint32_t key = 0;
  if (ldx == K) {
    // Each CTA streams one contiguous, equal share of the units (boundaries
    // on 32-unit lines), so no partly filled last round of the grid leaves
    // the read stream short of CTAs.
    const int64_t units = M * upr;
    const int64_t cta = (int64_t)(blockIdx.y * gridDim.x + blockIdx.x), ctas = (int64_t)gridDim.x * gridDim.y;
    const int64_t u0 = (units * cta / ctas) & ~int64_t(31);
    const int64_t u1 = cta + 1 == ctas ? units : (units * (cta + 1) / ctas) & ~int64_t(31);
    for (int64_t base = u0; base < u1; base += 256 * kUnroll) {
      Raw8<T> raw[kUnroll];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int64_t i = base + u * 256 + threadIdx.x;
        if (i < u1) raw[u].load(x + i * 8);
        else raw[u].zero();
      }
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) key = max(key, raw[u].abs_key_max());
    }
  } else {
    for (int64_t row = blockIdx.y; row < M; row += gridDim.y) {
      for (int64_t c8 = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; c8 < upr;
           c8 += (int64_t)gridDim.x * blockDim.x) {
        float v[8];
        load8(x + row * ldx + c8 * 8, v);
#pragma unroll
        for (int i = 0; i < 8; ++i) key = max(key, abs_key(v[i]));
      }
    }
  }
  finish_tensor_scale(key, &ws->amax_bits[slot], &ws->arrive[slot], s_out, st);
}

// One thread per 16-element block (two 16-byte bf16 loads), blocks numbered
// row-major over the whole tensor (M * K/16 < 2^31); each iteration loads
// kUnroll blocks per thread, then encodes them.  Launched as a programmatic dependent of the kernel that computes
// the tensor scale (when there is one): it issues its first loads, then waits
// for that grid before reading the scale.
template <typename T, int MODE>
__global__ void __launch_bounds__(256) k_quant(const T* __restrict__ x, int64_t M, int64_t K,
                                               int64_t ldx, const float* s_ptr,
                                               const float* sr_ptr, QOut q, QOut r, WsHeader* ws,
                                               int* st, DivMagic nb_div) {
  const uint32_t nb = (uint32_t)(K >> 4);
  const int64_t nblk = M * nb;
  const int64_t cta = (int64_t)(blockIdx.y * gridDim.x + blockIdx.x), ctas = (int64_t)gridDim.x * gridDim.y;
  Raw8<T> raw[kUnroll][2];
  auto load_blocks = [&](int64_t base) {
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int64_t j = base + u * 256 + threadIdx.x;
      if (j < nblk) {
        const uint32_t row = div_invariant((uint32_t)j, nb_div), b = (uint32_t)j - row * nb;
        const T* p = x + (int64_t)row * ldx + (int64_t)b * 16;
        raw[u][0].load(p);
        raw[u][1].load(p + 8);
      } else {
        raw[u][0].zero();
        raw[u][1].zero();
      }
    }
  };
  int64_t base = cta * 256 * kUnroll;
  load_blocks(base);   // the input does not depend on the preceding kernel
  tc::griddep_wait();
  const float s = *s_ptr;
  const float s_r = (MODE == Q_RES_ONLY || MODE == Q_BOTH) ? *sr_ptr : 0.0f;
  // per-code block scale and reciprocal for s (and for s_r)
  __shared__ float d_tab[256], inv_tab[256];
  __shared__ float dr_tab[(MODE == Q_RES_ONLY || MODE == Q_BOTH) ? 256 : 1];
  __shared__ float invr_tab[(MODE == Q_RES_ONLY || MODE == Q_BOTH) ? 256 : 1];
  make_scale_tables(s, d_tab, inv_tab);
  if constexpr (MODE == Q_RES_ONLY || MODE == Q_BOTH) make_scale_tables(s_r, dr_tab, invr_tab);
  __syncthreads();
  if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) {
    if (MODE != Q_RES_ONLY && q.s != s_ptr) *q.s = s;
    if (MODE == Q_BOTH && r.s != sr_ptr) *r.s = s_r;
  }
  uint32_t bad = 0, rkey = 0;
  for (bool first = true; base < nblk; base += ctas * 256 * kUnroll, first = false) {
    if (!first) load_blocks(base);
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int64_t j = base + u * 256 + threadIdx.x;
      if (j >= nblk) break;
      const uint32_t row = div_invariant((uint32_t)j, nb_div), b = (uint32_t)j - row * nb;
      float v[16];
      raw[u][0].get(v);
      raw[u][1].get(v + 8);
      uint32_t key;
      if constexpr (sizeof(T) == 2) {
        key = bf16x16_amax_key(raw[u][0].u, raw[u][1].u);
      } else {
        key = 0u;
#pragma unroll
        for (int i = 0; i < 16; ++i) key = max(key, abs_key(v[i]));
      }
      bad = max(bad, key);
      uint32_t db;
      float deq[16];
      const uint64_t codes = quant_block16_tab(v, key, s, d_tab, inv_tab, db, MODE == Q_PLAIN ? nullptr : deq);
      if (MODE != Q_RES_ONLY) store_block16(q, row, (int)b, codes, db);
      if (MODE != Q_PLAIN) {
        float rv[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) rv[i] = __fsub_rn(v[i], deq[i]);
        if (MODE == Q_MAIN_AMAXR) {
#pragma unroll
          for (int i = 0; i < 16; ++i) rkey = max(rkey, abs_key(rv[i]));
        } else {
          uint32_t rk = 0u;
#pragma unroll
          for (int i = 0; i < 16; ++i) rk = max(rk, abs_key(rv[i]));
          uint32_t dr;
          const uint64_t rc = quant_block16_tab(rv, rk, s_r, dr_tab, invr_tab, dr, nullptr);
          store_block16(r, row, (int)b, rc, dr);
        }
      }
    }
  }
  if (bad >= 0x7F800000u) report_status(st, NVFP4_ERR_NONFINITE);
  if (MODE == Q_MAIN_AMAXR) finish_tensor_scale(rkey, &ws->amax_bits[1], &ws->arrive[1], r.s, st);
}

// ------------------------------------------------- single-launch small inputs
// Decode-sized activations (a few rows) are too small to hide two or three
// dependent launches.  One cluster of kQC CTAs quantizes the whole tensor in
// one launch: each thread keeps its 16-element blocks in registers, the CTAs
// exchange their |x| maxima through distributed shared memory behind a cluster
// barrier, and every CTA derives the same tensor scale.  The arithmetic is the
// same per-block routine (quant_block16) as k_quant, so codes and scales are
// identical to the multi-launch path.

constexpr int kQC = 8;              // CTAs per cluster (portable cluster size)
constexpr int kQCWide = 16;         // CTAs per cluster for the largest inputs (non-portable size)
constexpr int kQThreads = 512;      // threads per CTA
constexpr int kQUnitsPerChunk = kQC * kQThreads;   // 16-element blocks per chunk of an 8-CTA cluster

// Block u (16 elements) of this thread's i-th chunk.  Grid: exactly one cluster
// of QC CTAs.
template <typename T, int R, bool RES, int QC>
__global__ void __launch_bounds__(kQThreads, 1)
    k_quant_cluster(const T* __restrict__ x, int M, int K, int64_t ldx, const float* s_in,
                    const float* sr_in, QOut q, QOut r, int* st) {
  __shared__ uint32_t red[kQThreads / 32];
  __shared__ uint32_t xch[2];       // published maxima: [0] |x|, [1] |residue|
  // programmatic dependent launch: let the next kernel set itself up, and wait
  // for the preceding one before reading x
  tc::griddep_launch_dependents();
  tc::griddep_wait();
  const uint32_t rank = tc::cluster_ctarank();
  const int nb = K >> 4;
  const int U = M * nb;
  const bool reporter = rank == 0 && threadIdx.x == 0;

  Raw8<T> raw[R][2];
  uint32_t key = 0u;
#pragma unroll
  for (int i = 0; i < R; ++i) {
    const int u = (i * QC + (int)rank) * kQThreads + (int)threadIdx.x;
    if (u < U) {
      const int row = u / nb, b = u - row * nb;
      const T* src = x + (int64_t)row * ldx + (int64_t)b * 16;
      raw[i][0].load(src);
      raw[i][1].load(src + 8);
    } else {
      raw[i][0].zero();
      raw[i][1].zero();
    }
  }
#pragma unroll
  for (int i = 0; i < R; ++i) key = max(key, max(raw[i][0].abs_key_max(), raw[i][1].abs_key_max()));
  if (key >= 0x7F800000u) report_status(st, NVFP4_ERR_NONFINITE);

  const bool exchange = s_in == nullptr || (RES && sr_in == nullptr);   // uniform
  const float s = s_in != nullptr ? *s_in : scale_from_key(cluster_max_u32(key, red, &xch[0]), reporter, st);
  float s_r = (RES && sr_in != nullptr) ? *sr_in : 0.0f;
  if (reporter) {
    if (q.s != s_in) *q.s = s;
    if (RES && sr_in != nullptr && r.s != sr_in) *r.s = s_r;
  }

  uint32_t rkey = 0u;
#pragma unroll
  for (int i = 0; i < R; ++i) {
    const int u = (i * QC + (int)rank) * kQThreads + (int)threadIdx.x;
    const bool act = u < U;
    const int row = act ? u / nb : 0, b = act ? u - row * nb : 0;
    float v[16], deq[16];
    raw[i][0].get(v);
    raw[i][1].get(v + 8);
    uint32_t db;
    const uint64_t codes = quant_block16(v, s, db, RES ? deq : nullptr);
    if (act) store_block16(q, row, b, codes, db);
    if (RES) {
      float rv[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) rv[j] = __fsub_rn(v[j], deq[j]);
      if (sr_in != nullptr) {
        uint32_t dr;
        const uint64_t rc = quant_block16(rv, s_r, dr, nullptr);
        if (act) store_block16(r, row, b, rc, dr);
      } else if (act) {
#pragma unroll
        for (int j = 0; j < 16; ++j) rkey = max(rkey, abs_key(rv[j]));
      }
    }
  }

  if (RES && sr_in == nullptr) {
    s_r = scale_from_key(cluster_max_u32(rkey, red, &xch[1]), reporter, st);
    if (reporter) *r.s = s_r;
#pragma unroll
    for (int i = 0; i < R; ++i) {
      const int u = (i * QC + (int)rank) * kQThreads + (int)threadIdx.x;
      if (u >= U) continue;
      const int row = u / nb, b = u - row * nb;
      float v[16], deq[16], rv[16];
      raw[i][0].get(v);
      raw[i][1].get(v + 8);
      uint32_t db, dr;
      (void)quant_block16(v, s, db, deq);
#pragma unroll
      for (int j = 0; j < 16; ++j) rv[j] = __fsub_rn(v[j], deq[j]);
      const uint64_t rc = quant_block16(rv, s_r, dr, nullptr);
      store_block16(r, row, b, rc, dr);
    }
  }
  if (exchange) tc::cluster_sync();  // peers may read this CTA's xch words until here
}

// ----------------------------------------------------------- ARCQuant path

// Binary64 power of two 2^e for -1022 <= e <= 1023.
__device__ __forceinline__ double pow2_f64(int e) {
  return __longlong_as_double((long long)(1023 + e) << 52);
}

// floor(log2(a)) for a finite positive fp32 bit pattern.
__device__ __forceinline__ int ilog2_key(uint32_t key) {
  return key >= 0x00800000u ? (int)(key >> 23) - 127 : (31 - __clz((int)key)) - 149;
}

// Pass 1, one CTA per row (grid-stride): rinv of the row and the running
// maximum of |y| = |fl32(fl32(x * rinv) * gamma)| over the tensor.  The three
// per-row reductions (|x| maximum for the exponent, the exact sum of squares,
// the |y| maximum) all need the whole row: with NC > 0 each thread keeps its
// NC 8-element units of the row in registers, so the row is read once; NC = 0
// is the general form that re-reads the row (from L1/L2) for each reduction.
template <typename T, int NC>
__global__ void __launch_bounds__(256) k_rms_stats(const T* __restrict__ x, int64_t M, int64_t K,
                                                   int64_t ldx, const T* __restrict__ gamma,
                                                   float eps, WsHeader* ws, float* rinv_out,
                                                   float* s_out, bool want_scale, int* st) {
  __shared__ uint32_t redu[32];
  __shared__ double redd[32];
  tc::griddep_launch_dependents();   // the reorder pass may launch; it waits for this grid's results
  const int64_t upr = K >> 3;
  uint32_t ykey = 0, bad = 0;
  // unit c8 of the row: NC > 0 -> c8 = threadIdx.x + 256 n, n < NC
  [[maybe_unused]] Raw8<T> rowv[NC > 0 ? NC : 1];
  for (int64_t row = blockIdx.x; row < M; row += gridDim.x) {
    const T* xr = x + row * ldx;
    uint32_t key = 0;
    if constexpr (NC > 0) {
#pragma unroll
      for (int n = 0; n < NC; ++n) {
        const int64_t c8 = threadIdx.x + 256 * n;
        if (c8 < upr) rowv[n].load(xr + c8 * 8);
        else rowv[n].zero();
      }
#pragma unroll
      for (int n = 0; n < NC; ++n) {
        float v[8];
        rowv[n].get(v);
#pragma unroll
        for (int i = 0; i < 8; ++i) key = max(key, abs_key(v[i]));
      }
    } else {
      for (int64_t c8 = threadIdx.x; c8 < upr; c8 += blockDim.x) {
        float v[8];
        load8(xr + c8 * 8, v);
#pragma unroll
        for (int i = 0; i < 8; ++i) key = max(key, abs_key(v[i]));
      }
    }
    key = block_max_u32(key, redu);
    bad = max(bad, key);
    double qsum = 0.0;
    int e = 0;
    if (key != 0u && key < 0x7F800000u) {
      e = ilog2_key(key);
      const double c = pow2_f64(17 - e);  // z = x * 2^(17-e), |z| < 2^18
      auto add_sq = [&](const float v[8]) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const double z = __dmul_rn((double)v[i], c);
          qsum = __dadd_rn(qsum, floor(__dmul_rn(z, z)));
        }
      };
      if constexpr (NC > 0) {
#pragma unroll
        for (int n = 0; n < NC; ++n) {
          float v[8];
          rowv[n].get(v);   // units past the row are zero and add nothing
          add_sq(v);
        }
      } else {
        for (int64_t c8 = threadIdx.x; c8 < upr; c8 += blockDim.x) {
          float v[8];
          load8(xr + c8 * 8, v);
          add_sq(v);
        }
      }
    }
    qsum = block_sum_f64(qsum, redd);  // exact: integers with total < 2^53
    const double mean = __ddiv_rn(__dmul_rn(qsum, pow2_f64(2 * e - 34)), (double)K);
    const float rinv = __double2float_rn(__drcp_rn(__dsqrt_rn(__dadd_rn(mean, (double)eps))));
    if (threadIdx.x == 0) rinv_out[row] = rinv;
    if (want_scale) {
      auto max_y = [&](const float v[8], const float g[8]) {
#pragma unroll
        for (int i = 0; i < 8; ++i) ykey = max(ykey, abs_key(__fmul_rn(__fmul_rn(v[i], rinv), g[i])));
      };
      if constexpr (NC > 0) {
#pragma unroll
        for (int n = 0; n < NC; ++n) {
          const int64_t c8 = threadIdx.x + 256 * n;
          if (c8 < upr) {
            float v[8], g[8];
            rowv[n].get(v);
            load8(gamma + c8 * 8, g);
            max_y(v, g);
          }
        }
      } else {
        for (int64_t c8 = threadIdx.x; c8 < upr; c8 += blockDim.x) {
          float v[8], g[8];
          load8(xr + c8 * 8, v);
          load8(gamma + c8 * 8, g);
          max_y(v, g);
        }
      }
    }
  }
  if (bad >= 0x7F800000u) report_status(st, NVFP4_ERR_NONFINITE);
  if (want_scale) finish_tensor_scale(ykey, &ws->amax_bits[0], &ws->arrive[0], s_out, st);
}

// Pass 2, persistent CTAs looping over rows.  Shared memory holds the channel
// permutation as 16-bit indices (K <= 65536) and gamma in its own type (both
// loaded once per CTA), and two row buffers: the next row's load (cp.async)
// is in flight while the current row is encoded.
__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gmem_src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(tc::saddr(smem_dst)), "l"(gmem_src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

// The channel permutation as 16-bit indices in shared memory (K <= 65536).  An
// entry outside 0..K-1 is replaced by 0, so no index is ever out of range; the
// return value says whether there was one.
__device__ __forceinline__ bool load_perm16(const int32_t* __restrict__ perm, int64_t K, uint16_t* sperm) {
  bool bad_perm = false;
  if (perm != nullptr && (reinterpret_cast<uintptr_t>(perm) & 15u) == 0) {
    // four 16-byte loads per thread in flight before any is used (K % 16 == 0)
    constexpr int U = 4;
    const int64_t n4 = K >> 2;
    const uint4* p4 = reinterpret_cast<const uint4*>(perm);
    for (int64_t c0 = threadIdx.x; c0 < n4; c0 += U * (int64_t)blockDim.x) {
      uint4 v[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int64_t c = c0 + u * (int64_t)blockDim.x;
        v[u] = c < n4 ? __ldg(p4 + c) : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int64_t c = c0 + u * (int64_t)blockDim.x;
        if (c < n4) {
          uint32_t e[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
          for (int i = 0; i < 4; ++i)
            if ((uint64_t)e[i] >= (uint64_t)K) {   // also catches negative entries
              bad_perm = true;
              e[i] = 0u;
            }
          *reinterpret_cast<uint2*>(sperm + 4 * c) = make_uint2(e[0] | (e[1] << 16), e[2] | (e[3] << 16));
        }
      }
    }
  } else {
    for (int64_t k = threadIdx.x; k < K; k += blockDim.x) {
      int32_t p = perm ? perm[k] : (int32_t)k;
      if (p < 0 || (int64_t)p >= K) {
        bad_perm = true;
        p = 0;
      }
      sperm[k] = (uint16_t)p;
    }
  }
  return bad_perm;
}

// Encode one row held in shared memory: y'[j] = fl32(fl32(x[perm[j]] * ri) *
// gamma[perm[j]]) (y' = x[perm] without gamma), one thread per 16-element block
// of the reordered row; the first nbr blocks' residues are quantized under the
// same scale and written as blocks nb .. nb + nbr - 1.
template <typename T>
__device__ __forceinline__ void encode_reordered_row(const T* srow, const uint16_t* sperm, const T* sgamma,
                                                     float ri, float s, const QOut& q, int64_t row, int nb,
                                                     int nbr, uint32_t& bad) {
  for (int b = threadIdx.x; b < nb; b += blockDim.x) {
    float v[16];
    uint16_t pv[16];
#pragma unroll
    for (int j = 0; j < 2; ++j)   // 16-byte reads of the cached permutation
      *reinterpret_cast<uint4*>(pv + 8 * j) = reinterpret_cast<const uint4*>(sperm)[b * 2 + j];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int p = pv[i];
      float y = load1(srow + p);
      bad = max(bad, abs_key(y));
      if (sgamma) y = __fmul_rn(__fmul_rn(y, ri), load1(sgamma + p));
      v[i] = y;
    }
    uint32_t db;
    float deq[16];
    const bool res = b < nbr;
    const uint64_t codes = quant_block16(v, s, db, res ? deq : nullptr);
    store_block16(q, row, b, codes, db);
    if (res) {
      float rv[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) rv[i] = __fsub_rn(v[i], deq[i]);
      uint32_t dr;
      const uint64_t rc = quant_block16(rv, s, dr, nullptr);
      store_block16(q, row, nb + b, rc, dr);
    }
  }
}

template <typename T>
__global__ void __launch_bounds__(256) k_reorder_quant(const T* __restrict__ x, int64_t M,
                                                       int64_t K, int64_t ldx,
                                                       const T* __restrict__ gamma,
                                                       const float* __restrict__ rinv,
                                                       const int32_t* __restrict__ perm, int64_t S,
                                                       const float* s_ptr, QOut q, int* st) {
  extern __shared__ __align__(16) unsigned char smem[];
  const int64_t row_bytes = K * (int64_t)sizeof(T);   // a multiple of 16 (K % 16 == 0)
  T* srow0 = reinterpret_cast<T*>(smem);
  T* srow1 = reinterpret_cast<T*>(smem + row_bytes);
  uint16_t* sperm = reinterpret_cast<uint16_t*>(smem + 2 * row_bytes);
  T* sgamma = reinterpret_cast<T*>(smem + 2 * row_bytes + ((K * 2 + 15) & ~int64_t(15)));
  auto fetch_row = [&](int64_t row, T* dst) {
    const T* xr = x + row * ldx;
    for (int64_t c = threadIdx.x; c < row_bytes / 16; c += blockDim.x)
      cp_async16(reinterpret_cast<uint4*>(dst) + c, reinterpret_cast<const uint4*>(xr) + c);
    cp_async_commit();
  };
  // gamma goes to shared memory by cp.async in the first row's group (its
  // pointer is 16-byte aligned and K * sizeof(T) a multiple of 16)
  if (gamma)
    for (int64_t c = threadIdx.x; c < row_bytes / 16; c += blockDim.x)
      cp_async16(reinterpret_cast<uint4*>(sgamma) + c, reinterpret_cast<const uint4*>(gamma) + c);
  if ((int64_t)blockIdx.x < M) fetch_row(blockIdx.x, srow0);   // overlaps the table set-up
  else cp_async_commit();
  if (load_perm16(perm, K, sperm)) report_status(st, NVFP4_ERR_INVALID_ARG);
  // X, gamma and perm are inputs of the call; the tensor scale and the row
  // factors come from the statistics pass, which may still be running
  tc::griddep_wait();
  const float s = *s_ptr;
  if (blockIdx.x == 0 && threadIdx.x == 0 && q.s != s_ptr) *q.s = s;
  const int nb = (int)(K >> 4);     // blocks of the reordered row
  const int nbr = (int)(S >> 4);    // residue blocks (the first S reordered columns)
  uint32_t bad = 0;
  int buf = 0;
  for (int64_t row = blockIdx.x; row < M; row += gridDim.x, buf ^= 1) {
    const T* srow = buf ? srow1 : srow0;
    cp_async_wait_all();
    __syncthreads();   // this row landed; every thread is done with the other buffer
    if (row + gridDim.x < M) fetch_row(row + gridDim.x, buf ? srow0 : srow1);
    encode_reordered_row(srow, sperm, gamma ? sgamma : nullptr, gamma ? rinv[row] : 1.0f, s, q, row, nb, nbr,
                         bad);
  }
  cp_async_wait_all();
  if (bad >= 0x7F800000u) report_status(st, NVFP4_ERR_NONFINITE);
}

// One-launch ARCQuant quantizer, for inputs whose rows fit in the shared
// memory of one wave of CTAs: one row per warp (or a few).  The launch is
// cooperative, so every CTA is resident.  Each warp:
//   1. loads its row with 16-byte loads, all in flight at once, keeps it in
//      registers and copies it to its row buffer in shared memory, and takes
//      from the registers the row's |x| maximum, its exact mean square (the
//      arithmetic of k_rms_stats), rinv and the row's |y| maximum (without
//      gamma: the |x| maximum);
//   2. the CTA meets the other CTAs at one exchange of the maximum through the
//      workspace header (atomics, a bounded wait; the last CTA to leave zeroes
//      the header again);
//   3. the warp encodes its own row from its row buffer, lanes over the
//      reordered 16-blocks (residue blocks included).
// X is read from DRAM once, no block barrier sits inside a row's work, and
// the result is identical to the two passes.
__device__ __forceinline__ uint32_t ld_acquire_gpu(const unsigned int* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// 8 consecutive elements from shared memory as fp32.
__device__ __forceinline__ void lds8(const __nv_bfloat16* p, float v[8]) {
  const uint4 u = *reinterpret_cast<const uint4*>(p);
  v[0] = __uint_as_float(u.x << 16); v[1] = __uint_as_float(u.x & 0xFFFF0000u);
  v[2] = __uint_as_float(u.y << 16); v[3] = __uint_as_float(u.y & 0xFFFF0000u);
  v[4] = __uint_as_float(u.z << 16); v[5] = __uint_as_float(u.z & 0xFFFF0000u);
  v[6] = __uint_as_float(u.w << 16); v[7] = __uint_as_float(u.w & 0xFFFF0000u);
}
__device__ __forceinline__ void lds8(const float* p, float v[8]) {
  const float4 a = reinterpret_cast<const float4*>(p)[0], b = reinterpret_cast<const float4*>(p)[1];
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

// Shared-memory layout of k_reorder_onepass: the permutation (16-bit), gamma
// in source and in permuted order, the d and 1/(d s) tables of the block
// encoder, then rpw row buffers for each of the CTA's wpc warps (4..8).
__host__ __device__ inline size_t onepass_fixed_bytes(size_t es, int64_t K, bool has_gamma) {
  return (((size_t)K * 2 + 15) & ~size_t(15)) + (has_gamma ? 2 * (size_t)K * es : 0) + 2 * 256 * 4;
}
inline size_t onepass_smem_bytes(size_t es, int64_t K, bool has_gamma, int rpw, int wpc) {
  return onepass_fixed_bytes(es, K, has_gamma) + (size_t)wpc * rpw * (size_t)K * es;
}

// 8 consecutive elements from global memory (16/32-byte aligned) as fp32.
__device__ __forceinline__ void ldg8(const __nv_bfloat16* p, float v[8]) {
  const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
  v[0] = __uint_as_float(u.x << 16); v[1] = __uint_as_float(u.x & 0xFFFF0000u);
  v[2] = __uint_as_float(u.y << 16); v[3] = __uint_as_float(u.y & 0xFFFF0000u);
  v[4] = __uint_as_float(u.z << 16); v[5] = __uint_as_float(u.z & 0xFFFF0000u);
  v[6] = __uint_as_float(u.w << 16); v[7] = __uint_as_float(u.w & 0xFFFF0000u);
}
__device__ __forceinline__ void ldg8(const float* p, float v[8]) {
  const float4 a = __ldg(reinterpret_cast<const float4*>(p)), b = __ldg(reinterpret_cast<const float4*>(p) + 1);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

// Gather reordered block b of a row held in shared memory: v[e] =
// y'[16 b + e] = fl32(fl32(x[perm[16 b + e]] * ri) * gp[16 b + e]) (gp: gamma in
// permuted order; no gamma: x[perm[.]]).  Returns the |.| maximum key.
template <typename T>
__device__ __forceinline__ uint32_t gather_block(const T* srow, const uint16_t* sperm, const T* sgp, float ri,
                                                 int b, float v[16]) {
  uint16_t pv[16];
#pragma unroll
  for (int j = 0; j < 2; ++j)   // 16-byte reads of the cached permutation
    *reinterpret_cast<uint4*>(pv + 8 * j) = reinterpret_cast<const uint4*>(sperm)[b * 2 + j];
  float g[16];
  if (sgp != nullptr) {
    lds8(sgp + b * 16, g);
    lds8(sgp + b * 16 + 8, g + 8);
  }
  uint32_t key = 0u;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    float y = load1(srow + pv[i]);
    if (sgp != nullptr) y = __fmul_rn(__fmul_rn(y, ri), g[i]);
    v[i] = y;
    key = max(key, abs_key(y));
  }
  return key;
}

// floor(z^2), z = x 2^(17-e), for a value x of 8 significant bits (bf16) as an
// exact fp32 computation: for |z| >= 1, z and z^2 (16 bits) are exact in fp32;
// for |z| < 1 the floor is 0 whatever z rounded to.  (c = 2^(17-e) in fp32,
// valid for e >= -110; the caller takes the binary64 form below that.)
__device__ __forceinline__ uint64_t sq_floor_bf16(float x, float c) {
  const float z = __fmul_rn(x, c);
  return (uint64_t)floorf(__fmul_rn(z, z));
}

// Units (8 elements) of a row a lane holds in registers at once.
template <typename T>
struct RowChunk {
  static constexpr int N = sizeof(T) == 2 ? 16 : 8;
};

template <typename T>
__global__ void __launch_bounds__(256, 2) k_reorder_onepass(const T* __restrict__ x, int64_t M, int64_t K,
                                                            int64_t ldx, const T* __restrict__ gamma, float eps,
                                                            const int32_t* __restrict__ perm, int64_t S,
                                                            const float* s_in, QOut q, WsHeader* ws, int rpw,
                                                            int* st) {
  constexpr int NCH = RowChunk<T>::N;   // units per lane loaded at once
  extern __shared__ __align__(16) unsigned char smem[];
  __shared__ uint32_t wkey[8];   // per warp: the |y| maximum of its rows (|x| without gamma)
  __shared__ uint32_t wbad[8];   // per warp: the |x| maximum (Inf/NaN detection)
  __shared__ float s_sh;
  __shared__ int ok_sh;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int wpc = (int)(blockDim.x >> 5);   // warps of this CTA, 4..8
  const int64_t row_bytes = K * (int64_t)sizeof(T);   // a multiple of 16 (K % 16 == 0)
  uint16_t* sperm = reinterpret_cast<uint16_t*>(smem);
  T* sg = reinterpret_cast<T*>(smem + ((K * 2 + 15) & ~int64_t(15)));   // gamma, source order
  T* sgp = sg + (gamma ? K : 0);                                         // gamma, permuted order
  float* d_tab = reinterpret_cast<float*>(reinterpret_cast<unsigned char*>(sgp) + (gamma ? row_bytes : 0));
  float* inv_tab = d_tab + 256;
  T* wrows = reinterpret_cast<T*>(smem + onepass_fixed_bytes(sizeof(T), K, gamma != nullptr)) +
             (int64_t)warp * rpw * K;
  const int64_t W = (int64_t)gridDim.x * wpc, wg = (int64_t)blockIdx.x * wpc + warp;   // warps, this warp
  int nrows = 0;   // rows of this warp: wg + i * W
  while (nrows < rpw && wg + nrows * W < M) ++nrows;

  // 0. gamma (source order) and the permutation, shared by the CTA's warps
  if (gamma)
    for (int64_t c = threadIdx.x; c < row_bytes / 16; c += blockDim.x)
      cp_async16(reinterpret_cast<uint4*>(sg) + c, reinterpret_cast<const uint4*>(gamma) + c);
  cp_async_commit();
  if (load_perm16(perm, K, sperm)) report_status(st, NVFP4_ERR_INVALID_ARG);
  cp_async_wait_all();
  __syncthreads();

  // 1. per warp, per row: load once (registers and the row buffer), statistics
  const int64_t upr = K >> 3;                     // 8-element units of a row
  const int npl = (int)((upr + 31) / 32);         // units per lane
  uint32_t ykey = 0u, bad = 0u;
  float ri_reg[4] = {1.0f, 1.0f, 1.0f, 1.0f};     // rinv of this warp's rows (rpw <= 4)
  for (int i = 0; i < nrows; ++i) {
    const T* xr = x + (wg + i * W) * ldx;
    T* sr = wrows + (int64_t)i * K;
    Raw8<T> raw[NCH];
    uint32_t key = 0u;
    for (int n0 = 0; n0 < npl; n0 += NCH) {       // load: all of a chunk in flight at once
#pragma unroll
      for (int n = 0; n < NCH; ++n) {
        const int64_t c8 = lane + 32 * (int64_t)(n0 + n);
        if (n0 + n < npl && c8 < upr) raw[n].load(xr + c8 * 8);
        else raw[n].zero();
      }
#pragma unroll
      for (int n = 0; n < NCH; ++n) {
        const int64_t c8 = lane + 32 * (int64_t)(n0 + n);
        if (n0 + n < npl && c8 < upr) raw[n].store_smem(sr + c8 * 8);
        key = max(key, raw[n].abs_key_max());
      }
    }
    key = warp_max_u32(key);
    bad = max(bad, key);
    if (gamma == nullptr) {
      ykey = max(ykey, key);
      continue;
    }
    // the exact sum of floor(z^2), z = x 2^(17-e), from the row buffer, four
    // independent 16-byte reads at a time
    uint64_t isum = 0;
    int e = 0;
    if (key != 0u && key < 0x7F800000u) {
      e = ilog2_key(key);
      const bool fast = sizeof(T) == 2 && e >= -110;
      const float c32 = fast ? __uint_as_float((uint32_t)(127 + 17 - e) << 23) : 0.0f;
      const double c64 = pow2_f64(17 - e);
      for (int n0 = 0; n0 < npl; n0 += 4) {
        float v[4][8];
#pragma unroll
        for (int n = 0; n < 4; ++n) {
          const int64_t c8 = lane + 32 * (int64_t)(n0 + n);
          if (n0 + n < npl && c8 < upr) lds8(sr + c8 * 8, v[n]);
          else
#pragma unroll
            for (int j = 0; j < 8; ++j) v[n][j] = 0.0f;
        }
#pragma unroll
        for (int n = 0; n < 4; ++n)
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            if (fast) {
              isum += sq_floor_bf16(v[n][j], c32);
            } else {
              const double z = __dmul_rn((double)v[n][j], c64);
              isum += (uint64_t)floor(__dmul_rn(z, z));
            }
          }
      }
    }
    // exact: integers with total < 2^53, so the order of the additions is free
    const double qsum = warp_sum_f64((double)isum);
    const double mean = __ddiv_rn(__dmul_rn(qsum, pow2_f64(2 * e - 34)), (double)K);
    const float ri = __double2float_rn(__drcp_rn(__dsqrt_rn(__dadd_rn(mean, (double)eps))));
    ri_reg[i & 3] = ri;
    if (s_in == nullptr) {
      for (int n0 = 0; n0 < npl; n0 += 4) {
        float v[4][8], g[4][8];
#pragma unroll
        for (int n = 0; n < 4; ++n) {
          const int64_t c8 = lane + 32 * (int64_t)(n0 + n);
          const bool ok = n0 + n < npl && c8 < upr;
#pragma unroll
          for (int j = 0; j < 8; ++j) v[n][j] = g[n][j] = 0.0f;
          if (ok) {
            lds8(sr + c8 * 8, v[n]);
            lds8(sg + c8 * 8, g[n]);
          }
        }
#pragma unroll
        for (int n = 0; n < 4; ++n)
#pragma unroll
          for (int j = 0; j < 8; ++j) ykey = max(ykey, abs_key(__fmul_rn(__fmul_rn(v[n][j], ri), g[n][j])));
      }
    }
  }
  ykey = warp_max_u32(ykey);
  if (lane == 0) {
    wkey[warp] = ykey;
    wbad[warp] = bad;
  }
  if (gamma)   // gamma in the permuted order, for 16-byte reads in the encoder
    for (int64_t j = threadIdx.x; j < K; j += blockDim.x) sgp[j] = sg[sperm[j]];
  __syncthreads();   // per-warp maxima and sgp are visible to every thread

  // 2. the tensor scale: one exchange of the CTA maxima through the workspace
  if (threadIdx.x == 0) {
    uint32_t m = 0u, xb = 0u;
    for (int w = 0; w < wpc; ++w) {
      m = max(m, wkey[w]);
      xb = max(xb, wbad[w]);
    }
    if (xb >= 0x7F800000u) report_status(st, NVFP4_ERR_NONFINITE);
    if (s_in == nullptr) {
      if (m != 0u) atomicMax(&ws->amax_bits[0], m);
      __threadfence();
      atomicAdd(&ws->arrive[0], 1u);
      const uint64_t t0 = tc::globaltimer();
      int ok = 1;
      while (ld_acquire_gpu(&ws->arrive[0]) < (uint32_t)gridDim.x) {
        __nanosleep(64);   // fewer polls of the shared counter while the others arrive
        if (tc::globaltimer() - t0 > tc::kTimeoutNs) {
          ok = 0;
          report_status(st, NVFP4_ERR_TIMEOUT);
          break;
        }
      }
      // every CTA's maximum was added before its arrival was counted
      const uint32_t a = ld_acquire_gpu(&ws->amax_bits[0]);
      s_sh = ok ? scale_from_key(a, blockIdx.x == 0, st) : 0.0f;
      ok_sh = ok;
    } else {
      s_sh = *s_in;
      ok_sh = 1;
    }
  }
  __syncthreads();
  if (s_in == nullptr && threadIdx.x == 32) {
    // leave after this CTA's read above; the last CTA to leave zeroes the
    // header for the next call (off the other threads' path)
    __threadfence();
    if (atomicAdd(&ws->arrive[1], 1u) == gridDim.x - 1u) {
      ws->amax_bits[0] = 0u;
      ws->arrive[0] = 0u;
      ws->arrive[1] = 0u;
      __threadfence();
    }
  }
  if (!ok_sh) return;
  const float s = s_sh;
  if (blockIdx.x == 0 && threadIdx.x == 0 && q.s != s_in) *q.s = s;
  make_scale_tables(s, d_tab, inv_tab);
  __syncthreads();

  // 3. each warp encodes its rows: lanes over the main blocks, then the residue
  // blocks (a residue block recomputes its main block's dequantized values);
  // two blocks per iteration, both gathers issued before either is encoded
  const int nb = (int)(K >> 4), nbr = (int)(S >> 4);
  const T* gp = gamma ? sgp : nullptr;
  auto finish = [&](int64_t row, bool res, int b, const float* v, uint32_t key) {
    uint32_t db;
    float deq[16];
    const uint64_t codes = quant_block16_tab(v, key, s, d_tab, inv_tab, db, res ? deq : nullptr);
    if (!res) {
      store_block16(q, row, b, codes, db);
    } else {
      float rv[16];
      uint32_t rkey = 0u;
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        rv[j] = __fsub_rn(v[j], deq[j]);
        rkey = max(rkey, abs_key(rv[j]));
      }
      uint32_t dr;
      const uint64_t rc = quant_block16_tab(rv, rkey, s, d_tab, inv_tab, dr, nullptr);
      store_block16(q, row, nb + b, rc, dr);
    }
  };
  for (int i = 0; i < nrows; ++i) {
    const int64_t row = wg + i * W;
    const T* sr = wrows + (int64_t)i * K;
    const float ri = gamma ? ri_reg[i & 3] : 1.0f;
    const int n_all = nb + nbr;
    for (int t = lane; t < n_all; t += 32) {
      const bool res = t >= nb;
      const int b = res ? t - nb : t;
      float v[16];
      const uint32_t k = gather_block(sr, sperm, gp, ri, b, v);
      finish(row, res, b, v, k);
    }
  }
}

// ------------------------------------------------------------ launchers

// ------------------------------------------------- single-launch small inputs

// capacity in 8-element units: each thread holds up to 8 (bf16) / 4 (fp32) 16-element blocks
int64_t quant_small_max_units(nvfp4_dtype dt) {
  return 2 * (int64_t)kQUnitsPerChunk * (dt == NVFP4_BF16 ? 8 : 4);
}

template <int QC>
void quant_cluster_config(cudaLaunchConfig_t& cfg, cudaLaunchAttribute* attr, cudaStream_t stream) {
  cfg = cudaLaunchConfig_t{};
  cfg.gridDim = dim3(QC, 1, 1);
  cfg.blockDim = dim3(kQThreads, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = QC;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;   // overlap the preceding kernel's tail
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
}

template <typename T, int R, bool RES, int QC = kQC>
cudaError_t launch_quant_cluster_r(const void* x, int64_t M, int64_t K, int64_t ldx, const float* s_in,
                                   const float* sr_in, const QOut& q, const QOut& r, int* st,
                                   cudaStream_t stream) {
  cudaLaunchConfig_t cfg;
  cudaLaunchAttribute attr[2];
  quant_cluster_config<QC>(cfg, attr, stream);
  return cudaLaunchKernelEx(&cfg, k_quant_cluster<T, R, RES, QC>, static_cast<const T*>(x), (int)M, (int)K, ldx,
                            s_in, sr_in, q, r, st);
}

// Whether a 16-CTA cluster of this instance can be resident on the device
// (the cluster must fit in one GPC); queried once per instance.
template <typename T, int R, bool RES>
bool wide_cluster_fits() {
  static int fits = -1;
  if (fits < 0) {
    auto kern = k_quant_cluster<T, R, RES, kQCWide>;
    int n = 0;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) == cudaSuccess) {
      cudaLaunchConfig_t cfg;
      cudaLaunchAttribute attr[2];
      quant_cluster_config<kQCWide>(cfg, attr, nullptr);
      cfg.numAttrs = 1;   // the cluster dimension only
      if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) n = 0;
    }
    (void)cudaGetLastError();   // a refused query leaves no error for the next launch
    fits = n >= 1 ? 1 : 0;
  }
  return fits == 1;
}

template <typename T, bool RES>
cudaError_t launch_quant_cluster_t(const void* x, int64_t M, int64_t K, int64_t ldx, const float* s_in,
                                   const float* sr_in, const QOut& q, const QOut& r, int* st,
                                   cudaStream_t stream) {
  // chunks of kQUnitsPerChunk 16-element blocks
  const int64_t chunks = (M * (K >> 4) + kQUnitsPerChunk - 1) / kQUnitsPerChunk;
  if (chunks <= 1) return launch_quant_cluster_r<T, 1, RES>(x, M, K, ldx, s_in, sr_in, q, r, st, stream);
  if (chunks <= 2) return launch_quant_cluster_r<T, 2, RES>(x, M, K, ldx, s_in, sr_in, q, r, st, stream);
  if (chunks <= 4) return launch_quant_cluster_r<T, 4, RES>(x, M, K, ldx, s_in, sr_in, q, r, st, stream);
  if constexpr (sizeof(T) == 2) {
    // twice the CTAs (16 SMs of one GPC) rather than twice the blocks per thread
    if (chunks <= 8 && wide_cluster_fits<T, 4, RES>())
      return launch_quant_cluster_r<T, 4, RES, kQCWide>(x, M, K, ldx, s_in, sr_in, q, r, st, stream);
    if (chunks <= 8) return launch_quant_cluster_r<T, 8, RES>(x, M, K, ldx, s_in, sr_in, q, r, st, stream);
  }
  return cudaErrorNotSupported;
}

cudaError_t launch_quant_small(bool residue, const void* x, nvfp4_dtype dt, int64_t M, int64_t K, int64_t ldx,
                               const float* s_in, const float* sr_in, const QOut& q, const QOut& r, int* st,
                               cudaStream_t stream) {
  if (M * (K >> 3) > quant_small_max_units(dt)) return cudaErrorNotSupported;
  if (dt == NVFP4_BF16)
    return residue ? launch_quant_cluster_t<__nv_bfloat16, true>(x, M, K, ldx, s_in, sr_in, q, r, st, stream)
                   : launch_quant_cluster_t<__nv_bfloat16, false>(x, M, K, ldx, s_in, sr_in, q, r, st, stream);
  return residue ? launch_quant_cluster_t<float, true>(x, M, K, ldx, s_in, sr_in, q, r, st, stream)
                 : launch_quant_cluster_t<float, false>(x, M, K, ldx, s_in, sr_in, q, r, st, stream);
}

// k_amax grid: contiguous input runs flat over 8-element units (x only);
// strided rows use (x) units of a row, (y) rows.
static inline dim3 quant_grid(int64_t M, int64_t K, int64_t ldx, int num_sms) {
  const int64_t upr = K >> 3;
  const int64_t target = (int64_t)num_sms * 8;
  if (ldx == K) {
    const int64_t per_cta = 256 * kUnroll;
    return dim3((unsigned)std::max<int64_t>(1, std::min<int64_t>(target, (M * upr + per_cta - 1) / per_cta)));
  }
  const int64_t gx = std::min<int64_t>((upr + 255) / 256, 65535);
  const int64_t gy = std::max<int64_t>(1, std::min<int64_t>({M, 65535, (target + gx - 1) / gx}));
  return dim3((unsigned)gx, (unsigned)gy);
}

template <typename T>
cudaError_t launch_amax_t(const void* x, int64_t M, int64_t K, int64_t ldx, WsHeader* ws, int slot,
                          float* s_out, int* st, int num_sms, cudaStream_t stream) {
  k_amax<T><<<quant_grid(M, K, ldx, num_sms), 256, 0, stream>>>(static_cast<const T*>(x), M, K, ldx, ws,
                                                           slot, s_out, st);
  return cudaGetLastError();
}

cudaError_t launch_amax(const void* x, nvfp4_dtype dt, int64_t M, int64_t K, int64_t ldx,
                        WsHeader* ws, int slot, float* s_out, int* st, int num_sms,
                        cudaStream_t stream) {
  return dt == NVFP4_BF16
             ? launch_amax_t<__nv_bfloat16>(x, M, K, ldx, ws, slot, s_out, st, num_sms, stream)
             : launch_amax_t<float>(x, M, K, ldx, ws, slot, s_out, st, num_sms, stream);
}

// k_quant grid: flat over 16-element blocks, up to 8 CTAs per SM.
static inline dim3 quant_block_grid(int64_t M, int64_t K, int num_sms) {
  const int64_t per_cta = 256 * kUnroll;
  return dim3((unsigned)std::max<int64_t>(1, std::min<int64_t>((int64_t)num_sms * 8, (M * (K >> 4) + per_cta - 1) / per_cta)));
}

template <typename T, int MODE>
cudaError_t launch_quant_m(const void* x, int64_t M, int64_t K, int64_t ldx, const float* s_ptr,
                           const float* sr_ptr, const QOut& q, const QOut& r, WsHeader* ws, int* st,
                           int num_sms, cudaStream_t stream, bool after_amax) {
  if (M * (K >> 4) >= ((int64_t)1 << 31)) return cudaErrorNotSupported;   // block numbers are 32-bit
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = quant_block_grid(M, K, num_sms);
  cfg.blockDim = dim3(256);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = after_amax ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, k_quant<T, MODE>, static_cast<const T*>(x), M, K, ldx, s_ptr, sr_ptr, q, r, ws,
                            st, make_div_magic((uint32_t)(K >> 4)));
}

template <typename T>
cudaError_t launch_quant_t(int mode, const void* x, int64_t M, int64_t K, int64_t ldx,
                           const float* s_ptr, const float* sr_ptr, const QOut& q, const QOut& r,
                           WsHeader* ws, int* st, int num_sms, cudaStream_t stream, bool after_amax) {
  switch (mode) {
    case Q_PLAIN:
      return launch_quant_m<T, Q_PLAIN>(x, M, K, ldx, s_ptr, sr_ptr, q, r, ws, st, num_sms, stream, after_amax);
    case Q_MAIN_AMAXR:
      return launch_quant_m<T, Q_MAIN_AMAXR>(x, M, K, ldx, s_ptr, sr_ptr, q, r, ws, st, num_sms, stream, after_amax);
    case Q_RES_ONLY:
      return launch_quant_m<T, Q_RES_ONLY>(x, M, K, ldx, s_ptr, sr_ptr, q, r, ws, st, num_sms, stream, after_amax);
    default:
      return launch_quant_m<T, Q_BOTH>(x, M, K, ldx, s_ptr, sr_ptr, q, r, ws, st, num_sms, stream, after_amax);
  }
}

cudaError_t launch_quant(int mode, const void* x, nvfp4_dtype dt, int64_t M, int64_t K, int64_t ldx,
                         const float* s_ptr, const float* sr_ptr, const QOut& q, const QOut& r,
                         WsHeader* ws, int* st, int num_sms, cudaStream_t stream, bool after_amax) {
  return dt == NVFP4_BF16
             ? launch_quant_t<__nv_bfloat16>(mode, x, M, K, ldx, s_ptr, sr_ptr, q, r, ws, st, num_sms, stream, after_amax)
             : launch_quant_t<float>(mode, x, M, K, ldx, s_ptr, sr_ptr, q, r, ws, st, num_sms, stream, after_amax);
}

template <typename T, int NC>
cudaError_t launch_rms_stats_nc(const void* x, int64_t M, int64_t K, int64_t ldx, const void* gamma,
                                float eps, WsHeader* ws, float* rinv, float* s_out, bool want_scale,
                                int* st, int num_sms, cudaStream_t stream) {
  const unsigned g = (unsigned)std::max<int64_t>(1, std::min<int64_t>(M, (int64_t)num_sms * 8));
  k_rms_stats<T, NC><<<g, 256, 0, stream>>>(static_cast<const T*>(x), M, K, ldx, static_cast<const T*>(gamma),
                                            eps, ws, rinv, s_out, want_scale, st);
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_rms_stats_t(const void* x, int64_t M, int64_t K, int64_t ldx, const void* gamma,
                               float eps, WsHeader* ws, float* rinv, float* s_out, bool want_scale,
                               int* st, int num_sms, cudaStream_t stream) {
  // 8-element units per thread when the row is held in registers (256 threads)
  const int64_t units = ((K >> 3) + 255) / 256;
  if (units <= 2) return launch_rms_stats_nc<T, 2>(x, M, K, ldx, gamma, eps, ws, rinv, s_out, want_scale, st, num_sms, stream);
  if (units <= 4) return launch_rms_stats_nc<T, 4>(x, M, K, ldx, gamma, eps, ws, rinv, s_out, want_scale, st, num_sms, stream);
  if (units <= 8) return launch_rms_stats_nc<T, 8>(x, M, K, ldx, gamma, eps, ws, rinv, s_out, want_scale, st, num_sms, stream);
  return launch_rms_stats_nc<T, 0>(x, M, K, ldx, gamma, eps, ws, rinv, s_out, want_scale, st, num_sms, stream);
}

cudaError_t launch_rms_stats(const void* x, nvfp4_dtype dt, int64_t M, int64_t K, int64_t ldx,
                             const void* gamma, float eps, WsHeader* ws, float* rinv, float* s_out,
                             bool want_scale, int* st, int num_sms, cudaStream_t stream) {
  return dt == NVFP4_BF16
             ? launch_rms_stats_t<__nv_bfloat16>(x, M, K, ldx, gamma, eps, ws, rinv, s_out, want_scale, st, num_sms, stream)
             : launch_rms_stats_t<float>(x, M, K, ldx, gamma, eps, ws, rinv, s_out, want_scale, st, num_sms, stream);
}

size_t reorder_smem_bytes(nvfp4_dtype dt, int64_t K, bool has_gamma) {
  const size_t es = dt == NVFP4_BF16 ? 2 : 4;
  return 2 * (size_t)K * es + (((size_t)K * 2 + 15) & ~size_t(15)) + (has_gamma ? (size_t)K * es : 0);
}

template <typename T>
cudaError_t launch_reorder_quant_t(const void* x, int64_t M, int64_t K, int64_t ldx, const void* gamma,
                                   const float* rinv, const int32_t* perm, int64_t S,
                                   const float* s_ptr, const QOut& q, int* st, int num_sms,
                                   cudaStream_t stream, bool after_stats) {
  const size_t smem = reorder_smem_bytes(sizeof(T) == 2 ? NVFP4_BF16 : NVFP4_F32, K, gamma != nullptr);
  cudaError_t e = cudaFuncSetAttribute(k_reorder_quant<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  // one wave of resident CTAs, several per SM so that rows overlap; a second
  // wave would repeat the table set-up for only a few rows each
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_reorder_quant<T>, 256, smem);
  if (e != cudaSuccess) return e;
  per_sm = std::max(1, std::min(per_sm, 8));
  const unsigned g = (unsigned)std::max<int64_t>(1, std::min<int64_t>(M, (int64_t)num_sms * per_sm));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(g);
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;   // after the statistics pass only
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = after_stats ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, k_reorder_quant<T>, static_cast<const T*>(x), M, K, ldx,
                            static_cast<const T*>(gamma), rinv, perm, S, s_ptr, q, st);
}

template <typename T>
cudaError_t launch_reorder_onepass_t(const void* x, int64_t M, int64_t K, int64_t ldx, const void* gamma,
                                     float eps, const int32_t* perm, int64_t S, const float* s_in,
                                     const QOut& q, WsHeader* ws, int* st, int num_sms, cudaStream_t stream) {
  constexpr size_t kMaxSmem = 227 * 1024;   // opt-in dynamic shared memory per CTA
  // The fewest rows per warp (up to 4) for which every row fits in the shared
  // memory of one wave of CTAs.  The kernel is bound by instruction issue, so
  // its time follows the busiest SM: the warps per CTA (4..8) are the ones
  // that put the fewest rows on any SM (2048 rows on 148 SMs: 7 warps, 14
  // rows per SM, where 8 warps leave 16 on most SMs and 8 on the rest).
  auto set_smem = [](size_t smem) {
    return cudaFuncSetAttribute(k_reorder_onepass<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  };
  cudaError_t e = cudaSuccess;
  for (int rpw = 1; rpw <= 4; ++rpw) {
    int wpc = 0;
    int64_t g = 0, best_load = INT64_MAX;
    for (int w = 8; w >= 4; --w) {
      const size_t smem = onepass_smem_bytes(sizeof(T), K, gamma != nullptr, rpw, w);
      if (smem > kMaxSmem) continue;
      e = set_smem(smem);
      if (e != cudaSuccess) return e;
      int occ = 0;
      e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, k_reorder_onepass<T>, 32 * w, smem);
      if (e != cudaSuccess) return e;
      const int64_t gw = (M + (int64_t)w * rpw - 1) / ((int64_t)w * rpw);   // CTAs of w warps
      if (occ < 1 || gw > (int64_t)occ * num_sms) continue;                 // not all resident at once
      const int64_t load = (gw + num_sms - 1) / num_sms * w;                // warps on the busiest SM
      if (load < best_load) {
        best_load = load;
        wpc = w;
        g = gw;
      }
    }
    if (wpc == 0) continue;
    const size_t smem = onepass_smem_bytes(sizeof(T), K, gamma != nullptr, rpw, wpc);
    e = set_smem(smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)g);
    cfg.blockDim = dim3(32 * wpc);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;   // all CTAs resident: they meet at the exchange
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, k_reorder_onepass<T>, static_cast<const T*>(x), M, K, ldx,
                           static_cast<const T*>(gamma), eps, perm, S, s_in, q, ws, rpw, st);
    if (e == cudaErrorCooperativeLaunchTooLarge) {
      (void)cudaGetLastError();
      return cudaErrorNotSupported;   // nothing ran; the two passes do the work
    }
    return e;
  }
  return cudaErrorNotSupported;
}

cudaError_t launch_reorder_onepass(const void* x, nvfp4_dtype dt, int64_t M, int64_t K, int64_t ldx,
                                   const void* gamma, float eps, const int32_t* perm, int64_t S,
                                   const float* s_in, const QOut& q, WsHeader* ws, int* st, int num_sms,
                                   cudaStream_t stream) {
  return dt == NVFP4_BF16
             ? launch_reorder_onepass_t<__nv_bfloat16>(x, M, K, ldx, gamma, eps, perm, S, s_in, q, ws, st, num_sms,
                                                       stream)
             : launch_reorder_onepass_t<float>(x, M, K, ldx, gamma, eps, perm, S, s_in, q, ws, st, num_sms, stream);
}

cudaError_t launch_reorder_quant(const void* x, nvfp4_dtype dt, int64_t M, int64_t K, int64_t ldx,
                                 const void* gamma, const float* rinv, const int32_t* perm,
                                 int64_t S, const float* s_ptr, const QOut& q, int* st, int num_sms,
                                 cudaStream_t stream, bool after_stats) {
  return dt == NVFP4_BF16
             ? launch_reorder_quant_t<__nv_bfloat16>(x, M, K, ldx, gamma, rinv, perm, S, s_ptr, q, st, num_sms,
                                                     stream, after_stats)
             : launch_reorder_quant_t<float>(x, M, K, ldx, gamma, rinv, perm, S, s_ptr, q, st, num_sms, stream,
                                             after_stats);
}

}  // namespace nvfp4
