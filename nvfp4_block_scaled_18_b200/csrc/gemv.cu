// Small-M (M <= 16) NVFP4 decode GEMV on CUDA cores, sm_100a.
//
// Computes Y[m,n] = s_a s_w * sum_b d_a[m,b] d_w[n,b] * sum_{k in b} v(a[m,k]) v(w[n,k])
// (+ s_r s_w * the same sum over the residue operand R), ResServe abstract:
// both contributions are accumulated on-chip and Y is written once.
// The small-M CUDA-core kernel of the ReSET summary (section "CUDA kernel
// optimisation") is the prior art this follows; the layout below is our own.
//
// Two kernels share the arithmetic below.  M <= 8 (k_gemv):
//   row-step = 1024 K-elements of one W row: 512 code bytes + 64 scale bytes.
//              The 32 lanes of a warp take consecutive 16-byte code chunks
//              (32 elements, two blocks) of the same row, so every copy of a
//              warp is one contiguous 512-byte segment.
//   warp     = RL = 2 rows of W at a time, one row-step of each per ring stage;
//              a cp.async ring of 4 stages per warp keeps 4.5 KB of W in flight.
//   CTA      = 8 warps on a block of rows (a multiple of 16), over one K slice.
//              The activation slice (and the residue's) is expanded once per
//              CTA into shared memory as int8 values 2 v(c) plus fp32 block
//              scales, so the inner loop only decodes W; the two rows of a
//              warp share every activation load.
//   cluster  = ks CTAs splitting K when the expanded activations of the whole
//              row do not fit (or to give small N more CTAs); each CTA keeps
//              its partial rows in shared memory and the owner of a row sums
//              the peers' partials through distributed shared memory.
//   end      = per row, the lane partials are reduced by a transposing
//              butterfly (V values over 32 lanes in V - 1 + 5 - log2 V
//              shuffles), scaled by 1/4 s_a s_w (the two doubled operands),
//              with the residue term s_r s_w folded in before the reduction.
// 8 < M <= 16 (k_gemv_lanes), where the dp4a rate bounds the time: one W row
// per lane, activations read at one address by the whole warp (see below).
// Math (both): W codes become int8 values 2 v(c) by a byte-permute table; a
// 16-element block dot is 4 dp4a (exact in int32, |dot| <= 2304); the block
// term dot * (d_a d_w) is exact in fp32 and is accumulated in fp32.
// k_gemv is a programmatic dependent: before griddepcontrol.wait it only asks
// L2 to prefetch its W rows (L2 is coherent), so every operand may come from
// the preceding kernel.
#include <algorithm>

#include "common.cuh"
#include "kernels.h"
#include "tcgen05.cuh"

namespace nvfp4 {
namespace {

using namespace tc;

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kStepCodes = 512;                      // 32 lanes x 16 code bytes
constexpr int kStepBytes = kStepCodes + 64;          // + 64 block scales
constexpr int kRingSteps = 8;                        // row-steps in flight per warp
constexpr int kRingBytes = kWarps * kRingSteps * kStepBytes;   // 36 KB
constexpr int kMaxKs = 8;
constexpr int kMaxRowsPerCta = 256;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async4(uint32_t dst, const void* src, int src_bytes) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;\n" ::"r"(dst), "l"(src), "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

// Eight E2M1 nibbles -> eight int8 values 2*v(c) (element i in byte i of lo:hi).
__device__ __forceinline__ void e2m1x8_to_i8(uint32_t c, uint32_t& lo, uint32_t& hi) {
  constexpr uint32_t kPosLo = 0x03020100u, kPosHi = 0x0C080604u;  // 0,1,2,3 | 4,6,8,12
  constexpr uint32_t kNegLo = 0xFDFEFF00u, kNegHi = 0xF4F8FAFCu;  // negated
  const uint32_t mag = c & 0x77777777u;
  const uint32_t sel = ((c >> 1) & 0x44444444u) | 0x32103210u;  // byte i of pos or of neg
  lo = __byte_perm(__byte_perm(kPosLo, kPosHi, mag), __byte_perm(kNegLo, kNegHi, mag), sel);
  hi = __byte_perm(__byte_perm(kPosLo, kPosHi, mag >> 16), __byte_perm(kNegLo, kNegHi, mag >> 16),
                   sel >> 16);
}

// Four E2M1 codes (bits 0-15) -> four int8 values 2 v(c) for the codes with a
// clear sign bit and 0 for the others: the codes themselves are the PRMT
// selectors (3-bit magnitude index + sign bit, which in the default PRMT mode
// replicates the selected byte's sign bit, 0 for every table byte).
__device__ __forceinline__ uint32_t e2m1x4_pos(uint32_t codes) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(0x03020100u), "r"(0x0C080604u), "r"(codes));
  return r;
}

// Two E4M3 bytes (first block in bits 0-7, second in bits 8-15) -> fp32
// (E4M3 values are exact in fp16).
__device__ __forceinline__ float2 e4m3x2_to_f32x2(uint32_t two) {
  uint32_t h2;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"((unsigned short)two));
  return __half22float2(*reinterpret_cast<const __half2*>(&h2));
}

// The V values v[] of every lane summed over the warp: afterwards each lane l
// holds the full sum of value l / (32 / V).
template <int V>
__device__ __forceinline__ float warp_transpose_sum(float (&v)[V], int lane) {
  int o = 16;
#pragma unroll
  for (int h = V / 2; h >= 1; h >>= 1, o >>= 1) {
    const bool up = (lane & o) != 0;
#pragma unroll
    for (int i = 0; i < h; ++i) {
      const float send = up ? v[i] : v[i + h];
      const float keep = up ? v[i + h] : v[i];
      v[i] = keep + __shfl_xor_sync(0xFFFFFFFFu, send, o);
    }
  }
  float s = v[0];
#pragma unroll
  for (; o >= 1; o >>= 1) s += __shfl_xor_sync(0xFFFFFFFFu, s, o);
  return s;
}

// Shared-memory layout of one CTA: the W ring, then the expanded activation
// (and residue) slice, then the partial rows a cluster exchanges.
struct GemvLayout {
  int slice_pairs;   // 64-element pairs in the largest K slice
  int xi, ri, xd, rd, part, bytes;
  __host__ __device__ GemvLayout(int MT, bool res, int pairs, int ks, int rows_per_cta) {
    slice_pairs = (pairs + ks - 1) / ks;
    const int xb = MT * slice_pairs * 64;    // int8 values
    const int db = MT * slice_pairs * 16;    // fp32 block scales, 4 per pair
    xi = kRingBytes;
    ri = xi + xb;
    xd = ri + (res ? xb : 0);
    rd = xd + db;
    part = rd + (res ? db : 0);
    bytes = part + (ks > 1 ? rows_per_cta * MT * 4 : 0);
  }
};

struct GemvParams {
  GemmArgs g;
  int ks, rows_per_cta, pairs;
  int prefetch;   // prefetch the W rows into L2 before the dependency wait
};

template <int MT, int RL, bool RES, bool BF16OUT>
__global__ void __launch_bounds__(kThreads, 2) k_gemv(const GemvParams p) {
  extern __shared__ __align__(128) unsigned char smem[];
  griddep_launch_dependents();
  const GemmArgs& g = p.g;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int K = (int)g.K, N = (int)g.N, M = (int)g.M;
  const int ks = p.ks;
  const int rank = ks > 1 ? (int)cluster_ctarank() : 0;
  const GemvLayout L(MT, RES, p.pairs, ks, p.rows_per_cta);
  // this CTA's K slice, in 64-element pairs
  const int pr0 = (rank * p.pairs) / ks, pr1 = ((rank + 1) * p.pairs) / ks;
  const int chunks = 2 * (pr1 - pr0);            // 32-element chunks in the slice
  const int k0 = pr0 * 64;
  const int steps = (chunks + 31) / 32;          // row-steps per row
  const int r0 = blockIdx.y * p.rows_per_cta;
  const int r1 = min(N, r0 + p.rows_per_cta);
  const int64_t cpitch = K / 2, spitch = K / 16;
  const int xpitch = L.slice_pairs * 64, dpitch = L.slice_pairs * 4;

  // warm L2 with this CTA's W rows while the preceding kernel finishes
  if (p.prefetch)
    for (int r = r0 + (int)threadIdx.x; r < r1; r += kThreads)
      prefetch_l2_bulk(g.w_codes + (int64_t)r * cpitch + k0 / 2, (uint32_t)chunks * 16u);
  griddep_wait();   // everything below may read the preceding kernel's results

  // ---- expand the activation (and residue) slice: int8 2 v(c) and fp32 scales
  for (int i = threadIdx.x; i < MT * chunks; i += kThreads) {
    const int m = i / chunks, c = i - m * chunks;
    uint4 cx = make_uint4(0u, 0u, 0u, 0u), cr = cx;
    if (m < M) {
      cx = __ldg(reinterpret_cast<const uint4*>(g.a_codes + (int64_t)m * cpitch + k0 / 2) + c);
      if (RES) cr = __ldg(reinterpret_cast<const uint4*>(g.r_codes + (int64_t)m * cpitch + k0 / 2) + c);
    }
    uint4 o0, o1;
    e2m1x8_to_i8(cx.x, o0.x, o0.y);
    e2m1x8_to_i8(cx.y, o0.z, o0.w);
    e2m1x8_to_i8(cx.z, o1.x, o1.y);
    e2m1x8_to_i8(cx.w, o1.z, o1.w);
    uint4* dst = reinterpret_cast<uint4*>(smem + L.xi + m * xpitch + c * 32);
    dst[0] = o0;
    dst[1] = o1;
    if (RES) {
      e2m1x8_to_i8(cr.x, o0.x, o0.y);
      e2m1x8_to_i8(cr.y, o0.z, o0.w);
      e2m1x8_to_i8(cr.z, o1.x, o1.y);
      e2m1x8_to_i8(cr.w, o1.z, o1.w);
      uint4* rdst = reinterpret_cast<uint4*>(smem + L.ri + m * xpitch + c * 32);
      rdst[0] = o0;
      rdst[1] = o1;
    }
  }
  for (int i = threadIdx.x; i < MT * 2 * chunks; i += kThreads) {
    const int m = i / (2 * chunks), b = i - m * 2 * chunks;
    float dx = 0.0f, dr = 0.0f;
    if (m < M) {
      dx = e4m3_value(g.a_scales[(int64_t)m * spitch + k0 / 16 + b]);
      if (RES) dr = e4m3_value(g.r_scales[(int64_t)m * spitch + k0 / 16 + b]);
    }
    reinterpret_cast<float*>(smem + L.xd)[m * dpitch + b] = dx;
    if (RES) reinterpret_cast<float*>(smem + L.rd)[m * dpitch + b] = dr;
  }
  const float alpha = 0.25f * (*g.a_s) * (*g.w_s);
  const float alpha_r = RES ? 0.25f * (*g.r_s) * (*g.w_s) : 0.0f;
  __syncthreads();

  // ---- stream W: warp w takes row groups w, w + 8, ... of RL rows each
  constexpr int kStages = kRingSteps / RL;
  constexpr bool kSplitSign = MT <= 2;   // fewer ALU operations per W element where the dp4a rate has room
  unsigned char* ring = smem + warp * (kRingSteps * kStepBytes);
  const int groups = (r1 - r0 + RL - 1) / RL;
  const int my_groups = groups > warp ? (groups - warp + kWarps - 1) / kWarps : 0;
  const int total = my_groups * steps;

  // Issue side: this lane's source pointers in the rows of the group being
  // issued, advanced by one row-step (512 code bytes, 64 scale bytes) per
  // issue.  A copy with nothing to read (past the slice or past N) reads 0
  // bytes from the matrix base and zero-fills its slot.
  const uint8_t* ic[RL];
  const uint8_t* isc[RL];
  bool iok[RL];
  int is_g = 0, is_t = 0;   // next (group, step) to issue
  auto set_group = [&](int gi) {
#pragma unroll
    for (int rr = 0; rr < RL; ++rr) {
      const int r = r0 + (warp + gi * kWarps) * RL + rr;
      iok[rr] = r < r1;
      const int64_t rc = iok[rr] ? r : r0;
      ic[rr] = g.w_codes + rc * cpitch + k0 / 2 + lane * 16;
      isc[rr] = g.w_scales + rc * spitch + k0 / 16 + lane * 4;
    }
  };
  set_group(0);
  auto issue = [&](int slot) {
    unsigned char* sb = ring + slot * (RL * kStepBytes);
    const bool cv = is_t * 32 + lane < chunks;          // this lane's 16 code bytes
    const bool bv = is_t * 64 + lane * 4 < 2 * chunks;  // lanes 0-15: 4 block scales (chunks 2 lane, 2 lane + 1)
#pragma unroll
    for (int rr = 0; rr < RL; ++rr) {
      const bool okc = iok[rr] && cv, oks = iok[rr] && bv;
      cp_async16(smem_u32(sb + rr * kStepBytes + lane * 16), okc ? ic[rr] : g.w_codes, okc ? 16 : 0);
      if (lane < 16)
        cp_async4(smem_u32(sb + rr * kStepBytes + kStepCodes + lane * 4), oks ? isc[rr] : g.w_scales, oks ? 4 : 0);
      ic[rr] += kStepCodes;
      isc[rr] += 64;
    }
    if (++is_t == steps) {
      is_t = 0;
      set_group(++is_g);
    }
  };

  float acc[RL][MT];
  float accr[RES ? RL : 1][RES ? MT : 1];
#pragma unroll
  for (int rr = 0; rr < RL; ++rr)
#pragma unroll
    for (int m = 0; m < MT; ++m) acc[rr][m] = 0.0f;
#pragma unroll
  for (int rr = 0; rr < (RES ? RL : 1); ++rr)
#pragma unroll
    for (int m = 0; m < (RES ? MT : 1); ++m) accr[rr][m] = 0.0f;

#pragma unroll
  for (int i = 0; i < kStages; ++i) {
    if (i < total) issue(i);
    cp_async_commit();
  }
  int slot = 0, cg = 0, ct = 0;   // group and step being computed
  for (int j = 0; j < total; ++j) {
    cp_async_wait<kStages - 1>();
    __syncwarp();
    const unsigned char* sb = ring + slot * (RL * kStepBytes);
    const int cx = min(ct * 32 + lane, chunks - 1);   // this lane's chunk (W is zero past the slice)
    // W as int8 2 v(c): signed values (w8), or with kSplitSign the magnitudes of
    // the positive codes (w8) and of the negative codes (wn) apart, 2 PRMT per 4
    // elements and no masking; the dot is then dp4a(w8, x) - dp4a(wn, x).
    uint32_t w8[RL][8];
    uint32_t wn[kSplitSign ? RL : 1][8];
    float2 dw[RL];
#pragma unroll
    for (int rr = 0; rr < RL; ++rr) {
      const uint4 wc = *reinterpret_cast<const uint4*>(sb + rr * kStepBytes + lane * 16);
      dw[rr] = e4m3x2_to_f32x2(*reinterpret_cast<const uint16_t*>(sb + rr * kStepBytes + kStepCodes + lane * 2));
      if constexpr (kSplitSign) {
        const uint32_t cw[4] = {wc.x, wc.y, wc.z, wc.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint32_t cn = cw[q] ^ 0x88888888u;
          w8[rr][2 * q] = e2m1x4_pos(cw[q]);
          w8[rr][2 * q + 1] = e2m1x4_pos(cw[q] >> 16);
          wn[kSplitSign ? rr : 0][2 * q] = e2m1x4_pos(cn);
          wn[kSplitSign ? rr : 0][2 * q + 1] = e2m1x4_pos(cn >> 16);
        }
      } else {
        e2m1x8_to_i8(wc.x, w8[rr][0], w8[rr][1]);
        e2m1x8_to_i8(wc.y, w8[rr][2], w8[rr][3]);
        e2m1x8_to_i8(wc.z, w8[rr][4], w8[rr][5]);
        e2m1x8_to_i8(wc.w, w8[rr][6], w8[rr][7]);
      }
    }
    // block dot of W row rr (words o..o+3) with activation words v
    auto bdot = [&](int rr, int o, const uint4& v) {
      int d = __dp4a((int)w8[rr][o], (int)v.x, 0);
      d = __dp4a((int)w8[rr][o + 1], (int)v.y, d);
      d = __dp4a((int)w8[rr][o + 2], (int)v.z, d);
      d = __dp4a((int)w8[rr][o + 3], (int)v.w, d);
      if constexpr (kSplitSign) {
        const int k = kSplitSign ? rr : 0;
        int e = __dp4a((int)wn[k][o], (int)v.x, 0);
        e = __dp4a((int)wn[k][o + 1], (int)v.y, e);
        e = __dp4a((int)wn[k][o + 2], (int)v.z, e);
        e = __dp4a((int)wn[k][o + 3], (int)v.w, e);
        d -= e;
      }
      return d;
    };
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      const uint4* xs = reinterpret_cast<const uint4*>(smem + L.xi + m * xpitch + cx * 32);
      const uint4 x0 = xs[0], x1 = xs[1];
      const float2 dx = *reinterpret_cast<const float2*>(smem + L.xd + (m * dpitch + 2 * cx) * 4);
#pragma unroll
      for (int rr = 0; rr < RL; ++rr) {
        const int d0 = bdot(rr, 0, x0), d1 = bdot(rr, 4, x1);
        acc[rr][m] = fmaf(__int2float_rn(d0), dx.x * dw[rr].x, acc[rr][m]);
        acc[rr][m] = fmaf(__int2float_rn(d1), dx.y * dw[rr].y, acc[rr][m]);
      }
      if (RES) {
        const uint4* rs = reinterpret_cast<const uint4*>(smem + L.ri + m * xpitch + cx * 32);
        const uint4 y0 = rs[0], y1 = rs[1];
        const float2 dr = *reinterpret_cast<const float2*>(smem + L.rd + (m * dpitch + 2 * cx) * 4);
#pragma unroll
        for (int rr = 0; rr < RL; ++rr) {
          float& a = accr[RES ? rr : 0][RES ? m : 0];
          const int d0 = bdot(rr, 0, y0), d1 = bdot(rr, 4, y1);
          a = fmaf(__int2float_rn(d0), dr.x * dw[rr].x, a);
          a = fmaf(__int2float_rn(d1), dr.y * dw[rr].y, a);
        }
      }
    }
    __syncwarp();
    if (j + kStages < total) issue(slot);
    cp_async_commit();
    if (++slot == kStages) slot = 0;

    if (++ct == steps) {   // the group's rows are complete: reduce over the lanes, store
      constexpr int V = RL * MT;
      float v[V];
#pragma unroll
      for (int rr = 0; rr < RL; ++rr)
#pragma unroll
        for (int m = 0; m < MT; ++m) {
          v[rr * MT + m] = RES ? fmaf(acc[rr][m], alpha, accr[RES ? rr : 0][RES ? m : 0] * alpha_r)
                               : acc[rr][m] * alpha;
          acc[rr][m] = 0.0f;
          if (RES) accr[RES ? rr : 0][RES ? m : 0] = 0.0f;
        }
      const float s = warp_transpose_sum<V>(v, lane);
      constexpr int kGroup = 32 / V;
      if (lane % kGroup == 0) {
        const int idx = lane / kGroup, rr = idx / MT, m = idx - rr * MT;
        const int rl = (warp + cg * kWarps) * RL + rr;   // row within the CTA's block
        if (m < M && r0 + rl < r1) {
          if (ks > 1)
            reinterpret_cast<float*>(smem + L.part)[rl * MT + m] = s;
          else if (BF16OUT)
            reinterpret_cast<__nv_bfloat16*>(g.y)[m * g.ldy + r0 + rl] = __float2bfloat16_rn(s);
          else
            reinterpret_cast<float*>(g.y)[m * g.ldy + r0 + rl] = s;
        }
      }
      ct = 0;
      ++cg;
    }
  }
  cp_async_wait<0>();
  if (ks == 1) return;

  // ---- K split: owner `rank` sums rows [rank R / ks, (rank + 1) R / ks) of the
  // block over every peer's partials, in rank order
  cluster_sync();
  const int rows = r1 - r0;
  const int q0 = (rank * rows) / ks, q1 = ((rank + 1) * rows) / ks;
  const uint32_t part = smem_u32(smem + L.part);
  for (int i = threadIdx.x; i < (q1 - q0) * MT; i += kThreads) {
    const int rl = q0 + i / MT, m = i % MT;
    if (m >= M) continue;
    float s = 0.0f;
    for (int src = 0; src < ks; ++src)
      s += ld_cluster_f32(mapa_shared(part + (uint32_t)(rl * MT + m) * 4u, (uint32_t)src));
    if (BF16OUT)
      reinterpret_cast<__nv_bfloat16*>(g.y)[m * g.ldy + r0 + rl] = __float2bfloat16_rn(s);
    else
      reinterpret_cast<float*>(g.y)[m * g.ldy + r0 + rl] = s;
  }
  cluster_sync();   // no CTA exits while a peer may still read its partials
}

// ------------------------------------------------------------------------
// 8 < M <= 16: one W row per lane.  A CTA of 8 warps takes 32 rows of W; K is
// split into 8 contiguous ranges, one per warp.  Each lane streams its row (32
// code bytes + 4 scale bytes per 64-element step) through a 6-deep per-warp
// cp.async ring together with the activation codes of the same step, which
// the warp expands once per step and every lane then reads at the same
// address (a broadcast).  With eight or more activation rows the dp4a rate,
// not the W stream, bounds the kernel, and the broadcast reads keep the
// shared-memory traffic per W element independent of M.

constexpr int kLaneStages = 6;

template <int MT, bool RES>
struct LaneLayout {
  // one ring slot
  static constexpr int kWc = 0;                        // 32 lanes x 32 code bytes
  static constexpr int kWs = 1024;                     // 32 lanes x 4 scale bytes
  static constexpr int kXc = 1152;                     // MT x 32 code bytes
  static constexpr int kXs = kXc + MT * 32;            // MT x 4 scale bytes
  static constexpr int kRc = ((kXs + MT * 4 + 15) / 16) * 16;
  static constexpr int kRs = kRc + MT * 32;
  static constexpr int kSlot = RES ? ((kRs + MT * 4 + 15) / 16) * 16 : kRc;
  // expanded activations of the current step (per warp)
  static constexpr int kXi = kLaneStages * kSlot;          // MT x 64 int8
  static constexpr int kXd = kXi + MT * 64;            // MT x 4 fp32
  static constexpr int kRi = kXd + MT * 16;
  static constexpr int kRd = kRi + MT * 64;
  static constexpr int kWarpBytes = RES ? kRd + MT * 16 : kRi;
  static constexpr int kCtaBytes = kWarps * kWarpBytes;
  static constexpr int kReduceBytes = kWarps * MT * 32 * 4 * (RES ? 2 : 1);
  static constexpr int kSmem = kCtaBytes > kReduceBytes ? kCtaBytes : kReduceBytes;
};

template <int MT, bool RES, bool BF16OUT>
__global__ void __launch_bounds__(256, 1) k_gemv_lanes(GemmArgs g) {
  using L = LaneLayout<MT, RES>;
  extern __shared__ __align__(128) unsigned char smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  unsigned char* wbase = smem + warp * L::kWarpBytes;
  const int64_t K = g.K, N = g.N;
  const int Mreal = (int)g.M;
  const int64_t n0 = (int64_t)blockIdx.x * 32;
  const int64_t n = n0 + lane;
  const bool row_ok = n < N;
  const int T = (int)(K / 64);
  const int t0 = (warp * T) / kWarps, t1 = ((warp + 1) * T) / kWarps;
  const int64_t cpitch = K / 2, spitch = K / 16;

  // per-lane source pointers, fixed for the whole kernel (step t adds t*32 / t*4)
  const uint8_t* wrow_c = g.w_codes + (row_ok ? n : 0) * cpitch;
  const uint8_t* wrow_s = g.w_scales + (row_ok ? n : 0) * spitch;
  const int wbytes16 = row_ok ? 16 : 0, wbytes4 = row_ok ? 4 : 0;
  const int swz = (lane >> 2) & 1;  // swaps the lane's two 16-byte halves: conflict-free reads
  // activation slices: lane i < 2*MT copies half h of row m's 32 code bytes, lane m < MT its 4 scale bytes
  const int xm = lane >> 1, xh = lane & 1;
  const bool x_lane = lane < 2 * MT, xrow_ok = x_lane && xm < Mreal;
  const uint8_t* xc_src = g.a_codes + (xrow_ok ? xm : 0) * cpitch + xh * 16;
  const uint8_t* rc_src = RES ? g.r_codes + (xrow_ok ? xm : 0) * cpitch + xh * 16 : nullptr;
  const bool s_lane = lane < MT, srow_ok = s_lane && lane < Mreal;
  const uint8_t* xs_src = g.a_scales + (srow_ok ? lane : 0) * spitch;
  const uint8_t* rs_src = RES ? g.r_scales + (srow_ok ? lane : 0) * spitch : nullptr;

  auto issue = [&](int t, int slot) {
    unsigned char* sb = wbase + slot * L::kSlot;
    const uint32_t wc = smem_u32(sb + L::kWc + lane * 32);
    cp_async16(wc + ((0 ^ swz) << 4), wrow_c + t * 32, wbytes16);
    cp_async16(wc + ((1 ^ swz) << 4), wrow_c + t * 32 + 16, wbytes16);
    cp_async4(smem_u32(sb + L::kWs + lane * 4), wrow_s + t * 4, wbytes4);
    if (x_lane) {
      cp_async16(smem_u32(sb + L::kXc + xm * 32 + xh * 16), xc_src + t * 32, xrow_ok ? 16 : 0);
      if (RES) cp_async16(smem_u32(sb + L::kRc + xm * 32 + xh * 16), rc_src + t * 32, xrow_ok ? 16 : 0);
    }
    if (s_lane) {
      cp_async4(smem_u32(sb + L::kXs + lane * 4), xs_src + t * 4, srow_ok ? 4 : 0);
      if (RES) cp_async4(smem_u32(sb + L::kRs + lane * 4), rs_src + t * 4, srow_ok ? 4 : 0);
    }
  };

  // activation codes -> int8, scales -> fp32 (cooperatively, once per step per warp)
  auto expand = [&](int slot) {
    const unsigned char* sb = wbase + slot * L::kSlot;
    for (int i = lane; i < 2 * MT; i += 32) {
      const int m = i >> 1, h = i & 1;
      const uint4 c = *reinterpret_cast<const uint4*>(sb + L::kXc + m * 32 + h * 16);
      uint4 o0, o1;
      e2m1x8_to_i8(c.x, o0.x, o0.y);
      e2m1x8_to_i8(c.y, o0.z, o0.w);
      e2m1x8_to_i8(c.z, o1.x, o1.y);
      e2m1x8_to_i8(c.w, o1.z, o1.w);
      uint4* dst = reinterpret_cast<uint4*>(wbase + L::kXi + m * 64 + h * 32);
      dst[0] = o0;
      dst[1] = o1;
      if (RES) {
        const uint4 rc = *reinterpret_cast<const uint4*>(sb + L::kRc + m * 32 + h * 16);
        e2m1x8_to_i8(rc.x, o0.x, o0.y);
        e2m1x8_to_i8(rc.y, o0.z, o0.w);
        e2m1x8_to_i8(rc.z, o1.x, o1.y);
        e2m1x8_to_i8(rc.w, o1.z, o1.w);
        uint4* rdst = reinterpret_cast<uint4*>(wbase + L::kRi + m * 64 + h * 32);
        rdst[0] = o0;
        rdst[1] = o1;
      }
    }
    for (int m = lane; m < MT; m += 32) {
      const uint32_t s4 = *reinterpret_cast<const uint32_t*>(sb + L::kXs + m * 4);
      *reinterpret_cast<float4*>(wbase + L::kXd + m * 16) =
          make_float4(e4m3_value(s4 & 0xFF), e4m3_value((s4 >> 8) & 0xFF),
                      e4m3_value((s4 >> 16) & 0xFF), e4m3_value(s4 >> 24));
      if (RES) {
        const uint32_t r4 = *reinterpret_cast<const uint32_t*>(sb + L::kRs + m * 4);
        *reinterpret_cast<float4*>(wbase + L::kRd + m * 16) =
            make_float4(e4m3_value(r4 & 0xFF), e4m3_value((r4 >> 8) & 0xFF),
                        e4m3_value((r4 >> 16) & 0xFF), e4m3_value(r4 >> 24));
      }
    }
  };

  float acc[MT], accr[RES ? MT : 1];
#pragma unroll
  for (int m = 0; m < MT; ++m) acc[m] = 0.0f;
#pragma unroll
  for (int m = 0; m < (RES ? MT : 1); ++m) accr[m] = 0.0f;

#pragma unroll
  for (int i = 0; i < kLaneStages; ++i) {
    if (t0 + i < t1) issue(t0 + i, i);
    cp_async_commit();
  }
  int slot = 0;
  for (int t = t0; t < t1; ++t) {
    cp_async_wait<kLaneStages - 1>();
    __syncwarp();
    expand(slot);
    __syncwarp();
    const unsigned char* sb = wbase + slot * L::kSlot;
    const uint4 wlo = *reinterpret_cast<const uint4*>(sb + L::kWc + lane * 32 + ((0 ^ swz) << 4));
    const uint4 whi = *reinterpret_cast<const uint4*>(sb + L::kWc + lane * 32 + ((1 ^ swz) << 4));
    const uint32_t wsc = *reinterpret_cast<const uint32_t*>(sb + L::kWs + lane * 4);
    const uint32_t wcw[8] = {wlo.x, wlo.y, wlo.z, wlo.w, whi.x, whi.y, whi.z, whi.w};
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      uint32_t w0, w1, w2, w3;
      e2m1x8_to_i8(wcw[2 * b], w0, w1);
      e2m1x8_to_i8(wcw[2 * b + 1], w2, w3);
      const float dw = e4m3_value((wsc >> (8 * b)) & 0xFF);
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        const uint4 xv = *reinterpret_cast<const uint4*>(wbase + L::kXi + m * 64 + b * 16);
        int dot = __dp4a((int)w0, (int)xv.x, 0);
        dot = __dp4a((int)w1, (int)xv.y, dot);
        dot = __dp4a((int)w2, (int)xv.z, dot);
        dot = __dp4a((int)w3, (int)xv.w, dot);
        const float dx = *reinterpret_cast<const float*>(wbase + L::kXd + m * 16 + b * 4);
        acc[m] = fmaf(__int2float_rn(dot), dx * dw, acc[m]);
        if (RES) {
          const uint4 rv = *reinterpret_cast<const uint4*>(wbase + L::kRi + m * 64 + b * 16);
          int rdot = __dp4a((int)w0, (int)rv.x, 0);
          rdot = __dp4a((int)w1, (int)rv.y, rdot);
          rdot = __dp4a((int)w2, (int)rv.z, rdot);
          rdot = __dp4a((int)w3, (int)rv.w, rdot);
          const float dr = *reinterpret_cast<const float*>(wbase + L::kRd + m * 16 + b * 4);
          accr[RES ? m : 0] = fmaf(__int2float_rn(rdot), dr * dw, accr[RES ? m : 0]);
        }
      }
    }
    __syncwarp();
    if (t + kLaneStages < t1) issue(t + kLaneStages, slot);
    cp_async_commit();
    if (++slot == kLaneStages) slot = 0;
  }
  cp_async_wait<0>();

  // cross-warp reduction of the K-split partial sums
  __syncthreads();
  float* red = reinterpret_cast<float*>(smem);
#pragma unroll
  for (int m = 0; m < MT; ++m) {
    red[(warp * MT + m) * 32 + lane] = acc[m];
    if (RES) red[((kWarps + warp) * MT + m) * 32 + lane] = accr[RES ? m : 0];
  }
  __syncthreads();
  const float alpha = 0.25f * (*g.a_s) * (*g.w_s);
  const float alpha_r = RES ? 0.25f * (*g.r_s) * (*g.w_s) : 0.0f;
  for (int idx = threadIdx.x; idx < MT * 32; idx += blockDim.x) {
    const int m = idx >> 5, l = idx & 31;
    float sum = 0.0f, sumr = 0.0f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      sum += red[(w * MT + m) * 32 + l];
      if (RES) sumr += red[((kWarps + w) * MT + m) * 32 + l];
    }
    const int64_t nn = n0 + l;
    if (m < Mreal && nn < N) {
      const float out = RES ? fmaf(sum, alpha, sumr * alpha_r) : sum * alpha;
      if (BF16OUT)
        reinterpret_cast<__nv_bfloat16*>(g.y)[m * g.ldy + nn] = __float2bfloat16_rn(out);
      else
        reinterpret_cast<float*>(g.y)[m * g.ldy + nn] = out;
    }
  }
}

template <int MT, bool RES, bool BF16OUT>
cudaError_t launch_lanes_t(const GemmArgs& g, cudaStream_t stream) {
  constexpr int smem = LaneLayout<MT, RES>::kSmem;
  cudaError_t e = cudaFuncSetAttribute(k_gemv_lanes<MT, RES, BF16OUT>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const unsigned grid = (unsigned)((g.N + 31) / 32);
  k_gemv_lanes<MT, RES, BF16OUT><<<grid, 256, smem, stream>>>(g);
  return cudaGetLastError();
}

template <int MT>
cudaError_t launch_lanes_m(const GemmArgs& g, cudaStream_t stream) {
  const bool res = g.r_codes != nullptr;
  if (res) return g.y_bf16 ? launch_lanes_t<MT, true, true>(g, stream) : launch_lanes_t<MT, true, false>(g, stream);
  return g.y_bf16 ? launch_lanes_t<MT, false, true>(g, stream) : launch_lanes_t<MT, false, false>(g, stream);
}


// ------------------------------------------------------------------ host side

constexpr int kSmemTwoPerSm = 233472 / 2 - 1024;   // two CTAs per SM (228 KB, 1 KB reserved per CTA)
constexpr int kSmemMax = 232448;

struct GemvChoice {
  int ks = 0, rows_per_cta = 0, smem = 0;
};

// The fewest CTAs per cluster whose expanded activation slice fits (two CTAs
// per SM if possible, else one), then more of them while the grid has fewer
// CTAs than resident slots, then rows per CTA so that one wave covers N.
GemvChoice choose(int MT, int RL, bool res, int N, int K, int num_sms) {
  const int pairs = K / 64;
  auto bytes = [&](int ks) { return GemvLayout(MT, res, pairs, ks, kMaxRowsPerCta).bytes; };
  GemvChoice c;
  int per_sm = 0, budget = 0;
  for (int b : {kSmemTwoPerSm, kSmemMax}) {
    ++per_sm;
    for (int ks = 1; ks <= std::min(kMaxKs, pairs) && c.ks == 0; ++ks)
      if (bytes(ks) <= b) c.ks = ks;
    if (c.ks > 0) {
      budget = b;
      per_sm = b == kSmemTwoPerSm ? 2 : 1;
      break;
    }
  }
  if (c.ks == 0) return c;
  const int group_rows = kWarps * RL;
  const int blocks_min = (N + group_rows - 1) / group_rows;   // one row group per warp
  const int slots = per_sm * num_sms;
  while (c.ks < std::min(kMaxKs, pairs / 16) && blocks_min * (c.ks + 1) <= slots && bytes(c.ks + 1) <= budget)
    ++c.ks;
  const int blocks_target = std::max(1, slots / c.ks);
  const int groups_per_cta = (blocks_min + blocks_target - 1) / blocks_target;
  c.rows_per_cta = std::min(kMaxRowsPerCta, groups_per_cta * group_rows);
  c.smem = GemvLayout(MT, res, pairs, c.ks, c.rows_per_cta).bytes;
  return c;
}

template <int MT, int RL, bool RES, bool BF16OUT>
cudaError_t launch_t(const GemmArgs& g, int num_sms, cudaStream_t stream) {
  const GemvChoice c = choose(MT, RL, RES, (int)g.N, (int)g.K, num_sms);
  if (c.ks == 0) return cudaErrorNotSupported;
  auto kern = k_gemv<MT, RL, RES, BF16OUT>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, c.smem);
  if (e != cudaSuccess) return e;
  const GemvParams p{g, c.ks, c.rows_per_cta, (int)(g.K / 64), prefetch_w(g.N, g.K) ? 1 : 0};
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)c.ks, (unsigned)((g.N + c.rows_per_cta - 1) / c.rows_per_cta), 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = (size_t)c.smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)c.ks;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;   // overlap the preceding kernel's tail
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kern, p);
}

template <int MT, int RL>
cudaError_t launch_m(const GemmArgs& g, int num_sms, cudaStream_t stream) {
  if (g.r_codes != nullptr)
    return g.y_bf16 ? launch_t<MT, RL, true, true>(g, num_sms, stream)
                    : launch_t<MT, RL, true, false>(g, num_sms, stream);
  return g.y_bf16 ? launch_t<MT, RL, false, true>(g, num_sms, stream)
                  : launch_t<MT, RL, false, false>(g, num_sms, stream);
}

}  // namespace

cudaError_t launch_gemv(const GemmArgs& g, int num_sms, cudaStream_t stream) {
  if (g.K % 64 != 0 || g.M < 1 || g.M > 16) return cudaErrorNotSupported;
  if (g.M <= 1) return launch_m<1, 2>(g, num_sms, stream);
  if (g.M <= 2) return launch_m<2, 2>(g, num_sms, stream);
  if (g.M <= 4) return launch_m<4, 2>(g, num_sms, stream);
  if (g.M <= 8) return launch_m<8, 2>(g, num_sms, stream);
  return launch_lanes_m<16>(g, stream);
}

}  // namespace nvfp4
