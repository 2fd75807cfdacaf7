// Small-M (M <= 16) NVFP4 decode GEMV on CUDA cores, sm_100a.
//
// Computes Y[m,n] = s_a s_w * sum_b d_a[m,b] d_w[n,b] * sum_{k in b} v(a[m,k]) v(w[n,k])
// (+ s_r s_w * the same sum over the residue operand R), ResServe abstract:
// both contributions are accumulated on-chip and Y is written once.
// The small-M CUDA-core kernel of the ReSET summary (section "CUDA kernel
// optimisation") is the prior art this follows; the layout below is our own.
//
// Layout of the work
//   CTA   = 8 warps on a tile of 32 rows of W (lane = row); the K dimension is
//           split into 8 contiguous ranges, one per warp; partial sums are
//           reduced through shared memory at the end.
//   step  = 64 K-elements (4 blocks of 16).  Each lane streams its own row's
//           32 code bytes + 4 scale bytes per step from HBM into a 6-deep
//           per-warp shared-memory ring with cp.async (zero-filled past N),
//           together with the activation codes/scales of the same K range.
//   math  = codes become int8 values 2*v(c) in {-12..12} through a byte
//           permute table; a 16-block dot product is 4 dp4a instructions
//           (exact in int32, |sum| <= 2304); the block term
//           idot * (d_a d_w) is exact in fp32 and is accumulated in fp32;
//           the factor 1/4 (two doubled operands) and s_a s_w are applied once.
#include "common.cuh"
#include "kernels.h"

namespace nvfp4 {
namespace {

constexpr int kWarps = 8;
constexpr int kStages = 6;

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

template <int MT, bool RES>
struct Layout {
  // one ring slot
  static constexpr int kWc = 0;                        // 32 lanes x 32 code bytes
  static constexpr int kWs = 1024;                     // 32 lanes x 4 scale bytes
  static constexpr int kXc = 1152;                     // MT x 32 code bytes
  static constexpr int kXs = kXc + MT * 32;            // MT x 4 scale bytes
  static constexpr int kRc = ((kXs + MT * 4 + 15) / 16) * 16;
  static constexpr int kRs = kRc + MT * 32;
  static constexpr int kSlot = RES ? ((kRs + MT * 4 + 15) / 16) * 16 : kRc;
  // expanded activations of the current step (per warp)
  static constexpr int kXi = kStages * kSlot;          // MT x 64 int8
  static constexpr int kXd = kXi + MT * 64;            // MT x 4 fp32
  static constexpr int kRi = kXd + MT * 16;
  static constexpr int kRd = kRi + MT * 64;
  static constexpr int kWarpBytes = RES ? kRd + MT * 16 : kRi;
  static constexpr int kCtaBytes = kWarps * kWarpBytes;
  static constexpr int kReduceBytes = kWarps * MT * 32 * 4 * (RES ? 2 : 1);
  static constexpr int kSmem = kCtaBytes > kReduceBytes ? kCtaBytes : kReduceBytes;
};

template <int MT, bool RES, bool BF16OUT>
__global__ void __launch_bounds__(256, 1) k_gemv(GemmArgs g) {
  using L = Layout<MT, RES>;
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
  for (int i = 0; i < kStages; ++i) {
    if (t0 + i < t1) issue(t0 + i, i);
    cp_async_commit();
  }
  int slot = 0;
  for (int t = t0; t < t1; ++t) {
    cp_async_wait<kStages - 1>();
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
    if (t + kStages < t1) issue(t + kStages, slot);
    cp_async_commit();
    if (++slot == kStages) slot = 0;
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
cudaError_t launch_t(const GemmArgs& g, cudaStream_t stream) {
  constexpr int smem = Layout<MT, RES>::kSmem;
  cudaError_t e = cudaFuncSetAttribute(k_gemv<MT, RES, BF16OUT>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const unsigned grid = (unsigned)((g.N + 31) / 32);
  k_gemv<MT, RES, BF16OUT><<<grid, 256, smem, stream>>>(g);
  return cudaGetLastError();
}

template <int MT>
cudaError_t launch_m(const GemmArgs& g, cudaStream_t stream) {
  const bool res = g.r_codes != nullptr;
  if (res) return g.y_bf16 ? launch_t<MT, true, true>(g, stream) : launch_t<MT, true, false>(g, stream);
  return g.y_bf16 ? launch_t<MT, false, true>(g, stream) : launch_t<MT, false, false>(g, stream);
}

}  // namespace

cudaError_t launch_gemv(const GemmArgs& g, int /*num_sms*/, cudaStream_t stream) {
  if (g.M <= 1) return launch_m<1>(g, stream);
  if (g.M <= 2) return launch_m<2>(g, stream);
  if (g.M <= 4) return launch_m<4>(g, stream);
  if (g.M <= 8) return launch_m<8>(g, stream);
  return launch_m<16>(g, stream);
}

}  // namespace nvfp4
