// Large-M NVFP4 W4A4 GEMM on the 5th-generation tensor cores (tcgen05), sm_100a.
//
// Y = s_a s_w * A W^T with A (M x K) and W (N x K) NVFP4, both K-major with
// block scales in the 128-row x 4-block atom layout (NVFP4_SF_TILED).  Each
// tcgen05.mma.kind::mxf4nvf4.block_scale.block16 multiplies a 128 x 64 slice of
// A by a 256 x 64 slice of W, applying one E4M3 scale per 16 elements of both
// operands, and accumulates in fp32 in tensor memory.  ARCQuant's K -> K+S
// compensation (ARCQuant blog post, section 3.1-3.2: one GEMM over the
// augmented K) runs through this kernel unchanged.
//
// Structure (persistent, one CTA per SM, 512 threads in four warpgroups with
// a register split):
//   warps 0-3  scale warps, one per TMEM lane quadrant (80 registers): for
//              every stage, each lane reads line l of the stage's 12 scale
//              atoms from shared memory and writes them with tcgen05.st into
//              its quadrant of the stage's own TMEM scale buffer, which is
//              the layout a 32x128b.warpx4 copy of the same atoms produces
//              (the atom's 32 lines repeated in all four quadrants).  Scale
//              copies issued to the tensor pipe (tcgen05.cp) would queue
//              behind the in-flight TMA traffic; these stores do not.
//   warp 4     one lane loads each stage (56 registers): the scale atoms
//              first, on their own barrier, then the A/W code tiles (128 B
//              K-slices, 128-byte swizzle) by TMA, into a 4-stage ring;
//   warp 5     allocates 512 TMEM columns; one lane issues the 4 MMAs (K = 64
//              each) of a stage once its codes have landed and all four
//              quadrants of its scales are written; tcgen05.commit frees the
//              stage and its scale buffer and, at the end of a tile, signals
//              the epilogue;
//   warps 8-15 read the 128 x 256 fp32 accumulator into registers (184
//              each; tcgen05.ld 32x32b.x32, two warps per TMEM lane quadrant,
//              128 columns each) and release it at once, so that the next
//              tile's MMAs start while they scale by s_a s_w, transpose 32 x 8
//              chunks through shared memory and store Y with 16-byte stores,
//              two lanes per 32-byte row segment.
// Tiles are 128 x 256 x 256 (M x N x K); tile order walks M fastest so that the
// CTAs in flight share W tiles through L2.  Every mbarrier wait is bounded: on
// timeout the kernel records NVFP4_ERR_TIMEOUT, every role leaves its loop, and
// TMEM is still released.
#include "kernels.h"
#include "tcgen05.cuh"

namespace nvfp4 {
using namespace tc;
namespace {

constexpr int BM = 128, BN = 256, BK = 256;
constexpr int BK_BYTES = BK / 2;                 // one 128-byte swizzle row per k-tile
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK_BYTES;           // 16 KB
constexpr int B_BYTES = BN * BK_BYTES;           // 32 KB
constexpr int SFA_BYTES = 4 * 512;               // 4 k-atoms of one 128-row group
constexpr int SFB_BYTES = 2 * 4 * 512;           // 2 row groups x 4 k-atoms
constexpr int STAGE_BYTES = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;  // 54 KB
constexpr int OFF_B = A_BYTES, OFF_SFA = A_BYTES + B_BYTES, OFF_SFB = OFF_SFA + SFA_BYTES;
constexpr int EPI_WARPS = 8, EPI_PITCH = 9;      // per epilogue warp: a 32 x 8 fp32 chunk (+1 pad)
constexpr int EPI_BYTES = EPI_WARPS * 32 * EPI_PITCH * 4;
constexpr int BAR_BYTES = 256;
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + EPI_BYTES + BAR_BYTES + 1024;    // + alignment slack
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t ACC_COL = 0;                  // 256 fp32 columns
constexpr uint32_t SF_COL = 256, SF_BUF = 48;    // one scale buffer per stage: SFA 4 k-blocks x 4
                                                 // columns, then SFB 4 k-blocks x 8
constexpr int NUM_THREADS = 512;
// Registers: the launch gives every thread 128 (the whole register file); the
// scale and control warpgroups hand some back for the epilogue's accumulator.
constexpr int LAUNCH_REGS = 65536 / NUM_THREADS;
constexpr int SF_REGS = 80, CTL_REGS = 56, EPI_REGS = 184;
static_assert(128 * SF_REGS + 128 * CTL_REGS + 256 * EPI_REGS <= NUM_THREADS * LAUNCH_REGS, "register split");
static_assert(STAGE_BYTES % 1024 == 0, "stages must keep 1024-byte alignment for 128B swizzle");
static_assert(SMEM_BYTES <= 232448, "shared memory budget");
static_assert((4 * STAGES + 3) * 8 + 16 + 8 <= BAR_BYTES, "barrier block");
static_assert(SF_COL % 4 == 0 && SF_BUF % 4 == 0 && SF_COL + STAGES * SF_BUF <= TMEM_COLS,
              "block-scaled MMA scale operands start on 4-column TMEM boundaries");

struct TcParams {
  const uint8_t* sfa;
  const uint8_t* sfb;
  const float* a_s;
  const float* w_s;
  void* y;
  int64_t ldy;
  int y_vec;       // Y base and row pitch allow 16-byte (fp32) / 8-byte (bf16) stores
  int M, N, K;
  const uint8_t* sfr;   // residue scales (RES)
  const float* r_s;     // residue tensor scale (RES)
  int katoms;      // scale atoms along K per 128-row group: ceil(K / 64) (MX: K / 128)
  int b_groups;    // 128-row groups of W = ceil(N / 128)
  int m_blocks, n_blocks, num_tiles, k_tiles;
  int* st;
  uint64_t wait_ns;   // bound on every mbarrier wait
  int hold;           // test of the timeout path: the producer loads nothing
};

// --------------------------------------------------------------- kernel

// MX: MXFP4 operands (32-element blocks, E8M0 scales, no tensor scales): the
// same stages, with the scale atoms covering K = 128 each, so half of each
// stage's scale area and of its TMEM scale buffer is used.
// RES: ResServe's full residue (Y = s_a s_w A W^T + s_r s_w R W^T).  Each tile
// runs two passes over its K-tiles, A W^T and then R W^T (the residue as a
// second run of K-tiles over the same W tiles).  NVFP4: two uses of the TMEM
// accumulator; the epilogue holds s_a s_w acc in registers while the second
// pass runs and adds s_r s_w acc before the single store of Y.  MXFP4 has no
// tensor scales, so the residue's K-tiles simply continue the same
// accumulation: Y = [A | R] [W | W]^T.
template <bool BF16OUT, bool MX, bool RES = false>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    k_gemm_nvf4(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const __grid_constant__ CUtensorMap tmR, const TcParams p) {
  constexpr int NPASS = RES ? 2 : 1;            // passes over the K-tiles per tile
  constexpr int NUSE = (RES && !MX) ? 2 : 1;    // accumulator uses per tile
  extern __shared__ __align__(16) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* epi = reinterpret_cast<float*>(smem + STAGES * STAGE_BYTES);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES + EPI_BYTES);
  uint64_t* full = bars;               // [STAGES] code tiles landed -> MMA
  uint64_t* empty = bars + STAGES;     // [STAGES] MMAs done -> TMA (stage and its scale buffer free)
  uint64_t* sf_land = bars + 2 * STAGES;   // [STAGES] scale atoms landed -> scale warps
  uint64_t* sf_full = bars + 3 * STAGES;   // [STAGES] scales in TMEM, all four quadrants -> MMA
  uint64_t* acc_full = bars + 4 * STAGES;
  uint64_t* acc_empty = acc_full + 1;  // the epilogue holds the accumulator in registers
  uint64_t* mma_drain = acc_empty + 1; // every MMA issued has completed (before TMEM is released)
  WaitState* abort_flag = reinterpret_cast<WaitState*>(mma_drain + 1);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(abort_flag + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(saddr(&full[s]), 1);
      mbar_init(saddr(&empty[s]), 1);
      mbar_init(saddr(&sf_land[s]), 1);
      mbar_init(saddr(&sf_full[s]), 4);
    }
    mbar_init(saddr(acc_full), 1);
    mbar_init(saddr(acc_empty), EPI_WARPS);
    mbar_init(saddr(mma_drain), 1);
    abort_flag->abort = 0;
    abort_flag->limit_ns = p.wait_ns;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 5) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(saddr(tmem_slot)),
                 "r"(TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp < 4) {
    regs_dec<SF_REGS>();
    // ------------------------------------------- scale warps: quadrant `warp`, every stage
    // TMEM scale buffer s was last read by the MMAs of the step STAGES earlier,
    // which completed before this step's loads were issued.
    const uint32_t quad = (uint32_t)(warp * 32) << 16;
    int g = 0;
    bool ok = true;
    for (int tile = blockIdx.x; ok && tile < p.num_tiles; tile += gridDim.x) {
      for (int t = 0; t < NPASS * p.k_tiles; ++t, ++g) {
        const int s = g % STAGES;
        // every lane waits; the warp goes on only if all saw the phase (the
        // TMEM stores are warp-collective)
        ok = __all_sync(0xFFFFFFFFu,
                        mbar_wait_inline(saddr(&sf_land[s]), (uint32_t)((g / STAGES) & 1), abort_flag, p.st)) != 0;
        if (!ok) break;
        tc_fence_after();
        const uint8_t* st_base = smem + s * STAGE_BYTES;
        const uint32_t buf = SF_COL + (uint32_t)s * SF_BUF;
        if constexpr (MX) {
          // two atoms per operand group: SFA atoms in columns 0-7, SFB atom a of
          // group g in columns 8 + 8a + 4g
          uint32_t rm[32];
#pragma unroll
          for (int a = 0; a < 2; ++a) {
            const uint4 va = *reinterpret_cast<const uint4*>(st_base + OFF_SFA + a * 512 + lane * 16);
            const uint4 v0 = *reinterpret_cast<const uint4*>(st_base + OFF_SFB + a * 512 + lane * 16);
            const uint4 v1 = *reinterpret_cast<const uint4*>(st_base + OFF_SFB + 2048 + a * 512 + lane * 16);
            rm[4 * a] = va.x; rm[4 * a + 1] = va.y; rm[4 * a + 2] = va.z; rm[4 * a + 3] = va.w;
            rm[8 + 8 * a] = v0.x; rm[8 + 8 * a + 1] = v0.y; rm[8 + 8 * a + 2] = v0.z; rm[8 + 8 * a + 3] = v0.w;
            rm[12 + 8 * a] = v1.x; rm[12 + 8 * a + 1] = v1.y; rm[12 + 8 * a + 2] = v1.z; rm[12 + 8 * a + 3] = v1.w;
          }
#pragma unroll
          for (int i = 24; i < 32; ++i) rm[i] = 0u;
          tmem_st32(tmem + quad + buf, rm);
        } else {
          uint32_t ra[16], rb[32];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint4 va = *reinterpret_cast<const uint4*>(st_base + OFF_SFA + j * 512 + lane * 16);
            const uint4 v0 = *reinterpret_cast<const uint4*>(st_base + OFF_SFB + j * 512 + lane * 16);
            const uint4 v1 = *reinterpret_cast<const uint4*>(st_base + OFF_SFB + 2048 + j * 512 + lane * 16);
            ra[4 * j] = va.x; ra[4 * j + 1] = va.y; ra[4 * j + 2] = va.z; ra[4 * j + 3] = va.w;
            rb[8 * j] = v0.x; rb[8 * j + 1] = v0.y; rb[8 * j + 2] = v0.z; rb[8 * j + 3] = v0.w;
            rb[8 * j + 4] = v1.x; rb[8 * j + 5] = v1.y; rb[8 * j + 6] = v1.z; rb[8 * j + 7] = v1.w;
          }
          tmem_st16(tmem + quad + buf, ra);
          tmem_st32(tmem + quad + buf + 16u, rb);
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(saddr(&sf_full[s]));
      }
    }
  } else if (warp < 8) {
    regs_dec<CTL_REGS>();
    if (warp == 4 && lane == 0) {
      // ------------------------------------------------------ TMA producer
      // the small scale atoms first, on their own barrier: their trip to TMEM
      // overlaps the code tiles' flight
      int g = 0;
      if (p.hold) goto producer_done;
      for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x) {
        const int mb = tile % p.m_blocks, nb = tile / p.m_blocks;
        const int ngroups = min(2, p.b_groups - nb * 2);
        for (int t = 0; t < NPASS * p.k_tiles; ++t, ++g) {
          const int pass = t >= p.k_tiles ? 1 : 0, kt = t - pass * p.k_tiles;
          const uint8_t* sfa = (RES && pass) ? p.sfr : p.sfa;            // A, then R
          const CUtensorMap* tma = (RES && pass) ? &tmR : &tmA;
          const int s = g % STAGES;
          if (!mbar_wait_inline(saddr(&empty[s]), (uint32_t)((g / STAGES) & 1) ^ 1u, abort_flag, p.st)) goto producer_done;
          const int jmax = min(4, (p.K - kt * BK) / 64);
          const int atoms = MX ? (jmax + 1) / 2 : jmax, apt = MX ? 2 : 4;   // atoms of this / a full k-tile
          const uint32_t sf_bytes = (uint32_t)atoms * 512u;
          uint8_t* st_base = smem + s * STAGE_BYTES;
          const uint32_t sbar = saddr(&sf_land[s]);
          mbar_expect_tx(sbar, sf_bytes * (1 + ngroups));
          bulk_load(saddr(st_base + OFF_SFA), sfa + ((size_t)mb * p.katoms + kt * apt) * 512, sf_bytes, sbar);
          for (int gi = 0; gi < ngroups; ++gi)
            bulk_load(saddr(st_base + OFF_SFB + gi * 2048),
                      p.sfb + ((size_t)(nb * 2 + gi) * p.katoms + kt * apt) * 512, sf_bytes, sbar);
          const uint32_t bar = saddr(&full[s]);
          mbar_expect_tx(bar, A_BYTES + B_BYTES);
          tma_load_2d(saddr(st_base), tma, kt * BK_BYTES, mb * BM, bar);
          tma_load_2d(saddr(st_base + OFF_B), &tmB, kt * BK_BYTES, nb * BN, bar);
        }
      }
    producer_done:
      // the last STAGES stages' copies may still be in flight if a consumer gave
      // up: let them land before the CTA can exit
      for (int g2 = max(0, g - STAGES); g2 < g; ++g2) {
        const uint32_t ph = (uint32_t)((g2 / STAGES) & 1);
        (void)mbar_drain(saddr(&sf_land[g2 % STAGES]), ph, abort_flag, p.st);
        (void)mbar_drain(saddr(&full[g2 % STAGES]), ph, abort_flag, p.st);
      }
    } else if (warp == 5 && lane == 0) {
      // -------------------------------------------------------- MMA issuer
      const uint32_t idesc = idesc_nvf4(BN);
      int g = 0, local = 0;
      for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x, ++local)
      for (int pass = 0; pass < NPASS; ++pass) {
        // accumulator use u: the epilogue has taken use u - 1 out of TMEM
        const bool fresh = NUSE == 2 || pass == 0;   // this pass starts a use of the accumulator
        const int u = NUSE * local + (NUSE == 2 ? pass : 0);
        if (fresh) {
          if (!mbar_wait_inline(saddr(acc_empty), (uint32_t)(u & 1) ^ 1u, abort_flag, p.st)) goto mma_done;
          tc_fence_after();
        }
        for (int kt = 0; kt < p.k_tiles; ++kt, ++g) {
          const int s = g % STAGES;
          const uint32_t ph = (uint32_t)((g / STAGES) & 1);
          if (!mbar_wait_inline(saddr(&sf_full[s]), ph, abort_flag, p.st)) goto mma_done;
          if (!mbar_wait_inline(saddr(&full[s]), ph, abort_flag, p.st)) goto mma_done;
          tc_fence_after();
          const int jmax = min(4, (p.K - kt * BK) / 64);
          const uint8_t* st_base = smem + s * STAGE_BYTES;
          const uint64_t da = desc_sw128(saddr(st_base)), db = desc_sw128(saddr(st_base + OFF_B));
          const uint32_t buf = SF_COL + (uint32_t)s * SF_BUF;
          for (int j = 0; j < jmax; ++j) {
            if constexpr (MX)   // K = 64 chunk j: atom j / 2, scale bytes 2 (j % 2) and 2 (j % 2) + 1
              tc_mma_mxf4(tmem + ACC_COL, da + (uint64_t)(2 * j), db + (uint64_t)(2 * j),
                          idesc_mxf4(BN, 2u * (uint32_t)(j & 1)), tmem + buf + 4 * (j >> 1),
                          tmem + buf + 8 + 8 * (j >> 1), (!fresh || kt > 0 || j > 0) ? 1u : 0u);
            else
              tc_mma_nvf4(tmem + ACC_COL, da + (uint64_t)(2 * j), db + (uint64_t)(2 * j), idesc, tmem + buf + 4 * j,
                          tmem + buf + 16 + 8 * j, (!fresh || kt > 0 || j > 0) ? 1u : 0u);
          }
          tc_commit(saddr(&empty[s]));
        }
        if (NUSE == 2 || pass == NPASS - 1) tc_commit(saddr(acc_full));
      }
    mma_done:
      // every MMA issued has completed before TMEM can be released
      tc_commit(saddr(mma_drain));
      (void)mbar_drain(saddr(mma_drain), 0u, abort_flag, p.st);
    }
  } else {
    regs_inc<EPI_REGS>();
    // ----------------------------------------------------------- epilogue
    const int q = warp & 3;  // TMEM lane quadrant this warp may access
    const int ew = warp - 8, half = ew / 4;
    float* buf = epi + ew * 32 * EPI_PITCH;
    const int sub_r = lane >> 1, sub_c = (lane & 1) * 4;
    int local = 0;
    const float alpha = MX ? 1.0f : (*p.a_s) * (*p.w_s);   // MXFP4 has no tensor scales
    const float alpha_r = NUSE == 2 ? (*p.r_s) * (*p.w_s) : 0.0f;
    const float out_scale = NUSE == 2 ? 1.0f : alpha;        // two uses: the registers hold the combined Y
    for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x, ++local) {
      const int mb = tile % p.m_blocks, nb = tile / p.m_blocks;
      if (!mbar_wait_inline(saddr(acc_full), (uint32_t)((NUSE * local) & 1), abort_flag, p.st)) break;
      tc_fence_after();
      // Each warp owns TMEM lanes (= tile rows) 32q..32q+31 and columns
      // [128 half, 128 half + 128): read them all, then free the accumulator.
      uint32_t r[BN / 64][32];
#pragma unroll
      for (int c = 0; c < BN / 64; ++c)
        tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + ACC_COL + (half * (BN / 64) + c) * 32, r[c]);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(saddr(acc_empty));
      if constexpr (NUSE == 2) {
        // s_a s_w acc1 stays in registers; add s_r s_w acc2 column chunk by column chunk
#pragma unroll
        for (int c = 0; c < BN / 64; ++c)
#pragma unroll
          for (int i = 0; i < 32; ++i) r[c][i] = __float_as_uint(__uint_as_float(r[c][i]) * alpha);
        if (!mbar_wait_inline(saddr(acc_full), (uint32_t)((NUSE * local + 1) & 1), abort_flag, p.st)) break;
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < BN / 64; ++c) {
          uint32_t t[32];
          tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + ACC_COL + (half * (BN / 64) + c) * 32, t);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i)
            r[c][i] = __float_as_uint(fmaf(alpha_r, __uint_as_float(t[i]), __uint_as_float(r[c][i])));
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(saddr(acc_empty));
      }
      // 32 x 8 chunks: lane = row while writing, then 2 lanes per 8-column row
      // segment, 16 rows per store instruction
#pragma unroll
      for (int c = 0; c < BN / 64; ++c) {
        const int col0 = nb * BN + (half * (BN / 64) + c) * 32;
        if (col0 >= p.N) continue;  // uniform across the warp
#pragma unroll
        for (int g8 = 0; g8 < 4; ++g8) {
#pragma unroll
          for (int i = 0; i < 8; ++i) buf[lane * EPI_PITCH + i] = __uint_as_float(r[c][g8 * 8 + i]) * out_scale;
          __syncwarp();
          const int cg = col0 + g8 * 8;
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int lr = h * 16 + sub_r;
            const int grow = mb * BM + q * 32 + lr;
            const float* src = buf + lr * EPI_PITCH + sub_c;
            const int64_t off = (int64_t)grow * p.ldy + cg + sub_c;
            if (grow < p.M) {
              if (p.y_vec && cg + 8 <= p.N) {
                if (BF16OUT)
                  *reinterpret_cast<uint2*>(reinterpret_cast<__nv_bfloat16*>(p.y) + off) =
                      make_uint2(pack_bf16x2(src[0], src[1]), pack_bf16x2(src[2], src[3]));
                else
                  *reinterpret_cast<float4*>(reinterpret_cast<float*>(p.y) + off) =
                      make_float4(src[0], src[1], src[2], src[3]);
              } else {
                // ragged last chunk or unaligned Y: element stores
                for (int e = 0; e < 4 && cg + sub_c + e < p.N; ++e) {
                  if (BF16OUT)
                    reinterpret_cast<__nv_bfloat16*>(p.y)[off + e] = __float2bfloat16_rn(src[e]);
                  else
                    reinterpret_cast<float*>(p.y)[off + e] = src[e];
                }
              }
            }
          }
          __syncwarp();
        }
      }
    }
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS) : "memory");
  }
}

}  // namespace

namespace tc {

// The driver's tensor-map encoder, resolved at run time through the runtime API
// so that the library does not link against libcuda.
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

bool encode_codes_map(CUtensorMap* map, const uint8_t* codes, int64_t rows, int64_t K, uint32_t box_rows) {
  PFN_cuTensorMapEncodeTiled_v12000 encode = tensor_map_encoder();
  if (encode == nullptr) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)(K / 2), (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)(K / 2)};
  const cuuint32_t box[2] = {(cuuint32_t)128, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(codes), dims,
                                strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                                CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace tc

template <bool MX>
cudaError_t launch_gemm_impl(const GemmArgs& g, int num_sms, cudaStream_t stream) {
  const bool res = g.r_codes != nullptr;   // ResServe residue: a second pass over the K-tiles
  if (MX ? (g.K % 128 != 0 || g.K < BK) : (g.K % 64 != 0 || g.K < BK)) return cudaErrorNotSupported;
  // sizes, tile coordinates and the tile count are 32-bit in the kernel
  if (g.M > INT32_MAX || g.N > INT32_MAX || g.K > INT32_MAX ||
      ((g.M + BM - 1) / BM) * ((g.N + BN - 1) / BN) > INT32_MAX)
    return cudaErrorNotSupported;
  CUtensorMap tmA, tmB, tmR;
  if (!encode_codes_map(&tmA, g.a_codes, g.M, g.K, BM) || !encode_codes_map(&tmB, g.w_codes, g.N, g.K, BN))
    return cudaErrorInvalidValue;
  if (res ? !encode_codes_map(&tmR, g.r_codes, g.M, g.K, BM) : false) return cudaErrorInvalidValue;
  if (!res) tmR = tmA;   // unused
  TcParams p{};
  p.sfa = g.a_scales; p.sfb = g.w_scales; p.a_s = g.a_s; p.w_s = g.w_s;
  p.sfr = g.r_scales; p.r_s = g.r_s;
  p.y = g.y; p.ldy = g.ldy;
  {
    const size_t vec_bytes = g.y_bf16 ? 8 : 16, esize = g.y_bf16 ? 2 : 4;
    p.y_vec = (reinterpret_cast<uintptr_t>(g.y) % vec_bytes == 0) && ((size_t)g.ldy * esize) % vec_bytes == 0;
  }
  p.M = (int)g.M; p.N = (int)g.N; p.K = (int)g.K;
  p.katoms = MX ? (int)(g.K / 128) : (int)((g.K + 63) / 64);
  p.b_groups = (int)((g.N + 127) / 128);
  p.m_blocks = (int)((g.M + BM - 1) / BM);
  p.n_blocks = (int)((g.N + BN - 1) / BN);
  p.num_tiles = p.m_blocks * p.n_blocks;
  p.k_tiles = (int)((g.K + BK - 1) / BK);
  p.st = g.st;
  const WaitTest wt = wait_test();
  p.wait_ns = wt.limit_ns;
  p.hold = wt.hold;
  auto kern = res ? (g.y_bf16 ? k_gemm_nvf4<true, MX, true> : k_gemm_nvf4<false, MX, true>)
                  : (g.y_bf16 ? k_gemm_nvf4<true, MX> : k_gemm_nvf4<false, MX>);
  // the register split assumes the launch allocates LAUNCH_REGS per thread
  cudaFuncAttributes fa{};
  if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess || fa.numRegs != LAUNCH_REGS) return cudaErrorNotSupported;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
  if (e != cudaSuccess) return e;
  const int grid = std::max(1, std::min(p.num_tiles, num_sms));
  kern<<<grid, NUM_THREADS, SMEM_BYTES, stream>>>(tmA, tmB, tmR, p);
  return cudaGetLastError();
}

cudaError_t launch_gemm_tc(const GemmArgs& g, int num_sms, cudaStream_t stream) {
  return launch_gemm_impl<false>(g, num_sms, stream);
}

cudaError_t launch_gemm_mx(const GemmArgs& g, int num_sms, cudaStream_t stream) {
  return launch_gemm_impl<true>(g, num_sms, stream);
}

}  // namespace nvfp4
