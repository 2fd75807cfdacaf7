// Few-row NVFP4 linear (M <= 128) on the tensor cores with the operands
// swapped, sm_100a.
//
// Y^T = W X^T: W (N x K) is the 128-row A operand of
// tcgen05.mma.kind::mxf4nvf4.block_scale.block16, the M activation rows (padded
// to NP = 16/32/64/128) are the B operand, so a decode step costs one pass over
// W at HBM speed instead of being limited by CUDA-core multiply rates.  With a
// residue operand R (ResServe abstract: FP4 base plus FP4 residue, combined
// on-chip) the same W tile feeds a second accumulator, and both are combined in
// the epilogue with their own tensor scales: Y = s_x s_w acc + s_r s_w acc_r.
//
// Grid: (ks, ceil(N/128)); the ks CTAs of one cluster split K between them and
// each accumulates a 128 x NP fp32 partial in TMEM.  Row r of the tile is owned
// by cluster rank floor(r*ks/128); every CTA pushes its partial rows straight
// into the owner's shared memory (distributed shared-memory stores), and after
// one cluster barrier each owner sums its rows and writes Y.  Roles inside a
// CTA (256 threads): warp 0 lane 0 issues TMA/bulk copies into a shared-memory
// ring; warps 4-7 (one per TMEM lane quadrant) write each k-tile's scale atoms
// into one of two alternating TMEM scale buffers with tcgen05.st; warp 1 lane 0
// issues the MMAs; then warps 0-3 drain the accumulators.
//
// Programmatic dependent launch: the kernel may start while the preceding
// kernel on the stream (normally the activation quantizer) is still running.
// Before griddepcontrol.wait it only sets up (barriers, TMEM) and asks L2 to
// prefetch this CTA's W tiles and scale atoms; L2 is the point of coherence,
// so a prefetch never yields stale data even if the preceding kernel writes W.
// Every load that feeds the result is issued after the wait.
//
// Safety: every mbarrier wait is bounded; every CTA reaches every cluster
// barrier on every path; the dynamic shared-memory request covers the whole
// layout and caps the CTAs per SM so that their TMEM allocations always fit
// side by side (no CTA can block in tcgen05.alloc behind a cluster peer).
#include "kernels.h"
#include "tcgen05.cuh"

namespace nvfp4 {
using namespace tc;
namespace {

constexpr int kThreads = 256;   // warps 0-3: roles and the drain; warps 4-7: scales into TMEM
constexpr int W_TILE = 128 * 128;   // 128 rows of W x 128 bytes (256 K-elements)
constexpr int SF4 = 4 * 512;         // 4 scale atoms: one 128-row group x 256 K

template <int NP, bool RES>
struct Cfg {
  static constexpr int X_TILE = NP * 128;
  static constexpr int OFF_X = W_TILE;
  static constexpr int OFF_R = OFF_X + X_TILE;
  static constexpr int OFF_SFW = OFF_R + (RES ? X_TILE : 0);
  static constexpr int OFF_SFX = OFF_SFW + SF4;
  static constexpr int OFF_SFR = OFF_SFX + SF4;
  static constexpr int STAGE = ((OFF_SFR + (RES ? SF4 : 0)) + 1023) / 1024 * 1024;
  // TMEM: acc [0,NP), acc_r [NP,2NP), then two scale buffers (alternating by
  // k-tile) of W, X (and R) scales, 16 columns each
  static constexpr uint32_t ACC = 0, ACC_R = NP;
  static constexpr uint32_t SF_COL = (RES ? 2 : 1) * NP, SF_BUF = RES ? 48 : 32;
  static constexpr uint32_t COLS_USED = SF_COL + 2 * SF_BUF;
  static constexpr uint32_t TMEM_COLS = COLS_USED <= 128 ? 128 : (COLS_USED <= 256 ? 256 : 512);
  static constexpr int TMEM_CTAS = 512 / TMEM_COLS;               // CTAs whose TMEM fits on one SM
  static constexpr int BAR = 256;
  // stages: as many as keep two CTAs per SM (the request plus the 1 KB the
  // runtime reserves per CTA must fit twice in the SM's 228 KB; four stages
  // when TMEM allows only one CTA)
  static constexpr int BUDGET = TMEM_CTAS >= 2 ? 233472 / 2 - 1024 : 224 * 1024;
  // pushed partial rows: every source rank has a slot of ceil(128/ks) rows in
  // its owner, ks * ceil(128/ks) <= 135 rows for ks <= 8
  static constexpr int PITCH = NP + 4;                            // floats per partial row (padded)
  static constexpr int PART_ROWS = 136;
  static constexpr int PART = PART_ROWS * PITCH * 4 * (RES ? 2 : 1);
  // a dedicated partial area (peers may push as soon as this CTA has started)
  // when it still leaves three stages; otherwise it overlays the stage ring
  static constexpr bool PART_OWN = PART <= 40 * 1024 && 3 * STAGE + PART + BAR + 1024 <= BUDGET;
  static constexpr int PART_DED = PART_OWN ? PART : 0;
  static constexpr int STAGES = (4 * STAGE + PART_DED + BAR + 1024 <= BUDGET)
                                    ? 4
                                    : ((3 * STAGE + PART_DED + BAR + 1024 <= BUDGET) ? 3 : 2);
  // layout from the 1024-aligned base: ring | dedicated partials | barriers;
  // +1024 covers the alignment of the dynamic shared-memory base
  static constexpr int SMEM_NEED = STAGES * STAGE + PART_DED + BAR + 1024;
  // request that keeps at most TMEM_CTAS CTAs on an SM, so tcgen05.alloc never waits on a peer
  static constexpr int SMEM_MIN = 233472 / (TMEM_CTAS + 1) + 1024;
  static constexpr int SMEM = SMEM_NEED > SMEM_MIN ? SMEM_NEED : SMEM_MIN;
  static constexpr int CTAS_PER_SM = (233472 / (SMEM + 1024)) < TMEM_CTAS ? (233472 / (SMEM + 1024)) : TMEM_CTAS;
  static_assert(1023 + STAGES * STAGE + PART_DED + BAR <= SMEM, "layout exceeds the shared-memory request");
  static_assert((2 * STAGES + 3) * 8 + 16 + 8 <= BAR, "barrier block");
  static_assert(SF_COL % 4 == 0 && SF_BUF % 4 == 0, "block-scaled MMA scale operands start on 4-column TMEM boundaries");
  static_assert(SMEM <= 232448, "shared memory budget");
  static_assert(PART_OWN || PART <= STAGES * STAGE, "partials overlay the stage ring");
  static_assert(233472 / (SMEM + 1024) <= TMEM_CTAS, "TMEM must fit every co-resident CTA");
  static_assert(CTAS_PER_SM >= 1, "residency");
};

struct SwapParams {
  const uint8_t* sfw;    // W scales, TILED
  const uint8_t* sfx;    // X scales, TILED (row group 0)
  const uint8_t* sfr;    // R scales, TILED (row group 0) or null
  const float* x_s;
  const float* w_s;
  const float* r_s;
  void* y;
  int64_t ldy;
  int M, N, K;
  int katoms_w, k_tiles;
  int* st;
  uint64_t wait_ns;   // bound on every mbarrier wait
  int hold;           // test of the timeout path: the producer loads nothing
  int prefetch;       // prefetch W into L2 before the dependency wait
};

template <int NP, bool RES, bool BF16OUT>
__global__ void __launch_bounds__(kThreads, 1)
    k_gemv_tc(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
              const __grid_constant__ CUtensorMap tmR, const SwapParams p) {
  using C = Cfg<NP, RES>;
  extern __shared__ __align__(16) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* part = reinterpret_cast<float*>(C::PART_OWN ? smem + C::STAGES * C::STAGE : smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::STAGES * C::STAGE + C::PART_DED);
  uint64_t* full = bars;
  uint64_t* empty = bars + C::STAGES;
  uint64_t* acc_full = bars + 2 * C::STAGES;
  uint64_t* sf_full = acc_full + 1;   // [2] a scale buffer written by all four quadrants
  WaitState* abort_flag = reinterpret_cast<WaitState*>(sf_full + 2);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(abort_flag + 1);

  griddep_launch_dependents();   // the next kernel may set itself up; it waits for this one's results

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank(), ks = cluster_nctarank();
  const int rt = blockIdx.y;                                       // 128-row tile of W
  const int kt0 = (int)((rank * (uint32_t)p.k_tiles) / ks);
  const int kt1 = (int)(((rank + 1) * (uint32_t)p.k_tiles) / ks);

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(saddr(&full[s]), 1);
      mbar_init(saddr(&empty[s]), 1);
    }
    mbar_init(saddr(acc_full), 1);
    mbar_init(saddr(&sf_full[0]), 4);
    mbar_init(saddr(&sf_full[1]), 4);
    abort_flag->abort = 0;
    abort_flag->limit_ns = p.wait_ns;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(saddr(tmem_slot)),
                 "r"(C::TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  // with a dedicated partial area, peers may push into it once they know this
  // CTA is running: announce it now, they wait for it before their first push
  if (C::PART_OWN) cluster_arrive_relaxed();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (p.prefetch && warp == 0 && lane == 0) {
    // warm L2 with this CTA's W tiles and scale atoms while the preceding kernel finishes
    for (int kt = kt0; kt < kt1; ++kt) {
      prefetch_l2_tile_2d(&tmW, kt * 128, rt * 128);
      prefetch_l2_bulk(p.sfw + ((size_t)rt * p.katoms_w + kt * 4) * 512,
                       (uint32_t)min(4, (p.K - kt * 256) / 64) * 512u);
    }
  }
  griddep_wait();   // X, R, the scales and the tensor scales come from the preceding kernel

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------- TMA producer
    int s = 0, issued = 0;
    uint32_t ph = 0;
    for (int kt = kt0; !p.hold && kt < kt1; ++kt, ++issued) {
      if (!mbar_wait(saddr(&empty[s]), ph ^ 1u, abort_flag, p.st)) break;
      const int jmax = min(4, (p.K - kt * 256) / 64);
      const uint32_t sf = (uint32_t)jmax * 512u;
      const uint32_t bar = saddr(&full[s]);
      uint8_t* sb = smem + s * C::STAGE;
      mbar_expect_tx(bar, W_TILE + C::X_TILE * (RES ? 2 : 1) + sf * (RES ? 3 : 2));
      tma_load_2d(saddr(sb), &tmW, kt * 128, rt * 128, bar);
      tma_load_2d(saddr(sb + C::OFF_X), &tmX, kt * 128, 0, bar);
      if (RES) tma_load_2d(saddr(sb + C::OFF_R), &tmR, kt * 128, 0, bar);
      bulk_load(saddr(sb + C::OFF_SFW), p.sfw + ((size_t)rt * p.katoms_w + kt * 4) * 512, sf, bar);
      bulk_load(saddr(sb + C::OFF_SFX), p.sfx + (size_t)kt * 4 * 512, sf, bar);
      if (RES) bulk_load(saddr(sb + C::OFF_SFR), p.sfr + (size_t)kt * 4 * 512, sf, bar);
      if (++s == C::STAGES) { s = 0; ph ^= 1u; }
    }
    // the last STAGES stages' copies may still be in flight if a consumer gave
    // up: let them land before the CTA can exit
    for (int g2 = max(0, issued - C::STAGES); g2 < issued; ++g2)
      (void)mbar_drain(saddr(&full[g2 % C::STAGES]), (uint32_t)((g2 / C::STAGES) & 1), abort_flag, p.st);
  } else if (warp >= 4) {
    // ------------------------------------------- scales into TMEM (tcgen05.st)
    // Warp w writes TMEM lane quadrant w - 4 of scale buffer g & 1 for the
    // CTA's g-th k-tile: line l of each W, X (and R) atom in every lane l of
    // the quadrant (the layout of a 32x128b.warpx4 copy of the atoms).  Scale
    // copies issued to the tensor pipe would queue behind the TMA stream;
    // these stores do not.  The buffer is reused once the MMAs of k-tile g-2
    // have completed.
    const uint32_t quad = (uint32_t)((warp - 4) * 32) << 16;
    for (int kt = kt0; kt < kt1; ++kt) {
      const int g = kt - kt0, s = g % C::STAGES;
      if (g >= 2) {
        const int g2 = g - 2;
        if (!__all_sync(0xFFFFFFFFu, mbar_wait(saddr(&empty[g2 % C::STAGES]), (uint32_t)((g2 / C::STAGES) & 1),
                                               abort_flag, p.st)))
          break;
      }
      if (!__all_sync(0xFFFFFFFFu, mbar_wait(saddr(&full[s]), (uint32_t)((g / C::STAGES) & 1), abort_flag, p.st)))
        break;
      tc_fence_after();
      const uint8_t* sb = smem + s * C::STAGE;
      const uint32_t buf = C::SF_COL + (uint32_t)(g & 1) * C::SF_BUF;
      uint32_t r[32];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint4 w = *reinterpret_cast<const uint4*>(sb + C::OFF_SFW + j * 512 + lane * 16);
        const uint4 x = *reinterpret_cast<const uint4*>(sb + C::OFF_SFX + j * 512 + lane * 16);
        r[4 * j] = w.x; r[4 * j + 1] = w.y; r[4 * j + 2] = w.z; r[4 * j + 3] = w.w;
        r[16 + 4 * j] = x.x; r[16 + 4 * j + 1] = x.y; r[16 + 4 * j + 2] = x.z; r[16 + 4 * j + 3] = x.w;
      }
      tmem_st32(tmem + quad + buf, r);   // W scales, then X scales
      if constexpr (RES) {
        uint32_t rr[16];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint4 v = *reinterpret_cast<const uint4*>(sb + C::OFF_SFR + j * 512 + lane * 16);
          rr[4 * j] = v.x; rr[4 * j + 1] = v.y; rr[4 * j + 2] = v.z; rr[4 * j + 3] = v.w;
        }
        tmem_st16(tmem + quad + buf + 32u, rr);
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(saddr(&sf_full[g & 1]));
    }
  } else if (warp == 1 && lane == 0) {
    // --------------------------------------------------------- MMA issuer
    const uint32_t idesc = idesc_nvf4(NP);
    int s = 0;
    uint32_t ph = 0;
    for (int kt = kt0; kt < kt1; ++kt) {
      const int g = kt - kt0;
      if (!mbar_wait(saddr(&full[s]), ph, abort_flag, p.st)) break;
      if (!mbar_wait(saddr(&sf_full[g & 1]), (uint32_t)((g >> 1) & 1), abort_flag, p.st)) break;
      tc_fence_after();
      const int jmax = min(4, (p.K - kt * 256) / 64);
      const uint8_t* sb = smem + s * C::STAGE;
      const uint32_t buf = C::SF_COL + (uint32_t)(g & 1) * C::SF_BUF;
      const uint64_t dw = desc_sw128(saddr(sb)), dx = desc_sw128(saddr(sb + C::OFF_X));
      const uint64_t dr = desc_sw128(saddr(sb + C::OFF_R));
      for (int j = 0; j < jmax; ++j) {
        const uint32_t acc = (kt > kt0 || j > 0) ? 1u : 0u;
        tc_mma_nvf4(tmem + C::ACC, dw + (uint64_t)(2 * j), dx + (uint64_t)(2 * j), idesc, tmem + buf + 4 * j,
                    tmem + buf + 16 + 4 * j, acc);
        if (RES)
          tc_mma_nvf4(tmem + C::ACC_R, dw + (uint64_t)(2 * j), dr + (uint64_t)(2 * j), idesc, tmem + buf + 4 * j,
                      tmem + buf + 32 + 4 * j, acc);
      }
      // waited for only when the stage is refilled (g + STAGES < nkt) or the
      // scale buffer reused (g + 2 < nkt): both are g + 2 < nkt with STAGES >= 2,
      // and a commit costs tensor-pipe time (acc_full covers the last two)
      if (kt + 2 < kt1) tc_commit(saddr(&empty[s]));
      if (++s == C::STAGES) { s = 0; ph ^= 1u; }
    }
    tc_commit(saddr(acc_full));
  }
  __syncwarp();

  // ------------------- push this CTA's partial rows to the CTA that owns them
  // Owner o = floor(r*ks/128) holds rows [ceil(o*128/ks), ceil((o+1)*128/ks))
  // of the tile, at most ceil(128/ks) rows, and keeps one slot of that many
  // rows per source rank.
  // the commit after the MMA loop is issued on every path: waiting for it also
  // waits for every MMA in flight, before TMEM is read and released
  const bool ok = mbar_drain(saddr(acc_full), 0u, abort_flag, p.st) && !wait_aborted(abort_flag);
  tc_fence_after();
  __syncwarp();     // the cluster barriers below are warp-aligned
  if (!C::PART_OWN) {
    // the partials overlay the ring: a peer's ring is free once its MMAs are done
    tc_fence_before();
    cluster_arrive();
  }
  cluster_wait();   // dedicated area: pairs with the arrive at start-up
  tc_fence_after();
  const int rows_max = (int)((128u + ks - 1) / ks);
  auto owner_row0 = [&](uint32_t o) { return (int)((o * 128u + ks - 1) / ks); };
  if (warp < 4) {
    const int row = warp * 32 + lane;                              // TMEM lane = W row of the tile
    const uint32_t o = (uint32_t)row * ks / 128u;
    const int slot = (int)rank * rows_max + (row - owner_row0(o));
    const uint32_t dst = mapa_shared(saddr(part + slot * C::PITCH), o);
    const uint32_t lane_addr = tmem + ((uint32_t)(warp * 32) << 16);
#pragma unroll
    for (int acc_i = 0; acc_i < (RES ? 2 : 1); ++acc_i) {
      const uint32_t dsti = dst + (uint32_t)(acc_i * C::PART_ROWS * C::PITCH * 4);
      const uint32_t src = lane_addr + (acc_i ? C::ACC_R : C::ACC);
#pragma unroll
      for (int c = 0; c < NP; c += 16) {
        uint32_t r[16];
        tmem_ld16(src + c, r);
        tmem_ld_wait();
        if (!ok) {
#pragma unroll
          for (int i = 0; i < 16; ++i) r[i] = 0u;
        }
#pragma unroll
        for (int i = 0; i < 16; i += 4)
          st_cluster_f32x4(dsti + (uint32_t)((c + i) * 4), __uint_as_float(r[i]), __uint_as_float(r[i + 1]),
                           __uint_as_float(r[i + 2]), __uint_as_float(r[i + 3]));
      }
    }
  }
  tc_fence_before();
  cluster_sync();   // every partial has landed in its owner's shared memory

  // ------------------------------------------------ owners sum their rows and store
  {
    const int r0 = owner_row0(rank), r1 = owner_row0(rank + 1);
    const int nrows = r1 - r0;
    const float alpha = (*p.x_s) * (*p.w_s);
    const float alpha_r = RES ? (*p.r_s) * (*p.w_s) : 0.0f;
    for (int idx = threadIdx.x; idx < nrows * p.M; idx += kThreads) {
      const int m = idx / nrows, i = idx - m * nrows;
      const int n = rt * 128 + r0 + i;
      if (n >= p.N) continue;
      float sum = 0.0f, sum_r = 0.0f;
      for (uint32_t src = 0; src < ks; ++src) {
        const int slot = (int)src * rows_max + i;
        sum += part[slot * C::PITCH + m];
        if (RES) sum_r += part[C::PART_ROWS * C::PITCH + slot * C::PITCH + m];
      }
      const float out = RES ? fmaf(sum, alpha, sum_r * alpha_r) : sum * alpha;
      if (BF16OUT)
        reinterpret_cast<__nv_bfloat16*>(p.y)[(int64_t)m * p.ldy + n] = __float2bfloat16_rn(out);
      else
        reinterpret_cast<float*>(p.y)[(int64_t)m * p.ldy + n] = out;
    }
  }

  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(C::TMEM_COLS)
                 : "memory");
  }
}

template <int NP, bool RES, bool BF16OUT>
cudaError_t launch_np(const GemmArgs& g, int num_sms, cudaStream_t stream) {
  using C = Cfg<NP, RES>;
  CUtensorMap tmW, tmX, tmR;
  if (!encode_codes_map(&tmW, g.w_codes, g.N, g.K, 128) || !encode_codes_map(&tmX, g.a_codes, g.M, g.K, NP))
    return cudaErrorInvalidValue;
  if (RES) {
    if (!encode_codes_map(&tmR, g.r_codes, g.M, g.K, NP)) return cudaErrorInvalidValue;
  } else {
    tmR = tmX;
  }
  SwapParams p{};
  p.sfw = g.w_scales; p.sfx = g.a_scales; p.sfr = g.r_scales;
  p.x_s = g.a_s; p.w_s = g.w_s; p.r_s = RES ? g.r_s : g.a_s;
  p.y = g.y; p.ldy = g.ldy;
  p.M = (int)g.M; p.N = (int)g.N; p.K = (int)g.K;
  p.katoms_w = (int)((g.K + 63) / 64);
  p.k_tiles = (int)((g.K + 255) / 256);
  p.st = g.st;
  const WaitTest wt = wait_test();
  p.wait_ns = wt.limit_ns;
  p.hold = wt.hold;
  p.prefetch = prefetch_w(g.N, g.K) ? 1 : 0;
  const int row_tiles = (int)((g.N + 127) / 128);
  auto kern = k_gemv_tc<NP, RES, BF16OUT>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = C::SMEM;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;   // overlap the preceding kernel's tail
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  // The largest K split whose clusters all fit at once (one wave).  A cluster
  // must fit inside one GPC, so count only the slots that whole clusters of c
  // CTAs fill in GPCs of 16 SMs (the smaller GPCs), not CTAs per SM x SMs.
  constexpr int kGpcSms = 16;
  const int per_gpc = kGpcSms * C::CTAS_PER_SM;
  int ks = 1;
  for (int c = std::min(8, p.k_tiles); c > 1; --c) {
    const int64_t slots = (int64_t)C::CTAS_PER_SM * num_sms * ((per_gpc / c) * c) / per_gpc;
    if ((int64_t)c * row_tiles <= slots) {
      ks = c;
      break;
    }
  }
  attr[0].val.clusterDim.x = (unsigned)ks;
  cfg.gridDim = dim3((unsigned)ks, (unsigned)row_tiles, 1);
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kern, tmW, tmX, tmR, p);
}

template <int NP>
cudaError_t launch_res(const GemmArgs& g, int num_sms, cudaStream_t stream) {
  if (g.r_codes != nullptr)
    return g.y_bf16 ? launch_np<NP, true, true>(g, num_sms, stream) : launch_np<NP, true, false>(g, num_sms, stream);
  return g.y_bf16 ? launch_np<NP, false, true>(g, num_sms, stream) : launch_np<NP, false, false>(g, num_sms, stream);
}

}  // namespace

cudaError_t launch_gemv_tc(const GemmArgs& g, int num_sms, cudaStream_t stream) {
  if (g.K % 64 != 0 || g.K < 256 || g.M > 128) return cudaErrorNotSupported;
  if (g.M <= 16) return launch_res<16>(g, num_sms, stream);
  if (g.M <= 32) return launch_res<32>(g, num_sms, stream);
  if (g.M <= 64) return launch_res<64>(g, num_sms, stream);
  return launch_res<128>(g, num_sms, stream);
}

}  // namespace nvfp4
