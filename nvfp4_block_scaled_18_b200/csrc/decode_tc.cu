// Decode-sized NVFP4 linear (M <= 16 activation rows) on the tensor cores,
// optionally fused with the online quantization of the activations, sm_100a.
//
// Y^T = W X^T with W (N x K, NVFP4, TILED scales) as the 128-row A operand of
// tcgen05.mma.kind::mxf4nvf4.block_scale.block16 and the activation rows
// (padded to 16) as the B operand.  With a residue R (ResServe abstract: FP4
// base plus FP4 residue, combined on-chip) X and R are stacked into one B
// operand, R's rows starting at row ro: ro = 8 for M <= 8 (one 16-row
// operand, the plain case's instructions), else ro = 16 (a 32-row operand).
// Each MMA then produces both products side by side in one accumulator, and
// Y = s_x s_w acc[:, 0:M] + s_r s_w acc[:, ro:ro+M].
//
// Fused mode (nvfp4_quantize_gemm): the kernel reads X in bf16/fp32 and
// quantizes it itself.  The ks CTAs of a cluster split K; together they cover
// the whole of X, so the tensor scale s = fl32(amax|X| / 2688) comes from one
// exchange of per-CTA maxima through distributed shared memory, and each CTA
// encodes its K-slice straight into shared memory in the MMA operand layout
// (the encoding routine is the quantizer's, so codes and scales are
// identical).  The cluster of the first 128-row tile also writes Q(X) (and
// Q(R)) to global memory.  This removes the separate quantizer launch and the
// hand-off between the two kernels from every decode call.
// Plain mode (nvfp4_gemm): X codes arrive by TMA, X scales are gathered.
//
// Activation scales sit in shared memory compactly: per k-tile and K=64 chunk,
// the 4 block scales of each of the 32 operand rows (X rows from 0, R rows
// from ro).  In TMEM they take the layout of a scale atom (lane l, column c:
// row 32c + l), with rows 32 and up absent (zero).  The scale operands of a
// block-scaled MMA start on a 4-column TMEM boundary: each K=64 MMA reads one
// atom's 4 columns.  With a residue, each CTA pushes s_x s_w acc_x + s_r s_w
// acc_r per row, so partial rows travel once.
//
// Grid: (ks, ceil(N/128)), cluster (ks, 1, 1), ks <= 8.  CTA rank r of a
// cluster handles k-tiles [r*kt/ks, (r+1)*kt/ks).  Roles (256 threads): every
// warp takes part in the activation quantization; warp 0 lane 0 streams W
// tiles and scale atoms through a TMA ring; warps 4-7 (one per TMEM lane
// quadrant) write each stage's W and activation scale atoms into the stage's
// TMEM scale buffer with tcgen05.st while warp 1 lane 0 issues the MMAs of the
// previous stage; warps 0-3 drain the accumulators and push their partial rows
// into a dedicated area of the owning CTA's shared memory (row r of the tile
// belongs to rank floor(r*ks/128)); each owner sums its rows and writes Y.
// Per-CTA maxima travel the same way: each CTA sends its maximum to every
// peer.  All traffic between CTAs is point to point: st.async stores whose
// bytes complete on an mbarrier of the receiving CTA, armed at start-up with
// the exact byte count it will receive, so a receiver waits only for its own
// data and no cluster-wide barrier sits on the critical path.  Every CTA
// announces at start-up that it is running (a relaxed cluster arrive) and
// waits for its peers' announcements before its first store into another CTA's
// shared memory; it exits only after every byte addressed to it has arrived.
//
// The kernel is a programmatic dependent of the preceding kernel: before
// griddepcontrol.wait it only sets up and asks L2 to prefetch its W tiles
// (L2 is coherent, so a prefetch never yields stale data); every load that
// feeds the result is issued after the wait.
//
// Safety: every mbarrier wait is bounded; every CTA reaches the start-up
// cluster barrier and sends every store its peers count on, on every path
// (both depend only on kernel arguments, which are uniform over the cluster,
// and a CTA whose pipeline gave up sends zeros); the shared-memory request
// covers the whole layout and the CTAs per SM are capped so that their TMEM
// allocations always fit side by side.
#include <cstring>

#include "kernels.h"
#include "quant_common.cuh"
#include "tcgen05.cuh"

namespace nvfp4 {
using namespace tc;
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int NP = 16;                       // activation rows, padded
constexpr int W_TILE = 128 * 128;            // 128 W rows x 256 K-elements
constexpr int SFW_BYTES = 4 * 512;           // one scale atom per K=64 chunk
constexpr int WSTAGE = W_TILE + SFW_BYTES;   // 18 KB, keeps 1024-byte alignment
constexpr int MAX_STAGES = 8;                // W ring depth limit; the launch picks p.stages in [2, 8]
constexpr int SF_BUFS = 2;                   // TMEM scale buffers, alternating by k-tile
constexpr int X_TILE = NP * 128;             // codes of one operand (X or R) in one k-tile (SW128)
constexpr int SF_TILE = 4 * 128;             // activation scales of one k-tile: 4 K=64 chunks x 32 rows
                                             // (rows 0-15 X, 16-31 R) x 4 block scales
// Residue row offset `ro`: 0 without a residue; otherwise R's rows start at
// operand row ro (8: X rows 0-7 and R rows 8-15 share one 16-row operand when
// M <= 8; 16: X rows 0-15, R rows 16-31).
__host__ __device__ constexpr int b_tile(int ro) { return ro == 16 ? 2 * X_TILE : X_TILE; }   // MMA B tile
__host__ __device__ constexpr int operand_rows(int ro) { return ro ? ro : NP; }   // rows per operand (X, R)
constexpr int BAR_BYTES = 256;
// floats per pushed partial row: M rounded up to 4 (16-byte rows)
__host__ __device__ constexpr int part_pitch(int M) { return (M + 3) & ~3; }
constexpr int MAX_KS = 8;   // portable cluster size: larger clusters wait for free slots inside one GPC

// Partial-row slots an owner holds: one slot of ceil(128/ks) rows per source
// rank, maximised over every cluster size the launcher may pick.
constexpr int max_part_rows() {
  int m = 0;
  for (int k = 1; k <= MAX_KS; ++k) m = (k * ((128 + k - 1) / k) > m) ? k * ((128 + k - 1) / k) : m;
  return m;
}
constexpr int PART_ROWS = max_part_rows();   // 133 (ks = 7)
// TMEM columns: acc [0,32) (X products in 0-15, R products in 16-31), then two
// scale buffers used by alternate k-tiles: W scales [+0,+16), X/R scales [+16,+32)
constexpr uint32_t ACC = 0, SF_COL = 32, SF_BUF = 32, SFX_OFF = 16, TMEM_COLS = 128;   // R products: column ro
static_assert(SFX_OFF == 16 && SF_BUF >= 32, "one 32-column TMEM store writes a stage's W and X scales");
static_assert(SF_COL % 4 == 0 && SF_BUF % 4 == 0 && SFX_OFF % 4 == 0,
              "block-scaled MMA scale operands start on 4-column TMEM boundaries");
static_assert(SF_COL + SF_BUFS * SF_BUF <= TMEM_COLS, "TMEM columns");
constexpr int TMEM_CTAS = 512 / TMEM_COLS;

static_assert(WSTAGE % 1024 == 0 && X_TILE % 1024 == 0, "SW128 tiles need 1024-byte alignment");
static_assert(PART_ROWS == 133, "slot count for ks <= 8");
// one pushed vector per row: the partial X product, or with a residue the
// already scaled sum s_x s_w acc_x + s_r s_w acc_r
__host__ __device__ constexpr int part_bytes(int M) { return PART_ROWS * part_pitch(M) * 4; }
static_assert((2 * MAX_STAGES + SF_BUFS + 5) * 8 + 16 + 8 <= BAR_BYTES, "barrier block");

struct DecodeParams {
  const void* x;        // fused: activations, M x K (ldx), bf16 or fp32
  int64_t ldx;
  const float* s_in;    // fused: given tensor scales or null (computed)
  const float* sr_in;
  QOut q, r;            // fused: Q(X), Q(R) written by the first row tile's cluster
  const uint8_t* sfx;   // plain: X / R scales (ROWMAJOR or TILED) and tensor scales
  const uint8_t* sfr;
  int x_tiled;
  const float* x_s;
  const float* r_s;
  const uint8_t* sfw;   // W scales, TILED
  const float* w_s;
  void* y;
  int64_t ldy;
  int M, N, K;
  int katoms_w;         // scale atoms per 128-row group of W = K / 64
  int k_tiles;          // ceil(K / 256)
  int kt_max;           // k-tiles per CTA held in the activation area
  int stages;           // W ring depth, 2..MAX_STAGES
  int* st;
  uint64_t wait_ns;     // bound on every mbarrier wait
  int hold;             // test of the timeout path: no W tile is loaded
  int prefetch;         // prefetch W into L2 before the dependency wait
};

// u / d for u < 2^16, d < 2^16 with m = ceil(2^32 / d): the error u*(m - 2^32/d)/2^32
// stays below 1/d, so the quotient is exact.
__device__ __forceinline__ int div_magic(int u, uint32_t m) { return (int)__umulhi((uint32_t)u, m); }

// Fused mode encodes the activation operand of all its k-tiles up front, and
// plain mode loads all of them at once (kt_max B tiles after the ring); plain
// mode with the 32-row X+R operand (ro = 16) streams each k-tile's B tile
// through the ring with its W tile instead (a stage is W_TILE + SFW_BYTES + B
// tile), since kt_max of its 4 KB tiles would leave one CTA per SM.
__host__ __device__ constexpr bool streams_b(int ro, bool fused) { return !fused && ro == 16; }
__host__ __device__ constexpr int stage_bytes(int ro, bool fused) {
  return streams_b(ro, fused) ? WSTAGE + b_tile(ro) : WSTAGE;
}
__host__ __device__ constexpr int smem_bytes(int stages, int kt_max, int ro, int M, bool fused) {
  return 1024 + stages * stage_bytes(ro, fused) + kt_max * ((streams_b(ro, fused) ? 0 : b_tile(ro)) + SF_TILE) +
         part_bytes(M) + BAR_BYTES;
}

template <typename T, bool FUSED, int RES, bool BF16OUT, int R>
__global__ void __launch_bounds__(kThreads, 1)
    k_decode_tc(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                const __grid_constant__ CUtensorMap tmR, const DecodeParams p) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int KT = p.kt_max;
  const int NS = p.stages;                                          // W ring depth
  constexpr int BT = b_tile(RES);                                   // B tile bytes per k-tile
  constexpr bool STREAM = streams_b(RES, FUSED);                    // B tiles travel with the W stages
  constexpr int SSTRIDE = stage_bytes(RES, FUSED);                  // ring stage: W (+ B tile)
  constexpr int OPR = operand_rows(RES);                            // rows of X (and of R)
  uint8_t* xcodes = smem + NS * SSTRIDE;                            // KT B tiles (unless STREAM)
  uint8_t* rcodes = xcodes + RES * 128;                             // R rows of each B tile
  uint8_t* sfxp = xcodes + (STREAM ? 0 : KT * BT);                  // KT x 512 B activation scales
  uint8_t* sfrp = sfxp + RES * 4;                                   // R scales: rows RES..
  const int pitch = part_pitch(p.M);
  float* part = reinterpret_cast<float*>(sfxp + KT * SF_TILE);      // pushed partial rows
  uint64_t* bars = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(part) + part_bytes(p.M));
  uint64_t* full = bars;                                            // [NS] W stage landed
  uint64_t* empty = bars + MAX_STAGES;                              // [NS] MMAs of the stage's k-tile done
  uint64_t* acc_full = bars + 2 * MAX_STAGES;
  uint64_t* x_full = acc_full + 1;
  uint64_t* sf_full = x_full + 1;                                   // [SF_BUFS] scale buffer written to TMEM
  uint64_t* xbar = sf_full + SF_BUFS;                               // [2] peers' |x|, |r| maxima arrived
  uint64_t* pbar = xbar + 2;                                        // peers' partial rows arrived
  WaitState* abort_flag = reinterpret_cast<WaitState*>(pbar + 1);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(abort_flag + 1);
  __shared__ uint32_t red[kWarps];
  __shared__ uint32_t xall[2][MAX_KS];                              // every CTA's |x|, |r| maximum

  griddep_launch_dependents();   // the next kernel may set itself up; it waits for this one's results

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank(), ks = cluster_nctarank();
  const int rt = blockIdx.y;                                        // 128-row tile of W
  const int kt0 = (int)((rank * (uint32_t)p.k_tiles) / ks);
  const int kt1 = (int)(((rank + 1) * (uint32_t)p.k_tiles) / ks);
  const int nkt = kt1 - kt0;
  // rows [owner_row0(o), owner_row0(o + 1)) of the tile are summed by rank o
  auto owner_row0 = [&](uint32_t o) { return (int)((o * 128u + ks - 1) / ks); };
  const bool x_exchange = FUSED && p.s_in == nullptr;
  const bool r_exchange = FUSED && RES && p.sr_in == nullptr;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(saddr(&full[s]), 1);
      mbar_init(saddr(&empty[s]), 1);
    }
    for (int b = 0; b < SF_BUFS; ++b) mbar_init(saddr(&sf_full[b]), 4);   // one arrival per scale warp
    mbar_init(saddr(acc_full), 1);
    mbar_init(saddr(x_full), 1);
    for (int i = 0; i < 2; ++i) mbar_init(saddr(&xbar[i]), 1);
    mbar_init(saddr(pbar), 1);
    // Arm the receive barriers with every byte the peers will send: one word
    // per exchanged maximum, and `pitch` floats per owned row.
    if (x_exchange) mbar_expect_tx(saddr(&xbar[0]), (ks - 1u) * 4u);
    if (r_exchange) mbar_expect_tx(saddr(&xbar[1]), (ks - 1u) * 4u);
    const uint32_t owned = (uint32_t)(owner_row0(rank + 1) - owner_row0(rank));
    mbar_expect_tx(saddr(pbar), (ks - 1u) * owned * (uint32_t)(pitch * 4));
    abort_flag->abort = 0;
    abort_flag->limit_ns = p.wait_ns;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(saddr(tmem_slot)),
                 "r"(TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  cluster_arrive_relaxed();   // this CTA is running: peers may store into its shared memory
  bool peers_running = false; // this thread has waited for the peers' start-up arrivals

  auto w_chunks = [&](int kt) { return min(4, (p.K - kt * 256) / 64); };   // K = 64 chunks in k-tile kt
  auto load_w = [&](int kt, int s) {   // the stage's W tile and scale atoms (STREAM: and its B tile)
    const uint32_t sf = (uint32_t)w_chunks(kt) * 512u;
    uint8_t* sb = smem + s * SSTRIDE;
    const uint32_t bar = saddr(&full[s]);
    mbar_expect_tx(bar, (uint32_t)W_TILE + sf + (STREAM ? (uint32_t)BT : 0u));
    tma_load_2d(saddr(sb), &tmW, kt * 128, rt * 128, bar);
    bulk_load(saddr(sb + W_TILE), p.sfw + ((size_t)rt * p.katoms_w + kt * 4) * 512, sf, bar);
    if (STREAM) {
      tma_load_2d(saddr(sb + WSTAGE), &tmX, kt * 128, 0, bar);
      if (RES) tma_load_2d(saddr(sb + WSTAGE + RES * 128), &tmR, kt * 128, 0, bar);
    }
  };

  if (p.prefetch && warp == 0 && lane == 0) {
    // warm L2 with this CTA's W tiles and scale atoms while the preceding kernel finishes
    for (int kt = kt0; kt < kt1; ++kt) {
      prefetch_l2_tile_2d(&tmW, kt * 128, rt * 128);
      prefetch_l2_bulk(p.sfw + ((size_t)rt * p.katoms_w + kt * 4) * 512, (uint32_t)w_chunks(kt) * 512u);
    }
  }
  griddep_wait();   // everything below may read the preceding kernel's results

  // fused: issue the activation loads first, so they are not queued behind the W stream
  [[maybe_unused]] Raw8<T> raw[FUSED ? R : 1];
  [[maybe_unused]] const int c0 = kt0 * 256;
  [[maybe_unused]] const int upr = (min(kt1 * 256, p.K) - c0) >> 3;   // 8-element units per row (multiple of 8)
  // 2^32 / upr, rounded up (slices of one launch have one of two widths)
  [[maybe_unused]] const uint32_t upr_m = (uint32_t)((0x100000000ull + (uint64_t)upr - 1) / (uint64_t)upr);
  [[maybe_unused]] const int U = p.M * upr;
  if constexpr (FUSED) {
    const T* x = static_cast<const T*>(p.x);
#pragma unroll
    for (int i = 0; i < R; ++i) {
      const int u = i * kThreads + (int)threadIdx.x;
      if (u < U) {
        const int row = div_magic(u, upr_m), c8 = u - row * upr;
        raw[i].load(x + (int64_t)row * p.ldx + c0 + c8 * 8);
      } else {
        raw[i].zero();
      }
    }
  }
  const int pre = p.hold ? 0 : min(nkt, NS);   // every stage of the ring is loaded at once
  int issued = pre;   // W stages loaded (warp 0 lane 0)
  if (warp == 0 && lane == 0) {
    if (!FUSED && !STREAM) {
      mbar_expect_tx(saddr(x_full), (uint32_t)(nkt * BT));
      for (int t = 0; t < nkt; ++t) {
        tma_load_2d(saddr(xcodes + t * BT), &tmX, (kt0 + t) * 128, 0, saddr(x_full));
        if (RES) tma_load_2d(saddr(rcodes + t * BT), &tmR, (kt0 + t) * 128, 0, saddr(x_full));
      }
    }
    for (int i = 0; i < pre; ++i) load_w(kt0 + i, i);   // the ring starts empty
  }

  // Cluster-wide maximum: send this CTA's maximum to every peer (st.async,
  // counted on the peer's barrier xbar[which]), then wait until all peers'
  // maxima have arrived here.  Every thread calls it.
  auto cluster_max = [&](uint32_t key, int which) {
    const uint32_t m = block_max_u32(key, red);
    if (!peers_running) {
      cluster_wait();
      peers_running = true;
    }
    if (threadIdx.x < ks && threadIdx.x != rank)
      st_async_u32(mapa_shared(saddr(&xall[which][rank]), threadIdx.x), m,
                   mapa_shared(saddr(&xbar[which]), threadIdx.x));
    (void)mbar_drain<true>(saddr(&xbar[which]), 0u, abort_flag, p.st);   // peers send on every path
    return max(m, warp_max_u32(lane < (int)ks && lane != (int)rank ? xall[which][lane] : 0u));
  };

  float sx = 0.0f, sr = 0.0f;   // activation / residue tensor scales for the epilogue
  if constexpr (!FUSED) {
    sx = *p.x_s;
    if (RES) sr = *p.r_s;
    // ---- gather the activation scales into atoms: line n of atom j of k-tile t
    // starts with the 4 block scales of row n in K chunk 4(kt0+t)+j
    const int nblk = p.K >> 4;
    for (int idx = threadIdx.x; idx < nkt * OPR * 4 * (RES ? 2 : 1); idx += kThreads) {
      const int which = idx / (nkt * OPR * 4);
      const int e = idx - which * (nkt * OPR * 4);
      const int t = e / (OPR * 4), n = (e >> 2) & (OPR - 1), j = e & 3;
      const int chunk = 4 * (kt0 + t) + j;
      const uint8_t* src = which ? p.sfr : p.sfx;
      uint32_t word = 0u;
      if (chunk * 4 < nblk) {
        if (p.x_tiled)
          word = *reinterpret_cast<const uint32_t*>(src + (size_t)chunk * 512 + n * 16);
        else if (n < p.M)
          word = *reinterpret_cast<const uint32_t*>(src + (size_t)n * nblk + chunk * 4);
      }
      *reinterpret_cast<uint32_t*>((which ? sfrp : sfxp) + t * SF_TILE + j * 128 + n * 4) = word;   // R: rows RES..
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  } else {
    // ---- quantize this CTA's K-slice of X into the operand layout
    if (U > R * kThreads) report_status(p.st, NVFP4_ERR_UNSUPPORTED);   // the host split rules this out
    const bool reporter = rank == 0 && threadIdx.x == 0;
    const bool writer = blockIdx.y == 0;                // this cluster also writes Q(X), Q(R)
    uint32_t key = 0u;
#pragma unroll
    for (int i = 0; i < R; ++i) key = max(key, raw[i].abs_key_max());
    if (key >= 0x7F800000u) report_status(p.st, NVFP4_ERR_NONFINITE);
    float s;
    if (p.s_in != nullptr) {
      s = *p.s_in;
    } else {
      s = scale_from_key(cluster_max(key, 0), reporter, p.st);
    }
    float s_r = (RES && p.sr_in != nullptr) ? *p.sr_in : 0.0f;
    if (writer && reporter) {
      if (p.q.s != p.s_in) *p.q.s = s;
      if (RES && p.sr_in != nullptr && p.r.s != p.sr_in) *p.r.s = s_r;
    }

    // place one encoded unit: codes into the SW128 tile, the block scale into its atom
    auto place = [&](uint8_t* codes_area, uint8_t* sf_area, const QOut& qo, int u, uint32_t codes, uint32_t db) {
      const int row = div_magic(u, upr_m), c8 = u - row * upr;
      const int t = c8 >> 5, kk = (c8 & 31) * 8;         // k-tile within the slice, column within it
      const int chunk16 = kk >> 5;                         // 16-byte chunk of the 128-byte row
      *reinterpret_cast<uint32_t*>(codes_area + t * BT + row * 128 + ((chunk16 ^ (row & 7)) << 4) +
                                   ((kk & 31) >> 1)) = codes;
      const int bt = kk >> 4;                              // 16-block within the k-tile
      if ((c8 & 1) == 0) sf_area[t * SF_TILE + (bt >> 2) * 128 + row * 4 + (bt & 3)] = (uint8_t)db;
      if (writer) store_half_block(qo, row, (c0 >> 3) + c8, codes, db);
    };

    uint32_t rkey = 0u;
#pragma unroll
    for (int i = 0; i < R; ++i) {
      const int u = i * kThreads + (int)threadIdx.x;
      const bool act = u < U;
      float v[8], deq[8];
      raw[i].get(v);
      uint32_t db;
      const uint32_t codes = quant_half_block(v, s, db, RES ? deq : nullptr);
      if (act) place(xcodes, sfxp, p.q, u, codes, db);
      if (RES) {
        float rv[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) rv[j] = __fsub_rn(v[j], deq[j]);
        if (p.sr_in != nullptr) {
          uint32_t dr;
          const uint32_t rc = quant_half_block(rv, s_r, dr, nullptr);
          if (act) place(rcodes, sfrp, p.r, u, rc, dr);
        } else if (act) {
#pragma unroll
          for (int j = 0; j < 8; ++j) rkey = max(rkey, abs_key(rv[j]));
        }
      }
    }
    if (RES && p.sr_in == nullptr) {
      s_r = scale_from_key(cluster_max(rkey, 1), reporter, p.st);
      if (writer && reporter) *p.r.s = s_r;
#pragma unroll
      for (int i = 0; i < R; ++i) {
        const int u = i * kThreads + (int)threadIdx.x;
        float v[8], deq[8], rv[8];
        raw[i].get(v);
        uint32_t db, dr;
        (void)quant_half_block(v, s, db, deq);
#pragma unroll
        for (int j = 0; j < 8; ++j) rv[j] = __fsub_rn(v[j], deq[j]);
        const uint32_t rc = quant_half_block(rv, s_r, dr, nullptr);
        if (u < U) place(rcodes, sfrp, p.r, u, rc, dr);
      }
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");   // generic writes -> tensor core reads
    sx = s;
    sr = s_r;
  }
  __syncthreads();   // activation operand (fused) / packed scales (plain) complete

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------- W producer (rest of the ring)
    int s = pre % NS;
    uint32_t ph = (pre == NS) ? 1u : 0u;
    for (int kt = kt0 + pre; !p.hold && kt < kt1; ++kt, ++issued) {
      if (!mbar_wait(saddr(&empty[s]), ph ^ 1u, abort_flag, p.st)) break;
      load_w(kt, s);
      if (++s == NS) { s = 0; ph ^= 1u; }
    }
    // the last NS stages' copies (and the activation codes) may still be in
    // flight if a consumer gave up: let them land before the CTA can exit
    for (int g2 = max(0, issued - NS); g2 < issued; ++g2)
      (void)mbar_drain(saddr(&full[g2 % NS]), (uint32_t)((g2 / NS) & 1), abort_flag, p.st);
    if (!FUSED && !STREAM) (void)mbar_drain(saddr(x_full), 0u, abort_flag, p.st);
  } else if (warp >= 4) {
    // ------------------------------------------- scales into TMEM (tcgen05.st)
    // Warp w writes TMEM lane quadrant w - 4 of scale buffer t & 1 for the
    // CTA's k-tile t: line l of each W atom, then of the k-tile's activation
    // atoms, in every lane l of the quadrant (the layout a 32x128b.warpx4 copy
    // of the same atoms gives).  Scale copies issued to the tensor pipe would
    // queue behind the stream of W tiles; these stores do not.  Buffer t & 1
    // was last read by the MMAs of k-tile t - 2, so its stores wait for that
    // k-tile's commit (the ring has at least two stages, so that commit's phase
    // is still the current one of its barrier).
    const uint32_t quad = (uint32_t)((warp - 4) * 32) << 16;
    auto write_tile = [&](int t, int s) {
      const uint8_t* sb = smem + s * SSTRIDE;
      uint32_t r[32];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint4 w = *reinterpret_cast<const uint4*>(sb + W_TILE + j * 512 + lane * 16);
        r[4 * j] = w.x; r[4 * j + 1] = w.y; r[4 * j + 2] = w.z; r[4 * j + 3] = w.w;
        // activation rows are 0-31 only: line l carries row l's 4 scales
        r[16 + 4 * j] = *reinterpret_cast<const uint32_t*>(sfxp + t * SF_TILE + j * 128 + lane * 4);
        r[16 + 4 * j + 1] = 0u; r[16 + 4 * j + 2] = 0u; r[16 + 4 * j + 3] = 0u;
      }
      tmem_st32(tmem + quad + SF_COL + (uint32_t)(t & 1) * SF_BUF, r);   // W scales, then X (and R) scales
    };
    auto buf_free = [&](int t) {   // the MMAs of k-tile t - 2 have completed
      return t < 2 || mbar_test_wait(saddr(&empty[(t - 2) % NS]), (uint32_t)(((t - 2) / NS) & 1));
    };
    for (int t = 0; t < nkt;) {
      // every lane waits; the warp goes on only if all saw the phase (the
      // TMEM store is warp-collective)
      if (t >= 2 && !__all_sync(0xFFFFFFFFu, mbar_wait(saddr(&empty[(t - 2) % NS]),
                                                       (uint32_t)(((t - 2) / NS) & 1), abort_flag, p.st)))
        break;
      if (!__all_sync(0xFFFFFFFFu, mbar_wait(saddr(&full[t % NS]), (uint32_t)((t / NS) & 1), abort_flag, p.st)))
        break;
      tc_fence_after();
      write_tile(t, t % NS);
      // k-tile t + 1 joins the batch if its stage has landed and its buffer is
      // free: one wait covers both stores
      const bool two = t + 1 < nkt &&
                       __all_sync(0xFFFFFFFFu, buf_free(t + 1) && mbar_test_wait(saddr(&full[(t + 1) % NS]),
                                                                                 (uint32_t)(((t + 1) / NS) & 1)));
      if (two) {
        tc_fence_after();
        write_tile(t + 1, (t + 1) % NS);
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(saddr(&sf_full[t & 1]));
        if (two) mbar_arrive(saddr(&sf_full[(t + 1) & 1]));
      }
      t += two ? 2 : 1;
    }
  } else if (warp == 1 && lane == 0) {
    // --------------------------------------------------------- MMA issuer
    bool ok = true;
    if (!FUSED && !STREAM) ok = mbar_wait(saddr(x_full), 0u, abort_flag, p.st);
    const uint32_t idesc = idesc_nvf4(RES == 16 ? 2 * NP : NP);
    for (int t = 0; ok && t < nkt; ++t) {
      const int s = t % NS;
      if (!mbar_wait(saddr(&full[s]), (uint32_t)((t / NS) & 1), abort_flag, p.st)) break;
      if (!mbar_wait(saddr(&sf_full[t & 1]), (uint32_t)((t >> 1) & 1), abort_flag, p.st)) break;
      tc_fence_after();
      const int kt = kt0 + t, jmax = w_chunks(kt);
      const uint8_t* sb = smem + s * SSTRIDE;
      const uint32_t sfw = SF_COL + (uint32_t)(t & 1) * SF_BUF, sfx = sfw + SFX_OFF;
      const uint64_t dw = desc_sw128(saddr(sb)), dx = desc_sw128(saddr(STREAM ? sb + WSTAGE : xcodes + t * BT));
      for (int j = 0; j < jmax; ++j) {
        const uint32_t acc = (t > 0 || j > 0) ? 1u : 0u;
        tc_mma_nvf4(tmem + ACC, dw + (uint64_t)(2 * j), dx + (uint64_t)(2 * j), idesc, tmem + sfw + 4 * j,
                    tmem + sfx + 4 * j, acc);
      }
      // Someone waits for this k-tile's MMAs only if its stage is refilled
      // (t + NS < nkt) or its scale buffer is reused (t + 2 < nkt); with
      // NS >= 2 both come down to t + 2 < nkt.  A commit costs tensor-pipe
      // time, so the last two k-tiles go without one (acc_full covers them).
      if (t + 2 < nkt) tc_commit(saddr(&empty[s]));
    }
    tc_commit(saddr(acc_full));
  }
  __syncwarp();

  // ------------------- push this CTA's partial rows to the CTA that owns them
  // the commit after the MMA loop is issued on every path: waiting for it also
  // waits for every MMA in flight, before TMEM is read and released
  const bool ok = mbar_drain(saddr(acc_full), 0u, abort_flag, p.st) && !wait_aborted(abort_flag);
  tc_fence_after();
  __syncwarp();     // the cluster barrier below is warp-aligned
  if (!peers_running) cluster_wait();   // uniform: no maximum was exchanged
  const int rows_max = (int)((128u + ks - 1) / ks);
  if (warp < 4) {
    // Own rows are stored locally; the others travel by st.async and are
    // counted on the owner's barrier pbar.
    const int row = warp * 32 + lane;                              // TMEM lane = W row of the tile
    const uint32_t o = (uint32_t)row * ks / 128u;
    const int slot = (int)rank * rows_max + (row - owner_row0(o));
    const bool local = o == rank;
    const uint32_t dst = mapa_shared(saddr(part + slot * pitch), o);
    const uint32_t dst_bar = mapa_shared(saddr(pbar), o);
    const uint32_t lane_addr = tmem + ((uint32_t)(warp * 32) << 16);
    uint32_t v[16];
    tmem_ld16(lane_addr + ACC, v);
    if constexpr (RES != 0) {
      // combine X and R products here: each row travels once, already scaled
      uint32_t vr[16];
      if constexpr (RES == 16) {
        tmem_ld16(lane_addr + ACC + 16, vr);
        tmem_ld_wait();
      } else {   // R products in columns 8-15 of the same load
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 8; ++i) vr[i] = v[8 + i];
      }
      const float ws = *p.w_s;
      const float alpha = __fmul_rn(sx, ws), alpha_r = __fmul_rn(sr, ws);
#pragma unroll
      for (int i = 0; i < RES; ++i)
        v[i] = __float_as_uint(__fmaf_rn(__uint_as_float(v[i]), alpha, __fmul_rn(__uint_as_float(vr[i]), alpha_r)));
    } else {
      tmem_ld_wait();
    }
    if (!ok) {
#pragma unroll
      for (int i = 0; i < 16; ++i) v[i] = 0u;
    }
    // the first `pitch` (>= M) products of the row
    if (local) {
#pragma unroll
      for (int i = 0; i < 16; i += 4)
        if (i < pitch)
          *reinterpret_cast<uint4*>(part + slot * pitch + i) = make_uint4(v[i], v[i + 1], v[i + 2], v[i + 3]);
    } else {
#pragma unroll
      for (int i = 0; i < 16; i += 4)
        if (i < pitch)
          st_async_f32x4(dst + (uint32_t)(i * 4), __uint_as_float(v[i]), __uint_as_float(v[i + 1]),
                         __uint_as_float(v[i + 2]), __uint_as_float(v[i + 3]), dst_bar);
    }
  }
  tc_fence_before();
  __syncthreads();  // own partial rows stored; TMEM reads done before the dealloc
  // Every peer's partial rows have landed here.  Each CTA also waits for all
  // bytes addressed to it before it exits, so no store targets an exited CTA.
  (void)mbar_drain<true>(saddr(pbar), 0u, abort_flag, p.st);

  // ------------------------------------------------ owners sum their rows and store
  {
    const int r0 = owner_row0(rank), r1 = owner_row0(rank + 1);
    const int nrows = r1 - r0;
    const float alpha = __fmul_rn(sx, *p.w_s);
    for (int idx = threadIdx.x; idx < nrows * p.M; idx += kThreads) {
      const int m = idx / nrows, i = idx - m * nrows;
      const int n = rt * 128 + r0 + i;
      if (n >= p.N) continue;
      float sum = 0.0f;
      for (uint32_t src = 0; src < ks; ++src) sum += part[((int)src * rows_max + i) * pitch + m];
      const float out = RES ? sum : sum * alpha;   // residue partials arrive scaled
      if (BF16OUT)
        reinterpret_cast<__nv_bfloat16*>(p.y)[(int64_t)m * p.ldy + n] = __float2bfloat16_rn(out);
      else
        reinterpret_cast<float*>(p.y)[(int64_t)m * p.ldy + n] = out;
    }
  }

  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS) : "memory");
  }
}


// ------------------------------------------------------------------ host side

constexpr double kFixedUs = 5.0;     // launch-to-exit latency of one wave of CTAs (measured, few k-tiles)
constexpr double kTileUs = 0.8;      // one k-tile (scale stores, 4 MMAs, 1 commit) per CTA, up to 4 CTAs per SM
constexpr double kQuantUs = 4.0;     // one-launch quantizer plus the hand-off to the next kernel
                                     // (with a computed residue scale, plus its second exchange)
constexpr double kExchangeUs = 1.3;  // fused: one cluster-wide maximum (stores into peers + wait)
constexpr double kUnitUs = 0.15;     // fused: encoding one 8-element unit per thread, per co-resident CTA
constexpr int kGpcSms = 16;          // SMs per GPC assumed when packing clusters (the smallest GPCs)
// A request of at least this many bytes keeps at most TMEM_CTAS CTAs on an SM
// (228 KB per SM, 1 KB reserved per CTA), so tcgen05.alloc never waits for a
// CTA of another cluster.
constexpr int kSmemFloor = 233472 / (TMEM_CTAS + 1) - 1024 + 16;
static_assert((kSmemFloor + 1024) * (TMEM_CTAS + 1) > 233472, "smem floor");

struct Choice {
  int ks = 0, kt_max = 0, stages = 0, smem = 0;
  double cost = 1e30;
};

// CTAs of `smem` bytes and `regs` registers per thread that one SM holds.
int ctas_per_sm(int smem, int regs) {
  int per_sm = std::min({233472 / (smem + 1024), TMEM_CTAS, 2048 / kThreads});
  if (regs > 0) per_sm = std::min(per_sm, 65536 / (((regs + 7) / 8) * 8 * kThreads));
  return per_sm;
}

// Cluster split of K for a kernel instance with `regs` registers per thread:
// waves of resident CTAs cost a fixed latency plus the per-CTA time of their
// k-tiles and, fused (units_cap > 0), the `exchanges` cluster-wide maxima and the encoding
// of the CTA's activation slice (every unit of which must fit in units_cap
// register arrays per thread).  The smaller split wins ties.  The W ring then
// takes as many stages (up to the CTA's k-tiles) as keep the same number of
// CTAs per SM: measured, a deeper ring gains a little where it costs no
// residency and loses a whole wave where it does.
Choice choose_split(int row_tiles, int k_tiles, int ro, int num_sms, int regs, int M, int K, int units_cap,
                    int exchanges) {
  const bool res = ro != 0;
  // waves of ks-CTA clusters with `per_sm` CTAs per SM: a cluster must fit
  // inside one GPC, so count only the slots that whole clusters fill in GPCs
  // of kGpcSms SMs
  auto waves_of = [&](int ks, int per_sm) {
    const int per_gpc = kGpcSms * per_sm;
    const int64_t ctas = (int64_t)row_tiles * ks,
                  slots = (int64_t)per_sm * num_sms * ((per_gpc / ks) * ks) / per_gpc;
    return slots > 0 ? (ctas + slots - 1) / slots : int64_t(1) << 40;
  };
  Choice best;
  for (int ks = 1; ks <= std::min(MAX_KS, k_tiles); ++ks) {
    const int kt_max = (k_tiles + ks - 1) / ks;
    const int smem = std::max(smem_bytes(2, kt_max, ro, M, units_cap > 0), kSmemFloor);
    if (smem > 232448) continue;
    const int slice = std::min(kt_max * 256, K);
    const int64_t units = (int64_t)M * (slice / 8);
    if (units_cap > 0 && units > (int64_t)units_cap * kThreads) continue;
    const int per_sm = ctas_per_sm(smem, regs);
    if (per_sm < 1) continue;
    const int64_t ctas = (int64_t)row_tiles * ks, slots = (int64_t)per_sm * num_sms;
    const int64_t waves = waves_of(ks, per_sm);
    double wave = kFixedUs + kTileUs * kt_max;
    if (units_cap > 0) {
      const double upt = (double)((units + kThreads - 1) / kThreads) * (res ? 2.0 : 1.0);
      const double co_resident = (double)std::min<int64_t>(per_sm, (std::min(ctas, slots) + num_sms - 1) / num_sms);
      wave += kExchangeUs * exchanges + kUnitUs * co_resident * upt;
    }
    const double cost = (double)waves * wave;
    if (cost < best.cost - 1e-9) best = Choice{ks, kt_max, 2, smem, cost};
  }
  // A ring that holds every W tile of the CTA, if the CTAs still fit in as
  // many waves (measured: all tiles in flight at once gains; a partly deeper
  // ring with fewer CTAs per SM can lose); else a deeper ring only while it
  // keeps the same number of CTAs per SM.
  if (best.ks > 0) {
    const int64_t waves = waves_of(best.ks, ctas_per_sm(best.smem, regs));
    const int all = best.kt_max;
    const int smem_all = std::max(smem_bytes(all, all, ro, M, units_cap > 0), kSmemFloor);
    const int per_sm_all = ctas_per_sm(smem_all, regs);
    if (all > 2 && all <= MAX_STAGES && smem_all <= 232448 && per_sm_all >= 1 &&
        waves_of(best.ks, per_sm_all) <= waves) {
      best.stages = all;
      best.smem = smem_all;
    } else {
      for (int st = 3; st <= std::min(MAX_STAGES, best.kt_max); ++st) {
        const int smem = std::max(smem_bytes(st, best.kt_max, ro, M, units_cap > 0), kSmemFloor);
        if (smem > 232448 || ctas_per_sm(smem, regs) < ctas_per_sm(best.smem, regs)) break;
        best.stages = st;
        best.smem = smem;
      }
    }
  }
  return best;
}

template <typename T, bool FUSED, int RES, bool BF16OUT, int R>
int regs_of() {
  static int regs = -1;
  if (regs < 0) {
    cudaFuncAttributes fa{};
    regs = cudaFuncGetAttributes(&fa, k_decode_tc<T, FUSED, RES, BF16OUT, R>) == cudaSuccess ? fa.numRegs : 255;
  }
  return regs;
}

template <typename T, bool FUSED, int RES, bool BF16OUT, int R>
cudaError_t launch_cfg(const DecodeArgs& a, DecodeParams p, const Choice& c, const CUtensorMap& tmW,
                       const CUtensorMap& tmX, const CUtensorMap& tmR, cudaStream_t stream) {
  if (a.dry_run) return cudaSuccess;
  auto kern = k_decode_tc<T, FUSED, RES, BF16OUT, R>;
  const int row_tiles = (int)((a.N + 127) / 128);
  p.kt_max = c.kt_max;
  p.stages = c.stages;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, c.smem);
  if (e != cudaSuccess) return e;
  if (c.ks > 8) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)c.ks, (unsigned)row_tiles, 1);
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
  return cudaLaunchKernelEx(&cfg, kern, tmW, tmX, tmR, p);
}

template <typename T, bool FUSED, int RES, bool BF16OUT>
cudaError_t launch_r(const DecodeArgs& a, const DecodeParams& p, const CUtensorMap& tmW, const CUtensorMap& tmX,
                     const CUtensorMap& tmR, int num_sms, cudaStream_t stream) {
  const int row_tiles = (int)((a.N + 127) / 128);
  const int M = (int)a.M, K = (int)a.K;
  // the same kernel on NVFP4 operands: the split for the plain instance
  const Choice plain = choose_split(row_tiles, p.k_tiles, RES, num_sms, regs_of<float, false, RES, BF16OUT, 0>(),
                                    M, K, 0, 0);
  if constexpr (!FUSED) {
    if (plain.ks == 0) return cudaErrorNotSupported;
    return launch_cfg<float, false, RES, BF16OUT, 0>(a, p, plain, tmW, tmX, tmR, stream);
  } else {
    // fused: the register-array size with the cheapest split; not worth it
    // (cudaErrorNotSupported) when quantizing separately is estimated faster
    // one cluster-wide maximum per tensor scale not given
    const int ex = (p.s_in == nullptr ? 1 : 0) + (RES && p.sr_in == nullptr ? 1 : 0);
    const Choice c1 = choose_split(row_tiles, p.k_tiles, RES, num_sms, regs_of<T, true, RES, BF16OUT, 1>(), M, K, 1, ex);
    const Choice c2 = choose_split(row_tiles, p.k_tiles, RES, num_sms, regs_of<T, true, RES, BF16OUT, 2>(), M, K, 2, ex);
    const Choice c4 = choose_split(row_tiles, p.k_tiles, RES, num_sms, regs_of<T, true, RES, BF16OUT, 4>(), M, K, 4, ex);
    const Choice c8 = choose_split(row_tiles, p.k_tiles, RES, num_sms, regs_of<T, true, RES, BF16OUT, 8>(), M, K, 8, ex);
    const Choice* best = &c1;
    int r = 1;
    if (c2.cost < best->cost - 1e-9) { best = &c2; r = 2; }
    if (c4.cost < best->cost - 1e-9) { best = &c4; r = 4; }
    if (c8.cost < best->cost - 1e-9) { best = &c8; r = 8; }
    const double quant_us = kQuantUs + (RES && p.sr_in == nullptr ? kExchangeUs : 0.0);
    if (best->ks == 0 || best->cost > plain.cost + quant_us) return cudaErrorNotSupported;
    switch (r) {
      case 1: return launch_cfg<T, true, RES, BF16OUT, 1>(a, p, *best, tmW, tmX, tmR, stream);
      case 2: return launch_cfg<T, true, RES, BF16OUT, 2>(a, p, *best, tmW, tmX, tmR, stream);
      case 4: return launch_cfg<T, true, RES, BF16OUT, 4>(a, p, *best, tmW, tmX, tmR, stream);
      default: return launch_cfg<T, true, RES, BF16OUT, 8>(a, p, *best, tmW, tmX, tmR, stream);
    }
  }
}

// residue row offset for this call (see b_tile)
int residue_rows(const DecodeArgs& a) {
  if (a.r_codes == nullptr && a.r_out.codes == nullptr) return 0;
  return a.M <= 8 ? 8 : 16;
}

template <typename T, bool FUSED>
cudaError_t launch_t(const DecodeArgs& a, const DecodeParams& p, const CUtensorMap& tmW, const CUtensorMap& tmX,
                     const CUtensorMap& tmR, int num_sms, cudaStream_t stream) {
  const int ro = residue_rows(a);
  if (ro == 8)
    return a.y_bf16 ? launch_r<T, FUSED, 8, true>(a, p, tmW, tmX, tmR, num_sms, stream)
                    : launch_r<T, FUSED, 8, false>(a, p, tmW, tmX, tmR, num_sms, stream);
  if (ro == 16)
    return a.y_bf16 ? launch_r<T, FUSED, 16, true>(a, p, tmW, tmX, tmR, num_sms, stream)
                    : launch_r<T, FUSED, 16, false>(a, p, tmW, tmX, tmR, num_sms, stream);
  return a.y_bf16 ? launch_r<T, FUSED, 0, true>(a, p, tmW, tmX, tmR, num_sms, stream)
                  : launch_r<T, FUSED, 0, false>(a, p, tmW, tmX, tmR, num_sms, stream);
}

}  // namespace

cudaError_t launch_decode_tc(const DecodeArgs& a, int num_sms, cudaStream_t stream) {
  if (a.M < 1 || a.M > NP || a.K % 64 != 0 || a.K < 256 || a.N < 1) return cudaErrorNotSupported;
  const bool fused = a.x != nullptr;
  CUtensorMap tmW, tmX, tmR;
  if (a.dry_run) {
    std::memset(&tmW, 0, sizeof(tmW));
    tmX = tmR = tmW;
  } else if (!encode_codes_map(&tmW, a.w_codes, a.N, a.K, 128)) {
    return cudaErrorInvalidValue;
  }
  if (a.dry_run) {
    // configuration only
  } else if (!fused) {
    const uint32_t box = (uint32_t)operand_rows(residue_rows(a));   // rows of X (and of R) per tile
    if (!encode_codes_map(&tmX, a.x_codes, a.M, a.K, box)) return cudaErrorInvalidValue;
    if (a.r_codes != nullptr) {
      if (!encode_codes_map(&tmR, a.r_codes, a.M, a.K, box)) return cudaErrorInvalidValue;
    } else {
      tmR = tmX;
    }
  } else {
    tmX = tmW;   // unused in fused mode
    tmR = tmW;
  }
  DecodeParams p{};
  p.x = a.x; p.ldx = a.ldx; p.s_in = a.s_in; p.sr_in = a.sr_in;
  p.q = a.q_out; p.r = a.r_out;
  p.sfx = a.x_scales; p.sfr = a.r_scales; p.x_tiled = a.x_tiled ? 1 : 0; p.x_s = a.x_s; p.r_s = a.r_s;
  p.sfw = a.w_scales; p.w_s = a.w_s;
  p.y = a.y; p.ldy = a.ldy;
  p.M = (int)a.M; p.N = (int)a.N; p.K = (int)a.K;
  p.katoms_w = (int)(a.K / 64);
  p.k_tiles = (int)((a.K + 255) / 256);
  p.st = a.st;
  const WaitTest wt = wait_test();
  p.wait_ns = wt.limit_ns;
  p.hold = wt.hold;
  p.prefetch = prefetch_w(a.N, a.K) ? 1 : 0;
  if (fused)
    return a.x_bf16 ? launch_t<__nv_bfloat16, true>(a, p, tmW, tmX, tmR, num_sms, stream)
                    : launch_t<float, true>(a, p, tmW, tmX, tmR, num_sms, stream);
  return launch_t<float, false>(a, p, tmW, tmX, tmR, num_sms, stream);   // element type unused
}

}  // namespace nvfp4
