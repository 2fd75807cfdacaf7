// Internal launch interface between the C-ABI layer (api.cu) and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>

#include "nvfp4.h"

namespace nvfp4 {

struct WsHeader;

// Output NVFP4 tensor as the quantizer kernels see it.
struct QOut {
  uint8_t* codes;
  uint8_t* scales;
  float* s;       // tensor scale (device)
  int64_t cols;   // columns of the whole tensor (row pitch = cols/2 bytes of codes)
  bool tiled;     // scale layout
};

enum QuantMode { Q_PLAIN = 0, Q_MAIN_AMAXR = 1, Q_RES_ONLY = 2, Q_BOTH = 3 };

cudaError_t launch_amax(const void* x, nvfp4_dtype dt, int64_t M, int64_t K, int64_t ldx,
                        WsHeader* ws, int slot, float* s_out, int* st, int num_sms,
                        cudaStream_t stream);
// after_amax: launched as a programmatic dependent of the k_amax launch just
// before it on the same stream (the quantizer overlaps that kernel's tail).
cudaError_t launch_quant(int mode, const void* x, nvfp4_dtype dt, int64_t M, int64_t K, int64_t ldx,
                         const float* s_ptr, const float* sr_ptr, const QOut& q, const QOut& r,
                         WsHeader* ws, int* st, int num_sms, cudaStream_t stream, bool after_amax = false);
cudaError_t launch_rms_stats(const void* x, nvfp4_dtype dt, int64_t M, int64_t K, int64_t ldx,
                             const void* gamma, float eps, WsHeader* ws, float* rinv, float* s_out,
                             bool want_scale, int* st, int num_sms, cudaStream_t stream);
// One-launch quantizer for inputs of at most quant_small_max_units(dt) 8-element
// units (M * K / 8); returns cudaErrorNotSupported above that.  With residue,
// r receives the residue; null s_in / sr_in mean "compute the tensor scale".
int64_t quant_small_max_units(nvfp4_dtype dt);
cudaError_t launch_quant_small(bool residue, const void* x, nvfp4_dtype dt, int64_t M, int64_t K, int64_t ldx,
                               const float* s_in, const float* sr_in, const QOut& q, const QOut& r, int* st,
                               cudaStream_t stream);
size_t reorder_smem_bytes(nvfp4_dtype dt, int64_t K, bool has_gamma);
// ARCQuant quantizer in one cooperative launch when every row fits in the
// shared memory of one wave of CTAs; cudaErrorNotSupported (nothing launched)
// otherwise.  Identical results to the statistics pass + launch_reorder_quant.
cudaError_t launch_reorder_onepass(const void* x, nvfp4_dtype dt, int64_t M, int64_t K, int64_t ldx,
                                   const void* gamma, float eps, const int32_t* perm, int64_t S,
                                   const float* s_in, const QOut& q, WsHeader* ws, int* st, int num_sms,
                                   cudaStream_t stream);
cudaError_t launch_reorder_quant(const void* x, nvfp4_dtype dt, int64_t M, int64_t K, int64_t ldx,
                                 const void* gamma, const float* rinv, const int32_t* perm,
                                 int64_t S, const float* s_ptr, const QOut& q, int* st, int num_sms,
                                 cudaStream_t stream, bool after_stats);

// Offline weight preparation: W_aug = [W' | W'[:, :S]], W'[:, j] = fl32(W[:, perm[j]] *
// sigma[perm[j]]) (sigma / perm may be null), quantized under s_in or its own
// computed tensor scale (written to q.s).
cudaError_t launch_weight_quant(const void* w, nvfp4_dtype dt, int64_t N, int64_t K, int64_t ldw,
                                const float* sigma, const int32_t* perm, int64_t S, const float* s_in,
                                const QOut& q, WsHeader* ws, int* st, int num_sms, cudaStream_t stream);

// Bounded-wait settings that the next tensor-core launches carry (process wide,
// host side): limit_ns bounds every device-side wait; hold != 0 makes the load
// issuers skip their operand loads, so that the waits run out and the launch
// reports NVFP4_ERR_TIMEOUT (a test of the timeout path, set through
// nvfp4_test_wait_fault).
struct WaitTest {
  uint64_t limit_ns;
  int hold;
};
WaitTest wait_test();
// The default bound on a device-side wait (4 s).
constexpr uint64_t tc_wait_default_ns() { return 4000000000ull; }

// The decode-sized kernels ask L2 to prefetch their W before their dependency
// wait, so that W streams while the preceding kernel finishes.  Beyond about a
// third of L2 (126 MB) the prefetched W and the W the preceding kernel is still
// streaming evict each other, so larger W is not prefetched.
constexpr int64_t kPrefetchMaxBytes = 40ll << 20;
inline bool prefetch_w(int64_t N, int64_t K) { return N * K / 16 * 9 <= kPrefetchMaxBytes; }

// Operands of the decode GEMV / tensor-core GEMM.
struct GemmArgs {
  const uint8_t* a_codes; const uint8_t* a_scales; const float* a_s;   // M x K
  const uint8_t* r_codes; const uint8_t* r_scales; const float* r_s;   // M x K (residue) or null
  const uint8_t* w_codes; const uint8_t* w_scales; const float* w_s;   // N x K
  void* y; int64_t ldy; bool y_bf16;
  int64_t M, N, K;
  int* st;
};

// Decode-sized linear (M <= 16) on the tensor cores.  Fused mode (x != null):
// X is quantized inside the kernel and Q(X) (and Q(R)) written to q_out
// (r_out); plain mode: X (and R) are NVFP4 tensors.  W must use TILED scales.
struct DecodeArgs {
  // fused mode
  const void* x; bool x_bf16; int64_t ldx;
  const float* s_in; const float* sr_in;
  QOut q_out, r_out;                      // r_out.codes != null selects the residue
  // plain mode
  const uint8_t* x_codes; const uint8_t* x_scales; const float* x_s;
  const uint8_t* r_codes; const uint8_t* r_scales; const float* r_s;
  bool x_tiled;                           // X / R scale layout
  // both
  const uint8_t* w_codes; const uint8_t* w_scales; const float* w_s;
  void* y; int64_t ldy; bool y_bf16;
  int64_t M, N, K;
  int* st;
  bool dry_run;                           // choose the configuration only; launch nothing
};
// cudaErrorNotSupported: fused mode is estimated slower than quantize-then-GEMM
// (or does not fit); nothing was launched.
cudaError_t launch_decode_tc(const DecodeArgs& a, int num_sms, cudaStream_t stream);

cudaError_t launch_gemv(const GemmArgs& g, int num_sms, cudaStream_t stream);
cudaError_t launch_gemm_tc(const GemmArgs& g, int num_sms, cudaStream_t stream);
// MXFP4 GEMM Y = deq(A) deq(W)^T: codes as for NVFP4, E8M0 scales in the TILED
// atom layout with 32-element blocks (a_s, w_s unused); K % 128 == 0.
cudaError_t launch_gemm_mx(const GemmArgs& g, int num_sms, cudaStream_t stream);
// MXFP4 (32-element blocks, E8M0 scales): codes row-major M x K/2, scales
// row-major M x K/32 or TILED; r_codes == nullptr: no residue.
cudaError_t launch_mx_quant(const void* x, nvfp4_dtype dt, int64_t M, int64_t K, int64_t ldx, uint8_t* codes,
                            uint8_t* scales, uint8_t* r_codes, uint8_t* r_scales, bool tiled, int* st, int num_sms,
                            cudaStream_t stream);
cudaError_t launch_gemv_tc(const GemmArgs& g, int num_sms, cudaStream_t stream);

}  // namespace nvfp4
