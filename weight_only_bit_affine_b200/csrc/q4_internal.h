// q4_internal.h -- host-side launcher declarations shared inside libq4.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <atomic>
#include <cstdint>
#include <vector>

namespace q4 {

// Device properties cached per device (first use of a device queries them).
struct DeviceInfo {
  int device = -1;
  int sm_count = 0;
  int cc_major = 0, cc_minor = 0;
  size_t smem_optin = 0;  // max dynamic shared memory per block (opt-in)
};
// Returns nullptr (and sets the error message) if the current device cannot
// be queried.
const DeviceInfo* current_device_info();

// One bit per device ordinal (< 64) for settings that are made once per
// kernel and device (cudaFuncSetAttribute applies to the current device).
// Two threads may both make the setting; it is idempotent.
struct PerDeviceOnce {
  std::atomic<uint64_t> done{0};
  bool needed(int device) const { return ((done.load(std::memory_order_acquire) >> device) & 1u) == 0; }
  void mark(int device) { done.fetch_or(uint64_t(1) << device, std::memory_order_release); }
};

// Output epilogue, applied to an fp32 accumulator before its single rounding
// to bf16.  The feed-forward block the projections belong to (SwiGLU MLP
// after the attention, each with its residual add) supplies the steps worth
// fusing into the matmul that produces their input:
//   kEpiResidual: y = r + acc        (o and down projections add the residual)
// SwiGLU, y = silu(acc_gate) * acc_up, is a problem with two weights
// (MatmulArgs::fused()), computed in one pass by every kernel family.
enum Epilogue : int { kEpiNone = 0, kEpiResidual = 1 };

// Launchers return cudaSuccess or the launch error.  Arguments are already
// validated by the ABI layer.
cudaError_t launch_quantize(const uint16_t* W, int64_t N, int64_t K, uint8_t* codes,
                            uint16_t* scales, uint16_t* biases, cudaStream_t stream,
                            const DeviceInfo& dev);
cudaError_t launch_dequantize(const uint8_t* codes, const uint16_t* scales,
                              const uint16_t* biases, int64_t N, int64_t K, uint16_t* W_out,
                              cudaStream_t stream, const DeviceInfo& dev);

struct MatmulArgs {
  const uint16_t* x;  // [M, K]
  const uint8_t* codes;
  const uint16_t* scales;
  const uint16_t* biases;
  uint16_t* y;  // [M, N]
  int64_t M, N, K;
  // Output epilogue (Epilogue above) with its bf16 operand r [M, N] (NULL
  // for kEpiNone; may equal y).
  int epi = 0;
  const uint16_t* r = nullptr;
  // SwiGLU in one pass: when up_codes is set, y = silu(x . w_hat^T) *
  // (x . w_hat_up^T), the up weights with the same shape.
  const uint8_t* up_codes = nullptr;
  const uint16_t* up_scales = nullptr;
  const uint16_t* up_biases = nullptr;
  bool fused() const { return up_codes != nullptr; }
};
// The 8-bit variant (q8.cu): codes [N, K] one byte each; K <= kQ8MaxK.
constexpr int64_t kQ8MaxK = 196608;  // per-group sums of two activation rows fill 48 KB of shared memory
cudaError_t launch_q8_quantize(const uint16_t* W, int64_t N, int64_t K, uint8_t* codes, uint16_t* scales,
                               uint16_t* biases, cudaStream_t stream, const DeviceInfo& dev);
cudaError_t launch_q8_dequantize(const uint8_t* codes, const uint16_t* scales, const uint16_t* biases, int64_t N,
                                 int64_t K, uint16_t* W_out, cudaStream_t stream, const DeviceInfo& dev);
cudaError_t launch_q8_matmul(const MatmulArgs& a, cudaStream_t stream, const DeviceInfo& dev);

// CUDA-core GEMV family, any M (activation rows in chunks of at most two;
// every chunk re-reads the weights).
cudaError_t launch_gemv(const MatmulArgs& a, cudaStream_t stream, const DeviceInfo& dev);
// Several independent matmuls; those the bulk-copy kernel takes share one
// launch (per chunk size).
cudaError_t launch_gemv_batch(const MatmulArgs* list, int count, cudaStream_t stream, const DeviceInfo& dev);
// 8-bit codes (q8_matmul, q8_matmul_batch) on the same bulk-copy GEMV:
// whether it takes a problem (no epilogue, K a multiple of 256, 16-byte
// aligned scale rows), and the launch of a list of such problems (activation
// rows in pairs; all pairs of one size share a launch of up to 256).
bool gemv8_supported(const MatmulArgs& a);
cudaError_t launch_gemv8_batch(const MatmulArgs* list, int count, cudaStream_t stream, const DeviceInfo& dev);
// A chain of dependent stages in one persistent launch (q4_matmul_chain):
// whether it takes `list` (one or two activation rows, every problem on the
// bulk-copy path), and the launch itself -- stage s is the next
// stage_counts[s] problems of `list`; done: n_stages counters, zero.
constexpr int kGemvChainMaxProblems = 256, kGemvChainMaxStages = 256;
bool gemv_chain_supported(const MatmulArgs* list, int count);
cudaError_t launch_gemv_chain(const MatmulArgs* list, int count, const int* stage_counts, int n_stages,
                              unsigned int* done, cudaStream_t stream, const DeviceInfo& dev);

// Tensor-core tiles (tcgen05, dequantized weights in tensor memory) for
// three or more activation rows (from kTensorCoreMinRows, or where the
// weight-streaming kernel does not take a problem).  One launch per problem;
// plan_tc does every host-side step (tensor-map encoding, configuration
// checks), so a call can plan all its problems before launching any.
constexpr int64_t kTensorCoreMinRows = 3;
bool tc_supported(const MatmulArgs& a);
struct TcParams {
  const uint16_t* scales;     // [N, K/32] (the gate's, for SwiGLU)
  const uint16_t* biases;
  const uint16_t* up_scales;  // SwiGLU: the up weight's; else NULL
  const uint16_t* up_biases;
  uint16_t* y;                // [M, N]
  const uint16_t* r;          // residual [M, N] (kEpiResidual), else NULL
  int64_t M, N;
  int K;
  int epi;                    // kEpiNone / kEpiResidual (SwiGLU: nacc == 2)
  int bn;                     // activation rows per tile (multiple of 16, <= 256)
  int nacc;                   // accumulators: 1, or 2 for SwiGLU (gate, up)
  int splits;                 // CTAs per cluster along K
  int stages;
  int a_slots;                // A ring slots in tensor memory
  uint32_t stage_bytes, b_atom_bytes;
  uint32_t a_col0;            // first tensor-memory column of the A ring
  uint32_t idesc;             // tcgen05 instruction descriptor
};
struct TcLaunch {
  CUtensorMap tmap_x, tmap_codes, tmap_up;
  TcParams p;
  dim3 grid;
  size_t smem;
  int atoms;  // 64-wide K atoms per pipeline stage
};
cudaError_t plan_tc(const MatmulArgs& a, const DeviceInfo& dev, TcLaunch* out);
cudaError_t launch_planned_tc(const TcLaunch& plan, cudaStream_t stream);

// Tensor-core weight streaming (tcgen05, A operand in tensor memory, segmented
// K) for kStreamMinRows..kStreamMaxRows activation rows; several problems share
// one launch.
constexpr int kStreamMinRows = 3, kStreamMaxRows = 8;
bool stream_supported(const MatmulArgs& a, const DeviceInfo& dev);
cudaError_t launch_stream_batch(const MatmulArgs* list, int count, cudaStream_t stream, const DeviceInfo& dev);

// Group-sum tensor-core kernel (q4_gmma.cu: tcgen05 sums of 128 + q per
// group, scales and biases applied in fp32) for kGmmaMinRows..kGmmaMaxRows
// activation rows (1 and 2 rows stay on the CUDA-core GEMV, which is faster
// there); a launch takes many problems of one M.  plan_gmma encodes every
// tensor map (and may fail) before anything is launched.
constexpr int64_t kGmmaMinRows = 3, kGmmaMaxRows = 16;
// A launch balances the steps (128 inputs of a 128-row tile) over all SMs;
// a tile that two or more CTAs share needs a workspace: counter_bytes of
// arrival counters (zero at launch) and partial_bytes of fp32 partial sums.
constexpr size_t kGmmaParamBytes = 32768;
struct GmmaPlan {
  alignas(64) unsigned char params[kGmmaParamBytes];  // the kernel's parameter block
  int grid;
  size_t smem;
  const void* kern;
  size_t counter_bytes, partial_bytes;  // both 0: no tile is shared
};
bool gmma_supported(const MatmulArgs& a, const DeviceInfo& dev);
cudaError_t plan_gmma(const MatmulArgs* list, int count, const DeviceInfo& dev, std::vector<GmmaPlan>& plans);
// counters / partials: the plan's workspace (NULL when its sizes are 0).
cudaError_t launch_planned_gmma(GmmaPlan& plan, unsigned int* counters, float* partials, cudaStream_t stream);

// One-time settings of a device's kernels (dynamic shared memory, cluster
// sizes), made before the first launch on the device.
cudaError_t gemv_prepare_device(const DeviceInfo& dev);
cudaError_t tc_prepare_device(const DeviceInfo& dev);
cudaError_t stream_prepare_device(const DeviceInfo& dev);
cudaError_t q8_prepare_device(const DeviceInfo& dev);
cudaError_t gmma_prepare_device(const DeviceInfo& dev);

// Counts every kernel launch libq4 enqueues (host side).
void count_launch();

// Diagnostics: the bounded-wait flags of each kernel family (synchronous copies).
cudaError_t gemv_device_flags(unsigned int* flags, bool clear);
cudaError_t tc_device_flags(unsigned int* flags, bool clear);
cudaError_t stream_device_flags(unsigned int* flags, bool clear);
cudaError_t gmma_device_flags(unsigned int* flags, bool clear);

}  // namespace q4
