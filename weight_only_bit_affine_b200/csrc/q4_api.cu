// q4_api.cu -- the extern "C" boundary of libq4 (declared in include/q4.h):
// argument validation on the host, device checks, dispatch to the kernels.
// Nothing throws across the boundary; a non-OK status from validation means
// nothing was enqueued on the stream.
#include "q4.h"
#include "q4_internal.h"

#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <mutex>
#include <algorithm>
#include <vector>

namespace q4 {
namespace {

thread_local char t_last_error[512] = "";

q4_status fail(q4_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(t_last_error, sizeof t_last_error, fmt, ap);
  va_end(ap);
  return st;
}

std::atomic<unsigned long long> g_launches{0};
std::atomic<unsigned int> g_disabled_kernels{0};  // q4_debug_disable_kernels

// Scratch for q4_matmul_batch_noalloc: the group-sum kernel's workspace
// (arrival counters, then fp32 partial sums) in a fixed device array instead
// of a stream-ordered allocation.  One array per device, shared by every
// such call on it.
constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];
std::mutex g_scratch_mutex;
void* g_scratch_addr[64] = {};  // per device ordinal, from cudaGetSymbolAddress (once per device)

// The scratch array's device address on the current device (dev.device).
cudaError_t noalloc_scratch(const DeviceInfo& dev, unsigned char** out) {
  if (dev.device < 0 || dev.device >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (g_scratch_addr[dev.device] == nullptr) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev.device] = p;
  }
  *out = static_cast<unsigned char*>(g_scratch_addr[dev.device]);
  return cudaSuccess;
}

constexpr int kMaxDevices = 64;
DeviceInfo g_devices[kMaxDevices];
std::atomic<bool> g_device_ready[kMaxDevices];
std::mutex g_device_mutex;

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

// Common checks of the current device.  Returns Q4_OK with *out set.
q4_status check_device(const DeviceInfo** out) {
  const DeviceInfo* d = current_device_info();
  if (!d) return Q4_ERR_CUDA;
  if (d->cc_major != 10 || d->cc_minor != 0)
    return fail(Q4_ERR_UNSUPPORTED, "device %d has compute capability %d.%d; libq4 is built for sm_100a (10.0)",
                d->device, d->cc_major, d->cc_minor);
  *out = d;
  return Q4_OK;
}

q4_status check_k_group(int64_t K, int group) {
  if (group != 32) return fail(Q4_ERR_UNSUPPORTED, "group size %d is not supported (only 32)", group);
  if (K < 32 || K % 32 != 0) return fail(Q4_ERR_SHAPE, "K = %lld must be a positive multiple of 32", (long long)K);
  return Q4_OK;
}

q4_status from_cuda(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return Q4_OK;
  return fail(Q4_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

// Host checks of one matmul; Q4_OK with *empty set when there is nothing to do.
q4_status check_matmul(const char* who, const uint16_t* x, int64_t M, int64_t K, const uint8_t* codes,
                       const uint16_t* scales, const uint16_t* biases, int64_t N, int group, const uint16_t* y,
                       bool* empty) {
  q4_status st = check_k_group(K, group);
  if (st != Q4_OK) return st;
  if (M < 0 || N < 0) return fail(Q4_ERR_SHAPE, "%s: negative size M = %lld, N = %lld", who, (long long)M, (long long)N);
  *empty = (M == 0 || N == 0);
  if (*empty) return Q4_OK;
  if (!x || !codes || !scales || !biases || !y) return fail(Q4_ERR_NULL, "%s: NULL pointer argument", who);
  if (!aligned(x, 16) || !aligned(codes, 16))
    return fail(Q4_ERR_ALIGN, "%s: x and codes must be 16-byte aligned", who);
  if (!aligned(scales, 2) || !aligned(biases, 2) || !aligned(y, 2))
    return fail(Q4_ERR_ALIGN, "%s: scales, biases and y must be 2-byte aligned", who);
  if (N > (int64_t(1) << 40) || M > (int64_t(1) << 31) || K > (int64_t(1) << 24))
    return fail(Q4_ERR_UNSUPPORTED, "%s: sizes beyond the supported range", who);
  return Q4_OK;
}

// Host checks of a problem's epilogue fields (q4.h, q4_epilogue); fills the
// epilogue part of *a.
q4_status check_epilogue(const char* who, int32_t epi, int32_t reserved, const uint16_t* r,
                         const uint8_t* up_codes, const uint16_t* up_scales, const uint16_t* up_biases,
                         MatmulArgs* a) {
  if (reserved != 0) return fail(Q4_ERR_UNSUPPORTED, "%s: reserved field must be 0", who);
  if (epi == Q4_EPI_NONE) return Q4_OK;
  if (epi == Q4_EPI_RESIDUAL) {
    if (!r) return fail(Q4_ERR_NULL, "%s: residual epilogue without its operand r", who);
    if (!aligned(r, 2)) return fail(Q4_ERR_ALIGN, "%s: r must be 2-byte aligned", who);
    const uintptr_t rb = reinterpret_cast<uintptr_t>(r), yb = reinterpret_cast<uintptr_t>(a->y);
    const uintptr_t bytes = static_cast<uintptr_t>(a->M) * static_cast<uintptr_t>(a->N) * 2u;
    if (rb != yb && rb < yb + bytes && yb < rb + bytes)
      return fail(Q4_ERR_SHAPE, "%s: r overlaps y without being y", who);
    a->epi = kEpiResidual;
    a->r = r;
    return Q4_OK;
  }
  if (epi == Q4_EPI_SWIGLU) {
    if (!up_codes || !up_scales || !up_biases) return fail(Q4_ERR_NULL, "%s: SwiGLU without its up weights", who);
    if (!aligned(up_codes, 16)) return fail(Q4_ERR_ALIGN, "%s: up codes must be 16-byte aligned", who);
    if (!aligned(up_scales, 2) || !aligned(up_biases, 2))
      return fail(Q4_ERR_ALIGN, "%s: up scales and biases must be 2-byte aligned", who);
    a->up_codes = up_codes;
    a->up_scales = up_scales;
    a->up_biases = up_biases;
    return Q4_OK;
  }
  return fail(Q4_ERR_UNSUPPORTED, "%s: unknown epilogue %d", who, static_cast<int>(epi));
}

// The launches of a validated, non-empty list.  Each problem takes the kernel
// it would take alone (so a batched result is bit-identical to the single
// call): the group-sum tensor-core kernel where it takes the problem (1..16
// activation rows), else the weight-streaming kernel (3..8 rows), else the
// tensor-core tiles (3 or more rows), else the CUDA-core GEMV.  Problems on
// the group-sum kernel, the bulk-copy GEMV and the weight-streaming kernel
// share launches per path; SwiGLU problems run in one pass on every path.
// Every host-side step that can fail for a valid call (tensor-map encoding,
// configuration checks) runs here, before the first launch.
struct ListPlan {
  std::vector<MatmulArgs> gemv, streamed;
  std::vector<TcLaunch> tc;
  std::vector<GmmaPlan> gm;
  size_t counter_bytes = 0, partial_bytes = 0;  // the group-sum launches' workspace
};

q4_status plan_problems(const std::vector<MatmulArgs>& list, const DeviceInfo& dev, const char* what,
                        ListPlan& pl) {
  std::vector<MatmulArgs> grouped;
  const unsigned int off = g_disabled_kernels.load(std::memory_order_relaxed);
  for (const MatmulArgs& a : list) {
    if (!(off & Q4_KERNEL_GROUP_SUM) && gmma_supported(a, dev)) {
      grouped.push_back(a);
    } else if (!(off & Q4_KERNEL_WEIGHT_STREAM) && stream_supported(a, dev)) {
      pl.streamed.push_back(a);
    } else if (!(off & Q4_KERNEL_TILES) && a.M >= kTensorCoreMinRows && tc_supported(a)) {
      pl.tc.emplace_back();
      const cudaError_t e = plan_tc(a, dev, &pl.tc.back());
      if (e != cudaSuccess) return from_cuda(e, what);
    } else {
      pl.gemv.push_back(a);
    }
  }
  if (!grouped.empty()) {
    const cudaError_t e = plan_gmma(grouped.data(), static_cast<int>(grouped.size()), dev, pl.gm);
    if (e != cudaSuccess) return from_cuda(e, what);
  }
  for (const GmmaPlan& g : pl.gm) {
    pl.counter_bytes += g.counter_bytes;
    pl.partial_bytes += g.partial_bytes;
  }
  return Q4_OK;
}

// Enqueues a plan's launches.  ws: the group-sum launches' workspace, its
// arrival counters zero ([0, counter_region) holds the counters, the partial
// sums start at counter_region); NULL when the plan needs none.  The launches
// leave every counter zero again, so one workspace serves a sequence of plans.
q4_status launch_plan(ListPlan& pl, const DeviceInfo& dev, cudaStream_t cs, const char* what, unsigned char* ws,
                      size_t counter_region) {
  q4_status st = Q4_OK;
  size_t co = 0, po = counter_region;
  for (GmmaPlan& g : pl.gm) {
    unsigned int* counters = g.counter_bytes ? reinterpret_cast<unsigned int*>(ws + co) : nullptr;
    float* partials = g.partial_bytes ? reinterpret_cast<float*>(ws + po) : nullptr;
    co += g.counter_bytes;
    po += g.partial_bytes;
    if ((st = from_cuda(launch_planned_gmma(g, counters, partials, cs), what)) != Q4_OK) return st;
  }
  for (const TcLaunch& t : pl.tc)
    if ((st = from_cuda(launch_planned_tc(t, cs), what)) != Q4_OK) return st;
  if (!pl.streamed.empty() &&
      (st = from_cuda(launch_stream_batch(pl.streamed.data(), static_cast<int>(pl.streamed.size()), cs, dev),
                      what)) != Q4_OK)
    return st;
  if (!pl.gemv.empty() &&
      (st = from_cuda(launch_gemv_batch(pl.gemv.data(), static_cast<int>(pl.gemv.size()), cs, dev), what)) != Q4_OK)
    return st;
  return Q4_OK;
}

// Plans and enqueues a list with its own workspace: a stream-ordered
// allocation (cudaMallocAsync, counters zeroed by cudaMemsetAsync, released
// by cudaFreeAsync), or with static_scratch the fixed array of
// q4_matmul_batch_noalloc.
q4_status run_problems(const std::vector<MatmulArgs>& list, const DeviceInfo& dev, cudaStream_t cs,
                       const char* what, bool static_scratch = false) {
  thread_local ListPlan pl;
  pl = ListPlan();
  q4_status st = plan_problems(list, dev, what, pl);
  if (st != Q4_OK) return st;
  const size_t cbytes = pl.counter_bytes, pbytes = pl.partial_bytes;
  unsigned char* ws = nullptr;
  if (cbytes + pbytes > 0 && static_scratch) {
    if (cbytes + pbytes > kNoAllocScratchBytes)
      return fail(Q4_ERR_UNSUPPORTED, "%s: the call needs %zu bytes of scratch, the fixed array holds %zu", what,
                  cbytes + pbytes, kNoAllocScratchBytes);
    cudaError_t e = noalloc_scratch(dev, &ws);
    if (e == cudaSuccess) e = cudaMemsetAsync(ws, 0, cbytes, cs);
    if (e != cudaSuccess) return from_cuda(e, what);
  } else if (cbytes + pbytes > 0) {
    cudaError_t e = cudaMallocAsync(reinterpret_cast<void**>(&ws), cbytes + pbytes, cs);
    if (e == cudaSuccess) e = cudaMemsetAsync(ws, 0, cbytes, cs);
    if (e != cudaSuccess) return from_cuda(e, what);
  }
  st = launch_plan(pl, dev, cs, what, ws, cbytes);
  if (ws != nullptr && !static_scratch) {
    const cudaError_t e = cudaFreeAsync(ws, cs);
    if (st == Q4_OK && e != cudaSuccess) st = from_cuda(e, what);
  }
  return st;
}

// One matmul with an epilogue (q4_matmul, q4_matmul_step, q4_matmul_residual,
// q4_matmul_swiglu).
q4_status matmul_impl(const char* who, const uint16_t* x, int64_t M, int64_t K, const uint8_t* codes,
                      const uint16_t* scales, const uint16_t* biases, int64_t N, int group, uint16_t* y,
                      int32_t epi, const uint16_t* r, const uint8_t* up_codes, const uint16_t* up_scales,
                      const uint16_t* up_biases, cudaStream_t stream) {
  bool empty = false;
  q4_status st = check_matmul(who, x, M, K, codes, scales, biases, N, group, y, &empty);
  if (st != Q4_OK || empty) return st;
  MatmulArgs a{x, codes, scales, biases, y, M, N, K};
  if ((st = check_epilogue(who, epi, 0, r, up_codes, up_scales, up_biases, &a)) != Q4_OK) return st;
  const DeviceInfo* dev = nullptr;
  if ((st = check_device(&dev)) != Q4_OK) return st;
  char what[64];
  snprintf(what, sizeof what, "%s launch", who);
  return run_problems(std::vector<MatmulArgs>{a}, *dev, stream, what);
}

}  // namespace

void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

const DeviceInfo* current_device_info() {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    fail(Q4_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
    return nullptr;
  }
  if (dev < 0 || dev >= kMaxDevices) {
    fail(Q4_ERR_UNSUPPORTED, "device ordinal %d out of range", dev);
    return nullptr;
  }
  if (g_device_ready[dev].load(std::memory_order_acquire)) return &g_devices[dev];
  std::lock_guard<std::mutex> lock(g_device_mutex);
  if (!g_device_ready[dev].load(std::memory_order_relaxed)) {
    DeviceInfo d;
    d.device = dev;
    int smem_optin = 0;
    if ((e = cudaDeviceGetAttribute(&d.sm_count, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess ||
        (e = cudaDeviceGetAttribute(&d.cc_major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess ||
        (e = cudaDeviceGetAttribute(&d.cc_minor, cudaDevAttrComputeCapabilityMinor, dev)) != cudaSuccess ||
        (e = cudaDeviceGetAttribute(&smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev)) != cudaSuccess) {
      fail(Q4_ERR_CUDA, "cudaDeviceGetAttribute: %s", cudaGetErrorString(e));
      return nullptr;
    }
    d.smem_optin = static_cast<size_t>(smem_optin);
    // The kernels' one-time settings on this device (only on the GPU they
    // are built for; check_device rejects any other before a launch).
    // cudaFuncSetAttribute applies to the current device, which is `dev`.
    if (d.cc_major == 10 && d.cc_minor == 0) {
      if ((e = gemv_prepare_device(d)) == cudaSuccess && (e = tc_prepare_device(d)) == cudaSuccess &&
          (e = stream_prepare_device(d)) == cudaSuccess && (e = gmma_prepare_device(d)) == cudaSuccess)
        e = q8_prepare_device(d);
      if (e != cudaSuccess) {
        fail(Q4_ERR_CUDA, "kernel attributes: %s", cudaGetErrorString(e));
        return nullptr;
      }
    }
    g_devices[dev] = d;
    g_device_ready[dev].store(true, std::memory_order_release);
  }
  return &g_devices[dev];
}

}  // namespace q4

using namespace q4;

extern "C" {

q4_status q4_quantize(const q4_bf16* W, int64_t N, int64_t K, int group, uint8_t* codes, q4_bf16* scales,
                      q4_bf16* biases, q4_stream_t stream) {
  q4_status st = check_k_group(K, group);
  if (st != Q4_OK) return st;
  if (N < 0) return fail(Q4_ERR_SHAPE, "negative N = %lld", (long long)N);
  if (N == 0) return Q4_OK;
  if (!W || !codes || !scales || !biases) return fail(Q4_ERR_NULL, "q4_quantize: NULL pointer argument");
  if (!aligned(W, 16) || !aligned(codes, 16))
    return fail(Q4_ERR_ALIGN, "q4_quantize: W and codes must be 16-byte aligned");
  if (!aligned(scales, 2) || !aligned(biases, 2))
    return fail(Q4_ERR_ALIGN, "q4_quantize: scales and biases must be 2-byte aligned");
  const DeviceInfo* dev = nullptr;
  if ((st = check_device(&dev)) != Q4_OK) return st;
  return from_cuda(launch_quantize(W, N, K, codes, scales, biases, reinterpret_cast<cudaStream_t>(stream), *dev),
                   "q4_quantize launch");
}

q4_status q4_dequantize(const uint8_t* codes, const q4_bf16* scales, const q4_bf16* biases, int64_t N, int64_t K,
                        int group, q4_bf16* W_out, q4_stream_t stream) {
  q4_status st = check_k_group(K, group);
  if (st != Q4_OK) return st;
  if (N < 0) return fail(Q4_ERR_SHAPE, "negative N = %lld", (long long)N);
  if (N == 0) return Q4_OK;
  if (!W_out || !codes || !scales || !biases) return fail(Q4_ERR_NULL, "q4_dequantize: NULL pointer argument");
  if (!aligned(W_out, 16) || !aligned(codes, 16))
    return fail(Q4_ERR_ALIGN, "q4_dequantize: W_out and codes must be 16-byte aligned");
  if (!aligned(scales, 2) || !aligned(biases, 2))
    return fail(Q4_ERR_ALIGN, "q4_dequantize: scales and biases must be 2-byte aligned");
  const DeviceInfo* dev = nullptr;
  if ((st = check_device(&dev)) != Q4_OK) return st;
  return from_cuda(
      launch_dequantize(codes, scales, biases, N, K, W_out, reinterpret_cast<cudaStream_t>(stream), *dev),
      "q4_dequantize launch");
}

q4_status q4_matmul(const q4_bf16* x, int64_t M, int64_t K, const uint8_t* codes, const q4_bf16* scales,
                    const q4_bf16* biases, int64_t N, int group, q4_bf16* y, q4_stream_t stream) {
  return matmul_impl("q4_matmul", x, M, K, codes, scales, biases, N, group, y, Q4_EPI_NONE, nullptr, nullptr,
                     nullptr, nullptr, reinterpret_cast<cudaStream_t>(stream));
}

q4_status q4_matmul_residual(const q4_bf16* x, int64_t M, int64_t K, const uint8_t* codes, const q4_bf16* scales,
                             const q4_bf16* biases, int64_t N, int group, const q4_bf16* r, q4_bf16* y,
                             q4_stream_t stream) {
  return matmul_impl("q4_matmul_residual", x, M, K, codes, scales, biases, N, group, y, Q4_EPI_RESIDUAL, r, nullptr,
                     nullptr, nullptr, reinterpret_cast<cudaStream_t>(stream));
}

q4_status q4_matmul_swiglu(const q4_bf16* x, int64_t M, int64_t K, const uint8_t* gate_codes,
                           const q4_bf16* gate_scales, const q4_bf16* gate_biases, const uint8_t* up_codes,
                           const q4_bf16* up_scales, const q4_bf16* up_biases, int64_t N, int group, q4_bf16* h,
                           q4_stream_t stream) {
  return matmul_impl("q4_matmul_swiglu", x, M, K, gate_codes, gate_scales, gate_biases, N, group, h, Q4_EPI_SWIGLU,
                     nullptr, up_codes, up_scales, up_biases, reinterpret_cast<cudaStream_t>(stream));
}

q4_status q4_matmul_step(const q4_bf16* x, int64_t M, int64_t K, const uint8_t* codes, const q4_bf16* scales,
                         const q4_bf16* biases, int64_t N, int64_t num_steps, int64_t step, int group, q4_bf16* y,
                         q4_stream_t stream) {
  q4_status st = check_k_group(K, group);
  if (st != Q4_OK) return st;
  if (num_steps < 1 || step < 0 || step >= num_steps)
    return fail(Q4_ERR_RANGE, "q4_matmul_step: step %lld outside [0, %lld)", (long long)step, (long long)num_steps);
  if (N < 0) return fail(Q4_ERR_SHAPE, "negative N = %lld", (long long)N);
  if (!codes || !scales || !biases) return fail(Q4_ERR_NULL, "q4_matmul_step: NULL pointer argument");
  const int64_t row0 = step * N;
  return matmul_impl("q4_matmul_step", x, M, K, codes + row0 * (K / 2), scales + row0 * (K / 32),
                     biases + row0 * (K / 32), N, group, y, Q4_EPI_NONE, nullptr, nullptr, nullptr, nullptr,
                     reinterpret_cast<cudaStream_t>(stream));
}

q4_status q4_matmul_chain(const q4_matmul_desc* descs, int count, const int* stage_counts, int n_stages, int64_t M,
                          int group, q4_stream_t stream) {
  if (count < 0 || n_stages < 0) return fail(Q4_ERR_SHAPE, "q4_matmul_chain: negative count or stage count");
  if (count == 0) return Q4_OK;
  if (!descs || !stage_counts) return fail(Q4_ERR_NULL, "q4_matmul_chain: NULL descriptor or stage array");
  int64_t sum = 0;
  for (int s = 0; s < n_stages; ++s) {
    if (stage_counts[s] < 0) return fail(Q4_ERR_SHAPE, "q4_matmul_chain: stage %d has a negative count", s);
    sum += stage_counts[s];
  }
  if (sum != count)
    return fail(Q4_ERR_SHAPE, "q4_matmul_chain: the stages hold %lld descriptors, count is %d", (long long)sum, count);
  // Validate every descriptor first (nothing is enqueued on failure); empty
  // problems and stages left empty drop out.
  std::vector<MatmulArgs> list;
  std::vector<int> stages;
  list.reserve(static_cast<size_t>(count));
  for (int s = 0, i = 0; s < n_stages; ++s) {
    int kept = 0;
    for (int k = 0; k < stage_counts[s]; ++k, ++i) {
      const q4_matmul_desc& d = descs[i];
      bool empty = false;
      char who[64];
      snprintf(who, sizeof who, "q4_matmul_chain[%d] (stage %d)", i, s);
      q4_status st = check_matmul(who, d.x, M, d.K, d.codes, d.scales, d.biases, d.N, group, d.y, &empty);
      if (st != Q4_OK) return st;
      MatmulArgs a{d.x, d.codes, d.scales, d.biases, d.y, M, d.N, d.K};
      if ((st = check_epilogue(who, d.epilogue, d.reserved, d.r, d.up_codes, d.up_scales, d.up_biases, &a)) != Q4_OK)
        return st;
      if (!empty) {
        list.push_back(a);
        ++kept;
      }
    }
    if (kept > 0) stages.push_back(kept);
  }
  if (list.empty()) return Q4_OK;
  const DeviceInfo* dev = nullptr;
  q4_status st;
  if ((st = check_device(&dev)) != Q4_OK) return st;
  const cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  const int n = static_cast<int>(stages.size());
  if (!gemv_chain_supported(list.data(), static_cast<int>(list.size()))) {
    // One batch launch (or set of launches) per stage, in order, every stage
    // planned first; the stages' group-sum launches share one workspace
    // (their counters return to zero after each launch), allocated and zeroed
    // once for the call.
    std::vector<ListPlan> plans(static_cast<size_t>(n));
    size_t cmax = 0, pmax = 0;
    for (int s = 0, i = 0; s < n; i += stages[s], ++s) {
      std::vector<MatmulArgs> part(list.begin() + i, list.begin() + i + stages[s]);
      if ((st = plan_problems(part, *dev, "q4_matmul_chain launch", plans[s])) != Q4_OK) return st;
      cmax = std::max(cmax, plans[s].counter_bytes);
      pmax = std::max(pmax, plans[s].partial_bytes);
    }
    unsigned char* ws = nullptr;
    if (cmax + pmax > 0) {
      cudaError_t e = cudaMallocAsync(reinterpret_cast<void**>(&ws), cmax + pmax, cs);
      if (e == cudaSuccess) e = cudaMemsetAsync(ws, 0, cmax, cs);
      if (e != cudaSuccess) return from_cuda(e, "q4_matmul_chain workspace");
    }
    for (int s = 0; s < n && st == Q4_OK; ++s) st = launch_plan(plans[s], *dev, cs, "q4_matmul_chain launch", ws, cmax);
    if (ws != nullptr) {
      const cudaError_t e = cudaFreeAsync(ws, cs);
      if (st == Q4_OK && e != cudaSuccess) st = from_cuda(e, "q4_matmul_chain workspace");
    }
    return st;
  }
  // Persistent launches, each over as many whole stages as its parameter
  // block holds, with one zeroed arrival counter per stage.
  unsigned int* done = nullptr;
  cudaError_t e = cudaMallocAsync(reinterpret_cast<void**>(&done), sizeof(unsigned int) * n, cs);
  if (e == cudaSuccess) e = cudaMemsetAsync(done, 0, sizeof(unsigned int) * n, cs);
  if (e != cudaSuccess) return from_cuda(e, "q4_matmul_chain workspace");
  for (int s = 0, i = 0; s < n && st == Q4_OK;) {
    int ns = 0, np = 0;
    while (s + ns < n && ns < kGemvChainMaxStages && np + stages[s + ns] <= kGemvChainMaxProblems) np += stages[s + ns++];
    if (ns == 0) {  // one stage of more problems than a launch holds: that stage as a batch
      std::vector<MatmulArgs> part(list.begin() + i, list.begin() + i + stages[s]);
      st = run_problems(part, *dev, cs, "q4_matmul_chain launch");
      i += stages[s++];
      continue;
    }
    st = from_cuda(launch_gemv_chain(list.data() + i, np, stages.data() + s, ns, done + s, cs, *dev),
                   "q4_matmul_chain launch");
    s += ns;
    i += np;
  }
  e = cudaFreeAsync(done, cs);
  if (st == Q4_OK && e != cudaSuccess) st = from_cuda(e, "q4_matmul_chain workspace");
  return st;
}

q4_status q4_matmul_batch(const q4_matmul_desc* descs, int count, int64_t M, int group, q4_stream_t stream) {
  if (count < 0) return fail(Q4_ERR_SHAPE, "q4_matmul_batch: negative count %d", count);
  if (count == 0) return Q4_OK;
  if (!descs) return fail(Q4_ERR_NULL, "q4_matmul_batch: NULL descriptor array");
  std::vector<MatmulArgs> list;
  list.reserve(static_cast<size_t>(count));
  for (int i = 0; i < count; ++i) {
    const q4_matmul_desc& d = descs[i];
    bool empty = false;
    char who[48];
    snprintf(who, sizeof who, "q4_matmul_batch[%d]", i);
    q4_status st = check_matmul(who, d.x, M, d.K, d.codes, d.scales, d.biases, d.N, group, d.y, &empty);
    if (st != Q4_OK) return st;
    MatmulArgs a{d.x, d.codes, d.scales, d.biases, d.y, M, d.N, d.K};
    if ((st = check_epilogue(who, d.epilogue, d.reserved, d.r, d.up_codes, d.up_scales, d.up_biases, &a)) != Q4_OK)
      return st;
    if (!empty) list.push_back(a);
  }
  if (list.empty()) return Q4_OK;
  const DeviceInfo* dev = nullptr;
  q4_status st;
  if ((st = check_device(&dev)) != Q4_OK) return st;
  return run_problems(list, *dev, reinterpret_cast<cudaStream_t>(stream), "q4_matmul_batch launch");
}

q4_status q4_matmul_batch_noalloc(const q4_matmul_desc* descs, int count, int64_t M, int group,
                                  q4_stream_t stream) {
  if (count < 0) return fail(Q4_ERR_SHAPE, "q4_matmul_batch_noalloc: negative count %d", count);
  if (count == 0) return Q4_OK;
  if (!descs) return fail(Q4_ERR_NULL, "q4_matmul_batch_noalloc: NULL descriptor array");
  std::vector<MatmulArgs> list;
  list.reserve(static_cast<size_t>(count));
  for (int i = 0; i < count; ++i) {
    const q4_matmul_desc& d = descs[i];
    bool empty = false;
    char who[56];
    snprintf(who, sizeof who, "q4_matmul_batch_noalloc[%d]", i);
    q4_status st = check_matmul(who, d.x, M, d.K, d.codes, d.scales, d.biases, d.N, group, d.y, &empty);
    if (st != Q4_OK) return st;
    MatmulArgs a{d.x, d.codes, d.scales, d.biases, d.y, M, d.N, d.K};
    if ((st = check_epilogue(who, d.epilogue, d.reserved, d.r, d.up_codes, d.up_scales, d.up_biases, &a)) != Q4_OK)
      return st;
    if (!empty) list.push_back(a);
  }
  if (list.empty()) return Q4_OK;
  const DeviceInfo* dev = nullptr;
  q4_status st;
  if ((st = check_device(&dev)) != Q4_OK) return st;
  return run_problems(list, *dev, reinterpret_cast<cudaStream_t>(stream), "q4_matmul_batch_noalloc launch", true);
}

// ---- the 8-bit variant (q8.cu) --------------------------------------------

q4_status q8_quantize(const q4_bf16* W, int64_t N, int64_t K, int group, uint8_t* codes, q4_bf16* scales,
                      q4_bf16* biases, q4_stream_t stream) {
  q4_status st = check_k_group(K, group);
  if (st != Q4_OK) return st;
  if (N < 0) return fail(Q4_ERR_SHAPE, "negative N = %lld", (long long)N);
  if (N == 0) return Q4_OK;
  if (!W || !codes || !scales || !biases) return fail(Q4_ERR_NULL, "q8_quantize: NULL pointer argument");
  if (!aligned(W, 16) || !aligned(codes, 16))
    return fail(Q4_ERR_ALIGN, "q8_quantize: W and codes must be 16-byte aligned");
  if (!aligned(scales, 2) || !aligned(biases, 2))
    return fail(Q4_ERR_ALIGN, "q8_quantize: scales and biases must be 2-byte aligned");
  const DeviceInfo* dev = nullptr;
  if ((st = check_device(&dev)) != Q4_OK) return st;
  return from_cuda(launch_q8_quantize(W, N, K, codes, scales, biases, reinterpret_cast<cudaStream_t>(stream), *dev),
                   "q8_quantize launch");
}

q4_status q8_dequantize(const uint8_t* codes, const q4_bf16* scales, const q4_bf16* biases, int64_t N, int64_t K,
                        int group, q4_bf16* W_out, q4_stream_t stream) {
  q4_status st = check_k_group(K, group);
  if (st != Q4_OK) return st;
  if (N < 0) return fail(Q4_ERR_SHAPE, "negative N = %lld", (long long)N);
  if (N == 0) return Q4_OK;
  if (!W_out || !codes || !scales || !biases) return fail(Q4_ERR_NULL, "q8_dequantize: NULL pointer argument");
  if (!aligned(W_out, 16) || !aligned(codes, 16))
    return fail(Q4_ERR_ALIGN, "q8_dequantize: W_out and codes must be 16-byte aligned");
  if (!aligned(scales, 2) || !aligned(biases, 2))
    return fail(Q4_ERR_ALIGN, "q8_dequantize: scales and biases must be 2-byte aligned");
  const DeviceInfo* dev = nullptr;
  if ((st = check_device(&dev)) != Q4_OK) return st;
  return from_cuda(
      launch_q8_dequantize(codes, scales, biases, N, K, W_out, reinterpret_cast<cudaStream_t>(stream), *dev),
      "q8_dequantize launch");
}

q4_status q8_matmul(const q4_bf16* x, int64_t M, int64_t K, const uint8_t* codes, const q4_bf16* scales,
                    const q4_bf16* biases, int64_t N, int group, q4_bf16* y, q4_stream_t stream) {
  bool empty = false;
  q4_status st = check_matmul("q8_matmul", x, M, K, codes, scales, biases, N, group, y, &empty);
  if (st != Q4_OK || empty) return st;
  if (K > kQ8MaxK) return fail(Q4_ERR_UNSUPPORTED, "q8_matmul: K = %lld above %lld", (long long)K, (long long)kQ8MaxK);
  const DeviceInfo* dev = nullptr;
  if ((st = check_device(&dev)) != Q4_OK) return st;
  MatmulArgs a{x, codes, scales, biases, y, M, N, K};
  return from_cuda(launch_q8_matmul(a, reinterpret_cast<cudaStream_t>(stream), *dev), "q8_matmul launch");
}

q4_status q8_matmul_batch(const q4_matmul_desc* descs, int count, int64_t M, int group, q4_stream_t stream) {
  if (count < 0) return fail(Q4_ERR_SHAPE, "q8_matmul_batch: negative count %d", count);
  if (count == 0) return Q4_OK;
  if (!descs) return fail(Q4_ERR_NULL, "q8_matmul_batch: NULL descriptor array");
  std::vector<MatmulArgs> fast, rest;
  for (int i = 0; i < count; ++i) {
    const q4_matmul_desc& d = descs[i];
    bool empty = false;
    char who[48];
    snprintf(who, sizeof who, "q8_matmul_batch[%d]", i);
    q4_status st = check_matmul(who, d.x, M, d.K, d.codes, d.scales, d.biases, d.N, group, d.y, &empty);
    if (st != Q4_OK) return st;
    if (d.epilogue != Q4_EPI_NONE || d.reserved != 0)
      return fail(Q4_ERR_UNSUPPORTED, "%s: 8-bit problems take no epilogue", who);
    if (d.K > kQ8MaxK)
      return fail(Q4_ERR_UNSUPPORTED, "%s: K = %lld above %lld", who, (long long)d.K, (long long)kQ8MaxK);
    if (empty) continue;
    const MatmulArgs a{d.x, d.codes, d.scales, d.biases, d.y, M, d.N, d.K};
    (gemv8_supported(a) ? fast : rest).push_back(a);
  }
  const DeviceInfo* dev = nullptr;
  q4_status st;
  if ((st = check_device(&dev)) != Q4_OK) return st;
  const cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  if (!fast.empty() &&
      (st = from_cuda(launch_gemv8_batch(fast.data(), static_cast<int>(fast.size()), cs, *dev),
                      "q8_matmul_batch launch")) != Q4_OK)
    return st;
  for (const MatmulArgs& a : rest)
    if ((st = from_cuda(launch_q8_matmul(a, cs, *dev), "q8_matmul_batch launch")) != Q4_OK) return st;
  return Q4_OK;
}

const char* q4_last_error(void) { return t_last_error; }

unsigned long long q4_debug_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

unsigned int q4_debug_disable_kernels(unsigned int mask) { return g_disabled_kernels.exchange(mask); }

int q4_device_status(int clear) {
  unsigned int f = 0, t = 0, s = 0, g = 0;
  if (gemv_device_flags(&f, clear != 0) != cudaSuccess || tc_device_flags(&t, clear != 0) != cudaSuccess ||
      stream_device_flags(&s, clear != 0) != cudaSuccess || gmma_device_flags(&g, clear != 0) != cudaSuccess)
    return -1;
  f |= t | s | g;
  return static_cast<int>(f);
}

}  // extern "C"
