// q4_quant.cu -- affine 4-bit group-32 quantize and dequantize kernels.
//
// The format is the model card "personaplex-edge-q4" ("Release details":
// affine Q4, group size 32, BF16), with the arithmetic read plainly:
// scale = bf16(fp32(max - min) / 15), bias = bf16(min), code = nearest-even
// of (w - bias) / scale in binary64, clamped to 0..15.  Reconstruction for
// validation ("Conversion and weight validation") is bf16(scale*q + bias).
//
// Rows are contiguous and every row holds K/32 whole groups, so the packed
// tensors are flat arrays of groups: group f = n*(K/32) + g owns 32 weights
// at W + 32f, 16 code bytes at codes + 16f, and scales[f], biases[f].  One
// thread handles one group; both kernels are bandwidth-trivial (offline and
// validation paths) and favour exact, order-identical arithmetic.
#include "q4_device.cuh"
#include "q4_internal.h"

#include <algorithm>

namespace q4 {

namespace {

__device__ __forceinline__ void unpack8_bf16(uint32_t lo_pair, float* out) {
  out[0] = __uint_as_float(lo_pair << 16);
  out[1] = __uint_as_float(lo_pair & 0xFFFF0000u);
}

__global__ void __launch_bounds__(256) quantize_kernel(const uint4* __restrict__ W, int64_t groups,
                                                       uint4* __restrict__ codes,
                                                       uint16_t* __restrict__ scales,
                                                       uint16_t* __restrict__ biases) {
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t f = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; f < groups; f += stride) {
    float w[32];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const uint4 v = W[4 * f + c];
      unpack8_bf16(v.x, w + 8 * c + 0);
      unpack8_bf16(v.y, w + 8 * c + 2);
      unpack8_bf16(v.z, w + 8 * c + 4);
      unpack8_bf16(v.w, w + 8 * c + 6);
    }
    // Same scan order and comparisons as a plain loop: the first minimal and
    // the first maximal element win (matters only for -0 vs +0).
    float mn = w[0], mx = w[0];
#pragma unroll
    for (int i = 1; i < 32; ++i) {
      if (w[i] < mn) mn = w[i];
      if (w[i] > mx) mx = w[i];
    }
    const float s32 = __fdiv_rn(__fsub_rn(mx, mn), 15.0f);
    const __nv_bfloat16 s_bf = __float2bfloat16_rn(s32);
    const __nv_bfloat16 b_bf = __float2bfloat16_rn(mn);  // exact: mn is a bf16 value
    const double s = static_cast<double>(__bfloat162float(s_bf));
    const double b = static_cast<double>(mn);
    uint32_t packed[4] = {0u, 0u, 0u, 0u};
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      uint32_t q = 0;
      if (s != 0.0) {
        double t = rint(__ddiv_rn(__dsub_rn(static_cast<double>(w[i]), b), s));
        t = fmin(fmax(t, 0.0), 15.0);
        q = static_cast<uint32_t>(t);
      }
      packed[i >> 3] |= q << (4 * (i & 7));
    }
    codes[f] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
    scales[f] = __bfloat16_as_ushort(s_bf);
    biases[f] = __bfloat16_as_ushort(b_bf);
  }
}

__global__ void __launch_bounds__(256) dequantize_kernel(const uint4* __restrict__ codes,
                                                         const uint16_t* __restrict__ scales,
                                                         const uint16_t* __restrict__ biases,
                                                         int64_t groups, uint4* __restrict__ W_out) {
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t f = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; f < groups; f += stride) {
    const uint4 c = codes[f];
    const uint32_t words[4] = {c.x, c.y, c.z, c.w};
    const double s = static_cast<double>(bf16_bits_to_float(scales[f]));
    const double b = static_cast<double>(bf16_bits_to_float(biases[f]));
#pragma unroll
    for (int wd = 0; wd < 4; ++wd) {
      uint32_t out[4];
#pragma unroll
      for (int p = 0; p < 4; ++p) {
        uint16_t h[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const uint32_t q = (words[wd] >> (4 * (2 * p + e))) & 0xFu;
          const double v = __dadd_rn(__dmul_rn(s, static_cast<double>(q)), b);
          h[e] = __bfloat16_as_ushort(__double2bfloat16(v));
        }
        out[p] = static_cast<uint32_t>(h[0]) | (static_cast<uint32_t>(h[1]) << 16);
      }
      W_out[4 * f + wd] = make_uint4(out[0], out[1], out[2], out[3]);
    }
  }
}

int grid_for(int64_t groups, const DeviceInfo& dev) {
  const int64_t blocks = (groups + 255) / 256;
  return static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(blocks, int64_t(dev.sm_count) * 8)));
}

}  // namespace

cudaError_t launch_quantize(const uint16_t* W, int64_t N, int64_t K, uint8_t* codes, uint16_t* scales,
                            uint16_t* biases, cudaStream_t stream, const DeviceInfo& dev) {
  const int64_t groups = N * (K / 32);
  count_launch();
  quantize_kernel<<<grid_for(groups, dev), 256, 0, stream>>>(reinterpret_cast<const uint4*>(W), groups,
                                                             reinterpret_cast<uint4*>(codes), scales, biases);
  return cudaGetLastError();
}

cudaError_t launch_dequantize(const uint8_t* codes, const uint16_t* scales, const uint16_t* biases,
                              int64_t N, int64_t K, uint16_t* W_out, cudaStream_t stream,
                              const DeviceInfo& dev) {
  const int64_t groups = N * (K / 32);
  count_launch();
  dequantize_kernel<<<grid_for(groups, dev), 256, 0, stream>>>(
      reinterpret_cast<const uint4*>(codes), scales, biases, groups, reinterpret_cast<uint4*>(W_out));
  return cudaGetLastError();
}

}  // namespace q4
