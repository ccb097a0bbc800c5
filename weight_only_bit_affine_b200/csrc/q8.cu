// q8.cu -- the 8-bit variant of the affine group-32 format: quantize,
// dequantize and matmul.
//
// Same rule as the 4-bit format with 255 levels (the pages compare a
// "standard 8-bit conversion" of the model -- TWX4 comparison page, opening
// section -- and ship an INT8 bundle -- ONNX README, "All four variants" --
// without stating its arithmetic): scale = bf16(fp32(max - min) / 255),
// bias = bf16(min), code = nearest-even of (w - bias) / scale in binary64,
// clamped to 0..255; one byte per code, codes [N, K]; scales and biases
// [N, K/32] bf16; w_hat = scale * q + bias.
//
// The matmul runs on the bulk-copy GEMV of q4_gemv.cu (8-bit rows: a lane's
// 32 codes become exact fp32 values meeting its x pairs in packed fp32 FMAs)
// where that kernel takes the problem (K a multiple of 256, 16-byte aligned
// scale rows); otherwise on the kernel below, a CUDA-core GEMV (one warp per
// weight row, lanes over the row's groups; activation rows in chunks of two).  At 1.125 bytes per weight
// an HBM-bound pass needs 1.8x fewer weights per second than the 4-bit one,
// so the arithmetic per weight can be heavier: each code becomes an exact
// fp32 (the byte under the exponent of 2^23, minus 2^23) and meets an fp32
// x in an FFMA; the bias term uses the group's sum of x, computed once per
// block into shared memory:  y = sum_g ( s * sum x q  +  b * sum x ).
#include "q4_device.cuh"
#include "q4_internal.h"

#include <algorithm>

namespace q4 {

namespace {

__global__ void __launch_bounds__(256) q8_quantize_kernel(const uint4* __restrict__ W, int64_t groups,
                                                          uint4* __restrict__ codes,
                                                          uint16_t* __restrict__ scales,
                                                          uint16_t* __restrict__ biases) {
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t f = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; f < groups; f += stride) {
    float w[32];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const uint4 v = W[4 * f + c];
      const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        w[8 * c + 2 * j] = __uint_as_float(u[j] << 16);
        w[8 * c + 2 * j + 1] = __uint_as_float(u[j] & 0xFFFF0000u);
      }
    }
    // the first minimal and the first maximal element in scan order
    float mn = w[0], mx = w[0];
#pragma unroll
    for (int i = 1; i < 32; ++i) {
      if (w[i] < mn) mn = w[i];
      if (w[i] > mx) mx = w[i];
    }
    const float s32 = __fdiv_rn(__fsub_rn(mx, mn), 255.0f);
    const __nv_bfloat16 s_bf = __float2bfloat16_rn(s32);
    const __nv_bfloat16 b_bf = __float2bfloat16_rn(mn);  // exact: mn is a bf16 value
    const double s = static_cast<double>(__bfloat162float(s_bf));
    const double b = static_cast<double>(mn);
    uint32_t packed[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      uint32_t q = 0;
      if (s != 0.0) {
        double t = rint(__ddiv_rn(__dsub_rn(static_cast<double>(w[i]), b), s));
        t = fmin(fmax(t, 0.0), 255.0);
        q = static_cast<uint32_t>(t);
      }
      packed[i >> 2] |= q << (8 * (i & 3));
    }
    codes[2 * f] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
    codes[2 * f + 1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
    scales[f] = __bfloat16_as_ushort(s_bf);
    biases[f] = __bfloat16_as_ushort(b_bf);
  }
}

__global__ void __launch_bounds__(256) q8_dequantize_kernel(const uint4* __restrict__ codes,
                                                            const uint16_t* __restrict__ scales,
                                                            const uint16_t* __restrict__ biases,
                                                            int64_t groups, uint4* __restrict__ W_out) {
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t f = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; f < groups; f += stride) {
    const double s = static_cast<double>(bf16_bits_to_float(scales[f]));
    const double b = static_cast<double>(bf16_bits_to_float(biases[f]));
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const uint4 c = codes[2 * f + half];
      const uint32_t words[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
      for (int wd = 0; wd < 4; ++wd) {  // 4 codes -> 4 bf16 = 8 bytes
        uint16_t h[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const uint32_t q = (words[wd] >> (8 * e)) & 0xFFu;
          h[e] = __bfloat16_as_ushort(__double2bfloat16(__dadd_rn(__dmul_rn(s, static_cast<double>(q)), b)));
        }
        const uint32_t lo = static_cast<uint32_t>(h[0]) | (static_cast<uint32_t>(h[1]) << 16);
        const uint32_t hi = static_cast<uint32_t>(h[2]) | (static_cast<uint32_t>(h[3]) << 16);
        reinterpret_cast<uint2*>(W_out)[8 * f + 4 * half + wd] = make_uint2(lo, hi);
      }
    }
  }
}

struct Q8Params {
  const uint16_t* x;  // [MR, K] (this chunk's activation rows)
  const uint8_t* codes;
  const uint16_t* scales;
  const uint16_t* biases;
  uint16_t* y;  // [MR, y_ld]
  int64_t N, y_ld;
  int K, G;
};

// q as an exact fp32: the byte under the exponent of 2^23 is 2^23 + q.
__device__ __forceinline__ float code_f32(uint32_t word, uint32_t sel) {
  return __uint_as_float(__byte_perm(word, 0x4B000000u, sel)) - 8388608.0f;
}

template <int MR>
__global__ void __launch_bounds__(256) q8_gemv_kernel(const __grid_constant__ Q8Params p) {
  extern __shared__ float xsum[];  // [MR][G]: per group sum of x
  pdl_launch_dependents();
  pdl_wait_predecessors();
  for (int i = threadIdx.x; i < MR * p.G; i += blockDim.x) {
    const int m = i / p.G, g = i - m * p.G;
    const uint4* xg = reinterpret_cast<const uint4*>(p.x + static_cast<int64_t>(m) * p.K + 32 * g);
    float t = 0.f;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const uint4 v = xg[c];
      const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) t += __uint_as_float(u[j] << 16) + __uint_as_float(u[j] & 0xFFFF0000u);
    }
    xsum[i] = t;
  }
  __syncthreads();

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t warps_total = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t row = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + warp; row < p.N; row += warps_total) {
    float acc[MR];
#pragma unroll
    for (int m = 0; m < MR; ++m) acc[m] = 0.f;
    const uint8_t* crow = p.codes + row * p.K;
    for (int g = lane; g < p.G; g += 32) {
      const uint4 c0 = ld_nc_v4(crow + 32 * g), c1 = ld_nc_v4(crow + 32 * g + 16);
      const uint32_t words[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
      const float s = bf16_bits_to_float(p.scales[row * p.G + g]);
      const float b = bf16_bits_to_float(p.biases[row * p.G + g]);
#pragma unroll
      for (int m = 0; m < MR; ++m) {
        const uint4* xg = reinterpret_cast<const uint4*>(p.x + static_cast<int64_t>(m) * p.K + 32 * g);
        float d0 = 0.f, d1 = 0.f;
#pragma unroll
        for (int c = 0; c < 4; ++c) {  // 8 inputs: two code words, four x pairs
          const uint4 v = __ldg(xg + c);
          const uint32_t xp[4] = {v.x, v.y, v.z, v.w};
          const uint32_t w0 = words[2 * c], w1 = words[2 * c + 1];
          d0 = fmaf(__uint_as_float(xp[0] << 16), code_f32(w0, 0x7540u), d0);
          d1 = fmaf(__uint_as_float(xp[0] & 0xFFFF0000u), code_f32(w0, 0x7541u), d1);
          d0 = fmaf(__uint_as_float(xp[1] << 16), code_f32(w0, 0x7542u), d0);
          d1 = fmaf(__uint_as_float(xp[1] & 0xFFFF0000u), code_f32(w0, 0x7543u), d1);
          d0 = fmaf(__uint_as_float(xp[2] << 16), code_f32(w1, 0x7540u), d0);
          d1 = fmaf(__uint_as_float(xp[2] & 0xFFFF0000u), code_f32(w1, 0x7541u), d1);
          d0 = fmaf(__uint_as_float(xp[3] << 16), code_f32(w1, 0x7542u), d0);
          d1 = fmaf(__uint_as_float(xp[3] & 0xFFFF0000u), code_f32(w1, 0x7543u), d1);
        }
        acc[m] = fmaf(s, d0 + d1, fmaf(b, xsum[m * p.G + g], acc[m]));
      }
    }
#pragma unroll
    for (int m = 0; m < MR; ++m) {
      float v = acc[m];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
      if (lane == 0) p.y[static_cast<int64_t>(m) * p.y_ld + row] = float_to_bf16_bits(v);
    }
  }
}

int grid_for(int64_t groups, const DeviceInfo& dev) {
  const int64_t blocks = (groups + 255) / 256;
  return static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(blocks, int64_t(dev.sm_count) * 8)));
}

template <int MR>
cudaError_t run_q8_gemv(const MatmulArgs& a, int64_t m0, const DeviceInfo& dev, cudaStream_t stream) {
  Q8Params p;
  p.x = a.x + m0 * a.K;
  p.codes = a.codes;
  p.scales = a.scales;
  p.biases = a.biases;
  p.y = a.y + m0 * a.N;
  p.N = a.N;
  p.y_ld = a.N;
  p.K = static_cast<int>(a.K);
  p.G = static_cast<int>(a.K / 32);
  const size_t smem = sizeof(float) * MR * p.G;
  const int64_t blocks = (a.N + 7) / 8;  // 8 warps = 8 rows per block per pass
  const int grid = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(blocks, int64_t(dev.sm_count) * 8)));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  count_launch();
  return cudaLaunchKernelEx(&cfg, q8_gemv_kernel<MR>, p);
}

}  // namespace

// The 8-bit kernels need no per-device settings (at most 48 KB of shared memory).
cudaError_t q8_prepare_device(const DeviceInfo&) { return cudaSuccess; }

cudaError_t launch_q8_quantize(const uint16_t* W, int64_t N, int64_t K, uint8_t* codes, uint16_t* scales,
                               uint16_t* biases, cudaStream_t stream, const DeviceInfo& dev) {
  const int64_t groups = N * (K / 32);
  count_launch();
  q8_quantize_kernel<<<grid_for(groups, dev), 256, 0, stream>>>(reinterpret_cast<const uint4*>(W), groups,
                                                                reinterpret_cast<uint4*>(codes), scales, biases);
  return cudaGetLastError();
}

cudaError_t launch_q8_dequantize(const uint8_t* codes, const uint16_t* scales, const uint16_t* biases, int64_t N,
                                 int64_t K, uint16_t* W_out, cudaStream_t stream, const DeviceInfo& dev) {
  const int64_t groups = N * (K / 32);
  count_launch();
  q8_dequantize_kernel<<<grid_for(groups, dev), 256, 0, stream>>>(
      reinterpret_cast<const uint4*>(codes), scales, biases, groups, reinterpret_cast<uint4*>(W_out));
  return cudaGetLastError();
}

cudaError_t launch_q8_matmul(const MatmulArgs& a, cudaStream_t stream, const DeviceInfo& dev) {
  // The bulk-copy GEMV (q4_gemv.cu, 8-bit rows) where it takes the problem;
  // this file's warp-per-row kernel otherwise.
  if (gemv8_supported(a)) return launch_gemv8_batch(&a, 1, stream, dev);
  for (int64_t m0 = 0; m0 < a.M; m0 += 2) {
    const cudaError_t e = (a.M - m0 >= 2) ? run_q8_gemv<2>(a, m0, dev, stream) : run_q8_gemv<1>(a, m0, dev, stream);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace q4
