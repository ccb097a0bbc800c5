// q4_gemv.cu -- the CUDA-core GEMV family of the affine Q4 group-32 matmul,
// for few activation rows (decode, M < 16):
//
//   y[m,n] = sum_g ( s[n,g] * sum_{k in g} x[m,k] q[n,k]  +  b[n,g] * sum_{k in g} x[m,k] )
//
// which is x . w_hat^T with w_hat = s*q + b (model card "personaplex-edge-q4":
// affine Q4, group size 32, the packed weights consumed directly by the
// matmul).  The weights are read once from HBM in packed form and never
// expanded in memory.
//
// Design (bandwidth-bound: ~1.6 flop per packed byte at M = 1):
//  * One persistent CTA per SM.  A producer warp streams tiles of `rt` whole
//    weight rows (codes, scales, biases: contiguous ranges) into a ring of
//    shared-memory stages with 1-D bulk (TMA) copies; the bytes in flight are
//    bounded by the ring, not by registers.
//  * Consumer threads form "teams" of K/KPL lanes; a team owns one weight row
//    at a time and lane j always covers the same KPL inputs k, so its slice of
//    x lives in registers for the whole kernel (the row reduction over K is
//    split across the team and finished with warp shuffles plus a
//    shared-memory step between the team's warps).
//  * Nibbles are unpacked in registers into bf16x2 values 128 + q (one LOP3
//    per two codes) and multiplied with bf16 x by fp32-accumulating FMAs; the
//    offset is removed per group exactly:  s*sum x(128+q) + (b - 128 s)*sum x.
//  * Programmatic dependent launch: each kernel lets the next one launch
//    early; before waiting for its predecessor the next kernel only issues L2
//    prefetches of its own weights (a hint with no effect on values), so the
//    weight stream of back-to-back matmuls keeps HBM busy across launches.
#include "q4_device.cuh"
#include "q4_internal.h"

#include <algorithm>

#ifndef Q4_GEMV_CTAS_PER_SM
#define Q4_GEMV_CTAS_PER_SM 1
#endif
#ifndef Q4_GEMV_SMEM_BUDGET
#define Q4_GEMV_SMEM_BUDGET (200 * 1024)
#endif
#ifndef Q4_GEMV_TARGET_THREADS
#define Q4_GEMV_TARGET_THREADS 512
#endif
#ifndef Q4_GEMV_MAC
#define Q4_GEMV_MAC 0
#endif

namespace q4 {

namespace {

// Inner-product variants (all exact products, fp32 accumulation):
//  kMacMixedBf16: bf16x2 "128 + q" unpack, fma.rn.f32.bf16 per weight;
//  kMacFfma2:     the same unpack widened to fp32 pairs, fma.rn.f32x2;
//  kMacMagicSub:  in-place fp32 unpack with exact offset removal
//                 (unpack_codes_f32), add/fma.rn.f32x2 on natural k pairs.
enum Mac { kMacMixedBf16 = 0, kMacFfma2 = 1, kMacMagicSub = 2 };
template <int MAC>
constexpr float mac_offset() { return MAC == kMacMagicSub ? 0.f : 128.f; }

struct TmaGemvParams {
  const uint16_t* x;       // [MR, K] (row stride K)
  const uint8_t* codes;    // [N, K/2]
  const uint16_t* scales;  // [N, G]
  const uint16_t* biases;  // [N, G]
  uint16_t* y;             // [MR, y_ld]
  int64_t N, y_ld;
  int K, G;
  int team;              // lanes per weight row (a multiple of 32, or a power of two below 32)
  int teams;             // teams per CTA
  int rt;                // rows per tile (= teams * RPT)
  int stages;
  int consumer_threads;  // teams * team (a multiple of 32)
  int chunk_tiles;       // tiles whose cross-warp partial sums are reduced together
  uint32_t codes_tile_bytes, sb_tile_bytes, stage_bytes;
};

template <int W>
__device__ __forceinline__ float seg_allreduce(float v) {
#pragma unroll
  for (int o = W / 2; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  return v;
}

__device__ __forceinline__ float seg_allreduce_dyn(float v, int width) {
  for (int o = width / 2; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  return v;
}

// x slice of one lane, per word w (8 inputs) and t = 0..3: the pair
// (x[8w + t], x[8w + t + 4]) matching the "128 + q" code pairs (bf16x2 for
// the mixed FMA, fp32 for FFMA2), or the natural pair (x[8w + 2t],
// x[8w + 2t + 1]) in fp32 for the in-place unpack.
template <int WORDS, int MAC>
struct XSlice {
  static constexpr int kRegs = (MAC == kMacMixedBf16) ? 1 : 2;
  uint32_t v[WORDS][4][kRegs];
  float sum;

  __device__ __forceinline__ void load(const uint16_t* src) {
    sum = 0.f;
#pragma unroll
    for (int w = 0; w < WORDS; ++w) {
      const uint4 e = *reinterpret_cast<const uint4*>(src + 8 * w);
      const uint32_t pr[4] = {__byte_perm(e.x, e.z, 0x5410), __byte_perm(e.x, e.z, 0x7632),
                              __byte_perm(e.y, e.w, 0x5410), __byte_perm(e.y, e.w, 0x7632)};
      const uint32_t nat[4] = {e.x, e.y, e.z, e.w};  // (x[8w+2t], x[8w+2t+1])
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        if constexpr (MAC == kMacMixedBf16) {
          v[w][t][0] = pr[t];
        } else if constexpr (MAC == kMacFfma2) {
          v[w][t][0] = pr[t] << 16;
          v[w][t][kRegs - 1] = pr[t] & 0xFFFF0000u;
        } else {
          v[w][t][0] = nat[t] << 16;
          v[w][t][kRegs - 1] = nat[t] & 0xFFFF0000u;
        }
        sum += __uint_as_float(pr[t] << 16) + __uint_as_float(pr[t] & 0xFFFF0000u);
      }
    }
  }
  __device__ __forceinline__ void zero() {
    sum = 0.f;
#pragma unroll
    for (int w = 0; w < WORDS; ++w)
#pragma unroll
      for (int t = 0; t < 4; ++t)
#pragma unroll
        for (int r = 0; r < kRegs; ++r) v[w][t][r] = 0u;
  }
};

// sum over the lane's inputs of x * (mac_offset + q), two partial accumulators.
template <int MR, int WORDS, int MAC>
__device__ __forceinline__ void dot_plus128(const uint32_t (&words)[WORDS], const XSlice<WORDS, MAC> (&xs)[MR],
                                            float (&a0)[MR], float (&a1)[MR]) {
  if constexpr (MAC == kMacMagicSub) {
#pragma unroll
    for (int w = 0; w < WORDS; ++w) {
      float q[8];
      unpack_codes_f32(words[w], q);
#pragma unroll
      for (int t = 0; t < 4; ++t)
#pragma unroll
        for (int m = 0; m < MR; ++m)
          ffma2(a0[m], a1[m], __uint_as_float(xs[m].v[w][t][0]), __uint_as_float(xs[m].v[w][t][1]), q[2 * t],
                q[2 * t + 1]);
    }
    return;
  }
  if constexpr (MAC == kMacMixedBf16) {
#pragma unroll
    for (int w = 0; w < WORDS; ++w)
#pragma unroll
      for (int m = 0; m < MR; ++m)
        word_dot_bf16(words[w], xs[m].v[w][0][0], xs[m].v[w][1][0], xs[m].v[w][2][0], xs[m].v[w][3][0], a0[m],
                      a1[m]);
    return;
  }
#pragma unroll
  for (int w = 0; w < WORDS; ++w) {
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const uint32_t v = nibbles_to_bf16x2_plus128(words[w], t);
      if constexpr (MAC == kMacMixedBf16) {
        (void)v;
      } else {
        const float lo = __uint_as_float(v << 16), hi = __uint_as_float(v & 0xFFFF0000u);
#pragma unroll
        for (int m = 0; m < MR; ++m)
          ffma2(a0[m], a1[m], __uint_as_float(xs[m].v[w][t][0]), __uint_as_float(xs[m].v[w][t][1]), lo, hi);
      }
    }
  }
}

template <int WORDS>
__device__ __forceinline__ void load_words_smem(const uint8_t* p, uint32_t (&words)[WORDS]) {
  if constexpr (WORDS == 4) {
    const uint4 v = *reinterpret_cast<const uint4*>(p);
    words[0] = v.x; words[1] = v.y; words[2] = v.z; words[3] = v.w;
  } else if constexpr (WORDS == 2) {
    const uint2 v = *reinterpret_cast<const uint2*>(p);
    words[0] = v.x; words[1] = v.y;
  } else {
    words[0] = *reinterpret_cast<const uint32_t*>(p);
  }
}

// Sum V values across the 32 lanes of a warp at once (V a power of two):
// after the call, lane l holds the total of value l >> (5 - log2 V).  Costs
// V - 1 + 5 - log2 V shuffles instead of 5 V.
template <int V>
__device__ __forceinline__ float transpose_reduce(float (&v)[V], int lane) {
  static_assert(V >= 1 && V <= 32 && (V & (V - 1)) == 0, "V must be a power of two <= 32");
  int o = 16;
#pragma unroll
  for (int cnt = V; cnt > 1; cnt >>= 1, o >>= 1) {
    const int half = cnt >> 1;
    const bool upper = (lane & o) != 0;
#pragma unroll
    for (int i = 0; i < half; ++i) {
      const float send = upper ? v[i] : v[i + half];
      const float keep = upper ? v[i + half] : v[i];
      v[i] = keep + __shfl_xor_sync(0xFFFFFFFFu, send, o);
    }
  }
  float r = v[0];
#pragma unroll
  for (; o > 0; o >>= 1) r += __shfl_xor_sync(0xFFFFFFFFu, r, o);
  return r;
}

constexpr int pow2_at_least(int v) { return v <= 1 ? 1 : 2 * pow2_at_least((v + 1) / 2); }
constexpr int ilog2(int v) { return v <= 1 ? 0 : 1 + ilog2(v / 2); }

__device__ __forceinline__ uint16_t to_bf16_bits(float v) { return __bfloat16_as_ushort(__float2bfloat16_rn(v)); }

template <int MR, int KPL, int RPT, int MAC, int MAXT>
__global__ void __launch_bounds__(MAXT, 1) gemv_tma_kernel(const __grid_constant__ TmaGemvParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  constexpr int WORDS = KPL / 8;
  constexpr int V = RPT * MR;
  constexpr int VP = pow2_at_least(V);
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int consumer_warps = p.consumer_threads >> 5;
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + static_cast<size_t>(p.stages) * p.stage_bytes);
  uint64_t* empty_bar = full_bar + p.stages;
  float* red = reinterpret_cast<float*>(empty_bar + p.stages);

  // This CTA's contiguous share of the weight rows (balanced to within one row).
  const int64_t r_begin = static_cast<int64_t>(blockIdx.x) * p.N / gridDim.x;
  const int64_t r_end = static_cast<int64_t>(blockIdx.x + 1) * p.N / gridDim.x;
  const int64_t cta_rows = r_end - r_begin;
  const int ntiles = static_cast<int>((cta_rows + p.rt - 1) / p.rt);

  if (tid == 0) {
    for (int s = 0; s < p.stages; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], consumer_warps);
    }
    fence_mbar_init();
  }
  __syncthreads();
  pdl_launch_dependents();

  const int half_k = p.K >> 1;
  if (warp == consumer_warps) {
    // ---------------- producer warp ----------------
    if (lane == 0) {
      // Warm L2 with the first tiles while the previous kernel may still run
      // (a prefetch is a hint: it changes no value any thread observes).
      for (int t = 0; t < ntiles && t < p.stages; ++t) {
        const int64_t row0 = r_begin + static_cast<int64_t>(t) * p.rt;
        const uint32_t rows = static_cast<uint32_t>((r_end - row0 < p.rt) ? (r_end - row0) : p.rt);
        bulk_prefetch_l2(p.codes + row0 * half_k, rows * half_k);
        bulk_prefetch_l2(p.scales + row0 * p.G, rows * p.G * 2);
        bulk_prefetch_l2(p.biases + row0 * p.G, rows * p.G * 2);
      }
    }
    pdl_wait_predecessors();
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;
      for (int t = 0; t < ntiles; ++t) {
        if (!mbar_wait(&empty_bar[stage], phase ^ 1u)) break;
        const int64_t row0 = r_begin + static_cast<int64_t>(t) * p.rt;
        const uint32_t rows = static_cast<uint32_t>((r_end - row0 < p.rt) ? (r_end - row0) : p.rt);
        const uint32_t cb = rows * half_k, sb = rows * p.G * 2;
        uint8_t* st = smem + static_cast<size_t>(stage) * p.stage_bytes;
        mbar_arrive_expect_tx(&full_bar[stage], cb + 2 * sb);
        bulk_g2s(st, p.codes + row0 * half_k, cb, &full_bar[stage]);
        bulk_g2s(st + p.codes_tile_bytes, p.scales + row0 * p.G, sb, &full_bar[stage]);
        bulk_g2s(st + p.codes_tile_bytes + p.sb_tile_bytes, p.biases + row0 * p.G, sb, &full_bar[stage]);
        ++issued;
        if (++stage == p.stages) { stage = 0; phase ^= 1u; }
      }
      // No copy may still target this CTA's shared memory when it exits: wait
      // (bounded) for the last issued tile of every stage.
      const int tail = min(issued, p.stages);
      for (int i = 0; i < tail; ++i) {
        int s = stage - 1 - i;
        uint32_t ph = phase;
        if (s < 0) { s += p.stages; ph ^= 1u; }
        mbar_wait(&full_bar[s], ph);
      }
    }
    return;
  }

  // ---------------- consumer threads ----------------
  const int team_idx = tid / p.team;
  const int j = tid - team_idx * p.team;
  const bool active = j < p.K / KPL;  // lanes past K own no inputs (padding)
  const int g = (j * KPL) >> 5;
  const int wpt = p.team >> 5;  // warps per team (0 when a warp holds several teams)
  const int warp_in_team = (p.team >= 32) ? (j >> 5) : 0;
  constexpr float kOffset = mac_offset<MAC>();

  pdl_wait_predecessors();

  XSlice<WORDS, MAC> xs[MR];
#pragma unroll
  for (int m = 0; m < MR; ++m) {
    if (active)
      xs[m].load(p.x + static_cast<int64_t>(m) * p.K + j * KPL);
    else
      xs[m].zero();
  }

  int stage = 0;
  uint32_t phase = 0;
  bool dead = false;
  for (int c0 = 0; c0 < ntiles; c0 += p.chunk_tiles) {
    const int c1 = min(ntiles, c0 + p.chunk_tiles);
    for (int t = c0; t < c1; ++t) {
      if (!dead && !mbar_wait(&full_bar[stage], phase)) dead = true;  // on timeout: finish without waiting
      const uint8_t* st = smem + static_cast<size_t>(stage) * p.stage_bytes;
      const uint16_t* ssc = reinterpret_cast<const uint16_t*>(st + p.codes_tile_bytes);
      const uint16_t* sbi = reinterpret_cast<const uint16_t*>(st + p.codes_tile_bytes + p.sb_tile_bytes);
      const int r_first = team_idx * RPT;                        // first row of this team in the tile
      const int64_t grow0 = r_begin + static_cast<int64_t>(t) * p.rt + r_first;

      float vals[VP];
#pragma unroll
      for (int i = 0; i < VP; ++i) vals[i] = 0.f;
      uint32_t words[RPT][WORDS];
      float sc[RPT], bi[RPT];
#pragma unroll
      for (int rr = 0; rr < RPT; ++rr) {  // issue all shared-memory loads first
        const int r = r_first + rr;
        if (active && grow0 + rr < r_end) {
          load_words_smem<WORDS>(st + static_cast<size_t>(r) * half_k + j * (KPL / 2), words[rr]);
          sc[rr] = bf16_bits_to_float(ssc[r * p.G + g]);
          bi[rr] = bf16_bits_to_float(sbi[r * p.G + g]);
        } else {
#pragma unroll
          for (int w = 0; w < WORDS; ++w) words[rr][w] = 0u;
          sc[rr] = bi[rr] = 0.f;
        }
      }
      // The stage's bytes are now in registers: hand it back to the producer.
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty_bar[stage]);
      if (++stage == p.stages) { stage = 0; phase ^= 1u; }

#pragma unroll
      for (int rr = 0; rr < RPT; ++rr) {
        float a0[MR], a1[MR];
#pragma unroll
        for (int m = 0; m < MR; ++m) a0[m] = a1[m] = 0.f;
        dot_plus128<MR, WORDS, MAC>(words[rr], xs, a0, a1);
        const float c = fmaf(-kOffset, sc[rr], bi[rr]);
#pragma unroll
        for (int m = 0; m < MR; ++m) vals[rr * MR + m] = fmaf(sc[rr], a0[m] + a1[m], c * xs[m].sum);
      }

      if (p.team >= 32) {
        const float tot = transpose_reduce<VP>(vals, lane);
        const int idx = lane >> (5 - ilog2(VP));
        const bool holder = (lane & ((32 / VP) - 1)) == 0 && idx < V;
        const int rr = idx / MR, m = idx % MR;
        if (holder && grow0 + rr < r_end) {
          if (wpt == 1) {
            p.y[static_cast<int64_t>(m) * p.y_ld + grow0 + rr] = to_bf16_bits(tot);
          } else {
            const int lr = (t - c0) * p.rt + r_first + rr;  // row within the chunk
            red[(lr * MR + m) * wpt + warp_in_team] = tot;
          }
        }
      } else {
#pragma unroll
        for (int i = 0; i < V; ++i) vals[i] = seg_allreduce_dyn(vals[i], p.team);
        if (j == 0) {
#pragma unroll
          for (int rr = 0; rr < RPT; ++rr)
            if (grow0 + rr < r_end) {
#pragma unroll
              for (int m = 0; m < MR; ++m)
                p.y[static_cast<int64_t>(m) * p.y_ld + grow0 + rr] = to_bf16_bits(vals[rr * MR + m]);
            }
        }
      }
    }
    if (wpt > 1) {
      // Cross-warp sums of this chunk's rows, once per chunk (consumers only).
      named_bar_sync(1, p.consumer_threads);
      const int64_t row_a = r_begin + static_cast<int64_t>(c0) * p.rt;
      const int64_t row_b = min(r_end, r_begin + static_cast<int64_t>(c1) * p.rt);
      const int n_out = static_cast<int>(row_b - row_a) * MR;
      for (int i = tid; i < n_out; i += p.consumer_threads) {
        const float* rp = red + i * wpt;
        float v = 0.f;
        for (int w = 0; w < wpt; ++w) v += rp[w];
        const int lr = i / MR, m = i - lr * MR;
        p.y[static_cast<int64_t>(m) * p.y_ld + row_a + lr] = to_bf16_bits(v);
      }
      named_bar_sync(1, p.consumer_threads);
    }
  }
}

// Generic path: any K, any 2-byte-aligned scales.  One warp per weight row,
// lanes stride over the row's groups; x is read through the L1 per group.
struct GenericParams {
  const uint16_t* x;
  const uint8_t* codes;
  const uint16_t* scales;
  const uint16_t* biases;
  uint16_t* y;
  int64_t N, y_ld;
  int K, G;
};

template <int MR>
__global__ void __launch_bounds__(256) gemv_generic_kernel(const __grid_constant__ GenericParams p) {
  pdl_launch_dependents();
  pdl_wait_predecessors();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t warps_total = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t row = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + warp; row < p.N; row += warps_total) {
    float acc[MR];
#pragma unroll
    for (int m = 0; m < MR; ++m) acc[m] = 0.f;
    for (int g = lane; g < p.G; g += 32) {
      const uint4 c4 = ld_nc_v4(p.codes + row * (p.K / 2) + static_cast<int64_t>(g) * 16);
      const uint32_t words[4] = {c4.x, c4.y, c4.z, c4.w};
      const float s = bf16_bits_to_float(p.scales[row * p.G + g]);
      const float b = bf16_bits_to_float(p.biases[row * p.G + g]);
      XSlice<4, kMacMixedBf16> xs[MR];
#pragma unroll
      for (int m = 0; m < MR; ++m) xs[m].load(p.x + static_cast<int64_t>(m) * p.K + g * 32);
      float a0[MR], a1[MR];
#pragma unroll
      for (int m = 0; m < MR; ++m) a0[m] = a1[m] = 0.f;
      dot_plus128<MR, 4, kMacMixedBf16>(words, xs, a0, a1);
      const float c = fmaf(-128.f, s, b);
#pragma unroll
      for (int m = 0; m < MR; ++m) acc[m] += fmaf(s, a0[m] + a1[m], c * xs[m].sum);
    }
#pragma unroll
    for (int m = 0; m < MR; ++m) {
      const float v = seg_allreduce<32>(acc[m]);
      if (lane == 0) p.y[static_cast<int64_t>(m) * p.y_ld + row] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
    }
  }
}

// ---------------------------------------------------------------- host side

template <typename Kern, typename Params>
cudaError_t launch_pdl(Kern kernel, dim3 grid, dim3 block, size_t smem, cudaStream_t stream, const Params& prm) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  count_launch();
  return cudaLaunchKernelEx(&cfg, kernel, prm);
}

constexpr int kKpl = 32;       // inputs per lane: one whole group (16 code bytes)
constexpr int kMaxRows = 4;    // activation rows per chunk (x slice: 16*MR registers)
constexpr int rpt_for(int mr) { return mr <= 2 ? 4 : 2; }  // weight rows per team per tile

template <int MR, int MAXT>
cudaError_t run_tma(const MatmulArgs& a, int64_t m0, const TmaGemvParams& base, size_t smem, int grid,
                    cudaStream_t stream) {
  TmaGemvParams p = base;
  p.x = a.x + m0 * a.K;
  p.y = a.y + m0 * a.N;
  auto kern = gemv_tma_kernel<MR, kKpl, rpt_for(MR), Q4_GEMV_MAC, MAXT>;
  static bool attr_set = false;  // per template instance; idempotent if raced
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  return launch_pdl(kern, dim3(grid), dim3(p.consumer_threads + 32), smem, stream, p);
}

template <int MR>
cudaError_t run_generic(const MatmulArgs& a, int64_t m0, const DeviceInfo& dev, cudaStream_t stream) {
  GenericParams p;
  p.x = a.x + m0 * a.K;
  p.codes = a.codes;
  p.scales = a.scales;
  p.biases = a.biases;
  p.y = a.y + m0 * a.N;
  p.N = a.N;
  p.y_ld = a.N;
  p.K = static_cast<int>(a.K);
  p.G = static_cast<int>(a.K / 32);
  const int64_t blocks = (a.N + 7) / 8;
  const int grid = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(blocks, int64_t(dev.sm_count) * 8)));
  return launch_pdl(gemv_generic_kernel<MR>, dim3(grid), dim3(256), 0, stream, p);
}

// Chooses the TMA kernel's shape for one chunk of `mr` activation rows.
// Returns false when the shape needs the generic kernel.
bool plan_tma(const MatmulArgs& a, int mr, const DeviceInfo& dev, TmaGemvParams& p, size_t& smem, int& grid) {
  const int64_t K = a.K, G = K / 32;
  if (G % 8 != 0) return false;  // scale rows must be whole 16-byte runs for bulk copies
  if ((reinterpret_cast<uintptr_t>(a.scales) | reinterpret_cast<uintptr_t>(a.biases)) & 15u) return false;
  const int64_t lanes = K / kKpl;
  int64_t team;
  if (lanes >= 32) {
    team = (lanes + 31) / 32 * 32;
  } else {
    team = 1;
    while (team < lanes) team <<= 1;
  }
  // Launch-bound instances: 384 and 640 threads, i.e. up to 170 and 102
  // registers per thread; only one activation row fits the 640-thread one
  // without spilling.
  const int max_consumers = (mr == 1) ? 608 : 352;
  if (team > max_consumers) return false;
  int teams = static_cast<int>(std::max<int64_t>(1, (Q4_GEMV_TARGET_THREADS + team / 2) / team));
  teams = std::min<int>(teams, static_cast<int>(max_consumers / team));
  if (team < 32) teams = std::max(teams, static_cast<int>(32 / team));
  if ((teams * team) % 32) return false;
  const int rpt = rpt_for(mr);
  const int rt = teams * rpt;
  const uint32_t codes_tile = static_cast<uint32_t>(rt * (K / 2));
  const uint32_t sb_tile = static_cast<uint32_t>((rt * G * 2 + 15) / 16 * 16);
  const uint32_t stage_bytes = (codes_tile + 2 * sb_tile + 127) / 128 * 128;
  const int wpt = (team >= 32) ? static_cast<int>(team / 32) : 0;
  grid = static_cast<int>(std::min<int64_t>(a.N, int64_t(dev.sm_count) * Q4_GEMV_CTAS_PER_SM));
  const int64_t cta_rows = (a.N + grid - 1) / grid;
  const int64_t cta_tiles = (cta_rows + rt - 1) / rt;
  // Cross-warp partials: one float per (row, activation row, warp), at most 16 KB.
  int chunk_tiles = static_cast<int>(cta_tiles);
  size_t red_bytes = 0;
  if (wpt > 1) {
    const size_t per_tile = static_cast<size_t>(rt) * mr * wpt * sizeof(float);
    chunk_tiles = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(cta_tiles, (16 * 1024) / per_tile)));
    red_bytes = per_tile * chunk_tiles;
  }
  const size_t budget = std::min<size_t>(Q4_GEMV_SMEM_BUDGET, dev.smem_optin);
  int stages = static_cast<int>((budget - red_bytes) / (stage_bytes + 16));
  stages = std::min<int64_t>(std::min(stages, 8), std::max<int64_t>(2, cta_tiles));
  if (stages < 2) stages = 2;
  smem = static_cast<size_t>(stages) * stage_bytes + 16 * stages + red_bytes;
  if (smem > dev.smem_optin) return false;
  p.N = a.N;
  p.y_ld = a.N;
  p.K = static_cast<int>(K);
  p.G = static_cast<int>(G);
  p.codes = a.codes;
  p.scales = a.scales;
  p.biases = a.biases;
  p.team = static_cast<int>(team);
  p.teams = teams;
  p.rt = rt;
  p.stages = stages;
  p.consumer_threads = static_cast<int>(team) * teams;
  p.chunk_tiles = chunk_tiles;
  p.codes_tile_bytes = codes_tile;
  p.sb_tile_bytes = sb_tile;
  p.stage_bytes = stage_bytes;
  return true;
}

template <int MR>
cudaError_t run_chunk(const MatmulArgs& a, int64_t m0, const DeviceInfo& dev, cudaStream_t stream) {
  TmaGemvParams p;
  size_t smem;
  int grid;
  if (plan_tma(a, MR, dev, p, smem, grid)) {
    const int threads = p.consumer_threads + 32;
    if (threads <= 384) return run_tma<MR, 384>(a, m0, p, smem, grid, stream);
    if constexpr (MR == 1) return run_tma<1, 640>(a, m0, p, smem, grid, stream);
  }
  return run_generic<MR>(a, m0, dev, stream);
}

}  // namespace

cudaError_t gemv_device_flags(unsigned int* flags, bool clear) {
  cudaError_t e = cudaMemcpyFromSymbol(flags, g_device_flags, sizeof(unsigned int));
  if (e == cudaSuccess && clear) {
    const unsigned int zero = 0;
    e = cudaMemcpyToSymbol(g_device_flags, &zero, sizeof(unsigned int));
  }
  return e;
}

cudaError_t launch_gemv(const MatmulArgs& a, cudaStream_t stream, const DeviceInfo& dev) {
  for (int64_t m0 = 0; m0 < a.M; m0 += kMaxRows) {
    const int mr = static_cast<int>(std::min<int64_t>(kMaxRows, a.M - m0));
    cudaError_t e;
    switch (mr) {
      case 1: e = run_chunk<1>(a, m0, dev, stream); break;
      case 2: e = run_chunk<2>(a, m0, dev, stream); break;
      case 3: e = run_chunk<3>(a, m0, dev, stream); break;
      default: e = run_chunk<4>(a, m0, dev, stream); break;
    }
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace q4
