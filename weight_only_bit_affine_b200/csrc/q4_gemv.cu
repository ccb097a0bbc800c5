// q4_gemv.cu -- the CUDA-core GEMV family of the affine Q4 group-32 matmul,
// for one or two activation rows (decode):
//
//   y[m,n] = sum_g ( s[n,g] * sum_{k in g} x[m,k] q[n,k]  +  b[n,g] * sum_{k in g} x[m,k] )
//
// which is x . w_hat^T with w_hat = s*q + b (model card "personaplex-edge-q4":
// affine Q4, group size 32, the packed weights consumed directly by the
// matmul).  The weights are read once from HBM in packed form and never
// expanded in memory.
//
// One launch runs a LIST of independent matmuls ("problems"): the temporal
// step's projections, or a single q4_matmul.  Design (bandwidth-bound at
// ~1.6 flop per packed byte):
//  * One persistent CTA per SM takes a balanced contiguous share of the
//    list's packed bytes (its rows of every problem in turn).  A producer
//    warp streams those rows (codes, scales, biases: contiguous byte ranges)
//    through a ring of shared-memory stages with 1-D bulk (TMA) copies, so
//    the ring never drains between problems.
//  * Consumer threads form "teams" of K/32 lanes; a team owns one weight row
//    at a time and lane j always covers input group j, so its slice of x
//    (read once per problem from global memory, L1 shared by the teams) sits
//    in registers for the whole problem.  Each warp sums its lanes with a
//    transpose-reduce; the sums across a team's warps are finished by an
//    epilogue warp behind mbarriers, so consumers never block on each other.
//  * Codes are unpacked in registers to bf16x2 "128 + q" (one LOP3 per two
//    codes) and multiplied with bf16 x by fma.rn.f32.bf16 (exact products,
//    fp32 accumulation); the offset is removed per group exactly:
//    s*sum x(128+q) + (b - 128 s)*sum x.
//  * Output epilogues (residual add; SwiGLU, whose tiles carry the gate rows
//    and then the same rows of the up weight, paired by the epilogue warp)
//    are compiled into a separate instantiation that only launches holding
//    such problems use.
//  * Programmatic dependent launch: before waiting for the previous kernel a
//    launch only prefetches its first weight tiles into L2 (a hint, no effect
//    on values); everything that reads memory another kernel may write comes
//    after the wait.
#include "q4_device.cuh"
#include "q4_internal.h"

#include <algorithm>
#include <cstdint>
#include <vector>

#ifndef Q4_GEMV_SMEM_BUDGET
#define Q4_GEMV_SMEM_BUDGET (227 * 1024)
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
    uint32_t kmask, kmagic;
    q4_lop3_constants(kmask, kmagic);
#pragma unroll
    for (int w = 0; w < WORDS; ++w)
#pragma unroll
      for (int m = 0; m < MR; ++m)
        word_dot_bf16(words[w], xs[m].v[w][0][0], xs[m].v[w][1][0], xs[m].v[w][2][0], xs[m].v[w][3][0], a0[m],
                      a1[m], kmask, kmagic);
  } else {
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
}

template <int WORDS>
__device__ __forceinline__ void load_words_smem(const uint8_t* p, uint32_t (&words)[WORDS]) {
  if constexpr (WORDS == 4) {
    const uint4 v = *reinterpret_cast<const uint4*>(p);
    words[0] = v.x; words[1] = v.y; words[2] = v.z; words[3] = v.w;
  } else if constexpr (WORDS == 8) {
    const uint4 v = *reinterpret_cast<const uint4*>(p), u = *reinterpret_cast<const uint4*>(p + 16);
    words[0] = v.x; words[1] = v.y; words[2] = v.z; words[3] = v.w;
    words[4] = u.x; words[5] = u.y; words[6] = u.z; words[7] = u.w;
  } else if constexpr (WORDS == 2) {
    const uint2 v = *reinterpret_cast<const uint2*>(p);
    words[0] = v.x; words[1] = v.y;
  } else {
    words[0] = *reinterpret_cast<const uint32_t*>(p);
  }
}

// A lane's code words of one row: 4-bit rows as load_words_smem; 8-bit rows
// (two 16-byte chunks) with the chunks in swapped order when swz is set.
template <int CW>
__device__ __forceinline__ void load_code_words(const uint8_t* p, bool swz, uint32_t (&words)[CW]) {
  if constexpr (CW == 8) {
    const uint4 v = *reinterpret_cast<const uint4*>(p + (swz ? 16 : 0));
    const uint4 u = *reinterpret_cast<const uint4*>(p + (swz ? 0 : 16));
    words[0] = v.x; words[1] = v.y; words[2] = v.z; words[3] = v.w;
    words[4] = u.x; words[5] = u.y; words[6] = u.z; words[7] = u.w;
  } else {
    load_words_smem<CW>(p, words);
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



// Problems per launch: their descriptors travel in the kernel parameters
// (a small instance for single calls, a large one for batches).
constexpr int kMaxProblems = 256;
constexpr int kFewProblems = 4;
// Weight rows per team per tile (4-bit codes), for one activation row and for
// two: larger tiles amortize the per-tile work (barriers, reductions, the
// scale and bias of every row) over more weights.  The temporal stream at one
// row: 805 us at 4 (four 56 KB ring stages), 774 us at 5 (three of 70 KB),
// 883 us at 3; at two rows 1346 us at 4, 1311 us at 5.  Six would overflow
// the epilogue warp's reduction slots at K = 11264.  A chain keeps four: its
// stages give each CTA a few tiles at most, where finer tiles balance better
// (the 129-stage decode chain: 1.53 ms at 4, 1.66 ms at 5).
#ifndef Q4_GEMV_RPT1
#define Q4_GEMV_RPT1 5
#endif
#ifndef Q4_GEMV_RPT2
#define Q4_GEMV_RPT2 5
#endif
constexpr int kRpt1 = Q4_GEMV_RPT1, kRpt2 = Q4_GEMV_RPT2, kRptChain = 4;
// 8-bit codes (q8_matmul): a row is twice the bytes, so a team takes two
// rows per tile and a tile stays near the 4-bit one's size.
constexpr int kRpt8 = 2;

struct GemvProblem {
  const uint16_t* x;       // [MR, K]
  const uint8_t* codes;    // [N, K/2] (4-bit codes) or [N, K] (8-bit)
  const uint16_t* scales;  // [N, K/32]
  const uint16_t* biases;  // [N, K/32]
  uint16_t* y;             // [MR, y_ld]
  const uint16_t* r;       // residual [MR, y_ld] (kEpiResidual), else NULL
  // SwiGLU in one pass: the up projection's weights (NULL otherwise).  A
  // tile then carries rt/2 gate rows followed by the same rows of up, and
  // the epilogue warp writes silu(gate) * up.
  const uint8_t* up_codes;
  const uint16_t* up_scales;
  const uint16_t* up_biases;
  int64_t N, y_ld;
  int64_t byte_begin;      // packed bytes of all earlier problems in the list
  int32_t K, epi;
};

// CTAs per launch at most (one per SM).
constexpr int kMaxCtas = 256;
// Stages of a chain launch at most.
constexpr int kMaxChainStages = kGemvChainMaxStages;
static_assert(kGemvChainMaxProblems == 256, "chain problems: the large parameter block");

template <int NP>
struct GemvLaunch {
  int count;
  int consumer_threads;  // a multiple of 32
  int stages;
  uint32_t stage_bytes;  // >= every problem's tile, 128-byte multiple
  int64_t total_bytes;   // packed bytes of the whole list (a batch launch)
  // A chain launch: stages run in order, stage s being the problems
  // [stage_begin[s], stage_begin[s + 1]) split over all CTAs like a batch of
  // stage_total[s] bytes (byte_begin counts from the stage's start); before
  // reading its inputs for stage s > 0 every CTA waits until done[s - 1]
  // (zero at launch) counts all CTAs.
  int n_stages;
  unsigned int* done;
  // first[c]: the first problem that ends after CTA c's first byte.  Every
  // role of the CTA starts its walk over the list there: the problems before
  // it hold none of its rows, and reading their descriptors (a constant-cache
  // miss each, ~0.4 us) delayed the last CTAs of a 225-problem launch enough
  // to cost the whole launch 5 %.  A launch of at most kFewProblems problems
  // walks from the first.
  uint16_t first[NP > kFewProblems ? kMaxCtas : 1];
  uint16_t stage_begin[NP > kFewProblems ? kMaxChainStages + 1 : 1];
  int64_t stage_total[NP > kFewProblems ? kMaxChainStages : 1];
  GemvProblem prob[NP];
};

constexpr float kNaN = __builtin_nanf("");  // written by a thread whose bounded wait gave up
constexpr int kRedSlots = 8;    // tiles of cross-warp partial sums in flight to the epilogue warp
constexpr int kRedSlotFloats = 64 * 2;  // >= rt * MR * warps-per-team (<= 110 at MR = 1, 120 at MR = 2)

// Shape of one problem for a given consumer count (host and device agree).
struct Geometry {
  int G;      // groups per row
  int team;   // lanes per weight row: G rounded up to 32, or to a power of two below 32
  int teams;  // teams in the CTA
  int wpt;    // warps per team (0 when a warp holds several teams)
  int rt;     // rows per tile
};
__host__ __device__ constexpr int rows_per_team(int bits, int mr, bool chain) {
  return bits == 8 ? kRpt8 : chain ? kRptChain : (mr == 1 ? kRpt1 : kRpt2);
}
__host__ __device__ inline Geometry geometry_of(int K, int consumer_threads, int bits, int mr, bool chain = false) {
  Geometry g;
  g.G = K / 32;
  if (g.G >= 32) {
    g.team = (g.G + 31) / 32 * 32;
  } else {
    g.team = 1;
    while (g.team < g.G) g.team <<= 1;
  }
  g.teams = consumer_threads / g.team;
  g.wpt = g.team >= 32 ? g.team / 32 : 0;
  g.rt = g.teams * rows_per_team(bits, mr, chain);
  return g;
}
// Code bytes of a weight row, and its packed bytes (codes, scales, biases).
__host__ __device__ inline int code_row_bytes(int K, int bits) { return bits == 4 ? K / 2 : K; }
__host__ __device__ inline int64_t packed_row_bytes(int K, int bits = 4) {
  return code_row_bytes(K, bits) + (K / 32) * 4;
}
__host__ __device__ inline bool is_fused(const GemvProblem& P) { return P.up_codes != nullptr; }
// Packed bytes per output row (gate + up when fused).
__host__ __device__ inline int64_t problem_row_bytes(const GemvProblem& P, int bits = 4) {
  return packed_row_bytes(P.K, bits) * (is_fused(P) ? 2 : 1);
}
// Does the problem's tile finish in the epilogue warp (sums across a team's
// warps, or the pairing of gate and up rows)?
__host__ __device__ inline bool uses_epilogue_warp(const GemvProblem& P, const Geometry& g) {
  return g.wpt > 1 || (is_fused(P) && g.wpt >= 1);
}

// Kernel-side views of the above.  A launch whose problems have no epilogue
// runs the EPI = false instantiation, where they fold to the plain matmul's
// constants and the epilogue code is compiled out of the hot loop (keeping it
// there cost the plain stream 4 %).
template <bool EPI>
__device__ __forceinline__ bool fused_k(const GemvProblem& P) {
  if constexpr (EPI) return is_fused(P);
  return false;
}
template <bool EPI>
__device__ __forceinline__ int rtile_k(const GemvProblem& P, const Geometry& g) {
  return fused_k<EPI>(P) ? g.rt / 2 : g.rt;
}
template <bool EPI>
__device__ __forceinline__ bool epilogue_warp_k(const GemvProblem& P, const Geometry& g) {
  return g.wpt > 1 || (fused_k<EPI>(P) && g.wpt >= 1);
}
// CHAIN: the residual may have been written by another CTA of the launch
// (an earlier stage), so it is read through L2.
template <bool EPI, bool CHAIN>
__device__ __forceinline__ uint16_t store_k(float v, const GemvProblem& P, int64_t idx) {
  if constexpr (EPI && CHAIN) {
    if (P.epi == kEpiResidual) return float_to_bf16_bits(v + bf16_bits_to_float(__ldcg(P.r + idx)));
    return float_to_bf16_bits(v);
  }
  if constexpr (EPI) return epilogue_bf16(v, P.epi, P.r, idx);
  return float_to_bf16_bits(v);
}

__device__ __forceinline__ uint32_t tile_rows(int64_t r_end, int64_t row0, int rt) {
  return static_cast<uint32_t>((r_end - row0 < rt) ? (r_end - row0) : rt);
}

// sum over this lane's 32 inputs of x * (mac_offset + q) for one weight row
// (four code words): the same operations in the same order on every path,
// so a row's result does not depend on where it falls in a tile.
__device__ __forceinline__ float row_acc(const uint32_t (&words)[4], const XSlice<4, Q4_GEMV_MAC>& xs, uint32_t kmask,
                                         uint32_t kmagic) {
  float acc = 0.f;
  if constexpr (Q4_GEMV_MAC == kMacMixedBf16) {
#pragma unroll
    for (int w = 0; w < 4; ++w)
      word_dot_bf16_acc(words[w], xs.v[w][0][0], xs.v[w][1][0], xs.v[w][2][0], xs.v[w][3][0], acc, kmask, kmagic);
  } else {
    float a0[1] = {0.f}, a1[1] = {0.f};
    dot_plus128<1, 4, Q4_GEMV_MAC>(words, *reinterpret_cast<const XSlice<4, Q4_GEMV_MAC>(*)[1]>(&xs), a0, a1);
    acc = a0[0] + a1[0];
  }
  return acc;
}

// The same for a row of 8-bit codes (eight words; byte i of word w is the
// code of input 4w + i): each code becomes an exact fp32 -- the byte under
// the exponent of 2^23, minus 2^23 -- and two at a time meet the lane's x
// pairs (x[8v + t], x[8v + t + 4]), whose codes are byte t of words 2v and
// 2v + 1, in one packed fp32 FMA.  The products are exact; no offset.
__device__ __forceinline__ float row_acc8(const uint32_t (&words)[8], const XSlice<4, kMacMixedBf16>& xs) {
  float a0 = 0.f, a1 = 0.f;
#pragma unroll
  for (int v = 0; v < 4; ++v)
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      float q0 = __uint_as_float(__byte_perm(words[2 * v], 0x4B000000u, 0x7540u | t));
      float q1 = __uint_as_float(__byte_perm(words[2 * v + 1], 0x4B000000u, 0x7540u | t));
      fadd2(q0, q1, -8388608.f, -8388608.f);
      const uint32_t xp = xs.v[v][t][0];
      ffma2(a0, a1, q0, q1, __uint_as_float(xp << 16), __uint_as_float(xp & 0xFFFF0000u));
    }
  return a0 + a1;
}

template <int BITS, int CW>
__device__ __forceinline__ float row_acc_bits(const uint32_t (&words)[CW], const XSlice<4, Q4_GEMV_MAC>& xs,
                                              uint32_t kmask, uint32_t kmagic) {
  if constexpr (BITS == 4) {
    return row_acc(words, xs, kmask, kmagic);
  } else {
    static_assert(Q4_GEMV_MAC == kMacMixedBf16, "8-bit rows use the bf16 pair layout of x");
    return row_acc8(words, xs);
  }
}

// The rows of problem `pi` that belong to this CTA's byte range [lo, hi) of
// the concatenated list: [*r0, *r1).  A row belongs to the CTA whose range
// holds its first packed byte, so each row of the list belongs to exactly one
// CTA; a row's arithmetic is the same wherever it falls in a tile (row_acc,
// the fixed reduction trees), so results do not depend on the split.
// Returns false when the problem lies entirely after the range (the caller
// stops scanning).
template <bool EPI, int BITS, int NP>
__device__ __forceinline__ bool segment_of(const GemvLaunch<NP>& L, int pi, int64_t lo, int64_t hi, int64_t* r0,
                                           int64_t* r1) {
  const GemvProblem& P = L.prob[pi];
  const int64_t rb = packed_row_bytes(P.K, BITS) * (fused_k<EPI>(P) ? 2 : 1);
  const int64_t pb = P.byte_begin, pe = pb + P.N * rb;
  *r0 = *r1 = 0;
  if (pb >= hi) return false;
  if (pe <= lo) return true;
  const int64_t a = (lo > pb ? lo : pb) - pb, b = (hi < pe ? hi : pe) - pb;
  *r0 = (a + rb - 1) / rb;
  *r1 = (b + rb - 1) / rb;
  if (*r0 > P.N) *r0 = P.N;
  if (*r1 > P.N) *r1 = P.N;
  return true;
}

// BITS: 4-bit codes (two per byte) or 8-bit codes (q8_matmul).
template <int MR, int MAXT, int NP, bool EPI, bool CHAIN, int BITS>
__global__ void __launch_bounds__(MAXT, 1) gemv_kernel(const __grid_constant__ GemvLaunch<NP> L) {
  static_assert(!CHAIN || NP > kFewProblems, "chains use the large parameter block");
  static_assert(BITS == 4 || BITS == 8, "code width");
  extern __shared__ __align__(128) uint8_t smem[];
  constexpr int RPT = rows_per_team(BITS, MR, CHAIN);  // rows per team per tile
  constexpr int CW = BITS == 4 ? 4 : 8;          // code words per lane per row (32 codes)
  constexpr int V = RPT * MR;
  constexpr int VP = pow2_at_least(V);
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int consumer_warps = L.consumer_threads >> 5;

  float* red = reinterpret_cast<float*>(smem + static_cast<size_t>(L.stages) * L.stage_bytes);
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(red + kRedSlots * kRedSlotFloats);
  uint64_t* empty_bar = full_bar + L.stages;
  uint64_t* rfull_bar = empty_bar + L.stages;   // [kRedSlots]
  uint64_t* rempty_bar = rfull_bar + kRedSlots;  // [kRedSlots]
  // Chains: go (phase s - 1 completes when this CTA may read the inputs of
  // stage s) and stage_done (phase s completes when every consumer warp and
  // the epilogue warp finished their writes of stage s).
  uint64_t* go_bar = rempty_bar + kRedSlots;
  uint64_t* stage_done_bar = go_bar + 1;
  // Set by any thread whose bounded wait gave up: the epilogue warp then
  // writes NaN for the partial sums it cannot vouch for.
  volatile uint32_t* gave_up = reinterpret_cast<volatile uint32_t*>(stage_done_bar + 1);

  if (tid == 0) {
    for (int s = 0; s < L.stages; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], consumer_warps);
    }
    for (int s = 0; s < kRedSlots; ++s) {
      mbar_init(&rfull_bar[s], consumer_warps);
      mbar_init(&rempty_bar[s], 1);
    }
    mbar_init(go_bar, 1);
    mbar_init(stage_done_bar, consumer_warps + 1);
    *gave_up = 0u;
    fence_mbar_init();
  }
  __syncthreads();
  pdl_launch_dependents();

  // The launch's stages (a batch is one) and this CTA's share of each: a
  // contiguous, balanced range [lo, hi) of the stage's packed bytes, and the
  // problems [pb, pe) to walk for it.
  const int n_st = CHAIN ? L.n_stages : 1;
  auto share = [&](int cs, int64_t& lo, int64_t& hi, int& pb, int& pe) {
    const int64_t T = CHAIN ? L.stage_total[cs] : L.total_bytes;
    lo = static_cast<int64_t>(blockIdx.x) * T / gridDim.x;
    hi = static_cast<int64_t>(blockIdx.x + 1) * T / gridDim.x;
    if constexpr (CHAIN) {
      pb = L.stage_begin[cs];
      pe = L.stage_begin[cs + 1];
    } else {
      pb = NP > kFewProblems ? L.first[blockIdx.x] : 0;
      pe = L.count;
    }
  };

  if (warp == consumer_warps) {
    // ---------------- producer warp ----------------
    if (lane == 0) {
      {  // warm L2 with the first tiles of the range (a hint; changes no value)
        int64_t r0, r1, lo, hi;
        int issued = 0, pb, pe;
        for (int cs = 0; cs < n_st && issued < L.stages; ++cs) {
        share(cs, lo, hi, pb, pe);
        for (int pi = pb; pi < pe && issued < L.stages; ++pi) {
          if (!segment_of<EPI, BITS>(L, pi, lo, hi, &r0, &r1)) break;
          const GemvProblem& P = L.prob[pi];
          const Geometry geo = geometry_of(P.K, L.consumer_threads, BITS, MR, CHAIN);
          const int code_bytes = code_row_bytes(P.K, BITS);  // code bytes per row
          const int rtile = rtile_k<EPI>(P, geo);
          for (int64_t row0 = r0; row0 < r1 && issued < L.stages; row0 += rtile, ++issued) {
            const uint32_t rows = tile_rows(r1, row0, rtile);
            bulk_prefetch_l2(P.codes + row0 * code_bytes, rows * code_bytes);
            bulk_prefetch_l2(P.scales + row0 * geo.G, rows * geo.G * 2);
            bulk_prefetch_l2(P.biases + row0 * geo.G, rows * geo.G * 2);
            if (fused_k<EPI>(P)) {
              bulk_prefetch_l2(P.up_codes + row0 * code_bytes, rows * code_bytes);
              bulk_prefetch_l2(P.up_scales + row0 * geo.G, rows * geo.G * 2);
              bulk_prefetch_l2(P.up_biases + row0 * geo.G, rows * geo.G * 2);
            }
          }
        }
        }
      }
      pdl_wait_predecessors();
      // The ring carries weight tiles only (the consumers read their
      // activations from global memory); the producer never waits for other
      // CTAs: across a chain's stages it streams weights ahead.
      int stage = 0, issued = 0;
      uint32_t phase = 0;
      bool dead = false;
      for (int cs = 0; cs < n_st && !dead; ++cs) {
      int64_t lo, hi;
      int pb, pe;
      share(cs, lo, hi, pb, pe);
      for (int pi = pb; pi < pe && !dead; ++pi) {
        int64_t r0, r1;
        if (!segment_of<EPI, BITS>(L, pi, lo, hi, &r0, &r1)) break;
        if (r0 >= r1) continue;
        const GemvProblem& P = L.prob[pi];
        const Geometry geo = geometry_of(P.K, L.consumer_threads, BITS, MR, CHAIN);
        const int code_bytes = code_row_bytes(P.K, BITS);  // code bytes per row
        const int rtile = rtile_k<EPI>(P, geo);
        for (int64_t row0 = r0; row0 < r1; row0 += rtile) {
          if (!mbar_wait(&empty_bar[stage], phase ^ 1u)) { dead = true; *gave_up = 1u; break; }
          uint8_t* st = smem + static_cast<size_t>(stage) * L.stage_bytes;
          {
            // Stage layout: codes of the tile's rows from 0, scales from
            // sb_off, biases from sb_off + sb_tile; a fused tile puts the up
            // rows right after the gate rows in each of the three regions
            // (2 * rows <= rt, and every offset stays a multiple of 16 bytes).
            const uint32_t rows = tile_rows(r1, row0, rtile);
            const uint32_t cb = rows * code_bytes, sb = rows * geo.G * 2;
            const uint32_t sb_off = static_cast<uint32_t>(geo.rt) * code_bytes;
            const uint32_t sb_tile = (static_cast<uint32_t>(geo.rt) * geo.G * 2 + 15u) & ~15u;
            const bool fused = fused_k<EPI>(P);
            mbar_arrive_expect_tx(&full_bar[stage], (fused ? 2u : 1u) * (cb + 2 * sb));
            bulk_g2s(st, P.codes + row0 * code_bytes, cb, &full_bar[stage]);
            bulk_g2s(st + sb_off, P.scales + row0 * geo.G, sb, &full_bar[stage]);
            bulk_g2s(st + sb_off + sb_tile, P.biases + row0 * geo.G, sb, &full_bar[stage]);
            if (fused) {
              bulk_g2s(st + cb, P.up_codes + row0 * code_bytes, cb, &full_bar[stage]);
              bulk_g2s(st + sb_off + sb, P.up_scales + row0 * geo.G, sb, &full_bar[stage]);
              bulk_g2s(st + sb_off + sb_tile + sb, P.up_biases + row0 * geo.G, sb, &full_bar[stage]);
            }
          }
          ++issued;
          if (++stage == L.stages) { stage = 0; phase ^= 1u; }
        }
      }
      }
      // No copy may still target this CTA's shared memory when it exits.
      for (int i = 0; i < min(issued, L.stages); ++i) {
        int s = stage - 1 - i;
        uint32_t ph = phase;
        if (s < 0) { s += L.stages; ph ^= 1u; }
        mbar_wait(&full_bar[s], ph);
      }
    }
    return;
  }

  pdl_wait_predecessors();  // consumers and epilogue read x and write y

  if (warp == consumer_warps + 1) {
    // ---------------- epilogue warp: sums across a team's warps, per tile ----------------
    int slot = 0;
    uint32_t sph = 0;
    bool dead = false;
    for (int cs = 0; cs < n_st; ++cs) {
    if constexpr (CHAIN) {
      if (cs > 0) {
        // Stage cs - 1 is complete in this CTA once its consumer warps and
        // this warp have arrived: announce it, wait for every CTA, then let
        // this CTA's consumers read the inputs of stage cs.  (A CTA whose
        // wait gave up still announces, so no other CTA waits on it.)
        if (!dead && !mbar_wait(stage_done_bar, static_cast<uint32_t>(cs - 1) & 1u)) { dead = true; *gave_up = 1u; }
        if (lane == 0) {
          grid_arrive(&L.done[cs - 1]);
          if (!dead && !grid_wait(&L.done[cs - 1], gridDim.x)) { dead = true; *gave_up = 1u; }
          mbar_arrive(go_bar);
        }
        dead = __shfl_sync(0xFFFFFFFFu, dead ? 1 : 0, 0) != 0;
      }
    }
    int64_t lo, hi;
    int pb, pe;
    share(cs, lo, hi, pb, pe);
    for (int pi = pb; pi < pe; ++pi) {
      int64_t r0, r1;
      if (!segment_of<EPI, BITS>(L, pi, lo, hi, &r0, &r1)) break;
      const GemvProblem& P = L.prob[pi];
      const Geometry geo = geometry_of(P.K, L.consumer_threads, BITS, MR, CHAIN);
      if (!epilogue_warp_k<EPI>(P, geo)) continue;
      const int rtile = rtile_k<EPI>(P, geo);
      const bool fused = fused_k<EPI>(P);
      for (int64_t row0 = r0; row0 < r1; row0 += rtile) {
        if (!dead && !mbar_wait(&rfull_bar[slot], sph)) { dead = true; *gave_up = 1u; }
        // Slot entry ((row * MR + m) * wpt + warp) holds one warp's partial
        // sum of the tile's row; a fused tile's up rows follow its n gate rows.
        const int n = static_cast<int>(tile_rows(r1, row0, rtile));
        const float* rs = red + slot * kRedSlotFloats;
        for (int i = lane; i < n * MR; i += 32) {
          const int lr = i / MR, m = i - lr * MR;
          float v = (dead || *gave_up) ? kNaN : 0.f;
          for (int w = 0; w < geo.wpt; ++w) v += rs[i * geo.wpt + w];
          const int64_t idx = static_cast<int64_t>(m) * P.y_ld + row0 + lr;
          if (fused) {
            float u = 0.f;
            for (int w = 0; w < geo.wpt; ++w) u += rs[(i + n * MR) * geo.wpt + w];
            P.y[idx] = float_to_bf16_bits(silu_f32(v) * u);
          } else {
            P.y[idx] = store_k<EPI, CHAIN>(v, P, idx);
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&rempty_bar[slot]);
        if (++slot == kRedSlots) { slot = 0; sph ^= 1u; }
      }
    }
    if constexpr (CHAIN) {
      __syncwarp();
      if (lane == 0 && cs + 1 < n_st) mbar_arrive(stage_done_bar);
    }
    }
    return;
  }

  // ---------------- consumer threads ----------------
  uint32_t kmask, kmagic;  // the dot product's LOP3 constants, held in registers
  q4_lop3_constants(kmask, kmagic);
  int stage = 0, slot = 0;
  uint32_t phase = 0, sph = 0;
  bool dead = false;
  for (int cs = 0; cs < n_st; ++cs) {
  if constexpr (CHAIN) {  // the inputs of stage cs are complete (every CTA finished stage cs - 1)
    if (cs > 0 && !dead && !mbar_wait(go_bar, static_cast<uint32_t>(cs - 1) & 1u)) { dead = true; *gave_up = 1u; }
  }
  int64_t lo, hi;
  int pb, pe;
  share(cs, lo, hi, pb, pe);
  for (int pi = pb; pi < pe; ++pi) {
    int64_t r_begin, r_end;
    if (!segment_of<EPI, BITS>(L, pi, lo, hi, &r_begin, &r_end)) break;
    if (r_begin >= r_end) continue;
    const GemvProblem& P = L.prob[pi];
    const Geometry geo = geometry_of(P.K, L.consumer_threads, BITS, MR, CHAIN);
    const int code_bytes = code_row_bytes(P.K, BITS);  // code bytes per row
    const int team_idx = tid / geo.team;
    const int j = tid - team_idx * geo.team;
    const bool active = team_idx < geo.teams && j < geo.G;
    const int warp_in_team = (geo.team >= 32) ? (j >> 5) : 0;
    const uint32_t sb_off = static_cast<uint32_t>(geo.rt) * code_bytes;
    const uint32_t sb_tile = (static_cast<uint32_t>(geo.rt) * geo.G * 2 + 15u) & ~15u;
    // Byte offsets inside a stage of this lane's first row (row team_idx) and
    // the step to its next row (teams rows further).
    const uint32_t code_off0 = static_cast<uint32_t>(team_idx) * code_bytes + j * (4 * CW);
    const uint32_t code_step = static_cast<uint32_t>(geo.teams) * code_bytes;
    const uint32_t sc_off0 = sb_off + (static_cast<uint32_t>(team_idx) * geo.G + j) * 2;
    const uint32_t sc_step = static_cast<uint32_t>(geo.teams) * geo.G * 2;

    // Activations: this lane's 32 inputs of each row, read from global memory
    // with plain loads once the launch's inputs are complete (after the
    // programmatic-dependent-launch wait; in a chain, after the stage barrier:
    // an acquire at GPU scope, then the go barrier).  The teams after the
    // first hit in L1.  (Sending them through the ring ahead of the tiles
    // took a stage per segment and was 2 % slower on the stream; in a chain a
    // read through L2 per team, or staging in shared memory at the cost of a
    // ring stage, were slower too.)
    XSlice<4, Q4_GEMV_MAC> xsl[MR];
#pragma unroll
    for (int m = 0; m < MR; ++m) {
      if (active)
        xsl[m].load(P.x + m * P.K + j * 32);
      else
        xsl[m].zero();
    }

    // 8-bit rows: a lane's 32 codes are two 16-byte chunks 32 bytes apart
    // from the next lane's; lanes 4..7 of every eight read their second chunk
    // first, so each quarter-warp load covers 128 distinct bytes (no bank
    // conflict), and their x slices swap halves to match.
    const bool swz = BITS == 8 && ((lane >> 2) & 1);
    if constexpr (BITS == 8) {
#pragma unroll
      for (int m = 0; m < MR; ++m)
#pragma unroll
        for (int w = 0; w < 2; ++w)
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            const uint32_t a = xsl[m].v[w][t][0], b = xsl[m].v[w + 2][t][0];
            xsl[m].v[w][t][0] = swz ? b : a;
            xsl[m].v[w + 2][t][0] = swz ? a : b;
          }
    }
    const bool use_red = epilogue_warp_k<EPI>(P, geo);
    const int rtile = rtile_k<EPI>(P, geo);
    constexpr float kOffset = BITS == 4 ? mac_offset<Q4_GEMV_MAC>() : 0.f;

    for (int64_t row0 = r_begin; row0 < r_end; row0 += rtile) {
      if (!dead && !mbar_wait(&full_bar[stage], phase)) { dead = true; *gave_up = 1u; }
      const uint8_t* st = smem + static_cast<size_t>(stage) * L.stage_bytes;
      // Rows of this tile are dealt to the teams round-robin (row r goes to
      // team r % teams), so a short last tile stays balanced; when a team
      // spans whole warps the row count below is warp-uniform and idle warps
      // skip the arithmetic entirely.  A fused tile of n output rows holds
      // 2n weight rows (gate rows, then up rows), all computed alike.
      const int tile_out = static_cast<int>((r_end - row0 < rtile) ? (r_end - row0) : rtile);
      const int tile_n = fused_k<EPI>(P) ? 2 * tile_out : tile_out;
      const int nv = (team_idx >= geo.teams || team_idx >= tile_n) ? 0
                     : (tile_n == geo.rt)                          ? RPT
                                                                   : (tile_n - team_idx + geo.teams - 1) / geo.teams;
      float vals[VP];
#pragma unroll
      for (int i = 0; i < VP; ++i) vals[i] = 0.f;
      bool compute = true;

      if (geo.team >= 32 && nv == RPT) {
        // Fast path: every row of this team is present (warp-uniform).
        // Lanes past G (padding) read in-stage bytes but take s = b = 0 and
        // a zero x slice, so they add exactly nothing.
        uint32_t words[RPT][CW];
        float sc[RPT], bi[RPT];
        const uint8_t* cp = st + code_off0;
        const uint8_t* sp = st + sc_off0;
#pragma unroll
        for (int rr = 0; rr < RPT; ++rr) {
          load_code_words<CW>(cp + rr * code_step, swz, words[rr]);
          const uint16_t sh = *reinterpret_cast<const uint16_t*>(sp + rr * sc_step);
          const uint16_t bh = *reinterpret_cast<const uint16_t*>(sp + rr * sc_step + sb_tile);
          sc[rr] = active ? bf16_bits_to_float(sh) : 0.f;
          bi[rr] = active ? bf16_bits_to_float(bh) : 0.f;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty_bar[stage]);
        if (++stage == L.stages) { stage = 0; phase ^= 1u; }
#pragma unroll
        for (int rr = 0; rr < RPT; ++rr) {
          const float c = fmaf(-kOffset, sc[rr], bi[rr]);
#pragma unroll
          for (int m = 0; m < MR; ++m)
            vals[rr * MR + m] = fmaf(sc[rr], row_acc_bits<BITS>(words[rr], xsl[m], kmask, kmagic), c * xsl[m].sum);
        }
      } else {
        uint32_t words[RPT][CW];
        float sc[RPT], bi[RPT];
        const bool lane_on = active && nv > 0;
#pragma unroll
        for (int rr = 0; rr < RPT; ++rr) {  // all shared-memory loads first
          if (lane_on && rr < nv) {
            load_code_words<CW>(st + code_off0 + rr * code_step, swz, words[rr]);
            sc[rr] = bf16_bits_to_float(*reinterpret_cast<const uint16_t*>(st + sc_off0 + rr * sc_step));
            bi[rr] = bf16_bits_to_float(*reinterpret_cast<const uint16_t*>(st + sc_off0 + rr * sc_step + sb_tile));
          } else {
#pragma unroll
            for (int w = 0; w < CW; ++w) words[rr][w] = 0u;
            sc[rr] = bi[rr] = 0.f;
          }
        }
        // The stage's bytes are in registers now: hand it back to the producer.
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty_bar[stage]);
        if (++stage == L.stages) { stage = 0; phase ^= 1u; }

        if (geo.team >= 32 && nv == 0) {
          compute = false;  // a whole idle warp
        } else {
#pragma unroll
          for (int rr = 0; rr < RPT; ++rr) {
            if (geo.team >= 32 && rr >= nv) break;  // warp-uniform
            const float c = fmaf(-kOffset, sc[rr], bi[rr]);
#pragma unroll
            for (int m = 0; m < MR; ++m)
              vals[rr * MR + m] = fmaf(sc[rr], row_acc_bits<BITS>(words[rr], xsl[m], kmask, kmagic), c * xsl[m].sum);
          }
        }
      }

      if (geo.team >= 32) {
        float* rs = red + slot * kRedSlotFloats;
        if (use_red && !dead && !mbar_wait(&rempty_bar[slot], sph ^ 1u)) { dead = true; *gave_up = 1u; }
        if (compute) {
          const float tot = transpose_reduce<VP>(vals, lane);
          const int idx = lane >> (5 - ilog2(VP));
          const int rr = idx / MR, m = idx % MR;
          const bool holder = (lane & ((32 / VP) - 1)) == 0 && idx < V && rr < nv;
          if (holder) {
            const int lr = team_idx + rr * geo.teams;  // row within the tile
            if (!use_red) {
              const int64_t idx = static_cast<int64_t>(m) * P.y_ld + row0 + lr;
              P.y[idx] = store_k<EPI, CHAIN>(dead ? kNaN : tot, P, idx);
            } else {
              rs[(lr * MR + m) * geo.wpt + warp_in_team] = tot;
            }
          }
        }
        if (use_red) {
          __syncwarp();
          if (lane == 0) mbar_arrive(&rfull_bar[slot]);
          if (++slot == kRedSlots) { slot = 0; sph ^= 1u; }
        }
      } else {
#pragma unroll
        for (int i = 0; i < V; ++i) vals[i] = seg_allreduce_dyn(vals[i], geo.team);
        if (j == 0) {
#pragma unroll
          for (int rr = 0; rr < RPT; ++rr)
            if (rr < nv) {
              const int64_t row = row0 + team_idx + rr * geo.teams;
#pragma unroll
              for (int m = 0; m < MR; ++m) {
                const int64_t idx = static_cast<int64_t>(m) * P.y_ld + row;
                P.y[idx] = store_k<EPI, CHAIN>(dead ? kNaN : vals[rr * MR + m], P, idx);
              }
            }
        }
      }
    }
  }
  if constexpr (CHAIN) {  // this warp's writes of stage cs are done
    __syncwarp();
    if (lane == 0 && cs + 1 < n_st) mbar_arrive(stage_done_bar);
  }
  }
}

// Generic path: any K, any 2-byte-aligned scales.  One warp per weight row,
// lanes stride over the row's groups; x is read through the L1 per group.
// A fused (SwiGLU) problem computes the gate and the up row of each output.
struct GenericParams {
  const uint16_t* x;
  const uint8_t* codes;
  const uint16_t* scales;
  const uint16_t* biases;
  uint16_t* y;
  const uint16_t* r;  // residual, or NULL
  const uint8_t* up_codes;  // SwiGLU up weights, or NULL
  const uint16_t* up_scales;
  const uint16_t* up_biases;
  int64_t N, y_ld;
  int K, G, epi;
};

// This lane's share of row `row` of one weight: sum over its groups of
// x * w_hat, per activation row.
template <int MR>
__device__ __forceinline__ void generic_row_dot(const GenericParams& p, const uint8_t* codes, const uint16_t* scales,
                                                const uint16_t* biases, int64_t row, int lane, float (&acc)[MR]) {
#pragma unroll
  for (int m = 0; m < MR; ++m) acc[m] = 0.f;
  for (int g = lane; g < p.G; g += 32) {
    const uint4 c4 = ld_nc_v4(codes + row * (p.K / 2) + static_cast<int64_t>(g) * 16);
    const uint32_t words[4] = {c4.x, c4.y, c4.z, c4.w};
    const float s = bf16_bits_to_float(scales[row * p.G + g]);
    const float b = bf16_bits_to_float(biases[row * p.G + g]);
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
}

template <int MR>
__global__ void __launch_bounds__(256) gemv_generic_kernel(const __grid_constant__ GenericParams p) {
  pdl_launch_dependents();
  pdl_wait_predecessors();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t warps_total = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t row = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + warp; row < p.N; row += warps_total) {
    float acc[MR];
    generic_row_dot<MR>(p, p.codes, p.scales, p.biases, row, lane, acc);
    if (p.up_codes != nullptr) {
      float up[MR];
      generic_row_dot<MR>(p, p.up_codes, p.up_scales, p.up_biases, row, lane, up);
#pragma unroll
      for (int m = 0; m < MR; ++m) {
        const float g = seg_allreduce<32>(acc[m]), u = seg_allreduce<32>(up[m]);
        if (lane == 0) p.y[static_cast<int64_t>(m) * p.y_ld + row] = float_to_bf16_bits(silu_f32(g) * u);
      }
      continue;
    }
#pragma unroll
    for (int m = 0; m < MR; ++m) {
      const float v = seg_allreduce<32>(acc[m]);
      const int64_t idx = static_cast<int64_t>(m) * p.y_ld + row;
      if (lane == 0) p.y[idx] = epilogue_bf16(v, p.epi, p.r, idx);
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

// Block shapes: consumers + producer warp + epilogue warp.  The thread
// counts bound the registers (768 threads: 80 per thread; 448: 128 -- the
// registers are split evenly over the SM's four schedulers, each holding at
// most ceil(warps / 4) of the block's warps).  One activation row: 22
// consumer warps -- teams of 4 warps for K = 4096 (five teams), of 11 for
// K = 11264 (two teams), and enough warps in flight to hide the
// shared-memory and dependency latencies of the dot products (measured: 704
// consumers stream the temporal step 30% faster than 512; 24 consumer warps,
// which need 72 registers, or a reduction by the team's last warp in place
// of the epilogue warp, were 12-15% slower).  Two rows: 12 consumer warps,
// three teams for K = 4096 (7% faster on a layer than 11 warps, two teams).
#ifndef Q4_GEMV_CONSUMERS1
#define Q4_GEMV_CONSUMERS1 704
#endif
constexpr int kConsumers1 = Q4_GEMV_CONSUMERS1, kThreads1 = kConsumers1 + 64;  // one activation row
#ifndef Q4_GEMV_CONSUMERS2
#define Q4_GEMV_CONSUMERS2 384
#endif
constexpr int kConsumers2 = Q4_GEMV_CONSUMERS2, kThreads2 = kConsumers2 + 64;  // two activation rows

int consumers_for(int mr) { return mr == 1 ? kConsumers1 : kConsumers2; }

// Does the bulk-copy kernel take this problem (else: the generic kernel)?
bool tma_ok(const MatmulArgs& a, int mr, int bits = 4) {
  const int64_t G = a.K / 32;
  if (G % 8 != 0) return false;  // scale rows must be whole 16-byte runs for bulk copies
  uintptr_t sb = reinterpret_cast<uintptr_t>(a.scales) | reinterpret_cast<uintptr_t>(a.biases);
  if (a.fused()) sb |= reinterpret_cast<uintptr_t>(a.up_scales) | reinterpret_cast<uintptr_t>(a.up_biases);
  if (sb & 15u) return false;
  const Geometry geo = geometry_of(static_cast<int>(a.K), consumers_for(mr), bits, mr);
  // A fused tile pairs gate and up rows in the epilogue warp, which needs
  // teams of whole warps.
  if (a.fused() && geo.team < 32) return false;
  return geo.teams >= 1 && geo.team <= consumers_for(mr);
}

template <int MR>
cudaError_t run_generic(const MatmulArgs& a, int64_t m0, const DeviceInfo& dev, cudaStream_t stream) {
  GenericParams p;
  p.x = a.x + m0 * a.K;
  p.codes = a.codes;
  p.scales = a.scales;
  p.biases = a.biases;
  p.y = a.y + m0 * a.N;
  p.r = a.r ? a.r + m0 * a.N : nullptr;
  p.up_codes = a.up_codes;
  p.up_scales = a.up_scales;
  p.up_biases = a.up_biases;
  p.N = a.N;
  p.y_ld = a.N;
  p.K = static_cast<int>(a.K);
  p.G = static_cast<int>(a.K / 32);
  p.epi = a.epi;
  const int64_t blocks = (a.N + 7) / 8;
  const int grid = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(blocks, int64_t(dev.sm_count) * 8)));
  return launch_pdl(gemv_generic_kernel<MR>, dim3(grid), dim3(256), 0, stream, p);
}

// Grows *stage_bytes to hold a tile of P; false if the epilogue warp's
// reduction slots cannot take P's tiles (they are sized for kConsumers1 /
// kConsumers2).
bool ring_stage_fits(const GemvProblem& P, int mr, int consumers, uint32_t& stage_bytes, int bits = 4,
                     bool chain = false) {
  const Geometry geo = geometry_of(P.K, consumers, bits, mr, chain);
  const uint32_t tile = static_cast<uint32_t>(geo.rt) * code_row_bytes(P.K, bits) +
                        2 * ((static_cast<uint32_t>(geo.rt) * geo.G * 2 + 15u) & ~15u);
  stage_bytes = std::max(stage_bytes, (tile + 127u) & ~127u);
  return !(uses_epilogue_warp(P, geo) && geo.rt * mr * geo.wpt > kRedSlotFloats);
}

// Ring depth and dynamic shared memory for stages of stage_bytes.
bool ring_of(uint32_t stage_bytes, const DeviceInfo& dev, int* stages, size_t* smem) {
  // reduction slots, their barriers, the chain's two barriers, the flag word
  const size_t fixed = sizeof(float) * kRedSlots * kRedSlotFloats + 16 * kRedSlots + 16 + 16;
  const size_t budget = std::min<size_t>(Q4_GEMV_SMEM_BUDGET, dev.smem_optin);
  if (fixed + 2 * (stage_bytes + 16) > dev.smem_optin) return false;
  *stages = std::max(2, std::min(static_cast<int>((budget - fixed) / (stage_bytes + 16)), 12));
  *smem = static_cast<size_t>(*stages) * stage_bytes + fixed + 16 * *stages;
  return true;
}

// Launches the bulk-copy kernel over `count` problems of `probs` (all taking
// this path, all with MR activation rows).
template <int MR, int NP, int BITS = 4>
cudaError_t run_list(const GemvProblem* probs, int count, const DeviceInfo& dev, cudaStream_t stream) {
  constexpr int kThreads = MR == 1 ? kThreads1 : kThreads2;
  const int consumers = consumers_for(MR);
  static_assert(sizeof(GemvLaunch<NP>) <= 32000, "kernel parameters exceed the launch limit");
  thread_local GemvLaunch<NP> L;  // copied into the launch parameters by cudaLaunchKernelEx
  uint32_t stage_bytes = 128;
  int64_t total = 0;
  for (int i = 0; i < count; ++i) {
    const GemvProblem& P = probs[i];
    if (!ring_stage_fits(P, MR, consumers, stage_bytes, BITS)) return cudaErrorInvalidConfiguration;
    L.prob[i] = P;
    L.prob[i].byte_begin = total;
    total += P.N * problem_row_bytes(P, BITS);
  }
  int stages = 0;
  size_t smem = 0;
  if (!ring_of(stage_bytes, dev, &stages, &smem)) return cudaErrorInvalidConfiguration;
  L.count = count;
  L.consumer_threads = consumers;
  L.stages = stages;
  L.stage_bytes = stage_bytes;
  L.total_bytes = total;
  // Enough CTAs that every one has work; one per SM.
  const int64_t rows = [&] { int64_t r = 0; for (int i = 0; i < count; ++i) r += probs[i].N; return r; }();
  const int grid = static_cast<int>(
      std::max<int64_t>(1, std::min<int64_t>(std::min(dev.sm_count, kMaxCtas), rows)));
  // each CTA's first problem: the first that ends after the CTA's first byte
  // (the kernel's byte range formula)
  int pi = 0;
  for (int c = 0; c < grid && NP > kFewProblems; ++c) {
    const int64_t lo = static_cast<int64_t>(c) * total / grid;
    while (pi < count && L.prob[pi].byte_begin + L.prob[pi].N * problem_row_bytes(L.prob[pi], BITS) <= lo) ++pi;
    L.first[c] = static_cast<uint16_t>(pi);
  }
  bool epi = false;
  for (int i = 0; i < count; ++i) epi = epi || probs[i].epi != kEpiNone || is_fused(probs[i]);
  auto kern = epi ? gemv_kernel<MR, kThreads, NP, true, false, BITS> : gemv_kernel<MR, kThreads, NP, false, false, BITS>;
  return launch_pdl(kern, dim3(grid), dim3(kThreads), smem, stream, L);
}

// One chain launch: `count` problems (all taking the bulk-copy kernel, MR
// activation rows) in n_stages stages of stage_counts[s] problems each;
// done: n_stages counters, zero.  Every CTA takes part in every stage, so
// the launch is cooperative (all CTAs resident at once, one per SM).
template <int MR>
cudaError_t run_chain(const GemvProblem* probs, int count, const int* stage_counts, int n_stages, unsigned int* done,
                      const DeviceInfo& dev, cudaStream_t stream) {
  constexpr int NP = kMaxProblems;
  constexpr int kThreads = MR == 1 ? kThreads1 : kThreads2;
  const int consumers = consumers_for(MR);
  if (count < 1 || count > NP || n_stages < 1 || n_stages > kMaxChainStages) return cudaErrorInvalidValue;
  thread_local GemvLaunch<NP> L;
  uint32_t stage_bytes = 128;
  bool epi = false;
  int i = 0;
  for (int s = 0; s < n_stages; ++s) {
    L.stage_begin[s] = static_cast<uint16_t>(i);
    int64_t total = 0;
    for (int k = 0; k < stage_counts[s]; ++k, ++i) {
      if (i >= count) return cudaErrorInvalidValue;
      const GemvProblem& P = probs[i];
      if (!ring_stage_fits(P, MR, consumers, stage_bytes, 4, true)) return cudaErrorInvalidConfiguration;
      L.prob[i] = P;
      L.prob[i].byte_begin = total;
      total += P.N * problem_row_bytes(P);
      epi = epi || P.epi != kEpiNone || is_fused(P);
    }
    L.stage_total[s] = total;
  }
  if (i != count) return cudaErrorInvalidValue;
  L.stage_begin[n_stages] = static_cast<uint16_t>(count);
  int stages = 0;
  size_t smem = 0;
  if (!ring_of(stage_bytes, dev, &stages, &smem)) return cudaErrorInvalidConfiguration;
  L.count = count;
  L.consumer_threads = consumers;
  L.stages = stages;
  L.stage_bytes = stage_bytes;
  L.total_bytes = 0;
  L.n_stages = n_stages;
  L.done = done;
  const int grid = std::min(dev.sm_count, kMaxCtas);
  auto kern = epi ? gemv_kernel<MR, kThreads, NP, true, true, 4> : gemv_kernel<MR, kThreads, NP, false, true, 4>;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  count_launch();
  return cudaLaunchKernelEx(&cfg, kern, L);
}

// Launches in groups of at most kMaxProblems problems.
template <int MR, int BITS = 4>
cudaError_t run_problems(std::vector<GemvProblem>& probs, const DeviceInfo& dev, cudaStream_t stream) {
  for (size_t i = 0; i < probs.size(); i += kMaxProblems) {
    const int n = static_cast<int>(std::min<size_t>(kMaxProblems, probs.size() - i));
    cudaError_t e = (n <= kFewProblems) ? run_list<MR, kFewProblems, BITS>(probs.data() + i, n, dev, stream)
                                        : run_list<MR, kMaxProblems, BITS>(probs.data() + i, n, dev, stream);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace

cudaError_t gemv_device_flags(unsigned int* flags, bool clear) { return tu_device_flags(flags, clear); }

cudaError_t gemv_prepare_device(const DeviceInfo& dev) {
  for (const void* kern : {reinterpret_cast<const void*>(gemv_kernel<1, kThreads1, kFewProblems, false, false, 4>),
                           reinterpret_cast<const void*>(gemv_kernel<1, kThreads1, kFewProblems, true, false, 4>),
                           reinterpret_cast<const void*>(gemv_kernel<1, kThreads1, kMaxProblems, false, false, 4>),
                           reinterpret_cast<const void*>(gemv_kernel<1, kThreads1, kMaxProblems, true, false, 4>),
                           reinterpret_cast<const void*>(gemv_kernel<1, kThreads1, kMaxProblems, false, true, 4>),
                           reinterpret_cast<const void*>(gemv_kernel<1, kThreads1, kMaxProblems, true, true, 4>),
                           reinterpret_cast<const void*>(gemv_kernel<2, kThreads2, kFewProblems, false, false, 4>),
                           reinterpret_cast<const void*>(gemv_kernel<2, kThreads2, kFewProblems, true, false, 4>),
                           reinterpret_cast<const void*>(gemv_kernel<2, kThreads2, kMaxProblems, false, false, 4>),
                           reinterpret_cast<const void*>(gemv_kernel<2, kThreads2, kMaxProblems, true, false, 4>),
                           reinterpret_cast<const void*>(gemv_kernel<2, kThreads2, kMaxProblems, false, true, 4>),
                           reinterpret_cast<const void*>(gemv_kernel<2, kThreads2, kMaxProblems, true, true, 4>),
                           reinterpret_cast<const void*>(gemv_kernel<1, kThreads1, kFewProblems, false, false, 8>),
                           reinterpret_cast<const void*>(gemv_kernel<1, kThreads1, kFewProblems, true, false, 8>),
                           reinterpret_cast<const void*>(gemv_kernel<1, kThreads1, kMaxProblems, false, false, 8>),
                           reinterpret_cast<const void*>(gemv_kernel<1, kThreads1, kMaxProblems, true, false, 8>),
                           reinterpret_cast<const void*>(gemv_kernel<2, kThreads2, kFewProblems, false, false, 8>),
                           reinterpret_cast<const void*>(gemv_kernel<2, kThreads2, kFewProblems, true, false, 8>),
                           reinterpret_cast<const void*>(gemv_kernel<2, kThreads2, kMaxProblems, false, false, 8>),
                           reinterpret_cast<const void*>(gemv_kernel<2, kThreads2, kMaxProblems, true, false, 8>)}) {
    const cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(dev.smem_optin));
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

cudaError_t launch_gemv_batch(const MatmulArgs* list, int count, cudaStream_t stream, const DeviceInfo& dev) {
  // Activation rows in chunks of at most two; every chunk of every problem
  // that fits the bulk-copy kernel joins one list per chunk size.
  std::vector<GemvProblem> one, two;
  for (int i = 0; i < count; ++i) {
    const MatmulArgs& a = list[i];
    for (int64_t m0 = 0; m0 < a.M; m0 += 2) {
      const int mr = static_cast<int>(std::min<int64_t>(2, a.M - m0));
      if (!tma_ok(a, mr)) {
        cudaError_t e = (mr == 1) ? run_generic<1>(a, m0, dev, stream) : run_generic<2>(a, m0, dev, stream);
        if (e != cudaSuccess) return e;
        continue;
      }
      GemvProblem P;
      P.x = a.x + m0 * a.K;
      P.codes = a.codes;
      P.scales = a.scales;
      P.biases = a.biases;
      P.y = a.y + m0 * a.N;
      P.r = a.r ? a.r + m0 * a.N : nullptr;
      P.up_codes = a.up_codes;
      P.up_scales = a.up_scales;
      P.up_biases = a.up_biases;
      P.N = a.N;
      P.y_ld = a.N;
      P.K = static_cast<int32_t>(a.K);
      P.epi = a.epi;
      P.byte_begin = 0;
      (mr == 1 ? one : two).push_back(P);
    }
  }
  cudaError_t e = cudaSuccess;
  if (!one.empty()) e = run_problems<1>(one, dev, stream);
  if (e == cudaSuccess && !two.empty()) e = run_problems<2>(two, dev, stream);
  return e;
}

cudaError_t launch_gemv(const MatmulArgs& a, cudaStream_t stream, const DeviceInfo& dev) {
  return launch_gemv_batch(&a, 1, stream, dev);
}

bool gemv8_supported(const MatmulArgs& a) {
  if (a.fused() || a.epi != kEpiNone) return false;
  for (int mr = 1; mr <= 2 && mr <= a.M; ++mr)
    if (!tma_ok(a, mr, 8)) return false;
  return true;
}

cudaError_t launch_gemv8_batch(const MatmulArgs* list, int count, cudaStream_t stream, const DeviceInfo& dev) {
  std::vector<GemvProblem> one, two;
  for (int i = 0; i < count; ++i) {
    const MatmulArgs& a = list[i];
    for (int64_t m0 = 0; m0 < a.M; m0 += 2) {
      GemvProblem P;
      P.x = a.x + m0 * a.K;
      P.codes = a.codes;
      P.scales = a.scales;
      P.biases = a.biases;
      P.y = a.y + m0 * a.N;
      P.r = nullptr;
      P.up_codes = nullptr;
      P.up_scales = nullptr;
      P.up_biases = nullptr;
      P.N = a.N;
      P.y_ld = a.N;
      P.K = static_cast<int32_t>(a.K);
      P.epi = kEpiNone;
      P.byte_begin = 0;
      (a.M - m0 >= 2 ? two : one).push_back(P);
    }
  }
  cudaError_t e = cudaSuccess;
  if (!two.empty()) e = run_problems<2, 8>(two, dev, stream);
  if (e == cudaSuccess && !one.empty()) e = run_problems<1, 8>(one, dev, stream);
  return e;
}

bool gemv_chain_supported(const MatmulArgs* list, int count) {
  if (count < 1) return false;
  const int64_t M = list[0].M;
  if (M < 1 || M > 2) return false;
  for (int i = 0; i < count; ++i)
    if (list[i].M != M || !tma_ok(list[i], static_cast<int>(M))) return false;
  return true;
}

cudaError_t launch_gemv_chain(const MatmulArgs* list, int count, const int* stage_counts, int n_stages,
                              unsigned int* done, cudaStream_t stream, const DeviceInfo& dev) {
  if (count > kGemvChainMaxProblems || n_stages > kGemvChainMaxStages) return cudaErrorInvalidValue;
  GemvProblem probs[kGemvChainMaxProblems];
  for (int i = 0; i < count; ++i) {
    const MatmulArgs& a = list[i];
    GemvProblem& P = probs[i];
    P.x = a.x;
    P.codes = a.codes;
    P.scales = a.scales;
    P.biases = a.biases;
    P.y = a.y;
    P.r = a.r;
    P.up_codes = a.up_codes;
    P.up_scales = a.up_scales;
    P.up_biases = a.up_biases;
    P.N = a.N;
    P.y_ld = a.N;
    P.K = static_cast<int32_t>(a.K);
    P.epi = a.epi;
    P.byte_begin = 0;
  }
  return list[0].M == 1 ? run_chain<1>(probs, count, stage_counts, n_stages, done, dev, stream)
                        : run_chain<2>(probs, count, stage_counts, n_stages, done, dev, stream);
}

}  // namespace q4
