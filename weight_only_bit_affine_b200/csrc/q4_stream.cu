// q4_stream.cu -- tensor-core weight streaming for three to eight activation
// rows (batched decode): the affine Q4 group-32 matmul
//
//   y[m,n] = sum_k x[m,k] * w_hat[n,k],   w_hat = s*q + b  (group 32 along k)
//
// with the products and the fp32 accumulation done by the 5th-generation
// tensor cores (tcgen05.mma, kind::f16) and the CUDA cores doing nothing but
// the dequantization, whatever the number of activation rows.  At these row
// counts the CUDA-core GEMV, which works on pairs of rows, would read the
// weights once per pair and multiply every weight by every row on the CUDA
// cores; this kernel reads them once and the rows cost tensor-core time only.
// Each weight enters the MMA as two bf16 parts hi + lo (q4_tcgen05.cuh,
// dequant_word_hilo), within ~2^-16 of the exact s*q + b.
//
// Segmented-K tiles.  The MMA's 128 rows (tensor-memory lanes) are not 128
// weight rows: a tile is R weight rows x `segs` segments of K (R * segs =
// 128; segs = 8, 16 or 32, so a segment is K / segs long), and lane
// r * segs + s holds the dequantized weights of row r, segment s, as the
// MMA's A operand in tensor memory.  The B operand is the activation rows cut
// the same way: row (m, s') of B is x[m, segment s'], so
//
//   D[lane (r, s), column (m, s')] = sum over segment s of w_hat[r, .] * x[m, segment s'],
//
// and the wanted partial sums are the "diagonal" columns s' = s; the
// off-diagonal columns are tensor-core work thrown away (the tensor cores
// have an order of magnitude to spare at these shapes).  A tile is R whole
// weight rows, contiguous in memory, so a tile arrives with three 1-D bulk
// copies (codes, scales, biases) exactly as the GEMV streams it (any mix of
// problems in one persistent launch, no tensor maps), and B is built once per
// problem in shared memory.  Because each lane keeps only its own column, the
// order of k inside a segment is free per segment: lane (r, s) takes its
// segment's 16-byte code runs rotated by s, so the eight lanes of a
// shared-memory phase (eight segments of one row) read eight different banks,
// and B holds each segment's x in the same rotated order.  The segments of a
// row sit in one warp, so the epilogue sums them with shuffles.
//
// SwiGLU (gate and up weights of the same shape) in one pass: each tile of a
// SwiGLU problem is two consecutive "virtual" tiles, the gate's R rows and
// then the same rows of the up weight; the epilogue keeps the gate's fp32
// sums in registers and writes silu(gate) * up when the up tile completes.
//
// Per CTA (one per SM, 608 threads):
//   warp 0       producer: three bulk copies per tile;
//   warps 1..2   MMA issue (warp 1 also allocates tensor memory): issuer i
//                takes chunks c == i (mod I) of every tile (I = 2 or 1 by
//                the problem's accumulator width) into its own double-buffered
//                fp32 tile.  One thread issues an MMA of these shapes only
//                every ~50 cycles (its instruction stream, not the tensor
//                core, is the limit), so several issuers keep pace with the
//                weight stream.  The split depends on the problem alone, so a
//                result never depends on the batch;
//   warps 3..14  dequantize: three groups of four warps (one warp per
//                tensor-memory lane quarter) take 64-wide K chunks in turn;
//                a thread turns 64 codes of its (row, segment) into 32 hi and
//                32 lo bf16 pairs (dequant_word_hilo) and stores them to
//                tensor memory (tcgen05.st);
//   warps 15..18 epilogue: per tile, read the diagonals of the issuers' fp32
//                tiles from tensor memory, sum them and the segments
//                (shuffles), write bf16 y; and, at each new problem, lay out
//                its B operand.
// Within a 16-byte run the order of k is natural in both operands (a
// tensor-memory column holds the bf16 pair k = 2i, 2i + 1).
// Every wait is bounded (q4_device.cuh); a thread whose wait gave up writes
// NaN.  Programmatic dependent launch as in the GEMV family.
#include "q4_device.cuh"
#include "q4_internal.h"
#include "q4_tcgen05.cuh"

#include <algorithm>
#include <cstdint>
#include <vector>

#ifndef Q4_STREAM_WAIT_SLEEP
#define Q4_STREAM_WAIT_SLEEP 1
#endif

namespace q4 {
namespace {

constexpr bool kSleepWaits = Q4_STREAM_WAIT_SLEEP != 0;

constexpr int kLanes = 128;                                  // tensor-memory lanes = MMA rows
constexpr int kChunkK = 64;                                  // K per lane per A chunk
constexpr int kChunkCols = 64;                               // A chunk in tensor memory: hi (32 columns), lo (32)
#ifndef Q4_STREAM_DQ_GROUPS
#define Q4_STREAM_DQ_GROUPS 3
#endif
// Dequantizing warp groups (4 warps each, one per tensor-memory lane quarter).
// Three keep the CTA at 19 warps, at most 5 per SM sub-partition, which
// leaves 96 registers a thread (at 23 warps it would be 80, and the
// dequantization spills).
constexpr int kGroups = Q4_STREAM_DQ_GROUPS;
constexpr int kMaxIssuers = 2;                               // MMA-issuing warps
constexpr int kFirstDqWarp = 1 + kMaxIssuers;                // 3
constexpr int kFirstEpiWarp = kFirstDqWarp + 4 * kGroups;   // 15 with three groups
constexpr int kThreads = 32 * (kFirstEpiWarp + 4);           // 608 with three dequantizing groups
constexpr int kMaxRows = kStreamMaxRows;                     // activation rows per launch
constexpr int kMinRows = kStreamMinRows;  // below this the CUDA-core GEMV is faster (it reads the weights once for 1-2 rows)
constexpr uint32_t kTmemCols = 512;
constexpr int kMaxASlots = 8;   // A ring in tensor memory: up to 8 chunks of 64 columns
constexpr int kMaxStages = 12;
constexpr int kMaxProblems = 256;
constexpr int kFewProblems = 4;
constexpr int kMaxCtas = 256;  // CTAs per launch at most (one per SM)
constexpr float kNaN = __builtin_nanf("");

struct StreamProblem {
  const uint16_t* x;  // [M, K]
  const uint8_t* codes;
  const uint16_t* scales;
  const uint16_t* biases;
  const uint8_t* up_codes;  // SwiGLU: the up weight (NULL otherwise)
  const uint16_t* up_scales;
  const uint16_t* up_biases;
  uint16_t* y;         // [M, N]
  const uint16_t* r;   // residual [M, N] (kEpiResidual), else NULL
  int64_t N;
  int64_t byte_begin;  // work offset of the first tile (packed bytes of all tiles before)
  int32_t K;
  int32_t segs;        // K segments per weight row; R = 128 / segs rows per tile
  int32_t tile_bytes;  // packed bytes of a full tile (both weights for SwiGLU): the unit of work balancing
  int32_t epi;         // output epilogue (q4_internal.h)
};

template <int NP>
struct StreamLaunch {
  int32_t count, M, stages, a_slots;  // a_slots: A ring chunks (a multiple of kGroups)
  uint32_t stage_bytes, b_bytes, a_col0, pad_;  // a_col0: first A ring column (after the accumulators)
  int64_t total_bytes;
  // first[c]: the first problem with a tile of CTA c (launches of more than
  // kFewProblems problems).  Every role walks the list from there and stops
  // at the first problem that starts at or after the CTA's last byte, so it
  // reads only its own problems' descriptors (each read of another problem's
  // is a constant-cache miss).
  uint16_t first[NP > kFewProblems ? kMaxCtas : 1];
  StreamProblem prob[NP];
};

__device__ __forceinline__ bool is_swiglu(const StreamProblem& P) { return P.up_codes != nullptr; }

template <int W>
__device__ __forceinline__ float pick(const uint32_t (&r)[W], int sel) {
  uint32_t v = r[0];
#pragma unroll
  for (int i = 1; i < W; ++i) v = (sel == i) ? r[i] : v;
  return __uint_as_float(v);
}

// part[m] += sum over the issuers in `mask` of column m * W + sel of this
// lane's accumulator tiles (W = segs: the lane's own segment's column).
template <int W>
__device__ __forceinline__ void gather_diag(uint32_t base, uint32_t issuer_stride, uint32_t mask, int I, int M,
                                            int sel, float (&part)[kMaxRows]) {
  for (int i = 0; i < I; ++i) {
    if (!((mask >> i) & 1u)) continue;
#pragma unroll
    for (int m = 0; m < kMaxRows; ++m)
      if (m < M) {
        // W columns in pieces of at most 16 (registers), both loads before one wait
        constexpr int P = W < 16 ? W : 16;
        uint32_t r[P], r2[P];
        const uint32_t col = base + static_cast<uint32_t>(i) * issuer_stride + static_cast<uint32_t>(m * W);
        if constexpr (W <= 16) {
          tmem_ld_cols<P>(col, r);
          tmem_wait_ld();
          part[m] += pick<P>(r, sel);
        } else {
          tmem_ld_cols<P>(col, r);
          tmem_ld_cols<P>(col + P, r2);
          tmem_wait_ld();
          part[m] += sel < P ? pick<P>(r, sel) : pick<P>(r2, sel - P);
        }
      }
  }
}

struct ProblemShape {
  int segs, R, kseg, pieces, chunks, full_chunks, nb, issuers;
  uint32_t dstride;  // columns per accumulator tile
  __device__ __forceinline__ ProblemShape(const StreamProblem& P, int M) {
    segs = P.segs;
    R = kLanes / segs;
    kseg = P.K / segs;
    pieces = kseg / 32;  // 16-byte code runs (one group each) per segment
    chunks = (kseg + kChunkK - 1) / kChunkK;
    full_chunks = kseg / kChunkK;  // the last chunk may be 32 wide
    nb = (segs * M + 15) & ~15;  // MMA N (B rows), a multiple of 16, at most 128
    issuers = nb <= 32 ? 2 : 1;
    dstride = static_cast<uint32_t>(nb);
  }
};

// The tiles of problem p that this CTA owns: those whose first byte (in the
// work order of all problems' tiles) falls in [lo, hi).  A SwiGLU problem's
// tile is its gate and up rows together, so the two always go to one CTA.
__device__ __forceinline__ void tile_range(const StreamProblem& P, int64_t lo, int64_t hi, int64_t& j0, int64_t& j1) {
  const int64_t R = kLanes / P.segs;
  const int64_t tiles = (P.N + R - 1) / R;
  auto first_from = [&](int64_t b) -> int64_t {
    const int64_t d = b - P.byte_begin;
    if (d <= 0) return 0;
    const int64_t j = (d + P.tile_bytes - 1) / P.tile_bytes;
    return j < tiles ? j : tiles;
  };
  j0 = first_from(lo);
  j1 = first_from(hi);
}

// Virtual tiles (v) of problem P for this CTA: [v0, v1); v maps to weight
// tile v >> sh and, for SwiGLU (sh = 1), to the gate (v even) or up (v odd).
__device__ __forceinline__ void vtile_range(const StreamProblem& P, int64_t lo, int64_t hi, int64_t& v0, int64_t& v1,
                                            int& sh) {
  int64_t j0, j1;
  tile_range(P, lo, hi, j0, j1);
  sh = is_swiglu(P) ? 1 : 0;
  v0 = j0 << sh;
  v1 = j1 << sh;
}

template <int NP, bool EPI>
__global__ void __launch_bounds__(kThreads, 1) stream_kernel(const __grid_constant__ StreamLaunch<NP> L) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* bmat = smem;               // B operand of the current problem, b_bytes (a multiple of 1024)
  uint8_t* ring = smem + L.b_bytes;   // stages x stage_bytes
  uint64_t* full = reinterpret_cast<uint64_t*>(ring + static_cast<size_t>(L.stages) * L.stage_bytes);
  uint64_t* empty = full + kMaxStages;
  // A chunk written: one set per issuer (chunk c of a tile goes to issuer
  // c % issuers).  With a single set, consecutive uses of a slot could belong
  // to different issuers (the chunk count per tile varies over a launch's
  // problems), and an issuer one use ahead would see the parity of the use
  // before the one it waits for still in progress as "complete".  Per issuer,
  // its own uses of a slot complete in order and at most one ahead of it.
  uint64_t* afull = empty + kMaxStages;                // [kMaxIssuers][kMaxASlots]
  uint64_t* aempty = afull + kMaxIssuers * kMaxASlots;
  uint64_t* dfull = aempty + kMaxASlots;
  uint64_t* dempty = dfull + 2;
  uint64_t* bfull = dempty + 2;
  uint64_t* bempty = bfull + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bempty + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int s = 0; s < L.stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 4 * kGroups);
    }
    for (int a = 0; a < L.a_slots; ++a) {
      for (int i = 0; i < kMaxIssuers; ++i) mbar_init(&afull[i * kMaxASlots + a], 4);
      mbar_init(&aempty[a], 1);
    }
    for (int d = 0; d < 2; ++d) {
      mbar_init(&dfull[d], kMaxIssuers);
      mbar_init(&dempty[d], 4);
    }
    mbar_init(bfull, 4);
    mbar_init(bempty, kMaxIssuers);
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // tensor-memory columns: the accumulator tiles (per issuer, double-buffered), then the A ring
  const uint32_t a_col0 = L.a_col0;
  const int A = L.a_slots;

  const int64_t G = gridDim.x;
  const int64_t lo = L.total_bytes * static_cast<int64_t>(blockIdx.x) / G;
  const int64_t hi = L.total_bytes * (static_cast<int64_t>(blockIdx.x) + 1) / G;
  const int p0 = NP > kFewProblems ? L.first[blockIdx.x] : 0;

  pdl_launch_dependents();
  if (warp == 0 && lane == 0) {
    // Before the wait: pull the first tile's codes toward L2 (a hint only).
    for (int p = p0; p < L.count && L.prob[p].byte_begin < hi; ++p) {
      const StreamProblem& P = L.prob[p];
      int64_t j0, j1;
      tile_range(P, lo, hi, j0, j1);
      if (j0 < j1) {
        const int64_t R = kLanes / P.segs;
        const int64_t rows = (P.N - j0 * R < R) ? P.N - j0 * R : R;
        bulk_prefetch_l2(P.codes + j0 * R * (P.K / 2), static_cast<uint32_t>(rows * (P.K / 2)));
        break;
      }
    }
  }
  pdl_wait_predecessors();

  if (warp == 0) {
    // ---------------- producer ----------------
    bool dead = false;
    int s = 0;
    uint32_t ph = 0;
    for (int p = p0; p < L.count && L.prob[p].byte_begin < hi; ++p) {
      const StreamProblem& P = L.prob[p];
      int64_t v0, v1;
      int sh;
      vtile_range(P, lo, hi, v0, v1, sh);
      const int R = kLanes / P.segs;
      const uint32_t row_bytes = static_cast<uint32_t>(P.K / 2), sb_row = static_cast<uint32_t>(P.K / 16);
      for (int64_t v = v0; v < v1; ++v) {
        if (lane == 0) {
          if (!dead && !mbar_wait<kSleepWaits>(&empty[s], ph ^ 1u)) dead = true;
          const int64_t row0 = (v >> sh) * R;
          const bool up = sh && (v & 1);
          const uint32_t rows = static_cast<uint32_t>((P.N - row0 < R) ? P.N - row0 : R);
          uint8_t* st = ring + static_cast<size_t>(s) * L.stage_bytes;
          mbar_arrive_expect_tx(&full[s], rows * (row_bytes + 2 * sb_row));
          // the tile's codes, scales and biases: three contiguous runs
          bulk_g2s(st, (up ? P.up_codes : P.codes) + row0 * row_bytes, rows * row_bytes, &full[s]);
          bulk_g2s(st + R * row_bytes, (up ? P.up_scales : P.scales) + row0 * (P.K / 32), rows * sb_row, &full[s]);
          bulk_g2s(st + R * (row_bytes + sb_row), (up ? P.up_biases : P.biases) + row0 * (P.K / 32), rows * sb_row,
                   &full[s]);
        }
        if (++s == L.stages) { s = 0; ph ^= 1u; }
      }
    }
  } else if (warp <= kMaxIssuers) {
    // ---------------- MMA issuers ----------------
    // The whole warp runs the loop (warp-uniform operands); the elected lane
    // issues the MMAs and commits.
    const int me = warp - 1;
    const bool leader = elect_one();
    {
      bool dead = false;
      int lp = 0;
      int slot0 = 0;      // A ring slot of the current tile's first chunk
      int64_t gt = 0;
      uint32_t aph = 0;  // bit a: parity of this issuer's next use of A slot a
      const uint64_t bdesc0 = sw128_desc(smem_u32(bmat));
      const uint32_t a_base = tmem + a_col0;
      for (int p = p0; p < L.count && L.prob[p].byte_begin < hi; ++p) {
        const StreamProblem& P = L.prob[p];
        int64_t v0, v1;
        int sh;
        vtile_range(P, lo, hi, v0, v1, sh);
        if (v0 >= v1) continue;
        const ProblemShape S(P, L.M);
        const bool active = me < S.issuers;
        const uint32_t idesc = idesc_bf16_m128(S.nb);
        const uint32_t atom16 = static_cast<uint32_t>(S.nb) * 128u >> 4;  // B atom size in 16-byte units
        // B of the previous problem is free once its MMAs are done.  Waiting
        // for this problem's B also means the epilogue has drained every
        // earlier tile, so the accumulator layout may change here.
        if (lp > 0 && leader) tc_commit(bempty);
        if (!dead && !mbar_wait<kSleepWaits>(bfull, static_cast<uint32_t>(lp & 1))) dead = true;
        tc_fence_after();
        for (int64_t v = v0; v < v1; ++v, ++gt) {
          const int db = static_cast<int>(gt & 1);
          const uint32_t dt = tmem + static_cast<uint32_t>(2 * me + db) * S.dstride;
          // every issuer waits, so none can arrive twice on one phase of dfull
          if (!dead && !mbar_wait<kSleepWaits>(&dempty[db], static_cast<uint32_t>((gt >> 1) & 1) ^ 1u)) dead = true;
          tc_fence_after();
          if (active) {
            for (int c = me; c < S.chunks; c += S.issuers) {
              int slot = slot0 + c;  // ring slot of chunk c
              while (slot >= A) slot -= A;
              if (!dead && !mbar_wait<kSleepWaits>(&afull[me * kMaxASlots + slot], (aph >> slot) & 1u)) dead = true;
              aph ^= 1u << slot;
              tc_fence_after();
              const uint32_t at = a_base + static_cast<uint32_t>(slot) * kChunkCols;
              const uint64_t bd = bdesc0 + static_cast<uint64_t>(c) * atom16;
              if (leader) {
                // the first MMA of this issuer in the tile overwrites its accumulator
                const uint32_t acc0 = c >= S.issuers ? 1u : 0u;
                if (c < S.full_chunks) {  // 64 k: four K16 steps of hi, then of lo
#pragma unroll
                  for (int kk = 0; kk < 4; ++kk) tc_mma_ts(dt, at + 8u * kk, bd + 2u * kk, idesc, kk ? 1u : acc0);
#pragma unroll
                  for (int kk = 0; kk < 4; ++kk) tc_mma_ts(dt, at + 32u + 8u * kk, bd + 2u * kk, idesc, 1u);
                } else {  // the segment's last 32 k
#pragma unroll
                  for (int kk = 0; kk < 2; ++kk) tc_mma_ts(dt, at + 8u * kk, bd + 2u * kk, idesc, kk ? 1u : acc0);
#pragma unroll
                  for (int kk = 0; kk < 2; ++kk) tc_mma_ts(dt, at + 32u + 8u * kk, bd + 2u * kk, idesc, 1u);
                }
                tc_commit(&aempty[slot]);
              }
              __syncwarp();
            }
          }
          // every issuer, every tile (count kMaxIssuers); an idle issuer's
          // commit arrives once its earlier MMAs are complete
          if (leader) tc_commit(&dfull[db]);
          __syncwarp();
          slot0 += S.chunks;
          while (slot0 >= A) slot0 -= A;
        }
        ++lp;
      }
    }
  } else if (warp < kFirstEpiWarp) {
    // ---------------- dequantize ----------------
    const int quarter = warp & 3;
    const int grp = (warp - kFirstDqWarp) >> 2;
    const int tl = 32 * quarter + lane;  // tensor-memory lane of this thread
    const uint32_t a_addr = tmem + (static_cast<uint32_t>(32 * quarter) << 16) + a_col0;
    bool dead = false;
    int s = 0;
    uint32_t ph = 0;
    int gmod = 0;             // chunks of this CTA before the current tile, mod kGroups
    int slot0 = 0;            // A ring slot of the current tile's first chunk
    uint32_t ph0 = 0;         // and its phase
    for (int p = p0; p < L.count && L.prob[p].byte_begin < hi; ++p) {
      const StreamProblem& P = L.prob[p];
      int64_t v0, v1;
      int sh;
      vtile_range(P, lo, hi, v0, v1, sh);
      if (v0 >= v1) continue;
      const ProblemShape S(P, L.M);
      const int r = tl / S.segs, seg = tl % S.segs;  // this lane: row r, segment seg
      const int rot = seg % S.pieces;                  // its code runs, rotated by seg
      const int groups = P.K / 32;
      for (int64_t v = v0; v < v1; ++v, gmod = (gmod + S.chunks) % kGroups) {
        if (!dead && !mbar_wait<kSleepWaits>(&full[s], ph)) dead = true;
        const uint8_t* st = ring + static_cast<size_t>(s) * L.stage_bytes;
        const uint8_t* crow = st + r * (P.K / 2) + seg * (S.kseg / 2);  // the segment's 16-byte code runs
        const uint16_t* srow = reinterpret_cast<const uint16_t*>(st + S.R * (P.K / 2)) + r * groups + seg * S.pieces;
        const uint16_t* brow = srow + S.R * groups;
        // the chunks of this group: global index == grp (mod kGroups)
        for (int c = (grp - gmod + kGroups) % kGroups; c < S.chunks; c += kGroups) {
          int slot = slot0 + c;  // ring slot and phase of chunk c
          uint32_t sph = ph0;
          while (slot >= A) { slot -= A; sph ^= 1u; }
          if (!dead && !mbar_wait<kSleepWaits>(&aempty[slot], sph ^ 1u)) dead = true;
          tc_fence_after();
          const uint32_t taddr = a_addr + static_cast<uint32_t>(slot) * kChunkCols;
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            if (h == 0 || c < S.full_chunks) {
              // position 2c + h of the segment holds its code run (2c + h + seg) mod pieces
              int run = 2 * c + h + rot;
              if (run >= S.pieces) run -= S.pieces;
              const uint4 cw = *reinterpret_cast<const uint4*>(crow + 16 * run);
              const uint64_t s2 = f32x2_splat(bf16_bits_to_float(srow[run]));
              const uint64_t b2 = f32x2_splat(bf16_bits_to_float(brow[run]));
              // 16 codes at a time (the register budget of 768 threads)
              uint32_t hh[8], ll[8];
              dequant_word_hilo(cw.x, s2, b2, hh + 0, ll + 0);
              dequant_word_hilo(cw.y, s2, b2, hh + 4, ll + 4);
              tmem_st_x8(taddr + 16u * h, hh);
              tmem_st_x8(taddr + 32u + 16u * h, ll);
              dequant_word_hilo(cw.z, s2, b2, hh + 0, ll + 0);
              dequant_word_hilo(cw.w, s2, b2, hh + 4, ll + 4);
              tmem_st_x8(taddr + 16u * h + 8u, hh);
              tmem_st_x8(taddr + 32u + 16u * h + 8u, ll);
            }
          }
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&afull[(c % S.issuers) * kMaxASlots + slot]);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);  // this warp's reads of the stage are done
        if (++s == L.stages) { s = 0; ph ^= 1u; }
        slot0 += S.chunks;
        while (slot0 >= A) { slot0 -= A; ph0 ^= 1u; }
      }
    }
  } else {
    // ---------------- epilogue (and B operand layout) ----------------
    const int quarter = warp & 3;
    const int et = tid - 32 * kFirstEpiWarp;  // 0..127
    const uint32_t lane_addr = static_cast<uint32_t>(32 * quarter) << 16;
    const int tl = 32 * quarter + lane;
    bool dead = false;
    int lp = 0;
    int64_t gt = 0;
    for (int p = p0; p < L.count && L.prob[p].byte_begin < hi; ++p) {
      const StreamProblem& P = L.prob[p];
      int64_t v0, v1;
      int sh;
      vtile_range(P, lo, hi, v0, v1, sh);
      if (v0 >= v1) continue;
      const ProblemShape S(P, L.M);
      // B: atom c (positions 2c, 2c + 1 of every segment: 64 k) holds rows
      // n = m * segs + s' of 128 bytes, 16-byte runs swizzled as the MMA's
      // 128-byte layout expects; position p of segment s' holds its x run
      // (p + s') mod pieces, as the dequantizing lanes take the code runs.
      // Rows beyond segs * M, and positions beyond the segment, are zero.
      if (lp > 0 && !dead && !mbar_wait<kSleepWaits>(bempty, static_cast<uint32_t>((lp - 1) & 1))) dead = true;
      {
        // four 16-byte runs per thread in flight at a time (their loads first)
        const int runs = S.chunks * S.nb * 8;
        for (int i0 = et; i0 < runs; i0 += 4 * 128) {
          uint4 v[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int i = i0 + 128 * u;
            const int run = i & 7, n = (i >> 3) % S.nb, c = (i >> 3) / S.nb;
            const int pos = 2 * c + (run >> 2);  // 32-wide position within the segment
            v[u] = make_uint4(0, 0, 0, 0);
            if (i < runs && n < S.segs * L.M && pos < S.pieces) {
              const int m = n / S.segs, sp = n % S.segs;
              int src = pos + sp % S.pieces;
              if (src >= S.pieces) src -= S.pieces;
              v[u] = *reinterpret_cast<const uint4*>(P.x + static_cast<int64_t>(m) * P.K +
                                                    static_cast<int64_t>(sp) * S.kseg + 32 * src + 8 * (run & 3));
            }
          }
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int i = i0 + 128 * u;
            if (i < runs) {
              const int run = i & 7, n = (i >> 3) % S.nb, c = (i >> 3) / S.nb;
              *reinterpret_cast<uint4*>(bmat + static_cast<size_t>(c) * S.nb * 128 + n * 128 + ((run ^ (n & 7)) << 4)) =
                  v[u];
            }
          }
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(bfull);

      const int seg = tl % S.segs;          // this lane's segment: its column of every accumulator tile
      const int rq = tl / S.segs;           // its row within the tile
      // issuers with chunks in a tile (the others' accumulators hold an older tile)
      const int I = S.issuers;
      const uint32_t mask = (1u << (S.chunks < I ? S.chunks : I)) - 1u;
      float gate[kMaxRows];  // SwiGLU: the gate's sums of the current tile, kept for its up tile
#pragma unroll
      for (int m = 0; m < kMaxRows; ++m) gate[m] = 0.f;
      for (int64_t v = v0; v < v1; ++v, ++gt) {
        const int db = static_cast<int>(gt & 1);
        if (!dead && !mbar_wait<kSleepWaits>(&dfull[db], static_cast<uint32_t>((gt >> 1) & 1))) dead = true;
        tc_fence_after();
        float part[kMaxRows];
#pragma unroll
        for (int m = 0; m < kMaxRows; ++m) part[m] = 0.f;
        const uint32_t dbase = tmem + lane_addr + static_cast<uint32_t>(db) * S.dstride;
        const uint32_t istride = 2 * S.dstride;
        if (S.segs == 8) gather_diag<8>(dbase, istride, mask, I, L.M, seg, part);
        else if (S.segs == 16) gather_diag<16>(dbase, istride, mask, I, L.M, seg, part);
        else gather_diag<32>(dbase, istride, mask, I, L.M, seg, part);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&dempty[db]);
        // sum the row's segments: lanes r * segs .. r * segs + segs - 1 of this warp
#pragma unroll
        for (int m = 0; m < kMaxRows; ++m)
          for (int o = 1; o < S.segs; o <<= 1) part[m] += __shfl_xor_sync(0xFFFFFFFFu, part[m], o);
        if (sh && !(v & 1)) {  // a SwiGLU gate tile: keep its sums for the up tile that follows
#pragma unroll
          for (int m = 0; m < kMaxRows; ++m) gate[m] = part[m];
          continue;
        }
        const int64_t row = (v >> sh) * S.R + rq;
        if (seg == 0 && row < P.N) {
#pragma unroll
          for (int m = 0; m < kMaxRows; ++m)
            if (m < L.M) {
              const int64_t idx = static_cast<int64_t>(m) * P.N + row;
              const float val = dead ? kNaN : part[m];
              if constexpr (EPI) {
                if (sh) P.y[idx] = float_to_bf16_bits(silu_f32(gate[m]) * val);
                else P.y[idx] = epilogue_bf16(val, P.epi, P.r, idx);
              } else {
                P.y[idx] = float_to_bf16_bits(val);
              }
            }
        }
      }
      ++lp;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ---------------------------------------------------------------- host side

// Segments per weight row: K / segs must be a multiple of 32 (whole groups,
// 16-byte code runs).  Fewer segments mean more rows per tile and fewer
// epilogues per byte; the tile must still leave room for three stages.
uint32_t stage_bytes_of(int64_t K, int segs) {
  const int64_t R = kLanes / segs;
  return static_cast<uint32_t>((R * (K / 2 + K / 8) + 127) & ~int64_t(127));
}
int segs_for(int64_t K) {
  if (K % 256 != 0) return 0;
  for (int s : {8, 16, 32})
    if (K % (32 * s) == 0 && 3 * stage_bytes_of(K, s) <= 168 * 1024) return s;
  return 0;
}

struct Plan {
  int segs = 0;
  uint32_t stage_bytes = 0, b_bytes = 0, nb = 0;
};

Plan plan_of(const MatmulArgs& a) {
  Plan pl;
  pl.segs = segs_for(a.K);
  if (pl.segs == 0) return pl;
  const int64_t kseg = a.K / pl.segs;
  pl.stage_bytes = stage_bytes_of(a.K, pl.segs);
  pl.nb = static_cast<uint32_t>((pl.segs * a.M + 15) & ~int64_t(15));
  const int64_t chunks = (kseg + kChunkK - 1) / kChunkK;
  pl.b_bytes = static_cast<uint32_t>(((chunks * pl.nb * 128) + 1023) & ~int64_t(1023));
  return pl;
}

constexpr size_t kFixedSmem = 1024 /* alignment */ + 8 * (2 * kMaxStages + (kMaxIssuers + 1) * kMaxASlots + 6) + 16;

uint32_t acc_cols_of(uint32_t nb) {
  const uint32_t issuers = nb <= 32 ? 2u : 1u;  // as ProblemShape
  return 2u * issuers * nb;
}

template <int NP>
cudaError_t run_stream(const MatmulArgs* list, int count, const DeviceInfo& dev, cudaStream_t stream) {
  static_assert(sizeof(StreamLaunch<NP>) <= 32000, "kernel parameters exceed the launch limit");
  thread_local StreamLaunch<NP> L;
  uint32_t stage_bytes = 128, b_bytes = 1024, acc_cols = 0;
  int64_t total = 0, tiles = 0;
  for (int i = 0; i < count; ++i) {
    const MatmulArgs& a = list[i];
    const Plan pl = plan_of(a);
    StreamProblem& P = L.prob[i];
    P.x = a.x;
    P.codes = a.codes;
    P.scales = a.scales;
    P.biases = a.biases;
    P.up_codes = a.up_codes;
    P.up_scales = a.up_scales;
    P.up_biases = a.up_biases;
    P.y = a.y;
    P.r = a.r;
    P.epi = a.epi;
    P.N = a.N;
    P.K = static_cast<int32_t>(a.K);
    P.segs = pl.segs;
    const int R = kLanes / pl.segs;
    P.tile_bytes = static_cast<int32_t>(R * (a.K / 2 + a.K / 8) * (a.fused() ? 2 : 1));
    P.byte_begin = total;
    const int64_t t = (a.N + R - 1) / R;
    total += t * P.tile_bytes;
    tiles += t;
    stage_bytes = std::max(stage_bytes, pl.stage_bytes);
    acc_cols = std::max(acc_cols, acc_cols_of(pl.nb));
    b_bytes = std::max(b_bytes, pl.b_bytes);
  }
  const size_t avail = dev.smem_optin - kFixedSmem - b_bytes;
  const int stages = static_cast<int>(std::min<size_t>(kMaxStages, avail / stage_bytes));
  if (stages < 2) return cudaErrorInvalidConfiguration;
  L.count = count;
  L.M = static_cast<int32_t>(list[0].M);
  L.stages = stages;
  L.pad_ = 0;
  // Tensor memory: the accumulator tiles of the widest problem, then as deep an
  // A ring as the rest holds (a multiple of kGroups chunks: the chunk of global
  // index c takes slot c mod a_slots and belongs to group c mod kGroups, so each
  // group owns its slots and never waits for another group's).
  L.a_col0 = (acc_cols + 31u) & ~31u;
  L.a_slots = static_cast<int32_t>(std::min<uint32_t>(kMaxASlots, (kTmemCols - L.a_col0) / kChunkCols) / kGroups *
                                   kGroups);
  if (L.a_slots < kGroups) return cudaErrorInvalidConfiguration;
  L.stage_bytes = stage_bytes;
  L.b_bytes = b_bytes;
  L.total_bytes = total;
  // All of the SM's shared memory: one CTA per SM (each allocates all 512
  // tensor-memory columns).
  const size_t smem = dev.smem_optin;
  const int grid =
      static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(std::min(dev.sm_count, kMaxCtas), tiles)));
  // each CTA's first problem: the first whose tiles end after the CTA's first
  // byte (the kernel's byte range formula)
  for (int64_t c = 0, i = 0; c < grid && NP > kFewProblems; ++c) {
    const int64_t lo = total * c / grid;
    while (i < count && L.prob[i].byte_begin + (L.prob[i].N + kLanes / L.prob[i].segs - 1) /
                                                   (kLanes / L.prob[i].segs) * L.prob[i].tile_bytes <= lo)
      ++i;
    L.first[c] = static_cast<uint16_t>(i);
  }
  bool epi = false;
  for (int i = 0; i < count; ++i) epi = epi || list[i].epi != kEpiNone || list[i].fused();
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  count_launch();
  return epi ? cudaLaunchKernelEx(&cfg, stream_kernel<NP, true>, L) : cudaLaunchKernelEx(&cfg, stream_kernel<NP, false>, L);
}

}  // namespace

cudaError_t stream_device_flags(unsigned int* flags, bool clear) { return tu_device_flags(flags, clear); }

cudaError_t stream_prepare_device(const DeviceInfo& dev) {
  for (const void* kern : {reinterpret_cast<const void*>(stream_kernel<kFewProblems, false>),
                           reinterpret_cast<const void*>(stream_kernel<kFewProblems, true>),
                           reinterpret_cast<const void*>(stream_kernel<kMaxProblems, false>),
                           reinterpret_cast<const void*>(stream_kernel<kMaxProblems, true>)}) {
    cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(dev.smem_optin));
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

bool stream_supported(const MatmulArgs& a, const DeviceInfo& dev) {
  if (a.M < kMinRows || a.M > kMaxRows) return false;
  uintptr_t sb = reinterpret_cast<uintptr_t>(a.scales) | reinterpret_cast<uintptr_t>(a.biases);
  if (a.fused()) sb |= reinterpret_cast<uintptr_t>(a.up_scales) | reinterpret_cast<uintptr_t>(a.up_biases);
  if (sb & 15u) return false;
  if (a.K > (int64_t(1) << 20)) return false;
  const Plan pl = plan_of(a);
  if (pl.segs == 0 || pl.nb > 128) return false;
  if ((kTmemCols - ((acc_cols_of(pl.nb) + 31u) & ~31u)) / kChunkCols < static_cast<uint32_t>(kGroups)) return false;
  return kFixedSmem + pl.b_bytes + 2 * static_cast<size_t>(pl.stage_bytes) <= dev.smem_optin;
}

// Problems share a launch while their combined layout fits: every problem
// fits alone (stream_supported), but the largest stage of one and the
// largest B operand of another may not fit together.
bool fits_together(uint32_t stage_bytes, uint32_t b_bytes, uint32_t acc_cols, const DeviceInfo& dev) {
  if (kFixedSmem + b_bytes + 2 * static_cast<size_t>(stage_bytes) > dev.smem_optin) return false;
  return (kTmemCols - ((acc_cols + 31u) & ~31u)) / kChunkCols >= static_cast<uint32_t>(kGroups);
}

cudaError_t launch_stream_batch(const MatmulArgs* list, int count, cudaStream_t stream, const DeviceInfo& dev) {
  int i = 0;
  while (i < count) {
    uint32_t sb = 0, bb = 0, ac = 0;
    int n = 0;
    while (i + n < count && n < kMaxProblems) {
      const Plan pl = plan_of(list[i + n]);
      const uint32_t sb2 = std::max(sb, pl.stage_bytes), bb2 = std::max(bb, pl.b_bytes),
                     ac2 = std::max(ac, acc_cols_of(pl.nb));
      if (n > 0 && !fits_together(sb2, bb2, ac2, dev)) break;
      sb = sb2;
      bb = bb2;
      ac = ac2;
      ++n;
    }
    cudaError_t e = (n <= kFewProblems) ? run_stream<kFewProblems>(list + i, n, dev, stream)
                                        : run_stream<kMaxProblems>(list + i, n, dev, stream);
    if (e != cudaSuccess) return e;
    i += n;
  }
  return cudaSuccess;
}

}  // namespace q4
