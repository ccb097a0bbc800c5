// q4_stream.cu -- tensor-core weight streaming for three or four activation
// rows (batched decode): the affine Q4 group-32 matmul
//
//   y[m,n] = sum_k x[m,k] * w_hat[n,k],   w_hat = bf16(s*q + b)  (group 32 along k)
//
// with the products and the fp32 accumulation done by the 5th-generation
// tensor cores (tcgen05.mma, kind::f16) and the CUDA cores doing nothing but
// the dequantization (about two instructions per weight, whatever the number
// of activation rows).  At three or four rows the CUDA-core GEMV, which works
// on pairs of rows, reads the weights twice and multiplies every weight by
// every row on the CUDA cores; this kernel reads them once and the rows cost
// tensor-core time only.  (At one or two rows the GEMV is faster: measured
// 4.7 TB/s at one row against this kernel's 2.7.)
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
// Per CTA (one per SM, 768 threads):
//   warp 0       producer: three bulk copies per tile;
//   warps 1..3   MMA issue (warp 1 also allocates tensor memory): issuer i
//                takes chunks c == i (mod I) of every tile (I = 3, 2 or 1 by
//                the problem's accumulator width) into its own double-buffered
//                fp32 tile.  One thread issues an MMA of these shapes only
//                every ~50 cycles (its instruction stream, not the tensor
//                core, is the limit), so several issuers keep pace with the
//                weight stream.  The split depends on the problem alone, so a
//                result never depends on the batch;
//   warps 4..19  dequantize: four groups of four warps (one warp per
//                tensor-memory lane quarter) take 64-wide K chunks in turn;
//                a thread turns 64 codes of its (row, segment) into 32 bf16x2
//                words -- "128 + q" by one LOP3 per two codes, q by an exact
//                packed subtract, bf16(s*q + b) by one packed FMA (one
//                rounding, as the dequantizer computes it) -- and stores them
//                to tensor memory (tcgen05.st);
//   warps 20..23 epilogue: per tile, read the diagonals of the issuers' fp32
//                tiles from tensor memory, sum them and the segments
//                (shuffles), write bf16 y; and, at each new problem, lay out
//                its B operand.
// The code pairs come out as (q[t], q[t+4]) of each 8-code word; the B
// operand is built with the same order of k, so the products pair up.
// Every wait is bounded (q4_device.cuh); programmatic dependent launch as in
// the GEMV family.
#include "q4_device.cuh"
#include "q4_internal.h"

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
constexpr int kChunkK = 64;                                  // K per lane per A chunk (32 columns)
constexpr int kGroups = 4;                                   // dequantizing warp groups
constexpr int kMaxIssuers = 3;                               // MMA-issuing warps
constexpr int kFirstDqWarp = 1 + kMaxIssuers;                // 4
constexpr int kFirstEpiWarp = kFirstDqWarp + 4 * kGroups;   // 20
constexpr int kThreads = 32 * (kFirstEpiWarp + 4);           // 768: 6 warps per SM sub-partition, <= 80 registers
constexpr int kMaxRows = 4;                                  // activation rows per launch
constexpr int kMinRows = 3;  // below this the CUDA-core GEMV is faster (it reads the weights once for 1-2 rows)
constexpr uint32_t kTmemCols = 512;
constexpr int kMaxASlots = 16;  // A ring in tensor memory: up to 16 chunks of 32 columns
constexpr int kMaxStages = 12;
constexpr int kMaxProblems = 256;
constexpr int kFewProblems = 4;

struct StreamProblem {
  const uint16_t* x;  // [M, K]
  const uint8_t* codes;
  const uint16_t* scales;
  const uint16_t* biases;
  uint16_t* y;         // [M, N]
  const uint16_t* r;   // epilogue operand [M, N] (kEpiResidual / kEpiSiluMul), else NULL
  int64_t N;
  int64_t byte_begin;  // work offset of the first tile (packed bytes of all tiles before)
  int32_t K;
  int32_t segs;        // K segments per weight row; R = 128 / segs rows per tile
  int32_t tile_bytes;  // packed bytes of a full tile (the unit of work balancing)
  int32_t epi;         // output epilogue (q4_device.cuh)
};

template <int NP>
struct StreamLaunch {
  int32_t count, M, stages, a_slots;  // a_slots: A ring chunks (a multiple of 4)
  uint32_t stage_bytes, b_bytes, a_col0, pad_;  // a_col0: first A ring column (after the accumulators)
  int64_t total_bytes;
  StreamProblem prob[NP];
};

// ---- tcgen05 wrappers -------------------------------------------------------

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// K-major operand with the 128-byte swizzle: rows of 128 bytes, 8-row groups
// 1024 bytes apart, base 1024-byte aligned.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t smem_addr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((smem_addr & 0x3FFFFu) >> 4);  // start address
  d |= static_cast<uint64_t>(16u >> 4) << 16;                // leading byte offset (unused)
  d |= static_cast<uint64_t>(1024u >> 4) << 32;              // stride byte offset
  d |= static_cast<uint64_t>(1) << 46;                       // descriptor version
  d |= static_cast<uint64_t>(2) << 61;                       // 128-byte swizzle
  return d;
}

// D (tensor memory) [+]= A (tensor memory) x B (shared memory descriptor).
__device__ __forceinline__ void tc_mma_ts(uint32_t tmem_d, uint32_t tmem_a, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{ .reg .pred p; setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p; }"
      ::"r"(tmem_d), "r"(tmem_a), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}


__device__ __forceinline__ void tmem_st_x16(uint32_t taddr, const uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
      "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
      : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// W (8, 16 or 32) consecutive fp32 columns of this thread's lane into r;
// complete with tmem_wait_ld().
template <int W>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, uint32_t (&r)[W]) {
  if constexpr (W == 8) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr));
  } else if constexpr (W == 16) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
  } else {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
  }
}

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
        uint32_t r[W];
        tmem_ld_cols<W>(base + static_cast<uint32_t>(i) * issuer_stride + static_cast<uint32_t>(m * W), r);
        tmem_wait_ld();
        part[m] += pick<W>(r, sel);
      }
  }
}

// tcgen05 instruction descriptor: D fp32, A and B bf16, both K-major, M = 128.
__device__ __forceinline__ uint32_t make_idesc(int n) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(n >> 3) << 17) |
         (static_cast<uint32_t>(kLanes >> 4) << 24);
}


// Eight codes (one word: q0..q7 of eight consecutive k) -> four bf16x2 words
// of w_hat for the k pairs (t, t + 4), t = 0..3: "128 + q" by one LOP3 per
// pair (0x43004300 is bf16 (128, 128), whose last significand bit weighs 1),
// q by an exact packed subtract, bf16(s*q + b) by one packed FMA (one
// rounding).  One PTX block with the two constants passed in registers (held
// by the caller across the loop), so none of them is rebuilt per use.
__device__ __forceinline__ void dequant_word(uint32_t w, uint32_t s2, uint32_t b2, uint32_t mask, uint32_t magic,
                                             uint32_t* o) {
  asm("{\n\t.reg .b32 t1, t2, t3, v0, v1, v2, v3;\n\t"
      "shr.b32 t1, %4, 4;\n\tshr.b32 t2, %4, 8;\n\tshr.b32 t3, %4, 12;\n\t"
      "lop3.b32 v0, %4, %7, %8, 0xEA;\n\tlop3.b32 v1, t1, %7, %8, 0xEA;\n\t"
      "lop3.b32 v2, t2, %7, %8, 0xEA;\n\tlop3.b32 v3, t3, %7, %8, 0xEA;\n\t"
      "sub.rn.bf16x2 v0, v0, %8;\n\tsub.rn.bf16x2 v1, v1, %8;\n\t"
      "sub.rn.bf16x2 v2, v2, %8;\n\tsub.rn.bf16x2 v3, v3, %8;\n\t"
      "fma.rn.bf16x2 %0, v0, %5, %6;\n\tfma.rn.bf16x2 %1, v1, %5, %6;\n\t"
      "fma.rn.bf16x2 %2, v2, %5, %6;\n\tfma.rn.bf16x2 %3, v3, %5, %6;\n\t}"
      : "=r"(o[0]), "=r"(o[1]), "=r"(o[2]), "=r"(o[3])
      : "r"(w), "r"(s2), "r"(b2), "r"(mask), "r"(magic));
}

// x[k..k+8) (one 16-byte run) in the (t, t + 4) pair order of dequant_word.
__device__ __forceinline__ uint4 pair_order(uint4 e) {
  return make_uint4(__byte_perm(e.x, e.z, 0x5410), __byte_perm(e.x, e.z, 0x7632), __byte_perm(e.y, e.w, 0x5410),
                    __byte_perm(e.y, e.w, 0x7632));
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
    issuers = nb <= 16 ? 3 : nb <= 32 ? 2 : 1;
    dstride = static_cast<uint32_t>(nb);
  }
};

// The tiles of problem p that this CTA owns: those whose first byte (in the
// work order of all problems' tiles) falls in [lo, hi).
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

// EPI: some problem of the launch has an output epilogue; the plain
// instantiation keeps the epilogue's code out of the kernel.
template <int NP, bool EPI>
__global__ void __launch_bounds__(kThreads, 1) stream_kernel(const __grid_constant__ StreamLaunch<NP> L) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* bmat = smem;               // B operand of the current problem, b_bytes (a multiple of 1024)
  uint8_t* ring = smem + L.b_bytes;   // stages x stage_bytes
  uint64_t* full = reinterpret_cast<uint64_t*>(ring + static_cast<size_t>(L.stages) * L.stage_bytes);
  uint64_t* empty = full + kMaxStages;
  uint64_t* afull = empty + kMaxStages;
  uint64_t* aempty = afull + kMaxASlots;
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
      mbar_init(&afull[a], 4);
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
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
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

  pdl_launch_dependents();
  if (warp == 0 && lane == 0) {
    // Before the wait: pull the first tile's codes toward L2 (a hint only).
    for (int p = 0; p < L.count; ++p) {
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
    for (int p = 0; p < L.count; ++p) {
      const StreamProblem& P = L.prob[p];
      int64_t j0, j1;
      tile_range(P, lo, hi, j0, j1);
      const int R = kLanes / P.segs;
      const uint32_t row_bytes = static_cast<uint32_t>(P.K / 2), sb_row = static_cast<uint32_t>(P.K / 16);
      for (int64_t j = j0; j < j1; ++j) {
        if (lane == 0) {
          if (!dead && !mbar_wait<kSleepWaits>(&empty[s], ph ^ 1u)) dead = true;
          const int64_t row0 = j * R;
          const uint32_t rows = static_cast<uint32_t>((P.N - row0 < R) ? P.N - row0 : R);
          uint8_t* st = ring + static_cast<size_t>(s) * L.stage_bytes;
          mbar_arrive_expect_tx(&full[s], rows * (row_bytes + 2 * sb_row));
          // the tile's codes, scales and biases: three contiguous runs
          bulk_g2s(st, P.codes + row0 * row_bytes, rows * row_bytes, &full[s]);
          bulk_g2s(st + R * row_bytes, P.scales + row0 * (P.K / 32), rows * sb_row, &full[s]);
          bulk_g2s(st + R * (row_bytes + sb_row), P.biases + row0 * (P.K / 32), rows * sb_row, &full[s]);
        }
        if (++s == L.stages) { s = 0; ph ^= 1u; }
      }
    }
  } else if (warp <= kMaxIssuers) {
    // ---------------- MMA issuers ----------------
    const int me = warp - 1;
    if (lane == 0) {
      bool dead = false;
      int lp = 0;
      int slot0 = 0;      // A ring slot of the current tile's first chunk
      uint32_t ph0 = 0;   // and its phase
      int64_t gt = 0;
      const uint64_t bdesc0 = sw128_desc(smem_u32(bmat));
      const uint32_t a_base = tmem + a_col0;
      for (int p = 0; p < L.count; ++p) {
        const StreamProblem& P = L.prob[p];
        int64_t j0, j1;
        tile_range(P, lo, hi, j0, j1);
        if (j0 >= j1) continue;
        const ProblemShape S(P, L.M);
        const bool active = me < S.issuers;
        const uint32_t idesc = make_idesc(S.nb);
        const uint32_t atom16 = static_cast<uint32_t>(S.nb) * 128u >> 4;  // B atom size in 16-byte units
        // B of the previous problem is free once its MMAs are done.  Waiting
        // for this problem's B also means the epilogue has drained every
        // earlier tile, so the accumulator layout may change here.
        if (lp > 0) tc_commit(bempty);
        if (!dead && !mbar_wait<kSleepWaits>(bfull, static_cast<uint32_t>(lp & 1))) dead = true;
        tc_fence_after();
        for (int64_t j = j0; j < j1; ++j, ++gt) {
          const int db = static_cast<int>(gt & 1);
          const uint32_t dt = tmem + static_cast<uint32_t>(2 * me + db) * S.dstride;
          // every issuer waits, so none can arrive twice on one phase of dfull
          if (!dead && !mbar_wait<kSleepWaits>(&dempty[db], static_cast<uint32_t>((gt >> 1) & 1) ^ 1u)) dead = true;
          tc_fence_after();
          if (active) {
            for (int c = me; c < S.chunks; c += S.issuers) {
              int slot = slot0 + c;  // ring slot and phase of chunk c
              uint32_t sph = ph0;
              while (slot >= A) { slot -= A; sph ^= 1u; }
              if (!dead && !mbar_wait<kSleepWaits>(&afull[slot], sph)) dead = true;
              tc_fence_after();
              const uint32_t at = a_base + static_cast<uint32_t>(slot) * 32u;
              const uint64_t bd = bdesc0 + static_cast<uint64_t>(c) * atom16;
              // the first MMA of this issuer in the tile overwrites its accumulator
              tc_mma_ts(dt, at, bd, idesc, c >= S.issuers ? 1u : 0u);
              tc_mma_ts(dt, at + 8u, bd + 2u, idesc, 1u);
              if (c < S.full_chunks) {
                tc_mma_ts(dt, at + 16u, bd + 4u, idesc, 1u);
                tc_mma_ts(dt, at + 24u, bd + 6u, idesc, 1u);
              }
              tc_commit(&aempty[slot]);
            }
          }
          // every issuer, every tile (count kMaxIssuers); an idle issuer's
          // commit arrives once its earlier MMAs are complete
          tc_commit(&dfull[db]);
          slot0 += S.chunks;
          while (slot0 >= A) { slot0 -= A; ph0 ^= 1u; }
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
    uint32_t kmask = 0x000F000Fu, kmagic = 0x43004300u;
    asm volatile("" : "+r"(kmask), "+r"(kmagic));  // opaque: kept in registers, not rebuilt per use
    bool dead = false;
    int s = 0;
    uint32_t ph = 0, gc = 0;  // gc: chunks of this CTA before the current tile
    int slot0 = 0;            // A ring slot of the current tile's first chunk
    uint32_t ph0 = 0;         // and its phase
    for (int p = 0; p < L.count; ++p) {
      const StreamProblem& P = L.prob[p];
      int64_t j0, j1;
      tile_range(P, lo, hi, j0, j1);
      if (j0 >= j1) continue;
      const ProblemShape S(P, L.M);
      const int r = tl / S.segs, seg = tl % S.segs;  // this lane: row r, segment seg
      const int rot = seg % S.pieces;                  // its code runs, rotated by seg
      const int groups = P.K / 32;
      for (int64_t j = j0; j < j1; ++j, gc += static_cast<uint32_t>(S.chunks)) {
        if (!dead && !mbar_wait<kSleepWaits>(&full[s], ph)) dead = true;
        const uint8_t* st = ring + static_cast<size_t>(s) * L.stage_bytes;
        const uint8_t* crow = st + r * (P.K / 2) + seg * (S.kseg / 2);  // the segment's 16-byte code runs
        const uint16_t* srow = reinterpret_cast<const uint16_t*>(st + S.R * (P.K / 2)) + r * groups + seg * S.pieces;
        const uint16_t* brow = srow + S.R * groups;
        // the chunks of this group: global index == grp (mod kGroups)
        for (int c = static_cast<int>((static_cast<uint32_t>(grp) - gc) & (kGroups - 1)); c < S.chunks; c += kGroups) {
          int slot = slot0 + c;  // ring slot and phase of chunk c
          uint32_t sph = ph0;
          while (slot >= A) { slot -= A; sph ^= 1u; }
          if (!dead && !mbar_wait<kSleepWaits>(&aempty[slot], sph ^ 1u)) dead = true;
          const uint32_t taddr = a_addr + static_cast<uint32_t>(slot) * 32u;
          uint32_t o[16];
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            if (h == 0 || c < S.full_chunks) {
              // position 2c + h of the segment holds its code run (2c + h + seg) mod pieces
              int run = 2 * c + h + rot;
              if (run >= S.pieces) run -= S.pieces;
              const uint4 cw = *reinterpret_cast<const uint4*>(crow + 16 * run);
              const uint32_t s2 = __byte_perm(static_cast<uint32_t>(srow[run]), 0, 0x1010);
              const uint32_t b2 = __byte_perm(static_cast<uint32_t>(brow[run]), 0, 0x1010);
              dequant_word(cw.x, s2, b2, kmask, kmagic, o + 0);
              dequant_word(cw.y, s2, b2, kmask, kmagic, o + 4);
              dequant_word(cw.z, s2, b2, kmask, kmagic, o + 8);
              dequant_word(cw.w, s2, b2, kmask, kmagic, o + 12);
              tmem_st_x16(taddr + 16u * h, o);
            }
          }
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&afull[slot]);
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
    for (int p = 0; p < L.count; ++p) {
      const StreamProblem& P = L.prob[p];
      int64_t j0, j1;
      tile_range(P, lo, hi, j0, j1);
      if (j0 >= j1) continue;
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
                  pair_order(v[u]);
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
      for (int64_t j = j0; j < j1; ++j, ++gt) {
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
        const int64_t row = j * S.R + rq;
        if (seg == 0 && row < P.N) {
#pragma unroll
          for (int m = 0; m < kMaxRows; ++m)
            if (m < L.M) {
              const int64_t idx = static_cast<int64_t>(m) * P.N + row;
              if constexpr (EPI) P.y[idx] = epilogue_bf16(part[m], P.epi, P.r, idx);
              else P.y[idx] = float_to_bf16_bits(part[m]);
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
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
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

constexpr size_t kFixedSmem = 1024 /* alignment */ + 8 * (2 * kMaxStages + 2 * kMaxASlots + 6) + 16;

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
    P.y = a.y;
    P.r = a.r;
    P.epi = a.epi;
    P.N = a.N;
    P.K = static_cast<int32_t>(a.K);
    P.segs = pl.segs;
    const int R = kLanes / pl.segs;
    P.tile_bytes = static_cast<int32_t>(R * (a.K / 2 + a.K / 8));
    P.byte_begin = total;
    const int64_t t = (a.N + R - 1) / R;
    total += t * P.tile_bytes;
    tiles += t;
    stage_bytes = std::max(stage_bytes, pl.stage_bytes);
    const uint32_t issuers = pl.nb <= 16 ? 3u : pl.nb <= 32 ? 2u : 1u;  // as ProblemShape
    acc_cols = std::max(acc_cols, 2u * issuers * pl.nb);
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
  // A ring as the rest holds (a multiple of 4 chunks: one slot per dequantizing
  // group per turn).
  L.a_col0 = (acc_cols + 31u) & ~31u;
  L.a_slots = static_cast<int32_t>(std::min<uint32_t>(kMaxASlots, (kTmemCols - L.a_col0) / 32u) & ~3u);
  if (L.a_slots < 4) return cudaErrorInvalidConfiguration;
  L.stage_bytes = stage_bytes;
  L.b_bytes = b_bytes;
  L.total_bytes = total;
  const size_t smem = kFixedSmem + b_bytes + static_cast<size_t>(stages) * stage_bytes;
  const int grid = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(dev.sm_count, tiles)));
  bool epi = false;
  for (int i = 0; i < count; ++i) epi = epi || list[i].epi != kEpiNone;
  auto kern = epi ? stream_kernel<NP, true> : stream_kernel<NP, false>;
  static PerDeviceOnce attr_once[2];
  if (attr_once[epi].needed(dev.device)) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(dev.smem_optin));
    if (e != cudaSuccess) return e;
    attr_once[epi].mark(dev.device);
  }
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
  return cudaLaunchKernelEx(&cfg, kern, L);
}

}  // namespace

cudaError_t stream_device_flags(unsigned int* flags, bool clear) { return tu_device_flags(flags, clear); }

bool stream_supported(const MatmulArgs& a, const DeviceInfo& dev) {
#if defined(Q4_STREAM_TC) && Q4_STREAM_TC == 0
  return false;
#endif
  if (a.M < kMinRows || a.M > kMaxRows) return false;
  if (a.fused()) return false;  // one-pass SwiGLU is a GEMV-family problem
  if ((reinterpret_cast<uintptr_t>(a.scales) | reinterpret_cast<uintptr_t>(a.biases)) & 15u) return false;
  if (a.K > (int64_t(1) << 20)) return false;
  const Plan pl = plan_of(a);
  if (pl.segs == 0) return false;
  return kFixedSmem + pl.b_bytes + 2 * static_cast<size_t>(pl.stage_bytes) <= dev.smem_optin;
}

cudaError_t launch_stream_batch(const MatmulArgs* list, int count, cudaStream_t stream, const DeviceInfo& dev) {
  for (int i = 0; i < count; i += kMaxProblems) {
    const int n = std::min(kMaxProblems, count - i);
    cudaError_t e = (n <= kFewProblems) ? run_stream<kFewProblems>(list + i, n, dev, stream)
                                        : run_stream<kMaxProblems>(list + i, n, dev, stream);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace q4
