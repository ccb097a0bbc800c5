// q4_gmma.cu -- the affine Q4 group-32 matmul for 1 to 16 activation rows
// (decode steps, a few concurrent streams) as per-group tensor-core sums:
//
//   y[m,n] = sum_g ( s[n,g] * D[n,g,m] + (b[n,g] - 128 s[n,g]) * X[m,g] ),
//   D[n,g,m] = sum_{k in g} (128 + q[n,k]) * x[m,k],   X[m,g] = sum_{k in g} x[m,k]
//
// which is x . w_hat^T with w_hat = s*q + b (model card "personaplex-edge-q4":
// affine Q4, group size 32; the packed weights are consumed as they are,
// never expanded in memory).  The 5th-generation tensor cores (tcgen05.mma,
// kind::f16) form the group sums D from the codes themselves: 128 + q is an
// exact bf16 (a byte permute and a LOP3 per two codes; no scale, no
// rounding), its products with the bf16 x are exact, and each group of 32
// inputs has its own fp32 accumulator in tensor memory (two K16 MMAs).  The
// CUDA cores apply the group's scale and bias in fp32, two FMAs per group and
// activation row -- the CUDA-core GEMV's arithmetic, with its dot products
// moved to the tensor cores and no dequantized weight formed at all.
//
// Tiles: 128 weight rows (the MMA's M and the tensor-memory lanes) x the
// whole K of one problem, in pipeline steps of 128 inputs (four groups); the
// MMA's N is 16 activation rows (rows beyond M are zero-filled by the TMA).
// The launch is persistent over a list of problems: each CTA takes the tiles
// whose first packed byte falls in its equal share of the list's bytes.
//
// Per CTA (608 threads, one CTA per SM):
//   warp 0        TMA producer: per step the x tile (16 rows x 128 inputs as
//                 two 128-byte-swizzled halves) and the code tile (128 rows x
//                 64 bytes, 64-byte swizzle, so that the dequantizing warps'
//                 16-byte reads do not conflict);
//   warps 1, 2    MMA issuers (whole warps; the elected lane issues), taking
//                 steps in turn: per step two MMAs per group into that group's
//                 16 accumulator columns, two waits and three commits;
//   warps 3..14   three groups of four warps, taking steps in turn: a thread
//                 turns its weight row's 128 codes into 64 bf16 pairs
//                 (128 + q, 128 + q') and stores them to its tensor-memory
//                 lane (tcgen05.st);
//   warps 15..18  epilogue, a thread per weight row: per problem, the group
//                 sums X of x into shared memory; per step, the four groups'
//                 D from tensor memory (tcgen05.ld) and acc += s*D + (b -
//                 128 s)*X in fp32, with the row's scales and biases fetched
//                 by cp.async three 8-group runs ahead; per tile, y (with the
//                 residual or SwiGLU epilogue).
// Tensor memory: 5 slots of A (64 columns each: 128 inputs as bf16 pairs),
// freed as soon as their MMAs complete, and 3 slots of D (64 columns each:
// four groups x 16 activation rows), freed once the epilogue has read them.
// Every wait is bounded (q4_device.cuh); an epilogue thread whose wait gave
// up writes NaN.  Programmatic dependent launch as in the other kernels.
#include "q4_device.cuh"
#include "q4_internal.h"
#include "q4_tcgen05.cuh"

#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstring>
#include <mutex>
#include <new>
#include <vector>

namespace q4 {
namespace {

constexpr int kRows = 128;                 // weight rows per tile (MMA M, tensor-memory lanes)
constexpr int kStepK = 128;                // inputs per pipeline step: four groups
constexpr int kGroupsPerStep = kStepK / 32;
constexpr int kSubK = 64;                  // inputs per 128-byte-swizzled x sub-tile
constexpr int kN = 16;                     // MMA N: activation rows, zero-padded
constexpr int kSuperK = 256;               // scale/bias run: 8 groups = 16 bytes of a row
constexpr int kStepsPerSuper = kSuperK / kStepK;
constexpr int kIssuers = 2;                // MMA-issuing warps, taking steps in turn
constexpr int kDqGroups = 3;               // dequantizing groups of four warps
constexpr int kFirstDq = 1 + kIssuers;
constexpr int kFirstEpi = kFirstDq + 4 * kDqGroups;  // 15
constexpr int kThreads = 32 * (kFirstEpi + 4);      // 608
constexpr int kASlots = 5;                 // steps' A operands in tensor memory
constexpr int kDSlots = 3;                 // steps' group sums in tensor memory
constexpr uint32_t kACols = 64;            // A columns per slot: 128 inputs as bf16 pairs
constexpr uint32_t kDCols = 64;            // D columns per slot: 4 groups x 16 activation rows
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kDCol0 = kASlots * kACols;        // 320: D after the A slots
constexpr int kXSubBytes = kN * kSubK * 2;           // 2 KB: 16 rows of 128 bytes
constexpr int kXTileBytes = 2 * kXSubBytes;          // 4 KB
constexpr int kCodeTileBytes = kRows * kStepK / 2;   // 8 KB: 128 rows of 64 bytes
constexpr int kStageBytes = kXTileBytes + kCodeTileBytes;  // 12 KB, a multiple of 1024
constexpr int kMaxStages = 16;
constexpr int kSbSlots = 4;                // scale/bias runs in flight per epilogue thread
constexpr int kSbPrefetch = kSbSlots - 1;
constexpr int kSbBytes = kSbSlots * 2 * kRows * 16;  // 16 KB
constexpr int kMaxXMaps = 8;
constexpr int kMaxEntries = 160;
constexpr int kMaxCtas = 256;  // CTAs per launch at most (one per SM)
static_assert(kMaxEntries <= 255, "entry indices fit a byte");
constexpr float kNaN = __builtin_nanf("");
// Sleep between polls of a barrier (ns), per role: the producer runs far
// ahead and waits long; the issuers are on the critical path.
#ifndef Q4_GMMA_SLEEP_PRODUCER
#define Q4_GMMA_SLEEP_PRODUCER 256
#endif
#ifndef Q4_GMMA_SLEEP_ISSUER
#define Q4_GMMA_SLEEP_ISSUER 32
#endif
#ifndef Q4_GMMA_SLEEP_DQ
#define Q4_GMMA_SLEEP_DQ 64
#endif
#ifndef Q4_GMMA_SLEEP_EPI
#define Q4_GMMA_SLEEP_EPI 64
#endif
constexpr unsigned kSleepProducer = Q4_GMMA_SLEEP_PRODUCER, kSleepIssuer = Q4_GMMA_SLEEP_ISSUER,
                   kSleepDq = Q4_GMMA_SLEEP_DQ, kSleepEpi = Q4_GMMA_SLEEP_EPI;
static_assert(kDCol0 + kDSlots * kDCols == kTmemCols, "tensor-memory layout");
constexpr int kMinStages = 4;  // >= kDqGroups, kIssuers: the cursors wrap a ring at most once per move
static_assert(kDqGroups <= kMinStages && kIssuers <= kMinStages && kDqGroups <= kASlots && kIssuers <= kDSlots,
              "cursor steps");

// One weight of a launch.  A SwiGLU problem takes two consecutive entries:
// the gate weight (fused = 1, with the problem's y) and then the up weight
// (fused = 2: only its codes map, scales and biases are used).
struct GmmaEntry {
  CUtensorMap codes_map;     // [N, K/2] bytes, box 64 x 128, 64-byte swizzle
  const uint16_t* scales;    // [N, K/32]
  const uint16_t* biases;
  uint16_t* y;               // [M, N]
  const uint16_t* r;         // residual [M, N] (kEpiResidual), else NULL
  int64_t step_begin;        // steps of all earlier tiles of the launch
  int32_t N, K;
  int32_t x_idx;             // x_map[x_idx] / x_ptr[x_idx]: this problem's activations
  int16_t epi, fused;
};
static_assert(sizeof(GmmaEntry) == 192, "entry layout");

struct GmmaLaunch {
  CUtensorMap x_map[kMaxXMaps];      // [M, K] bf16, box 64 x 16, 128-byte swizzle
  const uint16_t* x_ptr[kMaxXMaps];
  GmmaEntry e[kMaxEntries];
  // Tiles shared by several CTAs: each piece's fp32 partial sums, [2 * grid]
  // slots of kRows x (2 MC) floats (slot 2c: CTA c's first tile, 2c + 1 its
  // last), and [grid] arrival counters, zero at launch (NULL if no tile is
  // shared).
  float* partials;
  unsigned int* counters;
  int64_t total_steps;
  int32_t count, M, stages, x_floats;  // x_floats: group-sum area (largest K / 32) x MC, rounded up to 4
  // first[c]: the first entry (a SwiGLU pair's gate entry) whose tiles end
  // after CTA c's first step.  Every role of the CTA walks the entries from
  // there and stops at the first that starts at or after its last step, so
  // it reads only the descriptors of its own tiles (each read of another
  // entry's is a constant-cache miss).
  uint8_t first[kMaxCtas];
};
static_assert(sizeof(GmmaLaunch) <= 32764, "kernel parameter space");
static_assert(sizeof(GmmaLaunch) <= kGmmaParamBytes, "plan storage");
static_assert(kGmmaMaxRows <= kN, "activation rows per MMA");

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int c0, int c1, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
      ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(smem_u32(bar))
      : "memory");
}

// 16 bytes global -> shared; zero-filled when src_bytes == 0.
__device__ __forceinline__ void cp_async_16(void* dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Steps of one tile of entry E: K / 128 per weight (two weights for SwiGLU).
__device__ __forceinline__ int tile_steps(const GmmaEntry& E) { return (E.K / kStepK) * (E.fused ? 2 : 1); }

// First step of CTA c: the launch's steps in equal shares.
__device__ __forceinline__ int64_t cta_first_step(const GmmaLaunch& L, int64_t c) {
  return L.total_steps * c / gridDim.x;
}

// The tiles [j0, j1) of entry E that have steps in [lo, hi).
__device__ __forceinline__ void tile_range(const GmmaEntry& E, int64_t lo, int64_t hi, int64_t& j0, int64_t& j1) {
  const int64_t tiles = (static_cast<int64_t>(E.N) + kRows - 1) / kRows;
  const int64_t S = tile_steps(E);
  const int64_t a = lo - E.step_begin, b = hi - E.step_begin;
  j0 = a <= 0 ? 0 : a / S;
  j1 = b <= 0 ? 0 : (b + S - 1) / S;
  if (j0 > tiles) j0 = tiles;
  if (j1 > tiles) j1 = tiles;
}

// (a & b) | c in one LOP3.
__device__ __forceinline__ uint32_t and_or(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// Four code words (32 codes, k order) -> 16 bf16 pairs (128 + q[2i], 128 + q[2i+1]),
// the even k in the low half: per 8 codes a shift, four byte permutes and
// four LOP3s.  mask = 0x000F000F and bias = 0x43004300 (0x4300 is bf16 128,
// whose last 4 bits take q) come in registers, so that each LOP3 takes both.
__device__ __forceinline__ void codes_to_bf16(const uint4& c, uint32_t mask, uint32_t bias, uint32_t (&o)[16]) {
  const uint32_t words[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    const uint32_t wd = words[w], w4 = wd >> 4;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      // byte i of wd holds q[2i] in its low nibble, byte i of w4 holds q[2i+1]
      const uint32_t pr = __byte_perm(wd, w4, i | (i << 4) | ((4 + i) << 8) | ((4 + i) << 12));
      o[4 * w + i] = and_or(pr, mask, bias);
    }
  }
}

template <int W>
__device__ __forceinline__ void tmem_ld_d(uint32_t taddr, uint32_t (&r)[W]) {
  if constexpr (W == 1) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];" : "=r"(r[0]) : "r"(taddr));
  } else if constexpr (W == 2) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x2.b32 {%0, %1}, [%2];" : "=r"(r[0]), "=r"(r[1]) : "r"(taddr));
  } else if constexpr (W == 4) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(taddr));
  } else {
    tmem_ld_cols<W>(taddr, r);
  }
}

// MC: activation rows rounded up to 1, 2, 4, 8 or 16 (the epilogue's
// register arrays); EPI: some problem of the launch has an output epilogue.
template <int MC, bool EPI>
__global__ void __launch_bounds__(kThreads, 1) gmma_kernel(const __grid_constant__ GmmaLaunch L) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  uint8_t* ring = smem;  // stages x kStageBytes: the two x sub-tiles, then the code tile
  uint4* sb = reinterpret_cast<uint4*>(ring + static_cast<size_t>(L.stages) * kStageBytes);  // [slot][s, b][row]
  float* xsum = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(sb) + kSbBytes);         // [G][MC]
  uint64_t* tma_full = reinterpret_cast<uint64_t*>(xsum + L.x_floats);
  uint64_t* stage_free = tma_full + kMaxStages;
  uint64_t* a_full = stage_free + kMaxStages;  // A written (four dequantizing warps)
  uint64_t* a_free = a_full + kASlots;         // the MMAs reading the A slot are complete
  uint64_t* d_full = a_free + kASlots;         // the MMAs writing the D slot are complete
  uint64_t* d_free = d_full + kDSlots;         // D read (four epilogue warps)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(d_free + kDSlots);
  uint32_t* last_flag = tmem_slot + 1;         // epilogue: this CTA completes a shared tile

  if (tid == 0) {
    for (int s = 0; s < L.stages; ++s) {
      mbar_init(&tma_full[s], 1);
      mbar_init(&stage_free[s], 1);
    }
    for (int s = 0; s < kASlots; ++s) {
      mbar_init(&a_full[s], 4);
      mbar_init(&a_free[s], 1);
    }
    for (int s = 0; s < kDSlots; ++s) {
      mbar_init(&d_full[s], 1);
      mbar_init(&d_free[s], 4);
    }
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // All 512 columns: the allocation starts at lane 0, column 0, so the
  // tensor-memory addresses below are plain constants.
  const bool tmem_ok = *tmem_slot == 0u;
  if (!tmem_ok && tid == 0) atomicOr(&g_device_flags, kFlagWaitTimeout);

  const int64_t lo = cta_first_step(L, blockIdx.x), hi = cta_first_step(L, blockIdx.x + 1);
  pdl_launch_dependents();
  pdl_wait_predecessors();

  if (!tmem_ok) {
    // not reached; the flag tells the caller that nothing was computed
  } else if (warp == 0) {
    // ---------------- TMA producer (whole warp; the elected lane issues) ----------------
    const bool leader = elect_one();
    bool dead = false;
    int s = 0;
    uint32_t ph = 0;
    for (int p = L.first[blockIdx.x]; p < L.count && L.e[p].step_begin < hi; p += L.e[p].fused ? 2 : 1) {
      const GmmaEntry& E = L.e[p];
      int64_t j0, j1;
      tile_range(E, lo, hi, j0, j1);
      const int S = tile_steps(E), Sp = E.K / kStepK;
      const CUtensorMap* xmap = &L.x_map[E.x_idx];
      for (int64_t j = j0; j < j1; ++j) {
        const int64_t tb = E.step_begin + j * S;
        const int u0 = static_cast<int>(max(lo - tb, int64_t(0))), u1 = static_cast<int>(min(hi - tb, int64_t(S)));
        for (int u = u0; u < u1; ++u) {
          const int pass = u >= Sp ? 1 : 0, t = u - pass * Sp;  // the up weight after the gate's steps
          if (!dead && !mbar_wait_backoff<kSleepProducer>(&stage_free[s], ph ^ 1u)) dead = true;
          if (leader) {
            uint8_t* st = ring + static_cast<size_t>(s) * kStageBytes;
            mbar_arrive_expect_tx(&tma_full[s], kStageBytes);
            tma_load_2d(st, xmap, t * kStepK, 0, &tma_full[s]);
            tma_load_2d(st + kXSubBytes, xmap, t * kStepK + kSubK, 0, &tma_full[s]);
            tma_load_2d(st + kXTileBytes, &L.e[p + pass].codes_map, t * (kStepK / 2), static_cast<int>(j * kRows),
                        &tma_full[s]);
          }
          __syncwarp();
          if (++s == L.stages) { s = 0; ph ^= 1u; }
        }
      }
    }
  } else if (warp <= kIssuers) {
    // ---------------- MMA issuers (whole warps; the elected lane issues) ----------------
    // Issuer w takes the CTA's steps w - 1, w - 1 + kIssuers, ...; a commit
    // tracks the MMAs of its own thread, so the two need no coordination.
    // Waits for the dequantizing warps (they arrive after having waited for
    // the stage's TMA, so the x tile is in place too) and for the epilogue to
    // have read the D slot's previous sums.
    const bool leader = elect_one();
    const int me = warp - 1;
    const uint32_t idesc = idesc_bf16_m128(kN);
    const uint64_t bd0 = sw128_desc(smem_u32(ring));
    bool dead = false;
    int s = me % L.stages, aslot = me % kASlots, dslot = me % kDSlots;
    uint32_t aph = (me / kASlots) & 1u, dph = (me / kDSlots) & 1u;
    int t = me;  // step within the current segment; carried over segment ends
    for (int p = L.first[blockIdx.x]; p < L.count && L.e[p].step_begin < hi; p += L.e[p].fused ? 2 : 1) {
      const GmmaEntry& E = L.e[p];
      int64_t j0, j1;
      tile_range(E, lo, hi, j0, j1);
      const int S = tile_steps(E);
      for (int64_t j = j0; j < j1; ++j) {
        const int64_t tb = E.step_begin + j * S;
        const int len = static_cast<int>(min(hi - tb, int64_t(S)) - max(lo - tb, int64_t(0)));
        for (; t < len; t += kIssuers) {
          if (!dead && !mbar_wait_backoff<kSleepIssuer>(&a_full[aslot], aph)) dead = true;       // A written
          if (!dead && !mbar_wait_backoff<kSleepIssuer>(&d_free[dslot], dph ^ 1u)) dead = true;  // D read
          tc_fence_after();
          const uint64_t bd = bd0 + static_cast<uint64_t>(s * (kStageBytes >> 4));
          const uint32_t at = static_cast<uint32_t>(aslot) * kACols;
          const uint32_t dt = kDCol0 + static_cast<uint32_t>(dslot) * kDCols;
          if (leader) {
            // group g: inputs 32g .. 32g+31 = A columns 16g .. 16g+15, x sub-tile g / 2
            // (descriptor + 128 per 2 KB), K16 steps 2 (g % 2) and 2 (g % 2) + 1 (+ 2 each)
#pragma unroll
            for (int g = 0; g < kGroupsPerStep; ++g) {
              const uint64_t bg = bd + static_cast<uint64_t>((g >> 1) * (kXSubBytes >> 4) + 4 * (g & 1));
              tc_mma_ts(dt + 16u * g, at + 16u * g, bg, idesc, 0u);
              tc_mma_ts(dt + 16u * g, at + 16u * g + 8u, bg + 2u, idesc, 1u);
            }
            tc_commit(&a_free[aslot]);
            tc_commit(&d_full[dslot]);
            tc_commit(&stage_free[s]);
          }
          __syncwarp();
          // kIssuers steps on (kIssuers <= stages, kDSlots)
          s += kIssuers;
          if (s >= L.stages) s -= L.stages;
          aslot += kIssuers;
          if (aslot >= kASlots) { aslot -= kASlots; aph ^= 1u; }
          dslot += kIssuers;
          if (dslot >= kDSlots) { dslot -= kDSlots; dph ^= 1u; }
        }
        t -= len;
      }
    }
  } else if (warp < kFirstEpi) {
    // ---------------- codes -> 128 + q in tensor memory ----------------
    // Group grp takes the CTA's steps grp, grp + kDqGroups, ...
    const int quarter = warp & 3;  // a warp reaches tensor-memory lanes 32 * (warp % 4) and up
    const int grp = (warp - kFirstDq) / 4;
    const int row = 32 * quarter + lane;
    // The 64-byte swizzle stores 16-byte chunk c of row r at chunk c ^ ((r / 2) % 4).
    const int sw = (row >> 1) & 3;
    const uint32_t lane_addr = static_cast<uint32_t>(32 * quarter) << 16;
    uint32_t mask = 0x000F000Fu, bias = 0x43004300u;
    asm volatile("" : "+r"(mask), "+r"(bias));  // kept in registers for the LOP3s
    bool dead = false;
    int s = grp % L.stages, slot = grp % kASlots;
    uint32_t ph = (grp / L.stages) & 1u, sph = (grp / kASlots) & 1u;
    int t = grp;  // step within the current segment; carried over segment ends
    for (int p = L.first[blockIdx.x]; p < L.count && L.e[p].step_begin < hi; p += L.e[p].fused ? 2 : 1) {
      const GmmaEntry& E = L.e[p];
      int64_t j0, j1;
      tile_range(E, lo, hi, j0, j1);
      const int S = tile_steps(E);
      for (int64_t j = j0; j < j1; ++j) {
        const int64_t tb = E.step_begin + j * S;
        const int len = static_cast<int>(min(hi - tb, int64_t(S)) - max(lo - tb, int64_t(0)));
        for (; t < len; t += kDqGroups) {
          if (!dead && !mbar_wait_backoff<kSleepDq>(&tma_full[s], ph)) dead = true;
          const uint8_t* crow = ring + static_cast<size_t>(s) * kStageBytes + kXTileBytes + row * (kStepK / 2);
          if (!dead && !mbar_wait_backoff<kSleepDq>(&a_free[slot], sph ^ 1u)) dead = true;  // the slot's last MMAs are done
          tc_fence_after();
          const uint32_t taddr = lane_addr + static_cast<uint32_t>(slot) * kACols;
#pragma unroll
          for (int g = 0; g < kGroupsPerStep; ++g) {
            uint32_t o[16];
            codes_to_bf16(*reinterpret_cast<const uint4*>(crow + 16 * (g ^ sw)), mask, bias, o);
            tmem_st_x16(taddr + 16u * g, o);
          }
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&a_full[slot]);
          // kDqGroups steps on (kDqGroups <= stages, kASlots)
          s += kDqGroups;
          if (s >= L.stages) { s -= L.stages; ph ^= 1u; }
          slot += kDqGroups;
          if (slot >= kASlots) { slot -= kASlots; sph ^= 1u; }
        }
        t -= len;
      }
    }
  } else {
    // ---------------- epilogue: a thread per weight row ----------------
    const int quarter = warp & 3;
    const int et = tid - 32 * kFirstEpi;  // 0..127
    const int row = 32 * quarter + lane;
    const uint32_t lane_addr = (static_cast<uint32_t>(32 * quarter) << 16) + kDCol0;
    const int M = L.M;
    bool dead = false;
    int slot = 0;
    uint32_t sph = 0;
    for (int p = L.first[blockIdx.x]; p < L.count && L.e[p].step_begin < hi; p += L.e[p].fused ? 2 : 1) {
      const GmmaEntry& E = L.e[p];
      int64_t j0, j1;
      tile_range(E, lo, hi, j0, j1);
      if (j0 >= j1) continue;  // the same for all epilogue threads
      const int G = E.K / 32;
      const int Sp = E.K / kStepK, S = tile_steps(E);
      const int passes = EPI && E.fused ? 2 : 1;  // a fused problem makes the launch an EPI one
      // Group sums of x, X[g][m] in fp32 (added in k order), zero for m >= M.
      named_bar_sync(1, 128);  // all epilogue threads are done with the previous problem's sums
      const uint16_t* xp = L.x_ptr[E.x_idx];
      // From 8 rows, four sums per thread at a time with all their loads
      // issued before the adds: one L2 round trip per four sums instead of
      // per sum (the pipeline behind waits for these sums at every new
      // problem; a layer at 12 / 16 rows 92.8 -> 84.0 / 94.5 -> 87.0 us).  At
      // 4 rows the same made the decode step 8 % slower, so fewer rows keep
      // one sum at a time.
      constexpr int kXU = MC >= 8 ? 4 : 1;
      for (int i0 = et; i0 < MC * G; i0 += 128 * kXU) {
        uint4 v[kXU][4];
#pragma unroll
        for (int u = 0; u < kXU; ++u) {
          const int i = i0 + 128 * u;
          const int g = i / MC, m = i - g * MC;
          if (i < MC * G && m < M) {
            const uint4* src = reinterpret_cast<const uint4*>(xp + static_cast<int64_t>(m) * E.K + 32 * g);
#pragma unroll
            for (int c = 0; c < 4; ++c) v[u][c] = src[c];
          } else {
#pragma unroll
            for (int c = 0; c < 4; ++c) v[u][c] = make_uint4(0u, 0u, 0u, 0u);
          }
        }
#pragma unroll
        for (int u = 0; u < kXU; ++u) {
          const int i = i0 + 128 * u;
          float t = 0.f;
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const uint32_t w[4] = {v[u][c].x, v[u][c].y, v[u][c].z, v[u][c].w};
#pragma unroll
            for (int e = 0; e < 4; ++e) t = (t + __uint_as_float(w[e] << 16)) + __uint_as_float(w[e] & 0xFFFF0000u);
          }
          if (i < MC * G) xsum[i] = t;
        }
      }
      named_bar_sync(1, 128);
      for (int64_t j = j0; j < j1; ++j) {
        const int64_t grow = j * kRows + row;
        const bool row_ok = grow < E.N;
        const int64_t tb = E.step_begin + j * S;
        const int u0 = static_cast<int>(max(lo - tb, int64_t(0))), u1 = static_cast<int>(min(hi - tb, int64_t(S)));
        float acc[MC], gate[MC];
#pragma unroll
        for (int m = 0; m < MC; ++m) acc[m] = gate[m] = 0.f;
        for (int pass = 0; pass < passes; ++pass) {
          // this segment's steps [ta, tb2) of the pass (steps of 128 inputs of that weight)
          const int ta = max(u0 - pass * Sp, 0), tz = min(u1 - pass * Sp, Sp);
          if (ta < tz) {
            const GmmaEntry& W = L.e[p + pass];
            const uint16_t* srow = W.scales + (row_ok ? grow * G : 0);
            const uint16_t* brow = W.biases + (row_ok ? grow * G : 0);
            const uint32_t nbytes = row_ok ? 16u : 0u;
            const int r_end = (tz + 1) / kStepsPerSuper;  // runs [ta / 2, r_end)
            // scale/bias run r (groups 8r .. 8r+7) into slot r % kSbSlots; past
            // the last run an empty group keeps the group count uniform
            auto prefetch = [&](int r) {
              if (r < r_end) {
                const int sl = r % kSbSlots;
                cp_async_16(&sb[(2 * sl) * kRows + row], srow + 8 * r, nbytes);
                cp_async_16(&sb[(2 * sl + 1) * kRows + row], brow + 8 * r, nbytes);
              }
              cp_async_commit();
            };
#pragma unroll
            for (int r = 0; r < kSbPrefetch; ++r) prefetch(ta / kStepsPerSuper + r);
            const uint2* run = nullptr;  // this row's current scale run; its bias run is kRows uint4 on
            for (int t = ta; t < tz; ++t) {
              const int half = t % kStepsPerSuper;
              if (half == 0 || t == ta) {
                const int r = t / kStepsPerSuper;
                cp_async_wait<kSbPrefetch - 1>();  // run r has landed
                run = reinterpret_cast<const uint2*>(&sb[(2 * (r % kSbSlots)) * kRows + row]);
                prefetch(r + kSbPrefetch);  // into the slot run r - 1 used
              }
              // groups 4t .. 4t+3: words 2 * half and 2 * half + 1 of the runs
              const uint2 s2 = run[half], b2 = run[half + 2 * kRows];
              float sg[kGroupsPerStep], cg[kGroupsPerStep];
              sg[0] = __uint_as_float(s2.x << 16);
              sg[1] = __uint_as_float(s2.x & 0xFFFF0000u);
              sg[2] = __uint_as_float(s2.y << 16);
              sg[3] = __uint_as_float(s2.y & 0xFFFF0000u);
              cg[0] = fmaf(-128.f, sg[0], __uint_as_float(b2.x << 16));
              cg[1] = fmaf(-128.f, sg[1], __uint_as_float(b2.x & 0xFFFF0000u));
              cg[2] = fmaf(-128.f, sg[2], __uint_as_float(b2.y << 16));
              cg[3] = fmaf(-128.f, sg[3], __uint_as_float(b2.y & 0xFFFF0000u));
              const float* xg = xsum + kGroupsPerStep * MC * t;
              if (!dead && !mbar_wait_backoff<kSleepEpi>(&d_full[slot], sph)) dead = true;
              tc_fence_after();
              const uint32_t dcol = lane_addr + static_cast<uint32_t>(slot) * kDCols;
              // the groups' sums, several groups per load (one wait): 4 at 1..2
              // rows, 2 at 4 and at 16 (16 rows: 1,643 -> 1,558 us on the decode
              // step), 1 at 8 (2 measured slightly slower there)
              constexpr int kGL = MC <= 2 ? 4 : MC == 8 ? 1 : 2;
#pragma unroll
              for (int g0 = 0; g0 < kGroupsPerStep; g0 += kGL) {
                uint32_t d[kGL][MC];
#pragma unroll
                for (int gg = 0; gg < kGL; ++gg) tmem_ld_d<MC>(dcol + 16u * (g0 + gg), d[gg]);
                tmem_wait_ld();
                if (g0 + kGL == kGroupsPerStep) {  // all of the slot read
                  tc_fence_before();
                  __syncwarp();
                  if (lane == 0) mbar_arrive(&d_free[slot]);
                }
                // rows m >= M: D and X are zero, and acc[m] is not stored
#pragma unroll
                for (int gg = 0; gg < kGL; ++gg) {
                  const int g = g0 + gg;
#pragma unroll
                  for (int m = 0; m < MC; ++m)
                    acc[m] = fmaf(cg[g], xg[g * MC + m], fmaf(sg[g], __uint_as_float(d[gg][m]), acc[m]));
                }
              }
              if (++slot == kDSlots) { slot = 0; sph ^= 1u; }
            }
          }
          if (passes == 2 && pass == 0) {
#pragma unroll
            for (int m = 0; m < MC; ++m) {
              gate[m] = acc[m];
              acc[m] = 0.f;
            }
          }
        }
        if (dead) {
#pragma unroll
          for (int m = 0; m < MC; ++m) acc[m] = gate[m] = kNaN;
        }
        bool finish = true;  // this CTA writes y for the tile
        if (u0 != 0 || u1 != S) {
          // A tile shared with other CTAs: publish this piece's partial sums;
          // the CTA that arrives last adds all pieces in piece order and writes y.
          const int64_t T = L.total_steps, Gd = gridDim.x;
          const int64_t c0 = ((tb + 1) * Gd + T - 1) / T - 1;          // owner of the tile's first step
          const int64_t c1 = ((tb + S) * Gd + T - 1) / T - 1;          // owner of its last step
          const int64_t me = blockIdx.x;
          auto slot_of = [&](int64_t c) { return 2 * c + (cta_first_step(L, c) < tb ? 1 : 0); };
          float* mine = L.partials + (slot_of(me) * kRows + row) * (2 * MC);
#pragma unroll
          for (int m = 0; m < MC; ++m) {
            mine[m] = gate[m];
            mine[MC + m] = acc[m];
          }
          __threadfence();
          named_bar_sync(1, 128);
          if (et == 0) *last_flag = atomicAdd(&L.counters[c0], 1u) == static_cast<unsigned>(c1 - c0) ? 1u : 0u;
          named_bar_sync(1, 128);
          finish = *last_flag != 0;
          if (finish) {
            __threadfence();
            for (int64_t c = c0; c <= c1; ++c) {
              const float* part = L.partials + (slot_of(c) * kRows + row) * (2 * MC);
#pragma unroll
              for (int m = 0; m < MC; ++m) {
                const float g = __ldcg(part + m), v = __ldcg(part + MC + m);
                gate[m] = c == c0 ? g : gate[m] + g;
                acc[m] = c == c0 ? v : acc[m] + v;
              }
            }
            if (et == 0) L.counters[c0] = 0u;  // as found, for a launch that reuses the counters
          }
        }
        if (finish && row_ok) {
#pragma unroll
          for (int m = 0; m < MC; ++m)
            if (m < M) {
              const int64_t idx = static_cast<int64_t>(m) * E.N + grow;
              if constexpr (EPI) {
                if (passes == 2) E.y[idx] = float_to_bf16_bits(silu_f32(gate[m]) * acc[m]);
                else E.y[idx] = epilogue_bf16(acc[m], E.epi, E.r, idx);
              } else {
                E.y[idx] = float_to_bf16_bits(acc[m]);
              }
            }
        }
      }
    }
    cp_async_wait<0>();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(*tmem_slot, kTmemCols);
  }
}

// ---- host side ------------------------------------------------------------

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

constexpr size_t kBarrierBytes = 8 * (2 * kMaxStages + 2 * kASlots + 2 * kDSlots) + 16;
constexpr size_t kFixedSmem = kSbBytes + kBarrierBytes + 1024;  // + 1024: aligning the ring

bool encode_codes(CUtensorMap* map, const uint8_t* codes, int64_t N, int64_t K) {
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(K / 2), static_cast<cuuint64_t>(N)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(K / 2)};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(kStepK / 2), static_cast<cuuint32_t>(kRows)};
  cuuint32_t estr[2] = {1, 1};
  return encode_fn()(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(codes), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool encode_x(CUtensorMap* map, const uint16_t* x, int64_t M, int64_t K) {
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(M)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(K) * 2};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(kSubK), static_cast<cuuint32_t>(kN)};
  cuuint32_t estr[2] = {1, 1};
  return encode_fn()(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(x), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int MC>
const void* kernel_for(bool epi) {
  return epi ? reinterpret_cast<const void*>(gmma_kernel<MC, true>)
             : reinterpret_cast<const void*>(gmma_kernel<MC, false>);
}
const void* kernel_of(int mc, bool epi) {
  switch (mc) {
    case 1: return kernel_for<1>(epi);
    case 2: return kernel_for<2>(epi);
    case 4: return kernel_for<4>(epi);
    case 8: return kernel_for<8>(epi);
    default: return kernel_for<16>(epi);
  }
}

int rows_class(int64_t M) { return M <= 1 ? 1 : M <= 2 ? 2 : M <= 4 ? 4 : M <= 8 ? 8 : 16; }
// the group sums X [K/32][rows_class(M)] in fp32
size_t x_area_bytes(int64_t M, int64_t K) {
  return static_cast<size_t>(rows_class(M)) * static_cast<size_t>(K / 32) * 4 + 16;
}

}  // namespace

bool gmma_supported(const MatmulArgs& a, const DeviceInfo& dev) {
  if (a.M < kGmmaMinRows || a.M > kGmmaMaxRows) return false;
  if (a.K < kSuperK || a.K % kSuperK != 0 || a.K > (int64_t(1) << 20)) return false;
  if (a.N < 1 || a.N > (int64_t(1) << 31) - kRows) return false;
  uintptr_t al = reinterpret_cast<uintptr_t>(a.scales) | reinterpret_cast<uintptr_t>(a.biases) |
                 reinterpret_cast<uintptr_t>(a.codes) | reinterpret_cast<uintptr_t>(a.x);
  if (a.fused())
    al |= reinterpret_cast<uintptr_t>(a.up_scales) | reinterpret_cast<uintptr_t>(a.up_biases) |
          reinterpret_cast<uintptr_t>(a.up_codes);
  if (al & 15u) return false;
  // the group sums and kMinStages stages must fit beside the fixed areas
  if (x_area_bytes(a.M, a.K) + kMinStages * kStageBytes + kFixedSmem > dev.smem_optin) return false;
  return encode_fn() != nullptr;
}

// Splits `list` (every problem gmma_supported) into launches -- the same M,
// at most kMaxEntries weights, kMaxXMaps distinct activation tensors and
// group sums that fit in shared memory each -- and encodes every tensor map.
// Nothing is launched.
cudaError_t plan_gmma(const MatmulArgs* list, int count, const DeviceInfo& dev, std::vector<GmmaPlan>& plans) {
  int i = 0;
  while (i < count) {
    plans.emplace_back();
    GmmaPlan& pl = plans.back();
    GmmaLaunch& L = *new (pl.params) GmmaLaunch;
    std::memset(&L, 0, sizeof L);
    int nx = 0, ne = 0;
    int64_t x_k[kMaxXMaps] = {};
    size_t xbytes = 0;
    int64_t total = 0;  // steps
    bool epi = false;
    const int64_t M = list[i].M;
    while (i < count) {
      const MatmulArgs& a = list[i];
      const int need = a.fused() ? 2 : 1;
      if (ne + need > kMaxEntries || a.M != M) break;
      int xi = -1;  // an activation tensor is its pointer and its K
      for (int t = 0; t < nx; ++t)
        if (L.x_ptr[t] == a.x && x_k[t] == a.K) xi = t;
      if (xi < 0 && nx == kMaxXMaps) break;
      const size_t xb = std::max(xbytes, x_area_bytes(M, a.K));
      if (xb + kMinStages * kStageBytes + kFixedSmem > dev.smem_optin) break;
      if (xi < 0) {
        if (!encode_x(&L.x_map[nx], a.x, M, a.K)) return cudaErrorInvalidValue;
        L.x_ptr[nx] = a.x;
        x_k[nx] = a.K;
        xi = nx++;
      }
      for (int w = 0; w < need; ++w) {
        GmmaEntry& E = L.e[ne + w];
        if (!encode_codes(&E.codes_map, w ? a.up_codes : a.codes, a.N, a.K)) return cudaErrorInvalidValue;
        E.scales = w ? a.up_scales : a.scales;
        E.biases = w ? a.up_biases : a.biases;
        E.y = a.y;
        E.r = a.r;
        E.step_begin = total;
        E.N = static_cast<int32_t>(a.N);
        E.K = static_cast<int32_t>(a.K);
        E.x_idx = xi;
        E.epi = static_cast<int16_t>(a.epi);
        E.fused = static_cast<int16_t>(a.fused() ? 1 + w : 0);
      }
      total += (a.N + kRows - 1) / kRows * (a.K / kStepK) * need;
      xbytes = xb;
      epi = epi || a.epi != kEpiNone || a.fused();
      ne += need;
      ++i;
    }
    if (ne == 0) return cudaErrorInvalidValue;  // a problem that fits no launch alone
    L.count = ne;
    L.M = static_cast<int32_t>(M);
    L.x_floats = static_cast<int32_t>((xbytes / 4 + 3) & ~size_t(3));  // keeps the barriers after it aligned
    const size_t fixed = static_cast<size_t>(L.x_floats) * 4 + kFixedSmem;
    L.stages = static_cast<int32_t>(std::min<size_t>(kMaxStages, (dev.smem_optin - fixed) / kStageBytes));
    if (L.stages < kMinStages) return cudaErrorInvalidConfiguration;
    L.total_steps = total;
    // every SM takes an equal share of the steps (one CTA per SM: each
    // allocates all 512 tensor-memory columns)
    const int64_t grid = std::max<int64_t>(1, std::min<int64_t>(std::min(dev.sm_count, kMaxCtas), total));
    pl.grid = static_cast<int>(grid);
    // each CTA's first entry: the first whose tiles end after the CTA's first
    // step (the kernel's cta_first_step formula)
    for (int64_t c = 0, p = 0; c < grid; ++c) {
      const int64_t lo = total * c / grid;
      auto end_of = [&](int64_t q) {
        const GmmaEntry& E = L.e[q];
        return E.step_begin + (E.N + kRows - 1) / kRows * (E.K / kStepK) * (E.fused ? 2 : 1);
      };
      while (p < ne && end_of(p) <= lo) p += L.e[p].fused ? 2 : 1;
      L.first[c] = static_cast<uint8_t>(p);
    }
    pl.smem = dev.smem_optin;
    pl.kern = kernel_of(rows_class(M), epi);
    // Is a tile shared by two CTAs (a CTA boundary inside a tile)?
    bool shared = false;
    int e = 0;
    for (int64_t c = 1; c < grid && !shared; ++c) {
      const int64_t b = total * c / grid;
      while (e + 1 < ne && L.e[e + 1].step_begin <= b) ++e;
      const int64_t S = (L.e[e].K / kStepK) * (L.e[e].fused ? 2 : 1);
      shared = (b - L.e[e].step_begin) % S != 0;
    }
    pl.counter_bytes = shared ? (static_cast<size_t>(grid) * 4 + 255) / 256 * 256 : 0;
    pl.partial_bytes = shared ? static_cast<size_t>(2 * grid) * kRows * 2 * rows_class(M) * 4 : 0;
  }
  return cudaSuccess;
}

cudaError_t launch_planned_gmma(GmmaPlan& pl, unsigned int* counters, float* partials, cudaStream_t stream) {
  GmmaLaunch& L = *reinterpret_cast<GmmaLaunch*>(pl.params);
  L.counters = counters;
  L.partials = partials;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(pl.grid));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = pl.smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  count_launch();
  void* args[] = {const_cast<unsigned char*>(pl.params)};
  return cudaLaunchKernelExC(&cfg, pl.kern, args);
}

cudaError_t gmma_device_flags(unsigned int* flags, bool clear) { return tu_device_flags(flags, clear); }

cudaError_t gmma_prepare_device(const DeviceInfo& dev) {
  for (int mc : {1, 2, 4, 8, 16})
    for (bool epi : {false, true}) {
      const cudaError_t e = cudaFuncSetAttribute(kernel_of(mc, epi), cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 static_cast<int>(dev.smem_optin));
      if (e != cudaSuccess) return e;
    }
  return cudaSuccess;
}

}  // namespace q4
