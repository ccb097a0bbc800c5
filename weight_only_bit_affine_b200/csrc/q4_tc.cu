// q4_tc.cu -- tensor-core tiles of the affine Q4 group-32 matmul for many
// activation rows (prefill, concurrent conversations):
//
//   y[m,n] = sum_k x[m,k] * w_hat[n,k],   w_hat = s*q + b  (group 32 along k)
//
// The packed weights are dequantized tile by tile into tensor memory (never
// to HBM) and multiplied on the 5th-generation tensor cores (tcgen05.mma,
// kind::f16, bf16 x bf16 -> fp32 accumulation in tensor memory).  The Swift
// blog's prefill batching (voice prompt and prefill as one batched forward)
// and the four concurrent conversations of "A smaller voice model" are the
// workloads with several rows.
//
// Tile: 128 weight rows (the MMA's M side and the 128 tensor-memory lanes:
// D[n, m] = w_hat . x^T, so the output tile is y^T) x BN activation rows
// (the MMA's N side, 16..256) x the CTA's K range, walked in atoms of 64
// inputs (one 128-byte swizzle span of bf16 x).  Each weight enters the MMA
// as two bf16 parts, hi + lo (q4_tcgen05.cuh, dequant_word_hilo), so the operand
// is within ~2^-16 of the exact s*q + b; every atom is two groups of four
// K16 MMAs (hi, then lo) into the same accumulator.
//
// Per CTA (576 threads):
//   warp 0       TMA producer: per stage, the x tiles (tensor map, 128-byte
//                swizzle) and the code tile (tensor map, 128 rows x 32 bytes
//                per atom);
//   warp 1       allocates tensor memory; one thread issues the MMAs (A from
//                tensor memory, B = the x tile in shared memory) and commits
//                them to the barriers that free the A slot and the stage;
//   warps 2..17  dequantize, in four groups of four warps (one per
//                tensor-memory lane quarter) taking the atoms in turn, so
//                four atoms are in flight: the thread of weight row r turns
//                the row's 64 codes of an atom into 32 hi and 32 lo bf16
//                pairs and stores them to its tensor-memory lane
//                (tcgen05.st) in the atom's A slot, a ring of slots after
//                the accumulators; then the epilogue (tensor memory ->
//                registers -> bf16 y).
// SwiGLU (gate and up weights of the same shape): the up weight's atoms
// follow the gate's over the same K range into a second accumulator, and the
// epilogue writes silu(gate) * up from the two fp32 results.
// Split-K: when there are too few tiles to fill the GPU, the K range is split
// across the CTAs of a thread-block cluster, and the fp32 partial tiles are
// summed through distributed shared memory (no global workspace), laid out so
// that every warp's remote load reads 512 contiguous bytes.
// Every wait is bounded (q4_device.cuh); a thread whose wait gave up writes
// NaN.  Programmatic dependent launch as in the GEMV family.
#include "q4_device.cuh"
#include "q4_internal.h"
#include "q4_tcgen05.cuh"

#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>

namespace q4 {
namespace {

constexpr int kTileN = 128;                  // weight rows per tile (MMA M, tensor-memory lanes)
constexpr int kAtomK = 64;                   // K per atom (one 128-byte swizzle span of bf16)
constexpr int kSuperK = 256;                 // K per scale/bias load (8 groups = 16 bytes per row)
constexpr int kAtomsPerSuper = kSuperK / kAtomK;
constexpr int kDqGroups = 4;                 // dequantizing warp groups, taking atoms in turn
constexpr int kDqWarpsPerGroup = 4;          // one per tensor-memory lane quarter
constexpr int kDqWarps = kDqGroups * kDqWarpsPerGroup;
constexpr int kThreads = 64 + 32 * kDqWarps;  // 576
constexpr uint32_t kTmemCols = 512;
constexpr int kASlotCols = 64;               // one atom of A: hi (32 columns of bf16 pairs), then lo (32)
constexpr int kMaxASlots = 8;
constexpr int kMaxStages = 8;
constexpr int kCodeAtomBytes = kTileN * kAtomK / 2;  // 4 KB
constexpr float kNaN = __builtin_nanf("");


__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int c0, int c1, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
      ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ uint32_t dsmem_map(uint32_t local_addr, uint32_t rank) {
  uint32_t remote;
  asm("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(local_addr), "r"(rank));
  return remote;
}
__device__ __forceinline__ float4 ld_dsmem_v4(uint32_t remote_addr) {
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(remote_addr));
  return v;
}

// One output element from the tile's fp32 result(s).
template <bool EPI>
__device__ __forceinline__ uint16_t out_tc(float g, float u, const TcParams& p, int64_t idx) {
  if constexpr (EPI) {
    if (p.nacc == 2) return float_to_bf16_bits(silu_f32(g) * u);
    return epilogue_bf16(g, p.epi, p.r, idx);
  }
  return float_to_bf16_bits(g);
}

template <int ATOMS, bool EPI>
__global__ void __launch_bounds__(kThreads, 1)
    tc_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_codes,
              const __grid_constant__ CUtensorMap tmap_up, const __grid_constant__ TcParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // 1024-byte alignment for the swizzled x tiles.
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  uint64_t* tma_full = reinterpret_cast<uint64_t*>(smem + static_cast<size_t>(p.stages) * p.stage_bytes);
  uint64_t* stage_free = tma_full + kMaxStages;
  uint64_t* a_full = stage_free + kMaxStages;
  uint64_t* a_empty = a_full + kMaxASlots;
  uint64_t* accum_full = a_empty + kMaxASlots;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accum_full + 1);

  const int split = static_cast<int>(blockIdx.x);  // == cluster rank along x
  const int64_t n0 = static_cast<int64_t>(blockIdx.y) * kTileN;
  const int64_t m0 = static_cast<int64_t>(blockIdx.z) * p.bn;
  const int supers = p.K / kSuperK;
  const int sc_begin = split * supers / p.splits, sc_end = (split + 1) * supers / p.splits;
  const int pass_supers = sc_end - sc_begin;
  const int pass_atoms = pass_supers * kAtomsPerSuper;  // atoms of one weight over this CTA's K range
  const int natoms = pass_atoms * p.nacc;               // SwiGLU: the up weight's atoms follow the gate's
  const int k_begin = sc_begin * kSuperK;

  if (tid == 0) {
    for (int s = 0; s < p.stages; ++s) {
      mbar_init(&tma_full[s], 1);
      mbar_init(&stage_free[s], 1);
    }
    for (int a = 0; a < p.a_slots; ++a) {
      mbar_init(&a_full[a], kDqWarpsPerGroup);
      mbar_init(&a_empty[a], 1);
    }
    mbar_init(accum_full, 1);
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_launch_dependents();
  pdl_wait_predecessors();

  // Stage layout: ATOMS x tiles (bn rows x 128 B each), then the code tile
  // (128 rows x 32 * ATOMS bytes).
  const uint32_t b_atom = p.b_atom_bytes;
  auto b_tile = [&](int s) { return smem + static_cast<size_t>(s) * p.stage_bytes; };
  auto c_tile = [&](int s) { return b_tile(s) + ATOMS * b_atom; };
  const int nsteps = natoms / ATOMS;

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    // The whole warp runs the loop; the elected lane issues the copies.
    const bool leader = elect_one();
    {
      bool dead = false;
      int s = 0;
      uint32_t ph = 0;
      for (int j = 0; j < nsteps; ++j) {
        if (!dead && !mbar_wait<false>(&stage_free[s], ph ^ 1u)) dead = true;
        const int a = j * ATOMS;
        const bool up = a >= pass_atoms;
        const int k0 = k_begin + (a - (up ? pass_atoms : 0)) * kAtomK;
        if (leader) {
          mbar_arrive_expect_tx(&tma_full[s], ATOMS * (b_atom + kCodeAtomBytes));
#pragma unroll
          for (int at = 0; at < ATOMS; ++at)
            tma_load_2d(b_tile(s) + at * b_atom, &tmap_x, k0 + at * kAtomK, static_cast<int>(m0), &tma_full[s]);
          tma_load_2d(c_tile(s), up ? &tmap_up : &tmap_codes, k0 / 2, static_cast<int>(n0), &tma_full[s]);
        }
        __syncwarp();
        if (++s == p.stages) { s = 0; ph ^= 1u; }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    // Waits only for the dequantizing warps: they arrive after having waited
    // for the stage's TMA themselves, so the x tile is in place too.  The
    // whole warp runs the loop (warp-uniform operands); the elected lane
    // issues the MMAs and commits.
    const bool leader = elect_one();
    {
      bool dead = false;
      const uint32_t a_base = tmem_base + p.a_col0;
      int slot = 0, s = 0, sub = 0;
      uint32_t aph = 0, ph = 0;
      for (int a = 0; a < natoms; ++a) {
        if (!dead && !mbar_wait<false>(&a_full[slot], aph)) dead = true;
        tc_fence_after();
        const bool up = a >= pass_atoms;
        const uint32_t acc = tmem_base + (up ? static_cast<uint32_t>(p.bn) : 0u);
        const bool first = (a == 0) || (a == pass_atoms);
        const uint64_t bd = sw128_desc(smem_u32(b_tile(s) + sub * b_atom));
        const uint32_t at = a_base + static_cast<uint32_t>(slot) * kASlotCols;
        if (leader) {
#pragma unroll
          for (int kk = 0; kk < kAtomK / 16; ++kk)  // hi: 8 columns (16 bf16 along K) per MMA
            tc_mma_ts(acc, at + 8 * kk, bd + 2 * kk, p.idesc, (first && kk == 0) ? 0u : 1u);
#pragma unroll
          for (int kk = 0; kk < kAtomK / 16; ++kk)  // lo, same activations
            tc_mma_ts(acc, at + 32 + 8 * kk, bd + 2 * kk, p.idesc, 1u);
          tc_commit(&a_empty[slot]);
        }
        __syncwarp();
        if (++slot == p.a_slots) { slot = 0; aph ^= 1u; }
        if (++sub == ATOMS) {
          sub = 0;
          if (leader) tc_commit(&stage_free[s]);
          __syncwarp();
          if (++s == p.stages) { s = 0; ph ^= 1u; }
        }
      }
      if (leader) tc_commit(accum_full);
    }
  } else {
    // ---------------- dequantize, then epilogue ----------------
    const int quarter = warp & 3;  // the tensor-memory lanes this warp may access
    const int grp = (warp - 2) >> 2;
    const int row = 32 * quarter + lane;  // weight row within the tile
    const int64_t grow = n0 + row;
    const bool row_ok = grow < p.N;
    const int G = p.K / 32;
    const uint32_t lane_addr = tmem_base + (static_cast<uint32_t>(32 * quarter) << 16);
    // A group takes every kDqGroups-th atom: one per super-chunk (8 groups of
    // 32), always the same atom of it, so it needs one 32-bit word (two bf16)
    // of the row's scales and of its biases per super-chunk, fetched one
    // super-chunk ahead; u counts super-chunks over both passes of a SwiGLU
    // tile.
    static_assert(kDqGroups == kAtomsPerSuper, "one atom per super-chunk per group");
    auto load_sb = [&](int u, uint32_t& sv, uint32_t& bv) {
      sv = bv = 0u;
      if (!row_ok || u >= pass_supers * p.nacc) return;
      const bool up = u >= pass_supers;
      const int64_t off =
          grow * G + static_cast<int64_t>(sc_begin + u - (up ? pass_supers : 0)) * (kSuperK / 32) + 2 * grp;
      sv = *reinterpret_cast<const uint32_t*>((up ? p.up_scales : p.scales) + off);
      bv = *reinterpret_cast<const uint32_t*>((up ? p.up_biases : p.biases) + off);
    };
    uint32_t s_cur, b_cur, s_nxt, b_nxt;
    load_sb(0, s_cur, b_cur);
    load_sb(1, s_nxt, b_nxt);
    bool dead = false;
    // Stage and A slot of this group's atoms, advanced incrementally (atom a
    // sits in stage (a / ATOMS) mod stages and slot a mod a_slots).
    constexpr int kStageStep = kDqGroups / ATOMS;  // stages per group turn (ATOMS divides kDqGroups)
    int st = grp / ATOMS, slot = grp;
    uint32_t ph = 0, sph = 0;
    while (st >= p.stages) { st -= p.stages; ph ^= 1u; }
    while (slot >= p.a_slots) { slot -= p.a_slots; sph ^= 1u; }
    for (int a = grp, u = 0; a < natoms; a += kDqGroups, ++u) {
      if (u > 0) {
        s_cur = s_nxt;
        b_cur = b_nxt;
        load_sb(u + 1, s_nxt, b_nxt);
      }
      if (!dead && !mbar_wait(&tma_full[st], ph)) dead = true;  // codes arrived
      const uint4* cp = reinterpret_cast<const uint4*>(c_tile(st) + row * (32 * ATOMS) + (a % ATOMS) * 32);
      const uint4 cw0 = cp[0], cw1 = cp[1];  // the atom's two groups of 32 codes of this row
      const uint32_t sw = s_cur, bw = b_cur;
      const uint64_t s20 = f32x2_splat(__uint_as_float(sw << 16)), b20 = f32x2_splat(__uint_as_float(bw << 16));
      const uint64_t s21 = f32x2_splat(__uint_as_float(sw & 0xFFFF0000u));
      const uint64_t b21 = f32x2_splat(__uint_as_float(bw & 0xFFFF0000u));
      // All 64 codes into registers first (separate arrays: a tcgen05.st reads
      // its source registers after it issues, so none is overwritten early).
      uint32_t hi0[16], lo0[16], hi1[16], lo1[16];
      dequant_word_hilo(cw0.x, s20, b20, hi0, lo0);
      dequant_word_hilo(cw0.y, s20, b20, hi0 + 4, lo0 + 4);
      dequant_word_hilo(cw0.z, s20, b20, hi0 + 8, lo0 + 8);
      dequant_word_hilo(cw0.w, s20, b20, hi0 + 12, lo0 + 12);
      dequant_word_hilo(cw1.x, s21, b21, hi1, lo1);
      dequant_word_hilo(cw1.y, s21, b21, hi1 + 4, lo1 + 4);
      dequant_word_hilo(cw1.z, s21, b21, hi1 + 8, lo1 + 8);
      dequant_word_hilo(cw1.w, s21, b21, hi1 + 12, lo1 + 12);
      if (!dead && !mbar_wait(&a_empty[slot], sph ^ 1u)) dead = true;  // the MMAs of the slot's last atom are done
      tc_fence_after();
      const uint32_t taddr = lane_addr + p.a_col0 + static_cast<uint32_t>(slot) * kASlotCols;
      tmem_st_x16(taddr, hi0);
      tmem_st_x16(taddr + 16u, hi1);
      tmem_st_x16(taddr + 32u, lo0);
      tmem_st_x16(taddr + 48u, lo1);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&a_full[slot]);
      st += kStageStep;
      while (st >= p.stages) { st -= p.stages; ph ^= 1u; }
      slot += kDqGroups;
      while (slot >= p.a_slots) { slot -= p.a_slots; sph ^= 1u; }
    }

    // ---- epilogue: tensor memory -> y (or partial sums for the cluster) ----
    if (!dead && !mbar_wait(accum_full, 0)) dead = true;
    tc_fence_after();
    const int part = (warp - 2) >> 2;  // 0..3: which column octets this warp reads
    // Partial tile for the cluster's sum, in the stage area (all MMAs are
    // done): four columns per 16-byte unit, the 128 rows of a unit
    // consecutive (unit c4 of row r at c4 * 128 + r), so a warp's store and a
    // peer warp's load each cover 512 contiguous bytes.
    float4* red = reinterpret_cast<float4*>(smem);
    for (int c0 = 8 * part; c0 < p.bn; c0 += 32) {
      uint32_t gr[8], ur[8];
      tmem_ld_cols<8>(lane_addr + c0, gr);
      if (p.nacc == 2) tmem_ld_cols<8>(lane_addr + p.bn + c0, ur);
      tmem_wait_ld();
      float g[8], u[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        g[i] = dead ? kNaN : __uint_as_float(gr[i]);
        u[i] = (p.nacc == 2) ? (dead ? kNaN : __uint_as_float(ur[i])) : 0.f;
      }
      if (p.splits == 1) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int64_t m = m0 + c0 + i;
          if (row_ok && m < p.M) p.y[m * p.N + grow] = out_tc<EPI>(g[i], u[i], p, m * p.N + grow);
        }
      } else {
        red[(c0 / 4) * kTileN + row] = make_float4(g[0], g[1], g[2], g[3]);
        red[(c0 / 4 + 1) * kTileN + row] = make_float4(g[4], g[5], g[6], g[7]);
        if (p.nacc == 2) {
          red[((p.bn + c0) / 4) * kTileN + row] = make_float4(u[0], u[1], u[2], u[3]);
          red[((p.bn + c0) / 4 + 1) * kTileN + row] = make_float4(u[4], u[5], u[6], u[7]);
        }
      }
    }
  }

  if (p.splits > 1) {
    // Sum the cluster's partial tiles: CTA `split` finishes columns
    // [split * bn / splits, (split + 1) * bn / splits) of every row.
    cluster_sync_all();
    if (warp >= 2) {
      const int t = tid - 64;
      const int trow = t & (kTileN - 1);
      const int64_t grow = n0 + trow;
      // Column slice of this CTA, in float4 units (bn and the slice are multiples of 4).
      const int q_beg = split * (p.bn / 4) / p.splits, q_end = (split + 1) * (p.bn / 4) / p.splits;
      const uint32_t row_addr = smem_u32(smem) + static_cast<uint32_t>(trow) * 16u;
      uint32_t peer[8];
#pragma unroll
      for (int r = 0; r < 8; ++r) peer[r] = dsmem_map(row_addr, static_cast<uint32_t>(r < p.splits ? r : 0));
      for (int q = q_beg + (t >> 7); q < q_end; q += kDqWarps * 32 / kTileN) {
        float4 acc[2] = {make_float4(0.f, 0.f, 0.f, 0.f), make_float4(0.f, 0.f, 0.f, 0.f)};
#pragma unroll
        for (int w = 0; w < 2; ++w) {  // the gate's (or only) partial tiles, then the up weight's
          if (w >= p.nacc) break;
          float4 v[8];
#pragma unroll
          for (int r = 0; r < 8; ++r)  // all peers' loads first, then the sums
            if (r < p.splits)
              v[r] = ld_dsmem_v4(peer[r] + static_cast<uint32_t>((w * (p.bn / 4) + q) * kTileN) * 16u);
          float4 t = v[0];
#pragma unroll
          for (int r = 1; r < 8; ++r)
            if (r < p.splits) {
              t.x += v[r].x;
              t.y += v[r].y;
              t.z += v[r].z;
              t.w += v[r].w;
            }
          acc[w] = t;
        }
        const float4 ag = acc[0], au = acc[1];
        const float og[4] = {ag.x, ag.y, ag.z, ag.w}, ou[4] = {au.x, au.y, au.z, au.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int64_t m = m0 + 4 * q + i;
          if (grow < p.N && m < p.M) p.y[m * p.N + grow] = out_tc<EPI>(og[i], ou[i], p, m * p.N + grow);
        }
      }
    }
    cluster_sync_all();  // no CTA leaves while a peer may still read its shared memory
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
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

constexpr size_t kBarrierBytes = 8 * (2 * kMaxStages + 2 * kMaxASlots + 1) + 16;

template <int ATOMS, bool EPI>
void* kernel_of() {
  return reinterpret_cast<void*>(tc_kernel<ATOMS, EPI>);
}

}  // namespace

cudaError_t tc_device_flags(unsigned int* flags, bool clear) { return tu_device_flags(flags, clear); }

cudaError_t tc_prepare_device(const DeviceInfo& dev) {
  for (void* kern : {kernel_of<1, false>(), kernel_of<2, false>(), kernel_of<1, true>(), kernel_of<2, true>()}) {
    cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(dev.smem_optin));
    if (e == cudaSuccess) e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 0);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

bool tc_supported(const MatmulArgs& a) {
  if (a.K % kSuperK != 0) return false;
  uintptr_t sb = reinterpret_cast<uintptr_t>(a.scales) | reinterpret_cast<uintptr_t>(a.biases);
  if (a.fused()) sb |= reinterpret_cast<uintptr_t>(a.up_scales) | reinterpret_cast<uintptr_t>(a.up_biases);
  if (sb & 15u) return false;
  if (a.N > (int64_t(1) << 31) - kTileN || a.M > (int64_t(1) << 31) - 256) return false;
  return encode_fn() != nullptr;
}


cudaError_t plan_tc(const MatmulArgs& a, const DeviceInfo& dev, TcLaunch* out) {
  PFN_cuTensorMapEncodeTiled_v12000 encode = encode_fn();
  if (!encode) return cudaErrorNotSupported;
  const bool swiglu = a.fused();
  const int nacc = swiglu ? 2 : 1;
  const int bn_max = swiglu ? 128 : 256;  // the accumulators and a 4-slot A ring share 512 columns
  const int bn = static_cast<int>(std::min<int64_t>(bn_max, (a.M + 15) / 16 * 16));
  const int64_t n_tiles = (a.N + kTileN - 1) / kTileN;
  const int64_t m_tiles = (a.M + bn - 1) / bn;
  const int supers = static_cast<int>(a.K / kSuperK);
  // Split K over a cluster of up to 8 CTAs when the tiles alone would leave
  // SMs idle: the split minimising waves x (super-chunks per CTA + 4), the
  // "+ 4" standing for a CTA's fixed cost, measured at about four
  // super-chunks of main loop (the pipeline's fill, its drain and the
  // epilogue); ties go to the smaller split, which also saves the
  // cluster's sum.  One CTA per SM, so a wave is sm_count CTAs.
  int splits = 1;
  const int64_t tiles = n_tiles * m_tiles;
  {
    int64_t best = -1;
    for (int sp = 1; sp <= 8 && sp <= supers; ++sp) {
      const int64_t waves = (tiles * sp + dev.sm_count - 1) / dev.sm_count;
      const int64_t cost = waves * ((supers + sp - 1) / sp + 4);
      if (best < 0 || cost < best) { best = cost; splits = sp; }
    }
  }

  // Two atoms per stage when at least three such stages fit.
  const uint32_t b_atom = static_cast<uint32_t>(bn) * kAtomK * 2;
  auto stage_size = [&](int atoms) {
    return (static_cast<uint32_t>(atoms) * (b_atom + kCodeAtomBytes) + 1023u) & ~1023u;
  };
  const size_t avail = dev.smem_optin - 1024 - kBarrierBytes;
  const int atoms = (avail / stage_size(2) >= 3) ? 2 : 1;

  TcLaunch& L = *out;
  {
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(a.K), static_cast<cuuint64_t>(a.M)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(a.K) * 2};
    cuuint32_t box[2] = {static_cast<cuuint32_t>(kAtomK), static_cast<cuuint32_t>(bn)};
    cuuint32_t estr[2] = {1, 1};
    if (encode(&L.tmap_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(a.x), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  for (int w = 0; w < nacc; ++w) {
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(a.K / 2), static_cast<cuuint64_t>(a.N)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(a.K / 2)};
    cuuint32_t box[2] = {static_cast<cuuint32_t>(kAtomK / 2 * atoms), static_cast<cuuint32_t>(kTileN)};
    cuuint32_t estr[2] = {1, 1};
    const uint8_t* codes = w == 0 ? a.codes : a.up_codes;
    if (encode(w == 0 ? &L.tmap_codes : &L.tmap_up, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(codes),
               dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  if (!swiglu) L.tmap_up = L.tmap_codes;

  TcParams& p = L.p;
  p.scales = a.scales;
  p.biases = a.biases;
  p.up_scales = swiglu ? a.up_scales : nullptr;
  p.up_biases = swiglu ? a.up_biases : nullptr;
  p.y = a.y;
  p.r = a.r;
  p.epi = a.epi;
  p.M = a.M;
  p.N = a.N;
  p.K = static_cast<int>(a.K);
  p.bn = bn;
  p.nacc = nacc;
  p.splits = splits;
  p.b_atom_bytes = b_atom;
  p.stage_bytes = stage_size(atoms);
  const size_t red_bytes = static_cast<size_t>(kTileN) * nacc * bn * 4;  // the partial tile of the split-K sum
  p.stages = static_cast<int>(std::min<size_t>(kMaxStages, avail / p.stage_bytes));
  while (p.stages < kMaxStages && static_cast<size_t>(p.stages) * p.stage_bytes < red_bytes) ++p.stages;
  if (p.stages < 2 || static_cast<size_t>(p.stages) * p.stage_bytes < red_bytes ||
      static_cast<size_t>(p.stages) * p.stage_bytes > avail)
    return cudaErrorInvalidConfiguration;
  p.a_col0 = static_cast<uint32_t>((nacc * bn + kASlotCols - 1) / kASlotCols * kASlotCols);
  p.a_slots = static_cast<int>(std::min<uint32_t>(kMaxASlots, (kTmemCols - p.a_col0) / kASlotCols));
  if (p.a_slots < 2) return cudaErrorInvalidConfiguration;
  p.idesc = idesc_bf16_m128(bn);
  // All of the SM's shared memory, whatever the stages use: one CTA per SM,
  // so no two CTAs ever wait for each other's tensor memory (each allocates
  // all 512 columns; two clusters interleaved on the same SMs could deadlock).
  L.smem = dev.smem_optin;
  if (static_cast<size_t>(p.stages) * p.stage_bytes + kBarrierBytes + 1024 > L.smem) return cudaErrorInvalidConfiguration;
  L.grid = dim3(static_cast<unsigned>(splits), static_cast<unsigned>(n_tiles), static_cast<unsigned>(m_tiles));
  L.atoms = atoms;
  return cudaSuccess;
}

cudaError_t launch_planned_tc(const TcLaunch& L, cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = L.grid;
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = L.smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = L.grid.x;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  count_launch();
  const bool epi = L.p.epi != kEpiNone || L.p.nacc == 2;
  if (epi)
    return L.atoms == 2 ? cudaLaunchKernelEx(&cfg, tc_kernel<2, true>, L.tmap_x, L.tmap_codes, L.tmap_up, L.p)
                        : cudaLaunchKernelEx(&cfg, tc_kernel<1, true>, L.tmap_x, L.tmap_codes, L.tmap_up, L.p);
  return L.atoms == 2 ? cudaLaunchKernelEx(&cfg, tc_kernel<2, false>, L.tmap_x, L.tmap_codes, L.tmap_up, L.p)
                      : cudaLaunchKernelEx(&cfg, tc_kernel<1, false>, L.tmap_x, L.tmap_codes, L.tmap_up, L.p);
}

}  // namespace q4
