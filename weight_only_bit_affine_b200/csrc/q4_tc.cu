// q4_tc.cu -- tensor-core path of the affine Q4 group-32 matmul for many
// activation rows (prefill, concurrent conversations: M >= 16).
//
//   y[m,n] = sum_k x[m,k] * w_hat[n,k],   w_hat = s*q + b  (group 32 along k)
//
// The packed weights are dequantized tile by tile into shared memory (never
// to HBM) and multiplied on the 5th-generation tensor cores (tcgen05.mma,
// kind::f16, bf16 x bf16 -> fp32 accumulation in tensor memory).  The Swift
// blog's prefill batching (voice prompt and prefill as one batched forward)
// and the four concurrent conversations of "A smaller voice model" are the
// workloads with several rows.
//
// Tile: 128 weight rows (the MMA's M side: D[n, m] = w_hat . x^T, so the
// output tile is y^T) x BN activation rows (the MMA's N side, 16..256) x a
// K range; K advances in chunks of 64 (one 128-byte swizzle span of bf16).
// Per CTA (320 threads):
//   warp 0      TMA producer: x tile (tensor map, 128-byte swizzle) and the
//               4 KB code tile (tensor map, 32-byte rows) per chunk;
//   warp 1      allocates tensor memory; one thread issues 4 MMAs per chunk
//               and commits them to the stage's "free" barrier;
//   warps 2..9  dequantize: thread t owns group (t / 128) of weight row
//               (t % 128) in every chunk: bf16 "128 + q" by PRMT + LOP3, exact
//               q by a packed subtract, w_hat = fma.rn.bf16x2(q, s, b) (one
//               rounding), stored in the canonical K-major SWIZZLE_128B layout
//               the MMA descriptor reads; then the epilogue (tensor memory ->
//               registers -> bf16 y).
// Split-K: when there are too few tiles to fill the GPU, the K range is split
// across the CTAs of a thread-block cluster, and the fp32 partial tiles are
// summed through distributed shared memory (no global workspace).
// Every wait is bounded (q4_device.cuh); programmatic dependent launch as in
// the GEMV family.
#include "q4_device.cuh"
#include "q4_internal.h"

#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>

#ifndef Q4_TC_WAIT_SLEEP
#define Q4_TC_WAIT_SLEEP 0
#endif

namespace q4 {
namespace {

constexpr int kTileN = 128;        // weight rows per tile (MMA M)
constexpr int kChunkK = 64;        // K per pipeline stage (one 128-byte bf16 swizzle span)
constexpr int kSuperK = 256;       // K per scale/bias load (8 groups = 16 bytes per row)
constexpr int kDequantWarps = 8;
constexpr int kThreads = 64 + 32 * kDequantWarps;
constexpr int kATileBytes = kTileN * kChunkK * 2;   // 16 KB
constexpr int kCodeTileBytes = kTileN * kChunkK / 2;  // 4 KB

struct TcParams {
  const uint16_t* scales;  // [N, K/32]
  const uint16_t* biases;
  uint16_t* y;             // [M, N]
  const uint16_t* r;       // epilogue operand [M, N] (kEpiResidual / kEpiSiluMul), else NULL
  int64_t M, N;
  int K;
  int epi;                 // output epilogue (q4_device.cuh)
  int bn;          // activation rows per tile (multiple of 16, <= 256)
  int splits;      // CTAs per cluster along K
  int stages;
  uint32_t stage_bytes, b_tile_bytes;
  uint32_t tmem_cols;
  uint32_t idesc;  // tcgen05 instruction descriptor
};

// ---- tcgen05 / TMA wrappers ------------------------------------------------

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int c0, int c1, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
      ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// K-major operand tile with the 128-byte swizzle: rows of 128 bytes, 8-row
// groups 1024 bytes apart (stride byte offset), tile base 1024-byte aligned.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t smem_addr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((smem_addr & 0x3FFFFu) >> 4);  // start address
  d |= static_cast<uint64_t>(16u >> 4) << 16;                // leading byte offset (unused here)
  d |= static_cast<uint64_t>(1024u >> 4) << 32;              // stride byte offset
  d |= static_cast<uint64_t>(1) << 46;                       // descriptor version
  d |= static_cast<uint64_t>(2) << 61;                       // 128-byte swizzle
  return d;
}

__device__ __forceinline__ void tc_mma_f16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                           uint32_t accumulate) {
  asm volatile(
      "{ .reg .pred p; setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p; }"
      ::"r"(tmem_d), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void tc_ld_x8(uint32_t taddr, float (&v)[8]) {
  uint32_t r[8];
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
               : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[i]);
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

// ---- the kernel ------------------------------------------------------------
//
// A pipeline stage covers ATOMS x 64 inputs k (one or two 128-byte swizzle
// spans): fewer, larger stages cut the fixed per-stage cost of every role
// (barrier waits, TMA issue, MMA issue and commit) when shared memory allows
// at least three of them.

// Output store; the EPI = false instantiation (no epilogue in the launch)
// keeps the epilogue's code out of the kernel.
template <bool EPI>
__device__ __forceinline__ uint16_t store_tc(float v, const TcParams& p, int64_t idx) {
  if constexpr (EPI) return epilogue_bf16(v, p.epi, p.r, idx);
  return float_to_bf16_bits(v);
}

template <int ATOMS, bool EPI>
__global__ void __launch_bounds__(kThreads, 1)
    tc_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_codes,
              const __grid_constant__ TcParams p) {
  constexpr int kStageK = kChunkK * ATOMS;
  constexpr int kStagesPerSuper = kSuperK / kStageK;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // 1024-byte alignment for the swizzled operand tiles.
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  uint64_t* tma_full = reinterpret_cast<uint64_t*>(smem + static_cast<size_t>(p.stages) * p.stage_bytes);
  uint64_t* a_full = tma_full + p.stages;
  uint64_t* stage_free = a_full + p.stages;
  uint64_t* accum_full = stage_free + p.stages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accum_full + 1);

  const int split = static_cast<int>(blockIdx.x);  // == cluster rank along x
  const int64_t n0 = static_cast<int64_t>(blockIdx.y) * kTileN;
  const int64_t m0 = static_cast<int64_t>(blockIdx.z) * p.bn;
  const int supers = p.K / kSuperK;
  const int sc_begin = split * supers / p.splits, sc_end = (split + 1) * supers / p.splits;
  const int stage_begin = sc_begin * kStagesPerSuper;
  const int nstages = (sc_end - sc_begin) * kStagesPerSuper;

  if (tid == 0) {
    for (int s = 0; s < p.stages; ++s) {
      mbar_init(&tma_full[s], 1);
      mbar_init(&a_full[s], kDequantWarps);
      mbar_init(&stage_free[s], 1);
    }
    mbar_init(accum_full, 1);
    fence_mbar_init();
  }
  if (warp == 1) {  // tensor memory for the fp32 accumulator tile: 128 lanes x bn columns
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(p.tmem_cols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_launch_dependents();
  pdl_wait_predecessors();

  // Stage layout: ATOMS A tiles (128 rows x 128 B each, 16 KB apart), then
  // ATOMS x tiles (bn rows x 128 B each), then the code tile (128 rows x
  // 32*ATOMS bytes).
  const uint32_t b_atom = static_cast<uint32_t>(p.bn) * 128u;
  auto a_tile = [&](int s) { return smem + static_cast<size_t>(s) * p.stage_bytes; };
  auto b_tile = [&](int s) { return a_tile(s) + ATOMS * kATileBytes; };
  auto c_tile = [&](int s) { return b_tile(s) + ATOMS * b_atom; };

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      bool dead = false;
      int s = 0;
      uint32_t ph = 0;
      for (int c = 0; c < nstages; ++c) {
        if (!dead && !mbar_wait<Q4_TC_WAIT_SLEEP>(&stage_free[s], ph ^ 1u)) dead = true;
        const int k0 = (stage_begin + c) * kStageK;
        mbar_arrive_expect_tx(&tma_full[s], ATOMS * b_atom + kTileN * kStageK / 2);
#pragma unroll
        for (int at = 0; at < ATOMS; ++at)
          tma_load_2d(b_tile(s) + at * b_atom, &tmap_x, k0 + at * kChunkK, static_cast<int>(m0), &tma_full[s]);
        tma_load_2d(c_tile(s), &tmap_codes, k0 / 2, static_cast<int>(n0), &tma_full[s]);
        if (++s == p.stages) { s = 0; ph ^= 1u; }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    // Waits only for the dequantizing warps: they arrive after having waited
    // for this stage's TMA themselves, so the x tile is in place too.
    if (lane == 0) {
      bool dead = false;
      int s = 0;
      uint32_t ph = 0;
      for (int c = 0; c < nstages; ++c) {
        if (!dead && !mbar_wait<Q4_TC_WAIT_SLEEP>(&a_full[s], ph)) dead = true;
        tc_fence_after();
        const uint64_t ad = sw128_desc(smem_u32(a_tile(s)));
        const uint64_t bd = sw128_desc(smem_u32(b_tile(s)));
#pragma unroll
        for (int at = 0; at < ATOMS; ++at)
#pragma unroll
          for (int kk = 0; kk < kChunkK / 16; ++kk)  // 16 bf16 = 32 bytes per MMA step
            tc_mma_f16(tmem_base, ad + at * (kATileBytes >> 4) + 2 * kk, bd + at * (b_atom >> 4) + 2 * kk, p.idesc,
                       (c > 0 || at > 0 || kk > 0) ? 1u : 0u);
        tc_commit(&stage_free[s]);
        if (++s == p.stages) { s = 0; ph ^= 1u; }
      }
      tc_commit(accum_full);
    }
  } else {
    // ---------------- dequantize, then epilogue ----------------
    const int t = tid - 64;
    const int row = t & (kTileN - 1);  // weight row within the tile
    const int half = t >> 7;           // which group of each 64-wide atom
    const int64_t grow = n0 + row;
    const bool row_ok = grow < p.N;
    const int G = p.K / 32;
    // Scales and biases of this row, 8 groups (one super-chunk) per 16-byte load,
    // fetched one super-chunk ahead.
    uint4 s_cur = make_uint4(0, 0, 0, 0), b_cur = s_cur, s_nxt = s_cur, b_nxt = s_cur;
    auto load_sb = [&](int sc, uint4& sv, uint4& bv) {
      if (row_ok && sc < sc_end) {
        const int64_t off = grow * G + static_cast<int64_t>(sc) * (kSuperK / 32);
        sv = *reinterpret_cast<const uint4*>(p.scales + off);
        bv = *reinterpret_cast<const uint4*>(p.biases + off);
      } else {
        sv = make_uint4(0, 0, 0, 0);
        bv = sv;
      }
    };
    load_sb(sc_begin, s_cur, b_cur);
    load_sb(sc_begin + 1, s_nxt, b_nxt);
    bool dead = false;
    int s = 0, sub = 0, sc_next = sc_begin + 2;
    uint32_t ph = 0;
    for (int c = 0; c < nstages; ++c) {
      if (c > 0 && sub == 0) {
        s_cur = s_nxt;
        b_cur = b_nxt;
        load_sb(sc_next++, s_nxt, b_nxt);
      }
      if (!dead && !mbar_wait<Q4_TC_WAIT_SLEEP>(&stage_free[s], ph ^ 1u)) dead = true;  // A buffer no longer read
      if (!dead && !mbar_wait<Q4_TC_WAIT_SLEEP>(&tma_full[s], ph)) dead = true;         // codes arrived
      const uint8_t* crow = c_tile(s) + row * (32 * ATOMS);
#pragma unroll
      for (int at = 0; at < ATOMS; ++at) {
        // group (2*(sub*ATOMS + at) + half) of the current super-chunk
        const int gi = 2 * (sub * ATOMS + at) + half;
        const uint32_t sw = (gi < 2) ? s_cur.x : (gi < 4) ? s_cur.y : (gi < 6) ? s_cur.z : s_cur.w;
        const uint32_t bw = (gi < 2) ? b_cur.x : (gi < 4) ? b_cur.y : (gi < 6) ? b_cur.z : b_cur.w;
        const uint32_t sel = (gi & 1) ? 0x3232u : 0x1010u;  // broadcast one bf16 to both halves
        const uint32_t s2 = __byte_perm(sw, 0, sel);
        const uint32_t b2 = __byte_perm(bw, 0, sel);
        const uint4 cw = *reinterpret_cast<const uint4*>(crow + at * 32 + half * 16);
        const uint32_t words[4] = {cw.x, cw.y, cw.z, cw.w};
        uint8_t* arow = a_tile(s) + at * kATileBytes + row * 128;
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          const uint32_t wd = words[w], w4 = wd >> 4;
          uint32_t o[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            // bytes: [wd.byte_i, -, w4.byte_i, -] -> nibbles q[2i] at bits 0..3, q[2i+1] at 16..19
            const uint32_t pr = __byte_perm(wd, w4, (i) | (i << 4) | ((4 + i) << 8) | ((4 + i) << 12));
            const uint32_t v = (pr & 0x000F000Fu) | 0x43004300u;  // (128 + q, 128 + q') exactly
            const uint32_t q = bf16x2_sub(v, 0x43004300u);          // (q, q') exactly
            o[i] = bf16x2_fma(q, s2, b2);                           // bf16(s*q + b), one rounding
          }
          const int chunk16 = 4 * half + w;  // 16-byte chunk (8 k) within the 128-byte row
          *reinterpret_cast<uint4*>(arow + ((chunk16 ^ (row & 7)) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
        }
      }
      fence_proxy_async_smem();  // make the generic stores visible to the tensor core
      __syncwarp();
      if (lane == 0) mbar_arrive(&a_full[s]);
      if (++s == p.stages) { s = 0; ph ^= 1u; }
      if (++sub == kStagesPerSuper) sub = 0;
    }

    // ---- epilogue: tensor memory -> y (or partial sums for the cluster) ----
    if (!dead && !mbar_wait(accum_full, 0)) dead = true;
    tc_fence_after();
    const int lane_base = 32 * (warp & 3);
    const int trow = lane_base + lane;  // tile row held by this thread
    const int col_half = (warp - 2) >> 2;
    const int cols = p.bn / 2;
    const uint32_t taddr = tmem_base + (static_cast<uint32_t>(lane_base) << 16) + col_half * cols;
    float* red = reinterpret_cast<float*>(smem);  // reuses the stage area (all MMAs are done)
    const int red_ld = p.bn + 4;                  // 16-byte rows; row r and r + 1 four banks apart
    for (int c0 = 0; c0 < cols; c0 += 8) {
      float v[8];
      tc_ld_x8(taddr + c0, v);
      if (p.splits == 1) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int64_t m = m0 + col_half * cols + c0 + i;
          if (n0 + trow < p.N && m < p.M) p.y[m * p.N + n0 + trow] = store_tc<EPI>(v[i], p, m * p.N + n0 + trow);
        }
      } else {
        float4* dst = reinterpret_cast<float4*>(red + trow * red_ld + col_half * cols + c0);
        dst[0] = make_float4(v[0], v[1], v[2], v[3]);
        dst[1] = make_float4(v[4], v[5], v[6], v[7]);
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
      // Column slice of this CTA, in float4 units (bn and the slice are multiples of 4).
      const int q_beg = split * (p.bn / 4) / p.splits, q_end = (split + 1) * (p.bn / 4) / p.splits;
      const uint32_t row_addr = smem_u32(smem) + static_cast<uint32_t>(trow * (p.bn + 4)) * 4u;
      uint32_t peer[8];
#pragma unroll
      for (int r = 0; r < 8; ++r) peer[r] = dsmem_map(row_addr, static_cast<uint32_t>(r < p.splits ? r : 0));
      for (int q = q_beg + (t >> 7); q < q_end; q += 2) {
        // all peers' loads first, then the sums
        float4 v[8];
#pragma unroll
        for (int r = 0; r < 8; ++r)
          if (r < p.splits) v[r] = ld_dsmem_v4(peer[r] + static_cast<uint32_t>(q) * 16u);
        float4 acc = v[0];
#pragma unroll
        for (int r = 1; r < 8; ++r)
          if (r < p.splits) {
            acc.x += v[r].x;
            acc.y += v[r].y;
            acc.z += v[r].z;
            acc.w += v[r].w;
          }
        const float out[4] = {acc.x, acc.y, acc.z, acc.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int64_t m = m0 + 4 * q + i;
          if (n0 + trow < p.N && m < p.M) p.y[m * p.N + n0 + trow] = store_tc<EPI>(out[i], p, m * p.N + n0 + trow);
        }
      }
    }
    cluster_sync_all();  // no CTA leaves while a peer may still read its shared memory
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(p.tmem_cols)
                 : "memory");
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

uint32_t make_idesc(int bn) {
  uint32_t d = 0;
  d |= 1u << 4;                                  // D: fp32
  d |= 1u << 7;                                  // A: bf16
  d |= 1u << 10;                                 // B: bf16
  d |= static_cast<uint32_t>(bn >> 3) << 17;     // N
  d |= static_cast<uint32_t>(kTileN >> 4) << 24;  // M
  return d;                                      // both operands K-major, no negation
}

}  // namespace

cudaError_t tc_device_flags(unsigned int* flags, bool clear) { return tu_device_flags(flags, clear); }

bool tc_supported(const MatmulArgs& a) {
  if (a.fused()) return false;  // one-pass SwiGLU is a GEMV-family problem
  if (a.K % kSuperK != 0) return false;
  if ((reinterpret_cast<uintptr_t>(a.scales) | reinterpret_cast<uintptr_t>(a.biases)) & 15u) return false;
  if (a.N > (int64_t(1) << 31) - kTileN || a.M > (int64_t(1) << 31) - 256) return false;
  return encode_fn() != nullptr;
}

cudaError_t launch_tc(const MatmulArgs& a, cudaStream_t stream, const DeviceInfo& dev) {
  PFN_cuTensorMapEncodeTiled_v12000 encode = encode_fn();
  if (!encode) return cudaErrorNotSupported;
  const int bn = static_cast<int>(std::min<int64_t>(256, (a.M + 15) / 16 * 16));
  const int64_t n_tiles = (a.N + kTileN - 1) / kTileN;
  const int64_t m_tiles = (a.M + bn - 1) / bn;
  const int supers = static_cast<int>(a.K / kSuperK);
  // Split K over a cluster when the tiles alone would leave SMs idle.
  int splits = 1;
  const int64_t tiles = n_tiles * m_tiles;
  while (splits < 8 && splits * 2 <= supers && tiles * splits * 2 <= dev.sm_count) splits *= 2;
  if (splits < 8 && tiles * splits < dev.sm_count) {
    const int want = static_cast<int>(std::min<int64_t>(8, (dev.sm_count + tiles - 1) / tiles));
    if (want > splits && want <= supers && tiles * want <= dev.sm_count * 1.05) splits = want;
  }

  // Two 64-wide atoms per stage when at least three such stages fit.
  const uint32_t b_atom = static_cast<uint32_t>(bn) * kChunkK * 2;
  auto stage_size = [&](int atoms) {
    return (static_cast<uint32_t>(atoms) * (kATileBytes + b_atom + kCodeTileBytes) + 1023u) & ~1023u;
  };
  const size_t barrier_bytes = 8 * (3 * 12 + 1) + 16;
  const size_t avail = dev.smem_optin - 1024 - barrier_bytes;
  const int atoms = (avail / stage_size(2) >= 3) ? 2 : 1;

  CUtensorMap tmap_x, tmap_codes;
  {
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(a.K), static_cast<cuuint64_t>(a.M)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(a.K) * 2};
    cuuint32_t box[2] = {static_cast<cuuint32_t>(kChunkK), static_cast<cuuint32_t>(bn)};
    cuuint32_t estr[2] = {1, 1};
    if (encode(&tmap_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(a.x), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  {
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(a.K / 2), static_cast<cuuint64_t>(a.N)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(a.K / 2)};
    cuuint32_t box[2] = {static_cast<cuuint32_t>(kChunkK / 2 * atoms), static_cast<cuuint32_t>(kTileN)};
    cuuint32_t estr[2] = {1, 1};
    if (encode(&tmap_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(a.codes), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }

  TcParams p;
  p.scales = a.scales;
  p.biases = a.biases;
  p.y = a.y;
  p.r = a.r;
  p.epi = a.epi;
  p.M = a.M;
  p.N = a.N;
  p.K = static_cast<int>(a.K);
  p.bn = bn;
  p.splits = splits;
  p.b_tile_bytes = b_atom;
  p.stage_bytes = stage_size(atoms);
  const size_t red_bytes = static_cast<size_t>(kTileN) * (bn + 4) * 4;
  p.stages = static_cast<int>(std::min<size_t>(12, avail / p.stage_bytes));
  while (p.stages > 2 && static_cast<size_t>(p.stages) * p.stage_bytes < red_bytes) ++p.stages;
  if (p.stages < 2 || static_cast<size_t>(p.stages) * p.stage_bytes < red_bytes ||
      static_cast<size_t>(p.stages) * p.stage_bytes > avail)
    return cudaErrorInvalidConfiguration;
  uint32_t cols = 32;
  while (cols < static_cast<uint32_t>(bn)) cols <<= 1;
  p.tmem_cols = cols;
  p.idesc = make_idesc(bn);
  const size_t smem = static_cast<size_t>(p.stages) * p.stage_bytes + barrier_bytes + 1024;

  static PerDeviceOnce attr_once;
  if (attr_once.needed(dev.device)) {
    for (auto kern : {tc_kernel<1, false>, tc_kernel<2, false>, tc_kernel<1, true>, tc_kernel<2, true>}) {
      cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           static_cast<int>(dev.smem_optin));
      if (e == cudaSuccess) e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 0);
      if (e != cudaSuccess) return e;
    }
    attr_once.mark(dev.device);
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(splits), static_cast<unsigned>(n_tiles), static_cast<unsigned>(m_tiles));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = static_cast<unsigned>(splits);
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  count_launch();
  if (p.epi != kEpiNone)
    return atoms == 2 ? cudaLaunchKernelEx(&cfg, tc_kernel<2, true>, tmap_x, tmap_codes, p)
                      : cudaLaunchKernelEx(&cfg, tc_kernel<1, true>, tmap_x, tmap_codes, p);
  return atoms == 2 ? cudaLaunchKernelEx(&cfg, tc_kernel<2, false>, tmap_x, tmap_codes, p)
                    : cudaLaunchKernelEx(&cfg, tc_kernel<1, false>, tmap_x, tmap_codes, p);
}

}  // namespace q4
