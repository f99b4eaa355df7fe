// Persistent tcgen05 GEMM for sm_100a with fused epilogues.
//
//   C[M, N] = A[M, K] . B[N, K]^T,  A and B bf16 row-major (K contiguous), fp32 TMEM
//   accumulator, 128 x 256 output tile per CTA, 64-deep K slices.
//
// Warp roles (192 threads, one CTA per SM):
//   warp 0  lane 0 : TMA producer, 4-stage smem ring (A 16 KB + B 32 KB per stage)
//   warp 1  lane 0 : tcgen05.mma issuer; warp 1 also owns the TMEM allocation
//   warps 2-5      : epilogue; TMEM lane group (warp % 4) -> 32 output rows each
// The accumulator is double-buffered in TMEM (2 x 256 columns) so the epilogue of
// tile i overlaps the main loop of tile i + 1.
//
// Epilogues (the DiT block's projection steps, "Z-Image-Turbo port" DiT row and
// "Native creative jobs", "Recipes and precision": FP32 accumulators, SwiGLU gate in
// FP32, bf16 storage, never fp16):
//   EPI_F32    fp32 store (+ bias)                 embedders, final layer
//   EPI_BF16   bf16 store (+ bias)                 out-proj, w2 (y, normalized in FP32
//                                                  by the residual kernel)
//   EPI_QKV    q/k columns: real interleaved RoPE with per-token cos/sin, 32-column
//              chunks; bf16 store of [q | k | v]
//   EPI_QKV_NORM  same with a per-head RMSNorm of q and k first (whole head at once)
//   EPI_SWIGLU gate/up column blocks -> silu(gate) * up, bf16 store
#include <cudaTypedefs.h>

#include <cstdio>
#include <cstdlib>
#include <mutex>

#include "internal.h"
#include "ptx.cuh"

#ifndef ZDIT_L2_BAND_MB
#define ZDIT_L2_BAND_MB 32
#endif

namespace zdit {

namespace {

constexpr int BM = 128, BN = 256, BK = 64, STAGES = 4;
constexpr int A_TILE = BM * BK * 2;  // 16 KB
constexpr int B_TILE = BN * BK * 2;  // 32 KB
constexpr int STAGE_BYTES = A_TILE + B_TILE;
constexpr int THREADS = 192;
constexpr int TMEM_COLS = 2 * BN;
constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + 256;

struct KParams {
  int M, N, K, ldo;
  void* out;
  const float* bias;
  const float* rcos;
  const float* rsin;
  const float* qn;
  const float* kn;
  float eps;
  int dim;
  int num_m, num_n, num_k, group_m, group_n, raster;
  int* err;
  int* band_flags;  // per 128-row band arrival counters or nullptr
};

// Tile order of the persistent loop.  raster 0: bands of group_m M-tiles, M fastest
// inside a band (the band of A stays in L2 while B streams); raster 1: bands of
// group_n N-tiles, N fastest inside a band (the band of B stays in L2 while A
// streams).  The host sizes the band to a fraction of L2 and picks the order with
// less estimated HBM traffic.
__device__ __forceinline__ void tile_coords(int t, const KParams& p, int& mb, int& nb) {
  if (p.raster == 1) {
    const int group = p.group_n * p.num_m;
    const int g = t / group;
    const int first = g * p.group_n;
    const int gn = min(p.num_n - first, p.group_n);
    const int r = t - g * group;
    nb = first + r % gn;
    mb = r / gn;
    return;
  }
  const int group = p.group_m * p.num_n;
  const int g = t / group;
  const int first = g * p.group_m;
  const int gm = min(p.num_m - first, p.group_m);
  const int r = t - g * group;
  mb = first + r % gm;
  nb = r / gm;
}

__device__ __forceinline__ float silu_f(float g) { return g / (1.0f + __expf(-g)); }

template <int EPI>
__device__ __forceinline__ void epilogue_tile(const KParams& p, uint32_t taddr, int row, int nb) {
  const bool row_ok = row < p.M;
  if constexpr (EPI == EPI_F32 || EPI == EPI_BF16) {
#pragma unroll 1
    for (int c = 0; c < BN / 32; ++c) {
      const int col0 = nb * BN + c * 32;
      if (col0 >= p.N) break;  // warp-uniform
      uint32_t r[32];
      __syncwarp();  // tcgen05.ld is warp-collective: reconverge after the row-masked stores
      tmem_ld32(taddr + c * 32, r);
      tmem_ld_wait();
      float v[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
      if (p.bias != nullptr) {
#pragma unroll
        for (int j = 0; j < 32; j += 4) {
          const float4 b = *reinterpret_cast<const float4*>(p.bias + col0 + j);
          v[j] += b.x; v[j + 1] += b.y; v[j + 2] += b.z; v[j + 3] += b.w;
        }
      }
      if (row_ok) {
        if constexpr (EPI == EPI_F32) {
          float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.out) + (size_t)row * p.ldo + col0);
#pragma unroll
          for (int j = 0; j < 8; ++j) dst[j] = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
        } else {
          uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) + (size_t)row * p.ldo + col0);
#pragma unroll
          for (int j = 0; j < 4; ++j)
            dst[j] = make_uint4(pack_bf16x2(v[8 * j], v[8 * j + 1]), pack_bf16x2(v[8 * j + 2], v[8 * j + 3]),
                                pack_bf16x2(v[8 * j + 4], v[8 * j + 5]), pack_bf16x2(v[8 * j + 6], v[8 * j + 7]));
        }
      }
    }
  } else if constexpr (EPI == EPI_SWIGLU) {
    // tile columns [0,128) hold gate rows 128*nb.., [128,256) the matching up rows
#pragma unroll 1
    for (int c = 0; c < 4; ++c) {
      uint32_t g[32], u[32];
      __syncwarp();
      tmem_ld32(taddr + c * 32, g);
      tmem_ld32(taddr + 128 + c * 32, u);
      tmem_ld_wait();
      if (row_ok) {
        uint32_t h[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const float h0 = silu_f(__uint_as_float(g[2 * j])) * __uint_as_float(u[2 * j]);
          const float h1 = silu_f(__uint_as_float(g[2 * j + 1])) * __uint_as_float(u[2 * j + 1]);
          h[j] = pack_bf16x2(h0, h1);
        }
        uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) + (size_t)row * p.ldo +
                                              nb * 128 + c * 32);
#pragma unroll
        for (int j = 0; j < 4; ++j) dst[j] = make_uint4(h[4 * j], h[4 * j + 1], h[4 * j + 2], h[4 * j + 3]);
      }
    }
  } else if constexpr (EPI == EPI_QKV) {
    {
      // RoPE pairs never cross a 32-column chunk, so work chunk by chunk
      // (cos/sin of the 16 pairs of the chunk) and keep register use low.
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        const int col0 = nb * BN + c * 32;
        uint32_t r[32];
        __syncwarp();
        tmem_ld32(taddr + c * 32, r);
        tmem_ld_wait();
        if (!row_ok) continue;
        float v[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
        if (col0 < 2 * p.dim) {  // q or k columns: rotate
          const int pair0 = (col0 & 127) >> 1;  // first pair index of the chunk inside its head
          const float4* cs = reinterpret_cast<const float4*>(p.rcos + (size_t)row * 64 + pair0);
          const float4* sn = reinterpret_cast<const float4*>(p.rsin + (size_t)row * 64 + pair0);
#pragma unroll
          for (int i4 = 0; i4 < 4; ++i4) {
            const float4 c4 = cs[i4], s4 = sn[i4];
            const float cc[4] = {c4.x, c4.y, c4.z, c4.w};
            const float ss[4] = {s4.x, s4.y, s4.z, s4.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int i = i4 * 4 + e;
              const float x0 = v[2 * i], x1 = v[2 * i + 1];
              v[2 * i] = x0 * cc[e] - x1 * ss[e];
              v[2 * i + 1] = x0 * ss[e] + x1 * cc[e];
            }
          }
        }
        uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) + (size_t)row * p.ldo + col0);
#pragma unroll
        for (int j = 0; j < 4; ++j)
          dst[j] = make_uint4(pack_bf16x2(v[8 * j], v[8 * j + 1]), pack_bf16x2(v[8 * j + 2], v[8 * j + 3]),
                              pack_bf16x2(v[8 * j + 4], v[8 * j + 5]), pack_bf16x2(v[8 * j + 6], v[8 * j + 7]));
      }
    }
  } else if constexpr (EPI == EPI_QKV_NORM) {
#pragma unroll 1
    for (int hh = 0; hh < BN / 128; ++hh) {
      const int colh = nb * BN + hh * 128;
      float v[128];
      __syncwarp();
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t r[32];
        tmem_ld32(taddr + hh * 128 + c * 32, r);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 32; ++j) v[c * 32 + j] = __uint_as_float(r[j]);
      }
      if (!row_ok) continue;
      const bool is_q = colh < p.dim;
      const bool is_k = !is_q && colh < 2 * p.dim;
      if (is_q || is_k) {
        const float* nw = is_q ? p.qn : p.kn;
        if (nw != nullptr) {
          float ss = 0.f;
#pragma unroll
          for (int j = 0; j < 128; ++j) ss += v[j] * v[j];
          const float rinv = 1.0f / sqrtf(ss * (1.0f / 128.0f) + p.eps);
#pragma unroll
          for (int j = 0; j < 128; ++j) v[j] = v[j] * rinv * nw[j];
        }
        const float4* cs = reinterpret_cast<const float4*>(p.rcos + (size_t)row * 64);
        const float4* sn = reinterpret_cast<const float4*>(p.rsin + (size_t)row * 64);
#pragma unroll
        for (int i4 = 0; i4 < 16; ++i4) {
          const float4 c4 = cs[i4], s4 = sn[i4];
          const float cc[4] = {c4.x, c4.y, c4.z, c4.w};
          const float ssn[4] = {s4.x, s4.y, s4.z, s4.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int i = i4 * 4 + e;
            const float x0 = v[2 * i], x1 = v[2 * i + 1];
            v[2 * i] = x0 * cc[e] - x1 * ssn[e];
            v[2 * i + 1] = x0 * ssn[e] + x1 * cc[e];
          }
        }
      }
      uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) + (size_t)row * p.ldo + colh);
#pragma unroll
      for (int j = 0; j < 16; ++j)
        dst[j] = make_uint4(pack_bf16x2(v[8 * j], v[8 * j + 1]), pack_bf16x2(v[8 * j + 2], v[8 * j + 3]),
                            pack_bf16x2(v[8 * j + 4], v[8 * j + 5]), pack_bf16x2(v[8 * j + 6], v[8 * j + 7]));
    }
  }
}

template <int EPI>
__global__ void __launch_bounds__(THREADS, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const KParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* done = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], 4);
    }
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) tmem_alloc(tmem_slot, TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int num_tiles = p.num_m * p.num_n;
  griddep_wait();     // the predecessor's output (this GEMM's A operand) is complete
  griddep_trigger();  // every CTA has started: the successor may launch and set itself up

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------ TMA producer
    int stage = 0;
    uint32_t phase = 0;
    uint32_t armed = 0;  // bit s: stage s has an armed phase; parity in armed_par
    uint32_t armed_par = 0;
    for (int t = blockIdx.x; t < num_tiles && !*abort_flag; t += gridDim.x) {
      int mb, nb;
      tile_coords(t, p, mb, nb);
      for (int kb = 0; kb < p.num_k; ++kb) {
        if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag, p.err)) break;
        uint8_t* sa = smem + stage * STAGE_BYTES;
        mbar_arrive_expect_tx(&full[stage], STAGE_BYTES);
        tma_load_2d(sa, &tmA, &full[stage], kb * BK, mb * BM);
        tma_load_2d(sa + A_TILE, &tmB, &full[stage], kb * BK, nb * BN);
        armed |= 1u << stage;
        armed_par = (armed_par & ~(1u << stage)) | (phase << stage);
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1;
        }
      }
    }
    if (*abort_flag) {
      // let copies already in flight land before the CTA's shared memory is released
      int dummy = 0;
      for (int s = 0; s < STAGES; ++s)
        if (armed & (1u << s)) mbar_wait(&full[s], (armed_par >> s) & 1u, &dummy);
    }
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------------------ MMA issuer
    const uint32_t idesc = idesc_bf16_f32(BM, BN);
    int stage = 0;
    uint32_t phase = 0;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int t = blockIdx.x; t < num_tiles && !*abort_flag; t += gridDim.x) {
      if (!mbar_wait(&tempty[acc], acc_phase ^ 1, abort_flag, p.err)) break;
      tc_fence_after();
      const uint32_t d = tmem_base + acc * BN;
      bool ok = true;
      for (int kb = 0; kb < p.num_k; ++kb) {
        if (!mbar_wait(&full[stage], phase, abort_flag, p.err)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t a0 = smem_u32(smem + stage * STAGE_BYTES);
        const uint32_t b0 = a0 + A_TILE;
#pragma unroll
        for (int k = 0; k < BK / 16; ++k)
          umma_bf16_ss(d, sdesc_kmajor_sw128(a0 + k * 32), sdesc_kmajor_sw128(b0 + k * 32), idesc,
                       (kb | k) != 0 ? 1u : 0u);
        umma_commit(&empty[stage]);
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1;
        }
      }
      if (!ok) break;
      umma_commit(&tfull[acc]);
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1;
    }
    // all MMAs issued by this thread have finished once `done` fires
    umma_commit(done);
    int dummy = 0;
    mbar_wait(done, 0, &dummy);
  } else if (warp >= 2) {
    // ------------------------------------------------------------ epilogue
    const int lg = warp & 3;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int t = blockIdx.x; t < num_tiles; t += gridDim.x) {
      const bool ok = __all_sync(0xffffffffu, mbar_wait(&tfull[acc], acc_phase, abort_flag, p.err));
      if (!ok) break;
      tc_fence_after();
      int mb, nb;
      tile_coords(t, p, mb, nb);
      const uint32_t taddr = tmem_base + ((uint32_t)(lg * 32) << 16) + acc * BN;
      epilogue_tile<EPI>(p, taddr, mb * BM + lg * 32 + lane, nb);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1;
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

// ------------------------------------------------------------------------------
// CTA-pair variant (cta_group::2): a cluster of two CTAs computes a 256 x 256 tile.
// Each CTA TMA-loads its own 128 rows of A and its own 128 rows of B per k-slice and
// counts the bytes on the leader's barrier;
// the leader's single MMA thread issues M=256 x N=256 MMAs that read both CTAs'
// shared memory and write 128 rows x 256 columns into each CTA's TMEM; commits are
// multicast to both CTAs.  Each CTA runs the same epilogue on its 128 rows.  Per
// SM this halves the B traffic.  No TMA multicast is used.
// Ring: 192 KB either as 6 stages of 64-deep slices (32 KB) or as 3 stages of 128-deep
// slices (two 64-column swizzled halves per operand, 64 KB), which give the MMA thread 8
// UMMAs (1024 tensor clocks) per barrier wait instead of 4.  Measured per projection
// (ncu, one main block): the gate/up GEMM runs its tensor pipe 94% of the time with
// 128-deep slices against 89% with 64-deep ones; QKV and the out-projection (K = 3840)
// lose 3-4 points with them; so the SwiGLU projection takes 128 and the others 64.
template <int PBK>
struct PairRing {
  static constexpr int BKP = PBK;
  static constexpr int STAGES = PBK == 128 ? 3 : 6;
  static constexpr int A_TILE = 128 * PBK * 2;
  static constexpr int B_TILE = 128 * PBK * 2;
  static constexpr int STAGE_BYTES = A_TILE + B_TILE;
  static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + 256;
};
template <int EPI>
__host__ __device__ constexpr int pair_bk() { return EPI == EPI_SWIGLU ? 128 : 64; }

template <int EPI>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(THREADS, 1)
    gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const KParams p) {
  using Ring = PairRing<pair_bk<EPI>()>;
  constexpr int P_BK = Ring::BKP, P_STAGES = Ring::STAGES, P_A_TILE = Ring::A_TILE;
  constexpr int P_STAGE_BYTES = Ring::STAGE_BYTES;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + P_STAGES * P_STAGE_BYTES);
  uint64_t* empty = full + P_STAGES;
  uint64_t* tfull = empty + P_STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* done = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1;
  const int n_pairs = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < P_STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], 8);  // 4 epilogue warps in each CTA of the pair
    }
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) tmem_alloc_pair(tmem_slot, TMEM_COLS);
  tc_fence_before();
  cluster_sync();  // barriers of both CTAs initialised before any cross-CTA traffic
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int num_tiles = p.num_m * p.num_n;  // num_m counts 256-row pair tiles
  griddep_wait();     // the predecessor's output (this GEMM's A operand) is complete
  griddep_trigger();  // every CTA has started: the successor may launch and set itself up

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------ TMA producer (both CTAs)
    int stage = 0;
    uint32_t phase = 0;
    uint32_t armed = 0, armed_par = 0;
    for (int t = pair; t < num_tiles && !*abort_flag; t += n_pairs) {
      int mb, nb;
      tile_coords(t, p, mb, nb);
      const int m0 = mb * 256 + (int)rank * 128;
      const int n0 = nb * BN + (int)rank * 128;
      for (int kb = 0; kb < p.num_k; ++kb) {
        if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag, p.err)) break;
        uint8_t* sa = smem + stage * P_STAGE_BYTES;
        if (leader) mbar_arrive_expect_tx(&full[stage], 2 * P_STAGE_BYTES);
        const uint32_t bar = leader_smem_addr(&full[stage]);
#pragma unroll
        for (int h = 0; h < P_BK / 64; ++h) {
          tma_load_2d_pair(sa + h * 16384, &tmA, bar, kb * P_BK + h * 64, m0);
          tma_load_2d_pair(sa + P_A_TILE + h * 16384, &tmB, bar, kb * P_BK + h * 64, n0);
        }
        armed |= 1u << stage;
        armed_par = (armed_par & ~(1u << stage)) | (phase << stage);
        if (++stage == P_STAGES) {
          stage = 0;
          phase ^= 1;
        }
      }
    }
    if (*abort_flag && leader) {
      // the leader's full barriers also count the peer's bytes: drain both CTAs' copies
      int dummy = 0;
      for (int s = 0; s < P_STAGES; ++s)
        if (armed & (1u << s)) mbar_wait(&full[s], (armed_par >> s) & 1u, &dummy);
    }
  } else if (warp == 1 && lane == 0 && leader) {
    // ------------------------------------------------------------ MMA issuer (leader)
    const uint32_t idesc = idesc_bf16_f32(256, BN);
    int stage = 0;
    uint32_t phase = 0;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int t = pair; t < num_tiles && !*abort_flag; t += n_pairs) {
      if (!mbar_wait(&tempty[acc], acc_phase ^ 1, abort_flag, p.err)) break;
      tc_fence_after();
      const uint32_t d = tmem_base + acc * BN;
      bool ok = true;
      for (int kb = 0; kb < p.num_k; ++kb) {
        if (!mbar_wait(&full[stage], phase, abort_flag, p.err)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t a0 = smem_u32(smem + stage * P_STAGE_BYTES);
        const uint32_t b0 = a0 + P_A_TILE;
#pragma unroll
        for (int k = 0; k < P_BK / 16; ++k) {
          // K step k: (k / 4) 64-column swizzled halves of 16 KB + (k % 4) 32-byte slices
          const uint32_t off = (k >> 2) * 16384 + (k & 3) * 32;
          umma_pair_bf16_ss(d, sdesc_kmajor_sw128(a0 + off), sdesc_kmajor_sw128(b0 + off), idesc,
                            (kb | k) != 0 ? 1u : 0u);
        }
        umma_pair_commit_mc(&empty[stage], 0x3);
        if (++stage == P_STAGES) {
          stage = 0;
          phase ^= 1;
        }
      }
      if (!ok) break;
      umma_pair_commit_mc(&tfull[acc], 0x3);
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1;
    }
    umma_pair_commit(done);
    int dummy = 0;
    mbar_wait(done, 0, &dummy);
  } else if (warp >= 2) {
    // ------------------------------------------------------------ epilogue (both CTAs)
    const int lg = warp & 3;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int t = pair; t < num_tiles; t += n_pairs) {
      const bool ok = __all_sync(0xffffffffu, mbar_wait(&tfull[acc], acc_phase, abort_flag, p.err));
      if (!ok) break;
      tc_fence_after();
      int mb, nb;
      tile_coords(t, p, mb, nb);
      const uint32_t taddr = tmem_base + ((uint32_t)(lg * 32) << 16) + acc * BN;
      epilogue_tile<EPI>(p, taddr, mb * 256 + (int)rank * 128 + lg * 32 + lane, nb);
      if (p.band_flags != nullptr) {
        // this CTA's 128 rows of the tile are stored: one arrival on their band
        __threadfence();
        named_bar_sync(1, 128);
        if (warp == 2 && lane == 0) atomicAdd(p.band_flags + mb * 2 + (int)rank, 1);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (leader)
          mbar_arrive(&tempty[acc]);
        else
          mbar_arrive_cluster(&tempty[acc], 0);
      }
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1;
    }
  }
  tc_fence_before();
  cluster_sync();  // no CTA leaves while its pair may still touch its shared memory
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, TMEM_COLS);
  }
}

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

template <int EPI>
zdit_status launch_epi(const CUtensorMap& ta, const CUtensorMap& tb, const KParams& kp, int grid, bool pair,
                       cudaStream_t s) {
  // The shared-memory opt-in is a property of the current context: set on every launch
  // (cheap, and legal inside stream capture) so a second device, or a context created
  // again after a reset, never launches without it.
  if (pair) {
    if (cudaFuncSetAttribute(gemm_pair_kernel<EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             PairRing<pair_bk<EPI>()>::SMEM_BYTES) != cudaSuccess)
      return ZDIT_ERR_CUDA;
    launch_dependent(gemm_pair_kernel<EPI>, dim3(grid), dim3(THREADS), PairRing<pair_bk<EPI>()>::SMEM_BYTES, s, ta, tb,
                     kp);
  } else {
    if (cudaFuncSetAttribute(gemm_tc_kernel<EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES) !=
        cudaSuccess)
      return ZDIT_ERR_CUDA;
    launch_dependent(gemm_tc_kernel<EPI>, dim3(grid), dim3(THREADS), SMEM_BYTES, s, ta, tb, kp);
  }
  return cudaGetLastError() == cudaSuccess ? ZDIT_OK : ZDIT_ERR_CUDA;
}

}  // namespace

bool make_tmap_bf16_2d(CUtensorMap* m, const void* ptr, uint64_t rows, uint64_t cols, uint64_t ld_elems,
                       uint32_t box_rows, uint32_t box_cols) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {ld_elems * 2};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// ZDIT_GEMM_SINGLE_CTA=1 in the environment selects the single-CTA kernel for every
// shape (A/B comparisons of the two kernels).
bool force_single_cta() {
  static int v = -1;
  if (v < 0) {
    const char* e = getenv("ZDIT_GEMM_SINGLE_CTA");
    v = (e != nullptr && e[0] == '1') ? 1 : 0;
  }
  return v == 1;
}

bool gemm_uses_pair(int M, int N) { return M > 256 && N % BN == 0 && !force_single_cta(); }

zdit_status launch_gemm(const GemmArgs& a, cudaStream_t s) {
  if (a.M <= 0 || a.N <= 0 || a.K <= 0) return ZDIT_ERR_SHAPE;
  if (a.K % 8 || a.lda % 8 || a.ldb % 8 || a.N % 32) return ZDIT_ERR_SHAPE;
  if ((reinterpret_cast<uintptr_t>(a.A) | reinterpret_cast<uintptr_t>(a.B) |
       reinterpret_cast<uintptr_t>(a.out)) & 15)
    return ZDIT_ERR_ALIGNMENT;
  if (a.epi == EPI_SWIGLU && (a.N % BN)) return ZDIT_ERR_SHAPE;
  if (a.epi == EPI_QKV && (a.N != 3 * a.dim || a.dim % 128 || a.N % BN || !a.rope_cos || !a.rope_sin))
    return ZDIT_ERR_SHAPE;
  if ((a.epi == EPI_F32 || a.epi == EPI_BF16) && (a.ldo % 4)) return ZDIT_ERR_ALIGNMENT;
  // CTA pairs for every shape that fills several 256 x 256 tiles; the single-CTA
  // kernel for small or narrow problems (embedders, final layer, tiny blocks).
  const bool pair = a.M > 256 && a.N % BN == 0 && !force_single_cta();
  CUtensorMap ta, tb;
  if (!make_tmap_bf16_2d(&ta, a.A, a.M, a.K, a.lda, BM, BK)) return ZDIT_ERR_CUDA;
  if (!make_tmap_bf16_2d(&tb, a.B, a.N, a.K, a.ldb, pair ? 128 : BN, BK)) return ZDIT_ERR_CUDA;
  KParams kp;
  kp.M = a.M; kp.N = a.N; kp.K = a.K; kp.ldo = a.ldo; kp.out = a.out; kp.bias = a.bias;
  kp.rcos = a.rope_cos; kp.rsin = a.rope_sin; kp.qn = a.qn; kp.kn = a.kn; kp.eps = a.eps; kp.dim = a.dim;
  kp.num_m = pair ? (a.M + 255) / 256 : (a.M + BM - 1) / BM;
  kp.num_n = (a.N + BN - 1) / BN;
  const int kslice = !pair ? BK : (a.epi == EPI_SWIGLU ? pair_bk<EPI_SWIGLU>() : pair_bk<EPI_BF16>());
  kp.num_k = (a.K + kslice - 1) / kslice;
  // L2-aware raster: a band of tiles of one operand (about 32 MB, well inside one
  // die's share of the L2) stays resident while the other operand streams; the
  // streamed operand is re-read once per band.
  {
    const double band = (double)ZDIT_L2_BAND_MB * (1 << 20);
    const double a_tile = 2.0 * (pair ? 256 : BM) * a.K, b_tile = 2.0 * BN * a.K;
    const double a_all = 2.0 * a.M * a.K, b_all = 2.0 * a.N * a.K;
    int gm = (int)(band / a_tile), gn = (int)(band / b_tile);
    gm = gm < 1 ? 1 : (gm > kp.num_m ? kp.num_m : gm);
    gn = gn < 1 ? 1 : (gn > kp.num_n ? kp.num_n : gn);
    const double traffic_m = a_all + b_all * ((kp.num_m + gm - 1) / gm);
    const double traffic_n = b_all + a_all * ((kp.num_n + gn - 1) / gn);
    kp.group_m = gm;
    kp.group_n = gn;
    kp.raster = traffic_m <= traffic_n ? 0 : 1;
  }
  kp.err = device_error_ptr();
  kp.band_flags = pair ? a.band_flags : nullptr;
  const int tiles = kp.num_m * kp.num_n;
  int grid = tiles < num_sms() ? tiles : num_sms();
  if (pair) {
    const int pairs = num_sms() / 2;
    grid = 2 * (tiles < pairs ? tiles : pairs);
  }
  const double out_elt = (a.epi == EPI_F32) ? 4.0 : 2.0;
  const double out_cols = (a.epi == EPI_SWIGLU) ? a.N / 2.0 : (double)a.N;
  ProfScope ps(a.prof_kind, 2.0 * a.M * a.N * (double)a.K,
               2.0 * ((double)a.M * a.K + (double)a.N * a.K) + out_elt * a.M * out_cols, s);
  switch (a.epi) {
    case EPI_F32: return launch_epi<EPI_F32>(ta, tb, kp, grid, pair, s);
    case EPI_BF16: return launch_epi<EPI_BF16>(ta, tb, kp, grid, pair, s);
    case EPI_QKV:
      return a.qn != nullptr ? launch_epi<EPI_QKV_NORM>(ta, tb, kp, grid, pair, s)
                             : launch_epi<EPI_QKV>(ta, tb, kp, grid, pair, s);
    case EPI_SWIGLU: return launch_epi<EPI_SWIGLU>(ta, tb, kp, grid, pair, s);
  }
  return ZDIT_ERR_INVALID_ARG;
}

}  // namespace zdit
