// Varlen joint attention for sm_100a (head dim 128), flash-style with tcgen05.
//
// One CTA computes two 128-row query tiles of one (branch, head):
//   O = softmax(Q K^T / sqrt(128)) V over all L_b tokens of its branch segment.
// There is no mask inside a segment: caption pad tokens are ordinary context
// ("Z-Image-Turbo port", "The three things that each cost a wrong image", item 3),
// branches never see each other, and only the columns past the segment end of the
// last key tile are excluded.
//
// Warp roles (384 threads, three warpgroups):
//   warps 0-3 : softmax of query tile 0, one thread per query row (TMEM lane)
//   warps 4-7 : softmax of query tile 1
//   warp 8    : TMA producer (Q0, K0, then Q1; K and V tiles in separate 2-deep rings)
//   warp 9    : tcgen05.mma issuer
//   warps 10-11 complete the control warpgroup, which hands registers to the softmax
//   warpgroups (setmaxnreg: 168 at launch -> 208 softmax, 88 control).
// TMEM columns: S0 [0,128), S1 [128,256), O0 [256,384), O1 [384,512).  P_t (bf16,
// two per 32-bit column) is written back over the first 64 columns of S_t and fed
// to the PV product straight from TMEM, so P never touches shared memory.
// The tensor core alternates between the two tiles: PV0(j-1), S0(j), PV1(j-1),
// S1(j), ... so the softmax of one tile overlaps the MMAs of the other.  Because
// PV_t(j-1) is issued before S_t(j), the commit that signals S_t(j) also proves that
// PV_t(j-1) is done: the softmax may then overwrite P_t and rescale O_t freely.
// Online softmax in FP32 with a lazily moved reference max: the running max only
// moves (and O is rescaled) when a row's max grows by more than 16 (log2 units), so
// the common tile needs no O round trip; P = exp2(s - m_ref) <= 2^16 keeps bf16's
// relative precision, and O and the row sum stay far inside FP32 range.
// The epilogue stages O / l as bf16 in the shared memory that Q and the K ring no
// longer need, then writes two full 256-byte rows per warp store instruction.
#include <cstdio>

#include "internal.h"
#include "ptx.cuh"

namespace zdit {

bool make_tmap_bf16_2d(CUtensorMap* m, const void* ptr, uint64_t rows, uint64_t cols, uint64_t ld_elems,
                       uint32_t box_rows, uint32_t box_cols);

namespace {

constexpr int TILE = 128;            // query rows and key rows per tile
constexpr int HD = 128;              // head dim
constexpr int HALF = TILE * 64 * 2;  // one 64-column swizzled half tile: 16 KB
constexpr int TILE_BYTES = 2 * HALF;
constexpr int THREADS = 384;  // three warpgroups: softmax tile 0, softmax tile 1, control
constexpr int WARP_LOAD = 8, WARP_MMA = 9;
// smem: Q0 | Q1 | K[2] | V[2], then barriers
constexpr int OFF_Q = 0;
constexpr int OFF_K = OFF_Q + 2 * TILE_BYTES;
constexpr int OFF_V = OFF_K + 2 * TILE_BYTES;
constexpr int OFF_BAR = OFF_V + 2 * TILE_BYTES;
constexpr int SMEM_BYTES = 1024 + OFF_BAR + 256;
constexpr float kRescaleThreshold = 16.0f;  // log2 units

struct AParams {
  int ldo, n_heads, batch;
  void* o;
  const int* cu;
  float scale_log2;
  int* err;
};

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// Packed pairs of fp32 (Blackwell f32x2 arithmetic: one instruction, two lanes).
__device__ __forceinline__ uint64_t pk2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void unpk2(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}

__global__ void __launch_bounds__(THREADS, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const AParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint64_t* q_full = bars + 0;    // [2] one per query tile
  uint64_t* k_full = bars + 2;    // [2]
  uint64_t* k_empty = bars + 4;   // [2]
  uint64_t* v_full = bars + 6;    // [2]
  uint64_t* v_empty = bars + 8;   // [2]
  uint64_t* s_full = bars + 10;   // [2] one per query tile
  uint64_t* p_full = bars + 12;   // [2]
  uint64_t* o_full = bars + 14;   // [2]
  uint64_t* mma_done = bars + 16;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 17);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int head = blockIdx.y;
  griddep_wait();     // Q, K, V of the predecessor are complete
  griddep_trigger();  // every CTA has started: the successor may launch

  // locate (branch, query-tile pair) of this CTA
  int b = 0, pair = blockIdx.x;
  int seg0 = 0, L = 0;
  for (; b < p.batch; ++b) {
    seg0 = p.cu[b];
    L = p.cu[b + 1] - seg0;
    const int np = ((L + TILE - 1) / TILE + 1) / 2;
    if (pair < np) break;
    pair -= np;
  }
  if (b >= p.batch) return;  // (grid sized exactly; defensive, uniform per CTA)
  const int n_kv = (L + TILE - 1) / TILE;
  const int q0 = seg0 + pair * 2 * TILE;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], 1);
      mbar_init(&v_full[i], 1);
      mbar_init(&v_empty[i], 1);
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], 4);
      mbar_init(&o_full[i], 1);
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == WARP_LOAD && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  if (warp == WARP_MMA) tmem_alloc(tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int col0 = head * HD;

  // Register split: launched with 168 per thread (384 x 168 = 64512); the control
  // warpgroup drops to 88 and the two softmax warpgroups rise to 208:
  // 2 x 128 x 208 + 128 x 88 = 64512, exactly the launch's registers.
  if (warp >= 8) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 88;\n" ::: "memory");
    if (warp == WARP_LOAD && lane == 0) {
      // ------------------------------------------------------------ producer
      // Q0, then K0, then Q1: the first S product waits for 64 KB instead of 96 KB
      uint8_t* sQ = smem + OFF_Q;
      mbar_arrive_expect_tx(&q_full[0], TILE_BYTES);
      tma_load_2d(sQ, &tmQ, &q_full[0], col0, q0);
      tma_load_2d(sQ + HALF, &tmQ, &q_full[0], col0 + 64, q0);
      int nk_issued = 0, nv_issued = 0;
      for (int j = 0; j < n_kv; ++j) {
        const int st = j & 1;
        const uint32_t par = ((j >> 1) & 1) ^ 1;
        const int r0 = seg0 + j * TILE;
        if (!mbar_wait(&k_empty[st], par, abort_flag, p.err)) break;
        uint8_t* sK = smem + OFF_K + st * TILE_BYTES;
        mbar_arrive_expect_tx(&k_full[st], TILE_BYTES);
        tma_load_2d(sK, &tmK, &k_full[st], col0, r0);
        tma_load_2d(sK + HALF, &tmK, &k_full[st], col0 + 64, r0);
        ++nk_issued;
        if (j == 0) {
          mbar_arrive_expect_tx(&q_full[1], TILE_BYTES);
          tma_load_2d(sQ + TILE_BYTES, &tmQ, &q_full[1], col0, q0 + TILE);
          tma_load_2d(sQ + TILE_BYTES + HALF, &tmQ, &q_full[1], col0 + 64, q0 + TILE);
        }
        if (!mbar_wait(&v_empty[st], par, abort_flag, p.err)) break;
        uint8_t* sV = smem + OFF_V + st * TILE_BYTES;
        mbar_arrive_expect_tx(&v_full[st], TILE_BYTES);
        tma_load_2d(sV, &tmV, &v_full[st], col0, r0);
        tma_load_2d(sV + HALF, &tmV, &v_full[st], col0 + 64, r0);
        ++nv_issued;
      }
      if (*abort_flag) {
        int dummy = 0;
        mbar_wait(&q_full[0], 0, &dummy);
        if (nk_issued > 0) mbar_wait(&q_full[1], 0, &dummy);
        for (int j = (nk_issued > 2 ? nk_issued - 2 : 0); j < nk_issued; ++j)
          mbar_wait(&k_full[j & 1], (j >> 1) & 1, &dummy);
        for (int j = (nv_issued > 2 ? nv_issued - 2 : 0); j < nv_issued; ++j)
          mbar_wait(&v_full[j & 1], (j >> 1) & 1, &dummy);
      }
    } else if (warp == WARP_MMA && lane == 0) {
      // ------------------------------------------------------------ MMA issuer
      // Each UMMA here is only 64 tensor clocks of work, so the issuing thread must do
      // almost nothing per instruction: every shared-memory descriptor is precomputed
      // (a descriptor is linear in the address: desc(addr + off) = desc(addr) + off / 16).
      const uint32_t id_s = idesc_bf16_f32(TILE, TILE);             // Q, K both K-major
      const uint32_t id_o = idesc_bf16_f32(TILE, HD, false, true);  // P from TMEM, V MN-major
      uint64_t dq[2], dk[2], dv[2];
      for (int t = 0; t < 2; ++t) dq[t] = sdesc_kmajor_sw128(smem_u32(smem + OFF_Q + t * TILE_BYTES));
      for (int i = 0; i < 2; ++i) dk[i] = sdesc_kmajor_sw128(smem_u32(smem + OFF_K + i * TILE_BYTES));
      for (int i = 0; i < 2; ++i) dv[i] = sdesc_mnmajor_sw128(smem_u32(smem + OFF_V + i * TILE_BYTES), HALF, 1024);
      // K step k of a K-major 128-byte-swizzled tile: (k / 4) 64-column halves + (k % 4) 32-byte slices
      auto koff = [](int k) -> uint64_t { return (uint64_t)(((k >> 2) * HALF + (k & 3) * 32) >> 4); };
      // K step k of the MN-major V tile: 16 key rows of 128 bytes
      auto voff = [](int k) -> uint64_t { return (uint64_t)((k * 16 * 128) >> 4); };
      const uint32_t tm_s[2] = {tmem, tmem + 128};
      const uint32_t tm_o[2] = {tmem + 256, tmem + 384};
      // O_t += P_t V_i ; P_t read from TMEM columns [t*128, t*128 + 64)
      auto issue_pv = [&](int t, int i) -> bool {
        if (!mbar_wait(&p_full[t], i & 1, abort_flag, p.err)) return false;
        if (t == 0 && !mbar_wait(&v_full[i & 1], (i >> 1) & 1, abort_flag, p.err)) return false;
        tc_fence_after();
        const uint64_t vb = dv[i & 1];
        const uint32_t d = tm_o[t], pa = tm_s[t];
        umma_bf16_ts(d, pa, vb, id_o, i != 0 ? 1u : 0u);
  #pragma unroll
        for (int k = 1; k < TILE / 16; ++k) umma_bf16_ts(d, pa + k * 8, vb + voff(k), id_o, 1u);
        return true;
      };
      // S_t = Q_t K_j^T into TMEM columns [t*128, t*128 + 128)
      auto issue_s = [&](int t, int j) {
        const uint64_t kb = dk[j & 1], qb = dq[t];
        const uint32_t d = tm_s[t];
        umma_bf16_ss(d, qb, kb, id_s, 0u);
  #pragma unroll
        for (int k = 1; k < HD / 16; ++k) umma_bf16_ss(d, qb + koff(k), kb + koff(k), id_s, 1u);
        umma_commit(&s_full[t]);
      };
      bool ok = mbar_wait(&q_full[0], 0, abort_flag, p.err);
      for (int j = 0; ok && j < n_kv; ++j) {
        if (!mbar_wait(&k_full[j & 1], (j >> 1) & 1, abort_flag, p.err)) { ok = false; break; }
        tc_fence_after();
        if (j > 0 && !issue_pv(0, j - 1)) { ok = false; break; }
        issue_s(0, j);
        if (j > 0) {
          if (!issue_pv(1, j - 1)) { ok = false; break; }
          umma_commit(&v_empty[(j - 1) & 1]);
        }
        if (j == 0 && !mbar_wait(&q_full[1], 0, abort_flag, p.err)) { ok = false; break; }
        issue_s(1, j);
        umma_commit(&k_empty[j & 1]);
      }
      if (ok && issue_pv(0, n_kv - 1)) {
        umma_commit(&o_full[0]);
        if (issue_pv(1, n_kv - 1)) {
          umma_commit(&o_full[1]);
          umma_commit(&v_empty[(n_kv - 1) & 1]);
        }
      }
      umma_commit(mma_done);
      int dummy = 0;
      mbar_wait(mma_done, 0, &dummy);
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 208;\n" ::: "memory");
    // ------------------------------------------------------------ softmax
    const int t = warp >> 2;         // query tile of this warpgroup
    const int lg = warp & 3;         // TMEM lane group
    const uint32_t lane_off = (uint32_t)(lg * 32) << 16;
    const uint32_t tS = tmem + lane_off + t * 128;
    const uint32_t tO = tmem + lane_off + 256 + t * 128;
    float m_ref = -INFINITY, l_sum = 0.f;
    bool ok = true;
    for (int j = 0; j < n_kv; ++j) {
      ok = __all_sync(0xffffffffu, mbar_wait(&s_full[t], j & 1, abort_flag, p.err));
      if (!ok) break;
      tc_fence_after();
      float s[TILE];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t r[32];
        tmem_ld32(tS + c * 32, r);
#pragma unroll
        for (int e = 0; e < 32; ++e) s[c * 32 + e] = __uint_as_float(r[e]);
      }
      tmem_ld_wait();
      const int valid = L - j * TILE;  // keys past the segment end are excluded
      if (valid < TILE) {
#pragma unroll
        for (int e = 0; e < TILE; ++e)
          if (e >= valid) s[e] = -INFINITY;
      }
      // row max: 8 independent chains of 3-input max (a single chain is latency-bound)
      float m8[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) m8[i] = fmaxf(s[i], s[8 + i]);
#pragma unroll
      for (int e = 16; e < TILE; e += 16)
#pragma unroll
        for (int i = 0; i < 8; ++i) m8[i] = fmax3(m8[i], s[e + i], s[e + 8 + i]);
      float mx = fmaxf(fmax3(m8[0], m8[1], m8[2]), fmax3(m8[3], m8[4], fmax3(m8[5], m8[6], m8[7])));
      mx *= p.scale_log2;
      float alpha = 1.f;
      bool move = false;
      if (j == 0) {
        m_ref = mx;
      } else if (mx > m_ref + kRescaleThreshold) {
        alpha = ex2(m_ref - mx);
        m_ref = mx;
        move = true;
      }
      l_sum *= alpha;
      if (__any_sync(0xffffffffu, move)) {  // O_t is stable: PV_t(j-1) completed before S_t(j)
#pragma unroll 1
        for (int c = 0; c < 8; ++c) {
          uint32_t r[16];
          tmem_ld16(tO + c * 16, r);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 16; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
          tmem_st16(tO + c * 16, r);
        }
      }
      // P = exp2(s * scale - m_ref) with packed f32x2 arithmetic, bf16 pairs over the
      // first 64 columns of S_t
      const uint64_t sc2 = pk2(p.scale_log2, p.scale_log2);
      const uint64_t nm2 = pk2(-m_ref, -m_ref);
      uint64_t part[4] = {0ull, 0ull, 0ull, 0ull};  // 4 independent packed sum chains
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const uint64_t x2 = fma2(pk2(s[c * 32 + 2 * e], s[c * 32 + 2 * e + 1]), sc2, nm2);
          float a, b;
          unpk2(x2, a, b);
          const float p0 = ex2(a), p1 = ex2(b);
          part[e & 3] = add2(part[e & 3], pk2(p0, p1));
          pk[e] = pack_bf16x2(p0, p1);
        }
        tmem_st16(tS + c * 16, pk);
      }
      float q0, q1, q2, q3, q4, q5, q6, q7;
      unpk2(part[0], q0, q1);
      unpk2(part[1], q2, q3);
      unpk2(part[2], q4, q5);
      unpk2(part[3], q6, q7);
      l_sum += ((q0 + q1) + (q2 + q3)) + ((q4 + q5) + (q6 + q7));
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[t]);
    }
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&o_full[t], 0, abort_flag, p.err));
    if (ok) {
      tc_fence_after();
      // O_t / l, staged as bf16 in shared memory so the global stores are coalesced: once
      // O_t is final every S product has completed, so Q and the K ring are idle (tile t
      // uses the t-th 64 KB; rows padded to 272 B keep the row-per-lane writes
      // conflict-free).
      constexpr int kStageRow = 2 * HD + 16;
      uint8_t* stage = smem + OFF_Q + t * 65536 + lg * 32 * kStageRow;
      const float inv = 1.0f / l_sum;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t r[32];
        tmem_ld32(tO + c * 32, r);
        tmem_ld_wait();
        uint4* dst = reinterpret_cast<uint4*>(stage + lane * kStageRow + c * 64);
#pragma unroll
        for (int e = 0; e < 4; ++e)
          dst[e] = make_uint4(pack_bf16x2(__uint_as_float(r[8 * e]) * inv, __uint_as_float(r[8 * e + 1]) * inv),
                              pack_bf16x2(__uint_as_float(r[8 * e + 2]) * inv, __uint_as_float(r[8 * e + 3]) * inv),
                              pack_bf16x2(__uint_as_float(r[8 * e + 4]) * inv, __uint_as_float(r[8 * e + 5]) * inv),
                              pack_bf16x2(__uint_as_float(r[8 * e + 6]) * inv, __uint_as_float(r[8 * e + 7]) * inv));
      }
      __syncwarp();
      // two 256-byte rows per warp instruction
      const int row0 = pair * 2 * TILE + t * TILE + lg * 32;
#pragma unroll 4
      for (int it = 0; it < 16; ++it) {
        const int r = it * 2 + (lane >> 4);
        const uint4 v = *reinterpret_cast<const uint4*>(stage + r * kStageRow + (lane & 15) * 16);
        if (row0 + r < L)
          *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.o) + (size_t)(seg0 + row0 + r) * p.ldo + col0 +
                                    (lane & 15) * 8) = v;
      }
    }
  }
  __syncthreads();
  if (warp == WARP_MMA) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

zdit_status launch_attention(const AttnArgs& a, cudaStream_t s) {
  if (a.T <= 0 || a.batch <= 0 || a.n_heads <= 0) return ZDIT_ERR_SHAPE;
  if (a.ldq % 8 || a.ldk % 8 || a.ldv % 8 || a.ldo % 8) return ZDIT_ERR_ALIGNMENT;
  if ((reinterpret_cast<uintptr_t>(a.q) | reinterpret_cast<uintptr_t>(a.k) | reinterpret_cast<uintptr_t>(a.v) |
       reinterpret_cast<uintptr_t>(a.o)) & 15)
    return ZDIT_ERR_ALIGNMENT;
  int total_pairs = 0;
  for (int b = 0; b < a.batch; ++b) {
    const int L = a.cu_seqlens_host[b + 1] - a.cu_seqlens_host[b];
    if (L <= 0) return ZDIT_ERR_SHAPE;
    total_pairs += ((L + TILE - 1) / TILE + 1) / 2;
  }
  if (a.cu_seqlens_host[0] != 0 || a.cu_seqlens_host[a.batch] > a.T) return ZDIT_ERR_SHAPE;
  CUtensorMap tq, tk, tv;
  const int cols = a.n_heads * HD;
  if (!make_tmap_bf16_2d(&tq, a.q, a.T, cols, a.ldq, TILE, 64)) return ZDIT_ERR_CUDA;
  if (!make_tmap_bf16_2d(&tk, a.k, a.T, cols, a.ldk, TILE, 64)) return ZDIT_ERR_CUDA;
  if (!make_tmap_bf16_2d(&tv, a.v, a.T, cols, a.ldv, TILE, 64)) return ZDIT_ERR_CUDA;
  // per launch: the opt-in belongs to the current context (see launch_epi)
  if (cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES) != cudaSuccess)
    return ZDIT_ERR_CUDA;
  AParams p;
  p.ldo = a.ldo;
  p.n_heads = a.n_heads;
  p.batch = a.batch;
  p.o = a.o;
  p.cu = a.cu_seqlens_dev;
  p.scale_log2 = a.scale * 1.4426950408889634f;
  p.err = device_error_ptr();
  double l2 = 0.0;
  for (int b = 0; b < a.batch; ++b) {
    const double L = a.cu_seqlens_host[b + 1] - a.cu_seqlens_host[b];
    l2 += L * L;
  }
  ProfScope ps(PROF_ATTENTION, 4.0 * HD * a.n_heads * l2, 4.0 * 2.0 * a.T * (double)cols, s);
  dim3 grid(total_pairs, a.n_heads);
  launch_dependent(attn_tc_kernel, grid, dim3(THREADS), SMEM_BYTES, s, tq, tk, tv, p);
  return cudaGetLastError() == cudaSuccess ? ZDIT_OK : ZDIT_ERR_CUDA;
}

}  // namespace zdit
