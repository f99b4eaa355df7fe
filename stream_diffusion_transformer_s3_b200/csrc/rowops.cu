// Bandwidth-bound row and element kernels of the DiT hot path.
//
//   norm_modulate : a = Norm(x) * w * (1 + scale_b) -> bf16 GEMM operand
//                   (RMSNorm pre-norm of the block; LayerNorm without affine for the
//                   final layer; plain RMSNorm for the caption embedder)
//   residual      : x += gate_b * PostNorm(y) (y bf16), optionally fused with the
//                   next pre-norm so x is read once per step
//   adaln_gemv    : m_b = W_ada temb_b + b_ada (weight-streaming GEMV, 8 rows per warp)
//   euler_cfg     : x += (sigma_next - sigma_cur) * -(pos + g (pos - neg))
//   rope_table    : per-token cos/sin of the 3-axis rotary angles
//   timestep_embed, patchify / unpatchify, casts and row fills
//
// Row kernels use one 256-thread CTA per row; each thread keeps up to MAXV float4 of
// the row in registers so the row is read from HBM exactly once.
#include <cuda_bf16.h>

#include <cmath>

#include "internal.h"
#include "ptx.cuh"

namespace zdit {

// Latched device-side error word (0 = none); kernels get its address as a
// parameter; zdit_device_status reads and clears it.
__device__ int g_device_error = 0;

// Looked up on every call, not cached: the address belongs to the current device's
// context and changes when that context is destroyed and created again.
int* device_error_ptr() {
  void* p = nullptr;
  return cudaGetSymbolAddress(&p, g_device_error) == cudaSuccess ? static_cast<int*>(p) : nullptr;
}

zdit_status read_and_clear_device_error() {
  int err = 0;
  if (cudaMemcpyFromSymbol(&err, g_device_error, sizeof(int)) != cudaSuccess) return ZDIT_ERR_CUDA;
  if (err != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_device_error, &zero, sizeof(int)) != cudaSuccess) return ZDIT_ERR_CUDA;
  }
  return static_cast<zdit_status>(err);
}

namespace {

constexpr int RT = 256;  // threads per row CTA
constexpr int kGemvBatchMax = 40;

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ float block_sum(float v, float* sh) {
  v = warp_sum(v);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  if (l == 0) sh[w] = v;
  __syncthreads();
  float r = 0.f;
#pragma unroll
  for (int i = 0; i < RT / 32; ++i) r += sh[i];
  __syncthreads();
  return r;
}

__device__ __forceinline__ int branch_of(const int* cu, int batch, int t) {
  int b = 0;
  while (b + 1 < batch && t >= cu[b + 1]) ++b;
  return b;
}

__device__ __forceinline__ void store_bf16x4(__nv_bfloat16* dst, float a, float b, float c, float d) {
  uint2 u = make_uint2(pack_bf16x2(a, b), pack_bf16x2(c, d));
  *reinterpret_cast<uint2*>(dst) = u;
}

struct NormModParams {
  const float* x;
  int D;
  const float* w;
  const float* mod;
  int mod_stride;
  const int* cu;
  int batch;
  int fixed_branch;
  int layer_norm;
  float eps;
  __nv_bfloat16* out;
};

template <int MAXV>
__global__ void __launch_bounds__(RT) norm_modulate_kernel(NormModParams p) {
  __shared__ float sh[RT / 32];
  griddep_wait();
  griddep_trigger();
  const int t = blockIdx.x;
  const float* xr = p.x + (size_t)t * p.D;
  float4 v[MAXV];
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < MAXV; ++i) {
    const int idx = (i * RT + threadIdx.x) * 4;
    v[i] = idx < p.D ? *reinterpret_cast<const float4*>(xr + idx) : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  float mean = 0.f;
  if (p.layer_norm) {
#pragma unroll
    for (int i = 0; i < MAXV; ++i) s += v[i].x + v[i].y + v[i].z + v[i].w;
    mean = block_sum(s, sh) / p.D;
  }
  float ss = 0.f;
#pragma unroll
  for (int i = 0; i < MAXV; ++i) {
    const int idx = (i * RT + threadIdx.x) * 4;
    if (idx < p.D) {
      const float a = v[i].x - mean, b = v[i].y - mean, c = v[i].z - mean, d = v[i].w - mean;
      ss += a * a + b * b + c * c + d * d;
    }
  }
  const float rstd = 1.0f / sqrtf(block_sum(ss, sh) / p.D + p.eps);
  const int br = p.cu != nullptr ? branch_of(p.cu, p.batch, t) : p.fixed_branch;
  const float* sc = p.mod != nullptr ? p.mod + (size_t)br * p.mod_stride : nullptr;
  __nv_bfloat16* orow = p.out + (size_t)t * p.D;
#pragma unroll
  for (int i = 0; i < MAXV; ++i) {
    const int idx = (i * RT + threadIdx.x) * 4;
    if (idx < p.D) {
      float4 w4 = p.w != nullptr ? *reinterpret_cast<const float4*>(p.w + idx) : make_float4(1.f, 1.f, 1.f, 1.f);
      if (sc != nullptr) {
        const float4 s4 = *reinterpret_cast<const float4*>(sc + idx);
        w4.x *= 1.f + s4.x; w4.y *= 1.f + s4.y; w4.z *= 1.f + s4.z; w4.w *= 1.f + s4.w;
      }
      store_bf16x4(orow + idx, (v[i].x - mean) * rstd * w4.x, (v[i].y - mean) * rstd * w4.y,
                   (v[i].z - mean) * rstd * w4.z, (v[i].w - mean) * rstd * w4.w);
    }
  }
}

struct ResidParams {
  float* x;
  const __nv_bfloat16* y;
  int D;
  const float* post_w;
  const float* gate;
  int gate_stride;
  int tanh_gate;
  const int* cu;
  int batch;
  float eps;
  const float* next_w;
  const float* next_scale;
  int next_scale_stride;
  __nv_bfloat16* next_out;
  const int* band_flags;
  int band_target;
  int* err;
};

template <int MAXV>
__global__ void __launch_bounds__(RT) residual_kernel(ResidParams p) {
  __shared__ float sh[RT / 32];
  __shared__ int band_ok;
  const int t = blockIdx.x;
  if (p.band_flags != nullptr) {
    // The producing GEMM signals each 128-row band once all its tiles are stored, so
    // this row starts then instead of after the whole GEMM: the CTAs run beside the
    // GEMM's last tiles.  Everything else this kernel reads was complete before that
    // GEMM passed its own dependency wait, which precedes the launch of this grid.
    if (threadIdx.x == 0) {
      const int* f = p.band_flags + (t >> 7);
      const uint64_t t0 = globaltimer_ns();
      int v;
      while (true) {
        asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(f) : "memory");
        if (v >= p.band_target) break;
        if (globaltimer_ns() - t0 > kWaitLimitNs) {
          atomicCAS(p.err, 0, -7 /* ZDIT_ERR_DEVICE_TIMEOUT */);
          v = -1;
          break;
        }
        __nanosleep(200);
      }
      band_ok = v >= 0;
    }
    __syncthreads();
    griddep_trigger();
    if (!band_ok) return;  // uniform across the CTA
  } else {
    griddep_wait();
    griddep_trigger();
  }
  const __nv_bfloat16* yr = p.y + (size_t)t * p.D;
  float* xr = p.x + (size_t)t * p.D;
  float4 y[MAXV];
  float ss = 0.f;
#pragma unroll
  for (int i = 0; i < MAXV; ++i) {
    const int idx = (i * RT + threadIdx.x) * 4;
    if (idx < p.D) {
      // L2 loads: y may have been written by another SM moments ago (band-by-band start)
      const uint2 u = __ldcg(reinterpret_cast<const uint2*>(yr + idx));
      const __nv_bfloat162 lo = *reinterpret_cast<const __nv_bfloat162*>(&u.x);
      const __nv_bfloat162 hi = *reinterpret_cast<const __nv_bfloat162*>(&u.y);
      y[i] = make_float4(__low2float(lo), __high2float(lo), __low2float(hi), __high2float(hi));
    } else {
      y[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    ss += y[i].x * y[i].x + y[i].y * y[i].y + y[i].z * y[i].z + y[i].w * y[i].w;
  }
  // the residual row does not depend on the reduction: load it now so both streams
  // are in flight together
  float4 xv[MAXV];
#pragma unroll
  for (int i = 0; i < MAXV; ++i) {
    const int idx = (i * RT + threadIdx.x) * 4;
    xv[i] = idx < p.D ? *reinterpret_cast<const float4*>(xr + idx) : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  float r = 1.f;
  if (p.post_w != nullptr) r = 1.0f / sqrtf(block_sum(ss, sh) / p.D + p.eps);
  const int br = branch_of(p.cu, p.batch, t);
  const float* g = p.gate != nullptr ? p.gate + (size_t)br * p.gate_stride : nullptr;
  float ss2 = 0.f;
#pragma unroll
  for (int i = 0; i < MAXV; ++i) {
    const int idx = (i * RT + threadIdx.x) * 4;
    if (idx < p.D) {
      float4 x4 = xv[i];
      float4 w4 = p.post_w != nullptr ? *reinterpret_cast<const float4*>(p.post_w + idx)
                                      : make_float4(1.f, 1.f, 1.f, 1.f);
      float4 g4 = g != nullptr ? *reinterpret_cast<const float4*>(g + idx) : make_float4(1.f, 1.f, 1.f, 1.f);
      if (p.tanh_gate && g != nullptr) {
        g4.x = tanhf(g4.x); g4.y = tanhf(g4.y); g4.z = tanhf(g4.z); g4.w = tanhf(g4.w);
      }
      x4.x += g4.x * (y[i].x * r * w4.x);
      x4.y += g4.y * (y[i].y * r * w4.y);
      x4.z += g4.z * (y[i].z * r * w4.z);
      x4.w += g4.w * (y[i].w * r * w4.w);
      *reinterpret_cast<float4*>(xr + idx) = x4;
      y[i] = x4;  // keep the updated residual for the fused next norm
      ss2 += x4.x * x4.x + x4.y * x4.y + x4.z * x4.z + x4.w * x4.w;
    }
  }
  if (p.next_out == nullptr) return;  // uniform across the CTA
  const float r2 = 1.0f / sqrtf(block_sum(ss2, sh) / p.D + p.eps);
  const float* sc = p.next_scale != nullptr ? p.next_scale + (size_t)br * p.next_scale_stride : nullptr;
  __nv_bfloat16* orow = p.next_out + (size_t)t * p.D;
#pragma unroll
  for (int i = 0; i < MAXV; ++i) {
    const int idx = (i * RT + threadIdx.x) * 4;
    if (idx < p.D) {
      float4 w4 = *reinterpret_cast<const float4*>(p.next_w + idx);
      if (sc != nullptr) {
        const float4 s4 = *reinterpret_cast<const float4*>(sc + idx);
        w4.x *= 1.f + s4.x; w4.y *= 1.f + s4.y; w4.z *= 1.f + s4.z; w4.w *= 1.f + s4.w;
      }
      store_bf16x4(orow + idx, y[i].x * r2 * w4.x, y[i].y * r2 * w4.y, y[i].z * r2 * w4.z, y[i].w * r2 * w4.w);
    }
  }
}

// Several GEMVs of the same shape in one launch (every adaLN projection of a forward):
// blockIdx.y selects the matrix.
struct GemvBatch {
  const __nv_bfloat16* W[kGemvBatchMax];
  const float* bias[kGemvBatchMax];
  float* out[kGemvBatchMax];
};

// Weight-streaming GEMV of the adaLN projections: out_m[b, r] = sum_e W_m[r, e] temb[b, e]
// + bias_m[r].  The rows of every matrix are cut into groups of 8; a warp reduces one group
// at a time, lane l covering columns [8l, 8l + 8) of every 256-column chunk with the
// matching temb slice.  The warps of a grid of a few CTAs per SM stride over all groups of
// all matrices, and each loads the weights of its next (group, chunk) unit before reducing
// the current one, so every warp keeps 8 16-byte loads in flight while it computes (the
// weights are read once: the loads bypass L1).
template <int B>
__global__ void __launch_bounds__(128) adaln_gemv_kernel(const __grid_constant__ GemvBatch gb, int nm,
                                                         const float* __restrict__ temb, int E, int rows) {
  const int lane = threadIdx.x & 31;
  const int gpm = (rows + 7) / 8;              // groups per matrix
  const int nch = (E + 255) / 256;             // 256-column chunks per row
  const int64_t units_total = (int64_t)nm * gpm * nch;
  const int64_t wstride = (int64_t)gridDim.x * (blockDim.x >> 5);
  // unit k of this warp: group (gw + (k / nch) * wstride), chunk k % nch
  const int64_t gw = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  auto load_unit = [&](int64_t grp, int ch, uint4 (&u)[8]) {
    const int m = (int)(grp / gpm);
    const int r0 = (int)(grp - (int64_t)m * gpm) * 8;
    const int e0 = ch * 256 + lane * 8;
    const __nv_bfloat16* W = gb.W[m];
#pragma unroll
    for (int r = 0; r < 8; ++r)
      u[r] = (r0 + r < rows && e0 < E) ? __ldcs(reinterpret_cast<const uint4*>(W + (size_t)(r0 + r) * E + e0))
                                       : make_uint4(0u, 0u, 0u, 0u);
  };
  if (gw * nch >= units_total) return;
  uint4 cur[8], nxt[8];
  load_unit(gw, 0, cur);
  float acc[8][B];
#pragma unroll
  for (int r = 0; r < 8; ++r)
#pragma unroll
    for (int b = 0; b < B; ++b) acc[r][b] = 0.f;
  for (int64_t grp = gw, ch = 0;;) {
    // next unit of this warp
    int64_t ngrp = grp;
    int nchk = (int)ch + 1;
    if (nchk == nch) {
      nchk = 0;
      ngrp = grp + wstride;
    }
    const bool more = ngrp * nch < units_total;
    if (more) load_unit(ngrp, nchk, nxt);
    const int e0 = (int)ch * 256 + lane * 8;
    if (e0 < E) {
      float t[B][8];
#pragma unroll
      for (int b = 0; b < B; ++b) {
        const float4 lo = __ldg(reinterpret_cast<const float4*>(temb + (size_t)b * E + e0));
        const float4 hi = __ldg(reinterpret_cast<const float4*>(temb + (size_t)b * E + e0 + 4));
        t[b][0] = lo.x; t[b][1] = lo.y; t[b][2] = lo.z; t[b][3] = lo.w;
        t[b][4] = hi.x; t[b][5] = hi.y; t[b][6] = hi.z; t[b][7] = hi.w;
      }
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        const __nv_bfloat16* h = reinterpret_cast<const __nv_bfloat16*>(&cur[r]);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float w = __bfloat162float(h[j]);
#pragma unroll
          for (int b = 0; b < B; ++b) acc[r][b] = fmaf(w, t[b][j], acc[r][b]);
        }
      }
    }
    if (ch + 1 == nch) {
      // the group's last chunk: reduce across the warp and store its 8 rows
      const int m = (int)(grp / gpm);
      const int r0 = (int)(grp - (int64_t)m * gpm) * 8;
      const float* bias = gb.bias[m];
      float* out = gb.out[m];
#pragma unroll
      for (int r = 0; r < 8; ++r) {
#pragma unroll
        for (int b = 0; b < B; ++b) {
          const float v = warp_sum(acc[r][b]);
          acc[r][b] = 0.f;
          if (lane == 0 && r0 + r < rows) out[(size_t)b * rows + r0 + r] = v + (bias != nullptr ? bias[r0 + r] : 0.f);
        }
      }
    }
    if (!more) break;
#pragma unroll
    for (int r = 0; r < 8; ++r) cur[r] = nxt[r];
    grp = ngrp;
    ch = nchk;
  }
}

template <int B>
void launch_gemv_b(const GemvBatch& gb, int nm, const float* temb, int E, int rows, cudaStream_t s) {
  // 8 CTAs (32 warps) per SM at most; measured faster than a grid of only the resident
  // CTAs (4 per SM at B = 2) with or without L2 prefetches ahead of the loads
  const int64_t groups = (int64_t)nm * ((rows + 7) / 8);
  int64_t ctas = (groups + 3) / 4;  // 4 warps per CTA, at least one group per warp
  const int64_t cap = (int64_t)num_sms() * 8;
  if (ctas > cap) ctas = cap;
  adaln_gemv_kernel<B><<<(unsigned)ctas, 128, 0, s>>>(gb, nm, temb, E, rows);
}

void launch_gemv_any(const GemvBatch& gb, int nm, const float* temb, int B, int E, int rows, cudaStream_t s) {
  switch (B) {
    case 1: launch_gemv_b<1>(gb, nm, temb, E, rows, s); break;
    case 2: launch_gemv_b<2>(gb, nm, temb, E, rows, s); break;
    case 3: launch_gemv_b<3>(gb, nm, temb, E, rows, s); break;
    case 4: launch_gemv_b<4>(gb, nm, temb, E, rows, s); break;
    case 5: launch_gemv_b<5>(gb, nm, temb, E, rows, s); break;
    case 6: launch_gemv_b<6>(gb, nm, temb, E, rows, s); break;
    case 7: launch_gemv_b<7>(gb, nm, temb, E, rows, s); break;
    default: launch_gemv_b<8>(gb, nm, temb, E, rows, s); break;
  }
}

__global__ void euler_cfg_kernel(float* __restrict__ x, const float* __restrict__ vp,
                                 const float* __restrict__ vn, int64_t n, float g, float dsig) {
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  const int64_t n4 = n / 4;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += stride) {
    float4 xv = reinterpret_cast<float4*>(x)[i];
    const float4 p = reinterpret_cast<const float4*>(vp)[i];
    float4 q = p;
    if (vn != nullptr) q = reinterpret_cast<const float4*>(vn)[i];
    // v = -(pos + g (pos - neg)); x += dsig * v
    xv.x += dsig * -(p.x + g * (p.x - q.x));
    xv.y += dsig * -(p.y + g * (p.y - q.y));
    xv.z += dsig * -(p.z + g * (p.z - q.z));
    xv.w += dsig * -(p.w + g * (p.w - q.w));
    reinterpret_cast<float4*>(x)[i] = xv;
  }
  for (int64_t i = n4 * 4 + (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride) {
    const float p = vp[i];
    const float q = vn != nullptr ? vn[i] : p;
    x[i] += dsig * -(p + g * (p - q));
  }
}

// cos / sin of phi[t, i] = pos[t, axis(i)] * theta^(-2 j / width_axis) for a block of
// kRopeTokens tokens per CTA: the frequencies of the pairs are computed once per CTA into
// shared memory, then every (token, pair) angle and its cos / sin in double precision,
// rounded to fp32 (the phases reach ~130 rad, so fp32 angles would be off by ~1e-5).
constexpr int kRopeTokens = 32;

__global__ void rope_table_kernel(const int* __restrict__ pos, int64_t T, int half_dim, int a0, int a1, int a2,
                                  double theta, float* __restrict__ cs, float* __restrict__ sn) {
  extern __shared__ double omega[];  // [half_dim]
  const int start1 = a0 / 2, start2 = (a0 + a1) / 2;  // first pair of axes 1 and 2
  for (int i = threadIdx.x; i < half_dim; i += blockDim.x) {
    int j, width;
    if (i < a0 / 2) {
      j = i; width = a0;
    } else if (i < (a0 + a1) / 2) {
      j = i - a0 / 2; width = a1;
    } else {
      j = i - (a0 + a1) / 2; width = a2;
    }
    omega[i] = pow(theta, -2.0 * j / width);
  }
  __syncthreads();
  const int64_t t0 = (int64_t)blockIdx.x * kRopeTokens;
  const int64_t n = (T - t0 < kRopeTokens ? T - t0 : kRopeTokens) * half_dim;
  for (int64_t e = threadIdx.x; e < n; e += blockDim.x) {
    const int64_t t = t0 + e / half_dim;
    const int i = (int)(e % half_dim);
    const int axis = i < start1 ? 0 : (i < start2 ? 1 : 2);
    double s, c;
    sincos((double)pos[t * 3 + axis] * omega[i], &s, &c);
    cs[t * half_dim + i] = (float)c;
    sn[t * half_dim + i] = (float)s;
  }
}

struct TembParams {
  float t[8];
};

// temb_b = W2 . SiLU(W1 . [cos | sin](t_scale * t_b * freqs) + b1) + b2, E <= 1024.
__global__ void timestep_embed_kernel(TembParams tp, int E, float t_scale, const __nv_bfloat16* __restrict__ w1,
                                      const float* __restrict__ b1, const __nv_bfloat16* __restrict__ w2,
                                      const float* __restrict__ b2, float* __restrict__ temb) {
  extern __shared__ float sm[];  // [2E]
  float* emb = sm;
  float* hid = sm + E;
  const int b = blockIdx.x;
  const int half = E / 2;
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    const int i = e % half;
    const double freq = exp(-log(10000.0) * (double)i / (double)half);
    const double arg = (double)t_scale * (double)tp.t[b] * freq;
    emb[e] = (float)(e < half ? cos(arg) : sin(arg));
  }
  __syncthreads();
  // the two E x E products: a warp per output row, lanes split the row in 16-byte pieces
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  auto row_dot = [&](const __nv_bfloat16* wr, const float* v) {
    float a = 0.f;
    for (int k = lane * 8; k < E; k += 256) {
      const uint4 u = *reinterpret_cast<const uint4*>(wr + k);
      const __nv_bfloat16* h = reinterpret_cast<const __nv_bfloat16*>(&u);
#pragma unroll
      for (int j = 0; j < 8; ++j) a += __bfloat162float(h[j]) * v[k + j];
    }
    return warp_sum(a);
  };
  for (int e = warp; e < E; e += nw) {
    const float a = row_dot(w1 + (size_t)e * E, emb) + b1[e];
    if (lane == 0) hid[e] = a / (1.0f + expf(-a));
  }
  __syncthreads();
  for (int e = warp; e < E; e += nw) {
    const float a = row_dot(w2 + (size_t)e * E, hid) + b2[e];
    if (lane == 0) temb[(size_t)b * E + e] = a;
  }
}

// tokens[n, f] <-> latent[c, 2 hi + dy, 2 wi + dx] with n = hi * w + wi and
// f = (dy * 2 + dx) * C + c; `dir` 0 = patchify, 1 = unpatchify.
__global__ void patchify_kernel(const float* __restrict__ src, float* __restrict__ dst, int C, int h, int w,
                                int dir) {
  const int64_t total = (int64_t)h * w * 4 * C;
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= total) return;
  const int F = 4 * C;
  const int64_t n = idx / F;
  const int f = (int)(idx % F);
  const int q = f / C, c = f % C;
  const int dy = q >> 1, dx = q & 1;
  const int hi = (int)(n / w), wi = (int)(n % w);
  const int64_t li = ((int64_t)c * (2 * h) + (2 * hi + dy)) * (2 * w) + (2 * wi + dx);
  if (dir == 0)
    dst[idx] = src[li];
  else
    dst[li] = src[idx];
}

__global__ void cast_bf16_kernel(const float* __restrict__ src, __nv_bfloat16* __restrict__ dst, int64_t n) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) dst[i] = __float2bfloat16_rn(src[i]);
}

__global__ void fill_rows_kernel(float* __restrict__ x, int D, int nrows, const float* __restrict__ vec) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i < (int64_t)nrows * D) x[i] = vec[i % D];
}

struct LayoutParams {
  int B, grid_h, grid_w;
  int n_cap[8];
};

// Token layout of the stack: branch b is [image (n_img) | caption (n_cap_b)].
// Positions: image cell (h, w) -> (n_cap_b + 1, h, w); caption k -> (k + 1, 0, 0).
// Writes the positions of the image-only, caption-only and joint sequences and the
// three cu_seqlens arrays.
__global__ void stack_layout_kernel(LayoutParams lp, int* __restrict__ pos_img, int* __restrict__ pos_cap,
                                    int* __restrict__ pos_joint, int* __restrict__ cu_img, int* __restrict__ cu_cap,
                                    int* __restrict__ cu_joint) {
  const int n_img = lp.grid_h * lp.grid_w;
  int joff[9], coff[9];
  joff[0] = coff[0] = 0;
  for (int b = 0; b < lp.B; ++b) {
    joff[b + 1] = joff[b] + n_img + lp.n_cap[b];
    coff[b + 1] = coff[b] + lp.n_cap[b];
  }
  const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (t == 0) {
    for (int b = 0; b <= lp.B; ++b) {
      cu_img[b] = b * n_img;
      cu_cap[b] = coff[b];
      cu_joint[b] = joff[b];
    }
  }
  if (t >= joff[lp.B]) return;
  int b = 0;
  while (t >= joff[b + 1]) ++b;
  const int local = (int)(t - joff[b]);
  int p0, p1, p2;
  if (local < n_img) {
    p0 = lp.n_cap[b] + 1;
    p1 = local / lp.grid_w;
    p2 = local % lp.grid_w;
    const int64_t ii = (int64_t)b * n_img + local;
    pos_img[ii * 3] = p0; pos_img[ii * 3 + 1] = p1; pos_img[ii * 3 + 2] = p2;
  } else {
    const int k = local - n_img;
    p0 = k + 1; p1 = 0; p2 = 0;
    const int64_t ci = coff[b] + k;
    pos_cap[ci * 3] = p0; pos_cap[ci * 3 + 1] = p1; pos_cap[ci * 3 + 2] = p2;
  }
  pos_joint[t * 3] = p0; pos_joint[t * 3 + 1] = p1; pos_joint[t * 3 + 2] = p2;
}

}  // namespace

void launch_stack_layout(const int* n_cap, int B, int grid_h, int grid_w, int* pos_img, int* pos_cap, int* pos_joint,
                         int* cu_img, int* cu_cap, int* cu_joint, cudaStream_t s) {
  ProfScope ps(PROF_MISC, 0.0, 0.0, s);
  LayoutParams lp;
  lp.B = B; lp.grid_h = grid_h; lp.grid_w = grid_w;
  int64_t T = 0;
  for (int b = 0; b < 8; ++b) {
    lp.n_cap[b] = b < B ? n_cap[b] : 0;
    if (b < B) T += (int64_t)grid_h * grid_w + n_cap[b];
  }
  stack_layout_kernel<<<(unsigned)((T + 255) / 256), 256, 0, s>>>(lp, pos_img, pos_cap, pos_joint, cu_img, cu_cap,
                                                                  cu_joint);
}

void launch_norm_modulate_ex(const float* x, int T, int D, const float* w, const float* mod, int mod_stride,
                             const int* cu, int batch, int fixed_branch, int layer_norm, float eps,
                             __nv_bfloat16* out, cudaStream_t s) {
  ProfScope ps(PROF_NORM_MOD, 0.0, (double)T * D * (4.0 + 2.0), s);
  NormModParams p{x, D, w, mod, mod_stride, cu, batch, fixed_branch, layer_norm, eps, out};
  const int v = (D + RT * 4 - 1) / (RT * 4);
  if (T <= 0) return;
  if (v <= 1)
    launch_dependent(norm_modulate_kernel<1>, dim3(T), dim3(RT), 0, s, p);
  else if (v <= 2)
    launch_dependent(norm_modulate_kernel<2>, dim3(T), dim3(RT), 0, s, p);
  else if (v <= 4)
    launch_dependent(norm_modulate_kernel<4>, dim3(T), dim3(RT), 0, s, p);
  else
    launch_dependent(norm_modulate_kernel<8>, dim3(T), dim3(RT), 0, s, p);
}

void launch_norm_modulate(const RowModArgs& a, cudaStream_t s) {
  launch_norm_modulate_ex(a.x, a.T, a.D, a.w, a.mod, a.mod_stride, a.cu_seqlens, a.batch, 0, 0, a.eps, a.out, s);
}

void launch_residual(const ResidArgs& a, cudaStream_t s) {
  ProfScope ps(PROF_RESIDUAL, 0.0, (double)a.T * a.D * (10.0 + (a.next_out ? 2.0 : 0.0)), s);
  ResidParams p{a.x,       a.y,    a.D,          a.post_w,  a.gate,       a.gate_stride, a.tanh_gate,
                a.cu_seqlens, a.batch, a.eps,    a.next_w,  a.next_scale, a.next_scale_stride, a.next_out,
                a.band_flags, a.band_target, device_error_ptr()};
  const int v = (a.D + RT * 4 - 1) / (RT * 4);
  if (a.T <= 0) return;
  if (v <= 1)
    launch_dependent(residual_kernel<1>, dim3(a.T), dim3(RT), 0, s, p);
  else if (v <= 2)
    launch_dependent(residual_kernel<2>, dim3(a.T), dim3(RT), 0, s, p);
  else if (v <= 4)
    launch_dependent(residual_kernel<4>, dim3(a.T), dim3(RT), 0, s, p);
  else
    launch_dependent(residual_kernel<8>, dim3(a.T), dim3(RT), 0, s, p);
}

void launch_gemv(const __nv_bfloat16* W, const float* bias, const float* temb, int B, int E, int rows, float* out,
                 cudaStream_t s) {
  ProfScope ps(PROF_GEMV, 2.0 * rows * (double)E * B, 2.0 * rows * (double)E + 4.0 * rows * (B + 1.0), s);
  GemvBatch gb{};
  gb.W[0] = W;
  gb.bias[0] = bias;
  gb.out[0] = out;
  launch_gemv_any(gb, 1, temb, B, E, rows, s);
}

void launch_gemv_batched(const __nv_bfloat16* const* W, const float* const* bias, float* const* out, int nmat,
                         const float* temb, int B, int E, int rows, cudaStream_t s) {
  for (int m0 = 0; m0 < nmat; m0 += kGemvBatchMax) {
    const int nm = nmat - m0 < kGemvBatchMax ? nmat - m0 : kGemvBatchMax;
    GemvBatch gb{};
    for (int i = 0; i < nm; ++i) {
      gb.W[i] = W[m0 + i];
      gb.bias[i] = bias[m0 + i];
      gb.out[i] = out[m0 + i];
    }
    ProfScope ps(PROF_GEMV, 2.0 * rows * (double)E * B * nm, (2.0 * rows * (double)E + 4.0 * rows * (B + 1.0)) * nm, s);
    launch_gemv_any(gb, nm, temb, B, E, rows, s);
  }
}

void launch_euler_cfg(float* x, const float* vp, const float* vn, int64_t n, float g, float dsig, cudaStream_t s) {
  ProfScope ps(PROF_EULER, 0.0, 4.0 * (double)n * (vn != nullptr ? 4.0 : 3.0), s);
  int blocks = (int)((n / 4 + 255) / 256);
  if (blocks < 1) blocks = 1;
  if (blocks > 4 * num_sms()) blocks = 4 * num_sms();
  euler_cfg_kernel<<<blocks, 256, 0, s>>>(x, vp, vn, n, g, dsig);
}

void launch_rope_table(const int* pos, int64_t T, int head_dim, const int* axes, float theta, float* cs, float* sn,
                       cudaStream_t s) {
  ProfScope ps(PROF_ROPE, 0.0, 8.0 * (double)T * (head_dim / 2) + 12.0 * T, s);
  if (T <= 0 || head_dim <= 0) return;
  rope_table_kernel<<<(unsigned)((T + kRopeTokens - 1) / kRopeTokens), 256, (head_dim / 2) * sizeof(double), s>>>(
      pos, T, head_dim / 2, axes[0], axes[1], axes[2], (double)theta, cs, sn);
}

void launch_timestep_embed(const float* t_host, int B, int E, float t_scale, const __nv_bfloat16* w1,
                           const float* b1, const __nv_bfloat16* w2, const float* b2, float* temb, cudaStream_t s) {
  ProfScope ps(PROF_MISC, 0.0, 0.0, s);
  TembParams tp;
  for (int i = 0; i < 8; ++i) tp.t[i] = i < B ? t_host[i] : 0.f;
  timestep_embed_kernel<<<B, 256, 2 * E * sizeof(float), s>>>(tp, E, t_scale, w1, b1, w2, b2, temb);
}

void launch_patchify(const float* src, float* dst, int C, int h, int w, int dir, cudaStream_t s) {
  ProfScope ps(PROF_MISC, 0.0, 8.0 * (double)h * w * 4 * C, s);
  const int64_t total = (int64_t)h * w * 4 * C;
  if (total <= 0) return;
  patchify_kernel<<<(unsigned)((total + 255) / 256), 256, 0, s>>>(src, dst, C, h, w, dir);
}

void launch_cast_bf16(const float* src, __nv_bfloat16* dst, int64_t n, cudaStream_t s) {
  ProfScope ps(PROF_MISC, 0.0, 6.0 * (double)n, s);
  if (n <= 0) return;
  cast_bf16_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(src, dst, n);
}

void launch_fill_rows(float* x, int D, int nrows, const float* vec, cudaStream_t s) {
  ProfScope ps(PROF_MISC, 0.0, 4.0 * (double)nrows * D, s);
  const int64_t n = (int64_t)nrows * D;
  if (n <= 0) return;
  fill_rows_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(x, D, nrows, vec);
}

}  // namespace zdit
