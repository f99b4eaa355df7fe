// C-ABI entry points: host-side validation, workspace carving and the launch
// sequence of the block, the stack and the sampler update.  No compute happens here;
// every step runs in the kernels of gemm.cu, attention.cu and rowops.cu.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstring>
#include <mutex>
#include <vector>

#include "internal.h"

namespace zdit {

// rowops.cu
void launch_norm_modulate_ex(const float* x, int T, int D, const float* w, const float* mod, int mod_stride,
                             const int* cu, int batch, int fixed_branch, int layer_norm, float eps,
                             __nv_bfloat16* out, cudaStream_t s);
void launch_gemv(const __nv_bfloat16* W, const float* bias, const float* temb, int B, int E, int rows, float* out,
                 cudaStream_t s);
void launch_euler_cfg(float* x, const float* vp, const float* vn, int64_t n, float g, float dsig, cudaStream_t s);
void launch_gemv_batched(const __nv_bfloat16* const* W, const float* const* bias, float* const* out, int nmat,
                         const float* temb, int B, int E, int rows, cudaStream_t s);
void launch_rope_table(const int* pos, int64_t T, int head_dim, const int* axes, float theta, float* cs, float* sn,
                       cudaStream_t s);
void launch_timestep_embed(const float* t_host, int B, int E, float t_scale, const __nv_bfloat16* w1,
                           const float* b1, const __nv_bfloat16* w2, const float* b2, float* temb, cudaStream_t s);
void launch_patchify(const float* src, float* dst, int C, int h, int w, int dir, cudaStream_t s);
void launch_cast_bf16(const float* src, __nv_bfloat16* dst, int64_t n, cudaStream_t s);
void launch_fill_rows(float* x, int D, int nrows, const float* vec, cudaStream_t s);
void launch_stack_layout(const int* n_cap, int B, int grid_h, int grid_w, int* pos_img, int* pos_cap, int* pos_joint,
                         int* cu_img, int* cu_cap, int* cu_joint, cudaStream_t s);

zdit_status read_and_clear_device_error();

// SM count of the current device (queried per call: a process may drive several devices)
int num_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      n <= 0)
    n = 148;
  return n;
}

namespace {

constexpr int kMaxBatch = 8;
constexpr int kMaxBlocks = 256;

// the current device is a compute capability 10.x part (checked per call, like num_sms)
bool device_ok() {
  int dev = 0, major = 0;
  return cudaGetDevice(&dev) == cudaSuccess &&
         cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) == cudaSuccess && major == 10;
}

size_t align_up(size_t v, size_t a = 256) { return (v + a - 1) / a * a; }

// Bump allocator over a caller-provided workspace.
struct Carver {
  uint8_t* base;
  size_t off = 0;
  explicit Carver(void* b) : base(static_cast<uint8_t*>(b)) {}
  template <typename T>
  T* take(size_t count) {
    T* p = base ? reinterpret_cast<T*>(base + off) : nullptr;
    off = align_up(off + count * sizeof(T));
    return p;
  }
};

bool cfg_ok(const zdit_block_cfg* c) {
  if (c == nullptr) return false;
  // dim <= 8192: the row kernels hold a whole row in one CTA's registers
  if (c->head_dim != 128 || c->n_heads <= 0 || c->dim != c->n_heads * 128 || c->dim % 256 || c->dim > 8192)
    return false;
  if (c->ffn_hidden <= 0 || c->ffn_hidden % 128) return false;
  if (c->temb_dim <= 0 || c->temb_dim % 8 || c->temb_dim > 1024) return false;
  if (c->rope_axes[0] + c->rope_axes[1] + c->rope_axes[2] != c->head_dim) return false;
  for (int i = 0; i < 3; ++i)
    if (c->rope_axes[i] < 0 || c->rope_axes[i] % 2) return false;
  if (!(c->norm_eps > 0.f) || !(c->rope_theta > 0.f)) return false;
  if (c->flags & ~15u) return false;
  return true;
}

struct BlockWs {
  float* mod;           // [B, 4D]
  __nv_bfloat16* a;     // [T, D]
  __nv_bfloat16* qkvh;  // [T, max(3D, F)]
  __nv_bfloat16* o;     // [T, D]
  __nv_bfloat16* y;     // [T, D] projection output before the sandwich norm
  int* bands;           // [2 ceil(T / 256)] arrival counters of the out / down projections
};

size_t carve_block(Carver& c, BlockWs* ws, int64_t T, int B, int D, int F) {
  const int64_t wide = 3 * (int64_t)D > F ? 3 * (int64_t)D : F;
  BlockWs w;
  w.mod = c.take<float>((size_t)B * 4 * D);
  w.a = c.take<__nv_bfloat16>((size_t)T * D);
  w.qkvh = c.take<__nv_bfloat16>((size_t)T * wide);
  w.o = c.take<__nv_bfloat16>((size_t)T * D);
  w.y = c.take<__nv_bfloat16>((size_t)T * D);
  w.bands = c.take<int>((size_t)(T + 255) / 256 * 2);  // one per 128-row half of every 256-row pair tile
  if (ws) *ws = w;
  return c.off;
}

bool varlen_ok(const zdit_varlen* v) {
  if (v == nullptr || v->batch <= 0 || v->batch > kMaxBatch || !v->cu_seqlens_dev || !v->cu_seqlens_host)
    return false;
  if (v->cu_seqlens_host[0] != 0) return false;
  for (int b = 0; b < v->batch; ++b)
    if (v->cu_seqlens_host[b + 1] <= v->cu_seqlens_host[b]) return false;
  return true;
}

inline bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

// Band counters of one forward: zeroed when the token count changes, then every
// projection that signals them adds num_n arrivals per band, so the k-th one of the
// run is complete for a band at k * num_n.  A BandState lives for one block or stack
// call only (T starts at -1), so every call re-zeroes the counters in its workspace
// before the first projection that signals them: a reused workspace (the static
// scratch of zdit_block_forward_static included) never carries stale counts into the
// next call.  Caching a BandState across calls would break that.
struct BandState {
  int T = -1;
  int epoch = 0;
};

// Next block's pre-attention norm, fused into this block's last residual kernel.
struct NextNorm {
  const float* w;      // next block's n_attn
  const float* scale;  // next block's scale_attn [B, 4D] base (nullptr without adaLN)
};

// The block's launch sequence.  `mod` holds the adaLN vectors [B, 4D] (ignored
// without ADALN).  a_ready: ws.a already holds this block's pre-attention operand
// (written by the previous block's fused residual); next: fuse the next block's
// pre-attention norm into the final residual kernel.
zdit_status run_block(const zdit_block_cfg& cfg, const zdit_block_weights& w, const zdit_varlen& vl, int T,
                      float* x, const float* mod, const float* rcos, const float* rsin, const BlockWs& ws,
                      cudaStream_t s, BandState* band, bool a_ready = false, const NextNorm* next = nullptr) {
  const int D = cfg.dim, F = cfg.ffn_hidden, B = vl.batch;
  const bool adaln = cfg.flags & ZDIT_F_ADALN;
  const bool sandwich = cfg.flags & ZDIT_F_SANDWICH_NORM;
  const bool qkn = cfg.flags & ZDIT_F_QK_NORM;
  const float* s1 = adaln ? mod : nullptr;
  const float* g1 = adaln ? mod + D : nullptr;
  const float* s2 = adaln ? mod + 2 * D : nullptr;
  const float* g2 = adaln ? mod + 3 * D : nullptr;
  const int ms = 4 * D;
  // The residual kernels start band by band while their projection finishes (needs the
  // pair GEMM, and programmatic launches so the residual grid is resident early; off
  // under the event profiler, which times kernels one by one).
  const bool banded = band != nullptr && ws.bands != nullptr && gemm_uses_pair(T, D) && !profiling_on() &&
                      pdl_enabled();
  const int band_step = D / 256;  // arrivals per band per projection (N = D output tiles)
  if (banded && band->T != T) {
    if (cudaMemsetAsync(ws.bands, 0, (size_t)(T + 255) / 256 * 2 * sizeof(int), s) != cudaSuccess)
      return ZDIT_ERR_CUDA;
    band->T = T;
    band->epoch = 0;
  }

  // pre-attention norm + modulation -> bf16 operand
  if (!a_ready)
    launch_norm_modulate_ex(x, T, D, w.n_attn, s1, ms, vl.cu_seqlens_dev, B, 0, 0, cfg.norm_eps, ws.a, s);

  // QKV projection with (QK-norm +) RoPE epilogue -> [T, 3D] bf16
  GemmArgs g{};
  g.A = ws.a; g.lda = D; g.B = w.w_qkv; g.ldb = D; g.M = T; g.N = 3 * D; g.K = D;
  g.epi = EPI_QKV; g.out = ws.qkvh; g.ldo = 3 * D; g.rope_cos = rcos; g.rope_sin = rsin; g.dim = D;
  g.prof_kind = PROF_GEMM_QKV; g.qn = qkn ? w.n_q : nullptr; g.kn = qkn ? w.n_k : nullptr; g.eps = cfg.norm_eps;
  zdit_status st = launch_gemm(g, s);
  if (st != ZDIT_OK) return st;

  // joint attention over each branch segment
  AttnArgs at{};
  at.q = ws.qkvh; at.k = ws.qkvh + D; at.v = ws.qkvh + 2 * D;
  at.ldq = at.ldk = at.ldv = 3 * D; at.o = ws.o; at.ldo = D; at.T = T; at.n_heads = cfg.n_heads; at.batch = B;
  at.cu_seqlens_dev = vl.cu_seqlens_dev; at.cu_seqlens_host = vl.cu_seqlens_host;
  at.scale = 1.0f / sqrtf((float)cfg.head_dim);
  st = launch_attention(at, s);
  if (st != ZDIT_OK) return st;

  // output projection -> y fp32
  GemmArgs go{};
  go.A = ws.o; go.lda = D; go.B = w.w_out; go.ldb = D; go.M = T; go.N = D; go.K = D;
  go.epi = EPI_BF16; go.out = ws.y; go.ldo = D; go.prof_kind = PROF_GEMM_OUT;
  go.band_flags = banded ? ws.bands : nullptr;
  st = launch_gemm(go, s);
  if (st != ZDIT_OK) return st;

  // x += g1 * PostNorm(y), fused with the pre-FFN norm + modulation
  ResidArgs r{};
  r.x = x; r.y = ws.y; r.T = T; r.D = D; r.post_w = sandwich ? w.n_attn_post : nullptr;
  r.gate = g1; r.gate_stride = ms; r.tanh_gate = (cfg.flags & ZDIT_F_TANH_GATE) ? 1 : 0;
  r.cu_seqlens = vl.cu_seqlens_dev; r.batch = B; r.eps = cfg.norm_eps;
  r.next_w = w.n_ffn; r.next_scale = s2; r.next_scale_stride = ms; r.next_out = ws.a;
  r.band_flags = banded ? ws.bands : nullptr;
  r.band_target = banded ? ++band->epoch * band_step : 0;
  launch_residual(r, s);

  // gate/up projection with SwiGLU epilogue -> h bf16 [T, F]
  GemmArgs gu{};
  gu.A = ws.a; gu.lda = D; gu.B = w.w_gate_up; gu.ldb = D; gu.M = T; gu.N = 2 * F; gu.K = D;
  gu.epi = EPI_SWIGLU; gu.out = ws.qkvh; gu.ldo = F; gu.prof_kind = PROF_GEMM_GATE_UP;
  st = launch_gemm(gu, s);
  if (st != ZDIT_OK) return st;

  // down projection -> y fp32
  GemmArgs gd{};
  gd.A = ws.qkvh; gd.lda = F; gd.B = w.w_down; gd.ldb = F; gd.M = T; gd.N = D; gd.K = F;
  gd.epi = EPI_BF16; gd.out = ws.y; gd.ldo = D; gd.prof_kind = PROF_GEMM_DOWN;
  gd.band_flags = banded ? ws.bands : nullptr;
  st = launch_gemm(gd, s);
  if (st != ZDIT_OK) return st;

  // x += g2 * PostNorm(y)
  ResidArgs r2 = r;
  r2.post_w = sandwich ? w.n_ffn_post : nullptr;
  r2.gate = g2;
  r2.band_target = banded ? ++band->epoch * band_step : 0;
  if (next != nullptr) {
    r2.next_w = next->w; r2.next_scale = next->scale; r2.next_out = ws.a;
  } else {
    r2.next_w = nullptr; r2.next_scale = nullptr; r2.next_out = nullptr;
  }
  launch_residual(r2, s);
  return cudaGetLastError() == cudaSuccess ? ZDIT_OK : ZDIT_ERR_CUDA;
}

bool block_weights_ok(const zdit_block_cfg& cfg, const zdit_block_weights& w) {
  if (!w.w_qkv || !w.w_out || !w.w_gate_up || !w.w_down || !w.n_attn || !w.n_ffn) return false;
  if ((cfg.flags & ZDIT_F_ADALN) && (!w.w_ada || !w.b_ada)) return false;
  if ((cfg.flags & ZDIT_F_SANDWICH_NORM) && (!w.n_attn_post || !w.n_ffn_post)) return false;
  if ((cfg.flags & ZDIT_F_QK_NORM) && (!w.n_q || !w.n_k)) return false;
  const void* ptrs[] = {w.w_qkv, w.w_out, w.w_gate_up, w.w_down, w.w_ada, w.b_ada, w.n_attn,
                        w.n_attn_post, w.n_ffn, w.n_ffn_post, w.n_q, w.n_k};
  for (const void* p : ptrs)
    if (p && !al16(p)) return false;
  return true;
}

// ------------------------------------------------------------------ stack workspace
struct StackWs {
  int* pos_img;
  int* pos_cap;
  int* pos_joint;
  int* cu_img;
  int* cu_cap;
  int* cu_joint;
  float *cos_img, *sin_img, *cos_cap, *sin_cap, *cos_joint, *sin_joint;
  float* temb;
  float* mods;   // [n_blocks][B * 4D]
  float* fmod;   // [B, D]
  float* x_img;
  float* x_cap;
  float* x_joint;
  __nv_bfloat16* patches16;
  __nv_bfloat16* caps16;
  BlockWs blk;
};

struct StackDims {
  int B, n_img, T_img, T_cap, T, D, F, E, nblk, cap_dim, patch_dim;
  int n_cap[kMaxBatch], n_valid[kMaxBatch];
  int cu_img[kMaxBatch + 1], cu_cap[kMaxBatch + 1], cu_joint[kMaxBatch + 1], cap_off[kMaxBatch + 1];
};

bool stack_dims(const zdit_stack_cfg* cfg, const zdit_stack_inputs* in, StackDims* d) {
  if (!cfg || !in || !cfg_ok(&cfg->block)) return false;
  if (in->batch <= 0 || in->batch > kMaxBatch || in->grid_h <= 0 || in->grid_w <= 0) return false;
  if (!in->n_cap || !in->n_valid) return false;
  if (cfg->n_noise_refiner < 0 || cfg->n_context_refiner < 0 || cfg->n_main < 0) return false;
  if (cfg->n_noise_refiner + cfg->n_context_refiner + cfg->n_main > kMaxBlocks) return false;
  if (cfg->patch_dim <= 0 || cfg->patch_dim % 64 || cfg->cap_dim <= 0 || cfg->cap_dim % 64 || cfg->cap_dim > 8192)
    return false;
  d->B = in->batch;
  d->n_img = in->grid_h * in->grid_w;
  if (d->n_img % 32) return false;
  d->D = cfg->block.dim;
  d->F = cfg->block.ffn_hidden;
  d->E = cfg->block.temb_dim;
  d->nblk = cfg->n_noise_refiner + cfg->n_context_refiner + cfg->n_main;
  d->cap_dim = cfg->cap_dim;
  d->patch_dim = cfg->patch_dim;
  d->cu_img[0] = d->cu_cap[0] = d->cu_joint[0] = d->cap_off[0] = 0;
  for (int b = 0; b < d->B; ++b) {
    const int c = in->n_cap[b], v = in->n_valid[b];
    if (c < 32 || c % 32 || v < 0 || v > c) return false;
    d->n_cap[b] = c;
    d->n_valid[b] = v;
    d->cu_img[b + 1] = d->cu_img[b] + d->n_img;
    d->cu_cap[b + 1] = d->cu_cap[b] + c;
    d->cu_joint[b + 1] = d->cu_joint[b] + d->n_img + c;
    d->cap_off[b + 1] = d->cap_off[b] + v;
  }
  d->T_img = d->cu_img[d->B];
  d->T_cap = d->cu_cap[d->B];
  d->T = d->cu_joint[d->B];
  return true;
}

size_t carve_stack(Carver& c, StackWs* ws, const StackDims& d) {
  StackWs w;
  const int hd2 = 64;
  w.pos_img = c.take<int>((size_t)d.T_img * 3);
  w.pos_cap = c.take<int>((size_t)d.T_cap * 3);
  w.pos_joint = c.take<int>((size_t)d.T * 3);
  w.cu_img = c.take<int>(kMaxBatch + 1);
  w.cu_cap = c.take<int>(kMaxBatch + 1);
  w.cu_joint = c.take<int>(kMaxBatch + 1);
  w.cos_img = c.take<float>((size_t)d.T_img * hd2);
  w.sin_img = c.take<float>((size_t)d.T_img * hd2);
  w.cos_cap = c.take<float>((size_t)d.T_cap * hd2);
  w.sin_cap = c.take<float>((size_t)d.T_cap * hd2);
  w.cos_joint = c.take<float>((size_t)d.T * hd2);
  w.sin_joint = c.take<float>((size_t)d.T * hd2);
  w.temb = c.take<float>((size_t)d.B * d.E);
  w.mods = c.take<float>((size_t)(d.nblk > 0 ? d.nblk : 1) * d.B * 4 * d.D);
  w.fmod = c.take<float>((size_t)d.B * d.D);
  w.x_img = c.take<float>((size_t)d.T_img * d.D);
  w.x_cap = c.take<float>((size_t)d.T_cap * d.D);
  w.x_joint = c.take<float>((size_t)d.T * d.D);
  w.patches16 = c.take<__nv_bfloat16>((size_t)d.T_img * d.patch_dim);
  w.caps16 = c.take<__nv_bfloat16>((size_t)d.T_cap * d.cap_dim);
  carve_block(c, &w.blk, d.T, d.B, d.D, d.F);
  if (ws) *ws = w;
  return c.off;
}

// The stack's launch sequence.  opts.context_ready: ws.x_cap already holds the
// refined caption stream of these captions (the context refiner has no adaLN, so it
// does not depend on t); opts.dedup_noise: every branch reads the same patch tokens
// with the same t, so the noise refiner runs once on branch 0 and its result serves
// all branches (the image tokens of a branch differ only in the axis-0 position,
// whose rotation cancels in q.k).
struct StackOpts {
  bool context_ready = false;
  bool dedup_noise = false;
};

zdit_status stack_run(const zdit_stack_cfg* cfg, const zdit_stack_weights* w, const zdit_stack_inputs* in,
                      const StackDims& d, const StackWs& ws, float* out, const StackOpts& opts, cudaStream_t s) {
  const int D = d.D, B = d.B, E = d.E;
  const zdit_block_cfg& bcfg = cfg->block;

  // token layout: positions and segment offsets of the three sequences
  launch_stack_layout(d.n_cap, B, in->grid_h, in->grid_w, ws.pos_img, ws.pos_cap, ws.pos_joint, ws.cu_img,
                      ws.cu_cap, ws.cu_joint, s);
  launch_rope_table(ws.pos_img, d.T_img, 128, bcfg.rope_axes, bcfg.rope_theta, ws.cos_img, ws.sin_img, s);
  launch_rope_table(ws.pos_cap, d.T_cap, 128, bcfg.rope_axes, bcfg.rope_theta, ws.cos_cap, ws.sin_cap, s);
  launch_rope_table(ws.pos_joint, d.T, 128, bcfg.rope_axes, bcfg.rope_theta, ws.cos_joint, ws.sin_joint, s);

  // timestep embedding and every adaLN vector of the forward
  launch_timestep_embed(in->t, B, E, cfg->t_scale, static_cast<const __nv_bfloat16*>(w->w_t1), w->b_t1,
                        static_cast<const __nv_bfloat16*>(w->w_t2), w->b_t2, ws.temb, s);
  {
    // every adaLN projection of the forward in one launch
    const __nv_bfloat16* Ws[kMaxBlocks];
    const float* bs[kMaxBlocks];
    float* outs[kMaxBlocks];
    int nm = 0;
    for (int i = 0; i < d.nblk && (bcfg.flags & ZDIT_F_ADALN); ++i) {
      const bool ctx = i >= cfg->n_noise_refiner && i < cfg->n_noise_refiner + cfg->n_context_refiner;
      if (ctx) continue;
      Ws[nm] = static_cast<const __nv_bfloat16*>(w->blocks[i].w_ada);
      bs[nm] = w->blocks[i].b_ada;
      outs[nm] = ws.mods + (size_t)i * B * 4 * D;
      ++nm;
    }
    if (nm > 0) launch_gemv_batched(Ws, bs, outs, nm, ws.temb, B, E, 4 * D, s);
  }
  launch_gemv(static_cast<const __nv_bfloat16*>(w->w_fada), w->b_fada, ws.temb, B, E, D, ws.fmod, s);

  // image embedder: patches -> bf16 -> Linear(patch_dim, D) + bias
  const int B_img = opts.dedup_noise ? 1 : B;  // branches whose image stream is computed
  for (int b = 0; b < B_img; ++b)
    launch_cast_bf16(in->patches + (in->shared_patches ? 0 : (size_t)b * d.n_img * d.patch_dim),
                     ws.patches16 + (size_t)b * d.n_img * d.patch_dim, (int64_t)d.n_img * d.patch_dim, s);
  GemmArgs gx{};
  gx.A = ws.patches16; gx.lda = d.patch_dim; gx.B = w->w_x; gx.ldb = d.patch_dim; gx.M = B_img * d.n_img; gx.N = D;
  gx.K = d.patch_dim; gx.epi = EPI_F32; gx.out = ws.x_img; gx.ldo = D; gx.bias = w->b_x;
  zdit_status st = launch_gemm(gx, s);
  if (st != ZDIT_OK) return st;

  // caption embedder: RMSNorm(valid rows) -> Linear(cap_dim, D) + bias; pads <- pad_vec
  if (!opts.context_ready) {
  if (cudaMemsetAsync(ws.caps16, 0, (size_t)d.T_cap * d.cap_dim * sizeof(__nv_bfloat16), s) != cudaSuccess)
    return ZDIT_ERR_CUDA;
  for (int b = 0; b < B; ++b)
    if (d.n_valid[b] > 0)
      launch_norm_modulate_ex(in->cap_feats + (size_t)d.cap_off[b] * d.cap_dim, d.n_valid[b], d.cap_dim,
                              w->w_capnorm, nullptr, 0, nullptr, 1, 0, 0, bcfg.norm_eps,
                              ws.caps16 + (size_t)d.cu_cap[b] * d.cap_dim, s);
  GemmArgs gc{};
  gc.A = ws.caps16; gc.lda = d.cap_dim; gc.B = w->w_cap; gc.ldb = d.cap_dim; gc.M = d.T_cap; gc.N = D;
  gc.K = d.cap_dim; gc.epi = EPI_F32; gc.out = ws.x_cap; gc.ldo = D; gc.bias = w->b_cap;
  st = launch_gemm(gc, s);
  if (st != ZDIT_OK) return st;
  for (int b = 0; b < B; ++b)
    launch_fill_rows(ws.x_cap + (size_t)(d.cu_cap[b] + d.n_valid[b]) * D, D, d.n_cap[b] - d.n_valid[b],
                     w->pad_vec, s);
  }

  // refiners
  BandState band;
  zdit_varlen v_img{B_img, ws.cu_img, d.cu_img};
  zdit_varlen v_cap{B, ws.cu_cap, d.cu_cap};
  zdit_varlen v_joint{B, ws.cu_joint, d.cu_joint};
  for (int i = 0; i < d.nblk; ++i) {
    const bool noise = i < cfg->n_noise_refiner;
    const bool ctx = !noise && i < cfg->n_noise_refiner + cfg->n_context_refiner;
    if (!noise && !ctx) continue;
    if (ctx && opts.context_ready) continue;
    zdit_block_cfg bc = bcfg;
    if (ctx) bc.flags &= ~ZDIT_F_ADALN;
    const float* mod = ws.mods + (size_t)i * B * 4 * D;
    st = noise ? run_block(bc, w->blocks[i], v_img, B_img * d.n_img, ws.x_img, mod, ws.cos_img, ws.sin_img, ws.blk, s,
                           &band)
               : run_block(bc, w->blocks[i], v_cap, d.T_cap, ws.x_cap, mod, ws.cos_cap, ws.sin_cap, ws.blk, s, &band);
    if (st != ZDIT_OK) return st;
  }
  // concatenate each branch as [image | caption]
  for (int b = 0; b < B; ++b) {
    if (cudaMemcpyAsync(ws.x_joint + (size_t)d.cu_joint[b] * D, ws.x_img + (size_t)(opts.dedup_noise ? 0 : d.cu_img[b]) * D,
                        (size_t)d.n_img * D * sizeof(float), cudaMemcpyDeviceToDevice, s) != cudaSuccess)
      return ZDIT_ERR_CUDA;
    if (cudaMemcpyAsync(ws.x_joint + (size_t)(d.cu_joint[b] + d.n_img) * D, ws.x_cap + (size_t)d.cu_cap[b] * D,
                        (size_t)d.n_cap[b] * D * sizeof(float), cudaMemcpyDeviceToDevice, s) != cudaSuccess)
      return ZDIT_ERR_CUDA;
  }
  // main blocks; each one's last residual kernel also produces the next block's
  // pre-attention operand
  const int first_main = cfg->n_noise_refiner + cfg->n_context_refiner;
  const bool adaln = bcfg.flags & ZDIT_F_ADALN;
  for (int i = first_main; i < d.nblk; ++i) {
    NextNorm nn{};
    const bool has_next = i + 1 < d.nblk;
    if (has_next) {
      nn.w = w->blocks[i + 1].n_attn;
      nn.scale = adaln ? ws.mods + (size_t)(i + 1) * B * 4 * D : nullptr;
    }
    st = run_block(bcfg, w->blocks[i], v_joint, d.T, ws.x_joint, ws.mods + (size_t)i * B * 4 * D, ws.cos_joint,
                   ws.sin_joint, ws.blk, s, &band, i > first_main, has_next ? &nn : nullptr);
    if (st != ZDIT_OK) return st;
  }
  // final layer on the image rows of each branch
  for (int b = 0; b < B; ++b) {
    launch_norm_modulate_ex(ws.x_joint + (size_t)d.cu_joint[b] * D, d.n_img, D, nullptr, ws.fmod + (size_t)b * D, 0,
                            nullptr, 1, 0, 1, cfg->final_eps, ws.blk.a, s);
    GemmArgs gf{};
    gf.A = ws.blk.a; gf.lda = D; gf.B = w->w_final; gf.ldb = D; gf.M = d.n_img; gf.N = d.patch_dim; gf.K = D;
    gf.epi = EPI_F32; gf.out = out + (size_t)b * d.n_img * d.patch_dim; gf.ldo = d.patch_dim; gf.bias = w->b_final;
    st = launch_gemm(gf, s);
    if (st != ZDIT_OK) return st;
  }
  return cudaGetLastError() == cudaSuccess ? ZDIT_OK : ZDIT_ERR_CUDA;
}

}  // namespace
}  // namespace zdit

namespace zdit {

zdit_status check_block_call(const zdit_block_cfg* cfg, const zdit_block_weights* w, const zdit_varlen* varlen,
                             const float* x, const float* temb, const float* rope_cos, const float* rope_sin,
                             const void* workspace, bool with_workspace) {
  if (!cfg || !w || !varlen || !x || !rope_cos || !rope_sin || (with_workspace && !workspace))
    return ZDIT_ERR_INVALID_ARG;
  if (!cfg_ok(cfg) || !varlen_ok(varlen)) return ZDIT_ERR_SHAPE;
  if (!block_weights_ok(*cfg, *w)) return ZDIT_ERR_INVALID_ARG;
  if ((cfg->flags & ZDIT_F_ADALN) && !temb) return ZDIT_ERR_INVALID_ARG;
  if (!al16(x) || !al16(rope_cos) || !al16(rope_sin) ||
      (with_workspace && (reinterpret_cast<uintptr_t>(workspace) & 255)))
    return ZDIT_ERR_ALIGNMENT;
  if (!device_ok()) return ZDIT_ERR_UNSUPPORTED;
  return ZDIT_OK;
}

}  // namespace zdit

using namespace zdit;

extern "C" {

ZDIT_API int32_t zdit_version(void) { return 200; }

ZDIT_API const char* zdit_status_string(zdit_status s) {
  switch (s) {
    case ZDIT_OK: return "ZDIT_OK";
    case ZDIT_ERR_INVALID_ARG: return "ZDIT_ERR_INVALID_ARG";
    case ZDIT_ERR_SHAPE: return "ZDIT_ERR_SHAPE";
    case ZDIT_ERR_ALIGNMENT: return "ZDIT_ERR_ALIGNMENT";
    case ZDIT_ERR_WORKSPACE: return "ZDIT_ERR_WORKSPACE";
    case ZDIT_ERR_UNSUPPORTED: return "ZDIT_ERR_UNSUPPORTED";
    case ZDIT_ERR_CUDA: return "ZDIT_ERR_CUDA";
    case ZDIT_ERR_DEVICE_TIMEOUT: return "ZDIT_ERR_DEVICE_TIMEOUT";
  }
  return "ZDIT_ERR_UNKNOWN";
}

ZDIT_API size_t zdit_block_workspace_bytes(const zdit_block_cfg* cfg, int64_t total_tokens, int32_t batch) {
  if (!cfg_ok(cfg) || total_tokens <= 0 || batch <= 0 || batch > kMaxBatch) return 0;
  Carver c(nullptr);
  return carve_block(c, nullptr, total_tokens, batch, cfg->dim, cfg->ffn_hidden);
}

ZDIT_API zdit_status zdit_block_forward(const zdit_block_cfg* cfg, const zdit_block_weights* w,
                                        const zdit_varlen* varlen, float* x, const float* temb,
                                        const float* rope_cos, const float* rope_sin, void* workspace,
                                        size_t workspace_bytes, void* stream) {
  const zdit_status v = check_block_call(cfg, w, varlen, x, temb, rope_cos, rope_sin, workspace, true);
  if (v != ZDIT_OK) return v;
  const int T = varlen->cu_seqlens_host[varlen->batch];
  const size_t need = zdit_block_workspace_bytes(cfg, T, varlen->batch);
  if (workspace_bytes < need) return ZDIT_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  Carver c(workspace);
  BlockWs ws;
  carve_block(c, &ws, T, varlen->batch, cfg->dim, cfg->ffn_hidden);
  if (cfg->flags & ZDIT_F_ADALN)
    launch_gemv(static_cast<const __nv_bfloat16*>(w->w_ada), w->b_ada, temb, varlen->batch, cfg->temb_dim,
                4 * cfg->dim, ws.mod, s);
  BandState band;
  return run_block(*cfg, *w, *varlen, T, x, ws.mod, rope_cos, rope_sin, ws, s, &band);
}

ZDIT_API size_t zdit_stack_workspace_bytes(const zdit_stack_cfg* cfg, const zdit_stack_inputs* in) {
  StackDims d;
  if (!stack_dims(cfg, in, &d)) return 0;
  Carver c(nullptr);
  return carve_stack(c, nullptr, d);
}

// Host-side checks shared by zdit_stack_forward and zdit_sample.
zdit_status stack_validate(const zdit_stack_cfg* cfg, const zdit_stack_weights* w, const zdit_stack_inputs* in,
                           const float* out, void* workspace, StackDims* d) {
  if (!cfg || !w || !in || !out || !workspace || !in->patches || !in->t) return ZDIT_ERR_INVALID_ARG;
  if (!stack_dims(cfg, in, d)) return ZDIT_ERR_SHAPE;
  if (d->nblk > 0 && !w->blocks) return ZDIT_ERR_INVALID_ARG;
  if (d->cap_off[d->B] > 0 && !in->cap_feats) return ZDIT_ERR_INVALID_ARG;
  const void* req[] = {w->w_x, w->b_x, w->w_capnorm, w->w_cap, w->b_cap, w->pad_vec, w->w_t1, w->b_t1,
                       w->w_t2, w->b_t2, w->w_fada, w->b_fada, w->w_final, w->b_final};
  for (const void* p : req)
    if (!p) return ZDIT_ERR_INVALID_ARG;
  for (const void* p : req)
    if (!al16(p)) return ZDIT_ERR_ALIGNMENT;
  if (!al16(out) || !al16(in->patches) || (in->cap_feats && !al16(in->cap_feats)) ||
      (reinterpret_cast<uintptr_t>(workspace) & 255))
    return ZDIT_ERR_ALIGNMENT;
  for (int i = 0; i < d->nblk; ++i) {
    zdit_block_cfg bc = cfg->block;
    if (i >= cfg->n_noise_refiner && i < cfg->n_noise_refiner + cfg->n_context_refiner) bc.flags &= ~ZDIT_F_ADALN;
    if (!block_weights_ok(bc, w->blocks[i])) return ZDIT_ERR_INVALID_ARG;
  }
  if (!device_ok()) return ZDIT_ERR_UNSUPPORTED;
  return ZDIT_OK;
}

ZDIT_API zdit_status zdit_stack_forward(const zdit_stack_cfg* cfg, const zdit_stack_weights* w,
                                        const zdit_stack_inputs* in, float* out, void* workspace,
                                        size_t workspace_bytes, void* stream) {
  StackDims d;
  const zdit_status v = stack_validate(cfg, w, in, out, workspace, &d);
  if (v != ZDIT_OK) return v;
  Carver c0(nullptr);
  if (workspace_bytes < carve_stack(c0, nullptr, d)) return ZDIT_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  Carver c(workspace);
  StackWs ws;
  carve_stack(c, &ws, d);
  return stack_run(cfg, w, in, d, ws, out, StackOpts{}, s);
}

namespace {
size_t carve_sample(Carver& c, StackWs* ws, float** z, float** vel, const StackDims& d) {
  carve_stack(c, ws, d);
  float* zz = c.take<float>((size_t)d.n_img * d.patch_dim);
  float* vv = c.take<float>((size_t)d.B * d.n_img * d.patch_dim);
  if (z) *z = zz;
  if (vel) *vel = vv;
  return c.off;
}

// stack inputs of the sampler: the latent tokens are shared by every branch
bool sample_inputs(const zdit_stack_inputs* in, zdit_stack_inputs* in2, float* t_host, const void* some_device_ptr) {
  if (!in || in->batch <= 0 || in->batch > kMaxBatch) return false;
  *in2 = *in;
  for (int b = 0; b < in->batch; ++b) t_host[b] = 0.f;
  in2->t = t_host;
  in2->patches = static_cast<const float*>(some_device_ptr);
  in2->shared_patches = 1;
  return true;
}
}  // namespace

}  // extern "C"

namespace zdit {
namespace {

// The sampler's launch sequence: patchify, n_steps x (stack forward + CFG-Euler update),
// unpatchify.  Inputs are validated by the caller.
zdit_status sample_run(const zdit_stack_cfg* cfg, const zdit_stack_weights* w, const zdit_stack_inputs* in,
                       const zdit_sample_cfg* sc, float* latent, void* workspace, const StackDims& d,
                       zdit_stack_inputs& in2, float* t_host, cudaStream_t s) {
  Carver c(workspace);
  StackWs ws;
  float *z = nullptr, *vel = nullptr;
  carve_sample(c, &ws, &z, &vel, d);
  in2.patches = z;
  const int C = d.patch_dim / 4;
  const int64_t n = (int64_t)d.n_img * d.patch_dim;
  launch_patchify(latent, z, C, in->grid_h, in->grid_w, 0, s);
  StackOpts opts;
  opts.dedup_noise = sc->dedup_noise != 0 && d.B > 1;
  for (int i = 0; i < sc->n_steps; ++i) {
    // sigma_i = 3(1-u)/(3(1-u)+u), u = i / n_steps; the DiT sees t = 1 - sigma_i
    const double u0 = (double)i / sc->n_steps, u1 = (double)(i + 1) / sc->n_steps;
    const float s0 = (float)(3.0 * (1.0 - u0) / (3.0 * (1.0 - u0) + u0));
    const float s1 = (float)(3.0 * (1.0 - u1) / (3.0 * (1.0 - u1) + u1));
    for (int b = 0; b < d.B; ++b) t_host[b] = 1.0f - s0;
    opts.context_ready = sc->cache_context != 0 && i > 0;
    zdit_status st = stack_run(cfg, w, &in2, d, ws, vel, opts, s);
    if (st != ZDIT_OK) return st;
    launch_euler_cfg(z, vel, d.B > 1 ? vel + n : nullptr, n, sc->guidance, s1 - s0, s);
  }
  launch_patchify(z, latent, C, in->grid_h, in->grid_w, 1, s);
  return cudaGetLastError() == cudaSuccess ? ZDIT_OK : ZDIT_ERR_CUDA;
}

// Unique id of the current CUDA context (cuCtxGetId: ids are never reused within a
// process), 0 when it cannot be read.  Handles cached across calls (the sampler's graph and
// capture stream) belong to one context and are not reused after it is destroyed and
// created again.
unsigned long long current_context_id() {
  using GetCurrent = CUresult (*)(CUcontext*);
  using GetId = CUresult (*)(CUcontext, unsigned long long*);
  static GetCurrent get_current = nullptr;
  static GetId get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<GetCurrent>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<GetId>(p);
  });
  CUcontext c = nullptr;
  unsigned long long id = 0;
  if (get_current == nullptr || get_id == nullptr || get_current(&c) != CUDA_SUCCESS || c == nullptr ||
      get_id(c, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

// One cached executable graph of the sampler (zdit_sample_cfg.use_graph).
struct SampleGraph {
  std::mutex mu;
  std::vector<uint8_t> key;
  cudaGraphExec_t exec = nullptr;
  unsigned long long exec_context = 0;  // context the graph belongs to
  int64_t launches = 0;
  cudaStream_t capture_stream = nullptr;
  unsigned long long stream_context = 0;  // context the capture stream belongs to
};

SampleGraph& sample_graph() {
  static SampleGraph* g = new SampleGraph();  // never destroyed: outlives the CUDA context at exit
  return *g;
}

}  // namespace
}  // namespace zdit

extern "C" {

ZDIT_API size_t zdit_sample_workspace_bytes(const zdit_stack_cfg* cfg, const zdit_stack_inputs* in) {
  float t_host[kMaxBatch];
  zdit_stack_inputs in2;
  if (!sample_inputs(in, &in2, t_host, reinterpret_cast<const void*>(256))) return 0;
  StackDims d;
  if (!stack_dims(cfg, &in2, &d)) return 0;
  Carver c(nullptr);
  return carve_sample(c, nullptr, nullptr, nullptr, d);
}

ZDIT_API zdit_status zdit_sample(const zdit_stack_cfg* cfg, const zdit_stack_weights* w,
                                 const zdit_stack_inputs* in, const zdit_sample_cfg* sc, float* latent,
                                 void* workspace, size_t workspace_bytes, void* stream) {
  if (!sc || !latent || !in) return ZDIT_ERR_INVALID_ARG;
  if (sc->n_steps <= 0 || sc->n_steps > 1000 || in->batch > 2) return ZDIT_ERR_SHAPE;
  float t_host[kMaxBatch];
  zdit_stack_inputs in2;
  if (!sample_inputs(in, &in2, t_host, latent)) return ZDIT_ERR_SHAPE;
  StackDims d;
  const zdit_status v = stack_validate(cfg, w, &in2, latent, workspace, &d);
  if (v != ZDIT_OK) return v;
  if (d.patch_dim % 4) return ZDIT_ERR_SHAPE;
  Carver c0(nullptr);
  if (workspace_bytes < carve_sample(c0, nullptr, nullptr, nullptr, d)) return ZDIT_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (!sc->use_graph || profiling_on()) return sample_run(cfg, w, in, sc, latent, workspace, d, in2, t_host, s);
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(s, &cap) != cudaSuccess) return ZDIT_ERR_CUDA;
  if (cap != cudaStreamCaptureStatusNone)  // the caller is capturing: just add our launches
    return sample_run(cfg, w, in, sc, latent, workspace, d, in2, t_host, s);
  // key: every argument that shapes the launch sequence
  std::vector<uint8_t> key;
  auto put = [&key](const void* p, size_t n) {
    const uint8_t* b = static_cast<const uint8_t*>(p);
    key.insert(key.end(), b, b + n);
  };
  // the context, not only the device: after a context is destroyed its graph is not reused
  const unsigned long long ctx = current_context_id();
  if (ctx == 0) return sample_run(cfg, w, in, sc, latent, workspace, d, in2, t_host, s);
  put(&ctx, sizeof(ctx));
  put(cfg, sizeof(*cfg));
  put(w, sizeof(*w));
  put(w->blocks, sizeof(zdit_block_weights) * (size_t)(cfg->n_noise_refiner + cfg->n_context_refiner + cfg->n_main));
  put(&in->batch, sizeof(in->batch));
  put(&in->grid_h, sizeof(in->grid_h));
  put(&in->grid_w, sizeof(in->grid_w));
  put(in->n_cap, sizeof(int32_t) * (size_t)in->batch);
  put(in->n_valid, sizeof(int32_t) * (size_t)in->batch);
  put(&in->cap_feats, sizeof(in->cap_feats));
  put(sc, sizeof(*sc));
  put(&latent, sizeof(latent));
  put(&workspace, sizeof(workspace));
  put(&workspace_bytes, sizeof(workspace_bytes));
  SampleGraph& g = sample_graph();
  std::lock_guard<std::mutex> lock(g.mu);
  if (g.exec == nullptr || g.key != key) {
    // capture on a private stream (the caller's may be the legacy default stream, which
    // cannot capture); nothing runs during capture, the graph is then launched on `s`
    if (g.capture_stream == nullptr || g.stream_context != ctx) {
      // a stream of another context is left alone: it may no longer exist
      if (cudaStreamCreateWithFlags(&g.capture_stream, cudaStreamNonBlocking) != cudaSuccess) {
        g.capture_stream = nullptr;
        return ZDIT_ERR_CUDA;
      }
      g.stream_context = ctx;
    }
    cudaStream_t cs = g.capture_stream;
    const int64_t before = zdit_launch_count();
    if (cudaStreamBeginCapture(cs, cudaStreamCaptureModeRelaxed) != cudaSuccess) return ZDIT_ERR_CUDA;
    const zdit_status st = sample_run(cfg, w, in, sc, latent, workspace, d, in2, t_host, cs);
    cudaGraph_t graph = nullptr;
    const cudaError_t ce = cudaStreamEndCapture(cs, &graph);
    if (st != ZDIT_OK || ce != cudaSuccess || graph == nullptr) {
      if (graph != nullptr) cudaGraphDestroy(graph);
      return st != ZDIT_OK ? st : ZDIT_ERR_CUDA;
    }
    cudaGraphExec_t exec = nullptr;
    const cudaError_t ie = cudaGraphInstantiate(&exec, graph, 0);
    cudaGraphDestroy(graph);
    if (ie != cudaSuccess) return ZDIT_ERR_CUDA;
    if (g.exec != nullptr && g.exec_context == ctx) cudaGraphExecDestroy(g.exec);
    g.exec = exec;
    g.exec_context = ctx;
    g.key = key;
    g.launches = zdit_launch_count() - before;  // counted once at capture, once per replay below
    return cudaGraphLaunch(g.exec, s) == cudaSuccess ? ZDIT_OK : ZDIT_ERR_CUDA;
  }
  add_launches(g.launches);
  return cudaGraphLaunch(g.exec, s) == cudaSuccess ? ZDIT_OK : ZDIT_ERR_CUDA;
}

ZDIT_API zdit_status zdit_euler_cfg_step(float* x, const float* v_pos, const float* v_neg, int64_t n, float g,
                                         float sigma_cur, float sigma_next, void* stream) {
  if (!x || !v_pos || n < 0) return ZDIT_ERR_INVALID_ARG;
  if (!al16(x) || !al16(v_pos) || (v_neg && !al16(v_neg))) return ZDIT_ERR_ALIGNMENT;
  if (n == 0) return ZDIT_OK;
  if (!device_ok()) return ZDIT_ERR_UNSUPPORTED;
  launch_euler_cfg(x, v_pos, v_neg, n, g, sigma_next - sigma_cur, static_cast<cudaStream_t>(stream));
  return cudaGetLastError() == cudaSuccess ? ZDIT_OK : ZDIT_ERR_CUDA;
}

ZDIT_API zdit_status zdit_sigma_schedule(int32_t n_steps, float* sigmas) {
  if (n_steps <= 0 || !sigmas) return ZDIT_ERR_INVALID_ARG;
  for (int i = 0; i <= n_steps; ++i) {
    const double u = (double)i / n_steps;
    sigmas[i] = (float)(3.0 * (1.0 - u) / (3.0 * (1.0 - u) + u));
  }
  return ZDIT_OK;
}

ZDIT_API zdit_status zdit_rope_table(const int32_t* pos, int64_t T, int32_t head_dim, const int32_t rope_axes[3],
                                     float theta, float* cos_out, float* sin_out, void* stream) {
  if (!pos || !rope_axes || !cos_out || !sin_out || T < 0 || !(theta > 0.f)) return ZDIT_ERR_INVALID_ARG;
  if (head_dim <= 0 || head_dim % 2 || head_dim > 1024 || rope_axes[0] + rope_axes[1] + rope_axes[2] != head_dim)
    return ZDIT_ERR_SHAPE;
  for (int i = 0; i < 3; ++i)
    if (rope_axes[i] < 0 || rope_axes[i] % 2) return ZDIT_ERR_SHAPE;
  if (T == 0) return ZDIT_OK;
  if (!device_ok()) return ZDIT_ERR_UNSUPPORTED;
  launch_rope_table(pos, T, head_dim, rope_axes, theta, cos_out, sin_out, static_cast<cudaStream_t>(stream));
  return cudaGetLastError() == cudaSuccess ? ZDIT_OK : ZDIT_ERR_CUDA;
}

ZDIT_API zdit_status zdit_joint_attention(const void* q, int32_t ldq, const void* k, int32_t ldk, const void* v,
                                          int32_t ldv, void* o, int32_t ldo, const zdit_varlen* varlen,
                                          int32_t n_heads, int32_t head_dim, void* stream) {
  if (!q || !k || !v || !o || !varlen) return ZDIT_ERR_INVALID_ARG;
  if (head_dim != 128 || n_heads <= 0 || !varlen_ok(varlen)) return ZDIT_ERR_SHAPE;
  const int64_t HD = (int64_t)n_heads * head_dim;
  if (ldq < HD || ldk < HD || ldv < HD || ldo < HD) return ZDIT_ERR_SHAPE;
  if (!device_ok()) return ZDIT_ERR_UNSUPPORTED;
  AttnArgs a{};
  a.q = q; a.k = k; a.v = v; a.ldq = ldq; a.ldk = ldk; a.ldv = ldv; a.o = o; a.ldo = ldo;
  a.T = varlen->cu_seqlens_host[varlen->batch]; a.n_heads = n_heads; a.batch = varlen->batch;
  a.cu_seqlens_dev = varlen->cu_seqlens_dev; a.cu_seqlens_host = varlen->cu_seqlens_host;
  a.scale = 1.0f / sqrtf((float)head_dim);
  return launch_attention(a, static_cast<cudaStream_t>(stream));
}

ZDIT_API zdit_status zdit_adaln_project(const void* const* w_ada, const float* const* b_ada, float* const* out,
                                        int32_t n_mat, const float* temb, int32_t batch, int32_t temb_dim,
                                        int32_t rows, void* stream) {
  if (!w_ada || !out || !temb) return ZDIT_ERR_INVALID_ARG;
  if (n_mat <= 0 || n_mat > kMaxBlocks || batch <= 0 || batch > kMaxBatch || rows <= 0 || temb_dim <= 0 ||
      temb_dim % 8 || temb_dim > 1024)
    return ZDIT_ERR_SHAPE;
  for (int i = 0; i < n_mat; ++i) {
    if (!w_ada[i] || !out[i]) return ZDIT_ERR_INVALID_ARG;
    if (!al16(w_ada[i]) || (reinterpret_cast<uintptr_t>(out[i]) & 3) ||
        (b_ada && b_ada[i] && (reinterpret_cast<uintptr_t>(b_ada[i]) & 3)))
      return ZDIT_ERR_ALIGNMENT;
  }
  if (!al16(temb)) return ZDIT_ERR_ALIGNMENT;
  if (!device_ok()) return ZDIT_ERR_UNSUPPORTED;
  const float* bias[kMaxBlocks];
  for (int i = 0; i < n_mat; ++i) bias[i] = b_ada ? b_ada[i] : nullptr;
  launch_gemv_batched(reinterpret_cast<const __nv_bfloat16* const*>(w_ada), bias, out, n_mat, temb, batch, temb_dim,
                      rows, static_cast<cudaStream_t>(stream));
  return cudaGetLastError() == cudaSuccess ? ZDIT_OK : ZDIT_ERR_CUDA;
}

ZDIT_API zdit_status zdit_gemm_bf16(const void* A, const void* B, float* C, int64_t M, int64_t N, int64_t K,
                                    int64_t ldc, const float* bias, void* stream) {
  if (!A || !B || !C) return ZDIT_ERR_INVALID_ARG;
  if (M <= 0 || N <= 0 || K <= 0 || M > (1 << 30) || N > (1 << 30) || K > (1 << 30) || ldc < N)
    return ZDIT_ERR_SHAPE;
  if (bias && !al16(bias)) return ZDIT_ERR_ALIGNMENT;
  if (!device_ok()) return ZDIT_ERR_UNSUPPORTED;
  GemmArgs g{};
  g.A = A; g.B = B; g.M = (int)M; g.N = (int)N; g.K = (int)K; g.lda = (int)K; g.ldb = (int)K;
  g.epi = EPI_F32; g.out = C; g.ldo = (int)ldc; g.bias = bias;
  return launch_gemm(g, static_cast<cudaStream_t>(stream));
}

ZDIT_API zdit_status zdit_patchify(const float* latent, float* tokens, int32_t channels, int32_t height,
                                   int32_t width, void* stream) {
  if (!latent || !tokens) return ZDIT_ERR_INVALID_ARG;
  if (channels <= 0 || height <= 0 || width <= 0 || height % 2 || width % 2) return ZDIT_ERR_SHAPE;
  if (!device_ok()) return ZDIT_ERR_UNSUPPORTED;
  launch_patchify(latent, tokens, channels, height / 2, width / 2, 0, static_cast<cudaStream_t>(stream));
  return cudaGetLastError() == cudaSuccess ? ZDIT_OK : ZDIT_ERR_CUDA;
}

ZDIT_API zdit_status zdit_unpatchify(const float* tokens, float* latent, int32_t channels, int32_t height,
                                     int32_t width, void* stream) {
  if (!latent || !tokens) return ZDIT_ERR_INVALID_ARG;
  if (channels <= 0 || height <= 0 || width <= 0 || height % 2 || width % 2) return ZDIT_ERR_SHAPE;
  if (!device_ok()) return ZDIT_ERR_UNSUPPORTED;
  launch_patchify(tokens, latent, channels, height / 2, width / 2, 1, static_cast<cudaStream_t>(stream));
  return cudaGetLastError() == cudaSuccess ? ZDIT_OK : ZDIT_ERR_CUDA;
}

ZDIT_API zdit_status zdit_device_status(void* stream) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return ZDIT_ERR_CUDA;
  if (cudaGetLastError() != cudaSuccess) return ZDIT_ERR_CUDA;
  return read_and_clear_device_error();
}

}  // extern "C"
