/*
 * zdit.h - C ABI of the B200 (sm_100a) single-stream DiT hot path of Z-Image-Turbo.
 *
 * The library computes, on one GPU:
 *   - the single-stream DiT block over one packed caption+image token sequence
 *     (zdit_block_forward),
 *   - the whole DiT: embedders, 2 noise-refiner + 2 context-refiner + 30 main
 *     blocks and the final layer (zdit_stack_forward),
 *   - the fused negated-CFG FlowMatchEuler update (zdit_euler_cfg_step),
 * plus the pieces those are made of, exposed so they can be checked one by one
 * (joint attention, the projection GEMM, RoPE tables, patchify).
 *
 * Sources for what is computed (web pages, by title and section):
 *   [CoreAI] "Z-Image-Turbo port - a 6B diffusion DiT on Core AI, and why it is
 *            Mac-only" (Core AI model zoo): table "Architecture -> export mapping"
 *            (DiT and Sampler rows); "The three things that each cost a wrong image"
 *            (negated CFG, caption pad tokens); "fp16 does not work. bf16 does."
 *            (value ranges); "Hosting it from Swift" (patchify order, schedule).
 *   [Jobs]   "Native creative jobs" (1Cat-vLLM design note), "Recipes and
 *            precision" (FP32 latents, CFG, accumulators, SwiGLU gating).
 *   [Port]   "Z-Image Port Status" (FastVideo), "Pinned Official Pipeline Context"
 *            (sampler contract: endpoint-preserving schedule, no call at sigma 0).
 *
 * Conventions shared by every call:
 *   - Pointers marked "device" are CUDA device pointers on the current device;
 *     "host" pointers are read during the call only.  The caller owns every
 *     buffer; the library never allocates device memory in a compute call.
 *   - Every compute call is asynchronous on the CUDA stream passed as `stream`
 *     (NULL = legacy default stream) and never synchronizes, except
 *     zdit_device_status.
 *   - Arguments are validated on the host before any launch; a failed check
 *     returns an error status and launches nothing.  Nothing is thrown across
 *     the ABI.
 *   - Matrices are row-major.  bf16 = IEEE bfloat16 bit patterns (uint16).
 *     Device pointers handed to GEMMs or attention must be 16-byte aligned and
 *     their row strides multiples of 8 elements (TMA requirement).
 *   - fp16 is never used: activations reach 3.1e5 ([CoreAI] "fp16 does not work").
 *   - Every wait inside a kernel (a pipeline barrier, or a row waiting for its
 *     band of a projection) is bounded: one that exceeds the wait limit abandons
 *     the kernel and latches ZDIT_ERR_DEVICE_TIMEOUT, reported by
 *     zdit_device_status.  The limit is fixed when the library is built
 *     (ZDIT_WAIT_LIMIT_MS, default 2000 ms), one value for every wait: no wait of a
 *     healthy launch comes near it, but a run that is slowed down from outside (a
 *     profiler replaying kernels, a debugger, a GPU shared with a heavy job) could
 *     trip it; build with a larger ZDIT_WAIT_LIMIT_MS for such uses.
 */
#ifndef ZDIT_H_
#define ZDIT_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define ZDIT_API __attribute__((visibility("default")))

typedef enum {
  ZDIT_OK = 0,
  ZDIT_ERR_INVALID_ARG = -1,    /* null pointer, bad flag combination             */
  ZDIT_ERR_SHAPE = -2,          /* unsupported or inconsistent sizes              */
  ZDIT_ERR_ALIGNMENT = -3,      /* pointer or stride not 16-byte aligned          */
  ZDIT_ERR_WORKSPACE = -4,      /* workspace missing or smaller than required     */
  ZDIT_ERR_UNSUPPORTED = -5,    /* device is not sm_100                           */
  ZDIT_ERR_CUDA = -6,           /* a CUDA runtime / driver call failed            */
  ZDIT_ERR_DEVICE_TIMEOUT = -7  /* a kernel gave up on a bounded wait             */
} zdit_status;

/* Block feature flags. */
enum {
  ZDIT_F_ADALN = 1,         /* adaLN modulation from the timestep embedding; when
                               clear the block uses scale 0 and gate 1 (the
                               context refiner has none, [CoreAI] DiT row)      */
  ZDIT_F_SANDWICH_NORM = 2, /* RMSNorm(y) * w_post of each projection output before
                               its gated add (reading of [Jobs]: projection outputs
                               stay in FP32 range until normalized; and of the
                               3.1e5 output vs 6.7e3 residual ranges in [CoreAI]) */
  ZDIT_F_QK_NORM = 4,       /* per-head RMSNorm of q and k before RoPE (option) */
  ZDIT_F_TANH_GATE = 8      /* gate = tanh(adaLN gate chunk) (option)           */
};

/* Dimensions of one block.  Supported: head_dim == 128, dim == n_heads * 128,
 * dim % 256 == 0 (so q, k and v column blocks align with 256-wide GEMM tiles),
 * ffn_hidden % 128 == 0, temb_dim % 8 == 0 and <= 1024,
 * rope_axes[0] + rope_axes[1] + rope_axes[2] == head_dim with every entry even. */
typedef struct {
  int32_t dim;          /* D, model width (3840); n_heads * 128, <= 8192    */
  int32_t n_heads;      /* H (30)                                          */
  int32_t head_dim;     /* 128                                             */
  int32_t ffn_hidden;   /* F, SwiGLU hidden width (10240)                  */
  int32_t temb_dim;     /* E, adaLN input width (256)                      */
  int32_t rope_axes[3]; /* rotary widths per position axis (32, 48, 48)    */
  float norm_eps;       /* RMSNorm epsilon (1e-5)                          */
  float rope_theta;     /* rotary base (10000)                             */
  uint32_t flags;       /* ZDIT_F_*                                        */
} zdit_block_cfg;

/* Weights of one block, all device pointers.  Linear layers store W with the
 * output features as rows: y = a . W^T.
 *   w_ada     bf16 [4D, E]  adaLN; output chunks (scale_attn, gate_attn,
 *                           scale_ffn, gate_ffn), each D wide (NULL if !ADALN)
 *   b_ada     fp32 [4D]
 *   w_qkv     bf16 [3D, D]  rows q | k | v; head h owns rows h*128 .. h*128+127
 *                           of each
 *   w_out     bf16 [D, D]
 *   w_gate_up bf16 [2F, D]  SwiGLU gate (W1) and up (W3) rows interleaved in
 *                           128-row blocks: rows 256j .. 256j+127 are W1 rows
 *                           128j .. 128j+127 and rows 256j+128 .. 256j+255 are
 *                           the W3 rows with the same indices
 *   w_down    bf16 [D, F]   W2
 *   n_attn, n_ffn            fp32 [D] pre-norm weights
 *   n_attn_post, n_ffn_post  fp32 [D] post-projection norm weights (SANDWICH)
 *   n_q, n_k                 fp32 [128] per-head q / k norm weights (QK_NORM)
 */
typedef struct {
  const void* w_ada;
  const float* b_ada;
  const void* w_qkv;
  const void* w_out;
  const void* w_gate_up;
  const void* w_down;
  const float* n_attn;
  const float* n_attn_post;
  const float* n_ffn;
  const float* n_ffn_post;
  const float* n_q;
  const float* n_k;
} zdit_block_weights;

/* Packed variable-length batch: branch b owns tokens [cu[b], cu[b+1]).
 * Tokens of different branches never attend to each other. */
typedef struct {
  int32_t batch;                   /* number of branches B (1..8)          */
  const int32_t* cu_seqlens_dev;   /* device [B + 1], cu[0] = 0, increasing */
  const int32_t* cu_seqlens_host;  /* host copy of the same values          */
} zdit_varlen;

/* Workspace (device bytes) needed by zdit_block_forward for `total_tokens`
 * tokens in `batch` branches; 0 on invalid cfg. */
ZDIT_API size_t zdit_block_workspace_bytes(const zdit_block_cfg* cfg, int64_t total_tokens, int32_t batch);

/* One single-stream DiT block, in place on the residual stream x.
 *   m_b = W_ada temb_b + b_ada  -> (s1, g1, s2, g2)            (ADALN)
 *   a   = RMSNorm(x) * n_attn * (1 + s1_b)                     bf16
 *   q|k|v = a . W_qkv^T; (QK_NORM) q,k <- RMSNorm_head * n_q/k; RoPE(q, k)
 *   o   = per branch, per head softmax(q k^T / sqrt(128)) v     no mask
 *   y   = o . W_out^T; (SANDWICH) y <- RMSNorm(y) * n_attn_post
 *   x  += g1_b * y
 *   a   = RMSNorm(x) * n_ffn * (1 + s2_b)
 *   y   = (silu(a W1^T) * (a W3^T)) . W2^T; (SANDWICH) y <- RMSNorm(y) * n_ffn_post
 *   x  += g2_b * y
 * [CoreAI] DiT row (adaLN, 3-axis RoPE in real interleaved form with
 * precomputed cos/sin, 30 x 128 heads, width 3840); [CoreAI] "The three things",
 * item 3 (caption pad tokens are unmasked context); [Jobs] "Recipes and
 * precision" (FP32 accumulators, SwiGLU gate, residual).
 *   x         device fp32 [T, D], in/out; T = cu_seqlens_host[B]
 *   temb      device fp32 [B, E] (ignored without ADALN)
 *   rope_cos, rope_sin  device fp32 [T, head_dim / 2]: cos / sin of the angle of
 *             pair i of token t (see zdit_rope_table)
 *   workspace device, >= zdit_block_workspace_bytes, 256-byte aligned
 * Errors: ZDIT_ERR_INVALID_ARG (null pointers), ZDIT_ERR_SHAPE (cfg or varlen),
 * ZDIT_ERR_ALIGNMENT, ZDIT_ERR_WORKSPACE, ZDIT_ERR_CUDA (launch failure). */
ZDIT_API zdit_status zdit_block_forward(const zdit_block_cfg* cfg, const zdit_block_weights* w,
                                        const zdit_varlen* varlen, float* x, const float* temb,
                                        const float* rope_cos, const float* rope_sin, void* workspace,
                                        size_t workspace_bytes, void* stream);

/* zdit_block_forward without a caller workspace, for callers that cannot allocate
 * device memory: a plugin running inside a host framework that has already reserved
 * (nearly) all of the GPU for its own pool, so cudaMalloc would fail, or a
 * latency-critical loop that must not pay cudaMalloc's device-wide synchronization.
 * The pages describe no such entry point; it has no counterpart there.
 *   Same arguments and result as zdit_block_forward, minus the workspace.  The
 *   workspace is a 40 MiB device array owned by the library (held on every GPU that
 *   loads the library until the process exits); calls needing more than 40 MiB of
 *   workspace (zdit_block_workspace_bytes) return ZDIT_ERR_WORKSPACE and launch
 *   nothing.  At full width (D 3840, F 10240, two branches) that admits up to 907 tokens,
 *   e.g. the 256px cond/uncond pair (608 tokens, 26.8 MiB).
 *   The call allocates nothing (no cudaMalloc, cudaFree or allocating library call).
 *   Every call looks up the array's device address on the current device
 *   (cudaGetSymbolAddress); the first lookup on a device loads the library's module
 *   that holds the array, so make the first call on each device before any stream
 *   capture.
 *   All calls share the one array and it keeps the previous call's contents: the
 *   block writes every workspace byte it reads, except its per-band arrival
 *   counters, which each call zeroes on its stream before using them.  Calls whose
 *   execution overlaps on the GPU (different streams, or host threads) race on the
 *   array and must be serialized by the caller.
 *   Arguments are checked in the same order as zdit_block_forward; the size check
 *   comes after them.
 * Errors: as zdit_block_forward, plus ZDIT_ERR_WORKSPACE (too many tokens) and
 * ZDIT_ERR_CUDA (address lookup failed). */
ZDIT_API zdit_status zdit_block_forward_static(const zdit_block_cfg* cfg, const zdit_block_weights* w,
                                               const zdit_varlen* varlen, float* x, const float* temb,
                                               const float* rope_cos, const float* rope_sin, void* stream);

/* Whole DiT. */
typedef struct {
  zdit_block_cfg block;      /* shared by all blocks; ADALN is dropped for the
                                context refiner, kept for the others          */
  int32_t n_noise_refiner;   /* 2: adaLN blocks over the image tokens only     */
  int32_t n_context_refiner; /* 2: no-adaLN blocks over the caption tokens only */
  int32_t n_main;            /* 30: blocks over the joint sequence              */
  int32_t patch_dim;         /* 64 = 4 * latent channels                        */
  int32_t cap_dim;           /* caption feature width (2560), <= 8192           */
  float t_scale;             /* timestep scale inside the sinusoid (1000)       */
  float final_eps;           /* final LayerNorm epsilon (1e-6)                  */
} zdit_stack_cfg;

/* Stack weights (device pointers; `blocks` is a HOST array of
 * n_noise_refiner + n_context_refiner + n_main entries in that order).
 *   w_x [D, patch_dim] bf16, b_x [D]             image (x) embedder
 *   w_capnorm [cap_dim] fp32, w_cap [D, cap_dim] bf16, b_cap [D]
 *                                                caption embedder (RMSNorm, Linear)
 *   pad_vec [D] fp32                             learned caption pad token
 *   w_t1 [E, E] bf16, b_t1 [E], w_t2 [E, E] bf16, b_t2 [E]
 *                                                timestep MLP
 *   w_fada [D, E] bf16, b_fada [D]               final-layer modulation
 *   w_final [patch_dim, D] bf16, b_final [patch_dim]  final projection      */
typedef struct {
  const zdit_block_weights* blocks;
  const void* w_x;
  const float* b_x;
  const float* w_capnorm;
  const void* w_cap;
  const float* b_cap;
  const float* pad_vec;
  const void* w_t1;
  const float* b_t1;
  const void* w_t2;
  const float* b_t2;
  const void* w_fada;
  const float* b_fada;
  const void* w_final;
  const float* b_final;
} zdit_stack_weights;

/* Per-call inputs of the stack.  Branch b is laid out [image | caption]:
 * n_img = grid_h * grid_w image tokens, then n_cap[b] caption tokens of which the
 * first n_valid[b] are embedded caption features and the rest the pad token
 * ([CoreAI] "The three things", item 3: pad to round_up(L, 32), unmasked).
 * Positions: caption token k -> (k + 1, 0, 0); image cell (h, w) -> (n_cap + 1, h, w). */
typedef struct {
  int32_t batch;            /* B branches (cond, uncond, ...), 1..8           */
  int32_t grid_h, grid_w;   /* patch grid; n_img = grid_h * grid_w, n_img % 32 == 0 */
  const int32_t* n_cap;     /* host [B], multiples of 32, >= 32               */
  const int32_t* n_valid;   /* host [B], 0 <= n_valid <= n_cap                 */
  const float* patches;     /* device fp32 [B, n_img, patch_dim] patch tokens  */
  const float* cap_feats;   /* device fp32 [sum n_valid, cap_dim], branches concatenated */
  const float* t;           /* host [B] timestep fed to the DiT (t = 1 - sigma) */
  int32_t shared_patches;   /* 1: every branch reads the same [n_img, patch_dim]
                               tokens at `patches` (cond and uncond of one latent);
                               0: patches holds [B, n_img, patch_dim]           */
} zdit_stack_inputs;

ZDIT_API size_t zdit_stack_workspace_bytes(const zdit_stack_cfg* cfg, const zdit_stack_inputs* in);

/* out: device fp32 [B, n_img, patch_dim], the DiT output per branch in patch-token
 * layout.  [CoreAI] DiT row: x-embed + cap-embed, 2 noise-refiner (adaLN) +
 * 2 context-refiner (no adaLN) + 30 main + final.  Errors as zdit_block_forward. */
ZDIT_API zdit_status zdit_stack_forward(const zdit_stack_cfg* cfg, const zdit_stack_weights* w,
                                        const zdit_stack_inputs* in, float* out, void* workspace,
                                        size_t workspace_bytes, void* stream);

/* The 8-step sampler in one call: patchify the latent, then for i < n_steps run the
 * DiT on every branch at t = 1 - sigma_i (sigma_i = 3(1-u)/(3(1-u)+u), u = i/n_steps,
 * ending at sigma = 0 with no call there) and apply the negated-CFG Euler update,
 * then unpatchify ([CoreAI] Sampler row, "The three things", item 2 and "Hosting it
 * from Swift"; [Port] sampler contract).  Branch 0 is the conditional branch, branch
 * 1 (optional) the unconditional one; with one branch the update uses v = -pos.
 *   cache_context: embed and refine the captions once and reuse them for every step
 *     (the context refiner has no adaLN, so it does not depend on t).
 *   dedup_noise: run the noise refiner once for all branches (they share the latent
 *     and t, and their image tokens differ only in the axis-0 position, whose rotation
 *     cancels in q.k); equal to the full computation up to rounding. */
typedef struct {
  int32_t n_steps;        /* sampler updates (8)                         */
  float guidance;         /* g of -(pos + g (pos - neg)); two branches    */
  int32_t cache_context;  /* 1: caption stream computed once             */
  int32_t dedup_noise;    /* 1: noise refiner computed once for branches  */
  int32_t use_graph;      /* 1: the whole launch sequence is captured as one CUDA graph
                             on the first call and replayed while every argument (pointers,
                             sizes, steps, guidance) and the CUDA context stay the same (a
                             context created again captures afresh); not used while the
                             profiler records, nor when the context's id cannot be read
                             (the launches then run directly).  The library keeps one such
                             graph. */
} zdit_sample_cfg;

/* in: batch 1 or 2, grid, n_cap, n_valid, cap_feats as for zdit_stack_forward;
 * patches, t and shared_patches are ignored (the sampler supplies them).
 * latent: device fp32 [patch_dim / 4, 2 grid_h, 2 grid_w], the initial noise on
 * entry and the final latent on return.  Errors as zdit_stack_forward. */
ZDIT_API size_t zdit_sample_workspace_bytes(const zdit_stack_cfg* cfg, const zdit_stack_inputs* in);
ZDIT_API zdit_status zdit_sample(const zdit_stack_cfg* cfg, const zdit_stack_weights* w,
                                 const zdit_stack_inputs* in, const zdit_sample_cfg* sc, float* latent,
                                 void* workspace, size_t workspace_bytes, void* stream);

/* Fused negated CFG + FlowMatchEuler update over n fp32 values (device):
 *   v = -(v_pos + g * (v_pos - v_neg));  x += (sigma_next - sigma_cur) * v
 * v_neg == NULL means a single branch: v = -v_pos (g ignored).
 * [CoreAI] "The three things", item 2 (negated CFG); Sampler row (FlowMatchEuler);
 * [Jobs] "Recipes and precision" (latents and CFG in FP32).  The update is
 * elementwise, so it applies unchanged to patch-token layout.
 * Errors: ZDIT_ERR_INVALID_ARG (null x / v_pos, n < 0), ZDIT_ERR_ALIGNMENT
 * (pointers not 16-byte aligned), ZDIT_ERR_CUDA. */
ZDIT_API zdit_status zdit_euler_cfg_step(float* x, const float* v_pos, const float* v_neg, int64_t n, float g,
                                         float sigma_cur, float sigma_next, void* stream);

/* Host: the n_steps + 1 sigmas sigma_i = 3(1-u)/(3(1-u)+u), u = i / n_steps,
 * ending at exactly 0 ([CoreAI] "Hosting it from Swift"; [Port] scheduler
 * contract).  sigmas: host fp32 [n_steps + 1].  Errors: ZDIT_ERR_INVALID_ARG. */
ZDIT_API zdit_status zdit_sigma_schedule(int32_t n_steps, float* sigmas);

/* Per-token rotary tables: for pair i (0 <= i < head_dim/2) of token t,
 * angle = pos[t, a] * theta^(-2 j / rope_axes[a]), where a is the axis of pair i
 * (pairs [0, axes0/2) -> axis 0, next axes1/2 -> axis 1, rest -> axis 2) and j the
 * pair index inside that axis.  pos: device int32 [T, 3]; cos_out, sin_out:
 * device fp32 [T, head_dim / 2]; head_dim even, at most 1024.  Angles and their
 * cos / sin are computed in double precision and rounded to fp32.  [CoreAI] DiT
 * row (3-axis RoPE, precomputed cos/sin).  Errors: ZDIT_ERR_INVALID_ARG,
 * ZDIT_ERR_SHAPE. */
ZDIT_API zdit_status zdit_rope_table(const int32_t* pos, int64_t T, int32_t head_dim, const int32_t rope_axes[3],
                                     float theta, float* cos_out, float* sin_out, void* stream);

/* Joint attention alone (head_dim 128): for every branch and head,
 * O = softmax(Q K^T / sqrt(128)) V over the branch's tokens, no mask.
 * q, k, v: device bf16 [T, ld*] with head h at columns h*128 .. h*128+127;
 * o: device bf16 [T, ldo].  [CoreAI] DiT row and "The three things", item 3.
 * Errors: ZDIT_ERR_INVALID_ARG, ZDIT_ERR_SHAPE, ZDIT_ERR_ALIGNMENT, ZDIT_ERR_CUDA. */
ZDIT_API zdit_status zdit_joint_attention(const void* q, int32_t ldq, const void* k, int32_t ldk, const void* v,
                                          int32_t ldv, void* o, int32_t ldo, const zdit_varlen* varlen,
                                          int32_t n_heads, int32_t head_dim, void* stream);

/* The adaLN projections of several blocks in one launch (the first step of every block
 * with ADALN; zdit_stack_forward computes all of a forward's at once):
 *   out_i[b, r] = sum_e w_ada_i[r, e] temb[b, e] + b_ada_i[r],  i < n_mat
 * [CoreAI] DiT row (adaLN in the refiners and main blocks); [Jobs] "Recipes and
 * precision" (adaLN scaling in FP32).  Each out_i holds the four D-wide chunks
 * (scale_attn, gate_attn, scale_ffn, gate_ffn) of one block when rows = 4D.
 *   w_ada    host array of n_mat device pointers, each bf16 [rows, temb_dim], 16-byte aligned
 *   b_ada    host array of n_mat device pointers, each fp32 [rows]; the array or an entry may
 *            be NULL (no bias)
 *   out      host array of n_mat device pointers, each fp32 [batch, rows]
 *   temb     device fp32 [batch, temb_dim], 16-byte aligned
 *   n_mat 1..256, batch 1..8, temb_dim a multiple of 8 up to 1024, rows >= 1.
 * The weights are streamed once (HBM-bound); accumulation in FP32.
 * Errors: ZDIT_ERR_INVALID_ARG (null pointers), ZDIT_ERR_SHAPE, ZDIT_ERR_ALIGNMENT. */
ZDIT_API zdit_status zdit_adaln_project(const void* const* w_ada, const float* const* b_ada, float* const* out,
                                        int32_t n_mat, const float* temb, int32_t batch, int32_t temb_dim,
                                        int32_t rows, void* stream);

/* Projection GEMM alone: C[M, N] (fp32, row stride ldc) = A[M, K] . B[N, K]^T
 * (+ bias[N] if non-NULL); A, B device bf16 row-major.  The tensor-core kernel
 * behind every projection of the block.  Requires N % 32 == 0, K % 8 == 0,
 * ldc % 4 == 0.  Errors: ZDIT_ERR_INVALID_ARG, ZDIT_ERR_SHAPE, ZDIT_ERR_ALIGNMENT,
 * ZDIT_ERR_CUDA. */
ZDIT_API zdit_status zdit_gemm_bf16(const void* A, const void* B, float* C, int64_t M, int64_t N, int64_t K,
                                    int64_t ldc, const float* bias, void* stream);

/* Patchify a latent [C, 2h, 2w] (device fp32) into tokens [h*w, 4C] (device fp32),
 * token n = hi * w + wi, feature f = (dy * 2 + dx) * C + c ([CoreAI] "Hosting it
 * from Swift": patchify feature order); zdit_unpatchify is the inverse.
 * Errors: ZDIT_ERR_INVALID_ARG, ZDIT_ERR_SHAPE. */
ZDIT_API zdit_status zdit_patchify(const float* latent, float* tokens, int32_t channels, int32_t height,
                                   int32_t width, void* stream);
ZDIT_API zdit_status zdit_unpatchify(const float* tokens, float* latent, int32_t channels, int32_t height,
                                     int32_t width, void* stream);

/* Per-kernel timing of the library's own launches.
 * zdit_profile_begin(max_records) turns recording on: every kernel launch of the
 * library is bracketed by two CUDA events on the stream it is launched on (at most
 * max_records launches are recorded; later ones are counted but not timed).
 * zdit_profile_end waits for the recorded events, turns recording off and writes
 * one entry per kernel kind that ran (at most max_entries, which must be >= 16):
 * its name, launch count, summed event time in ms, summed algorithmic FLOPs
 * (2 M N K for a GEMM, 4 * 128 * H * sum L^2 for attention) and summed algorithmic
 * DRAM bytes (each input read once, each output written once).  Host-only
 * bookkeeping plus cudaEventRecord; intended for benchmarks, not for CUDA-graph
 * capture.  Errors: ZDIT_ERR_INVALID_ARG, ZDIT_ERR_CUDA. */
typedef struct {
  char name[40];
  int32_t launches;
  double total_ms;
  double flops;
  double bytes;
} zdit_profile_entry;
ZDIT_API zdit_status zdit_profile_begin(int32_t max_records);
ZDIT_API zdit_status zdit_profile_end(zdit_profile_entry* entries, int32_t max_entries, int32_t* n_entries);

/* Number of kernel launches issued by the library since it was loaded. */
ZDIT_API int64_t zdit_launch_count(void);

/* Synchronizes `stream`, then returns (and clears) the first device-side error
 * latched by any kernel of this library (ZDIT_ERR_DEVICE_TIMEOUT), or
 * ZDIT_ERR_CUDA if the stream reports a CUDA error, else ZDIT_OK.
 * The latched error lives in one word per device, shared by every stream and host
 * thread that uses the library on that device: it reports an error of any of their
 * launches, not only of `stream`'s, and reading it clears it for all of them.  Callers
 * that run the library on several streams of one device at once must coordinate who
 * reads it. */
ZDIT_API zdit_status zdit_device_status(void* stream);

/* Health check of the bounded waits used by every pipelined kernel: launches one
 * kernel that waits on a barrier nothing arrives on; after the library's wait limit
 * (ZDIT_WAIT_LIMIT_MS, 2 s by default) it gives up, latches ZDIT_ERR_DEVICE_TIMEOUT (read with
 * zdit_device_status) and writes 2 to *result_dev (device int32; 1 would mean the
 * wait wrongly succeeded).  The context stays usable.  Not part of the DiT path.
 * Errors: ZDIT_ERR_INVALID_ARG, ZDIT_ERR_CUDA. */
ZDIT_API zdit_status zdit_selftest_wait_timeout(int32_t* result_dev, void* stream);

/* Static string naming a status code. */
ZDIT_API const char* zdit_status_string(zdit_status s);

/* ABI version (major * 10000 + minor * 100 + patch). */
ZDIT_API int32_t zdit_version(void);

#ifdef __cplusplus
}
#endif

#endif /* ZDIT_H_ */
