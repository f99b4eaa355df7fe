// Internal interfaces between the C-ABI layer and the kernel translation units.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "../../include/zdit.h"

namespace zdit {

// ---------------------------------------------------------------- launch accounting
enum ProfKind : int {
  PROF_GEMM_QKV = 0, PROF_GEMM_OUT, PROF_GEMM_GATE_UP, PROF_GEMM_DOWN, PROF_GEMM_OTHER,
  PROF_ATTENTION, PROF_NORM_MOD, PROF_RESIDUAL, PROF_GEMV, PROF_EULER, PROF_ROPE, PROF_MISC,
  PROF_NUM_KINDS
};

// Counts one kernel launch; when profiling is on, brackets it with CUDA events on
// stream `s` (construct just before the launch, destroy just after).
class ProfScope {
 public:
  ProfScope(int kind, double flops, double bytes, cudaStream_t s);
  ~ProfScope();
  ProfScope(const ProfScope&) = delete;
  ProfScope& operator=(const ProfScope&) = delete;

 private:
  int kind_;
  double flops_, bytes_;
  cudaStream_t s_;
  cudaEvent_t a_ = nullptr, b_ = nullptr;
  bool active_ = false;
};

// ---------------------------------------------------------------- GEMM (tcgen05)
// C[M, N] = A[M, K] . B[N, K]^T with bf16 A, B (both K-major, row-major in memory)
// and an fp32 accumulator in TMEM, followed by one of the fused epilogues.
enum GemmEpilogue : int {
  EPI_F32 = 0,     // out fp32 [M, ldo] = acc (+ bias[n])
  EPI_BF16 = 1,    // out bf16 [M, ldo] = acc (+ bias[n])
  EPI_QKV = 2,     // out bf16 [M, 3D]; columns < 2D: optional per-head RMSNorm, then RoPE
  EPI_SWIGLU = 3,  // out bf16 [M, N/2]; tile columns [gate 128 | up 128] -> silu(g) * u
  EPI_QKV_NORM = 4,  // EPI_QKV with per-head RMSNorm of q and k before RoPE (selected when qn != null)
};

struct GemmArgs {
  const void* A;  // bf16 [M, K], row stride lda elements
  const void* B;  // bf16 [N, K], row stride ldb elements
  int M, N, K, lda, ldb;
  int epi;
  void* out;
  int ldo;
  const float* bias;      // [N] or nullptr (EPI_F32 / EPI_BF16)
  const float* rope_cos;  // [M, 64] (EPI_QKV)
  const float* rope_sin;
  int dim;                // D (EPI_QKV): columns < 2D are q | k
  const float* qn;        // [128] per-head RMSNorm weights (EPI_QKV, optional)
  const float* kn;
  float eps;
  int prof_kind = PROF_GEMM_OTHER;
  // Optional per-128-row-band arrival counters: every CTA of the pair kernel adds 1 to
  // the counter of its 128 output rows once they are stored (num_n arrivals per band
  // per launch), so a row consumer can start on a band before the whole GEMM ends.
  // Only honoured on the pair path (gemm_uses_pair).
  int* band_flags = nullptr;
};

zdit_status launch_gemm(const GemmArgs& a, cudaStream_t s);
bool gemm_uses_pair(int M, int N);

// ---------------------------------------------------------------- attention
struct AttnArgs {
  const void* q;  // bf16 [T, ldq] ; head h at columns h*128 .. h*128+127
  const void* k;
  const void* v;
  int ldq, ldk, ldv;  // row strides in elements
  void* o;            // bf16 [T, ldo]
  int ldo;
  int T, n_heads, batch;
  const int* cu_seqlens_dev;   // [batch + 1]
  const int* cu_seqlens_host;  // [batch + 1]
  float scale;                 // 1 / sqrt(head_dim)
};
zdit_status launch_attention(const AttnArgs& a, cudaStream_t s);

// ---------------------------------------------------------------- row / small kernels
struct RowModArgs {
  const float* x;        // [T, D]
  int T, D;
  const float* w;        // [D] norm weight
  const float* mod;      // per-branch modulation base or nullptr; scale at mod[b*mod_stride + d]
  int mod_stride;
  const int* cu_seqlens; // [B + 1] device (branch of each row)
  int batch;
  float eps;
  __nv_bfloat16* out;    // [T, D]
};
void launch_norm_modulate(const RowModArgs& a, cudaStream_t s);

struct ResidArgs {
  float* x;              // [T, D] in/out residual stream
  const __nv_bfloat16* y;  // [T, D] projection output (bf16)
  int T, D;
  const float* post_w;   // sandwich norm weight or nullptr (no post-norm)
  const float* gate;     // per-branch gate: gate[b*gate_stride + d], or nullptr (gate 1)
  int gate_stride;
  int tanh_gate;
  const int* cu_seqlens;
  int batch;
  float eps;
  // optional fused next pre-norm: a = RMS(x_new) * w_next * (1 + scale_next[b])
  const float* next_w;
  const float* next_scale;
  int next_scale_stride;
  __nv_bfloat16* next_out;
  // Optional: instead of waiting for the whole producing GEMM, row t waits until
  // band_flags[t / 128] >= band_target (that GEMM's counters, see GemmArgs).
  const int* band_flags = nullptr;
  int band_target = 0;
};
void launch_residual(const ResidArgs& a, cudaStream_t s);


// Host-side argument checks of one block call, in the order zdit_block_forward runs
// them (null pointers, cfg and varlen shapes, weights, temb, alignment, device);
// with_workspace adds the caller workspace (non-null, 256-byte aligned).
zdit_status check_block_call(const zdit_block_cfg* cfg, const zdit_block_weights* w, const zdit_varlen* varlen,
                             const float* x, const float* temb, const float* rope_cos, const float* rope_sin,
                             const void* workspace, bool with_workspace);

int num_sms();
// true while zdit_profile_begin .. zdit_profile_end is recording
bool profiling_on();
// adds n to the launch counter (kernels replayed from a captured graph)
void add_launches(int64_t n);

// Device address of the library's latched device-error word on the current device.
int* device_error_ptr();

// ---------------------------------------------------------------- dependent launches
// The per-block chain (GEMMs, attention, residual and norm kernels) is launched with
// programmatic stream serialization: each of these kernels lets its successor launch
// once all its CTAs have started (griddep_trigger after its prologue), and waits for its
// predecessor's completion and memory (griddep_wait) before its first global access, so a
// successor's launch, barrier setup, TMEM allocation and descriptor prefetch overlap the
// predecessor's last wave.  ZDIT_PDL=0 in the environment turns it off.
bool pdl_enabled();

__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

template <typename... KArgs, typename... Args>
cudaError_t launch_dependent(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                             Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = pdl_enabled() ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

}  // namespace zdit
