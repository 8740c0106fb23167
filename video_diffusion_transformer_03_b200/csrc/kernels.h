// Internal launcher interface between the C ABI (h3b_api.cu) and the kernel translation
// units.  Not part of the public ABI.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace h3b {

using bf16 = __nv_bfloat16;

// Per-device facts the launchers need.
struct DevCtx {
  int device;
  int num_sms;
  uint32_t* err_flag;  // device address of this device's wait-timeout flag
};

// Record a message for h3b_last_error (thread-local) and return `code`.
int set_error(int code, const char* fmt, ...);

// Check the launch that just happened; returns 0 or H3B_ECUDA with a message.
int check_launch(const char* what);

// ---------------------------------------------------------------- GEMM (tcgen05)
enum GemmEpi : int {
  kEpiBias = 0,       // out = bf16(acc + bias)
  kEpiGelu = 1,       // out = bf16(gelu_tanh(acc + bias))
  kEpiRope = 2,       // out = bf16(rope(acc + bias)) on columns < rope_cols
  kEpiGateResid = 3,  // out = bf16(out + gate * (acc + bias))
  kEpiInt8Deq = 4,    // int8 path: out = bf16(out + gate * (acc * row_scale * col_scale + bias))
  // LN-folded forms: A is the raw bf16 residual x and B the AdaLN-folded weights W'
  // (launch_fold_adaln); pre = rstd_r (acc - mean_r c_j) + dv_j with the row statistics
  // merged from stats_in, then the base epilogue
  kEpiRopeLN = 5,     // out = bf16(rope(pre)) on columns < rope_cols
  kEpiGeluLN = 6,     // out = bf16(gelu_tanh(pre))
  kEpiHeadEuler = 7,  // out_f32 += euler_dt * pre (fp32 state, in place): a final head
  // int8 operands with one scale per A row (row_scale [M]) and per B row (col_scale [N]):
  // pre = (float(acc) * row_scale) * col_scale + bias_f32, then the base epilogue
  kEpiI8Rope = 8,     // out = bf16(rope(pre)) on columns < rope_cols
  kEpiI8Gelu = 9,     // out = bf16(gelu_tanh(pre))
  // grouped int8 (launch_gemm_i8_grouped): acc is the fp32 sum over K groups of
  // float(acc_g) * row_scale[m, g]; out = bf16(out + gate * (acc * col_scale + bias_f32))
  kEpiI8GroupGate = 10,
};

// The base epilogue of a kind (the LN-folded kinds share their base's arithmetic).
__host__ __device__ constexpr int epi_base(int k) {
  return (k == kEpiRopeLN || k == kEpiI8Rope) ? kEpiRope
         : (k == kEpiGeluLN || k == kEpiI8Gelu) ? kEpiGelu
                                                 : k;
}
// Kinds whose accumulator is int32 with row and column scales.
__host__ __device__ constexpr bool epi_int8(int k) {
  return k == kEpiInt8Deq || k == kEpiI8Rope || k == kEpiI8Gelu;
}
// Kinds that add a gated branch to the residual held in `out`.
__host__ __device__ constexpr bool epi_gated(int k) {
  return k == kEpiGateResid || k == kEpiInt8Deq || k == kEpiI8GroupGate;
}
__host__ __device__ constexpr bool epi_ln_fold(int k) {
  return k == kEpiRopeLN || k == kEpiGeluLN || k == kEpiHeadEuler;
}

struct GemmEpilogue {
  int kind = kEpiBias;
  const bf16* bias = nullptr;        // bf16 paths, [N]
  const float* bias_f32 = nullptr;   // int8 path, [N] or null
  const float* gate = nullptr;       // [N]
  const float* rope_cs = nullptr;    // [M, head_dim/2, 2]
  int rope_cols = 0;
  int head_dim = 128;
  bf16* out = nullptr;               // [M, ld_out]
  int ld_out = 0;
  const float* row_scale = nullptr;  // int8 path, [M]
  const float* col_scale = nullptr;  // int8 path, [N]
  int32_t* acc_out = nullptr;        // int8 path, [M, N] or null
  // kEpiGateResid, kEpiBias: per row, (mean, M2) of each 256-column group of the stored
  // bf16 output, [M, ld_out / 256]; or null
  float2* stats_out = nullptr;
  // kEpiHeadEuler: the fp32 state [M, ld_out] updated in place, and the Euler step
  float* out_f32 = nullptr;
  float euler_dt = 0.f;
  // LN-folded kinds: the A rows' group statistics [M, stats_parts], the folded weights'
  // row sums c [N] (dv [N] comes in bias_f32) and the LayerNorm epsilon
  const float2* stats_in = nullptr;
  const float* fold_c = nullptr;
  int stats_parts = 0;
  float ln_eps = 1e-6f;
  // RoPE kinds: per-head RMSNorm of q (columns < rope_cols / 2) and k (up to rope_cols)
  // before the rotation, gains [head_dim] each (eps = ln_eps); both null = off.  Runs
  // data-parallel (the norm needs the whole head from one accumulator).
  const float* q_gain = nullptr;
  const float* k_gain = nullptr;
  // kEpiI8GroupGate: groups of 1024 K columns; row_scale is [M, act_groups]
  int act_groups = 0;
};

// Kernel scratch: one caller buffer per stream, used by one kernel at a time.  Layout:
//   [0, kSkFlagsOffset)                 partial tiles: the GEMM's stream-K slots
//                                       ([CTA][128][256] words), or the attention's split
//                                       query tiles ([CTA][head_dim/4][128] float4, then
//                                       [CTA][128] (m, l) pairs)
//   [kSkFlagsOffset, kAttnFlagsOffset)  GEMM flags, [CTA][8 epilogue warps]
//   [kAttnFlagsOffset, kScratchBytes)   attention flags, [CTA][4 softmax warps]
// A flag holds the launch's sequence number (next_scratch_seq) once the 32 partial rows
// of that warp are written, and is put back to zero by the reader.
constexpr int kMaxSkCtas = 160;  // grid cap of the split schedules
constexpr size_t kSkFlagsOffset = size_t(kMaxSkCtas) * 128 * 256 * 4;
constexpr size_t kAttnFlagsOffset = kSkFlagsOffset + size_t(kMaxSkCtas) * 8 * 8;
constexpr size_t kScratchBytes = kAttnFlagsOffset + size_t(kMaxSkCtas) * 4 * 8;

// Bytes of kernel scratch (kScratchBytes).
size_t gemm_scratch_bytes();
// A value no flag can hold from an earlier launch of this process.
unsigned long long next_scratch_seq();
// Host enumeration of one scheduling unit's GEMM work items (h3b_gemm_schedule).
int gemm_schedule_items(int tiles, int k_blocks, int units, int mode, int unit, int* items,
                        int max_items);
// Process-wide GEMM dispatch overrides (h3b_set_gemm_override); -1 on bad values.
int set_gemm_override(int tile, int sched, int trans);

// out = A[M, K] * B[N, K]^T with epilogue; bf16 inputs.  K % 64 == 0, N % 128 == 0.
// scratch (>= gemm_scratch_bytes(), or null) enables the stream-K schedule when the
// tile count quantises badly onto the SMs.
int launch_gemm_bf16(const DevCtx& ctx, const bf16* A, const bf16* B, int M, int N, int K,
                     const GemmEpilogue& epi, void* scratch, size_t scratch_bytes,
                     cudaStream_t stream);
// Same for int8 inputs (int32 accumulate; kEpiInt8Deq, kEpiI8Rope, kEpiI8Gelu).
// K % 128 == 0, N % 128 == 0.
int launch_gemm_i8(const DevCtx& ctx, const int8_t* A, const int8_t* B, int M, int N, int K,
                   const GemmEpilogue& epi, void* scratch, size_t scratch_bytes,
                   cudaStream_t stream);
// Grouped int8 product (kEpiI8GroupGate): one A scale per row and 1024-column group.
// K % 1024 == 0, N % 128 == 0.  scratch (>= gemm_scratch_bytes(), or null) lets a partial
// last wave run stream-K over groups.
int launch_gemm_i8_grouped(const DevCtx& ctx, const int8_t* A, const int8_t* B, int M, int N,
                           int K, const GemmEpilogue& epi, void* scratch, size_t scratch_bytes,
                           cudaStream_t stream);

// ---------------------------------------------------------------- attention (tcgen05)
// scratch (>= gemm_scratch_bytes(), or null) enables the persistent split schedule:
// one CTA per SM, each taking an equal share of the (query tile, KV tile) steps.
int launch_attention(const DevCtx& ctx, const bf16* qkv, int n_tokens, int n_heads,
                     int head_dim, bf16* out, void* scratch, size_t scratch_bytes,
                     cudaStream_t stream);

// Attention form for later launches: 0 automatic (two query tiles per CTA), 1 one tile,
// 2 two tiles; -1 on a bad value.
int set_attention_variant(int v);

// ---------------------------------------------------------------- row kernels
int launch_ln_modulate(const bf16* x, int n, int d, float eps, const float* shift,
                       const float* scale, bf16* h, cudaStream_t stream);
// x_res = bf16(x_state); h = LN(x_res)(1 + scale) + shift
int launch_ln_modulate_from_state(const float* x_state, int n, int d, float eps,
                                  const float* shift, const float* scale, bf16* x_res,
                                  bf16* h, cudaStream_t stream);
// x_res = bf16(x_state) and the (mean, M2) of each 256-column group of its rows,
// stats [n, d / 256] (the row statistics the LN-folded GEMM epilogues consume)
int launch_state_to_residual(const float* x_state, int n, int d, bf16* x_res, float2* stats,
                             cudaStream_t stream);
// (mean, M2) of each 256-column group of the rows of x, stats [n, d / 256]
int launch_row_stats(const bf16* x, int n, int d, float2* stats, cudaStream_t stream);
// W' = bf16(W diag(1 + scale)), c = row sums of W', dv = W shift + b (see k_fold_adaln)
int launch_fold_adaln(const bf16* w, const bf16* b, const float* shift, const float* scale,
                      int n_out, int d, bf16* w_out, float* c_out, float* d_out,
                      cudaStream_t stream);
int launch_final_euler(const bf16* x_l, int n, int n_video, int d, float eps,
                       const float* final_mod, float dt_sigma, float* x_state,
                       cudaStream_t stream);
// final_euler that also stores the velocity and / or the core residual
// r = x_l - bf16(x_state) (either may be null)
int launch_final_euler_keep(const bf16* x_l, int n, int n_video, int d, float eps,
                            const float* final_mod, float dt_sigma, float* x_state, float* v_out,
                            float* r_out, cudaStream_t stream);
// skipped core: x_l = bf16(bf16(x_state) + r_in), then final AdaLN + Euler
int launch_core_reuse_final(const float* r_in, int n, int n_video, int d, float eps,
                            const float* final_mod, float dt_sigma, float* x_state,
                            cudaStream_t stream);
// h = LN(x)(1 + scale) + shift quantised to int8 with one scale per row (q [n, d],
// q_scale [n]); the quantisation rule of launch_quantize_rows
int launch_ln_modulate_q8(const bf16* x, int n, int d, float eps, const float* shift,
                          const float* scale, int8_t* q, float* q_scale, cudaStream_t stream);
// int8 quantisation with one scale per row and 1024-column group: q [rows, cols],
// scale [rows, cols / 1024]; cols % 1024 == 0
int launch_quantize_groups(const bf16* a, int rows, int cols, int8_t* q, float* scale,
                           cudaStream_t stream);
// dst = bf16(src), n elements (n % 8 == 0)
int launch_f32_to_bf16(const float* src, long long n, bf16* dst, cudaStream_t stream);
// x_state += dt * v (n elements, n % 4 == 0)
int launch_euler_axpy(const float* v, long long n, float dt_sigma, float* x_state,
                      cudaStream_t stream);
int launch_token_pair(const bf16* src, bf16* dst, int t, int h, int w, int n_audio, int d,
                      cudaStream_t stream);
int launch_token_unpair(const bf16* src, bf16* dst, const bf16* saved, int t, int h, int w,
                        int n_audio, int d, cudaStream_t stream);
int launch_quantize_rows(const bf16* a, int rows, int cols, int8_t* q, float* scale,
                         cudaStream_t stream);
int launch_adaln_gemv(const bf16* w, const bf16* b, const bf16* c, int n_out, int c_dim,
                      float* out, cudaStream_t stream);
int launch_rope_table(int t, int h, int w, int n_audio, int halved, int paired,
                      int head_dim, const int* split, float theta, float* rope_cs,
                      cudaStream_t stream);

}  // namespace h3b
