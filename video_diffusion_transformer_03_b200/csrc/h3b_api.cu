// C ABI of the h3b library: argument validation, workspace layout and the order of the
// kernels inside a DiT block and an Euler step.  See include/h3b.h for the contract of
// every entry point.
#include "../../include/h3b.h"
#include "kernels.h"

#include <algorithm>
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <vector>

// Set (first code wins) by any kernel whose bounded wait gave up; one per device.
__device__ uint32_t g_h3b_wait_error = 0u;

// Block workspace of h3b_block_forward_noalloc: a fixed array in the module's device
// image, so that entry point never allocates.  In host code this name only stands for
// the symbol; its device address comes from cudaGetSymbolAddress (per device).
static __device__ __align__(256) uint8_t g_noalloc_ws[H3B_NOALLOC_WORKSPACE_BYTES];

namespace h3b {

namespace {

thread_local char g_last_error[512] = "";
std::atomic<uint64_t> g_launches{0};

bool debug_mode() {
  static const bool on = [] {
    const char* v = std::getenv("H3B_DEBUG");
    return v && v[0] && v[0] != '0';
  }();
  return on;
}

constexpr int kMaxDevices = 64;

// Captured whole denoises of the host entry points (see denoise_graph), per device.
struct DenoiseGraph {
  std::vector<uint8_t> key;
  cudaGraphExec_t exec = nullptr;
};
std::mutex g_graph_mu;
std::vector<DenoiseGraph> g_graphs[kMaxDevices];

// Forget a device's captured denoises: after a wait timed out, the split schedules'
// flags in the workspace may hold a sequence number a replay would reuse.
void drop_graphs(int device) {
  if (device < 0 || device >= kMaxDevices) return;
  std::lock_guard<std::mutex> lock(g_graph_mu);
  for (DenoiseGraph& g : g_graphs[device]) cudaGraphExecDestroy(g.exec);
  g_graphs[device].clear();
}

}  // namespace

int set_error(int code, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  std::vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
  return code;
}

int check_launch(const char* what) {
  g_launches.fetch_add(1, std::memory_order_relaxed);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return set_error(H3B_ECUDA, "%s: launch failed: %s", what, cudaGetErrorString(e));
  if (debug_mode()) {
    e = cudaDeviceSynchronize();
    if (e != cudaSuccess)
      return set_error(H3B_ECUDA, "%s: kernel failed: %s", what, cudaGetErrorString(e));
    uint32_t flag = 0;
    cudaMemcpyFromSymbol(&flag, g_h3b_wait_error, sizeof(flag));
    if (flag) return set_error(H3B_ETIMEOUT, "%s: device wait gave up (code %u)", what, flag);
  }
  return H3B_OK;
}

namespace {

int get_ctx(DevCtx* ctx) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return set_error(H3B_ECUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices) return set_error(H3B_EUNSUPPORTED, "device %d", dev);
  static std::mutex mu;
  static DevCtx cache[kMaxDevices];
  static bool have[kMaxDevices] = {};
  std::lock_guard<std::mutex> lock(mu);
  if (!have[dev]) {
    int major = 0, minor = 0, sms = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (major != 10 || minor != 0)
      return set_error(H3B_EUNSUPPORTED, "device %d is sm_%d%d; this library is built for sm_100a",
                       dev, major, minor);
    void* flag = nullptr;
    e = cudaGetSymbolAddress(&flag, g_h3b_wait_error);
    if (e != cudaSuccess)
      return set_error(H3B_ECUDA, "cudaGetSymbolAddress: %s", cudaGetErrorString(e));
    cache[dev] = DevCtx{dev, sms, static_cast<uint32_t*>(flag)};
    have[dev] = true;
  }
  *ctx = cache[dev];
  return H3B_OK;
}

inline bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline size_t a256(size_t b) { return (b + 255) & ~size_t(255); }

int check_dims(const h3b_dims* d) {
  if (!d) return set_error(H3B_EINVAL, "dims is NULL");
  if (d->head_dim != 64 && d->head_dim != 128)
    return set_error(H3B_EINVAL, "head_dim %d must be 64 or 128", d->head_dim);
  if (d->n_heads <= 0 || d->d != d->n_heads * d->head_dim)
    return set_error(H3B_EINVAL, "d=%d must equal n_heads*head_dim", d->d);
  if (d->d % 256 != 0 || d->d > 4096)
    return set_error(H3B_EINVAL, "d=%d must be a multiple of 256 and <= 4096", d->d);
  if (d->d_ff <= 0 || d->d_ff % 256 != 0)
    return set_error(H3B_EINVAL, "d_ff=%d must be a positive multiple of 256", d->d_ff);
  if (d->c_dim <= 0 || d->c_dim % 8 != 0)
    return set_error(H3B_EINVAL, "c_dim=%d must be a positive multiple of 8", d->c_dim);
  const int* s = d->rope_split;
  if (s[0] < 0 || s[1] < 0 || s[2] < 0 || (s[0] | s[1] | s[2]) & 1 ||
      s[0] + s[1] + s[2] != d->head_dim)
    return set_error(H3B_EINVAL, "rope_split (%d,%d,%d) must be even and sum to head_dim",
                     s[0], s[1], s[2]);
  if (!(d->ln_eps > 0.f) || !(d->rope_theta > 0.f))
    return set_error(H3B_EINVAL, "ln_eps and rope_theta must be positive");
  return H3B_OK;
}

int check_grid(const h3b_grid* g, bool need_even_w) {
  if (!g) return set_error(H3B_EINVAL, "grid is NULL");
  if (g->t < 0 || g->h < 0 || g->w < 0 || g->n_audio < 0)
    return set_error(H3B_EINVAL, "grid sizes must be non-negative");
  if (need_even_w && (g->w & 1)) return set_error(H3B_EINVAL, "w=%d must be even to pair tokens", g->w);
  const long long n = 1LL * g->t * g->h * g->w + g->n_audio;
  if (n > (1LL << 24)) return set_error(H3B_EINVAL, "too many tokens (%lld)", n);
  return H3B_OK;
}

int check_weights(const h3b_block_weights* w) {
  if (!w) return set_error(H3B_EINVAL, "weights NULL");
  const void* p[8] = {w->w_qkv, w->b_qkv, w->w_o, w->b_o, w->w_fc1, w->b_fc1, w->w_fc2, w->b_fc2};
  for (const void* q : p)
    if (!q || !al16(q)) return set_error(H3B_EINVAL, "block weight pointer NULL or not 16-byte aligned");
  if ((w->q_norm == nullptr) != (w->k_norm == nullptr) || (w->q_norm && !al16(w->q_norm)) ||
      (w->k_norm && !al16(w->k_norm)))
    return set_error(H3B_EINVAL, "q_norm and k_norm: both or neither, 16-byte aligned");
  return H3B_OK;
}

bool has_fold(const h3b_block_weights* w) {
  return w->w_qkv_fold && w->c_qkv && w->d_qkv && w->w_fc1_fold && w->c_fc1 && w->d_fc1;
}

int check_fold(const h3b_block_weights* w) {
  if (!has_fold(w)) return set_error(H3B_EINVAL, "folded block weights missing");
  const void* p[6] = {w->w_qkv_fold, w->c_qkv, w->d_qkv, w->w_fc1_fold, w->c_fc1, w->d_fc1};
  for (const void* q : p)
    if (!al16(q)) return set_error(H3B_EINVAL, "folded weight pointer not 16-byte aligned");
  return H3B_OK;
}

size_t activations_bytes(const h3b_dims* d, int n) {
  return a256(size_t(n) * std::max(4 * d->d, d->d_ff) * 2);
}

size_t arena_bytes(const h3b_dims* d, int n) {
  return activations_bytes(d, n) + a256(gemm_scratch_bytes());
}

// Buffers of one block inside the arena: qkv [n, 3d] then attention output [n, d]; the
// MLP hidden activations [n, d_ff] reuse the same bytes once both are dead.  The GEMMs'
// stream-K scratch follows.
struct BlockBufs {
  bf16* qkv;
  bf16* attn;
  bf16* g;
  void* gemm_scratch;
};

BlockBufs carve_block(const h3b_dims* d, int n, void* arena) {
  bf16* base = static_cast<bf16*>(arena);
  return BlockBufs{base, base + size_t(n) * 3 * d->d, base,
                   static_cast<uint8_t*>(arena) + activations_bytes(d, n)};
}

int block_forward_impl(const DevCtx& ctx, const h3b_dims* d, const h3b_block_weights* w,
                       const float* mod, const float* mod_next, const float* rope_cs, int n,
                       bool compute_h, bf16* x, bf16* h, void* arena, cudaStream_t s) {
  const int D = d->d;
  const BlockBufs b = carve_block(d, n, arena);
  int rc;
  if (compute_h && (rc = launch_ln_modulate(x, n, D, d->ln_eps, mod, mod + D, h, s))) return rc;

  GemmEpilogue e;
  e.kind = kEpiRope;
  e.bias = reinterpret_cast<const bf16*>(w->b_qkv);
  e.q_gain = w->q_norm;
  e.k_gain = w->k_norm;
  e.ln_eps = d->ln_eps;
  e.rope_cs = rope_cs;
  e.rope_cols = 2 * D;
  e.head_dim = d->head_dim;
  e.out = b.qkv;
  e.ld_out = 3 * D;
  if ((rc = launch_gemm_bf16(ctx, h, reinterpret_cast<const bf16*>(w->w_qkv), n, 3 * D, D, e, b.gemm_scratch, gemm_scratch_bytes(), s)))
    return rc;
  if ((rc = launch_attention(ctx, b.qkv, n, d->n_heads, d->head_dim, b.attn, b.gemm_scratch,
                             gemm_scratch_bytes(), s)))
    return rc;

  e = GemmEpilogue();
  e.kind = kEpiGateResid;
  e.bias = reinterpret_cast<const bf16*>(w->b_o);
  e.gate = mod + 2 * D;
  e.out = x;
  e.ld_out = D;
  if ((rc = launch_gemm_bf16(ctx, b.attn, reinterpret_cast<const bf16*>(w->w_o), n, D, D, e, b.gemm_scratch, gemm_scratch_bytes(), s)))
    return rc;
  if ((rc = launch_ln_modulate(x, n, D, d->ln_eps, mod + 3 * D, mod + 4 * D, h, s))) return rc;

  e = GemmEpilogue();
  e.kind = kEpiGelu;
  e.bias = reinterpret_cast<const bf16*>(w->b_fc1);
  e.out = b.g;
  e.ld_out = d->d_ff;
  if ((rc = launch_gemm_bf16(ctx, h, reinterpret_cast<const bf16*>(w->w_fc1), n, d->d_ff, D, e, b.gemm_scratch, gemm_scratch_bytes(), s)))
    return rc;

  e = GemmEpilogue();
  e.kind = kEpiGateResid;
  e.bias = reinterpret_cast<const bf16*>(w->b_fc2);
  e.gate = mod + 5 * D;
  e.out = x;
  e.ld_out = D;
  if ((rc = launch_gemm_bf16(ctx, b.g, reinterpret_cast<const bf16*>(w->w_fc2), n, D, d->d_ff, e, b.gemm_scratch, gemm_scratch_bytes(), s)))
    return rc;
  if (mod_next && (rc = launch_ln_modulate(x, n, D, d->ln_eps, mod_next, mod_next + D, h, s)))
    return rc;
  return H3B_OK;
}

// The block with both AdaLN LayerNorms folded into the QKV and FC1 projections: the
// gated-residual epilogues of the out-projection and FC2 write the residual's row
// statistics, which the next folded projection's epilogue applies (no LayerNorm pass).
int block_forward_folded_impl(const DevCtx& ctx, const h3b_dims* d, const h3b_block_weights* w,
                              const float* mod, const float* rope_cs, int n, bf16* x,
                              float2* stats, void* arena, cudaStream_t s) {
  const int D = d->d;
  const BlockBufs b = carve_block(d, n, arena);
  int rc;
  GemmEpilogue e;
  e.kind = kEpiRopeLN;
  e.bias_f32 = w->d_qkv;
  e.fold_c = w->c_qkv;
  e.q_gain = w->q_norm;
  e.k_gain = w->k_norm;
  e.stats_in = stats;
  e.stats_parts = D / 256;
  e.ln_eps = d->ln_eps;
  e.rope_cs = rope_cs;
  e.rope_cols = 2 * D;
  e.head_dim = d->head_dim;
  e.out = b.qkv;
  e.ld_out = 3 * D;
  if ((rc = launch_gemm_bf16(ctx, x, reinterpret_cast<const bf16*>(w->w_qkv_fold), n, 3 * D, D, e,
                             b.gemm_scratch, gemm_scratch_bytes(), s)))
    return rc;
  if ((rc = launch_attention(ctx, b.qkv, n, d->n_heads, d->head_dim, b.attn, b.gemm_scratch,
                             gemm_scratch_bytes(), s)))
    return rc;

  e = GemmEpilogue();
  e.kind = kEpiGateResid;
  e.bias = reinterpret_cast<const bf16*>(w->b_o);
  e.gate = mod + 2 * D;
  e.out = x;
  e.ld_out = D;
  e.stats_out = stats;
  if ((rc = launch_gemm_bf16(ctx, b.attn, reinterpret_cast<const bf16*>(w->w_o), n, D, D, e,
                             b.gemm_scratch, gemm_scratch_bytes(), s)))
    return rc;

  e = GemmEpilogue();
  e.kind = kEpiGeluLN;
  e.bias_f32 = w->d_fc1;
  e.fold_c = w->c_fc1;
  e.stats_in = stats;
  e.stats_parts = D / 256;
  e.ln_eps = d->ln_eps;
  e.out = b.g;
  e.ld_out = d->d_ff;
  if ((rc = launch_gemm_bf16(ctx, x, reinterpret_cast<const bf16*>(w->w_fc1_fold), n, d->d_ff, D,
                             e, b.gemm_scratch, gemm_scratch_bytes(), s)))
    return rc;

  e = GemmEpilogue();
  e.kind = kEpiGateResid;
  e.bias = reinterpret_cast<const bf16*>(w->b_fc2);
  e.gate = mod + 5 * D;
  e.out = x;
  e.ld_out = D;
  e.stats_out = stats;
  return launch_gemm_bf16(ctx, b.g, reinterpret_cast<const bf16*>(w->w_fc2), n, D, d->d_ff, e,
                          b.gemm_scratch, gemm_scratch_bytes(), s);
}

// Buffers of the int8 block after the shared arena: the quantised AdaLN output [n, d] and
// its row scales [n], the quantised GELU output [n, d_ff] and its group scales
// [n, d_ff / 1024].
struct Int8Bufs {
  int8_t* hq;
  float* hs;
  int8_t* gq;
  float* gs;
  size_t total;
};

Int8Bufs carve_int8(const h3b_dims* d, int n, void* base) {
  uint8_t* p = static_cast<uint8_t*>(base);
  Int8Bufs b{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    uint8_t* q = p ? p + off : nullptr;
    off += a256(bytes);
    return q;
  };
  b.hq = reinterpret_cast<int8_t*>(take(size_t(n) * d->d));
  b.hs = reinterpret_cast<float*>(take(size_t(n) * 4));
  b.gq = reinterpret_cast<int8_t*>(take(size_t(n) * d->d_ff));
  b.gs = reinterpret_cast<float*>(take(size_t(n) * (d->d_ff / 1024) * 4));
  b.total = off;
  return b;
}

// The block on the int8 path (dothoosh.com, "The powerful int8 path"): the AdaLN outputs
// quantised per row inside the LayerNorm kernel, int8 QKV and FC1 with per-row and
// per-output-channel scales (RoPE / GELU in their epilogues), the GELU output quantised
// per 1024-channel group, and the grouped int8 FC2 with the gated residual; attention and
// the output projection stay bf16.
int block_forward_int8_impl(const DevCtx& ctx, const h3b_dims* d, const h3b_block_weights* w,
                            const h3b_int8_block* q, const float* mod, const float* rope_cs,
                            int n, bf16* x, void* arena, cudaStream_t s) {
  const int D = d->d;
  const BlockBufs b = carve_block(d, n, arena);
  const Int8Bufs ib = carve_int8(d, n, static_cast<uint8_t*>(arena) + arena_bytes(d, n));
  int rc;
  if ((rc = launch_ln_modulate_q8(x, n, D, d->ln_eps, mod, mod + D, ib.hq, ib.hs, s))) return rc;
  GemmEpilogue e;
  e.kind = kEpiI8Rope;
  e.bias = reinterpret_cast<const bf16*>(w->b_qkv);
  e.row_scale = ib.hs;
  e.col_scale = q->s_qkv;
  e.q_gain = w->q_norm;
  e.k_gain = w->k_norm;
  e.ln_eps = d->ln_eps;
  e.rope_cs = rope_cs;
  e.rope_cols = 2 * D;
  e.head_dim = d->head_dim;
  e.out = b.qkv;
  e.ld_out = 3 * D;
  if ((rc = launch_gemm_i8(ctx, ib.hq, q->w_qkv_q, n, 3 * D, D, e, b.gemm_scratch,
                           gemm_scratch_bytes(), s)))
    return rc;
  if ((rc = launch_attention(ctx, b.qkv, n, d->n_heads, d->head_dim, b.attn, b.gemm_scratch,
                             gemm_scratch_bytes(), s)))
    return rc;
  e = GemmEpilogue();
  e.kind = kEpiGateResid;
  e.bias = reinterpret_cast<const bf16*>(w->b_o);
  e.gate = mod + 2 * D;
  e.out = x;
  e.ld_out = D;
  if ((rc = launch_gemm_bf16(ctx, b.attn, reinterpret_cast<const bf16*>(w->w_o), n, D, D, e,
                             b.gemm_scratch, gemm_scratch_bytes(), s)))
    return rc;
  if ((rc = launch_ln_modulate_q8(x, n, D, d->ln_eps, mod + 3 * D, mod + 4 * D, ib.hq, ib.hs, s)))
    return rc;
  e = GemmEpilogue();
  e.kind = kEpiI8Gelu;
  e.bias = reinterpret_cast<const bf16*>(w->b_fc1);
  e.row_scale = ib.hs;
  e.col_scale = q->s_fc1;
  e.out = b.g;
  e.ld_out = d->d_ff;
  if ((rc = launch_gemm_i8(ctx, ib.hq, q->w_fc1_q, n, d->d_ff, D, e, b.gemm_scratch,
                           gemm_scratch_bytes(), s)))
    return rc;
  if ((rc = launch_quantize_groups(b.g, n, d->d_ff, ib.gq, ib.gs, s))) return rc;
  e = GemmEpilogue();
  e.kind = kEpiI8GroupGate;
  e.bias = reinterpret_cast<const bf16*>(w->b_fc2);
  e.row_scale = ib.gs;
  e.act_groups = d->d_ff / 1024;
  e.col_scale = q->s_fc2;
  e.gate = mod + 5 * D;
  e.out = x;
  e.ld_out = D;
  return launch_gemm_i8_grouped(ctx, ib.gq, q->w_fc2_q, n, D, d->d_ff, e, b.gemm_scratch,
                                gemm_scratch_bytes(), s);
}

// Workspace of one denoise step.
struct StepBufs {
  bf16* x_res;      // [N, d] residual stream (bf16)
  bf16* h;          // [N, d] AdaLN output feeding the next projection
  float* rope;      // [N, hd/2, 2]
  float* rope_red;  // [N_red, hd/2, 2]
  bf16* x_red;      // [N_red, d]
  float2* stats;    // [N, d / 256] row statistics of the residual (folded blocks)
  float2* stats_red;  // [N_red, d / 256]
  bf16* lat;        // [N, c_lat] the latent as the patch embedding's operand (latent steps)
  void* arena;      // block arena sized for N tokens
  size_t total;
};

StepBufs carve_step(const h3b_dims* d, const h3b_grid* g, bool reduce, void* ws,
                    int c_lat = 0) {
  const size_t n = size_t(g->t) * g->h * g->w + g->n_audio;
  const size_t nr = size_t(g->t) * g->h * (g->w / 2) + g->n_audio;
  uint8_t* p = static_cast<uint8_t*>(ws);
  StepBufs b{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    uint8_t* q = p ? p + off : nullptr;
    off += a256(bytes);
    return q;
  };
  b.x_res = reinterpret_cast<bf16*>(take(n * d->d * 2));
  b.h = reinterpret_cast<bf16*>(take(n * d->d * 2));
  b.rope = reinterpret_cast<float*>(take(n * d->head_dim * 4));
  b.stats = reinterpret_cast<float2*>(take(n * (d->d / 256) * sizeof(float2)));
  if (reduce) {
    b.rope_red = reinterpret_cast<float*>(take(nr * d->head_dim * 4));
    b.x_red = reinterpret_cast<bf16*>(take(nr * d->d * 2));
    b.stats_red = reinterpret_cast<float2*>(take(nr * (d->d / 256) * sizeof(float2)));
  }
  if (c_lat > 0) b.lat = reinterpret_cast<bf16*>(take(n * size_t(c_lat) * 2));
  b.arena = take(arena_bytes(d, static_cast<int>(n)));
  b.total = off;
  return b;
}

// The active blocks in their folded form on b.x_res (row statistics in b.stats), with the
// token pairing after `reduce_after` executed blocks and the restore at the end: b.x_res
// then holds x_L.  *stats_valid tells whether b.stats still describes it (not after a
// restore).
int folded_stack(const DevCtx& ctx, const h3b_dims* d, const h3b_grid* g,
                 const std::vector<int>& order, const h3b_block_weights* blocks,
                 const float* mods, int reduce_after, int unpair_bypass, const StepBufs& b,
                 cudaStream_t s, bool* stats_valid) {
  const int D = d->d;
  const int n = g->t * g->h * g->w + g->n_audio;
  const int n_red = g->t * g->h * (g->w / 2) + g->n_audio;
  int rc;
  bf16* cur = b.x_res;
  float2* cur_stats = b.stats;
  int cur_n = n;
  const float* rope = b.rope;
  for (size_t k = 0; k < order.size(); ++k) {
    const int blk = order[k];
    if ((rc = block_forward_folded_impl(ctx, d, &blocks[blk], mods + size_t(blk) * 6 * D, rope,
                                        cur_n, cur, cur_stats, b.arena, s)))
      return rc;
    if (reduce_after > 0 && int(k + 1) == reduce_after && k + 1 < order.size()) {
      if ((rc = launch_token_pair(b.x_res, b.x_red, g->t, g->h, g->w, g->n_audio, D, s)))
        return rc;
      cur = b.x_red;
      cur_n = n_red;
      cur_stats = b.stats_red;
      rope = b.rope_red;
      if ((rc = launch_row_stats(cur, cur_n, D, cur_stats, s))) return rc;
    }
  }
  *stats_valid = cur != b.x_red;
  if (cur == b.x_red &&
      (rc = launch_token_unpair(b.x_red, b.x_res, unpair_bypass ? b.x_res : nullptr, g->t, g->h,
                                g->w, g->n_audio, D, s)))
    return rc;
  return H3B_OK;
}

int denoise_step_impl(const DevCtx& ctx, const h3b_dims* d, const h3b_grid* g, int n_blocks,
                      const h3b_block_weights* blocks, const unsigned char* active,
                      const float* mods, const float* final_mod, int reduce_after,
                      int unpair_bypass, float sigma, float sigma_next, float* x_state,
                      const StepBufs& b, cudaStream_t s, float* v_out = nullptr,
                      float* r_out = nullptr) {
  const int D = d->d;
  const int nv = g->t * g->h * g->w;
  const int n = nv + g->n_audio;
  const int n_red = g->t * g->h * (g->w / 2) + g->n_audio;
  const bool may_reduce = reduce_after > 0;
  int rc;
  if ((rc = launch_rope_table(g->t, g->h, g->w, g->n_audio, g->rope_halved, 0, d->head_dim,
                              d->rope_split, d->rope_theta, b.rope, s)))
    return rc;
  if (may_reduce &&
      (rc = launch_rope_table(g->t, g->h, g->w, g->n_audio, g->rope_halved, 1, d->head_dim,
                              d->rope_split, d->rope_theta, b.rope_red, s)))
    return rc;

  std::vector<int> order;
  bool folded = true;
  for (int i = 0; i < n_blocks; ++i)
    if (!active || active[i]) {
      order.push_back(i);
      folded = folded && has_fold(&blocks[i]);
    }
  if (folded && !order.empty()) {
    // every block reads the raw residual and its row statistics (no LayerNorm pass)
    if ((rc = launch_state_to_residual(x_state, n, D, b.x_res, b.stats, s))) return rc;
    bool stats_valid = false;
    if ((rc = folded_stack(ctx, d, g, order, blocks, mods, reduce_after, unpair_bypass, b, s,
                           &stats_valid)))
      return rc;
    if (v_out || r_out)
      return launch_final_euler_keep(b.x_res, n, nv, D, d->ln_eps, final_mod, sigma_next - sigma,
                                     x_state, v_out, r_out, s);
    return launch_final_euler(b.x_res, n, nv, D, d->ln_eps, final_mod, sigma_next - sigma,
                              x_state, s);
  }
  const float* first_mod = order.empty() ? final_mod : mods + size_t(order[0]) * 6 * D;
  if ((rc = launch_ln_modulate_from_state(x_state, n, D, d->ln_eps, first_mod, first_mod + D,
                                          b.x_res, b.h, s)))
    return rc;

  bf16* cur = b.x_res;
  int cur_n = n;
  const float* rope = b.rope;
  for (size_t k = 0; k < order.size(); ++k) {
    const int blk = order[k];
    const bool has_next = k + 1 < order.size();
    const bool pair_now = may_reduce && int(k + 1) == reduce_after && has_next;
    const float* mod = mods + size_t(blk) * 6 * D;
    const float* mod_next = (has_next && !pair_now) ? mods + size_t(order[k + 1]) * 6 * D : nullptr;
    if ((rc = block_forward_impl(ctx, d, &blocks[blk], mod, mod_next, rope, cur_n, false, cur,
                                 b.h, b.arena, s)))
      return rc;
    if (pair_now) {
      if ((rc = launch_token_pair(b.x_res, b.x_red, g->t, g->h, g->w, g->n_audio, D, s)))
        return rc;
      cur = b.x_red;
      cur_n = n_red;
      rope = b.rope_red;
      const float* nm = mods + size_t(order[k + 1]) * 6 * D;
      if ((rc = launch_ln_modulate(cur, cur_n, D, d->ln_eps, nm, nm + D, b.h, s))) return rc;
    }
  }
  if (cur == b.x_red &&
      (rc = launch_token_unpair(b.x_red, b.x_res, unpair_bypass ? b.x_res : nullptr, g->t, g->h,
                                g->w, g->n_audio, D, s)))
    return rc;
  if (v_out || r_out)
    return launch_final_euler_keep(b.x_res, n, nv, D, d->ln_eps, final_mod, sigma_next - sigma,
                                   x_state, v_out, r_out, s);
  return launch_final_euler(b.x_res, n, nv, D, d->ln_eps, final_mod, sigma_next - sigma, x_state, s);
}

// One Euler step on the per-token latent: patch embedding per stream into the residual
// (its epilogue writing the row statistics), the folded block stack, the final AdaLN
// folded into each stream's head with the Euler update in the head's epilogue.
int denoise_step_latent_impl(const DevCtx& ctx, const h3b_dims* d, const h3b_grid* g,
                             int n_blocks, const h3b_block_weights* blocks,
                             const unsigned char* active, const float* mods,
                             const h3b_latent_heads* hd, int reduce_after, int unpair_bypass,
                             float sigma, float sigma_next, float* latent, const StepBufs& b,
                             cudaStream_t s) {
  const int D = d->d, C = hd->c_lat;
  const int nv = g->t * g->h * g->w;
  const int n = nv + g->n_audio;
  const int parts = D / 256;
  int rc;
  if ((rc = launch_rope_table(g->t, g->h, g->w, g->n_audio, g->rope_halved, 0, d->head_dim,
                              d->rope_split, d->rope_theta, b.rope, s)))
    return rc;
  if (reduce_after > 0 &&
      (rc = launch_rope_table(g->t, g->h, g->w, g->n_audio, g->rope_halved, 1, d->head_dim,
                              d->rope_split, d->rope_theta, b.rope_red, s)))
    return rc;
  if ((rc = launch_f32_to_bf16(latent, static_cast<long long>(n) * C, b.lat, s))) return rc;
  const int rows[2] = {nv, g->n_audio};
  const int first[2] = {0, nv};
  for (int st = 0; st < 2; ++st) {  // patch embedding, video rows then audio rows
    GemmEpilogue e;
    e.kind = kEpiBias;
    e.bias = reinterpret_cast<const bf16*>(hd->b_patch[st]);
    e.out = b.x_res + size_t(first[st]) * D;
    e.ld_out = D;
    e.stats_out = b.stats + size_t(first[st]) * parts;
    if ((rc = launch_gemm_bf16(ctx, b.lat + size_t(first[st]) * C,
                               reinterpret_cast<const bf16*>(hd->w_patch[st]), rows[st], D, C, e,
                               b.arena, 0, s)))
      return rc;
  }
  std::vector<int> order;
  for (int i = 0; i < n_blocks; ++i)
    if (!active || active[i]) order.push_back(i);
  bool stats_valid = true;
  if (!order.empty() && (rc = folded_stack(ctx, d, g, order, blocks, mods, reduce_after,
                                           unpair_bypass, b, s, &stats_valid)))
    return rc;
  if (!stats_valid && (rc = launch_row_stats(b.x_res, n, D, b.stats, s))) return rc;
  for (int st = 0; st < 2; ++st) {  // final AdaLN + head + Euler, per stream
    GemmEpilogue e;
    e.kind = kEpiHeadEuler;
    e.bias_f32 = hd->dv_head[st];
    e.fold_c = hd->c_head[st];
    e.stats_in = b.stats + size_t(first[st]) * parts;
    e.stats_parts = parts;
    e.ln_eps = d->ln_eps;
    e.out_f32 = latent + size_t(first[st]) * C;
    e.ld_out = C;
    e.euler_dt = sigma_next - sigma;
    if ((rc = launch_gemm_bf16(ctx, b.x_res + size_t(first[st]) * D,
                               reinterpret_cast<const bf16*>(hd->w_head_fold[st]), rows[st], C, D,
                               e, b.arena, 0, s)))
      return rc;
  }
  return H3B_OK;
}

int check_step_args(const h3b_dims* dims, const h3b_grid* grid, int n_blocks,
                    const h3b_block_weights* blocks, const unsigned char* active,
                    const float* mods, const float* final_mod, int reduce_after,
                    const float* x_state, void* ws, size_t ws_bytes, StepBufs* bufs) {
  int rc;
  if ((rc = check_dims(dims))) return rc;
  if ((rc = check_grid(grid, reduce_after > 0))) return rc;
  if (n_blocks < 0 || (n_blocks > 0 && !blocks)) return set_error(H3B_EINVAL, "bad block list");
  for (int i = 0; i < n_blocks; ++i)
    if ((!active || active[i]) &&
        ((rc = check_weights(&blocks[i])) || (has_fold(&blocks[i]) && (rc = check_fold(&blocks[i])))))
      return rc;
  if (!mods && n_blocks > 0) return set_error(H3B_EINVAL, "mods is NULL");
  if (!final_mod || !x_state || !al16(mods) || !al16(final_mod) || !al16(x_state))
    return set_error(H3B_EINVAL, "final_mod / x_state NULL or not 16-byte aligned");
  const StepBufs need = carve_step(dims, grid, reduce_after > 0, nullptr);
  if (!ws || !al16(ws) || ws_bytes < need.total)
    return set_error(H3B_EWORKSPACE, "workspace of %zu bytes needed, %zu given", need.total, ws_bytes);
  *bufs = carve_step(dims, grid, reduce_after > 0, ws);
  return H3B_OK;
}

}  // namespace
}  // namespace h3b

using namespace h3b;

// ============================================================================ C ABI
extern "C" {

int h3b_version(void) { return H3B_VERSION; }

const char* h3b_last_error(void) { return g_last_error; }

uint64_t h3b_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

int h3b_sync_status(void* stream) {
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return set_error(H3B_ECUDA, "stream sync: %s", cudaGetErrorString(e));
  uint32_t flag = 0;
  e = cudaMemcpyFromSymbol(&flag, g_h3b_wait_error, sizeof(flag));
  if (e != cudaSuccess) return set_error(H3B_ECUDA, "read wait flag: %s", cudaGetErrorString(e));
  if (flag) {
    const uint32_t zero = 0;
    cudaMemcpyToSymbol(g_h3b_wait_error, &zero, sizeof(zero));
    int dev = -1;
    if (cudaGetDevice(&dev) == cudaSuccess) drop_graphs(dev);
    return set_error(H3B_ETIMEOUT, "a device-side wait gave up (code %u)", flag);
  }
  return H3B_OK;
}

size_t h3b_gemm_workspace_size(void) { return gemm_scratch_bytes(); }

int h3b_gemm_schedule(int tiles, int k_blocks, int units, int mode, int unit, int* items,
                      int max_items) {
  if (tiles <= 0 || k_blocks <= 0 || units <= 0 || unit < 0 || unit >= units)
    return set_error(H3B_EINVAL, "gemm_schedule: tiles=%d k_blocks=%d units=%d unit=%d", tiles,
                     k_blocks, units, unit);
  if (mode < 0 || mode > 3) return set_error(H3B_EINVAL, "gemm_schedule: mode %d", mode);
  if (max_items < 0 || (max_items > 0 && !items))
    return set_error(H3B_EINVAL, "gemm_schedule: items buffer");
  const int n = gemm_schedule_items(tiles, k_blocks, units, mode, unit, items, max_items);
  if (n < 0)
    return set_error(H3B_EINVAL, "gemm_schedule: too few split K slices per unit for mode %d",
                     mode);
  return n;
}

int h3b_set_gemm_override(int tile, int sched, int trans) {
  if (set_gemm_override(tile, sched, trans))
    return set_error(H3B_EINVAL, "set_gemm_override: tile=%d sched=%d trans=%d", tile, sched,
                     trans);
  return H3B_OK;
}

int h3b_set_attention_variant(int variant) {
  if (set_attention_variant(variant))
    return set_error(H3B_EINVAL, "set_attention_variant: %d (0, 1 or 2)", variant);
  return H3B_OK;
}

size_t h3b_workspace_size(const h3b_dims* dims, int n_tokens) {
  if (check_dims(dims) || n_tokens < 0) return 0;
  return arena_bytes(dims, n_tokens);
}

size_t h3b_denoise_workspace_size(const h3b_dims* dims, const h3b_grid* grid, int reduce) {
  if (check_dims(dims) || check_grid(grid, reduce != 0)) return 0;
  return carve_step(dims, grid, reduce != 0, nullptr).total;
}

int h3b_adaln_modulation(const h3b_bf16* w, const h3b_bf16* b, const h3b_bf16* c, int n_out,
                         int c_dim, float* mod, void* stream) {
  if (!w || !b || !c || !mod || !al16(w) || !al16(c))
    return set_error(H3B_EINVAL, "adaln_modulation: NULL or misaligned pointer");
  if (n_out < 0 || c_dim <= 0 || c_dim % 8)
    return set_error(H3B_EINVAL, "adaln_modulation: c_dim=%d must be a positive multiple of 8", c_dim);
  DevCtx ctx;
  if (int rc = get_ctx(&ctx)) return rc;
  return launch_adaln_gemv(reinterpret_cast<const bf16*>(w), reinterpret_cast<const bf16*>(b),
                           reinterpret_cast<const bf16*>(c), n_out, c_dim, mod,
                           static_cast<cudaStream_t>(stream));
}

int h3b_rope_table(const h3b_dims* dims, const h3b_grid* grid, int paired, float* rope_cs,
                   void* stream) {
  int rc;
  if ((rc = check_dims(dims)) || (rc = check_grid(grid, paired != 0))) return rc;
  if (!rope_cs || !al16(rope_cs)) return set_error(H3B_EINVAL, "rope_table: bad output pointer");
  DevCtx ctx;
  if ((rc = get_ctx(&ctx))) return rc;
  return launch_rope_table(grid->t, grid->h, grid->w, grid->n_audio, grid->rope_halved,
                           paired != 0, dims->head_dim, dims->rope_split, dims->rope_theta,
                           rope_cs, static_cast<cudaStream_t>(stream));
}

int h3b_ln_modulate(const h3b_bf16* x, int n_tokens, int d, float eps, const float* shift,
                    const float* scale, h3b_bf16* h, void* stream) {
  if (n_tokens < 0 || d <= 0 || d % 256 || d > 4096)
    return set_error(H3B_EINVAL, "ln_modulate: d=%d must be a multiple of 256 <= 4096", d);
  if (!x || !h || !shift || !scale || !al16(x) || !al16(h) || !al16(shift) || !al16(scale))
    return set_error(H3B_EINVAL, "ln_modulate: NULL or misaligned pointer");
  if (!(eps > 0.f)) return set_error(H3B_EINVAL, "ln_modulate: eps must be positive");
  DevCtx ctx;
  if (int rc = get_ctx(&ctx)) return rc;
  return launch_ln_modulate(reinterpret_cast<const bf16*>(x), n_tokens, d, eps, shift, scale,
                            reinterpret_cast<bf16*>(h), static_cast<cudaStream_t>(stream));
}

int h3b_block_forward(const h3b_dims* dims, const h3b_block_weights* w, const float* mod,
                      const float* mod_next, const float* rope_cs, int n_tokens, int compute_h,
                      h3b_bf16* x, h3b_bf16* h, void* ws, size_t ws_bytes, void* stream) {
  int rc;
  if ((rc = check_dims(dims)) || (rc = check_weights(w))) return rc;
  if (n_tokens < 0 || n_tokens > (1 << 24)) return set_error(H3B_EINVAL, "n_tokens=%d", n_tokens);
  if (!mod || !rope_cs || !x || !h || !al16(mod) || !al16(rope_cs) || !al16(x) || !al16(h) ||
      (mod_next && !al16(mod_next)))
    return set_error(H3B_EINVAL, "block_forward: NULL or misaligned pointer");
  if (!ws || !al16(ws) || ws_bytes < arena_bytes(dims, n_tokens))
    return set_error(H3B_EWORKSPACE, "block_forward: workspace of %zu bytes needed, %zu given",
                     arena_bytes(dims, n_tokens), ws_bytes);
  DevCtx ctx;
  if ((rc = get_ctx(&ctx))) return rc;
  return block_forward_impl(ctx, dims, w, mod, mod_next, rope_cs, n_tokens, compute_h != 0,
                            reinterpret_cast<bf16*>(x), reinterpret_cast<bf16*>(h), ws,
                            static_cast<cudaStream_t>(stream));
}

int h3b_fold_adaln(const h3b_bf16* w, const h3b_bf16* b, const float* shift, const float* scale,
                   int n_out, int d, h3b_bf16* w_out, float* c_out, float* dv_out,
                   void* stream) {
  if (n_out < 0 || d <= 0 || d % 8)
    return set_error(H3B_EINVAL, "fold_adaln: d=%d must be a positive multiple of 8", d);
  const void* ptrs[7] = {w, b, shift, scale, w_out, c_out, dv_out};
  for (const void* q : ptrs)
    if (!q || !al16(q)) return set_error(H3B_EINVAL, "fold_adaln: NULL or misaligned pointer");
  const uintptr_t w0 = reinterpret_cast<uintptr_t>(w), o0 = reinterpret_cast<uintptr_t>(w_out);
  const uintptr_t bytes = uintptr_t(n_out) * d * 2;
  if (w0 < o0 + bytes && o0 < w0 + bytes)
    return set_error(H3B_EINVAL, "fold_adaln: w_out overlaps w");
  DevCtx ctx;
  if (int rc = get_ctx(&ctx)) return rc;
  return launch_fold_adaln(reinterpret_cast<const bf16*>(w), reinterpret_cast<const bf16*>(b),
                           shift, scale, n_out, d, reinterpret_cast<bf16*>(w_out), c_out, dv_out,
                           static_cast<cudaStream_t>(stream));
}

int h3b_row_stats(const h3b_bf16* x, int n_tokens, int d, float* stats, void* stream) {
  if (n_tokens < 0 || d <= 0 || d % 256 || d > 4096)
    return set_error(H3B_EINVAL, "row_stats: d=%d must be a multiple of 256 <= 4096", d);
  if (!x || !stats || !al16(x) || !al16(stats))
    return set_error(H3B_EINVAL, "row_stats: NULL or misaligned pointer");
  DevCtx ctx;
  if (int rc = get_ctx(&ctx)) return rc;
  return launch_row_stats(reinterpret_cast<const bf16*>(x), n_tokens, d,
                          reinterpret_cast<float2*>(stats), static_cast<cudaStream_t>(stream));
}

int h3b_block_forward_folded(const h3b_dims* dims, const h3b_block_weights* w, const float* mod,
                             const float* rope_cs, int n_tokens, h3b_bf16* x, float* stats,
                             void* ws, size_t ws_bytes, void* stream) {
  int rc;
  if ((rc = check_dims(dims)) || (rc = check_weights(w)) || (rc = check_fold(w))) return rc;
  if (n_tokens < 0 || n_tokens > (1 << 24)) return set_error(H3B_EINVAL, "n_tokens=%d", n_tokens);
  if (!mod || !rope_cs || !x || !stats || !al16(mod) || !al16(rope_cs) || !al16(x) || !al16(stats))
    return set_error(H3B_EINVAL, "block_forward_folded: NULL or misaligned pointer");
  if (!ws || !al16(ws) || ws_bytes < arena_bytes(dims, n_tokens))
    return set_error(H3B_EWORKSPACE, "block_forward_folded: workspace of %zu bytes needed, %zu given",
                     arena_bytes(dims, n_tokens), ws_bytes);
  DevCtx ctx;
  if ((rc = get_ctx(&ctx))) return rc;
  return block_forward_folded_impl(ctx, dims, w, mod, rope_cs, n_tokens, reinterpret_cast<bf16*>(x),
                                   reinterpret_cast<float2*>(stats), ws,
                                   static_cast<cudaStream_t>(stream));
}

size_t h3b_workspace_size_int8(const h3b_dims* dims, int n_tokens) {
  if (check_dims(dims) || n_tokens < 0 || dims->d_ff % 1024) return 0;
  return arena_bytes(dims, n_tokens) + carve_int8(dims, n_tokens, nullptr).total;
}

int h3b_block_forward_int8(const h3b_dims* dims, const h3b_block_weights* w,
                           const h3b_int8_block* wq, const float* mod, const float* rope_cs,
                           int n_tokens, h3b_bf16* x, void* ws, size_t ws_bytes, void* stream) {
  int rc;
  if ((rc = check_dims(dims)) || (rc = check_weights(w))) return rc;
  if (dims->d_ff % 1024)
    return set_error(H3B_EINVAL, "block_forward_int8: d_ff=%d must be a multiple of 1024", dims->d_ff);
  if (n_tokens < 0 || n_tokens > (1 << 24)) return set_error(H3B_EINVAL, "n_tokens=%d", n_tokens);
  if (!wq) return set_error(H3B_EINVAL, "block_forward_int8: int8 weights NULL");
  const void* ptrs[6] = {wq->w_qkv_q, wq->s_qkv, wq->w_fc1_q, wq->s_fc1, wq->w_fc2_q, wq->s_fc2};
  for (const void* p : ptrs)
    if (!p || !al16(p)) return set_error(H3B_EINVAL, "block_forward_int8: int8 weight NULL or misaligned");
  if (!mod || !rope_cs || !x || !al16(mod) || !al16(rope_cs) || !al16(x))
    return set_error(H3B_EINVAL, "block_forward_int8: NULL or misaligned pointer");
  const size_t need = arena_bytes(dims, n_tokens) + carve_int8(dims, n_tokens, nullptr).total;
  if (!ws || !al16(ws) || ws_bytes < need)
    return set_error(H3B_EWORKSPACE, "block_forward_int8: workspace of %zu bytes needed, %zu given",
                     need, ws_bytes);
  DevCtx ctx;
  if ((rc = get_ctx(&ctx))) return rc;
  return block_forward_int8_impl(ctx, dims, w, wq, mod, rope_cs, n_tokens,
                                 reinterpret_cast<bf16*>(x), ws, static_cast<cudaStream_t>(stream));
}

int h3b_quantize_groups(const h3b_bf16* a, int rows, int cols, int8_t* q, float* scale,
                        void* stream) {
  if (rows < 0 || cols <= 0 || cols % 1024)
    return set_error(H3B_EINVAL, "quantize_groups: cols=%d must be a positive multiple of 1024", cols);
  if (!a || !q || !scale || !al16(a) || !al16(q) || !al16(scale))
    return set_error(H3B_EINVAL, "quantize_groups: NULL or misaligned pointer");
  DevCtx ctx;
  if (int rc = get_ctx(&ctx)) return rc;
  return launch_quantize_groups(reinterpret_cast<const bf16*>(a), rows, cols, q, scale,
                                static_cast<cudaStream_t>(stream));
}

int h3b_ln_modulate_q8(const h3b_bf16* x, int n_tokens, int d, float eps, const float* shift,
                       const float* scale, int8_t* q, float* q_scale, void* stream) {
  if (n_tokens < 0 || d <= 0 || d % 256 || d > 4096)
    return set_error(H3B_EINVAL, "ln_modulate_q8: d=%d must be a multiple of 256 <= 4096", d);
  if (!x || !q || !q_scale || !shift || !scale || !al16(x) || !al16(q) || !al16(shift) ||
      !al16(scale))
    return set_error(H3B_EINVAL, "ln_modulate_q8: NULL or misaligned pointer");
  DevCtx ctx;
  if (int rc = get_ctx(&ctx)) return rc;
  return launch_ln_modulate_q8(reinterpret_cast<const bf16*>(x), n_tokens, d, eps, shift, scale,
                               q, q_scale, static_cast<cudaStream_t>(stream));
}

int h3b_gemm_i8_grouped(const int8_t* A, const float* a_scale, int M, int K, int N,
                        const int8_t* w_q, const float* w_scale, const h3b_bf16* bias,
                        const float* gate, h3b_bf16* resid, void* ws, size_t ws_bytes,
                        void* stream) {
  if (M < 0 || K <= 0 || K % 1024 || N <= 0 || N % 128)
    return set_error(H3B_EINVAL, "gemm_i8_grouped: K=%d must be a multiple of 1024, N=%d of 128", K, N);
  const void* ptrs[6] = {A, a_scale, w_q, w_scale, gate, resid};
  for (const void* p : ptrs)
    if (!p || !al16(p)) return set_error(H3B_EINVAL, "gemm_i8_grouped: NULL or misaligned pointer");
  if (bias && !al16(bias)) return set_error(H3B_EINVAL, "gemm_i8_grouped: misaligned bias");
  DevCtx ctx;
  if (int rc = get_ctx(&ctx)) return rc;
  GemmEpilogue e;
  e.kind = kEpiI8GroupGate;
  e.bias = reinterpret_cast<const bf16*>(bias);
  e.row_scale = a_scale;
  e.act_groups = K / 1024;
  e.col_scale = w_scale;
  e.gate = gate;
  e.out = reinterpret_cast<bf16*>(resid);
  e.ld_out = N;
  return launch_gemm_i8_grouped(ctx, A, w_q, M, N, K, e, ws, ws ? ws_bytes : 0,
                                static_cast<cudaStream_t>(stream));
}

int h3b_block_forward_noalloc(const h3b_dims* dims, const h3b_block_weights* w,
                              const float* mod, const float* mod_next, const float* rope_cs,
                              int n_tokens, int compute_h, h3b_bf16* x, h3b_bf16* h,
                              void* stream) {
  int rc;
  if ((rc = check_dims(dims)) || (rc = check_weights(w))) return rc;
  if (n_tokens < 0 || n_tokens > (1 << 24)) return set_error(H3B_EINVAL, "n_tokens=%d", n_tokens);
  if (!mod || !rope_cs || !x || !h || !al16(mod) || !al16(rope_cs) || !al16(x) || !al16(h) ||
      (mod_next && !al16(mod_next)))
    return set_error(H3B_EINVAL, "block_forward_noalloc: NULL or misaligned pointer");
  const size_t need = arena_bytes(dims, n_tokens);
  if (need > H3B_NOALLOC_WORKSPACE_BYTES)
    return set_error(H3B_EWORKSPACE,
                     "block_forward_noalloc: %d tokens need %zu workspace bytes, the static "
                     "workspace holds %zu",
                     n_tokens, need, size_t(H3B_NOALLOC_WORKSPACE_BYTES));
  DevCtx ctx;
  if ((rc = get_ctx(&ctx))) return rc;
  // Device address of the static workspace, looked up once per device with that device
  // current (the host-side name of a __device__ array is not a device pointer).
  static std::mutex mu;
  static void* addr[kMaxDevices] = {};
  void* ws = nullptr;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[ctx.device]) {
      void* p = nullptr;
      cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_ws);
      if (e != cudaSuccess || !p)
        return set_error(H3B_ECUDA, "block_forward_noalloc: cudaGetSymbolAddress: %s",
                         cudaGetErrorString(e));
      addr[ctx.device] = p;
    }
    ws = addr[ctx.device];
  }
  return block_forward_impl(ctx, dims, w, mod, mod_next, rope_cs, n_tokens, compute_h != 0,
                            reinterpret_cast<bf16*>(x), reinterpret_cast<bf16*>(h), ws,
                            static_cast<cudaStream_t>(stream));
}

int h3b_final_euler(const h3b_bf16* x_l, int n_tokens, int n_video, int d, float eps,
                    const float* final_mod, float sigma, float sigma_next, float* x_state,
                    void* stream) {
  if (n_tokens < 0 || n_video < 0 || n_video > n_tokens || d <= 0 || d % 256 || d > 4096)
    return set_error(H3B_EINVAL, "final_euler: bad sizes (n=%d n_video=%d d=%d)", n_tokens, n_video, d);
  if (!x_l || !final_mod || !x_state || !al16(x_l) || !al16(final_mod) || !al16(x_state))
    return set_error(H3B_EINVAL, "final_euler: NULL or misaligned pointer");
  DevCtx ctx;
  if (int rc = get_ctx(&ctx)) return rc;
  return launch_final_euler(reinterpret_cast<const bf16*>(x_l), n_tokens, n_video, d, eps,
                            final_mod, sigma_next - sigma, x_state,
                            static_cast<cudaStream_t>(stream));
}

int h3b_denoise_step(const h3b_dims* dims, const h3b_grid* grid, int n_blocks,
                     const h3b_block_weights* blocks, const unsigned char* active,
                     const float* mods, const float* final_mod, int reduce_after,
                     int unpair_bypass, float sigma, float sigma_next, float* x_state,
                     void* ws, size_t ws_bytes, void* stream) {
  StepBufs b;
  int rc = check_step_args(dims, grid, n_blocks, blocks, active, mods, final_mod, reduce_after,
                           x_state, ws, ws_bytes, &b);
  if (rc) return rc;
  DevCtx ctx;
  if ((rc = get_ctx(&ctx))) return rc;
  return denoise_step_impl(ctx, dims, grid, n_blocks, blocks, active, mods, final_mod,
                           reduce_after, unpair_bypass, sigma, sigma_next, x_state, b,
                           static_cast<cudaStream_t>(stream));
}

size_t h3b_denoise_latent_workspace_size(const h3b_dims* dims, const h3b_grid* grid, int reduce,
                                         int c_lat) {
  if (check_dims(dims) || check_grid(grid, reduce != 0) || c_lat <= 0 || c_lat % 128) return 0;
  return carve_step(dims, grid, reduce != 0, nullptr, c_lat).total;
}

int h3b_denoise_step_latent(const h3b_dims* dims, const h3b_grid* grid, int n_blocks,
                            const h3b_block_weights* blocks, const unsigned char* active,
                            const float* mods, const h3b_latent_heads* heads, int reduce_after,
                            int unpair_bypass, float sigma, float sigma_next, float* latent,
                            void* ws, size_t ws_bytes, void* stream) {
  int rc;
  if ((rc = check_dims(dims)) || (rc = check_grid(grid, reduce_after > 0))) return rc;
  if (!heads || heads->c_lat <= 0 || heads->c_lat % 128 || heads->c_lat > 4096)
    return set_error(H3B_EINVAL, "denoise_step_latent: c_lat must be a positive multiple of 128");
  for (int st = 0; st < 2; ++st) {
    const void* p[6] = {heads->w_patch[st], heads->b_patch[st], heads->w_head_fold[st],
                        heads->c_head[st], heads->dv_head[st], nullptr};
    for (int i = 0; i < 5; ++i)
      if (!p[i] || !al16(p[i]))
        return set_error(H3B_EINVAL, "denoise_step_latent: head pointer NULL or misaligned");
  }
  if (n_blocks < 0 || (n_blocks > 0 && (!blocks || !mods)))
    return set_error(H3B_EINVAL, "bad block list");
  for (int i = 0; i < n_blocks; ++i)
    if ((!active || active[i]) && ((rc = check_weights(&blocks[i])) || (rc = check_fold(&blocks[i]))))
      return rc;
  if (!latent || !al16(latent)) return set_error(H3B_EINVAL, "latent NULL or misaligned");
  const StepBufs need = carve_step(dims, grid, reduce_after > 0, nullptr, heads->c_lat);
  if (!ws || !al16(ws) || ws_bytes < need.total)
    return set_error(H3B_EWORKSPACE, "workspace of %zu bytes needed, %zu given", need.total,
                     ws_bytes);
  const StepBufs b = carve_step(dims, grid, reduce_after > 0, ws, heads->c_lat);
  DevCtx ctx;
  if ((rc = get_ctx(&ctx))) return rc;
  return denoise_step_latent_impl(ctx, dims, grid, n_blocks, blocks, active, mods, heads,
                                  reduce_after, unpair_bypass, sigma, sigma_next, latent, b,
                                  static_cast<cudaStream_t>(stream));
}

int h3b_denoise_step_keep(const h3b_dims* dims, const h3b_grid* grid, int n_blocks,
                          const h3b_block_weights* blocks, const unsigned char* active,
                          const float* mods, const float* final_mod, int reduce_after,
                          int unpair_bypass, float sigma, float sigma_next, float* x_state,
                          float* v_out, float* core_res_out, void* ws, size_t ws_bytes,
                          void* stream) {
  StepBufs b;
  int rc = check_step_args(dims, grid, n_blocks, blocks, active, mods, final_mod, reduce_after,
                           x_state, ws, ws_bytes, &b);
  if (rc) return rc;
  if ((v_out && !al16(v_out)) || (core_res_out && !al16(core_res_out)))
    return set_error(H3B_EINVAL, "denoise_step_keep: misaligned v_out / core_res_out");
  DevCtx ctx;
  if ((rc = get_ctx(&ctx))) return rc;
  return denoise_step_impl(ctx, dims, grid, n_blocks, blocks, active, mods, final_mod,
                           reduce_after, unpair_bypass, sigma, sigma_next, x_state, b,
                           static_cast<cudaStream_t>(stream), v_out, core_res_out);
}

int h3b_euler_velocity(const float* v, int n_tokens, int d, float sigma, float sigma_next,
                       float* x_state, void* stream) {
  if (n_tokens < 0 || d <= 0 || d % 4)
    return set_error(H3B_EINVAL, "euler_velocity: bad sizes (n=%d d=%d)", n_tokens, d);
  if (!v || !x_state || !al16(v) || !al16(x_state))
    return set_error(H3B_EINVAL, "euler_velocity: NULL or misaligned pointer");
  DevCtx ctx;
  if (int rc = get_ctx(&ctx)) return rc;
  return launch_euler_axpy(v, static_cast<long long>(n_tokens) * d, sigma_next - sigma, x_state,
                           static_cast<cudaStream_t>(stream));
}

int h3b_euler_core_reuse(const float* core_res, int n_tokens, int n_video, int d, float eps,
                         const float* final_mod, float sigma, float sigma_next, float* x_state,
                         void* stream) {
  if (n_tokens < 0 || n_video < 0 || n_video > n_tokens || d <= 0 || d % 256 || d > 4096)
    return set_error(H3B_EINVAL, "euler_core_reuse: bad sizes (n=%d n_video=%d d=%d)", n_tokens,
                     n_video, d);
  if (!core_res || !final_mod || !x_state || !al16(core_res) || !al16(final_mod) ||
      !al16(x_state))
    return set_error(H3B_EINVAL, "euler_core_reuse: NULL or misaligned pointer");
  DevCtx ctx;
  if (int rc = get_ctx(&ctx)) return rc;
  return launch_core_reuse_final(core_res, n_tokens, n_video, d, eps, final_mod,
                                 sigma_next - sigma, x_state, static_cast<cudaStream_t>(stream));
}

int h3b_reuse_schedule(int steps, int every, unsigned char* fresh_out) {
  if (steps <= 0 || every <= 0 || !fresh_out)
    return set_error(H3B_EINVAL, "reuse_schedule: steps=%d every=%d", steps, every);
  int n = 0;
  for (int i = 0; i < steps; ++i) {
    fresh_out[i] = (i % every == 0 || i == steps - 1) ? 1 : 0;
    n += fresh_out[i];
  }
  return n;
}

namespace {

// Captured whole denoises (the Euler steps of one request on one state buffer), kept per
// device and keyed by every argument that shapes the launches: a replay relaunches the
// same kernels with the same arguments (the split schedules' flags are handed back at zero
// by their readers, so replays stay correct; after a timed-out wait h3b_sync_status drops
// them all).  Captured on a stream of the library's and launched on the caller's.
constexpr size_t kGraphCacheSize = 4;

void key_bytes(std::vector<uint8_t>& k, const void* v, size_t n) {
  const uint8_t* b = static_cast<const uint8_t*>(v);
  k.insert(k.end(), b, b + n);
}
#define H3B_KEY_PUT(k, v) key_bytes((k), &(v), sizeof(v))

int denoise_graph(const DevCtx& ctx, const h3b_dims* dims, const h3b_grid* grid, int n_blocks,
                  const h3b_block_weights* blocks, const unsigned char* active,
                  const float* mods, const float* final_mod, int reduce_after,
                  int unpair_bypass, int n_steps, int first_step, int n_run, float* state,
                  const StepBufs& b, void* ws, size_t ws_bytes, cudaGraphExec_t* out) {
  static cudaStream_t capture_stream[kMaxDevices] = {};
  std::vector<uint8_t> key;
  H3B_KEY_PUT(key, *dims);
  H3B_KEY_PUT(key, *grid);
  H3B_KEY_PUT(key, n_blocks);
  for (int i = 0; i < n_blocks; ++i) {
    H3B_KEY_PUT(key, blocks[i]);
    const unsigned char on = active ? active[i] : 1;
    H3B_KEY_PUT(key, on);
  }
  H3B_KEY_PUT(key, mods);
  H3B_KEY_PUT(key, final_mod);
  H3B_KEY_PUT(key, reduce_after);
  H3B_KEY_PUT(key, unpair_bypass);
  H3B_KEY_PUT(key, n_steps);
  H3B_KEY_PUT(key, first_step);
  H3B_KEY_PUT(key, n_run);
  H3B_KEY_PUT(key, state);
  H3B_KEY_PUT(key, ws);
  H3B_KEY_PUT(key, ws_bytes);
  std::lock_guard<std::mutex> lock(g_graph_mu);
  auto& c = g_graphs[ctx.device];
  for (const DenoiseGraph& gph : c)
    if (gph.key == key) {
      *out = gph.exec;
      return 0;
    }
  cudaError_t e = cudaSuccess;
  if (!capture_stream[ctx.device])
    e = cudaStreamCreateWithFlags(&capture_stream[ctx.device], cudaStreamNonBlocking);
  if (e != cudaSuccess)
    return set_error(H3B_ECUDA, "denoise graph: stream: %s", cudaGetErrorString(e));
  cudaStream_t cs = capture_stream[ctx.device];
  if ((e = cudaStreamBeginCapture(cs, cudaStreamCaptureModeThreadLocal)) != cudaSuccess)
    return set_error(H3B_ECUDA, "denoise graph: begin capture: %s", cudaGetErrorString(e));
  int rc = 0;
  for (int i = first_step; i < first_step + n_run && rc == 0; ++i) {
    const float sg = static_cast<float>(1.0 - double(i) / n_steps);
    const float sn = static_cast<float>(1.0 - double(i + 1) / n_steps);
    rc = denoise_step_impl(ctx, dims, grid, n_blocks, blocks, active, mods, final_mod,
                           reduce_after, unpair_bypass, sg, sn, state, b, cs);
  }
  cudaGraph_t graph = nullptr;
  e = cudaStreamEndCapture(cs, &graph);
  if (rc != 0 || e != cudaSuccess) {
    if (graph) cudaGraphDestroy(graph);
    cudaGetLastError();
    return rc ? rc : set_error(H3B_ECUDA, "denoise graph: capture: %s", cudaGetErrorString(e));
  }
  cudaGraphExec_t exec = nullptr;
  e = cudaGraphInstantiate(&exec, graph, 0);
  cudaGraphDestroy(graph);
  if (e != cudaSuccess)
    return set_error(H3B_ECUDA, "denoise graph: instantiate: %s", cudaGetErrorString(e));
  if (c.size() >= kGraphCacheSize) {
    cudaGraphExecDestroy(c.front().exec);
    c.erase(c.begin());
  }
  c.push_back({std::move(key), exec});
  *out = exec;
  return 0;
}

}  // namespace

int h3b_denoise_host(const h3b_dims* dims, const h3b_grid* grid, int n_blocks,
                     const h3b_block_weights* blocks, const unsigned char* active,
                     const float* mods, const float* final_mod, int reduce_after,
                     int unpair_bypass, int n_steps, int first_step, int n_run,
                     const float* x_host_in, float* x_host_out, float* x_state_dev,
                     void* ws, size_t ws_bytes, void* stream) {
  StepBufs b;
  int rc = check_step_args(dims, grid, n_blocks, blocks, active, mods, final_mod, reduce_after,
                           x_state_dev, ws, ws_bytes, &b);
  if (rc) return rc;
  if (!x_host_in || !x_host_out) return set_error(H3B_EINVAL, "denoise_host: NULL host buffer");
  if (n_steps <= 0 || first_step < 0 || n_run < 0 || first_step + n_run > n_steps)
    return set_error(H3B_EINVAL, "denoise_host: steps %d..%d of %d", first_step,
                     first_step + n_run, n_steps);
  DevCtx ctx;
  if ((rc = get_ctx(&ctx))) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // the Euler steps as one cached CUDA graph (direct launches with H3B_DEBUG)
  cudaGraphExec_t graph = nullptr;
  if (!debug_mode() &&
      (rc = denoise_graph(ctx, dims, grid, n_blocks, blocks, active, mods, final_mod,
                          reduce_after, unpair_bypass, n_steps, first_step, n_run, x_state_dev,
                          b, ws, ws_bytes, &graph)))
    return rc;
  const size_t bytes = (size_t(grid->t) * grid->h * grid->w + grid->n_audio) * dims->d * 4;
  cudaError_t e = cudaMemcpyAsync(x_state_dev, x_host_in, bytes, cudaMemcpyHostToDevice, s);
  if (e != cudaSuccess) return set_error(H3B_ECUDA, "denoise_host H2D: %s", cudaGetErrorString(e));
  if (graph) {
    if ((e = cudaGraphLaunch(graph, s)) != cudaSuccess)
      return set_error(H3B_ECUDA, "denoise_host graph launch: %s", cudaGetErrorString(e));
  } else {
    for (int i = first_step; i < first_step + n_run; ++i) {
      const float sg = static_cast<float>(1.0 - double(i) / n_steps);
      const float sn = static_cast<float>(1.0 - double(i + 1) / n_steps);
      if ((rc = denoise_step_impl(ctx, dims, grid, n_blocks, blocks, active, mods, final_mod,
                                  reduce_after, unpair_bypass, sg, sn, x_state_dev, b, s)))
        return rc;
    }
  }
  e = cudaMemcpyAsync(x_host_out, x_state_dev, bytes, cudaMemcpyDeviceToHost, s);
  if (e != cudaSuccess) return set_error(H3B_ECUDA, "denoise_host D2H: %s", cudaGetErrorString(e));
  return h3b_sync_status(stream);
}

namespace {

// Copy streams and events of the pipelined host entry point, created once per device.
struct CopyLanes {
  cudaStream_t up = nullptr, down = nullptr;
  cudaEvent_t start = nullptr, in[2] = {}, done[2] = {}, out[2] = {};
};

int copy_lanes(int device, CopyLanes** out) {
  static std::mutex mu;
  static CopyLanes lanes[kMaxDevices];
  static bool ready[kMaxDevices] = {};
  std::lock_guard<std::mutex> lock(mu);
  CopyLanes& l = lanes[device];
  if (!ready[device]) {
    cudaError_t e = cudaStreamCreateWithFlags(&l.up, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&l.down, cudaStreamNonBlocking);
    cudaEvent_t* evs[] = {&l.start, &l.in[0], &l.in[1], &l.done[0], &l.done[1], &l.out[0],
                          &l.out[1]};
    for (cudaEvent_t* ev : evs)
      if (e == cudaSuccess) e = cudaEventCreateWithFlags(ev, cudaEventDisableTiming);
    if (e != cudaSuccess)
      return set_error(H3B_ECUDA, "denoise_host_pipelined: stream/event creation: %s",
                       cudaGetErrorString(e));
    ready[device] = true;
  }
  *out = &l;
  return 0;
}

}  // namespace

int h3b_denoise_host_pipelined(const h3b_dims* dims, const h3b_grid* grid, int n_blocks,
                               const h3b_block_weights* blocks, const unsigned char* active,
                               const float* mods, const float* final_mod, int reduce_after,
                               int unpair_bypass, int n_steps, int first_step, int n_run,
                               int n_requests, const float* x_host_in, float* x_host_out,
                               float* x_state_dev, void* ws, size_t ws_bytes, void* stream) {
  StepBufs b;
  int rc = check_step_args(dims, grid, n_blocks, blocks, active, mods, final_mod, reduce_after,
                           x_state_dev, ws, ws_bytes, &b);
  if (rc) return rc;
  if (!x_host_in || !x_host_out || n_requests < 0)
    return set_error(H3B_EINVAL, "denoise_host_pipelined: NULL host buffer or %d requests",
                     n_requests);
  if (n_steps <= 0 || first_step < 0 || n_run < 0 || first_step + n_run > n_steps)
    return set_error(H3B_EINVAL, "denoise_host_pipelined: steps %d..%d of %d", first_step,
                     first_step + n_run, n_steps);
  DevCtx ctx;
  if ((rc = get_ctx(&ctx))) return rc;
  CopyLanes* l = nullptr;
  if ((rc = copy_lanes(ctx.device, &l))) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t elems = (size_t(grid->t) * grid->h * grid->w + grid->n_audio) * dims->d;
  const size_t bytes = elems * sizeof(float);
  auto fail = [](cudaError_t e, const char* what) {
    return set_error(H3B_ECUDA, "denoise_host_pipelined: %s: %s", what, cudaGetErrorString(e));
  };
  cudaError_t e;
  // one captured denoise per state buffer (reused across calls with the same arguments);
  // with H3B_DEBUG the steps are launched directly so that each launch is checked
  cudaGraphExec_t graphs[2] = {nullptr, nullptr};
  if (!debug_mode())
    for (int k = 0; k < 2 && k < n_requests; ++k)
      if ((rc = denoise_graph(ctx, dims, grid, n_blocks, blocks, active, mods, final_mod,
                              reduce_after, unpair_bypass, n_steps, first_step, n_run,
                              x_state_dev + k * elems, b, ws, ws_bytes, &graphs[k])))
        return rc;
  // everything below is ordered after the work already on `stream`
  if ((e = cudaEventRecord(l->start, s)) != cudaSuccess) return fail(e, "record");
  if ((e = cudaStreamWaitEvent(l->up, l->start, 0)) != cudaSuccess) return fail(e, "wait");
  for (int r = 0; r < n_requests; ++r) {
    const int k = r & 1;
    float* state = x_state_dev + k * elems;
    // upload r into state buffer k once request r - 2 has been downloaded from it
    if (r >= 2 && (e = cudaStreamWaitEvent(l->up, l->out[k], 0)) != cudaSuccess)
      return fail(e, "wait");
    if ((e = cudaMemcpyAsync(state, x_host_in + r * elems, bytes, cudaMemcpyHostToDevice,
                             l->up)) != cudaSuccess)
      return fail(e, "H2D");
    if ((e = cudaEventRecord(l->in[k], l->up)) != cudaSuccess) return fail(e, "record");
    if ((e = cudaStreamWaitEvent(s, l->in[k], 0)) != cudaSuccess) return fail(e, "wait");
    if (graphs[k]) {
      if ((e = cudaGraphLaunch(graphs[k], s)) != cudaSuccess) return fail(e, "graph launch");
    } else {
      for (int i = first_step; i < first_step + n_run; ++i) {
        const float sg = static_cast<float>(1.0 - double(i) / n_steps);
        const float sn = static_cast<float>(1.0 - double(i + 1) / n_steps);
        if ((rc = denoise_step_impl(ctx, dims, grid, n_blocks, blocks, active, mods, final_mod,
                                    reduce_after, unpair_bypass, sg, sn, state, b, s)))
          return rc;
      }
    }
    if ((e = cudaEventRecord(l->done[k], s)) != cudaSuccess) return fail(e, "record");
    if ((e = cudaStreamWaitEvent(l->down, l->done[k], 0)) != cudaSuccess) return fail(e, "wait");
    if ((e = cudaMemcpyAsync(x_host_out + r * elems, state, bytes, cudaMemcpyDeviceToHost,
                             l->down)) != cudaSuccess)
      return fail(e, "D2H");
    if ((e = cudaEventRecord(l->out[k], l->down)) != cudaSuccess) return fail(e, "record");
  }
  // the call ends on `stream` after the last download
  for (int k = 0; k < 2 && k < n_requests; ++k)
    if ((e = cudaStreamWaitEvent(s, l->out[(n_requests - 1 - k) & 1], 0)) != cudaSuccess)
      return fail(e, "wait");
  return h3b_sync_status(stream);
}

int h3b_token_reduce(int mode, const h3b_bf16* src, h3b_bf16* dst, const h3b_bf16* saved, int t,
                     int h, int w, int n_audio, int d, void* stream) {
  if (mode != H3B_PAIR && mode != H3B_UNPAIR) return set_error(H3B_EINVAL, "token_reduce: mode %d", mode);
  if (t < 0 || h < 0 || w < 0 || (w & 1) || n_audio < 0 || d <= 0 || d % 8)
    return set_error(H3B_EINVAL, "token_reduce: bad sizes (t=%d h=%d w=%d audio=%d d=%d)", t, h, w, n_audio, d);
  if (!src || !dst || !al16(src) || !al16(dst) || (saved && !al16(saved)))
    return set_error(H3B_EINVAL, "token_reduce: NULL or misaligned pointer");
  if (mode == H3B_PAIR && saved) return set_error(H3B_EINVAL, "token_reduce: saved is for UNPAIR");
  if (src == dst) return set_error(H3B_EINVAL, "token_reduce: src and dst must differ");
  DevCtx ctx;
  if (int rc = get_ctx(&ctx)) return rc;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (mode == H3B_PAIR)
    return launch_token_pair(reinterpret_cast<const bf16*>(src), reinterpret_cast<bf16*>(dst), t,
                             h, w, n_audio, d, s);
  return launch_token_unpair(reinterpret_cast<const bf16*>(src), reinterpret_cast<bf16*>(dst),
                             reinterpret_cast<const bf16*>(saved), t, h, w, n_audio, d, s);
}

int h3b_quantize_rows(const h3b_bf16* a, int rows, int cols, int8_t* q, float* scale,
                      void* stream) {
  if (rows < 0 || cols <= 0 || cols % 16 || cols > 32768)
    return set_error(H3B_EINVAL, "quantize_rows: cols=%d must be a multiple of 16 <= 32768", cols);
  if (!a || !q || !scale || !al16(a) || !al16(q))
    return set_error(H3B_EINVAL, "quantize_rows: NULL or misaligned pointer");
  DevCtx ctx;
  if (int rc = get_ctx(&ctx)) return rc;
  return launch_quantize_rows(reinterpret_cast<const bf16*>(a), rows, cols, q, scale,
                              static_cast<cudaStream_t>(stream));
}

int h3b_fc2_int8_row(const h3b_bf16* act, int M, int K, int n_out, const int8_t* w_q,
                     const float* w_scale, const float* bias, const float* gate, h3b_bf16* resid,
                     int8_t* act_q, float* row_scale, int32_t* acc_out, void* ws,
                     size_t ws_bytes, void* stream) {
  if (M < 0 || K <= 0 || K % 128 || K > 32768 || n_out <= 0 || n_out % 128)
    return set_error(H3B_EINVAL, "fc2_int8_row: K=%d must be a multiple of 128 <= 32768, n_out=%d a multiple of 128", K, n_out);
  const void* ptrs[7] = {act, w_q, w_scale, gate, resid, act_q, row_scale};
  for (const void* p : ptrs)
    if (!p || !al16(p)) return set_error(H3B_EINVAL, "fc2_int8_row: NULL or misaligned pointer");
  if ((bias && !al16(bias)) || (acc_out && !al16(acc_out)))
    return set_error(H3B_EINVAL, "fc2_int8_row: misaligned bias / acc_out");
  DevCtx ctx;
  int rc;
  if ((rc = get_ctx(&ctx))) return rc;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  if ((rc = launch_quantize_rows(reinterpret_cast<const bf16*>(act), M, K, act_q, row_scale, s)))
    return rc;
  GemmEpilogue e;
  e.kind = kEpiInt8Deq;
  e.bias_f32 = bias;
  e.gate = gate;
  e.out = reinterpret_cast<bf16*>(resid);
  e.ld_out = n_out;
  e.row_scale = row_scale;
  e.col_scale = w_scale;
  e.acc_out = acc_out;
  if (ws && !al16(ws)) return set_error(H3B_EINVAL, "fc2_int8_row: misaligned workspace");
  return launch_gemm_i8(ctx, act_q, w_q, M, n_out, K, e, ws, ws_bytes, s);
}

int h3b_gemm_bf16(const h3b_bf16* A, const h3b_bf16* B, int M, int N, int K, int epilogue,
                  const h3b_bf16* bias, const float* gate, const float* rope_cs, int rope_cols,
                  int head_dim, h3b_bf16* out, void* ws, size_t ws_bytes, void* stream) {
  if (M < 0 || K <= 0 || K % 64 || N <= 0 || N % 128)
    return set_error(H3B_EINVAL, "gemm_bf16: K=%d must be a multiple of 64, N=%d of 128", K, N);
  if (epilogue < H3B_EPI_BIAS || epilogue > H3B_EPI_GATE_RESID)
    return set_error(H3B_EINVAL, "gemm_bf16: epilogue %d", epilogue);
  if (!A || !B || !bias || !out || !al16(A) || !al16(B) || !al16(bias) || !al16(out))
    return set_error(H3B_EINVAL, "gemm_bf16: NULL or misaligned pointer");
  if (epilogue == H3B_EPI_GATE_RESID && (!gate || !al16(gate)))
    return set_error(H3B_EINVAL, "gemm_bf16: gate required");
  if (epilogue == H3B_EPI_BIAS_ROPE &&
      (!rope_cs || !al16(rope_cs) || (head_dim != 64 && head_dim != 128) || rope_cols < 0 ||
       rope_cols % head_dim || rope_cols > N))
    return set_error(H3B_EINVAL, "gemm_bf16: bad RoPE arguments");
  DevCtx ctx;
  if (int rc = get_ctx(&ctx)) return rc;
  GemmEpilogue e;
  e.kind = epilogue;
  e.bias = reinterpret_cast<const bf16*>(bias);
  e.gate = gate;
  e.rope_cs = rope_cs;
  e.rope_cols = rope_cols;
  e.head_dim = head_dim;
  e.out = reinterpret_cast<bf16*>(out);
  e.ld_out = N;
  if (ws && !al16(ws)) return set_error(H3B_EINVAL, "gemm_bf16: misaligned workspace");
  return launch_gemm_bf16(ctx, reinterpret_cast<const bf16*>(A), reinterpret_cast<const bf16*>(B),
                          M, N, K, e, ws, ws_bytes, static_cast<cudaStream_t>(stream));
}

int h3b_gemm_bf16_ln(const h3b_bf16* A, const h3b_bf16* B, int M, int N, int K, int epilogue,
                     const h3b_bf16* bias, const float* gate, const float* fold_c,
                     const float* fold_dv, const float* stats_in, float* stats_out,
                     float ln_eps, const float* rope_cs, int rope_cols, int head_dim,
                     const float* q_gain, const float* k_gain, h3b_bf16* out, void* ws,
                     size_t ws_bytes, void* stream) {
  if (M < 0 || K <= 0 || K % 64 || N <= 0 || N % 128)
    return set_error(H3B_EINVAL, "gemm_bf16_ln: K=%d must be a multiple of 64, N=%d of 128", K, N);
  if (!A || !B || !out || !al16(A) || !al16(B) || !al16(out) || (ws && !al16(ws)))
    return set_error(H3B_EINVAL, "gemm_bf16_ln: NULL or misaligned pointer");
  GemmEpilogue e;
  e.out = reinterpret_cast<bf16*>(out);
  e.ld_out = N;
  if (epilogue == H3B_EPI_LN_ROPE || epilogue == H3B_EPI_LN_GELU) {
    if (K % 256 || K > 4096 || !fold_c || !fold_dv || !stats_in || !al16(fold_c) ||
        !al16(fold_dv) || !al16(stats_in) || !(ln_eps > 0.f))
      return set_error(H3B_EINVAL, "gemm_bf16_ln: LN-folded form needs K %% 256 == 0, c, dv, stats_in, eps > 0");
    if (epilogue == H3B_EPI_LN_ROPE &&
        (!rope_cs || !al16(rope_cs) || (head_dim != 64 && head_dim != 128) || rope_cols < 0 ||
         rope_cols % head_dim || rope_cols > N))
      return set_error(H3B_EINVAL, "gemm_bf16_ln: bad RoPE arguments");
    e.kind = epilogue == H3B_EPI_LN_ROPE ? kEpiRopeLN : kEpiGeluLN;
    e.fold_c = fold_c;
    e.bias_f32 = fold_dv;
    e.stats_in = reinterpret_cast<const float2*>(stats_in);
    e.stats_parts = K / 256;
    e.ln_eps = ln_eps;
    e.rope_cs = rope_cs;
    e.rope_cols = rope_cols;
    e.head_dim = head_dim;
  } else if (epilogue == H3B_EPI_BIAS_ROPE) {
    if (!bias || !al16(bias) || !rope_cs || !al16(rope_cs) || (head_dim != 64 && head_dim != 128) ||
        rope_cols < 0 || rope_cols % head_dim || rope_cols > N)
      return set_error(H3B_EINVAL, "gemm_bf16_ln: bad bias / RoPE arguments");
    e.kind = kEpiRope;
    e.bias = reinterpret_cast<const bf16*>(bias);
    e.ln_eps = ln_eps;
    e.rope_cs = rope_cs;
    e.rope_cols = rope_cols;
    e.head_dim = head_dim;
  } else if (epilogue == H3B_EPI_GATE_RESID) {
    if (!bias || !gate || !al16(bias) || !al16(gate) || (stats_out && (N % 256 || !al16(stats_out))))
      return set_error(H3B_EINVAL, "gemm_bf16_ln: gated residual needs bias, gate (and N %% 256 == 0 for stats)");
    e.kind = kEpiGateResid;
    e.bias = reinterpret_cast<const bf16*>(bias);
    e.gate = gate;
    e.stats_out = reinterpret_cast<float2*>(stats_out);
  } else {
    return set_error(H3B_EINVAL, "gemm_bf16_ln: epilogue %d", epilogue);
  }
  if ((q_gain == nullptr) != (k_gain == nullptr) ||
      (q_gain && (e.kind != kEpiRope && e.kind != kEpiRopeLN)) ||
      (q_gain && (!al16(q_gain) || !al16(k_gain) || e.rope_cols % 2 || (e.rope_cols / 2) % e.head_dim)))
    return set_error(H3B_EINVAL, "gemm_bf16_ln: q_gain / k_gain need a RoPE form, both or neither");
  e.q_gain = q_gain;
  e.k_gain = k_gain;
  DevCtx ctx;
  if (int rc = get_ctx(&ctx)) return rc;
  return launch_gemm_bf16(ctx, reinterpret_cast<const bf16*>(A), reinterpret_cast<const bf16*>(B),
                          M, N, K, e, ws, ws_bytes, static_cast<cudaStream_t>(stream));
}

int h3b_attention(const h3b_bf16* qkv, int n_tokens, int n_heads, int head_dim, h3b_bf16* out,
                  void* ws, size_t ws_bytes, void* stream) {
  if (n_tokens < 0 || n_heads <= 0 || (head_dim != 64 && head_dim != 128))
    return set_error(H3B_EINVAL, "attention: bad sizes (n=%d heads=%d hd=%d)", n_tokens, n_heads, head_dim);
  if (!qkv || !out || !al16(qkv) || !al16(out) || (ws && !al16(ws)))
    return set_error(H3B_EINVAL, "attention: NULL or misaligned pointer");
  DevCtx ctx;
  if (int rc = get_ctx(&ctx)) return rc;
  return launch_attention(ctx, reinterpret_cast<const bf16*>(qkv), n_tokens, n_heads, head_dim,
                          reinterpret_cast<bf16*>(out), ws, ws_bytes,
                          static_cast<cudaStream_t>(stream));
}

int h3b_layer_mask(const float* mods_host, int n_blocks, int d, int n_active,
                   unsigned char* mask_out) {
  if (!mods_host || !mask_out || n_blocks <= 0 || d <= 0)
    return set_error(H3B_EINVAL, "layer_mask: bad arguments");
  const int n_drop = n_blocks - n_active;
  if (n_drop > 0 && n_drop > n_blocks - 2)
    return set_error(H3B_EINVAL, "layer_mask: the first and last blocks are always kept");
  for (int b = 0; b < n_blocks; ++b) mask_out[b] = 1;
  if (n_drop <= 0) return H3B_OK;
  std::vector<std::pair<double, int>> score;
  for (int b = 1; b < n_blocks - 1; ++b) {
    const float* m = mods_host + size_t(b) * 6 * d;
    double ga = 0.0, gm = 0.0;
    for (int j = 0; j < d; ++j) {
      ga += std::fabs(double(m[2 * d + j]));
      gm += std::fabs(double(m[5 * d + j]));
    }
    score.emplace_back(ga / d + gm / d, b);
  }
  std::sort(score.begin(), score.end(), [](const auto& a, const auto& b) {
    return a.first != b.first ? a.first < b.first : a.second > b.second;
  });
  for (int i = 0; i < n_drop; ++i) mask_out[score[i].second] = 0;
  return H3B_OK;
}

}  // extern "C"
