/*
 * h3b -- B200 (sm_100a) DiT-block denoising path: public C ABI.
 *
 * The library computes the transformer-block forward inside the Euler denoising loop of a
 * MiniMax-H3-style video+audio diffusion model: AdaLN-modulated LayerNorm, QKV projection,
 * 3D RoPE over the (t, h, w) token grid, joint video+audio self-attention, an output
 * projection whose gated residual feeds the MLP's AdaLN, a GELU MLP whose gated residual
 * feeds the next block's AdaLN, the per-stream final AdaLN and the Euler update; plus
 * horizontal token pairing and an int8 row-scaled FC2.
 *
 * Sources, cited by page title and section:
 *   "How h3.c cuts MiniMax-H3 video inference to 3.5 seconds" (dothoosh.com), sections
 *     "DiT fusions and memory management", "Aggressive optimisation levers",
 *     "The powerful int8 path";
 *   "H3-metal: running MiniMax-H3 directly on Apple Silicon" (aihot.vn, README
 *     translation), sections 2 "First fast video", 4 "Speed/quality presets",
 *     5 "Resolution and duration";
 *   "h3: native MiniMax-H3 on Apple Silicon" (news.ditty.ir).
 *
 * Conventions for every entry point:
 *   - Pointers marked "device" are CUDA device pointers owned by the caller; pointers
 *     marked "host" are host pointers.  The library never allocates or frees device
 *     memory (h3b_denoise_host_pipelined creates two copy streams and a few events per
 *     device on its first call and keeps them).
 *   - Tensors are dense row-major; "[a, b]" means b is the contiguous dimension.
 *     Every device pointer must be 16-byte aligned.
 *   - h3b_bf16 is bfloat16 storage (IEEE-754 binary32 with the low 16 bits dropped).
 *   - `stream` is a cudaStream_t passed as void*; NULL means the legacy default stream.
 *     Calls are asynchronous on that stream; no host synchronisation happens inside
 *     (except h3b_sync_status, h3b_denoise_host and h3b_denoise_host_pipelined).
 *   - Return value: H3B_OK (0) or a negative H3B_E* code.  All argument validation
 *     happens before the first launch, so a call that fails validation launches
 *     nothing.  h3b_last_error() returns a message for the calling thread's last error.
 *   - Device-side waits inside the kernels give up after about two seconds; the kernel
 *     then returns early and records the event in a per-device flag, which the next
 *     h3b_sync_status call reports as H3B_ETIMEOUT.  The outputs of that work are
 *     invalid, and so are split-schedule flags it left in the caller's workspace: when
 *     h3b_sync_status reports H3B_ETIMEOUT the library drops its cached denoise graphs
 *     (the next host call captures fresh ones with new sequence numbers); a CUDA graph
 *     the caller captured around library calls must be captured again too.
 *   - Per device, the library caches the device addresses of its module variables, its
 *     copy streams and its captured graphs for the life of the process; it assumes the
 *     device's primary context lives as long (cudaDeviceReset while the library is in
 *     use is not supported).
 */
#ifndef H3B_H_
#define H3B_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define H3B_VERSION 1

enum {
  H3B_OK = 0,
  H3B_EINVAL = -1,        /* bad sizes, layout or alignment */
  H3B_EWORKSPACE = -2,    /* workspace missing or smaller than the size function says */
  H3B_ECUDA = -3,         /* a CUDA runtime call or kernel launch failed */
  H3B_ETIMEOUT = -4,      /* a device-side wait gave up (reported by h3b_sync_status) */
  H3B_EUNSUPPORTED = -5   /* the current device is not sm_100 */
};

typedef uint16_t h3b_bf16;

/* Model dimensions.  d = n_heads * head_dim; head_dim is 64 or 128; rope_split are the
 * widths of the (t, h, w) chunks of the head dimension (even, summing to head_dim);
 * d % 256 == 0, d <= 4096, d_ff % 256 == 0, c_dim % 8 == 0. */
typedef struct h3b_dims {
  int d;
  int n_heads;
  int head_dim;
  int d_ff;
  int c_dim;
  int rope_split[3];
  float rope_theta;   /* RoPE base, 10000 in the workloads */
  float ln_eps;       /* LayerNorm epsilon, 1e-6 */
} h3b_dims;

/* Token grid: video tokens (t, h, w) in raster order, then n_audio audio tokens.
 * rope_halved != 0 halves the spatial RoPE coordinates (small-canvas variant: aihot.vn
 * README section 5).  Audio tokens sit at RoPE position (0, 0, 0). */
typedef struct h3b_grid {
  int t, h, w;
  int n_audio;
  int rope_halved;
} h3b_grid;

/* Parameters of one block (device, bf16).  Weights are [out, in]: w_qkv [3d, d] (q rows,
 * then k, then v; head j at rows j*head_dim), w_o [d, d], w_fc1 [d_ff, d], w_fc2 [d, d_ff];
 * biases b_qkv [3d], b_o [d], b_fc1 [d_ff], b_fc2 [d].
 *
 * The last six fields are optional (all NULL = absent): the block's two AdaLN
 * modulations folded into the projections that consume them, as h3b_fold_adaln writes
 * them -- w_qkv_fold [3d, d] bf16 with c_qkv, d_qkv [3d] fp32 from (shift_msa,
 * scale_msa); w_fc1_fold [d_ff, d] bf16 with c_fc1, d_fc1 [d_ff] fp32 from (shift_mlp,
 * scale_mlp).  With them the block reads the raw residual and no LayerNorm pass runs
 * (h3b_block_forward_folded; h3b_denoise_step uses them when every active block has
 * them).  h3b_block_forward ignores them.
 *
 * q_norm, k_norm (optional, both or neither): per-head RMSNorm gains [head_dim] fp32 for
 * q and k.  When present, every head of q and k is normalised inside the QKV
 * projection's epilogue, before the rotation: q_h <- q_h / sqrt(mean(q_h^2) + ln_eps) *
 * q_norm (dothoosh.com, "The powerful int8 path": RMS normalisation and RoPE for Q/K in
 * the QKV tile). */
typedef struct h3b_block_weights {
  const h3b_bf16* w_qkv;
  const h3b_bf16* b_qkv;
  const h3b_bf16* w_o;
  const h3b_bf16* b_o;
  const h3b_bf16* w_fc1;
  const h3b_bf16* b_fc1;
  const h3b_bf16* w_fc2;
  const h3b_bf16* b_fc2;
  const h3b_bf16* w_qkv_fold;
  const float* c_qkv;
  const float* d_qkv;
  const h3b_bf16* w_fc1_fold;
  const float* c_fc1;
  const float* d_fc1;
  const float* q_norm;
  const float* k_norm;
} h3b_block_weights;

/* ---------------------------------------------------------------- library information */
int h3b_version(void);
const char* h3b_last_error(void);

/* Number of kernels this library has launched in this process (all devices, all
 * threads), for launch accounting by callers. */
uint64_t h3b_launch_count(void);

/* Synchronise `stream`, then read and clear this device's wait-timeout flag.
 * Returns H3B_OK, H3B_ETIMEOUT (a kernel gave up waiting; its outputs are invalid) or
 * H3B_ECUDA (an asynchronous CUDA error). */
int h3b_sync_status(void* stream);

/* ---------------------------------------------------------------- workspace sizes */
/* Bytes of workspace h3b_block_forward needs for n_tokens tokens.  One arena, laid out by
 * lifetime: the QKV and attention-output regions are reused for the MLP hidden
 * activations (dothoosh.com, "DiT fusions and memory management": activation arenas
 * aliased by lifetime). */
size_t h3b_workspace_size(const h3b_dims* dims, int n_tokens);

/* Bytes of the optional scratch that lets h3b_gemm_bf16 and h3b_fc2_int8_row use the
 * stream-K schedule (K loop split across all SMs when the output tiles do not fill the
 * SMs evenly).  The block and step workspaces already include it. */
size_t h3b_gemm_workspace_size(void);

/* Bytes of workspace h3b_denoise_step needs for this grid; reduce != 0 adds the paired
 * stream's buffers. */
size_t h3b_denoise_workspace_size(const h3b_dims* dims, const h3b_grid* grid, int reduce);

/* ---------------------------------------------------------------- diagnostics */
/* The GEMM kernels' work schedule, computed on the host by the same functions the kernels
 * run (no GPU, no CUDA call): the work items of scheduling unit `unit` (a CTA pair of the
 * pair kernel, a CTA of the single-SM kernel) out of `units`, for `tiles` output tiles of
 * `k_blocks` K slices each.  mode: 0 data-parallel; 1 hybrid stream-K (the pair kernel's
 * form: whole waves but the last data-parallel, the rest split evenly); 2 stream-K over
 * every tile (the single-SM kernel's form); 3 remainder stream-K (the grouped int8 kernel's
 * form, K slices being its 1024-column groups: every whole wave data-parallel, the tiles
 * past them split evenly).  Item i goes to items[4 i .. 4 i + 3] (host,
 * caller-owned) as (tile, first K slice, end K slice, merge), in processing order: merge
 * is -1 for a partial tile the unit parks for a higher unit, else the first unit whose
 * parked partial the item's epilogue adds (the unit itself when it adds none).  At most
 * max_items items are written.  Returns the number of items, or H3B_EINVAL for
 * non-positive sizes, a unit outside [0, units), a mode outside 0-3, a missing buffer, or
 * a stream-K mode with fewer than 4 split K slices per unit (mode 3: fewer than one, or
 * no partial wave past at least one whole one); the GEMM calls run those shapes
 * data-parallel. */
int h3b_gemm_schedule(int tiles, int k_blocks, int units, int mode, int unit, int* items,
                      int max_items);

/* Force the GEMM dispatch for every later GEMM launch of this process, for measurements
 * and tests (the automatic choice is the product path; this call exists so that each
 * tile configuration and schedule can be exercised and timed on purpose, in place of
 * environment switches).  -1 restores the automatic choice for that field.
 *   tile:  0 CTA-pair 256-wide, 1 CTA-pair 128-wide, 2 single-CTA 256, 3 single-CTA 128
 *          (used where the shape allows it);
 *   sched: 0 data-parallel, 1 hybrid stream-K, 2 stream-K over every tile (where the
 *          scratch allows it and each unit gets at least 4 split K slices);
 *   trans: 0 never, 1 always use the transposed pair kernel where the shape allows it.
 * Returns H3B_OK, or H3B_EINVAL (nothing changed) for a value out of range.  Applies to
 * launches issued after the call, on every thread; a CUDA graph keeps the launches it
 * captured. */
int h3b_set_gemm_override(int tile, int sched, int trans);

/* Select the attention kernel's form for later launches of this process, for tests and
 * measurements: 0 automatic (the default: two 128-query tiles per CTA sharing each K/V
 * tile, one softmax warpgroup each), 1 one query tile per CTA, 2 two tiles, 3 two tiles
 * with a quarter of the exponentials on the FMA pipe (a cubic on the reduced argument)
 * instead of the MUFU unit.  Returns H3B_OK or H3B_EINVAL. */
int h3b_set_attention_variant(int variant);

/* ---------------------------------------------------------------- hot-path steps */
/* AdaLN modulation vectors: mod[j] = sum_k w[j, k] c[k] + b[j], j < n_out.
 * w [n_out, c_dim] bf16, b [n_out] bf16, c [c_dim] bf16, mod [n_out] fp32 (all device).
 * A block's six vectors are rows of mod [6, d] in the order shift_msa, scale_msa,
 * gate_msa, shift_mlp, scale_mlp, gate_mlp; a stream's final pair is (shift, scale).
 * (dothoosh.com, "DiT fusions and memory management" and "Aggressive optimisation
 * levers": per-block AdaLN gates.) */
int h3b_adaln_modulation(const h3b_bf16* w, const h3b_bf16* b, const h3b_bf16* c,
                         int n_out, int c_dim, float* mod, void* stream);

/* RoPE cos/sin table for a grid: rope_cs [n_tokens, head_dim / 2, 2] fp32 (device),
 * entry (i, p) = (cos a, sin a) of pair p of token i.  Pair p lies in the chunk of axis
 * x (t, h, w in that order); with k its index inside the chunk of width D_x,
 * a = pos_x(i) * rope_theta^(-2k / D_x).  paired != 0 builds the table of the paired
 * grid (w / 2 columns, merged token j at w = 2j + 0.5).  n_tokens = t*h*w (or t*h*(w/2)
 * when paired) + n_audio.  (aihot.vn README section 5: spatial RoPE coordinates.) */
int h3b_rope_table(const h3b_dims* dims, const h3b_grid* grid, int paired, float* rope_cs,
                   void* stream);

/* LayerNorm (no affine, biased variance) + AdaLN modulation:
 * h = LN(x) * (1 + scale) + shift.  x, h [n_tokens, d] bf16; shift, scale [d] fp32.
 * x and h must not overlap. */
int h3b_ln_modulate(const h3b_bf16* x, int n_tokens, int d, float eps, const float* shift,
                    const float* scale, h3b_bf16* h, void* stream);

/* One DiT block (dothoosh.com, "DiT fusions and memory management"):
 *   h  = LN(x)(1 + scale_msa) + shift_msa          (computed here iff compute_h != 0,
 *                                                     else h must already hold it)
 *   qkv = h W_qkv^T + b_qkv; q, k rotated by RoPE (rope_cs from h3b_rope_table)
 *   o  = softmax(q k^T / sqrt(head_dim)) v           per head, all tokens, no mask
 *   x  = x + gate_msa (o W_o^T + b_o)                (in place, bf16)
 *   h  = LN(x)(1 + scale_mlp) + shift_mlp
 *   x  = x + gate_mlp (GELU_tanh(h W_fc1^T + b_fc1) W_fc2^T + b_fc2)
 *   h  = LN(x)(1 + mod_next.scale_msa) + mod_next.shift_msa     iff mod_next != NULL
 * mod, mod_next: [6, d] fp32 device; x, h: [n_tokens, d] bf16 device (in/out);
 * ws: device workspace of at least h3b_workspace_size(dims, n_tokens) bytes. */
int h3b_block_forward(const h3b_dims* dims, const h3b_block_weights* w, const float* mod,
                      const float* mod_next, const float* rope_cs, int n_tokens,
                      int compute_h, h3b_bf16* x, h3b_bf16* h, void* ws, size_t ws_bytes,
                      void* stream);

/* AdaLN folded into the projection that consumes it (dothoosh.com, "DiT fusions and
 * memory management": the attention gate fused with the MLP AdaLN, the MLP gate producing
 * the next block's attention AdaLN).  For h = LN(x)(1 + scale) + shift (LN without affine,
 * biased variance) feeding y = h W^T + b:
 *   y[r, j] = rstd_r (sum_k x[r, k] W'[j, k] - mean_r c_j) + dv_j,  with
 *   W'[j, k] = bf16(W[j, k] (1 + scale_k)),  c_j = sum_k W'[j, k] (over the stored W'),
 *   dv_j = sum_k shift_k W[j, k] + b_j.
 * Exact in real arithmetic whenever the modulation vectors are fixed for the run (they are
 * here: the conditioning vector is constant over the steps).  w [n_out, d] bf16, b [n_out]
 * bf16, shift, scale [d] fp32; outputs w_out [n_out, d] bf16 (must not overlap w), c_out,
 * dv_out [n_out] fp32; all device, d % 8 == 0.  Run once per block per conditioning:
 * (shift_msa, scale_msa) with w_qkv, (shift_mlp, scale_mlp) with w_fc1. */
int h3b_fold_adaln(const h3b_bf16* w, const h3b_bf16* b, const float* shift, const float* scale,
                   int n_out, int d, h3b_bf16* w_out, float* c_out, float* dv_out,
                   void* stream);

/* Row statistics of the residual in the form the folded block consumes and produces:
 * stats [n_tokens, d / 256] float2, per row and 256-column group (mean, M2) of the bf16
 * values (M2 = sum of squared deviations from the group mean).  x [n_tokens, d] bf16
 * device, d % 256 == 0.  (The denoise step computes these itself.) */
int h3b_row_stats(const h3b_bf16* x, int n_tokens, int d, float* stats, void* stream);

/* One DiT block with both AdaLN LayerNorms folded into the projections (the folded fields
 * of w, from h3b_fold_adaln with this block's mod):
 *   qkv = the folded QKV of x (reads x and its row statistics `stats`), RoPE in the epilogue
 *   o   = attention; x = x + gate_msa (o W_o^T + b_o), the epilogue writing x's new
 *         row statistics into stats
 *   g   = GELU of the folded FC1 of x (reads x and stats)
 *   x   = x + gate_mlp (g W_fc2^T + b_fc2), the epilogue writing the new statistics
 * The result equals h3b_block_forward's x up to rounding; no h is produced: the next
 * block (folded) reads x and stats.  mod [6, d] fp32 (the gates); x [n_tokens, d] bf16
 * in/out; stats [n_tokens, d / 256] float2 in/out (see h3b_row_stats); ws as
 * h3b_block_forward.  All device. */
int h3b_block_forward_folded(const h3b_dims* dims, const h3b_block_weights* w, const float* mod,
                             const float* rope_cs, int n_tokens, h3b_bf16* x, float* stats,
                             void* ws, size_t ws_bytes, void* stream);

/* h3b_block_forward without a caller-supplied workspace, for callers that cannot allocate
 * device memory: plug-in hosts that hand a module only its input and output buffers,
 * deployments whose memory plan is fixed before launch, and latency-critical loops that
 * must not call cudaMalloc (it can synchronise the device).  The paper has no
 * counterpart; the block math, arguments and results are those of h3b_block_forward.
 *
 * The workspace is one static device array of H3B_NOALLOC_WORKSPACE_BYTES (64 MiB) inside
 * the library; every GPU that loads the library holds it until the process exits.  A call
 * needs h3b_workspace_size(dims, n_tokens) bytes of it (at d = 3072, d_ff = 12288 that is
 * 1,877 tokens at most) and returns H3B_EWORKSPACE, launching nothing, when the block does
 * not fit.  The first call on a device looks up the array's device address (make that
 * first call before any stream capture).  All calls share the array and nothing in it has
 * to start at zero (every region is written before it is read); calls whose executions
 * overlap on the GPU -- concurrent streams, or threads sharing a device -- race on it, so
 * serialise them.  Nothing here allocates or frees memory. */
#define H3B_NOALLOC_WORKSPACE_BYTES (64u << 20)
int h3b_block_forward_noalloc(const h3b_dims* dims, const h3b_block_weights* w,
                              const float* mod, const float* mod_next, const float* rope_cs,
                              int n_tokens, int compute_h, h3b_bf16* x, h3b_bf16* h,
                              void* stream);

/* Per-stream final AdaLN fused with the Euler update (dothoosh.com, "DiT fusions and
 * memory management": final AdaLN bound to the video/audio offsets of one residual
 * buffer; aihot.vn section 2: linear sigma grid):
 *   v = LN(x_l)(1 + scale_s) + shift_s, s = video for rows < n_video, else audio;
 *   x_state += (sigma_next - sigma) v.
 * x_l [n_tokens, d] bf16; final_mod [2 streams, 2 (shift, scale), d] fp32;
 * x_state [n_tokens, d] fp32 (in/out); all device. */
int h3b_final_euler(const h3b_bf16* x_l, int n_tokens, int n_video, int d, float eps,
                    const float* final_mod, float sigma, float sigma_next, float* x_state,
                    void* stream);

/* One Euler step of the denoising loop over all active blocks:
 *   x = bf16(x_state); for each active block b: h3b_block_forward (or, when every active
 *   block carries its folded weights, h3b_block_forward_folded); after `reduce_after`
 *   executed blocks (if > 0 and blocks remain) pair horizontal video tokens; restore
 *   before the final AdaLN (bypass restore if unpair_bypass, else duplicate);
 *   x_state += (sigma_next - sigma) final_adaln(x).
 * blocks: host array of n_blocks weight sets; active: host [n_blocks] (NULL = all);
 * mods: device [n_blocks, 6, d] fp32; final_mod: device [2, 2, d] fp32;
 * x_state: device [n_tokens, d] fp32, n_tokens = t*h*w + n_audio;
 * ws: device, at least h3b_denoise_workspace_size(dims, grid, reduce_after > 0).
 * (ditty.ir and dothoosh.com "Aggressive optimisation levers": token pairing after
 * block 3, layer thinning; aihot.vn section 2: --steps N means exactly N passes.) */
int h3b_denoise_step(const h3b_dims* dims, const h3b_grid* grid, int n_blocks,
                     const h3b_block_weights* blocks, const unsigned char* active,
                     const float* mods, const float* final_mod, int reduce_after,
                     int unpair_bypass, float sigma, float sigma_next, float* x_state,
                     void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------- latent steps */
/* The steps on either side of the block stack (dothoosh.com, "DiT fusions and memory
 * management": the final BF16 heads apply the AdaLN as they load their tiles; aihot.vn
 * section 4: the patch and head work around the core).  The state is a per-token latent
 * [n_tokens, c_lat] fp32; each stream (video rows, then audio rows) has its own patch
 * embedding and head.  w_head_fold[s], c_head[s], dv_head[s] are the stream's head with
 * its final AdaLN folded in (h3b_fold_adaln with the stream's final (shift, scale)). */
typedef struct h3b_latent_heads {
  int c_lat;                          /* latent channels per token, multiple of 128 */
  const h3b_bf16* w_patch[2];         /* [d, c_lat] bf16, per stream (video, audio) */
  const h3b_bf16* b_patch[2];         /* [d] bf16 */
  const h3b_bf16* w_head_fold[2];     /* [c_lat, d] bf16 */
  const float* c_head[2];             /* [c_lat] fp32 */
  const float* dv_head[2];            /* [c_lat] fp32 */
} h3b_latent_heads;

/* Bytes of workspace h3b_denoise_step_latent needs (0 on bad arguments). */
size_t h3b_denoise_latent_workspace_size(const h3b_dims* dims, const h3b_grid* grid, int reduce,
                                         int c_lat);

/* One Euler step on the latent:
 *   x = bf16(bf16(latent) W_patch,s^T + b_patch,s)   (GEMM per stream; its epilogue also
 *       writes x's row statistics)
 *   every active block in its folded form (each must carry its folded weights), with the
 *   token pairing / restore of h3b_denoise_step
 *   latent += (sigma_next - sigma) ((LN(x_L)(1 + scale_s) + shift_s) W_head,s^T + b_head,s)
 *       (the head GEMM per stream applies the folded final AdaLN and the Euler update in
 *       its epilogue; no normalised activation is stored).
 * latent: device [n_tokens, c_lat] fp32 in/out; mods: device [n_blocks, 6, d];
 * ws: h3b_denoise_latent_workspace_size bytes. */
int h3b_denoise_step_latent(const h3b_dims* dims, const h3b_grid* grid, int n_blocks,
                            const h3b_block_weights* blocks, const unsigned char* active,
                            const float* mods, const h3b_latent_heads* heads, int reduce_after,
                            int unpair_bypass, float sigma, float sigma_next, float* latent,
                            void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------- reuse policies */
/* Whole-velocity reuse and core-residual reuse (dothoosh.com, "Aggressive optimisation
 * levers"; aihot.vn section 4 "Speed/quality presets": --reuse and --core-reuse; the two
 * are mutually exclusive).  The schedule: step i of `steps` runs the model when
 * i % every == 0, and the last step always does (20 steps: every = 1, 2, 3 give 20, 11,
 * 8 fresh evaluations, the counts the pages print).  fresh_out: host [steps], 1 = run
 * the model.  Returns the number of fresh steps, or H3B_EINVAL. */
int h3b_reuse_schedule(int steps, int every, unsigned char* fresh_out);

/* h3b_denoise_step that also keeps what a skipped step needs: v_out [n_tokens, d] fp32,
 * the velocity the step applied (whole-velocity reuse); core_res_out [n_tokens, d] fp32,
 * the block stack's residual r = x_L - bf16(x_state) with x_state the step's input
 * (core-residual reuse).  Either may be NULL; device. */
int h3b_denoise_step_keep(const h3b_dims* dims, const h3b_grid* grid, int n_blocks,
                          const h3b_block_weights* blocks, const unsigned char* active,
                          const float* mods, const float* final_mod, int reduce_after,
                          int unpair_bypass, float sigma, float sigma_next, float* x_state,
                          float* v_out, float* core_res_out, void* ws, size_t ws_bytes,
                          void* stream);

/* A skipped step of whole-velocity reuse: x_state += (sigma_next - sigma) v, with v the
 * last fresh step's velocity.  v, x_state [n_tokens, d] fp32 device; d % 4 == 0. */
int h3b_euler_velocity(const float* v, int n_tokens, int d, float sigma, float sigma_next,
                       float* x_state, void* stream);

/* A skipped step of core-residual reuse: the block stack is replaced by the residual of the
 * last fresh step, x_L = bf16(bf16(x_state) + core_res); the final AdaLN and the Euler
 * update run as in h3b_final_euler.  core_res, x_state [n_tokens, d] fp32; final_mod
 * [2, 2, d] fp32; all device. */
int h3b_euler_core_reuse(const float* core_res, int n_tokens, int n_video, int d, float eps,
                         const float* final_mod, float sigma, float sigma_next, float* x_state,
                         void* stream);

/* Whole denoise from a HOST latent: copies x_host_in [n_tokens, d] fp32 to the device,
 * runs Euler steps first_step .. first_step + n_run - 1 of the linear grid with n_steps
 * intervals (sigma_i = 1 - i / n_steps), copies the state back into x_host_out and
 * synchronises `stream`.  x_state_dev: device [n_tokens, d] fp32 scratch for the state.
 * Host buffers should be pinned for full copy bandwidth.  The steps run as a CUDA graph
 * captured on the first call with these arguments (see h3b_denoise_host_pipelined). */
int h3b_denoise_host(const h3b_dims* dims, const h3b_grid* grid, int n_blocks,
                     const h3b_block_weights* blocks, const unsigned char* active,
                     const float* mods, const float* final_mod, int reduce_after,
                     int unpair_bypass, int n_steps, int first_step, int n_run,
                     const float* x_host_in, float* x_host_out, float* x_state_dev,
                     void* ws, size_t ws_bytes, void* stream);

/* Serving form of h3b_denoise_host: n_requests independent whole denoises of HOST
 * latents, request r read from x_host_in + r * n_tokens * d and written to
 * x_host_out + r * n_tokens * d ([n_requests, n_tokens, d] fp32, pinned for full copy
 * bandwidth).  Request r computes on `stream` while the library's copy streams upload
 * request r + 1 and download request r - 1, so the copies overlap the compute; every
 * request still makes its own host-to-device and device-to-host trip.  x_state_dev:
 * device [2, n_tokens, d] fp32 (two state buffers, alternating).  The work is ordered
 * after what `stream` already holds, and `stream` is synchronised before returning.
 * Each request's Euler steps run as a CUDA graph captured on the first call with these
 * arguments (the library keeps the last four per device; H3B_DEBUG=1 launches directly).
 * Calls on one device must not overlap (the copy streams are shared).  No counterpart
 * on the pages: the host-side pipelining of a serving loop around the denoise. */
int h3b_denoise_host_pipelined(const h3b_dims* dims, const h3b_grid* grid, int n_blocks,
                               const h3b_block_weights* blocks, const unsigned char* active,
                               const float* mods, const float* final_mod, int reduce_after,
                               int unpair_bypass, int n_steps, int first_step, int n_run,
                               int n_requests, const float* x_host_in, float* x_host_out,
                               float* x_state_dev, void* ws, size_t ws_bytes, void* stream);

/* Horizontal token pairing (ditty.ir; dothoosh.com "Aggressive optimisation levers").
 * mode H3B_PAIR:   dst[t,h,j] = (src[t,h,2j] + src[t,h,2j+1]) / 2, audio rows copied;
 *                  src [t*h*w + n_audio, d], dst [t*h*(w/2) + n_audio, d].
 * mode H3B_UNPAIR: dst[t,h,2j+k] = saved[t,h,2j+k] + (src[t,h,j] - pair(saved)[t,h,j])
 *                  when saved != NULL (bypass restore; pair(saved) rounded to bf16 as
 *                  H3B_PAIR would store it), else dst[t,h,2j+k] = src[t,h,j];
 *                  audio rows copied; src is the paired stream, dst and saved full.
 *                  dst may equal saved (in place).
 * All bf16 device; w must be even; averages and corrections in fp32, one rounding. */
enum { H3B_PAIR = 0, H3B_UNPAIR = 1 };
int h3b_token_reduce(int mode, const h3b_bf16* src, h3b_bf16* dst, const h3b_bf16* saved,
                     int t, int h, int w, int n_audio, int d, void* stream);

/* Symmetric int8 quantisation, one fp32 scale per row (aihot.vn section 4 and
 * dothoosh.com "The powerful int8 path": one activation scale per FC2 row):
 * absmax = max|a_row|; q = clamp(rne(a * (127 / absmax)), -127, 127) with IEEE fp32
 * division and multiply; scale = absmax / 127; a zero row gives q = 0, scale = 0.
 * a [rows, cols] bf16, q [rows, cols] int8, scale [rows] fp32 (device); cols % 16 == 0.
 * Used for FC2 activations (rows = tokens) and for weights (rows = output channels). */
int h3b_quantize_rows(const h3b_bf16* a, int rows, int cols, int8_t* q, float* scale,
                      void* stream);

/* Int8 row-scaled FC2 with gated residual (aihot.vn section 4, --use-int8-row-fc2):
 *   act_q, row_scale = h3b_quantize_rows(act);
 *   acc = act_q w_q^T (int32, exact);  y = float(acc) * row_scale[m] * w_scale[n] (+ bias[n]);
 *   resid = bf16(resid + gate[n] y).
 * act [M, K] bf16; w_q [n_out, K] int8; w_scale, gate [n_out] fp32; bias [n_out] fp32 or
 * NULL; resid [M, n_out] bf16 in/out; act_q [M, K] int8 and row_scale [M] fp32 outputs;
 * acc_out [M, n_out] int32 output or NULL.  All device.  K % 128 == 0,
 * n_out % 128 == 0.  ws: NULL, or device scratch of h3b_gemm_workspace_size() bytes that
 * enables the stream-K schedule (the result is the same either way: int32 sums are exact). */
int h3b_fc2_int8_row(const h3b_bf16* act, int M, int K, int n_out, const int8_t* w_q,
                     const float* w_scale, const float* bias, const float* gate,
                     h3b_bf16* resid, int8_t* act_q, float* row_scale, int32_t* acc_out,
                     void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------- int8 block path */
/* Weights of one block on the int8 path (dothoosh.com, "The powerful int8 path": int8
 * MLP with dynamic activation quantisation and per-output-channel weight scales, the FC2
 * input with one scale per 1024 channels, quantised QKV).  Weights [out, in] int8 from
 * h3b_quantize_rows of the bf16 weights, with their per-output-channel scales [out] fp32.
 * The biases, the output projection and the Q/K norm gains come from h3b_block_weights. */
typedef struct h3b_int8_block {
  const int8_t* w_qkv_q;   /* [3d, d] */
  const float* s_qkv;      /* [3d] */
  const int8_t* w_fc1_q;   /* [d_ff, d] */
  const float* s_fc1;      /* [d_ff] */
  const int8_t* w_fc2_q;   /* [d, d_ff] */
  const float* s_fc2;      /* [d] */
} h3b_int8_block;

/* Bytes of workspace h3b_block_forward_int8 needs (0 on bad arguments; d_ff % 1024). */
size_t h3b_workspace_size_int8(const h3b_dims* dims, int n_tokens);

/* One DiT block on the int8 path:
 *   hq, hs = quantise_rows(LN(x)(1 + scale_msa) + shift_msa)      (one fused kernel)
 *   qkv    = rope(rmsnorm?((hq w_qkv_q^T) hs s_qkv + b_qkv))          (int8 GEMM epilogue)
 *   o      = attention (bf16);  x = x + gate_msa (o W_o^T + b_o)  (bf16)
 *   hq, hs = quantise_rows(LN(x)(1 + scale_mlp) + shift_mlp)
 *   g      = GELU((hq w_fc1_q^T) hs s_fc1 + b_fc1)                   (bf16)
 *   gq, gs = quantise_groups(g), one scale per row and 1024 channels
 *   x      = x + gate_mlp (s_fc2 sum_groups gs acc_group + b_fc2)   (grouped int8 GEMM)
 * Quantisation: the rule of h3b_quantize_rows.  mod [6, d] fp32; x [n_tokens, d] bf16
 * in/out; ws: h3b_workspace_size_int8 bytes.  All device.  d_ff % 1024 == 0. */
int h3b_block_forward_int8(const h3b_dims* dims, const h3b_block_weights* w,
                           const h3b_int8_block* wq, const float* mod, const float* rope_cs,
                           int n_tokens, h3b_bf16* x, void* ws, size_t ws_bytes, void* stream);

/* h = LN(x)(1 + scale) + shift (fp32) quantised per row: q [n_tokens, d] int8,
 * q_scale [n_tokens] fp32 (the rule of h3b_quantize_rows); x bf16.  All device. */
int h3b_ln_modulate_q8(const h3b_bf16* x, int n_tokens, int d, float eps, const float* shift,
                       const float* scale, int8_t* q, float* q_scale, void* stream);

/* The rule of h3b_quantize_rows applied to every 1024-column group of every row:
 * a [rows, cols] bf16, q [rows, cols] int8, scale [rows, cols / 1024] fp32; cols % 1024
 * == 0.  All device. */
int h3b_quantize_groups(const h3b_bf16* a, int rows, int cols, int8_t* q, float* scale,
                        void* stream);

/* The grouped int8 FC2 with gated residual:
 *   resid = bf16(resid + gate (w_scale[n] sum_g a_scale[m, g] acc_g[m, n] + bias[n])),
 *   acc_g = the exact int32 product of group g (1024 K columns) of A [M, K] and w_q [N, K].
 * a_scale [M, K / 1024], w_scale, gate [N] fp32; bias [N] bf16 or NULL; resid [M, N]
 * bf16 in/out.  All device.  K % 1024 == 0, N % 128 == 0.  ws: NULL, or ws_bytes >=
 * h3b_gemm_workspace_size() of device scratch, which lets a partial last wave of tiles run
 * stream-K over the groups (the same sums, added in a fixed order); one call at a time per
 * scratch. */
int h3b_gemm_i8_grouped(const int8_t* A, const float* a_scale, int M, int K, int N,
                        const int8_t* w_q, const float* w_scale, const h3b_bf16* bias,
                        const float* gate, h3b_bf16* resid, void* ws, size_t ws_bytes,
                        void* stream);

/* ---------------------------------------------------------------- single kernels */
/* The projection GEMM used by the block: out = A B^T with an epilogue.
 * A [M, K] bf16, B [N, K] bf16 (device), K % 64 == 0, N % 128 == 0.
 *   H3B_EPI_BIAS:       out[M, N] = bf16(acc + bias)
 *   H3B_EPI_BIAS_GELU:  out = bf16(GELU_tanh(acc + bias))
 *   H3B_EPI_BIAS_ROPE:  out = bf16(rope(acc + bias)) on columns < rope_cols (pairs of
 *                       adjacent columns, head_dim-periodic, table rope_cs), plain after
 *   H3B_EPI_GATE_RESID: out = bf16(out + gate (acc + bias)), in place (out is the residual)
 * bias [N] bf16; gate [N] fp32 (GATE_RESID only); rope_cs as h3b_rope_table.
 * ws: NULL, or device scratch of h3b_gemm_workspace_size() bytes enabling stream-K. */
enum { H3B_EPI_BIAS = 0, H3B_EPI_BIAS_GELU = 1, H3B_EPI_BIAS_ROPE = 2, H3B_EPI_GATE_RESID = 3 };
int h3b_gemm_bf16(const h3b_bf16* A, const h3b_bf16* B, int M, int N, int K, int epilogue,
                  const h3b_bf16* bias, const float* gate, const float* rope_cs,
                  int rope_cols, int head_dim, h3b_bf16* out, void* ws, size_t ws_bytes,
                  void* stream);

/* The projection GEMM in the forms of the folded block path (h3b_block_forward_folded) and
 * with the Q/K RMSNorm:
 *   H3B_EPI_LN_ROPE, H3B_EPI_LN_GELU: A [M, K] is the raw bf16 residual and B the folded
 *     weights (h3b_fold_adaln); pre[r, j] = rstd_r (acc - mean_r fold_c[j]) + fold_dv[j],
 *     with mean_r and rstd_r = 1 / sqrt(var_r + ln_eps) merged from stats_in
 *     [M, K / 256] (h3b_row_stats form), then RoPE on columns < rope_cols (as
 *     H3B_EPI_BIAS_ROPE) or GELU_tanh; K % 256 == 0.  bias and gate are unused.
 *   H3B_EPI_BIAS_ROPE: as in h3b_gemm_bf16.
 *   H3B_EPI_GATE_RESID: as in h3b_gemm_bf16, and the output rows' group statistics go to
 *     stats_out [M, N / 256] (h3b_row_stats form) when it is not NULL; N % 256 == 0.
 * q_gain, k_gain (RoPE forms only; both or neither): each head_dim slice of columns
 * [0, rope_cols / 2) (q) and [rope_cols / 2, rope_cols) (k) is RMS-normalised with
 * eps = ln_eps and multiplied by the gains [head_dim] before the rotation (as the block
 * does with q_norm, k_norm).
 * fold_c, fold_dv [N] fp32; other arguments as h3b_gemm_bf16.  All device. */
enum { H3B_EPI_LN_ROPE = 4, H3B_EPI_LN_GELU = 5 };
int h3b_gemm_bf16_ln(const h3b_bf16* A, const h3b_bf16* B, int M, int N, int K, int epilogue,
                     const h3b_bf16* bias, const float* gate, const float* fold_c,
                     const float* fold_dv, const float* stats_in, float* stats_out,
                     float ln_eps, const float* rope_cs, int rope_cols, int head_dim,
                     const float* q_gain, const float* k_gain, h3b_bf16* out, void* ws,
                     size_t ws_bytes, void* stream);

/* Joint self-attention over one packed QKV buffer: qkv [n_tokens, 3 n_heads head_dim]
 * bf16 (q, then k, then v; head j at column j*head_dim of each), out [n_tokens,
 * n_heads head_dim] bf16 (device).  out = softmax(q k^T / sqrt(head_dim)) v per head.
 * ws: NULL, or 16-byte aligned device scratch of h3b_gemm_workspace_size() bytes (the
 * same scratch the GEMM calls take; one kernel at a time per buffer).  With it the work
 * is split evenly over the SMs (a query block may be finished by two CTAs, merged through
 * the scratch); without it, one CTA per (head, query block).  A query block is 256 rows
 * (two 128-row tiles sharing each K/V load; see h3b_set_attention_variant).  A smaller
 * ws is ignored. */
int h3b_attention(const h3b_bf16* qkv, int n_tokens, int n_heads, int head_dim,
                  h3b_bf16* out, void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------- host policy */
/* Layer thinning mask (dothoosh.com "Aggressive optimisation levers": rank blocks by
 * their AdaLN gates, always keep the first and last block).  score_b = mean|gate_msa| +
 * mean|gate_mlp| from mods_host [n_blocks, 6, d] fp32 (host); the n_blocks - n_active
 * lowest-scoring interior blocks are dropped, the higher index first on ties.
 * mask_out: host [n_blocks], 1 = active. */
int h3b_layer_mask(const float* mods_host, int n_blocks, int d, int n_active,
                   unsigned char* mask_out);

#ifdef __cplusplus
}
#endif

#endif /* H3B_H_ */
