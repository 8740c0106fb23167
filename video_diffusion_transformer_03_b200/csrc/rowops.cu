// Memory-bound kernels of the path: LayerNorm + AdaLN modulation (a warp per token row,
// 16-byte vector loads, the row held in registers for an exact two-pass mean/variance,
// warp-shuffle reductions), the per-stream final AdaLN fused with the Euler update,
// horizontal token pairing and its bypass restore, the int8 row quantiser, the AdaLN
// modulation GEMV and the RoPE cos/sin table.
#include "kernels.h"
#include "ptx.cuh"

#include <algorithm>
#include <cmath>

namespace h3b {

namespace {

constexpr int kRowWarps = 4;  // rows per 128-thread block

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

__device__ __forceinline__ void unpack8(const uint4& u, float (&f)[8]) {
  float2 a = unpack_bf16x2(u.x), b = unpack_bf16x2(u.y), c = unpack_bf16x2(u.z),
         d = unpack_bf16x2(u.w);
  f[0] = a.x; f[1] = a.y; f[2] = b.x; f[3] = b.y; f[4] = c.x; f[5] = c.y; f[6] = d.x; f[7] = d.y;
}
__device__ __forceinline__ uint4 pack8(const float (&f)[8]) {
  uint4 u;
  u.x = pack_bf16x2(f[0], f[1]);
  u.y = pack_bf16x2(f[2], f[3]);
  u.z = pack_bf16x2(f[4], f[5]);
  u.w = pack_bf16x2(f[6], f[7]);
  return u;
}
__device__ __forceinline__ void load8f(const float* p, float (&f)[8]) {
  const float4 a = __ldg(reinterpret_cast<const float4*>(p));
  const float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
  f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w; f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
}

// Mean and reciprocal standard deviation of one row held as NV x 8 values per lane
// (biased variance, two passes over registers).
template <int NV>
__device__ __forceinline__ void row_stats(const float (&v)[NV][8], int d, float eps,
                                          float& mean, float& rstd) {
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < NV; ++i)
#pragma unroll
    for (int k = 0; k < 8; ++k) s += v[i][k];
  mean = warp_sum(s) / static_cast<float>(d);
  float q = 0.f;
#pragma unroll
  for (int i = 0; i < NV; ++i)
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const float t = v[i][k] - mean;
      q = fmaf(t, t, q);
    }
  const float var = warp_sum(q) / static_cast<float>(d);
  rstd = rsqrtf(var + eps);
}

// h = LN(x)(1 + scale) + shift.  FROM_STATE: x is the fp32 state; it is first rounded to
// bf16 (the block input) and written to x_res.
template <int NV, bool FROM_STATE>
__global__ void __launch_bounds__(128) k_ln_modulate(const void* __restrict__ xin, int n,
                                                     float eps, const float* __restrict__ shift,
                                                     const float* __restrict__ scale,
                                                     bf16* __restrict__ x_res,
                                                     bf16* __restrict__ h) {
  constexpr int D = NV * 256;
  const int row = blockIdx.x * kRowWarps + (threadIdx.x >> 5);
  if (row >= n) return;
  const int lane = threadIdx.x & 31;
  float v[NV][8];
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    const int col = (i * 32 + lane) * 8;
    if constexpr (FROM_STATE) {
      const float* xs = static_cast<const float*>(xin) + size_t(row) * D + col;
      float f[8];
      load8f(xs, f);
      const uint4 u = pack8(f);
      reinterpret_cast<uint4*>(x_res + size_t(row) * D + col)[0] = u;
      unpack8(u, v[i]);
    } else {
      const bf16* xb = static_cast<const bf16*>(xin) + size_t(row) * D + col;
      unpack8(__ldg(reinterpret_cast<const uint4*>(xb)), v[i]);
    }
  }
  float mean, rstd;
  row_stats<NV>(v, D, eps, mean, rstd);
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    const int col = (i * 32 + lane) * 8;
    float sh[8], sc[8], o[8];
    load8f(shift + col, sh);
    load8f(scale + col, sc);
#pragma unroll
    for (int k = 0; k < 8; ++k) o[k] = fmaf((v[i][k] - mean) * rstd, 1.0f + sc[k], sh[k]);
    reinterpret_cast<uint4*>(h + size_t(row) * D + col)[0] = pack8(o);
  }
}

// Symmetric int8 code of v with inv = 127 / absmax (IEEE fp32 multiply, round to nearest
// even, clamp): the rule of k_quantize_rows.
__device__ __forceinline__ uint32_t q8x4(float a, float b, float c, float d, float inv) {
  const int qa = max(-127, min(127, __float2int_rn(__fmul_rn(a, inv))));
  const int qb = max(-127, min(127, __float2int_rn(__fmul_rn(b, inv))));
  const int qc = max(-127, min(127, __float2int_rn(__fmul_rn(c, inv))));
  const int qd = max(-127, min(127, __float2int_rn(__fmul_rn(d, inv))));
  return (static_cast<uint32_t>(qa) & 0xFFu) | ((static_cast<uint32_t>(qb) & 0xFFu) << 8) |
         ((static_cast<uint32_t>(qc) & 0xFFu) << 16) | ((static_cast<uint32_t>(qd) & 0xFFu) << 24);
}

// LayerNorm + AdaLN fused with the int8 quantisation of its output (the int8 path's input
// to QKV and FC1): h = LN(x)(1 + scale) + shift in fp32, then one scale per row,
// absmax / 127, and q = clamp(rne(h * (127 / absmax))).  The row stays in registers.
template <int NV>
__global__ void __launch_bounds__(128) k_ln_modulate_q8(const bf16* __restrict__ x, int n,
                                                        float eps, const float* __restrict__ shift,
                                                        const float* __restrict__ scale,
                                                        int8_t* __restrict__ q,
                                                        float* __restrict__ q_scale) {
  constexpr int D = NV * 256;
  const int row = blockIdx.x * kRowWarps + (threadIdx.x >> 5);
  if (row >= n) return;
  const int lane = threadIdx.x & 31;
  float v[NV][8];
#pragma unroll
  for (int i = 0; i < NV; ++i)
    unpack8(__ldg(reinterpret_cast<const uint4*>(x + size_t(row) * D + (i * 32 + lane) * 8)), v[i]);
  float mean, rstd;
  row_stats<NV>(v, D, eps, mean, rstd);
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    const int col = (i * 32 + lane) * 8;
    float sh[8], sc[8];
    load8f(shift + col, sh);
    load8f(scale + col, sc);
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      v[i][k] = fmaf((v[i][k] - mean) * rstd, 1.0f + sc[k], sh[k]);
      amax = fmaxf(amax, fabsf(v[i][k]));
    }
  }
  amax = warp_max(amax);
  const float inv = amax > 0.f ? __fdiv_rn(127.0f, amax) : 0.0f;
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    const int col = (i * 32 + lane) * 8;
    reinterpret_cast<uint2*>(q + size_t(row) * D + col)[0] =
        make_uint2(q8x4(v[i][0], v[i][1], v[i][2], v[i][3], inv),
                   q8x4(v[i][4], v[i][5], v[i][6], v[i][7], inv));
  }
  if (lane == 0) q_scale[row] = amax > 0.f ? __fdiv_rn(amax, 127.0f) : 0.0f;
}

// Group quantisation: a warp per (row, 1024-column group) of a [rows, cols] bf16 matrix,
// the rule of k_quantize_rows within each group; scale [rows, cols / 1024].
__global__ void __launch_bounds__(256) k_quantize_groups(const bf16* __restrict__ a, int rows,
                                                         int cols, int8_t* __restrict__ q,
                                                         float* __restrict__ scale) {
  constexpr int G = 1024;
  const int groups = cols / G;
  const long long gw = blockIdx.x * 8ll + (threadIdx.x >> 5);
  if (gw >= static_cast<long long>(rows) * groups) return;
  const int row = static_cast<int>(gw / groups), g = static_cast<int>(gw % groups);
  const int lane = threadIdx.x & 31;
  const uint4* src = reinterpret_cast<const uint4*>(a + size_t(row) * cols + size_t(g) * G);
  float v[4][8];
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    unpack8(__ldg(src + i * 32 + lane), v[i]);
#pragma unroll
    for (int k = 0; k < 8; ++k) amax = fmaxf(amax, fabsf(v[i][k]));
  }
  amax = warp_max(amax);
  const float inv = amax > 0.f ? __fdiv_rn(127.0f, amax) : 0.0f;
  uint2* dst = reinterpret_cast<uint2*>(q + size_t(row) * cols + size_t(g) * G);
#pragma unroll
  for (int i = 0; i < 4; ++i)
    dst[i * 32 + lane] = make_uint2(q8x4(v[i][0], v[i][1], v[i][2], v[i][3], inv),
                                    q8x4(v[i][4], v[i][5], v[i][6], v[i][7], inv));
  if (lane == 0) scale[size_t(row) * groups + g] = amax > 0.f ? __fdiv_rn(amax, 127.0f) : 0.0f;
}

// v = LN(x_l)(1 + scale_s) + shift_s (s = video below n_video, else audio);
// x_state += dt * v.
template <int NV>
__global__ void __launch_bounds__(128) k_final_euler(const bf16* __restrict__ xl, int n,
                                                     int n_video, float eps,
                                                     const float* __restrict__ fmod,
                                                     float dt, float* __restrict__ xs) {
  constexpr int D = NV * 256;
  const int row = blockIdx.x * kRowWarps + (threadIdx.x >> 5);
  if (row >= n) return;
  const int lane = threadIdx.x & 31;
  float v[NV][8];
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    const int col = (i * 32 + lane) * 8;
    unpack8(__ldg(reinterpret_cast<const uint4*>(xl + size_t(row) * D + col)), v[i]);
  }
  float mean, rstd;
  row_stats<NV>(v, D, eps, mean, rstd);
  const float* shift = fmod + (row < n_video ? 0 : 2 * D);
  const float* scale = shift + D;
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    const int col = (i * 32 + lane) * 8;
    float sh[8], sc[8];
    load8f(shift + col, sh);
    load8f(scale + col, sc);
    float4* st = reinterpret_cast<float4*>(xs + size_t(row) * D + col);
    float4 a = st[0], b = st[1];
    float x8[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const float vel = fmaf((v[i][k] - mean) * rstd, 1.0f + sc[k], sh[k]);
      x8[k] = fmaf(dt, vel, x8[k]);
    }
    st[0] = make_float4(x8[0], x8[1], x8[2], x8[3]);
    st[1] = make_float4(x8[4], x8[5], x8[6], x8[7]);
  }
}

// The final AdaLN + Euler step of the reuse policies.  !CORE_IN: as k_final_euler on
// x_l, also storing the velocity (v_out) and the core residual r = x_l - bf16(x_state)
// (r_out) when those are not null.  CORE_IN: a skipped core, x_l = bf16(bf16(x_state) +
// r_in) built in registers.
template <int NV, bool CORE_IN>
__global__ void __launch_bounds__(128) k_final_euler_ex(const bf16* __restrict__ xl,
                                                        const float* __restrict__ r_in, int n,
                                                        int n_video, float eps,
                                                        const float* __restrict__ fmod,
                                                        float dt, float* __restrict__ xs,
                                                        float* __restrict__ v_out,
                                                        float* __restrict__ r_out) {
  constexpr int D = NV * 256;
  const int row = blockIdx.x * kRowWarps + (threadIdx.x >> 5);
  if (row >= n) return;
  const int lane = threadIdx.x & 31;
  float v[NV][8];
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    const size_t off = size_t(row) * D + (i * 32 + lane) * 8;
    if constexpr (CORE_IN) {
      float f[8], x_in[8], r[8];
      load8f(xs + off, f);
      unpack8(pack8(f), x_in);
      load8f(r_in + off, r);
#pragma unroll
      for (int k = 0; k < 8; ++k) f[k] = x_in[k] + r[k];
      unpack8(pack8(f), v[i]);
    } else {
      unpack8(__ldg(reinterpret_cast<const uint4*>(xl + off)), v[i]);
      if (r_out) {
        float f[8], x_in[8];
        load8f(xs + off, f);
        unpack8(pack8(f), x_in);
        float4* ro = reinterpret_cast<float4*>(r_out + off);
        ro[0] = make_float4(v[i][0] - x_in[0], v[i][1] - x_in[1], v[i][2] - x_in[2], v[i][3] - x_in[3]);
        ro[1] = make_float4(v[i][4] - x_in[4], v[i][5] - x_in[5], v[i][6] - x_in[6], v[i][7] - x_in[7]);
      }
    }
  }
  float mean, rstd;
  row_stats<NV>(v, D, eps, mean, rstd);
  const float* shift = fmod + (row < n_video ? 0 : 2 * D);
  const float* scale = shift + D;
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    const int col = (i * 32 + lane) * 8;
    const size_t off = size_t(row) * D + col;
    float sh[8], sc[8], vel[8];
    load8f(shift + col, sh);
    load8f(scale + col, sc);
#pragma unroll
    for (int k = 0; k < 8; ++k) vel[k] = fmaf((v[i][k] - mean) * rstd, 1.0f + sc[k], sh[k]);
    if (!CORE_IN && v_out) {
      float4* vo = reinterpret_cast<float4*>(v_out + off);
      vo[0] = make_float4(vel[0], vel[1], vel[2], vel[3]);
      vo[1] = make_float4(vel[4], vel[5], vel[6], vel[7]);
    }
    float4* st = reinterpret_cast<float4*>(xs + off);
    float4 a = st[0], b = st[1];
    st[0] = make_float4(fmaf(dt, vel[0], a.x), fmaf(dt, vel[1], a.y), fmaf(dt, vel[2], a.z),
                        fmaf(dt, vel[3], a.w));
    st[1] = make_float4(fmaf(dt, vel[4], b.x), fmaf(dt, vel[5], b.y), fmaf(dt, vel[6], b.z),
                        fmaf(dt, vel[7], b.w));
  }
}

// dst = bf16(src) over n8 groups of 8 values (the latent as a GEMM operand).
__global__ void __launch_bounds__(256) k_f32_to_bf16(const float* __restrict__ src, long long n8,
                                                     bf16* __restrict__ dst) {
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n8;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    float f[8];
    load8f(src + i * 8, f);
    reinterpret_cast<uint4*>(dst)[i] = pack8(f);
  }
}

// x_state += dt * v over n4 float4 elements (a skipped step of whole-velocity reuse).
__global__ void __launch_bounds__(256) k_euler_axpy(const float4* __restrict__ v, long long n4,
                                                    float dt, float4* __restrict__ xs) {
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n4;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const float4 a = __ldg(v + i);
    float4 x = xs[i];
    x.x = fmaf(dt, a.x, x.x);
    x.y = fmaf(dt, a.y, x.y);
    x.z = fmaf(dt, a.z, x.z);
    x.w = fmaf(dt, a.w, x.w);
    xs[i] = x;
  }
}

// Statistics of one 256-column group of a row, held as 8 values per lane: the group's
// mean and M2 (sum of squared deviations from it), accumulated about the group's first
// value so that a large common offset does not cancel.  The GEMM epilogues write the
// same (mean, M2) per group for the rows they produce; a consumer merges a row's groups.
__device__ __forceinline__ float2 group_stats(const float (&v)[8]) {
  const float k = __shfl_sync(0xffffffffu, v[0], 0);
  float s1 = 0.f, s2 = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float t = v[i] - k;
    s1 += t;
    s2 = fmaf(t, t, s2);
  }
  s1 = warp_sum(s1);
  s2 = warp_sum(s2);
  return make_float2(k + s1 * (1.0f / 256.0f), s2 - s1 * s1 * (1.0f / 256.0f));
}

// x_res = bf16(x_state) (the block input) and the (mean, M2) of each 256-column group of
// the stored bf16 row: stats [n, D / 256].
template <int NV>
__global__ void __launch_bounds__(128) k_state_to_residual(const float* __restrict__ xs, int n,
                                                           bf16* __restrict__ x_res,
                                                           float2* __restrict__ stats) {
  constexpr int D = NV * 256;
  const int row = blockIdx.x * kRowWarps + (threadIdx.x >> 5);
  if (row >= n) return;
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    const int col = (i * 32 + lane) * 8;
    float f[8], v[8];
    load8f(xs + size_t(row) * D + col, f);
    const uint4 u = pack8(f);
    reinterpret_cast<uint4*>(x_res + size_t(row) * D + col)[0] = u;
    unpack8(u, v);
    const float2 g = group_stats(v);
    if (lane == 0) stats[size_t(row) * NV + i] = g;
  }
}

// (mean, M2) of each 256-column group of the bf16 rows of x: stats [n, D / 256].
template <int NV>
__global__ void __launch_bounds__(128) k_row_stats(const bf16* __restrict__ x, int n,
                                                   float2* __restrict__ stats) {
  constexpr int D = NV * 256;
  const int row = blockIdx.x * kRowWarps + (threadIdx.x >> 5);
  if (row >= n) return;
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    float v[8];
    unpack8(__ldg(reinterpret_cast<const uint4*>(x + size_t(row) * D + (i * 32 + lane) * 8)), v);
    const float2 g = group_stats(v);
    if (lane == 0) stats[size_t(row) * NV + i] = g;
  }
}

// AdaLN folded into the projection that consumes the modulated LayerNorm output: for
// h = LN(x)(1 + scale) + shift and y = h W^T + b,
//   y[r, j] = rstd_r (sum_k x[r, k] W'[j, k] - mean_r c_j) + d_j,
//   W'[j, k] = bf16(W[j, k] (1 + scale_k)),  c_j = sum_k W'[j, k],  d_j = sum_k shift_k W[j, k] + b_j.
// One warp per output row j; c is summed over the stored (rounded) W' so that the mean
// term cancels exactly what the tensor cores accumulate.
__global__ void __launch_bounds__(256) k_fold_adaln(const bf16* __restrict__ w,
                                                    const bf16* __restrict__ b,
                                                    const float* __restrict__ shift,
                                                    const float* __restrict__ scale, int n_out,
                                                    int d, bf16* __restrict__ w_out,
                                                    float* __restrict__ c_out,
                                                    float* __restrict__ d_out) {
  const int j = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (j >= n_out) return;
  const int lane = threadIdx.x & 31;
  const uint4* wr = reinterpret_cast<const uint4*>(w + size_t(j) * d);
  uint4* wo = reinterpret_cast<uint4*>(w_out + size_t(j) * d);
  float cs = 0.f, ds = 0.f;
  for (int v = lane; v < (d >> 3); v += 32) {
    float a[8], sh[8], sc[8], f[8], r[8];
    unpack8(__ldg(wr + v), a);
    load8f(shift + v * 8, sh);
    load8f(scale + v * 8, sc);
#pragma unroll
    for (int k = 0; k < 8; ++k) f[k] = fmaf(a[k], sc[k], a[k]);
    const uint4 u = pack8(f);
    wo[v] = u;
    unpack8(u, r);
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      cs += r[k];
      ds = fmaf(sh[k], a[k], ds);
    }
  }
  cs = warp_sum(cs);
  ds = warp_sum(ds);
  if (lane == 0) {
    c_out[j] = cs;
    d_out[j] = ds + __bfloat162float(b[j]);
  }
}

// Pairing: reduced video token r averages full tokens 2r and 2r + 1 (w is even, so the
// horizontal neighbours (t, h, 2j), (t, h, 2j+1) are consecutive rows).
__global__ void k_token_pair(const bf16* __restrict__ src, bf16* __restrict__ dst, int nv_red,
                             int n_audio, int vecs) {
  const long long idx = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x;
  const long long total = static_cast<long long>(nv_red + n_audio) * vecs;
  if (idx >= total) return;
  const int tok = static_cast<int>(idx / vecs);
  const int vec = static_cast<int>(idx % vecs);
  const uint4* s = reinterpret_cast<const uint4*>(src);
  uint4* o = reinterpret_cast<uint4*>(dst);
  if (tok < nv_red) {
    float a[8], b[8], m[8];
    unpack8(__ldg(s + size_t(2 * tok) * vecs + vec), a);
    unpack8(__ldg(s + size_t(2 * tok + 1) * vecs + vec), b);
#pragma unroll
    for (int k = 0; k < 8; ++k) m[k] = 0.5f * (a[k] + b[k]);
    o[size_t(tok) * vecs + vec] = pack8(m);
  } else {
    o[size_t(tok) * vecs + vec] = __ldg(s + size_t(2 * nv_red + (tok - nv_red)) * vecs + vec);
  }
}

// Restore: full tokens 2r, 2r + 1 from reduced token r; bypass form when saved != null.
__global__ void k_token_unpair(const bf16* __restrict__ src, bf16* dst, const bf16* saved,
                               int nv_red, int n_audio, int vecs) {
  const long long idx = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x;
  const long long total = static_cast<long long>(nv_red + n_audio) * vecs;
  if (idx >= total) return;
  const int tok = static_cast<int>(idx / vecs);
  const int vec = static_cast<int>(idx % vecs);
  const uint4* s = reinterpret_cast<const uint4*>(src);
  uint4* o = reinterpret_cast<uint4*>(dst);
  const uint4 r = __ldg(s + size_t(tok) * vecs + vec);
  if (tok < nv_red) {
    if (saved) {
      const uint4* sv = reinterpret_cast<const uint4*>(saved);
      float x[8], a[8], b[8], pa[8];
      unpack8(r, x);
      unpack8(sv[size_t(2 * tok) * vecs + vec], a);
      unpack8(sv[size_t(2 * tok + 1) * vecs + vec], b);
#pragma unroll
      for (int k = 0; k < 8; ++k) pa[k] = 0.5f * (a[k] + b[k]);
      float pr[8];
      unpack8(pack8(pa), pr);  // the pair value exactly as pairing stores it
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const float delta = x[k] - pr[k];
        a[k] += delta;
        b[k] += delta;
      }
      o[size_t(2 * tok) * vecs + vec] = pack8(a);
      o[size_t(2 * tok + 1) * vecs + vec] = pack8(b);
    } else {
      o[size_t(2 * tok) * vecs + vec] = r;
      o[size_t(2 * tok + 1) * vecs + vec] = r;
    }
  } else {
    o[size_t(2 * nv_red + (tok - nv_red)) * vecs + vec] = r;
  }
}

// One block per row; the row stays in registers (cols <= 256 * 8 * MAXV).
template <int MAXV>
__global__ void __launch_bounds__(256, 3) k_quantize_rows(const bf16* __restrict__ a, int cols,
                                                          int8_t* __restrict__ q,
                                                          float* __restrict__ scale) {
  __shared__ float red[8];
  const int row = blockIdx.x;
  const int nvec = cols >> 3;
  const uint4* src = reinterpret_cast<const uint4*>(a + size_t(row) * cols);
  // the row stays packed (4 registers per 8 values) so that three blocks fit on an SM
  uint4 raw[MAXV];
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < MAXV; ++i) {
    const int vi = i * 256 + threadIdx.x;
    raw[i] = vi < nvec ? __ldg(src + vi) : make_uint4(0u, 0u, 0u, 0u);
  }
#pragma unroll
  for (int i = 0; i < MAXV; ++i) {
    float v[8];
    unpack8(raw[i], v);
#pragma unroll
    for (int k = 0; k < 8; ++k) amax = fmaxf(amax, fabsf(v[k]));
  }
  amax = warp_max(amax);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
  __syncthreads();
  amax = red[0];
#pragma unroll
  for (int w = 1; w < 8; ++w) amax = fmaxf(amax, red[w]);
  const float inv = amax > 0.f ? __fdiv_rn(127.0f, amax) : 0.0f;
  uint2* dst = reinterpret_cast<uint2*>(q + size_t(row) * cols);
#pragma unroll
  for (int i = 0; i < MAXV; ++i) {
    const int vi = i * 256 + threadIdx.x;
    if (vi < nvec) {
      float v[8];
      unpack8(raw[i], v);
      uint32_t w[2] = {0u, 0u};
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        int qi = __float2int_rn(__fmul_rn(v[k], inv));
        qi = max(-127, min(127, qi));
        w[k >> 2] |= (static_cast<uint32_t>(qi) & 0xFFu) << (8 * (k & 3));
      }
      dst[vi] = make_uint2(w[0], w[1]);
    }
  }
  if (threadIdx.x == 0) scale[row] = amax > 0.f ? __fdiv_rn(amax, 127.0f) : 0.0f;
}

// out[j] = sum_k w[j, k] c[k] + b[j]; a warp per output.
__global__ void __launch_bounds__(256) k_adaln_gemv(const bf16* __restrict__ w,
                                                    const bf16* __restrict__ b,
                                                    const bf16* __restrict__ c, int n_out,
                                                    int c_dim, float* __restrict__ out) {
  const int j = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (j >= n_out) return;
  const int lane = threadIdx.x & 31;
  const uint4* wr = reinterpret_cast<const uint4*>(w + size_t(j) * c_dim);
  const uint4* cv = reinterpret_cast<const uint4*>(c);
  float acc = 0.f;
  for (int v = lane; v < (c_dim >> 3); v += 32) {
    float a[8], x[8];
    unpack8(__ldg(wr + v), a);
    unpack8(__ldg(cv + v), x);
#pragma unroll
    for (int k = 0; k < 8; ++k) acc = fmaf(a[k], x[k], acc);
  }
  acc = warp_sum(acc);
  if (lane == 0) out[j] = acc + __bfloat162float(b[j]);
}

// rope_cs[tok, p] = (cos, sin) of pos_axis(tok) * theta^(-2k / D_axis); positions and
// angles in double precision, rounded once to fp32.
__global__ void k_rope_table(int t, int h, int wg, int n_audio, int halved, int paired,
                             int half, int s0, int s1, int s2, double log2_theta,
                             float* __restrict__ cs) {
  const int nv = t * h * wg;
  const long long idx = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x;
  if (idx >= static_cast<long long>(nv + n_audio) * half) return;
  const int tok = static_cast<int>(idx / half);
  const int pi = static_cast<int>(idx % half);
  double pos3[3] = {0.0, 0.0, 0.0};
  if (tok < nv) {
    const int ti = tok / (h * wg);
    const int hi = (tok / wg) % h;
    const int wi = tok % wg;
    pos3[0] = ti;
    pos3[1] = hi;
    pos3[2] = paired ? 2.0 * wi + 0.5 : static_cast<double>(wi);
    if (halved) {
      pos3[1] *= 0.5;
      pos3[2] *= 0.5;
    }
  }
  int axis, k, width;
  if (pi < s0 / 2) {
    axis = 0; k = pi; width = s0;
  } else if (pi < (s0 + s1) / 2) {
    axis = 1; k = pi - s0 / 2; width = s1;
  } else {
    axis = 2; k = pi - (s0 + s1) / 2; width = s2;
  }
  const double freq = exp2(-2.0 * k / width * log2_theta);
  double sn, cn;
  sincos(pos3[axis] * freq, &sn, &cn);
  cs[2 * idx] = static_cast<float>(cn);
  cs[2 * idx + 1] = static_cast<float>(sn);
}

}  // namespace

// ------------------------------------------------------------------------ launchers
#define H3B_NV_SWITCH(NV_EXPR, CALL)                                          \
  switch (NV_EXPR) {                                                          \
    case 1: { constexpr int NV = 1; CALL; } break;                            \
    case 2: { constexpr int NV = 2; CALL; } break;                            \
    case 3: { constexpr int NV = 3; CALL; } break;                            \
    case 4: { constexpr int NV = 4; CALL; } break;                            \
    case 5: { constexpr int NV = 5; CALL; } break;                            \
    case 6: { constexpr int NV = 6; CALL; } break;                            \
    case 7: { constexpr int NV = 7; CALL; } break;                            \
    case 8: { constexpr int NV = 8; CALL; } break;                            \
    case 9: { constexpr int NV = 9; CALL; } break;                            \
    case 10: { constexpr int NV = 10; CALL; } break;                          \
    case 11: { constexpr int NV = 11; CALL; } break;                          \
    case 12: { constexpr int NV = 12; CALL; } break;                          \
    case 13: { constexpr int NV = 13; CALL; } break;                          \
    case 14: { constexpr int NV = 14; CALL; } break;                          \
    case 15: { constexpr int NV = 15; CALL; } break;                          \
    case 16: { constexpr int NV = 16; CALL; } break;                          \
    default: return set_error(-1, "row kernels: d=%d unsupported", (NV_EXPR) * 256); \
  }

int launch_ln_modulate(const bf16* x, int n, int d, float eps, const float* shift,
                       const float* scale, bf16* h, cudaStream_t stream) {
  if (n <= 0) return 0;
  const int grid = (n + kRowWarps - 1) / kRowWarps;
  H3B_NV_SWITCH(d / 256, (k_ln_modulate<NV, false><<<grid, 32 * kRowWarps, 0, stream>>>(
                             x, n, eps, shift, scale, nullptr, h)));
  return check_launch("ln_modulate");
}

int launch_ln_modulate_from_state(const float* x_state, int n, int d, float eps,
                                  const float* shift, const float* scale, bf16* x_res,
                                  bf16* h, cudaStream_t stream) {
  if (n <= 0) return 0;
  const int grid = (n + kRowWarps - 1) / kRowWarps;
  H3B_NV_SWITCH(d / 256, (k_ln_modulate<NV, true><<<grid, 32 * kRowWarps, 0, stream>>>(
                             x_state, n, eps, shift, scale, x_res, h)));
  return check_launch("ln_modulate_from_state");
}

int launch_state_to_residual(const float* x_state, int n, int d, bf16* x_res, float2* stats,
                             cudaStream_t stream) {
  if (n <= 0) return 0;
  const int grid = (n + kRowWarps - 1) / kRowWarps;
  H3B_NV_SWITCH(d / 256, (k_state_to_residual<NV><<<grid, 32 * kRowWarps, 0, stream>>>(
                             x_state, n, x_res, stats)));
  return check_launch("state_to_residual");
}

int launch_row_stats(const bf16* x, int n, int d, float2* stats, cudaStream_t stream) {
  if (n <= 0) return 0;
  const int grid = (n + kRowWarps - 1) / kRowWarps;
  H3B_NV_SWITCH(d / 256, (k_row_stats<NV><<<grid, 32 * kRowWarps, 0, stream>>>(x, n, stats)));
  return check_launch("row_stats");
}

int launch_fold_adaln(const bf16* w, const bf16* b, const float* shift, const float* scale,
                      int n_out, int d, bf16* w_out, float* c_out, float* d_out,
                      cudaStream_t stream) {
  if (n_out <= 0) return 0;
  const int grid = (n_out + 7) / 8;
  k_fold_adaln<<<grid, 256, 0, stream>>>(w, b, shift, scale, n_out, d, w_out, c_out, d_out);
  return check_launch("fold_adaln");
}

int launch_final_euler(const bf16* x_l, int n, int n_video, int d, float eps,
                       const float* final_mod, float dt_sigma, float* x_state,
                       cudaStream_t stream) {
  if (n <= 0) return 0;
  const int grid = (n + kRowWarps - 1) / kRowWarps;
  H3B_NV_SWITCH(d / 256, (k_final_euler<NV><<<grid, 32 * kRowWarps, 0, stream>>>(
                             x_l, n, n_video, eps, final_mod, dt_sigma, x_state)));
  return check_launch("final_euler");
}

int launch_final_euler_keep(const bf16* x_l, int n, int n_video, int d, float eps,
                            const float* final_mod, float dt_sigma, float* x_state, float* v_out,
                            float* r_out, cudaStream_t stream) {
  if (n <= 0) return 0;
  const int grid = (n + kRowWarps - 1) / kRowWarps;
  H3B_NV_SWITCH(d / 256, (k_final_euler_ex<NV, false><<<grid, 32 * kRowWarps, 0, stream>>>(
                             x_l, nullptr, n, n_video, eps, final_mod, dt_sigma, x_state, v_out,
                             r_out)));
  return check_launch("final_euler_keep");
}

int launch_core_reuse_final(const float* r_in, int n, int n_video, int d, float eps,
                            const float* final_mod, float dt_sigma, float* x_state,
                            cudaStream_t stream) {
  if (n <= 0) return 0;
  const int grid = (n + kRowWarps - 1) / kRowWarps;
  H3B_NV_SWITCH(d / 256, (k_final_euler_ex<NV, true><<<grid, 32 * kRowWarps, 0, stream>>>(
                             nullptr, r_in, n, n_video, eps, final_mod, dt_sigma, x_state,
                             nullptr, nullptr)));
  return check_launch("core_reuse_final");
}

int launch_ln_modulate_q8(const bf16* x, int n, int d, float eps, const float* shift,
                          const float* scale, int8_t* q, float* q_scale, cudaStream_t stream) {
  if (n <= 0) return 0;
  const int grid = (n + kRowWarps - 1) / kRowWarps;
  H3B_NV_SWITCH(d / 256, (k_ln_modulate_q8<NV><<<grid, 32 * kRowWarps, 0, stream>>>(
                             x, n, eps, shift, scale, q, q_scale)));
  return check_launch("ln_modulate_q8");
}

int launch_quantize_groups(const bf16* a, int rows, int cols, int8_t* q, float* scale,
                           cudaStream_t stream) {
  const long long warps = static_cast<long long>(rows) * (cols / 1024);
  if (warps <= 0) return 0;
  k_quantize_groups<<<static_cast<unsigned>((warps + 7) / 8), 256, 0, stream>>>(a, rows, cols, q,
                                                                               scale);
  return check_launch("quantize_groups");
}

int launch_f32_to_bf16(const float* src, long long n, bf16* dst, cudaStream_t stream) {
  const long long n8 = n / 8;
  if (n8 <= 0) return 0;
  const int grid = static_cast<int>(std::min<long long>((n8 + 255) / 256, 148 * 8));
  k_f32_to_bf16<<<grid, 256, 0, stream>>>(src, n8, dst);
  return check_launch("f32_to_bf16");
}

int launch_euler_axpy(const float* v, long long n, float dt_sigma, float* x_state,
                      cudaStream_t stream) {
  const long long n4 = n / 4;
  if (n4 <= 0) return 0;
  const int grid = static_cast<int>(std::min<long long>((n4 + 255) / 256, 148 * 8));
  k_euler_axpy<<<grid, 256, 0, stream>>>(reinterpret_cast<const float4*>(v), n4, dt_sigma,
                                         reinterpret_cast<float4*>(x_state));
  return check_launch("euler_axpy");
}

int launch_token_pair(const bf16* src, bf16* dst, int t, int h, int w, int n_audio, int d,
                      cudaStream_t stream) {
  const int nv_red = t * h * (w / 2);
  const long long total = static_cast<long long>(nv_red + n_audio) * (d / 8);
  if (total == 0) return 0;
  const int grid = static_cast<int>((total + 255) / 256);
  k_token_pair<<<grid, 256, 0, stream>>>(src, dst, nv_red, n_audio, d / 8);
  return check_launch("token_pair");
}

int launch_token_unpair(const bf16* src, bf16* dst, const bf16* saved, int t, int h, int w,
                        int n_audio, int d, cudaStream_t stream) {
  const int nv_red = t * h * (w / 2);
  const long long total = static_cast<long long>(nv_red + n_audio) * (d / 8);
  if (total == 0) return 0;
  const int grid = static_cast<int>((total + 255) / 256);
  k_token_unpair<<<grid, 256, 0, stream>>>(src, dst, saved, nv_red, n_audio, d / 8);
  return check_launch("token_unpair");
}

int launch_quantize_rows(const bf16* a, int rows, int cols, int8_t* q, float* scale,
                         cudaStream_t stream) {
  if (rows <= 0) return 0;
  const int nvec = cols / 8;
  if (nvec <= 256 * 2)
    k_quantize_rows<2><<<rows, 256, 0, stream>>>(a, cols, q, scale);
  else if (nvec <= 256 * 8)
    k_quantize_rows<8><<<rows, 256, 0, stream>>>(a, cols, q, scale);
  else if (nvec <= 256 * 16)
    k_quantize_rows<16><<<rows, 256, 0, stream>>>(a, cols, q, scale);
  else
    return set_error(-1, "quantize_rows: cols=%d above 32768", cols);
  return check_launch("quantize_rows");
}

int launch_adaln_gemv(const bf16* w, const bf16* b, const bf16* c, int n_out, int c_dim,
                      float* out, cudaStream_t stream) {
  if (n_out <= 0) return 0;
  const int grid = (n_out + 7) / 8;
  k_adaln_gemv<<<grid, 256, 0, stream>>>(w, b, c, n_out, c_dim, out);
  return check_launch("adaln_gemv");
}

int launch_rope_table(int t, int h, int w, int n_audio, int halved, int paired, int head_dim,
                      const int* split, float theta, float* rope_cs, cudaStream_t stream) {
  const int wg = paired ? w / 2 : w;
  const int half = head_dim / 2;
  const long long total = static_cast<long long>(t * h * wg + n_audio) * half;
  if (total == 0) return 0;
  const int grid = static_cast<int>((total + 255) / 256);
  k_rope_table<<<grid, 256, 0, stream>>>(t, h, wg, n_audio, halved, paired, half, split[0],
                                         split[1], split[2], std::log2(double(theta)),
                                         rope_cs);
  return check_launch("rope_table");
}

}  // namespace h3b
