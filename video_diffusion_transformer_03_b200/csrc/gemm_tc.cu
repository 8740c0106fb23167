// Persistent, warp-specialised tcgen05 GEMMs for the block's projections (QKV, out-proj,
// FC1, FC2) and the int8 row-scaled and grouped FC2:  out = A[M, K] * B[N, K]^T  with a
// fused epilogue.
//
// Main form, a CTA pair (cluster of 2, cta_group::2) per 256 x BN tile:
//   warp 0      TMA producer: 128-byte-swizzled [128 x 128 B] A tiles and [BN/2 x 128 B]
//               B tiles into a STAGES-deep shared-memory ring in each CTA;
//   warp 1      TMEM allocator; in the even CTA the MMA issuer (one thread): 4 x
//               tcgen05.mma per stage into a 256 x BN fp32 / int32 accumulator; two
//               accumulator buffers, so the epilogue of tile i overlaps tile i + 1's MMAs;
//   warps 2..   epilogue (4 warps, 8 for 256-wide tiles): tcgen05.ld of the accumulator
//               (thread = row, 32 columns per load), bias / LayerNorm fold / GELU / RoPE /
//               gated residual / int8 dequant, staged through shared memory, coalesced.
// Single-CTA 128 x BN tiles (192 threads) serve M < 256.  Tiles are visited in groups of
// 16 M-tiles (M fastest) so that CTAs running together share weight tiles in L2; schedules
// data-parallel, stream-K or both (a cost model picks), all waits bounded.
#include "kernels.h"
#include "ptx.cuh"
#include "tmap.h"

#include <algorithm>
#include <atomic>
#include <cstdio>
#include <cstdlib>
#include <random>

namespace h3b {

namespace {

constexpr int kBM = 128;
constexpr int kTransBN = 160;  // token tile of the transposed pair kernel
constexpr int kTileBytesK = 128;  // bytes of K per smem tile row (one swizzle span)
constexpr int kGroupM = 16;

template <int BN>
struct GemmCfg {
  static constexpr int kStages = (BN == 256) ? 4 : 6;
  static constexpr uint32_t kABytes = kBM * kTileBytesK;
  static constexpr uint32_t kBBytes = BN * kTileBytesK;
  static constexpr uint32_t kTmemCols = 2 * BN;
  static constexpr size_t kSmem =
      1024 + size_t(kStages) * (kABytes + kBBytes) + 256;  // align pad + ring + barriers
};

struct GemmParams {
  int M, N, k_blocks, m_tiles, n_tiles;
  int tokens;  // transposed pair kernel: output rows (the B operand's rows); else unused
  // Stream-K: the iterations (tile, k-block) of tiles [sk_tile0, tiles) are cut into one
  // equal contiguous range per scheduling unit (CTA or CTA pair).  Each unit walks its
  // range backwards, tile by tile (k-blocks inside a tile still run forwards), so the
  // partial tile at the end of its range is computed first: the unit stores it in its slot
  // and publishes sk_seq in its flag.  The unit holding the tile's last k-block reaches
  // that tile last and adds the slots of the lower-numbered units that computed the rest
  // of it: waits only ever point at lower-numbered units, which are dispatched first.
  // Tiles [0, sk_tile0), whole waves of one tile per unit, then run data-parallel.
  int sk;
  int sk_tile0;
  long long sk_iters;  // (tiles - sk_tile0) x k_blocks
  uint32_t* sk_slots;            // [gridDim.x][BN / 4][128] uint4 of raw accumulator words
  unsigned long long* sk_flags;  // [gridDim.x][4]
  unsigned long long sk_seq;
  GemmEpilogue epi;
  uint32_t* err;
};

// Stream-K slots are sized for the widest tile (same offsets for every tile width, so
// launches of different widths may share one scratch buffer).  One flag per (CTA,
// epilogue warp): a warp publishes the 32 slot rows it wrote, and the owner's warp with
// the same TMEM lane quarter reads exactly those rows.
static_assert(kSkFlagsOffset >= size_t(kMaxSkCtas) * kBM * 256 * 4,
              "stream-K slots must hold the widest tile");

// Scheduling units are CTAs (single-SM kernel) or CTA pairs (pair kernel): `me` is this
// unit's index and `count` the number of units in the grid.
__host__ __device__ __forceinline__ long long sk_begin(const GemmParams& p, int c, int count) {
  return p.sk_iters * c / count;
}

// Unit whose range contains iteration i (counted from the first stream-K tile).
__host__ __device__ __forceinline__ int sk_owner(const GemmParams& p, long long i, int count) {
  int c = static_cast<int>(i * count / p.sk_iters);
  while (c + 1 < count && sk_begin(p, c + 1, count) <= i) ++c;
  while (c > 0 && sk_begin(p, c, count) > i) --c;
  return c;
}

// Work items of this unit: (tile, k-block range).  Every role walks the same sequence.
struct Sched {
  long long it, it_end;  // stream-K phase
  int tile, dp_end;      // data-parallel phase: tiles me, me + count, ... below dp_end
  int count;
};

__host__ __device__ __forceinline__ void sched_init(const GemmParams& p, Sched& s, int me,
                                                   int count) {
  s.count = count;
  s.tile = me;
  if (p.sk) {
    s.it = sk_begin(p, me, count);
    s.it_end = sk_begin(p, me + 1, count);
    s.dp_end = p.sk_tile0;
  } else {
    s.it = s.it_end = 0;
    s.dp_end = p.m_tiles * p.n_tiles;
  }
}

__host__ __device__ __forceinline__ bool sched_next(const GemmParams& p, Sched& s, int& tile,
                                                    int& kb0, int& kb1) {
  if (s.it_end > s.it) {  // stream-K: backwards over [it, it_end), it_end moves down
    const int rel = static_cast<int>((s.it_end - 1) / p.k_blocks);
    const long long t0 = static_cast<long long>(rel) * p.k_blocks;
    const long long start = s.it > t0 ? s.it : t0;
    tile = p.sk_tile0 + rel;
    kb0 = static_cast<int>(start - t0);
    kb1 = static_cast<int>(s.it_end - t0);
    s.it_end = start;
    return true;
  }
  if (s.tile >= s.dp_end) return false;
  tile = s.tile;
  kb0 = 0;
  kb1 = p.k_blocks;
  s.tile += s.count;
  return true;
}

__device__ __forceinline__ void tile_coords(int tile, int m_tiles, int n_tiles, int& mb,
                                            int& nb) {
  const int per_group = kGroupM * n_tiles;
  const int group = tile / per_group;
  const int first_m = group * kGroupM;
  const int gsize = min(m_tiles - first_m, kGroupM);
  const int in_group = tile - group * per_group;
  mb = first_m + in_group % gsize;
  nb = in_group / gsize;
}

// Time-bounded wait that ignores the abort flag (used to drain in-flight copies).
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_timer_ns() - t0 > kWaitLimitNs) return;
  }
}

__device__ __forceinline__ float gelu_tanh(float x) {
  // 0.5 x (1 + tanh(u)) == x / (1 + exp(-2u)),  u = sqrt(2/pi) (x + 0.044715 x^3)
  const float u = 0.7978845608028654f * fmaf(0.044715f * x, x * x, x);
  return __fdividef(x, 1.0f + __expf(-2.0f * u));
}

__device__ __forceinline__ void load_bf16x32(const bf16* src, float (&v)[32]) {
  const uint4* s = reinterpret_cast<const uint4*>(src);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint4 u = __ldg(s + i);
    float2 a = unpack_bf16x2(u.x), b = unpack_bf16x2(u.y), c = unpack_bf16x2(u.z),
           d = unpack_bf16x2(u.w);
    v[8 * i + 0] = a.x; v[8 * i + 1] = a.y; v[8 * i + 2] = b.x; v[8 * i + 3] = b.y;
    v[8 * i + 4] = c.x; v[8 * i + 5] = c.y; v[8 * i + 6] = d.x; v[8 * i + 7] = d.y;
  }
}

__device__ __forceinline__ void store_bf16x32(bf16* dst, const float (&v)[32]) {
  uint4* d = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint4 u;
    u.x = pack_bf16x2(v[8 * i + 0], v[8 * i + 1]);
    u.y = pack_bf16x2(v[8 * i + 2], v[8 * i + 3]);
    u.z = pack_bf16x2(v[8 * i + 4], v[8 * i + 5]);
    u.w = pack_bf16x2(v[8 * i + 6], v[8 * i + 7]);
    d[i] = u;
  }
}

__device__ __forceinline__ void load_f32x32(const float* src, float (&v)[32]) {
  const float4* s = reinterpret_cast<const float4*>(src);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    float4 f = __ldg(s + i);
    v[4 * i + 0] = f.x; v[4 * i + 1] = f.y; v[4 * i + 2] = f.z; v[4 * i + 3] = f.w;
  }
}

// Per-row scalars of an epilogue row: for the LN-folded kinds the mean and
// 1 / sqrt(var + eps); for the int8 kinds the activation row scale rs.
struct LnRow {
  float mu, rstd;
  float rs = 0.f;
};

// Merge a row's group statistics (mean, M2 of each 256-column group, in group order) into
// the row's mean and reciprocal standard deviation (biased variance over all columns).
__device__ __forceinline__ LnRow ln_row(const GemmEpilogue& e, int row) {
  const float2* s = e.stats_in + size_t(row) * e.stats_parts;
  float mu = 0.f;
  for (int g = 0; g < e.stats_parts; ++g) mu += __ldg(s + g).x;
  mu /= static_cast<float>(e.stats_parts);
  float m2 = 0.f;
  for (int g = 0; g < e.stats_parts; ++g) {
    const float2 v = __ldg(s + g);
    const float t = v.x - mu;
    m2 += fmaf(256.0f * t, t, v.y);
  }
  const float var = fmaxf(m2 / (256.0f * static_cast<float>(e.stats_parts)), 0.0f);
  return LnRow{mu, rsqrtf(var + e.ln_eps)};
}

// Shifted sums of one output row over a 256-column tile, about the row's first stored
// value k: s1 = sum (x - k), s2 = sum (x - k)^2 of the bf16 values written.
struct StatAcc {
  float k, s1, s2;
};

// Add 32 output values of this lane's row (the fp32 values the bf16 output rounds: the
// statistics then describe the residual before its storage rounding, as the LayerNorm of
// the unrounded sum would); `first` marks the tile's first chunk, whose first value
// becomes the shift.  Two independent partial sums keep the dependency chains short.
__device__ __forceinline__ void stat_add(StatAcc& a, const float (&v)[32], bool first) {
  if (first) {
    a.k = v[0];
    a.s1 = 0.f;
    a.s2 = 0.f;
  }
  float s1a = 0.f, s1b = 0.f, s2a = 0.f, s2b = 0.f;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const float x0 = v[2 * i] - a.k, x1 = v[2 * i + 1] - a.k;
    s1a += x0;
    s1b += x1;
    s2a = fmaf(x0, x0, s2a);
    s2b = fmaf(x1, x1, s2b);
  }
  a.s1 += s1a + s1b;
  a.s2 += s2a + s2b;
}

// The tile row's group statistics (mean, M2) over its 256 columns.
__device__ __forceinline__ float2 stat_final(const StatAcc& a) {
  return make_float2(a.k + a.s1 * (1.0f / 256.0f), a.s2 - a.s1 * a.s1 * (1.0f / 256.0f));
}

// Row operands of one 32-column chunk that come from global memory, loaded one chunk
// ahead of their use so that their latency overlaps the previous chunk's work.
struct RowIn {
  uint4 res[4];  // residual, 32 bf16 (gated-residual epilogues)
  float4 cs[8];  // RoPE (cos, sin) of 16 pairs (RoPE epilogue)
};

template <int EPI>
__device__ __forceinline__ void load_row_in(const GemmEpilogue& e, int row, int col, RowIn& in) {
  if constexpr (epi_gated(EPI)) {
    const uint4* s = reinterpret_cast<const uint4*>(e.out + size_t(row) * e.ld_out + col);
#pragma unroll
    for (int i = 0; i < 4; ++i) in.res[i] = s[i];  // coherent: this kernel rewrites it
  }
  if constexpr (epi_base(EPI) == kEpiRope) {
    if (col < e.rope_cols) {
      const int half = e.head_dim >> 1;
      const float4* cs = reinterpret_cast<const float4*>(
          e.rope_cs + (size_t(row) * half + ((col % e.head_dim) >> 1)) * 2);
#pragma unroll
      for (int i = 0; i < 8; ++i) in.cs[i] = __ldg(cs + i);
    }
  }
}

// The per-row scalars an epilogue row needs (LN-folded kinds: the merged statistics; int8
// kinds: the activation row scale), read before the accumulator is ready so that their
// latency overlaps the tile's MMAs.
template <int EPI>
__device__ __forceinline__ LnRow row_scalars(const GemmEpilogue& e, int row, bool valid) {
  LnRow ln{0.f, 1.f};
  if constexpr (epi_ln_fold(EPI)) {
    if (valid) ln = ln_row(e, row);
  }
  if constexpr (epi_int8(EPI)) ln.rs = valid ? __ldg(e.row_scale + row) : 0.f;
  return ln;
}

// a[i] for i in 0..3 without indexing a register array by a runtime value.
__device__ __forceinline__ float pick4(const float (&a)[4], int i) {
  float v = a[0];
#pragma unroll
  for (int k = 1; k < 4; ++k) v = (i == k) ? a[k] : v;
  return v;
}

// Q/K RMSNorm first pass of the single-CTA kernel (vectors read from global memory): the
// reciprocal RMS of each head of this lane's row over a BN-column tile at col0.
template <int BN, int EPI>
__device__ __forceinline__ void qk_rms_pass_global(const GemmEpilogue& e, uint32_t tbase,
                                                   int col0, const LnRow& ln,
                                                   float (&qks)[4]) {
  float ss[4] = {0.f, 0.f, 0.f, 0.f};
  const int cpd = e.head_dim >> 5;
#pragma unroll 1
  for (int c = 0; c < BN / 32; ++c) {
    uint32_t r[32];
    tmem_ld32(tbase + c * 32, r);
    tmem_wait_ld(r);
    float v[32];
    const int col = col0 + c * 32;
    if constexpr (epi_int8(EPI)) {
      float cs[32], b[32];
      load_f32x32(e.col_scale + col, cs);
      if (e.bias_f32) {
        load_f32x32(e.bias_f32 + col, b);
      } else if (e.bias) {
        load_bf16x32(e.bias + col, b);
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) b[j] = 0.0f;
      }
#pragma unroll
      for (int j = 0; j < 32; ++j)
        v[j] = __fmul_rn(__fmul_rn(static_cast<float>(static_cast<int32_t>(r[j])), ln.rs), cs[j]) +
               b[j];
    } else if constexpr (epi_ln_fold(EPI)) {
      float cv[32], dv[32];
      load_f32x32(e.fold_c + col, cv);
      load_f32x32(e.bias_f32 + col, dv);
#pragma unroll
      for (int j = 0; j < 32; ++j)
        v[j] = fmaf(ln.rstd, fmaf(-ln.mu, cv[j], __uint_as_float(r[j])), dv[j]);
    } else {
      float b[32];
      load_bf16x32(e.bias + col, b);
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]) + b[j];
    }
    float s = 0.f;
#pragma unroll
    for (int j = 0; j < 32; ++j) s = fmaf(v[j], v[j], s);
    const int h = c / cpd;
#pragma unroll
    for (int k = 0; k < 4; ++k) ss[k] += (h == k) ? s : 0.f;
  }
  const float inv_hd = 1.0f / static_cast<float>(e.head_dim);
#pragma unroll
  for (int k = 0; k < 4; ++k) qks[k] = rsqrtf(fmaf(ss[k], inv_hd, e.ln_eps));
}

// Epilogue of one 32-column chunk of one row.  ln: the row's statistics (LN-folded
// kinds); sa: the row's running statistics of the stored output, or null; qk_s: the Q/K
// RMSNorm scale of the chunk's head (RoPE kinds with gains).
template <int EPI>
__device__ __forceinline__ void epilogue_chunk(const GemmEpilogue& e, int row, int col,
                                               const uint32_t (&r)[32], const RowIn& in,
                                               const LnRow& ln, StatAcc* sa, bool first,
                                               float qk_s = 1.0f) {
  float v[32];
  if constexpr (epi_int8(EPI)) {
    const float rs = __ldg(e.row_scale + row);
    float cs[32];
    load_f32x32(e.col_scale + col, cs);
    if (e.acc_out) {
      int4* dst = reinterpret_cast<int4*>(e.acc_out + size_t(row) * e.ld_out + col);
#pragma unroll
      for (int i = 0; i < 8; ++i)
        dst[i] = make_int4(int(r[4 * i]), int(r[4 * i + 1]), int(r[4 * i + 2]),
                           int(r[4 * i + 3]));
    }
#pragma unroll
    for (int j = 0; j < 32; ++j)
      v[j] = __fmul_rn(__fmul_rn(static_cast<float>(static_cast<int32_t>(r[j])), rs), cs[j]);
    if (e.bias_f32 || e.bias) {
      float b[32];
      if (e.bias_f32)
        load_f32x32(e.bias_f32 + col, b);
      else
        load_bf16x32(e.bias + col, b);
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] += b[j];
    }
  } else if constexpr (epi_ln_fold(EPI)) {
    float c[32], dv[32];
    load_f32x32(e.fold_c + col, c);
    load_f32x32(e.bias_f32 + col, dv);
#pragma unroll
    for (int j = 0; j < 32; ++j)
      v[j] = fmaf(ln.rstd, fmaf(-ln.mu, c[j], __uint_as_float(r[j])), dv[j]);
  } else {
    float b[32];
    load_bf16x32(e.bias + col, b);
#pragma unroll
    for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]) + b[j];
  }

  if constexpr (EPI == kEpiHeadEuler) {
    float4* st = reinterpret_cast<float4*>(e.out_f32 + size_t(row) * e.ld_out + col);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      float4 x = st[i];
      x.x = fmaf(e.euler_dt, v[4 * i + 0], x.x);
      x.y = fmaf(e.euler_dt, v[4 * i + 1], x.y);
      x.z = fmaf(e.euler_dt, v[4 * i + 2], x.z);
      x.w = fmaf(e.euler_dt, v[4 * i + 3], x.w);
      st[i] = x;
    }
    return;
  }
  if constexpr (epi_base(EPI) == kEpiGelu) {
#pragma unroll
    for (int j = 0; j < 32; ++j) v[j] = gelu_tanh(v[j]);
  }
  if constexpr (epi_base(EPI) == kEpiRope) {
    if (col < e.rope_cols) {
      if (e.q_gain != nullptr) {
        float gn[32];
        load_f32x32((col < (e.rope_cols >> 1) ? e.q_gain : e.k_gain) + col % e.head_dim, gn);
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] *= qk_s * gn[j];
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) {  // 2 pairs per float4 (cos0, sin0, cos1, sin1)
        const float4 c = in.cs[i];
        const float x0 = v[4 * i], x1 = v[4 * i + 1], y0 = v[4 * i + 2], y1 = v[4 * i + 3];
        v[4 * i + 0] = x0 * c.x - x1 * c.y;
        v[4 * i + 1] = x0 * c.y + x1 * c.x;
        v[4 * i + 2] = y0 * c.z - y1 * c.w;
        v[4 * i + 3] = y0 * c.w + y1 * c.z;
      }
    }
  }
  bf16* dst = e.out + size_t(row) * e.ld_out + col;
  if constexpr (epi_gated(EPI)) {
    float g[32];
    load_f32x32(e.gate + col, g);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t w[4] = {in.res[i].x, in.res[i].y, in.res[i].z, in.res[i].w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float2 rr = unpack_bf16x2(w[k]);
        v[8 * i + 2 * k] = fmaf(g[8 * i + 2 * k], v[8 * i + 2 * k], rr.x);
        v[8 * i + 2 * k + 1] = fmaf(g[8 * i + 2 * k + 1], v[8 * i + 2 * k + 1], rr.y);
      }
    }
  }
  uint32_t pk[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) pk[i] = pack_bf16x2(v[2 * i], v[2 * i + 1]);
  if constexpr (EPI == kEpiGateResid || EPI == kEpiBias) {
    if (sa != nullptr) stat_add(*sa, v, first);
  }
  uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int i = 0; i < 4; ++i) d4[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
}

// Stream-K slot of a unit: BN / 4 column groups of 128 rows, so that the 32 rows of a warp
// read or write 512 contiguous bytes per column group.
template <int BN>
__device__ __forceinline__ uint4* sk_slot(const GemmParams& p, int slot_id) {
  return reinterpret_cast<uint4*>(p.sk_slots) + size_t(slot_id) * (BN / 4) * kBM;
}

// Park a 128 x BN partial accumulator (this thread's row from TMEM) in a slot: the
// 32-column chunks [c_first, c_first + nchunks) of the tile; tbase addresses chunk c_first.
template <int BN>
__device__ __forceinline__ void sk_park(const GemmParams& p, int slot_id, uint32_t tbase,
                                        int row_in_tile, int c_first = 0,
                                        int nchunks = BN / 32) {
  uint4* slot = sk_slot<BN>(p, slot_id) + row_in_tile;
#pragma unroll 1
  for (int c = 0; c < nchunks; ++c) {
    uint32_t r[32];
    tmem_ld32(tbase + c * 32, r);
    tmem_wait_ld(r);
#pragma unroll
    for (int i = 0; i < 8; ++i)
      __stcg(slot + size_t((c_first + c) * 8 + i) * kBM,
             make_uint4(r[4 * i], r[4 * i + 1], r[4 * i + 2], r[4 * i + 3]));
  }
}

template <bool INT8>
__device__ __forceinline__ void add_part(uint32_t (&r)[32], const uint4 (&part)[8]) {
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint32_t u[4] = {part[i].x, part[i].y, part[i].z, part[i].w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      if constexpr (INT8)
        r[4 * i + k] = uint32_t(int32_t(r[4 * i + k]) + int32_t(u[k]));
      else
        r[4 * i + k] = __float_as_uint(__uint_as_float(r[4 * i + k]) + __uint_as_float(u[k]));
    }
  }
}

// Epilogue of one output tile row (BN columns): accumulator from TMEM, plus the partial
// tiles parked by units [src_lo, src_hi) (slot src * stride + off), then the fused
// epilogue.  The next column chunk's row inputs and first partial are fetched while the
// current chunk is finished.
template <int BN, bool INT8, int EPI>
__device__ __forceinline__ void epilogue_unit(const GemmParams& p, uint32_t tbase, int row,
                                              int row_in_tile, int col0, int src_lo,
                                              int src_hi, int stride, int off, LnRow ln_in) {
  constexpr int NC = BN / 32;
  const bool valid = row < p.M;
  const bool has_part = src_lo < src_hi;
  const uint4* first = has_part ? sk_slot<BN>(p, src_lo * stride + off) + row_in_tile : nullptr;
  LnRow ln = ln_in;
  StatAcc sa{0.f, 0.f, 0.f};
  const bool want_stats =
      (EPI == kEpiGateResid || EPI == kEpiBias) && BN == 256 && p.epi.stats_out != nullptr;
  float qks[4] = {1.f, 1.f, 1.f, 1.f};
  if constexpr (epi_base(EPI) == kEpiRope) {
    if (p.epi.q_gain != nullptr && col0 < p.epi.rope_cols)
      qk_rms_pass_global<BN, EPI>(p.epi, tbase, col0, ln, qks);
  }
  RowIn in[2];
  uint4 part[2][8];
  if (valid) load_row_in<EPI>(p.epi, row, col0, in[0]);
  if (has_part) {
#pragma unroll
    for (int i = 0; i < 8; ++i) part[0][i] = __ldcg(first + size_t(i) * kBM);
  }
#pragma unroll 2
  for (int c = 0; c < NC; ++c) {
    uint32_t r[32];
    tmem_ld32(tbase + c * 32, r);
    if (c + 1 < NC) {
      if (valid) load_row_in<EPI>(p.epi, row, col0 + (c + 1) * 32, in[(c + 1) & 1]);
      if (has_part) {
#pragma unroll
        for (int i = 0; i < 8; ++i)
          part[(c + 1) & 1][i] = __ldcg(first + size_t((c + 1) * 8 + i) * kBM);
      }
    }
    tmem_wait_ld(r);
    if (has_part) {
      add_part<INT8>(r, part[c & 1]);
      for (int src = src_lo + 1; src < src_hi; ++src) {
        const uint4* ps = sk_slot<BN>(p, src * stride + off) + row_in_tile;
        uint4 more[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) more[i] = __ldcg(ps + size_t(c * 8 + i) * kBM);
        add_part<INT8>(r, more);
      }
    }
    if (valid)
      epilogue_chunk<EPI>(p.epi, row, col0 + c * 32, r, in[c & 1], ln,
                          want_stats ? &sa : nullptr, c == 0,
                          pick4(qks, (c * 32) / p.epi.head_dim));
  }
  if (want_stats && valid)
    p.epi.stats_out[size_t(row) * (p.epi.ld_out / 256) + col0 / 256] = stat_final(sa);
}

// ---------------------------------------------------------------- staged pair epilogue
// Each epilogue warp of the pair kernels owns kWarpStage bytes of shared memory: a 4 KB
// block through which a 32 x 32 chunk passes between the row-per-lane form of the TMEM
// accumulator and the coalesced form of global memory, and the tile's column vectors as
// fp32, which all lanes read at the same address.  With one row per lane a warp-wide
// 16-byte access touches 32 cache lines; through the block it touches 8 (bf16 rows of 64
// bytes) or 4 (fp32 rows of 128 bytes), and the vectors cost one global round trip per
// tile, issued while the warp waits for the accumulator, instead of one per chunk.
constexpr int kVecLen = 256;                               // widest tile
constexpr uint32_t kWarpStage = 4096 + 3 * kVecLen * 4;   // block + 3 vectors
constexpr int kVecBias = 0, kVecGate = kVecLen, kVecScale = 2 * kVecLen;

// 16-byte piece j of row r of a 32 x 32 block: bf16 rows hold 4 pieces, fp32 rows 8.  The
// XOR keeps both access forms (one row per lane; 8 or 4 whole rows per instruction) free of
// bank conflicts within each quarter warp.
__device__ __forceinline__ int blk16(int r, int j) { return r * 4 + (j ^ ((r >> 1) & 3)); }
__device__ __forceinline__ int blk32(int r, int j) { return r * 8 + (j ^ (r & 7)); }

// The NV column vectors starting at col0 into vec (fp32): bias (int8: the fp32 bias, zero
// when absent), gate, int8 column scales.
template <int EPI, int NV>
__device__ __forceinline__ void stage_vectors(const GemmEpilogue& e, int col0, float* vec,
                                              int lane) {
#pragma unroll
  for (int k = 0; k < NV / 32; ++k) {
    const int i = k * 32 + lane;
    const int col = col0 + i;
    if constexpr (epi_int8(EPI) || EPI == kEpiI8GroupGate) {
      float bv = 0.0f;
      if (e.bias_f32)
        bv = __ldg(e.bias_f32 + col);
      else if (e.bias)
        bv = __uint_as_float(static_cast<uint32_t>(
                 __ldg(reinterpret_cast<const unsigned short*>(e.bias) + col)) << 16);
      vec[kVecBias + i] = bv;
      vec[kVecScale + i] = __ldg(e.col_scale + col);
    } else if constexpr (epi_ln_fold(EPI)) {
      vec[kVecBias + i] = __ldg(e.bias_f32 + col);   // dv
      vec[kVecScale + i] = __ldg(e.fold_c + col);    // c
    } else {
      const uint32_t b = __ldg(reinterpret_cast<const unsigned short*>(e.bias) + col);
      vec[kVecBias + i] = __uint_as_float(b << 16);
    }
    if constexpr (epi_gated(EPI))
      vec[kVecGate + i] = __ldg(e.gate + col);
    if constexpr (epi_base(EPI) == kEpiRope) {
      // Q/K RMSNorm gains of the column's head dimension (1 outside q and k, or when off)
      float gn = 1.0f;
      if (e.q_gain != nullptr && col < e.rope_cols)
        gn = __ldg((col < (e.rope_cols >> 1) ? e.q_gain : e.k_gain) + col % e.head_dim);
      vec[kVecGate + i] = gn;
    }
  }
}

// Global inputs of the 32 x 32 chunk (rows row0 + [0, nrows), columns col + [0, 32)) in
// coalesced form: residual pieces (row k * 8 + lane / 4, piece lane % 4) and RoPE (cos, sin)
// pieces (row k * 4 + lane / 8, piece lane % 8).
template <int EPI>
__device__ __forceinline__ void load_block_in(const GemmEpilogue& e, int row0, int nrows,
                                              int col, int lane, RowIn& in) {
  if constexpr (epi_gated(EPI)) {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int r = k * 8 + (lane >> 2);
      in.res[k] = r < nrows ? *reinterpret_cast<const uint4*>(
                                  e.out + size_t(row0 + r) * e.ld_out + col + (lane & 3) * 8)
                            : make_uint4(0u, 0u, 0u, 0u);  // coherent: this kernel rewrites it
    }
  }
  if constexpr (epi_base(EPI) == kEpiRope) {
    if (col < e.rope_cols) {
      const int half = e.head_dim >> 1;
      const int pair0 = (col % e.head_dim) >> 1;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int r = k * 4 + (lane >> 3);
        in.cs[k] = r < nrows ? __ldg(reinterpret_cast<const float4*>(
                                         e.rope_cs + (size_t(row0 + r) * half + pair0) * 2) +
                                     (lane & 7))
                             : make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
  }
}

// Values before the activation / rotation of a bf16 chunk from staged vectors: acc + bias,
// or the LN-folded form rstd (acc - mean c) + dv.
template <int EPI>
__device__ __forceinline__ void pre_values(const uint32_t (&r)[32], const float* vec,
                                           const LnRow& ln, float (&v)[32]) {
  if constexpr (epi_int8(EPI)) {
#pragma unroll
    for (int j = 0; j < 32; ++j)
      v[j] = __fmul_rn(__fmul_rn(static_cast<float>(static_cast<int32_t>(r[j])), ln.rs),
                       vec[kVecScale + j]) +
             vec[kVecBias + j];
  } else if constexpr (epi_ln_fold(EPI)) {
#pragma unroll
    for (int j = 0; j < 32; ++j)
      v[j] = fmaf(ln.rstd, fmaf(-ln.mu, vec[kVecScale + j], __uint_as_float(r[j])),
                  vec[kVecBias + j]);
  } else {
#pragma unroll
    for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]) + vec[kVecBias + j];
  }
}

// Q/K RMSNorm, first pass: the reciprocal RMS of each head of this lane's row in a
// 32-column-chunk tile (heads of head_dim columns; the tile lies inside q, k or v).  The
// scale of chunk c is qks[c * 32 / head_dim]; the chunks are re-read from TMEM.
template <int BN, int EPI>
__device__ __forceinline__ void qk_rms_pass(const GemmEpilogue& e, uint32_t tbase,
                                            const float* vec, const LnRow& ln,
                                            float (&qks)[4]) {
  float ss[4] = {0.f, 0.f, 0.f, 0.f};
  const int cpd = e.head_dim >> 5;  // chunks per head
#pragma unroll 1
  for (int c = 0; c < BN / 32; ++c) {
    uint32_t r[32];
    tmem_ld32(tbase + c * 32, r);
    tmem_wait_ld(r);
    float v[32];
    pre_values<EPI>(r, vec + c * 32, ln, v);
    float s = 0.f;
#pragma unroll
    for (int j = 0; j < 32; ++j) s = fmaf(v[j], v[j], s);
    const int h = c / cpd;
#pragma unroll
    for (int k = 0; k < 4; ++k) ss[k] += (h == k) ? s : 0.f;
  }
  const float inv_hd = 1.0f / static_cast<float>(e.head_dim);
#pragma unroll
  for (int k = 0; k < 4; ++k) qks[k] = rsqrtf(fmaf(ss[k], inv_hd, e.ln_eps));
}

// Epilogue of one 32 x 32 chunk held one row per lane (lane L: row row0 + L, columns col +
// [0, 32)); vec points at the chunk's first column in the staged vectors.  ln: this lane's
// row statistics (LN-folded kinds); sa: its running output statistics, or null; qk_s: the
// Q/K RMSNorm scale of the chunk's head (RoPE kinds with gains).
template <int EPI>
__device__ __forceinline__ void epilogue_block(const GemmEpilogue& e, int row0, int nrows,
                                               int col, const uint32_t (&r)[32],
                                               const RowIn& in, uint4* blk, const float* vec,
                                               int lane, const LnRow& ln, StatAcc* sa,
                                               bool first, float qk_s = 1.0f) {
  const bool valid = lane < nrows;
  float v[32];
  if constexpr (EPI == kEpiI8GroupGate) {
#pragma unroll
    for (int j = 0; j < 32; ++j)
      v[j] = __fmul_rn(__uint_as_float(r[j]), vec[kVecScale + j]) + vec[kVecBias + j];
  } else if constexpr (epi_int8(EPI)) {
    const float rs = valid ? __ldg(e.row_scale + row0 + lane) : 0.0f;
    if (e.acc_out && valid) {
      int4* dst = reinterpret_cast<int4*>(e.acc_out + size_t(row0 + lane) * e.ld_out + col);
#pragma unroll
      for (int i = 0; i < 8; ++i)
        dst[i] = make_int4(int(r[4 * i]), int(r[4 * i + 1]), int(r[4 * i + 2]),
                           int(r[4 * i + 3]));
    }
#pragma unroll
    for (int j = 0; j < 32; ++j)
      v[j] = __fmul_rn(__fmul_rn(static_cast<float>(static_cast<int32_t>(r[j])), rs),
                       vec[kVecScale + j]);
    if (e.bias_f32 || e.bias) {  // staged as fp32 from either form
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] += vec[kVecBias + j];
    }
  } else {
    pre_values<EPI>(r, vec, ln, v);
  }
  if constexpr (EPI == kEpiHeadEuler) {
    // state += dt * v: the chunk's fp32 rows pass through the block, so each warp
    // instruction reads and writes 4 whole rows of 128 bytes
    __syncwarp();
#pragma unroll
    for (int i = 0; i < 8; ++i)
      blk[blk32(lane, i)] = make_uint4(__float_as_uint(v[4 * i]), __float_as_uint(v[4 * i + 1]),
                                       __float_as_uint(v[4 * i + 2]), __float_as_uint(v[4 * i + 3]));
    __syncwarp();
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int rr = k * 4 + (lane >> 3);
      if (rr < nrows) {
        float4* st =
            reinterpret_cast<float4*>(e.out_f32 + size_t(row0 + rr) * e.ld_out + col) + (lane & 7);
        const uint4 u = blk[blk32(rr, lane & 7)];
        float4 x = *st;
        x.x = fmaf(e.euler_dt, __uint_as_float(u.x), x.x);
        x.y = fmaf(e.euler_dt, __uint_as_float(u.y), x.y);
        x.z = fmaf(e.euler_dt, __uint_as_float(u.z), x.z);
        x.w = fmaf(e.euler_dt, __uint_as_float(u.w), x.w);
        *st = x;
      }
    }
    __syncwarp();
    return;
  }
  if constexpr (epi_base(EPI) == kEpiGelu) {
#pragma unroll
    for (int j = 0; j < 32; ++j) v[j] = gelu_tanh(v[j]);
  }
  if constexpr (epi_base(EPI) == kEpiRope) {
    if (col < e.rope_cols) {
      if (e.q_gain != nullptr) {
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] *= qk_s * vec[kVecGate + j];
      }
      __syncwarp();
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const float4 c = in.cs[k];
        blk[blk32(k * 4 + (lane >> 3), lane & 7)] =
            make_uint4(__float_as_uint(c.x), __float_as_uint(c.y), __float_as_uint(c.z),
                       __float_as_uint(c.w));
      }
      __syncwarp();
#pragma unroll
      for (int i = 0; i < 8; ++i) {  // 2 pairs per piece (cos0, sin0, cos1, sin1)
        const uint4 u = blk[blk32(lane, i)];
        const float cx = __uint_as_float(u.x), sx = __uint_as_float(u.y);
        const float cy = __uint_as_float(u.z), sy = __uint_as_float(u.w);
        const float x0 = v[4 * i], x1 = v[4 * i + 1], y0 = v[4 * i + 2], y1 = v[4 * i + 3];
        v[4 * i + 0] = x0 * cx - x1 * sx;
        v[4 * i + 1] = x0 * sx + x1 * cx;
        v[4 * i + 2] = y0 * cy - y1 * sy;
        v[4 * i + 3] = y0 * sy + y1 * cy;
      }
    }
  }
  if constexpr (epi_gated(EPI)) {
    __syncwarp();
#pragma unroll
    for (int k = 0; k < 4; ++k) blk[blk16(k * 8 + (lane >> 2), lane & 3)] = in.res[k];
    __syncwarp();
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint4 u = blk[blk16(lane, i)];
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float2 rr = unpack_bf16x2(w[k]);
        v[8 * i + 2 * k] = fmaf(vec[kVecGate + 8 * i + 2 * k], v[8 * i + 2 * k], rr.x);
        v[8 * i + 2 * k + 1] =
            fmaf(vec[kVecGate + 8 * i + 2 * k + 1], v[8 * i + 2 * k + 1], rr.y);
      }
    }
  }
  uint32_t pk[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) pk[i] = pack_bf16x2(v[2 * i], v[2 * i + 1]);
  if constexpr (EPI == kEpiGateResid || EPI == kEpiBias) {
    if (sa != nullptr) stat_add(*sa, v, first);
  }
  __syncwarp();
#pragma unroll
  for (int i = 0; i < 4; ++i)
    blk[blk16(lane, i)] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
  __syncwarp();
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int rr = k * 8 + (lane >> 2);
    if (rr < nrows)
      *reinterpret_cast<uint4*>(e.out + size_t(row0 + rr) * e.ld_out + col + (lane & 3) * 8) =
          blk[blk16(rr, lane & 3)];
  }
  __syncwarp();  // the block is free for the next chunk
}

// Epilogue of one 128-row half tile of the pair kernel, this warp's 32 rows (row0 + lane):
// accumulator from TMEM, plus the partial tiles parked by units [src_lo, src_hi) (slot
// src * stride + off), then the staged epilogue chunk by chunk.  The next chunk's global
// inputs and first partial are fetched while the current chunk is finished.
template <int BN, bool INT8, int EPI, int NCW>
__device__ __forceinline__ StatAcc epilogue_unit_pair(const GemmParams& p, uint32_t tbase,
                                                      int row0, int row_in_tile, int col0,
                                                      int c_first, int src_lo, int src_hi,
                                                      int stride, int off, uint4* blk,
                                                      const float* vec, int lane, LnRow ln) {
  // NCW 32-column chunks of the tile, [c_first, c_first + NCW): tbase, col0 and vec address
  // the first of them; the partial slots hold the whole tile.  Returns this row's output
  // statistics over those columns (when the epilogue keeps them).
  const int nrows = p.M - row0;
  const bool has_part = src_lo < src_hi;
  const uint4* first =
      has_part ? sk_slot<BN>(p, src_lo * stride + off) + row_in_tile + size_t(c_first) * 8 * kBM
               : nullptr;
  StatAcc sa{0.f, 0.f, 0.f};
  const bool want_stats =
      (EPI == kEpiGateResid || EPI == kEpiBias) && BN == 256 && p.epi.stats_out != nullptr;
  float qks[4] = {1.f, 1.f, 1.f, 1.f};
  if constexpr (epi_base(EPI) == kEpiRope) {
    if (p.epi.q_gain != nullptr && col0 < p.epi.rope_cols)
      qk_rms_pass<NCW * 32, EPI>(p.epi, tbase, vec, ln, qks);
  }
  // Each chunk's global inputs are fetched while its accumulator columns come out of
  // tensor memory (two epilogue warps per SMSP hide the rest of the latency; double
  // buffering them would not fit the registers of a 10-warp CTA).  The loop is unrolled by
  // two only: fully unrolled, a 256-wide tile's epilogue is large enough that its warps
  // stall on instruction fetch.  With RoPE (32 more registers of (cos, sin) per chunk) two
  // chunks in flight overflow the 168 registers, so one.
  constexpr int kUnroll = epi_base(EPI) == kEpiRope ? 1 : 2;
#pragma unroll kUnroll
  for (int c = 0; c < NCW; ++c) {
    uint32_t r[32];
    tmem_ld32(tbase + c * 32, r);
    RowIn in;
    load_block_in<EPI>(p.epi, row0, nrows, col0 + c * 32, lane, in);
    uint4 part[8];
    if (has_part) {
#pragma unroll
      for (int i = 0; i < 8; ++i) part[i] = __ldcg(first + size_t(c * 8 + i) * kBM);
    }
    tmem_wait_ld(r);
    if (has_part) {
      add_part<INT8>(r, part);
      for (int src = src_lo + 1; src < src_hi; ++src) {
        const uint4* ps = sk_slot<BN>(p, src * stride + off) + row_in_tile;
        uint4 more[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) more[i] = __ldcg(ps + size_t((c_first + c) * 8 + i) * kBM);
        add_part<INT8>(r, more);
      }
    }
    epilogue_block<EPI>(p.epi, row0, nrows, col0 + c * 32, r, in, blk, vec + c * 32, lane, ln,
                        want_stats ? &sa : nullptr, c == 0,
                        pick4(qks, (c * 32) / p.epi.head_dim));
  }
  return sa;
}

// Group statistics (mean, M2) of a row's 256 columns from two halves of 128 columns, each
// kept as shifted sums (StatAcc) by its own warp (Chan et al.'s pairwise combination).
__device__ __forceinline__ float2 stat_half(const StatAcc& a) {
  return make_float2(a.k + a.s1 * (1.0f / 128.0f), a.s2 - a.s1 * a.s1 * (1.0f / 128.0f));
}
__device__ __forceinline__ float2 stat_combine(float2 a, float2 b) {
  const float d = b.x - a.x;
  return make_float2(0.5f * (a.x + b.x), a.y + b.y + 64.0f * d * d);
}

// Epilogue of the transposed pair kernel (A = weights, B = activations, so the TMEM lane
// is an output feature and the column a token).  For each 32-token chunk the warp turns
// its 32 features x 32 tokens around in its block (rotated columns: conflict-free both
// ways), after which lane L owns token L's 32 consecutive features and the chunk takes the
// same staged epilogue as the untransposed kernel.
template <int BN, int EPI>
__device__ __forceinline__ void epilogue_unit_trans(const GemmParams& p, uint32_t tbase,
                                                    int lane, int feat0, int tok0, uint4* blk,
                                                    const float* vec) {
  constexpr int NC = BN / 32;
  float* stage = reinterpret_cast<float*>(blk);
#pragma unroll 2
  for (int c = 0; c < NC; ++c) {
    uint32_t r[32];
    tmem_ld32(tbase + c * 32, r);
    const int row0 = tok0 + c * 32;
    RowIn in;
    load_block_in<EPI>(p.epi, row0, p.tokens - row0, feat0, lane, in);
    tmem_wait_ld(r);
#pragma unroll
    for (int t = 0; t < 32; ++t) stage[t * 32 + ((lane + t) & 31)] = __uint_as_float(r[t]);
    __syncwarp();
    uint32_t v[32];
#pragma unroll
    for (int f = 0; f < 32; ++f) v[f] = __float_as_uint(stage[lane * 32 + ((f + lane) & 31)]);
    epilogue_block<EPI>(p.epi, row0, p.tokens - row0, feat0, v, in, blk, vec, lane,
                        LnRow{0.f, 1.f}, nullptr, false);
  }
}

template <int BN, bool INT8, int EPI>
__global__ void __launch_bounds__(192, 1)
    k_gemm_tc(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
              const GemmParams p) {
  using Cfg = GemmCfg<BN>;
  constexpr int STAGES = Cfg::kStages;
  constexpr uint32_t A_BYTES = Cfg::kABytes, B_BYTES = Cfg::kBBytes;
  constexpr uint32_t IDESC = INT8 ? idesc_s8(kBM, BN) : idesc_bf16(kBM, BN, false);
  constexpr int BK_ELEMS = INT8 ? 128 : 64;
  constexpr int K_STEPS = kTileBytesK / 32;  // one MMA consumes 32 bytes of K

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * A_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + STAGES * B_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile uint32_t* abort_flag = tmem_slot + 1;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 4);
    }
    mbar_init(drain, 1);
    *abort_flag = 0u;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_map(&tmA);
    tma_prefetch_map(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, Cfg::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------------------------------------------------------- producer
      int stage = 0;
      uint32_t phase = 0;
      int armed[STAGES];
#pragma unroll
      for (int s = 0; s < STAGES; ++s) armed[s] = -1;
      bool ok = true;
      Sched sc;
      sched_init(p, sc, blockIdx.x, gridDim.x);
      int tile, kb0, kb1;
      while (ok && sched_next(p, sc, tile, kb0, kb1)) {
        int mb, nb;
        tile_coords(tile, p.m_tiles, p.n_tiles, mb, nb);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!wait_bar(&empty[stage], phase ^ 1u, abort_flag, p.err, kErrGemmWait)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[stage], A_BYTES + B_BYTES);
          tma_load_2d(sA + stage * A_BYTES, &tmA, &full[stage], kb * BK_ELEMS, mb * kBM);
          tma_load_2d(sB + stage * B_BYTES, &tmB, &full[stage], kb * BK_ELEMS, nb * BN);
          armed[stage] = static_cast<int>(phase);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {  // let copies already issued land before the CTA exits
        for (int s = 0; s < STAGES; ++s)
          if (armed[s] >= 0) drain_wait(&full[s], static_cast<uint32_t>(armed[s]));
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------------------------------------------------------- MMA issuer
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int local = 0;
      Sched sc;
      sched_init(p, sc, blockIdx.x, gridDim.x);
      int tile, kb0, kb1;
      for (; ok && sched_next(p, sc, tile, kb0, kb1); ++local) {
        const int buf = local & 1;
        const uint32_t use = static_cast<uint32_t>(local >> 1);
        if (!wait_bar(&tempty[buf], (use & 1u) ^ 1u, abort_flag, p.err, kErrGemmWait)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf * BN);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!wait_bar(&full[stage], phase, abort_flag, p.err, kErrGemmWait)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + stage * A_BYTES);
          const uint32_t b0 = smem_u32(sB + stage * B_BYTES);
#pragma unroll
          for (int k = 0; k < K_STEPS; ++k) {
            const uint64_t ad = sdesc_sw128(a0 + k * 32, 16, 1024);
            const uint64_t bd = sdesc_sw128(b0 + k * 32, 16, 1024);
            const uint32_t acc = (kb > kb0 || k > 0) ? 1u : 0u;
            if constexpr (INT8)
              umma_i8(d_tmem, ad, bd, IDESC, acc);
            else
              umma_f16(d_tmem, ad, bd, IDESC, acc);
          }
          tc_commit(&empty[stage]);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (ok) tc_commit(&tfull[buf]);
      }
      tc_commit(drain);
      drain_wait(drain, 0);
    }
  } else {
    // ------------------------------------------------------------------ epilogue
    const int quarter = warp & 3;  // TMEM lanes this warp may access
    const int row_in_tile = quarter * 32 + lane;
    const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
    int local = 0;
    Sched sc;
    sched_init(p, sc, blockIdx.x, gridDim.x);
    int tile, kb0, kb1;
    for (; sched_next(p, sc, tile, kb0, kb1); ++local) {
      int mb, nb;
      tile_coords(tile, p.m_tiles, p.n_tiles, mb, nb);
      const int buf = local & 1;
      const uint32_t use = static_cast<uint32_t>(local >> 1);
      const int row = mb * kBM + row_in_tile;
      const LnRow ln_pre = row_scalars<EPI>(p.epi, row, row < p.M);
      bool ok = wait_bar(&tfull[buf], use & 1u, abort_flag, p.err, kErrGemmWait);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const uint32_t tbase = tmem_base + lane_addr + static_cast<uint32_t>(buf * BN);
      if (kb1 < p.k_blocks) {
        // stream-K contributor: park the partial tile in this CTA's slot
        sk_park<BN>(p, static_cast<int>(blockIdx.x), tbase, row_in_tile);
        __threadfence();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&tempty[buf]);
          st_release_u64(p.sk_flags + blockIdx.x * 4 + quarter, p.sk_seq);
        }
        continue;
      }
      // tile owner: add the partials of the CTAs that computed the rest of this tile
      int c_lo = static_cast<int>(blockIdx.x);
      if (kb0 > 0) {
        c_lo = sk_owner(p, static_cast<long long>(tile - p.sk_tile0) * p.k_blocks, gridDim.x);
        for (int c = c_lo; c < static_cast<int>(blockIdx.x) && ok; ++c) {
          const unsigned long long* f = p.sk_flags + c * 4 + quarter;
          bool seen = ld_acquire_u64(f) == p.sk_seq;
          if (!seen) {
            const uint64_t t0 = global_timer_ns();
            while (!seen) {
              seen = ld_acquire_u64(f) == p.sk_seq;
              if (!seen && (*abort_flag || global_timer_ns() - t0 > kWaitLimitNs)) {
                *abort_flag = 1u;
                atomicCAS(p.err, 0u, kErrGemmWait);
                break;
              }
            }
          }
          ok = __all_sync(0xffffffffu, seen);
        }
      }
      epilogue_unit<BN, INT8, EPI>(p, tbase, row, row_in_tile, nb * BN, c_lo,
                                   static_cast<int>(blockIdx.x), 1, 0, ln_pre);
      // hand the consumed flags back at zero, so a replay of this launch (same sequence
      // value, e.g. from a CUDA graph) waits for its own contributors again
      __syncwarp();
      if (lane == 0)
        for (int src = c_lo; src < static_cast<int>(blockIdx.x); ++src)
          p.sk_flags[src * 4 + quarter] = 0ull;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[buf]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, Cfg::kTmemCols);
  }
}

// ---------------------------------------------------------------------------------------
// CTA-pair variant (tcgen05 cta_group::2): a cluster of two CTAs on two SMs computes a
// 256 x 256 tile.  Each CTA loads its own 128 rows of A and its own 128 rows (half) of B
// per 128-byte K slice, so per SM the operand traffic per MMA is two thirds of the
// single-CTA 128 x 256 tile and the ring holds 6 stages.  The even CTA issues the MMAs
// (M = 256) and signals both CTAs; each CTA's epilogue reads its own 128 accumulator
// lanes.  Work units (tiles or stream-K ranges) are scheduled per pair.
// 256-wide tiles (not transposed) get eight epilogue warps, two per TMEM lane quarter,
// each taking one 128-column half: one warp per SMSP was slow enough that the last tile's
// epilogue and the stream-K merges stood out at the end of the kernel.  Narrower and
// transposed tiles keep four.  Flags are laid out for eight either way.
constexpr int kPairEpiWarps = 8;
template <int BN, bool TRANS>
constexpr int pair_epi_warps() { return BN == 256 && !TRANS ? 8 : 4; }
// Row statistics of the two halves meet in shared memory: [2 accumulators][4 quarters][32].
constexpr uint32_t kPairStatBytes = 2 * 4 * 32 * sizeof(float2);

template <int BN, bool TRANS = false, int EPIW = pair_epi_warps<BN, TRANS>()>
struct PairCfg {
  static constexpr int kEpiWarps = EPIW;
  static constexpr int kThreads = 64 + 32 * EPIW;
  static constexpr uint32_t kABytes = 128 * kTileBytesK;       // this CTA's 128 rows of A
  static constexpr uint32_t kBBytes = (BN / 2) * kTileBytesK;  // this CTA's half of B
  static constexpr uint32_t kTmemCols = 2 * BN <= 256 ? 256 : 512;  // two accumulators
  static constexpr uint32_t kStageOut = EPIW * kWarpStage + kPairStatBytes;
  // as many stages as fit (5 at BN 256: one fewer than with four epilogue warps measured
  // no slower on the block shapes), at most 8
  static constexpr int kFit =
      static_cast<int>((232448 - 1024 - 512 - kStageOut) / (kABytes + kBBytes));
  static constexpr int kStages = kFit < 8 ? kFit : 8;
  static constexpr size_t kSmem =
      1024 + size_t(kStages) * (kABytes + kBBytes) + kStageOut + 512;
  static_assert(kStages >= 4, "pair kernel ring below 4 stages");
  static_assert(kSmem <= 232448, "pair kernel shared memory above the 227 KB limit");
};

template <int BN, bool INT8, int EPI, bool TRANS>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(PairCfg<BN, TRANS>::kThreads, 1)
    k_gemm_pair(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const GemmParams p) {
  using Cfg = PairCfg<BN, TRANS>;
  constexpr int STAGES = Cfg::kStages;
  constexpr uint32_t HA = Cfg::kABytes;
  constexpr uint32_t HB = Cfg::kBBytes;
  constexpr uint32_t IDESC = INT8 ? idesc_s8(256, BN) : idesc_bf16(256, BN, false);
  constexpr int BK_ELEMS = INT8 ? 128 : 64;
  constexpr int K_STEPS = kTileBytesK / 32;
  constexpr uint32_t kTmemCols = Cfg::kTmemCols;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * HA;
  uint8_t* sEpi = sB + STAGES * HB;  // epilogue staging, kWarpStage per epilogue warp
  float2* sStat = reinterpret_cast<float2*>(sEpi + Cfg::kEpiWarps * kWarpStage);
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + STAGES * HB + Cfg::kStageOut);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint64_t* stat_bar = drain + 1;  // [2 accumulators][4 quarters]: the second half's
                                   // statistics of the tile are in sStat
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(stat_bar + 8);
  volatile uint32_t* abort_flag = tmem_slot + 1;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int pair = static_cast<int>(blockIdx.x >> 1);
  const int npairs = static_cast<int>(gridDim.x >> 1);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 2 * Cfg::kEpiWarps);  // every epilogue warp of both CTAs
    }
    mbar_init(drain, 1);
    for (int q = 0; q < 8; ++q) mbar_init(&stat_bar[q], 1);
    *abort_flag = 0u;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_map(&tmA);
    tma_prefetch_map(&tmB);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // the even CTA's barriers, addressed from either CTA
  const uint32_t full0 = mapa_shared(smem_u32(full), 0);
  const uint32_t tempty0 = mapa_shared(smem_u32(tempty), 0);

  if (warp == 0) {
    if (lane == 0) {
      // ---------------------------------------------------------------- producer (both)
      int stage = 0;
      uint32_t phase = 0;
      int armed[STAGES];
#pragma unroll
      for (int s = 0; s < STAGES; ++s) armed[s] = -1;
      bool ok = true;
      Sched sc;
      sched_init(p, sc, pair, npairs);
      int tile, kb0, kb1;
      while (ok && sched_next(p, sc, tile, kb0, kb1)) {
        int mb, nb;
        tile_coords(tile, p.m_tiles, p.n_tiles, mb, nb);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!wait_bar(&empty[stage], phase ^ 1u, abort_flag, p.err, kErrGemmWait)) {
            ok = false;
            break;
          }
          if (rank == 0) mbar_arrive_expect_tx(&full[stage], 2 * (HA + HB));
          const uint32_t fb = full0 + stage * 8;
          tma_load_2d_pair(sA + stage * HA, &tmA, fb, kb * BK_ELEMS, mb * 256 + rank * 128);
          tma_load_2d_pair(sB + stage * HB, &tmB, fb, kb * BK_ELEMS,
                           nb * BN + static_cast<int>(rank) * (BN / 2));
          armed[stage] = static_cast<int>(phase);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok && rank == 0) {  // the even CTA's full barriers count both CTAs' bytes
        for (int s = 0; s < STAGES; ++s)
          if (armed[s] >= 0) drain_wait(&full[s], static_cast<uint32_t>(armed[s]));
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      // ---------------------------------------------------------------- MMA issuer (even CTA)
      // Each stage's four K steps are issued from one asm block: the tensor pipe queues
      // little behind the MMA it executes, so instructions between MMAs can idle it.
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int local = 0;
      const uint64_t a_desc0 = sdesc_sw128(smem_u32(sA), 16, 1024);
      const uint64_t b_desc0 = sdesc_sw128(smem_u32(sB), 16, 1024);
      Sched sc;
      sched_init(p, sc, pair, npairs);
      int tile, kb0, kb1;
      for (; ok && sched_next(p, sc, tile, kb0, kb1); ++local) {
        const int buf = local & 1;
        const uint32_t use = static_cast<uint32_t>(local >> 1);
        if (!wait_bar(&tempty[buf], (use & 1u) ^ 1u, abort_flag, p.err, kErrGemmWait)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf * BN);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!wait_bar(&full[stage], phase, abort_flag, p.err, kErrGemmWait)) {
            ok = false;
            break;
          }
          tc_fence_after();
          static_assert(K_STEPS == 4, "one stage is four K steps of 32 bytes");
          umma_pair_x4<INT8>(d_tmem, a_desc0 + static_cast<uint64_t>(stage) * (HA >> 4),
                             b_desc0 + static_cast<uint64_t>(stage) * (HB >> 4), IDESC,
                             kb > kb0 ? 1u : 0u);
          tc_commit_pair_mc(&empty[stage], 0x3);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (ok) tc_commit_pair_mc(&tfull[buf], 0x3);
      }
      tc_commit_pair(drain);
      drain_wait(drain, 0);
    }
  } else {
    // ------------------------------------------------------------------ epilogue (both)
    // Warp 2 + e: TMEM lane quarter (2 + e) & 3, column half e >> 2 of a 256-wide tile
    // (with a narrower or transposed tile the second four warps only keep the tile count).
    constexpr bool kSplit = Cfg::kEpiWarps == 8;
    constexpr int NCW = kSplit ? BN / 64 : BN / 32;  // 32-column chunks per warp
    const int ew = warp - 2;
    const int half = ew >> 2;
    const bool worker = kSplit || half == 0;
    const int ch0 = kSplit ? half * (BN / 2) : 0;  // the warp's first column in the tile
    const int quarter = warp & 3;
    const int row_in_tile = quarter * 32 + lane;
    const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
    const int slot_id = pair * 2 + static_cast<int>(rank);
    uint4* blk = reinterpret_cast<uint4*>(sEpi + ew * kWarpStage);
    float* vec = reinterpret_cast<float*>(sEpi + ew * kWarpStage + 4096);
    int local = 0;
    int n_stats[2] = {0, 0};  // per accumulator: tiles whose statistics the halves combined
    Sched sc;
    sched_init(p, sc, pair, npairs);
    int tile, kb0, kb1;
    auto release_acc = [&](int buf) {
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (rank == 0)
          mbar_arrive(&tempty[buf]);
        else
          mbar_arrive_cluster(tempty0 + buf * 8);
      }
    };
    for (; sched_next(p, sc, tile, kb0, kb1); ++local) {
      int mb, nb;
      tile_coords(tile, p.m_tiles, p.n_tiles, mb, nb);
      const int buf = local & 1;
      const uint32_t use = static_cast<uint32_t>(local >> 1);
      if (!worker) {
        // paced by the accumulator like the workers, so its arrival counts for this tile
        const bool ok = __all_sync(0xffffffffu,
                                   wait_bar(&tfull[buf], use & 1u, abort_flag, p.err, kErrGemmWait));
        if (!ok) break;
        release_acc(buf);
        continue;
      }
      // the tile's column vectors, fetched while the accumulator is being computed
      if constexpr (TRANS)
        stage_vectors<EPI, 32>(p.epi, mb * 256 + static_cast<int>(rank) * 128 + quarter * 32,
                               vec, lane);
      else
        stage_vectors<EPI, NCW * 32>(p.epi, nb * BN + ch0, vec, lane);
      const int row_pre = mb * 256 + static_cast<int>(rank) * 128 + row_in_tile;
      const LnRow ln_pre = row_scalars<EPI>(p.epi, row_pre, !TRANS && row_pre < p.M);
      bool ok = wait_bar(&tfull[buf], use & 1u, abort_flag, p.err, kErrGemmWait);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const int row = mb * 256 + static_cast<int>(rank) * 128 + row_in_tile;
      const uint32_t tbase = tmem_base + lane_addr + static_cast<uint32_t>(buf * BN + ch0);
      if (kb1 < p.k_blocks) {
        // stream-K contributor: park this warp's part of the partial tile in its slot
        sk_park<BN>(p, slot_id, tbase, row_in_tile, ch0 / 32, NCW);
        __threadfence();
        release_acc(buf);
        if (lane == 0) st_release_u64(p.sk_flags + slot_id * kPairEpiWarps + ew, p.sk_seq);
        continue;
      }
      int c_lo = pair;
      if (kb0 > 0) {
        c_lo = sk_owner(p, static_cast<long long>(tile - p.sk_tile0) * p.k_blocks, npairs);
        for (int c = c_lo; c < pair && ok; ++c) {
          const unsigned long long* f =
              p.sk_flags + (c * 2 + static_cast<int>(rank)) * kPairEpiWarps + ew;
          bool seen = ld_acquire_u64(f) == p.sk_seq;
          if (!seen) {
            const uint64_t t0 = global_timer_ns();
            while (!seen) {
              seen = ld_acquire_u64(f) == p.sk_seq;
              if (!seen && (*abort_flag || global_timer_ns() - t0 > kWaitLimitNs)) {
                *abort_flag = 1u;
                atomicCAS(p.err, 0u, kErrGemmWait);
                break;
              }
            }
          }
          ok = __all_sync(0xffffffffu, seen);
        }
      }
      __syncwarp();  // staged vectors visible to every lane
      StatAcc sa{0.f, 0.f, 0.f};
      if constexpr (TRANS)
        epilogue_unit_trans<BN, EPI>(p, tbase, lane, mb * 256 + static_cast<int>(rank) * 128 +
                                     quarter * 32, nb * BN, blk, vec);
      else
        sa = epilogue_unit_pair<BN, INT8, EPI, NCW>(p, tbase, row - lane, row_in_tile,
                                                    nb * BN + ch0, ch0 / 32, c_lo, pair, 2,
                                                    static_cast<int>(rank), blk, vec, lane,
                                                    ln_pre);
      __syncwarp();
      if (lane == 0)
        for (int src = c_lo; src < pair; ++src)
          p.sk_flags[(src * 2 + static_cast<int>(rank)) * kPairEpiWarps + ew] = 0ull;
      if constexpr (kSplit && (EPI == kEpiGateResid || EPI == kEpiBias)) {
        if (p.epi.stats_out != nullptr) {
          // the row's statistics over the tile's 256 columns: the second half hands its
          // 128 to the first, which combines and stores them
          // (one barrier per accumulator: the second half can be a tile ahead, never two
          // on the same accumulator, which waits for the first half's release)
          float2* xs = sStat + (buf * 4 + quarter) * 32;
          const int ns = buf ? n_stats[1] : n_stats[0];
          if (half == 1) {
            xs[lane] = stat_half(sa);
            __syncwarp();
            if (lane == 0) mbar_arrive(&stat_bar[buf * 4 + quarter]);
          } else {
            ok = __all_sync(0xffffffffu, wait_bar(&stat_bar[buf * 4 + quarter],
                                                  static_cast<uint32_t>(ns) & 1u, abort_flag,
                                                  p.err, kErrGemmWait));
            if (ok && row < p.M)
              p.epi.stats_out[size_t(row) * (p.epi.ld_out / 256) + nb] =
                  stat_combine(stat_half(sa), xs[lane]);
          }
          if (buf)
            ++n_stats[1];
          else
            ++n_stats[0];
        }
      }
      release_acc(buf);
      if (!ok) break;
    }
  }

  // Neither CTA leaves while the other may still signal its barriers or read its tiles.
  tc_fence_before();
  cluster_sync();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, kTmemCols);
  }
}

// ---------------------------------------------------------------------------------------
// Grouped int8 pair GEMM: the A operand carries one scale per row and per group of 1024 K
// columns (the int8 MLP's FC2 input), so the group products cannot share one integer
// accumulator.  Pair tiles of 256 x 128; with the scratch, the tiles past the whole waves
// are split stream-K in groups (lower units park their fp32 sums, the owner adds them).
// TMEM (per CTA, 128 lanes): two int32 group accumulators (columns 0-127, 128-255) and the
// fp32 running sum (256-383).  The MMA issuer fills accumulator g & 1 with group g's
// products and signals gfull; the epilogue warps fold it into the sum, sum += float(acc_g)
// * s_a[row, g], and hand it back (gempty), so the fold of group g overlaps the products
// of group g + 1.  After a tile's last group the same warps run the staged epilogue.
constexpr int kGroupK = 1024;

template <int EPI>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(192, 1)
    k_gemm_pair_grouped(const __grid_constant__ CUtensorMap tmA,
                        const __grid_constant__ CUtensorMap tmB, const GemmParams p) {
  constexpr int BN = 128;
  using Cfg = PairCfg<BN, false, 4>;
  constexpr int STAGES = Cfg::kStages;
  constexpr uint32_t HA = Cfg::kABytes;
  constexpr uint32_t HB = Cfg::kBBytes;
  constexpr uint32_t IDESC = idesc_s8(256, BN);
  constexpr int K_STEPS = kTileBytesK / 32;
  constexpr uint32_t kTmemCols = 512;
  constexpr uint32_t kSumCol = 256;
  constexpr int KB_PER_GROUP = kGroupK / 128;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * HA;
  uint8_t* sEpi = sB + STAGES * HB;
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + STAGES * HB + Cfg::kStageOut);
  uint64_t* empty = full + STAGES;
  uint64_t* gfull = empty + STAGES;
  uint64_t* gempty = gfull + 2;
  uint64_t* drain = gempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile uint32_t* abort_flag = tmem_slot + 1;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int pair = static_cast<int>(blockIdx.x >> 1);
  const int npairs = static_cast<int>(gridDim.x >> 1);
  // the schedule counts K in groups (p.k_blocks = groups of kGroupK columns), so that a
  // stream-K cut always falls between two groups
  const int groups = p.k_blocks;

  if (threadIdx.x == 0) {
    for (int st = 0; st < STAGES; ++st) {
      mbar_init(&full[st], 1);
      mbar_init(&empty[st], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&gfull[b], 1);
      mbar_init(&gempty[b], 8);  // four epilogue warps in each CTA of the pair
    }
    mbar_init(drain, 1);
    *abort_flag = 0u;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_map(&tmA);
    tma_prefetch_map(&tmB);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const uint32_t full0 = mapa_shared(smem_u32(full), 0);
  const uint32_t gempty0 = mapa_shared(smem_u32(gempty), 0);

  if (warp == 0) {
    if (lane == 0) {
      // ---------------------------------------------------------------- producer (both)
      int stage = 0;
      uint32_t phase = 0;
      int armed[STAGES];
#pragma unroll
      for (int st = 0; st < STAGES; ++st) armed[st] = -1;
      bool ok = true;
      Sched sc;
      sched_init(p, sc, pair, npairs);
      int tile, g0, g1;
      while (ok && sched_next(p, sc, tile, g0, g1)) {
        int mb, nb;
        tile_coords(tile, p.m_tiles, p.n_tiles, mb, nb);
        for (int kb = g0 * KB_PER_GROUP; kb < g1 * KB_PER_GROUP; ++kb) {
          if (!wait_bar(&empty[stage], phase ^ 1u, abort_flag, p.err, kErrGemmWait)) {
            ok = false;
            break;
          }
          if (rank == 0) mbar_arrive_expect_tx(&full[stage], 2 * (HA + HB));
          const uint32_t fb = full0 + stage * 8;
          tma_load_2d_pair(sA + stage * HA, &tmA, fb, kb * 128, mb * 256 + rank * 128);
          tma_load_2d_pair(sB + stage * HB, &tmB, fb, kb * 128,
                           nb * BN + static_cast<int>(rank) * (BN / 2));
          armed[stage] = static_cast<int>(phase);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok && rank == 0) {
        for (int st = 0; st < STAGES; ++st)
          if (armed[st] >= 0) drain_wait(&full[st], static_cast<uint32_t>(armed[st]));
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      // ---------------------------------------------------------------- MMA issuer (even CTA)
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int gi = 0;  // groups issued by this pair so far
      const uint64_t a_desc0 = sdesc_sw128(smem_u32(sA), 16, 1024);
      const uint64_t b_desc0 = sdesc_sw128(smem_u32(sB), 16, 1024);
      Sched sc;
      sched_init(p, sc, pair, npairs);
      int tile, g0, g1;
      while (ok && sched_next(p, sc, tile, g0, g1)) {
        for (int g = g0; g < g1 && ok; ++g, ++gi) {
          const int buf = gi & 1;
          const uint32_t use = static_cast<uint32_t>(gi >> 1);
          if (!wait_bar(&gempty[buf], (use & 1u) ^ 1u, abort_flag, p.err, kErrGemmWait)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf * BN);
          // two stages per step: their eight K steps from one asm block (a 256 x 128 int8
          // MMA is short, and what the thread issues between MMAs idles the tensor pipe)
          static_assert(K_STEPS == 4, "one stage is four K steps of 32 bytes");
          static_assert(STAGES % 2 == 0 && KB_PER_GROUP % 2 == 0, "stages taken in pairs");
          for (int kb = 0; kb < KB_PER_GROUP; kb += 2) {
            if (!wait_bar(&full[stage], phase, abort_flag, p.err, kErrGemmWait) ||
                !wait_bar(&full[stage + 1], phase, abort_flag, p.err, kErrGemmWait)) {
              ok = false;
              break;
            }
            tc_fence_after();
            umma_pair_i8_x8<(HA >> 4), (HB >> 4)>(
                d_tmem, a_desc0 + static_cast<uint64_t>(stage) * (HA >> 4),
                b_desc0 + static_cast<uint64_t>(stage) * (HB >> 4), IDESC, kb > 0 ? 1u : 0u);
            tc_commit_pair_mc(&empty[stage], 0x3);
            tc_commit_pair_mc(&empty[stage + 1], 0x3);
            stage += 2;
            if (stage == STAGES) {
              stage = 0;
              phase ^= 1u;
            }
          }
          if (ok) tc_commit_pair_mc(&gfull[buf], 0x3);
        }
      }
      tc_commit_pair(drain);
      drain_wait(drain, 0);
    }
  } else {
    // ------------------------------------------------------------------ fold + epilogue
    const int quarter = warp & 3;
    const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
    uint4* blk = reinterpret_cast<uint4*>(sEpi + quarter * kWarpStage);
    float* vec = reinterpret_cast<float*>(sEpi + quarter * kWarpStage + 4096);
    int gi = 0;
    bool ok = true;
    const int ew = warp - 2;  // epilogue warp 0..3 (its flag in the slot's flag row)
    const int slot_id = pair * 2 + static_cast<int>(rank);
    const int row_in_tile = quarter * 32 + lane;
    Sched sc;
    sched_init(p, sc, pair, npairs);
    int tile, g0, g1;
    while (ok && sched_next(p, sc, tile, g0, g1)) {
      int mb, nb;
      tile_coords(tile, p.m_tiles, p.n_tiles, mb, nb);
      stage_vectors<EPI, BN>(p.epi, nb * BN, vec, lane);
      const int row0 = mb * 256 + static_cast<int>(rank) * 128 + quarter * 32;
      const int row = row0 + lane;
      const uint32_t sum_addr = tmem_base + lane_addr + kSumCol;
      for (int g = g0; g < g1; ++g, ++gi) {
        const int buf = gi & 1;
        const uint32_t use = static_cast<uint32_t>(gi >> 1);
        ok = __all_sync(0xffffffffu,
                        wait_bar(&gfull[buf], use & 1u, abort_flag, p.err, kErrGemmWait));
        if (!ok) break;
        tc_fence_after();
        const float sa = row < p.M ? __ldg(p.epi.row_scale + size_t(row) * groups + g) : 0.f;
        const uint32_t acc_addr = tmem_base + lane_addr + static_cast<uint32_t>(buf * BN);
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
          uint32_t a[32];
          tmem_ld32(acc_addr + c * 32, a);
          tmem_wait_ld(a);
          uint32_t sm[32];
          if (g > g0) {
            tmem_ld32(sum_addr + c * 32, sm);
            tmem_wait_ld(sm);
#pragma unroll
            for (int j = 0; j < 32; ++j)
              sm[j] = __float_as_uint(fmaf(static_cast<float>(static_cast<int32_t>(a[j])), sa,
                                           __uint_as_float(sm[j])));
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              sm[j] = __float_as_uint(__fmul_rn(static_cast<float>(static_cast<int32_t>(a[j])), sa));
          }
          tmem_st32(sum_addr + c * 32, sm);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {  // the group accumulator may be refilled
          if (rank == 0)
            mbar_arrive(&gempty[buf]);
          else
            mbar_arrive_cluster(gempty0 + buf * 8);
        }
      }
      if (!ok) break;
      if (g1 < groups) {
        // stream-K contributor: park this warp's rows of the running sum in its slot (the
        // sum is rewritten only by this warp's next fold, after the stores have read it)
        tc_fence_after();
        sk_park<BN>(p, slot_id, sum_addr, row_in_tile);
        __threadfence();
        __syncwarp();
        if (lane == 0) st_release_u64(p.sk_flags + slot_id * kPairEpiWarps + ew, p.sk_seq);
        tc_fence_before();
        __syncwarp();
        continue;
      }
      int c_lo = pair;
      if (g0 > 0) {
        // the tile's earlier groups were summed by the units below: wait for their parks
        c_lo = sk_owner(p, static_cast<long long>(tile - p.sk_tile0) * p.k_blocks, npairs);
        for (int c = c_lo; c < pair && ok; ++c) {
          const unsigned long long* f =
              p.sk_flags + (c * 2 + static_cast<int>(rank)) * kPairEpiWarps + ew;
          bool seen = ld_acquire_u64(f) == p.sk_seq;
          if (!seen) {
            const uint64_t t0 = global_timer_ns();
            while (!seen) {
              seen = ld_acquire_u64(f) == p.sk_seq;
              if (!seen && (*abort_flag || global_timer_ns() - t0 > kWaitLimitNs)) {
                *abort_flag = 1u;
                atomicCAS(p.err, 0u, kErrGemmWait);
                break;
              }
            }
          }
          ok = __all_sync(0xffffffffu, seen);
        }
        if (!ok) break;
      }
      __syncwarp();  // staged vectors visible to every lane
      const int nrows = p.M - row0;
      RowIn in[2];
      load_block_in<EPI>(p.epi, row0, nrows, nb * BN, lane, in[0]);
#pragma unroll 2
      for (int c = 0; c < BN / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(sum_addr + c * 32, r);
        if (c + 1 < BN / 32) load_block_in<EPI>(p.epi, row0, nrows, nb * BN + (c + 1) * 32, lane, in[(c + 1) & 1]);
        tmem_wait_ld(r);
        for (int src = c_lo; src < pair; ++src) {  // the parked partial sums, fp32
          const uint4* ps = sk_slot<BN>(p, src * 2 + static_cast<int>(rank)) + row_in_tile;
          uint4 part[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) part[i] = __ldcg(ps + size_t(c * 8 + i) * kBM);
          add_part<false>(r, part);
        }
        epilogue_block<EPI>(p.epi, row0, nrows, nb * BN + c * 32, r, in[c & 1], blk, vec + c * 32,
                            lane, LnRow{0.f, 1.f}, nullptr, false);
      }
      if (lane == 0)
        for (int src = c_lo; src < pair; ++src)
          p.sk_flags[(src * 2 + static_cast<int>(rank)) * kPairEpiWarps + ew] = 0ull;
      tc_fence_before();
      __syncwarp();
    }
  }

  tc_fence_before();
  cluster_sync();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, kTmemCols);
  }
}

std::atomic<unsigned long long> g_sk_seq{0};
bool trace_gemm();
int forced_sched();

// A value no flag of the scratch can hold from an earlier launch: a per-process random
// high half and a launch counter.
unsigned long long next_sk_seq() {
  static const unsigned long long salt =
      (static_cast<unsigned long long>(std::random_device{}()) << 32) | 1ull;
  return salt + (g_sk_seq.fetch_add(1) << 1);
}

// First stream-K tile of the pair kernel's hybrid schedule: every whole wave of tiles but
// the last runs data-parallel, so the split part holds between one and two tiles per unit
// (all tiles, when there are fewer than two waves).
int hybrid_tile0(int tiles, int units) { return std::max(0, tiles / units - 1) * units; }

// First stream-K tile of the grouped int8 kernel's schedule: every whole wave runs
// data-parallel and only the tiles past them are split (K counted in 1024-column groups).
int remainder_tile0(int tiles, int units) { return (tiles / units) * units; }

// Schedule costs in units of one K slice of one tile on one scheduling unit.
// Data-parallel: ceil(tiles / units) waves of k_blocks slices.  Stream-K over the tiles
// from dp_tiles on: the whole waves before it, plus the even share of the split tiles
// times 1.28, plus 17 (partial-tile parking and merging, the exposed epilogue of the merged
// tile).  The constants fit the CTA-pair kernel on B200 (CUDA graphs of 20 launches) at
// M = 832, 1600 and 11344 with the four block GEMM shapes of a 3072-wide model; the choice
// they make was the faster schedule for all ten shapes measured.
double dp_cost(int tiles, int units, int k_blocks) {
  return double((tiles + units - 1) / units) * k_blocks;
}
double sk_cost(int tiles, int units, int k_blocks, int dp_tiles) {
  return double(dp_tiles / units) * k_blocks +
         1.28 * double(tiles - dp_tiles) * k_blocks / units + 17.0;
}
bool want_stream_k(int tiles, int units, int k_blocks, int dp_tiles = 0) {
  return sk_cost(tiles, units, k_blocks, dp_tiles) < dp_cost(tiles, units, k_blocks);
}

template <int BN, bool INT8, int EPI>
int launch_impl(const DevCtx& ctx, const void* A, const void* B, int M, int N, int K,
                const GemmEpilogue& epi, void* scratch, size_t scratch_bytes,
                cudaStream_t stream) {
  using Cfg = GemmCfg<BN>;
  const CUtensorMapDataType dt =
      INT8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const int esize = INT8 ? 1 : 2;
  const int bk = kTileBytesK / esize;
  CUtensorMap ta, tb;
  if (!make_tmap_2d(&ta, A, dt, uint64_t(M), uint64_t(K), uint64_t(K) * esize, kBM, bk) ||
      !make_tmap_2d(&tb, B, dt, uint64_t(N), uint64_t(K), uint64_t(K) * esize, BN, bk))
    return set_error(-3, "gemm: cuTensorMapEncodeTiled failed (M=%d N=%d K=%d)", M, N, K);

  auto kernel = k_gemm_tc<BN, INT8, EPI>;
  static std::atomic<uint32_t> attr_done{0};  // one bit per device
  const uint32_t bit = 1u << (ctx.device & 31);
  if (!(attr_done.load() & bit)) {
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(Cfg::kSmem));
    if (e != cudaSuccess)
      return set_error(-3, "gemm: cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    attr_done.fetch_or(bit);
  }

  GemmParams p{};
  p.M = M;
  p.N = N;
  p.k_blocks = K / bk;
  p.m_tiles = (M + kBM - 1) / kBM;
  p.n_tiles = N / BN;
  p.epi = epi;
  p.err = ctx.err_flag;
  const int tiles = p.m_tiles * p.n_tiles;
  const int sk_ctas = std::min(ctx.num_sms, kMaxSkCtas);
  const long long iters = static_cast<long long>(tiles) * p.k_blocks;
  // (the Q/K RMSNorm needs whole heads from one accumulator: no split tiles)
  const bool sk_ok = scratch != nullptr && scratch_bytes >= kScratchBytes &&
                     iters >= 4LL * sk_ctas && epi.q_gain == nullptr;
  const bool use_sk = sk_ok && (forced_sched() >= 0 ? forced_sched() >= 1
                                                    : want_stream_k(tiles, ctx.num_sms, p.k_blocks));
  if (trace_gemm())
    std::fprintf(stderr, "h3b gemm 1cta BN=%d M=%d N=%d K=%d tiles=%d sms=%d -> %s grid=%d\n", BN,
                 M, N, K, tiles, ctx.num_sms, use_sk ? "stream-K" : "data-parallel",
                 use_sk ? sk_ctas : std::min(tiles, ctx.num_sms));
  if (!use_sk) {
    const int grid = std::min(tiles, ctx.num_sms);
    kernel<<<grid, 192, Cfg::kSmem, stream>>>(ta, tb, p);
    return check_launch("gemm");
  }
  p.sk = 1;
  p.sk_iters = iters;
  p.sk_slots = static_cast<uint32_t*>(scratch);
  p.sk_flags =
      reinterpret_cast<unsigned long long*>(static_cast<uint8_t*>(scratch) + kSkFlagsOffset);
  p.sk_seq = next_sk_seq();
  // one CTA per SM, never more CTAs than SMs: every CTA is resident at once
  kernel<<<sk_ctas, 192, Cfg::kSmem, stream>>>(ta, tb, p);
  return check_launch("gemm");
}

// Largest number of CTA pairs of the pair kernel that can be resident at once.
template <int BN, bool INT8, int EPI, bool TRANS = false>
int pair_capacity(const DevCtx& ctx) {
  static std::atomic<int> cap[64];
  const int dev = ctx.device & 63;
  int c = cap[dev].load();
  if (c > 0) return c;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * (ctx.num_sms / 2));
  cfg.blockDim = dim3(PairCfg<BN, TRANS>::kThreads);
  cfg.dynamicSmemBytes = PairCfg<BN, TRANS>::kSmem;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, k_gemm_pair<BN, INT8, EPI, TRANS>, &cfg) !=
          cudaSuccess ||
      n <= 0) {
    cudaGetLastError();
    n = 0;
  }
  c = std::min(n, ctx.num_sms / 2);
  if (c > 0) cap[dev].store(c);
  return c;
}

// Returns 1 if the pair kernel is not usable here (caller falls back to single-CTA tiles).
template <int BN, bool INT8, int EPI>
int launch_pair(const DevCtx& ctx, const void* A, const void* B, int M, int N, int K,
                const GemmEpilogue& epi, void* scratch, size_t scratch_bytes,
                cudaStream_t stream, int* rc) {
  using Cfg = PairCfg<BN>;
  auto kernel = k_gemm_pair<BN, INT8, EPI, false>;
  static std::atomic<uint32_t> attr_done{0};
  const uint32_t bit = 1u << (ctx.device & 31);
  if (!(attr_done.load() & bit)) {
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(Cfg::kSmem)) != cudaSuccess) {
      cudaGetLastError();
      return 1;
    }
    attr_done.fetch_or(bit);
  }
  const int cap = pair_capacity<BN, INT8, EPI>(ctx);
  if (cap <= 0) return 1;
  const CUtensorMapDataType dt =
      INT8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const int esize = INT8 ? 1 : 2;
  const int bk = kTileBytesK / esize;
  CUtensorMap ta, tb;
  if (!make_tmap_2d(&ta, A, dt, uint64_t(M), uint64_t(K), uint64_t(K) * esize, 128, bk) ||
      !make_tmap_2d(&tb, B, dt, uint64_t(N), uint64_t(K), uint64_t(K) * esize, BN / 2, bk)) {
    *rc = set_error(-3, "gemm: cuTensorMapEncodeTiled failed (M=%d N=%d K=%d)", M, N, K);
    return 0;
  }
  GemmParams p{};
  p.M = M;
  p.N = N;
  p.k_blocks = K / bk;
  p.m_tiles = (M + 255) / 256;
  p.n_tiles = N / BN;
  p.epi = epi;
  p.err = ctx.err_flag;
  const int tiles = p.m_tiles * p.n_tiles;
  const int sk_pairs = std::min(cap, kMaxSkCtas / 2);
  // hybrid: all whole waves but the last run data-parallel, the rest is split stream-K
  const int sk_tile0 = forced_sched() == 2 ? 0 : hybrid_tile0(tiles, sk_pairs);
  const long long iters = static_cast<long long>(tiles - sk_tile0) * p.k_blocks;
  const bool sk_ok = scratch != nullptr && scratch_bytes >= kScratchBytes &&
                     iters >= 4LL * sk_pairs && epi.q_gain == nullptr;
  const bool use_sk =
      sk_ok && (forced_sched() >= 0 ? forced_sched() >= 1
                                    : want_stream_k(tiles, sk_pairs, p.k_blocks, sk_tile0));
  if (trace_gemm())
    std::fprintf(stderr,
                 "h3b gemm pair BN=%d M=%d N=%d K=%d tiles=%d cap=%d -> %s pairs=%d sk_tile0=%d\n",
                 BN, M, N, K, tiles, cap, use_sk ? "stream-K" : "data-parallel",
                 use_sk ? sk_pairs : std::min(tiles, cap), use_sk ? sk_tile0 : 0);
  if (use_sk) {
    GemmParams q = p;
    q.sk = 1;
    q.sk_tile0 = sk_tile0;
    q.sk_iters = iters;
    q.sk_slots = static_cast<uint32_t*>(scratch);
    q.sk_flags =
        reinterpret_cast<unsigned long long*>(static_cast<uint8_t*>(scratch) + kSkFlagsOffset);
    q.sk_seq = next_sk_seq();
    // never more pairs than can be resident at once (occupancy query above)
    kernel<<<2 * sk_pairs, Cfg::kThreads, Cfg::kSmem, stream>>>(ta, tb, q);
    *rc = check_launch("gemm_pair");
    return 0;
  }
  kernel<<<2 * std::min(tiles, cap), Cfg::kThreads, Cfg::kSmem, stream>>>(ta, tb, p);
  *rc = check_launch("gemm_pair");
  return 0;
}

// Transposed CTA-pair GEMM, out[M, N] = X[M, K] W[N, K]^T computed as W X^T: the weight
// rows fill the 256-row MMA side and the M activation rows (tokens) the 160-wide N side,
// so a token count that is not a multiple of 256 wastes little (1,600 = 10 x 160).
// Data-parallel only.  Returns 1 if the kernel cannot run here.
template <int EPI>
int launch_pair_trans(const DevCtx& ctx, const bf16* X, const bf16* W, int M, int N, int K,
                      const GemmEpilogue& epi, cudaStream_t stream, int* rc) {
  constexpr int BN = kTransBN;
  using Cfg = PairCfg<BN, true>;
  auto kernel = k_gemm_pair<BN, false, EPI, true>;
  static std::atomic<uint32_t> attr_done{0};
  const uint32_t bit = 1u << (ctx.device & 31);
  if (!(attr_done.load() & bit)) {
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(Cfg::kSmem)) != cudaSuccess) {
      cudaGetLastError();
      return 1;
    }
    attr_done.fetch_or(bit);
  }
  const int cap = pair_capacity<BN, false, EPI, true>(ctx);
  if (cap <= 0) return 1;
  CUtensorMap ta, tb;
  if (!make_tmap_2d(&ta, W, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, uint64_t(N), uint64_t(K),
                    uint64_t(K) * 2, 128, 64) ||
      !make_tmap_2d(&tb, X, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, uint64_t(M), uint64_t(K),
                    uint64_t(K) * 2, BN / 2, 64)) {
    *rc = set_error(-3, "gemm: cuTensorMapEncodeTiled failed (M=%d N=%d K=%d)", M, N, K);
    return 0;
  }
  GemmParams p{};
  p.M = N;
  p.N = M;
  p.tokens = M;
  p.k_blocks = K / 64;
  p.m_tiles = N / 256;
  p.n_tiles = (M + BN - 1) / BN;
  p.epi = epi;
  p.err = ctx.err_flag;
  const int tiles = p.m_tiles * p.n_tiles;
  if (trace_gemm())
    std::fprintf(stderr, "h3b gemm pair transposed BN=%d M=%d N=%d K=%d tiles=%d cap=%d\n", BN,
                 M, N, K, tiles, cap);
  kernel<<<2 * std::min(tiles, cap), Cfg::kThreads, Cfg::kSmem, stream>>>(ta, tb, p);
  *rc = check_launch("gemm_pair_trans");
  return 0;
}

// Process-wide overrides of the GEMM dispatch (h3b_set_gemm_override; diagnostics and
// measurements only, -1 = automatic).  Set through the C ABI, never from the environment.
std::atomic<int> g_force_tile{-1}, g_force_sched{-1}, g_force_trans{-1};

// Forced schedule: 2 stream-K over every tile, 1 hybrid stream-K (the pair kernel's
// default form), 0 data-parallel, -1 the cost model's choice; where the scratch allows it.
int forced_sched() { return g_force_sched.load(std::memory_order_relaxed); }

// H3B_TRACE_GEMM=1 prints each GEMM's schedule to stderr (diagnostics only).
bool trace_gemm() {
  static const bool on = [] {
    const char* v = std::getenv("H3B_TRACE_GEMM");
    return v && v[0] == '1';
  }();
  return on;
}

// Tile configurations of the bf16 / int8 GEMM.
enum TileCfg { kPair256 = 0, kPair128 = 1, kSingle256 = 2, kSingle128 = 3, kAuto = -1 };

// Forced tile configuration (a TileCfg value), where the shape allows it.
int forced_tile() { return g_force_tile.load(std::memory_order_relaxed); }

bool tile_allowed(int cfg, int M, int N) {
  switch (cfg) {
    case kPair256: return N % 256 == 0 && M >= 256;
    case kPair128: return N % 128 == 0 && M >= 256;
    case kSingle256: return N % 256 == 0;
    case kSingle128: return N % 128 == 0;
    default: return false;
  }
}

// Shape-based choice: CTA-pair 256-wide tiles unless the problem is too small for pairs.
int choose_tile(int M, int N) {
  const int f = forced_tile();
  if (f != kAuto && tile_allowed(f, M, N)) return f;
  if (tile_allowed(kPair256, M, N)) return kPair256;
  if (tile_allowed(kSingle256, M, N)) return kSingle256;
  return kSingle128;
}

template <int BN>
int dispatch_bf16(const DevCtx& ctx, const bf16* A, const bf16* B, int M, int N, int K,
                  const GemmEpilogue& epi, void* ws, size_t wsb, cudaStream_t s) {
  switch (epi.kind) {
    case kEpiBias: return launch_impl<BN, false, kEpiBias>(ctx, A, B, M, N, K, epi, ws, wsb, s);
    case kEpiGelu: return launch_impl<BN, false, kEpiGelu>(ctx, A, B, M, N, K, epi, ws, wsb, s);
    case kEpiRope: return launch_impl<BN, false, kEpiRope>(ctx, A, B, M, N, K, epi, ws, wsb, s);
    case kEpiGateResid:
      return launch_impl<BN, false, kEpiGateResid>(ctx, A, B, M, N, K, epi, ws, wsb, s);
    case kEpiRopeLN:
      return launch_impl<BN, false, kEpiRopeLN>(ctx, A, B, M, N, K, epi, ws, wsb, s);
    case kEpiGeluLN:
      return launch_impl<BN, false, kEpiGeluLN>(ctx, A, B, M, N, K, epi, ws, wsb, s);
    case kEpiHeadEuler:
      return launch_impl<BN, false, kEpiHeadEuler>(ctx, A, B, M, N, K, epi, ws, wsb, s);
    default: return set_error(-1, "gemm: unknown epilogue %d", epi.kind);
  }
}

}  // namespace

size_t gemm_scratch_bytes() { return kScratchBytes; }

int set_gemm_override(int tile, int sched, int trans) {
  if (tile < -1 || tile > kSingle128 || sched < -1 || sched > 2 || trans < -1 || trans > 1)
    return -1;
  g_force_tile.store(tile);
  g_force_sched.store(sched);
  g_force_trans.store(trans);
  return 0;
}

// The work items of one scheduling unit, from the functions the kernels run: (tile, first
// K slice, end K slice, merge) with merge = -1 for a partial tile the unit parks for a
// higher unit, else the first unit whose parked partial the item's epilogue adds (the unit
// itself when it adds none).  -1 for a stream-K schedule the launches never run (fewer
// than 4 split K slices per unit: a unit with an empty range would leave its flag unset).
int gemm_schedule_items(int tiles, int k_blocks, int units, int mode, int unit, int* items,
                        int max_items) {
  GemmParams p{};
  p.k_blocks = k_blocks;
  p.m_tiles = tiles;
  p.n_tiles = 1;
  if (mode != 0) {
    p.sk = 1;
    p.sk_tile0 = mode == 1 ? hybrid_tile0(tiles, units)
                           : mode == 3 ? remainder_tile0(tiles, units) : 0;
    p.sk_iters = static_cast<long long>(tiles - p.sk_tile0) * k_blocks;
    // the pair kernels split only with at least 4 K slices per unit; the grouped kernel
    // with at least one group per unit, and only a partial wave past whole ones
    if (mode == 3 ? (tiles <= units || p.sk_iters < units) : p.sk_iters < 4LL * units)
      return -1;
  }
  Sched sc;
  sched_init(p, sc, unit, units);
  int n = 0, tile, kb0, kb1;
  while (sched_next(p, sc, tile, kb0, kb1)) {
    int merge = unit;
    if (kb1 < k_blocks)
      merge = -1;
    else if (kb0 > 0)
      merge = sk_owner(p, static_cast<long long>(tile - p.sk_tile0) * k_blocks, units);
    if (n < max_items) {
      items[4 * n + 0] = tile;
      items[4 * n + 1] = kb0;
      items[4 * n + 2] = kb1;
      items[4 * n + 3] = merge;
    }
    ++n;
  }
  return n;
}

unsigned long long next_scratch_seq() { return next_sk_seq(); }

template <int EPI>
bool try_pair_bf16(int bn, const DevCtx& ctx, const bf16* A, const bf16* B, int M, int N, int K,
                   const GemmEpilogue& epi, void* ws, size_t wsb, cudaStream_t s, int* rc) {
  if (bn == 256) return launch_pair<256, false, EPI>(ctx, A, B, M, N, K, epi, ws, wsb, s, rc) == 0;
  return launch_pair<128, false, EPI>(ctx, A, B, M, N, K, epi, ws, wsb, s, rc) == 0;
}

// Forced use (1) or exclusion (0) of the transposed pair kernel where the shape allows it.
int forced_trans() { return g_force_trans.load(std::memory_order_relaxed); }

// Transposed (tokens on the 160-wide side) or not, from the same cost reasoning as the
// stream-K choice, in units of one 256 x 256 tile on one CTA pair: the untransposed
// kernel's best schedule against ceil(tiles / pairs) waves of 160 / 256 of a tile, times
// kTransCost for the narrower tile's lower efficiency.  Measured on B200 (CUDA graphs of
// 20 launches): the 160-wide tile does ~1.5x the time per FLOP of the 256-wide one, so the
// transposed kernel is picked only where it wins: the out-projection at 832 tokens (24.9
// vs 25.5 us data-parallel); at 1,600 tokens stream-K does it in 36.9 us against 39.5.
constexpr double kTransCost = 1.5;

bool want_trans(const DevCtx& ctx, int M, int N, int K, bool sk_possible) {
  if (N % 256 != 0 || M < kTransBN || forced_tile() != kAuto) return false;
  if (forced_trans() >= 0) return forced_trans() == 1;
  const int pairs = std::max(1, ctx.num_sms / 2);
  const double kb = K / 64;
  const int tiles_n = ((M + 255) / 256) * (N / 256);
  double best_n = dp_cost(tiles_n, pairs, 1);
  if (sk_possible)
    best_n = std::min(best_n, sk_cost(tiles_n, pairs, K / 64, hybrid_tile0(tiles_n, pairs)) / kb);
  const int tiles_t = (N / 256) * ((M + kTransBN - 1) / kTransBN);
  const double t = double((tiles_t + pairs - 1) / pairs) * kTransBN / 256.0 * kTransCost;
  return t < best_n;
}

int launch_gemm_bf16(const DevCtx& ctx, const bf16* A, const bf16* B, int M, int N, int K,
                     const GemmEpilogue& epi, void* scratch, size_t scratch_bytes,
                     cudaStream_t stream) {
  if (M <= 0) return 0;
  int tile = choose_tile(M, N);
  // Row statistics of the output need a tile that covers a whole 256-column group, and the
  // transposed kernel spreads a token's columns over several warps: 256-wide untransposed
  // tiles for them, and for the LN-folded kinds (row statistics read per row).
  const bool row_stats =
      epi.stats_out != nullptr || epi_ln_fold(epi.kind) || epi.q_gain != nullptr;
  if (epi.stats_out != nullptr) tile = M >= 256 ? kPair256 : kSingle256;
  if (tile == kPair256 && !row_stats &&
      want_trans(ctx, M, N, K, scratch != nullptr && scratch_bytes >= kScratchBytes)) {
    int rc = 0, r = 1;
    switch (epi.kind) {
      case kEpiBias: r = launch_pair_trans<kEpiBias>(ctx, A, B, M, N, K, epi, stream, &rc); break;
      case kEpiGelu: r = launch_pair_trans<kEpiGelu>(ctx, A, B, M, N, K, epi, stream, &rc); break;
      case kEpiRope: r = launch_pair_trans<kEpiRope>(ctx, A, B, M, N, K, epi, stream, &rc); break;
      case kEpiGateResid:
        r = launch_pair_trans<kEpiGateResid>(ctx, A, B, M, N, K, epi, stream, &rc);
        break;
      default: return set_error(-1, "gemm: unknown epilogue %d", epi.kind);
    }
    if (r == 0) return rc;
  }
  if (tile == kPair256 || tile == kPair128) {
    const int bn = tile == kPair256 ? 256 : 128;
    int rc = 0;
    bool done = false;
    switch (epi.kind) {
      case kEpiBias:
        done = try_pair_bf16<kEpiBias>(bn, ctx, A, B, M, N, K, epi, scratch, scratch_bytes,
                                       stream, &rc);
        break;
      case kEpiGelu:
        done = try_pair_bf16<kEpiGelu>(bn, ctx, A, B, M, N, K, epi, scratch, scratch_bytes,
                                       stream, &rc);
        break;
      case kEpiRope:
        done = try_pair_bf16<kEpiRope>(bn, ctx, A, B, M, N, K, epi, scratch, scratch_bytes,
                                       stream, &rc);
        break;
      case kEpiGateResid:
        done = try_pair_bf16<kEpiGateResid>(bn, ctx, A, B, M, N, K, epi, scratch,
                                            scratch_bytes, stream, &rc);
        break;
      case kEpiRopeLN:
        done = try_pair_bf16<kEpiRopeLN>(bn, ctx, A, B, M, N, K, epi, scratch, scratch_bytes,
                                         stream, &rc);
        break;
      case kEpiGeluLN:
        done = try_pair_bf16<kEpiGeluLN>(bn, ctx, A, B, M, N, K, epi, scratch, scratch_bytes,
                                         stream, &rc);
        break;
      case kEpiHeadEuler:
        done = try_pair_bf16<kEpiHeadEuler>(bn, ctx, A, B, M, N, K, epi, scratch, scratch_bytes,
                                            stream, &rc);
        break;
      default: return set_error(-1, "gemm: unknown epilogue %d", epi.kind);
    }
    if (done) return rc;
  }
  if (tile == kSingle256 || (tile != kSingle128 && N % 256 == 0))
    return dispatch_bf16<256>(ctx, A, B, M, N, K, epi, scratch, scratch_bytes, stream);
  return dispatch_bf16<128>(ctx, A, B, M, N, K, epi, scratch, scratch_bytes, stream);
}

template <int EPI>
int launch_i8_kind(const DevCtx& ctx, const int8_t* A, const int8_t* B, int M, int N, int K,
                   const GemmEpilogue& epi, void* scratch, size_t scratch_bytes,
                   cudaStream_t stream) {
  const int tile = choose_tile(M, N);
  if (tile == kPair256 || tile == kPair128) {
    int rc = 0;
    const int r = tile == kPair256
                      ? launch_pair<256, true, EPI>(ctx, A, B, M, N, K, epi, scratch,
                                                    scratch_bytes, stream, &rc)
                      : launch_pair<128, true, EPI>(ctx, A, B, M, N, K, epi, scratch,
                                                    scratch_bytes, stream, &rc);
    if (r == 0) return rc;
  }
  if (tile == kSingle128 || N % 256 != 0)
    return launch_impl<128, true, EPI>(ctx, A, B, M, N, K, epi, scratch, scratch_bytes, stream);
  return launch_impl<256, true, EPI>(ctx, A, B, M, N, K, epi, scratch, scratch_bytes, stream);
}

int launch_gemm_i8(const DevCtx& ctx, const int8_t* A, const int8_t* B, int M, int N, int K,
                   const GemmEpilogue& epi, void* scratch, size_t scratch_bytes,
                   cudaStream_t stream) {
  if (M <= 0) return 0;
  switch (epi.kind) {
    case kEpiInt8Deq:
      return launch_i8_kind<kEpiInt8Deq>(ctx, A, B, M, N, K, epi, scratch, scratch_bytes, stream);
    case kEpiI8Rope:
      return launch_i8_kind<kEpiI8Rope>(ctx, A, B, M, N, K, epi, scratch, scratch_bytes, stream);
    case kEpiI8Gelu:
      return launch_i8_kind<kEpiI8Gelu>(ctx, A, B, M, N, K, epi, scratch, scratch_bytes, stream);
    default: return set_error(-1, "gemm_i8: unknown epilogue %d", epi.kind);
  }
}

int launch_gemm_i8_grouped(const DevCtx& ctx, const int8_t* A, const int8_t* B, int M, int N,
                           int K, const GemmEpilogue& epi, void* scratch, size_t scratch_bytes,
                           cudaStream_t stream) {
  if (M <= 0) return 0;
  if (epi.kind != kEpiI8GroupGate || K % kGroupK || N % 128)
    return set_error(-1, "gemm_i8_grouped: K=%d must be a multiple of %d, N=%d of 128", K, kGroupK, N);
  using Cfg = PairCfg<128, false, 4>;
  auto kernel = k_gemm_pair_grouped<kEpiI8GroupGate>;
  static std::atomic<uint32_t> attr_done{0};
  const uint32_t bit = 1u << (ctx.device & 31);
  if (!(attr_done.load() & bit)) {
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(Cfg::kSmem));
    if (e != cudaSuccess)
      return set_error(-3, "gemm_i8_grouped: cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    attr_done.fetch_or(bit);
  }
  static std::atomic<int> cap_cache[64];
  int cap = cap_cache[ctx.device & 63].load();
  if (cap <= 0) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * (ctx.num_sms / 2));
    cfg.blockDim = dim3(192);
    cfg.dynamicSmemBytes = Cfg::kSmem;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kernel, &cfg) != cudaSuccess || n <= 0) {
      cudaGetLastError();
      return set_error(-3, "gemm_i8_grouped: no resident CTA pair");
    }
    cap = std::min(n, ctx.num_sms / 2);
    cap_cache[ctx.device & 63].store(cap);
  }
  CUtensorMap ta, tb;
  if (!make_tmap_2d(&ta, A, CU_TENSOR_MAP_DATA_TYPE_UINT8, uint64_t(M), uint64_t(K), uint64_t(K),
                    128, 128) ||
      !make_tmap_2d(&tb, B, CU_TENSOR_MAP_DATA_TYPE_UINT8, uint64_t(N), uint64_t(K), uint64_t(K),
                    64, 128))
    return set_error(-3, "gemm_i8_grouped: cuTensorMapEncodeTiled failed (M=%d N=%d K=%d)", M, N, K);
  GemmParams p{};
  p.M = M;
  p.N = N;
  p.k_blocks = K / kGroupK;  // the kernel schedules K in groups
  p.m_tiles = (M + 255) / 256;
  p.n_tiles = N / 128;
  p.epi = epi;
  p.err = ctx.err_flag;
  const int tiles = p.m_tiles * p.n_tiles;
  // A last wave that would leave pairs idle is split stream-K by groups over all pairs,
  // ahead of the whole waves (which run data-parallel): every pair gets at least one group
  // of it, the units below a split tile park their fp32 sums, the one holding its last group
  // adds them in its epilogue.
  const int sk_pairs = std::min(cap, kMaxSkCtas / 2);
  const int sk_tile0 = remainder_tile0(tiles, sk_pairs);
  const long long iters = static_cast<long long>(tiles - sk_tile0) * p.k_blocks;
  const bool use_sk = scratch != nullptr && scratch_bytes >= kScratchBytes &&
                      tiles > sk_pairs && iters >= sk_pairs && forced_sched() != 0;
  if (trace_gemm())
    std::fprintf(stderr, "h3b gemm i8 grouped M=%d N=%d K=%d tiles=%d cap=%d -> %s sk_tile0=%d\n",
                 M, N, K, tiles, cap, use_sk ? "hybrid stream-K" : "data-parallel",
                 use_sk ? sk_tile0 : 0);
  if (use_sk) {
    p.sk = 1;
    p.sk_tile0 = sk_tile0;
    p.sk_iters = iters;
    p.sk_slots = static_cast<uint32_t*>(scratch);
    p.sk_flags =
        reinterpret_cast<unsigned long long*>(static_cast<uint8_t*>(scratch) + kSkFlagsOffset);
    p.sk_seq = next_sk_seq();
    kernel<<<2 * sk_pairs, 192, Cfg::kSmem, stream>>>(ta, tb, p);
  } else {
    kernel<<<2 * std::min(tiles, cap), 192, Cfg::kSmem, stream>>>(ta, tb, p);
  }
  return check_launch("gemm_i8_grouped");
}

}  // namespace h3b
