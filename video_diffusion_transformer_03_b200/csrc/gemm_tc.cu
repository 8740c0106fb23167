// Persistent, warp-specialised tcgen05 GEMM for the block's projections (QKV, out-proj,
// FC1, FC2) and the int8 row-scaled FC2:  out = A[M, K] * B[N, K]^T  with a fused
// epilogue.
//
// Roles (192 threads, one CTA per SM):
//   warp 0      TMA producer: 128-byte-swizzled [128 x 128 B] A tiles and [BN x 128 B] B
//               tiles into a STAGES-deep shared-memory ring;
//   warp 1      TMEM allocator and MMA issuer (one thread): 4 x tcgen05.mma per stage,
//               accumulating a 128 x BN fp32 / int32 tile in tensor memory; two
//               accumulator buffers so the epilogue of tile i overlaps the MMAs of
//               tile i + 1;
//   warps 2..5  epilogue: tcgen05.ld of the accumulator (thread = row, 32 columns per
//               load), bias / GELU / RoPE / gated residual / int8 dequant, 16-byte
//               global stores.
// Tiles are visited in groups of 16 M-tiles (M fastest) so that CTAs running together
// share weight tiles in L2.
#include "kernels.h"
#include "ptx.cuh"
#include "tmap.h"

#include <algorithm>
#include <atomic>

namespace h3b {

namespace {

constexpr int kBM = 128;
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
  GemmEpilogue epi;
  uint32_t* err;
};

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

// Same as load_bf16x32 but through the coherent path (the residual is read and written
// by this kernel).
__device__ __forceinline__ void load_bf16x32_rw(const bf16* src, float (&v)[32]) {
  const uint4* s = reinterpret_cast<const uint4*>(src);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint4 u = s[i];
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

// Epilogue of one 32-column chunk of one row.
template <int EPI>
__device__ __forceinline__ void epilogue_chunk(const GemmEpilogue& e, int row, int col,
                                               const uint32_t (&r)[32]) {
  float v[32];
  if constexpr (EPI == kEpiInt8Deq) {
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
    if (e.bias_f32) {
      float b[32];
      load_f32x32(e.bias_f32 + col, b);
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] += b[j];
    }
  } else {
    float b[32];
    load_bf16x32(e.bias + col, b);
#pragma unroll
    for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]) + b[j];
  }

  if constexpr (EPI == kEpiGelu) {
#pragma unroll
    for (int j = 0; j < 32; ++j) v[j] = gelu_tanh(v[j]);
  }
  if constexpr (EPI == kEpiRope) {
    if (col < e.rope_cols) {
      const int half = e.head_dim >> 1;
      const float4* cs = reinterpret_cast<const float4*>(
          e.rope_cs + (size_t(row) * half + ((col % e.head_dim) >> 1)) * 2);
#pragma unroll
      for (int i = 0; i < 8; ++i) {  // 2 pairs per float4 (cos0, sin0, cos1, sin1)
        const float4 c = __ldg(cs + i);
        const float x0 = v[4 * i], x1 = v[4 * i + 1], y0 = v[4 * i + 2], y1 = v[4 * i + 3];
        v[4 * i + 0] = x0 * c.x - x1 * c.y;
        v[4 * i + 1] = x0 * c.y + x1 * c.x;
        v[4 * i + 2] = y0 * c.z - y1 * c.w;
        v[4 * i + 3] = y0 * c.w + y1 * c.z;
      }
    }
  }
  bf16* dst = e.out + size_t(row) * e.ld_out + col;
  if constexpr (EPI == kEpiGateResid || EPI == kEpiInt8Deq) {
    float g[32], res[32];
    load_f32x32(e.gate + col, g);
    load_bf16x32_rw(dst, res);
#pragma unroll
    for (int j = 0; j < 32; ++j) v[j] = fmaf(g[j], v[j], res[j]);
  }
  store_bf16x32(dst, v);
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
  const int num_tiles = p.m_tiles * p.n_tiles;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------------------------------------------------------- producer
      int stage = 0;
      uint32_t phase = 0;
      int armed[STAGES];
#pragma unroll
      for (int s = 0; s < STAGES; ++s) armed[s] = -1;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        int mb, nb;
        tile_coords(tile, p.m_tiles, p.n_tiles, mb, nb);
        for (int kb = 0; kb < p.k_blocks; ++kb) {
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
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++local) {
        const int buf = local & 1;
        const uint32_t use = static_cast<uint32_t>(local >> 1);
        if (!wait_bar(&tempty[buf], (use & 1u) ^ 1u, abort_flag, p.err, kErrGemmWait)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf * BN);
        for (int kb = 0; kb < p.k_blocks; ++kb) {
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
            const uint32_t acc = (kb | k) != 0 ? 1u : 0u;
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
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++local) {
      int mb, nb;
      tile_coords(tile, p.m_tiles, p.n_tiles, mb, nb);
      const int buf = local & 1;
      const uint32_t use = static_cast<uint32_t>(local >> 1);
      bool ok = wait_bar(&tfull[buf], use & 1u, abort_flag, p.err, kErrGemmWait);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const int row = mb * kBM + row_in_tile;
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(tmem_base + lane_addr + static_cast<uint32_t>(buf * BN + c * 32), r);
        tmem_wait_ld(r);
        if (row < p.M) epilogue_chunk<EPI>(p.epi, row, nb * BN + c * 32, r);
      }
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

template <int BN, bool INT8, int EPI>
int launch_impl(const DevCtx& ctx, const void* A, const void* B, int M, int N, int K,
                const GemmEpilogue& epi, cudaStream_t stream) {
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

  GemmParams p;
  p.M = M;
  p.N = N;
  p.k_blocks = K / bk;
  p.m_tiles = (M + kBM - 1) / kBM;
  p.n_tiles = N / BN;
  p.epi = epi;
  p.err = ctx.err_flag;
  const int tiles = p.m_tiles * p.n_tiles;
  const int grid = std::min(tiles, ctx.num_sms);
  kernel<<<grid, 192, Cfg::kSmem, stream>>>(ta, tb, p);
  return check_launch("gemm");
}

template <int BN>
int dispatch_bf16(const DevCtx& ctx, const bf16* A, const bf16* B, int M, int N, int K,
                  const GemmEpilogue& epi, cudaStream_t s) {
  switch (epi.kind) {
    case kEpiBias: return launch_impl<BN, false, kEpiBias>(ctx, A, B, M, N, K, epi, s);
    case kEpiGelu: return launch_impl<BN, false, kEpiGelu>(ctx, A, B, M, N, K, epi, s);
    case kEpiRope: return launch_impl<BN, false, kEpiRope>(ctx, A, B, M, N, K, epi, s);
    case kEpiGateResid:
      return launch_impl<BN, false, kEpiGateResid>(ctx, A, B, M, N, K, epi, s);
    default: return set_error(-1, "gemm: unknown epilogue %d", epi.kind);
  }
}

}  // namespace

int launch_gemm_bf16(const DevCtx& ctx, const bf16* A, const bf16* B, int M, int N, int K,
                     const GemmEpilogue& epi, cudaStream_t stream) {
  if (M <= 0) return 0;
  if (N % 256 == 0) return dispatch_bf16<256>(ctx, A, B, M, N, K, epi, stream);
  return dispatch_bf16<128>(ctx, A, B, M, N, K, epi, stream);
}

int launch_gemm_i8(const DevCtx& ctx, const int8_t* A, const int8_t* B, int M, int N, int K,
                   const GemmEpilogue& epi, cudaStream_t stream) {
  if (M <= 0) return 0;
  if (N % 256 == 0) return launch_impl<256, true, kEpiInt8Deq>(ctx, A, B, M, N, K, epi, stream);
  return launch_impl<128, true, kEpiInt8Deq>(ctx, A, B, M, N, K, epi, stream);
}

}  // namespace h3b
