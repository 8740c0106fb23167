// Joint video+audio self-attention, flash style, on tcgen05.
//
// One CTA per (128-query tile, head); full non-causal attention over all tokens of the
// joint stream.  The q and k columns of the packed QKV buffer are already rotated by
// 3D RoPE in the QKV projection's epilogue, so tiles are consumed as loaded.
//
// Roles (192 threads):
//   warp 0      TMA producer: Q tile once, then K_j and V_j tiles into 2-stage rings
//               (K stages are released as soon as S_j = Q K_j^T completes, V stages after
//               O += P_j V_j);
//   warp 1      MMA issuer: S_j into one of two TMEM score buffers (128 fp32 columns each),
//               then O += P_{j-1} V_{j-1} (P from shared memory, V as an MN-major operand)
//               into a TMEM output accumulator;
//   warps 2..5  softmax: thread = query row; the whole 128-wide score row is in registers,
//               so row max and row sum need no shuffles.  Exponentials are base 2 with
//               the 1/sqrt(head_dim) scale folded in.  Rescaling of O is lazy: the
//               running max used for the exponentials only moves when the tile max
//               exceeds it by more than 8 (a factor 256), and then O (in TMEM) and the
//               row sum are multiplied by 2^(m_old - m_new).
// TMEM map: S0 [0,128), S1 [128,256), O [256, 256 + head_dim).
#include "kernels.h"
#include "ptx.cuh"
#include "tmap.h"

#include <atomic>
#include <cmath>

namespace h3b {

namespace {

constexpr uint32_t kBox = 128 * 128;  // [128 rows x 128 B] swizzled box

template <int HD>
struct AttnCfg {
  static constexpr int kNBox = HD / 64;
  static constexpr uint32_t kQBytes = kNBox * kBox;
  static constexpr uint32_t kKVBytes = kNBox * kBox;
  static constexpr uint32_t kPBytes = 2 * kBox;
  static constexpr size_t kSmem = 1024 + kQBytes + 4 * size_t(kKVBytes) + 2 * kPBytes + 256;
};

struct AttnParams {
  int n;            // tokens
  int d;            // n_heads * head_dim
  int n_kv;         // ceil(n / 128)
  float scale_log2; // log2(e) / sqrt(head_dim)
  bf16* out;        // [n, d]
  uint32_t* err;
};

// 2^x on the FMA pipe, for a share of the probabilities so that the MUFU unit (16 ex2 per
// clock per SM, the same time per 128 x 128 tile as the tile's MMAs) is not the limit.
// Range reduction to n = round(x) by adding the 1.5 * 2^23 shifter, f = x - n in
// [-1/2, 1/2], 2^f by a degree-3 polynomial fitted here by iteratively reweighted least
// squares on the relative error (max 7.5e-5 over x in [-125, 8]), then 2^n added to the
// exponent field.  x is clamped at -125 so the exponent add cannot underflow.
__device__ __forceinline__ float exp2_fma(float x) {
  x = fmaxf(x, -125.0f);
  const float shifter = 12582912.0f;
  const float t = x + shifter;
  const int n = __float_as_int(t) - __float_as_int(shifter);
  const float f = x - (t - shifter);
  float p = 0.05517259240150452f;
  p = fmaf(p, f, 0.24261370301246643f);
  p = fmaf(p, f, 0.6932610273361206f);
  p = fmaf(p, f, 0.9999278783798218f);
  return __int_as_float(__float_as_int(p) + (n << 23));
}

__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_timer_ns() - t0 > kWaitLimitNs) return;
  }
}

template <int HD>
__global__ void __launch_bounds__(192, 1)
    k_attention_tc(const __grid_constant__ CUtensorMap tm, const AttnParams p) {
  using Cfg = AttnCfg<HD>;
  constexpr uint32_t IDESC_S = idesc_bf16(128, 128, false);
  constexpr uint32_t IDESC_PV = idesc_bf16(128, HD, true);
  constexpr uint32_t kTmemCols = 512;
  constexpr uint32_t kOCol = 256;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sK = sQ + Cfg::kQBytes;          // 2 stages
  uint8_t* sV = sK + 2 * Cfg::kKVBytes;     // 2 stages
  uint8_t* sP = sV + 2 * Cfg::kKVBytes;     // 2 buffers
  uint64_t* bars = reinterpret_cast<uint64_t*>(sP + 2 * Cfg::kPBytes);
  uint64_t* q_full = bars + 0;
  uint64_t* k_full = bars + 1;
  uint64_t* k_empty = bars + 3;
  uint64_t* v_full = bars + 5;
  uint64_t* v_empty = bars + 7;
  uint64_t* s_full = bars + 9;
  uint64_t* s_free = bars + 11;
  uint64_t* p_full = bars + 13;
  uint64_t* p_free = bars + 15;
  uint64_t* drain = bars + 17;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 18);
  volatile uint32_t* abort_flag = tmem_slot + 1;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int qt = blockIdx.x;
  const int head = blockIdx.y;
  const int n_kv = p.n_kv;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
      mbar_init(&s_full[s], 1);
      mbar_init(&s_free[s], 4);
      mbar_init(&p_full[s], 4);
      mbar_init(&p_free[s], 1);
    }
    mbar_init(drain, 1);
    *abort_flag = 0u;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) tma_prefetch_map(&tm);
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------------ producer
      const int xq = head * HD, xk = p.d + head * HD, xv = 2 * p.d + head * HD;
      int k_armed[2] = {-1, -1}, v_armed[2] = {-1, -1};
      mbar_arrive_expect_tx(q_full, Cfg::kQBytes);
#pragma unroll
      for (int b = 0; b < Cfg::kNBox; ++b)
        tma_load_2d(sQ + b * kBox, &tm, q_full, xq + 64 * b, qt * 128);
      bool ok = true;
      for (int j = 0; j < n_kv && ok; ++j) {
        const int st = j & 1;
        const uint32_t ph = static_cast<uint32_t>(j >> 1) & 1u;
        if (!wait_bar(&k_empty[st], ph ^ 1u, abort_flag, p.err, kErrAttnWait)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&k_full[st], Cfg::kKVBytes);
#pragma unroll
        for (int b = 0; b < Cfg::kNBox; ++b)
          tma_load_2d(sK + st * Cfg::kKVBytes + b * kBox, &tm, &k_full[st], xk + 64 * b,
                      j * 128);
        k_armed[st] = static_cast<int>(ph);
        if (!wait_bar(&v_empty[st], ph ^ 1u, abort_flag, p.err, kErrAttnWait)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&v_full[st], Cfg::kKVBytes);
#pragma unroll
        for (int b = 0; b < Cfg::kNBox; ++b)
          tma_load_2d(sV + st * Cfg::kKVBytes + b * kBox, &tm, &v_full[st], xv + 64 * b,
                      j * 128);
        v_armed[st] = static_cast<int>(ph);
      }
      if (!ok) {
        drain_wait(q_full, 0);
        for (int s = 0; s < 2; ++s) {
          if (k_armed[s] >= 0) drain_wait(&k_full[s], static_cast<uint32_t>(k_armed[s]));
          if (v_armed[s] >= 0) drain_wait(&v_full[s], static_cast<uint32_t>(v_armed[s]));
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------------ MMA issuer
      bool ok = wait_bar(q_full, 0, abort_flag, p.err, kErrAttnWait);
      const uint32_t q0 = smem_u32(sQ);
      for (int j = 0; j <= n_kv && ok; ++j) {
        if (j < n_kv) {
          const int st = j & 1;
          const uint32_t ph = static_cast<uint32_t>(j >> 1) & 1u;
          if (!wait_bar(&k_full[st], ph, abort_flag, p.err, kErrAttnWait)) break;
          if (j >= 2 && !wait_bar(&s_free[st], ph ^ 1u, abort_flag, p.err, kErrAttnWait))
            break;
          tc_fence_after();
          const uint32_t k0 = smem_u32(sK + st * Cfg::kKVBytes);
#pragma unroll
          for (int kk = 0; kk < HD / 16; ++kk) {
            const uint32_t off = (kk >> 2) * kBox + (kk & 3) * 32;
            umma_f16(tmem + st * 128, sdesc_sw128(q0 + off, 16, 1024),
                     sdesc_sw128(k0 + off, 16, 1024), IDESC_S, kk > 0 ? 1u : 0u);
          }
          tc_commit(&s_full[st]);
          tc_commit(&k_empty[st]);
        }
        if (j >= 1) {
          const int i = j - 1;
          const int pb = i & 1;
          const uint32_t ph = static_cast<uint32_t>(i >> 1) & 1u;
          if (!wait_bar(&p_full[pb], ph, abort_flag, p.err, kErrAttnWait)) break;
          if (!wait_bar(&v_full[pb], ph, abort_flag, p.err, kErrAttnWait)) break;
          tc_fence_after();
          const uint32_t p0 = smem_u32(sP + pb * Cfg::kPBytes);
          const uint32_t v0 = smem_u32(sV + pb * Cfg::kKVBytes);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t poff = (kk >> 2) * kBox + (kk & 3) * 32;
            umma_f16(tmem + kOCol, sdesc_sw128(p0 + poff, 16, 1024),
                     sdesc_sw128(v0 + kk * 2048, kBox, 1024), IDESC_PV,
                     (i > 0 || kk > 0) ? 1u : 0u);
          }
          tc_commit(&p_free[pb]);
          tc_commit(&v_empty[pb]);
        }
      }
      tc_commit(drain);
      drain_wait(drain, 0);
    }
  } else {
    // ------------------------------------------------------------------ softmax
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;  // query row within the tile
    const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
    const float sl2 = p.scale_log2;
    float m_used = -INFINITY;
    float l = 0.f;
    bool ok = true;
    for (int j = 0; j < n_kv; ++j) {
      const int sb = j & 1;
      const uint32_t ph = static_cast<uint32_t>(j >> 1) & 1u;
      ok = __all_sync(0xffffffffu, wait_bar(&s_full[sb], ph, abort_flag, p.err, kErrAttnWait));
      if (!ok) break;
      tc_fence_after();
      float s[128];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t r[32];
        tmem_ld32(tmem + lane_addr + sb * 128 + c * 32, r);
        tmem_wait_ld(r);
#pragma unroll
        for (int t = 0; t < 32; ++t) s[c * 32 + t] = __uint_as_float(r[t]);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_free[sb]);

      if ((j + 1) * 128 > p.n) {
        const int valid = p.n - j * 128;
#pragma unroll
        for (int c = 0; c < 128; ++c)
          if (c >= valid) s[c] = -INFINITY;
      }
      float m8[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) m8[i] = s[i];
#pragma unroll
      for (int c = 8; c < 128; ++c) m8[c & 7] = fmaxf(m8[c & 7], s[c]);
#pragma unroll
      for (int i = 4; i > 0; i >>= 1)
#pragma unroll
        for (int k = 0; k < i; ++k) m8[k] = fmaxf(m8[k], m8[k + i]);
      const float mxs = m8[0] * sl2;
      if (j == 0) {
        m_used = mxs;
      } else {
        const bool need = mxs > m_used + 8.0f;
        if (__any_sync(0xffffffffu, need)) {
          // O must hold every earlier P V product before it is rescaled
          const int i = j - 1;
          ok = __all_sync(0xffffffffu,
                          wait_bar(&p_free[i & 1], static_cast<uint32_t>(i >> 1) & 1u,
                                   abort_flag, p.err, kErrAttnWait));
          if (!ok) break;
          tc_fence_after();
          const float alpha = need ? ex2_approx(m_used - mxs) : 1.0f;
#pragma unroll
          for (int c = 0; c < HD / 32; ++c) {
            uint32_t r[32];
            const uint32_t addr = tmem + lane_addr + kOCol + c * 32;
            tmem_ld32(addr, r);
            tmem_wait_ld(r);
#pragma unroll
            for (int t = 0; t < 32; ++t) r[t] = __float_as_uint(__uint_as_float(r[t]) * alpha);
            tmem_st32(addr, r);
          }
          tmem_wait_st();
          l *= alpha;
          if (need) m_used = mxs;
        }
      }
      float sum8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int c = 0; c < 128; ++c) {
        const float x = fmaf(s[c], sl2, -m_used);
        const float e = (c & 3) == 3 ? exp2_fma(x) : ex2_approx(x);
        sum8[c & 7] += e;
        s[c] = e;
      }
#pragma unroll
      for (int i = 4; i > 0; i >>= 1)
#pragma unroll
        for (int k = 0; k < i; ++k) sum8[k] += sum8[k + i];
      l += sum8[0];
      if (j >= 2) {
        ok = __all_sync(0xffffffffu,
                        wait_bar(&p_free[sb], ph ^ 1u, abort_flag, p.err, kErrAttnWait));
        if (!ok) break;
      }
      uint8_t* pbuf = sP + sb * Cfg::kPBytes + row * 128;
#pragma unroll
      for (int c16 = 0; c16 < 16; ++c16) {
        uint4 u;
        u.x = pack_bf16x2(s[c16 * 8 + 0], s[c16 * 8 + 1]);
        u.y = pack_bf16x2(s[c16 * 8 + 2], s[c16 * 8 + 3]);
        u.z = pack_bf16x2(s[c16 * 8 + 4], s[c16 * 8 + 5]);
        u.w = pack_bf16x2(s[c16 * 8 + 6], s[c16 * 8 + 7]);
        const int chunk = (c16 & 7) ^ (row & 7);
        *reinterpret_cast<uint4*>(pbuf + (c16 >> 3) * kBox + chunk * 16) = u;
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[sb]);
    }
    if (ok) {
      const int last = n_kv - 1;
      ok = __all_sync(0xffffffffu,
                      wait_bar(&p_free[last & 1], static_cast<uint32_t>(last >> 1) & 1u,
                               abort_flag, p.err, kErrAttnWait));
    }
    if (ok) {
      tc_fence_after();
      const float inv_l = 1.0f / l;
      const int grow = qt * 128 + row;
#pragma unroll
      for (int c = 0; c < HD / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(tmem + lane_addr + kOCol + c * 32, r);
        tmem_wait_ld(r);
        if (grow < p.n) {
          uint4* dst =
              reinterpret_cast<uint4*>(p.out + size_t(grow) * p.d + head * HD + c * 32);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            uint4 u;
            u.x = pack_bf16x2(__uint_as_float(r[8 * i + 0]) * inv_l,
                              __uint_as_float(r[8 * i + 1]) * inv_l);
            u.y = pack_bf16x2(__uint_as_float(r[8 * i + 2]) * inv_l,
                              __uint_as_float(r[8 * i + 3]) * inv_l);
            u.z = pack_bf16x2(__uint_as_float(r[8 * i + 4]) * inv_l,
                              __uint_as_float(r[8 * i + 5]) * inv_l);
            u.w = pack_bf16x2(__uint_as_float(r[8 * i + 6]) * inv_l,
                              __uint_as_float(r[8 * i + 7]) * inv_l);
            dst[i] = u;
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <int HD>
int launch_hd(const DevCtx& ctx, const bf16* qkv, int n, int heads, bf16* out,
              cudaStream_t stream) {
  using Cfg = AttnCfg<HD>;
  const int d = heads * HD;
  CUtensorMap tm;
  if (!make_tmap_2d(&tm, qkv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, uint64_t(n), uint64_t(3 * d),
                    uint64_t(3 * d) * 2, 128, 64))
    return set_error(-3, "attention: cuTensorMapEncodeTiled failed (n=%d d=%d)", n, d);
  auto kernel = k_attention_tc<HD>;
  static std::atomic<uint32_t> attr_done{0};
  const uint32_t bit = 1u << (ctx.device & 31);
  if (!(attr_done.load() & bit)) {
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(Cfg::kSmem));
    if (e != cudaSuccess)
      return set_error(-3, "attention: cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    attr_done.fetch_or(bit);
  }
  AttnParams p;
  p.n = n;
  p.d = d;
  p.n_kv = (n + 127) / 128;
  p.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(double(HD)));
  p.out = out;
  p.err = ctx.err_flag;
  dim3 grid((n + 127) / 128, heads);
  kernel<<<grid, 192, Cfg::kSmem, stream>>>(tm, p);
  return check_launch("attention");
}

}  // namespace

int launch_attention(const DevCtx& ctx, const bf16* qkv, int n_tokens, int n_heads,
                     int head_dim, bf16* out, cudaStream_t stream) {
  if (n_tokens <= 0) return 0;
  if (head_dim == 128) return launch_hd<128>(ctx, qkv, n_tokens, n_heads, out, stream);
  if (head_dim == 64) return launch_hd<64>(ctx, qkv, n_tokens, n_heads, out, stream);
  return set_error(-1, "attention: head_dim %d unsupported (64 or 128)", head_dim);
}

}  // namespace h3b
