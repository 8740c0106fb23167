// Joint video+audio self-attention, flash style, on tcgen05.
//
// Full non-causal attention over all tokens of the joint stream, per head.  The q and k
// columns of the packed QKV buffer are already rotated by 3D RoPE in the QKV projection's
// epilogue, so tiles are consumed as loaded.
//
// Work: a unit is one (head, 128-query tile) pair and has n_kv steps, one per 128-key
// tile.  The units' steps, laid end to end (u * n_kv + j), are cut into one equal
// contiguous range per CTA.  With a scratch buffer the grid is persistent (one CTA per
// SM), so every SM gets the same number of steps whatever the unit count; a unit cut
// between two CTAs is finished by the CTA holding its last key tile (the owner), which
// merges the running state (unnormalised O, row max, row sum) that the lower CTA left in
// the scratch.  Each CTA walks its units from last to first, so its contribution to a
// split unit is computed first and the owner's merge, done last, does not wait in
// practice.  Without scratch the grid has one CTA per unit (nothing is split).
//
// Roles (192 threads):
//   warp 0      TMA producer: the Q tile of each unit (once the previous unit's last S
//               has read the buffer), then K_j and V_j tiles into 2-stage rings (K stages are released as soon as S_j = Q K_j^T completes,
//               V stages after O += P_j V_j);
//   warp 1      MMA issuer: S_j into one of two TMEM score buffers (128 fp32 columns
//               each), then O += P_{j-1} V_{j-1} (P from shared memory, V as an MN-major
//               operand) into a TMEM output accumulator.  At the first step of a unit the
//               previous unit's last P V goes first, so its end does not wait for the
//               new unit's first S;
//   warps 2..5  softmax: thread = query row; the whole 128-wide score row is in registers,
//               so row max and row sum need no shuffles.  Exponentials are base 2 with
//               the 1/sqrt(head_dim) scale folded in, all on the MUFU unit (the score
//               row's load-exp-pack chain is latency bound, so moving a share of the
//               exponentials to FMA-pipe polynomials only adds instructions).  Rescaling of O is lazy: the
//               running max used for the exponentials only moves when the tile max
//               exceeds it by more than 8 (a factor 256), and then O (in TMEM) and the
//               row sum are multiplied by 2^(m_old - m_new).  At the end of a unit the
//               same warps normalise and store O, or park / merge a split unit's state.
// TMEM map: S0 [0,128), S1 [128,256), O [256, 256 + head_dim).
#include "kernels.h"
#include "ptx.cuh"
#include "tmap.h"

#include <algorithm>
#include <atomic>
#include <cmath>

namespace h3b {

namespace {

constexpr uint32_t kBox = 128 * 128;  // [128 rows x 128 B] swizzled box

// Shared memory: Q, K x 2, V x 2, P x 2 (the softmax writes P_j while P_{j-1} V_{j-1}
// may still be running).
template <int HD>
struct AttnCfg {
  static constexpr int kNBox = HD / 64;
  static constexpr uint32_t kQBytes = kNBox * kBox;
  static constexpr uint32_t kKVBytes = kNBox * kBox;
  static constexpr uint32_t kPBytes = 2 * kBox;
  static constexpr size_t kSmem =
      1024 + size_t(kQBytes) + 4 * size_t(kKVBytes) + 2 * size_t(kPBytes) + 256;
};

struct AttnParams {
  int n;             // tokens
  int d;             // n_heads * head_dim
  int n_kv;          // ceil(n / 128): key tiles, and steps per unit
  int n_qt;          // ceil(n / 128): query tiles per head
  long long steps;   // units * n_kv
  float scale_log2;  // log2(e) / sqrt(head_dim)
  bf16* out;         // [n, d]
  float4* part_o;    // [gridDim.x][head_dim / 4][128] unnormalised O of a split unit
  float2* part_ml;   // [gridDim.x][128] (running max, row sum) of a split unit
  unsigned long long* flags;  // [gridDim.x][4]
  unsigned long long seq;
  uint32_t* err;
};

__device__ __forceinline__ float max3(float a, float b, float c) {
  float m;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(m) : "f"(a), "f"(b), "f"(c));
  return m;
}

__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_timer_ns() - t0 > kWaitLimitNs) return;
  }
}

// This CTA's step range [begin, end) and the units it touches.
struct Range {
  long long begin, end;
  int u_first, u_last;
};

__device__ __forceinline__ long long range_begin(const AttnParams& p, int c) {
  return p.steps * c / static_cast<long long>(gridDim.x);
}

__device__ __forceinline__ Range cta_range(const AttnParams& p) {
  Range r;
  r.begin = range_begin(p, static_cast<int>(blockIdx.x));
  r.end = range_begin(p, static_cast<int>(blockIdx.x) + 1);
  r.u_first = static_cast<int>(r.begin / p.n_kv);
  r.u_last = static_cast<int>((r.end - 1) / p.n_kv);
  return r;
}

// Segment k of the walk (units from the last to the first): unit u_last - k, key tiles
// [j0, j1).  j1 < n_kv: the lower part of a split unit; j0 > 0: the upper part.  A range
// is at least n_kv steps long, so no segment is both.
__device__ __forceinline__ void segment(const AttnParams& p, const Range& r, int k, int& unit,
                                        int& j0, int& j1) {
  unit = r.u_last - k;
  const long long base = static_cast<long long>(unit) * p.n_kv;
  j0 = static_cast<int>(r.begin > base ? r.begin - base : 0ll);
  j1 = static_cast<int>(r.end - base < p.n_kv ? r.end - base : static_cast<long long>(p.n_kv));
}

// Wait until the flag holds `seq`; false on abort or time-out (records kErrAttnWait).
__device__ __forceinline__ bool wait_flag(const unsigned long long* f, unsigned long long seq,
                                          volatile uint32_t* abort_flag, uint32_t* err) {
  if (ld_acquire_u64(f) == seq) return true;
  const uint64_t t0 = global_timer_ns();
  while (ld_acquire_u64(f) != seq) {
    if (*abort_flag || global_timer_ns() - t0 > kWaitLimitNs) {
      *abort_flag = 1u;
      atomicCAS(err, 0u, kErrAttnWait);
      return false;
    }
  }
  return true;
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
  uint64_t* q_empty = bars + 1;
  uint64_t* k_full = bars + 2;   // [2]
  uint64_t* k_empty = bars + 4;  // [2]
  uint64_t* v_full = bars + 6;   // [2]
  uint64_t* v_empty = bars + 8;  // [2]
  uint64_t* s_full = bars + 10;  // [2]
  uint64_t* s_free = bars + 12;  // [2]
  uint64_t* p_full = bars + 14;  // [2]
  uint64_t* p_free = bars + 16;  // [2]
  uint64_t* o_empty = bars + 18;
  uint64_t* drain = bars + 19;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 20);
  volatile uint32_t* abort_flag = tmem_slot + 1;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const Range rg = cta_range(p);
  const int n_seg = rg.u_last - rg.u_first + 1;

  if (threadIdx.x == 0) {
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
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    mbar_init(o_empty, 4);
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
      int k_armed[2] = {-1, -1}, v_armed[2] = {-1, -1}, q_armed = -1;
      bool ok = true;
      int t = 0;  // step counter of this CTA (ring position)
      for (int k = 0; k < n_seg && ok; ++k) {
        int unit, j0, j1;
        segment(p, rg, k, unit, j0, j1);
        const int head = unit / p.n_qt, qt = unit % p.n_qt;
        const int xq = head * HD, xk = p.d + head * HD, xv = 2 * p.d + head * HD;
        if (k > 0 && !wait_bar(q_empty, static_cast<uint32_t>(k - 1) & 1u, abort_flag, p.err,
                               kErrAttnWait)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(q_full, Cfg::kQBytes);
#pragma unroll
        for (int b = 0; b < Cfg::kNBox; ++b)
          tma_load_2d(sQ + b * kBox, &tm, q_full, xq + 64 * b, qt * 128);
        q_armed = k & 1;
        for (int j = j0; j < j1; ++j, ++t) {
          const int st = t & 1;
          const uint32_t ph = static_cast<uint32_t>(t >> 1) & 1u;
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
      }
      if (!ok) {
        // let the copies in flight land before the CTA's shared memory is released
        if (q_armed >= 0) drain_wait(q_full, static_cast<uint32_t>(q_armed));
        for (int s = 0; s < 2; ++s) {
          if (k_armed[s] >= 0) drain_wait(&k_full[s], static_cast<uint32_t>(k_armed[s]));
          if (v_armed[s] >= 0) drain_wait(&v_full[s], static_cast<uint32_t>(v_armed[s]));
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------------ MMA issuer
      // Two cursors over the same walk: the S side (step t) runs one step ahead of the
      // P V side (step t - 1).
      int ks = 0, js = 0, js0 = 0, js1 = 0, unit_s = 0;  // S cursor: segment, key tile
      int kp = 0, jp = 0, jp0 = 0, jp1 = 0, unit_p = 0;  // P V cursor
      segment(p, rg, 0, unit_s, js0, js1);
      js = js0;
      segment(p, rg, 0, unit_p, jp0, jp1);
      jp = jp0;
      auto issue_s = [&](long long t) -> bool {
        const int st = static_cast<int>(t & 1);
        const uint32_t ph = static_cast<uint32_t>(t >> 1) & 1u;
        if (js == js0 &&
            !wait_bar(q_full, static_cast<uint32_t>(ks) & 1u, abort_flag, p.err, kErrAttnWait))
          return false;
        if (!wait_bar(&k_full[st], ph, abort_flag, p.err, kErrAttnWait)) return false;
        if (t >= 2 && !wait_bar(&s_free[st], ph ^ 1u, abort_flag, p.err, kErrAttnWait))
          return false;
        tc_fence_after();
        const uint32_t q0 = smem_u32(sQ);
        const uint32_t k0 = smem_u32(sK + st * Cfg::kKVBytes);
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint32_t off = (kk >> 2) * kBox + (kk & 3) * 32;
          umma_f16(tmem + st * 128, sdesc_sw128(q0 + off, 16, 1024),
                   sdesc_sw128(k0 + off, 16, 1024), IDESC_S, kk > 0 ? 1u : 0u);
        }
        tc_commit(&s_full[st]);
        tc_commit(&k_empty[st]);
        if (++js == js1) {  // last S of this unit: the Q buffer may be refilled
          tc_commit(q_empty);
          if (++ks < n_seg) {
            segment(p, rg, ks, unit_s, js0, js1);
            js = js0;
          }
        }
        return true;
      };
      auto issue_pv = [&](long long i) -> bool {
        const int vb = static_cast<int>(i & 1);
        const uint32_t ph = static_cast<uint32_t>(i >> 1) & 1u;
        const bool first = jp == jp0;
        // the previous unit's O must have been read out before it is overwritten
        if (first && kp > 0 &&
            !wait_bar(o_empty, static_cast<uint32_t>(kp - 1) & 1u, abort_flag, p.err,
                      kErrAttnWait))
          return false;
        if (!wait_bar(&p_full[vb], ph, abort_flag, p.err, kErrAttnWait)) return false;
        if (!wait_bar(&v_full[vb], ph, abort_flag, p.err, kErrAttnWait)) return false;
        tc_fence_after();
        const uint32_t p0 = smem_u32(sP + vb * Cfg::kPBytes);
        const uint32_t v0 = smem_u32(sV + vb * Cfg::kKVBytes);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t poff = (kk >> 2) * kBox + (kk & 3) * 32;
          umma_f16(tmem + kOCol, sdesc_sw128(p0 + poff, 16, 1024),
                   sdesc_sw128(v0 + kk * 2048, kBox, 1024), IDESC_PV,
                   (!first || kk > 0) ? 1u : 0u);
        }
        tc_commit(&p_free[vb]);
        tc_commit(&v_empty[vb]);
        if (++jp == jp1 && ++kp < n_seg) {
          segment(p, rg, kp, unit_p, jp0, jp1);
          jp = jp0;
        }
        return true;
      };
      const long long total = rg.end - rg.begin;
      for (long long t = 0; t <= total; ++t) {
        // at a unit's first step (not the walk's first), finish the previous unit first
        const bool pv_first = t >= 1 && t < total && js == js0;
        if (pv_first && !issue_pv(t - 1)) break;
        if (t < total && !issue_s(t)) break;
        if (t >= 1 && !pv_first && !issue_pv(t - 1)) break;
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
    bool ok = true;
    int t = 0;
    for (int k = 0; k < n_seg && ok; ++k) {
      int unit, j0, j1;
      segment(p, rg, k, unit, j0, j1);
      float m_used = -INFINITY;
      float l = 0.f;
      for (int j = j0; j < j1; ++j, ++t) {
        const int sb = t & 1;
        const uint32_t ph = static_cast<uint32_t>(t >> 1) & 1u;
        ok = __all_sync(0xffffffffu, wait_bar(&s_full[sb], ph, abort_flag, p.err, kErrAttnWait));
        if (!ok) break;
        tc_fence_after();
        float s[128];
        {
          uint32_t r[128];
          tmem_ld128_sync(tmem + lane_addr + sb * 128, r);
#pragma unroll
          for (int q = 0; q < 128; ++q) s[q] = __uint_as_float(r[q]);
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
        // row max: eight independent chains of three-input maxima
        float m8[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          m8[i] = fmaxf(s[i], s[8 + i]);
#pragma unroll
          for (int c = 16; c < 128; c += 16) m8[i] = max3(m8[i], s[c + i], s[c + 8 + i]);
        }
        const float mx = max3(max3(m8[0], m8[1], m8[2]), max3(m8[3], m8[4], m8[5]),
                              fmaxf(m8[6], m8[7]));
        const float mxs = mx * sl2;
        if (j == j0) {
          m_used = mxs;
        } else {
          const bool need = mxs > m_used + 8.0f;
          if (__any_sync(0xffffffffu, need)) {
            // O must hold every earlier P V product of this unit before it is rescaled
            const int i = t - 1;
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
              for (int q = 0; q < 32; ++q) r[q] = __float_as_uint(__uint_as_float(r[q]) * alpha);
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
          const float e = ex2_approx(x);
          sum8[c & 7] += e;
          s[c] = e;
        }
#pragma unroll
        for (int i = 4; i > 0; i >>= 1)
#pragma unroll
          for (int q = 0; q < i; ++q) sum8[q] += sum8[q + i];
        l += sum8[0];
        if (t >= 2) {  // P buffer sb is free once P_{t-2} V_{t-2} has completed
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
      if (!ok) break;
      // ---- end of the unit: O holds every P V product once the last one completes
      {
        const int last = t - 1;
        ok = __all_sync(0xffffffffu,
                        wait_bar(&p_free[last & 1], static_cast<uint32_t>(last >> 1) & 1u,
                                 abort_flag, p.err, kErrAttnWait));
        if (!ok) break;
      }
      tc_fence_after();
      const int head = unit / p.n_qt, qt = unit % p.n_qt;
      const uint32_t o_addr = tmem + lane_addr + kOCol;
      if (j1 < p.n_kv) {
        // lower part of a split unit: park the running state for the owner (next CTA)
        float4* po = p.part_o + size_t(blockIdx.x) * (HD / 4) * 128 + row;
#pragma unroll 1
        for (int c = 0; c < HD / 32; ++c) {
          uint32_t r[32];
          tmem_ld32(o_addr + c * 32, r);
          tmem_wait_ld(r);
#pragma unroll
          for (int i = 0; i < 8; ++i)
            __stcg(po + size_t(c * 8 + i) * 128,
                   make_float4(__uint_as_float(r[4 * i]), __uint_as_float(r[4 * i + 1]),
                               __uint_as_float(r[4 * i + 2]), __uint_as_float(r[4 * i + 3])));
        }
        __stcg(p.part_ml + size_t(blockIdx.x) * 128 + row, make_float2(m_used, l));
        __threadfence();
        __syncwarp();
        if (lane == 0) st_release_u64(p.flags + blockIdx.x * 4 + quarter, p.seq);
      } else {
        // whole unit, or upper part of a split unit: merge the lower CTA's state, then
        // normalise and store
        float wa = 0.f, wb = 1.f;
        const float4* po = nullptr;
        if (j0 > 0) {
          const int src = static_cast<int>(blockIdx.x) - 1;
          ok = __all_sync(0xffffffffu, wait_flag(p.flags + src * 4 + quarter, p.seq,
                                                 abort_flag, p.err));
          if (!ok) break;
          const float2 ml = __ldcg(p.part_ml + size_t(src) * 128 + row);
          const float m = fmaxf(ml.x, m_used);
          wa = ex2_approx(ml.x - m);
          wb = ex2_approx(m_used - m);
          l = ml.y * wa + l * wb;
          po = p.part_o + size_t(src) * (HD / 4) * 128 + row;
        }
        const float inv_l = 1.0f / l;
        wa *= inv_l;
        wb *= inv_l;
        const int grow = qt * 128 + row;
#pragma unroll
        for (int c = 0; c < HD / 32; ++c) {
          uint32_t r[32];
          tmem_ld32(o_addr + c * 32, r);
          tmem_wait_ld(r);
          float o[32];
#pragma unroll
          for (int q = 0; q < 32; ++q) o[q] = __uint_as_float(r[q]) * wb;
          if (po != nullptr) {
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const float4 a = __ldcg(po + size_t(c * 8 + i) * 128);
              o[4 * i + 0] = fmaf(a.x, wa, o[4 * i + 0]);
              o[4 * i + 1] = fmaf(a.y, wa, o[4 * i + 1]);
              o[4 * i + 2] = fmaf(a.z, wa, o[4 * i + 2]);
              o[4 * i + 3] = fmaf(a.w, wa, o[4 * i + 3]);
            }
          }
          if (grow < p.n) {
            uint4* dst =
                reinterpret_cast<uint4*>(p.out + size_t(grow) * p.d + head * HD + c * 32);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              uint4 u;
              u.x = pack_bf16x2(o[8 * i + 0], o[8 * i + 1]);
              u.y = pack_bf16x2(o[8 * i + 2], o[8 * i + 3]);
              u.z = pack_bf16x2(o[8 * i + 4], o[8 * i + 5]);
              u.w = pack_bf16x2(o[8 * i + 6], o[8 * i + 7]);
              dst[i] = u;
            }
          }
        }
        if (po != nullptr) {
          // hand the flag back at zero, so a replay of this launch (same sequence value,
          // e.g. from a CUDA graph) waits for the lower CTA again
          __syncwarp();
          if (lane == 0) p.flags[(blockIdx.x - 1) * 4 + quarter] = 0ull;
        }
      }
      // O may now be overwritten by the next unit's first P V
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(o_empty);
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


// ============================================================================ two-tile form
// The unit is (head, 256-query block): two 128-query tiles that share every K and V tile
// load, each with its own softmax warpgroup, so the two softmax streams overlap each
// other and the tensor core (one softmax warpgroup per CTA was the critical path).
// Roles (384 threads, three warpgroups):
//   warpgroup 0  warp 0 TMA producer; warps 1 and 2 MMA issuers of query tiles 0 and 1
//                (one thread each, on different SMSPs); warp 3 idle;
//   warpgroup 1  softmax of query tile 0 (rows 0-127 of the unit);
//   warpgroup 2  softmax of query tile 1 (rows 128-255).
// The softmax fits the 168 registers a thread is launched with; the polynomial-exp2 form
// needs more and moves registers from warpgroup 0 (104) to the softmax (200), which adds
// up to the 384 x 168 of the launch.
// The tensor pipe keeps almost nothing queued behind the MMA it is executing, so any time
// an issuing thread spends between two MMAs (barrier waits, fences, commits, address
// arithmetic) leaves it idle: each 8-step product is issued from one asm block, and two
// issuers, one per tile, keep the pipe fed while either of them waits.
// TMEM: S0 [0,128), S1 [128,256), O0 [256,384), O1 [384,512): one score buffer per tile,
// so S_j+1 of a tile is computed as soon as its softmax has read S_j into registers.
// Shared memory: Q0, Q1, P0, P1 and a 3-slot ring of K/V tiles loaded in the order the
// tensor core consumes them (K_j+1 before V_j); both issuers release every slot (the empty
// barriers count two arrivals).  Per step an issuer issues S of key tile j, then O += P V of
// key tile j - 1 (at a unit's first step, the previous unit's last P V goes first).  A
// query block whose second tile starts past the last token skips that tile (its MMAs and
// its softmax).  The split schedule is that of the one-tile form, with the parked running
// state of both tiles (O in bf16, (max, sum) in fp32).

constexpr int kRing = 3;

// 2^x on the FMA and integer pipes (the MUFU unit has 16 results per clock per SM and is
// shared by both softmax warpgroups): x = n + f with n the nearest integer (added to
// 1.5 * 2^23, x's integer part lands in the low mantissa bits) and f in [-0.5, 0.5];
// 2^f from a cubic fitted to minimise the relative error on that interval (Remez
// exchange; max relative error 7.5e-5, below the 2^-9 of the bf16 P it feeds); 2^n added
// to the exponent field.  x is clamped to -125 so the result stays normal.
__device__ __forceinline__ float exp2_poly(float x) {
  x = fmaxf(x, -125.0f);
  const float t = x + 12582912.0f;
  const int n = __float_as_int(t) - 0x4B400000;
  const float f = x - (t - 12582912.0f);
  const float p = fmaf(fmaf(fmaf(0.05517166853f, f, 0.24261112511f), f, 0.69326096773f), f,
                       0.99992805719f);
  return __int_as_float(__float_as_int(p) + static_cast<int>(static_cast<unsigned>(n) << 23));
}

template <int HD>
struct Attn2Cfg {
  static constexpr int kNBox = HD / 64;
  static constexpr uint32_t kQBytes = kNBox * kBox;   // one 128-row tile
  static constexpr uint32_t kKVBytes = kNBox * kBox;
  static constexpr uint32_t kPBytes = 2 * kBox;
  static constexpr size_t kSmem = 1024 + 2 * size_t(kQBytes) + 2 * size_t(kPBytes) +
                                  size_t(kRing) * kKVBytes + 512;
  static_assert(kSmem <= 232448, "two-tile attention shared memory above 227 KB");
};

struct Attn2Params {
  int n, d, n_kv, n_qb;  // tokens, n_heads * head_dim, key tiles, 256-query blocks per head
  long long steps;       // units * n_kv
  long long work;        // the steps weighted by their cost (see work_to_step)
  int half_last;         // 1: the last block of each head has one query tile
  int weighted;          // CTA ranges cut by work instead of steps
  float scale_log2;
  bf16* out;
  uint4* part_o;         // [gridDim.x][2 tiles][head_dim / 8][128] uint4 (8 bf16)
  float2* part_ml;       // [gridDim.x][2 tiles][128]
  unsigned long long* flags;  // [gridDim.x][2 tiles][4]
  unsigned long long seq;
  uint32_t* err;
};

// Relative cost of a key-tile step of a block with two query tiles and of one whose second
// tile is empty (the last block of each head when n % 256 is in (0, 128]): the second runs
// one softmax warp per SMSP instead of two, which takes ~63% of the time, not half
// (measured on B200: CTAs holding such a block finished 30% before the others).
constexpr long long kWorkFull = 8, kWorkHalf = 5;

// The first step (u * n_kv + j) whose work starts at or after work position P.
__host__ __device__ inline long long work_to_step(const Attn2Params& p, long long P) {
  const long long nkv = p.n_kv, h1 = p.half_last;
  const long long per_head = (kWorkFull * (p.n_qb - h1) + kWorkHalf * h1) * nkv;
  const long long head = P / per_head;
  const long long r = P - head * per_head;
  long long qb = r / (kWorkFull * nkv);
  if (qb > p.n_qb - 1) qb = p.n_qb - 1;
  const long long wu = (h1 && qb == p.n_qb - 1) ? kWorkHalf : kWorkFull;
  const long long j = (r - qb * kWorkFull * nkv + wu - 1) / wu;
  return (head * p.n_qb + qb) * nkv + j;
}

// This CTA's steps.  Cut by work where every range still holds at least n_kv steps (a unit
// is then cut at most once, between two neighbouring CTAs), else by steps.
__device__ __forceinline__ Range cta_range2(const Attn2Params& p) {
  Range r;
  const long long b = blockIdx.x, g = gridDim.x;
  if (p.weighted) {
    r.begin = work_to_step(p, p.work * b / g);
    r.end = work_to_step(p, p.work * (b + 1) / g);
  } else {
    r.begin = p.steps * b / g;
    r.end = p.steps * (b + 1) / g;
  }
  r.u_first = static_cast<int>(r.begin / p.n_kv);
  r.u_last = static_cast<int>((r.end - 1) / p.n_kv);
  return r;
}

__device__ __forceinline__ void segment2(const Attn2Params& p, const Range& r, int k, int& unit,
                                         int& j0, int& j1) {
  unit = r.u_last - k;
  const long long base = static_cast<long long>(unit) * p.n_kv;
  j0 = static_cast<int>(r.begin > base ? r.begin - base : 0ll);
  j1 = static_cast<int>(r.end - base < p.n_kv ? r.end - base : static_cast<long long>(p.n_kv));
}

// Whether the unit's second query tile holds any token.
__device__ __forceinline__ bool tile1_valid(const Attn2Params& p, int unit) {
  return (unit % p.n_qb) * 256 + 128 < p.n;
}

// POLY: every fourth exponential of a score row on the FMA pipe (exp2_poly).
template <int HD, bool POLY>
__global__ void __launch_bounds__(384, 1)
    k_attention_tc2(const __grid_constant__ CUtensorMap tm, const Attn2Params p) {
  using Cfg = Attn2Cfg<HD>;
  constexpr uint32_t IDESC_S = idesc_bf16(128, 128, false);
  constexpr uint32_t IDESC_PV = idesc_bf16(128, HD, true);
  constexpr uint32_t kTmemCols = 512;
  constexpr uint32_t kOCol = 256;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;                          // 2 tiles
  uint8_t* sP = sQ + 2 * Cfg::kQBytes;         // 2 tiles
  uint8_t* sKV = sP + 2 * Cfg::kPBytes;        // kRing slots
  uint64_t* bars = reinterpret_cast<uint64_t*>(sKV + kRing * Cfg::kKVBytes);
  uint64_t* q_full = bars + 0;
  uint64_t* q_empty = bars + 1;
  uint64_t* kv_full = bars + 2;   // [kRing]
  uint64_t* kv_empty = bars + 5;  // [kRing]
  uint64_t* s_full = bars + 8;    // [2 tiles]
  uint64_t* s_free = bars + 10;   // [2]
  uint64_t* p_full = bars + 12;   // [2]
  uint64_t* p_free = bars + 14;   // [2]
  uint64_t* o_empty = bars + 16;  // [2]
  uint64_t* drain = bars + 18;    // [2 issuers]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 20);
  volatile uint32_t* abort_flag = tmem_slot + 1;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const Range rg = cta_range2(p);
  const int n_seg = rg.u_last - rg.u_first + 1;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 2);
    for (int s = 0; s < kRing; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 2);
    }
    for (int w = 0; w < 2; ++w) {
      mbar_init(&s_full[w], 1);
      mbar_init(&s_free[w], 4);
      mbar_init(&p_full[w], 4);
      mbar_init(&p_free[w], 1);
      mbar_init(&o_empty[w], 4);
    }
    mbar_init(&drain[0], 1);
    mbar_init(&drain[1], 1);
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

  if (warp < 4) {
    if constexpr (POLY) regs_dealloc<104>();
    if (warp == 0 && lane == 0) {
      // ------------------------------------------------------------------ producer
      // Loads in the MMA's consumption order: per step t, K(t) then V(t - 1), except at a
      // unit's first step (not the walk's first), where V(t - 1) goes first; the Q tiles
      // of a unit before its first K.
      bool ok = true;
      int slot = 0;
      uint32_t ring_phase = 0;
      int armed[kRing] = {-1, -1, -1};
      int q_armed = -1;
      const long long total = rg.end - rg.begin;
      int ks = 0, js = 0, js0 = 0, js1 = 0, unit_s = 0;  // step t's segment and key tile
      int kp = 0, jp = 0, jp0 = 0, jp1 = 0, unit_p = 0;  // step t - 1's
      segment2(p, rg, 0, unit_s, js0, js1);
      js = js0;
      segment2(p, rg, 0, unit_p, jp0, jp1);
      jp = jp0;
      auto load = [&](int x, int y) -> bool {
        if (!wait_bar(&kv_empty[slot], ring_phase ^ 1u, abort_flag, p.err, kErrAttnWait))
          return false;
        mbar_arrive_expect_tx(&kv_full[slot], Cfg::kKVBytes);
#pragma unroll
        for (int b = 0; b < Cfg::kNBox; ++b)
          tma_load_2d(sKV + slot * Cfg::kKVBytes + b * kBox, &tm, &kv_full[slot], x + 64 * b, y);
        armed[slot] = static_cast<int>(ring_phase);
        if (++slot == kRing) {
          slot = 0;
          ring_phase ^= 1u;
        }
        return true;
      };
      auto load_k = [&]() -> bool {  // K of step t, and the unit's Q tiles first
        const int head = unit_s / p.n_qb, qb = unit_s % p.n_qb;
        if (js == js0) {
          if (ks > 0 && !wait_bar(q_empty, static_cast<uint32_t>(ks - 1) & 1u, abort_flag, p.err,
                                  kErrAttnWait))
            return false;
          mbar_arrive_expect_tx(q_full, 2 * Cfg::kQBytes);
#pragma unroll
          for (int w = 0; w < 2; ++w)
#pragma unroll
            for (int b = 0; b < Cfg::kNBox; ++b)
              tma_load_2d(sQ + w * Cfg::kQBytes + b * kBox, &tm, q_full, head * HD + 64 * b,
                          qb * 256 + w * 128);
          q_armed = ks & 1;
        }
        if (!load(p.d + head * HD, js * 128)) return false;
        if (++js == js1 && ++ks < n_seg) {
          segment2(p, rg, ks, unit_s, js0, js1);
          js = js0;
        }
        return true;
      };
      auto load_v = [&]() -> bool {  // V of step t - 1
        const int head = unit_p / p.n_qb;
        if (!load(2 * p.d + head * HD, jp * 128)) return false;
        if (++jp == jp1 && ++kp < n_seg) {
          segment2(p, rg, kp, unit_p, jp0, jp1);
          jp = jp0;
        }
        return true;
      };
      for (long long t = 0; t <= total && ok; ++t) {
        const bool first = t >= 1 && t < total && js == js0;
        if (first) ok = load_v() && load_k();
        else ok = (t >= total || load_k()) && (t < 1 || load_v());
      }
      if (!ok) {
        if (q_armed >= 0) drain_wait(q_full, static_cast<uint32_t>(q_armed));
        for (int s = 0; s < kRing; ++s)
          if (armed[s] >= 0) drain_wait(&kv_full[s], static_cast<uint32_t>(armed[s]));
      }
    } else if ((warp == 1 || warp == 2) && lane == 0) {
      // ------------------------------------------------------------------ MMA issuers
      // Warp 1 issues tile 0's products, warp 2 tile 1's (different SMSPs): each walks the
      // same steps and ring slots, so while one thread waits on a barrier the other feeds
      // the tensor pipe, and neither tile's chain waits on the other's.  Both commit every
      // ring slot and the Q buffer (their empty barriers count two arrivals).
      const int w = warp - 1;
      int slot = 0;
      uint32_t ring_phase = 0;
      int cnt = 0;         // S products issued for this tile (P V products run one behind)
      int pvc = 0;         // P V products issued
      int units_done = 0;  // units whose last P V was issued (tile present)
      int ks = 0, js = 0, js0 = 0, js1 = 0, unit_s = 0;
      int kp = 0, jp = 0, jp0 = 0, jp1 = 0, unit_p = 0;
      segment2(p, rg, 0, unit_s, js0, js1);
      js = js0;
      segment2(p, rg, 0, unit_p, jp0, jp1);
      jp = jp0;
      // (pinned here: hoisted above the role split they would stay live through the softmax)
      const uint64_t q_desc = opaque_u64(sdesc_sw128(smem_u32(sQ + w * Cfg::kQBytes), 16, 1024));
      const uint64_t p_desc = opaque_u64(sdesc_sw128(smem_u32(sP + w * Cfg::kPBytes), 16, 1024));
      const uint64_t k_desc0 = opaque_u64(sdesc_sw128(smem_u32(sKV), 16, 1024));
      const uint64_t v_desc0 = opaque_u64(sdesc_sw128(smem_u32(sKV), kBox, 1024));
      const uint32_t s_tmem = tmem + w * 128;
      const uint32_t o_tmem = tmem + kOCol + w * 128;
      auto ring_take = [&](int& s_out) -> bool {
        if (!wait_bar(&kv_full[slot], ring_phase, abort_flag, p.err, kErrAttnWait)) return false;
        s_out = slot;
        if (++slot == kRing) {
          slot = 0;
          ring_phase ^= 1u;
        }
        return true;
      };
      auto issue_s = [&]() -> bool {
        const bool here = w == 0 || tile1_valid(p, unit_s);
        if (js == js0 &&
            !wait_bar(q_full, static_cast<uint32_t>(ks) & 1u, abort_flag, p.err, kErrAttnWait))
          return false;
        int ksl;
        if (!ring_take(ksl)) return false;
        if (here) {
          if (cnt >= 1 && !wait_bar(&s_free[w], static_cast<uint32_t>(cnt - 1) & 1u,
                                    abort_flag, p.err, kErrAttnWait))
            return false;
          tc_fence_after();
          const uint64_t k_desc = k_desc0 + static_cast<uint64_t>(ksl) * (Cfg::kKVBytes >> 4);
          if constexpr (HD == 128)
            umma_f16_x8_kk<kBox / 16>(s_tmem, q_desc, k_desc, IDESC_S, 0u);
          else
            umma_f16_x4_kk(s_tmem, q_desc, k_desc, IDESC_S, 0u);
          tc_commit(&s_full[w]);
          ++cnt;
        }
        tc_commit(&kv_empty[ksl]);
        if (++js == js1) {
          tc_commit(q_empty);
          if (++ks < n_seg) {
            segment2(p, rg, ks, unit_s, js0, js1);
            js = js0;
          }
        }
        return true;
      };
      auto issue_pv = [&]() -> bool {
        const bool here = w == 0 || tile1_valid(p, unit_p);
        const bool first = jp == jp0;
        int vsl;
        if (!ring_take(vsl)) return false;
        if (here) {
          // the tile's previous unit must have read O out before it is overwritten
          if (first && units_done > 0 &&
              !wait_bar(&o_empty[w], static_cast<uint32_t>(units_done - 1) & 1u, abort_flag,
                        p.err, kErrAttnWait))
            return false;
          if (!wait_bar(&p_full[w], static_cast<uint32_t>(pvc) & 1u, abort_flag, p.err,
                        kErrAttnWait))
            return false;
          tc_fence_after();
          umma_f16_x8_kmn<kBox / 16>(
              o_tmem, p_desc, v_desc0 + static_cast<uint64_t>(vsl) * (Cfg::kKVBytes >> 4),
              IDESC_PV, first ? 0u : 1u);
          tc_commit(&p_free[w]);
          ++pvc;
        }
        tc_commit(&kv_empty[vsl]);
        if (++jp == jp1) {
          if (here) ++units_done;
          if (++kp < n_seg) {
            segment2(p, rg, kp, unit_p, jp0, jp1);
            jp = jp0;
          }
        }
        return true;
      };
      const long long total = rg.end - rg.begin;
      for (long long t = 0; t <= total; ++t) {
        const bool pv_first = t >= 1 && t < total && js == js0;
        if (pv_first && !issue_pv()) break;
        if (t < total && !issue_s()) break;
        if (t >= 1 && !pv_first && !issue_pv()) break;
      }
      tc_commit(&drain[w]);
      drain_wait(&drain[w], 0);
    }
  } else {
    if constexpr (POLY) regs_alloc<200>();
    // ------------------------------------------------------------------ softmax (tile w)
    const int w = (warp - 4) >> 2;
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t s_addr = tmem + lane_addr + w * 128;
    const uint32_t o_addr = tmem + lane_addr + kOCol + w * 128;
    const float sl2 = p.scale_log2;
    uint8_t* pbuf = sP + w * Cfg::kPBytes + row * 128;
    bool ok = true;
    int c = 0;  // steps of this tile so far
    for (int k = 0; k < n_seg && ok; ++k) {
      int unit, j0, j1;
      segment2(p, rg, k, unit, j0, j1);
      if (w == 1 && !tile1_valid(p, unit)) continue;
      float m_used = -INFINITY;
      float l = 0.f;
      for (int j = j0; j < j1; ++j, ++c) {
        const uint32_t ph = static_cast<uint32_t>(c) & 1u;
        ok = __all_sync(0xffffffffu, wait_bar(&s_full[w], ph, abort_flag, p.err, kErrAttnWait));
        if (!ok) break;
        tc_fence_after();
        float s[128];
        {
          uint32_t r[128];
          tmem_ld128_sync(s_addr, r);
#pragma unroll
          for (int q = 0; q < 128; ++q) s[q] = __uint_as_float(r[q]);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&s_free[w]);
        if ((j + 1) * 128 > p.n) {
          const int valid = p.n - j * 128;
#pragma unroll
          for (int q = 0; q < 128; ++q)
            if (q >= valid) s[q] = -INFINITY;
        }
        float m8[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          m8[i] = fmaxf(s[i], s[8 + i]);
#pragma unroll
          for (int q = 16; q < 128; q += 16) m8[i] = max3(m8[i], s[q + i], s[q + 8 + i]);
        }
        const float mx = max3(max3(m8[0], m8[1], m8[2]), max3(m8[3], m8[4], m8[5]),
                              fmaxf(m8[6], m8[7]));
        const float mxs = mx * sl2;
        // lazy rescale: the running max moves only when the tile max exceeds it by more
        // than 8; O is rescaled below, once the scores are dead (after P is stored)
        float alpha = 1.0f;
        bool need = false;
        if (j == j0) {
          m_used = mxs;
        } else if (mxs > m_used + 8.0f) {
          need = true;
          alpha = ex2_approx(m_used - mxs);
          m_used = mxs;
        }
        float sum8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int q = 0; q < 128; ++q) {
          const float x = fmaf(s[q], sl2, -m_used);
          const float e = (POLY && (q & 3) == 3) ? exp2_poly(x) : ex2_approx(x);
          sum8[q & 7] += e;
          s[q] = e;
        }
#pragma unroll
        for (int i = 4; i > 0; i >>= 1)
#pragma unroll
          for (int q = 0; q < i; ++q) sum8[q] += sum8[q + i];
        l = fmaf(l, alpha, sum8[0]);
        if (c >= 1) {
          // the tile's P buffer is free, and O complete, once its previous P V has finished
          ok = __all_sync(0xffffffffu, wait_bar(&p_free[w], static_cast<uint32_t>(c - 1) & 1u,
                                                abort_flag, p.err, kErrAttnWait));
          if (!ok) break;
        }
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
        if (__any_sync(0xffffffffu, need)) {
          // O holds every earlier P V product of the unit (the wait above) and the next one
          // is not released yet: scale it to the new running max
          tc_fence_after();
#pragma unroll 1
          for (int cc = 0; cc < HD / 32; ++cc) {
            uint32_t r[32];
            tmem_ld32(o_addr + cc * 32, r);
            tmem_wait_ld(r);
#pragma unroll
            for (int q = 0; q < 32; ++q) r[q] = __float_as_uint(__uint_as_float(r[q]) * alpha);
            tmem_st32(o_addr + cc * 32, r);
          }
          tmem_wait_st();
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[w]);
      }
      if (!ok) break;
      // ---- end of the unit: O holds every P V product once the last one completes
      ok = __all_sync(0xffffffffu, wait_bar(&p_free[w], static_cast<uint32_t>(c - 1) & 1u,
                                            abort_flag, p.err, kErrAttnWait));
      if (!ok) break;
      tc_fence_after();
      const int head = unit / p.n_qb, qb = unit % p.n_qb;
      const int part = static_cast<int>(blockIdx.x) * 2 + w;
      if (j1 < p.n_kv) {
        // lower part of a split unit: park the running state for the owner (next CTA)
        uint4* po = p.part_o + size_t(part) * (HD / 8) * 128 + row;
#pragma unroll 1
        for (int cc = 0; cc < HD / 32; ++cc) {
          uint32_t r[32];
          tmem_ld32(o_addr + cc * 32, r);
          tmem_wait_ld(r);
#pragma unroll
          for (int i = 0; i < 4; ++i)
            __stcg(po + size_t(cc * 4 + i) * 128,
                   make_uint4(pack_bf16x2(__uint_as_float(r[8 * i]), __uint_as_float(r[8 * i + 1])),
                              pack_bf16x2(__uint_as_float(r[8 * i + 2]), __uint_as_float(r[8 * i + 3])),
                              pack_bf16x2(__uint_as_float(r[8 * i + 4]), __uint_as_float(r[8 * i + 5])),
                              pack_bf16x2(__uint_as_float(r[8 * i + 6]), __uint_as_float(r[8 * i + 7]))));
        }
        __stcg(p.part_ml + size_t(part) * 128 + row, make_float2(m_used, l));
        __threadfence();
        __syncwarp();
        if (lane == 0) st_release_u64(p.flags + part * 4 + quarter, p.seq);
      } else {
        float wa = 0.f, wb = 1.f;
        const uint4* po = nullptr;
        if (j0 > 0) {
          const int src = part - 2;  // the same tile of the previous CTA
          ok = __all_sync(0xffffffffu,
                          wait_flag(p.flags + src * 4 + quarter, p.seq, abort_flag, p.err));
          if (!ok) break;
          const float2 ml = __ldcg(p.part_ml + size_t(src) * 128 + row);
          const float m = fmaxf(ml.x, m_used);
          wa = ex2_approx(ml.x - m);
          wb = ex2_approx(m_used - m);
          l = ml.y * wa + l * wb;
          po = p.part_o + size_t(src) * (HD / 8) * 128 + row;
        }
        const float inv_l = 1.0f / l;
        wa *= inv_l;
        wb *= inv_l;
        const int grow = qb * 256 + w * 128 + row;
#pragma unroll
        for (int cc = 0; cc < HD / 32; ++cc) {
          uint32_t r[32];
          tmem_ld32(o_addr + cc * 32, r);
          tmem_wait_ld(r);
          float o[32];
#pragma unroll
          for (int q = 0; q < 32; ++q) o[q] = __uint_as_float(r[q]) * wb;
          if (po != nullptr) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const uint4 a = __ldcg(po + size_t(cc * 4 + i) * 128);
              const float2 a0 = unpack_bf16x2(a.x), a1 = unpack_bf16x2(a.y);
              const float2 a2 = unpack_bf16x2(a.z), a3 = unpack_bf16x2(a.w);
              o[8 * i + 0] = fmaf(a0.x, wa, o[8 * i + 0]);
              o[8 * i + 1] = fmaf(a0.y, wa, o[8 * i + 1]);
              o[8 * i + 2] = fmaf(a1.x, wa, o[8 * i + 2]);
              o[8 * i + 3] = fmaf(a1.y, wa, o[8 * i + 3]);
              o[8 * i + 4] = fmaf(a2.x, wa, o[8 * i + 4]);
              o[8 * i + 5] = fmaf(a2.y, wa, o[8 * i + 5]);
              o[8 * i + 6] = fmaf(a3.x, wa, o[8 * i + 6]);
              o[8 * i + 7] = fmaf(a3.y, wa, o[8 * i + 7]);
            }
          }
          if (grow < p.n) {
            uint4* dst =
                reinterpret_cast<uint4*>(p.out + size_t(grow) * p.d + head * HD + cc * 32);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              uint4 u;
              u.x = pack_bf16x2(o[8 * i + 0], o[8 * i + 1]);
              u.y = pack_bf16x2(o[8 * i + 2], o[8 * i + 3]);
              u.z = pack_bf16x2(o[8 * i + 4], o[8 * i + 5]);
              u.w = pack_bf16x2(o[8 * i + 6], o[8 * i + 7]);
              dst[i] = u;
            }
          }
        }
        if (po != nullptr) {
          __syncwarp();
          if (lane == 0) p.flags[(part - 2) * 4 + quarter] = 0ull;
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&o_empty[w]);
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

template <int HD, bool POLY>
int launch_hd2(const DevCtx& ctx, const bf16* qkv, int n, int heads, bf16* out, void* scratch,
               size_t scratch_bytes, cudaStream_t stream) {
  using Cfg = Attn2Cfg<HD>;
  const int d = heads * HD;
  CUtensorMap tm;
  if (!make_tmap_2d(&tm, qkv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, uint64_t(n), uint64_t(3 * d),
                    uint64_t(3 * d) * 2, 128, 64))
    return set_error(-3, "attention: cuTensorMapEncodeTiled failed (n=%d d=%d)", n, d);
  auto kernel = k_attention_tc2<HD, POLY>;
  static std::atomic<uint32_t> attr_done{0};
  const uint32_t bit = 1u << (ctx.device & 31);
  if (!(attr_done.load() & bit)) {
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(Cfg::kSmem));
    if (e != cudaSuccess)
      return set_error(-3, "attention: cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    attr_done.fetch_or(bit);
  }
  Attn2Params p = {};
  p.n = n;
  p.d = d;
  p.n_kv = (n + 127) / 128;
  p.n_qb = (n + 255) / 256;
  const long long units = static_cast<long long>(p.n_qb) * heads;
  p.steps = units * p.n_kv;
  p.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(double(HD)));
  p.out = out;
  p.err = ctx.err_flag;
  long long grid = units;
  if (scratch != nullptr && scratch_bytes >= kScratchBytes) {
    static_assert(size_t(kMaxSkCtas) * 2 * 128 * (128 * 2 + 8) <= kSkFlagsOffset,
                  "two-tile attention partial states must fit the slot area");
    static_assert(size_t(kMaxSkCtas) * 2 * 4 * 8 <= kScratchBytes - kSkFlagsOffset,
                  "two-tile attention flags must fit the flag area");
    grid = std::min<long long>(units, std::min(ctx.num_sms, kMaxSkCtas));
    uint8_t* base = static_cast<uint8_t*>(scratch);
    p.part_o = reinterpret_cast<uint4*>(base);
    p.part_ml = reinterpret_cast<float2*>(base + size_t(kMaxSkCtas) * 2 * 128 * HD * 2);
    p.flags = reinterpret_cast<unsigned long long*>(base + kSkFlagsOffset);
    p.seq = next_scratch_seq();
  }
  if (grid > 0x7fffffffll) return set_error(-1, "attention: %lld units", units);
  p.half_last = (n % 256 != 0 && n % 256 <= 128) ? 1 : 0;
  p.work = (kWorkFull * (p.n_qb - p.half_last) + kWorkHalf * p.half_last) * heads * p.n_kv;
  p.weighted = p.half_last && p.work >= kWorkFull * p.n_kv * grid;
  kernel<<<static_cast<unsigned>(grid), 384, Cfg::kSmem, stream>>>(tm, p);
  return check_launch("attention");
}

template <int HD>
int launch_hd(const DevCtx& ctx, const bf16* qkv, int n, int heads, bf16* out, void* scratch,
              size_t scratch_bytes, cudaStream_t stream) {
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
  AttnParams p = {};
  p.n = n;
  p.d = d;
  p.n_kv = (n + 127) / 128;
  p.n_qt = p.n_kv;
  const long long units = static_cast<long long>(p.n_qt) * heads;
  p.steps = units * p.n_kv;
  p.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(double(HD)));
  p.out = out;
  p.err = ctx.err_flag;
  // Split schedule: one CTA per SM, never more CTAs than units, so a range is at least
  // n_kv steps long: a unit is cut at most once and each CTA parks at most one partial
  // state.  Without scratch: one CTA per unit.
  long long grid = units;
  if (scratch != nullptr && scratch_bytes >= kScratchBytes) {
    static_assert(size_t(kMaxSkCtas) * 128 * (128 + 2) * 4 <= kSkFlagsOffset,
                  "attention partial states must fit the slot area");
    grid = std::min<long long>(units, std::min(ctx.num_sms, kMaxSkCtas));
    uint8_t* base = static_cast<uint8_t*>(scratch);
    p.part_o = reinterpret_cast<float4*>(base);
    p.part_ml = reinterpret_cast<float2*>(base + size_t(kMaxSkCtas) * 128 * HD * 4);
    p.flags = reinterpret_cast<unsigned long long*>(base + kAttnFlagsOffset);
    p.seq = next_scratch_seq();
  }
  if (grid > 0x7fffffffll) return set_error(-1, "attention: %lld units", units);
  kernel<<<static_cast<unsigned>(grid), 192, Cfg::kSmem, stream>>>(tm, p);
  return check_launch("attention");
}

}  // namespace

std::atomic<int> g_attn_variant{0};

int set_attention_variant(int v) {
  if (v < 0 || v > 3) return -1;
  g_attn_variant.store(v);
  return 0;
}

int launch_attention(const DevCtx& ctx, const bf16* qkv, int n_tokens, int n_heads,
                     int head_dim, bf16* out, void* scratch, size_t scratch_bytes,
                     cudaStream_t stream) {
  if (n_tokens <= 0) return 0;
  // two query tiles per CTA unless the one-tile form is asked for
  const int v = g_attn_variant.load(std::memory_order_relaxed);
  const bool poly = v == 3;
  if (head_dim == 128) {
    if (v == 1) return launch_hd<128>(ctx, qkv, n_tokens, n_heads, out, scratch, scratch_bytes, stream);
    return poly ? launch_hd2<128, true>(ctx, qkv, n_tokens, n_heads, out, scratch, scratch_bytes, stream)
                : launch_hd2<128, false>(ctx, qkv, n_tokens, n_heads, out, scratch, scratch_bytes, stream);
  }
  if (head_dim == 64) {
    if (v == 1) return launch_hd<64>(ctx, qkv, n_tokens, n_heads, out, scratch, scratch_bytes, stream);
    return poly ? launch_hd2<64, true>(ctx, qkv, n_tokens, n_heads, out, scratch, scratch_bytes, stream)
                : launch_hd2<64, false>(ctx, qkv, n_tokens, n_heads, out, scratch, scratch_bytes, stream);
  }
  return set_error(-1, "attention: head_dim %d unsupported (64 or 128)", head_dim);
}

}  // namespace h3b
