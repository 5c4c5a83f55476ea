// Causal grouped-query flash attention on tcgen05 (sm_100a).
//
// O[i, h, :] = softmax_j( Q[i, h, :] . K[j, g, :] / sqrt(hd) ) V[j, g, :],
// g = h / (hq / hkv), over keys j visible to query i:
//   kstart(i) <= j <= qpos(i),  j < T_kv,
// kstart(i) = kstart[i] when given (varlen batches: the first key of row i's
// own sequence, so attention is block-diagonal causal), else 0.
// qpos(i) = qpos[i] when a position list is given (halt mode: compacted
// queries at their original positions attend over all T keys), else i
// (dense and prune mode: causal over the rows' own order).  This is the
// attention module whose output, after o_proj, is the update U that the DASH
// blog post (§2.1) scores; the T x T matrix is never materialised.
//
// One CTA = two 128-row query tiles (Q0, Q1) of one query head, sharing every
// K/V tile.  Warp roles (320 threads):
//   warp 0      TMA producer: Q0/Q1 once, then load groups (2-stage ring):
//               group 0 = K_0, group g = V_(g-1) and K_g, the operands the
//               MMAs of one key step consume
//   warp 1      TMEM allocator and MMA issue, in the order
//                 S0_0 S1_0 | PV0_0 S0_1 PV1_0 S1_1 | PV0_1 S0_2 ...
//               so each softmax warpgroup overlaps two MMAs of the other tile.
//               The warp runs the issue loop converged; elect.sync picks the
//               lane that issues each MMA and commit.
//   warps 2..5  softmax of Q0, warps 6..9 softmax of Q1: one query row per
//               thread (TMEM lane = row); S_j is read from TMEM, the running
//               max / sum kept in registers, O rescaled in TMEM only when the
//               max grows by more than 2^8 (exact: l and O share the stale
//               reference), and P_j written back to TMEM as packed 16-bit
//               pairs (the model's format, DT) over the upper half of S_j, where the P*V MMA reads it as its
//               A operand.
// TMEM columns: S0/P0 [0,128) S1/P1 [128,256) O0 [256,384) O1 [384,512).
// MMAs issued by one thread complete in order, so the commit that signals
// S_i(j+1) also proves that P_i(j) V_j is finished: the softmax may then
// overwrite P_i and rescale O_i without another barrier.
// A tcgen05.mma holds its issuing warp for about its execution time, so the
// warp's other work (barrier waits, commits, fences) idles the tensor pipe:
// it waits once per load group and once per P, fences only before P*V (the
// softmax threads' TMEM writes), and commits three times per key step.
// Issuing from the converged warp measured faster than from a lone lane-0
// thread in a divergent branch.
#pragma once

#include "common.cuh"

namespace dash {
namespace attn {

constexpr int BQ = 128;   // query rows per tile (two tiles per CTA)
constexpr int BKV = 128;  // keys per tile
constexpr int kStages = 2;  // load groups in flight
constexpr int kThreads = 320;
constexpr float kRescaleThreshold = 8.0f;  // log2 units
// One exponential in every 2 * kEmuPeriod columns is computed on the FMA pipe
// (ex2_fma); the rest use MUFU, whose 16 per clock per SM match the tensor
// pipe's rate for this tile shape.  0 disables the FMA path.
#ifndef DASH_ATTN_EMU_PERIOD
#define DASH_ATTN_EMU_PERIOD 8
#endif
constexpr int kEmuPeriod = DASH_ATTN_EMU_PERIOD;

struct Params {
  s16* out;  // [M, hq*hd]
  int64_t ldo;
  const int32_t* qpos;    // [M] or NULL
  const int32_t* kstart;  // [M] or NULL (non-decreasing)
  int M, T_kv, hq, hkv, hd, n_qblocks;
  float scale_log2;  // log2(e) / sqrt(hd)
};

template <int HD>
struct Cfg {
  static constexpr int kPanels = HD / 64;  // 128-byte swizzle panels per row
  static constexpr int kTileBytes = 128 * HD * 2;
  static constexpr int kOffQ = 0;  // Q0, Q1
  static constexpr int kOffK = kOffQ + 2 * kTileBytes;  // K of group g in stage g % 2
  static constexpr int kOffV = kOffK + kStages * kTileBytes;
  static constexpr int kOffBar = kOffV + kStages * kTileBytes;
  // q_full, g_full[2], g_empty[2], s_full[2], p_full[2], o_done[2] (last P*V of a tile), drain
  static constexpr int kNumBars = 1 + 2 * kStages + 2 + 2 + 2 + 1;
  static constexpr int kSmemBytes = kOffBar + 8 * kNumBars + 16 + 1024;
  static constexpr uint32_t kTmemCols = 512;
};

// max of three fp32 values in one instruction (sm_100)
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// 2^x on the FMA / integer pipes, relieving the MUFU unit that the other half
// of the softmax exponentials use.  Range split: x = j + f with j = round(x)
// (the 1.5 * 2^23 addition rounds to an integer held in the low mantissa
// bits) and f in [-0.5, 0.5]; 2^f by a cubic whose coefficients were fitted
// here to minimise the relative error on [-0.5, 0.5] (iteratively reweighted
// least squares on Chebyshev nodes; max relative error 7.5e-5 in fp32, far
// below the 16-bit P's rounding); 2^j is added to the exponent field.  Inputs are
// clamped at -125 so the exponent add stays within normal numbers (j <= -127
// would wrap into the sign bit); fully masked scores give ~2e-38 instead of 0,
// negligible next to any stored weight.
__device__ __forceinline__ float ex2_fma(float x) {
  constexpr float kRound = 12582912.0f;  // 1.5 * 2^23
  x = fmaxf(x, -125.0f);
  const float t = x + kRound;
  const float f = x - (t - kRound);
  const float q = fmaf(fmaf(fmaf(0.0551716685f, f, 0.2426111251f), f, 0.6932609677f), f, 0.9999280572f);
  return __int_as_float(__float_as_int(q) + (__float_as_int(t) << 23));
}

__device__ __forceinline__ void umma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                             uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// P*V with A = P from TMEM, issued by one elected lane of a converged warp.
__device__ __forceinline__ void umma_ts_elect(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                              uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t.reg .b32 r;\n\t"
      "elect.sync r|e, 0xffffffff;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
template <int HD, int DT>
__global__ void __launch_bounds__(kThreads, 1)
    attn_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
                const __grid_constant__ CUtensorMap tmap_v, const Params p) {
  using C = Cfg<HD>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  const uint32_t bar_q = smem_u32(bars);
  const uint32_t bar_gfull = smem_u32(bars + 1);
  const uint32_t bar_gempty = smem_u32(bars + 1 + kStages);
  const uint32_t bar_sfull = smem_u32(bars + 1 + 2 * kStages);
  const uint32_t bar_pfull = bar_sfull + 16;
  const uint32_t bar_odone = bar_sfull + 32;
  const uint32_t bar_drain = bar_sfull + 48;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::kNumBars);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int head = blockIdx.x % p.hq;
  const int qb = p.n_qblocks - 1 - static_cast<int>(blockIdx.x / p.hq);  // heavy blocks first
  const int kvh = head / (p.hq / p.hkv);
  const int q0 = qb * 2 * BQ;
  const bool has1 = q0 + BQ < p.M;
  // Key tiles [jb_t, n_t) each query tile needs (positions and key starts ascend
  // within the block).
  int n_t[2], jb_t[2], pos_first[2], ks_last[2];
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    const int first = min(q0 + t * BQ, p.M - 1);
    const int last = min(q0 + t * BQ + BQ - 1, p.M - 1);
    pos_first[t] = p.qpos ? p.qpos[first] : first;
    const int pos_last = p.qpos ? p.qpos[last] : last;
    const int lim = min(pos_last + 1, p.T_kv);
    n_t[t] = (lim + BKV - 1) / BKV;
    jb_t[t] = p.kstart ? p.kstart[first] / BKV : 0;
    ks_last[t] = p.kstart ? p.kstart[last] : 0;
  }
  if (!has1) {
    n_t[1] = 0;
    jb_t[1] = jb_t[0];
  }
  const int j0 = jb_t[0];  // first key tile of the block
  const int n_kv = max(n_t[0], n_t[1]);

  if (threadIdx.x == 0) {
    mbar_init(bar_q, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar_gfull + 8 * s, 1);
      mbar_init(bar_gempty + 8 * s, 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(bar_sfull + 8 * t, 1);
      mbar_init(bar_pfull + 8 * t, 128);
      mbar_init(bar_odone + 8 * t, 1);
    }
    mbar_init(bar_drain, 1);
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmap_q);
    prefetch_tmap(&tmap_k);
    prefetch_tmap(&tmap_v);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer
      const uint32_t sq = smem_u32(smem + C::kOffQ);
      mbar_arrive_expect_tx(bar_q, (has1 ? 2 : 1) * C::kTileBytes);
      for (int t = 0; t < (has1 ? 2 : 1); ++t)
        for (int pn = 0; pn < C::kPanels; ++pn)
          tma_load_2d(&tmap_q, sq + t * C::kTileBytes + pn * (BQ * 128), bar_q, head * HD + pn * 64, q0 + t * BQ);
      uint32_t armed = 0, apar = 0;
      for (int g = 0; g <= n_kv - j0; ++g) {
        const bool has_k = j0 + g < n_kv, has_v = g >= 1;
        const int st = g % kStages;
        const uint32_t ph = (g / kStages) & 1;
        if (!mbar_wait(bar_gempty + 8 * st, ph ^ 1u)) break;
        const uint32_t fb = bar_gfull + 8 * st;
        mbar_arrive_expect_tx(fb, ((has_k ? 1 : 0) + (has_v ? 1 : 0)) * C::kTileBytes);
        const uint32_t sk = smem_u32(smem + C::kOffK + st * C::kTileBytes);
        const uint32_t sv = smem_u32(smem + C::kOffV + st * C::kTileBytes);
        for (int pn = 0; pn < C::kPanels; ++pn) {
          if (has_k) tma_load_2d(&tmap_k, sk + pn * (BKV * 128), fb, kvh * HD + pn * 64, (j0 + g) * BKV);
          if (has_v) tma_load_2d(&tmap_v, sv + pn * (BKV * 128), fb, kvh * HD + pn * 64, (j0 + g - 1) * BKV);
        }
        armed |= 1u << st;
        apar = (apar & ~(1u << st)) | (ph << st);
      }
      mbar_wait_drain(bar_q, 0);
      for (int st = 0; st < kStages; ++st)
        if ((armed >> st) & 1u) mbar_wait_drain(bar_gfull + 8 * st, (apar >> st) & 1u);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA
    {  // converged warp; elected lanes issue
      const uint32_t idesc_s = umma_idesc<DT>(BQ, BKV, false, false);
      const uint32_t idesc_o = umma_idesc<DT>(BQ, HD, false, true);
      // Descriptors are built once and advanced by adding (byte offset >> 4)
      // to the start-address field.
      const uint64_t qdesc0 = umma_desc_sw128(smem_u32(smem + C::kOffQ), 16, 1024);
      const uint64_t kdesc0 = umma_desc_sw128(smem_u32(smem + C::kOffK), 16, 1024);
      const uint64_t vdesc0 = umma_desc_sw128(smem_u32(smem + C::kOffV), BKV * 128, 1024);
      // a wait with an inline first try (the barrier is usually ready)
      // lane 0's outcome, broadcast: every decision stays warp-uniform, so
      // elect.sync always sees the whole warp
      auto wait = [](uint32_t bar, uint32_t par) { return warp_wait(bar, par); };
      auto issue_s = [&](int t, int st) {  // S_t = Q_t K^T, K in stage st
        const uint64_t kd = kdesc0 + static_cast<uint64_t>((st * C::kTileBytes) >> 4);
        const uint64_t qd = qdesc0 + static_cast<uint64_t>((t * C::kTileBytes) >> 4);
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          constexpr int kPanelStep = (BQ * 128) >> 4;
          const int off = (kk >> 2) * kPanelStep + (kk & 3) * 2;  // (panel, 32-byte column step) >> 4
          umma_ss_elect(tmem_base + t * BKV, qd + off, kd + off, idesc_s, kk != 0 ? 1u : 0u);
        }
        umma_commit_elect(bar_sfull + 8 * t);
      };
      // group 0 holds K_j0 only
      bool ok = wait(bar_q, 0) && wait(bar_gfull, 0);
      if (ok) {
        for (int t = 0; t < 2; ++t)
          if (jb_t[t] == j0 && j0 < n_t[t]) issue_s(t, 0);
        umma_commit_elect(bar_gempty);
      }
      for (int j = j0; ok && j < n_kv; ++j) {
        const int g = j - j0 + 1, st = g % kStages;  // group g: V_j and K_(j+1)
        if (!wait(bar_gfull + 8 * st, (g / kStages) & 1)) {
          ok = false;
          break;
        }
        for (int t = 0; t < 2; ++t) {
          if (jb_t[t] <= j && j < n_t[t]) {  // O_t += P_t V_j  (P from TMEM)
            if (!wait(bar_pfull + 8 * t, (j - jb_t[t]) & 1)) {
              ok = false;
              break;
            }
            tc_fence_after();  // P_t and any O_t rescale by the softmax threads precede P*V
            const uint64_t vd = vdesc0 + static_cast<uint64_t>((st * C::kTileBytes) >> 4);
            const uint32_t pa = tmem_base + t * BKV + BKV / 2;
            const uint32_t acc0 = j != jb_t[t] ? 1u : 0u;
#pragma unroll
            for (int kk = 0; kk < BKV / 16; ++kk)  // 16 keys = 16 rows of 128 bytes
              umma_ts_elect(tmem_base + 256 + t * 128, pa + kk * 8, vd + kk * ((16 * 128) >> 4), idesc_o,
                           kk != 0 ? 1u : acc0);
            if (j == n_t[t] - 1) umma_commit_elect(bar_odone + 8 * t);
          }
          if (jb_t[t] <= j + 1 && j + 1 < n_t[t]) issue_s(t, st);
        }
        if (!ok) break;
        umma_commit_elect(bar_gempty + 8 * st);
      }
      umma_commit_elect(bar_drain);
      mbar_wait_drain(bar_drain, 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax
    const int t = (warp - 2) >> 2;   // query tile of this warpgroup
    const int wq = warp & 3;         // TMEM lane quarter
    const int r = wq * 32 + lane;    // row within the tile == TMEM lane
    const int m = q0 + t * BQ + r;
    const int mrow = min(m, p.M - 1);
    const int row_pos = p.qpos ? p.qpos[mrow] : m;
    const int row_ks = p.kstart ? p.kstart[mrow] : 0;
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t s_addr = tmem_base + lane_off + t * BKV;
    const uint32_t o_addr = tmem_base + lane_off + 256 + t * 128;
    const int n = n_t[t], jb = jb_t[t];
    const float sc = p.scale_log2;
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int j = jb; j < n; ++j) {
      // warp-uniform outcomes keep the warp converged for __any_sync and tcgen05.ld
      if (!__all_sync(0xffffffffu, mbar_wait(bar_sfull + 8 * t, (j - jb) & 1))) {
        ok = false;
        break;
      }
      tc_fence_after();
      // S in two halves: the max of the first runs while the second loads
      uint32_t u[BKV];
      tmem_ld32(s_addr + 0, *reinterpret_cast<uint32_t(*)[32]>(u + 0));
      tmem_ld32(s_addr + 32, *reinterpret_cast<uint32_t(*)[32]>(u + 32));
      tmem_ld_wait();
      tmem_ld32(s_addr + 64, *reinterpret_cast<uint32_t(*)[32]>(u + 64));
      tmem_ld32(s_addr + 96, *reinterpret_cast<uint32_t(*)[32]>(u + 96));
      float* s = reinterpret_cast<float*>(u);
      const int kv0 = j * BKV;
      const bool edge = kv0 + BKV - 1 > pos_first[t] || kv0 + BKV > p.T_kv || kv0 < ks_last[t];
      const int hi = min(row_pos, p.T_kv - 1) - kv0;  // visible columns of this row: [lo, hi]
      const int lo = row_ks - kv0;
      float mx[8];
      if (edge) {
#pragma unroll
        for (int c = 0; c < BKV / 2; ++c) s[c] = (c >= lo && c <= hi) ? s[c] : -INFINITY;
      }
#pragma unroll
      for (int k = 0; k < 8; ++k) mx[k] = fmax3(s[k], s[8 + k], s[16 + k]);
#pragma unroll
      for (int c = 24; c + 16 <= BKV / 2; c += 16)
#pragma unroll
        for (int k = 0; k < 8; ++k) mx[k] = fmax3(mx[k], s[c + k], s[c + 8 + k]);
#pragma unroll
      for (int k = 0; k < 8; ++k) mx[k] = fmaxf(mx[k], s[BKV / 2 - 8 + k]);
      tmem_ld_wait();
      if (edge) {
#pragma unroll
        for (int c = BKV / 2; c < BKV; ++c) s[c] = (c >= lo && c <= hi) ? s[c] : -INFINITY;
      }
#pragma unroll
      for (int c = BKV / 2; c < BKV; c += 16)
#pragma unroll
        for (int k = 0; k < 8; ++k) mx[k] = fmax3(mx[k], s[c + k], s[c + 8 + k]);
      const float rmax = fmax3(fmax3(mx[0], mx[1], mx[2]), fmax3(mx[3], mx[4], mx[5]), fmaxf(mx[6], mx[7])) * sc;
      // Each row moves its own reference (rarely); the warp-wide vote on
      // whether O needs rescaling waits until after the exponentials.
      float alpha = 1.f;
      if (j == jb) {
        m_run = rmax;  // -inf if this row's keys start in a later tile
      } else if (rmax > m_run + kRescaleThreshold) {
        alpha = ex2_approx(m_run - rmax);  // 0 for a row fully masked so far (m_run = -inf)
        m_run = rmax;
      }
      const float neg = m_run == -INFINITY ? 0.f : -m_run;  // fully masked so far: p = 0
      // row sum of the exponentials: even and odd columns in packed fp32x2 adds
      float2 ls[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) ls[k] = make_float2(0.f, 0.f);
      float lsum = 0.f;
#pragma unroll
      for (int half = 0; half < 2; ++half) {  // 64 columns at a time keeps pk small
        uint32_t pk[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int c = half * 64 + 2 * i;
          // s * scale - max for both columns in one packed fp32x2 FMA (two fmaf)
          const float2 x = __ffma2_rn(make_float2(s[c], s[c + 1]), make_float2(sc, sc), make_float2(neg, neg));
          const float e0 = ex2_approx(x.x);  // MUFU
          const float e1 = (kEmuPeriod > 0 && (i % (kEmuPeriod > 0 ? kEmuPeriod : 1)) == kEmuPeriod - 1)
                               ? ex2_fma(x.y)  // FMA pipe
                               : ex2_approx(x.y);
          ls[i & 3] = __fadd2_rn(ls[i & 3], make_float2(e0, e1));
          pk[i] = Num<DT>::pack(e0, e1);
        }
        tmem_st32(s_addr + BKV / 2 + 32 * half, pk);
      }
      lsum = ((ls[0].x + ls[0].y) + (ls[1].x + ls[1].y)) + ((ls[2].x + ls[2].y) + (ls[3].x + ls[3].y));
      l_run = fmaf(l_run, alpha, lsum);
      if (__any_sync(0xffffffffu, alpha != 1.f)) {
        // P_t(j-1) V_(j-1) is complete (in-order MMAs): O_t may be rescaled.
#pragma unroll 1
        for (int c = 0; c < HD; c += 32) {
          uint32_t o[32];
          tmem_ld32(o_addr + c, o);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
          tmem_st32(o_addr + c, o);
        }
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar_pfull + 8 * t);
    }
    // o_done[t] completes once, after the last P*V of this tile
    if (__all_sync(0xffffffffu, ok && n > jb && mbar_wait(bar_odone + 8 * t, 0))) {
      tc_fence_after();
      const float inv_l = 1.f / l_run;
      s16* dst = p.out + static_cast<int64_t>(mrow) * p.ldo + head * HD;
#pragma unroll 1
      for (int c = 0; c < HD; c += 32) {
        uint32_t o[32];
        tmem_ld32(o_addr + c, o);
        tmem_ld_wait();
        if (m < p.M) {
          uint4* d4 = reinterpret_cast<uint4*>(dst + c);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            uint4 w;
            w.x = Num<DT>::pack(__uint_as_float(o[8 * i + 0]) * inv_l, __uint_as_float(o[8 * i + 1]) * inv_l);
            w.y = Num<DT>::pack(__uint_as_float(o[8 * i + 2]) * inv_l, __uint_as_float(o[8 * i + 3]) * inv_l);
            w.z = Num<DT>::pack(__uint_as_float(o[8 * i + 4]) * inv_l, __uint_as_float(o[8 * i + 5]) * inv_l);
            w.w = Num<DT>::pack(__uint_as_float(o[8 * i + 6]) * inv_l, __uint_as_float(o[8 * i + 7]) * inv_l);
            d4[i] = w;
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::kTmemCols);
  }
}

}  // namespace attn
}  // namespace dash
