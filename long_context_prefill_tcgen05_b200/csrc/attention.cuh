// Causal grouped-query flash attention on tcgen05 (sm_100a).
//
// O[i, h, :] = softmax_j( Q[i, h, :] . K[j, g, :] / sqrt(hd) ) V[j, g, :],
// g = h / (hq / hkv), over keys j visible to query i:  j <= qpos(i), j < T_kv.
// qpos(i) = qpos[i] when a position list is given (halt mode: compacted
// queries at their original positions attend over all T keys), else i
// (dense and prune mode: causal over the rows' own order).  This is the
// attention module whose output, after o_proj, is the update U that the DASH
// blog post (§2.1) scores; it never materialises the T x T matrix.
//
// One CTA = one 128-row query tile of one query head.  Warp roles:
//   warp 0      TMA producer: Q once, then K_j / V_j tiles into a 2-stage ring
//   warp 1      TMEM allocator and MMA issuer:
//                 S_j = Q K_j^T   into S[j % 2] (TMEM, fp32)
//                 O  += P_j V_j   into O        (TMEM, fp32), V as an MN-major operand
//   warps 2..5  softmax: one query row per thread; reads S_j from TMEM, keeps
//               the running max / sum, rescales O in TMEM when the max grows by
//               more than 2^8 (lazy rescaling keeps the result exact), writes
//               P_j (bf16) into swizzled shared memory, and finally writes
//               O / l to global memory.
#pragma once

#include "common.cuh"

namespace dash {
namespace attn {

constexpr int BQ = 128;  // query rows per CTA
constexpr int BKV = 128; // keys per tile
constexpr int kStages = 2;
constexpr int kThreads = 192;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

struct Params {
  __nv_bfloat16* out;  // [M, hq*hd]
  int64_t ldo;
  const int32_t* qpos; // [M] or NULL
  int M, T_kv, hq, hkv, hd, n_qtiles;
  float scale_log2;    // log2(e) / sqrt(hd)
};

template <int HD>
struct Cfg {
  static constexpr int kPanels = HD / 64;            // 128-byte swizzle panels per row
  static constexpr int kQBytes = BQ * HD * 2;
  static constexpr int kKBytes = BKV * HD * 2;
  static constexpr int kPBytes = BQ * BKV * 2;
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + kQBytes;
  static constexpr int kOffV = kOffK + kStages * kKBytes;
  static constexpr int kOffP = kOffV + kStages * kKBytes;
  static constexpr int kOffBar = kOffP + kPBytes;
  static constexpr int kNumBars = 1 + 3 * kStages + 2 + 1 + 1 + 1;
  static constexpr int kSmemBytes = kOffBar + 8 * kNumBars + 16 + 1024;
  static constexpr uint32_t kTmemCols = 512;  // S0 [0,128), S1 [128,256), O [256, 256+HD)
};

template <int HD>
__global__ void __launch_bounds__(kThreads, 1)
    attn_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
                const __grid_constant__ CUtensorMap tmap_v, const Params p) {
  using C = Cfg<HD>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  // barrier slots
  const uint32_t bar_q = smem_u32(bars + 0);
  const uint32_t bar_kfull0 = smem_u32(bars + 1);
  const uint32_t bar_vfull0 = smem_u32(bars + 1 + kStages);
  const uint32_t bar_kvempty0 = smem_u32(bars + 1 + 2 * kStages);
  const uint32_t bar_sfull0 = smem_u32(bars + 1 + 3 * kStages);
  const uint32_t bar_pfull = smem_u32(bars + 3 + 3 * kStages);
  const uint32_t bar_odone = smem_u32(bars + 4 + 3 * kStages);
  const uint32_t bar_drain = smem_u32(bars + 5 + 3 * kStages);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::kNumBars);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int head = blockIdx.x % p.hq;
  const int qt = p.n_qtiles - 1 - static_cast<int>(blockIdx.x / p.hq);  // heavy tiles first
  const int kvh = head / (p.hq / p.hkv);
  const int q0 = qt * BQ;
  const int q_last = min(p.M - 1, q0 + BQ - 1);
  const int pos_first = p.qpos ? p.qpos[q0] : q0;
  const int pos_last = p.qpos ? p.qpos[q_last] : q_last;
  const int kv_limit = min(pos_last + 1, p.T_kv);
  const int n_tiles = (kv_limit + BKV - 1) / BKV;

  if (threadIdx.x == 0) {
    mbar_init(bar_q, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar_kfull0 + 8 * s, 1);
      mbar_init(bar_vfull0 + 8 * s, 1);
      mbar_init(bar_kvempty0 + 8 * s, 1);
    }
    mbar_init(bar_sfull0, 1);
    mbar_init(bar_sfull0 + 8, 1);
    mbar_init(bar_pfull, 128);
    mbar_init(bar_odone, 1);
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
  const uint32_t tmem_o = tmem_base + 256;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------------------------------------------------- producer
      const uint32_t sq = smem_u32(smem + C::kOffQ);
      mbar_arrive_expect_tx(bar_q, C::kQBytes);
      for (int pn = 0; pn < C::kPanels; ++pn)
        tma_load_2d(&tmap_q, sq + pn * (BQ * 128), bar_q, head * HD + pn * 64, q0);
      uint32_t armed = 0, armed_par = 0;
      for (int j = 0; j < n_tiles; ++j) {
        const int st = j % kStages;
        const uint32_t ph = (j / kStages) & 1;
        if (!mbar_wait(bar_kvempty0 + 8 * st, ph ^ 1u)) break;
        const uint32_t sk = smem_u32(smem + C::kOffK + st * C::kKBytes);
        const uint32_t sv = smem_u32(smem + C::kOffV + st * C::kKBytes);
        mbar_arrive_expect_tx(bar_kfull0 + 8 * st, C::kKBytes);
        for (int pn = 0; pn < C::kPanels; ++pn)
          tma_load_2d(&tmap_k, sk + pn * (BKV * 128), bar_kfull0 + 8 * st, kvh * HD + pn * 64,
                      j * BKV);
        mbar_arrive_expect_tx(bar_vfull0 + 8 * st, C::kKBytes);
        for (int pn = 0; pn < C::kPanels; ++pn)
          tma_load_2d(&tmap_v, sv + pn * (BKV * 128), bar_vfull0 + 8 * st, kvh * HD + pn * 64,
                      j * BKV);
        armed |= 1u << st;
        armed_par = (armed_par & ~(1u << st)) | (ph << st);
      }
      mbar_wait_drain(bar_q, 0);
      for (int s = 0; s < kStages; ++s) {
        if ((armed >> s) & 1u) {
          mbar_wait_drain(bar_kfull0 + 8 * s, (armed_par >> s) & 1u);
          mbar_wait_drain(bar_vfull0 + 8 * s, (armed_par >> s) & 1u);
        }
      }
    }
  } else if (warp == 1) {
    // -------------------------------------------------------------- MMA
    const uint32_t idesc_s = umma_idesc_bf16(BQ, BKV, false, false);
    const uint32_t idesc_o = umma_idesc_bf16(BQ, HD, false, true);
    const uint32_t sq = smem_u32(smem + C::kOffQ);
    const uint32_t sp = smem_u32(smem + C::kOffP);
    bool ok = mbar_wait(bar_q, 0);
    for (int j = 0; ok && j <= n_tiles; ++j) {
      if (j < n_tiles) {
        const int st = j % kStages;
        const uint32_t ph = (j / kStages) & 1;
        if (!mbar_wait(bar_kfull0 + 8 * st, ph)) break;
        tc_fence_after();
        if (lane == 0) {
          const uint32_t sk = smem_u32(smem + C::kOffK + st * C::kKBytes);
          const uint32_t d = tmem_base + (j & 1) * BKV;
#pragma unroll
          for (int kk = 0; kk < HD / 16; ++kk) {
            const uint32_t off = (kk >> 2) * (BQ * 128) + (kk & 3) * 32;
            umma_bf16_ss(d, umma_desc_sw128(sq + off, 16, 1024), umma_desc_sw128(sk + off, 16, 1024),
                         idesc_s, kk != 0 ? 1u : 0u);
          }
          umma_commit(bar_sfull0 + 8 * (j & 1));
        }
        __syncwarp();
      }
      if (j >= 1) {
        const int jp = j - 1;
        const int st = jp % kStages;
        const uint32_t ph = (jp / kStages) & 1;
        if (!mbar_wait(bar_pfull, jp & 1)) break;
        if (!mbar_wait(bar_vfull0 + 8 * st, ph)) break;
        tc_fence_after();
        if (lane == 0) {
          const uint32_t sv = smem_u32(smem + C::kOffV + st * C::kKBytes);
#pragma unroll
          for (int kk = 0; kk < BKV / 16; ++kk) {
            const uint32_t aoff = (kk >> 2) * (BQ * 128) + (kk & 3) * 32;
            umma_bf16_ss(tmem_o, umma_desc_sw128(sp + aoff, 16, 1024),
                         umma_desc_sw128(sv + kk * 16 * 128, BKV * 128, 1024), idesc_o,
                         (jp | kk) != 0 ? 1u : 0u);
          }
          umma_commit(bar_odone);
          umma_commit(bar_kvempty0 + 8 * st);
        }
        __syncwarp();
      }
    }
    if (lane == 0) umma_commit(bar_drain);
    __syncwarp();
    mbar_wait_drain(bar_drain, 0);
  } else {
    // ---------------------------------------------------------- softmax
    const int wq = warp & 3;
    const int r = wq * 32 + lane;  // row within the tile == TMEM lane
    const int m = q0 + r;
    const int mrow = min(m, p.M - 1);
    const int row_pos = p.qpos ? p.qpos[mrow] : m;
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    uint8_t* sp_row = smem + C::kOffP + r * 128;
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int j = 0; j < n_tiles; ++j) {
      if (!mbar_wait(bar_sfull0 + 8 * (j & 1), (j >> 1) & 1)) {
        ok = false;
        break;
      }
      tc_fence_after();
      // Four loads in flight, one wait; the registers are read only after it.
      uint32_t u0[32], u1[32], u2[32], u3[32];
      const uint32_t srow = tmem_base + lane_off + (j & 1) * BKV;
      tmem_ld32(srow + 0, u0);
      tmem_ld32(srow + 32, u1);
      tmem_ld32(srow + 64, u2);
      tmem_ld32(srow + 96, u3);
      tmem_ld_wait();
      float s[BKV];
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        s[i] = __uint_as_float(u0[i]);
        s[32 + i] = __uint_as_float(u1[i]);
        s[64 + i] = __uint_as_float(u2[i]);
        s[96 + i] = __uint_as_float(u3[i]);
      }
      const int kv0 = j * BKV;
      const bool need_mask = (kv0 + BKV - 1 > pos_first) || (kv0 + BKV > p.T_kv);
      float rmax = -INFINITY;
      if (need_mask) {
        const int lim = min(row_pos, p.T_kv - 1) - kv0;  // last visible column of this row
#pragma unroll
        for (int c = 0; c < BKV; ++c) {
          s[c] = (c <= lim) ? s[c] * p.scale_log2 : -INFINITY;
          rmax = fmaxf(rmax, s[c]);
        }
      } else {
#pragma unroll
        for (int c = 0; c < BKV; ++c) {
          s[c] *= p.scale_log2;
          rmax = fmaxf(rmax, s[c]);
        }
      }
      // P_j may be written and O rescaled only once O += P_{j-1} V_{j-1} is done.
      if (j >= 1 && !mbar_wait(bar_odone, (j - 1) & 1)) {
        ok = false;
        break;
      }
      tc_fence_after();
      if (j == 0) {
        m_run = rmax;  // every row sees key 0, so rmax is finite here
      } else if (__any_sync(0xffffffffu, rmax > m_run + kRescaleThreshold)) {
        const float m_new = fmaxf(m_run, rmax);
        const float alpha = exp2f(m_run - m_new);
        m_run = m_new;
        l_run *= alpha;
#pragma unroll 1
        for (int c = 0; c < HD; c += 32) {
          uint32_t o[32];
          tmem_ld32(tmem_o + lane_off + c, o);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
          tmem_st32(tmem_o + lane_off + c, o);
        }
        tmem_st_wait();
      }
      float lsum = 0.f;
#pragma unroll
      for (int ch = 0; ch < BKV / 8; ++ch) {
        float e[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          e[i] = exp2f(s[8 * ch + i] - m_run);
          lsum += e[i];
        }
        uint4 w;
        w.x = pack_bf16(e[0], e[1]);
        w.y = pack_bf16(e[2], e[3]);
        w.z = pack_bf16(e[4], e[5]);
        w.w = pack_bf16(e[6], e[7]);
        const int pn = ch >> 3, cc = ch & 7;
        *reinterpret_cast<uint4*>(sp_row + pn * (BQ * 128) + ((cc ^ (r & 7)) << 4)) = w;
      }
      l_run += lsum;
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(bar_pfull);
    }
    if (ok && n_tiles > 0 && mbar_wait(bar_odone, (n_tiles - 1) & 1)) {
      tc_fence_after();
      const float inv_l = 1.f / l_run;
      __nv_bfloat16* dst = p.out + static_cast<int64_t>(mrow) * p.ldo + head * HD;
#pragma unroll 1
      for (int c = 0; c < HD; c += 32) {
        uint32_t o[32];
        tmem_ld32(tmem_o + lane_off + c, o);
        tmem_ld_wait();
        if (m < p.M) {
          float f[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) f[i] = __uint_as_float(o[i]) * inv_l;
          uint4* d4 = reinterpret_cast<uint4*>(dst + c);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            uint4 w;
            w.x = pack_bf16(f[8 * i + 0], f[8 * i + 1]);
            w.y = pack_bf16(f[8 * i + 2], f[8 * i + 3]);
            w.z = pack_bf16(f[8 * i + 4], f[8 * i + 5]);
            w.w = pack_bf16(f[8 * i + 6], f[8 * i + 7]);
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
