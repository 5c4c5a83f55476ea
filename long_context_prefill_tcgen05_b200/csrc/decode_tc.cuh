// decode_tc.cuh -- the projections of a generation step for several
// sequences at once ([DASH blog] §3.1, generation stage: every layer runs on
// the new tokens) on the tensor cores.
//
// With n new rows a projection Y[n, R] = X[n, K] W[R, K]^T does 2n FLOP per
// weight byte: at n >= 3 the CUDA-core GEMV (gemv_kernel) spends more issue
// slots on the dot products than HBM leaves it.  Here the weight rows go on
// the MMA's M dimension (tiles of 128 rows streamed by TMA) and the n input
// rows, padded to 16, on N; the fp32 sums of a tile sit in 16 TMEM columns,
// lane r = weight row r.  Short weight matrices are split along K so that
// every SM streams: each (row block, K range) item writes its partial sums,
// and the last CTA to finish a row block adds them in split order (fixed, so
// the result does not depend on timing) and applies the epilogue -- the same
// epilogues as gemv_kernel (RMSNorm scale, RoPE + cache append, SwiGLU,
// residual add).
#pragma once

#include "decode.cuh"

namespace dash {
namespace decode {

constexpr int kTcRows = 128;      // weight rows per tile (MMA M = TMEM lanes)
constexpr int kTcN = 16;          // input rows, padded (MMA N)
constexpr int kTcThreads = 192;   // warp 0 TMA, warp 1 MMA, warps 2..5 epilogue; all stage x
constexpr int kTcMaxStages = 8;
constexpr int kTcMaxItems = 512;  // (row block, K range) items of a split launch
constexpr int kTcMinRows = 3;     // input rows from which the tensor-core form is used

struct TcMaps {
  CUtensorMap w;   // [R, K] 16-bit, box {64, 128}, 128B swizzle
  CUtensorMap w2;  // kGvSwiglu: the up projection (same shape; W holds the gate)
};

struct TcParams {
  const s16* x;     // [n, K]
  const s16* gain;  // kGvQkv / kGvSwiglu: RMSNorm gain [K] (the norm is fused)
  float eps;
  int n, K;
  int blocks;    // R / 128
  int splits;    // K ranges per row block
  int ksteps;    // K / 64
  int stages;    // weight ring depth
  float* part;   // [blocks * splits][128][16 * accumulators] partial sums (splits > 1)
  int* counters; // [blocks] finished items per row block (zero before the launch; left zero)
  s16* out;      // kGvResid: residual stream [n, ldo] (in/out); kGvSwiglu: act [n, ldo]
  int64_t ldo;
  s16* q;        // kGvQkv: [n, hq*hd]
  int hq, hkv, hd;
  double theta;
  SeqSlots seq;
};

__device__ __forceinline__ void named_bar_sync(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}
// Barrier `id` over `count` threads that also ANDs their predicates.
__device__ __forceinline__ bool named_bar_and(int id, int count, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %3, 0;\n\t"
      "bar.red.and.pred q, %1, %2, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(id), "r"(count), "r"(pred ? 1u : 0u)
      : "memory");
  return r != 0u;
}

template <int EPI>
struct TcCfg {
  static constexpr int kAcc = EPI == kGvSwiglu ? 2 : 1;    // accumulators: (gate, up) or one
  static constexpr uint32_t kTileBytes = kTcRows * 128;   // 128 rows x 64 elements
  static constexpr uint32_t kStageBytes = kAcc * kTileBytes;
  static constexpr uint32_t kPanelBytes = kTcN * 128;     // x: 16 rows x 64 elements
  static constexpr uint32_t kTmemCols = 32;
};

template <int EPI, int DT>
__global__ void __launch_bounds__(kTcThreads, 1) gemv_tc_kernel(const __grid_constant__ TcMaps maps,
                                                                const TcParams p) {
  using C = TcCfg<EPI>;
  constexpr bool kNorm = EPI != kGvResid;
  extern __shared__ uint8_t tc_smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(tc_smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* ring = smem;                                   // [stages][kAcc][128 x 64] swizzled
  uint8_t* xs = smem + p.stages * C::kStageBytes;         // x slice: [k-steps][16 x 64] swizzled
  __shared__ float rs_s[kMaxSeq];
  __shared__ float red[kTcThreads / 32][kMaxSeq];
  __shared__ float2 rope_cs[EPI == kGvQkv ? kMaxSeq * 64 : 1];       // [m][i]: (cos, sin)
  __shared__ float ysm[EPI == kGvQkv ? kTcRows * kMaxSeq : 1];        // [row][m]: RoPE partners
  __shared__ int s_ticket;
  __shared__ __align__(8) uint64_t bars[2 * kTcMaxStages + 2];
  __shared__ uint32_t tmem_slot;
  const uint32_t bar_full = smem_u32(&bars[0]);
  const uint32_t bar_empty = smem_u32(&bars[kTcMaxStages]);
  const uint32_t bar_acc = smem_u32(&bars[2 * kTcMaxStages]);        // a tile's sums are in TMEM
  const uint32_t bar_accfree = smem_u32(&bars[2 * kTcMaxStages + 1]); // the epilogue has read them

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int K = p.K, nv = K >> 3;
  pdl_trigger();
  if (threadIdx.x == 0) {
    for (int i = 0; i < p.stages; ++i) {
      mbar_init(bar_full + 8 * i, 1);
      mbar_init(bar_empty + 8 * i, 1);
    }
    mbar_init(bar_acc, 1);
    mbar_init(bar_accfree, 128);
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&maps.w);
    if (C::kAcc == 2) prefetch_tmap(&maps.w2);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&tmem_slot), C::kTmemCols);
    tmem_relinquish();
  }
  if constexpr (EPI == kGvQkv) {  // RoPE rotations (launch arguments: before the PDL wait)
    const int half = p.hd >> 1;
    for (int t = threadIdx.x; t < p.n * half; t += kTcThreads) {
      const int m = t / half, i = t - m * half;
      const double inv = pow(p.theta, -2.0 * i / static_cast<double>(p.hd));
      double sn, cs;
      sincos(static_cast<double>(p.seq.p[m]) * inv, &sn, &cs);
      rope_cs[t] = make_float2(static_cast<float>(cs), static_cast<float>(sn));
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  // Weights do not depend on the previous kernel: the producer fills the
  // ring with the first item's leading tiles before the PDL wait.
  const int items = p.blocks * p.splits;
  auto item_range = [&](int item, int& rb, int& k0, int& nk) {
    rb = item / p.splits;
    const int ks = item - rb * p.splits;
    k0 = static_cast<int>(static_cast<int64_t>(p.ksteps) * ks / p.splits);
    nk = static_cast<int>(static_cast<int64_t>(p.ksteps) * (ks + 1) / p.splits) - k0;
  };
  auto load_tile = [&](uint32_t i, int rb, int k) {  // ring slot i % stages is free
    const int st = static_cast<int>(i % p.stages);
    mbar_arrive_expect_tx(bar_full + 8 * st, C::kStageBytes);
    const uint32_t dst = smem_u32(ring + st * C::kStageBytes);
    tma_load_2d(&maps.w, dst, bar_full + 8 * st, k * 64, rb * kTcRows);
    if (C::kAcc == 2) tma_load_2d(&maps.w2, dst + C::kTileBytes, bar_full + 8 * st, k * 64, rb * kTcRows);
  };
  int early = 0;  // tiles of the first item already issued (producer lane)
  if (warp == 0 && lane == 0 && static_cast<int>(blockIdx.x) < items) {
    int rb, k0, nk;
    item_range(blockIdx.x, rb, k0, nk);
    early = nk < p.stages ? nk : p.stages;
    for (int j = 0; j < early; ++j) load_tile(j, rb, k0 + j);  // fresh slots: nothing to wait for
  }
  pdl_wait();
  const uint4* xg = reinterpret_cast<const uint4*>(p.x);
  if constexpr (kNorm) {  // 1/rms of every input row, over all of K
    float ss[kMaxSeq];
#pragma unroll
    for (int m = 0; m < kMaxSeq; ++m) ss[m] = 0.f;
    for (int c = threadIdx.x; c < nv; c += kTcThreads)
#pragma unroll
      for (int m = 0; m < kMaxSeq; ++m)
        if (m < p.n) ss[m] += sumsq8<DT>(__ldg(xg + static_cast<int64_t>(m) * nv + c));
#pragma unroll
    for (int m = 0; m < kMaxSeq; ++m) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) ss[m] += __shfl_xor_sync(0xffffffffu, ss[m], o);
      if (lane == 0) red[warp][m] = ss[m];
    }
    __syncthreads();
    if (threadIdx.x < p.n) {
      float t = 0.f;
      for (int w = 0; w < kTcThreads / 32; ++w) t += red[w][threadIdx.x];
      rs_s[threadIdx.x] = rsqrtf(t / static_cast<float>(K) + p.eps);
    }
  }

  uint32_t ring_i = 0;     // k-steps through the ring so far (producer and MMA warp alike)
  uint32_t acc_phase = 0;  // items finished
  bool ok = true;
  for (int item = blockIdx.x; item < items; item += gridDim.x) {
    int rb, k0, nk;
    item_range(item, rb, k0, nk);
    __syncthreads();  // the previous item's MMAs have read xs (its sums were read after them)
    // x[:, 64 k0 : 64 (k0 + nk)] (times the gain) as 16-row swizzled panels; rows >= n are zero
    for (int i = threadIdx.x; i < kTcN * nk * 8; i += kTcThreads) {
      const int m = i / (nk * 8), cc = i - m * (nk * 8);
      uint4 v = make_uint4(0, 0, 0, 0);
      if (m < p.n) {
        const int c = k0 * 8 + cc;
        v = __ldg(xg + static_cast<int64_t>(m) * nv + c);
        if constexpr (kNorm) v = mul8<DT>(v, __ldg(reinterpret_cast<const uint4*>(p.gain) + c));
      }
      *reinterpret_cast<uint4*>(xs + sw128_offset(m, cc * 8, C::kPanelBytes)) = v;
    }
    fence_proxy_async_smem();
    __syncthreads();
    if (warp == 0) {
      // ------------------------------------------------------------ producer
      if (lane == 0) {
        for (int j = early; j < nk; ++j) {
          const uint32_t i = ring_i + j;
          if (!mbar_wait(bar_empty + 8 * (i % p.stages), ((i / p.stages) & 1u) ^ 1u)) break;
          load_tile(i, rb, k0 + j);
        }
        early = 0;
      }
      __syncwarp();
    } else if (warp == 1) {
      // ------------------------------------------------------------ MMA
      const uint32_t idesc = umma_idesc<DT>(kTcRows, kTcN, false, false);
      ok = ok && warp_wait(bar_accfree, (acc_phase & 1u) ^ 1u);  // previous item's sums read
      tc_fence_after();
      for (int j = 0; ok && j < nk; ++j) {
        const uint32_t i = ring_i + j;
        const int st = static_cast<int>(i % p.stages);
        ok = warp_wait(bar_full + 8 * st, (i / p.stages) & 1u);
        if (!ok) break;
        tc_fence_after();
        const uint32_t sa = smem_u32(ring + st * C::kStageBytes);
        const uint32_t sb = smem_u32(xs + j * C::kPanelBytes);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint32_t acc = (j | kk) != 0 ? 1u : 0u;
          umma_ss_elect(tmem, umma_desc_sw128(sa + kk * 32, 16, 1024), umma_desc_sw128(sb + kk * 32, 16, 1024),
                        idesc, acc);
          if (C::kAcc == 2)
            umma_ss_elect(tmem + kTcN, umma_desc_sw128(sa + C::kTileBytes + kk * 32, 16, 1024),
                          umma_desc_sw128(sb + kk * 32, 16, 1024), idesc, acc);
        }
        umma_commit_elect(bar_empty + 8 * st);
      }
      umma_commit_elect(bar_acc);
    } else {
      // ------------------------------------------------------------ epilogue
      const int r = (warp & 3) * 32 + lane;  // TMEM lane = weight row r of the block
      const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
      // the four epilogue warps take every decision below alike, so that
      // their named barriers always see all 128 threads
      const bool got = named_bar_and(1, 128, mbar_wait(bar_acc, acc_phase & 1u));
      float y[C::kAcc][kTcN];
#pragma unroll
      for (int a = 0; a < C::kAcc; ++a)
#pragma unroll
        for (int m = 0; m < kTcN; ++m) y[a][m] = 0.f;
      if (got) {
        uint32_t u[C::kAcc][kTcN];
        tc_fence_after();
        tmem_ld16(tmem + lane_off, u[0]);
        if (C::kAcc == 2) tmem_ld16(tmem + lane_off + kTcN, u[C::kAcc - 1]);
        tmem_ld_wait();
#pragma unroll
        for (int a = 0; a < C::kAcc; ++a)
#pragma unroll
          for (int m = 0; m < kTcN; ++m) y[a][m] = __uint_as_float(u[a][m]);
      }
      tc_fence_before();
      mbar_arrive(bar_accfree);
      bool last = got;
      if (p.splits > 1) {
        // this item's partial sums out; the row block's last item adds all of them in split order
        if (got) {
          float4* dst =
              reinterpret_cast<float4*>(p.part + (static_cast<int64_t>(item) * kTcRows + r) * kTcN * C::kAcc);
#pragma unroll
          for (int a = 0; a < C::kAcc; ++a)
#pragma unroll
            for (int m = 0; m < kTcN; m += 4)
              dst[(a * kTcN + m) / 4] = make_float4(y[a][m], y[a][m + 1], y[a][m + 2], y[a][m + 3]);
          __threadfence();
        }
        named_bar_sync(1, 128);
        if (r == 0) s_ticket = got && atomicAdd(&p.counters[rb], 1) == p.splits - 1 ? 1 : 0;
        named_bar_sync(1, 128);
        last = s_ticket != 0;
        if (last) {
          __threadfence();
#pragma unroll
          for (int a = 0; a < C::kAcc; ++a)
#pragma unroll
            for (int m = 0; m < kTcN; ++m) y[a][m] = 0.f;
          for (int s = 0; s < p.splits; ++s) {
            const float4* src = reinterpret_cast<const float4*>(
                p.part + ((static_cast<int64_t>(rb) * p.splits + s) * kTcRows + r) * kTcN * C::kAcc);
#pragma unroll
            for (int a = 0; a < C::kAcc; ++a)
#pragma unroll
              for (int m = 0; m < kTcN; m += 4) {
                const float4 v = __ldcg(src + (a * kTcN + m) / 4);  // written by other CTAs: not from L1
                y[a][m] += v.x;
                y[a][m + 1] += v.y;
                y[a][m + 2] += v.z;
                y[a][m + 3] += v.w;
              }
          }
          if (r == 0) p.counters[rb] = 0;  // ready for the next launch
        }
      }
      const int row = rb * kTcRows + r;  // output row (weight row) of this thread
      if constexpr (EPI == kGvQkv) {
        const int hd = p.hd, half = hd >> 1;
        const int head = row / hd, i = row - head * hd;
        if (last)
#pragma unroll
          for (int m = 0; m < kMaxSeq; ++m)
            if (m < p.n) ysm[r * kMaxSeq + m] = y[0][m] * rs_s[m];
        named_bar_sync(2, 128);
        const int partner = i < half ? r + half : r - half;  // same head: hd divides 128
        if (last) {
#pragma unroll
          for (int m = 0; m < kMaxSeq; ++m) {
            if (m >= p.n) continue;
            const float self = ysm[r * kMaxSeq + m];
            float o = self;
            if (head < p.hq + p.hkv) {  // rotate-half RoPE at the token's position
              const float other = ysm[partner * kMaxSeq + m];
              const float2 cs = rope_cs[m * half + (i < half ? i : i - half)];
              o = i < half ? self * cs.x - other * cs.y : self * cs.x + other * cs.y;
            }
            s16* dst;
            if (head < p.hq) {
              dst = p.q + static_cast<int64_t>(m) * p.hq * hd + row;
            } else {
              const int kvd = p.hkv * hd;
              const bool is_k = head < p.hq + p.hkv;
              const int c = row - p.hq * hd - (is_k ? 0 : kvd);
              dst = (is_k ? p.seq.k[m] : p.seq.v[m]) + p.seq.row[m] * kvd + c;
              if (head == p.hq && i == 0 && p.seq.pos[m]) p.seq.pos[m][p.seq.row[m]] = p.seq.p[m];
            }
            *dst = Num<DT>::from_f(o);
          }
        }
        named_bar_sync(2, 128);  // ysm is rewritten by the next item
      } else if constexpr (EPI == kGvSwiglu) {
        if (last)
#pragma unroll
          for (int m = 0; m < kMaxSeq; ++m) {
            if (m >= p.n) continue;
            const float g = y[0][m] * rs_s[m], up = y[C::kAcc - 1][m] * rs_s[m];
            p.out[static_cast<int64_t>(m) * p.ldo + row] = Num<DT>::from_f(g / (1.f + __expf(-g)) * up);
          }
      } else {
        if (last)
#pragma unroll
          for (int m = 0; m < kMaxSeq; ++m) {
            if (m >= p.n) continue;
            s16* o = p.out + static_cast<int64_t>(m) * p.ldo + row;
            *o = Num<DT>::from_f(Num<DT>::to_f(*o) + y[0][m]);
          }
      }
    }
    ring_i += nk;
    ++acc_phase;
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

}  // namespace decode
}  // namespace dash
