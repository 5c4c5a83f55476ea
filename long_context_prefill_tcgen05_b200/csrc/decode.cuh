// Generation on the KV cache a DASH prefill leaves behind (sm_100a).
//
// The DASH blog post (§3.1, generation stage; §5.1, KV cache) notes that
// generated tokens are not pruned, but every layer past the halting layer
// cached only the active tokens, so a new token attends to fewer keys.  One
// step runs one new token per sequence (n <= kMaxSeq) through a layer:
//
//   gemv_kernel<kGvQkv>     q/k/v = rmsnorm(x) W_qkv^T, RoPE on q and k, the
//                           new k/v (and position) appended to each cache
//   decode_attn_kernel      split-key attention over each cache on tcgen05; the
//                           last CTA of each (sequence, kv head) merges the
//                           partial softmax results
//   gemv_kernel<kGvResid>   x += o W_o^T
//   gemv_kernel<kGvSwiglu>  act = silu(rmsnorm(x) W_g^T) * (rmsnorm(x) W_u^T)
//   gemv_kernel<kGvResid>   x += act W_d^T
//
// With n <= 8 rows the projections are HBM-bound on the weights (2 bytes
// per multiply-add), so they run on the CUDA cores: one warp streams two
// weight rows with 16-byte loads and keeps n dot products per row; one
// 16-warp CTA per SM takes the row pairs strided over the grid, so the
// weights spread evenly over the SMs.  Every kernel of the step is launched
// with programmatic dependent launch (griddepcontrol) to hide launch gaps.
//
// The attention is HBM-bound on the cache.  Its query group (hq / hkv <= 16
// heads) is too small for a tcgen05 M dimension, so the kernel puts the keys
// on M instead:
//   S^T [128 keys, 16]  = K_tile [128 keys, hd] . Q^T          (A = K, K-major)
//   O^T [hd, 16]       += V_tile^T [hd, 128 keys] . P^T          (A = V^T, MN-major)
// with the group padded to N = 16 columns.  TMEM lane r holds key r of the
// tile for S^T and dimension r for O^T, so the four softmax warps own both.
// K/V tiles arrive by TMA (128B swizzle, no multicast) in a 3-stage ring.
#pragma once

#include "common.cuh"

namespace dash {
namespace decode {

constexpr int kMaxSeq = 8;
constexpr int kMaxSegs = 64;   // sequences x kv heads in one launch
constexpr int kMaxCtas = 256;  // decode-attention CTAs (partial-result slots)
constexpr int kGroupPad = 16;  // query heads per kv head, padded (MMA N)
constexpr int BKV = 128;       // keys per tile (MMA M)
constexpr int kStages = 3;
constexpr int kPrefetchTiles = 3;  // decode attention: tiles sent to L2 before the PDL wait
constexpr int kAttnThreads = 192;
constexpr float kRescaleThreshold = 8.0f;  // log2 units, as in the prefill softmax

// ============================================================ async copies
// (Prefetching the next kernel's weights or cache into L2 during a kernel
// measured slower: a step's kernels are bandwidth-bound while they stream,
// and the prefetch only moved bytes between them.)
__device__ __forceinline__ void prefetch_l2(const void* ptr, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(reinterpret_cast<uint64_t>(ptr)), "r"(bytes)
               : "memory");
}

// Bulk async copy global -> shared (no tensor map), completing on `bar`.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
               : "memory");
}

// =================================================================== GEMV
enum GemvEpi : int { kGvQkv = 0, kGvResid = 1, kGvSwiglu = 2 };

struct SeqSlots {
  s16* k[kMaxSeq];  // cache arrays of this layer
  s16* v[kMaxSeq];
  int32_t* pos[kMaxSeq];      // may be NULL
  int64_t row[kMaxSeq];       // row the new token's k/v go to
  int32_t p[kMaxSeq];         // RoPE position of the new token
};

struct GemvParams {
  const s16* W;     // [rows, K] row-major
  const s16* W2;    // kGvSwiglu: up-projection [rows, K]
  const s16* x;     // [n, K]
  const s16* gain;  // kGvQkv / kGvSwiglu: RMSNorm gain [K] (the norm is fused)
  float eps;
  int n, K, tasks;
  int stage_x;                // kGvResid: copy x to shared memory first (it fits)
  int x_smem;                 // bytes of dynamic shared memory taken by staged x (16-byte multiple)
  int pre_bytes;              // leading bytes of each row of a warp's first task loaded to shared
                              // memory before the PDL wait (16-byte multiple, <= 2K; 0: none)
  s16* out;  // kGvResid: residual stream [n, ldo] (in/out); kGvSwiglu: act [n, ldo]
  int64_t ldo;
  s16* q;  // kGvQkv: [n, hq*hd]
  int hq, hkv, hd;
  double theta;
  SeqSlots seq;
};

constexpr int kGemvWarps = 16;  // one CTA per SM; warps take tasks strided over the grid

// Programmatic dependent launch: let the next kernel of the stream be
// scheduled now, and wait until the previous one has finished and its
// writes are visible.  (No-ops for a launch without the PDL attribute.)
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Dot product of 8 16-bit pairs: the even and the odd elements accumulate in
// two fp32 chains, each step one packed fp32x2 multiply-add (two IEEE fmaf,
// one instruction on sm_100), and the chains are added at the end.
template <int DT>
__device__ __forceinline__ float2 pair(uint32_t v) {
  return make_float2(Num<DT>::lo(v), Num<DT>::hi(v));
}
template <int DT>
__device__ __forceinline__ float dot8(const uint4& w, const uint4& x) {
  float2 c = __fmul2_rn(pair<DT>(w.x), pair<DT>(x.x));
  c = __ffma2_rn(pair<DT>(w.y), pair<DT>(x.y), c);
  c = __ffma2_rn(pair<DT>(w.z), pair<DT>(x.z), c);
  c = __ffma2_rn(pair<DT>(w.w), pair<DT>(x.w), c);
  return c.x + c.y;
}

template <int DT>
__device__ __forceinline__ float sumsq8(const uint4& v) {
  using N = Num<DT>;
  float s = 0.f;
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int e = 0; e < 4; ++e) s = fmaf(N::lo(w[e]), N::lo(w[e]), fmaf(N::hi(w[e]), N::hi(w[e]), s));
  return s;
}

template <int DT>
__device__ __forceinline__ uint4 mul8(const uint4& x, const uint4& g) {
  using N = Num<DT>;
  return make_uint4(N::pack(N::lo(x.x) * N::lo(g.x), N::hi(x.x) * N::hi(g.x)),
                    N::pack(N::lo(x.y) * N::lo(g.y), N::hi(x.y) * N::hi(g.y)),
                    N::pack(N::lo(x.z) * N::lo(g.z), N::hi(x.z) * N::hi(g.z)),
                    N::pack(N::lo(x.w) * N::lo(g.w), N::hi(x.w) * N::hi(g.w)));
}

// Streaming read of weights: not kept in L1, 256-byte L2 fetch granularity.
__device__ __forceinline__ uint4 ldg_stream(const uint4* ptr) {
  uint4 v;
  asm("ld.global.nc.L1::no_allocate.L2::256B.v4.u32 {%0, %1, %2, %3}, [%4];"
      : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
      : "l"(ptr));
  return v;
}

// Each task = two weight rows (r0, r1) against all n inputs:
//   kGvQkv     rows (i, i + hd/2) of one q/k/v head: the RoPE pair
//   kGvSwiglu  row t of W (gate) and row t of W2 (up)
//   kGvResid   rows (2t, 2t + 1)
// With the norm fused (kGvQkv, kGvSwiglu) the CTA first computes each
// input row's 1/rms and stages x * gain in shared memory, in the model's
// 16-bit format (exact for unit gains); the 1/rms multiplies the finished dot products, as the
// prefill's GEMM epilogues do.  kGvResid stages x as is when it fits.
//
// Weights are never written during a step, so they need not wait for the
// previous kernel: before its PDL wait every warp starts bulk copies of the
// leading pre_bytes of its first task's two rows into its own shared-memory
// slot.  A CTA starts as soon as the previous kernel's CTA on its SM exits,
// so these copies fill the previous kernel's tail (its SMs finish unevenly,
// the attention's merge runs on a few) with this kernel's own bytes.
template <int EPI, int NS, int DT>
__global__ void __launch_bounds__(32 * kGemvWarps, 1) gemv_kernel(const GemvParams p) {
  constexpr bool kNorm = EPI != kGvResid;
  extern __shared__ uint4 xg_smem[];  // kNorm: [n][K/8]
  __shared__ float red[kGemvWarps][kMaxSeq];
  __shared__ float rs_s[kMaxSeq];
  __shared__ __align__(8) uint64_t pre_bar[kGemvWarps];
  __shared__ float2 rope_cs[EPI == kGvQkv ? kMaxSeq * 64 : 1];  // [m][i]: (cos, sin)
  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int K = p.K, nv = K >> 3;
  if constexpr (EPI == kGvQkv) {
    // RoPE rotation of every (input row, frequency) pair: the positions are
    // launch arguments, so this fp64 work runs before the PDL wait, off the
    // critical path (fp64 angle, as the prefill's table)
    const int half = p.hd >> 1;
    if (threadIdx.x < p.n * half) {
      const int m = threadIdx.x / half, i = threadIdx.x - m * half;
      const double inv = pow(p.theta, -2.0 * i / static_cast<double>(p.hd));
      double sn, cs;
      sincos(static_cast<double>(p.seq.p[m]) * inv, &sn, &cs);
      rope_cs[threadIdx.x] = make_float2(static_cast<float>(cs), static_cast<float>(sn));
    }
  }
  // the two weight rows of a task
  auto rows = [&](int task, const s16*& w0, const s16*& w1) {
    if constexpr (EPI == kGvQkv) {
      const int half = p.hd >> 1;
      const int head = task / half, i = task - head * half;
      w0 = p.W + static_cast<int64_t>(head * p.hd + i) * K;
      w1 = w0 + static_cast<int64_t>(half) * K;
    } else if constexpr (EPI == kGvSwiglu) {
      w0 = p.W + static_cast<int64_t>(task) * K;
      w1 = p.W2 + static_cast<int64_t>(task) * K;
    } else {
      w0 = p.W + static_cast<int64_t>(2 * task) * K;
      w1 = w0 + K;
    }
  };
  const int task0 = blockIdx.x + gridDim.x * warp;
  const bool pre = p.pre_bytes > 0 && task0 < p.tasks;  // warp-uniform
  const uint4* pre_w = reinterpret_cast<const uint4*>(reinterpret_cast<const uint8_t*>(xg_smem) + p.x_smem +
                                                      static_cast<int64_t>(warp) * 2 * p.pre_bytes);
  const uint32_t bar = smem_u32(&pre_bar[warp]);
  if (pre && lane == 0) {
    const s16* r0;
    const s16* r1;
    rows(task0, r0, r1);
    mbar_init(bar, 1);
    fence_mbar_init();
    mbar_arrive_expect_tx(bar, 2u * p.pre_bytes);
    bulk_load(smem_u32(pre_w), r0, p.pre_bytes, bar);
    bulk_load(smem_u32(pre_w) + p.pre_bytes, r1, p.pre_bytes, bar);
  }
  constexpr int U = NS <= 4 ? 8 : 4;  // 16-byte chunks per row in flight per lane
  // A round of a task's two rows: U 16-byte chunks per row per lane.
  // Without a shared-memory preload, the first task's first round is loaded
  // into these registers before the PDL wait (weights do not depend on the
  // previous kernel), so its latency overlaps the wait and the staging of x.
  uint4 ra[U], rb[U];
  const bool reg0 = !pre && task0 < p.tasks;  // warp-uniform
  if (reg0) {
    const s16* r0;
    const s16* r1;
    rows(task0, r0, r1);
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int c = lane + 32 * u;
      if (c < nv) {
        ra[u] = ldg_stream(reinterpret_cast<const uint4*>(r0) + c);
        rb[u] = ldg_stream(reinterpret_cast<const uint4*>(r1) + c);
      }
    }
  }
  pdl_wait();
  const uint4* xg = reinterpret_cast<const uint4*>(p.x);
  if constexpr (kNorm) {
    float ss[NS];
#pragma unroll
    for (int m = 0; m < NS; ++m) ss[m] = 0.f;
    const uint4* gv = reinterpret_cast<const uint4*>(p.gain);
    for (int c = threadIdx.x; c < nv; c += blockDim.x) {
      const uint4 g = __ldg(gv + c);
#pragma unroll
      for (int m = 0; m < NS; ++m)
        if (m < p.n) {
          const uint4 v = __ldg(xg + static_cast<int64_t>(m) * nv + c);
          ss[m] += sumsq8<DT>(v);
          xg_smem[m * nv + c] = mul8<DT>(v, g);
        }
    }
#pragma unroll
    for (int m = 0; m < NS; ++m) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) ss[m] += __shfl_xor_sync(0xffffffffu, ss[m], o);
      if (lane == 0) red[warp][m] = ss[m];
    }
    __syncthreads();
    if (threadIdx.x < p.n) {
      float t = 0.f;
      for (int w = 0; w < kGemvWarps; ++w) t += red[w][threadIdx.x];
      rs_s[threadIdx.x] = rsqrtf(t / static_cast<float>(K) + p.eps);
    }
    __syncthreads();
    xg = xg_smem;
  } else if (p.stage_x) {
    for (int c = threadIdx.x; c < p.n * nv; c += blockDim.x) xg_smem[c] = __ldg(xg + c);
    __syncthreads();
    xg = xg_smem;
  }
  const bool from_smem = kNorm || p.stage_x;
  const int stride = gridDim.x * kGemvWarps;
  // chunks of the first task's rows in shared memory
  int pv = 0;
  if (pre) {
    // every lane observes the phase (the copies' writes are then visible to it)
    if (!__all_sync(0xffffffffu, mbar_wait(bar, 0))) {  // bounded; flagged as a timeout
      if (lane == 0) mbar_wait_drain(bar, 0);
      return;
    }
    pv = p.pre_bytes >> 4;
  }
  // One task; `first` (the warp's first task) takes the preloaded bytes.
  auto run_task = [&](int task, bool first) {
    int head = 0, i = 0;
    if constexpr (EPI == kGvQkv) {
      head = task / (p.hd >> 1);
      i = task - head * (p.hd >> 1);
    }
    const s16* w0;
    const s16* w1;
    rows(task, w0, w1);
    // kGvResid: lane m loads the two residual values of input row m now, so
    // the load's latency hides behind the task's dot products
    uint32_t res = 0;
    if constexpr (EPI == kGvResid) {
      if (lane < p.n) res = *reinterpret_cast<const uint32_t*>(p.out + static_cast<int64_t>(lane) * p.ldo + 2 * task);
    }
    // The next task's rows go to L2 while this one streams.  (Prefetching the
    // current task's rows as well measured slower: the demand loads race
    // their own prefetch.)
    if (lane == 0) {
      if (task + stride < p.tasks) {
        const s16* n0;
        const s16* n1;
        rows(task + stride, n0, n1);
        prefetch_l2(n0, K * 2);
        prefetch_l2(n1, K * 2);
      }
    }
    const uint4* wa = reinterpret_cast<const uint4*>(w0);
    const uint4* wb = reinterpret_cast<const uint4*>(w1);
    float a0[NS], a1[NS];
#pragma unroll
    for (int m = 0; m < NS; ++m) a0[m] = a1[m] = 0.f;
    const int npv = first ? pv : 0;
    for (int c0 = lane; c0 < nv; c0 += 32 * U) {
      if (!(first && reg0 && c0 == lane)) {  // else: the first round is in ra, rb already
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const int c = c0 + 32 * u;
          if (c < npv) {
            ra[u] = pre_w[c];
            rb[u] = pre_w[npv + c];
          } else if (c < nv) {
            ra[u] = ldg_stream(wa + c);  // weights stream through once per step
            rb[u] = ldg_stream(wb + c);
          }
        }
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int c = c0 + 32 * u;
        if (c < nv) {
#pragma unroll
          for (int m = 0; m < NS; ++m) {
            if (m < p.n) {
              const uint4 xm = from_smem ? xg[m * nv + c] : __ldg(xg + static_cast<int64_t>(m) * nv + c);
              a0[m] += dot8<DT>(ra[u], xm);
              a1[m] += dot8<DT>(rb[u], xm);
            }
          }
        }
      }
    }
#pragma unroll
    for (int m = 0; m < NS; ++m) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        a0[m] += __shfl_xor_sync(0xffffffffu, a0[m], o);
        a1[m] += __shfl_xor_sync(0xffffffffu, a1[m], o);
      }
    }
    // Epilogue: lane m finishes input row m.
#pragma unroll
    for (int m = 0; m < NS; ++m) {
      if (m >= p.n || lane != m) continue;
      const float sc = kNorm ? rs_s[m] : 1.f;
      const float y0 = a0[m] * sc, y1 = a1[m] * sc;
      if constexpr (EPI == kGvQkv) {
        const int hd = p.hd, half = hd >> 1;
        float o0 = y0, o1 = y1;
        if (head < p.hq + p.hkv) {  // rotate-half RoPE at the token's position
          const float2 r = rope_cs[m * half + i];
          const float c = r.x, s = r.y;
          o0 = y0 * c - y1 * s;
          o1 = y1 * c + y0 * s;
        }
        s16* dst;
        if (head < p.hq) {
          dst = p.q + static_cast<int64_t>(m) * p.hq * hd + head * hd;
        } else {
          const int kvd = p.hkv * hd;
          const bool is_k = head < p.hq + p.hkv;
          const int h = is_k ? head - p.hq : head - p.hq - p.hkv;
          dst = (is_k ? p.seq.k[m] : p.seq.v[m]) + p.seq.row[m] * kvd + h * hd;
          if (head == p.hq && i == 0 && p.seq.pos[m]) p.seq.pos[m][p.seq.row[m]] = p.seq.p[m];
        }
        dst[i] = Num<DT>::from_f(o0);
        dst[i + half] = Num<DT>::from_f(o1);
      } else if constexpr (EPI == kGvSwiglu) {
        p.out[static_cast<int64_t>(m) * p.ldo + task] = Num<DT>::from_f(y0 / (1.f + __expf(-y0)) * y1);
      } else {
        s16* o = p.out + static_cast<int64_t>(m) * p.ldo + 2 * task;
        const float r0 = Num<DT>::lo(res) + y0, r1 = Num<DT>::hi(res) + y1;
        *reinterpret_cast<uint32_t*>(o) = Num<DT>::pack(r0, r1);
      }
    }
  };
  if (task0 < p.tasks) run_task(task0, true);
  for (int task = task0 + stride; task < p.tasks; task += stride) run_task(task, false);
}

// ========================================================= decode attention
struct AttnParams {
  const s16* q;  // [n, hq*HD], RoPE applied
  s16* out;      // [n, hq*HD]
  float* part_o;           // [CTA c][g < group][HD]: unnormalised O of each CTA (a segment's CTAs adjacent)
  float* part_ml;          // [CTA c][16][2]: (running max in log2 units, sum); 128 bytes per CTA, so
                           // a segment's block starts 16-byte aligned for the bulk copy
  int n, hq, hkv, group, tiles_per_cta;
  int len[kMaxSeq];                // keys of each sequence (cache rows incl. the new one)
  int seg_cta0[kMaxSegs + 1];      // first CTA of segment s * hkv + h; [nseg] = CTA count
  float scale_log2;                // log2(e) / sqrt(HD)
};

struct AttnMaps {
  CUtensorMap k[kMaxSeq];  // [len, hkv*HD] 16-bit, box {64, 128}, 128B swizzle
  CUtensorMap v[kMaxSeq];
};

template <int HD>
struct ACfg {
  static constexpr int kPanels = HD / 64;
  static constexpr int kTile = BKV * HD * 2;  // one K or V tile
  static constexpr int kOffK = 0;
  static constexpr int kOffV = kStages * kTile;
  // HD = 64: V^T has only 64 rows; the MMA (M = 128) reads its second 64-row
  // panel from here (zeros), and those O^T rows are never used.
  static constexpr int kOffZero = 2 * kStages * kTile;
  static constexpr int kZeroBytes = HD == 64 ? BKV * 128 : 0;
  static constexpr int kOffQ = kOffZero + kZeroBytes;   // [16, HD] K-major, kPanels x 2 KB
  static constexpr int kOffP = kOffQ + kPanels * 2048;  // 2 buffers of [16, 128 keys] K-major, 2 x 2 KB each
  static constexpr int kOffRed = kOffP + 2 * 4096;      // [2][4 warps][16] floats
  static constexpr int kOffBar = kOffRed + 2 * 4 * 16 * 4;
  // full[kStages], empty[kStages], q_ready, s_full[2], p_full[2], pv_done[2], red[2], drain, o_read
  static constexpr int kNumBars = 2 * kStages + 1 + 2 + 2 + 2 + 2 + 1 + 1;
  static constexpr int kSmemBytes = kOffBar + 8 * kNumBars + 16 + 1024;
  static constexpr uint32_t kTmemCols = 64;  // S^T buffers [0,16) [16,32), O^T [32,48)
};

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32"
      " {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0],"
      " {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}
__device__ __forceinline__ float ex2f(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
// Byte offset of element (row, col) in a K-major 128B-swizzled operand whose
// 64-column panels are `panel_bytes` apart (rows of 128 bytes, 8-row atoms).
__device__ __forceinline__ uint32_t sw128_offset(int row, int col, int panel_bytes) {
  const int pn = col >> 6, cc = col & 63;
  return pn * panel_bytes + row * 128 + ((((cc >> 3) ^ (row & 7)) & 7) << 4) + ((cc & 7) << 1);
}


// One CTA = a run of up to tiles_per_cta key tiles of one (sequence, kv head)
// segment.  Warp 0: TMA producer.  Warp 1: TMEM owner and MMA issuer.
// Warps 2..5: Q staging, softmax (lane r = key r of the tile), and the
// epilogue (lane r = dimension r of O^T), writing the CTA's partial result.
template <int HD, int DT>
__global__ void __launch_bounds__(kAttnThreads, 1)
    decode_attn_kernel(const __grid_constant__ AttnMaps maps, const AttnParams p) {
  using C = ACfg<HD>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  pdl_trigger();
  const int b = blockIdx.x;
  const int nseg = p.n * p.hkv;
  int seg = 0;
  while (seg + 1 < nseg && p.seg_cta0[seg + 1] <= b) ++seg;
  const int s = seg / p.hkv, kvh = seg - s * p.hkv;
  const int L = p.len[s];
  const int tiles = (L + BKV - 1) / BKV;
  const int t0 = (b - p.seg_cta0[seg]) * p.tiles_per_cta;
  const int nt = min(t0 + p.tiles_per_cta, tiles) - t0;
  // The CTA's first tiles go to L2 while the previous kernel finishes (an L2
  // prefetch is only a hint: the tile holding the row that kernel appends is
  // read again, coherently, after the wait).
  if (threadIdx.x == 0)
    for (int i = 0; i < min(nt, kPrefetchTiles); ++i)
      for (int pn = 0; pn < HD / 64; ++pn) {
        tma_prefetch_l2_2d(&maps.k[s], kvh * HD + pn * 64, (t0 + i) * BKV);
        tma_prefetch_l2_2d(&maps.v[s], kvh * HD + pn * 64, (t0 + i) * BKV);
      }
  pdl_wait();  // q and the appended cache row come from the previous kernel
  if (nt <= 0) return;  // uniform for the whole CTA

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  const uint32_t bar_full = smem_u32(bars);
  const uint32_t bar_empty = smem_u32(bars + kStages);
  const uint32_t bar_q = smem_u32(bars + 2 * kStages);
  const uint32_t bar_sfull = bar_q + 8;    // [2] S^T buffer b holds tile i (i & 1 == b)
  const uint32_t bar_pfull = bar_q + 24;   // [2] P^T buffer b written for tile i
  const uint32_t bar_pvdone = bar_q + 40;  // [2] P^T(i) V(i) finished, buffer i & 1 free
  const uint32_t bar_red = bar_q + 56;     // [2]
  const uint32_t bar_drain = bar_q + 72;
  const uint32_t bar_oread = bar_q + 80;  // the 128 epilogue threads no longer read TMEM
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::kNumBars);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(bar_full + 8 * i, 1);
      mbar_init(bar_empty + 8 * i, 1);
    }
    mbar_init(bar_q, 128);
    mbar_init(bar_sfull, 1);
    mbar_init(bar_sfull + 8, 1);
    mbar_init(bar_pfull, 128);
    mbar_init(bar_pfull + 8, 128);
    mbar_init(bar_pvdone, 1);
    mbar_init(bar_pvdone + 8, 1);
    mbar_init(bar_red, 128);
    mbar_init(bar_red + 8, 128);
    mbar_init(bar_drain, 1);
    mbar_init(bar_oread, 128);
    fence_mbar_init();
  }
  if (HD == 64) {  // zero panel read as the upper half of V^T
    uint4* z = reinterpret_cast<uint4*>(smem + C::kOffZero);
    for (int i = threadIdx.x; i < C::kZeroBytes / 16; i += kAttnThreads) z[i] = make_uint4(0, 0, 0, 0);
    fence_proxy_async_smem();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&maps.k[s]);
    prefetch_tmap(&maps.v[s]);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  bool tmem_freed = false;  // warp 1

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer
      uint32_t armed = 0, par = 0;
      for (int i = 0; i < nt; ++i) {
        const int st = i % kStages;
        const uint32_t ph = (i / kStages) & 1;
        if (!mbar_wait(bar_empty + 8 * st, ph ^ 1u)) break;
        const uint32_t sk = smem_u32(smem + C::kOffK + st * C::kTile);
        const uint32_t sv = smem_u32(smem + C::kOffV + st * C::kTile);
        mbar_arrive_expect_tx(bar_full + 8 * st, 2 * C::kTile);
        const int row = (t0 + i) * BKV;
        for (int pn = 0; pn < C::kPanels; ++pn) {
          tma_load_2d(&maps.k[s], sk + pn * (BKV * 128), bar_full + 8 * st, kvh * HD + pn * 64, row);
          tma_load_2d(&maps.v[s], sv + pn * (BKV * 128), bar_full + 8 * st, kvh * HD + pn * 64, row);
        }
        armed |= 1u << st;
        par = (par & ~(1u << st)) | (ph << st);
      }
      for (int st = 0; st < kStages; ++st)
        if ((armed >> st) & 1u) mbar_wait_drain(bar_full + 8 * st, (par >> st) & 1u);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA
    const uint32_t idesc_s = umma_idesc<DT>(BKV, kGroupPad, false, false);
    const uint32_t idesc_o = umma_idesc<DT>(BKV, kGroupPad, true, false);
    const uint32_t sq = smem_u32(smem + C::kOffQ);
    const uint32_t sp = smem_u32(smem + C::kOffP);
    const uint32_t sz = smem_u32(smem + C::kOffZero);
    auto issue_s = [&](int i) {  // S^T_i = K_i Q^T
      const int st = i % kStages;
      if (!mbar_wait(bar_full + 8 * st, (i / kStages) & 1)) return false;
      tc_fence_after();
      if (lane == 0) {
        const uint32_t sk = smem_u32(smem + C::kOffK + st * C::kTile);
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint32_t oa = (kk >> 2) * (BKV * 128) + (kk & 3) * 32;
          const uint32_t ob = (kk >> 2) * 2048 + (kk & 3) * 32;
          umma_ss(tmem_base + (i & 1) * kGroupPad, umma_desc_sw128(sk + oa, 16, 1024),
                       umma_desc_sw128(sq + ob, 16, 1024), idesc_s, kk != 0 ? 1u : 0u);
        }
        umma_commit(bar_sfull + 8 * (i & 1));
      }
      __syncwarp();
      return true;
    };
    auto issue_pv = [&](int i) {  // O^T += V_i^T P_i^T
      if (!mbar_wait(bar_pfull + 8 * (i & 1), (i >> 1) & 1)) return false;
      tc_fence_after();
      if (lane == 0) {
        const int st = i % kStages;
        const uint32_t sv = smem_u32(smem + C::kOffV + st * C::kTile);
        const uint32_t lbo = HD == 128 ? BKV * 128 : sz - sv;  // stride of V^T's two 64-row panels
#pragma unroll
        for (int kk = 0; kk < BKV / 16; ++kk) {
          const uint32_t ob = (kk >> 2) * 2048 + (kk & 3) * 32;
          umma_ss(tmem_base + 2 * kGroupPad, umma_desc_sw128(sv + kk * 16 * 128, lbo, 1024),
                       umma_desc_sw128(sp + (i & 1) * 4096 + ob, 16, 1024), idesc_o,
                       (i != 0 || kk != 0) ? 1u : 0u);
        }
        umma_commit(bar_pvdone + 8 * (i & 1));
        umma_commit(bar_empty + 8 * st);
      }
      __syncwarp();
      return true;
    };
    bool ok = mbar_wait(bar_q, 0);
    if (ok) ok = issue_s(0);
    for (int i = 0; ok && i < nt; ++i) {
      if (i + 1 < nt) ok = issue_s(i + 1);
      if (ok) ok = issue_pv(i);
    }
    if (lane == 0) umma_commit(bar_drain);
    __syncwarp();
    mbar_wait_drain(bar_drain, 0);
    // TMEM is freed as soon as the epilogue has read O (a dealloc takes a
    // few microseconds; it then overlaps the partials' stores)
    if (warp_wait(bar_oread, 0)) {
      tc_fence_after();
      tmem_dealloc(tmem_base, C::kTmemCols);
      tmem_freed = true;
    }
  } else {
    // ---------------------------------------------- Q staging, softmax, epilogue
    const int wq = warp & 3;
    const int r = wq * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const int G = p.group;
    // Q of this kv head's group, rows G..15 zero, K-major 128B-swizzled.
    {
      const s16* qs = p.q + static_cast<int64_t>(s) * p.hq * HD + static_cast<int64_t>(kvh) * G * HD;
      constexpr int kChunks = kGroupPad * HD / 8;
      for (int ch = r; ch < kChunks; ch += 128) {
        const int g = ch / (HD / 8), c = ch - g * (HD / 8);
        uint4 v = make_uint4(0, 0, 0, 0);
        if (g < G) v = *reinterpret_cast<const uint4*>(qs + g * HD + c * 8);
        *reinterpret_cast<uint4*>(smem + C::kOffQ + sw128_offset(g, c * 8, 2048)) = v;
      }
      fence_proxy_async_smem();
      mbar_arrive(bar_q);
    }
    float* red = reinterpret_cast<float*>(smem + C::kOffRed);
    const float sc = p.scale_log2;
    float m_run[kGroupPad], l_part[kGroupPad];
#pragma unroll
    for (int g = 0; g < kGroupPad; ++g) {
      m_run[g] = -INFINITY;
      l_part[g] = 0.f;
    }
    bool ok = true;
    for (int i = 0; i < nt; ++i) {
      ok = __all_sync(0xffffffffu, mbar_wait(bar_sfull + 8 * (i & 1), (i >> 1) & 1));
      if (!ok) break;
      tc_fence_after();
      uint32_t u[kGroupPad];
      tmem_ld16(tmem_base + lane_off + (i & 1) * kGroupPad, u);
      tmem_ld_wait();
      const bool valid = (t0 + i) * BKV + r < L;
      float sv[kGroupPad], mx[kGroupPad];
#pragma unroll
      for (int g = 0; g < kGroupPad; ++g) {
        sv[g] = valid ? __uint_as_float(u[g]) * sc : -INFINITY;
        mx[g] = sv[g];
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1)
#pragma unroll
        for (int g = 0; g < kGroupPad; ++g) mx[g] = fmaxf(mx[g], __shfl_xor_sync(0xffffffffu, mx[g], o));
      // tile maximum per head over the four warps (mbarrier exchange)
      float* rb = red + (i & 1) * 64;
      if (lane < kGroupPad) {
        float v = mx[0];
#pragma unroll
        for (int g = 1; g < kGroupPad; ++g) v = lane == g ? mx[g] : v;
        rb[wq * 16 + lane] = v;
      }
      mbar_arrive(bar_red + 8 * (i & 1));
      ok = __all_sync(0xffffffffu, mbar_wait(bar_red + 8 * (i & 1), (i >> 1) & 1));
      if (!ok) break;
      bool rescale = false;
      float alpha[kGroupPad];
#pragma unroll
      for (int g = 0; g < kGroupPad; ++g) {
        const float mt = fmaxf(fmaxf(rb[g], rb[16 + g]), fmaxf(rb[32 + g], rb[48 + g]));
        alpha[g] = 1.f;
        if (i == 0) {
          m_run[g] = mt;  // the first tile of a run always holds a valid key
        } else if (mt > m_run[g] + kRescaleThreshold) {
          rescale = true;
        }
        mx[g] = mt;
      }
      if (rescale) {  // identical decision in every thread (same inputs)
#pragma unroll
        for (int g = 0; g < kGroupPad; ++g) {
          const float mn = fmaxf(m_run[g], mx[g]);
          alpha[g] = mn == m_run[g] ? 1.f : ex2f(m_run[g] - mn);
          m_run[g] = mn;
          l_part[g] *= alpha[g];
        }
      }
      uint16_t pb[kGroupPad];
#pragma unroll
      for (int g = 0; g < kGroupPad; ++g) {
        const float e = valid ? ex2f(sv[g] - m_run[g]) : 0.f;
        l_part[g] += e;
        pb[g] = Num<DT>::from_f(e);
      }
      // P^T buffer i & 1 is free once P_(i-2) V_(i-2) is done; a rescale of
      // O^T also needs P_(i-1) V_(i-1) done.  (Each pv_done barrier is at
      // most one completion ahead of these waits.)
      if (i >= 2) {
        ok = __all_sync(0xffffffffu, mbar_wait(bar_pvdone + 8 * (i & 1), ((i >> 1) - 1) & 1));
        if (!ok) break;
      }
      if (rescale) {
        ok = __all_sync(0xffffffffu, mbar_wait(bar_pvdone + 8 * ((i - 1) & 1), ((i - 1) >> 1) & 1));
        if (!ok) break;
      }
      tc_fence_after();
      if (rescale) {
        uint32_t o[kGroupPad];
        tmem_ld16(tmem_base + lane_off + 2 * kGroupPad, o);
        tmem_ld_wait();
#pragma unroll
        for (int g = 0; g < kGroupPad; ++g) o[g] = __float_as_uint(__uint_as_float(o[g]) * alpha[g]);
        tmem_st16(tmem_base + lane_off + 2 * kGroupPad, o);
        tmem_st_wait();
      }
#pragma unroll
      for (int g = 0; g < kGroupPad; ++g)
        *reinterpret_cast<uint16_t*>(smem + C::kOffP + (i & 1) * 4096 + sw128_offset(g, r, 2048)) = pb[g];
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(bar_pfull + 8 * (i & 1));
    }
    // MMAs complete in order: PV(nt-1) done means all are.
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar_pvdone + 8 * ((nt - 1) & 1), ((nt - 1) >> 1) & 1));
    uint32_t o[kGroupPad];
    if (ok) {
      tc_fence_after();
      tmem_ld16(tmem_base + lane_off + 2 * kGroupPad, o);
      tmem_ld_wait();
    }
    tc_fence_before();
    mbar_arrive(bar_oread);  // on every path, so the MMA warp's wait ends
    if (ok) {
      // sum of each head's exponentials over the CTA's keys
#pragma unroll
      for (int off = 16; off > 0; off >>= 1)
#pragma unroll
        for (int g = 0; g < kGroupPad; ++g) l_part[g] += __shfl_xor_sync(0xffffffffu, l_part[g], off);
      float* rb = red + (nt & 1) * 64;  // the buffer tile nt would use: free now
      if (lane < kGroupPad) {
        float v = l_part[0];
#pragma unroll
        for (int g = 1; g < kGroupPad; ++g) v = lane == g ? l_part[g] : v;
        rb[wq * 16 + lane] = v;
      }
      mbar_arrive(bar_red + 8 * (nt & 1));
      ok = __all_sync(0xffffffffu, mbar_wait(bar_red + 8 * (nt & 1), (nt >> 1) & 1));
      if (ok) {
        float* po = p.part_o + static_cast<int64_t>(b) * G * HD;
        if (r < HD)
#pragma unroll
          for (int g = 0; g < kGroupPad; ++g)
            if (g < G) po[g * HD + r] = __uint_as_float(o[g]);
        if (r < G) {
          float mr = m_run[0], lr = 0.f;
#pragma unroll
          for (int g = 0; g < kGroupPad; ++g)
            if (g == r) {
              mr = m_run[g];
              lr = (rb[g] + rb[16 + g]) + (rb[32 + g] + rb[48 + g]);
            }
          float* pm = p.part_ml + (static_cast<int64_t>(b) * kGroupPad + r) * 2;
          pm[0] = mr;
          pm[1] = lr;
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1 && !tmem_freed) {  // the early free's wait gave up
    tc_fence_after();
    tmem_dealloc(tmem_base, C::kTmemCols);
  }
}

// Merge of every (sequence, kv head) segment's partial results, launched
// after the attention kernel.  One warp per (segment, head g of its
// group, 32 dimensions); lane = dimension:
//   M_g = max_c m_cg,  w_cg = 2^(m_cg - M_g) / sum_c' 2^(m_c'g - M_g) l_c'g,
//   O_g = sum_c w_cg o_cg  (c ascending).
// (The last CTA of each segment used to merge inside the attention kernel:
// one SM then read all of the segment's partials while the others idled.)
struct MergeParams {
  const float* part_o;   // as AttnParams
  const float* part_ml;
  s16* out;              // [n, hq*hd]
  int n, hq, hkv, group, hd, items;
  int seg_cta0[kMaxSegs + 1];
};
constexpr int kMergeWarps = 1;  // one warp per CTA: the merge's loads spread over more SMs

template <int DT>
__global__ void __launch_bounds__(32 * kMergeWarps) decode_merge_kernel(const MergeParams p) {
  __shared__ float wsm[kMergeWarps][kMaxCtas];
  pdl_trigger();
  pdl_wait();  // the partials come from the attention kernel
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int item = blockIdx.x * kMergeWarps + warp;
  if (item >= p.items) return;
  const int slices = p.hd >> 5, G = p.group;
  const int seg = item / (G * slices);
  const int rem = item - seg * G * slices;
  const int g = rem / slices, sl = rem - g * slices;
  const int c0 = p.seg_cta0[seg], nch = p.seg_cta0[seg + 1] - c0;
  // the first batch of o values and every (m, l) are loaded together (one
  // round trip); later batches (segments of more than kBatch CTAs) follow
  constexpr int kBatch = 64;
  const float* po = p.part_o + (static_cast<int64_t>(c0) * G + g) * p.hd + sl * 32 + lane;
  const int64_t cstride = static_cast<int64_t>(G) * p.hd;
  float o[kBatch];
#pragma unroll
  for (int k = 0; k < kBatch; ++k) o[k] = k < nch ? po[k * cstride] : 0.f;
  const float2* ml = reinterpret_cast<const float2*>(p.part_ml) + static_cast<int64_t>(c0) * kGroupPad + g;
  constexpr int kPer = kMaxCtas / 32;
  float2 v[kPer];
#pragma unroll
  for (int k = 0; k < kPer; ++k) {
    const int c = lane + 32 * k;
    v[k] = c < nch ? ml[static_cast<int64_t>(c) * kGroupPad] : make_float2(-INFINITY, 0.f);
  }
  float M = -INFINITY;
#pragma unroll
  for (int k = 0; k < kPer; ++k) M = fmaxf(M, v[k].x);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
  float L = 0.f;
#pragma unroll
  for (int k = 0; k < kPer; ++k)
    if (lane + 32 * k < nch) L = fmaf(ex2f(v[k].x - M), v[k].y, L);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) L += __shfl_xor_sync(0xffffffffu, L, off);
  const float inv = 1.f / L;
#pragma unroll
  for (int k = 0; k < kPer; ++k)
    if (lane + 32 * k < nch) wsm[warp][lane + 32 * k] = ex2f(v[k].x - M) * inv;
  __syncwarp();
  float acc = 0.f;
  for (int cb = 0;;) {
#pragma unroll
    for (int k = 0; k < kBatch; ++k)
      if (cb + k < nch) acc = fmaf(wsm[warp][cb + k], o[k], acc);
    cb += kBatch;
    if (cb >= nch) break;
#pragma unroll
    for (int k = 0; k < kBatch; ++k) o[k] = cb + k < nch ? po[(cb + k) * cstride] : 0.f;
  }
  const int s = seg / p.hkv, kvh = seg - s * p.hkv;
  p.out[static_cast<int64_t>(s) * p.hq * p.hd + static_cast<int64_t>(kvh * G + g) * p.hd + sl * 32 + lane] =
      Num<DT>::from_f(acc);
}

// ============================================================ cache store
// Rows [a, a + rows) of the prefill's per-layer K/V buffers -> cache rows
// [0, rows); pos[r] = pos_src[a + r] (or r when pos_src is NULL).
__global__ void kv_store_kernel(const s16* __restrict__ Kb, const s16* __restrict__ Vb, int kvd, int64_t a,
                                int64_t rows, const int32_t* __restrict__ pos_src, s16* __restrict__ k,
                                s16* __restrict__ v, int32_t* __restrict__ pos) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t wpb = blockDim.x >> 5;
  const int nv = kvd >> 3;
  for (int64_t r = static_cast<int64_t>(blockIdx.x) * wpb + warp; r < rows; r += gridDim.x * wpb) {
    const uint4* sk = reinterpret_cast<const uint4*>(Kb + (a + r) * kvd);
    const uint4* svv = reinterpret_cast<const uint4*>(Vb + (a + r) * kvd);
    uint4* dk = reinterpret_cast<uint4*>(k + r * kvd);
    uint4* dv = reinterpret_cast<uint4*>(v + r * kvd);
    for (int c = lane; c < nv; c += 32) {
      dk[c] = sk[c];
      dv[c] = svv[c];
    }
    if (pos && lane == 0) pos[r] = pos_src ? pos_src[a + r] : static_cast<int32_t>(r);
  }
}

}  // namespace decode
}  // namespace dash
