// Persistent tcgen05 GEMM for sm_100a: D[M, N] = A[M, K] * B[N, K]^T with
// 16-bit operands (bf16 or fp16, template parameter DT; the outputs take the
// same format), fp32 accumulation in tensor memory, and epilogues fused for
// the decoder block of the DASH prefill path:
//
//   kEpiStore     out = D
//   kEpiResid     out = out + D             (residual add, in place)
//   kEpiResidSsq  out = out + D, plus per-row partial sums of D^2 and out_in^2
//                 over the tile's columns -> the attention-update norm
//                 ||U_t||_2 (and ||H_t||_2) of the DASH blog post, §2.1,
//                 with no extra pass over U
//   kEpiSwiglu    out = silu(D_gate) * D_up  (B tile = BN/2 gate rows + BN/2 up rows)
//   kEpiQkv       rotate-half RoPE on q/k heads, split into q / k / v buffers,
//                 k/v rows optionally remapped (halt mode writes them at the
//                 tokens' original positions)
//
// Warp roles (192 threads, one CTA per SM):
//   warp 0      TMA producer: A and B tiles (128B swizzle) into a smem ring
//   warp 1      TMEM allocator and MMA issuer (one thread issues tcgen05.mma)
//   warps 2..5  epilogue: tcgen05.ld of the accumulator, fused math, stores
// The accumulator is double-buffered in TMEM so the epilogue of tile i
// overlaps the main loop of tile i+1.
#pragma once

#include "common.cuh"

namespace dash {
namespace gemm {

constexpr int BM = 128;
constexpr int BK = 64;  // 64 16-bit elements = one 128-byte swizzle row
constexpr int kThreads = 192;
constexpr int kGroupM = 16;  // M tiles per raster group (L2 reuse of B)

enum Epi : int { kEpiStore = 0, kEpiResid = 1, kEpiResidSsq = 2, kEpiSwiglu = 3, kEpiQkv = 4 };

struct EpiArgs {
  s16* out;  // store / resid / swiglu destination
  int64_t ldo;
  float* ssq_u;  // [tiles_n, M] partial sums of D^2 (kEpiResidSsq)
  float* ssq_h;  // [tiles_n, M] partial sums of out_in^2
  s16* q;
  s16* k;
  s16* v;
  int64_t ldq, ldkv;
  const int32_t* pos;        // RoPE position of row m (NULL: m)
  const int32_t* kv_rowmap;  // k/v destination row of row m (NULL: m)
  const float4* rope;        // [max_pos, hd/2] float2 (cos, sin), read as float4 pairs
  const float* row_scale;    // [M] or NULL: per-row factor on the accumulator (RMSNorm 1/rms)
  int col_offset;            // qkv column of this GEMM's column 0
  int hq, hkv, hd;
  int64_t rope_rows;         // kEpiQkv: positions in the RoPE table (pos must lie in [0, rope_rows))
  int64_t kv_rows;           // kEpiQkv: rows of the k / v buffers (kv rows must lie in [0, kv_rows))
  int row0;                  // kEpiQkv: row m of this launch is row row0 + m of the whole GEMM (its
                             // position and k/v row when pos / kv_rowmap are NULL)
};

struct Shape {
  int M, N, K;
  int tiles_m, tiles_n, num_tiles;
};

template <int BN>
struct Cfg {
  static constexpr int kStages = BN == 256 ? 4 : 6;
  static constexpr int kABytes = BM * BK * 2;
  static constexpr int kBBytes = BN * BK * 2;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kTmemCols = 2 * BN;
  static constexpr int kBarBytes = 8 * (2 * kStages + 5) + 8;
  static constexpr int kSmemBytes = kStages * kStageBytes + 1024 + kBarBytes;
};

__device__ __forceinline__ void tile_coords(int t, int tiles_m, int tiles_n, int& tm, int& tn,
                                            int group_m = kGroupM) {
  const int per_group = group_m * tiles_n;
  const int g = t / per_group;
  const int first_m = g * group_m;
  const int gsize = min(tiles_m - first_m, group_m);
  const int r = t - g * per_group;
  tm = first_m + r % gsize;
  tn = r / gsize;
}

template <int DT>
__device__ __forceinline__ void store32(s16* dst, const float* v) {
  uint4* d = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint4 w;
    w.x = Num<DT>::pack(v[8 * i + 0], v[8 * i + 1]);
    w.y = Num<DT>::pack(v[8 * i + 2], v[8 * i + 3]);
    w.z = Num<DT>::pack(v[8 * i + 4], v[8 * i + 5]);
    w.w = Num<DT>::pack(v[8 * i + 6], v[8 * i + 7]);
    d[i] = w;
  }
}

// ----------------------------------------------------------------- epilogues
template <int BN, int EPI, int DT>
__device__ __forceinline__ void epilogue_tile(uint32_t tbase, int m, int tn, const Shape& sh,
                                              const EpiArgs& ep) {
  const bool live = m < sh.M;
  if constexpr (EPI == kEpiStore || EPI == kEpiResid || EPI == kEpiResidSsq) {
    float su = 0.f, sq = 0.f;
#pragma unroll 1
    for (int c = 0; c < BN; c += 32) {
      uint32_t r[32];
      tmem_ld32(tbase + c, r);
      tmem_ld_wait();
      if (live) {
        s16* p = ep.out + static_cast<int64_t>(m) * ep.ldo + tn * BN + c;
        float o[32];
        if constexpr (EPI == kEpiStore) {
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __uint_as_float(r[i]);
        } else {
          const uint4* hp = reinterpret_cast<const uint4*>(p);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint4 hv = hp[j];
            const uint32_t hw[4] = {hv.x, hv.y, hv.z, hv.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float h0 = Num<DT>::lo(hw[e]), h1 = Num<DT>::hi(hw[e]);
              const float a0 = __uint_as_float(r[8 * j + 2 * e]);
              const float a1 = __uint_as_float(r[8 * j + 2 * e + 1]);
              o[8 * j + 2 * e] = h0 + a0;
              o[8 * j + 2 * e + 1] = h1 + a1;
              if constexpr (EPI == kEpiResidSsq) {
                su = fmaf(a0, a0, fmaf(a1, a1, su));
                sq = fmaf(h0, h0, fmaf(h1, h1, sq));
              }
            }
          }
        }
        store32<DT>(p, o);
      }
    }
    if constexpr (EPI == kEpiResidSsq) {
      if (live) {
        ep.ssq_u[static_cast<int64_t>(tn) * sh.M + m] = su;
        ep.ssq_h[static_cast<int64_t>(tn) * sh.M + m] = sq;
      }
    }
  } else if constexpr (EPI == kEpiSwiglu) {
#pragma unroll 1
    for (int c = 0; c < BN / 2; c += 32) {
      uint32_t g[32], u[32];
      tmem_ld32(tbase + c, g);
      tmem_ld32(tbase + BN / 2 + c, u);
      tmem_ld_wait();
      if (live) {
        const float sc = ep.row_scale ? ep.row_scale[m] : 1.f;
        float o[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float gf = __uint_as_float(g[i]) * sc;
          o[i] = gf / (1.f + __expf(-gf)) * (__uint_as_float(u[i]) * sc);
        }
        store32<DT>(ep.out + static_cast<int64_t>(m) * ep.ldo + tn * (BN / 2) + c, o);
      }
    }
  } else {  // kEpiQkv
    const int hd = ep.hd, half = hd >> 1;
    int p = 0, kvrow = 0;
    float sc = 1.f;
    bool ok = live;
    if (ok) {
      p = ep.pos ? ep.pos[m] : ep.row0 + m;
      kvrow = ep.kv_rowmap ? ep.kv_rowmap[m] : ep.row0 + m;
      // Caller-supplied positions index the RoPE table and row maps pick the
      // k / v row written: a row with either out of range is flagged and
      // left unwritten.
      if (p < 0 || p >= ep.rope_rows || kvrow < 0 || kvrow >= ep.kv_rows) {
        flag_error(kDevErrIndex);
        ok = false;
      }
      if (ep.row_scale) sc = ep.row_scale[m];
    }
#pragma unroll 1
    for (int hb = 0; hb < BN / hd; ++hb) {
      const int head = (ep.col_offset + tn * BN + hb * hd) / hd;  // warp-uniform
      s16* dst;
      bool rope = true;
      if (head < ep.hq) {
        dst = ep.q + static_cast<int64_t>(m) * ep.ldq + head * hd;
      } else if (head < ep.hq + ep.hkv) {
        dst = ep.k + static_cast<int64_t>(kvrow) * ep.ldkv + (head - ep.hq) * hd;
      } else {
        dst = ep.v + static_cast<int64_t>(kvrow) * ep.ldkv + (head - ep.hq - ep.hkv) * hd;
        rope = false;
      }
      const uint32_t tb = tbase + hb * hd;
      if (rope) {
#pragma unroll 1
        for (int c = 0; c < half; c += 32) {
          uint32_t x1[32], x2[32];
          tmem_ld32(tb + c, x1);
          tmem_ld32(tb + half + c, x2);
          tmem_ld_wait();
          if (ok) {
            const float4* cs = ep.rope + ((static_cast<int64_t>(p) * half + c) >> 1);
            float y1[32], y2[32];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const float4 t = cs[i];  // (cos_2i, sin_2i, cos_2i+1, sin_2i+1)
              const float a0 = __uint_as_float(x1[2 * i]) * sc, b0 = __uint_as_float(x2[2 * i]) * sc;
              const float a1 = __uint_as_float(x1[2 * i + 1]) * sc, b1 = __uint_as_float(x2[2 * i + 1]) * sc;
              y1[2 * i] = a0 * t.x - b0 * t.y;
              y2[2 * i] = b0 * t.x + a0 * t.y;
              y1[2 * i + 1] = a1 * t.z - b1 * t.w;
              y2[2 * i + 1] = b1 * t.z + a1 * t.w;
            }
            store32<DT>(dst + c, y1);
            store32<DT>(dst + half + c, y2);
          }
        }
      } else {
#pragma unroll 1
        for (int c = 0; c < hd; c += 32) {
          uint32_t r[32];
          tmem_ld32(tb + c, r);
          tmem_ld_wait();
          if (ok) {
            float o[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __uint_as_float(r[i]) * sc;
            store32<DT>(dst + c, o);
          }
        }
      }
    }
  }
}

// -------------------------------------------------------------------- kernel
template <int BN, int EPI, int DT>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                const __grid_constant__ CUtensorMap tmap_b2, const Shape sh, const EpiArgs ep) {
  using C = Cfg<BN>;
  constexpr int S = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + S * C::kABytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S * C::kStageBytes);
  // bars: full[S], empty[S], tfull[2], tempty[2], drain[1]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * S + 5);
  const uint32_t full0 = smem_u32(bars), empty0 = smem_u32(bars + S);
  const uint32_t tfull0 = smem_u32(bars + 2 * S), tempty0 = smem_u32(bars + 2 * S + 2);
  const uint32_t drain = smem_u32(bars + 2 * S + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull0 + 8 * a, 1);
      mbar_init(tempty0 + 8 * a, 128);
    }
    mbar_init(drain, 1);
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmap_a);
    prefetch_tmap(&tmap_b);
    if (EPI == kEpiSwiglu) prefetch_tmap(&tmap_b2);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int nk = sh.K / BK;

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0, armed = 0, armed_par = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < sh.num_tiles && ok; t += gridDim.x) {
        int tm, tn;
        tile_coords(t, sh.tiles_m, sh.tiles_n, tm, tn);
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(empty0 + 8 * stage, phase ^ 1u)) {
            ok = false;
            break;
          }
          const uint32_t fb = full0 + 8 * stage;
          mbar_arrive_expect_tx(fb, C::kStageBytes);
          const uint32_t a_dst = smem_u32(sA + stage * C::kABytes);
          const uint32_t b_dst = smem_u32(sB + stage * C::kBBytes);
          tma_load_2d(&tmap_a, a_dst, fb, kb * BK, tm * BM);
          if constexpr (EPI == kEpiSwiglu) {
            tma_load_2d(&tmap_b, b_dst, fb, kb * BK, tn * (BN / 2));
            tma_load_2d(&tmap_b2, b_dst + (BN / 2) * BK * 2, fb, kb * BK, tn * (BN / 2));
          } else {
            tma_load_2d(&tmap_b, b_dst, fb, kb * BK, tn * BN);
          }
          armed |= 1u << stage;
          armed_par = (armed_par & ~(1u << stage)) | (phase << stage);
          if (++stage == S) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // Let every load this thread issued land before the CTA can exit.
      for (int s = 0; s < S; ++s)
        if ((armed >> s) & 1u) mbar_wait_drain(full0 + 8 * s, (armed_par >> s) & 1u);
    }
  } else if (warp == 1) {
    // One thread issues: a tcgen05.mma holds its issuing thread for about its
    // execution time, so time spent on warp syncs or fences here idles the
    // tensor pipe.  The TMA-loaded stages are ordered by the full-barrier wait
    // alone; a tcgen05 fence is taken only after the epilogue's release of an
    // accumulator (other threads' tcgen05.ld before this thread's MMAs).
    if (lane == 0) {
      const uint32_t idesc = umma_idesc<DT>(BM, BN, false, false);
      // Descriptors differ only in their start-address field (bytes >> 4), so
      // they are advanced by integer adds.
      const uint64_t adesc0 = umma_desc_sw128(smem_u32(sA), 16, 1024);
      const uint64_t bdesc0 = umma_desc_sw128(smem_u32(sB), 16, 1024);
      int stage = 0, local = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < sh.num_tiles && ok; t += gridDim.x, ++local) {
        const int acc = local & 1;
        const uint32_t acc_par = (local >> 1) & 1;
        if (!mbar_wait(tempty0 + 8 * acc, acc_par ^ 1u)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_try_wait(full0 + 8 * stage, phase) && !mbar_wait(full0 + 8 * stage, phase)) {
            ok = false;
            break;
          }
          const uint64_t ad = adesc0 + static_cast<uint64_t>((stage * C::kABytes) >> 4);
          const uint64_t bd = bdesc0 + static_cast<uint64_t>((stage * C::kBBytes) >> 4);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)  // 16 columns = 32 bytes along the 128-byte swizzle row
            umma_ss(d_tmem, ad + 2 * kk, bd + 2 * kk, idesc, (kb | kk) != 0 ? 1u : 0u);
          umma_commit(empty0 + 8 * stage);
          if (++stage == S) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit(tfull0 + 8 * acc);
      }
      // Every MMA this thread issued must finish before TMEM is released.
      umma_commit(drain);
      mbar_wait_drain(drain, 0);
    }
    __syncwarp();
  } else {
    const int wq = warp & 3;  // TMEM lane quarter this warp may access
    int local = 0;
    for (int t = blockIdx.x; t < sh.num_tiles; t += gridDim.x, ++local) {
      const int acc = local & 1;
      const uint32_t acc_par = (local >> 1) & 1;
      if (!mbar_wait(tfull0 + 8 * acc, acc_par)) break;
      tc_fence_after();
      int tm, tn;
      tile_coords(t, sh.tiles_m, sh.tiles_n, tm, tn);
      const int m = tm * BM + wq * 32 + lane;
      const uint32_t tbase = tmem_base + (static_cast<uint32_t>(wq * 32) << 16) + acc * BN;
      epilogue_tile<BN, EPI, DT>(tbase, m, tn, sh, ep);
      tc_fence_before();
      mbar_arrive(tempty0 + 8 * acc);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::kTmemCols);
  }
}


// ------------------------------------------------------- CTA-pair kernel
// The same contraction and epilogues on a pair of SMs (a 2-CTA cluster) that
// share one 256 x 256 tile.  The even CTA issues tcgen05.mma.cta_group::2
// with M = 256: each CTA holds 128 rows of A and 128 rows of B (for SwiGLU:
// CTA 0 the gate rows, CTA 1 the up rows) in its own shared memory and gets
// its 128 x 256 fp32 half of the accumulator in its own TMEM, so its
// epilogue is the single-CTA BN = 256 epilogue on rows tm*256 + rank*128.
// Per SM a k-block stages 32 KB (A 16 KB + half of B 16 KB) instead of 48 KB
// at the same MMA rate, a third less L2 -> SMEM traffic and a third fewer
// shared-memory operand reads by the tensor core.
//
// Barriers: full[s] lives in the even CTA; both CTAs' loads count their bytes
// on it (.cta_group::2) and the even CTA's producer arms it for both.  The
// MMA commits arrive on empty[s] and tfull[a] of both CTAs; all 8 epilogue
// warps of the pair arrive on the even CTA's tempty[a].
struct PairCfg {
  static constexpr int BN = 256;
  static constexpr int kRows = 2 * BM;  // rows of A per pair tile
  static constexpr int kStages = 6;
  static constexpr int kABytes = BM * BK * 2;
  static constexpr int kBBytes = (BN / 2) * BK * 2;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kTmemCols = 2 * BN;
  static constexpr int kGroupM = 8;  // pair tiles per raster group (2048 rows of A)
  static constexpr int kBarBytes = 8 * (2 * kStages + 5) + 8;
  static constexpr int kSmemBytes = kStages * kStageBytes + 1024 + kBarBytes;
};

// sh.tiles_m counts 256-row pair tiles; gridDim.x = 2 * number of pairs.
template <int EPI, int DT>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_pair_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                     const __grid_constant__ CUtensorMap tmap_b2, const Shape sh, const EpiArgs ep) {
  using C = PairCfg;
  constexpr int S = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + S * C::kABytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S * C::kStageBytes);
  // bars: full[S], empty[S], tfull[2], tempty[2], drain[1]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * S + 5);
  const uint32_t full0 = smem_u32(bars), empty0 = smem_u32(bars + S);
  const uint32_t tfull0 = smem_u32(bars + 2 * S), tempty0 = smem_u32(bars + 2 * S + 2);
  const uint32_t drain = smem_u32(bars + 2 * S + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = static_cast<int>(blockIdx.x >> 1), npairs = static_cast<int>(gridDim.x >> 1);
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull0 + 8 * a, 1);
      mbar_init(tempty0 + 8 * a, 8);
    }
    mbar_init(drain, 1);
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmap_a);
    prefetch_tmap(leader || EPI != kEpiSwiglu ? &tmap_b : &tmap_b2);
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_slot), C::kTmemCols);
    tmem_relinquish_pair();
  }
  // The peer's barriers must be initialised before any load or commit
  // reaches them.
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int nk = sh.K / BK;

  if (warp == 0) {
    if (lane == 0) {
      const uint32_t full_pair0 = mapa_shared(full0, 0);
      const CUtensorMap* map_b = EPI == kEpiSwiglu && !leader ? &tmap_b2 : &tmap_b;
      int stage = 0;
      uint32_t phase = 0, armed = 0, armed_par = 0;
      bool ok = true;
      for (int t = pair; t < sh.num_tiles && ok; t += npairs) {
        int tm, tn;
        tile_coords(t, sh.tiles_m, sh.tiles_n, tm, tn, C::kGroupM);
        // A rows past M are loaded from row 0 instead of as an all-out-of-range
        // box: their products land in accumulator rows the epilogue never stores.
        int a_row = tm * C::kRows + static_cast<int>(rank) * BM;
        if (a_row >= sh.M) a_row = 0;
        const int b_row = EPI == kEpiSwiglu ? tn * (C::BN / 2) : tn * C::BN + static_cast<int>(rank) * (C::BN / 2);
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(empty0 + 8 * stage, phase ^ 1u)) {
            ok = false;
            break;
          }
          if (leader) mbar_arrive_expect_tx(full0 + 8 * stage, 2 * C::kStageBytes);
          const uint32_t fb = full_pair0 + 8 * stage;
          tma_load_2d_pair(&tmap_a, smem_u32(sA + stage * C::kABytes), fb, kb * BK, a_row);
          tma_load_2d_pair(map_b, smem_u32(sB + stage * C::kBBytes), fb, kb * BK, b_row);
          armed |= 1u << stage;
          armed_par = (armed_par & ~(1u << stage)) | (phase << stage);
          if (++stage == S) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // Before the CTA may exit: the even CTA waits for every armed stage to
      // land (its full barriers count both CTAs' bytes); both wait for the
      // last commit on each of their empty barriers, which may come from
      // the other SM.
      for (int s = 0; s < S; ++s) {
        if (!((armed >> s) & 1u)) continue;
        if (leader) mbar_wait_drain(full0 + 8 * s, (armed_par >> s) & 1u);
        mbar_wait(empty0 + 8 * s, (armed_par >> s) & 1u);
      }
      if (!ok && !leader) {
        // After an error the even CTA may not arm the phase this CTA's last
        // loads count on; give those copies time to land.
        const unsigned long long t0 = globaltimer();
        while (globaltimer() - t0 < 100000ull) {
        }
      }
    }
  } else if (warp == 1) {
    if (leader && lane == 0) {  // one issuing thread, as in gemm_kernel
      const uint32_t idesc = umma_idesc<DT>(C::kRows, C::BN, false, false);
      const uint64_t adesc0 = umma_desc_sw128(smem_u32(sA), 16, 1024);
      const uint64_t bdesc0 = umma_desc_sw128(smem_u32(sB), 16, 1024);
      int stage = 0, local = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int t = pair; t < sh.num_tiles && ok; t += npairs, ++local) {
        const int acc = local & 1;
        const uint32_t acc_par = (local >> 1) & 1;
        if (!mbar_wait(tempty0 + 8 * acc, acc_par ^ 1u)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * C::BN;
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_try_wait(full0 + 8 * stage, phase) && !mbar_wait(full0 + 8 * stage, phase)) {
            ok = false;
            break;
          }
          const uint64_t ad = adesc0 + static_cast<uint64_t>((stage * C::kABytes) >> 4);
          const uint64_t bd = bdesc0 + static_cast<uint64_t>((stage * C::kBBytes) >> 4);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)
            umma_ss_pair(d_tmem, ad + 2 * kk, bd + 2 * kk, idesc, (kb | kk) != 0 ? 1u : 0u);
          umma_commit_pair(empty0 + 8 * stage, 3);
          if (++stage == S) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit_pair(tfull0 + 8 * acc, 3);
      }
      // Every MMA must finish before either CTA releases its TMEM.
      umma_commit_pair(drain, 1);
      mbar_wait_drain(drain, 0);
    }
    __syncwarp();
  } else {
    const int wq = warp & 3;  // TMEM lane quarter this warp may access
    const uint32_t tempty_pair0 = mapa_shared(tempty0, 0);
    int local = 0;
    for (int t = pair; t < sh.num_tiles; t += npairs, ++local) {
      const int acc = local & 1;
      const uint32_t acc_par = (local >> 1) & 1;
      if (!mbar_wait(tfull0 + 8 * acc, acc_par)) break;
      tc_fence_after();
      int tm, tn;
      tile_coords(t, sh.tiles_m, sh.tiles_n, tm, tn, C::kGroupM);
      const int m = tm * C::kRows + static_cast<int>(rank) * BM + wq * 32 + lane;
      const uint32_t tbase = tmem_base + (static_cast<uint32_t>(wq * 32) << 16) + acc * C::BN;
      epilogue_tile<C::BN, EPI, DT>(tbase, m, tn, sh, ep);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(tempty_pair0 + 8 * acc);
    }
  }
  // barrier.cluster is .aligned: the producer lane rejoins its warp first.
  __syncwarp();
  tc_fence_before();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, C::kTmemCols);
  }
  cluster_sync();
}

}  // namespace gemm
}  // namespace dash
