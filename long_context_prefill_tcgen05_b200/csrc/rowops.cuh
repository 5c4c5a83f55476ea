// Row-wise kernels of the DASH prefill path (SIMT, HBM- or latency-bound):
// RMSNorm, the Δattn score, its reduction from GEMM-epilogue partial sums,
// the active-set selection (radix top-k / threshold + ordered compaction),
// row gather / scatter, and the RoPE cos/sin table.
#pragma once

#include "common.cuh"

namespace dash {
namespace rows {

constexpr int kMaxVec = 16;  // 16-byte vectors per lane: rows of up to 4096 16-bit elements

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

template <int DT>
__device__ __forceinline__ float sumsq8(const uint4& v) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  float s = 0.f;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float a = Num<DT>::lo(w[e]), b = Num<DT>::hi(w[e]);
    s = fmaf(a, a, fmaf(b, b, s));
  }
  return s;
}

// ------------------------------------------------------------------ RMSNorm
// y[r] = x[src(r)] * rsqrt(mean(x^2) + eps) * g, one warp per row, fp32 math.
// src(r) = rowmap[r] when a row map is given (halt mode normalises the frozen
// rows straight from the full hidden-state buffer).
// With row_scale given, the kernel writes y[r] = x[src(r)] * g and
// row_scale[r] = rsqrt(mean(x^2) + eps) instead: the GEMM that consumes y
// applies the scale to its fp32 accumulator, so the normalised activation is
// never rounded to 16 bits (x * g is exact when g = 1).
// Each warp issues its row's loads first; the block then stages g (d
// elements, dynamic shared memory) while they are in flight, so the scaling after the
// row's reduction waits on no second global load.
template <int DT>
__global__ void rmsnorm_kernel(const s16* __restrict__ x, int64_t x_rows, const int32_t* __restrict__ rowmap,
                               int64_t rows, int d, const s16* __restrict__ g, float eps, s16* __restrict__ y,
                               float* __restrict__ row_scale) {
  extern __shared__ uint4 g_s[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t r = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + warp;
  const int nv = d >> 3;
  bool live = r < rows;
  int64_t src = r;
  if (live && rowmap) {
    src = rowmap[r];
    if (src < 0 || src >= x_rows) {  // warp-uniform
      if (lane == 0) flag_error(kDevErrIndex);
      live = false;
    }
  }
  uint4 v[kMaxVec];
  if (live) {
    const uint4* xr = reinterpret_cast<const uint4*>(x + src * d);
#pragma unroll
    for (int i = 0; i < kMaxVec; ++i) {
      const int c = lane + 32 * i;
      if (c < nv) v[i] = xr[c];
    }
  }
  for (int c = threadIdx.x; c < nv; c += blockDim.x) g_s[c] = reinterpret_cast<const uint4*>(g)[c];
  __syncthreads();
  if (!live) return;
  float ss = 0.f;
#pragma unroll
  for (int i = 0; i < kMaxVec; ++i)
    if (lane + 32 * i < nv) ss += sumsq8<DT>(v[i]);
  ss = warp_sum(ss);
  float rs = rsqrtf(ss / static_cast<float>(d) + eps);
  if (row_scale) {
    if (lane == 0) row_scale[r] = rs;
    rs = 1.f;
  }
  uint4* yr = reinterpret_cast<uint4*>(y + r * d);
#pragma unroll
  for (int i = 0; i < kMaxVec; ++i) {
    const int c = lane + 32 * i;
    if (c < nv) {
      const uint4 gv = g_s[c];
      const uint32_t xw[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
      const uint32_t gw[4] = {gv.x, gv.y, gv.z, gv.w};
      uint32_t o[4];
#pragma unroll
      for (int e = 0; e < 4; ++e)
        o[e] = Num<DT>::pack(Num<DT>::lo(xw[e]) * rs * Num<DT>::lo(gw[e]),
                             Num<DT>::hi(xw[e]) * rs * Num<DT>::hi(gw[e]));
      yr[c] = make_uint4(o[0], o[1], o[2], o[3]);
    }
  }
}

// -------------------------------------------------------------------- score
// Δ_t = ||U_t||_2, or ||U_t||_2 / ||H_t||_2 (one warp per row).
constexpr int kRowChunks = 16;  // 16-byte chunks per lane in flight (a 4096-wide 16-bit row)

template <int DT>
__global__ void score_kernel(const s16* __restrict__ u, const s16* __restrict__ h, int64_t T, int d,
                             int relative, float* __restrict__ delta) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t r = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + warp;
  if (r >= T) return;
  const int nv = d >> 3;
  const uint4* ur = reinterpret_cast<const uint4*>(u + r * d);
  float su = 0.f, sh = 0.f;
  // all of a lane's chunks of the row in flight before the reduction
  auto sumsq_row = [&](const uint4* row) {
    float acc = 0.f;
    for (int c0 = lane; c0 < nv; c0 += 32 * kRowChunks) {
      uint4 v[kRowChunks];
#pragma unroll
      for (int u = 0; u < kRowChunks; ++u)
        if (c0 + 32 * u < nv) v[u] = __ldcs(row + c0 + 32 * u);
#pragma unroll
      for (int u = 0; u < kRowChunks; ++u)
        if (c0 + 32 * u < nv) acc += sumsq8<DT>(v[u]);
    }
    return acc;
  };
  su = sumsq_row(ur);
  if (relative) sh = sumsq_row(reinterpret_cast<const uint4*>(h + r * d));
  su = warp_sum(su);
  if (relative) sh = warp_sum(sh);
  if (lane == 0) {
    const float dl = relative ? sqrtf(su) / sqrtf(sh) : sqrtf(su);
    if (!isfinite(dl)) flag_error(kDevErrNonfinite);
    delta[r] = dl;
  }
}

// Δ from the o_proj epilogue's per-tile partial sums [ntiles, M], reduced in
// a fixed order so the result is deterministic.  With accumulate set, delta
// keeps the maximum of its current value and the new Δ (consecutive-layer
// monitoring).
__global__ void score_from_ssq_kernel(const float* __restrict__ ssq_u, const float* __restrict__ ssq_h,
                                      int ntiles, int64_t M, int relative, int accumulate,
                                      float* __restrict__ delta) {
  const int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (t >= M) return;
  float su = 0.f, sh = 0.f;
  for (int j = 0; j < ntiles; ++j) su += ssq_u[j * M + t];
  if (relative)
    for (int j = 0; j < ntiles; ++j) sh += ssq_h[j * M + t];
  const float dl = relative ? sqrtf(su) / sqrtf(sh) : sqrtf(su);
  if (!isfinite(dl)) flag_error(kDevErrNonfinite);
  delta[t] = accumulate ? fmaxf(delta[t], dl) : dl;
}

// ------------------------------------------------------------------- select
// Monotone 32-bit key of an fp32 score: larger score -> larger key; -0 and +0
// share a key (they compare equal).
__device__ __forceinline__ uint32_t score_key(float f) {
  uint32_t u = __float_as_uint(f);
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

constexpr int kSelThreads = 1024;
constexpr int kSelPerThread = 4;  // consecutive elements per thread in a chunk
constexpr int kSelChunk = kSelThreads * kSelPerThread;

// Exclusive block-wide prefix sum of one value per thread; also returns the total.
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, uint32_t* warp_tot, uint32_t& total) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint32_t incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t n = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += n;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const uint32_t wv = warp_tot[lane];
    uint32_t wi = wv;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t n = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += n;
    }
    warp_tot[32 + lane] = wi - wv;  // exclusive
    if (lane == 31) warp_tot[64] = wi;
  }
  __syncthreads();
  const uint32_t res = warp_tot[32 + warp] + incl - v;
  total = warp_tot[64];
  __syncthreads();
  return res;
}

// Selection over T scores, one CTA per segment (one sequence of a varlen
// batch; a single segment [0, T) when seg is NULL).  Within segment b,
// [s0, s1) = [seg[b], seg[b+1]):
//   kind 0 (top-k): among tokens in [lo, hi) choose the k_dyn best by
//     (score desc, index asc); kind 1 (threshold): score >= thr.
//   Tokens outside [lo, hi) (the first keep_first / last keep_last tokens of
//   the segment) are always kept; k_dyn = floor(keep * (hi - lo)) in double.
// Writes the kept (absolute) indices ascending to idx[s0 ...], the others to
// halted[s0 ...] (optional), and the count to count[b]; a NaN/Inf score in
// the segment writes count[b] = -3 instead.
// Top-k finds the k-th key by an 8-bit MSB-first radix select over
// shared-memory histograms, then compacts in index order with block-wide
// ballot prefix sums; among keys equal to the k-th, the lowest indices win.
__global__ void __launch_bounds__(kSelThreads, 1)
    select_kernel(const float* __restrict__ scores_all, int64_t T_all, const int32_t* __restrict__ seg, int kind,
                  double keep, float thr, int keep_first, int keep_last, int32_t* __restrict__ idx_all,
                  int32_t* __restrict__ halted_all, int32_t* __restrict__ count_all) {
  __shared__ uint32_t hist[256];
  __shared__ uint32_t warp_tot[65];
  __shared__ uint32_t s_prefix, s_k;
  __shared__ int s_bad;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t s0 = seg ? seg[blockIdx.x] : 0;
  const int64_t T = seg ? seg[blockIdx.x + 1] - s0 : T_all;
  const float* scores = scores_all + s0;
  int32_t* idx = idx_all + s0;
  int32_t* halted = halted_all ? halted_all + s0 : nullptr;
  int32_t* count = count_all + blockIdx.x;
  const int64_t lo = keep_first < T ? keep_first : T;
  int64_t hi = keep_last > 0 ? T - keep_last : T;
  if (hi < lo) hi = lo;
  const int64_t k_dyn = kind == 0 ? static_cast<int64_t>(floor(keep * static_cast<double>(hi - lo))) : 0;

  if (tid == 0) s_bad = 0;
  __syncthreads();
  int bad = 0;
  for (int64_t t = tid; t < T; t += kSelThreads) bad |= !isfinite(scores[t]);
  if (__any_sync(0xffffffffu, bad) && lane == 0) s_bad = 1;
  __syncthreads();
  if (s_bad) {
    if (tid == 0) {
      count[0] = -3;
      flag_error(kDevErrNonfinite);
    }
    return;
  }

  const int64_t n_mid = hi - lo;
  // mode: 0 none of the middle, 1 all of the middle, 2 radix cut, 3 threshold
  int mode;
  if (kind == 1) mode = 3;
  else if (k_dyn <= 0) mode = 0;
  else if (k_dyn >= n_mid) mode = 1;
  else mode = 2;

  uint32_t kth = 0, k_rem = 0;
  if (mode == 2) {
    uint32_t prefix = 0, mask = 0, k = static_cast<uint32_t>(k_dyn);
    for (int shift = 24; shift >= 0; shift -= 8) {
      for (int b = tid; b < 256; b += kSelThreads) hist[b] = 0;
      __syncthreads();
      for (int64_t base = lo; base < hi; base += kSelThreads) {
        const int64_t t = base + tid;
        const bool in = t < hi;
        uint32_t key = in ? score_key(scores[t]) : 0u;
        const bool match = in && ((key & mask) == prefix);
        const uint32_t bin = (key >> shift) & 255u;
        const uint32_t active = __ballot_sync(0xffffffffu, match);
        if (match) {
          const uint32_t peers = __match_any_sync(active, bin);
          if (lane == __ffs(peers) - 1) atomicAdd(&hist[bin], __popc(peers));
        }
      }
      __syncthreads();
      if (warp == 0) {
        // lane l owns bins [8l, 8l + 8); find the bin holding the k-th largest
        uint32_t cnt[8], own = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          cnt[i] = hist[8 * lane + i];
          own += cnt[i];
        }
        // suffix sum over lanes: incl[l] = keys in bins of lanes >= l
        uint32_t incl = own;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const uint32_t n = __shfl_down_sync(0xffffffffu, incl, o);
          if (lane + o < 32) incl += n;
        }
        const uint32_t above = incl - own;  // keys in bins of higher lanes
        if (above < k && k <= incl) {
          uint32_t acc = above;
          int b = 7;
          for (; b > 0; --b) {
            if (acc + cnt[b] >= k) break;
            acc += cnt[b];
          }
          s_prefix = prefix | (static_cast<uint32_t>(8 * lane + b) << shift);
          s_k = k - acc;
        }
      }
      __syncthreads();
      prefix = s_prefix;
      k = s_k;
      mask |= 255u << shift;
      __syncthreads();
    }
    kth = prefix;
    k_rem = k;  // how many keys equal to kth (lowest indices first) are taken
  }

  // Ordered compaction, kSelChunk consecutive tokens per round.
  uint32_t sel_base = 0, hal_base = 0, eq_base = 0;
  for (int64_t c0 = 0; c0 < T; c0 += kSelChunk) {
    const int64_t t0 = c0 + static_cast<int64_t>(tid) * kSelPerThread;
    bool gt[kSelPerThread], eq[kSelPerThread], valid[kSelPerThread], forced[kSelPerThread];
    uint32_t n_eq = 0;
#pragma unroll
    for (int i = 0; i < kSelPerThread; ++i) {
      const int64_t t = t0 + i;
      valid[i] = t < T;
      forced[i] = valid[i] && (t < lo || t >= hi);
      gt[i] = eq[i] = false;
      if (valid[i] && !forced[i]) {
        const float s = scores[t];
        if (mode == 1) gt[i] = true;
        else if (mode == 3) gt[i] = s >= thr;
        else if (mode == 2) {
          const uint32_t key = score_key(s);
          gt[i] = key > kth;
          eq[i] = key == kth;
        }
      }
      n_eq += eq[i];
    }
    uint32_t tot_eq;
    uint32_t eq_rank = eq_base + block_excl_scan(n_eq, warp_tot, tot_eq);
    bool sel[kSelPerThread];
    uint32_t n_sel = 0, n_hal = 0;
#pragma unroll
    for (int i = 0; i < kSelPerThread; ++i) {
      bool take_eq = false;
      if (eq[i]) {
        take_eq = eq_rank < k_rem;
        ++eq_rank;
      }
      sel[i] = valid[i] && (forced[i] || gt[i] || take_eq);
      n_sel += sel[i];
      n_hal += valid[i] && !sel[i];
    }
    uint32_t tot_pk;
    const uint32_t pk = block_excl_scan((n_sel << 16) | n_hal, warp_tot, tot_pk);
    uint32_t ps = sel_base + (pk >> 16), ph = hal_base + (pk & 0xffffu);
#pragma unroll
    for (int i = 0; i < kSelPerThread; ++i) {
      if (!valid[i]) continue;
      if (sel[i]) idx[ps++] = static_cast<int32_t>(s0 + t0 + i);
      else if (halted) halted[ph++] = static_cast<int32_t>(s0 + t0 + i);
    }
    sel_base += tot_pk >> 16;
    hal_base += tot_pk & 0xffffu;
    eq_base += tot_eq;
  }
  if (tid == 0) count[0] = static_cast<int32_t>(sel_base);
}

// ------------------------------------------------------ multi-SM select
// Selection for one sequence spread over all SMs ([DASH blog] §3.1 step 3
// and the final ascending sort of §3.3; threshold form from [DASH news]).
// Same result, bit for bit, as select_kernel on one segment:
//   1. sel_hist_kernel     one pass over the scores: a histogram of the 11
//                          most significant bits of every middle token's
//                          monotone key, summed over the CTAs (top-k only)
//   2. sel_scan_kernel     every CTA finds the bucket holding the cut from
//                          that histogram, counts the tokens of its chunk
//                          whose fate is certain (bucket above the cut, or
//                          the threshold test), and appends the cut bucket's
//                          tokens to a candidate list
//   3. sel_resolve_kernel  one CTA resolves the exact cut key among the
//                          candidates and how many keys equal to it are
//                          taken (lowest indices first), then the output
//                          offset of every chunk
//   4. sel_compact_kernel  every CTA writes its chunk's kept and halted
//                          indices in ascending order at those offsets
// A chunk is kSelCtaTok consecutive tokens; its CTA owns them in every pass.
constexpr int kSelCtaThreads = 256;
constexpr int kSelCtaTok = kSelCtaThreads * kSelPerThread;  // tokens per chunk
constexpr int kSelBits = 11;
constexpr int kSelBins = 1 << kSelBits;
constexpr int kSelShift = 32 - kSelBits;
constexpr int kResolveThreads = 1024;

// Scratch in the caller's workspace; the header (hist, n_cand, bad) must be
// zero when sel_hist_kernel starts.
struct SelState {
  uint32_t hist[kSelBins];  // middle tokens per key bucket
  uint32_t n_cand;          // candidates appended
  int32_t bad;              // a non-finite score was seen
  uint32_t kth;             // the cut key (top-k)
  uint32_t k_rem;           // keys equal to kth that are kept, lowest indices first
};
struct SelArgs {
  const float* scores;
  int64_t T, lo, hi;   // the middle [lo, hi) is ranked; the rest is forced
  int64_t k_dyn;       // middle tokens to keep (top-k)
  int mode;            // 0 none of the middle, 1 all of it, 2 top-k cut, 3 threshold
  float thr;
  int64_t n_chunks;
  SelState* st;
  uint32_t* cand_key;  // [T]
  int32_t* cand_idx;   // [T]
  uint32_t* n_flag;    // [n_chunks] middle tokens kept for certain
  uint32_t* gt_extra;  // [n_chunks] candidates above the cut key
  uint32_t* eq_cnt;    // [n_chunks] candidates equal to the cut key
  uint32_t* sel_off;   // [n_chunks] first output slot of the chunk's kept tokens
  uint32_t* hal_off;   // [n_chunks] ... and of its halted tokens
  uint32_t* eq_before; // [n_chunks] keys equal to the cut in earlier chunks
  int32_t* idx;        // [T] kept indices, ascending
  int32_t* halted;     // [T] or NULL: the others, ascending
  int32_t* count;      // [1] kept count, or -3 after a non-finite score
};

// Exclusive prefix sum over a block of NT threads (one value each) and the total.
template <int NT>
__device__ __forceinline__ uint32_t block_scan_excl(uint32_t v, uint32_t* sh, uint32_t& total) {
  constexpr int kWarps = NT / 32;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint32_t incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t n = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += n;
  }
  if (lane == 31) sh[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const uint32_t wv = lane < kWarps ? sh[lane] : 0u;
    uint32_t wi = wv;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t n = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += n;
    }
    sh[32 + lane] = wi - wv;
    if (lane == 31) sh[64] = wi;
  }
  __syncthreads();
  const uint32_t res = sh[32 + warp] + incl - v;
  total = sh[64];
  __syncthreads();
  return res;
}

// The bucket holding the k-th largest middle key and the count above it,
// from the global histogram (every caller gets the same answer).
template <int NT>
__device__ __forceinline__ void find_cut_bucket(const SelState* st, int64_t k, uint32_t* sh, int& bucket,
                                                uint32_t& above) {
  constexpr int kPerT = kSelBins / NT;
  __shared__ int s_bucket;
  __shared__ uint32_t s_above;
  if (threadIdx.x == 0) {  // no bucket when fewer than k keys are finite (then the caller sees `bad`)
    s_bucket = -1;
    s_above = 0;
  }
  // thread i owns buckets [kSelBins - (i + 1) * kPerT, kSelBins - i * kPerT): thread 0 the highest
  uint32_t c[kPerT], own = 0;
#pragma unroll
  for (int j = 0; j < kPerT; ++j) {
    c[j] = st->hist[kSelBins - 1 - (threadIdx.x * kPerT + j)];
    own += c[j];
  }
  uint32_t tot;
  const uint32_t before = block_scan_excl<NT>(own, sh, tot);  // keys in higher buckets
  if (before < static_cast<uint64_t>(k) && static_cast<uint64_t>(k) <= static_cast<uint64_t>(before) + own) {
    uint32_t acc = before;
    int j = 0;
    for (; j < kPerT - 1; ++j) {
      if (acc + c[j] >= k) break;
      acc += c[j];
    }
    s_bucket = kSelBins - 1 - (threadIdx.x * kPerT + j);
    s_above = acc;
  }
  __syncthreads();
  bucket = s_bucket;
  above = s_above;
  __syncthreads();
}

__global__ void __launch_bounds__(kSelCtaThreads) sel_hist_kernel(const SelArgs a) {
  __shared__ uint32_t h[kSelBins];
  for (int i = threadIdx.x; i < kSelBins; i += kSelCtaThreads) h[i] = 0;
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int64_t t0 = static_cast<int64_t>(blockIdx.x) * kSelCtaTok + threadIdx.x * kSelPerThread;
#pragma unroll
  for (int i = 0; i < kSelPerThread; ++i) {
    const int64_t t = t0 + i;
    bool in = t >= a.lo && t < a.hi;
    uint32_t bin = 0;
    if (in) {
      const float f = a.scores[t];
      in = isfinite(f);
      bin = score_key(f) >> kSelShift;
    }
    const uint32_t active = __ballot_sync(0xffffffffu, in);
    if (in) {  // one shared atomic per distinct bucket of the warp
      const uint32_t peers = __match_any_sync(active, bin);
      if (lane == __ffs(peers) - 1) atomicAdd(&h[bin], __popc(peers));
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < kSelBins; i += kSelCtaThreads)
    if (h[i]) atomicAdd(&a.st->hist[i], h[i]);
}

__global__ void __launch_bounds__(kSelCtaThreads) sel_scan_kernel(const SelArgs a) {
  __shared__ uint32_t sh[65];
  const int lane = threadIdx.x & 31;
  const int64_t c = blockIdx.x;
  int bucket = -1;
  uint32_t above = 0;
  if (a.mode == 2) find_cut_bucket<kSelCtaThreads>(a.st, a.k_dyn, sh, bucket, above);
  const int64_t t0 = c * kSelCtaTok + threadIdx.x * kSelPerThread;
  uint32_t n = 0;
  int bad = 0;
#pragma unroll
  for (int i = 0; i < kSelPerThread; ++i) {
    const int64_t t = t0 + i;
    bool cand = false;
    uint32_t key = 0;
    if (t < a.T) {
      const float f = a.scores[t];
      bad |= !isfinite(f);
      if (t >= a.lo && t < a.hi) {
        if (a.mode == 1) n += 1;
        else if (a.mode == 3) n += f >= a.thr;
        else if (a.mode == 2 && isfinite(f)) {
          key = score_key(f);
          const int b = static_cast<int>(key >> kSelShift);
          n += b > bucket;
          cand = b == bucket;
        }
      }
    }
    // warp-aggregated append of the cut bucket's tokens
    const uint32_t m = __ballot_sync(0xffffffffu, cand);
    if (m) {
      uint32_t base = 0;
      if (lane == __ffs(m) - 1) base = atomicAdd(&a.st->n_cand, __popc(m));
      base = __shfl_sync(0xffffffffu, base, __ffs(m) - 1);
      if (cand) {
        const uint32_t slot = base + __popc(m & ((1u << lane) - 1u));
        a.cand_key[slot] = key;
        a.cand_idx[slot] = static_cast<int32_t>(t);
      }
    }
  }
  if (__any_sync(0xffffffffu, bad) && lane == 0) atomicOr(&a.st->bad, 1);
  uint32_t tot;
  block_scan_excl<kSelCtaThreads>(n, sh, tot);
  if (threadIdx.x == 0) {
    a.n_flag[c] = tot;
    a.gt_extra[c] = 0;
    a.eq_cnt[c] = 0;
  }
}

__global__ void __launch_bounds__(kResolveThreads, 1) sel_resolve_kernel(const SelArgs a) {
  __shared__ uint32_t sh[65];
  __shared__ uint32_t hist[256];
  __shared__ uint32_t s_prefix, s_k;
  const int tid = threadIdx.x, lane = tid & 31;
  if (a.st->bad) {
    if (tid == 0) {
      a.count[0] = -3;
      flag_error(kDevErrNonfinite);
    }
    return;
  }
  uint32_t kth = 0, k_rem = 0;
  if (a.mode == 2) {
    int bucket;
    uint32_t above;
    find_cut_bucket<kResolveThreads>(a.st, a.k_dyn, sh, bucket, above);
    const uint32_t C = a.st->n_cand;
    // radix select of the (k_dyn - above)-th largest candidate key over the
    // bits below the bucket's, 8 at a time
    uint32_t prefix = static_cast<uint32_t>(bucket) << kSelShift, mask = ~0u << kSelShift;
    uint32_t k = static_cast<uint32_t>(a.k_dyn - above);
    for (int shift = 16; shift >= 0; shift -= 8) {
      for (int b = tid; b < 256; b += kResolveThreads) hist[b] = 0;
      __syncthreads();
      for (uint32_t base = 0; base < C; base += kResolveThreads) {
        const uint32_t j = base + tid;
        const uint32_t key = j < C ? a.cand_key[j] : 0u;
        const bool match = j < C && (key & mask) == prefix;
        const uint32_t bin = (key >> shift) & 255u;
        const uint32_t active = __ballot_sync(0xffffffffu, match);
        if (match) {
          const uint32_t peers = __match_any_sync(active, bin);
          if (lane == __ffs(peers) - 1) atomicAdd(&hist[bin], __popc(peers));
        }
      }
      __syncthreads();
      if (tid < 32) {  // lane l owns bins [8l, 8l + 8)
        uint32_t cnt[8], own = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          cnt[i] = hist[8 * lane + i];
          own += cnt[i];
        }
        uint32_t incl = own;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const uint32_t n = __shfl_down_sync(0xffffffffu, incl, o);
          if (lane + o < 32) incl += n;
        }
        const uint32_t abv = incl - own;
        if (abv < k && k <= incl) {
          uint32_t acc = abv;
          int b = 7;
          for (; b > 0; --b) {
            if (acc + cnt[b] >= k) break;
            acc += cnt[b];
          }
          s_prefix = prefix | (static_cast<uint32_t>(8 * lane + b) << shift);
          s_k = k - acc;
        }
      }
      __syncthreads();
      prefix = s_prefix;
      k = s_k;
      mask |= 255u << shift;
      __syncthreads();
    }
    kth = prefix;
    k_rem = k;
    // per chunk: candidates above the cut key, and equal to it (one atomic
    // per distinct (chunk, kind) of a warp: a warp's candidates mostly share
    // a chunk, appended together)
    for (uint32_t base = 0; base < C; base += kResolveThreads) {
      const uint32_t j = base + tid;
      uint32_t kind = 0;
      int64_t ch = 0;
      if (j < C) {
        const uint32_t key = a.cand_key[j];
        ch = a.cand_idx[j] / kSelCtaTok;
        kind = key > kth ? 1u : (key == kth ? 2u : 0u);
      }
      const uint32_t active = __ballot_sync(0xffffffffu, kind != 0u);
      if (kind != 0u) {
        const uint32_t peers = __match_any_sync(active, static_cast<uint32_t>(ch) * 4u + kind);
        if (lane == __ffs(peers) - 1) atomicAdd(kind == 1u ? &a.gt_extra[ch] : &a.eq_cnt[ch], __popc(peers));
      }
    }
    __syncthreads();
  }
  // output offsets of every chunk, in chunk order
  uint32_t sel_carry = 0, hal_carry = 0, eq_carry = 0;
  for (int64_t c0 = 0; c0 < a.n_chunks; c0 += kResolveThreads) {
    const int64_t c = c0 + tid;
    uint32_t n_sel = 0, n_hal = 0, n_eq = 0;
    if (c < a.n_chunks) {
      const int64_t b = c * kSelCtaTok, e = min(b + kSelCtaTok, a.T);
      const int64_t mid = max(int64_t(0), min(e, a.hi) - max(b, a.lo));
      n_sel = static_cast<uint32_t>((e - b) - mid) + a.n_flag[c];
      if (a.mode == 2) {
        n_eq = a.eq_cnt[c];
        n_sel += a.gt_extra[c];
      }
      n_hal = static_cast<uint32_t>(e - b);  // minus the kept ones, below
    }
    uint32_t tot_eq;
    const uint32_t eq_b = eq_carry + block_scan_excl<kResolveThreads>(n_eq, sh, tot_eq);
    if (a.mode == 2 && c < a.n_chunks) {
      const uint32_t taken = eq_b >= k_rem ? 0u : min(n_eq, k_rem - eq_b);
      n_sel += taken;
    }
    n_hal -= n_sel;
    uint32_t tot_sel, tot_hal;
    const uint32_t so = sel_carry + block_scan_excl<kResolveThreads>(n_sel, sh, tot_sel);
    const uint32_t ho = hal_carry + block_scan_excl<kResolveThreads>(n_hal, sh, tot_hal);
    if (c < a.n_chunks) {
      a.sel_off[c] = so;
      a.hal_off[c] = ho;
      a.eq_before[c] = eq_b;
    }
    sel_carry += tot_sel;
    hal_carry += tot_hal;
    eq_carry += tot_eq;
  }
  if (tid == 0) {
    a.st->kth = kth;
    a.st->k_rem = k_rem;
    a.count[0] = static_cast<int32_t>(sel_carry);
  }
}

__global__ void __launch_bounds__(kSelCtaThreads) sel_compact_kernel(const SelArgs a) {
  __shared__ uint32_t sh[65];
  if (a.st->bad) return;  // uniform
  const int64_t c = blockIdx.x;
  const uint32_t kth = a.st->kth, k_rem = a.st->k_rem;
  const int64_t t0 = c * kSelCtaTok + threadIdx.x * kSelPerThread;
  bool gt[kSelPerThread], eq[kSelPerThread], valid[kSelPerThread], forced[kSelPerThread];
  uint32_t n_eq = 0;
#pragma unroll
  for (int i = 0; i < kSelPerThread; ++i) {
    const int64_t t = t0 + i;
    valid[i] = t < a.T;
    forced[i] = valid[i] && (t < a.lo || t >= a.hi);
    gt[i] = eq[i] = false;
    if (valid[i] && !forced[i]) {
      const float f = a.scores[t];
      if (a.mode == 1) gt[i] = true;
      else if (a.mode == 3) gt[i] = f >= a.thr;
      else if (a.mode == 2) {
        const uint32_t key = score_key(f);
        gt[i] = key > kth;
        eq[i] = key == kth;
      }
    }
    n_eq += eq[i];
  }
  uint32_t tot;
  uint32_t eq_rank = a.eq_before[c] + block_scan_excl<kSelCtaThreads>(n_eq, sh, tot);
  bool sel[kSelPerThread];
  uint32_t n_sel = 0, n_hal = 0;
#pragma unroll
  for (int i = 0; i < kSelPerThread; ++i) {
    bool take_eq = false;
    if (eq[i]) {
      take_eq = eq_rank < k_rem;
      ++eq_rank;
    }
    sel[i] = valid[i] && (forced[i] || gt[i] || take_eq);
    n_sel += sel[i];
    n_hal += valid[i] && !sel[i];
  }
  const uint32_t pk = block_scan_excl<kSelCtaThreads>((n_sel << 16) | n_hal, sh, tot);
  uint32_t ps = a.sel_off[c] + (pk >> 16), ph = a.hal_off[c] + (pk & 0xffffu);
#pragma unroll
  for (int i = 0; i < kSelPerThread; ++i) {
    if (!valid[i]) continue;
    if (sel[i]) a.idx[ps++] = static_cast<int32_t>(t0 + i);
    else if (a.halted) a.halted[ph++] = static_cast<int32_t>(t0 + i);
  }
}

// ---------------------------------------------------------- varlen layout
// For each row i (original token orig = rows ? rows[i] : i) of a varlen batch
// with sequence starts cu[0..nseq]: pos[i] = orig - cu[s] (the RoPE position
// within its sequence s) and, when kstart is given, kstart[i] = kspace[s] (or
// cu[s] without kspace): the first key the row may attend to.
__global__ void seq_layout_kernel(const int32_t* __restrict__ cu, int nseq, const int32_t* __restrict__ rows,
                                  int64_t M, const int32_t* __restrict__ kspace, int32_t* __restrict__ pos,
                                  int32_t* __restrict__ kstart) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < M;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int32_t orig = rows ? rows[i] : static_cast<int32_t>(i);
    int a = 0, b = nseq;  // largest s with cu[s] <= orig
    while (b - a > 1) {
      const int mid = (a + b) >> 1;
      if (cu[mid] <= orig) a = mid;
      else b = mid;
    }
    if (pos) pos[i] = orig - cu[a];
    if (kstart) kstart[i] = kspace ? kspace[a] : cu[a];
  }
}

// -------------------------------------------------------- gather / scatter
// Y[i] = X[idx[i]] (gather) or X[idx[i]] = Y[i] (scatter); one warp per row.
template <bool kScatter>
__global__ void move_rows_kernel(const s16* __restrict__ src, s16* __restrict__ dst,
                                 const int32_t* __restrict__ idx, int64_t K, int64_t T, int d) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t wpb = blockDim.x >> 5;
  const int nv = d >> 3;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * wpb + warp; i < K; i += gridDim.x * wpb) {
    const int64_t t = idx[i];
    if (t < 0 || t >= T) {
      if (lane == 0) flag_error(kDevErrIndex);
      continue;
    }
    const uint4* s = reinterpret_cast<const uint4*>(src + (kScatter ? i : t) * d);
    uint4* o = reinterpret_cast<uint4*>(dst + (kScatter ? t : i) * d);
    // all of a lane's chunks of the row in flight before the first store
    for (int c0 = lane; c0 < nv; c0 += 32 * kRowChunks) {
      uint4 v[kRowChunks];
#pragma unroll
      for (int u = 0; u < kRowChunks; ++u)
        if (c0 + 32 * u < nv) v[u] = __ldcs(s + c0 + 32 * u);
#pragma unroll
      for (int u = 0; u < kRowChunks; ++u)
        if (c0 + 32 * u < nv) o[c0 + 32 * u] = v[u];
    }
  }
}

// ------------------------------------------------------------- RoPE table
// tab[p * half + i] = (cos, sin) of p * theta^(-2i / (2 half)), evaluated in
// fp64 and rounded to fp32.
__global__ void rope_table_kernel(float2* __restrict__ tab, int64_t max_pos, int half, double theta) {
  const int64_t n = max_pos * half;
  for (int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < n;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t p = e / half;
    const int i = static_cast<int>(e - p * half);
    const double inv = pow(theta, -2.0 * i / (2.0 * half));
    double s, c;
    sincos(static_cast<double>(p) * inv, &s, &c);
    tab[e] = make_float2(static_cast<float>(c), static_cast<float>(s));
  }
}

}  // namespace rows
}  // namespace dash
