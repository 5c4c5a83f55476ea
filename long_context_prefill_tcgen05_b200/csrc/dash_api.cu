// C ABI of libdash (declared in include/dash.h and include/dash_ops.h):
// argument checks, workspace carving, tensor-map encoding, kernel launches,
// and the host-side layer loop of the single-shot DASH prefill.
#include <algorithm>
#include <cstddef>
#include <atomic>
#include <cmath>
#include <cstring>
#include <mutex>
#include <utility>
#include <vector>

#include "dash.h"
#include "dash_ops.h"

#include "attention.cuh"
#include "common.cuh"
#include "decode.cuh"
#include "decode_tc.cuh"
#include "gemm.cuh"
#include "rowops.cuh"

namespace {

using dash::kBf16;
using dash::kF16;
using dash::Num;
using dash::s16;
using dash::attn::attn_kernel;
using dash::gemm::EpiArgs;
using dash::gemm::gemm_kernel;

// ------------------------------------------------------------- device info
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

struct DeviceInfo {
  int num_sms = 0;
};
constexpr int kMaxDevices = 64;
DeviceInfo g_dev[kMaxDevices];
std::mutex g_mu;
EncodeTiledFn g_encode = nullptr;

dash_status device_info(DeviceInfo** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return DASH_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_encode) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || fn == nullptr)
      return DASH_ERR_CUDA;
    g_encode = reinterpret_cast<EncodeTiledFn>(fn);
  }
  if (g_dev[dev].num_sms == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      return DASH_ERR_CUDA;
    g_dev[dev].num_sms = n;
  }
  *out = &g_dev[dev];
  return DASH_OK;
}

inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }
inline const s16* cb(const dash_bf16* p) { return reinterpret_cast<const s16*>(p); }
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline dash_status launch_status() {
  return cudaGetLastError() == cudaSuccess ? DASH_OK : DASH_ERR_CUDA;
}

// ------------------------------------------------------------ launch timing
// While recording, each kernel launch is bracketed by two CUDA events on its
// stream (host-side bookkeeping; meant for a single host thread).
struct TimingRec {
  dash_launch_record r;
  cudaEvent_t e0, e1;
};
struct Timing {
  bool on = false;
  int cap = 0;
  int layer = -1;
  std::vector<TimingRec> recs;
  std::vector<cudaEvent_t> pool;
  size_t used = 0;
} g_timing;

cudaEvent_t next_event() {
  if (g_timing.used == g_timing.pool.size()) {
    cudaEvent_t e;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    g_timing.pool.push_back(e);
  }
  return g_timing.pool[g_timing.used++];
}

class TimedLaunch {
 public:
  // kind < 0: not recorded (a launch inside another record's span);
  // launches: kernel launches the record spans
  TimedLaunch(int kind, int64_t m, int64_t n, int64_t k, cudaStream_t st, int launches = 1) : st_(st) {
    if (!g_timing.on || kind < 0 || static_cast<int>(g_timing.recs.size()) >= g_timing.cap) return;
    cudaEvent_t e0 = next_event(), e1 = next_event();
    if (!e0 || !e1) return;
    TimingRec t;
    t.r.kind = kind;
    t.r.layer = g_timing.layer;
    t.r.m = m;
    t.r.n = n;
    t.r.k = k;
    t.r.ms = 0.f;
    t.r.launches = launches;
    t.e0 = e0;
    t.e1 = e1;
    g_timing.recs.push_back(t);
    idx_ = static_cast<int>(g_timing.recs.size()) - 1;
    cudaEventRecord(e0, st_);
  }
  ~TimedLaunch() {
    if (idx_ >= 0) cudaEventRecord(g_timing.recs[idx_].e1, st_);
  }

 private:
  cudaStream_t st_;
  int idx_ = -1;
};

// 2D tensor map of 16-bit elements (format dt) with a 64-element (128-byte)
// inner box and 128B swizzle.
bool make_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint64_t ld, uint32_t box_rows,
              CUtensorMapDataType dt) {
  if (!aligned16(base) || (ld * 2) % 16 != 0 || rows == 0 || cols % 64 != 0) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {ld * 2};
  const cuuint32_t box[2] = {64, box_rows};
  const cuuint32_t es[2] = {1, 1};
  return g_encode(m, dt, 2, const_cast<void*>(base), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ------------------------------------------------------------------- GEMM
template <int BN, int EPI, int DT>
dash_status launch_gemm(const DeviceInfo& di, const s16* A, int64_t lda, int64_t M, int K, const s16* B,
                        const s16* B2, int N, const EpiArgs& ep, cudaStream_t st, int kind) {
  using C = dash::gemm::Cfg<BN>;
  if (M == 0) return DASH_OK;
  static std::once_flag attr_once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(attr_once, [] {
    attr_err = cudaFuncSetAttribute(gemm_kernel<BN, EPI, DT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    C::kSmemBytes);
  });
  if (attr_err != cudaSuccess) return DASH_ERR_CUDA;
  constexpr CUtensorMapDataType kMt = Num<DT>::kMapType;
  CUtensorMap ma, mb, mb2;
  if (!make_map(&ma, A, M, K, lda, dash::gemm::BM, kMt)) return DASH_ERR_INVALID_ARG;
  if (EPI == dash::gemm::kEpiSwiglu) {
    if (!make_map(&mb, B, N / 2, K, K, BN / 2, kMt) || !make_map(&mb2, B2, N / 2, K, K, BN / 2, kMt))
      return DASH_ERR_INVALID_ARG;
  } else {
    if (!make_map(&mb, B, N, K, K, BN, kMt)) return DASH_ERR_INVALID_ARG;
    mb2 = mb;
  }
  dash::gemm::Shape sh;
  sh.M = static_cast<int>(M);
  sh.N = N;
  sh.K = K;
  sh.tiles_m = static_cast<int>((M + dash::gemm::BM - 1) / dash::gemm::BM);
  sh.tiles_n = N / BN;
  sh.num_tiles = sh.tiles_m * sh.tiles_n;
  const int grid = sh.num_tiles < di.num_sms ? sh.num_tiles : di.num_sms;
  TimedLaunch tl(kind, M, N, K, st);
  gemm_kernel<BN, EPI, DT><<<grid, dash::gemm::kThreads, C::kSmemBytes, st>>>(ma, mb, mb2, sh, ep);
  return launch_status();
}

// 256 x 256 tiles on SM pairs (2-CTA clusters).
std::atomic<int> g_gemm_pairs{1};

// How many pairs of this kernel the device runs at once (0: none, e.g. the
// attribute or the occupancy query failed; the single-SM kernel is used).
template <int EPI, int DT>
int gemm_pair_capacity(const DeviceInfo& di) {
  using C = dash::gemm::PairCfg;
  auto kernel = dash::gemm::gemm_pair_kernel<EPI, DT>;
  static std::once_flag once;
  static int max_pairs = 0;
  std::call_once(once, [&] {
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes) != cudaSuccess)
      return;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(static_cast<unsigned>(di.num_sms & ~1));
    cfg.blockDim = dim3(dash::gemm::kThreads);
    cfg.dynamicSmemBytes = C::kSmemBytes;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kernel, &cfg) == cudaSuccess) max_pairs = n;
    cudaGetLastError();
  });
  return max_pairs;
}

template <int EPI, int DT>
dash_status launch_gemm_pair(int max_pairs, const s16* A, int64_t lda, int64_t M, int K, const s16* B,
                             const s16* B2, int N, const EpiArgs& ep, cudaStream_t st, int kind,
                             int64_t tile_limit = 0) {
  using C = dash::gemm::PairCfg;
  auto kernel = dash::gemm::gemm_pair_kernel<EPI, DT>;
  if (M == 0) return DASH_OK;
  constexpr CUtensorMapDataType kMt = Num<DT>::kMapType;
  CUtensorMap ma, mb, mb2;
  if (!make_map(&ma, A, M, K, lda, dash::gemm::BM, kMt)) return DASH_ERR_INVALID_ARG;
  if (EPI == dash::gemm::kEpiSwiglu) {
    if (!make_map(&mb, B, N / 2, K, K, C::BN / 2, kMt) || !make_map(&mb2, B2, N / 2, K, K, C::BN / 2, kMt))
      return DASH_ERR_INVALID_ARG;
  } else {
    if (!make_map(&mb, B, N, K, K, C::BN / 2, kMt)) return DASH_ERR_INVALID_ARG;
    mb2 = mb;
  }
  dash::gemm::Shape sh;
  sh.M = static_cast<int>(M);
  sh.N = N;
  sh.K = K;
  sh.tiles_m = static_cast<int>((M + C::kRows - 1) / C::kRows);
  sh.tiles_n = N / C::BN;
  sh.num_tiles = sh.tiles_m * sh.tiles_n;
  if (tile_limit > 0 && tile_limit < sh.num_tiles) sh.num_tiles = static_cast<int>(tile_limit);
  const int pairs = sh.num_tiles < max_pairs ? sh.num_tiles : max_pairs;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.gridDim = dim3(static_cast<unsigned>(2 * pairs));
  cfg.blockDim = dim3(dash::gemm::kThreads);
  cfg.dynamicSmemBytes = C::kSmemBytes;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  TimedLaunch tl(kind, M, N, K, st);
  if (cudaLaunchKernelEx(&cfg, kernel, ma, mb, mb2, sh, ep) != cudaSuccess) return DASH_ERR_CUDA;
  return launch_status();
}

template <int EPI, int DT>
dash_status gemm(const DeviceInfo& di, const s16* A, int64_t lda, int64_t M, int K, const s16* B,
                 const s16* B2, int N, const EpiArgs& ep, cudaStream_t st, int kind, int* bn_used = nullptr) {
  if (K % dash::gemm::BK != 0 || M > INT32_MAX) return DASH_ERR_SHAPE;
  // SwiGLU tiles hold BN/2 gate + BN/2 up columns, so N = 2F must split into
  // whole tiles on both halves.
  const bool can256 = EPI == dash::gemm::kEpiSwiglu ? (N / 2) % 128 == 0 : N % 256 == 0;
  const bool can128 = EPI == dash::gemm::kEpiSwiglu ? (N / 2) % 64 == 0 : N % 128 == 0;
  if (can256) {
    if (bn_used) *bn_used = 256;
    if (M > dash::gemm::BM && g_gemm_pairs.load(std::memory_order_relaxed)) {
      const int pairs = gemm_pair_capacity<EPI, DT>(di);
      if (pairs > 0) {
        // Tiles run in waves of `pairs`; a last wave that is only partly full
        // idles most SM pairs.  Its tiles come last in the grouped raster, so
        // (once rounded up to whole columns of the last group) they form the
        // rectangle rows [m0, M) x columns [n0, N).  When that rectangle fits
        // one wave of 128 x 128 single-SM tiles, the pair kernel stops before
        // it and the single-SM kernel computes it: each output element is
        // still one tile's sum over k in the same order.
        constexpr bool kSplittable = EPI == dash::gemm::kEpiStore || EPI == dash::gemm::kEpiResid ||
                                     EPI == dash::gemm::kEpiQkv;
        using PC = dash::gemm::PairCfg;
        const int64_t tiles_m = (M + PC::kRows - 1) / PC::kRows, tiles_n = N / PC::BN;
        const int64_t num = tiles_m * tiles_n, rem = num % pairs;
        const int64_t g_last = tiles_m - ((tiles_m - 1) / PC::kGroupM) * PC::kGroupM;
        const int64_t cols = (rem + g_last - 1) / g_last, rect = cols * g_last;
        if (kSplittable && num > pairs && rem > 0 && cols < tiles_n && 4 * rect <= di.num_sms) {
          TimedLaunch tl(kind, M, N, K, st, 2);  // one record for both launches
          dash_status r = launch_gemm_pair<EPI, DT>(pairs, A, lda, M, K, B, B2, N, ep, st, -1, num - rect);
          if (r != DASH_OK) return r;
          const int64_t m0 = (tiles_m - g_last) * PC::kRows, n0 = (tiles_n - cols) * PC::BN;
          EpiArgs e = ep;
          if (EPI == dash::gemm::kEpiQkv) {
            e.q = ep.q ? ep.q + m0 * ep.ldq : nullptr;
            if (ep.pos) e.pos = ep.pos + m0;
            if (ep.kv_rowmap) e.kv_rowmap = ep.kv_rowmap + m0;
            if (ep.row_scale) e.row_scale = ep.row_scale + m0;
            e.row0 = ep.row0 + static_cast<int>(m0);
            e.col_offset = ep.col_offset + static_cast<int>(n0);
          } else {
            e.out = ep.out + m0 * ep.ldo + n0;
          }
          return launch_gemm<128, EPI, DT>(di, A + m0 * lda, lda, M - m0, K, B + n0 * K, nullptr,
                                           static_cast<int>(cols * PC::BN), e, st, -1);
        }
        return launch_gemm_pair<EPI, DT>(pairs, A, lda, M, K, B, B2, N, ep, st, kind);
      }
    }
    return launch_gemm<256, EPI, DT>(di, A, lda, M, K, B, B2, N, ep, st, kind);
  }
  if (can128) {
    if (bn_used) *bn_used = 128;
    return launch_gemm<128, EPI, DT>(di, A, lda, M, K, B, B2, N, ep, st, kind);
  }
  return DASH_ERR_SHAPE;
}

inline int o_proj_tiles(int d) { return d % 256 == 0 ? d / 256 : d / 128; }

// -------------------------------------------------------------- attention
template <int HD, int DT>
dash_status launch_attn_hd(const s16* Q, int64_t ldq, const s16* K, const s16* V, int64_t ldkv, int64_t M,
                           int64_t T_kv, int hq, int hkv, const int32_t* qpos, const int32_t* kstart, s16* O,
                           int64_t ldo, cudaStream_t st) {
  using C = dash::attn::Cfg<HD>;
  static std::once_flag attr_once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(attr_once, [] {
    attr_err = cudaFuncSetAttribute(attn_kernel<HD, DT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    C::kSmemBytes);
  });
  if (attr_err != cudaSuccess) return DASH_ERR_CUDA;
  CUtensorMap mq, mk, mv;
  constexpr CUtensorMapDataType kMt = Num<DT>::kMapType;
  if (!make_map(&mq, Q, M, static_cast<uint64_t>(hq) * HD, ldq, dash::attn::BQ, kMt) ||
      !make_map(&mk, K, T_kv, static_cast<uint64_t>(hkv) * HD, ldkv, dash::attn::BKV, kMt) ||
      !make_map(&mv, V, T_kv, static_cast<uint64_t>(hkv) * HD, ldkv, dash::attn::BKV, kMt))
    return DASH_ERR_INVALID_ARG;
  dash::attn::Params p;
  p.out = O;
  p.ldo = ldo;
  p.qpos = qpos;
  p.kstart = kstart;
  p.M = static_cast<int>(M);
  p.T_kv = static_cast<int>(T_kv);
  p.hq = hq;
  p.hkv = hkv;
  p.hd = HD;
  p.n_qblocks = static_cast<int>((M + 2 * dash::attn::BQ - 1) / (2 * dash::attn::BQ));
  p.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(HD)));
  const int64_t grid = static_cast<int64_t>(p.n_qblocks) * hq;
  TimedLaunch tl(DASH_K_ATTENTION, M, T_kv, (qpos || kstart) ? -1 : M * (M + 1) / 2, st);
  attn_kernel<HD, DT><<<static_cast<unsigned>(grid), dash::attn::kThreads, C::kSmemBytes, st>>>(mq, mk, mv, p);
  return launch_status();
}

template <int DT>
dash_status attention(const s16* Q, int64_t ldq, const s16* K, const s16* V, int64_t ldkv, int64_t M,
                      int64_t T_kv, int hq, int hkv, int hd, const int32_t* qpos, const int32_t* kstart, s16* O,
                      int64_t ldo, cudaStream_t st) {
  if (M == 0) return DASH_OK;
  if (T_kv <= 0 || M > INT32_MAX || T_kv > INT32_MAX || hkv <= 0 || hq % hkv != 0) return DASH_ERR_SHAPE;
  if (hd == 128) return launch_attn_hd<128, DT>(Q, ldq, K, V, ldkv, M, T_kv, hq, hkv, qpos, kstart, O, ldo, st);
  if (hd == 64) return launch_attn_hd<64, DT>(Q, ldq, K, V, ldkv, M, T_kv, hq, hkv, qpos, kstart, O, ldo, st);
  return DASH_ERR_SHAPE;
}

// ---------------------------------------------------------------- row ops
template <int DT>
dash_status rmsnorm(const s16* X, int64_t x_rows, const int32_t* rowmap, int64_t rows, int d, const s16* g,
                    double eps, s16* Y, cudaStream_t st, float* row_scale = nullptr) {
  if (rows == 0) return DASH_OK;
  // 4-warp blocks, one row per warp
  constexpr int kWarps = 4;
  const int64_t blocks = (rows + kWarps - 1) / kWarps;
  TimedLaunch tl(DASH_K_RMSNORM, rows, d, 0, st);
  dash::rows::rmsnorm_kernel<DT><<<static_cast<unsigned>(blocks), 32 * kWarps, static_cast<size_t>(d) * sizeof(s16),
                               st>>>(X, x_rows, rowmap, rows, d, g, static_cast<float>(eps), Y, row_scale);
  return launch_status();
}

dash_status move_rows(bool scatter, const s16* src, s16* dst, const int32_t* idx, int64_t K, int64_t T, int d,
                      const DeviceInfo& di, cudaStream_t st) {
  if (K == 0) return DASH_OK;
  const int warps = 8;
  int64_t blocks = (K + warps - 1) / warps;
  const int64_t cap = static_cast<int64_t>(di.num_sms) * 16;
  if (blocks > cap) blocks = cap;
  TimedLaunch tl(scatter ? DASH_K_SCATTER : DASH_K_GATHER, K, d, 0, st);
  if (scatter)
    dash::rows::move_rows_kernel<true><<<static_cast<unsigned>(blocks), 32 * warps, 0, st>>>(src, dst, idx, K, T, d);
  else
    dash::rows::move_rows_kernel<false><<<static_cast<unsigned>(blocks), 32 * warps, 0, st>>>(src, dst, idx, K, T, d);
  return launch_status();
}

dash_status rope_table(float2* tab, int64_t max_pos, int hd, double theta, const DeviceInfo& di, cudaStream_t st) {
  const int64_t n = max_pos * (hd / 2);
  int64_t blocks = (n + 255) / 256;
  const int64_t cap = static_cast<int64_t>(di.num_sms) * 32;
  if (blocks > cap) blocks = cap;
  if (blocks == 0) return DASH_OK;
  TimedLaunch tl(DASH_K_ROPE_TABLE, max_pos, hd / 2, 0, st);
  dash::rows::rope_table_kernel<<<static_cast<unsigned>(blocks), 256, 0, st>>>(tab, max_pos, hd / 2, theta);
  return launch_status();
}

// -------------------------------------------------------------- workspace
struct Carver {
  uint8_t* base;
  size_t off = 0;
  template <class T>
  T* take(size_t count) {
    off = (off + 255) & ~static_cast<size_t>(255);
    T* p = base ? reinterpret_cast<T*>(base + off) : nullptr;
    off += count * sizeof(T);
    return p;
  }
};

struct LayerWs {
  float2* rope;  // [max_pos, hd/2]
  s16* X;       // [M, max(d, hq*hd)]: norm output, then attention output
  s16* Q;       // [M, hq*hd]
  s16* Kb;      // [T_kv, hkv*hd]
  s16* Vb;      // [T_kv, hkv*hd]
  s16* Act;     // [max(M*F, (T_kv-M)*d)]: SwiGLU output; halt-mode frozen-row norms
  float* ssq_u;  // [o_proj tiles, M]
  float* ssq_h;
  float* rs;     // [max(M, T_kv - M)] RMSNorm 1/rms per row, applied in the GEMM epilogues
  int64_t rope_rows;  // positions held by the RoPE table
};

bool dims_ok(const dash_dims* D) {
  if (!D) return false;
  const int d = D->d_model, hq = D->n_heads, hkv = D->n_kv_heads, hd = D->head_dim, F = D->ffn_dim;
  if (D->n_layers <= 0 || d <= 0 || hq <= 0 || hkv <= 0 || F <= 0) return false;
  if (hd != 64 && hd != 128) return false;
  if (hq % hkv != 0) return false;
  if (d % 128 != 0 || d > 4096 || F % 64 != 0 || (hq * hd) % 128 != 0) return false;
  if (!(D->rms_eps >= 0.0) || !(D->rope_theta > 0.0)) return false;
  if (D->dtype != DASH_DTYPE_BF16 && D->dtype != DASH_DTYPE_F16) return false;
  return true;
}

void carve_layer(const dash_dims& D, int64_t M, int64_t T_kv, int64_t max_pos, Carver& c, LayerWs& w) {
  const int64_t d = D.d_model, qd = static_cast<int64_t>(D.n_heads) * D.head_dim;
  const int64_t kvd = static_cast<int64_t>(D.n_kv_heads) * D.head_dim, F = D.ffn_dim;
  w.rope = c.take<float2>(static_cast<size_t>(max_pos) * (D.head_dim / 2));
  w.rope_rows = max_pos;
  w.X = c.take<s16>(static_cast<size_t>(M) * (d > qd ? d : qd));
  w.Q = c.take<s16>(static_cast<size_t>(M) * qd);
  w.Kb = c.take<s16>(static_cast<size_t>(T_kv) * kvd);
  w.Vb = c.take<s16>(static_cast<size_t>(T_kv) * kvd);
  const int64_t act = M * F > (T_kv - M) * d ? M * F : (T_kv - M) * d;
  w.Act = c.take<s16>(static_cast<size_t>(act));
  const int nt = o_proj_tiles(D.d_model);
  w.ssq_u = c.take<float>(static_cast<size_t>(nt) * M);
  w.ssq_h = c.take<float>(static_cast<size_t>(nt) * M);
  w.rs = c.take<float>(static_cast<size_t>(M > T_kv - M ? M : T_kv - M));
}

// One pre-norm decoder block on H [M, d] in place (rope table already built).
// pos: RoPE position of each row (NULL: row index); kstart: first key each
// row may attend to (NULL: 0; varlen batches); halted_pos: RoPE positions of
// the halted rows (NULL: their original index).
template <int DT>
dash_status layer_impl(const DeviceInfo& di, const dash_dims& D, const dash_layer_weights& w, s16* H, int64_t M,
                       const int32_t* pos, const dash_halt_ctx* halt, float* delta, int relative,
                       const LayerWs& ws, cudaStream_t st, const int32_t* kstart = nullptr,
                       const int32_t* halted_pos = nullptr, int delta_accumulate = 0) {
  if (M == 0) return DASH_OK;
  const int d = D.d_model, hq = D.n_heads, hkv = D.n_kv_heads, hd = D.head_dim, F = D.ffn_dim;
  const int qd = hq * hd, kvd = hkv * hd;
  const int64_t T_kv = halt ? halt->T : M;
  dash_status s;

  EpiArgs qkv{};
  qkv.q = ws.Q;
  qkv.k = ws.Kb;
  qkv.v = ws.Vb;
  qkv.ldq = qd;
  qkv.ldkv = kvd;
  qkv.rope = reinterpret_cast<const float4*>(ws.rope);
  qkv.hq = hq;
  qkv.hkv = hkv;
  qkv.hd = hd;
  qkv.rope_rows = ws.rope_rows;
  qkv.kv_rows = T_kv;

  // Keys / values of the halted rows, from their frozen states, at their
  // original positions ([DASH news] "选择性停止机制").
  if (halt && T_kv > M) {
    const int64_t nh = T_kv - M;
    if ((s = rmsnorm<DT>(cb(halt->h_full), T_kv, halt->halted_idx, nh, d, cb(w.attn_norm), D.rms_eps, ws.Act, st,
                     ws.rs)) != DASH_OK)
      return s;
    EpiArgs kv = qkv;
    kv.row_scale = ws.rs;
    kv.q = nullptr;
    kv.pos = halted_pos ? halted_pos : halt->halted_idx;
    kv.kv_rowmap = halt->halted_idx;
    kv.col_offset = qd;
    if ((s = gemm<dash::gemm::kEpiQkv, DT>(di, ws.Act, d, nh, d, cb(w.w_qkv) + static_cast<int64_t>(qd) * d, nullptr,
                                       2 * kvd, kv, st, DASH_K_GEMM_KV_HALTED)) != DASH_OK)
      return s;
  }

  // a1: input RMSNorm (its 1/rms is applied to the QKV accumulator)
  if ((s = rmsnorm<DT>(H, M, nullptr, M, d, cb(w.attn_norm), D.rms_eps, ws.X, st, ws.rs)) != DASH_OK) return s;
  // a2: QKV projection + RoPE (k/v of active rows land at their original rows in halt mode)
  qkv.row_scale = ws.rs;
  qkv.pos = pos;
  qkv.kv_rowmap = halt ? halt->active_idx : nullptr;
  qkv.col_offset = 0;
  if ((s = gemm<dash::gemm::kEpiQkv, DT>(di, ws.X, d, M, d, cb(w.w_qkv), nullptr, qd + 2 * kvd, qkv, st, DASH_K_GEMM_QKV)) != DASH_OK)
    return s;
  // a3: causal GQA attention -> O (into X)
  if ((s = attention<DT>(ws.Q, qd, ws.Kb, ws.Vb, kvd, M, T_kv, hq, hkv, hd, halt ? halt->active_idx : nullptr, kstart,
                     ws.X, qd, st)) != DASH_OK)
    return s;
  // a4: o_proj + residual (+ per-row sums of U^2 and H^2 for Δ)
  EpiArgs o{};
  o.out = H;
  o.ldo = d;
  o.ssq_u = ws.ssq_u;
  o.ssq_h = ws.ssq_h;
  int bn = 0;
  if (delta)
    s = gemm<dash::gemm::kEpiResidSsq, DT>(di, ws.X, qd, M, qd, cb(w.w_o), nullptr, d, o, st, DASH_K_GEMM_O, &bn);
  else
    s = gemm<dash::gemm::kEpiResid, DT>(di, ws.X, qd, M, qd, cb(w.w_o), nullptr, d, o, st, DASH_K_GEMM_O, &bn);
  if (s != DASH_OK) return s;
  if (delta) {
    const int64_t blocks = (M + 255) / 256;
    TimedLaunch tl(DASH_K_SCORE, M, d / bn, 0, st);
    dash::rows::score_from_ssq_kernel<<<static_cast<unsigned>(blocks), 256, 0, st>>>(ws.ssq_u, ws.ssq_h, d / bn,
                                                                                     M, relative, delta_accumulate,
                                                                                     delta);
    if ((s = launch_status()) != DASH_OK) return s;
  }
  // a5: post-attention RMSNorm, gate/up GEMM with SwiGLU
  if ((s = rmsnorm<DT>(H, M, nullptr, M, d, cb(w.ffn_norm), D.rms_eps, ws.X, st, ws.rs)) != DASH_OK) return s;
  EpiArgs sw{};
  sw.out = ws.Act;
  sw.ldo = F;
  sw.row_scale = ws.rs;
  if ((s = gemm<dash::gemm::kEpiSwiglu, DT>(di, ws.X, d, M, d, cb(w.w_gate), cb(w.w_up), 2 * F, sw, st, DASH_K_GEMM_GATE_UP)) != DASH_OK) return s;
  // a6: down projection + residual
  EpiArgs dn{};
  dn.out = H;
  dn.ldo = d;
  return gemm<dash::gemm::kEpiResid, DT>(di, ws.Act, F, M, F, cb(w.w_down), nullptr, d, dn, st, DASH_K_GEMM_DOWN);
}

// The decoder block in the model's 16-bit format (dims.dtype).
template <typename... A>
dash_status layer_fmt(const DeviceInfo& di, const dash_dims& D, A&&... a) {
  if (D.dtype == DASH_DTYPE_F16) return layer_impl<kF16>(di, D, std::forward<A>(a)...);
  return layer_impl<kBf16>(di, D, std::forward<A>(a)...);
}

bool weights_ok(const dash_layer_weights* w) {
  return w && w->attn_norm && w->w_qkv && w->w_o && w->ffn_norm && w->w_gate && w->w_up && w->w_down &&
         aligned16(w->attn_norm) && aligned16(w->w_qkv) && aligned16(w->w_o) && aligned16(w->ffn_norm) &&
         aligned16(w->w_gate) && aligned16(w->w_up) && aligned16(w->w_down);
}

// Scratch of the multi-SM selection of one sequence (none for varlen
// batches, whose sequences each take one CTA).
struct SelWs {
  dash::rows::SelState* st = nullptr;
  uint32_t* cand_key = nullptr;
  int32_t* cand_idx = nullptr;
  uint32_t* chunk = nullptr;  // 6 arrays of n_chunks entries
  int64_t n_chunks = 0;
};

void carve_select(int64_t T, Carver& c, SelWs& w) {
  namespace r = dash::rows;
  w.n_chunks = (T + r::kSelCtaTok - 1) / r::kSelCtaTok;
  w.st = c.take<r::SelState>(1);
  w.cand_key = c.take<uint32_t>(static_cast<size_t>(T > 0 ? T : 1));
  w.cand_idx = c.take<int32_t>(static_cast<size_t>(T > 0 ? T : 1));
  w.chunk = c.take<uint32_t>(static_cast<size_t>(6 * (w.n_chunks > 0 ? w.n_chunks : 1)));
}

struct PrefillWs {
  LayerWs L;
  SelWs sel_ws;     // single-sequence selection scratch
  s16* Hc;         // [T, d] compacted active rows
  float* delta;     // [T]
  int32_t* idx;     // [T]
  int32_t* halted;  // [T]
  int32_t* count;   // [nseq]
  // varlen batches only (nseq > 1 or a sequence layout given)
  int32_t* cu;      // [nseq + 1] sequence starts
  int32_t* cuc;     // [nseq + 1] sequence starts among the active rows
  int32_t* sel;     // [T] per-sequence selection regions before packing
  int32_t* selh;    // [T]
  int32_t* pos;     // [T] RoPE positions of the current rows
  int32_t* kst;     // [T] first visible key of the current rows
  int32_t* hpos;    // [T] RoPE positions of halted rows
};

void carve_prefill(const dash_dims& D, int64_t T, int nseq, Carver& c, PrefillWs& w) {
  carve_layer(D, T, T, T, c, w.L);
  w.Hc = c.take<s16>(static_cast<size_t>(T) * D.d_model);
  w.delta = c.take<float>(static_cast<size_t>(T));
  w.idx = c.take<int32_t>(static_cast<size_t>(T));
  w.halted = c.take<int32_t>(static_cast<size_t>(T));
  w.count = c.take<int32_t>(static_cast<size_t>(nseq > 0 ? nseq : 1));
  const bool varlen = nseq > 1;
  w.cu = varlen ? c.take<int32_t>(static_cast<size_t>(nseq) + 1) : nullptr;
  w.cuc = varlen ? c.take<int32_t>(static_cast<size_t>(nseq) + 1) : nullptr;
  w.sel = varlen ? c.take<int32_t>(static_cast<size_t>(T)) : nullptr;
  w.selh = varlen ? c.take<int32_t>(static_cast<size_t>(T)) : nullptr;
  w.pos = varlen ? c.take<int32_t>(static_cast<size_t>(T)) : nullptr;
  w.kst = varlen ? c.take<int32_t>(static_cast<size_t>(T)) : nullptr;
  w.hpos = varlen ? c.take<int32_t>(static_cast<size_t>(T)) : nullptr;
  if (!varlen) carve_select(T, c, w.sel_ws);
}

// Selection ([DASH blog] §3.1; threshold form from [DASH news]).  One
// sequence (seg == NULL): the multi-SM kernels over sel's scratch; nseg
// sequences of a varlen batch (seg = their starts on the device): one CTA each.
dash_status select_impl(const float* scores, int64_t T, const int32_t* seg, int nseg, int kind, double keep,
                        float thr, int keep_first, int keep_last, int32_t* idx, int32_t* halted, int32_t* count,
                        const SelWs* sel, const DeviceInfo& di, cudaStream_t st) {
  (void)di;
  namespace r = dash::rows;
  if (T == 0 || nseg == 0)
    return cudaMemsetAsync(count, 0, sizeof(int32_t) * (nseg > 0 ? nseg : 1), st) == cudaSuccess ? DASH_OK
                                                                                            : DASH_ERR_CUDA;
  // the same middle range, k and mode as select_kernel computes on the device
  const int64_t lo = keep_first < T ? keep_first : T;
  int64_t hi = keep_last > 0 ? T - keep_last : T;
  if (hi < lo) hi = lo;
  const int64_t k_dyn = kind == DASH_SELECT_TOPK ? static_cast<int64_t>(std::floor(keep * static_cast<double>(hi - lo)))
                                                  : 0;
  const int mode = kind == DASH_SELECT_THRESHOLD ? 3 : (k_dyn <= 0 ? 0 : (k_dyn >= hi - lo ? 1 : 2));
  // one CTA per sequence, or the multi-SM passes (the histogram only for a top-k cut)
  TimedLaunch tl(DASH_K_SELECT, T, nseg, 0, st, seg ? 1 : (mode == 2 ? 4 : 3));
  if (seg) {
    r::select_kernel<<<nseg, r::kSelThreads, 0, st>>>(scores, T, seg, kind, keep, thr, keep_first, keep_last, idx,
                                                      halted, count);
    return launch_status();
  }
  if (!sel || !sel->st) return DASH_ERR_NO_MEMORY;
  r::SelArgs a;
  a.scores = scores;
  a.T = T;
  a.lo = lo;
  a.hi = hi;
  a.k_dyn = k_dyn;
  a.mode = mode;
  a.thr = thr;
  a.n_chunks = sel->n_chunks;
  a.st = sel->st;
  a.cand_key = sel->cand_key;
  a.cand_idx = sel->cand_idx;
  const int64_t G = sel->n_chunks;
  a.n_flag = sel->chunk;
  a.gt_extra = sel->chunk + G;
  a.eq_cnt = sel->chunk + 2 * G;
  a.sel_off = sel->chunk + 3 * G;
  a.hal_off = sel->chunk + 4 * G;
  a.eq_before = sel->chunk + 5 * G;
  a.idx = idx;
  a.halted = halted;
  a.count = count;
  if (cudaMemsetAsync(sel->st, 0, offsetof(r::SelState, kth), st) != cudaSuccess) return DASH_ERR_CUDA;
  const unsigned grid = static_cast<unsigned>(G);
  if (a.mode == 2) r::sel_hist_kernel<<<grid, r::kSelCtaThreads, 0, st>>>(a);
  r::sel_scan_kernel<<<grid, r::kSelCtaThreads, 0, st>>>(a);
  r::sel_resolve_kernel<<<1, r::kResolveThreads, 0, st>>>(a);
  r::sel_compact_kernel<<<grid, r::kSelCtaThreads, 0, st>>>(a);
  return launch_status();
}

dash_status seq_layout(const int32_t* cu, int nseq, const int32_t* rows, int64_t M, const int32_t* kspace,
                       int32_t* pos, int32_t* kstart, const DeviceInfo& di, cudaStream_t st) {
  if (M == 0) return DASH_OK;
  int64_t blocks = (M + 255) / 256;
  if (blocks > di.num_sms * 8) blocks = di.num_sms * 8;
  dash::rows::seq_layout_kernel<<<static_cast<unsigned>(blocks), 256, 0, st>>>(cu, nseq, rows, M, kspace, pos,
                                                                               kstart);
  return launch_status();
}

// Scratch of dash_layer_forward_noalloc: a file-scope device array, so that
// entry point never allocates.  Every GPU that loads the library holds it
// until the process exits.  In host code the array's name is only a
// host-side stand-in; its device address comes from cudaGetSymbolAddress.
constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;
__device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of g_noalloc_scratch on the current device, looked up on
// every call (cheap; allocates nothing), so it stays valid across a device
// reset or a re-created primary context.
dash_status noalloc_scratch(void** out) {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return DASH_ERR_CUDA;
  *out = p;
  return DASH_OK;
}

// A wait that nothing will ever satisfy: the bounded wait must give up,
// record kDevErrTimeout and let the kernel return (the failure path of every
// pipelined kernel, exercised without faulting the GPU).
__global__ void wait_timeout_selftest_kernel(int* done) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    dash::mbar_init(dash::smem_u32(&bar), 1);
    dash::fence_mbar_init();
  }
  __syncthreads();
  const bool ok = dash::mbar_wait(dash::smem_u32(&bar), 0);
  if (threadIdx.x == 0) done[0] = ok ? 1 : 2;
}

__global__ void exp2_fma_kernel(const float* __restrict__ x, int64_t n, float* __restrict__ y) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    y[i] = dash::attn::ex2_fma(x[i]);
}


// ---------------------------------------------------------------- KV cache
dash_status kv_store(const s16* Kb, const s16* Vb, int kvd, int64_t a, int64_t rows, const int32_t* pos_src,
                     const dash_kv_cache& c, const DeviceInfo& di, cudaStream_t st) {
  if (rows == 0) return DASH_OK;
  const int warps = 8;
  int64_t blocks = (rows + warps - 1) / warps;
  const int64_t cap = static_cast<int64_t>(di.num_sms) * 16;
  if (blocks > cap) blocks = cap;
  TimedLaunch tl(DASH_K_KV_STORE, rows, kvd, 0, st);
  dash::decode::kv_store_kernel<<<static_cast<unsigned>(blocks), 32 * warps, 0, st>>>(
      Kb, Vb, kvd, a, rows, pos_src, reinterpret_cast<s16*>(c.k), reinterpret_cast<s16*>(c.v), c.pos);
  return launch_status();
}

bool cache_ok(const dash_kv_cache& c) {
  return c.k && c.v && aligned16(c.k) && aligned16(c.v) && c.capacity >= 0 && c.len >= 0 && c.len <= c.capacity &&
         (!c.pos || (reinterpret_cast<uintptr_t>(c.pos) & 3u) == 0);
}

// Capacities a prefill needs: every layer holds its sequence's T_s rows,
// except the layers after L_s in prune mode, which hold K_s rows (known here
// for top-k selection; checked after the selection for threshold selection).
dash_status check_prefill_caches(const dash_dims& D, const dash_config& cfg, const int32_t* cu, int nseq,
                                 const dash_kv_cache* caches) {
  for (int q = 0; q < nseq; ++q) {
    const int64_t Tq = cu[q + 1] - cu[q];
    for (int l = 0; l < D.n_layers; ++l) {
      const dash_kv_cache& c = caches[static_cast<size_t>(q) * D.n_layers + l];
      if (!cache_ok(c)) return DASH_ERR_INVALID_ARG;
      int64_t need = Tq;
      if (cfg.mode == DASH_MODE_PRUNE && l > cfg.halt_layer)
        need = cfg.select == DASH_SELECT_TOPK ? dash_topk_count(Tq, cfg.keep_ratio, cfg.keep_first, cfg.keep_last)
                                              : 0;
      if (c.capacity < need) return DASH_ERR_SHAPE;
    }
  }
  return DASH_OK;
}

dash_status check_config(const dash_dims* dims, const dash_config* cfg) {
  if (cfg->mode != DASH_MODE_PRUNE && cfg->mode != DASH_MODE_HALT && cfg->mode != DASH_MODE_DENSE)
    return DASH_ERR_INVALID_ARG;
  if (cfg->mode != DASH_MODE_DENSE) {
    if (cfg->halt_layer < 0 || cfg->halt_layer >= dims->n_layers) return DASH_ERR_INVALID_ARG;
    if (cfg->select != DASH_SELECT_TOPK && cfg->select != DASH_SELECT_THRESHOLD) return DASH_ERR_INVALID_ARG;
    if (cfg->score != DASH_SCORE_ABS && cfg->score != DASH_SCORE_REL) return DASH_ERR_INVALID_ARG;
    if (cfg->select == DASH_SELECT_TOPK && !(cfg->keep_ratio >= 0.0 && cfg->keep_ratio <= 1.0))
      return DASH_ERR_INVALID_ARG;
    if (cfg->keep_first < 0 || cfg->keep_last < 0) return DASH_ERR_INVALID_ARG;
    if (cfg->monitor_layers < 0 || cfg->monitor_layers > cfg->halt_layer + 1) return DASH_ERR_INVALID_ARG;
  }
  return DASH_OK;
}

// Single-shot DASH prefill over nseq independent sequences concatenated in H
// (sequence s = rows [cu[s], cu[s+1]), cu in host memory): block-diagonal
// causal attention, RoPE positions counted from each sequence's start, and a
// separate selection per sequence ([DASH blog] §5.1: decisions are made per
// sample).  nseq == 1 is the plain single-sequence prefill.
dash_status prefill_impl(const dash_dims* dims, const dash_layer_weights* layers, dash_bf16* H, const int32_t* cu,
                         int nseq, const dash_config* cfg, int32_t* idx_out, int64_t* K_out, int32_t* seq_counts,
                         float* delta_out, void* ws, size_t ws_bytes, void* stream,
                         dash_kv_cache* caches = nullptr) {
  if (!dims_ok(dims)) return DASH_ERR_SHAPE;
  if (!layers || !H || !cfg || !aligned16(H)) return DASH_ERR_INVALID_ARG;
  const int64_t T = cu[nseq];
  if (T < 0 || T > INT32_MAX) return DASH_ERR_SHAPE;
  dash_status s = check_config(dims, cfg);
  if (s != DASH_OK) return s;
  for (int l = 0; l < dims->n_layers; ++l)
    if (!weights_ok(&layers[l])) return DASH_ERR_INVALID_ARG;
  if (caches && (s = check_prefill_caches(*dims, *cfg, cu, nseq, caches)) != DASH_OK) return s;
  if (T == 0) {
    if (caches)
      for (int q = 0; q < nseq * dims->n_layers; ++q) caches[q].len = 0;
    if (K_out) *K_out = 0;
    if (seq_counts)
      for (int q = 0; q < nseq; ++q) seq_counts[q] = 0;
    return DASH_OK;
  }
  Carver probe{nullptr};
  PrefillWs sizes;
  carve_prefill(*dims, T, nseq, probe, sizes);
  if (!ws || ws_bytes < probe.off + 256) return DASH_ERR_NO_MEMORY;
  DeviceInfo* di;
  if ((s = device_info(&di)) != DASH_OK) return s;
  Carver c{reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(ws) + 255) & ~static_cast<uintptr_t>(255))};
  PrefillWs P;
  carve_prefill(*dims, T, nseq, c, P);
  cudaStream_t st = as_stream(stream);
  s16* h = reinterpret_cast<s16*>(H);
  const dash_dims& D = *dims;
  const bool varlen = nseq > 1;
  if ((s = rope_table(P.L.rope, T, D.head_dim, D.rope_theta, *di, st)) != DASH_OK) return s;

  // Row layout of the full sequence(s): RoPE positions and key starts.
  const int32_t* pos_full = nullptr;
  const int32_t* kst_full = nullptr;
  if (varlen) {
    if (cudaMemcpyAsync(P.cu, cu, sizeof(int32_t) * (nseq + 1), cudaMemcpyHostToDevice, st) != cudaSuccess)
      return DASH_ERR_CUDA;
    if ((s = seq_layout(P.cu, nseq, nullptr, T, nullptr, P.pos, P.kst, *di, st)) != DASH_OK) return s;
    pos_full = P.pos;
    kst_full = P.kst;
  }

  // KV cache rows of each sequence after a layer: kv_start/kv_rows index the
  // layer's K/V buffers; kv_pos (NULL: row order) gives their positions.
  std::vector<int64_t> kv_start(static_cast<size_t>(nseq)), kv_rows(static_cast<size_t>(nseq));
  for (int q = 0; q < nseq; ++q) {
    kv_start[q] = cu[q];
    kv_rows[q] = cu[q + 1] - cu[q];
  }
  const int32_t* kv_pos = nullptr;

  // Δ is taken at the layers [delta_first, delta_last] and combined by maximum.
  auto run_layers = [&](int l0, int l1, s16* rows, int64_t M, const int32_t* pos, const dash_halt_ctx* hc,
                        const int32_t* kst, const int32_t* hpos, int delta_first, int delta_last,
                        float* delta) -> dash_status {
    for (int l = l0; l < l1; ++l) {
      g_timing.layer = l;
      const bool take = l >= delta_first && l <= delta_last;
      dash_status r = layer_fmt(*di, D, layers[l], rows, M, pos, hc, take ? delta : nullptr,
                                 cfg->score == DASH_SCORE_REL, P.L, st, kst, hpos, l > delta_first ? 1 : 0);
      for (int q = 0; r == DASH_OK && caches && q < nseq; ++q) {
        dash_kv_cache& c = caches[static_cast<size_t>(q) * D.n_layers + l];
        r = kv_store(P.L.Kb, P.L.Vb, D.n_kv_heads * D.head_dim, kv_start[q], kv_rows[q], kv_pos, c, *di, st);
        c.len = kv_rows[q];
      }
      g_timing.layer = -1;
      if (r != DASH_OK) return r;
    }
    return DASH_OK;
  };

  if (cfg->mode == DASH_MODE_DENSE) {
    if ((s = run_layers(0, D.n_layers, h, T, pos_full, nullptr, kst_full, nullptr, -1, -1, nullptr)) != DASH_OK)
      return s;
    if (K_out) *K_out = T;
    if (seq_counts)
      for (int q = 0; q < nseq; ++q) seq_counts[q] = cu[q + 1] - cu[q];
    return DASH_OK;
  }

  // Layers 0..L_s on all T tokens; Δ from the halting layer's o_proj epilogue.
  const int Ls = cfg->halt_layer;
  float* delta = delta_out ? delta_out : P.delta;
  const int window = cfg->monitor_layers > 1 ? cfg->monitor_layers : 1;
  if ((s = run_layers(0, Ls + 1, h, T, pos_full, nullptr, kst_full, nullptr, Ls - window + 1, Ls, delta)) != DASH_OK)
    return s;

  // One-shot selection of the active set S*, per sequence.
  int32_t* idx = idx_out ? idx_out : P.idx;
  std::vector<int32_t> counts(static_cast<size_t>(nseq));
  if ((s = select_impl(delta, T, varlen ? P.cu : nullptr, nseq, cfg->select, cfg->keep_ratio, cfg->threshold,
                       cfg->keep_first, cfg->keep_last, varlen ? P.sel : idx, varlen ? P.selh : P.halted, P.count,
                       varlen ? nullptr : &P.sel_ws, *di, st)) != DASH_OK)
    return s;
  if (cudaMemcpyAsync(counts.data(), P.count, sizeof(int32_t) * nseq, cudaMemcpyDeviceToHost, st) != cudaSuccess ||
      cudaStreamSynchronize(st) != cudaSuccess)
    return DASH_ERR_CUDA;
  int64_t K = 0;
  for (int q = 0; q < nseq; ++q) {
    if (counts[q] < 0) return DASH_ERR_NONFINITE;
    K += counts[q];
  }
  if (K_out) *K_out = K;
  if (seq_counts)
    for (int q = 0; q < nseq; ++q) seq_counts[q] = counts[q];
  if (varlen) {
    // Pack the per-sequence regions into contiguous ascending lists.
    std::vector<int32_t> cuc(static_cast<size_t>(nseq) + 1, 0);
    int64_t hoff = 0;
    for (int q = 0; q < nseq; ++q) {
      const int64_t len = cu[q + 1] - cu[q], kq = counts[q];
      cuc[q + 1] = cuc[q] + counts[q];
      if (kq > 0 && cudaMemcpyAsync(idx + cuc[q], P.sel + cu[q], sizeof(int32_t) * kq, cudaMemcpyDeviceToDevice,
                                    st) != cudaSuccess)
        return DASH_ERR_CUDA;
      if (len - kq > 0 && cudaMemcpyAsync(P.halted + hoff, P.selh + cu[q], sizeof(int32_t) * (len - kq),
                                          cudaMemcpyDeviceToDevice, st) != cudaSuccess)
        return DASH_ERR_CUDA;
      hoff += len - kq;
    }
    // (a copy from pageable host memory has consumed its source when it returns)
    if (cudaMemcpyAsync(P.cuc, cuc.data(), sizeof(int32_t) * (nseq + 1), cudaMemcpyHostToDevice, st) != cudaSuccess)
      return DASH_ERR_CUDA;
  }

  // Gather the active rows; later layers run on them only.
  if ((s = move_rows(false, h, P.Hc, idx, K, T, D.d_model, *di, st)) != DASH_OK) return s;
  if (cfg->mode == DASH_MODE_PRUNE) {
    const int32_t* pos_c = idx;  // original positions
    const int32_t* kst_c = nullptr;
    if (varlen) {  // positions within each sequence; keys from the sequence's first active row
      if ((s = seq_layout(P.cu, nseq, idx, K, P.cuc, P.pos, P.kst, *di, st)) != DASH_OK) return s;
      pos_c = P.pos;
      kst_c = P.kst;
    }
    if (caches) {  // later layers cache the active rows only
      int64_t a = 0;
      for (int q = 0; q < nseq; ++q) {
        kv_start[q] = a;
        kv_rows[q] = counts[q];
        a += counts[q];
        for (int l = Ls + 1; l < D.n_layers; ++l)
          if (caches[static_cast<size_t>(q) * D.n_layers + l].capacity < counts[q]) return DASH_ERR_SHAPE;
      }
      kv_pos = pos_c;
    }
    if ((s = run_layers(Ls + 1, D.n_layers, P.Hc, K, pos_c, nullptr, kst_c, nullptr, -1, -1, nullptr)) != DASH_OK)
      return s;
    if (K > 0 && cudaMemcpyAsync(h, P.Hc, static_cast<size_t>(K) * D.d_model * sizeof(s16),
                                 cudaMemcpyDeviceToDevice, st) != cudaSuccess)
      return DASH_ERR_CUDA;
    return DASH_OK;
  }
  dash_halt_ctx hc;
  hc.active_idx = idx;
  hc.halted_idx = P.halted;
  hc.h_full = H;
  hc.T = T;
  const int32_t* pos_a = idx;
  const int32_t* kst_a = nullptr;
  const int32_t* hpos = nullptr;
  if (varlen) {
    if ((s = seq_layout(P.cu, nseq, idx, K, nullptr, P.pos, P.kst, *di, st)) != DASH_OK) return s;
    if ((s = seq_layout(P.cu, nseq, P.halted, T - K, nullptr, P.hpos, nullptr, *di, st)) != DASH_OK) return s;
    pos_a = P.pos;
    kst_a = P.kst;
    hpos = P.hpos;
  }
  if ((s = run_layers(Ls + 1, D.n_layers, P.Hc, K, pos_a, &hc, kst_a, hpos, -1, -1, nullptr)) != DASH_OK) return s;
  return move_rows(true, P.Hc, h, idx, K, T, D.d_model, *di, st);
}


// ------------------------------------------------------------ generation
namespace dec = dash::decode;

struct DecodeWs {
  float* tc_part;    // [kTcMaxItems][128][32] partial sums of split tensor-core GEMVs
  int* tc_counters;  // [kTcMaxItems] (zeroed per step; the kernels leave them zero)
  s16* Q;         // [n, hq*hd]
  s16* O;         // [n, hq*hd] attention output
  s16* Act;       // [n, F]
  float* part_o;   // [kMaxCtas, 16, hd]
  float* part_ml;  // [kMaxCtas, 16, 2]
};

void carve_decode(const dash_dims& D, int n, Carver& c, DecodeWs& w) {
  const size_t qd = static_cast<size_t>(D.n_heads) * D.head_dim;
  w.tc_part = nullptr;  // the tensor-core projections (3 or more sequences) only
  w.tc_counters = nullptr;
  if (n >= dec::kTcMinRows) {
    w.tc_part = c.take<float>(static_cast<size_t>(dec::kTcMaxItems) * dec::kTcRows * 2 * dec::kTcN);
    w.tc_counters = c.take<int>(dec::kTcMaxItems);
  }
  w.Q = c.take<s16>(n * qd);
  w.O = c.take<s16>(n * qd);
  w.Act = c.take<s16>(static_cast<size_t>(n) * D.ffn_dim);
  w.part_o = c.take<float>(static_cast<size_t>(dec::kMaxCtas) * dec::kGroupPad * D.head_dim);
  w.part_ml = c.take<float>(static_cast<size_t>(dec::kMaxCtas) * dec::kGroupPad * 2);
}

// Launch with programmatic dependent launch: the kernel may be scheduled
// while its predecessor on the stream finishes; it waits (griddepcontrol)
// before reading that predecessor's results.
template <typename... ExpTypes, typename... ActTypes>
cudaError_t launch_pdl(void (*kernel)(ExpTypes...), unsigned grid, unsigned block, size_t smem, cudaStream_t st,
                       ActTypes&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(block);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<ActTypes>(args)...);
}

constexpr size_t kGemvSmemMax = 160 * 1024;    // x staged in shared memory up to this size
constexpr size_t kGemvSmemTotal = 224 * 1024;  // staged x + the warps' first-task weight slots

template <int EPI, int NS, int DT>
dash_status launch_gemv_ns(const DeviceInfo& di, const dec::GemvParams& gp, int kind, int64_t n_out,
                           bool preload, cudaStream_t st) {
  if (gp.tasks == 0) return DASH_OK;
  constexpr bool kNorm = EPI != dec::kGvResid;
  const size_t xbytes = static_cast<size_t>(gp.n) * gp.K * 2;
  const bool stage = kNorm || xbytes <= kGemvSmemMax;
  if (kNorm && xbytes > kGemvSmemMax) return DASH_ERR_SHAPE;
  dec::GemvParams q = gp;
  q.stage_x = !kNorm && stage;
  const size_t xs = stage ? xbytes : 0;
  // preload: the rest of shared memory holds two rows' leading bytes per
  // warp, loaded before the PDL wait (whole rows when they fit).  Only for
  // the down projection: a kernel's PDL wait is released after the copies
  // then in flight on the device complete, so behind a short predecessor
  // (the attention merge before o_proj, the down projection before QKV)
  // a preload delays the kernel more than it saves.
  size_t pre = !preload || kNorm ? 0 : (kGemvSmemTotal - xs) / (2 * dec::kGemvWarps) & ~static_cast<size_t>(15);
  if (pre > static_cast<size_t>(gp.K) * 2) pre = static_cast<size_t>(gp.K) * 2;
  if (pre < 1024) pre = 0;
  q.x_smem = static_cast<int>(xs);
  q.pre_bytes = static_cast<int>(pre);
  const size_t smem = xs + 2 * dec::kGemvWarps * pre;
  static std::once_flag attr_once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(attr_once, [] {
    attr_err = cudaFuncSetAttribute(dec::gemv_kernel<EPI, NS, DT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    static_cast<int>(kNorm ? kGemvSmemMax : kGemvSmemTotal));
  });
  if (attr_err != cudaSuccess) return DASH_ERR_CUDA;
  // one CTA per SM (tasks strided over the grid), so every SM streams weights
  const unsigned grid = static_cast<unsigned>(gp.tasks < di.num_sms ? gp.tasks : di.num_sms);
  TimedLaunch tl(kind, gp.n, n_out, gp.K, st);
  if (launch_pdl(dec::gemv_kernel<EPI, NS, DT>, grid, 32 * dec::kGemvWarps, smem, st, q) != cudaSuccess)
    return DASH_ERR_CUDA;
  return launch_status();
}

template <int EPI, int DT>
dash_status launch_gemv_n(const DeviceInfo& di, const dec::GemvParams& gp, int kind, int64_t n_out, cudaStream_t st,
                          bool preload) {
  if (gp.n <= 1) return launch_gemv_ns<EPI, 1, DT>(di, gp, kind, n_out, preload, st);
  if (gp.n <= 2) return launch_gemv_ns<EPI, 2, DT>(di, gp, kind, n_out, preload, st);
  if (gp.n <= 4) return launch_gemv_ns<EPI, 4, DT>(di, gp, kind, n_out, preload, st);
  return launch_gemv_ns<EPI, 8, DT>(di, gp, kind, n_out, preload, st);
}

constexpr size_t kTcSmemBudget = 208 * 1024;  // weight ring + x slice (dynamic shared memory)
bool g_gemv_tc = true;                         // dash_set_decode_tensor_cores

// The tensor-core form (decode_tc.cuh) for gp.n >= kTcMinRows.  Returns
// DASH_ERR_SHAPE, before launching anything, when the shape does not suit it.
template <int EPI, int DT>
dash_status launch_gemv_tc(const DeviceInfo& di, const dec::GemvParams& gp, int kind, int64_t n_out,
                           const DecodeWs& w, cudaStream_t st) {
  using C = dec::TcCfg<EPI>;
  const int R = EPI == dec::kGvSwiglu ? gp.tasks : 2 * gp.tasks;  // weight rows
  if (R % dec::kTcRows != 0 || gp.K % 64 != 0 || gp.n > dec::kTcN) return DASH_ERR_SHAPE;
  if (EPI == dec::kGvQkv && (gp.hd > dec::kTcRows || dec::kTcRows % gp.hd != 0)) return DASH_ERR_SHAPE;
  const int blocks = R / dec::kTcRows, ksteps = gp.K / 64;
  // K ranges per row block: at most one item per SM (a second round on a few
  // SMs would double their time), each range's x slice and a ring of at least
  // two stages within the shared-memory budget
  int splits = 1;
  if (blocks < di.num_sms) splits = std::min(ksteps, di.num_sms / blocks);
  auto slice = [&](int sp) { return static_cast<size_t>((ksteps + sp - 1) / sp) * C::kPanelBytes; };
  while (splits < ksteps && slice(splits) + 2 * C::kStageBytes > kTcSmemBudget) ++splits;
  if (slice(splits) + 2 * C::kStageBytes > kTcSmemBudget) return DASH_ERR_SHAPE;
  if (splits > 1 && blocks * splits > dec::kTcMaxItems) return DASH_ERR_SHAPE;
  const int stages = static_cast<int>(
      std::min<size_t>(dec::kTcMaxStages, (kTcSmemBudget - slice(splits)) / C::kStageBytes));
  const size_t smem = 1024 + static_cast<size_t>(stages) * C::kStageBytes + slice(splits);
  static std::once_flag attr_once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(attr_once, [] {
    attr_err = cudaFuncSetAttribute(dec::gemv_tc_kernel<EPI, DT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    static_cast<int>(1024 + kTcSmemBudget));
  });
  if (attr_err != cudaSuccess) return DASH_ERR_CUDA;
  constexpr CUtensorMapDataType kMt = Num<DT>::kMapType;
  dec::TcMaps maps;
  std::memset(&maps, 0, sizeof(maps));
  if (!make_map(&maps.w, gp.W, static_cast<uint64_t>(R), gp.K, gp.K, dec::kTcRows, kMt)) return DASH_ERR_INVALID_ARG;
  if (EPI == dec::kGvSwiglu && !make_map(&maps.w2, gp.W2, static_cast<uint64_t>(R), gp.K, gp.K, dec::kTcRows, kMt))
    return DASH_ERR_INVALID_ARG;
  dec::TcParams tp;
  std::memset(&tp, 0, sizeof(tp));
  tp.x = gp.x;
  tp.gain = gp.gain;
  tp.eps = gp.eps;
  tp.n = gp.n;
  tp.K = gp.K;
  tp.blocks = blocks;
  tp.splits = splits;
  tp.ksteps = ksteps;
  tp.stages = stages;
  tp.part = w.tc_part;
  tp.counters = w.tc_counters;
  tp.out = gp.out;
  tp.ldo = gp.ldo;
  tp.q = gp.q;
  tp.hq = gp.hq;
  tp.hkv = gp.hkv;
  tp.hd = gp.hd;
  tp.theta = gp.theta;
  tp.seq = gp.seq;
  const int items = blocks * splits;
  const unsigned grid = static_cast<unsigned>(items < di.num_sms ? items : di.num_sms);
  TimedLaunch tl(kind, gp.n, n_out, gp.K, st);
  if (launch_pdl(dec::gemv_tc_kernel<EPI, DT>, grid, dec::kTcThreads, smem, st, maps, tp) != cudaSuccess)
    return DASH_ERR_CUDA;
  return launch_status();
}

template <int EPI, int DT>
dash_status launch_gemv(const DeviceInfo& di, const dec::GemvParams& gp, int kind, int64_t n_out, cudaStream_t st,
                        bool preload = false, const DecodeWs* w = nullptr) {
  // three or more input rows: the tensor-core form when the shape suits it
  if (w && gp.n >= dec::kTcMinRows && g_gemv_tc) {
    const dash_status s = launch_gemv_tc<EPI, DT>(di, gp, kind, n_out, *w, st);
    if (s != DASH_ERR_SHAPE) return s;
  }
  // o_proj / down whose input rows do not all fit in shared memory: one launch
  // per group of rows that does (the weights are read once per group, at the
  // streaming rate; read from global memory per chunk, x cost ~5x more)
  if constexpr (EPI == dec::kGvResid) {
    const int per = static_cast<int>(kGemvSmemMax / (static_cast<size_t>(gp.K) * 2));
    if (gp.n > 1 && per >= 1 && gp.n > per) {
      TimedLaunch tl(kind, gp.n, n_out, gp.K, st, (gp.n + per - 1) / per);
      for (int m0 = 0; m0 < gp.n; m0 += per) {
        dec::GemvParams q = gp;
        q.n = gp.n - m0 < per ? gp.n - m0 : per;
        q.x = gp.x + static_cast<int64_t>(m0) * gp.K;
        q.out = gp.out + static_cast<int64_t>(m0) * gp.ldo;
        const dash_status s = launch_gemv_n<EPI, DT>(di, q, -1, n_out, st, preload);
        if (s != DASH_OK) return s;
      }
      return DASH_OK;
    }
  }
  return launch_gemv_n<EPI, DT>(di, gp, kind, n_out, st, preload);
}

// Split-key decode attention of one layer: the CTA count is held to one
// wave (at most one CTA per SM, at most kMaxCtas) by giving each CTA a run of
// tiles_per_cta key tiles of one (sequence, kv head) segment.
template <int HD, int DT>
dash_status decode_attention_hd(const DeviceInfo& di, const dash_dims& D, int n, const int64_t* len,
                                const dash_kv_cache* const* layer_caches, const DecodeWs& w, cudaStream_t st) {
  using C = dec::ACfg<HD>;
  static std::once_flag attr_once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(attr_once, [] {
    attr_err = cudaFuncSetAttribute(dec::decode_attn_kernel<HD, DT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    C::kSmemBytes);
  });
  if (attr_err != cudaSuccess) return DASH_ERR_CUDA;
  const int hkv = D.n_kv_heads, kvd = hkv * HD;
  dec::AttnMaps maps;
  std::memset(&maps, 0, sizeof(maps));
  dec::AttnParams ap;
  std::memset(&ap, 0, sizeof(ap));
  int64_t total_tiles = 0, max_tiles = 0, keys = 0;
  for (int q = 0; q < n; ++q) {
    const dash_kv_cache& c = *layer_caches[q];
    if (!make_map(&maps.k[q], c.k, static_cast<uint64_t>(len[q]), kvd, kvd, dec::BKV, Num<DT>::kMapType) ||
        !make_map(&maps.v[q], c.v, static_cast<uint64_t>(len[q]), kvd, kvd, dec::BKV, Num<DT>::kMapType))
      return DASH_ERR_INVALID_ARG;
    ap.len[q] = static_cast<int>(len[q]);
    const int64_t t = (len[q] + dec::BKV - 1) / dec::BKV;
    total_tiles += t * hkv;
    max_tiles = t > max_tiles ? t : max_tiles;
    keys += len[q];
  }
  const int64_t cap = di.num_sms < dec::kMaxCtas ? di.num_sms : dec::kMaxCtas;
  int64_t per = (total_tiles + cap - 1) / cap;
  if (per < 1) per = 1;
  auto ctas_for = [&](int64_t tpc) {
    int64_t c = 0;
    for (int q = 0; q < n; ++q) c += hkv * (((len[q] + dec::BKV - 1) / dec::BKV + tpc - 1) / tpc);
    return c;
  };
  while (ctas_for(per) > cap && per < max_tiles) ++per;
  const int64_t nctas = ctas_for(per);
  if (nctas > dec::kMaxCtas) return DASH_ERR_SHAPE;
  int c0 = 0;
  for (int q = 0; q < n; ++q) {
    const int64_t chunks = ((len[q] + dec::BKV - 1) / dec::BKV + per - 1) / per;
    for (int h = 0; h < hkv; ++h) {
      ap.seg_cta0[q * hkv + h] = c0;
      c0 += static_cast<int>(chunks);
    }
  }
  ap.seg_cta0[n * hkv] = c0;
  ap.q = w.Q;
  ap.out = w.O;
  ap.part_o = w.part_o;
  ap.part_ml = w.part_ml;
  ap.n = n;
  ap.hq = D.n_heads;
  ap.hkv = hkv;
  ap.group = D.n_heads / hkv;
  ap.tiles_per_cta = static_cast<int>(per);
  ap.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(HD)));
  dec::MergeParams mp;
  std::memset(&mp, 0, sizeof(mp));
  mp.part_o = w.part_o;
  mp.part_ml = w.part_ml;
  mp.out = w.O;
  mp.n = n;
  mp.hq = D.n_heads;
  mp.hkv = hkv;
  mp.group = ap.group;
  mp.hd = HD;
  mp.items = n * hkv * ap.group * (HD / 32);
  std::memcpy(mp.seg_cta0, ap.seg_cta0, sizeof(mp.seg_cta0));
  TimedLaunch tl(DASH_K_DEC_ATTENTION, n, keys, nctas, st, 2);
  if (launch_pdl(dec::decode_attn_kernel<HD, DT>, static_cast<unsigned>(nctas), dec::kAttnThreads, C::kSmemBytes, st,
                 maps, ap) != cudaSuccess)
    return DASH_ERR_CUDA;
  // The merge is launched in plain stream order (it starts once the attention
  // has completed).  Launched with PDL it was resident early, and o_proj's
  // CTAs, which cannot start before the attention grid completes, then
  // started ~3 us after the attention's CTAs exited and the merge's wait was
  // released ~4 us after the attention ended; the step measured 2% slower.
  const unsigned mgrid = static_cast<unsigned>((mp.items + dec::kMergeWarps - 1) / dec::kMergeWarps);
  dec::decode_merge_kernel<DT><<<mgrid, 32 * dec::kMergeWarps, 0, st>>>(mp);
  if (cudaGetLastError() != cudaSuccess) return DASH_ERR_CUDA;
  return launch_status();
}

template <int DT>
dash_status decode_impl(const dash_dims* dims, const dash_layer_weights* layers, dash_bf16* X, int n,
                        const int32_t* pos, dash_kv_cache* caches, void* ws, size_t ws_bytes, void* stream) {
  if (!dims_ok(dims)) return DASH_ERR_SHAPE;
  const dash_dims& D = *dims;
  if (n < 1 || n > dec::kMaxSeq) return DASH_ERR_SHAPE;
  if (D.n_heads / D.n_kv_heads > dec::kGroupPad || n * D.n_kv_heads > dec::kMaxSegs) return DASH_ERR_SHAPE;
  if (!layers || !X || !aligned16(X) || !pos || !caches) return DASH_ERR_INVALID_ARG;
  for (int l = 0; l < D.n_layers; ++l)
    if (!weights_ok(&layers[l])) return DASH_ERR_INVALID_ARG;
  for (int q = 0; q < n; ++q) {
    if (pos[q] < 0) return DASH_ERR_INVALID_ARG;
    for (int l = 0; l < D.n_layers; ++l) {
      const dash_kv_cache& c = caches[static_cast<size_t>(q) * D.n_layers + l];
      if (!cache_ok(c)) return DASH_ERR_INVALID_ARG;
      if (c.len >= c.capacity || c.len + 1 > INT32_MAX) return DASH_ERR_SHAPE;
    }
  }
  Carver probe{nullptr};
  DecodeWs sizes;
  carve_decode(D, n, probe, sizes);
  if (!ws || ws_bytes < probe.off + 256) return DASH_ERR_NO_MEMORY;
  DeviceInfo* di;
  dash_status s = device_info(&di);
  if (s != DASH_OK) return s;
  if (di->num_sms < dec::kMaxSegs) return DASH_ERR_SHAPE;
  Carver c{reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(ws) + 255) & ~static_cast<uintptr_t>(255))};
  DecodeWs w;
  carve_decode(D, n, c, w);
  cudaStream_t st = as_stream(stream);
  s16* x = reinterpret_cast<s16*>(X);
  const int d = D.d_model, hq = D.n_heads, hkv = D.n_kv_heads, hd = D.head_dim, F = D.ffn_dim;
  const int qd = hq * hd;
  if (n >= dec::kTcMinRows &&
      cudaMemsetAsync(w.tc_counters, 0, sizeof(int) * dec::kTcMaxItems, st) != cudaSuccess)
    return DASH_ERR_CUDA;

  for (int l = 0; l < D.n_layers; ++l) {
    g_timing.layer = l;
    const dash_layer_weights& lw = layers[l];
    const dash_kv_cache* lc[dec::kMaxSeq];
    int64_t len[dec::kMaxSeq];
    dec::GemvParams qkv;
    std::memset(&qkv, 0, sizeof(qkv));
    for (int q = 0; q < n; ++q) {
      lc[q] = &caches[static_cast<size_t>(q) * D.n_layers + l];
      qkv.seq.k[q] = reinterpret_cast<s16*>(lc[q]->k);
      qkv.seq.v[q] = reinterpret_cast<s16*>(lc[q]->v);
      qkv.seq.pos[q] = lc[q]->pos;
      qkv.seq.row[q] = lc[q]->len;
      qkv.seq.p[q] = pos[q];
      len[q] = lc[q]->len + 1;
    }
    // RMSNorm (fused) -> QKV with RoPE, appended to the caches
    qkv.W = cb(lw.w_qkv);
    qkv.x = x;
    qkv.gain = cb(lw.attn_norm);
    qkv.eps = static_cast<float>(D.rms_eps);
    qkv.n = n;
    qkv.K = d;
    qkv.tasks = (hq + 2 * hkv) * hd / 2;
    qkv.q = w.Q;
    qkv.hq = hq;
    qkv.hkv = hkv;
    qkv.hd = hd;
    qkv.theta = D.rope_theta;
    if ((s = launch_gemv<dec::kGvQkv, DT>(*di, qkv, DASH_K_DEC_GEMV_QKV, qd + 2 * hkv * hd, st, false, &w)) !=
        DASH_OK)
      break;
    // attention over each sequence's cache (including the new row)
    s = hd == 128 ? decode_attention_hd<128, DT>(*di, D, n, len, lc, w, st)
                  : decode_attention_hd<64, DT>(*di, D, n, len, lc, w, st);
    if (s != DASH_OK) break;
    // o_proj + residual
    dec::GemvParams o;
    std::memset(&o, 0, sizeof(o));
    o.W = cb(lw.w_o);
    o.x = w.O;
    o.n = n;
    o.K = qd;
    o.tasks = d / 2;
    o.out = x;
    o.ldo = d;
    if ((s = launch_gemv<dec::kGvResid, DT>(*di, o, DASH_K_DEC_GEMV_O, d, st, false, &w)) != DASH_OK) break;
    // RMSNorm (fused) -> gate/up with SwiGLU
    dec::GemvParams gu;
    std::memset(&gu, 0, sizeof(gu));
    gu.W = cb(lw.w_gate);
    gu.W2 = cb(lw.w_up);
    gu.x = x;
    gu.gain = cb(lw.ffn_norm);
    gu.eps = static_cast<float>(D.rms_eps);
    gu.n = n;
    gu.K = d;
    gu.tasks = F;
    gu.out = w.Act;
    gu.ldo = F;
    if ((s = launch_gemv<dec::kGvSwiglu, DT>(*di, gu, DASH_K_DEC_GEMV_GATE_UP, 2 * F, st, false, &w)) != DASH_OK)
      break;
    // down + residual
    dec::GemvParams dn;
    std::memset(&dn, 0, sizeof(dn));
    dn.W = cb(lw.w_down);
    dn.x = w.Act;
    dn.n = n;
    dn.K = F;
    dn.tasks = d / 2;
    dn.out = x;
    dn.ldo = d;
    if ((s = launch_gemv<dec::kGvResid, DT>(*di, dn, DASH_K_DEC_GEMV_DOWN, d, st, true, &w)) != DASH_OK) break;
    for (int q = 0; q < n; ++q) caches[static_cast<size_t>(q) * D.n_layers + l].len += 1;
  }
  g_timing.layer = -1;
  return s;
}
}  // namespace

// =================================================================== C ABI
extern "C" {

const char* dash_status_string(dash_status s) {
  switch (s) {
    case DASH_OK: return "ok";
    case DASH_ERR_INVALID_ARG: return "invalid argument";
    case DASH_ERR_SHAPE: return "unsupported shape";
    case DASH_ERR_NONFINITE: return "non-finite score";
    case DASH_ERR_NO_MEMORY: return "workspace too small";
    case DASH_ERR_CUDA: return "CUDA error";
    case DASH_ERR_TIMEOUT: return "device wait timed out";
    case DASH_ERR_INDEX: return "index out of range";
  }
  return "unknown status";
}

dash_status dash_device_error(void) {
  if (cudaDeviceSynchronize() != cudaSuccess) return DASH_ERR_CUDA;
  unsigned v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, dash::g_dash_dev_error, sizeof(v)) != cudaSuccess) return DASH_ERR_CUDA;
  if (v && cudaMemcpyToSymbol(dash::g_dash_dev_error, &zero, sizeof(zero)) != cudaSuccess) return DASH_ERR_CUDA;
  if (v & dash::kDevErrTimeout) return DASH_ERR_TIMEOUT;
  if (v & dash::kDevErrIndex) return DASH_ERR_INDEX;
  if (v & dash::kDevErrNonfinite) return DASH_ERR_NONFINITE;
  return DASH_OK;
}

dash_status dash_score(const dash_bf16* U, const dash_bf16* H, int64_t T, int32_t d, int32_t relative, float* delta,
                       void* stream) {
  if (T < 0 || d <= 0 || d % 8 != 0) return DASH_ERR_SHAPE;
  if (T == 0) return DASH_OK;
  if (!U || !delta || (relative && !H) || !aligned16(U) || (relative && !aligned16(H))) return DASH_ERR_INVALID_ARG;
  const int warps = 8;
  const int64_t blocks = (T + warps - 1) / warps;
  TimedLaunch tl(DASH_K_SCORE, T, d, relative ? 1 : 0, as_stream(stream));
  dash::rows::score_kernel<kBf16><<<static_cast<unsigned>(blocks), 32 * warps, 0, as_stream(stream)>>>(
      reinterpret_cast<const s16*>(U), reinterpret_cast<const s16*>(H), T, d, relative ? 1 : 0, delta);
  return launch_status();
}

int64_t dash_topk_count(int64_t T, double keep_ratio, int32_t keep_first, int32_t keep_last) {
  if (T <= 0) return 0;
  const int64_t lo = keep_first > 0 ? (keep_first < T ? keep_first : T) : 0;
  int64_t hi = keep_last > 0 ? T - keep_last : T;
  if (hi < lo) hi = lo;
  return (T - (hi - lo)) + static_cast<int64_t>(std::floor(keep_ratio * static_cast<double>(hi - lo)));
}

size_t dash_select_workspace_size(int64_t T) {
  if (T < 0) return 0;
  Carver c{nullptr};
  SelWs w;
  carve_select(T, c, w);
  return c.off + 256;
}

dash_status dash_select(const float* scores, int64_t T, int32_t kind, double keep_ratio, float threshold,
                        int32_t keep_first, int32_t keep_last, int32_t* idx, int32_t* halted, int32_t* count,
                        void* ws, size_t ws_bytes, void* stream) {
  if (T < 0 || T > INT32_MAX) return DASH_ERR_SHAPE;
  if (!count || (T > 0 && (!scores || !idx))) return DASH_ERR_INVALID_ARG;
  if (kind != DASH_SELECT_TOPK && kind != DASH_SELECT_THRESHOLD) return DASH_ERR_INVALID_ARG;
  if (keep_first < 0 || keep_last < 0) return DASH_ERR_INVALID_ARG;
  if (kind == DASH_SELECT_TOPK && !(keep_ratio >= 0.0 && keep_ratio <= 1.0)) return DASH_ERR_INVALID_ARG;
  if (T > 0 && (!ws || ws_bytes < dash_select_workspace_size(T))) return DASH_ERR_NO_MEMORY;
  DeviceInfo* di;
  dash_status s = device_info(&di);
  if (s != DASH_OK) return s;
  Carver c{reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(ws) + 255) & ~static_cast<uintptr_t>(255))};
  SelWs w;
  carve_select(T, c, w);
  return select_impl(scores, T, nullptr, 1, kind, keep_ratio, threshold, keep_first, keep_last, idx, halted, count,
                     &w, *di, as_stream(stream));
}

dash_status dash_compact(const dash_bf16* X, int64_t T, const int32_t* idx, int64_t K, int32_t d, dash_bf16* Y,
                         void* stream) {
  if (K < 0 || T < 0 || d <= 0 || d % 8 != 0) return DASH_ERR_SHAPE;
  if (K == 0) return DASH_OK;
  if (!X || !idx || !Y || !aligned16(X) || !aligned16(Y)) return DASH_ERR_INVALID_ARG;
  DeviceInfo* di;
  dash_status s = device_info(&di);
  if (s != DASH_OK) return s;
  return move_rows(false, reinterpret_cast<const s16*>(X), reinterpret_cast<s16*>(Y), idx, K, T, d, *di,
                   as_stream(stream));
}

dash_status dash_scatter(const dash_bf16* Y, const int32_t* idx, int64_t K, int32_t d, dash_bf16* X, int64_t T,
                         void* stream) {
  if (K < 0 || T < 0 || d <= 0 || d % 8 != 0) return DASH_ERR_SHAPE;
  if (K == 0) return DASH_OK;
  if (!X || !idx || !Y || !aligned16(X) || !aligned16(Y)) return DASH_ERR_INVALID_ARG;
  DeviceInfo* di;
  dash_status s = device_info(&di);
  if (s != DASH_OK) return s;
  return move_rows(true, reinterpret_cast<const s16*>(Y), reinterpret_cast<s16*>(X), idx, K, T, d, *di,
                   as_stream(stream));
}

dash_status dash_rmsnorm(const dash_bf16* X, int64_t M, int32_t d, const dash_bf16* g, double eps, dash_bf16* Y,
                         void* stream) {
  if (M < 0 || d <= 0 || d % 8 != 0 || d > 8 * 32 * dash::rows::kMaxVec) return DASH_ERR_SHAPE;
  if (M == 0) return DASH_OK;
  if (!X || !g || !Y || !aligned16(X) || !aligned16(g) || !aligned16(Y)) return DASH_ERR_INVALID_ARG;
  return rmsnorm<kBf16>(reinterpret_cast<const s16*>(X), M, nullptr, M, d, reinterpret_cast<const s16*>(g), eps,
                 reinterpret_cast<s16*>(Y), as_stream(stream));
}

int32_t dash_set_decode_tensor_cores(int32_t enable) {
  const bool prev = g_gemv_tc;
  g_gemv_tc = enable != 0;
  return prev ? 1 : 0;
}

int32_t dash_set_gemm_pairs(int32_t enable) { return g_gemm_pairs.exchange(enable != 0 ? 1 : 0); }

dash_status dash_linear(const dash_bf16* A, int64_t M, int32_t K, const dash_bf16* W, int32_t N, dash_bf16* Y,
                        void* stream) {
  if (M < 0 || K <= 0 || N <= 0 || K % 64 != 0 || N % 128 != 0) return DASH_ERR_SHAPE;
  if (M == 0) return DASH_OK;
  if (!A || !W || !Y || !aligned16(A) || !aligned16(W) || !aligned16(Y)) return DASH_ERR_INVALID_ARG;
  DeviceInfo* di;
  dash_status s = device_info(&di);
  if (s != DASH_OK) return s;
  EpiArgs ep{};
  ep.out = reinterpret_cast<s16*>(Y);
  ep.ldo = N;
  return gemm<dash::gemm::kEpiStore, kBf16>(*di, reinterpret_cast<const s16*>(A), K, M, K, reinterpret_cast<const s16*>(W),
                                     nullptr, N, ep, as_stream(stream), DASH_K_GEMM);
}

dash_status dash_selftest_wait_timeout(int32_t* done) {
  if (!done) return DASH_ERR_INVALID_ARG;
  if (cudaDeviceSynchronize() != cudaSuccess) return DASH_ERR_CUDA;
  wait_timeout_selftest_kernel<<<1, 32>>>(done);
  if (cudaGetLastError() != cudaSuccess) return DASH_ERR_CUDA;
  return dash_device_error();
}

dash_status dash_exp2_fma(const float* x, int64_t n, float* y, void* stream) {
  if (n < 0) return DASH_ERR_SHAPE;
  if (n == 0) return DASH_OK;
  if (!x || !y) return DASH_ERR_INVALID_ARG;
  const int64_t blocks = (n + 255) / 256 < 4096 ? (n + 255) / 256 : 4096;
  exp2_fma_kernel<<<static_cast<unsigned>(blocks), 256, 0, as_stream(stream)>>>(x, n, y);
  return launch_status();
}

dash_status dash_attention(const dash_bf16* Q, const dash_bf16* K, const dash_bf16* V, int64_t M, int64_t T_kv,
                           int32_t hq, int32_t hkv, int32_t hd, const int32_t* qpos, const int32_t* kstart,
                           dash_bf16* O, void* stream) {
  if (M < 0 || T_kv < 0 || hq <= 0 || hkv <= 0 || hq % hkv != 0 || (hd != 64 && hd != 128)) return DASH_ERR_SHAPE;
  if (M == 0) return DASH_OK;
  if (T_kv == 0) return DASH_ERR_SHAPE;
  if (!Q || !K || !V || !O || !aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O))
    return DASH_ERR_INVALID_ARG;
  if (!qpos && M > T_kv) return DASH_ERR_SHAPE;
  DeviceInfo* di;
  dash_status s = device_info(&di);
  if (s != DASH_OK) return s;
  const int64_t qd = static_cast<int64_t>(hq) * hd, kvd = static_cast<int64_t>(hkv) * hd;
  return attention<kBf16>(reinterpret_cast<const s16*>(Q), qd, reinterpret_cast<const s16*>(K),
                   reinterpret_cast<const s16*>(V), kvd, M, T_kv, hq, hkv, hd, qpos, kstart,
                   reinterpret_cast<s16*>(O), qd, as_stream(stream));
}

size_t dash_layer_workspace_size(const dash_dims* dims, int64_t M, int64_t T_kv, int64_t max_pos) {
  if (!dims_ok(dims) || M < 0 || T_kv < M || max_pos < 0) return 0;
  Carver c{nullptr};
  LayerWs w;
  carve_layer(*dims, M, T_kv, max_pos, c, w);
  return c.off + 256;
}

dash_status dash_layer_forward(const dash_dims* dims, const dash_layer_weights* w, dash_bf16* H, int64_t M,
                               const int32_t* pos, int64_t max_pos, const dash_halt_ctx* halt, float* delta,
                               int32_t relative, void* ws, size_t ws_bytes, void* stream) {
  if (!dims_ok(dims)) return DASH_ERR_SHAPE;
  if (!weights_ok(w) || !H || !aligned16(H)) return DASH_ERR_INVALID_ARG;
  if (M < 0 || M > INT32_MAX) return DASH_ERR_SHAPE;
  if (M == 0) return DASH_OK;
  int64_t T_kv = M;
  if (halt) {
    if (!halt->active_idx || !halt->h_full || halt->T < M || pos != halt->active_idx) return DASH_ERR_INVALID_ARG;
    if (halt->T > M && !halt->halted_idx) return DASH_ERR_INVALID_ARG;
    T_kv = halt->T;
    if (max_pos < halt->T) return DASH_ERR_INVALID_ARG;
  }
  if (!pos && max_pos < M) return DASH_ERR_INVALID_ARG;
  if (max_pos > INT32_MAX) return DASH_ERR_SHAPE;
  const size_t need = dash_layer_workspace_size(dims, M, T_kv, max_pos);
  if (!ws || ws_bytes < need) return DASH_ERR_NO_MEMORY;
  DeviceInfo* di;
  dash_status s = device_info(&di);
  if (s != DASH_OK) return s;
  Carver c{reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(ws) + 255) & ~static_cast<uintptr_t>(255))};
  LayerWs L;
  carve_layer(*dims, M, T_kv, max_pos, c, L);
  cudaStream_t st = as_stream(stream);
  if ((s = rope_table(L.rope, max_pos, dims->head_dim, dims->rope_theta, *di, st)) != DASH_OK) return s;
  return layer_fmt(*di, *dims, *w, reinterpret_cast<s16*>(H), M, pos, halt, delta, relative, L, st);
}

dash_status dash_layer_forward_noalloc(const dash_dims* dims, const dash_layer_weights* w, dash_bf16* H,
                                       int64_t M, const int32_t* pos, int64_t max_pos, const dash_halt_ctx* halt,
                                       float* delta, int32_t relative, void* stream) {
  if (!dims_ok(dims)) return DASH_ERR_SHAPE;
  if (M < 0 || max_pos < 0) return DASH_ERR_SHAPE;
  if (M == 0) return DASH_OK;
  const int64_t T_kv = halt ? halt->T : M;
  const size_t need = dash_layer_workspace_size(dims, M, T_kv, max_pos);
  if (need == 0) return DASH_ERR_INVALID_ARG;
  if (need > kNoAllocScratchBytes) return DASH_ERR_NO_MEMORY;
  void* scratch = nullptr;
  const dash_status s = noalloc_scratch(&scratch);
  if (s != DASH_OK) return s;
  return dash_layer_forward(dims, w, H, M, pos, max_pos, halt, delta, relative, scratch, kNoAllocScratchBytes,
                            stream);
}

size_t dash_prefill_workspace_size(const dash_dims* dims, int64_t T, const dash_config* cfg) {
  if (!dims_ok(dims) || T < 0 || !cfg) return 0;
  Carver c{nullptr};
  PrefillWs w;
  carve_prefill(*dims, T, 1, c, w);
  return c.off + 256;
}

size_t dash_prefill_varlen_workspace_size(const dash_dims* dims, int64_t T, int32_t nseq, const dash_config* cfg) {
  if (!dims_ok(dims) || T < 0 || nseq < 1 || !cfg) return 0;
  Carver c{nullptr};
  PrefillWs w;
  carve_prefill(*dims, T, nseq, c, w);
  return c.off + 256;
}

dash_status dash_prefill(const dash_dims* dims, const dash_layer_weights* layers, dash_bf16* H, int64_t T,
                         const dash_config* cfg, int32_t* idx_out, int64_t* K_out, float* delta_out, void* ws,
                         size_t ws_bytes, void* stream) {
  if (T < 0 || T > INT32_MAX) return DASH_ERR_SHAPE;
  const int32_t cu[2] = {0, static_cast<int32_t>(T)};
  return prefill_impl(dims, layers, H, cu, 1, cfg, idx_out, K_out, nullptr, delta_out, ws, ws_bytes, stream);
}

dash_status dash_prefill_varlen(const dash_dims* dims, const dash_layer_weights* layers, dash_bf16* H,
                                const int32_t* cu_seqlens, int32_t nseq, const dash_config* cfg, int32_t* idx_out,
                                int64_t* K_out, int32_t* seq_counts, float* delta_out, void* ws, size_t ws_bytes,
                                void* stream) {
  if (!cu_seqlens || nseq < 1) return DASH_ERR_INVALID_ARG;
  if (cu_seqlens[0] != 0) return DASH_ERR_INVALID_ARG;
  for (int s = 0; s < nseq; ++s)
    if (cu_seqlens[s + 1] < cu_seqlens[s]) return DASH_ERR_INVALID_ARG;
  return prefill_impl(dims, layers, H, cu_seqlens, nseq, cfg, idx_out, K_out, seq_counts, delta_out, ws, ws_bytes,
                      stream);
}

dash_status dash_prefill_kv(const dash_dims* dims, const dash_layer_weights* layers, dash_bf16* H, int64_t T,
                            const dash_config* cfg, int32_t* idx_out, int64_t* K_out, float* delta_out,
                            dash_kv_cache* caches, void* ws, size_t ws_bytes, void* stream) {
  if (T < 0 || T > INT32_MAX) return DASH_ERR_SHAPE;
  if (!caches) return DASH_ERR_INVALID_ARG;
  const int32_t cu[2] = {0, static_cast<int32_t>(T)};
  return prefill_impl(dims, layers, H, cu, 1, cfg, idx_out, K_out, nullptr, delta_out, ws, ws_bytes, stream,
                      caches);
}

dash_status dash_prefill_varlen_kv(const dash_dims* dims, const dash_layer_weights* layers, dash_bf16* H,
                                   const int32_t* cu_seqlens, int32_t nseq, const dash_config* cfg,
                                   int32_t* idx_out, int64_t* K_out, int32_t* seq_counts, float* delta_out,
                                   dash_kv_cache* caches, void* ws, size_t ws_bytes, void* stream) {
  if (!cu_seqlens || nseq < 1 || !caches) return DASH_ERR_INVALID_ARG;
  if (cu_seqlens[0] != 0) return DASH_ERR_INVALID_ARG;
  for (int s = 0; s < nseq; ++s)
    if (cu_seqlens[s + 1] < cu_seqlens[s]) return DASH_ERR_INVALID_ARG;
  return prefill_impl(dims, layers, H, cu_seqlens, nseq, cfg, idx_out, K_out, seq_counts, delta_out, ws, ws_bytes,
                      stream, caches);
}

size_t dash_decode_attention_workspace_size(int32_t hd) {
  if (hd != 64 && hd != 128) return 0;
  return static_cast<size_t>(dash::decode::kMaxCtas) * dash::decode::kGroupPad * (hd + 2) * sizeof(float) + 1024;
}

dash_status dash_decode_attention(const dash_bf16* Q, int32_t nseq, const dash_kv_cache* caches, int32_t hq,
                                  int32_t hkv, int32_t hd, dash_bf16* O, void* ws, size_t ws_bytes,
                                  void* stream) {
  namespace dec = dash::decode;
  if (nseq < 1 || nseq > dec::kMaxSeq || hkv <= 0 || hq <= 0 || hq % hkv != 0 || (hd != 64 && hd != 128) ||
      hq / hkv > dec::kGroupPad || nseq * hkv > dec::kMaxSegs || (hq * hd) % 8 != 0)
    return DASH_ERR_SHAPE;
  if (!Q || !O || !caches || !aligned16(Q) || !aligned16(O)) return DASH_ERR_INVALID_ARG;
  const dash_kv_cache* lc[dec::kMaxSeq];
  int64_t len[dec::kMaxSeq];
  for (int q = 0; q < nseq; ++q) {
    if (!caches[q].k || !caches[q].v || !aligned16(caches[q].k) || !aligned16(caches[q].v))
      return DASH_ERR_INVALID_ARG;
    if (caches[q].len < 1 || caches[q].len > INT32_MAX) return DASH_ERR_SHAPE;
    lc[q] = &caches[q];
    len[q] = caches[q].len;
  }
  const size_t need = dash_decode_attention_workspace_size(hd);
  if (!ws || ws_bytes < need) return DASH_ERR_NO_MEMORY;
  DeviceInfo* di;
  dash_status s = device_info(&di);
  if (s != DASH_OK) return s;
  if (di->num_sms < dec::kMaxSegs) return DASH_ERR_SHAPE;
  dash_dims D{};
  D.n_layers = 1;
  D.n_heads = hq;
  D.n_kv_heads = hkv;
  D.head_dim = hd;
  Carver c{reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(ws) + 255) & ~static_cast<uintptr_t>(255))};
  DecodeWs w{};
  w.Q = const_cast<s16*>(reinterpret_cast<const s16*>(Q));
  w.O = reinterpret_cast<s16*>(O);
  w.part_o = c.take<float>(static_cast<size_t>(dec::kMaxCtas) * dec::kGroupPad * hd);
  w.part_ml = c.take<float>(static_cast<size_t>(dec::kMaxCtas) * dec::kGroupPad * 2);
  cudaStream_t st = as_stream(stream);
  return hd == 128 ? decode_attention_hd<128, kBf16>(*di, D, nseq, len, lc, w, st)
                   : decode_attention_hd<64, kBf16>(*di, D, nseq, len, lc, w, st);
}

size_t dash_decode_workspace_size(const dash_dims* dims, int32_t nseq) {
  if (!dims_ok(dims) || nseq < 1 || nseq > dash::decode::kMaxSeq) return 0;
  Carver c{nullptr};
  DecodeWs w;
  carve_decode(*dims, nseq, c, w);
  return c.off + 256;
}

dash_status dash_decode_step(const dash_dims* dims, const dash_layer_weights* layers, dash_bf16* X,
                             int32_t nseq, const int32_t* pos, dash_kv_cache* caches, void* ws, size_t ws_bytes,
                             void* stream) {
  if (dims && dims->dtype == DASH_DTYPE_F16)
    return decode_impl<kF16>(dims, layers, X, nseq, pos, caches, ws, ws_bytes, stream);
  return decode_impl<kBf16>(dims, layers, X, nseq, pos, caches, ws, ws_bytes, stream);
}

dash_status dash_timing_start(int32_t capacity) {
  if (capacity <= 0) return DASH_ERR_INVALID_ARG;
  g_timing.recs.clear();
  g_timing.recs.reserve(static_cast<size_t>(capacity));
  g_timing.cap = capacity;
  g_timing.used = 0;
  g_timing.layer = -1;
  g_timing.on = true;
  return DASH_OK;
}

int32_t dash_timing_stop(dash_launch_record* out, int32_t cap) {
  g_timing.on = false;
  int32_t n = 0;
  for (TimingRec& t : g_timing.recs) {
    if (cudaEventSynchronize(t.e1) != cudaSuccess) return -1;
    float ms = 0.f;
    if (cudaEventElapsedTime(&ms, t.e0, t.e1) != cudaSuccess) return -1;
    t.r.ms = ms;
    if (out && n < cap) out[n] = t.r;
    ++n;
  }
  g_timing.recs.clear();
  g_timing.used = 0;
  return n < cap || !out ? n : cap;
}

const char* dash_kernel_name(int32_t kind) {
  static const char* names[DASH_K_COUNT] = {"rope_table", "rmsnorm", "gemm_qkv_rope", "gemm_kv_halted",
                                            "attention", "gemm_o_resid_delta", "score", "gemm_gate_up_swiglu",
                                            "gemm_down_resid", "select", "gather", "scatter", "gemm",
                                            "kv_store", "gemv_qkv_rope_append", "decode_attention",
                                            "gemv_o_resid", "gemv_gate_up_swiglu", "gemv_down_resid"};
  return kind >= 0 && kind < DASH_K_COUNT ? names[kind] : "unknown";
}

}  // extern "C"
