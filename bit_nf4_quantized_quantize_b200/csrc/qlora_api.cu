// Host side of the C ABI declared in include/qlora_nf4.h: argument checks,
// the NF4 tables, workspace layout, TMA descriptors and kernel launches.
// Everything here runs on the host; all arithmetic of the layer runs in the
// kernels of quantize.cuh and gemm_tc.cuh.
#include "qlora_nf4.h"

#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <atomic>
#include <map>
#include <mutex>
#include <tuple>
#include <utility>
#include <vector>

#include "ptx_sm100.cuh"
#include "quantize.cuh"
#include "gemm_tc.cuh"
#include "lora_tc.cuh"
#include "fused2_tc.cuh"
#include "decode_tc.cuh"
#include "decode_lut.cuh"
#include "merge.cuh"
#include "dropout.cuh"

using namespace qlora;

namespace {

// ------------------------------------------------------------------ NF4 table
// Standard normal quantile by Newton's method on Phi(x) = erfc(-x/sqrt2)/2
// (on the upper tail erfc(x/sqrt2)/2 = 1-p for p > 1/2), started at 0.
double normal_quantile(double p) {
  const double inv_sqrt_2pi = 0.39894228040143267794;
  const bool upper = p > 0.5;
  const double target = upper ? 1.0 - p : p;
  double x = 0.0;
  for (int it = 0; it < 100; ++it) {
    const double f = upper ? (target - 0.5 * std::erfc(x / std::sqrt(2.0)))
                           : (0.5 * std::erfc(-x / std::sqrt(2.0)) - target);
    const double step = f / (inv_sqrt_2pi * std::exp(-0.5 * x * x));
    const double nx = x - step;
    if (nx == x || std::fabs(step) < 1e-17) { x = nx; break; }
    x = nx;
  }
  return x;
}

// "QLoRAの理論と実装", listing create_nf4_codebook: Phi^-1(i/18) for i = 1..8,
// the level 0, Phi^-1(j/16) for j = 9..15, divided by the largest magnitude.
// Decision thresholds: code(n) = #{i : n > (level_i + level_{i+1})/2}, the
// exact nearest level with the lower index on a tie; thr_i is the smallest
// fp32 above that exact midpoint, so code(n) = #{i : n >= thr_i}.  The
// 33-cell table indexes floor(16 n) + 16 for n in [-1, 1].
Nf4Tables build_tables() {
  Nf4Tables T;
  std::memset(&T, 0, sizeof(T));
  double v[16];
  int n = 0;
  for (int i = 1; i <= 8; ++i) v[n++] = normal_quantile(i / 18.0);
  v[n++] = 0.0;
  for (int j = 9; j <= 15; ++j) v[n++] = normal_quantile(j / 16.0);
  double mx = 0.0;
  for (double a : v) mx = std::max(mx, std::fabs(a));
  for (int i = 0; i < 16; ++i) T.level[i] = static_cast<float>(v[i] / mx);
  std::sort(T.level, T.level + 16);
  double mid[15];
  float thr[15];
  for (int i = 0; i < 15; ++i) {
    mid[i] = (static_cast<double>(T.level[i]) + static_cast<double>(T.level[i + 1])) * 0.5;
    float f = static_cast<float>(mid[i]);
    if (static_cast<double>(f) <= mid[i]) f = std::nextafter(f, INFINITY);
    thr[i] = f;
  }
  // cells of width 1/16: cell c covers [(c-16)/16, (c-15)/16)
  T.fast_ok = 1;
  for (int c = 0; c < kLutCells; ++c) {
    const double lo = (c - 16) / 16.0, hi = (c - 15) / 16.0;
    int cnt = 0, inside_n = 0, inside_i = -1;
    for (int i = 0; i < 15; ++i) {
      if (mid[i] < lo) ++cnt;
      else if (mid[i] < hi) { if (inside_i < 0) inside_i = i; ++inside_n; }
    }
    T.cell_lo[c] = cnt;
    T.cell_thr[c] = inside_i < 0 ? INFINITY : thr[inside_i];
    if (inside_n > 1) T.fast_ok = 0;  // (cannot happen for this table: midpoints are >= 0.088 apart)
    // fast entry, in units of t = 16 n + 15.875: the midpoint (64.0 when the
    // cell has none, above every t) with the code in its 4 low mantissa bits
    const float f = inside_i < 0 ? 64.0f : static_cast<float>(16.0 * mid[inside_i] + 15.875);
    uint32_t bits;
    std::memcpy(&bits, &f, 4);
    T.cell_fast[c] = (bits & ~15u) | static_cast<uint32_t>(cnt);
  }
  // every midpoint must be farther than 2^-17 from every cell edge
  for (int i = 0; i < 15; ++i) {
    const double d = std::fabs(mid[i] * 16.0 - std::nearbyint(mid[i] * 16.0)) / 16.0;
    if (d <= std::ldexp(1.0, -17)) T.fast_ok = 0;
  }
  return T;
}

const Nf4Tables& tables() {
  static const Nf4Tables t = build_tables();
  return t;
}

// ------------------------------------------------------------------ device
constexpr int kMaxDevices = 64;

int check_device(int* dev_out, int* num_sms) {
  // caches shared by host threads: cached_sms is written before cached_ok publishes it
  static std::atomic<int> cached_ok[kMaxDevices];  // 0 unknown, 1 ok, -1 bad
  static std::atomic<int> cached_sms[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) { cudaGetLastError(); return QLORA_ERR_NO_DEVICE; }
  if (dev < 0 || dev >= kMaxDevices) return QLORA_ERR_NO_DEVICE;
  if (cached_ok[dev] == 0) {
    cudaDeviceProp prop;
    if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) { cudaGetLastError(); return QLORA_ERR_NO_DEVICE; }
    cached_sms[dev] = prop.multiProcessorCount;
    cached_ok[dev] = (prop.major == 10) ? 1 : -1;
  }
  if (cached_ok[dev] != 1) return QLORA_ERR_NO_DEVICE;
  *dev_out = dev;
  *num_sms = cached_sms[dev];
  return QLORA_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// ------------------------------------------------------------------ TMA
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    else
      cudaGetLastError();
  });
  return fn;
}

// 2-D row-major tensor: `cols` contiguous elements per row, `rows` rows,
// `row_bytes` between rows; box of box_cols x box_rows.
bool make_map(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t cols, uint64_t rows,
              uint64_t row_bytes, uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle sw) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool map_bf16(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, uint32_t box_cols, uint32_t box_rows) {
  return make_map(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, base, cols, rows, cols * 2, box_cols, box_rows,
                  CU_TENSOR_MAP_SWIZZLE_128B);
}

// ------------------------------------------------------------------ timing
struct TimingRec {
  int kind;
  cudaEvent_t start, stop;
};
std::mutex g_timing_mu;
std::atomic<bool> g_timing_on{false};   // read by every launch, set by qlora_timing_enable
std::vector<TimingRec> g_timing_recs;
std::vector<cudaEvent_t> g_event_pool;

cudaEvent_t take_event() {
  if (!g_event_pool.empty()) {
    cudaEvent_t e = g_event_pool.back();
    g_event_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  if (cudaEventCreate(&e) != cudaSuccess) { cudaGetLastError(); return nullptr; }
  return e;
}

// Run `launch` (which enqueues one kernel on st); bracket it with events when
// timing is on.
std::atomic<int64_t> g_launch_count{0};

template <class F>
int timed(int kind, cudaStream_t st, F&& launch) {
  g_launch_count.fetch_add(1, std::memory_order_relaxed);
  if (!g_timing_on) return launch();
  std::lock_guard<std::mutex> lk(g_timing_mu);
  cudaEvent_t a = take_event(), b = take_event();
  if (a) cudaEventRecord(a, st);
  const int rc = launch();
  if (b) cudaEventRecord(b, st);
  if (a && b) g_timing_recs.push_back({kind, a, b});
  return rc;
}

// ------------------------------------------------------------------ launches
// Launch with programmatic stream serialisation (see griddep_wait in
// ptx_sm100.cuh), optionally as clusters of cluster_x x 1 x cluster_z CTAs.
template <typename... KArgs, typename... Args>
int launch_ex(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, unsigned cluster_x,
              unsigned cluster_z, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  int n = 0;
  attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[n].val.programmaticStreamSerializationAllowed = 1;
  ++n;
  if (cluster_x * cluster_z > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = cluster_x;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = cluster_z;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  if (cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...) != cudaSuccess) {
    cudaGetLastError();
    return QLORA_ERR_CUDA;
  }
  return QLORA_OK;
}

template <int BN, int NSTAGE, bool A_MN, int BSRC, int OUT, int NDW, int MH = 1>
int launch_gemm(dim3 grid, const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& a2,
                const CUtensorMap& b2, const GemmArgs& args, cudaStream_t st, int dev) {
  using L = GemmSmem<BN, NSTAGE, BSRC, NDW, MH, OUT>;
  auto kern = qlora_gemm_kernel<BN, NSTAGE, A_MN, BSRC, OUT, NDW, MH>;
  // the adapter slices must fit in the first pass over the stages
  if (args.n_lora > NSTAGE) return QLORA_ERR_UNSUPPORTED_SHAPE;
  static std::atomic<bool> attr_set[kMaxDevices];   // one-time setup done (stored last)
  if (!attr_set[dev]) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kDynBytes) != cudaSuccess) {
      cudaGetLastError();
      return QLORA_ERR_CUDA;
    }
    attr_set[dev] = true;
  }
  const int kind = (OUT == kOutDropoutAdd) ? QLORA_KERNEL_DROPOUT
                 : (BSRC == kBDeqK) ? QLORA_KERNEL_FWD
                 : (BSRC == kBDeqMN) ? QLORA_KERNEL_DX
                 : A_MN ? QLORA_KERNEL_GRAD_GEMM : QLORA_KERNEL_LORA_GEMM;
  return timed(kind, st, [&] {
    return launch_ex(kern, grid, dim3(64 + 32 * NDW), L::kDynBytes, st, 1, grid.z, a, b, a2, b2, args);
  });
}

// Fused dequant-GEMM on CTA pairs (cluster of 2), tile (256*MH) x 256.
template <int BSRC, int MH>
int launch_pair(int num_pairs, const CUtensorMap& a, const CUtensorMap& p, const CUtensorMap& a2,
                const CUtensorMap& b2, const GemmArgs& args, cudaStream_t st, int dev) {
  // output: bf16 [m_rows x n_cols] (row stride ld_out), stored in 32 x 32 blocks with 64-byte swizzle
  CUtensorMap out;
  if (!make_map(&out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, args.out, static_cast<uint64_t>(args.n_cols),
                static_cast<uint64_t>(args.m_rows), static_cast<uint64_t>(args.ld_out) * 2, 32, 32,
                CU_TENSOR_MAP_SWIZZLE_64B))
    return QLORA_ERR_CUDA;
  using L = PairSmem<MH>;
  auto kern = qlora_fused_pair_kernel<BSRC, MH>;
  static std::atomic<bool> attr_set[kMaxDevices];   // one-time setup done (stored last)
  if (!attr_set[dev]) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kDynBytes) != cudaSuccess) {
      cudaGetLastError();
      return QLORA_ERR_CUDA;
    }
    attr_set[dev] = true;
  }
  const int kind = (BSRC == kBDeqK) ? QLORA_KERNEL_FWD : QLORA_KERNEL_DX;
  return timed(kind, st, [&] {
    return launch_ex(kern, dim3(static_cast<unsigned>(2 * num_pairs)), dim3(kPairThreads), L::kDynBytes, st, 2, 1,
                     a, p, a2, b2, out, args);
  });
}

// Small-M forward (decode_tc.cuh): row tiles of T = 128 - r weight rows, the
// K range split over a cluster of S CTAs.  S is the largest cluster size
// (<= 8) for which every row tile's cluster is resident at once (the
// occupancy query accounts for how clusters pack into the GPU's processing
// clusters) and every rank gets at least two k-steps.
template <int MP>
int launch_decode(const CUtensorMap& tx, const CUtensorMap& tp, const CUtensorMap& ta, const CUtensorMap& tb,
                  DecodeArgs& d, cudaStream_t st, int dev) {
  using L = DecodeSmem<MP>;
  auto kern = qlora_decode_kernel<MP>;
  static std::atomic<bool> attr_set[kMaxDevices];   // one-time setup done (stored last)
  static std::atomic<int> max_clusters[kMaxDevices][9];
  if (!attr_set[dev]) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kDynBytes) != cudaSuccess) {
      cudaGetLastError();
      return QLORA_ERR_CUDA;
    }
    for (int S = 1; S <= 8; ++S) {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(1, 1, static_cast<unsigned>(S));
      cfg.blockDim = dim3(kDecThreads);
      cfg.dynamicSmemBytes = L::kDynBytes;
      cudaLaunchAttribute attr;
      attr.id = cudaLaunchAttributeClusterDimension;
      attr.val.clusterDim.x = 1;
      attr.val.clusterDim.y = 1;
      attr.val.clusterDim.z = static_cast<unsigned>(S);
      cfg.attrs = &attr;
      cfg.numAttrs = 1;
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) {
        cudaGetLastError();
        n = 0;
      }
      max_clusters[dev][S] = n;
    }
    attr_set[dev] = true;
  }
  const int T = d.tile_rows;
  const int tiles = (d.n_cols + T - 1) / T;
  int S = 1;
  for (int c = 2; c <= 8; ++c) {
    const int per = (d.k_steps + c - 1) / c;
    if (per < 2 || (c - 1) * per >= d.k_steps) continue;   // every rank gets work
    if (tiles <= max_clusters[dev][c]) S = c;
  }
  d.steps_per_split = (d.k_steps + S - 1) / S;
  d.slice_rows = ((T + S - 1) / S + 7) / 8 * 8;
  d.slice_u = (d.r + S - 1) / S;
  if (S * d.slice_rows > 192 || S * d.slice_u > 72) return QLORA_ERR_UNSUPPORTED_SHAPE;  // not reached: r <= 64
  return timed(QLORA_KERNEL_FWD_DECODE, st, [&] {
    return launch_ex(kern, dim3(static_cast<unsigned>(tiles), 1, static_cast<unsigned>(S)), dim3(kDecThreads),
                     L::kDynBytes, st, 1, static_cast<unsigned>(S), tx, tp, ta, tb, d);
  });
}

int run_decode(const uint8_t* codes, const uint8_t* q8, const float* s2, int64_t N, int64_t K, const uint16_t* X,
               int64_t M, const uint16_t* A, const uint16_t* B, int r, float s, uint16_t* Y, uint16_t* U_save,
               cudaStream_t st, int dev) {
  const int mp = M <= 16 ? 16 : 32;
  const int T = kDecLanes - r;
  CUtensorMap tx, tp, ta, tb;
  if (!map_bf16(&tx, X, M, K, 64, static_cast<uint32_t>(mp)) ||
      !make_map(&tp, CU_TENSOR_MAP_DATA_TYPE_UINT8, codes, K / 2, N, K / 2, 32, static_cast<uint32_t>(T),
                CU_TENSOR_MAP_SWIZZLE_32B) ||
      !map_bf16(&ta, A, r, K, 64, static_cast<uint32_t>(r)) || !map_bf16(&tb, B, N, r, 64, kDecLanes))
    return QLORA_ERR_CUDA;
  DecodeArgs d{};
  d.m_rows = static_cast<int>(M);
  d.n_cols = static_cast<int>(N);
  d.k_steps = static_cast<int>(K / 64);
  d.steps_per_split = d.k_steps;
  d.r = r;
  d.tile_rows = T;
  d.s = s;
  d.q8 = q8;
  d.s2 = s2;
  for (int i = 0; i < 16; ++i) d.level[i] = tables().level[i];
  d.y = Y;
  d.ld_y = N;
  d.u_save = U_save;
  if (mp == 16) return launch_decode<16>(tx, tp, ta, tb, d, st, dev);
  return launch_decode<32>(tx, tp, ta, tb, d, st, dev);
}

size_t a256(size_t x) { return (x + 255) & ~size_t(255); }

constexpr int kLutRouteTokens = 4;   // the forward takes the table-lookup path up to this many tokens

// One to eight tokens (decode_lut.cuh): U = X A^T in a small launch that also
// prefetches the weight into L2, then the table-lookup kernel.  A CTA owns
// T = ceil(N / 16 / SMs) tiles of 16 rows and all of K.  Returns
// QLORA_ERR_UNSUPPORTED_SHAPE (nothing launched) when the shape is outside the
// kernel's limits; the caller then takes the other few-token path.
int run_decode_lut(const uint8_t* codes, const uint8_t* q8, const float* s2, int64_t N, int64_t K,
                   const uint16_t* X, int64_t M, const uint16_t* A, const uint16_t* B, int r, float s, uint16_t* Y,
                   uint16_t* U_save, float* U32, int sms, cudaStream_t st, int dev) {
  // the X rows and the 8-bit constants arrive by bulk copies: 16-byte aligned
  if (M > kLutMaxTokens || !aligned16(X) || (q8 && !aligned16(q8)) || N * (K / 64) >= (int64_t(1) << 31))
    return QLORA_ERR_UNSUPPORTED_SHAPE;
  const int tiles_total = static_cast<int>(N / kLutTile);
  const int T = (tiles_total + sms - 1) / sms;
  const int grid = (tiles_total + T - 1) / T;
  const int mi = static_cast<int>(M), ki = static_cast<int>(K);
  int n_slots = std::min(T, kLutMaxSlots);
  while (n_slots > 1 && lut_layout(mi, ki, T, n_slots, r, q8 == nullptr).total > kLutMaxSmem) --n_slots;
  const int smem = lut_layout(mi, ki, T, n_slots, r, q8 == nullptr).total;
  if (smem > kLutMaxSmem) return QLORA_ERR_UNSUPPORTED_SHAPE;
  LutArgs a{};
  a.codes = codes;
  a.q8 = q8;
  a.s2 = s2;
  a.x = X;
  a.b = B;
  a.u = U32;
  a.y = Y;
  a.m = mi;
  a.n = static_cast<int>(N);
  a.k = ki;
  a.r = r;
  a.tiles_per_cta = T;
  a.n_slots = n_slots;
  a.s = s;
  for (int i = 0; i < 16; ++i) a.level[i] = tables().level[i];
  DecUArgs u{};
  u.x = X;
  u.a = A;
  u.m = mi;
  u.k = ki;
  u.r = r;
  u.u32 = U32;
  u.u_save = U_save;
  u.codes = codes;
  u.consts = q8 ? q8 : reinterpret_cast<const uint8_t*>(s2);
  u.consts_size = q8 ? 1 : 4;
  u.n = static_cast<int>(N);
  u.rows_per_cta = T * kLutTile;
  static std::atomic<bool> attr_set[kMaxDevices];   // one-time setup done (stored last)
  if (!attr_set[dev]) {
    if (cudaFuncSetAttribute(qlora_decode_lut_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kLutMaxSmem) !=
        cudaSuccess) {
      cudaGetLastError();
      return QLORA_ERR_CUDA;
    }
    attr_set[dev] = true;
  }
  const unsigned u_grid = static_cast<unsigned>(std::max(grid, r));
  if (int rc = timed(QLORA_KERNEL_LORA_GEMM, st, [&] {
        if (M == 1) return launch_ex(qlora_decode_u_kernel<1>, dim3(u_grid), dim3(kDecUThreads), 0, st, 1, 1, u);
        if (M == 2) return launch_ex(qlora_decode_u_kernel<2>, dim3(u_grid), dim3(kDecUThreads), 0, st, 1, 1, u);
        if (M <= 4) return launch_ex(qlora_decode_u_kernel<4>, dim3(u_grid), dim3(kDecUThreads), 0, st, 1, 1, u);
        return launch_ex(qlora_decode_u_kernel<8>, dim3(u_grid), dim3(kDecUThreads), 0, st, 1, 1, u);
      }))
    return rc;
  return timed(QLORA_KERNEL_FWD_DECODE, st, [&] {
    return launch_ex(qlora_decode_lut_kernel, dim3(static_cast<unsigned>(grid)), dim3(kLutThreads),
                     static_cast<size_t>(smem), st, 1, 1, a);
  });
}

struct WsLayout {
  size_t us, v, vs, u, xm, bits, total;
};

// bf16 scratch of M x r each: s*U (forward adapter operand), V and s*V
// (backward), U (recomputed when the caller passes no saved U).
// With dropout, xm holds the masked adapter input X * keep (bf16 M x K) and
// bits the keep mask, one bit per element (M x K / 8 bytes).
WsLayout ws_layout(int64_t M, int64_t N, int64_t K, int r, int num_sms, bool dropout = false) {
  (void)N; (void)num_sms;
  WsLayout w;
  const size_t mr = a256(static_cast<size_t>(M) * r * 2);
  w.us = 0;
  w.v = w.us + mr;
  w.vs = w.v + mr;
  w.u = w.vs + mr;
  w.xm = w.u + mr;
  w.bits = w.xm + (dropout ? a256(static_cast<size_t>(M) * K * 2) : 0);
  w.total = w.bits + (dropout ? a256(static_cast<size_t>(M) * K / 8) : 0);
  return w;
}


// How many clusters of S CTAs (along z) of `kern` can be resident at once,
// from the occupancy API (it accounts for how clusters pack into the GPU's
// processing clusters), cached per kernel, device and S.
int cluster_capacity(const void* kern, int threads, size_t smem, int S, int dev) {
  static std::mutex mu;
  static std::map<std::tuple<const void*, int, int>, int> cache;
  std::lock_guard<std::mutex> lk(mu);
  const auto key = std::make_tuple(kern, dev, S);
  auto it = cache.find(key);
  if (it != cache.end()) return it->second;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) != cudaSuccess)
    cudaGetLastError();
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(1, 1, static_cast<unsigned>(S));
  cfg.blockDim = dim3(static_cast<unsigned>(threads));
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr;
  attr.id = cudaLaunchAttributeClusterDimension;
  attr.val.clusterDim.x = 1;
  attr.val.clusterDim.y = 1;
  attr.val.clusterDim.z = static_cast<unsigned>(S);
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) {
    cudaGetLastError();
    n = 0;
  }
  cache.emplace(key, n);
  return n;
}

// The largest split S <= 8 of k_steps reduction steps over a cluster along z
// such that every tile's cluster is resident at once (one wave) and every
// rank gets at least min_per steps; 1 when no split fits.  pow2: S must be a
// power of two (the kernel's reduction divides 128 tile rows by S).
int one_wave_split(const void* kern, int threads, size_t smem, int tiles, int k_steps, int min_per, bool pow2,
                   int dev) {
  int S = 1;
  for (int c = 2; c <= 8; ++c) {
    if (pow2 && (c & (c - 1)) != 0) continue;
    const int per = (k_steps + c - 1) / c;
    if (per < min_per || (c - 1) * per >= k_steps) continue;   // every rank gets work
    if (tiles <= cluster_capacity(kern, threads, smem, c, dev)) S = c;
  }
  return S;
}

// Split of a split-K adapter product (qlora_lora_kernel): the largest power
// of two <= 8 with tiles x S <= 2 x SMs and at least one reduction step per
// rank.  (The occupancy API reports one CTA of this kernel per SM; splits
// sized to that measured slower on the train4096 shapes: dA/dB 26.7 us at
// S = 2 against 23.9 us at S = 4.)
int lora_cluster(int tiles, int k_steps, int num_sms) {
  int S = 1;
  while (S < 8 && tiles * S * 2 <= 2 * num_sms && S * 2 <= k_steps) S *= 2;
  return S;
}

// Split of the small-M single-CTA fused kernel (one CTA per 128 x 256 tile):
// at least two reduction steps per rank.
template <int BSRC>
int gemm_split(int tiles, int k_steps, int dev) {
  using L = GemmSmem<256, 4, BSRC, 8, 1>;
  return one_wave_split(reinterpret_cast<const void*>(qlora_gemm_kernel<256, 4, false, BSRC, kOutBf16, 8, 1>),
                        64 + 32 * 8, L::kDynBytes, tiles, k_steps, 2, false, dev);
}

// Pipeline shape of the adapter kernel: stages x reduction steps per stage.
constexpr int kLoraStagesDefault = 4;
constexpr int kLoraKbDefault = 1;

// Grid: tiles_total CTAs along x (rounded up to cx) times S along z, in
// clusters of cx x 1 x S.
template <bool A_MN, bool B_MN, int STAGES = kLoraStagesDefault, int KB = kLoraKbDefault>
int launch_lora(const CUtensorMap& a0, const CUtensorMap& b0, const CUtensorMap& a1, const CUtensorMap& b1,
                const LoraArgs& args, int tiles_total, int S, cudaStream_t st, int dev, int kind, int cx = 1) {
  auto kern = qlora_lora_kernel<A_MN, B_MN, STAGES, KB>;
  using L = LoraSmem<STAGES, KB>;
  static std::atomic<bool> attr_set[kMaxDevices];   // one-time setup done (stored last)
  if (!attr_set[dev]) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kDynBytes) != cudaSuccess) {
      cudaGetLastError();
      return QLORA_ERR_CUDA;
    }
    attr_set[dev] = true;
  }
  return timed(kind, st, [&] {
    const unsigned gx = static_cast<unsigned>((tiles_total + cx - 1) / cx * cx);
    return launch_ex(kern, dim3(gx, 1, static_cast<unsigned>(S)), dim3(kLoraThreads), L::kDynBytes, st,
                     static_cast<unsigned>(cx), static_cast<unsigned>(S), a0, b0, a1, b1, args);
  });
}

LoraProblem lora_problem(int rows, int k_steps, int S, int rpad, int kind, void* out0, void* out1, int ld_t,
                         float scale0, float scale1) {
  LoraProblem p{};
  p.scale0 = scale0;
  p.scale1 = scale1;
  p.rows = rows;
  p.k_steps = k_steps;
  p.per_split = (k_steps + S - 1) / S;
  p.tiles_m = (rows + 127) / 128;
  p.tiles_n = rpad / 64;
  p.out_kind = kind;
  p.out0 = out0;
  p.out1 = out1;
  p.ld_t = ld_t;
  return p;
}

// q8 == NULL: single quantization, s2 holds the fp32 absmax of every block.
int check_weight(const uint8_t* codes, const uint8_t* q8, const float* s2, int64_t N, int64_t K) {
  (void)q8;
  if (!codes || !s2) return QLORA_ERR_INVALID_ARG;
  if (N <= 0 || K <= 0 || K % 64 != 0 || N % 64 != 0) return QLORA_ERR_UNSUPPORTED_SHAPE;
  if (N > (1 << 24) || K > (1 << 24)) return QLORA_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(codes) || !aligned16(s2)) return QLORA_ERR_UNSUPPORTED_SHAPE;
  return QLORA_OK;
}

// M == 0 (an empty batch) is valid, and X may then be NULL.
int check_lora(const void* X, int64_t M, const void* A, const void* B, int r, float alpha) {
  if ((M != 0 && !X) || !A || !B) return QLORA_ERR_INVALID_ARG;
  if (M < 0 || M > (1 << 24)) return QLORA_ERR_UNSUPPORTED_SHAPE;
  if (r < 1 || r > 256 || !std::isfinite(alpha)) return QLORA_ERR_INVALID_ARG;
  if (r % 8 != 0) return QLORA_ERR_UNSUPPORTED_SHAPE;
  if ((X && !aligned16(X)) || !aligned16(A) || !aligned16(B)) return QLORA_ERR_UNSUPPORTED_SHAPE;
  return QLORA_OK;
}

// Shape of a weight for the quantizer, the dequantizer and the merge: n_out,
// k_in >= 0 with k_in % 64 == 0.  Sets *empty when it holds no element (the
// call is then a no-op and its pointers may be NULL).
int check_weight_shape(int64_t n_out, int64_t k_in, bool* empty) {
  if (n_out < 0 || k_in < 0 || k_in % 64 != 0) return QLORA_ERR_UNSUPPORTED_SHAPE;
  *empty = n_out == 0 || k_in == 0;
  return QLORA_OK;
}

void fill_levels(GemmArgs& g) {
  for (int i = 0; i < 16; ++i) g.level[i] = tables().level[i];
}

// V runs beside dX as U runs beside the forward's fused kernel; dX's empty
// slots also take the gradient kernel (second stream).
constexpr bool kVBesideDx = true;

// Whether an adapter product (U = X A^T or V = dY B: ceil(M/128) x rpad/64
// tiles) can run beside the fused kernel that consumes it (`pairs` CTA-pair
// tiles over the same reduction length).  It then runs unsplit, one CTA per
// tile, two neighbouring tiles per TPC (a cluster of 2 along x): each of its
// C clusters takes one CTA-pair slot from the fused kernel's first wave for
// less than one of that kernel's tiles (one tile is twice the reduction
// steps at half the rate).  That costs nothing when C does not exceed the
// pair slots the fused kernel's last wave leaves empty.
bool adapter_beside(int64_t M, int rpad, int pairs, int num_sms) {
  if (num_sms < 2) return false;
  const int64_t tiles = (M + 127) / 128 * (rpad / 64);
  const int64_t clusters = (tiles + 1) / 2;
  const int64_t slots = num_sms / 2;
  const int64_t waves = (pairs + slots - 1) / slots;
  return clusters <= waves * slots - pairs;
}

// acc = X A^T; `plain` = bf16(scale0 acc) and `scaled` = bf16(scale1 acc), each may be NULL.
// beside: the unsplit grid of adapter_beside.
int run_lora_down(const uint16_t* X, int64_t M, int64_t K, const uint16_t* Amat, int r, float scale0, float scale1,
                  uint16_t* plain, uint16_t* scaled, int num_sms, cudaStream_t st, int dev, bool beside = false) {
  const int rpad = (r + 63) / 64 * 64;
  CUtensorMap ta, tb;
  if (!map_bf16(&ta, X, M, K, 64, 128) || !map_bf16(&tb, Amat, r, K, 64, 64)) return QLORA_ERR_CUDA;
  const int k_steps = static_cast<int>(K / 64);
  const int tiles = static_cast<int>((M + 127) / 128) * (rpad / 64);
  const int S = beside ? 1 : lora_cluster(tiles, k_steps, num_sms);
  LoraArgs la{};
  la.p[0] = lora_problem(static_cast<int>(M), k_steps, S, rpad, kLoraOutPlainScaled, plain, scaled, 0, scale0,
                         scale1);
  la.p[1] = la.p[0];
  la.p[1].tiles_m = 0;   // no second problem: a CTA padding the grid has no tile
  la.tiles0 = tiles;
  la.r = r;
  return launch_lora<false, false>(ta, tb, ta, tb, la, tiles, S, st, dev, QLORA_KERNEL_LORA_GEMM, beside ? 2 : 1);
}

// ------------------------------------------------------------------ LoRA dropout
// Dropout on the adapter input (dropout.cuh): 16-bit keep threshold t =
// floor(p * 2^16) and scale inv = fp32(1 / (1 - p)), both from the fp32 p.
struct DropoutSpec {
  bool on = false;
  uint32_t t = 0;
  float inv = 1.f;
  uint64_t seed = 0, offset = 0;
  // the masked input X * keep and the keep bits: written by the forward when the caller
  // asks to keep them, read by the backward instead of being generated again
  uint16_t* xd = nullptr;
  uint16_t* bits = nullptr;
};

// Returns false if p is not in [0, 1).  p == 0 leaves the spec off.
bool make_dropout(float p, uint64_t seed, uint64_t offset, DropoutSpec* d) {
  if (!(p >= 0.f && p < 1.f)) return false;
  *d = DropoutSpec{};
  if (p == 0.f) return true;
  const double pd = static_cast<double>(p);
  d->on = true;
  d->t = static_cast<uint32_t>(std::floor(pd * 65536.0));   // <= 0xFFFF for p < 1
  d->inv = static_cast<float>(1.0 / (1.0 - pd));
  d->seed = seed;
  d->offset = offset;
  return true;
}

// X * keep (bf16 M x K) into `out`.
// out = X * keep; bits (or NULL) receives the keep mask, one bit per element.
int launch_dropout_mask(const uint16_t* X, int64_t M, int64_t K, const DropoutSpec& d, uint16_t* out, int sms,
                        cudaStream_t st, uint16_t* bits = nullptr) {
  const int64_t n16 = M * K / 16;   // K % 64 == 0
  const int64_t want = (n16 + 255) / 256;
  // one round of resident blocks: the grid-stride loop then ends evenly on every SM
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return QLORA_ERR_CUDA;
  }
  static std::atomic<int> resident[kMaxDevices];   // blocks of 256 threads per SM, 0 = not yet asked
  if (resident[dev] == 0) {
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, dropout_mask_kernel, 256, 0) != cudaSuccess || n < 1) {
      cudaGetLastError();
      n = 1;
    }
    resident[dev] = n;
  }
  const unsigned blocks =
      static_cast<unsigned>(std::min<int64_t>(want, static_cast<int64_t>(sms) * resident[dev]));
  return timed(QLORA_KERNEL_DROPOUT, st, [&] {
    return launch_ex(dropout_mask_kernel, dim3(blocks), dim3(256), 0, st, 1, 1, X, n16, d.t, d.seed, d.offset, out,
                     bits);
  });
}

// ------------------------------------------------------------------ failure-path self-test
// One warp waits, bounded, on an mbarrier that nothing arrives at.  The wait
// gives up after kWaitLimitNs, latches the device error flag (as any kernel's
// expired wait does) and the kernel exits normally; *waited_ns (if given)
// receives how long it waited.
__global__ void selftest_wait_kernel(unsigned long long* waited_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_word;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_word = 0;
    fence_barrier_init();
  }
  __syncthreads();
  const uint64_t t0 = globaltimer_ns();
  const bool ok = mbar_wait(&bar, 0, &abort_word);
  __syncwarp();
  if (threadIdx.x == 0 && waited_ns != nullptr) *waited_ns = ok ? 0ull : globaltimer_ns() - t0;
}

// ------------------------------------------------------------------ fixed scratch
// Scratch of qlora_linear_fwd_noalloc: a file-scope device array, so that the
// library never allocates for that entry point.  Every GPU that loads the
// library holds these bytes until the process exits.
constexpr size_t kNoAllocScratchBytes = size_t(4) << 20;  // 4 MiB

}  // namespace

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {

// Device address of g_noalloc_scratch on the current device.  In host code the
// array's name only stands in for the symbol, so the address is looked up once
// per device (with that device current) and cached.
void* noalloc_scratch(int dev) {
  static std::mutex mu;
  static void* addr[kMaxDevices];
  std::lock_guard<std::mutex> lk(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
      cudaGetLastError();
      return nullptr;
    }
    addr[dev] = p;
  }
  return addr[dev];
}

}  // namespace

// ======================================================================= ABI
// A second stream per device for backward: the gradient kernel (dA, dB)
// needs only V, U, X and dY, so it runs beside the dX kernel and takes the
// SMs that the dX grid's last wave leaves idle.  The library forks it off the
// caller's stream with an event and joins it back before returning, so the
// caller sees one ordered stream.  Created on first use, kept for the
// process's lifetime.
struct AuxStream {
  cudaStream_t s = nullptr;
  cudaEvent_t fork = nullptr;
  cudaEvent_t join = nullptr;
  bool ok = false;
};
std::mutex g_aux_mu;
AuxStream g_aux[kMaxDevices];

// Caller holds g_aux_mu.  nullptr if the stream or events cannot be made.
AuxStream* aux_stream(int dev) {
  AuxStream& a = g_aux[dev];
  if (!a.ok) {
    if (cudaStreamCreateWithFlags(&a.s, cudaStreamNonBlocking) != cudaSuccess ||
        cudaEventCreateWithFlags(&a.fork, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&a.join, cudaEventDisableTiming) != cudaSuccess) {
      cudaGetLastError();
      return nullptr;
    }
    a.ok = true;
  }
  return &a;
}

// Whether work of a call on stream st may go to the second stream: it must
// not be inside a stream capture other than st's own.  A capture that st
// runs takes the second stream in through the fork event (and the graph then
// keeps the two branches); a capture that another caller left open on it
// must not receive this call's kernel, which then stays on st.
bool aux_usable(cudaStream_t st, cudaStream_t aux) {
  cudaStreamCaptureStatus sa = cudaStreamCaptureStatusNone, ss = cudaStreamCaptureStatusNone;
  unsigned long long ida = 0, ids = 0;
  if (cudaStreamGetCaptureInfo(aux, &sa, &ida) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  if (sa == cudaStreamCaptureStatusNone) return true;
  if (cudaStreamGetCaptureInfo(st, &ss, &ids) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  return sa == cudaStreamCaptureStatusActive && ss == cudaStreamCaptureStatusActive && ids == ida;
}

// Persistent quantizer: one CTA per SM (its shared-memory ring fills most of
// the SM), never more CTAs than groups.
template <int kMode>
int launch_quantize(int64_t groups, int sms, int dev, cudaStream_t st, const float* W, int64_t n_blocks,
                    uint8_t* codes, uint8_t* q8, float* s2) {
  auto kern = quantize_nf4_kernel<kMode>;
  static std::atomic<bool> attr_set[kMaxDevices];   // one-time setup done (stored last)
  if (!attr_set[dev]) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, sizeof(QuantSmem)) != cudaSuccess) {
      cudaGetLastError();
      return QLORA_ERR_CUDA;
    }
    attr_set[dev] = true;
  }
  const int64_t grid = std::min<int64_t>(groups, sms);
  return launch_ex(kern, dim3(static_cast<unsigned>(grid)), dim3(kQuantThreads), sizeof(QuantSmem), st, 1, 1, W,
                   n_blocks, groups, codes, q8, s2, tables());
}

extern "C" {

const char* qlora_strerror(int code) {
  switch (code) {
    case QLORA_OK: return "ok";
    case QLORA_ERR_INVALID_ARG: return "invalid argument (NULL pointer, r or alpha out of range)";
    case QLORA_ERR_UNSUPPORTED_SHAPE: return "unsupported shape or alignment (K, N multiple of 64; r multiple of 8; 16-byte aligned pointers)";
    case QLORA_ERR_CUDA: return "CUDA runtime error";
    case QLORA_ERR_DEVICE_TIMEOUT: return "a kernel's bounded wait expired";
    case QLORA_ERR_WORKSPACE: return "workspace missing or too small";
    case QLORA_ERR_NO_DEVICE: return "no sm_100 device is current";
    case QLORA_ERR_UNAVAILABLE: return "available in the checked build (libqlora_nf4_debug.so) only";
    default: return "unknown error code";
  }
}

int qlora_debug_record(int64_t* out) {
#ifdef QLORA_DEBUG
  if (!out) return QLORA_ERR_INVALID_ARG;
  int dev, sms;
  if (int rc = check_device(&dev, &sms)) return rc;
  unsigned long long h[4];
  const unsigned long long zero[4] = {0ull, 0ull, 0ull, 0ull};
  if (cudaMemcpyFromSymbol(h, qlora::g_debug_record, sizeof(h)) != cudaSuccess ||
      cudaMemcpyToSymbol(qlora::g_debug_record, zero, sizeof(zero)) != cudaSuccess) {
    cudaGetLastError();
    return QLORA_ERR_CUDA;
  }
  for (int i = 0; i < 4; ++i) out[i] = static_cast<int64_t>(h[i]);
  return QLORA_OK;
#else
  (void)out;
  return QLORA_ERR_UNAVAILABLE;
#endif
}

int qlora_nf4_codebook(float* out) {
  if (!out) return QLORA_ERR_INVALID_ARG;
  std::memcpy(out, tables().level, sizeof(float) * 16);
  return QLORA_OK;
}

int qlora_quantize_nf4_dq(const float* W, int64_t n_out, int64_t k_in, uint8_t* codes, uint8_t* q8, float* s2,
                          void* stream) {
  bool empty;
  if (int rc = check_weight_shape(n_out, k_in, &empty)) return rc;
  if (empty) return QLORA_OK;
  if (!W || !codes || !q8 || !s2) return QLORA_ERR_INVALID_ARG;
  if (!aligned16(W) || (reinterpret_cast<uintptr_t>(codes) & 3u) || (reinterpret_cast<uintptr_t>(s2) & 3u))
    return QLORA_ERR_UNSUPPORTED_SHAPE;
  int dev, sms;
  if (int rc = check_device(&dev, &sms)) return rc;
  const int64_t n_blocks = n_out * k_in / kBlock;
  const int64_t groups = (n_blocks + kGroup - 1) / kGroup;
  if (groups > INT32_MAX) return QLORA_ERR_UNSUPPORTED_SHAPE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return timed(QLORA_KERNEL_QUANTIZE, st, [&] {
    return launch_quantize<kQuantLinear8>(groups, sms, dev, st, W, n_blocks, codes, q8, s2);
  });
}

int qlora_quantize_nf4_dq_fp8(const float* W, int64_t n_out, int64_t k_in, uint8_t* codes, uint8_t* q8, float* s2,
                              void* stream) {
  bool empty;
  if (int rc = check_weight_shape(n_out, k_in, &empty)) return rc;
  if (empty) return QLORA_OK;
  if (!W || !codes || !q8 || !s2) return QLORA_ERR_INVALID_ARG;
  if (!aligned16(W) || (reinterpret_cast<uintptr_t>(codes) & 3u) || (reinterpret_cast<uintptr_t>(s2) & 3u))
    return QLORA_ERR_UNSUPPORTED_SHAPE;
  int dev, sms;
  if (int rc = check_device(&dev, &sms)) return rc;
  const int64_t n_blocks = n_out * k_in / kBlock;
  const int64_t groups = (n_blocks + kGroup - 1) / kGroup;
  if (groups > INT32_MAX) return QLORA_ERR_UNSUPPORTED_SHAPE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return timed(QLORA_KERNEL_QUANTIZE, st, [&] {
    return launch_quantize<kQuantFp8>(groups, sms, dev, st, W, n_blocks, codes, q8, s2);
  });
}

int qlora_quantize_nf4(const float* W, int64_t n_out, int64_t k_in, uint8_t* codes, float* absmax, void* stream) {
  bool empty;
  if (int rc = check_weight_shape(n_out, k_in, &empty)) return rc;
  if (empty) return QLORA_OK;
  if (!W || !codes || !absmax) return QLORA_ERR_INVALID_ARG;
  if (!aligned16(W) || (reinterpret_cast<uintptr_t>(codes) & 3u) || (reinterpret_cast<uintptr_t>(absmax) & 3u))
    return QLORA_ERR_UNSUPPORTED_SHAPE;
  int dev, sms;
  if (int rc = check_device(&dev, &sms)) return rc;
  const int64_t n_blocks = n_out * k_in / kBlock;
  const int64_t groups = (n_blocks + kGroup - 1) / kGroup;
  if (groups > INT32_MAX) return QLORA_ERR_UNSUPPORTED_SHAPE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* no_q8 = nullptr;
  return timed(QLORA_KERNEL_QUANTIZE, st, [&] {
    return launch_quantize<kQuantSingle>(groups, sms, dev, st, W, n_blocks, codes, no_q8, absmax);
  });
}

int qlora_merge_adapter(const float* W, int64_t n_out, int64_t k_in, const uint16_t* A, const uint16_t* B, int r,
                        float alpha, void* out, int out_dtype, void* stream) {
  if (out_dtype != QLORA_OUT_BF16 && out_dtype != QLORA_OUT_FP32) return QLORA_ERR_INVALID_ARG;
  if (r < 1 || r > 256 || !std::isfinite(alpha)) return QLORA_ERR_INVALID_ARG;
  bool empty;
  if (int rc = check_weight_shape(n_out, k_in, &empty)) return rc;
  if (n_out > (1 << 24) || k_in > (1 << 24)) return QLORA_ERR_UNSUPPORTED_SHAPE;
  if (empty) return QLORA_OK;
  if (!W || !A || !B || !out) return QLORA_ERR_INVALID_ARG;
  if (!aligned16(W) || !aligned16(A) || !aligned16(B) || !aligned16(out)) return QLORA_ERR_UNSUPPORTED_SHAPE;
  int dev, sms;
  if (int rc = check_device(&dev, &sms)) return rc;
  const double s = static_cast<double>(alpha / static_cast<float>(r));
  if ((n_out + kMergeRows - 1) / kMergeRows > 65535) return QLORA_ERR_UNSUPPORTED_SHAPE;   // grid y
  const dim3 grid(static_cast<unsigned>((k_in + kMergeCols - 1) / kMergeCols),
                  static_cast<unsigned>((n_out + kMergeRows - 1) / kMergeRows));
  const size_t smem = sizeof(double) * kMergeRows * static_cast<size_t>(r);   // <= 32 KiB
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return timed(QLORA_KERNEL_MERGE, st, [&] {
    if (out_dtype == QLORA_OUT_BF16)
      return launch_ex(merge_adapter_kernel<true>, grid, dim3(kMergeCols), smem, st, 1, 1, W, n_out, k_in, A, B, r,
                       s, out);
    return launch_ex(merge_adapter_kernel<false>, grid, dim3(kMergeCols), smem, st, 1, 1, W, n_out, k_in, A, B, r,
                     s, out);
  });
}

int qlora_dequant(const uint8_t* codes, const uint8_t* q8, const float* s2, int64_t n_out, int64_t k_in,
                  void* out, int out_dtype, void* stream) {
  if (out_dtype != QLORA_OUT_BF16 && out_dtype != QLORA_OUT_FP32) return QLORA_ERR_INVALID_ARG;
  bool empty;
  if (int rc = check_weight_shape(n_out, k_in, &empty)) return rc;
  if (empty) return QLORA_OK;
  if (!codes || !s2 || !out) return QLORA_ERR_INVALID_ARG;   // q8 == NULL: single quantization
  if ((reinterpret_cast<uintptr_t>(codes) & 3u) || !aligned16(out)) return QLORA_ERR_UNSUPPORTED_SHAPE;
  int dev, sms;
  if (int rc = check_device(&dev, &sms)) return rc;
  const int64_t n_oct = n_out * k_in / 8;
  const int blocks = static_cast<int>(std::min<int64_t>((n_oct + 255) / 256, 64LL * sms));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return timed(QLORA_KERNEL_DEQUANT, st, [&] {
    if (out_dtype == QLORA_OUT_BF16)
      return launch_ex(dequant_kernel<true>, dim3(blocks), dim3(256), 0, st, 1, 1, codes, q8, s2, n_oct, out,
                       tables());
    return launch_ex(dequant_kernel<false>, dim3(blocks), dim3(256), 0, st, 1, 1, codes, q8, s2, n_oct, out,
                     tables());
  });
}

size_t qlora_workspace_bytes(int64_t M, int64_t n_out, int64_t k_in, int r) {
  if (M < 1 || n_out < 64 || k_in < 64 || r < 1 || r > 256) return 0;   // M == 0 needs no workspace
  int dev = 0, sms = 148;
  if (check_device(&dev, &sms) != QLORA_OK) sms = 148;
  return ws_layout(M, n_out, k_in, r, sms).total;
}

// The forward with (dr.on) or without dropout on the adapter input.
static int fwd_impl(const uint8_t* codes, const uint8_t* q8, const float* s2, int64_t n_out, int64_t k_in,
                    const uint16_t* X, int64_t M, const uint16_t* A, const uint16_t* B, int r, float alpha,
                    uint16_t* Y, uint16_t* U_save, void* workspace, size_t workspace_bytes, void* stream,
                    const DropoutSpec& dr) {
  if (int rc = check_weight(codes, q8, s2, n_out, k_in)) return rc;
  if (int rc = check_lora(X, M, A, B, r, alpha)) return rc;
  if (M == 0) return QLORA_OK;   // an empty batch: Y and U have no rows
  if (!Y) return QLORA_ERR_INVALID_ARG;
  if (!aligned16(Y) || (U_save && !aligned16(U_save))) return QLORA_ERR_UNSUPPORTED_SHAPE;
  int dev, sms;
  if (int rc = check_device(&dev, &sms)) return rc;
  const WsLayout L = ws_layout(M, n_out, k_in, r, sms, dr.on);
  if (!workspace || workspace_bytes < L.total || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return QLORA_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint16_t* Us = reinterpret_cast<uint16_t*>(ws + L.us);
  const float s = alpha / static_cast<float>(r);
  const int rpad = (r + 63) / 64 * 64;

  // one to four tokens: table-lookup kernel (two launches); measured faster than the
  // tensor-memory kernel below up to four tokens (decode_lut.cuh)
  if (M <= kLutRouteTokens && !dr.on) {
    const int rc = run_decode_lut(codes, q8, s2, n_out, k_in, X, M, A, B, r, s, Y, U_save,
                                  reinterpret_cast<float*>(ws + L.v), sms, st, dev);
    if (rc != QLORA_ERR_UNSUPPORTED_SHAPE) return rc;
  }
  // a few tokens: one launch, weight rows on the MMA's M side, U computed in-kernel
  if (M <= kDecMaxTokens && r <= kDecMaxRank && !dr.on)
    return run_decode(codes, q8, s2, n_out, k_in, X, M, A, B, r, s, Y, U_save, st, dev);

  // the pair path's tiles, and whether U can run beside the fused kernel
  const int mh = M > 256 ? 2 : 1;
  const int pairs = static_cast<int>((M + 256 * mh - 1) / (256 * mh)) * static_cast<int>((n_out + 255) / 256);
  const bool beside = M > 128 && adapter_beside(M, rpad, pairs, sms);
  if (dr.on) {
    // the adapter's input goes through dropout: U = (X * keep) A^T / (1 - p)
    uint16_t* Xm = dr.xd ? dr.xd : reinterpret_cast<uint16_t*>(ws + L.xm);
    if (int rc = launch_dropout_mask(X, M, k_in, dr, Xm, sms, st, dr.bits)) return rc;
    if (int rc = run_lora_down(Xm, M, k_in, A, r, dr.inv, s * dr.inv, U_save, Us, sms, st, dev, beside)) return rc;
  } else if (int rc = run_lora_down(X, M, k_in, A, r, 1.f, s, U_save, Us, sms, st, dev, beside)) {
    return rc;
  }

  GemmArgs g{};
  g.m_rows = static_cast<int>(M);
  g.n_cols = static_cast<int>(n_out);
  g.k_steps = static_cast<int>(k_in / 64);
  g.steps_per_split = g.k_steps;
  g.n_lora = rpad / 64;
  g.q8 = q8;
  g.s2 = s2;
  g.w_rows = static_cast<int>(n_out);
  g.w_kblocks = static_cast<int>(k_in / 64);
  fill_levels(g);
  g.out = Y;
  g.ld_out = n_out;
  g.split_stride = 0;
  if (M > 128) {
    // CTA pairs: tile (256*MH) x 256, each CTA expanding 128 weight rows per step
    CUtensorMap tx, tp, tus, tb;
    if (!map_bf16(&tx, X, M, k_in, 64, 128) ||
        !make_map(&tp, CU_TENSOR_MAP_DATA_TYPE_UINT8, codes, k_in / 2, n_out, k_in / 2, 32, 128,
                  CU_TENSOR_MAP_SWIZZLE_32B) ||
        !map_bf16(&tus, Us, M, r, 64, 128) || !map_bf16(&tb, B, n_out, r, 64, 128))
      return QLORA_ERR_CUDA;
    return mh == 2 ? launch_pair<kBDeqK, 2>(pairs, tx, tp, tus, tb, g, st, dev)
                   : launch_pair<kBDeqK, 1>(pairs, tx, tp, tus, tb, g, st, dev);
  }
  CUtensorMap tx, tp, tus, tb;
  if (!map_bf16(&tx, X, M, k_in, 64, 128) ||
      !make_map(&tp, CU_TENSOR_MAP_DATA_TYPE_UINT8, codes, k_in / 2, n_out, k_in / 2, 32, 256,
                CU_TENSOR_MAP_SWIZZLE_32B) ||
      !map_bf16(&tus, Us, M, r, 64, 128) || !map_bf16(&tb, B, n_out, r, 64, 256))
    return QLORA_ERR_CUDA;
  // small M: split the reduction over a cluster of up to 8 CTAs (DSMEM sum)
  const int tiles = static_cast<int>((M + 127) / 128) * static_cast<int>((n_out + 255) / 256);
  const int S = gemm_split<kBDeqK>(tiles, g.k_steps, dev);
  g.steps_per_split = (g.k_steps + S - 1) / S;
  const dim3 grid(static_cast<unsigned>((M + 127) / 128), static_cast<unsigned>((n_out + 255) / 256),
                  static_cast<unsigned>(S));
  return launch_gemm<256, 4, false, kBDeqK, kOutBf16, 8, 1>(grid, tx, tp, tus, tb, g, st, dev);
}

int qlora_linear_fwd(const uint8_t* codes, const uint8_t* q8, const float* s2, int64_t n_out, int64_t k_in,
                     const uint16_t* X, int64_t M, const uint16_t* A, const uint16_t* B, int r, float alpha,
                     uint16_t* Y, uint16_t* U_save, void* workspace, size_t workspace_bytes, void* stream) {
  return fwd_impl(codes, q8, s2, n_out, k_in, X, M, A, B, r, alpha, Y, U_save, workspace, workspace_bytes, stream,
                  DropoutSpec{});
}

// The kept dropout state: the masked input and the keep bits, both or neither.
static int dropout_state(const void* xd, const void* bits, DropoutSpec* dr) {
  if ((xd == nullptr) != (bits == nullptr)) return QLORA_ERR_INVALID_ARG;
  if ((xd && !aligned16(xd)) || (bits && !aligned16(bits))) return QLORA_ERR_UNSUPPORTED_SHAPE;
  if (dr->on) {
    dr->xd = const_cast<uint16_t*>(static_cast<const uint16_t*>(xd));
    dr->bits = const_cast<uint16_t*>(static_cast<const uint16_t*>(bits));
  }
  return QLORA_OK;
}

int qlora_linear_fwd_dropout(const uint8_t* codes, const uint8_t* q8, const float* s2, int64_t n_out, int64_t k_in,
                             const uint16_t* X, int64_t M, const uint16_t* A, const uint16_t* B, int r, float alpha,
                             float p, uint64_t seed, uint64_t offset, uint16_t* Y, uint16_t* U_save,
                             uint16_t* Xd_save, uint32_t* keep_save, void* workspace, size_t workspace_bytes,
                             void* stream) {
  DropoutSpec dr;
  if (!make_dropout(p, seed, offset, &dr)) return QLORA_ERR_INVALID_ARG;
  if (int rc = dropout_state(Xd_save, keep_save, &dr)) return rc;
  return fwd_impl(codes, q8, s2, n_out, k_in, X, M, A, B, r, alpha, Y, U_save, workspace, workspace_bytes, stream,
                  dr);
}

// Forward with the library's own fixed scratch instead of a caller workspace:
// for callers that cannot allocate device memory (see include/qlora_nf4.h).
int qlora_linear_fwd_noalloc(const uint8_t* codes, const uint8_t* q8, const float* s2, int64_t n_out,
                             int64_t k_in, const uint16_t* X, int64_t M, const uint16_t* A, const uint16_t* B,
                             int r, float alpha, uint16_t* Y, uint16_t* U_save, void* stream) {
  if (int rc = check_weight(codes, q8, s2, n_out, k_in)) return rc;
  if (int rc = check_lora(X, M, A, B, r, alpha)) return rc;
  if (M == 0) return QLORA_OK;   // an empty batch: nothing to compute
  if (!Y) return QLORA_ERR_INVALID_ARG;
  int dev, sms;
  if (int rc = check_device(&dev, &sms)) return rc;
  const size_t need = ws_layout(M, n_out, k_in, r, sms).total;
  if (need > kNoAllocScratchBytes) return QLORA_ERR_WORKSPACE;  // beyond the fixed 4 MiB
  void* scratch = noalloc_scratch(dev);
  if (!scratch) return QLORA_ERR_CUDA;
  return qlora_linear_fwd(codes, q8, s2, n_out, k_in, X, M, A, B, r, alpha, Y, U_save, scratch,
                          kNoAllocScratchBytes, stream);
}

// The backward with (dr.on) or without dropout on the adapter input.
static int bwd_impl(const uint8_t* codes, const uint8_t* q8, const float* s2, int64_t n_out, int64_t k_in,
                    const uint16_t* X, int64_t M, const uint16_t* A, const uint16_t* B, int r, float alpha,
                    const uint16_t* dY, const uint16_t* U_saved, uint16_t* dX, float* dA, float* dB,
                    void* workspace, size_t workspace_bytes, void* stream, const DropoutSpec& dr) {
  if (int rc = check_weight(codes, q8, s2, n_out, k_in)) return rc;
  if (int rc = check_lora(X, M, A, B, r, alpha)) return rc;
  if ((M != 0 && !dY) || !dA || !dB) return QLORA_ERR_INVALID_ARG;
  if ((dY && !aligned16(dY)) || !aligned16(dA) || !aligned16(dB) || (U_saved && !aligned16(U_saved)) ||
      (dX && !aligned16(dX)))
    return QLORA_ERR_UNSUPPORTED_SHAPE;
  int dev, sms;
  if (int rc = check_device(&dev, &sms)) return rc;
  if (M == 0) {
    // an empty batch: the sums over tokens that make dA and dB are empty, so both are zero
    cudaStream_t st0 = static_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(dA, 0, sizeof(float) * static_cast<size_t>(r) * static_cast<size_t>(k_in), st0) != cudaSuccess ||
        cudaMemsetAsync(dB, 0, sizeof(float) * static_cast<size_t>(n_out) * static_cast<size_t>(r), st0) != cudaSuccess) {
      cudaGetLastError();
      return QLORA_ERR_CUDA;
    }
    return QLORA_OK;
  }
  const WsLayout L = ws_layout(M, n_out, k_in, r, sms, dr.on);
  if (!workspace || workspace_bytes < L.total || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return QLORA_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint16_t* V = reinterpret_cast<uint16_t*>(ws + L.v);
  uint16_t* Vs = reinterpret_cast<uint16_t*>(ws + L.vs);
  uint16_t* Ubuf = reinterpret_cast<uint16_t*>(ws + L.u);
  const float s = alpha / static_cast<float>(r);
  const int rpad = (r + 63) / 64 * 64;
  const int N = static_cast<int>(n_out), K = static_cast<int>(k_in);

  // the adapter's input: X, or X * keep with dropout (the 1/(1-p) goes into the scales); the
  // keep bits are read by the masked dX term.  Both come from the forward when it kept them.
  const uint16_t* Xa = X;
  const uint16_t* keep_bits = nullptr;
  if (dr.on && dr.xd) {
    Xa = dr.xd;
    keep_bits = dr.bits;
  } else if (dr.on) {
    uint16_t* Xm = reinterpret_cast<uint16_t*>(ws + L.xm);
    uint16_t* bits = reinterpret_cast<uint16_t*>(ws + L.bits);
    if (int rc = launch_dropout_mask(X, M, K, dr, Xm, sms, st, bits)) return rc;
    Xa = Xm;
    keep_bits = bits;
  }
  // U (from the forward, or recomputed)
  const uint16_t* U = U_saved;
  if (!U) {
    // the forward's grid for U (split or not), so the recomputed U is bit-identical to a saved one
    const int fmh = M > 256 ? 2 : 1;
    const int fwd_pairs = static_cast<int>((M + 256 * fmh - 1) / (256 * fmh)) * ((N + 255) / 256);
    const bool fwd_beside = M > 128 && adapter_beside(M, rpad, fwd_pairs, sms);
    if (int rc = run_lora_down(Xa, M, K, A, r, dr.inv, s, Ubuf, nullptr, sms, st, dev, fwd_beside)) return rc;
    U = Ubuf;
  }
  // V = dY B  (B viewed MN-major: its rows are the reduction index)
  {
    CUtensorMap ta, tb;
    if (!map_bf16(&ta, dY, M, N, 64, 128) || !map_bf16(&tb, B, N, r, 64, 64)) return QLORA_ERR_CUDA;
    const int k_steps = N / 64;
    const int tiles = static_cast<int>((M + 127) / 128) * (rpad / 64);
    // The grid depends on the shapes alone, so V (and with it dA) is the same
    // bit for bit whichever outputs are requested.  V is launched last before dX
    // (after any mask pass and U recompute), so it can run beside dX.
    const int mh = M > 256 ? 2 : 1;
    const int pairs = static_cast<int>((M + 256 * mh - 1) / (256 * mh)) * ((K + 255) / 256);
    const bool beside = kVBesideDx && M > 128 && adapter_beside(M, rpad, pairs, sms);
    const int S = beside ? 1 : lora_cluster(tiles, k_steps, sms);
    LoraArgs la{};
    la.p[0] = lora_problem(static_cast<int>(M), k_steps, S, rpad, kLoraOutPlainScaled, V, Vs, 0, 1.f, s);
    la.p[1] = la.p[0];
    la.p[1].tiles_m = 0;   // no second problem: a CTA padding the grid has no tile
    la.tiles0 = tiles;
    la.r = r;
    if (int rc = launch_lora<false, true>(ta, tb, ta, tb, la, tiles, S, st, dev, QLORA_KERNEL_LORA_GEMM,
                                          beside ? 2 : 1))
      return rc;
  }
  // The gradient kernel goes to the device's second stream, forked here and
  // launched after dX so that dX's CTAs are queued first; with per-kernel
  // timing on, every kernel stays on the caller's stream (each timed alone),
  // and so does it while another caller's capture holds the second stream.
  std::unique_lock<std::mutex> aux_lk(g_aux_mu, std::defer_lock);
  AuxStream* aux = nullptr;
  if (!g_timing_on && dX) {
    aux_lk.lock();
    aux = aux_stream(dev);
    if (aux && !aux_usable(st, aux->s)) aux = nullptr;
    if (aux && cudaEventRecord(aux->fork, st) != cudaSuccess) {
      cudaGetLastError();
      return QLORA_ERR_CUDA;
    }
  }
  // dX = dY dequant(W) + (s V) A; with dropout the adapter term is masked, so
  // the fused kernel computes dY dequant(W) alone and a tensor-core GEMM V A
  // adds s/(1-p) (V A) where the input was kept (masked-add epilogue)
  if (dX) {
    GemmArgs g{};
    g.m_rows = static_cast<int>(M);
    g.n_cols = K;
    g.k_steps = N / 64;
    g.steps_per_split = g.k_steps;
    g.n_lora = dr.on ? 0 : rpad / 64;
    g.q8 = q8;
    g.s2 = s2;
    g.w_rows = N;
    g.w_kblocks = K / 64;
    fill_levels(g);
    g.out = dX;
    g.ld_out = K;
    int rc;
    if (M > 128) {
      const int mh = M > 256 ? 2 : 1;
      CUtensorMap ta, tp, ta2, tb2;
      if (!map_bf16(&ta, dY, M, N, 64, 128) ||
          !make_map(&tp, CU_TENSOR_MAP_DATA_TYPE_UINT8, codes, K / 2, N, K / 2, 64, 64, CU_TENSOR_MAP_SWIZZLE_64B) ||
          !map_bf16(&ta2, Vs, M, r, 64, 128) || !map_bf16(&tb2, A, r, K, 64, 64))
        return QLORA_ERR_CUDA;
      const int pairs = static_cast<int>((M + 256 * mh - 1) / (256 * mh)) * ((K + 255) / 256);
      rc = mh == 2 ? launch_pair<kBDeqMN, 2>(pairs, ta, tp, ta2, tb2, g, st, dev)
                   : launch_pair<kBDeqMN, 1>(pairs, ta, tp, ta2, tb2, g, st, dev);
    } else {
      CUtensorMap ta, tp, ta2, tb2;
      if (!map_bf16(&ta, dY, M, N, 64, 128) ||
          !make_map(&tp, CU_TENSOR_MAP_DATA_TYPE_UINT8, codes, K / 2, N, K / 2, 128, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
          !map_bf16(&ta2, Vs, M, r, 64, 128) || !map_bf16(&tb2, A, r, K, 64, 64))
        return QLORA_ERR_CUDA;
      const int tiles = static_cast<int>((M + 127) / 128) * ((K + 255) / 256);
      const int S = gemm_split<kBDeqMN>(tiles, g.k_steps, dev);
      g.steps_per_split = (g.k_steps + S - 1) / S;
      const dim3 grid(static_cast<unsigned>((M + 127) / 128), static_cast<unsigned>((K + 255) / 256),
                      static_cast<unsigned>(S));
      rc = launch_gemm<256, 4, false, kBDeqMN, kOutBf16, 8, 1>(grid, ta, tp, ta2, tb2, g, st, dev);
    }
    if (rc) return rc;
    if (dr.on) {
      // D = V A: A operand V (M x r, K-major), B operand the adapter's A (r x K, MN-major);
      // r is one to four reduction steps of 64 (zero-filled past r)
      CUtensorMap tv, ta, tdx;
      if (!map_bf16(&tv, V, M, r, 64, 128) || !map_bf16(&ta, A, r, K, 64, 64) || !map_bf16(&tdx, dX, M, K, 64, 128))
        return QLORA_ERR_CUDA;
      GemmArgs gd{};
      gd.m_rows = static_cast<int>(M);
      gd.n_cols = K;
      gd.k_steps = rpad / 64;
      gd.steps_per_split = gd.k_steps;
      gd.n_lora = 0;
      gd.out = dX;
      gd.ld_out = K;
      gd.drop_scale = s * dr.inv;
      gd.drop_bits = reinterpret_cast<const uint32_t*>(keep_bits);
      // 128 x 128 tiles, one stage, four epilogue warps: two CTAs per SM, so one CTA's
      // loads overlap another's masked update
      const dim3 grid(static_cast<unsigned>((M + 127) / 128), static_cast<unsigned>((K + 127) / 128), 1);
      rc = launch_gemm<128, 1, false, kBTmaMN, kOutDropoutAdd, 4, 1>(grid, tv, ta, tdx, ta, gd, st, dev);
      if (rc) return rc;
    }
  }
  // dA^T = X^T V and dB = dY^T U in one grouped launch, reduced over M (X * keep and s/(1-p)
  // for dA with dropout)
  {
    CUtensorMap ta0, tb0, ta1, tb1;
    if (!map_bf16(&ta0, Xa, M, K, 64, 64) || !map_bf16(&tb0, V, M, r, 64, 64) ||
        !map_bf16(&ta1, dY, M, N, 64, 64) || !map_bf16(&tb1, U, M, r, 64, 64))
      return QLORA_ERR_CUDA;
    const int k_steps = static_cast<int>((M + 63) / 64);
    const int tiles_a = ((K + 127) / 128) * (rpad / 64);
    const int tiles_b = ((N + 127) / 128) * (rpad / 64);
    // With dX on the CTA-pair path the gradient kernel runs beside it (second
    // stream) in the slots of dX's last wave: unsplit there, two tiles per TPC,
    // it takes fewer SM-microseconds than split (train4096 step 238.0 -> 232.0
    // us) although it is slower alone.  The grid depends on the shapes alone,
    // so dA and dB have the same bits with or without dX.
    const bool unsplit = M > 128;
    const int S = unsplit ? 1 : lora_cluster(tiles_a + tiles_b, k_steps, sms);
    LoraArgs la{};
    la.p[0] = lora_problem(K, k_steps, S, rpad, kLoraOutTransposed, dA, nullptr, K, 1.f, s * dr.inv);
    la.p[1] = lora_problem(N, k_steps, S, rpad, kLoraOutRowMajor, dB, nullptr, 0, 1.f, s);
    la.tiles0 = tiles_a;
    la.r = r;
    cudaStream_t gst = st;
    if (aux) {
      if (cudaStreamWaitEvent(aux->s, aux->fork, 0) != cudaSuccess) {
        cudaGetLastError();
        return QLORA_ERR_CUDA;
      }
      gst = aux->s;
    }
    const int rc = launch_lora<true, true>(ta0, tb0, ta1, tb1, la, tiles_a + tiles_b, S, gst, dev,
                                           QLORA_KERNEL_GRAD_GEMM, unsplit ? 2 : 1);
    // the second stream joins back even when the launch failed, so that a capture on the
    // caller's stream never ends with an unjoined branch
    if (aux && (cudaEventRecord(aux->join, aux->s) != cudaSuccess || cudaStreamWaitEvent(st, aux->join, 0) != cudaSuccess)) {
      cudaGetLastError();
      return rc ? rc : QLORA_ERR_CUDA;
    }
    if (rc) return rc;
  }
  return QLORA_OK;
}

int qlora_linear_bwd(const uint8_t* codes, const uint8_t* q8, const float* s2, int64_t n_out, int64_t k_in,
                     const uint16_t* X, int64_t M, const uint16_t* A, const uint16_t* B, int r, float alpha,
                     const uint16_t* dY, const uint16_t* U_saved, uint16_t* dX, float* dA, float* dB,
                     void* workspace, size_t workspace_bytes, void* stream) {
  return bwd_impl(codes, q8, s2, n_out, k_in, X, M, A, B, r, alpha, dY, U_saved, dX, dA, dB, workspace,
                  workspace_bytes, stream, DropoutSpec{});
}

int qlora_linear_bwd_dropout(const uint8_t* codes, const uint8_t* q8, const float* s2, int64_t n_out, int64_t k_in,
                             const uint16_t* X, int64_t M, const uint16_t* A, const uint16_t* B, int r, float alpha,
                             float p, uint64_t seed, uint64_t offset, const uint16_t* dY, const uint16_t* U_saved,
                             const uint16_t* Xd_saved, const uint32_t* keep_saved, uint16_t* dX, float* dA, float* dB,
                             void* workspace, size_t workspace_bytes, void* stream) {
  DropoutSpec dr;
  if (!make_dropout(p, seed, offset, &dr)) return QLORA_ERR_INVALID_ARG;
  if (int rc = dropout_state(Xd_saved, keep_saved, &dr)) return rc;
  return bwd_impl(codes, q8, s2, n_out, k_in, X, M, A, B, r, alpha, dY, U_saved, dX, dA, dB, workspace,
                  workspace_bytes, stream, dr);
}

size_t qlora_workspace_bytes_dropout(int64_t M, int64_t n_out, int64_t k_in, int r) {
  if (M < 1 || n_out < 64 || k_in < 64 || r < 1 || r > 256) return 0;
  int dev = 0, sms = 148;
  if (check_device(&dev, &sms) != QLORA_OK) sms = 148;
  return ws_layout(M, n_out, k_in, r, sms, true).total;
}

int qlora_dropout_apply(const uint16_t* X, int64_t M, int64_t k_in, float p, uint64_t seed, uint64_t offset,
                        uint16_t* out, void* stream) {
  if (M < 0 || k_in <= 0 || k_in % 64 != 0) return QLORA_ERR_UNSUPPORTED_SHAPE;
  DropoutSpec dr;
  if (!make_dropout(p, seed, offset, &dr)) return QLORA_ERR_INVALID_ARG;
  if (M == 0) return QLORA_OK;   // an empty batch
  if (!X || !out) return QLORA_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(out)) return QLORA_ERR_UNSUPPORTED_SHAPE;
  int dev, sms;
  if (int rc = check_device(&dev, &sms)) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (!dr.on) dr.t = 0;   // p == 0: every element kept (the same kernel, threshold 0)
  return launch_dropout_mask(X, M, k_in, dr, out, sms, st);
}

int64_t qlora_launch_count(void) { return g_launch_count.load(std::memory_order_relaxed); }

int qlora_timing_enable(int on) {
  std::lock_guard<std::mutex> lk(g_timing_mu);
  for (auto& r : g_timing_recs) {
    g_event_pool.push_back(r.start);
    g_event_pool.push_back(r.stop);
  }
  g_timing_recs.clear();
  g_timing_on = on != 0;
  return QLORA_OK;
}

int qlora_timing_collect(double* ms, int64_t* counts, int n_kinds) {
  if (!ms || !counts || n_kinds < QLORA_KERNEL_COUNT) return QLORA_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lk(g_timing_mu);
  int rc = QLORA_OK;
  for (auto& r : g_timing_recs) {
    float t = 0.f;
    if (cudaEventSynchronize(r.stop) != cudaSuccess || cudaEventElapsedTime(&t, r.start, r.stop) != cudaSuccess) {
      cudaGetLastError();
      rc = QLORA_ERR_CUDA;
    } else {
      ms[r.kind] += t;
      counts[r.kind] += 1;
    }
    g_event_pool.push_back(r.start);
    g_event_pool.push_back(r.stop);
  }
  g_timing_recs.clear();
  return rc;
}

int qlora_selftest_device_timeout(unsigned long long* waited_ns, void* stream) {
  int dev, sms;
  if (int rc = check_device(&dev, &sms)) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  selftest_wait_kernel<<<1, 32, 0, st>>>(waited_ns);
  if (cudaGetLastError() != cudaSuccess) return QLORA_ERR_CUDA;
  g_launch_count.fetch_add(1, std::memory_order_relaxed);
  return QLORA_OK;
}

int qlora_device_status(void* stream) {
  int dev, sms;
  if (int rc = check_device(&dev, &sms)) return rc;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) {
    cudaGetLastError();
    return QLORA_ERR_CUDA;
  }
  int flag = 0;
  if (cudaMemcpyFromSymbol(&flag, g_device_error, sizeof(int)) != cudaSuccess) return QLORA_ERR_CUDA;
  if (flag) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_device_error, &zero, sizeof(int)) != cudaSuccess) return QLORA_ERR_CUDA;
    return QLORA_ERR_DEVICE_TIMEOUT;
  }
  return QLORA_OK;
}

}  // extern "C"
