// Small-M forward of the NF4 linear layer (a few tokens against a large frozen
// weight: the bandwidth-bound "decode" shapes), sm_100a.
//
//   Y = X dequant(W)^T + s (X A^T) B^T,   M <= 32 tokens, r <= 64
//
// At small M the packed weight stream is the whole cost, so the layout is
// turned around: the MMA's 128-row side holds weight rows (and adapter rows,
// below) and its N side is the M tokens padded to MP (16 or 32).  An MMA
// instruction of this shape costs about as much as one with N = 64 no
// matter how few tokens there are, so the kernel is organised to issue as few
// of them as possible:
//
// * Adapter rows share the MMA with the weight rows.  The 128 TMEM lanes of
//   the A operand are r rows of the adapter's A followed by T = 128 - r weight
//   rows, so one MMA per 16-wide slice of K yields both the partial U_z^T =
//   A[:, Kz] X[:, Kz]^T (lanes < r) and the partial Y_z^T (lanes >= r).  A
//   CTA owns T weight rows [c0, c0+T) and one K range Kz.
// * The A operand lives in tensor memory: a thread owns one TMEM lane (one
//   weight row, or one adapter row) and writes its 64 values of a k-step with
//   one tcgen05.st.  Shared memory holds only what TMA stages per k-step: the
//   packed codes of the T rows, the token tile and the adapter slice
//   A[:, k..k+64) (which every CTA reads, so it comes from L2).
//
// * A thread that waits on any barrier while its own MMAs are in flight
//   stalls until they drain, so two threads in different warps issue the
//   MMAs of alternate k-steps, each into its own accumulator (summed in the
//   epilogue); one issues while the other waits.
//
// The K ranges of a row tile form a cluster along z.  The adapter needs
// U = sum_z U_z, but its up-projection is linear in U, so every rank adds
// B[rows, :] (s U_z)^T to its own partial tile and the cluster sum yields
// s U B^T.  Each rank then sends its fp32 partials with st.async into the
// shared memory of the rank that owns those rows; the owner waits on a local
// mbarrier for the bytes it expects, adds the S partials in rank order and
// stores bf16 Y (and U, for the first row tile).  There is no cluster
// barrier at the end.
//
// * Filling a stage is a chain of dependent latencies (barrier wait, table,
//   expansion, tcgen05.st, its wait, fence, arrive), so four warpgroups take
//   every fourth k-step and each scheduler interleaves four such chains.
//
// Warp roles (608 threads):
//   warp 0        TMA producer (one elected lane)
//   warps 1, 2    MMA issuers for even / odd k-steps (one elected lane each);
//                 warp 1 also allocates TMEM
//   warps 3..18   fill the A operand; warpgroup g (warps 3+4g .. 6+4g) takes
//                 k-steps t = g mod 4.  Afterwards warps 8, 9 (lanes 0..63)
//                 turn U_z into the adapter operand, warps 3..6 send the
//                 partial tile, and warps 3..18 reduce the rows this rank
//                 owns.
// Every mbarrier wait is bounded (ptx_sm100.cuh).
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include "ptx_sm100.cuh"
#include "gemm_tc.cuh"

namespace qlora {

constexpr int kDecLanes = 128;       // TMEM lanes = rows of the MMA
constexpr int kDecMaxRank = 64;      // adapter rank handled by this kernel
constexpr int kDecMaxTokens = 32;    // tokens handled by this kernel
constexpr int kDecWG = 4;            // warpgroups filling the A operand
constexpr int kDecThreads = 96 + 128 * kDecWG;
constexpr int kDecStages = 8;        // a multiple of kDecWG: a stage always belongs to one warpgroup
constexpr int kDecACols = 32;        // TMEM columns of one 128 x 64 bf16 A stage

// Offset of the adapter slice from the packed codes within a stage.
__host__ __device__ constexpr int dec_a_off(int r) { return ((kDecLanes - r) * 32 + 1023) / 1024 * 1024; }

struct DecodeArgs {
  int m_rows;             // tokens M (<= MP)
  int n_cols;             // N: weight rows = columns of Y
  int k_steps;            // K / 64
  int steps_per_split;    // k-steps per cluster rank
  int r;                  // adapter rank (multiple of 8, <= 64)
  int tile_rows;          // T = 128 - r weight rows per CTA
  int slice_rows;         // rows of the tile each rank reduces and stores (multiple of 8)
  int slice_u;            // columns of U each rank of the first tile reduces and stores
  float s;                // alpha / r
  const uint8_t* q8;
  const float* s2;
  float level[16];        // NF4 levels (fp32)
  uint16_t* y;            // bf16 [M x N], rows ld_y elements apart
  int64_t ld_y;
  uint16_t* u_save;       // bf16 [M x r] (U = X A^T), or NULL
};

template <int MP>
struct DecodeSmem {
  static_assert(MP == 16 || MP == 32, "MP");
  // one stage: [token tile MP x 128 B, 128-byte swizzle]
  //            [packed codes, T rows x 32 B][adapter slice, r rows x 128 B, 128-byte swizzle]
  // the adapter slice starts at the first 1024-byte boundary after the codes:
  // roundup(32 (128 - r), 1024) + 128 r <= 10240 for every r in [8, 64]
  static constexpr int kXOff = 0;
  static constexpr int kPOff = MP * 128;
  static constexpr int kStageBytes = kPOff + 10240;
  static_assert(kStageBytes % 1024 == 0, "stages stay 1024-byte aligned");
  static constexpr int kBwOff = kDecStages * kStageBytes;    // B rows of the lanes x 64 (adapter up-projection)
  static constexpr int kSuOff = kBwOff + kDecLanes * 128;    // bf16(s U_z): MP x 64
  static constexpr int kRecvOff = kSuOff + MP * 128;         // fp32 [S][MP][slice_rows], S * slice_rows <= 192
  static constexpr int kRecvUOff = kRecvOff + MP * 192 * 4;  // fp32 [S][MP][slice_u],   S * slice_u <= 72
  static constexpr int kBarOff = kRecvUOff + MP * 72 * 4;
  static constexpr int kNumBars = 3 * kDecStages + 5;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kBytes = kMiscOff + 16;
  static constexpr int kDynBytes = kBytes + 1024;            // slack to align the base to 1024 B
  static_assert(kDynBytes <= 232448, "shared memory");
  // TMEM: A stages at columns [32 s, 32 s + 32), then the two accumulators
  static constexpr uint32_t kAccCol = kDecStages * kDecACols;
  static constexpr uint32_t kTmemCols = kAccCol + 2 * MP <= 256 ? 256 : 512;
};

// MP consecutive fp32 TMEM columns of the warp's 32 lanes.
template <int MP>
__device__ __forceinline__ void tmem_read_cols(uint32_t taddr, float (&out)[MP]) {
  if constexpr (MP == 16) {
    uint32_t v[16];
    tmem_ld_32x32b_x16(taddr, v);
    tmem_ld_wait();
#pragma unroll
    for (int i = 0; i < 16; ++i) out[i] = __uint_as_float(v[i]);
  } else {
#pragma unroll
    for (int c = 0; c < MP / 32; ++c) {
      uint32_t v[32];
      tmem_ld_32x32b_x32(taddr + 32 * c, v);
      tmem_ld_wait();
#pragma unroll
      for (int i = 0; i < 32; ++i) out[32 * c + i] = __uint_as_float(v[i]);
    }
  }
}

template <int MP>
__global__ void __launch_bounds__(kDecThreads, 1)
qlora_decode_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmP,
                    const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const DecodeArgs args) {
  using L = DecodeSmem<MP>;
  constexpr int NS = kDecStages;
  constexpr uint32_t kIdesc = idesc_bf16_m128(MP, 0u, 0u);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full_tma = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  uint64_t* full_w = full_tma + NS;
  uint64_t* empty = full_w + NS;
  uint64_t* mma_done = empty + NS;    // both issuers' main products have completed
  uint64_t* su_full = mma_done + 1;   // bf16(s U_z) written (warps 8, 9)
  uint64_t* bw_full = su_full + 1;    // B rows landed
  uint64_t* accum_full = bw_full + 1; // adapter product completed
  uint64_t* recv_full = accum_full + 1;  // every peer's partials for the rows this rank owns
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int r = args.r;
  const int T = args.tile_rows;
  const int c0 = blockIdx.x * T;
  const int step_begin = blockIdx.z * args.steps_per_split;
  const int step_end = min(args.k_steps, step_begin + args.steps_per_split);
  const int n_steps = max(0, step_end - step_begin);
  // the K ranges of a row tile are one cluster along z (none when there is one range)
  const bool clustered = gridDim.z > 1;
  const int S = static_cast<int>(gridDim.z);
  const int rank = clustered ? static_cast<int>(cluster_ctarank()) : 0;
  const int a_off = L::kPOff + dec_a_off(r);
  const int mv = min(args.m_rows, MP);
  const bool want_u = blockIdx.x == 0 && args.u_save != nullptr;
  const int sl = args.slice_rows;
  const int su_n = args.slice_u;
  const int own_rows = max(0, min(sl, T - rank * sl));
  const int own_cols = max(0, min(su_n, r - rank * su_n));

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full_tma[s], 1);
      mbar_init(&full_w[s], 4);
      mbar_init(&empty[s], 1);
    }
    mbar_init(mma_done, 2);
    mbar_init(su_full, 2);
    mbar_init(bw_full, 1);
    mbar_init(accum_full, 1);
    mbar_init(recv_full, 1);
    *abort_flag = 0;
    fence_barrier_init();
    // the bytes the peers will send: mv values of each owned row (and owned
    // U column) from every rank
    if (clustered)
      mbar_arrive_expect_tx(recv_full, static_cast<uint32_t>(S * mv * (own_rows + (want_u ? own_cols : 0)) * 4));
  }
  if (warp == 0 && lane == 0) {
    // descriptors are kernel parameters: fetch them while the previous grid finishes
    tma_prefetch_desc(&tmX);
    tma_prefetch_desc(&tmP);
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) tmem_alloc(tmem_slot, L::kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // barriers initialised and this CTA running: peers may send once they have
  // waited on this phase (every thread waits once, before any remote store)
  if (clustered) cluster_arrive_release();
  const uint32_t tmem_d = *tmem_slot;
  const uint32_t d_acc = tmem_d + L::kAccCol;   // accumulator p at d_acc + p * MP
  griddep_wait();   // no global access before the previous grid is complete

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      // B[c0 - r + lane, 0 .. 64) for TMEM lane `lane`: rows before 0 and
      // columns past r arrive as zeros; lanes < r are never read back
      mbar_arrive_expect_tx(bw_full, kDecLanes * 128);
      tma_load_2d(smem + L::kBwOff, &tmB, bw_full, 0, c0 - r);
      for (int t = 0; t < n_steps; ++t) {
        const int s = t % NS;
        if (t >= NS && !mbar_wait(&empty[s], ((t / NS) - 1) & 1, abort_flag)) break;
        const int ks = step_begin + t;
        uint8_t* st = smem + s * L::kStageBytes;
        mbar_arrive_expect_tx(&full_tma[s], MP * 128 + T * 32 + r * 128);
        tma_load_2d(st + L::kXOff, &tmX, &full_tma[s], ks * 64, 0);
        tma_load_2d(st + L::kPOff, &tmP, &full_tma[s], ks * 32, c0, 1);
        tma_load_2d(st + a_off, &tmA, &full_tma[s], ks * 64, 0);
      }
    }
    __syncwarp();
    if (clustered) cluster_wait();
  } else if (warp <= 2) {
    // ------------------------------------------------------------ MMA issuers
    const int p = warp - 1;                              // k-steps t = p, p + 2, ...
    const uint32_t d_mine = d_acc + static_cast<uint32_t>(p * MP);
    bool ok = true;
    for (int t = p; t < n_steps && ok; t += 2) {
      const int s = t % NS;
      const uint32_t ph = (t / NS) & 1;
      ok = mbar_wait(&full_tma[s], ph, abort_flag) && mbar_wait(&full_w[s], ph, abort_flag);
      if (!ok) break;
      tc_fence_after();
      if (lane == 0) {
        const uint32_t a_tm = tmem_d + static_cast<uint32_t>(s * kDecACols);
        const uint32_t x_base = smem_u32(smem + s * L::kStageBytes + L::kXOff);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          umma_bf16_tmem_a(d_mine, a_tm + kk * 8, smem_desc_sw128(x_base + kk * 32, 16), kIdesc,
                           (t > p || kk > 0) ? 1u : 0u);
        umma_commit(&empty[s]);
      }
      __syncwarp();
    }
    if (lane == 0) umma_commit(mma_done);
    __syncwarp();
    if (p == 0) {
      // adapter up-projection into accumulator 0: D += B[rows, :] (s U_z)^T
      if (ok) ok = mbar_wait(su_full, 0, abort_flag) && mbar_wait(bw_full, 0, abort_flag);
      if (ok) {
        tc_fence_after();
        if (lane == 0) {
          const uint32_t bw = smem_u32(smem + L::kBwOff);
          const uint32_t su = smem_u32(smem + L::kSuOff);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_bf16(d_acc, smem_desc_sw128(bw + kk * 32, 16), smem_desc_sw128(su + kk * 32, 16), kIdesc,
                      (n_steps > 0 || kk > 0) ? 1u : 0u);
        }
        __syncwarp();
      }
      if (lane == 0) umma_commit(accum_full);
      __syncwarp();
    }
    if (clustered) cluster_wait();
  } else {
    // ------------------------------------------------------------ A operand
    const int wg = (warp - 3) >> 2;
    const int q = warp & 3;                 // TMEM lane quarter this warp may access
    const int ln = q * 32 + lane;           // TMEM lane = row of the A operand
    const bool is_adapter = ln < r;         // lanes < r: adapter row ln; else weight row c0 + ln - r
    const int i = ln - r;
    const int w_row = c0 + i;
    const uint32_t lane_addr = static_cast<uint32_t>(q * 32) << 16;
    bool ok = true;
    float level[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) level[j] = args.level[j];
    const int kblocks = args.k_steps;
    auto load_scale = [&](int ks) -> float {
      if (is_adapter || w_row >= args.n_cols) return 0.f;
      const int64_t blk = static_cast<int64_t>(w_row) * kblocks + ks;
      return block_scale(args.q8, args.s2, blk);
    };
    // this warpgroup's steps are t = wg, wg + kDecWG, ...: scales two of them ahead
    float c1_a = (wg < n_steps) ? load_scale(step_begin + wg) : 0.f;
    float c1_b = (wg + kDecWG < n_steps) ? load_scale(step_begin + wg + kDecWG) : 0.f;
    for (int t = wg; t < n_steps; t += kDecWG) {
      const int s = t % NS;
      const uint32_t ph = (t / NS) & 1;
      const float c1 = c1_a;
      c1_a = c1_b;
      if (t + 2 * kDecWG < n_steps) c1_b = load_scale(step_begin + t + 2 * kDecWG);
      uint32_t w[32];
      const DeqTable tab = make_table(level, c1);
      if (!mbar_wait(&full_tma[s], ph, abort_flag)) { ok = false; break; }
      tc_fence_after();
      if (is_adapter) {
        // adapter row ln: 128 B, 128-byte swizzle (16-byte chunk c at c ^ (ln & 7))
        const uint32_t a_base = smem_u32(smem + s * L::kStageBytes + a_off) + ln * 128;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint4 e = ld_shared_v4(a_base + ((static_cast<uint32_t>(c) ^ (ln & 7)) << 4));
          w[4 * c] = e.x;
          w[4 * c + 1] = e.y;
          w[4 * c + 2] = e.z;
          w[4 * c + 3] = e.w;
        }
      } else {
        // packed row i: 32 B, 32-byte swizzle (16-byte chunk h at h ^ ((i >> 2) & 1))
        const uint32_t p_base = smem_u32(smem + s * L::kStageBytes + L::kPOff);
        const uint32_t sw = (i >> 2) & 1;
        const uint4 p0 = ld_shared_v4(p_base + i * 32 + ((0u ^ sw) << 4));
        const uint4 p1 = ld_shared_v4(p_base + i * 32 + ((1u ^ sw) << 4));
        const uint32_t words[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint4 e = expand8(tab, words[c]);
          w[4 * c] = e.x;
          w[4 * c + 1] = e.y;
          w[4 * c + 2] = e.z;
          w[4 * c + 3] = e.w;
        }
      }
      tmem_st_32x32b_x32(tmem_d + lane_addr + static_cast<uint32_t>(s * kDecACols), w);
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&full_w[s]);
    }
    griddep_launch_dependents();
    const uint32_t recv_bar = smem_u32(recv_full);
    if (warp == 8 || warp == 9) {
      // ---------------------------------------------------------- U_z -> adapter operand
      // lanes 0..63 = adapter index j
      const int j = ln;
      if (ok) ok = mbar_wait(mma_done, 0, abort_flag);
      float u[MP], u1[MP];
#pragma unroll
      for (int m = 0; m < MP; ++m) u[m] = 0.f;
      if (ok) {
        tc_fence_after();
        tmem_read_cols<MP>(d_acc + lane_addr, u);
        tmem_read_cols<MP>(d_acc + lane_addr + MP, u1);
        const bool live = (n_steps > 0) && (j < r);
        const bool has1 = n_steps > 1;   // accumulator 1 holds nothing otherwise
        uint8_t* su = smem + L::kSuOff;
#pragma unroll
        for (int m = 0; m < MP; ++m) {
          u[m] = live ? u[m] + (has1 ? u1[m] : 0.f) : 0.f;
          // s U_z as a K-major operand: row m (token), element j, 128-byte swizzle
          const __nv_bfloat16 h = __float2bfloat16_rn(__fmul_rn(args.s, u[m]));
          *reinterpret_cast<__nv_bfloat16*>(su + m * 128 + (((j >> 3) ^ (m & 7)) << 4) + (j & 7) * 2) = h;
        }
        fence_proxy_async_smem();
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(su_full);
      if (clustered) cluster_wait();   // every peer is running
      if (ok && want_u && j < r) {
        // partial U -> the rank that stores columns [o * slice_u, (o+1) * slice_u) of U
        const int o = j / su_n;
        const int jl = j - o * su_n;
        const uint32_t base = smem_u32(smem + L::kRecvUOff);
#pragma unroll
        for (int m = 0; m < MP; ++m) {
          if (m >= mv) break;
          const int uidx = (rank * MP + m) * su_n + jl;
          if (!QLORA_CHECK(uidx < MP * 72 && o < S, kDbgCluster, uidx)) continue;
          const uint32_t off = base + static_cast<uint32_t>(uidx * 4);
          if (clustered) st_async_f32(map_to_rank(off, o), u[m], map_to_rank(recv_bar, o));
          else *reinterpret_cast<float*>(smem + L::kRecvUOff + (off - base)) = u[m];
        }
      }
    } else if (warp <= 6) {
      // ---------------------------------------------------------- partial tile -> owners
      if (ok) ok = mbar_wait(accum_full, 0, abort_flag);
      float v[MP], v1[MP];
      if (ok) {
        tc_fence_after();
        tmem_read_cols<MP>(d_acc + lane_addr, v);
        tmem_read_cols<MP>(d_acc + lane_addr + MP, v1);
        if (n_steps > 1) {   // accumulator 1 holds nothing otherwise
#pragma unroll
          for (int m = 0; m < MP; ++m) v[m] += v1[m];
        }
      }
      __syncwarp();
      if (clustered) cluster_wait();   // every peer is running
      if (ok && ln >= r && i < T) {
        const int o = i / sl;
        const int il = i - o * sl;
        const uint32_t base = smem_u32(smem + L::kRecvOff);
#pragma unroll
        for (int m = 0; m < MP; ++m) {
          if (m >= mv) break;
          const int yidx = (rank * MP + m) * sl + il;
          if (!QLORA_CHECK(yidx < MP * 192 && o < S, kDbgCluster, yidx)) continue;
          const uint32_t off = base + static_cast<uint32_t>(yidx * 4);
          if (clustered) st_async_f32(map_to_rank(off, o), v[m], map_to_rank(recv_bar, o));
          else *reinterpret_cast<float*>(smem + L::kRecvOff + (off - base)) = v[m];
        }
      }
    } else {
      if (clustered) cluster_wait();
    }

    // ------------------------------------------------------------ owned rows
    if (clustered) {
      if (!mbar_wait(recv_full, 0, abort_flag)) ok = false;
    } else {
      named_bar_sync(1, 128 * kDecWG);   // warps 3..: the local partials are written
    }
    if (!*abort_flag) {
      const int tid = static_cast<int>(threadIdx.x) - 96;
      {
        // Y rows [rank * slice_rows, ...) of the tile: sum the S partials in rank order
        const int pairs = own_rows / 2;   // even: T and slice_rows are multiples of 8
        const float* recv = reinterpret_cast<const float*>(smem + L::kRecvOff);
        for (int idx = tid; idx < mv * pairs; idx += 128 * kDecWG) {
          const int m = idx / pairs;
          const int il = 2 * (idx - m * pairs);
          float a0 = 0.f, a1 = 0.f;
          for (int pp = 0; pp < S; ++pp) {
            const float2 x = *reinterpret_cast<const float2*>(recv + (pp * MP + m) * sl + il);
            a0 += x.x;
            a1 += x.y;
          }
          const int col = c0 + rank * sl + il;
          if (col < args.n_cols) {
            __nv_bfloat162 h = __floats2bfloat162_rn(a0, a1);
            *reinterpret_cast<__nv_bfloat162*>(args.y + static_cast<int64_t>(m) * args.ld_y + col) = h;
          }
        }
      }
      if (want_u) {
        const float* recv = reinterpret_cast<const float*>(smem + L::kRecvUOff);
        for (int idx = tid; idx < mv * own_cols; idx += 128 * kDecWG) {
          const int m = idx / own_cols;
          const int jl = idx - m * own_cols;
          float a = 0.f;
          for (int pp = 0; pp < S; ++pp) a += recv[(pp * MP + m) * su_n + jl];
          reinterpret_cast<__nv_bfloat16*>(args.u_save)[static_cast<int64_t>(m) * r + rank * su_n + jl] =
              __float2bfloat16_rn(a);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_d, L::kTmemCols);
  }
}

}  // namespace qlora
