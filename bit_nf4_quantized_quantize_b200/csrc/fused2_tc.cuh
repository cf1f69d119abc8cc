// Fused NF4 dequant-GEMM on a CTA pair (tcgen05 cta_group::2), sm_100a.
//
//   forward  Y  = X dequant(W)^T + (s U) B^T    (B operand K-major: weight rows)
//   backward dX = dY dequant(W)  + (s V) A      (B operand MN-major: weight columns)
//
// A cluster of two CTAs computes a (256*MH) x 256 output tile.  Each MMA is
// M = 256 (both CTAs' 128-row A halves) x N = 256 (both CTAs' 128-row B
// halves) x K = 16, issued by the even CTA; each CTA's TMEM receives its own
// 128 rows.  With MH = 2 two such MMAs share every B tile, so each CTA expands
// only 128 x 64 NF4 weights per 2 x 128 x 256 x 64 MMA: a quarter of the
// dequant work per MMA of a 128-row single-CTA tile.
//
// Per CTA and stage: A (MH x 128 rows x 64, TMA, 128B swizzle), the packed
// codes of its 128 B rows (TMA), and its B half (dequantized in registers and
// written in the UMMA layout).  Synchronisation:
//   full_tma[s]   local: this CTA's TMA bytes landed (waited by its dequant warps)
//   full_w[s]     in the even CTA, count 2*NDW: both CTAs' dequant warps
//                 arrive (remote arrive for the odd CTA) after their A and B
//                 halves are in place; the MMA issuer waits on it alone
//   empty[s]      local, completed in both CTAs by one multicast commit
//   accum_full    local, completed in both CTAs by one multicast commit
// Every wait is bounded; both CTAs always reach the final cluster barrier.
// No TMA load uses cluster multicast.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include "ptx_sm100.cuh"
#include "gemm_tc.cuh"

namespace qlora {

// ---------------------------------------------------------------- PTX (pair)
__device__ __forceinline__ void tmem_alloc_pair(uint32_t* smem_result, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;"
               ::"r"(smem_u32(smem_result)), "r"(ncols) : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void umma_bf16_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                               uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}"
      ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive once on `bar` (same offset) in every CTA of cta_mask when the pair's
// MMAs issued so far have completed.
__device__ __forceinline__ void umma_commit_pair_mc(uint64_t* bar, uint16_t cta_mask) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;"
      ::"r"(smem_u32(bar)), "h"(cta_mask) : "memory");
}
// Arrive on the mbarrier at the same offset in CTA `rank` of the cluster.
// Default (release, CTA-scope) semantics: the operand tile it announces was
// written to this CTA's shared memory and published to the async proxy by
// fence.proxy.async beforehand, which is what the pair's MMA reads through.
// (A release at cluster scope added ~0.6 us per k-step on this path.)
__device__ __forceinline__ void mbar_arrive_remote(uint64_t* bar, uint32_t rank) {
  asm volatile(
      "{\n\t.reg .b32 ra;\n\t"
      "mapa.shared::cluster.u32 ra, %0, %1;\n\t"
      "mbarrier.arrive.shared::cluster.b64 _, [ra];\n\t}"
      ::"r"(smem_u32(bar)), "r"(rank) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait_cluster(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
  return ok != 0;
}
// Bounded wait with cluster-scope acquire (for barriers that the peer CTA arrives on).
__device__ __forceinline__ bool mbar_wait_cluster(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
  if (mbar_try_wait_cluster(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait_cluster(bar, parity)) return true;
    if ((i & 255u) == 0) {
      if (*abort_flag) return false;
      if (globaltimer_ns() - t0 > kWaitLimitNs) {
        *abort_flag = 1;
        atomicExch(&g_device_error, kDevErrTimeout);
        return false;
      }
      if (i > 4096) __nanosleep(128);
    }
  }
}
__device__ __forceinline__ uint32_t cta_rank_in_cluster() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_barrier() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Instruction descriptor for the pair: M = 256 (>>4 = 16 at bits [24,29)).
__host__ __device__ constexpr uint32_t idesc_bf16_m256(uint32_t n, uint32_t b_mn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (b_mn << 16) | ((n >> 3) << 17) | ((256u >> 4) << 24);
}

// Two warpgroups of dequant / epilogue warps per CTA.  Warpgroup g expands
// the B half of steps t with t % 2 == g (one B row, or one 64-column block of
// a reduction row, per thread), so two stages are in flight at once.
constexpr int kPairNDW = 8;
constexpr int kPairThreads = 64 + 32 * kPairNDW;
constexpr int kPairBHalf = 128;        // B rows (N) held by each CTA
constexpr int kPairN = 2 * kPairBHalf; // N of each MMA

template <int MH>
struct PairSmem {
  static constexpr int kATile = MH * kAHalfBytes;              // MH x 16 KiB
  static constexpr int kBTile = kPairBHalf * kBK * 2;          // 16 KiB
  static constexpr int kPTile = kPairBHalf * kBK / 2;          // 4 KiB
  static constexpr int kStages = MH == 2 ? 4 : 6;
  static constexpr int kAOff = 0;
  static constexpr int kBOff = kAOff + kStages * kATile;
  static constexpr int kPOff = kBOff + kStages * kBTile;
  static constexpr int kBarOff = kPOff + kStages * kPTile;
  static constexpr int kMiscOff = kBarOff + (3 * kStages + 1) * 8;
  static constexpr int kBytes = kMiscOff + 16;
  static constexpr int kDynBytes = kBytes + 1024;
  static_assert(kDynBytes <= 232448, "shared memory");
};

template <int BSRC, int MH>
__global__ void __launch_bounds__(kPairThreads, 1)
qlora_fused_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmP,
                        const __grid_constant__ CUtensorMap tmA2, const __grid_constant__ CUtensorMap tmB2,
                        const __grid_constant__ CUtensorMap tmOut, const GemmArgs args) {
  static_assert(BSRC == kBDeqK || BSRC == kBDeqMN, "dequant sources only");
  using L = PairSmem<MH>;
  constexpr int NST = L::kStages;
  constexpr bool kBMN = (BSRC == kBDeqMN);
  constexpr uint32_t kIdesc = idesc_bf16_m256(kPairN, kBMN ? 1u : 0u);
  constexpr uint32_t kTmemCols = MH * kPairN;   // 256 or 512

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full_tma = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  uint64_t* full_w = full_tma + NST;
  uint64_t* empty = full_w + NST;
  uint64_t* accum_full = empty + NST;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cta_rank_in_cluster();        // 0: issues the MMAs
  const int pair = blockIdx.x >> 1;
  const int tiles_n = (args.n_cols + kPairN - 1) / kPairN;
  const int m0 = (pair / tiles_n) * (256 * MH);       // first row of the pair's tile
  const int c0 = (pair % tiles_n) * kPairN;           // first column of the pair's tile
  const int cb = c0 + kPairBHalf * static_cast<int>(rank);  // first B row held here
  const int n_main = args.k_steps;
  const int n_lora = args.n_lora;
  const int total = n_lora + n_main;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(&full_tma[s], 1);
      mbar_init(&full_w[s], 2 * (kPairNDW / 2));   // one warpgroup of each CTA per step
      mbar_init(&empty[s], 1);
    }
    mbar_init(accum_full, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc_pair(tmem_slot, kTmemCols);
  tc_fence_before();
  __syncthreads();
  cluster_barrier();     // barriers of both CTAs initialised before any remote arrive
  tc_fence_after();
  const uint32_t tmem_d = *tmem_slot;
  // The previous grid on the stream is the adapter kernel that writes s U
  // (or s V); it releases this grid as soon as it is running.  The main steps
  // read only X (or dY) and the packed weight, which are complete before that
  // kernel started, so the wait for its completion comes just before the
  // first adapter slice (producer) and before the first store (epilogue).

  if (warp == 0) {
    // ------------------------------------------------------------ producer (each CTA its own halves)
    if (lane == 0) {
      tma_prefetch_desc(&tmA);
      tma_prefetch_desc(&tmP);
      if (n_lora > 0) { tma_prefetch_desc(&tmA2); tma_prefetch_desc(&tmB2); }
      for (int t = 0; t < total; ++t) {
        const int s = t % NST;
        if (t >= NST && !mbar_wait(&empty[s], ((t / NST) - 1) & 1, abort_flag)) break;
        uint8_t* a_dst = smem + L::kAOff + s * L::kATile;
        uint8_t* b_dst = smem + L::kBOff + s * L::kBTile;
        if (t >= n_main) {
          const int j = t - n_main;   // adapter slice: the previous grid's output
          if (j == 0) griddep_wait();
          mbar_arrive_expect_tx(&full_tma[s], L::kATile + L::kBTile);
#pragma unroll
          for (int h = 0; h < MH; ++h)
            tma_load_2d(a_dst + h * kAHalfBytes, &tmA2, &full_tma[s], j * kBK, m0 + 256 * h + 128 * rank);
          if (!kBMN) {
            tma_load_2d(b_dst, &tmB2, &full_tma[s], j * kBK, cb);
          } else {
            tma_load_2d(b_dst, &tmB2, &full_tma[s], cb, j * kBK);
            tma_load_2d(b_dst + kBK * 128, &tmB2, &full_tma[s], cb + 64, j * kBK);
          }
        } else {
          const int ks = t;
          mbar_arrive_expect_tx(&full_tma[s], L::kATile + L::kPTile);
#pragma unroll
          for (int h = 0; h < MH; ++h)
            tma_load_2d(a_dst + h * kAHalfBytes, &tmA, &full_tma[s], ks * kBK, m0 + 256 * h + 128 * rank);
          uint8_t* p_dst = smem + L::kPOff + s * L::kPTile;
          if (!kBMN) tma_load_2d(p_dst, &tmP, &full_tma[s], ks * (kBK / 2), cb, 1);   // 128 rows x 32 B
          else tma_load_2d(p_dst, &tmP, &full_tma[s], cb / 2, ks * kBK, 1);        // 64 rows x 64 B
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (even CTA only)
    if (rank == 0) {
      for (int t = 0; t < total; ++t) {
        const int s = t % NST;
        if (!mbar_wait_cluster(&full_w[s], (t / NST) & 1, abort_flag)) break;
        tc_fence_after();
        if (lane == 0) {
          const uint32_t a_base = smem_u32(smem + L::kAOff + s * L::kATile);
          const uint32_t b_base = smem_u32(smem + L::kBOff + s * L::kBTile);
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk) {
            const uint64_t bd = kBMN ? smem_desc_sw128(b_base + kk * 2048, kBK * 128)
                                     : smem_desc_sw128(b_base + kk * 32, 16);
#pragma unroll
            for (int h = 0; h < MH; ++h)
              umma_bf16_pair(tmem_d + h * kPairN, smem_desc_sw128(a_base + h * kAHalfBytes + kk * 32, 16), bd,
                             kIdesc, (t > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit_pair_mc(&empty[s], 0x3);
        }
        __syncwarp();
      }
      if (lane == 0) umma_commit_pair_mc(accum_full, 0x3);
      __syncwarp();
    }
  } else {
    // ------------------------------------------------------------ dequant, then epilogue
    const int item = (threadIdx.x - 64) & 127;   // 0..127
    const int wg = (threadIdx.x - 64) >> 7;      // warpgroup: steps t with t % 2 == wg
    bool ok = true;
    float level[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) level[i] = args.level[i];
    // item -> (weight row, 64-block) whose 64 values this thread expands per step
    auto load_scale = [&](int ks) -> float {
      int wr, kb;
      if (!kBMN) { wr = cb + item; kb = ks; }
      else { wr = ks * 64 + (item & 63); kb = cb / 64 + (item >> 6); }
      if (wr >= args.w_rows || kb >= args.w_kblocks) return 0.f;
      const int64_t blk = static_cast<int64_t>(wr) * args.w_kblocks + kb;
      return block_scale(args.q8, args.s2, blk);
    };
    // this warpgroup's main steps are ks = t = wg, wg+2, ...; scales prefetched two ahead
    float c1_a = (wg < n_main) ? load_scale(wg) : 0.f;
    float c1_b = (wg + 2 < n_main) ? load_scale(wg + 2) : 0.f;
    for (int t = wg; t < total; t += 2) {
      const int s = t % NST;
      const uint32_t ph = (t / NST) & 1;
      if (!mbar_wait(&full_tma[s], ph, abort_flag)) { ok = false; break; }
      if (t < n_main) {
        const int ks = t;
        const float c1 = c1_a;
        c1_a = c1_b;
        if (ks + 4 < n_main) c1_b = load_scale(ks + 4);
        const DeqTable tab = make_table(level, c1);
        const uint32_t p_base = smem_u32(smem + L::kPOff + s * L::kPTile);
        const uint32_t b_base = smem_u32(smem + L::kBOff + s * L::kBTile);
        if (!kBMN) {
          // packed row `item`: 32 B, 32-byte swizzle (16 B chunk h at h ^ ((row >> 2) & 1))
          const int r = item;
          const uint32_t sw = (r >> 2) & 1;
          const uint4 p0 = ld_shared_v4(p_base + r * 32 + ((0u ^ sw) << 4));
          const uint4 p1 = ld_shared_v4(p_base + r * 32 + ((1u ^ sw) << 4));
          const uint32_t words[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
          const uint32_t row_addr = b_base + r * 128;
#pragma unroll
          for (int c = 0; c < 8; ++c)
            st_shared_v4(row_addr + ((static_cast<uint32_t>(c) ^ (r & 7)) << 4), expand8(tab, words[c]));
        } else {
          // packed row nr: 64 B (128 columns), 64-byte swizzle (chunk c at c ^ ((row >> 1) & 3));
          // block jb is chunks 2jb and 2jb+1
          const int nr = item & 63;
          const int jb = item >> 6;
          const uint32_t sw = (nr >> 1) & 3;
          const uint32_t prow = p_base + nr * 64;
          const uint4 p0 = ld_shared_v4(prow + ((static_cast<uint32_t>(2 * jb) ^ sw) << 4));
          const uint4 p1 = ld_shared_v4(prow + ((static_cast<uint32_t>(2 * jb + 1) ^ sw) << 4));
          const uint32_t words[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
          const uint32_t row_addr = b_base + jb * (kBK * 128) + nr * 128;
#pragma unroll
          for (int c = 0; c < 8; ++c)
            st_shared_v4(row_addr + ((static_cast<uint32_t>(c) ^ (nr & 7)) << 4), expand8(tab, words[c]));
        }
        fence_proxy_async_smem();
      }
      __syncwarp();
      if (lane == 0) {
        if (rank == 0) mbar_arrive(&full_w[s]);
        else mbar_arrive_remote(&full_w[s], 0);
      }
    }
    // ------------------------------------------------------------ epilogue (own 128 rows per half)
    if (ok) ok = mbar_wait_cluster(accum_full, 0, abort_flag);
    griddep_wait();   // the previous grid is complete before this grid writes anything
    griddep_launch_dependents();
    if (ok) {
      tc_fence_after();
      const int q = warp & 3;
      // This warp owns TMEM lanes 32q..32q+31 (its 32 output rows) and the
      // 32-column chunks ch = wg, wg+2, wg+4, wg+6 of each half.  Each 32 x 32
      // block is converted to bf16 into a private 2 KiB staging tile in the
      // (now idle) stage memory and written by one TMA bulk tensor store,
      // which also clips rows >= M and columns >= N.
      uint8_t* stage = smem + (warp - 2) * (MH * 4 * 2048);
      // The warp's 4 * MH chunks of 32 columns, c = 4 h + j at half h, column chunk wg + 2 j.
      // Two register buffers: the load of chunk c + 1 is in flight while chunk c is
      // converted and staged; the wait that follows hands its registers over.
      constexpr int kChunks = 4 * MH;
      const uint32_t tlane = tmem_d + (static_cast<uint32_t>(q * 32) << 16);
      auto chunk_col = [&](int c) -> uint32_t {
        return static_cast<uint32_t>((c >> 2) * kPairN + (wg + 2 * (c & 3)) * 32);
      };
      auto stage_chunk = [&](int c, const uint32_t (&v)[32]) {
        // row `lane` of the block: 64 bytes, 16-byte chunk i at (i ^ ((lane >> 1) & 3))
        const uint32_t blk = smem_u32(stage + c * 2048);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          uint4 o;
          __nv_bfloat162 h0 = __floats2bfloat162_rn(__uint_as_float(v[8 * i + 0]), __uint_as_float(v[8 * i + 1]));
          __nv_bfloat162 h1 = __floats2bfloat162_rn(__uint_as_float(v[8 * i + 2]), __uint_as_float(v[8 * i + 3]));
          __nv_bfloat162 h2 = __floats2bfloat162_rn(__uint_as_float(v[8 * i + 4]), __uint_as_float(v[8 * i + 5]));
          __nv_bfloat162 h3 = __floats2bfloat162_rn(__uint_as_float(v[8 * i + 6]), __uint_as_float(v[8 * i + 7]));
          o.x = *reinterpret_cast<uint32_t*>(&h0);
          o.y = *reinterpret_cast<uint32_t*>(&h1);
          o.z = *reinterpret_cast<uint32_t*>(&h2);
          o.w = *reinterpret_cast<uint32_t*>(&h3);
          st_shared_v4(blk + lane * 64 + ((static_cast<uint32_t>(i) ^ ((lane >> 1) & 3)) << 4), o);
        }
        if ((c & 3) == 3) {
          // the half's four blocks are staged: store them
          const int h = c >> 2;
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            const int row0 = m0 + 256 * h + 128 * static_cast<int>(rank) + q * 32;
#pragma unroll
            for (int j = 0; j < 4; ++j)
              tma_store_2d(&tmOut, stage + (h * 4 + j) * 2048, c0 + (wg + 2 * j) * 32, row0);
          }
        }
      };
      uint32_t va[32], vb[32];
      tmem_ld_32x32b_x32(tlane + chunk_col(0), va);
      tmem_ld_wait_regs(va);
#pragma unroll
      for (int c = 0; c < kChunks; c += 2) {
        if (c + 1 < kChunks) tmem_ld_32x32b_x32(tlane + chunk_col(c + 1), vb);
        stage_chunk(c, va);
        if (c + 1 < kChunks) {
          tmem_ld_wait_regs(vb);
          if (c + 2 < kChunks) tmem_ld_32x32b_x32(tlane + chunk_col(c + 2), va);
          stage_chunk(c + 1, vb);
          if (c + 2 < kChunks) tmem_ld_wait_regs(va);
        }
      }
      if (lane == 0) {
        tma_store_commit();
        tma_store_wait_read();
      }
      __syncwarp();
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_barrier();     // the peer's MMAs and reads of this CTA's shared memory are over
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_d, kTmemCols);
  }
}

}  // namespace qlora
