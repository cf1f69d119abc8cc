// Skinny adapter products of the QLoRA layer on tcgen05, split-K across a
// thread-block cluster and reduced through distributed shared memory.
//
//   U    = X A^T      (M x r)   -> U (bf16) and s*U (bf16)      reduction over K
//   V    = dY B       (M x r)   -> V (bf16) and s*V (bf16)      reduction over N
//   dA^T = X^T V      (K x r)   -> dA = s * (.)^T  (fp32 r x K) reduction over M
//   dB   = dY^T U     (N x r)   -> dB = s * (.)    (fp32 N x r) reduction over M
//
// ("逆伝播と勾配の流れ" of "QLoRAの理論と実装": dL/dB = (alpha/r) dL/dY (A X)^T and
// dL/dA = (alpha/r) B^T dL/dY X^T, written row-major.)
//
// Each output tile is 128 rows x 64 columns (one 64-wide slice of r).  The S
// CTAs of a cluster (S = 1, 2, 4 or 8, along grid z) take consecutive slices
// of the reduction; after the mainloop each CTA copies its TMEM accumulator to
// its own shared memory, the cluster synchronises, and CTA c sums rows
// [c*128/S, (c+1)*128/S) over the S CTAs in rank order (deterministic) and
// writes the final values.  No partial sums go to global memory and no
// reduction kernel follows.  Two independent problems (dA and dB) can share
// one launch: blockIdx.x below tiles0 selects problem 0.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include "ptx_sm100.cuh"

namespace qlora {

constexpr int kLoraBN = 64;
constexpr int kLoraThreads = 192;  // warp 0 TMA, warp 1 MMA, warps 2-5 epilogue

enum LoraOut : int {
  kLoraOutPlainScaled = 0,  // bf16 out0 = scale0 * sum (may be NULL), bf16 out1 = scale1 * sum; [rows][r]
  kLoraOutTransposed = 1,   // fp32 out0[col][row] = scale1 * sum  (dA from dA^T tiles)
  kLoraOutRowMajor = 2,     // fp32 out0[row][col] = scale1 * sum  (dB)
};

struct LoraProblem {
  int rows;        // rows of D (M, K or N)
  int k_steps;     // reduction steps of 64
  int per_split;   // reduction steps per cluster rank
  int tiles_m;     // 128-row tiles
  int tiles_n;     // 64-column slices of r
  int out_kind;
  void* out0;
  void* out1;
  int ld_t;        // kLoraOutTransposed: elements between out0 rows (= rows)
  float scale0;    // kLoraOutPlainScaled: factor of out0 (1 for U or V itself)
  float scale1;    // factor of out1 (PlainScaled) or of out0 (fp32 outputs)
};

struct LoraArgs {
  LoraProblem p[2];
  int tiles0;      // blocks of problem 0 along x (tiles_m * tiles_n)
  int r;
};

// Shared memory of one CTA: STAGES pipeline stages, each KB reduction steps
// of 64 (an A tile of 128 x 64 and a B tile of 64 x 64 bf16 per step).
template <int STAGES, int KB>
struct LoraSmem {
  static constexpr int kATile = 128 * 64 * 2;   // 16 KiB
  static constexpr int kBTile = 64 * 64 * 2;    // 8 KiB
  static constexpr int kAStage = KB * kATile;
  static constexpr int kBStage = KB * kBTile;
  static constexpr int kAOff = 0;
  static constexpr int kBOff = kAOff + STAGES * kAStage;
  static constexpr int kBarOff = kBOff + STAGES * kBStage;
  static constexpr int kMiscOff = kBarOff + (2 * STAGES + 1) * 8;
  static constexpr int kBytes = kMiscOff + 16;
  static constexpr int kDynBytes = kBytes + 1024;
  static constexpr int kRedBytes = 128 * 64 * 4;  // fp32 accumulator copy (reuses the A stages)
  static_assert(kRedBytes <= kBOff, "reduction buffer fits in the A stages");
  static_assert(kDynBytes <= 232448, "shared memory");
};

// A_MN: A operand MN-major (dA^T = X^T V, dB = dY^T U); else K-major (U, V).
// B_MN: B operand MN-major (V = dY B and the gradient products); else K-major (U).
// STAGES pipeline stages of KB reduction steps each.
template <bool A_MN, bool B_MN, int STAGES, int KB>
__global__ void __launch_bounds__(kLoraThreads, 1)
qlora_lora_kernel(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmB0,
                  const __grid_constant__ CUtensorMap tmA1, const __grid_constant__ CUtensorMap tmB1,
                  const LoraArgs args) {
  using L = LoraSmem<STAGES, KB>;
  constexpr uint32_t kIdesc = idesc_bf16_m128(kLoraBN, A_MN ? 1u : 0u, B_MN ? 1u : 0u);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  uint64_t* empty = full + STAGES;
  uint64_t* accum_full = empty + STAGES;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int which = static_cast<int>(blockIdx.x) < args.tiles0 ? 0 : 1;
  const LoraProblem P = which ? args.p[1] : args.p[0];
  const CUtensorMap* tA = which ? &tmA1 : &tmA0;
  const CUtensorMap* tB = which ? &tmB1 : &tmB0;
  const int tile = static_cast<int>(blockIdx.x) - (which ? args.tiles0 : 0);
  const int m0 = (tile / P.tiles_n) * 128;
  const int c0 = (tile % P.tiles_n) * kLoraBN;
  // The cluster is cx x 1 x S CTAs: the S ranks along z split the reduction;
  // cx = 2 only places two neighbouring tiles on one TPC (S = 1 then).  The
  // peer with split rank p has cluster rank x_local + cx * p.
  const int S = static_cast<int>(gridDim.z);
  const int rank = static_cast<int>(blockIdx.z);
  const uint32_t cx = cluster_dim_x();
  const uint32_t x_local = cluster_ctarank() % cx;
  const int ks0 = rank * P.per_split;
  const bool live = tile < P.tiles_m * P.tiles_n;   // false: a CTA that only pads the grid to the cluster
  const int n_steps = live ? max(0, min(P.k_steps, ks0 + P.per_split) - ks0) : 0;   // reduction steps of 64
  const int n_stages = (n_steps + KB - 1) / KB;                             // pipeline iterations

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(accum_full, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, kLoraBN);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_d = *tmem_slot;
  griddep_wait();   // no global access before the previous grid is complete
  // Release the next grid now: every CTA of this one is running, so a next
  // grid that waits for this one's completion (griddep_wait) before reading
  // its outputs cannot starve it of SMs, and it can start work that does not
  // depend on them on the SMs this grid leaves free.
  griddep_launch_dependents();

  bool ok = true;
  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(tA);
      tma_prefetch_desc(tB);
      for (int t = 0; t < n_stages; ++t) {
        const int s = t % STAGES;
        if (t >= STAGES && !mbar_wait(&empty[s], ((t / STAGES) - 1) & 1, abort_flag)) break;
        const int nb = min(KB, n_steps - t * KB);
        mbar_arrive_expect_tx(&full[s], static_cast<uint32_t>(nb * (L::kATile + L::kBTile)));
        for (int b = 0; b < nb; ++b) {
          const int ks = ks0 + t * KB + b;
          uint8_t* a_dst = smem + L::kAOff + s * L::kAStage + b * L::kATile;
          uint8_t* b_dst = smem + L::kBOff + s * L::kBStage + b * L::kBTile;
          if (A_MN) {
            tma_load_2d(a_dst, tA, &full[s], m0, ks * 64);
            tma_load_2d(a_dst + 64 * 128, tA, &full[s], m0 + 64, ks * 64);
          } else {
            tma_load_2d(a_dst, tA, &full[s], ks * 64, m0);
          }
          if (B_MN) tma_load_2d(b_dst, tB, &full[s], c0, ks * 64);
          else tma_load_2d(b_dst, tB, &full[s], ks * 64, c0);
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    for (int t = 0; t < n_stages; ++t) {
      const int s = t % STAGES;
      if (!mbar_wait(&full[s], (t / STAGES) & 1, abort_flag)) break;
      tc_fence_after();
      if (lane == 0) {
        const int nb = min(KB, n_steps - t * KB);
        for (int b = 0; b < nb; ++b) {
          const uint32_t a_base = smem_u32(smem + L::kAOff + s * L::kAStage + b * L::kATile);
          const uint32_t b_base = smem_u32(smem + L::kBOff + s * L::kBStage + b * L::kBTile);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t ad = A_MN ? smem_desc_sw128(a_base + kk * 2048, 64 * 128) : smem_desc_sw128(a_base + kk * 32, 16);
            const uint64_t bd = B_MN ? smem_desc_sw128(b_base + kk * 2048, 64 * 128) : smem_desc_sw128(b_base + kk * 32, 16);
            umma_bf16(tmem_d, ad, bd, kIdesc, (t > 0 || b > 0 || kk > 0) ? 1u : 0u);
          }
        }
        umma_commit(&empty[s]);
      }
      __syncwarp();
    }
    if (lane == 0) umma_commit(accum_full);
    __syncwarp();
  } else {
    // copy the accumulator (or zeros, for a rank with no steps) to shared memory
    ok = mbar_wait(accum_full, 0, abort_flag);
    float* red = reinterpret_cast<float*>(smem + L::kAOff);
    const int q = warp & 3;
    const int row = q * 32 + lane;
    if (ok) {
      tc_fence_after();
      uint32_t v[2][32];   // both 32-column chunks in flight before one wait
      tmem_ld_32x32b_x32(tmem_d + (static_cast<uint32_t>(q * 32) << 16), v[0]);
      tmem_ld_32x32b_x32(tmem_d + (static_cast<uint32_t>(q * 32) << 16) + 32, v[1]);
      tmem_ld_wait();
      // row-major [128][64] with the 16-byte chunk index rotated by the row
      // to spread the stores over the banks
      float4* dst = reinterpret_cast<float4*>(red + row * 64);
#pragma unroll
      for (int ch = 0; ch < 2; ++ch) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int c16 = ((ch * 8 + i) + row) & 15;
          float4 val = make_float4(__uint_as_float(v[ch][4 * i]), __uint_as_float(v[ch][4 * i + 1]),
                                   __uint_as_float(v[ch][4 * i + 2]), __uint_as_float(v[ch][4 * i + 3]));
          if (n_steps == 0) val = make_float4(0.f, 0.f, 0.f, 0.f);
          dst[c16] = val;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync_all();   // every rank's accumulator is in its shared memory

  if (warp >= 2 && live && !*abort_flag) {
    // rows [rank*128/S, (rank+1)*128/S) of the tile, summed over ranks 0..S-1
    const int t = threadIdx.x - 64;            // 0..127
    const int rows_here = 128 / S;
    const uint32_t red_base = smem_u32(smem + L::kAOff);
    const int items = rows_here * 16;          // 16 four-column chunks per row
    for (int it = t; it < items; it += 128) {
      int lr, c16;
      if (P.out_kind == kLoraOutTransposed) {  // lanes along rows: coalesced transposed stores
        lr = it % rows_here;
        c16 = it / rows_here;
      } else {
        lr = it / 16;
        c16 = it % 16;
      }
      const int trow = rank * rows_here + lr;
      const uint32_t off = static_cast<uint32_t>(trow * 64 + ((c16 + trow) & 15) * 4) * 4u;
      if (!QLORA_CHECK(off + 16u <= 128u * 64u * 4u, kDbgCluster, off)) continue;
      // issue all remote loads before the first add, then sum in rank order
      float4 v[8];
#pragma unroll
      for (int p = 0; p < 8; ++p)
        if (p < S) v[p] = ld_cluster_v4(map_to_rank(red_base + off, x_local + cx * static_cast<uint32_t>(p)));
      float4 acc = v[0];
#pragma unroll
      for (int p = 1; p < 8; ++p)
        if (p < S) { acc.x += v[p].x; acc.y += v[p].y; acc.z += v[p].z; acc.w += v[p].w; }
      const int grow = m0 + trow;
      const int gcol = c0 + c16 * 4;
      if (grow < P.rows && gcol < args.r) {
        const float s = P.scale1;
        if (P.out_kind == kLoraOutPlainScaled) {
          const int64_t o = static_cast<int64_t>(grow) * args.r + gcol;
          if (P.out0) {
            const float s0 = P.scale0;
            __nv_bfloat162 h0 = __floats2bfloat162_rn(s0 * acc.x, s0 * acc.y);
            __nv_bfloat162 h1 = __floats2bfloat162_rn(s0 * acc.z, s0 * acc.w);
            uint2 u;
            u.x = *reinterpret_cast<uint32_t*>(&h0);
            u.y = *reinterpret_cast<uint32_t*>(&h1);
            *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(P.out0) + o) = u;
          }
          if (P.out1) {
            __nv_bfloat162 h0 = __floats2bfloat162_rn(s * acc.x, s * acc.y);
            __nv_bfloat162 h1 = __floats2bfloat162_rn(s * acc.z, s * acc.w);
            uint2 u;
            u.x = *reinterpret_cast<uint32_t*>(&h0);
            u.y = *reinterpret_cast<uint32_t*>(&h1);
            *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(P.out1) + o) = u;
          }
        } else if (P.out_kind == kLoraOutRowMajor) {
          *reinterpret_cast<float4*>(static_cast<float*>(P.out0) + static_cast<int64_t>(grow) * args.r + gcol) =
              make_float4(s * acc.x, s * acc.y, s * acc.z, s * acc.w);
        } else {
          float* o = static_cast<float*>(P.out0);
          o[static_cast<int64_t>(gcol + 0) * P.ld_t + grow] = s * acc.x;
          o[static_cast<int64_t>(gcol + 1) * P.ld_t + grow] = s * acc.y;
          o[static_cast<int64_t>(gcol + 2) * P.ld_t + grow] = s * acc.z;
          o[static_cast<int64_t>(gcol + 3) * P.ld_t + grow] = s * acc.w;
        }
      }
    }
  }

  // No rank leaves while another still reads its shared memory.  Every remote
  // value was consumed before this point, so a relaxed arrive suffices and
  // the barrier does not wait for this CTA's global stores to complete.
  cluster_arrive_relaxed();
  cluster_wait();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_d, kLoraBN);
  }
}

}  // namespace qlora
