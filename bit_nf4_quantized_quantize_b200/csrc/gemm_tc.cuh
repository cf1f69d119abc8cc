// tcgen05 (5th-generation tensor core) GEMM for the QLoRA linear layer, sm_100a.
//
// D[128 x BN] tile (+)= A[128 x K] * B[BN x K]^T with bf16 operands staged in
// 128-byte-swizzled shared memory and an fp32 accumulator in TMEM.  One
// template covers every product of the layer:
//
//   forward   Y  = X dequant(W)^T + (s U) B^T      B operand = NF4 weight, K-major
//   backward  dX = dY dequant(W)  + (s V) A        B operand = NF4 weight, MN-major
//   LoRA      U  = X A^T, V = dY B                 split-K, fp32 partials
//   grads     dA^T = X^T V, dB = dY^T U            split-M, fp32 partials
//
// For the two weight products the B tile is never read from HBM in bf16: the
// producer warp streams the packed 4-bit codes with TMA, the dequant warps
// expand them in registers (one 16-entry bf16 table per 64-block, looked up
// with byte permutes) and write the bf16 tile straight into the swizzled
// layout UMMA reads.  The adapter term runs as extra K=64 slices of the same
// accumulator (U or V pre-scaled by s on the A side, B or A on the B side), so
// the LoRA up-projection costs no separate pass over Y.
//
// Warp roles (64 + 32*NDW threads):
//   warp 0        TMA producer (one elected lane)
//   warp 1        TMEM allocator and MMA issuer (one elected lane)
//   warps 2..     dequant (weight products), then epilogue (TMEM -> registers
//                 -> global).  Warp w reads TMEM lanes 32*(w%4)...
// Pipelines: full_tma[s] (TMA bytes landed), full_w[s] (dequant wrote the B
// tile), empty[s] (the MMAs that read stage s completed), accum_full.  Every
// wait is bounded (ptx_sm100.cuh): on expiry the CTA latches the device error
// flag, every role leaves its loop, TMEM is freed and the CTA exits.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include "ptx_sm100.cuh"

namespace qlora {

enum BSource : int {
  kBTmaK = 0,    // B tile loaded by TMA, K-major
  kBTmaMN = 1,   // B tile loaded by TMA, MN-major
  kBDeqK = 2,    // B = dequant(W) rows (weight row n = B row), K-major   (forward)
  kBDeqMN = 3,   // B = dequant(W)^T (weight row = reduction index), MN-major (dX)
};
// kOutDropoutAdd: bf16 out(m, n) = bf16(fp32(out(m, n)) + drop_scale * D(m, n)) where bit
// e = m * ld_out + n of the LoRA-dropout keep mask drop_bits (bit e & 31 of word e >> 5) is
// set, out unchanged where it is clear (the adapter's share of dX under dropout).  In this mode the tensor map
// tmA2 covers the output (bf16, box 64 x 128): the output tile comes in by TMA.
enum OutMode : int { kOutBf16 = 0, kOutF32Partial = 1, kOutDropoutAdd = 2 };

constexpr int kBK = 64;                 // reduction elements per stage (128 B of bf16)
constexpr int kBM = 128;                // MMA M
constexpr int kAHalfBytes = kBM * kBK * 2;  // one 128-row A half (16 KiB)

struct GemmArgs {
  int m_rows;             // rows of D (MMA M side) in total
  int n_cols;             // columns of D in total
  int k_steps;            // main reduction steps (of 64) in total
  int steps_per_split;    // main steps per CTA along blockIdx.z
  int n_lora;             // adapter slices (of 64) issued before the main steps
  // NF4 weight (dequant sources only)
  const uint8_t* q8;
  const float* s2;
  int w_rows;             // N of the weight
  int w_kblocks;          // K/64 of the weight
  float level[16];        // NF4 levels (fp32)
  // output
  void* out;
  int64_t ld_out;         // elements between consecutive D rows
  int64_t split_stride;   // elements between splits (partial mode)
  // kOutDropoutAdd: scale and keep bits
  float drop_scale;
  const uint32_t* drop_bits;
};

template <int BN, int NSTAGE, int BSRC, int NDW, int MH, int OUT = kOutBf16>
struct GemmSmem {
  static constexpr bool kDeq = (BSRC == kBDeqK || BSRC == kBDeqMN);
  // kOutDropoutAdd: the output tile (bf16, MH x 128 rows x BN, 64-column boxes of 128-byte
  // swizzled rows) is loaded by TMA while the MMAs run, and read back by the epilogue
  static constexpr int kOutTileBytes = OUT == kOutDropoutAdd ? MH * kBM * BN * 2 : 0;
  static constexpr int kATileBytes = MH * kAHalfBytes;
  static constexpr int kBTileBytes = BN * kBK * 2;
  static constexpr int kPTileBytes = kDeq ? BN * kBK / 2 : 0;
  static constexpr int kAOff = 0;
  static constexpr int kBOff = kAOff + NSTAGE * kATileBytes;
  static_assert(kBOff + NSTAGE * (kBTileBytes + kPTileBytes) + kOutTileBytes + 1024 + 8 * (3 * NSTAGE + 2) + 16 <=
                    232448,
                "shared memory");
  static constexpr int kPOff = kBOff + NSTAGE * kBTileBytes;
  static constexpr int kOutOff = kPOff + NSTAGE * kPTileBytes;   // 1024-byte aligned
  static constexpr int kBarOff = kOutOff + kOutTileBytes;
  static constexpr int kNumBars = 3 * NSTAGE + 2;   // full_tma, full_w, empty per stage; accum_full; out_full
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kBytes = kMiscOff + 16;
  static constexpr int kDynBytes = kBytes + 1024;  // slack to align the base to 1024 B
};

// ---------------------------------------------------------------------------
// Register-level NF4 expansion.  For one 64-block with combined scale c1, the
// 16 values bf16(fp32(level[i] * c1)) are split into low bytes (lo[0..3]) and
// high bytes (hi[0..3]), 4 per register; a byte permute then looks up 4 codes
// at once.
struct DeqTable {
  uint32_t lo[4], hi[4];
};

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

__device__ __forceinline__ DeqTable make_table(const float (&level)[16], float c1) {
  uint32_t pr[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    __nv_bfloat162 h = __floats2bfloat162_rn(__fmul_rn(level[2 * j], c1), __fmul_rn(level[2 * j + 1], c1));
    pr[j] = *reinterpret_cast<uint32_t*>(&h);
  }
  DeqTable t;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    t.lo[q] = prmt(pr[2 * q], pr[2 * q + 1], 0x6420u);
    t.hi[q] = prmt(pr[2 * q], pr[2 * q + 1], 0x7531u);
  }
  return t;
}

// 8 codes (one packed word, element j in bits 4j..4j+3) -> 4 bf16 pairs.
__device__ __forceinline__ uint4 expand8(const DeqTable& t, uint32_t p) {
  const uint32_t s = p & 0x77777777u;                 // low three bits of each code
  const uint32_t x = (p >> 1) & 0x44444444u;          // bit 3 of each code, moved to bit 2
  uint4 o;
  {
    const uint32_t sel = x | 0x3210u;
    const uint32_t lo = prmt(prmt(t.lo[0], t.lo[1], s), prmt(t.lo[2], t.lo[3], s), sel);
    const uint32_t hi = prmt(prmt(t.hi[0], t.hi[1], s), prmt(t.hi[2], t.hi[3], s), sel);
    o.x = prmt(lo, hi, 0x5140u);
    o.y = prmt(lo, hi, 0x7362u);
  }
  {
    const uint32_t s1 = s >> 16;
    const uint32_t sel = (x >> 16) | 0x3210u;
    const uint32_t lo = prmt(prmt(t.lo[0], t.lo[1], s1), prmt(t.lo[2], t.lo[3], s1), sel);
    const uint32_t hi = prmt(prmt(t.hi[0], t.hi[1], s1), prmt(t.hi[2], t.hi[3], s1), sel);
    o.z = prmt(lo, hi, 0x5140u);
    o.w = prmt(lo, hi, 0x7362u);
  }
  return o;
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint4 v) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}
__device__ __forceinline__ uint4 ld_shared_v4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}

// ---------------------------------------------------------------------------
// MH = number of 128-row halves of the M tile.  With MH = 2 the tile is
// 256 x BN: two accumulators (TMEM columns [0, BN) and [BN, 2 BN)) share each
// B tile, which halves the dequant work per MMA.
template <int BN, int NSTAGE, bool A_MN, int BSRC, int OUT, int NDW, int MH>
__global__ void __launch_bounds__(64 + 32 * NDW, 1)
qlora_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                  const __grid_constant__ CUtensorMap tmA2, const __grid_constant__ CUtensorMap tmB2,
                  const GemmArgs args) {
  using L = GemmSmem<BN, NSTAGE, BSRC, NDW, MH, OUT>;
  constexpr bool kDeq = L::kDeq;
  constexpr int kATileBytes = L::kATileBytes;
  static_assert(MH == 1 || MH == 2, "MH");
  static_assert(MH == 1 || !A_MN, "MN-major A uses one half");
  constexpr bool kBMN = (BSRC == kBTmaMN || BSRC == kBDeqMN);
  static_assert(BN % 64 == 0 && BN >= 64 && BN <= 256, "BN");
  static_assert(!kDeq || NDW * 32 == BN, "one dequant item per thread");
  static_assert(NDW % 4 == 0, "epilogue warps must cover the four TMEM lane quarters");
  constexpr uint32_t kIdesc = idesc_bf16_m128(BN, A_MN ? 1u : 0u, kBMN ? 1u : 0u);
  constexpr uint32_t kTmemCols = (MH * BN) < 32 ? 32 : MH * BN;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full_tma = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  uint64_t* full_w = full_tma + NSTAGE;
  uint64_t* empty = full_w + NSTAGE;
  uint64_t* accum_full = empty + NSTAGE;
  uint64_t* out_full = accum_full + 1;   // kOutDropoutAdd: the output tile landed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * (kBM * MH);
  const int c0 = blockIdx.y * BN;
  const int split = blockIdx.z;
  const int step_begin = split * args.steps_per_split;
  const int step_end = min(args.k_steps, step_begin + args.steps_per_split);
  const int n_main = max(0, step_end - step_begin);
  const int n_lora = (split == 0) ? args.n_lora : 0;
  const int total = n_lora + n_main;
  // bf16 output with the reduction split over a cluster along z (the launch
  // sets cluster dims (1, 1, gridDim.z)); MH == 1 only
  const bool csplit = (OUT == kOutBf16) && MH == 1 && gridDim.z > 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NSTAGE; ++s) {
      mbar_init(&full_tma[s], 1);
      mbar_init(&full_w[s], NDW);
      mbar_init(&empty[s], 1);
    }
    mbar_init(accum_full, 1);
    mbar_init(out_full, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_d = *tmem_slot;
  griddep_wait();   // no global access before the previous grid is complete

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tmA);
      tma_prefetch_desc(&tmB);
      if (n_lora > 0) { tma_prefetch_desc(&tmA2); tma_prefetch_desc(&tmB2); }
      if (OUT == kOutDropoutAdd) {
        // the output tile the epilogue updates (tmA2 maps the output: bf16, box 64 x 128)
        mbar_arrive_expect_tx(out_full, static_cast<uint32_t>(L::kOutTileBytes));
#pragma unroll
        for (int h = 0; h < MH; ++h)
#pragma unroll
          for (int c = 0; c < BN / 64; ++c)
            tma_load_2d(smem + L::kOutOff + (h * (BN / 64) + c) * (kBM * 128), &tmA2, out_full, c0 + 64 * c,
                        m0 + h * kBM);
      }
      for (int t = 0; t < total; ++t) {
        const int s = t % NSTAGE;
        if (t >= NSTAGE && !mbar_wait(&empty[s], ((t / NSTAGE) - 1) & 1, abort_flag)) break;
        uint8_t* a_dst = smem + L::kAOff + s * kATileBytes;
        uint8_t* b_dst = smem + L::kBOff + s * L::kBTileBytes;
        if (t < n_lora) {
          // adapter slice: A2 = (s*U or s*V) [rows x r], K-major; B2 like the main B
          mbar_arrive_expect_tx(&full_tma[s], kATileBytes + L::kBTileBytes);
          tma_load_2d(a_dst, &tmA2, &full_tma[s], t * kBK, m0);
          if (BSRC == kBDeqK || BSRC == kBTmaK) {
            tma_load_2d(b_dst, &tmB2, &full_tma[s], t * kBK, c0);
          } else {
#pragma unroll
            for (int c = 0; c < BN / 64; ++c)
              tma_load_2d(b_dst + c * (kBK * 128), &tmB2, &full_tma[s], c0 + 64 * c, t * kBK);
          }
        } else {
          const int ks = step_begin + (t - n_lora);
          const uint32_t bbytes = kDeq ? L::kPTileBytes : L::kBTileBytes;
          mbar_arrive_expect_tx(&full_tma[s], kATileBytes + bbytes);
          if (A_MN) {
            tma_load_2d(a_dst, &tmA, &full_tma[s], m0, ks * kBK);
            tma_load_2d(a_dst + kBK * 128, &tmA, &full_tma[s], m0 + 64, ks * kBK);
          } else {
            tma_load_2d(a_dst, &tmA, &full_tma[s], ks * kBK, m0);
          }
          if (BSRC == kBTmaK) {
            tma_load_2d(b_dst, &tmB, &full_tma[s], ks * kBK, c0);
          } else if (BSRC == kBTmaMN) {
#pragma unroll
            for (int c = 0; c < BN / 64; ++c)
              tma_load_2d(b_dst + c * (kBK * 128), &tmB, &full_tma[s], c0 + 64 * c, ks * kBK);
          } else if (BSRC == kBDeqK) {
            // packed codes of weight rows [c0, c0+BN), k-step ks: BN rows x 32 B
            tma_load_2d(smem + L::kPOff + s * L::kPTileBytes, &tmB, &full_tma[s], ks * (kBK / 2), c0, 1);
          } else {
            // packed codes of weight rows [64 ks, 64 ks + 64), columns [c0, c0+BN): 64 rows x BN/2 B
            tma_load_2d(smem + L::kPOff + s * L::kPTileBytes, &tmB, &full_tma[s], c0 / 2, ks * kBK, 1);
          }
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    bool ok = true;
    for (int t = 0; t < total && ok; ++t) {
      const int s = t % NSTAGE;
      const uint32_t ph = (t / NSTAGE) & 1;
      ok = mbar_wait(&full_tma[s], ph, abort_flag);
      // full_w[s] completes one phase per use of stage s (the dequant warps
      // also arrive, without work, on adapter steps), so its parity is ph too
      if (ok && kDeq) ok = mbar_wait(&full_w[s], ph, abort_flag);
      if (!ok) break;
      tc_fence_after();
      if (lane == 0) {
        const uint32_t a_base = smem_u32(smem + L::kAOff + s * kATileBytes);
        const uint32_t b_base = smem_u32(smem + L::kBOff + s * L::kBTileBytes);
        // the adapter slices' A operand is always K-major
        const bool a_mn_now = A_MN && (t >= n_lora);
#pragma unroll
        for (int kk = 0; kk < kBK / 16; ++kk) {
          const uint64_t ad = a_mn_now ? smem_desc_sw128(a_base + kk * 2048, kBK * 128)
                                       : smem_desc_sw128(a_base + kk * 32, 16);
          const uint64_t bd = kBMN ? smem_desc_sw128(b_base + kk * 2048, kBK * 128)
                                   : smem_desc_sw128(b_base + kk * 32, 16);
          umma_bf16(tmem_d, ad, bd, kIdesc, (t > 0 || kk > 0) ? 1u : 0u);
          if (MH == 2)
            umma_bf16(tmem_d + BN, smem_desc_sw128(a_base + kAHalfBytes + kk * 32, 16), bd, kIdesc,
                      (t > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(&empty[s]);
      }
      __syncwarp();
    }
    if (lane == 0) umma_commit(accum_full);  // also fires (immediately) when nothing was issued
    __syncwarp();
  } else {
    // ------------------------------------------------------------ dequant
    const int item = threadIdx.x - 64;  // 0 .. NDW*32-1
    bool ok = true;
    if constexpr (kDeq) {
      float level[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) level[i] = args.level[i];
      // item -> (weight row, 64-block) of this thread, and where its bytes live
      int w_row_base, kb_base, row_stride_steps;
      if (BSRC == kBDeqK) {
        // row `item` of the B tile = weight row c0+item, block = k-step
        w_row_base = c0 + item;
        kb_base = 0;
        row_stride_steps = 0;
      } else {
        // item = (reduction row nr, 64-column block jb of the tile)
        w_row_base = item & 63;           // + 64*ks
        kb_base = c0 / 64 + (item >> 6);  // fixed block column
        row_stride_steps = 64;
      }
      auto load_scale = [&](int ks) -> float {
        const int wr = (BSRC == kBDeqK) ? w_row_base : (w_row_base + ks * row_stride_steps);
        const int kb = (BSRC == kBDeqK) ? ks : kb_base;
        if (wr >= args.w_rows || kb >= args.w_kblocks) return 0.f;
        const int64_t blk = static_cast<int64_t>(wr) * args.w_kblocks + kb;
        return block_scale(args.q8, args.s2, blk);
      };
      // scales are prefetched two steps ahead (c1_a: this step, c1_b: next)
      float c1_a = (n_main > 0) ? load_scale(step_begin) : 0.f;
      float c1_b = (n_main > 1) ? load_scale(step_begin + 1) : 0.f;
      for (int t = 0; t < total; ++t) {
        const int s = t % NSTAGE;
        const uint32_t ph = (t / NSTAGE) & 1;
        if (t < n_lora) {
          // adapter slice: B comes from TMA.  Wait for the stage's bytes like
          // any step (so these warps never run a phase ahead: a wait on a
          // later phase of a barrier whose current phase is incomplete would
          // return at once), then keep full_w[s]'s phase count in step.
          if (!mbar_wait(&full_tma[s], ph, abort_flag)) { ok = false; break; }
          __syncwarp();
          if (lane == 0) mbar_arrive(&full_w[s]);
          continue;
        }
        const int ks = step_begin + (t - n_lora);
        const float c1 = c1_a;
        c1_a = c1_b;
        if (t + 2 < total) c1_b = load_scale(ks + 2);
        const DeqTable tab = make_table(level, c1);
        if (!mbar_wait(&full_tma[s], ph, abort_flag)) { ok = false; break; }
        const uint32_t p_base = smem_u32(smem + L::kPOff + s * L::kPTileBytes);
        const uint32_t b_base = smem_u32(smem + L::kBOff + s * L::kBTileBytes);
        if (BSRC == kBDeqK) {
          // packed row `item`: 32 B, 32-byte-swizzled (16 B chunk h at h ^ ((row>>2)&1))
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
          // packed row nr: BN/2 = 128 B, 128-byte-swizzled; block jb is chunks 2jb, 2jb+1
          const int nr = item & 63;
          const int jb = item >> 6;
          const uint32_t prow = p_base + nr * 128;
          const uint4 p0 = ld_shared_v4(prow + ((static_cast<uint32_t>(2 * jb) ^ (nr & 7)) << 4));
          const uint4 p1 = ld_shared_v4(prow + ((static_cast<uint32_t>(2 * jb + 1) ^ (nr & 7)) << 4));
          const uint32_t words[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
          const uint32_t row_addr = b_base + jb * (kBK * 128) + nr * 128;
#pragma unroll
          for (int c = 0; c < 8; ++c)
            st_shared_v4(row_addr + ((static_cast<uint32_t>(c) ^ (nr & 7)) << 4), expand8(tab, words[c]));
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&full_w[s]);
      }
    }
    // ------------------------------------------------------------ epilogue
    if (ok) ok = mbar_wait(accum_full, 0, abort_flag);
    griddep_launch_dependents();
    if (ok && csplit) {
      // split-K over the cluster: copy the tile's valid rows to this CTA's
      // shared memory (fp32 [128][BN], 16-byte chunks rotated by the row);
      // they are summed across the cluster below
      float* red = reinterpret_cast<float*>(smem);
      const int q = warp & 3;
      const int grp = (warp - 2) >> 2;
      const int m_valid = min(kBM, args.m_rows - m0);
      if (q * 32 < m_valid) {
        tc_fence_after();
        const int row = q * 32 + lane;
        for (int ch = grp; ch < BN / 32; ch += NDW / 4) {
          uint32_t v[32];
          tmem_ld_32x32b_x32(tmem_d + (static_cast<uint32_t>(q * 32) << 16) + ch * 32, v);
          tmem_ld_wait();
          if (row < m_valid) {
            float4* dst = reinterpret_cast<float4*>(red + row * BN);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              float4 val = make_float4(__uint_as_float(v[4 * i]), __uint_as_float(v[4 * i + 1]),
                                       __uint_as_float(v[4 * i + 2]), __uint_as_float(v[4 * i + 3]));
              if (total == 0) val = make_float4(0.f, 0.f, 0.f, 0.f);
              dst[(ch * 8 + i + row) & (BN / 4 - 1)] = val;
            }
          }
        }
      }
    } else if (OUT == kOutDropoutAdd) {
      // masked update of the output tile (MH == 1): this thread owns row q*32 + lane and
      // the 32-column chunks ch = grp, grp + NDW/4, ...  Every keep word is loaded up
      // front and two chunks leave TMEM per wait, so the latencies overlap.
      static_assert(MH == 1, "masked update: one 128-row half");
      constexpr int kChunks = BN / 32 / (NDW / 4);
      static_assert(kChunks % 2 == 0, "chunks go in pairs");
      const int q = warp & 3;
      const int grp = (warp - 2) >> 2;
      const int rl = q * 32 + lane;
      const int row = m0 + rl;
      const bool live = ok && total > 0 && row < args.m_rows;
      uint32_t keep[kChunks];
#pragma unroll
      for (int c = 0; c < kChunks; ++c) {
        const int col = c0 + (grp + c * (NDW / 4)) * 32;
        keep[c] = (live && col < args.n_cols)
                      ? __ldg(args.drop_bits + ((static_cast<int64_t>(row) * args.ld_out + col) >> 5)) : 0u;
      }
      if (ok && total > 0) ok = mbar_wait(out_full, 0, abort_flag);
      if (ok && total > 0) {
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < kChunks; c += 2) {
          uint32_t v[2][32];
#pragma unroll
          for (int u = 0; u < 2; ++u)
            tmem_ld_32x32b_x32(tmem_d + (static_cast<uint32_t>(q * 32) << 16) + (grp + (c + u) * (NDW / 4)) * 32,
                               v[u]);
          tmem_ld_wait();
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int ch = grp + (c + u) * (NDW / 4);
            const int col = c0 + ch * 32;
            if (!live || col >= args.n_cols) continue;
            const int64_t e = static_cast<int64_t>(row) * args.ld_out + col;   // a multiple of 32
            // the current values, from the tile TMA brought in: row rl of 64-column box
            // ch / 2, 16-byte chunks (ch % 2) * 4 + i at (chunk ^ (rl & 7)) * 16
            const uint32_t box = smem_u32(smem + L::kOutOff + (ch / 2) * (kBM * 128)) + rl * 128;
            uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(args.out) + e);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const uint32_t c16 = static_cast<uint32_t>((ch & 1) * 4 + i);
              const uint4 d = ld_shared_v4(box + ((c16 ^ static_cast<uint32_t>(rl & 7)) << 4));
              const uint32_t in[4] = {d.x, d.y, d.z, d.w};
              uint32_t o[4];
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                const int b = 8 * i + 2 * j;   // element e + b (low half), e + b + 1 (high half)
                const float lo = __uint_as_float(in[j] << 16), hi = __uint_as_float(in[j] & 0xFFFF0000u);
                const float x0 = ((keep[c + u] >> b) & 1u) ? lo + args.drop_scale * __uint_as_float(v[u][b]) : lo;
                const float x1 = ((keep[c + u] >> (b + 1)) & 1u) ? hi + args.drop_scale * __uint_as_float(v[u][b + 1]) : hi;
                __nv_bfloat162 hb = __floats2bfloat162_rn(x0, x1);
                o[j] = *reinterpret_cast<uint32_t*>(&hb);
              }
              dst[i] = make_uint4(o[0], o[1], o[2], o[3]);
            }
          }
        }
      }
    } else if (ok && total > 0) {
      tc_fence_after();
      const int q = warp & 3;
      const int grp = (warp - 2) >> 2;
#pragma unroll 1
      for (int h = 0; h < MH; ++h) {
        const int row = m0 + h * kBM + q * 32 + lane;
#pragma unroll 1
        for (int ch = grp; ch < BN / 32; ch += NDW / 4) {
          uint32_t v[32];
          tmem_ld_32x32b_x32(tmem_d + (static_cast<uint32_t>(q * 32) << 16) + h * BN + ch * 32, v);
          tmem_ld_wait();
          const int col = c0 + ch * 32;
          if (row < args.m_rows && col < args.n_cols) {
            if (OUT == kOutBf16) {
              uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(args.out) +
                                                    static_cast<int64_t>(row) * args.ld_out + col);
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
                dst[i] = o;
              }
            } else {
              float4* dst = reinterpret_cast<float4*>(static_cast<float*>(args.out) + split * args.split_stride +
                                                      static_cast<int64_t>(row) * args.ld_out + col);
#pragma unroll
              for (int i = 0; i < 8; ++i)
                dst[i] = make_float4(__uint_as_float(v[4 * i]), __uint_as_float(v[4 * i + 1]),
                                     __uint_as_float(v[4 * i + 2]), __uint_as_float(v[4 * i + 3]));
            }
          }
        }
      }
    } else if (ok && OUT == kOutF32Partial) {
      // a split with no work still owns its slice of the partial buffer: zero it
      const int q = warp & 3;
      const int grp = (warp - 2) >> 2;
      for (int h = 0; h < MH; ++h) {
        const int row = m0 + h * kBM + q * 32 + lane;
        for (int ch = grp; ch < BN / 32; ch += NDW / 4) {
          const int col = c0 + ch * 32;
          if (row < args.m_rows && col < args.n_cols) {
            float4* dst = reinterpret_cast<float4*>(static_cast<float*>(args.out) + split * args.split_stride +
                                                    static_cast<int64_t>(row) * args.ld_out + col);
#pragma unroll
            for (int i = 0; i < 8; ++i) dst[i] = make_float4(0.f, 0.f, 0.f, 0.f);
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (csplit) {
    cluster_sync_all();   // every rank's partial tile is in its shared memory
    if (warp >= 2 && !*abort_flag) {
      // rank r sums its share of the valid rows' float4s over all ranks, in rank order
      const int S = static_cast<int>(gridDim.z);
      const int rank = static_cast<int>(cluster_ctarank());
      const int m_valid = min(kBM, args.m_rows - m0);
      const int n4 = m_valid * (BN / 4);
      const int lo = static_cast<int>((static_cast<int64_t>(n4) * rank) / S);
      const int hi = static_cast<int>((static_cast<int64_t>(n4) * (rank + 1)) / S);
      const uint32_t red_base = smem_u32(smem);
      for (int idx = lo + static_cast<int>(threadIdx.x) - 64; idx < hi; idx += 32 * NDW) {
        const int row = idx / (BN / 4);
        const int c4 = idx - row * (BN / 4);
        const uint32_t off = static_cast<uint32_t>(row * BN + ((c4 + row) & (BN / 4 - 1)) * 4) * 4u;
        if (!QLORA_CHECK(off + 16u <= static_cast<uint32_t>(kBM * BN * 4), kDbgCluster, off)) continue;
        float4 v[8];
#pragma unroll
        for (int p = 0; p < 8; ++p)
          if (p < S) v[p] = ld_cluster_v4(map_to_rank(red_base + off, p));
        float4 a = v[0];
#pragma unroll
        for (int p = 1; p < 8; ++p)
          if (p < S) { a.x += v[p].x; a.y += v[p].y; a.z += v[p].z; a.w += v[p].w; }
        const int col = c0 + 4 * c4;
        if (col < args.n_cols) {
          __nv_bfloat162 h0 = __floats2bfloat162_rn(a.x, a.y), h1 = __floats2bfloat162_rn(a.z, a.w);
          uint2 u;
          u.x = *reinterpret_cast<uint32_t*>(&h0);
          u.y = *reinterpret_cast<uint32_t*>(&h1);
          *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(args.out) +
                                    static_cast<int64_t>(m0 + row) * args.ld_out + col) = u;
        }
      }
    }
    cluster_sync_all();   // no rank leaves while another still reads its shared memory
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_d, kTmemCols);
  }
}

}  // namespace qlora
