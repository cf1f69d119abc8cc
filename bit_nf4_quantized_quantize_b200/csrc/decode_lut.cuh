// Few-token forward of the NF4 linear layer (M <= 8 tokens), sm_100a:
//
//   Y = X dequant(W)^T + s (X A^T) B^T
//
// At a few tokens the layer is a matrix-vector product whose only real cost
// is reading the packed weight once (0.53 byte per weight with its block
// constants).  Expanding every code to bf16 with byte permutes costs about
// three integer instructions per weight, more than the HBM stream allows, so
// this path never expands a code on its own:
//
// * One byte of packed codes holds two weights (the low nibble is the even
//   element).  A shared-memory table maps the byte to the pair of NF4 levels
//   (fp16): one byte permute forms the table address and one shared load
//   returns the pair, which is directly an f16x2 operand register of
//   mma.sync.m16n8k16.  The table has one copy per lane in the address bits
//   that pick the bank (entry e of lane copy c at e * 256 + c * 4), so the 32
//   lanes of a warp never conflict whatever bytes they look up.
// * The tensor core does the dot products: 16 weight rows x 16 columns per
//   instruction against up to 8 tokens (the N side), fp32 accumulation.  An
//   instruction's 16 k slots may stand for any 16 columns as long as the
//   weight and activation operands agree, so a lane's four code bytes per
//   instruction are contiguous in memory (8 bytes per row and 64-column
//   block).  Each 64-column block of a row is one instruction group of four,
//   whose fresh fp32 result is scaled by the block constant c1 and added to
//   the row's total, so the weight the product uses is the fp32 dequantized
//   value level * c1 (to the level's fp16 rounding, 2^-11 relative), not the
//   bf16 rounding of it that the larger-M paths multiply with; both are within
//   the layer's tolerance of the bf16 reference.
// * Activations are fp16 after scaling each 64-column block of a token by a
//   power of two that brings its largest magnitude into [2^14, 2^15) (exact
//   for every bf16 value in fp16's normal range); a block's fp32 result is
//   multiplied by the inverse power of two together with c1.
//
// Work split: a CTA owns T tiles of 16 consecutive rows and all of K.  A
// producer warp first copies the M token rows of X (bf16, one bulk copy per
// token, into padded rows that the compute warps convert to scaled fp16 in
// place) and the 8-bit block constants of all the CTA's rows, then streams
// the tiles through a ring of shared-memory slots, one bulk asynchronous copy
// per row into rows padded so that the consumers' 8-byte operand loads never
// conflict.  The compute warps build the lookup table while those copies
// land.  The c1 and activation-scale tables are stored by row with a stride
// of 4 mod 32 floats, so one 16-byte load brings four blocks' scales of a row
// without bank conflicts.  The 16 compute warps work on one tile at a time,
// each on its own range of 64-column blocks, and leave their partial row
// totals in shared memory; the epilogue adds the 16 partials in warp order
// (so the result does not depend on timing), adds s (U B^T) and writes bf16 Y.
//
// Ordering.  qlora_decode_u_kernel (U = X A^T, launched just before this
// kernel on the same stream) starts early, prefetches this kernel's weight
// lines into L2 (a hint: it changes no value any read returns), waits for the
// previous grid, and only then lets this kernel be scheduled.  So when this
// kernel starts every grid before the adapter kernel has completed, and it
// reads the weight, X and B at once; it waits for the adapter kernel itself
// (griddepcontrol.wait) only before it reads U and writes Y.  It lets the next
// grid be scheduled as soon as it starts, so the next layer's adapter kernel
// prefetches that layer's weight while this one computes.  Every wait on a
// copy or a slot is bounded.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include "ptx_sm100.cuh"
#include "gemm_tc.cuh"

namespace qlora {

constexpr int kLutMaxTokens = 8;                 // the kernel's limit (the MMA's N side)
constexpr int kLutWarps = 16;                     // compute warps
constexpr int kLutThreads = 32 * (kLutWarps + 1); // and one producer warp
constexpr int kLutTableBytes = 256 * 256;         // 256 byte values x 256-byte rows (32 lane copies of 4 B used)
constexpr int kLutTile = 16;                      // weight rows of one tile (the MMA's M)
constexpr int kLutMaxSlots = 4;
constexpr int kLutMaxSmem = 224 * 1024;
constexpr int kDecUThreads = 128;

struct LutArgs {
  const uint8_t* codes;  // packed codes, N rows of K/2 bytes
  const uint8_t* q8;     // 8-bit block constants (16-byte aligned), or NULL (single quantization: s2 = absmax)
  const float* s2;
  const uint16_t* x;     // bf16 [M x K]
  const uint16_t* b;     // bf16 [N x r]
  const float* u;        // fp32 [M x r] = X A^T (qlora_decode_u_kernel)
  uint16_t* y;           // bf16 [M x N]
  int m, n, k, r;
  int tiles_per_cta;     // T
  int n_slots;           // ring slots (<= kLutMaxSlots)
  float s;               // alpha / r
  float level[16];       // NF4 levels (fp32)
};

// Row stride of a tile slot: K/2 bytes padded so that the stride in 4-byte
// words is 8 mod 32 (the 16 lanes of a half warp then hit 16 distinct bank
// pairs with their 8-byte loads); a multiple of 16 bytes.
__host__ __device__ constexpr int lut_row_stride(int k) { return k / 2 + 4 * ((8 - (k / 8) % 32 + 32) % 32); }

// Row stride of X in shared memory (halves): K padded by 8, so that the rows
// of different tokens fall in different banks.
__host__ __device__ constexpr int lut_x_stride(int k) { return k + 8; }
// Row stride (floats) of the c1 table ([row][block]) and of the activation scales
// ([token][block]): at least the number of blocks, a multiple of 4 and 4 mod 32, so that a
// lane's 16-byte load of four consecutive blocks is aligned and the 8 rows (tokens) a warp
// reads at once fall in 8 distinct groups of 4 banks.
__host__ __device__ constexpr int lut_scale_stride(int kblocks) { return kblocks + ((4 - kblocks) % 32 + 32) % 32; }
// Floats per (row, token) of the partial totals: the 16 warps' values and one
// of padding, so that consecutive rows fall in different banks.
constexpr int kLutPartStride = kLutWarps + 1;

// Shared-memory layout of one CTA; every part starts on a 16-byte boundary.
//   table | ring (slots x 16 padded rows) | block constants of the CTA's rows (the
//   16-byte aligned span holding them: q8 bytes, or fp32 absmax when single) |
//   group scales s2 of those rows | c1 of every block of those rows (fp32,
//   [row][block], rows of lut_scale_stride) | X (fp16, scaled per 64-column block,
//   rows of lut_x_stride) | 2^e per token and block (rows of lut_scale_stride) | partial totals
//   [T * 16 rows][m][kLutPartStride] | U (fp32) | B rows (bf16) | barriers: full, empty
//   per slot, constants, X | abort word
struct LutLayout {
  int ring, consts, s2g, c1, x, xsc, part, u, b, bars, abort_word, total;
};
__host__ __device__ constexpr int lut_align16(int x) { return (x + 15) / 16 * 16; }
__host__ __device__ inline LutLayout lut_layout(int m, int k, int tiles, int n_slots, int r, bool single) {
  LutLayout L{};
  const int rows = tiles * kLutTile;
  const int kblocks = k / 64;
  L.ring = kLutTableBytes;
  L.consts = L.ring + n_slots * kLutTile * lut_row_stride(k);
  L.s2g = L.consts + lut_align16(rows * kblocks * (single ? 4 : 1) + 32);
  L.c1 = L.s2g + lut_align16((single ? 0 : rows * kblocks / 256 + 2) * 4);
  L.x = L.c1 + lut_align16(rows * lut_scale_stride(kblocks) * 4);
  L.xsc = L.x + lut_align16(m * lut_x_stride(k) * 2);
  L.part = L.xsc + lut_align16(m * lut_scale_stride(kblocks) * 4);
  L.u = L.part + lut_align16(rows * m * kLutPartStride * 4);
  L.b = L.u + lut_align16(m * r * 4);
  L.bars = L.b + lut_align16(rows * r * 2);
  L.abort_word = L.bars + (2 * kLutMaxSlots + 2) * 8;
  L.total = L.abort_word + 16;
  return L;
}

__device__ __forceinline__ uint4 ld_cg_v4(const void* p) {
  uint4 v;
  asm volatile("ld.global.cg.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
  return v;
}

// Bulk asynchronous copy global -> this CTA's shared memory, completion as
// transaction bytes on `bar`.  Both addresses and the size are multiples of 16.
__device__ __forceinline__ void lut_bulk_copy(void* smem_dst, const void* gsrc, uint32_t bytes, uint64_t* bar) {
  if (!QLORA_CHECK((bytes & 15u) == 0 && (reinterpret_cast<uintptr_t>(gsrc) & 15u) == 0, kDbgBulk, bytes) ||
      !QLORA_CHECK((smem_u32(smem_dst) & 15u) == 0, kDbgSmemAlign, smem_u32(smem_dst)))
    return;
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
               ::"r"(smem_u32(smem_dst)), "l"(gsrc), "r"(bytes), "r"(smem_u32(bar)) : "memory");
}

// Wait for a copy that may still be in flight when the CTA gives up: bounded,
// and not cut short by the abort word (the CTA must not exit while a copy can
// still write its shared memory).
__device__ __forceinline__ void lut_drain(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > kWaitLimitNs) {
      atomicExch(&g_device_error, kDevErrTimeout);
      return;
    }
    __nanosleep(256);
  }
}

// Bring the 128-byte line holding p into L2 (a hint: it changes no value that
// any later read returns, so it may run before the grid-dependency wait).
__device__ __forceinline__ void prefetch_l2_line(const void* p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

// c1 of a block from its raw stored constants (the forms of block_scale).
__device__ __forceinline__ float lut_block_scale(bool has_q8, uint32_t q, float sv) {
  if (!has_q8) return sv;
  if (signbit(sv)) return __fmul_rn(e4m3_to_f32(q), -sv);
  return __fmul_rn(static_cast<float>(q), sv);
}

// Shared-memory loads at 32-bit shared-window addresses (no generic-address
// conversion per access).
__device__ __forceinline__ uint32_t lds_u32(uint32_t a) {
  uint32_t v;
  asm("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a));
  return v;
}
__device__ __forceinline__ uint2 lds_v2(uint32_t a) {
  uint2 v;
  asm("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(a));
  return v;
}
__device__ __forceinline__ uint4 lds_v4(uint32_t a) {
  uint4 v;
  asm("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
  return v;
}
__device__ __forceinline__ float lds_f32(uint32_t a) {
  float v;
  asm("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(a));
  return v;
}

// 2^e as fp32 for e in [-126, 127].
__device__ __forceinline__ float exp2_int(int e) { return __uint_as_float(static_cast<uint32_t>(e + 127) << 23); }

// D = A B (fp16 operands, fp32 result), m16n8k16, fragments as the PTX ISA
// lays them out for lane (g = lane / 4, t = lane % 4).
__device__ __forceinline__ void mma_f16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                              uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%10, %11, %12, %13};"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(d[0]), "f"(d[1]), "f"(d[2]), "f"(d[3]));
}

__global__ void __launch_bounds__(kLutThreads, 1) qlora_decode_lut_kernel(const LutArgs args) {
  extern __shared__ __align__(1024) uint8_t lut_smem[];
  const int K = args.k;
  const int m = args.m;
  const int r = args.r;
  const int T = args.tiles_per_cta;
  const int n_slots = args.n_slots;
  const bool has_q8 = args.q8 != nullptr;
  const LutLayout L = lut_layout(m, K, T, n_slots, r, !has_q8);
  uint8_t* ring = lut_smem + L.ring;
  uint8_t* consts = lut_smem + L.consts;
  float* s2g = reinterpret_cast<float*>(lut_smem + L.s2g);
  float* c1s = reinterpret_cast<float*>(lut_smem + L.c1);   // [local row][block]
  __half* xs = reinterpret_cast<__half*>(lut_smem + L.x);
  float* xsc = reinterpret_cast<float*>(lut_smem + L.xsc);   // [token][block]: 2^e
  float* part = reinterpret_cast<float*>(lut_smem + L.part);
  float* us = reinterpret_cast<float*>(lut_smem + L.u);
  uint16_t* bs = reinterpret_cast<uint16_t*>(lut_smem + L.b);
  uint64_t* full = reinterpret_cast<uint64_t*>(lut_smem + L.bars);   // [slot]
  uint64_t* empty = full + kLutMaxSlots;                              // [slot]
  uint64_t* consts_bar = empty + kLutMaxSlots;
  uint64_t* x_bar = consts_bar + 1;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(lut_smem + L.abort_word);
  int* issued = reinterpret_cast<int*>(lut_smem + L.abort_word) + 1;   // tiles the producer copied

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int tiles_total = args.n / kLutTile;
  const int tile0 = blockIdx.x * T;
  const int tiles_here = max(0, min(T, tiles_total - tile0));
  const int row0 = tile0 * kLutTile;
  const int rows_here = tiles_here * kLutTile;
  const int64_t row_bytes = K / 2;
  const int rs = lut_row_stride(K);
  const int slot_bytes = kLutTile * rs;
  const int kblocks = K / 64;
  const int ss = lut_scale_stride(kblocks);   // row stride of the c1 and X-scale tables
  const uint8_t* cta_codes = args.codes + static_cast<int64_t>(row0) * row_bytes;
  // the 16-byte aligned span holding the block constants of the CTA's rows
  const int csize = has_q8 ? 1 : 4;
  const uint8_t* cbase = has_q8 ? args.q8 : reinterpret_cast<const uint8_t*>(args.s2);
  const int64_t c_lo = static_cast<int64_t>(row0) * kblocks * csize;
  const int64_t c_hi = static_cast<int64_t>(row0 + rows_here) * kblocks * csize;
  const int c_delta = static_cast<int>(c_lo & 15);
  const uint8_t* cspan = cbase + (c_lo & ~int64_t(15));
  const uint32_t cbytes = static_cast<uint32_t>(((c_hi + 15) & ~int64_t(15)) - (c_lo & ~int64_t(15)));
  const int64_t g_lo = (static_cast<int64_t>(row0) * kblocks) >> 8;   // first group scale of the CTA's rows

  griddep_launch_dependents();   // the next grid may be scheduled now
  // the compute threads' global loads go out first: B rows, group scales (X comes by bulk copy)
  const int xpieces = m * K / 8;
  uint4 bq = make_uint4(0u, 0u, 0u, 0u);
  float sgq = 0.f;
  if (warp < kLutWarps) {
    if (tid < rows_here * r / 8) bq = ld_cg_v4(args.b + static_cast<int64_t>(row0) * r + tid * 8);
    if (has_q8 && rows_here > 0) {
      const int64_t g_hi = (static_cast<int64_t>(row0 + rows_here) * kblocks - 1) >> 8;
      if (tid <= g_hi - g_lo) sgq = __ldg(args.s2 + g_lo + tid);
    }
  }
  if (tid == kLutWarps * 32) {
    for (int i = 0; i < kLutMaxSlots; ++i) {
      mbar_init(full + i, 1);
      mbar_init(empty + i, kLutWarps);
    }
    mbar_init(consts_bar, 1);
    mbar_init(x_bar, 1);
    *abort_flag = 0;
    *issued = 0;
    fence_barrier_init();
  }
  __syncthreads();

  if (warp == kLutWarps) {
    // ---------------------------------------------------------------- producer
    // X rows first (one bulk copy per token, bf16, into the token's padded row: converted in
    // place), then the block constants
    if (lane == 0) mbar_arrive_expect_tx(x_bar, static_cast<uint32_t>(m * K * 2));
    __syncwarp();
    if (lane < m)
      lut_bulk_copy(xs + lane * lut_x_stride(K), args.x + static_cast<int64_t>(lane) * K, static_cast<uint32_t>(K * 2),
                    x_bar);
    if (lane == 0 && rows_here > 0) {
      mbar_arrive_expect_tx(consts_bar, cbytes);
      lut_bulk_copy(consts, cspan, cbytes, consts_bar);
    }
    bool ok = true;
    for (int c = 0; c < tiles_here && ok; ++c) {
      const int slot = c % n_slots;
      if (c >= n_slots) ok = __all_sync(0xffffffffu, mbar_wait(empty + slot, (c / n_slots - 1) & 1, abort_flag));
      if (!ok) break;
      if (lane == 0) mbar_arrive_expect_tx(full + slot, static_cast<uint32_t>(kLutTile * row_bytes));
      __syncwarp();
      if (lane < kLutTile)
        lut_bulk_copy(ring + slot * slot_bytes + lane * rs, cta_codes + static_cast<int64_t>(c * kLutTile + lane) * row_bytes,
                      static_cast<uint32_t>(row_bytes), full + slot);
      if (lane == 0) *issued = c + 1;
    }
    // then U, once the adapter kernel has completed (the epilogue reads it after the CTA barrier)
    griddep_wait();
    for (int i = lane; i < m * r; i += 32) us[i] = args.u[i];
  } else {
    // ---------------------------------------------------------------- compute warps
    const int ctid = tid;   // 0 .. 511
    // table: entry for byte value e, lane copy c = fp16 (level[e & 15], level[e >> 4]) at e * 256 + c * 4
    // (built while the X rows are in flight)
    for (int i = ctid; i < 256 * 8; i += kLutWarps * 32) {
      const int e = i >> 3;
      const __half2 h = __floats2half2_rn(args.level[e & 15], args.level[e >> 4]);
      const uint32_t v = *reinterpret_cast<const uint32_t*>(&h);
      *reinterpret_cast<uint4*>(lut_smem + e * 256 + (i & 7) * 16) = make_uint4(v, v, v, v);
    }
    if (ctid < rows_here * r / 8) *reinterpret_cast<uint4*>(bs + ctid * 8) = bq;
    for (int i = ctid + kLutWarps * 32; i < rows_here * r / 8; i += kLutWarps * 32)
      *reinterpret_cast<uint4*>(bs + i * 8) = ld_cg_v4(args.b + static_cast<int64_t>(row0) * r + i * 8);
    if (has_q8 && rows_here > 0) {
      const int64_t g_hi = (static_cast<int64_t>(row0 + rows_here) * kblocks - 1) >> 8;
      if (ctid <= g_hi - g_lo) s2g[ctid] = sgq;
      for (int i = ctid + kLutWarps * 32; i <= g_hi - g_lo; i += kLutWarps * 32) s2g[i] = __ldg(args.s2 + g_lo + i);
    }
    // X, in place: 16-byte pieces (8 values); the 8 pieces of a 64-column block sit in 8 consecutive lanes
    const bool x_ok = __all_sync(0xffffffffu, mbar_wait(x_bar, 0, abort_flag));
    for (int i0 = warp * 32; x_ok && i0 < xpieces; i0 += kLutWarps * 32) {
      const int i = i0 + lane;
      const int tk = i / (K / 8), col8 = i - tk * (K / 8);   // token, 8-column piece
      uint4* px = reinterpret_cast<uint4*>(xs + tk * lut_x_stride(K) + col8 * 8);
      const uint4 v = i < xpieces ? *px : make_uint4(0u, 0u, 0u, 0u);
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
      uint32_t mx = 0u;
#pragma unroll
      for (int q = 0; q < 4; ++q) mx = max(mx, max(w[q] & 0x7FFFu, (w[q] >> 16) & 0x7FFFu));
      mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
      // largest magnitude in [2^(E-127), 2^(E-126)) for biased exponent E: scale by 2^(141-E)
      const int e = max(static_cast<int>(mx >> 7) - 141, -126);
      const float down = exp2_int(-e);
      if (i < xpieces) {
        uint32_t h[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const __half2 hv = __floats2half2_rn(__fmul_rn(__uint_as_float(w[q] << 16), down),
                                               __fmul_rn(__uint_as_float(w[q] & 0xFFFF0000u), down));
          h[q] = *reinterpret_cast<const uint32_t*>(&hv);
        }
        *px = make_uint4(h[0], h[1], h[2], h[3]);
        if ((lane & 7) == 0) xsc[tk * ss + col8 / 8] = exp2_int(e);   // [token][block]
      }
    }
    named_bar_sync(1, kLutWarps * 32);   // table, X, block scales of X, B rows

    const int g = lane >> 2;   // fragment row (and token) group
    const int t = lane & 3;    // thread in group
    const int seg_lo = (kblocks * warp) / kLutWarps;   // this warp's 64-column blocks
    const int seg_hi = (kblocks * (warp + 1)) / kLutWarps;
    const uint32_t lane_sel = static_cast<uint32_t>(lane * 4);   // byte 0 of the table address
    const bool tok_ok = g < m;                                   // this lane's B operand column is a real token
    // 32-bit shared-memory offsets of this lane's operands (block seg adds seg * 32, seg * 64 or seg)
    const uint32_t code_g = static_cast<uint32_t>(g * rs + 8 * t), code_h = code_g + 8u * static_cast<uint32_t>(rs);
    const uint32_t x_off = static_cast<uint32_t>(g * lut_x_stride(K) + 16 * t);   // in halves
    const uint32_t xsc0 = static_cast<uint32_t>(2 * t * ss), xsc1 = xsc0 + static_cast<uint32_t>(ss);   // + block
    const bool sx0_ok = 2 * t < m, sx1_ok = 2 * t + 1 < m;
    bool ok = x_ok && (rows_here == 0 || __all_sync(0xffffffffu, mbar_wait(consts_bar, 0, abort_flag)));
    // c1 of every block of the CTA's rows, from the stored constants
    if (ok) {
      const uint32_t s2_first = static_cast<uint32_t>(row0) * static_cast<uint32_t>(kblocks);
      for (int i = ctid; i < rows_here * kblocks; i += kLutWarps * 32) {
        const int rl = i / kblocks, bl = i - rl * kblocks;
        float v;
        if (has_q8)
          v = lut_block_scale(true, consts[c_delta + i], s2g[((s2_first + i) >> 8) - static_cast<uint32_t>(g_lo)]);
        else
          v = *reinterpret_cast<const float*>(consts + c_delta + i * 4);
        c1s[rl * ss + bl] = v;
      }
    }
    named_bar_sync(1, kLutWarps * 32);   // c1
    // one 64-column block: code bytes of rows g, g + 8 at code_g / code_h + blk * 32 of the slot
    const uint32_t lut_base = smem_u32(lut_smem);
    const uint32_t c1_base = smem_u32(c1s), xsc_base = smem_u32(xsc), x_base = smem_u32(xs) + 2u * x_off;
    auto block = [&](uint32_t slot_base, uint32_t blk, float cg, float ch, float sx0, float sx1, float (&acc)[4]) {
      const uint2 wg = lds_v2(slot_base + code_g + blk * 32u);
      const uint2 wh = lds_v2(slot_base + code_h + blk * 32u);
      uint4 xa = make_uint4(0u, 0u, 0u, 0u), xb = make_uint4(0u, 0u, 0u, 0u);
      if (tok_ok) {
        xa = lds_v4(x_base + blk * 128u);
        xb = lds_v4(x_base + blk * 128u + 16u);
      }
      const uint32_t xv[8] = {xa.x, xa.y, xa.z, xa.w, xb.x, xb.y, xb.z, xb.w};
      float d[4] = {0.f, 0.f, 0.f, 0.f}, e[4] = {0.f, 0.f, 0.f, 0.f};   // two chains: j even, j odd
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        // code bytes 2j, 2j + 1 of this lane's 8: columns 16t + 4j + {0, 1} and + {2, 3}
        const uint32_t wgj = j < 2 ? wg.x : wg.y, whj = j < 2 ? wh.x : wh.y;
        const uint32_t s0b = 0x5504u | (static_cast<uint32_t>((2 * j) & 3) << 4);
        const uint32_t s1b = 0x5504u | (static_cast<uint32_t>((2 * j + 1) & 3) << 4);
        const uint32_t a0 = lds_u32(lut_base + prmt(wgj, lane_sel, s0b));
        const uint32_t a1 = lds_u32(lut_base + prmt(whj, lane_sel, s0b));
        const uint32_t a2 = lds_u32(lut_base + prmt(wgj, lane_sel, s1b));
        const uint32_t a3 = lds_u32(lut_base + prmt(whj, lane_sel, s1b));
        if (j & 1) mma_f16_16816(e, a0, a1, a2, a3, xv[2 * j], xv[2 * j + 1]);
        else mma_f16_16816(d, a0, a1, a2, a3, xv[2 * j], xv[2 * j + 1]);
      }
      acc[0] = __fmaf_rn(__fmul_rn(cg, sx0), __fadd_rn(d[0], e[0]), acc[0]);
      acc[1] = __fmaf_rn(__fmul_rn(cg, sx1), __fadd_rn(d[1], e[1]), acc[1]);
      acc[2] = __fmaf_rn(__fmul_rn(ch, sx0), __fadd_rn(d[2], e[2]), acc[2]);
      acc[3] = __fmaf_rn(__fmul_rn(ch, sx1), __fadd_rn(d[3], e[3]), acc[3]);
    };
    for (int c = 0; c < tiles_here && ok; ++c) {
      const int slot = c % n_slots;
      ok = __all_sync(0xffffffffu, mbar_wait(full + slot, (c / n_slots) & 1, abort_flag));
      if (!ok) break;
      const uint32_t sbase = smem_u32(ring) + static_cast<uint32_t>(slot * slot_bytes);
      const uint32_t c1_row = static_cast<uint32_t>(c * kLutTile + g);
      float acc[4] = {0.f, 0.f, 0.f, 0.f};   // rows g, g + 8 x tokens 2t, 2t + 1
      const uint32_t cg_row = c1_base + 4u * c1_row * static_cast<uint32_t>(ss);
      const uint32_t ch_row = cg_row + 4u * 8u * static_cast<uint32_t>(ss);
      // one block with its scales loaded one by one (tokens past m: scale 0)
      auto block1 = [&](int b) {
        const uint32_t ub = static_cast<uint32_t>(b);
        block(sbase, ub, lds_f32(cg_row + 4u * ub), lds_f32(ch_row + 4u * ub),
              sx0_ok ? lds_f32(xsc_base + 4u * (xsc0 + ub)) : 0.f, sx1_ok ? lds_f32(xsc_base + 4u * (xsc1 + ub)) : 0.f,
              acc);
      };
      int blk = seg_lo;
      for (; blk < seg_hi && (blk & 3) != 0; ++blk) block1(blk);
      for (; blk + 4 <= seg_hi; blk += 4) {   // four blocks at a time: one 16-byte load per scale row
        const uint32_t ub = static_cast<uint32_t>(blk);
        const uint4 cg4 = lds_v4(cg_row + 4u * ub), ch4 = lds_v4(ch_row + 4u * ub);
        uint4 s04 = make_uint4(0u, 0u, 0u, 0u), s14 = make_uint4(0u, 0u, 0u, 0u);
        if (sx0_ok) s04 = lds_v4(xsc_base + 4u * (xsc0 + ub));
        if (sx1_ok) s14 = lds_v4(xsc_base + 4u * (xsc1 + ub));
        block(sbase, ub, __uint_as_float(cg4.x), __uint_as_float(ch4.x), __uint_as_float(s04.x), __uint_as_float(s14.x), acc);
        block(sbase, ub + 1u, __uint_as_float(cg4.y), __uint_as_float(ch4.y), __uint_as_float(s04.y), __uint_as_float(s14.y), acc);
        block(sbase, ub + 2u, __uint_as_float(cg4.z), __uint_as_float(ch4.z), __uint_as_float(s04.z), __uint_as_float(s14.z), acc);
        block(sbase, ub + 3u, __uint_as_float(cg4.w), __uint_as_float(ch4.w), __uint_as_float(s04.w), __uint_as_float(s14.w), acc);
      }
      for (; blk < seg_hi; ++blk) block1(blk);
      // partial totals of this warp, [tile row][token][warp]; then the slot is free
      float* pt = part + static_cast<int64_t>(c * kLutTile) * m * kLutPartStride;
      if (2 * t < m) {
        pt[(g * m + 2 * t) * kLutPartStride + warp] = acc[0];
        pt[((g + 8) * m + 2 * t) * kLutPartStride + warp] = acc[2];
      }
      if (2 * t + 1 < m) {
        pt[(g * m + 2 * t + 1) * kLutPartStride + warp] = acc[1];
        pt[((g + 8) * m + 2 * t + 1) * kLutPartStride + warp] = acc[3];
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(empty + slot);
    }
  }
  __syncthreads();
  if (*abort_flag) {
    if (tid == kLutWarps * 32) {
      // a wait gave up: let every copy still in flight land before the CTA exits
      // (the last tile the producer copied into each slot)
      const int n_issued = *issued;
      for (int sl = 0; sl < min(n_issued, n_slots); ++sl) {
        const int last = sl + ((n_issued - 1 - sl) / n_slots) * n_slots;
        lut_drain(full + sl, (last / n_slots) & 1);
      }
      if (rows_here > 0) lut_drain(consts_bar, 0);
      lut_drain(x_bar, 0);
    }
    return;
  }

  // ---------------------------------------------------------------- epilogue
  // (the producer waited for the adapter kernel and loaded U before the CTA barrier above)
  for (int idx = tid; idx < rows_here * m; idx += kLutThreads) {
    const int tk = idx / rows_here;
    const int rl = idx - tk * rows_here;
    const float* pp = part + (static_cast<int64_t>(rl) * m + tk) * kLutPartStride;
    float y = 0.f;
#pragma unroll
    for (int w = 0; w < kLutWarps; ++w) y = __fadd_rn(y, pp[w]);
    float a = 0.f;
    const uint16_t* brow = bs + rl * r;
    const float* urow = us + tk * r;
    for (int j = 0; j < r; j += 8) {
      const uint4 bv = *reinterpret_cast<const uint4*>(brow + j);
      const uint32_t bw[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        a = __fmaf_rn(__uint_as_float(bw[q] << 16), urow[j + 2 * q], a);
        a = __fmaf_rn(__uint_as_float(bw[q] & 0xFFFF0000u), urow[j + 2 * q + 1], a);
      }
    }
    y = __fmaf_rn(args.s, a, y);
    const __nv_bfloat16 yb = __float2bfloat16_rn(y);
    args.y[static_cast<int64_t>(tk) * args.n + row0 + rl] = *reinterpret_cast<const uint16_t*>(&yb);
  }
}

// U = X A^T for the few-token forward: CTA j < r computes column j of U
// (every token), fp32 into u32 and bf16 into u_save when given.  Before its
// dependency wait every CTA prefetches into L2 the packed codes and block
// constants that CTA j of the table kernel will read (rows [16 T j,
// 16 T (j + 1))): a hint only.  It lets the table kernel be scheduled only
// after the wait, so that kernel starts after every earlier grid completed.
struct DecUArgs {
  const uint16_t* x;     // bf16 [M x K]
  const uint16_t* a;     // bf16 [r x K]
  int m, k, r;
  float* u32;            // fp32 [M x r]
  uint16_t* u_save;      // bf16 [M x r] or NULL
  const uint8_t* codes;  // the table kernel's weight, for the prefetch
  const uint8_t* consts; // q8 bytes, or fp32 absmax (single quantization)
  int consts_size;       // bytes per block constant (1 or 4)
  int n, rows_per_cta;
};

template <int MT>
__global__ void __launch_bounds__(kDecUThreads) qlora_decode_u_kernel(const DecUArgs args) {
  __shared__ float red[kDecUThreads / 32][MT];
  const int j = blockIdx.x;
  const int k = args.k;
  {
    const int64_t r0 = static_cast<int64_t>(j) * args.rows_per_cta;
    const int64_t r1 = min(static_cast<int64_t>(args.n), r0 + args.rows_per_cta);
    if (r1 > r0) {
      const uint8_t* cp = args.codes + r0 * (k / 2);
      const int64_t cb = (r1 - r0) * (k / 2);
      for (int64_t off = static_cast<int64_t>(threadIdx.x) * 128; off < cb; off += kDecUThreads * 128)
        prefetch_l2_line(cp + off);
      const int64_t q0 = r0 * (k / 64) * args.consts_size, q1 = r1 * (k / 64) * args.consts_size;
      for (int64_t off = (q0 & ~int64_t(127)) + threadIdx.x * 128; off < q1; off += kDecUThreads * 128)
        prefetch_l2_line(args.consts + off);
    }
  }
  griddep_wait();
  griddep_launch_dependents();   // every earlier grid has completed: the table kernel may start
  if (j >= args.r) return;
  const int m = args.m;
  const uint16_t* arow = args.a + static_cast<int64_t>(j) * k;
  float acc[MT];
#pragma unroll
  for (int tk = 0; tk < MT; ++tk) acc[tk] = 0.f;
  // columns c0 + 1024 i (i < 4) per pass: the pass's loads are issued together
  for (int c0 = threadIdx.x * 8; c0 < k; c0 += kDecUThreads * 8 * 4) {
    uint4 av[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int c = c0 + i * kDecUThreads * 8;
      av[i] = c < k ? *reinterpret_cast<const uint4*>(arow + c) : make_uint4(0u, 0u, 0u, 0u);
    }
    uint4 xv[MT][4];   // every token's loads of this pass go out together
#pragma unroll
    for (int tk = 0; tk < MT; ++tk)
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int c = c0 + i * kDecUThreads * 8;
        xv[tk][i] = (tk < m && c < k) ? *reinterpret_cast<const uint4*>(args.x + static_cast<int64_t>(tk) * k + c)
                                      : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
    for (int tk = 0; tk < MT; ++tk) {
      if (tk >= m) break;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint32_t aw[4] = {av[i].x, av[i].y, av[i].z, av[i].w};
        const uint32_t xw[4] = {xv[tk][i].x, xv[tk][i].y, xv[tk][i].z, xv[tk][i].w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          acc[tk] = __fmaf_rn(__uint_as_float(aw[q] << 16), __uint_as_float(xw[q] << 16), acc[tk]);
          acc[tk] = __fmaf_rn(__uint_as_float(aw[q] & 0xFFFF0000u), __uint_as_float(xw[q] & 0xFFFF0000u), acc[tk]);
        }
      }
    }
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
#pragma unroll
  for (int tk = 0; tk < MT; ++tk) {
    float v = acc[tk];
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0) red[warp][tk] = v;
  }
  __syncthreads();
  if (threadIdx.x < m) {
    const int tk = threadIdx.x;
    float v = 0.f;
    for (int w = 0; w < kDecUThreads / 32; ++w) v = __fadd_rn(v, red[w][tk]);
    args.u32[static_cast<int64_t>(tk) * args.r + j] = v;
    if (args.u_save) {
      const __nv_bfloat16 h = __float2bfloat16_rn(v);
      args.u_save[static_cast<int64_t>(tk) * args.r + j] = *reinterpret_cast<const uint16_t*>(&h);
    }
  }
}

}  // namespace qlora
