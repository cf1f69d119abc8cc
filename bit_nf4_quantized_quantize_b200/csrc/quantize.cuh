// NF4 quantization with double quantization, and dequantization, for sm_100a.
//
// "QLoRAの理論と実装" §5-1 (absmax per 64-block, w/absmax, nearest of the 16
// NormalFloat levels, 4-bit code) and §5-2 (8-bit re-quantization of the fp32
// absmax constants in groups of 256, one fp32 second-level constant; without
// that second stage the fp32 absmax constants are stored as they are).
//
// quantize_nf4_kernel<kMode>: a persistent grid, one CTA of 1024 threads per
// SM.  A group is 256 blocks (16384 weights, 64 KiB of fp32 input); CTA b
// takes groups b, b + grid, b + 2 grid, ...  The groups stream into a ring of
// three shared-memory stages with bulk asynchronous copies (one copy per
// group, completion counted in bytes on the stage's mbarrier), so the loads
// of the next two groups are in flight while the warps code the current one.
// Eight threads share a 64-block (8 consecutive weights each, two 16-byte
// shared loads whose order alternates with lane bit 2, so a warp's 512 bytes
// fall on 32 distinct banks); the block absmax is a 3-step xor-shuffle max.
// The warps run free of block-wide barriers: a warp that has coded its part
// of a group counts itself on the stage's counter, and the warp that
// completes the count refills the stage with the group three ahead.  The
// absmax values stay in a shared-memory ring, so the fp32 constants never go
// to HBM; the second-level quantization of the CTA's i-th group runs three
// groups later, on the eight warps 8 (i mod 4) .. 8 (i mod 4) + 7 (one absmax
// value per lane), right after they see group i + 3 arrive -- which proves
// every warp has finished group i -- so that work is spread evenly over the
// warps instead of delaying one of them.  The last three groups get theirs
// after a final barrier.  Traffic per weight: 4 B read, 0.5 + 1/64 + 4/16384
// B written with a second stage, or 0.5 + 4/64 B written when the second
// stage is off and the absmax constants are stored.
//
// Nearest level.  The code of n = fp32(w / absmax) is #{i : n > mid_i}, mid_i
// the exact midpoint of levels i and i+1; with thr_i the smallest fp32 above
// mid_i this is #{i : n >= thr_i}.  Cells of width 1/16 over [-1, 1] hold at
// most one midpoint each (the midpoints are >= 0.088 apart), so code =
// lo[cell] + (n > mid[cell]) with cell = floor(16 n) + 16.  Both the cell and
// the comparison use the scaled value t = 16 n + 15.875 in [-0.125, 31.875]:
// fp32(t + 1.5 * 2^21) lies in the binade of ulp 1/4, so its bits, masked to
// 0xFC, are 4 * floor(t + 1/8) = 4 * cell (ties of the rounding fall on the
// cell that owns them) -- the byte offset of a 4-byte table entry, taken
// modulo 64 entries.
//
// Fast path: t' = fp32(w * rcp16 + 15.875), rcp16 = 16 * rcp.approx(absmax)
// (relative error at most 2^-23), is within 2^-18 of t (the reciprocal's and
// the fma's rounding, plus the rounding of n).  The fast table holds B =
// fp32(16 mid + 15.875) with the cell's left-edge code in its 4 low mantissa
// bits (moving B by less than 2^-15), and the code is lo + sign(B - t').
// That decision equals the exact one whenever |B - t'| > 2^-14; each thread
// keeps the smallest |B - t'| of its 8 weights, and a thread with a value at
// or below 2^-14 (or a block whose 16 / absmax would not be a normal fp32)
// recomputes its 8 weights on the exact path: one IEEE division n = fp32(w /
// absmax) and the exact table {thr, lo}.  The exact path is taken by a warp
// only when one of its lanes needs it.  The host checks that no midpoint lies
// within 2^-17 of a cell edge (so a cell taken one off near an edge decides
// the same code) and otherwise disables the fast
// path.  The result always equals the exact-division code.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>
#include "ptx_sm100.cuh"

namespace qlora {

constexpr int kBlock = 64;     // first-level block
constexpr int kGroup = 256;    // second-level group (blocks per s2)
constexpr int kLutCells = 33;  // floor(16 n) + 16 for n in [-1, 1]
constexpr int kLutPad = 64;    // table entries in shared memory: any 6-bit index is in range
constexpr float kCellOffset = 15.875f;     // t = 16 n + 15.875
constexpr float kQuarterMagic = 3145728.f;  // 1.5 * 2^21: fp32 values in [2^21, 2^22) have ulp 1/4
// Guard of the fast path, in units of t.  With n = fp32(w / absmax), |w / absmax| <= 1,
// and the exact decision "n > mid" read as 16 n + 15.875 > T, T = 16 mid + 15.875:
//   |t' - (16 w/absmax + 15.875)| <= 16 * 2^-23 (rcp.approx, relative error <= 2^-23)
//                                    + 2^-20 (the fma's rounding: t' < 32, ulp <= 2^-19)
//   |16 n - 16 w/absmax|          <= 16 * 2^-25 = 2^-21 (the rounding of n)
//   so |t' - (16 n + 15.875)|     <  2^-18;
//   |B - T| <= 2^-20 (rounding T to fp32) + 15 * 2^-19 (the code in the 4 low mantissa
//   bits)  <  2^-15.
// If |B - t'| > 2^-14 > 2^-15 + 2^-18, B - t' and T - (16 n + 15.875) have the same sign, so
// the fast code is the exact one; the margin is about 1.8x.  fabsf(B - t') is exact where it
// is near 2^-14 (B and t' within a factor 2 of each other), so the test itself cannot err.
constexpr float kFastGuard = 6.103515625e-05f;  // 2^-14

// Host-built tables handed to the kernels by value.
struct Nf4Tables {
  float level[16];             // NF4 levels, ascending (fp32)
  float cell_thr[kLutCells];   // smallest fp32 above the cell's midpoint, or +inf
  int cell_lo[kLutCells];      // code of the cell's left edge
  uint32_t cell_fast[kLutCells];  // bits of fp32(16 mid + 15.875) (or 64.0f) with the low 4 bits = cell_lo
  int fast_ok;                 // the fast path's preconditions hold for this table
};

constexpr int kQuantThreads = 1024;  // 32 warps; 8 threads per 64-block
constexpr int kQuantStages = 3;      // shared-memory ring of groups
constexpr int kGroupFloats = kGroup * kBlock;                        // 16384
constexpr int kQuantPasses = kGroupFloats / 8 / kQuantThreads;       // 2 passes of 8 weights per thread

// Group i's absmax values are read until its second level runs (while the
// designated warps handle group i + kQuantStages); group i + 8 cannot start
// before every warp has finished group i + 8 - kQuantStages >= i + kQuantStages.
constexpr int kAbsmaxRing = 8;
static_assert(kAbsmaxRing >= 2 * kQuantStages, "absmax ring too short for the second-level lag");

struct QuantSmem {
  float stage[kQuantStages][kGroupFloats];   // 3 x 64 KiB, 128-byte aligned
  float absmax[kAbsmaxRing][kGroup];
  int2 exact[kLutPad];       // {threshold bits, left-edge code}
  uint32_t fast[kLutPad];
  uint64_t full[kQuantStages];
  uint32_t done[kQuantStages];     // warps that finished the stage, counted over all its uses
  uint32_t issued[kQuantStages];   // copies issued into the stage
  int abort_flag;
};

// Second stage of the quantizer.
enum QuantMode : int {
  kQuantSingle = 0,   // none: s2 receives the n_blocks fp32 absmax constants, q8 unused
  kQuantLinear8 = 1,  // q8 = min(255, rint(fp32(absmax / s2))), s2 = fp32(c2 / 255)
  kQuantFp8 = 2,      // q8 = E4M3(fp32(absmax / s)), s = fp32(c2 / 448), stored as s2 = -s
};

// {d0, d1} = {a0 * b + c, a1 * b + c}, two fp32 fmas in one instruction, each rounded on its own.
__device__ __forceinline__ void fma2_rn(float& d0, float& d1, float a0, float a1, float b, float c) {
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %4};\n\tmov.b64 rc, {%5, %5};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d0), "=f"(d1) : "f"(a0), "f"(a1), "f"(b), "f"(c));
}
// {d0, d1} = {a0 + b, a1 + b}, each rounded on its own.
__device__ __forceinline__ void add2_rn(float& d0, float& d1, float a0, float a1, float b) {
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %4};\n\t"
      "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d0), "=f"(d1) : "f"(a0), "f"(a1), "f"(b));
}

// Three-input fp32 max and min (exact, like a chain of two fmaxf / fminf).
__device__ __forceinline__ float max3f(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
__device__ __forceinline__ float min3f(float a, float b, float c) {
  float d;
  asm("min.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

__device__ __forceinline__ void bulk_load_g2s(void* smem_dst, const void* gsrc, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
               ::"r"(smem_u32(smem_dst)), "l"(gsrc), "r"(bytes), "r"(smem_u32(bar)) : "memory");
}

// Codes of the 8 weights f[0..7] of one block (block absmax am), packed with
// f[j] in bits 4j..4j+3.
__device__ __forceinline__ uint32_t nf4_code8(const float (&f)[8], float am, bool fast_table,
                                              const QuantSmem& sm) {
  // fast path needs 16 / absmax to be a normal fp32: absmax in [2^-120, 2^125]
  const bool fast = fast_table && am >= 7.52316385e-37f && am <= 4.2535296e37f;
  uint32_t packed = 0x88888888u;   // an all-zero block: every code is 8 (the level 0.0)
  bool need = !fast && am > 0.f;   // weights the fast path cannot decide
  if (fast) {
    float rcp;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(rcp) : "f"(am));   // am and 1/am are normal here
    const float r16 = 16.f * rcp;   // exact scaling
    float dmin = 1.f;
    uint32_t pair[4];   // byte j / 2: the codes of f[j] (low nibble) and f[j + 1]
#pragma unroll
    for (int j = 0; j < 8; j += 2) {
      float t[2], u[2];
      uint32_t x[2];
      fma2_rn(t[0], t[1], f[j], f[j + 1], r16, kCellOffset);
      add2_rn(u[0], u[1], t[0], t[1], kQuarterMagic);
      float d[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const uint32_t off = __float_as_uint(u[h]) & 0xFCu;
        const uint32_t ent = *reinterpret_cast<const uint32_t*>(reinterpret_cast<const char*>(sm.fast) + off);
        d[h] = __uint_as_float(ent) - t[h];
        // the code in the low 4 bits: the cell's left-edge code, plus one above its midpoint
        // (a cell whose left-edge code is 15 holds no midpoint, so the nibble never carries)
        x[h] = ent + (__float_as_uint(d[h]) >> 31);
      }
      dmin = min3f(dmin, fabsf(d[0]), fabsf(d[1]));
      pair[j / 2] = (x[1] << 4) + (x[0] & 15u);   // bits above 7 are dropped by the byte permutes
    }
    packed = __byte_perm(__byte_perm(pair[0], pair[1], 0x0040u), __byte_perm(pair[2], pair[3], 0x0040u), 0x5410u);
    need = dmin <= kFastGuard;
  }
  if (__any_sync(0xffffffffu, need)) {
    if (need) {
      // one IEEE fp32 division per weight, round to nearest (never the reciprocal form)
      packed = 0;
#pragma unroll
      for (int j = 7; j >= 0; --j) {
        const float wn = __fdiv_rn(f[j], am);
        const uint32_t off = __float_as_uint(__fadd_rn(__fmaf_rn(wn, 16.f, kCellOffset), kQuarterMagic)) & 0xFCu;
        const int2 ent = sm.exact[off >> 2];
        packed = (packed << 4) + static_cast<uint32_t>(ent.y) + (wn >= __int_as_float(ent.x) ? 1u : 0u);
      }
    }
  }
  return packed;
}

template <int kMode>
__global__ void __launch_bounds__(kQuantThreads, 1)
quantize_nf4_kernel(const float* __restrict__ W, int64_t n_blocks, int64_t groups, uint8_t* __restrict__ codes,
                    uint8_t* __restrict__ q8, float* __restrict__ s2, const Nf4Tables tabs) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  QuantSmem& sm = *reinterpret_cast<QuantSmem*>(smem_raw);
  const int tid = threadIdx.x;
  if (tid < kLutPad) {
    // index 63 is cell 0: the fast path's t' of a weight equal to -absmax may
    // round one quarter below 0; indices 33..62 repeat cell 32 (only NaN
    // input, a caller error, reaches them)
    const int c = tid < kLutCells ? tid : (tid == kLutPad - 1 ? 0 : kLutCells - 1);
    sm.exact[tid] = make_int2(__float_as_int(tabs.cell_thr[c]), tabs.cell_lo[c]);
    sm.fast[tid] = tabs.cell_fast[c];
  }
  if (tid == 0) {
    sm.abort_flag = 0;
    for (int s = 0; s < kQuantStages; ++s) {
      mbar_init(&sm.full[s], 1);
      sm.done[s] = 0;
      sm.issued[s] = 0;
    }
    fence_barrier_init();
  }
  __syncthreads();
  const bool fast_table = tabs.fast_ok != 0;
  const int64_t gstep = gridDim.x;
  auto group_blocks = [&](int64_t g) {
    const int64_t left = n_blocks - g * kGroup;
    return left < kGroup ? static_cast<int>(left) : kGroup;
  };
  auto issue = [&](int64_t g, int s) {
    const uint32_t bytes = static_cast<uint32_t>(group_blocks(g)) * kBlock * 4u;
    if (!QLORA_CHECK((bytes & 15u) == 0 && (reinterpret_cast<uintptr_t>(W + g * kGroupFloats) & 15u) == 0 &&
                         (smem_u32(sm.stage[s]) & 15u) == 0,
                     kDbgBulk, bytes))
      return;
    ++sm.issued[s];
    mbar_arrive_expect_tx(&sm.full[s], bytes);
    bulk_load_g2s(sm.stage[s], W + g * kGroupFloats, bytes, &sm.full[s]);
  };

  griddep_wait();   // the previous grid's writes are visible from here on
  if (tid == 0) {
    for (int s = 0; s < kQuantStages; ++s) {
      const int64_t g = blockIdx.x + s * gstep;
      if (g < groups) issue(g, s);
    }
  }
  __syncthreads();   // issued[] as thread 0 left it
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const int sub = lane & 7;        // 8 threads per 64-block
  const int swz = (lane >> 2) & 1; // which half of the 8 weights the first shared load takes
  constexpr uint32_t kWarps = kQuantThreads / 32;

  // Second level of the CTA's i-th group (group gg), on warps 8 (i mod 4) ..
  // 8 (i mod 4) + 7: c2 = max of the group's absmax, s2 = fp32(c2/255), q =
  // min(255, rint_half_even(fp32(absmax/s2))) (or the E4M3 form); a lane codes
  // one absmax value.
  auto second_level = [&](int64_t gg, int i) {
    const int nbb = group_blocks(gg);
    const float* amb = sm.absmax[i % kAbsmaxRing];
    float c2 = 0.f;
#pragma unroll
    for (int k = 0; k < kGroup / 32; ++k) {
      const int b = k * 32 + lane;
      c2 = fmaxf(c2, b < nbb ? amb[b] : 0.f);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) c2 = fmaxf(c2, __shfl_xor_sync(0xffffffffu, c2, o));
    const float sc = __fdiv_rn(c2, kMode == kQuantFp8 ? 448.f : 255.f);
    const int b = (warp & 7) * 32 + lane;
    if (b < nbb) {
      uint32_t q = 0;
      if (sc != 0.f) {
        const float ratio = __fdiv_rn(amb[b], sc);
        if (kMode == kQuantFp8) {
          uint16_t pr;   // round to nearest even, saturating at 448; both halves hold the same code
          asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(pr) : "f"(ratio), "f"(ratio));
          q = pr & 0xFFu;
        } else {
          q = static_cast<uint32_t>(min(255, __float2int_rn(ratio)));  // round half to even
        }
      }
      q8[gg * kGroup + b] = static_cast<uint8_t>(q);
    }
    // the FP8 form stores -s: the sign bit marks the group's format
    if (b == 0) s2[gg] = kMode == kQuantFp8 ? -sc : sc;
  };

  int it = 0;
  for (int64_t g = blockIdx.x; g < groups; g += gstep, ++it) {
    const int buf = it % kQuantStages;
    const int use = it / kQuantStages;   // earlier uses of this stage
    const int nb = group_blocks(g);
    float* amb = sm.absmax[it % kAbsmaxRing];
    if (!mbar_wait(&sm.full[buf], static_cast<uint32_t>(use) & 1u, &sm.abort_flag)) break;
    // group it arrived, so every warp has finished group it - kQuantStages
    if (kMode != kQuantSingle && it >= kQuantStages && (warp >> 3) == ((it - kQuantStages) & 3))
      second_level(g - kQuantStages * gstep, it - kQuantStages);
#pragma unroll
    for (int p = 0; p < kQuantPasses; ++p) {
      const int lb = p * (kQuantThreads / 8) + (tid >> 3);
      const float* src = sm.stage[buf] + lb * kBlock + sub * 8;
      const float4 a = *reinterpret_cast<const float4*>(src + 4 * swz);
      const float4 b = *reinterpret_cast<const float4*>(src + 4 * (swz ^ 1));
      const float f[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
      float am = max3f(max3f(fabsf(f[0]), fabsf(f[1]), fabsf(f[2])), max3f(fabsf(f[3]), fabsf(f[4]), fabsf(f[5])),
                       fmaxf(fabsf(f[6]), fabsf(f[7])));
      am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 1));
      am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 2));
      am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 4));
      if (lb >= nb) am = 0.f;   // past the end of the weight: the stage holds stale data
      uint32_t packed = nf4_code8(f, am, fast_table, sm);
      if (swz) packed = __funnelshift_l(packed, packed, 16);   // f[0..3] were weights 4..7
      if (lb < nb) {
        *reinterpret_cast<uint32_t*>(codes + ((g * kGroup + lb) * kBlock + sub * 8) / 2) = packed;
        if (sub == 0) {
          if (kMode != kQuantSingle) amb[lb] = am;
          else s2[g * kGroup + lb] = am;
        }
      }
    }
    // this warp is done with the stage and has written its absmax values; the
    // warp that completes the count refills the stage
    __syncwarp();
    if (lane == 0) {
      __threadfence_block();
      if (atomicAdd(&sm.done[buf], 1u) == kWarps * static_cast<uint32_t>(use + 1) - 1u) {
        __threadfence_block();
        if (g + kQuantStages * gstep < groups && !sm.abort_flag) issue(g + kQuantStages * gstep, buf);
      }
    }
  }
  __syncthreads();
  if (!sm.abort_flag) {
    // second level of the CTA's last kQuantStages groups (no later group proves them finished)
    if (kMode != kQuantSingle) {
      for (int i = it > kQuantStages ? it - kQuantStages : 0; i < it; ++i)
        if ((warp >> 3) == (i & 3)) second_level(blockIdx.x + static_cast<int64_t>(i) * gstep, i);
    }
  } else if (tid == 0) {
    // a copy did not complete in time: wait (bounded) for the ones still in flight before exiting
    int none = 0;
    for (int s = 0; s < kQuantStages; ++s)
      if (sm.issued[s] > 0) mbar_wait(&sm.full[s], (sm.issued[s] - 1u) & 1u, &none);
  }
  griddep_launch_dependents();
}

// Dense dequantization: w = fp32(level[code] * c1), c1 the block scale in any
// of its stored forms (block_scale), fp32 or bf16 out.  One thread per 8
// consecutive weights (4 packed bytes).
template <bool kBf16>
__global__ void __launch_bounds__(256)
dequant_kernel(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ q8,
               const float* __restrict__ s2, int64_t n_oct, void* __restrict__ out,
               const Nf4Tables tabs) {
  __shared__ float s_level[16];
  if (threadIdx.x < 16) s_level[threadIdx.x] = tabs.level[threadIdx.x];
  __syncthreads();
  griddep_wait();
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n_oct;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const uint32_t p = __ldg(reinterpret_cast<const uint32_t*>(codes) + i);
    const int64_t blk = (i * 8) / kBlock;
    const float c1 = block_scale(q8, s2, blk);
    float w[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) w[j] = __fmul_rn(s_level[(p >> (4 * j)) & 15u], c1);
    if (kBf16) {
      uint4 o;
      __nv_bfloat162 h0 = __floats2bfloat162_rn(w[0], w[1]);
      __nv_bfloat162 h1 = __floats2bfloat162_rn(w[2], w[3]);
      __nv_bfloat162 h2 = __floats2bfloat162_rn(w[4], w[5]);
      __nv_bfloat162 h3 = __floats2bfloat162_rn(w[6], w[7]);
      o.x = *reinterpret_cast<uint32_t*>(&h0);
      o.y = *reinterpret_cast<uint32_t*>(&h1);
      o.z = *reinterpret_cast<uint32_t*>(&h2);
      o.w = *reinterpret_cast<uint32_t*>(&h3);
      reinterpret_cast<uint4*>(out)[i] = o;
    } else {
      float4* o = reinterpret_cast<float4*>(out) + 2 * i;
      o[0] = make_float4(w[0], w[1], w[2], w[3]);
      o[1] = make_float4(w[4], w[5], w[6], w[7]);
    }
  }
}

}  // namespace qlora
