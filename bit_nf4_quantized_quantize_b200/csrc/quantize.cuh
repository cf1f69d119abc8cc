// NF4 quantization with double quantization, and dequantization, for sm_100a.
//
// "QLoRAの理論と実装" §5-1 (absmax per 64-block, w/absmax, nearest of the 16
// NormalFloat levels, 4-bit code) and §5-2 (8-bit re-quantization of the fp32
// absmax constants in groups of 256, one fp32 second-level constant; without
// that second stage the fp32 absmax constants are stored as they are).
//
// quantize_nf4_kernel<kMode>: one CTA of 512 threads per group of 256 blocks (16384
// weights, 64 KiB of fp32 input).  Eight threads share a 64-block (8
// consecutive weights each, two 16-byte loads), so a warp reads 1 KiB
// contiguous per pass; the block absmax is a 3-step xor-shuffle max.  The
// group's 256 absmax values then stay in shared memory for the second-level
// quantization, so the fp32 constants never go to HBM.  Traffic per weight:
// 4 B read, 0.5 + 1/64 + 4/16384 B written with a second stage, or 0.5 + 4/64
// B written when the second stage is off and the absmax constants are stored.
//
// Nearest level.  The code of n = fp32(w / absmax) is #{i : n >= thr_i}, thr_i
// the smallest fp32 above the exact midpoint of levels i and i+1.  Cells of
// width 1/16 over [-1, 1] hold at most one threshold each (the thresholds are
// >= 0.088 apart), so code = lo[cell] + (n >= thr[cell]) with cell =
// floor(16 n) + 16.  The cell comes from the float adder rather than a
// conversion: u = fp32(fp32(16 n + 15.5) + 1.5 * 2^23) lies in the binade of
// ulp 1, whose low 6 mantissa bits are then RN(16 n + 15.5) = floor(16 n + 16)
// away from the cell edges; within 2^-17 of an edge the cell may be the left
// or right neighbour, which decides the same code because no threshold lies
// within 2^-17 of an edge (the host checks this).  Fast path: q0 = fp32(w * fp32(1/absmax)) is within 2.5
// ulp of n, so every threshold that is not within 2^-18 of q0 lies on the
// same side of q0 and n; the fast table packs the cell's left-edge code into
// the 4 low mantissa bits of its threshold (a perturbation below 2^-19) and
// one 4-byte shared-memory load serves the lookup.  When q0 is within 2^-18 of
// the cell's threshold, or absmax is outside [2^-125, 2^125], the weight takes
// the exact path: one IEEE division and the exact table.  The host checks
// that no threshold lies within 2^-17 of a cell edge and otherwise disables
// the fast path.  The result always equals the exact-division code.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>
#include "ptx_sm100.cuh"

namespace qlora {

constexpr int kBlock = 64;     // first-level block
constexpr int kGroup = 256;    // second-level group (blocks per s2)
constexpr int kLutCells = 33;  // floor(16 n) + 16 for n in [-1, 1]
constexpr int kLutPad = 64;    // table entries in shared memory: any 6-bit index is in range
constexpr float kFastGuard = 3.814697265625e-06f;  // 2^-18

// Host-built tables handed to the kernels by value.
struct Nf4Tables {
  float level[16];             // NF4 levels, ascending (fp32)
  float cell_thr[kLutCells];   // exact threshold inside the cell, or +inf
  int cell_lo[kLutCells];      // code of the cell's left edge
  uint32_t cell_fast[kLutCells];  // threshold bits (or 4.0f) with the low 4 bits = cell_lo
  int fast_ok;                 // the fast path's preconditions hold for this table
};

constexpr int kQuantThreads = 512;  // 16 warps; 8 threads per 64-block, 4 passes of 64 blocks

// Second stage of the quantizer.
enum QuantMode : int {
  kQuantSingle = 0,   // none: s2 receives the n_blocks fp32 absmax constants, q8 unused
  kQuantLinear8 = 1,  // q8 = min(255, rint(fp32(absmax / s2))), s2 = fp32(c2 / 255)
  kQuantFp8 = 2,      // q8 = E4M3(fp32(absmax / s)), s = fp32(c2 / 448), stored as s2 = -s
};
template <int kMode>
__global__ void __launch_bounds__(kQuantThreads, 2)
quantize_nf4_kernel(const float* __restrict__ W, int64_t n_blocks, uint8_t* __restrict__ codes,
                    uint8_t* __restrict__ q8, float* __restrict__ s2, const Nf4Tables tabs) {
  __shared__ int2 s_exact[kLutPad];     // {threshold bits, left-edge code}
  __shared__ uint32_t s_fast[kLutPad];
  __shared__ float s_absmax[kGroup];
  __shared__ float s_warpmax[kGroup / 32];

  const int tid = threadIdx.x;
  if (tid < kLutPad) {
    // entries past the last cell repeat it (only NaN input, a caller error, reaches them)
    const int c = tid < kLutCells ? tid : kLutCells - 1;
    s_exact[tid] = make_int2(__float_as_int(tabs.cell_thr[c]), tabs.cell_lo[c]);
    s_fast[tid] = tabs.cell_fast[c];
  }
  const bool fast_table = tabs.fast_ok != 0;

  const int64_t g = blockIdx.x;
  const int64_t b_first = g * kGroup;
  const int64_t left = n_blocks - b_first;
  const int nb = left < kGroup ? static_cast<int>(left) : kGroup;
  const int sub = tid & 7;     // 8 threads per 64-block
  const int lb0 = tid >> 3;    // block within a pass (64 blocks per pass)
  constexpr int kPasses = kGroup / (kQuantThreads / 8);

  griddep_wait();   // the previous grid's writes are visible from here on
  // Issue every load of the thread up front (8 x 16 B in flight per thread).
  float4 v[kPasses][2];
#pragma unroll
  for (int p = 0; p < kPasses; ++p) {
    const int lb = p * (kQuantThreads / 8) + lb0;
    if (lb < nb) {
      const float4* src = reinterpret_cast<const float4*>(W + (b_first + lb) * kBlock + sub * 8);
      v[p][0] = __ldcs(src);
      v[p][1] = __ldcs(src + 1);
    } else {
      v[p][0] = make_float4(0.f, 0.f, 0.f, 0.f);
      v[p][1] = v[p][0];
    }
  }
  __syncthreads();  // lookup table ready

#pragma unroll
  for (int p = 0; p < kPasses; ++p) {
    const int lb = p * (kQuantThreads / 8) + lb0;
    const float e[8] = {v[p][0].x, v[p][0].y, v[p][0].z, v[p][0].w,
                        v[p][1].x, v[p][1].y, v[p][1].z, v[p][1].w};
    float am = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j) am = fmaxf(am, fabsf(e[j]));
    am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 1));
    am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 2));
    am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 4));
    // every lane takes part (the warp-wide vote below); blocks past the end hold
    // zeros and are not stored
    // fast path needs fp32(1/absmax) to be a normal number
    const bool fast = fast_table && am >= 2.35098870e-38f * 4.0f && am <= 4.2535296e37f;
    uint32_t packed = 0x88888888u;   // an all-zero block: every code is 8 (the level 0.0)
    uint32_t slow = 0;               // weights the fast path cannot decide
    if (fast) {
      const float rcp = __frcp_rn(am);
      packed = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float q0 = __fmul_rn(e[j], rcp);
        const uint32_t cell = __float_as_uint(__fadd_rn(__fmaf_rn(q0, 16.f, 15.5f), 12582912.f)) & 63u;
        const uint32_t ent = s_fast[cell];
        const float thr = __uint_as_float(ent);
        packed |= ((ent & 15u) + (q0 >= thr ? 1u : 0u)) << (4 * j);
        slow |= (fabsf(q0 - thr) <= kFastGuard ? 1u : 0u) << j;
      }
    } else if (am > 0.f) {
      slow = 0xFFu;
    }
    if (__any_sync(0xffffffffu, slow != 0u)) {
      // one IEEE fp32 division per undecided weight, round to nearest (never the reciprocal form)
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if ((slow >> j) & 1u) {
          const float wn = __fdiv_rn(e[j], am);
          const uint32_t cell = __float_as_uint(__fadd_rn(__fmaf_rn(wn, 16.f, 15.5f), 12582912.f)) & 63u;
          const int2 ent = s_exact[cell];
          const uint32_t code = static_cast<uint32_t>(ent.y) + (wn >= __int_as_float(ent.x) ? 1u : 0u);
          packed = (packed & ~(15u << (4 * j))) | (code << (4 * j));
        }
      }
    }
    if (lb < nb) {
      *reinterpret_cast<uint32_t*>(codes + ((b_first + lb) * kBlock + sub * 8) / 2) = packed;
      if (sub == 0) {
        if (kMode != kQuantSingle) s_absmax[lb] = am;
        else s2[b_first + lb] = am;
      }
    }
  }
  griddep_launch_dependents();
  if (kMode == kQuantSingle) return;
  __syncthreads();

  // Second level: c2 = max of the group's absmax, s2 = fp32(c2/255),
  // q = min(255, rint_half_even(fp32(absmax/s2))).  Threads 0..255 own one
  // absmax each (warps 0..7).
  if (tid < kGroup) {
    const float my = tid < nb ? s_absmax[tid] : 0.f;
    float m = my;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if ((tid & 31) == 0) s_warpmax[tid >> 5] = m;
  }
  __syncthreads();
  if (tid < kGroup) {
    float c2 = s_warpmax[0];
#pragma unroll
    for (int w = 1; w < kGroup / 32; ++w) c2 = fmaxf(c2, s_warpmax[w]);
    const float sc = __fdiv_rn(c2, kMode == kQuantFp8 ? 448.f : 255.f);
    if (tid < nb) {
      uint32_t q = 0;
      if (sc != 0.f) {
        const float ratio = __fdiv_rn(s_absmax[tid], sc);
        if (kMode == kQuantFp8) {
          uint16_t pr;   // round to nearest even, saturating at 448; both halves hold the same code
          asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(pr) : "f"(ratio), "f"(ratio));
          q = pr & 0xFFu;
        } else {
          q = static_cast<uint32_t>(min(255, __float2int_rn(ratio)));  // round half to even
        }
      }
      q8[b_first + tid] = static_cast<uint8_t>(q);
    }
    // the FP8 form stores -s: the sign bit marks the group's format
    if (tid == 0) s2[g] = kMode == kQuantFp8 ? -sc : sc;
  }
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
