// LoRA dropout on the adapter input, sm_100a.
//
// The PEFT LoraConfig of "QLoRAの理論と実装" (lora_dropout=0.05) puts dropout on
// the adapter's input only: the adapter sees x * keep / (1 - p), the frozen
// NF4 path sees x.  The keep decision of element e (row-major index m*K + k
// of X) is word (e & 3) of Philox4x32-10 at counter (lo32(e >> 2),
// hi32(e >> 2), lo32(offset), hi32(offset)) under key (lo32(seed),
// hi32(seed)); the element is kept when that word is >= t = floor(p * 2^32).
// Philox4x32-10 is the counter-based generator of Salmon, Moraes, Dror and
// Shaw ("Parallel Random Numbers: As Easy as 1, 2, 3", SC'11), written here
// from that definition.
//
// The masks are applied where the adapter consumes x:
//   dropout_mask_kernel   X_keep = X * keep (bf16, exact), the input of U = X_keep A^T
//                         and dA = V^T X_keep (their 1/(1-p) goes into the scales);
//   dropout_dx_kernel     dX += s/(1-p) * (V A) * keep, the adapter's share of dX,
//                         after the fused kernel wrote dY dequant(W) alone.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>
#include "ptx_sm100.cuh"

namespace qlora {

__device__ __forceinline__ uint4 philox4x32_10(uint4 c, uint2 k) {
#pragma unroll
  for (int round = 0; round < 10; ++round) {
    const uint32_t hi0 = __umulhi(0xD2511F53u, c.x), lo0 = 0xD2511F53u * c.x;
    const uint32_t hi1 = __umulhi(0xCD9E8D57u, c.z), lo1 = 0xCD9E8D57u * c.z;
    c = make_uint4(hi1 ^ c.y ^ k.x, lo1, hi0 ^ c.w ^ k.y, lo0);
    k.x += 0x9E3779B9u;
    k.y += 0xBB67AE85u;
  }
  return c;
}

// The four words deciding elements 4q .. 4q+3.
__device__ __forceinline__ uint4 dropout_words(uint64_t q, uint64_t seed, uint64_t offset) {
  return philox4x32_10(make_uint4(static_cast<uint32_t>(q), static_cast<uint32_t>(q >> 32),
                                  static_cast<uint32_t>(offset), static_cast<uint32_t>(offset >> 32)),
                       make_uint2(static_cast<uint32_t>(seed), static_cast<uint32_t>(seed >> 32)));
}

// out = X with every dropped element replaced by +0 (bf16 bit patterns); four
// elements (8 bytes, one Philox block) per thread and step.  n4 = M*K/4.
__global__ void __launch_bounds__(256)
dropout_mask_kernel(const uint16_t* __restrict__ X, int64_t n4, uint32_t t, uint64_t seed, uint64_t offset,
                    uint16_t* __restrict__ out) {
  griddep_wait();
  for (int64_t q = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; q < n4;
       q += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const uint4 w = dropout_words(static_cast<uint64_t>(q), seed, offset);
    uint2 x = __ldg(reinterpret_cast<const uint2*>(X) + q);
    // element 4q is the low half of the first word
    if (w.x < t) x.x &= 0xFFFF0000u;
    if (w.y < t) x.x &= 0x0000FFFFu;
    if (w.z < t) x.y &= 0xFFFF0000u;
    if (w.w < t) x.y &= 0x0000FFFFu;
    reinterpret_cast<uint2*>(out)[q] = x;
  }
  griddep_launch_dependents();
}

constexpr int kDxRows = 8;      // rows of dX per thread
constexpr int kDxThreads = 256; // a thread owns 4 consecutive columns: 1024 columns per CTA

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// dX[m, k] = bf16(fp32(dX[m, k]) + scale * sum_j V[m, j] A[j, k]) where element
// (m, k) is kept; dX unchanged where it was dropped.  V: bf16 M x r, A: bf16
// r x K.  Shared memory: the CTA's kDxRows rows of V as fp32.
__global__ void __launch_bounds__(kDxThreads)
dropout_dx_kernel(uint16_t* __restrict__ dX, const uint16_t* __restrict__ V, const uint16_t* __restrict__ A,
                  int64_t M, int64_t K, int r, float scale, uint32_t t, uint64_t seed, uint64_t offset) {
  extern __shared__ float s_v[];
  const int64_t m0 = static_cast<int64_t>(blockIdx.y) * kDxRows;
  const int64_t k0 = (static_cast<int64_t>(blockIdx.x) * kDxThreads + threadIdx.x) * 4;
  griddep_wait();
  for (int i = threadIdx.x; i < kDxRows * r; i += kDxThreads) {
    const int rr = i / r, j = i - rr * r;
    s_v[i] = (m0 + rr < M) ? __uint_as_float(static_cast<uint32_t>(__ldg(V + (m0 + rr) * r + j)) << 16) : 0.f;
  }
  __syncthreads();
  griddep_launch_dependents();
  if (k0 >= K) return;
  float acc[kDxRows][4];
#pragma unroll
  for (int rr = 0; rr < kDxRows; ++rr) acc[rr][0] = acc[rr][1] = acc[rr][2] = acc[rr][3] = 0.f;
  for (int j = 0; j < r; ++j) {
    const uint2 a = __ldg(reinterpret_cast<const uint2*>(A + static_cast<int64_t>(j) * K + k0));
    const float a0 = bf16_lo(a.x), a1 = bf16_hi(a.x), a2 = bf16_lo(a.y), a3 = bf16_hi(a.y);
#pragma unroll
    for (int rr = 0; rr < kDxRows; ++rr) {
      const float v = s_v[rr * r + j];
      acc[rr][0] = fmaf(v, a0, acc[rr][0]);
      acc[rr][1] = fmaf(v, a1, acc[rr][1]);
      acc[rr][2] = fmaf(v, a2, acc[rr][2]);
      acc[rr][3] = fmaf(v, a3, acc[rr][3]);
    }
  }
#pragma unroll
  for (int rr = 0; rr < kDxRows; ++rr) {
    const int64_t m = m0 + rr;
    if (m >= M) break;
    const int64_t e = m * K + k0;   // a multiple of 4: one Philox block
    const uint4 w = dropout_words(static_cast<uint64_t>(e >> 2), seed, offset);
    uint2* p = reinterpret_cast<uint2*>(dX + e);
    uint2 d = *p;
    const float o0 = w.x >= t ? bf16_lo(d.x) + scale * acc[rr][0] : bf16_lo(d.x);
    const float o1 = w.y >= t ? bf16_hi(d.x) + scale * acc[rr][1] : bf16_hi(d.x);
    const float o2 = w.z >= t ? bf16_lo(d.y) + scale * acc[rr][2] : bf16_lo(d.y);
    const float o3 = w.w >= t ? bf16_hi(d.y) + scale * acc[rr][3] : bf16_hi(d.y);
    __nv_bfloat162 h0 = __floats2bfloat162_rn(o0, o1), h1 = __floats2bfloat162_rn(o2, o3);
    d.x = *reinterpret_cast<uint32_t*>(&h0);
    d.y = *reinterpret_cast<uint32_t*>(&h1);
    *p = d;
  }
}

}  // namespace qlora
