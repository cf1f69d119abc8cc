// Adapter merge into the 16-bit base, for distribution, sm_100a.
//
// "QLoRAとは？4bit量子化＋LoRAの仕組み・VRAM目安・実装手順と採用判断を解説",
// section on merging a trained adapter: merging onto the 4-bit base rounds
// the adapter's small differences onto the 4-bit grid, so the adapter is
// folded into the unquantized base loaded in bf16, and that merged 16-bit
// weight is what gets quantized again (qlora_quantize_nf4_dq or
// qlora_quantize_nf4 on this kernel's fp32 output).
//
//   merged[n, k] = bf16( fp64(bf16(W[n, k])) + fp64(s) * sum_j B[n, j] A[j, k] )
//
// The sum runs in fp64 in the order j = 0, 1, ..., r-1, every product and
// every addition rounded on its own (a product of two bf16 values is exact
// in fp64), and the result is rounded to bf16 once, straight from fp64.  The
// explicit __dmul_rn / __dadd_rn keep the compiler from fusing them.
//
// A CTA covers kMergeRows rows x 256 columns; a thread owns one column and
// keeps one fp64 accumulator per row.  The tile's rows of B sit in shared
// memory as fp64 (every thread reads the same element: a broadcast); A is
// read once per CTA with coalesced loads.  The kernel is bound by fp64
// issue (two instructions per term), not by its 4 + 4 bytes of traffic per
// weight.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>
#include "ptx_sm100.cuh"

namespace qlora {

constexpr int kMergeRows = 16;
constexpr int kMergeCols = 256;   // = threads per CTA

__device__ __forceinline__ double bf16_bits_to_f64(uint16_t b) {
  return static_cast<double>(__uint_as_float(static_cast<uint32_t>(b) << 16));
}

// fp64 -> bf16 bits, round to nearest even, one rounding.
__device__ __forceinline__ uint16_t f64_to_bf16_bits(double x) {
  uint16_t b;
  asm("cvt.rn.bf16.f64 %0, %1;" : "=h"(b) : "d"(x));
  return b;
}

// Shared memory: B rows of the tile as fp64, kMergeRows x r.
template <bool kBf16Out>
__global__ void __launch_bounds__(kMergeCols)
merge_adapter_kernel(const float* __restrict__ W, int64_t n_rows, int64_t k_cols, const uint16_t* __restrict__ A,
                     const uint16_t* __restrict__ B, int r, double s, void* __restrict__ out) {
  extern __shared__ double s_b[];
  const int64_t n0 = static_cast<int64_t>(blockIdx.y) * kMergeRows;
  const int64_t k = static_cast<int64_t>(blockIdx.x) * kMergeCols + threadIdx.x;
  const int64_t left = n_rows - n0;
  const int rows = left < kMergeRows ? static_cast<int>(left) : kMergeRows;
  griddep_wait();
  for (int i = threadIdx.x; i < kMergeRows * r; i += kMergeCols) {
    const int n = i / r, j = i - n * r;
    s_b[i] = n < rows ? bf16_bits_to_f64(__ldg(B + (n0 + n) * r + j)) : 0.0;
  }
  __syncthreads();
  griddep_launch_dependents();
  if (k >= k_cols) return;
  double acc[kMergeRows];
#pragma unroll
  for (int n = 0; n < kMergeRows; ++n) acc[n] = 0.0;
  for (int j = 0; j < r; ++j) {
    const double a = bf16_bits_to_f64(__ldg(A + static_cast<int64_t>(j) * k_cols + k));
#pragma unroll
    for (int n = 0; n < kMergeRows; ++n) acc[n] = __dadd_rn(acc[n], __dmul_rn(s_b[n * r + j], a));
  }
#pragma unroll
  for (int n = 0; n < kMergeRows; ++n) {
    if (n >= rows) break;
    const int64_t idx = (n0 + n) * k_cols + k;
    const double w16 = static_cast<double>(__bfloat162float(__float2bfloat16_rn(__ldg(W + idx))));
    const uint16_t m = f64_to_bf16_bits(__dadd_rn(w16, __dmul_rn(s, acc[n])));
    if (kBf16Out) static_cast<uint16_t*>(out)[idx] = m;
    else static_cast<float*>(out)[idx] = __uint_as_float(static_cast<uint32_t>(m) << 16);
  }
}

}  // namespace qlora
