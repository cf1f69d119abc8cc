// LoRA dropout on the adapter input, sm_100a.
//
// The PEFT LoraConfig of "QLoRAの理論と実装" (lora_dropout=0.05) puts dropout on
// the adapter's input only: the adapter sees x * keep / (1 - p), the frozen
// NF4 path sees x.  The keep decision of element e (row-major index m*K + k
// of X) is the 16-bit half (e & 1) (the low half first) of word
// ((e >> 1) & 3) of Philox4x32-10 at counter (lo32(e >> 3), hi32(e >> 3),
// lo32(offset), hi32(offset)) under key (lo32(seed), hi32(seed)); the
// element is kept when that half is >= t = floor(p * 2^16).  One block thus
// decides 8 elements, and the two elements of a bf16 pair read the two
// halves of one word.  Philox4x32-10 is the counter-based generator of
// Salmon, Moraes, Dror and Shaw ("Parallel Random Numbers: As Easy as 1, 2,
// 3", SC'11), written here from that definition.
//
// The masks are applied where the adapter consumes x:
//   dropout_mask_kernel   X_keep = X * keep (bf16, exact), the input of U = X_keep A^T
//                         and dA = V^T X_keep (their 1/(1-p) goes into the scales);
//   dX += s/(1-p) * (V A) * keep, the adapter's share of dX, after the fused
//                         kernel wrote dY dequant(W) alone: the masked-add epilogue
//                         of the tensor-core GEMM V A (gemm_tc.cuh, kOutDropoutAdd),
//                         which reads the keep bits the backward's mask kernel wrote.
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

// The four words deciding elements 8q .. 8q+7 (two per word, the low half first).
__device__ __forceinline__ uint4 dropout_words(uint64_t q, uint64_t seed, uint64_t offset) {
  return philox4x32_10(make_uint4(static_cast<uint32_t>(q), static_cast<uint32_t>(q >> 32),
                                  static_cast<uint32_t>(offset), static_cast<uint32_t>(offset >> 32)),
                       make_uint2(static_cast<uint32_t>(seed), static_cast<uint32_t>(seed >> 32)));
}

// out = X with every dropped element replaced by +0 (bf16 bit patterns).  A
// thread takes 16 consecutive elements (32 bytes, two Philox blocks) per
// step; its loads are issued before the generator runs, so they are in
// flight meanwhile.  Word m of the pair of blocks decides the bf16 pair in
// data word m, one 16-bit half each, so one per-halfword compare against
// t2 = t | t << 16 gives that data word's mask.  n16 = M*K/16 (M*K is a
// multiple of 64).  If `bits` is not NULL, bit j of bits[q] is the keep
// decision of element 16 q + j (M*K/8 bytes), for consumers that apply the
// same mask later without regenerating it.
__global__ void __launch_bounds__(256)
dropout_mask_kernel(const uint16_t* __restrict__ X, int64_t n16, uint32_t t, uint64_t seed, uint64_t offset,
                    uint16_t* __restrict__ out, uint16_t* __restrict__ bits) {
  const uint32_t t2 = t | (t << 16);   // t <= 0xFFFF
  griddep_wait();
  for (int64_t q = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; q < n16;
       q += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const uint4* src = reinterpret_cast<const uint4*>(X) + 2 * q;
    const uint4 x0 = __ldg(src), x1 = __ldg(src + 1);
    const uint4 w0 = dropout_words(static_cast<uint64_t>(2 * q), seed, offset);
    const uint4 w1 = dropout_words(static_cast<uint64_t>(2 * q + 1), seed, offset);
    const uint32_t rnd[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
    uint32_t v[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
    uint32_t k = 0;
#pragma unroll
    for (int m = 0; m < 8; ++m) {
      const uint32_t keep = __vcmpgeu2(rnd[m], t2);   // 0xFFFF in each kept half
      v[m] &= keep;
      k |= ((keep & 1u) | ((keep >> 15) & 2u)) << (2 * m);
    }
    uint4* dst = reinterpret_cast<uint4*>(out) + 2 * q;
    dst[0] = make_uint4(v[0], v[1], v[2], v[3]);
    dst[1] = make_uint4(v[4], v[5], v[6], v[7]);
    if (bits) bits[q] = static_cast<uint16_t>(k);
  }
  griddep_launch_dependents();
}

}  // namespace qlora
