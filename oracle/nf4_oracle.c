/*
 * CPU oracle for the QLoRA NF4 + double-quantization linear layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library links, loads or
 * calls this file; only the test suite, the package's smoke check and the
 * bench's CPU-baseline / reference arm do.  It shares no code, header, table or
 * constant with the CUDA path: the NF4 table is derived here from its quantile
 * definition with this file's own inverse normal CDF.
 *
 * Every step is written to be read against the pages:
 *   [p1] "QLoRAの理論と実装" (disassemble-channel.com)
 *   [p2] Qiita article on why QLoRA survives 4-bit (TaiyoYamada)
 *   [p4] "QLoRAとは？4bit量子化＋LoRAの仕組み・VRAM目安・実装手順と採用判断を解説"
 *        (issoh.co.jp)
 * Quantisation follows the algorithm's steps in order (it is an encoding, so
 * there is no shorter closed form); the linear layer is the plain definition
 * evaluated in fp64 on the exact bf16 operands.
 *
 * Readings of points the pages leave open (all listed in the design notes):
 *   - codebook: the p1 listing "create_nf4_codebook" (quantiles i/18, i=1..8 on
 *     the negative side, j/16, j=9..15 on the positive side, zero pinned,
 *     divided by the largest magnitude), because the p1 §5-1 formula with
 *     i/(2^b+1), i=0 gives Phi^-1(0) = -inf;
 *   - nearest code: exact argmin over the 16 levels, the lowest index winning
 *     a tie (numpy argmin, p1 listing "quantize_nf4");
 *   - w/absmax is one IEEE fp32 division;
 *   - an all-zero block gets absmax 0 and code 8 (the level 0.0);
 *   - nibble order: element 2j in the low nibble of byte j, row-major flatten;
 *   - double quantization: linear unsigned 8-bit absmax quantization of each
 *     group of 256 fp32 absmax constants, s2 = fp32(c2/255),
 *     q = min(255, round-half-even(fp32(absmax/s2))), s2 == 0 gives q = 0;
 *   - dequant: w = bf16( fp32( c[code] * fp32(q * s2) ) );
 *   - single quantization (second stage off): w = bf16( fp32( c[code] * absmax ) );
 *   - FP8 reading of the second stage ("8bit量子化（FP8相当）"): s2 = fp32(c2/448),
 *     q = E4M3(fp32(absmax/s2)) rounded to nearest even and saturated at 448,
 *     stored with the sign bit of s2 set to mark the group's format;
 *   - adapter merge: into the 16-bit base, not the 4-bit one (p4), as one
 *     rounding of the fp64 value bf16(W) + s * sum_j B[n,j] A[j,k].
 *
 * Build: gcc -O2 -fopenmp -ffp-contract=off -fno-fast-math -shared -fPIC.
 * fp-contract is off so that no multiply-add is fused: every fp32 operation
 * below rounds once, as written.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>
#include <stdlib.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_BLOCK 64   /* first-level block, p1 §5-1 step 1 and §5-2 */
#define ORACLE_GROUP 256  /* second-level block of absmax constants, p1 §5-2 */

int oracle_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ------------------------------------------------------------------------ */
/* Standard normal CDF and its inverse.                                      */
/* Phi(x) = erfc(-x/sqrt(2)) / 2 and its upper tail 1 - Phi(x) =             */
/* erfc(x/sqrt(2)) / 2 (textbook identities).  The inverse is found by       */
/* bisection until the bracket is two adjacent doubles.  For p > 1/2 the     */
/* upper tail is matched against 1 - p (exact for such p), so that no        */
/* precision is lost to 1 - tiny.                                            */
/* ------------------------------------------------------------------------ */
static double oracle_phi(double x) { return 0.5 * erfc(-x / sqrt(2.0)); }
static double oracle_phi_upper(double x) { return 0.5 * erfc(x / sqrt(2.0)); }

double oracle_norm_ppf(double p) {
    if (!(p > 0.0 && p < 1.0)) return NAN;
    int upper = p > 0.5;
    double target = upper ? 1.0 - p : p;
    double lo = -40.0, hi = 40.0;
    for (int it = 0; it < 4000; ++it) {
        double mid = 0.5 * (lo + hi);
        if (mid <= lo || mid >= hi) break;  /* adjacent doubles */
        /* both branches move lo up while mid is below the quantile */
        int below = upper ? (oracle_phi_upper(mid) > target) : (oracle_phi(mid) < target);
        if (below) lo = mid; else hi = mid;
    }
    double elo = upper ? fabs(oracle_phi_upper(lo) - target) : fabs(oracle_phi(lo) - target);
    double ehi = upper ? fabs(oracle_phi_upper(hi) - target) : fabs(oracle_phi(hi) - target);
    return (elo < ehi) ? lo : hi;
}

/* ------------------------------------------------------------------------ */
/* NF4 codebook.  [p1] "NF4量子化の仕組みの実装（教育目的）", listing         */
/* create_nf4_codebook: eight negative levels at the quantiles i/18,        */
/* i = 1..8, the level 0, seven positive levels at the quantiles j/16,      */
/* j = 9..15; all divided by the largest magnitude; sorted ascending.       */
/* This matches the "8 negative, 7 positive, zero pinned" statement of      */
/* p1 §5-1 "数学的な構成".  out64 gets the fp64 levels, out32 their fp32     */
/* rounding (the table the quantizer uses).                                  */
/* ------------------------------------------------------------------------ */
void oracle_nf4_codebook(double out64[16], float out32[16]) {
    double v[16];
    int n = 0;
    for (int i = 1; i <= 8; ++i) v[n++] = oracle_norm_ppf((double)i / 18.0);
    v[n++] = 0.0;
    for (int j = 9; j <= 15; ++j) v[n++] = oracle_norm_ppf((double)j / 16.0);
    double mx = 0.0;
    for (int i = 0; i < 16; ++i) if (fabs(v[i]) > mx) mx = fabs(v[i]);
    for (int i = 0; i < 16; ++i) v[i] = v[i] / mx;
    /* insertion sort, ascending (the values are already ascending) */
    for (int i = 1; i < 16; ++i) {
        double t = v[i]; int j = i - 1;
        while (j >= 0 && v[j] > t) { v[j + 1] = v[j]; --j; }
        v[j + 1] = t;
    }
    for (int i = 0; i < 16; ++i) { out64[i] = v[i]; out32[i] = (float)v[i]; }
}

/* ------------------------------------------------------------------------ */
/* Nearest level.  [p1] §5-1 step 2: i* = argmin_i |w_norm - c_i|.  The     */
/* distances are formed in fp64 from the fp32 operands; near any tie the     */
/* two operands are within a factor 2^28 of each other (or one is 0), so the */
/* differences are exact there and the comparison is the exact-real one.     */
/* Strict '<' keeps the lowest index on a tie, as numpy's argmin does.      */
/* ------------------------------------------------------------------------ */
int oracle_nearest_code(float wn, const float table[16]) {
    int best = 0;
    double bd = fabs((double)wn - (double)table[0]);
    for (int i = 1; i < 16; ++i) {
        double d = fabs((double)wn - (double)table[i]);
        if (d < bd) { bd = d; best = i; }
    }
    return best;
}

/* ------------------------------------------------------------------------ */
/* Blockwise NF4 quantization, [p1] §5-1 steps 1-2 and the listing          */
/* quantize_nf4 (semantics only): per block of 64 consecutive row-major     */
/* elements, absmax = max |w| (exact); absmax == 0 leaves the block at 0;   */
/* else w_norm = fp32(w / absmax) and the nearest level's index is stored   */
/* in 4 bits.  n must be a multiple of 64 (every K is; the listing's zero    */
/* padding of a ragged tail is therefore never exercised).                   */
/* codes: n/2 bytes, absmax: n/64 floats.  Returns 0, or -1 on a bad n.     */
/* ------------------------------------------------------------------------ */
int oracle_quantize_nf4(const float* w, int64_t n, const float table[16],
                        uint8_t* codes, float* absmax) {
    if (n < 0 || n % ORACLE_BLOCK != 0) return -1;
    int64_t nb = n / ORACLE_BLOCK;
#pragma omp parallel for schedule(static)
    for (int64_t b = 0; b < nb; ++b) {
        const float* blk = w + b * ORACLE_BLOCK;
        float am = 0.0f;
        for (int j = 0; j < ORACLE_BLOCK; ++j) {
            float a = fabsf(blk[j]);
            if (a > am) am = a;
        }
        absmax[b] = am;
        uint8_t* out = codes + b * (ORACLE_BLOCK / 2);
        for (int j = 0; j < ORACLE_BLOCK; j += 2) {
            int c0, c1;
            if (am == 0.0f) {
                c0 = c1 = oracle_nearest_code(0.0f, table);
            } else {
                volatile float n0 = blk[j] / am;      /* one fp32 rounding */
                volatile float n1 = blk[j + 1] / am;
                c0 = oracle_nearest_code(n0, table);
                c1 = oracle_nearest_code(n1, table);
            }
            out[j / 2] = (uint8_t)(c0 | (c1 << 4));   /* even element: low nibble */
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Double quantization.  [p1] §5-2 (the fp32 absmax constants of the first  */
/* stage are quantized to 8 bits in blocks of 256) and [p2] "Double          */
/* Quantization の仕組み" (W ~ (c2 * c1_quant) * W_quant).  Per group:       */
/* c2 = max absmax, s2 = fp32(c2/255) is the stored fp32 second-level        */
/* constant, q = min(255, rint_half_even(fp32(absmax/s2))), s2 == 0 -> q = 0.*/
/* nb absmax values; the last group may be partial.                          */
/* ------------------------------------------------------------------------ */
void oracle_double_quant(const float* absmax, int64_t nb, uint8_t* q8, float* s2) {
    int64_t ng = (nb + ORACLE_GROUP - 1) / ORACLE_GROUP;
#pragma omp parallel for schedule(static)
    for (int64_t g = 0; g < ng; ++g) {
        int64_t b0 = g * ORACLE_GROUP;
        int64_t b1 = b0 + ORACLE_GROUP < nb ? b0 + ORACLE_GROUP : nb;
        float c2 = 0.0f;
        for (int64_t b = b0; b < b1; ++b) if (absmax[b] > c2) c2 = absmax[b];
        volatile float s = c2 / 255.0f;
        s2[g] = s;
        for (int64_t b = b0; b < b1; ++b) {
            if (s == 0.0f) { q8[b] = 0; continue; }
            volatile float ratio = absmax[b] / s;
            float r = rintf(ratio);                 /* default mode: half-even */
            if (r > 255.0f) r = 255.0f;
            q8[b] = (uint8_t)r;
        }
    }
}

/* FP8 E4M3 (1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits, no   */
/* infinities, largest finite value 448, smallest subnormal 2^-9).  Encode:  */
/* round to nearest even, then clamp to 448 (saturating); input >= 0.        */
uint8_t oracle_f32_to_e4m3(float x) {
    if (!(x > 0.0f)) return 0;
    double a = (double)x;
    int e;
    frexp(a, &e);                        /* a = m * 2^e, 0.5 <= m < 1          */
    int ue = e - 4;                      /* 4 significant bits                 */
    if (ue < -9) ue = -9;                /* subnormal step 2^-9                */
    double r = ldexp(rint(ldexp(a, -ue)), ue);
    if (r > 448.0) r = 448.0;
    if (r == 0.0) return 0;
    int E;
    double m = frexp(r, &E);
    int ef = E - 1 + 7;                  /* biased exponent of r               */
    if (ef <= 0) return (uint8_t)ldexp(r, 9);          /* subnormal: r / 2^-9 */
    return (uint8_t)((ef << 3) | ((int)ldexp(m, 4) - 8));
}

float oracle_e4m3_to_f32(uint8_t b) {
    int e = (b >> 3) & 15, m = b & 7;
    double v = e == 0 ? ldexp((double)m, -9) : ldexp(1.0 + m / 8.0, e - 7);
    return (float)((b & 0x80) ? -v : v);
}

/* The FP8 reading of the second stage of p1 §5-2 ("8bit量子化（FP8相当）"),     */
/* [p2] "Double Quantization の仕組み" (c1 quantized to 8 bits with the FP32  */
/* c2 above it): per group of 256 blocks, s = fp32(c2 / 448) so that the    */
/* group maximum maps to E4M3's largest finite value, q = E4M3(fp32(absmax  */
/* / s)), q = 0 when s == 0.  s2 stores -s: its sign bit marks the group as */
/* FP8 (every linear-format s2 is >= 0), and c1' = fp32(E4M3 value * |s2|). */
void oracle_double_quant_fp8(const float* absmax, int64_t nb, uint8_t* q8, float* s2) {
    int64_t ng = (nb + ORACLE_GROUP - 1) / ORACLE_GROUP;
#pragma omp parallel for schedule(static)
    for (int64_t g = 0; g < ng; ++g) {
        int64_t b0 = g * ORACLE_GROUP;
        int64_t b1 = b0 + ORACLE_GROUP < nb ? b0 + ORACLE_GROUP : nb;
        float c2 = 0.0f;
        for (int64_t b = b0; b < b1; ++b) if (absmax[b] > c2) c2 = absmax[b];
        volatile float s = c2 / 448.0f;
        s2[g] = -s;
        for (int64_t b = b0; b < b1; ++b) {
            if (s == 0.0f) { q8[b] = 0; continue; }
            volatile float ratio = absmax[b] / s;
            q8[b] = oracle_f32_to_e4m3(ratio);
        }
    }
}


/* Round an fp32 value to bf16 (round to nearest, ties to even), returned as */
/* its 16-bit pattern.  NaN stays a quiet NaN.                               */
uint16_t oracle_f32_to_bf16(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7f800000u) == 0x7f800000u && (u & 0x007fffffu))
        return (uint16_t)((u >> 16) | 0x0040u);
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7fffu + lsb;
    return (uint16_t)(u >> 16);
}

/* ------------------------------------------------------------------------ */
/* Dequantization.  [p1] §5-1 step 3 (w_hat = c_i* x absmax), with the       */
/* absmax rebuilt from the double-quantized pair as [p2] gives it            */
/* (c1' = c2-scale x c1_quant), computed to bf16 as the storage/compute      */
/* split of [p2] "4bitのまま計算しているわけではない" requires:               */
/*   c1' = fp32(q * s2);  w32 = fp32(c[code] * c1');  w = bf16_rn(w32).      */
/* out_f32 (may be NULL) gets w32, out_bf16 (may be NULL) gets w.           */
/* ------------------------------------------------------------------------ */
void oracle_dequant(const uint8_t* codes, const uint8_t* q8, const float* s2,
                    int64_t n, const float table[16], float* out_f32,
                    uint16_t* out_bf16) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) {
        int64_t b = i / ORACLE_BLOCK, g = b / ORACLE_GROUP;
        int code = (i & 1) ? (codes[i / 2] >> 4) : (codes[i / 2] & 15);
        /* a set sign bit marks an FP8-format group (oracle_double_quant_fp8) */
        volatile float c1 = signbit(s2[g]) ? oracle_e4m3_to_f32(q8[b]) * -s2[g] : (float)q8[b] * s2[g];
        volatile float w32 = table[code] * c1;
        if (out_f32) out_f32[i] = w32;
        if (out_bf16) out_bf16[i] = oracle_f32_to_bf16(w32);
    }
}

/* Single quantization: only the first stage of p1 §5-2 ("Double
 * Quantization", memory arithmetic: first stage only = 4 + 32/64 = 4.5
 * bit/param; the p1 bitsandbytes listing's bnb_4bit_use_double_quant knob
 * turns the second stage off).  The fp32 absmax of each 64-block is kept as
 * is, so the block scale is absmax itself:
 * w = bf16( fp32( c[code] * absmax ) ). */
void oracle_dequant_single(const uint8_t* codes, const float* absmax, int64_t n,
                           const float table[16], float* out_f32, uint16_t* out_bf16) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) {
        int64_t b = i / ORACLE_BLOCK;
        int code = (i & 1) ? (codes[i / 2] >> 4) : (codes[i / 2] & 15);
        volatile float w32 = table[code] * absmax[b];
        if (out_f32) out_f32[i] = w32;
        if (out_bf16) out_bf16[i] = oracle_f32_to_bf16(w32);
    }
}

/* fp64 -> bf16, round to nearest, ties to even, in one step (no detour     */
/* through fp32).  Finite input; values past the largest bf16 become inf.   */
uint16_t oracle_f64_to_bf16(double x) {
    if (x == 0.0) return signbit(x) ? 0x8000u : 0x0000u;
    double a = fabs(x);
    int e;
    frexp(a, &e);                        /* a = m * 2^e, 0.5 <= m < 1          */
    int ue = e - 8;                      /* bf16 keeps 8 significant bits       */
    if (ue < -133) ue = -133;            /* subnormal bf16: ulp 2^-133          */
    double q = rint(ldexp(a, -ue));      /* exact scaling, then round-half-even */
    double r = ldexp(q, ue);             /* exactly representable in fp32       */
    float f = (float)r;
    if (r > 3.3895313892515355e38) f = INFINITY;   /* beyond the largest bf16 */
    uint32_t u;
    memcpy(&u, &f, 4);
    uint16_t b = (uint16_t)(u >> 16);
    return x < 0 ? (uint16_t)(b | 0x8000u) : b;
}

static double oracle_bf16_to_f64(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* Adapter merge for distribution, [p4] "学習済みアダプタのマージと配布で精度が */
/* 崩れる分岐点を整理する": merging into the 4-bit base rounds the adapter's    */
/* small differences onto the 4-bit grid, so the adapter is folded into the  */
/* unquantized base loaded in bf16, and the merged 16-bit weight is then     */
/* quantized again.  Here: W16 = bf16(W); each output element is            */
/*   v = fp64(W16) + fp64(s) * sum_{j=0..r-1} B[n,j] A[j,k]                  */
/* with the sum taken in fp64 in the order j = 0, 1, ..., one rounding per   */
/* product and per addition (products of two bf16 values are exact in fp64), */
/* and merged = bf16(v), rounded once.  s = fp32(alpha / r).  W is N x K     */
/* fp32, A is r x K and B is N x r as bf16 bit patterns; out is N x K bf16.  */
void oracle_merge_adapter(const float* W, int64_t N, int64_t K, const uint16_t* A, const uint16_t* B,
                          int r, double alpha, uint16_t* out) {
    volatile float s32 = (float)(alpha / (double)r);
    double s = (double)s32;
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t k = 0; k < K; ++k) {
            volatile double acc = 0.0;
            for (int j = 0; j < r; ++j) {
                volatile double prod = oracle_bf16_to_f64(B[n * r + j]) * oracle_bf16_to_f64(A[(int64_t)j * K + k]);
                acc = acc + prod;
            }
            volatile double t = s * acc;
            volatile double v = oracle_bf16_to_f64(oracle_f32_to_bf16(W[n * K + k])) + t;
            out[n * K + k] = oracle_f64_to_bf16(v);
        }
    }
}

/* ------------------------------------------------------------------------ */
/* LoRA dropout on the adapter input ([p1] PEFT listing LoraConfig(...,     */
/* lora_dropout=0.05); the adapter sees dropout(x) = x * keep / (1 - p)).    */
/* The keep decisions come from Philox4x32-10, the counter-based generator  */
/* of Salmon, Moraes, Dror and Shaw, "Parallel Random Numbers: As Easy as   */
/* 1, 2, 3" (SC'11), written here from that definition: 10 rounds of two    */
/* 32x32->64 multiplications (multipliers 0xD2511F53, 0xCD9E8D57) with the  */
/* key bumped by the Weyl constants (0x9E3779B9, 0xBB67AE85) between rounds. */
void oracle_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4]) {
    uint32_t c0 = ctr[0], c1 = ctr[1], c2 = ctr[2], c3 = ctr[3];
    uint32_t k0 = key[0], k1 = key[1];
    for (int round = 0; round < 10; ++round) {
        uint64_t p0 = (uint64_t)0xD2511F53u * c0;
        uint64_t p1 = (uint64_t)0xCD9E8D57u * c2;
        uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
        uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
        uint32_t n0 = hi1 ^ c1 ^ k0;
        uint32_t n1 = lo1;
        uint32_t n2 = hi0 ^ c3 ^ k1;
        uint32_t n3 = lo0;
        c0 = n0; c1 = n1; c2 = n2; c3 = n3;
        k0 += 0x9E3779B9u;
        k1 += 0xBB67AE85u;
    }
    out[0] = c0; out[1] = c1; out[2] = c2; out[3] = c3;
}

/* Keep decision of element e (row-major index m*K + k of X).  One block of */
/* Philox4x32-10, counter (lo32(e>>3), hi32(e>>3), lo32(offset),            */
/* hi32(offset)) and key (lo32(seed), hi32(seed)), decides 8 elements: e    */
/* reads the 16-bit half (e & 1) (0 = the low half) of word ((e >> 1) & 3) */
/* and is kept when that half is >= t, t = floor(p * 2^16) (the caller's    */
/* integer threshold), so the drop probability is t / 2^16.                 */
void oracle_dropout_keep(int64_t M, int64_t K, uint32_t t, uint64_t seed, uint64_t offset, uint8_t* keep) {
    const uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
#pragma omp parallel for schedule(static)
    for (int64_t q = 0; q < (M * K + 7) / 8; ++q) {
        uint32_t ctr[4] = {(uint32_t)q, (uint32_t)((uint64_t)q >> 32), (uint32_t)offset, (uint32_t)(offset >> 32)};
        uint32_t w[4];
        oracle_philox4x32_10(ctr, key, w);
        for (int j = 0; j < 8; ++j) {
            int64_t e = q * 8 + j;
            uint32_t half = (w[j >> 1] >> (16 * (j & 1))) & 0xFFFFu;
            if (e < M * K) keep[e] = half >= t ? 1 : 0;
        }
    }
}

/* ------------------------------------------------------------------------ */
/* The linear layer in fp64, row-major.  W is N x K (out x in), X is M x K,  */
/* A is r x K, B is N x r, s = alpha / r.                                    */
/* [p1] "LoRAの復習" h = W0 x + (alpha/r) B A x, and "QLoRAの計算フロー"     */
/* steps 1-4 (dequant, main product, A x then B, sum).  Column vectors of    */
/* the pages become rows here: Y = X W^T + s (X A^T) B^T.                    */
/* rows: if non-NULL, only those nrows rows of Y (and U) are computed and    */
/* written compactly (row i of the output is row rows[i] of the full Y).     */
/* ------------------------------------------------------------------------ */
void oracle_linear_fwd(const double* X, const double* W, const double* A,
                       const double* B, int64_t M, int64_t N, int64_t K, int r,
                       double alpha, const int64_t* rows, int64_t nrows,
                       double* Y, double* U) {
    double s = alpha / (double)r;
    int64_t count = rows ? nrows : M;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t i = 0; i < count; ++i) {
        int64_t m = rows ? rows[i] : i;
        const double* x = X + m * K;
        double* u = U + i * r;
        for (int j = 0; j < r; ++j) {               /* U = X A^T (r values) */
            const double* a = A + (int64_t)j * K;
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k) acc += x[k] * a[k];
            u[j] = acc;
        }
        for (int64_t nn = 0; nn < N; ++nn) {        /* Y = X W^T + s U B^T */
            const double* wr = W + nn * K;
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k) acc += x[k] * wr[k];
            double lora = 0.0;
            for (int j = 0; j < r; ++j) lora += u[j] * B[nn * r + j];
            Y[i * N + nn] = acc + s * lora;
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Backward, [p1] "逆伝播と勾配の流れ":                                       */
/*   dL/dB = (alpha/r) dL/dY (A X)^T   ->  dB = s dY^T U      (N x r)        */
/*   dL/dA = (alpha/r) B^T dL/dY X^T   ->  dA = s (dY B)^T X  (r x K)        */
/* W is frozen (no gradient).  dX is the chain rule through both paths:      */
/*   dX = dY W + s (dY B) A                                   (M x K)        */
/* Only dX's rows may be sampled (rows/nrows as in the forward); dA and dB   */
/* are always full reductions over all M rows.                               */
/* ------------------------------------------------------------------------ */
void oracle_linear_bwd(const double* X, const double* W, const double* A,
                       const double* B, const double* dY, int64_t M, int64_t N,
                       int64_t K, int r, double alpha, const int64_t* rows,
                       int64_t nrows, double* dX, double* dA, double* dB) {
    double s = alpha / (double)r;
    double* V = (double*)malloc(sizeof(double) * (size_t)M * (size_t)r);
    double* U = (double*)malloc(sizeof(double) * (size_t)M * (size_t)r);
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        const double* dy = dY + m * N;
        const double* x = X + m * K;
        for (int j = 0; j < r; ++j) {
            double acc = 0.0;                        /* V = dY B */
            for (int64_t nn = 0; nn < N; ++nn) acc += dy[nn] * B[nn * r + j];
            V[m * r + j] = acc;
            const double* a = A + (int64_t)j * K;   /* U = X A^T */
            double au = 0.0;
            for (int64_t k = 0; k < K; ++k) au += x[k] * a[k];
            U[m * r + j] = au;
        }
    }
    int64_t count = rows ? nrows : M;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t i = 0; i < count; ++i) {
        int64_t m = rows ? rows[i] : i;
        const double* dy = dY + m * N;
        double* out = dX + i * K;
        for (int64_t k = 0; k < K; ++k) out[k] = 0.0;
        for (int64_t nn = 0; nn < N; ++nn) {         /* dY W */
            double g = dy[nn];
            const double* wr = W + nn * K;
            for (int64_t k = 0; k < K; ++k) out[k] += g * wr[k];
        }
        for (int j = 0; j < r; ++j) {                /* + s V A */
            double g = s * V[m * r + j];
            const double* a = A + (int64_t)j * K;
            for (int64_t k = 0; k < K; ++k) out[k] += g * a[k];
        }
    }
#pragma omp parallel for schedule(static)
    for (int64_t k = 0; k < K; ++k) {                /* dA = s V^T X */
        for (int j = 0; j < r; ++j) {
            double acc = 0.0;
            for (int64_t m = 0; m < M; ++m) acc += V[m * r + j] * X[m * K + k];
            dA[(int64_t)j * K + k] = s * acc;
        }
    }
#pragma omp parallel for schedule(static)
    for (int64_t nn = 0; nn < N; ++nn) {             /* dB = s dY^T U */
        for (int j = 0; j < r; ++j) {
            double acc = 0.0;
            for (int64_t m = 0; m < M; ++m) acc += dY[m * N + nn] * U[m * r + j];
            dB[nn * r + j] = s * acc;
        }
    }
    free(V);
    free(U);
}
