/*
 * Ternary BitLinear oracle: plain, slow, single-threaded CPU C.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may include, link or
 * call this code; only the tests, the smoke check and the benchmark's CPU
 * baseline leg use it.  It shares no code, header, table or constant with the
 * CUDA library under ternary_weight_bit_bitlinear_b200/csrc.
 *
 * What it computes (BitNet b1.58 BitLinear, I2_S-style "int2 with scale"):
 *   alpha  = mean |W| over the whole weight tensor, rounded once to fp32
 *   c[m,k] = clamp(round_half_even(W[m,k] / alpha), -1, 1)
 *   amax_n = max_k |x[n,k]|,  s_n = 127 / amax_n  (fp32)
 *   q[n,k] = clamp(round_half_even(x[n,k] * s_n), -128, 127)
 *   acc[n,m] = sum_k c[m,k] * q[n,k]                      (int32)
 *   y[n,m] = (float)acc * (alpha * (amax_n / 127))        (fp32, each op RN)
 *
 * Sources: "Bitnet.cpp: Efficient Edge Inference for Ternary LLMs" reading
 * notes, section 1.1 (weights in {-1,0,1}), section 2.3 (I2_S: ternary weights
 * with one scale, int8 activations, 2.0 bits per weight, lossless), section 4.1
 * (lossless-inference conditions); FairyFuse article, "ternary quantisation
 * scheme" (threshold +-0.5 alpha) and "fused kernel design" (add/subtract
 * accumulation over bit-packed codes).
 *
 * Packed layout (defined by this project; the pages fix only 2.0 bpw):
 *   row m of W occupies 4*ceil(K/64) little-endian uint32 words (K/16 when K
 *   is a multiple of 64; otherwise the row is padded to a 16-byte boundary);
 *   weight k sits in word k/16 of its row at bit 8*(k%4) + 2*((k%16)/4);
 *   the 2-bit field holds the offset-binary code c+1 in {0,1,2}; 3 never
 *   occurs; padding fields past K hold 01, i.e. code 0, weight nothing.
 *
 * Error convention: functions returning int give 0 on success, a negative
 * value on a rejected input (documented per function).
 */
#ifndef BITLINEAR_ORACLE_H
#define BITLINEAR_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Exponent-binned exact |w| sum: bins[e] += 24-bit significand of |w| whose
 * biased exponent is e (subnormals go to e=1 with their raw fraction).
 * Adds to bins (caller zeroes them).  Returns -1 if any w is inf/NaN. */
int oracle_abs_bins(const float* w, int64_t n, uint64_t bins[256]);

/* alpha = sum|w| / count rounded to nearest-even fp32, from exact bins.
 * count must be in [1, 2^40].  Returns 0.0f when the sum is zero. */
float oracle_alpha_from_bins(const uint64_t bins[256], int64_t count);

/* alpha for a whole tensor; *status = 0 or -1 (non-finite input). */
float oracle_absmean(const float* w, int64_t n, int* status);

/* codes[i] = clamp(rint(w[i]/alpha), -1, 1); all zero when alpha == 0. */
void oracle_ternarize(const float* w, int64_t n, float alpha, int8_t* codes);

/* Words per packed row: 4*ceil(K/64). */
int64_t oracle_packed_row_words(int64_t K);

/* Pack codes [M,K] (K % 16 == 0) into M*oracle_packed_row_words(K) words.
 * Returns -1 on a code outside {-1,0,1} or a bad K. */
int oracle_pack(const int8_t* codes, int64_t M, int64_t K, uint32_t* packed);

/* Inverse of oracle_pack.  Returns -1 if a field holds 3 or a padding field
 * is not code 0. */
int oracle_unpack(const uint32_t* packed, int64_t M, int64_t K, int8_t* codes);

/* TL2-style storage, 5 bits per three weights (defined by this project; the
 * pages fix the 1-bit sign + 4-bit index split and the 5/3 bits per weight).
 * Per row, with nb = floor(K/96) blocks of 96 weights and K2 = K - 96*nb:
 *   bytes [0, 16*nb)        index plane: block b's group g (weights 96b+3g ..
 *                           96b+3g+2) has its 4-bit index in byte 16b + g/2,
 *                           low nibble for even g;
 *   next 16*ceil(nb/4)      sign plane: block b's 32 signs in the
 *                           little-endian uint32 at 4b (bit g), zero padding;
 *   next 16*ceil(K2/64)     the last K2 weights in the 2-bit layout of
 *                           oracle_pack (a K2-wide row, padded with code 0).
 * A group's v = 9(c0+1) + 3(c1+1) + (c2+1): index |v - 13|, sign (v < 13).
 * Negating a group's codes flips its sign bit only.  K % 16 == 0. */
int64_t oracle_tl2_row_bytes(int64_t K);
int oracle_tl2_encode(const int8_t* codes, int64_t M, int64_t K, uint8_t* out);
/* Inverse; -1 on an index above 13, a negative zero group, or bad padding. */
int oracle_tl2_decode(const uint8_t* in, int64_t M, int64_t K, int8_t* codes);

/* Per-token absmax int8 quantisation of x [N,K].  qsum may be NULL. */
void oracle_quant_act(const float* x, int64_t N, int64_t K,
                      int8_t* q, float* amax, int32_t* qsum);

/* Per-tensor variant: one absmax over the whole x [N,K]; every amax[n] gets
 * that value and every element uses s = 127/amax. */
void oracle_quant_act_per_tensor(const float* x, int64_t N, int64_t K,
                                 int8_t* q, float* amax, int32_t* qsum);

/* Triple-loop int32 matmul acc[n*M+m] = sum_k codes[m*K+k] * q[n*K+k]. */
void oracle_matmul_i32(const int8_t* codes, int64_t M, int64_t K,
                       const int8_t* q, int64_t N, int32_t* acc);

/* The same product evaluated with additions and subtractions only. */
void oracle_matmul_addsub(const int8_t* codes, int64_t M, int64_t K,
                          const int8_t* q, int64_t N, int32_t* acc);

/* y[n*M+m] = (float)acc[n*M+m] * (alpha * (amax[n] / 127.0f)). */
void oracle_rescale(const int32_t* acc, int64_t N, int64_t M, float alpha,
                    const float* amax, float* y);

/* Whole layer from latent weights: alpha, packed, q/amax/qsum, acc, y.
 * Scratch (codes) is allocated here.  Returns 0, -1 (non-finite W) or -2
 * (allocation failure / bad shape). */
int oracle_bitlinear(const float* W, int64_t M, int64_t K,
                     const float* x, int64_t N,
                     float* alpha, uint32_t* packed, int8_t* q, float* amax,
                     int32_t* qsum, int32_t* acc, float* y);

#ifdef __cplusplus
}
#endif

#endif
