/*
 * Ternary BitLinear oracle -- TEST INFRASTRUCTURE ONLY (see bitlinear_oracle.h).
 *
 * Plain C99, single thread, no SIMD intrinsics, built with
 * -O2 -fno-fast-math -ffp-contract=off so that every fp32 operation below is
 * one IEEE round-to-nearest-even operation in the order written.
 */
#include "bitlinear_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------- */
/* alpha = mean|W|                                                           */
/*                                                                           */
/* Bitnet.cpp reading notes, section 1.1 and section 4.1 "lossless inference */
/* conditions": BitNet b1.58 weights are ternary with one per-tensor scale.  */
/* The formula itself did not survive extraction; the scale is read here as  */
/* the absolute mean of W (BitNet b1.58's absmean rule), computed exactly and */
/* rounded once to fp32 so that the result does not depend on summation     */
/* order.                                                                    */
/* ------------------------------------------------------------------------- */

int oracle_abs_bins(const float* w, int64_t n, uint64_t bins[256])
{
    int bad = 0;
    for (int64_t i = 0; i < n; ++i) {
        uint32_t bits;
        memcpy(&bits, &w[i], sizeof bits);
        uint32_t e = (bits >> 23) & 0xFFu;
        uint32_t frac = bits & 0x7FFFFFu;
        if (e == 255u) {          /* inf or NaN */
            bad = 1;
            continue;
        }
        uint64_t significand;
        if (e == 0u) {            /* zero or subnormal: frac * 2^-149 */
            significand = frac;
            e = 1u;
        } else {                  /* normal: (2^23 + frac) * 2^(e-150) */
            significand = (uint64_t)frac | 0x800000u;
        }
        bins[e] += significand;
    }
    return bad ? -1 : 0;
}

/* Big unsigned integer, 32-bit little-endian limbs. */
#define BIG_LIMBS 16   /* 512 bits: the sum needs < 318, plus the 128-bit shift */

static void big_add_shifted(uint32_t* big, uint64_t v, int shift)
{
    int limb = shift / 32;
    int off = shift % 32;
    /* v << off spans at most three limbs */
    uint64_t lo = (v << off) & 0xFFFFFFFFu;
    uint64_t mid = (off == 0) ? (v >> 32) : ((v >> (32 - off)) & 0xFFFFFFFFu);
    uint64_t hi = (off == 0) ? 0 : (v >> (64 - off));
    uint64_t parts[3] = {lo, mid, hi};
    uint64_t carry = 0;
    for (int i = 0; limb + i < BIG_LIMBS; ++i) {
        uint64_t add = (i < 3) ? parts[i] : 0;
        if (i >= 3 && carry == 0) break;
        uint64_t s = (uint64_t)big[limb + i] + add + carry;
        big[limb + i] = (uint32_t)s;
        carry = s >> 32;
    }
}

static int big_top_bit(const uint32_t* big)
{
    for (int i = BIG_LIMBS - 1; i >= 0; --i) {
        if (big[i] != 0) {
            int b = 31;
            while (((big[i] >> b) & 1u) == 0) --b;
            return i * 32 + b;
        }
    }
    return -1;
}

static int big_bit(const uint32_t* big, int pos)
{
    return (int)((big[pos / 32] >> (pos % 32)) & 1u);
}

float oracle_alpha_from_bins(const uint64_t bins[256], int64_t count)
{
    /* B = sum_e bins[e] * 2^(e-1), so that sum|w| = B * 2^-149. */
    uint32_t B[BIG_LIMBS];
    memset(B, 0, sizeof B);
    for (int e = 1; e < 255; ++e)
        if (bins[e] != 0) big_add_shifted(B, bins[e], e - 1);
    if (big_top_bit(B) < 0) return 0.0f;

    /* Q = floor(B * 2^128 / count), rem = remainder.  Long division in
     * 16-bit digits keeps every intermediate below 2^56 (count <= 2^40). */
    const int SHIFT = 128;
    uint32_t S[BIG_LIMBS];
    memset(S, 0, sizeof S);
    for (int i = 0; i + SHIFT / 32 < BIG_LIMBS; ++i) S[i + SHIFT / 32] = B[i];
    uint32_t Q[BIG_LIMBS];
    memset(Q, 0, sizeof Q);
    uint64_t rem = 0;
    uint64_t d = (uint64_t)count;
    for (int i = BIG_LIMBS - 1; i >= 0; --i) {
        uint32_t qlimb = 0;
        for (int h = 1; h >= 0; --h) {
            uint64_t digit = (S[i] >> (16 * h)) & 0xFFFFu;
            rem = (rem << 16) | digit;
            uint64_t qd = rem / d;
            rem = rem % d;
            qlimb |= (uint32_t)qd << (16 * h);
        }
        Q[i] = qlimb;
    }

    /* mean = (Q + rem/count) * 2^(-149-128).  Round to fp32, ties to even. */
    int p = big_top_bit(Q);               /* Q >= 2^88 > 0 */
    int E = p - (149 + SHIFT);            /* mean in [2^E, 2^(E+1)) */
    int cut = (E >= -126) ? (p - 23) : SHIFT;  /* lowest kept bit of Q */
    uint64_t mant = 0;
    for (int b = p; b >= cut; --b) mant = (mant << 1) | (uint64_t)big_bit(Q, b);
    int half = big_bit(Q, cut - 1);
    int below = (rem != 0);
    for (int b = cut - 2; b >= 0 && !below; --b) below = big_bit(Q, b);
    if (half && (below || (mant & 1u))) mant += 1;
    /* value = mant * 2^(cut - 277); exact in double, and representable in fp32 */
    return (float)ldexp((double)mant, cut - (149 + SHIFT));
}

float oracle_absmean(const float* w, int64_t n, int* status)
{
    uint64_t bins[256];
    memset(bins, 0, sizeof bins);
    int rc = oracle_abs_bins(w, n, bins);
    if (status) *status = rc;
    if (rc != 0 || n <= 0) return rc != 0 ? NAN : 0.0f;
    return oracle_alpha_from_bins(bins, n);
}

/* ------------------------------------------------------------------------- */
/* Ternarisation.  Reading notes section 1.1: weights take values in         */
/* {-1,0,1}.  Round-to-nearest of w/alpha clamped to [-1,1]; an exact tie    */
/* (|w/alpha| == 0.5) rounds to even, i.e. to 0, which agrees with the       */
/* FairyFuse threshold rule (w > 0.5 alpha -> +1, w < -0.5 alpha -> -1).     */
/* ------------------------------------------------------------------------- */

void oracle_ternarize(const float* w, int64_t n, float alpha, int8_t* codes)
{
    for (int64_t i = 0; i < n; ++i) {
        if (alpha == 0.0f) {
            codes[i] = 0;
            continue;
        }
        float r = w[i] / alpha;
        float t = rintf(r);          /* default rounding mode: nearest-even */
        int c;
        if (t > 1.0f) c = 1;
        else if (t < -1.0f) c = -1;
        else c = (int)t;
        codes[i] = (int8_t)c;
    }
}

/* ------------------------------------------------------------------------- */
/* 2-bit packing: 2.0 bits per weight, the I2_S storage size in the reading  */
/* notes' section 2.3 method table.  Layout as stated in the header.          */
/* ------------------------------------------------------------------------- */

static int field_bit(int64_t k)
{
    return (int)(8 * (k % 4) + 2 * ((k % 16) / 4));
}

int64_t oracle_packed_row_words(int64_t K)
{
    return 4 * ((K + 63) / 64);
}

int oracle_pack(const int8_t* codes, int64_t M, int64_t K, uint32_t* packed)
{
    if (K % 16 != 0 || M < 0) return -1;
    int64_t wpr = oracle_packed_row_words(K);
    /* every field starts as 01 (code 0), so the padding past K stays code 0 */
    for (int64_t i = 0; i < M * wpr; ++i) packed[i] = 0x55555555u;
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t k = 0; k < K; ++k) {
            int c = codes[m * K + k];
            if (c < -1 || c > 1) return -1;
            uint32_t field = (uint32_t)(c + 1);
            uint32_t* w = &packed[m * wpr + k / 16];
            *w = (*w & ~(3u << field_bit(k))) | (field << field_bit(k));
        }
    }
    return 0;
}

int oracle_unpack(const uint32_t* packed, int64_t M, int64_t K, int8_t* codes)
{
    if (K % 16 != 0 || M < 0) return -1;
    int64_t wpr = oracle_packed_row_words(K);
    int bad = 0;
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t k = 0; k < 16 * wpr; ++k) {
            uint32_t field = (packed[m * wpr + k / 16] >> field_bit(k)) & 3u;
            if (field == 3u) bad = 1;
            if (k < K)
                codes[m * K + k] = (int8_t)((int)field - 1);
            else if (field != 1u)
                bad = 1;       /* padding must hold code 0 */
        }
    }
    return bad ? -1 : 0;
}

/* ------------------------------------------------------------------------- */
/* TL2-style storage at 5/3 bits per weight (reading notes section 2.3       */
/* "technical details": three ternary weights stored as a 1-bit sign plus a  */
/* 4-bit index, 5 bits in all, by folding each combination onto its mirror  */
/* image; K split into a part stored in groups of three and a remainder).    */
/* The index table and byte layout are this project's own (see header).     */
/* ------------------------------------------------------------------------- */

static int64_t tl2_blocks(int64_t K) { return K / 96; }

int64_t oracle_tl2_row_bytes(int64_t K)
{
    int64_t nb = tl2_blocks(K);
    int64_t k2 = K - 96 * nb;
    return 16 * nb + 16 * ((nb + 3) / 4) + 16 * ((k2 + 63) / 64);
}

/* One group of three codes -> (sign, index): the base-3 number of the codes
 * plus one, v = 9(c0+1) + 3(c1+1) + (c2+1) in [0, 26], mirrors to 26 - v when
 * every code is negated; v = 13 is (0,0,0), its own mirror.  The index is
 * |v - 13| in [0, 13] and the sign says which side of 13 v lies on. */
static void tl2_encode_group(int c0, int c1, int c2, int* sign, int* index)
{
    int v = 9 * (c0 + 1) + 3 * (c1 + 1) + (c2 + 1);
    if (v >= 13) { *sign = 0; *index = v - 13; }
    else         { *sign = 1; *index = 13 - v; }
}

static void tl2_decode_group(int sign, int index, int* c)
{
    int v = sign ? 13 - index : 13 + index;
    c[0] = v / 9 - 1;
    c[1] = (v / 3) % 3 - 1;
    c[2] = v % 3 - 1;
}

int oracle_tl2_encode(const int8_t* codes, int64_t M, int64_t K, uint8_t* out)
{
    if (K % 16 != 0 || M < 0) return -1;
    int64_t nb = tl2_blocks(K), k3 = 96 * nb, k2 = K - k3;
    int64_t rb = oracle_tl2_row_bytes(K);
    int64_t sign_off = 16 * nb, tail_off = sign_off + 16 * ((nb + 3) / 4);
    for (int64_t m = 0; m < M; ++m) {
        const int8_t* c = codes + m * K;
        uint8_t* row = out + m * rb;
        for (int64_t i = 0; i < rb; ++i) row[i] = 0;
        for (int64_t k = 0; k < K; ++k)
            if (c[k] < -1 || c[k] > 1) return -1;
        for (int64_t b = 0; b < nb; ++b) {
            uint32_t signs = 0;
            for (int g = 0; g < 32; ++g) {
                int64_t k = 96 * b + 3 * g;
                int s, idx;
                tl2_encode_group(c[k], c[k + 1], c[k + 2], &s, &idx);
                row[16 * b + g / 2] |= (uint8_t)(idx << (4 * (g % 2)));
                signs |= (uint32_t)s << g;
            }
            for (int j = 0; j < 4; ++j)
                row[sign_off + 4 * b + j] = (uint8_t)(signs >> (8 * j));
        }
        /* the remainder: the 2-bit layout of oracle_pack, padded with code 0 */
        int64_t tail_words = 4 * ((k2 + 63) / 64);
        for (int64_t w = 0; w < tail_words; ++w) {
            uint32_t word = 0x55555555u;
            for (int64_t i = 0; i < 16; ++i) {
                int64_t j = 16 * w + i;
                if (j >= k2) break;
                int bit = field_bit(j);
                word = (word & ~(3u << bit)) | ((uint32_t)(c[k3 + j] + 1) << bit);
            }
            for (int j = 0; j < 4; ++j)
                row[tail_off + 4 * w + j] = (uint8_t)(word >> (8 * j));
        }
    }
    return 0;
}

int oracle_tl2_decode(const uint8_t* in, int64_t M, int64_t K, int8_t* codes)
{
    if (K % 16 != 0 || M < 0) return -1;
    int64_t nb = tl2_blocks(K), k3 = 96 * nb, k2 = K - k3;
    int64_t rb = oracle_tl2_row_bytes(K);
    int64_t sign_off = 16 * nb, tail_off = sign_off + 16 * ((nb + 3) / 4);
    int bad = 0;
    for (int64_t m = 0; m < M; ++m) {
        const uint8_t* row = in + m * rb;
        int8_t* c = codes + m * K;
        for (int64_t b = 0; b < nb; ++b) {
            uint32_t signs = 0;
            for (int j = 0; j < 4; ++j) signs |= (uint32_t)row[sign_off + 4 * b + j] << (8 * j);
            for (int g = 0; g < 32; ++g) {
                int idx = (row[16 * b + g / 2] >> (4 * (g % 2))) & 15;
                int s = (signs >> g) & 1;
                if (idx > 13 || (idx == 0 && s)) bad = 1;   /* never written */
                int d[3];
                tl2_decode_group(s, idx > 13 ? 0 : idx, d);
                for (int i = 0; i < 3; ++i) c[96 * b + 3 * g + i] = (int8_t)d[i];
            }
        }
        for (int64_t i = sign_off + 4 * nb; i < tail_off; ++i)
            if (row[i] != 0) bad = 1;                        /* sign-plane padding */
        int64_t tail_words = 4 * ((k2 + 63) / 64);
        for (int64_t w = 0; w < tail_words; ++w) {
            uint32_t word = 0;
            for (int j = 0; j < 4; ++j) word |= (uint32_t)row[tail_off + 4 * w + j] << (8 * j);
            for (int64_t i = 0; i < 16; ++i) {
                int64_t j = 16 * w + i;
                uint32_t f = (word >> field_bit(j)) & 3u;
                if (f == 3u) bad = 1;
                if (j < k2) c[k3 + j] = (int8_t)((int)f - 1);
                else if (f != 1u) bad = 1;                   /* padding holds code 0 */
            }
        }
    }
    return bad ? -1 : 0;
}

/* ------------------------------------------------------------------------- */
/* Activation quantisation: absmax to int8 (reading notes section 2.3 and    */
/* 4.1: int8 activations).  Per token (one scale per row of x).  The scale   */
/* s = 127/amax is one fp32 division; the product x*s is rounded half-even   */
/* and clamped.  amax == 0 gives q = 0.  If s overflows to inf (amax below   */
/* 127/FLT_MAX), x*s is +-inf (clamped to 127 / -128) or NaN for x == 0,     */
/* which is taken as 0.                                                      */
/* ------------------------------------------------------------------------- */

void oracle_quant_act(const float* x, int64_t N, int64_t K,
                      int8_t* q, float* amax, int32_t* qsum)
{
    for (int64_t n = 0; n < N; ++n) {
        const float* row = x + n * K;
        float a = 0.0f;
        for (int64_t k = 0; k < K; ++k) {
            float v = fabsf(row[k]);
            if (v > a) a = v;
        }
        amax[n] = a;
        int32_t sum = 0;
        if (a == 0.0f) {
            for (int64_t k = 0; k < K; ++k) q[n * K + k] = 0;
        } else {
            float s = 127.0f / a;
            for (int64_t k = 0; k < K; ++k) {
                float p = row[k] * s;
                float t = rintf(p);
                int v;
                if (isnan(t)) v = 0;
                else if (t > 127.0f) v = 127;
                else if (t < -128.0f) v = -128;
                else v = (int)t;
                q[n * K + k] = (int8_t)v;
                sum += v;
            }
        }
        if (qsum) qsum[n] = sum;
    }
}

/* The reading notes' I2_S setting, section 2.3 "technical details" and
 * section 4.1 "lossless inference conditions": per-tensor int8 activations.
 * The same rule as above with the maximum taken over the whole tensor. */
void oracle_quant_act_per_tensor(const float* x, int64_t N, int64_t K,
                                 int8_t* q, float* amax, int32_t* qsum)
{
    float a = 0.0f;
    for (int64_t i = 0; i < N * K; ++i) {
        float v = fabsf(x[i]);
        if (v > a) a = v;
    }
    for (int64_t n = 0; n < N; ++n) {
        amax[n] = a;
        int32_t sum = 0;
        for (int64_t k = 0; k < K; ++k) {
            int v = 0;
            if (a != 0.0f) {
                float s = 127.0f / a;
                float t = rintf(x[n * K + k] * s);
                if (isnan(t)) v = 0;
                else if (t > 127.0f) v = 127;
                else if (t < -128.0f) v = -128;
                else v = (int)t;
            }
            q[n * K + k] = (int8_t)v;
            sum += v;
        }
        if (qsum) qsum[n] = sum;
    }
}

/* ------------------------------------------------------------------------- */
/* The mpGEMM: int32 accumulation of ternary x int8 products (reading notes   */
/* section 4.1: MAD-based int8 multiply-add).                                */
/* ------------------------------------------------------------------------- */

void oracle_matmul_i32(const int8_t* codes, int64_t M, int64_t K,
                       const int8_t* q, int64_t N, int32_t* acc)
{
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t m = 0; m < M; ++m) {
            int32_t s = 0;
            for (int64_t k = 0; k < K; ++k)
                s += (int32_t)codes[m * K + k] * (int32_t)q[n * K + k];
            acc[n * M + m] = s;
        }
    }
}

/* FairyFuse "fused kernel design": skip a zero weight, add the activation
 * for +1, subtract it for -1 -- no multiplication anywhere. */
void oracle_matmul_addsub(const int8_t* codes, int64_t M, int64_t K,
                          const int8_t* q, int64_t N, int32_t* acc)
{
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t m = 0; m < M; ++m) {
            int32_t s = 0;
            for (int64_t k = 0; k < K; ++k) {
                int8_t c = codes[m * K + k];
                if (c == 1) s += q[n * K + k];
                else if (c == -1) s -= q[n * K + k];
            }
            acc[n * M + m] = s;
        }
    }
}

/* Dequantisation: y = acc * alpha * amax / 127, evaluated as
 * (float)acc * (alpha * (amax / 127)), one RN operation per step. */
void oracle_rescale(const int32_t* acc, int64_t N, int64_t M, float alpha,
                    const float* amax, float* y)
{
    for (int64_t n = 0; n < N; ++n) {
        float step = amax[n] / 127.0f;
        float scale = alpha * step;
        for (int64_t m = 0; m < M; ++m)
            y[n * M + m] = (float)acc[n * M + m] * scale;
    }
}

int oracle_bitlinear(const float* W, int64_t M, int64_t K,
                     const float* x, int64_t N,
                     float* alpha, uint32_t* packed, int8_t* q, float* amax,
                     int32_t* qsum, int32_t* acc, float* y)
{
    if (M < 0 || K < 0 || N < 0 || K % 16 != 0) return -2;
    int status = 0;
    float a = oracle_absmean(W, M * K, &status);
    if (status != 0) return -1;
    *alpha = a;
    int8_t* codes = (int8_t*)malloc((size_t)(M * K > 0 ? M * K : 1));
    if (!codes) return -2;
    oracle_ternarize(W, M * K, a, codes);
    oracle_pack(codes, M, K, packed);
    oracle_quant_act(x, N, K, q, amax, qsum);
    oracle_matmul_i32(codes, M, K, q, N, acc);
    oracle_rescale(acc, N, M, a, amax, y);
    free(codes);
    return 0;
}
