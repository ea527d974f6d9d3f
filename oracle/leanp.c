/*
 * Lean-P / power-of-two block-scale emulator, plain C, bit level.
 * TEST INFRASTRUCTURE ONLY (see oracle/__init__.py): only the tests, the smoke check and
 * the bench's CPU-baseline leg load this file's library.  It shares no code with the CUDA
 * path and includes nothing from it.
 *
 * What the pages say ([ZYFA-mb] "Como o motor de atenção FP8 da Zyphra funciona";
 * [ZYFA-pt] "Como o ZYFA funciona?", cut off at the first technique; [ZYFA-fr] "Ce que
 * couvrent les noyaux"):
 *   - each FP8 probability is produced by one multiply-add and one integer conversion
 *     that yields the FP8 bit pattern, exploiting the bit structure of the format, with
 *     no exponential;
 *   - each 64-key block is scaled by a power of two before the FP8 rounding, and the
 *     scaled matrix instruction removes that factor;
 *   - the row normaliser is the sum of the *rounded* probabilities, formed by one extra
 *     matrix instruction per block.
 *
 * Reading (the plainest one the pages support; all arithmetic float32 with one rounding
 * per operation, fmaf = fused multiply-add with a single rounding):
 *   The e4m3 code n = 8e + m (exponent field e, mantissa m) decodes to about
 *   2^(n/8 - 7) (the logarithm of 1 + m/8 taken as m/8: Mitchell 1962), so a code
 *   linear in the score approximates the exponential (the exponential-by-integer idea of
 *   Schraudolph 1999).  With a = 8 log2(e) * scale * dq * dk (code units per raw score
 *   unit), per row and per 128-key tile in ascending key order:
 *     m      reference max in code units, an integer, raised lazily:
 *            cand = ceil(float32(a * mu_tile)) (mu_tile = tile max of the raw scores);
 *            m = cand on the first tile, afterwards m = cand only if cand > m + H
 *            (H = 14, the headroom between the block-max code 112 and the largest
 *            finite code 126); otherwise m is kept
 *     k_b    per 64-key block b with block max mu_b:
 *            t = fmaf(mu_b, a, -m);  k_b = clamp(floor(-t / 8), 0, KMAX)
 *            (a block whose max sits below m by 8 k_b or more is lifted by 2^k_b)
 *     code   the multiply-add, saturating to [0, 1] (negative codes clamp to 0):
 *              u = sat(fmaf(s, a / 256, (112 + 8 k_b - m) / 256))
 *            and the integer conversion, one fma whose rounding at magnitude 2^23 is the
 *            round-to-nearest-even integer:  r = fmaf(u, 256, 1.5 * 2^23);
 *            byte = low 8 bits of r  (at most 126: never the NaN code 127)
 *     value  decode(byte) ~ 2^((a s - m)/8) * 2^(7 + k_b); the matrix instruction
 *            applies 2^-(7 + k_b) per (row, 64-key block) through UE8M0 scale factors
 *     l      l <- alpha l + sum_j decode(byte_j) 2^-(7+k_b(j));   O likewise with v_j
 *     alpha  2^((m_old - m_new)/8) when m is raised (0 on the first tile)
 *   final:   o = O * dv / l,  lse = ln 2 * (m / 8 + log2 l)
 * Masked scores are -inf: their code is 0.  A fully masked block gets k_b = KMAX (its
 * codes are all 0, so its scale multiplies zeros).
 *
 * Build: gcc -O2 -ffp-contract=off -fno-fast-math -shared -fPIC (every a*b+c here is
 * written as the operation it is; the compiler must not fuse or reorder them).
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define LEANP_MAGIC 12582912.0f /* 1.5 * 2^23 */
#define LEANP_TOP 112          /* code of a block maximum at the reference */
#define LEANP_HEADROOM 14      /* 126 - LEANP_TOP */

/* ---- e4m3fn decode by the format definition (independent of the Python codec) ---- */
double leanp_e4m3_decode(uint8_t c) {
    int e = (c >> 3) & 15, m = c & 7;
    double mag;
    if ((c & 0x7F) == 0x7F) return NAN;
    if (e == 0) mag = ldexp((double)m, -9);
    else mag = ldexp(1.0 + m / 8.0, e - 7);
    return (c & 0x80) ? -mag : mag;
}

/* exposed for the tests' exact-rounding pin */
float leanp_fmaf(float x, float y, float z) { return fmaf(x, y, z); }

/* reference max in code units after seeing a tile whose raw-score maximum is mu_tile */
int leanp_update_max(float mu_tile, float a, int m_old, int m_valid) {
    if (isinf(mu_tile) && mu_tile < 0) return m_old;  /* no visible key in the tile */
    float prod = a * mu_tile;                          /* one float32 rounding */
    int cand = (int)ceilf(prod);
    if (!m_valid) return cand;
    return cand > m_old + LEANP_HEADROOM ? cand : m_old;
}

/* power-of-two shift of one 64-key block */
int leanp_kshift(float mu_b, float a, int m, int kmax) {
    if (isinf(mu_b) && mu_b < 0) return kmax;          /* fully masked block */
    float t = fmaf(mu_b, a, -(float)m);
    float g = -t * 0.125f;                             /* exact */
    if (g >= (float)kmax) return kmax;
    float f = floorf(g);
    if (f <= 0.0f) return 0;
    return (int)f;
}

/* code of one score given the block shift */
uint8_t leanp_code(float s, float a, int m, int kb) {
    const float inv256 = 0.00390625f;
    float c = (float)(LEANP_TOP + 8 * kb - m) * inv256; /* exact: small integer / 256 */
    float u = fmaf(s, a * inv256, c);                  /* a / 256 exact */
    if (!(u > 0.0f)) u = 0.0f;                         /* saturate (NaN, -inf, <= 0 -> 0) */
    if (u > 1.0f) u = 1.0f;
    float r = fmaf(u, 256.0f, LEANP_MAGIC);
    uint32_t bits;
    memcpy(&bits, &r, 4);
    return (uint8_t)(bits & 0xFF);
}

/*
 * Encode one row of one key tile.  s: n raw scores (n a multiple of 64, -inf = masked),
 * m: the running max already updated with this tile.  Writes n codes and n/64 shifts.
 */
void leanp_encode_row_tile(const float* s, int n, float a, int m, int kmax,
                           uint8_t* codes, uint8_t* kshift) {
    for (int b = 0; b < n / 64; ++b) {
        float mu = -INFINITY;
        for (int j = 0; j < 64; ++j) mu = fmaxf(mu, s[b * 64 + j]);
        int kb = leanp_kshift(mu, a, m, kmax);
        kshift[b] = (uint8_t)kb;
        for (int j = 0; j < 64; ++j) codes[b * 64 + j] = leanp_code(s[b * 64 + j], a, m, kb);
    }
}

/*
 * Replay the kernel's per-row state machine over a row of raw scores, tile by tile in
 * ascending key order, and return codes, shifts and the reference max used per tile.
 *   s       [ntiles * tile] raw scores of one query row (-inf where masked)
 *   codes   [ntiles * tile] out, kshift [ntiles * tile / 64] out, mref [ntiles] out
 * Tiles with no visible key are skipped (their codes are 0 and shifts KMAX).
 */
void leanp_encode_row(const float* s, int ntiles, int tile, float a, int kmax,
                      uint8_t* codes, uint8_t* kshift, int* mref) {
    int m = 0, m_valid = 0;
    for (int t = 0; t < ntiles; ++t) {
        const float* st = s + (size_t)t * tile;
        float mu = -INFINITY;
        for (int j = 0; j < tile; ++j) mu = fmaxf(mu, st[j]);
        m = leanp_update_max(mu, a, m, m_valid);
        if (!(isinf(mu) && mu < 0)) m_valid = 1;
        mref[t] = m_valid ? m : 0;
        if (!m_valid) {
            memset(codes + (size_t)t * tile, 0, tile);
            for (int b = 0; b < tile / 64; ++b) kshift[(size_t)t * tile / 64 + b] = (uint8_t)kmax;
            continue;
        }
        leanp_encode_row_tile(st, tile, a, m, kmax, codes + (size_t)t * tile,
                              kshift + (size_t)t * tile / 64);
    }
}

/*
 * End-to-end tile driver for one query row: from the row's raw scores (float32) and the
 * value rows (float64, already dequantised), the lean-P output row and lse.
 *   s [S_k] raw scores (-inf masked), v [S_k * dv] dequantised values (row-major),
 *   scale_nat = softmax scale * dq * dk (natural units per raw score unit) for lse.
 * The products and sums of this step are formed in float64 (the tensor core's float32
 * accumulation order is not specified), so this predicts the kernel within float32
 * accumulation error, not bit for bit.
 */
void leanp_attention_row(const float* s, int S_k, int tile, const double* v, int dv,
                         float a, int kmax, double* o_out, double* lse_out) {
    int ntiles = (S_k + tile - 1) / tile;
    double acc[1024];
    double l = 0.0;
    int m = 0, m_valid = 0;
    float buf[512];
    uint8_t codes[512], ks[8];
    for (int d = 0; d < dv; ++d) acc[d] = 0.0;
    for (int t = 0; t < ntiles; ++t) {
        int n = tile;
        for (int j = 0; j < n; ++j) {
            int key = t * tile + j;
            buf[j] = key < S_k ? s[key] : -INFINITY;
        }
        float mu = -INFINITY;
        for (int j = 0; j < n; ++j) mu = fmaxf(mu, buf[j]);
        if (isinf(mu) && mu < 0) continue;
        int m_new = leanp_update_max(mu, a, m, m_valid);
        double alpha = m_valid ? exp2((double)(m - m_new) / 8.0) : 0.0;
        m = m_new;
        m_valid = 1;
        leanp_encode_row_tile(buf, n, a, m, kmax, codes, ks);
        l *= alpha;
        for (int d = 0; d < dv; ++d) acc[d] *= alpha;
        for (int j = 0; j < n; ++j) {
            int key = t * tile + j;
            if (key >= S_k || codes[j] == 0) continue;
            double w = leanp_e4m3_decode(codes[j]) * ldexp(1.0, -(7 + ks[j / 64]));
            l += w;
            for (int d = 0; d < dv; ++d) acc[d] += w * v[(size_t)key * dv + d];
        }
    }
    for (int d = 0; d < dv; ++d) o_out[d] = acc[d] / l;
    *lse_out = log(2.0) * ((double)m / 8.0 + log2(l));
}

/*
 * Exact-P ablation ([ZYFA-mb] "Como o motor de atenção FP8 da Zyphra funciona" contrasts
 * lean P with "exact P", the probabilities formed with an exponential and then rounded to
 * FP8).  Reading: same reference max m and block shifts k_b as lean P; the value written
 * is e4m3_rn(2^x) with the float32 exponent
 *     x = fmaf(s, a / 8, (8 (7 + k_b) - m) / 8)      (a / 8 and the constant are exact)
 * so that 2^x = 2^((a s - m)/8) 2^(7 + k_b), the quantity lean P approximates.  This
 * function forms x for n scores; the exponential and the e4m3 rounding are done by the
 * caller (oracle/leanp.py) in float64 and with the table codec.
 */
void leanp_exact_arg(const float* s, int n, float a, int m, int kb, float* x) {
    const float a8 = a * 0.125f;
    const float c = (float)(8 * (7 + kb) - m) * 0.125f;
    for (int i = 0; i < n; ++i) x[i] = fmaf(s[i], a8, c);
}

