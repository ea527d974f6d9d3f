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
 *            (H = 14, the headroom between the block-max code T = 112 and the largest
 *            finite code 126); otherwise m is kept
 *     k_b    per 64-key block b with block max mu_b:
 *            t = fmaf(mu_b, a, -m);  k_b = clamp(floor(-t / 8), KMIN, KMAX), KMIN = 0,
 *            KMAX = 16 (a block whose max sits below m by 8 k_b or more is lifted by
 *            2^k_b, so its maximum codes into (T - 8, T])
 *     code   the multiply-add, saturating to [0, 1] (negative codes clamp to 0):
 *              u = sat(fmaf(s, a / 256, (T + 8 k_b - m) / 256))
 *            and the integer conversion, one fma whose rounding at magnitude 2^23 is the
 *            round-to-nearest-even integer:  r = fmaf(u, 256, 1.5 * 2^23);
 *            byte = low 8 bits of r  (at most T + H = 126: never the NaN code 127)
 *     value  decode(byte) ~ 2^((a s - m)/8) * 2^(T/8 - 7 + k_b); the matrix instruction
 *            applies 2^-(T/8 - 7 + k_b) per (row, 64-key block) through UE8M0 scale
 *            factors, so a score at the reference weighs 1
 *     l      l <- alpha l + sum_j decode(byte_j) 2^-(T/8-7+k_b(j));   O likewise with v_j
 *     alpha  2^((m_old - m_new)/8) when m is raised (0 on the first tile)
 *   final:   o = O * dv / l,  lse = ln 2 * (m / 8 + log2 l)
 * Masked scores are -inf: their code is 0.  A fully masked block gets k_b = KMAX (its
 * codes are all 0, so its scale multiplies zeros).
 *
 * The eager reading (the reference follows the running maximum on every tile, H = 0, with
 * block maxima at T = 120 as first proposed for this method) is the other plain reading of
 * the pages; every function taking (top, headroom, kmin) accepts any reading (T, H, KMIN)
 * with T + H <= 126, and the functions without those arguments use the one above.  The
 * tests compare the two readings' accuracy.
 *
 * Build: gcc -O2 -ffp-contract=off -fno-fast-math -shared -fPIC (every a*b+c here is
 * written as the operation it is; the compiler must not fuse or reorder them).
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define LEANP_MAGIC 12582912.0f /* 1.5 * 2^23 */
#define LEANP_TOP 112          /* T: a block maximum codes into (T - 8, T] */
#define LEANP_HEADROOM 14      /* H: codes the tile max may exceed the reference by */
#define LEANP_KMIN 0           /* blocks above the reference keep k_b = 0 */

/* the reading the functions without reading arguments use */
int leanp_reading_top(void) { return LEANP_TOP; }
int leanp_reading_headroom(void) { return LEANP_HEADROOM; }
int leanp_reading_kmin(void) { return LEANP_KMIN; }

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

/* reference max in code units after seeing a tile whose raw-score maximum is mu_tile.
 * headroom: how far (in codes) the tile maximum may rise above the reference before the
 * reference is raised -- LEANP_HEADROOM for the lazy reading, 0 for the eager one (the
 * reference follows the running maximum on every tile). */
int leanp_update_max_ex(float mu_tile, float a, int m_old, int m_valid, int headroom) {
    if (isinf(mu_tile) && mu_tile < 0) return m_old;  /* no visible key in the tile */
    float prod = a * mu_tile;                          /* one float32 rounding */
    int cand = (int)ceilf(prod);
    if (!m_valid) return cand;
    return cand > m_old + headroom ? cand : m_old;
}

int leanp_update_max(float mu_tile, float a, int m_old, int m_valid) {
    return leanp_update_max_ex(mu_tile, a, m_old, m_valid, LEANP_HEADROOM);
}

/* power-of-two shift of one 64-key block: floor(-t/8) clamped to [kmin, kmax] */
int leanp_kshift_ex(float mu_b, float a, int m, int kmin, int kmax) {
    if (isinf(mu_b) && mu_b < 0) return kmax;          /* fully masked block */
    float t = fmaf(mu_b, a, -(float)m);
    float g = -t * 0.125f;                             /* exact */
    if (g >= (float)kmax) return kmax;
    float f = floorf(g);
    if (f <= (float)kmin) return kmin;
    return (int)f;
}

int leanp_kshift(float mu_b, float a, int m, int kmax) {
    return leanp_kshift_ex(mu_b, a, m, LEANP_KMIN, kmax);
}

/* code of one score given the block shift; top = code of a block maximum at the
 * reference (LEANP_TOP in the lazy reading, 120 in the eager one) */
uint8_t leanp_code_ex(float s, float a, int m, int kb, int top) {
    const float inv256 = 0.00390625f;
    float c = (float)(top + 8 * kb - m) * inv256;      /* exact: small integer / 256 */
    float u = fmaf(s, a * inv256, c);                  /* a / 256 exact */
    if (!(u > 0.0f)) u = 0.0f;                         /* saturate (NaN, -inf, <= 0 -> 0) */
    if (u > 1.0f) u = 1.0f;
    float r = fmaf(u, 256.0f, LEANP_MAGIC);
    uint32_t bits;
    memcpy(&bits, &r, 4);
    return (uint8_t)(bits & 0xFF);
}

uint8_t leanp_code(float s, float a, int m, int kb) {
    return leanp_code_ex(s, a, m, kb, LEANP_TOP);
}

/*
 * Encode one row of one key tile.  s: n raw scores (n a multiple of 64, -inf = masked),
 * m: the running max already updated with this tile.  Writes n codes and n/64 shifts.
 */
/* kshift holds k_b as a signed byte */
static void encode_row_tile_top(const float* s, int n, float a, int m, int kmin, int kmax,
                                int top, uint8_t* codes, int8_t* kshift) {
    for (int b = 0; b < n / 64; ++b) {
        float mu = -INFINITY;
        for (int j = 0; j < 64; ++j) mu = fmaxf(mu, s[b * 64 + j]);
        int kb = leanp_kshift_ex(mu, a, m, kmin, kmax);
        kshift[b] = (int8_t)kb;
        for (int j = 0; j < 64; ++j) codes[b * 64 + j] = leanp_code_ex(s[b * 64 + j], a, m, kb, top);
    }
}

void leanp_encode_row_tile(const float* s, int n, float a, int m, int kmax,
                           uint8_t* codes, int8_t* kshift) {
    encode_row_tile_top(s, n, a, m, LEANP_KMIN, kmax, LEANP_TOP, codes, kshift);
}

/*
 * Replay the kernel's per-row state machine over a row of raw scores, tile by tile in
 * ascending key order, and return codes, shifts and the reference max used per tile.
 *   s       [ntiles * tile] raw scores of one query row (-inf where masked)
 *   codes   [ntiles * tile] out, kshift [ntiles * tile / 64] out (signed), mref [ntiles] out
 * Tiles with no visible key are skipped (their codes are 0 and shifts KMAX).
 */
void leanp_encode_row_ex(const float* s, int ntiles, int tile, float a, int kmax, int top,
                         int headroom, int kmin, uint8_t* codes, int8_t* kshift, int* mref) {
    int m = 0, m_valid = 0;
    for (int t = 0; t < ntiles; ++t) {
        const float* st = s + (size_t)t * tile;
        float mu = -INFINITY;
        for (int j = 0; j < tile; ++j) mu = fmaxf(mu, st[j]);
        m = leanp_update_max_ex(mu, a, m, m_valid, headroom);
        if (!(isinf(mu) && mu < 0)) m_valid = 1;
        mref[t] = m_valid ? m : 0;
        if (!m_valid) {
            memset(codes + (size_t)t * tile, 0, tile);
            for (int b = 0; b < tile / 64; ++b) kshift[(size_t)t * tile / 64 + b] = (int8_t)kmax;
            continue;
        }
        encode_row_tile_top(st, tile, a, m, kmin, kmax, top, codes + (size_t)t * tile,
                            kshift + (size_t)t * tile / 64);
    }
}

void leanp_encode_row(const float* s, int ntiles, int tile, float a, int kmax,
                      uint8_t* codes, int8_t* kshift, int* mref) {
    leanp_encode_row_ex(s, ntiles, tile, a, kmax, LEANP_TOP, LEANP_HEADROOM, LEANP_KMIN, codes,
                        kshift, mref);
}

/*
 * End-to-end tile driver for one query row: from the row's raw scores (float32) and the
 * value rows (float64, already dequantised), the lean-P output row and lse, under the
 * reading (top, headroom, kmin) -- the one above is (120, 16, -2); the eager reading is
 * (120, 0, 0).
 *   s [S_k] raw scores (-inf masked), v [S_k * dv] dequantised values (row-major).
 * The products and sums of this step are formed in float64 (the tensor core's float32
 * accumulation order is not specified), so this predicts the kernel within float32
 * accumulation error, not bit for bit.  The weight of a code is
 * decode(byte) 2^-(top/8 - 7 + k_b), so a score at the reference weighs 1.
 */
void leanp_attention_row_ex(const float* s, int S_k, int tile, const double* v, int dv,
                            float a, int kmax, int top, int headroom, int kmin,
                            double* o_out, double* lse_out) {
    int ntiles = (S_k + tile - 1) / tile;
    double acc[1024];
    double l = 0.0;
    int m = 0, m_valid = 0;
    float buf[512];
    uint8_t codes[512];
    int8_t ks[8];
    const double unit = ldexp(1.0, -(top / 8 - 7));
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
        int m_new = leanp_update_max_ex(mu, a, m, m_valid, headroom);
        double alpha = m_valid ? exp2((double)(m - m_new) / 8.0) : 0.0;
        m = m_new;
        m_valid = 1;
        encode_row_tile_top(buf, n, a, m, kmin, kmax, top, codes, ks);
        l *= alpha;
        for (int d = 0; d < dv; ++d) acc[d] *= alpha;
        for (int j = 0; j < n; ++j) {
            int key = t * tile + j;
            if (key >= S_k || codes[j] == 0) continue;
            double w = leanp_e4m3_decode(codes[j]) * unit * ldexp(1.0, -ks[j / 64]);
            l += w;
            for (int d = 0; d < dv; ++d) acc[d] += w * v[(size_t)key * dv + d];
        }
    }
    for (int d = 0; d < dv; ++d) o_out[d] = acc[d] / l;
    *lse_out = log(2.0) * ((double)m / 8.0 + log2(l));
}

void leanp_attention_row(const float* s, int S_k, int tile, const double* v, int dv,
                         float a, int kmax, double* o_out, double* lse_out) {
    leanp_attention_row_ex(s, S_k, tile, v, dv, a, kmax, LEANP_TOP, LEANP_HEADROOM, LEANP_KMIN,
                           o_out, lse_out);
}

/*
 * Exact-P ablation ([ZYFA-mb] "Como o motor de atenção FP8 da Zyphra funciona" contrasts
 * lean P with "exact P", the probabilities formed with an exponential and then rounded to
 * FP8).  Reading: same reference max m and block shifts k_b as lean P; the value written
 * is e4m3_rn(2^x) with the float32 exponent
 *     x = fmaf(s, a / 8, (T - 56 + 8 k_b - m) / 8)   (a / 8 and the constant are exact)
 * so that 2^x = 2^((a s - m)/8) 2^(T/8 - 7 + k_b), the value whose log-linear code lean P
 * writes (a score at the reference gives 2^(T/8 - 7) with k_b = 0).  This function forms
 * x for n scores; the exponential and the e4m3 rounding are done by the caller
 * (oracle/leanp.py) in float64 and with the table codec.
 */
void leanp_exact_arg(const float* s, int n, float a, int m, int kb, float* x) {
    const float a8 = a * 0.125f;
    const float c = (float)(LEANP_TOP - 56 + 8 * kb - m) * 0.125f;
    for (int i = 0; i < n; ++i) x[i] = fmaf(s[i], a8, c);
}
