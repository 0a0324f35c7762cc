/*
 * bitnet_oracle.c -- plain, slow, scalar CPU oracle for the BitNet b1.58
 * BitLinear path.  TEST INFRASTRUCTURE ONLY: it is loaded by the tests, by
 * the smoke check and by the benchmark's CPU-baseline leg, never by the
 * product library.  It shares no code, header or constant table with the
 * CUDA path.
 *
 * Every function states the passage it restates.  Page names used below:
 *   [KeyTech]  "Key Technologies Enabling the BitNET Family" (edgeai-for-
 *              beginners, BitNET family module): "Advanced Quantization
 *              Methodologies" (absmean ternary weights, per-token absmax
 *              8-bit activations) and "Architectural Innovations" (BitLinear,
 *              RMSNorm, no bias).
 *   [Gartu]    "BitNet / Ternary / Binary -- Les LLMs 1-bit" (brain.gartu.xyz),
 *              section "Apercu de l'entrainement d'un BitLinear": the
 *              BitLinear forward (beta = mean|w|, round(w/(beta+1e-8)),
 *              clamp to [-1, 1], F.linear).
 *   [HN-b158]  Hacker News thread on the b1.58 paper (srizon.com reader):
 *              the ternary dot product as "sum of activations where the
 *              weight is +1 minus sum where it is -1", and "activations are
 *              int8 during inference".
 *   [KeyTech] also gives the feed-forward activation (squared ReLU, the
 *              ReLU^2 gate below).
 *   [Gartu] also names the binary variant, BitNet b1 ("BitNet b1 (binaire)":
 *              weights exactly +1 or -1), restated in orc_binarise below.
 *   [Notes]    "BitNet Technical Notes" (afondiel.github.io), "System
 *              Design" / Appendix glossary: bit-packing at 2 bits per
 *              ternary weight.
 *
 * Floating point: every float operation is a single IEEE-754 binary32 or
 * binary64 operation in round-to-nearest-even.  The file must be compiled
 * without fast-math and with -ffp-contract=off (the build script does so).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* Exact sum of |W| (absmean numerator).                                    */
/*                                                                          */
/* [KeyTech] "ternary weight quantization using absmean"; [Gartu] computes   */
/* beta = w.abs().mean().  The mean is a plain definition, so the oracle     */
/* computes it exactly: the real-number sum of |W| is accumulated without    */
/* rounding in a wide fixed-point register (a Kulisch accumulator) whose     */
/* least significant bit is 2^-149, the smallest binary32 step, and is then  */
/* rounded once to binary64.                                                */
/* ------------------------------------------------------------------------ */

/* 2^-149 .. 2^(127+1+64): 12 limbs of 32 bits = 384 bits is ample for any  */
/* count of elements below 2^60.                                           */
#define ORC_LIMBS 12

static void kulisch_add(uint32_t acc[ORC_LIMBS], uint32_t mant, int shift)
{
    /* add mant * 2^shift (in units of 2^-149) */
    int limb = shift / 32;
    int off = shift % 32;
    uint64_t v = (uint64_t)mant << off;          /* at most 24+31 = 55 bits */
    uint64_t carry = 0;
    for (int i = limb; i < ORC_LIMBS; ++i) {
        uint64_t add = (v & 0xffffffffu) + carry;
        uint64_t s = (uint64_t)acc[i] + add;
        acc[i] = (uint32_t)s;
        carry = s >> 32;
        v >>= 32;
        if (v == 0 && carry == 0) break;
    }
}

/* Round the fixed-point value acc * 2^-149 to the nearest binary64.        */
static double kulisch_to_double(const uint32_t acc[ORC_LIMBS])
{
    int top = -1;
    for (int i = ORC_LIMBS - 1; i >= 0; --i)
        if (acc[i]) { top = i; break; }
    if (top < 0) return 0.0;
    int hb = 31;
    while (!((acc[top] >> hb) & 1u)) --hb;
    int p = top * 32 + hb;                         /* highest set bit index */
    if (p < 64) {
        uint64_t lo = (uint64_t)acc[0] | ((uint64_t)acc[1] << 32);
        /* integer below 2^64: one correctly rounded conversion */
        return ldexp((double)lo, -149);
    }
    /* take bits [p-63, p] as a 64-bit integer; OR a sticky bit for any   */
    /* nonzero bit below; 64 > 53 + 2, so one conversion rounds correctly */
    int lo_bit = p - 63;
    uint64_t word = 0;
    for (int b = 0; b < 64; ++b) {
        int bit = lo_bit + b;
        if ((acc[bit / 32] >> (bit % 32)) & 1u) word |= (uint64_t)1 << b;
    }
    int sticky = 0;
    for (int bit = 0; bit < lo_bit && !sticky; ++bit)
        if ((acc[bit / 32] >> (bit % 32)) & 1u) sticky = 1;
    if (sticky) word |= 1u;
    return ldexp((double)word, lo_bit - 149);
}

/* Correctly rounded binary64 value of sum_i |W[i]| (W finite).             */
double orc_abs_sum(const float *W, int64_t n)
{
    uint32_t acc[ORC_LIMBS];
    memset(acc, 0, sizeof acc);
    for (int64_t i = 0; i < n; ++i) {
        uint32_t bits;
        memcpy(&bits, &W[i], 4);
        bits &= 0x7fffffffu;                       /* |w| */
        uint32_t e = bits >> 23;
        uint32_t m = bits & 0x7fffffu;
        if (e == 0) {                              /* zero or subnormal: m * 2^-149 */
            if (m) kulisch_add(acc, m, 0);
        } else {                                   /* (2^23 + m) * 2^(e-150) */
            kulisch_add(acc, m | 0x800000u, (int)e - 1);
        }
    }
    return kulisch_to_double(acc);
}

/* gamma = mean |W| over all N*K entries, [Gartu] beta = w.abs().mean().   */
/* Reading: the exact sum rounded to binary64, divided by N*K in binary64, */
/* rounded to binary32.  An all-zero W gives gamma = 0.                    */
float orc_gamma(const float *W, int64_t n)
{
    if (n <= 0) return 0.0f;
    double s = orc_abs_sum(W, n);
    double mean = s / (double)n;
    return (float)mean;
}

/* ------------------------------------------------------------------------ */
/* Ternarisation.  [Gartu] w_quant = clamp(round(w / (beta + 1e-8)), -1, 1); */
/* torch.round rounds half to even, which is rintf in the default mode.      */
/* The arithmetic is binary32, as in the page's float32 PyTorch code:        */
/* d = gamma + eps rounded to binary32, then one IEEE division.              */
/* ------------------------------------------------------------------------ */
void orc_ternarise(const float *W, int64_t n, float gamma, float eps, int8_t *Wq)
{
    float d = gamma + eps;
    for (int64_t i = 0; i < n; ++i) {
        float t = W[i] / d;
        float r = rintf(t);
        /* r is integer-valued, so clamping to [-1, 1] is a three-way test; */
        /* a NaN quotient (0/0 when gamma + eps == 0) compares false: 0.     */
        int8_t q;
        if (r >= 1.0f) q = 1;
        else if (r <= -1.0f) q = -1;
        else q = 0;
        Wq[i] = q;
    }
}

/* ------------------------------------------------------------------------ */
/* 2-bit packing.  [Notes] "bit-packing (e.g., 2 bits per ternary weight)".  */
/* The pages fix no encoding or layout; this library's layout is:            */
/*   code c = q + 1  (0 -> -1, 1 -> 0, 2 -> +1; 3 is never written),         */
/*   row n occupies bytes [n*K/4, (n+1)*K/4),                                */
/*   byte j (0..3) of the 4-byte group g of the row holds the weights        */
/*   k = 16g + 4s + j for s = 0..3, weight s in bits [2s, 2s+1].             */
/* Written byte by byte here, with no word arithmetic.                       */
/* Returns the number of entries of Wq outside {-1, 0, 1}; such entries are  */
/* stored as code 3.                                                         */
/* ------------------------------------------------------------------------ */
int64_t orc_pack(const int8_t *Wq, int64_t N, int64_t K, uint8_t *Wp)
{
    int64_t bad = 0;
    int64_t row_bytes = K / 4;
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t g = 0; g < K / 16; ++g) {
            for (int j = 0; j < 4; ++j) {
                unsigned byte = 0;
                for (int s = 0; s < 4; ++s) {
                    int64_t k = 16 * g + 4 * s + j;
                    int q = Wq[n * K + k];
                    unsigned c;
                    if (q >= -1 && q <= 1) c = (unsigned)(q + 1);
                    else { c = 3u; ++bad; }
                    byte |= c << (2 * s);
                }
                Wp[n * row_bytes + 4 * g + j] = (uint8_t)byte;
            }
        }
    }
    return bad;
}

/* Inverse of orc_pack.  Code 3 decodes to 0 and is counted.                */
int64_t orc_unpack(const uint8_t *Wp, int64_t N, int64_t K, int8_t *Wq)
{
    int64_t bad = 0;
    int64_t row_bytes = K / 4;
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t k = 0; k < K; ++k) {
            int64_t g = k / 16;
            int s = (int)((k % 16) / 4);
            int j = (int)(k % 4);
            unsigned byte = Wp[n * row_bytes + 4 * g + j];
            unsigned c = (byte >> (2 * s)) & 3u;
            if (c == 3u) { ++bad; Wq[n * K + k] = 0; }
            else Wq[n * K + k] = (int8_t)((int)c - 1);
        }
    }
    return bad;
}

/* ------------------------------------------------------------------------ */
/* Per-token absmax int8 activation quantisation.                           */
/* [KeyTech] "8-bit activation quantization using absmax quantization per-  */
/* token"; [HN-b158] activations are int8 at inference.  Per row m:          */
/*   a   = max(max_k |t_k|, floor_eps)        (floor_eps guards a zero row)  */
/*   q_k = clamp(rint(t_k * (127 / a)), -128, 127)                           */
/*   s   = a / 127                 (x ~= s * q)                              */
/* with t = x when no norm gain is given.                                    */
/*                                                                          */
/* Optional RMSNorm prologue ([KeyTech] "uses RMSNorm for normalization",    */
/* no bias): RMSNorm(x)_k = x_k * r * g_k with r = 1/sqrt(mean_k x_k^2 +     */
/* rms_eps).  Since r > 0 is common to the whole row it cancels in           */
/* u_k * 127 / max|u|, so the codes are taken from t_k = x_k * g_k and r     */
/* enters only the scale: s = r * a / 127 (r and s formed in binary64,       */
/* s rounded once to binary32).                                              */
/* Also returns xsum[m] = sum_k q_k (exact int32).                           */
/* ------------------------------------------------------------------------ */
void orc_quant_act(const float *x, int64_t M, int64_t K, const float *gain,
                   float rms_eps, float floor_eps,
                   int8_t *xq, float *scale, int32_t *xsum)
{
    for (int64_t m = 0; m < M; ++m) {
        const float *row = x + m * K;
        float a = 0.0f;
        for (int64_t k = 0; k < K; ++k) {
            float t = gain ? row[k] * gain[k] : row[k];
            float at = fabsf(t);
            if (at > a) a = at;
        }
        if (a < floor_eps) a = floor_eps;
        float inv = 127.0f / a;
        int32_t s = 0;
        for (int64_t k = 0; k < K; ++k) {
            float t = gain ? row[k] * gain[k] : row[k];
            float v = rintf(t * inv);
            int q;
            if (v > 127.0f) q = 127;
            else if (v < -128.0f) q = -128;
            else q = (int)v;
            xq[m * K + k] = (int8_t)q;
            s += q;
        }
        xsum[m] = s;
        if (gain) {
            double ss = 0.0;
            for (int64_t k = 0; k < K; ++k) ss += (double)row[k] * (double)row[k];
            double r = 1.0 / sqrt(ss / (double)K + (double)rms_eps);
            scale[m] = (float)(r * (double)a / 127.0);
        } else {
            scale[m] = a / 127.0f;
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Integer contraction acc[m,n] = sum_k xq[m,k] * Wq[n,k].                   */
/* [Gartu] F.linear(x, w) computes x @ w^T; with int8 x and ternary w the    */
/* result is an exact integer.  Plain triple loop, int64 accumulation.       */
/* ------------------------------------------------------------------------ */
void orc_linear_i32(const int8_t *xq, int64_t M, int64_t K, const int8_t *Wq,
                    int64_t N, int32_t *acc)
{
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            int64_t s = 0;
            for (int64_t k = 0; k < K; ++k)
                s += (int64_t)xq[m * K + k] * (int64_t)Wq[n * K + k];
            acc[m * N + n] = (int32_t)s;
        }
}

/* Dequantised output y[m,n] = acc[m,n] * (gamma * s[m]) in binary32:       */
/* the weight scale gamma and the activation scale max|x|/127 undo the two  */
/* quantisers ([KeyTech] absmean and absmax quantisers).                    */
void orc_output(const int32_t *acc, int64_t M, int64_t N, float gamma,
                const float *scale, float *y)
{
    for (int64_t m = 0; m < M; ++m) {
        float sm = gamma * scale[m];
        for (int64_t n = 0; n < N; ++n)
            y[m * N + n] = (float)acc[m * N + n] * sm;
    }
}

/* ------------------------------------------------------------------------ */
/* Binary weights (BitNet b1).  [Gartu] "BitNet b1 (binaire)": every weight */
/* of the BitLinear layer is exactly +1 or -1.  The pages give no rule, so  */
/* the reading is the sign, ties (zero) to +1: W_b = +1 where W >= 0, else  */
/* -1 (a NaN compares false and gives -1).  The scale is the same absmean   */
/* beta = mean|W| as the ternary case (orc_gamma): sign(W) * mean|W| is the */
/* binary approximation of W with the least sum of squared errors.          */
/* ------------------------------------------------------------------------ */
void orc_binarise(const float *W, int64_t n, int8_t *Wb)
{
    for (int64_t i = 0; i < n; ++i) Wb[i] = (W[i] >= 0.0f) ? (int8_t)1 : (int8_t)-1;
}

/* 1-bit pack: bit 1 for +1, 0 for -1.  K is split into groups of 32       */
/* weights, one little-endian uint32 each (group g of row n at byte offset  */
/* n*K/8 + 4g); weight k = 32g + 4s + j (s in 0..7, j in 0..3) sits at bit  */
/* 8j + s, so (word >> s) & 0x01010101 holds the bits of k = 32g+4s .. +3    */
/* one per byte in order.  Values other than +-1 are stored as 0 (-1) and   */
/* counted.  Requires K % 32 == 0.                                          */
int64_t orc_pack_b1(const int8_t *Wb, int64_t N, int64_t K, uint8_t *Wp)
{
    int64_t bad = 0;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t g = 0; g < K / 32; ++g) {
            uint32_t word = 0;
            for (int s = 0; s < 8; ++s)
                for (int j = 0; j < 4; ++j) {
                    int8_t v = Wb[n * K + 32 * g + 4 * s + j];
                    if (v != 1 && v != -1) ++bad;
                    if (v == 1) word |= 1u << (8 * j + s);
                }
            uint8_t *o = Wp + n * (K / 8) + 4 * g;
            o[0] = (uint8_t)(word & 0xff);
            o[1] = (uint8_t)((word >> 8) & 0xff);
            o[2] = (uint8_t)((word >> 16) & 0xff);
            o[3] = (uint8_t)(word >> 24);
        }
    return bad;
}

void orc_unpack_b1(const uint8_t *Wp, int64_t N, int64_t K, int8_t *Wb)
{
    for (int64_t n = 0; n < N; ++n)
        for (int64_t g = 0; g < K / 32; ++g) {
            const uint8_t *b = Wp + n * (K / 8) + 4 * g;
            uint32_t word = (uint32_t)b[0] | ((uint32_t)b[1] << 8) | ((uint32_t)b[2] << 16) | ((uint32_t)b[3] << 24);
            for (int s = 0; s < 8; ++s)
                for (int j = 0; j < 4; ++j)
                    Wb[n * K + 32 * g + 4 * s + j] = ((word >> (8 * j + s)) & 1u) ? (int8_t)1 : (int8_t)-1;
        }
}

/* ------------------------------------------------------------------------ */
/* Base-3 packing ("BitNET Family", Memory Efficiency: 0.4 GB for the 2B     */
/* model, i.e. about 1.6 bits per weight; Hacker News thread (bitsplea.se):  */
/* "2 bits instead of 1.58").  Five ternary weights fit one byte            */
/* (3^5 = 243 <= 256): a byte holds sum_i c_i 3^i with codes c = q + 1.     */
/* Layout (this library's): K is cut into groups of 20 weights, one         */
/* little-endian uint32 each; byte j of group g holds the weights           */
/* k = 20g + 4i + j (i = 0..4, c_i the i-th base-3 digit), so digit i of the */
/* four bytes gives four consecutive weights.  Weights past K code as 1     */
/* (q = 0).  A row takes ceil(K / 80) * 16 bytes (whole 16-byte chunks).     */
/* Values outside {-1, 0, 1} are stored as code 1 and counted.               */
/* ------------------------------------------------------------------------ */
int64_t orc_t3_row_bytes(int64_t K) { return (K + 79) / 80 * 16; }

int64_t orc_pack_t3(const int8_t *Wq, int64_t N, int64_t K, uint8_t *Wp)
{
    int64_t bad = 0, rb = orc_t3_row_bytes(K);
    for (int64_t n = 0; n < N; ++n)
        for (int64_t g = 0; g < rb / 4; ++g)
            for (int j = 0; j < 4; ++j) {
                int v = 0, p3 = 1;
                for (int i = 0; i < 5; ++i) {
                    int64_t k = 20 * g + 4 * i + j;
                    int c = 1;
                    if (k < K) {
                        int q = Wq[n * K + k];
                        if (q >= -1 && q <= 1) c = q + 1;
                        else ++bad;
                    }
                    v += c * p3;
                    p3 *= 3;
                }
                Wp[n * rb + 4 * g + j] = (uint8_t)v;
            }
    return bad;
}

/* Inverse of orc_pack_t3 for k < K; bytes above 242 are invalid: counted,  */
/* their weights read as 0.                                                 */
int64_t orc_unpack_t3(const uint8_t *Wp, int64_t N, int64_t K, int8_t *Wq)
{
    int64_t bad = 0, rb = orc_t3_row_bytes(K);
    for (int64_t n = 0; n < N; ++n)
        for (int64_t g = 0; g < rb / 4; ++g)
            for (int j = 0; j < 4; ++j) {
                int v = Wp[n * rb + 4 * g + j];
                int valid = v <= 242;
                if (!valid && 20 * g + j < K) ++bad;
                for (int i = 0; i < 5; ++i) {
                    int64_t k = 20 * g + 4 * i + j;
                    int c = v % 3;
                    v /= 3;
                    if (k < K) Wq[n * K + k] = valid ? (int8_t)(c - 1) : (int8_t)0;
                }
            }
    return bad;
}

/* ------------------------------------------------------------------------ */
/* ReLU^2 gate of the feed-forward layers.  [KeyTech] "Architectural        */
/* Innovations": squared ReLU activations in the feed-forward layers.  The  */
/* down projection's input is the gate projection's output squared after    */
/* ReLU, times the up projection's output:                                  */
/*   t = (r * r) * u,  r = max(g, 0)                                        */
/* in binary32, one rounding per operation, in that order.  A NaN gate      */
/* counts as 0 (the comparison g > 0 is false).                             */
/* ------------------------------------------------------------------------ */
void orc_relu2_gate(const float *gate, const float *up, int64_t n, float *t)
{
    for (int64_t i = 0; i < n; ++i) {
        float g = gate[i];
        float r = (g > 0.0f) ? g : 0.0f;
        float rr = r * r;
        t[i] = rr * up[i];
    }
}

/* Output with the block's residual stream added (a Transformer feed-forward */
/* block adds its output to its input; the pages name only the gate):       */
/*   y[m,n] = resid[m,n] + (float)acc[m,n] * (gamma * s[m])                 */
/* binary32: the product rounded, then the sum rounded.                      */
void orc_output_resid(const int32_t *acc, int64_t M, int64_t N, float gamma,
                      const float *scale, const float *resid, float *y)
{
    for (int64_t m = 0; m < M; ++m) {
        float sm = gamma * scale[m];
        for (int64_t n = 0; n < N; ++n) {
            float prod = (float)acc[m * N + n] * sm;
            y[m * N + n] = resid[m * N + n] + prod;
        }
    }
}

/* binary32 -> bfloat16 bits, round to nearest, ties to even; NaN stays NaN */
void orc_to_bf16(const float *v, int64_t n, uint16_t *out)
{
    for (int64_t i = 0; i < n; ++i) {
        uint32_t u;
        memcpy(&u, &v[i], 4);
        if ((u & 0x7fffffffu) > 0x7f800000u) { out[i] = (uint16_t)((u >> 16) | 0x40u); continue; }
        uint32_t lsb = (u >> 16) & 1u;
        u += 0x7fffu + lsb;
        out[i] = (uint16_t)(u >> 16);
    }
}

/* Whole BitLinear forward for convenience: quantise x, contract, rescale.  */
void orc_bitlinear(const float *x, int64_t M, int64_t K, const int8_t *Wq,
                   int64_t N, float gamma, const float *gain, float rms_eps,
                   float floor_eps, float *y)
{
    int8_t *xq = (int8_t *)malloc((size_t)(M * K > 0 ? M * K : 1));
    float *sc = (float *)malloc((size_t)(M > 0 ? M : 1) * sizeof(float));
    int32_t *xs = (int32_t *)malloc((size_t)(M > 0 ? M : 1) * sizeof(int32_t));
    int32_t *acc = (int32_t *)malloc((size_t)(M * N > 0 ? M * N : 1) * sizeof(int32_t));
    orc_quant_act(x, M, K, gain, rms_eps, floor_eps, xq, sc, xs);
    orc_linear_i32(xq, M, K, Wq, N, acc);
    orc_output(acc, M, N, gamma, sc, y);
    free(xq); free(sc); free(xs); free(acc);
}
