/*
 * kvq oracle -- plain, slow, CPU reference for the quantized KV cache hot path.
 *
 * THIS IS TEST INFRASTRUCTURE.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load it.  The product library never links,
 * loads or calls anything in this directory, and this file includes nothing
 * from the product (no shared headers, tables or helpers).
 *
 * Built with:  gcc -O2 -std=c11 -fPIC -shared -ffp-contract=off -fno-fast-math
 * so that every float expression below is a sequence of correctly rounded
 * IEEE-754 binary32 / binary64 operations in the order written.
 *
 * Sources (web pages; cited by title and section):
 *  [COBRA]   "KV-COBRA splits the KV-cache budget per head -- Rank vs bit-width
 *             allocation" (learnaivisually.com explainer)
 *  [BEE]     "BeeLlama.cpp v0.4.0 发布：聚焦 KV cache 量化，新增 KVarN 与精度尾部机制"
 *             (taozi.news)
 *  [VBR]     "Introducing a new KV format: VBR (Variable Bit Rate)" (thread)
 *  [FORUM]   forum thread explaining decode attention and the memory-bandwidth
 *             bound (swe-vps threads?id=maurelius2)
 * Where the pages are silent this file takes a reading, stated at the code that
 * uses it and tagged R1, R2, ... so that one choice keeps one name wherever it
 * recurs (the GPU side carries the same tags).
 *
 * Every function here is pinned by CPU tests against something other than
 * itself (closed forms, exhaustive comparisons with numpy's float16, worked
 * examples, invariants).  No function is "parity unpinned".
 */
#include <stdint.h>
#include <string.h>
#include <math.h>
#include <stdlib.h>

#define D 128                      /* head_dim, fixed by every workload */

float orc_f16_to_f32(uint16_t h);

/* ------------------------------------------------------------------------- */
/* binary16 conversions, written out by hand (pinned exhaustively vs numpy)   */
/* ------------------------------------------------------------------------- */

/* Shift a non-negative integer right by s bits, rounding to nearest, ties to
 * even.  m < 2^25. */
static uint32_t shr_rne(uint32_t m, int s) {
    if (s <= 0) return m << (-s);
    if (s >= 26) return 0;
    uint32_t q = m >> s;
    uint32_t rem = m & ((1u << s) - 1u);
    uint32_t half = 1u << (s - 1);
    if (rem > half || (rem == half && (q & 1u))) q++;
    return q;
}

/* float -> binary16, round to nearest even (IEEE default). */
uint16_t orc_f16_rn(float f) {
    uint32_t x; memcpy(&x, &f, 4);
    uint32_t sign = (x >> 16) & 0x8000u;
    uint32_t ax = x & 0x7fffffffu;
    if (ax > 0x7f800000u) return (uint16_t)(sign | 0x7e00u);      /* NaN */
    if (ax >= 0x477ff000u) return (uint16_t)(sign | 0x7c00u);     /* >= 65520 -> inf */
    int e = (int)(ax >> 23);                                        /* biased fp32 exponent */
    uint32_t m = (ax & 0x7fffffu);
    if (e == 0) return (uint16_t)sign;                              /* fp32 subnormal: |f| < 2^-126 -> 0 */
    m |= 0x800000u;                                                 /* value = m * 2^(e-150) */
    /* fp16 value = h * 2^(he-25) for normals with he = e-112, or h * 2^-24 for subnormals */
    if (e >= 113) {
        /* normal fp16: keep 11 significant bits */
        uint32_t h = shr_rne(m, 13);                                /* 1024..2048 */
        uint32_t he = (uint32_t)(e - 112);
        /* h may have rounded up to 2048: carry into exponent */
        uint32_t bits = (he << 10) + (h - 1024u);
        return (uint16_t)(sign | bits);
    }
    /* subnormal fp16: units of 2^-24; m*2^(e-150) / 2^-24 = m * 2^(e-126) */
    uint32_t h = shr_rne(m, 126 - e);
    return (uint16_t)(sign | h);                                    /* h==1024 is the smallest normal */
}

/* float -> binary16, round toward -infinity (R5: the _1 minimum). */
uint16_t orc_f16_rd(float f) {
    uint16_t h = orc_f16_rn(f);
    uint32_t x; memcpy(&x, &f, 4);
    if ((x & 0x7fffffffu) > 0x7f800000u) return h;                 /* NaN */
    /* compare the rounded value with f; step down one ulp if it rounded up */
    float back = orc_f16_to_f32(h);
    if (back > f) {
        /* next binary16 toward -inf */
        if (h == 0x0000u) return 0x8001u;                            /* +0 -> -min subnormal */
        if (h & 0x8000u) return (uint16_t)(h + 1u);                  /* negative: magnitude up */
        return (uint16_t)(h - 1u);                                   /* positive: magnitude down */
    }
    return h;
}

float orc_f16_to_f32(uint16_t h) {
    uint32_t sign = ((uint32_t)h & 0x8000u) << 16;
    uint32_t e = (h >> 10) & 0x1fu;
    uint32_t m = h & 0x3ffu;
    float mag;
    if (e == 0x1f) {
        uint32_t bits = sign | 0x7f800000u | (m << 13);
        memcpy(&mag, &bits, 4);
        return mag;
    }
    if (e == 0) mag = ldexpf((float)m, -24);                         /* exact */
    else mag = ldexpf((float)(m | 0x400u), (int)e - 25);             /* exact */
    return sign ? -mag : mag;
}

/* bf16 -> fp32: a bf16 value is the upper half of a binary32 (sign, 8-bit
 * exponent, 7 fraction bits), so widening appends 16 zero bits.  Exact. */
float orc_bf16_to_f32(uint16_t h) {
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* A raw 16-bit row element (the plan's kv dtype: bf16 if nonzero, else fp16). */
static float raw_to_f32(uint16_t h, int bf16) { return bf16 ? orc_bf16_to_f32(h) : orc_f16_to_f32(h); }

void orc_f16_rn_array(const float* x, uint16_t* h, int64_t n) { for (int64_t i = 0; i < n; ++i) h[i] = orc_f16_rn(x[i]); }
void orc_f16_rd_array(const float* x, uint16_t* h, int64_t n) { for (int64_t i = 0; i < n; ++i) h[i] = orc_f16_rd(x[i]); }
void orc_f16_to_f32_array(const uint16_t* h, float* x, int64_t n) { for (int64_t i = 0; i < n; ++i) x[i] = orc_f16_to_f32(h[i]); }

/* ------------------------------------------------------------------------- */
/* Hadamard rotation [COBRA §Jargon "Hadamard rotation"; BEE §KVarN]          */
/* ------------------------------------------------------------------------- */

/* Sylvester construction: H_1 = [1], H_2n = [[H, H], [H, -H]].  Entry (i, j)
 * is (-1)^popcount(i & j).  Written out by the recursive definition. */
void orc_hadamard_matrix(int n, int8_t* H) {
    H[0] = 1;
    for (int m = 1; m < n; m *= 2) {
        for (int i = 0; i < m; ++i)
            for (int j = 0; j < m; ++j) {
                int8_t v = H[i * n + j];
                H[i * n + (j + m)] = v;
                H[(i + m) * n + j] = v;
                H[(i + m) * n + (j + m)] = (int8_t)-v;
            }
    }
}

/* c = fp32RN(1/sqrt(128)) (R: the normalisation of the rotation). */
float orc_hadamard_c(void) { return (float)(1.0 / sqrt((double)D)); }

/* y = H x / sqrt(128) in double: the orthonormal rotation, dense. */
void orc_rotate_dense(int64_t n_rows, const double* x, double* y) {
    static int8_t H[D * D];
    static int init = 0;
    if (!init) { orc_hadamard_matrix(D, H); init = 1; }
    const double s = 1.0 / sqrt((double)D);
    for (int64_t r = 0; r < n_rows; ++r) {
        const double* xr = x + r * D;
        double* yr = y + r * D;
        for (int i = 0; i < D; ++i) {
            double acc = 0.0;
            for (int j = 0; j < D; ++j) acc += (double)H[i * D + j] * xr[j];
            yr[i] = acc * s;
        }
    }
}

/* The rotation as it is computed on the quantize side (R8/R9 spec FWHT):
 * binary32, butterfly stages with half-width h = 1, 2, 4, ..., 64 in that
 * order; the pair (i, i+h) with bit h of i clear becomes (a+b, a-b); then
 * every element is multiplied by c.  Because each output of every stage is a
 * single correctly rounded add or subtract, any implementation that performs
 * the same stages in the same order produces identical bits. */
void orc_fwht_spec(int64_t n_rows, float* x) {
    const float c = orc_hadamard_c();
    for (int64_t r = 0; r < n_rows; ++r) {
        float* v = x + r * D;
        for (int h = 1; h < D; h *= 2)
            for (int i = 0; i < D; ++i)
                if ((i & h) == 0) {
                    float a = v[i], b = v[i + h];
                    v[i] = a + b;
                    v[i + h] = a - b;
                }
        for (int i = 0; i < D; ++i) v[i] = v[i] * c;
    }
}

/* ------------------------------------------------------------------------- */
/* Codecs [BEE §新增标准 KV cache 类型; config text for q4_0]                  */
/* ------------------------------------------------------------------------- */

/* Codec ids (shared numbering with the public header by value only). */
enum { C_F16 = 0, C_Q8_0, C_Q6_0, C_Q4_0, C_Q3_0, C_Q2_0,
       C_Q8_1, C_Q6_1, C_Q4_1, C_Q3_1, C_Q2_1, C_RANK = 11, C_Q5_0 = 12, C_Q5_1 = 13 };

static int codec_bits(int codec) {
    switch (codec) {
        case C_Q8_0: case C_Q8_1: return 8;
        case C_Q6_0: case C_Q6_1: return 6;
        case C_Q5_0: case C_Q5_1: return 5;
        case C_Q4_0: case C_Q4_1: return 4;
        case C_Q3_0: case C_Q3_1: return 3;
        case C_Q2_0: case C_Q2_1: return 2;
        default: return 16;
    }
}
static int codec_is_1(int codec) { return (codec >= C_Q8_1 && codec <= C_Q2_1) || codec == C_Q5_1; }

/* Bytes of one packed row (R7): codes for n values at b bits, plus fp16
 * scales.  For the rank variant n = r and the block is min(32, r). */
int orc_row_bytes(int codec, int r, int b, int* code_bytes, int* scale_bytes) {
    int n = (codec == C_RANK) ? r : D;
    int bits = (codec == C_RANK) ? b : codec_bits(codec);
    int blk = n < 32 ? n : 32;
    int nb = n / blk;
    *code_bytes = n * bits / 8;
    if (codec == C_F16) *scale_bytes = 0;
    else if (codec == C_RANK) *scale_bytes = 2 * nb;
    else *scale_bytes = codec_is_1(codec) ? 4 * nb : 2 * nb;
    return 0;
}

/* R1-R4: symmetric block quantizer ("_0"), qmax = 2^(b-1)-1, codes clamped to
 * [-2^(b-1), qmax], stored offset-binary u = code + 2^(b-1).  The scale is
 * computed in fp32, stored as fp16 (RNE), and codes are taken against the
 * stored scale. */
static void quant_block_sym(const float* x, int n, int bits, uint8_t* u, uint16_t* dh_out) {
    float amax = 0.0f;
    for (int j = 0; j < n; ++j) { float a = fabsf(x[j]); if (a > amax) amax = a; }
    const int qmax = (1 << (bits - 1)) - 1;
    const int qmin = -(1 << (bits - 1));
    float d = amax / (float)qmax;
    if (d > 65504.0f) d = 65504.0f;
    uint16_t dh = orc_f16_rn(d);
    float df = orc_f16_to_f32(dh);
    *dh_out = dh;
    if (df == 0.0f) { for (int j = 0; j < n; ++j) u[j] = (uint8_t)(-qmin); return; }
    float inv = 1.0f / df;
    for (int j = 0; j < n; ++j) {
        float t = x[j] * inv;
        float r = rintf(t);                                  /* ties to even (R3) */
        if (r < (float)qmin) r = (float)qmin;
        if (r > (float)qmax) r = (float)qmax;
        u[j] = (uint8_t)((int)r - qmin);
    }
}

/* R5: asymmetric block quantizer ("_1"): m = fp16 round-down of the block
 * minimum, d = (max - m)/(2^b - 1) stored fp16 RNE, u = clamp(RNE((x-m)/d)). */
/* Block minimum / maximum with IEEE-754 minimum / maximum semantics for signed
 * zeros (-0 < +0), so the result does not depend on the order of the values. */
static float block_minimum(const float* x, int n) {
    float mn = x[0];
    for (int j = 1; j < n; ++j)
        if (x[j] < mn || (x[j] == 0.0f && mn == 0.0f && signbit(x[j]))) mn = x[j];
    return mn;
}
static float block_maximum(const float* x, int n) {
    float mx = x[0];
    for (int j = 1; j < n; ++j)
        if (x[j] > mx || (x[j] == 0.0f && mx == 0.0f && !signbit(x[j]))) mx = x[j];
    return mx;
}

static void quant_block_asym(const float* x, int n, int bits, uint8_t* u, uint16_t* dh_out, uint16_t* mh_out) {
    float mn = block_minimum(x, n), mx = block_maximum(x, n);
    if (mn < -65504.0f) mn = -65504.0f;
    if (mn > 65504.0f) mn = 65504.0f;
    uint16_t mh = orc_f16_rd(mn);
    float mf = orc_f16_to_f32(mh);
    const int umax = (1 << bits) - 1;
    float d = (mx - mf) / (float)umax;
    if (d > 65504.0f) d = 65504.0f;
    uint16_t dh = orc_f16_rn(d);
    float df = orc_f16_to_f32(dh);
    *dh_out = dh; *mh_out = mh;
    if (df == 0.0f) { for (int j = 0; j < n; ++j) u[j] = 0; return; }
    float inv = 1.0f / df;
    for (int j = 0; j < n; ++j) {
        float t = (x[j] - mf) * inv;
        float r = rintf(t);
        if (r < 0.0f) r = 0.0f;
        if (r > (float)umax) r = (float)umax;
        u[j] = (uint8_t)(int)r;
    }
}

/* R11: mid-rise symmetric quantizer with all 2^b levels for the rank variant
 * [COBRA §Jargon "Scalar quantization": one of 2^b levels].  Levels are
 * (k + 1/2) d for k in [-2^(b-1), 2^(b-1)-1]; d = amax / (2^(b-1) - 1/2). */
static void quant_block_midrise(const float* x, int n, int bits, uint8_t* u, uint16_t* dh_out) {
    float amax = 0.0f;
    for (int j = 0; j < n; ++j) { float a = fabsf(x[j]); if (a > amax) amax = a; }
    const int half = 1 << (bits - 1);
    float L = (float)half - 0.5f;
    float d = amax / L;
    if (d > 65504.0f) d = 65504.0f;
    uint16_t dh = orc_f16_rn(d);
    float df = orc_f16_to_f32(dh);
    *dh_out = dh;
    if (df == 0.0f) { for (int j = 0; j < n; ++j) u[j] = (uint8_t)half; return; }
    float inv = 1.0f / df;
    for (int j = 0; j < n; ++j) {
        float t = x[j] * inv;
        float k = floorf(t);
        if (k < (float)-half) k = (float)-half;
        if (k > (float)(half - 1)) k = (float)(half - 1);
        u[j] = (uint8_t)((int)k + half);
    }
}

/* R7 packing.  u[0..n) with b bits each into a canonical row:
 *  b=8: byte j = u_j;  b=4: nibble j (LSB first);  b=2: 2-bit field j;
 *  b=1: bit j;  b=6: 4-bit plane of (u & 15) followed by 2-bit plane of u>>4;
 *  b=5: 4-bit plane of (u & 15) followed by 1-bit plane of u>>4;
 *  b=3: 2-bit plane of (u & 3) followed by 1-bit plane of u>>2;
 *  b=16 (F16): little-endian binary16 values. */
static void pack_field(const uint8_t* v, int n, int w, uint8_t* out) {
    int per = 8 / w;
    memset(out, 0, (size_t)(n * w / 8));
    for (int j = 0; j < n; ++j) out[j / per] |= (uint8_t)(v[j] << (w * (j % per)));
}
static void unpack_field(const uint8_t* in, int n, int w, uint8_t* v) {
    int per = 8 / w;
    uint8_t mask = (uint8_t)((1u << w) - 1u);
    for (int j = 0; j < n; ++j) v[j] = (uint8_t)((in[j / per] >> (w * (j % per))) & mask);
}
void orc_pack_codes(const uint8_t* u, int n, int bits, uint8_t* out) {
    uint8_t lo[128], hi[128];
    switch (bits) {
        case 8: memcpy(out, u, (size_t)n); break;
        case 4: pack_field(u, n, 4, out); break;
        case 2: pack_field(u, n, 2, out); break;
        case 1: pack_field(u, n, 1, out); break;
        case 6:
            for (int j = 0; j < n; ++j) { lo[j] = u[j] & 15; hi[j] = u[j] >> 4; }
            pack_field(lo, n, 4, out); pack_field(hi, n, 2, out + n / 2); break;
        case 5:
            for (int j = 0; j < n; ++j) { lo[j] = u[j] & 15; hi[j] = u[j] >> 4; }
            pack_field(lo, n, 4, out); pack_field(hi, n, 1, out + n / 2); break;
        case 3:
            for (int j = 0; j < n; ++j) { lo[j] = u[j] & 3; hi[j] = u[j] >> 2; }
            pack_field(lo, n, 2, out); pack_field(hi, n, 1, out + n / 4); break;
        default: break;
    }
}
void orc_unpack_codes(const uint8_t* in, int n, int bits, uint8_t* u) {
    uint8_t lo[128], hi[128];
    switch (bits) {
        case 8: memcpy(u, in, (size_t)n); break;
        case 4: unpack_field(in, n, 4, u); break;
        case 2: unpack_field(in, n, 2, u); break;
        case 1: unpack_field(in, n, 1, u); break;
        case 6:
            unpack_field(in, n, 4, lo); unpack_field(in + n / 2, n, 2, hi);
            for (int j = 0; j < n; ++j) u[j] = (uint8_t)(lo[j] | (hi[j] << 4));
            break;
        case 5:
            unpack_field(in, n, 4, lo); unpack_field(in + n / 2, n, 1, hi);
            for (int j = 0; j < n; ++j) u[j] = (uint8_t)(lo[j] | (hi[j] << 4));
            break;
        case 3:
            unpack_field(in, n, 2, lo); unpack_field(in + n / 4, n, 1, hi);
            for (int j = 0; j < n; ++j) u[j] = (uint8_t)(lo[j] | (hi[j] << 2));
            break;
        default: break;
    }
}

/* Quantize rows (already in the stored basis, fp32) into canonical packed
 * rows: codes[n_rows][cb], scales[n_rows][sb/2] (fp16 bit patterns).
 * Scale row layout: _0 and rank: d_0..d_{nb-1};  _1: d_0, m_0, d_1, m_1, ...
 * For F16 the "codes" are the fp16 values of the row (stored unrotated, R8). */
void orc_quantize_rows(int codec, int r, int b, int64_t n_rows, const float* y, uint8_t* codes, uint16_t* scales) {
    int cb, sb;
    orc_row_bytes(codec, r, b, &cb, &sb);
    const int n = (codec == C_RANK) ? r : D;
    const int bits = (codec == C_RANK) ? b : codec_bits(codec);
    const int blk = n < 32 ? n : 32;
    const int nb = n / blk;
    for (int64_t row = 0; row < n_rows; ++row) {
        const float* x = y + row * n;
        uint8_t* crow = codes + row * cb;
        uint16_t* srow = scales + row * (sb / 2);
        if (codec == C_F16) {
            for (int j = 0; j < n; ++j) { uint16_t h = orc_f16_rn(x[j]); crow[2 * j] = (uint8_t)(h & 0xff); crow[2 * j + 1] = (uint8_t)(h >> 8); }
            continue;
        }
        uint8_t u[128];
        for (int k = 0; k < nb; ++k) {
            if (codec == C_RANK) quant_block_midrise(x + k * blk, blk, bits, u + k * blk, &srow[k]);
            else if (codec_is_1(codec)) quant_block_asym(x + k * blk, blk, bits, u + k * blk, &srow[2 * k], &srow[2 * k + 1]);
            else quant_block_sym(x + k * blk, blk, bits, u + k * blk, &srow[k]);
        }
        orc_pack_codes(u, n, bits, crow);
    }
}

/* R6 dequantization in the stored basis (each result is one correctly rounded
 * binary32 value):  _0: code * d;  _1: u * d + m (u*d is exact);
 * rank: (2u - (2^b - 1)) * (d/2). */
void orc_dequantize_rows(int codec, int r, int b, int64_t n_rows, const uint8_t* codes, const uint16_t* scales, float* y) {
    int cb, sb;
    orc_row_bytes(codec, r, b, &cb, &sb);
    const int n = (codec == C_RANK) ? r : D;
    const int bits = (codec == C_RANK) ? b : codec_bits(codec);
    const int blk = n < 32 ? n : 32;
    for (int64_t row = 0; row < n_rows; ++row) {
        const uint8_t* crow = codes + row * cb;
        const uint16_t* srow = scales + row * (sb / 2);
        float* x = y + row * n;
        if (codec == C_F16) {
            for (int j = 0; j < n; ++j) x[j] = orc_f16_to_f32((uint16_t)(crow[2 * j] | (crow[2 * j + 1] << 8)));
            continue;
        }
        uint8_t u[128];
        orc_unpack_codes(crow, n, bits, u);
        for (int j = 0; j < n; ++j) {
            int k = j / blk;
            if (codec == C_RANK) {
                float df = orc_f16_to_f32(srow[k]);
                float lev = (float)(2 * (int)u[j] - ((1 << bits) - 1));
                x[j] = lev * (0.5f * df);
            } else if (codec_is_1(codec)) {
                float df = orc_f16_to_f32(srow[2 * k]);
                float mf = orc_f16_to_f32(srow[2 * k + 1]);
                float p = (float)u[j] * df;
                x[j] = p + mf;
            } else {
                float df = orc_f16_to_f32(srow[k]);
                int code = (int)u[j] - (1 << (bits - 1));
                x[j] = (float)code * df;
            }
        }
    }
}

/* ------------------------------------------------------------------------- */
/* Variance normalisation [BEE §核心新特性：KVarN]; R10                       */
/* ------------------------------------------------------------------------- */

/* inv_s[c] = fp32RN(1 / sqrt(mean_t x[t][c]^2)), the mean taken in double in
 * token order; 1 where the rms is below 1e-6.  x is fp16 [n_tok][stride]. */
void orc_varnorm_inv_rms(int64_t n_tok, int n_ch, int64_t stride, const uint16_t* x, float* inv_s) {
    for (int c = 0; c < n_ch; ++c) {
        double s = 0.0;
        for (int64_t t = 0; t < n_tok; ++t) {
            double v = (double)orc_f16_to_f32(x[t * stride + c]);
            s += v * v;
        }
        double rms = sqrt(s / (double)n_tok);
        inv_s[c] = (rms < 1e-6) ? 1.0f : (float)(1.0 / rms);
    }
}

/* ------------------------------------------------------------------------- */
/* Rotation fused into the per-head projection [COBRA §The news, last but one */
/* paragraph: the rotation is folded into the head's projection matrix]; R12  */
/* ------------------------------------------------------------------------- */

/* M = R_r P^T, with P the 128 x r orthonormal basis of the head (row-major
 * [128][r]) and R_r = H_r / sqrt(r) (Sylvester) for r in {16,32,64,128}, or
 * I_3 (x) H_32 / sqrt(32) for r = 96.  Computed in double, stored fp32 [r][128]. */
void orc_fuse_projection(int r, const double* P, float* M) {
    int8_t H[128 * 128];
    int blk = (r == 96) ? 32 : r;
    orc_hadamard_matrix(blk, H);       /* H is blk x blk with row stride blk */
    /* orc_hadamard_matrix writes with stride n = blk */
    const double s = 1.0 / sqrt((double)blk);
    for (int i = 0; i < r; ++i) {
        int bi = i / blk, ii = i % blk;
        for (int c = 0; c < D; ++c) {
            double acc = 0.0;
            for (int k = 0; k < blk; ++k) acc += (double)H[ii * blk + k] * P[c * r + bi * blk + k];
            M[i * D + c] = (float)(acc * s);
        }
    }
}

/* ------------------------------------------------------------------------- */
/* Encode: the append-quantize path for whole rows                             */
/* ------------------------------------------------------------------------- */

/* Rotation modes (by value, matching the public header's numbering). */
enum { ROT_NONE = 0, ROT_HADAMARD = 1, ROT_VARNORM_HADAMARD = 2, ROT_PROJECTION = 3 };

/* Bring fp16 rows [n_rows][128] into the stored basis, as fp32:
 *  F16 codec: the raw values (R8);
 *  Hadamard:  spec FWHT of x;  varnorm: spec FWHT of (x * inv_s) (one fp32
 *  multiply per element, R10);
 *  projection: z = M x accumulated in double, rounded to fp32 (R12). */
void orc_to_stored_basis_dt(int bf16, int codec, int rot, int r, const float* inv_s, const float* M,
                            int64_t n_rows, const uint16_t* x, float* y) {
    const int n_out = (codec == C_RANK) ? r : D;
    for (int64_t row = 0; row < n_rows; ++row) {
        float v[D];
        for (int j = 0; j < D; ++j) v[j] = raw_to_f32(x[row * D + j], bf16);
        float* out = y + row * n_out;
        if (codec == C_F16 || rot == ROT_NONE) { memcpy(out, v, sizeof(float) * D); continue; }
        if (codec == C_RANK) {
            for (int i = 0; i < r; ++i) {
                double acc = 0.0;
                for (int j = 0; j < D; ++j) acc += (double)M[i * D + j] * (double)v[j];
                out[i] = (float)acc;
            }
            continue;
        }
        if (rot == ROT_VARNORM_HADAMARD) for (int j = 0; j < D; ++j) v[j] = v[j] * inv_s[j];
        orc_fwht_spec(1, v);
        memcpy(out, v, sizeof(float) * D);
    }
}

void orc_to_stored_basis(int codec, int rot, int r, const float* inv_s, const float* M,
                         int64_t n_rows, const uint16_t* x, float* y) {
    orc_to_stored_basis_dt(0, codec, rot, r, inv_s, M, n_rows, x, y);
}

/* Full encode of raw 16-bit rows (fp16, or bf16 if bf16 != 0) into canonical
 * packed rows. */
void orc_encode_rows_dt(int bf16, int codec, int rot, int r, int b, const float* inv_s, const float* M,
                        int64_t n_rows, const uint16_t* x, uint8_t* codes, uint16_t* scales) {
    const int n_out = (codec == C_RANK) ? r : D;
    float* y = (float*)malloc(sizeof(float) * (size_t)(n_rows * n_out));
    orc_to_stored_basis_dt(bf16, codec, rot, r, inv_s, M, n_rows, x, y);
    orc_quantize_rows(codec, r, b, n_rows, y, codes, scales);
    free(y);
}

void orc_encode_rows(int codec, int rot, int r, int b, const float* inv_s, const float* M,
                     int64_t n_rows, const uint16_t* x, uint8_t* codes, uint16_t* scales) {
    orc_encode_rows_dt(0, codec, rot, r, b, inv_s, M, n_rows, x, codes, scales);
}

/* Dequantize canonical rows and return them in the ORIGINAL basis, double:
 *  F16 / no rotation: the stored values;
 *  Hadamard: R yhat (dense double);  varnorm: (R yhat) / inv_s;
 *  projection: M^T zhat (double). */
void orc_decode_rows_original(int codec, int rot, int r, int b, const float* inv_s, const float* M,
                              int64_t n_rows, const uint8_t* codes, const uint16_t* scales, double* out) {
    const int n = (codec == C_RANK) ? r : D;
    float* y = (float*)malloc(sizeof(float) * (size_t)(n_rows * n));
    orc_dequantize_rows(codec, r, b, n_rows, codes, scales, y);
    for (int64_t row = 0; row < n_rows; ++row) {
        double* o = out + row * D;
        const float* yr = y + row * n;
        if (codec == C_F16 || rot == ROT_NONE) { for (int j = 0; j < D; ++j) o[j] = (double)yr[j]; continue; }
        if (codec == C_RANK) {
            for (int c = 0; c < D; ++c) {
                double acc = 0.0;
                for (int i = 0; i < r; ++i) acc += (double)M[i * D + c] * (double)yr[i];
                o[c] = acc;
            }
            continue;
        }
        double t[D];
        for (int j = 0; j < D; ++j) t[j] = (double)yr[j];
        orc_rotate_dense(1, t, o);
        if (rot == ROT_VARNORM_HADAMARD) for (int j = 0; j < D; ++j) o[j] = o[j] / (double)inv_s[j];
    }
    free(y);
}

/* ------------------------------------------------------------------------- */
/* Decode attention [FORUM, attention paragraph]: dot the query with every     */
/* prior key, softmax, weighted average of the values.                         */
/* ------------------------------------------------------------------------- */

/* One query head over n keys/values [n][128] (double), softmax scale given. */
void orc_attention(int64_t n, const double* q, const double* K, const double* V, double scale, double* out) {
    double* s = (double*)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
    double m = -INFINITY;
    for (int64_t i = 0; i < n; ++i) {
        double acc = 0.0;
        for (int j = 0; j < D; ++j) acc += q[j] * K[i * D + j];
        s[i] = acc * scale;
        if (s[i] > m) m = s[i];
    }
    double l = 0.0;
    for (int64_t i = 0; i < n; ++i) { s[i] = exp(s[i] - m); l += s[i]; }
    for (int j = 0; j < D; ++j) out[j] = 0.0;
    for (int64_t i = 0; i < n; ++i)
        for (int j = 0; j < D; ++j) out[j] += s[i] * V[i * D + j];
    for (int j = 0; j < D; ++j) out[j] = (n > 0) ? out[j] / l : 0.0;
    free(s);
}

/* Decode attention for one (sequence, layer, kv-head) of a cache whose history
 * is given as fp16 rows [len][128] for K and V.  The newest T rows are the
 * F16 precision tail [BEE §KV cache 精度尾部]; rows older than that were
 * quantized with the head's codecs after the head's transform.  G query heads
 * (fp16 [G][128]) share this kv-head (grouped-query attention).  The cache is
 * rebuilt here from the history with this file's own encoder, dequantized to
 * the original basis in double, and attended densely.  When T >= len every
 * row is a tail row and the path is exactly the plain F16 attention below.
 * out: fp32 [G][128].  k_codec/v_codec: codec ids; kb/vb: bits for the rank
 * codec; r: rank. */
void orc_decode_head_dt(int bf16, int64_t len, int T, int G, const uint16_t* Kx, const uint16_t* Vx,
                        const uint16_t* q, int k_codec, int v_codec, int rot, int r, int kb, int vb,
                        const float* inv_s_k, const float* inv_s_v, const float* M, float scale, float* out) {
    int64_t nq = len > T ? len - T : 0;
    double* Kd = (double*)malloc(sizeof(double) * (size_t)((len > 0 ? len : 1) * D));
    double* Vd = (double*)malloc(sizeof(double) * (size_t)((len > 0 ? len : 1) * D));
    int cbk, sbk, cbv, sbv;
    orc_row_bytes(k_codec, r, kb, &cbk, &sbk);
    orc_row_bytes(v_codec, r, vb, &cbv, &sbv);
    if (nq > 0) {
        uint8_t* ck = (uint8_t*)malloc((size_t)(nq * cbk));
        uint16_t* sk = (uint16_t*)malloc((size_t)(nq * (sbk > 0 ? sbk : 2)));
        uint8_t* cv = (uint8_t*)malloc((size_t)(nq * cbv));
        uint16_t* sv = (uint16_t*)malloc((size_t)(nq * (sbv > 0 ? sbv : 2)));
        orc_encode_rows_dt(bf16, k_codec, rot, r, kb, inv_s_k, M, nq, Kx, ck, sk);
        orc_encode_rows_dt(bf16, v_codec, rot, r, vb, inv_s_v, M, nq, Vx, cv, sv);
        orc_decode_rows_original(k_codec, rot, r, kb, inv_s_k, M, nq, ck, sk, Kd);
        orc_decode_rows_original(v_codec, rot, r, vb, inv_s_v, M, nq, cv, sv, Vd);
        free(ck); free(sk); free(cv); free(sv);
    }
    for (int64_t i = nq; i < len; ++i)
        for (int j = 0; j < D; ++j) {
            Kd[i * D + j] = (double)raw_to_f32(Kx[i * D + j], bf16);
            Vd[i * D + j] = (double)raw_to_f32(Vx[i * D + j], bf16);
        }
    for (int g = 0; g < G; ++g) {
        double qd[D], o[D];
        for (int j = 0; j < D; ++j) qd[j] = (double)raw_to_f32(q[g * D + j], bf16);
        orc_attention(len, qd, Kd, Vd, (double)scale, o);
        for (int j = 0; j < D; ++j) out[g * D + j] = (float)o[j];
    }
    free(Kd); free(Vd);
}

void orc_decode_head(int64_t len, int T, int G, const uint16_t* Kx, const uint16_t* Vx, const uint16_t* q,
                     int k_codec, int v_codec, int rot, int r, int kb, int vb,
                     const float* inv_s_k, const float* inv_s_v, const float* M, float scale, float* out) {
    orc_decode_head_dt(0, len, T, G, Kx, Vx, q, k_codec, v_codec, rot, r, kb, vb, inv_s_k, inv_s_v, M, scale, out);
}

/* Decode attention from already packed canonical rows (the oracle's own), for
 * timing the decode step alone: nq quantized rows + nt raw fp16 tail rows. */
void orc_decode_packed_dt(int bf16, int64_t nq, const uint8_t* ck, const uint16_t* sk, const uint8_t* cv,
                          const uint16_t* sv, int64_t nt, const uint16_t* Kt, const uint16_t* Vt, int G,
                          const uint16_t* q, int k_codec, int v_codec, int rot, int r, int kb, int vb,
                          const float* inv_s_k, const float* inv_s_v, const float* M, float scale, float* out) {
    int64_t len = nq + nt;
    double* Kd = (double*)malloc(sizeof(double) * (size_t)((len > 0 ? len : 1) * D));
    double* Vd = (double*)malloc(sizeof(double) * (size_t)((len > 0 ? len : 1) * D));
    if (nq > 0) {
        orc_decode_rows_original(k_codec, rot, r, kb, inv_s_k, M, nq, ck, sk, Kd);
        orc_decode_rows_original(v_codec, rot, r, vb, inv_s_v, M, nq, cv, sv, Vd);
    }
    for (int64_t i = 0; i < nt; ++i)
        for (int j = 0; j < D; ++j) {
            Kd[(nq + i) * D + j] = (double)raw_to_f32(Kt[i * D + j], bf16);
            Vd[(nq + i) * D + j] = (double)raw_to_f32(Vt[i * D + j], bf16);
        }
    for (int g = 0; g < G; ++g) {
        double qd[D], o[D];
        for (int j = 0; j < D; ++j) qd[j] = (double)raw_to_f32(q[g * D + j], bf16);
        orc_attention(len, qd, Kd, Vd, (double)scale, o);
        for (int j = 0; j < D; ++j) out[g * D + j] = (float)o[j];
    }
    free(Kd); free(Vd);
}

void orc_decode_packed(int64_t nq, const uint8_t* ck, const uint16_t* sk, const uint8_t* cv, const uint16_t* sv,
                       int64_t nt, const uint16_t* Kt, const uint16_t* Vt, int G, const uint16_t* q,
                       int k_codec, int v_codec, int rot, int r, int kb, int vb,
                       const float* inv_s_k, const float* inv_s_v, const float* M, float scale, float* out) {
    orc_decode_packed_dt(0, nq, ck, sk, cv, sv, nt, Kt, Vt, G, q, k_codec, v_codec, rot, r, kb, vb, inv_s_k, inv_s_v,
                         M, scale, out);
}

/* ------------------------------------------------------------------------- */
/* KV-COBRA allocation of rank and bits per head [COBRA §The news (steps C1   */
/* and C2) and §Where the bits actually go]                                   */
/* ------------------------------------------------------------------------- */

static const int COBRA_R[5] = {16, 32, 64, 96, 128};

/* Error of keeping the top r directions of a head at b bits: the variance of
 * the dropped directions (lost outright) plus the rounding noise of the kept
 * ones, eps[b-1] times their variance.  lambda: the head's 128 direction
 * variances, sorted in decreasing order. */
double orc_cobra_error(const double* lambda, int r, int b, const double* eps) {
    double kept = 0.0, lost = 0.0;
    for (int i = 0; i < D; ++i) {
        if (i < r) kept += lambda[i];
        else lost += lambda[i];
    }
    return lost + eps[b - 1] * kept;
}

/* C1: the (r, b) with r*b <= budget of least error (ties: fewer bits, then
 * smaller r).  Returns 0 and leaves r, b untouched if nothing fits. */
int orc_cobra_best(const double* lambda, int budget, const double* eps, int* r_out, int* b_out) {
    double best = INFINITY;
    int found = 0, best_bits = 0;
    for (int ri = 0; ri < 5; ++ri)
        for (int b = 1; b <= 4; ++b) {
            int bits = COBRA_R[ri] * b;
            if (bits > budget) continue;
            double e = orc_cobra_error(lambda, COBRA_R[ri], b, eps);
            if (!found || e < best || (e == best && bits < best_bits) ||
                (e == best && bits == best_bits && COBRA_R[ri] < *r_out)) {
                best = e; best_bits = bits; *r_out = COBRA_R[ri]; *b_out = b; found = 1;
            }
        }
    return found;
}

/* C2: water-filling over heads.  Every head starts at the cheapest setting
 * (r = 16, b = 1); the remaining bits of the budget (bpd * 128 per head) go,
 * one upgrade at a time, to the head whose best affordable upgrade removes the
 * most error per extra bit (ties: lower head index, then fewer bits), until no
 * upgrade fits or none lowers the error.  lambdas: [n_heads][128], each sorted
 * in decreasing order.  Returns the bits used. */
int orc_cobra_allocate(int n_heads, const double* lambdas, double bpd, const double* eps, int* r, int* b) {
    const int budget = (int)(bpd * D * n_heads + 0.5);
    int used = 0;
    for (int h = 0; h < n_heads; ++h) { r[h] = 16; b[h] = 1; used += 16; }
    for (;;) {
        int bh = -1, br = 0, bb = 0, bbits = 0;
        double bgain = 0.0;
        for (int h = 0; h < n_heads; ++h) {
            const double* lam = lambdas + (size_t)h * D;
            const double e0 = orc_cobra_error(lam, r[h], b[h], eps);
            const int cur = r[h] * b[h];
            for (int ri = 0; ri < 5; ++ri)
                for (int bi = 1; bi <= 4; ++bi) {
                    int bits = COBRA_R[ri] * bi;
                    if (bits <= cur || used - cur + bits > budget) continue;
                    double gain = (e0 - orc_cobra_error(lam, COBRA_R[ri], bi, eps)) / (double)(bits - cur);
                    if (gain > bgain || (gain == bgain && gain > 0.0 && bh == h && bits < bbits)) {
                        bgain = gain; bh = h; br = COBRA_R[ri]; bb = bi; bbits = bits;
                    }
                }
        }
        if (bh < 0) break;
        used += bbits - r[bh] * b[bh];
        r[bh] = br; b[bh] = bb;
    }
    return used;
}
