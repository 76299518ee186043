/*
 * moe_oracle.c -- CPU oracle of the MoE layer.
 *
 * TEST INFRASTRUCTURE ONLY. Only tests/, __graft_entry__.smoke() and the
 * cpu_baseline / reference legs of bench.py may load this library. It shares
 * no code with the CUDA path and never calls it.
 *
 * What it computes, and where that is stated:
 *
 *  - The per-token MoE step of "Megatron-Core MoE -- 大规模稀疏专家并行实践"
 *    (study notes, estelledc.github.io), section 实践案例 / 案例 1: score every
 *    expert, keep the top-k, and sum gate(e) * Expert_e(x) over the kept ones.
 *  - The memory-efficient permutation of "《使用 Megatron Core 大规模训练混合专家
 *    模型（MoE）》技术总结" (gist.science), section 2.2: the routing weight is
 *    absorbed into the activation, i.e. W_d (g a) is computed instead of
 *    g (W_d a). oc_moe_fwd_tokens() can evaluate both orders.
 *  - The load-balancing auxiliary loss named in section 2.4 of the same summary
 *    ("fuse routing, permutation and aux-loss computation") and in 案例 3 of the
 *    study notes. The pages give no formula; the reading used is
 *    aux = E * sum_e f_e P_e with f_e = count_e / (T k) and P_e the mean full
 *    softmax probability of expert e.
 *  - MXFP8 (section 3 of the summary names the MXFP8 recipe for Blackwell):
 *    OCP Microscaling Formats v1.0, section 6.3: per block of 32 elements the
 *    shared scale is 2^(floor(log2(amax)) - 8) (8 = E4M3 emax), stored as an
 *    UE8M0 byte, and each element is v/scale rounded to E4M3 (nearest-even,
 *    clamped to +-448).
 *
 *  - NVFP4 (section 2.4 of the summary runs the expert GEMMs in FP8/FP4, and
 *    section 3 lists an NVFP4 recipe): NVIDIA's 4-bit format. Elements are
 *    OCP MX v1.0 FP4 E2M1 (section 5.3.3: magnitudes 0, 0.5, 1, 1.5, 2, 3, 4,
 *    6); every 16 consecutive elements along K share one positive E4M3 scale
 *    (amax / 6 times a per-tensor encode scale G, rounded to E4M3), and the
 *    tensor's fp32 G = 6 * 448 / amax(tensor) makes the largest block scale
 *    448. The pages fix none of this; the readings used: G per expert
 *    weight matrix, G = 1 for activations, nearest-even everywhere.
 *
 * Everything is plain loops in double precision. Expert operands are reached
 * through oc_mat, which decodes one row at a time from bf16, MXFP8 or fp64
 * storage; decoding is exact in every case.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------ scalars */

static double bf16_to_double(uint16_t v) {
    uint32_t u = (uint32_t)v << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* Round to bf16 the way a kernel that works in fp32 does: first to fp32, then
 * to the nearest bf16 with ties to even (IEEE round-to-nearest-even on the
 * upper 16 bits of the fp32 pattern). Inf/NaN pass through. */
double oc_bf16_round(double v) {
    float f = (float)v;
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7f800000u) == 0x7f800000u) return (double)f;
    u += 0x7fffu + ((u >> 16) & 1u);
    u &= 0xffff0000u;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* Rounding points of the layer's precision recipes:
 *   OC_EXACT  no rounding at all (fp64 throughout; used by the pins);
 *   OC_MX     MXFP8 recipe: the expert GEMM operands are MXFP8 (x and the
 *             gate-folded activation, 1x32 blocks along K), the expert GEMM
 *             outputs are bf16;
 *   OC_BF16R  BF16 recipe: the expert GEMM operands and outputs are bf16 (the
 *             gate-folded activation, each expert's output; in the backward
 *             the saved pre-activations, dgate/dup, the per-row dXp and the
 *             router-gradient operand). */
enum { OC_EXACT = 0, OC_MX = 1, OC_BF16R = 2, OC_NV = 3, OC_MXQ = 4, OC_NVQ = 5 };
/*   OC_NV     NVFP4 recipe: as OC_MX with NVFP4 operands (16-blocks along K,
 *             activations with G = 1), bf16 expert GEMM outputs.
 *   OC_MXQ, OC_NVQ  the block-scaled formats' quantisation points only: the
 *             operands are quantised exactly as under OC_MX / OC_NV (and, in
 *             the backward, every MXFP8 operand of OC_MX), but no value is
 *             rounded to bf16 anywhere (not the expert outputs, the saved
 *             pre-activations, dgate/dup, dXp nor the router-gradient
 *             operand): fp64 everywhere else. This is the exact layer up to
 *             the quantisation the format itself defines. */
static int is_mx(int recipe) { return recipe == OC_MX || recipe == OC_MXQ; }
static int is_nv(int recipe) { return recipe == OC_NV || recipe == OC_NVQ; }

static void round_vec(double* v, int n, int recipe) {
    if (recipe == OC_BF16R || recipe == OC_MX || recipe == OC_NV)
        for (int i = 0; i < n; ++i) v[i] = oc_bf16_round(v[i]);
}

/* E4M3 (OCP "fn" variant): 1 sign, 4 exponent (bias 7), 3 mantissa bits;
 * exponent field 0 is subnormal (m * 2^-9); S.1111.111 is NaN; max 448. */
double oc_e4m3_decode(uint8_t c) {
    int s = c >> 7, ef = (c >> 3) & 15, m = c & 7;
    double v;
    if (ef == 15 && m == 7) return NAN;
    if (ef == 0) v = ldexp((double)m, -9);
    else v = ldexp(1.0 + m / 8.0, ef - 7);
    return s ? -v : v;
}

/* The binade of a positive finite double: the e with 2^e <= a < 2^(e+1).
 * frexp returns a = m 2^x with m in [0.5, 1) exactly, so e = x - 1. */
static int binade(double a) {
    int x;
    frexp(a, &x);
    return x - 1;
}

/* Round |v| to the E4M3 grid, nearest-even, clamp to 448. v is finite. */
uint8_t oc_e4m3_encode(double v) {
    uint8_t sign = (signbit(v) ? 0x80 : 0x00);
    double a = fabs(v);
    if (a == 0.0) return sign;
    int e = binade(a);
    if (e < -6) e = -6;                     /* subnormal range shares the 2^-9 quantum */
    double q = ldexp(1.0, e - 3);           /* spacing of the grid in this binade */
    double r = a / q;                       /* exact: power-of-two division */
    double fl = floor(r);
    double frac = r - fl;
    double n;
    if (frac > 0.5) n = fl + 1.0;
    else if (frac < 0.5) n = fl;
    else n = (fmod(fl, 2.0) == 0.0) ? fl : fl + 1.0;
    double val = n * q;
    if (val > 448.0) val = 448.0;
    if (val == 0.0) return sign;
    /* encode val */
    int ve = binade(val);
    uint8_t code;
    if (ve < -6) {
        code = (uint8_t)(val / ldexp(1.0, -9));          /* subnormal: m = val / 2^-9 */
    } else {
        int mant = (int)(val / ldexp(1.0, ve - 3)) - 8;  /* 0..7 */
        code = (uint8_t)(((ve + 7) << 3) | mant);
    }
    return sign | code;
}

/* UE8M0 scale byte of one block, OCP MX v1.0 section 6.3 with E4M3 emax = 8. */
uint8_t oc_mx_scale_byte(double amax) {
    if (!(amax > 0.0)) return 0;
    int e = binade(amax);
    int b = e - 8 + 127;
    if (b < 0) b = 0;
    if (b > 254) b = 254;
    return (uint8_t)b;
}

/* Quantise rows x K (K % 32 == 0) of fp32 values to E4M3 codes + UE8M0 bytes,
 * 1x32 blocks along K. */
void oc_mxfp8_quantize(long rows, int K, const float* src, uint8_t* codes, uint8_t* scales) {
    long r;
#pragma omp parallel for schedule(static)
    for (r = 0; r < rows; ++r) {
        for (int b = 0; b < K / 32; ++b) {
            const float* v = src + r * (long)K + b * 32;
            double amax = 0.0;
            for (int i = 0; i < 32; ++i) {
                double a = fabs((double)v[i]);
                if (a > amax) amax = a;
            }
            uint8_t sb = oc_mx_scale_byte(amax);
            scales[r * (long)(K / 32) + b] = sb;
            double X = ldexp(1.0, (int)sb - 127);
            for (int i = 0; i < 32; ++i)
                codes[r * (long)K + b * 32 + i] = oc_e4m3_encode((double)v[i] / X);
        }
    }
}

/* Same, from bf16 storage. */
void oc_mxfp8_quantize_bf16(long rows, int K, const uint16_t* src, uint8_t* codes, uint8_t* scales) {
    long r;
#pragma omp parallel for schedule(static)
    for (r = 0; r < rows; ++r) {
        float tmp[32];
        for (int b = 0; b < K / 32; ++b) {
            double amax = 0.0;
            for (int i = 0; i < 32; ++i) {
                tmp[i] = (float)bf16_to_double(src[r * (long)K + b * 32 + i]);
                double a = fabs((double)tmp[i]);
                if (a > amax) amax = a;
            }
            uint8_t sb = oc_mx_scale_byte(amax);
            scales[r * (long)(K / 32) + b] = sb;
            double X = ldexp(1.0, (int)sb - 127);
            for (int i = 0; i < 32; ++i)
                codes[r * (long)K + b * 32 + i] = oc_e4m3_encode((double)tmp[i] / X);
        }
    }
}

/* ------------------------------------------------------------ NVFP4 */

/* E2M1 (OCP MX v1.0 section 5.3.3): code bits s.ee.m, exponent bias 1,
 * exponent field 0 is subnormal (m * 0.5); no Inf or NaN; largest 6. */
double oc_e2m1_decode(uint8_t c) {
    int s = (c >> 3) & 1, ef = (c >> 1) & 3, m = c & 1;
    double v = ef == 0 ? 0.5 * m : ldexp(1.0 + 0.5 * m, ef - 1);
    return s ? -v : v;
}

/* Nearest E2M1 code of v: magnitudes above 6 saturate to 6, a tie goes to the
 * code whose mantissa bit is 0 (round half to even); the sign is kept, zero
 * included. v is finite. */
uint8_t oc_e2m1_encode(double v) {
    uint8_t sign = signbit(v) ? 8 : 0;
    double a = fabs(v);
    if (a > 6.0) a = 6.0;
    int best = 0;
    double bd = INFINITY;
    for (int c = 0; c < 8; ++c) {
        double d = fabs(oc_e2m1_decode((uint8_t)c) - a);
        if (d < bd || (d == bd && (c & 1) == 0)) {
            best = c;
            bd = d;
        }
    }
    return sign | (uint8_t)best;
}

/* Encode scale G of a tensor with largest magnitude amax: 6 * 448 / amax in
 * fp32, so that the block holding amax gets the largest E4M3 scale; 1 for an
 * all-zero tensor. */
float oc_nvfp4_global_scale(float amax) { return amax > 0.0f ? 2688.0f / amax : 1.0f; }

/* E4M3 scale byte of a 16-block with largest magnitude amax, tensor scale G:
 * (amax / 6) * G in fp32, rounded to E4M3 (nearest-even, at most 448). */
uint8_t oc_nvfp4_scale_byte(float amax, float G) {
    float s = amax / 6.0f;
    s = s * G;
    return oc_e4m3_encode((double)s);
}

/* One 16-block t[16] -> codes[16] (one E2M1 code per byte) and its scale byte.
 * Element i is t[i] * (G / scale) in fp32, rounded to E2M1; a zero scale
 * multiplies by 0. Decoding: code * scale / G. */
static uint8_t nv_block(const float* t, float G, uint8_t* codes) {
    float amax = 0.0f;
    for (int i = 0; i < 16; ++i)
        if (fabsf(t[i]) > amax) amax = fabsf(t[i]);
    uint8_t sb = oc_nvfp4_scale_byte(amax, G);
    float sd = (float)oc_e4m3_decode(sb);
    float r = sd > 0.0f ? G / sd : 0.0f;
    for (int i = 0; i < 16; ++i) {
        float u = t[i] * r;
        codes[i] = oc_e2m1_encode((double)u);
    }
    return sb;
}

/* Quantise rows x K (K % 16 == 0) of bf16 values with tensor scale G:
 * packed [rows, K/2] (element 2i in the low nibble of byte i, 2i+1 in the
 * high nibble), scales [rows, K/16]. */
void oc_nvfp4_quantize_bf16(long rows, int K, const uint16_t* src, float G, uint8_t* packed, uint8_t* scales) {
    long r;
#pragma omp parallel for schedule(static)
    for (r = 0; r < rows; ++r) {
        float t[16];
        uint8_t c[16];
        for (int b = 0; b < K / 16; ++b) {
            for (int i = 0; i < 16; ++i) t[i] = (float)bf16_to_double(src[r * (long)K + b * 16 + i]);
            scales[r * (long)(K / 16) + b] = nv_block(t, G, c);
            for (int i = 0; i < 8; ++i)
                packed[r * (long)(K / 2) + b * 8 + i] = (uint8_t)(c[2 * i] | (c[2 * i + 1] << 4));
        }
    }
}

/* Same, from fp32 values. */
void oc_nvfp4_quantize_f32(long rows, int K, const float* src, float G, uint8_t* packed, uint8_t* scales) {
    long r;
#pragma omp parallel for schedule(static)
    for (r = 0; r < rows; ++r) {
        uint8_t c[16];
        for (int b = 0; b < K / 16; ++b) {
            scales[r * (long)(K / 16) + b] = nv_block(src + r * (long)K + b * 16, G, c);
            for (int i = 0; i < 8; ++i)
                packed[r * (long)(K / 2) + b * 8 + i] = (uint8_t)(c[2 * i] | (c[2 * i + 1] << 4));
        }
    }
}

/* Largest magnitude of n bf16 values (the input of oc_nvfp4_global_scale). */
float oc_bf16_amax(long n, const uint16_t* src) {
    double m = 0.0;
    for (long i = 0; i < n; ++i) {
        double a = fabs(bf16_to_double(src[i]));
        if (a > m) m = a;
    }
    return (float)m;
}

/* ------------------------------------------------------------ matrices */

enum { OC_BF16 = 0, OC_MXFP8 = 1, OC_F64 = 2, OC_NVFP4 = 3 };

/* Row-major matrix [rows, cols]; for OC_MXFP8, sf holds rows x cols/32 bytes.
 * OC_NVFP4: data holds rows x cols/2 packed E2M1 bytes, sf rows x cols/16 E4M3
 * scales, and gs one encode scale G per gs_rows consecutive rows (one per
 * expert matrix; NULL: G = 1). */
typedef struct {
    int32_t kind;
    int32_t cols;
    int64_t rows;
    const void* data;
    const uint8_t* sf;
    const float* gs;
    int64_t gs_rows;
} oc_mat;

/* Every E4M3 and E2M1 value, read from the decoders above once at load time
 * (the matrix reader looks codes up here instead of decoding each element). */
static double g_e4m3[256], g_e2m1[16];
__attribute__((constructor)) static void oc_decode_tables(void) {
    for (int c = 0; c < 256; ++c) g_e4m3[c] = oc_e4m3_decode((uint8_t)c);
    for (int c = 0; c < 16; ++c) g_e2m1[c] = oc_e2m1_decode((uint8_t)c);
}

static void oc_row(const oc_mat* m, int64_t r, double* out) {
    int C = m->cols;
    if (m->kind == OC_BF16) {
        const uint16_t* p = (const uint16_t*)m->data + r * C;
        for (int c = 0; c < C; ++c) out[c] = bf16_to_double(p[c]);
    } else if (m->kind == OC_MXFP8) {
        const uint8_t* p = (const uint8_t*)m->data + r * C;
        const uint8_t* s = m->sf + r * (C / 32);
        for (int b = 0; b < C / 32; ++b) {
            const double X = ldexp(1.0, (int)s[b] - 127);
            for (int c = 32 * b; c < 32 * b + 32; ++c) out[c] = g_e4m3[p[c]] * X;
        }
    } else if (m->kind == OC_NVFP4) {
        const uint8_t* p = (const uint8_t*)m->data + r * (C / 2);
        const uint8_t* s = m->sf + r * (C / 16);
        double G = m->gs ? (double)m->gs[r / m->gs_rows] : 1.0;
        for (int c = 0; c < C; ++c) {
            uint8_t code = (p[c / 2] >> (4 * (c & 1))) & 15;
            out[c] = g_e2m1[code] * g_e4m3[s[c / 16]] / G;
        }
    } else {
        const double* p = (const double*)m->data + r * C;
        for (int c = 0; c < C; ++c) out[c] = p[c];
    }
}

/* Sub-matrix view: rows [r0, r0+nrows) of m (an expert's slice of [E*R, C]). */
static oc_mat oc_slice(const oc_mat* m, int64_t r0, int64_t nrows) {
    oc_mat s = *m;
    s.rows = nrows;
    if (m->kind == OC_BF16) s.data = (const uint16_t*)m->data + r0 * m->cols;
    else if (m->kind == OC_MXFP8) {
        s.data = (const uint8_t*)m->data + r0 * m->cols;
        s.sf = m->sf + r0 * (m->cols / 32);
    } else if (m->kind == OC_NVFP4) {
        /* slices start on a G boundary (one expert matrix) */
        s.data = (const uint8_t*)m->data + r0 * (m->cols / 2);
        s.sf = m->sf + r0 * (m->cols / 16);
        if (m->gs) s.gs = m->gs + r0 / m->gs_rows;
    } else s.data = (const double*)m->data + r0 * m->cols;
    return s;
}

static double dot(const double* a, const double* b, int n) {
    double s = 0.0;
    for (int i = 0; i < n; ++i) s += a[i] * b[i];
    return s;
}

/* y = M v  (M [R, C], v [C]) */
static void matvec(const oc_mat* M, const double* v, double* y, double* rowbuf) {
    for (int64_t r = 0; r < M->rows; ++r) {
        oc_row(M, r, rowbuf);
        y[r] = dot(rowbuf, v, M->cols);
    }
}

/* y += M^T v  (M [R, C], v [R], y [C]) */
static void matvec_t_acc(const oc_mat* M, const double* v, double* y, double* rowbuf) {
    for (int64_t r = 0; r < M->rows; ++r) {
        oc_row(M, r, rowbuf);
        for (int c = 0; c < M->cols; ++c) y[c] += rowbuf[c] * v[r];
    }
}

static double sigmoid(double z) { return 1.0 / (1.0 + exp(-z)); }
static double silu(double z) { return z * sigmoid(z); }
static double silu_grad(double z) { double s = sigmoid(z); return s * (1.0 + z * (1.0 - s)); }

/* Round a double to the MXFP8 grid of its 32-block, in place, blocks along n.
 * The values are first rounded to fp32 (the precision in which the quantiser
 * takes its decisions), then quantised and decoded back. */
static void mx_roundtrip(double* v, int n) {
    for (int b = 0; b < n / 32; ++b) {
        float t[32];
        double amax = 0.0;
        for (int i = 0; i < 32; ++i) {
            t[i] = (float)v[b * 32 + i];
            if (fabs((double)t[i]) > amax) amax = fabs((double)t[i]);
        }
        uint8_t sb = oc_mx_scale_byte(amax);
        double X = ldexp(1.0, (int)sb - 127);
        for (int i = 0; i < 32; ++i) v[b * 32 + i] = oc_e4m3_decode(oc_e4m3_encode((double)t[i] / X)) * X;
    }
}

/* The same along a strided column: v[i * stride] for i in [0, n), in blocks of
 * 32 consecutive i (the last block zero-padded; padding never changes amax). */
static void mx_roundtrip_strided(double* v, long n, long stride) {
    for (long b0 = 0; b0 < n; b0 += 32) {
        long nb = n - b0 < 32 ? n - b0 : 32;
        float t[32];
        double amax = 0.0;
        for (long i = 0; i < nb; ++i) {
            t[i] = (float)v[(b0 + i) * stride];
            if (fabs((double)t[i]) > amax) amax = fabs((double)t[i]);
        }
        uint8_t sb = oc_mx_scale_byte(amax);
        double X = ldexp(1.0, (int)sb - 127);
        for (long i = 0; i < nb; ++i) v[(b0 + i) * stride] = oc_e4m3_decode(oc_e4m3_encode((double)t[i] / X)) * X;
    }
}

/* Round a double vector to the NVFP4 grid of its 16-blocks with G = 1 (the
 * activation reading), in place: fp32 first, then quantised and decoded. */
static void nv_roundtrip(double* v, int n) {
    for (int b = 0; b < n / 16; ++b) {
        float t[16];
        uint8_t c[16];
        for (int i = 0; i < 16; ++i) t[i] = (float)v[b * 16 + i];
        uint8_t sb = nv_block(t, 1.0f, c);
        double sd = oc_e4m3_decode(sb);
        for (int i = 0; i < 16; ++i) v[b * 16 + i] = oc_e2m1_decode(c[i]) * sd;
    }
}

/* ------------------------------------------------------------ routing */

/* logits[t,e] = sum_h x[t,h] W_r[e,h] (+ bias[e]); fp64 sum, one final rounding
 * to fp32 when round_f32 (router logits are kept in high precision: the study
 * notes' 踩过的坑 section warns that low-precision logits collapse routing). */
void oc_router_logits(int T, int H, int E, const oc_mat* x, const oc_mat* Wr, const float* bias,
                      int round_f32, double* logits) {
    int t;
#pragma omp parallel for schedule(static)
    for (t = 0; t < T; ++t) {
        double* xr = (double*)malloc(sizeof(double) * H);
        double* wr = (double*)malloc(sizeof(double) * H);
        oc_row(x, t, xr);
        for (int e = 0; e < E; ++e) {
            oc_row(Wr, e, wr);
            double s = dot(xr, wr, H);
            if (bias) s += (double)bias[e];
            logits[(long)t * E + e] = round_f32 ? (double)(float)s : s;
        }
        free(xr);
        free(wr);
    }
}

/* s[t,:] = softmax(l[t,:]) (score 0) or sigmoid(l[t,e]) (score 1). */
void oc_scores(int T, int E, int score, const double* logits, double* s) {
    for (int t = 0; t < T; ++t) {
        const double* l = logits + (long)t * E;
        double* o = s + (long)t * E;
        if (score == 0) {
            double mx = l[0];
            for (int e = 1; e < E; ++e) if (l[e] > mx) mx = l[e];
            double z = 0.0;
            for (int e = 0; e < E; ++e) { o[e] = exp(l[e] - mx); z += o[e]; }
            for (int e = 0; e < E; ++e) o[e] /= z;
        } else {
            for (int e = 0; e < E; ++e) o[e] = sigmoid(l[e]);
        }
    }
}

/* Top-k by logit value, descending; equal values go to the lower expert index
 * first. Slot j holds the j-th largest. (Selecting on logits is the same as
 * selecting on softmax or sigmoid scores: both maps are increasing.) */
void oc_topk(int T, int E, int k, const double* logits, int32_t* idx) {
    for (int t = 0; t < T; ++t) {
        const double* l = logits + (long)t * E;
        for (int j = 0; j < k; ++j) {
            int best = -1;
            for (int e = 0; e < E; ++e) {
                int taken = 0;
                for (int i = 0; i < j; ++i) if (idx[(long)t * k + i] == e) taken = 1;
                if (taken) continue;
                if (best < 0 || l[e] > l[best]) best = e;   /* strict: ties keep the lower index */
            }
            idx[(long)t * k + j] = best;
        }
    }
}

/*
 * Group-limited top-k on selection scores (the DeepSeek-V3 router variant; the
 * pages name DeepSeek-V3's routing but give no rule, so this is the reading):
 * the E experts form n_group equal groups of consecutive indices; a group's
 * score is the sum of its two largest selection scores (its one score when a
 * group holds a single expert); the topk_group best groups are kept
 * (descending, lower group index first on ties); then the k best experts of
 * the kept groups by selection score (descending, lower index first). The
 * selection score is sel[t,e] = s[t,e] + b[e], a per-expert bias that moves
 * selection only, never the gate values. n_group <= 1 is plain top-k on sel.
 */
void oc_topk_grouped(int T, int E, int k, int n_group, int topk_group, const double* sel, int32_t* idx) {
    int G = n_group > 1 ? E / n_group : E;
    int ng = n_group > 1 ? n_group : 1;
    int tg = n_group > 1 ? topk_group : 1;
    double* gscore = (double*)malloc(sizeof(double) * ng);
    int* gkeep = (int*)malloc(sizeof(int) * ng);
    for (int t = 0; t < T; ++t) {
        const double* v = sel + (long)t * E;
        for (int g = 0; g < ng; ++g) {
            double a1 = -INFINITY, a2 = -INFINITY;
            for (int e = g * G; e < (g + 1) * G; ++e) {
                if (v[e] > a1) { a2 = a1; a1 = v[e]; }
                else if (v[e] > a2) { a2 = v[e]; }
            }
            gscore[g] = (G >= 2) ? a1 + a2 : a1;
            gkeep[g] = 0;
        }
        for (int r = 0; r < tg; ++r) {
            int best = -1;
            for (int g = 0; g < ng; ++g) {
                if (gkeep[g]) continue;
                if (best < 0 || gscore[g] > gscore[best]) best = g;   /* strict: ties keep the lower group */
            }
            gkeep[best] = 1;
        }
        for (int j = 0; j < k; ++j) {
            int best = -1;
            for (int e = 0; e < E; ++e) {
                if (!gkeep[e / G]) continue;
                int taken = 0;
                for (int i = 0; i < j; ++i) if (idx[(long)t * k + i] == e) taken = 1;
                if (taken) continue;
                if (best < 0 || v[e] > v[best]) best = e;
            }
            idx[(long)t * k + j] = best;
        }
    }
    free(gscore);
    free(gkeep);
}

/* gates[t,j] = s[t, idx[t,j]] (/ sum over the selected when norm) * route_scale */
void oc_gates(int T, int E, int k, int norm, double route_scale, const double* s, const int32_t* idx,
              double* gates) {
    for (int t = 0; t < T; ++t) {
        double z = 0.0;
        for (int j = 0; j < k; ++j) z += s[(long)t * E + idx[(long)t * k + j]];
        for (int j = 0; j < k; ++j) {
            double g = s[(long)t * E + idx[(long)t * k + j]];
            if (norm) g /= z;
            gates[(long)t * k + j] = g * route_scale;
        }
    }
}

/* Expert-contiguous order: counts, exclusive-scan offsets, and a stable
 * counting sort of the flattened pairs (t*k + j) by expert. */
void oc_maps(int T, int E, int k, const int32_t* idx, int32_t* counts, int32_t* offsets, int32_t* row_of,
             int32_t* src_of) {
    for (int e = 0; e < E; ++e) counts[e] = 0;
    for (long p = 0; p < (long)T * k; ++p) counts[idx[p]] += 1;
    offsets[0] = 0;
    for (int e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];
    int32_t* fill = (int32_t*)malloc(sizeof(int32_t) * E);
    for (int e = 0; e < E; ++e) fill[e] = offsets[e];
    for (long p = 0; p < (long)T * k; ++p) {
        int e = idx[p];
        int r = fill[e]++;
        row_of[p] = r;
        src_of[r] = (int32_t)(p / k);
    }
    free(fill);
}

/*
 * Capacity factor (the expert-slot limit the practice cases name as the first
 * knob for imbalance: an expert whose slots are full drops the excess tokens).
 * Reading: C = ceil(cf * T * k / E) slots per expert; an expert keeps the
 * first C of its (token, slot) pairs in ascending token order and drops the
 * rest; cf <= 0 means no limit. keep[t*k + j] = 1 for kept pairs, 0 for
 * dropped ones. Returns C (or T*k without a limit).
 */
int oc_capacity_keep(int T, int E, int k, double cf, const int32_t* idx, uint8_t* keep) {
    long cap = (long)T * k;
    if (cf > 0.0) {
        double c = ceil(cf * (double)T * (double)k / (double)E);
        cap = c < (double)cap ? (long)c : cap;
    }
    long* seen = (long*)calloc(E, sizeof(long));
    for (long p = 0; p < (long)T * k; ++p) {
        int e = idx[p];
        keep[p] = (uint8_t)(seen[e] < cap);
        seen[e] += 1;
    }
    free(seen);
    return (int)cap;
}

/* Maps of the kept pairs only (keep == NULL: every pair): counts of kept pairs,
 * offsets, the stable order, and row_of = -1 for dropped pairs. */
void oc_maps_kept(int T, int E, int k, const int32_t* idx, const uint8_t* keep, int32_t* counts, int32_t* offsets,
                  int32_t* row_of, int32_t* src_of) {
    for (int e = 0; e < E; ++e) counts[e] = 0;
    for (long p = 0; p < (long)T * k; ++p)
        if (!keep || keep[p]) counts[idx[p]] += 1;
    offsets[0] = 0;
    for (int e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];
    int32_t* fill = (int32_t*)malloc(sizeof(int32_t) * E);
    for (int e = 0; e < E; ++e) fill[e] = offsets[e];
    for (long p = 0; p < (long)T * k; ++p) {
        if (keep && !keep[p]) {
            row_of[p] = -1;
            continue;
        }
        int e = idx[p];
        int r = fill[e]++;
        row_of[p] = r;
        src_of[r] = (int32_t)(p / k);
    }
    free(fill);
}

/* aux = E * sum_e f_e P_e, f_e = counts[e]/(T k), P_e = mean_t s[t,e] (full softmax). */
double oc_aux(int T, int E, int k, const double* s, const int32_t* counts) {
    double acc = 0.0;
    for (int e = 0; e < E; ++e) {
        double P = 0.0;
        for (int t = 0; t < T; ++t) P += s[(long)t * E + e];
        P /= (double)T;
        double f = (double)counts[e] / ((double)T * k);
        acc += f * P;
    }
    return (double)E * acc;
}

/* ------------------------------------------------------------ experts */

/* One expert on one token vector xv [H]:
 *   z_g = W_g xv, z_u = W_u xv, a = silu(z_g) * z_u   (W_g, W_u: [F, H])
 * With mx != 0 the activation fed to the down projection is rounded to MXFP8
 * after the gate is folded in (see oc_moe_fwd_tokens). */
static void expert_act(const oc_mat* Wg, const oc_mat* Wu, const double* xv, double* zg, double* zu, double* a,
                       double* rowbuf) {
    int F = (int)Wg->rows;
    matvec(Wg, xv, zg, rowbuf);
    matvec(Wu, xv, zu, rowbuf);
    for (int f = 0; f < F; ++f) a[f] = silu(zg[f]) * zu[f];
}

/* The gate-folded activation as the down projection's operand: MXFP8 blocks
 * along F (MXFP8 recipe) or bf16 (BF16 recipe). */
static void round_act(double* a, int F, int recipe) {
    if (is_mx(recipe)) mx_roundtrip(a, F);
    else if (is_nv(recipe)) nv_roundtrip(a, F);
    else if (recipe == OC_BF16R) round_vec(a, F, recipe);
}

/*
 * Forward output rows for a list of tokens, given the routing.
 *
 *   y[t] = sum_j g[t,j] * W_d[e_j] (silu(W_g[e_j] x_t) * (W_u[e_j] x_t))
 *          (+ shared expert on every token, weight 1)
 *
 * A slot with idx < 0 (a pair dropped at an expert's capacity) is skipped.
 * fold = 1 evaluates W_d (g a) (the memory-efficient permutation order),
 * fold = 0 evaluates g (W_d a); the two agree up to rounding.
 * recipe (OC_EXACT / OC_MX / OC_BF16R / OC_NV) selects the rounding points:
 *   OC_MX: x is rounded to MXFP8 (1x32 blocks along H) before the expert
 *     GEMMs, the gate-folded activation g*a (and the shared expert's a) to
 *     MXFP8 along F before the down projection; the weights are given as
 *     OC_MXFP8 matrices (already quantised);
 *   OC_NV: as OC_MX with NVFP4 (16-blocks, G = 1) in place of MXFP8 and
 *     OC_NVFP4 weight matrices;
 *   OC_BF16R: g*a (and the shared a) is rounded to bf16;
 *   all three: each expert's down-projection output is rounded to bf16 before
 *     the sum. y itself is returned unrounded.
 *   OC_MXQ / OC_NVQ: the quantisation points of OC_MX / OC_NV only (x, the
 *     weights and the gate-folded activation); expert outputs stay unrounded.
 * Weight layouts: Wg, Wu [E*F, H]; Wd [E*H, F]; shared Wgs, Wus [F, H], Wds [H, F].
 */
int oc_moe_fwd_tokens(int T, int H, int E, int k, int F, int S, int recipe, int fold, const oc_mat* x,
                      const oc_mat* Wg, const oc_mat* Wu, const oc_mat* Wd, const oc_mat* Wgs, const oc_mat* Wus,
                      const oc_mat* Wds, const int32_t* idx, const double* gates, int n_tok, const int32_t* toks,
                      double* y_out, double* shared_out) {
    int i;
    (void)T;
    (void)E;
#pragma omp parallel for schedule(dynamic, 1)
    for (i = 0; i < n_tok; ++i) {
        int t = toks[i];
        int maxd = H > F ? H : F;
        double* xv = (double*)malloc(sizeof(double) * H);
        double* zg = (double*)malloc(sizeof(double) * F);
        double* zu = (double*)malloc(sizeof(double) * F);
        double* a = (double*)malloc(sizeof(double) * F);
        double* o = (double*)malloc(sizeof(double) * H);
        double* rowbuf = (double*)malloc(sizeof(double) * maxd);
        double* y = y_out + (long)i * H;
        oc_row(x, t, xv);
        if (is_mx(recipe)) mx_roundtrip(xv, H);
        else if (is_nv(recipe)) nv_roundtrip(xv, H);
        for (int h = 0; h < H; ++h) y[h] = 0.0;
        for (int j = 0; j < k; ++j) {
            int e = idx[(long)t * k + j];
            double g = gates[(long)t * k + j];
            if (e < 0) continue; /* a pair dropped at an expert's capacity contributes nothing */
            oc_mat we_g = oc_slice(Wg, (int64_t)e * F, F);
            oc_mat we_u = oc_slice(Wu, (int64_t)e * F, F);
            oc_mat we_d = oc_slice(Wd, (int64_t)e * H, H);
            expert_act(&we_g, &we_u, xv, zg, zu, a, rowbuf);
            if (fold) {
                for (int f = 0; f < F; ++f) a[f] *= g;
                round_act(a, F, recipe);
                matvec(&we_d, a, o, rowbuf);
                round_vec(o, H, recipe);
                for (int h = 0; h < H; ++h) y[h] += o[h];
            } else {
                round_act(a, F, recipe);
                matvec(&we_d, a, o, rowbuf);
                round_vec(o, H, recipe);
                for (int h = 0; h < H; ++h) y[h] += g * o[h];
            }
        }
        if (S) {
            expert_act(Wgs, Wus, xv, zg, zu, a, rowbuf);
            round_act(a, F, recipe);
            matvec(Wds, a, o, rowbuf);
            round_vec(o, H, recipe);
            for (int h = 0; h < H; ++h) y[h] += o[h];
            if (shared_out)
                for (int h = 0; h < H; ++h) shared_out[(long)i * H + h] = o[h];
        }
        free(xv); free(zg); free(zu); free(a); free(o); free(rowbuf);
    }
    return 0;
}

/*
 * Dense all-experts brute force (a pin for the per-token loop): every expert is
 * evaluated on every token and the results are combined with a dense [T,E]
 * gate matrix that is zero off the selected experts. No routing lists at all.
 */
int oc_moe_fwd_dense(int T, int H, int E, int F, const oc_mat* x, const oc_mat* Wg, const oc_mat* Wu,
                     const oc_mat* Wd, const double* gate_dense, double* y_out) {
    int t;
#pragma omp parallel for schedule(dynamic, 1)
    for (t = 0; t < T; ++t) {
        int maxd = H > F ? H : F;
        double* xv = (double*)malloc(sizeof(double) * H);
        double* zg = (double*)malloc(sizeof(double) * F);
        double* zu = (double*)malloc(sizeof(double) * F);
        double* a = (double*)malloc(sizeof(double) * F);
        double* o = (double*)malloc(sizeof(double) * H);
        double* rowbuf = (double*)malloc(sizeof(double) * maxd);
        oc_row(x, t, xv);
        for (int h = 0; h < H; ++h) y_out[(long)t * H + h] = 0.0;
        for (int e = 0; e < E; ++e) {
            oc_mat we_g = oc_slice(Wg, (int64_t)e * F, F);
            oc_mat we_u = oc_slice(Wu, (int64_t)e * F, F);
            oc_mat we_d = oc_slice(Wd, (int64_t)e * H, H);
            expert_act(&we_g, &we_u, xv, zg, zu, a, rowbuf);
            matvec(&we_d, a, o, rowbuf);
            for (int h = 0; h < H; ++h) y_out[(long)t * H + h] += gate_dense[(long)t * E + e] * o[h];
        }
        free(xv); free(zg); free(zu); free(a); free(o); free(rowbuf);
    }
    return 0;
}

/* Expert part of the layer for explicit (row -> expert, gate) lists, the way
 * the grouped GEMM stage sees it: a row r holds activation xp[r] routed to
 * expert e_of[r] with gate g_of[r]. Outputs z_g, z_u [n, F] (unrounded),
 * ap [n, F] = g * silu(z_g) * z_u rounded per `recipe` (it is the down
 * projection's operand), and o [n, H] = W_d ap (rounded to bf16 under the MX
 * and BF16 recipes). Rows are independent. */
int oc_expert_rows(int H, int F, int recipe, const oc_mat* xp, const int32_t* e_of, const double* g_of,
                   const oc_mat* Wg, const oc_mat* Wu, const oc_mat* Wd, int n, const int32_t* rows,
                   double* zg_out, double* zu_out, double* ap_out, double* o_out) {
    int i;
#pragma omp parallel for schedule(dynamic, 1)
    for (i = 0; i < n; ++i) {
        int r = rows[i];
        int e = e_of[r];
        int maxd = H > F ? H : F;
        double* xv = (double*)malloc(sizeof(double) * H);
        double* zg = (double*)malloc(sizeof(double) * F);
        double* zu = (double*)malloc(sizeof(double) * F);
        double* a = (double*)malloc(sizeof(double) * F);
        double* rowbuf = (double*)malloc(sizeof(double) * maxd);
        oc_row(xp, r, xv);
        if (is_mx(recipe)) mx_roundtrip(xv, H);
        else if (is_nv(recipe)) nv_roundtrip(xv, H);
        oc_mat we_g = oc_slice(Wg, (int64_t)e * F, F);
        oc_mat we_u = oc_slice(Wu, (int64_t)e * F, F);
        oc_mat we_d = oc_slice(Wd, (int64_t)e * H, H);
        expert_act(&we_g, &we_u, xv, zg, zu, a, rowbuf);
        for (int f = 0; f < F; ++f) a[f] *= g_of[r];
        round_act(a, F, recipe);
        if (zg_out) for (int f = 0; f < F; ++f) zg_out[(long)i * F + f] = zg[f];
        if (zu_out) for (int f = 0; f < F; ++f) zu_out[(long)i * F + f] = zu[f];
        if (ap_out) for (int f = 0; f < F; ++f) ap_out[(long)i * F + f] = a[f];
        if (o_out) {
            matvec(&we_d, a, o_out + (long)i * H, rowbuf);
            round_vec(o_out + (long)i * H, H, recipe);
        }
        free(xv); free(zg); free(zu); free(a); free(rowbuf);
    }
    return 0;
}

/* ------------------------------------------------------------ backward */

/*
 * Derivative of the forward (bf16 / fp64 operands, softmax or sigmoid scores
 * with selected-normalised gates), for upstream dY [T,H] and d_aux.
 * Per token t of the list:
 *   for each selected j (e = idx[t,j]):
 *     z_g, z_u, a = silu(z_g) z_u, v = W_d[e]^T dY_t,  dg_j = <v, a>
 *     da = g_j v, dz_g = da z_u silu'(z_g), dz_u = da silu(z_g)
 *     dx_t += W_g[e]^T dz_g + W_u[e]^T dz_u
 *   gate path (c = route_scale, p = softmax over the selected logits):
 *     softmax, normalised: g_j = c p_j, so
 *       dl[sel_j] = g_j dg_j - g_j (sum_i g_i dg_i) / c
 *     sigmoid, normalised: g_j = c s_j / Z, s = sigmoid(l), Z = sum_sel s_i, so
 *       dl[sel_j] = s_j (1 - s_j) (c/Z) (dg_j - (sum_i g_i dg_i) / c)
 *     softmax, unnormalised: g_j = c s_j, dl = s (ds - <s, ds>), ds_{e_j} = c dg_j
 *   aux path (softmax only, counts are constants):
 *     c_e = E count_e / (T k) / T,  dl[t,e] += d_aux s_e (c_e - sum_i s_i c_i)
 *   router: dx_t += sum_e dl[t,e] W_r[e]
 * recipe OC_BF16R applies the BF16 recipe's rounding points: z_g and z_u are
 * the saved bf16 pre-activations (a, silu, silu' are computed from them),
 * dz_g and dz_u are rounded to bf16, each selected expert's contribution
 * W_g^T dz_g + W_u^T dz_u is rounded to bf16, and the router path uses dl
 * rounded to bf16 and rounds its result to bf16. dl itself stays unrounded.
 * Under OC_MX (the MXFP8 backward): z is recomputed from MXFP8 x and the
 * forward's MXFP8 weights and rounded to bf16 (the saved pre-activations);
 * v = W_d^T dY takes WdT (W_d^T [E*F, H], MXFP8 along H) and dY in MXFP8 along
 * H; dz_g, dz_u are rounded to bf16 and then to MXFP8 along F, and the gate/up
 * dgrad takes WgT, WuT (W_g^T, W_u^T [E*H, F], MXFP8 along F); its result and
 * the router path are rounded as under OC_BF16R. (WdT, WgT, WuT are unused
 * otherwise and may be NULL.) OC_MXQ takes the same MXFP8 operands as OC_MX
 * but rounds nothing to bf16 (z, dz_g, dz_u, the dXp contributions and the
 * router path stay fp64).
 * logits, s (scores), gates, idx and counts are the forward's (counts: every
 * selected pair, as the router counted them for aux). keep: NULL, or the
 * capacity mask of oc_capacity_keep: a dropped pair contributes nothing to y,
 * so it gets dg = 0 and no expert gradient, while its score still enters the
 * normalisation of the other gates.
 */
int oc_moe_bwd_tokens(int T, int H, int E, int k, int F, int score, int norm, double route_scale, int aux_on,
                      double d_aux, int recipe, const oc_mat* x, const oc_mat* Wr, const oc_mat* Wg,
                      const oc_mat* Wu, const oc_mat* Wd, const oc_mat* WdT, const oc_mat* WgT, const oc_mat* WuT,
                      const oc_mat* dY, const int32_t* idx, const double* s_all,
                      const double* s_softmax, const int32_t* counts, const uint8_t* keep, int n_tok,
                      const int32_t* toks, double* dx_out, double* dl_out, double* dg_out) {
    int i;
#pragma omp parallel for schedule(dynamic, 1)
    for (i = 0; i < n_tok; ++i) {
        int t = toks[i];
        int maxd = H > F ? H : F;
        double* xv = (double*)malloc(sizeof(double) * H);
        double* dy = (double*)malloc(sizeof(double) * H);
        double* zg = (double*)malloc(sizeof(double) * F);
        double* zu = (double*)malloc(sizeof(double) * F);
        double* a = (double*)malloc(sizeof(double) * F);
        double* v = (double*)malloc(sizeof(double) * F);
        double* dzg = (double*)malloc(sizeof(double) * F);
        double* dzu = (double*)malloc(sizeof(double) * F);
        double* dxp = (double*)malloc(sizeof(double) * H);
        double* rowbuf = (double*)malloc(sizeof(double) * maxd);
        double* dg = (double*)malloc(sizeof(double) * k);
        double* g = (double*)malloc(sizeof(double) * k);
        double* dx = dx_out + (long)i * H;
        double* dl = dl_out + (long)i * E;
        const double* s = s_all + (long)t * E;
        oc_row(x, t, xv);
        oc_row(dY, t, dy);
        double* xe = xv;           /* the expert GEMMs' copy of x (MXFP8 along H under OC_MX) */
        double* dye = dy;          /* dY as the down dgrad's operand */
        double* xq = NULL;
        double* dyq = NULL;
        if (is_mx(recipe)) {
            xq = (double*)malloc(sizeof(double) * H);
            dyq = (double*)malloc(sizeof(double) * H);
            memcpy(xq, xv, sizeof(double) * H);
            memcpy(dyq, dy, sizeof(double) * H);
            mx_roundtrip(xq, H);
            mx_roundtrip(dyq, H);
            xe = xq;
            dye = dyq;
        }
        for (int h = 0; h < H; ++h) dx[h] = 0.0;
        for (int e = 0; e < E; ++e) dl[e] = 0.0;
        /* gates again from the scores (as the forward defined them) */
        double Z = 0.0;
        for (int j = 0; j < k; ++j) Z += s[idx[(long)t * k + j]];
        for (int j = 0; j < k; ++j) {
            double gj = s[idx[(long)t * k + j]];
            if (norm) gj /= Z;
            g[j] = gj * route_scale;
        }
        for (int j = 0; j < k; ++j) {
            int e = idx[(long)t * k + j];
            if (keep && !keep[(long)t * k + j]) {
                dg[j] = 0.0; /* dropped at capacity: the output does not depend on its gate */
                continue;
            }
            oc_mat we_g = oc_slice(Wg, (int64_t)e * F, F);
            oc_mat we_u = oc_slice(Wu, (int64_t)e * F, F);
            oc_mat we_d = oc_slice(Wd, (int64_t)e * H, H);
            expert_act(&we_g, &we_u, xe, zg, zu, a, rowbuf);
            if (recipe == OC_BF16R || recipe == OC_MX) {
                /* the backward reads the forward's gate/up pre-activations saved in bf16 */
                for (int f = 0; f < F; ++f) { zg[f] = oc_bf16_round(zg[f]); zu[f] = oc_bf16_round(zu[f]); }
                for (int f = 0; f < F; ++f) a[f] = silu(zg[f]) * zu[f];
            }
            if (is_mx(recipe)) {
                oc_mat wt_d = oc_slice(WdT, (int64_t)e * F, F);   /* W_d^T [F, H], MXFP8 along H */
                matvec(&wt_d, dye, v, rowbuf);                      /* v = W_d^T dY_t */
            } else {
                for (int f = 0; f < F; ++f) v[f] = 0.0;
                matvec_t_acc(&we_d, dy, v, rowbuf);           /* v = W_d^T dY_t */
            }
            dg[j] = dot(v, a, F);
            for (int f = 0; f < F; ++f) {
                double da = g[j] * v[f];
                dzg[f] = da * zu[f] * silu_grad(zg[f]);
                dzu[f] = da * silu(zg[f]);
            }
            if (recipe == OC_BF16R || recipe == OC_MX) {
                for (int f = 0; f < F; ++f) { dzg[f] = oc_bf16_round(dzg[f]); dzu[f] = oc_bf16_round(dzu[f]); }
            }
            for (int h = 0; h < H; ++h) dxp[h] = 0.0;
            if (is_mx(recipe)) {
                /* dgate/dup as the gate/up dgrad's operand: MXFP8 along F; W_g^T, W_u^T [H, F] MXFP8 along F */
                mx_roundtrip(dzg, F);
                mx_roundtrip(dzu, F);
                oc_mat wt_g = oc_slice(WgT, (int64_t)e * H, H);
                oc_mat wt_u = oc_slice(WuT, (int64_t)e * H, H);
                double* tmp = (double*)malloc(sizeof(double) * H);
                matvec(&wt_g, dzg, tmp, rowbuf);
                for (int h = 0; h < H; ++h) dxp[h] += tmp[h];
                matvec(&wt_u, dzu, tmp, rowbuf);
                for (int h = 0; h < H; ++h) dxp[h] += tmp[h];
                free(tmp);
            } else {
                matvec_t_acc(&we_g, dzg, dxp, rowbuf);
                matvec_t_acc(&we_u, dzu, dxp, rowbuf);
            }
            if (recipe == OC_BF16R || recipe == OC_MX) round_vec(dxp, H, OC_BF16R);
            for (int h = 0; h < H; ++h) dx[h] += dxp[h];
        }
        if (dg_out) for (int j = 0; j < k; ++j) dg_out[(long)i * k + j] = dg[j];
        /* gate path */
        double sgd = 0.0;
        for (int j = 0; j < k; ++j) sgd += g[j] * dg[j];
        for (int j = 0; j < k; ++j) {
            int e = idx[(long)t * k + j];
            if (score == 0) {
                if (norm) {
                    /* g_j = c exp(l_j) / sum_sel exp(l_i):  c p_j (dg_j - sum_i p_i dg_i) */
                    dl[e] += g[j] * dg[j] - g[j] * sgd / route_scale;
                }
                /* unnormalised softmax gates are handled below (all E logits move) */
            } else {
                double sj = s[e];
                if (norm) {
                    /* g_j = c s_j / Z, dg/ds_j: c/Z (dg_j - sum_i g_i dg_i / c) */
                    double dsj = (route_scale / Z) * (dg[j] - sgd / route_scale);
                    dl[e] += dsj * sj * (1.0 - sj);
                } else {
                    dl[e] += route_scale * dg[j] * sj * (1.0 - sj);
                }
            }
        }
        if (score == 0 && !norm) {
            /* g_j = c s_{e_j}, s = softmax over all E: ds_e = c dg_j at e = e_j */
            double* ds = (double*)calloc(E, sizeof(double));
            for (int j = 0; j < k; ++j) ds[idx[(long)t * k + j]] += route_scale * dg[j];
            double sds = 0.0;
            for (int e = 0; e < E; ++e) sds += s[e] * ds[e];
            for (int e = 0; e < E; ++e) dl[e] += s[e] * (ds[e] - sds);
            free(ds);
        }
        /* aux path */
        if (aux_on) {
            const double* ss = s_softmax + (long)t * E;
            double sc = 0.0;
            for (int e = 0; e < E; ++e) {
                double ce = (double)E * (double)counts[e] / ((double)T * k) / (double)T;
                sc += ss[e] * ce;
            }
            for (int e = 0; e < E; ++e) {
                double ce = (double)E * (double)counts[e] / ((double)T * k) / (double)T;
                dl[e] += d_aux * ss[e] * (ce - sc);
            }
        }
        /* router path */
        for (int h = 0; h < H; ++h) dxp[h] = 0.0;
        for (int e = 0; e < E; ++e) {
            double c = (recipe == OC_BF16R || recipe == OC_MX) ? oc_bf16_round(dl[e]) : dl[e];
            if (c == 0.0) continue;
            oc_row(Wr, e, rowbuf);
            for (int h = 0; h < H; ++h) dxp[h] += c * rowbuf[h];
        }
        if (recipe == OC_BF16R || recipe == OC_MX) round_vec(dxp, H, OC_BF16R);
        for (int h = 0; h < H; ++h) dx[h] += dxp[h];
        free(xq); free(dyq);
        free(xv); free(dy); free(zg); free(zu); free(a); free(v); free(dzg); free(dzu); free(dxp); free(rowbuf);
        free(dg); free(g);
    }
    return 0;
}

/*
 * Expert weight gradients for a list of experts, summing over every token
 * routed to each one (rows of the stable order, i.e. ascending token index):
 *   dW_d[e] += dY_t (x) (g a),  dW_g[e] += dz_g (x) x_t,  dW_u[e] += dz_u (x) x_t
 * Outputs: dWg, dWu [n_exp, F, H]; dWd [n_exp, H, F]. Experts with no token
 * get exact zeros. gates are the forward's [T,k]. Under OC_BF16R, g a is the
 * forward's bf16 activation (from the unrounded z), and dz_g, dz_u are the
 * bf16 values of the backward (from the saved bf16 z, rounded).
 * Under OC_MX (the MXFP8 backward): z is recomputed from MXFP8 x and weights
 * and rounded to bf16 (the saved pre-activations), g a is recomputed from it;
 * v = W_d^T dY uses WdT (W_d^T [E*F, H], MXFP8 along H) and dY in MXFP8 along
 * H; dz_g, dz_u are rounded to bf16; then every weight-gradient operand (g a,
 * dz_g, dz_u, x, dY) is quantised to MXFP8 along the expert's tokens, in blocks
 * of 32 consecutive tokens of its stable order. OC_MXQ: the same quantisation
 * with z, dz_g and dz_u unrounded.
 */
int oc_moe_bwd_expert_dw(int T, int H, int E, int k, int F, int recipe, const oc_mat* x, const oc_mat* Wg,
                         const oc_mat* Wu, const oc_mat* Wd, const oc_mat* WdT, const oc_mat* dY, const int32_t* idx,
                         const double* gates, int n_exp, const int32_t* exps, double* dWg, double* dWu,
                         double* dWd) {
    (void)E;
    for (int q = 0; q < n_exp; ++q) {
        int e = exps[q];
        double* gG = dWg + (long)q * F * H;
        double* gU = dWu + (long)q * F * H;
        double* gD = dWd + (long)q * H * F;
        memset(gG, 0, sizeof(double) * (size_t)F * H);
        memset(gU, 0, sizeof(double) * (size_t)F * H);
        memset(gD, 0, sizeof(double) * (size_t)F * H);
        /* tokens routed to e, with their gate */
        int n = 0;
        int32_t* tl = (int32_t*)malloc(sizeof(int32_t) * (T > 0 ? T : 1));
        double* gl = (double*)malloc(sizeof(double) * (T > 0 ? T : 1));
        for (int t = 0; t < T; ++t)
            for (int j = 0; j < k; ++j)
                if (idx[(long)t * k + j] == e) { tl[n] = t; gl[n] = gates[(long)t * k + j]; ++n; }
        oc_mat we_g = oc_slice(Wg, (int64_t)e * F, F);
        oc_mat we_u = oc_slice(Wu, (int64_t)e * F, F);
        oc_mat we_d = oc_slice(Wd, (int64_t)e * H, H);
        /* per-token intermediates, then the outer products; parallel over the
         * output rows so each thread owns its rows and the token order of each
         * sum stays ascending. */
        double* A = (double*)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1) * F);
        double* DZG = (double*)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1) * F);
        double* DZU = (double*)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1) * F);
        double* XV = (double*)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1) * H);
        double* DY = (double*)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1) * H);
        int i;
#pragma omp parallel for schedule(dynamic, 1)
        for (i = 0; i < n; ++i) {
            int maxd = H > F ? H : F;
            double* zg = (double*)malloc(sizeof(double) * F);
            double* zu = (double*)malloc(sizeof(double) * F);
            double* v = (double*)malloc(sizeof(double) * F);
            double* rowbuf = (double*)malloc(sizeof(double) * maxd);
            double* xv = XV + (long)i * H;
            double* dy = DY + (long)i * H;
            double* a = A + (long)i * F;
            oc_row(x, tl[i], xv);
            oc_row(dY, tl[i], dy);
            if (is_mx(recipe)) {
                /* the forward's gate/up GEMM saw x in MXFP8 along H; its bf16 pre-activations were
                 * saved (OC_MX; unrounded under OC_MXQ), and the backward recomputes g a from them */
                double* xq = (double*)malloc(sizeof(double) * H);
                double* dyq = (double*)malloc(sizeof(double) * H);
                memcpy(xq, xv, sizeof(double) * H);
                memcpy(dyq, dy, sizeof(double) * H);
                mx_roundtrip(xq, H);
                mx_roundtrip(dyq, H);
                expert_act(&we_g, &we_u, xq, zg, zu, a, rowbuf);
                if (recipe == OC_MX)
                    for (int f = 0; f < F; ++f) { zg[f] = oc_bf16_round(zg[f]); zu[f] = oc_bf16_round(zu[f]); }
                for (int f = 0; f < F; ++f) a[f] = gl[i] * silu(zg[f]) * zu[f];
                oc_mat wt_d = oc_slice(WdT, (int64_t)e * F, F);
                matvec(&wt_d, dyq, v, rowbuf);                      /* v = W_d^T dY_t, MXFP8 along H */
                free(xq);
                free(dyq);
            } else {
                expert_act(&we_g, &we_u, xv, zg, zu, a, rowbuf);
                /* A holds the down projection's operand g a */
                for (int f = 0; f < F; ++f) a[f] *= gl[i];
                if (recipe == OC_BF16R) {
                    round_vec(a, F, recipe);
                    round_vec(zg, F, recipe);
                    round_vec(zu, F, recipe);
                }
                for (int f = 0; f < F; ++f) v[f] = 0.0;
                matvec_t_acc(&we_d, dy, v, rowbuf);
            }
            for (int f = 0; f < F; ++f) {
                double da = gl[i] * v[f];
                DZG[(long)i * F + f] = da * zu[f] * silu_grad(zg[f]);
                DZU[(long)i * F + f] = da * silu(zg[f]);
            }
            if (recipe == OC_BF16R || recipe == OC_MX) {
                round_vec(DZG + (long)i * F, F, OC_BF16R);
                round_vec(DZU + (long)i * F, F, OC_BF16R);
            }
            free(zg); free(zu); free(v); free(rowbuf);
        }
        if (is_mx(recipe)) {
            /* weight-gradient GEMM operands: MXFP8 along the expert's tokens (K = its rows), in blocks of
             * 32 consecutive tokens of its stable order; x and dY from their bf16 values */
            int c;
#pragma omp parallel for schedule(static)
            for (c = 0; c < F; ++c) {
                mx_roundtrip_strided(A + c, n, F);
                mx_roundtrip_strided(DZG + c, n, F);
                mx_roundtrip_strided(DZU + c, n, F);
            }
#pragma omp parallel for schedule(static)
            for (c = 0; c < H; ++c) {
                mx_roundtrip_strided(XV + c, n, H);
                mx_roundtrip_strided(DY + c, n, H);
            }
        }
        int f;
#pragma omp parallel for schedule(static)
        for (f = 0; f < F; ++f) {
            for (int ii = 0; ii < n; ++ii) {
                double cg = DZG[(long)ii * F + f], cu = DZU[(long)ii * F + f];
                const double* xv = XV + (long)ii * H;
                for (int h = 0; h < H; ++h) {
                    gG[(long)f * H + h] += cg * xv[h];
                    gU[(long)f * H + h] += cu * xv[h];
                }
            }
        }
        int h;
#pragma omp parallel for schedule(static)
        for (h = 0; h < H; ++h) {
            for (int ii = 0; ii < n; ++ii) {
                double c = DY[(long)ii * H + h];
                const double* a = A + (long)ii * F;
                for (int f2 = 0; f2 < F; ++f2) gD[(long)h * F + f2] += c * a[f2];
            }
        }
        free(tl); free(gl); free(A); free(DZG); free(DZU); free(XV); free(DY);
    }
    return 0;
}

/* dW_r[e,h] = sum_t dl[t,e] x[t,h] over all T tokens (ascending t); with
 * round_dl the bf16 value of dl is used (the BF16 recipe's operand). */
void oc_router_dwr(int T, int H, int E, const double* dl, int round_dl, const oc_mat* x, double* dWr) {
    int e;
#pragma omp parallel for schedule(static)
    for (e = 0; e < E; ++e) {
        double* xr = (double*)malloc(sizeof(double) * H);
        double* out = dWr + (long)e * H;
        for (int h = 0; h < H; ++h) out[h] = 0.0;
        for (int t = 0; t < T; ++t) {
            double c = dl[(long)t * E + e];
            if (round_dl) c = oc_bf16_round(c);
            if (c == 0.0) continue;
            oc_row(x, t, xr);
            for (int h = 0; h < H; ++h) out[h] += c * xr[h];
        }
        free(xr);
    }
}

/* Unpermute-sum with unit weights: y[t] = sum_j o[row_of[t,j]] (+ shared[t]). */
void oc_unpermute(int T, int H, int k, const double* o, const int32_t* row_of, const double* shared, double* y) {
    for (int t = 0; t < T; ++t)
        for (int h = 0; h < H; ++h) {
            double s = 0.0;
            for (int j = 0; j < k; ++j) s += o[(long)row_of[(long)t * k + j] * H + h];
            if (shared) s += shared[(long)t * H + h];
            y[(long)t * H + h] = s;
        }
}

int oc_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
