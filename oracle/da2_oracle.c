/*
 * da2_oracle.c -- plain, slow float64 CPU oracle for the DraftAttention2
 * attention hot path ("DraftAttention2", paperpeel.com/paper/2609.32628.md).
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the parity checker for the CUDA
 * library; only the tests, the smoke check and the CPU-baseline leg of the
 * benchmark may load it.  It shares no code, header, table or constant
 * generator with the CUDA path.
 *
 * What it computes, step by step, in the order of the paper:
 *   1. spatial partition of each frame into R_f = ceil(Hv*Wv/C) connected,
 *      balanced regions (Sec. 3.3 "Fused quantization and reordering";
 *      App. C.2, whose formula is cut off on the page);
 *   2. pooled draft descriptors: region mean and channel-wise max of Q and K
 *      over the valid tokens (Eq. 2; App. C.1);
 *   3. draft map A = (1-lambda) softmax_row(Qbar Kbar^T/sqrt d)
 *                   + lambda softmax_row(Qmax Kmax^T/sqrt d)      (Eq. 3);
 *   4. per-head ranking of all R^2 region pairs, ties by pair index, integer
 *      quotas, precision assignment 8 / 4 / skip (Sec. 3.1 "Joint allocation
 *      of sparsity and precision"; App. C.1);
 *   5. operand quantization: FP8 e4m3 with one scale per 64-token tile, and
 *      two-level NVFP4 (e2m1 codes, e4m3 scale per 16 elements, fp32 tile
 *      scale) (App. C.1 "Routing and precision formats");
 *   6. block-sparse attention with one softmax state and one numerator shared
 *      by both precision phases, the probabilities quantized for the
 *      probability-value product, and the unquantized denominator Z^q
 *      (App. B.3 "Weight quantization under shared normalization"; Sec. 3.3
 *      "Cross-precision accumulation", Eq. 8, whose body is garbled on the
 *      page); rows without a retained valid key return zero (App. C.1);
 *      the original token order is restored on output.
 *
 * Floating point: all attention arithmetic is float64.  The draft map is
 * computed in float64 with a fixed operation order (fma chains in ascending
 * channel order, sums in ascending index order, and the exponential o_exp
 * below) so that the ranking it induces is reproducible bit for bit.  The
 * quantizers use float32 IEEE round-to-nearest operations, as the formats
 * they feed are float32-scaled.  Build with -ffp-contract=off so that no
 * multiply-add is fused behind our back.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define O_BLOCK 64 /* attention block size: one region per 64-token block */

/* ------------------------------------------------------------------------ */
/* Number formats (OCP FP8 E4M3 "fn" and FP4 E2M1), written from the format  */
/* definitions: sign, exponent, mantissa, round to nearest even, saturating. */
/* ------------------------------------------------------------------------ */

/* E4M3: bias 7, 3 mantissa bits, no infinities, largest finite 448,
   smallest subnormal 2^-9. */
double oracle_e4m3_decode(uint8_t code) {
    int s = (code >> 7) & 1, e = (code >> 3) & 15, m = code & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) v = ldexp((double)m, -9);
    else v = ldexp(1.0 + m / 8.0, e - 7);
    return s ? -v : v;
}

static uint8_t e4m3_bits_of_value(double v) { /* v >= 0, exactly representable */
    if (v == 0.0) return 0;
    int ex;
    frexp(v, &ex);
    int E = ex - 1; /* v in [2^E, 2^(E+1)) */
    if (E < -6) return (uint8_t)(v / ldexp(1.0, -9)); /* subnormal */
    int mant = (int)((v / ldexp(1.0, E) - 1.0) * 8.0);
    return (uint8_t)(((E + 7) << 3) | mant);
}

uint8_t oracle_e4m3_encode(float x) {
    uint8_t sign = signbit(x) ? 0x80 : 0x00;
    double a = fabs((double)x);
    if (isnan(x)) return 0x7F;
    if (a >= 448.0) return (uint8_t)(sign | 0x7E); /* saturate to 448 */
    int ex;
    frexp(a, &ex);
    int E = ex - 1;
    if (a == 0.0 || E < -6) E = -6;            /* subnormal spacing 2^-9 */
    double ulp = ldexp(1.0, E - 3);
    double v = rint(a / ulp) * ulp;           /* ties to even */
    if (v > 448.0) v = 448.0;
    return (uint8_t)(sign | e4m3_bits_of_value(v));
}

/* E2M1: bias 1, 1 mantissa bit; values 0, 0.5, 1, 1.5, 2, 3, 4, 6. */
double oracle_e2m1_decode(uint8_t code) {
    static const double mag[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};
    double v = mag[code & 7];
    return (code & 8) ? -v : v;
}

uint8_t oracle_e2m1_encode(float x) {
    uint8_t sign = signbit(x) ? 0x8 : 0x0;
    double a = fabs((double)x);
    if (a >= 6.0) return (uint8_t)(sign | 0x7);
    int ex;
    frexp(a, &ex);
    int E = ex - 1;
    if (a == 0.0 || E < 0) E = 0;              /* subnormal spacing 0.5 */
    double ulp = ldexp(1.0, E - 1);
    double v = rint(a / ulp) * ulp;
    if (v > 6.0) v = 6.0;
    uint8_t bits;
    if (v == 0.0) bits = 0;
    else if (v == 0.5) bits = 1;
    else {
        int vex;
        frexp(v, &vex);
        int VE = vex - 1; /* 0..2 */
        int mant = (int)((v / ldexp(1.0, VE) - 1.0) * 2.0);
        bits = (uint8_t)(((VE + 1) << 1) | mant);
    }
    return (uint8_t)(sign | bits);
}

/* ------------------------------------------------------------------------ */
/* exp for the draft softmax: Cody-Waite argument reduction x = k ln2 + r    */
/* (two-part ln2), e^r by its Taylor series to degree 13 in Horner form with */
/* fma, scaling by 2^k.  Results that would be subnormal are flushed to 0.   */
/* The constants are the correctly rounded doubles of 1/ln2, of ln2 cut to   */
/* 32 significant bits (LN2_HI) and of the remainder (LN2_LO), and of 1/n!.  */
/* ------------------------------------------------------------------------ */
static const double O_LOG2E = 0x1.71547652b82fep+0;
static const double O_LN2_HI = 0x1.62e42fee00000p-1;
static const double O_LN2_LO = 0x1.a39ef35793c76p-33;
static const double O_INV_FACT[14] = {
    0x1.0000000000000p+0,  0x1.0000000000000p+0,  0x1.0000000000000p-1,
    0x1.5555555555555p-3,  0x1.5555555555555p-5,  0x1.1111111111111p-7,
    0x1.6c16c16c16c17p-10, 0x1.a01a01a01a01ap-13, 0x1.a01a01a01a01ap-16,
    0x1.71de3a556c734p-19, 0x1.27e4fb7789f5cp-22, 0x1.ae64567f544e4p-26,
    0x1.1eed8eff8d898p-29, 0x1.6124613a86d09p-33};

double oracle_exp(double x) {
    if (x < -708.0) return 0.0;
    if (x > 709.0) return INFINITY;
    double k = rint(x * O_LOG2E);
    double r = fma(-k, O_LN2_HI, x);
    r = fma(-k, O_LN2_LO, r);
    double p = O_INV_FACT[13];
    for (int n = 12; n >= 0; --n) p = fma(p, r, O_INV_FACT[n]);
    return ldexp(p, (int)k);
}

/* ------------------------------------------------------------------------ */
/* 1. Spatial partition (Sec. 3.3; App. C.2).                                */
/* Reading of the truncated C.2: R_f = ceil(n/C) regions per frame with      */
/* balanced sizes (the first n mod R_f regions one token larger).  Candidate */
/* partitions: for nb = 1..Hv, split the rows into nb bands of balanced      */
/* height (taller bands first); walk the bands boustrophedon (even bands     */
/* left to right, odd bands right to left), inside a band column by column, */
/* alternating top-down and bottom-up; cut the walk into the R_f chunks.     */
/* Keep candidates whose regions are all 4-connected; take the smallest      */
/* total perimeter, ties to the smaller nb.  Region j of frame f is block    */
/* a = f*R_f + j; a token's slot is its position in the walk of its region.  */
/* ------------------------------------------------------------------------ */
static void walk_order(int Hv, int Wv, int nb, int* cell_of_step) {
    int base = Hv / nb, rem = Hv % nb, r0 = 0, step = 0;
    for (int i = 0; i < nb; ++i) {
        int h = base + (i < rem ? 1 : 0);
        for (int k = 0; k < Wv; ++k) {
            int x = (i % 2 == 0) ? k : (Wv - 1 - k);
            for (int t = 0; t < h; ++t) {
                int y = (k % 2 == 0) ? (r0 + t) : (r0 + h - 1 - t);
                cell_of_step[step++] = y * Wv + x;
            }
        }
        r0 += h;
    }
}

static int region_connected(int Hv, int Wv, const int* reg, int j, int start_cell, int count,
                            int* stack, char* seen) {
    int top = 0, found = 0;
    stack[top++] = start_cell;
    seen[start_cell] = 1;
    while (top) {
        int c = stack[--top];
        ++found;
        int y = c / Wv, x = c % Wv;
        int nbr[4] = {y > 0 ? c - Wv : -1, y < Hv - 1 ? c + Wv : -1, x > 0 ? c - 1 : -1,
                      x < Wv - 1 ? c + 1 : -1};
        for (int q = 0; q < 4; ++q) {
            int n = nbr[q];
            if (n >= 0 && !seen[n] && reg[n] == j) {
                seen[n] = 1;
                stack[top++] = n;
            }
        }
    }
    return found == count;
}

/* Returns R_f (>0) and fills region_of[Hv*Wv], slot_of[Hv*Wv], n_a[R_f];
   returns -1 on bad arguments. */
int oracle_partition(int Hv, int Wv, int C, int* region_of, int* slot_of, int* n_a) {
    if (Hv <= 0 || Wv <= 0 || C <= 0) return -1;
    int n = Hv * Wv;
    int Rf = (n + C - 1) / C;
    int* sizes = (int*)malloc(sizeof(int) * Rf);
    for (int j = 0; j < Rf; ++j) sizes[j] = n / Rf + (j < n % Rf ? 1 : 0);
    int* walk = (int*)malloc(sizeof(int) * n);
    int* reg = (int*)malloc(sizeof(int) * n);
    int* slot = (int*)malloc(sizeof(int) * n);
    int* stack = (int*)malloc(sizeof(int) * n);
    char* seen = (char*)malloc(n);
    long best_perim = -1;
    int best_nb = -1, any_connected = 0;
    for (int pass = 0; pass < 2 && best_nb < 0; ++pass) {
        for (int nb = 1; nb <= Hv; ++nb) {
            walk_order(Hv, Wv, nb, walk);
            int step = 0;
            for (int j = 0; j < Rf; ++j)
                for (int s = 0; s < sizes[j]; ++s, ++step) {
                    reg[walk[step]] = j;
                    slot[walk[step]] = s;
                }
            int ok = 1;
            memset(seen, 0, n);
            step = 0;
            for (int j = 0; j < Rf && ok; ++j) {
                ok = region_connected(Hv, Wv, reg, j, walk[step], sizes[j], stack, seen);
                step += sizes[j];
            }
            if (!ok && pass == 0) continue;
            any_connected |= ok;
            long perim = 0;
            for (int c = 0; c < n; ++c) {
                int y = c / Wv, x = c % Wv;
                perim += (y == 0 || reg[c - Wv] != reg[c]);
                perim += (y == Hv - 1 || reg[c + Wv] != reg[c]);
                perim += (x == 0 || reg[c - 1] != reg[c]);
                perim += (x == Wv - 1 || reg[c + 1] != reg[c]);
            }
            if (best_nb < 0 || perim < best_perim) {
                best_perim = perim;
                best_nb = nb;
            }
        }
    }
    (void)any_connected;
    walk_order(Hv, Wv, best_nb, walk);
    int step = 0;
    for (int j = 0; j < Rf; ++j) {
        n_a[j] = sizes[j];
        for (int s = 0; s < sizes[j]; ++s, ++step) {
            region_of[walk[step]] = j;
            slot_of[walk[step]] = s;
        }
    }
    free(sizes); free(walk); free(reg); free(slot); free(stack); free(seen);
    return Rf;
}

/* ------------------------------------------------------------------------ */
/* Shapes and the token <-> slot tables.                                     */
/* ------------------------------------------------------------------------ */
/* Prefix (text) tokens, App. C.1: the precision budget counts only pairs  */
/* of video regions.  Reading of the sequence layout, which the pages       */
/* do not give: the P prefix tokens come first (positions 0..P-1), the      */
/* video tokens follow in raster order (P + f*Hv*Wv + y*Wv + x).  The       */
/* prefix is packed into Rp = ceil(P/64) blocks of consecutive tokens, which */
/* follow the Rv video blocks: block Rv + i holds tokens 64i .. 64i+63.     */
typedef struct {
    int B, H, d, F, Hv, Wv, P;
    int Rf, Rv, Rp, R, N, Npad; /* R = Rv + Rp blocks */
    int* slot_token; /* [Npad] token index of packed slot, -1 for padding */
    int* n_a;        /* [R] valid tokens of region (block) a */
} o_geom;

static int geom_make_p(o_geom* g, int B, int H, int d, int F, int Hv, int Wv, int P) {
    if (P < 0) return -1;
    g->B = B; g->H = H; g->d = d; g->F = F; g->Hv = Hv; g->Wv = Wv; g->P = P;
    int n = Hv * Wv;
    int* region_of = (int*)malloc(sizeof(int) * n);
    int* slot_of = (int*)malloc(sizeof(int) * n);
    int* nf = (int*)malloc(sizeof(int) * n);
    int Rf = oracle_partition(Hv, Wv, O_BLOCK, region_of, slot_of, nf);
    if (Rf <= 0) { free(region_of); free(slot_of); free(nf); return -1; }
    g->Rf = Rf; g->Rv = F * Rf; g->Rp = (P + O_BLOCK - 1) / O_BLOCK; g->R = g->Rv + g->Rp;
    g->N = P + F * n; g->Npad = g->R * O_BLOCK;
    g->slot_token = (int*)malloc(sizeof(int) * g->Npad);
    g->n_a = (int*)malloc(sizeof(int) * g->R);
    for (int i = 0; i < g->Npad; ++i) g->slot_token[i] = -1;
    for (int f = 0; f < F; ++f) {
        for (int j = 0; j < Rf; ++j) g->n_a[f * Rf + j] = nf[j];
        for (int c = 0; c < n; ++c) {
            int a = f * Rf + region_of[c];
            g->slot_token[a * O_BLOCK + slot_of[c]] = P + f * n + c;
        }
    }
    for (int i = 0; i < g->Rp; ++i) {
        int a = g->Rv + i, cnt = P - i * O_BLOCK < O_BLOCK ? P - i * O_BLOCK : O_BLOCK;
        g->n_a[a] = cnt;
        for (int s2 = 0; s2 < cnt; ++s2) g->slot_token[a * O_BLOCK + s2] = i * O_BLOCK + s2;
    }
    free(region_of); free(slot_of); free(nf);
    return 0;
}

static int geom_make(o_geom* g, int B, int H, int d, int F, int Hv, int Wv) {
    return geom_make_p(g, B, H, d, F, Hv, Wv, 0);
}

static void geom_free(o_geom* g) { free(g->slot_token); free(g->n_a); }

/* Packed-slot -> token table for a shape with P prefix tokens; returns the
   number of blocks (video, then prefix), or -1. */
int oracle_slot_tokens_p(int F, int Hv, int Wv, int P, int* slot_token, int* n_a) {
    o_geom g;
    if (geom_make_p(&g, 1, 1, 64, F, Hv, Wv, P)) return -1;
    memcpy(slot_token, g.slot_token, sizeof(int) * g.Npad);
    memcpy(n_a, g.n_a, sizeof(int) * g.R);
    int R = g.R;
    geom_free(&g);
    return R;
}

/* Packed-slot -> token table for a shape; returns R, or -1. */
int oracle_slot_tokens(int F, int Hv, int Wv, int* slot_token, int* n_a) {
    o_geom g;
    if (geom_make(&g, 1, 1, 64, F, Hv, Wv)) return -1;
    memcpy(slot_token, g.slot_token, sizeof(int) * g.Npad);
    memcpy(n_a, g.n_a, sizeof(int) * g.R);
    int R = g.R;
    geom_free(&g);
    return R;
}

static inline double bf16_to_double(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* Gather the 64 x d tile of block a of head (b,h) in slot order; padding rows
   are zero. x is [B,H,N,d] bf16 bits, contiguous. */
/* bf16 of a double, round to nearest even (8 significant bits, the
   exponent range of float32 with its subnormals).  Used for the weights of
   the 16-bit path, whose values are at most 1. */
double oracle_bf16_round(double x) {
    if (x == 0.0 || !isfinite(x)) return x;
    int e;
    frexp(fabs(x), &e); /* |x| in [2^(e-1), 2^e) */
    int ex = e - 1;
    if (ex < -126) ex = -126; /* subnormal spacing 2^-133 */
    double q = ldexp(1.0, ex - 7); /* spacing of the bf16 values near |x| */
    return nearbyint(x / q) * q;   /* x / q is exact; nearbyint rounds half to even */
}

static void gather_tile(const o_geom* g, const uint16_t* x, int bh, int a, double* tile) {
    int d = g->d;
    const uint16_t* base = x + (size_t)bh * g->N * d;
    for (int j = 0; j < O_BLOCK; ++j) {
        int t = g->slot_token[a * O_BLOCK + j];
        for (int c = 0; c < d; ++c) tile[j * d + c] = (t < 0) ? 0.0 : bf16_to_double(base[(size_t)t * d + c]);
    }
}

/* ------------------------------------------------------------------------ */
/* 5. Operand quantization (App. C.1 formats; scale placement is a reading).  */
/* FP8: one fp32 scale per 64-token tile, s = amax/448, codes                */
/*      e4m3(x * (448/amax)).                                                */
/* NVFP4 (two-level): tile scale g = amax/2688 (2688 = 448*6); per group of  */
/*      16 consecutive elements sf = ue4m3(amax16 * (448/amax)); codes       */
/*      e2m1(x * (1/(sf*g))).  Dequantized value = code * sf * g.            */
/* A tile whose amax is 0 gets scale 0 and all-zero codes; a group whose sf  */
/* rounds to 0 gets zero codes.  All scalar ops are fp32 round-to-nearest.   */
/* ------------------------------------------------------------------------ */
static float tile_amax(const double* tile, int count) {
    double m = 0.0;
    for (int i = 0; i < count; ++i) m = fmax(m, fabs(tile[i]));
    return (float)m; /* a bf16 value, exact in fp32 */
}

static void quant_fp8(const double* vals, int count, float amax, uint8_t* codes, float* scale) {
    if (amax == 0.0f) {
        *scale = 0.0f;
        memset(codes, 0, count);
        return;
    }
    *scale = amax / 448.0f;
    float inv = 448.0f / amax;
    for (int i = 0; i < count; ++i) codes[i] = oracle_e4m3_encode((float)vals[i] * inv);
}

/* Quantize one group of 16 values with tile amax; writes 16 e2m1 codes and
   its ue4m3 scale code. */
static void quant_fp4_group(const float* v16, float amax, float g, uint8_t* codes16, uint8_t* sf_code) {
    float t = 448.0f / amax;
    float a16 = 0.0f;
    for (int i = 0; i < 16; ++i) a16 = fmaxf(a16, fabsf(v16[i]));
    uint8_t sf = oracle_e4m3_encode(a16 * t);
    *sf_code = sf;
    if (sf == 0) {
        memset(codes16, 0, 16);
        return;
    }
    float sfg = (float)oracle_e4m3_decode(sf) * g;
    float r = 1.0f / sfg;
    for (int i = 0; i < 16; ++i) codes16[i] = oracle_e2m1_encode(v16[i] * r);
}

/* Outputs of the preparation step, logical layouts (row-major):
 *   desc     f64 [4][B][H][R][d]     Qbar, Qmax, Kbar, Kmax
 *   q8,k8    u8  [B][H][R][64][d]    e4m3 codes
 *   v8t      u8  [B][H][R][d][64]    e4m3 codes of V^T
 *   s8       f32 [3][B][H][R]        FP8 tile scales of Q, K, V
 *   q4,k4    u8  [B][H][R][64][d]    e2m1 codes, one per byte (unpacked)
 *   v4t      u8  [B][H][R][d][64]    e2m1 codes of V^T, one per byte
 *   sfq,sfk  u8  [B][H][R][64][d/16] ue4m3 group scales (groups along d)
 *   sfv      u8  [B][H][R][d][4]     ue4m3 group scales of V^T (groups along tokens)
 *   g4       f32 [3][B][H][R]        NVFP4 tile scales of Q, K, V
 *   vmax     f32 [2][B][H]           max_kb s8_V[kb], max_kb g4_V[kb]
 */
/* With P prefix tokens every block (video, then prefix) is prepared; the V
   maxima (the units of the 8-bit and 4-bit phases, which only video pairs
   use) are taken over the video blocks. */
int oracle_prepare_p(int B, int H, int d, int F, int Hv, int Wv, int P, const uint16_t* q, const uint16_t* k,
                     const uint16_t* v, double* desc, uint8_t* q8, uint8_t* k8, uint8_t* v8t, float* s8,
                     uint8_t* q4, uint8_t* k4, uint8_t* v4t, uint8_t* sfq, uint8_t* sfk, uint8_t* sfv,
                     float* g4, float* vmax) {
    o_geom g;
    if (d % 16 || geom_make_p(&g, B, H, d, F, Hv, Wv, P)) return -1;
    int R = g.R, BH = B * H;
    size_t tile = (size_t)O_BLOCK * d;
#pragma omp parallel for schedule(dynamic)
    for (int bh = 0; bh < BH; ++bh) {
        double* t = (double*)malloc(sizeof(double) * tile);
        double* tt = (double*)malloc(sizeof(double) * tile);
        float* f16 = (float*)malloc(sizeof(float) * 16);
        float vm8 = 0.0f, vm4 = 0.0f;
        for (int a = 0; a < R; ++a) {
            size_t ba = (size_t)bh * R + a;
            int na = g.n_a[a];
            for (int which = 0; which < 3; ++which) {
                const uint16_t* src = which == 0 ? q : (which == 1 ? k : v);
                gather_tile(&g, src, bh, a, t);
                /* Eq. 2: mean and channel max over the n_a valid slots. */
                if (which < 2) {
                    double* avg = desc + ((size_t)(2 * which) * BH * R + ba) * d;
                    double* mx = desc + ((size_t)(2 * which + 1) * BH * R + ba) * d;
                    for (int c = 0; c < d; ++c) {
                        double s = 0.0, m = t[c];
                        for (int j = 0; j < na; ++j) {
                            s += t[j * d + c];
                            m = fmax(m, t[j * d + c]);
                        }
                        avg[c] = s / (double)na;
                        mx[c] = m;
                    }
                }
                float amax = tile_amax(t, (int)tile);
                float gt = amax / 2688.0f;
                g4[(size_t)which * BH * R + ba] = gt;
                if (which < 2) {
                    uint8_t* c8 = (which == 0 ? q8 : k8) + ba * tile;
                    quant_fp8(t, (int)tile, amax, c8, &s8[(size_t)which * BH * R + ba]);
                    uint8_t* c4 = (which == 0 ? q4 : k4) + ba * tile;
                    uint8_t* sf = (which == 0 ? sfq : sfk) + ba * (tile / 16);
                    for (int j = 0; j < O_BLOCK; ++j)
                        for (int gi = 0; gi < d / 16; ++gi) {
                            if (amax == 0.0f) {
                                memset(c4 + j * d + gi * 16, 0, 16);
                                sf[j * (d / 16) + gi] = 0;
                                continue;
                            }
                            for (int i = 0; i < 16; ++i) f16[i] = (float)t[j * d + gi * 16 + i];
                            quant_fp4_group(f16, amax, gt, c4 + j * d + gi * 16, sf + j * (d / 16) + gi);
                        }
                } else {
                    /* Value path: transpose the tile to [d][64] (Sec. 3.3). */
                    for (int j = 0; j < O_BLOCK; ++j)
                        for (int c = 0; c < d; ++c) tt[c * O_BLOCK + j] = t[j * d + c];
                    quant_fp8(tt, (int)tile, amax, v8t + ba * tile, &s8[(size_t)2 * BH * R + ba]);
                    uint8_t* c4 = v4t + ba * tile;
                    uint8_t* sf = sfv + ba * (size_t)d * 4;
                    for (int c = 0; c < d; ++c)
                        for (int gi = 0; gi < 4; ++gi) {
                            if (amax == 0.0f) {
                                memset(c4 + c * O_BLOCK + gi * 16, 0, 16);
                                sf[c * 4 + gi] = 0;
                                continue;
                            }
                            for (int i = 0; i < 16; ++i) f16[i] = (float)tt[c * O_BLOCK + gi * 16 + i];
                            quant_fp4_group(f16, amax, gt, c4 + c * O_BLOCK + gi * 16, sf + c * 4 + gi);
                        }
                    if (a < g.Rv) {
                        vm8 = fmaxf(vm8, s8[(size_t)2 * BH * R + ba]);
                        vm4 = fmaxf(vm4, gt);
                    }
                }
            }
        }
        vmax[bh] = vm8;
        vmax[BH + bh] = vm4;
        free(t); free(tt); free(f16);
    }
    geom_free(&g);
    return 0;
}

int oracle_prepare(int B, int H, int d, int F, int Hv, int Wv, const uint16_t* q, const uint16_t* k,
                   const uint16_t* v, double* desc, uint8_t* q8, uint8_t* k8, uint8_t* v8t, float* s8,
                   uint8_t* q4, uint8_t* k4, uint8_t* v4t, uint8_t* sfq, uint8_t* sfk, uint8_t* sfv,
                   float* g4, float* vmax) {
    return oracle_prepare_p(B, H, d, F, Hv, Wv, 0, q, k, v, desc, q8, k8, v8t, s8, q4, k4, v4t, sfq, sfk, sfv, g4,
                            vmax);
}

/* ------------------------------------------------------------------------ */
/* 5b. INT8 operands of the paper's 8-bit QK^T (App. C.1: its 8-bit path   */
/* multiplies Q and K in INT8 and keeps P V in FP8; the scale placement is  */
/* a reading, as for FP8): per 64-token tile                                */
/* s = amax/127 (fp32 divide), code = clamp(RNE(x * (127/amax)), -127, 127) */
/* with the product rounded in fp32; dequantized value = code * s; a zero   */
/* tile has s = 0 and all-zero codes.                                        */
/*   q8i,k8i s8 [B][H][R][64][d]; si8 f32 [2][B][H][R] (Q, K)                */
/* ------------------------------------------------------------------------ */
int8_t oracle_int8_encode(float x) {
    float r = nearbyintf(x); /* round half to even */
    if (r > 127.0f) r = 127.0f;
    if (r < -127.0f) r = -127.0f;
    return (int8_t)r;
}

int oracle_prepare_int8_p(int B, int H, int d, int F, int Hv, int Wv, int P, const uint16_t* q, const uint16_t* k,
                          int8_t* q8i, int8_t* k8i, float* si8) {
    o_geom g;
    if (d % 16 || geom_make_p(&g, B, H, d, F, Hv, Wv, P)) return -1;
    int R = g.R, BH = B * H;
    size_t tile = (size_t)O_BLOCK * d;
#pragma omp parallel for schedule(dynamic)
    for (int bh = 0; bh < BH; ++bh) {
        double* t = (double*)malloc(sizeof(double) * tile);
        for (int a = 0; a < R; ++a) {
            size_t ba = (size_t)bh * R + a;
            for (int which = 0; which < 2; ++which) {
                gather_tile(&g, which == 0 ? q : k, bh, a, t);
                float amax = tile_amax(t, (int)tile);
                int8_t* c = (which == 0 ? q8i : k8i) + ba * tile;
                float* sc = si8 + (size_t)which * BH * R + ba;
                if (amax == 0.0f) {
                    *sc = 0.0f;
                    memset(c, 0, tile);
                    continue;
                }
                *sc = amax / 127.0f;
                float inv = 127.0f / amax;
                for (size_t i = 0; i < tile; ++i) c[i] = oracle_int8_encode((float)t[i] * inv);
            }
        }
        free(t);
    }
    geom_free(&g);
    return 0;
}

int oracle_prepare_int8(int B, int H, int d, int F, int Hv, int Wv, const uint16_t* q, const uint16_t* k,
                        int8_t* q8i, int8_t* k8i, float* si8) {
    return oracle_prepare_int8_p(B, H, d, F, Hv, Wv, 0, q, k, q8i, k8i, si8);
}

/* ------------------------------------------------------------------------ */
/* 3. Draft map (Eq. 3; App. C.1: both branches normalize over key regions). */
/* logit = (sum_c q_c k_c, as an fma chain in ascending c from 0) * (1/sqrt d);*/
/* row softmax with m = row max, e_b = o_exp(l_b - m), Z = sum_b e_b in       */
/* ascending b, S_b = e_b / Z; A = fma(lambda, S^max, (1-lambda) * S^avg).    */
/* desc as produced by oracle_prepare; A is f64 [B][H][R][R].               */
/* ------------------------------------------------------------------------ */
static void softmax_row(const double* qd, const double* kd, int R, int d, double rd, double* S) {
    double m = -INFINITY;
    for (int b = 0; b < R; ++b) {
        double acc = 0.0;
        for (int c = 0; c < d; ++c) acc = fma(qd[c], kd[(size_t)b * d + c], acc);
        S[b] = acc * rd;
        m = fmax(m, S[b]);
    }
    double Z = 0.0;
    for (int b = 0; b < R; ++b) {
        S[b] = oracle_exp(S[b] - m);
        Z += S[b];
    }
    for (int b = 0; b < R; ++b) S[b] = S[b] / Z;
}

int oracle_draft(int BH, int R, int d, const double* desc, double lambda, double* A) {
    double rd = 1.0 / sqrt((double)d);
    double oml = 1.0 - lambda;
#pragma omp parallel for schedule(dynamic)
    for (int bh = 0; bh < BH; ++bh) {
        double* Sa = (double*)malloc(sizeof(double) * R);
        double* Sm = (double*)malloc(sizeof(double) * R);
        const double* qa = desc + (size_t)(0 * BH + bh) * R * d;
        const double* qm = desc + (size_t)(1 * BH + bh) * R * d;
        const double* ka = desc + (size_t)(2 * BH + bh) * R * d;
        const double* km = desc + (size_t)(3 * BH + bh) * R * d;
        for (int a = 0; a < R; ++a) {
            softmax_row(qa + (size_t)a * d, ka, R, d, rd, Sa);
            softmax_row(qm + (size_t)a * d, km, R, d, rd, Sm);
            double* row = A + ((size_t)bh * R + a) * R;
            for (int b = 0; b < R; ++b) row[b] = fma(lambda, Sm[b], oml * Sa[b]);
        }
        free(Sa); free(Sm);
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* 4. Ranking, quotas and assignment (Sec. 3.1; App. C.1).                   */
/* All R^2 pairs of a head are sorted by A descending, ties to the smaller   */
/* pair index a*R+b.  Quotas from basis points: T8 = floor(R^2 bp8/10^4),    */
/* Tkeep = floor(R^2 (bp8+bp4)/10^4).  rank < T8 -> 8, rank < Tkeep -> 4,    */
/* else skip (0).  Per query row a the list holds its 8-bit key blocks in    */
/* ascending order, then its 4-bit key blocks in ascending order.            */
/* prec u8 [BH][R][R]; cnt i32 [2][BH][R] (8-bit, 4-bit); kidx u16 [BH][R][R].*/
/* ------------------------------------------------------------------------ */
typedef struct { double a; int idx; } o_pair;

static int pair_cmp(const void* x, const void* y) {
    const o_pair* p = (const o_pair*)x;
    const o_pair* q = (const o_pair*)y;
    if (p->a > q->a) return -1;
    if (p->a < q->a) return 1;
    return (p->idx < q->idx) ? -1 : (p->idx > q->idx);
}

int oracle_assign(int BH, int R, const double* A, int bp8, int bp4, uint8_t* prec, int* cnt, uint16_t* kidx) {
    if (bp8 < 0 || bp4 < 0 || bp8 + bp4 > 10000) return -1;
    long long RR = (long long)R * R;
    long long T8 = RR * bp8 / 10000, Tk = RR * (bp8 + bp4) / 10000;
#pragma omp parallel for schedule(dynamic)
    for (int bh = 0; bh < BH; ++bh) {
        o_pair* pr = (o_pair*)malloc(sizeof(o_pair) * RR);
        const double* Ah = A + (size_t)bh * RR;
        for (long long i = 0; i < RR; ++i) { pr[i].a = Ah[i]; pr[i].idx = (int)i; }
        qsort(pr, (size_t)RR, sizeof(o_pair), pair_cmp);
        uint8_t* P = prec + (size_t)bh * RR;
        for (long long r = 0; r < RR; ++r) P[pr[r].idx] = (r < T8) ? 8 : (r < Tk ? 4 : 0);
        for (int a = 0; a < R; ++a) {
            int n8 = 0, n4 = 0;
            uint16_t* L = kidx + ((size_t)bh * R + a) * R;
            for (int b = 0; b < R; ++b) if (P[(size_t)a * R + b] == 8) L[n8++] = (uint16_t)b;
            for (int b = 0; b < R; ++b) if (P[(size_t)a * R + b] == 4) L[n8 + n4++] = (uint16_t)b;
            cnt[(size_t)bh * R + a] = n8;
            cnt[(size_t)BH * R + (size_t)bh * R + a] = n4;
        }
        free(pr);
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* 4b. Per-query-row ranking option (a reading of "ranks blocks per query    */
/* row"; the pages rank all R^2 pairs of a head, item 4): the R key blocks  */
/* of each query block a are sorted by A descending, ties to the smaller     */
/* key block b.  Quotas per row: T8 = floor(R bp8/10^4), Tkeep =             */
/* floor(R (bp8+bp4)/10^4); rank < T8 -> 8, rank < Tkeep -> 4, else skip.    */
/* Outputs as oracle_assign.                                                 */
/* ------------------------------------------------------------------------ */
int oracle_assign_rows(int BH, int R, const double* A, int bp8, int bp4, uint8_t* prec, int* cnt,
                       uint16_t* kidx) {
    if (bp8 < 0 || bp4 < 0 || bp8 + bp4 > 10000) return -1;
    long long T8 = (long long)R * bp8 / 10000, Tk = (long long)R * (bp8 + bp4) / 10000;
#pragma omp parallel for schedule(dynamic)
    for (int bh = 0; bh < BH; ++bh) {
        o_pair* pr = (o_pair*)malloc(sizeof(o_pair) * R);
        for (int a = 0; a < R; ++a) {
            size_t row = (size_t)bh * R + a;
            const double* Ar = A + row * R;
            for (int b = 0; b < R; ++b) { pr[b].a = Ar[b]; pr[b].idx = b; }
            qsort(pr, (size_t)R, sizeof(o_pair), pair_cmp);
            uint8_t* P = prec + row * R;
            for (int r = 0; r < R; ++r) P[pr[r].idx] = (r < T8) ? 8 : (r < Tk ? 4 : 0);
            int n8 = 0, n4 = 0;
            uint16_t* L = kidx + row * R;
            for (int b = 0; b < R; ++b) if (P[b] == 8) L[n8++] = (uint16_t)b;
            for (int b = 0; b < R; ++b) if (P[b] == 4) L[n8 + n4++] = (uint16_t)b;
            cnt[row] = n8;
            cnt[(size_t)BH * R + row] = n4;
        }
        free(pr);
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* 4c. Three tiers (Table 1's 16-bit share; App. B.6: the 16-bit path takes */
/* the largest masses, INT8/FP8 the next, NVFP4 the rest).  Cumulative       */
/* quotas over the ranking of item 4 (per head) or 4b (per row, n = R):      */
/* C16 = floor(n bp16/10^4), C8 = floor(n (bp16+bp8)/10^4),                  */
/* Ck = floor(n (bp16+bp8+bp4)/10^4), n = R^2 per head; rank < C16 -> 16,    */
/* < C8 -> 8, < Ck -> 4, else 0.  With bp16 = 0 this is items 4 / 4b.        */
/* Lists: 16-bit key blocks ascending, then 8-bit, then 4-bit (the phase     */
/* order).  cnt i32 [3][BH][R] holds the 8-bit, 4-bit and 16-bit counts.     */
/* ------------------------------------------------------------------------ */
int oracle_assign_tiers(int BH, int R, const double* A, int bp16, int bp8, int bp4, int per_row, uint8_t* prec,
                        int* cnt, uint16_t* kidx) {
    if (bp16 < 0 || bp8 < 0 || bp4 < 0 || bp16 + bp8 + bp4 > 10000) return -1;
    long long n = per_row ? (long long)R : (long long)R * R;
    long long C16 = n * bp16 / 10000, C8 = n * (bp16 + bp8) / 10000, Ck = n * (bp16 + bp8 + bp4) / 10000;
    size_t BHR = (size_t)BH * R;
#pragma omp parallel for schedule(dynamic)
    for (int bh = 0; bh < BH; ++bh) {
        o_pair* pr = (o_pair*)malloc(sizeof(o_pair) * (size_t)n);
        uint8_t* P = prec + (size_t)bh * R * R;
        const double* Ah = A + (size_t)bh * R * R;
        for (int a0 = 0; a0 < (per_row ? R : 1); ++a0) {
            /* the ranked set: row a0 (per row) or all pairs of the head */
            size_t base = per_row ? (size_t)a0 * R : 0;
            for (long long i = 0; i < n; ++i) {
                pr[i].a = Ah[base + i];
                pr[i].idx = (int)i;
            }
            qsort(pr, (size_t)n, sizeof(o_pair), pair_cmp);
            for (long long r = 0; r < n; ++r)
                P[base + pr[r].idx] = (r < C16) ? 16 : (r < C8) ? 8 : (r < Ck) ? 4 : 0;
        }
        for (int a = 0; a < R; ++a) {
            int c[3] = {0, 0, 0}, k = 0;
            uint16_t* L = kidx + ((size_t)bh * R + a) * R;
            const uint8_t* Pa = P + (size_t)a * R;
            for (int b = 0; b < R; ++b) if (Pa[b] == 16) { L[k++] = (uint16_t)b; ++c[2]; }
            for (int b = 0; b < R; ++b) if (Pa[b] == 8) { L[k++] = (uint16_t)b; ++c[0]; }
            for (int b = 0; b < R; ++b) if (Pa[b] == 4) { L[k++] = (uint16_t)b; ++c[1]; }
            for (int t = 0; t < 3; ++t) cnt[t * BHR + (size_t)bh * R + a] = c[t];
        }
        free(pr);
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* 4d. Prefix keys and queries (App. C.1: a video query keeps every valid  */
/* prefix key, a prefix query attends to every key, and neither kind of     */
/* pair counts against the video-region budget).  Reading of the            */
/* unstated precision: both run on the 16-bit path, the reference precision */
/* (the budget that assigns the lower precisions covers only video-region   */
/* pairs).  From a video plan (cnt [3][BH][Rv], lists [BH][Rv][Rv] of item  */
/* 4c, 16-bit blocks first) build the plan over all Rt = Rv + Rp blocks: a  */
/* video row gets the prefix blocks Rv..Rt-1 after its 16-bit video blocks  */
/* (ascending block order within the phase); a prefix row gets every block  */
/* 0..Rt-1 at 16 bits.  cnt_t [3][BH][Rt], kidx_t [BH][Rt][Rt].              */
/* ------------------------------------------------------------------------ */
int oracle_prefix_plan(int BH, int Rv, int Rp, const int* cnt_v, const uint16_t* kidx_v, int* cnt_t,
                       uint16_t* kidx_t) {
    if (BH <= 0 || Rv <= 0 || Rp < 0) return -1;
    int Rt = Rv + Rp;
    size_t BHRv = (size_t)BH * Rv, BHRt = (size_t)BH * Rt;
    for (int bh = 0; bh < BH; ++bh) {
        for (int a = 0; a < Rt; ++a) {
            size_t rt = (size_t)bh * Rt + a;
            uint16_t* L = kidx_t + rt * Rt;
            if (a < Rv) {
                size_t rv = (size_t)bh * Rv + a;
                int n8 = cnt_v[rv], n4 = cnt_v[BHRv + rv], n16 = cnt_v[2 * BHRv + rv];
                const uint16_t* Lv = kidx_v + rv * Rv;
                int k = 0;
                for (int i = 0; i < n16; ++i) L[k++] = Lv[i];
                for (int i = 0; i < Rp; ++i) L[k++] = (uint16_t)(Rv + i);
                for (int i = n16; i < n16 + n8 + n4; ++i) L[k++] = Lv[i];
                cnt_t[rt] = n8;
                cnt_t[BHRt + rt] = n4;
                cnt_t[2 * BHRt + rt] = n16 + Rp;
            } else {
                for (int b = 0; b < Rt; ++b) L[b] = (uint16_t)b;
                cnt_t[rt] = 0;
                cnt_t[BHRt + rt] = 0;
                cnt_t[2 * BHRt + rt] = Rt;
            }
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* 6. Block-sparse attention with shared normalization (App. B.3, C.1;       */
/*    Sec. 3.3 phased execution and cross-precision accumulation).           */
/* For each valid query u of block a, in fp64:                               */
/*   phases: the 16-bit key blocks of row a (ascending; only with the tiers  */
/*   of item 4c), then the 8-bit ones, then the 4-bit ones;                  */
/*   per key block kb: s_v = (q_u . k_v)/sqrt d with the operands of the     */
/*   pair's precision, padded keys excluded; m' = max(m, max_v s_v); the     */
/*   numerator and l are rescaled by e^(m-m'); p_v = e^(s_v - m');           */
/*   l += sum_v p_v (the unquantized denominator Z^q of App. B.3); the       */
/*   numerator adds weight_v * valuecode_v.                                  */
/* 16-bit phase (unit 1): Q, K, V are the bf16 inputs and the weight is      */
/*   bf16(p_v); entering the 8-bit phase from it the numerator is divided by */
/*   sigma8 (and by sigma4 when it goes straight to the 4-bit phase).        */
/* Value codes: 8-bit: e4m3 code of V^T; 4-bit: e2m1 code * ue4m3 group      */
/*   scale; the tile scale sv[kb] (s8 or g4 of the V tile) is moved into the */
/*   weight.  Weights and units (reading of the garbled Eq. 8, "entry and    */
/*   exit scalings are inverse changes of numerical units", App. B.3):       */
/*   8-bit phase, unit sigma8 = vmax8/448:                                   */
/*     weight = e4m3(float(p_v) * float(sv[kb]/sigma8));                     */
/*   4-bit phase, unit sigma4 = vmax4/2688: y_v = float(p_v) *               */
/*     float(sv[kb]/sigma4); per 16 consecutive key slots sf = ue4m3(max y/6)*/
/*     and weight = e2m1(y_v * (1/sf)) * sf;                                 */
/*   entering the 4-bit phase the numerator is multiplied by unit/sigma4;    */
/*   at the end O = numerator * unit / l, or 0 when no valid key was kept.   */
/* flags: bit0 quantize Q/K/V; bit1 quantize the weights (needs bit2);       */
/* bit3 (with the operands of item 5b) the 8-bit phase's QK^T in INT8;       */
/* bit2 carry the numerator in phase units (production = 7).  Without bit0  */
/* the value "codes" are the exact values divided by sv[kb]; without bit1    */
/* the weights are the exact p_v * sv[kb] / unit.                            */
/* out is f64 [B][H][N][d] in original token order.                          */
/* ------------------------------------------------------------------------ */
static int attention_impl(int B, int H, int d, int F, int Hv, int Wv, int P, const uint16_t* q, const uint16_t* k,
                          const uint16_t* v, const uint8_t* q8, const uint8_t* k8, const uint8_t* v8t,
                          const float* s8, const uint8_t* q4, const uint8_t* k4, const uint8_t* v4t,
                          const uint8_t* sfq, const uint8_t* sfk, const uint8_t* sfv, const float* g4,
                          const float* vmax, const int* cnt, int tiers, const uint16_t* kidx, int flags,
                          const uint8_t* sel, const int8_t* q8i, const int8_t* k8i, const float* si8,
                          double* out) {
    /* sel: NULL, or one byte per (b,h,block); blocks with sel == 0 are not computed. */
    o_geom g;
    int qops = flags & 1, qw = flags & 2, units = flags & 4;
    int i8 = (flags & 8) && q8i && k8i && si8; /* the 8-bit phase's QK^T in INT8 */
    if (qw && !units) return -2;
    if (geom_make_p(&g, B, H, d, F, Hv, Wv, P)) return -1;
    int R = g.R, BH = B * H, N = g.N, G = d / 16;
    size_t tile = (size_t)O_BLOCK * d, BHR = (size_t)BH * R;
    double rd = 1.0 / sqrt((double)d);
    double e4[256], e2[16];
    for (int c = 0; c < 256; ++c) e4[c] = oracle_e4m3_decode((uint8_t)c);
    for (int c = 0; c < 16; ++c) e2[c] = oracle_e2m1_decode((uint8_t)c);
#pragma omp parallel for schedule(dynamic)
    for (int bh = 0; bh < BH; ++bh) {
        double* Qt = (double*)malloc(sizeof(double) * tile);
        double* Qd = (double*)malloc(sizeof(double) * 3 * tile); /* Q per phase (8, 4, 16-bit), [slot][c] */
        double* Kd = (double*)malloc(sizeof(double) * tile);     /* [slot][c] */
        double* Vc = (double*)malloc(sizeof(double) * tile);     /* value codes [slot][c] */
        double* O = (double*)malloc(sizeof(double) * tile);      /* numerators [query slot][c] */
        double m[O_BLOCK], l[O_BLOCK], s[O_BLOCK], p[O_BLOCK], w[O_BLOCK];
        float sig8 = vmax[bh] / 448.0f, sig4 = vmax[BH + bh] / 2688.0f;
        for (int a = 0; a < R; ++a) {
            size_t ba = (size_t)bh * R + a;
            if (sel && !sel[ba]) continue;
            int n16 = tiers == 3 ? cnt[2 * BHR + ba] : 0, n8 = cnt[ba], n4 = cnt[BHR + ba], nq = g.n_a[a];
            const uint16_t* L = kidx + ba * R;
            gather_tile(&g, q, bh, a, Qt);
            for (int j = 0; j < O_BLOCK; ++j)
                for (int c = 0; c < d; ++c) {
                    size_t e = ba * tile + (size_t)j * d + c;
                    double x = Qt[j * d + c];
                    Qd[j * d + c] = qops ? (i8 ? (double)q8i[e] * (double)si8[ba] : e4[q8[e]] * (double)s8[ba]) : x;
                    Qd[tile + j * d + c] =
                        qops ? e2[q4[e]] * e4[sfq[ba * tile / 16 + (size_t)j * G + c / 16]] * (double)g4[ba] : x;
                    Qd[2 * tile + j * d + c] = x; /* the 16-bit path uses the bf16 operands as they are */
                }
            /* one softmax state and one numerator per query, shared by both phases */
            for (int u = 0; u < O_BLOCK; ++u) {
                m[u] = -INFINITY;
                l[u] = 0.0;
            }
            for (size_t i = 0; i < tile; ++i) O[i] = 0.0;
            /* phases in order: 16-bit (unit 1), 8-bit (unit sigma8), 4-bit (unit sigma4) */
            double unit = units ? (n16 > 0 ? 1.0 : (double)sig8) : 1.0;
            for (int it = 0; it < n16 + n8 + n4; ++it) {
                int ph = it < n16 ? 2 : (it < n16 + n8 ? 0 : 1); /* 0: 8-bit, 1: 4-bit, 2: 16-bit phase */
                int kb = L[it], nk = g.n_a[kb];
                size_t bk = (size_t)bh * R + kb;
                double sv = ph == 2 ? 1.0 : (ph == 0 ? (double)s8[2 * BHR + bk] : (double)g4[2 * BHR + bk]);
                if (units && n16 > 0 && n8 > 0 && it == n16) {
                    /* Eq. 8, entering the 8-bit phase from the 16-bit one. */
                    double f = (sig8 > 0.0f) ? unit / (double)sig8 : 1.0;
                    for (size_t i = 0; i < tile; ++i) O[i] *= f;
                    unit = (double)sig8;
                }
                if (it == n16 + n8 && units) {
                    /* Eq. 8, entering the 4-bit phase: change of numerical units. */
                    double f = (sig4 > 0.0f) ? unit / (double)sig4 : 1.0;
                    for (size_t i = 0; i < tile; ++i) O[i] *= f;
                    unit = (double)sig4;
                }
                /* operands of this key block at the pair's precision */
                gather_tile(&g, k, bh, kb, Kd);
                gather_tile(&g, v, bh, kb, Vc);
                for (int j = 0; j < O_BLOCK; ++j)
                    for (int c = 0; c < d; ++c) {
                        size_t ek = bk * tile + (size_t)j * d + c;
                        size_t ev = bk * tile + (size_t)c * O_BLOCK + j;
                        if (qops && ph == 2) {
                            /* 16-bit: the gathered bf16 values of K and V */
                        } else if (qops) {
                            Kd[j * d + c] = ph == 0 ? (i8 ? (double)k8i[ek] * (double)si8[BHR + bk]
                                                          : e4[k8[ek]] * (double)s8[BHR + bk])
                                                    : e2[k4[ek]] * e4[sfk[bk * tile / 16 + (size_t)j * G + c / 16]] *
                                                          (double)g4[BHR + bk];
                            Vc[j * d + c] = ph == 0 ? e4[v8t[ev]]
                                                    : e2[v4t[ev]] * e4[sfv[bk * (size_t)d * 4 + (size_t)c * 4 + j / 16]];
                        } else {
                            Vc[j * d + c] = (sv > 0.0) ? Vc[j * d + c] / sv : 0.0;
                        }
                    }
                for (int u = 0; u < nq; ++u) {
                    const double* qu = Qd + (size_t)ph * tile + (size_t)u * d;
                    for (int j = 0; j < nk; ++j) {
                        double acc = 0.0;
                        for (int c = 0; c < d; ++c) acc += qu[c] * Kd[j * d + c];
                        s[j] = acc * rd;
                    }
                    double mb = -INFINITY;
                    for (int j = 0; j < nk; ++j) mb = fmax(mb, s[j]);
                    double mn = fmax(m[u], mb);
                    double corr = (m[u] == -INFINITY) ? 0.0 : exp(m[u] - mn);
                    l[u] *= corr;
                    double* Ou = O + (size_t)u * d;
                    for (int c = 0; c < d; ++c) Ou[c] *= corr;
                    m[u] = mn;
                    for (int j = 0; j < O_BLOCK; ++j) p[j] = (j < nk) ? exp(s[j] - mn) : 0.0;
                    for (int j = 0; j < nk; ++j) l[u] += p[j];
                    if (!qw) {
                        for (int j = 0; j < O_BLOCK; ++j) w[j] = (unit > 0.0) ? p[j] * sv / unit : 0.0;
                    } else if (ph == 2) {
                        for (int j = 0; j < O_BLOCK; ++j) w[j] = oracle_bf16_round(p[j]);
                    } else if (ph == 0) {
                        float ratio = sig8 > 0.0f ? s8[2 * BHR + bk] / sig8 : 0.0f;
                        for (int j = 0; j < O_BLOCK; ++j) w[j] = e4[oracle_e4m3_encode((float)p[j] * ratio)];
                    } else {
                        float ratio = sig4 > 0.0f ? g4[2 * BHR + bk] / sig4 : 0.0f;
                        for (int gi = 0; gi < O_BLOCK / 16; ++gi) {
                            float y[16], ym = 0.0f;
                            for (int i = 0; i < 16; ++i) {
                                y[i] = (float)p[gi * 16 + i] * ratio;
                                ym = fmaxf(ym, y[i]);
                            }
                            uint8_t sf = oracle_e4m3_encode(ym / 6.0f);
                            double sfd = e4[sf];
                            float r = sf ? 1.0f / (float)sfd : 0.0f;
                            for (int i = 0; i < 16; ++i) w[gi * 16 + i] = sf ? e2[oracle_e2m1_encode(y[i] * r)] * sfd : 0.0;
                        }
                    }
                    for (int j = 0; j < nk; ++j)
                        for (int c = 0; c < d; ++c) Ou[c] += w[j] * Vc[j * d + c];
                }
            }
            for (int u = 0; u < nq; ++u) {
                int t = g.slot_token[a * O_BLOCK + u];
                double* o = out + ((size_t)bh * N + t) * d;
                for (int c = 0; c < d; ++c) o[c] = (l[u] > 0.0) ? O[(size_t)u * d + c] * unit / l[u] : 0.0;
            }
        }
        free(Qt); free(Qd); free(Kd); free(Vc); free(O);
    }
    geom_free(&g);
    return 0;
}

int oracle_attention(int B, int H, int d, int F, int Hv, int Wv, const uint16_t* q, const uint16_t* k,
                     const uint16_t* v, const uint8_t* q8, const uint8_t* k8, const uint8_t* v8t,
                     const float* s8, const uint8_t* q4, const uint8_t* k4, const uint8_t* v4t,
                     const uint8_t* sfq, const uint8_t* sfk, const uint8_t* sfv, const float* g4,
                     const float* vmax, const int* cnt, const uint16_t* kidx, int flags, const uint8_t* sel,
                     double* out) {
    return attention_impl(B, H, d, F, Hv, Wv, 0, q, k, v, q8, k8, v8t, s8, q4, k4, v4t, sfq, sfk, sfv, g4, vmax, cnt, 2,
                          kidx, flags, sel, NULL, NULL, NULL, out);
}

/* The same with the 16-bit tier: cnt i32 [3][BH][R] (8-bit, 4-bit, 16-bit
   counts) and lists holding the 16-bit key blocks first (oracle_assign_tiers). */
int oracle_attention_tiers(int B, int H, int d, int F, int Hv, int Wv, const uint16_t* q, const uint16_t* k,
                           const uint16_t* v, const uint8_t* q8, const uint8_t* k8, const uint8_t* v8t,
                           const float* s8, const uint8_t* q4, const uint8_t* k4, const uint8_t* v4t,
                           const uint8_t* sfq, const uint8_t* sfk, const uint8_t* sfv, const float* g4,
                           const float* vmax, const int* cnt, const uint16_t* kidx, int flags, const uint8_t* sel,
                           double* out) {
    return attention_impl(B, H, d, F, Hv, Wv, 0, q, k, v, q8, k8, v8t, s8, q4, k4, v4t, sfq, sfk, sfv, g4, vmax, cnt, 3,
                          kidx, flags, sel, NULL, NULL, NULL, out);
}

/* Either tier layout (tiers = 2 or 3) with the 8-bit phase's QK^T in INT8
   (flags bit 3, item 5b operands; FP8 PV as before). */
int oracle_attention_int8(int B, int H, int d, int F, int Hv, int Wv, const uint16_t* q, const uint16_t* k,
                          const uint16_t* v, const uint8_t* q8, const uint8_t* k8, const uint8_t* v8t,
                          const float* s8, const uint8_t* q4, const uint8_t* k4, const uint8_t* v4t,
                          const uint8_t* sfq, const uint8_t* sfk, const uint8_t* sfv, const float* g4,
                          const float* vmax, const int* cnt, int tiers, const uint16_t* kidx, int flags,
                          const uint8_t* sel, const int8_t* q8i, const int8_t* k8i, const float* si8, double* out) {
    if (tiers != 2 && tiers != 3) return -1;
    return attention_impl(B, H, d, F, Hv, Wv, 0, q, k, v, q8, k8, v8t, s8, q4, k4, v4t, sfq, sfk, sfv, g4, vmax, cnt,
                          tiers, kidx, flags | 8, sel, q8i, k8i, si8, out);
}

/* The attention with P prefix tokens: operands of all Rt blocks (video,
   then prefix; oracle_prepare_p), the three-tier plan over Rt blocks
   (oracle_prefix_plan) and, optionally (q8i non-null), the INT8 operands of
   the 8-bit phase's QK^T.  out f64 [B][H][P + F*Hv*Wv][d] in token order. */
int oracle_attention_p(int B, int H, int d, int F, int Hv, int Wv, int P, const uint16_t* q, const uint16_t* k,
                       const uint16_t* v, const uint8_t* q8, const uint8_t* k8, const uint8_t* v8t,
                       const float* s8, const uint8_t* q4, const uint8_t* k4, const uint8_t* v4t,
                       const uint8_t* sfq, const uint8_t* sfk, const uint8_t* sfv, const float* g4,
                       const float* vmax, const int* cnt, const uint16_t* kidx, int flags, const uint8_t* sel,
                       const int8_t* q8i, const int8_t* k8i, const float* si8, double* out) {
    return attention_impl(B, H, d, F, Hv, Wv, P, q, k, v, q8, k8, v8t, s8, q4, k4, v4t, sfq, sfk, sfv, g4, vmax, cnt,
                          3, kidx, q8i ? (flags | 8) : flags, sel, q8i, k8i, si8, out);
}

/* Dense softmax attention, for checking the oracle against brute force. */
int oracle_dense(int BH, int N, int d, const uint16_t* q, const uint16_t* k, const uint16_t* v, double* out) {
    double rd = 1.0 / sqrt((double)d);
#pragma omp parallel for schedule(dynamic)
    for (int bh = 0; bh < BH; ++bh) {
        double* s = (double*)malloc(sizeof(double) * N);
        for (int u = 0; u < N; ++u) {
            const uint16_t* qu = q + ((size_t)bh * N + u) * d;
            double m = -INFINITY, l = 0.0;
            for (int t = 0; t < N; ++t) {
                const uint16_t* kt = k + ((size_t)bh * N + t) * d;
                double acc = 0.0;
                for (int c = 0; c < d; ++c) acc += bf16_to_double(qu[c]) * bf16_to_double(kt[c]);
                s[t] = acc * rd;
                m = fmax(m, s[t]);
            }
            double* o = out + ((size_t)bh * N + u) * d;
            for (int c = 0; c < d; ++c) o[c] = 0.0;
            for (int t = 0; t < N; ++t) {
                double p = exp(s[t] - m);
                l += p;
                const uint16_t* vt = v + ((size_t)bh * N + t) * d;
                for (int c = 0; c < d; ++c) o[c] += p * bf16_to_double(vt[c]);
            }
            for (int c = 0; c < d; ++c) o[c] /= l;
        }
        free(s);
    }
    return 0;
}

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
