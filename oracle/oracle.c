/*
 * oracle.c - plain, slow, single-threaded fp64 CPU oracle of the routed-MoE layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check of the build
 * entry point and the benchmark's CPU-baseline leg may load this library.  It shares
 * no code, header or table with the CUDA library: it reads expert weights in the
 * generator's interchange form (natural code order), and it has its own reader of
 * the packed format (used only to check the packer).
 *
 * The pages (five web pages about the Xolotl engine) state the problem but no
 * formula: each token picks a few experts and only those experts' weights are read
 * and applied (ossradar.top, Xolotl README, "How it works, in one paragraph";
 * yoney.dev news item, third paragraph).  What is computed here is the plain
 * DeepSeek-style routed layer that reading implies:
 *
 *   L[t,e] = sum_h x[t,h] Wr[e,h] + b[e]            oracle_logits, oracle_select
 *   p = softmax(L[t,:]); ids = top-k of p (ties: lower id); g = p[ids] / sum p[ids]
 *   counts / offsets / perm (expert asc, token asc) / inv_perm   oracle_permute
 *   y_e(x) = Wd (silu(Wg x) * (Wu x))                oracle_expert_ffn
 *   y[t] = sum_j g[t,j] y_{ids[t,j]}(x[t]) + sum_s y_shared_s(x[t])   oracle_combine
 *
 * Weights are dequantised exactly in fp64: w = (c - o) * s with o = 1 (ternary),
 * 1.5 (2-bit), 3.5 (3-bit) and s the fp16 group scale, one per 64 weights along K.
 * Those value sets ({-1,0,1}, {-1.5,-0.5,0.5,1.5}, -3.5..3.5, times the scale) are
 * the layer's stated quantisation (ternary / 2-bit / 3-bit mix: ossradar.top README,
 * "Get a model"; shadowgraph.io README, "Get a model").
 *
 * Build: cc -O2 -std=c11 -shared -fPIC oracle.c -lm   (no fast-math, no threads).
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <string.h>

#define ORACLE_GROUP 64

/* ---- scalar decoding of the input encodings ---------------------------- */

/* IEEE binary16 bit pattern -> double (exact). */
double oracle_f16_to_f64(uint16_t h) {
    int sign = (h >> 15) & 1;
    int expo = (h >> 10) & 0x1F;
    int mant = h & 0x3FF;
    double v;
    if (expo == 0) {
        v = ldexp((double)mant, -24);                /* subnormal: mant * 2^-24 */
    } else if (expo == 31) {
        v = mant ? NAN : INFINITY;
    } else {
        v = ldexp((double)(mant | 0x400), expo - 25); /* (1024 + mant) * 2^(e-15-10) */
    }
    return sign ? -v : v;
}

/* bfloat16 bit pattern -> double (exact: the high half of a binary32). */
double oracle_bf16_to_f64(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static double code_offset(int fmt) {
    return fmt == 0 ? 1.0 : (fmt == 1 ? 1.5 : 3.5);
}

/* Code of element (n, k) of a matrix in the interchange form. */
static int nat_code(const uint8_t* codes, const uint8_t* hi, int fmt, int K, int n, int k) {
    int c = (codes[(size_t)n * (K / 4) + k / 4] >> (2 * (k % 4))) & 3;
    if (fmt == 2) c += 4 * ((hi[(size_t)n * (K / 8) + k / 8] >> (k % 8)) & 1);
    return c;
}

/* Dequantise row n of W[N][K] into w[K] (fp64, exact). Returns -1 on a bad code. */
static int dequant_row(const uint8_t* codes, const uint8_t* hi, const uint16_t* scales, int fmt,
                       int K, int n, double* w) {
    double o = code_offset(fmt);
    for (int k = 0; k < K; ++k) {
        int c = nat_code(codes, hi, fmt, K, n, k);
        if (fmt == 0 && c > 2) return -1;
        w[k] = ((double)c - o) * oracle_f16_to_f64(scales[(size_t)n * (K / ORACLE_GROUP) + k / ORACLE_GROUP]);
    }
    return 0;
}

/* ---- router logits ------------------------------------------------------- */

/* L[t][e] = sum_h x[t][h] * Wr[e][h], in fp64 (x bf16, Wr fp32, both exact in fp64). */
void oracle_logits(int T, int H, int E, const uint16_t* x, const float* Wr, double* L) {
    for (int t = 0; t < T; ++t) {
        for (int e = 0; e < E; ++e) {
            double acc = 0.0;
            for (int h = 0; h < H; ++h)
                acc += oracle_bf16_to_f64(x[(size_t)t * H + h]) * (double)Wr[(size_t)e * H + h];
            L[(size_t)t * E + e] = acc;
        }
    }
}

/* ---- softmax, top-k, renormalised gates ---------------------------------- */

/* For each token: z = L + b (b may be NULL), p = softmax(z) (max subtracted),
 * ids = k largest p in descending order (equal p: lower id first),
 * gates = p[ids] / sum p[ids].  p_out [T][E] may be NULL. */
void oracle_select(int T, int E, int k, const double* L, const float* bias, int32_t* ids,
                   double* gates, double* p_out) {
    double p[1024];
    unsigned char taken[1024];
    for (int t = 0; t < T; ++t) {
        const double* row = L + (size_t)t * E;
        double zmax = -INFINITY;
        for (int e = 0; e < E; ++e) {
            double z = row[e] + (bias ? (double)bias[e] : 0.0);
            p[e] = z;
            if (z > zmax) zmax = z;
        }
        double sum = 0.0;
        for (int e = 0; e < E; ++e) {
            p[e] = exp(p[e] - zmax);
            sum += p[e];
        }
        for (int e = 0; e < E; ++e) {
            p[e] /= sum;
            taken[e] = 0;
            if (p_out) p_out[(size_t)t * E + e] = p[e];
        }
        double psel = 0.0;
        for (int j = 0; j < k; ++j) {
            int best = -1;
            for (int e = 0; e < E; ++e) {
                if (taken[e]) continue;
                if (best < 0 || p[e] > p[best]) best = e;   /* strict '>' keeps the lower id on ties */
            }
            taken[best] = 1;
            ids[(size_t)t * k + j] = best;
            psel += p[best];
        }
        for (int j = 0; j < k; ++j) gates[(size_t)t * k + j] = p[ids[(size_t)t * k + j]] / psel;
    }
}

/* ---- histogram, exclusive scan, permutation ------------------------------- */

/* counts[e] = #{(t,j): ids[t][j] == e}; offsets = exclusive prefix sum (E+1 entries);
 * perm lists pairs t*k + j expert by expert (ascending), token ascending within an
 * expert; inv_perm is its inverse. */
void oracle_permute(int T, int E, int k, const int32_t* ids, int32_t* counts, int32_t* offsets,
                    int32_t* perm, int32_t* inv_perm) {
    for (int e = 0; e < E; ++e) counts[e] = 0;
    for (int i = 0; i < T * k; ++i) counts[ids[i]]++;
    offsets[0] = 0;
    for (int e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];
    int r = 0;
    for (int e = 0; e < E; ++e)
        for (int t = 0; t < T; ++t)
            for (int j = 0; j < k; ++j)
                if (ids[(size_t)t * k + j] == e) perm[r++] = t * k + j;
    for (int i = 0; i < T * k; ++i) inv_perm[perm[i]] = i;
}

/* ---- one expert FFN (routed or shared) on a list of tokens ----------------- */

/* y[i][:] = Wd (silu(Wg x_i) * (Wu x_i)) for n_tok tokens x_i (bf16 rows of H).
 * Gate/up are [I][H], down is [H][I], each as (codes, hi, scales) in the
 * interchange form.  scratch must hold 2*max(H, I) + I*n_tok doubles.
 * Returns 0, or -1 on a bad code. */
int oracle_expert_ffn(int H, int I, int fmt,
                      const uint8_t* g_codes, const uint8_t* g_hi, const uint16_t* g_scales,
                      const uint8_t* u_codes, const uint8_t* u_hi, const uint16_t* u_scales,
                      const uint8_t* d_codes, const uint8_t* d_hi, const uint16_t* d_scales,
                      int n_tok, const uint16_t* x, double* y, double* scratch) {
    int KW = H > I ? H : I;
    double* w = scratch;                 /* one dequantised row, up to max(H, I)   */
    double* w2 = scratch + KW;           /* second row (up)                         */
    double* hbuf = scratch + 2 * KW;     /* h[i][n] for all tokens, I per token      */
    for (int n = 0; n < I; ++n) {
        if (dequant_row(g_codes, g_hi, g_scales, fmt, H, n, w)) return -1;
        if (dequant_row(u_codes, u_hi, u_scales, fmt, H, n, w2)) return -1;
        for (int i = 0; i < n_tok; ++i) {
            const uint16_t* xi = x + (size_t)i * H;
            double a = 0.0, b = 0.0;
            for (int h = 0; h < H; ++h) {
                double xv = oracle_bf16_to_f64(xi[h]);
                a += w[h] * xv;
                b += w2[h] * xv;
            }
            hbuf[(size_t)i * I + n] = a / (1.0 + exp(-a)) * b;
        }
    }
    for (int m = 0; m < H; ++m) {
        if (dequant_row(d_codes, d_hi, d_scales, fmt, I, m, w)) return -1;
        for (int i = 0; i < n_tok; ++i) {
            double acc = 0.0;
            const double* hi_ = hbuf + (size_t)i * I;
            for (int n = 0; n < I; ++n) acc += w[n] * hi_[n];
            y[(size_t)i * H + m] = acc;
        }
    }
    return 0;
}

/* ---- gate-weighted combine -------------------------------------------------- */

/* y[h] = sum_j gates[j] * y_routed[j][h] + sum_s y_shared[s][h], slot order j = 0..k-1. */
void oracle_combine(int H, int k, int S, const double* gates, const double* y_routed,
                    const double* y_shared, double* y) {
    for (int h = 0; h < H; ++h) {
        double acc = 0.0;
        for (int j = 0; j < k; ++j) acc += gates[j] * y_routed[(size_t)j * H + h];
        for (int s = 0; s < S; ++s) acc += y_shared[(size_t)s * H + h];
        y[h] = acc;
    }
}

/* ---- reader of the packed format (checks the packer; not used by the layer) ---- */

static uint32_t rd32(const uint8_t* p) {
    return (uint32_t)p[0] | ((uint32_t)p[1] << 8) | ((uint32_t)p[2] << 16) | ((uint32_t)p[3] << 24);
}
static uint64_t rd64(const uint8_t* p) { return (uint64_t)rd32(p) | ((uint64_t)rd32(p + 4) << 32); }

/* Reads matrix `which` (0 gate [I][H], 1 up [I][H], 2 down [H][I]) of expert table
 * entry `table` from a packed buffer: codes as int8 [rows][K] (full code 0..7) and
 * scales as fp16 bits [rows][K/64].  *fmt receives the format.
 * Layout read here (packed format version 2): header of 256 bytes (magic 'MOEP',
 * version 2, H, I, E, S, group 64, interleave 8); table of 64-byte entries at 256
 * ({u32 fmt, u32 0, u64 gu_scales, gu_codes, gu_hi, dn_scales, dn_codes, dn_hi});
 * gate/up fused as GU[2I][H] with rows interleaved 8 gate / 8 up.  Each array holds
 * one block per (16-row tile j, chunk c of up to 8 groups of 64, ng groups):
 *   codes  at 4*K*j + 2048*c; word wl = 4*gl + quarter of tile row r at u32 index
 *          r*32 + (wl ^ 4*(r%8)) when ng == 8, else r*4*ng + wl; element 16w+2p+h of
 *          a code word at bits 16h+2p..+1;
 *   hi     at 128*G*j + 1024*c; word vl = 2*gl + half at r*16 + (vl ^ 2*((r%8)/2)) when
 *          ng == 8, else r*2*ng + vl; element 32v+16q+2p+h at bit 16h+8q+p;
 *   scales at 256*NC*j + 256*c; scale of group 8c+gl of row r at half r*8 + gl.
 * Format 3 (ternary, five codes per byte, a storage form): the scales as above; the
 * codes of physical row pr (the fused gate/up row order) in ceil(K/5) bytes from
 * pr*ceil(K/5), element k in byte k/5 as base-3 digit k%5 (the byte is the sum of
 * c_{5i+j} 3^j, at most 242); no third bits.
 * Returns 0 or a negative error. */
int oracle_unpack(const uint8_t* buf, size_t bytes, int table, int which, int8_t* codes,
                  uint16_t* scales, int* fmt) {
    if (bytes < 256 || rd32(buf) != 0x50454F4Du || rd32(buf + 4) != 2u) return -1;
    int H = (int)rd32(buf + 8), I = (int)rd32(buf + 12), E = (int)rd32(buf + 16);
    int S = (int)rd32(buf + 20), R = (int)rd32(buf + 28);
    if ((int)rd32(buf + 24) != ORACLE_GROUP || R != 8) return -2;
    if (table < 0 || table >= E + S) return -3;
    const uint8_t* ent = buf + 256 + (size_t)table * 64;
    int f = (int)rd32(ent);
    *fmt = f;
    int rows = which == 2 ? H : I;
    int K = which == 2 ? I : H;
    int G = K / ORACLE_GROUP;
    int NC = (G + 7) / 8;
    uint64_t off_s = rd64(ent + (which == 2 ? 32 : 8));
    uint64_t off_c = rd64(ent + (which == 2 ? 40 : 16));
    uint64_t off_h = rd64(ent + (which == 2 ? 48 : 24));
    for (int n = 0; n < rows; ++n) {
        /* physical row in the packed matrix */
        int pr = which == 2 ? n : 16 * (n / 8) + (which == 1 ? 8 : 0) + n % 8;
        int j = pr / 16, r = pr % 16;
        for (int g = 0; g < G; ++g) {
            int c = g / 8, gl = g % 8;
            const uint8_t* sp = buf + off_s + (size_t)256 * NC * j + 256 * (size_t)c + 16 * r + 2 * gl;
            scales[(size_t)n * G + g] = (uint16_t)(sp[0] | (sp[1] << 8));
        }
        for (int k = 0; k < K; ++k) {
            int g = k / 64, c = g / 8, gl = g % 8;
            int ng = G - 8 * c < 8 ? G - 8 * c : 8;
            int wl = 4 * gl + (k % 64) / 16;
            int pos = ng == 8 ? r * 32 + (wl ^ (4 * (r % 8))) : r * 4 * ng + wl;
            uint32_t word = rd32(buf + off_c + (size_t)4 * K * j + 2048 * (size_t)c + 4 * (size_t)pos);
            int i = k % 16, p = i / 2, h = i % 2;
            int code = (int)((word >> (16 * h + 2 * p)) & 3u);
            if (f == 3) {
                /* dense ternary: physical row pr holds ceil(K/5) bytes, element k in
                   byte k/5 as base-3 digit k%5 (byte = sum of c_{5i+j} 3^j) */
                size_t rb = (size_t)(K + 4) / 5;
                int v = buf[off_c + (size_t)pr * rb + (size_t)(k / 5)];
                if (v > 242) return -4;
                for (int d = 0; d < k % 5; ++d) v /= 3;
                code = v % 3;
            }
            if (f == 2) {
                int vl = 2 * gl + (k % 64) / 32;
                int hpos = ng == 8 ? r * 16 + (vl ^ (2 * ((r % 8) / 2))) : r * 2 * ng + vl;
                uint32_t hw = rd32(buf + off_h + (size_t)128 * G * j + 1024 * (size_t)c + 4 * (size_t)hpos);
                int e = k % 32, q = e / 16, p1 = (e % 16) / 2, h1 = e % 2;
                code += 4 * (int)((hw >> (16 * h1 + 8 * q + p1)) & 1u);
            }
            codes[(size_t)n * K + k] = (int8_t)code;
        }
    }
    return 0;
}
