/*
 * oracle.c -- plain, slow, fp64 CPU oracle for the quantized decode-step linear layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path (the CUDA library and its Python
 * binding) may include, link or call this file; only tests/, the smoke check and the CPU
 * baseline leg of bench.py use it.  It shares no code, header, table or helper with the CUDA
 * path: every decoder below is written out from the format definitions.
 *
 * Sources for what is computed (the pages are a set of web pages about two inference
 * engines, "imp" for the RTX 5090 and "Imparo"):
 *   - imp README, "Features" table, rows "Quantization" and "sm_120a kernels": GGUF Q8_0/Q4_0 and
 *     NVFP4 weights, NVFP4 block-scaled GEMM/GEMV, e2m1 / e4m3 decode.
 *   - Imparo README intro: Q4_0 MoE decode with CUDA expert routing (LFM2.5-8B-A1B).
 *   - imp README, "Features" table, row "Server": an ordered (deterministic) MoE reduction.
 *   - imp release notes, v0.6 "Native MXFP4 GGUF weight format": E2M1 codes with UE8M0 block
 *     scales, 4.25 bits per weight (one 8-bit scale per 32 values).
 *   - imp README, "Features" table, row "Quantization": GGUF K-quants (Q4_K_M and others) among
 *     the weight formats.
 * The pages name the formats but never print their byte layout.  The layouts used here are the
 * public conventions (GGUF block_q8_0 / block_q4_0; NVFP4 = E2M1 codes, one E4M3 scale per 16
 * values, one FP32 per-tensor scale), the plainest reading the pages support.
 *
 * All arithmetic is fp64 except where a rule fixes fp32 (the activation quantizer of the chunk
 * path, which is a rounding rule stated in fp32).  Sums are plain sequential loops.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

enum { QO_Q8_0 = 1, QO_Q4_0 = 2, QO_NVFP4 = 3, QO_MXFP4 = 4, QO_Q4_K = 5, QO_Q6_K = 6 };

/* ---------------------------------------------------------------- scalar decoders */

/* IEEE 754 binary16: 1 sign, 5 exponent (bias 15), 10 mantissa bits. */
double qo_fp16(uint16_t h) {
    int s = (h >> 15) & 1, e = (h >> 10) & 0x1f, m = h & 0x3ff;
    double v;
    if (e == 0)
        v = ldexp((double)m, -24); /* subnormal: m * 2^-14 * 2^-10 */
    else if (e == 31)
        v = m ? NAN : INFINITY;
    else
        v = ldexp(1.0 + m / 1024.0, e - 15);
    return s ? -v : v;
}

/* OCP FP8 E4M3 ("fn": no infinities): 1 sign, 4 exponent (bias 7), 3 mantissa bits.
 * Exponent 0 is subnormal (m * 2^-9); S.1111.111 is NaN; the largest finite value is 448. */
double qo_e4m3(uint8_t b) {
    int s = (b >> 7) & 1, e = (b >> 3) & 0xf, m = b & 7;
    double v;
    if (e == 15 && m == 7)
        return NAN;
    if (e == 0)
        v = ldexp((double)m, -9);
    else
        v = ldexp(1.0 + m / 8.0, e - 7);
    return s ? -v : v;
}

/* OCP FP4 E2M1: 1 sign, 2 exponent (bias 1), 1 mantissa bit; exponent 0 is subnormal (m * 0.5). */
double qo_e2m1(uint8_t c) {
    int s = (c >> 3) & 1, e = (c >> 1) & 3, m = c & 1;
    double v = (e == 0) ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
    return s ? -v : v;
}

/* OCP MX UE8M0 scale: an 8-bit biased exponent (bias 127), no sign, no mantissa; 0xFF is NaN. */
double qo_e8m0(uint8_t b) {
    if (b == 0xff) return NAN;
    return ldexp(1.0, (int)b - 127);
}

/* ---------------------------------------------------------------- block dequantization */

/* Bytes of one canonical row of K weights. */
int64_t qo_row_bytes(int fmt, int64_t K) {
    if (fmt == QO_Q8_0) return (K / 32) * 34;
    if (fmt == QO_Q4_0) return (K / 32) * 18;
    if (fmt == QO_NVFP4 || fmt == QO_MXFP4) return K / 2;
    if (fmt == QO_Q4_K) return (K / 256) * 144;
    if (fmt == QO_Q6_K) return (K / 256) * 210;
    return -1;
}

/* GGUF Q4_K super-block (256 values, 144 bytes): fp16 d, fp16 dmin, 12 bytes holding eight 6-bit
 * scales and eight 6-bit mins (one pair per 32-value sub-block), 128 bytes of 4-bit codes.
 * Sub-blocks 0..3 keep their scale and min in the low 6 bits of bytes 0..3 and 4..7; sub-blocks
 * 4..7 keep the low 4 bits of each in byte 8..11 (scale low nibble, min high nibble) and the top
 * 2 bits in the spare high bits of bytes 0..3 (scale) and 4..7 (min) of sub-block j - 4. */
void qo_q4k_scale_min(const uint8_t* sc12, int j, int* sc, int* m) {
    if (j < 4) {
        *sc = sc12[j] & 63;
        *m = sc12[j + 4] & 63;
    } else {
        *sc = (sc12[j + 4] & 0xf) | ((sc12[j - 4] >> 6) << 4);
        *m = (sc12[j + 4] >> 4) | ((sc12[j] >> 6) << 4);
    }
}

/* Dequantize row n of a canonical tensor into w[0..K) (fp64, exact real value).
 *   Q8_0 block (34 B): fp16 d, int8 q[32];          w_j = d * q_j
 *   Q4_0 block (18 B): fp16 d, uint8 qs[16];        element j (j<16) is the low nibble of qs[j],
 *                                                   element j+16 its high nibble; w = d * (nib - 8)
 *   NVFP4: codes [N][K/2], byte i = elements 2i (low nibble) and 2i+1 (high nibble);
 *          scales [N][K/16] E4M3; w = e2m1(code) * e4m3(scale of k/16) * g
 *   MXFP4: codes as NVFP4; scales [N][K/32] UE8M0; w = e2m1(code) * 2^(scale of k/32 - 127)
 *   Q4_K super-block (144 B per 256 values, see qo_q4k_scale_min): the codes of the 64 values
 *          64c .. 64c+63 are bytes 32c .. 32c+31 of the code area, values 64c + l in the low
 *          nibble of byte l, 64c + 32 + l in its high nibble; value k of sub-block j = k / 32:
 *          w = d * scale_j * code - dmin * min_j
 *   Q6_K super-block (210 B per 256 values): ql[128] (low 4 bits of the codes), qh[64] (high 2
 *          bits), int8 scales[16] (one per 16 values), fp16 d.  In half h (values 128h .. 128h+127,
 *          bytes ql[64h ..], qh[32h ..], scales[8h ..]) value 128h + 32s + l (s = 0..3, l = 0..31)
 *          takes its low 4 bits from the low nibble of ql[64h + l] (s = 0), of ql[64h + 32 + l]
 *          (s = 1), or the high nibbles of those bytes (s = 2, 3), its high 2 bits from bits
 *          2s, 2s+1 of qh[32h + l], and scale scales[8h + 2s + l / 16]:  w = d * scale * (code - 32) */
static void dequant_row(int fmt, int64_t K, const uint8_t* blocks, const uint8_t* scales, float g,
                        int64_t n, double* w) {
    if (fmt == QO_Q8_0 || fmt == QO_Q4_0) {
        int64_t bsz = fmt == QO_Q8_0 ? 34 : 18;
        const uint8_t* row = blocks + n * (K / 32) * bsz;
        for (int64_t b = 0; b < K / 32; ++b) {
            const uint8_t* blk = row + b * bsz;
            double d = qo_fp16((uint16_t)(blk[0] | (blk[1] << 8)));
            for (int j = 0; j < 32; ++j) {
                double q;
                if (fmt == QO_Q8_0)
                    q = (double)(int8_t)blk[2 + j];
                else
                    q = (double)((j < 16 ? (blk[2 + j] & 0xf) : (blk[2 + j - 16] >> 4)) - 8);
                w[b * 32 + j] = d * q;
            }
        }
    } else if (fmt == QO_NVFP4) {
        const uint8_t* row = blocks + n * (K / 2);
        const uint8_t* srow = scales + n * (K / 16);
        for (int64_t k = 0; k < K; ++k) {
            uint8_t byte = row[k / 2];
            uint8_t c = (k & 1) ? (byte >> 4) : (byte & 0xf);
            w[k] = qo_e2m1(c) * qo_e4m3(srow[k / 16]) * (double)g;
        }
    } else if (fmt == QO_Q4_K) {
        const uint8_t* row = blocks + n * (K / 256) * 144;
        for (int64_t b = 0; b < K / 256; ++b) {
            const uint8_t* blk = row + b * 144;
            double d = qo_fp16((uint16_t)(blk[0] | (blk[1] << 8)));
            double dmin = qo_fp16((uint16_t)(blk[2] | (blk[3] << 8)));
            const uint8_t* sc12 = blk + 4;
            const uint8_t* qs = blk + 16;
            for (int k = 0; k < 256; ++k) {
                int sc, m;
                qo_q4k_scale_min(sc12, k / 32, &sc, &m);
                int c = k / 64, l = k % 32;
                int code = (k % 64) < 32 ? (qs[32 * c + l] & 0xf) : (qs[32 * c + l] >> 4);
                w[b * 256 + k] = d * sc * code - dmin * m;
            }
        }
    } else if (fmt == QO_Q6_K) {
        const uint8_t* row = blocks + n * (K / 256) * 210;
        for (int64_t b = 0; b < K / 256; ++b) {
            const uint8_t* blk = row + b * 210;
            const uint8_t* ql = blk;
            const uint8_t* qh = blk + 128;
            const int8_t* sc = (const int8_t*)(blk + 192);
            double d = qo_fp16((uint16_t)(blk[208] | (blk[209] << 8)));
            for (int v = 0; v < 256; ++v) {
                int h = v / 128, s = (v % 128) / 32, l = v % 32;
                uint8_t lb = ql[64 * h + 32 * (s & 1) + l];
                int lo = (s < 2) ? (lb & 0xf) : (lb >> 4);
                int hi = (qh[32 * h + l] >> (2 * s)) & 3;
                int code = lo | (hi << 4);
                w[b * 256 + v] = d * sc[8 * h + 2 * s + l / 16] * (code - 32);
            }
        }
    } else {
        const uint8_t* row = blocks + n * (K / 2);
        const uint8_t* srow = scales + n * (K / 32);
        for (int64_t k = 0; k < K; ++k) {
            uint8_t byte = row[k / 2];
            uint8_t c = (k & 1) ? (byte >> 4) : (byte & 0xf);
            w[k] = qo_e2m1(c) * qo_e8m0(srow[k / 32]);
        }
    }
}

/* Values per block along K (the granularity K must respect): 16 for NVFP4, 256 for the K-quant
 * super-blocks (Q4_K, Q6_K), 32 otherwise. */
static int64_t qo_block_k(int fmt) { return fmt == QO_NVFP4 ? 16 : (fmt == QO_Q4_K || fmt == QO_Q6_K) ? 256 : 32; }

/* Full-tensor dequantization to fp64.  Returns 0, or -1 on a bad argument. */
int qo_dequant(int fmt, int64_t N, int64_t K, const uint8_t* blocks, const uint8_t* scales,
               float g, double* W) {
    if (qo_row_bytes(fmt, K) < 0 || K % qo_block_k(fmt)) return -1;
    for (int64_t n = 0; n < N; ++n) dequant_row(fmt, K, blocks, scales, g, n, W + n * K);
    return 0;
}

/* The fp32 value of each weight ("bit-exact dequant").  For Q8_0 / Q4_0 and for the NVFP4
 * product e2m1*e4m3 the fp64 value is exactly representable in fp32; the NVFP4 per-tensor
 * scale g is the one rounding: w32 = fp32( (e2m1*e4m3) * g ), rounded once to nearest-even.
 * Q4_K: both products d*scale*code and dmin*min are exact; their difference is rounded once.
 * Q6_K: d*scale*(code - 32) has at most 11 + 7 + 5 significant bits: exact in fp32. */
int qo_dequant_f32(int fmt, int64_t N, int64_t K, const uint8_t* blocks, const uint8_t* scales,
                   float g, float* W) {
    if (qo_row_bytes(fmt, K) < 0 || K % qo_block_k(fmt)) return -1;
    double* w = (double*)malloc(sizeof(double) * K);
    if (!w) return -1;
    for (int64_t n = 0; n < N; ++n) {
        dequant_row(fmt, K, blocks, scales, g, n, w);
        for (int64_t k = 0; k < K; ++k) W[n * K + k] = (float)w[k];
    }
    free(w);
    return 0;
}

/* ---------------------------------------------------------------- GEMV / GEMM */

/* y[m][j] = sum_k W[rows[j]][k] * x[m][k] and A[m][j] = sum_k |W[rows[j]][k] * x[m][k]|, fp64,
 * plain sequential sums, for the listed output rows (all rows when rows == NULL, nrows = N).
 * x is M x K (row stride K) already widened to fp64 by the caller (exactly).  Outputs are
 * M x nrows.  Returns 0 or -1. */
int qo_gemv_rows(int fmt, int64_t N, int64_t K, const uint8_t* blocks, const uint8_t* scales,
                 float g, int M, const double* x, const int64_t* rows, int64_t nrows, double* y,
                 double* A) {
    if (qo_row_bytes(fmt, K) < 0 || K % qo_block_k(fmt)) return -1;
    double* w = (double*)malloc(sizeof(double) * (K ? K : 1));
    if (!w) return -1;
    for (int64_t j = 0; j < nrows; ++j) {
        int64_t n = rows ? rows[j] : j;
        if (n < 0 || n >= N) { free(w); return -1; }
        dequant_row(fmt, K, blocks, scales, g, n, w);
        for (int m = 0; m < M; ++m) {
            double s = 0.0, a = 0.0;
            for (int64_t k = 0; k < K; ++k) {
                double p = w[k] * x[(int64_t)m * K + k];
                s += p;
                a += fabs(p);
            }
            y[(int64_t)m * nrows + j] = s;
            if (A) A[(int64_t)m * nrows + j] = a;
        }
    }
    free(w);
    return 0;
}

int qo_gemv(int fmt, int64_t N, int64_t K, const uint8_t* blocks, const uint8_t* scales, float g,
            int M, const double* x, double* y, double* A) {
    return qo_gemv_rows(fmt, N, K, blocks, scales, g, M, x, NULL, N, y, A);
}

/* SiLU gate, the activation of a gated MLP: silu(z) = z / (1 + exp(-z)). */
double qo_silu(double z) { return z / (1.0 + exp(-z)); }

/* h[m][i] = silu(gu[m][i]) * gu[m][I + i] for a gate_up output laid out as [gate ; up]
 * (the gate rows first, then the up rows).  Also returns the magnitude
 * Ah[m][i] = |silu'(g)| * Ag * |u| + |silu(g)| * Au  -- a first-order error scale used only
 * to size the tolerance of the fused epilogue. */
void qo_silu_gate(int M, int64_t I, const double* gu, const double* Agu, double* h, double* Ah) {
    for (int m = 0; m < M; ++m)
        for (int64_t i = 0; i < I; ++i) {
            double gv = gu[(int64_t)m * 2 * I + i], uv = gu[(int64_t)m * 2 * I + I + i];
            double sg = 1.0 / (1.0 + exp(-gv));
            h[(int64_t)m * I + i] = gv * sg * uv;
            if (Ah) {
                double dsil = sg * (1.0 + gv * (1.0 - sg)); /* d silu / dz */
                double ag = Agu ? Agu[(int64_t)m * 2 * I + i] : fabs(gv);
                double au = Agu ? Agu[(int64_t)m * 2 * I + I + i] : fabs(uv);
                Ah[(int64_t)m * I + i] = fabs(dsil) * ag * fabs(uv) + fabs(gv * sg) * au;
            }
        }
}

/* ---------------------------------------------------------------- MoE routing */

/* Router for one token: p = softmax(logits) in fp64; the top_k experts by descending p (a tie
 * goes to the lower expert index); weights renormalised over the selected experts.
 * softmax is strictly increasing in each logit, so ranking by p is ranking by the logits
 * themselves: the selection compares the given logits (exact comparisons of the inputs, the same
 * decision in any precision), and p is used only for the weights. */
void qo_route(int E, int top_k, const double* logits, int32_t* ids, double* wts) {
    double mx = -INFINITY, z = 0.0;
    double* p = (double*)malloc(sizeof(double) * E);
    char* taken = (char*)calloc(E, 1);
    for (int e = 0; e < E; ++e) mx = logits[e] > mx ? logits[e] : mx;
    for (int e = 0; e < E; ++e) { p[e] = exp(logits[e] - mx); z += p[e]; }
    for (int e = 0; e < E; ++e) p[e] /= z;
    double tot = 0.0;
    for (int s = 0; s < top_k; ++s) {
        int best = -1;
        for (int e = 0; e < E; ++e)
            if (!taken[e] && (best < 0 || logits[e] > logits[best])) best = e;
        taken[best] = 1;
        ids[s] = best;
        wts[s] = p[best];
        tot += p[best];
    }
    for (int s = 0; s < top_k; ++s) wts[s] /= tot;
    free(p);
    free(taken);
}

/* Full routed MoE layer in fp64 for M tokens:
 *   route each token; for each slot, gu = W_gu[e] x, h = silu(gate)*up, o = W_dn[e] h;
 *   y[m] = sum over slots (in slot order) of wts[m][slot] * o.
 * Experts are stacked: gate_up blocks [E][2I rows][...], down blocks [E][H rows][...]
 * (NVFP4: the matching scale planes, and one per-tensor scale per expert and matrix).
 * Outputs: ids, wts (M x top_k), h (M x top_k x I), y (M x H), A (M x H) with
 * A = sum_slot wts * sum_j |W_dn[j] * h_j| (the magnitude of the final contraction). */
int qo_moe(int fmt, int E, int64_t H, int64_t I, int top_k, const uint8_t* gu_blocks,
           const uint8_t* gu_scales, const float* gu_g, const uint8_t* dn_blocks,
           const uint8_t* dn_scales, const float* dn_g, int M, const double* logits,
           const double* x, int32_t* ids, double* wts, double* h, double* y, double* A) {
    int64_t gu_rb = qo_row_bytes(fmt, H), dn_rb = qo_row_bytes(fmt, I);
    if (gu_rb < 0 || dn_rb < 0) return -1;
    double* gu = (double*)malloc(sizeof(double) * 2 * I);
    double* o = (double*)malloc(sizeof(double) * H);
    double* oa = (double*)malloc(sizeof(double) * H);
    for (int m = 0; m < M; ++m) {
        qo_route(E, top_k, logits + (int64_t)m * E, ids + (int64_t)m * top_k,
                 wts + (int64_t)m * top_k);
        for (int64_t j = 0; j < H; ++j) { y[(int64_t)m * H + j] = 0.0; A[(int64_t)m * H + j] = 0.0; }
        for (int s = 0; s < top_k; ++s) {
            int e = ids[(int64_t)m * top_k + s];
            double ws = wts[(int64_t)m * top_k + s];
            const uint8_t* gb = gu_blocks + (int64_t)e * 2 * I * gu_rb;
            const int fp4 = fmt == QO_NVFP4 || fmt == QO_MXFP4;
            const uint8_t* gsc = fp4 ? gu_scales + (int64_t)e * 2 * I * (H / qo_block_k(fmt)) : NULL;
            const uint8_t* db = dn_blocks + (int64_t)e * H * dn_rb;
            const uint8_t* dsc = fp4 ? dn_scales + (int64_t)e * H * (I / qo_block_k(fmt)) : NULL;
            qo_gemv(fmt, 2 * I, H, gb, gsc, gu_g ? gu_g[e] : 1.0f, 1, x + (int64_t)m * H, gu, NULL);
            double* hm = h + ((int64_t)m * top_k + s) * I;
            qo_silu_gate(1, I, gu, NULL, hm, NULL);
            qo_gemv(fmt, H, I, db, dsc, dn_g ? dn_g[e] : 1.0f, 1, hm, o, oa);
            for (int64_t j = 0; j < H; ++j) {
                y[(int64_t)m * H + j] += ws * o[j];
                A[(int64_t)m * H + j] += fabs(ws) * oa[j];
            }
        }
    }
    free(gu);
    free(o);
    free(oa);
    return 0;
}

/* ---------------------------------------------------------------- NVFP4 activation quantizer */

/* Round a non-negative fp32 value to OCP E4M3 (fn), nearest-even, saturating at 448.
 * Written as a search over the 127 non-negative finite codes: the nearest code wins, and of two
 * equally near codes the one with an even mantissa (even code) wins. */
uint8_t qo_round_e4m3_satfinite(float v) {
    if (!(v > 0.0f)) return 0; /* zero, negative zero and NaN inputs never occur here */
    if (v >= 448.0f) return 0x7e;
    double dv = v;
    int best = 0;
    double bd = INFINITY;
    for (int c = 0; c <= 0x7e; ++c) {
        double d = fabs(qo_e4m3((uint8_t)c) - dv);
        if (d < bd || (d == bd && (c & 1) == 0 && (best & 1) == 1)) { bd = d; best = c; }
    }
    return (uint8_t)best;
}

/* Round an fp32 value to OCP E2M1, nearest-even, saturating at +-6; the sign of the input is
 * kept (a negative value that rounds to zero gives code 8, negative zero).  A search over the
 * eight magnitudes, as above. */
uint8_t qo_round_e2m1_satfinite(float v) {
    int neg = signbit(v) ? 1 : 0;
    double a = fabs((double)v);
    int best = 0;
    double bd = INFINITY;
    for (int c = 0; c < 8; ++c) {
        double d = fabs(qo_e2m1((uint8_t)c) - a);
        if (d < bd || (d == bd && (c & 1) == 0 && (best & 1) == 1)) { bd = d; best = c; }
    }
    if (a >= 6.0) best = 7;
    return (uint8_t)(best | (neg << 3));
}

/* NVFP4 quantization of a bf16 activation matrix X (M x K, given as fp32 values that are exact
 * bf16 numbers), the A operand of the chunk GEMM.  The pages name NVFP4 activations only through
 * the "mxf4nvf4" block-scaled MMA; the rule below is the adopted reading, all steps in fp32 with
 * IEEE round-to-nearest-even:
 *   a_g   = amax|X| / (6 * 448)                              (per-tensor fp32 scale)
 *   s_b   = E4M3_rne_satfinite( amax_b / (6 * a_g) )         (per 16 consecutive k of a row)
 *   code  = E2M1_rne_satfinite( x / (fp32(s_b) * a_g) )      (0 where s_b == 0)
 * When amax == 0 every scale and code is 0 and a_g = 0.
 * Output: codes [M][K/2] (two per byte, element 2i in the low nibble), scales [M][K/16], a_g. */
int qo_act_quant(int M, int64_t K, const float* X, uint8_t* codes, uint8_t* scales, float* a_g_out) {
    if (K % 16) return -1;
    float amax = 0.0f;
    for (int64_t i = 0; i < (int64_t)M * K; ++i) {
        float a = fabsf(X[i]);
        if (a > amax) amax = a;
    }
    volatile float six448 = 6.0f * 448.0f;
    volatile float a_g = amax / six448;
    *a_g_out = a_g;
    for (int m = 0; m < M; ++m)
        for (int64_t b = 0; b < K / 16; ++b) {
            const float* xb = X + (int64_t)m * K + b * 16;
            float bmax = 0.0f;
            for (int j = 0; j < 16; ++j) {
                float a = fabsf(xb[j]);
                if (a > bmax) bmax = a;
            }
            uint8_t s = 0;
            if (a_g > 0.0f) {
                volatile float den = 6.0f * a_g;
                volatile float q = bmax / den;
                s = qo_round_e4m3_satfinite(q);
            }
            scales[(int64_t)m * (K / 16) + b] = s;
            volatile float sf = (float)qo_e4m3(s);
            volatile float div = sf * a_g;
            for (int j = 0; j < 16; j += 2) {
                uint8_t c0 = 0, c1 = 0;
                if (div > 0.0f) {
                    volatile float v0 = xb[j] / div, v1 = xb[j + 1] / div;
                    c0 = qo_round_e2m1_satfinite(v0);
                    c1 = qo_round_e2m1_satfinite(v1);
                }
                codes[(int64_t)m * (K / 2) + b * 8 + j / 2] = (uint8_t)(c0 | (c1 << 4));
            }
        }
    return 0;
}

/* ---------------------------------------------------------------- MXFP4 activation quantizer */

/* MXFP4 quantization of a bf16 activation matrix X (M x K, fp32 values that are exact bf16
 * numbers), the A operand of the MXFP4 chunk GEMM.  The pages give MXFP4 as "E2M1 + UE8M0 block
 * scales, 4.25 bits per weight" (imp release notes v0.6) and nothing on quantizing activations;
 * the rule below is the OCP MX v1.0 conversion, the plainest reading for an MX operand.  For each
 * block of 32 consecutive k of a row, with amax_b its largest magnitude:
 *   e     = floor(log2(amax_b)) - 2        (2: the exponent of E2M1's largest value, 6 = 1.5 * 2^2)
 *   byte  = e + 127, clamped to [0, 254]  (the UE8M0 scale X = 2^(byte - 127))
 *   code  = E2M1_rne_satfinite( x / X )    (x / X is exact: a power-of-two scaling)
 * A block whose amax is 0 (or below 2^-125) gets byte 0.  A block holding an Inf or NaN gets the
 * UE8M0 NaN byte 0xFF and all-zero codes (finite activations are the case the chunk path serves).
 * Output: codes [M][K/2] (element 2i in the low nibble), scales [M][K/32]. */
int qo_act_quant_mx(int M, int64_t K, const float* X, uint8_t* codes, uint8_t* scales) {
    if (K % 32) return -1;
    for (int m = 0; m < M; ++m)
        for (int64_t b = 0; b < K / 32; ++b) {
            const float* xb = X + (int64_t)m * K + b * 32;
            double amax = 0.0;
            int special = 0;
            for (int j = 0; j < 32; ++j) {
                if (!isfinite(xb[j])) special = 1;
                double a = fabs((double)xb[j]);
                if (a > amax) amax = a;
            }
            uint8_t byte = 0;
            if (special) {
                byte = 0xFF;
            } else if (amax > 0.0) {
                int E;
                frexp(amax, &E); /* amax = f * 2^E, f in [0.5, 1): floor(log2(amax)) = E - 1 */
                int e = (E - 1) - 2;
                int bi = e + 127;
                byte = (uint8_t)(bi < 0 ? 0 : (bi > 254 ? 254 : bi));
            }
            scales[(int64_t)m * (K / 32) + b] = byte;
            for (int j = 0; j < 32; j += 2) {
                uint8_t c0 = 0, c1 = 0;
                if (!special) {
                    double inv = ldexp(1.0, 127 - (int)byte); /* 1 / X */
                    float v0 = (float)((double)xb[j] * inv), v1 = (float)((double)xb[j + 1] * inv);
                    c0 = qo_round_e2m1_satfinite(v0);
                    c1 = qo_round_e2m1_satfinite(v1);
                }
                codes[(int64_t)m * (K / 2) + b * 16 + j / 2] = (uint8_t)(c0 | (c1 << 4));
            }
        }
    return 0;
}
