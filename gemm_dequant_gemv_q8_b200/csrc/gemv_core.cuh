// gemv_core.cuh -- device routines shared by the dense GEMV and the MoE expert kernels:
// per-warp bulk-copy ring configuration, in-register code decoders, the per-unit dot products,
// the 8-lane reduce-scatter and the SiLU gate.
#pragma once
#include "qlin_common.cuh"

namespace qlin {

constexpr int kGemvWarps = 4;  // warps per CTA

template <int FMT>
struct RingCfg {
    static constexpr int D = 2;  // ring depth (units) per warp
    static constexpr int UB = unit_bytes(FMT);
    static constexpr int kSmem = kGemvWarps * D * (UB + 8);
    static constexpr int kCtasPerSm = (FMT == QLIN_Q8_0) ? 3 : 4;  // 12-16 warps per SM
};


// ------------------------------------------------------------------ code decoders
// Magic-exponent construction: OR-ing a nibble/byte into the mantissa of 2^E, placed so that its
// unit bit is the float's unit-in-last-place, gives exactly 2^E + code; subtracting (2^E + bias)
// leaves the signed code exactly.  Different nibble positions use different E, so no shifts.
__device__ __forceinline__ float magic(uint32_t w, uint32_t mask, uint32_t expbits) {
    return __uint_as_float((w & mask) | expbits);
}

// Q4_0 word: elements 8k..8k+7 (nibble i = element i).  One shared exponent 2^23 for every
// nibble position: the nibble at bits 4j (j = i mod 4, taken from w or w >> 16) gives the exact
// float 2^23 + code * 16^j, and subtracting 2^23 + 8 * 16^j leaves (code - 8) * 16^j exactly.
// The matching activations are pre-scaled by 16^-j (exact), see prescale_x_q4.  Returns four
// pairs for elements (0,1), (2,3), (4,5), (6,7).
__device__ __forceinline__ void dec_q4(uint32_t w, float2 (&p)[4]) {
    const uint32_t e23 = 0x4b000000u;
    const float2 c01 = make_float2(-(8388608.0f + 8.0f), -(8388608.0f + 128.0f));
    const float2 c23 = make_float2(-(8388608.0f + 2048.0f), -(8388608.0f + 32768.0f));
    const uint32_t h = w >> 16;
    p[0] = __fadd2_rn(make_float2(__uint_as_float((w & 0xfu) | e23), __uint_as_float((w & 0xf0u) | e23)), c01);
    p[1] = __fadd2_rn(make_float2(__uint_as_float((w & 0xf00u) | e23), __uint_as_float((w & 0xf000u) | e23)), c23);
    p[2] = __fadd2_rn(make_float2(__uint_as_float((h & 0xfu) | e23), __uint_as_float((h & 0xf0u) | e23)), c01);
    p[3] = __fadd2_rn(make_float2(__uint_as_float((h & 0xf00u) | e23), __uint_as_float((h & 0xf000u) | e23)), c23);
}

// Pre-scale a lane's 32 activations for dec_q4: element e (pair e/2) times 16^-(e mod 4).
template <int MP>
__device__ __forceinline__ void prescale_x_q4(float2 (&xv)[MP][16]) {
    const float2 s01 = make_float2(1.0f, 0.0625f), s23 = make_float2(0.00390625f, 0.000244140625f);
#pragma unroll
    for (int mm = 0; mm < MP; ++mm)
#pragma unroll
        for (int q = 0; q < 16; ++q) xv[mm][q] = __fmul2_rn(xv[mm][q], (q & 1) ? s23 : s01);
}

// Q8_0 word: 4 elements stored as q + 128 -> two pairs of q.
__device__ __forceinline__ void dec_q8(uint32_t w, float2 (&p)[2]) {
    const float2 c = make_float2(-(8388608.0f + 128.0f), -(32768.0f + 128.0f));
    const uint32_t h = w >> 16;
    p[0] = __fadd2_rn(make_float2(magic(w, 0xffu, 0x4b000000u), magic(w, 0xff00u, 0x47000000u)), c);
    p[1] = __fadd2_rn(make_float2(magic(h, 0xffu, 0x4b000000u), magic(h, 0xff00u, 0x47000000u)), c);
}

// NVFP4 word: elements 8k..8k+7, byte j = elements 2j (low nibble), 2j+1 -> four pairs of e2m1.
__device__ __forceinline__ void dec_fp4(uint32_t w, float2 (&p)[4]) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        uint32_t h2 = e2m1x2_to_f16x2(w >> (8 * j));
        p[j] = __half22float2(*reinterpret_cast<__half2*>(&h2));
    }
}

// ------------------------------------------------------------------ activations
// Lane's 32 activations of one part (elements k0 .. k0+31) for MP rows given by pointers (NULL
// row = zeros); elements at or beyond K read as 0 (NVFP4 K may end in the middle of a part).
template <bool XBF16, int MP>
__device__ __forceinline__ void load_x_rows(const void* const (&rows)[MP], int64_t k0, int64_t K,
                                            float2 (&xv)[MP][16]) {
    const int64_t left = K - k0;
#pragma unroll
    for (int mm = 0; mm < MP; ++mm) {
        const bool row_ok = rows[mm] != nullptr;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const bool ok = row_ok && left >= 16 * (h + 1);
            if (XBF16) {
                const uint4* src =
                    reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(rows[mm]) + k0 + 16 * h);
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                    uint4 v = ok ? src[q] : make_uint4(0, 0, 0, 0);
                    uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        xv[mm][8 * h + 4 * q + j] =
                            make_float2(__uint_as_float(u[j] << 16), __uint_as_float(u[j] & 0xffff0000u));
                }
            } else {
                const float4* src = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(rows[mm]) + k0 + 16 * h);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    float4 v = ok ? src[q] : make_float4(0.f, 0.f, 0.f, 0.f);
                    xv[mm][8 * h + 2 * q] = make_float2(v.x, v.y);
                    xv[mm][8 * h + 2 * q + 1] = make_float2(v.z, v.w);
                }
            }
        }
    }
}

// ------------------------------------------------------------------ NVFP4 x bf16: f16 products
// With bf16 activations every product e2m1 * x is exact in f16 arithmetic terms: e2m1 values are
// exact f16 numbers and a bf16 value (8 significant bits) is an exact f16 number once it is
// brought into f16's range.  Each 16-element block of a lane's activations is multiplied by a
// power of two 2^-s chosen so its largest magnitude lands in [2^14, 2^15) (exact), converted to
// f16 (exact except for elements more than 2^38 below the block maximum, whose contribution is
// far below fp32 rounding), and 2^s is folded into the block's E4M3 scale.  Products then go
// through fma.rn.f32.f16: exact products, fp32 sums.
template <int MP>
__device__ __forceinline__ void load_x_fp4h(const void* const (&rows)[MP], int64_t k0, int64_t K,
                                            uint32_t (&xh)[MP][16], float (&xsc)[MP][2]) {
    const int64_t left = K - k0;
#pragma unroll
    for (int mm = 0; mm < MP; ++mm) {
#pragma unroll
        for (int b = 0; b < 2; ++b) {
            const bool ok = rows[mm] != nullptr && left >= 16 * (b + 1);
            const uint4* src =
                reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(rows[mm]) + k0 + 16 * b);
            uint32_t u[8];
            {
                uint4 v0 = ok ? src[0] : make_uint4(0, 0, 0, 0);
                uint4 v1 = ok ? src[1] : make_uint4(0, 0, 0, 0);
                u[0] = v0.x; u[1] = v0.y; u[2] = v0.z; u[3] = v0.w;
                u[4] = v1.x; u[5] = v1.y; u[6] = v1.z; u[7] = v1.w;
            }
            uint32_t mx = 0;
#pragma unroll
            for (int q = 0; q < 8; ++q) mx = __vmaxu2(mx, u[q] & 0x7fff7fffu);
            const uint32_t mb = max(mx & 0xffffu, mx >> 16);
            int s = (int)(mb >> 7) - 141;  // block max exponent - 127 - 14
            s = s < -110 ? -110 : s;
            const float down = __uint_as_float((uint32_t)(127 - s) << 23);  // 2^-s
            xsc[mm][b] = __uint_as_float((uint32_t)(127 + s) << 23);        // 2^s
            const float2 dd = make_float2(down, down);
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                float2 f = make_float2(__uint_as_float(u[q] << 16), __uint_as_float(u[q] & 0xffff0000u));
                f = __fmul2_rn(f, dd);
                uint32_t h;
                asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(h) : "f"(f.y), "f"(f.x));  // low half = even element
                xh[mm][8 * b + q] = h;
            }
        }
    }
}

// acc0 += w.lo * x.lo, acc1 += w.hi * x.hi  (f16 operands, exact products, fp32 sums)
__device__ __forceinline__ void fma2_f16_f32(uint32_t w2, uint32_t x2, float& acc0, float& acc1) {
    asm("{\n .reg .f16 wl, wh, xl, xu;\n mov.b32 {wl, wh}, %2;\n mov.b32 {xl, xu}, %3;\n"
        " fma.rn.f32.f16 %0, wl, xl, %0;\n fma.rn.f32.f16 %1, wh, xu, %1;\n}\n"
        : "+f"(acc0), "+f"(acc1)
        : "r"(w2), "r"(x2));
}

// Four E2M1 codes pairs of one word -> four f16x2 (low half = even element).
__device__ __forceinline__ void dec_fp4_h(uint32_t w, uint32_t (&h)[4]) {
    asm("{\n .reg .b8 b0, b1, b2, b3;\n mov.b32 {b0, b1, b2, b3}, %4;\n"
        " cvt.rn.f16x2.e2m1x2 %0, b0;\n cvt.rn.f16x2.e2m1x2 %1, b1;\n"
        " cvt.rn.f16x2.e2m1x2 %2, b2;\n cvt.rn.f16x2.e2m1x2 %3, b3;\n}\n"
        : "=r"(h[0]), "=r"(h[1]), "=r"(h[2]), "=r"(h[3])
        : "r"(w));
}

// NVFP4 unit dot with f16 products (see load_x_fp4h); same contract as unit_dot.
template <int MP, bool ACC = false>
__device__ __forceinline__ void unit_dot_fp4h(const uint8_t* ub, int lane, const uint32_t (&xh)[MP][16],
                                              const float (&xsc)[MP][2], float (&res)[8][MP]) {
    const uint4 sv = lds128(ub + 4096 + lane * 16);
    const uint32_t sw[4] = {sv.x, sv.y, sv.z, sv.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const uint32_t sc = sw[i >> 1] >> (16 * (i & 1));
        const float e0 = e4m3_to_f32(sc & 0xffu), e1 = e4m3_to_f32((sc >> 8) & 0xffu);
        const uint4 c = lds128(ub + (lane + 32 * i) * 16);
        const uint32_t cw[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
        for (int b = 0; b < 2; ++b) {
            float a0[MP], a1[MP];
#pragma unroll
            for (int mm = 0; mm < MP; ++mm) a0[mm] = a1[mm] = 0.f;
#pragma unroll
            for (int kk = 0; kk < 2; ++kk) {
                const int k = 2 * b + kk;
                uint32_t wh[4];
                dec_fp4_h(cw[k], wh);
#pragma unroll
                for (int mm = 0; mm < MP; ++mm)
#pragma unroll
                    for (int jj = 0; jj < 4; ++jj) fma2_f16_f32(wh[jj], xh[mm][4 * k + jj], a0[mm], a1[mm]);
            }
            const float e = b ? e1 : e0;
#pragma unroll
            for (int mm = 0; mm < MP; ++mm) {
                const float sc_b = e * xsc[mm][b];
                res[i][mm] = (ACC || b) ? fmaf(sc_b, a0[mm] + a1[mm], res[i][mm]) : sc_b * (a0[mm] + a1[mm]);
            }
        }
    }
}

// ------------------------------------------------------------------ one unit, rows of one m-pass
// res[i][mm] = contribution of (row (lane/8) + 4i, part lane%8) for activation row m0 + mm;
// with ACC the contribution is added to res instead (one fused multiply-add per block).
template <int FMT, int MP, bool ACC = false>
__device__ __forceinline__ void unit_dot(const uint8_t* ub, int lane, const float2 (&xv)[MP][16],
                                         float (&res)[8][MP]) {
    const uint4 sv = lds128(ub + code_bytes(FMT) + lane * 16);
    const uint32_t sw[4] = {sv.x, sv.y, sv.z, sv.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const uint32_t sc = sw[i >> 1] >> (16 * (i & 1));  // 16 bits of scale for (row, part)
        if (FMT == QLIN_Q4_0) {
            const uint4 c = lds128(ub + (lane + 32 * i) * 16);
            const uint32_t cw[4] = {c.x, c.y, c.z, c.w};
            float2 s0[MP], s1[MP];
#pragma unroll
            for (int mm = 0; mm < MP; ++mm) s0[mm] = s1[mm] = make_float2(0.f, 0.f);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                float2 p[4];
                dec_q4(cw[k], p);
#pragma unroll
                for (int mm = 0; mm < MP; ++mm) {
                    s0[mm] = __ffma2_rn(p[0], xv[mm][4 * k + 0], s0[mm]);
                    s1[mm] = __ffma2_rn(p[1], xv[mm][4 * k + 1], s1[mm]);
                    s0[mm] = __ffma2_rn(p[2], xv[mm][4 * k + 2], s0[mm]);
                    s1[mm] = __ffma2_rn(p[3], xv[mm][4 * k + 3], s1[mm]);
                }
            }
            const float d = fp16_bits_to_f32(sc & 0xffffu);
#pragma unroll
            for (int mm = 0; mm < MP; ++mm) {
                const float bsum = (s0[mm].x + s0[mm].y) + (s1[mm].x + s1[mm].y);
                res[i][mm] = ACC ? fmaf(d, bsum, res[i][mm]) : d * bsum;
            }
        } else if (FMT == QLIN_Q8_0) {
            const uint4 c0 = lds128(ub + (lane + 32 * i) * 16);
            const uint4 c1 = lds128(ub + 4096 + (lane + 32 * i) * 16);
            const uint32_t cw[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
            float2 s0[MP], s1[MP];
#pragma unroll
            for (int mm = 0; mm < MP; ++mm) s0[mm] = s1[mm] = make_float2(0.f, 0.f);
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                float2 p[2];
                dec_q8(cw[k], p);
#pragma unroll
                for (int mm = 0; mm < MP; ++mm) {
                    s0[mm] = __ffma2_rn(p[0], xv[mm][2 * k + 0], s0[mm]);
                    s1[mm] = __ffma2_rn(p[1], xv[mm][2 * k + 1], s1[mm]);
                }
            }
            const float d = fp16_bits_to_f32(sc & 0xffffu);
#pragma unroll
            for (int mm = 0; mm < MP; ++mm) {
                const float bsum = (s0[mm].x + s0[mm].y) + (s1[mm].x + s1[mm].y);
                res[i][mm] = ACC ? fmaf(d, bsum, res[i][mm]) : d * bsum;
            }
        } else {  // NVFP4: two 16-element blocks per part, one E4M3 scale each
            const uint4 c = lds128(ub + (lane + 32 * i) * 16);
            const uint32_t cw[4] = {c.x, c.y, c.z, c.w};
            float bs[2][MP];
#pragma unroll
            for (int b = 0; b < 2; ++b) {
                float2 s0[MP], s1[MP];
#pragma unroll
                for (int mm = 0; mm < MP; ++mm) s0[mm] = s1[mm] = make_float2(0.f, 0.f);
#pragma unroll
                for (int kk = 0; kk < 2; ++kk) {
                    const int k = 2 * b + kk;
                    float2 p[4];
                    dec_fp4(cw[k], p);
#pragma unroll
                    for (int mm = 0; mm < MP; ++mm) {
                        s0[mm] = __ffma2_rn(p[0], xv[mm][4 * k + 0], s0[mm]);
                        s1[mm] = __ffma2_rn(p[1], xv[mm][4 * k + 1], s1[mm]);
                        s0[mm] = __ffma2_rn(p[2], xv[mm][4 * k + 2], s0[mm]);
                        s1[mm] = __ffma2_rn(p[3], xv[mm][4 * k + 3], s1[mm]);
                    }
                }
#pragma unroll
                for (int mm = 0; mm < MP; ++mm) bs[b][mm] = (s0[mm].x + s0[mm].y) + (s1[mm].x + s1[mm].y);
            }
            const float e0 = e4m3_to_f32(sc & 0xffu), e1 = e4m3_to_f32((sc >> 8) & 0xffu);
#pragma unroll
            for (int mm = 0; mm < MP; ++mm)
                res[i][mm] = ACC ? fmaf(e1, bs[1][mm], fmaf(e0, bs[0][mm], res[i][mm])) : e0 * bs[0][mm] + e1 * bs[1][mm];
        }
    }
}

// Reduce-scatter over the 8 lanes that share (lane / 8): lane ends with the sum over parts of
// row slot i = lane % 8 (that is, tile row (lane / 8) + 4 * (lane % 8)).  Fixed order.
template <int MP>
__device__ __forceinline__ void reduce_scatter8(float (&res)[8][MP], int lane, float (&out)[MP]) {
#pragma unroll
    for (int mm = 0; mm < MP; ++mm) {
        float v4[4], v2[2];
        const bool b2 = lane & 4, b1 = lane & 2, b0 = lane & 1;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            float send = b2 ? res[j][mm] : res[j + 4][mm];
            float keep = b2 ? res[j + 4][mm] : res[j][mm];
            float got = __shfl_xor_sync(0xffffffffu, send, 4);
            v4[j] = b2 ? (got + keep) : (keep + got);  // lower lane's value first
        }
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            float send = b1 ? v4[j] : v4[j + 2];
            float keep = b1 ? v4[j + 2] : v4[j];
            float got = __shfl_xor_sync(0xffffffffu, send, 2);
            v2[j] = b1 ? (got + keep) : (keep + got);
        }
        float send = b0 ? v2[0] : v2[1];
        float keep = b0 ? v2[1] : v2[0];
        float got = __shfl_xor_sync(0xffffffffu, send, 1);
        out[mm] = b0 ? (got + keep) : (keep + got);
    }
}

// ------------------------------------------------------------------ tile output
// silu(g) = g * sigmoid(g), with exp taken of -|g| only (no overflow for very negative g).
__device__ __forceinline__ float silu_f32(float g) {
    const float e = expf(-fabsf(g));
    const float sig = g >= 0.f ? 1.0f / (1.0f + e) : e / (1.0f + e);
    return g * sig;
}

}  // namespace qlin
