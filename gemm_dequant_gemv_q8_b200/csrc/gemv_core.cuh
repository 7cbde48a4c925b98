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
    static constexpr int kCtasPerSm = (FMT == QLIN_Q8_0 || FMT == QLIN_Q6_K) ? 3 : 4;  // 12-16 warps per SM
};
// CTAs per SM of the persistent grids (the ring's shared memory allows 3 for the byte-code formats).
inline int ring_ctas_per_sm(int fmt) { return (fmt == QLIN_Q8_0 || fmt == QLIN_Q6_K) ? 3 : 4; }


// ------------------------------------------------------------------ code decoders
// Q4_0 / Q8_0 codes as denormal floats.  A 32-bit pattern P < 2^24 read as an fp32 number is
// exactly P * 2^-149 (patterns below 2^23 are denormals, 2^23 .. 2^24-1 continue seamlessly as
// the first binade).  So a nibble or byte masked in place at bit 4j (8j), with nothing else set,
// IS the float n * 2^(4j) * 2^-149: one AND per weight, no shift, no subtraction.  Codes are
// unsigned (Q4_0 nibble n = q + 8, Q8_0 byte = q + 128, Q6_K byte = q + 32).  The offset is
// removed from each decoded value before it is multiplied: adding -offset * 2^(position - 149)
// to n * 2^(position - 149) is exact (both are multiples of 2^-149 below 2^-125), one packed add
// per two values, so every product and partial sum is of the signed weight q.  (Removing the
// offset once per block instead, from a sum of the activations, leaves rounding errors of the
// size of offset * sum|x| in the block sum: for blocks of small codes that is far above
// 2e-6 * sum|q x|.)  Q4_K codes (0..15, placed as Q4_0's) go through the same decoder without an
// offset; their sub-block min multiplies a sum of the activations (prep_x_q4), as the format
// defines w = d * scale * code - dmin * min.
// Activations are pre-scaled by 2^(kXExp - 4j) (2^(kXExp - 8j) for Q8_0), so every product is
// the exact n * x * 2^(kXExp - 149) computed inside an fp32 FMA; block sums carry 2^(kXExp - 149)
// and the tile output multiplies by kDenormUnscale = 2^(149 - kXExp).  Products stay normal and
// exact for 2^-40 <= |x| < 2^65; smaller activations lose relative precision (each product is
// then exact to 2^-63 in absolute terms), larger ones overflow.
constexpr int kXExp = 63;
constexpr float kDenormUnscale = 0x1p86f;  // 2^(149 - kXExp)

// Output scale of a format's block sums: the NVFP4 per-tensor scale, 1 for MXFP4 (its block
// scales are applied in full per block), or 2^86 for Q4_0 / Q8_0 / Q4_K.
template <int FMT>
__device__ __forceinline__ float format_out_scale(const uint8_t* packed) {
    if (FMT == QLIN_NVFP4) return reinterpret_cast<const PackedHeader*>(packed)->global_scale;
    if (FMT == QLIN_MXFP4) return 1.0f;
    return kDenormUnscale;
}

// Q4_0 words w0, w1 (elements 8k..8k+7 and 8k+8..8k+15, element i of a word at bits 4i).
// Elements 0..5 of each word are masked in place (position j = i).  The top bytes of the two
// words (elements 6 and 7 of each) are gathered by one byte permute into bits 0..15 of a third
// word, where they sit at positions 0, 1 (word w0) and 2, 3 (word w1).  Pairs per word: (0,1)
// (2,3) (4,5) (6,7).  SIGNED (Q4_0): the offset 8 is removed from each value (positions 4j:
// -8 * 2^(4j - 149) = -2^(4j - 146)).
template <bool SIGNED>
__device__ __forceinline__ void dec_q4_pair(uint32_t w0, uint32_t w1, float2 (&p0)[4], float2 (&p1)[4]) {
    const uint32_t top = __byte_perm(w0, w1, 0x0073u);  // byte 0 = w0 byte 3, byte 1 = w1 byte 3
    p0[0] = make_float2(__uint_as_float(w0 & 0xfu), __uint_as_float(w0 & 0xf0u));
    p0[1] = make_float2(__uint_as_float(w0 & 0xf00u), __uint_as_float(w0 & 0xf000u));
    p0[2] = make_float2(__uint_as_float(w0 & 0xf0000u), __uint_as_float(w0 & 0xf00000u));
    p0[3] = make_float2(__uint_as_float(top & 0xfu), __uint_as_float(top & 0xf0u));
    p1[0] = make_float2(__uint_as_float(w1 & 0xfu), __uint_as_float(w1 & 0xf0u));
    p1[1] = make_float2(__uint_as_float(w1 & 0xf00u), __uint_as_float(w1 & 0xf000u));
    p1[2] = make_float2(__uint_as_float(w1 & 0xf0000u), __uint_as_float(w1 & 0xf00000u));
    p1[3] = make_float2(__uint_as_float(top & 0xf00u), __uint_as_float(top & 0xf000u));
    if (SIGNED) {
        const float2 b01 = make_float2(-0x1p-146f, -0x1p-142f), b23 = make_float2(-0x1p-138f, -0x1p-134f);
        const float2 b45 = make_float2(-0x1p-130f, -0x1p-126f);
        p0[0] = __fadd2_rn(p0[0], b01), p0[1] = __fadd2_rn(p0[1], b23), p0[2] = __fadd2_rn(p0[2], b45);
        p0[3] = __fadd2_rn(p0[3], b01);  // positions 0, 1
        p1[0] = __fadd2_rn(p1[0], b01), p1[1] = __fadd2_rn(p1[1], b23), p1[2] = __fadd2_rn(p1[2], b45);
        p1[3] = __fadd2_rn(p1[3], b23);  // positions 2, 3
    }
}

// Q8_0 word: elements 4k..4k+3 stored as q + 128 in bytes 0..3 (Q6_K: q + 32).  Bytes 0..2 are
// masked in place (positions 0, 1, 2); byte 3 is w >> 24 (position 0).  Pairs: (0,1) (2,3).  The
// offset OFF is removed from each value: -OFF * 2^(8j - 149) at position j.
template <int OFF>
__device__ __forceinline__ void dec_q8(uint32_t w, float2 (&p)[2]) {
    constexpr float b0 = -(float)OFF * 0x1p-149f, b1 = -(float)OFF * 0x1p-141f, b2 = -(float)OFF * 0x1p-133f;
    p[0] = __fadd2_rn(make_float2(__uint_as_float(w & 0xffu), __uint_as_float(w & 0xff00u)), make_float2(b0, b1));
    p[1] = __fadd2_rn(make_float2(__uint_as_float(w & 0xff0000u), __uint_as_float(w >> 24)), make_float2(b2, b0));
}

// Sum of one lane's 32 activations (the Q4_K min term), in the order unit_dot adds its products:
// two interleaved pair chains, then the pairs combined lane-wise, then the two halves.
__device__ __forceinline__ float offset_sum(const float2 (&x)[16]) {
    float2 t0 = x[0], t1 = x[1];
#pragma unroll
    for (int q = 2; q < 16; q += 2) {
        t0 = __fadd2_rn(t0, x[q]);
        t1 = __fadd2_rn(t1, x[q + 1]);
    }
    const float2 u = __fadd2_rn(t0, t1);
    return u.x + u.y;
}

// Prepare a lane's 32 activations for the Q4_0 / Q4_K decoder: element e (pair e/2) times
// 2^(kXExp - 4 j) with j the decoder's position of element e mod 8.  Q4_K also takes
// xb = sum * 2^(kXExp - 149), the factor of its min term; Q4_0 needs none (xb = 0).
template <int MP, bool K4 = false>
__device__ __forceinline__ void prep_x_q4(float2 (&xv)[MP][16], float2 (&xb)[MP]) {
    constexpr float c = 0x1p-86f;  // 2^(kXExp - 149)
    const float2 s0 = make_float2(0x1p63f, 0x1p59f), s1 = make_float2(0x1p55f, 0x1p51f);
    const float2 s2 = make_float2(0x1p47f, 0x1p43f);
#pragma unroll
    for (int mm = 0; mm < MP; ++mm) {
        xb[mm] = make_float2(K4 ? c * offset_sum(xv[mm]) : 0.f, 0.f);
#pragma unroll
        for (int q = 0; q < 16; ++q)  // pair q = 4k + (q & 3); pair 4k+3 sits at positions 0,1 (k even) or 2,3
            xv[mm][q] = __fmul2_rn(xv[mm][q], (q & 3) == 0 ? s0 : (q & 3) == 1 ? s1 : (q & 3) == 2 ? s2 : ((q >> 2) & 1) ? s1 : s0);
    }
}

// Prepare a lane's 32 activations for the Q8_0 / Q6_K decoder (codes in the same byte positions;
// the decoder removes their offsets): pairs (4k, 4k+1) times (2^63, 2^55) and (4k+2, 4k+3) times
// (2^47, 2^63).  No activation sum is needed (xb = 0).
template <int MP>
__device__ __forceinline__ void prep_x_q8(float2 (&xv)[MP][16], float2 (&xb)[MP]) {
    const float2 s0 = make_float2(0x1p63f, 0x1p55f), s1 = make_float2(0x1p47f, 0x1p63f);
#pragma unroll
    for (int mm = 0; mm < MP; ++mm) {
        xb[mm] = make_float2(0.f, 0.f);
#pragma unroll
        for (int q = 0; q < 16; ++q) xv[mm][q] = __fmul2_rn(xv[mm][q], (q & 1) ? s1 : s0);
    }
}

// Prepare a lane's activations for unit_dot<FMT> (NVFP4 needs no preparation; xb is unused).
template <int FMT, int MP>
__device__ __forceinline__ void prep_x(float2 (&xv)[MP][16], float2 (&xb)[MP]) {
    if (FMT == QLIN_Q4_0) prep_x_q4<MP>(xv, xb);
    else if (FMT == QLIN_Q4_K) prep_x_q4<MP, true>(xv, xb);
    else if (FMT == QLIN_Q8_0) prep_x_q8<MP>(xv, xb);
    else if (FMT == QLIN_Q6_K) prep_x_q8<MP>(xv, xb);
    else {
#pragma unroll
        for (int mm = 0; mm < MP; ++mm) xb[mm] = make_float2(0.f, 0.f);
    }
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
// 16-byte activation load; CG = through L2 only (activations written earlier by the same grid).
template <bool CG, typename V>
__device__ __forceinline__ V ldx16(const V* p) {
    if constexpr (CG) return __ldcg(p);
    else return *p;
}

// Lane's 32 activations of one part (elements k0 .. k0+31) for MP rows given by pointers (NULL
// row = zeros); elements at or beyond K read as 0 (NVFP4 K may end in the middle of a part).
template <bool XBF16, int MP, bool CG = false>
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
                    uint4 v = ok ? ldx16<CG>(src + q) : make_uint4(0, 0, 0, 0);
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
                    float4 v = ok ? ldx16<CG>(src + q) : make_float4(0.f, 0.f, 0.f, 0.f);
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
// One 16-element block of bf16 activations (8 words, two elements each) -> eight f16x2 words
// scaled by 2^-s, and 2^s.
__device__ __forceinline__ void fp4h_block(const uint32_t (&u)[8], uint32_t* xh, float& xsc) {
    uint32_t mx = 0;
#pragma unroll
    for (int q = 0; q < 8; ++q) mx = __vmaxu2(mx, u[q] & 0x7fff7fffu);
    const uint32_t mb = max(mx & 0xffffu, mx >> 16);
    int s = (int)(mb >> 7) - 141;  // block max exponent - 127 - 14
    s = s < -110 ? -110 : s;
    const float down = __uint_as_float((uint32_t)(127 - s) << 23);  // 2^-s
    xsc = __uint_as_float((uint32_t)(127 + s) << 23);               // 2^s
    const float2 dd = make_float2(down, down);
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        float2 f = make_float2(__uint_as_float(u[q] << 16), __uint_as_float(u[q] & 0xffff0000u));
        f = __fmul2_rn(f, dd);
        uint32_t h;
        asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(h) : "f"(f.y), "f"(f.x));  // low half = even element
        xh[q] = h;
    }
}

template <int MP, bool CG = false>
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
                uint4 v0 = ok ? ldx16<CG>(src) : make_uint4(0, 0, 0, 0);
                uint4 v1 = ok ? ldx16<CG>(src + 1) : make_uint4(0, 0, 0, 0);
                u[0] = v0.x; u[1] = v0.y; u[2] = v0.z; u[3] = v0.w;
                u[4] = v1.x; u[5] = v1.y; u[6] = v1.z; u[7] = v1.w;
            }
            fp4h_block(u, &xh[mm][8 * b], xsc[mm][b]);
        }
    }
}

// ------------------------------------------------------------------ activations staged in smem
// A unit's activation slice (256 values per row) staged in shared memory by per-lane 16-byte
// cp.async copies, one unit ahead of its use, so the L2 latency of the activations overlaps the
// previous unit's arithmetic.  Part p (32 values) of row m sits at m * 8 * pitch + p * pitch:
// the 16-byte pad per part puts the eight parts that a quarter-warp reads at once on disjoint
// banks.  Values at or beyond K are zero-filled by the copy (K is a multiple of 16).
template <bool XBF16>
struct XStage {
    static constexpr int kPitch = XBF16 ? 80 : 144;   // bytes per part (64 or 128 + 16)
    static constexpr int kVecPerPart = XBF16 ? 4 : 8;  // 16-byte vectors per part
    static constexpr int kRowBytes = 8 * kPitch;
};

__device__ __forceinline__ void cp_async16_zfill(void* smem_dst, const void* gsrc, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(smem_dst)), "l"(gsrc),
                 "r"(src_bytes)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

// Issue the copies of k-group g of MP rows (row m at x + m * ldx; rows >= M zero-filled).
// Stage the k-group g slice of MP activation rows (row mm at rows[mm]; NULL rows and values at or
// beyond K are zero-filled) into buf, 16-byte cp.async copies in the XStage layout.  `any` is a
// valid global address given to the zero-filling copies (they read nothing from it).
template <bool XBF16, int MP>
__device__ __forceinline__ void stage_x_rows(const void* const (&rows)[MP], int64_t K, int g, uint8_t* buf, int lane,
                                             const void* any) {
    using S = XStage<XBF16>;
    constexpr int kEl = XBF16 ? 8 : 4;  // values per vector
    constexpr int kEs = XBF16 ? 2 : 4;  // bytes per value
#pragma unroll
    for (int mm = 0; mm < MP; ++mm) {
        const uint8_t* row = reinterpret_cast<const uint8_t*>(rows[mm]);
#pragma unroll
        for (int i = 0; i < (8 * S::kVecPerPart) / 32; ++i) {
            const int vi = lane + 32 * i, p = vi / S::kVecPerPart, q = vi % S::kVecPerPart;
            const int64_t el = (int64_t)g * kGroupK + (int64_t)vi * kEl;
            const bool ok = row != nullptr && el < K;
            cp_async16_zfill(buf + mm * S::kRowBytes + p * S::kPitch + q * 16,
                             ok ? (const void*)(row + el * kEs) : any, ok ? 16u : 0u);
        }
    }
    cp_async_commit();
}

template <bool XBF16, int MP>
__device__ __forceinline__ void stage_x(const void* x, int64_t ldx, int M, int64_t K, int g, uint8_t* buf, int lane) {
    constexpr int kEs = XBF16 ? 2 : 4;
    const void* rows[MP];
#pragma unroll
    for (int mm = 0; mm < MP; ++mm)
        rows[mm] = mm < M ? (const void*)(reinterpret_cast<const uint8_t*>(x) + (int64_t)mm * ldx * kEs) : nullptr;
    stage_x_rows<XBF16, MP>(rows, K, g, buf, lane, x);
}

// A lane's 32 activations of its part from the staged slice (same result as load_x_rows).
template <bool XBF16, int MP>
__device__ __forceinline__ void load_x_staged(const uint8_t* buf, int part, float2 (&xv)[MP][16]) {
    using S = XStage<XBF16>;
#pragma unroll
    for (int mm = 0; mm < MP; ++mm) {
        const uint8_t* b = buf + mm * S::kRowBytes + part * S::kPitch;
        if (XBF16) {
#pragma unroll
            for (int vq = 0; vq < 4; ++vq) {
                const uint4 v = lds128(b + 16 * vq);
                const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    xv[mm][4 * vq + j] = make_float2(__uint_as_float(u[j] << 16), __uint_as_float(u[j] & 0xffff0000u));
            }
        } else {
#pragma unroll
            for (int vq = 0; vq < 8; ++vq) {
                const uint4 v = lds128(b + 16 * vq);
                xv[mm][2 * vq] = make_float2(__uint_as_float(v.x), __uint_as_float(v.y));
                xv[mm][2 * vq + 1] = make_float2(__uint_as_float(v.z), __uint_as_float(v.w));
            }
        }
    }
}

// The NVFP4 f16-product activations (see load_x_fp4h) from a staged bf16 slice.
template <int MP>
__device__ __forceinline__ void load_x_fp4h_staged(const uint8_t* buf, int part, uint32_t (&xh)[MP][16],
                                                   float (&xsc)[MP][2]) {
    using S = XStage<true>;
#pragma unroll
    for (int mm = 0; mm < MP; ++mm) {
        const uint8_t* bp = buf + mm * S::kRowBytes + part * S::kPitch;
#pragma unroll
        for (int b = 0; b < 2; ++b) {
            const uint4 v0 = lds128(bp + 32 * b), v1 = lds128(bp + 32 * b + 16);
            const uint32_t u[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
            fp4h_block(u, &xh[mm][8 * b], xsc[mm][b]);
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

// NVFP4 / MXFP4 unit dot with f16 products (see load_x_fp4h); same contract as unit_dot.
// FMT: QLIN_NVFP4 (two E4M3 scales per part) or QLIN_MXFP4 (one UE8M0 scale for both halves).
template <int MP, bool ACC = false, int FMT = QLIN_NVFP4>
__device__ __forceinline__ void unit_dot_fp4h(const uint8_t* ub, int lane, const uint32_t (&xh)[MP][16],
                                              const float (&xsc)[MP][2], float (&res)[8][MP]) {
    uint32_t sw[4];
    if (FMT == QLIN_MXFP4) {
        const uint2 s2 = *reinterpret_cast<const uint2*>(ub + 4096 + lane * 8);
        sw[0] = s2.x, sw[1] = s2.y, sw[2] = sw[3] = 0u;
    } else {
        const uint4 sv = lds128(ub + 4096 + lane * 16);
        sw[0] = sv.x, sw[1] = sv.y, sw[2] = sv.z, sw[3] = sv.w;
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        float e0, e1;
        if (FMT == QLIN_MXFP4) {
            e0 = e1 = e8m0_to_f32(sw[i >> 2] >> (8 * (i & 3)));
        } else {
            const uint32_t sc = sw[i >> 1] >> (16 * (i & 1));
            e0 = e4m3_to_f32(sc & 0xffu), e1 = e4m3_to_f32((sc >> 8) & 0xffu);
        }
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
                                         const float2 (&xb)[MP], float (&res)[8][MP]) {
    uint32_t sw[4];
    if (FMT == QLIN_MXFP4) {  // 8 bits of scale per (row, part)
        const uint2 s2 = *reinterpret_cast<const uint2*>(ub + code_bytes(FMT) + lane * 8);
        sw[0] = s2.x, sw[1] = s2.y, sw[2] = sw[3] = 0u;
    } else {
        const uint4 sv = lds128(ub + code_bytes(FMT) + lane * 16);
        sw[0] = sv.x, sw[1] = sv.y, sw[2] = sv.z, sw[3] = sv.w;
    }
    constexpr bool kRowD = FMT == QLIN_Q4_K || FMT == QLIN_Q6_K;
    uint32_t dmw[kRowD ? 8 : 1];  // K-quants: {d, dmin} (Q6_K: {d, 0}) of the lane's 8 rows
    if (kRowD) {
        const uint8_t* dp = ub + row_d_off(FMT) + (lane >> 3) * 32;
        const uint4 d0 = lds128(dp), d1 = lds128(dp + 16);
        const uint32_t t[8] = {d0.x, d0.y, d0.z, d0.w, d1.x, d1.y, d1.z, d1.w};
#pragma unroll
        for (int i = 0; i < (kRowD ? 8 : 1); ++i) dmw[i] = t[i];
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        // 16 bits of scale for (row, part); MXFP4: 8 bits
        const uint32_t sc = FMT == QLIN_MXFP4 ? (sw[i >> 2] >> (8 * (i & 3))) : (sw[i >> 1] >> (16 * (i & 1)));
        if (FMT == QLIN_Q4_0 || FMT == QLIN_Q4_K) {
            const uint4 c = lds128(ub + (lane + 32 * i) * 16);
            const uint32_t cw[4] = {c.x, c.y, c.z, c.w};
            float2 s0[MP], s1[MP];
#pragma unroll
            for (int mm = 0; mm < MP; ++mm) s0[mm] = s1[mm] = make_float2(0.f, 0.f);
#pragma unroll
            for (int kp = 0; kp < 2; ++kp) {
                float2 p[2][4];
                dec_q4_pair<FMT == QLIN_Q4_0>(cw[2 * kp], cw[2 * kp + 1], p[0], p[1]);
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int k = 2 * kp + h;
#pragma unroll
                    for (int mm = 0; mm < MP; ++mm) {
                        s0[mm] = __ffma2_rn(p[h][0], xv[mm][4 * k + 0], s0[mm]);
                        s1[mm] = __ffma2_rn(p[h][1], xv[mm][4 * k + 1], s1[mm]);
                        s0[mm] = __ffma2_rn(p[h][2], xv[mm][4 * k + 2], s0[mm]);
                        s1[mm] = __ffma2_rn(p[h][3], xv[mm][4 * k + 3], s1[mm]);
                    }
                }
            }
            if (FMT == QLIN_Q4_K) {  // d * scale * sum(code x) - dmin * min * sum(x), both factors exact
                const float2 dd = __half22float2(*reinterpret_cast<const __half2*>(&dmw[kRowD ? i : 0]));
                const float ka = dd.x * (float)(sc & 63u), kb = dd.y * (float)((sc >> 6) & 63u);
#pragma unroll
                for (int mm = 0; mm < MP; ++mm) {
                    const float2 u = __fadd2_rn(s0[mm], s1[mm]);
                    const float base = ACC ? fmaf(-kb, xb[mm].x, res[i][mm]) : -kb * xb[mm].x;
                    res[i][mm] = fmaf(ka, u.x + u.y, base);
                }
            } else {
                const float d = fp16_bits_to_f32(sc & 0xffffu);
#pragma unroll
                for (int mm = 0; mm < MP; ++mm) {
                    const float2 u = __fadd2_rn(s0[mm], s1[mm]);
                    const float bsum = u.x + u.y;
                    res[i][mm] = ACC ? fmaf(d, bsum, res[i][mm]) : d * bsum;
                }
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
                dec_q8<128>(cw[k], p);
#pragma unroll
                for (int mm = 0; mm < MP; ++mm) {
                    s0[mm] = __ffma2_rn(p[0], xv[mm][2 * k + 0], s0[mm]);
                    s1[mm] = __ffma2_rn(p[1], xv[mm][2 * k + 1], s1[mm]);
                }
            }
            const float d = fp16_bits_to_f32(sc & 0xffffu);
#pragma unroll
            for (int mm = 0; mm < MP; ++mm) {
                const float2 u = __fadd2_rn(s0[mm], s1[mm]);
                const float bsum = u.x + u.y;
                res[i][mm] = ACC ? fmaf(d, bsum, res[i][mm]) : d * bsum;
            }
        } else if (FMT == QLIN_Q6_K) {  // Q8_0's byte planes holding 6-bit codes; a scale per 16 values
            const uint4 c0 = lds128(ub + (lane + 32 * i) * 16);
            const uint4 c1 = lds128(ub + 4096 + (lane + 32 * i) * 16);
            const uint32_t cw[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
            float2 s0[2][MP], s1[2][MP];  // [16-value block][row]
#pragma unroll
            for (int b = 0; b < 2; ++b)
#pragma unroll
                for (int mm = 0; mm < MP; ++mm) s0[b][mm] = s1[b][mm] = make_float2(0.f, 0.f);
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                float2 p[2];
                dec_q8<32>(cw[k], p);
#pragma unroll
                for (int mm = 0; mm < MP; ++mm) {
                    s0[k >> 2][mm] = __ffma2_rn(p[0], xv[mm][2 * k + 0], s0[k >> 2][mm]);
                    s1[k >> 2][mm] = __ffma2_rn(p[1], xv[mm][2 * k + 1], s1[k >> 2][mm]);
                }
            }
            const float d = __half2float(__ushort_as_half((unsigned short)(dmw[kRowD ? i : 0] & 0xffffu)));
            const float e0 = d * (float)(int8_t)(sc & 0xffu), e1 = d * (float)(int8_t)((sc >> 8) & 0xffu);  // exact
#pragma unroll
            for (int mm = 0; mm < MP; ++mm) {
                const float2 u0 = __fadd2_rn(s0[0][mm], s1[0][mm]), u1 = __fadd2_rn(s0[1][mm], s1[1][mm]);
                const float b0 = u0.x + u0.y, b1 = u1.x + u1.y;
                res[i][mm] = fmaf(e1, b1, ACC ? fmaf(e0, b0, res[i][mm]) : e0 * b0);
            }
        } else if (FMT == QLIN_MXFP4) {  // one 32-element block per part, one UE8M0 scale
            const uint4 c = lds128(ub + (lane + 32 * i) * 16);
            const uint32_t cw[4] = {c.x, c.y, c.z, c.w};
            float2 s0[MP], s1[MP];
#pragma unroll
            for (int mm = 0; mm < MP; ++mm) s0[mm] = s1[mm] = make_float2(0.f, 0.f);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
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
            const float e = e8m0_to_f32(sc);
#pragma unroll
            for (int mm = 0; mm < MP; ++mm) {
                const float bsum = (s0[mm].x + s0[mm].y) + (s1[mm].x + s1[mm].y);
                res[i][mm] = ACC ? fmaf(e, bsum, res[i][mm]) : e * bsum;
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
