// chunk_common.cuh -- operand layouts of the NVFP4 / MXFP4 prefill-chunk GEMM (tcgen05 block-scaled
// MMA).
//
// Both operands are stored in global memory exactly as the tensor core reads them from shared
// memory, so each pipeline stage is filled by plain bulk copies:
//   codes : rows of 128 bytes (256 E2M1 values of one k-group), 16-byte chunk c of row r stored at
//           chunk position c ^ (r % 8) -- the 128-byte-swizzled K-major canonical layout; 8-row
//           groups are 1024 bytes apart.
//   scales: per 128 rows and per 4 scale blocks along k, a 512-byte atom; the scale of row r
//           (0..127) and block j (0..3) is at byte (r % 32) * 16 + (r / 32) * 4 + j, the layout the
//           32x128b scale-factor copy into tensor memory expects.  NVFP4: E4M3 scales of 16 values,
//           an atom per 64-value k-block (4 per k-group); MXFP4: UE8M0 scales of 32 values, an atom
//           per 128-value span (2 per k-group; the two MMAs of a span take bytes 0-1 and 2-3).
// Weights (QLIN_PACK_MMA): units of 256 rows x 256 values = 32768 B codes + 8 atoms (4 k-blocks x
// 2 row halves) = 36864 B, in [row tile][k-group] order after the 256-byte header (MXFP4: 4 atoms,
// the unit keeps the NVFP4 size).
// Activations (quantized by the chunk path): units of 128 rows x 256 values = 16384 B codes +
// 4 atoms = 18432 B (MXFP4: 2 atoms), in [row tile][k-group] order.
#pragma once
#include "qlin_common.cuh"

namespace qlin {

constexpr int kMmaWRows = 256;   // weight rows per tile (the MMA N dimension)
constexpr int kMmaARows = 128;   // activation rows per tile (the MMA M dimension)
constexpr int kMmaWUnit = 256 * 128 + 8 * 512;  // 36864
constexpr int kMmaAUnit = 128 * 128 + 4 * 512;  // 18432

__host__ __device__ inline int64_t mma_code_off(int r, int chunk) {
    return (int64_t)r * 128 + ((chunk ^ (r & 7)) << 4);
}
// scale atom byte offset inside a unit's scale region: kb = 64-value block, r = row in the tile
__host__ __device__ inline int64_t mma_scale_off(int kb, int r, int j, int halves) {
    const int h = r >> 7, rr = r & 127;
    return (int64_t)(kb * halves + h) * 512 + (rr & 31) * 16 + (rr >> 5) * 4 + j;
}

// ------------------------------------------------------------------ activation quantization
// The rule (every step in fp32 with IEEE round-to-nearest-even):
//   a_g  = amax|X| / (6 * 448)                       per tensor
//   s_b  = E4M3_rne_satfinite( amax_b / (6 * a_g) )  per 16 consecutive values of a row
//   code = E2M1_rne_satfinite( x / (e4m3(s_b) * a_g) ), 0 where that divisor is 0
__device__ __forceinline__ float act_global_scale(float amax) { return __fdiv_rn(amax, __fmul_rn(6.0f, 448.0f)); }

__device__ __forceinline__ uint8_t e4m3_rne_sat(float v) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(v));
    return (uint8_t)(r & 0xffu);
}

// two E2M1 codes: low nibble from lo, high nibble from hi
__device__ __forceinline__ uint32_t e2m1x2_rne_sat(float lo, float hi) {
    uint32_t r;
    asm("{\n .reg .b8 t;\n cvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n cvt.u32.u8 %0, t;\n}\n" : "=r"(r) : "f"(hi), "f"(lo));
    return r & 0xffu;
}

// Max |x| over the M x K bf16 activations, one partial per thread (fmaxf: a NaN input is skipped).
// `vec`: x is 16-byte aligned and ldx % 8 == 0 (8 values per load).
__device__ __forceinline__ float act_amax_partial(const __nv_bfloat16* __restrict__ x, int M, int64_t K, int64_t ldx,
                                                  bool vec, int64_t tid, int64_t nthreads) {
    float m = 0.f;
    if (vec) {
        const int64_t per_row = K / 8;
        const int64_t total = (int64_t)M * per_row;
        for (int64_t i = tid; i < total; i += nthreads) {
            const int64_t r = i / per_row, c = i - r * per_row;
            const uint4 v = __ldg(reinterpret_cast<const uint4*>(x + r * ldx) + c);
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                m = fmaxf(m, fabsf(__uint_as_float(w[j] << 16)));
                m = fmaxf(m, fabsf(__uint_as_float(w[j] & 0xffff0000u)));
            }
        }
    } else {
        const int64_t total = (int64_t)M * K;
        for (int64_t i = tid; i < total; i += nthreads) {
            const int64_t r = i / K, c = i - r * K;
            m = fmaxf(m, fabsf(__bfloat162float(x[r * ldx + c])));
        }
    }
    return m;
}

// The 16 bf16 values of item (row m, 16-value block b) as 8 words (value 2j in the low half of
// word j); zeros outside the M x K activations.
__device__ __forceinline__ void act_load_item(const __nv_bfloat16* __restrict__ x, int M, int64_t K, int64_t ldx,
                                              bool vec, int m, int64_t b, uint32_t (&w)[8]) {
    const int64_t k = b * 16;
#pragma unroll
    for (int j = 0; j < 8; ++j) w[j] = 0u;
    if (m >= M || k >= K) return;
    const __nv_bfloat16* xr = x + (int64_t)m * ldx + k;
    if (vec) {
        const uint4 a0 = __ldg(reinterpret_cast<const uint4*>(xr));
        const uint4 a1 = __ldg(reinterpret_cast<const uint4*>(xr) + 1);
        w[0] = a0.x, w[1] = a0.y, w[2] = a0.z, w[3] = a0.w, w[4] = a1.x, w[5] = a1.y, w[6] = a1.z, w[7] = a1.w;
    } else {
        const unsigned short* xs = reinterpret_cast<const unsigned short*>(xr);
#pragma unroll
        for (int j = 0; j < 8; ++j) w[j] = (uint32_t)xs[2 * j] | ((uint32_t)xs[2 * j + 1] << 16);
    }
}

__device__ __forceinline__ float act_item_amax(const uint32_t (&w)[8]) {
    float bmax = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        bmax = fmaxf(bmax, fabsf(__uint_as_float(w[j] << 16)));
        bmax = fmaxf(bmax, fabsf(__uint_as_float(w[j] & 0xffff0000u)));
    }
    return bmax;
}

// x / d rounded to nearest even, for d in [2^-96, 2^100] and finite x: the correctly rounded
// reciprocal and two FMA-based remainder corrections (Markstein, "Computation of elementary
// functions on the IBM RISC System/6000 processor", IBM J. Res. Dev. 34(1), 1990); the sign is
// taken from x so that -0 stays -0.  Over every finite bf16 x and every divisor the quantizer can
// form (E4M3 scale times a_g) this equals __fdiv_rn bit for bit wherever the quotient can reach a
// nonzero E2M1 code, and gives a signed code 0 elsewhere (checked exhaustively on the host; a
// sampled check is part of the CPU tests).
__device__ __forceinline__ float div_by_recip(float x, float d, float y) {
    const float q0 = __fmul_rn(x, y);
    const float r0 = __fmaf_rn(-q0, d, x);
    const float q1 = __fmaf_rn(r0, y, q0);
    const float r1 = __fmaf_rn(-q1, d, x);
    return copysignf(__fmaf_rn(r1, y, q1), x);
}

// Two quotients at once: the same steps on a pair of values with the packed fp32 operations, each
// lane rounded as the scalar operation rounds it (so the results are div_by_recip's, bit for bit);
// -q * d + x is taken as fma(q, -d, x), the same value.
__device__ __forceinline__ float2 div_by_recip2(float2 x, float d, float y) {
    const float2 yy = make_float2(y, y), nd = make_float2(-d, -d);
    const float2 q0 = __fmul2_rn(x, yy);
    const float2 r0 = __ffma2_rn(q0, nd, x);
    const float2 q1 = __ffma2_rn(r0, yy, q0);
    const float2 r1 = __ffma2_rn(q1, nd, x);
    const float2 q = __ffma2_rn(r1, yy, q1);
    return make_float2(copysignf(q.x, x.x), copysignf(q.y, x.y));
}

// Scale byte and 8 code bytes (element 2j in the low nibble of byte j) of one 16-value block.
__device__ __forceinline__ uint8_t act_quant_block(const uint32_t (&w)[8], float bmax, float ag, uint32_t (&c8)[2]) {
    c8[0] = c8[1] = 0u;
    uint8_t s = 0;
    if (ag > 0.f) s = e4m3_rne_sat(__fdiv_rn(bmax, __fmul_rn(6.0f, ag)));
    const float div = __fmul_rn(e4m3_to_f32(s), ag);
    if (div > 0.f) {
        uint32_t special = 0u;  // any Inf or NaN among the 16 values
#pragma unroll
        for (int j = 0; j < 8; ++j)
            special |= (uint32_t)((w[j] & 0x7f80u) == 0x7f80u) | (uint32_t)((w[j] & 0x7f800000u) == 0x7f800000u);
        if (special == 0u && div >= 0x1p-96f && div <= 0x1p100f) {
            const float y = __frcp_rn(div);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const float2 qv =
                    div_by_recip2(make_float2(__uint_as_float(w[j] << 16), __uint_as_float(w[j] & 0xffff0000u)), div, y);
                c8[j >> 2] |= e2m1x2_rne_sat(qv.x, qv.y) << (8 * (j & 3));
            }
        } else {
#pragma unroll
            for (int j = 0; j < 8; ++j)
                c8[j >> 2] |= e2m1x2_rne_sat(__fdiv_rn(__uint_as_float(w[j] << 16), div),
                                             __fdiv_rn(__uint_as_float(w[j] & 0xffff0000u), div))
                              << (8 * (j & 3));
        }
    }
    return s;
}

// Store item (m, b) of the padded operand (TM*128 rows x G*16 blocks) in the MMA unit layout and,
// optionally, in the canonical layout (codes [M][K/2], scales [M][K/16]).
__device__ __forceinline__ void act_store_item(int M, int64_t K, int64_t G, int m, int64_t b, uint8_t s,
                                               const uint32_t (&c8)[2], uint8_t* __restrict__ aq,
                                               uint8_t* __restrict__ canon_codes, uint8_t* __restrict__ canon_scales) {
    const int64_t k = b * 16;
    const int tm = m / kMmaARows, r = m % kMmaARows;
    const int64_t g = k / kGroupK;
    const int kin = (int)(k % kGroupK);
    uint8_t* ub = aq + ((int64_t)tm * G + g) * kMmaAUnit;
    const int chunk = kin / 32, within = (kin % 32) / 2;  // 8 code bytes at byte 0 or 8 of the chunk
    *reinterpret_cast<uint2*>(ub + mma_code_off(r, chunk) + within) = make_uint2(c8[0], c8[1]);
    ub[kMmaARows * 128 + mma_scale_off(kin / 64, r, (kin % 64) / 16, 1)] = s;
    if (canon_codes && m < M && k < K) {
        memcpy(canon_codes + (int64_t)m * (K / 2) + k / 2, c8, 8);
        canon_scales[(int64_t)m * (K / 16) + k / 16] = s;
    }
}

// Load, quantize and store item (m, b); rows >= M and values >= K are written as zeros.
__device__ __forceinline__ void act_quant_item(const __nv_bfloat16* __restrict__ x, int M, int64_t K, int64_t ldx,
                                               int64_t G, float ag, bool vec, int m, int64_t b,
                                               uint8_t* __restrict__ aq, uint8_t* __restrict__ canon_codes,
                                               uint8_t* __restrict__ canon_scales) {
    uint32_t w[8], c8[2];
    act_load_item(x, M, K, ldx, vec, m, b, w);
    const uint8_t s = act_quant_block(w, act_item_amax(w), ag, c8);
    act_store_item(M, K, G, m, b, s, c8, aq, canon_codes, canon_scales);
}

// ------------------------------------------------------------------ MXFP4 activation quantization
// The OCP MX conversion, per 32 consecutive values of a row: scale byte = floor(log2 amax) - 2 + 127
// clamped to [0, 254] (0xFF when the block holds an Inf or NaN), X = 2^(byte - 127), code =
// E2M1_rne_satfinite(x / X), the division exact (a power of two).  A 32-value block is two 16-value
// items, 2c and 2c + 1, which the quantizers place in adjacent lanes: one shuffle gives each the
// block's amax.  For a normal amax with biased exponent be, floor(log2 amax) = be - 127, so the
// byte is be - 2; amax below 2^-125 (be < 2, zero and subnormals included) clamps to 0.
__device__ __forceinline__ uint8_t mx_scale_byte(float amax, bool special) {
    if (special) return 0xFF;
    const uint32_t be = (__float_as_uint(amax) >> 23) & 0xffu;
    return (uint8_t)(be >= 2u ? be - 2u : 0u);
}

__device__ __forceinline__ bool act_item_special(const uint32_t (&w)[8]) {
    uint32_t sp = 0u;
#pragma unroll
    for (int j = 0; j < 8; ++j) sp |= (uint32_t)((w[j] & 0x7f80u) == 0x7f80u) | (uint32_t)((w[j] & 0x7f800000u) == 0x7f800000u);
    return sp != 0u;
}

// Codes of one 16-value item under the scale byte of its 32-value block.
__device__ __forceinline__ void act_quant_item_mx_codes(const uint32_t (&w)[8], uint8_t byte, uint32_t (&c8)[2]) {
    c8[0] = c8[1] = 0u;
    if (byte == 0xFF) return;
    const float inv = __uint_as_float((254u - byte) << 23);  // 2^(127 - byte), a normal number
#pragma unroll
    for (int j = 0; j < 8; ++j)
        c8[j >> 2] |= e2m1x2_rne_sat(__fmul_rn(__uint_as_float(w[j] << 16), inv),
                                     __fmul_rn(__uint_as_float(w[j] & 0xffff0000u), inv))
                      << (8 * (j & 3));
}

// Block scale byte of the 32-value block of an item whose partner item sits in lane ^ 1 (every
// lane of the warp calls this).
__device__ __forceinline__ uint8_t act_mx_pair_byte(float bmax, bool special) {
    const float pm = __shfl_xor_sync(0xffffffffu, bmax, 1);
    const int ps = __shfl_xor_sync(0xffffffffu, special ? 1 : 0, 1);
    return mx_scale_byte(fmaxf(bmax, pm), special || ps != 0);
}

// Store item (m, b) of the padded MXFP4 operand: codes as act_store_item; the block's scale byte
// is written by the even item of the pair (atom layout: 4 scales of 32 values per 128-value span).
__device__ __forceinline__ void act_store_item_mx(int M, int64_t K, int64_t G, int m, int64_t b, uint8_t byte,
                                                  const uint32_t (&c8)[2], uint8_t* __restrict__ aq,
                                                  uint8_t* __restrict__ canon_codes,
                                                  uint8_t* __restrict__ canon_scales) {
    const int64_t k = b * 16;
    const int tm = m / kMmaARows, r = m % kMmaARows;
    const int64_t g = k / kGroupK;
    const int kin = (int)(k % kGroupK);
    uint8_t* ub = aq + ((int64_t)tm * G + g) * kMmaAUnit;
    const int chunk = kin / 32, within = (kin % 32) / 2;
    *reinterpret_cast<uint2*>(ub + mma_code_off(r, chunk) + within) = make_uint2(c8[0], c8[1]);
    if ((b & 1) == 0) ub[kMmaARows * 128 + mma_scale_off(kin / 128, r, (kin % 128) / 32, 1)] = byte;
    if (canon_codes && m < M && k < K) {
        memcpy(canon_codes + (int64_t)m * (K / 2) + k / 2, c8, 8);
        if ((b & 1) == 0) canon_scales[(int64_t)m * (K / 32) + k / 32] = byte;
    }
}

}  // namespace qlin
