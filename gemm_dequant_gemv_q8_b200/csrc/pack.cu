// pack.cu -- canonical GGUF / NVFP4 / MXFP4 tensors -> the packed tile layout, and its inverse for tests.
//
// The repacker is the offline step that re-lays weights once per tensor (the pages' prior art:
// Imparo README intro, a "private GateUp layout" built from the canonical GGUF; imp README "Why
// this exists", an NVFP4 decode cache transformed at init).  It moves bytes only: no rounding.
#include "qlin_common.cuh"

namespace qlin {

// Source row of packed tile row r, or -1 for padding.
__device__ __forceinline__ int64_t source_row(int64_t t, int r, int64_t N, int gate_up) {
    if (gate_up) {
        int64_t half = N / 2;
        int64_t i = t * 16 + (r & 15);
        if (i >= half) return -1;
        return r < 16 ? i : half + i;
    }
    int64_t n = t * kTileRows + r;
    return n < N ? n : -1;
}

// One CTA per unit; thread (r, p) = (tid / 8, tid % 8) writes row r, part p.
template <int FMT>
__global__ void __launch_bounds__(256) pack_kernel(const uint8_t* __restrict__ blocks,
                                                   const uint8_t* __restrict__ scales, int64_t N,
                                                   int64_t K, int gate_up, uint8_t* __restrict__ packed,
                                                   int64_t G) {
    const int64_t unit = blockIdx.x;
    const int64_t t = unit / G, g = unit % G;
    const int r = threadIdx.x >> 3, p = threadIdx.x & 7;
    uint8_t* ub = packed + kHdrBytes + unit * (int64_t)unit_bytes(FMT);
    const int64_t n = source_row(t, r, N, gate_up);
    const int64_t k0 = g * kGroupK + p * 32;  // first element of this part
    const int lane = (r & 3) * 8 + p, slot = r >> 2;
    uint8_t* sc = ub + code_bytes(FMT) + (FMT == QLIN_MXFP4 ? lane * 8 + slot : lane * 16 + slot * 2);

    if (FMT == QLIN_Q4_0) {
        uint8_t out[16];
        uint16_t d = 0;
        if (n >= 0 && k0 < K) {
            const uint8_t* blk = blocks + n * (K / 32) * 18 + (k0 / 32) * 18;
            d = (uint16_t)(blk[0] | (blk[1] << 8));
            uint8_t e[32];
            for (int j = 0; j < 16; ++j) {
                e[j] = blk[2 + j] & 0xf;
                e[j + 16] = blk[2 + j] >> 4;
            }
            for (int j = 0; j < 16; ++j) out[j] = (uint8_t)(e[2 * j] | (e[2 * j + 1] << 4));
        } else {
            for (int j = 0; j < 16; ++j) out[j] = 0x88;  // code 8 -> value 0, with d = 0
        }
        uint4 v;
        memcpy(&v, out, 16);
        *reinterpret_cast<uint4*>(ub + (r * 8 + p) * 16) = v;
        sc[0] = (uint8_t)(d & 0xff);
        sc[1] = (uint8_t)(d >> 8);
    } else if (FMT == QLIN_Q8_0) {
        uint8_t out[32];
        uint16_t d = 0;
        if (n >= 0 && k0 < K) {
            const uint8_t* blk = blocks + n * (K / 32) * 34 + (k0 / 32) * 34;
            d = (uint16_t)(blk[0] | (blk[1] << 8));
            for (int j = 0; j < 32; ++j) out[j] = (uint8_t)(blk[2 + j] ^ 0x80u);  // q + 128
        } else {
            for (int j = 0; j < 32; ++j) out[j] = 0x80;  // q = 0
        }
        uint4 v0, v1;
        memcpy(&v0, out, 16);
        memcpy(&v1, out + 16, 16);
        *reinterpret_cast<uint4*>(ub + (r * 8 + p) * 16) = v0;
        *reinterpret_cast<uint4*>(ub + 4096 + (r * 8 + p) * 16) = v1;
        sc[0] = (uint8_t)(d & 0xff);
        sc[1] = (uint8_t)(d >> 8);
    } else if (FMT == QLIN_Q4_K) {
        // GGUF Q4_K super-block (144 B per 256 values = one k-group): fp16 d, fp16 dmin, 12 bytes
        // of packed 6-bit sub-block scales and mins, 128 bytes of codes (values 64c + l in the
        // low nibble of byte 32c + l, values 64c + 32 + l in its high nibble).  Part p is
        // sub-block p; its codes move to the 4-bit part order, its scale and min to the slot.
        uint8_t out[16];
        uint16_t scm = 0;
        uint32_t dm = 0;
        for (int j = 0; j < 16; ++j) out[j] = 0;
        if (n >= 0) {
            const uint8_t* blk = blocks + n * (K / 256) * 144 + g * 144;
            const uint8_t* s12 = blk + 4;
            const uint8_t* qs = blk + 16 + 32 * (p >> 1);
            for (int j = 0; j < 16; ++j) {
                const uint8_t lo = (p & 1) ? (qs[2 * j] >> 4) : (qs[2 * j] & 0xf);
                const uint8_t hi = (p & 1) ? (qs[2 * j + 1] >> 4) : (qs[2 * j + 1] & 0xf);
                out[j] = (uint8_t)(lo | (hi << 4));
            }
            int scv, mv;
            if (p < 4) {
                scv = s12[p] & 63;
                mv = s12[p + 4] & 63;
            } else {
                scv = (s12[p + 4] & 0xf) | ((s12[p - 4] >> 6) << 4);
                mv = (s12[p + 4] >> 4) | ((s12[p] >> 6) << 4);
            }
            scm = (uint16_t)(scv | (mv << 6));
            dm = (uint32_t)blk[0] | ((uint32_t)blk[1] << 8) | ((uint32_t)blk[2] << 16) | ((uint32_t)blk[3] << 24);
        }
        uint4 v;
        memcpy(&v, out, 16);
        *reinterpret_cast<uint4*>(ub + (r * 8 + p) * 16) = v;
        sc[0] = (uint8_t)(scm & 0xff);
        sc[1] = (uint8_t)(scm >> 8);
        if (p == 0) *reinterpret_cast<uint32_t*>(ub + row_d_off(FMT) + ((r & 3) * 8 + (r >> 2)) * 4) = dm;
    } else if (FMT == QLIN_Q6_K) {
        // GGUF Q6_K super-block (210 B per 256 values = one k-group): ql[128], qh[64], int8
        // scales[16], fp16 d.  Part p holds values 32p .. 32p+31 = half h = p / 4, quarter s = p % 4
        // of the super-block; each 6-bit code is assembled into a byte of the Q8_0 planes.
        uint8_t out[32];
        uint16_t scs = 0;
        uint32_t dm = 0;
        for (int j = 0; j < 32; ++j) out[j] = 32;  // padding: code 32 (value 0), scale 0
        if (n >= 0) {
            const uint8_t* blk = blocks + n * (K / 256) * 210 + g * 210;
            const int h = p >> 2, q = p & 3;
            const uint8_t* ql = blk + 64 * h + 32 * (q & 1);
            const uint8_t* qh = blk + 128 + 32 * h;
            for (int e = 0; e < 32; ++e) {
                const int lo = (q < 2) ? (ql[e] & 0xf) : (ql[e] >> 4);
                const int hi = (qh[e] >> (2 * q)) & 3;
                out[e] = (uint8_t)(lo | (hi << 4));
            }
            scs = (uint16_t)(blk[192 + 8 * h + 2 * q] | (blk[192 + 8 * h + 2 * q + 1] << 8));
            dm = (uint32_t)blk[208] | ((uint32_t)blk[209] << 8);
        }
        uint4 v0, v1;
        memcpy(&v0, out, 16);
        memcpy(&v1, out + 16, 16);
        *reinterpret_cast<uint4*>(ub + (r * 8 + p) * 16) = v0;
        *reinterpret_cast<uint4*>(ub + 4096 + (r * 8 + p) * 16) = v1;
        sc[0] = (uint8_t)(scs & 0xff);
        sc[1] = (uint8_t)(scs >> 8);
        if (p == 0) *reinterpret_cast<uint32_t*>(ub + row_d_off(FMT) + ((r & 3) * 8 + (r >> 2)) * 4) = dm;
    } else if (FMT == QLIN_MXFP4) {  // codes as NVFP4, one UE8M0 scale per part
        uint8_t out[16];
        uint8_t s = 0;
        for (int j = 0; j < 16; ++j) out[j] = 0;
        if (n >= 0 && k0 < K) {
            const uint8_t* row = blocks + n * (K / 2);
            for (int j = 0; j < 16; ++j) out[j] = row[k0 / 2 + j];
            s = scales[n * (K / 32) + k0 / 32];
        }
        uint4 v;
        memcpy(&v, out, 16);
        *reinterpret_cast<uint4*>(ub + (r * 8 + p) * 16) = v;
        sc[0] = s;
    } else {  // NVFP4: codes already two per byte in element order
        uint8_t out[16];
        uint8_t s0 = 0, s1 = 0;
        for (int j = 0; j < 16; ++j) out[j] = 0;
        if (n >= 0 && k0 < K) {
            const uint8_t* row = blocks + n * (K / 2);
            const uint8_t* srow = scales + n * (K / 16);
            const int64_t valid = (K - k0) >= 32 ? 32 : (K - k0);  // 16 or 32
            for (int j = 0; j < valid / 2; ++j) out[j] = row[k0 / 2 + j];
            s0 = srow[k0 / 16];
            if (valid == 32) s1 = srow[k0 / 16 + 1];
        }
        uint4 v;
        memcpy(&v, out, 16);
        *reinterpret_cast<uint4*>(ub + (r * 8 + p) * 16) = v;
        sc[0] = s0;
        sc[1] = s1;
    }
}

__global__ void write_header_kernel(uint8_t* packed, uint32_t fmt, int64_t N, int64_t K,
                                    uint32_t flags, float gs, int32_t T, int32_t G) {
    PackedHeader* h = reinterpret_cast<PackedHeader*>(packed);
    if (threadIdx.x == 0) {
        h->magic = kMagic;  // unit_bytes below is the GEMV unit; QLIN_PACK_MMA units are 36864 B
        h->fmt = fmt;
        h->N = N;
        h->K = K;
        h->flags = flags;
        h->global_scale = gs;
        h->T = T;
        h->G = G;
        h->unit_bytes = (uint32_t)unit_bytes((int)fmt);
    }
    if (threadIdx.x >= 1 && threadIdx.x < 54) h->reserved[threadIdx.x - 1] = 0;
}

// Inverse for tests: one CTA per unit, thread (r, p) writes the 32 fp32 weights of its part.
template <int FMT>
__global__ void __launch_bounds__(256) unpack_kernel(const uint8_t* __restrict__ packed, int64_t N,
                                                     int64_t K, int gate_up, int64_t G,
                                                     float* __restrict__ w) {
    const int64_t unit = blockIdx.x;
    const int64_t t = unit / G, g = unit % G;
    const int r = threadIdx.x >> 3, p = threadIdx.x & 7;
    const uint8_t* ub = packed + kHdrBytes + unit * (int64_t)unit_bytes(FMT);
    const int64_t n = source_row(t, r, N, gate_up);
    const int64_t k0 = g * kGroupK + p * 32;
    if (n < 0 || k0 >= K) return;
    const int lane = (r & 3) * 8 + p, slot = r >> 2;
    const uint8_t* sc = ub + code_bytes(FMT) + (FMT == QLIN_MXFP4 ? lane * 8 + slot : lane * 16 + slot * 2);
    const float gs = reinterpret_cast<const PackedHeader*>(packed)->global_scale;
    const int64_t valid = (K - k0) >= 32 ? 32 : (K - k0);
    float* out = w + n * K + k0;
    const uint8_t* cv = ub + (r * 8 + p) * 16;
    if (FMT == QLIN_Q4_0) {
        float d = fp16_bits_to_f32(sc[0] | (sc[1] << 8));
        for (int e = 0; e < 32; ++e) {
            int nib = (cv[e / 2] >> (4 * (e & 1))) & 0xf;
            out[e] = d * (float)(nib - 8);
        }
    } else if (FMT == QLIN_Q8_0) {
        float d = fp16_bits_to_f32(sc[0] | (sc[1] << 8));
        for (int e = 0; e < 32; ++e) {
            int b = (e < 16 ? cv[e] : cv[4096 + e - 16]);
            out[e] = d * (float)(b - 128);
        }
    } else if (FMT == QLIN_Q4_K) {
        // w = d * scale * code - dmin * min: both products exact in fp32, one rounding
        const uint32_t dm = *reinterpret_cast<const uint32_t*>(ub + row_d_off(FMT) + ((r & 3) * 8 + (r >> 2)) * 4);
        const int scm = sc[0] | (sc[1] << 8);
        const float a = fp16_bits_to_f32(dm & 0xffffu) * (float)(scm & 63);
        const float b = fp16_bits_to_f32(dm >> 16) * (float)((scm >> 6) & 63);
        for (int e = 0; e < 32; ++e) {
            const int nib = (cv[e / 2] >> (4 * (e & 1))) & 0xf;
            out[e] = __fmaf_rn(a, (float)nib, -b);
        }
    } else if (FMT == QLIN_Q6_K) {
        // w = d * scale * (code - 32): d * scale and the product are exact in fp32 (<= 23 bits)
        const uint32_t dm = *reinterpret_cast<const uint32_t*>(ub + row_d_off(FMT) + ((r & 3) * 8 + (r >> 2)) * 4);
        const float d = fp16_bits_to_f32(dm & 0xffffu);
        const float e0 = d * (float)(int8_t)sc[0], e1 = d * (float)(int8_t)sc[1];
        for (int e = 0; e < 32; ++e) {
            const int b = e < 16 ? cv[e] : cv[4096 + e - 16];
            out[e] = __fmul_rn(e < 16 ? e0 : e1, (float)(b - 32));
        }
    } else if (FMT == QLIN_MXFP4) {
        const float s = e8m0_to_f32(sc[0]);
        for (int e = 0; e < valid; ++e) {
            uint32_t h2 = e2m1x2_to_f16x2(cv[e / 2]);
            float v = __half2float(__ushort_as_half((unsigned short)((e & 1) ? (h2 >> 16) : (h2 & 0xffff))));
            out[e] = __fmul_rn(v, s);  // a power of two times an E2M1 value: exact unless it overflows
        }
    } else {
        for (int e = 0; e < valid; ++e) {
            uint32_t h2 = e2m1x2_to_f16x2(cv[e / 2]);
            float v = __half2float(__ushort_as_half((unsigned short)((e & 1) ? (h2 >> 16) : (h2 & 0xffff))));
            float s = e4m3_to_f32(sc[e / 16]);
            out[e] = __fmul_rn(__fmul_rn(v, s), gs);  // v*s is exact; the tensor scale rounds once
        }
    }
}

// QLIN_PACK_MMA for the formats other than NVFP4, and QLIN_PACK_MMA_BF16: the dequantized weights
// as bf16 rows of Kc values (K rounded up to 64, the tail zero), each the fp32 value
// qlin_dequant_debug gives rounded to nearest-even bf16 -- the operand of the bf16 prefill-chunk
// GEMM.  NVFP4: e2m1 * e4m3 without the per-tensor scale (exact in bf16; the GEMM applies the scale
// from the header).  Thread = (row, 32 values).
template <int FMT>
__global__ void __launch_bounds__(256) pack_bf16_kernel(const uint8_t* __restrict__ blocks,
                                                        const uint8_t* __restrict__ scales, int64_t N, int64_t K,
                                                        int64_t Kc, __nv_bfloat16* __restrict__ out) {
    const int64_t nb = Kc / 32, Np = (N + 255) / 256 * 256;
    const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= Np * nb) return;
    const int64_t n = idx / nb, b = idx - n * nb, k0 = b * 32;
    float w[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) w[j] = 0.f;
    if (n < N && k0 < K) {
        if (FMT == QLIN_Q8_0 || FMT == QLIN_Q4_0) {
            const int bsz = FMT == QLIN_Q8_0 ? 34 : 18;
            const uint8_t* blk = blocks + n * (K / 32) * bsz + b * bsz;
            const float d = fp16_bits_to_f32(blk[0] | (blk[1] << 8));
            for (int j = 0; j < 32; ++j) {
                const int q = FMT == QLIN_Q8_0 ? (int)(int8_t)blk[2 + j]
                                               : (j < 16 ? (blk[2 + j] & 0xf) : (blk[2 + j - 16] >> 4)) - 8;
                w[j] = d * (float)q;  // exact
            }
        } else if (FMT == QLIN_NVFP4) {  // K % 16 == 0: the last 32-value part may be half valid
            const uint8_t* row = blocks + n * (K / 2) + k0 / 2;
            for (int j = 0; j < 32 && k0 + j < K; ++j) {
                const uint32_t h2 = e2m1x2_to_f16x2(row[j / 2]);
                const float v = __half2float(__ushort_as_half((unsigned short)((j & 1) ? (h2 >> 16) : (h2 & 0xffff))));
                w[j] = __fmul_rn(v, e4m3_to_f32(scales[n * (K / 16) + (k0 + j) / 16]));  // exact
            }
        } else if (FMT == QLIN_MXFP4) {
            const uint8_t* row = blocks + n * (K / 2) + k0 / 2;
            const float sc = e8m0_to_f32(scales[n * (K / 32) + b]);
            for (int j = 0; j < 32; ++j) {
                const uint32_t h2 = e2m1x2_to_f16x2(row[j / 2]);
                const float v = __half2float(__ushort_as_half((unsigned short)((j & 1) ? (h2 >> 16) : (h2 & 0xffff))));
                w[j] = __fmul_rn(v, sc);  // exact unless it overflows
            }
        } else if (FMT == QLIN_Q4_K) {
            const uint8_t* blk = blocks + n * (K / 256) * 144 + (k0 / 256) * 144;
            const int p = (int)((k0 % 256) / 32);
            const uint8_t* s12 = blk + 4;
            const int scv = p < 4 ? (s12[p] & 63) : ((s12[p + 4] & 0xf) | ((s12[p - 4] >> 6) << 4));
            const int mv = p < 4 ? (s12[p + 4] & 63) : ((s12[p + 4] >> 4) | ((s12[p] >> 6) << 4));
            const float ka = fp16_bits_to_f32(blk[0] | (blk[1] << 8)) * (float)scv;  // exact
            const float kb = fp16_bits_to_f32(blk[2] | (blk[3] << 8)) * (float)mv;   // exact
            const uint8_t* qs = blk + 16 + 32 * (p >> 1);
            for (int j = 0; j < 32; ++j) {
                const int code = (p & 1) ? (qs[j] >> 4) : (qs[j] & 0xf);
                w[j] = __fmaf_rn(ka, (float)code, -kb);  // one rounding
            }
        } else if (FMT == QLIN_Q6_K) {
            const uint8_t* blk = blocks + n * (K / 256) * 210 + (k0 / 256) * 210;
            const int p = (int)((k0 % 256) / 32), h = p >> 2, q = p & 3;
            const uint8_t* ql = blk + 64 * h + 32 * (q & 1);
            const uint8_t* qh = blk + 128 + 32 * h;
            const float d = fp16_bits_to_f32(blk[208] | (blk[209] << 8));
            const float e0 = d * (float)(int8_t)blk[192 + 8 * h + 2 * q], e1 = d * (float)(int8_t)blk[192 + 8 * h + 2 * q + 1];
            for (int j = 0; j < 32; ++j) {
                const int code = ((q < 2) ? (ql[j] & 0xf) : (ql[j] >> 4)) | (((qh[j] >> (2 * q)) & 3) << 4);
                w[j] = __fmul_rn(j < 16 ? e0 : e1, (float)(code - 32));  // exact
            }
        }
    }
    uint32_t pk[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) {
        const __nv_bfloat162 h = __floats2bfloat162_rn(w[2 * j], w[2 * j + 1]);
        pk[j] = *reinterpret_cast<const uint32_t*>(&h);
    }
    // blocked: 256 rows x 64 values per (row block, k-block), 32 KB contiguous
    const int64_t blk = (n / 256) * (Kc / 64) + k0 / 64;
    uint4* dst = reinterpret_cast<uint4*>(out + (blk * 256 + n % 256) * 64 + k0 % 64);
#pragma unroll
    for (int v = 0; v < 4; ++v) dst[v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
}

}  // namespace qlin

using namespace qlin;

extern "C" int64_t qlin_bf16_cache_cols(int64_t K);

extern "C" cudaError_t qlin_launch_pack_mma(int fmt, const void* codes, const void* scales, int64_t N, int64_t K,
                                            int gate_up, void* packed, cudaStream_t s);

extern "C" cudaError_t qlin_launch_pack(int fmt, const void* blocks, const void* scales, int64_t N,
                                        int64_t K, int pack_flags, float gs, void* packed,
                                        cudaStream_t s) {
    if ((pack_flags & ~QLIN_PACK_GATE_UP) == QLIN_PACK_MMA && (fmt == QLIN_NVFP4 || fmt == QLIN_MXFP4)) {
        const int gu = (pack_flags & QLIN_PACK_GATE_UP) ? 1 : 0;
        write_header_kernel<<<1, 64, 0, s>>>((uint8_t*)packed, (uint32_t)fmt, N, K, (uint32_t)pack_flags, gs,
                                             (int32_t)(gu ? (N / 2 + 127) / 128 : (N + 255) / 256),
                                             (int32_t)((K + 255) / 256));
        return qlin_launch_pack_mma(fmt, blocks, scales, N, K, gu, packed, s);
    }
    if (pack_flags == QLIN_PACK_MMA || pack_flags == QLIN_PACK_MMA_BF16) {
        write_header_kernel<<<1, 64, 0, s>>>((uint8_t*)packed, (uint32_t)fmt, N, K, (uint32_t)pack_flags, gs,
                                             (int32_t)((N + 255) / 256), (int32_t)((K + 255) / 256));
        const int64_t Kc = qlin_bf16_cache_cols(K);
        const int64_t threads = (N + 255) / 256 * 256 * (Kc / 32);
        const dim3 grid((unsigned)((threads + 255) / 256));
        const uint8_t* bl = (const uint8_t*)blocks;
        const uint8_t* sc = (const uint8_t*)scales;
        __nv_bfloat16* out = (__nv_bfloat16*)((uint8_t*)packed + kHdrBytes);
        if (fmt == QLIN_Q8_0) pack_bf16_kernel<QLIN_Q8_0><<<grid, 256, 0, s>>>(bl, sc, N, K, Kc, out);
        else if (fmt == QLIN_Q4_0) pack_bf16_kernel<QLIN_Q4_0><<<grid, 256, 0, s>>>(bl, sc, N, K, Kc, out);
        else if (fmt == QLIN_MXFP4) pack_bf16_kernel<QLIN_MXFP4><<<grid, 256, 0, s>>>(bl, sc, N, K, Kc, out);
        else if (fmt == QLIN_Q4_K) pack_bf16_kernel<QLIN_Q4_K><<<grid, 256, 0, s>>>(bl, sc, N, K, Kc, out);
        else if (fmt == QLIN_Q6_K) pack_bf16_kernel<QLIN_Q6_K><<<grid, 256, 0, s>>>(bl, sc, N, K, Kc, out);
        else pack_bf16_kernel<QLIN_NVFP4><<<grid, 256, 0, s>>>(bl, sc, N, K, Kc, out);
        return cudaGetLastError();
    }
    Geometry geo = geometry(fmt, N, K, pack_flags);
    const int gu = (pack_flags & QLIN_PACK_GATE_UP) ? 1 : 0;
    write_header_kernel<<<1, 64, 0, s>>>((uint8_t*)packed, (uint32_t)fmt, N, K, (uint32_t)pack_flags,
                                         gs, (int32_t)geo.T, (int32_t)geo.G);
    dim3 grid((unsigned)geo.U);
    if (fmt == QLIN_Q4_0)
        pack_kernel<QLIN_Q4_0><<<grid, 256, 0, s>>>((const uint8_t*)blocks, nullptr, N, K, gu,
                                                     (uint8_t*)packed, geo.G);
    else if (fmt == QLIN_Q8_0)
        pack_kernel<QLIN_Q8_0><<<grid, 256, 0, s>>>((const uint8_t*)blocks, nullptr, N, K, gu,
                                                     (uint8_t*)packed, geo.G);
    else if (fmt == QLIN_MXFP4)
        pack_kernel<QLIN_MXFP4><<<grid, 256, 0, s>>>((const uint8_t*)blocks, (const uint8_t*)scales,
                                                      N, K, gu, (uint8_t*)packed, geo.G);
    else if (fmt == QLIN_Q4_K)
        pack_kernel<QLIN_Q4_K><<<grid, 256, 0, s>>>((const uint8_t*)blocks, nullptr, N, K, gu,
                                                     (uint8_t*)packed, geo.G);
    else if (fmt == QLIN_Q6_K)
        pack_kernel<QLIN_Q6_K><<<grid, 256, 0, s>>>((const uint8_t*)blocks, nullptr, N, K, gu,
                                                     (uint8_t*)packed, geo.G);
    else
        pack_kernel<QLIN_NVFP4><<<grid, 256, 0, s>>>((const uint8_t*)blocks, (const uint8_t*)scales,
                                                      N, K, gu, (uint8_t*)packed, geo.G);
    return cudaGetLastError();
}

extern "C" cudaError_t qlin_launch_unpack(int fmt, const void* packed, int64_t N, int64_t K,
                                          int pack_flags, float* w, cudaStream_t s) {
    Geometry geo = geometry(fmt, N, K, pack_flags);
    const int gu = (pack_flags & QLIN_PACK_GATE_UP) ? 1 : 0;
    dim3 grid((unsigned)geo.U);
    if (fmt == QLIN_Q4_0)
        unpack_kernel<QLIN_Q4_0><<<grid, 256, 0, s>>>((const uint8_t*)packed, N, K, gu, geo.G, w);
    else if (fmt == QLIN_Q8_0)
        unpack_kernel<QLIN_Q8_0><<<grid, 256, 0, s>>>((const uint8_t*)packed, N, K, gu, geo.G, w);
    else if (fmt == QLIN_MXFP4)
        unpack_kernel<QLIN_MXFP4><<<grid, 256, 0, s>>>((const uint8_t*)packed, N, K, gu, geo.G, w);
    else if (fmt == QLIN_Q4_K)
        unpack_kernel<QLIN_Q4_K><<<grid, 256, 0, s>>>((const uint8_t*)packed, N, K, gu, geo.G, w);
    else if (fmt == QLIN_Q6_K)
        unpack_kernel<QLIN_Q6_K><<<grid, 256, 0, s>>>((const uint8_t*)packed, N, K, gu, geo.G, w);
    else
        unpack_kernel<QLIN_NVFP4><<<grid, 256, 0, s>>>((const uint8_t*)packed, N, K, gu, geo.G, w);
    return cudaGetLastError();
}
