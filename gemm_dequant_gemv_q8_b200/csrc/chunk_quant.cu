// chunk_quant.cu -- the chunk path's operand preparation (sm_100a):
//   * QLIN_PACK_MMA weight packing: canonical NVFP4 -> the tensor-core operand layout;
//   * NVFP4 quantization of bf16 activations (the A operand).
//
// Activation quantization rule (the pages name NVFP4 activations only through the block-scaled
// "mxf4nvf4" MMA -- imp README, "Features", row "sm_120a kernels"; the rule is the adopted reading,
// every step in fp32 with IEEE round-to-nearest-even):
//   a_g  = amax|X| / (6 * 448)                       per tensor
//   s_b  = E4M3_rne_satfinite( amax_b / (6 * a_g) )  per 16 consecutive values of a row
//   code = E2M1_rne_satfinite( x / (e4m3(s_b) * a_g) ), 0 where that divisor is 0
#include "chunk_common.cuh"

namespace qlin {

// ------------------------------------------------------------------ weight packing
// One CTA per unit (256-row tile, k-group); thread r writes row r.
__global__ void __launch_bounds__(256) pack_mma_kernel(const uint8_t* __restrict__ codes,
                                                       const uint8_t* __restrict__ scales, int64_t N,
                                                       int64_t K, int64_t G, uint8_t* __restrict__ packed) {
    const int64_t unit = blockIdx.x;
    const int64_t t = unit / G, g = unit % G;
    const int r = threadIdx.x;
    const int64_t n = t * kMmaWRows + r;
    uint8_t* ub = packed + kHdrBytes + unit * (int64_t)kMmaWUnit;
    const int64_t k0 = g * kGroupK;
#pragma unroll 1
    for (int c = 0; c < 8; ++c) {  // 16-byte chunk c holds values k0 + 32c .. +31
        uint8_t buf[16];
        for (int j = 0; j < 16; ++j) buf[j] = 0;
        const int64_t kc = k0 + 32 * c;
        if (n < N && kc < K) {
            const int64_t valid = (K - kc) >= 32 ? 16 : (K - kc) / 2;
            for (int j = 0; j < valid; ++j) buf[j] = codes[n * (K / 2) + kc / 2 + j];
        }
        uint4 v;
        memcpy(&v, buf, 16);
        *reinterpret_cast<uint4*>(ub + mma_code_off(r, c)) = v;
    }
    uint8_t* sc = ub + kMmaWRows * 128;
    for (int b = 0; b < 16; ++b) {  // 16-value block b of the k-group
        const int64_t kb16 = k0 + 16 * b;
        const uint8_t s = (n < N && kb16 < K) ? scales[n * (K / 16) + kb16 / 16] : 0;
        sc[mma_scale_off(b >> 2, r, b & 3, 2)] = s;
    }
}

// ------------------------------------------------------------------ activation quantization
// Block-wide max of |x| folded into one word with atomicMax (order-independent, deterministic);
// the last block to finish turns it into a_g and clears the accumulator for the next call.
__global__ void __launch_bounds__(256) act_amax_kernel(const __nv_bfloat16* __restrict__ x, int M, int64_t K,
                                                       int64_t ldx, unsigned* __restrict__ words) {
    // words[0] = amax bits (accumulating), words[1] = ticket, words[2] = a_g (float bits, output)
    griddep_wait();
    float m = 0.f;
    const int64_t total = (int64_t)M * K;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t r = i / K, c = i - r * K;
        m = fmaxf(m, fabsf(__bfloat162float(x[r * ldx + c])));
    }
    for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    __shared__ float wmax[8];
    if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
        float b = 0.f;
        for (int w = 0; w < (int)(blockDim.x >> 5); ++w) b = fmaxf(b, wmax[w]);
        atomicMax(&words[0], __float_as_uint(b));  // non-negative floats order as their bits
        __threadfence();
        const unsigned ticket = atomicAdd(&words[1], 1u);
        if (ticket == gridDim.x - 1) {
            __threadfence();
            const float amax = __uint_as_float(atomicAdd(&words[0], 0u));
            const float ag = __fdiv_rn(amax, __fmul_rn(6.0f, 448.0f));
            words[2] = __float_as_uint(ag);
            words[0] = 0u;
            words[1] = 0u;
        }
    }
}

__device__ __forceinline__ uint8_t e4m3_rne_sat(float v) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(v));
    return (uint8_t)(r & 0xffu);
}

// two E2M1 codes: low nibble from lo, high nibble from hi
__device__ __forceinline__ uint8_t e2m1x2_rne_sat(float lo, float hi) {
    uint32_t r;
    asm("{\n .reg .b8 t;\n cvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n cvt.u32.u8 %0, t;\n}\n" : "=r"(r) : "f"(hi), "f"(lo));
    return (uint8_t)(r & 0xffu);
}

// One thread per (row, 16-value block) of the padded operand.  Writes the MMA layout and,
// optionally, the canonical layout (codes [M][K/2], scales [M][K/16]) for inspection.
__global__ void __launch_bounds__(256) act_quant_kernel(const __nv_bfloat16* __restrict__ x, int M, int64_t K,
                                                        int64_t ldx, int64_t G, int TM, const unsigned* __restrict__ words,
                                                        uint8_t* __restrict__ aq, uint8_t* __restrict__ canon_codes,
                                                        uint8_t* __restrict__ canon_scales) {
    griddep_wait();
    const int64_t nblk16 = G * 16;  // 16-value blocks per padded row
    const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= (int64_t)TM * kMmaARows * nblk16) return;
    const int m = (int)(idx / nblk16);
    const int64_t b = idx - (int64_t)m * nblk16;
    const int64_t k = b * 16;
    const float ag = __uint_as_float(words[2]);
    uint8_t codes[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    uint8_t s = 0;
    if (m < M && k < K) {
        float v[16];
        float bmax = 0.f;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            v[j] = __bfloat162float(x[(int64_t)m * ldx + k + j]);
            bmax = fmaxf(bmax, fabsf(v[j]));
        }
        if (ag > 0.f) s = e4m3_rne_sat(__fdiv_rn(bmax, __fmul_rn(6.0f, ag)));
        const float div = __fmul_rn(e4m3_to_f32(s), ag);
        if (div > 0.f) {
#pragma unroll
            for (int j = 0; j < 8; ++j) codes[j] = e2m1x2_rne_sat(__fdiv_rn(v[2 * j], div), __fdiv_rn(v[2 * j + 1], div));
        }
    }
    const int tm = m / kMmaARows, r = m % kMmaARows;
    const int64_t g = k / kGroupK;
    const int kin = (int)(k % kGroupK);
    uint8_t* ub = aq + ((int64_t)tm * G + g) * kMmaAUnit;
    const int chunk = kin / 32, within = (kin % 32) / 2;  // 8 code bytes at byte 0 or 8 of the chunk
    uint2 cv;
    memcpy(&cv, codes, 8);
    *reinterpret_cast<uint2*>(ub + mma_code_off(r, chunk) + within) = cv;
    ub[kMmaARows * 128 + mma_scale_off(kin / 64, r, (kin % 64) / 16, 1)] = s;
    if (canon_codes && m < M && k < K) {
        memcpy(canon_codes + (int64_t)m * (K / 2) + k / 2, codes, 8);
        canon_scales[(int64_t)m * (K / 16) + k / 16] = s;
    }
}

}  // namespace qlin

using namespace qlin;

extern "C" cudaError_t qlin_launch_pack_mma(const void* codes, const void* scales, int64_t N, int64_t K, float gs,
                                            void* packed, cudaStream_t s) {
    const int64_t T = (N + kMmaWRows - 1) / kMmaWRows, G = (K + kGroupK - 1) / kGroupK;
    (void)gs;  // the header (with the per-tensor scale) is written by qlin_launch_pack
    pack_mma_kernel<<<(unsigned)(T * G), 256, 0, s>>>((const uint8_t*)codes, (const uint8_t*)scales, N, K, G,
                                                       (uint8_t*)packed);
    return cudaGetLastError();
}

extern "C" cudaError_t qlin_launch_act_quant(const void* x, int M, int64_t K, int64_t ldx, void* words, void* aq,
                                             void* canon_codes, void* canon_scales, cudaStream_t s, bool pdl) {
    const int64_t G = (K + kGroupK - 1) / kGroupK;
    const int TM = (M + kMmaARows - 1) / kMmaARows;
    int blocks = (int)(((int64_t)M * K + 255) / 256);
    if (blocks > 1184) blocks = 1184;
    if (blocks < 1) blocks = 1;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    cfg.blockDim = dim3(256);
    cfg.stream = s;
    cfg.gridDim = dim3((unsigned)blocks);
    cudaError_t e = cudaLaunchKernelEx(&cfg, act_amax_kernel, (const __nv_bfloat16*)x, M, K, ldx, (unsigned*)words);
    if (e != cudaSuccess) return e;
    const int64_t threads = (int64_t)TM * kMmaARows * G * 16;
    cfg.gridDim = dim3((unsigned)((threads + 255) / 256));
    cfg.numAttrs = 1;  // depends only on the amax kernel just launched
    return cudaLaunchKernelEx(&cfg, act_quant_kernel, (const __nv_bfloat16*)x, M, K, ldx, G, TM,
                              (const unsigned*)words, (uint8_t*)aq, (uint8_t*)canon_codes, (uint8_t*)canon_scales);
}
