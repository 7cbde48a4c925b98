// chunk_quant.cu -- the chunk path's operand preparation (sm_100a):
//   * QLIN_PACK_MMA weight packing: canonical NVFP4 / MXFP4 -> the tensor-core operand layout;
//   * NVFP4 / MXFP4 quantization of bf16 activations (the A operand; MXFP4 by the OCP MX rule,
//     see chunk_common.cuh).
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
// One CTA per unit (256-row tile, k-group); thread r writes row r.  MX: UE8M0 scales of 32 values
// (canonical [N][K/32]) instead of E4M3 scales of 16 ([N][K/16]).  gate_half > 0 (QLIN_PACK_GATE_UP,
// the N = 2 * gate_half rows being [gate ; up]): tile t holds gate rows 128t .. 128t + 127 in its
// rows 0..127 and the matching up rows in rows 128..255, so an output tile holds g and u of the same
// 128 outputs (rows past gate_half are zero).
template <bool MX>
__global__ void __launch_bounds__(256) pack_mma_kernel(const uint8_t* __restrict__ codes,
                                                       const uint8_t* __restrict__ scales, int64_t N,
                                                       int64_t K, int64_t G, int64_t gate_half,
                                                       uint8_t* __restrict__ packed) {
    const int64_t unit = blockIdx.x;
    const int64_t t = unit / G, g = unit % G;
    const int r = threadIdx.x;
    int64_t n = t * kMmaWRows + r;
    if (gate_half > 0) {
        const int64_t i = t * 128 + (r & 127);
        n = i < gate_half ? (r < 128 ? i : gate_half + i) : N;  // N: a zero row
    }
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
    if (MX) {
        for (int b = 0; b < 8; ++b) {  // 32-value block b of the k-group
            const int64_t kb32 = k0 + 32 * b;
            const uint8_t s = (n < N && kb32 < K) ? scales[n * (K / 32) + kb32 / 32] : 0;
            sc[mma_scale_off(b >> 2, r, b & 3, 2)] = s;
        }
    } else {
        for (int b = 0; b < 16; ++b) {  // 16-value block b of the k-group
            const int64_t kb16 = k0 + 16 * b;
            const uint8_t s = (n < N && kb16 < K) ? scales[n * (K / 16) + kb16 / 16] : 0;
            sc[mma_scale_off(b >> 2, r, b & 3, 2)] = s;
        }
    }
}

// ------------------------------------------------------------------ activation quantization
// The standalone form of step 1 of the chunk path, used by the inspection entry point
// (qlin_act_quant_debug); qlin_gemm_chunk runs the same per-item code inside its persistent kernel.
// Block-wide max of |x| folded into one word with atomicMax (order-independent, deterministic);
// the last block to finish turns it into a_g and clears the accumulator for the next call.
__global__ void __launch_bounds__(256) act_amax_kernel(const __nv_bfloat16* __restrict__ x, int M, int64_t K,
                                                       int64_t ldx, bool vec, unsigned* __restrict__ words) {
    // words[0] = amax bits (accumulating), words[1] = ticket, words[2] = a_g (float bits, output)
    float m = act_amax_partial(x, M, K, ldx, vec, (int64_t)blockIdx.x * blockDim.x + threadIdx.x,
                               (int64_t)gridDim.x * blockDim.x);
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
            words[2] = __float_as_uint(act_global_scale(amax));
            words[0] = 0u;
            words[1] = 0u;
        }
    }
}

// One thread per (row, 16-value block) of the padded operand.
__global__ void __launch_bounds__(256) act_quant_kernel(const __nv_bfloat16* __restrict__ x, int M, int64_t K,
                                                        int64_t ldx, int64_t G, int TM, bool vec,
                                                        const unsigned* __restrict__ words, uint8_t* __restrict__ aq,
                                                        uint8_t* __restrict__ canon_codes,
                                                        uint8_t* __restrict__ canon_scales) {
    const int64_t nblk16 = G * 16;  // 16-value blocks per padded row
    const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= (int64_t)TM * kMmaARows * nblk16) return;
    const int m = (int)(idx / nblk16);
    act_quant_item(x, M, K, ldx, G, __uint_as_float(words[2]), vec, m, idx - (int64_t)m * nblk16, aq, canon_codes,
                   canon_scales);
}

// MXFP4: one thread per (row, 16-value item) of the padded operand; the two items of a 32-value
// block are adjacent threads of one warp (no global scale, no max pass).
__global__ void __launch_bounds__(256) act_quant_mx_kernel(const __nv_bfloat16* __restrict__ x, int M, int64_t K,
                                                           int64_t ldx, int64_t G, int TM, bool vec,
                                                           uint8_t* __restrict__ aq, uint8_t* __restrict__ canon_codes,
                                                           uint8_t* __restrict__ canon_scales) {
    const int64_t nblk16 = G * 16;
    const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const bool live = idx < (int64_t)TM * kMmaARows * nblk16;  // a multiple of 32: whole warps
    const int m = live ? (int)(idx / nblk16) : 0;
    const int64_t b = live ? idx - (int64_t)m * nblk16 : 0;
    uint32_t w[8], c8[2];
    act_load_item(x, live ? M : 0, K, ldx, vec, m, b, w);
    const uint8_t byte = act_mx_pair_byte(act_item_amax(w), act_item_special(w));
    if (!live) return;
    act_quant_item_mx_codes(w, byte, c8);
    act_store_item_mx(M, K, G, m, b, byte, c8, aq, canon_codes, canon_scales);
}

}  // namespace qlin

using namespace qlin;

// Weight tiles of the MMA layout: 256 rows each, or (gate_up) one per 128 gate rows.
extern "C" int64_t qlin_mma_tiles(int64_t N, int gate_up) {
    return gate_up ? (N / 2 + 127) / 128 : (N + kMmaWRows - 1) / kMmaWRows;
}

extern "C" cudaError_t qlin_launch_pack_mma(int fmt, const void* codes, const void* scales, int64_t N, int64_t K,
                                            int gate_up, void* packed, cudaStream_t s) {
    const int64_t T = qlin_mma_tiles(N, gate_up), G = (K + kGroupK - 1) / kGroupK;
    const int64_t half = gate_up ? N / 2 : 0;
    // (the header, with the per-tensor scale, is written by qlin_launch_pack)
    if (fmt == QLIN_MXFP4)
        pack_mma_kernel<true><<<(unsigned)(T * G), 256, 0, s>>>((const uint8_t*)codes, (const uint8_t*)scales, N, K, G,
                                                                 half, (uint8_t*)packed);
    else
        pack_mma_kernel<false><<<(unsigned)(T * G), 256, 0, s>>>((const uint8_t*)codes, (const uint8_t*)scales, N, K,
                                                                  G, half, (uint8_t*)packed);
    return cudaGetLastError();
}

extern "C" cudaError_t qlin_launch_act_quant_mx(const void* x, int M, int64_t K, int64_t ldx, void* aq,
                                                void* canon_codes, void* canon_scales, cudaStream_t s) {
    const int64_t G = (K + kGroupK - 1) / kGroupK;
    const int TM = (M + kMmaARows - 1) / kMmaARows;
    const bool vec = ((reinterpret_cast<uintptr_t>(x) & 15) == 0) && (ldx % 8 == 0);
    const int64_t threads = (int64_t)TM * kMmaARows * G * 16;
    act_quant_mx_kernel<<<(unsigned)((threads + 255) / 256), 256, 0, s>>>(
        (const __nv_bfloat16*)x, M, K, ldx, G, TM, vec, (uint8_t*)aq, (uint8_t*)canon_codes, (uint8_t*)canon_scales);
    return cudaGetLastError();
}

extern "C" cudaError_t qlin_launch_act_quant(const void* x, int M, int64_t K, int64_t ldx, void* words, void* aq,
                                             void* canon_codes, void* canon_scales, cudaStream_t s) {
    const int64_t G = (K + kGroupK - 1) / kGroupK;
    const int TM = (M + kMmaARows - 1) / kMmaARows;
    const bool vec = ((reinterpret_cast<uintptr_t>(x) & 15) == 0) && (ldx % 8 == 0);
    int blocks = (int)(((int64_t)M * K + 255) / 256);
    if (blocks > 1184) blocks = 1184;
    if (blocks < 1) blocks = 1;
    act_amax_kernel<<<blocks, 256, 0, s>>>((const __nv_bfloat16*)x, M, K, ldx, vec, (unsigned*)words);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const int64_t threads = (int64_t)TM * kMmaARows * G * 16;
    act_quant_kernel<<<(unsigned)((threads + 255) / 256), 256, 0, s>>>(
        (const __nv_bfloat16*)x, M, K, ldx, G, TM, vec, (const unsigned*)words, (uint8_t*)aq, (uint8_t*)canon_codes,
        (uint8_t*)canon_scales);
    return cudaGetLastError();
}
