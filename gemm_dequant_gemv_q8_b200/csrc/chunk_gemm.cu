// chunk_gemm.cu -- NVFP4 prefill-chunk GEMM on the 5th-generation tensor cores (sm_100a).
//
// y[m][n] = (a_g * g_w) * sum_k A_q[m][k] * W_q[n][k], with A_q the NVFP4-quantized activations
// (chunk_quant.cu) and W_q the NVFP4 weights, both as E2M1 codes with one E4M3 scale per 16 values.
// The block scales are applied inside the MMA (tcgen05.mma kind::mxf4nvf4, block16), the
// per-tensor scales in the epilogue.  The pages' counterpart is imp's NVFP4 block-scaled GEMM for
// prefill (README "Features", row "sm_120a kernels", written there with mma.sync for sm_120a);
// this is the datacenter-Blackwell form: TMEM accumulators, smem descriptors, a single thread
// issuing MMAs.
//
// One CTA per SM, persistent over 128 x 256 output tiles.  Warp roles:
//   warp 0  : producer -- bulk copies of one A unit (128 rows x 256 values + scales, 18 KB) and one
//             W unit (256 rows x 256 values + scales, 36 KB) per stage into a 3-stage ring;
//   warp 1  : one thread copies the stage's scale factors into tensor memory (tcgen05.cp) and
//             issues 4 block-scaled MMAs (K = 64 each), then commits the stage back to the producer
//             and, after the tile's last stage, the accumulator to the epilogue;
//   warps 2-5: epilogue -- tcgen05.ld of the 128 x 256 fp32 accumulator, scale, store y.
// Every mbarrier wait is bounded; a timeout sets the status word and the CTA winds down.
#include "chunk_common.cuh"

namespace qlin {

constexpr int kChunkStages = 3;
constexpr int kChunkStageBytes = kMmaAUnit + kMmaWUnit;                    // 55296, multiple of 1024
constexpr int kChunkSmem = kChunkStages * kChunkStageBytes + 1024 + 256;  // + alignment + barriers/flags
constexpr int kTmemCols = 512;
constexpr int kAccCols = 256;

struct ChunkArgs {
    const uint8_t* w;   // QLIN_PACK_MMA buffer (header + units)
    const uint8_t* aq;  // quantized activations (units)
    const unsigned* ag_word;
    float* y;
    int64_t ldy;
    int M;
    int64_t N, K;
    int T2, G, TM;
    unsigned* status;
};

__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr) {
    uint64_t d = (uint64_t)((saddr >> 4) & 0x3fffu);
    d |= (uint64_t)1 << 16;             // leading byte offset (unused for swizzled K-major)
    d |= (uint64_t)(1024 >> 4) << 32;   // stride byte offset: 8-row groups 1024 B apart
    d |= (uint64_t)1 << 46;             // descriptor version for sm_100
    d |= (uint64_t)2 << 61;             // 128-byte swizzle
    return d;
}

__device__ __forceinline__ uint64_t sdesc_sf(uint32_t saddr) {
    uint64_t d = (uint64_t)((saddr >> 4) & 0x3fffu);
    d |= (uint64_t)1 << 16;
    d |= (uint64_t)(128 >> 4) << 32;    // 8 rows x 16 B core matrices, contiguous
    d |= (uint64_t)1 << 46;
    return d;                           // no swizzle
}

// Instruction descriptor: E2M1 x E2M1, E4M3 scales, K-major A and B, M = 128, N = 256, K = 64.
__host__ __device__ constexpr uint32_t chunk_idesc() {
    return (1u << 7) | (1u << 10) | ((uint32_t)(256 >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
}

__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                       uint32_t sfa, uint32_t sfb, uint32_t accumulate) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n}\n" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
        : "memory");
}

__device__ __forceinline__ void tc_cp_sf(uint32_t taddr, uint64_t sdesc) {
    asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

__device__ __forceinline__ void tc_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tc_ld32(uint32_t taddr, float (&v)[32]) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

__global__ void __launch_bounds__(192, 1) chunk_gemm_kernel(const ChunkArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + kChunkStages * kChunkStageBytes);
    uint64_t* empty = full + kChunkStages;
    uint64_t* acc_full = empty + kChunkStages;
    uint64_t* acc_empty = acc_full + 1;
    uint64_t* mma_done = acc_empty + 1;
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(mma_done + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
    volatile int* issued = abort_flag + 1;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kChunkStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(acc_full, 1);
        mbar_init(acc_empty, 4);
        mbar_init(mma_done, 1);
        *abort_flag = 0;
        *issued = 0;
        fence_mbar_init();
    }
    if (warp == 0) {  // the whole warp allocates (and later frees) tensor memory
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_holder)),
                     "r"(kTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;
    griddep_wait();  // the quantized activations come from the previous kernels

    const int ntiles = a.T2 * a.TM;
    const uint32_t idesc = chunk_idesc();
    if (warp == 0) {
        if (lane == 0) {
            int it = 0;
            for (int tile = blockIdx.x; tile < ntiles && !*abort_flag; tile += gridDim.x) {
                const int t2 = tile / a.TM, tm = tile % a.TM;
                for (int g = 0; g < a.G; ++g, ++it) {
                    const int s = it % kChunkStages;
                    if (it >= kChunkStages && !mbar_wait_bounded(&empty[s], ((it / kChunkStages) - 1) & 1)) {
                        atomicOr(a.status, 1u);
                        *abort_flag = 1;
                        break;
                    }
                    uint8_t* st = smem + s * kChunkStageBytes;
                    mbar_arrive_expect_tx(&full[s], kChunkStageBytes);
                    bulk_g2s(st, a.aq + ((int64_t)tm * a.G + g) * kMmaAUnit, kMmaAUnit, &full[s]);
                    bulk_g2s(st + kMmaAUnit, a.w + kHdrBytes + ((int64_t)t2 * a.G + g) * kMmaWUnit, kMmaWUnit, &full[s]);
                    *issued = it + 1;
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            int it = 0, tcount = 0;
            for (int tile = blockIdx.x; tile < ntiles && !*abort_flag; tile += gridDim.x, ++tcount) {
                if (tcount > 0) {
                    if (!mbar_wait_bounded(acc_empty, (tcount - 1) & 1)) {
                        atomicOr(a.status, 1u);
                        *abort_flag = 1;
                        break;
                    }
                    tc_fence_after();
                }
                bool ok = true;
                for (int g = 0; g < a.G; ++g, ++it) {
                    const int s = it % kChunkStages;
                    if (!mbar_wait_bounded(&full[s], (it / kChunkStages) & 1)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sa = smem_u32(smem + s * kChunkStageBytes);
                    const uint32_t sb = sa + kMmaAUnit;
#pragma unroll
                    for (int kb = 0; kb < 4; ++kb) {
                        const uint32_t col = kAccCols + (uint32_t)((s * 4 + kb) * 12);
                        const uint32_t sfa = tmem + col, sfb = tmem + col + 4;
                        tc_cp_sf(sfa, sdesc_sf(sa + 128 * 128 + kb * 512));
                        tc_cp_sf(sfb, sdesc_sf(sb + 256 * 128 + (kb * 2 + 0) * 512));
                        tc_cp_sf(sfb + 4, sdesc_sf(sb + 256 * 128 + (kb * 2 + 1) * 512));
                        tc_mma(tmem, sdesc_sw128(sa + kb * 32), sdesc_sw128(sb + kb * 32), idesc, sfa, sfb,
                               (g > 0 || kb > 0) ? 1u : 0u);
                    }
                    tc_commit(&empty[s]);  // frees the stage once these MMAs have read it
                }
                if (!ok) {
                    atomicOr(a.status, 1u);
                    *abort_flag = 1;
                    break;
                }
                tc_commit(acc_full);
            }
            // every tcgen05 operation of this thread has completed before the CTA winds down
            tc_commit(mma_done);
            if (!mbar_wait_bounded(mma_done, 0)) atomicOr(a.status, 1u);
        }
    } else {  // epilogue warps 2..5: TMEM lane quarter = warp % 4
        const int q = warp & 3;
        float gw_ag = 0.f;
        {
            const float gw = reinterpret_cast<const PackedHeader*>(a.w)->global_scale;
            gw_ag = __fmul_rn(gw, __uint_as_float(*a.ag_word));
        }
        int tcount = 0;
        for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++tcount) {
            if (!mbar_wait_bounded(acc_full, tcount & 1)) {
                if (lane == 0) atomicOr(a.status, 1u);
                *abort_flag = 1;
                break;
            }
            tc_fence_after();
            const int t2 = tile / a.TM, tm = tile % a.TM;
            const int m = tm * kMmaARows + q * 32 + lane;
            float* yrow = a.y + (int64_t)m * a.ldy;
            const int64_t n0 = (int64_t)t2 * kMmaWRows;
#pragma unroll 1
            for (int c = 0; c < kAccCols; c += 32) {
                float v[32];
                tc_ld32(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)c, v);
                if (m < a.M) {
                    if (n0 + c + 32 <= a.N && ((reinterpret_cast<uintptr_t>(yrow + n0 + c) & 15) == 0)) {
#pragma unroll
                        for (int i = 0; i < 32; i += 4)
                            *reinterpret_cast<float4*>(yrow + n0 + c + i) =
                                make_float4(v[i] * gw_ag, v[i + 1] * gw_ag, v[i + 2] * gw_ag, v[i + 3] * gw_ag);
                    } else {
                        for (int i = 0; i < 32; ++i)
                            if (n0 + c + i < a.N) yrow[n0 + c + i] = v[i] * gw_ag;
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_expect_tx(acc_empty, 0);
        }
    }
    __syncthreads();
    if (warp == 0) {
        if (lane == 0 && *abort_flag) {
            // wait (bounded) for the last bulk copies issued to land before shared memory is released
            const int n_it = *issued;
            for (int j = n_it > kChunkStages ? n_it - kChunkStages : 0; j < n_it; ++j)
                mbar_wait_bounded(&full[j % kChunkStages], (j / kChunkStages) & 1, 50000000ull);
        }
        __syncwarp();
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols));
    }
}

}  // namespace qlin

using namespace qlin;

extern "C" size_t qlin_chunk_ws_bytes(int M, int64_t N, int64_t K) {
    (void)N;
    const int64_t G = (K + kGroupK - 1) / kGroupK;
    const int64_t TM = (M + kMmaARows - 1) / kMmaARows;
    return 256 + (size_t)(TM * G) * kMmaAUnit;
}

extern "C" cudaError_t qlin_launch_act_quant(const void* x, int M, int64_t K, int64_t ldx, void* words, void* aq,
                                             void* canon_codes, void* canon_scales, cudaStream_t s, bool pdl);

extern "C" cudaError_t qlin_launch_chunk(const void* packed, int64_t N, int64_t K, const void* x, int M, int64_t ldx,
                                         float* y, int64_t ldy, void* ws, int flags, cudaStream_t s) {
    uint8_t* w8 = (uint8_t*)ws;
    unsigned* words = (unsigned*)(w8 + 64);  // [amax, ticket, a_g]
    uint8_t* aq = w8 + 256;
    const bool pdl = (flags & QLIN_FLAG_PDL) != 0;
    cudaError_t e = qlin_launch_act_quant(x, M, K, ldx, words, aq, nullptr, nullptr, s, pdl);
    if (e != cudaSuccess) return e;
    static bool attr_set = false;
    if (!attr_set) {
        e = cudaFuncSetAttribute(chunk_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kChunkSmem);
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
    ChunkArgs a;
    a.w = (const uint8_t*)packed;
    a.aq = aq;
    a.ag_word = words + 2;
    a.y = y;
    a.ldy = ldy;
    a.M = M;
    a.N = N;
    a.K = K;
    a.T2 = (int)((N + kMmaWRows - 1) / kMmaWRows);
    a.G = (int)((K + kGroupK - 1) / kGroupK);
    a.TM = (M + kMmaARows - 1) / kMmaARows;
    a.status = (unsigned*)ws;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int ntiles = a.T2 * a.TM;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(ntiles < sms ? ntiles : sms));
    cfg.blockDim = dim3(192);
    cfg.dynamicSmemBytes = kChunkSmem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, chunk_gemm_kernel, a);
}

extern "C" cudaError_t qlin_launch_act_quant_debug(const void* x, int M, int64_t K, int64_t ldx, void* ws,
                                                   void* codes, void* scales, float* ag, cudaStream_t s) {
    uint8_t* w8 = (uint8_t*)ws;
    unsigned* words = (unsigned*)(w8 + 64);
    cudaError_t e = qlin_launch_act_quant(x, M, K, ldx, words, w8 + 256, codes, scales, s, false);
    if (e != cudaSuccess) return e;
    return cudaMemcpyAsync(ag, words + 2, 4, cudaMemcpyDeviceToDevice, s);
}
