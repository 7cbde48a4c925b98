// chunk_gemm.cu -- NVFP4 prefill-chunk GEMM on the 5th-generation tensor cores (sm_100a).
//
// y[m][n] = (a_g * g_w) * sum_k A_q[m][k] * W_q[n][k], with A_q the NVFP4-quantized activations
// and W_q the NVFP4 weights, both as E2M1 codes with one E4M3 scale per 16 values.  The block
// scales are applied inside the MMA (tcgen05.mma kind::mxf4nvf4, block16), the per-tensor scales
// in the epilogue.  The pages' counterpart is imp's NVFP4 block-scaled GEMM for prefill (README
// "Features", row "sm_120a kernels", written there with mma.sync for sm_120a); this is the
// datacenter-Blackwell form: TMEM accumulators, smem descriptors, a single thread issuing MMAs.
//
// One launch, one persistent CTA per SM:
//   phase Q (all warps of all CTAs): max |x| over the whole tensor (one atomicMax per CTA), a
//            bounded grid-wide barrier, a_g, then every CTA quantizes its share of the
//            (row, 16-value block) items into the MMA operand layout; a second grid barrier.
//   phase G (warp roles), over 128 x 256 output tiles:
//     warp 0   : producer -- bulk copies of one A unit (128 rows x 256 values + scales, 18 KB) and
//                one W unit (256 rows x 256 values + scales, 36 KB) per stage, 4-stage ring;
//     warp 1   : one thread issues the stage's 4 block-scaled MMAs (K = 64 each), commits the
//                stage back and, after the tile's last stage, the accumulator to the epilogue;
//     warps 2-5: scale-factor writers -- move the stage's E4M3 scales from shared memory into
//                tensor memory with tcgen05.st (one TMEM lane quarter each), so that the tensor
//                pipe spends its time on MMAs only;
//     warps 6-9: epilogue -- tcgen05.ld of the 128 x 256 fp32 accumulator, 32 columns at a time,
//                released to the MMAs as soon as it has been read; the scaled values go out
//                through a small per-warp transpose buffer so that stores are row-contiguous.
// Every wait is bounded; a timeout sets the status word and the CTA winds down.
#include "chunk_common.cuh"

namespace qlin {

constexpr int kChunkStages = 4;
constexpr int kChunkStageBytes = kMmaAUnit + kMmaWUnit;  // 55296, multiple of 1024
constexpr int kEpiWarps = 4;
constexpr int kEpiBuf = 32 * 64;                          // one 32 x 16 fp32 transpose buffer per warp
constexpr int kChunkRingBytes = kChunkStages * kChunkStageBytes;
constexpr int kChunkEpiBytes = kEpiWarps * kEpiBuf;
constexpr int kChunkSmem = 1024 + kChunkRingBytes + kChunkEpiBytes + 256;
constexpr int kChunkThreads = 320;
constexpr int kTmemCols = 512;
constexpr int kAccCols = 256;
constexpr int kSfCols = 48;  // per stage: 4 k-blocks x (4 SFA + 8 SFB) columns
constexpr int kQItems = 8;   // activation items held in registers per thread in phase Q

// workspace words (after the status word): amax accumulator, barrier counters, a_g
constexpr int kWAmax = 0, kWArrive1 = 1, kWAg = 2, kWArrive2 = 3, kWExit = 4;

struct ChunkArgs {
    const uint8_t* w;   // QLIN_PACK_MMA buffer (header + units)
    const __nv_bfloat16* x;
    int64_t ldx;
    uint8_t* aq;        // quantized activations (units), in the workspace
    unsigned* words;
    float* y;
    int64_t ldy;
    int M;
    int64_t N, K;
    int T2, G, TM;
    int xvec;
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

// 16 consecutive 32-bit TMEM columns of this warp's lane quarter from r[O .. O+15] of each thread.
template <int O>
__device__ __forceinline__ void tc_st16(uint32_t taddr, const uint32_t (&r)[48]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
            taddr),
        "r"(r[O + 0]), "r"(r[O + 1]), "r"(r[O + 2]), "r"(r[O + 3]), "r"(r[O + 4]), "r"(r[O + 5]), "r"(r[O + 6]),
        "r"(r[O + 7]), "r"(r[O + 8]), "r"(r[O + 9]), "r"(r[O + 10]), "r"(r[O + 11]), "r"(r[O + 12]), "r"(r[O + 13]),
        "r"(r[O + 14]), "r"(r[O + 15])
        : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ unsigned ld_acquire_gpu(const unsigned* p) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void fence_proxy_async_global() {
    asm volatile("fence.proxy.async.global;" ::: "memory");
}

// Grid-wide barrier on a counter that only grows within one launch (reset by the last CTA out).
// Called by one thread per CTA; false after ~2 s without all CTAs arriving.
__device__ __forceinline__ bool grid_arrive_wait(unsigned* counter, unsigned target) {
    __threadfence();
    atomicAdd(counter, 1u);
    if (ld_acquire_gpu(counter) >= target) return true;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t it = 1;; ++it) {
        if (ld_acquire_gpu(counter) >= target) return true;
        if ((it & 63u) == 0 && globaltimer_ns() - t0 > 2000000000ull) return false;
        __nanosleep(64);
    }
}

__global__ void __launch_bounds__(kChunkThreads, 1) chunk_gemm_kernel(const ChunkArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    uint8_t* epi = smem + kChunkRingBytes;
    uint64_t* full = reinterpret_cast<uint64_t*>(epi + kChunkEpiBytes);
    uint64_t* empty = full + kChunkStages;
    uint64_t* sfready = empty + kChunkStages;
    uint64_t* acc_full = sfready + kChunkStages;
    uint64_t* acc_empty = acc_full + 1;
    uint64_t* mma_done = acc_empty + 1;
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(mma_done + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
    volatile int* issued = abort_flag + 1;
    volatile float* ag_sm = reinterpret_cast<volatile float*>(issued + 1);
    float* red = const_cast<float*>(ag_sm + 1);  // one partial max per warp
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kChunkStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
            mbar_init(&sfready[s], 4);
        }
        mbar_init(acc_full, 1);
        mbar_init(acc_empty, kEpiWarps);
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
    const int ntiles = a.T2 * a.TM;
    griddep_wait();  // x comes from the previous kernels

    // ---------------------------------------------------------------- phase Q: quantize x
    // When every thread has at most kQItems (row, 16-value block) items, the items stay in
    // registers between the max pass and the quantization (x is read once, all loads in flight
    // together); otherwise x is read twice.
    {
        const int64_t gtid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
        const int64_t gthreads = (int64_t)gridDim.x * blockDim.x;
        const int64_t nblk16 = (int64_t)a.G * 16;
        const int64_t items = (int64_t)a.TM * kMmaARows * nblk16;
        const bool resident = items <= gthreads * kQItems;
        const bool vec = a.xvec != 0;
        uint32_t xw[kQItems][8];
        float bmax[kQItems];
        float m = 0.f;
        // item i = m * nblk16 + b; thread items i0 + j * gthreads, coordinates advanced without division
        const int64_t qstep = gthreads / nblk16, rstep = gthreads - qstep * nblk16;
        const int m_first = (int)(gtid / nblk16);
        const int64_t b_first = gtid - (int64_t)m_first * nblk16;
        if (resident) {
            int mj = m_first;
            int64_t bj = b_first;
#pragma unroll
            for (int j = 0; j < kQItems; ++j) {
                act_load_item(a.x, gtid + j * gthreads < items ? a.M : 0, a.K, a.ldx, vec, mj, bj, xw[j]);
                mj += (int)qstep;
                bj += rstep;
                if (bj >= nblk16) bj -= nblk16, ++mj;
            }
#pragma unroll
            for (int j = 0; j < kQItems; ++j) {
                bmax[j] = act_item_amax(xw[j]);
                m = fmaxf(m, bmax[j]);
            }
        } else {
            m = act_amax_partial(a.x, a.M, a.K, a.ldx, vec, gtid, gthreads);
        }
        for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if (lane == 0) red[warp] = m;
        __syncthreads();
        if (threadIdx.x == 0) {
            float b = 0.f;
            for (int w = 0; w < kChunkThreads / 32; ++w) b = fmaxf(b, red[w]);
            atomicMax(&a.words[kWAmax], __float_as_uint(b));  // non-negative floats order as their bits
            float ag = 0.f;
            if (grid_arrive_wait(&a.words[kWArrive1], gridDim.x)) {
                ag = act_global_scale(__uint_as_float(ld_acquire_gpu(&a.words[kWAmax])));
                if (blockIdx.x == 0) a.words[kWAg] = __float_as_uint(ag);
            } else {
                atomicOr(a.status, 1u);
                *abort_flag = 1;
            }
            *ag_sm = ag;
        }
        __syncthreads();
        if (!*abort_flag) {
            const float ag = *ag_sm;
            if (resident) {
                int mj = m_first;
                int64_t bj = b_first;
#pragma unroll
                for (int j = 0; j < kQItems; ++j) {
                    if (gtid + j * gthreads < items) {
                        uint32_t c8[2];
                        const uint8_t sc = act_quant_block(xw[j], bmax[j], ag, c8);
                        act_store_item(a.M, a.K, a.G, mj, bj, sc, c8, a.aq, nullptr, nullptr);
                    }
                    mj += (int)qstep;
                    bj += rstep;
                    if (bj >= nblk16) bj -= nblk16, ++mj;
                }
            } else {
                for (int64_t i = gtid; i < items; i += gthreads) {
                    const int mrow = (int)(i / nblk16);
                    act_quant_item(a.x, a.M, a.K, a.ldx, a.G, ag, vec, mrow, i - (int64_t)mrow * nblk16, a.aq,
                                   nullptr, nullptr);
                }
            }
            fence_proxy_async_global();  // the operand is read back by bulk copies (async proxy)
        }
        __syncthreads();
        if (threadIdx.x == 0) {
            if (!grid_arrive_wait(&a.words[kWArrive2], gridDim.x)) {
                atomicOr(a.status, 1u);
                *abort_flag = 1;
            }
            fence_proxy_async_global();
        }
        __syncthreads();
    }

    // ---------------------------------------------------------------- phase G: the GEMM
    if (warp == 0) {
        if (lane == 0) {
            fence_proxy_async_global();  // this thread's bulk copies read what phase Q wrote
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
            const uint32_t idesc = chunk_idesc();
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
                    const uint32_t par = (it / kChunkStages) & 1;
                    if (!mbar_wait_bounded(&full[s], par) || !mbar_wait_bounded(&sfready[s], par)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sa = smem_u32(smem + s * kChunkStageBytes);
                    const uint32_t sb = sa + kMmaAUnit;
#pragma unroll
                    for (int kb = 0; kb < 4; ++kb) {
                        const uint32_t col = kAccCols + (uint32_t)(s * kSfCols + kb * 12);
                        tc_mma(tmem, sdesc_sw128(sa + kb * 32), sdesc_sw128(sb + kb * 32), idesc, tmem + col,
                               tmem + col + 4, (g > 0 || kb > 0) ? 1u : 0u);
                    }
                    tc_commit(&empty[s]);  // frees the stage (smem and its scale columns) once read
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
    } else if (warp < 2 + 4) {  // scale-factor writers: TMEM lane quarter = warp % 4
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        int it = 0;
        for (int tile = blockIdx.x; tile < ntiles && !*abort_flag; tile += gridDim.x) {
            bool ok = true;
            for (int g = 0; g < a.G; ++g, ++it) {
                const int s = it % kChunkStages;
                if (it >= kChunkStages && !mbar_wait_bounded(&empty[s], ((it / kChunkStages) - 1) & 1)) {
                    ok = false;
                    break;
                }
                if (!mbar_wait_bounded(&full[s], (it / kChunkStages) & 1)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                // Atom layout (both operands): the 4 scales of row r (0..127 of a 128-row half) are
                // word r / 32 of 16-byte row r % 32.  Every lane quarter of TMEM gets the whole atom:
                // lane 32q + i, columns c..c+3 = the atom's 16-byte row i.
                const uint8_t* st = smem + s * kChunkStageBytes;
                const uint8_t* sfa = st + kMmaARows * 128 + lane * 16;
                const uint8_t* sfb = st + kMmaAUnit + kMmaWRows * 128 + lane * 16;
                uint32_t r[48];
#pragma unroll
                for (int kb = 0; kb < 4; ++kb) {
                    const uint4 va = lds128(sfa + kb * 512);
                    const uint4 vb0 = lds128(sfb + (kb * 2 + 0) * 512);
                    const uint4 vb1 = lds128(sfb + (kb * 2 + 1) * 512);
                    r[kb * 12 + 0] = va.x, r[kb * 12 + 1] = va.y, r[kb * 12 + 2] = va.z, r[kb * 12 + 3] = va.w;
                    r[kb * 12 + 4] = vb0.x, r[kb * 12 + 5] = vb0.y, r[kb * 12 + 6] = vb0.z, r[kb * 12 + 7] = vb0.w;
                    r[kb * 12 + 8] = vb1.x, r[kb * 12 + 9] = vb1.y, r[kb * 12 + 10] = vb1.z, r[kb * 12 + 11] = vb1.w;
                }
                const uint32_t cbase = tmem + lane_base + kAccCols + (uint32_t)(s * kSfCols);
                tc_st16<0>(cbase, r);
                tc_st16<16>(cbase + 16, r);
                tc_st16<32>(cbase + 32, r);
                asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sfready[s]);
            }
            if (!ok) {
                if (lane == 0) atomicOr(a.status, 1u);
                *abort_flag = 1;
                break;
            }
        }
    } else {  // epilogue warps 6..9: TMEM lane quarter = warp % 4
        const int q = warp & 3;
        const uint32_t lane_base = (uint32_t)(q * 32) << 16;
        const float gw_ag = __fmul_rn(reinterpret_cast<const PackedHeader*>(a.w)->global_scale, *ag_sm);
        // 32 rows x 16 columns, row pitch 64 B, 16-byte chunk j of row r at position j ^ (r % 4)
        uint8_t* tb = epi + (warp - 6) * kEpiBuf;
        int tcount = 0;
        for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++tcount) {
            if (*abort_flag || !mbar_wait_bounded(acc_full, tcount & 1)) {
                if (lane == 0) atomicOr(a.status, 1u);
                *abort_flag = 1;
                break;
            }
            tc_fence_after();
            const int t2 = tile / a.TM, tm = tile % a.TM;
            const int m0 = tm * kMmaARows + q * 32;  // this warp's first row
            const int64_t n0 = (int64_t)t2 * kMmaWRows;
#pragma unroll 1
            for (int c = 0; c < kAccCols; c += 32) {
                float v[32];
                tc_ld32(tmem + lane_base + (uint32_t)c, v);
                if (c == kAccCols - 32) {  // the accumulator has been read: release it to the MMAs
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(acc_empty);
                }
                if (m0 >= a.M || n0 + c >= a.N) continue;
                // Transpose through shared memory so that each store instruction writes 8 rows x
                // 64 contiguous bytes instead of 32 rows x 16 bytes.
#pragma unroll
                for (int h = 0; h < 2; ++h) {
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        *reinterpret_cast<float4*>(tb + lane * 64 + ((j ^ (lane & 3)) << 4)) =
                            make_float4(v[16 * h + 4 * j] * gw_ag, v[16 * h + 4 * j + 1] * gw_ag,
                                        v[16 * h + 4 * j + 2] * gw_ag, v[16 * h + 4 * j + 3] * gw_ag);
                    __syncwarp();
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int r = 8 * i + (lane >> 2), ch = lane & 3;
                        const float4 val = *reinterpret_cast<const float4*>(tb + r * 64 + ((ch ^ (r & 3)) << 4));
                        const int mrow = m0 + r;
                        const int64_t ncol = n0 + c + 16 * h + 4 * ch;
                        if (mrow < a.M && ncol < a.N) {
                            float* dst = a.y + (int64_t)mrow * a.ldy + ncol;
                            if (ncol + 4 <= a.N && (reinterpret_cast<uintptr_t>(dst) & 15) == 0) {
                                *reinterpret_cast<float4*>(dst) = val;
                            } else {
                                const float e[4] = {val.x, val.y, val.z, val.w};
                                for (int u = 0; u < 4 && ncol + u < a.N; ++u) dst[u] = e[u];
                            }
                        }
                    }
                    __syncwarp();
                }
            }
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
    if (threadIdx.x == 0) {  // the last CTA out clears the counters for the next call
        __threadfence();
        if (atomicAdd(&a.words[kWExit], 1u) == gridDim.x - 1) {
            a.words[kWAmax] = 0u;
            a.words[kWArrive1] = 0u;
            a.words[kWArrive2] = 0u;
            a.words[kWExit] = 0u;
            __threadfence();
        }
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
                                             void* canon_codes, void* canon_scales, cudaStream_t s);

extern "C" cudaError_t qlin_launch_chunk(const void* packed, int64_t N, int64_t K, const void* x, int M, int64_t ldx,
                                         float* y, int64_t ldy, void* ws, int flags, cudaStream_t s) {
    static bool attr_set = false;
    cudaError_t e;
    if (!attr_set) {
        e = cudaFuncSetAttribute(chunk_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kChunkSmem);
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
    uint8_t* w8 = (uint8_t*)ws;
    ChunkArgs a;
    a.w = (const uint8_t*)packed;
    a.x = (const __nv_bfloat16*)x;
    a.ldx = ldx;
    a.aq = w8 + 256;
    a.words = (unsigned*)(w8 + 64);
    a.y = y;
    a.ldy = ldy;
    a.M = M;
    a.N = N;
    a.K = K;
    a.T2 = (int)((N + kMmaWRows - 1) / kMmaWRows);
    a.G = (int)((K + kGroupK - 1) / kGroupK);
    a.TM = (M + kMmaARows - 1) / kMmaARows;
    a.xvec = ((reinterpret_cast<uintptr_t>(x) & 15) == 0 && ldx % 8 == 0) ? 1 : 0;
    a.status = (unsigned*)ws;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    // All CTAs must be co-resident (grid-wide barriers): one per SM at most.
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, chunk_gemm_kernel, kChunkThreads, kChunkSmem);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    const int ntiles = a.T2 * a.TM;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(ntiles < sms ? ntiles : sms));
    cfg.blockDim = dim3(kChunkThreads);
    cfg.dynamicSmemBytes = kChunkSmem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = (flags & QLIN_FLAG_PDL) ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, chunk_gemm_kernel, a);
}

extern "C" cudaError_t qlin_launch_act_quant_debug(const void* x, int M, int64_t K, int64_t ldx, void* ws,
                                                   void* codes, void* scales, float* ag, cudaStream_t s) {
    uint8_t* w8 = (uint8_t*)ws;
    unsigned* words = (unsigned*)(w8 + 64);
    cudaError_t e = qlin_launch_act_quant(x, M, K, ldx, words, w8 + 256, codes, scales, s);
    if (e != cudaSuccess) return e;
    return cudaMemcpyAsync(ag, words + 2, 4, cudaMemcpyDeviceToDevice, s);
}
