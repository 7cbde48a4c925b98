// chunk_bf16.cu -- prefill-chunk GEMM for the GGUF / MXFP4 weight formats on the 5th-generation
// tensor cores (sm_100a): y[m][n] = g * sum_k x[m][k] * Wb[n][k], x bf16 as given, Wb the bf16 copy
// of the dequantized weights that qlin_pack_weights(QLIN_PACK_MMA / QLIN_PACK_MMA_BF16) builds once
// (each weight the fp32 dequantized value rounded to nearest-even bf16; for NVFP4 the exact product
// of code and block scale), fp32 accumulation in tensor memory, g the per-tensor scale of the
// packed header (1 for every format but NVFP4) applied once per output.
//
// The pages' counterpart: imp keeps "full-precision prefill via source dequant" for GGUF models
// (README "Why this exists") and runs its prefill GEMMs on the tensor cores; here the dequantized
// copy is bf16 and the GEMM is tcgen05.mma kind::f16 with TMEM accumulators.
//
// One launch, persistent CTAs (at most one per SM), K in stages of 64, tiles of 128 x 256 (CG = 1)
// or 256 x 256 per pair of CTAs (CG = 2, cta_group::2: each CTA stages its 128 activation rows and
// half of the 256 weight rows, so each SM writes and the MMA reads 32 KB of shared memory per
// stage instead of 48 KB):
//   warp 0   : producer -- two TMA tensor loads per stage (x rows and weight rows, 64 values each,
//              128-byte swizzled by the tensor maps) into the ring; rows and columns outside the
//              tensors read as zero.  The weight copy is stored in blocks of 256 rows x 64 values,
//              so a stage's weight tile is one contiguous 32 KB block (a 4-D tensor map).  With CG = 2 both CTAs' loads complete on the first CTA's
//              stage barrier (the .cta_group::2 form), which alone tracks a stage's bytes;
//   warp 1   : one thread (of the first CTA) issues the stage's four M128/M256 N256 K16 MMAs,
//              commits the stage back to the producers (both CTAs) and, after the tile's last
//              stage, the accumulator to the epilogues;
//   warps 2-5: epilogue -- tcgen05.ld of this CTA's 128 x 256 fp32 accumulator rows (one TMEM lane
//              quarter each), released to the MMAs once read, stored to y through a transpose buffer.
// Tensor memory holds two accumulators, used by alternate tiles, so a tile's drain overlaps the next
// tile's MMAs.
// Every wait is bounded; a timeout sets the status word and the CTA winds down.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "qlin_common.cuh"

namespace qlin {

namespace cb {

constexpr int kRows = 128;          // activation rows per CTA (MMA M per CTA)
constexpr int kCols = 256;          // weight rows per tile (MMA N)
constexpr int kKStage = 64;         // K per stage: one 128-byte swizzle span of bf16
constexpr int kABytes = kRows * 128;
constexpr int kEpiWarps = 4, kFirstEpi = 2;
constexpr int kThreads = (kFirstEpi + kEpiWarps) * 32;
constexpr int kEpiBuf = 32 * 64;  // one warp's 32 x 16 fp32 transpose buffer
constexpr int kTmemCols = 512;  // two 256-column accumulators: the next tile's MMAs run while one drains
template <int CG>
struct Cfg {
    static constexpr int kBRows = kCols / CG;                 // weight rows staged by this CTA
    static constexpr int kBBytes = kBRows * 128;
    static constexpr int kStageBytes = kABytes + kBBytes;    // 48 KB (CG = 1) or 32 KB (CG = 2)
    static constexpr int kStages = CG == 1 ? 4 : 6;
    static constexpr int kSmem = 1024 + kStages * kStageBytes + kEpiWarps * kEpiBuf + 256;
};
static_assert(Cfg<1>::kSmem <= 232448 && Cfg<2>::kSmem <= 232448, "shared memory budget");

struct Args {
    const float* gscale;  // the per-tensor scale in the packed header
    float* y;
    int64_t ldy;
    int M;
    int64_t N, K;
    int TM, TN, KS;  // row tiles, weight-row tiles, K stages
    unsigned* status;
};

__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr) {
    uint64_t d = (uint64_t)((saddr >> 4) & 0x3fffu);
    d |= (uint64_t)1 << 16;            // leading byte offset (unused for swizzled K-major)
    d |= (uint64_t)(1024 >> 4) << 32;  // stride byte offset: 8-row groups 1024 B apart
    d |= (uint64_t)1 << 46;            // descriptor version for sm_100
    d |= (uint64_t)2 << 61;            // 128-byte swizzle
    return d;
}

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
            smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}
// CTA pairs: the load lands in this CTA's shared memory and completes on the barrier at the same
// offset in the pair's first CTA (no multicast: each CTA loads its own rows).
__device__ __forceinline__ void tma_load_2d_pair(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
    asm volatile(
        "{\n .reg .b32 rb;\n mapa.shared::cluster.u32 rb, %4, 0;\n"
        " cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [rb];\n}\n" ::"r"(
            smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}

// The weight copy is blocked (256 rows x 64 values contiguous, 32 KB): a 4-D tensor map {value,
// row in block, k-block, row block}; one box is this CTA's rows of one block.
__device__ __forceinline__ void tma_load_4d(void* dst, const CUtensorMap* map, int c1, int c2, int c3,
                                            uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(
            smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(0), "r"(c1), "r"(c2), "r"(c3), "r"(smem_u32(bar))
        : "memory");
}
__device__ __forceinline__ void tma_load_4d_pair(void* dst, const CUtensorMap* map, int c1, int c2, int c3,
                                                 uint64_t* bar) {
    asm volatile(
        "{\n .reg .b32 rb;\n mapa.shared::cluster.u32 rb, %6, 0;\n"
        " cp.async.bulk.tensor.4d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4, %5}], [rb];\n}\n" ::"r"(
            smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(0), "r"(c1), "r"(c2), "r"(c3), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ uint32_t cta_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Arrive on the mbarrier at the same offset in CTA `rank` of the cluster.
__device__ __forceinline__ void mbar_arrive_remote(uint64_t* bar, uint32_t rank) {
    asm volatile(
        "{\n .reg .b32 ra;\n mapa.shared::cluster.u32 ra, %0, %1;\n"
        " mbarrier.arrive.release.cluster.shared::cluster.b64 _, [ra];\n}\n" ::"r"(smem_u32(bar)),
        "r"(rank)
        : "memory");
}

template <int CG>
__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t accumulate) {
    if constexpr (CG == 1)
        asm volatile(
            "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
            " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
            "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
            : "memory");
    else
        asm volatile(
            "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
            " tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
            "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
            : "memory");
}

// Commit this thread's MMAs to the barrier at `bar` (CG = 2: in both CTAs of the pair).
template <int CG>
__device__ __forceinline__ void commit(uint64_t* bar) {
    if constexpr (CG == 1)
        asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                     : "memory");
    else
        asm volatile(
            "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
                smem_u32(bar)),
            "h"((uint16_t)3)
            : "memory");
}
// Commit to this CTA's own barrier only.
template <int CG>
__device__ __forceinline__ void commit_self(uint64_t* bar) {
    if constexpr (CG == 1)
        asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                     : "memory");
    else
        asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                     : "memory");
}

__device__ __forceinline__ void fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void ld32(uint32_t taddr, float (&v)[32]) {
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

__device__ __forceinline__ void mbar_arrive_local(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

}  // namespace cb

template <int CG>
__global__ void __launch_bounds__(cb::kThreads, 1)
    chunk_bf16_kernel(const cb::Args a, const __grid_constant__ CUtensorMap xmap,
                      const __grid_constant__ CUtensorMap wmap) {
    using namespace cb;
    using C = Cfg<CG>;
    constexpr int S = C::kStages;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    uint8_t* epi = smem + S * C::kStageBytes;
    uint64_t* full = reinterpret_cast<uint64_t*>(epi + kEpiWarps * kEpiBuf);
    uint64_t* empty = full + S;
    uint64_t* acc_full = empty + S;     // [2]: accumulator b holds a finished tile
    uint64_t* acc_empty = acc_full + 2;  // [2]: accumulator b has been read
    uint64_t* mma_done = acc_empty + 2;
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(mma_done + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
    volatile int* issued = abort_flag + 1;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = CG == 1 ? 0u : cta_rank();  // rank 0 issues the pair's MMAs

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);  // CG = 2: rank 0's counts the bytes of both CTAs
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], kEpiWarps * CG);  // the epilogue warps of every CTA of the group
        }
        mbar_init(mma_done, 1);
        *abort_flag = 0;
        *issued = 0;
        fence_mbar_init();
    }
    if (warp == 0) {  // the whole warp allocates (and later frees) the accumulator columns
        if constexpr (CG == 1) {
            asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                             smem_u32(tmem_holder)),
                         "r"(kTmemCols));
            asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
        } else {
            asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                             smem_u32(tmem_holder)),
                         "r"(kTmemCols));
            asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;");
        }
    }
    fence_before();
    __syncthreads();
    if constexpr (CG == 2) cluster_sync();  // the pair's barriers exist before either CTA signals the other
    fence_after();
    const uint32_t tmem = *tmem_holder;
    const int ntiles = a.TM * a.TN;  // TM: tiles of 128 * CG activation rows
    const int tile0 = blockIdx.x / CG, tstep = gridDim.x / CG;
    griddep_wait();  // x comes from the previous kernels
    // No CTA of this grid waits for another: a dependent launch may take SMs as CTAs leave them (it
    // reads nothing of ours before its own wait).
    griddep_launch_dependents();

    if (warp == 0) {
        if (lane == 0) {
            int it = 0;
            for (int tile = tile0; tile < ntiles && !*abort_flag; tile += tstep) {
                const int tn = tile / a.TM, tm = tile % a.TM;  // groups at work together share weight tiles
                const int xrow = (tm * CG + (int)rank) * kRows;
                for (int ks = 0; ks < a.KS; ++ks, ++it) {
                    const int s = it % S;
                    if (it >= S && !mbar_wait_bounded(&empty[s], ((it / S) - 1) & 1)) {
                        atomicOr(a.status, 1u);
                        *abort_flag = 1;
                        break;
                    }
                    uint8_t* st = smem + s * C::kStageBytes;
                    if constexpr (CG == 1) {
                        mbar_arrive_expect_tx(&full[s], C::kStageBytes);
                        tma_load_2d(st, &xmap, ks * kKStage, xrow, &full[s]);
                        tma_load_4d(st + kABytes, &wmap, 0, ks, tn, &full[s]);
                    } else {
                        if (rank == 0) mbar_arrive_expect_tx(&full[s], 2 * C::kStageBytes);
                        tma_load_2d_pair(st, &xmap, ks * kKStage, xrow, &full[s]);
                        tma_load_4d_pair(st + kABytes, &wmap, (int)rank * C::kBRows, ks, tn, &full[s]);
                    }
                    *issued = it + 1;
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && rank == 0) {
            // bf16 x bf16 -> fp32, both operands K-major, M = 128 * CG, N = 256
            const uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(kCols >> 3) << 17) |
                                   ((uint32_t)((kRows * CG) >> 4) << 24);
            int it = 0, tcount = 0;
            for (int tile = tile0; tile < ntiles && !*abort_flag; tile += tstep, ++tcount) {
                const int ab = tcount & 1;  // accumulator of this tile
                if (tcount >= 2) {          // its previous tile (tcount - 2) has been read out
                    if (!mbar_wait_bounded(&acc_empty[ab], ((tcount - 2) >> 1) & 1)) {
                        atomicOr(a.status, 1u);
                        *abort_flag = 1;
                        break;
                    }
                    fence_after();
                }
                const uint32_t dacc = tmem + (uint32_t)(ab * kCols);
                bool ok = true;
                for (int ks = 0; ks < a.KS; ++ks, ++it) {
                    const int s = it % S;
                    if (!mbar_wait_bounded(&full[s], (it / S) & 1)) {
                        ok = false;
                        break;
                    }
                    fence_after();
                    const uint32_t sa = smem_u32(smem + s * C::kStageBytes), sb = sa + kABytes;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)  // K = 16 per MMA: 32 bytes along the swizzled row
                        mma_bf16<CG>(dacc, sdesc_sw128(sa + kk * 32), sdesc_sw128(sb + kk * 32), idesc,
                                     (ks > 0 || kk > 0) ? 1u : 0u);
                    commit<CG>(&empty[s]);  // frees the stage in every CTA of the group
                }
                if (!ok) {
                    atomicOr(a.status, 1u);
                    *abort_flag = 1;
                    break;
                }
                commit<CG>(&acc_full[ab]);
            }
            commit_self<CG>(mma_done);  // every tcgen05 operation of this thread completes before teardown
            if (!mbar_wait_bounded(mma_done, 0)) atomicOr(a.status, 1u);
        }
    } else {  // epilogue: TMEM lane quarter = warp % 4, all 256 columns of this CTA's 128 rows
        const int q = warp & 3;
        const uint32_t lane_base = (uint32_t)(q * 32) << 16;
        uint8_t* tb = epi + (warp - kFirstEpi) * kEpiBuf;
        const float gs = *a.gscale;  // written by the packing kernel, before this launch
        int tcount = 0;
        for (int tile = tile0; tile < ntiles; tile += tstep, ++tcount) {
            const int ab = tcount & 1;
            if (*abort_flag || !mbar_wait_bounded(&acc_full[ab], (tcount >> 1) & 1)) {
                if (lane == 0) atomicOr(a.status, 1u);
                *abort_flag = 1;
                break;
            }
            fence_after();
            const int tn = tile / a.TM, tm = tile % a.TM;
            const int m0 = (tm * CG + (int)rank) * kRows + q * 32;  // this warp's first row
            const int64_t n0 = (int64_t)tn * kCols;
#pragma unroll 1
            for (int c = 0; c < kCols; c += 32) {
                float v[32];
                ld32(tmem + lane_base + (uint32_t)(ab * kCols + c), v);
                if (c == kCols - 32) {  // this warp's columns are read: release the accumulator
                    fence_before();
                    __syncwarp();
                    if (lane == 0) {
                        if (CG == 1 || rank == 0)
                            mbar_arrive_local(&acc_empty[ab]);
                        else
                            mbar_arrive_remote(&acc_empty[ab], 0);
                    }
                }
                if (m0 >= a.M || n0 + c >= a.N) continue;
                // Transpose through shared memory so that each store instruction writes 8 rows x
                // 64 contiguous bytes instead of 32 rows x 16 bytes.
#pragma unroll
                for (int h = 0; h < 2; ++h) {
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        *reinterpret_cast<float4*>(tb + lane * 64 + ((j ^ (lane & 3)) << 4)) =
                            make_float4(v[16 * h + 4 * j] * gs, v[16 * h + 4 * j + 1] * gs,
                                        v[16 * h + 4 * j + 2] * gs, v[16 * h + 4 * j + 3] * gs);
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
    if (warp == 0 && lane == 0 && *abort_flag) {
        // wait (bounded) for the last tensor loads issued to land before shared memory is released
        // (CG = 2: they complete on rank 0's barriers; rank 1 waits out the same bound instead)
        const int n_it = *issued;
        for (int j = n_it > S ? n_it - S : 0; j < n_it; ++j) {
            if (CG == 1 || rank == 0)
                mbar_wait_bounded(&full[j % S], (j / S) & 1, 50000000ull);
        }
        if (CG == 2 && rank != 0) {
            const uint64_t t0 = globaltimer_ns();
            while (globaltimer_ns() - t0 < 50000000ull) __nanosleep(1000);
        }
    }
    // CG = 2: the pair's MMAs read both CTAs' shared memory and write both CTAs' tensor memory;
    // neither CTA frees either before the issuing CTA has seen them complete (mma_done above).
    if constexpr (CG == 2) cluster_sync();
    if (warp == 0) {
        __syncwarp();
        fence_after();
        if constexpr (CG == 1)
            asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols));
        else
            asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols));
    }
}

}  // namespace qlin

using namespace qlin;

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link-time libcuda dependency).
static PFN_cuTensorMapEncodeTiled_v12000 bf16_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static bool tried = false;
    if (!tried) {
        tried = true;
        void* p = nullptr;
        cudaDriverEntryPointQueryResult qr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &qr) == cudaSuccess &&
            qr == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

// A bf16 matrix {cols (inner), rows} with a row pitch of `pitch` elements, read in boxes of 64
// columns (128 bytes) x box_rows rows with the 128-byte swizzle; out-of-range elements read as 0.
static bool make_bf16_map(CUtensorMap* map, const void* base, int64_t rows, int64_t cols, int64_t pitch,
                          int box_rows) {
    PFN_cuTensorMapEncodeTiled_v12000 enc = bf16_map_encoder();
    if (!enc) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)pitch * 2};
    const cuuint32_t box[2] = {(cuuint32_t)cb::kKStage, (cuuint32_t)box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Columns of the bf16 weight copy: K rounded up to whole 64-value stages (zero-filled).
extern "C" int64_t qlin_bf16_cache_cols(int64_t K) { return (K + cb::kKStage - 1) / cb::kKStage * cb::kKStage; }
// Bytes of the bf16 weight copy: blocks of 256 rows x 64 values, N rounded up to 256 (zero rows).
extern "C" int64_t qlin_bf16_cache_bytes(int64_t N, int64_t K) {
    return (N + cb::kCols - 1) / cb::kCols * cb::kCols * qlin_bf16_cache_cols(K) * 2;
}

// The blocked weight copy as a 4-D bf16 tensor {64 values, 256 rows, Kc / 64 k-blocks, Np / 256 row
// blocks}, read in boxes of 64 values x box_rows rows with the 128-byte swizzle.
static bool make_wblock_map(CUtensorMap* map, const void* base, int64_t N, int64_t K, int box_rows) {
    PFN_cuTensorMapEncodeTiled_v12000 enc = bf16_map_encoder();
    if (!enc) return false;
    const int64_t kb = qlin_bf16_cache_cols(K) / cb::kKStage, nb = (N + cb::kCols - 1) / cb::kCols;
    const cuuint64_t dims[4] = {(cuuint64_t)cb::kKStage, (cuuint64_t)cb::kCols, (cuuint64_t)kb, (cuuint64_t)nb};
    const cuuint64_t strides[3] = {(cuuint64_t)cb::kKStage * 2, (cuuint64_t)cb::kCols * cb::kKStage * 2,
                                   (cuuint64_t)kb * cb::kCols * cb::kKStage * 2};
    const cuuint32_t box[4] = {(cuuint32_t)cb::kKStage, (cuuint32_t)box_rows, 1, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int CG>
static cudaError_t launch_bf16_cg(const cb::Args& a, const CUtensorMap& xmap, const CUtensorMap& wmap, int flags,
                                  cudaStream_t s) {
    using C = cb::Cfg<CG>;
    static bool attr_set = false;
    static int max_units = 0, cached_dev = -1;  // CTAs (CG = 1) or pairs (CG = 2) resident at once
    cudaError_t e;
    if (!attr_set) {
        e = cudaFuncSetAttribute(chunk_bf16_kernel<CG>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
    int dev = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[2];
    int na = 0;
    if (CG == 2) {
        attr[na].id = cudaLaunchAttributeClusterDimension;
        attr[na].val.clusterDim.x = 2;
        attr[na].val.clusterDim.y = 1;
        attr[na].val.clusterDim.z = 1;
        ++na;
    }
    cfg.blockDim = dim3(cb::kThreads);
    cfg.dynamicSmemBytes = C::kSmem;
    cfg.stream = s;
    cfg.attrs = attr;
    if (cached_dev != dev) {
        int sms = 0;
        if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
        int units = sms;
        if (CG == 2) {
            cfg.gridDim = dim3((unsigned)(sms & ~1));
            cfg.numAttrs = na;
            int clusters = 0;
            if ((e = cudaOccupancyMaxActiveClusters(&clusters, chunk_bf16_kernel<CG>, &cfg)) != cudaSuccess) return e;
            if (clusters < 1) return cudaErrorInvalidConfiguration;
            units = clusters;
        }
        max_units = units;
        cached_dev = dev;
    }
    const int ntiles = a.TM * a.TN;
    cfg.gridDim = dim3((unsigned)((ntiles < max_units ? ntiles : max_units) * CG));
    if (flags & QLIN_FLAG_PDL) {
        attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[na].val.programmaticStreamSerializationAllowed = 1;
        ++na;
    }
    cfg.numAttrs = na;
    return cudaLaunchKernelEx(&cfg, chunk_bf16_kernel<CG>, a, xmap, wmap);
}

// packed: the 256-byte header (its per-tensor scale multiplies every output), then the blocked bf16
// weights: for row block nb and k-block kb, 256 rows x 64 values at element
// ((nb * Kc / 64 + kb) * 256 + row) * 64;
// x: bf16 [M][K] with row pitch ldx (16-byte aligned base, ldx % 8 == 0, checked by the caller).
// QLIN_FLAG_CTA_PAIRS with M > 128: 256 x 256 tiles on pairs of CTAs.
extern "C" cudaError_t qlin_launch_chunk_bf16(const void* packed, int64_t N, int64_t K, const void* x, int M,
                                              int64_t ldx, float* y, int64_t ldy, void* ws, int flags,
                                              cudaStream_t s) {
    const int cg = (flags & QLIN_FLAG_CTA_PAIRS) && M > cb::kRows ? 2 : 1;
    const void* wb = reinterpret_cast<const uint8_t*>(packed) + kHdrBytes;
    cb::Args a;
    a.gscale = &reinterpret_cast<const PackedHeader*>(packed)->global_scale;
    a.y = y;
    a.ldy = ldy;
    a.M = M;
    a.N = N;
    a.K = K;
    a.TM = (M + cb::kRows * cg - 1) / (cb::kRows * cg);
    a.TN = (int)((N + cb::kCols - 1) / cb::kCols);
    a.KS = (int)(qlin_bf16_cache_cols(K) / cb::kKStage);
    a.status = (unsigned*)ws;
    CUtensorMap xmap, wmap;
    memset(&xmap, 0, sizeof(xmap));
    memset(&wmap, 0, sizeof(wmap));
    if (!make_bf16_map(&xmap, x, M, K, ldx, cb::kRows)) return cudaErrorInvalidValue;
    if (!make_wblock_map(&wmap, wb, N, K, cb::kCols / cg)) return cudaErrorInvalidValue;
    return cg == 2 ? launch_bf16_cg<2>(a, xmap, wmap, flags, s) : launch_bf16_cg<1>(a, xmap, wmap, flags, s);
}
