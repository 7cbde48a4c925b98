// chunk_gemm.cu -- NVFP4 prefill-chunk GEMM on the 5th-generation tensor cores (sm_100a).
//
// y[m][n] = (a_g * g_w) * sum_k A_q[m][k] * W_q[n][k], with A_q the NVFP4-quantized activations
// and W_q the NVFP4 weights, both as E2M1 codes with one E4M3 scale per 16 values.  The block
// scales are applied inside the MMA (tcgen05.mma kind::mxf4nvf4, block16), the per-tensor scales
// in the epilogue.  The pages' counterpart is imp's NVFP4 block-scaled GEMM for prefill (README
// "Features", row "sm_120a kernels", written there with mma.sync for sm_120a); this is the
// datacenter-Blackwell form: TMEM accumulators, smem descriptors, a single thread issuing MMAs.
//
// One launch, persistent CTAs (one per SM):
//   phase Q (all warps of all CTAs): max |x| over the whole tensor (one atomicMax per CTA), a
//            bounded grid-wide barrier, a_g, then every CTA quantizes its share of the
//            (row, 16-value block) items into the MMA operand layout, taken unit by unit, and
//            counts them into a per-unit ready counter (no second grid barrier: each producer
//            waits only for the units of its own tiles).
//   phase G (warp roles), over output tiles of 128 * CG activation rows x 256 weight rows:
//     warp 0   : producer -- bulk copies of one A unit (128 rows x 256 values + scales, 18 KB) and
//                this CTA's part of one W unit (CG = 1: 256 rows, 36 KB; CG = 2: 128 rows' codes
//                plus all 256 rows' scales, 20 KB) per stage into a shared-memory ring;
//     warp 1   : (CG = 1, or rank 0 of a pair) one thread issues the stage's 4 block-scaled MMAs
//                (K = 64 each), commits the stage back to every CTA of the group and, after the
//                tile's last stage, the accumulator to the epilogues; (rank 1 of a pair) one thread
//                tells rank 0 when a stage of this CTA is ready (data landed, scales written);
//     warps 2-5: scale-factor writers -- move the stage's E4M3 scales from shared memory into
//                tensor memory with tcgen05.st (one TMEM lane quarter each), off the tensor pipe;
//     warps 6-9: epilogue -- tcgen05.ld of the 128 x 256 fp32 accumulator, 32 columns at a time,
//                released to the MMAs as soon as it has been read; scaled values leave through
//                shared memory, as TMA tensor stores of 32 x 32 boxes (CG = 2, 16-byte aligned y)
//                or as row-contiguous plain stores.
// Every wait is bounded; a timeout sets the status word and the CTA winds down.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "chunk_common.cuh"

namespace qlin {

constexpr int kAccCols = 256;

// CG = 1: one CTA per 128 x 256 output tile (tcgen05 cta_group::1, M = 128).
// CG = 2: a cluster of two CTAs per 256 x 256 tile (cta_group::2, M = 256): each CTA holds its
//         128 activation rows and half of the 256 weight rows; the tensor cores of the pair
//         exchange the halves, so each SM streams 38 KB per k-group instead of 54 KB.
// MX = false: NVFP4 operands (E4M3 scales of 16 values); MX = true: MXFP4 operands (UE8M0 scales of
// 32 values, half the scale bytes).  The stage layout is the same; MXFP4 copies fewer scale bytes.
template <int CG, bool MX = false>
struct ChunkCfg {
    static constexpr int kWCodes = 32768 / CG;                      // weight code bytes per CTA per k-group
    static constexpr int kStageBytes = kMmaAUnit + kWCodes + 4096;  // + all 256 weight rows' scales
    static constexpr int kAScale = MX ? 1024 : 2048;                 // activation scale bytes per k-group
    static constexpr int kWScale = MX ? 2048 : 4096;                 // weight scale bytes (256 rows)
    static constexpr int kScaleBytes = kAScale + kWScale;            // completes on the scale barrier
    static constexpr int kCodeBytes = kMmaARows * 128 + kWCodes;
    static constexpr int kStages = CG == 1 ? 4 : 5;
    static constexpr int kRingBytes = kStages * kStageBytes;
    static constexpr int kSfCols = MX ? 24 : 48;  // TMEM columns of one stage's scale factors
};
static_assert(ChunkCfg<1>::kStageBytes % 1024 == 0 && ChunkCfg<2>::kStageBytes % 1024 == 0, "stage alignment");
// Epilogue warps 6-9, each with a staging box of kBoxRows rows x 32 fp32 columns (128-byte rows,
// 128B-swizzled) for TMA tensor stores; the same buffer serves as a 32 x 16 transpose buffer
// when y is not 16-byte aligned.  CG = 1 leaves room for 16-row boxes beside its 4-stage ring.
template <int CG>
struct EpiCfg {
    static constexpr int kWarps = 4;
    static constexpr int kFirstWarp = 6;
    static constexpr int kCols = kAccCols;  // accumulator columns per warp
    static constexpr int kBoxRows = CG == 1 ? 16 : 32;
    static constexpr int kBuf = kBoxRows * 128;
    static constexpr int kBytes = kWarps * kBuf;
};
template <int CG>
constexpr int chunk_smem() { return 1024 + ChunkCfg<CG>::kRingBytes + EpiCfg<CG>::kBytes + 512; }
constexpr int kChunkThreads = 320;
constexpr int kTmemCols = 512;
constexpr int kSfCols = 48;  // per stage, NVFP4: 4 k-blocks x (4 SFA + 8 SFB) columns (MXFP4: 2 spans, 24)
constexpr int kQItems = 8;   // activation items held in registers per thread in phase Q
static_assert(kAccCols + ChunkCfg<1>::kStages * kSfCols <= kTmemCols, "TMEM budget");
static_assert(kAccCols + ChunkCfg<2>::kStages * kSfCols <= kTmemCols, "TMEM budget");
static_assert(chunk_smem<1>() <= 232448 && chunk_smem<2>() <= 232448, "shared memory budget");

// workspace words (after the status word): amax accumulator, barrier counter, a_g, exit counter
constexpr int kWAmax = 0, kWArrive1 = 1, kWAg = 2, kWExit = 4;
constexpr int kUnitItems = kMmaARows * 16;  // (row, 16-value block) items of one 128 x 256 operand unit

struct ChunkArgs {
    const uint8_t* w;   // QLIN_PACK_MMA buffer (header + units)
    const __nv_bfloat16* x;
    int64_t ldx;
    uint8_t* aq;        // quantized activations (units), in the workspace
    unsigned* words;
    unsigned* ready;    // per activation unit: items quantized so far (kUnitItems when complete)
    float* y;
    int64_t ldy;
    int M;
    int64_t N, K;
    int T2, G, TM;  // TM: 128-row activation units (a multiple of CG)
    int KS, GS;     // k-splits per output tile (1 or 2) and k-groups per split
    int xvec, yvec, tma_store;  // yvec: y 16-byte aligned with a row pitch of a multiple of 4 floats
    unsigned* status;
    // Grouped mode (the MoE prefill), tile_expert != nullptr, single CTAs, no k-split: the rows of x
    // are sorted by expert, each expert's rows padded to whole 128-row tiles; row tile tm belongs to
    // expert tile_expert[tm], the first *used_tm row tiles are in use (written by an earlier kernel
    // of the stream), and expert e's packed weights (header included) start at w + e * w_stride.
    const int* tile_expert;
    const int* tile_rows;  // rows of tile tm that hold data (the epilogue stores no others)
    const int* used_tm;
    int64_t w_stride;
    // SiLU-gate epilogue (h != nullptr; weights packed with QLIN_PACK_GATE_UP, so accumulator columns
    // 0..127 are the gate and 128..255 the up rows of outputs 128 t2 .. 128 t2 + 127): h[m][i] =
    // bf16(silu(g) * u) for i < h_cols, row pitch ldh; y is not written.
    __nv_bfloat16* h;
    int64_t ldh, h_cols;
    // Grouped mode: aq already holds the quantized operand (written by an earlier kernel of the
    // stream); amax_in: the max |x| it was quantized with (the bits of a non-negative float; NVFP4's
    // a_g follows from it).  amax_out != nullptr (SiLU-gate epilogue): max |h| over the stored bf16
    // values is folded in with atomicMax.
    const unsigned* amax_in;
    unsigned* amax_out;
};

// silu(z) = z * sigmoid(z) with e = exp(-|z|) = 2^(-|z| log2 e) from the MUFU ex2 unit and the
// reciprocal from the MUFU rcp unit (each within about 2^-22 relative; the rounding of the argument
// adds |z| 2^-23 relative to e; subnormal e flushes to 0).  The result is rounded to bf16 (2^-9
// relative) right after, so the approximations cost nothing visible while taking the epilogue from
// ~25 instructions per output (IEEE exp and division) to ~6.
__device__ __forceinline__ float chunk_silu(float z) {
    float e, r;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(e) : "f"(-fabsf(z) * 1.44269504088896341f));
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(1.0f + e));
    return z * (z >= 0.f ? r : e * r);
}

__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr) {
    uint64_t d = (uint64_t)((saddr >> 4) & 0x3fffu);
    d |= (uint64_t)1 << 16;             // leading byte offset (unused for swizzled K-major)
    d |= (uint64_t)(1024 >> 4) << 32;   // stride byte offset: 8-row groups 1024 B apart
    d |= (uint64_t)1 << 46;             // descriptor version for sm_100
    d |= (uint64_t)2 << 61;             // 128-byte swizzle
    return d;
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
template <int O, int R>
__device__ __forceinline__ void tc_st16(uint32_t taddr, const uint32_t (&r)[R]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
            taddr),
        "r"(r[O + 0]), "r"(r[O + 1]), "r"(r[O + 2]), "r"(r[O + 3]), "r"(r[O + 4]), "r"(r[O + 5]), "r"(r[O + 6]),
        "r"(r[O + 7]), "r"(r[O + 8]), "r"(r[O + 9]), "r"(r[O + 10]), "r"(r[O + 11]), "r"(r[O + 12]), "r"(r[O + 13]),
        "r"(r[O + 14]), "r"(r[O + 15])
        : "memory");
}

__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, const void* src, int x, int y) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(x), "r"(y), "r"(smem_u32(src))
                 : "memory");
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// The same box added element-wise into global memory (f32 add, the tensor map's type).
__device__ __forceinline__ void tma_add_2d(const CUtensorMap* map, const void* src, int x, int y) {
    asm volatile("cp.reduce.async.bulk.tensor.2d.global.shared::cta.add.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(x), "r"(y), "r"(smem_u32(src))
                 : "memory");
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_read_all() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ unsigned ld_acquire_gpu(const unsigned* p) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ unsigned ld_relaxed_gpu(const unsigned* p) {
    unsigned v;
    asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void fence_proxy_async_global() {
    asm volatile("fence.proxy.async.global;" ::: "memory");
}

// Grid-wide barrier on a counter that only grows within one launch (reset by the last CTA out).
// Called by one thread per CTA; false after ~2 s (or the workspace's wait budget) without all
// CTAs arriving.
__device__ __forceinline__ bool grid_arrive_wait(unsigned* counter, unsigned target, const void* ws) {
    __threadfence();
    atomicAdd(counter, 1u);
    if (ld_acquire_gpu(counter) >= target) return true;
    const uint64_t t0 = globaltimer_ns(), budget = ws_wait_budget_ns(ws);
    for (uint32_t it = 1;; ++it) {
        if (ld_acquire_gpu(counter) >= target) return true;
        if (globaltimer_ns() - t0 > budget) return false;
        __nanosleep(64);
    }
}


// ------------------------------------------------------------------ CTA-pair helpers (CG = 2)
__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
// All threads of both CTAs of the cluster.
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Arrive on the mbarrier at the same shared-memory offset in CTA `rank` of the cluster.
__device__ __forceinline__ void mbar_arrive_cluster(uint64_t* bar, uint32_t rank) {
    asm volatile(
        "{\n .reg .b32 ra;\n mapa.shared::cluster.u32 ra, %0, %1;\n"
        " mbarrier.arrive.release.cluster.shared::cluster.b64 _, [ra];\n}\n" ::"r"(smem_u32(bar)),
        "r"(rank)
        : "memory");
}
__device__ __forceinline__ bool mbar_try_wait_cluster(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n"
        " selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
// Bounded wait that also acquires what the other CTA of the pair released before arriving.
__device__ __forceinline__ bool mbar_wait_cluster_bounded(uint64_t* bar, uint32_t parity) {
    if (mbar_try_wait_cluster(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait_cluster(bar, parity)) return true;
        if ((it & 255u) == 0 && globaltimer_ns() - t0 > 2000000000ull) return false;
    }
}

// MXFP4 x MXFP4 with UE8M0 scales of 32 values (kind::mxf4, scale_vec::2X); the scale byte pair of
// this K = 64 step is selected by the scale-factor ids of idesc and the top two bits of sfa / sfb.
template <int CG>
__device__ __forceinline__ void tc_mma_mx_cg(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                             uint32_t sfa, uint32_t sfb, uint32_t accumulate) {
    if constexpr (CG == 1)
        asm volatile(
            "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
            " tcgen05.mma.cta_group::1.kind::mxf4.block_scale.block32 [%0], %1, %2, %3, [%5], [%6], p;\n}\n" ::"r"(d_tmem),
            "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
            : "memory");
    else
        asm volatile(
            "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
            " tcgen05.mma.cta_group::2.kind::mxf4.block_scale.block32 [%0], %1, %2, %3, [%5], [%6], p;\n}\n" ::"r"(d_tmem),
            "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
            : "memory");
}

// 8 consecutive 32-bit TMEM columns of this warp's lane quarter from r[O .. O+7] of each thread.
template <int O, int R>
__device__ __forceinline__ void tc_st8(uint32_t taddr, const uint32_t (&r)[R]) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr), "r"(r[O + 0]),
                 "r"(r[O + 1]), "r"(r[O + 2]), "r"(r[O + 3]), "r"(r[O + 4]), "r"(r[O + 5]), "r"(r[O + 6]),
                 "r"(r[O + 7])
                 : "memory");
}

template <int CG>
__device__ __forceinline__ void tc_mma_cg(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t sfa, uint32_t sfb, uint32_t accumulate) {
    if constexpr (CG == 1) {
        tc_mma(d_tmem, adesc, bdesc, idesc, sfa, sfb, accumulate);
    } else {
        asm volatile(
            "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
            " tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n}\n" ::"r"(
                d_tmem),
            "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
            : "memory");
    }
}
// Commit this thread's MMAs to the mbarrier at `bar` in every CTA of the group.
template <int CG>
__device__ __forceinline__ void tc_commit_cg(uint64_t* bar) {
    if constexpr (CG == 1) {
        tc_commit(bar);
    } else {
        asm volatile(
            "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
                smem_u32(bar)),
            "h"((uint16_t)3)
            : "memory");
    }
}
// Commit to this CTA's own mbarrier only.
template <int CG>
__device__ __forceinline__ void tc_commit_self(uint64_t* bar) {
    if constexpr (CG == 1)
        tc_commit(bar);
    else
        asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                     : "memory");
}
template <int CG>
__device__ __forceinline__ void tmem_alloc(uint32_t* holder) {
    if constexpr (CG == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(holder)),
                     "r"(kTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    } else {
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(holder)),
                     "r"(kTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;");
    }
}
template <int CG>
__device__ __forceinline__ void tmem_free(uint32_t tmem) {
    if constexpr (CG == 1)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols));
    else
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols));
}

// GR: grouped mode (the MoE prefill; CG = 1): pre-quantized activations, per-tile expert weights,
// the optional SiLU-gate epilogue.  The plain chunk GEMM (GR = false) carries none of that code.
template <int CG, bool MX, bool GR>
__global__ void __launch_bounds__(kChunkThreads, 1) chunk_gemm_kernel(const ChunkArgs a,
                                                                       const __grid_constant__ CUtensorMap ymap) {
    using Cfg = ChunkCfg<CG, MX>;
    using Epi = EpiCfg<CG>;
    constexpr int S = Cfg::kStages;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    uint8_t* epi = smem + Cfg::kRingBytes;
    uint64_t* full = reinterpret_cast<uint64_t*>(epi + Epi::kBytes);
    uint64_t* empty = full + S;
    uint64_t* sfready = empty + S;  // this CTA's scale writers are done with the stage
    uint64_t* pfull = sfready + S;  // CG = 2, rank 0: the other CTA's stage is ready
    uint64_t* sfull = pfull + S;    // the stage's scale bytes have landed (the codes: full)
    uint64_t* acc_full = sfull + S;
    uint64_t* acc_empty = acc_full + 1;
    uint64_t* mma_done = acc_empty + 1;
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(mma_done + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
    volatile int* issued = abort_flag + 1;
    volatile float* ag_sm = reinterpret_cast<volatile float*>(issued + 1);
    float* red = const_cast<float*>(ag_sm + 1);  // one partial max per warp
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = CG == 1 ? 0u : cluster_ctarank();  // rank 0 issues the pair's MMAs

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
            mbar_init(&sfready[s], 4);
            mbar_init(&pfull[s], 1);
            mbar_init(&sfull[s], 1);
        }
        mbar_init(acc_full, 1);
        mbar_init(acc_empty, Epi::kWarps * CG);  // the epilogue warps of every CTA of the group
        mbar_init(mma_done, 1);
        *abort_flag = 0;
        *issued = 0;
        fence_mbar_init();
    }
    if (warp == 0) tmem_alloc<CG>(tmem_holder);  // the whole warp allocates (and later frees) tensor memory
    tc_fence_before();
    __syncthreads();
    if constexpr (CG == 2) cluster_sync_all();  // the pair's barriers exist before either CTA signals the other
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;
    const int TMA = GR ? *a.used_tm : a.TM;  // activation row tiles in use
    const int TMP = TMA / CG;  // activation tiles of 128 * CG rows
    const int ntiles = a.T2 * TMP * a.KS;
    const int tile0 = blockIdx.x / CG, tstep = gridDim.x / CG;
    // Work item `tile`: weight tile t2, activation tile tm (this CTA's 128 rows of it) and the
    // k-groups [g0, g1) of split tile % KS.  With KS = 2 the two halves of an output tile add into
    // y, which phase Q zeroes: two addends onto zero give the same sum in either order.
    auto tile_of = [&](int tile, int& t2, int& tm, int& g0, int& g1) {
        const int ks = tile % a.KS, rest = tile / a.KS;
        t2 = rest / TMP;
        tm = (rest % TMP) * CG + (int)rank;
        g0 = ks * a.GS;
        g1 = g0 + a.GS < a.G ? g0 + a.GS : a.G;
    };
    // Packed weights of the expert of row tile tm (grouped mode), else of the one matrix.
    auto wbase = [&](int tm) -> const uint8_t* {
        if constexpr (GR)
            return a.w + (int64_t)a.tile_expert[tm] * a.w_stride;
        else
            return a.w;
    };
    // The weights do not depend on x: the producer starts the first stages' weight copies now, so
    // they land during phase Q (the stage barriers also expect the activation bytes, copied once
    // quantized).
    // A stage's copies: the scale bytes (2 KB of the activation unit, 4 KB of the weight unit)
    // complete on sfull, so the scale writers start before the 48 KB (or 32 KB) of codes land.
    auto expect_stage = [&](int s) {
        mbar_arrive_expect_tx(&full[s], Cfg::kCodeBytes);
        mbar_arrive_expect_tx(&sfull[s], Cfg::kScaleBytes);
    };
    auto copy_w = [&](uint8_t* st, const uint8_t* wu, int s) {
        bulk_g2s(st + kMmaAUnit + Cfg::kWCodes, wu + kMmaWRows * 128, Cfg::kWScale, &sfull[s]);
        bulk_g2s(st + kMmaAUnit, wu + rank * Cfg::kWCodes, Cfg::kWCodes, &full[s]);
    };
    auto copy_a = [&](uint8_t* st, const uint8_t* au, int s) {
        bulk_g2s(st + kMmaARows * 128, au + kMmaARows * 128, Cfg::kAScale, &sfull[s]);
        bulk_g2s(st, au, kMmaARows * 128, &full[s]);
    };
    int npre = 0;  // stages of the first tile whose weight part is already in flight (thread 0)
    if (threadIdx.x == 0 && tile0 < ntiles) {
        int t2, tm, g0, g1;
        tile_of(tile0, t2, tm, g0, g1);
        npre = g1 - g0 < S ? g1 - g0 : S;
        for (int it = 0; it < npre; ++it) {
            uint8_t* st = smem + it * Cfg::kStageBytes;
            const uint8_t* wu = wbase(tm) + kHdrBytes + ((int64_t)t2 * a.G + g0 + it) * kMmaWUnit;
            expect_stage(it);
            copy_w(st, wu, it);
        }
        *issued = npre;  // in flight (the abort path waits for them, bounded)
    }
    griddep_wait();  // x comes from the previous kernels

    // ---------------------------------------------------------------- phase Q: quantize x
    // Items in unit-major order: item i belongs to unit u = i / kUnitItems (u = tm * G + g), row
    // (i % kUnitItems) / 16 of the unit's 128 and 16-value block i % 16 of its k-group.  When every
    // thread has at most kQItems items, they stay in registers between the max pass and the
    // quantization (x is read once, all loads in flight together); otherwise x is read twice.
    // Grouped mode: the operand was quantized by an earlier kernel; only a_g is taken here.
    if constexpr (GR) {
        if (threadIdx.x == 0) *ag_sm = MX ? 1.0f : act_global_scale(__uint_as_float(__ldcg(a.amax_in)));
        __syncthreads();
        griddep_launch_dependents();
    } else {
        const int64_t gtid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
        const int64_t gthreads = (int64_t)gridDim.x * blockDim.x;
        const int64_t items = (int64_t)TMA * a.G * kUnitItems;
        const bool resident = items <= gthreads * kQItems;
        const bool vec = a.xvec != 0;
        auto item_mb = [&](int64_t i, int& m, int64_t& b) {
            const int64_t u = i / kUnitItems;
            const int within = (int)(i - u * kUnitItems);
            const int64_t tm = u / a.G;
            m = (int)(tm * kMmaARows) + (within >> 4);
            b = (u - tm * a.G) * 16 + (within & 15);
        };
        uint32_t xw[kQItems][8];
        float bmax[kQItems];
        float m = 0.f;
        if (resident) {
#pragma unroll
            for (int j = 0; j < kQItems; ++j) {
                const int64_t i = gtid + j * gthreads;
                int mj = 0;
                int64_t bj = 0;
                if (i < items) item_mb(i, mj, bj);
                act_load_item(a.x, i < items ? a.M : 0, a.K, a.ldx, vec, mj, bj, xw[j]);
            }
#pragma unroll
            for (int j = 0; j < kQItems; ++j) {
                bmax[j] = act_item_amax(xw[j]);
                m = fmaxf(m, bmax[j]);
            }
        } else {
            m = act_amax_partial(a.x, a.M, a.K, a.ldx, vec, gtid, gthreads);
        }
        // The per-unit ready counters start from zero: cleared here, before the grid barrier that
        // orders every CTA's increments after them.  (Their place in the workspace depends on the
        // shape, so what a call with other shapes left there is not zero.)
        for (int64_t u = gtid; u < (int64_t)a.TM * a.G; u += gthreads) a.ready[u] = 0u;
        __threadfence();
        if (a.KS > 1) {  // the k-split halves add into y: zero it (ordered before them by the barrier)
            const int64_t nq = (a.N + 3) / 4;
            for (int64_t i = gtid; i < (int64_t)a.M * nq; i += gthreads) {
                const int64_t row = i / nq, c = (i - row * nq) * 4;
                float* dst = a.y + row * a.ldy + c;
                if (a.yvec && c + 4 <= a.N)
                    *reinterpret_cast<float4*>(dst) = make_float4(0.f, 0.f, 0.f, 0.f);
                else
                    for (int u = 0; u < 4 && c + u < a.N; ++u) dst[u] = 0.f;
            }
        }
        for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if (lane == 0) red[warp] = m;
        __syncthreads();
        if (threadIdx.x == 0) {
            float b = 0.f;
            for (int w = 0; w < kChunkThreads / 32; ++w) b = fmaxf(b, red[w]);
            atomicMax(&a.words[kWAmax], __float_as_uint(b));  // non-negative floats order as their bits
            float ag = 0.f;
            if (grid_arrive_wait(&a.words[kWArrive1], gridDim.x, a.status)) {
                ag = act_global_scale(__uint_as_float(ld_acquire_gpu(&a.words[kWAmax])));
                if (blockIdx.x == 0) a.words[kWAg] = __float_as_uint(ag);
            } else {
                atomicOr(a.status, 1u);
                *abort_flag = 1;
            }
            *ag_sm = MX ? 1.0f : ag;  // MXFP4 activations carry no per-tensor scale
        }
        __syncthreads();
        // Every CTA of this grid is resident (all passed the barrier): a dependent launch may now
        // take SMs as this grid's CTAs leave them; it reads nothing of ours before its own wait.
        griddep_launch_dependents();
        if (!*abort_flag) {
            const float ag = *ag_sm;
            // (the items of one warp are 32 consecutive indices and `items` is a multiple of 32, so
            // the MXFP4 pair shuffles below run with every lane of the warp)
            if (resident) {
#pragma unroll
                for (int j = 0; j < kQItems; ++j) {
                    const int64_t i = gtid + j * gthreads;
                    if constexpr (MX) {
                        const uint8_t byte = act_mx_pair_byte(bmax[j], act_item_special(xw[j]));
                        if (i < items) {
                            int mj;
                            int64_t bj;
                            item_mb(i, mj, bj);
                            uint32_t c8[2];
                            act_quant_item_mx_codes(xw[j], byte, c8);
                            act_store_item_mx(a.M, a.K, a.G, mj, bj, byte, c8, a.aq, nullptr, nullptr);
                        }
                    } else if (i < items) {
                        int mj;
                        int64_t bj;
                        item_mb(i, mj, bj);
                        uint32_t c8[2];
                        const uint8_t sc = act_quant_block(xw[j], bmax[j], ag, c8);
                        act_store_item(a.M, a.K, a.G, mj, bj, sc, c8, a.aq, nullptr, nullptr);
                    }
                }
            } else {
                for (int64_t i = gtid; i < items; i += gthreads) {
                    int mi;
                    int64_t bi;
                    item_mb(i, mi, bi);
                    if constexpr (MX) {
                        uint32_t w[8], c8[2];
                        act_load_item(a.x, a.M, a.K, a.ldx, vec, mi, bi, w);
                        const uint8_t byte = act_mx_pair_byte(act_item_amax(w), act_item_special(w));
                        act_quant_item_mx_codes(w, byte, c8);
                        act_store_item_mx(a.M, a.K, a.G, mi, bi, byte, c8, a.aq, nullptr, nullptr);
                    } else {
                        act_quant_item(a.x, a.M, a.K, a.ldx, a.G, ag, vec, mi, bi, a.aq, nullptr, nullptr);
                    }
                }
            }
            fence_proxy_async_global();  // the operand is read back by bulk copies (async proxy)
            __syncthreads();
            // This CTA's items form, per pass j, the range [blockIdx.x * 320 + j * gthreads, +320):
            // at most two units each.  Count them into the units' ready counters.
            if (threadIdx.x == 0) __threadfence();
            __syncthreads();
            const int64_t first = (int64_t)blockIdx.x * blockDim.x;
            const int64_t npass = first < items ? (items - first + gthreads - 1) / gthreads : 0;
            for (int64_t t = threadIdx.x; t < 2 * npass; t += blockDim.x) {
                const int64_t lo = first + (t >> 1) * gthreads;
                const int64_t hi = lo + blockDim.x < items ? lo + blockDim.x : items;
                const int64_t u0 = lo / kUnitItems, split = (u0 + 1) * kUnitItems;
                if ((t & 1) == 0) {
                    atomicAdd(&a.ready[u0], (unsigned)((hi < split ? hi : split) - lo));
                } else if (hi > split) {
                    atomicAdd(&a.ready[u0 + 1], (unsigned)(hi - split));
                }
            }
        }
        __syncthreads();
    }

    // ---------------------------------------------------------------- phase G: the GEMM
    if (warp == 0) {
        if (lane == 0) {
            fence_proxy_async_global();  // this thread's bulk copies read what phase Q wrote
            int it = 0;
            for (int tile = tile0; tile < ntiles && !*abort_flag; tile += tstep) {
                int t2, tm, g0, g1;
                tile_of(tile, t2, tm, g0, g1);
                if constexpr (!GR) {  // every unit of this tile's activation rows and k-groups quantized (bounded wait)
                    const unsigned* rd = a.ready + (int64_t)tm * a.G;
                    const uint64_t t0 = globaltimer_ns(), budget = ws_wait_budget_ns(a.status);
                    bool ready = false;
                    while (!ready) {
                        ready = true;
                        for (int g = g0; g < g1; ++g) ready &= ld_relaxed_gpu(rd + g) >= (unsigned)kUnitItems;
                        if (!ready) {
                            if (globaltimer_ns() - t0 > budget) break;
                            __nanosleep(64);
                        }
                    }
                    if (!ready) {
                        atomicOr(a.status, 1u);
                        *abort_flag = 1;
                        break;
                    }
                    __threadfence();             // acquire what the quantizing CTAs released
                    fence_proxy_async_global();  // ... for the bulk copies that read it
                }
                for (int g = g0; g < g1; ++g, ++it) {
                    const int s = it % S;
                    if (it >= S && !mbar_wait_bounded(&empty[s], ((it / S) - 1) & 1)) {
                        atomicOr(a.status, 1u);
                        *abort_flag = 1;
                        break;
                    }
                    uint8_t* st = smem + s * Cfg::kStageBytes;
                    const uint8_t* wu = wbase(tm) + kHdrBytes + ((int64_t)t2 * a.G + g) * kMmaWUnit;
                    if (it >= npre) {  // (the first stages' weights were started before phase Q)
                        expect_stage(s);
                        copy_w(st, wu, s);
                    }
                    copy_a(st, a.aq + ((int64_t)tm * a.G + g) * kMmaAUnit, s);
                    *issued = it + 1 > npre ? it + 1 : npre;
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && rank == 0) {
            // Instruction descriptor: E2M1 x E2M1, E4M3 scales (MXFP4: UE8M0, bit 23), K-major A and B,
            // M = 128 * CG, N = 256.
            const uint32_t idesc = (1u << 7) | (1u << 10) | ((uint32_t)(256 >> 3) << 17) |
                                   ((uint32_t)((128 * CG) >> 4) << 24) | (MX ? (1u << 23) : 0u);
            int it = 0, tcount = 0;
            for (int tile = tile0; tile < ntiles && !*abort_flag; tile += tstep, ++tcount) {
                if (tcount > 0) {
                    if (!mbar_wait_cluster_bounded(acc_empty, (tcount - 1) & 1)) {
                        atomicOr(a.status, 1u);
                        *abort_flag = 1;
                        break;
                    }
                    tc_fence_after();
                }
                int t2, tm, g0, g1;
                tile_of(tile, t2, tm, g0, g1);
                bool ok = true;
                for (int g = 0; g < g1 - g0; ++g, ++it) {
                    const int s = it % S;
                    const uint32_t par = (it / S) & 1;
                    if (!mbar_wait_bounded(&full[s], par) || !mbar_wait_bounded(&sfready[s], par) ||
                        (CG == 2 && !mbar_wait_cluster_bounded(&pfull[s], par))) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sa = smem_u32(smem + s * Cfg::kStageBytes);
                    const uint32_t sb = sa + kMmaAUnit;
#pragma unroll
                    for (int kb = 0; kb < 4; ++kb) {
                        if constexpr (MX) {
                            // span kb / 2 of the stage's scale columns (SFA 4, SFB 8); bytes 0-1 or 2-3
                            const uint32_t col = tmem + kAccCols + (uint32_t)(s * Cfg::kSfCols + (kb >> 1) * 12);
                            const uint32_t sid = (uint32_t)(kb & 1) * 2u;
                            tc_mma_mx_cg<CG>(tmem, sdesc_sw128(sa + kb * 32), sdesc_sw128(sb + kb * 32),
                                             idesc | (sid << 29) | (sid << 4), col | (sid << 30), (col + 4) | (sid << 30),
                                             (g > 0 || kb > 0) ? 1u : 0u);
                        } else {
                            const uint32_t col = tmem + kAccCols + (uint32_t)(s * kSfCols + kb * 12);  // SFA 4, SFB 8
                            tc_mma_cg<CG>(tmem, sdesc_sw128(sa + kb * 32), sdesc_sw128(sb + kb * 32), idesc, col,
                                          col + 4, (g > 0 || kb > 0) ? 1u : 0u);
                        }
                    }
                    tc_commit_cg<CG>(&empty[s]);  // frees the stage (smem and its scale columns) in every CTA
                }
                if (!ok) {
                    atomicOr(a.status, 1u);
                    *abort_flag = 1;
                    break;
                }
                tc_commit_cg<CG>(acc_full);
            }
            // every tcgen05 operation of this thread has completed before the CTAs wind down
            tc_commit_self<CG>(mma_done);
            if (!mbar_wait_bounded(mma_done, 0)) atomicOr(a.status, 1u);
        } else if (CG == 2 && lane == 0) {
            // rank 1: tell rank 0 when each stage of this CTA is ready (its scale writers waited for
            // the data before writing the scales)
            int it = 0;
            for (int tile = tile0; tile < ntiles && !*abort_flag; tile += tstep) {
                int t2, tm, g0, g1;
                tile_of(tile, t2, tm, g0, g1);
                bool ok = true;
                for (int g = g0; g < g1; ++g, ++it) {
                    const int s = it % S;
                    if (!mbar_wait_bounded(&sfready[s], (it / S) & 1)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_cluster(&pfull[s], 0);
                }
                if (!ok) {
                    atomicOr(a.status, 1u);
                    *abort_flag = 1;
                    break;
                }
            }
        }
    } else if (warp < Epi::kFirstWarp) {  // scale-factor writers: TMEM lane quarter = warp % 4
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        int it = 0;
        for (int tile = tile0; tile < ntiles && !*abort_flag; tile += tstep) {
            int t2, tm, g0, g1;
            tile_of(tile, t2, tm, g0, g1);
            bool ok = true;
            for (int g = g0; g < g1; ++g, ++it) {
                const int s = it % S;
                if (it >= S && !mbar_wait_bounded(&empty[s], ((it / S) - 1) & 1)) {
                    ok = false;
                    break;
                }
                if (!mbar_wait_bounded(&sfull[s], (it / S) & 1)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                // Atom layout (both operands): the 4 scales of row r (0..127 of a 128-row half) are
                // word r / 32 of 16-byte row r % 32.  Every lane quarter of TMEM gets the whole atom:
                // lane 32q + i, columns c..c+3 = the atom's 16-byte row i.  Each CTA holds the
                // scales of its own activation rows and of all 256 weight rows.
                // (MXFP4: the same, per 128-value span: 2 atoms of activation scales, 4 of weight scales)
                const uint8_t* st = smem + s * Cfg::kStageBytes;
                const uint8_t* sfa = st + kMmaARows * 128 + lane * 16;
                const uint8_t* sfb = st + kMmaAUnit + Cfg::kWCodes + lane * 16;
                constexpr int NB = MX ? 2 : 4;  // atoms of activation scales per stage
                uint32_t r[NB * 12];
#pragma unroll
                for (int kb = 0; kb < NB; ++kb) {
                    const uint4 va = lds128(sfa + kb * 512);
                    const uint4 vb0 = lds128(sfb + (kb * 2 + 0) * 512);
                    const uint4 vb1 = lds128(sfb + (kb * 2 + 1) * 512);
                    r[kb * 12 + 0] = va.x, r[kb * 12 + 1] = va.y, r[kb * 12 + 2] = va.z, r[kb * 12 + 3] = va.w;
                    r[kb * 12 + 4] = vb0.x, r[kb * 12 + 5] = vb0.y, r[kb * 12 + 6] = vb0.z, r[kb * 12 + 7] = vb0.w;
                    r[kb * 12 + 8] = vb1.x, r[kb * 12 + 9] = vb1.y, r[kb * 12 + 10] = vb1.z, r[kb * 12 + 11] = vb1.w;
                }
                const uint32_t cbase = tmem + lane_base + kAccCols + (uint32_t)(s * Cfg::kSfCols);
                if constexpr (MX) {
                    tc_st16<0>(cbase, r);
                    tc_st8<16>(cbase + 16, r);
                } else {
                    tc_st16<0>(cbase, r);
                    tc_st16<16>(cbase + 16, r);
                    tc_st16<32>(cbase + 32, r);
                }
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
    } else {  // epilogue: TMEM lane quarter = warp % 4
        const int q = warp & 3;
        const int c_lo = ((warp - Epi::kFirstWarp) >> 2) * Epi::kCols;  // this warp's first column
        const uint32_t lane_base = (uint32_t)(q * 32) << 16;
        float gw_ag = __fmul_rn(reinterpret_cast<const PackedHeader*>(a.w)->global_scale, *ag_sm);
        uint8_t* tb = epi + (warp - Epi::kFirstWarp) * Epi::kBuf;
        constexpr int R = Epi::kBoxRows;
        const bool tma = a.tma_store != 0;
        const bool add = a.KS > 1;  // k-split: add this half into y (zeroed in phase Q)
        if (add && lane == 0) fence_proxy_async_global();  // the zeroing stores before the TMA adds
        int tcount = 0, nstore = 0;
        float hmax = 0.f;  // max |h| over this thread's stored values (amax_out)
        for (int tile = tile0; tile < ntiles; tile += tstep, ++tcount) {
            int t2, tm, g0, g1;
            tile_of(tile, t2, tm, g0, g1);
            // grouped: this tile's expert's per-tensor scale and its rows holding data, loaded while
            // its MMAs run
            const float ws_g = GR ? reinterpret_cast<const PackedHeader*>(wbase(tm))->global_scale : 0.f;
            const int mlim = GR ? tm * kMmaARows + a.tile_rows[tm] : a.M;  // rows past it: not stored
            if (*abort_flag || !mbar_wait_bounded(acc_full, tcount & 1)) {
                if (lane == 0) atomicOr(a.status, 1u);
                *abort_flag = 1;
                break;
            }
            tc_fence_after();
            const int m0 = tm * kMmaARows + q * 32;  // this warp's first row
            const int64_t n0 = (int64_t)t2 * kMmaWRows;
            if (GR) gw_ag = __fmul_rn(ws_g, *ag_sm);
            if (GR && a.h) {
                // SiLU-gate epilogue: columns c (gate) and c + 128 (up) of output 128 t2 + c; this
                // thread's row m0 + lane; 32 outputs of one row per step, stored as bf16.
                const int row = m0 + lane;
#pragma unroll 1
                for (int c = 0; c < 128; c += 32) {
                    float g[32], u[32];
                    tc_ld32(tmem + lane_base + (uint32_t)c, g);
                    tc_ld32(tmem + lane_base + (uint32_t)(128 + c), u);
                    if (c == 96) {  // every column of this warp's rows is read: release them
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(acc_empty);
                    }
                    const int64_t i0 = (int64_t)t2 * 128 + c;
                    if (row >= mlim || i0 >= a.h_cols) continue;
                    __nv_bfloat16* dst = a.h + (int64_t)row * a.ldh + i0;
                    uint32_t pk[16];
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const float h0 = chunk_silu(g[2 * j] * gw_ag) * (u[2 * j] * gw_ag);
                        const float h1 = chunk_silu(g[2 * j + 1] * gw_ag) * (u[2 * j + 1] * gw_ag);
                        const __nv_bfloat162 hb = __floats2bfloat162_rn(h0, h1);
                        pk[j] = *reinterpret_cast<const uint32_t*>(&hb);
                        hmax = fmaxf(hmax, fmaxf(fabsf(__uint_as_float(pk[j] << 16)),
                                                 fabsf(__uint_as_float(pk[j] & 0xffff0000u))));
                    }
                    if (i0 + 32 <= a.h_cols && (reinterpret_cast<uintptr_t>(dst) & 15) == 0) {
#pragma unroll
                        for (int v = 0; v < 4; ++v)
                            reinterpret_cast<uint4*>(dst)[v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
                    } else {
                        for (int j = 0; j < 32 && i0 + j < a.h_cols; ++j)
                            dst[j] = __ushort_as_bfloat16((unsigned short)(pk[j >> 1] >> (16 * (j & 1))));
                    }
                }
                continue;
            }
#pragma unroll 1
            for (int c = c_lo; c < c_lo + Epi::kCols; c += 32) {
                float v[32];
                tc_ld32(tmem + lane_base + (uint32_t)c, v);
                if (c == c_lo + Epi::kCols - 32) {  // this warp's columns are read: release them
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) {
                        if (CG == 1 || rank == 0)
                            mbar_arrive(acc_empty);
                        else
                            mbar_arrive_cluster(acc_empty, 0);
                    }
                }
                if (m0 >= mlim || n0 + c >= a.N) continue;
                if (tma) {
                    // rows hh*R .. hh*R+R-1 of the warp's 32 as one R x 32 box; row r's 16-byte chunk j
                    // at position j ^ (r % 8) (the 128B swizzle of the tensor map)
#pragma unroll
                    for (int hh = 0; hh < 32 / R; ++hh) {
                        if (m0 + hh * R >= mlim) break;
                        if (lane == 0 && nstore > 0) bulk_wait_read_all();  // the previous store has read the box
                        __syncwarp();
                        if (lane / R == hh) {
                            const int r = lane % R;
#pragma unroll
                            for (int j = 0; j < 8; ++j)
                                *reinterpret_cast<float4*>(tb + r * 128 + ((j ^ (r & 7)) << 4)) =
                                    make_float4(v[4 * j] * gw_ag, v[4 * j + 1] * gw_ag, v[4 * j + 2] * gw_ag,
                                                v[4 * j + 3] * gw_ag);
                        }
                        fence_proxy_async_smem();
                        __syncwarp();
                        if (lane == 0) {
                            if (add)
                                tma_add_2d(&ymap, tb, (int)(n0 + c), m0 + hh * R);
                            else
                                tma_store_2d(&ymap, tb, (int)(n0 + c), m0 + hh * R);
                        }
                        ++nstore;
                    }
                    continue;
                }
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
                        if (mrow < mlim && ncol < a.N) {
                            float* dst = a.y + (int64_t)mrow * a.ldy + ncol;
                            if (add) {
                                const float e[4] = {val.x, val.y, val.z, val.w};
                                for (int u = 0; u < 4 && ncol + u < a.N; ++u) atomicAdd(dst + u, e[u]);
                            } else if (ncol + 4 <= a.N && (reinterpret_cast<uintptr_t>(dst) & 15) == 0) {
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
        if (tma && lane == 0) bulk_wait_all();
        if (GR && a.amax_out) {  // (fmaxf skips a NaN, as the quantizer's own max pass does)
            for (int o = 16; o; o >>= 1) hmax = fmaxf(hmax, __shfl_xor_sync(0xffffffffu, hmax, o));
            if (lane == 0) atomicMax(a.amax_out, __float_as_uint(hmax));
        }
        __syncwarp();
    }
    __syncthreads();
    if (warp == 0 && lane == 0 && *abort_flag) {
        // wait (bounded) for the last bulk copies issued to land before shared memory is released
        const int n_it = *issued;
        for (int j = n_it > S ? n_it - S : 0; j < n_it; ++j) {
            mbar_wait_bounded(&full[j % S], (j / S) & 1, 50000000ull);
            mbar_wait_bounded(&sfull[j % S], (j / S) & 1, 50000000ull);
        }
    }
    // CG = 2: the pair's MMAs read both CTAs' shared memory and write both CTAs' tensor memory;
    // neither CTA frees either before the issuing CTA has seen them complete (mma_done above).
    if constexpr (CG == 2) cluster_sync_all();
    if (warp == 0) {
        __syncwarp();
        tc_fence_after();
        tmem_free<CG>(tmem);
    }
    // The last CTA out clears the words of phase Q for the next call (grouped mode uses none).
    if constexpr (!GR) {
        if (threadIdx.x == 0) {
            __threadfence();
            *issued = atomicAdd(&a.words[kWExit], 1u) == gridDim.x - 1 ? -1 : 0;
        }
        __syncthreads();
        if (*issued == -1 && threadIdx.x == 0) {
            a.words[kWAmax] = 0u;
            a.words[kWArrive1] = 0u;
            a.words[kWExit] = 0u;
            __threadfence();
        }
    }
}

}  // namespace qlin

using namespace qlin;

// CTA pairs (cta_group::2) on request (QLIN_FLAG_CTA_PAIRS) when there are more than 128
// activation rows; single CTAs otherwise.
static inline int chunk_cg(int M, int flags) { return (flags & QLIN_FLAG_CTA_PAIRS) && M > kMmaARows ? 2 : 1; }
static inline int64_t chunk_units_m(int M, int flags) {  // 128-row activation units, a multiple of the group size
    const int cg = chunk_cg(M, flags);
    const int64_t rows = (int64_t)kMmaARows * cg;
    return ((M + rows - 1) / rows) * cg;
}

// Workspace: status word and counters (256 B), quantized activation units, per-unit ready counters.
// Sized for the larger (CTA-pair) layout, so one workspace serves both.
extern "C" size_t qlin_chunk_ws_bytes(int M, int64_t N, int64_t K) {
    (void)N;
    const int64_t units = chunk_units_m(M, QLIN_FLAG_CTA_PAIRS) * ((K + kGroupK - 1) / kGroupK);
    return 256 + (size_t)units * kMmaAUnit + (size_t)((units * 4 + 255) / 256) * 256;
}

extern "C" cudaError_t qlin_launch_act_quant(const void* x, int M, int64_t K, int64_t ldx, void* words, void* aq,
                                             void* canon_codes, void* canon_scales, cudaStream_t s);

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link-time libcuda dependency).
static PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
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

// y as a 2-D fp32 tensor {N (inner), M} with row pitch ldy * 4 bytes, stored in 32 x 32 boxes with
// the 128-byte swizzle.  False when y does not meet the tensor-map rules (16-byte aligned base and
// pitch) or the encoder is unavailable; the kernel then stores y with plain stores.
static bool make_y_map(CUtensorMap* map, float* y, int M, int64_t N, int64_t ldy, int box_rows) {
    if ((reinterpret_cast<uintptr_t>(y) & 15) != 0 || (ldy * 4) % 16 != 0) return false;
    PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
    if (!enc) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)N, (cuuint64_t)M};
    const cuuint64_t strides[1] = {(cuuint64_t)ldy * 4};
    const cuuint32_t box[2] = {32, (cuuint32_t)box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, y, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int CG, bool MX, bool GR>
static cudaError_t launch_chunk_cg(ChunkArgs a, int flags, cudaStream_t s) {
    static bool attr_set = false;
    cudaError_t e;
    if (!attr_set) {
        e = cudaFuncSetAttribute(chunk_gemm_kernel<CG, MX, GR>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 chunk_smem<CG>());
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
    // All CTAs must be co-resident (grid-wide barriers): one CTA per SM, and for CG = 2 no more
    // pairs than the device can hold at once.
    static int max_units = 0;  // CTAs (CG = 1) or clusters (CG = 2) resident at once, per device
    static int cached_dev = -1;
    int dev = 0;
    e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
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
    cfg.blockDim = dim3(kChunkThreads);
    cfg.dynamicSmemBytes = chunk_smem<CG>();
    cfg.stream = s;
    cfg.attrs = attr;
    if (cached_dev != dev) {
        int sms = 0;
        e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return e;
        int per_sm = 0;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, chunk_gemm_kernel<CG, MX, GR>, kChunkThreads,
                                                          chunk_smem<CG>());
        if (e != cudaSuccess) return e;
        if (per_sm < 1) return cudaErrorInvalidConfiguration;
        int units = sms;
        if (CG == 2) {
            cfg.gridDim = dim3((unsigned)(sms & ~1));
            cfg.numAttrs = na;
            int clusters = 0;
            e = cudaOccupancyMaxActiveClusters(&clusters, chunk_gemm_kernel<CG, MX, GR>, &cfg);
            if (e != cudaSuccess) return e;
            if (clusters < 1) return cudaErrorInvalidConfiguration;
            units = clusters;
        }
        max_units = units;
        cached_dev = dev;
    }
    // Too few output tiles to give every CTA one: split each tile's k-groups in two halves.
    const int base_tiles = a.T2 * (a.TM / CG);
    a.KS = (CG == 1 && !GR && a.G >= 2 && 2 * base_tiles <= max_units) ? 2 : 1;
    a.GS = (a.G + a.KS - 1) / a.KS;
    const int ntiles = base_tiles * a.KS;
    const int units = ntiles < max_units ? ntiles : max_units;
    cfg.gridDim = dim3((unsigned)(units * CG));
    if (flags & QLIN_FLAG_PDL) {
        attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[na].val.programmaticStreamSerializationAllowed = 1;
        ++na;
    }
    cfg.numAttrs = na;
    CUtensorMap ymap;
    memset(&ymap, 0, sizeof(ymap));
    a.tma_store = (!a.h && a.y && make_y_map(&ymap, a.y, a.M, a.N, a.ldy, EpiCfg<CG>::kBoxRows)) ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, chunk_gemm_kernel<CG, MX, GR>, a, ymap);
}

extern "C" cudaError_t qlin_launch_chunk(int fmt, const void* packed, int64_t N, int64_t K, const void* x, int M,
                                         int64_t ldx, float* y, int64_t ldy, void* ws, int flags, cudaStream_t s) {
    uint8_t* w8 = (uint8_t*)ws;
    ChunkArgs a;
    memset(&a, 0, sizeof(a));  // (grouped-mode fields off)
    a.w = (const uint8_t*)packed;
    a.x = (const __nv_bfloat16*)x;
    a.ldx = ldx;
    a.aq = w8 + 256;
    a.words = (unsigned*)(w8 + 64);
    a.ready = (unsigned*)(w8 + 256 + chunk_units_m(M, QLIN_FLAG_CTA_PAIRS) * ((K + kGroupK - 1) / kGroupK) * kMmaAUnit);
    a.y = y;
    a.ldy = ldy;
    a.M = M;
    a.N = N;
    a.K = K;
    a.T2 = (int)((N + kMmaWRows - 1) / kMmaWRows);
    a.G = (int)((K + kGroupK - 1) / kGroupK);
    a.TM = (int)chunk_units_m(M, flags);
    a.xvec = ((reinterpret_cast<uintptr_t>(x) & 15) == 0 && ldx % 8 == 0) ? 1 : 0;
    a.tma_store = 0;
    a.yvec = ((reinterpret_cast<uintptr_t>(y) & 15) == 0 && ldy % 4 == 0) ? 1 : 0;
    a.KS = 1;
    a.GS = a.G;
    a.status = (unsigned*)ws;
    a.tile_expert = nullptr;
    a.used_tm = nullptr;
    a.w_stride = 0;
    a.h = nullptr;
    a.ldh = a.h_cols = 0;
    if (fmt == QLIN_MXFP4)
        return chunk_cg(M, flags) == 2 ? launch_chunk_cg<2, true, false>(a, flags, s)
                                       : launch_chunk_cg<1, true, false>(a, flags, s);
    return chunk_cg(M, flags) == 2 ? launch_chunk_cg<2, false, false>(a, flags, s)
                                   : launch_chunk_cg<1, false, false>(a, flags, s);
}

extern "C" cudaError_t qlin_launch_act_quant_debug(const void* x, int M, int64_t K, int64_t ldx, void* ws,
                                                   void* codes, void* scales, float* ag, cudaStream_t s) {
    uint8_t* w8 = (uint8_t*)ws;
    unsigned* words = (unsigned*)(w8 + 64);
    cudaError_t e = qlin_launch_act_quant(x, M, K, ldx, words, w8 + 256, codes, scales, s);
    if (e != cudaSuccess) return e;
    return cudaMemcpyAsync(ag, words + 2, 4, cudaMemcpyDeviceToDevice, s);
}

// Grouped launch (the MoE prefill): the activations are expert-sorted rows (rows_max at most, the
// first *used_tm * 128 in use, each expert's rows padded to whole 128-row tiles), already quantized
// into the workspace's operand units by an earlier kernel of the stream, with max |x| = *amax_in;
// w = E packed weight buffers w_stride bytes apart, T2 weight tiles per expert, row tile tm against
// expert tile_expert[tm].  h != nullptr: the SiLU-gate epilogue (weights packed QLIN_PACK_MMA |
// QLIN_PACK_GATE_UP) writing h_cols bf16 outputs per row and folding max |h| into *amax_out; else
// y (fp32, N columns).  Either way rows past tile_rows[tm] of tile tm are not stored.  Errors go to
// *status (the first word of the caller's workspace, whose wait budget word the waits read).  Single CTAs,
// no k-split, launched as a programmatic dependent of the kernel before it.
extern "C" cudaError_t qlin_launch_chunk_grouped(int fmt, const void* w, int64_t w_stride, int T2, int64_t N,
                                                 int64_t K, int rows_max, float* y, int64_t ldy, void* h,
                                                 int64_t ldh, int64_t h_cols, const int* tile_expert,
                                                 const int* tile_rows, const int* used_tm, const unsigned* amax_in,
                                                 unsigned* amax_out, unsigned* status, void* ws, cudaStream_t s) {
    uint8_t* w8 = (uint8_t*)ws;
    ChunkArgs a;
    memset(&a, 0, sizeof(a));
    a.w = (const uint8_t*)w;
    a.ldx = K;
    a.aq = w8 + 256;
    a.words = (unsigned*)(w8 + 64);
    a.ready = (unsigned*)(w8 + 256 +
                          chunk_units_m(rows_max, QLIN_FLAG_CTA_PAIRS) * ((K + kGroupK - 1) / kGroupK) * kMmaAUnit);
    a.y = y;
    a.ldy = ldy;
    a.M = rows_max;
    a.N = N;
    a.K = K;
    a.T2 = T2;
    a.G = (int)((K + kGroupK - 1) / kGroupK);
    a.TM = (int)chunk_units_m(rows_max, 0);
    a.yvec = (y && (reinterpret_cast<uintptr_t>(y) & 15) == 0 && ldy % 4 == 0) ? 1 : 0;
    a.KS = 1;
    a.GS = a.G;
    a.status = status;  // the caller's status word (its wait budget word 32 bytes on)
    a.tile_expert = tile_expert;
    a.tile_rows = tile_rows;
    a.used_tm = used_tm;
    a.w_stride = w_stride;
    a.h = (__nv_bfloat16*)h;
    a.ldh = ldh;
    a.h_cols = h_cols;
    a.amax_in = amax_in;
    a.amax_out = amax_out;
    // programmatic dependent launch: the tile table, the row counts and the weights read before
    // the kernel's wait come from kernels that finished before the previous one passed its own wait
    return fmt == QLIN_MXFP4 ? launch_chunk_cg<1, true, true>(a, QLIN_FLAG_PDL, s)
                             : launch_chunk_cg<1, false, true>(a, QLIN_FLAG_PDL, s);
}

// ---------------------------------------------------------------------------------------------
// MMA-only rate of the FP4 tensor path on this device (a measurement aid, not on the hot path).
// One CTA per SM; one thread issues `iters` back-to-back kind::mxf4nvf4 block16 MMAs of M 128,
// N 256, K 64 into one TMEM accumulator. These use the chunk GEMM's own instruction, shared-memory
// descriptors and instruction word, on fixed operands: arbitrary E2M1 bytes (every 4-bit pattern
// is a finite value) and E4M3 1.0 in every scale factor. No operand moves while the MMAs run, so
// the rate is the tensor pipe's own. Each CTA records its clock64 span from the first issue to the
// commit's arrival; the caller times the launch with events.
constexpr int kProbeABytes = kMmaARows * 128;  // 128 rows x 256 E2M1 values: four K = 64 steps
constexpr int kProbeBBytes = kMmaWRows * 128;  // 256 rows x 256 values
constexpr int kProbePad = 128 * 1024;          // keeps one CTA, and one TMEM allocation, per SM
constexpr int kProbeSmem = 1024 + kProbeABytes + kProbeBBytes + 64 + kProbePad;
static_assert(kProbeSmem <= 232448 && 2 * kProbeSmem > 233472, "one probe CTA per SM");

__global__ void __launch_bounds__(128, 1) fp4_mma_rate_kernel(int iters, unsigned long long* cycles,
                                                              unsigned* status) {
    extern __shared__ uint8_t probe_raw[];
    uint8_t* sm = (uint8_t*)(((uintptr_t)probe_raw + 1023) & ~(uintptr_t)1023);
    uint64_t* bar = (uint64_t*)(sm + kProbeABytes + kProbeBBytes);
    uint32_t* holder = (uint32_t*)(bar + 1);
    const int warp = threadIdx.x >> 5;
    for (int i = threadIdx.x; i < (kProbeABytes + kProbeBBytes) / 4; i += blockDim.x) {
        uint32_t v = (uint32_t)i * 2654435761u ^ (blockIdx.x * 40503u);
        v ^= v >> 15;
        v *= 0x2c1b3c6du;
        v ^= v >> 12;
        ((uint32_t*)sm)[i] = v;
    }
    if (threadIdx.x == 0) {
        mbar_init(bar, 1);
        fence_mbar_init();
    }
    fence_proxy_async_smem();  // the operands were written through the generic proxy
    if (warp == 0) tmem_alloc<1>(holder);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *holder;
    {  // scale-factor columns kAccCols .. kAccCols + 15 of this warp's lane quarter: E4M3 1.0
        uint32_t r[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) r[j] = 0x38383838u;
        tc_st16<0, 16>(tmem + ((uint32_t)(warp * 32) << 16) + kAccCols, r);
        asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (threadIdx.x == 0) {
        const uint32_t idesc = (1u << 7) | (1u << 10) | ((uint32_t)(kMmaWRows >> 3) << 17) |
                               ((uint32_t)(kMmaARows >> 4) << 24);
        const uint32_t sa = smem_u32(sm), sb = sa + kProbeABytes, sf = tmem + kAccCols;
        const unsigned long long t0 = clock64();
        for (int i = 0; i < iters; ++i) {
            const uint32_t kb = (uint32_t)(i & 3) * 32;  // the K = 64 step inside the 128-byte swizzle row
            tc_mma(tmem, sdesc_sw128(sa + kb), sdesc_sw128(sb + kb), idesc, sf, sf + 4, i > 0 ? 1u : 0u);
        }
        tc_commit(bar);
        if (!mbar_wait_bounded(bar, 0)) atomicOr(status, 1u);
        cycles[blockIdx.x] = clock64() - t0;
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_free<1>(tmem);
    }
}

extern "C" cudaError_t qlin_launch_fp4_mma_rate(int iters, unsigned long long* cycles, int max_ctas,
                                                unsigned* status, int* ctas, cudaStream_t s) {
    int dev = 0, sms = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    *ctas = sms;
    if (sms > max_ctas) return cudaErrorInvalidValue;
    e = cudaFuncSetAttribute(fp4_mma_rate_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kProbeSmem);
    if (e != cudaSuccess) return e;
    fp4_mma_rate_kernel<<<sms, 128, kProbeSmem, s>>>(iters, cycles, status);
    return cudaGetLastError();
}
