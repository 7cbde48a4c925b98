// chain.cu -- a sequence of dequantize-and-multiply GEMVs in one persistent launch.
//
// A decode step is a long run of GEMVs over different weight matrices (per layer: q/k/v, o,
// gate_up + SiLU, down).  Launched one by one, each GEMV pays the HBM pipeline's ramp-up at its
// start and its slowest warp at its end; for the 2-30 MB matrices of a decode step that fixed cost
// is as large as the streaming itself.  Weights never depend on activations, so this kernel
// streams the weights of the whole sequence back to back through every warp's copy ring, and
// only the activations wait: an op whose input is the output of an earlier op of the same launch
// waits (bounded) until that op's tiles are all written, while its weights are already arriving.
// (The pages' engines capture the decode step in CUDA graphs for the same reason: imp release
// notes v0.4, "CUDA graphs"; the per-launch overhead is what a persistent launch removes.)
//
// Work split.  Every op is split across ALL warps of the grid into contiguous unit ranges of q or
// q+1 units; the warps receiving the extra units rotate from op to op, so that over a chain each
// warp streams the same number of units to within one.  A tile split between warps is finished
// by the last-arriving contributor (atomic ticket), which sums the partials in range order:
// results are deterministic and independent of timing.
#include <algorithm>

#include "gemv_core.cuh"

namespace qlin {

constexpr int kMaxChainOps = 256;

struct ChainOp {
    const uint8_t* packed;
    const void* x;
    float* y;
    int64_t ws_off;     // byte offset of this op's tile tickets in the workspace
    int32_t ldx, ldy;
    int32_t N, K;       // packed rows (gate + up rows for SiLU-gate ops) and inputs
    int32_t T, G;       // tiles, k-groups
    int32_t U;          // units = T * G
    int32_t q, r;       // split: range v has q + (v < r) units
    int32_t rot;        // warp w has range v = (w - rot) mod W
    int32_t smax;       // partial slots per tile
    int32_t wait_for;   // earlier op whose y this op reads, or -1
    int32_t epi;        // QLIN_EPI_*; bit 8: a later op waits for this one
    int32_t part_rel;   // partials start at ws_off + part_rel
};

struct ChainArgs {
    ChainOp op[kMaxChainOps];
    uint8_t* ws;
    int32_t n_ops;
    int32_t M;
    int32_t W;  // warps in the grid
    int32_t pad;
};

constexpr int kChainSignal = 0x100;
// Workspace: [0,4) status word; [64,68) exit counter; [256, 256 + 4 n_ops) per-op count of
// written tiles; then per op: T tickets (rounded to 256 B) and T x smax x 32 x M fp32 partials.
constexpr int64_t kChainExitOff = 64;
constexpr int64_t kChainDoneOff = 256;

__device__ __forceinline__ uint32_t ld_acquire_u32(const unsigned int* p) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void red_release_add(unsigned int* p, uint32_t v) {
    asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Unit range [b, e) of warp gw in op o.
__device__ __forceinline__ void chain_range(const ChainOp& o, int gw, int W, int& b, int& e) {
    int v = gw - o.rot;
    if (v < 0) v += W;
    b = v * o.q + min(v, o.r);
    e = b + o.q + (v < o.r ? 1 : 0);
}

// Range index (v) of the warp that owns unit u of op o.
__device__ __forceinline__ int chain_owner(const ChainOp& o, int u) {
    const int big = o.r * (o.q + 1);
    if (u < big) return u / (o.q + 1);
    return o.r + (u - big) / o.q;  // q >= 1 here: u < U = W q + r
}

// A warp's position in its sequence of units: op j, unit u of that op, end of its range in op j.
struct ChainCursor {
    int j, u, e;
};

__device__ __forceinline__ void chain_seek(const ChainArgs& a, int gw, ChainCursor& c, int j) {
    for (; j < a.n_ops; ++j) {
        int b, e;
        chain_range(a.op[j], gw, a.W, b, e);
        if (e > b) {
            c.j = j;
            c.u = b;
            c.e = e;
            return;
        }
    }
    c.j = a.n_ops;
    c.u = c.e = 0;
}

__device__ __forceinline__ void chain_step(const ChainArgs& a, int gw, ChainCursor& c) {
    if (++c.u >= c.e) chain_seek(a, gw, c, c.j + 1);
}

template <int FMT>
__device__ __forceinline__ void chain_issue(const ChainArgs& a, const ChainCursor& p, uint8_t* dst, uint64_t* bar) {
    constexpr int UB = RingCfg<FMT>::UB;
    mbar_arrive_expect_tx(bar, UB);
    bulk_g2s(dst, a.op[p.j].packed + kHdrBytes + (int64_t)p.u * UB, UB, bar);
}

// Write tile t of op o from the reduced values (lane holds tile row (lane/8) + 4 (lane%8)).
template <int MAXM>
__device__ __forceinline__ void chain_write_tile(const ChainOp& o, int M, int t, int lane, float (&v)[MAXM],
                                                 float gs) {
    const int row = (lane >> 3) + 4 * (lane & 7);
#pragma unroll
    for (int m = 0; m < MAXM; ++m) v[m] = v[m] * gs;
    if ((o.epi & 0xff) == QLIN_EPI_SILU_GATE) {
        float u[MAXM];
#pragma unroll
        for (int m = 0; m < MAXM; ++m) u[m] = __shfl_down_sync(0xffffffffu, v[m], 4);
        const int64_t i = (int64_t)t * 16 + row;
        if ((lane & 7) < 4 && i < o.N / 2) {
#pragma unroll
            for (int m = 0; m < MAXM; ++m)
                if (m < M) o.y[m * (int64_t)o.ldy + i] = silu_f32(v[m]) * u[m];
        }
    } else {
        const int64_t n = (int64_t)t * kTileRows + row;
        if (n < o.N) {
#pragma unroll
            for (int m = 0; m < MAXM; ++m)
                if (m < M) o.y[m * (int64_t)o.ldy + n] = v[m];
        }
    }
}

// Finish tile t of op j held by this warp: write it if the warp's range covers it, else store the
// partial and take a ticket; the last contributor sums all partials in range order and writes.
// Whoever writes the tile counts it for ops that a later op waits for.
template <int MAXM>
__device__ __forceinline__ void chain_finish_tile(const ChainArgs& a, int j, int t, int b, int e, int lane,
                                                  float (&acc)[MAXM], float gs) {
    const ChainOp& o = a.op[j];
    const int f = t * o.G, l = f + o.G - 1;
    bool wrote = false;
    if (f >= b && l < e) {
        chain_write_tile<MAXM>(o, a.M, t, lane, acc, gs);
        wrote = true;
    } else {
        const int v_first = chain_owner(o, f), v_last = chain_owner(o, l);
        const int n_t = v_last - v_first + 1;
        const int slot = chain_owner(o, b > f ? b : f) - v_first;
        float* part = reinterpret_cast<float*>(a.ws + o.ws_off + o.part_rel);
        int* cnt = reinterpret_cast<int*>(a.ws + o.ws_off);
        float* mine = part + (((int64_t)t * o.smax + slot) * 32 + lane) * a.M;
#pragma unroll
        for (int m = 0; m < MAXM; ++m)
            if (m < a.M) __stcg(mine + m, acc[m]);
        __threadfence();
        __syncwarp();
        int ticket = 0;
        if (lane == 0) ticket = atomicAdd(cnt + t, 1);
        ticket = __shfl_sync(0xffffffffu, ticket, 0);
        if (ticket == n_t - 1) {
            __threadfence();
            float sum[MAXM];
#pragma unroll
            for (int m = 0; m < MAXM; ++m) sum[m] = 0.f;
            for (int s = 0; s < n_t; ++s) {
                const float* src = part + (((int64_t)t * o.smax + s) * 32 + lane) * a.M;
#pragma unroll
                for (int m = 0; m < MAXM; ++m)
                    if (m < a.M) sum[m] += __ldcg(src + m);
            }
            chain_write_tile<MAXM>(o, a.M, t, lane, sum, gs);
            if (lane == 0) cnt[t] = 0;  // leave the workspace reusable
            wrote = true;
        }
    }
    if (wrote && (o.epi & kChainSignal)) {
        __threadfence();
        __syncwarp();
        if (lane == 0) red_release_add(reinterpret_cast<unsigned int*>(a.ws + kChainDoneOff) + j, 1u);
    }
}

// Bounded wait until every tile of op j is written (2 s); false on timeout.
__device__ __forceinline__ bool chain_wait_op(const ChainArgs& a, int j) {
    const unsigned int* done = reinterpret_cast<const unsigned int*>(a.ws + kChainDoneOff) + j;
    const uint32_t target = (uint32_t)a.op[j].T;
    if (__all_sync(0xffffffffu, ld_acquire_u32(done) >= target)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t it = 1;; ++it) {
        __nanosleep(64);
        if (__all_sync(0xffffffffu, ld_acquire_u32(done) >= target)) return true;
        if ((it & 63u) == 0 && globaltimer_ns() - t0 > 2000000000ull) return false;
    }
}

template <int FMT, int MAXM, bool XBF16>
__global__ void __launch_bounds__(kGemvWarps * 32, RingCfg<FMT>::kCtasPerSm)
    chain_kernel(const __grid_constant__ ChainArgs a) {
    using C = RingCfg<FMT>;
    constexpr int MP = MAXM >= 2 ? 2 : 1;
    constexpr bool kOnePass = MAXM <= 2;
    constexpr bool kH = (FMT == QLIN_NVFP4) && XBF16;
    extern __shared__ __align__(128) uint8_t smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int gw = blockIdx.x * kGemvWarps + warp;
    uint8_t* ring = smem + warp * C::D * C::UB;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kGemvWarps * C::D * C::UB) + warp * C::D;

    griddep_launch_dependents();
    ChainCursor c;
    chain_seek(a, gw, c, 0);
    ChainCursor p = c;  // producer cursor, C::D units ahead once primed
    if (lane == 0) {
#pragma unroll
        for (int s = 0; s < C::D; ++s) mbar_init(&bars[s], 1);
        fence_mbar_init();
        for (int s = 0; s < C::D && p.j < a.n_ops; ++s) {  // weights: independent of earlier kernels
            chain_issue<FMT>(a, p, ring + s * C::UB, &bars[s]);
            chain_step(a, gw, p);
        }
    }
    p.j = __shfl_sync(0xffffffffu, p.j, 0);
    p.u = __shfl_sync(0xffffffffu, p.u, 0);
    p.e = __shfl_sync(0xffffffffu, p.e, 0);
    __syncwarp();
    griddep_wait();  // activations, outputs and the workspace may belong to the previous kernel

    const int part = lane & 7;
    float acc[MAXM];
#pragma unroll
    for (int m = 0; m < MAXM; ++m) acc[m] = 0.f;
    float acc8[8][MP];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int mm = 0; mm < MP; ++mm) acc8[i][mm] = 0.f;

    bool failed = false;
    int seq = 0;        // units consumed
    int cur_op = -1;    // op of the previous unit
    int b = 0, e = 0;   // this warp's range in cur_op
    float gs = 1.f;
    while (c.j < a.n_ops) {
        const ChainOp& o = a.op[c.j];
        if (c.j != cur_op) {
            cur_op = c.j;
            chain_range(o, gw, a.W, b, e);
            gs = format_out_scale<FMT>(o.packed);
            if (o.wait_for >= 0 && !chain_wait_op(a, o.wait_for)) {
                failed = true;
                break;
            }
        }
        const int slot = seq % C::D;
        if (!mbar_wait_bounded(&bars[slot], (uint32_t)((seq / C::D) & 1))) {
            failed = true;
            break;
        }
        const uint8_t* ubuf = ring + slot * C::UB;
        const int t = c.u / o.G, g = c.u - t * o.G;
        const int64_t k0 = (int64_t)g * kGroupK + part * 32;
        if (kOnePass) {
            const void* rows[MP];
#pragma unroll
            for (int mm = 0; mm < MP; ++mm)
                rows[mm] = (mm < a.M) ? (XBF16 ? (const void*)(reinterpret_cast<const __nv_bfloat16*>(o.x) + mm * (int64_t)o.ldx)
                                               : (const void*)(reinterpret_cast<const float*>(o.x) + mm * (int64_t)o.ldx))
                                      : nullptr;
            if constexpr (kH) {
                uint32_t xh[MP][16];
                float xsc[MP][2];
                load_x_fp4h<MP, true>(rows, k0, o.K, xh, xsc);
                unit_dot_fp4h<MP, true>(ubuf, lane, xh, xsc, acc8);
            } else {
                float2 xv[MP][16];
                float xb[MP];
                load_x_rows<XBF16, MP, true>(rows, k0, o.K, xv);
                prep_x<FMT, MP>(xv, xb);
                unit_dot<FMT, MP, true>(ubuf, lane, xv, xb, acc8);
            }
        } else {
#pragma unroll 1
            for (int m0 = 0; m0 < a.M; m0 += MP) {
                const void* rows[MP];
#pragma unroll
                for (int mm = 0; mm < MP; ++mm)
                    rows[mm] = (m0 + mm < a.M)
                                   ? (XBF16 ? (const void*)(reinterpret_cast<const __nv_bfloat16*>(o.x) + (m0 + mm) * (int64_t)o.ldx)
                                            : (const void*)(reinterpret_cast<const float*>(o.x) + (m0 + mm) * (int64_t)o.ldx))
                                   : nullptr;
                float res[8][MP];
                if constexpr (kH) {
                    uint32_t xh[MP][16];
                    float xsc[MP][2];
                    load_x_fp4h<MP, true>(rows, k0, o.K, xh, xsc);
                    unit_dot_fp4h<MP>(ubuf, lane, xh, xsc, res);
                } else {
                    float2 xv[MP][16];
                    float xb[MP];
                    load_x_rows<XBF16, MP, true>(rows, k0, o.K, xv);
                    prep_x<FMT, MP>(xv, xb);
                    unit_dot<FMT, MP>(ubuf, lane, xv, xb, res);
                }
                float r[MP];
                reduce_scatter8<MP>(res, lane, r);
#pragma unroll
                for (int q = 0; q < MAXM; ++q)
#pragma unroll
                    for (int mm = 0; mm < MP; ++mm)
                        if (q == m0 + mm) acc[q] += r[mm];
            }
        }
        __syncwarp();
        // Refill this slot with the producer's next unit (the ring runs C::D units ahead).
        if (lane == 0 && p.j < a.n_ops) {
            fence_proxy_async_smem();
            chain_issue<FMT>(a, p, ring + slot * C::UB, &bars[slot]);
        }
        if (p.j < a.n_ops) chain_step(a, gw, p);
        ++seq;
        const int j_now = c.j;
        chain_step(a, gw, c);
        if (c.j != j_now || c.u / o.G != t) {  // tile t of op j_now ends in this warp
            if (kOnePass) {
                float r[MP];
                reduce_scatter8<MP>(acc8, lane, r);
#pragma unroll
                for (int mm = 0; mm < MP; ++mm) acc[mm] = r[mm];
#pragma unroll
                for (int i = 0; i < 8; ++i)
#pragma unroll
                    for (int mm = 0; mm < MP; ++mm) acc8[i][mm] = 0.f;
            }
            chain_finish_tile<MAXM>(a, j_now, t, b, e, lane, acc, gs);
#pragma unroll
            for (int m = 0; m < MAXM; ++m) acc[m] = 0.f;
        }
    }
    if (failed && lane == 0) {
        atomicOr(reinterpret_cast<unsigned int*>(a.ws), 1u);
        // Wait (bounded) for this warp's copies still in flight: the C::D units after seq.
        ChainCursor q = c;
        for (int s = 0; s < C::D && q.j < a.n_ops; ++s) {
            mbar_wait_bounded(&bars[(seq + s) % C::D], (uint32_t)(((seq + s) / C::D) & 1), 100000000ull);
            chain_step(a, gw, q);
        }
    }
    // The last CTA to leave resets the per-op tile counts for the next launch.
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        unsigned int* ex = reinterpret_cast<unsigned int*>(a.ws + kChainExitOff);
        if (atomicAdd(ex, 1u) == gridDim.x - 1) {
            __threadfence();
            unsigned int* done = reinterpret_cast<unsigned int*>(a.ws + kChainDoneOff);
            for (int j = 0; j < a.n_ops; ++j) done[j] = 0u;
            *ex = 0u;
        }
    }
}

}  // namespace qlin

// ------------------------------------------------------------------ host side
namespace qlin {

static int chain_sm_count() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
    return n;
}

// CTAs of the persistent grid: every SM holds RingCfg<FMT>::kCtasPerSm of them (the register
// and shared-memory budget of the kernel is sized for exactly that).
static int chain_grid(int fmt) {
    const int cps = fmt == QLIN_Q8_0 ? RingCfg<QLIN_Q8_0>::kCtasPerSm : RingCfg<QLIN_Q4_0>::kCtasPerSm;
    return chain_sm_count() * cps;
}

static int64_t al256(int64_t v) { return (v + 255) / 256 * 256; }

// Fill the device descriptors; returns the workspace bytes the chain needs.
static int64_t chain_plan(int fmt, int M, const qlin_gemv_op* ops, int n, int W, ChainArgs* a) {
    int64_t off = kChainDoneOff + al256(4 * (int64_t)n);
    int64_t before = 0;  // units of the ops before this one
    for (int j = 0; j < n; ++j) {
        const qlin_gemv_op& u = ops[j];
        const int epi = u.epilogue & 0xff;
        const Geometry geo = geometry(fmt, u.N, u.K, epi == QLIN_EPI_SILU_GATE ? QLIN_PACK_GATE_UP : 0);
        ChainOp o = {};
        o.packed = (const uint8_t*)u.packed;
        o.x = u.x;
        o.y = u.y;
        o.ldx = (int32_t)u.ldx;
        o.ldy = (int32_t)u.ldy;
        o.N = (int32_t)u.N;
        o.K = (int32_t)u.K;
        o.T = (int32_t)geo.T;
        o.G = (int32_t)geo.G;
        o.U = (int32_t)geo.U;
        o.q = (int32_t)(geo.U / W);
        o.r = (int32_t)(geo.U % W);
        o.rot = (int32_t)(before % W);
        o.smax = (int32_t)(o.q == 0 ? o.G : std::min<int64_t>(o.G, (o.G + o.q - 1) / o.q + 1));
        o.wait_for = u.wait_for;
        o.epi = epi;
        for (int k = j + 1; k < n; ++k)
            if (ops[k].wait_for == j) o.epi |= kChainSignal;
        o.ws_off = off;
        o.part_rel = (int32_t)al256(4 * (int64_t)o.T);
        off += o.part_rel + al256((int64_t)o.T * o.smax * 32 * M * 4);
        before += geo.U;
        if (a) a->op[j] = o;
    }
    return off;
}

template <int FMT, int MAXM, bool XBF16>
static cudaError_t chain_launch(const ChainArgs* a, int grid, cudaStream_t s, bool pdl) {
    using C = RingCfg<FMT>;
    auto kern = chain_kernel<FMT, MAXM, XBF16>;
    static bool attr_set = false;  // per instantiation; idempotent
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
        if (e != cudaSuccess) return e;
        // The dependency waits need every CTA of the grid resident at once.
        int occ = 0;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, kGemvWarps * 32, C::kSmem);
        if (e != cudaSuccess) return e;
        if (occ < C::kCtasPerSm) return cudaErrorLaunchOutOfResources;
        attr_set = true;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kGemvWarps * 32);
    cfg.dynamicSmemBytes = C::kSmem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kern, *a);
}

template <int FMT, bool XBF16>
static cudaError_t chain_launch_m(const ChainArgs* a, int grid, cudaStream_t s, bool pdl) {
    if (a->M == 1) return chain_launch<FMT, 1, XBF16>(a, grid, s, pdl);
    if (a->M == 2) return chain_launch<FMT, 2, XBF16>(a, grid, s, pdl);
    if (a->M <= 4) return chain_launch<FMT, 4, XBF16>(a, grid, s, pdl);
    return chain_launch<FMT, 8, XBF16>(a, grid, s, pdl);
}

}  // namespace qlin

using namespace qlin;

extern "C" int qlin_chain_max_ops() { return kMaxChainOps; }

extern "C" size_t qlin_chain_ws_bytes(int fmt, int M, const qlin_gemv_op* ops, int n_ops) {
    return (size_t)chain_plan(fmt, M, ops, n_ops, chain_grid(fmt) * kGemvWarps, nullptr);
}

// Launch after host-side validation (done in api.cu).
extern "C" cudaError_t qlin_launch_chain(int fmt, int xdt, int M, const qlin_gemv_op* ops, int n_ops, int flags,
                                         void* ws, cudaStream_t s) {
    static_assert(sizeof(ChainArgs) <= 32000, "kernel parameter space");
    const int grid = chain_grid(fmt);
    ChainArgs* a = new ChainArgs();  // ~20 KB: not on the caller's stack
    chain_plan(fmt, M, ops, n_ops, grid * kGemvWarps, a);
    a->ws = (uint8_t*)ws;
    a->n_ops = n_ops;
    a->M = M;
    a->W = grid * kGemvWarps;
    const bool pdl = (flags & QLIN_FLAG_PDL) != 0, bf16 = xdt == QLIN_BF16;
    cudaError_t e;
    if (fmt == QLIN_Q4_0) e = bf16 ? chain_launch_m<QLIN_Q4_0, true>(a, grid, s, pdl) : chain_launch_m<QLIN_Q4_0, false>(a, grid, s, pdl);
    else if (fmt == QLIN_Q8_0) e = bf16 ? chain_launch_m<QLIN_Q8_0, true>(a, grid, s, pdl) : chain_launch_m<QLIN_Q8_0, false>(a, grid, s, pdl);
    else e = bf16 ? chain_launch_m<QLIN_NVFP4, true>(a, grid, s, pdl) : chain_launch_m<QLIN_NVFP4, false>(a, grid, s, pdl);
    delete a;
    return e;
}
