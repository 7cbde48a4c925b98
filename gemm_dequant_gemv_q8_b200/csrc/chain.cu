// chain.cu -- a sequence of dequantize-and-multiply GEMVs in one persistent launch.
//
// A decode step is a long run of GEMVs over different weight matrices (per layer: q/k/v, o,
// gate_up + SiLU, down).  Launched one by one, each GEMV pays the HBM pipeline's ramp-up at its
// start and its slowest warp at its end; for the 2-30 MB matrices of a decode step that fixed cost
// is as large as the streaming itself.  Weights never depend on activations, so this kernel
// streams the weights of the whole sequence back to back through every warp's copy ring, and only
// the activations wait.  (The pages' engines capture the decode step in CUDA graphs for the
// per-launch overhead: imp release notes v0.4, "CUDA graphs".)
//
// Segments.  The ops are grouped by dependency level: level 0 = ops that wait for nothing, level
// d+1 = ops waiting for an op of level d.  One level is one segment; its ops' units, concatenated
// in the given op order, are split into one contiguous range per warp (equal to within one unit,
// the warps receiving the extra unit rotating from segment to segment).  So a warp's range ends in
// at most one tile shared with the next warp, whatever the number of ops in the segment, and a
// segment never waits for itself: an op of segment d+1 waits (bounded) for the op of segment d
// it reads, normally already finished.  A chain of independent projections is one segment; a
// fully sequential chain is one segment per op.
//
// Split tiles.  A tile crossing a range boundary is computed in pieces by consecutive warps.
// Every piece is published as 64-bit words {fp32 partial, launch tag} (single-copy atomic stores;
// no fence, no read-modify-write), and the warp owning the tile's first unit -- its piece ends that
// warp's range -- finishes the tile when it moves on to the next segment (or before it waits, or
// at the end): it reads the pieces in range order, re-reading (bounded) any word whose tag is not
// this launch's, adds them in that order and writes the tile.  Results are deterministic and
// independent of timing; no warp waits for work another warp has not started.
#include <algorithm>
#include <vector>

#include "gemv_core.cuh"

namespace qlin {

constexpr int kMaxChainOps = 192;

struct ChainOp {
    const uint8_t* packed;
    const void* x;
    float* y;
    int64_t ws_off;     // byte offset of this op's partial words in the workspace
    int32_t ldx, ldy;
    int32_t N, K;       // packed rows (gate + up rows for SiLU-gate ops) and inputs
    int32_t T, G;       // tiles, k-groups
    int32_t U;          // units = T * G
    int32_t base;       // first unit of this op in its segment's concatenated units
    int32_t smax;       // partial slots per tile
    int32_t wait_for;   // op (execution index) whose y this op reads, or -1
    int32_t epi;        // QLIN_EPI_* | QLIN_OUT_BF16; bit 8: a later op waits for this one
    int32_t seg;        // segment index
};

struct ChainSeg {
    int32_t first, end;  // ops [first, end)
    int32_t U;           // units
    int32_t q, r;        // range v has q + (v < r) units
    int32_t rot;         // warp w has range v = (w - rot) mod W
};

struct ChainArgs {
    ChainOp op[kMaxChainOps];
    ChainSeg seg[kMaxChainOps];
    uint8_t* ws;
    int32_t n_ops, n_seg;
    int32_t M;
    int32_t W;  // warps in the grid
};

constexpr int kChainSignal = 0x100;
// Workspace: [0,4) status word; [64,68) exit counter; [128,132) launch counter; [256, 256 +
// 4 n_ops) per-op count of written tiles; then per op T x smax x 32 x M partial words (8 B).
constexpr int64_t kChainExitOff = 64;
constexpr int64_t kChainEpochOff = 128;
constexpr int64_t kChainDoneOff = 256;

__device__ __forceinline__ void st_relaxed_u64(uint64_t* p, uint64_t v) {
    asm volatile("st.relaxed.gpu.global.b64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

__device__ __forceinline__ uint64_t ld_relaxed_u64(const uint64_t* p) {
    uint64_t v;
    asm volatile("ld.relaxed.gpu.global.b64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ uint32_t ld_acquire_u32(const unsigned int* p) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void red_release_add(unsigned int* p, uint32_t v) {
    asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Range [b, e) (segment units) of warp gw in segment s.
__device__ __forceinline__ void seg_range(const ChainSeg& s, int gw, int W, int& b, int& e) {
    int v = gw - s.rot;
    if (v < 0) v += W;
    b = v * s.q + min(v, s.r);
    e = b + s.q + (v < s.r ? 1 : 0);
}

// Range index of the warp owning segment unit u.
__device__ __forceinline__ int seg_owner(const ChainSeg& s, int u) {
    const int big = s.r * (s.q + 1);
    if (u < big) return u / (s.q + 1);
    return s.r + (u - big) / s.q;  // q >= 1 here: u < U = W q + r
}

// A warp's position: segment s, op j, segment unit u (tile t, k-group g of op j); its range in s
// ends at e.  t and g advance incrementally: no division per unit.
struct ChainCursor {
    int s, j, u, e, t, g;
};

// First unit of the first non-empty range of this warp in segments >= s.
__device__ __forceinline__ void chain_seek(const ChainArgs& a, int gw, ChainCursor& c, int s) {
    for (; s < a.n_seg; ++s) {
        int b, e;
        seg_range(a.seg[s], gw, a.W, b, e);
        if (e > b) {
            int j = a.seg[s].first;
            while (b >= a.op[j].base + a.op[j].U) ++j;
            c.s = s;
            c.j = j;
            c.u = b;
            c.e = e;
            c.t = (b - a.op[j].base) / a.op[j].G;
            c.g = b - a.op[j].base - c.t * a.op[j].G;
            return;
        }
    }
    c.s = a.n_seg;
    c.j = a.n_ops;
    c.u = c.e = c.t = c.g = 0;
}

__device__ __forceinline__ void chain_step(const ChainArgs& a, int gw, ChainCursor& c) {
    if (++c.u >= c.e) {
        chain_seek(a, gw, c, c.s + 1);
        return;
    }
    if (c.u >= a.op[c.j].base + a.op[c.j].U) {  // ops of a segment are contiguous
        ++c.j;
        c.t = c.g = 0;
    } else if (++c.g == a.op[c.j].G) {
        c.g = 0;
        ++c.t;
    }
}

template <int FMT>
__device__ __forceinline__ void chain_issue(const ChainArgs& a, const ChainCursor& p, uint8_t* dst, uint64_t* bar) {
    constexpr int UB = RingCfg<FMT>::UB;
    const ChainOp& o = a.op[p.j];
    mbar_arrive_expect_tx(bar, UB);
    bulk_g2s(dst, o.packed + kHdrBytes + (int64_t)(p.u - o.base) * UB, UB, bar);
}

// Write tile t of op o from the reduced values (lane holds tile row (lane/8) + 4 (lane%8)).
template <int MAXM>
__device__ __forceinline__ void chain_write_tile(const ChainOp& o, int M, int t, int lane, float (&v)[MAXM],
                                                 float gs) {
    const int row = (lane >> 3) + 4 * (lane & 7);
#pragma unroll
    for (int m = 0; m < MAXM; ++m) v[m] = v[m] * gs;
    const bool bf16 = (o.epi & QLIN_OUT_BF16) != 0;
    auto store = [&](int64_t idx, float val) {
        if (bf16) reinterpret_cast<__nv_bfloat16*>(o.y)[idx] = __float2bfloat16_rn(val);
        else o.y[idx] = val;
    };
    if ((o.epi & 0xf) == QLIN_EPI_SILU_GATE) {
        float u[MAXM];
#pragma unroll
        for (int m = 0; m < MAXM; ++m) u[m] = __shfl_down_sync(0xffffffffu, v[m], 4);
        const int64_t i = (int64_t)t * 16 + row;
        if ((lane & 7) < 4 && i < o.N / 2) {
#pragma unroll
            for (int m = 0; m < MAXM; ++m)
                if (m < M) store(m * (int64_t)o.ldy + i, silu_f32(v[m]) * u[m]);
        }
    } else {
        const int64_t n = (int64_t)t * kTileRows + row;
        if (n < o.N) {
#pragma unroll
            for (int m = 0; m < MAXM; ++m)
                if (m < M) store(m * (int64_t)o.ldy + n, v[m]);
        }
    }
}

// Count n written tiles of op j for the ops waiting for it (one release per batch of tiles).  The
// warp barrier orders every lane's tile stores before lane 0's release, which is cumulative over
// them.
__device__ __forceinline__ void chain_signal(const ChainArgs& a, int j, uint32_t n, int lane) {
    __syncwarp();
    if (lane == 0) red_release_add(reinterpret_cast<unsigned int*>(a.ws + kChainDoneOff) + j, n);
}

// Write tile t of op j (values already summed); with `signal`, count it at once.
template <int MAXM>
__device__ __forceinline__ void chain_emit(const ChainArgs& a, int j, int t, int lane, float (&v)[MAXM], float gs,
                                           bool signal) {
    const ChainOp& o = a.op[j];
    chain_write_tile<MAXM>(o, a.M, t, lane, v, gs);
    if (signal && (o.epi & kChainSignal)) chain_signal(a, j, 1u, lane);
}

// Split-tile geometry of tile t of op j: range index of its first piece and number of pieces.
__device__ __forceinline__ void chain_pieces(const ChainArgs& a, int j, int t, int& v_first, int& n_t) {
    const ChainOp& o = a.op[j];
    const ChainSeg& s = a.seg[o.seg];
    const int f = o.base + t * o.G;
    v_first = seg_owner(s, f);
    n_t = seg_owner(s, f + o.G - 1) - v_first + 1;
}

// Publish this warp's piece (slot = its place in range order) of split tile t of op j.
template <int MAXM>
__device__ __forceinline__ void chain_publish(const ChainArgs& a, int j, int t, int slot, int lane,
                                              const float (&acc)[MAXM], uint32_t tag) {
    const ChainOp& o = a.op[j];
    uint64_t* w = reinterpret_cast<uint64_t*>(a.ws + o.ws_off) + (((int64_t)t * o.smax + slot) * 32 + lane) * a.M;
#pragma unroll
    for (int m = 0; m < MAXM; ++m)
        if (m < a.M) st_relaxed_u64(w + m, ((uint64_t)tag << 32) | __float_as_uint(acc[m]));
}

// Finish split tile t of op j: add its n_t published pieces in range order (re-reading, bounded,
// any word not yet tagged with this launch), then write it.  False if a piece never arrived (~2 s, or the workspace's
// wait budget).
template <int MAXM>
__device__ __noinline__ bool chain_flush(const ChainArgs& a, int j, int t, int lane, float gs, uint32_t tag) {
    const ChainOp& o = a.op[j];
    int v_first, n_t;
    chain_pieces(a, j, t, v_first, n_t);
    const uint64_t* part = reinterpret_cast<const uint64_t*>(a.ws + o.ws_off) + ((int64_t)t * o.smax * 32 + lane) * a.M;
    const int64_t sstride = 32 * (int64_t)a.M;  // words per slot
    constexpr int CH = MAXM >= 16 ? 1 : 16 / MAXM;
    float sum[MAXM];
#pragma unroll
    for (int m = 0; m < MAXM; ++m) sum[m] = 0.f;
    for (int s0 = 0; s0 < n_t; s0 += CH) {
        uint64_t w[CH][MAXM];
#pragma unroll
        for (int c = 0; c < CH; ++c)
#pragma unroll
            for (int m = 0; m < MAXM; ++m)
                w[c][m] = (s0 + c < n_t && m < a.M) ? ld_relaxed_u64(part + (s0 + c) * sstride + m)
                                                    : ((uint64_t)tag << 32);
        bool ready = true;
#pragma unroll
        for (int c = 0; c < CH; ++c)
#pragma unroll
            for (int m = 0; m < MAXM; ++m) ready &= (uint32_t)(w[c][m] >> 32) == tag;
        if (!__all_sync(0xffffffffu, ready)) {  // a piece is not visible yet: re-read (bounded)
            const uint64_t t0 = globaltimer_ns(), budget = ws_wait_budget_ns(a.ws);
            for (uint32_t it = 1;; ++it) {
                __nanosleep(100);
                ready = true;
#pragma unroll
                for (int c = 0; c < CH; ++c)
#pragma unroll
                    for (int m = 0; m < MAXM; ++m)
                        if (s0 + c < n_t && m < a.M && (uint32_t)(w[c][m] >> 32) != tag) {
                            w[c][m] = ld_relaxed_u64(part + (s0 + c) * sstride + m);
                            ready &= (uint32_t)(w[c][m] >> 32) == tag;
                        }
                if (__all_sync(0xffffffffu, ready)) break;
                if (globaltimer_ns() - t0 > budget) return false;
            }
        }
#pragma unroll
        for (int c = 0; c < CH; ++c)
#pragma unroll
            for (int m = 0; m < MAXM; ++m)
                if (s0 + c < n_t) sum[m] += __uint_as_float((uint32_t)w[c][m]);
    }
    chain_emit<MAXM>(a, j, t, lane, sum, gs, true);
    return true;
}

// Which ops this CTA has seen complete (set by the warp that saw it; zeroed at kernel start), and
// whether one of its warps is polling the global counts right now.
__shared__ unsigned int s_chain_seen[kMaxChainOps];
__shared__ unsigned int s_chain_poll;

// Bounded wait until every tile of op j is written (~2 s, or the workspace's wait budget); false
// on timeout.  One warp of the CTA at a time reads the global count (with a pause between reads);
// the others wait for the shared-memory flag the reading warp sets when the count is complete.
// Thousands of warps polling one L2 line slow every other load of the grid.
__device__ __forceinline__ bool chain_wait_op(const ChainArgs& a, int j) {
    const unsigned int* done = reinterpret_cast<const unsigned int*>(a.ws + kChainDoneOff) + j;
    const uint32_t target = (uint32_t)a.op[j].T;
    const int lane = threadIdx.x & 31;
    uint32_t seen = 0;
    if (lane == 0) {
        asm volatile("ld.acquire.cta.shared.u32 %0, [%1];" : "=r"(seen) : "r"(smem_u32(&s_chain_seen[j])) : "memory");
        if (!seen && ld_acquire_u32(done) >= target) seen = 1;
    }
    if (__shfl_sync(0xffffffffu, seen, 0)) {
        __syncwarp();
        return true;
    }
    const uint64_t t0 = globaltimer_ns(), budget = ws_wait_budget_ns(a.ws);
    for (;;) {
        __nanosleep(256);
        if (lane == 0) {
            asm volatile("ld.acquire.cta.shared.u32 %0, [%1];" : "=r"(seen) : "r"(smem_u32(&s_chain_seen[j])) : "memory");
            if (!seen && atomicExch(&s_chain_poll, 1u) == 0u) {
                if (ld_acquire_u32(done) >= target) {
                    asm volatile("st.release.cta.shared.u32 [%0], 1;" ::"r"(smem_u32(&s_chain_seen[j])) : "memory");
                    seen = 1;
                }
                atomicExch(&s_chain_poll, 0u);
            }
        }
        if (__shfl_sync(0xffffffffu, seen, 0)) {
            __syncwarp();  // the other lanes read after lane 0's acquire
            return true;
        }
        if (globaltimer_ns() - t0 > budget) return false;
    }
}

// Shared memory of the chain kernel: the per-warp weight rings and their barriers, then (for
// M <= 2, except Q8_0 / Q6_K whose rings leave no room) two activation stages per warp.
template <int FMT, int MAXM, bool XBF16>
struct ChainSmem {
    static constexpr int MP = MAXM >= 2 ? 2 : 1;
    static constexpr bool kStaged = MAXM <= 2 && FMT != QLIN_Q8_0 && FMT != QLIN_Q6_K;
    static constexpr int kStageBytes = MP * XStage<XBF16>::kRowBytes;  // one stage of one warp
    static constexpr int kXOff = (RingCfg<FMT>::kSmem + 127) / 128 * 128;
    static constexpr int kBytes = kStaged ? kXOff + kGemvWarps * 2 * kStageBytes : RingCfg<FMT>::kSmem;
};

template <int FMT, int MAXM, bool XBF16>
__global__ void __launch_bounds__(kGemvWarps * 32, RingCfg<FMT>::kCtasPerSm)
    chain_kernel(const __grid_constant__ ChainArgs a) {
    using C = RingCfg<FMT>;
    constexpr int MP = MAXM >= 2 ? 2 : 1;
    constexpr bool kOnePass = MAXM <= 2;
    constexpr bool kH = (FMT == QLIN_NVFP4 || FMT == QLIN_MXFP4) && XBF16;
    extern __shared__ __align__(128) uint8_t smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int gw = blockIdx.x * kGemvWarps + warp;
    uint8_t* ring = smem + warp * C::D * C::UB;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kGemvWarps * C::D * C::UB) + warp * C::D;

    griddep_launch_dependents();
    for (int i = threadIdx.x; i < kMaxChainOps; i += blockDim.x) s_chain_seen[i] = 0u;
    if (threadIdx.x == 0) s_chain_poll = 0u;
    __syncthreads();
    ChainCursor c;
    chain_seek(a, gw, c, 0);
    ChainCursor p = c;  // producer cursor, C::D units ahead once primed
    if (lane == 0) {
#pragma unroll
        for (int s = 0; s < C::D; ++s) mbar_init(&bars[s], 1);
        fence_mbar_init();
        for (int s = 0; s < C::D && p.s < a.n_seg; ++s) {  // weights: independent of earlier kernels
            chain_issue<FMT>(a, p, ring + s * C::UB, &bars[s]);
            chain_step(a, gw, p);
        }
    }
    p.s = __shfl_sync(0xffffffffu, p.s, 0);
    p.j = __shfl_sync(0xffffffffu, p.j, 0);
    p.u = __shfl_sync(0xffffffffu, p.u, 0);
    p.e = __shfl_sync(0xffffffffu, p.e, 0);
    p.t = __shfl_sync(0xffffffffu, p.t, 0);
    p.g = __shfl_sync(0xffffffffu, p.g, 0);
    __syncwarp();
    griddep_wait();  // activations, outputs and the workspace may belong to the previous kernel
    const uint32_t tag = __ldcg(reinterpret_cast<const unsigned int*>(a.ws + kChainEpochOff)) + 1u;

    using XS = ChainSmem<FMT, MAXM, XBF16>;
    uint8_t* xst = smem + XS::kXOff + warp * 2 * XS::kStageBytes;  // used only if XS::kStaged
    bool xready = false;  // the current unit's activations were staged by the previous iteration
    int sig_j = -1;       // written tiles of op sig_j not yet counted
    uint32_t sig_n = 0;
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
    int pend_j = -1, pend_t = 0;  // split tile this warp finishes on leaving the segment
    float pend_gs = 1.f;
    int seq = 0;                  // units consumed
    int cur_seg = -1, cur_op = -1;
    int b = 0, e = 0;             // this warp's range in cur_seg
    float gs = 1.f;
    while (c.s < a.n_seg) {
        const ChainOp& o = a.op[c.j];
        if (c.s != cur_seg) {
            cur_seg = c.s;
            seg_range(a.seg[c.s], gw, a.W, b, e);
            if (pend_j >= 0) {
                if (!chain_flush<MAXM>(a, pend_j, pend_t, lane, pend_gs, tag)) {
                    failed = true;
                    break;
                }
                pend_j = -1;
            }
        }
        if (c.j != cur_op) {
            cur_op = c.j;
            gs = format_out_scale<FMT>(o.packed);
            if (sig_n) {
                chain_signal(a, sig_j, sig_n, lane);
                sig_n = 0;
            }
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
        const int t = c.t, g = c.g;
        const int64_t k0 = (int64_t)g * kGroupK + part * 32;
        ChainCursor cn = c;  // the next unit of this warp
        chain_step(a, gw, cn);
        if constexpr (XS::kStaged) {
            uint8_t* xcur = xst + (seq & 1) * XS::kStageBytes;
            if (!xready) stage_x<XBF16, MP>(o.x, o.ldx, a.M, o.K, g, xcur, lane);
            cp_async_wait_all();
            __syncwarp();
            // Stage the next unit's slice now, unless its op must first wait for another op.
            xready = false;
            if (cn.s < a.n_seg && (cn.j == c.j || a.op[cn.j].wait_for < 0)) {
                const ChainOp& on = a.op[cn.j];
                stage_x<XBF16, MP>(on.x, on.ldx, a.M, on.K, cn.g,
                                   xst + ((seq + 1) & 1) * XS::kStageBytes, lane);
                xready = true;
            }
            if constexpr (kH) {
                uint32_t xh[MP][16];
                float xsc[MP][2];
                load_x_fp4h_staged<MP>(xcur, part, xh, xsc);
                unit_dot_fp4h<MP, true, FMT>(ubuf, lane, xh, xsc, acc8);
            } else {
                float2 xv[MP][16];
                float2 xb[MP];
                load_x_staged<XBF16, MP>(xcur, part, xv);
                prep_x<FMT, MP>(xv, xb);
                unit_dot<FMT, MP, true>(ubuf, lane, xv, xb, acc8);
            }
        } else if (kOnePass) {
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
                unit_dot_fp4h<MP, true, FMT>(ubuf, lane, xh, xsc, acc8);
            } else {
                float2 xv[MP][16];
                float2 xb[MP];
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
                    unit_dot_fp4h<MP, false, FMT>(ubuf, lane, xh, xsc, res);
                } else {
                    float2 xv[MP][16];
                    float2 xb[MP];
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
        if (lane == 0 && p.s < a.n_seg) {
            fence_proxy_async_smem();
            chain_issue<FMT>(a, p, ring + slot * C::UB, &bars[slot]);
        }
        if (p.s < a.n_seg) chain_step(a, gw, p);
        ++seq;
        const int s_now = c.s, j_now = c.j;
        c = cn;
        if (c.s != s_now || c.j != j_now || c.t != t) {  // tile t of op j_now ends here
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
            const int f = o.base + t * o.G;  // the tile in segment units: [f, f + G)
            if (f >= b && f + o.G <= e) {  // the whole tile is this warp's
                chain_emit<MAXM>(a, j_now, t, lane, acc, gs, false);
                if (o.epi & kChainSignal) {
                    if (sig_n && sig_j != j_now) chain_signal(a, sig_j, sig_n, lane), sig_n = 0;
                    sig_j = j_now;
                    ++sig_n;
                }
            } else {
                const ChainSeg& sg = a.seg[s_now];
                const int sl = seg_owner(sg, b > f ? b : f) - seg_owner(sg, f);
                chain_publish<MAXM>(a, j_now, t, sl, lane, acc, tag);
                if (sl == 0) {  // first piece: this warp's range ends in the tile; finish it later
                    pend_j = j_now;
                    pend_t = t;
                    pend_gs = gs;
                }
            }
#pragma unroll
            for (int m = 0; m < MAXM; ++m) acc[m] = 0.f;
        }
    }
    if (sig_n) chain_signal(a, sig_j, sig_n, lane);
    if (!failed && pend_j >= 0 && !chain_flush<MAXM>(a, pend_j, pend_t, lane, pend_gs, tag)) failed = true;
    if constexpr (XS::kStaged) cp_async_wait_all();  // no copy into this CTA's memory outlives it
    if (failed && lane == 0) {
        atomicOr(reinterpret_cast<unsigned int*>(a.ws), 1u);
        // Wait (bounded) for this warp's copies still in flight: the C::D units from seq on.
        ChainCursor q = c;
        for (int s = 0; s < C::D && q.s < a.n_seg; ++s) {
            mbar_wait_bounded(&bars[(seq + s) % C::D], (uint32_t)(((seq + s) / C::D) & 1), 100000000ull);
            chain_step(a, gw, q);
        }
    }
    // The last CTA to leave resets the per-op tile counts and advances the launch counter.
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        unsigned int* ex = reinterpret_cast<unsigned int*>(a.ws + kChainExitOff);
        if (atomicAdd(ex, 1u) == gridDim.x - 1) {
            __threadfence();
            unsigned int* done = reinterpret_cast<unsigned int*>(a.ws + kChainDoneOff);
            for (int j = 0; j < a.n_ops; ++j) done[j] = 0u;
            *reinterpret_cast<unsigned int*>(a.ws + kChainEpochOff) = tag;  // next launch tags with tag + 1
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
    const int cps = ring_ctas_per_sm(fmt);
    return chain_sm_count() * cps;
}

static int64_t al256(int64_t v) { return (v + 255) / 256 * 256; }

// Execution order: by dependency level (0 = waits for nothing, d + 1 = waits for an op of level
// d), then by the given order.  Each level becomes one segment.
static std::vector<int> chain_levels(const qlin_gemv_op* ops, int n, std::vector<int>& level) {
    level.assign(n, 0);
    for (int j = 0; j < n; ++j) level[j] = ops[j].wait_for >= 0 ? level[ops[j].wait_for] + 1 : 0;
    std::vector<int> order(n);
    for (int j = 0; j < n; ++j) order[j] = j;
    std::stable_sort(order.begin(), order.end(), [&](int x, int y) { return level[x] < level[y]; });
    return order;
}

// Fill the device descriptors (if a is not null); returns the workspace bytes the chain needs.
static int64_t chain_plan(int fmt, int M, const qlin_gemv_op* ops, int n, int W, ChainArgs* a) {
    std::vector<int> level;
    const std::vector<int> order = chain_levels(ops, n, level);
    std::vector<int> pos(n);
    for (int i = 0; i < n; ++i) pos[order[i]] = i;
    std::vector<ChainOp> op(n);
    std::vector<ChainSeg> seg;
    int64_t off = kChainDoneOff + al256(4 * (int64_t)n);
    for (int i = 0; i < n; ++i) {
        const int j = order[i];
        const qlin_gemv_op& u = ops[j];
        if (i == 0 || level[j] != level[order[i - 1]]) seg.push_back(ChainSeg{i, i, 0, 0, 0, 0});
        ChainSeg& sg = seg.back();
        const int epi = u.epilogue & (0xf | QLIN_OUT_BF16);
        const Geometry geo = geometry(fmt, u.N, u.K, (epi & 0xf) == QLIN_EPI_SILU_GATE ? QLIN_PACK_GATE_UP : 0);
        ChainOp& o = op[i];
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
        o.base = sg.U;
        o.seg = (int32_t)seg.size() - 1;
        o.wait_for = u.wait_for >= 0 ? pos[u.wait_for] : -1;
        o.epi = epi;
        for (int k = j + 1; k < n; ++k)
            if (ops[k].wait_for == j) o.epi |= kChainSignal;
        sg.U += o.U;
        sg.end = i + 1;
    }
    int64_t rot = 0;
    for (ChainSeg& sg : seg) {
        sg.q = sg.U / W;
        sg.r = sg.U % W;
        sg.rot = (int32_t)rot;
        rot = (rot + sg.r) % W;  // the next segment's extra units go to the warps after these
    }
    for (int i = 0; i < n; ++i) {
        ChainOp& o = op[i];
        const int q = seg[o.seg].q;
        o.smax = (int32_t)(q == 0 ? o.G : std::min<int64_t>(o.G, (o.G + q - 1) / q + 1));
        o.ws_off = off;
        off += al256((int64_t)o.T * o.smax * 32 * M * 8);
    }
    if (a) {
        for (int i = 0; i < n; ++i) a->op[i] = op[i];
        for (size_t s = 0; s < seg.size(); ++s) a->seg[s] = seg[s];
        a->n_ops = n;
        a->n_seg = (int32_t)seg.size();
    }
    return off;
}

template <int FMT, int MAXM, bool XBF16>
static cudaError_t chain_launch(const ChainArgs* a, int grid, cudaStream_t s, bool pdl) {
    using C = RingCfg<FMT>;
    auto kern = chain_kernel<FMT, MAXM, XBF16>;
    constexpr int kSmem = ChainSmem<FMT, MAXM, XBF16>::kBytes;
    static bool attr_set = false;  // per instantiation; idempotent
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
        if (e != cudaSuccess) return e;
        // The dependency waits need every CTA of the grid resident at once.
        int occ = 0;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, kGemvWarps * 32, kSmem);
        if (e != cudaSuccess) return e;
        if (occ < C::kCtasPerSm) return cudaErrorLaunchOutOfResources;
        attr_set = true;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kGemvWarps * 32);
    cfg.dynamicSmemBytes = kSmem;
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
    a->M = M;
    a->W = grid * kGemvWarps;
    const bool pdl = (flags & QLIN_FLAG_PDL) != 0, bf16 = xdt == QLIN_BF16;
    cudaError_t e;
    if (fmt == QLIN_Q4_0) e = bf16 ? chain_launch_m<QLIN_Q4_0, true>(a, grid, s, pdl) : chain_launch_m<QLIN_Q4_0, false>(a, grid, s, pdl);
    else if (fmt == QLIN_Q8_0) e = bf16 ? chain_launch_m<QLIN_Q8_0, true>(a, grid, s, pdl) : chain_launch_m<QLIN_Q8_0, false>(a, grid, s, pdl);
    else if (fmt == QLIN_MXFP4) e = bf16 ? chain_launch_m<QLIN_MXFP4, true>(a, grid, s, pdl) : chain_launch_m<QLIN_MXFP4, false>(a, grid, s, pdl);
    else if (fmt == QLIN_Q4_K) e = bf16 ? chain_launch_m<QLIN_Q4_K, true>(a, grid, s, pdl) : chain_launch_m<QLIN_Q4_K, false>(a, grid, s, pdl);
    else if (fmt == QLIN_Q6_K) e = bf16 ? chain_launch_m<QLIN_Q6_K, true>(a, grid, s, pdl) : chain_launch_m<QLIN_Q6_K, false>(a, grid, s, pdl);
    else e = bf16 ? chain_launch_m<QLIN_NVFP4, true>(a, grid, s, pdl) : chain_launch_m<QLIN_NVFP4, false>(a, grid, s, pdl);
    delete a;
    return e;
}
