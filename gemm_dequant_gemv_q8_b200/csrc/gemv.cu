// gemv.cu -- dequantize-and-multiply GEMV for M = 1..8 activation rows (sm_100a).
//
// What it computes: y[m][n] = sum_k x[m][k] * W[n][k] for block-quantized W (GGUF Q8_0 / Q4_0,
// NVFP4), the decode-step linear layer of the imp pages (README "Features": NVFP4 block-scaled
// GEMM/GEMV, "dp4a Q8_0 decode"; release notes v0.4.1), optionally followed by the gated-MLP
// epilogue silu(gate) * up (a fused SiLU epilogue is prior art there: release notes v0.4,
// "Fused RMSNormGated+SiLU").  Decode streams every weight byte once, so the kernel is built to
// stream HBM at full rate:
//   * work = units of (32 rows x 256 inputs), contiguous in memory; every warp owns a contiguous,
//     equal share of units (no wave quantization), fetched by cp.async.bulk into a per-warp
//     shared-memory ring that completes on mbarriers (bounded waits, no hangs);
//   * with QLIN_FLAG_PDL the first ring stages are issued before griddepcontrol.wait, so weight
//     streaming overlaps the tail of the previous kernel;
//   * codes are decoded in registers (magic-exponent float construction for Q4_0 / Q8_0,
//     cvt.e2m1x2 for NVFP4) and multiplied with packed fp32x2 FMAs; every product and sum is
//     fp32 and chains stay short (per 32-element block, then per unit, then per tile);
//   * a tile split between warps is finished by the last-arriving warp (atomic ticket, no
//     waiting), which sums the partials in a fixed order: results are deterministic.
#include "gemv_core.cuh"

namespace qlin {

struct GemvArgs {
    const uint8_t* packed;
    int64_t N, K, T, G, U;
    const void* x;
    int64_t ldx;
    int M;
    float* y;
    int64_t ldy;
    uint8_t* ws;
    int64_t Wt;   // number of CTAs sharing the units
    int smax;     // partial slots per tile
};

template <int MAXM>
__device__ __forceinline__ void write_tile(const GemvArgs& a, int64_t t, int lane, float (&v)[MAXM],
                                           int epi, float gs) {
    const int row = (lane >> 3) + 4 * (lane & 7);
#pragma unroll
    for (int m = 0; m < MAXM; ++m) v[m] = v[m] * gs;
    if (epi == QLIN_EPI_SILU_GATE) {
        float u[MAXM];
#pragma unroll
        for (int m = 0; m < MAXM; ++m) u[m] = __shfl_down_sync(0xffffffffu, v[m], 4);
        const int64_t i = t * 16 + row;
        if ((lane & 7) < 4 && i < a.N / 2) {
#pragma unroll
            for (int m = 0; m < MAXM; ++m)
                if (m < a.M) {
                    a.y[m * a.ldy + i] = silu_f32(v[m]) * u[m];
                }
        }
    } else {
        const int64_t n = t * kTileRows + row;
        if (n < a.N) {
#pragma unroll
            for (int m = 0; m < MAXM; ++m)
                if (m < a.M) a.y[m * a.ldy + n] = v[m];
        }
    }
}

// Workspace: [0,256) status word; [256, 256 + 4T rounded to 256) tile tickets; then partials
// [T][smax][32 rows][M] fp32.
__host__ __device__ inline int64_t ws_counters_off() { return 256; }
__host__ __device__ inline int64_t ws_partials_off(int64_t T) { return 256 + ((4 * T + 255) / 256) * 256; }

// Global split-tile fixup between CTAs: store this CTA's partial of tile t, take a ticket; the
// CTA that arrives last sums every partial in CTA order (deterministic) and writes the tile.
template <int MAXM>
__device__ __forceinline__ void global_fixup(const GemvArgs& a, int64_t t, int64_t c, int lane,
                                             float (&acc)[MAXM], int epi, float gs) {
    const int64_t f = t * a.G, l = f + a.G - 1;
    const int64_t C = a.Wt;  // number of CTAs sharing the units
    const int64_t c_first = ((f + 1) * C - 1) / a.U, c_last = ((l + 1) * C - 1) / a.U;
    const int n_t = (int)(c_last - c_first + 1);
    const int slot = (int)(c - c_first);
    float* part = reinterpret_cast<float*>(a.ws + ws_partials_off(a.T));
    int* cnt = reinterpret_cast<int*>(a.ws + ws_counters_off());
    float* mine = part + ((t * a.smax + slot) * 32 + lane) * a.M;
#pragma unroll
    for (int m = 0; m < MAXM; ++m)
        if (m < a.M) __stcg(mine + m, acc[m]);
    __threadfence();
    __syncwarp();
    int ticket = 0;
    if (lane == 0) ticket = atomicAdd(cnt + t, 1);
    ticket = __shfl_sync(0xffffffffu, ticket, 0);
    if (ticket != n_t - 1) return;
    __threadfence();
    float sum[MAXM];
#pragma unroll
    for (int m = 0; m < MAXM; ++m) sum[m] = 0.f;
    for (int s = 0; s < n_t; ++s) {
        const float* src = part + ((t * a.smax + s) * 32 + lane) * a.M;
#pragma unroll
        for (int m = 0; m < MAXM; ++m)
            if (m < a.M) sum[m] += __ldcg(src + m);
    }
    write_tile<MAXM>(a, t, lane, sum, epi, gs);
    if (lane == 0) cnt[t] = 0;  // leave the workspace reusable
}

// ------------------------------------------------------------------ the kernel
// Work split: CTA c owns the contiguous units [c U / C, (c+1) U / C); its warp w owns the w-th
// quarter of that range.  A tile wholly inside one warp's range is written by that warp.  A tile
// shared by warps of one CTA is combined in shared memory, in warp order, after one barrier; only
// tiles at the CTA's two ends can be shared with other CTAs and go through the global fixup.
// Rows of x per pass is MP (1 or 2).  With MAXM <= 2 all rows fit one pass: each lane keeps its 8
// row-part accumulators across the units of a tile (one FMA per block) and reduces once per tile.
// With MAXM > 2 each pass reduces at once.
template <int FMT, int MAXM, bool XBF16, int EPI>
__global__ void __launch_bounds__(kGemvWarps * 32, RingCfg<FMT>::kCtasPerSm) gemv_kernel(const GemvArgs a) {
    using C = RingCfg<FMT>;
    constexpr int MP = MAXM >= 2 ? 2 : 1;
    constexpr bool kOnePass = MAXM <= 2;
    constexpr bool kH = (FMT == QLIN_NVFP4 || FMT == QLIN_MXFP4) && XBF16;  // f16-product path (see load_x_fp4h)
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ float slots[kGemvWarps][2][32][MAXM];  // warp-boundary tile partials
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint8_t* ring = smem + warp * C::D * C::UB;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kGemvWarps * C::D * C::UB) + warp * C::D;
    const uint8_t* units = a.packed + kHdrBytes;

    griddep_launch_dependents();
    // The per-tensor scale lives in the packed header (immutable, like the weights).
    const float gs = format_out_scale<FMT>(a.packed);

    const int U = (int)a.U, nC = (int)a.Wt, G = (int)a.G;
    const int cu0 = (int)((int64_t)blockIdx.x * U / nC), cu1 = (int)((int64_t)(blockIdx.x + 1) * U / nC);
    const int ub = cu0 + (int)((int64_t)warp * (cu1 - cu0) / kGemvWarps);
    const int ue = cu0 + (int)((int64_t)(warp + 1) * (cu1 - cu0) / kGemvWarps);
    const int n = ue - ub;

    if (lane == 0 && n > 0) {
#pragma unroll
        for (int s = 0; s < C::D; ++s) mbar_init(&bars[s], 1);
        fence_mbar_init();
        // Weight prefetch: independent of the previous kernel in the stream.
        for (int s = 0; s < C::D && s < n; ++s) {
            mbar_arrive_expect_tx(&bars[s], C::UB);
            bulk_g2s(ring + s * C::UB, units + (int64_t)(ub + s) * C::UB, C::UB, &bars[s]);
        }
    }
    __syncwarp();
    griddep_wait();  // x, y and the workspace may belong to the previous kernel

    const int part = lane & 7;
    int t = n > 0 ? ub / G : 0, g = n > 0 ? ub - t * G : 0;
    const int t_first = t, t_last = n > 0 ? (ue - 1) / G : -1;
    float acc[MAXM];
#pragma unroll
    for (int m = 0; m < MAXM; ++m) acc[m] = 0.f;
    float acc8[8][MP];
    float2 xv[MP][16];
    float2 xb[MP];
    uint32_t xh[MP][16];
    float xsc[MP][2];
    const void* rows0[MP];
#pragma unroll
    for (int mm = 0; mm < MP; ++mm)
        rows0[mm] = (mm < a.M) ? (XBF16 ? (const void*)(reinterpret_cast<const __nv_bfloat16*>(a.x) + mm * a.ldx)
                                        : (const void*)(reinterpret_cast<const float*>(a.x) + mm * a.ldx))
                               : nullptr;
    if (kOnePass) {
#pragma unroll
        for (int i = 0; i < 8; ++i)
#pragma unroll
            for (int mm = 0; mm < MP; ++mm) acc8[i][mm] = 0.f;
        if (n > 0) {
            if constexpr (kH) {
                load_x_fp4h<MP>(rows0, (int64_t)g * kGroupK + part * 32, a.K, xh, xsc);
            } else {
                load_x_rows<XBF16, MP>(rows0, (int64_t)g * kGroupK + part * 32, a.K, xv);
                prep_x<FMT, MP>(xv, xb);
            }
        }
    }
    bool failed = false;
    int j = 0;
    for (; j < n; ++j) {
        int tn = t, gn = g + 1;
        if (gn == G) {
            gn = 0;
            ++tn;
        }
        const int slot = j % C::D;
        if (!mbar_wait_bounded(&bars[slot], (uint32_t)((j / C::D) & 1))) {
            failed = true;
            break;
        }
        const uint8_t* ubuf = ring + slot * C::UB;
        if (kOnePass && j > 0) {  // activations of this unit (the first unit's were loaded above)
            if constexpr (kH) {
                load_x_fp4h<MP>(rows0, (int64_t)g * kGroupK + part * 32, a.K, xh, xsc);
            } else {
                load_x_rows<XBF16, MP>(rows0, (int64_t)g * kGroupK + part * 32, a.K, xv);
                prep_x<FMT, MP>(xv, xb);
            }
        }
        if (kOnePass) {
            if constexpr (kH) unit_dot_fp4h<MP, true, FMT>(ubuf, lane, xh, xsc, acc8);
            else unit_dot<FMT, MP, true>(ubuf, lane, xv, xb, acc8);
        } else {
            const int64_t k0 = (int64_t)g * kGroupK + part * 32;
#pragma unroll 1
            for (int m0 = 0; m0 < a.M; m0 += MP) {  // passes over pairs of activation rows
                float2 xp[MP][16];
                const void* rows[MP];
#pragma unroll
                for (int mm = 0; mm < MP; ++mm)
                    rows[mm] = (m0 + mm < a.M)
                                   ? (XBF16 ? (const void*)(reinterpret_cast<const __nv_bfloat16*>(a.x) + (m0 + mm) * a.ldx)
                                            : (const void*)(reinterpret_cast<const float*>(a.x) + (m0 + mm) * a.ldx))
                                   : nullptr;
                float res[8][MP];
                if constexpr (kH) {
                    uint32_t xph[MP][16];
                    float xps[MP][2];
                    load_x_fp4h<MP>(rows, k0, a.K, xph, xps);
                    unit_dot_fp4h<MP, false, FMT>(ubuf, lane, xph, xps, res);
                } else {
                    float2 xpb[MP];
                    load_x_rows<XBF16, MP>(rows, k0, a.K, xp);
                    prep_x<FMT, MP>(xp, xpb);
                    unit_dot<FMT, MP>(ubuf, lane, xp, xpb, res);
                }
                float r[MP];
                reduce_scatter8<MP>(res, lane, r);
#pragma unroll
                for (int q = 0; q < MAXM; ++q)  // static register indexing of acc[m0 + mm]
#pragma unroll
                    for (int mm = 0; mm < MP; ++mm)
                        if (q == m0 + mm) acc[q] += r[mm];
            }
        }
        __syncwarp();
        if (lane == 0 && j + C::D < n) {
            fence_proxy_async_smem();
            mbar_arrive_expect_tx(&bars[slot], C::UB);
            bulk_g2s(ring + slot * C::UB, units + (int64_t)(ub + j + C::D) * C::UB, C::UB, &bars[slot]);
        }
        if (tn != t || j + 1 == n) {  // last unit of tile t in this warp's range
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
            if ((int64_t)t * G >= ub && (int64_t)t * G + G <= ue) {
                write_tile<MAXM>(a, t, lane, acc, EPI, gs);  // whole tile inside this warp
            } else {
                const int k = (t == t_first) ? 0 : 1;  // shared tiles are a warp's first or last
#pragma unroll
                for (int m = 0; m < MAXM; ++m) slots[warp][k][lane][m] = acc[m];
            }
#pragma unroll
            for (int m = 0; m < MAXM; ++m) acc[m] = 0.f;
        }
        t = tn;
        g = gn;
    }
    if (failed && lane == 0) {
        // Report, then wait (bounded) for this warp's copies still in flight.
        atomicOr(reinterpret_cast<unsigned int*>(a.ws), 1u);
        const int issued = (j + C::D < n) ? j + C::D : n;
        for (int q = j; q < issued; ++q)
            mbar_wait_bounded(&bars[q % C::D], (uint32_t)((q / C::D) & 1), 100000000ull);
    }
    __syncthreads();  // every warp reaches this, with or without units
    if (failed || n <= 0) return;
    // Combine the tiles this warp is the lowest-index toucher of and that it does not own whole.
    const int range_len = cu1 - cu0;
#pragma unroll 1
    for (int k = 0; k < 2; ++k) {
        const int tt = k == 0 ? t_first : t_last;
        if (k == 1 && t_last == t_first) break;
        const int64_t f = (int64_t)tt * G;
        if (f >= ub && f + G <= ue) continue;  // owned whole by this warp, already written
        // The nearest lower warp with units ends exactly at ub, so a lower warp of this CTA touches
        // the tile iff f < ub and some lower warp has units (ub > cu0).  Then it combines instead.
        if (f < ub && ub > cu0) continue;
        float sum[MAXM];
#pragma unroll
        for (int m = 0; m < MAXM; ++m) sum[m] = 0.f;
        for (int w2 = warp; w2 < kGemvWarps; ++w2) {
            const int b2 = cu0 + (int)((int64_t)w2 * range_len / kGemvWarps);
            const int e2 = cu0 + (int)((int64_t)(w2 + 1) * range_len / kGemvWarps);
            if (e2 <= b2) continue;
            if (b2 >= f + G) break;                      // past the tile
            const int k2 = (b2 / G == tt) ? 0 : 1;        // tt is w2's first or last tile
#pragma unroll
            for (int m = 0; m < MAXM; ++m) sum[m] += slots[w2][k2][lane][m];
        }
        if (f >= cu0 && f + G <= cu1) write_tile<MAXM>(a, tt, lane, sum, EPI, gs);
        else global_fixup<MAXM>(a, tt, blockIdx.x, lane, sum, EPI, gs);
    }
}

// ------------------------------------------------------------------ host side
static int sm_count_cached() {
    static int cache[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    if (!cache[dev]) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        cache[dev] = n;
    }
    return cache[dev];
}

struct GemvPlan {
    int64_t T, G, U, Wt;
    int grid, smax;
    size_t ws_bytes;
};

static GemvPlan plan_gemv(int fmt, int M, int64_t N, int64_t K, int pack_flags) {
    GemvPlan p;
    Geometry geo = geometry(fmt, N, K, pack_flags);
    p.T = geo.T;
    p.G = geo.G;
    p.U = geo.U;
    const int cps = ring_ctas_per_sm(fmt);
    const int64_t cmax = (int64_t)sm_count_cached() * cps;
    int64_t c = (p.U + kGemvWarps - 1) / kGemvWarps;  // at least one unit per warp
    if (c > cmax) c = cmax;
    if (c < 1) c = 1;
    p.grid = (int)c;
    p.Wt = c;  // the kernel splits units between CTAs, then between a CTA's warps
    const int64_t per = p.U / c;  // >= 1 unit per CTA
    int64_t smax = (p.G + per - 1) / per + 1;
    if (smax > c) smax = c;
    p.smax = (int)smax;
    p.ws_bytes = (size_t)ws_partials_off(p.T) + (size_t)p.T * p.smax * 32 * (M > 0 ? M : 1) * 4;
    return p;
}

template <int FMT, int MAXM, bool XBF16, int EPI>
static cudaError_t launch_one(const GemvArgs& a, int grid, cudaStream_t s, bool pdl) {
    using C = RingCfg<FMT>;
    auto kern = gemv_kernel<FMT, MAXM, XBF16, EPI>;
    static bool attr_set = false;  // per instantiation; benign race (idempotent)
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
        if (e != cudaSuccess) return e;
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
    return cudaLaunchKernelEx(&cfg, kern, a);
}

template <int FMT, bool XBF16, int EPI>
static cudaError_t launch_m(const GemvArgs& a, int grid, cudaStream_t s, bool pdl) {
    if (a.M == 1) return launch_one<FMT, 1, XBF16, EPI>(a, grid, s, pdl);
    if (a.M == 2) return launch_one<FMT, 2, XBF16, EPI>(a, grid, s, pdl);
    if (a.M <= 4) return launch_one<FMT, 4, XBF16, EPI>(a, grid, s, pdl);
    return launch_one<FMT, 8, XBF16, EPI>(a, grid, s, pdl);
}

template <int FMT>
static cudaError_t launch_fmt(const GemvArgs& a, bool bf16, int epi, int grid, cudaStream_t s, bool pdl) {
    if (bf16)
        return epi ? launch_m<FMT, true, 1>(a, grid, s, pdl) : launch_m<FMT, true, 0>(a, grid, s, pdl);
    return epi ? launch_m<FMT, false, 1>(a, grid, s, pdl) : launch_m<FMT, false, 0>(a, grid, s, pdl);
}

}  // namespace qlin

using namespace qlin;

extern "C" size_t qlin_gemv_ws_bytes(int fmt, int M, int64_t N, int64_t K, int pack_flags) {
    return plan_gemv(fmt, M, N, K, pack_flags).ws_bytes;
}

// Launch after host-side validation (done in api.cu).
extern "C" cudaError_t qlin_launch_gemv(int fmt, const void* packed, int64_t N, int64_t K,
                                        const void* x, int xdt, int M, int64_t ldx, float* y,
                                        int64_t ldy, int flags, void* ws, cudaStream_t s) {
    const int epi = flags & 0xff;
    const bool pdl = (flags & QLIN_FLAG_PDL) != 0;
    const int pack_flags = epi == QLIN_EPI_SILU_GATE ? QLIN_PACK_GATE_UP : 0;
    GemvPlan p = plan_gemv(fmt, M, N, K, pack_flags);
    GemvArgs a;
    a.packed = (const uint8_t*)packed;
    a.N = N;
    a.K = K;
    a.T = p.T;
    a.G = p.G;
    a.U = p.U;
    a.x = x;
    a.ldx = ldx;
    a.M = M;
    a.y = y;
    a.ldy = ldy;
    a.ws = (uint8_t*)ws;
    a.Wt = p.Wt;
    a.smax = p.smax;
    const bool bf16 = xdt == QLIN_BF16;
    if (fmt == QLIN_Q4_0) return launch_fmt<QLIN_Q4_0>(a, bf16, epi, p.grid, s, pdl);
    if (fmt == QLIN_Q8_0) return launch_fmt<QLIN_Q8_0>(a, bf16, epi, p.grid, s, pdl);
    if (fmt == QLIN_MXFP4) return launch_fmt<QLIN_MXFP4>(a, bf16, epi, p.grid, s, pdl);
    if (fmt == QLIN_Q4_K) return launch_fmt<QLIN_Q4_K>(a, bf16, epi, p.grid, s, pdl);
    if (fmt == QLIN_Q6_K) return launch_fmt<QLIN_Q6_K>(a, bf16, epi, p.grid, s, pdl);
    return launch_fmt<QLIN_NVFP4>(a, bf16, epi, p.grid, s, pdl);
}

// ------------------------------------------------------------------ allocation-free variant
// qlin_gemv_noalloc: the same GEMV for callers that cannot allocate device memory themselves.
// Its workspace is a fixed array in the library's own device memory (held by every GPU that
// loads the library, until the process exits) instead of a caller-provided buffer.
#include <mutex>

namespace qlin {
constexpr size_t kNoAllocScratchBytes = (size_t)8 << 20;  // 8 MiB
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];
static void* g_noalloc_addr[64] = {nullptr};  // device address of the array, per device
static std::mutex g_noalloc_mu;

// Device address of the scratch array on the current device (looked up once per device; in host
// code the array's name is only a stand-in, never a device address).
static cudaError_t noalloc_scratch(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    if (!g_noalloc_addr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        g_noalloc_addr[dev] = p;
    }
    *out = g_noalloc_addr[dev];
    return cudaSuccess;
}
}  // namespace qlin

extern "C" qlin_status_t qlin_gemv_noalloc(qlin_format_t fmt, const void* packed, int64_t N, int64_t K,
                                           const void* x, qlin_dtype_t xdt, int M, int64_t ldx, float* y,
                                           int64_t ldy, int flags, qlin_stream_t stream) {
    if (fmt != QLIN_Q8_0 && fmt != QLIN_Q4_0 && fmt != QLIN_NVFP4 && fmt != QLIN_MXFP4 && fmt != QLIN_Q4_K &&
        fmt != QLIN_Q6_K)
        return QLIN_ERR_INVALID_ARG;
    if (N < 1 || K < 1 || N > ((int64_t)1 << 31) || K > ((int64_t)1 << 31)) return QLIN_ERR_INVALID_ARG;
    if (fmt == QLIN_NVFP4 ? (K % 16) : (fmt == QLIN_Q4_K || fmt == QLIN_Q6_K) ? (K % 256) : (K % 32))
        return QLIN_ERR_INVALID_ARG;
    if (M < 1 || M > 8) return QLIN_ERR_INVALID_ARG;
    if (xdt != QLIN_F32 && xdt != QLIN_BF16) return QLIN_ERR_INVALID_ARG;
    const int epi = flags & 0xff;
    if (epi != QLIN_EPI_NONE && epi != QLIN_EPI_SILU_GATE) return QLIN_ERR_INVALID_ARG;
    if (flags & ~(0xff | QLIN_FLAG_PDL)) return QLIN_ERR_INVALID_ARG;
    if (epi == QLIN_EPI_SILU_GATE && (N % 2)) return QLIN_ERR_INVALID_ARG;
    if (!packed || !x || !y) return QLIN_ERR_INVALID_ARG;
    const int64_t ncols = epi == QLIN_EPI_SILU_GATE ? N / 2 : N;
    if (ldx < K || ldy < ncols) return QLIN_ERR_INVALID_ARG;
    if ((uintptr_t)packed % 256 || (uintptr_t)x % 16 || (uintptr_t)y % 4) return QLIN_ERR_ALIGNMENT;
    if (ldx % (xdt == QLIN_F32 ? 4 : 8)) return QLIN_ERR_ALIGNMENT;
    const int pack_flags = epi == QLIN_EPI_SILU_GATE ? QLIN_PACK_GATE_UP : 0;
    if (geometry(fmt, N, K, pack_flags).U >= ((int64_t)1 << 31)) return QLIN_ERR_UNSUPPORTED;
    const GemvPlan p = plan_gemv(fmt, M, N, K, pack_flags);
    if (p.ws_bytes > kNoAllocScratchBytes) return QLIN_ERR_WORKSPACE;  // beyond the fixed maximum
    void* scratch = nullptr;
    if (noalloc_scratch(&scratch) != cudaSuccess) return QLIN_ERR_CUDA;
    // The array keeps the previous call's contents.  The tile tickets must start at zero (a call
    // that gave up on a wait can leave them set); the partial sums are always written before they
    // are read.  The status word at offset 0 is left alone: it is sticky, like a workspace's, until
    // qlin_gemv_noalloc_status reads and clears it (the array starts zeroed when the library loads).
    if (cudaMemsetAsync((uint8_t*)scratch + ws_counters_off(), 0,
                        (size_t)(ws_partials_off(p.T) - ws_counters_off()), (cudaStream_t)stream) != cudaSuccess)
        return QLIN_ERR_CUDA;
    return qlin_launch_gemv(fmt, packed, N, K, x, xdt, M, ldx, y, ldy, flags, scratch, (cudaStream_t)stream) ==
                   cudaSuccess
               ? QLIN_OK
               : QLIN_ERR_CUDA;
}

extern "C" qlin_status_t qlin_gemv_noalloc_status(qlin_stream_t stream) {
    void* scratch = nullptr;
    if (noalloc_scratch(&scratch) != cudaSuccess) return QLIN_ERR_CUDA;
    return qlin_ws_status(scratch, stream);
}
