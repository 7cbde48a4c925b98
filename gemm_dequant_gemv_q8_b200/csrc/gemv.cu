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
    int64_t Wt;   // total warps sharing the units
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

template <int MAXM>
__device__ __forceinline__ void flush_tile(const GemvArgs& a, int64_t t, int64_t gw, int64_t ub,
                                           int64_t ue, int lane, float (&acc)[MAXM], int epi,
                                           float gs) {
    const int64_t f = t * a.G, l = f + a.G - 1;
    if (f >= ub && l < ue) {  // whole tile inside this warp's range
        write_tile<MAXM>(a, t, lane, acc, epi, gs);
        return;
    }
    const int64_t c_first = ((f + 1) * a.Wt - 1) / a.U;
    const int64_t c_last = ((l + 1) * a.Wt - 1) / a.U;
    const int n_t = (int)(c_last - c_first + 1);
    const int slot = (int)(gw - c_first);
    const int row = (lane >> 3) + 4 * (lane & 7);
    float* part = reinterpret_cast<float*>(a.ws + ws_partials_off(a.T));
    int* cnt = reinterpret_cast<int*>(a.ws + ws_counters_off());
    float* mine = part + ((t * a.smax + slot) * 32 + row) * a.M;
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
        const float* src = part + ((t * a.smax + s) * 32 + row) * a.M;
#pragma unroll
        for (int m = 0; m < MAXM; ++m)
            if (m < a.M) sum[m] += __ldcg(src + m);
    }
    write_tile<MAXM>(a, t, lane, sum, epi, gs);
    if (lane == 0) cnt[t] = 0;  // leave the workspace reusable
}

// ------------------------------------------------------------------ the kernel
// Rows of x handled per pass is MP (1 or 2).  With MAXM <= 2 every row fits one pass: each lane
// keeps its 8 row-part accumulators across all units of a tile (one FMA per block) and the
// 8-lane reduce-scatter runs once per tile; x of the next unit is loaded while this one computes.
// With MAXM > 2 the unit is processed in passes of two rows, each pass reduced at once.
template <int FMT, int MAXM, bool XBF16, int EPI>
__global__ void __launch_bounds__(kGemvWarps * 32) gemv_kernel(const GemvArgs a) {
    using C = RingCfg<FMT>;
    constexpr int MP = MAXM >= 2 ? 2 : 1;
    constexpr bool kOnePass = MAXM <= 2;
    extern __shared__ __align__(128) uint8_t smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint8_t* ring = smem + warp * C::D * C::UB;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kGemvWarps * C::D * C::UB) + warp * C::D;
    const uint8_t* units = a.packed + kHdrBytes;

    griddep_launch_dependents();
    // The per-tensor scale lives in the packed header (immutable, like the weights).
    const float gs = FMT == QLIN_NVFP4 ? reinterpret_cast<const PackedHeader*>(a.packed)->global_scale : 1.0f;

    const int U = (int)a.U, Wt = (int)a.Wt, G = (int)a.G;
    const int gw = blockIdx.x * kGemvWarps + warp;
    const int ub = (int)((int64_t)gw * U / Wt), ue = (int)((int64_t)(gw + 1) * U / Wt);
    const int n = ue - ub;
    if (n <= 0) return;

    if (lane == 0) {
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
    int t = ub / G, g = ub - t * G;
    float acc[MAXM];
#pragma unroll
    for (int m = 0; m < MAXM; ++m) acc[m] = 0.f;
    float acc8[8][MP];
    float2 xv[MP][16];
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
        load_x_rows<XBF16, MP>(rows0, (int64_t)g * kGroupK + part * 32, a.K, xv);
    }
    bool failed = false;
    int j = 0;
    for (; j < n; ++j) {
        int tn = t, gn = g + 1;
        if (gn == G) {
            gn = 0;
            ++tn;
        }
        float2 xn[MP][16];
        if (kOnePass && j + 1 < n) load_x_rows<XBF16, MP>(rows0, (int64_t)gn * kGroupK + part * 32, a.K, xn);
        const int slot = j % C::D;
        if (!mbar_wait_bounded(&bars[slot], (uint32_t)((j / C::D) & 1))) {
            failed = true;
            break;
        }
        const uint8_t* ubuf = ring + slot * C::UB;
        if (kOnePass) {
            unit_dot<FMT, MP, true>(ubuf, lane, xv, acc8);
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
                load_x_rows<XBF16, MP>(rows, k0, a.K, xp);
                float res[8][MP];
                unit_dot<FMT, MP>(ubuf, lane, xp, res);
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
            flush_tile<MAXM>(a, t, gw, ub, ue, lane, acc, EPI, gs);
#pragma unroll
            for (int m = 0; m < MAXM; ++m) acc[m] = 0.f;
        }
        t = tn;
        g = gn;
        if (kOnePass) {
#pragma unroll
            for (int mm = 0; mm < MP; ++mm)
#pragma unroll
                for (int q = 0; q < 16; ++q) xv[mm][q] = xn[mm][q];
        }
    }
    if (failed) {
        // Report, then wait (bounded) for this warp's copies still in flight before exiting.
        if (lane == 0) {
            atomicOr(reinterpret_cast<unsigned int*>(a.ws), 1u);
            const int issued = (j + C::D < n) ? j + C::D : n;
            for (int q = j; q < issued; ++q)
                mbar_wait_bounded(&bars[q % C::D], (uint32_t)((q / C::D) & 1), 100000000ull);
        }
        __syncwarp();
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
    const int cps = fmt == QLIN_Q8_0 ? RingCfg<QLIN_Q8_0>::kCtasPerSm : RingCfg<QLIN_Q4_0>::kCtasPerSm;
    const int64_t wmax = (int64_t)sm_count_cached() * cps * kGemvWarps;
    int64_t wt = p.U < wmax ? p.U : wmax;
    p.grid = (int)((wt + kGemvWarps - 1) / kGemvWarps);
    p.Wt = wt;
    const int64_t per = p.U / p.Wt;  // >= 1
    int64_t smax = (p.G + per - 1) / per + 1;
    if (smax > p.Wt) smax = p.Wt;
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
    if (fmt != QLIN_Q8_0 && fmt != QLIN_Q4_0 && fmt != QLIN_NVFP4) return QLIN_ERR_INVALID_ARG;
    if (N < 1 || K < 1 || N > ((int64_t)1 << 31) || K > ((int64_t)1 << 31)) return QLIN_ERR_INVALID_ARG;
    if (fmt == QLIN_NVFP4 ? (K % 16) : (K % 32)) return QLIN_ERR_INVALID_ARG;
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
    // The array keeps the previous call's contents: the status word and the tile tickets must
    // start at zero (the partial sums are always written before they are read).
    if (cudaMemsetAsync(scratch, 0, (size_t)ws_partials_off(p.T), (cudaStream_t)stream) != cudaSuccess)
        return QLIN_ERR_CUDA;
    return qlin_launch_gemv(fmt, packed, N, K, x, xdt, M, ldx, y, ldy, flags, scratch, (cudaStream_t)stream) ==
                   cudaSuccess
               ? QLIN_OK
               : QLIN_ERR_CUDA;
}
