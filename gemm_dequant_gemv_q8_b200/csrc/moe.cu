// moe.cu -- top-k routed MoE expert projections for M = 1..8 tokens (sm_100a).
//
// What it computes (Imparo README intro: a Q4_0 MoE decode through "CUDA expert routing"; imp
// README "Features": MoE top-k grouped GEMM, and an ordered, deterministic MoE reduction):
//   route : p = softmax(logits[m]); the top_k experts by p (ties -> lower expert index); weights
//           renormalised over the selected experts;
//   expert: h = silu(W_gate[e] x) * (W_up[e] x), o = W_down[e] h, for every (token, slot);
//   output: y[m] = sum over slots, in slot order, of weight * o.
// Two launches, both graph-capturable and with no device-to-host traffic (the routing is
// computed on the device -- the lesson of the imp release notes v0.7.0, where a host round trip
// of the routing made MoE decode incompatible with CUDA graphs):
//   phase 0: every CTA routes all tokens redundantly in shared memory (M x E is tiny), then the
//            warps stream only the SELECTED experts' gate_up weights, each expert once for all
//            tokens routed to it, and write h with the SiLU-gate epilogue;
//   phase 1: the same for the down weights; each finished (expert, tile) bumps a per-(token, tile)
//            ticket and the last of the token's experts sums the slots in slot order into y.
#include "gemv_core.cuh"

namespace qlin {

constexpr int kMoeMaxTopK = 8;
constexpr int kMoeMaxM = 8;
constexpr int kMoeMaxAct = kMoeMaxM * kMoeMaxTopK;

struct MoeArgs {
    const uint8_t* packed;  // this phase's stacked expert buffers
    int64_t stride;         // bytes between experts' packed buffers
    int E;
    int64_t H, I;
    int top_k;
    const float* logits;  // M x E or NULL (ids / weights are inputs)
    int32_t* ids;         // M x top_k
    float* wts;           // M x top_k
    const void* x;        // phase 0: M x H activations (fp32 / bf16); phase 1: unused
    int M;
    float* y;  // M x H
    float* h;  // M x top_k x I
    float* o;  // M x top_k x H (phase 1 scratch)
    uint8_t* ws;
    int64_t Kin;  // input length of this phase's matrices (H or I)
    int64_t Nout; // output rows (2I or H)
    int64_t T, G, Ue;
    int64_t Wt;
    int smax;
    int64_t cnt_off, part_off, comb_off;
};

struct RouteSmem {
    int n_act;
    int expert[kMoeMaxAct];
    int nrows[kMoeMaxAct];
    int8_t row_m[kMoeMaxAct][kMoeMaxM];
    int8_t row_s[kMoeMaxAct][kMoeMaxM];
    int ids[kMoeMaxM][kMoeMaxTopK];
    float w[kMoeMaxM][kMoeMaxTopK];
    int kvalid[kMoeMaxM];
};

// Routing of all tokens into shared memory (whole CTA participates).
template <int PHASE>
__device__ void moe_route(const MoeArgs& a, RouteSmem& r) {
    const int tid = threadIdx.x;
    if (PHASE == 0 && a.logits) {
        if (tid < a.M) {
            const float* l = a.logits + (int64_t)tid * a.E;
            for (int s = 0; s < a.top_k; ++s) {
                int best = -1;
                for (int e = 0; e < a.E; ++e) {
                    bool taken = false;
                    for (int q = 0; q < s; ++q) taken |= (r.ids[tid][q] == e);
                    if (!taken && (best < 0 || l[e] > l[best])) best = e;
                }
                r.ids[tid][s] = best;
            }
            // renormalised softmax over the selected experts (the full normaliser cancels)
            const float lmax = l[r.ids[tid][0]];
            float z = 0.f;
            for (int s = 0; s < a.top_k; ++s) {
                r.w[tid][s] = expf(l[r.ids[tid][s]] - lmax);
                z += r.w[tid][s];
            }
            for (int s = 0; s < a.top_k; ++s) r.w[tid][s] = r.w[tid][s] / z;
            r.kvalid[tid] = a.top_k;
            if (blockIdx.x == 0)
                for (int s = 0; s < a.top_k; ++s) {
                    a.ids[(int64_t)tid * a.top_k + s] = r.ids[tid][s];
                    a.wts[(int64_t)tid * a.top_k + s] = r.w[tid][s];
                }
        }
    } else {
        if (tid < a.M) {
            int kv = 0;
            for (int s = 0; s < a.top_k; ++s) {
                int e = a.ids[(int64_t)tid * a.top_k + s];
                bool bad = e < 0 || e >= a.E;
                for (int q = 0; q < s; ++q) bad |= (r.ids[tid][q] == e);
                if (bad) {  // invalid or repeated expert: the slot is skipped and reported
                    if (blockIdx.x == 0) atomicOr(reinterpret_cast<unsigned int*>(a.ws), 2u);
                    e = -1;
                } else {
                    ++kv;
                }
                r.ids[tid][s] = e;
                r.w[tid][s] = a.wts[(int64_t)tid * a.top_k + s];
            }
            r.kvalid[tid] = kv;
        }
    }
    __syncthreads();
    if (threadIdx.x < 32) {  // warp 0 compacts the active experts in ascending order
        const int lane = threadIdx.x;
        int n = 0;
        for (int base = 0; base < a.E; base += 32) {
            const int e = base + lane;
            int cnt = 0;
            int8_t rm[kMoeMaxM], rs[kMoeMaxM];
            if (e < a.E)
                for (int m = 0; m < a.M; ++m)
                    for (int s = 0; s < a.top_k; ++s)
                        if (r.ids[m][s] == e && cnt < kMoeMaxM) {
                            rm[cnt] = (int8_t)m;
                            rs[cnt] = (int8_t)s;
                            ++cnt;
                        }
            const unsigned mask = __ballot_sync(0xffffffffu, cnt > 0);
            if (cnt > 0) {
                const int idx = n + __popc(mask & ((1u << lane) - 1u));
                r.expert[idx] = e;
                r.nrows[idx] = cnt;
                for (int c = 0; c < cnt; ++c) {
                    r.row_m[idx][c] = rm[c];
                    r.row_s[idx][c] = rs[c];
                }
            }
            n += __popc(mask);
        }
        if (lane == 0) r.n_act = n;
    }
    __syncthreads();
}

template <int PHASE, int MAXM>
__device__ __forceinline__ void moe_write_tile(const MoeArgs& a, const RouteSmem& r, int act,
                                               int64_t t, int lane, float (&v)[MAXM], float gs) {
    const int row = (lane >> 3) + 4 * (lane & 7);
    const int nr = r.nrows[act];
#pragma unroll
    for (int m = 0; m < MAXM; ++m) v[m] *= gs;
    if (PHASE == 0) {
        float u[MAXM];
#pragma unroll
        for (int m = 0; m < MAXM; ++m) u[m] = __shfl_down_sync(0xffffffffu, v[m], 4);
        const int64_t i = t * 16 + row;
        if ((lane & 7) < 4 && i < a.I) {
#pragma unroll
            for (int q = 0; q < MAXM; ++q)
                if (q < nr) a.h[((int64_t)r.row_m[act][q] * a.top_k + r.row_s[act][q]) * a.I + i] = silu_f32(v[q]) * u[q];
        }
        return;
    }
    const int64_t n = t * kTileRows + row;
    if (n < a.H) {
#pragma unroll
        for (int q = 0; q < MAXM; ++q)
            if (q < nr) __stcg(a.o + ((int64_t)r.row_m[act][q] * a.top_k + r.row_s[act][q]) * a.H + n, v[q]);
    }
    __threadfence();
    __syncwarp();
    int* comb = reinterpret_cast<int*>(a.ws + a.comb_off);
    for (int q = 0; q < nr; ++q) {
        const int m = r.row_m[act][q];
        int ticket = 0;
        if (lane == 0) ticket = atomicAdd(comb + (int64_t)m * a.T + t, 1);
        ticket = __shfl_sync(0xffffffffu, ticket, 0);
        if (ticket == r.kvalid[m] - 1) {  // last of the token's experts for this tile
            __threadfence();
            if (n < a.H) {
                float acc = 0.f;
                for (int s = 0; s < a.top_k; ++s)
                    if (r.ids[m][s] >= 0) acc += r.w[m][s] * __ldcg(a.o + ((int64_t)m * a.top_k + s) * a.H + n);
                a.y[(int64_t)m * a.H + n] = acc;
            }
            if (lane == 0) comb[(int64_t)m * a.T + t] = 0;
        }
    }
}

template <int PHASE, int MAXM>
__device__ __forceinline__ void moe_flush(const MoeArgs& a, const RouteSmem& r, int64_t key, int64_t gw,
                                          int64_t ub, int64_t ue, int64_t Wt, int64_t U, int lane,
                                          float (&acc)[MAXM], float gs) {
    const int act = (int)(key / a.T);
    const int64_t t = key - (int64_t)act * a.T;
    const int64_t f = key * a.G, l = f + a.G - 1;
    if (f >= ub && l < ue) {
        moe_write_tile<PHASE, MAXM>(a, r, act, t, lane, acc, gs);
        return;
    }
    const int64_t c_first = ((f + 1) * Wt - 1) / U, c_last = ((l + 1) * Wt - 1) / U;
    const int n_t = (int)(c_last - c_first + 1);
    const int slot = (int)(gw - c_first);
    const int row = (lane >> 3) + 4 * (lane & 7);
    float* part = reinterpret_cast<float*>(a.ws + a.part_off);
    int* cnt = reinterpret_cast<int*>(a.ws + a.cnt_off);
    float* mine = part + ((key * a.smax + slot) * 32 + row) * a.M;
#pragma unroll
    for (int m = 0; m < MAXM; ++m)
        if (m < a.M) __stcg(mine + m, acc[m]);
    __threadfence();
    __syncwarp();
    int ticket = 0;
    if (lane == 0) ticket = atomicAdd(cnt + key, 1);
    ticket = __shfl_sync(0xffffffffu, ticket, 0);
    if (ticket != n_t - 1) return;
    __threadfence();
    float sum[MAXM];
#pragma unroll
    for (int m = 0; m < MAXM; ++m) sum[m] = 0.f;
    for (int s = 0; s < n_t; ++s) {
        const float* src = part + ((key * a.smax + s) * 32 + row) * a.M;
#pragma unroll
        for (int m = 0; m < MAXM; ++m)
            if (m < a.M) sum[m] += __ldcg(src + m);
    }
    moe_write_tile<PHASE, MAXM>(a, r, act, t, lane, sum, gs);
    if (lane == 0) cnt[key] = 0;
}

template <int FMT, int MAXM, bool XBF16, int PHASE>
__global__ void __launch_bounds__(kGemvWarps * 32, RingCfg<FMT>::kCtasPerSm) moe_kernel(const MoeArgs a) {
    using C = RingCfg<FMT>;
    constexpr int MP = MAXM >= 2 ? 2 : 1;
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ RouteSmem r;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint8_t* ring = smem + warp * C::D * C::UB;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kGemvWarps * C::D * C::UB) + warp * C::D;

    griddep_launch_dependents();
    griddep_wait();  // logits / ids / h come from earlier kernels
    moe_route<PHASE>(a, r);

    const int64_t U = (int64_t)r.n_act * a.Ue;
    const int64_t Wt = a.Wt < U ? a.Wt : U;
    const int64_t gw = (int64_t)blockIdx.x * kGemvWarps + warp;
    if (gw >= Wt) return;
    const int64_t ub = gw * U / Wt, ue = (gw + 1) * U / Wt;
    const int64_t n = ue - ub;
    if (n <= 0) return;

    auto unit_src = [&](int64_t u) -> const uint8_t* {
        const int64_t act = u / a.Ue, v = u - act * a.Ue;
        return a.packed + (int64_t)r.expert[act] * a.stride + kHdrBytes + v * C::UB;
    };
    if (lane == 0) {
#pragma unroll
        for (int s = 0; s < C::D; ++s) mbar_init(&bars[s], 1);
        fence_mbar_init();
        for (int s = 0; s < C::D && s < n; ++s) {
            mbar_arrive_expect_tx(&bars[s], C::UB);
            bulk_g2s(ring + s * C::UB, unit_src(ub + s), C::UB, &bars[s]);
        }
    }
    __syncwarp();

    float acc[MAXM];
#pragma unroll
    for (int m = 0; m < MAXM; ++m) acc[m] = 0.f;
    int64_t cur_key = ub / a.G;  // key = act * T + t  (units of one expert are contiguous)
    float gs = format_out_scale<FMT>(a.packed + (int64_t)r.expert[cur_key / a.T] * a.stride);
    bool failed = false;
    int64_t j = 0;
    for (; j < n; ++j) {
        const int64_t u = ub + j;
        const int64_t key = u / a.G, g = u - key * a.G;
        if (key != cur_key) {
            moe_flush<PHASE, MAXM>(a, r, cur_key, gw, ub, ue, Wt, U, lane, acc, gs);
#pragma unroll
            for (int m = 0; m < MAXM; ++m) acc[m] = 0.f;
            cur_key = key;
            if (FMT == QLIN_NVFP4)
                gs = reinterpret_cast<const PackedHeader*>(a.packed + (int64_t)r.expert[key / a.T] * a.stride)->global_scale;
        }
        const int slot = (int)(j % C::D);
        if (!mbar_wait_bounded(&bars[slot], (uint32_t)((j / C::D) & 1))) {
            failed = true;
            break;
        }
        const uint8_t* ubuf = ring + slot * C::UB;
        const int act = (int)(key / a.T);
        const int nr = r.nrows[act];
        const int64_t k0 = g * kGroupK + (lane & 7) * 32;
#pragma unroll 1
        for (int q0 = 0; q0 < nr; q0 += MP) {
            const void* rows[MP];
#pragma unroll
            for (int mm = 0; mm < MP; ++mm) {
                const int q = q0 + mm;
                if (q >= nr) {
                    rows[mm] = nullptr;
                } else if (PHASE == 0) {
                    const int64_t off = (int64_t)r.row_m[act][q] * a.H;
                    rows[mm] = XBF16 ? (const void*)(reinterpret_cast<const __nv_bfloat16*>(a.x) + off)
                                     : (const void*)(reinterpret_cast<const float*>(a.x) + off);
                } else {
                    rows[mm] = a.h + ((int64_t)r.row_m[act][q] * a.top_k + r.row_s[act][q]) * a.I;
                }
            }
            constexpr bool kXB = (PHASE == 0) && XBF16;
            float res[8][MP];
            if constexpr (kXB && FMT == QLIN_NVFP4) {
                uint32_t xh[MP][16];
                float xsc[MP][2];
                load_x_fp4h<MP>(rows, k0, a.Kin, xh, xsc);
                unit_dot_fp4h<MP>(ubuf, lane, xh, xsc, res);
            } else {
                float2 xv[MP][16];
                float xb[MP];
                load_x_rows<kXB, MP>(rows, k0, a.Kin, xv);
                prep_x<FMT, MP>(xv, xb);
                unit_dot<FMT, MP>(ubuf, lane, xv, xb, res);
            }
            float rr[MP];
            reduce_scatter8<MP>(res, lane, rr);
#pragma unroll
            for (int qq = 0; qq < MAXM; ++qq)
#pragma unroll
                for (int mm = 0; mm < MP; ++mm)
                    if (qq == q0 + mm) acc[qq] += rr[mm];
        }
        __syncwarp();
        if (lane == 0 && j + C::D < n) {
            fence_proxy_async_smem();
            mbar_arrive_expect_tx(&bars[slot], C::UB);
            bulk_g2s(ring + slot * C::UB, unit_src(u + C::D), C::UB, &bars[slot]);
        }
    }
    if (failed) {
        if (lane == 0) {
            atomicOr(reinterpret_cast<unsigned int*>(a.ws), 1u);
            const int64_t issued = (j + C::D < n) ? j + C::D : n;
            for (int64_t qd = j; qd < issued; ++qd)
                mbar_wait_bounded(&bars[qd % C::D], (uint32_t)((qd / C::D) & 1), 100000000ull);
        }
        __syncwarp();
        return;
    }
    moe_flush<PHASE, MAXM>(a, r, cur_key, gw, ub, ue, Wt, U, lane, acc, gs);
}

// ------------------------------------------------------------------ host side
struct MoePlan {
    int64_t nmax;
    int64_t T0, G0, Ue0, T1, G1, Ue1;
    int64_t Wt;
    int grid, smax0, smax1;
    int64_t cnt0, cnt1, comb, part0, part1, o, h;
    size_t bytes;
};

static int moe_sm_count() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
    return n;
}

static int64_t al256(int64_t b) { return (b + 255) / 256 * 256; }

static MoePlan plan_moe(int fmt, int M, int64_t H, int64_t I, int E, int top_k, bool need_h) {
    MoePlan p;
    Geometry g0 = geometry(fmt, 2 * I, H, QLIN_PACK_GATE_UP);
    Geometry g1 = geometry(fmt, H, I, 0);
    p.nmax = (int64_t)M * top_k < E ? (int64_t)M * top_k : E;
    p.T0 = g0.T; p.G0 = g0.G; p.Ue0 = g0.U;
    p.T1 = g1.T; p.G1 = g1.G; p.Ue1 = g1.U;
    const int cps = fmt == QLIN_Q8_0 ? RingCfg<QLIN_Q8_0>::kCtasPerSm : RingCfg<QLIN_Q4_0>::kCtasPerSm;
    p.Wt = (int64_t)moe_sm_count() * cps * kGemvWarps;
    p.grid = (int)(p.Wt / kGemvWarps);
    auto smax_for = [&](int64_t Ue, int64_t G) {
        int64_t per = Ue / p.Wt;  // smallest per-warp share: one active expert
        if (per < 1) per = 1;
        int64_t s = (G + per - 1) / per + 1;
        return (int)(s > p.Wt ? p.Wt : s);
    };
    p.smax0 = smax_for(p.Ue0, p.G0);
    p.smax1 = smax_for(p.Ue1, p.G1);
    int64_t off = 256;
    p.cnt0 = off; off += al256(4 * p.nmax * p.T0);
    p.cnt1 = off; off += al256(4 * p.nmax * p.T1);
    p.comb = off; off += al256(4 * (int64_t)M * p.T1);
    p.part0 = off; off += al256(4 * p.nmax * p.T0 * p.smax0 * 32 * M);
    p.part1 = off; off += al256(4 * p.nmax * p.T1 * p.smax1 * 32 * M);
    p.o = off; off += al256(4 * (int64_t)M * top_k * H);
    p.h = off; if (need_h) off += al256(4 * (int64_t)M * top_k * I);
    p.bytes = (size_t)off;
    return p;
}

template <int FMT, int MAXM, bool XBF16, int PHASE>
static cudaError_t moe_launch(const MoeArgs& a, int grid, cudaStream_t s, bool pdl) {
    using C = RingCfg<FMT>;
    auto kern = moe_kernel<FMT, MAXM, XBF16, PHASE>;
    static bool attr_set = false;
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

template <int FMT, bool XBF16, int PHASE>
static cudaError_t moe_launch_m(const MoeArgs& a, int grid, cudaStream_t s, bool pdl) {
    if (a.M == 1) return moe_launch<FMT, 1, XBF16, PHASE>(a, grid, s, pdl);
    if (a.M == 2) return moe_launch<FMT, 2, XBF16, PHASE>(a, grid, s, pdl);
    return moe_launch<FMT, 8, XBF16, PHASE>(a, grid, s, pdl);
}

template <int FMT>
static cudaError_t moe_fmt(const MoeArgs& a0, const MoeArgs& a1, bool bf16, int grid, cudaStream_t s, bool pdl) {
    cudaError_t e = bf16 ? moe_launch_m<FMT, true, 0>(a0, grid, s, pdl) : moe_launch_m<FMT, false, 0>(a0, grid, s, pdl);
    if (e != cudaSuccess) return e;
    return moe_launch_m<FMT, false, 1>(a1, grid, s, true);  // phase 1 always follows phase 0
}

}  // namespace qlin

using namespace qlin;

extern "C" size_t qlin_moe_ws_bytes(int fmt, int M, int64_t H, int64_t I, int E, int top_k) {
    return plan_moe(fmt, M, H, I, E, top_k, true).bytes;
}

extern "C" cudaError_t qlin_launch_moe(int fmt, const void* gu, const void* dn, int E, int64_t H, int64_t I,
                                       int top_k, const float* logits, int32_t* ids, float* wts, const void* x,
                                       int xdt, int M, float* y, float* h, int flags, void* ws, cudaStream_t s) {
    MoePlan p = plan_moe(fmt, M, H, I, E, top_k, h == nullptr);
    uint8_t* w = (uint8_t*)ws;
    MoeArgs a0 = {};
    a0.E = E; a0.H = H; a0.I = I; a0.top_k = top_k; a0.logits = logits; a0.ids = ids; a0.wts = wts;
    a0.x = x; a0.M = M; a0.y = y; a0.h = h ? h : (float*)(w + p.h); a0.o = (float*)(w + p.o); a0.ws = w;
    a0.Wt = p.Wt;
    MoeArgs a1 = a0;
    a0.packed = (const uint8_t*)gu;
    a0.stride = (int64_t)qlin_packed_bytes((qlin_format_t)fmt, 2 * I, H, QLIN_PACK_GATE_UP);
    a0.Kin = H; a0.Nout = 2 * I; a0.T = p.T0; a0.G = p.G0; a0.Ue = p.Ue0; a0.smax = p.smax0;
    a0.cnt_off = p.cnt0; a0.part_off = p.part0; a0.comb_off = p.comb;
    a1.packed = (const uint8_t*)dn;
    a1.stride = (int64_t)qlin_packed_bytes((qlin_format_t)fmt, H, I, 0);
    a1.logits = nullptr;  // phase 1 reads the routing written by phase 0
    a1.Kin = I; a1.Nout = H; a1.T = p.T1; a1.G = p.G1; a1.Ue = p.Ue1; a1.smax = p.smax1;
    a1.cnt_off = p.cnt1; a1.part_off = p.part1; a1.comb_off = p.comb;
    const bool pdl = (flags & QLIN_FLAG_PDL) != 0;
    const bool bf16 = xdt == QLIN_BF16;
    if (fmt == QLIN_Q4_0) return moe_fmt<QLIN_Q4_0>(a0, a1, bf16, p.grid, s, pdl);
    if (fmt == QLIN_Q8_0) return moe_fmt<QLIN_Q8_0>(a0, a1, bf16, p.grid, s, pdl);
    return moe_fmt<QLIN_NVFP4>(a0, a1, bf16, p.grid, s, pdl);
}
