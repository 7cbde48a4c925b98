// moe.cu -- top-k routed MoE expert projections for M = 1..8 tokens, in one launch (sm_100a).
//
// What it computes (Imparo README intro: a Q4_0 MoE decode through "CUDA expert routing"; imp
// README "Features": MoE top-k grouped GEMM, and an ordered, deterministic MoE reduction):
//   route : p = softmax(logits[m]); the top_k experts by p (ties -> lower expert index); weights
//           renormalised over the selected experts;
//   expert: h = silu(W_gate[e] x) * (W_up[e] x), o = W_down[e] h, for every (token, slot);
//   output: y[m] = sum over slots, in slot order, of weight * o.
// The routing is computed on the device -- no host round trip, so the layer is graph-capturable
// (the lesson of the imp release notes v0.7.0, where a host round trip of the routing made MoE
// decode incompatible with CUDA graphs) -- redundantly by every CTA in shared memory (M x E is
// tiny), which then plans the launch on the device: the work entries (a selected expert with up
// to two of the tokens routed to it; an expert chosen by more tokens gets more entries) put their
// gate_up tiles in step 0 and their down tiles in step 1, and each step's tiles are split into
// one contiguous range per CTA.  A CTA owns its tiles whole: its four warps take the tiles' units
// (k-groups) in turn, each through its own ring of bulk copies, and add their parts in shared
// memory.  A CTA reaching an entry's down tiles waits (bounded) only for that entry's gate_up
// tiles.  The last of a token's experts to write a down tile adds the token's slot outputs for
// that tile in slot order (a ticket per token and tile): deterministic.
#include "gemv_core.cuh"

namespace qlin {

constexpr int kMoeMaxTopK = 8;
constexpr int kMoeMaxM = 8;
constexpr int kMoeMaxAct = kMoeMaxM * kMoeMaxTopK;  // work entries (an entry holds >= 1 row)
constexpr int kMoeEntryRows = 2;                     // rows per work entry

struct MoeArgs {
    const uint8_t* gu;  // E stacked gate_up buffers (QLIN_PACK_GATE_UP, 2I x H)
    const uint8_t* dn;  // E stacked down buffers (H x I)
    int64_t gu_stride, dn_stride;
    int E, H, I, top_k, M;
    const float* logits;  // M x E or NULL (ids / weights are inputs)
    int32_t* ids;         // M x top_k
    float* wts;           // M x top_k
    const void* x;        // M x H activations (fp32 / bf16)
    float* y;             // M x H
    float* h;             // M x top_k x I  (SiLU-gate outputs)
    float* o;             // M x top_k x H  (down outputs, workspace)
    uint8_t* ws;
    int T0, G0, U0;       // per expert, gate_up: tiles (16 gate + 16 up rows), k-groups over H, units
    int T1, G1, U1;       // per expert, down: tiles of 32 rows of H, k-groups over I, units
};

// Workspace: [0,4) status word (bit 0 timeout, bit 1 bad expert id); [64,68) exit counter;
// [256, ...) per-work-entry gate_up tile counts (reset by the last CTA to leave); per-(token, down
// tile) combine tickets (reset by the combine that uses them, or, after a failed wait, by the
// last CTA to leave); then the down outputs o and the SiLU-gate outputs h.
constexpr int64_t kMoeExitOff = 64;
constexpr int64_t kMoeDoneOff = 256;
constexpr int kMoeMaxT1 = 1024;  // down tiles per expert (H <= 32768)
__host__ __device__ inline int64_t moe_comb_off() { return kMoeDoneOff + 4 * kMoeMaxAct; }
__host__ __device__ inline int64_t moe_head_bytes() { return moe_comb_off() + 4 * (int64_t)kMoeMaxM * kMoeMaxT1; }

// ------------------------------------------------------------------ device-side plan
// Segment s (0 = gate_up, 1 = down) of the work entries: Tt = n_act T tiles of G k-group units
// each.  CTA v = (blockIdx - rot) mod gridDim owns tiles [v q + min(v, r), + q + (v < r)) whole:
// its four warps take the tiles' units in turn and add their parts in shared memory, so no tile
// is shared between CTAs and nothing waits for another CTA's piece of a tile.
struct MoeSeg {
    int Tt, q, r, rot, G, T;
};

struct RouteSmem {
    MoeSeg sg[2];  // the device-side plan (identical in every CTA)
    int tb[2], te[2];  // this CTA's tiles of each step
    int n_act;
    int expert[kMoeMaxAct];
    int nrows[kMoeMaxAct];
    int8_t row_m[kMoeMaxAct][kMoeEntryRows];
    int8_t row_s[kMoeMaxAct][kMoeEntryRows];
    int ids[kMoeMaxM][kMoeMaxTopK];
    float w[kMoeMaxM][kMoeMaxTopK];
    int kvalid[kMoeMaxM];  // valid slots of each token
};

// Routing of all tokens into shared memory (whole CTA participates).  With logits, one warp per
// token: lane l holds the logits of experts l + 32 j, and every expert's slot is its rank in the
// order "larger logit first, a tie to the lower expert index" (NaN ranks as -inf), counted
// against all experts at once -- independent comparisons, where top_k argmax rounds would be a
// chain of dependent shuffles.  The selection is the one a sequential scan with a strict
// comparison makes.  CTA 0 also writes ids and weights out.  Without logits, invalid or repeated
// input ids skip their slot and set status bit 1.
constexpr int kMoeMaxE = 256;

__device__ __forceinline__ float moe_key(float v) { return v != v ? -INFINITY : v; }

__device__ __forceinline__ void moe_route(const MoeArgs& a, RouteSmem& r) {
    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31, nw = blockDim.x >> 5;
    if (a.logits) {
        constexpr int kTokPerWarp = (kMoeMaxM + kGemvWarps - 1) / kGemvWarps;
        constexpr int kJ = kMoeMaxE / 32;
        const int J = (a.E + 31) >> 5;
        float vall[kTokPerWarp][kJ];  // all of this warp's logits first: their loads fly together
#pragma unroll
        for (int i = 0; i < kTokPerWarp; ++i) {
            const int m = warp + i * nw;
#pragma unroll
            for (int j = 0; j < kJ; ++j) {
                const int e = lane + 32 * j;
                vall[i][j] = (m < a.M && e < a.E) ? moe_key(__ldcg(a.logits + (int64_t)m * a.E + e)) : -INFINITY;
            }
        }
#pragma unroll
        for (int i = 0; i < kTokPerWarp; ++i) {
            const int m = warp + i * nw;
            if (m >= a.M) break;
            int rank[kJ];
#pragma unroll
            for (int j = 0; j < kJ; ++j) rank[j] = 0;
            if (J == 1) {
                const float v = vall[i][0];
#pragma unroll
                for (int src = 0; src < 32; ++src) {
                    const float ov = __shfl_sync(0xffffffffu, v, src);
                    rank[0] += (src < a.E) & ((ov > v) | ((ov == v) & (src < lane)));
                }
            } else {
#pragma unroll
                for (int jj = 0; jj < kJ; ++jj) {
                    if (jj >= J) break;
#pragma unroll 4
                    for (int src = 0; src < 32; ++src) {
                        const float ov = __shfl_sync(0xffffffffu, vall[i][jj], src);
                        const int oe = src + 32 * jj;
#pragma unroll
                        for (int j = 0; j < kJ; ++j)
                            if (j < J)
                                rank[j] += (oe < a.E) & ((ov > vall[i][j]) | ((ov == vall[i][j]) & (oe < lane + 32 * j)));
                    }
                }
            }
#pragma unroll
            for (int j = 0; j < kJ; ++j) {
                const int e = lane + 32 * j;
                if (e < a.E && rank[j] < a.top_k) {
                    r.ids[m][rank[j]] = e;
                    r.w[m][rank[j]] = vall[i][j];
                }
            }
            __syncwarp();
            // weights renormalised over the selected experts: exp(l_s - l_0) / sum
            const float ex = lane < a.top_k ? expf(r.w[m][lane] - r.w[m][0]) : 0.f;
            float z = ex;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
            __syncwarp();
            if (lane < a.top_k) {
                const float w = ex / z;
                r.w[m][lane] = w;
                if (blockIdx.x == 0) {
                    a.ids[(int64_t)m * a.top_k + lane] = r.ids[m][lane];
                    a.wts[(int64_t)m * a.top_k + lane] = w;
                }
            }
        }
    } else if (tid < a.M) {
        for (int s = 0; s < a.top_k; ++s) {
            int e = a.ids[(int64_t)tid * a.top_k + s];
            bool bad = e < 0 || e >= a.E;
            for (int q = 0; q < s; ++q) bad |= (r.ids[tid][q] == e);
            if (bad) {
                if (blockIdx.x == 0) atomicOr(reinterpret_cast<unsigned int*>(a.ws), 2u);
                e = -1;
            }
            r.ids[tid][s] = e;
            r.w[tid][s] = a.wts[(int64_t)tid * a.top_k + s];
        }
    }
    __syncthreads();
    if (tid < a.M) {
        int kv = 0;
        for (int q = 0; q < a.top_k; ++q) kv += r.ids[tid][q] >= 0;
        r.kvalid[tid] = kv;
        if (kv == 0 && blockIdx.x == 0)  // no expert: the token's output is zero
            for (int n = 0; n < a.H; ++n) a.y[(int64_t)tid * a.H + n] = 0.f;
    }
    if (warp == 0) {
        // Warp 0 lists the work entries: the selected experts in ascending order, each expert's
        // rows in (token, slot) order, cut into entries of at most kMoeEntryRows rows (an expert
        // chosen by more tokens streams its weights once per entry, the later reads mostly from L2).
        int n = 0;
        for (int base = 0; base < a.E; base += 32) {
            const int e = base + lane;
            int cnt = 0;  // at most one slot per token: cnt <= M
            for (int m = 0; m < a.M; ++m)
                for (int q = 0; q < a.top_k; ++q) cnt += r.ids[m][q] == e;
            const int ne = (cnt + kMoeEntryRows - 1) / kMoeEntryRows;
            int incl = ne;  // inclusive prefix sum of the entries over the lanes
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int t = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += t;
            }
            int idx = n + incl - ne, c = 0;
            for (int m = 0; m < a.M; ++m)
                for (int q = 0; q < a.top_k; ++q)
                    if (r.ids[m][q] == e) {
                        if (c == 0) {
                            r.expert[idx] = e;
                            r.nrows[idx] = min(kMoeEntryRows, cnt);
                        }
                        r.row_m[idx][c] = (int8_t)m;
                        r.row_s[idx][c] = (int8_t)q;
                        if (++c == kMoeEntryRows) {
                            c = 0;
                            ++idx;
                            cnt -= kMoeEntryRows;
                        }
                    }
            n += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) r.n_act = n;
    }
    __syncthreads();
}

// A warp's position in its CTA's units of segment s (tile-major, k-group minor): list index i
// (this warp takes i = warp, warp + 4, ...), local tile jl and k-group g, work entry act and its
// tile t; n = units of the CTA in the segment.  Advanced incrementally (no division per unit).
struct MoeCursor {
    int s, i, jl, g, act, t, n;
};

__device__ __forceinline__ void moe_seek(const MoeSeg (&sg)[2], const int (&tb)[2], const int (&te)[2], int warp,
                                         MoeCursor& c, int s) {
    for (; s < 2; ++s) {
        const int n = (te[s] - tb[s]) * sg[s].G;
        if (warp < n) {
            c.s = s;
            c.i = warp;
            c.jl = warp / sg[s].G;
            c.g = warp - c.jl * sg[s].G;
            const int T = tb[s] + c.jl;
            c.act = T / sg[s].T;
            c.t = T - c.act * sg[s].T;
            c.n = n;
            return;
        }
    }
    c.s = 2;
    c.i = c.jl = c.g = c.act = c.t = c.n = 0;
}

__device__ __forceinline__ void moe_step(const MoeSeg (&sg)[2], const int (&tb)[2], const int (&te)[2], int warp,
                                         MoeCursor& c) {
    c.i += kGemvWarps;
    if (c.i >= c.n) {
        moe_seek(sg, tb, te, warp, c, c.s + 1);
        return;
    }
    const MoeSeg& S = sg[c.s];
    c.g += kGemvWarps;
    while (c.g >= S.G) {
        c.g -= S.G;
        ++c.jl;
        if (++c.t == S.T) {
            c.t = 0;
            ++c.act;
        }
    }
}

template <int FMT>
__device__ __forceinline__ const uint8_t* moe_unit_src(const MoeArgs& a, const RouteSmem& r, const MoeSeg (&sg)[2],
                                                       const MoeCursor& c) {
    const uint8_t* base = c.s == 0 ? a.gu + (int64_t)r.expert[c.act] * a.gu_stride
                                   : a.dn + (int64_t)r.expert[c.act] * a.dn_stride;
    return base + kHdrBytes + ((int64_t)c.t * sg[c.s].G + c.g) * RingCfg<FMT>::UB;
}

// Write tile t of active expert `act` in segment s: h rows with the SiLU gate (s = 0) or the
// down outputs o (s = 1), one row per (token, slot) routed to the expert.
template <int MAXM>
__device__ __forceinline__ void moe_write_tile(const MoeArgs& a, const RouteSmem& r, int s, int act, int t,
                                               int lane, float (&v)[MAXM], float gs) {
    const int row = (lane >> 3) + 4 * (lane & 7);
    const int nr = r.nrows[act];
#pragma unroll
    for (int m = 0; m < MAXM; ++m) v[m] *= gs;
    if (s == 0) {
        float u[MAXM];
#pragma unroll
        for (int m = 0; m < MAXM; ++m) u[m] = __shfl_down_sync(0xffffffffu, v[m], 4);
        const int i = t * 16 + row;
        if ((lane & 7) < 4 && i < a.I) {
#pragma unroll
            for (int q = 0; q < MAXM; ++q)
                if (q < nr) a.h[((int64_t)r.row_m[act][q] * a.top_k + r.row_s[act][q]) * a.I + i] = silu_f32(v[q]) * u[q];
        }
        // Count the tile for the down units of this expert: the warp barrier orders every lane's
        // stores before lane 0's release (which is cumulative over them).
        __syncwarp();
        if (lane == 0) {
            unsigned int* done = reinterpret_cast<unsigned int*>(a.ws + kMoeDoneOff);
            asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(done + act) : "memory");
        }
        return;
    }
    // Down tile: store the slot outputs, then take a ticket per token (lane q for the expert's row
    // q, all at once); the last of a token's experts for this tile adds the token's slot outputs
    // in slot order into y.  The warp barriers carry the lanes' stores into the tickets' release
    // and the tickets' acquire into every lane's loads.
    const int n = t * kTileRows + row;
    if (n < a.H) {
#pragma unroll
        for (int q = 0; q < MAXM; ++q)
            if (q < nr) __stcg(a.o + ((int64_t)r.row_m[act][q] * a.top_k + r.row_s[act][q]) * a.H + n, v[q]);
    }
    __syncwarp();
    unsigned int* comb = reinterpret_cast<unsigned int*>(a.ws + moe_comb_off());
    unsigned int tk = 0;
    if (lane < nr)
        asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;"
                     : "=r"(tk)
                     : "l"(comb + r.row_m[act][lane] * a.T1 + t)
                     : "memory");
    __syncwarp();
    for (int q = 0; q < nr; ++q) {
        const int m = r.row_m[act][q];
        const unsigned int ticket = __shfl_sync(0xffffffffu, tk, q);
        if (ticket == (unsigned)r.kvalid[m] - 1u) {
            if (n < a.H) {
                float sum = 0.f;
                for (int k = 0; k < a.top_k; ++k)
                    if (r.ids[m][k] >= 0) sum += r.w[m][k] * __ldcg(a.o + ((int64_t)m * a.top_k + k) * a.H + n);
                a.y[(int64_t)m * a.H + n] = sum;
            }
            if (lane == 0) comb[m * a.T1 + t] = 0u;  // leave the workspace reusable
        }
    }
}

// Bounded wait until *p >= target (~2 s, or the workspace's wait budget); false on timeout.
__device__ __forceinline__ bool moe_wait_count(const unsigned int* p, uint32_t target, const void* ws) {
    auto ld = [&]() {
        uint32_t v;
        asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
        return v;
    };
    if (__all_sync(0xffffffffu, ld() >= target)) return true;
    const uint64_t t0 = globaltimer_ns(), budget = ws_wait_budget_ns(ws);
    for (uint32_t it = 1;; ++it) {
        __nanosleep(64);
        if (__all_sync(0xffffffffu, ld() >= target)) return true;
        if (globaltimer_ns() - t0 > budget) return false;
    }
}

// Row pointers of the pass starting at row q0 of active expert `act` in segment s (segment 0:
// the tokens' x rows, XB: bf16; segment 1: their fp32 h rows); NULL past the expert's rows.
template <int MP, bool XB>
__device__ __forceinline__ void moe_rows(const MoeArgs& a, const RouteSmem& r, int s, int act, int q0,
                                         const void* (&rows)[MP]) {
    const int nr = r.nrows[act];
#pragma unroll
    for (int mm = 0; mm < MP; ++mm) {
        const int q = q0 + mm;
        if (q >= nr) {
            rows[mm] = nullptr;
        } else if (s == 0) {
            const int64_t off = (int64_t)r.row_m[act][q] * a.H;
            rows[mm] = XB ? (const void*)(reinterpret_cast<const __nv_bfloat16*>(a.x) + off)
                          : (const void*)(reinterpret_cast<const float*>(a.x) + off);
        } else {
            rows[mm] = a.h + ((int64_t)r.row_m[act][q] * a.top_k + r.row_s[act][q]) * a.I;
        }
    }
}

// One unit of segment s for the rows of work entry `act` (at most kMoeEntryRows = MAXM rows),
// accumulated into acc8 across a tile's units.  xs: the rows already staged in shared memory (or
// NULL); after_first_load() runs once the activations are in registers.
template <int FMT, int MAXM, bool XB, typename F>
__device__ __forceinline__ void moe_unit(const MoeArgs& a, const RouteSmem& r, int s, int act, int g,
                                         const uint8_t* ubuf, int lane, float (&acc8)[8][MAXM],
                                         const uint8_t* xs, F&& after_first_load) {
    constexpr int MP = MAXM;
    const int64_t Kin = s == 0 ? a.H : a.I;
    const int part = lane & 7;
    const int64_t k0 = (int64_t)g * kGroupK + part * 32;
    const void* rows[MP];
    moe_rows<MP, XB>(a, r, s, act, 0, rows);
    if constexpr (XB && (FMT == QLIN_NVFP4 || FMT == QLIN_MXFP4)) {
        uint32_t xh[MP][16];
        float xsc[MP][2];
        if (xs != nullptr)
            load_x_fp4h_staged<MP>(xs, part, xh, xsc);
        else
            load_x_fp4h<MP, true>(rows, k0, Kin, xh, xsc);
        after_first_load();
        unit_dot_fp4h<MP, true, FMT>(ubuf, lane, xh, xsc, acc8);
    } else {
        float2 xv[MP][16];
        float2 xb[MP];
        if (xs != nullptr)
            load_x_staged<XB, MP>(xs, part, xv);
        else
            load_x_rows<XB, MP, true>(rows, k0, Kin, xv);
        after_first_load();
        prep_x<FMT, MP>(xv, xb);
        unit_dot<FMT, MP, true>(ubuf, lane, xv, xb, acc8);
    }
}

// Shared memory of the MoE kernel: the per-warp weight rings and their barriers, then (except
// Q8_0 and Q6_K, whose rings leave no room) one activation stage per warp: the next unit's rows, copied
// while the current unit computes.
template <int FMT, int MAXM>
struct MoeSmem {
    static constexpr int MP = MAXM;
    static constexpr bool kStaged = FMT != QLIN_Q8_0 && FMT != QLIN_Q6_K;
    static constexpr int kStageBytes = MP * XStage<false>::kRowBytes;  // fp32 layout; bf16 rows fit
    static constexpr int kXOff = (RingCfg<FMT>::kSmem + 127) / 128 * 128;
    static constexpr int kBytes = kStaged ? kXOff + kGemvWarps * kStageBytes : RingCfg<FMT>::kSmem;
};

template <int FMT>
__device__ __forceinline__ float moe_scale(const MoeArgs& a, const RouteSmem& r, int s, int act) {
    return format_out_scale<FMT>(s == 0 ? a.gu + (int64_t)r.expert[act] * a.gu_stride
                                        : a.dn + (int64_t)r.expert[act] * a.dn_stride);
}

template <int FMT, int MAXM, bool XBF16>
__global__ void __launch_bounds__(kGemvWarps * 32, RingCfg<FMT>::kCtasPerSm) moe_kernel(const __grid_constant__ MoeArgs a) {
    using C = RingCfg<FMT>;
    using MS = MoeSmem<FMT, MAXM>;
    constexpr int MP = MAXM;
    static_assert(MAXM >= 1 && MAXM <= kMoeEntryRows, "rows per work entry");
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ RouteSmem r;
    __shared__ float red[2][kGemvWarps][32][MP];  // the warps' parts of a tile (by tile parity)
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint8_t* ring = smem + warp * C::D * C::UB;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kGemvWarps * C::D * C::UB) + warp * C::D;
    uint8_t* xst = smem + MS::kXOff + warp * MS::kStageBytes;  // used only if MS::kStaged

    griddep_launch_dependents();
    griddep_wait();  // logits / ids / x come from earlier kernels
    moe_route(a, r);
    if (threadIdx.x == 0) {
        MoeSeg* sp = r.sg;
        sp[0].G = a.G0; sp[0].T = a.T0;
        sp[1].G = a.G1; sp[1].T = a.T1;
        for (int s = 0; s < 2; ++s) {
            sp[s].Tt = r.n_act * sp[s].T;
            sp[s].q = sp[s].Tt / (int)gridDim.x;
            sp[s].r = sp[s].Tt % (int)gridDim.x;
        }
        sp[0].rot = 0;
        sp[1].rot = sp[0].r;  // the second step's extra tiles go to the CTAs after the first's
        for (int s = 0; s < 2; ++s) {
            int v = (int)blockIdx.x - sp[s].rot;
            if (v < 0) v += gridDim.x;
            r.tb[s] = v * sp[s].q + min(v, sp[s].r);
            r.te[s] = r.tb[s] + sp[s].q + (v < sp[s].r ? 1 : 0);
        }
    }
    __syncthreads();
    const MoeSeg (&sg)[2] = r.sg;
    const int (&tb)[2] = r.tb;
    const int (&te)[2] = r.te;

    MoeCursor c;
    moe_seek(sg, tb, te, warp, c, 0);
    MoeCursor p = c;  // producer cursor, C::D units ahead once primed
    if (lane == 0) {
#pragma unroll
        for (int s = 0; s < C::D; ++s) mbar_init(&bars[s], 1);
        fence_mbar_init();
        for (int s = 0; s < C::D && p.s < 2; ++s) {
            mbar_arrive_expect_tx(&bars[s], C::UB);
            bulk_g2s(ring + s * C::UB, moe_unit_src<FMT>(a, r, sg, p), C::UB, &bars[s]);
            moe_step(sg, tb, te, warp, p);
        }
    }
    __syncwarp();
    p.s = __shfl_sync(0xffffffffu, p.s, 0);
    p.i = __shfl_sync(0xffffffffu, p.i, 0);
    p.jl = __shfl_sync(0xffffffffu, p.jl, 0);
    p.g = __shfl_sync(0xffffffffu, p.g, 0);
    p.act = __shfl_sync(0xffffffffu, p.act, 0);
    p.t = __shfl_sync(0xffffffffu, p.t, 0);
    p.n = __shfl_sync(0xffffffffu, p.n, 0);

    float acc8[8][MP];
    bool failed = false;
    int seq = 0, waited = -1, tc = 0;
    bool xready = false;  // the current unit's rows are already staged
    auto stage_unit = [&](const MoeCursor& u) {
        const void* rows[MP];
        if (!XBF16 || u.s == 1) {  // fp32 rows: x (step 0) or h (step 1)
            moe_rows<MP, false>(a, r, u.s, u.act, 0, rows);
            stage_x_rows<false, MP>(rows, u.s == 0 ? a.H : a.I, u.g, xst, lane, a.ws);
        } else {
            moe_rows<MP, true>(a, r, 0, u.act, 0, rows);
            stage_x_rows<true, MP>(rows, a.H, u.g, xst, lane, a.ws);
        }
    };
    const unsigned int* done = reinterpret_cast<const unsigned int*>(a.ws + kMoeDoneOff);
    for (int s = 0; s < 2; ++s) {
        const int T = sg[s].T;
        int act = tb[s] / T, t = tb[s] - act * T;  // the CTA's current tile
        float gs = act < r.n_act ? moe_scale<FMT>(a, r, s, act) : 1.f;
        for (int jl = 0; jl < te[s] - tb[s]; ++jl, ++tc) {
            // down units read h: wait (bounded) for this entry's gate_up tiles
            if (s == 1 && act != waited && !failed) {
                waited = act;
                if (!moe_wait_count(done + act, (uint32_t)a.T0, a.ws)) failed = true;
            }
#pragma unroll
            for (int i = 0; i < 8; ++i)
#pragma unroll
                for (int mm = 0; mm < MP; ++mm) acc8[i][mm] = 0.f;
            while (!failed && c.s == s && c.jl == jl) {
                const int slot = seq % C::D;
                if (!mbar_wait_bounded(&bars[slot], (uint32_t)((seq / C::D) & 1))) {
                    failed = true;
                    break;
                }
                const uint8_t* ubuf = ring + slot * C::UB;
                const uint8_t* xs = nullptr;
                MoeCursor cn = c;  // the next unit of this warp
                bool stage_next = false;
                if constexpr (MS::kStaged) {
                    if (!xready) stage_unit(c);
                    cp_async_wait_all();
                    __syncwarp();
                    xs = xst;
                    moe_step(sg, tb, te, warp, cn);
                    // h rows of a down unit may be read only after that entry's wait
                    stage_next = cn.s < 2 && (cn.s == 0 || (c.s == 1 && cn.act == c.act));
                }
                auto after_first_load = [&]() {  // the stage is free: copy the next unit's rows into it
                    if constexpr (MS::kStaged) {
                        __syncwarp();
                        if (stage_next) stage_unit(cn);
                    }
                };
                if constexpr (!XBF16)  // one copy of the unit code for both steps (instruction cache)
                    moe_unit<FMT, MAXM, false>(a, r, s, c.act, c.g, ubuf, lane, acc8, xs, after_first_load);
                else if (s == 0)
                    moe_unit<FMT, MAXM, true>(a, r, 0, c.act, c.g, ubuf, lane, acc8, xs, after_first_load);
                else
                    moe_unit<FMT, MAXM, false>(a, r, 1, c.act, c.g, ubuf, lane, acc8, xs, after_first_load);
                xready = stage_next;
                __syncwarp();
                // Refill this slot with the producer's next unit (the ring runs C::D units ahead).
                if (lane == 0 && p.s < 2) {
                    fence_proxy_async_smem();
                    mbar_arrive_expect_tx(&bars[slot], C::UB);
                    bulk_g2s(ring + slot * C::UB, moe_unit_src<FMT>(a, r, sg, p), C::UB, &bars[slot]);
                }
                if (p.s < 2) moe_step(sg, tb, te, warp, p);
                ++seq;
                moe_step(sg, tb, te, warp, c);
            }
            // The tile's parts: each warp's (zero if it had no unit of the tile), added in warp
            // order by one warp (rotating) -- deterministic.
            float rr[MP];
            reduce_scatter8<MP>(acc8, lane, rr);
#pragma unroll
            for (int mm = 0; mm < MP; ++mm) red[tc & 1][warp][lane][mm] = rr[mm];
            __syncthreads();
            if (warp == tc % kGemvWarps) {
                float v[MP];
#pragma unroll
                for (int mm = 0; mm < MP; ++mm) v[mm] = 0.f;
#pragma unroll
                for (int w = 0; w < kGemvWarps; ++w)
#pragma unroll
                    for (int mm = 0; mm < MP; ++mm) v[mm] += red[tc & 1][w][lane][mm];
                moe_write_tile<MAXM>(a, r, s, act, t, lane, v, gs);
            }
            if (++t == T && jl + 1 < te[s] - tb[s]) {
                t = 0;
                ++act;
                gs = moe_scale<FMT>(a, r, s, act);
            }
        }
    }
    if constexpr (MS::kStaged) cp_async_wait_all();  // no copy into this CTA's memory outlives it
    if (failed && lane == 0) {
        atomicOr(reinterpret_cast<unsigned int*>(a.ws), 1u);
        MoeCursor q = c;  // wait (bounded) for this warp's copies still in flight
        for (int s = 0; s < C::D && q.s < 2; ++s) {
            mbar_wait_bounded(&bars[(seq + s) % C::D], (uint32_t)(((seq + s) / C::D) & 1), 100000000ull);
            moe_step(sg, tb, te, warp, q);
        }
    }
    __syncwarp();
    // The last CTA to leave resets the tile counts, and after a failed wait also the combine
    // tickets (a unit that gave up took none, so some tokens' tickets stopped short of zero).
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        unsigned int* ex = reinterpret_cast<unsigned int*>(a.ws + kMoeExitOff);
        if (atomicAdd(ex, 1u) == gridDim.x - 1) {
            __threadfence();
            unsigned int* dn = reinterpret_cast<unsigned int*>(a.ws + kMoeDoneOff);
            for (int j = 0; j < kMoeMaxAct; ++j) dn[j] = 0u;
            if (__ldcg(reinterpret_cast<const unsigned int*>(a.ws)) & 1u) {
                unsigned int* comb = reinterpret_cast<unsigned int*>(a.ws + moe_comb_off());
                for (int j = 0; j < a.M * a.T1; ++j) comb[j] = 0u;
            }
            *ex = 0u;
        }
    }
}

}  // namespace qlin

// ------------------------------------------------------------------ host side
namespace qlin {

static int moe_sm_count() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
    return n;
}

static int64_t al256(int64_t b) { return (b + 255) / 256 * 256; }

struct MoePlan {
    int grid;
    int64_t o_off, h_off;
    size_t bytes;
};

static MoePlan plan_moe(int fmt, int M, int64_t H, int64_t I, int top_k, bool need_h) {
    MoePlan p;
    const int cps = ring_ctas_per_sm(fmt);
    p.grid = moe_sm_count() * cps;
    int64_t off = al256(moe_head_bytes());
    p.o_off = off;
    off += al256(4 * (int64_t)M * top_k * H);
    p.h_off = off;
    if (need_h) off += al256(4 * (int64_t)M * top_k * I);
    p.bytes = (size_t)off;
    return p;
}

template <int FMT, int MAXM, bool XBF16>
static cudaError_t moe_launch(const MoeArgs& a, int grid, cudaStream_t s, bool pdl) {
    using C = RingCfg<FMT>;
    constexpr int kSmem = MoeSmem<FMT, MAXM>::kBytes;
    auto kern = moe_kernel<FMT, MAXM, XBF16>;
    static bool attr_set = false;  // per instantiation; idempotent
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
        if (e != cudaSuccess) return e;
        // The waits between the steps need every CTA of the grid resident at once.
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
    return cudaLaunchKernelEx(&cfg, kern, a);
}

// Work entries hold at most kMoeEntryRows rows whatever M is.
template <int FMT, bool XBF16>
static cudaError_t moe_launch_m(const MoeArgs& a, int grid, cudaStream_t s, bool pdl) {
    if (a.M == 1) return moe_launch<FMT, 1, XBF16>(a, grid, s, pdl);
    return moe_launch<FMT, kMoeEntryRows, XBF16>(a, grid, s, pdl);
}

}  // namespace qlin

using namespace qlin;

extern "C" size_t qlin_moe_ws_bytes(int fmt, int M, int64_t H, int64_t I, int E, int top_k) {
    (void)E;
    return plan_moe(fmt, M, H, I, top_k, true).bytes;
}

extern "C" cudaError_t qlin_launch_moe(int fmt, const void* gu, const void* dn, int E, int64_t H, int64_t I,
                                       int top_k, const float* logits, int32_t* ids, float* wts, const void* x,
                                       int xdt, int M, float* y, float* h, int flags, void* ws, cudaStream_t s) {
    const MoePlan p = plan_moe(fmt, M, H, I, top_k, h == nullptr);
    uint8_t* w = (uint8_t*)ws;
    const Geometry g0 = geometry(fmt, 2 * I, H, QLIN_PACK_GATE_UP);
    const Geometry g1 = geometry(fmt, H, I, 0);
    MoeArgs a = {};
    a.gu = (const uint8_t*)gu;
    a.dn = (const uint8_t*)dn;
    a.gu_stride = (int64_t)qlin_packed_bytes((qlin_format_t)fmt, 2 * I, H, QLIN_PACK_GATE_UP);
    a.dn_stride = (int64_t)qlin_packed_bytes((qlin_format_t)fmt, H, I, 0);
    a.E = E;
    a.H = (int)H;
    a.I = (int)I;
    a.top_k = top_k;
    a.M = M;
    a.logits = logits;
    a.ids = ids;
    a.wts = wts;
    a.x = x;
    a.y = y;
    a.h = h ? h : (float*)(w + p.h_off);
    a.o = (float*)(w + p.o_off);
    a.ws = w;
    a.T0 = (int)g0.T;
    a.G0 = (int)g0.G;
    a.U0 = (int)g0.U;
    a.T1 = (int)g1.T;
    a.G1 = (int)g1.G;
    a.U1 = (int)g1.U;
    const bool pdl = (flags & QLIN_FLAG_PDL) != 0, bf16 = xdt == QLIN_BF16;
    if (fmt == QLIN_Q4_0) return bf16 ? moe_launch_m<QLIN_Q4_0, true>(a, p.grid, s, pdl) : moe_launch_m<QLIN_Q4_0, false>(a, p.grid, s, pdl);
    if (fmt == QLIN_Q8_0) return bf16 ? moe_launch_m<QLIN_Q8_0, true>(a, p.grid, s, pdl) : moe_launch_m<QLIN_Q8_0, false>(a, p.grid, s, pdl);
    if (fmt == QLIN_MXFP4) return bf16 ? moe_launch_m<QLIN_MXFP4, true>(a, p.grid, s, pdl) : moe_launch_m<QLIN_MXFP4, false>(a, p.grid, s, pdl);
    if (fmt == QLIN_Q4_K) return bf16 ? moe_launch_m<QLIN_Q4_K, true>(a, p.grid, s, pdl) : moe_launch_m<QLIN_Q4_K, false>(a, p.grid, s, pdl);
    if (fmt == QLIN_Q6_K) return bf16 ? moe_launch_m<QLIN_Q6_K, true>(a, p.grid, s, pdl) : moe_launch_m<QLIN_Q6_K, false>(a, p.grid, s, pdl);
    return bf16 ? moe_launch_m<QLIN_NVFP4, true>(a, p.grid, s, pdl) : moe_launch_m<QLIN_NVFP4, false>(a, p.grid, s, pdl);
}
