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
// tiny), which then plans the launch on the device exactly as the GEMV chain plans it on the
// host (chain.cu): the gate_up units of the selected experts (each expert once, for all tokens
// routed to it) form segment 0, their down units segment 1, and each segment is split into one
// contiguous range per warp.  A warp reaching an expert's down units waits (bounded) only for that
// expert's gate_up tiles.  The last of a token's experts to write a down tile adds the token's
// slot outputs for that tile in slot order (a ticket per token and tile): deterministic.  Split
// tiles use the chain's tagged partial words, stored per warp.
#include "gemv_core.cuh"

namespace qlin {

constexpr int kMoeMaxTopK = 8;
constexpr int kMoeMaxM = 8;
constexpr int kMoeMaxAct = kMoeMaxM * kMoeMaxTopK;

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
    int W;                // warps in the grid
};

// Workspace: [0,4) status word (bit 0 timeout, bit 1 bad expert id); [64,68) exit counter;
// [128,132) launch counter; [256, ...) per-active-expert gate_up tile counts; per-(token, down
// tile) combine tickets (self-resetting); partial words [segment][warp range][first piece, last
// piece][32][M].
constexpr int64_t kMoeExitOff = 64;
constexpr int64_t kMoeEpochOff = 128;
constexpr int64_t kMoeDoneOff = 256;
constexpr int kMoeMaxT1 = 1024;  // down tiles per expert (H <= 32768)
__host__ __device__ inline int64_t moe_comb_off() { return kMoeDoneOff + 4 * kMoeMaxAct; }
__host__ __device__ inline int64_t moe_part_off() { return moe_comb_off() + 4 * (int64_t)kMoeMaxM * kMoeMaxT1; }

// ------------------------------------------------------------------ device-side plan
// Segment s (0 = gate_up, 1 = down) of the selected experts: per expert Ue units (T tiles x G
// k-groups), U = n_act Ue in all, warp range v holding q + (v < r) of them, v = (gw - rot) mod W.
struct MoeSeg {
    int U, q, r, rot, Ue, G, T;
};

struct RouteSmem {
    MoeSeg sg[2];  // the device-side plan (identical in every CTA)
    int n_act;
    int expert[kMoeMaxAct];
    int nrows[kMoeMaxAct];
    int8_t row_m[kMoeMaxAct][kMoeMaxM];
    int8_t row_s[kMoeMaxAct][kMoeMaxM];
    int ids[kMoeMaxM][kMoeMaxTopK];
    float w[kMoeMaxM][kMoeMaxTopK];
    int kvalid[kMoeMaxM];  // valid slots of each token
};

// Routing of all tokens into shared memory (whole CTA participates).  With logits, CTA 0 also
// writes ids and weights out.  Invalid or repeated input ids skip their slot and set status bit 1.
constexpr int kMoeMaxE = 256;

__device__ void moe_route(const MoeArgs& a, RouteSmem& r) {
    const int tid = threadIdx.x;
    if (a.logits) {
        // One warp per token: each lane holds the logits of experts lane + 32 j; top_k rounds of a
        // warp-wide argmax (largest logit, ties to the lower expert index -- the order a
        // sequential scan with a strict comparison gives).
        const int warp = tid >> 5, lane = tid & 31, nw = blockDim.x >> 5;
        // all of this warp's logits first, so that their loads are in flight together
        constexpr int kTokPerWarp = (kMoeMaxM + kGemvWarps - 1) / kGemvWarps;
        float vall[kTokPerWarp][kMoeMaxE / 32];
#pragma unroll
        for (int i = 0; i < kTokPerWarp; ++i) {
            const int m = warp + i * nw;
#pragma unroll
            for (int j = 0; j < kMoeMaxE / 32; ++j) {
                const int e = lane + 32 * j;
                vall[i][j] = (m < a.M && e < a.E) ? __ldcg(a.logits + (int64_t)m * a.E + e) : -INFINITY;
            }
        }
#pragma unroll
        for (int i = 0; i < kTokPerWarp; ++i) {
            const int m = warp + i * nw;
            if (m >= a.M) break;
            float v[kMoeMaxE / 32];
#pragma unroll
            for (int j = 0; j < kMoeMaxE / 32; ++j) v[j] = vall[i][j];
            float lsel[kMoeMaxTopK];
            unsigned taken = 0;  // bit j: expert lane + 32 j already selected
            for (int s = 0; s < a.top_k; ++s) {
                float bv = -INFINITY;
                int be = 0x7fffffff;
#pragma unroll
                for (int j = 0; j < kMoeMaxE / 32; ++j) {
                    const int e = lane + 32 * j;
                    if (e < a.E && !((taken >> j) & 1u) && (be == 0x7fffffff || v[j] > bv || (v[j] == bv && e < be))) {
                        bv = v[j];
                        be = e;
                    }
                }
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) {
                    const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
                    const int oe = __shfl_xor_sync(0xffffffffu, be, o);
                    if (oe != 0x7fffffff && (be == 0x7fffffff || ov > bv || (ov == bv && oe < be))) {
                        bv = ov;
                        be = oe;
                    }
                }
#pragma unroll
                for (int j = 0; j < kMoeMaxE / 32; ++j)  // take it out of later rounds
                    if (lane + 32 * j == be) taken |= 1u << j;
                lsel[s] = bv;
                if (lane == 0) r.ids[m][s] = be;
            }
            if (lane == 0) {  // renormalised softmax over the selected experts
                float z = 0.f;
                for (int s = 0; s < a.top_k; ++s) {
                    r.w[m][s] = expf(lsel[s] - lsel[0]);
                    z += r.w[m][s];
                }
                for (int s = 0; s < a.top_k; ++s) r.w[m][s] = r.w[m][s] / z;
                if (blockIdx.x == 0)
                    for (int s = 0; s < a.top_k; ++s) {
                        a.ids[(int64_t)m * a.top_k + s] = r.ids[m][s];
                        a.wts[(int64_t)m * a.top_k + s] = r.w[m][s];
                    }
            }
        }
    } else if (tid < a.M) {
        {
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
    }
    __syncthreads();
    if (tid < a.M) {
        int kv = 0;
        for (int q = 0; q < a.top_k; ++q) kv += r.ids[tid][q] >= 0;
        r.kvalid[tid] = kv;
        if (kv == 0 && blockIdx.x == 0)  // no expert: the token's output is zero
            for (int n = 0; n < a.H; ++n) a.y[(int64_t)tid * a.H + n] = 0.f;
    }
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

__device__ __forceinline__ void moe_range(const MoeSeg& s, int gw, int W, int& b, int& e) {
    int v = gw - s.rot;
    if (v < 0) v += W;
    b = v * s.q + min(v, s.r);
    e = b + s.q + (v < s.r ? 1 : 0);
}

__device__ __forceinline__ int moe_owner(const MoeSeg& s, int u) {
    const int big = s.r * (s.q + 1);
    if (u < big) return u / (s.q + 1);
    return s.r + (u - big) / s.q;
}

// Position: segment s (2 = done), active expert a, unit uo of it (tile t, k-group g), segment
// unit u; the warp's range in s ends at e.  Advanced incrementally (no division per unit).
struct MoeCursor {
    int s, a, uo, t, g, u, e;
};

__device__ __forceinline__ void moe_seek(const MoeSeg (&sg)[2], int gw, int W, MoeCursor& c, int s) {
    for (; s < 2; ++s) {
        int b, e;
        moe_range(sg[s], gw, W, b, e);
        if (e > b) {
            c.s = s;
            c.a = b / sg[s].Ue;
            c.uo = b - c.a * sg[s].Ue;
            c.t = c.uo / sg[s].G;
            c.g = c.uo - c.t * sg[s].G;
            c.u = b;
            c.e = e;
            return;
        }
    }
    c.s = 2;
    c.a = c.uo = c.t = c.g = c.u = c.e = 0;
}

__device__ __forceinline__ void moe_step(const MoeSeg (&sg)[2], int gw, int W, MoeCursor& c) {
    if (++c.u >= c.e) {
        moe_seek(sg, gw, W, c, c.s + 1);
        return;
    }
    if (++c.uo == sg[c.s].Ue) {
        ++c.a;
        c.uo = c.t = c.g = 0;
    } else if (++c.g == sg[c.s].G) {
        c.g = 0;
        ++c.t;
    }
}

template <int FMT>
__device__ __forceinline__ const uint8_t* moe_unit_src(const MoeArgs& a, const RouteSmem& r, const MoeCursor& c) {
    const uint8_t* base = c.s == 0 ? a.gu + (int64_t)r.expert[c.a] * a.gu_stride
                                   : a.dn + (int64_t)r.expert[c.a] * a.dn_stride;
    return base + kHdrBytes + (int64_t)c.uo * RingCfg<FMT>::UB;
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
        __threadfence();  // count the tile for the down units of this expert
        __syncwarp();
        if (lane == 0) {
            unsigned int* done = reinterpret_cast<unsigned int*>(a.ws + kMoeDoneOff);
            asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(done + act) : "memory");
        }
        return;
    }
    // Down tile: store the slot outputs, then take a ticket per token; the last of a token's
    // experts for this tile adds the token's slot outputs in slot order into y.
    const int n = t * kTileRows + row;
    if (n < a.H) {
#pragma unroll
        for (int q = 0; q < MAXM; ++q)
            if (q < nr) __stcg(a.o + ((int64_t)r.row_m[act][q] * a.top_k + r.row_s[act][q]) * a.H + n, v[q]);
    }
    __threadfence();
    __syncwarp();
    unsigned int* comb = reinterpret_cast<unsigned int*>(a.ws + moe_comb_off());
    for (int q = 0; q < nr; ++q) {
        const int m = r.row_m[act][q];
        unsigned int ticket = 0;
        if (lane == 0) ticket = atomicAdd(comb + m * a.T1 + t, 1u);
        ticket = __shfl_sync(0xffffffffu, ticket, 0);
        if (ticket == (unsigned)r.kvalid[m] - 1u) {
            __threadfence();
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

// Partial words of range index v, piece kind k (0: the first piece of its range, 1: the last).
__device__ __forceinline__ uint64_t* moe_part(const MoeArgs& a, int s, int v, int k, int lane) {
    return reinterpret_cast<uint64_t*>(a.ws + moe_part_off()) + ((((int64_t)s * a.W + v) * 2 + k) * 32 + lane) * a.M;
}

template <int MAXM>
__device__ __forceinline__ void moe_publish(const MoeArgs& a, int s, int v, int k, int lane, const float (&acc)[MAXM],
                                            uint32_t tag) {
    uint64_t* w = moe_part(a, s, v, k, lane);
#pragma unroll
    for (int m = 0; m < MAXM; ++m)
        if (m < a.M)
            asm volatile("st.relaxed.gpu.global.b64 [%0], %1;" ::"l"(w + m),
                         "l"(((uint64_t)tag << 32) | __float_as_uint(acc[m]))
                         : "memory");
}

__device__ __forceinline__ uint64_t moe_ld_relaxed(const uint64_t* p) {
    uint64_t v;
    asm volatile("ld.relaxed.gpu.global.b64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

// Finish split tile t of expert `act` in segment s, whose first piece is range v's last piece and
// whose other n_t - 1 pieces are the first pieces of ranges v+1 ..: add them in range order
// (re-reading, bounded, words not yet tagged with this launch) and write the tile.
template <int MAXM>
__device__ __noinline__ bool moe_flush(const MoeArgs& a, const RouteSmem& r, int s, int act, int t, int v, int n_t,
                                       int lane, float gs, uint32_t tag) {
    float sum[MAXM];
#pragma unroll
    for (int m = 0; m < MAXM; ++m) sum[m] = 0.f;
    // pieces fetched together (their loads in flight at once), then added in order; one at a time
    // with 8 rows, where the wider batch costs more in registers than it saves
    constexpr int kB = MAXM > 2 ? 1 : 4;
    for (int i0 = 0; i0 < n_t; i0 += kB) {
        uint64_t x[kB][MAXM];
#pragma unroll
        for (int b = 0; b < kB; ++b) {
            const int i = i0 + b;
            const uint64_t* w = i < n_t ? moe_part(a, s, v + i, i == 0 ? 1 : 0, lane) : nullptr;
#pragma unroll
            for (int m = 0; m < MAXM; ++m)
                x[b][m] = (w != nullptr && m < a.M) ? moe_ld_relaxed(w + m) : ((uint64_t)tag << 32);
        }
        bool ready = true;
#pragma unroll
        for (int b = 0; b < kB; ++b)
#pragma unroll
            for (int m = 0; m < MAXM; ++m) ready &= (uint32_t)(x[b][m] >> 32) == tag;
        if (!__all_sync(0xffffffffu, ready)) {
            const uint64_t t0 = globaltimer_ns();
            for (uint32_t it = 1;; ++it) {
                __nanosleep(100);
                ready = true;
#pragma unroll
                for (int b = 0; b < kB; ++b) {
                    const int i = i0 + b;
#pragma unroll
                    for (int m = 0; m < MAXM; ++m)
                        if (i < n_t && m < a.M && (uint32_t)(x[b][m] >> 32) != tag) {
                            x[b][m] = moe_ld_relaxed(moe_part(a, s, v + i, i == 0 ? 1 : 0, lane) + m);
                            ready &= (uint32_t)(x[b][m] >> 32) == tag;
                        }
                }
                if (__all_sync(0xffffffffu, ready)) break;
                if ((it & 63u) == 0 && globaltimer_ns() - t0 > 2000000000ull) return false;
            }
        }
#pragma unroll
        for (int b = 0; b < kB; ++b)
            if (i0 + b < n_t)
#pragma unroll
                for (int m = 0; m < MAXM; ++m) sum[m] += __uint_as_float((uint32_t)x[b][m]);
    }
    moe_write_tile<MAXM>(a, r, s, act, t, lane, sum, gs);
    return true;
}

// Bounded wait until *p >= target (2 s); false on timeout.
__device__ __forceinline__ bool moe_wait_count(const unsigned int* p, uint32_t target) {
    auto ld = [&]() {
        uint32_t v;
        asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
        return v;
    };
    if (__all_sync(0xffffffffu, ld() >= target)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t it = 1;; ++it) {
        __nanosleep(64);
        if (__all_sync(0xffffffffu, ld() >= target)) return true;
        if ((it & 63u) == 0 && globaltimer_ns() - t0 > 2000000000ull) return false;
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

// One unit of segment s for the rows of active expert `act`.  One-pass (MAXM <= 2, or an expert
// with at most 2 rows) accumulates into acc8 across a tile's units; otherwise each pass is
// reduced at once into acc.  xs: the first pass's rows already staged in shared memory (or
// NULL); after_first_load() runs once the first pass's activations are in registers.
template <int FMT, int MAXM, bool XB, typename F>
__device__ __forceinline__ void moe_unit(const MoeArgs& a, const RouteSmem& r, int s, int act, int g,
                                         const uint8_t* ubuf, int lane, float (&acc8)[8][MAXM >= 2 ? 2 : 1],
                                         float (&acc)[MAXM], const uint8_t* xs, F&& after_first_load) {
    constexpr int MP = MAXM >= 2 ? 2 : 1;
    const int nr = r.nrows[act];
    const bool kOnePass = MAXM <= 2 || nr <= 2;  // an expert with at most 2 rows: accumulate in acc8
    const int64_t Kin = s == 0 ? a.H : a.I;
    const int part = lane & 7;
    const int64_t k0 = (int64_t)g * kGroupK + part * 32;
#pragma unroll 1
    for (int q0 = 0; q0 < (kOnePass ? 1 : nr); q0 += MP) {
        const void* rows[MP];
        moe_rows<MP, XB>(a, r, s, act, q0, rows);
        if constexpr (XB && FMT == QLIN_NVFP4) {
            uint32_t xh[MP][16];
            float xsc[MP][2];
            if (q0 == 0 && xs != nullptr)
                load_x_fp4h_staged<MP>(xs, part, xh, xsc);
            else
                load_x_fp4h<MP, true>(rows, k0, Kin, xh, xsc);
            if (q0 == 0) after_first_load();
            if (kOnePass) {
                unit_dot_fp4h<MP, true>(ubuf, lane, xh, xsc, acc8);
            } else {
                float res[8][MP];
                unit_dot_fp4h<MP>(ubuf, lane, xh, xsc, res);
                float rr[MP];
                reduce_scatter8<MP>(res, lane, rr);
#pragma unroll
                for (int qq = 0; qq < MAXM; ++qq)
#pragma unroll
                    for (int mm = 0; mm < MP; ++mm)
                        if (qq == q0 + mm) acc[qq] += rr[mm];
            }
        } else {
            float2 xv[MP][16];
            float xb[MP];
            if (q0 == 0 && xs != nullptr)
                load_x_staged<XB, MP>(xs, part, xv);
            else
                load_x_rows<XB, MP, true>(rows, k0, Kin, xv);
            if (q0 == 0) after_first_load();
            prep_x<FMT, MP>(xv, xb);
            if (kOnePass) {
                unit_dot<FMT, MP, true>(ubuf, lane, xv, xb, acc8);
            } else {
                float res[8][MP];
                unit_dot<FMT, MP>(ubuf, lane, xv, xb, res);
                float rr[MP];
                reduce_scatter8<MP>(res, lane, rr);
#pragma unroll
                for (int qq = 0; qq < MAXM; ++qq)
#pragma unroll
                    for (int mm = 0; mm < MP; ++mm)
                        if (qq == q0 + mm) acc[qq] += rr[mm];
            }
        }
    }
}

// Shared memory of the MoE kernel: the per-warp weight rings and their barriers, then (for at most
// 2 rows, except Q8_0 whose ring leaves no room) one activation stage per warp: the next unit's
// rows, copied while the current unit computes.  (With 8 rows the staging measured slower.)
template <int FMT, int MAXM>
struct MoeSmem {
    static constexpr int MP = MAXM >= 2 ? 2 : 1;
    static constexpr bool kStaged = FMT != QLIN_Q8_0 && MAXM <= 2;
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
__global__ void __launch_bounds__(kGemvWarps * 32, RingCfg<FMT>::kCtasPerSm) moe_kernel(const MoeArgs a) {
    using C = RingCfg<FMT>;
    using MS = MoeSmem<FMT, MAXM>;
    constexpr int MP = MAXM >= 2 ? 2 : 1;
    constexpr bool kOnePass = MAXM <= 2;
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ RouteSmem r;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int gw = blockIdx.x * kGemvWarps + warp;
    uint8_t* ring = smem + warp * C::D * C::UB;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kGemvWarps * C::D * C::UB) + warp * C::D;
    uint8_t* xst = smem + MS::kXOff + warp * MS::kStageBytes;  // used only if MS::kStaged

    griddep_launch_dependents();
    griddep_wait();  // logits / ids / x come from earlier kernels
    moe_route(a, r);
    const uint32_t tag = __ldcg(reinterpret_cast<const unsigned int*>(a.ws + kMoeEpochOff)) + 1u;
    if (threadIdx.x == 0) {
        MoeSeg* sp = r.sg;
        sp[0].Ue = a.U0; sp[0].G = a.G0; sp[0].T = a.T0;
        sp[1].Ue = a.U1; sp[1].G = a.G1; sp[1].T = a.T1;
        for (int s = 0; s < 2; ++s) {
            sp[s].U = r.n_act * sp[s].Ue;
            sp[s].q = sp[s].U / a.W;
            sp[s].r = sp[s].U % a.W;
        }
        sp[0].rot = 0;
        sp[1].rot = sp[0].r;  // the second step's extra units go to the warps after the first's
    }
    __syncthreads();
    const MoeSeg (&sg)[2] = r.sg;

    MoeCursor c;
    moe_seek(sg, gw, a.W, c, 0);
    MoeCursor p = c;
    if (lane == 0) {
#pragma unroll
        for (int s = 0; s < C::D; ++s) mbar_init(&bars[s], 1);
        fence_mbar_init();
        for (int s = 0; s < C::D && p.s < 2; ++s) {
            mbar_arrive_expect_tx(&bars[s], C::UB);
            bulk_g2s(ring + s * C::UB, moe_unit_src<FMT>(a, r, p), C::UB, &bars[s]);
            moe_step(sg, gw, a.W, p);
        }
    }
    __syncwarp();
    p.s = __shfl_sync(0xffffffffu, p.s, 0);
    p.a = __shfl_sync(0xffffffffu, p.a, 0);
    p.uo = __shfl_sync(0xffffffffu, p.uo, 0);
    p.t = __shfl_sync(0xffffffffu, p.t, 0);
    p.g = __shfl_sync(0xffffffffu, p.g, 0);
    p.u = __shfl_sync(0xffffffffu, p.u, 0);
    p.e = __shfl_sync(0xffffffffu, p.e, 0);

    float acc[MAXM];
#pragma unroll
    for (int m = 0; m < MAXM; ++m) acc[m] = 0.f;
    float acc8[8][MP];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int mm = 0; mm < MP; ++mm) acc8[i][mm] = 0.f;
    bool failed = false;
    int pend_s = -1, pend_a = 0, pend_t = 0, pend_v = 0, pend_n = 0;  // split tile finished later
    float pend_gs = 1.f;
    int seq = 0, cur_s = -1, cur_a = -1, b = 0, e = 0;
    bool xready = false;  // the current unit's first-pass rows are already staged
    auto stage_unit = [&](const MoeCursor& u) {
        const void* rows[MP];
        if (u.s == 0) {
            moe_rows<MP, XBF16>(a, r, 0, u.a, 0, rows);
            stage_x_rows<XBF16, MP>(rows, a.H, u.g, xst, lane, a.ws);
        } else {
            moe_rows<MP, false>(a, r, 1, u.a, 0, rows);
            stage_x_rows<false, MP>(rows, a.I, u.g, xst, lane, a.ws);
        }
    };
    float gs = 1.f;
    while (c.s < 2) {
        if (c.s != cur_s) {  // new segment: finish the pending tile of the previous one
            cur_s = c.s;
            cur_a = -1;
            moe_range(sg[c.s], gw, a.W, b, e);
            if (pend_s >= 0) {
                if (!moe_flush<MAXM>(a, r, pend_s, pend_a, pend_t, pend_v, pend_n, lane, pend_gs, tag)) {
                    failed = true;
                    break;
                }
                pend_s = -1;
            }
        }
        if (c.a != cur_a) {
            cur_a = c.a;
            gs = moe_scale<FMT>(a, r, c.s, c.a);
            // down units read h: wait for this expert's gate_up tiles
            if (c.s == 1 && !moe_wait_count(reinterpret_cast<const unsigned int*>(a.ws + kMoeDoneOff) + c.a,
                                            (uint32_t)a.T0)) {
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
        const uint8_t* xs = nullptr;
        MoeCursor cn = c;  // the next unit of this warp
        bool stage_next = false;
        if constexpr (MS::kStaged) {
            if (!xready) stage_unit(c);
            cp_async_wait_all();
            __syncwarp();
            xs = xst;
            moe_step(sg, gw, a.W, cn);
            // h rows of a down unit may be read only after that expert's wait
            stage_next = cn.s < 2 && (cn.s == 0 || (c.s == 1 && cn.a == c.a));
        }
        auto after_first_load = [&]() {  // the stage is free: copy the next unit's rows into it
            if constexpr (MS::kStaged) {
                __syncwarp();
                if (stage_next) stage_unit(cn);
            }
        };
        if (c.s == 0)
            moe_unit<FMT, MAXM, XBF16>(a, r, 0, c.a, c.g, ubuf, lane, acc8, acc, xs, after_first_load);
        else
            moe_unit<FMT, MAXM, false>(a, r, 1, c.a, c.g, ubuf, lane, acc8, acc, xs, after_first_load);
        xready = stage_next;
        __syncwarp();
        if (lane == 0 && p.s < 2) {
            fence_proxy_async_smem();
            mbar_arrive_expect_tx(&bars[slot], C::UB);
            bulk_g2s(ring + slot * C::UB, moe_unit_src<FMT>(a, r, p), C::UB, &bars[slot]);
        }
        if (p.s < 2) moe_step(sg, gw, a.W, p);
        ++seq;
        const int s_now = c.s, a_now = c.a, t = c.t;
        moe_step(sg, gw, a.W, c);
        if (c.s != s_now || c.a != a_now || c.t != t) {  // tile t of expert a_now ends here
            if (kOnePass || r.nrows[a_now] <= 2) {  // the tile was accumulated in acc8
                float rr[MP];
                reduce_scatter8<MP>(acc8, lane, rr);
#pragma unroll
                for (int mm = 0; mm < MP; ++mm) acc[mm] = rr[mm];
#pragma unroll
                for (int i = 0; i < 8; ++i)
#pragma unroll
                    for (int mm = 0; mm < MP; ++mm) acc8[i][mm] = 0.f;
            }
            const MoeSeg& S = sg[s_now];
            const int f = a_now * S.Ue + t * S.G;  // the tile in segment units
            if (f >= b && f + S.G <= e) {
                moe_write_tile<MAXM>(a, r, s_now, a_now, t, lane, acc, gs);
            } else {
                const int v_first = moe_owner(S, f);
                const int v = moe_owner(S, b > f ? b : f);
                if (v > v_first) {
                    moe_publish<MAXM>(a, s_now, v, 0, lane, acc, tag);  // first piece of range v
                } else {  // range v ends in the tile and owns its first unit: finish it later
                    moe_publish<MAXM>(a, s_now, v, 1, lane, acc, tag);
                    pend_s = s_now;
                    pend_a = a_now;
                    pend_t = t;
                    pend_v = v;
                    pend_n = moe_owner(S, f + S.G - 1) - v_first + 1;
                    pend_gs = gs;
                }
            }
#pragma unroll
            for (int m = 0; m < MAXM; ++m) acc[m] = 0.f;
        }
    }
    if (!failed && pend_s >= 0 &&
        !moe_flush<MAXM>(a, r, pend_s, pend_a, pend_t, pend_v, pend_n, lane, pend_gs, tag))
        failed = true;
    if constexpr (MS::kStaged) cp_async_wait_all();  // no copy into this CTA's memory outlives it
    if (failed && lane == 0) {
        atomicOr(reinterpret_cast<unsigned int*>(a.ws), 1u);
        MoeCursor q = c;  // wait (bounded) for this warp's copies still in flight
        for (int s = 0; s < C::D && q.s < 2; ++s) {
            mbar_wait_bounded(&bars[(seq + s) % C::D], (uint32_t)(((seq + s) / C::D) & 1), 100000000ull);
            moe_step(sg, gw, a.W, q);
        }
    }
    __syncwarp();
    // The last CTA to leave resets the tile counts and advances the launch counter.
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        unsigned int* ex = reinterpret_cast<unsigned int*>(a.ws + kMoeExitOff);
        if (atomicAdd(ex, 1u) == gridDim.x - 1) {
            __threadfence();
            unsigned int* done = reinterpret_cast<unsigned int*>(a.ws + kMoeDoneOff);
            for (int j = 0; j < kMoeMaxAct; ++j) done[j] = 0u;
            *reinterpret_cast<unsigned int*>(a.ws + kMoeEpochOff) = tag;
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
    int grid, W;
    int64_t o_off, h_off;
    size_t bytes;
};

static MoePlan plan_moe(int fmt, int M, int64_t H, int64_t I, int top_k, bool need_h) {
    MoePlan p;
    const int cps = fmt == QLIN_Q8_0 ? RingCfg<QLIN_Q8_0>::kCtasPerSm : RingCfg<QLIN_Q4_0>::kCtasPerSm;
    p.grid = moe_sm_count() * cps;
    p.W = p.grid * kGemvWarps;
    int64_t off = moe_part_off() + al256((int64_t)2 * p.W * 2 * 32 * M * 8);
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

template <int FMT, bool XBF16>
static cudaError_t moe_launch_m(const MoeArgs& a, int grid, cudaStream_t s, bool pdl) {
    if (a.M == 1) return moe_launch<FMT, 1, XBF16>(a, grid, s, pdl);
    if (a.M == 2) return moe_launch<FMT, 2, XBF16>(a, grid, s, pdl);
    return moe_launch<FMT, 8, XBF16>(a, grid, s, pdl);
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
    a.W = p.W;
    const bool pdl = (flags & QLIN_FLAG_PDL) != 0, bf16 = xdt == QLIN_BF16;
    if (fmt == QLIN_Q4_0) return bf16 ? moe_launch_m<QLIN_Q4_0, true>(a, p.grid, s, pdl) : moe_launch_m<QLIN_Q4_0, false>(a, p.grid, s, pdl);
    if (fmt == QLIN_Q8_0) return bf16 ? moe_launch_m<QLIN_Q8_0, true>(a, p.grid, s, pdl) : moe_launch_m<QLIN_Q8_0, false>(a, p.grid, s, pdl);
    return bf16 ? moe_launch_m<QLIN_NVFP4, true>(a, p.grid, s, pdl) : moe_launch_m<QLIN_NVFP4, false>(a, p.grid, s, pdl);
}
