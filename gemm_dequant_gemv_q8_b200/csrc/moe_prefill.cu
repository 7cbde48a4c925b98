// moe_prefill.cu -- top-k routed MoE expert projections for a prefill chunk of M tokens on the
// tcgen05 tensor cores (sm_100a): the grouped-GEMM counterpart of moe.cu's decode kernel.
//
// What it computes is what qlin_moe_experts computes (route; h = silu(W_gate[e] x) * (W_up[e] x);
// o = W_down[e] h; y[m] = sum over slots, in slot order, of weight * o), with NVFP4 / MXFP4 expert
// weights and the chunk path's activation quantization.  The pages' counterpart: imp's MoE "top-k
// grouped GEMM" and its NVFP4 grouped GEMM for MoE prefill (imp README, "Features" table, row
// "Architectures"; release notes v0.7.0), there on sm_120a.  Six launches on one stream, no host
// synchronisation (the counts and the tile table live on the device, so the sequence can be
// captured in a CUDA graph); every launch after the first is a programmatic dependent of the one
// before it and reads that one's results only after griddepcontrol.wait:
//   1. route (a warp per token): top_k (ties to the lower expert index, a NaN logit ranks as
//      -inf), renormalised weights, max |x| folded into one word, and for each valid slot its
//      index among the expert's entries (a shared-memory count per CTA, then one atomic per expert
//      and CTA on the global count); the last CTA to finish turns the counts into each expert's
//      first sorted row (rows padded to whole 128-row tiles), the table row tile -> expert and
//      each tile's count of rows holding entries;
//   2. gather-quantize (a CTA per token): the token's row quantized once as the chunk path
//      quantizes (NVFP4: one per-tensor scale from max |x| over the chunk; MXFP4: the OCP MX rule)
//      and stored, in the tensor-core operand layout, at each of its sorted rows; extra CTAs zero
//      each expert's padding rows;
//   3. grouped chunk GEMM, gate_up: each 128-row tile against its expert's gate/up-interleaved
//      weights, the SiLU-gate fused in the epilogue, h stored as bf16 (padding rows not stored) and
//      max |h| folded into a word;
//   4. h quantized the same way (NVFP4: its own per-tensor scale, from that word), a thread per
//      64 values of a row;
//   5. grouped chunk GEMM, down: each tile against its expert's down weights, o (fp32) per sorted row
//      (padding rows not stored);
//   6. combine: y[m] = sum over slots, in slot order, of weight * o[row of (m, slot)] (deterministic),
//      and the optional h output.  The GEMMs report their errors in the caller's status word.
// Which sorted row an entry takes depends on the order of the atomic counter, but every row is
// computed on its own (the MMA rows are independent and the per-tensor scales are maxima), so the
// results do not: y, h, ids and weights are the same from run to run.
#include "chunk_common.cuh"

extern "C" cudaError_t qlin_launch_chunk_grouped(int fmt, const void* w, int64_t w_stride, int T2, int64_t N,
                                                 int64_t K, int rows_max, float* y, int64_t ldy, void* h,
                                                 int64_t ldh, int64_t h_cols, const int* tile_expert,
                                                 const int* tile_rows, const int* used_tm, const unsigned* amax_in,
                                                 unsigned* amax_out, unsigned* status, void* ws, cudaStream_t s);
extern "C" size_t qlin_chunk_ws_bytes(int M, int64_t N, int64_t K);
extern "C" int64_t qlin_mma_tiles(int64_t N, int gate_up);

namespace qlin {

constexpr int kPfMaxTopK = 8;
constexpr int kPfMaxE = 256;
constexpr int kPfRouteWarps = 16;  // tokens per route CTA
constexpr int kPfGatherThreads = 128;
constexpr int kPfPadCtas = 4;  // CTAs zeroing one expert's padding rows

static inline int64_t pf_al256(int64_t v) { return (v + 255) / 256 * 256; }

// Sorted rows at most: every (token, slot) entry plus up to 127 padding rows per expert.
static inline int pf_rows_max(int M, int E, int top_k) {
    const int64_t r = (int64_t)M * top_k + (int64_t)E * 127;
    return (int)((r + 127) / 128 * 128);
}

// Workspace layout (offsets in bytes).  [0, 256): the status word (and the wait budget word).
// rt, at a fixed offset (its counters start each call at zero, whatever the shapes of the call
// before): cnt[256] at 0, fill[256] at 1024, off[257] at 2048, words at 3328: [0] ticket, [1] max |x|,
// [2] max |h|, [3] row tiles in use.
struct PfLayout {
    int64_t lpos, pos, rt, tile_expert, ws_a, hs, ws_b, os, total;
    int rows_max;
};

static PfLayout pf_layout(int M, int64_t H, int64_t I, int E, int top_k) {
    PfLayout L;
    L.rows_max = pf_rows_max(M, E, top_k);
    const int64_t R = L.rows_max, TMx = R / 128;
    int64_t o = 256;
    L.rt = o;
    o += 4096;
    L.lpos = o;
    o += pf_al256(4 * (int64_t)M * top_k);
    L.pos = o;
    o += pf_al256(4 * (int64_t)M * top_k);
    L.tile_expert = o;  // then tile_rows
    o += pf_al256(8 * TMx);
    L.ws_a = o;
    o += pf_al256((int64_t)qlin_chunk_ws_bytes((int)R, 2 * I, H));
    L.hs = o;
    o += pf_al256(2 * R * I);
    L.ws_b = o;
    o += pf_al256((int64_t)qlin_chunk_ws_bytes((int)R, H, I));
    L.os = o;
    o += pf_al256(4 * R * H);
    L.total = o;
    return L;
}

struct PfArgs {
    const float* logits;  // M x E, or nullptr (ids / weights given)
    int32_t* ids;         // M x top_k
    float* wts;           // M x top_k
    const __nv_bfloat16* x;  // M x H
    int64_t H;
    int M, E, top_k, TMx;
    int* lpos;            // M x top_k: index of (token, slot) among its expert's entries, -1 skipped
    int* pos;             // M x top_k: sorted row of (token, slot), -1 for a skipped slot
    int* cnt;             // E: entries per expert (counted in step 1, cleared by its last CTA)
    int* fill;            // E: the counts, kept for step 2 (an expert's padding rows start at off + fill)
    int* off;             // E + 1: first sorted row of each expert
    unsigned* words;      // [0] ticket, [1] max |x|, [2] max |h|, [3] row tiles in use
    int* tile_expert;     // TMx
    int* tile_rows;       // TMx: rows of the tile that hold entries (the rest is padding)
    unsigned* status;     // bit 1: an invalid or repeated given expert id (the slot is skipped)
};

// Larger logit first, ties to the lower index; a NaN logit ranks as -inf.
__device__ __forceinline__ bool pf_before(float a, int ia, float b, int ib) {
    const float fa = a != a ? -INFINITY : a, fb = b != b ? -INFINITY : b;
    return fa > fb || (fa == fb && ia < ib);
}

__global__ void __launch_bounds__(kPfRouteWarps * 32) moe_prefill_route_kernel(const PfArgs a) {
    __shared__ int s_cnt[kPfMaxE];  // this CTA's entries per expert, then their first index
    __shared__ int s_off[kPfMaxE + 1];
    __shared__ float s_max[kPfRouteWarps];
    __shared__ int s_last;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, k = a.top_k;
    const int m = blockIdx.x * kPfRouteWarps + warp;
    griddep_launch_dependents();  // (the gather reads nothing of this grid before its own wait)
    for (int e = threadIdx.x; e < a.E; e += blockDim.x) s_cnt[e] = 0;
    __syncthreads();
    int my_e = -1, my_li = 0;  // lane r < top_k: slot r's expert and its index among this CTA's
    float mx = 0.f;
    if (m < a.M) {
        // the token's logits (lane l holds experts l, l + 32, ...), in flight with the x loads below
        float v[kPfMaxE / 32];
        const float* l = a.logits ? a.logits + (int64_t)m * a.E : nullptr;
#pragma unroll
        for (int j = 0; j < kPfMaxE / 32; ++j) {
            const int e = lane + 32 * j;
            v[j] = (l && e < a.E) ? l[e] : -INFINITY;
        }
        // max |x| of the token (fmaxf skips a NaN, as the chunk quantizer's max pass does)
        const uint4* xr = reinterpret_cast<const uint4*>(a.x + (int64_t)m * a.H);
#pragma unroll 8
        for (int64_t v = lane; v < a.H / 8; v += 32) {
            const uint4 q = __ldg(xr + v);
            const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
            for (int j = 0; j < 4; ++j)
                mx = fmaxf(mx, fmaxf(fabsf(__uint_as_float(w[j] << 16)), fabsf(__uint_as_float(w[j] & 0xffff0000u))));
        }
        for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));

        int32_t* id = a.ids + (int64_t)m * k;
        int sel[kPfMaxTopK];
#pragma unroll
        for (int r = 0; r < kPfMaxTopK; ++r) sel[r] = -1;
        if (l) {
            // top_k rounds of a warp-wide argmax under pf_before
            unsigned taken = 0u;
            float selv[kPfMaxTopK];  // the selected logits (as given)
#pragma unroll
            for (int r = 0; r < kPfMaxTopK; ++r) {
                if (r >= k) break;
                float bv = -INFINITY;
                int bi = 0x7fffffff;
#pragma unroll
                for (int j = 0; j < kPfMaxE / 32; ++j) {
                    const int e = lane + 32 * j;
                    if (e < a.E && !((taken >> j) & 1u) && pf_before(v[j], e, bv, bi)) {
                        bv = v[j];
                        bi = e;
                    }
                }
                for (int o = 16; o; o >>= 1) {
                    const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
                    const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
                    if (pf_before(ov, oi, bv, bi)) {
                        bv = ov;
                        bi = oi;
                    }
                }
                sel[r] = bi;
                selv[r] = bv;
                if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
            }
            // weights: softmax over the selected logits (the largest first), fp32
            const float lmax = selv[0] != selv[0] ? 0.f : selv[0];
            float ex[kPfMaxTopK], sum = 0.f;
#pragma unroll
            for (int r = 0; r < kPfMaxTopK; ++r) {
                if (r >= k) break;
                ex[r] = expf(selv[r] - lmax);
                sum += ex[r];
            }
            if (lane == 0) {
#pragma unroll
                for (int r = 0; r < kPfMaxTopK; ++r) {
                    if (r >= k) break;
                    id[r] = sel[r];
                    a.wts[(int64_t)m * k + r] = ex[r] / sum;
                }
            }
        } else {
#pragma unroll
            for (int r = 0; r < kPfMaxTopK; ++r)
                if (r < k) sel[r] = id[r];
        }
        // each valid slot's index among its expert's entries (lane r takes slot r)
        if (lane < k) {
            int e = sel[0];
            bool ok = true;
#pragma unroll
            for (int r = 1; r < kPfMaxTopK; ++r)
                if (r == lane) e = sel[r];
#pragma unroll
            for (int r2 = 0; r2 < kPfMaxTopK; ++r2)
                if (r2 < lane && sel[r2] == e) ok = false;  // a repeated id counts once
            ok = ok && e >= 0 && e < a.E;
            if (ok) {
                my_e = e;
                my_li = atomicAdd(&s_cnt[e], 1);
            } else {
                a.lpos[(int64_t)m * k + lane] = -1;
                atomicOr(a.status, 2u);
            }
        }
    }
    // One global atomic per expert present in this CTA gives its entries' first index; one per CTA
    // folds max |x| in (non-negative floats order as their bits).
    if (lane == 0) s_max[warp] = mx;
    __syncthreads();
    for (int e = threadIdx.x; e < a.E; e += blockDim.x) {
        const int c = s_cnt[e];
        if (c) s_cnt[e] = atomicAdd(&a.cnt[e], c);
    }
    if (threadIdx.x == 0) {
        float b = 0.f;
        for (int w = 0; w < kPfRouteWarps; ++w) b = fmaxf(b, s_max[w]);
        atomicMax(&a.words[1], __float_as_uint(b));
    }
    __syncthreads();
    if (my_e >= 0) a.lpos[(int64_t)m * k + lane] = s_cnt[my_e] + my_li;
    // The last CTA to finish: first sorted row of each expert, the tile table, and the counters
    // cleared for the next call.
    if (threadIdx.x == 0) {
        __threadfence();
        s_last = atomicAdd(&a.words[0], 1u) == gridDim.x - 1;
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    for (int e = threadIdx.x; e < a.E; e += blockDim.x) {  // the counts, read once and cleared
        const int c = __ldcg(&a.cnt[e]);
        s_cnt[e] = c;
        a.fill[e] = c;
        a.cnt[e] = 0;
    }
    __syncthreads();
    if (warp == 0) {  // exclusive scan of the padded counts: lane l takes experts 8l .. 8l + 7
        int c[kPfMaxE / 32], sum = 0;
#pragma unroll
        for (int j = 0; j < kPfMaxE / 32; ++j) {
            const int e = lane * (kPfMaxE / 32) + j;
            c[j] = e < a.E ? (s_cnt[e] + 127) / 128 * 128 : 0;
            sum += c[j];
        }
        int incl = sum;
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
        }
        int run = incl - sum;
#pragma unroll
        for (int j = 0; j < kPfMaxE / 32; ++j) {
            const int e = lane * (kPfMaxE / 32) + j;
            if (e < a.E) s_off[e] = run;
            run += c[j];
        }
        if (lane == 31) {
            s_off[a.E] = incl;
            a.words[3] = (unsigned)(incl / 128);
        }
    }
    __syncthreads();
    for (int e = threadIdx.x; e <= a.E; e += blockDim.x) a.off[e] = s_off[e];
    for (int t = threadIdx.x; t < a.TMx; t += blockDim.x) {
        // the expert whose rows hold tile t: the last e with s_off[e] <= 128 t (an expert without
        // entries holds no rows), -1 past the rows in use
        int ex = -1;
        if (128 * t < s_off[a.E]) {
            int lo = 0, hi = a.E - 1;
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if (s_off[mid] <= 128 * t) lo = mid;
                else hi = mid - 1;
            }
            ex = lo;
        }
        a.tile_expert[t] = ex;
        const int live = ex < 0 ? 0 : s_off[ex] + s_cnt[ex] - 128 * t;
        a.tile_rows[t] = live < 0 ? 0 : (live > 128 ? 128 : live);
    }
    if (threadIdx.x == 0) {
        a.words[0] = 0u;  // the ticket
        a.words[2] = 0u;  // max |h|, accumulated by the gate_up GEMM that follows
    }
}

// Blocks [0, M): token m's row quantized once (item = 16 values; NVFP4 with a_g from max |x|, MXFP4
// by the pair rule) and stored at each of its sorted rows, in the operand units of the gate_up
// GEMM's workspace (G k-groups of 256 values per 128-row tile; values past H are zeros); the
// sorted row of each (m, slot) recorded.  Blocks [M, M + kPfPadCtas E): expert e's padding rows
// zeroed, per row and k-group its 8 16-byte code chunks and its 4 (MXFP4: 2) scale words.
template <bool MX>
__global__ void __launch_bounds__(kPfGatherThreads) moe_prefill_gather_quant_kernel(const PfArgs a, int64_t G,
                                                                                  uint8_t* __restrict__ aq) {
    const int b = blockIdx.x, k = a.top_k;
    const int64_t nitems = G * 16;
    if (b < a.M) {
        const int m = b;
        // the token's first item (the caller's x) in flight before the wait for the routing
        uint32_t w[8], c8[2];
        act_load_item(a.x, threadIdx.x < nitems ? a.M : 0, a.H, a.H, true, m, threadIdx.x < nitems ? threadIdx.x : 0, w);
        griddep_wait();
        griddep_launch_dependents();  // after the wait: the next grid's early reads see the routing
        int rows[kPfMaxTopK];
#pragma unroll
        for (int r = 0; r < kPfMaxTopK; ++r) {
            rows[r] = -1;
            if (r < k) {
                const int li = a.lpos[(int64_t)m * k + r];
                if (li >= 0) rows[r] = a.off[a.ids[(int64_t)m * k + r]] + li;
                if (threadIdx.x == 0) a.pos[(int64_t)m * k + r] = rows[r];
            }
        }
        const float ag = MX ? 1.0f : act_global_scale(__uint_as_float(__ldcg(&a.words[1])));
        // (nitems is even, so the two items of a 32-value block are both live or both not, and the
        // loop bounds are the same for every lane: the MXFP4 pair shuffles run with the whole warp)
        for (int64_t i0 = 0; i0 < nitems; i0 += kPfGatherThreads) {
            const int64_t it = i0 + threadIdx.x;
            const bool live = it < nitems;
            if (i0 > 0) act_load_item(a.x, live ? a.M : 0, a.H, a.H, true, m, live ? it : 0, w);
            uint8_t sc;
            if constexpr (MX) {
                sc = act_mx_pair_byte(act_item_amax(w), act_item_special(w));
                act_quant_item_mx_codes(w, sc, c8);
            } else {
                sc = act_quant_block(w, act_item_amax(w), ag, c8);
            }
            if (!live) continue;
#pragma unroll
            for (int r = 0; r < kPfMaxTopK; ++r) {
                if (r >= k || rows[r] < 0) continue;
                if constexpr (MX)
                    act_store_item_mx(0, a.H, G, rows[r], it, sc, c8, aq, nullptr, nullptr);
                else
                    act_store_item(0, a.H, G, rows[r], it, sc, c8, aq, nullptr, nullptr);
            }
        }
    } else {
        griddep_wait();
        griddep_launch_dependents();
        const int e = (b - a.M) / kPfPadCtas, part = (b - a.M) % kPfPadCtas;
        const int r0 = a.off[e] + a.fill[e], npad = a.off[e + 1] - r0;  // < 128 rows, one tile
        const int per_row = (int)G * 12;
        for (int i = part * kPfGatherThreads + threadIdx.x; i < npad * per_row; i += kPfPadCtas * kPfGatherThreads) {
            const int rr = i / per_row, rem = i - rr * per_row;
            const int g = rem / 12, piece = rem - g * 12;
            const int row = r0 + rr, r = row & (kMmaARows - 1);
            uint8_t* ub = aq + ((int64_t)(row / kMmaARows) * G + g) * kMmaAUnit;
            if (piece < 8)
                *reinterpret_cast<uint4*>(ub + mma_code_off(r, piece)) = make_uint4(0u, 0u, 0u, 0u);
            else if (!MX || piece < 10)
                *reinterpret_cast<uint32_t*>(ub + kMmaARows * 128 + mma_scale_off(piece - 8, r, 0, 1)) = 0u;
        }
    }
}

// h (the sorted rows in use, bf16) quantized for the down GEMM: one thread per 64 consecutive
// values of a row (four 16-value items; NVFP4 with a_g from max |h|, word [2], folded in by the
// gate_up epilogue; MXFP4 by the OCP MX rule, the two 32-value blocks within the thread), stored
// in the down GEMM's operand units (G k-groups per 128-row tile; values past I are zeros) as two
// 16-byte code chunks and one scale word.  Padding rows (not written by the gate_up epilogue) are
// not read: their operand rows are zeros.  The grid covers every row the workspace can hold;
// threads past the rows in use return at once.
template <bool MX>
__global__ void __launch_bounds__(256) moe_prefill_quant_h_kernel(const __nv_bfloat16* __restrict__ hs, int64_t I,
                                                                  int64_t G, const unsigned* __restrict__ words,
                                                                  const int* __restrict__ tile_rows,
                                                                  uint8_t* __restrict__ aq) {
    griddep_wait();  // h and max |h| come from the gate_up GEMM
    griddep_launch_dependents();
    const int64_t nq = G * 4;  // 64-value quads per (padded) row
    const int64_t qd = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int rows = (int)words[3] * kMmaARows;
    if (qd >= (int64_t)rows * nq) return;
    const int row = (int)(qd / nq);
    const int64_t qi = qd - (int64_t)row * nq;
    const int tm = row / kMmaARows, r = row % kMmaARows;
    const int lim = r < tile_rows[tm] ? rows : 0;  // a padding row reads as zeros
    uint32_t w[4][8], c8[4][2];
    uint8_t sc[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) act_load_item(hs, lim, I, I, true, row, 4 * qi + j, w[j]);
    if constexpr (MX) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const uint8_t byte = mx_scale_byte(fmaxf(act_item_amax(w[2 * h]), act_item_amax(w[2 * h + 1])),
                                               act_item_special(w[2 * h]) || act_item_special(w[2 * h + 1]));
            sc[2 * h] = sc[2 * h + 1] = byte;
            act_quant_item_mx_codes(w[2 * h], byte, c8[2 * h]);
            act_quant_item_mx_codes(w[2 * h + 1], byte, c8[2 * h + 1]);
        }
    } else {
        const float ag = act_global_scale(__uint_as_float(__ldcg(&words[2])));
#pragma unroll
        for (int j = 0; j < 4; ++j) sc[j] = act_quant_block(w[j], act_item_amax(w[j]), ag, c8[j]);
    }
    const int64_t k0 = 64 * qi;
    const int kin = (int)(k0 % kGroupK);
    uint8_t* ub = aq + ((int64_t)tm * G + k0 / kGroupK) * kMmaAUnit;
#pragma unroll
    for (int h = 0; h < 2; ++h)  // 16-byte chunk kin / 32 + h: items 2h and 2h + 1
        *reinterpret_cast<uint4*>(ub + mma_code_off(r, kin / 32 + h)) =
            make_uint4(c8[2 * h][0], c8[2 * h][1], c8[2 * h + 1][0], c8[2 * h + 1][1]);
    uint8_t* sb = ub + kMmaARows * 128;
    if constexpr (MX)  // the two block scales of this half span: bytes j, j + 1 of the row's word
        *reinterpret_cast<uint16_t*>(sb + mma_scale_off(kin / 128, r, (kin % 128) / 32, 1)) =
            (uint16_t)(sc[0] | (sc[2] << 8));
    else  // the four 16-value scales of this 64-value block: the row's word of atom kin / 64
        *reinterpret_cast<uint32_t*>(sb + mma_scale_off(kin / 64, r, 0, 1)) =
            (uint32_t)sc[0] | ((uint32_t)sc[1] << 8) | ((uint32_t)sc[2] << 16) | ((uint32_t)sc[3] << 24);
}

// One CTA per token: y[m] = sum over slots in slot order of w * o[row]; the optional h output
// (fp32 values of the bf16 h of each (token, slot)); max |x| cleared for the next call.
__global__ void __launch_bounds__(256) moe_prefill_combine_kernel(const PfArgs a, const float* __restrict__ os,
                                                                  const __nv_bfloat16* __restrict__ hs, int64_t I,
                                                                  float* __restrict__ y, float* __restrict__ h) {
    const int m = blockIdx.x, top_k = a.top_k;
    const int64_t H = a.H;
    griddep_wait();  // o comes from the down GEMM
    if (m == 0 && threadIdx.x == 0) a.words[1] = 0u;
    int rows[kPfMaxTopK];
    float w[kPfMaxTopK];
#pragma unroll
    for (int r = 0; r < kPfMaxTopK; ++r) {
        rows[r] = r < top_k ? a.pos[(int64_t)m * top_k + r] : -1;
        w[r] = r < top_k ? a.wts[(int64_t)m * top_k + r] : 0.f;
    }
    // four columns per thread (H % 32 == 0; the o rows are 16-byte aligned), one fused multiply-add
    // per slot and column
    const bool yvec = (reinterpret_cast<uintptr_t>(y) & 15) == 0;
    for (int64_t n4 = threadIdx.x; n4 < H / 4; n4 += blockDim.x) {
        float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int r = 0; r < kPfMaxTopK; ++r) {
            if (r < top_k && rows[r] >= 0) {
                const float4 o = *reinterpret_cast<const float4*>(os + (int64_t)rows[r] * H + 4 * n4);
                sum.x = __fmaf_rn(w[r], o.x, sum.x);
                sum.y = __fmaf_rn(w[r], o.y, sum.y);
                sum.z = __fmaf_rn(w[r], o.z, sum.z);
                sum.w = __fmaf_rn(w[r], o.w, sum.w);
            }
        }
        float* dst = y + (int64_t)m * H + 4 * n4;
        if (yvec) {
            *reinterpret_cast<float4*>(dst) = sum;
        } else {
            dst[0] = sum.x, dst[1] = sum.y, dst[2] = sum.z, dst[3] = sum.w;
        }
    }
    if (h) {
        for (int r = 0; r < top_k; ++r)
            for (int64_t i = threadIdx.x; i < I; i += blockDim.x)
                h[((int64_t)m * top_k + r) * I + i] =
                    rows[r] >= 0 ? __bfloat162float(hs[(int64_t)rows[r] * I + i]) : 0.f;
    }
}

}  // namespace qlin

using namespace qlin;

// A launch that may begin while the previous kernel of the stream finishes (programmatic dependent
// launch); the kernel waits (griddepcontrol.wait) before it reads that kernel's results.
template <typename... KArgs, typename... Args>
static cudaError_t pf_launch_pdl(void (*kernel)(KArgs...), unsigned grid, unsigned block, cudaStream_t s,
                                 Args... args) {
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(block);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

extern "C" size_t qlin_moe_prefill_ws_bytes(int M, int64_t H, int64_t I, int E, int top_k) {
    return (size_t)pf_layout(M, H, I, E, top_k).total;
}

// After host-side validation (api.cu).  gu / dn: E stacked packed buffers (QLIN_PACK_MMA |
// QLIN_PACK_GATE_UP over [gate ; up] rows 2I x H, and QLIN_PACK_MMA over H x I).
extern "C" cudaError_t qlin_launch_moe_prefill(int fmt, const void* gu, const void* dn, int E, int64_t H, int64_t I,
                                               int top_k, const float* logits, int32_t* ids, float* wts,
                                               const void* x, int M, float* y, float* h, void* ws, size_t gu_stride,
                                               size_t dn_stride, cudaStream_t s) {
    const PfLayout L = pf_layout(M, H, I, E, top_k);
    uint8_t* w8 = (uint8_t*)ws;
    uint8_t* rt = w8 + L.rt;
    PfArgs pa;
    pa.logits = logits;
    pa.ids = ids;
    pa.wts = wts;
    pa.x = (const __nv_bfloat16*)x;
    pa.H = H;
    pa.M = M;
    pa.E = E;
    pa.top_k = top_k;
    pa.TMx = L.rows_max / 128;
    pa.lpos = (int*)(w8 + L.lpos);
    pa.pos = (int*)(w8 + L.pos);
    pa.cnt = (int*)rt;
    pa.fill = (int*)(rt + 1024);
    pa.off = (int*)(rt + 2048);
    pa.words = (unsigned*)(rt + 3328);
    pa.tile_expert = (int*)(w8 + L.tile_expert);
    pa.tile_rows = pa.tile_expert + pa.TMx;
    pa.status = (unsigned*)ws;
    const int* used_tm = (const int*)(pa.words + 3);
    moe_prefill_route_kernel<<<(M + kPfRouteWarps - 1) / kPfRouteWarps, kPfRouteWarps * 32, 0, s>>>(pa);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const int64_t Gh = (H + kGroupK - 1) / kGroupK;
    uint8_t* aq = w8 + L.ws_a + 256;  // the gate_up GEMM's operand units (its workspace layout)
    e = fmt == QLIN_MXFP4
            ? pf_launch_pdl(moe_prefill_gather_quant_kernel<true>, M + kPfPadCtas * E, kPfGatherThreads, s, pa, Gh, aq)
            : pf_launch_pdl(moe_prefill_gather_quant_kernel<false>, M + kPfPadCtas * E, kPfGatherThreads, s, pa, Gh, aq);
    if (e != cudaSuccess) return e;
    __nv_bfloat16* hs = (__nv_bfloat16*)(w8 + L.hs);
    float* os = (float*)(w8 + L.os);
    e = qlin_launch_chunk_grouped(fmt, gu, (int64_t)gu_stride, (int)qlin_mma_tiles(2 * I, 1), 2 * I, H, L.rows_max,
                                  nullptr, 0, hs, I, I, pa.tile_expert, pa.tile_rows, used_tm, pa.words + 1,
                                  pa.words + 2, pa.status, w8 + L.ws_a, s);
    if (e != cudaSuccess) return e;
    const int64_t Gi = (I + kGroupK - 1) / kGroupK;
    const int64_t hquads = (int64_t)L.rows_max * Gi * 4;
    uint8_t* aq_b = w8 + L.ws_b + 256;  // the down GEMM's operand units
    const unsigned hgrid = (unsigned)((hquads + 255) / 256);
    e = fmt == QLIN_MXFP4 ? pf_launch_pdl(moe_prefill_quant_h_kernel<true>, hgrid, 256, s, hs, I, Gi,
                                          (const unsigned*)pa.words, (const int*)pa.tile_rows, aq_b)
                          : pf_launch_pdl(moe_prefill_quant_h_kernel<false>, hgrid, 256, s, hs, I, Gi,
                                          (const unsigned*)pa.words, (const int*)pa.tile_rows, aq_b);
    if (e != cudaSuccess) return e;
    e = qlin_launch_chunk_grouped(fmt, dn, (int64_t)dn_stride, (int)qlin_mma_tiles(H, 0), H, I, L.rows_max, os, H,
                                  nullptr, 0, 0, pa.tile_expert, pa.tile_rows, used_tm, pa.words + 2, nullptr,
                                  pa.status, w8 + L.ws_b, s);
    if (e != cudaSuccess) return e;
    return pf_launch_pdl(moe_prefill_combine_kernel, (unsigned)M, 256, s, pa, (const float*)os,
                         (const __nv_bfloat16*)hs, I, y, h);
}
