// moe_prefill.cu -- top-k routed MoE expert projections for a prefill chunk of M tokens on the
// tcgen05 tensor cores (sm_100a): the grouped-GEMM counterpart of moe.cu's decode kernel.
//
// What it computes is what qlin_moe_experts computes (route; h = silu(W_gate[e] x) * (W_up[e] x);
// o = W_down[e] h; y[m] = sum over slots, in slot order, of weight * o), with NVFP4 / MXFP4 expert
// weights and the chunk path's activation quantization.  The pages' counterpart: imp's MoE "top-k
// grouped GEMM" and its NVFP4 grouped GEMM for MoE prefill (imp README, "Features" table, row
// "Architectures"; release notes v0.7.0), there on sm_120a.  Five launches on one stream, no host
// synchronisation (the counts and the tile table live on the device, so the sequence can be
// captured in a CUDA graph):
//   1. route + counting sort (one CTA): top_k per token (ties to the lower expert index, a NaN logit
//      ranks as -inf), renormalised weights, then the (token, slot) entries sorted by expert --
//      tokens ascending within an expert, each expert's rows padded to whole 128-row tiles -- and
//      the table row tile -> expert;
//   2. gather: x rows into the sorted bf16 matrix (padding rows zero);
//   3. grouped chunk GEMM, gate_up: the sorted rows quantized as the chunk path quantizes (NVFP4:
//      one per-tensor scale over them; MXFP4: the OCP MX rule), each 128-row tile against its
//      expert's gate/up-interleaved weights, the SiLU-gate fused in the epilogue, h stored as bf16;
//   4. grouped chunk GEMM, down: h quantized the same way (NVFP4: its own per-tensor scale), each
//      tile against its expert's down weights, o (fp32) per sorted row;
//   5. combine: y[m] = sum over slots, in slot order, of weight * o[row of (m, slot)] (deterministic),
//      the optional h output, and the two GEMMs' status words folded into the caller's.
#include "chunk_common.cuh"

extern "C" cudaError_t qlin_launch_chunk_grouped(int fmt, const void* w, int64_t w_stride, int T2, int64_t N,
                                                 int64_t K, const void* x, int rows_max, float* y, int64_t ldy,
                                                 void* h, int64_t ldh, int64_t h_cols, const int* tile_expert,
                                                 const int* used_tm, void* ws, cudaStream_t s);
extern "C" size_t qlin_chunk_ws_bytes(int M, int64_t N, int64_t K);
extern "C" int64_t qlin_mma_tiles(int64_t N, int gate_up);

namespace qlin {

constexpr int kPfMaxTopK = 8;
constexpr int kPfMaxE = 256;
constexpr int kPfThreads = 1024;

static inline int64_t pf_al256(int64_t v) { return (v + 255) / 256 * 256; }

// Sorted rows at most: every (token, slot) entry plus up to 127 padding rows per expert.
static inline int pf_rows_max(int M, int E, int top_k) {
    const int64_t r = (int64_t)M * top_k + (int64_t)E * 127;
    return (int)((r + 127) / 128 * 128);
}

// Workspace layout (offsets in bytes).
struct PfLayout {
    int64_t pos, tile_expert, used_tm, row_token, xs, ws_a, hs, ws_b, os, total;
    int rows_max;
};

static PfLayout pf_layout(int M, int64_t H, int64_t I, int E, int top_k) {
    PfLayout L;
    L.rows_max = pf_rows_max(M, E, top_k);
    const int64_t R = L.rows_max, TMx = R / 128;
    int64_t o = 256;  // [0, 256): the status word
    L.pos = o;
    o += pf_al256(4 * (int64_t)M * top_k);
    L.tile_expert = o;
    o += pf_al256(4 * TMx);
    L.used_tm = o;
    o += 256;
    L.row_token = o;
    o += pf_al256(4 * R);
    L.xs = o;
    o += pf_al256(2 * R * H);
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
    int M, E, top_k, TMx;
    int* pos;             // M x top_k: sorted row of (token, slot), -1 for a skipped slot
    int* tile_expert;     // TMx
    int* used_tm;
    int* row_token;       // rows_max: token of a sorted row, -1 for padding
    unsigned* status;     // bit 1: an invalid or repeated given expert id (the slot is skipped)
};

// Larger logit first, ties to the lower index; a NaN logit ranks as -inf.
__device__ __forceinline__ bool pf_before(float a, int ia, float b, int ib) {
    const float fa = a != a ? -INFINITY : a, fb = b != b ? -INFINITY : b;
    return fa > fb || (fa == fb && ia < ib);
}

__global__ void __launch_bounds__(kPfThreads) moe_prefill_route_kernel(const PfArgs a) {
    __shared__ int cnt[kPfMaxE];
    __shared__ int off[kPfMaxE + 1];
    __shared__ int warp_sum[kPfThreads / 32];
    __shared__ int chunk_base;
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int k = a.top_k;
    for (int e = tid; e < a.E; e += blockDim.x) cnt[e] = 0;
    __syncthreads();
    // 1. routing (or validation of the given ids), and the per-expert counts
    for (int m = tid; m < a.M; m += blockDim.x) {
        int32_t* id = a.ids + (int64_t)m * k;
        if (a.logits) {
            const float* l = a.logits + (int64_t)m * a.E;
            int sel[kPfMaxTopK];
            for (int e = 0; e < a.E; ++e) {
                int r = 0;
                const float le = l[e];
                for (int e2 = 0; e2 < a.E && r < k; ++e2) r += pf_before(l[e2], e2, le, e) ? 1 : 0;
                if (r < k) sel[r] = e;
            }
            const float lmax = l[sel[0]] != l[sel[0]] ? 0.f : l[sel[0]];
            float ex[kPfMaxTopK], sum = 0.f;
            for (int r = 0; r < k; ++r) {
                ex[r] = expf(l[sel[r]] - lmax);
                sum += ex[r];
            }
            for (int r = 0; r < k; ++r) {
                id[r] = sel[r];
                a.wts[(int64_t)m * k + r] = ex[r] / sum;
            }
        }
        for (int r = 0; r < k; ++r) {
            const int e = id[r];
            bool ok = e >= 0 && e < a.E;
            for (int r2 = 0; r2 < r && ok; ++r2) ok = id[r2] != e;
            if (ok) atomicAdd(&cnt[e], 1);
            else atomicOr(a.status, 2u);
        }
    }
    __syncthreads();
    // 2. offsets: each expert's rows padded to whole 128-row tiles; the tile table
    if (tid == 0) {
        int run = 0;
        for (int e = 0; e < a.E; ++e) {
            off[e] = run;
            run += (cnt[e] + 127) / 128 * 128;
        }
        off[a.E] = run;
        *a.used_tm = run / 128;
    }
    __syncthreads();
    for (int e = 0; e < a.E; ++e)
        for (int t = off[e] / 128 + tid; t < off[e + 1] / 128; t += blockDim.x) a.tile_expert[t] = e;
    for (int t = off[a.E] / 128 + tid; t < a.TMx; t += blockDim.x) a.tile_expert[t] = -1;
    for (int r = tid; r < a.TMx * 128; r += blockDim.x) a.row_token[r] = -1;
    for (int i = tid; i < a.M * k; i += blockDim.x) a.pos[i] = -1;
    __syncthreads();
    // 3. sorted rows: the entry (m, slot) of expert e goes to off[e] + #{m' < m routed to e}
    for (int e = 0; e < a.E; ++e) {
        if (cnt[e] == 0) continue;  // (uniform: every thread reads the same shared count)
        if (tid == 0) chunk_base = 0;
        __syncthreads();
        for (int m0 = 0; m0 < a.M; m0 += blockDim.x) {
            const int m = m0 + tid;
            int slot = -1;
            if (m < a.M) {
                const int32_t* id = a.ids + (int64_t)m * k;
                for (int r = 0; r < k; ++r) {
                    bool ok = id[r] == e;
                    for (int r2 = 0; r2 < r && ok; ++r2) ok = id[r2] != e;  // a repeated id counts once
                    if (ok) slot = r;
                }
            }
            const unsigned bal = __ballot_sync(0xffffffffu, slot >= 0);
            if (lane == 0) warp_sum[wid] = __popc(bal);
            __syncthreads();
            int before = chunk_base;
            for (int w = 0; w < wid; ++w) before += warp_sum[w];
            before += __popc(bal & ((1u << lane) - 1u));
            if (slot >= 0) {
                const int row = off[e] + before;
                a.pos[(int64_t)m * k + slot] = row;
                a.row_token[row] = m;
            }
            __syncthreads();
            if (tid == 0) {
                int tot = 0;
                for (int w = 0; w < (int)(blockDim.x >> 5); ++w) tot += warp_sum[w];
                chunk_base += tot;
            }
            __syncthreads();
        }
    }
}

// One CTA per sorted row in use: the token's bf16 activations, or zeros for a padding row.
__global__ void __launch_bounds__(128) moe_prefill_gather_kernel(const __nv_bfloat16* __restrict__ x, int64_t H,
                                                                 const int* __restrict__ row_token,
                                                                 const int* __restrict__ used_tm,
                                                                 __nv_bfloat16* __restrict__ xs) {
    const int r = blockIdx.x;
    if (r >= *used_tm * 128) return;
    const int t = row_token[r];
    uint4* dst = reinterpret_cast<uint4*>(xs + (int64_t)r * H);
    const uint4* src = reinterpret_cast<const uint4*>(x + (int64_t)(t < 0 ? 0 : t) * H);
    for (int64_t v = threadIdx.x; v < H / 8; v += blockDim.x) dst[v] = t < 0 ? make_uint4(0, 0, 0, 0) : src[v];
}

// One CTA per token: y[m] = sum over slots in slot order of w * o[row]; the optional h output
// (fp32 values of the bf16 h of each (token, slot)); the GEMMs' status words folded in.
__global__ void __launch_bounds__(256) moe_prefill_combine_kernel(const int* __restrict__ pos,
                                                                  const float* __restrict__ wts, int top_k,
                                                                  const float* __restrict__ os, int64_t H,
                                                                  const __nv_bfloat16* __restrict__ hs, int64_t I,
                                                                  float* __restrict__ y, float* __restrict__ h,
                                                                  unsigned* status, const unsigned* st_a,
                                                                  const unsigned* st_b) {
    const int m = blockIdx.x;
    if (m == 0 && threadIdx.x == 0) {
        const unsigned s = *st_a | *st_b;
        if (s) atomicOr(status, s & 1u);
    }
    int rows[kPfMaxTopK];
    float w[kPfMaxTopK];
    for (int r = 0; r < top_k; ++r) {
        rows[r] = pos[(int64_t)m * top_k + r];
        w[r] = wts[(int64_t)m * top_k + r];
    }
    for (int64_t n = threadIdx.x; n < H; n += blockDim.x) {
        float sum = 0.f;
        for (int r = 0; r < top_k; ++r)
            if (rows[r] >= 0) sum += w[r] * os[(int64_t)rows[r] * H + n];
        y[(int64_t)m * H + n] = sum;
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
    PfArgs pa;
    pa.logits = logits;
    pa.ids = ids;
    pa.wts = wts;
    pa.M = M;
    pa.E = E;
    pa.top_k = top_k;
    pa.TMx = L.rows_max / 128;
    pa.pos = (int*)(w8 + L.pos);
    pa.tile_expert = (int*)(w8 + L.tile_expert);
    pa.used_tm = (int*)(w8 + L.used_tm);
    pa.row_token = (int*)(w8 + L.row_token);
    pa.status = (unsigned*)ws;
    moe_prefill_route_kernel<<<1, kPfThreads, 0, s>>>(pa);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    __nv_bfloat16* xs = (__nv_bfloat16*)(w8 + L.xs);
    __nv_bfloat16* hs = (__nv_bfloat16*)(w8 + L.hs);
    float* os = (float*)(w8 + L.os);
    moe_prefill_gather_kernel<<<L.rows_max, 128, 0, s>>>((const __nv_bfloat16*)x, H, pa.row_token, pa.used_tm, xs);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    e = qlin_launch_chunk_grouped(fmt, gu, (int64_t)gu_stride, (int)qlin_mma_tiles(2 * I, 1), 2 * I, H, xs,
                                  L.rows_max, nullptr, 0, hs, I, I, pa.tile_expert, pa.used_tm, w8 + L.ws_a, s);
    if (e != cudaSuccess) return e;
    e = qlin_launch_chunk_grouped(fmt, dn, (int64_t)dn_stride, (int)qlin_mma_tiles(H, 0), H, I, hs, L.rows_max, os, H,
                                  nullptr, 0, 0, pa.tile_expert, pa.used_tm, w8 + L.ws_b, s);
    if (e != cudaSuccess) return e;
    moe_prefill_combine_kernel<<<M, 256, 0, s>>>(pa.pos, wts, top_k, os, H, hs, I, y, h, pa.status,
                                                 (const unsigned*)(w8 + L.ws_a), (const unsigned*)(w8 + L.ws_b));
    return cudaGetLastError();
}
