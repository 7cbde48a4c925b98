// api.cu -- the C ABI of libqlin: host-side validation, status codes, launches on the caller's
// stream.  Declarations and the contract of every entry point are in include/qlin.h.
#include <stdio.h>

#include "qlin_common.cuh"

extern "C" cudaError_t qlin_launch_pack(int fmt, const void* blocks, const void* scales, int64_t N,
                                        int64_t K, int pack_flags, float gs, void* packed,
                                        cudaStream_t s);
extern "C" cudaError_t qlin_launch_unpack(int fmt, const void* packed, int64_t N, int64_t K,
                                          int pack_flags, float* w, cudaStream_t s);
extern "C" size_t qlin_gemv_ws_bytes(int fmt, int M, int64_t N, int64_t K, int pack_flags);
extern "C" size_t qlin_moe_ws_bytes(int fmt, int M, int64_t H, int64_t I, int E, int top_k);
extern "C" cudaError_t qlin_launch_moe(int fmt, const void* gu, const void* dn, int E, int64_t H, int64_t I,
                                       int top_k, const float* logits, int32_t* ids, float* wts, const void* x,
                                       int xdt, int M, float* y, float* h, int flags, void* ws, cudaStream_t s);
extern "C" size_t qlin_chunk_ws_bytes(int M, int64_t N, int64_t K);
extern "C" int64_t qlin_bf16_cache_cols(int64_t K);
extern "C" int64_t qlin_bf16_cache_bytes(int64_t N, int64_t K);
extern "C" cudaError_t qlin_launch_chunk_bf16(const void* packed, int64_t N, int64_t K, const void* x, int M,
                                              int64_t ldx, float* y, int64_t ldy, void* ws, int flags,
                                              cudaStream_t s);
extern "C" cudaError_t qlin_launch_chunk(int fmt, const void* packed, int64_t N, int64_t K, const void* x, int M,
                                         int64_t ldx, float* y, int64_t ldy, void* ws, int flags, cudaStream_t s);
extern "C" cudaError_t qlin_launch_act_quant_mx(const void* x, int M, int64_t K, int64_t ldx, void* aq,
                                                void* canon_codes, void* canon_scales, cudaStream_t s);
extern "C" cudaError_t qlin_launch_act_quant_debug(const void* x, int M, int64_t K, int64_t ldx, void* ws,
                                                   void* codes, void* scales, float* ag, cudaStream_t s);
extern "C" cudaError_t qlin_launch_gemv(int fmt, const void* packed, int64_t N, int64_t K,
                                        const void* x, int xdt, int M, int64_t ldx, float* y,
                                        int64_t ldy, int flags, void* ws, cudaStream_t s);

extern "C" size_t qlin_moe_prefill_ws_bytes(int M, int64_t H, int64_t I, int E, int top_k);
extern "C" cudaError_t qlin_launch_moe_prefill(int fmt, const void* gu, const void* dn, int E, int64_t H, int64_t I,
                                               int top_k, const float* logits, int32_t* ids, float* wts,
                                               const void* x, int M, float* y, float* h, void* ws, size_t gu_stride,
                                               size_t dn_stride, cudaStream_t s);

extern "C" cudaError_t qlin_launch_fp4_mma_rate(int iters, unsigned long long* cycles, int max_ctas,
                                                unsigned* status, int* ctas, cudaStream_t s);
extern "C" int qlin_chain_max_ops();
extern "C" size_t qlin_chain_ws_bytes(int fmt, int M, const qlin_gemv_op* ops, int n_ops);
extern "C" cudaError_t qlin_launch_chain(int fmt, int xdt, int M, const qlin_gemv_op* ops, int n_ops, int flags,
                                         void* ws, cudaStream_t s);

namespace {

constexpr int64_t kMaxDim = (int64_t)1 << 31;

bool valid_fmt(int f) {
    return f == QLIN_Q8_0 || f == QLIN_Q4_0 || f == QLIN_NVFP4 || f == QLIN_MXFP4 || f == QLIN_Q4_K || f == QLIN_Q6_K;
}

bool valid_shape(int fmt, int64_t N, int64_t K) {
    if (N < 1 || K < 1 || N > kMaxDim || K > kMaxDim) return false;
    return fmt == QLIN_NVFP4 ? (K % 16 == 0) : (fmt == QLIN_Q4_K || fmt == QLIN_Q6_K) ? (K % 256 == 0) : (K % 32 == 0);
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

qlin_status_t cuda_status(cudaError_t e) { return e == cudaSuccess ? QLIN_OK : QLIN_ERR_CUDA; }

// One chain op against the qlin_gemv rules (op j of the chain).
qlin_status_t check_chain_op(int fmt, int xdt, const qlin_gemv_op& o, int j) {
    if (!valid_shape(fmt, o.N, o.K)) return QLIN_ERR_INVALID_ARG;
    if (o.epilogue & ~(0xf | QLIN_OUT_BF16)) return QLIN_ERR_INVALID_ARG;
    const int epi = o.epilogue & 0xf;
    if (epi != QLIN_EPI_NONE && epi != QLIN_EPI_SILU_GATE) return QLIN_ERR_INVALID_ARG;
    if (epi == QLIN_EPI_SILU_GATE && (o.N % 2)) return QLIN_ERR_INVALID_ARG;
    if (!o.packed || !o.x || !o.y) return QLIN_ERR_INVALID_ARG;
    const int64_t ncols = epi == QLIN_EPI_SILU_GATE ? o.N / 2 : o.N;
    if (o.ldx < o.K || o.ldy < ncols || o.ldx >= kMaxDim || o.ldy >= kMaxDim) return QLIN_ERR_INVALID_ARG;
    if (o.wait_for < -1 || o.wait_for >= j) return QLIN_ERR_INVALID_ARG;
    if (!aligned(o.packed, 256) || !aligned(o.x, 16) || !aligned(o.y, (o.epilogue & QLIN_OUT_BF16) ? 2 : 4))
        return QLIN_ERR_ALIGNMENT;
    if (o.ldx % (xdt == QLIN_F32 ? 4 : 8)) return QLIN_ERR_ALIGNMENT;
    const int pack_flags = epi == QLIN_EPI_SILU_GATE ? QLIN_PACK_GATE_UP : 0;
    if (qlin::geometry(fmt, o.N, o.K, pack_flags).U >= ((int64_t)1 << 30)) return QLIN_ERR_UNSUPPORTED;
    return QLIN_OK;
}

qlin_status_t check_chain(int fmt, int xdt, int M, const qlin_gemv_op* ops, int n_ops) {
    if (!valid_fmt(fmt) || (xdt != QLIN_F32 && xdt != QLIN_BF16) || M < 1 || M > 8) return QLIN_ERR_INVALID_ARG;
    if (!ops || n_ops < 1 || n_ops > qlin_chain_max_ops()) return QLIN_ERR_INVALID_ARG;
    for (int j = 0; j < n_ops; ++j) {
        const qlin_status_t st = check_chain_op(fmt, xdt, ops[j], j);
        if (st != QLIN_OK) return st;
    }
    return QLIN_OK;
}

}  // namespace

extern "C" {

size_t qlin_chain_workspace_bytes(qlin_format_t fmt, int M, const qlin_gemv_op* ops, int n_ops) {
    if (check_chain(fmt, QLIN_F32, M, ops, n_ops) != QLIN_OK && check_chain(fmt, QLIN_BF16, M, ops, n_ops) != QLIN_OK)
        return 0;
    return qlin_chain_ws_bytes(fmt, M, ops, n_ops);
}

qlin_status_t qlin_gemv_chain(qlin_format_t fmt, qlin_dtype_t xdt, int M, const qlin_gemv_op* ops, int n_ops,
                              int flags, void* ws, size_t ws_bytes, qlin_stream_t stream) {
    const qlin_status_t st = check_chain(fmt, xdt, M, ops, n_ops);
    if (st != QLIN_OK) return st;
    if (flags & ~QLIN_FLAG_PDL) return QLIN_ERR_INVALID_ARG;
    if (!ws || ws_bytes < qlin_chain_ws_bytes(fmt, M, ops, n_ops)) return QLIN_ERR_WORKSPACE;
    if (!aligned(ws, 256)) return QLIN_ERR_ALIGNMENT;
    return cuda_status(qlin_launch_chain(fmt, xdt, M, ops, n_ops, flags, ws, (cudaStream_t)stream));
}

size_t qlin_packed_bytes(qlin_format_t fmt, int64_t N, int64_t K, int pack_flags) {
    if (!valid_fmt(fmt) || !valid_shape(fmt, N, K)) return 0;
    if (pack_flags == (QLIN_PACK_MMA | QLIN_PACK_GATE_UP)) {  // NVFP4 / MXFP4: gate and up rows interleaved
        if ((fmt != QLIN_NVFP4 && fmt != QLIN_MXFP4) || N % 2) return 0;
        return (size_t)qlin::kHdrBytes + (size_t)((N / 2 + 127) / 128) * (size_t)((K + 255) / 256) * 36864u;
    }
    if (pack_flags == QLIN_PACK_MMA_BF16)  // the bf16 copy, every format
        return (size_t)qlin::kHdrBytes + (size_t)qlin_bf16_cache_bytes(N, K);
    if (pack_flags == QLIN_PACK_MMA) {
        if (fmt != QLIN_NVFP4 && fmt != QLIN_MXFP4)  // the bf16 copy of the dequantized weights, rows of K rounded up to 64
            return (size_t)qlin::kHdrBytes + (size_t)qlin_bf16_cache_bytes(N, K);
        return (size_t)qlin::kHdrBytes + (size_t)((N + 255) / 256) * (size_t)((K + 255) / 256) * 36864u;
    }
    if (pack_flags & ~QLIN_PACK_GATE_UP) return 0;
    if ((pack_flags & QLIN_PACK_GATE_UP) && (N % 2)) return 0;
    qlin::Geometry g = qlin::geometry(fmt, N, K, pack_flags);
    return (size_t)qlin::kHdrBytes + (size_t)g.U * (size_t)qlin::unit_bytes(fmt);
}

qlin_status_t qlin_pack_weights(qlin_format_t fmt, int64_t N, int64_t K, const void* blocks,
                                const void* scales, float global_scale, int pack_flags,
                                void* packed, size_t packed_bytes, qlin_stream_t stream) {
    if (!valid_fmt(fmt)) return QLIN_ERR_INVALID_ARG;
    if (!valid_shape(fmt, N, K)) return QLIN_ERR_INVALID_ARG;
    if (pack_flags != QLIN_PACK_MMA && pack_flags != QLIN_PACK_MMA_BF16 && (pack_flags & ~QLIN_PACK_GATE_UP) &&
        pack_flags != (QLIN_PACK_MMA | QLIN_PACK_GATE_UP))
        return QLIN_ERR_INVALID_ARG;
    if (pack_flags == (QLIN_PACK_MMA | QLIN_PACK_GATE_UP) && fmt != QLIN_NVFP4 && fmt != QLIN_MXFP4)
        return QLIN_ERR_UNSUPPORTED;
    if ((pack_flags & QLIN_PACK_GATE_UP) && (N % 2)) return QLIN_ERR_INVALID_ARG;
    if (!blocks || !packed) return QLIN_ERR_INVALID_ARG;
    if ((fmt == QLIN_NVFP4 || fmt == QLIN_MXFP4) && !scales) return QLIN_ERR_INVALID_ARG;
    if (!aligned(packed, 256)) return QLIN_ERR_ALIGNMENT;
    if (packed_bytes < qlin_packed_bytes(fmt, N, K, pack_flags)) return QLIN_ERR_INVALID_ARG;
    const float gs = fmt == QLIN_NVFP4 ? global_scale : 1.0f;
    return cuda_status(qlin_launch_pack(fmt, blocks, scales, N, K, pack_flags, gs, packed,
                                        (cudaStream_t)stream));
}

size_t qlin_workspace_bytes(int op, qlin_format_t fmt, int M, int64_t N, int64_t K, int E, int top_k) {
    (void)E;
    (void)top_k;
    if (!valid_fmt(fmt) || !valid_shape(fmt, N, K)) return 0;
    if (op == QLIN_OP_MOE) {  /* N = H, K = I */
        if (M < 1 || M > 8 || E < 1 || E > 256 || top_k < 1 || top_k > 8 || top_k > E) return 0;
        if (!valid_shape(fmt, 2 * K, N) || !valid_shape(fmt, N, K)) return 0;
        return qlin_moe_ws_bytes(fmt, M, N, K, E, top_k);
    }
    if (op == QLIN_OP_MOE_PREFILL) {  /* N = H, K = I */
        if ((fmt != QLIN_NVFP4 && fmt != QLIN_MXFP4) || M < 1 || M > (1 << 20) || E < 1 || E > 256 || top_k < 1 ||
            top_k > 8 || top_k > E || N % 32 || K % 32)
            return 0;
        return qlin_moe_prefill_ws_bytes(M, N, K, E, top_k);
    }
    if (op == QLIN_OP_CHUNK) {
        if (M < 1 || M > (1 << 20)) return 0;
        return (fmt == QLIN_NVFP4 || fmt == QLIN_MXFP4) ? qlin_chunk_ws_bytes(M, N, K) : 256;  // bf16 path: the status word
    }
    if (op == QLIN_OP_GEMV) {
        if (M < 1 || M > 8) return 0;
        size_t a = qlin_gemv_ws_bytes(fmt, M, N, K, 0);
        size_t b = (N % 2 == 0) ? qlin_gemv_ws_bytes(fmt, M, N, K, QLIN_PACK_GATE_UP) : 0;
        return a > b ? a : b;
    }
    return 0;
}

qlin_status_t qlin_gemv(qlin_format_t fmt, const void* packed, int64_t N, int64_t K, const void* x,
                        qlin_dtype_t xdt, int M, int64_t ldx, float* y, int64_t ldy, int flags,
                        void* ws, size_t ws_bytes, qlin_stream_t stream) {
    if (!valid_fmt(fmt) || !valid_shape(fmt, N, K)) return QLIN_ERR_INVALID_ARG;
    if (M < 1 || M > 8) return QLIN_ERR_INVALID_ARG;
    if (xdt != QLIN_F32 && xdt != QLIN_BF16) return QLIN_ERR_INVALID_ARG;
    const int epi = flags & 0xff;
    if (epi != QLIN_EPI_NONE && epi != QLIN_EPI_SILU_GATE) return QLIN_ERR_INVALID_ARG;
    if (flags & ~(0xff | QLIN_FLAG_PDL)) return QLIN_ERR_INVALID_ARG;
    if (epi == QLIN_EPI_SILU_GATE && (N % 2)) return QLIN_ERR_INVALID_ARG;
    if (!packed || !x || !y) return QLIN_ERR_INVALID_ARG;
    const int64_t ncols = epi == QLIN_EPI_SILU_GATE ? N / 2 : N;
    if (ldx < K || ldy < ncols) return QLIN_ERR_INVALID_ARG;
    if (!aligned(packed, 256) || !aligned(x, 16) || !aligned(y, 4)) return QLIN_ERR_ALIGNMENT;
    if (ldx % (xdt == QLIN_F32 ? 4 : 8)) return QLIN_ERR_ALIGNMENT;
    const int pack_flags = epi == QLIN_EPI_SILU_GATE ? QLIN_PACK_GATE_UP : 0;
    if (qlin::geometry(fmt, N, K, pack_flags).U >= ((int64_t)1 << 31)) return QLIN_ERR_UNSUPPORTED;
    const size_t need = qlin_gemv_ws_bytes(fmt, M, N, K, pack_flags);
    if (!ws || ws_bytes < need) return QLIN_ERR_WORKSPACE;
    if (!aligned(ws, 256)) return QLIN_ERR_ALIGNMENT;
    return cuda_status(qlin_launch_gemv(fmt, packed, N, K, x, xdt, M, ldx, y, ldy, flags, ws,
                                        (cudaStream_t)stream));
}

qlin_status_t qlin_moe_experts(qlin_format_t fmt, const void* gate_up_packed, const void* down_packed,
                               int E, int64_t H, int64_t I, int top_k, const float* router_logits,
                               int32_t* topk_ids, float* topk_w, const void* x, qlin_dtype_t xdt, int M,
                               float* y, float* h, int flags, void* ws, size_t ws_bytes,
                               qlin_stream_t stream) {
    if (!valid_fmt(fmt)) return QLIN_ERR_INVALID_ARG;
    if (M < 1 || M > 8 || E < 1 || E > 256 || top_k < 1 || top_k > 8 || top_k > E) return QLIN_ERR_INVALID_ARG;
    if (!valid_shape(fmt, 2 * I, H) || !valid_shape(fmt, H, I)) return QLIN_ERR_INVALID_ARG;
    if (H > 32768) return QLIN_ERR_UNSUPPORTED;  // down tiles per expert are tracked per token
    if (xdt != QLIN_F32 && xdt != QLIN_BF16) return QLIN_ERR_INVALID_ARG;
    if (flags & ~QLIN_FLAG_PDL) return QLIN_ERR_INVALID_ARG;
    if (!gate_up_packed || !down_packed || !topk_ids || !topk_w || !x || !y) return QLIN_ERR_INVALID_ARG;
    if (!aligned(gate_up_packed, 256) || !aligned(down_packed, 256) || !aligned(x, 16) || !aligned(y, 4) ||
        !aligned(topk_ids, 4) || !aligned(topk_w, 4) || (router_logits && !aligned(router_logits, 4)) ||
        (h && !aligned(h, 16)))
        return QLIN_ERR_ALIGNMENT;
    const size_t need = qlin_moe_ws_bytes(fmt, M, H, I, E, top_k);
    if (!ws || ws_bytes < need) return QLIN_ERR_WORKSPACE;
    if (!aligned(ws, 256)) return QLIN_ERR_ALIGNMENT;
    return cuda_status(qlin_launch_moe(fmt, gate_up_packed, down_packed, E, H, I, top_k, router_logits, topk_ids,
                                       topk_w, x, xdt, M, y, h, flags, ws, (cudaStream_t)stream));
}

qlin_status_t qlin_moe_prefill(qlin_format_t fmt, const void* gate_up_packed, const void* down_packed, int E,
                               int64_t H, int64_t I, int top_k, const float* router_logits, int32_t* topk_ids,
                               float* topk_w, const void* x, int M, float* y, float* h, int flags, void* ws,
                               size_t ws_bytes, qlin_stream_t stream) {
    if (!valid_fmt(fmt)) return QLIN_ERR_INVALID_ARG;
    if (fmt != QLIN_NVFP4 && fmt != QLIN_MXFP4) return QLIN_ERR_UNSUPPORTED;
    if (M < 1 || M > (1 << 20) || E < 1 || E > 256 || top_k < 1 || top_k > 8 || top_k > E) return QLIN_ERR_INVALID_ARG;
    if (H < 32 || I < 32 || H % 32 || I % 32 || H > kMaxDim || I > kMaxDim) return QLIN_ERR_INVALID_ARG;
    if (flags != 0) return QLIN_ERR_INVALID_ARG;
    if (!gate_up_packed || !down_packed || !topk_ids || !topk_w || !x || !y) return QLIN_ERR_INVALID_ARG;
    if (!aligned(gate_up_packed, 256) || !aligned(down_packed, 256) || !aligned(x, 16) || !aligned(y, 4) ||
        !aligned(topk_ids, 4) || !aligned(topk_w, 4) || (router_logits && !aligned(router_logits, 4)) ||
        (h && !aligned(h, 4)))
        return QLIN_ERR_ALIGNMENT;
    const size_t need = qlin_moe_prefill_ws_bytes(M, H, I, E, top_k);
    if (!ws || ws_bytes < need) return QLIN_ERR_WORKSPACE;
    if (!aligned(ws, 256)) return QLIN_ERR_ALIGNMENT;
    const size_t gu_stride = qlin_packed_bytes(fmt, 2 * I, H, QLIN_PACK_MMA | QLIN_PACK_GATE_UP);
    const size_t dn_stride = qlin_packed_bytes(fmt, H, I, QLIN_PACK_MMA);
    return cuda_status(qlin_launch_moe_prefill(fmt, gate_up_packed, down_packed, E, H, I, top_k, router_logits,
                                               topk_ids, topk_w, x, M, y, h, ws, gu_stride, dn_stride,
                                               (cudaStream_t)stream));
}

qlin_status_t qlin_gemm_chunk(qlin_format_t fmt, const void* packed, int64_t N, int64_t K, const void* x,
                              int M, int64_t ldx, float* y, int64_t ldy, int flags, void* ws,
                              size_t ws_bytes, qlin_stream_t stream) {
    if (!valid_fmt(fmt)) return QLIN_ERR_INVALID_ARG;
    if (!valid_shape(fmt, N, K) || M < 1 || M > (1 << 20)) return QLIN_ERR_INVALID_ARG;
    if (flags & ~(QLIN_FLAG_PDL | QLIN_FLAG_CTA_PAIRS | QLIN_FLAG_BF16_COPY)) return QLIN_ERR_INVALID_ARG;
    if (!packed || !x || !y) return QLIN_ERR_INVALID_ARG;
    if (ldx < K || ldy < N) return QLIN_ERR_INVALID_ARG;
    if (!aligned(packed, 256) || !aligned(x, 2) || !aligned(y, 4)) return QLIN_ERR_ALIGNMENT;
    if ((fmt != QLIN_NVFP4 && fmt != QLIN_MXFP4) || (flags & QLIN_FLAG_BF16_COPY)) {
        // bf16 path: x is read by tensor-map loads (16-byte aligned rows)
        if (!aligned(x, 16) || ldx % 8) return QLIN_ERR_ALIGNMENT;
        if (!ws || ws_bytes < 256) return QLIN_ERR_WORKSPACE;
        if (!aligned(ws, 256)) return QLIN_ERR_ALIGNMENT;
        return cuda_status(qlin_launch_chunk_bf16(packed, N, K, x, M, ldx, y, ldy, ws, flags & ~QLIN_FLAG_BF16_COPY,
                                                  (cudaStream_t)stream));
    }
    if (!ws || ws_bytes < qlin_chunk_ws_bytes(M, N, K)) return QLIN_ERR_WORKSPACE;
    if (!aligned(ws, 256)) return QLIN_ERR_ALIGNMENT;
    return cuda_status(qlin_launch_chunk(fmt, packed, N, K, x, M, ldx, y, ldy, ws, flags, (cudaStream_t)stream));
}

qlin_status_t qlin_act_quant_debug(const void* x, int M, int64_t K, int64_t ldx, void* codes, void* scales,
                                   float* a_g, void* ws, size_t ws_bytes, qlin_stream_t stream) {
    if (!x || !codes || !scales || !a_g || M < 1 || K < 16 || K % 16 || ldx < K) return QLIN_ERR_INVALID_ARG;
    if (!ws || ws_bytes < qlin_chunk_ws_bytes(M, 256, K)) return QLIN_ERR_WORKSPACE;
    if (!aligned(ws, 256) || !aligned(codes, 8) || !aligned(a_g, 4)) return QLIN_ERR_ALIGNMENT;
    return cuda_status(qlin_launch_act_quant_debug(x, M, K, ldx, ws, codes, scales, a_g, (cudaStream_t)stream));
}

qlin_status_t qlin_act_quant_mx_debug(const void* x, int M, int64_t K, int64_t ldx, void* codes, void* scales,
                                      void* ws, size_t ws_bytes, qlin_stream_t stream) {
    if (!x || !codes || !scales || M < 1 || K < 32 || K % 32 || ldx < K) return QLIN_ERR_INVALID_ARG;
    if (!ws || ws_bytes < qlin_chunk_ws_bytes(M, 256, K)) return QLIN_ERR_WORKSPACE;
    if (!aligned(ws, 256) || !aligned(codes, 8)) return QLIN_ERR_ALIGNMENT;
    return cuda_status(qlin_launch_act_quant_mx(x, M, K, ldx, (uint8_t*)ws + 256, codes, scales, (cudaStream_t)stream));
}

qlin_status_t qlin_dequant_debug(qlin_format_t fmt, const void* packed, int64_t N, int64_t K,
                                 int pack_flags, float* w, qlin_stream_t stream) {
    if (!valid_fmt(fmt) || !valid_shape(fmt, N, K)) return QLIN_ERR_INVALID_ARG;
    if (pack_flags & ~QLIN_PACK_GATE_UP) return QLIN_ERR_INVALID_ARG;
    if ((pack_flags & QLIN_PACK_GATE_UP) && (N % 2)) return QLIN_ERR_INVALID_ARG;
    if (!packed || !w) return QLIN_ERR_INVALID_ARG;
    if (!aligned(packed, 256) || !aligned(w, 4)) return QLIN_ERR_ALIGNMENT;
    return cuda_status(qlin_launch_unpack(fmt, packed, N, K, pack_flags, w, (cudaStream_t)stream));
}

qlin_status_t qlin_ws_status(void* ws, qlin_stream_t stream) {
    if (!ws) return QLIN_ERR_INVALID_ARG;
    unsigned int word = 0;
    cudaError_t e = cudaMemcpyAsync(&word, ws, sizeof(word), cudaMemcpyDeviceToHost, (cudaStream_t)stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize((cudaStream_t)stream);
    if (e != cudaSuccess) return QLIN_ERR_CUDA;
    if (word == 0) return QLIN_OK;
    e = cudaMemsetAsync(ws, 0, sizeof(word), (cudaStream_t)stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize((cudaStream_t)stream);
    if (e != cudaSuccess) return QLIN_ERR_CUDA;
    return (word & 1u) ? QLIN_ERR_TIMEOUT : QLIN_ERR_INVALID_ARG;  /* bit 1: bad expert id */
}

qlin_status_t qlin_ws_set_wait_budget(void* ws, uint32_t ns, qlin_stream_t stream) {
    if (!ws) return QLIN_ERR_INVALID_ARG;
    if (!aligned(ws, 256)) return QLIN_ERR_ALIGNMENT;
    cudaError_t e = cudaMemcpyAsync((uint8_t*)ws + qlin::kWsWaitBudgetOff, &ns, sizeof(ns), cudaMemcpyHostToDevice,
                                    (cudaStream_t)stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize((cudaStream_t)stream);  // ns lives on this stack
    return cuda_status(e);
}

qlin_status_t qlin_probe_fp4_mma(int iters, unsigned long long* cycles, int max_ctas, unsigned int* status,
                                 int* ctas, qlin_stream_t stream) {
    if (iters < 1 || iters > (1 << 20) || max_ctas < 1 || !cycles || !status || !ctas) return QLIN_ERR_INVALID_ARG;
    if (!aligned(cycles, 8) || !aligned(status, 4)) return QLIN_ERR_ALIGNMENT;
    *ctas = 0;
    const cudaError_t e = qlin_launch_fp4_mma_rate(iters, cycles, max_ctas, status, ctas, (cudaStream_t)stream);
    if (e == cudaErrorInvalidValue && *ctas > max_ctas) return QLIN_ERR_INVALID_ARG;  // nothing launched
    return cuda_status(e);
}

const char* qlin_status_string(qlin_status_t s) {
    switch (s) {
        case QLIN_OK: return "QLIN_OK";
        case QLIN_ERR_INVALID_ARG: return "QLIN_ERR_INVALID_ARG";
        case QLIN_ERR_UNSUPPORTED: return "QLIN_ERR_UNSUPPORTED";
        case QLIN_ERR_ALIGNMENT: return "QLIN_ERR_ALIGNMENT";
        case QLIN_ERR_WORKSPACE: return "QLIN_ERR_WORKSPACE";
        case QLIN_ERR_CUDA: return "QLIN_ERR_CUDA";
        case QLIN_ERR_TIMEOUT: return "QLIN_ERR_TIMEOUT";
    }
    return "QLIN_ERR_UNKNOWN";
}

}  // extern "C"
