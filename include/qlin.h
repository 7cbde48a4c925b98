/*
 * qlin.h -- C ABI of libqlin, a B200 (sm_100a) library for the decode-step linear layer over
 * block-quantized weights: fused dequantize-and-multiply of GGUF Q8_0 / Q4_0 / Q4_K / Q6_K blocks and
 * NVFP4 / MXFP4 tensors against a small batch of activation rows, the routed MoE expert projections, and
 * an NVFP4 prefill-chunk GEMM on the tcgen05 tensor cores.
 *
 * What the operations compute comes from the pages describing the "imp" engine (README
 * "Features" table, rows "Quantization", "Architectures" and "sm_120a kernels"; README "Why this
 * exists"; release notes v0.6, "Native MXFP4 GGUF weight format") and the "Imparo" engine (README
 * intro: Q4_0 MoE decode with CUDA expert routing).  The pages name the formats but not their byte
 * layout; the layouts below are the public conventions (MXFP4: the OCP MX one, with the code byte
 * order of NVFP4; Q4_K / Q6_K: GGUF's block_q4_K / block_q6_K, the K-quants of the "Quantization"
 * row's GGUF files).
 *
 * Conventions for every entry point
 *   - W is N x K (output x input), row-major along K; y[m][n] = sum_k x[m][k] * W[n][k].
 *   - Every pointer argument is a caller-owned DEVICE pointer unless stated otherwise.  The
 *     library allocates nothing and keeps no global state, with two exceptions: a per-device
 *     SM-count cache, and qlin_gemv_noalloc's fixed 8 MiB __device__ scratch array (held by every
 *     GPU that loads the library) with its per-device address cache and the mutex guarding it.
 *     All work is enqueued asynchronously on `stream` (NULL = the legacy default stream).
 *   - Arguments are validated on the host before anything is launched; a failed check returns
 *     its status code and enqueues nothing.  A launch failure returns QLIN_ERR_CUDA.
 *   - No C++ exception crosses this boundary.
 *   - Workspaces ("ws") are caller-owned device buffers of at least qlin_workspace_bytes(...)
 *     bytes, 256-byte aligned, ZERO-FILLED before their first use.  Every call leaves the
 *     workspace's counters zero again when it completes, so a workspace can be reused by calls
 *     that run one after another on one stream; calls that overlap on the GPU must not share one.
 *     Where the counters sit depends on the call's shapes for qlin_gemv, qlin_gemv_chain and
 *     qlin_moe_experts: reuse their workspace only for calls with the same op and shapes (or zero
 *     it again).  qlin_gemm_chunk and qlin_moe_prefill keep theirs at fixed places or clear them
 *     themselves, so any later call may reuse their workspace.
 */
#ifndef QLIN_H
#define QLIN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* qlin_stream_t; /* a cudaStream_t */

typedef enum { QLIN_Q8_0 = 1, QLIN_Q4_0 = 2, QLIN_NVFP4 = 3, QLIN_MXFP4 = 4, QLIN_Q4_K = 5, QLIN_Q6_K = 6 } qlin_format_t;
typedef enum { QLIN_F32 = 0, QLIN_BF16 = 1 } qlin_dtype_t;
typedef enum {
    QLIN_OK = 0,
    QLIN_ERR_INVALID_ARG = 1, /* a null pointer, a size out of range, an unknown enum value   */
    QLIN_ERR_UNSUPPORTED = 2, /* a valid combination this library does not implement          */
    QLIN_ERR_ALIGNMENT = 3,   /* a pointer or leading dimension breaks the alignment rules    */
    QLIN_ERR_WORKSPACE = 4,   /* ws is NULL or smaller than qlin_workspace_bytes()            */
    QLIN_ERR_CUDA = 5,        /* a CUDA runtime call failed (launch, attribute query)         */
    QLIN_ERR_TIMEOUT = 6      /* a bounded device wait gave up (reported by qlin_ws_status)   */
} qlin_status_t;

/* qlin_gemv flags (OR-able) */
enum {
    QLIN_EPI_NONE = 0,      /* y[m][n] for n < N                                                 */
    QLIN_EPI_SILU_GATE = 1, /* gated MLP epilogue: rows [0, N/2) are the gate g, rows [N/2, N) the
                               up projection u; y[m][i] = silu(g_i) * u_i for i < N/2, with
                               silu(z) = z / (1 + exp(-z)).  Requires a QLIN_PACK_GATE_UP buffer. */
    QLIN_OUT_BF16 = 0x10,   /* qlin_gemv_chain ops only: y is bf16 (round to nearest even), ldy in
                               elements -- so that a later op of a bf16 chain can read it as x */
    QLIN_FLAG_PDL = 0x100,  /* launch with programmatic dependent launch: the kernel starts
                               streaming its weights while the previous kernel on the stream is
                               still running, and waits for it before touching x or y.  Only
                               valid when the packed weights were written before the previous
                               kernel on the stream started.                                      */
    QLIN_FLAG_CTA_PAIRS = 0x200, /* qlin_gemm_chunk only, M > 128: tile with pairs of CTAs
                               (tcgen05 cta_group::2, 256 activation rows per tile; each SM streams
                               half of every weight tile).  Same results; the default single-CTA
                               tiling is faster on the sizes measured so far. */
    QLIN_FLAG_BF16_COPY = 0x400  /* qlin_gemm_chunk only: `packed` is a QLIN_PACK_MMA_BF16 buffer, so
                               the bf16-operand path runs (for NVFP4 and MXFP4 weights too: bf16 x,
                               no activation quantization).  Optional for the GGUF formats, whose
                               chunk path is always the bf16 one. */
};

/* qlin_pack_weights flags */
enum {
    QLIN_PACK_DEFAULT = 0,
    QLIN_PACK_GATE_UP = 1, /* the N rows are [gate ; up] halves (N even): each packed tile pairs
                             16 gate rows with their 16 up rows so the SiLU-gate epilogue fuses */
    QLIN_PACK_MMA = 2,     /* the weight operand of qlin_gemm_chunk.  NVFP4 / MXFP4: the tensor-core
                             layout (tiles of 256 rows x 256 values, 128-byte-swizzled K-major codes,
                             scale factors in 512-byte atoms: E4M3 per 16 values, or UE8M0 per 32),
                             36864 B per tile (0.5625 B/weight) plus padding to 256 x 256.
                             Q8_0 / Q4_0 / Q4_K / Q6_K: a bf16 copy of the dequantized
                             weights after the 256-byte header, in blocks of 256 rows x 64 values
                             (32 KB contiguous, rows of 128 bytes): with Kc = roundup(K, 64), row n
                             and column k at element ((n / 256 * Kc / 64 + k / 64) * 256 + n % 256)
                             * 64 + k % 64; each weight the fp32 value of qlin_dequant_debug rounded
                             to nearest-even bf16, columns >= K and rows >= N (to a multiple of
                             256) zero (2 B/weight: the full-precision prefill copy; imp README
                             "Why this exists": prefill via source dequant) */
    QLIN_PACK_MMA_BF16 = 4  /* the bf16 copy, for every format (the same buffer as QLIN_PACK_MMA for the
                             GGUF formats; MXFP4: e2m1 * 2^(scale - 127), exact in bf16).  NVFP4: each element is the product of its
                             E2M1 code and its E4M3 block scale (at most 2 + 4 significant bits,
                             2^-10 <= |v| <= 2688: exact in bf16); the per-tensor scale stays in the
                             header and qlin_gemm_chunk applies it to each output once.  Layout and
                             size as the QLIN_PACK_MMA bf16 copy. */
};

/* qlin_workspace_bytes ops */
enum { QLIN_OP_GEMV = 1, QLIN_OP_MOE = 2, QLIN_OP_CHUNK = 3, QLIN_OP_MOE_PREFILL = 4 };

/* ------------------------------------------------------------------------- weight repacking */

/* Bytes of the packed buffer for an N x K tensor (0 for invalid arguments).
 * The packed layout is library-private: a 256-byte header (format, sizes, the NVFP4 per-tensor
 * scale), then tiles of 32 output rows x 256 inputs, each stored as 16-byte code vectors that a
 * warp reads contiguously, followed by that tile's scales; K is padded to a multiple of 256 and N
 * to a multiple of 32 (16 per half for QLIN_PACK_GATE_UP) with zero codes and zero scales.
 * The packed size is the canonical size plus that padding (Q8_0 1.0625 B/weight, Q4_0 and NVFP4
 * 0.5625 B/weight, MXFP4 0.53125 B/weight), except the K-quants: Q4_K 0.578125 B/weight against the
 * canonical 0.5625 (each sub-block's 6-bit scale and min take a 16-bit slot), Q6_K 1.078 B/weight
 * against 0.8203 (each 6-bit code takes a byte, decoded like Q8_0).  Prior art for a private re-laid-out weight copy: Imparo README intro
 * ("private GateUp layout"); imp README "Why this exists" (an NVFP4 decode cache built at init). */
size_t qlin_packed_bytes(qlin_format_t fmt, int64_t N, int64_t K, int pack_flags);

/* Re-lay a canonical tensor into the packed layout (one kernel, enqueued on `stream`).
 *   Q8_0 : blocks = GGUF block_q8_0 rows [N][K/32] x 34 B (fp16 d, int8 q[32]), scales = NULL
 *   Q4_0 : blocks = GGUF block_q4_0 rows [N][K/32] x 18 B (fp16 d, 16 B of nibbles; byte j holds
 *          element j low, element j+16 high), scales = NULL
 *   NVFP4: blocks = E2M1 codes [N][K/2] (byte i: element 2i low nibble, 2i+1 high nibble),
 *          scales = E4M3 [N][K/16], global_scale = the fp32 per-tensor scale
 *   MXFP4: blocks = E2M1 codes as NVFP4, scales = UE8M0 bytes [N][K/32] (value 2^(byte - 127),
 *          0xFF = NaN), global_scale ignored (imp release notes v0.6: E2M1 + UE8M0 block scales,
 *          4.25 bits per weight)
 *   Q4_K : blocks = GGUF block_q4_K rows [N][K/256] x 144 B: fp16 d, fp16 dmin, 12 bytes of
 *          6-bit sub-block scales and mins (sub-blocks 0..3 in the low 6 bits of bytes 0..3 /
 *          4..7; sub-blocks 4..7 with their low 4 bits in the nibbles of bytes 8..11 and their top
 *          2 bits in bits 6..7 of bytes 0..3 / 4..7), 128 bytes of codes (values 64c + l in the low
 *          nibble of byte 32c + l, values 64c + 32 + l in its high nibble); value k of sub-block
 *          j = k / 32 is d * scale_j * code - dmin * min_j; scales = NULL
 *   Q6_K : blocks = GGUF block_q6_K rows [N][K/256] x 210 B: ql[128] (low 4 code bits), qh[64]
 *          (high 2 bits), int8 scales[16] (one per 16 values), fp16 d; value 128h + 32s + l takes
 *          the low (s < 2) or high nibble of ql[64h + 32 (s & 1) + l], bits 2s..2s+1 of
 *          qh[32h + l] and scales[8h + 2s + l / 16]: w = d * scale * (code - 32); scales = NULL
 * K % 32 == 0 for Q8_0 / Q4_0 / MXFP4, K % 16 == 0 for NVFP4, K % 256 == 0 for Q4_K / Q6_K; N >= 1;
 * QLIN_PACK_GATE_UP needs N even.
 * `packed` must be 256-byte aligned and hold qlin_packed_bytes(...) bytes.  Canonical inputs
 * have no alignment requirement.  The canonical buffers may be freed once the kernel has run. */
qlin_status_t qlin_pack_weights(qlin_format_t fmt, int64_t N, int64_t K, const void* blocks,
                                const void* scales, float global_scale, int pack_flags,
                                void* packed, size_t packed_bytes, qlin_stream_t stream);

/* ------------------------------------------------------------------------- dense GEMV (M = 1..8) */

/* Workspace bytes for an op.  QLIN_OP_GEMV: (fmt, M, N, K); QLIN_OP_MOE: (fmt, M, N = H,
 * K = I, E, top_k); QLIN_OP_CHUNK: (fmt, M, N, K).  0 for invalid arguments. */
size_t qlin_workspace_bytes(int op, qlin_format_t fmt, int M, int64_t N, int64_t K, int E,
                            int top_k);

/* y = x * W^T for M activation rows, W packed by qlin_pack_weights with the same fmt, N, K
 * (QLIN_PACK_GATE_UP with QLIN_EPI_SILU_GATE, QLIN_PACK_DEFAULT otherwise).
 *   x   : M rows of K values, fp32 or bf16 (xdt), row stride ldx elements; 16-byte aligned with
 *         ldx a multiple of 4 (fp32) or 8 (bf16)
 *   y   : fp32, row stride ldy elements; N columns per row, or N/2 with QLIN_EPI_SILU_GATE
 *   flags: QLIN_EPI_* | QLIN_FLAG_PDL
 * Weights stream from HBM once; dequantization happens in registers; products and sums are fp32
 * (activations are never quantized).  Results are deterministic for a given device and shape.
 * Q8_0 / Q4_0 / Q4_K / Q6_K products are exact in fp32 for activations with 2^-40 <= |x| < 2^65; below that
 * range a product is exact to 2^-63 in absolute terms, at or above it the result overflows.  A 32-value
 * block whose scaled sum |d * sum q x| falls below 2^-40 (a tiny scale times tiny activations) is exact
 * to about 2^-64 in absolute terms.
 * The dequantize-and-multiply of quantized weight blocks against activations is the "NVFP4
 * block-scaled GEMM/GEMV" and "dp4a Q8_0 decode" of the imp pages (README "Features"; release
 * notes v0.4.1), re-designed here for sm_100a. */
qlin_status_t qlin_gemv(qlin_format_t fmt, const void* packed, int64_t N, int64_t K, const void* x,
                        qlin_dtype_t xdt, int M, int64_t ldx, float* y, int64_t ldy, int flags,
                        void* ws, size_t ws_bytes, qlin_stream_t stream);

/* Allocation-free variant of qlin_gemv.  The pages have no counterpart: this entry point exists
 * for callers that cannot allocate device memory for a workspace -- for example a plugin inside
 * a host application that owns every device allocation and hands out only the tensors it
 * manages, or a latency-critical decode loop that must not call cudaMalloc (which can
 * synchronise the device) once it is running.  Same arguments, semantics and results as
 * qlin_gemv, minus the workspace: the split-tile partial sums and tickets live in a fixed 8 MiB
 * array of the library's own device memory, which every GPU that loads the library holds until
 * the process exits.  It calls no cudaMalloc / cudaFree and no allocating library routine.
 *   - A shape whose workspace (qlin_workspace_bytes(QLIN_OP_GEMV, ...)) exceeds 8 MiB is rejected
 *     with QLIN_ERR_WORKSPACE before anything is enqueued.
 *   - The first call on each device looks up the array's device address (cudaGetSymbolAddress,
 *     with that device current); make that first call before any stream capture.
 *   - Every call clears the array's tile tickets on `stream` (cudaMemsetAsync), then launches the
 *     kernel.  All calls share the one array: calls that can overlap on the GPU (different
 *     streams without ordering between them) race and must not be issued.
 *   - The array's status word is sticky across calls, as a workspace's is: a bounded device wait
 *     that gave up sets it, and qlin_gemv_noalloc_status reads and clears it. */
qlin_status_t qlin_gemv_noalloc(qlin_format_t fmt, const void* packed, int64_t N, int64_t K,
                                const void* x, qlin_dtype_t xdt, int M, int64_t ldx, float* y,
                                int64_t ldy, int flags, qlin_stream_t stream);

/* Read and clear the status word of qlin_gemv_noalloc's scratch array on the current device, as
 * qlin_ws_status does for a workspace (synchronises `stream`): QLIN_OK, or QLIN_ERR_TIMEOUT if a
 * bounded device wait of some qlin_gemv_noalloc call on this device gave up since the last check. */
qlin_status_t qlin_gemv_noalloc_status(qlin_stream_t stream);

/* ------------------------------------------------------------------------- GEMV chains */

/* One GEMV of a chain: the arguments of qlin_gemv for one weight matrix, plus a dependency. */
typedef struct qlin_gemv_op {
    const void* packed; /* qlin_pack_weights output for (fmt, N, K); QLIN_PACK_GATE_UP iff SiLU gate */
    int64_t N, K;       /* packed rows and inputs, as for qlin_gemv (N, K < 2^31)                    */
    const void* x;      /* M x K activations in the chain's xdt, row stride ldx (qlin_gemv rules)    */
    int64_t ldx;
    float* y;           /* M x N (N/2 with QLIN_EPI_SILU_GATE) fp32 (bf16 with QLIN_OUT_BF16, passed
                           through this pointer), row stride ldy elements                           */
    int64_t ldy;
    int32_t epilogue;   /* QLIN_EPI_NONE or QLIN_EPI_SILU_GATE, optionally | QLIN_OUT_BF16           */
    int32_t wait_for;   /* -1, or the index of an EARLIER op of the same chain whose y this op's x
                           reads: the op then reads x only after every tile of that op is written */
} qlin_gemv_op;

/* Most ops in one chain. */
int qlin_chain_max_ops(void);

/* Workspace bytes of qlin_gemv_chain for these ops on the current device (0 if invalid). */
size_t qlin_chain_workspace_bytes(qlin_format_t fmt, int M, const qlin_gemv_op* ops, int n_ops);

/* Run n_ops GEMVs (all with format fmt, activation dtype xdt and M rows) in ONE persistent
 * launch.  Each op computes what qlin_gemv computes for its arguments, to the same tolerance (the
 * split of the K sums between warps differs, so the last bits can differ from qlin_gemv's;
 * repeated runs of one chain on one device agree bit for bit).  The weights of all ops stream back to back: the ramp-up and tail of
 * the HBM pipeline are paid once per chain instead of once per matrix, which is what a decode step
 * of many 2-30 MB projections needs (the pages capture their decode steps in CUDA graphs for the
 * per-launch overhead: imp release notes v0.4).  Ops run concurrently, in any order that respects
 * wait_for: an op with wait_for = i reads its x only after op i has written all of its y (a
 * bounded device-side wait; a wait that gives up after ~2 s sets the workspace status word,
 * reported by qlin_ws_status as QLIN_ERR_TIMEOUT), and the library may issue such an op a few
 * places later than given, after ops that do not wait.  No op may write memory that another op of
 * the chain reads or writes, except the y that a waiting op reads as its x.  The grid holds a fixed number of CTAs per SM; the dependency waits
 * assume nothing else keeps SMs busy for seconds while the chain runs.
 *   ops   : host array of n_ops descriptors (1 <= n_ops <= qlin_chain_max_ops()), read during the
 *           call only
 *   flags : 0 or QLIN_FLAG_PDL
 *   ws    : qlin_chain_workspace_bytes(fmt, M, ops, n_ops) bytes, zero-filled before first use
 * Errors: as qlin_gemv, per op; QLIN_ERR_INVALID_ARG also for n_ops out of range or a wait_for
 * that does not name an earlier op. */
qlin_status_t qlin_gemv_chain(qlin_format_t fmt, qlin_dtype_t xdt, int M, const qlin_gemv_op* ops, int n_ops,
                              int flags, void* ws, size_t ws_bytes, qlin_stream_t stream);

/* ------------------------------------------------------------------------- routed MoE experts */

/* Top-k routed MoE expert projections for M = 1..8 tokens.  Follows the Imparo README intro (a
 * Q4_0 MoE decode through "CUDA expert routing", LFM2.5-8B-A1B) and the imp README "Features"
 * table (MoE top-k grouped GEMM; an ordered, deterministic MoE reduction):
 *   route  : p = softmax(router_logits[m]); the top_k experts by p (a tie goes to the lower expert
 *            index; a NaN logit ranks as -inf); weights renormalised over the selected experts
 *   experts: h = silu(W_gate[e] x) * (W_up[e] x);  o = W_down[e] h   (fp32, as qlin_gemv)
 *   output : y[m] = sum over slots in slot order of weight * o
 * Only the selected experts' weights are read: once per call for every two tokens routed to the
 * expert (an expert chosen by 3..8 tokens is streamed 2..4 times, the repeats mostly from L2).
 * Arguments:
 *   gate_up_packed: E consecutive buffers, each qlin_packed_bytes(fmt, 2I, H, QLIN_PACK_GATE_UP)
 *                   bytes, expert e packed from its [gate ; up] rows (2I x H)
 *   down_packed   : E consecutive buffers, each qlin_packed_bytes(fmt, H, I, 0) bytes (H x I)
 *   router_logits : M x E fp32, or NULL -- then topk_ids / topk_w are inputs (ids in [0, E), no
 *                   repeats within a token; a bad slot is skipped and qlin_ws_status() reports
 *                   QLIN_ERR_INVALID_ARG)
 *   topk_ids, topk_w: M x top_k int32 / fp32, written when router_logits is given
 *   x : M x H rows (fp32 or bf16), contiguous;  y : M x H fp32, contiguous
 *   h : optional M x top_k x I fp32 output of the SiLU-gated intermediate (NULL: kept in ws)
 *   flags: 0 or QLIN_FLAG_PDL;  ws: qlin_workspace_bytes(QLIN_OP_MOE, fmt, M, H, I, E, top_k)
 * E <= 256, top_k <= min(8, E), H <= 32768 (else QLIN_ERR_UNSUPPORTED), any format.  One kernel launch on
 * `stream` (routing, gate_up of the selected experts, down, weighted sum), no host
 * synchronisation.  The status word (qlin_ws_status) reports a bad input expert id (the slot is
 * skipped) or a timed-out device wait. */
qlin_status_t qlin_moe_experts(qlin_format_t fmt, const void* gate_up_packed, const void* down_packed,
                               int E, int64_t H, int64_t I, int top_k, const float* router_logits,
                               int32_t* topk_ids, float* topk_w, const void* x, qlin_dtype_t xdt, int M,
                               float* y, float* h, int flags, void* ws, size_t ws_bytes,
                               qlin_stream_t stream);

/* Top-k routed MoE expert projections for a prefill chunk of M tokens (M >= 1; built for M >= 64)
 * on the tcgen05 tensor cores: what qlin_moe_experts computes -- the same routing (top_k by logit,
 * ties to the lower expert index, a NaN logit ranks as -inf, weights renormalised over the selected
 * experts), h = silu(W_gate[e] x) * (W_up[e] x), o = W_down[e] h, y[m] = sum over slots in slot
 * order of weight * o -- with NVFP4 or MXFP4 expert weights and the chunk path's quantization of
 * the activations:
 *   - x is quantized once per token as qlin_gemm_chunk quantizes it (NVFP4: one per-tensor scale
 *     from max |x| over all M tokens; MXFP4: the OCP MX rule) and copied to the token's sorted rows
 *     (the routed (token, slot) entries grouped by expert, each expert padded to whole 128-row
 *     tiles);
 *   - each 128-row tile is multiplied by its expert's gate/up weights with the SiLU-gate fused in
 *     the epilogue (silu from the MUFU ex2 / rcp units: within (2^-19 + |g| 2^-22) |h| of the fp32
 *     expression before h is rounded to bf16);
 *   - h (bf16) is quantized the same way for the down projection (NVFP4: its own per-tensor scale
 *     from max |h| over every routed row).
 * Which sorted row an entry takes depends on the order of device atomics, but every row is computed
 * on its own, so y, h, ids and weights are the same from run to run (and under graph replay).  The
 * pages' counterpart is imp's MoE top-k grouped GEMM, an NVFP4 grouped GEMM on sm_120a (imp README,
 * "Features" table, row "Architectures"; release notes v0.7.0).  Six launches on `stream` (route,
 * gather-quantize, grouped gate_up GEMM, h quantization, grouped down GEMM, combine), no host
 * synchronisation.
 *   gate_up_packed: E consecutive buffers, each qlin_packed_bytes(fmt, 2I, H, QLIN_PACK_MMA |
 *                   QLIN_PACK_GATE_UP) bytes, expert e packed from its [gate ; up] rows (2I x H)
 *   down_packed   : E consecutive buffers, each qlin_packed_bytes(fmt, H, I, QLIN_PACK_MMA) bytes
 *   router_logits : M x E fp32, or NULL -- then topk_ids / topk_w are inputs (a bad or repeated id is
 *                   skipped, its h row is zero, and qlin_ws_status() reports QLIN_ERR_INVALID_ARG)
 *   topk_ids, topk_w: M x top_k int32 / fp32, written when router_logits is given
 *   x : M x H bf16, contiguous, 16-byte aligned;  y : M x H fp32, contiguous
 *   h : optional M x top_k x I fp32: the bf16 h of each (token, slot), as fp32 (NULL: not written)
 *   flags: 0;  ws: qlin_workspace_bytes(QLIN_OP_MOE_PREFILL, fmt, M, H, I, E, top_k) bytes, zero-filled
 *       before its first use like every workspace
 * fmt NVFP4 or MXFP4 (else QLIN_ERR_UNSUPPORTED); E <= 256, top_k <= min(8, E); H % 32 == 0 and
 * I % 32 == 0 (QLIN_ERR_INVALID_ARG otherwise).  Bounded device waits as qlin_gemm_chunk. */
qlin_status_t qlin_moe_prefill(qlin_format_t fmt, const void* gate_up_packed, const void* down_packed, int E,
                               int64_t H, int64_t I, int top_k, const float* router_logits, int32_t* topk_ids,
                               float* topk_w, const void* x, int M, float* y, float* h, int flags, void* ws,
                               size_t ws_bytes, qlin_stream_t stream);

/* ------------------------------------------------------------------------- prefill-chunk GEMM */

/* GEMM for prefill chunks (M rows of bf16 activations, M >= 1; built for M >= 64) on the tcgen05
 * tensor cores.  NVFP4 weights take the block-scaled FP4 path described here; the other formats
 * the bf16 path described after it.  The counterpart on the pages is imp's NVFP4 block-scaled GEMM for
 * prefill (README "Features", row "sm_120a kernels": block-scaled mxf4nvf4 MMA, there with
 * mma.sync for sm_120a).  One persistent launch on `stream`, two steps:
 *   1. quantize x to NVFP4 (the A operand), all in fp32 with round-to-nearest-even:
 *        a_g = amax|x| / (6 * 448);  s_b = E4M3_rne_satfinite(amax_b / (6 * a_g)) per 16 values;
 *        code = E2M1_rne_satfinite(x / (e4m3(s_b) * a_g)), 0 where that divisor is 0
 *      (a bounded grid-wide barrier between the max and the quantization; all CTAs of the launch
 *      are resident at once, one per SM);
 *   2. y[m][n] = (a_g * g_w) * sum_k A_q[m][k] * W_q[n][k], block scales applied inside the MMA
 *      (kind::mxf4nvf4 block16), fp32 accumulation in tensor memory.  When the 128 x 256 output
 *      tiles number at most half the CTAs (M <= 128 with N <= 37 * 256 on 148 SMs, ...), each tile
 *      runs as two halves of its k-groups that add into y, which step 1 zeroes; two addends onto
 *      zero give the same sum in either order, so y stays deterministic.
 *   packed: qlin_pack_weights(QLIN_NVFP4, N, K, ..., QLIN_PACK_MMA);  x: bf16 M x K, row stride ldx;
 *   y: fp32, row stride ldy (16-byte aligned y and ldy % 4 == 0 take the TMA-store epilogue);
 *   flags: QLIN_FLAG_PDL and/or QLIN_FLAG_CTA_PAIRS;
 *   ws: qlin_workspace_bytes(QLIN_OP_CHUNK, QLIN_NVFP4, M, N, K, 0, 0) bytes.
 * bf16 path (Q8_0, Q4_0, MXFP4, Q4_K, Q6_K): y[m][n] = sum_k x[m][k] * Wb[n][k] with Wb the bf16
 * copy written by qlin_pack_weights(fmt, N, K, ..., QLIN_PACK_MMA), tcgen05.mma kind::f16 (bf16
 * operands loaded by tensor-map copies, fp32 accumulation in tensor memory); x must be 16-byte
 * aligned with ldx % 8 == 0 (else QLIN_ERR_ALIGNMENT); QLIN_FLAG_CTA_PAIRS (M > 128): 256 x 256
 * tiles on pairs of CTAs (cta_group::2), each staging its 128 activation rows and 128 weight rows;
 * ws: qlin_workspace_bytes(QLIN_OP_CHUNK, fmt, M, N, K, 0, 0) bytes (256: the status word).
 * Bounded device waits: a timeout sets the workspace status word (qlin_ws_status). */
/* bf16-operand path for NVFP4 weights (QLIN_FLAG_BF16_COPY with a QLIN_PACK_MMA_BF16 buffer):
 * y[m][n] = fl(g * sum_k x[m][k] * (e2m1 * e4m3)[n][k]): the bf16 x as given against the exact block
 * products, fp32 accumulation in tensor memory, the per-tensor scale g applied once per output.  The
 * activations are not quantized, so this path meets the bf16-operand chunk bound |y - y_ref| <=
 * 1e-2 * sum|w x| against the unquantized product, which the FP4-activation path above does not
 * guarantee (its per-output error against y_ref is that of NVFP4-quantized activations, up to about
 * 1e-2 * sum|w x| on random data).  It streams 2 bytes per weight instead of 0.5625. */
qlin_status_t qlin_gemm_chunk(qlin_format_t fmt, const void* packed, int64_t N, int64_t K, const void* x,
                              int M, int64_t ldx, float* y, int64_t ldy, int flags, void* ws,
                              size_t ws_bytes, qlin_stream_t stream);

/* MXFP4 weights (QLIN_PACK_MMA) take the same one-launch form with MXFP4 activations and the
 * kind::mxf4 MMA (UE8M0 scales of 32 values, the scale byte pair of each K = 64 step selected in the
 * instruction descriptor): step 1 quantizes x by the OCP MX rule -- per 32 consecutive values of a
 * row, scale byte = floor(log2 amax) - 2 + 127 clamped to [0, 254] (0xFF for a block holding an Inf
 * or NaN), code = E2M1_rne_satfinite(x / 2^(byte - 127)) -- with no per-tensor scale, and step 2 is
 * y[m][n] = sum_k A_q[m][k] * W_q[n][k].  The pages give MXFP4 as E2M1 codes with UE8M0 block scales
 * (imp release notes v0.6, "Native MXFP4 GGUF weight format"); the activation rule is the OCP MX
 * conversion. */

/* Test and inspection aid: run step 1 of qlin_gemm_chunk alone and also write the quantized
 * activations in the canonical NVFP4 layout: codes [M][K/2] (element 2i in the low nibble), E4M3
 * scales [M][K/16], and a_g (one float, device memory).  ws as for qlin_gemm_chunk. */
qlin_status_t qlin_act_quant_debug(const void* x, int M, int64_t K, int64_t ldx, void* codes, void* scales,
                                   float* a_g, void* ws, size_t ws_bytes, qlin_stream_t stream);

/* The same for the MXFP4 chunk path: the MX-quantized activations in canonical layout, codes
 * [M][K/2] and UE8M0 scale bytes [M][K/32] (K % 32 == 0).  ws as for qlin_gemm_chunk. */
qlin_status_t qlin_act_quant_mx_debug(const void* x, int M, int64_t K, int64_t ldx, void* codes, void* scales,
                                      void* ws, size_t ws_bytes, qlin_stream_t stream);

/* Dequantize a packed buffer back to fp32 W[N][K] (row-major, canonical row order, also for
 * QLIN_PACK_GATE_UP buffers; pass the pack_flags the buffer was packed with).  The value of every
 * weight is the exact fp32 number d*q (Q8_0), d*(q-8) (Q4_0), fp32(e2m1*e4m3*g) rounded once
 * (NVFP4), e2m1 * 2^(scale - 127) (MXFP4: exact, +-Inf where it overflows fp32), or
 * fp32(d*scale*code - dmin*min) rounded once (Q4_K: both products are exact in fp32), or the
 * exact d*scale*(code - 32) (Q6_K).  A test and inspection aid; not on the hot path.  w must be 4-byte aligned. */
qlin_status_t qlin_dequant_debug(qlin_format_t fmt, const void* packed, int64_t N, int64_t K,
                                 int pack_flags, float* w, qlin_stream_t stream);

/* Read and clear the sticky device status word of a workspace (synchronises `stream`).
 * Returns QLIN_OK, QLIN_ERR_TIMEOUT if a bounded device wait gave up since the last check, or
 * QLIN_ERR_INVALID_ARG if qlin_moe_experts met an invalid or repeated expert id. */
qlin_status_t qlin_ws_status(void* ws, qlin_stream_t stream);

/* Test and fault-injection aid: set the budget, in nanoseconds, of the bounded device waits between
 * CTAs in the calls that use workspace `ws` -- qlin_gemv_chain's dependency and partial-sum waits,
 * qlin_moe_experts' waits for an expert's gate_up tiles, qlin_gemm_chunk's (NVFP4) grid barrier and
 * activation-ready waits.  0 restores the default of about 2 s.  The value is kept in the workspace
 * (the uint32 at byte 32, which a zero-filled workspace has at 0) until it is set again.  A wait
 * that runs out sets the status word (qlin_ws_status then reports QLIN_ERR_TIMEOUT), its warp
 * abandons the rest of its work and waits (bounded) for its own copies in flight, and the launch
 * finishes; that call's outputs are unspecified, and the workspace is usable again by the next
 * call.  Waits for this CTA's own bulk copies are not affected.  Synchronises `stream`.  The pages
 * have no counterpart (the Imparo README, "Why Imparo", reports failures rather than hiding them). */
qlin_status_t qlin_ws_set_wait_budget(void* ws, uint32_t ns, qlin_stream_t stream);

/* Measurement aid, not on the hot path: the MMA-only rate of the FP4 tensor path on this device,
 * the denominator beside the 9 PFLOP/s dense FP4 figure of the datacenter part (imp README, "Why
 * this exists": tcgen05 and TMEM are the datacenter path). Launches one CTA per SM on `stream`.
 * One thread of each CTA issues `iters` (1 .. 2^20) dependent tcgen05.mma kind::mxf4nvf4
 * block16 MMAs of M 128, N 256, K 64 (4,194,304 flops each). They use the instruction,
 * descriptors and instruction word of qlin_gemm_chunk's NVFP4 path, on fixed shared-memory
 * operands into one TMEM accumulator; the operands hold arbitrary E2M1 codes and E4M3 1.0 scales,
 * and nothing is written back.
 * cycles: device array of max_ctas uint64 (8-byte aligned). CTA i writes its clock64 span from
 *   the first issue to the MMAs' completion into cycles[i].
 * status: a device uint32 word; bit 0 is or-ed in if a CTA's bounded wait for its MMAs gave up
 *   (after about 2 s).
 * *ctas (host) receives the number of CTAs, the SM count. If that exceeds max_ctas, the call
 *   returns QLIN_ERR_INVALID_ARG and launches nothing.
 * The caller times the launch (CUDA events on `stream`): flops = 4,194,304 * iters * *ctas. */
qlin_status_t qlin_probe_fp4_mma(int iters, unsigned long long* cycles, int max_ctas, unsigned int* status,
                                 int* ctas, qlin_stream_t stream);

const char* qlin_status_string(qlin_status_t status);

#ifdef __cplusplus
}
#endif
#endif /* QLIN_H */
