"""Python binding of libqlin (the C ABI declared in include/qlin.h).

Argument marshalling only: every step of the computation runs in the CUDA library.  PyTorch
supplies device memory and the current stream.  The library is loaded on first use from this
directory (build it with ``python -m gemm_dequant_gemv_q8_b200.build``); if it is missing or
cannot be loaded every call raises -- there is no fallback of any kind.

The functions keep the C names (``qlin_pack_weights``, ``qlin_gemv``, ...).  They take torch
tensors, check dtype/device/contiguity, and pass raw pointers, sizes and the current stream.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

QLIN_Q8_0, QLIN_Q4_0, QLIN_NVFP4, QLIN_MXFP4, QLIN_Q4_K, QLIN_Q6_K = 1, 2, 3, 4, 5, 6
QLIN_F32, QLIN_BF16 = 0, 1
QLIN_EPI_NONE, QLIN_EPI_SILU_GATE, QLIN_OUT_BF16, QLIN_FLAG_PDL, QLIN_FLAG_CTA_PAIRS = 0, 1, 0x10, 0x100, 0x200
QLIN_FLAG_BF16_COPY = 0x400
QLIN_PACK_DEFAULT, QLIN_PACK_GATE_UP, QLIN_PACK_MMA, QLIN_PACK_MMA_BF16 = 0, 1, 2, 4
QLIN_OP_GEMV, QLIN_OP_MOE, QLIN_OP_CHUNK, QLIN_OP_MOE_PREFILL = 1, 2, 3, 4
STATUS = {0: "QLIN_OK", 1: "QLIN_ERR_INVALID_ARG", 2: "QLIN_ERR_UNSUPPORTED",
          3: "QLIN_ERR_ALIGNMENT", 4: "QLIN_ERR_WORKSPACE", 5: "QLIN_ERR_CUDA",
          6: "QLIN_ERR_TIMEOUT"}

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libqlin.so")
_lock = threading.Lock()
_lib = None

_P, _I64, _I, _F, _SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
# name -> (restype, argtypes); mirrors include/qlin.h
SIGNATURES = {
    "qlin_packed_bytes": (_SZ, [_I, _I64, _I64, _I]),
    "qlin_pack_weights": (_I, [_I, _I64, _I64, _P, _P, _F, _I, _P, _SZ, _P]),
    "qlin_workspace_bytes": (_SZ, [_I, _I, _I, _I64, _I64, _I, _I]),
    "qlin_gemv": (_I, [_I, _P, _I64, _I64, _P, _I, _I, _I64, _P, _I64, _I, _P, _SZ, _P]),
    "qlin_gemv_noalloc": (_I, [_I, _P, _I64, _I64, _P, _I, _I, _I64, _P, _I64, _I, _P]),
    "qlin_gemv_noalloc_status": (_I, [_P]),
    "qlin_moe_experts": (_I, [_I, _P, _P, _I, _I64, _I64, _I, _P, _P, _P, _P, _I, _I, _P, _P, _I, _P, _SZ, _P]),
    "qlin_gemm_chunk": (_I, [_I, _P, _I64, _I64, _P, _I, _I64, _P, _I64, _I, _P, _SZ, _P]),
    "qlin_moe_prefill": (_I, [_I, _P, _P, _I, _I64, _I64, _I, _P, _P, _P, _P, _I, _P, _P, _I, _P, _SZ, _P]),
    "qlin_act_quant_debug": (_I, [_P, _I, _I64, _I64, _P, _P, _P, _P, _SZ, _P]),
    "qlin_act_quant_mx_debug": (_I, [_P, _I, _I64, _I64, _P, _P, _P, _SZ, _P]),
    "qlin_dequant_debug": (_I, [_I, _P, _I64, _I64, _I, _P, _P]),
    "qlin_chain_max_ops": (_I, []),
    "qlin_chain_workspace_bytes": (_SZ, [_I, _I, _P, _I]),
    "qlin_gemv_chain": (_I, [_I, _I, _I, _P, _I, _I, _P, _SZ, _P]),
    "qlin_ws_status": (_I, [_P, _P]),
    "qlin_ws_set_wait_budget": (_I, [_P, ctypes.c_uint32, _P]),
    "qlin_probe_fp4_mma": (_I, [_I, _P, _I, _P, ctypes.POINTER(_I), _P]),
    "qlin_status_string": (ctypes.c_char_p, [_I]),
}


class GemvOp(ctypes.Structure):
    """struct qlin_gemv_op of include/qlin.h (64 bytes)."""
    _fields_ = [("packed", _P), ("N", _I64), ("K", _I64), ("x", _P), ("ldx", _I64), ("y", _P),
                ("ldy", _I64), ("epilogue", ctypes.c_int32), ("wait_for", ctypes.c_int32)]


class QlinError(RuntimeError):
    def __init__(self, fn, status):
        self.status = status
        super().__init__(f"{fn} failed: {STATUS.get(status, status)}")


def lib():
    """The loaded libqlin.so; raises if it is missing (no fallback path exists)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(f"libqlin.so not built at {LIB_PATH}; run "
                                   "`python -m gemm_dequant_gemv_q8_b200.build`")
            l = ctypes.CDLL(LIB_PATH)
            for name, (res, args) in SIGNATURES.items():
                fn = getattr(l, name)
                fn.restype, fn.argtypes = res, args
            _lib = l
    return _lib


def _stream(stream=None):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dev(t, name, dtype=None):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    return ctypes.c_void_p(t.data_ptr())


def _check(fn, st):
    if st != 0:
        raise QlinError(fn, st)


def _alloc_aligned(nbytes, device, align=256):
    buf = torch.empty(nbytes + align, dtype=torch.uint8, device=device)
    off = (-buf.data_ptr()) % align
    return buf[off:off + nbytes]


# ----------------------------------------------------------------------------- entry points
def qlin_packed_bytes(fmt, N, K, pack_flags=QLIN_PACK_DEFAULT):
    return lib().qlin_packed_bytes(fmt, N, K, pack_flags)


def qlin_pack_weights(fmt, N, K, blocks, scales=None, global_scale=1.0,
                      pack_flags=QLIN_PACK_DEFAULT, packed=None, stream=None):
    """Pack a canonical device tensor; returns the packed uint8 device buffer."""
    nbytes = qlin_packed_bytes(fmt, N, K, pack_flags)
    if nbytes == 0:
        raise QlinError("qlin_packed_bytes", 1)
    if packed is None:
        packed = _alloc_aligned(nbytes, blocks.device)
    st = lib().qlin_pack_weights(fmt, N, K, _dev(blocks, "blocks"), _dev(scales, "scales"),
                                 float(global_scale), pack_flags, _dev(packed, "packed"),
                                 packed.numel() * packed.element_size(), _stream(stream))
    _check("qlin_pack_weights", st)
    return packed


def qlin_workspace_bytes(op, fmt, M, N, K, E=0, top_k=0):
    return lib().qlin_workspace_bytes(op, fmt, M, N, K, E, top_k)


def workspace(nbytes, device="cuda"):
    """A zero-filled, 256-byte-aligned workspace of at least nbytes."""
    ws = _alloc_aligned(max(int(nbytes), 256), device)
    ws.zero_()
    return ws


def qlin_gemv(fmt, packed, N, K, x, y=None, flags=QLIN_EPI_NONE, ws=None, stream=None):
    """y = x @ W^T (or the SiLU-gate epilogue).  x: (M, K) fp32/bf16 CUDA, rows may be strided."""
    if x.dim() == 1:
        x = x.unsqueeze(0)
    M = x.shape[0]
    if x.stride(1) != 1:
        raise ValueError("x rows must be contiguous")
    xdt = {torch.float32: QLIN_F32, torch.bfloat16: QLIN_BF16}.get(x.dtype)
    if xdt is None:
        raise TypeError("x must be float32 or bfloat16")
    ncols = N // 2 if (flags & 0xFF) == QLIN_EPI_SILU_GATE else N
    if y is None:
        y = torch.empty(M, ncols, dtype=torch.float32, device=x.device)
    if ws is None:
        ws = workspace(qlin_workspace_bytes(QLIN_OP_GEMV, fmt, M, N, K), x.device)
    st = lib().qlin_gemv(fmt, _dev(packed, "packed"), N, K, _dev(x, "x"), xdt, M, x.stride(0),
                         _dev(y, "y", torch.float32), y.stride(0), flags, _dev(ws, "ws"),
                         ws.numel() * ws.element_size(), _stream(stream))
    _check("qlin_gemv", st)
    return y


def qlin_moe_experts(fmt, gate_up_packed, down_packed, E, H, I, top_k, x, router_logits=None,
                     topk_ids=None, topk_w=None, y=None, h=None, flags=0, ws=None, stream=None):
    """Routed MoE layer for M = x.shape[0] tokens.  Returns (y, topk_ids, topk_w, h)."""
    M = x.shape[0]
    xdt = {torch.float32: QLIN_F32, torch.bfloat16: QLIN_BF16}.get(x.dtype)
    if xdt is None or not x.is_contiguous():
        raise TypeError("x must be a contiguous float32 or bfloat16 tensor")
    dev = x.device
    if topk_ids is None:
        topk_ids = torch.empty(M, top_k, dtype=torch.int32, device=dev)
    if topk_w is None:
        topk_w = torch.empty(M, top_k, dtype=torch.float32, device=dev)
    if y is None:
        y = torch.empty(M, H, dtype=torch.float32, device=dev)
    if ws is None:
        ws = workspace(qlin_workspace_bytes(QLIN_OP_MOE, fmt, M, H, I, E, top_k), dev)
    st = lib().qlin_moe_experts(fmt, _dev(gate_up_packed, "gate_up_packed"), _dev(down_packed, "down_packed"),
                                E, H, I, top_k, _dev(router_logits, "router_logits", torch.float32),
                                _dev(topk_ids, "topk_ids", torch.int32), _dev(topk_w, "topk_w", torch.float32),
                                _dev(x, "x"), xdt, M, _dev(y, "y", torch.float32),
                                _dev(h, "h", torch.float32), flags, _dev(ws, "ws"),
                                ws.numel() * ws.element_size(), _stream(stream))
    _check("qlin_moe_experts", st)
    return y, topk_ids, topk_w, h


def qlin_moe_prefill(fmt, gate_up_packed, down_packed, E, H, I, top_k, x, router_logits=None, topk_ids=None,
                     topk_w=None, y=None, h=None, ws=None, stream=None):
    """Routed MoE layer for a prefill chunk of M = x.shape[0] bf16 tokens on the tensor cores
    (NVFP4 / MXFP4 experts packed with pack_experts(..., QLIN_PACK_MMA[ | QLIN_PACK_GATE_UP])).
    Returns (y, topk_ids, topk_w, h)."""
    if x.dtype != torch.bfloat16 or not x.is_contiguous():
        raise TypeError("x must be a contiguous bfloat16 tensor")
    M, dev = x.shape[0], x.device
    if topk_ids is None:
        topk_ids = torch.empty(M, top_k, dtype=torch.int32, device=dev)
    if topk_w is None:
        topk_w = torch.empty(M, top_k, dtype=torch.float32, device=dev)
    if y is None:
        y = torch.empty(M, H, dtype=torch.float32, device=dev)
    if ws is None:
        ws = workspace(qlin_workspace_bytes(QLIN_OP_MOE_PREFILL, fmt, M, H, I, E, top_k), dev)
    st = lib().qlin_moe_prefill(fmt, _dev(gate_up_packed, "gate_up_packed"), _dev(down_packed, "down_packed"), E, H,
                                I, top_k, _dev(router_logits, "router_logits", torch.float32),
                                _dev(topk_ids, "topk_ids", torch.int32), _dev(topk_w, "topk_w", torch.float32),
                                _dev(x, "x"), M, _dev(y, "y", torch.float32), _dev(h, "h", torch.float32), 0,
                                _dev(ws, "ws"), ws.numel() * ws.element_size(), _stream(stream))
    _check("qlin_moe_prefill", st)
    return y, topk_ids, topk_w, h


def pack_experts(fmt, E, N, K, canon, pack_flags=QLIN_PACK_DEFAULT, stream=None):
    """Pack E canonical expert tensors into one stacked buffer (E consecutive packed buffers).
    canon: list of (blocks, scales or None, global_scale) device tensors."""
    stride = qlin_packed_bytes(fmt, N, K, pack_flags)
    buf = _alloc_aligned(stride * E, canon[0][0].device)
    for e, (b, s, g) in enumerate(canon):
        qlin_pack_weights(fmt, N, K, b, s, g, pack_flags, packed=buf[e * stride:(e + 1) * stride], stream=stream)
    return buf


def qlin_gemm_chunk(fmt, packed, N, K, x, y=None, flags=0, ws=None, stream=None):
    """Prefill-chunk GEMM: y (M, N) fp32 = x (M, K) bf16 times W^T.  NVFP4 / MXFP4 weights packed
    with QLIN_PACK_MMA: x quantized in the same launch.  GGUF weights packed with QLIN_PACK_MMA,
    or any format packed with QLIN_PACK_MMA_BF16 and called with QLIN_FLAG_BF16_COPY: bf16 x
    times the bf16 copy of the weights."""
    if x.dtype != torch.bfloat16 or x.stride(1) != 1:
        raise TypeError("x must be bfloat16 with contiguous rows")
    M = x.shape[0]
    if y is None:
        y = torch.empty(M, N, dtype=torch.float32, device=x.device)
    if ws is None:
        ws = workspace(qlin_workspace_bytes(QLIN_OP_CHUNK, fmt, M, N, K), x.device)
    st = lib().qlin_gemm_chunk(fmt, _dev(packed, "packed"), N, K, _dev(x, "x"), M, x.stride(0),
                               _dev(y, "y", torch.float32), y.stride(0), flags, _dev(ws, "ws"),
                               ws.numel() * ws.element_size(), _stream(stream))
    _check("qlin_gemm_chunk", st)
    return y


def qlin_act_quant_debug(x, ws=None, stream=None):
    """Quantized activations of the chunk path in the canonical layout: (codes, scales, a_g)."""
    M, K = x.shape
    codes = torch.empty(M, K // 2, dtype=torch.uint8, device=x.device)
    scales = torch.empty(M, K // 16, dtype=torch.uint8, device=x.device)
    ag = torch.empty(1, dtype=torch.float32, device=x.device)
    if ws is None:
        ws = workspace(qlin_workspace_bytes(QLIN_OP_CHUNK, QLIN_NVFP4, M, 256, K), x.device)
    st = lib().qlin_act_quant_debug(_dev(x, "x"), M, K, x.stride(0), _dev(codes, "codes"), _dev(scales, "scales"),
                                    _dev(ag, "a_g"), _dev(ws, "ws"), ws.numel() * ws.element_size(), _stream(stream))
    _check("qlin_act_quant_debug", st)
    return codes, scales, ag


def qlin_act_quant_mx_debug(x, ws=None, stream=None):
    """The MXFP4 chunk path's quantized activations: (codes [M][K/2], UE8M0 scales [M][K/32])."""
    if x.dtype != torch.bfloat16 or x.stride(1) != 1:
        raise TypeError("x must be bfloat16 with contiguous rows")
    M, K = x.shape
    codes = torch.empty(M, K // 2, dtype=torch.uint8, device=x.device)
    scales = torch.empty(M, K // 32, dtype=torch.uint8, device=x.device)
    if ws is None:
        ws = workspace(qlin_workspace_bytes(QLIN_OP_CHUNK, QLIN_MXFP4, M, 256, K), x.device)
    st = lib().qlin_act_quant_mx_debug(_dev(x, "x"), M, K, x.stride(0), _dev(codes, "codes"), _dev(scales, "scales"),
                                       _dev(ws, "ws"), ws.numel() * ws.element_size(), _stream(stream))
    _check("qlin_act_quant_mx_debug", st)
    return codes, scales


def qlin_dequant_debug(fmt, packed, N, K, pack_flags=QLIN_PACK_DEFAULT, stream=None):
    w = torch.empty(N, K, dtype=torch.float32, device=packed.device)
    st = lib().qlin_dequant_debug(fmt, _dev(packed, "packed"), N, K, pack_flags,
                                  _dev(w, "w"), _stream(stream))
    _check("qlin_dequant_debug", st)
    return w


def qlin_ws_status(ws, stream=None):
    """Read and clear the workspace's sticky device status word (synchronises the stream)."""
    return lib().qlin_ws_status(_dev(ws, "ws"), _stream(stream))


def qlin_ws_set_wait_budget(ws, ns, stream=None):
    """Budget (ns) of the bounded inter-CTA waits of calls using ws; 0 = the default (~2 s)."""
    _check("qlin_ws_set_wait_budget", lib().qlin_ws_set_wait_budget(_dev(ws, "ws"), int(ns), _stream(stream)))


def qlin_probe_fp4_mma(iters, cycles, status, stream=None):
    """Launch the MMA-only FP4 rate probe: `iters` M128 N256 K64 mxf4nvf4 MMAs per SM.  cycles:
    an int64 CUDA tensor with one entry per possible CTA (its length is max_ctas); status: an
    int32 CUDA word that bit 0 is or-ed into if a wait gave up.  Returns the number of CTAs
    launched.  The caller times the launch."""
    if cycles.dtype != torch.int64 or status.dtype != torch.int32:
        raise TypeError("cycles must be int64 and status int32")
    ctas = _I(0)
    _check("qlin_probe_fp4_mma", lib().qlin_probe_fp4_mma(int(iters), _dev(cycles, "cycles"), cycles.numel(),
                                                          _dev(status, "status"), ctypes.byref(ctas),
                                                          _stream(stream)))
    return ctas.value


def qlin_status_string(status):
    return lib().qlin_status_string(status).decode()


def gemv_op(packed, N, K, x, y, epilogue=QLIN_EPI_NONE, wait_for=-1):
    """One op of a chain: the qlin_gemv arguments for one matrix (x, y CUDA tensors with
    contiguous rows; y bf16 with QLIN_OUT_BF16 in epilogue) and the index of an earlier op whose
    y this op's x reads (or -1)."""
    if x.dim() == 1:
        x = x.unsqueeze(0)
    if y.dim() == 1:
        y = y.unsqueeze(0)
    if x.stride(1) != 1 or y.stride(1) != 1:
        raise ValueError("x and y rows must be contiguous")
    ydt = torch.bfloat16 if epilogue & QLIN_OUT_BF16 else torch.float32
    return GemvOp(_dev(packed, "packed").value, N, K, _dev(x, "x").value, x.stride(0),
                  _dev(y, "y", ydt).value, y.stride(0), epilogue, wait_for)


def _op_array(ops):
    arr = (GemvOp * len(ops))(*ops)
    return arr, ctypes.cast(arr, ctypes.c_void_p)


def qlin_chain_max_ops():
    return lib().qlin_chain_max_ops()


def qlin_chain_workspace_bytes(fmt, M, ops):
    arr, ptr = _op_array(ops)
    return lib().qlin_chain_workspace_bytes(fmt, M, ptr, len(ops))


def qlin_gemv_chain(fmt, xdt, M, ops, flags=0, ws=None, stream=None):
    """Run the GEMVs `ops` (a list of gemv_op(...)) in one persistent launch; returns ws."""
    arr, ptr = _op_array(ops)
    if ws is None:
        ws = workspace(lib().qlin_chain_workspace_bytes(fmt, M, ptr, len(ops)))
    st = lib().qlin_gemv_chain(fmt, xdt, M, ptr, len(ops), flags, _dev(ws, "ws"),
                               ws.numel() * ws.element_size(), _stream(stream))
    _check("qlin_gemv_chain", st)
    return ws
