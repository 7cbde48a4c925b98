"""fp64 CPU oracle for the quantized decode-step linear layer -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference legs of ``bench.py``
may import this package.  The product path (``gemm_dequant_gemv_q8_b200``) never imports it and
shares no code with it.  The arithmetic lives in ``oracle.c`` (plain C, fp64, sequential sums);
this module compiles it with gcc on first use and marshals numpy arrays.

Every function cites what it follows; the format layouts are the public GGUF / NVFP4 / OCP MX
conventions (the pages name the formats -- imp README, "Features" table, row "Quantization";
imp release notes v0.6, "Native MXFP4 GGUF weight format" -- but do not print their layout).

Parity pins for every function here live in ``tests/test_oracle_pins.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

Q8_0, Q4_0, NVFP4, MXFP4, Q4_K, Q6_K = 1, 2, 3, 4, 5, 6
_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so (plain -O2, no fast-math, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
                               "-fno-fast-math", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _l():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            P, I64, I, F, D = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float, ctypes.c_double
            lib.qo_fp16.restype = D; lib.qo_fp16.argtypes = [ctypes.c_uint16]
            lib.qo_e4m3.restype = D; lib.qo_e4m3.argtypes = [ctypes.c_uint8]
            lib.qo_e2m1.restype = D; lib.qo_e2m1.argtypes = [ctypes.c_uint8]
            lib.qo_e8m0.restype = D; lib.qo_e8m0.argtypes = [ctypes.c_uint8]
            lib.qo_silu.restype = D; lib.qo_silu.argtypes = [D]
            lib.qo_row_bytes.restype = I64; lib.qo_row_bytes.argtypes = [I, I64]
            lib.qo_dequant.restype = I; lib.qo_dequant.argtypes = [I, I64, I64, P, P, F, P]
            lib.qo_dequant_f32.restype = I; lib.qo_dequant_f32.argtypes = [I, I64, I64, P, P, F, P]
            lib.qo_gemv_rows.restype = I
            lib.qo_gemv_rows.argtypes = [I, I64, I64, P, P, F, I, P, P, I64, P, P]
            lib.qo_silu_gate.restype = None; lib.qo_silu_gate.argtypes = [I, I64, P, P, P, P]
            lib.qo_route.restype = None; lib.qo_route.argtypes = [I, I, P, P, P]
            lib.qo_moe.restype = I
            lib.qo_moe.argtypes = [I, I, I64, I64, I, P, P, P, P, P, P, I, P, P, P, P, P, P, P]
            lib.qo_round_e4m3_satfinite.restype = ctypes.c_uint8
            lib.qo_round_e4m3_satfinite.argtypes = [F]
            lib.qo_round_e2m1_satfinite.restype = ctypes.c_uint8
            lib.qo_round_e2m1_satfinite.argtypes = [F]
            lib.qo_act_quant.restype = I; lib.qo_act_quant.argtypes = [I, I64, P, P, P, P]
            lib.qo_act_quant_mx.restype = I; lib.qo_act_quant_mx.argtypes = [I, I64, P, P, P]
            _lib = lib
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _u8(a):
    if a is None:
        return None
    a = np.ascontiguousarray(np.asarray(a))
    return a.view(np.uint8)


# ----------------------------------------------------------------------------- scalar decoders
def fp16(bits: int) -> float:
    """IEEE binary16 decode (sign, 5-bit exponent bias 15, 10-bit mantissa)."""
    return _l().qo_fp16(bits)


def e4m3(bits: int) -> float:
    """OCP FP8 E4M3 'fn' decode (bias 7, subnormal m*2^-9, S.1111.111 = NaN, max 448)."""
    return _l().qo_e4m3(bits)


def e2m1(code: int) -> float:
    """OCP FP4 E2M1 decode (bias 1, subnormal m*0.5, max 6)."""
    return _l().qo_e2m1(code)


def e8m0(bits: int) -> float:
    """OCP MX UE8M0 scale decode: 2^(bits - 127), bits 0xFF = NaN."""
    return _l().qo_e8m0(bits)


def silu(z: float) -> float:
    return _l().qo_silu(z)


def row_bytes(fmt: int, K: int) -> int:
    return _l().qo_row_bytes(fmt, K)


# ----------------------------------------------------------------------------- tensors
def dequant(fmt, N, K, blocks, scales=None, g=1.0):
    """fp64 weights W[N][K] (exact real values of the blocks)."""
    W = np.empty((N, K), np.float64)
    rc = _l().qo_dequant(fmt, N, K, _p(_u8(blocks)), _p(_u8(scales)), g, _p(W))
    assert rc == 0, "bad arguments"
    return W


def dequant_f32(fmt, N, K, blocks, scales=None, g=1.0):
    """fp32 weights: the value the 'bit-exact dequant' check compares against."""
    W = np.empty((N, K), np.float32)
    rc = _l().qo_dequant_f32(fmt, N, K, _p(_u8(blocks)), _p(_u8(scales)), g, _p(W))
    assert rc == 0, "bad arguments"
    return W


def gemv(fmt, N, K, blocks, x, scales=None, g=1.0, rows=None):
    """y = W x and A = sum |W*x| in fp64 for x of shape (M, K); optional output-row subset.

    Returns (y, A), each (M, nrows)."""
    x = np.ascontiguousarray(np.asarray(x, np.float64).reshape(-1, K))
    M = x.shape[0]
    if rows is not None:
        rows = np.ascontiguousarray(np.asarray(rows, np.int64))
        nr = rows.size
    else:
        nr = N
    y = np.empty((M, nr), np.float64)
    A = np.empty((M, nr), np.float64)
    rc = _l().qo_gemv_rows(fmt, N, K, _p(_u8(blocks)), _p(_u8(scales)), g, M, _p(x),
                           _p(rows), nr, _p(y), _p(A))
    assert rc == 0, "bad arguments"
    return y, A


def silu_gate(gu, Agu=None):
    """h = silu(gate) * up for gate_up outputs laid out [gate ; up] along the last axis.

    Returns (h, Ah) where Ah is a first-order error magnitude for the fused epilogue."""
    gu = np.ascontiguousarray(np.asarray(gu, np.float64))
    M, twoI = gu.shape
    I = twoI // 2
    h = np.empty((M, I), np.float64)
    Ah = np.empty((M, I), np.float64)
    Agu = None if Agu is None else np.ascontiguousarray(np.asarray(Agu, np.float64))
    _l().qo_silu_gate(M, I, _p(gu), _p(Agu), _p(h), _p(Ah))
    return h, Ah


def route(logits, top_k):
    """Softmax, top-k by descending probability (tie -> lower expert), renormalised weights."""
    logits = np.ascontiguousarray(np.asarray(logits, np.float64))
    M, E = logits.shape
    ids = np.empty((M, top_k), np.int32)
    wts = np.empty((M, top_k), np.float64)
    for m in range(M):
        _l().qo_route(E, top_k, _p(logits[m]), _p(ids[m]), _p(wts[m]))
    return ids, wts


def moe(fmt, E, H, I, top_k, gu_blocks, dn_blocks, logits, x, gu_scales=None, dn_scales=None,
        gu_g=None, dn_g=None):
    """Routed MoE layer in fp64.  Returns dict(ids, wts, h, y, A)."""
    logits = np.ascontiguousarray(np.asarray(logits, np.float64))
    x = np.ascontiguousarray(np.asarray(x, np.float64))
    M = x.shape[0]
    ids = np.empty((M, top_k), np.int32)
    wts = np.empty((M, top_k), np.float64)
    h = np.empty((M, top_k, I), np.float64)
    y = np.empty((M, H), np.float64)
    A = np.empty((M, H), np.float64)
    gug = None if gu_g is None else np.ascontiguousarray(np.asarray(gu_g, np.float32))
    dng = None if dn_g is None else np.ascontiguousarray(np.asarray(dn_g, np.float32))
    rc = _l().qo_moe(fmt, E, H, I, top_k, _p(_u8(gu_blocks)), _p(_u8(gu_scales)), _p(gug),
                     _p(_u8(dn_blocks)), _p(_u8(dn_scales)), _p(dng), M, _p(logits), _p(x),
                     _p(ids), _p(wts), _p(h), _p(y), _p(A))
    assert rc == 0, "bad arguments"
    return dict(ids=ids, wts=wts, h=h, y=y, A=A)


def round_e4m3(v: float) -> int:
    return _l().qo_round_e4m3_satfinite(v)


def round_e2m1(v: float) -> int:
    return _l().qo_round_e2m1_satfinite(v)


def act_quant(X):
    """NVFP4 activation quantizer of the chunk path (fp32 rule).  X: (M, K) fp32 values that are
    exact bf16 numbers.  Returns (codes [M][K/2] u8, scales [M][K/16] u8, a_g float)."""
    X = np.ascontiguousarray(np.asarray(X, np.float32))
    M, K = X.shape
    codes = np.empty((M, K // 2), np.uint8)
    scales = np.empty((M, K // 16), np.uint8)
    ag = np.empty(1, np.float32)
    rc = _l().qo_act_quant(M, K, _p(X), _p(codes), _p(scales), _p(ag))
    assert rc == 0, "bad arguments"
    return codes, scales, float(ag[0])


def gemm_same_quant(w_codes, w_scales, w_g, a_codes, a_scales, a_g, N, K):
    """y_q[m][n] = sum_k A_q[m][k] * W[n][k] with both operands the exact NVFP4 values, fp64.

    Returns (y, A) as gemv does."""
    Aq = dequant(NVFP4, a_codes.shape[0], K, a_codes, a_scales, a_g)
    return gemv(NVFP4, N, K, w_codes, Aq, scales=w_scales, g=w_g)


def act_quant_mx(X):
    """MXFP4 activation quantizer of the MXFP4 chunk path (OCP MX rule: one UE8M0 scale
    2^(floor(log2 amax) - 2) per 32 values, E2M1 codes rounded to nearest even, saturating).
    X: (M, K) fp32 values that are exact bf16 numbers.  Returns (codes [M][K/2], scales [M][K/32])."""
    X = np.ascontiguousarray(np.asarray(X, np.float32))
    M, K = X.shape
    codes = np.empty((M, K // 2), np.uint8)
    scales = np.empty((M, K // 32), np.uint8)
    rc = _l().qo_act_quant_mx(M, K, _p(X), _p(codes), _p(scales))
    assert rc == 0, "bad arguments"
    return codes, scales


def gemm_same_quant_mx(w_codes, w_scales, a_codes, a_scales, N, K):
    """y_q[m][n] = sum_k A_q[m][k] * W[n][k] with both operands the exact MXFP4 values, fp64.

    Returns (y, A) as gemv does."""
    Aq = dequant(MXFP4, a_codes.shape[0], K, a_codes, a_scales)
    return gemv(MXFP4, N, K, w_codes, Aq, scales=w_scales)
