"""Host-side checks of the C ABI (no GPU needed): the library loads, exports every entry point
declared in include/qlin.h, and rejects bad arguments before launching anything."""
import ctypes
import os
import re

import pytest
import torch

import gemm_dequant_gemv_q8_b200 as q
from gemm_dequant_gemv_q8_b200 import build as qbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    qbuild.build()
    return q.lib()


# The argument-check tests below hand the library made-up device addresses and expect every call
# to be rejected on the host. Where a device is visible, a regression in a check would launch a
# kernel on unmapped memory, so they run only on machines without one.
made_up_addresses = pytest.mark.skipif(torch.cuda.is_available(),
                                       reason="made-up device addresses: run only where no kernel can launch")


def declared_functions():
    names = []
    for h in os.listdir(os.path.join(ROOT, "include")):
        if h.endswith(".h"):
            txt = open(os.path.join(ROOT, "include", h)).read()
            txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
            names += re.findall(r"\b(qlin_\w+)\s*\(", txt)
    return sorted(set(names))


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert "qlin_gemv" in names and "qlin_pack_weights" in names
    for n in names:
        assert hasattr(lib, n), n
    assert set(q.SIGNATURES) <= set(names)


def test_status_strings(lib):
    for code, name in q.STATUS.items():
        assert q.qlin_status_string(code) == name


def test_packed_bytes_sizes(lib):
    # Q4_0 / NVFP4: 0.5625 B per weight, Q8_0: 1.0625, plus a 256-byte header; N->32, K->256 pad.
    assert q.qlin_packed_bytes(q.QLIN_Q4_0, 4096, 2560) == 256 + 4096 * 2560 * 9 // 16
    assert q.qlin_packed_bytes(q.QLIN_Q8_0, 1024, 256) == 256 + 1024 * 256 * 17 // 16
    assert q.qlin_packed_bytes(q.QLIN_NVFP4, 32, 16) == 256 + 4608
    assert q.qlin_packed_bytes(q.QLIN_Q4_0, 33, 288) == 256 + 2 * 2 * 4608
    assert q.qlin_packed_bytes(q.QLIN_Q4_0, 64, 256, q.QLIN_PACK_GATE_UP) == 256 + 2 * 4608
    assert q.qlin_packed_bytes(q.QLIN_Q4_0, 64, 100) == 0  # K % 32
    assert q.qlin_packed_bytes(q.QLIN_NVFP4, 64, 40) == 0  # K % 16
    # MXFP4: codes as NVFP4, one scale byte per 32 values: 4096 + 256 bytes per 32 x 256 unit
    assert q.qlin_packed_bytes(q.QLIN_MXFP4, 4096, 2560) == 256 + 4096 * 2560 * 17 // 32
    assert q.qlin_packed_bytes(q.QLIN_MXFP4, 64, 272) == 0  # K % 32
    # QLIN_PACK_MMA for the GGUF / MXFP4 formats: the bf16 copy in blocks of 256 rows x 64 values,
    # K rounded up to 64 and N to 256
    assert q.qlin_packed_bytes(q.QLIN_Q4_0, 100, 96, q.QLIN_PACK_MMA) == 256 + 256 * 128 * 2
    assert q.qlin_packed_bytes(q.QLIN_Q6_K, 64, 512, q.QLIN_PACK_MMA) == 256 + 256 * 512 * 2
    assert q.qlin_packed_bytes(q.QLIN_Q4_0, 17408, 5120, q.QLIN_PACK_MMA) == 256 + 17408 * 5120 * 2
    # Q4_K: 4096 B of codes + 512 B of sub-block scale/min slots + 128 B of per-row d/dmin per unit
    assert q.qlin_packed_bytes(q.QLIN_Q4_K, 4096, 2560) == 256 + (4096 // 32) * (2560 // 256) * 4736
    assert q.qlin_packed_bytes(q.QLIN_Q4_K, 33, 512) == 256 + 2 * 2 * 4736
    assert q.qlin_packed_bytes(q.QLIN_Q4_K, 64, 288) == 0  # K % 256
    # Q6_K: two 4096 B byte planes of 6-bit codes + 512 B of int8 scale pairs + 128 B of per-row d
    assert q.qlin_packed_bytes(q.QLIN_Q6_K, 4096, 2560) == 256 + (4096 // 32) * (2560 // 256) * 8832
    assert q.qlin_packed_bytes(q.QLIN_Q6_K, 64, 288) == 0  # K % 256
    assert q.qlin_packed_bytes(7, 64, 256) == 0
    assert q.qlin_packed_bytes(q.QLIN_Q4_0, 63, 256, q.QLIN_PACK_GATE_UP) == 0  # odd N


def _gemv(lib, fmt=2, packed=0x100000, N=64, K=256, x=0x200000, xdt=0, M=1, ldx=256, y=0x300000,
          ldy=64, flags=0, ws=0x400000, ws_bytes=1 << 30):
    P = ctypes.c_void_p
    return lib.qlin_gemv(fmt, P(packed), N, K, P(x), xdt, M, ldx, P(y), ldy, flags, P(ws), ws_bytes, None)


@made_up_addresses
def test_gemv_argument_checks_return_before_launch(lib):
    E_ARG, E_ALIGN, E_WS = 1, 3, 4
    assert _gemv(lib, fmt=9) == E_ARG
    assert _gemv(lib, M=0) == E_ARG and _gemv(lib, M=9) == E_ARG
    assert _gemv(lib, K=100) == E_ARG
    assert _gemv(lib, xdt=5) == E_ARG
    assert _gemv(lib, flags=7) == E_ARG
    assert _gemv(lib, flags=q.QLIN_EPI_SILU_GATE, N=63) == E_ARG
    assert _gemv(lib, packed=0) == E_ARG and _gemv(lib, x=0) == E_ARG and _gemv(lib, y=0) == E_ARG
    assert _gemv(lib, ldx=128) == E_ARG and _gemv(lib, ldy=10) == E_ARG
    assert _gemv(lib, x=0x200004) == E_ALIGN
    assert _gemv(lib, packed=0x100010) == E_ALIGN
    assert _gemv(lib, ldx=258) == E_ALIGN
    assert _gemv(lib, ws=0) == E_WS and _gemv(lib, ws_bytes=16) == E_WS
    assert _gemv(lib, ws=0x400010) == E_ALIGN


@made_up_addresses
def test_pack_argument_checks(lib):
    P = ctypes.c_void_p
    f = lib.qlin_pack_weights
    assert f(2, 64, 256, P(0), None, 1.0, 0, P(0x1000), 1 << 30, None) == 1
    assert f(3, 64, 256, P(0x1000), None, 1.0, 0, P(0x10000), 1 << 30, None) == 1  # NVFP4 needs scales
    assert f(4, 64, 256, P(0x1000), None, 1.0, 0, P(0x10000), 1 << 30, None) == 1  # MXFP4 needs scales
    assert f(2, 64, 256, P(0x1000), None, 1.0, 3, P(0x10000), 1 << 30, None) == 2  # gate_up MMA form: FP4 only
    assert f(4, 63, 256, P(0x1000), P(0x2000), 1.0, 3, P(0x10000), 1 << 30, None) == 1  # ... with N even
    assert f(2, 64, 256, P(0x1000), None, 1.0, 2, P(0x10000), 256 + 64 * 256, None) == 1  # bf16 copy needs 2 B/w
    assert f(2, 64, 256, P(0x1000), None, 1.0, 0, P(0x10010), 1 << 30, None) == 3
    assert f(2, 64, 256, P(0x1000), None, 1.0, 0, P(0x10000), 10, None) == 1
    assert f(2, 64, 256, P(0x1000), None, 1.0, 8, P(0x10000), 1 << 30, None) == 1


def test_workspace_bytes_cover_partials(lib):
    b1 = q.qlin_workspace_bytes(q.QLIN_OP_GEMV, q.QLIN_Q4_0, 1, 4096, 2560)
    b8 = q.qlin_workspace_bytes(q.QLIN_OP_GEMV, q.QLIN_Q4_0, 8, 4096, 2560)
    assert 0 < b1 < b8
    assert q.qlin_workspace_bytes(q.QLIN_OP_GEMV, q.QLIN_Q4_0, 0, 4096, 2560) == 0


def _chain_op(packed=0x100000, N=64, K=256, x=0x200000, ldx=256, y=0x300000, ldy=64, epi=0, wait_for=-1):
    return q.GemvOp(packed, N, K, x, ldx, y, ldy, epi, wait_for)


@made_up_addresses
def test_chain_argument_checks_return_before_launch(lib):
    E_ARG, E_ALIGN, E_WS = 1, 3, 4
    P = ctypes.c_void_p

    def call(ops, n=None, fmt=2, xdt=0, M=1, flags=0, ws=0x400000, ws_bytes=1 << 30):
        arr = (q.GemvOp * max(len(ops), 1))(*ops)
        return lib.qlin_gemv_chain(fmt, xdt, M, ctypes.cast(arr, P), len(ops) if n is None else n, flags,
                                   P(ws), ws_bytes, None)

    ok = _chain_op()
    assert call([ok], n=0) == E_ARG and call([ok], n=lib.qlin_chain_max_ops() + 1) == E_ARG
    assert call([ok], M=9) == E_ARG and call([ok], fmt=7) == E_ARG and call([ok], xdt=3) == E_ARG
    assert call([ok], flags=1) == E_ARG
    assert call([ok, _chain_op(wait_for=1)]) == E_ARG   # must name an EARLIER op
    assert call([ok, _chain_op(wait_for=-2)]) == E_ARG
    assert call([ok, _chain_op(K=100)]) == E_ARG
    assert call([ok, _chain_op(epi=1, N=63)]) == E_ARG
    assert call([ok, _chain_op(ldy=10)]) == E_ARG
    assert call([ok, _chain_op(packed=0x100010)]) == E_ALIGN
    assert call([ok, _chain_op(x=0x200008)]) == E_ALIGN
    assert call([ok], ws=0) == E_WS and call([ok], ws_bytes=64) == E_WS
    assert call([ok], ws=0x400010) == E_ALIGN


def test_chain_workspace_bytes(lib):
    ops = [_chain_op(), _chain_op(N=2 * 9728, K=2560, epi=1, ldy=9728, ldx=2560),
           _chain_op(N=2560, K=9728, ldx=9728, ldy=2560, wait_for=1)]
    b1 = q.qlin_chain_workspace_bytes(q.QLIN_Q4_0, 1, ops)
    b8 = q.qlin_chain_workspace_bytes(q.QLIN_Q4_0, 8, ops)
    assert 256 < b1 < b8 and b1 % 256 == 0
    assert q.qlin_chain_workspace_bytes(q.QLIN_Q4_0, 1, [_chain_op(wait_for=0)]) == 0


@made_up_addresses
def test_moe_rejects_oversized_hidden_before_launch(lib):
    P = ctypes.c_void_p
    st = lib.qlin_moe_experts(q.QLIN_MXFP4, P(0x100000), P(0x200000), 32, 32768 + 256, 1792, 4, P(0x300000),
                              P(0x400000), P(0x500000), P(0x600000), 1, 1, P(0x700000), None, 0,
                              P(0x800000), 1 << 30, None)
    assert st == 2  # QLIN_ERR_UNSUPPORTED: down tiles per expert are tracked for H <= 32768


@made_up_addresses
def test_moe_prefill_argument_checks_return_before_launch(lib):
    """Every bad argument of qlin_moe_prefill is reported before anything is enqueued (the device
    pointers below are never dereferenced: the checks run on the host)."""
    P = ctypes.c_void_p
    N4, MX = q.QLIN_NVFP4, q.QLIN_MXFP4
    ok = dict(fmt=N4, gu=P(0x100000), dn=P(0x200000), E=32, H=2048, I=1792, k=4, logits=P(0x300000),
              ids=P(0x400000), w=P(0x500000), x=P(0x600000), M=64, y=P(0x700000), h=None, flags=0,
              ws=P(0x800000), wsb=1 << 34)

    def call(**kw):
        a = dict(ok, **kw)
        return lib.qlin_moe_prefill(a["fmt"], a["gu"], a["dn"], a["E"], a["H"], a["I"], a["k"], a["logits"], a["ids"],
                                    a["w"], a["x"], a["M"], a["y"], a["h"], a["flags"], a["ws"], a["wsb"], None)

    assert call(fmt=q.QLIN_Q4_0) == 2       # GGUF experts: not on this path
    assert call(fmt=q.QLIN_Q8_0) == 2
    assert call(fmt=99) == 1                # unknown format
    assert call(E=0) == 1 and call(E=257) == 1
    assert call(k=0) == 1 and call(k=9) == 1 and call(E=2, k=3) == 1
    assert call(H=2047) == 1 and call(I=1800) == 1 and call(H=16) == 1
    assert call(M=0) == 1
    assert call(flags=1) == 1
    assert call(gu=None) == 1 and call(y=None) == 1 and call(ids=None) == 1
    assert call(x=P(0x600008)) == 3         # x not 16-byte aligned
    assert call(gu=P(0x100010)) == 3        # packed buffers 256-byte aligned
    assert call(wsb=16) == 4 and call(ws=None) == 4
    assert call(fmt=MX, wsb=16) == 4


def test_moe_prefill_workspace_bytes(lib):
    N4 = q.QLIN_NVFP4
    assert q.qlin_workspace_bytes(q.QLIN_OP_MOE_PREFILL, q.QLIN_Q4_0, 64, 2048, 1792, 32, 4) == 0
    assert q.qlin_workspace_bytes(q.QLIN_OP_MOE_PREFILL, N4, 64, 2048, 1800, 32, 4) == 0
    sizes = [q.qlin_workspace_bytes(q.QLIN_OP_MOE_PREFILL, N4, M, 2048, 1792, 32, 4) for M in (1, 64, 512, 4096)]
    assert all(s > 0 for s in sizes) and sizes == sorted(sizes)
    # the same for MXFP4 experts (the operand units keep the NVFP4 size)
    assert q.qlin_workspace_bytes(q.QLIN_OP_MOE_PREFILL, q.QLIN_MXFP4, 512, 2048, 1792, 32, 4) == sizes[2]


@made_up_addresses
def test_probe_fp4_mma_argument_checks(lib):
    P = ctypes.c_void_p
    ctas = ctypes.c_int(-1)

    def call(iters=64, cycles=0x100000, max_ctas=1024, status=0x200000):
        return lib.qlin_probe_fp4_mma(iters, P(cycles), max_ctas, P(status), ctypes.byref(ctas), None)

    assert call(iters=0) == 1 and call(iters=(1 << 20) + 1) == 1
    assert call(max_ctas=0) == 1
    assert call(cycles=0) == 1 and call(status=0) == 1
    assert call(cycles=0x100004) == 3 and call(status=0x200002) == 3
