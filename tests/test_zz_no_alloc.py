"""The allocation-free GEMV entry point (qlin_gemv_noalloc), called through the C ABI.

It is for callers that cannot allocate device memory for a workspace (a plugin whose host
application owns all device allocations, or a decode loop that must not call cudaMalloc once it
runs).  Both calls run the same kernel on the same plan as qlin_gemv, so on two calls in a row
(the shared scratch array keeps the first call's contents) the output must equal qlin_gemv's bit
for bit, and it must also meet the GEMV tolerance against the oracle directly.  A shape whose
workspace exceeds the fixed scratch size must be rejected before anything runs.  This file is
collected last and needs no state from the other tests.
"""
import ctypes

import numpy as np
import pytest
import torch

import gemm_dequant_gemv_q8_b200 as q
import oracle
import synth

pytestmark = pytest.mark.gpu


def call_noalloc(fmt, packed, N, K, x, y, flags=0):
    xdt = q.QLIN_BF16 if x.dtype == torch.bfloat16 else q.QLIN_F32
    P = ctypes.c_void_p
    return q.lib().qlin_gemv_noalloc(fmt, P(packed.data_ptr()), N, K, P(x.data_ptr()), xdt, x.shape[0],
                                     x.stride(0), P(y.data_ptr()), y.stride(0), flags,
                                     P(torch.cuda.current_stream().cuda_stream))


def noalloc_status():
    return q.lib().qlin_gemv_noalloc_status(ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


@pytest.mark.parametrize("fmt,N,K,M,flags", [
    (q.QLIN_Q4_0, 2560, 9728, 1, 0),
    (q.QLIN_Q8_0, 1000, 1024, 3, 0),
    (q.QLIN_NVFP4, 2 * 1088, 5120, 4, q.QLIN_EPI_SILU_GATE),
])
def test_noalloc_matches_qlin_gemv_and_oracle_twice(fmt, N, K, M, flags):
    blocks, scales, g = synth.weights(fmt, N, K, synth.gen(N + K + M))
    pf = q.QLIN_PACK_GATE_UP if flags == q.QLIN_EPI_SILU_GATE else q.QLIN_PACK_DEFAULT
    packed = q.qlin_pack_weights(fmt, N, K, blocks.cuda(), None if scales is None else scales.cuda(), g, pf)
    xdt = torch.bfloat16 if fmt == q.QLIN_NVFP4 else torch.float32
    ncols = N // 2 if flags == q.QLIN_EPI_SILU_GATE else N
    rows = np.arange(0, ncols, 7)
    for call in range(2):
        x = synth.activations(M, K, synth.gen(100 * call + N), dtype=xdt).cuda()
        ref = q.qlin_gemv(fmt, packed, N, K, x, flags=flags)
        y = torch.full((M, ncols), float("nan"), device="cuda")
        assert call_noalloc(fmt, packed, N, K, x, y, flags) == 0
        torch.cuda.synchronize()
        assert noalloc_status() == 0
        # same kernel, same plan: identical bits
        assert torch.equal(y, ref), call
        # and directly against the oracle: 2e-6 * sum|w*x| per output (for the SiLU gate, the
        # bound propagated through silu(g)*u, as in the other GEMV tests)
        xs = x.cpu().double().numpy()
        sc = None if scales is None else scales.numpy()
        yd = y[:, rows].double().cpu().numpy()
        if flags == q.QLIN_EPI_SILU_GATE:
            sel = np.concatenate([rows, rows + N // 2])
            gu, A = oracle.gemv(fmt, N, K, blocks.numpy(), xs, scales=sc, g=g, rows=sel)
            href, Ah = oracle.silu_gate(gu, A)
            tol = 2e-6 * Ah + 8 * 2.0 ** -24 * np.abs(href) + 4 * 2.0 ** -126 * (1 + np.abs(gu[:, len(rows):]))
            err = np.abs(yd - href)
        else:
            yref, A = oracle.gemv(fmt, N, K, blocks.numpy(), xs, scales=sc, g=g, rows=rows)
            tol = 2e-6 * A
            err = np.abs(yd - yref)
        assert (err <= tol).all(), (call, float(np.max(err / np.maximum(tol, 1e-300))))


def test_noalloc_rejects_shapes_beyond_its_scratch():
    # N = 262144, K = 256, M = 8 needs a 16 MiB workspace; the fixed scratch is 8 MiB.  Real
    # buffers of the right sizes, so that a regression of the size check gives a wrong status or
    # output, never an access outside an allocation.
    N, K, M = 262144, 256, 8
    need = q.qlin_workspace_bytes(q.QLIN_OP_GEMV, q.QLIN_Q4_0, M, N, K)
    assert need > 8 << 20
    packed = q._alloc_aligned(q.qlin_packed_bytes(q.QLIN_Q4_0, N, K), "cuda")
    packed.zero_()
    x = torch.zeros(M, K, device="cuda")
    y = torch.full((M, N), 7.0, device="cuda")
    assert call_noalloc(q.QLIN_Q4_0, packed, N, K, x, y) == 4  # QLIN_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert bool((y == 7.0).all())  # nothing was enqueued
