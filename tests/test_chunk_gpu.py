"""GPU parity of the NVFP4 prefill-chunk path (activation quantizer + tcgen05 GEMM).

The quantized activations must equal the oracle's bit for bit (codes, scales, a_g: the rule is
stated in fp32 and both sides take each rounding in fp32).  The GEMM output must match the fp64
product of the same quantized operands within 2e-6 * sum|a_q * w| (fp32 accumulation).  Against
the fp64 product of the unquantized bf16 activations two checks hold at the configured K = 5120:
per output, the triangle-inequality bound 2e-6 * sum|a_q * w| + sum|w| * |x - a_q| (always true if
the kernel multiplies the quantized operands it was given), and over all sampled outputs an rms of
|y - y_exact| / sum|x * w| below 5e-3 (the activation quantization alone gives about 2.5e-3 for
N(0,1) activations; single outputs reach 1e-2, so a per-output 1e-2 bound is not a valid check).
"""
import numpy as np
import pytest
import torch

import gemm_dequant_gemv_q8_b200 as q
import oracle
import synth

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("M,K", [(1, 256), (64, 5120), (130, 272), (512, 1024)])
def test_act_quant_bit_exact(M, K):
    x = synth.activations(M, K, synth.gen(M + K), dtype=torch.bfloat16)
    codes, scales, ag = q.qlin_act_quant_debug(x.cuda())
    rc, rs, rag = oracle.act_quant(x.float().numpy())
    assert float(ag.item()) == rag
    assert np.array_equal(scales.cpu().numpy(), rs)
    assert np.array_equal(codes.cpu().numpy(), rc)


def test_act_quant_zero_and_outlier_rows():
    x = torch.zeros(4, 64, dtype=torch.bfloat16)
    x[1, 3] = 1000.0
    x[2, :] = 1e-3
    x[3, 17] = -0.5
    codes, scales, ag = q.qlin_act_quant_debug(x.cuda())
    rc, rs, rag = oracle.act_quant(x.float().numpy())
    assert float(ag.item()) == rag
    assert np.array_equal(scales.cpu().numpy(), rs) and np.array_equal(codes.cpu().numpy(), rc)


def _chunk(M, N, K, seed, rows=None, flags=0):
    codes, scales, g = synth.nvfp4(N, K, synth.gen(seed))
    packed = q.qlin_pack_weights(q.QLIN_NVFP4, N, K, codes.cuda(), scales.cuda(), g, q.QLIN_PACK_MMA)
    x = synth.activations(M, K, synth.gen(seed + 1), dtype=torch.bfloat16)
    y = q.qlin_gemm_chunk(q.QLIN_NVFP4, packed, N, K, x.cuda(), flags=flags)
    torch.cuda.synchronize()
    ac, asc, ag = oracle.act_quant(x.float().numpy())
    if rows is None:
        rows = np.arange(N)
    xq = oracle.dequant(q.QLIN_NVFP4, M, K, ac, asc, ag)
    yq, Aq = oracle.gemv(q.QLIN_NVFP4, N, K, codes.numpy(), xq, scales=scales.numpy(), g=g, rows=rows)
    xd = x.double().numpy()
    ye, Ae = oracle.gemv(q.QLIN_NVFP4, N, K, codes.numpy(), xd, scales=scales.numpy(), g=g, rows=rows)
    _, Ed = oracle.gemv(q.QLIN_NVFP4, N, K, codes.numpy(), xd - xq, scales=scales.numpy(), g=g, rows=rows)
    return y.cpu().double().numpy()[:, rows], yq, Aq, ye, Ae, Ed


@pytest.mark.parametrize("flags", [0, q.QLIN_FLAG_CTA_PAIRS])
@pytest.mark.parametrize("M,N,K", [(128, 256, 256), (70, 300, 272), (200, 512, 1024), (64, 264, 768)])
def test_chunk_gemm_small(M, N, K, flags):
    # Few output tiles (all but the first shape): each tile's k-groups run as two halves that add
    # into y; K = 768 splits its three k-groups 2 + 1, K = 272 ends in a partial k-group.
    y, yq, Aq, _, _, _ = _chunk(M, N, K, 10 * M + N, flags=flags)
    err = np.abs(y - yq)
    assert (err <= 2e-6 * Aq).all(), float(np.max(err / np.maximum(Aq, 1e-300)))


@pytest.mark.parametrize("M,flags", [(64, 0), (512, 0), (512, q.QLIN_FLAG_CTA_PAIRS)])
def test_chunk_gemm_27b_shape_sampled(M, flags):
    N, K = 17408, 5120
    rows = np.unique(np.concatenate([[0, 255, 256, N - 1], np.random.default_rng(M).integers(0, N, 60)]))
    y, yq, Aq, ye, Ae, Ed = _chunk(M, N, K, 77, rows, flags=flags)
    assert (np.abs(y - yq) <= 2e-6 * Aq).all(), float(np.max(np.abs(y - yq) / np.maximum(Aq, 1e-300)))
    assert (np.abs(y - ye) <= 2e-6 * Aq + Ed + 1e-12 * Ae).all()
    rel = np.abs(y - ye) / Ae
    assert float(np.sqrt(np.mean(rel * rel))) < 5e-3, float(np.sqrt(np.mean(rel * rel)))


def test_chunk_gemm_status_clean_and_deterministic():
    N, K, M = 512, 512, 128
    codes, scales, g = synth.nvfp4(N, K, synth.gen(5))
    packed = q.qlin_pack_weights(q.QLIN_NVFP4, N, K, codes.cuda(), scales.cuda(), g, q.QLIN_PACK_MMA)
    x = synth.activations(M, K, synth.gen(6), dtype=torch.bfloat16).cuda()
    ws = q.workspace(q.qlin_workspace_bytes(q.QLIN_OP_CHUNK, q.QLIN_NVFP4, M, N, K))
    y1 = q.qlin_gemm_chunk(q.QLIN_NVFP4, packed, N, K, x, ws=ws).clone()
    y2 = q.qlin_gemm_chunk(q.QLIN_NVFP4, packed, N, K, x, ws=ws)
    assert torch.equal(y1, y2)
    assert q.qlin_ws_status(ws) == 0


@pytest.mark.parametrize("flags", [0, q.QLIN_FLAG_CTA_PAIRS])
@pytest.mark.parametrize("xpad,ypad", [(0, 4), (4, 3), (8, 0)])
def test_chunk_gemm_strided_operands(xpad, ypad, flags):
    """Row strides other than K and N: x rows ldx = K + xpad apart (xpad = 4: 8-byte-aligned rows,
    the quantizer's scalar loads), y rows ldy = N + ypad apart (ypad = 3: rows not 16-byte aligned,
    the epilogue's plain stores; otherwise the tensor-store epilogue with a pitch)."""
    M, N, K = 170, 300, 272
    codes, scales, g = synth.nvfp4(N, K, synth.gen(31))
    packed = q.qlin_pack_weights(q.QLIN_NVFP4, N, K, codes.cuda(), scales.cuda(), g, q.QLIN_PACK_MMA)
    x = synth.activations(M, K, synth.gen(32), dtype=torch.bfloat16)
    xbig = torch.zeros(M, K + xpad, dtype=torch.bfloat16)
    xbig[:, :K] = x
    ybig = torch.full((M, N + ypad), float("nan"), device="cuda")
    y = ybig[:, :N]
    q.qlin_gemm_chunk(q.QLIN_NVFP4, packed, N, K, xbig.cuda()[:, :K], y=y, flags=flags)
    torch.cuda.synchronize()
    ac, asc, ag = oracle.act_quant(x.float().numpy())
    xq = oracle.dequant(q.QLIN_NVFP4, M, K, ac, asc, ag)
    yq, Aq = oracle.gemv(q.QLIN_NVFP4, N, K, codes.numpy(), xq, scales=scales.numpy(), g=g)
    yy = y.cpu().double().numpy()
    assert (np.abs(yy - yq) <= 2e-6 * Aq).all(), float(np.nanmax(np.abs(yy - yq) / np.maximum(Aq, 1e-300)))
    if ypad:  # the padding columns are untouched
        assert torch.isnan(ybig[:, N:]).all()


@pytest.mark.parametrize("flags", [0, q.QLIN_FLAG_CTA_PAIRS])
@pytest.mark.parametrize("M", [1, 33, 127, 129, 257, 300])
def test_chunk_gemm_ragged_rows(M, flags):
    """Row counts that leave part of a 128-row tile (or of a 256-row tile of a CTA pair), and of a
    warp's 32 rows, empty; M = 300 leaves one CTA of the second pair without any row."""
    y, yq, Aq, _, _, _ = _chunk(M, 288, 512, 500 + M, flags=flags)
    assert (np.abs(y - yq) <= 2e-6 * Aq).all(), float(np.max(np.abs(y - yq) / np.maximum(Aq, 1e-300)))


def test_chunk_gemm_alternating_shapes_one_workspace():
    """The workspace's barrier counters return to zero after every call: calls of different M
    (different grid sizes) on one workspace all succeed with a clean status."""
    N, K = 512, 512
    codes, scales, g = synth.nvfp4(N, K, synth.gen(41))
    packed = q.qlin_pack_weights(q.QLIN_NVFP4, N, K, codes.cuda(), scales.cuda(), g, q.QLIN_PACK_MMA)
    ws = q.workspace(q.qlin_workspace_bytes(q.QLIN_OP_CHUNK, q.QLIN_NVFP4, 512, N, K))
    for M, fl in ((512, 0), (3, 0), (256, q.QLIN_FLAG_CTA_PAIRS), (64, 0), (512, q.QLIN_FLAG_CTA_PAIRS), (300, 0)):
        x = synth.activations(M, K, synth.gen(42 + M), dtype=torch.bfloat16)
        y = q.qlin_gemm_chunk(q.QLIN_NVFP4, packed, N, K, x.cuda(), ws=ws, flags=fl)
        torch.cuda.synchronize()
        assert q.qlin_ws_status(ws) == 0
        ac, asc, ag = oracle.act_quant(x.float().numpy())
        xq = oracle.dequant(q.QLIN_NVFP4, M, K, ac, asc, ag)
        yq, Aq = oracle.gemv(q.QLIN_NVFP4, N, K, codes.numpy(), xq, scales=scales.numpy(), g=g)
        assert (np.abs(y.cpu().double().numpy() - yq) <= 2e-6 * Aq).all()


def test_chunk_gemm_back_to_back_pdl_one_workspace():
    """Calls enqueued back to back with QLIN_FLAG_PDL on one workspace (no host synchronisation
    between them): each may start while the previous drains, yet every result and the status
    stay as if they ran one after another."""
    N, K = 1024, 768
    codes, scales, g = synth.nvfp4(N, K, synth.gen(51))
    packed = q.qlin_pack_weights(q.QLIN_NVFP4, N, K, codes.cuda(), scales.cuda(), g, q.QLIN_PACK_MMA)
    ws = q.workspace(q.qlin_workspace_bytes(q.QLIN_OP_CHUNK, q.QLIN_NVFP4, 512, N, K))
    runs = []
    for M, fl in ((512, 0), (64, 0), (300, q.QLIN_FLAG_CTA_PAIRS), (7, 0), (512, 0), (129, 0)):
        x = synth.activations(M, K, synth.gen(52 + M), dtype=torch.bfloat16)
        y = q.qlin_gemm_chunk(q.QLIN_NVFP4, packed, N, K, x.cuda(), ws=ws, flags=fl | q.QLIN_FLAG_PDL)
        runs.append((x, y))
    torch.cuda.synchronize()
    assert q.qlin_ws_status(ws) == 0
    for x, y in runs:
        ac, asc, ag = oracle.act_quant(x.float().numpy())
        xq = oracle.dequant(q.QLIN_NVFP4, x.shape[0], K, ac, asc, ag)
        yq, Aq = oracle.gemv(q.QLIN_NVFP4, N, K, codes.numpy(), xq, scales=scales.numpy(), g=g)
        assert (np.abs(y.cpu().double().numpy() - yq) <= 2e-6 * Aq).all()
