"""GPU parity of the MXFP4 prefill-chunk path (MX activation quantizer + tcgen05 kind::mxf4 GEMM).

The quantized activations must equal the oracle's bit for bit (codes and UE8M0 scale bytes; the OCP
MX rule scales by a power of two, so both sides take the same single rounding to E2M1).  The GEMM
output must match the fp64 product of the same quantized operands within 2e-6 * sum|a_q * w| (fp32
accumulation in tensor memory).  Against the fp64 product of the unquantized bf16 activations, per
output the triangle bound 2e-6 * sum|a_q * w| + sum|w| * |x - a_q| holds, and over the sampled
outputs the rms of |y - y_exact| / sum|x * w| is that of the oracle's own quantized product plus at
most 2e-6 (the activation quantization is the method's; the kernel adds only its fp32 sums).
"""
import numpy as np
import pytest
import torch

import gemm_dequant_gemv_q8_b200 as q
import oracle
import synth

pytestmark = pytest.mark.gpu
MX = q.QLIN_MXFP4


@pytest.mark.parametrize("M,K", [(1, 256), (64, 5120), (130, 288), (512, 1024)])
def test_act_quant_mx_bit_exact(M, K):
    x = synth.activations(M, K, synth.gen(M + K + 7), dtype=torch.bfloat16)
    codes, scales = q.qlin_act_quant_mx_debug(x.cuda())
    rc, rs = oracle.act_quant_mx(x.float().numpy())
    assert np.array_equal(scales.cpu().numpy(), rs)
    assert np.array_equal(codes.cpu().numpy(), rc)


def test_act_quant_mx_special_rows():
    """A zero row, an outlier, values near the bottom and top of bf16, negative zeros, an Inf."""
    x = torch.zeros(6, 128, dtype=torch.bfloat16)
    x[1, 3] = 1000.0
    x[1, 40:70] = 0.01
    x[2, :] = 1e-38
    x[2, 64:96] = 3e38
    x[3, 17] = -0.0
    x[3, 33] = -0.5
    x[4] = torch.linspace(-7.9, 7.9, 128)
    x[5, 65] = float("inf")
    x[5, 66] = 2.0
    codes, scales = q.qlin_act_quant_mx_debug(x.cuda())
    rc, rs = oracle.act_quant_mx(x.float().numpy())
    assert np.array_equal(scales.cpu().numpy(), rs)
    assert np.array_equal(codes.cpu().numpy(), rc)
    assert rs[5, 2] == 0xFF and rs[0, 0] == 0


def _mx_chunk(M, N, K, seed, rows=None, flags=0):
    codes, scales, _ = synth.mxfp4(N, K, synth.gen(seed))
    packed = q.qlin_pack_weights(MX, N, K, codes.cuda(), scales.cuda(), 1.0, q.QLIN_PACK_MMA)
    assert packed.numel() == q.qlin_packed_bytes(MX, N, K, q.QLIN_PACK_MMA)
    x = synth.activations(M, K, synth.gen(seed + 1), dtype=torch.bfloat16)
    ws = q.workspace(q.qlin_workspace_bytes(q.QLIN_OP_CHUNK, MX, M, N, K))
    y = q.qlin_gemm_chunk(MX, packed, N, K, x.cuda(), flags=flags, ws=ws)
    torch.cuda.synchronize()
    assert q.qlin_ws_status(ws) == 0
    ac, asc = oracle.act_quant_mx(x.float().numpy())
    if rows is None:
        rows = np.arange(N)
    xq = oracle.dequant(MX, M, K, ac, asc)
    yq, Aq = oracle.gemv(MX, N, K, codes.numpy(), xq, scales=scales.numpy(), rows=rows)
    xd = x.double().numpy()
    ye, Ae = oracle.gemv(MX, N, K, codes.numpy(), xd, scales=scales.numpy(), rows=rows)
    _, Ed = oracle.gemv(MX, N, K, codes.numpy(), xd - xq, scales=scales.numpy(), rows=rows)
    return y.cpu().double().numpy()[:, rows], yq, Aq, ye, Ae, Ed


@pytest.mark.parametrize("flags", [0, q.QLIN_FLAG_CTA_PAIRS])
@pytest.mark.parametrize("M,N,K", [(1, 256, 256), (37, 70, 288), (64, 300, 512), (200, 520, 2560),
                                   (513, 1000, 1024)])
def test_mx_chunk_same_quant_parity(M, N, K, flags):
    y, yq, Aq, ye, Ae, Ed = _mx_chunk(M, N, K, 900 + M + N, flags=flags)
    err = np.abs(y - yq)
    bad = err > 2e-6 * Aq + 1e-30
    assert not bad.any(), (int(bad.sum()), float(np.max(err / np.maximum(Aq, 1e-300))))
    # against the unquantized product: the triangle bound per output
    assert (np.abs(y - ye) <= 2e-6 * Aq + Ed + 1e-30).all()


@pytest.mark.parametrize("flags", [0, q.QLIN_FLAG_CTA_PAIRS])
def test_mx_chunk_full_size_sampled(flags):
    """The prefill-chunk workload's shape (K = 5120, N = 17408, M = 512), sampled output rows."""
    M, N, K = 512, 17408, 5120
    rows = np.unique(np.linspace(0, N - 1, 63).astype(np.int64))
    y, yq, Aq, ye, Ae, Ed = _mx_chunk(M, N, K, 5150, rows=rows, flags=flags)
    err = np.abs(y - yq)
    assert (err <= 2e-6 * Aq + 1e-30).all(), float(np.max(err / Aq))
    rel_gpu = np.abs(y - ye) / Ae
    rel_oracle = np.abs(yq - ye) / Ae
    rms_gpu, rms_oracle = np.sqrt(np.mean(rel_gpu ** 2)), np.sqrt(np.mean(rel_oracle ** 2))
    print("MXFP4 chunk vs unquantized x: rms %.3g (oracle's quantized product %.3g), max %.3g" %
          (rms_gpu, rms_oracle, rel_gpu.max()))
    assert rms_gpu <= rms_oracle + 2e-6


def test_mx_chunk_bf16_copy_option():
    """MXFP4 weights also take the bf16-operand path (QLIN_PACK_MMA_BF16 + QLIN_FLAG_BF16_COPY)."""
    M, N, K = 64, 300, 512
    codes, scales, _ = synth.mxfp4(N, K, synth.gen(77))
    packed = q.qlin_pack_weights(MX, N, K, codes.cuda(), scales.cuda(), 1.0, q.QLIN_PACK_MMA_BF16)
    x = synth.activations(M, K, synth.gen(78), dtype=torch.bfloat16)
    y = q.qlin_gemm_chunk(MX, packed, N, K, x.cuda(), flags=q.QLIN_FLAG_BF16_COPY)
    torch.cuda.synchronize()
    ye, Ae = oracle.gemv(MX, N, K, codes.numpy(), x.double().numpy(), scales=scales.numpy())
    assert (np.abs(y.cpu().double().numpy() - ye) <= (2 * K + 1) * 2.0 ** -24 * Ae + 1e-30).all()
