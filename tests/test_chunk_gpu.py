"""GPU parity of the NVFP4 prefill-chunk path (activation quantizer + tcgen05 GEMM).

The quantized activations must equal the oracle's bit for bit (codes, scales, a_g: the rule is
stated in fp32 and both sides take each rounding in fp32).  The GEMM output must match the fp64
product of the same quantized operands within 2e-6 * sum|a_q * w| (fp32 accumulation).  Against
the fp64 product of the unquantized bf16 activations the bound is 1e-2 * sum|x * w| (the
bf16-operand tolerance of the chunk path) at the configured K = 5120: the activation quantization
error relative to sum|x * w| shrinks like 1/sqrt(K) (about 0.15% rms at K = 5120, about 0.6% at
K = 256, where single outputs exceed 1%), so that check is made at K = 5120 only.
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


def _chunk(M, N, K, seed, rows=None):
    codes, scales, g = synth.nvfp4(N, K, synth.gen(seed))
    packed = q.qlin_pack_weights(q.QLIN_NVFP4, N, K, codes.cuda(), scales.cuda(), g, q.QLIN_PACK_MMA)
    x = synth.activations(M, K, synth.gen(seed + 1), dtype=torch.bfloat16)
    y = q.qlin_gemm_chunk(q.QLIN_NVFP4, packed, N, K, x.cuda())
    torch.cuda.synchronize()
    ac, asc, ag = oracle.act_quant(x.float().numpy())
    if rows is None:
        rows = np.arange(N)
    yq, Aq = oracle.gemv(q.QLIN_NVFP4, N, K, codes.numpy(), oracle.dequant(q.QLIN_NVFP4, M, K, ac, asc, ag),
                         scales=scales.numpy(), g=g, rows=rows)
    ye, Ae = oracle.gemv(q.QLIN_NVFP4, N, K, codes.numpy(), x.double().numpy(), scales=scales.numpy(), g=g, rows=rows)
    return y.cpu().double().numpy()[:, rows], yq, Aq, ye, Ae


@pytest.mark.parametrize("M,N,K", [(128, 256, 256), (70, 300, 272), (200, 512, 1024)])
def test_chunk_gemm_small(M, N, K):
    y, yq, Aq, ye, Ae = _chunk(M, N, K, 10 * M + N)
    err = np.abs(y - yq)
    assert (err <= 2e-6 * Aq).all(), float(np.max(err / np.maximum(Aq, 1e-300)))


@pytest.mark.parametrize("M", [64, 512])
def test_chunk_gemm_27b_shape_sampled(M):
    N, K = 17408, 5120
    rows = np.unique(np.concatenate([[0, 255, 256, N - 1], np.random.default_rng(M).integers(0, N, 60)]))
    y, yq, Aq, ye, Ae = _chunk(M, N, K, 77, rows)
    assert (np.abs(y - yq) <= 2e-6 * Aq).all(), float(np.max(np.abs(y - yq) / np.maximum(Aq, 1e-300)))
    assert (np.abs(y - ye) <= 1e-2 * Ae).all()


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
