"""GPU parity of the dense GEMV path against the fp64 oracle (element by element).

Bars: dequantized weights bit-exact (sign included); y within 2e-6 * sum_k |w*x| of the oracle
(fp32 products and sums); the SiLU-gate epilogue within the first-order propagation of that
bound plus a few fp32 roundings of the epilogue itself.
"""
import numpy as np
import pytest
import torch

import gemm_dequant_gemv_q8_b200 as q
import oracle
import synth

pytestmark = pytest.mark.gpu
FMTS = [q.QLIN_Q8_0, q.QLIN_Q4_0, q.QLIN_NVFP4, q.QLIN_MXFP4, q.QLIN_Q4_K, q.QLIN_Q6_K]
TOL = 2e-6


def k_ok(fmt, K):
    """K-quant rows are whole 256-value super-blocks: skip shapes they cannot hold."""
    if fmt in (q.QLIN_Q4_K, q.QLIN_Q6_K) and K % 256:
        pytest.skip("K-quants need K % 256 == 0")


def make(fmt, N, K, seed, pack_flags=q.QLIN_PACK_DEFAULT):
    blocks, scales, g = synth.weights(fmt, N, K, synth.gen(seed))
    packed = q.qlin_pack_weights(fmt, N, K, blocks.cuda(), None if scales is None else scales.cuda(),
                                 g, pack_flags)
    return blocks.numpy(), None if scales is None else scales.numpy(), g, packed


def silu_tol(href, Ah, u):
    """Tolerance of the fp32 SiLU-gate epilogue: the propagated GEMV bound, a few fp32 roundings
    of the epilogue (expf, add, divide, two products), and fp32's underflow floor (no normal
    numbers below 2^-126: silu(g) for g below about -87 is not representable)."""
    return TOL * Ah + 8 * 2.0 ** -24 * np.abs(href) + 4 * 2.0 ** -126 * (1 + np.abs(u))


def check_y(y, yref, A, tol=TOL):
    y = y.double().cpu().numpy()
    err = np.abs(y - yref)
    bad = err > tol * A
    assert not bad.any(), f"{bad.sum()} of {bad.size} outside tol; worst ratio {np.max(err / np.maximum(A, 1e-300)):.3g}"


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("N,K", [(32, 256), (100, 288), (257, 2560), (64, 1024)])
def test_dequant_bit_exact(fmt, N, K):
    k_ok(fmt, K)
    blocks, scales, g, packed = make(fmt, N, K, 100 + N)
    w = q.qlin_dequant_debug(fmt, packed, N, K).cpu().numpy()
    ref = oracle.dequant_f32(fmt, N, K, blocks, scales, g)
    assert np.array_equal(w.view(np.uint32), ref.view(np.uint32))


def test_dequant_mxfp4_special_scale_bytes():
    """UE8M0 bytes at the ends of the range: 0 (2^-127, subnormal products), 1, 126..128, 254
    (6 * 2^127 overflows fp32 to Inf on both sides) and 255 (NaN).  Non-NaN weights bit-exact,
    NaN exactly where the oracle has NaN."""
    N, K = 32, 512
    codes, _, _ = synth.weights(q.QLIN_MXFP4, N, K, synth.gen(8))
    special = torch.tensor([0, 1, 126, 127, 128, 254, 255, 130], dtype=torch.uint8)
    scales = special.repeat(N * K // 32 // 8 + 1)[: N * K // 32].reshape(N, K // 32).contiguous()
    packed = q.qlin_pack_weights(q.QLIN_MXFP4, N, K, codes.cuda(), scales.cuda())
    w = q.qlin_dequant_debug(q.QLIN_MXFP4, packed, N, K).cpu().numpy()
    ref = oracle.dequant_f32(q.QLIN_MXFP4, N, K, codes.numpy(), scales.numpy())
    nan = np.isnan(ref)
    assert nan.any() and np.isinf(ref).any()
    assert np.array_equal(np.isnan(w), nan)
    assert np.array_equal(w[~nan].view(np.uint32), ref[~nan].view(np.uint32))


def test_dequant_nvfp4_k_multiple_of_16_only():
    N, K = 40, 272  # K % 32 == 16: the last part is half padding
    blocks, scales, g, packed = make(q.QLIN_NVFP4, N, K, 7)
    w = q.qlin_dequant_debug(q.QLIN_NVFP4, packed, N, K).cpu().numpy()
    assert np.array_equal(w.view(np.uint32), oracle.dequant_f32(q.QLIN_NVFP4, N, K, blocks, scales, g).view(np.uint32))


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("M", [1, 2, 3, 4, 8])
@pytest.mark.parametrize("xdt", [torch.float32, torch.bfloat16])
def test_gemv_parity(fmt, M, xdt):
    N, K = 200, 1280  # several tiles, a ragged last tile, 5 k-groups
    blocks, scales, g, packed = make(fmt, N, K, 11 + M)
    x = synth.activations(M, K, synth.gen(50 + M), dtype=xdt)
    y = q.qlin_gemv(fmt, packed, N, K, x.cuda())
    yref, A = oracle.gemv(fmt, N, K, blocks, x.double().numpy(), scales=scales, g=g)
    check_y(y, yref, A)


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("N,K,M", [(1, 32, 1), (31, 96, 2), (33, 544, 5), (4096, 2560, 1), (1024, 9728, 1),
                                   (2560, 17408, 4)])
def test_gemv_shapes(fmt, N, K, M):
    k_ok(fmt, K)
    blocks, scales, g, packed = make(fmt, N, K, N + K)
    xdt = torch.bfloat16 if fmt == q.QLIN_NVFP4 else torch.float32
    x = synth.activations(M, K, synth.gen(K), dtype=xdt)
    y = q.qlin_gemv(fmt, packed, N, K, x.cuda())
    rows = np.unique(np.linspace(0, N - 1, min(N, 97)).astype(np.int64))
    yref, A = oracle.gemv(fmt, N, K, blocks, x.double().numpy(), scales=scales, g=g, rows=rows)
    check_y(y[:, rows], yref, A)


def test_gemv_nvfp4_ragged_k16():
    N, K, M = 70, 272, 3
    blocks, scales, g, packed = make(q.QLIN_NVFP4, N, K, 3)
    x = synth.activations(M, K, synth.gen(4), dtype=torch.bfloat16)
    y = q.qlin_gemv(q.QLIN_NVFP4, packed, N, K, x.cuda())
    yref, A = oracle.gemv(q.QLIN_NVFP4, N, K, blocks, x.double().numpy(), scales=scales, g=g)
    check_y(y, yref, A)


@pytest.mark.parametrize("fmt", FMTS)
def test_one_hot_x_gives_dequantized_column(fmt):
    N, K = 96, 768
    blocks, scales, g, packed = make(fmt, N, K, 21)
    W = oracle.dequant_f32(fmt, N, K, blocks, scales, g)
    ks = [0, 31, 32, 255, 256, 767]
    x = torch.zeros(len(ks), K)
    for i, k in enumerate(ks):
        x[i, k] = 1.0
    y = q.qlin_gemv(fmt, packed, N, K, x.cuda()).cpu().numpy()
    for i, k in enumerate(ks):
        assert np.array_equal(y[i], W[:, k]), k  # by value: -0 and +0 compare equal


def test_dequant_q4k_extreme_fields():
    """Q4_K super-blocks with the largest and smallest fields: 6-bit scales and mins of 0 and 63,
    d / dmin of 0, the fp16 maximum 65504 and the smallest subnormal 2^-24, every code; fp32 of
    d*scale*code - dmin*min rounded once, bit for bit (both products are exact in fp32)."""
    N, K = 48, 512
    blocks, _, _ = synth.weights(q.QLIN_Q4_K, N, K, synth.gen(9))
    b = blocks.clone().view(N, K // 256, 144)
    fp16 = torch.tensor([0.0, 65504.0, 2.0 ** -24, 1.0], dtype=torch.float16).view(torch.uint8).view(4, 2)
    for n in range(N):
        b[n, :, 0:2] = fp16[n % 4]
        b[n, :, 2:4] = fp16[(n // 4) % 4]
        if n % 3 == 0:
            b[n, :, 4:16] = 0xFF  # every scale and min 63
        elif n % 3 == 1:
            b[n, :, 4:16] = 0
    blocks = b.reshape(N, -1).contiguous()
    packed = q.qlin_pack_weights(q.QLIN_Q4_K, N, K, blocks.cuda())
    w = q.qlin_dequant_debug(q.QLIN_Q4_K, packed, N, K).cpu().numpy()
    ref = oracle.dequant_f32(q.QLIN_Q4_K, N, K, blocks.numpy())
    assert np.array_equal(w.view(np.uint32), ref.view(np.uint32))


def test_dequant_q6k_extreme_fields():
    """Q6_K super-blocks with every code 0 or 63 and int8 scales -128 / 127 / 0, d of 0, the fp16
    maximum and the smallest subnormal: d*scale*(code-32) is exact in fp32, bit for bit."""
    N, K = 48, 512
    blocks, _, _ = synth.weights(q.QLIN_Q6_K, N, K, synth.gen(10))
    b = blocks.clone().view(N, K // 256, 210)
    fp16 = torch.tensor([0.0, 65504.0, 2.0 ** -24, 1.0], dtype=torch.float16).view(torch.uint8).view(4, 2)
    for n in range(N):
        b[n, :, 208:210] = fp16[n % 4]
        if n % 3 == 0:
            b[n, :, 0:192] = 0xFF  # every code 63
            b[n, :, 192:208] = 0x80  # scale -128
        elif n % 3 == 1:
            b[n, :, 0:192] = 0  # every code 0
            b[n, :, 192:208] = 0x7F  # scale 127
    blocks = b.reshape(N, -1).contiguous()
    packed = q.qlin_pack_weights(q.QLIN_Q6_K, N, K, blocks.cuda())
    w = q.qlin_dequant_debug(q.QLIN_Q6_K, packed, N, K).cpu().numpy()
    ref = oracle.dequant_f32(q.QLIN_Q6_K, N, K, blocks.numpy())
    assert np.array_equal(w.view(np.uint32), ref.view(np.uint32))


def test_strided_x_and_y():
    fmt, N, K, M = q.QLIN_Q4_0, 96, 512, 3
    blocks, scales, g, packed = make(fmt, N, K, 31)
    xb = synth.activations(M, K + 64, synth.gen(32)).cuda()
    x = xb[:, :K]
    y = torch.full((M, N + 8), float("nan"), device="cuda")
    q.qlin_gemv(fmt, packed, N, K, x, y=y[:, :N])
    yref, A = oracle.gemv(fmt, N, K, blocks, x.cpu().double().numpy())
    check_y(y[:, :N], yref, A)
    assert torch.isnan(y[:, N:]).all()


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("M", [1, 4])
def test_silu_gate_epilogue(fmt, M):
    I, K = 272, 1024  # N = 2I gate_up rows; ragged 16-row half-tiles
    N = 2 * I
    blocks, scales, g, packed = make(fmt, N, K, 41 + M, q.QLIN_PACK_GATE_UP)
    xdt = torch.bfloat16 if fmt == q.QLIN_NVFP4 else torch.float32
    x = synth.activations(M, K, synth.gen(42), dtype=xdt)
    h = q.qlin_gemv(fmt, packed, N, K, x.cuda(), flags=q.QLIN_EPI_SILU_GATE).double().cpu().numpy()
    gu, Agu = oracle.gemv(fmt, N, K, blocks, x.double().numpy(), scales=scales, g=g)
    href, Ah = oracle.silu_gate(gu, Agu)
    err = np.abs(h - href)
    tol = silu_tol(href, Ah, gu[:, I:])
    assert (err <= tol).all(), np.max(err / np.maximum(tol, 1e-300))
    w = q.qlin_dequant_debug(fmt, packed, N, K, q.QLIN_PACK_GATE_UP).cpu().numpy()
    assert np.array_equal(w.view(np.uint32), oracle.dequant_f32(fmt, N, K, blocks, scales, g).view(np.uint32))


def test_deterministic_and_workspace_reusable():
    fmt, N, K, M = q.QLIN_Q4_0, 2560, 4096, 2
    blocks, scales, g, packed = make(fmt, N, K, 61)
    x = synth.activations(M, K, synth.gen(62)).cuda()
    ws = q.workspace(q.qlin_workspace_bytes(q.QLIN_OP_GEMV, fmt, M, N, K))
    ys = [q.qlin_gemv(fmt, packed, N, K, x, ws=ws) for _ in range(5)]
    for y in ys[1:]:
        assert torch.equal(y, ys[0])
    assert q.qlin_ws_status(ws) == 0
    cnt = ws[256:256 + 4 * ((N + 31) // 32)]
    assert not cnt.any()  # tile tickets back at zero


def test_pdl_launches_in_a_chain_match():
    fmt, N, K = q.QLIN_Q4_0, 1024, 1024
    blocks, scales, g, packed = make(fmt, N, K, 71)
    x = synth.activations(1, K, synth.gen(72)).cuda()
    ws = q.workspace(q.qlin_workspace_bytes(q.QLIN_OP_GEMV, fmt, 1, N, K))
    ref = q.qlin_gemv(fmt, packed, N, K, x, ws=ws)
    # chain: y_{i+1} = W y_i / ||.|| style dependency through the same buffers, with PDL
    a = x.clone()
    b = torch.empty(1, N, device="cuda")
    outs = []
    for _ in range(6):
        q.qlin_gemv(fmt, packed, N, K, a, y=b, ws=ws, flags=q.QLIN_FLAG_PDL)
        a, b = b, a
        outs.append(a.clone())
    torch.cuda.synchronize()
    a2 = x.clone()
    for i in range(6):
        y2 = q.qlin_gemv(fmt, packed, N, K, a2, ws=ws)
        assert torch.equal(y2, outs[i])
        a2 = y2
    assert torch.equal(outs[0], ref)
