"""GPU parity of the prefill-chunk GEMM for the GGUF and MXFP4 formats (the bf16 path).

qlin_pack_weights(QLIN_PACK_MMA_BF16) builds a bf16 copy of the dequantized weights: every weight is the
fp32 value the oracle's dequant gives, rounded to nearest-even bf16 (torch's conversion is the
reference rounding) -- checked bit for bit, tail columns zero.  qlin_gemm_chunk then multiplies bf16
x by that copy on the tensor cores with fp32 accumulation: checked against the fp64 product with
the same bf16 weights (|y - ref| <= 2 K 2^-24 sum|x w_bf16|: the fp32 summation bound, with one ulp
per addition allowed for the tensor core's order and rounding) and against the
unrounded weights within the chunk path's 1e-2 sum|x w| bound.
"""
import numpy as np
import pytest
import torch

import gemm_dequant_gemv_q8_b200 as q
import oracle
import synth

pytestmark = pytest.mark.gpu

FMTS = [q.QLIN_Q4_0, q.QLIN_Q8_0, q.QLIN_MXFP4, q.QLIN_Q4_K, q.QLIN_Q6_K]


def kquant(fmt):
    return fmt in (q.QLIN_Q4_K, q.QLIN_Q6_K)


def make(fmt, N, K, seed):
    blocks, scales, g = synth.weights(fmt, N, K, synth.gen(seed))
    packed = q.qlin_pack_weights(fmt, N, K, blocks.cuda(), None if scales is None else scales.cuda(), g,
                                 q.QLIN_PACK_MMA_BF16)
    w32 = oracle.dequant_f32(fmt, N, K, blocks.numpy(), None if scales is None else scales.numpy(), g)
    return packed, w32


def cache(packed, N, K):
    # blocks of 256 rows x 64 values: block (nb, kb) holds rows 256 nb.. and columns 64 kb..
    kc = (K + 63) // 64 * 64
    npad = (N + 255) // 256 * 256
    blocks = packed[256:256 + npad * kc * 2].view(torch.bfloat16).view(npad // 256, kc // 64, 256, 64)
    return blocks.permute(0, 2, 1, 3).reshape(npad, kc), kc


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("N,K", [(40, 256), (33, 96), (300, 2560)])
def test_bf16_cache_bit_exact(fmt, N, K):
    if kquant(fmt) and K % 256:
        pytest.skip("K-quants need K % 256 == 0")
    packed, w32 = make(fmt, N, K, 900 + N)
    assert packed.numel() == q.qlin_packed_bytes(fmt, N, K, q.QLIN_PACK_MMA_BF16)
    wb, kc = cache(packed, N, K)
    ref = torch.from_numpy(w32).to(torch.bfloat16)
    got = wb[:N, :K].cpu()
    assert torch.equal(got.view(torch.int16), ref.view(torch.int16))
    assert (wb[:, K:].cpu().float() == 0).all() and (wb[N:].cpu().float() == 0).all()


def check(y, x, w32, tol_exact=1e-2):
    xd = x.double().cpu().numpy()
    wb = torch.from_numpy(w32).to(torch.bfloat16).double().numpy()
    ref = xd @ wb.T
    A = np.abs(xd) @ np.abs(wb).T
    K = xd.shape[1]
    err = np.abs(y.double().cpu().numpy() - ref)
    bound = 2 * K * 2.0 ** -24 * A + 1e-30
    assert (err <= bound).all(), float(np.max(err / bound))
    exact = xd @ w32.astype(np.float64).T
    A0 = np.abs(xd) @ np.abs(w32.astype(np.float64)).T
    assert (np.abs(y.double().cpu().numpy() - exact) <= tol_exact * A0 + 1e-30).all()


@pytest.mark.parametrize("flags", [0, q.QLIN_FLAG_CTA_PAIRS])
@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("M,N,K", [(1, 256, 256), (64, 300, 512), (200, 520, 2560), (513, 1000, 1024),
                                   (37, 70, 96), (300, 264, 768)])
def test_chunk_bf16_parity(fmt, M, N, K, flags):
    # QLIN_FLAG_CTA_PAIRS: 256-row tiles on pairs of CTAs when M > 128 (single CTAs otherwise)
    if kquant(fmt) and K % 256:
        pytest.skip("K-quants need K % 256 == 0")
    packed, w32 = make(fmt, N, K, 1000 + M)
    if fmt == q.QLIN_MXFP4:  # MXFP4's own chunk path is the FP4 one; the bf16 copy asks for this flag
        flags |= q.QLIN_FLAG_BF16_COPY
    x = synth.activations(M, K, synth.gen(1100 + M), dtype=torch.bfloat16).cuda()
    ws = q.workspace(q.qlin_workspace_bytes(q.QLIN_OP_CHUNK, fmt, M, N, K))
    y = q.qlin_gemm_chunk(fmt, packed, N, K, x, ws=ws, flags=flags)
    torch.cuda.synchronize()
    assert q.qlin_ws_status(ws) == 0
    check(y, x, w32)


def test_chunk_bf16_strided_operands_and_reuse():
    fmt, M, N, K = q.QLIN_Q4_0, 150, 264, 768
    packed, w32 = make(fmt, N, K, 77)
    xb = synth.activations(M, K + 40, synth.gen(78), dtype=torch.bfloat16).cuda()  # ldx = K + 40 (8-aligned)
    x = xb[:, :K]
    y = torch.full((M, N + 5), float("nan"), device="cuda")
    ws = q.workspace(q.qlin_workspace_bytes(q.QLIN_OP_CHUNK, fmt, M, N, K))
    for _ in range(2):
        q.qlin_gemm_chunk(fmt, packed, N, K, x, y=y[:, :N], ws=ws)
    torch.cuda.synchronize()
    assert q.qlin_ws_status(ws) == 0
    check(y[:, :N], x, w32)
    assert torch.isnan(y[:, N:]).all()


@pytest.mark.parametrize("flags", [0, q.QLIN_FLAG_CTA_PAIRS])
def test_chunk_bf16_full_size_sampled(flags):
    # a prefill chunk of the Q4_0 4B stack's gate_up: M = 512, K = 2560, N = 2 x 9728; sampled rows
    fmt, M, N, K = q.QLIN_Q4_0, 512, 19456, 2560
    blocks, _, _ = synth.weights(fmt, N, K, synth.gen(4242))
    packed = q.qlin_pack_weights(fmt, N, K, blocks.cuda(), pack_flags=q.QLIN_PACK_MMA)
    x = synth.activations(M, K, synth.gen(4243), dtype=torch.bfloat16).cuda()
    ws = q.workspace(q.qlin_workspace_bytes(q.QLIN_OP_CHUNK, fmt, M, N, K))
    y = q.qlin_gemm_chunk(fmt, packed, N, K, x, ws=ws, flags=flags)
    torch.cuda.synchronize()
    assert q.qlin_ws_status(ws) == 0
    rows = np.unique(np.linspace(0, N - 1, 61).astype(np.int64))
    w32 = oracle.dequant_f32(fmt, N, K, blocks.numpy())[rows]
    check(y[:, rows], x, w32)


def test_chunk_bf16_argument_checks():
    fmt, M, N, K = q.QLIN_Q8_0, 8, 64, 256
    packed, _ = make(fmt, N, K, 5)
    lib = q.lib()
    ws = q.workspace(256)
    xb = torch.zeros(M, K + 4, dtype=torch.bfloat16, device="cuda")
    y = torch.empty(M, N, device="cuda")
    # ldx not a multiple of 8: the tensor-map rows would not be 16-byte aligned
    st = lib.qlin_gemm_chunk(fmt, q._dev(packed, "p"), N, K, q._dev(xb, "x"), M, K + 4, q._dev(y, "y"), N, 0,
                             q._dev(ws, "ws"), 256, q._stream(None))
    assert st == 3  # QLIN_ERR_ALIGNMENT
    st = lib.qlin_gemm_chunk(fmt, q._dev(packed, "p"), N, K, q._dev(xb, "x"), M, K, q._dev(y, "y"), N, 0,
                             q._dev(ws, "ws"), 255, q._stream(None))
    assert st == 4  # QLIN_ERR_WORKSPACE


def test_chunk_bf16_back_to_back_pdl():
    # calls enqueued back to back with QLIN_FLAG_PDL (each may start while the previous drains)
    fmt, N, K = q.QLIN_Q4_0, 520, 1024
    packed, w32 = make(fmt, N, K, 61)
    ws = q.workspace(q.qlin_workspace_bytes(q.QLIN_OP_CHUNK, fmt, 512, N, K))
    runs = []
    for M, fl in ((512, 0), (64, 0), (300, q.QLIN_FLAG_CTA_PAIRS), (5, 0)):
        x = synth.activations(M, K, synth.gen(62 + M), dtype=torch.bfloat16).cuda()
        runs.append((x, q.qlin_gemm_chunk(fmt, packed, N, K, x, ws=ws, flags=fl | q.QLIN_FLAG_PDL)))
    torch.cuda.synchronize()
    assert q.qlin_ws_status(ws) == 0
    for x, y in runs:
        check(y, x, w32)


# ------------------------------------------------------------------ NVFP4 weights on the bf16 path
def make_nvfp4_bf16(N, K, seed):
    codes, scales, g = synth.weights(q.QLIN_NVFP4, N, K, synth.gen(seed))
    packed = q.qlin_pack_weights(q.QLIN_NVFP4, N, K, codes.cuda(), scales.cuda(), g, q.QLIN_PACK_MMA_BF16)
    return codes.numpy(), scales.numpy(), g, packed


def test_nvfp4_bf16_copy_holds_exact_block_products():
    """QLIN_PACK_MMA_BF16 for NVFP4: every element is e2m1 * e4m3 (the oracle's dequant with a
    per-tensor scale of 1, exact in bf16), the per-tensor scale kept in the header."""
    N, K = 300, 272  # ragged rows and a K that ends in the middle of a 64-value stage
    codes, scales, g, packed = make_nvfp4_bf16(N, K, 77)
    assert packed.numel() == q.qlin_packed_bytes(q.QLIN_NVFP4, N, K, q.QLIN_PACK_MMA_BF16)
    wb, kc = cache(packed, N, K)
    prod = oracle.dequant(q.QLIN_NVFP4, N, K, codes, scales, 1.0)
    ref = torch.from_numpy(prod).to(torch.bfloat16)
    assert np.array_equal(ref.double().numpy(), prod)  # the products are bf16 numbers
    assert torch.equal(wb[:N, :K].cpu().view(torch.int16), ref.view(torch.int16))
    assert (wb[:, K:].cpu().float() == 0).all() and (wb[N:].cpu().float() == 0).all()
    hdr_g = packed[:256].cpu().view(torch.float32)[7].item()  # PackedHeader.global_scale (byte 28)
    assert hdr_g == g


@pytest.mark.parametrize("flags", [q.QLIN_FLAG_BF16_COPY, q.QLIN_FLAG_BF16_COPY | q.QLIN_FLAG_CTA_PAIRS])
@pytest.mark.parametrize("M,N,K", [(64, 300, 512), (200, 520, 2560), (513, 1000, 1024), (37, 70, 272)])
def test_nvfp4_bf16_path_meets_the_bf16_operand_bound(M, N, K, flags):
    """y = g * sum x * (e2m1 * e4m3): exact products in the tensor core, fp32 accumulation, one
    rounding for g.  Against the fp64 product of the bf16 x as given and the exact NVFP4 weights
    (no activation quantization): |y - y_ref| <= (2K + 1) 2^-24 sum|w x| (the fp32 summation bound of
    the other bf16-path tests plus the scale's rounding), which implies the bf16-operand chunk bound
    of 1e-2 sum|w x| by a wide margin."""
    codes, scales, g, packed = make_nvfp4_bf16(N, K, 3000 + M)
    x = synth.activations(M, K, synth.gen(3100 + M), dtype=torch.bfloat16)
    y = q.qlin_gemm_chunk(q.QLIN_NVFP4, packed, N, K, x.cuda(), flags=flags)
    torch.cuda.synchronize()
    rows = np.unique(np.linspace(0, N - 1, min(N, 64)).astype(np.int64))
    yref, A = oracle.gemv(q.QLIN_NVFP4, N, K, codes, x.double().numpy(), scales=scales, g=g, rows=rows)
    err = np.abs(y[:, rows].double().cpu().numpy() - yref)
    bound = (2 * K + 1) * 2.0 ** -24 * A + 1e-30
    assert (err <= bound).all(), float(np.max(err / bound))
    assert (err <= 1e-2 * A + 1e-30).all()
