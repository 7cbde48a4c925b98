"""GPU parity on hand-built blocks at the edges of the Q8_0, Q4_0, Q6_K and NVFP4 formats.

The seeded workloads never produce these fields, so they are built here byte by byte:
  Q8_0 / Q4_0: every code, including Q8_0's -128 (legal in the format, outside the workload's
      [-127, 127]); blocks of one small constant code (+-1), where a decoder that removes the
      unsigned offset from a block sum instead of from each value loses the 2e-6 bound; fp16
      scales d in {+0, -0, -1, 1, 2^-24 (the smallest subnormal), 65504 (the largest finite)}.
  NVFP4: E4M3 block scales 0 (+0 and -0), the smallest subnormal 2^-9, 448 (the largest), a
      negative scale and NaN (0x7F); the per-tensor scale fp32(1/448) of the workload.
  activations at the ends of the range in which the Q4_0 / Q8_0 products are exact:
      2^-40 <= |x| < 2^65.
Bars (as the other GEMV tests): dequantized weights bit-exact (NaN exactly where the oracle has
NaN); one-hot x reproduces a dequantized column; y within 2e-6 * sum|w*x| of the fp64 oracle,
element by element, NaN exactly where the oracle's y is NaN.
"""
import numpy as np
import pytest
import torch

import gemm_dequant_gemv_q8_b200 as q
import oracle
import synth

pytestmark = pytest.mark.gpu
TOL = 2e-6
D_EDGE = [0.0, -0.0, -1.0, 1.0, 2.0 ** -24, 65504.0]


def fp16_bytes(v):
    return np.frombuffer(np.array([v], dtype=np.float16).tobytes(), dtype=np.uint8)


def q8_0_edge(N, K, rng):
    """Q8_0 rows of hand-built blocks: block b of row n takes d = D_EDGE[(n + b) % 6] and one of
    four code patterns: every code -128..127 across the row's blocks, all +1, all -1, or random
    codes over the full int8 range."""
    nb = K // 32
    out = np.zeros((N, nb, 34), dtype=np.uint8)
    ramp = np.arange(-128, 128, dtype=np.int16)
    for n in range(N):
        for b in range(nb):
            out[n, b, 0:2] = fp16_bytes(D_EDGE[(n + b) % len(D_EDGE)])
            kind = (n // 2 + b) % 4
            if kind == 0:
                codes = ramp[(32 * (b + n)) % 256:][:32]
                if len(codes) < 32:
                    codes = np.concatenate([codes, ramp[:32 - len(codes)]])
            elif kind == 1:
                codes = np.ones(32, np.int16)
            elif kind == 2:
                codes = -np.ones(32, np.int16)
            else:
                codes = rng.integers(-128, 128, 32).astype(np.int16)
            out[n, b, 2:] = codes.astype(np.int8).view(np.uint8)
    return torch.from_numpy(out.reshape(N, nb * 34).copy())


def q4_0_edge(N, K, rng):
    """Q4_0 rows: d as for Q8_0; code patterns: every nibble 0..15 twice, all q = +1 (nibble 9),
    all q = -1 (nibble 7), all q = -8 (nibble 0), or random nibbles."""
    nb = K // 32
    out = np.zeros((N, nb, 18), dtype=np.uint8)
    for n in range(N):
        for b in range(nb):
            out[n, b, 0:2] = fp16_bytes(D_EDGE[(n + b) % len(D_EDGE)])
            kind = (n // 2 + b) % 5
            if kind == 0:
                nib = np.concatenate([np.arange(16), np.arange(16)[::-1]])
            elif kind == 1:
                nib = np.full(32, 9)
            elif kind == 2:
                nib = np.full(32, 7)
            elif kind == 3:
                nib = np.zeros(32, np.int64)
            else:
                nib = rng.integers(0, 16, 32)
            out[n, b, 2:] = (nib[:16] | (nib[16:] << 4)).astype(np.uint8)  # element j low, j+16 high
    return torch.from_numpy(out.reshape(N, nb * 18).copy())


E4M3_EDGE = [0x00, 0x80, 0x01, 0x7E, 0xB8, 0x38, 0x7F]  # +0, -0, 2^-9, 448, -1, 1, NaN


def nvfp4_edge(N, K, rng, with_nan=True):
    """NVFP4 codes covering all 16 values; E4M3 scales cycling through E4M3_EDGE (NaN only in rows
    n % 4 == 3 when with_nan, so the other rows stay finite); per-tensor scale fp32(1/448)."""
    codes = np.zeros((N, K // 2), dtype=np.uint8)
    for n in range(N):
        c = (np.arange(K) + n) % 16 if n % 2 == 0 else rng.integers(0, 16, K)
        codes[n] = (c[0::2] | (c[1::2] << 4)).astype(np.uint8)
    scales = np.zeros((N, K // 16), dtype=np.uint8)
    edge = E4M3_EDGE if with_nan else E4M3_EDGE[:-1]
    for n in range(N):
        for b in range(K // 16):
            s = edge[(n + b) % len(edge)]
            if s == 0x7F and n % 4 != 3:
                s = 0x3C  # 1.5
            scales[n, b] = s
    return torch.from_numpy(codes), torch.from_numpy(scales), synth.NVFP4_G


def edge_activations(M, K, rng, dtype=torch.float32):
    """Row 0: |x| in [2^-40, 2^-39) with random signs; row 1: |x| in [2^63, 2^65); row 2: all
    positive N(0,1) magnitudes (every product of a constant-code block has one sign); further rows
    N(0,1)."""
    x = rng.standard_normal((M, K))
    mant = rng.uniform(1.0, 2.0, (M, K)) * np.where(rng.random((M, K)) < 0.5, -1.0, 1.0)
    if M > 0:
        x[0] = mant[0] * 2.0 ** -40
    if M > 1:
        x[1] = mant[1] * 2.0 ** 63 * np.where(rng.random(K) < 0.5, 1.0, 1.99)
    if M > 2:
        x[2] = np.abs(x[2])
    t = torch.from_numpy(x).to(torch.float32)
    return t.to(dtype).contiguous()


def pack(fmt, N, K, blocks, scales, g):
    return q.qlin_pack_weights(fmt, N, K, blocks.cuda(), None if scales is None else scales.cuda(), g)


def bitwise_equal_or_both_nan(a, b):
    nan = np.isnan(b)
    assert np.array_equal(np.isnan(a), nan)
    assert np.array_equal(a[~nan].view(np.uint32), b[~nan].view(np.uint32))


def check_y(y, yref, A):
    y = y.double().cpu().numpy()
    nan = np.isnan(yref) | np.isnan(A)
    assert np.array_equal(np.isnan(y), nan), "NaN outputs differ from the oracle's"
    err = np.abs(y - yref)[~nan]
    tol = TOL * A[~nan]
    bad = err > tol
    assert not bad.any(), f"{bad.sum()} outside; worst {np.max(err / np.maximum(tol, 1e-300)):.3g} x tol"


BUILDERS = {
    q.QLIN_Q8_0: lambda N, K, rng: (q8_0_edge(N, K, rng), None, 1.0),
    q.QLIN_Q4_0: lambda N, K, rng: (q4_0_edge(N, K, rng), None, 1.0),
    q.QLIN_NVFP4: nvfp4_edge,
}


@pytest.mark.parametrize("fmt", [q.QLIN_Q8_0, q.QLIN_Q4_0, q.QLIN_NVFP4])
def test_edge_dequant_bit_exact(fmt):
    N, K = 72, 512
    blocks, scales, g = BUILDERS[fmt](N, K, np.random.default_rng(fmt))
    w = q.qlin_dequant_debug(fmt, pack(fmt, N, K, blocks, scales, g), N, K).cpu().numpy()
    ref = oracle.dequant_f32(fmt, N, K, blocks.numpy(), None if scales is None else scales.numpy(), g)
    bitwise_equal_or_both_nan(w, ref)
    if fmt != q.QLIN_NVFP4:
        assert (ref.view(np.uint32) == 0x80000000).any()  # d = -0 reached the decoder


@pytest.mark.parametrize("fmt", [q.QLIN_Q8_0, q.QLIN_Q4_0, q.QLIN_NVFP4])
def test_edge_one_hot_columns(fmt):
    N, K = 72, 512
    rng = np.random.default_rng(10 + fmt)
    # no NaN scales here: a NaN weight anywhere in a row makes the whole output row NaN (NaN * 0)
    blocks, scales, g = nvfp4_edge(N, K, rng, with_nan=False) if fmt == q.QLIN_NVFP4 else BUILDERS[fmt](N, K, rng)
    packed = pack(fmt, N, K, blocks, scales, g)
    W = oracle.dequant_f32(fmt, N, K, blocks.numpy(), None if scales is None else scales.numpy(), g)
    ks = [0, 1, 17, 31, 32, 255, 256, 300, 511]
    x = torch.zeros(len(ks), K)
    for i, k in enumerate(ks):
        x[i, k] = 1.0
    for m0 in range(0, len(ks), 8):
        y = q.qlin_gemv(fmt, packed, N, K, x[m0:m0 + 8].cuda()).cpu().numpy()
        for i, k in enumerate(ks[m0:m0 + 8]):
            col = W[:, k]
            nan = np.isnan(col)
            assert np.array_equal(np.isnan(y[i]), nan)
            assert np.array_equal(y[i][~nan], col[~nan]), k  # by value: -0 and +0 compare equal


@pytest.mark.parametrize("fmt", [q.QLIN_Q8_0, q.QLIN_Q4_0, q.QLIN_NVFP4])
@pytest.mark.parametrize("M", [1, 3, 8])
@pytest.mark.parametrize("xdt", [torch.float32, torch.bfloat16])
def test_edge_gemv_parity(fmt, M, xdt):
    N, K = 200, 2048  # several tiles, a ragged last tile, 8 k-groups
    rng = np.random.default_rng(100 * fmt + M)
    blocks, scales, g = BUILDERS[fmt](N, K, rng)
    packed = pack(fmt, N, K, blocks, scales, g)
    x = edge_activations(M, K, rng, xdt)
    y = q.qlin_gemv(fmt, packed, N, K, x.cuda())
    yref, A = oracle.gemv(fmt, N, K, blocks.numpy(), x.double().numpy(),
                          scales=None if scales is None else scales.numpy(), g=g)
    check_y(y, yref, A)


def small_code_rows(fmt, N, K, rng):
    """Rows of blocks whose codes are small: even rows one constant code (+1 in rows 0 mod 4, -1
    in rows 2 mod 4), odd rows sparse (every code 0 but one +-1 per block).  Scales as the
    workload's."""
    nb = K // 32
    per = 34 if fmt == q.QLIN_Q8_0 else 18
    b = np.zeros((N, nb, per), np.uint8)
    lo, hi = (1e-3, 1e-2) if fmt == q.QLIN_Q8_0 else (1e-3, 2e-2)
    for n in range(N):
        for blk in range(nb):
            b[n, blk, 0:2] = fp16_bytes(float(rng.uniform(lo, hi)))
            if n % 2 == 0:
                codes = np.full(32, 1 if n % 4 == 0 else -1)
            else:
                codes = np.zeros(32, np.int64)
                codes[rng.integers(0, 32)] = rng.choice([-1, 1])
            if fmt == q.QLIN_Q8_0:
                b[n, blk, 2:] = codes.astype(np.int8).view(np.uint8)
            else:
                nib = codes + 8
                b[n, blk, 2:] = (nib[:16] | (nib[16:] << 4)).astype(np.uint8)
    return torch.from_numpy(b.reshape(N, -1).copy())


@pytest.mark.parametrize("fmt", [q.QLIN_Q8_0, q.QLIN_Q4_0])
@pytest.mark.parametrize("K", [32, 4096])
def test_edge_small_and_sparse_codes(fmt, K):
    """Blocks of one small constant code with all-positive activations (the products of a block
    have one sign), and sparse blocks (one code +-1 among zeros).  A decoder that adds the unsigned
    codes (q + 8, q + 128) and removes the offset once per block from a sum of the activations
    leaves rounding errors of the size of offset * sum|x| there: with K = 32 (one block per row) it
    misses 2e-6 * sum|w*x| on most of these outputs (by fp32 emulation: ~80% of the constant-code
    Q8_0 rows, ~50-95% of the sparse rows, errors up to 5e-2 of sum|w*x|).  The bound must hold on
    every output."""
    N, M = 64, 3
    rng = np.random.default_rng(5 + K)
    blocks = small_code_rows(fmt, N, K, rng)
    packed = pack(fmt, N, K, blocks, None, 1.0)
    x = np.abs(rng.standard_normal((M, K)))
    x[1] = rng.uniform(0.5, 1.0, K)
    x[2] = rng.standard_normal(K)
    x = torch.from_numpy(x).float()
    for rows in (x[:1], x):  # M = 1 and M = 3 (two rows per pass)
        y = q.qlin_gemv(fmt, packed, N, K, rows.cuda())
        yref, A = oracle.gemv(fmt, N, K, blocks.numpy(), rows.double().numpy())
        check_y(y, yref, A)


def test_edge_q6k_constant_small_codes():
    """Q6_K rows whose codes are all 33 or 31 (q = +1 / -1) with positive activations: the Q6_K
    decoder removes its offset 32 per value as Q8_0's does."""
    N, K, M = 64, 1024, 1
    rng = np.random.default_rng(6)
    b = np.zeros((N, K // 256, 210), np.uint8)
    for n in range(N):
        code = 33 if n % 2 == 0 else 31
        b[n, :, 0:128] = (code & 15) | ((code & 15) << 4)  # low 4 bits, both nibbles
        hi = code >> 4
        b[n, :, 128:192] = hi | (hi << 2) | (hi << 4) | (hi << 6)
        b[n, :, 192:208] = np.uint8(rng.integers(1, 127))
        b[n, :, 208:210] = fp16_bytes(float(rng.uniform(2e-5, 2e-4)))
    blocks = torch.from_numpy(b.reshape(N, -1).copy())
    packed = pack(q.QLIN_Q6_K, N, K, blocks, None, 1.0)
    x = torch.from_numpy(np.abs(rng.standard_normal((M, K)))).float()
    y = q.qlin_gemv(q.QLIN_Q6_K, packed, N, K, x.cuda())
    yref, A = oracle.gemv(q.QLIN_Q6_K, N, K, blocks.numpy(), x.double().numpy())
    assert np.all(np.abs(oracle.dequant_f32(q.QLIN_Q6_K, N, K, blocks.numpy())) > 0)
    check_y(y, yref, A)


@pytest.mark.parametrize("fmt", [q.QLIN_Q8_0, q.QLIN_Q4_0, q.QLIN_NVFP4])
def test_edge_chain_matches_oracle(fmt):
    """The same edge blocks through qlin_gemv_chain (the decode-step launch), two ops, the second
    reading the first's output."""
    N = K = 512
    rng = np.random.default_rng(40 + fmt)
    blocks, scales, g = BUILDERS[fmt](N, K, rng)
    if fmt == q.QLIN_NVFP4:
        blocks, scales, g = nvfp4_edge(N, K, rng, with_nan=False)
    packed = pack(fmt, N, K, blocks, scales, g)
    x = torch.from_numpy(rng.standard_normal((1, K))).float()
    xd = x.cuda()
    y1 = torch.empty(1, N, device="cuda")
    y2 = torch.empty(1, N, device="cuda")
    ops = [q.gemv_op(packed, N, K, xd, y1), q.gemv_op(packed, N, K, y1, y2, wait_for=0)]
    q.qlin_gemv_chain(fmt, q.QLIN_F32, 1, ops)
    sc = None if scales is None else scales.numpy()
    r1, A1 = oracle.gemv(fmt, N, K, blocks.numpy(), x.double().numpy(), scales=sc, g=g)
    check_y(y1, r1, A1)
    r2, A2 = oracle.gemv(fmt, N, K, blocks.numpy(), y1.double().cpu().numpy(), scales=sc, g=g)
    check_y(y2, r2, A2)
