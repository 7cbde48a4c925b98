"""Pins of the fp64 oracle against what the formats and the mathematics fix (CPU only).

Each check is chosen so that a plausible mistake in the oracle (a swapped nibble, a wrong
exponent bias, a dropped term, a transposed operand, a wrong tie rule) fails one of them.  None of
them re-derives a value through the oracle's own code path: the references are golden fixtures
worked by hand from the format definitions, library routines (numpy float16, torch float8,
torch silu, numpy argsort), exact rational arithmetic, and closed forms.
"""
import math
import struct
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
import synth
from conftest import read_golden


def f32_bits(v):
    return struct.unpack("<I", struct.pack("<f", v))[0]


# ----------------------------------------------------------------------------- scalar decoders
def test_fp16_all_codes_match_numpy():
    ref = np.arange(65536, dtype=np.uint32).astype(np.uint16).view(np.float16).astype(np.float64)
    got = np.array([oracle.fp16(b) for b in range(65536)])
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(got))
    assert np.array_equal(ref[~nan], got[~nan])
    assert np.array_equal(np.signbit(ref[~nan]), np.signbit(got[~nan]))


def test_e4m3_all_codes_match_torch():
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = np.array([oracle.e4m3(b) for b in range(256)])
    nan = np.isnan(ref)
    assert nan.sum() == 2  # S.1111.111 only: the "fn" variant has no infinities
    assert np.array_equal(nan, np.isnan(got))
    assert np.array_equal(ref[~nan], got[~nan])
    assert oracle.e4m3(0x7E) == 448.0 and oracle.e4m3(0x01) == 2.0 ** -9


def test_e2m1_all_codes_match_golden():
    rows = [l.split() for l in read_golden("e2m1_values.txt")]
    assert len(rows) == 16
    for code, val in rows:
        c, v = int(code, 16), float(val)
        got = oracle.e2m1(c)
        assert got == v and math.copysign(1, got) == math.copysign(1, v), (c, got, v)


def test_e8m0_all_codes_match_fp32_bit_construction():
    # UE8M0 byte b is the biased exponent of a power of two: the fp32 number with exponent field b
    # and a zero mantissa for b = 1..254, the fp32 subnormal 0x00400000 (2^-127) for b = 0, NaN
    # for 0xFF.  Built from bits here, not through the oracle's ldexp.
    for b in range(1, 255):
        ref = float(np.array([b << 23], np.uint32).view(np.float32)[0])
        assert oracle.e8m0(b) == ref, b
    assert oracle.e8m0(0) == float(np.array([0x00400000], np.uint32).view(np.float32)[0]) == 2.0 ** -127
    assert math.isnan(oracle.e8m0(255))


# ----------------------------------------------------------------------------- block dequant
def _golden_blocks(name):
    lines = read_golden(name)
    out = []
    for i in range(0, len(lines), 2):
        assert lines[i].startswith("bytes:") and lines[i + 1].startswith("values:")
        b = bytes(int(t, 16) for t in lines[i].split()[1:])
        v = [float(t) for t in lines[i + 1].split()[1:]]
        out.append((b, v))
    return out


@pytest.mark.parametrize("fmt,name", [(oracle.Q8_0, "q8_0_block.txt"), (oracle.Q4_0, "q4_0_block.txt")])
def test_gguf_block_dequant_matches_golden(fmt, name):
    for b, v in _golden_blocks(name):
        blocks = np.frombuffer(b, np.uint8)
        w = oracle.dequant(fmt, 1, 32, blocks)[0]
        assert list(w) == v
        w32 = oracle.dequant_f32(fmt, 1, 32, blocks)[0]
        assert np.array_equal(w32.astype(np.float64), np.array(v))


def test_gguf_blocks_stack_along_k_and_rows():
    # Two golden blocks side by side in one row, and the same row twice: block b of row n covers
    # k in [32b, 32b+32); rows are independent.
    (b0, v0), (b1, v1) = _golden_blocks("q4_0_block.txt")[:2]
    row = np.frombuffer(b0 + b1, np.uint8)
    W = oracle.dequant(oracle.Q4_0, 2, 64, np.concatenate([row, row[::-1][::-1]]))
    assert list(W[0]) == v0 + v1 and list(W[1]) == v0 + v1


def test_nvfp4_dequant_rounding_golden():
    for line in read_golden("nvfp4_rounding.txt"):
        code, sc, gb, wb = (int(t, 16) for t in line.split())
        g = struct.unpack("<f", struct.pack("<I", gb))[0]
        codes = np.zeros((1, 8), np.uint8)
        codes[0, 0] = code  # element 0 is the low nibble of byte 0
        codes[0, 7] = code << 4  # element 15 is the high nibble of byte 7
        scales = np.array([[sc]], np.uint8)
        w32 = oracle.dequant_f32(oracle.NVFP4, 1, 16, codes, scales, g)[0]
        assert f32_bits(float(w32[0])) == wb, (hex(code), hex(f32_bits(float(w32[0]))), hex(wb))
        assert f32_bits(float(w32[15])) == wb
        assert all(f32_bits(float(t)) == 0 for t in w32[1:15])


def test_nvfp4_scale_applies_per_16():
    # Codes all 0x2 (1.0); scales 1.0, 2.0, 0.5 for k in [0,16), [16,32), [32,48).
    codes = np.full((1, 24), 0x22, np.uint8)
    scales = np.array([[0x38, 0x40, 0x30]], np.uint8)  # E4M3 1.0, 2.0, 0.5
    w = oracle.dequant(oracle.NVFP4, 1, 48, codes, scales, 1.0)[0]
    assert list(w) == [1.0] * 16 + [2.0] * 16 + [0.5] * 16


def test_mxfp4_dequant_matches_golden():
    lines = read_golden("mxfp4_block.txt")
    codes = np.array([[int(t, 16) for t in lines[0].split()[1:]]], np.uint8)
    scales = np.array([[int(t, 16) for t in lines[1].split()[1:]]], np.uint8)
    v = [float(t) for t in lines[2].split()[1:]]
    w = oracle.dequant(oracle.MXFP4, 1, 64, codes, scales)[0]
    assert list(w) == v and list(np.signbit(w)) == [math.copysign(1, t) < 0 for t in v]
    w32 = oracle.dequant_f32(oracle.MXFP4, 1, 64, codes, scales)[0]
    assert np.array_equal(w32.astype(np.float64), np.array(v))


def test_mxfp4_equals_nvfp4_with_the_same_power_of_two_scales():
    # A UE8M0 scale 2^(e-127) with e in [120, 134] is exactly an E4M3 value (2^-7 .. 2^7); giving
    # both 16-value halves of each 32-value block that E4M3 scale (converted by torch) and the
    # per-tensor scale 1 must give the same weights through the (separately pinned) NVFP4 decode.
    N, K = 6, 128
    codes, _, _ = synth.weights(oracle.MXFP4, N, K, synth.gen(11))
    e = torch.randint(120, 135, (N, K // 32), generator=synth.gen(12), dtype=torch.int32)
    pow2 = torch.pow(2.0, (e - 127).to(torch.float64)).to(torch.float32)
    e4 = pow2.to(torch.float8_e4m3fn)
    assert torch.equal(e4.to(torch.float32), pow2)
    nv_scales = e4.view(torch.uint8).repeat_interleave(2, dim=1).numpy()
    Wmx = oracle.dequant(oracle.MXFP4, N, K, codes.numpy(), e.to(torch.uint8).numpy())
    Wnv = oracle.dequant(oracle.NVFP4, N, K, codes.numpy(), nv_scales, 1.0)
    assert np.array_equal(Wmx, Wnv)


def test_mxfp4_scale_ff_is_nan_only_in_its_block():
    codes = np.full((1, 32), 0x22, np.uint8)  # every element 1.0
    w = oracle.dequant(oracle.MXFP4, 1, 64, codes, np.array([[0xFF, 0x7F]], np.uint8))[0]
    assert np.isnan(w[:32]).all() and list(w[32:]) == [1.0] * 32


# ----------------------------------------------------------------------------- GEMV
def _identity_q8(K):
    blk = np.zeros((K, K // 32, 34), np.uint8)
    blk[:, :, 0:2] = np.frombuffer(np.float16(1.0).tobytes(), np.uint8)
    for n in range(K):
        blk[n, n // 32, 2 + n % 32] = 1
    return blk.reshape(K, -1)


def _identity_q4(K):
    blk = np.zeros((K, K // 32, 18), np.uint8)
    blk[:, :, 0:2] = np.frombuffer(np.float16(1.0).tobytes(), np.uint8)
    blk[:, :, 2:] = 0x88  # every nibble 8 -> 0
    for n in range(K):
        j = n % 32
        if j < 16:
            blk[n, n // 32, 2 + j] = (blk[n, n // 32, 2 + j] & 0xF0) | 9
        else:
            blk[n, n // 32, 2 + j - 16] = (blk[n, n // 32, 2 + j - 16] & 0x0F) | (9 << 4)
    return blk.reshape(K, -1)


def _identity_nvfp4(K):
    codes = np.zeros((K, K // 2), np.uint8)
    for n in range(K):
        codes[n, n // 2] = 0x2 << (4 * (n & 1))
    return codes, np.full((K, K // 16), 0x38, np.uint8)


# ----------------------------------------------------------------------------- Q4_K
def _q4k_block(d_bits, dmin_bits, sc, m, codes):
    """One GGUF Q4_K super-block packed from its fields, written here from the block_q4_K
    definition in the packing direction (the oracle only unpacks): 6-bit scales and mins of
    sub-blocks 0..3 in the low bits of bytes 0..3 / 4..7, the low 4 bits of those of sub-blocks
    4..7 in the nibbles of bytes 8..11, their top 2 bits in bits 6..7 of bytes 0..3 / 4..7; code k
    (c = k / 64, l = k % 32) in the low nibble of qs[32c + l] for k % 64 < 32, else the high one."""
    head = bytearray(struct.pack("<HH", d_bits, dmin_bits))
    s12 = bytearray(12)
    for j in range(8):
        if j < 4:
            s12[j] |= sc[j]
            s12[j + 4] |= m[j]
        else:
            s12[j + 4] |= (sc[j] & 15) | ((m[j] & 15) << 4)
            s12[j - 4] |= (sc[j] >> 4) << 6
            s12[j] |= (m[j] >> 4) << 6
    qs = bytearray(128)
    for k in range(256):
        c, l = k // 64, k % 32
        qs[32 * c + l] |= codes[k] if k % 64 < 32 else codes[k] << 4
    return bytes(head + s12 + qs)


def test_q4k_dequant_matches_golden():
    lines = read_golden("q4k_block.txt")
    blk = bytearray(int(t, 16) for t in lines[0].split()[1:])
    qs = bytearray(128)
    for t in lines[1].split()[1:]:
        i, v = t.split(":")
        qs[int(i)] = int(v, 16)
    w = oracle.dequant(oracle.Q4_K, 1, 256, np.frombuffer(bytes(blk + qs), np.uint8)[None, :])[0]
    for t in lines[2].split()[1:]:
        k, v = t.split(":")
        assert w[int(k)] == float(v), (k, w[int(k)], v)


def test_q4k_packed_fields_decode_exactly():
    # Every 6-bit scale and min value in every sub-block position, random codes, fp16 d / dmin
    # drawn by numpy: the oracle must return d * sc * code - dmin * m exactly (fp64 holds it).
    rng = np.random.default_rng(7)
    for rep in range(64):
        sc = [int(v) for v in (np.arange(8) * 8 + rep) % 64]
        m = [int(v) for v in (63 - np.arange(8) * 8 - rep) % 64]
        codes = [int(v) for v in rng.integers(0, 16, 256)]
        d16, dm16 = np.float16(rng.uniform(1e-3, 2.0)), np.float16(rng.uniform(1e-3, 2.0))
        blk = _q4k_block(int(d16.view(np.uint16)), int(dm16.view(np.uint16)), sc, m, codes)
        w = oracle.dequant(oracle.Q4_K, 1, 256, np.frombuffer(blk, np.uint8)[None, :])[0]
        ref = [Fraction(float(d16)) * sc[k // 32] * codes[k] - Fraction(float(dm16)) * m[k // 32] for k in range(256)]
        assert all(Fraction(w[k]) == ref[k] for k in range(256)), rep


def test_q4k_rows_of_several_superblocks_and_identity():
    # Identity through Q4_K: d = 1, dmin = 0, every sub-block scale 1 and min 0, code 1 at k = n.
    K = 512
    rows = []
    for n in range(K):
        codes = [0] * K
        codes[n] = 1
        rows.append(b"".join(_q4k_block(0x3C00, 0, [1] * 8, [0] * 8, codes[256 * b:256 * (b + 1)])
                             for b in range(K // 256)))
    blocks = np.frombuffer(b"".join(rows), np.uint8).reshape(K, -1)
    assert blocks.shape[1] == oracle.row_bytes(oracle.Q4_K, K) == 288
    x = synth.activations(2, K, synth.gen(21)).double().numpy()
    y, A = oracle.gemv(oracle.Q4_K, K, K, blocks, x)
    assert np.array_equal(y, x) and np.array_equal(A, np.abs(x))


def test_q4k_gemv_matches_exact_rational_sum_and_one_hot():
    N, K, M = 6, 512, 2
    blocks, _, _ = synth.weights(oracle.Q4_K, N, K, synth.gen(22))
    blocks = blocks.numpy()
    W = oracle.dequant(oracle.Q4_K, N, K, blocks)
    x = synth.activations(M, K, synth.gen(23)).double().numpy()
    y, A = oracle.gemv(oracle.Q4_K, N, K, blocks, x)
    for m in range(M):
        for n in range(N):
            exact = sum(Fraction(W[n, k]) * Fraction(x[m, k]) for k in range(K))
            absum = sum(abs(Fraction(W[n, k]) * Fraction(x[m, k])) for k in range(K))
            assert abs(Fraction(y[m, n]) - exact) <= Fraction(K * 2.0 ** -52) * absum
    for k in (0, 31, 32, 255, 256, 300, 511):
        e = np.zeros((1, K))
        e[0, k] = 1.0
        assert np.array_equal(oracle.gemv(oracle.Q4_K, N, K, blocks, e)[0][0], W[:, k])


def test_q4k_f32_value_is_one_rounding_of_the_exact_difference():
    # d = 1, scale 63, code 15: 945; dmin = 2^-24 (fp16 0x0001), min 1: w = 945 - 2^-24, which fp32
    # rounds (to nearest even) to 945; a min of 0 leaves 945 exactly.
    codes = [15] * 256
    blk = _q4k_block(0x3C00, 0x0001, [63] * 8, [1] * 8, codes)
    a = np.frombuffer(blk, np.uint8)[None, :]
    w = oracle.dequant(oracle.Q4_K, 1, 256, a)[0]
    assert Fraction(w[0]) == 945 - Fraction(1, 2 ** 24)
    w32 = oracle.dequant_f32(oracle.Q4_K, 1, 256, a)[0]
    assert w32[0] == np.float32(945.0) and np.float32(945.0 - 2.0 ** -24) == np.float32(945.0)


# ----------------------------------------------------------------------------- Q6_K
def _q6k_block(d_bits, scales, codes):
    """One GGUF Q6_K super-block packed from its fields (packing direction, written here from the
    block_q6_K definition): value v = 128h + 32s + l puts its low 4 bits in the low (s < 2) or high
    (s >= 2) nibble of ql[64h + 32 (s & 1) + l] and its high 2 bits at bits 2s of qh[32h + l]."""
    ql, qh = bytearray(128), bytearray(64)
    for v in range(256):
        h, s, l = v // 128, (v % 128) // 32, v % 32
        i = 64 * h + 32 * (s & 1) + l
        ql[i] |= (codes[v] & 15) << (4 if s >= 2 else 0)
        qh[32 * h + l] |= (codes[v] >> 4) << (2 * s)
    return bytes(ql + qh + bytes(int(t) & 0xFF for t in scales) + struct.pack("<H", d_bits))


def test_q6k_dequant_matches_golden():
    lines = read_golden("q6k_block.txt")
    blk = bytearray(210)
    blk[192:208] = bytes(int(t, 16) for t in lines[0].split()[1:])
    blk[208:210] = struct.pack("<H", 0x3C00)
    for t in lines[1].split()[1:]:
        i, v = t.split(":")
        blk[int(i)] = int(v, 16)
    for t in lines[2].split()[1:]:
        i, v = t.split(":")
        blk[128 + int(i)] = int(v, 16)
    w = oracle.dequant(oracle.Q6_K, 1, 256, np.frombuffer(bytes(blk), np.uint8)[None, :])[0]
    for t in lines[3].split()[1:]:
        k, v = t.split(":")
        assert w[int(k)] == float(v), (k, w[int(k)], v)


def test_q6k_packed_fields_decode_exactly():
    # every 6-bit code and every int8 scale value at every position, fp16 d from numpy: the oracle
    # returns d * scale * (code - 32) exactly, and that value is exact in fp32 too
    rng = np.random.default_rng(9)
    for rep in range(32):
        codes = [int(v) for v in (np.arange(256) * 7 + rep) % 64]
        scales = [int(v) for v in ((np.arange(16) * 17 + 8 * rep) % 256) - 128]
        d16 = np.float16(rng.uniform(1e-3, 4.0))
        blk = np.frombuffer(_q6k_block(int(d16.view(np.uint16)), scales, codes), np.uint8)[None, :]
        w = oracle.dequant(oracle.Q6_K, 1, 256, blk)[0]
        for v in range(256):
            h, s, l = v // 128, (v % 128) // 32, v % 32
            ref = Fraction(float(d16)) * scales[8 * h + 2 * s + l // 16] * (codes[v] - 32)
            assert Fraction(w[v]) == ref, (rep, v)
        assert np.array_equal(oracle.dequant_f32(oracle.Q6_K, 1, 256, blk)[0].astype(np.float64), w)


def test_q6k_identity_exact_sum_and_one_hot():
    K = 512
    rows = []
    for n in range(K):
        codes = [32] * K
        codes[n] = 33
        rows.append(b"".join(_q6k_block(0x3C00, [1] * 16, codes[256 * b:256 * (b + 1)]) for b in range(2)))
    blocks = np.frombuffer(b"".join(rows), np.uint8).reshape(K, -1)
    assert blocks.shape[1] == oracle.row_bytes(oracle.Q6_K, K) == 420
    x = synth.activations(2, K, synth.gen(31)).double().numpy()
    y, A = oracle.gemv(oracle.Q6_K, K, K, blocks, x)
    assert np.array_equal(y, x) and np.array_equal(A, np.abs(x))
    N, M = 5, 2
    blocks, _, _ = synth.weights(oracle.Q6_K, N, K, synth.gen(32))
    blocks = blocks.numpy()
    W = oracle.dequant(oracle.Q6_K, N, K, blocks)
    x = synth.activations(M, K, synth.gen(33)).double().numpy()
    y, _ = oracle.gemv(oracle.Q6_K, N, K, blocks, x)
    for m in range(M):
        for n in range(N):
            exact = sum(Fraction(W[n, k]) * Fraction(x[m, k]) for k in range(K))
            absum = sum(abs(Fraction(W[n, k]) * Fraction(x[m, k])) for k in range(K))
            assert abs(Fraction(y[m, n]) - exact) <= Fraction(K * 2.0 ** -52) * absum
    for k in (0, 15, 16, 127, 128, 300, 511):
        e = np.zeros((1, K))
        e[0, k] = 1.0
        assert np.array_equal(oracle.gemv(oracle.Q6_K, N, K, blocks, e)[0][0], W[:, k])


def _identity_mxfp4(K):
    codes, _ = _identity_nvfp4(K)
    return codes, np.full((K, K // 32), 0x7F, np.uint8)  # UE8M0 2^0


FMTS_ALL = [oracle.Q8_0, oracle.Q4_0, oracle.NVFP4, oracle.MXFP4]


@pytest.mark.parametrize("fmt", FMTS_ALL)
def test_gemv_identity_gives_x(fmt):
    K = 96
    x = synth.activations(3, K, synth.gen(1)).double().numpy()
    if fmt == oracle.Q8_0:
        blocks, scales = _identity_q8(K), None
    elif fmt == oracle.Q4_0:
        blocks, scales = _identity_q4(K), None
    elif fmt == oracle.NVFP4:
        blocks, scales = _identity_nvfp4(K)
    else:
        blocks, scales = _identity_mxfp4(K)
    y, A = oracle.gemv(fmt, K, K, blocks, x, scales=scales, g=1.0)
    assert np.array_equal(y, x)
    assert np.array_equal(A, np.abs(x))


@pytest.mark.parametrize("fmt", FMTS_ALL)
def test_gemv_one_hot_selects_a_column(fmt):
    N, K = 40, 64  # N != K so a transposed operand cannot pass
    blocks, scales, g = synth.weights(fmt, N, K, synth.gen(2))
    blocks, scales = blocks.numpy(), None if scales is None else scales.numpy()
    W = oracle.dequant(fmt, N, K, blocks, scales, g)
    for k in (0, 17, 31, 32, 63):
        x = np.zeros((1, K))
        x[0, k] = 1.0
        y, _ = oracle.gemv(fmt, N, K, blocks, x, scales=scales, g=g)
        assert np.array_equal(y[0], W[:, k])


@pytest.mark.parametrize("fmt", FMTS_ALL)
def test_gemv_matches_exact_rational_sum(fmt):
    N, K, M = 5, 64, 3
    blocks, scales, g = synth.weights(fmt, N, K, synth.gen(3))
    blocks, scales = blocks.numpy(), None if scales is None else scales.numpy()
    W = oracle.dequant(fmt, N, K, blocks, scales, g)
    x = synth.activations(M, K, synth.gen(4)).double().numpy()
    y, A = oracle.gemv(fmt, N, K, blocks, x, scales=scales, g=g)
    for m in range(M):
        for n in range(N):
            exact = sum(Fraction(W[n, k]) * Fraction(x[m, k]) for k in range(K))
            absum = sum(abs(Fraction(W[n, k]) * Fraction(x[m, k])) for k in range(K))
            assert abs(Fraction(y[m, n]) - exact) <= Fraction(K * 2.0 ** -52) * absum
            assert abs(Fraction(A[m, n]) - absum) <= Fraction(K * 2.0 ** -52) * absum


def test_gemv_row_subset_matches_full():
    N, K = 33, 128
    blocks, _, _ = synth.weights(oracle.Q4_0, N, K, synth.gen(5))
    x = synth.activations(2, K, synth.gen(6)).double().numpy()
    y, A = oracle.gemv(oracle.Q4_0, N, K, blocks.numpy(), x)
    rows = [32, 0, 7]
    ys, As = oracle.gemv(oracle.Q4_0, N, K, blocks.numpy(), x, rows=rows)
    assert np.array_equal(ys, y[:, rows]) and np.array_equal(As, A[:, rows])


# ----------------------------------------------------------------------------- SiLU gate
def test_silu_matches_torch_and_identities():
    z = np.linspace(-30, 30, 601)
    ref = torch.nn.functional.silu(torch.tensor(z, dtype=torch.float64)).numpy()
    got = np.array([oracle.silu(t) for t in z])
    assert np.allclose(got, ref, rtol=1e-15, atol=1e-300)
    assert oracle.silu(0.0) == 0.0
    for t in (0.3, 2.0, 7.5):  # silu(-z) = silu(z) - z
        assert abs(oracle.silu(-t) - (oracle.silu(t) - t)) < 1e-15 * 10


def test_silu_gate_uses_first_half_as_gate():
    gu = np.array([[1.0, -2.0, 3.0, 5.0]])  # gate = [1, -2], up = [3, 5]
    h, _ = oracle.silu_gate(gu)
    sig = lambda t: 1.0 / (1.0 + math.exp(-t))
    assert np.allclose(h[0], [1.0 * sig(1.0) * 3.0, -2.0 * sig(-2.0) * 5.0], rtol=1e-15)


# ----------------------------------------------------------------------------- routing / MoE
def test_route_matches_stable_sort_and_renormalises():
    logits = synth.router_logits(8, 32, synth.gen(7)).double().numpy()
    ids, wts = oracle.route(logits, 4)
    p = torch.softmax(torch.tensor(logits), dim=1).numpy()
    for m in range(8):
        order = np.argsort(-p[m], kind="stable")[:4]
        assert list(ids[m]) == list(order)
        assert np.allclose(wts[m], p[m, order] / p[m, order].sum(), rtol=1e-14)
        assert abs(wts[m].sum() - 1.0) < 1e-15 * 8


def test_route_tie_goes_to_lower_expert():
    ids, wts = oracle.route(np.zeros((1, 6)), 3)
    assert list(ids[0]) == [0, 1, 2]
    assert np.allclose(wts[0], 1.0 / 3.0)


def _moe_case(fmt, E, H, I, seed):
    gu = [synth.weights(fmt, 2 * I, H, synth.gen(seed + e)) for e in range(E)]
    dn = [synth.weights(fmt, H, I, synth.gen(seed + 100 + e)) for e in range(E)]
    cat = lambda ts, j: None if ts[0][j] is None else np.stack([t[j].numpy() for t in ts])
    return (cat(gu, 0), cat(gu, 1), np.array([t[2] for t in gu], np.float32),
            cat(dn, 0), cat(dn, 1), np.array([t[2] for t in dn], np.float32))


def _mlp(fmt, H, I, gu_b, gu_s, gu_g, dn_b, dn_s, dn_g, x):
    gu, _ = oracle.gemv(fmt, 2 * I, H, gu_b, x, scales=gu_s, g=gu_g)
    h, _ = oracle.silu_gate(gu)
    y, _ = oracle.gemv(fmt, H, I, dn_b, h, scales=dn_s, g=dn_g)
    return y


@pytest.mark.parametrize("fmt", [oracle.Q4_0, oracle.NVFP4])
def test_moe_all_experts_uniform_logits_is_mean(fmt):
    E, H, I = 4, 64, 32
    gub, gus, gug, dnb, dns, dng = _moe_case(fmt, E, H, I, 10)
    x = synth.activations(2, H, synth.gen(11)).double().numpy()
    r = oracle.moe(fmt, E, H, I, E, gub, dnb, np.zeros((2, E)), x, gus, dns, gug, dng)
    mean = sum(_mlp(fmt, H, I, gub[e], None if gus is None else gus[e], gug[e], dnb[e],
                    None if dns is None else dns[e], dng[e], x) for e in range(E)) / E
    assert np.allclose(r["y"], mean, rtol=1e-12, atol=1e-12)
    assert np.allclose(r["wts"], 1.0 / E)


def test_moe_top1_is_dense_mlp_of_argmax():
    fmt, E, H, I = oracle.Q4_0, 5, 64, 32
    gub, gus, gug, dnb, dns, dng = _moe_case(fmt, E, H, I, 20)
    logits = synth.router_logits(3, E, synth.gen(21)).double().numpy()
    x = synth.activations(3, H, synth.gen(22)).double().numpy()
    r = oracle.moe(fmt, E, H, I, 1, gub, dnb, logits, x, gus, dns, gug, dng)
    for m in range(3):
        e = int(np.argmax(logits[m]))
        ref = _mlp(fmt, H, I, gub[e], None, 1.0, dnb[e], None, 1.0, x[m:m + 1])
        assert r["ids"][m, 0] == e and r["wts"][m, 0] == 1.0
        assert np.array_equal(r["y"][m], ref[0])


def test_moe_identical_experts_is_dense_and_permutation_invariant():
    fmt, E, H, I = oracle.Q4_0, 6, 64, 32
    gub, gus, gug, dnb, dns, dng = _moe_case(fmt, E, H, I, 30)
    logits = synth.router_logits(2, E, synth.gen(31)).double().numpy()
    x = synth.activations(2, H, synth.gen(32)).double().numpy()
    same = oracle.moe(fmt, E, H, I, 3, np.stack([gub[0]] * E), np.stack([dnb[0]] * E), logits, x)
    dense = _mlp(fmt, H, I, gub[0], None, 1.0, dnb[0], None, 1.0, x)
    assert np.allclose(same["y"], dense, rtol=1e-12, atol=1e-12)
    perm = np.array([3, 5, 0, 1, 4, 2])
    a = oracle.moe(fmt, E, H, I, 3, gub, dnb, logits, x)
    b = oracle.moe(fmt, E, H, I, 3, gub[perm], dnb[perm], logits[:, perm], x)
    # the softmax denominator is summed in a different order, so equal up to fp64 rounding
    assert np.allclose(a["y"], b["y"], rtol=1e-13, atol=1e-16)
    assert np.array_equal(perm[b["ids"]], a["ids"])


# ----------------------------------------------------------------------------- NVFP4 act quant
def test_round_e2m1_golden_ties_and_nearest():
    for line in read_golden("e2m1_ties.txt"):
        v, c = line.split()
        assert oracle.round_e2m1(float(v)) == int(c, 16), (v, c)
    grid = [oracle.e2m1(c) for c in range(8)]
    rng = np.random.default_rng(0)
    for v in rng.uniform(-8, 8, 2000).astype(np.float32):
        c = oracle.round_e2m1(float(v))
        got = oracle.e2m1(c)
        if abs(v) < 6:
            assert all(abs(abs(v) - abs(got)) <= abs(abs(v) - t) for t in grid)
        assert (c >> 3) == (1 if v < 0 else 0)
    for c in range(16):  # every grid value round-trips
        assert oracle.round_e2m1(oracle.e2m1(c)) == c


def test_round_e4m3_matches_torch():
    rng = np.random.default_rng(1)
    vals = np.concatenate([rng.uniform(0, 448, 3000), np.exp(rng.uniform(-12, 6, 3000))])
    vals = vals[vals <= 448].astype(np.float32)
    # midpoints between consecutive codes: exact ties
    pos = [oracle.e4m3(c) for c in range(0x7F)]
    mids = np.array([(a + b) / 2 for a, b in zip(pos[:-1], pos[1:])], np.float32)
    allv = np.concatenate([vals, mids])
    ref = torch.tensor(allv).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.round_e4m3(float(v)) for v in allv], np.uint8)
    assert np.array_equal(got, ref)
    assert oracle.round_e4m3(1000.0) == 0x7E and oracle.round_e4m3(0.0) == 0


def test_act_quant_grid_values_are_exact():
    grid = [0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0, -6.0, -0.5, 0.0, 1.0, -1.5, 2.0, -3.0, 4.0, 6.0]
    X = np.array([grid], np.float32)
    codes, scales, ag = oracle.act_quant(X)
    assert scales[0, 0] == 0x7E  # amax_b / (6 a_g) = 448 exactly after rounding
    dec = [oracle.e2m1((codes[0, j // 2] >> (4 * (j & 1))) & 0xF) for j in range(16)]
    assert dec == grid
    assert ag == np.float32(np.float32(6.0) / np.float32(6.0 * 448.0))


def test_act_quant_error_bound_and_zero_tensor():
    X = synth.activations(3, 64, synth.gen(40), dtype=torch.bfloat16).float().numpy()
    codes, scales, ag = oracle.act_quant(X)
    Aq = oracle.dequant(oracle.NVFP4, 3, 64, codes, scales, ag)
    for m in range(3):
        for b in range(4):
            s = oracle.e4m3(int(scales[m, b])) * ag
            blk = X[m, 16 * b:16 * b + 16].astype(np.float64)
            # inside the E2M1 range the error is at most half of the largest grid step (1.0)
            assert np.all(np.abs(blk - Aq[m, 16 * b:16 * b + 16]) <= 1.0 * s * (1 + 1e-6))
    z_codes, z_scales, z_ag = oracle.act_quant(np.zeros((2, 32), np.float32))
    assert z_ag == 0.0 and not z_codes.any() and not z_scales.any()


# ----------------------------------------------------------------------------- MXFP4 act quant
E2M1_MAG = [Fraction(0), Fraction(1, 2), Fraction(1), Fraction(3, 2), Fraction(2), Fraction(3), Fraction(4),
            Fraction(6)]


def _mx_decode(codes, scales, m, j):
    c = (int(codes[m, j // 2]) >> (4 * (j & 1))) & 0xF
    return c, int(scales[m, j // 32])


def test_act_quant_mx_scale_puts_the_block_max_in_the_top_binade():
    """OCP MX: X = 2^(floor(log2 amax) - emax_elem) with emax_elem = 2 for E2M1, so amax / X lies
    in [4, 8) -- the binade of E2M1's 4 and 6 -- for every block not clamped at the UE8M0 range."""
    rng = np.random.default_rng(11)
    X = (rng.standard_normal((4, 256)) * np.exp2(rng.integers(-30, 30, (4, 1)))).astype(np.float32)
    X = torch.tensor(X).to(torch.bfloat16).float().numpy()
    codes, scales = oracle.act_quant_mx(X)
    for m in range(4):
        for b in range(8):
            amax = Fraction(float(np.max(np.abs(X[m, 32 * b:32 * b + 32].astype(np.float64)))))
            Xs = Fraction(2) ** (int(scales[m, b]) - 127)
            assert 4 <= amax / Xs < 8, (m, b, scales[m, b])


def test_act_quant_mx_codes_are_nearest_ties_even_saturating():
    """Every code is the E2M1 value nearest to x / X in exact arithmetic (ties to the even code),
    with magnitudes from 6 up to 8 saturating to 6 and the sign kept."""
    rng = np.random.default_rng(12)
    X = (rng.standard_normal((3, 128)) * 3).astype(np.float32)
    X[0, :32] = np.linspace(-8, 8, 32)  # block max 8: scale 2^1, every grid point and midpoint region
    # block max 6 (scale 2^0) holding every midpoint between E2M1 magnitudes: exact ties
    X[1, :32] = [6.0, 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, -0.25, -0.75, -1.25, -1.75, -2.5, -3.5, -5.0,
                 7.0, -7.5] + [0.0] * 15
    X = torch.tensor(X).to(torch.bfloat16).float().numpy()
    codes, scales = oracle.act_quant_mx(X)
    for m in range(3):
        for j in range(128):
            c, byte = _mx_decode(codes, scales, m, j)
            q = Fraction(float(X[m, j])) / Fraction(2) ** (byte - 127)
            a = abs(q)
            dists = [abs(a - v) for v in E2M1_MAG]
            best = min(range(8), key=lambda i: (dists[i], i % 2))  # nearest, then even code
            if a >= 6:
                best = 7
            assert (c & 7) == best, (m, j, float(q), c)
            assert (c >> 3) == (1 if math.copysign(1.0, float(X[m, j])) < 0 else 0)


def test_act_quant_mx_grid_round_trip_and_special_blocks():
    grid = [0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0, -6.0] * 4  # block max 6: scale 2^0 (byte 127)
    X = np.array([grid + [v * 2.0 ** -20 for v in grid]], np.float32)
    codes, scales = oracle.act_quant_mx(X)
    assert list(scales[0]) == [127, 107]
    for j in range(64):
        c, byte = _mx_decode(codes, scales, 0, j)
        val = float(E2M1_MAG[c & 7]) * (-1 if c & 8 else 1) * 2.0 ** (byte - 127)
        assert val == X[0, j], j
    # an all-zero block: byte 0 and zero codes; negative zero keeps its sign (code 8)
    Z = np.zeros((1, 32), np.float32)
    Z[0, 3] = -0.0
    zc, zs = oracle.act_quant_mx(Z)
    assert zs[0, 0] == 0 and (int(zc[0, 1]) >> 4) == 8 and int(zc[0, 0]) == 0
    # a block below 2^-125 clamps to byte 0 (X = 2^-127): 2^-130 * 4.5 -> x / X = 0.5625 -> code 1
    T = np.zeros((1, 32), np.float32)
    T[0, 0] = np.float32(4.5 * 2.0 ** -130)
    tc, ts = oracle.act_quant_mx(T)
    assert ts[0, 0] == 0 and (int(tc[0, 0]) & 0xF) == 1
    # the largest finite bf16 block: floor(log2(3.39e38)) - 2 = 125 -> byte 252
    B = np.zeros((1, 32), np.float32)
    B[0, 5] = torch.tensor(3.3895314e38).to(torch.bfloat16).float().item()
    bc, bs = oracle.act_quant_mx(B)
    assert bs[0, 0] == 252
    # a block holding an infinity: the UE8M0 NaN byte and zero codes
    I = np.ones((1, 32), np.float32)
    I[0, 7] = np.inf
    ic, isc = oracle.act_quant_mx(I)
    assert isc[0, 0] == 0xFF and not ic.any()


# ----------------------------------------------------------------------------- same-quant products
def _fp4_value(codes, r, j):
    c = (int(codes[r, j // 2]) >> (4 * (j & 1))) & 0xF
    return -E2M1_MAG[c & 7] if c & 8 else E2M1_MAG[c & 7]


def _e4m3_fraction(b):
    return Fraction(torch.tensor([b], dtype=torch.uint8).view(torch.float8_e4m3fn).double().item())


@pytest.mark.parametrize("mx", [False, True])
def test_gemm_same_quant_is_the_exact_product_of_the_decoded_operands(mx):
    """y[m][n] = sum_k a[m][k] w[n][k], both operands decoded here from their codes by the format
    definitions (E2M1 table, E4M3 through torch's float8, UE8M0 as a power of two), in exact
    arithmetic.  M, N and K differ, so a transposed operand, a scale applied to the wrong row or a
    block index off by one fails."""
    M, N, K = 3, 5, 96
    rng = np.random.default_rng(21 + mx)
    bs = 32 if mx else 16
    a_codes = rng.integers(0, 256, (M, K // 2), dtype=np.uint8)
    w_codes = rng.integers(0, 256, (N, K // 2), dtype=np.uint8)
    if mx:
        a_sc = rng.integers(118, 136, (M, K // bs), dtype=np.uint8)
        w_sc = rng.integers(118, 136, (N, K // bs), dtype=np.uint8)
        y, A = oracle.gemm_same_quant_mx(w_codes, w_sc, a_codes, a_sc, N, K)
        scale = lambda b: Fraction(2) ** (int(b) - 127)
        a_g = w_g = Fraction(1)
    else:
        a_sc = rng.integers(0x08, 0x7F, (M, K // bs), dtype=np.uint8)   # finite E4M3, no NaN
        w_sc = rng.integers(0x08, 0x7F, (N, K // bs), dtype=np.uint8)
        ag, wg = float(np.float32(1 / 448)), float(np.float32(3 / 1000))
        y, A = oracle.gemm_same_quant(w_codes, w_sc, wg, a_codes, a_sc, ag, N, K)
        scale = _e4m3_fraction
        a_g, w_g = Fraction(ag), Fraction(wg)
    assert y.shape == (M, N) and A.shape == (M, N)
    for m in range(M):
        for n in range(N):
            terms = [_fp4_value(a_codes, m, k) * scale(a_sc[m, k // bs]) * a_g *
                     _fp4_value(w_codes, n, k) * scale(w_sc[n, k // bs]) * w_g for k in range(K)]
            exact, absum = sum(terms), sum(abs(t) for t in terms)
            assert abs(Fraction(float(y[m, n])) - exact) <= Fraction(K * 2.0 ** -52) * absum, (m, n)
            assert abs(Fraction(float(A[m, n])) - absum) <= Fraction(K * 2.0 ** -52) * absum, (m, n)
