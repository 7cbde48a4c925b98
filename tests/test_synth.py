"""The seeded input generators produce what the input recipe states (CPU only): canonical byte
layouts and sizes, scale ranges after their fp16 / E4M3 / UE8M0 rounding, every code value in use,
N(0,1) activations and logits, and the same bytes for the same seed."""
import numpy as np
import pytest
import torch

import synth


def fp16_of(blocks, nbytes, off):
    """The fp16 field at byte offset `off` of every nbytes-long block."""
    b = blocks.reshape(-1, nbytes)[:, off:off + 2].contiguous()
    return b.view(torch.float16).float().flatten()


def test_q8_0_layout_scales_and_codes():
    N, K = 64, 256
    t = synth.q8_0(N, K, synth.gen(1))
    assert t.dtype == torch.uint8 and t.shape == (N, K // 32 * 34)
    d = fp16_of(t, 34, 0)
    assert d.min() >= 1e-3 * (1 - 2 ** -11) and d.max() <= 1e-2 * (1 + 2 ** -11)
    q = t.reshape(-1, 34)[:, 2:].contiguous().view(torch.int8)
    assert int(q.min()) == -127 and int(q.max()) == 127  # the full range, never -128 by default


def test_q4_0_layout_scales_and_nibbles():
    N, K = 64, 256
    t = synth.q4_0(N, K, synth.gen(2))
    assert t.shape == (N, K // 32 * 18)
    d = fp16_of(t, 18, 0)
    assert d.min() >= 1e-3 * (1 - 2 ** -11) and d.max() <= 2e-2 * (1 + 2 ** -11)
    qs = t.reshape(-1, 18)[:, 2:]
    nib = torch.cat([qs & 15, qs >> 4]).flatten()
    assert set(nib.tolist()) == set(range(16))


def test_nvfp4_scales_codes_and_tensor_scale():
    N, K = 64, 512
    codes, scales, g = synth.nvfp4(N, K, synth.gen(3))
    assert codes.shape == (N, K // 2) and scales.shape == (N, K // 16)
    s = scales.view(torch.float8_e4m3fn).float()
    assert s.min() >= 0.5 and s.max() <= 448.0 and not torch.isnan(s).any()
    nib = torch.cat([codes & 15, codes >> 4]).flatten()
    assert set(nib.tolist()) == set(range(16))
    assert g == float(np.float32(1.0 / 448.0))


def test_mxfp4_scale_bytes_and_codes():
    N, K = 64, 512
    codes, scales, g = synth.mxfp4(N, K, synth.gen(4))
    assert codes.shape == (N, K // 2) and scales.shape == (N, K // 32) and g == 1.0
    assert int(scales.min()) == 118 and int(scales.max()) == 130


def test_k_quant_layouts():
    N, K = 32, 512
    t4 = synth.q4_k(N, K, synth.gen(5))
    assert t4.shape == (N, K // 256 * 144)
    d = fp16_of(t4, 144, 0)
    dmin = fp16_of(t4, 144, 2)
    for v in (d, dmin):
        assert v.min() >= 2e-4 * (1 - 2 ** -11) and v.max() <= 2e-3 * (1 + 2 ** -11)
    t6 = synth.q6_k(N, K, synth.gen(6))
    assert t6.shape == (N, K // 256 * 210)
    d6 = fp16_of(t6, 210, 208)  # d is the last field of the 210-byte block
    assert d6.min() >= 2e-5 * (1 - 2 ** -11) and d6.max() <= 2e-4 * (1 + 2 ** -11)


def test_activations_and_logits_are_standard_normal():
    x = synth.activations(64, 4096, synth.gen(7))
    assert x.dtype == torch.float32
    assert abs(float(x.mean())) < 0.01 and abs(float(x.std()) - 1.0) < 0.01
    xb = synth.activations(4, 256, synth.gen(7), dtype=torch.bfloat16)
    assert xb.dtype == torch.bfloat16
    assert torch.equal(xb, synth.activations(4, 256, synth.gen(7)).to(torch.bfloat16))
    lg = synth.router_logits(512, 32, synth.gen(8))
    assert lg.shape == (512, 32) and abs(float(lg.mean())) < 0.02 and abs(float(lg.std()) - 1.0) < 0.02


@pytest.mark.parametrize("fmt", [synth.Q8_0, synth.Q4_0, synth.NVFP4, synth.MXFP4, synth.Q4_K, synth.Q6_K])
def test_same_seed_same_bytes(fmt):
    a = synth.weights(fmt, 32, 256, synth.gen(11))
    b = synth.weights(fmt, 32, 256, synth.gen(11))
    c = synth.weights(fmt, 32, 256, synth.gen(12))
    assert torch.equal(a[0], b[0]) and not torch.equal(a[0], c[0])
    if a[1] is not None:
        assert torch.equal(a[1], b[1])
    assert synth.seed_for(2, 3, 4) == 2034
