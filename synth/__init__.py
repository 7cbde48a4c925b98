"""Seeded synthetic inputs shared by the tests, the smoke check and the bench.

This module only draws random numbers and lays them out in the canonical storage formats
(GGUF Q8_0 / Q4_0 blocks, NVFP4 / MXFP4 code and scale planes); it holds none of the layer's arithmetic.
Rounding of drawn reals to fp16 / bf16 / E4M3 storage uses torch's own conversions
(round-to-nearest-even).

Canonical layouts (the public conventions; the pages name the formats but not their bytes):
  Q8_0  one row = K/32 blocks of 34 bytes: fp16 scale d (little endian), then 32 int8 codes
  Q4_0  one row = K/32 blocks of 18 bytes: fp16 scale d, then 16 bytes; byte j holds element j
        in its low nibble and element j+16 in its high nibble
  NVFP4 codes [N][K/2] (byte i = element 2i low nibble, 2i+1 high nibble), E4M3 scales [N][K/16],
        one fp32 per-tensor scale
  MXFP4 codes as NVFP4, UE8M0 scale bytes [N][K/32] (one per 32 values), no per-tensor scale
  Q4_K  one row = K/256 super-blocks of 144 bytes: fp16 d, fp16 dmin, 12 bytes of packed 6-bit
        sub-block scales and mins, 128 bytes of 4-bit codes (GGUF block_q4_K)
  Q6_K  one row = K/256 super-blocks of 210 bytes: ql[128] (low code bits), qh[64] (high 2 bits),
        int8 scales[16] (one per 16 values), fp16 d (GGUF block_q6_K)

Workload recipes (seeded; shapes from the synthetic layer stacks the bench and tests use):
  Q8_0:  codes uniform over [-127, 127], scale uniform real in [1e-3, 1e-2] rounded to fp16
  Q4_0:  4-bit codes uniform over 0..15 (value = code - 8), scale uniform real in [1e-3, 2e-2]
  NVFP4: codes uniform over all 16, E4M3 scales uniform real in [0.5, 448] rounded to E4M3,
         per-tensor scale fp32(1/448)
  MXFP4: codes uniform over all 16, scale bytes uniform integers in [118, 130] (2^-9 .. 2^3)
  Q4_K:  d and dmin uniform real in [2e-4, 2e-3] rounded to fp16; the 12 scale bytes and the
         128 code bytes uniform over 0..255 (every byte pattern is a valid encoding: sub-block
         scales and mins uniform over 0..63, codes uniform over 0..15)
  Q6_K:  code bytes (ql, qh) and int8 scales uniform over all byte values (6-bit codes uniform
         over 0..63), d uniform real in [2e-5, 2e-4] rounded to fp16
  activations N(0, 1) (fp32, or fp32 draws rounded to bf16); router logits N(0, 1)
"""
from __future__ import annotations

import torch

Q8_0, Q4_0, NVFP4, MXFP4, Q4_K, Q6_K = 1, 2, 3, 4, 5, 6
FMT_NAMES = {Q8_0: "q8_0", Q4_0: "q4_0", NVFP4: "nvfp4", MXFP4: "mxfp4", Q4_K: "q4_k", Q6_K: "q6_k"}
NVFP4_G = float(torch.tensor(1.0 / 448.0, dtype=torch.float32))


def gen(seed: int, device="cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def seed_for(config: int, layer: int = 0, tensor: int = 0) -> int:
    """Per-tensor seed: config id * 1000 + layer * 10 + tensor index."""
    return config * 1000 + layer * 10 + tensor


def _fp16_bytes(vals: torch.Tensor) -> torch.Tensor:
    return vals.to(torch.float16).contiguous().view(torch.uint8).reshape(*vals.shape, 2)


def q8_0(N, K, g, device="cpu", d_range=(1e-3, 1e-2), q_range=(-127, 127)):
    """Canonical Q8_0 tensor, uint8 [N, K/32*34]."""
    assert K % 32 == 0
    nb = K // 32
    d = torch.empty(N, nb, dtype=torch.float32, device=device).uniform_(*d_range, generator=g)
    q = torch.randint(q_range[0], q_range[1] + 1, (N, nb, 32), generator=g, device=device,
                      dtype=torch.int16).to(torch.int8).view(torch.uint8)
    return torch.cat([_fp16_bytes(d), q], dim=2).reshape(N, nb * 34).contiguous()


def q4_0(N, K, g, device="cpu", d_range=(1e-3, 2e-2)):
    """Canonical Q4_0 tensor, uint8 [N, K/32*18]."""
    assert K % 32 == 0
    nb = K // 32
    d = torch.empty(N, nb, dtype=torch.float32, device=device).uniform_(*d_range, generator=g)
    qs = torch.randint(0, 256, (N, nb, 16), generator=g, device=device,
                       dtype=torch.int16).to(torch.uint8)
    return torch.cat([_fp16_bytes(d), qs], dim=2).reshape(N, nb * 18).contiguous()


def q4_k(N, K, g, device="cpu", d_range=(2e-4, 2e-3)):
    """Canonical Q4_K tensor, uint8 [N, K/256*144]."""
    assert K % 256 == 0
    nb = K // 256
    d = torch.empty(N, nb, 2, dtype=torch.float32, device=device).uniform_(*d_range, generator=g)
    rest = torch.randint(0, 256, (N, nb, 140), generator=g, device=device, dtype=torch.int16).to(torch.uint8)
    return torch.cat([_fp16_bytes(d).reshape(N, nb, 4), rest], dim=2).reshape(N, nb * 144).contiguous()


def q6_k(N, K, g, device="cpu", d_range=(2e-5, 2e-4)):
    """Canonical Q6_K tensor, uint8 [N, K/256*210]."""
    assert K % 256 == 0
    nb = K // 256
    rest = torch.randint(0, 256, (N, nb, 208), generator=g, device=device, dtype=torch.int16).to(torch.uint8)
    d = torch.empty(N, nb, dtype=torch.float32, device=device).uniform_(*d_range, generator=g)
    return torch.cat([rest, _fp16_bytes(d)], dim=2).reshape(N, nb * 210).contiguous()


def nvfp4(N, K, g, device="cpu", s_range=(0.5, 448.0)):
    """Canonical NVFP4 tensor: (codes uint8 [N, K/2], scales uint8 [N, K/16], fp32 tensor scale)."""
    assert K % 16 == 0
    codes = torch.randint(0, 256, (N, K // 2), generator=g, device=device,
                          dtype=torch.int16).to(torch.uint8)
    s = torch.empty(N, K // 16, dtype=torch.float32, device=device).uniform_(*s_range, generator=g)
    scales = s.to(torch.float8_e4m3fn).view(torch.uint8).contiguous()
    return codes.contiguous(), scales, NVFP4_G


def mxfp4(N, K, g, device="cpu", e_range=(118, 130)):
    """Canonical MXFP4 tensor: (codes uint8 [N, K/2], UE8M0 scale bytes [N, K/32], 1.0).
    Codes uniform over all 16; scale bytes uniform integers in e_range (2^-9 .. 2^3)."""
    assert K % 32 == 0
    codes = torch.randint(0, 256, (N, K // 2), generator=g, device=device,
                          dtype=torch.int16).to(torch.uint8)
    scales = torch.randint(e_range[0], e_range[1] + 1, (N, K // 32), generator=g, device=device,
                           dtype=torch.int16).to(torch.uint8)
    return codes.contiguous(), scales.contiguous(), 1.0


def weights(fmt, N, K, g, device="cpu"):
    """Canonical tensor of the given format: (blocks, scales or None, per-tensor scale)."""
    if fmt == Q8_0:
        return q8_0(N, K, g, device), None, 1.0
    if fmt == Q4_0:
        return q4_0(N, K, g, device), None, 1.0
    if fmt == MXFP4:
        return mxfp4(N, K, g, device=device)
    if fmt == NVFP4:
        return nvfp4(N, K, g, device)
    if fmt == Q4_K:
        return q4_k(N, K, g, device), None, 1.0
    if fmt == Q6_K:
        return q6_k(N, K, g, device), None, 1.0
    raise ValueError(fmt)


def activations(M, K, g, dtype=torch.float32, device="cpu"):
    """N(0,1) activations; bf16 rows are fp32 draws rounded to bf16."""
    x = torch.randn(M, K, generator=g, dtype=torch.float32, device=device)
    return x.to(dtype).contiguous()


def router_logits(M, E, g, device="cpu"):
    return torch.randn(M, E, generator=g, dtype=torch.float32, device=device)
