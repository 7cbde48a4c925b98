"""The MMA-only FP4 rate probe (qlin_probe_fp4_mma): every SM's CTA runs its MMAs to completion,
reports a positive clock span and a clean status word, and the rate it implies lies between a
fraction of and the B200's dense FP4 figure (9 PFLOP/s) with some margin for clocks above the
base.  It is a measurement aid; the bench prints it beside that figure."""
import pytest
import torch

import gemm_dequant_gemv_q8_b200 as q

pytestmark = pytest.mark.gpu

FLOP_PER_MMA = 2 * 128 * 256 * 64


def test_probe_fp4_mma_runs_on_every_sm_and_reports_a_plausible_rate():
    cycles = torch.zeros(1024, dtype=torch.int64, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    iters = 4096
    q.qlin_probe_fp4_mma(iters, cycles, status)  # warm-up
    cycles.zero_()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    ctas = q.qlin_probe_fp4_mma(iters, cycles, status)
    e.record()
    torch.cuda.synchronize()
    assert ctas == torch.cuda.get_device_properties(0).multi_processor_count
    assert int(status.item()) == 0
    c = cycles[:ctas].cpu()
    assert (c > 0).all() and not cycles[ctas:].any()
    per_mma = float(c.max()) / iters
    assert 32 <= per_mma <= 4096, per_mma  # the tensor pipe's issue rate, in SM cycles
    tflops = FLOP_PER_MMA * iters * ctas / (s.elapsed_time(e) * 1e-3) / 1e12
    assert 500 < tflops < 12000, tflops


def test_probe_fp4_mma_rejects_too_small_a_cycles_array():
    cycles = torch.zeros(8, dtype=torch.int64, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    with pytest.raises(q.QlinError) as ei:
        q.qlin_probe_fp4_mma(64, cycles, status)
    assert ei.value.status == 1
    torch.cuda.synchronize()
    assert not cycles.any() and int(status.item()) == 0
