"""The bench's workload at full size, in the launch configurations bench.py times (graph-captured;
one persistent GEMV chain per step, one chain per layer, or one launch per projection with PDL
between kernels): sampled outputs of every projection checked one by one against the oracle."""
import numpy as np
import pytest
import torch

import bench
import oracle
import synth

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("mode,pdl,dataflow", [("chain", True, "stated"), ("chain", False, "stated"),
                                               ("chain", True, "serial"), ("layer_chain", True, "stated"),
                                               ("layer_chain", True, "serial"), ("launches", True, "stated"),
                                               ("launches", False, "serial")])
def test_stack_sampled_outputs_match_oracle(mode, pdl, dataflow):
    fmt, layers = synth.Q4_0, 2
    st = bench.DenseStack(fmt, layers, mode=mode, dataflow=dataflow)
    g = st.capture(pdl=pdl)
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    rng = np.random.default_rng(5)
    for l in range(layers):
        for pi, (name, N, K, epi) in enumerate(bench.STACK):
            blocks, scales, gs = synth.weights(fmt, N, K, synth.gen(synth.seed_for(2, l, pi), device="cuda"),
                                               device="cuda")
            x = st.x[(l, pi)].double().cpu().numpy()
            y = st.y[(l, pi)].double().cpu().numpy()
            ncols = N // 2 if epi else N
            cols = np.unique(np.concatenate([[0, ncols - 1], rng.integers(0, ncols, 40)]))
            if epi:
                rows = np.concatenate([cols, cols + N // 2])
                sel = blocks[torch.as_tensor(rows, device="cuda")].cpu().numpy()
                gu, Agu = oracle.gemv(fmt, len(rows), K, sel, x)
                n = len(cols)
                gu2 = np.concatenate([gu[:, :n], gu[:, n:]], axis=1)
                A2 = np.concatenate([Agu[:, :n], Agu[:, n:]], axis=1)
                href, Ah = oracle.silu_gate(gu2, A2)
                tol = 2e-6 * Ah + 8 * 2.0 ** -24 * np.abs(href) + 4 * 2.0 ** -126 * (1 + np.abs(gu[:, n:]))
                assert (np.abs(y[:, cols] - href) <= tol).all(), (l, name)
            else:
                sel = blocks[torch.as_tensor(cols, device="cuda")].cpu().numpy()
                yref, A = oracle.gemv(fmt, len(cols), K, sel, x)
                assert (np.abs(y[:, cols] - yref) <= 2e-6 * A).all(), (l, name)
    del g
