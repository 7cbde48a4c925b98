"""GPU parity of qlin_gemv_chain: every op of a chain against the fp64 oracle.

The bars are qlin_gemv's: y within 2e-6 * sum_k |w*x| (fp32 products and sums), the SiLU-gate
epilogue within the propagated bound.  An op whose activations are the output of an earlier op
of the same launch is checked against the oracle applied to the activations that op actually
read (the earlier op's GPU output): the check is of the op, and of the wait that makes it read a
finished input.  Chains also run twice and must give identical bits, with a clean status word.
"""
import numpy as np
import pytest
import torch

import gemm_dequant_gemv_q8_b200 as q
import oracle
import synth

pytestmark = pytest.mark.gpu
FMTS = [q.QLIN_Q8_0, q.QLIN_Q4_0, q.QLIN_NVFP4, q.QLIN_MXFP4]
TOL = 2e-6


class Op:
    def __init__(self, fmt, N, K, M, seed, epi=q.QLIN_EPI_NONE, x=None, wait_for=-1, xdt=torch.float32):
        pf = q.QLIN_PACK_GATE_UP if (epi & 0xF) == q.QLIN_EPI_SILU_GATE else q.QLIN_PACK_DEFAULT
        blocks, scales, g = synth.weights(fmt, N, K, synth.gen(seed))
        self.packed = q.qlin_pack_weights(fmt, N, K, blocks.cuda(), None if scales is None else scales.cuda(), g, pf)
        self.blocks, self.scales, self.g = blocks.numpy(), None if scales is None else scales.numpy(), g
        self.fmt, self.N, self.K, self.epi, self.wait_for = fmt, N, K, epi, wait_for
        self.x = x if x is not None else synth.activations(M, K, synth.gen(seed + 1), dtype=xdt).cuda()
        ncols = N // 2 if (epi & 0xF) == q.QLIN_EPI_SILU_GATE else N
        ydt = torch.bfloat16 if epi & q.QLIN_OUT_BF16 else torch.float32
        self.y = torch.full((M, ncols), float("nan"), device="cuda", dtype=ydt)

    def op(self):
        return q.gemv_op(self.packed, self.N, self.K, self.x, self.y, self.epi, self.wait_for)

    def check(self):
        x = self.x.double().cpu().numpy()
        y = self.y.double().cpu().numpy()
        ref, A = oracle.gemv(self.fmt, self.N, self.K, self.blocks, x, scales=self.scales, g=self.g)
        if (self.epi & 0xF) == q.QLIN_EPI_SILU_GATE:
            href, Ah = oracle.silu_gate(ref, A)
            tol = TOL * Ah + 8 * 2.0 ** -24 * np.abs(href) + 4 * 2.0 ** -126 * (1 + np.abs(ref[:, self.N // 2:]))
            err = np.abs(y - href)
        else:
            tol, err = TOL * A, np.abs(y - ref)
            href = ref
        if self.epi & q.QLIN_OUT_BF16:  # one rounding to bf16 (8 significant bits): half an ulp
            tol = tol + 2.0 ** -8 * np.abs(href) + 2.0 ** -133
        assert (err <= tol).all(), (self.N, self.K, float(np.max(err / np.maximum(tol, 1e-300))))


def run(fmt, xdt, M, ops, ws=None):
    return q.qlin_gemv_chain(fmt, q.QLIN_F32 if xdt == torch.float32 else q.QLIN_BF16, M,
                             [o.op() for o in ops], ws=ws)


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("M", [1, 3])
def test_chain_mixed_with_dependencies(fmt, M):
    A = Op(fmt, 200, 1280, M, 10)
    B = Op(fmt, 2 * 96, 544, M, 20, epi=q.QLIN_EPI_SILU_GATE)
    C = Op(fmt, 160, 96, M, 30, x=B.y, wait_for=1)          # reads B's SiLU output
    D = Op(fmt, 33, 160, M, 40, x=C.y, wait_for=2)          # reads C's output
    E = Op(fmt, 1024, 2560, M, 50)
    ops = [A, B, C, D, E]
    ws = run(fmt, torch.float32, M, ops)
    torch.cuda.synchronize()
    assert q.qlin_ws_status(ws) == 0
    for o in ops:
        o.check()


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("M", [1, 2, 4, 8])
def test_chain_bf16_activations(fmt, M):
    ops = [Op(fmt, N, K, M, 60 + i, xdt=torch.bfloat16) for i, (N, K) in
           enumerate([(256, 512), (96, 2560), (520, 272 if fmt == q.QLIN_NVFP4 else 288), (64, 4096)])]
    ws = run(fmt, torch.bfloat16, M, ops)
    torch.cuda.synchronize()
    assert q.qlin_ws_status(ws) == 0
    for o in ops:
        o.check()


@pytest.mark.parametrize("fmt", [q.QLIN_Q4_K, q.QLIN_Q6_K])
@pytest.mark.parametrize("M", [1, 2, 4, 8])
@pytest.mark.parametrize("xdt", [torch.float32, torch.bfloat16])
def test_chain_kquant_mlp_with_dependencies(fmt, M, xdt):
    """K-quants (K a multiple of 256): two gated MLP layers plus an independent projection; down
    reads its layer's SiLU output, the second layer's gate_up reads the first layer's down.  With
    bf16 activations every op writes bf16 (the next op's input)."""
    ob = q.QLIN_OUT_BF16 if xdt == torch.bfloat16 else 0
    ops = []
    x = synth.activations(M, 1024, synth.gen(300), dtype=xdt).cuda()
    for l in range(2):
        gu = Op(fmt, 2 * 512, 1024, M, 310 + l, epi=q.QLIN_EPI_SILU_GATE | ob, x=x,
                wait_for=-1 if l == 0 else len(ops) - 1, xdt=xdt)
        ops.append(gu)
        dn = Op(fmt, 1024, 512, M, 320 + l, epi=ob, x=gu.y, wait_for=len(ops) - 1, xdt=xdt)
        ops.append(dn)
        x = dn.y
    ops.append(Op(fmt, 200, 2560, M, 330, xdt=xdt))
    ws = run(fmt, xdt, M, ops)
    torch.cuda.synchronize()
    assert q.qlin_ws_status(ws) == 0
    for o in ops:
        o.check()


def test_chain_serial_dependencies_and_reuse():
    """Eight ops, each reading the previous op's output; the same workspace is used three times
    (its counters must come back to zero) and the three runs agree bit for bit."""
    fmt, M, n = q.QLIN_Q4_0, 2, 512
    x0 = synth.activations(M, n, synth.gen(70)).cuda()
    ops = []
    for i in range(8):
        ops.append(Op(fmt, n, n, M, 80 + i, x=x0 if i == 0 else ops[-1].y, wait_for=i - 1))
    ws = run(fmt, torch.float32, M, ops)
    outs = [o.y.clone() for o in ops]
    for _ in range(2):
        for o in ops:
            o.y.fill_(float("nan"))
        run(fmt, torch.float32, M, ops, ws=ws)
        torch.cuda.synchronize()
        for o, y0 in zip(ops, outs):
            assert torch.equal(o.y, y0)
    assert q.qlin_ws_status(ws) == 0
    for o in ops:
        o.check()


def test_chain_many_ops_stack_shapes():
    """Two layers of the 4B stack shapes plus small ops (12 ops), Q4_0, M = 1: rotation of the
    extra units across ops, ops smaller than the grid, down reading gate_up's output."""
    fmt, M = q.QLIN_Q4_0, 1
    ops = []
    for l in range(2):
        ops.append(Op(fmt, 6144, 2560, M, 100 + 10 * l))
        ops.append(Op(fmt, 2560, 4096, M, 101 + 10 * l))
        gu = Op(fmt, 2 * 9728, 2560, M, 102 + 10 * l, epi=q.QLIN_EPI_SILU_GATE)
        ops.append(gu)
        ops.append(Op(fmt, 2560, 9728, M, 103 + 10 * l, x=gu.y, wait_for=len(ops) - 1))
        ops.append(Op(fmt, 32, 256, M, 104 + 10 * l))
        ops.append(Op(fmt, 1, 32, M, 105 + 10 * l))
    ws = run(fmt, torch.float32, M, ops)
    torch.cuda.synchronize()
    assert q.qlin_ws_status(ws) == 0
    rng = np.random.default_rng(3)
    for o in ops:
        if o.N <= 1024:
            o.check()
            continue
        # large ops: sampled rows against the oracle
        ncols = o.y.shape[1]
        cols = np.unique(np.concatenate([[0, ncols - 1], rng.integers(0, ncols, 48)]))
        x = o.x.double().cpu().numpy()
        y = o.y.double().cpu().numpy()[:, cols]
        if o.epi == q.QLIN_EPI_SILU_GATE:
            rows = np.concatenate([cols, cols + o.N // 2])
            ref, A = oracle.gemv(fmt, o.N, o.K, o.blocks, x, rows=rows)
            href, Ah = oracle.silu_gate(ref, A)
            tol = TOL * Ah + 8 * 2.0 ** -24 * np.abs(href) + 4 * 2.0 ** -126 * (1 + np.abs(ref[:, len(cols):]))
            assert (np.abs(y - href) <= tol).all()
        else:
            ref, A = oracle.gemv(fmt, o.N, o.K, o.blocks, x, rows=cols)
            assert (np.abs(y - ref) <= TOL * A).all()


def test_chain_argument_checks():
    fmt, M = q.QLIN_Q4_0, 1
    a = Op(fmt, 64, 256, M, 5)
    ok = a.op()
    bad_wait = q.gemv_op(a.packed, 64, 256, a.x, a.y, q.QLIN_EPI_NONE, 1)  # names itself, not an earlier op
    lib = q.lib()
    ws = q.workspace(1 << 20)
    arr, ptr = q._op_array([ok, bad_wait])
    st = lib.qlin_gemv_chain(fmt, q.QLIN_F32, M, ptr, 2, 0, q._dev(ws, "ws"), ws.numel(), q._stream())
    assert st == 1
    arr, ptr = q._op_array([ok])
    assert lib.qlin_gemv_chain(fmt, q.QLIN_F32, M, ptr, 0, 0, q._dev(ws, "ws"), ws.numel(), q._stream()) == 1
    assert lib.qlin_gemv_chain(fmt, q.QLIN_F32, 9, ptr, 1, 0, q._dev(ws, "ws"), ws.numel(), q._stream()) == 1
    assert lib.qlin_gemv_chain(fmt, q.QLIN_F32, M, ptr, 1, 0, q._dev(ws, "ws"), 16, q._stream()) == 4


@pytest.mark.parametrize("fmt", [q.QLIN_NVFP4, q.QLIN_Q4_0, q.QLIN_MXFP4, q.QLIN_Q4_K, q.QLIN_Q6_K])
@pytest.mark.parametrize("M", [1, 4])
def test_chain_bf16_mlp(fmt, M):
    """A bf16 chain of gated MLPs: gate_up writes h in bf16 (QLIN_OUT_BF16), down reads it."""
    ops = []
    for l in range(2):
        I = 512 if fmt in (q.QLIN_Q4_K, q.QLIN_Q6_K) else 352  # K-quants: K a multiple of 256
        gu = Op(fmt, 2 * I, 1024, M, 200 + l, epi=q.QLIN_EPI_SILU_GATE | q.QLIN_OUT_BF16, xdt=torch.bfloat16)
        dn = Op(fmt, 288, I, M, 210 + l, x=gu.y, wait_for=len(ops), xdt=torch.bfloat16)
        ops += [gu, dn]
    ws = run(fmt, torch.bfloat16, M, ops)
    torch.cuda.synchronize()
    assert q.qlin_ws_status(ws) == 0
    for o in ops:
        o.check()
