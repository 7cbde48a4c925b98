"""GPU parity of the MoE prefill path (qlin_moe_prefill: route + sort, grouped tcgen05 GEMMs).

Checked stage by stage against the fp64 oracle, with every bound derived from the arithmetic:
  routing   ids equal to the oracle's (the decision is taken on the fp32 logits on both sides),
            weights within 1e-6 relative (fp32 softmax over the selected experts);
  gate_up   h of each (token, slot) against silu(g) * u of the oracle's product of the same
            quantized activations (NVFP4: one per-tensor scale from max |x| over the chunk; MXFP4:
            the OCP MX rule, row-local) with the expert's weights: the GEMM bound 2e-6 sum|a_q w|
            carried through silu(g) * u, the epilogue's error (silu_tol below), and h's rounding
            to bf16 (half an ulp, at most 2^-8 relative);
  down      y against the slot-ordered sum of the oracle's down projections of the kernel's own
            h quantized the same way (NVFP4: a per-tensor scale over all h): 2e-6 sum|h_q w| per
            slot and gamma(top_k) for the fp32 combine, as for the decode MoE.
"""
import numpy as np
import pytest
import torch

import gemm_dequant_gemv_q8_b200 as q
import oracle
import synth

pytestmark = pytest.mark.gpu
U32 = 2.0 ** -24


def gamma(n):
    return n * U32 / (1 - n * U32)


def silu_tol(href, Ah, g, u):
    """The epilogue forms z = g s, e = exp(-|z|) with the MUFU ex2 unit (argument -|z| log2 e
    rounded: |z| 2^-23 relative on e; the unit itself taken as 2^-21 relative) and 1 / (1 + e)
    with the MUFU rcp unit (2^-21); sigmoid is r (z >= 0) or e r (z < 0), so within
    2 (2^-21 + |z| 2^-23) + 2^-21 + 2^-23 relative; four fp32 roundings (z, u s, z sig, times u)
    add 2^-22.  Together under (2^-19 + |g| 2^-22) |h|, plus the GEMM bound carried through
    silu(g) u (2e-6 Ah), plus (|g| + 4) 2^-126 (1 + |u|) for e flushed to zero below 2^-126
    (|h| <= |z| e^-|z| |u| there)."""
    return (2e-6 * Ah + (2.0 ** -19 + np.abs(g) * 2.0 ** -22) * np.abs(href) +
            (np.abs(g) + 4) * 2.0 ** -126 * (1 + np.abs(u)))


class Experts:
    def __init__(self, fmt, E, H, I, seed):
        self.fmt, self.E, self.H, self.I = fmt, E, H, I
        self.gu = [synth.weights(fmt, 2 * I, H, synth.gen(seed + e)) for e in range(E)]
        self.dn = [synth.weights(fmt, H, I, synth.gen(seed + 500 + e)) for e in range(E)]
        dev = lambda b, s, g: (b.cuda(), None if s is None else s.cuda(), g)
        self.gu_p = q.pack_experts(fmt, E, 2 * I, H, [dev(*t) for t in self.gu], q.QLIN_PACK_MMA | q.QLIN_PACK_GATE_UP)
        self.dn_p = q.pack_experts(fmt, E, H, I, [dev(*t) for t in self.dn], q.QLIN_PACK_MMA)

    def w(self, t):
        b, s, g = t
        return b.numpy(), None if s is None else s.numpy(), g


def quantize(fmt, X):
    """The chunk path's quantized activations (fp64 values) of the rows of X."""
    X = np.ascontiguousarray(X, np.float32)
    if fmt == q.QLIN_NVFP4:
        c, s, ag = oracle.act_quant(X)
        return oracle.dequant(fmt, X.shape[0], X.shape[1], c, s, ag)
    c, s = oracle.act_quant_mx(X)
    return oracle.dequant(fmt, X.shape[0], X.shape[1], c, s)


def run_and_check(ex, M, top_k, seed, tokens=None, logits=None, given=None):
    fmt, E, H, I = ex.fmt, ex.E, ex.H, ex.I
    x = synth.activations(M, H, synth.gen(seed), dtype=torch.bfloat16)
    h = torch.full((M, top_k, I), float("nan"), device="cuda")
    ws = q.workspace(q.qlin_workspace_bytes(q.QLIN_OP_MOE_PREFILL, fmt, M, H, I, E, top_k))
    if given is None:
        if logits is None:
            logits = synth.router_logits(M, E, synth.gen(seed + 1))
        y, ids, w, _ = q.qlin_moe_prefill(fmt, ex.gu_p, ex.dn_p, E, H, I, top_k, x.cuda(),
                                          router_logits=logits.cuda(), h=h, ws=ws)
    else:
        y, ids, w, _ = q.qlin_moe_prefill(fmt, ex.gu_p, ex.dn_p, E, H, I, top_k, x.cuda(),
                                          topk_ids=torch.as_tensor(given[0], dtype=torch.int32).cuda(),
                                          topk_w=torch.as_tensor(given[1], dtype=torch.float32).cuda(), h=h, ws=ws)
    torch.cuda.synchronize()
    bad = given is not None and any(not (0 <= int(e) < E) or int(e) in [int(v) for v in r[:i]]
                                    for r in given[0] for i, e in enumerate(r))
    assert q.qlin_ws_status(ws) == (1 if bad else 0)  # QLIN_ERR_INVALID_ARG: a bad expert id
    ids, w = ids.cpu().numpy(), w.cpu().double().numpy()
    h, y = h.cpu().double().numpy(), y.cpu().double().numpy()
    if given is None:
        rids, rw = oracle.route(logits.double().numpy(), top_k)
        assert np.array_equal(ids, rids)
        assert np.allclose(w, rw, rtol=1e-6, atol=0)
    xq = quantize(fmt, x.float().numpy())           # every token is routed: the same rows, same scale
    hq = quantize(fmt, h.reshape(M * top_k, I)).reshape(M, top_k, I)  # the kernel's h, quantized
    for m in (range(M) if tokens is None else tokens):
        yref = np.zeros(H)
        A = np.zeros(H)
        for s in range(top_k):
            e = int(ids[m, s])
            if not (0 <= e < E) or e in [int(v) for v in ids[m, :s]]:  # a skipped slot
                assert (h[m, s] == 0).all()
                continue
            gb, gs, gg = ex.w(ex.gu[e])
            gu, Agu = oracle.gemv(fmt, 2 * I, H, gb, xq[m:m + 1], scales=gs, g=gg)
            href, Ah = oracle.silu_gate(gu, Agu)
            tol = silu_tol(href[0], Ah[0], gu[0, :I], gu[0, I:])
            tol = tol + 2.0 ** -8 * (np.abs(href[0]) + tol)
            err = np.abs(h[m, s] - href[0])
            assert (err <= tol).all(), (m, s, float(np.max(err / tol)))
            db, ds, dg = ex.w(ex.dn[e])
            o, Ao = oracle.gemv(fmt, H, I, db, hq[m, s][None], scales=ds, g=dg)
            yref += w[m, s] * o[0]
            A += abs(w[m, s]) * Ao[0]
        tol_y = (2e-6 + gamma(top_k) * (1 + 2e-6)) * A
        assert (np.abs(y[m] - yref) <= tol_y + 1e-30).all(), (m, float(np.max(np.abs(y[m] - yref) / tol_y)))
    return ids, w, y


@pytest.mark.parametrize("fmt", [q.QLIN_NVFP4, q.QLIN_MXFP4])
@pytest.mark.parametrize("M", [1, 37, 200])
def test_moe_prefill_small(fmt, M):
    # 8 experts of gate_up 512 -> 2 x 288 (a ragged 128-row tile) and down 288 -> 512, top-2
    ex = Experts(fmt, 8, 512, 288, 7000 + fmt)
    run_and_check(ex, M, 2, 7100 + M)


@pytest.mark.parametrize("fmt,E,H,I,M,k", [
    (q.QLIN_NVFP4, 256, 64, 64, 5, 8),     # the largest expert count and top_k the entry point takes
    (q.QLIN_MXFP4, 1, 96, 160, 70, 1),     # one expert: every token on it
    (q.QLIN_NVFP4, 4, 32, 32, 9, 4),       # the smallest H and I, top_k = E
    (q.QLIN_MXFP4, 16, 64, 96, 4096, 2),   # many tokens: 256 routing CTAs, 64 tiles per expert on average
])
def test_moe_prefill_edge_shapes(fmt, E, H, I, M, k):
    ex = Experts(fmt, E, H, I, 7600 + E)
    tokens = None if M <= 128 else [0, 1, 2047, 2048, 4095]
    run_and_check(ex, M, k, 7700 + M, tokens=tokens)


@pytest.mark.parametrize("fmt", [q.QLIN_NVFP4, q.QLIN_MXFP4])
def test_moe_prefill_lfm2_shape_sampled(fmt):
    # the 8B-A1B MoE layer (H 2048, 32 experts of gate_up 2048 -> 2 x 1792, down 1792 -> 2048, top-4)
    # over a prefill chunk of 512 tokens; every routed row goes through the GEMMs, a sample of tokens
    # is checked against the oracle
    ex = Experts(fmt, 32, 2048, 1792, 7200 + fmt)
    run_and_check(ex, 512, 4, 7300, tokens=[0, 1, 77, 255, 256, 400, 511])


def test_moe_prefill_given_ids_uneven_load():
    # ids as inputs: every token on expert 3 (a 2-tile expert at M = 150) and one other
    fmt, E, H, I, M, k = q.QLIN_NVFP4, 6, 256, 128, 150, 2
    ex = Experts(fmt, E, H, I, 7400)
    rng = np.random.default_rng(3)
    ids = np.stack([np.array([3, [0, 1, 2, 4, 5][m % 5]]) for m in range(M)]).astype(np.int32)
    w = rng.uniform(0.1, 1.0, (M, k)).astype(np.float32)
    out_ids, _, _ = run_and_check(ex, M, k, 7401, given=(ids, w))
    assert np.array_equal(out_ids, ids)


@pytest.mark.parametrize("fmt", [q.QLIN_NVFP4, q.QLIN_MXFP4])
def test_moe_prefill_bad_ids_reported_and_skipped(fmt):
    # given ids with an out-of-range id and a repeated one: status bit 1 set, those slots skipped
    E, H, I, M, k = 6, 256, 160, 40, 3
    ex = Experts(fmt, E, H, I, 7450)
    rng = np.random.default_rng(5)
    ids = np.stack([rng.permutation(E)[:k] for _ in range(M)]).astype(np.int32)
    ids[3, 1] = E + 2
    ids[7, 2] = ids[7, 0]
    ids[9, 0] = -1
    w = rng.uniform(0.1, 1.0, (M, k)).astype(np.float32)
    run_and_check(ex, M, k, 7451, given=(ids, w))


def test_moe_prefill_deterministic_and_graph_capturable():
    fmt, E, H, I, M, k = q.QLIN_NVFP4, 8, 512, 256, 130, 2
    ex = Experts(fmt, E, H, I, 7500)
    x = synth.activations(M, H, synth.gen(7501), dtype=torch.bfloat16).cuda()
    logits = synth.router_logits(M, E, synth.gen(7502)).cuda()
    ws = q.workspace(q.qlin_workspace_bytes(q.QLIN_OP_MOE_PREFILL, fmt, M, H, I, E, k))
    ids = torch.empty(M, k, dtype=torch.int32, device="cuda")
    w = torch.empty(M, k, device="cuda")
    y = torch.empty(M, H, device="cuda")
    ref = q.qlin_moe_prefill(fmt, ex.gu_p, ex.dn_p, E, H, I, k, x, router_logits=logits, ws=ws)[0].clone()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())  # calls sharing a workspace must not overlap
    with torch.cuda.stream(s):
        q.qlin_moe_prefill(fmt, ex.gu_p, ex.dn_p, E, H, I, k, x, router_logits=logits, topk_ids=ids, topk_w=w, y=y,
                           ws=ws)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        q.qlin_moe_prefill(fmt, ex.gu_p, ex.dn_p, E, H, I, k, x, router_logits=logits, topk_ids=ids, topk_w=w, y=y,
                           ws=ws)
    for _ in range(3):
        y.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(y, ref)
    assert q.qlin_ws_status(ws) == 0


def test_moe_prefill_tied_logits():
    """Equal logits go to the lower expert index: the routing equals the oracle's on rows built
    with ties, and the layer matches as in the other tests."""
    fmt, E, H, I, M, k = q.QLIN_NVFP4, 8, 128, 96, 6, 3
    ex = Experts(fmt, E, H, I, 7950)
    logits = synth.router_logits(M, E, synth.gen(7951)).clone()
    logits[1, :] = 0.25                       # all tied: experts 0, 1, 2
    logits[2, [1, 5, 6]] = 8.0                # a three-way tie at the top
    logits[4, [0, 3]] = -8.0                  # a tie at the bottom, never selected
    run_and_check(ex, M, k, 7952, logits=logits)


def test_moe_prefill_workspace_reused_across_shapes():
    """One workspace (sized for the largest call) through calls of different M: each result equals
    the same call on a fresh workspace, bit for bit, and the status stays clean."""
    fmt, E, H, I, k = q.QLIN_NVFP4, 8, 256, 160, 2
    ex = Experts(fmt, E, H, I, 7800)
    ws = q.workspace(q.qlin_workspace_bytes(q.QLIN_OP_MOE_PREFILL, fmt, 300, H, I, E, k))
    for M in (300, 17, 129, 300, 1):
        x = synth.activations(M, H, synth.gen(7801 + M), dtype=torch.bfloat16).cuda()
        logits = synth.router_logits(M, E, synth.gen(7901 + M)).cuda()
        y = q.qlin_moe_prefill(fmt, ex.gu_p, ex.dn_p, E, H, I, k, x, router_logits=logits, ws=ws)[0]
        ref = q.qlin_moe_prefill(fmt, ex.gu_p, ex.dn_p, E, H, I, k, x, router_logits=logits)[0]
        torch.cuda.synchronize()
        assert q.qlin_ws_status(ws) == 0
        assert torch.equal(y, ref), M


def test_moe_prefill_argument_checks():
    lib, P = q.lib(), q._dev
    x = torch.zeros(4, 256, dtype=torch.bfloat16, device="cuda")
    # GGUF formats are not on this path
    assert q.qlin_workspace_bytes(q.QLIN_OP_MOE_PREFILL, q.QLIN_Q4_0, 4, 256, 128, 4, 2) == 0
    st = lib.qlin_moe_prefill(q.QLIN_Q4_0, P(x, "a"), P(x, "b"), 4, 256, 128, 2, None, P(x, "c"), P(x, "d"),
                              P(x, "x"), 4, P(x, "y"), None, 0, P(x, "ws"), 1 << 20, q._stream(None))
    assert st == 2  # QLIN_ERR_UNSUPPORTED
