"""GPU parity of the routed MoE expert path against the fp64 oracle, stage by stage.

ids exact (the decision is taken on the fp32 logits on both sides); weights within 1e-6
relative; h against the oracle's silu(gate)*up of the same x; y against the oracle's down
projections of the kernel's own h, combined with the kernel's weights in slot order; and y end to
end against the pure fp64 chain.  Every bound past the GEMV's 2e-6 * sum|w*x| is derived below
from the arithmetic the kernel performs (combine_tol, e2e_tol), not chosen.

Weights: the kernel forms p_i = exp(l_i - l_max) / sum over the top_k of exp(l_j - l_max) in
fp32; with expf within 2 ulp that is at most (2 + 2 + (top_k - 1) + 1) * 2^-24 <= 4.8e-7
relative for top_k <= 4 (6.5e-7 for top_k = 8), inside the 1e-6 the routing check asserts.
"""
import numpy as np
import pytest
import torch

import gemm_dequant_gemv_q8_b200 as q
import oracle
import synth

pytestmark = pytest.mark.gpu


U32 = 2.0 ** -24
W_RTOL = 1e-6  # the routing weights' relative bound, asserted by run_and_check


def silu_tol(href, Ah, u):
    return 2e-6 * Ah + 8 * U32 * np.abs(href) + 4 * 2.0 ** -126 * (1 + np.abs(u))


def gamma(n):
    """Bound on the relative error of a sequential fp32 sum of n terms, fused multiply-adds
    included (one rounding each): n u / (1 - n u)."""
    return n * U32 / (1 - n * U32)


def combine_tol(A, top_k):
    """y = sum over slots, in slot order, of w_s * o_s, each o_s a down-projection GEMV of the
    kernel's own h (so within 2e-6 * A_s), summed by top_k fused multiply-adds from 0:
    |y - sum w_s o_s| <= sum |w_s| 2e-6 A_s + gamma(top_k) sum |w_s| |o_s + err_s|
                      <= (2e-6 + gamma(top_k) (1 + 2e-6)) * A,   A = sum_s |w_s| A_s."""
    return (2e-6 + gamma(top_k) * (1 + 2e-6)) * A


def e2e_tol(ex, ids, w_ref, xd, top_k):
    """First-order bound on y against the pure fp64 chain, propagated stage by stage:
      h: the bound the stage check asserts, dh = silu_tol (GEMV bound of gate and up carried
         through silu(g) * u, plus the epilogue's fp32 roundings);
      o = W_dn h: the GEMV bound on the kernel's h (2e-6 * |W_dn| (|h| + dh)) plus the
         propagated h error |W_dn| dh;
      y = sum w_s o_s: weight error W_RTOL |w_s| |o_s|, slot error |w_s| (1 + W_RTOL) do_s, and
         the combine's gamma(top_k) * sum |w_s| (1 + W_RTOL) (|o_s| + do_s)."""
    M, fmt, H, I = xd.shape[0], ex.fmt, ex.H, ex.I
    tol = np.zeros((M, H))
    for m in range(M):
        acc = np.zeros(H)
        mag = np.zeros(H)
        for s in range(top_k):
            e = int(ids[m, s])
            gb, gs, gg = ex.np(ex.gu[e])
            gu, Agu = oracle.gemv(fmt, 2 * I, H, gb, xd[m:m + 1], scales=gs, g=gg)
            h, Ah = oracle.silu_gate(gu, Agu)
            dh = silu_tol(h[0], Ah[0], gu[0, I:])
            db, ds, dg = ex.np(ex.dn[e])
            W = oracle.dequant(fmt, H, I, db, ds, dg)
            Wa = np.abs(W)
            o = W @ h[0]
            do = 2e-6 * (Wa @ (np.abs(h[0]) + dh)) + Wa @ dh
            ws = abs(w_ref[m, s])
            acc += W_RTOL * ws * np.abs(o) + ws * (1 + W_RTOL) * do
            mag += ws * (1 + W_RTOL) * (np.abs(o) + do)
        tol[m] = acc + gamma(top_k) * mag
    return tol


class Experts:
    def __init__(self, fmt, E, H, I, seed, device="cuda"):
        self.fmt, self.E, self.H, self.I = fmt, E, H, I
        self.gu = [synth.weights(fmt, 2 * I, H, synth.gen(seed + e)) for e in range(E)]
        self.dn = [synth.weights(fmt, H, I, synth.gen(seed + 1000 + e)) for e in range(E)]
        dev = lambda t: None if t[1] is None else t[1].to(device)
        self.gu_p = q.pack_experts(fmt, E, 2 * I, H, [(b.to(device), dev((b, s)), g) for b, s, g in self.gu],
                                   q.QLIN_PACK_GATE_UP)
        self.dn_p = q.pack_experts(fmt, E, H, I, [(b.to(device), dev((b, s)), g) for b, s, g in self.dn])

    def np(self, t):
        b, s, g = t
        return b.numpy(), None if s is None else s.numpy(), g


def run_and_check(ex, M, top_k, logits, x, given=None, ws=None):
    fmt, E, H, I = ex.fmt, ex.E, ex.H, ex.I
    h = torch.empty(M, top_k, I, device="cuda")
    if given is None:
        y, ids, w, _ = q.qlin_moe_experts(fmt, ex.gu_p, ex.dn_p, E, H, I, top_k, x.cuda(),
                                          router_logits=logits.cuda(), h=h, ws=ws)
    else:
        ids_in = torch.as_tensor(given[0], dtype=torch.int32).cuda()
        w_in = torch.as_tensor(given[1], dtype=torch.float32).cuda()
        y, ids, w, _ = q.qlin_moe_experts(fmt, ex.gu_p, ex.dn_p, E, H, I, top_k, x.cuda(), topk_ids=ids_in,
                                          topk_w=w_in, h=h, ws=ws)
    torch.cuda.synchronize()
    ids, w, h, y = ids.cpu().numpy(), w.cpu().double().numpy(), h.cpu().double().numpy(), y.cpu().double().numpy()
    xd = x.double().numpy()
    if given is None:
        rids, rw = oracle.route(logits.double().numpy(), top_k)
        assert np.array_equal(ids, rids)
        assert np.allclose(w, rw, rtol=1e-6, atol=0)
    for m in range(M):
        yref = np.zeros(H)
        A = np.zeros(H)
        for s in range(top_k):
            e = int(ids[m, s])
            gb, gs, gg = ex.np(ex.gu[e])
            gu, Agu = oracle.gemv(fmt, 2 * I, H, gb, xd[m:m + 1], scales=gs, g=gg)
            href, Ah = oracle.silu_gate(gu, Agu)
            assert (np.abs(h[m, s] - href[0]) <= silu_tol(href[0], Ah[0], gu[0, I:])).all(), (m, s)
            db, ds, dg = ex.np(ex.dn[e])
            o, Ao = oracle.gemv(fmt, H, I, db, h[m, s][None], scales=ds, g=dg)
            yref += w[m, s] * o[0]
            A += abs(w[m, s]) * Ao[0]
        assert (np.abs(y[m] - yref) <= combine_tol(A, top_k)).all(), m
    return ids, w, y


@pytest.mark.parametrize("M", [1, 8])
def test_moe_q4_0_lfm2_shape(M):
    # H = 2048, 32 experts of gate_up 2048 -> 2 x 1792 and down 1792 -> 2048, top-4
    ex = Experts(q.QLIN_Q4_0, 32, 2048, 1792, 4000)
    logits = synth.router_logits(M, 32, synth.gen(4100 + M))
    x = synth.activations(M, 2048, synth.gen(4200 + M))
    ids, w, y = run_and_check(ex, M, 4, logits, x)
    # end to end against the pure fp64 chain, within the propagated bound
    r = oracle.moe(q.QLIN_Q4_0, 32, 2048, 1792, 4, np.stack([ex.np(t)[0] for t in ex.gu]),
                   np.stack([ex.np(t)[0] for t in ex.dn]), logits.double().numpy(), x.double().numpy())
    assert np.array_equal(ids, r["ids"])
    tol = e2e_tol(ex, r["ids"], r["wts"], x.double().numpy(), 4)
    err = np.abs(y - r["y"])
    assert (err <= tol).all(), float(np.max(err / tol))
    # for scale: the derived bound relative to the chain's own sum |w * x| terms
    print("e2e bound / A: max %.3g, median %.3g" % (np.max(tol / r["A"]), np.median(tol / r["A"])))


@pytest.mark.parametrize("fmt,xdt", [(q.QLIN_Q8_0, torch.float32), (q.QLIN_NVFP4, torch.bfloat16),
                                     (q.QLIN_Q4_0, torch.bfloat16), (q.QLIN_MXFP4, torch.bfloat16),
                                     (q.QLIN_MXFP4, torch.float32)])
@pytest.mark.parametrize("M", [1, 3, 8])
def test_moe_formats_small(fmt, xdt, M):
    ex = Experts(fmt, 6, 256, 96, 5000 + fmt)
    logits = synth.router_logits(M, 6, synth.gen(5100 + M))
    x = synth.activations(M, 256, synth.gen(5200 + M), dtype=xdt)
    run_and_check(ex, M, 2, logits, x)


@pytest.mark.parametrize("fmt", [q.QLIN_Q4_K, q.QLIN_Q6_K])
@pytest.mark.parametrize("M", [1, 8])
def test_moe_kquant_experts(fmt, M):
    # K-quant experts (K a multiple of 256 for both projections): H = 512, I = 256, top-2 of 6
    ex = Experts(fmt, 6, 512, 256, 5500)
    logits = synth.router_logits(M, 6, synth.gen(5600 + M))
    x = synth.activations(M, 512, synth.gen(5700 + M))
    run_and_check(ex, M, 2, logits, x)


@pytest.mark.parametrize("M", [2, 8])
def test_moe_all_experts_uniform_is_mean(M):
    # equal logits: ties go to the lower expert index; with M = 8 every expert serves all 8
    # tokens, four work entries of two rows each
    fmt, E, H, I = q.QLIN_Q4_0, 4, 256, 64
    ex = Experts(fmt, E, H, I, 6000)
    x = synth.activations(M, H, synth.gen(6001))
    ids, w, y = run_and_check(ex, M, E, torch.zeros(M, E), x)
    assert (ids == np.arange(E)).all() and np.allclose(w, 1.0 / E, rtol=1e-7)


def test_moe_given_ids_and_weights():
    fmt, E, H, I, M, k = q.QLIN_Q4_0, 8, 512, 128, 4, 3
    ex = Experts(fmt, E, H, I, 7000)
    rng = np.random.default_rng(0)
    ids = np.stack([rng.permutation(E)[:k] for _ in range(M)]).astype(np.int32)
    w = rng.uniform(0.1, 1.0, (M, k)).astype(np.float32)
    x = synth.activations(M, H, synth.gen(7001))
    out_ids, out_w, _ = run_and_check(ex, M, k, None, x, given=(ids, w))
    assert np.array_equal(out_ids, ids)


def test_moe_bad_expert_id_is_reported_and_skipped():
    fmt, E, H, I, M, k = q.QLIN_Q4_0, 4, 256, 64, 1, 2
    ex = Experts(fmt, E, H, I, 8000)
    x = synth.activations(M, H, synth.gen(8001))
    ws = q.workspace(q.qlin_workspace_bytes(q.QLIN_OP_MOE, fmt, M, H, I, E, k))
    ids = torch.tensor([[1, 9]], dtype=torch.int32, device="cuda")  # 9 is out of range
    w = torch.tensor([[0.5, 0.5]], device="cuda")
    y, _, _, _ = q.qlin_moe_experts(fmt, ex.gu_p, ex.dn_p, E, H, I, k, x.cuda(), topk_ids=ids, topk_w=w, ws=ws)
    assert q.qlin_ws_status(ws) == 1  # QLIN_ERR_INVALID_ARG
    # the valid slot alone
    ids1 = torch.tensor([[1]], dtype=torch.int32, device="cuda")
    y1, _, _, _ = q.qlin_moe_experts(fmt, ex.gu_p, ex.dn_p, E, H, I, 1, x.cuda(), topk_ids=ids1,
                                     topk_w=torch.tensor([[0.5]], device="cuda"))
    assert torch.equal(y, y1)


def test_moe_deterministic_and_graph_capturable():
    fmt, E, H, I, M, k = q.QLIN_Q4_0, 32, 2048, 1792, 8, 4
    ex = Experts(fmt, E, H, I, 9000)
    logits = synth.router_logits(M, E, synth.gen(9001)).cuda()
    x = synth.activations(M, H, synth.gen(9002)).cuda()
    ws = q.workspace(q.qlin_workspace_bytes(q.QLIN_OP_MOE, fmt, M, H, I, E, k))
    ids = torch.empty(M, k, dtype=torch.int32, device="cuda")
    w = torch.empty(M, k, device="cuda")
    y = torch.empty(M, H, device="cuda")
    ref = q.qlin_moe_experts(fmt, ex.gu_p, ex.dn_p, E, H, I, k, x, router_logits=logits, ws=ws)[0].clone()
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())  # calls sharing a workspace must not overlap
    with torch.cuda.stream(s):
        q.qlin_moe_experts(fmt, ex.gu_p, ex.dn_p, E, H, I, k, x, router_logits=logits, topk_ids=ids, topk_w=w,
                           y=y, ws=ws, flags=q.QLIN_FLAG_PDL)
    torch.cuda.synchronize()
    with torch.cuda.graph(g):
        q.qlin_moe_experts(fmt, ex.gu_p, ex.dn_p, E, H, I, k, x, router_logits=logits, topk_ids=ids, topk_w=w,
                           y=y, ws=ws, flags=q.QLIN_FLAG_PDL)
    for _ in range(3):
        y.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(y, ref)
    assert q.qlin_ws_status(ws) == 0
