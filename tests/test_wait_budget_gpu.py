"""Bounded device waits that run out, made to run out on purpose (no fault, no endless loop).

A wait between CTAs is given a budget of 1 ns (qlin_ws_set_wait_budget) and a dependency that
cannot be met yet when it is first checked: warps or CTAs that have no share of the producing op
(fewer producer units than warps, fewer gate_up tiles than CTAs) reach the dependent op as soon as
the launch starts, while the producers' tiles need at least one trip to HBM.  The kernel must then
return on its own, report QLIN_ERR_TIMEOUT through qlin_ws_status, and leave the workspace usable:
the next call, with the default budget, gives the same bits as a call on a fresh workspace.  The
outputs of the call whose waits ran out are unspecified and not checked.
"""
import pytest
import torch

import gemm_dequant_gemv_q8_b200 as q
import synth

pytestmark = pytest.mark.gpu
TINY_NS = 1


def packed_q4(N, K, seed):
    blocks, _, _ = synth.weights(q.QLIN_Q4_0, N, K, synth.gen(seed))
    return q.qlin_pack_weights(q.QLIN_Q4_0, N, K, blocks.cuda())


def run_out(call, ws, attempts=3):
    """Run call() with the tiny budget until a wait runs out (normally the first time)."""
    q.qlin_ws_set_wait_budget(ws, TINY_NS)
    for _ in range(attempts):
        call()
        torch.cuda.synchronize()  # the launch ended by itself
        st = q.qlin_ws_status(ws)
        if st == 6:  # QLIN_ERR_TIMEOUT
            break
    q.qlin_ws_set_wait_budget(ws, 0)
    return st


def test_chain_wait_runs_out_and_workspace_recovers():
    # op 0: 32 tiles x 10 k-groups = 320 units, fewer than the grid's warps: the warps without
    # op 0 units go straight to op 1, whose wait for op 0 runs out.
    N0, K0, N1 = 1024, 2560, 1024
    p0, p1 = packed_q4(N0, K0, 1), packed_q4(N1, N0, 2)
    x = synth.activations(1, K0, synth.gen(3)).cuda()
    y0 = torch.empty(1, N0, device="cuda")
    y1 = torch.empty(1, N1, device="cuda")
    ops = [q.gemv_op(p0, N0, K0, x, y0), q.gemv_op(p1, N1, N0, y0, y1, wait_for=0)]
    ref_ws = q.qlin_gemv_chain(q.QLIN_Q4_0, q.QLIN_F32, 1, ops)
    ref0, ref1 = y0.clone(), y1.clone()
    assert q.qlin_ws_status(ref_ws) == 0

    ws = q.workspace(q.qlin_chain_workspace_bytes(q.QLIN_Q4_0, 1, ops))
    assert run_out(lambda: q.qlin_gemv_chain(q.QLIN_Q4_0, q.QLIN_F32, 1, ops, ws=ws), ws) == 6
    assert not ws[256:256 + 8].any()  # the last CTA out reset the per-op tile counts
    for _ in range(2):
        y0.fill_(float("nan"))
        y1.fill_(float("nan"))
        q.qlin_gemv_chain(q.QLIN_Q4_0, q.QLIN_F32, 1, ops, ws=ws)
        torch.cuda.synchronize()
        assert q.qlin_ws_status(ws) == 0
        assert torch.equal(y0, ref0) and torch.equal(y1, ref1)


@pytest.mark.parametrize("M", [1, 2])
def test_moe_wait_runs_out_and_workspace_recovers(M):
    # I = 256: 16 gate_up tiles per selected expert, at most 8 experts (128 tiles) for M <= 2,
    # fewer than the CTAs: the CTAs without gate_up tiles start on down units, whose wait for
    # their expert's gate_up tiles runs out.
    fmt, E, H, I, k = q.QLIN_Q4_0, 8, 1024, 256, 4
    gu = [synth.weights(fmt, 2 * I, H, synth.gen(100 + e)) for e in range(E)]
    dn = [synth.weights(fmt, H, I, synth.gen(200 + e)) for e in range(E)]
    gu_p = q.pack_experts(fmt, E, 2 * I, H, [(b.cuda(), None, g) for b, s, g in gu], q.QLIN_PACK_GATE_UP)
    dn_p = q.pack_experts(fmt, E, H, I, [(b.cuda(), None, g) for b, s, g in dn])
    logits = synth.router_logits(M, E, synth.gen(300 + M)).cuda()
    x = synth.activations(M, H, synth.gen(400 + M)).cuda()
    nbytes = q.qlin_workspace_bytes(q.QLIN_OP_MOE, fmt, M, H, I, E, k)
    ref = q.qlin_moe_experts(fmt, gu_p, dn_p, E, H, I, k, x, router_logits=logits,
                             ws=q.workspace(nbytes))[0].clone()

    ws = q.workspace(nbytes)
    call = lambda: q.qlin_moe_experts(fmt, gu_p, dn_p, E, H, I, k, x, router_logits=logits, ws=ws)
    assert run_out(call, ws) == 6
    for _ in range(2):  # the combine tickets left by the abandoned units were cleared
        y = call()[0]
        torch.cuda.synchronize()
        assert q.qlin_ws_status(ws) == 0
        assert torch.equal(y, ref)


def test_wait_budget_argument_checks():
    assert q.lib().qlin_ws_set_wait_budget(None, 5, None) == 1
    ws = q.workspace(512)
    q.qlin_ws_set_wait_budget(ws, 123456)
    assert int(ws[32:36].view(torch.int32).item()) == 123456
    q.qlin_ws_set_wait_budget(ws, 0)
    assert not ws[32:36].any()
