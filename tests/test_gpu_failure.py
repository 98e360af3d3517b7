"""Failure handling on the GPU without faulting it: the bounded wait of the streaming pass is made
to run out by its test hook (a barrier that nothing completes, a short limit), and the call must
report GSPARSE_DERR_TIMEOUT, skip the rest of its work, and leave the context usable for the next
call, which must match the oracle bit for bit. Also the per-call events around the streaming
pass (no process-wide state)."""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests.gpu_util import bits, dev, host

import compressed_sgd_b200 as gs

pytestmark = pytest.mark.gpu


def test_expired_wait_reports_timeout_and_the_next_call_is_exact():
    n, keep, m = (1 << 22) + 5, (1, 100), 0.9
    g = synth.flat_mixture(n, seed=70)
    u = synth.gaussian(n, 71, sigma=1e-3)
    r = synth.gaussian(n, 72, sigma=1e-4)
    gd, ud, rd = dev(g), dev(u), dev(r)
    cap = gs.k_for(n, keep)
    sentinel = -7
    idx = torch.full((cap,), sentinel, dtype=torch.int32, device="cuda")
    val = torch.zeros(cap, device="cuda")
    st = gs.status_tensor()
    gs.residual_topk(gd, rd, keep, out_idx=idx, out_val=val, d_status=st, momentum=(ud, m),
                     flags=gs.GSPARSE_SELECT_TEST_EXPIRE_WAIT)
    torch.cuda.synchronize()
    assert int(st.item()) & gs.DERR_TIMEOUT
    # the steps after the streaming pass did nothing: no entry was emitted
    assert bool((idx == sentinel).all())
    # the context is usable: the same step again from the saved state, without the hook
    ud.copy_(dev(u))
    rd.copy_(dev(r))
    st2 = gs.status_tensor()
    gi, gv, go = gs.residual_topk(gd, rd, keep, d_status=st2, momentum=(ud, m))
    wi, wv, wo, wr, wu = oracle.residual_topk_momentum(g, u, m, r, keep)
    assert int(host(st2)[0]) == 0
    K = int(host(go)[-1])
    assert np.array_equal(host(go), wo)
    assert np.array_equal(host(gi)[:K], wi)
    assert np.array_equal(bits(host(gv)[:K]), bits(wv))
    assert np.array_equal(bits(host(rd)), bits(wr))
    assert np.array_equal(bits(host(ud)), bits(wu))


def test_expired_wait_in_plain_topk_reports_timeout():
    # plain top-k streams through the same ring: the hook makes its first waits run out too, and
    # the next call (residual restored) equals the oracle
    n, keep = (1 << 22) + 9, (1, 100)
    g = synth.flat_mixture(n, seed=75)
    r = synth.gaussian(n, 76, sigma=1e-4)
    gd, rd = dev(g), dev(r)
    st = gs.status_tensor()
    gs.residual_topk(gd, rd, keep, d_status=st, flags=gs.GSPARSE_SELECT_TEST_EXPIRE_WAIT)
    torch.cuda.synchronize()
    assert int(st.item()) & gs.DERR_TIMEOUT
    rd.copy_(dev(r))
    st2 = gs.status_tensor()
    gi, gv, go = gs.residual_topk(gd, rd, keep, d_status=st2)
    wi, wv, wo, wr = oracle.residual_topk(g, r, keep)
    K = int(host(go)[-1])
    assert int(host(st2)[0]) == 0
    assert np.array_equal(host(gi)[:K], wi) and np.array_equal(bits(host(gv)[:K]), bits(wv))
    assert np.array_equal(bits(host(rd)), bits(wr))


def test_the_hook_does_nothing_in_binarize():
    # sparse binarisation streams through registers (no waits): the flag changes nothing
    n, keep = 300001, (1, 1000)
    g = synth.gaussian(n, 73, sigma=1e-2)
    r = synth.gaussian(n, 74, sigma=1e-3)
    rd = dev(r)
    st = gs.status_tensor()
    gi, gv, gm, go = gs.binarize(dev(g), rd, keep, d_status=st, flags=gs.GSPARSE_SELECT_TEST_EXPIRE_WAIT)
    wi, wv, wm, wo, wr = oracle.binarize(g, r, keep)
    K = int(host(go)[-1])
    assert int(host(st)[0]) == 0
    assert np.array_equal(host(gi)[:K], wi) and np.array_equal(bits(host(gm)), bits(wm))
    assert np.array_equal(bits(host(rd)), bits(wr))


def test_pass_events_are_per_call():
    # two calls on two streams, each with its own events: both record a positive pass time that
    # lies inside its own call
    n, keep = 1 << 24, (1, 100)
    g = [dev(synth.flat_mixture(n, seed=80 + w)) for w in range(2)]
    r = [torch.zeros(n, device="cuda") for _ in range(2)]
    streams = [torch.cuda.Stream() for _ in range(2)]
    torch.cuda.synchronize()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(2)]
    for w in range(2):
        with torch.cuda.stream(streams[w]):
            ev[w][0].record()
            gs.residual_topk(g[w], r[w], keep, pass_events=(ev[w][1], ev[w][2]))
            ev[w][3].record()
    torch.cuda.synchronize()
    for w in range(2):
        p = ev[w][1].elapsed_time(ev[w][2])
        whole = ev[w][0].elapsed_time(ev[w][3])
        assert 0.0 < p <= whole
        assert ev[w][0].elapsed_time(ev[w][1]) >= 0.0 and ev[w][2].elapsed_time(ev[w][3]) >= 0.0
