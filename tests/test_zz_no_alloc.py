"""The allocation-free residual top-k (scratch in the library's own fixed device array, for
callers that cannot allocate device memory themselves) against the workspace entry point.

Collected last on purpose: if it fails, a run stopped at the first failure has already run every
other test. It needs no state from earlier tests."""
import numpy as np
import pytest
import torch

import oracle
import synth

import compressed_sgd_b200 as gs

pytestmark = pytest.mark.gpu


def _bits(t):
    return t.detach().cpu().numpy().view(np.uint32)


def test_noalloc_matches_workspace_entry_point_on_two_calls_in_a_row():
    n, keep = 3_000_017, (1, 100)
    r0 = synth.gaussian(n, 23, sigma=1e-4)
    ra = torch.from_numpy(r0).cuda()
    rb = ra.clone()
    sa, sb = gs.status_tensor(), gs.status_tensor()
    for seed in (21, 22):                       # residual carried from the first call to the second
        gd = torch.from_numpy(synth.flat_mixture(n, seed=seed)).cuda()
        ia, va, oa = gs.residual_topk(gd, ra, keep, d_status=sa)
        ib, vb, ob = gs.residual_topk_noalloc(gd, rb, keep, d_status=sb)
        torch.cuda.synchronize()
        assert int(sa.item()) == 0 and int(sb.item()) == 0
        assert torch.equal(oa, ob)
        K = int(oa[-1].item())
        assert K == gs.k_for(n, keep)
        assert torch.equal(ia[:K], ib[:K])
        assert np.array_equal(_bits(va[:K]), _bits(vb[:K]))
        assert np.array_equal(_bits(ra), _bits(rb))


def test_noalloc_rejects_sizes_above_its_maximum():
    n = gs.NOALLOC_MAX_N + 1
    g = torch.zeros(n, device="cuda")
    with pytest.raises(gs.GsparseError, match="unsupported"):
        gs.residual_topk_noalloc(g, g.clone(), (1, 100))


@pytest.mark.parametrize("keep", [(1, 10), (1, 1)])
def test_noalloc_near_its_maximum_with_a_large_keep(keep):
    # here the fixed array is far below the recommended workspace, so the call runs with small
    # candidate stores, no pool, and pieces re-read from the residual; the full-workspace call
    # must give the same result bit for bit
    n = gs.NOALLOC_MAX_N - 3
    assert gs.residual_topk_workspace_size(n, 1, keep) > 16 << 20
    g = synth.flat_mixture(n, seed=31)
    ra = torch.from_numpy(synth.gaussian(n, 32, sigma=1e-4)).cuda()
    rb = ra.clone()
    gd = torch.from_numpy(g).cuda()
    sa, sb = gs.status_tensor(), gs.status_tensor()
    ia, va, oa = gs.residual_topk(gd, ra, keep, d_status=sa)
    ib, vb, ob = gs.residual_topk_noalloc(gd, rb, keep, d_status=sb)
    torch.cuda.synchronize()
    assert int(sa.item()) == 0 and int(sb.item()) == 0
    assert torch.equal(oa, ob)
    K = int(oa[-1].item())
    assert K == gs.k_for(n, keep)
    assert torch.equal(ia[:K], ib[:K])
    assert np.array_equal(_bits(va[:K]), _bits(vb[:K]))
    assert np.array_equal(_bits(ra), _bits(rb))


def test_noalloc_at_its_maximum_against_the_oracle():
    # n = the maximum, keep 1/2: the reduced-capacity route, compared with the CPU oracle
    n, keep = gs.NOALLOC_MAX_N, (1, 2)
    g = synth.flat_mixture(n, seed=33)
    r = synth.gaussian(n, 34, sigma=1e-4)
    rd = torch.from_numpy(r).cuda()
    st = gs.status_tensor()
    gi, gv, go = gs.residual_topk_noalloc(torch.from_numpy(g).cuda(), rd, keep, d_status=st)
    torch.cuda.synchronize()
    wi, wv, wo, wr = oracle.residual_topk(g, r, keep)
    assert int(st.item()) == 0
    assert np.array_equal(go.cpu().numpy(), wo)
    K = int(wo[-1])
    assert np.array_equal(gi[:K].cpu().numpy(), wi)
    assert np.array_equal(_bits(gv[:K]), wv.view(np.uint32))
    assert np.array_equal(_bits(rd), wr.view(np.uint32))
