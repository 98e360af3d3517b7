"""CUDA path vs the CPU oracle, element by element, on seeded inputs (bit-exact on indices,
counts, residuals, bitstreams; fp32 means and sums are compared bitwise too, which is stricter
than the 1e-6 relative bound)."""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests.gpu_util import bits, dev, gpu_binarize, gpu_topk, host

import compressed_sgd_b200 as gs

pytestmark = pytest.mark.gpu


def assert_topk_equal(got, want):
    gi, gv, go, gr, st = got
    wi, wv, wo, wr = want
    assert st == 0
    assert np.array_equal(go, wo), (go, wo)
    assert np.array_equal(gi, wi)
    assert np.array_equal(bits(gv), bits(wv))
    assert np.array_equal(bits(gr), bits(wr))


# ------------------------------------------------------------------------------------ top-k

SIZES = [0, 1, 2, 5, 31, 32, 33, 127, 1000, 4097, 65537, 300001, (1 << 20) + 3]
KEEPS = [(1, 100), (1, 10), (1, 2), (1, 1), (0, 1), (1, 1000), (7, 9)]


@pytest.mark.parametrize("n", SIZES)
def test_topk_global_sizes(n):
    g = synth.gaussian(n, n)
    r = synth.gaussian(n, n + 1, sigma=3e-4)
    for keep in KEEPS:
        assert_topk_equal(gpu_topk(g, r, keep), oracle.residual_topk(g, r, keep))


@pytest.mark.parametrize("seed", range(4))
def test_topk_ties_and_zeros(seed):
    n = 20000 + 977 * seed
    g = synth.tied_values(n, seed, levels=3, zero_frac=0.3)
    r = synth.tied_values(n, seed + 50, levels=2, zero_frac=0.6)
    for keep in [(1, 100), (1, 4), (1, 2), (9, 10), (1, 1)]:
        assert_topk_equal(gpu_topk(g, r, keep), oracle.residual_topk(g, r, keep))


def test_topk_all_zero_and_constant():
    n = 50001
    z = np.zeros(n, np.float32)
    for keep in [(1, 100), (1, 2)]:
        assert_topk_equal(gpu_topk(z, z, keep), oracle.residual_topk(z, z, keep))
    c = np.full(n, -0.5, np.float32)
    assert_topk_equal(gpu_topk(c, z, (1, 7)), oracle.residual_topk(c, z, (1, 7)))


@pytest.mark.parametrize("layout", [
    [37, 1, 500, 64, 0, 1023],
    [0, 0, 5],
    [100000, 3, 250000, 1],
    [16384, 16385, 16383, 70000],
    [1] * 200,
])
def test_topk_per_segment(layout):
    seg = np.concatenate([[0], np.cumsum(layout)]).astype(np.int64)
    n = int(seg[-1])
    g = synth.gaussian(n, 7)
    r = synth.tied_values(n, 8, levels=3) * np.float32(1e-3)
    for keep in [(1, 100), (1, 10), (1, 1), (0, 1)]:
        assert_topk_equal(gpu_topk(g, r, keep, seg=seg), oracle.residual_topk(g, r, keep, seg=seg))


@pytest.mark.parametrize("route", ["exhaustive", "min_workspace", "tiny_workspace"])
def test_topk_fallback_routes_identical(route):
    n = 400003
    g = synth.flat_mixture(n, seed=3)
    r = synth.gaussian(n, 4, sigma=1e-4)
    seg = np.array([0, 1000, 200000, n], np.int64)
    for keep, s in [((1, 100), None), ((1, 10), seg), ((1, 2), None)]:
        T = 1 if s is None else len(s) - 1
        kw = {}
        if route == "exhaustive":
            kw["flags"] = gs.GSPARSE_SELECT_EXHAUSTIVE
        elif route == "min_workspace":
            kw["workspace_bytes"] = int(gs.lib().gsparse_residual_topk_workspace_min(n, T))
        else:
            kw["workspace_bytes"] = int(gs.lib().gsparse_residual_topk_workspace_min(n, T)) + 64 * 1024
        assert_topk_equal(gpu_topk(g, r, keep, seg=s, **kw), oracle.residual_topk(g, r, keep, seg=s))


def test_topk_sample_threshold_too_high_is_redone():
    # a segment whose sampled runs miss a dense block of large values: the sampled threshold
    # leaves fewer than k candidates and the segment is redone exhaustively
    n = 1 << 20
    g = synth.gaussian(n, 11, sigma=1e-6)
    g[777000:777000 + 20000] = synth.gaussian(20000, 12, sigma=1.0)
    r = np.zeros(n, np.float32)
    assert_topk_equal(gpu_topk(g, r, (1, 60)), oracle.residual_topk(g, r, (1, 60)))


def clustered_rows(n, seed, row=512, frac_rows=0.6, tokens=1000):
    """Embedding-like gradient: rows of `row` entries, only the rows of Zipf-drawn token ids are
    non-zero (N(0, 1e-2^2)) in the first `frac_rows` of the vector; the rest is dense N(0, 1e-4^2).
    The large entries come in long runs, so whole pieces of the streaming pass are candidates."""
    gen = synth.rng(seed, 91)
    m = int(n * frac_rows) // row
    g = synth.normal(gen, n, 1e-4)
    g[:m * row] = 0.0
    rows = np.unique(synth.zipf_ids(gen, tokens, m, 1.1))
    for r_ in rows:
        g[r_ * row:(r_ + 1) * row] = synth.normal(gen, row, 1e-2)
    return g


@pytest.mark.parametrize("pool", [1.0, 0.6, 0.3, 0.0])
def test_topk_clustered_candidates_pool_and_reread(pool):
    # candidates concentrated in dense rows overflow the per-piece stores: they continue in pool
    # chunks, and pieces that find the pool empty are re-read; every split gives the same result
    n = (1 << 22) + 4321
    g = clustered_rows(n, 5)
    r = synth.gaussian(n, 6, sigma=1e-5)
    seg = np.array([0, 1 << 20, 3 << 20, n], np.int64)
    for keep, s in [((1, 100), None), ((1, 100), seg), ((1, 20), None)]:
        T = 1 if s is None else len(s) - 1
        lo = int(gs.lib().gsparse_residual_topk_workspace_min(n, T))
        hi = int(gs.lib().gsparse_residual_topk_workspace_size(n, T, *keep))
        ws = lo + int((hi - lo) * pool) if pool < 1.0 else None
        assert_topk_equal(gpu_topk(g, r, keep, seg=s, workspace_bytes=ws), oracle.residual_topk(g, r, keep, seg=s))


def test_binarize_clustered_candidates():
    n = (1 << 21) + 77
    g = clustered_rows(n, 8, frac_rows=0.8)
    r = np.zeros(n, np.float32)
    for keep in [(1, 10), (1, 4)]:
        lo = int(gs.lib().gsparse_binarize_workspace_min(n, 1, *keep))
        hi = int(gs.lib().gsparse_binarize_workspace_size(n, 1, *keep))
        for ws in [None, lo + (hi - lo) // 3]:
            assert_binarize_equal(gpu_binarize(g, r, keep, workspace_bytes=ws), oracle.binarize(g, r, keep))


def test_topk_multi_step_residual_carried():
    lay = synth.mlp_layout()
    seg = synth.offsets(lay)
    n = int(seg[-1])
    r_o = np.zeros(n, np.float32)
    rd = dev(r_o)
    for step in range(4):
        g = synth.mlp_gradient(0, step)
        wi, wv, wo, r_o = oracle.residual_topk(g, r_o, (1, 100), seg=seg)
        idx, val, off = gs.residual_topk(dev(g), rd, (1, 100), seg_offsets=dev(seg))
        K = int(host(off)[-1])
        assert np.array_equal(host(off), wo)
        assert np.array_equal(host(idx)[:K], wi)
        assert np.array_equal(bits(host(val)[:K]), bits(wv))
        assert np.array_equal(bits(host(rd)), bits(r_o))


# --------------------------------------------------------- momentum correction and momentum masking

def gpu_topk_momentum(g, u, m, r, keep, seg=None, flags=0, workspace_bytes=None):
    gd, ud, rd = dev(g), dev(u), dev(r)
    segd = None if seg is None else dev(np.asarray(seg, np.int64))
    st = gs.status_tensor()
    ws = None
    if workspace_bytes is not None:
        ws = torch.empty(max(workspace_bytes, 256), dtype=torch.uint8, device="cuda")
    idx, val, off = gs.residual_topk(gd, rd, keep, seg_offsets=segd, flags=flags, workspace=ws, d_status=st,
                                     momentum=(ud, m))
    offh = host(off)
    K = int(offh[-1])
    return host(idx)[:K], host(val)[:K], offh, host(rd), host(ud), int(host(st)[0])


def assert_momentum_equal(got, want):
    gi, gv, go, gr, gu, st = got
    wi, wv, wo, wr, wu = want
    assert st == 0
    assert np.array_equal(go, wo)
    assert np.array_equal(gi, wi)
    assert np.array_equal(bits(gv), bits(wv))
    assert np.array_equal(bits(gr), bits(wr))
    assert np.array_equal(bits(gu), bits(wu))


@pytest.mark.parametrize("n", [1, 1000, 300001, (1 << 21) + 3])
def test_topk_momentum_multi_step(n):
    for m, keep in [(0.9, (1, 100)), (0.5, (1, 10)), (0.0, (1, 100)), (0.9, (1, 1)), (0.9, (0, 1))]:
        u = np.zeros(n, np.float32)
        r = np.zeros(n, np.float32)
        for step in range(3):
            g = synth.flat_mixture(n, seed=10 + step)
            want = oracle.residual_topk_momentum(g, u, m, r, keep)
            got = gpu_topk_momentum(g, u, m, r, keep)
            assert_momentum_equal(got, want)
            r, u = want[3], want[4]


@pytest.mark.parametrize("route", ["default", "exhaustive", "min_workspace", "clustered"])
def test_topk_momentum_segments_and_routes(route):
    n = (1 << 20) + 77
    g = clustered_rows(n, 21) if route == "clustered" else synth.flat_mixture(n, seed=21)
    u = synth.gaussian(n, 22, sigma=1e-3)
    r = synth.gaussian(n, 23, sigma=1e-4)
    seg = np.array([0, 5000, 600000, n], np.int64)
    for keep, s in [((1, 100), None), ((1, 50), seg)]:
        T = 1 if s is None else len(s) - 1
        kw = {}
        if route == "exhaustive":
            kw["flags"] = gs.GSPARSE_SELECT_EXHAUSTIVE
        elif route == "min_workspace":
            kw["workspace_bytes"] = int(gs.lib().gsparse_residual_topk_workspace_min(n, T))
        assert_momentum_equal(gpu_topk_momentum(g, u, 0.9, r, keep, seg=s, **kw),
                              oracle.residual_topk_momentum(g, u, 0.9, r, keep, seg=s))


def test_topk_momentum_with_pending_writes():
    # the quantisation error of the previous step arrives as pending writes to the residual
    n = 500003
    keep = (1, 100)
    u = np.zeros(n, np.float32)
    r = np.zeros(n, np.float32)
    ud, rd = dev(u), dev(r)
    st = gs.status_tensor()
    pend = None
    keep_alive = []
    for step in range(3):
        g = synth.flat_mixture(n, seed=40 + step)
        idx, val, off, r_o, u_o = oracle.residual_topk_momentum(g, u, 0.9, r, keep)
        _, _, qv, r_o = oracle.quantize(idx, val, residual=r_o, write_dequantized=True)
        gi, gv, go = gs.residual_topk(dev(g), rd, keep, d_status=st, pending=pend, momentum=(ud, 0.9))
        K = int(host(go)[-1])
        fb = torch.empty(max(K, 1), device="cuda")
        gs.quantize(gi, gv, go[1:2], write_dequantized=True, feedback_out=fb, d_status=st, capacity=gi.numel())
        pend = gs.make_pending(gi, fb, go[1:2], capacity=gi.numel())
        keep_alive.append((gi, gv, go, fb))
        assert int(host(st)[0]) == 0
        assert np.array_equal(host(gi)[:K], idx) and np.array_equal(bits(host(gv)[:K]), bits(qv))
        assert np.array_equal(bits(host(ud)), bits(u_o))
        u, r = u_o, r_o
    # the last feedback is still pending: applying it must give the oracle's residual
    gs.residual_topk(torch.zeros(n, device="cuda"), rd, (0, 1), d_status=st, pending=pend)
    assert np.array_equal(bits(host(rd)), bits(r))


def test_topk_momentum_argument_errors():
    n = 1024
    g = torch.zeros(n, device="cuda")
    r = torch.zeros(n, device="cuda")
    with pytest.raises(RuntimeError):
        gs.residual_topk(g, r, (1, 100), momentum=(r, 0.9))   # u aliases the residual
    with pytest.raises(RuntimeError):
        gs.residual_topk(g, r, (1, 100), momentum=(torch.zeros(n + 1, device="cuda")[1:], 0.9))  # misaligned


def test_topk_warmup_schedule_carried_residual():
    # keep fractions 25% -> 0.1% over the warm-up (large k first), residual carried
    n = (1 << 21) + 11
    r = np.zeros(n, np.float32)
    for t in range(6):
        keep = gs.warmup_keep(t, 4)
        assert keep == oracle.warmup_keep(t, 4)
        g = synth.flat_mixture(n, seed=60 + t)
        want = oracle.residual_topk(g, r, keep)
        assert_topk_equal(gpu_topk(g, r, keep), want)
        r = want[3]


def test_topk_bad_segments_and_capacity_flagged():
    n = 1000
    g = synth.gaussian(n, 1)
    r = np.zeros(n, np.float32)
    _, _, _, rr, st = gpu_topk(g, r, (1, 10), seg=np.array([0, 600, 500, n], np.int64))
    assert st & gs.DERR_SEGMENTS and np.array_equal(rr, r)     # nothing touched
    _, _, _, rr, st = gpu_topk(g, r, (1, 10), seg=np.array([0, 600, n - 1], np.int64))
    assert st & gs.DERR_SEGMENTS
    _, _, _, rr, st = gpu_topk(g, r, (1, 10), capacity=50)
    assert st & gs.DERR_CAPACITY and np.array_equal(rr, r)


def test_topk_host_argument_errors():
    x = torch.zeros(16, device="cuda")
    with pytest.raises(gs.GsparseError):
        gs.residual_topk(x, x, (2, 1))                      # keep fraction above 1
    with pytest.raises(gs.GsparseError):
        gs.residual_topk(x[1:], x[1:], (1, 2))              # misaligned
    with pytest.raises(gs.GsparseError):
        ws = torch.empty(64, dtype=torch.uint8, device="cuda")
        gs.residual_topk(x, x.clone(), (1, 2), workspace=ws)


# ------------------------------------------------------------------------------------ quantise

@pytest.mark.parametrize("K", [0, 1, 31, 33, 255, 256, 257, 5000, 70001, 600000])
def test_quantize_parity(K):
    n = max(4 * K, 1)
    gen = np.random.default_rng(K)
    idx = np.sort(gen.choice(n, K, replace=False)).astype(np.int32)
    val = synth.gaussian(K, K, sigma=1e-2)
    if K > 10:
        val[::11] = 0.0
        val[5::13] = -0.0
    res = synth.gaussian(n, 3, sigma=1e-4)
    wb, wm, wval, wres = oracle.quantize(idx, val, residual=res, write_dequantized=True)
    vd, rd = dev(val), dev(res)
    end = torch.tensor([K], dtype=torch.int64, device="cuda")
    st = gs.status_tensor()
    sb, means = gs.quantize(dev(idx), vd, end, residual=rd, write_dequantized=True, d_status=st, capacity=K)
    assert int(host(st)[0]) == 0
    assert np.array_equal(bits(host(means)), bits(wm))
    assert np.array_equal(host(sb)[:(K + 31) // 32].view(np.uint32), wb)
    assert np.array_equal(bits(host(vd)), bits(wval))
    assert np.array_equal(bits(host(rd)), bits(wres))


def test_quantize_sublist_with_begin_end():
    K = 3000
    idx = np.arange(0, 3 * K, 3, dtype=np.int32)
    val = synth.gaussian(K, 5, sigma=1e-2)
    b, e = 700, 2333
    wb, wm, _, _ = oracle.quantize(idx[b:e], val[b:e])
    sb, means = gs.quantize(dev(idx), dev(val), torch.tensor([e], device="cuda"),
                            d_begin=torch.tensor([b], device="cuda"), capacity=K)
    assert np.array_equal(bits(host(means)), bits(wm))
    assert np.array_equal(host(sb)[:(e - b + 31) // 32].view(np.uint32), wb)


# ------------------------------------------------------------------------------------ binarise

def assert_binarize_equal(got, want):
    gi, gv, gm, go, gr, st = got
    wi, wv, wm, wo, wr = want
    assert st == 0
    assert np.array_equal(go, wo)
    assert np.array_equal(gi, wi)
    assert np.array_equal(bits(gm), bits(wm))
    assert np.array_equal(bits(gv), bits(wv))
    assert np.array_equal(bits(gr), bits(wr))


@pytest.mark.parametrize("n", [1, 2, 33, 1000, 65537, 300001, (1 << 20) + 5])
def test_binarize_global(n):
    g = synth.gaussian(n, n, sigma=1e-2)
    r = synth.gaussian(n, n + 2, sigma=1e-3)
    for keep in [(1, 1000), (1, 100), (1, 3), (1, 1)]:
        assert_binarize_equal(gpu_binarize(g, r, keep), oracle.binarize(g, r, keep))


def test_binarize_skewed_ties_segments_and_routes():
    n = 200000
    g = synth.tied_values(n, 4, levels=3, zero_frac=0.2)
    g[: n // 2] = np.abs(g[: n // 2])
    r = np.zeros(n, np.float32)
    seg = np.array([0, 10, 10, 150000, n], np.int64)
    for keep in [(1, 1000), (1, 50), (1, 2)]:
        want = oracle.binarize(g, r, keep, seg=seg)
        assert_binarize_equal(gpu_binarize(g, r, keep, seg=seg), want)
        assert_binarize_equal(gpu_binarize(g, r, keep, seg=seg, flags=gs.GSPARSE_SELECT_EXHAUSTIVE), want)
        mn = int(gs.lib().gsparse_binarize_workspace_min(n, 4, *keep))
        assert_binarize_equal(gpu_binarize(g, r, keep, seg=seg, workspace_bytes=mn), want)


@pytest.mark.parametrize("n", [1, 2, 1000, 300001, (1 << 21) + 9])
def test_binarize_by_magnitude(n):
    # the magnitude-first reading: top fraction by |acc|, then the sign with the larger mean
    r = np.zeros(n, np.float32)
    for step, keep in enumerate([(1, 1000), (1, 100), (1, 10), (1, 1)]):
        g = synth.gaussian(n, 300 + step, sigma=1e-2) + np.float32(2e-3)   # a sign imbalance
        want = oracle.binarize(g, r, keep, by_magnitude=True)
        assert_binarize_equal(gpu_binarize(g, r, keep, by_magnitude=True), want)
        r = want[4]


@pytest.mark.parametrize("route", ["segments", "exhaustive", "min_workspace", "ties"])
def test_binarize_by_magnitude_routes(route):
    n = 400009
    g = synth.gaussian(n, 310, sigma=1e-2)
    r = synth.gaussian(n, 311, sigma=1e-3)
    seg = None
    kw = {}
    if route == "segments":
        seg = np.array([0, 17, 1000, 250000, 250000, n], np.int64)
    elif route == "exhaustive":
        kw["flags"] = gs.GSPARSE_SELECT_EXHAUSTIVE
    elif route == "ties":
        g = synth.tied_values(n, 312, levels=4) * np.float32(1e-2)
        r = np.zeros(n, np.float32)
    for keep in [(1, 100), (1, 7)]:
        if route == "min_workspace":
            kw["workspace_bytes"] = int(gs.lib().gsparse_binarize_workspace_min(n, 1, *keep))
        assert_binarize_equal(gpu_binarize(g, r, keep, seg=seg, by_magnitude=True, **kw),
                              oracle.binarize(g, r, keep, seg=seg, by_magnitude=True))


def test_binarize_one_sign_only():
    n = 5000
    g = np.abs(synth.gaussian(n, 1))
    r = np.zeros(n, np.float32)
    assert_binarize_equal(gpu_binarize(g, r, (1, 100)), oracle.binarize(g, r, (1, 100)))
    assert_binarize_equal(gpu_binarize(-g, r, (1, 100)), oracle.binarize(-g, r, (1, 100)))
    z = np.zeros(n, np.float32)
    assert_binarize_equal(gpu_binarize(z, z, (1, 100)), oracle.binarize(z, z, (1, 100)))


# ------------------------------------------------------------------------------------ Golomb

@pytest.mark.parametrize("b", [0, 1, 3, 6, 9, 15, 30])
@pytest.mark.parametrize("K", [0, 1, 31, 32, 33, 1000, 65537])
def test_golomb_parity(b, K):
    n = 1 << 22 if b else 1 << 14
    gen = np.random.default_rng(b * 1000 + K)
    idx = np.sort(gen.choice(n, min(K, n), replace=False)).astype(np.int32)
    K = idx.size
    base = 0
    wwords, wbits, wtable = oracle.golomb_encode(idx, b, base, chunk=64)
    end = torch.tensor([K], dtype=torch.int64, device="cuda")
    st = gs.status_tensor()
    words, nbits, table = gs.golomb_encode(dev(idx), end, b, n, base=base, chunk=64, d_status=st, capacity=K)
    nb = int(host(nbits)[0])
    assert int(host(st)[0]) == 0 and nb == wbits
    assert np.array_equal(host(words)[:(nb + 31) // 32].view(np.uint32), wwords)
    if K:
        assert np.array_equal(host(table)[: wtable.shape[0]], wtable)
    out = gs.golomb_decode(words, nbits, end, K, b, base=base, table=table, chunk=64, n_limit=n, d_status=st)
    assert int(host(st)[0]) == 0
    assert np.array_equal(host(out)[:K], idx)
    out2 = gs.golomb_decode(words, nbits, end, K, b, base=base, table=None, n_limit=n, d_status=st)
    assert np.array_equal(host(out2)[:K], idx)


@pytest.mark.parametrize("chunk", [4, 7, 64])
@pytest.mark.parametrize("b, K", [(3, (1 << 20) + 7), (9, 25_558), (0, 4097)])
def test_golomb_parity_chunks_and_list_lengths(b, K, chunk):
    # short lists (2 codewords per encoding thread) and long ones (8), small and odd side-table
    # chunks (the decoder's 16-byte output path and its scalar tail)
    n = 1 << 27 if b else 1 << 14
    gen = np.random.default_rng(b * 7 + K + chunk)
    idx = np.unique(gen.integers(0, n, size=int(K * 1.2)))[:K].astype(np.int32)
    K = idx.size
    wwords, wbits, wtable = oracle.golomb_encode(idx, b, 0, chunk=chunk)
    end = torch.tensor([K], dtype=torch.int64, device="cuda")
    st = gs.status_tensor()
    words, nbits, table = gs.golomb_encode(dev(idx), end, b, n, chunk=chunk, d_status=st, capacity=K)
    nb = int(host(nbits)[0])
    assert int(host(st)[0]) == 0 and nb == wbits
    assert np.array_equal(host(words)[:(nb + 31) // 32].view(np.uint32), wwords)
    assert np.array_equal(host(table)[: wtable.shape[0]], wtable)
    out = gs.golomb_decode(words, nbits, end, K, b, table=table, chunk=chunk, n_limit=n, d_status=st)
    assert int(host(st)[0]) == 0
    assert np.array_equal(host(out)[:K], idx)


def test_golomb_huge_gaps_and_base():
    idx = np.array([5, 6, 100000, 100001, 2_000_000_000], np.int32)
    for b in [0, 2, 20]:
        ww, wb, wt = oracle.golomb_encode(idx, b, base=5, chunk=2)
        end = torch.tensor([idx.size], device="cuda")
        words, nbits, table = gs.golomb_encode(dev(idx), end, b, 2**31 - 1, base=5, chunk=2)
        nb = int(host(nbits)[0])
        assert nb == wb and np.array_equal(host(words)[:(nb + 31) // 32].view(np.uint32), ww)
        out = gs.golomb_decode(words, nbits, end, idx.size, b, base=5, table=table, chunk=2)
        assert np.array_equal(host(out)[: idx.size], idx)


def test_golomb_corrupt_streams_flagged():
    idx = np.sort(np.random.default_rng(0).choice(100000, 3000, replace=False)).astype(np.int32)
    end = torch.tensor([idx.size], device="cuda")
    words, nbits, table = gs.golomb_encode(dev(idx), end, 6, 100000, chunk=32)
    # truncated stream
    st = gs.status_tensor()
    short = nbits - 5
    gs.golomb_decode(words, short, end, idx.size, 6, table=table, chunk=32, d_status=st)
    assert int(host(st)[0]) & gs.DERR_CORRUPT_STREAM
    # flipped bits (host-made corruption), both decoders: flagged or, if still a valid code,
    # the decoded indices differ; never a fault
    for flip in [3, 1000, 7777]:
        w = words.clone()
        w.view(torch.int32)[flip // 32] ^= (1 << (flip % 32))
        for tb in [table, None]:
            st = gs.status_tensor()
            out = gs.golomb_decode(w, nbits, end, idx.size, 6, table=tb, chunk=32, n_limit=100000, d_status=st)
            s = int(host(st)[0])
            assert s != 0 or not np.array_equal(host(out)[: idx.size], idx)
    # not ascending
    bad = idx.copy()
    bad[10] = bad[9]
    st = gs.status_tensor()
    gs.golomb_encode(dev(bad), end, 6, 100000, d_status=st)
    assert int(host(st)[0]) & gs.DERR_INDEX_RANGE


# ------------------------------------------------------------------------------------ scatter

@pytest.mark.parametrize("W", [1, 2, 4, 8])
@pytest.mark.parametrize("n", [1, 8191, 8192, 100003])
def test_scatter_parity(W, n):
    gen = np.random.default_rng(W * n)
    host_lists, lists, keep = [], [], []
    for w in range(W):
        k = int(min(n, gen.integers(0, max(n // 10, 2))))
        idx = np.sort(gen.choice(n, k, replace=False)).astype(np.int32)
        val = synth.gaussian(k, w, sigma=1e-2)
        cnt = torch.tensor([k], dtype=torch.int64, device="cuda")
        if w == 1:   # a binarised worker: one value for every entry
            u = torch.tensor([0.125], device="cuda")
            host_lists.append((idx, None, np.float32(0.125)))
            t = (dev(idx), cnt, u)
            lists.append(gs.make_list(t[0], cnt, uniform_val=u, capacity=k))
        else:
            host_lists.append((idx, val))
            t = (dev(idx), cnt, dev(val))
            lists.append(gs.make_list(t[0], cnt, val=t[2], capacity=k))
        keep.append(t)
    wd, wi, wv = oracle.scatter_accumulate(host_lists, n)
    st = gs.status_tensor()
    dense, mi, mv, mc = gs.scatter_accumulate(lists, n, merged=True, d_status=st)
    assert int(host(st)[0]) == 0
    assert np.array_equal(bits(host(dense)[:n]), bits(wd))
    U = int(host(mc)[0])
    assert U == wi.size
    assert np.array_equal(host(mi)[:U], wi)
    assert np.array_equal(bits(host(mv)[:U]), bits(wv))


def test_scatter_bad_indices_flagged():
    n = 1000
    idx = torch.tensor([5, 3, 7], dtype=torch.int32, device="cuda")
    val = torch.ones(3, device="cuda")
    cnt = torch.tensor([3], device="cuda")
    st = gs.status_tensor()
    gs.scatter_accumulate([gs.make_list(idx, cnt, val=val)], n, d_status=st)
    assert int(host(st)[0]) & gs.DERR_INDEX_RANGE
    idx = torch.tensor([5, 3000], dtype=torch.int32, device="cuda")
    st = gs.status_tensor()
    gs.scatter_accumulate([gs.make_list(idx, torch.tensor([2], device="cuda"), val=val[:2])], n, d_status=st)
    assert int(host(st)[0]) & gs.DERR_INDEX_RANGE


# ------------------------------------------------------------------------------------ combine

@pytest.mark.parametrize("n", [1, 3, 4, 1000, 100001])
def test_combine_parity(n):
    G = synth.gaussian(n, 1, sigma=1e-2)
    L = synth.gaussian(n, 2, sigma=1e-2)
    for alpha, beta in [(1.0, 1.0), (0.25, 0.25), (0.0, 0.5), (1.0 / 3, 0.7)]:
        want = oracle.combine_local(G, L, alpha, beta)
        got = gs.combine_local(dev(G), dev(L), alpha=alpha, beta=beta)
        assert np.array_equal(bits(host(got)), bits(want))
    k = max(n // 7, 1)
    own_idx = np.sort(np.random.default_rng(n).choice(n, k, replace=False)).astype(np.int32)
    own_val = synth.gaussian(k, 9, sigma=1e-2)
    want = oracle.combine_local(G, L, 1.0, 1.0, mode=1, own_idx=own_idx, own_val=own_val)
    got = gs.combine_local(dev(G), dev(L), mode=1, own_idx=dev(own_idx), own_val=dev(own_val),
                           own_count=torch.tensor([k], device="cuda"), own_capacity=k)
    assert np.array_equal(bits(host(got)), bits(want))


# ------------------------------------------------------------------------------------ fused receive

@pytest.mark.parametrize("W", [1, 2, 4, 8])
@pytest.mark.parametrize("n", [3, 8192, 8193, 200003])
def test_accumulate_combine_parity(W, n):
    gen = np.random.default_rng(77 * W + n)
    host_lists, lists, keep = [], [], []
    for w in range(W):
        k = int(min(n, gen.integers(1, max(n // 10, 2) + 1)))
        idx = np.sort(gen.choice(n, k, replace=False)).astype(np.int32)
        val = synth.gaussian(k, 40 + w, sigma=1e-2)
        cnt = torch.tensor([k], dtype=torch.int64, device="cuda")
        t = (dev(idx), cnt, dev(val))
        keep.append(t)
        host_lists.append((idx, val))
        lists.append(gs.make_list(t[0], cnt, val=t[2], capacity=k))
    Lh = synth.gaussian(n, 5, sigma=1e-2)
    L = dev(Lh)
    wd, _, _ = oracle.scatter_accumulate(host_lists, n, merged=False)
    for alpha, beta in [(1.0, 1.0), (0.25, 0.75)]:
        for mode in (0, 1):
            own = W - 1 if mode == 1 else -1
            kw = {} if mode == 0 else {"own_idx": host_lists[own][0], "own_val": host_lists[own][1]}
            want = oracle.combine_local(wd, Lh, alpha, beta, mode=mode, **kw)
            dense = torch.empty(n, device="cuda")
            st = gs.status_tensor()
            out = gs.accumulate_combine(lists, n, L, alpha=alpha, beta=beta, mode=mode, own=own, dense_out=dense,
                                        d_status=st)
            assert int(host(st)[0]) == 0
            assert np.array_equal(bits(host(out)), bits(want))
            assert np.array_equal(bits(host(dense)), bits(wd))
            out2 = gs.accumulate_combine(lists, n, L, alpha=alpha, beta=beta, mode=mode, own=own)
            assert np.array_equal(bits(host(out2)), bits(want))


def test_accumulate_combine_crowded_tiles():
    # most entries of every worker fall in a few tiles (dense rows), the rest are spread thin:
    # tiles are taken dynamically and crowded ones walk thousands of entries per worker
    n = (1 << 22) + 999
    W = 4
    gen = np.random.default_rng(4242)
    host_lists, lists, keep = [], [], []
    for w in range(W):
        dense_part = gen.choice(np.arange(50000, 50000 + 40000), 30000, replace=False)
        sparse_part = gen.choice(n, 20000, replace=False)
        idx = np.unique(np.concatenate([dense_part, sparse_part])).astype(np.int32)
        val = synth.gaussian(idx.size, 60 + w, sigma=1e-2)
        cnt = torch.tensor([idx.size], dtype=torch.int64, device="cuda")
        t = (dev(idx), cnt, dev(val))
        keep.append(t)
        host_lists.append((idx, val))
        lists.append(gs.make_list(t[0], cnt, val=t[2], capacity=idx.size))
    Lh = synth.gaussian(n, 9, sigma=1e-2)
    wd, _, _ = oracle.scatter_accumulate(host_lists, n, merged=False)
    for mode in (0, 1):
        own = 1 if mode == 1 else -1
        kw = {} if mode == 0 else {"own_idx": host_lists[own][0], "own_val": host_lists[own][1]}
        want = oracle.combine_local(wd, Lh, 1.0, 1.0, mode=mode, **kw)
        st = gs.status_tensor()
        dense = torch.empty(n, device="cuda")
        out = gs.accumulate_combine(lists, n, dev(Lh), mode=mode, own=own, dense_out=dense, d_status=st)
        assert int(host(st)[0]) == 0
        assert np.array_equal(bits(host(out)), bits(want))
        assert np.array_equal(bits(host(dense)), bits(wd))


# ------------------------------------------------------------------------------------ pending writes

@pytest.mark.parametrize("mode", ["global", "per_tensor", "delay"])
def test_quantisation_feedback_as_pending_writes_matches_immediate(mode):
    """Quantise with feedback_out, hand (idx, feedback) to the next residual_topk as pending writes:
    after every top-k the residual and the outputs equal the oracle chain that writes the
    quantisation error into the residual at once."""
    lay = [70000, 3, 130001, 64] if mode == "per_tensor" else [200071]
    seg = np.concatenate([[0], np.cumsum(lay)]).astype(np.int64)
    n, T = int(seg[-1]), len(lay)
    seg_arg = seg if mode == "per_tensor" else None
    r_o = np.zeros(n, np.float32)
    r_d = torch.zeros(n, device="cuda")
    pend = None
    keepalive = []
    st = gs.status_tensor()
    for step in range(6):
        keep = (0, 1) if (mode == "delay" and step % 2 == 1) else (1, 50)
        g = synth.flat_mixture(n, seed=300 + step)
        wi, wv, wo, r_o = oracle.residual_topk(g, r_o, keep, seg=seg_arg)
        idx, val, off = gs.residual_topk(dev(g), r_d, keep, seg_offsets=None if seg_arg is None else dev(seg),
                                         d_status=st, pending=pend)
        K = int(wo[-1])
        assert np.array_equal(host(off), wo), step
        assert np.array_equal(host(idx)[:K], wi), step
        assert np.array_equal(bits(host(val)[:K]), bits(wv)), step
        assert np.array_equal(bits(host(r_d)), bits(r_o)), step
        pend = None
        if K:
            fb = torch.empty(idx.numel(), device="cuda")
            for s in range(T):
                b, e = int(wo[s]), int(wo[s + 1])
                _, _, wv_s, r_o = oracle.quantize(wi[b:e], wv[b:e], residual=r_o, write_dequantized=True)
                gs.quantize(idx, val, off[s + 1:s + 2], d_begin=off[s:s + 1], write_dequantized=True,
                            feedback_out=fb[b:], d_status=st, capacity=idx.numel())
            pend = gs.make_pending(idx, fb, off[T:T + 1])
            keepalive.append((idx, val, off, fb))
    assert int(host(st)[0]) == 0


def test_pending_writes_must_be_ascending():
    n = 5000
    g = synth.gaussian(n, 1)
    r = torch.zeros(n, device="cuda")
    pidx = torch.tensor([10, 20, 15], dtype=torch.int32, device="cuda")
    pval = torch.ones(3, device="cuda")
    st = gs.status_tensor()
    gs.residual_topk(dev(g), r, (1, 10), d_status=st,
                     pending=gs.make_pending(pidx, pval, torch.tensor([3], device="cuda")))
    assert int(host(st)[0]) & gs.DERR_INDEX_RANGE
    assert bool((r == 0).all())                       # nothing written


@pytest.mark.parametrize("defect", ["descent", "repeat", "past_n", "negative", "first_negative"])
def test_pending_writes_invalid_inside_a_long_list(defect):
    # the same check on a list long enough that the defect sits inside a full run of writes
    n = 200_000
    g = synth.gaussian(n, 3)
    r = torch.zeros(n, device="cuda")
    base = np.arange(1000, dtype=np.int64) * 150 + 7
    if defect == "descent":
        base[500] = base[499] - 3
    elif defect == "repeat":
        base[500] = base[499]
    elif defect == "past_n":
        base[500:] += n          # ascending, but out of range from entry 500 on
    elif defect == "negative":
        base[:501] -= base[500] + 1   # entries 0..500 negative, still ascending
    else:
        base[0] = -1
    pidx = torch.tensor(base.astype(np.int32), device="cuda")
    pval = torch.ones(1000, device="cuda")
    st = gs.status_tensor()
    gs.residual_topk(dev(g), r, (1, 10), d_status=st,
                     pending=gs.make_pending(pidx, pval, torch.tensor([1000], device="cuda")))
    assert int(host(st)[0]) & gs.DERR_INDEX_RANGE
    assert bool((r == 0).all())                       # nothing written


# ------------------------------------------------------------------- segmented quantisation

@pytest.mark.parametrize("layout", [[1000], [37, 0, 5000, 256, 1, 70001], [0], [300, 0, 0]])
def test_quantize_segments_parity(layout):
    # one call over T sub-lists equals T separate quantisations of the oracle, each with its own
    # two means; sign bits and feedback over positions from the first offset
    off = np.concatenate([[0], np.cumsum(layout)]).astype(np.int64)
    K = int(off[-1])
    n = max(3 * K, 1)
    gen = np.random.default_rng(K + len(layout))
    idx = np.sort(gen.choice(n, K, replace=False)).astype(np.int32)
    val = synth.gaussian(K, K + 7, sigma=1e-2)
    if K > 20:
        val[::17] = 0.0
        val[3::19] = -0.0
    res = synth.gaussian(n, 9, sigma=1e-4)
    want_res = res.copy()
    want_val = val.copy()
    want_bits = np.zeros(max((K + 31) // 32, 1), np.uint32)
    want_means = np.zeros(2 * len(layout), np.float32)
    for s in range(len(layout)):
        b, e = int(off[s]), int(off[s + 1])
        wb, wm, wv, want_res = oracle.quantize(idx[b:e], val[b:e], residual=want_res, write_dequantized=True)
        want_val[b:e] = wv
        want_means[2 * s:2 * s + 2] = wm
        for j in range(b, e):
            if val[j] < 0:
                want_bits[j // 32] |= np.uint32(1 << (j % 32))
    vd, rd = dev(val), dev(res)
    fb = torch.zeros(max(K, 1), device="cuda")
    st = gs.status_tensor()
    sb, means = gs.quantize_segments(dev(idx), vd, dev(off), residual=rd, write_dequantized=True, feedback_out=fb,
                                     d_status=st, capacity=K)
    assert int(host(st)[0]) == 0
    assert np.array_equal(bits(host(means)), bits(want_means))
    assert np.array_equal(host(sb)[:(K + 31) // 32].view(np.uint32), want_bits[:(K + 31) // 32])
    assert np.array_equal(bits(host(vd)), bits(want_val))
    assert np.array_equal(bits(host(rd)), bits(want_res))
    # the feedback list holds the same errors the residual received
    got_fb = host(fb)[:K]
    assert np.array_equal(bits(got_fb), bits(want_res[idx])) if K else True


def test_quantize_segments_bad_offsets_flagged():
    idx = dev(np.arange(100, dtype=np.int32))
    val = dev(synth.gaussian(100, 1))
    st = gs.status_tensor()
    gs.quantize_segments(idx, val, dev(np.array([0, 60, 40, 100], np.int64)), d_status=st, capacity=100)
    assert int(host(st)[0]) & gs.DERR_CAPACITY
    st = gs.status_tensor()
    gs.quantize_segments(idx, val, dev(np.array([0, 101], np.int64)), d_status=st, capacity=100)
    assert int(host(st)[0]) & gs.DERR_CAPACITY
