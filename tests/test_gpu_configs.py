"""The five workloads at full size, in the launch configuration bench.py uses (same entry points,
same sizes). Where the oracle finishes in seconds it is compared element by element; for the 2^30
workload the oracle checks worker 0 at the 99% drop and every other case is checked through
properties that hold at any size (exact k, the bitwise residual invariant, the threshold and
tie rule, Golomb round trip and closed-form length, the worker-ordered sum)."""
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import pytest
import torch

import oracle
import synth
from tests.gpu_util import bits, dev, host

import compressed_sgd_b200 as gs

pytestmark = pytest.mark.gpu


def check_topk_properties(g_d, r_old_d, r_new_d, idx_d, val_d, K):
    """Exact selection properties on the GPU (torch ops, independent of the library)."""
    acc = g_d + r_old_d                           # one IEEE fp32 add
    n = acc.numel()
    idx = idx_d[:K].long()
    assert K == 0 or bool((idx[1:] > idx[:-1]).all())
    mask = torch.zeros(n, dtype=torch.bool, device=acc.device)
    mask[idx] = True
    ab = acc.view(torch.int32)
    assert torch.equal(val_d[:K].view(torch.int32), ab[idx])
    assert bool((r_new_d.view(torch.int32)[mask] == 0).all())            # +0 exactly
    assert torch.equal(r_new_d.view(torch.int32)[~mask], ab[~mask])
    keys = ab & 0x7FFFFFFF
    if K == 0 or K == n:
        return
    T = int(keys[idx].min())
    assert int(keys[~mask].max()) <= T
    tie_in = torch.nonzero(mask & (keys == T)).flatten()
    tie_out = torch.nonzero(~mask & (keys == T)).flatten()
    if tie_out.numel() and tie_in.numel():
        assert int(tie_in.max()) < int(tie_out.min())


# ------------------------------------------------------------------------------------ 1

def test_config1_flat_mixture_exact():
    n = 1 << 20
    g = synth.flat_mixture(n, seed=0)
    r = np.zeros(n, np.float32)
    wi, wv, wo, wr = oracle.residual_topk(g, r, (1, 100))
    assert wi.size == 10486
    gd, rd = dev(g), dev(r)
    idx, val, off = gs.residual_topk(gd, rd, (1, 100))
    assert np.array_equal(host(off), wo)
    assert np.array_equal(host(idx)[:10486], wi)
    assert np.array_equal(bits(host(val)[:10486]), bits(wv))
    assert np.array_equal(bits(host(rd)), bits(wr))


# ------------------------------------------------------------------------------------ 2

@pytest.mark.parametrize("mode", ["per_tensor", "global"])
@pytest.mark.parametrize("quantise", [False, True])
def test_config2_mlp_50_steps_4_workers(mode, quantise):
    lay = synth.mlp_layout()
    seg = synth.offsets(lay)
    n, W, steps, keep = int(seg[-1]), 4, 50, (1, 100)
    seg_arg = seg if mode == "per_tensor" else None
    T = len(lay) if mode == "per_tensor" else 1
    seg_d = dev(seg) if seg_arg is not None else None
    r_host = [np.zeros(n, np.float32) for _ in range(W)]
    r_dev = [torch.zeros(n, device="cuda") for _ in range(W)]
    st = gs.status_tensor()

    def oracle_worker(w, g):
        oi, ov, oo, rr = oracle.residual_topk(g, r_host[w], keep, seg=seg_arg)
        if quantise:
            parts = []
            for s in range(T):
                b, e = int(oo[s]), int(oo[s + 1])
                bits_s, means_s, ov_s, rr = oracle.quantize(oi[b:e], ov[b:e], residual=rr, write_dequantized=True)
                parts.append((bits_s, means_s))
                ov[b:e] = ov_s
        else:
            parts = None
        r_host[w] = rr
        return oi, ov, oo, parts

    pool = ThreadPoolExecutor(W)
    for step in range(steps):
        grads = [synth.mlp_gradient(w, step) for w in range(W)]
        want = list(pool.map(lambda w: oracle_worker(w, grads[w]), range(W)))
        lists, keepalive = [], []
        for w in range(W):
            idx, val, off = gs.residual_topk(dev(grads[w]), r_dev[w], keep, seg_offsets=seg_d, d_status=st)
            segmented = quantise and step % 2 == 1   # odd steps: all tensors in one call
            if quantise and not segmented:
                qparts = []
                for s in range(T):
                    sb, mm = gs.quantize(idx, val, off[s + 1:s + 2], d_begin=off[s:s + 1], residual=r_dev[w],
                                         write_dequantized=True, d_status=st, capacity=idx.numel())
                    qparts.append((sb, mm))
            elif segmented:
                sb_all, mm_all = gs.quantize_segments(idx, val, off, residual=r_dev[w], write_dequantized=True,
                                                      d_status=st, capacity=idx.numel())
            oi, ov, oo, parts = want[w]
            K = int(oo[-1])
            assert np.array_equal(host(off), oo), (step, w)
            assert np.array_equal(host(idx)[:K], oi), (step, w)
            assert np.array_equal(bits(host(val)[:K]), bits(ov)), (step, w)
            assert np.array_equal(bits(host(r_dev[w])), bits(r_host[w])), (step, w)
            if quantise and not segmented:
                for s in range(T):
                    sb, mm = qparts[s]
                    wb, wm = parts[s]
                    assert np.array_equal(bits(host(mm)), bits(wm))
                    assert np.array_equal(host(sb)[:wb.size].view(np.uint32), wb)
            elif segmented:
                wm_all = np.concatenate([parts[s][1] for s in range(T)])
                assert np.array_equal(bits(host(mm_all)), bits(wm_all))
                neg = np.zeros(((K + 31) // 32) * 32, bool)
                neg[:K] = ov < 0
                want_words = np.packbits(neg.reshape(-1, 32)[:, ::-1], axis=1).view(">u4").ravel().astype(np.uint32)
                assert np.array_equal(host(sb_all)[:want_words.size].view(np.uint32), want_words)
            cnt = off[T:T + 1]
            lists.append(gs.make_list(idx, cnt, val=val))
            keepalive.append((idx, val, off))
        dense, mi, mv, mc = gs.scatter_accumulate(lists, n, merged=True, d_status=st)
        wd, wmi, wmv = oracle.scatter_accumulate([(want[w][0], want[w][1]) for w in range(W)], n)
        assert np.array_equal(bits(host(dense)[:n]), bits(wd))
        U = int(host(mc)[0])
        assert np.array_equal(host(mi)[:U], wmi) and np.array_equal(bits(host(mv)[:U]), bits(wmv))
    assert int(host(st)[0]) == 0


# ------------------------------------------------------------------------------------ 3

def test_config3_nmt_20_steps_4_workers_combine():
    n = int(synth.offsets(synth.nmt_layout())[-1])
    W, steps, keep = 4, 20, (1, 100)
    r_host = [np.zeros(n, np.float32) for _ in range(W)]
    r_dev = [torch.zeros(n, device="cuda") for _ in range(W)]
    st = gs.status_tensor()
    pool = ThreadPoolExecutor(W)
    for step in range(steps):
        grads = list(pool.map(lambda w: synth.nmt_gradient(w, step), range(W)))

        def oracle_worker(w):
            oi, ov, oo, rr = oracle.residual_topk(grads[w], r_host[w], keep)
            r_host[w] = rr
            return oi, ov
        want = list(pool.map(oracle_worker, range(W)))
        lists, outs = [], []
        g_dev = [dev(x) for x in grads]
        for w in range(W):
            idx, val, off = gs.residual_topk(g_dev[w], r_dev[w], keep, d_status=st)
            oi, ov = want[w]
            K = oi.size
            assert int(host(off)[-1]) == K
            assert np.array_equal(host(idx)[:K], oi), (step, w)
            assert np.array_equal(bits(host(val)[:K]), bits(ov)), (step, w)
            if step in (0, steps - 1) or w == 0:
                assert np.array_equal(bits(host(r_dev[w])), bits(r_host[w])), (step, w)
            lists.append(gs.make_list(idx, off[1:2], val=val))
            outs.append((idx, val, off))
        dense, _, _, _ = gs.scatter_accumulate(lists, n, d_status=st)
        wd, _, _ = oracle.scatter_accumulate(want, n, merged=False)
        assert np.array_equal(bits(host(dense)[:n]), bits(wd)), step
        if step in (0, steps - 1):
            for w in (0, W - 1):
                out = gs.combine_local(dense[:n], g_dev[w])
                assert np.array_equal(bits(host(out)), bits(oracle.combine_local(wd, grads[w])))
                idx, val, off = outs[w]
                K = want[w][0].size
                outp = gs.combine_local(dense[:n], g_dev[w], mode=1, own_idx=idx, own_val=val, own_count=off[1:2],
                                        own_capacity=K)
                wantp = oracle.combine_local(wd, grads[w], mode=1, own_idx=want[w][0], own_val=want[w][1])
                assert np.array_equal(bits(host(outp)), bits(wantp))
    assert int(host(st)[0]) == 0


# ------------------------------------------------------------------------------------ 4

def test_config4_resnet50_delay10_binarise_golomb_8_workers():
    lay = synth.resnet50_layout()
    n = int(synth.offsets(lay)[-1])
    assert len(lay) == 161 and n == 25_557_032
    W, delay, keep = 8, 10, (1, 1000)
    b = gs.golomb_b_star(0.001)
    assert b == 9
    st = gs.status_tensor()
    gpu_lists, host_lists, keepalive = [], [], []
    for w in range(W):
        r_o = np.zeros(n, np.float32)
        r = torch.zeros(n, device="cuda")
        for step in range(delay - 1):          # communication delay: accumulate only
            g = synth.resnet50_gradient(w, step)
            _, _, _, r_o = oracle.residual_topk(g, r_o, (0, 1))
            gs.residual_topk(dev(g), r, (0, 1), d_status=st)
        assert np.array_equal(bits(host(r)), bits(r_o))
        g = synth.resnet50_gradient(w, delay - 1)
        oi, ov, om, oo, rr = oracle.binarize(g, r_o, keep)
        idx, val, mean, off = gs.binarize(dev(g), r, keep, d_status=st)
        K = oi.size
        assert int(host(off)[-1]) == K
        assert np.array_equal(host(idx)[:K], oi)
        assert np.array_equal(bits(host(mean)), bits(om))
        assert np.array_equal(bits(host(val)[:K]), bits(ov))
        assert np.array_equal(bits(host(r)), bits(rr))
        words_o, nb_o, table_o = oracle.golomb_encode(oi, b, chunk=64)
        dec_o = oracle.golomb_decode(words_o, nb_o, K, b, n_limit=n)
        end = off[1:2]
        words, nbits, table = gs.golomb_encode(idx, end, b, n, chunk=64, d_status=st, capacity=idx.numel())
        assert int(host(nbits)[0]) == nb_o
        assert np.array_equal(host(words)[:words_o.size].view(np.uint32), words_o)
        assert np.array_equal(host(table)[:table_o.shape[0]], table_o)
        dec = gs.golomb_decode(words, nbits, end, idx.numel(), b, table=table, chunk=64, n_limit=n, d_status=st)
        assert np.array_equal(host(dec)[:K], dec_o)
        gpu_lists.append(gs.make_list(dec, end, uniform_val=mean[0:1], capacity=idx.numel()))
        host_lists.append((dec_o, None, om[0]))
        keepalive.append((dec, end, mean, r))
    dense, mi, mv, mc = gs.scatter_accumulate(gpu_lists, n, merged=True, d_status=st)
    wd, wmi, wmv = oracle.scatter_accumulate(host_lists, n)
    assert np.array_equal(bits(host(dense)[:n]), bits(wd))
    U = int(host(mc)[0])
    assert np.array_equal(host(mi)[:U], wmi) and np.array_equal(bits(host(mv)[:U]), bits(wmv))
    assert int(host(st)[0]) == 0


# ------------------------------------------------------------------------------------ 5

def test_config5_2e30_two_workers_three_drops():
    n, W = 1 << 30, 2
    st = gs.status_tensor()
    g_host = [synth.laplace_outliers(w, n) for w in range(W)]
    g_dev = [dev(x) for x in g_host]
    zero = torch.zeros(n, device="cuda")
    for drop_den in (10, 100, 1000):
        keep = (1, drop_den)
        b = gs.golomb_b_star(1.0 / drop_den)
        lists, keepalive = [], []
        for w in range(W):
            r = torch.zeros(n, device="cuda")
            idx, val, off = gs.residual_topk(g_dev[w], r, keep, d_status=st)
            K = int(host(off)[-1])
            assert K == oracle.k_for(n, *keep)
            check_topk_properties(g_dev[w], zero, r, idx, val, K)
            if w == 0 and drop_den == 100:
                # the bench workload: element-by-element against the oracle
                wi, wv, wo, wr = oracle.residual_topk(g_host[0], np.zeros(n, np.float32), keep)
                assert np.array_equal(host(idx)[:K], wi)
                assert np.array_equal(bits(host(val)[:K]), bits(wv))
                assert np.array_equal(bits(host(r)), bits(wr))
                del wr
                qb, qm, qv, _ = oracle.quantize(wi, wv, write_dequantized=True)
                sb, mm = gs.quantize(idx, val.clone(), off[1:2], d_status=st)
                assert np.array_equal(bits(host(mm)), bits(qm))
                assert np.array_equal(host(sb)[:qb.size].view(np.uint32), qb)
                ww, wnb, wt = oracle.golomb_encode(wi, b, chunk=64)
            elif w == 0:
                # 90% and 99.9%: quantisation and Golomb words of the library's own list (pinned
                # above by exact k, order, threshold, ties and the residual invariant), bitwise
                # against the oracle on the same list
                hi, hv = host(idx)[:K], host(val)[:K]
                qb, qm, qv, _ = oracle.quantize(hi, hv, write_dequantized=True)
                sb, mm = gs.quantize(idx, val.clone(), off[1:2], d_status=st)
                assert np.array_equal(bits(host(mm)), bits(qm))
                assert np.array_equal(host(sb)[:qb.size].view(np.uint32), qb)
                ww, wnb, wt = oracle.golomb_encode(hi, b, chunk=64)
                del hi, hv, qv
            end = off[1:2]
            words, nbits, table = gs.golomb_encode(idx, end, b, n, chunk=64, d_status=st)
            ids = idx[:K].long()
            gaps = torch.diff(ids, prepend=torch.tensor([-1], device="cuda")) - 1
            assert int(host(nbits)[0]) == K * (b + 1) + int((gaps >> b).sum())        # closed form
            if w == 0:
                assert int(host(nbits)[0]) == wnb
                assert np.array_equal(host(words)[:ww.size].view(np.uint32), ww)
                assert np.array_equal(host(table)[:wt.shape[0]], wt)                     # side table
            dec = gs.golomb_decode(words, nbits, end, idx.numel(), b, table=table, chunk=64, n_limit=n, d_status=st)
            assert torch.equal(dec[:K], idx[:K])
            lists.append(gs.make_list(dec, end, val=val))
            keepalive.append((idx, val, off, dec, r))
        dense, _, _, _ = gs.scatter_accumulate(lists, n, d_status=st)
        check = torch.zeros(n, device="cuda")
        for (idx, val, off, dec, r) in keepalive:      # worker order, distinct indices per worker
            K = int(off[-1])
            check.index_add_(0, idx[:K].long(), val[:K])
        assert torch.equal(dense[:n].view(torch.int32), check.view(torch.int32))
        del keepalive, lists, dense, check
    assert int(host(st)[0]) == 0
