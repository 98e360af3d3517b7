"""The exchange of compressed updates between ranks (compressed_sgd_b200.exchange), run as two
gloo ranks on CPU: each rank compresses its own seeded gradient with the oracle (residual top-k
and Golomb coding), the payloads of different lengths are all-gathered, and every rank decodes all
of them and forms the worker-ordered sum, which must equal the sum formed from the original
lists bit for bit."""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
import synth


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


N = 200003
KEEPS = [(1, 100), (0, 1)]   # rank 1 sends nothing in the second exchange


def _compress(rank, rnd):
    g = synth.flat_mixture(N, seed=1000 * rnd + rank)
    keep = (1, 10 * (rank + 1)) if rnd == 0 else KEEPS[rank]
    idx, val, _, _ = oracle.residual_topk(g, np.zeros(N, np.float32), keep)
    b = oracle.golomb_b_star(0.01)
    words, nbits, table = oracle.golomb_encode(idx, b, chunk=64)
    return idx, val, words, nbits, table, b


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from compressed_sgd_b200 import exchange
        results = []
        for rnd in range(2):
            idx, val, words, nbits, table, b = _compress(rank, rnd)
            tab = torch.from_numpy(table.astype(np.int64)) if table is not None else torch.zeros(0, dtype=torch.int64)
            p = exchange.pack(torch.from_numpy(words.view(np.int32).copy()), nbits, idx.size, tab,
                              torch.from_numpy(val.copy()), b, chunk=64)
            got = exchange.all_gather_payloads(p, dist)
            lists = []
            for q in got:
                m = exchange.unpack_meta(q["meta"])
                dec = oracle.golomb_decode(q["words"].numpy().view(np.uint32), m["nbits"], m["count"], m["b"],
                                           n_limit=N)
                lists.append((dec, q["values"].numpy()))
            dense, _, _ = oracle.scatter_accumulate(lists, N, merged=False)
            results.append((dense.copy(), exchange.payload_bytes(got)))
        out[rank] = results
    finally:
        dist.destroy_process_group()


def test_all_gather_of_compressed_payloads_two_ranks():
    world = 2
    out = mp.Manager().dict()
    mp.spawn(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True)
    for rnd in range(2):
        lists = []
        for r in range(world):
            idx, val, *_ = _compress(r, rnd)
            lists.append((idx, val))
        want, _, _ = oracle.scatter_accumulate(lists, N, merged=False)
        for r in range(world):
            dense, nbytes = out[r][rnd]
            assert np.array_equal(dense.view(np.uint32), want.view(np.uint32))
            assert nbytes > 0


import pytest  # noqa: E402


@pytest.mark.gpu
def test_exchange_nccl_one_rank_then_library_decode_and_sum():
    # CUDA tensors over NCCL (one rank on this GPU), then the library's decoder and
    # worker-ordered sum on the gathered payloads
    import compressed_sgd_b200 as gs
    from compressed_sgd_b200 import exchange
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=torch.device("cuda", 0))
    try:
        idx, val, words, nbits, table, b = _compress(0, 0)
        dev = torch.device("cuda", 0)
        p = exchange.pack(torch.from_numpy(words.view(np.int32).copy()).to(dev), nbits, idx.size,
                          torch.from_numpy(table.astype(np.int64)).to(dev), torch.from_numpy(val.copy()).to(dev),
                          b, chunk=64)
        (q,) = exchange.all_gather_payloads(p, dist)
        m = exchange.unpack_meta(q["meta"])
        K = m["count"]
        cnt = torch.tensor([K], dtype=torch.int64, device=dev)
        nb = torch.tensor([m["nbits"]], dtype=torch.int64, device=dev)
        st = gs.status_tensor(dev)
        dec = gs.golomb_decode(q["words"], nb, cnt, K, m["b"], table=q["table"].reshape(-1, 2), chunk=m["chunk"],
                               n_limit=N, d_status=st)
        vals = q["values"].clone()
        dense, _, _, _ = gs.scatter_accumulate([gs.make_list(dec, cnt, val=vals, capacity=K)], N, device=dev,
                                               d_status=st)
        want, _, _ = oracle.scatter_accumulate([(idx, val)], N, merged=False)
        assert int(st.item()) == 0
        assert np.array_equal(dense.cpu().numpy().view(np.uint32), want.view(np.uint32))
    finally:
        dist.destroy_process_group()


# ------------------------------------------------------------------ fixed-capacity exchange

CAP_KEEP = (1, 50)


def _fixed_payload(rank, rnd):
    """Oracle payload laid out in fixed-capacity buffers: words, side table, values and an int64
    header {bits, count}; rank 1 sends nothing in exchange 1 (the second)."""
    g = synth.flat_mixture(N, seed=3000 * rnd + rank)
    keep = CAP_KEEP if not (rank == 1 and rnd == 1) else (0, 1)
    idx, val, _, _ = oracle.residual_topk(g, np.zeros(N, np.float32), keep)
    b = oracle.golomb_b_star(0.02)
    words, nbits, table = oracle.golomb_encode(idx, b, chunk=64)
    cap = oracle.k_for(N, *CAP_KEEP)
    nw = (cap * (b + 1) + ((N + 1) >> b) + 64 + 31) // 32
    W = np.zeros(nw, np.int32)
    W[:words.size] = words.view(np.int32)
    T = np.zeros(((cap + 63) // 64) * 2, np.int64)
    if table is not None and idx.size:
        T[:table.size] = table.reshape(-1)
    V = np.zeros(cap, np.float32)
    V[:val.size] = val
    M = np.array([nbits, idx.size], np.int64)
    return (idx, val, b), [torch.from_numpy(W), torch.from_numpy(T), torch.from_numpy(V), torch.from_numpy(M)]


def _fixed_rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from compressed_sgd_b200 import exchange
        res = []
        for rnd in range(2):
            (_, _, b), sections = _fixed_payload(rank, rnd)
            rows = exchange.all_gather_fixed(sections, dist)
            lists = []
            for W, T, V, M in rows:
                nbits, count = int(M[0]), int(M[1])
                dec = oracle.golomb_decode(W.numpy().view(np.uint32), nbits, count, b, n_limit=N)
                lists.append((dec, V.numpy()[:count].copy()))
            dense, _, _ = oracle.scatter_accumulate(lists, N, merged=False)
            res.append(dense.copy())
        out[rank] = res
    finally:
        dist.destroy_process_group()


def test_fixed_capacity_gather_two_ranks():
    world = 2
    out = mp.Manager().dict()
    mp.spawn(_fixed_rank_main, args=(world, _free_port(), out), nprocs=world, join=True)
    for rnd in range(2):
        lists = [_fixed_payload(r, rnd)[0][:2] for r in range(world)]
        want, _, _ = oracle.scatter_accumulate(lists, N, merged=False)
        for r in range(world):
            assert np.array_equal(out[r][rnd].view(np.uint32), want.view(np.uint32))


# ------------------------------------------------ two ranks, payloads from the library's encoder

def _lib_keep(rank, rnd):
    if rnd == 0:
        return (1, 10) if rank == 0 else (1, 100)
    return (1, 100) if rank == 0 else (0, 1)      # rank 1 sends nothing in exchange 1


def _lib_rank_main(rank, world, port, out):
    import compressed_sgd_b200 as gs
    from compressed_sgd_b200 import exchange
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        dev = torch.device("cuda", 0)
        torch.cuda.set_device(dev)
        b = gs.golomb_b_star(0.01)
        res = []
        for rnd in range(2):
            keep = _lib_keep(rank, rnd)
            g = synth.flat_mixture(N, seed=5000 * rnd + rank)
            gd = torch.from_numpy(g).to(dev)
            rd = torch.zeros(N, device=dev)
            st = gs.status_tensor(dev)
            idx, val, off = gs.residual_topk(gd, rd, keep, d_status=st)
            end = off[1:2]
            gs.quantize(idx, val, end, residual=rd, write_dequantized=True, d_status=st)
            words, nbits, table = gs.golomb_encode(idx, end, b, N, chunk=64, d_status=st)
            torch.cuda.synchronize()
            assert int(st.item()) == 0
            K, nb = int(end.item()), int(nbits.item())
            # the payload as the library wrote it, moved to the host for the gloo exchange
            p = exchange.pack(words.cpu(), nb, K, table[:(K + 63) // 64].cpu(), val[:K].cpu(), b, chunk=64)
            got = exchange.all_gather_payloads(p, dist)
            lists, keep_alive = [], []
            for q in got:
                m = exchange.unpack_meta(q["meta"])
                cnt = torch.tensor([m["count"]], dtype=torch.int64, device=dev)
                nbq = torch.tensor([m["nbits"]], dtype=torch.int64, device=dev)
                wq = q["words"].to(dev) if q["words"].numel() else torch.zeros(1, dtype=torch.int32, device=dev)
                tq = q["table"].to(dev).reshape(-1, 2) if q["table"].numel() else None
                capq = max(m["count"], 1)
                dec = gs.golomb_decode(wq, nbq, cnt, capq, m["b"], table=tq, chunk=64, n_limit=N, d_status=st)
                vq = q["values"].to(dev) if q["values"].numel() else torch.zeros(1, device=dev)
                lists.append(gs.make_list(dec, cnt, val=vq, capacity=capq))
                keep_alive += [cnt, nbq, wq, tq, dec, vq]
            outd = gs.accumulate_combine(lists, N, gd, d_status=st)
            torch.cuda.synchronize()
            res.append((int(st.item()), p["words"].numpy().copy(), nb, outd.cpu().numpy().copy(),
                        rd.cpu().numpy().copy()))
        out[rank] = res
    finally:
        dist.destroy_process_group()


@pytest.mark.gpu
def test_two_ranks_exchange_library_payloads_against_oracle():
    # both ranks run on cuda:0 (independent kernels, no waiting between processes); the payloads
    # travel through gloo on the host with different lengths, one of them empty
    world = 2
    out = mp.Manager().dict()
    mp.spawn(_lib_rank_main, args=(world, _free_port(), out), nprocs=world, join=True)
    b = oracle.golomb_b_star(0.01)
    for rnd in range(2):
        lists, grads, resid, streams = [], [], [], []
        for r in range(world):
            g = synth.flat_mixture(N, seed=5000 * rnd + r)
            oi, ov, _, orr = oracle.residual_topk(g, np.zeros(N, np.float32), _lib_keep(r, rnd))
            _, _, oq, orr = oracle.quantize(oi, ov, residual=orr, write_dequantized=True)
            ww, nb, _ = oracle.golomb_encode(oi, b, chunk=64)
            lists.append((oi, oq))
            grads.append(g)
            resid.append(orr)
            streams.append((ww, nb))
        dense, _, _ = oracle.scatter_accumulate(lists, N, merged=False)
        for r in range(world):
            status, words, nb, outd, rd = out[r][rnd]
            assert status == 0
            ww, wnb = streams[r]
            assert nb == wnb and np.array_equal(words.view(np.uint32)[:ww.size], ww)
            assert np.array_equal(rd.view(np.uint32), resid[r].view(np.uint32))
            want = oracle.combine_local(dense, grads[r])
            assert np.array_equal(outd.view(np.uint32), want.view(np.uint32))
