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
KEEPS = [(1, 100), (0, 1)]   # rank 1 sends nothing in the second round


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
