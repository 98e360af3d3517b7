"""Exchange of compressed updates between data-parallel ranks (one worker per rank).

After compression every worker holds a variable-length payload: the Golomb-coded positions of
its sent entries (words, bit count, side table) and their values (fp32, or the 2-bit form: sign
bits and two means). Every worker needs every other worker's payload to form the global sparse
sum ("Sparse Communication for Distributed Gradient Descent", Abstract: workers exchange sparse
updates; "Sparse Binary Compression", §I: the clients' updates are summed). The exchange is an
all-gather of variable-length sections: the section lengths are all-gathered first, then each
section is padded to the longest and all-gathered, and every rank trims the received rows to
their own lengths. With CUDA tensors and the NCCL backend the transfers run over NVLink; with CPU
tensors and gloo the same code runs on the host. Decoding and the worker-ordered sum then use the
library's calls on the gathered payloads (rank order = worker order).

all_gather_payloads learns the lengths on the host (one small gather and a synchronisation per
call). all_gather_fixed instead gathers buffers of a fixed capacity whose used lengths travel
inside them (the stream's bit count and the entry count in a device header), so a training loop
can run the exchange with no host synchronisation; the decoder reads the lengths on the device.
"""
from typing import Dict, List, Optional, Sequence

import torch

# payload sections, in a fixed order; each is a 1-D tensor
SECTIONS = ("words", "table", "values", "meta")


def pack(words: torch.Tensor, nbits: int, count: int, table: torch.Tensor, values: torch.Tensor,
         b: int, base: int = 0, chunk: int = 0) -> Dict[str, torch.Tensor]:
    """One worker's payload. words: int32 Golomb stream (at least ceil(nbits / 32) words); table:
    int64 side table flattened (or empty); values: fp32 values of the sent entries, or the 2-bit
    form laid out by the caller. meta carries nbits, count, b, base and chunk as int64."""
    dev = words.device
    nw = (int(nbits) + 31) // 32
    meta = torch.tensor([int(nbits), int(count), int(b), int(base), int(chunk)], dtype=torch.int64, device=dev)
    return {"words": words[:nw].contiguous(), "table": table.reshape(-1).contiguous(),
            "values": values.reshape(-1).contiguous(), "meta": meta}


def unpack_meta(meta: torch.Tensor) -> Dict[str, int]:
    m = [int(x) for x in meta.tolist()]
    return {"nbits": m[0], "count": m[1], "b": m[2], "base": m[3], "chunk": m[4]}


def _gather_section(t: torch.Tensor, lengths: List[int], dist, group) -> List[torch.Tensor]:
    longest = max(lengths)
    padded = torch.zeros(max(longest, 1), dtype=t.dtype, device=t.device)
    if t.numel():
        padded[:t.numel()] = t
    rows = [torch.empty_like(padded) for _ in lengths]
    dist.all_gather(rows, padded, group=group)
    return [row[:ln] for row, ln in zip(rows, lengths)]


def all_gather_payloads(payload: Dict[str, torch.Tensor], dist, group=None) -> List[Dict[str, torch.Tensor]]:
    """Every rank's payload, in rank order. All ranks call this with payloads of the same dtypes
    on the same kind of device; the lengths may differ."""
    dev = payload["meta"].device
    world = dist.get_world_size(group)
    mine = torch.tensor([payload[s].numel() for s in SECTIONS], dtype=torch.int64, device=dev)
    sizes = [torch.empty_like(mine) for _ in range(world)]
    dist.all_gather(sizes, mine, group=group)
    sizes = [[int(x) for x in s.tolist()] for s in sizes]
    out: List[Dict[str, torch.Tensor]] = [dict() for _ in range(world)]
    for k, name in enumerate(SECTIONS):
        rows = _gather_section(payload[name], [s[k] for s in sizes], dist, group)
        for r in range(world):
            out[r][name] = rows[r]
    return out


def payload_bytes(payloads: Sequence[Dict[str, torch.Tensor]]) -> int:
    """Bytes that cross the interconnect per rank and step (before padding)."""
    return sum(t.numel() * t.element_size() for p in payloads for t in p.values())


def gather_buffers(sections: Sequence[torch.Tensor], world: int) -> List[torch.Tensor]:
    """Receive buffers for all_gather_fixed: one tensor of world x numel per section."""
    return [torch.empty(world * t.numel(), dtype=t.dtype, device=t.device) for t in sections]


def all_gather_fixed(sections: Sequence[torch.Tensor], dist, group=None,
                     out: Optional[Sequence[torch.Tensor]] = None) -> List[List[torch.Tensor]]:
    """Gathers same-shaped buffers from every rank, one collective per section. sections: 1-D
    contiguous tensors of the same length and dtype on every rank (fixed capacities, e.g. the
    Golomb word buffer, the side table, the values and an int64 header holding the bit count and
    the entry count). out: receive buffers from gather_buffers (allocated here if None). With
    dist None there is one rank and its sections are returned as they are.
    Returns rows[r][k] = section k of rank r (views into the receive buffers)."""
    if dist is None:
        return [list(sections)]
    world = dist.get_world_size(group)
    if out is None:
        out = gather_buffers(sections, world)
    per_rank: List[List[torch.Tensor]] = [[] for _ in range(world)]
    for t, gathered in zip(sections, out):
        dist.all_gather_into_tensor(gathered, t, group=group)
        rows = gathered.view(world, t.numel())
        for r in range(world):
            per_rank[r].append(rows[r])
    return per_rank
