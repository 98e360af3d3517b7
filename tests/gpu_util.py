"""Shared helpers for the GPU parity tests: run the CUDA path through the C ABI on host inputs
and bring results back as numpy arrays."""
import numpy as np
import torch

import compressed_sgd_b200 as gs


def dev(x, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(x))
    if dtype is not None:
        t = t.to(dtype)
    return t.cuda()


def host(t):
    torch.cuda.synchronize()
    return t.detach().cpu().numpy()


def bits(a):
    return np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)


def gpu_topk(g, r, keep, seg=None, flags=0, workspace_bytes=None, capacity=None):
    """Returns (idx, val, offsets, new_r, status) as numpy."""
    gd, rd = dev(g), dev(r)
    segd = None if seg is None else dev(np.asarray(seg, np.int64))
    st = gs.status_tensor()
    ws = None
    if workspace_bytes is not None:
        ws = torch.empty(max(workspace_bytes, 256), dtype=torch.uint8, device="cuda")
    idx, val, off = gs.residual_topk(gd, rd, keep, seg_offsets=segd, flags=flags, workspace=ws, d_status=st,
                                     capacity=capacity)
    offh = host(off)
    K = int(offh[-1])
    return host(idx)[:K], host(val)[:K], offh, host(rd), int(host(st)[0])


def gpu_binarize(g, r, keep, seg=None, flags=0, workspace_bytes=None, by_magnitude=False):
    gd, rd = dev(g), dev(r)
    segd = None if seg is None else dev(np.asarray(seg, np.int64))
    st = gs.status_tensor()
    ws = None
    if workspace_bytes is not None:
        ws = torch.empty(max(workspace_bytes, 256), dtype=torch.uint8, device="cuda")
    idx, val, mean, off = gs.binarize(gd, rd, keep, seg_offsets=segd, flags=flags, workspace=ws, d_status=st,
                                      by_magnitude=by_magnitude)
    offh = host(off)
    K = int(offh[-1])
    return host(idx)[:K], host(val)[:K], host(mean), offh, host(rd), int(host(st)[0])
