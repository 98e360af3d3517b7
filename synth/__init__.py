"""Seeded synthetic gradients for the gradient-compression hot path.

This module only draws random numbers and lays out tensor shapes; it holds none of the
compression arithmetic. Its host arrays feed both the CUDA library (copied to the device) and
the CPU oracle, so the two always read identical bytes.

The workloads stand in for the training runs on the pages (MNIST MLP and NMT in "Sparse
Communication for Distributed Gradient Descent", Introduction; ResNet50/ImageNet in "Sparse Binary
Compression", §III-A Networks and Datasets), which need datasets that are not available: only the
gradient shapes and value distributions are reproduced.

Every draw comes from numpy's PCG64 seeded by ``SeedSequence([seed, tag, *coords])``, so a
(config, worker, step, part) coordinate always yields the same values, independent of thread
count or of which other coordinates were generated.
"""
from __future__ import annotations

import math
from concurrent.futures import ThreadPoolExecutor
from typing import List, Tuple

import numpy as np

# ----------------------------------------------------------------------------------------------
# generators


def rng(*coords: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([int(c) for c in coords])))


def normal(gen: np.random.Generator, n: int, sigma: float) -> np.ndarray:
    """N(0, sigma^2) drawn in fp64 and rounded once to fp32."""
    return (gen.standard_normal(n) * sigma).astype(np.float32)


# ----------------------------------------------------------------------------------------------
# layouts: (name, numel, fan_in) per tensor, flat concatenation in list order


def mlp_layout() -> List[Tuple[str, int, int]]:
    """3-layer MNIST MLP 784-1024-1024-10 with biases; each bias takes its layer's fan_in."""
    return [("fc1.w", 784 * 1024, 784), ("fc1.b", 1024, 784),
            ("fc2.w", 1024 * 1024, 1024), ("fc2.b", 1024, 1024),
            ("fc3.w", 1024 * 10, 1024), ("fc3.b", 10, 1024)]


NMT_VOCAB, NMT_DIM, NMT_TOKENS = 85000, 512, 80 * 50


def nmt_layout() -> List[Tuple[str, int, int]]:
    """Three vocabulary matrices 85000x512 (source/target embedding, output) + 16 dense 1024x1024."""
    lay = [(name, NMT_VOCAB * NMT_DIM, NMT_DIM) for name in ("src_emb", "tgt_emb", "out_proj")]
    lay += [(f"rnn{i}", 1024 * 1024, 1024) for i in range(16)]
    return lay


def resnet50_layout() -> List[Tuple[str, int, int]]:
    """ResNet-50 parameter tensors: 7x7 stem, bottleneck stages 64/128/256/512 x 3/4/6/3 blocks
    (1x1, 3x3, 1x1 convs, expansion 4, 1x1 projection on each stage's first block), BN gamma and
    beta after every conv, fc 2048->1000 with bias. BN vectors take their conv's fan_in."""
    lay: List[Tuple[str, int, int]] = []

    def conv(name, cin, cout, k):
        fan = cin * k * k
        lay.append((name + ".w", cout * fan, fan))
        lay.append((name + ".bn.gamma", cout, fan))
        lay.append((name + ".bn.beta", cout, fan))

    conv("stem", 3, 64, 7)
    cin = 64
    for stage, (width, blocks) in enumerate(zip((64, 128, 256, 512), (3, 4, 6, 3))):
        for blk in range(blocks):
            p = f"s{stage}.b{blk}"
            conv(p + ".c1", cin, width, 1)
            conv(p + ".c2", width, width, 3)
            conv(p + ".c3", width, width * 4, 1)
            if blk == 0:
                conv(p + ".proj", cin, width * 4, 1)
            cin = width * 4
    lay.append(("fc.w", 1000 * 2048, 2048))
    lay.append(("fc.b", 1000, 2048))
    return lay


def offsets(layout) -> np.ndarray:
    return np.concatenate([[0], np.cumsum([t[1] for t in layout])]).astype(np.int64)


# ----------------------------------------------------------------------------------------------
# the five workloads


def flat_mixture(n: int = 1 << 20, seed: int = 0) -> np.ndarray:
    """95% N(0, 1e-4^2) and 5% N(0, 1e-2^2), the component chosen per element."""
    gen = rng(seed, 1)
    wide = gen.random(n) < 0.05
    x = gen.standard_normal(n) * np.where(wide, 1e-2, 1e-4)
    return x.astype(np.float32)


def mlp_gradient(worker: int, step: int, seed: int = 0) -> np.ndarray:
    """Each entry N(0, 1e-3^2) scaled by 1/sqrt(fan_in) of its layer; fresh per (worker, step)."""
    parts = []
    for t, (_, numel, fan) in enumerate(mlp_layout()):
        parts.append(normal(rng(seed, 2, worker, step, t), numel, 1e-3 / math.sqrt(fan)))
    return np.concatenate(parts)


def zipf_ids(gen: np.random.Generator, count: int, vocab: int, s: float) -> np.ndarray:
    """Token ids 0..vocab-1, id = rank - 1 with P(rank) proportional to rank^-s (inverse CDF)."""
    w = np.arange(1, vocab + 1, dtype=np.float64) ** (-s)
    cdf = np.cumsum(w)
    cdf /= cdf[-1]
    return np.minimum(np.searchsorted(cdf, gen.random(count), side="right"), vocab - 1)


def nmt_gradient(worker: int, step: int, seed: int = 0) -> np.ndarray:
    """Vocabulary matrices: only rows of the token ids in an 80x50 batch (Zipf s=1.1) are non-zero,
    N(0, 1e-2^2); the 16 dense matrices are N(0, 1e-4^2)."""
    parts = []
    for t, (_, numel, _) in enumerate(nmt_layout()):
        gen = rng(seed, 3, worker, step, t)
        if t < 3:
            m = np.zeros((NMT_VOCAB, NMT_DIM), np.float32)
            rows = np.unique(zipf_ids(gen, NMT_TOKENS, NMT_VOCAB, 1.1))
            m[rows] = normal(gen, rows.size * NMT_DIM, 1e-2).reshape(rows.size, NMT_DIM)
            parts.append(m.reshape(-1))
        else:
            parts.append(normal(gen, numel, 1e-4))
    return np.concatenate(parts)


def resnet50_gradient(worker: int, step: int, seed: int = 0) -> np.ndarray:
    """Entries N(0, sigma_l^2), sigma_l = 1/sqrt(fan_in) of the tensor's layer."""
    parts = []
    for t, (_, numel, fan) in enumerate(resnet50_layout()):
        parts.append(normal(rng(seed, 4, worker, step, t), numel, 1.0 / math.sqrt(fan)))
    return np.concatenate(parts)


def laplace_outliers(worker: int, n: int = 1 << 30, seed: int = 0, chunk: int = 1 << 22,
                     threads: int = 8) -> np.ndarray:
    """Laplace(0, 1e-3); independently with probability 0.001 an entry is Laplace(0, 1e-1)
    instead. Drawn in chunks of `chunk` entries, each from its own seeded stream."""
    out = np.empty(n, np.float32)

    def fill(c):
        lo, hi = c * chunk, min(n, (c + 1) * chunk)
        gen = rng(seed, 5, worker, c)
        x = gen.laplace(0.0, 1e-3, hi - lo)
        out_mask = gen.random(hi - lo) < 1e-3
        x[out_mask] = gen.laplace(0.0, 1e-1, int(out_mask.sum()))
        out[lo:hi] = x

    nchunks = (n + chunk - 1) // chunk
    with ThreadPoolExecutor(max_workers=threads) as ex:
        list(ex.map(fill, range(nchunks)))
    return out


# ----------------------------------------------------------------------------------------------
# small adversarial inputs for parity cases


def tied_values(n: int, seed: int, levels: int = 5, zero_frac: float = 0.2) -> np.ndarray:
    """Magnitudes from a handful of levels with both signs, +0 and -0: many exact ties."""
    gen = rng(seed, 90)
    mags = np.float32(2.0) ** gen.integers(-8, -8 + levels, n).astype(np.float32)
    sign = np.where(gen.random(n) < 0.5, -1.0, 1.0).astype(np.float32)
    x = (mags * sign).astype(np.float32)
    z = gen.random(n) < zero_frac
    x[z] = np.where(gen.random(int(z.sum())) < 0.5, np.float32(0.0), np.float32(-0.0))
    return x


def gaussian(n: int, seed: int, sigma: float = 1e-3) -> np.ndarray:
    return normal(rng(seed, 91), n, sigma)
