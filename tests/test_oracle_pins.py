"""Pins of the CPU oracle against facts that do not come from the oracle itself: brute force on
tiny inputs, exact rational arithmetic, hand-worked codes, closed forms, the figure printed on
the pages, invariants and special cases. CPU only."""
import itertools
import math
import os
import struct
from fractions import Fraction

import numpy as np
import pytest

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def f32(x):
    return np.float32(x)


def bits(x):
    return struct.unpack("<I", struct.pack("<f", float(x)))[0]


def ieee_add(a, b):
    """fp32 sum of two fp32 numbers: the exact rational sum rounded once to nearest even. An exact
    zero is +0 unless both operands are -0 (IEEE 754 rule for round to nearest)."""
    s = Fraction(float(a)) + Fraction(float(b))
    if s == 0:
        both_neg = math.copysign(1.0, a) < 0 and math.copysign(1.0, b) < 0
        return np.float32(-0.0 if both_neg else 0.0)
    return np.float32(float(s)) if abs(s) < 2 ** 100 else np.float32(float(a) + float(b))


def round_f32_exact(x):
    """Round a rational to the nearest fp32 (ties to even) without passing through fp64."""
    f = np.float32(float(x))
    cands = {f, np.nextafter(f, np.float32(np.inf)), np.nextafter(f, np.float32(-np.inf))}
    best = sorted(cands, key=lambda c: (abs(Fraction(float(c)) - x), int(c.view(np.uint32)) & 1))
    return best[0]


def acc_of(g, r):
    return np.array([ieee_add(a, b) for a, b in zip(g.tolist(), r.tolist())], np.float32)


def brute_topk_subsets(acc, k):
    """The unique k-subset S with: for i in S, j not in S: |a_i| > |a_j| or (|a_i| == |a_j| and i < j)."""
    n = len(acc)
    mags = [abs(float(a)) for a in acc]
    found = []
    for S in itertools.combinations(range(n), k):
        s = set(S)
        ok = all(mags[i] > mags[j] or (mags[i] == mags[j] and i < j) for i in s for j in range(n) if j not in s)
        if ok:
            found.append(S)
    assert len(found) == 1
    return list(found[0])


def rank_count_topk(acc, k):
    """O(n^2) rank count: i is kept iff fewer than k entries come before it in the order."""
    mags = [abs(float(a)) for a in acc]
    n = len(acc)
    out = []
    for i in range(n):
        rank = sum(1 for j in range(n) if mags[j] > mags[i] or (mags[j] == mags[i] and j < i))
        if rank < k:
            out.append(i)
    return out


# ------------------------------------------------------------------------------------ k and b*

def test_k_is_ceiling_of_fraction():
    # the flat 2^20 workload states k = 10,486 for a 99% drop
    assert oracle.k_for(1 << 20, 1, 100) == 10486
    for n in [0, 1, 7, 99, 100, 101, 12345, (1 << 30), (1 << 31) - 1]:
        for num, den in [(0, 1), (1, 100), (1, 10), (1, 1000), (3, 7), (1, 1)]:
            want = min(n, math.ceil(Fraction(n * num, den)))
            assert oracle.k_for(n, num, den) == want


def test_golomb_b_star_values():
    # b* = 1 + floor(log2(log(phi-1)/log(1-p))): hand evaluation
    #   p=0.01: log(0.6180)/log(0.99) = 47.88 -> log2 5.58 -> 6
    #   p=0.001: 480.97 -> 8.91 -> 9 ;  p=0.1: 4.567 -> 2.19 -> 3
    assert oracle.golomb_b_star(0.01) == 6
    assert oracle.golomb_b_star(0.001) == 9
    assert oracle.golomb_b_star(0.1) == 3
    assert oracle.golomb_b_star(0.0) == -1


# ------------------------------------------------------------------------------------ top-k

@pytest.mark.parametrize("seed", range(12))
def test_topk_brute_force_subsets(seed):
    gen = np.random.default_rng(seed)
    n = int(gen.integers(16, 21))
    g = synth.tied_values(n, seed, levels=3, zero_frac=0.25)
    r = synth.tied_values(n, seed + 100, levels=3, zero_frac=0.5) * np.float32(0.5)
    acc = acc_of(g, r)
    for k in sorted({0, 1, int(gen.integers(2, n)), n - 1, n}):
        idx, val, off, rn = oracle.residual_topk(g, r, keep=(k, n))
        assert oracle.k_for(n, k, n) == k
        want = brute_topk_subsets(acc, k)
        assert idx.tolist() == want
        assert [bits(v) for v in val] == [bits(acc[i]) for i in want]
        assert off.tolist() == [0, k]


@pytest.mark.parametrize("seed", range(10))
def test_topk_rank_count(seed):
    gen = np.random.default_rng(1000 + seed)
    n = int(gen.integers(21, 65))
    g = synth.tied_values(n, seed + 7, levels=4)
    r = synth.gaussian(n, seed, sigma=0.01) if seed % 2 else np.zeros(n, np.float32)
    acc = acc_of(g, r)
    for num, den in [(1, 100), (1, 10), (1, 3), (1, 2), (7, 8)]:
        idx, _, _, _ = oracle.residual_topk(g, r, keep=(num, den))
        assert idx.tolist() == rank_count_topk(acc, oracle.k_for(n, num, den))


@pytest.mark.parametrize("seed", range(6))
def test_topk_residual_invariant_bitwise(seed):
    n = 2000 + 37 * seed
    g = synth.gaussian(n, seed)
    r = synth.tied_values(n, seed, levels=6) * np.float32(1e-3)
    acc = acc_of(g, r)
    idx, val, off, rn = oracle.residual_topk(g, r, keep=(1, 20))
    sent = np.zeros(n, np.float32)
    sent[idx] = val
    for i in range(n):
        pair = (bits(sent[i]), bits(rn[i]))
        assert bits(acc[i]) in pair and 0 in pair           # one of them is acc_i, the other +0
    assert len(set(idx.tolist())) == idx.size == oracle.k_for(n, 1, 20)
    assert np.all(np.diff(idx) > 0)
    # selected keys dominate unselected keys; equal keys go to the lower index
    mags = np.abs(acc.astype(np.float64))
    T = mags[idx].min()
    unsent = np.setdiff1d(np.arange(n), idx)
    assert mags[unsent].max() <= T
    ties_out = unsent[mags[unsent] == T]
    ties_in = idx[mags[idx] == T]
    if ties_out.size:
        assert ties_in.max() < ties_out.min()


def test_topk_special_cases():
    n = 333
    g = synth.gaussian(n, 3)
    r = synth.gaussian(n, 4)
    acc = acc_of(g, r)
    idx, val, off, rn = oracle.residual_topk(g, r, keep=(1, 1))          # k = n
    assert idx.tolist() == list(range(n)) and np.all(rn == 0) and np.array_equal(val, acc)
    idx, val, off, rn = oracle.residual_topk(g, r, keep=(0, 1))          # k = 0: accumulate only
    assert idx.size == 0 and off.tolist() == [0, 0] and np.array_equal(rn.view(np.uint32), acc.view(np.uint32))
    idx, val, off, rn = oracle.residual_topk(np.zeros(0, np.float32), np.zeros(0, np.float32))
    assert idx.size == 0 and off.tolist() == [0, 0]


# ------------------------------------------------------------------ momentum correction and masking
# "Sparse Binary Compression", §II and Appendix A: the momentum-corrected gradient goes into the
# residual, and the momentum of the sent entries is zeroed.

def test_momentum_delay_only_closed_form():
    # keep 0 (nothing sent), m = 1/2, g = 1, u = r = 0 at the start: after t steps
    # u_t = 2 - 2^(1-t) and r_t = sum_{s<=t} u_s = 2t - 2 + 2^(1-t), all exact in fp32
    n = 7
    g = np.ones(n, np.float32)
    u = np.zeros(n, np.float32)
    r = np.zeros(n, np.float32)
    for t in range(1, 13):
        idx, _, off, r, u = oracle.residual_topk_momentum(g, u, 0.5, r, keep=(0, 1))
        assert idx.size == 0 and off.tolist() == [0, 0]
        assert np.all(u == np.float32(2.0 - 2.0 ** (1 - t)))
        assert np.all(r == np.float32(2.0 * t - 2.0 + 2.0 ** (1 - t)))


def test_momentum_send_all_masks_everything():
    # keep 1 (everything sent every step): the residual and the momentum are zeroed each step, so
    # the sent values are the raw gradient at every step whatever m is
    n = 50
    u = np.zeros(n, np.float32)
    r = np.zeros(n, np.float32)
    for t in range(4):
        g = synth.gaussian(n, 70 + t)
        idx, val, _, r, u = oracle.residual_topk_momentum(g, u, 0.9, r, keep=(1, 1))
        assert idx.tolist() == list(range(n))
        assert np.array_equal(val.view(np.uint32), g.view(np.uint32))
        assert np.all(r.view(np.uint32) == 0) and np.all(u.view(np.uint32) == 0)


def test_momentum_zero_reduces_to_plain_topk():
    n = 1000
    for step in range(3):
        g = synth.gaussian(n, 80 + step)
        r0 = synth.gaussian(n, 90 + step, sigma=1e-4)
        u0 = synth.gaussian(n, 95 + step)
        idx, val, off, rn, un = oracle.residual_topk_momentum(g, u0, 0.0, r0, keep=(1, 10))
        pi, pv, po, pr = oracle.residual_topk(g, r0, keep=(1, 10))
        assert np.array_equal(idx, pi) and np.array_equal(val.view(np.uint32), pv.view(np.uint32))
        assert np.array_equal(off, po) and np.array_equal(rn.view(np.uint32), pr.view(np.uint32))
        want_u = g.copy()
        want_u[idx] = 0.0
        assert np.array_equal(un.view(np.uint32), want_u.view(np.uint32))


def test_momentum_small_exact_case():
    # integer-valued inputs, m = 1/2: v = (u / 2) + g exactly; the two largest |r + v| are sent
    g = np.array([1, -4, 2, 0, 3], np.float32)
    u = np.array([4, 2, -6, 8, 0], np.float32)
    r = np.array([0, 1, 0, -1, 0], np.float32)
    # v = [3, -3, -1, 4, 3]; acc = [3, -2, -1, 3, 3]; k = 2 -> indices 0 and 3 (ties -> lower)
    idx, val, _, rn, un = oracle.residual_topk_momentum(g, u, 0.5, r, keep=(2, 5))
    assert idx.tolist() == [0, 3] and val.tolist() == [3.0, 3.0]
    assert rn.tolist() == [0.0, -2.0, -1.0, 0.0, 3.0]
    assert un.tolist() == [0.0, -3.0, -1.0, 0.0, 3.0]


def test_warmup_schedule_endpoints_and_ratio():
    # "Sparse Binary Compression", Appendix A: sparsity raised exponentially from 25% to 0.1% kept
    T = 4
    nums = [oracle.warmup_keep(t, T)[0] for t in range(T + 3)]
    assert nums[0] == 250000 and all(x == 1000 for x in nums[T:])
    # geometric: each step multiplies the keep fraction by (0.001 / 0.25)^(1/4) = 0.2515 (4 steps)
    q = (0.001 / 0.25) ** 0.25
    for t in range(1, T + 1):
        assert abs(nums[t] - nums[t - 1] * q) <= 1.0
    assert nums[1] in (62872, 62873) and nums[2] == 15811
    assert oracle.warmup_keep(0, 0)[0] == 1000          # no warm-up: the final fraction at once
    assert oracle.warmup_keep(3, 4, 0.5, 0.5)[0] == 500000
    assert oracle.warmup_keep(1, 4, 0.0, 0.1)[0] == -1


# ------------------------------------------- sparse binarisation, magnitude-first reading
# "Sparse Binary Compression", §II Sparse Binarization: keep the largest-magnitude fraction, then
# the sign with the larger absolute mean decides which values remain.

def test_binarize_magnitude_hand_worked():
    g = np.array([3, -5, 1, -4, 2, 0, -1], np.float32)
    r = np.zeros(7, np.float32)
    # k = 3: S = {0, 1, 3} (|3|, |-5|, |-4|); mu+ = 3, mu- = 4.5 -> the negatives, mean -4.5
    idx, val, mean, off, rn = oracle.binarize(g, r, (3, 7), by_magnitude=True)
    assert idx.tolist() == [1, 3] and val.tolist() == [-4.5, -4.5] and mean.tolist() == [-4.5]
    assert off.tolist() == [0, 2] and rn.tolist() == [3.0, -0.5, 1.0, 0.5, 2.0, 0.0, -1.0]


def test_binarize_magnitude_equal_means_take_positive():
    # mu+ = mu- = 1.5 with everything kept: the positive set is sent (ties go to the positive sign)
    g = np.array([2, -2, 1, -1], np.float32)
    idx, val, mean, off, rn = oracle.binarize(g, np.zeros(4, np.float32), (1, 1), by_magnitude=True)
    assert idx.tolist() == [0, 2] and mean.tolist() == [1.5] and rn.tolist() == [0.5, -2.0, -0.5, -1.0]


@pytest.mark.parametrize("seed", range(12))
def test_binarize_magnitude_brute_force(seed):
    # integer-valued inputs: every mean is an exact rational, rounded once to fp32
    gen = np.random.default_rng(500 + seed)
    n = int(gen.integers(1, 40))
    g = gen.integers(-9, 10, n).astype(np.float32)
    r = gen.integers(-3, 4, n).astype(np.float32)
    keep = (int(gen.integers(0, 5)), 4)
    acc = g + r
    k = math.ceil(n * keep[0] / keep[1])
    S = sorted(sorted(range(n), key=lambda i: (-abs(float(acc[i])), i))[:k])
    P = [i for i in S if acc[i] > 0]
    N = [i for i in S if acc[i] < 0]
    mp = float(np.float32(Fraction(int(sum(acc[i] for i in P))) / len(P))) if P else 0.0
    mn = float(np.float32(Fraction(int(-sum(acc[i] for i in N))) / len(N))) if N else 0.0
    if P and mp >= mn:
        sent, m = P, mp
    elif N:
        sent, m = N, -mn
    else:
        sent, m = [], 0.0
    idx, val, mean, off, rn = oracle.binarize(g, r, keep, by_magnitude=True)
    assert idx.tolist() == sent and mean.tolist() == [np.float32(m)]
    assert all(v == np.float32(m) for v in val)
    want_r = acc.copy()
    for i in sent:
        want_r[i] = acc[i] - np.float32(m)
    assert np.array_equal(rn, want_r)


def test_binarize_magnitude_keep_all_equals_sign_sets():
    # k = n: S is everything, so both readings compare all positives against all negatives
    n = 301
    gen = np.random.default_rng(9)
    g = gen.integers(-50, 51, n).astype(np.float32)
    r = np.zeros(n, np.float32)
    a = oracle.binarize(g, r, (1, 1), by_magnitude=True)
    b = oracle.binarize(g, r, (1, 1))
    for x, y in zip(a, b):
        assert np.array_equal(x, y)


def test_topk_negative_zero_ties_positive_zero():
    g = np.array([-0.0, 0.0, -0.0, 1.0], np.float32)
    r = np.array([-0.0, -0.0, 0.0, 0.0], np.float32)
    # acc = -0, +0, +0, 1 ; k = 3 -> 3, then the two lowest indices among the zeros
    idx, val, _, rn = oracle.residual_topk(g, r, keep=(3, 4))
    assert idx.tolist() == [0, 1, 3]
    assert bits(val[0]) == 0x80000000 and bits(val[1]) == 0
    assert bits(rn[0]) == 0 and bits(rn[2]) == 0


@pytest.mark.parametrize("seed", range(4))
def test_per_tensor_equals_separate_selections(seed):
    lay = [37, 1, 500, 64, 0, 1023]
    seg = np.concatenate([[0], np.cumsum(lay)])
    n = int(seg[-1])
    g = synth.gaussian(n, seed)
    r = synth.tied_values(n, seed, levels=3) * np.float32(1e-3)
    acc = acc_of(g, r)
    idx, val, off, rn = oracle.residual_topk(g, r, keep=(1, 10), seg=seg)
    for s in range(len(lay)):
        part = idx[off[s]:off[s + 1]]
        want = [int(seg[s]) + i for i in rank_count_topk(acc[seg[s]:seg[s + 1]], oracle.k_for(lay[s], 1, 10))]
        assert part.tolist() == want


# ------------------------------------------------------------------------------------ quantise

def exact_mean_f32(values):
    """fp32 of the fp64 of the exact rational mean (the oracle divides once in fp64 and rounds to fp32)."""
    if not values:
        return np.float32(0.0)
    s = sum(Fraction(float(v)) for v in values)
    return np.float32(float(s / len(values)))


@pytest.mark.parametrize("seed", range(5))
def test_quantize_means_and_bits(seed):
    K = 1000 + 513 * seed
    # values on a 2^-20 grid keep every fp64 partial sum exact, so the exact mean is the target
    val = (np.round(synth.gaussian(K, seed, sigma=1e-2) * 2.0 ** 20) / 2.0 ** 20).astype(np.float32)
    val[::97] = 0.0
    idx = np.sort(np.random.default_rng(seed).choice(10 * K, K, replace=False)).astype(np.int32)
    res = np.zeros(10 * K, np.float32)
    bits_, means, deq, res2 = oracle.quantize(idx, val, residual=res, write_dequantized=True)
    pos = [v for v in val if v > 0]
    neg = [v for v in val if v < 0]
    assert means[0] == exact_mean_f32(pos) and means[1] == exact_mean_f32(neg)
    assert means[1] < 0 < means[0]
    for j in range(K):
        assert ((bits_[j // 32] >> (j % 32)) & 1) == (1 if val[j] < 0 else 0)
        q = means[0] if val[j] > 0 else (means[1] if val[j] < 0 else np.float32(0))
        assert bits(deq[j]) == bits(q)
        # error fed back: exact difference rounded once
        assert res2[idx[j]] == np.float32(Fraction(float(val[j])) - Fraction(float(q)))
    untouched = np.setdiff1d(np.arange(10 * K), idx)
    assert np.all(res2[untouched] == 0)


def test_quantize_all_positive_and_constant():
    val = np.full(777, 0.375, np.float32)
    idx = np.arange(777, dtype=np.int32)
    b, means, _, _ = oracle.quantize(idx, val)
    assert means[0] == np.float32(0.375) and means[1] == 0 and np.all(b == 0)


def test_fixed_order_sum_absorbs_inside_a_block():
    # Members 2, 2^-60, 1, 1 + 2^-22 at positions 0, 1, 256, 512 (zeros elsewhere are not members).
    # Block 0 adds 2 + 2^-60 = 2 in fp64; blocks give 2, 1, 1 + 2^-22; tree: (2 + 1) + (1 + 2^-22)
    # = 4 + 2^-22; mean 1 + 2^-24 is the fp32 midpoint of 1 and 1 + 2^-23 and ties to even: 1.0.
    # The exact mean lies just above the midpoint (1 + 2^-23): summing exactly would be caught.
    val = np.zeros(513, np.float32)
    val[0], val[1], val[256], val[512] = 2.0, 2.0 ** -60, 1.0, 1.0 + 2.0 ** -22
    _, means, _, _ = oracle.quantize(np.arange(val.size, dtype=np.int32), val)
    assert means[0] == np.float32(1.0)
    exact = sum(Fraction(float(v)) for v in val if v > 0) / 4
    assert round_f32_exact(exact) == np.float32(1.0 + 2.0 ** -23)


def test_fixed_order_sum_keeps_a_later_block_whole():
    # 512 members: 512 and 254 copies of t = 2^-45 in block 0 (each t vanishes next to 512 in
    # fp64: half an ulp there is 2^-44), then 256 copies of t in block 1 (sum 2^-37, exact), then
    # A2 = 3*2^-15 - 2^-37 in block 2. Rule: (512 + 2^-37) + A2 = 512 + 3*2^-15; /512 = 1 + 3*2^-24,
    # the fp32 midpoint of 1 + 2^-23 and 1 + 2^-22, which ties to the even 1 + 2^-22. Summing the
    # list left to right in one pass loses every t and gives 1 + 2^-23 instead.
    t = 2.0 ** -45
    val = np.zeros(3 * 256, np.float32)
    val[0] = 512.0
    val[1:255] = t
    val[256:512] = t
    val[512] = 3 * 2.0 ** -15 - 2.0 ** -37
    assert float(val[512]) == 3 * 2.0 ** -15 - 2.0 ** -37           # exactly representable
    _, means, _, _ = oracle.quantize(np.arange(val.size, dtype=np.int32), val)
    assert means[0] == np.float32(1.0 + 2.0 ** -22)
    seq = 0.0
    for v in val:
        seq += float(v)
    assert np.float32(seq / 512) == np.float32(1.0 + 2.0 ** -23)


def test_fixed_order_sum_pairs_four_block_sums_as_a_tree():
    # Four blocks of 256 positions. Members: 4 and 2^-22 in block 0 (block sum A = 4 + 2^-22, exact
    # in fp64), none in block 1 (sum +0), 2^-51 in block 2, 2^-51 in block 3. In fp64 one ulp of A
    # is 2^-50, so adding 2^-51 to A alone is an exact tie, which goes to A (its last mantissa bit
    # is 0). Pairwise tree: (A + 0) + (2^-51 + 2^-51) = A + 2^-50 exactly; mean over 4 members
    # 1 + 2^-24 + 2^-52, just above the fp32 midpoint of 1 and 1 + 2^-23, rounds up to 1 + 2^-23.
    # Left to right: ((A + 0) + 2^-51) + 2^-51 = A; mean 1 + 2^-24 is the midpoint itself and ties
    # to the even 1.0. So this case fails a block-sum combination that runs left to right.
    val = np.zeros(4 * 256, np.float32)
    val[0], val[1], val[512], val[768] = 4.0, 2.0 ** -22, 2.0 ** -51, 2.0 ** -51
    _, means, _, _ = oracle.quantize(np.arange(val.size, dtype=np.int32), val)
    assert means[0] == np.float32(1.0 + 2.0 ** -23)
    assert means[0].view(np.uint32) == np.uint32(0x3F800001)
    A = 4.0 + 2.0 ** -22
    assert A + 2.0 ** -51 == A and A + 2.0 ** -50 == 4.0 + 2.0 ** -22 + 2.0 ** -50   # the fp64 facts used
    blocks = [A, 0.0, 2.0 ** -51, 2.0 ** -51]
    tree = (blocks[0] + blocks[1]) + (blocks[2] + blocks[3])
    left_to_right = ((blocks[0] + blocks[1]) + blocks[2]) + blocks[3]
    assert np.float32(tree / 4) == np.float32(1.0 + 2.0 ** -23)
    assert np.float32(left_to_right / 4) == np.float32(1.0)


def test_fixed_order_sum_lifts_an_odd_last_block_unchanged():
    # Five blocks: 4 | 2^-22 | (none) | 2^-51 | 2^-51, one member each where present. Level 1 of the
    # tree pairs (b0 + b1) = A = 4 + 2^-22 and (b2 + b3) = 2^-51; b4 moves up alone. Level 2:
    # A + 2^-51 = A (an exact tie to even, as above); b4 moves up. Level 3: A + 2^-51 = A. Mean over
    # 4 members 1 + 2^-24 ties to 1.0. Pairing from the right end instead (b0 alone, (b1 + b2),
    # (b3 + b4) = 2^-50) gives A + 2^-50 and 1 + 2^-23, as does the exact sum; folding the odd
    # block into the last pair, (b2 + b3 + b4), gives 2^-50 there and 1 + 2^-23 as well.
    val = np.zeros(5 * 256, np.float32)
    val[0], val[256], val[768], val[1024] = 4.0, 2.0 ** -22, 2.0 ** -51, 2.0 ** -51
    _, means, _, _ = oracle.quantize(np.arange(val.size, dtype=np.int32), val)
    assert means[0] == np.float32(1.0)
    b = [4.0, 2.0 ** -22, 0.0, 2.0 ** -51, 2.0 ** -51]
    from_right = (b[0] + (b[1] + b[2])) + (b[3] + b[4])
    folded = (b[0] + b[1]) + ((b[2] + b[3]) + b[4])
    assert np.float32(from_right / 4) == np.float32(1.0 + 2.0 ** -23)
    assert np.float32(folded / 4) == np.float32(1.0 + 2.0 ** -23)
    exact = sum(Fraction(x) for x in b) / 4
    assert round_f32_exact(exact) == np.float32(1.0 + 2.0 ** -23)


# ------------------------------------------------------------------------------------ binarise

def brute_binarize(acc, k):
    n = len(acc)
    pos = [i for i in range(n) if acc[i] > 0]
    neg = [i for i in range(n) if acc[i] < 0]

    def top(cands):
        kk = min(k, len(cands))
        mags = {i: abs(float(acc[i])) for i in cands}
        out = [i for i in cands
               if sum(1 for j in cands if mags[j] > mags[i] or (mags[j] == mags[i] and j < i)) < kk]
        return sorted(out)

    P, N = top(pos), top(neg)
    mp = exact_mean_f32([acc[i] for i in P])
    mn = exact_mean_f32([-acc[i] for i in N])
    if P and mp >= mn:
        return P, mp
    if N:
        return N, -mn
    return [], np.float32(0.0)


@pytest.mark.parametrize("seed", range(10))
def test_binarize_brute_force(seed):
    gen = np.random.default_rng(50 + seed)
    n = int(gen.integers(16, 48))
    g = synth.tied_values(n, seed, levels=4, zero_frac=0.1)
    if seed % 3 == 0:
        g = np.abs(g) * np.float32(0.5) + g        # skew towards positive
    r = np.zeros(n, np.float32)
    acc = acc_of(g, r)
    for num, den in [(1, 10), (1, 4), (1, 2), (1, 1)]:
        k = oracle.k_for(n, num, den)
        idx, val, mean, off, rn = oracle.binarize(g, r, keep=(num, den))
        S, m = brute_binarize(acc, k)
        assert idx.tolist() == S and bits(mean[0]) == bits(m)
        assert np.all(val == m)
        for i in range(n):
            want = np.float32(Fraction(float(acc[i])) - Fraction(float(m))) if i in S else acc[i]
            assert bits(rn[i]) == bits(want)


def test_binarize_picks_larger_mean_side():
    g = np.array([5, -1, 4, -1, 3, -1, 0, -9], np.float32)
    # k = 2: P = {0, 2} mean 4.5 ; N = {7, 1} mean 5 -> N wins with -5
    idx, val, mean, off, _ = oracle.binarize(g, np.zeros(8, np.float32), keep=(1, 4))
    assert idx.tolist() == [1, 7] and mean[0] == -5.0
    g[7] = -7.0   # N mean 4 < 4.5 -> P
    idx, val, mean, off, _ = oracle.binarize(g, np.zeros(8, np.float32), keep=(1, 4))
    assert idx.tolist() == [0, 2] and mean[0] == 4.5
    g = np.array([2, -2, 0], np.float32)   # equal means -> positive
    idx, _, mean, _, _ = oracle.binarize(g, np.zeros(3, np.float32), keep=(1, 3))
    assert idx.tolist() == [0] and mean[0] == 2.0
    z = np.zeros(5, np.float32)             # nothing to send
    idx, _, mean, off, rn = oracle.binarize(z, z, keep=(1, 1))
    assert idx.size == 0 and mean[0] == 0 and off.tolist() == [0, 0]


# ------------------------------------------------------------------------------------ Golomb

def read_golden(name):
    d = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, *vals = line.split()
            d[key] = vals
    return d


def test_golomb_hand_worked_example():
    d = read_golden("golomb_rice_b2.txt")
    b, base = int(d["b"][0]), int(d["base"][0])
    idx = np.array([int(x) for x in d["indices"]], np.int32)
    words, nbits, _ = oracle.golomb_encode(idx, b, base)
    assert nbits == int(d["nbits"][0])
    assert words.tolist() == [int(x) for x in d["words"]]
    assert oracle.golomb_decode(words, nbits, idx.size, b, base).tolist() == idx.tolist()


def test_golomb_unary_when_b_is_zero():
    idx = np.array([3, 4, 6], np.int32)          # gaps 3, 0, 1 -> 1110 0 10
    words, nbits, _ = oracle.golomb_encode(idx, 0)
    assert nbits == 7 and words.tolist() == [0b0100111]


@pytest.mark.parametrize("b", [0, 1, 3, 6, 9, 12])
def test_golomb_roundtrip_and_length(b):
    gen = np.random.default_rng(b)
    n = 200000
    idx = np.sort(gen.choice(n, 3000, replace=False)).astype(np.int32)
    base = 5 if idx[0] >= 5 else 0
    words, nbits, table = oracle.golomb_encode(idx, b, base, chunk=64)
    gaps = np.diff(np.concatenate([[base - 1], idx.astype(np.int64)])) - 1
    assert nbits == idx.size * (b + 1) + int((gaps >> b).sum())          # closed form
    assert oracle.golomb_decode(words, nbits, idx.size, b, base).tolist() == idx.tolist()
    # side table: codeword c*64 starts at the summed lengths of the codewords before it
    lens = (gaps >> b) + 1 + b
    starts = np.concatenate([[0], np.cumsum(lens)])
    for c in range(table.shape[0]):
        assert table[c, 0] == starts[64 * c]
        assert table[c, 1] == (base - 1 if c == 0 else idx[64 * c - 1])


def test_golomb_mean_length_matches_printed_figure():
    d = read_golden("golomb_bits_per_position.txt")
    p, b = float(d["p"][0]), int(d["b"][0])
    gen = np.random.default_rng(7)
    gaps = gen.geometric(p, 200000) - 1                    # Bernoulli(p) positions
    idx = np.cumsum(gaps + 1) - 1
    idx = idx[idx < 2 ** 31 - 1].astype(np.int32)
    words, nbits, _ = oracle.golomb_encode(idx, b)
    per_pos = nbits / idx.size
    assert abs(per_pos - float(d["bits_per_position"][0])) < 0.01 * 8.38
    assert round(16 / per_pos, 1) == float(d["ratio_vs_16bit"][0])


def test_golomb_decoder_rejects_bad_streams():
    idx = np.array([1, 5, 9, 100], np.int32)
    words, nbits, _ = oracle.golomb_encode(idx, 3)
    with pytest.raises(oracle.OracleError):
        oracle.golomb_decode(words, nbits - 1, idx.size, 3)           # truncated
    with pytest.raises(oracle.OracleError):
        oracle.golomb_decode(words, nbits, idx.size - 1, 3)           # bits left over
    with pytest.raises(oracle.OracleError):
        oracle.golomb_decode(words, nbits, idx.size, 3, n_limit=100)  # index out of range
    with pytest.raises(oracle.OracleError):
        oracle.golomb_encode(np.array([5, 5], np.int32), 3)           # not strictly ascending


# ------------------------------------------------------------------------------------ scatter

def test_scatter_worker_order():
    # workers 0,1,2 add 2^24, 1, 1 at index 0: (2^24 + 1) rounds to 2^24 (ties to even), then again
    lists = [(np.array([0, 3], np.int32), np.array([2.0 ** 24, 1.5], np.float32)),
             (np.array([0], np.int32), np.array([1.0], np.float32)),
             (np.array([0, 2], np.int32), np.array([1.0, -0.0], np.float32))]
    dense, mi, mv = oracle.scatter_accumulate(lists, 5)
    assert dense[0] == 2.0 ** 24 and dense[3] == 1.5 and bits(dense[2]) == 0 and dense[1] == 0
    assert mi.tolist() == [0, 2, 3] and mv.tolist() == [2.0 ** 24, 0.0, 1.5]


@pytest.mark.parametrize("W", [1, 2, 4, 8])
def test_scatter_sum_within_rounding(W):
    n = 5000
    gen = np.random.default_rng(W)
    lists, exact, absum = [], [Fraction(0)] * n, [Fraction(0)] * n
    for w in range(W):
        idx = np.sort(gen.choice(n, 300, replace=False)).astype(np.int32)
        val = synth.gaussian(300, w)
        if w == W - 1 and W > 1:
            lists.append((idx, None, 0.25))
            val = np.full(300, 0.25, np.float32)
        else:
            lists.append((idx, val))
        for i, v in zip(idx.tolist(), val.tolist()):
            exact[i] += Fraction(v)
            absum[i] += abs(Fraction(v))
    dense, mi, mv = oracle.scatter_accumulate(lists, n)
    union = sorted(set(np.concatenate([l[0] for l in lists]).tolist()))
    assert mi.tolist() == union
    for i in range(n):
        assert abs(Fraction(float(dense[i])) - exact[i]) <= Fraction(W) * Fraction(1, 2 ** 23) * absum[i]
    if W == 1:
        want = np.zeros(n, np.float32)
        want[lists[0][0]] = lists[0][1]
        assert np.array_equal(dense, want)
    assert np.array_equal(mv, dense[mi])


# ------------------------------------------------------------------------------------ combine

def test_combine_modes():
    n = 1000
    G = synth.gaussian(n, 1)
    L = synth.gaussian(n, 2)
    out = oracle.combine_local(G, L, alpha=0.0, beta=0.5)
    assert np.array_equal(out, L * np.float32(0.5))
    # small integers: every step exact, so the sum mode is plain addition
    Gi = np.arange(n, dtype=np.float32)
    Li = -2 * np.arange(n, dtype=np.float32)
    assert np.array_equal(oracle.combine_local(Gi, Li), -np.arange(n, dtype=np.float32))
    # partial mode with one worker: G equals the worker's own sparse update, so only L remains
    idx = np.array([3, 10, 999], np.int32)
    val = np.array([1.5, -2.25, 7.0], np.float32)
    dense, _, _ = oracle.scatter_accumulate([(idx, val)], n)
    out = oracle.combine_local(dense, L, mode=1, own_idx=idx, own_val=val)
    assert np.array_equal(out.view(np.uint32), (L + np.float32(0)).view(np.uint32))
