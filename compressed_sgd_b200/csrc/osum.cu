// Fixed-order fp64 sums (see osum.cuh for the order).
#include "osum.cuh"

namespace gs {

// One warp sums 32 consecutive leaves (one per lane). The values are read coalesced, 32 leaves x
// 64 positions at a time, into a padded shared tile; each lane then adds its own leaf's positions
// strictly left to right, so every leaf sum is the plain sequential fp64 sum of its block.
constexpr int kLeafWarps = 4;
constexpr int kLeafRound = 64;

__global__ void __launch_bounds__(kLeafWarps * 32) osum_leaves_kernel(SumJob* jobs, int32_t njobs,
                                                                      double* leaves, int64_t leaf_bound,
                                                                      const int32_t* abort_flag) {
  pdl_begin();
  __shared__ float tile[kLeafWarps][32][kLeafRound + 1];
  __shared__ const float* lptr[kLeafWarps][32];
  __shared__ int lcnt[kLeafWarps][32];
  if (abort_flag && *abort_flag) return;
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int64_t t = ((int64_t)blockIdx.x * kLeafWarps + wid) * 32 + lane;
  int32_t job = -1, mode = kSumAll, cnt = 0;
  const float* ptr = nullptr;
  if (t < leaf_bound) {
    // the job owning leaf t: the last job whose first leaf is <= t
    int32_t lo = 0, hi = njobs;
    while (lo < hi) {
      const int32_t mid = (lo + hi) >> 1;
      if (jobs[mid].leaf_base <= t) lo = mid + 1; else hi = mid;
    }
    job = lo - 1;
    if (job >= 0) {
      const SumJob& J = jobs[job];
      const int64_t leaf = t - J.leaf_base;
      if (leaf < cdiv(J.len, kSumBlock)) {
        const int64_t b = leaf * kSumBlock;
        cnt = (int)((J.len - b) < kSumBlock ? (J.len - b) : kSumBlock);
        ptr = J.vals + b;
        mode = J.mode;
      } else {
        job = -1;
      }
    }
  }
  lptr[wid][lane] = ptr;
  lcnt[wid][lane] = cnt;
  __syncwarp();
  double s = 0.0;
  unsigned long long members = 0;
  for (int base = 0; base < kSumBlock; base += kLeafRound) {
    // 32 leaves x 64 positions: lane l fetches position (base + l) and (base + 32 + l) of every
    // leaf, all 64 loads independent, then the values go to the shared tile
    float v0[32], v1[32];
#pragma unroll
    for (int c = 0; c < 32; ++c) {
      const float* pc = lptr[wid][c];
      const int nc = lcnt[wid][c];
      v0[c] = base + lane < nc ? pc[base + lane] : 0.0f;
      v1[c] = base + 32 + lane < nc ? pc[base + 32 + lane] : 0.0f;
    }
#pragma unroll
    for (int c = 0; c < 32; ++c) {
      tile[wid][c][lane] = v0[c];
      tile[wid][c][32 + lane] = v1[c];
    }
    __syncwarp();
    const int m = cnt - base < kLeafRound ? cnt - base : kLeafRound;
    // a value outside the job's sign class is added as +0, which leaves the sum's bits as they
    // are (a positive-class sum starts at +0 and only grows; a negative-class one is +0 until its
    // first member and negative after); no divergent branch when lanes hold different modes
    for (int j = 0; j < m; ++j) {
      const float x = tile[wid][lane][j];
      const bool take = mode == kSumPositive ? x > 0.0f : (mode == kSumNegative ? x < 0.0f : true);
      const double v = mode == kSumNegated ? -(double)x : (double)x;
      s = __dadd_rn(s, take ? v : 0.0);
      members += take;
    }
    __syncwarp();
  }
  if (job >= 0) leaves[t] = s;
  // member counts are integers, so the order of the atomics does not matter: the lowest lane of
  // each group of lanes working on the same job adds the group's total
  const uint32_t same = __match_any_sync(kFull, job);
  unsigned long long grp = 0;
  for (int l = 0; l < 32; ++l) {
    const unsigned long long ml = __shfl_sync(kFull, members, l);
    if ((same >> l) & 1u) grp += ml;
  }
  if (job >= 0 && (int)(threadIdx.x & 31) == __ffs(same) - 1 && grp) atomicAdd(&jobs[job].count, grp);
}

// Paired leaves: jobs 2p (positive members) and 2p + 1 (negative members) of the same list. One
// lane per 256-position block reads the block once and forms both sequential fp64 sums; leaf t of
// the pair numbering (pair p owns leaves [jobs[2p].leaf_base, + its leaf count)) is leaf
// t - jobs[2p].leaf_base of both jobs.
__global__ void __launch_bounds__(kLeafWarps * 32) osum_pair_leaves_kernel(SumJob* jobs, int32_t npairs,
                                                                           double* leaves,
                                                                           int64_t pair_leaf_bound,
                                                                           const int32_t* abort_flag) {
  pdl_begin();
  __shared__ float tile[kLeafWarps][32][kLeafRound + 1];
  __shared__ const float* lptr[kLeafWarps][32];
  __shared__ int lcnt[kLeafWarps][32];
  if (abort_flag && *abort_flag) return;
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int64_t t = ((int64_t)blockIdx.x * kLeafWarps + wid) * 32 + lane;
  int32_t pair = -1, cnt = 0;
  int64_t leaf = 0;
  const float* ptr = nullptr;
  if (t < pair_leaf_bound) {
    int32_t lo = 0, hi = npairs;
    while (lo < hi) {
      const int32_t mid = (lo + hi) >> 1;
      if (jobs[2 * mid].leaf_base <= t) lo = mid + 1; else hi = mid;
    }
    pair = lo - 1;
    if (pair >= 0) {
      const SumJob& J = jobs[2 * pair];
      leaf = t - J.leaf_base;
      if (leaf < cdiv(J.len, kSumBlock)) {
        const int64_t b = leaf * kSumBlock;
        cnt = (int)((J.len - b) < kSumBlock ? (J.len - b) : kSumBlock);
        ptr = J.vals + b;
      } else {
        pair = -1;
      }
    }
  }
  lptr[wid][lane] = ptr;
  lcnt[wid][lane] = cnt;
  __syncwarp();
  double sp = 0.0, sn = 0.0;
  uint32_t np = 0, nn = 0;
  for (int base = 0; base < kSumBlock; base += kLeafRound) {
    float v0[32], v1[32];
#pragma unroll
    for (int c = 0; c < 32; ++c) {
      const float* pc = lptr[wid][c];
      const int nc = lcnt[wid][c];
      v0[c] = base + lane < nc ? pc[base + lane] : 0.0f;
      v1[c] = base + 32 + lane < nc ? pc[base + 32 + lane] : 0.0f;
    }
#pragma unroll
    for (int c = 0; c < 32; ++c) {
      tile[wid][c][lane] = v0[c];
      tile[wid][c][32 + lane] = v1[c];
    }
    __syncwarp();
    const int m = cnt - base < kLeafRound ? cnt - base : kLeafRound;
    // both sums take every position, the other sign's values as +0: sp starts at +0 and only
    // grows, sn is +0 until its first negative value and negative after, so adding +0 changes
    // neither (the same bits as adding each value to its own sum only); no divergent branch
    for (int j = 0; j < m; ++j) {
      const float x = tile[wid][lane][j];
      const bool pos = x > 0.0f, neg = x < 0.0f;
      sp = __dadd_rn(sp, (double)(pos ? x : 0.0f));
      sn = __dadd_rn(sn, (double)(neg ? x : 0.0f));
      np += pos;
      nn += neg;
    }
    __syncwarp();
  }
  if (pair >= 0) {
    leaves[jobs[2 * pair].leaf_base + leaf] = sp;
    leaves[jobs[2 * pair + 1].leaf_base + leaf] = sn;
  }
  // member counts: the lowest lane of each group of lanes on the same pair adds the group's total
  const uint32_t same = __match_any_sync(kFull, pair);
  unsigned long long gp = 0, gn = 0;
  for (int l = 0; l < 32; ++l) {
    const unsigned long long a = __shfl_sync(kFull, (unsigned long long)np, l);
    const unsigned long long b = __shfl_sync(kFull, (unsigned long long)nn, l);
    if ((same >> l) & 1u) { gp += a; gn += b; }
  }
  if (pair >= 0 && lane == __ffs(same) - 1) {
    if (gp) atomicAdd(&jobs[2 * pair].count, gp);
    if (gn) atomicAdd(&jobs[2 * pair + 1].count, gn);
  }
}

// Pairwise reduction of m values held in a[] (shared), ping-ponging with b[]. Returns the result
// in thread 0's view via the returned pointer's element 0 after the final barrier.
__device__ double* tree_reduce_shared(double* a, double* b, int m) {
  int len = m;
  while (len > 1) {
    const int pairs = len >> 1;
    for (int i = threadIdx.x; i < pairs; i += blockDim.x) b[i] = __dadd_rn(a[2 * i], a[2 * i + 1]);
    if ((len & 1) && threadIdx.x == 0) b[pairs] = a[len - 1];
    __syncthreads();
    double* t = a; a = b; b = t;
    len = (len + 1) >> 1;
  }
  return a;
}

__global__ void __launch_bounds__(1024) osum_tree_kernel(SumJob* jobs, int32_t njobs, const double* leaves,
                                 double* partials, int64_t partial_stride,
                                 const int32_t* abort_flag) {
  pdl_begin();
  if (abort_flag && *abort_flag) return;
  __shared__ double sa[kTreeLeaves], sb[kTreeLeaves];
  __shared__ int is_last;
  const int32_t job = blockIdx.y;
  if (job >= njobs) return;
  SumJob& J = jobs[job];
  const int64_t nleaves = cdiv(J.len, kSumBlock);
  const int64_t nblk = cdiv(nleaves, kTreeLeaves);
  const int64_t blk = blockIdx.x;
  if (nleaves == 0) {
    if (blk == 0 && threadIdx.x == 0) { J.sum = 0.0; J.mean = 0.0f; }
    return;
  }
  if (blk >= nblk) return;
  const int64_t first = blk * kTreeLeaves;
  const int m = (int)((nleaves - first) < kTreeLeaves ? (nleaves - first) : kTreeLeaves);
  for (int i = threadIdx.x; i < m; i += blockDim.x) sa[i] = leaves[J.leaf_base + first + i];
  __syncthreads();
  double* r = tree_reduce_shared(sa, sb, m);
  if (nblk == 1) {
    if (threadIdx.x == 0) {
      const double s = r[0];
      J.sum = s;
      J.mean = J.count ? __double2float_rn(__ddiv_rn(s, (double)J.count)) : 0.0f;
    }
    return;
  }
  if (threadIdx.x == 0) {
    partials[job * partial_stride + blk] = r[0];
    __threadfence();
    const uint32_t prev = atomicAdd(&J.done_blocks, 1u);
    is_last = (prev == (uint32_t)(nblk - 1));
  }
  __syncthreads();
  if (!is_last) return;
  __threadfence();
  // the aligned blocks of 2048 leaves are whole subtrees of the pairwise tree, so reducing
  // their results with the same rule continues the same tree
  const int mp = (int)nblk;
  for (int i = threadIdx.x; i < mp; i += blockDim.x)
    sa[i] = ((volatile double*)partials)[job * partial_stride + i];
  __syncthreads();
  r = tree_reduce_shared(sa, sb, mp);
  if (threadIdx.x == 0) {
    const double s = r[0];
    J.sum = s;
    J.mean = J.count ? __double2float_rn(__ddiv_rn(s, (double)J.count)) : 0.0f;
    J.done_blocks = 0;
  }
}

void osum_launch_pairs(SumJob* jobs, int32_t npairs, double* leaves, int64_t pair_leaf_bound,
                       int64_t per_job_leaf_bound, double* partials, const int32_t* abort_flag,
                       cudaStream_t s) {
  if (npairs <= 0) return;
  if (pair_leaf_bound > 0) {
    const int threads = kLeafWarps * 32;
    launch(osum_pair_leaves_kernel, (unsigned)cdiv(pair_leaf_bound, threads), threads, 0, s, 
        jobs, npairs, leaves, pair_leaf_bound, abort_flag);
  }
  const int64_t stride = osum_partial_stride(per_job_leaf_bound);
  dim3 grid((unsigned)stride, (unsigned)(2 * npairs));
  launch(osum_tree_kernel, grid, 1024, 0, s, jobs, 2 * npairs, leaves, partials, stride, abort_flag);
}

void osum_launch(SumJob* jobs, int32_t njobs, double* leaves, int64_t leaf_bound,
                 int64_t per_job_leaf_bound, double* partials, const int32_t* abort_flag,
                 cudaStream_t s) {
  if (njobs <= 0) return;
  if (leaf_bound > 0) {
    const int threads = kLeafWarps * 32;
    launch(osum_leaves_kernel, (unsigned)cdiv(leaf_bound, threads), threads, 0, s, jobs, njobs, leaves,
                                                                               leaf_bound, abort_flag);
  }
  const int64_t stride = osum_partial_stride(per_job_leaf_bound);
  dim3 grid((unsigned)stride, (unsigned)njobs);
  launch(osum_tree_kernel, grid, 1024, 0, s, jobs, njobs, leaves, partials, stride, abort_flag);
}

}  // namespace gs
