// Fixed-order fp64 sums (see osum.cuh for the order).
#include "osum.cuh"

namespace gs {

__global__ void osum_leaves_kernel(SumJob* jobs, int32_t njobs, double* leaves, int64_t leaf_bound,
                                   const int32_t* abort_flag) {
  if (abort_flag && *abort_flag) return;
  const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  unsigned long long members = 0;
  int32_t job = -1;
  if (t < leaf_bound) {
    // the job owning leaf t: the last job whose first leaf is <= t
    int32_t lo = 0, hi = njobs;
    while (lo < hi) {
      int32_t mid = (lo + hi) >> 1;
      if (jobs[mid].leaf_base <= t) lo = mid + 1; else hi = mid;
    }
    job = lo - 1;
    if (job >= 0) {
      const SumJob& J = jobs[job];
      const int64_t leaf = t - J.leaf_base;
      const int64_t nleaves = cdiv(J.len, kSumBlock);
      if (leaf < nleaves) {
        const int64_t b = leaf * kSumBlock;
        const int64_t e = b + kSumBlock < J.len ? b + kSumBlock : J.len;
        double s = 0.0;
        const float* v = J.vals;
        switch (J.mode) {
          case kSumPositive:
            for (int64_t j = b; j < e; ++j) { float x = v[j]; if (x > 0.0f) { s = __dadd_rn(s, (double)x); ++members; } }
            break;
          case kSumNegative:
            for (int64_t j = b; j < e; ++j) { float x = v[j]; if (x < 0.0f) { s = __dadd_rn(s, (double)x); ++members; } }
            break;
          case kSumNegated:
            for (int64_t j = b; j < e; ++j) s = __dadd_rn(s, -(double)v[j]);
            members = (unsigned long long)(e - b);
            break;
          default:
            for (int64_t j = b; j < e; ++j) s = __dadd_rn(s, (double)v[j]);
            members = (unsigned long long)(e - b);
        }
        leaves[t] = s;
      } else {
        job = -1;
      }
    }
  }
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

void osum_launch(SumJob* jobs, int32_t njobs, double* leaves, int64_t leaf_bound,
                 int64_t per_job_leaf_bound, double* partials, const int32_t* abort_flag,
                 cudaStream_t s) {
  if (njobs <= 0) return;
  if (leaf_bound > 0) {
    const int threads = 256;
    osum_leaves_kernel<<<(unsigned)cdiv(leaf_bound, threads), threads, 0, s>>>(jobs, njobs, leaves,
                                                                               leaf_bound, abort_flag);
  }
  const int64_t stride = osum_partial_stride(per_job_leaf_bound);
  dim3 grid((unsigned)stride, (unsigned)njobs);
  osum_tree_kernel<<<grid, 1024, 0, s>>>(jobs, njobs, leaves, partials, stride, abort_flag);
}

}  // namespace gs
