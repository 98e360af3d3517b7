// Fixed-order fp64 sums and means over lists of fp32 values (internal).
//
// The order: list positions are cut into blocks of 256; each block adds its member values left
// to right in fp64 starting from +0.0; the block sums are then combined pairwise, level by level
// (next[m] = cur[2m] + cur[2m+1], an unpaired last element moves up unchanged) until one value
// remains; mean = (float)(sum / (double)count), +0.0f for no members. The pages give no
// summation order; fixing one makes the sent means, and hence the residuals, bitwise
// reproducible.
//
// A "job" is one such sum: a list (device pointer + length) and a membership rule. Jobs are
// described in device memory so that their lengths can come from earlier kernels.
#pragma once

#include "common.cuh"

namespace gs {

constexpr int kSumBlock = 256;       // list positions per leaf block
constexpr int kTreeLeaves = 2048;    // leaf sums reduced by one CTA of the tree kernel

enum SumMode : int32_t { kSumAll = 0, kSumPositive = 1, kSumNegative = 2, kSumNegated = 3 };

struct SumJob {
  const float* vals;   // list base
  int64_t len;         // list length
  int32_t mode;        // SumMode: which entries are members (kSumNegated: all, value negated)
  int32_t pad;
  int64_t leaf_base;   // first leaf of this job in the shared leaf array
  unsigned long long count;  // members (filled by the leaf kernel)
  double sum;          // filled by the tree kernel
  float mean;          // filled by the tree kernel
  uint32_t done_blocks;  // completion counter of the tree kernel (must start at 0)
};

// Leaf sums: one sequential fp64 sum per 256-position block of one job (one lane per block).
__global__ void osum_leaves_kernel(SumJob* jobs, int32_t njobs, double* leaves, int64_t leaf_bound,
                                   const int32_t* abort_flag);

// Tree: grid (x = tree blocks of 2048 leaves per job, bound; y = job). The last CTA of a job to
// finish reduces the block partials and writes sum and mean.
__global__ void __launch_bounds__(1024) osum_tree_kernel(SumJob* jobs, int32_t njobs, const double* leaves,
                                 double* partials, int64_t partial_stride,
                                 const int32_t* abort_flag);

// Host: grid sizes for a set of jobs whose total leaves are bounded by leaf_bound and whose
// per-job leaves are bounded by per_job_leaf_bound.
void osum_launch(SumJob* jobs, int32_t njobs, double* leaves, int64_t leaf_bound,
                 int64_t per_job_leaf_bound, double* partials, const int32_t* abort_flag,
                 cudaStream_t s);

// Paired jobs: jobs[2p] (positive members) and jobs[2p + 1] (negative members) of one list, with
// jobs[2p].leaf_base the pair's first leaf in a numbering of pair_leaf_bound leaves and
// jobs[2p + 1].leaf_base its own leaf range; the list is read once per pair.
void osum_launch_pairs(SumJob* jobs, int32_t npairs, double* leaves, int64_t pair_leaf_bound,
                       int64_t per_job_leaf_bound, double* partials, const int32_t* abort_flag,
                       cudaStream_t s);

inline int64_t osum_partial_stride(int64_t per_job_leaf_bound) {
  return cdiv(per_job_leaf_bound > 0 ? per_job_leaf_bound : 1, kTreeLeaves);
}

}  // namespace gs
