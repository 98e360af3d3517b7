// 2-bit quantisation of a sent list: positives -> their mean, negatives -> their mean, one sign
// bit per entry ("Sparse Communication for Distributed Gradient Descent", Abstract: sparse
// exchange combined with quantisation), with the quantisation error fed back into the residual
// ("Sparse Binary Compression", §II Residual Accumulation).
//
// Kernels: setup (two sum jobs over the list) -> fixed-order fp64 leaf sums -> pairwise tree ->
// apply (q_j, sign words by warp ballot, error feedback, optional in-place dequantisation).
#include "common.cuh"
#include "osum.cuh"

namespace gs {
namespace {

__global__ void q_setup_kernel(const float* val, const int64_t* d_begin, const int64_t* d_end,
                               int64_t capacity, SumJob* jobs, int32_t* ctl, int32_t* d_status) {
  pdl_begin();
  const int64_t b = d_begin ? *d_begin : 0;
  const int64_t e = *d_end;
  int64_t len = e - b;
  if (b < 0 || len < 0 || len > capacity) {
    raise(d_status, GSPARSE_DERR_CAPACITY);
    ctl[0] = 1;
    len = 0;
  } else {
    ctl[0] = 0;
  }
  ctl[2] = 0;
  const int64_t leaves = cdiv(len, kSumBlock);
  for (int c = 0; c < 2; ++c) {
    SumJob J;
    J.vals = val + b;
    J.len = len;
    J.mode = c == 0 ? kSumPositive : kSumNegative;
    J.pad = 0;
    J.leaf_base = c * leaves;   // the pair's leaves are leaves [0, leaves) of both jobs
    J.count = 0;
    J.sum = 0.0;
    J.mean = 0.0f;
    J.done_blocks = 0;
    jobs[c] = J;
  }
}

// Four list positions per thread, j = blockIdx.x * 1024 + k * 256 + threadIdx.x (k = 0..3), so
// the 32 lanes of a warp always hold 32 consecutive positions and one ballot is one sign word.
constexpr int kApplyThreads = 256, kApplyPer = 4;

__global__ void __launch_bounds__(kApplyThreads) q_apply_kernel(
    const int32_t* idx, float* val, const int64_t* d_begin, const int64_t* d_end, const SumJob* jobs,
    float* residual, int64_t n, float* feedback, uint32_t* sign_bits, float* d_means,
    int32_t write_deq, const int32_t* ctl, int32_t* d_status) {
  pdl_begin();
  if (ctl[0]) return;
  const int64_t b = d_begin ? *d_begin : 0;
  const int64_t len = *d_end - b;
  const float mp = jobs[0].mean, mn = jobs[1].mean;
  const int64_t j0 = (int64_t)blockIdx.x * (kApplyThreads * kApplyPer);
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    d_means[0] = mp;
    d_means[1] = mn;
  }
  float xv[kApplyPer];
#pragma unroll
  for (int k = 0; k < kApplyPer; ++k) {
    const int64_t j = j0 + k * kApplyThreads + threadIdx.x;
    xv[k] = j < len ? val[b + j] : 0.0f;
  }
#pragma unroll
  for (int k = 0; k < kApplyPer; ++k) {
    const int64_t j = j0 + k * kApplyThreads + threadIdx.x;
    if ((j & ~(int64_t)31) >= len) break;  // warp-uniform: the warp's 32 positions all lie beyond
    const bool in = j < len;
    const float x = xv[k];
    const bool neg = in && x < 0.0f;
    const uint32_t word = __ballot_sync(kFull, neg);
    if ((threadIdx.x & 31) == 0) sign_bits[j >> 5] = word;
    if (!in) continue;
    const float q = x > 0.0f ? mp : (neg ? mn : 0.0f);
    const float err = __fsub_rn(x, q);
    if (residual) {
      const int32_t i = idx[b + j];
      if (i < 0 || (int64_t)i >= n) raise(d_status, GSPARSE_DERR_INDEX_RANGE);
      else residual[i] = err;
    }
    if (feedback) feedback[j] = err;
    if (write_deq) val[b + j] = q;
  }
}

// ------------------------------------------------------------------------------------------
// segmented form: one call quantises T consecutive sub-lists [off[s], off[s+1]) (e.g. the
// per-tensor outputs of a segmented top-k), each with its own two means

// Validates the offsets and writes two sum jobs per segment (positive, negative members).
__global__ void __launch_bounds__(1024) q_setup_seg_kernel(const float* val, const int64_t* off, int32_t T,
                                                           int64_t capacity, int64_t pair_bound, SumJob* jobs,
                                                           int32_t* ctl, int32_t* d_status) {
  pdl_begin();
  __shared__ int64_t sh[33];
  __shared__ int bad;
  if (threadIdx.x == 0) bad = 0;
  __syncthreads();
  for (int64_t s = threadIdx.x; s <= T; s += blockDim.x) {
    const int64_t o = off[s];
    if (o < 0 || o > capacity || (s > 0 && off[s - 1] > o)) bad = 1;
  }
  __syncthreads();
  if (bad) {
    if (threadIdx.x == 0) {
      raise(d_status, GSPARSE_DERR_CAPACITY);
      ctl[0] = 1;
    }
    return;
  }
  // pair s (positive job 2s, negative job 2s + 1) owns leaves [pb_s, pb_s + L_s) of the pair
  // numbering; the positive job's leaves sit there and the negative job's at pair_bound + pb_s
  int64_t carry = 0;
  for (int64_t base = 0; base < (int64_t)T; base += blockDim.x) {
    const int64_t s = base + threadIdx.x;
    const int64_t len = s < T ? off[s + 1] - off[s] : 0;
    int64_t tot;
    const int64_t ex = block_exclusive_scan(cdiv(len, kSumBlock), sh, &tot);
    for (int c = 0; c < 2 && s < T; ++c) {
      SumJob J;
      J.vals = val + off[s];
      J.len = len;
      J.mode = c ? kSumNegative : kSumPositive;
      J.pad = 0;
      J.leaf_base = carry + ex + (c ? pair_bound : 0);
      J.count = 0;
      J.sum = 0.0;
      J.mean = 0.0f;
      J.done_blocks = 0;
      jobs[2 * s + c] = J;
    }
    carry += tot;
  }
  if (threadIdx.x == 0) ctl[0] = 0;
}

// As q_apply_kernel over positions [off[0], off[T]), each entry with its segment's means; sign
// bits, feedback and positions are counted from off[0].
__global__ void __launch_bounds__(kApplyThreads) q_apply_seg_kernel(
    const int32_t* idx, float* val, const int64_t* off, int32_t T, const SumJob* jobs, float* residual,
    int64_t n, float* feedback, uint32_t* sign_bits, float* d_means, int32_t write_deq, const int32_t* ctl,
    int32_t* d_status) {
  pdl_begin();
  if (ctl[0]) return;
  const int64_t b = off[0];
  const int64_t len = off[T] - b;
  const int64_t j0 = (int64_t)blockIdx.x * (kApplyThreads * kApplyPer);
  if (blockIdx.x == 0)
    for (int64_t s = threadIdx.x; s < T; s += blockDim.x) {
      d_means[2 * s] = jobs[2 * s].mean;
      d_means[2 * s + 1] = jobs[2 * s + 1].mean;
    }
  float xv[kApplyPer];
#pragma unroll
  for (int k = 0; k < kApplyPer; ++k) {
    const int64_t j = j0 + k * kApplyThreads + threadIdx.x;
    xv[k] = j < len ? val[b + j] : 0.0f;
  }
#pragma unroll
  for (int k = 0; k < kApplyPer; ++k) {
    const int64_t j = j0 + k * kApplyThreads + threadIdx.x;
    if ((j & ~(int64_t)31) >= len) break;  // warp-uniform: the warp's 32 positions all lie beyond
    const bool in = j < len;
    const float x = xv[k];
    const bool neg = in && x < 0.0f;
    const uint32_t word = __ballot_sync(kFull, neg);
    if ((threadIdx.x & 31) == 0) sign_bits[j >> 5] = word;
    if (!in) continue;
    const int64_t s = upper_bound_i64(off, (int64_t)T + 1, b + j) - 1;   // the segment of b + j
    const float q = x > 0.0f ? jobs[2 * s].mean : (neg ? jobs[2 * s + 1].mean : 0.0f);
    const float err = __fsub_rn(x, q);
    if (residual) {
      const int32_t i = idx[b + j];
      if (i < 0 || (int64_t)i >= n) raise(d_status, GSPARSE_DERR_INDEX_RANGE);
      else residual[i] = err;
    }
    if (feedback) feedback[j] = err;
    if (write_deq) val[b + j] = q;
  }
}

struct QSegLayout {
  SumJob* jobs;
  double* leaves;
  double* partials;
  int32_t* ctl;
  int64_t leaf_bound, per_job;
  size_t bytes;
};

QSegLayout qs_carve(int64_t capacity, int32_t T, void* ws) {
  QSegLayout L;
  Carver cv(ws);
  L.per_job = cdiv(capacity, kSumBlock);
  L.leaf_bound = L.per_job + T;   // leaves of the pair numbering; each job kind has this many
  L.jobs = cv.take<SumJob>(2 * (int64_t)T);
  L.ctl = cv.take<int32_t>(4);
  L.leaves = cv.take<double>(2 * L.leaf_bound);
  L.partials = cv.take<double>(2 * (int64_t)T * osum_partial_stride(L.per_job));
  L.bytes = cv.off + 256;
  return L;
}

struct QLayout {
  SumJob* jobs;
  double* leaves;
  double* partials;
  int32_t* ctl;
  int64_t leaf_bound, per_job;
  size_t bytes;
};

QLayout q_carve(int64_t capacity, void* ws) {
  QLayout L;
  Carver cv(ws);
  L.per_job = cdiv(capacity, kSumBlock);
  L.leaf_bound = 2 * L.per_job;
  L.jobs = cv.take<SumJob>(2);
  L.ctl = cv.take<int32_t>(4);
  L.leaves = cv.take<double>(L.leaf_bound);
  L.partials = cv.take<double>(2 * osum_partial_stride(L.per_job));
  L.bytes = cv.off + 256;
  return L;
}

}  // namespace
}  // namespace gs

using namespace gs;

extern "C" {

size_t gsparse_quantize_workspace_size(int64_t capacity) {
  if (capacity < 0) return 0;
  return q_carve(capacity, nullptr).bytes;
}

int gsparse_quantize(const int32_t* idx, float* val, const int64_t* d_begin, const int64_t* d_end,
                     int64_t capacity, float* residual, int64_t n, float* feedback_out,
                     uint32_t* sign_bits, float* d_means, int32_t write_dequantized,
                     void* workspace, size_t workspace_bytes, int32_t* d_status,
                     gsparse_stream stream) {
  cudaStream_t st = (cudaStream_t)stream;
  if (capacity < 0 || n < 0 || !d_end || !d_means || (capacity > 0 && (!val || !sign_bits)) ||
      (residual && capacity > 0 && !idx))
    return GSPARSE_ERR_INVALID_ARG;
  if (capacity > INT32_MAX) return GSPARSE_ERR_UNSUPPORTED;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return GSPARSE_ERR_WORKSPACE;
  QLayout L = q_carve(capacity, workspace);
  if (workspace_bytes < L.bytes) return GSPARSE_ERR_WORKSPACE;
  launch(q_setup_kernel, 1, 1, 0, st, val, d_begin, d_end, capacity, L.jobs, L.ctl, d_status);
  osum_launch_pairs(L.jobs, 1, L.leaves, L.per_job, L.per_job, L.partials, L.ctl, st);
  const int64_t blocks = cdiv(capacity > 0 ? capacity : 1, kApplyThreads * kApplyPer);
  launch(q_apply_kernel, (unsigned)blocks, kApplyThreads, 0, st, 
      idx, val, d_begin, d_end, L.jobs, residual, n, feedback_out, sign_bits, d_means,
      write_dequantized, L.ctl, d_status);
  return launch_status();
}

size_t gsparse_quantize_segments_workspace_size(int64_t capacity, int32_t num_segments) {
  if (capacity < 0 || num_segments < 1) return 0;
  return qs_carve(capacity, num_segments, nullptr).bytes;
}

int gsparse_quantize_segments(const int32_t* idx, float* val, const int64_t* d_offsets,
                              int32_t num_segments, int64_t capacity, float* residual, int64_t n,
                              float* feedback_out, uint32_t* sign_bits, float* d_means,
                              int32_t write_dequantized, void* workspace, size_t workspace_bytes,
                              int32_t* d_status, gsparse_stream stream) {
  cudaStream_t st = (cudaStream_t)stream;
  const int32_t T = num_segments;
  if (T < 1 || capacity < 0 || n < 0 || !d_offsets || !d_means || (capacity > 0 && (!val || !sign_bits)) ||
      (residual && capacity > 0 && !idx))
    return GSPARSE_ERR_INVALID_ARG;
  if (capacity > INT32_MAX) return GSPARSE_ERR_UNSUPPORTED;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return GSPARSE_ERR_WORKSPACE;
  QSegLayout L = qs_carve(capacity, T, workspace);
  if (workspace_bytes < L.bytes) return GSPARSE_ERR_WORKSPACE;
  launch(q_setup_seg_kernel, 1, 1024, 0, st, val, d_offsets, T, capacity, L.leaf_bound, L.jobs, L.ctl, d_status);
  osum_launch_pairs(L.jobs, T, L.leaves, L.leaf_bound, L.per_job, L.partials, L.ctl, st);
  const int64_t blocks = cdiv(capacity > 0 ? capacity : 1, kApplyThreads * kApplyPer);
  launch(q_apply_seg_kernel, (unsigned)blocks, kApplyThreads, 0, st, idx, val, d_offsets, T, L.jobs, residual, n,
                                                                 feedback_out, sign_bits, d_means,
                                                                 write_dequantized, L.ctl, d_status);
  return launch_status();
}

}  // extern "C"
