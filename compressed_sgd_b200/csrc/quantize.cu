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
    J.leaf_base = c * leaves;
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
  q_setup_kernel<<<1, 1, 0, st>>>(val, d_begin, d_end, capacity, L.jobs, L.ctl, d_status);
  osum_launch(L.jobs, 2, L.leaves, L.leaf_bound, L.per_job, L.partials, L.ctl, st);
  const int64_t blocks = cdiv(capacity > 0 ? capacity : 1, kApplyThreads * kApplyPer);
  q_apply_kernel<<<(unsigned)blocks, kApplyThreads, 0, st>>>(
      idx, val, d_begin, d_end, L.jobs, residual, n, feedback_out, sign_bits, d_means,
      write_dequantized, L.ctl, d_status);
  return launch_status();
}

}  // extern "C"
