// Host helpers of the C ABI: status strings, keep counts, Golomb parameter.
#include <math.h>

#include "common.cuh"

namespace gs {

int sm_count() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (dev < 0 || dev >= 64) return 148;
  if (!cached[dev]) {
    int v = 0;
    cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
    cached[dev] = v > 0 ? v : 148;
  }
  return cached[dev];
}

}  // namespace gs

extern "C" {

const char* gsparse_status_string(int status) {
  switch (status) {
    case GSPARSE_OK: return "ok";
    case GSPARSE_ERR_INVALID_ARG: return "invalid argument";
    case GSPARSE_ERR_WORKSPACE: return "workspace too small or misaligned";
    case GSPARSE_ERR_CUDA: return "CUDA launch error";
    case GSPARSE_ERR_UNSUPPORTED: return "unsupported size or parameter";
    default: return "unknown status";
  }
}

const char* gsparse_version(void) { return "gsparse 0.1 (sm_100a)"; }

int64_t gsparse_k_for(int64_t n_s, int64_t keep_num, int64_t keep_den) {
  if (keep_den <= 0 || keep_num < 0 || keep_num > keep_den) return -1;
  return gs::kept_count(n_s, keep_num, keep_den);
}

int32_t gsparse_golomb_b_star(double p) {
  if (!(p > 0.0) || !(p < 1.0)) return -1;
  const double phi = (1.0 + sqrt(5.0)) / 2.0;
  return 1 + (int32_t)floor(log2(log(phi - 1.0) / log(1.0 - p)));
}

int32_t gsparse_golomb_chunk_hint(int64_t capacity) {
  int32_t c = 64;
  while (c > 4 && capacity / c < 16384) c >>= 1;
  return c;
}

int64_t gsparse_warmup_keep_num(int64_t t, int64_t T, double start, double end, int64_t den) {
  if (den <= 0 || t < 0 || T < 0 || !(start > 0.0) || !(start <= 1.0) || !(end > 0.0) || !(end <= 1.0))
    return -1;
  const double f = (T == 0 || t >= T) ? end : start * pow(end / start, (double)t / (double)T);
  int64_t num = llround(f * (double)den);
  if (num < 1) num = 1;
  if (num > den) num = den;
  return num;
}

}  // extern "C"
