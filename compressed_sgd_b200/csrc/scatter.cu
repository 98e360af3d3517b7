// Receive side: sum of W workers' sparse updates and its combination with the local gradient
// ("Combining Global Sparse Gradients with Local Gradients in Distributed Neural Network
// Training", Abstract; "Sparse Binary Compression", §I: the clients' updates are summed).
//
// Scatter-accumulate works on tiles of 8192 consecutive indices. A streaming pass over the sorted
// lists first records where each worker's entries of every tile start. One CTA owns a tile: it
// adds the workers' entries of the tile worker by worker into a shared-memory accumulator (fixed
// worker order, one fp32 add per entry, so the result is bitwise reproducible), writes the dense
// tile with coalesced stores and counts the touched indices. The merged sparse output is an
// ordered compaction of the touched indices after a scan over the tile counts.
#include "common.cuh"

namespace gs {
namespace {

constexpr int kTile = 8192;
constexpr int kTileShift = 13;
static_assert(kTile == 1 << kTileShift, "tiles are a power of two");
constexpr int kTileThreads = 256;

struct Lists {
  const int32_t* idx[GSPARSE_MAX_WORKERS];
  const float* val[GSPARSE_MAX_WORKERS];
  const float* uni[GSPARSE_MAX_WORKERS];
  const int64_t* cnt[GSPARSE_MAX_WORKERS];
  int64_t cap[GSPARSE_MAX_WORKERS];
};

__device__ __forceinline__ int64_t list_count(const Lists& L, int w) {
  int64_t c = *L.cnt[w];
  if (c < 0) c = 0;
  return c > L.cap[w] ? L.cap[w] : c;
}

// start[t * W + w] = first entry of worker w with index >= t * kTile, for t = 0..ntiles, in one
// streaming pass over each list: entry j starts every tile after its predecessor's tile up to its
// own (index clamped to [0, n] by tile), and the end of the list closes the remaining tiles. For
// an ascending list every table entry is written exactly once; a descent between tiles is flagged
// (and the readers clamp the table to the list). Grid: (x, W).
__device__ __forceinline__ int64_t tile_of_index(int32_t i, int64_t ntiles) {
  if (i < 0) return 0;
  const int64_t t = (int64_t)i / kTile;
  return t < ntiles ? t : ntiles;
}

__device__ __forceinline__ void starts_at(const int32_t* ix, int64_t j, int64_t c, int32_t cur,
                                          int32_t prev, int64_t ntiles, int32_t W, int w,
                                          int64_t* start, int32_t* d_status) {
  const int64_t tj = j < c ? tile_of_index(cur, ntiles) : ntiles;
  const int64_t tp = j > 0 ? tile_of_index(prev, ntiles) : -1;
  if (tj < tp) raise(d_status, GSPARSE_DERR_INDEX_RANGE);
  for (int64_t t = tp + 1; t <= tj; ++t) start[t * W + w] = j;
}

// Sixteen consecutive entries per thread (four 16-byte loads in flight when the list is 16-byte
// aligned).
constexpr int kStartsPer = 16;

__global__ void __launch_bounds__(256) sa_starts_kernel(Lists L, int32_t W, int64_t n, int64_t ntiles,
                                                        int64_t* start, uint32_t* next_tile,
                                                        int32_t* d_status) {
  pdl_begin();
  const int w = blockIdx.y;
  const int64_t c = list_count(L, w);
  const int32_t* ix = L.idx[w];
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    if (w == 0 && next_tile) *next_tile = 0u;  // the combine kernel's tile counter
    if (*L.cnt[w] > L.cap[w]) raise(d_status, GSPARSE_DERR_CAPACITY);
    if (c > 0 && (ix[0] < 0 || (int64_t)ix[c - 1] >= n)) raise(d_status, GSPARSE_DERR_INDEX_RANGE);
  }
  const int64_t j0 = kStartsPer * ((int64_t)blockIdx.x * blockDim.x + threadIdx.x);
  // lanes past the list stay for the shuffle below (they mark nothing)
  int32_t v[kStartsPer];
  if (j0 > c) {
#pragma unroll
    for (int e = 0; e < kStartsPer; ++e) v[e] = 0;
  } else if (j0 + kStartsPer <= c && (reinterpret_cast<uintptr_t>(ix) & 15u) == 0) {
#pragma unroll
    for (int h = 0; h < kStartsPer / 4; ++h) {
      const int4 q = *reinterpret_cast<const int4*>(ix + j0 + 4 * h);
      v[4 * h] = q.x; v[4 * h + 1] = q.y; v[4 * h + 2] = q.z; v[4 * h + 3] = q.w;
    }
  } else {
#pragma unroll
    for (int e = 0; e < kStartsPer; ++e) v[e] = j0 + e < c ? ix[j0 + e] : 0;
  }
  // fast scan, 32-bit: an entry is marked when its raw tile (index >> 13, as unsigned) differs
  // from its predecessor's, which includes every change of the clamped tile and every negative
  // index, and so is the end of the list; starts_at clamps, and a marked entry whose clamped tile
  // equals its predecessor's starts nothing. The predecessor of a thread's first entry is the
  // last entry of the lane before (one load per warp).
  const int lane = threadIdx.x & 31;
  int32_t p0 = __shfl_up_sync(kFull, v[kStartsPer - 1], 1);
  if (j0 > c) return;
  if (lane == 0) p0 = j0 > 0 ? ix[j0 - 1] : -1;
  uint32_t change = 0;
  uint32_t tp = (uint32_t)p0 >> kTileShift;
#pragma unroll
  for (int e = 0; e < kStartsPer; ++e) {
    const uint32_t tv = (uint32_t)v[e] >> kTileShift;
    change |= (uint32_t)(tv != tp) << e;
    tp = tv;
  }
  const int64_t left = c - j0;   // entries of the list from j0 on (>= 0 here)
  uint32_t mark = left < kStartsPer ? (change & ((1u << (uint32_t)left) - 1u)) | (1u << (uint32_t)left)
                                    : change;   // entries of the list, and the list's end
  // the marked entries, in order (rolled loop: the list values come again from L1)
  while (mark) {
    const int e = __ffs(mark) - 1;
    mark &= mark - 1;
    const int64_t j = j0 + e;
    const int32_t cur = j < c ? ix[j] : 0;
    const int32_t prev = j > 0 ? ix[j - 1] : 0;
    starts_at(ix, j, c, cur, prev, ntiles, W, w, start, d_status);
  }
}

// The entries [b, e) of worker w in tile t, clamped to the list.
__device__ __forceinline__ void tile_range(const int64_t* start, int64_t t, int32_t W, int w,
                                           int64_t c, int64_t* b, int64_t* e) {
  int64_t lo = start[t * W + w], hi = start[(t + 1) * W + w];
  lo = lo < 0 ? 0 : (lo > c ? c : lo);
  hi = hi < lo ? lo : (hi > c ? c : hi);
  *b = lo;
  *e = hi;
}

// Accumulates tile t into acc[] (zeroed) and sets touched bits.
__device__ void accumulate_tile(const Lists& L, int32_t W, int64_t t, const int64_t* start,
                                float* acc, uint32_t* touched, int32_t* d_status) {
  const int64_t t0 = t * kTile;
  for (int w = 0; w < W; ++w) {
    int64_t b, e;
    tile_range(start, t, W, w, list_count(L, w), &b, &e);
    const int32_t* ix = L.idx[w];
    const float* vv = L.val[w];
    const float u = (vv || !L.uni[w]) ? 0.0f : *L.uni[w];
    for (int64_t j = b + threadIdx.x; j < e; j += blockDim.x) {
      const int32_t i = ix[j];
      if (j > 0 && ix[j - 1] >= i) { raise(d_status, GSPARSE_DERR_INDEX_RANGE); continue; }
      const int off = (int)(i - t0);
      if (off < 0 || off >= kTile) continue;  // out of range, reported by the bounds pass
      acc[off] = __fadd_rn(acc[off], vv ? vv[j] : u);
      atomicOr(&touched[off >> 5], 1u << (off & 31));
    }
    __syncthreads();  // worker order: all of worker w before any of worker w + 1
  }
}

__global__ void __launch_bounds__(kTileThreads) sa_tile_kernel(Lists L, int32_t W, int64_t n,
                                                               const int64_t* start, float* dense,
                                                               int64_t* tile_count,
                                                               int32_t* d_status) {
  pdl_begin();
  __shared__ __align__(16) float acc[kTile];
  __shared__ uint32_t touched[kTile / 32];
  const int64_t t = blockIdx.x;
  for (int i = threadIdx.x; i < kTile; i += blockDim.x) acc[i] = 0.0f;
  for (int i = threadIdx.x; i < kTile / 32; i += blockDim.x) touched[i] = 0u;
  __syncthreads();
  accumulate_tile(L, W, t, start, acc, touched, d_status);
  const int64_t t0 = t * kTile;
  const int64_t m = (n - t0) < kTile ? (n - t0) : kTile;
  if (dense) {
    if (m == kTile) {
      for (int v = threadIdx.x; v < kTile / 4; v += blockDim.x)
        st_stream(dense + t0 + 4 * v, reinterpret_cast<const float4*>(acc)[v]);
    } else {
      for (int i = threadIdx.x; i < m; i += blockDim.x) dense[t0 + i] = acc[i];
    }
  }
  if (tile_count) {
    __shared__ int64_t sh[33];
    int64_t c = 0;
    for (int i = threadIdx.x; i < kTile / 32; i += blockDim.x) c += __popc(touched[i]);
    int64_t tot;
    block_exclusive_scan(c, sh, &tot);
    if (threadIdx.x == 0) tile_count[t] = tot;
  }
}

__global__ void __launch_bounds__(1024) sa_scan_kernel(int64_t* tile_count, int64_t ntiles,
                                                       int64_t* d_merged_count, int64_t capacity,
                                                       int32_t* ctl, int32_t* d_status) {
  pdl_begin();
  __shared__ int64_t sh[33];
  int64_t carry = 0;
  for (int64_t base = 0; base < ntiles; base += blockDim.x) {
    const int64_t i = base + threadIdx.x;
    const int64_t v = i < ntiles ? tile_count[i] : 0;
    int64_t tot;
    const int64_t ex = block_exclusive_scan(v, sh, &tot);
    if (i < ntiles) tile_count[i] = carry + ex;
    carry += tot;
  }
  if (threadIdx.x == 0) {
    *d_merged_count = carry;
    ctl[0] = carry > capacity;
    if (carry > capacity) raise(d_status, GSPARSE_DERR_CAPACITY);
  }
}

__global__ void __launch_bounds__(kTileThreads) sa_merge_kernel(Lists L, int32_t W, const int64_t* start,
                                                                const int64_t* tile_off,
                                                                int32_t* merged_idx, float* merged_val,
                                                                const int32_t* ctl) {
  pdl_begin();
  __shared__ float acc[kTile];
  __shared__ uint32_t touched[kTile / 32];
  __shared__ int64_t sh[33];
  if (ctl[0]) return;
  const int64_t t = blockIdx.x;
  // skip tiles no worker touches
  bool any = false;
  for (int w = 0; w < W; ++w) {
    int64_t b, e;
    tile_range(start, t, W, w, list_count(L, w), &b, &e);
    any |= b != e;
  }
  if (!any) return;
  for (int i = threadIdx.x; i < kTile; i += blockDim.x) acc[i] = 0.0f;
  for (int i = threadIdx.x; i < kTile / 32; i += blockDim.x) touched[i] = 0u;
  __syncthreads();
  accumulate_tile(L, W, t, start, acc, touched, nullptr);
  // thread k owns bitmap word k (kTile / 32 == blockDim.x)
  const uint32_t word = touched[threadIdx.x];
  int64_t tot;
  const int64_t pre = block_exclusive_scan(__popc(word), sh, &tot);
  int64_t o = tile_off[t] + pre;
  uint32_t wbits = word;
  while (wbits) {
    const int b = __ffs(wbits) - 1;
    wbits &= wbits - 1;
    const int off = threadIdx.x * 32 + b;
    merged_idx[o] = (int32_t)(t * kTile + off);
    merged_val[o] = acc[off];
    ++o;
  }
}

// Fused receive side. The tile-start table (the bounds kernel above) gives each worker's entries
// of every tile. Persistent CTAs take tiles from a shared counter, so tiles crowded with entries
// (dense embedding rows) do not hold up the others. For each tile a CTA requests the
// local-gradient tile first, adds the workers' entries of the tile into a shared accumulator
// (worker by worker, so the sums keep the fixed order; four independent list loads per thread in
// flight), streams out fl(fl(alpha * G) + fl(beta * L)) and finally clears only the entries it
// touched, so the accumulator is zeroed once per CTA rather than once per tile.
constexpr int kCombThreads = 256;
constexpr int kCombPer = 4;

constexpr int kCombPre = 2;  // workers whose first batch of entries is requested together

__global__ void __launch_bounds__(kCombThreads, 4) sa_combine_kernel(Lists L, int32_t W, int64_t n,
                                                                  const int64_t* start,
                                                                  uint32_t* next_tile,
                                                                  const float* Lg, float* out,
                                                                  float alpha, float beta,
                                                                  int32_t own, float* dense,
                                                                  int32_t* d_status) {
  pdl_begin();
  constexpr int kVec = kTile / 4 / kCombThreads;  // float4s of a tile per thread
  __shared__ __align__(16) float acc[kTile];
  __shared__ uint32_t touched[kTile / 32];
  __shared__ uint32_t tnext;
  __shared__ int64_t cnt[GSPARSE_MAX_WORKERS], rb[GSPARSE_MAX_WORKERS], re[GSPARSE_MAX_WORKERS];
  const int64_t ntiles = cdiv(n, kTile);
  for (int i = threadIdx.x; i < kTile; i += blockDim.x) acc[i] = 0.0f;
  for (int i = threadIdx.x; i < kTile / 32; i += blockDim.x) touched[i] = 0u;
  if (threadIdx.x == 0) tnext = atomicAdd(next_tile, 1u);
  __syncthreads();
  int64_t t = tnext;
  // the entry ranges of the tile being worked on sit in rb/re; those of the next tile are loaded
  // (by thread w for worker w) while the current tile is finished
  for (int w = threadIdx.x; w < W; w += blockDim.x) {
    cnt[w] = list_count(L, w);
    if (t < ntiles) tile_range(start, t, W, w, cnt[w], &rb[w], &re[w]);
  }
  while (t < ntiles) {
    __syncthreads();  // every thread has read tnext; rb/re hold tile t
    if (threadIdx.x == 0) tnext = atomicAdd(next_tile, 1u);  // claimed now, read after the tile
    const int64_t t0 = t * kTile;
    const int64_t m = (n - t0) < kTile ? (n - t0) : kTile;
    float4 lv[kVec];
    if (m == kTile) {
#pragma unroll
      for (int k = 0; k < kVec; ++k) lv[k] = ld_stream(Lg + t0 + 4 * (threadIdx.x + k * kCombThreads));
    }
    // first batch of the first kCombPre workers, requested together
    int32_t pi[kCombPre];
    float px[kCombPre];
#pragma unroll
    for (int w = 0; w < kCombPre; ++w) {
      pi[w] = 0;
      px[w] = 0.0f;
      if (w < W) {
        const int64_t j = rb[w] + threadIdx.x;
        if (j < re[w]) {
          pi[w] = L.idx[w][j];
          px[w] = L.val[w] ? L.val[w][j] : (L.uni[w] ? *L.uni[w] : 0.0f);
        }
      }
    }
    for (int w = 0; w < W; ++w) {
      const int32_t* ix = L.idx[w];
      const float* vv = L.val[w];
      const float u = (vv || !L.uni[w]) ? 0.0f : *L.uni[w];
      const int64_t b = rb[w], e = re[w];
      for (int64_t jb = b; jb < e; jb += kCombThreads * kCombPer) {
        int32_t iv[kCombPer];
        float xv[kCombPer];
#pragma unroll
        for (int k = 0; k < kCombPer; ++k) {
          const int64_t j = jb + k * kCombThreads + threadIdx.x;
          if (k == 0 && jb == b && w < kCombPre) {
#pragma unroll
            for (int ww = 0; ww < kCombPre; ++ww)
              if (ww == w) { iv[0] = pi[ww]; xv[0] = px[ww]; }
          } else {
            iv[k] = j < e ? ix[j] : 0;
            xv[k] = j < e ? (vv ? vv[j] : u) : 0.0f;
          }
        }
#pragma unroll
        for (int k = 0; k < kCombPer; ++k) {
          const int64_t j = jb + k * kCombThreads + threadIdx.x;
          if (j >= e) continue;
          if (j > 0 && ix[j - 1] >= iv[k]) { raise(d_status, GSPARSE_DERR_INDEX_RANGE); continue; }
          const int off = (int)(iv[k] - t0);
          if (off < 0 || off >= kTile) continue;  // out of range, reported by the bounds pass
          acc[off] = __fadd_rn(acc[off], xv[k]);
          atomicOr(&touched[off >> 5], 1u << (off & 31));
        }
      }
      __syncthreads();  // worker order: all of worker w before any of worker w + 1
    }
    // the next tile's ranges (tnext is visible after the syncs above)
    const int64_t tn = tnext;
    int64_t nb_ = 0, ne_ = 0;
    if (threadIdx.x < W && tn < ntiles) tile_range(start, tn, W, threadIdx.x, cnt[threadIdx.x], &nb_, &ne_);
    if (dense) {
      if (m == kTile) {
        for (int v = threadIdx.x; v < kTile / 4; v += blockDim.x)
          st_stream(dense + t0 + 4 * v, reinterpret_cast<const float4*>(acc)[v]);
      } else {
        for (int i = threadIdx.x; i < m; i += blockDim.x) dense[t0 + i] = acc[i];
      }
    }
    if (own >= 0) {
      // partial mode: the worker's own sent values leave G before the combination
      const int32_t* ix = L.idx[own];
      const float* vv = L.val[own];
      const float u = (vv || !L.uni[own]) ? 0.0f : *L.uni[own];
      for (int64_t j = rb[own] + threadIdx.x; j < re[own]; j += blockDim.x) {
        const int off = (int)(ix[j] - t0);
        if (off >= 0 && off < kTile) acc[off] = __fsub_rn(acc[off], vv ? vv[j] : u);
      }
      __syncthreads();
    }
    if (m == kTile) {
#pragma unroll
      for (int k = 0; k < kVec; ++k) {
        const int v = threadIdx.x + k * kCombThreads;
        const float4 g = reinterpret_cast<const float4*>(acc)[v];
        float4 o;
        o.x = __fadd_rn(__fmul_rn(alpha, g.x), __fmul_rn(beta, lv[k].x));
        o.y = __fadd_rn(__fmul_rn(alpha, g.y), __fmul_rn(beta, lv[k].y));
        o.z = __fadd_rn(__fmul_rn(alpha, g.z), __fmul_rn(beta, lv[k].z));
        o.w = __fadd_rn(__fmul_rn(alpha, g.w), __fmul_rn(beta, lv[k].w));
        st_stream(out + t0 + 4 * v, o);
      }
    } else {
      for (int i = threadIdx.x; i < m; i += blockDim.x)
        out[t0 + i] = __fadd_rn(__fmul_rn(alpha, acc[i]), __fmul_rn(beta, Lg[t0 + i]));
    }
    __syncthreads();
    // clear what this tile touched (thread k owns bitmap word k)
    for (int k = threadIdx.x; k < kTile / 32; k += blockDim.x) {
      uint32_t word = touched[k];
      touched[k] = 0u;
      while (word) {
        const int bit = __ffs(word) - 1;
        word &= word - 1;
        acc[k * 32 + bit] = 0.0f;
      }
    }
    if (threadIdx.x < W) {
      rb[threadIdx.x] = nb_;
      re[threadIdx.x] = ne_;
    }
    t = tn;
  }
}

// ---------------------------------------------------------------------------------------------
// combine

__global__ void combine_kernel(const float* G, const float* Lg, float* out, int64_t n, float alpha,
                               float beta) {
  pdl_begin();
  const int64_t nv = n >> 2;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t v = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; v < nv; v += stride) {
    const float4 g = ld_stream(G + 4 * v), l = ld_stream(Lg + 4 * v);
    float4 o;
    o.x = __fadd_rn(__fmul_rn(alpha, g.x), __fmul_rn(beta, l.x));
    o.y = __fadd_rn(__fmul_rn(alpha, g.y), __fmul_rn(beta, l.y));
    o.z = __fadd_rn(__fmul_rn(alpha, g.z), __fmul_rn(beta, l.z));
    o.w = __fadd_rn(__fmul_rn(alpha, g.w), __fmul_rn(beta, l.w));
    st_stream(out + 4 * v, o);
  }
  const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (t < (n & 3)) {
    const int64_t i = 4 * nv + t;
    out[i] = __fadd_rn(__fmul_rn(alpha, G[i]), __fmul_rn(beta, Lg[i]));
  }
}

__global__ void combine_partial_kernel(const float* G, const float* Lg, float* out, int64_t n,
                                       float alpha, float beta, const int32_t* own_idx,
                                       const float* own_val, const int64_t* d_count,
                                       int64_t capacity, int32_t* d_status) {
  pdl_begin();
  int64_t K = *d_count;
  if (K > capacity) {
    if (blockIdx.x == 0 && threadIdx.x == 0) raise(d_status, GSPARSE_DERR_CAPACITY);
    K = capacity;
  }
  const int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= K) return;
  const int32_t i = own_idx[j];
  if (i < 0 || (int64_t)i >= n) { raise(d_status, GSPARSE_DERR_INDEX_RANGE); return; }
  const float gi = __fsub_rn(G[i], own_val[j]);
  out[i] = __fadd_rn(__fmul_rn(alpha, gi), __fmul_rn(beta, Lg[i]));
}

struct SLayout {
  int64_t* start;
  int64_t* tile_count;
  int32_t* ctl;
  size_t bytes;
};

void launch_starts(const Lists& L, int32_t W, int64_t n, int64_t ntiles, int64_t* start,
                   uint32_t* next_tile, int32_t* d_status, cudaStream_t st) {
  int64_t most = 0;
  for (int w = 0; w < W; ++w) most = L.cap[w] > most ? L.cap[w] : most;
  const int64_t bx = cdiv(most + 1, kStartsPer * 256);  // entries 0..count of every list
  launch(sa_starts_kernel, dim3((unsigned)bx, (unsigned)W), 256, 0, st, L, W, n, ntiles, start, next_tile,
                                                                      d_status);
}

SLayout s_carve(int32_t W, int64_t n, void* ws) {
  SLayout L;
  Carver cv(ws);
  const int64_t ntiles = cdiv(n, kTile);
  L.start = cv.take<int64_t>((ntiles + 1) * W);
  L.tile_count = cv.take<int64_t>(ntiles + 1);
  L.ctl = cv.take<int32_t>(4);
  L.bytes = cv.off + 256;
  return L;
}

}  // namespace
}  // namespace gs

using namespace gs;

extern "C" {

size_t gsparse_scatter_accumulate_workspace_size(int32_t W, int64_t n) {
  if (W < 1 || n < 0) return 0;
  return s_carve(W, n, nullptr).bytes;
}

int gsparse_scatter_accumulate(const gsparse_list* lists, int32_t W, int64_t n, float* dense_out,
                               int32_t* merged_idx, float* merged_val, int64_t* d_merged_count,
                               int64_t merged_capacity, void* workspace, size_t workspace_bytes,
                               int32_t* d_status, gsparse_stream stream) {
  cudaStream_t st = (cudaStream_t)stream;
  if (!lists || W < 1 || n < 0 || merged_capacity < 0) return GSPARSE_ERR_INVALID_ARG;
  if (W > GSPARSE_MAX_WORKERS || n > INT32_MAX) return GSPARSE_ERR_UNSUPPORTED;
  const bool merged = d_merged_count != nullptr;
  if (merged && merged_capacity > 0 && (!merged_idx || !merged_val)) return GSPARSE_ERR_INVALID_ARG;
  if (dense_out && !aligned16(dense_out)) return GSPARSE_ERR_INVALID_ARG;
  Lists L{};
  for (int w = 0; w < W; ++w) {
    const gsparse_list& x = lists[w];
    if (!x.d_count || x.capacity < 0 || (x.capacity > 0 && (!x.idx || (!x.val && !x.uniform_val))))
      return GSPARSE_ERR_INVALID_ARG;
    L.idx[w] = x.idx;
    L.val[w] = x.val;
    L.uni[w] = x.uniform_val;
    L.cnt[w] = x.d_count;
    L.cap[w] = x.capacity;
  }
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return GSPARSE_ERR_WORKSPACE;
  SLayout S = s_carve(W, n, workspace);
  if (workspace_bytes < S.bytes) return GSPARSE_ERR_WORKSPACE;
  const int64_t ntiles = cdiv(n, kTile);
  if (ntiles == 0) {
    if (merged && cudaMemsetAsync(d_merged_count, 0, sizeof(int64_t), st) != cudaSuccess)
      return GSPARSE_ERR_CUDA;
    return launch_status();
  }
  launch_starts(L, W, n, ntiles, S.start, nullptr, d_status, st);
  launch(sa_tile_kernel, (unsigned)ntiles, kTileThreads, 0, st, L, W, n, S.start, dense_out,
                                                            merged ? S.tile_count : nullptr, d_status);
  if (merged) {
    launch(sa_scan_kernel, 1, 1024, 0, st, S.tile_count, ntiles, d_merged_count, merged_capacity, S.ctl,
                                       d_status);
    launch(sa_merge_kernel, (unsigned)ntiles, kTileThreads, 0, st, L, W, S.start, S.tile_count,
                                                               merged_idx, merged_val, S.ctl);
  }
  return launch_status();
}

size_t gsparse_accumulate_combine_workspace_size(int32_t W, int64_t n) {
  return gsparse_scatter_accumulate_workspace_size(W, n);
}

int gsparse_accumulate_combine(const gsparse_list* lists, int32_t W, int64_t n, const float* L,
                               float* out, float alpha, float beta, int32_t mode, int32_t own,
                               float* dense_out, void* workspace, size_t workspace_bytes,
                               int32_t* d_status, gsparse_stream stream) {
  cudaStream_t st = (cudaStream_t)stream;
  if (!lists || W < 1 || n < 0 || (mode != 0 && mode != 1)) return GSPARSE_ERR_INVALID_ARG;
  if (W > GSPARSE_MAX_WORKERS || n > INT32_MAX) return GSPARSE_ERR_UNSUPPORTED;
  if (mode == 1 && (own < 0 || own >= W)) return GSPARSE_ERR_INVALID_ARG;
  if (n > 0 && (!L || !out || !aligned16(L) || !aligned16(out))) return GSPARSE_ERR_INVALID_ARG;
  if (dense_out && !aligned16(dense_out)) return GSPARSE_ERR_INVALID_ARG;
  Lists Ls{};
  for (int w = 0; w < W; ++w) {
    const gsparse_list& x = lists[w];
    if (!x.d_count || x.capacity < 0 || (x.capacity > 0 && (!x.idx || (!x.val && !x.uniform_val))))
      return GSPARSE_ERR_INVALID_ARG;
    Ls.idx[w] = x.idx;
    Ls.val[w] = x.val;
    Ls.uni[w] = x.uniform_val;
    Ls.cnt[w] = x.d_count;
    Ls.cap[w] = x.capacity;
  }
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return GSPARSE_ERR_WORKSPACE;
  SLayout S = s_carve(W, n, workspace);
  if (workspace_bytes < S.bytes) return GSPARSE_ERR_WORKSPACE;
  const int64_t ntiles = cdiv(n, kTile);
  if (ntiles == 0) return launch_status();
  uint32_t* next_tile = reinterpret_cast<uint32_t*>(S.ctl + 1);
  launch_starts(Ls, W, n, ntiles, S.start, next_tile, d_status, st);
  const int64_t ctas = (int64_t)sm_count() * 4 < ntiles ? (int64_t)sm_count() * 4 : ntiles;
  launch(sa_combine_kernel, (unsigned)ctas, kCombThreads, 0, st, 
      Ls, W, n, S.start, next_tile, L, out, alpha, beta, mode == 1 ? own : -1, dense_out, d_status);
  return launch_status();
}

int gsparse_combine_local(const float* G, const float* L, float* out, int64_t n, float alpha,
                          float beta, int32_t mode, const int32_t* own_idx, const float* own_val,
                          const int64_t* d_own_count, int64_t own_capacity, int32_t* d_status,
                          gsparse_stream stream) {
  cudaStream_t st = (cudaStream_t)stream;
  if (n < 0 || (mode != 0 && mode != 1)) return GSPARSE_ERR_INVALID_ARG;
  if (n > 0 && (!G || !L || !out || !aligned16(G) || !aligned16(L) || !aligned16(out)))
    return GSPARSE_ERR_INVALID_ARG;
  if (mode == 1 && (!d_own_count || own_capacity < 0 || (own_capacity > 0 && (!own_idx || !own_val))))
    return GSPARSE_ERR_INVALID_ARG;
  if (mode == 1 && (out == G || out == L)) return GSPARSE_ERR_INVALID_ARG;
  if (n > 0) {
    const int64_t blocks = cdiv(n, 4 * 256) < 148 * 8 ? cdiv(n, 4 * 256) : 148 * 8;
    launch(combine_kernel, (unsigned)(blocks > 0 ? blocks : 1), 256, 0, st, G, L, out, n, alpha, beta);
  }
  if (mode == 1 && own_capacity > 0)
    launch(combine_partial_kernel, (unsigned)cdiv(own_capacity, 256), 256, 0, st, 
        G, L, out, n, alpha, beta, own_idx, own_val, d_own_count, own_capacity, d_status);
  return launch_status();
}

}  // extern "C"
