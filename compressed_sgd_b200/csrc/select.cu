// Exact residual top-k and sparse binarisation on B200.
//
// Method: "Sparse Communication for Distributed Gradient Descent" (Aji & Heafield 2017),
// Abstract — drop the 99% smallest updates by |value|; "Sparse Binary Compression" (Sattler et
// al. 2018), §II Residual Accumulation, Sparse Binarization, Communication Delay.
//
// Design (one call = a fixed sequence of kernels on the caller's stream, no host sync):
//  1. plan     per-segment sizes, k_s, output bases and the split of each segment into "pieces"
//              (contiguous ranges of <= Lp entries, one warp each).
//  2. sample   per segment, a 16384-entry sample of acc = g + r gives a candidate threshold
//              T_lo that a little more than k_s entries reach (the exact k_s-th key when the
//              whole segment fits in the sample).
//  3. pass 1   the only full stream over the data: 128-bit loads of g and r, acc = fl(g + r),
//              residual <- acc (or +0 for candidates in top-k mode, so sent entries never need
//              a second write), candidates (key >= T_lo) appended per piece in index order by a
//              warp-ballot compaction, and a shared-memory histogram of candidate keys.
//  4. check    a segment whose sample threshold was too high (fewer than k_s candidates) is
//              redone exhaustively; pieces whose candidate store overflowed are re-read from
//              the residual. Both routes give the same result, only slower.
//  5-7.        three radix-select levels (11 + 11 + 9 bits of the key) over the candidates give
//              the exact k_s-th key T and how many entries equal to T are taken.
//  8-9. count + scan per piece, then emit: selected candidates are written in index order;
//              candidates not selected get their acc back into the residual.
// Ties: keys equal to T are taken in ascending index order, so the lowest indices win.
#include <math.h>

#include <atomic>
#include <type_traits>

#include "common.cuh"
#include "osum.cuh"

namespace gs {
namespace {

constexpr uint32_t kNone = 0x80000000u;  // a threshold no 31-bit key reaches
constexpr int kBins1 = 2048, kBins2 = 2048, kBins3 = 512;
constexpr int kHist = kBins1 + kBins2 + kBins3;  // per problem
constexpr int64_t kGranule = 512;                // entries per warp iteration (32 lanes x 16)
constexpr int64_t kTargetPieces = 148 * 64;      // four pieces per pass-1 warp slot of a B200 (16 per
                                                  // SM), so a crowded piece holds up less of the pass
constexpr int kSample = 1 << 18;                 // sampled entries per segment
constexpr int kSampleRuns = kSample / 32;        // ... as evenly spaced runs of 32 entries
constexpr int kSampleCtas = 256;                 // CTAs sharing one segment's sample
static_assert(kSample % (32 * kSampleCtas) == 0 && kSample / kSampleCtas <= 1024,
              "each sample CTA takes whole runs, at most 32 of them");
constexpr int kWarps = 8;                        // warps (pieces) per CTA
constexpr int kMaxChunks = 64;                   // pool chunks one piece may claim
constexpr int kUnitShift = 11;                   // work unit after pass 1: >= 2048 store positions,
constexpr int kReadUnits = 8;                    // ... or 1/8 of a re-read piece
constexpr int kThreads = kWarps * 32;

struct Sel {
  const float* g;
  float* r;
  float* u;    // momentum (null: none): v = fl(fl(mom * u) + g) replaces g, u <- v, sent u <- 0
  float mom;
  int64_t n;
  int32_t T, C;       // segments; classes: 1 = |x| (top-k), 2 = x > 0 and x < 0 (binarise)
  int32_t zero_mode;  // top-k: write +0 for candidates in pass 1
  int32_t wait_test;  // test hook: the first ring wait of every warp is on a barrier nothing completes
  int64_t Lp, Q, cap;
  int64_t *seg_lo, *seg_n, *seg_k, *seg_kbase, *seg_pbase;
  uint32_t *tlo, *redo, *pfx, *thr;
  int64_t *keff, *krem, *need_eq;
  uint32_t* hist;  // [P][kHist]
  uint32_t *pcnt, *prsrc, *pgt, *peq, *ptake;  // pgt..poff: per work unit and class
  int64_t* poff;
  int64_t* uoff;    // [Q + 1] first work unit of each piece (the last entry: the number of units)
  int32_t* upiece;  // [units] the piece of each work unit
  int64_t Ur, units_bound;
  int32_t ushift;   // a stored piece's unit: 2^ushift store positions
  // candidate stores: Q primary stores of cap slots, then a pool of chunks of 2^chunk_shift slots
  // that a piece claims (at most max_chunks) once its primary store is full
  int32_t* cidx;
  float* cval;
  int32_t* pchunk;    // [Q][max_chunks] pool chunk ids claimed by each piece, in order
  uint32_t* pnch;     // [Q] chunks claimed
  int64_t pool_chunks;
  int32_t chunk_shift, max_chunks;
  int32_t* ctl;  // [0] abort, [1] any redo, [2] next free pool chunk
  // sample: two-level histogram of the sampled keys per problem
  uint32_t *shist, *scount, *sdone, *sb1, *sblo, *ssub;
  int64_t *srank, *sabove, *smcap;
  unsigned long long* svar;  // per problem: sum and sum of squares of the per-run counts
  // pending residual writes applied in the sample and pass 1 (null: none); pstart[q] is the
  // first write at or after piece q's first entry ([Q + 1])
  uint32_t* pstart;
  uint32_t* srun;   // [T][kSampleRuns][2]: each sampled run's range of pending writes (level 1 -> 2)
  const int32_t* pw_idx;
  const float* pw_val;
  const int64_t* pw_count;
  int64_t pw_cap;
  int32_t* d_status;
  // binarise
  int32_t* lidx;
  float* lval;
  int32_t* bsel;
};

struct Piece {
  int64_t lo, hi;
  int32_t s;
};

__device__ __forceinline__ int64_t total_pieces(const Sel& a) { return a.seg_pbase[a.T]; }

__device__ __forceinline__ Piece piece_of(const Sel& a, int64_t q) {
  Piece p;
  p.s = (int32_t)(upper_bound_i64(a.seg_pbase, a.T + 1, q) - 1);
  p.lo = a.seg_lo[p.s] + (q - a.seg_pbase[p.s]) * a.Lp;
  const int64_t end = a.seg_lo[p.s] + a.seg_n[p.s];
  p.hi = p.lo + a.Lp < end ? p.lo + a.Lp : end;
  return p;
}

// The piece holding entry i (0 <= i < n).
__device__ __forceinline__ int64_t piece_containing(const Sel& a, int64_t i) {
  const int64_t s = upper_bound_i64(a.seg_lo, a.T, i) - 1;  // the last segment starting at or before i
  const int64_t sc = s < 0 ? 0 : s;
  const int64_t q = a.seg_pbase[sc] + (i - a.seg_lo[sc]) / a.Lp;
  const int64_t qmax = a.seg_pbase[sc + 1] - 1;
  return q > qmax ? qmax : q;
}

// Slots of a piece's candidate store: positions [0, cap) in its primary store, later positions in
// its pool chunks (chunk c holds positions cap + c * 2^chunk_shift onwards).
__device__ __forceinline__ uint32_t room_of(const Sel& a, int64_t q) {
  return (uint32_t)a.cap + (a.pnch[q] << a.chunk_shift);
}

__device__ __forceinline__ int64_t slot_of(const Sel& a, int64_t q, uint32_t pos) {
  if (pos < (uint32_t)a.cap) return q * a.cap + pos;
  const uint32_t o = pos - (uint32_t)a.cap;
  const int64_t c = a.pchunk[q * a.max_chunks + (o >> a.chunk_shift)];
  return a.Q * a.cap + (c << a.chunk_shift) + (o & ((1u << a.chunk_shift) - 1u));
}

// Work units of the steps after pass 1 (histogram levels 2-3, count, scan, emit): a piece with a
// candidate store is split into units of 2^ushift store positions (at least its primary store,
// so only pieces that spilled into the pool have more than one), a re-read piece into units of
// Ur entries, so a piece crowded with candidates is shared by several warps.
__device__ __forceinline__ int64_t unit_count(const Sel& a) { return a.uoff[total_pieces(a)]; }

__device__ __forceinline__ int64_t unit_piece(const Sel& a, int64_t u) { return a.upiece[u]; }

__device__ __forceinline__ int64_t units_of_piece(const Sel& a, int64_t q) {
  if (a.prsrc[q]) {
    const Piece P = piece_of(a, q);
    return cdiv(P.hi - P.lo, a.Ur);
  }
  return cdiv((int64_t)a.pcnt[q], (int64_t)1 << a.ushift);
}

// The range of unit k of piece q: store positions [b, e), or for a re-read piece entries [b, e).
__device__ __forceinline__ void unit_range(const Sel& a, int64_t q, const Piece& P, int64_t k,
                                           int64_t* b, int64_t* e) {
  if (a.prsrc[q]) {
    *b = P.lo + k * a.Ur;
    *e = *b + a.Ur < P.hi ? *b + a.Ur : P.hi;
  } else {
    const int64_t cnt = a.pcnt[q];
    *b = k << a.ushift;
    *e = *b + ((int64_t)1 << a.ushift) < cnt ? *b + ((int64_t)1 << a.ushift) : cnt;
  }
}

// class of an accumulated value: top-k has one class; binarise splits by sign (zeros in none)
template <int C>
__device__ __forceinline__ int class_of(float x) {
  if (C == 1) return 0;
  return x > 0.0f ? 0 : (x < 0.0f ? 1 : -1);
}

__device__ __forceinline__ uint32_t* hist_of(const Sel& a, int64_t p, int level) {
  return a.hist + p * kHist + (level == 1 ? 0 : (level == 2 ? kBins1 : kBins1 + kBins2));
}

// Histogram sink of a CTA: counts for the CTA's first segment go to shared memory and are
// flushed once; counts for other segments (CTAs straddling a segment boundary) go straight to
// global memory.
template <int C, int BINS>
struct CtaHist {
  uint32_t sh[C * BINS];
  int64_t primary;
  __device__ void add(const Sel& a, int32_t s, int c, uint32_t bin, int level) {
    if (s == primary) atomicAdd(&sh[c * BINS + bin], 1u);
    else atomicAdd(hist_of(a, (int64_t)s * C + c, level) + bin, 1u);
  }
  __device__ void init(const Sel& a, int64_t q0) {
    init_seg(q0 < total_pieces(a) ? piece_of(a, q0).s : -1);
  }
  __device__ void init_seg(int64_t seg) {
    for (int i = threadIdx.x; i < C * BINS; i += blockDim.x) sh[i] = 0;
    if (threadIdx.x == 0) primary = seg;
  }
  // adds the shared counts of bins [0, bins) to the primary segment's histograms
  __device__ void flush(const Sel& a, int level, int bins) {
    if (primary < 0) return;
    for (int i = threadIdx.x; i < C * BINS; i += blockDim.x) {
      const uint32_t h = sh[i];
      if (h && (i % BINS) < bins) atomicAdd(hist_of(a, primary * C + i / BINS, level) + (i % BINS), h);
    }
  }
};

// ------------------------------------------------------------------------------------------
// block helpers for the select steps (blockDim.x == 1024)

// Given bin counts h[0..B) and a rank (1 = largest), find the bin b holding the rank-th largest
// entry: sum(h[b+1..B)) < rank <= sum(h[b..B)). Returns b and the count above it.
__device__ void block_find_bin(const uint32_t* h, int B, int64_t rank, uint32_t* bin_out,
                               int64_t* above_out) {
  __shared__ int64_t sh[33];
  __shared__ uint32_t fb;
  __shared__ int64_t fa;
  const int per = (B + (int)blockDim.x - 1) / (int)blockDim.x;
  // thread t owns bins [B - (t+1)*per, B - t*per) walked downwards
  const int hi = B - (int)threadIdx.x * per;
  int64_t mine = 0;
  for (int j = 0; j < per; ++j) {
    const int b = hi - 1 - j;
    if (b >= 0) mine += h[b];
  }
  int64_t tot;
  int64_t above = block_exclusive_scan(mine, sh, &tot);
  if (threadIdx.x == 0) { fb = 0; fa = 0; }
  __syncthreads();
  for (int j = 0; j < per; ++j) {
    const int b = hi - 1 - j;
    if (b < 0) break;
    const int64_t c = h[b];
    if (above < rank && rank <= above + c) { fb = (uint32_t)b; fa = above; }
    above += c;
  }
  __syncthreads();
  *bin_out = fb;
  *above_out = fa;
  __syncthreads();
}

// ------------------------------------------------------------------------------------------
// 1. plan

__global__ void __launch_bounds__(1024) plan_kernel(Sel a, const int64_t* seg, int64_t knum, int64_t kden,
                            int64_t out_capacity, int64_t* out_offsets) {
  pdl_begin();
  __shared__ int64_t sh[33];
  __shared__ int bad;
  if (threadIdx.x == 0) bad = 0;
  __syncthreads();
  int64_t carry_k = 0, carry_p = 0;
  for (int64_t base = 0; base < a.T; base += blockDim.x) {
    const int64_t s = base + threadIdx.x;
    int64_t k = 0, np = 0;
    if (s < a.T) {
      const int64_t lo = seg ? seg[s] : 0;
      const int64_t hi = seg ? seg[s + 1] : a.n;
      if (hi < lo || lo < 0 || hi > a.n || (s == 0 && lo != 0) || (s == a.T - 1 && hi != a.n)) bad = 1;
      const int64_t ns = hi > lo ? hi - lo : 0;
      k = kept_count(ns, knum, kden);
      np = cdiv(ns, a.Lp);
      a.seg_lo[s] = lo;
      a.seg_n[s] = ns;
      a.seg_k[s] = k;
    }
    int64_t tk, tp;
    const int64_t ek = block_exclusive_scan(k, sh, &tk);
    const int64_t ep = block_exclusive_scan(np, sh, &tp);
    if (s < a.T) {
      a.seg_kbase[s] = carry_k + ek;
      a.seg_pbase[s] = carry_p + ep;
    }
    carry_k += tk;
    carry_p += tp;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    a.seg_kbase[a.T] = carry_k;
    a.seg_pbase[a.T] = carry_p;
    if (bad || carry_p > a.Q) {
      raise(a.d_status, GSPARSE_DERR_SEGMENTS);
      a.ctl[0] = 1;
      a.seg_pbase[a.T] = 0;
    } else if (carry_k > out_capacity) {
      raise(a.d_status, GSPARSE_DERR_CAPACITY);
      a.ctl[0] = 1;
      a.seg_pbase[a.T] = 0;
    }
  }
  __syncthreads();
  if (out_offsets && !a.ctl[0])
    for (int64_t s = threadIdx.x; s <= a.T; s += blockDim.x) out_offsets[s] = a.seg_kbase[s];
}

// ------------------------------------------------------------------------------------------
// 2. sample: candidate thresholds
//
// Each segment's sample (the whole segment when it has at most kSample entries, else kSample
// entries in evenly spaced runs of 32) is split over kSampleCtas CTAs. Level 1 histograms the
// top 11 key bits. Level 2 re-reads the sample and histograms the keys of a range of level-1
// bins at a finer resolution; its last CTA sets T_lo to the lower edge of the fine bucket holding
// the m-th largest sampled key. With the whole segment in the sample m = k, so at least k
// entries reach T_lo. Otherwise m sits three standard deviations (plus 16) above the expected
// sample count e = k * S / n_s. Entries of one run can be strongly correlated (a run inside an
// all-zero embedding row, or inside a tensor of larger scale), so the deviation is estimated
// from the spread of the per-run counts measured at level 2, never below the independent-entry
// figure sqrt(e) and never above sqrt(32 e), which bounds the variance of a sum of run counts in
// [0, 32]. Level 1 therefore picks the bins of both ends, m0 = e + 3 sqrt(e) + 16 and
// m_max = e + 3 sqrt(32 e) + 16, and level 2 covers the bins between them. A shortfall (fewer than
// k entries reaching T_lo) is still caught and redone by the check step.

__device__ __forceinline__ uint32_t pending_count(const Sel& a) {
  if (!a.pw_idx) return 0;
  int64_t c = *a.pw_count;
  c = c < 0 ? 0 : (c > a.pw_cap ? a.pw_cap : c);
  return (uint32_t)c;
}

// The gradient term of entry i: g_i, or with momentum v_i = fl(fl(mom * u_i) + g_i).
__device__ __forceinline__ float grad_at(const Sel& a, int64_t i) {
  return a.u ? __fadd_rn(__fmul_rn(a.mom, a.u[i]), a.g[i]) : a.g[i];
}

__device__ __forceinline__ float4 momentum4(float m, float4 u, float4 g) {
  return make_float4(__fadd_rn(__fmul_rn(m, u.x), g.x), __fadd_rn(__fmul_rn(m, u.y), g.y),
                     __fadd_rn(__fmul_rn(m, u.z), g.z), __fadd_rn(__fmul_rn(m, u.w), g.w));
}

// First pending write at or after entry x: searched only among the writes of x's piece.
__device__ __forceinline__ uint32_t pending_lower_bound(const Sel& a, int64_t x) {
  if (x <= 0) return 0;
  if (x >= a.n) return pending_count(a);
  const int64_t q = piece_containing(a, x);
  const uint32_t b = a.pstart[q], e = a.pstart[q + 1];
  return b + (uint32_t)lower_bound_i32(a.pw_idx + b, e > b ? e - b : 0, x);
}

// The residual value of entry i with the pending writes applied (the writes in [b, e) of the
// list, which must hold every write of the caller's range).
__device__ __forceinline__ float residual_at(const Sel& a, int64_t i, uint32_t b, uint32_t e) {
  if (b < e) {
    const int64_t pos = lower_bound_i32(a.pw_idx + b, e - b, i);
    if (pos < (int64_t)(e - b) && a.pw_idx[b + pos] == i) return a.pw_val[b + pos];
  }
  return a.r[i];
}

__device__ __forceinline__ int64_t sample_pos(int64_t lo, int64_t ns, int64_t j) {
  if (ns <= kSample) return lo + j;
  return lo + (j >> 5) * (ns - 32) / (kSampleRuns - 1) + (j & 31);
}

__device__ __forceinline__ uint32_t* shist_of(const Sel& a, int64_t p, int level) {
  return a.shist + p * (2 * kBins1) + (level == 1 ? 0 : kBins1);
}

// smallest s with 2^s >= v (v >= 1)
__device__ __forceinline__ uint32_t ceil_log2(uint32_t v) { return v <= 1 ? 0u : 32u - __clz(v - 1u); }

constexpr int kSampleThreads = 512;    // two sampled entries per thread, two CTAs per SM

template <int C>
__global__ void __launch_bounds__(kSampleThreads) sample_kernel(Sel a, int level, int exhaustive) {
  pdl_begin();
  __shared__ uint32_t h[C * kBins1];
  __shared__ uint32_t cnt[C];
  __shared__ unsigned long long vsum[C], vsq[C];
  __shared__ int last;
  if (a.ctl[0]) return;
  const int32_t s = blockIdx.y;
  const int64_t lo = a.seg_lo[s], ns = a.seg_n[s], k = a.seg_k[s];
  const int64_t P0 = (int64_t)s * C;
  if (k == 0 || ns == 0 || exhaustive) {
    if (level == 1 && blockIdx.x == 0 && threadIdx.x < C) {
      a.tlo[P0 + threadIdx.x] = (k == 0 || ns == 0) ? kNone : 0u;
      a.sb1[P0 + threadIdx.x] = kNone;
    }
    return;
  }
  // level 2: per class the level-1 bins [blo, b1] at 2^sub fine bins each
  uint32_t b1[C], blo[C], sub[C];
#pragma unroll
  for (int c = 0; c < C; ++c) {
    b1[c] = level == 2 ? a.sb1[P0 + c] : kNone;
    blo[c] = level == 2 && b1[c] != kNone ? a.sblo[P0 + c] : 0u;
    sub[c] = level == 2 && b1[c] != kNone ? a.ssub[P0 + c] : 0u;
  }
  if (level == 2) {
    bool any = false;
#pragma unroll
    for (int c = 0; c < C; ++c) any |= b1[c] != kNone;
    if (!any) return;
  }
  for (int i = threadIdx.x; i < C * kBins1; i += blockDim.x) h[i] = 0;
  if (threadIdx.x < C) {
    cnt[threadIdx.x] = 0;
    vsum[threadIdx.x] = 0;
    vsq[threadIdx.x] = 0;
  }
  __syncthreads();
  const int64_t S = ns < kSample ? ns : kSample;
  const int64_t j0 = S * blockIdx.x / gridDim.x, j1 = S * (blockIdx.x + 1) / gridDim.x;
  // The sample sees the pending residual writes. A fully sampled segment: the writes of this
  // CTA's contiguous slice. A sparsely sampled one: per run of 32 entries, the writes falling in
  // the run (one binary search per run, by the lanes of the first warp).
  __shared__ uint32_t pwb, pwe;
  __shared__ uint32_t run_b[32], run_e[32];
  const uint32_t pc = pending_count(a);
  const bool sparse = ns > kSample;  // then j1 - j0 is a multiple of blockDim.x and one warp
                                     // iteration is one run
  const bool runs = pc && sparse;
  if (threadIdx.x == 0) {
    pwb = pwe = 0;
    if (pc && ns <= kSample) {
      pwb = pending_lower_bound(a, lo + j0);
      pwe = pending_lower_bound(a, lo + j1);
    }
  }
  if (runs && threadIdx.x < 32) {
    const int64_t jr = j0 + 32 * threadIdx.x;       // j0 is a multiple of 32 here
    uint32_t b = 0, e = 0;
    if (jr < j1) {
      uint32_t* rr = a.srun + 2 * ((int64_t)s * kSampleRuns + (jr >> 5));
      if (level == 1) {
        const int64_t start = sample_pos(lo, ns, jr);
        b = pending_lower_bound(a, start);
        const uint32_t span = pc - b < 33u ? pc - b : 33u;
        e = b + (uint32_t)lower_bound_i32(a.pw_idx + b, span, start + 32);
        rr[0] = b;
        rr[1] = e;
      } else {
        b = rr[0];   // found by level 1 (same runs, same CTA split)
        e = rr[1];
      }
    }
    run_b[threadIdx.x] = b;
    run_e[threadIdx.x] = e;
  }
  __syncthreads();
  // the CTA's slice holds at most 1024 entries: every thread loads its (at most two) before any
  // is histogrammed
  static_assert(kSample / kSampleCtas <= 2 * kSampleThreads, "two sampled entries per thread");
  constexpr int kIt = (kSample / kSampleCtas + kSampleThreads - 1) / kSampleThreads;
  float xs[kIt];
#pragma unroll
  for (int it = 0; it < kIt; ++it) {
    const int64_t j = j0 + threadIdx.x + (int64_t)it * blockDim.x;
    xs[it] = 0.0f;
    if (j < j1) {
      const int64_t i = sample_pos(lo, ns, j);
      const uint32_t cb = runs ? run_b[(j - j0) >> 5] : pwb;
      const uint32_t ce = runs ? run_e[(j - j0) >> 5] : pwe;
      xs[it] = __fadd_rn(grad_at(a, i), residual_at(a, i, cb, ce));
    }
  }
#pragma unroll
  for (int it = 0; it < kIt; ++it) {
    const int64_t j = j0 + threadIdx.x + (int64_t)it * blockDim.x;
    const float x = xs[it];
    const int c = j < j1 ? class_of<C>(x) : -1;
    const uint32_t key = mag_key(x);
    if (level == 2 && sparse) {
      // this run's count of class members in bin b1 or above
#pragma unroll
      for (int cc = 0; cc < C; ++cc) {
        const bool hit = c == cc && b1[cc] != kNone && (key >> 20) >= b1[cc];
        const uint32_t nr = __popc(__ballot_sync(kFull, hit));
        if ((threadIdx.x & 31) == 0 && nr) {
          atomicAdd(&vsum[cc], (unsigned long long)nr);
          atomicAdd(&vsq[cc], (unsigned long long)(nr * nr));
        }
      }
    }
    if (c < 0) continue;
    if (level == 1) {
      atomicAdd(&h[c * kBins1 + (key >> 20)], 1u);
      atomicAdd(&cnt[c], 1u);
    } else if (b1[c] != kNone && (key >> 20) >= blo[c] && (key >> 20) <= b1[c]) {
      atomicAdd(&h[c * kBins1 + ((key >> (20 - sub[c])) - (blo[c] << sub[c]))], 1u);
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < C * kBins1; i += blockDim.x)
    if (h[i]) atomicAdd(shist_of(a, P0 + i / kBins1, level) + (i % kBins1), h[i]);
  if (level == 1 && threadIdx.x < C && cnt[threadIdx.x]) atomicAdd(&a.scount[P0 + threadIdx.x], cnt[threadIdx.x]);
  if (level == 2 && threadIdx.x < C && vsum[threadIdx.x]) {
    atomicAdd(&a.svar[2 * (P0 + threadIdx.x)], vsum[threadIdx.x]);
    atomicAdd(&a.svar[2 * (P0 + threadIdx.x) + 1], vsq[threadIdx.x]);
  }
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) last = atomicAdd(&a.sdone[2 * s + level - 1], 1u) == gridDim.x - 1;
  __syncthreads();
  if (!last) return;
  __threadfence();
  const double e = (double)k * (double)S / (double)ns;
  for (int c = 0; c < C; ++c) {
    const int64_t p = P0 + c;
    if (level == 2 && b1[c] == kNone) continue;
    for (int i = threadIdx.x; i < kBins1; i += blockDim.x) h[i] = ((volatile uint32_t*)shist_of(a, p, level))[i];
    __syncthreads();
    if (level == 1) {
      const int64_t count = ((volatile uint32_t*)a.scount)[p];
      int64_t m0, mmax;
      if (!sparse) {
        m0 = mmax = k < count ? k : count;          // the whole segment is in the sample
      } else {
        m0 = (int64_t)ceil(e + 3.0 * sqrt(e) + 16.0);
        mmax = (int64_t)ceil(e + 3.0 * sqrt(32.0 * e) + 16.0);
      }
      if (count == 0 || m0 >= count) {
        // every member is needed (or the class is absent from a fully sampled segment)
        if (threadIdx.x == 0) {
          a.tlo[p] = (count == 0 && !sparse) ? kNone : 0u;
          a.sb1[p] = kNone;
        }
      } else {
        if (mmax > count) mmax = count;
        uint32_t bin, binlo;
        int64_t above, above_lo;
        block_find_bin(h, kBins1, m0, &bin, &above);
        block_find_bin(h, kBins1, mmax, &binlo, &above_lo);
        if (threadIdx.x == 0) {
          a.sb1[p] = bin;
          a.sblo[p] = binlo;
          a.ssub[p] = 11u - ceil_log2(bin - binlo + 1u);
          a.srank[p] = m0;
          a.sabove[p] = above;
          a.smcap[p] = mmax;
        }
      }
    } else {
      int64_t m = a.srank[p];
      if (sparse) {
        // the deviation of the sampled count, from the spread of the per-run counts
        const double R = (double)kSampleRuns;
        const double mean = (double)((volatile unsigned long long*)a.svar)[2 * p] / R;
        const double sq = (double)((volatile unsigned long long*)a.svar)[2 * p + 1] / R;
        const double var = sq - mean * mean > 0.0 ? sq - mean * mean : 0.0;
        const double sd = sqrt(R * var) > sqrt(e) ? sqrt(R * var) : sqrt(e);
        const int64_t ma = (int64_t)ceil(e + 3.0 * sd + 16.0);
        const int64_t mcap = a.smcap[p];
        m = ma < m ? m : (ma > mcap ? mcap : ma);
      }
      uint32_t bin;
      int64_t above;
      block_find_bin(h, kBins1, m - a.sabove[p], &bin, &above);
      if (threadIdx.x == 0) a.tlo[p] = ((blo[c] << sub[c]) + bin) << (20 - sub[c]);
    }
    __syncthreads();
  }
}

// ------------------------------------------------------------------------------------------
// 3. pass 1: the streaming pass

// Candidate test of one accumulated value: its key reaches T_lo of its class. Binarise: the sign
// picks the class, and zeros and NaN belong to neither (same classes as class_of<2>).
template <int C>
__device__ __forceinline__ uint32_t cand_bit(float x, const uint32_t* tl) {
  const uint32_t u = __float_as_uint(x);
  const uint32_t key = u & 0x7fffffffu;
  if (C == 1) return key >= tl[0];
  const uint32_t t = (u >> 31) ? tl[1] : tl[0];
  return key >= t && key != 0u && key <= 0x7f800000u;
}

template <int C>
__device__ __forceinline__ int cand_class(float x) {
  return C == 1 ? 0 : (int)(__float_as_uint(x) >> 31);
}

// Per-warp state of pass 1 over one piece.
struct P1State {
  uint32_t count;   // candidates found so far
  uint32_t cp;      // next pending write of this piece
  // pending window of 64 writes (entries cp + lane and cp + 32 + lane), loaded one chunk ahead
  int32_t win_idx, win_idx2;
  float win_val, win_val2;
  // the store: positions below `room` have slots; the newest region (primary store or pool
  // chunk) starts at position ch_lo, slot ch_base; the one before it at pv_lo, pv_base
  uint32_t room, nch, ch_lo, pv_lo;
  int64_t ch_base, pv_base;
};

// Makes room for `need` more candidates (need <= 512 <= a chunk) by claiming one pool chunk.
// Warp-uniform; once a candidate has been dropped nothing more is claimed (the piece is re-read).
// A piece whose candidates so far are more than a quarter of the `seen` entries it has streamed
// (once it has streamed four chunks, so that one dense row at its start does not decide) claims
// none either: candidates that dense are cheaper to re-read from the residual in the later steps
// (4 bytes per entry) than to store here (8 bytes per candidate and a scattered write each), and
// refusing early leaves little to restore.
__device__ __forceinline__ void p1_reserve(const Sel& a, int64_t q, uint32_t need, uint32_t seen,
                                           P1State& S, int lane) {
  if (S.count + need <= S.room || S.count > S.room) return;
  uint32_t c = 0xFFFFFFFFu;
  if (lane == 0 && S.nch < (uint32_t)a.max_chunks &&
      (seen < 4u * (uint32_t)kGranule || 4ull * (S.count + need) <= (uint64_t)seen)) {
    c = atomicAdd(reinterpret_cast<uint32_t*>(a.ctl + 2), 1u);
    if (c >= (uint64_t)a.pool_chunks) c = 0xFFFFFFFFu;
    else a.pchunk[q * a.max_chunks + S.nch] = (int32_t)c;
  }
  c = __shfl_sync(kFull, c, 0);
  if (c == 0xFFFFFFFFu) return;
  S.pv_lo = S.ch_lo;
  S.pv_base = S.ch_base;
  S.ch_lo = S.room;
  S.ch_base = a.Q * a.cap + ((int64_t)c << a.chunk_shift);
  S.room += 1u << a.chunk_shift;
  S.nch += 1;
}

__device__ __forceinline__ void load_window(const Sel& a, uint32_t cp, uint32_t cend, int lane,
                                            P1State& S) {
  const uint32_t j = cp + lane;
  S.win_idx = j < cend ? a.pw_idx[j] : INT32_MAX;
  S.win_val = j < cend ? a.pw_val[j] : 0.0f;
  S.win_idx2 = j + 32 < cend ? a.pw_idx[j + 32] : INT32_MAX;
  S.win_val2 = j + 32 < cend ? a.pw_val[j + 32] : 0.0f;
}

// One chunk of 512 entries [base, base + 512) of the piece [lo, hi): pending writes, acc, the
// candidate test and ordered store, the histogram, and the residual write-back. gv/rv hold the
// chunk (entries outside the piece, as marked by `valid`, are ignored). Ring mode (full chunks
// only): the chunk is in shared memory instead, g in `gs_`, r in `st`; pending writes go straight
// into st and gv/rv are read from there.
template <int C, bool kRing = false>
__device__ __forceinline__ void pass1_chunk(const Sel& a, int64_t q, uint32_t base, uint32_t lo,
                                            uint32_t hi, bool full, uint32_t valid,
                                            float4 (&gv)[4], float4 (&rv)[4], P1State& S,
                                            uint32_t cend, const uint32_t (&tl)[C], float* st,
                                            uint32_t* hsink, int hstride, int lane,
                                            const float* gs_ = nullptr, const float* us_ = nullptr) {
  float4* st4 = reinterpret_cast<float4*>(st);
  float* r = a.r;
  if (kRing) {
    // pending writes that fall in this chunk replace those residual entries in the slot
    if (S.cp < cend) {
      const uint32_t lim = base + (uint32_t)kGranule;
      for (;;) {
        // the window's writes inside the chunk are a prefix of it (the list ascends)
        const bool in = S.win_idx >= (int32_t)base && S.win_idx < (int32_t)lim;
        const bool in2 = S.win_idx2 >= (int32_t)base && S.win_idx2 < (int32_t)lim;
        const uint32_t mask = __ballot_sync(kFull, in), mask2 = __ballot_sync(kFull, in2);
        if (!mask) break;
        if (in) st[S.win_idx - (int32_t)base] = S.win_val;
        if (in2) st[S.win_idx2 - (int32_t)base] = S.win_val2;
        S.cp += __popc(mask) + __popc(mask2);
        __syncwarp();
        load_window(a, S.cp, cend, lane, S);
        if (mask2 != kFull) break;
      }
    }
    const float4* g4 = reinterpret_cast<const float4*>(gs_);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      gv[u] = g4[u * 32 + lane];
      rv[u] = st4[u * 32 + lane];
    }
    if (us_) {
      // momentum correction: v = fl(fl(m u) + g) stands in for g and becomes the new momentum
      const float4* u4 = reinterpret_cast<const float4*>(us_);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        gv[u] = momentum4(a.mom, u4[u * 32 + lane], gv[u]);
        st_stream(a.u + base + u * 128 + lane * 4, gv[u]);
      }
    }
    __syncwarp();
  } else if (S.cp < cend) {
    // pending residual writes that fall in this chunk replace those residual entries
    const uint32_t lim = base + (uint32_t)kGranule < hi ? base + (uint32_t)kGranule : hi;
    bool staged = false;
    for (;;) {
      // the window's writes inside the chunk are a prefix of it (the list ascends)
      const bool in = S.win_idx >= (int32_t)base && S.win_idx < (int32_t)lim;
      const bool in2 = S.win_idx2 >= (int32_t)base && S.win_idx2 < (int32_t)lim;
      const uint32_t mask = __ballot_sync(kFull, in), mask2 = __ballot_sync(kFull, in2);
      if (!mask) break;
      if (!staged) {
#pragma unroll
        for (int u = 0; u < 4; ++u) st4[u * 32 + lane] = rv[u];
        __syncwarp();
        staged = true;
      }
      if (in) st[S.win_idx - (int32_t)base] = S.win_val;
      if (in2) st[S.win_idx2 - (int32_t)base] = S.win_val2;
      S.cp += __popc(mask) + __popc(mask2);
      __syncwarp();
      load_window(a, S.cp, cend, lane, S);   // the next window (for this chunk if it was full)
      if (mask2 != kFull) break;
    }
    if (staged) {
#pragma unroll
      for (int u = 0; u < 4; ++u) rv[u] = st4[u * 32 + lane];
      __syncwarp();
    }
  }
  float4 av[4];
  uint32_t m16 = 0;
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    av[u] = make_float4(__fadd_rn(gv[u].x, rv[u].x), __fadd_rn(gv[u].y, rv[u].y),
                        __fadd_rn(gv[u].z, rv[u].z), __fadd_rn(gv[u].w, rv[u].w));
    m16 |= (cand_bit<C>(av[u].x, tl) | (cand_bit<C>(av[u].y, tl) << 1) |
            (cand_bit<C>(av[u].z, tl) << 2) | (cand_bit<C>(av[u].w, tl) << 3)) << (4 * u);
  }
  m16 &= valid;
  // per-quarter counts packed in bytes; one warp scan serves all four quarters
  const uint32_t packed = __popc(m16 & 0xFu) | (__popc(m16 & 0xF0u) << 8) |
                          (__popc(m16 & 0xF00u) << 16) | (__popc(m16 & 0xF000u) << 24);
  const uint32_t incl = warp_inclusive_scan(packed);
  const uint32_t tot = __shfl_sync(kFull, incl, 31);
  bool from_stage = false;
  if (tot && S.count > S.room) {
    // the piece is past its store and will be re-read: only the histogram
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const float xs[4] = {av[u].x, av[u].y, av[u].z, av[u].w};
#pragma unroll
      for (int e = 0; e < 4; ++e)
        if ((m16 >> (4 * u + e)) & 1u)
          atomicAdd(hsink + cand_class<C>(xs[e]) * hstride + (mag_key(xs[e]) >> 20), 1u);
    }
    S.count += (tot & 0xFFu) + ((tot >> 8) & 0xFFu) + ((tot >> 16) & 0xFFu) + (tot >> 24);
  } else if (kRing && (tot & 0xFFu) + ((tot >> 8) & 0xFFu) + ((tot >> 16) & 0xFFu) + (tot >> 24) - 32u <
                         (uint32_t)kGranule / 2 - 31u) {
    // Ring chunk with 32 to 256 candidates: the slot's g half is free (every lane has read its
    // g), so each lane places its candidates there at their ranks, index and value side by side,
    // and the warp then stores them and counts their keys 32 at a time: the per-lane loop, whose
    // trip count is the busiest lane's, only writes shared memory. (Below one candidate per lane
    // the extra staging costs more than it saves: a 99.9% drop and small per-tensor steps were
    // slower with it; at a 90% drop pass 1 ran 5.42 vs 5.03 TB/s.)
#pragma unroll
    for (int u = 0; u < 4; ++u) st4[u * 32 + lane] = av[u];
    const uint32_t excl = incl - packed;
    const uint32_t t0 = tot & 0xFFu, t1 = (tot >> 8) & 0xFFu, t2 = (tot >> 16) & 0xFFu;
    const uint32_t total = t0 + t1 + t2 + (tot >> 24);
    p1_reserve(a, q, total, base + (uint32_t)kGranule - lo, S, lane);
    int32_t* ci_s = reinterpret_cast<int32_t*>(const_cast<float*>(gs_));
    float* cv_s = const_cast<float*>(gs_) + kGranule / 2;
    __syncwarp();
    uint32_t stored = 0;
    for (uint32_t m = m16; m; m &= m - 1) {
      const int b = __ffs(m) - 1;
      const int u = b >> 2, e = b & 3;
      const uint32_t before = (u >= 1 ? t0 : 0u) + (u >= 2 ? t1 : 0u) + (u >= 3 ? t2 : 0u);
      const uint32_t rank = before + ((excl >> (8 * u)) & 0xFFu) +
                            __popc(m16 & ((1u << b) - 1u) & (0xFu << (4 * u)));
      ci_s[rank] = (int32_t)(base + u * 128 + lane * 4 + e);
      cv_s[rank] = st[(u * 32 + lane) * 4 + e];
      stored |= (uint32_t)(S.count + rank < S.room) << b;
    }
    __syncwarp();
    for (uint32_t k = (uint32_t)lane; k < total; k += 32) {
      const uint32_t pos = S.count + k;
      const float x = cv_s[k];
      if (pos < S.room) {
        const int64_t slot = pos >= S.ch_lo ? S.ch_base + (pos - S.ch_lo) : S.pv_base + (pos - S.pv_lo);
        a.cidx[slot] = ci_s[k];
        a.cval[slot] = x;
      }
      atomicAdd(hsink + cand_class<C>(x) * hstride + (mag_key(x) >> 20), 1u);
    }
    S.count += total;
    if (a.zero_mode) {
      // stored candidates leave the residual as +0 (the not-sent ones get acc back later)
      for (uint32_t m = stored; m; m &= m - 1) {
        const int b = __ffs(m) - 1;
        st[((b >> 2) * 32 + lane) * 4 + (b & 3)] = 0.0f;
      }
      __syncwarp();
      from_stage = true;
    }
  } else if (tot) {
#pragma unroll
    for (int u = 0; u < 4; ++u) st4[u * 32 + lane] = av[u];
    __syncwarp();
    const uint32_t excl = incl - packed;
    const uint32_t t0 = tot & 0xFFu, t1 = (tot >> 8) & 0xFFu, t2 = (tot >> 16) & 0xFFu;
    p1_reserve(a, q, t0 + t1 + t2 + (tot >> 24), base + (uint32_t)kGranule - lo, S, lane);
    uint32_t stored = 0;
    for (uint32_t m = m16; m; m &= m - 1) {
      const int b = __ffs(m) - 1;
      const int u = b >> 2, e = b & 3;
      const uint32_t before = (u >= 1 ? t0 : 0u) + (u >= 2 ? t1 : 0u) + (u >= 3 ? t2 : 0u);
      const uint32_t pos = S.count + before + ((excl >> (8 * u)) & 0xFFu) +
                           __popc(m16 & ((1u << b) - 1u) & (0xFu << (4 * u)));
      const float x = st[(u * 32 + lane) * 4 + e];
      if (pos < S.room) {
        const int64_t slot = pos >= S.ch_lo ? S.ch_base + (pos - S.ch_lo) : S.pv_base + (pos - S.pv_lo);
        a.cidx[slot] = (int32_t)(base + u * 128 + lane * 4 + e);
        a.cval[slot] = x;
        stored |= 1u << b;
      }
      atomicAdd(hsink + cand_class<C>(x) * hstride + (mag_key(x) >> 20), 1u);
    }
    S.count += t0 + t1 + t2 + (tot >> 24);
    if (a.zero_mode) {
      // stored candidates leave the residual as +0 (the not-sent ones get acc back later)
      for (uint32_t m = stored; m; m &= m - 1) {
        const int b = __ffs(m) - 1;
        st[((b >> 2) * 32 + lane) * 4 + (b & 3)] = 0.0f;
      }
      __syncwarp();
      from_stage = true;
    }
  }
  if (full) {
#pragma unroll
    for (int u = 0; u < 4; ++u)
      st_stream(r + base + u * 128 + lane * 4, from_stage ? st4[u * 32 + lane] : av[u]);
  } else {
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const float4 o = from_stage ? st4[u * 32 + lane] : av[u];
      const float ov[4] = {o.x, o.y, o.z, o.w};
#pragma unroll
      for (int e = 0; e < 4; ++e)
        if ((valid >> (4 * u + e)) & 1u) r[base + u * 128 + lane * 4 + e] = ov[e];
    }
  }
  __syncwarp();
}

// First or last chunk of a piece: entry-wise bounds.
__device__ __forceinline__ uint32_t load_edge(const Sel& a, uint32_t base, uint32_t lo, uint32_t hi,
                                              int lane, float4 (&gv)[4], float4 (&rv)[4]) {
  uint32_t valid = 0;
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    float t0[4], t1[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const uint32_t i = base + u * 128 + lane * 4 + e;
      const bool in = i >= lo && i < hi;
      t0[e] = in ? a.g[i] : 0.0f;
      t1[e] = in ? a.r[i] : 0.0f;
      valid |= (uint32_t)in << (4 * u + e);
    }
    gv[u] = make_float4(t0[0], t0[1], t0[2], t0[3]);
    rv[u] = make_float4(t1[0], t1[1], t1[2], t1[3]);
  }
  return valid;
}

__device__ __forceinline__ void load_full(const Sel& a, uint32_t base, int lane, float4 (&gv)[4],
                                          float4 (&rv)[4]) {
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    gv[u] = ld_stream(a.g + base + u * 128 + lane * 4);
    rv[u] = ld_stream(a.r + base + u * 128 + lane * 4);
  }
}

// The streaming pass: one warp per piece. Interior chunks are software pipelined: the next
// chunk's g and r (and the next window of pending writes) are in flight while this one is
// processed.
template <int C>
__global__ void __launch_bounds__(kThreads, 2) pass1_kernel(Sel a) {
  pdl_begin();
  __shared__ CtaHist<C, kBins1> H;
  __shared__ __align__(16) float stage[kWarps * kGranule];  // per warp: one chunk, entry order
  if (a.ctl[0]) return;
  const int64_t q0 = (int64_t)blockIdx.x * kWarps;
  H.init(a, q0);
  __syncthreads();
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int64_t q = q0 + wid;
  if (q < total_pieces(a)) {
    const Piece P = piece_of(a, q);
    uint32_t tl[C];
#pragma unroll
    for (int c = 0; c < C; ++c) tl[c] = a.tlo[(int64_t)P.s * C + c];
    // histogram sink: this CTA's shared counts, or global counts for a second segment
    const bool sh_sink = P.s == H.primary;
    uint32_t* hsink = sh_sink ? H.sh : hist_of(a, (int64_t)P.s * C, 1);
    const int hstride = sh_sink ? kBins1 : kHist;
    const uint32_t lo = (uint32_t)P.lo, hi = (uint32_t)P.hi;  // indices are below 2^31
    float* st = stage + wid * kGranule;
    // pending residual writes of this piece start at the first index >= lo
    const uint32_t cend = pending_count(a);
    P1State S;
    S.count = 0;
    S.cp = 0;
    S.room = (uint32_t)a.cap;
    S.nch = 0;
    S.ch_lo = S.pv_lo = 0;
    S.ch_base = S.pv_base = q * a.cap;
    if (cend) S.cp = a.pstart[q];
    load_window(a, S.cp, cend, lane, S);
    uint32_t base = lo & ~3u;
    float4 gv[4], rv[4];
    if (base < lo || base + (uint32_t)kGranule > hi) {
      const uint32_t valid = load_edge(a, base, lo, hi, lane, gv, rv);
      pass1_chunk<C>(a, q, base, lo, hi, false, valid, gv, rv, S, cend, tl, st, hsink, hstride, lane);
      base += (uint32_t)kGranule;
    }
    if (base < hi && base + (uint32_t)kGranule <= hi) {
      float4 gn[4], rn[4];
      load_full(a, base, lane, gn, rn);
      for (;;) {
#pragma unroll
        for (int u = 0; u < 4; ++u) { gv[u] = gn[u]; rv[u] = rn[u]; }
        const uint32_t nb = base + (uint32_t)kGranule;
        const bool more = nb + (uint32_t)kGranule <= hi;
        if (more) load_full(a, nb, lane, gn, rn);
        pass1_chunk<C>(a, q, base, lo, hi, true, 0xFFFFu, gv, rv, S, cend, tl, st, hsink, hstride,
                       lane);
        base = nb;
        if (!more) break;
      }
    }
    if (base < hi) {
      const uint32_t valid = load_edge(a, base, lo, hi, lane, gv, rv);
      pass1_chunk<C>(a, q, base, lo, hi, false, valid, gv, rv, S, cend, tl, st, hsink, hstride, lane);
    }
    if (lane == 0) {
      a.pcnt[q] = S.count;
      a.pnch[q] = S.nch;
    }
  }
  __syncthreads();
  H.flush(a, 1, kBins1);
}

// ------------------------------------------------------------------------------------------
// 3b. pass 1 through a shared-memory ring (fp32 top-k, with or without momentum)
//
// The same pass, with the interior chunks of a piece brought into shared memory by bulk
// asynchronous copies (one lane issues 2 KB per stream and chunk, completion is counted on a
// per-slot mbarrier), kStages - 1 chunks ahead of the one being processed (two streams, g and r)
// or kStagesM - 1 ahead (three streams, g, u and r), so a warp keeps its loads outstanding
// without holding them in registers. The register pipeline above serves the sign-split
// binarisation (two classes per problem). Every wait is bounded (about a second of SM
// clock); a wait that gives up raises GSPARSE_DERR_TIMEOUT, stops the call and lets the warp's
// remaining copies land before it exits.

constexpr int kStages = 3;
constexpr uint32_t kPendChunks = 3;    // chunks of pending writes kept requested ahead in L2
constexpr uint32_t kChunkBytes = (uint32_t)kGranule * 4u;
constexpr long long kTestWaitCycles = 1ll << 16;   // the test hook's wait (about 33 us)

struct __align__(128) RingSlot {
  float g[kGranule];
  float r[kGranule];
};
// with momentum a slot also holds the chunk of u, and the ring is one stage shorter (same bytes)
struct __align__(128) RingSlotM {
  float g[kGranule];
  float r[kGranule];
  float u[kGranule];
};
constexpr int kStagesM = 2;
constexpr size_t kRingBytesM = sizeof(RingSlotM) * kStagesM * kWarps;

// Momentum correction of an edge chunk held in registers: gv <- v, and u <- v for the entries
// inside the piece.
__device__ __forceinline__ void momentum_edge(const Sel& a, uint32_t base, uint32_t valid, int lane,
                                              float4 (&gv)[4]) {
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    float gx[4] = {gv[u].x, gv[u].y, gv[u].z, gv[u].w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      if (!((valid >> (4 * u + e)) & 1u)) continue;
      const uint32_t i = base + u * 128 + lane * 4 + e;
      gx[e] = __fadd_rn(__fmul_rn(a.mom, a.u[i]), gx[e]);
      a.u[i] = gx[e];
    }
    gv[u] = make_float4(gx[0], gx[1], gx[2], gx[3]);
  }
}

template <int C, bool kMom>
__global__ void __launch_bounds__(kThreads, 2) pass1_ring_kernel(Sel a) {
  pdl_begin();
  using Slot = typename std::conditional<kMom, RingSlotM, RingSlot>::type;
  constexpr int kSt = kMom ? kStagesM : kStages;
  extern __shared__ __align__(128) unsigned char ring_mem[];
  __shared__ CtaHist<C, kBins1> H;
  // per warp: one barrier per ring slot, and one that nothing ever arrives at (the test hook's)
  __shared__ uint64_t bars[kWarps][kSt + 1];
  if (a.ctl[0]) return;
  const int64_t q0 = (int64_t)blockIdx.x * kWarps;
  H.init(a, q0);
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  if (lane == 0)
    for (int k = 0; k <= kSt; ++k) mbar_init(&bars[wid][k], 1);
  fence_mbarrier_init();
  __syncthreads();
  const int64_t q = q0 + wid;
  if (q < total_pieces(a)) {
    const Piece P = piece_of(a, q);
    uint32_t tl[C];
#pragma unroll
    for (int c = 0; c < C; ++c) tl[c] = a.tlo[(int64_t)P.s * C + c];
    const bool sh_sink = P.s == H.primary;
    uint32_t* hsink = sh_sink ? H.sh : hist_of(a, (int64_t)P.s * C, 1);
    const int hstride = sh_sink ? kBins1 : kHist;
    const uint32_t lo = (uint32_t)P.lo, hi = (uint32_t)P.hi;  // indices are below 2^31
    Slot* ring = reinterpret_cast<Slot*>(ring_mem) + wid * kSt;
    uint64_t* mb = bars[wid];
    const uint32_t cend = pending_count(a);
    P1State S;
    S.count = 0;
    S.cp = 0;
    S.room = (uint32_t)a.cap;
    S.nch = 0;
    S.ch_lo = S.pv_lo = 0;
    S.ch_base = S.pv_base = q * a.cap;
    if (cend) S.cp = a.pstart[q];
    load_window(a, S.cp, cend, lane, S);
    // pending writes up to entry pf have been requested into L2 (see the chunk loop), at most up
    // to pf_end (the piece's last write) and about kPendChunks chunks' worth ahead of the window
    uint32_t pf = S.cp, pf_end = S.cp, lead = 0;
    if (cend) {
      pf_end = a.pstart[q + 1];
      const uint64_t per = (uint64_t)(pf_end - S.cp) * (kPendChunks * (uint64_t)kGranule) / (hi > lo ? hi - lo : 1u);
      lead = (uint32_t)(per + 32u < 512u ? per + 32u : 512u);
    }
    uint32_t base = lo & ~3u;
    float4 gv[4], rv[4];
    if (base < lo || base + (uint32_t)kGranule > hi) {
      const uint32_t valid = load_edge(a, base, lo, hi, lane, gv, rv);
      if (kMom) momentum_edge(a, base, valid, lane, gv);
      pass1_chunk<C>(a, q, base, lo, hi, false, valid, gv, rv, S, cend, tl, ring[0].r, hsink, hstride, lane);
      base += (uint32_t)kGranule;
    }
    // interior chunks [base, base + nint * 512) through the ring (base is 16-byte aligned)
    const uint32_t nint = base < hi ? (hi - base) / (uint32_t)kGranule : 0u;
    auto issue = [&](uint32_t c) {
      Slot& sl = ring[c % kSt];
      uint64_t* bar = &mb[c % kSt];
      const size_t off = (size_t)base + (size_t)c * kGranule;
      mbar_arrive_expect_tx(bar, (kMom ? 3u : 2u) * kChunkBytes);
      bulk_load(sl.g, a.g + off, kChunkBytes, bar);
      bulk_load(sl.r, a.r + off, kChunkBytes, bar);
      if constexpr (kMom) bulk_load(sl.u, a.u + off, kChunkBytes, bar);
    };
    if (lane == 0)
      for (uint32_t c = 0; c + 1 < (uint32_t)kSt && c < nint; ++c) issue(c);
    uint32_t parity = 0;   // bit k: the phase parity slot k waits for next
    uint32_t issued = nint < (uint32_t)kSt - 1 ? nint : (uint32_t)kSt - 1;
    bool failed = false;
    uint32_t c_fail = 0;
    for (uint32_t c = 0; c < nint; ++c) {
      const uint32_t k = c % kSt;
      if (issued < nint) {
        // the slot of chunk c - 1 is free: order this warp's accesses to it before the copy
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) issue(issued);
        ++issued;
      }
      // test hook: the first wait is on the extra barrier, which never completes, with a short limit
      const bool ok = (a.wait_test && c == 0) ? mbar_wait_bounded(&mb[kSt], 0u, kTestWaitCycles)
                                              : mbar_wait_bounded(&mb[k], (parity >> k) & 1u);
      if (!ok) {
        failed = true;
        c_fail = c;
        break;
      }
      parity ^= 1u << k;
      // Keep the pending writes of the next few chunks requested into L2: a window load that
      // missed would queue behind the ring's copies in flight (several microseconds), while the
      // line is needed one chunk later; a longer lead loses the lines to the stream before use.
      // Lanes 0-15 take index lines, 16-31 value lines, one 32-entry line each, only lines not
      // requested before.
      if (pf < pf_end) {
        const uint32_t want = S.cp + lead < pf_end ? S.cp + lead : pf_end;
        if (pf < want) {
          const uint32_t j = pf + 32u * (uint32_t)(lane & 15);
          if (j < want) prefetch_l2(lane < 16 ? (const void*)(a.pw_idx + j) : (const void*)(a.pw_val + j));
          pf = pf + 512u < want ? pf + 512u : want;
        }
      }
      const float* us_ = nullptr;
      if constexpr (kMom) us_ = ring[k].u;
      pass1_chunk<C, true>(a, q, base + c * (uint32_t)kGranule, lo, hi, true, 0xFFFFu, gv, rv, S, cend,
                           tl, ring[k].r, hsink, hstride, lane, ring[k].g, us_);
    }
    if (failed) {
      if (lane == 0) {
        raise(a.d_status, GSPARSE_DERR_TIMEOUT);
        a.ctl[0] = 1;
      }
      // let the copies still in flight land before the warp leaves (bounded as well): chunks
      // c_fail .. issued - 1, at most one per slot, each still waiting for its slot's next phase
      for (uint32_t c = c_fail; c < issued; ++c) {
        const uint32_t k = c % kSt;
        mbar_wait_bounded(&mb[k], (parity >> k) & 1u);
      }
    } else {
      base += nint * (uint32_t)kGranule;
      if (base < hi) {
        const uint32_t valid = load_edge(a, base, lo, hi, lane, gv, rv);
        if (kMom) momentum_edge(a, base, valid, lane, gv);
        pass1_chunk<C>(a, q, base, lo, hi, false, valid, gv, rv, S, cend, tl, ring[0].r, hsink, hstride, lane);
      }
    }
    if (lane == 0) {
      a.pcnt[q] = S.count;
      a.pnch[q] = S.nch;
    }
  }
  __syncthreads();
  H.flush(a, 1, kBins1);
}

// The pending residual writes must be strictly ascending indices in [0, n): anything else stops
// the call before it touches the residual. The same pass records pstart: the pieces whose first
// entry lies in (idx[j-1], idx[j]] start their writes at j. A thread takes kCheckPer consecutive
// writes and keeps the first entry of the next piece, so it locates a piece only when a write
// crosses a piece start.
constexpr int kCheckPer = 16;

__global__ void __launch_bounds__(256) pending_check_kernel(Sel a) {
  pdl_begin();
  const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (t == 0 && *a.pw_count > a.pw_cap) {
    raise(a.d_status, GSPARSE_DERR_CAPACITY);
    a.ctl[0] = 1;
  }
  const uint32_t c = pending_count(a);
  const int64_t Qn = total_pieces(a);
  const int64_t j0 = t * kCheckPer;
  bool bad = false;
  if (j0 <= c) {
    const int32_t* x = a.pw_idx;
    int32_t v[kCheckPer];
    if (j0 + kCheckPer <= c && (reinterpret_cast<uintptr_t>(x + j0) & 15u) == 0) {
#pragma unroll
      for (int h = 0; h < kCheckPer / 4; ++h) {
        const int4 w = *reinterpret_cast<const int4*>(x + j0 + 4 * h);
        v[4 * h] = w.x; v[4 * h + 1] = w.y; v[4 * h + 2] = w.z; v[4 * h + 3] = w.w;
      }
    } else {
#pragma unroll
      for (int e = 0; e < kCheckPer; ++e) v[e] = j0 + e < c ? x[j0 + e] : 0;
    }
    const int64_t ip0 = j0 > 0 ? x[j0 - 1] : -1;
    auto clampi = [&](int64_t i) { return i < 0 ? (int64_t)0 : (i < a.n ? i : a.n - 1); };
    // the last piece already started before this thread's first write, and the next piece's start
    int64_t q_prev = (ip0 < 0 || Qn == 0) ? -1 : piece_containing(a, clampi(ip0));
    int64_t next_lo = q_prev + 1 < Qn ? piece_of(a, q_prev + 1).lo : INT64_MAX;
    // fast scan: validity, and a mark on every write at or beyond the next piece's start
    uint32_t mark = 0;
    if (j0 + kCheckPer <= c) {
      // a full run: 32-bit tests (indices are int32; n <= 2^31 - 1, so an unsigned compare with n
      // also catches negative indices)
      const uint32_t un = (uint32_t)a.n;
      const uint32_t nl = next_lo <= (int64_t)UINT32_MAX ? (uint32_t)next_lo : UINT32_MAX;
      int32_t ip = (int32_t)ip0;
#pragma unroll
      for (int e = 0; e < kCheckPer; ++e) {
        bad |= (uint32_t)v[e] >= un || ((j0 + e) > 0 && ip >= v[e]);
        mark |= (uint32_t)((uint32_t)v[e] >= nl && (uint32_t)v[e] < un) << e;
        ip = v[e];
      }
      // every write at or beyond the next start is marked; out-of-range ones raise anyway
    } else {
      int64_t ip = ip0;
#pragma unroll
      for (int e = 0; e < kCheckPer; ++e) {
        const int64_t j = j0 + e;
        const int64_t i = v[e];
        if (j < c) bad |= i < 0 || i >= a.n || (j > 0 && ip >= i);
        mark |= (uint32_t)(j <= c && (j == c || i >= next_lo)) << e;
        ip = i;
      }
    }
    // the marked writes, in order (rolled loop)
    while (mark && Qn > 0) {
      const int e = __ffs(mark) - 1;
      mark &= mark - 1;
      const int64_t j = j0 + e;
      const int64_t i = j < c ? (int64_t)x[j] : a.n;
      if (j < c && i < next_lo) continue;
      const int64_t q_cur = j < c ? piece_containing(a, clampi(i)) : Qn;
      for (int64_t q = q_prev + 1; q <= q_cur; ++q) a.pstart[q] = (uint32_t)j;
      if (q_cur > q_prev) q_prev = q_cur;
      next_lo = q_prev + 1 < Qn ? piece_of(a, q_prev + 1).lo : INT64_MAX;
    }
  }
  if (__any_sync(kFull, bad) && (threadIdx.x & 31) == 0) {
    raise(a.d_status, GSPARSE_DERR_INDEX_RANGE);
    a.ctl[0] = 1;
  }
}

// ------------------------------------------------------------------------------------------
// candidate iteration for the later steps (order not needed)

// Calls f(x, c, key) for every candidate value of piece q in [b, e): store positions (values
// only; four float4 loads per lane in flight), or, for pieces marked to be re-read, entries of
// the residual (which then holds acc) filtered by class and T_lo. b is a multiple of 4 for the
// store.
template <int C, class F>
__device__ __forceinline__ void for_each_candidate(const Sel& a, int64_t q, const Piece& P,
                                                   int64_t b, int64_t e, F f) {
  const int lane = threadIdx.x & 31;
  if (!a.prsrc[q]) {
    // every store region starts 16-byte aligned (cap and the chunk size are multiples of 4)
    const uint32_t cnt = (uint32_t)e;
    const uint32_t n4 = (cnt + 3) / 4;
    for (uint32_t j4 = (uint32_t)b / 4 + lane; j4 < n4; j4 += 128) {
      float4 X[4];
#pragma unroll
      for (int h = 0; h < 4; ++h)
        X[h] = j4 + 32 * h < n4 ? *reinterpret_cast<const float4*>(a.cval + slot_of(a, q, 4 * (j4 + 32 * h)))
                                : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        const float xv[4] = {X[h].x, X[h].y, X[h].z, X[h].w};
#pragma unroll
        for (int e4 = 0; e4 < 4; ++e4) {
          const uint32_t j = 4 * (j4 + 32 * h) + e4;
          if (j < cnt) {
            const int c = class_of<C>(xv[e4]);
            f(xv[e4], c < 0 ? 0 : c, mag_key(xv[e4]));
          }
        }
      }
    }
    return;
  }
  uint32_t tl[C];
#pragma unroll
  for (int c = 0; c < C; ++c) tl[c] = a.tlo[(int64_t)P.s * C + c];
  for (int64_t base = b & ~(int64_t)3; base < e; base += 128) {
    const int64_t v = base + lane * 4;
    float x[4] = {0.f, 0.f, 0.f, 0.f};
    if (v >= b && v + 4 <= e) {
      const float4 t = *reinterpret_cast<const float4*>(a.r + v);
      x[0] = t.x; x[1] = t.y; x[2] = t.z; x[3] = t.w;
    } else {
#pragma unroll
      for (int e4 = 0; e4 < 4; ++e4)
        if (v + e4 >= b && v + e4 < e) x[e4] = a.r[v + e4];
    }
#pragma unroll
    for (int e4 = 0; e4 < 4; ++e4) {
      const int64_t i = v + e4;
      if (i < b || i >= e) continue;
      const int c = class_of<C>(x[e4]);
      if (c < 0) continue;
      const uint32_t key = mag_key(x[e4]);
      if (key >= tl[c]) f(x[e4], c, key);
    }
  }
}

// ------------------------------------------------------------------------------------------
// 4. check + restore

__global__ void check_kernel(Sel a) {
  pdl_begin();
  __shared__ int64_t sh[33];
  if (a.ctl[0]) return;
  const int64_t p = blockIdx.x;
  const int32_t s = (int32_t)(p / a.C);
  uint32_t* h = hist_of(a, p, 1);
  int64_t mine = 0;
  for (int i = threadIdx.x; i < kBins1; i += blockDim.x) mine += h[i];
  int64_t total;
  block_exclusive_scan(mine, sh, &total);
  const uint32_t t = a.tlo[p];
  if (t != kNone && t != 0 && total < a.seg_k[s]) {
    for (int i = threadIdx.x; i < kBins1; i += blockDim.x) h[i] = 0;
    if (threadIdx.x == 0) {
      a.redo[p] = 1;
      a.tlo[p] = 0;
      a.ctl[1] = 1;
    }
  }
}

template <int C>
__global__ void __launch_bounds__(kThreads) restore_kernel(Sel a) {
  pdl_begin();
  __shared__ CtaHist<C, kBins1> H;
  if (a.ctl[0]) return;
  const int64_t q0 = (int64_t)blockIdx.x * kWarps;
  H.init(a, q0);
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int64_t q = q0 + (threadIdx.x >> 5);
  if (q < total_pieces(a)) {
    const Piece P = piece_of(a, q);
    bool redo = false;
#pragma unroll
    for (int c = 0; c < C; ++c) redo |= a.redo[(int64_t)P.s * C + c] != 0;
    const uint32_t cnt = a.pcnt[q];
    const uint32_t room = room_of(a, q);
    if (redo || cnt > room) {
      if (a.zero_mode) {
        // the stored candidates get their acc back, eight per lane with their loads in flight
        const uint32_t stored = cnt < room ? cnt : room;
        constexpr int kB = 8;
        for (uint32_t j0 = lane; j0 < stored; j0 += 32 * kB) {
          int32_t ix[kB];
          float xv[kB];
#pragma unroll
          for (int k = 0; k < kB; ++k) {
            const uint32_t j = j0 + 32u * k;
            const int64_t sl = j < stored ? slot_of(a, q, j) : 0;
            ix[k] = j < stored ? a.cidx[sl] : -1;
            xv[k] = j < stored ? a.cval[sl] : 0.0f;
          }
#pragma unroll
          for (int k = 0; k < kB; ++k)
            if (ix[k] >= 0) a.r[ix[k]] = xv[k];
        }
      }
      __syncwarp();
      if (lane == 0) a.prsrc[q] = 1;
      __syncwarp();
      if (redo) {
        // the redone classes count every member (their T_lo is now 0)
        for_each_candidate<C>(a, q, P, P.lo, P.hi, [&](float, int c, uint32_t key) {
          if (a.redo[(int64_t)P.s * C + c]) H.add(a, P.s, c, key >> 20, 1);
        });
      }
    }
  }
  __syncthreads();
  // only redone problems received counts here
  H.flush(a, 1, kBins1);
}

// ------------------------------------------------------------------------------------------
// 5-7. radix-select levels

// Numbers the work units of every piece (pieces and their stores are final after restore):
// uoff and the unit -> piece table. One CTA; thread t owns a contiguous run of pieces.
__device__ void number_units(const Sel& a, int64_t* sh) {
  const int64_t Qn = total_pieces(a);
  const int64_t per = cdiv(Qn, (int64_t)blockDim.x);
  const int64_t q_lo = threadIdx.x * per < Qn ? threadIdx.x * per : Qn;
  const int64_t q_hi = q_lo + per < Qn ? q_lo + per : Qn;
  // the run is taken eight pieces at a time, so their loads are in flight together
  constexpr int kB = 8;
  int64_t mine = 0;
  for (int64_t q = q_lo; q < q_hi; q += kB) {
    int64_t nu[kB];
#pragma unroll
    for (int k = 0; k < kB; ++k) nu[k] = q + k < q_hi ? units_of_piece(a, q + k) : 0;
#pragma unroll
    for (int k = 0; k < kB; ++k) mine += nu[k];
  }
  int64_t total;
  int64_t run = block_exclusive_scan(mine, sh, &total);
  for (int64_t q = q_lo; q < q_hi; q += kB) {
    int64_t nu[kB];
#pragma unroll
    for (int k = 0; k < kB; ++k) nu[k] = q + k < q_hi ? units_of_piece(a, q + k) : 0;
#pragma unroll
    for (int k = 0; k < kB; ++k) {
      if (q + k >= q_hi) break;
      a.uoff[q + k] = run;
      for (int64_t j = 0; j < nu[k]; ++j) a.upiece[run + j] = (int32_t)(q + k);
      run += nu[k];
    }
  }
  if (threadIdx.x == 0) a.uoff[Qn] = total;
}

// One radix-select level of problem p by the whole CTA (any block size): the bin holding the
// remaining rank, narrowing the prefix (levels 1-2) or fixing the threshold (level 3). h: the
// CTA's shared scratch of kBins1 counts. The histogram is read through L2 (written by atomics of
// other CTAs of the same or the previous kernel).
__device__ void select_problem(const Sel& a, int64_t p, int level, uint32_t* h, int64_t* sh) {
  const int32_t s = (int32_t)(p / a.C);
  if (level > 1 && a.pfx[p] == kNone) return;   // CTA-uniform
  const int B = level == 3 ? kBins3 : kBins1;
  const uint32_t* src = hist_of(a, p, level);
  int64_t mine = 0;
  for (int i = threadIdx.x; i < B; i += blockDim.x) {
    h[i] = __ldcg(src + i);
    mine += h[i];
  }
  int64_t total;
  block_exclusive_scan(mine, sh, &total);
  int64_t rank;
  if (level == 1) {
    const int64_t k = a.seg_k[s] < total ? a.seg_k[s] : total;
    if (threadIdx.x == 0) a.keff[p] = k;
    if (k == 0) {
      if (threadIdx.x == 0) {
        a.pfx[p] = kNone;
        a.thr[p] = kNone;
        a.need_eq[p] = 0;
      }
      __syncthreads();
      return;
    }
    rank = k;
  } else {
    rank = a.krem[p];
  }
  uint32_t bin;
  int64_t above;
  block_find_bin(h, B, rank, &bin, &above);
  if (threadIdx.x == 0) {
    if (level == 1) {
      a.pfx[p] = bin;
      a.krem[p] = rank - above;
    } else if (level == 2) {
      a.pfx[p] = (a.pfx[p] << 11) | bin;
      a.krem[p] = rank - above;
    } else {
      a.thr[p] = (a.pfx[p] << 9) | bin;
      a.need_eq[p] = rank - above;
    }
  }
  __syncthreads();
}

__global__ void __launch_bounds__(1024) select_kernel(Sel a, int level) {
  pdl_begin();
  __shared__ uint32_t h[kBins1];
  __shared__ int64_t sh[33];
  if (a.ctl[0]) return;
  if (level == 1 && blockIdx.x == 0) number_units(a, sh);
  select_problem(a, blockIdx.x, level, h, sh);
}


template <int C>
__global__ void __launch_bounds__(kThreads) hist_kernel(Sel a, int level) {
  pdl_begin();
  constexpr int B = kBins1;  // level 3 uses the first 512 bins
  __shared__ CtaHist<C, B> H;
  if (a.ctl[0]) return;
  const int64_t U = unit_count(a);
  const int64_t u0 = (int64_t)blockIdx.x * kWarps;
  H.init_seg(u0 < U ? piece_of(a, unit_piece(a, u0)).s : -1);
  __syncthreads();
  for (int64_t u = u0 + (threadIdx.x >> 5); u < U; u += (int64_t)gridDim.x * kWarps) {
    const int64_t q = unit_piece(a, u);
    const Piece P = piece_of(a, q);
    int64_t b, e;
    unit_range(a, q, P, u - a.uoff[q], &b, &e);
    uint32_t pf[C];
#pragma unroll
    for (int c = 0; c < C; ++c) pf[c] = a.pfx[(int64_t)P.s * C + c];
    for_each_candidate<C>(a, q, P, b, e, [&](float, int c, uint32_t key) {
      if (level == 2) {
        if ((key >> 20) == pf[c]) H.add(a, P.s, c, (key >> 9) & 2047u, 2);
      } else {
        if ((key >> 9) == pf[c]) H.add(a, P.s, c, key & 511u, 3);
      }
    });
  }
  __syncthreads();
  H.flush(a, level, level == 2 ? kBins2 : kBins3);
}

// ------------------------------------------------------------------------------------------
// 8. count + scan

template <int C>
__global__ void __launch_bounds__(kThreads) count_kernel(Sel a) {
  pdl_begin();
  if (a.ctl[0]) return;
  const int64_t U = unit_count(a);
  for (int64_t u = (int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5); u < U;
       u += (int64_t)gridDim.x * kWarps) {
    const int64_t q = unit_piece(a, u);
    const Piece P = piece_of(a, q);
    int64_t b, e;
    unit_range(a, q, P, u - a.uoff[q], &b, &e);
    uint32_t th[C], gt[C], eq[C];
#pragma unroll
    for (int c = 0; c < C; ++c) {
      th[c] = a.thr[(int64_t)P.s * C + c];
      gt[c] = 0;
      eq[c] = 0;
    }
    for_each_candidate<C>(a, q, P, b, e, [&](float, int c, uint32_t key) {
#pragma unroll
      for (int cc = 0; cc < C; ++cc) {
        if (cc == c) {
          gt[cc] += key > th[cc] && th[cc] != kNone;
          eq[cc] += key == th[cc];
        }
      }
    });
#pragma unroll
    for (int c = 0; c < C; ++c) {
      const uint32_t G = warp_sum(gt[c]), E = warp_sum(eq[c]);
      if ((threadIdx.x & 31) == 0) {
        a.pgt[u * C + c] = G;
        a.peq[u * C + c] = E;
      }
    }
  }
}

// Offsets of every work unit's selected entries within problem p's output, and how many keys
// equal to the threshold it takes (the first need_eq of them in unit order), by the whole CTA.
// The per-unit counts are read through L2.
__device__ void scan_problem(const Sel& a, int64_t p, int64_t* sh) {
  const int32_t s = (int32_t)(p / a.C);
  const int c = (int)(p % a.C);
  // the work units of segment s, in index order; thread t owns a contiguous run of them
  const int64_t first = a.uoff[a.seg_pbase[s]], last = a.uoff[a.seg_pbase[s + 1]];
  const int64_t need = a.need_eq[p];
  const int64_t per = cdiv(last - first, (int64_t)blockDim.x);
  const int64_t u_lo = first + threadIdx.x * per < last ? first + threadIdx.x * per : last;
  const int64_t u_hi = u_lo + per < last ? u_lo + per : last;
  // each loop takes the run eight units at a time, so their loads are in flight together
  constexpr int kB = 8;
  int64_t eq_mine = 0;
  for (int64_t u = u_lo; u < u_hi; u += kB) {
    uint32_t eq[kB];
#pragma unroll
    for (int k = 0; k < kB; ++k) eq[k] = u + k < u_hi ? __ldcg(a.peq + (u + k) * a.C + c) : 0u;
#pragma unroll
    for (int k = 0; k < kB; ++k) eq_mine += eq[k];
  }
  int64_t teq;
  int64_t eq_before = block_exclusive_scan(eq_mine, sh, &teq);
  // keys equal to the threshold: the first `need` of them in unit order are taken
  int64_t sel_mine = 0;
  for (int64_t u = u_lo; u < u_hi; u += kB) {
    uint32_t eq[kB], gt[kB];
#pragma unroll
    for (int k = 0; k < kB; ++k) {
      eq[k] = u + k < u_hi ? __ldcg(a.peq + (u + k) * a.C + c) : 0u;
      gt[k] = u + k < u_hi ? __ldcg(a.pgt + (u + k) * a.C + c) : 0u;
    }
#pragma unroll
    for (int k = 0; k < kB; ++k) {
      int64_t take = need - eq_before;
      take = take < 0 ? 0 : (take > (int64_t)eq[k] ? (int64_t)eq[k] : take);
      sel_mine += gt[k] + take;
      eq_before += eq[k];
    }
  }
  int64_t tsel;
  int64_t sel_before = block_exclusive_scan(sel_mine, sh, &tsel);
  eq_before -= eq_mine;
  for (int64_t u = u_lo; u < u_hi; u += kB) {
    uint32_t eq[kB], gt[kB];
#pragma unroll
    for (int k = 0; k < kB; ++k) {
      eq[k] = u + k < u_hi ? __ldcg(a.peq + (u + k) * a.C + c) : 0u;
      gt[k] = u + k < u_hi ? __ldcg(a.pgt + (u + k) * a.C + c) : 0u;
    }
#pragma unroll
    for (int k = 0; k < kB; ++k) {
      if (u + k >= u_hi) break;
      int64_t take = need - eq_before;
      take = take < 0 ? 0 : (take > (int64_t)eq[k] ? (int64_t)eq[k] : take);
      a.poff[(u + k) * a.C + c] = sel_before;
      a.ptake[(u + k) * a.C + c] = (uint32_t)take;
      sel_before += gt[k] + take;
      eq_before += eq[k];
    }
  }
}

__global__ void __launch_bounds__(1024) scan_kernel(Sel a) {
  pdl_begin();
  __shared__ int64_t sh[33];
  if (a.ctl[0]) return;
  scan_problem(a, blockIdx.x, sh);
}

// ------------------------------------------------------------------------------------------
// 9. emit, in index order

// A warp's staging rows for the ordered output: the selected entries of 128 candidates, compacted.
struct EmitStage {
  int32_t idx[128];
  float val[128];
};

template <int C>
__device__ __forceinline__ void emit_unit(const Sel& a, int64_t u, int32_t* out_idx, float* out_val,
                                          int64_t limit, EmitStage& stg);

template <int C>
__global__ void __launch_bounds__(kThreads, 4) emit_kernel(Sel a, int32_t* out_idx, float* out_val,
                                                        int64_t limit) {
  pdl_begin();
  __shared__ EmitStage stage[kWarps];
  if (a.ctl[0]) return;
  const int64_t U = unit_count(a);
  for (int64_t u = (int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5); u < U;
       u += (int64_t)gridDim.x * kWarps)
    emit_unit<C>(a, u, out_idx, out_val, limit, stage[threadIdx.x >> 5]);
}

template <int C>
__device__ __forceinline__ void emit_unit(const Sel& a, int64_t u, int32_t* out_idx, float* out_val,
                                          int64_t limit, EmitStage& stg) {
  const int lane = threadIdx.x & 31;
  const uint32_t lt = lanemask_lt();
  const int64_t q = unit_piece(a, u);
  const Piece P = piece_of(a, q);
  int64_t ub, ue;
  unit_range(a, q, P, u - a.uoff[q], &ub, &ue);
  uint32_t th[C], take[C], eq_run[C], sel_run[C];
  int64_t base_out[C];
#pragma unroll
  for (int c = 0; c < C; ++c) {
    const int64_t p = (int64_t)P.s * C + c;
    th[c] = a.thr[p];
    take[c] = a.ptake[u * C + c];
    eq_run[c] = 0;
    sel_run[c] = 0;
    // top-k: the segment's block of the output; binarise: the class list of the problem
    base_out[c] = (C == 1 ? a.seg_kbase[P.s] : 2 * a.seg_kbase[P.s] + c * a.seg_k[P.s]) + a.poff[u * C + c];
  }
  auto is_sel = [&](int c, uint32_t key, bool eq_taken) {
    return c >= 0 && th[c] != kNone && (key > th[c] || eq_taken);
  };
  if (!a.prsrc[q]) {
    // the unit's store positions [ub, ue) in index order, four consecutive candidates per lane
    const uint32_t cnt = (uint32_t)ue, jbeg = (uint32_t)ub;
    auto ci = [&](uint32_t pos) { return *reinterpret_cast<const int4*>(a.cidx + slot_of(a, q, pos)); };
    auto cv = [&](uint32_t pos) { return *reinterpret_cast<const float4*>(a.cval + slot_of(a, q, pos)); };
    // software pipelined: three batches of 128 candidates are in flight while one is placed
    constexpr int kAhead = 3;
    int4 Iq[kAhead];
    float4 Xq[kAhead];
#pragma unroll
    for (int h = 0; h < kAhead; ++h) {
      const uint32_t jj = jbeg + 128 * h + 4 * lane;
      Iq[h] = jj < cnt ? ci(jj) : make_int4(0, 0, 0, 0);
      Xq[h] = jj < cnt ? cv(jj) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    for (uint32_t j0 = jbeg; j0 < cnt; j0 += 128) {
      const uint32_t j = j0 + 4 * lane;
      const int4 I = Iq[0];
      const float4 X = Xq[0];
#pragma unroll
      for (int h = 0; h + 1 < kAhead; ++h) { Iq[h] = Iq[h + 1]; Xq[h] = Xq[h + 1]; }
      {
        const uint32_t jj = j + 128 * kAhead;
        Iq[kAhead - 1] = jj < cnt ? ci(jj) : make_int4(0, 0, 0, 0);
        Xq[kAhead - 1] = jj < cnt ? cv(jj) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
      int32_t iv[4] = {0, 0, 0, 0};
      float xv[4] = {0.f, 0.f, 0.f, 0.f};
      if (j < cnt) {
        iv[0] = I.x; iv[1] = I.y; iv[2] = I.z; iv[3] = I.w;
        xv[0] = X.x; xv[1] = X.y; xv[2] = X.z; xv[3] = X.w;
      }
      int cls[4];
      uint32_t key[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        cls[e] = j + e < cnt ? class_of<C>(xv[e]) : -1;
        key[e] = mag_key(xv[e]);
      }
      uint32_t selm = 0;
#pragma unroll
      for (int cc = 0; cc < C; ++cc) {
        uint32_t eqm = 0, gtm = 0;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          eqm |= (uint32_t)(cls[e] == cc && key[e] == th[cc]) << e;
          gtm |= (uint32_t)(cls[e] == cc && th[cc] != kNone && key[e] > th[cc]) << e;
        }
        uint32_t sm = gtm;
        if (__any_sync(kFull, eqm)) {
          // keys equal to the threshold: the first `take` of them in index order are sent
          uint32_t teq;
          const uint32_t pre_eq = warp_prefix_small(__popc(eqm), &teq);
#pragma unroll
          for (int e = 0; e < 4; ++e)
            if (((eqm >> e) & 1u) && (eq_run[cc] + pre_eq + __popc(eqm & ((1u << e) - 1u))) < take[cc])
              sm |= 1u << e;
          eq_run[cc] += teq;
        }
        uint32_t tsel;
        const uint32_t pre_sel = warp_prefix_small(__popc(sm), &tsel);
        if (tsel) {
          // the selected entries of these 128 candidates, compacted in index order, leave as one
          // contiguous run of output positions (coalesced rows)
          uint32_t k = pre_sel;
#pragma unroll
          for (int e = 0; e < 4; ++e)
            if ((sm >> e) & 1u) { stg.idx[k] = iv[e]; stg.val[k] = xv[e]; ++k; }
          __syncwarp();
          const int64_t o0 = base_out[cc] + sel_run[cc];
          int32_t* oi = (C == 1 ? out_idx : a.lidx) + o0;
          float* ov = (C == 1 ? out_val : a.lval) + o0;
          // positions past the output's capacity are dropped (and reported)
          const int64_t room = limit - o0;
          const uint32_t nfit = room <= 0 ? 0u : (room < (int64_t)tsel ? (uint32_t)room : tsel);
          if (nfit < tsel && lane == 0) raise(a.d_status, GSPARSE_DERR_CAPACITY);
          for (uint32_t t = (uint32_t)lane; t < nfit; t += 32) {
            const int32_t i = stg.idx[t];
            oi[t] = i;
            ov[t] = stg.val[t];
            if (C == 1 && a.u) a.u[i] = 0.0f;  // momentum masking of the sent entry
          }
          __syncwarp();
        }
        sel_run[cc] += tsel;
        selm |= sm;
      }
      if (a.zero_mode) {
        // a candidate that is not sent keeps its acc in the residual
#pragma unroll
        for (int e = 0; e < 4; ++e)
          if (j + e < cnt && !((selm >> e) & 1u)) a.r[iv[e]] = xv[e];
      }
    }
    return;
  }
  // re-read piece: the residual holds acc; walk the unit's entries [ub, ue) in index order
  for (int64_t vb = ub & ~(int64_t)3; vb < ue; vb += 128) {
    const int64_t v = vb + lane * 4;
    float x[4] = {0.f, 0.f, 0.f, 0.f};
    if (v >= ub && v + 4 <= ue) {
      const float4 t = *reinterpret_cast<const float4*>(a.r + v);
      x[0] = t.x; x[1] = t.y; x[2] = t.z; x[3] = t.w;
    } else {
#pragma unroll
      for (int e = 0; e < 4; ++e)
        if (v + e >= ub && v + e < ue) x[e] = a.r[v + e];
    }
    int cls[4];
    uint32_t key[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const bool in = v + e >= ub && v + e < ue;
      cls[e] = in ? class_of<C>(x[e]) : -1;
      key[e] = mag_key(x[e]);
    }
    uint32_t selm = 0;
#pragma unroll
    for (int cc = 0; cc < C; ++cc) {
      uint32_t eqm = 0;
#pragma unroll
      for (int e = 0; e < 4; ++e) eqm |= (uint32_t)(cls[e] == cc && key[e] == th[cc]) << e;
      uint32_t teq;
      const uint32_t pre_eq = warp_prefix_small(__popc(eqm), &teq);
      uint32_t sm = 0;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const bool eq = (eqm >> e) & 1u;
        const bool taken = eq && (eq_run[cc] + pre_eq + __popc(eqm & ((1u << e) - 1u))) < take[cc];
        sm |= (uint32_t)(cls[e] == cc && is_sel(cc, key[e], taken)) << e;
      }
      uint32_t tsel;
      const uint32_t pre_sel = warp_prefix_small(__popc(sm), &tsel);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        if ((sm >> e) & 1u) {
          const int64_t o = base_out[cc] + sel_run[cc] + pre_sel + __popc(sm & ((1u << e) - 1u));
          if (o >= limit) raise(a.d_status, GSPARSE_DERR_CAPACITY);
          else if (C == 1) {
            out_idx[o] = (int32_t)(v + e);
            out_val[o] = x[e];
            if (a.u) a.u[v + e] = 0.0f;  // momentum masking of the sent entry
          } else { a.lidx[o] = (int32_t)(v + e); a.lval[o] = x[e]; }
        }
      }
      eq_run[cc] += teq;
      sel_run[cc] += tsel;
      selm |= sm;
    }
    if (a.zero_mode && selm) {
#pragma unroll
      for (int e = 0; e < 4; ++e)
        if ((selm >> e) & 1u) a.r[v + e] = 0.0f;
    }
  }
}

// ------------------------------------------------------------------------------------------
// binarise: means, choice, output

__global__ void __launch_bounds__(1024) bjobs_kernel(Sel a, SumJob* jobs) {
  pdl_begin();
  __shared__ int64_t sh[33];
  if (a.ctl[0]) return;
  const int64_t P = (int64_t)a.T * 2;
  int64_t carry = 0;
  for (int64_t base = 0; base < P; base += blockDim.x) {
    const int64_t p = base + threadIdx.x;
    int64_t leaves = 0;
    if (p < P) leaves = cdiv(a.keff[p], kSumBlock);
    int64_t tot;
    const int64_t ex = block_exclusive_scan(leaves, sh, &tot);
    if (p < P) {
      const int32_t s = (int32_t)(p >> 1);
      const int c = (int)(p & 1);
      SumJob J;
      J.vals = a.lval + 2 * a.seg_kbase[s] + c * a.seg_k[s];
      J.len = a.keff[p];
      J.mode = c == 0 ? kSumAll : kSumNegated;
      J.pad = 0;
      J.leaf_base = carry + ex;
      J.count = 0;
      J.sum = 0.0;
      J.mean = 0.0f;
      J.done_blocks = 0;
      jobs[p] = J;
    }
    carry += tot;
  }
}

__global__ void __launch_bounds__(1024) bchoose_kernel(Sel a, const SumJob* jobs, float* d_mean, int64_t* out_offsets) {
  pdl_begin();
  __shared__ int64_t sh[33];
  if (a.ctl[0]) return;
  int64_t carry = 0;
  for (int64_t base = 0; base < a.T; base += blockDim.x) {
    const int64_t s = base + threadIdx.x;
    int64_t cnt = 0;
    if (s < a.T) {
      const int64_t kp = a.keff[2 * s], kn = a.keff[2 * s + 1];
      const float mp = jobs[2 * s].mean, mn = jobs[2 * s + 1].mean;
      const bool pos = kp > 0 && mp >= mn;
      const bool neg = !pos && kn > 0;
      a.bsel[s] = pos ? 0 : (neg ? 1 : -1);
      d_mean[s] = pos ? mp : (neg ? -mn : 0.0f);
      cnt = pos ? kp : (neg ? kn : 0);
    }
    int64_t tot;
    const int64_t ex = block_exclusive_scan(cnt, sh, &tot);
    if (s < a.T) out_offsets[s] = carry + ex;
    carry += tot;
  }
  if (threadIdx.x == 0) out_offsets[a.T] = carry;
}

__global__ void bemit_kernel(Sel a, const float* d_mean, const int64_t* out_offsets,
                             int64_t bound, int32_t* out_idx, float* out_val) {
  pdl_begin();
  if (a.ctl[0]) return;
  const int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= bound || j >= out_offsets[a.T]) return;
  const int32_t s = (int32_t)(upper_bound_i64(out_offsets, a.T + 1, j) - 1);
  const int c = a.bsel[s];
  const int64_t src = 2 * a.seg_kbase[s] + c * a.seg_k[s] + (j - out_offsets[s]);
  const int32_t i = a.lidx[src];
  const float m = d_mean[s];
  out_idx[j] = i;
  if (out_val) out_val[j] = m;
  a.r[i] = __fsub_rn(a.lval[src], m);
}

// ------------------------------------------------------------------------------------------
// binarise, magnitude-first reading: the top-k list S of each segment (residual top-k), then the
// means of its positive and of its negative members (fixed-order sums over the positions of S),
// the choice per segment, and an ordered compaction of the chosen members

constexpr int kMagBlock = 1024;  // list positions per compaction block (4 per thread)

// Two sum jobs per segment over the members of S: positive (job 2s) and negative (job 2s + 1),
// summed as a pair (the list is read once): the pair's leaves are leaves [pb_s, pb_s + L_s) of the
// positive job and [pair_bound + pb_s, ...) of the negative job.
__global__ void __launch_bounds__(1024) mjobs_kernel(const float* lval, const int64_t* loff, int32_t T,
                                                     int64_t pair_bound, SumJob* jobs,
                                                     const int32_t* abort_flag) {
  pdl_begin();
  __shared__ int64_t sh[33];
  if (*abort_flag) return;
  int64_t carry = 0;
  for (int64_t base = 0; base < (int64_t)T; base += blockDim.x) {
    const int64_t s = base + threadIdx.x;
    const int64_t len = s < T ? loff[s + 1] - loff[s] : 0;
    int64_t tot;
    const int64_t ex = block_exclusive_scan(cdiv(len, kSumBlock), sh, &tot);
    for (int c = 0; c < 2 && s < T; ++c) {
      SumJob J;
      J.vals = lval + loff[s];
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
}

// mu+ = mean of the positive members, mu- = -(mean of the negative members); the larger is sent
// (ties to positive), with the signed mean.
__global__ void __launch_bounds__(1024) mchoose_kernel(const SumJob* jobs, int32_t T, int32_t* bsel,
                                                       float* d_mean, int64_t* out_offsets,
                                                       const int32_t* abort_flag) {
  pdl_begin();
  __shared__ int64_t sh[33];
  if (*abort_flag) return;
  int64_t carry = 0;
  for (int64_t base = 0; base < T; base += blockDim.x) {
    const int64_t s = base + threadIdx.x;
    int64_t cnt = 0;
    if (s < T) {
      const int64_t np = (int64_t)jobs[2 * s].count, nn = (int64_t)jobs[2 * s + 1].count;
      const float mp = jobs[2 * s].mean, mn = -jobs[2 * s + 1].mean;
      const bool pos = np > 0 && mp >= mn;
      const bool neg = !pos && nn > 0;
      bsel[s] = pos ? 0 : (neg ? 1 : -1);
      d_mean[s] = pos ? mp : (neg ? -mn : 0.0f);
      cnt = pos ? np : (neg ? nn : 0);
    }
    int64_t tot;
    const int64_t ex = block_exclusive_scan(cnt, sh, &tot);
    if (s < T) out_offsets[s] = carry + ex;
    carry += tot;
  }
  if (threadIdx.x == 0) out_offsets[T] = carry;
}

__device__ __forceinline__ bool mag_chosen(const int32_t* bsel, const int64_t* loff, int32_t T,
                                           const float* lval, int64_t j, int32_t* seg_out) {
  const int32_t s = (int32_t)(upper_bound_i64(loff, T + 1, j) - 1);
  *seg_out = s;
  const int c = bsel[s];
  return c == 0 ? lval[j] > 0.0f : (c == 1 ? lval[j] < 0.0f : false);
}

__global__ void __launch_bounds__(256) mcount_kernel(const int32_t* bsel, const int64_t* loff, int32_t T,
                                                     const float* lval, int64_t* bcnt,
                                                     const int32_t* abort_flag) {
  pdl_begin();
  __shared__ int64_t sh[33];
  if (*abort_flag) return;
  const int64_t K = loff[T];
  const int64_t j0 = (int64_t)blockIdx.x * kMagBlock + 4 * threadIdx.x;
  int64_t mine = 0;
  for (int e = 0; e < 4; ++e) {
    int32_t s;
    if (j0 + e < K && mag_chosen(bsel, loff, T, lval, j0 + e, &s)) ++mine;
  }
  int64_t tot;
  block_exclusive_scan(mine, sh, &tot);
  if (threadIdx.x == 0) bcnt[blockIdx.x] = tot;
}

__global__ void __launch_bounds__(1024) mscan_kernel(int64_t* bcnt, int64_t nblk, const int32_t* abort_flag) {
  pdl_begin();
  __shared__ int64_t sh[33];
  if (*abort_flag) return;
  int64_t carry = 0;
  for (int64_t base = 0; base < nblk; base += blockDim.x) {
    const int64_t b = base + threadIdx.x;
    const int64_t v = b < nblk ? bcnt[b] : 0;
    int64_t tot;
    const int64_t ex = block_exclusive_scan(v, sh, &tot);
    if (b < nblk) bcnt[b] = carry + ex;
    carry += tot;
  }
}

// The chosen members of S leave in list order (their global rank among the chosen is their output
// position, since the segments' outputs are consecutive); every member of S gets its residual:
// fl(acc - m_s) when sent, acc otherwise (the top-k left +0 there).
__global__ void __launch_bounds__(256) memit_kernel(const int32_t* bsel, const int64_t* loff, int32_t T,
                                                    const int32_t* lidx, const float* lval,
                                                    const int64_t* bcnt, const float* d_mean, float* r,
                                                    int32_t* out_idx, float* out_val, int64_t out_capacity,
                                                    int32_t* d_status, const int32_t* abort_flag) {
  pdl_begin();
  __shared__ int64_t sh[33];
  if (*abort_flag) return;
  const int64_t K = loff[T];
  const int64_t j0 = (int64_t)blockIdx.x * kMagBlock + 4 * threadIdx.x;
  bool ch[4];
  int32_t sg[4];
  int64_t mine = 0;
  for (int e = 0; e < 4; ++e) {
    ch[e] = j0 + e < K && mag_chosen(bsel, loff, T, lval, j0 + e, &sg[e]);
    mine += ch[e];
  }
  int64_t tot;
  int64_t o = bcnt[blockIdx.x] + block_exclusive_scan(mine, sh, &tot);
  for (int e = 0; e < 4; ++e) {
    const int64_t j = j0 + e;
    if (j >= K) break;
    const int32_t i = lidx[j];
    if (ch[e]) {
      const float m = d_mean[sg[e]];
      if (o >= out_capacity) {
        raise(d_status, GSPARSE_DERR_CAPACITY);
      } else {
        out_idx[o] = i;
        if (out_val) out_val[o] = m;
      }
      r[i] = __fsub_rn(lval[j], m);
      ++o;
    } else {
      r[i] = lval[j];
    }
  }
}

// ------------------------------------------------------------------------------------------
// accumulate only (keep 0): residual <- fl(g + residual)

// ctl null: no plan ran (one segment), and the kernel itself reports the empty output offsets.
// With momentum (u non-null) the gradient term is v = fl(fl(mom * u) + g), and u <- v.
__global__ void accumulate_kernel(const float* g, float* r, int64_t n, const int32_t* ctl,
                                  int64_t* out_offsets, float* u, float mom) {
  pdl_begin();
  if (ctl && ctl[0]) return;
  if (!ctl && out_offsets && blockIdx.x == 0 && threadIdx.x < 2) out_offsets[threadIdx.x] = 0;
  const int64_t nv = n >> 2;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t v = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; v < nv; v += stride) {
    float4 a = ld_stream(g + 4 * v);
    const float4 b = ld_stream(r + 4 * v);
    if (u) {
      a = momentum4(mom, ld_stream(u + 4 * v), a);
      st_stream(u + 4 * v, a);
    }
    st_stream(r + 4 * v, make_float4(__fadd_rn(a.x, b.x), __fadd_rn(a.y, b.y), __fadd_rn(a.z, b.z),
                                     __fadd_rn(a.w, b.w)));
  }
  const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (t < (n & 3)) {
    const int64_t i = 4 * nv + t;
    float gi = g[i];
    if (u) {
      gi = __fadd_rn(__fmul_rn(mom, u[i]), gi);
      u[i] = gi;
    }
    r[i] = __fadd_rn(gi, r[i]);
  }
}

// ------------------------------------------------------------------------------------------
// host side

struct Layout {
  int64_t n, Lp, Q, cap, cap_rec;
  int32_t T, C;
  size_t fixed_bytes, total_bytes;
  Sel a;
  // binarise extras
  SumJob* jobs;
  double* leaves;
  double* partials;
  int64_t leaf_bound, per_job_leaf_bound, kbound;
  char* zero_begin;
  size_t zero_bytes;
};

int64_t pick_lp(int64_t n) {
  int64_t lp = cdiv(n > 0 ? n : 1, kTargetPieces);
  return round_up(lp < kGranule ? kGranule : lp, kGranule);
}

// k bound over all segmentations: sum_s ceil(n_s f) <= ceil(n f) + T
int64_t k_bound(int64_t n, int32_t T, int64_t num, int64_t den) {
  const int64_t kb = kept_count(n, num, den) + T;
  return kb < n ? kb : n;
}

int64_t rec_cap(int64_t Lp, int32_t C, int64_t num, int64_t den) {
  const double q = den > 0 ? (double)num / (double)den : 1.0;
  const double f = q + 3.0 * sqrt(q / kSample) + 16.0 / kSample;
  double cap = ceil((double)Lp * f * C * 1.25) + 64.0;
  if (cap > (double)Lp) cap = (double)Lp;
  return round_up((int64_t)cap, 32);
}

// Carves the workspace (ws may be null to measure). cap_req < 0: recommended capacity.
Layout carve(int64_t n, int32_t T, int32_t C, int64_t num, int64_t den, void* ws, size_t ws_bytes,
             bool measure_rec) {
  Layout L{};
  L.n = n;
  L.T = T;
  L.C = C;
  L.Lp = pick_lp(n);
  L.Q = cdiv(n, L.Lp) + T;
  const int64_t P = (int64_t)T * C;
  Carver cv(ws);
  Sel& a = L.a;
  a.seg_lo = cv.take<int64_t>(T);
  a.seg_n = cv.take<int64_t>(T);
  a.seg_k = cv.take<int64_t>(T);
  a.seg_kbase = cv.take<int64_t>(T + 1);
  a.seg_pbase = cv.take<int64_t>(T + 1);
  a.tlo = cv.take<uint32_t>(P);
  a.pfx = cv.take<uint32_t>(P);
  a.thr = cv.take<uint32_t>(P);
  a.keff = cv.take<int64_t>(P);
  a.krem = cv.take<int64_t>(P);
  a.need_eq = cv.take<int64_t>(P);
  a.uoff = cv.take<int64_t>(L.Q + 1);
  a.pstart = cv.take<uint32_t>(L.Q + 1);
  a.srun = cv.take<uint32_t>((int64_t)T * kSampleRuns * 2);
  // work units: a stored piece holds at most as many candidates as entries, so at most
  // n / 2^kUnitShift + Q units; a re-read piece at most kReadUnits
  a.Ur = round_up(cdiv(L.Lp, kReadUnits), 128);
  a.units_bound = L.Q * (kReadUnits + 1) + (n >> kUnitShift) + 1;
  a.upiece = cv.take<int32_t>(a.units_bound);
  a.pgt = cv.take<uint32_t>(a.units_bound * C);
  a.peq = cv.take<uint32_t>(a.units_bound * C);
  a.ptake = cv.take<uint32_t>(a.units_bound * C);
  a.poff = cv.take<int64_t>(a.units_bound * C);
  // zero-initialised block
  const size_t zoff = (size_t)round_up((int64_t)cv.off, 256);
  a.ctl = cv.take<int32_t>(64);
  a.redo = cv.take<uint32_t>(P);
  a.pcnt = cv.take<uint32_t>(L.Q);
  a.prsrc = cv.take<uint32_t>(L.Q);
  a.hist = cv.take<uint32_t>(P * kHist);
  a.shist = cv.take<uint32_t>(P * 2 * kBins1);
  a.scount = cv.take<uint32_t>(P);
  a.sdone = cv.take<uint32_t>(2 * (int64_t)T);
  a.svar = cv.take<unsigned long long>(2 * P);
  const size_t zend = cv.off;
  a.sb1 = cv.take<uint32_t>(P);
  a.sblo = cv.take<uint32_t>(P);
  a.ssub = cv.take<uint32_t>(P);
  a.srank = cv.take<int64_t>(P);
  a.sabove = cv.take<int64_t>(P);
  a.smcap = cv.take<int64_t>(P);
  L.zero_begin = ws ? (char*)ws + zoff : nullptr;
  L.zero_bytes = zend - zoff;
  if (C == 2) {
    L.kbound = k_bound(n, T, num, den);
    a.lidx = cv.take<int32_t>(2 * L.kbound);
    a.lval = cv.take<float>(2 * L.kbound);
    a.bsel = cv.take<int32_t>(T);
    L.jobs = cv.take<SumJob>(P);
    L.leaf_bound = cdiv(2 * L.kbound, kSumBlock) + P;
    L.per_job_leaf_bound = cdiv(kept_count(n, num, den), kSumBlock);
    L.leaves = cv.take<double>(L.leaf_bound);
    L.partials = cv.take<double>(P * osum_partial_stride(L.per_job_leaf_bound));
  }
  // pool chunks: a power of two >= 512 slots (one 512-entry chunk of pass 1 never needs more than
  // one new chunk), with kMaxChunks of them covering a whole piece
  int32_t shift = 9;
  while ((kMaxChunks << shift) < L.Lp) ++shift;
  a.chunk_shift = shift;
  a.max_chunks = kMaxChunks;
  a.pchunk = cv.take<int32_t>(L.Q * kMaxChunks);
  a.pnch = cv.take<uint32_t>(L.Q);
  L.fixed_bytes = cv.off + 512;
  L.cap_rec = rec_cap(L.Lp, C, num, den);
  const int64_t csz = (int64_t)1 << shift;
  int64_t cap, pool;
  if (measure_rec) {
    cap = L.cap_rec;
    // room for about twice the kept entries beyond the primary stores, as whole chunks
    pool = cdiv(2 * C * k_bound(n, T, num, den), csz) + 64;
  } else {
    // the primary stores up to the recommended size (int4-aligned), the rest as pool chunks
    const int64_t room = ws_bytes > L.fixed_bytes ? (int64_t)(ws_bytes - L.fixed_bytes) : 0;
    cap = (room / (L.Q * 8 > 0 ? L.Q * 8 : 1)) & ~(int64_t)3;
    if (cap > L.cap_rec) cap = L.cap_rec;
    if (cap > L.Lp) cap = L.Lp;
    pool = (room - L.Q * cap * 8 - 512) / (csz * 8);
    if (pool < 0) pool = 0;
  }
  if (pool > INT32_MAX) pool = INT32_MAX;
  L.cap = cap;
  a.pool_chunks = pool;
  // a stored piece's work unit covers at least its primary store (pieces that did not spill are
  // one unit each)
  int32_t us = kUnitShift;
  while (((int64_t)1 << us) < cap) ++us;
  a.ushift = us;
  a.cidx = cv.take<int32_t>(L.Q * cap + pool * csz);
  a.cval = cv.take<float>(L.Q * cap + pool * csz);
  L.total_bytes = cv.off;
  a.cap = cap;
  a.Lp = L.Lp;
  a.Q = L.Q;
  a.n = n;
  a.T = T;
  a.C = C;
  return L;
}

bool bad_keep(int64_t num, int64_t den) { return den <= 0 || num < 0 || num > den; }

template <int C>
int run_select(const float* g, float* r, int64_t n, const int64_t* seg, int32_t T, int64_t num,
               int64_t den, int32_t* out_idx, float* out_val, float* d_mean, int64_t* out_offsets,
               int64_t out_capacity, const gsparse_pending* pending, uint32_t flags, void* ws,
               size_t ws_bytes, int32_t* d_status, cudaStream_t st,
               const gsparse_pass_events* events, float* u = nullptr, float mom = 0.0f) {
  if (pending && (!pending->d_count || pending->capacity < 0 ||
                  (pending->capacity > 0 && (!pending->idx || !pending->val))))
    return GSPARSE_ERR_INVALID_ARG;
  if (n < 0 || T < 1 || (seg == nullptr && T != 1) || bad_keep(num, den) || !out_offsets ||
      out_capacity < 0)
    return GSPARSE_ERR_INVALID_ARG;
  if (n > INT32_MAX) return GSPARSE_ERR_UNSUPPORTED;
  if (n > 0 && (!g || !r || !aligned16(g) || !aligned16(r))) return GSPARSE_ERR_INVALID_ARG;
  if (u && (C != 1 || !aligned16(u) || u == r || u == g)) return GSPARSE_ERR_INVALID_ARG;
  if (n == 0) u = nullptr;
  if (out_capacity > 0 && !out_idx) return GSPARSE_ERR_INVALID_ARG;
  if (C == 1 && out_capacity > 0 && !out_val) return GSPARSE_ERR_INVALID_ARG;
  if (C == 2 && !d_mean) return GSPARSE_ERR_INVALID_ARG;
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u)) return GSPARSE_ERR_WORKSPACE;
  Layout L = carve(n, T, C, num, den, ws, ws_bytes, false);
  if (ws_bytes < L.total_bytes || ws_bytes < L.fixed_bytes) return GSPARSE_ERR_WORKSPACE;
  Sel a = L.a;
  a.g = g;
  a.r = r;
  a.u = u;
  a.mom = mom;
  a.zero_mode = C == 1;
  a.wait_test = (flags & GSPARSE_SELECT_TEST_EXPIRE_WAIT) ? 1 : 0;
  a.d_status = d_status;
  const bool has_pending = pending && pending->capacity > 0;
  if (num == 0 && C == 1 && !has_pending && seg == nullptr) {
    // communication delay step on one segment: accumulate only, nothing to plan
    const int64_t blocks = cdiv(n, 4 * 256) < 148 * 8 ? cdiv(n, 4 * 256) : 148 * 8;
    launch(accumulate_kernel, (unsigned)(blocks > 0 ? blocks : 1), 256, 0, st, g, r, n, nullptr, out_offsets,
                                                                          u, mom);
    return launch_status();
  }
  a.pw_idx = has_pending ? pending->idx : nullptr;
  a.pw_val = has_pending ? pending->val : nullptr;
  a.pw_count = has_pending ? pending->d_count : nullptr;
  a.pw_cap = has_pending ? pending->capacity : 0;
  if (cudaMemsetAsync(L.zero_begin, 0, L.zero_bytes, st) != cudaSuccess) return GSPARSE_ERR_CUDA;
  launch(plan_kernel, 1, 1024, 0, st, a, seg, num, den, out_capacity, C == 1 ? out_offsets : nullptr);
  if (has_pending)
    launch(pending_check_kernel, (unsigned)cdiv(a.pw_cap + 1, 256 * kCheckPer), 256, 0, st, a);
  if (num == 0 && C == 1 && !has_pending) {  // communication delay step: accumulate only
    if (n > 0) {
      const int64_t blocks = cdiv(n, 4 * 256) < 148 * 8 ? cdiv(n, 4 * 256) : 148 * 8;
      launch(accumulate_kernel, (unsigned)(blocks > 0 ? blocks : 1), 256, 0, st, g, r, n, a.ctl, nullptr, u,
                                                                            mom);
    }
    return launch_status();
  }
  const unsigned piece_ctas = (unsigned)cdiv(L.Q, kWarps);
  const int exhaustive = (flags & GSPARSE_SELECT_EXHAUSTIVE) ? 1 : 0;
  const dim3 sgrid(kSampleCtas, (unsigned)T);
  launch(sample_kernel<C>, sgrid, kSampleThreads, 0, st, a, 1, exhaustive);
  launch(sample_kernel<C>, sgrid, kSampleThreads, 0, st, a, 2, exhaustive);
  const bool timed = events && events->before && events->after;
  if (timed) cudaEventRecord((cudaEvent_t)events->before, st);
  if (piece_ctas) {
    if constexpr (C == 1) {
      if (a.u) {
        if (cudaFuncSetAttribute(pass1_ring_kernel<1, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)kRingBytesM) != cudaSuccess)
          return GSPARSE_ERR_CUDA;
        launch(pass1_ring_kernel<1, true>, piece_ctas, kThreads, kRingBytesM, st, a);
      } else {
        // two streams through the 3-stage ring: faster than the register pipeline on flat
        // gradients (2% at a 99% drop, 9% at 90%), 4% slower when candidates cluster
        constexpr size_t kRingBytes = sizeof(RingSlot) * kStages * kWarps;
        if (cudaFuncSetAttribute(pass1_ring_kernel<1, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)kRingBytes) != cudaSuccess)
          return GSPARSE_ERR_CUDA;
        launch(pass1_ring_kernel<1, false>, piece_ctas, kThreads, kRingBytes, st, a);
      }
    } else {
      launch(pass1_kernel<C>, piece_ctas, kThreads, 0, st, a);
    }
  }
  if (timed) cudaEventRecord((cudaEvent_t)events->after, st);
  launch(check_kernel, (unsigned)(T * C), 256, 0, st, a);
  // the steps after pass 1 run over work units, at most a.units_bound of them
  int64_t uc = cdiv(a.units_bound, kWarps);
  if (uc > (int64_t)sm_count() * 8) uc = (int64_t)sm_count() * 8;
  const unsigned unit_ctas = piece_ctas ? (unsigned)uc : 0u;
  if (piece_ctas) launch(restore_kernel<C>, piece_ctas, kThreads, 0, st, a);
  launch(select_kernel, (unsigned)(T * C), 1024, 0, st, a, 1);
  if (unit_ctas) launch(hist_kernel<C>, unit_ctas, kThreads, 0, st, a, 2);
  launch(select_kernel, (unsigned)(T * C), 1024, 0, st, a, 2);
  if (unit_ctas) launch(hist_kernel<C>, unit_ctas, kThreads, 0, st, a, 3);
  launch(select_kernel, (unsigned)(T * C), 1024, 0, st, a, 3);
  if (unit_ctas) launch(count_kernel<C>, unit_ctas, kThreads, 0, st, a);
  launch(scan_kernel, (unsigned)(T * C), 1024, 0, st, a);
  if (unit_ctas)
    launch(emit_kernel<C>, unit_ctas, kThreads, 0, st, a, out_idx, out_val,
                                                    C == 1 ? out_capacity : 2 * L.kbound);
  if (C == 2) {
    launch(bjobs_kernel, 1, 1024, 0, st, a, L.jobs);
    osum_launch(L.jobs, T * 2, L.leaves, L.leaf_bound, L.per_job_leaf_bound, L.partials, a.ctl, st);
    launch(bchoose_kernel, 1, 1024, 0, st, a, L.jobs, d_mean, out_offsets);
    if (L.kbound > 0)
      launch(bemit_kernel, (unsigned)cdiv(L.kbound, 256), 256, 0, st, a, d_mean, out_offsets, L.kbound,
                                                                  out_idx, out_val);
  }
  return launch_status();
}

// Magnitude-first binarisation: its own lists and sums at the front of the workspace, the
// residual top-k's workspace behind them.
struct MagLayout {
  int32_t* lidx;
  float* lval;
  int64_t* loff;
  SumJob* jobs;
  double* leaves;
  double* partials;
  int32_t* bsel;
  int64_t* bcnt;
  int64_t kb, leaf_bound, per_job, nblk;
  size_t bytes;
};

MagLayout mag_carve(int64_t n, int32_t T, int64_t num, int64_t den, void* ws) {
  MagLayout M;
  Carver cv(ws);
  M.kb = k_bound(n, T, num, den);
  M.lidx = cv.take<int32_t>(M.kb);
  M.lval = cv.take<float>(M.kb);
  M.loff = cv.take<int64_t>((int64_t)T + 1);
  M.per_job = cdiv(M.kb, kSumBlock);
  M.leaf_bound = M.per_job + T;   // leaves of the pair numbering (each sign has this many)
  M.jobs = cv.take<SumJob>(2 * (int64_t)T);
  M.leaves = cv.take<double>(2 * M.leaf_bound);
  M.partials = cv.take<double>(2 * (int64_t)T * osum_partial_stride(M.per_job));
  M.bsel = cv.take<int32_t>(T);
  M.nblk = cdiv(M.kb > 0 ? M.kb : 1, kMagBlock);
  M.bcnt = cv.take<int64_t>(M.nblk + 1);
  M.bytes = (size_t)round_up((int64_t)cv.off, 256);
  return M;
}

int run_binarize_magnitude(const float* g, float* r, int64_t n, const int64_t* seg, int32_t T,
                           int64_t num, int64_t den, int32_t* out_idx, float* out_val, float* d_mean,
                           int64_t* out_offsets, int64_t out_capacity, uint32_t flags, void* ws,
                           size_t ws_bytes, int32_t* d_status, cudaStream_t st,
                           const gsparse_pass_events* events) {
  if (n < 0 || T < 1 || bad_keep(num, den) || !d_mean || !out_offsets || out_capacity < 0)
    return GSPARSE_ERR_INVALID_ARG;
  if (n > INT32_MAX) return GSPARSE_ERR_UNSUPPORTED;
  if (out_capacity > 0 && !out_idx) return GSPARSE_ERR_INVALID_ARG;
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u)) return GSPARSE_ERR_WORKSPACE;
  const MagLayout M = mag_carve(n, T, num, den, ws);
  if (ws_bytes < M.bytes) return GSPARSE_ERR_WORKSPACE;
  void* tws = static_cast<char*>(ws) + M.bytes;
  const size_t tws_bytes = ws_bytes - M.bytes;
  // S: the residual top-k into the internal lists (the caller's capacity bounds sum k_s, as for
  // the two-set reading)
  const int rc = run_select<1>(g, r, n, seg, T, num, den, M.lidx, M.lval, nullptr, M.loff,
                               out_capacity < M.kb ? out_capacity : M.kb, nullptr,
                               flags & GSPARSE_SELECT_EXHAUSTIVE, tws, tws_bytes, d_status, st, events);
  if (rc != GSPARSE_OK) return rc;
  const int32_t* abort_flag = carve(n, T, 1, num, den, tws, tws_bytes, false).a.ctl;
  launch(mjobs_kernel, 1, 1024, 0, st, M.lval, M.loff, T, M.leaf_bound, M.jobs, abort_flag);
  osum_launch_pairs(M.jobs, T, M.leaves, M.leaf_bound, M.per_job, M.partials, abort_flag, st);
  launch(mchoose_kernel, 1, 1024, 0, st, M.jobs, T, M.bsel, d_mean, out_offsets, abort_flag);
  if (M.kb > 0) {
    launch(mcount_kernel, (unsigned)M.nblk, 256, 0, st, M.bsel, M.loff, T, M.lval, M.bcnt, abort_flag);
    launch(mscan_kernel, 1, 1024, 0, st, M.bcnt, M.nblk, abort_flag);
    launch(memit_kernel, (unsigned)M.nblk, 256, 0, st, M.bsel, M.loff, T, M.lidx, M.lval, M.bcnt, d_mean, r,
                                                   out_idx, out_val, out_capacity, d_status, abort_flag);
  }
  return launch_status();
}

// Scratch of gsparse_residual_topk_noalloc: one array per device, in the library's own memory.
static __device__ __align__(256) unsigned char g_noalloc_scratch[GSPARSE_NOALLOC_SCRATCH_BYTES];

// Device address of the array on the current device, looked up once per device. In host code
// the symbol itself is only a host-side stand-in, never a device address. Several host threads
// may look it up at once: each writes the same address, published with release ordering.
int noalloc_scratch(void** out) {
  static std::atomic<void*> addr[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return GSPARSE_ERR_CUDA;
  }
  if (dev < 0 || dev >= 64) return GSPARSE_ERR_UNSUPPORTED;
  void* p = addr[dev].load(std::memory_order_acquire);
  if (!p) {
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
      cudaGetLastError();   // leave no error behind for the caller's next launch check
      return GSPARSE_ERR_CUDA;
    }
    addr[dev].store(p, std::memory_order_release);
  }
  *out = p;
  return GSPARSE_OK;
}

}  // namespace
}  // namespace gs

using namespace gs;

extern "C" {

size_t gsparse_residual_topk_workspace_size(int64_t n, int32_t T, int64_t num, int64_t den) {
  if (n < 0 || T < 1 || bad_keep(num, den)) return 0;
  return carve(n, T, 1, num, den, nullptr, 0, true).total_bytes + 256;
}

size_t gsparse_residual_topk_workspace_min(int64_t n, int32_t T) {
  if (n < 0 || T < 1) return 0;
  return carve(n, T, 1, 1, 1, nullptr, 0, false).fixed_bytes;
}

int gsparse_residual_topk_momentum(const float* g, float* momentum_buf, float momentum,
                                   float* residual, int64_t n, const int64_t* seg_offsets,
                                   int32_t num_segments, int64_t keep_num, int64_t keep_den,
                                   int32_t* out_idx, float* out_val, int64_t* out_offsets,
                                   int64_t out_capacity, const gsparse_pending* pending,
                                   uint32_t flags, void* workspace, size_t workspace_bytes,
                                   int32_t* d_status, gsparse_stream stream,
                                   const gsparse_pass_events* pass_events) {
  if (n > 0 && !momentum_buf) return GSPARSE_ERR_INVALID_ARG;
  return run_select<1>(g, residual, n, seg_offsets, num_segments, keep_num, keep_den, out_idx,
                       out_val, nullptr, out_offsets, out_capacity, pending, flags, workspace,
                       workspace_bytes, d_status, (cudaStream_t)stream, pass_events, momentum_buf,
                       momentum);
}

int gsparse_residual_topk(const float* g, float* residual, int64_t n, const int64_t* seg_offsets,
                          int32_t num_segments, int64_t keep_num, int64_t keep_den, int32_t* out_idx,
                          float* out_val, int64_t* out_offsets, int64_t out_capacity,
                          const gsparse_pending* pending, uint32_t flags, void* workspace,
                          size_t workspace_bytes, int32_t* d_status, gsparse_stream stream,
                          const gsparse_pass_events* pass_events) {
  return run_select<1>(g, residual, n, seg_offsets, num_segments, keep_num, keep_den, out_idx,
                       out_val, nullptr, out_offsets, out_capacity, pending, flags, workspace,
                       workspace_bytes, d_status, (cudaStream_t)stream, pass_events);
}

size_t gsparse_binarize_workspace_size(int64_t n, int32_t T, int64_t num, int64_t den) {
  if (n < 0 || T < 1 || bad_keep(num, den)) return 0;
  const size_t two_sets = carve(n, T, 2, num, den, nullptr, 0, true).total_bytes + 256;
  const size_t by_mag = mag_carve(n, T, num, den, nullptr).bytes +
                        carve(n, T, 1, num, den, nullptr, 0, true).total_bytes + 256;
  return two_sets > by_mag ? two_sets : by_mag;
}

size_t gsparse_binarize_workspace_min(int64_t n, int32_t T, int64_t num, int64_t den) {
  if (n < 0 || T < 1 || bad_keep(num, den)) return 0;
  const size_t two_sets = carve(n, T, 2, num, den, nullptr, 0, false).fixed_bytes;
  const size_t by_mag = mag_carve(n, T, num, den, nullptr).bytes +
                        carve(n, T, 1, num, den, nullptr, 0, false).fixed_bytes;
  return two_sets > by_mag ? two_sets : by_mag;
}

int gsparse_residual_topk_noalloc(const float* g, float* residual, int64_t n, int64_t keep_num,
                                  int64_t keep_den, int32_t* out_idx, float* out_val,
                                  int64_t* out_offsets, int64_t out_capacity, int32_t* d_status,
                                  gsparse_stream stream) {
  if (n > GSPARSE_NOALLOC_MAX_N) return GSPARSE_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  const int st = noalloc_scratch(&scratch);
  if (st != GSPARSE_OK) return st;
  return run_select<1>(g, residual, n, nullptr, 1, keep_num, keep_den, out_idx, out_val, nullptr,
                       out_offsets, out_capacity, nullptr, 0, scratch, GSPARSE_NOALLOC_SCRATCH_BYTES,
                       d_status, (cudaStream_t)stream, nullptr);
}

int gsparse_binarize(const float* g, float* residual, int64_t n, const int64_t* seg_offsets,
                     int32_t num_segments, int64_t keep_num, int64_t keep_den, int32_t* out_idx,
                     float* out_val, float* d_mean, int64_t* out_offsets, int64_t out_capacity,
                     uint32_t flags, void* workspace, size_t workspace_bytes, int32_t* d_status,
                     gsparse_stream stream, const gsparse_pass_events* pass_events) {
  if (flags & GSPARSE_BINARIZE_BY_MAGNITUDE)
    return run_binarize_magnitude(g, residual, n, seg_offsets, num_segments, keep_num, keep_den,
                                  out_idx, out_val, d_mean, out_offsets, out_capacity, flags, workspace,
                                  workspace_bytes, d_status, (cudaStream_t)stream, pass_events);
  return run_select<2>(g, residual, n, seg_offsets, num_segments, keep_num, keep_den, out_idx,
                       out_val, d_mean, out_offsets, out_capacity, nullptr, flags, workspace,
                       workspace_bytes, d_status, (cudaStream_t)stream, pass_events);
}

}  // extern "C"
