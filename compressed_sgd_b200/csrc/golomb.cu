// Golomb (Rice, M = 2^b) coding of the gaps between sent positions ("Sparse Binary
// Compression", §II Optimal Position Encoding; Appendix A: the decoder needs no shapes).
//
// Codeword of gap d: q = d >> b one-bits, a zero-bit, then d mod 2^b in b bits, most significant
// first; stream bit t is bit t % 32 of word t / 32.
//
// Encoder, one pass over the indices: a block of 2048 codewords sums its codeword lengths, finds
// its first bit by a decoupled look-back over the blocks before it (bounded waits; blocks are
// numbered in the order they start, so a block only waits on running blocks), packs its
// codewords into a shared word buffer and writes each of its words once. The two words a block
// may share with its neighbours go to a side array and a small fix-up kernel merges them.
// Decoder: with the side table, one thread per chunk of codewords decodes sequentially from its
// recorded bit offset and checks that it ends where the next chunk starts.
#include "common.cuh"

namespace gs {
namespace {

constexpr int kCodeThreads = 256;
// codewords per thread: 8 for long lists; 2 for short ones (below kShortList), which then spread
// over four times as many blocks
constexpr int kPerLong = 8, kPerShort = 2;
constexpr int64_t kShortList = 1 << 20;
constexpr int kPackWords = 4096;             // shared word buffer of a block (128 Kbit)
constexpr long long kLookbackCycles = 1ll << 31;  // bound of one block's look-back (about a second)

// Look-back descriptors: flag in the top two bits, a bit count below.
constexpr uint64_t kFlagAgg = 1ull << 62;    // the block's own total is published
constexpr uint64_t kFlagInc = 2ull << 62;    // the total of this block and all before it
constexpr uint64_t kValMask = (1ull << 62) - 1ull;

struct GState {
  uint32_t next_block;  // dynamic block numbering (blocks start in this order)
  int32_t abort;        // a look-back gave up
};

__device__ __forceinline__ uint64_t ld_relaxed(const uint64_t* p) {
  uint64_t v;
  asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_relaxed(uint64_t* p, uint64_t v) {
  asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

// The list [begin, begin + len) from the device bounds; false (len 0) if they are invalid.
__device__ __forceinline__ bool list_bounds(const int64_t* d_begin, const int64_t* d_end,
                                            int64_t capacity, int64_t* begin, int64_t* len) {
  const int64_t b = d_begin ? *d_begin : 0;
  const int64_t l = *d_end - b;
  *begin = b;
  *len = (b < 0 || l < 0 || l > capacity) ? 0 : l;
  return !(b < 0 || l < 0 || l > capacity);
}

// Gaps of this thread's KP consecutive codewords (entries j0 .. j0+KP-1 of the list); an
// invalid (negative) gap is reported and coded as 0. Indices are non-negative int32, so a gap
// fits 32 bits. The entries come in as 16-byte loads when they are aligned.
template <int KP>
__device__ __forceinline__ void thread_gaps(const int32_t* x, int64_t len, int64_t base, int64_t j0,
                                            uint32_t (&d)[KP], int32_t* d_status) {
  int32_t v[KP];
  if (KP % 4 == 0 && j0 > 0 && j0 + KP <= len && (reinterpret_cast<uintptr_t>(x + j0) & 15u) == 0) {
    // a full run after the list's first entry: 32-bit differences (indices are int32, so
    // idx - prev - 1 fits 32 unsigned bits whenever idx > prev)
#pragma unroll
    for (int h = 0; h < KP / 4; ++h) {
      const int4 a = *reinterpret_cast<const int4*>(x + j0 + 4 * h);
      v[4 * h] = a.x; v[4 * h + 1] = a.y; v[4 * h + 2] = a.z; v[4 * h + 3] = a.w;
    }
    int32_t prev = x[j0 - 1];
    bool bad = false;
#pragma unroll
    for (int e = 0; e < KP; ++e) {
      const bool up = v[e] > prev;
      bad |= !up;
      d[e] = up ? (uint32_t)v[e] - (uint32_t)prev - 1u : 0u;
      prev = v[e];
    }
    if (bad) raise(d_status, GSPARSE_DERR_INDEX_RANGE);
    return;
  }
  if (KP % 4 == 0 && j0 + KP <= len && (reinterpret_cast<uintptr_t>(x + j0) & 15u) == 0) {
#pragma unroll
    for (int h = 0; h < KP / 4; ++h) {
      const int4 a = *reinterpret_cast<const int4*>(x + j0 + 4 * h);
      v[4 * h] = a.x; v[4 * h + 1] = a.y; v[4 * h + 2] = a.z; v[4 * h + 3] = a.w;
    }
  } else {
#pragma unroll
    for (int e = 0; e < KP; ++e) v[e] = j0 + e < len ? x[j0 + e] : 0;
  }
  int64_t prev = j0 == 0 ? base - 1 : (j0 - 1 < len ? (int64_t)x[j0 - 1] : 0);
  bool bad = false;
#pragma unroll
  for (int e = 0; e < KP; ++e) {
    d[e] = 0;
    if (j0 + e < len) {
      const int64_t g = (int64_t)v[e] - prev - 1;
      if (g < 0) bad = true;
      else d[e] = (uint32_t)g;
      prev = v[e];
    }
  }
  if (bad) raise(d_status, GSPARSE_DERR_INDEX_RANGE);
}

struct Code {
  uint64_t o;     // first bit
  uint64_t q;     // unary length
  uint32_t tail;  // (1 + b)-bit field after the unary run: terminator 0 then reversed remainder
  uint32_t len_tail;
};

// bits of codeword c that fall in word w
__device__ __forceinline__ uint32_t code_bits_in_word(const Code& c, uint64_t w) {
  const uint64_t lo = w * 32, hi = lo + 32;
  uint32_t bits = 0;
  // unary ones [o, o + q)
  const uint64_t a = c.o > lo ? c.o : lo;
  const uint64_t e = (c.o + c.q) < hi ? (c.o + c.q) : hi;
  if (a < e) {
    const uint32_t n = (uint32_t)(e - a), s = (uint32_t)(a - lo);
    bits |= (n == 32 ? 0xffffffffu : ((1u << n) - 1u)) << s;
  }
  // tail field at p = o + q
  const uint64_t p = c.o + c.q;
  if (p < hi && p + c.len_tail > lo) {
    const uint64_t f = (uint64_t)c.tail;
    if (p >= lo) bits |= (uint32_t)(f << (p - lo));
    else bits |= (uint32_t)(f >> (lo - p));
  }
  return bits;
}

// Exclusive prefix of block vb (the bits of all blocks before it), by warp 0 looking back over
// the descriptors of blocks vb-1, vb-2, ... 32 at a time: aggregates are added until a block
// whose inclusive total is published. Blocks are numbered in the order they start, so every
// block waited on is already running and publishes its aggregate without waiting itself.
// Returns false if a descriptor stayed unpublished for kLookbackCycles.
__device__ bool lookback(const uint64_t* flags, uint32_t vb, int lane, uint64_t* prefix) {
  uint64_t acc = 0;
  int64_t p = (int64_t)vb - 1;
  const long long t0 = clock64();
  while (p >= 0) {
    const int64_t q = p - lane;
    uint64_t f = q >= 0 ? ld_relaxed(flags + q) : kFlagInc;   // before block 0: an inclusive 0
    for (;;) {
      const bool missing = (f >> 62) == 0;
      if (!__any_sync(kFull, missing)) break;
      const bool late = lane == 0 && clock64() - t0 > kLookbackCycles;
      if (__any_sync(kFull, late)) return false;
      if (missing) f = ld_relaxed(flags + q);
    }
    const uint32_t inc = __ballot_sync(kFull, (f >> 62) == 2u);
    const int first = inc ? __ffs(inc) - 1 : 32;   // the nearest block with an inclusive total
    acc += warp_sum(lane <= first ? (f & kValMask) : 0ull);
    if (inc) break;
    p -= 32;
  }
  *prefix = acc;
  return true;
}

// One pass: codeword lengths and the block's bit count (published at once), packing into a shared
// word buffer relative to the block's own first bit, then the look-back for that bit's stream
// position (by warp 0, after the packing, so the blocks before have had time to publish) and one
// write per word, shifted into place with a funnel shift. The first and the last word of a block
// may hold bits of the neighbouring block: those two go to head[]/tail[] and the fix-up kernel
// merges them. A block whose bits do not fit the shared buffer (very long unary runs) looks back
// first, zeroes its interior words and ORs its codewords into them.
template <int KP>
__global__ void __launch_bounds__(kCodeThreads, 5) g_encode_kernel(
    const int32_t* idx, const int64_t* d_begin, const int64_t* d_end, int64_t capacity, int64_t base,
    int b, uint32_t* words, int64_t word_capacity, uint64_t* d_nbits, int64_t* table, int32_t chunk,
    GState* state, uint64_t* flags, uint32_t* head, uint32_t* tail, int32_t* d_status) {
  pdl_begin();
  __shared__ uint32_t wbuf[kPackWords + 1];
  __shared__ int64_t sh[33];
  __shared__ uint32_t s_vb;
  __shared__ uint64_t s_prefix;
  __shared__ int s_ok;
  __shared__ uint32_t s_head, s_tail;
  if (threadIdx.x == 0) s_vb = atomicAdd(&state->next_block, 1u);
  int64_t lb, len;
  const bool valid = list_bounds(d_begin, d_end, capacity, &lb, &len);
  __syncthreads();
  const uint32_t vb = s_vb;
  if (!valid) {
    if (vb == 0 && threadIdx.x == 0) {
      raise(d_status, GSPARSE_DERR_CAPACITY);
      *d_nbits = 0;
    }
    return;
  }
  const int64_t nact = cdiv(len, (KP * kCodeThreads));
  if (len == 0) {
    if (vb == 0 && threadIdx.x == 0) *d_nbits = 0;
    return;
  }
  if ((int64_t)vb >= nact) return;
  const int32_t* x = idx + lb;
  const int64_t jb = (int64_t)vb * (KP * kCodeThreads);
  const int64_t j0 = jb + (int64_t)threadIdx.x * KP;
  uint32_t d[KP];
  thread_gaps<KP>(x, len, base, j0, d, d_status);
  // codewords of this thread: entries j0 .. j0 + nv - 1 of the list
  const int nv = len - j0 >= KP ? KP : (len > j0 ? (int)(len - j0) : 0);
  // this thread's bits: 32-bit sums unless a unary part reaches 2^26
  uint32_t l32 = 0;
  bool wide = false;
#pragma unroll
  for (int e = 0; e < KP; ++e) {
    if (e < nv) {
      const uint32_t q = d[e] >> b;
      wide |= q >= (1u << 26);
      l32 += q + 1u + (uint32_t)b;
    }
  }
  uint64_t lu = l32;
  if (wide) {
    lu = 0;
#pragma unroll
    for (int e = 0; e < KP; ++e)
      if (e < nv) lu += (uint64_t)(d[e] >> b) + 1u + (uint32_t)b;
  }
  const int64_t l = (int64_t)lu;
  int64_t tot;
  const int64_t ex = block_exclusive_scan(l, sh, &tot);   // this thread's first bit in the block
  if (threadIdx.x == 0) st_relaxed(flags + vb, (vb == 0 ? kFlagInc : kFlagAgg) | (uint64_t)tot);
  const bool last = (int64_t)vb == nact - 1;
  // relative words [0, nrel): the block's bits from its own first bit
  const int64_t nrel = cdiv(tot, 32);
  const bool fits = nrel + 1 <= kPackWords;
  auto find_prefix = [&]() {
    if (threadIdx.x < 32) {
      uint64_t prefix = 0;
      const bool ok = vb == 0 ? true : lookback(flags, vb, (int)threadIdx.x, &prefix);
      if (threadIdx.x == 0) {
        s_ok = ok;
        s_prefix = prefix;
        if (ok && vb > 0) st_relaxed(flags + vb, kFlagInc | (prefix + (uint64_t)tot));
        if (!ok) {
          raise(d_status, GSPARSE_DERR_TIMEOUT);
          state->abort = 1;
        }
      }
    }
    __syncthreads();
  };
  if (fits) {
    for (int64_t i = threadIdx.x; i <= nrel; i += blockDim.x) wbuf[i] = 0u;
    __syncthreads();
    uint32_t p = (uint32_t)ex;   // relative bit position (< 2^17 here)
#pragma unroll
    for (int e = 0; e < KP; ++e) {
      if (e >= nv) break;
      const uint32_t q = d[e] >> b;
      const uint32_t rem = d[e] & ((1u << b) - 1u);
      // terminator 0, then the remainder most significant bit first
      const uint32_t tl = b ? (__brev(rem) >> (32 - b)) << 1 : 0u;
      if (q + 1u + (uint32_t)b <= 32u) {
        // the whole codeword as one pattern: at most two words
        const uint32_t pat = (q ? 0xffffffffu >> (32u - q) : 0u) | (tl << q);
        const uint64_t v = (uint64_t)pat << (p & 31u);
        if ((uint32_t)v) atomicOr(&wbuf[p >> 5], (uint32_t)v);
        if ((uint32_t)(v >> 32)) atomicOr(&wbuf[(p >> 5) + 1], (uint32_t)(v >> 32));
      } else {
        uint32_t pp = p, qq = q;
        while (qq) {  // the unary run of ones
          const uint32_t s2 = pp & 31u, nrun = qq < 32u - s2 ? qq : 32u - s2;
          atomicOr(&wbuf[pp >> 5], (nrun == 32u ? 0xffffffffu : ((1u << nrun) - 1u)) << s2);
          pp += nrun;
          qq -= nrun;
        }
        const uint64_t v = (uint64_t)tl << (pp & 31u);  // terminator + remainder, <= 32 bits
        if ((uint32_t)v) atomicOr(&wbuf[pp >> 5], (uint32_t)v);
        if ((uint32_t)(v >> 32)) atomicOr(&wbuf[(pp >> 5) + 1], (uint32_t)(v >> 32));
      }
      p += q + 1u + (uint32_t)b;
    }
    find_prefix();   // includes the barrier that completes the packing
  } else {
    find_prefix();
  }
  if (!s_ok) return;
  const uint64_t S = s_prefix, E = S + (uint64_t)tot;
  if (last && threadIdx.x == 0) {
    *d_nbits = E;
    if ((int64_t)cdiv((int64_t)E, 32) > word_capacity) raise(d_status, GSPARSE_DERR_CAPACITY);
  }
  const int64_t o0 = (int64_t)S + ex;
  // side table: bit offset and preceding index at every chunk start (one 32-bit division per
  // thread; indices < 2^31)
  if (table) {
    // the chunk starts among this thread's codewords: e = e0, e0 + chunk, ... below nv
    const bool p2 = (chunk & (chunk - 1)) == 0;   // power-of-two chunks: masks and shifts
    const uint32_t cm = (uint32_t)chunk - 1u;
    const int cs = __ffs(chunk) - 1;
    const uint32_t e0 = p2 ? (((uint32_t)chunk - ((uint32_t)j0 & cm)) & cm)
                           : (uint32_t)((chunk - (int64_t)((uint32_t)j0 % (uint32_t)chunk)) % chunk);
    if (e0 < (uint32_t)nv) {
      int64_t o = o0;
      uint32_t next = e0;
#pragma unroll
      for (int e = 0; e < KP; ++e) {
        if (e >= nv) break;
        if ((uint32_t)e == next) {
          next += (uint32_t)chunk;
          const int64_t j = j0 + e;
          const int64_t c = (int64_t)(p2 ? (uint32_t)j >> cs : (uint32_t)j / (uint32_t)chunk);
          table[2 * c] = o;
          table[2 * c + 1] = j == 0 ? base - 1 : (int64_t)x[j - 1];
        }
        o += (int64_t)(d[e] >> b) + 1 + b;
      }
    }
  }
  const uint64_t wf = S >> 5, wl = (E - 1) >> 5;
  if ((int64_t)wl >= word_capacity) return;   // capacity raised by the last block
  // the first word is shared with the block before when the block starts inside it, the last
  // with the block after when it ends inside it (the last block's final word is its own)
  const bool head_shared = vb > 0 && (S & 31);
  const bool tail_shared = !last && (E & 31);
  const uint32_t span = (uint32_t)(wl - wf + 1);
  if (fits) {
    // stream word wf + i holds relative bits [32 i - sh, 32 i - sh + 32): a funnel shift of
    // relative words i - 1 and i (span <= nrel + 1, and wbuf[nrel] is zero)
    const uint32_t shf = (uint32_t)(S & 31);
    for (uint32_t i = threadIdx.x; i < span; i += blockDim.x) {
      const uint32_t hi = wbuf[i], lo = i ? wbuf[i - 1] : 0u;
      const uint32_t bits = __funnelshift_l(lo, hi, shf);
      if (i == 0 && head_shared) head[vb] = bits;
      else if (i == span - 1 && tail_shared) tail[vb] = bits;
      else words[wf + i] = bits;
    }
    return;
  }
  // long unary runs: interior words zeroed, then every codeword OR-ed in; the two edge words
  // are gathered in shared memory
  if (threadIdx.x == 0) { s_head = 0u; s_tail = 0u; }
  for (uint64_t w = wf + 1 + threadIdx.x; w < wl; w += blockDim.x) words[w] = 0u;
  __syncthreads();
  int64_t o = o0;
#pragma unroll
  for (int e = 0; e < KP; ++e) {
    if (e >= nv) break;
    Code c;
    c.o = (uint64_t)o;
    c.q = (uint64_t)(d[e] >> b);
    const uint32_t rem = d[e] & ((1u << b) - 1u);
    c.tail = b ? (__brev(rem) >> (32 - b)) << 1 : 0u;
    c.len_tail = 1u + (uint32_t)b;
    const uint64_t w0 = c.o >> 5, w1 = (c.o + c.q + c.len_tail - 1) >> 5;
    for (uint64_t w = w0; w <= w1; ++w) {
      const uint32_t bits = code_bits_in_word(c, w);
      if (!bits) continue;
      if (w == wf) atomicOr(&s_head, bits);
      else if (w == wl) atomicOr(&s_tail, bits);
      else atomicOr(&words[w], bits);
    }
    o += (int64_t)c.q + c.len_tail;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    if (head_shared) head[vb] = s_head; else words[wf] = s_head;
    if (tail_shared) tail[vb] = s_tail; else if (wl != wf) words[wl] = s_tail;
  }
}

// The words shared by two blocks: word (S_j >> 5) for every block j > 0 that starts inside a
// word holds the end of block j - 1 (its tail) and the start of block j (its head).
__global__ void g_fix_kernel(const int64_t* d_begin, const int64_t* d_end, int64_t capacity,
                             int32_t block_codes, const GState* state, const uint64_t* flags,
                             const uint32_t* head, const uint32_t* tail, uint32_t* words,
                             int64_t word_capacity) {
  pdl_begin();
  int64_t lb, len;
  if (!list_bounds(d_begin, d_end, capacity, &lb, &len) || state->abort) return;
  const int64_t nact = cdiv(len, block_codes);
  const int64_t j = 1 + (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= nact) return;
  const uint64_t S = flags[j - 1] & kValMask;   // inclusive total of the blocks before j
  const int64_t w = (int64_t)(S >> 5);
  if ((S & 31) && w < word_capacity) words[w] = tail[j - 1] | head[j];
}

// ---------------------------------------------------------------------------------------------
// decoder

// Word w of the stream, read from a window holding words [base_w, lim_w) (zero outside).
__device__ __forceinline__ uint32_t word_at(const uint32_t* src, int64_t base_w, int64_t lim_w,
                                            int64_t w) {
  return (w >= base_w && w < lim_w) ? src[w - base_w] : 0u;
}

// Decodes `count` codewords from bit t; returns false (and raises) on a corrupt stream.
__device__ bool decode_run(const uint32_t* src, int64_t base_w, int64_t lim_w, uint64_t nbits,
                           uint64_t& t, int64_t& prev, int64_t count, int b, int64_t n_limit,
                           int32_t* out, int32_t* d_status) {
  for (int64_t k = 0; k < count; ++k) {
    uint64_t q = 0;
    for (;;) {
      if (t >= nbits) { raise(d_status, GSPARSE_DERR_CORRUPT_STREAM); return false; }
      const uint32_t sh = (uint32_t)(t & 31);
      const uint32_t avail = 32 - sh;
      const uint32_t v = word_at(src, base_w, lim_w, (int64_t)(t >> 5)) >> sh;
      const uint32_t zeros = ~v & (avail == 32 ? 0xffffffffu : ((1u << avail) - 1u));
      if (zeros) {
        const uint32_t z = (uint32_t)__ffs(zeros) - 1u;
        q += z;
        t += z + 1;
        break;
      }
      q += avail;
      t += avail;
    }
    if (t > nbits) { raise(d_status, GSPARSE_DERR_CORRUPT_STREAM); return false; }
    uint32_t rem = 0;
    if (b > 0) {
      if (t + (uint64_t)b > nbits) { raise(d_status, GSPARSE_DERR_CORRUPT_STREAM); return false; }
      const int64_t w = (int64_t)(t >> 5);
      const uint64_t win = (uint64_t)word_at(src, base_w, lim_w, w) |
                           ((uint64_t)word_at(src, base_w, lim_w, w + 1) << 32);
      const uint32_t raw = (uint32_t)(win >> (t & 31)) & ((1u << b) - 1u);
      rem = __brev(raw) >> (32 - b);
      t += (uint64_t)b;
    }
    if (q > (uint64_t)INT32_MAX) { raise(d_status, GSPARSE_DERR_INDEX_RANGE); return false; }
    const int64_t i = prev + 1 + (int64_t)((q << b) | rem);
    if (i >= n_limit || i > INT32_MAX) { raise(d_status, GSPARSE_DERR_INDEX_RANGE); return false; }
    out[k] = (int32_t)i;
    prev = i;
  }
  return true;
}

// Decodes one codeword from a staged window, word by word (any length): the general path.
__device__ __forceinline__ bool decode_one_local_slow(const uint32_t* sw, uint32_t nb_rel, uint32_t& t,
                                                      uint32_t& q_out, uint32_t& rem_out, int b,
                                                      int32_t* d_status) {
  uint32_t q = 0;
  for (;;) {
    if (t >= nb_rel) { raise(d_status, GSPARSE_DERR_CORRUPT_STREAM); return false; }
    const uint32_t sh = t & 31u;
    const uint32_t zeros = ~(sw[t >> 5] >> sh) & (0xffffffffu >> sh);
    if (zeros) {
      const uint32_t z = (uint32_t)__ffs(zeros) - 1u;
      q += z;
      t += z + 1u;
      break;
    }
    q += 32u - sh;
    t += 32u - sh;
  }
  uint32_t rem = 0;
  if (b > 0) {
    if (t > nb_rel || nb_rel - t < (uint32_t)b) { raise(d_status, GSPARSE_DERR_CORRUPT_STREAM); return false; }
    const uint32_t w = t >> 5;
    const uint64_t win = (uint64_t)sw[w] | ((uint64_t)sw[w + 1] << 32);
    rem = __brev((uint32_t)(win >> (t & 31u)) & ((1u << b) - 1u)) >> (32 - b);
    t += (uint32_t)b;
  } else if (t > nb_rel) {
    raise(d_status, GSPARSE_DERR_CORRUPT_STREAM);
    return false;
  }
  q_out = q;
  rem_out = rem;
  return true;
}

// Decodes `count` codewords of one chunk from a staged window with a 64-bit register bit buffer:
// sw holds stream words [wa, ...) (two zero spares past the window), t0 is the chunk's first bit
// relative to bit 32 * wa and nb_rel the window's end. The buffer holds `avail` unread bits, LSB
// first, and takes the next stream word whenever 32 or fewer remain, so one codeword of up to
// 33 - b bits needs no refill; a longer one is finished word by word from the window. Outputs go
// out four at a time when the chunk's output row is 16-byte aligned. Returns false (and raises)
// on a corrupt stream; on success t0 is the bit after the last codeword.
__device__ bool decode_chunk_buffered(const uint32_t* sw, uint32_t nb_rel, uint32_t wlim, uint32_t& t0,
                                      int64_t& prev64, int count, int b, int64_t n_limit, int32_t* out,
                                      int32_t* d_status) {
  const uint32_t mask = b > 0 ? 0xffffffffu >> (32 - b) : 0u;
  // indices live in [0, 2^31): 32-bit arithmetic; qmax keeps (q << b) below 2^31
  const uint32_t qmax = 0x7fffffffu >> b;
  const uint32_t lim = (uint32_t)(n_limit < (int64_t)INT32_MAX ? n_limit : (int64_t)INT32_MAX);
  uint32_t prev1 = (uint32_t)(prev64 + 1);   // the index after the previous one (>= 0)
  uint32_t wi = t0 >> 5;                      // next word to take into the buffer
  const uint32_t s0 = t0 & 31u;
  uint64_t buf = ((uint64_t)sw[wi] | ((uint64_t)sw[wi + 1] << 32)) >> s0;
  uint32_t avail = 64u - s0;
  wi += 2;
  // one codeword; false on a corrupt stream or an index out of range
  auto next = [&](int32_t& outv) -> bool {
    if (avail <= 32u) {
      if (wi >= wlim) { raise(d_status, GSPARSE_DERR_CORRUPT_STREAM); return false; }   // ran off the window
      buf |= (uint64_t)sw[wi] << avail;
      avail += 32u;
      ++wi;
    }
    const uint32_t lo = (uint32_t)buf;
    uint32_t z;                                // ones before the first zero bit
    if (~lo) z = (uint32_t)__ffs(~lo) - 1u;
    else z = ~(uint32_t)(buf >> 32) ? 31u + (uint32_t)__ffs(~(uint32_t)(buf >> 32)) : 64u;
    uint32_t q, rem = 0;
    const uint32_t used = z + 1u + (uint32_t)b;
    if (used <= avail) {
      q = z;
      if (b > 0) rem = __brev((uint32_t)(buf >> (z + 1u)) & mask) >> (32 - b);
      buf = used == 64u ? 0ull : buf >> used;
      avail -= used;
    } else {
      // a long unary run: finish this codeword from the window, then restart the buffer after it
      uint32_t t = 32u * wi - avail;
      if (t >= nb_rel) { raise(d_status, GSPARSE_DERR_CORRUPT_STREAM); return false; }
      if (!decode_one_local_slow(sw, nb_rel, t, q, rem, b, d_status)) return false;
      wi = t >> 5;
      const uint32_t s = t & 31u;
      buf = ((uint64_t)sw[wi] | ((uint64_t)sw[wi + 1] << 32)) >> s;
      avail = 64u - s;
      wi += 2;
    }
    if (q > qmax) { raise(d_status, GSPARSE_DERR_INDEX_RANGE); return false; }
    const uint32_t i = prev1 + ((q << b) | rem);   // < 2^32: prev1 <= 2^31, gap < 2^31
    if (i >= lim) { raise(d_status, GSPARSE_DERR_INDEX_RANGE); return false; }
    prev1 = i + 1u;
    outv = (int32_t)i;
    return true;
  };
  int k = 0;
  bool ok = true;
  if ((reinterpret_cast<uintptr_t>(out) & 15u) == 0) {
    for (; k + 4 <= count; k += 4) {
      int32_t v0, v1, v2, v3;
      if (!next(v0) || !next(v1) || !next(v2) || !next(v3)) { ok = false; break; }
      *reinterpret_cast<int4*>(out + k) = make_int4(v0, v1, v2, v3);
    }
  }
  for (; ok && k < count; ++k) {
    int32_t v;
    if (!next(v)) { ok = false; break; }
    out[k] = v;
  }
  if (!ok) return false;
  t0 = 32u * wi - avail;
  if (t0 > nb_rel) { raise(d_status, GSPARSE_DERR_CORRUPT_STREAM); return false; }
  prev64 = (int64_t)prev1 - 1;
  return true;
}

// One thread per chunk of codewords, kDecThreads chunks per CTA. The CTA's stream words (a
// contiguous bit range given by the side table) are staged in shared memory when they fit and
// decoded there through a register bit buffer; otherwise the thread reads global memory.
constexpr int kDecThreads = 128;
constexpr int kDecWords = 4096;   // 128 Kbit of staged stream per CTA

__global__ void __launch_bounds__(kDecThreads) g_decode_chunks_kernel(
    const uint32_t* words, int64_t word_capacity, const uint64_t* d_nbits, const int64_t* d_count,
    int64_t capacity, int b, const int64_t* table, int32_t chunk, int64_t n_limit, int32_t* out,
    int32_t* d_status) {
  pdl_begin();
  __shared__ __align__(16) uint32_t sw[kDecWords];
  const int64_t K = *d_count;
  if (K < 0 || K > capacity) {
    if (blockIdx.x == 0 && threadIdx.x == 0) raise(d_status, GSPARSE_DERR_CAPACITY);
    return;
  }
  const uint64_t nbits = *d_nbits;
  if (nbits > (uint64_t)word_capacity * 32u) {
    if (blockIdx.x == 0 && threadIdx.x == 0) raise(d_status, GSPARSE_DERR_CORRUPT_STREAM);
    return;
  }
  const int64_t nch = cdiv(K, chunk);
  const int64_t c0 = (int64_t)blockIdx.x * kDecThreads;
  if (c0 >= nch) return;
  const int64_t c = c0 + threadIdx.x;
  const int64_t c1 = c0 + kDecThreads < nch ? c0 + kDecThreads : nch;  // chunks of this CTA
  // the CTA's bit range, clamped to the stream
  uint64_t ba = (uint64_t)table[2 * c0];
  uint64_t bz = c1 < nch ? (uint64_t)table[2 * c1] : nbits;
  ba = ba < nbits ? ba : nbits;
  bz = bz < nbits ? (bz > ba ? bz : ba) : nbits;
  const int64_t nw = cdiv((int64_t)nbits, 32);
  const int64_t wa = (int64_t)(ba >> 5), wz = cdiv((int64_t)bz, 32) + 3;   // three zero spare words
  const bool staged = wz - wa <= kDecWords;
  if (staged) {
    // the window with 16-byte loads (the stream's words only; zero past its end), all of a
    // thread's loads issued before any is stored
    const int span = (int)(wz - wa);
    const bool vec = (reinterpret_cast<uintptr_t>(words + wa) & 15u) == 0;
    constexpr int kStageIt = kDecWords / (4 * kDecThreads);
    uint4 vbuf[kStageIt];
#pragma unroll
    for (int it = 0; it < kStageIt; ++it) {
      const int k = 4 * (threadIdx.x + it * kDecThreads);
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (k < span) {
        if (vec && wa + k + 3 < nw) {
          v = *reinterpret_cast<const uint4*>(words + wa + k);
        } else {
          v.x = wa + k < nw ? words[wa + k] : 0u;
          v.y = wa + k + 1 < nw ? words[wa + k + 1] : 0u;
          v.z = wa + k + 2 < nw ? words[wa + k + 2] : 0u;
          v.w = wa + k + 3 < nw ? words[wa + k + 3] : 0u;
        }
      }
      vbuf[it] = v;
    }
#pragma unroll
    for (int it = 0; it < kStageIt; ++it) {
      const int k = 4 * (threadIdx.x + it * kDecThreads);
      if (k < span) *reinterpret_cast<uint4*>(sw + k) = vbuf[it];
    }
    __syncthreads();
  }
  if (c >= nch) return;
  uint64_t t = (uint64_t)table[2 * c];
  int64_t prev = table[2 * c + 1];
  const int64_t first = c * chunk;
  const int count = (int)((K - first) < chunk ? (K - first) : chunk);
  if (t > nbits || (staged && (t < ba || t > bz))) {
    raise(d_status, GSPARSE_DERR_CORRUPT_STREAM);   // the side table does not fit the stream
    return;
  }
  bool ok;
  if (staged) {
    // the window's end: this CTA's range, so a chunk cannot run into the next CTA's bits
    uint32_t tl = (uint32_t)(t - 32u * (uint64_t)wa);
    const uint32_t nb_rel = (uint32_t)(bz - 32u * (uint64_t)wa);
    // refills stop two words short of the staged span (the last words are zero spares)
    ok = decode_chunk_buffered(sw, nb_rel, (uint32_t)(wz - wa) - 1u, tl, prev, count, b, n_limit, out + first,
                               d_status);
    t = 32u * (uint64_t)wa + tl;
  } else {
    ok = decode_run(words, 0, nw, nbits, t, prev, count, b, n_limit, out + first, d_status);
  }
  if (ok) {
    const bool last = c + 1 == nch;
    const uint64_t end = last ? nbits : (uint64_t)table[2 * (c + 1)];
    if (t != end || (!last && prev != table[2 * (c + 1) + 1])) raise(d_status, GSPARSE_DERR_CORRUPT_STREAM);
  }
}

__global__ void g_decode_serial_kernel(const uint32_t* words, int64_t word_capacity,
                                       const uint64_t* d_nbits,
                                       const int64_t* d_count, int64_t capacity, int64_t base,
                                       int b, int64_t n_limit, int32_t* out, int32_t* d_status) {
  pdl_begin();
  const int64_t K = *d_count;
  if (K < 0 || K > capacity) { raise(d_status, GSPARSE_DERR_CAPACITY); return; }
  const uint64_t nbits = *d_nbits;
  if (nbits > (uint64_t)word_capacity * 32u) { raise(d_status, GSPARSE_DERR_CORRUPT_STREAM); return; }
  uint64_t t = 0;
  int64_t prev = base - 1;
  if (!decode_run(words, 0, cdiv((int64_t)nbits, 32), nbits, t, prev, K, b, n_limit, out, d_status))
    return;
  if (t != nbits) raise(d_status, GSPARSE_DERR_CORRUPT_STREAM);
}

struct GLayout {
  GState* state;
  uint64_t* flags;
  uint32_t* head;
  uint32_t* tail;
  int64_t nblk;
  size_t zero_bytes;   // state and flags, cleared per call
  size_t bytes;
};

int32_t codes_per_thread(int64_t capacity) { return capacity < kShortList ? kPerShort : kPerLong; }

GLayout g_carve(int64_t capacity, void* ws) {
  GLayout L;
  Carver cv(ws);
  L.nblk = cdiv(capacity > 0 ? capacity : 1, (int64_t)codes_per_thread(capacity) * kCodeThreads);
  L.state = cv.take<GState>(1);
  L.flags = cv.take<uint64_t>(L.nblk);
  L.zero_bytes = cv.off;
  L.head = cv.take<uint32_t>(L.nblk);
  L.tail = cv.take<uint32_t>(L.nblk);
  L.bytes = cv.off + 256;
  return L;
}

}  // namespace
}  // namespace gs

using namespace gs;

extern "C" {

size_t gsparse_golomb_encode_workspace_size(int64_t capacity) {
  if (capacity < 0) return 0;
  return g_carve(capacity, nullptr).bytes;
}

int gsparse_golomb_encode(const int32_t* idx, const int64_t* d_begin, const int64_t* d_end,
                          int64_t capacity, int64_t base, int32_t b, uint32_t* words,
                          int64_t word_capacity, uint64_t* d_nbits, int64_t* chunk_table,
                          int32_t chunk, void* workspace, size_t workspace_bytes,
                          int32_t* d_status, gsparse_stream stream) {
  cudaStream_t st = (cudaStream_t)stream;
  if (capacity < 0 || word_capacity < 0 || !d_end || !d_nbits || (capacity > 0 && (!idx || !words)) ||
      (chunk_table && chunk <= 0))
    return GSPARSE_ERR_INVALID_ARG;
  if (b < 0 || b > 30 || capacity > INT32_MAX) return GSPARSE_ERR_UNSUPPORTED;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return GSPARSE_ERR_WORKSPACE;
  GLayout L = g_carve(capacity, workspace);
  if (workspace_bytes < L.bytes) return GSPARSE_ERR_WORKSPACE;
  if (cudaMemsetAsync(workspace, 0, L.zero_bytes, st) != cudaSuccess) return GSPARSE_ERR_CUDA;
  const int32_t kp = codes_per_thread(capacity);
  if (kp == kPerShort)
    launch(g_encode_kernel<kPerShort>, (unsigned)L.nblk, kCodeThreads, 0, st, idx, d_begin, d_end, capacity,
           base, b, words, word_capacity, d_nbits, chunk_table, chunk, L.state, L.flags, L.head, L.tail,
           d_status);
  else
    launch(g_encode_kernel<kPerLong>, (unsigned)L.nblk, kCodeThreads, 0, st, idx, d_begin, d_end, capacity,
           base, b, words, word_capacity, d_nbits, chunk_table, chunk, L.state, L.flags, L.head, L.tail,
           d_status);
  if (L.nblk > 1)
    launch(g_fix_kernel, (unsigned)cdiv(L.nblk - 1, 256), 256, 0, st, d_begin, d_end, capacity,
           kp * kCodeThreads, L.state, L.flags, L.head, L.tail, words, word_capacity);
  return launch_status();
}

int gsparse_golomb_decode(const uint32_t* words, int64_t word_capacity, const uint64_t* d_nbits,
                          const int64_t* d_count, int64_t capacity, int64_t base, int32_t b,
                          const int64_t* chunk_table, int32_t chunk, int64_t n_limit,
                          int32_t* out_idx, int32_t* d_status, gsparse_stream stream) {
  cudaStream_t st = (cudaStream_t)stream;
  if (capacity < 0 || word_capacity < 0 || !d_nbits || !d_count || (capacity > 0 && (!words || !out_idx)) ||
      (chunk_table && chunk <= 0))
    return GSPARSE_ERR_INVALID_ARG;
  if (b < 0 || b > 30 || capacity > INT32_MAX) return GSPARSE_ERR_UNSUPPORTED;
  if (chunk_table) {
    const int64_t nch = cdiv(capacity > 0 ? capacity : 1, chunk);
    launch(g_decode_chunks_kernel, (unsigned)cdiv(nch, kDecThreads), kDecThreads, 0, st, 
        words, word_capacity, d_nbits, d_count, capacity, b, chunk_table, chunk, n_limit, out_idx,
        d_status);
  } else {
    launch(g_decode_serial_kernel, 1, 1, 0, st, words, word_capacity, d_nbits, d_count, capacity, base,
                                            b, n_limit, out_idx, d_status);
  }
  return launch_status();
}

}  // extern "C"
