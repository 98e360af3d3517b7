// CPU oracle for residual gradient sparsification — TEST INFRASTRUCTURE ONLY.
//
// Plain, slow, single-threaded C++17 statement of what the compression hot path computes.
// Only tests/, the smoke check in __graft_entry__.py and bench.py's CPU-baseline leg may load
// this library. It shares no code, header, table or constant with the CUDA library, and it
// never includes a CUDA header.
//
// Sources (web pages on the method):
//  [AH17]  "Sparse Communication for Distributed Gradient Descent", Aji & Heafield, EMNLP 2017,
//          Abstract: drop the 99% smallest updates by absolute value, exchange sparse
//          matrices, optionally combine with quantisation.
//  [SBC]   "Sparse Binary Compression: Towards Distributed Deep Learning with minimal
//          Communication", Sattler et al., arXiv 1805.08768v1, §II (Communication Delay,
//          Sparse Binarization, Residual Accumulation, Optimal Position Encoding) and
//          Appendix A (Golomb position decoding without shape information).
//  [AHB19] "Combining Global Sparse Gradients with Local Gradients in Distributed Neural
//          Network Training", Aji, Heafield & Bogoychev, EMNLP-IJCNLP 2019, Abstract.
//
// Where the pages leave a step open, the plainest reading is taken and marked READING.
// Compile with -ffp-contract=off: every fp32 operation below is one IEEE round-to-nearest op.
//
// Status codes returned by every entry point: 0 ok, 1 invalid argument, 2 output capacity too
// small, 3 corrupt bitstream, 4 index out of range.

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <numeric>
#include <vector>

namespace {

constexpr int kOk = 0, kBadArg = 1, kCapacity = 2, kCorrupt = 3, kRange = 4;

// Order key of a float by magnitude: the IEEE bit pattern with the sign bit cleared. For finite
// values, a larger key means a larger |x|; +0 and -0 share key 0. [AH17] Abstract ranks updates
// "by absolute value"; READING: the bit pattern is that order (NaN keys sort above +inf).
uint32_t mag_key(float x) {
  uint32_t u;
  std::memcpy(&u, &x, sizeof u);
  return u & 0x7fffffffu;
}

// Number kept in a segment of n_s entries for keep fraction num/den: ceil(n_s*num/den), computed
// exactly. [AH17] Abstract fixes the fraction (drop 99% => keep 1/100); READING: ceil, so every
// non-empty segment sends at least one entry when num > 0.
int64_t kept_count(int64_t n_s, int64_t num, int64_t den) {
  if (n_s <= 0 || num <= 0) return 0;
  unsigned __int128 prod = (unsigned __int128)n_s * (unsigned __int128)num;
  unsigned __int128 k = (prod + (unsigned __int128)(den - 1)) / (unsigned __int128)den;
  return k > (unsigned __int128)n_s ? n_s : (int64_t)k;
}

// The k largest of `cand` under the total order (key descending, index ascending), returned in
// ascending index order. Each entry is packed as (~key << 32 | index) so that ascending order of
// the packed integer is exactly that total order ("largest by magnitude, ties to the lower
// index"); std::nth_element then places the k smallest packed values first.
std::vector<int64_t> top_k_packed(std::vector<uint64_t>& packed, int64_t k) {
  if (k > (int64_t)packed.size()) k = (int64_t)packed.size();
  if (k < (int64_t)packed.size()) std::nth_element(packed.begin(), packed.begin() + k, packed.end());
  std::vector<int64_t> out(k);
  for (int64_t j = 0; j < k; ++j) out[j] = (int64_t)(uint32_t)(packed[j] & 0xffffffffu);
  std::sort(out.begin(), out.end());
  return out;
}

uint64_t pack(uint32_t key, int64_t index) { return ((uint64_t)(~key) << 32) | (uint64_t)(uint32_t)index; }

template <class KeyFn>
std::vector<int64_t> top_k(const std::vector<int64_t>& cand, int64_t k, KeyFn key) {
  std::vector<uint64_t> packed(cand.size());
  for (size_t j = 0; j < cand.size(); ++j) packed[j] = pack(key(cand[j]), cand[j]);
  return top_k_packed(packed, k);
}

// Fixed-order fp64 sum of the member entries of a list. READING: the pages give no summation
// order, but the sent mean decides the new residual bit for bit, so the order is fixed here:
// the list is cut into consecutive blocks of 256 positions; each block adds its members left to
// right in fp64 starting from +0.0; the block sums are then combined pairwise level by level
// (element m of the next level = element 2m + element 2m+1; an unpaired last element moves up
// unchanged) until one value remains. An empty list sums to +0.0.
double ordered_sum(const std::vector<double>& v, const std::vector<char>& member) {
  std::vector<double> level;
  for (size_t c = 0; c < v.size(); c += 256) {
    double s = 0.0;
    size_t end = std::min(v.size(), c + 256);
    for (size_t j = c; j < end; ++j)
      if (member[j]) s += v[j];
    level.push_back(s);
  }
  if (level.empty()) return 0.0;
  while (level.size() > 1) {
    std::vector<double> next;
    for (size_t a = 0; a + 1 < level.size(); a += 2) next.push_back(level[a] + level[a + 1]);
    if (level.size() % 2 == 1) next.push_back(level.back());
    level.swap(next);
  }
  return level[0];
}

// Mean of the members: (float)(sum / count) with one fp64 division and one rounding to fp32;
// no members => +0.0f.
float ordered_mean(const std::vector<double>& v, const std::vector<char>& member) {
  int64_t count = 0;
  for (char m : member) count += m ? 1 : 0;
  if (count == 0) return 0.0f;
  return (float)(ordered_sum(v, member) / (double)count);
}

bool valid_segments(int64_t n, const int64_t* seg, int32_t T) {
  if (T < 1 || seg == nullptr || seg[0] != 0 || seg[T] != n) return false;
  for (int32_t s = 0; s < T; ++s)
    if (seg[s + 1] < seg[s]) return false;
  return true;
}

}  // namespace

extern "C" {

int64_t orc_k_for(int64_t n_s, int64_t num, int64_t den) { return kept_count(n_s, num, den); }

// b* = 1 + floor(log2(log(phi - 1) / log(1 - p))), phi the golden ratio: the Golomb parameter for
// position coding at density p ([SBC] §II Optimal Position Encoding names Golomb coding of the
// distances; the formula for b* is the workload's stated rule).
int32_t orc_golomb_b_star(double p) {
  if (!(p > 0.0) || !(p < 1.0)) return -1;
  const double phi = (1.0 + std::sqrt(5.0)) / 2.0;
  return 1 + (int32_t)std::floor(std::log2(std::log(phi - 1.0) / std::log(1.0 - p)));
}

// Warm-up schedule ([SBC] Appendix A: sparsity raised exponentially from 25% to 0.1% kept during
// the first epochs). READING: keep(t) = start * (end/start)^(t/T) for t < T, end afterwards;
// returned as a numerator over den, rounded to nearest and clamped to [1, den].
int64_t orc_warmup_keep_num(int64_t t, int64_t T, double start, double end, int64_t den) {
  if (den <= 0 || t < 0 || T < 0 || !(start > 0.0) || !(start <= 1.0) || !(end > 0.0) || !(end <= 1.0))
    return -1;
  double keep = end;
  if (T > 0 && t < T) keep = start * std::exp(std::log(end / start) * (double)t / (double)T);
  int64_t num = (int64_t)std::llround(keep * (double)den);
  return std::min<int64_t>(std::max<int64_t>(num, 1), den);
}

// Residual top-k ([AH17] Abstract; [SBC] §II Residual Accumulation).
//   acc_i = fl(g_i + r_i)                                   (fp32, round to nearest even)
//   per segment s: send the k_s entries of largest |acc| (ties to the lower index), ascending;
//   r_i <- 0 for the sent entries and acc_i for all others.
// seg: T+1 offsets (seg[0] = 0, seg[T] = n); one segment = global selection, one per tensor =
// per-tensor selection (READING: the pages allow both). num = 0 accumulates only ([SBC] §II
// Communication Delay: updates are summed locally between exchanges).
// Outputs: out_idx/out_val in segment order, out_off[T+1] exclusive offsets.
int orc_residual_topk(const float* g, float* r, int64_t n, const int64_t* seg, int32_t T,
                      int64_t num, int64_t den, int32_t* out_idx, float* out_val, int64_t* out_off,
                      int64_t capacity) {
  if (n < 0 || n > INT32_MAX || !valid_segments(n, seg, T) || num < 0 || den <= 0 || num > den)
    return kBadArg;
  std::vector<float> acc(n);
  for (int64_t i = 0; i < n; ++i) acc[i] = g[i] + r[i];
  auto key = [&](int64_t i) { return mag_key(acc[i]); };

  int64_t total = 0;
  for (int32_t s = 0; s < T; ++s) total += kept_count(seg[s + 1] - seg[s], num, den);
  if (total > capacity) return kCapacity;

  int64_t o = 0;
  out_off[0] = 0;
  for (int64_t i = 0; i < n; ++i) r[i] = acc[i];
  for (int32_t s = 0; s < T; ++s) {
    std::vector<uint64_t> packed(seg[s + 1] - seg[s]);
    for (int64_t i = seg[s]; i < seg[s + 1]; ++i) packed[i - seg[s]] = pack(key(i), i);
    std::vector<int64_t> sent = top_k_packed(packed, kept_count(seg[s + 1] - seg[s], num, den));
    for (int64_t i : sent) {
      out_idx[o] = (int32_t)i;
      out_val[o] = acc[i];
      r[i] = 0.0f;
      ++o;
    }
    out_off[s + 1] = o;
  }
  return kOk;
}

// Residual top-k with momentum correction and momentum masking ([SBC] §II "Momentum Correction,
// Warm-up Training and Momentum Masking" and Appendix A: the momentum-corrected gradient is added
// to the residual; the momentum of the entries that were sent is set to zero). READING of the
// arithmetic, one fp32 operation at a time:
//   v_i = fl(fl(m * u_i) + g_i)        the momentum-corrected gradient; u_i <- v_i
//   acc_i = fl(r_i + v_i)              then the residual top-k above on acc
//   for the sent i: r_i <- 0 and u_i <- 0 (masking); all other entries keep r_i = acc_i.
// With m = 0 this is orc_residual_topk plus u <- g with the sent entries zeroed.
int orc_residual_topk_momentum(const float* g, float* u, float m, float* r, int64_t n,
                               const int64_t* seg, int32_t T, int64_t num, int64_t den,
                               int32_t* out_idx, float* out_val, int64_t* out_off,
                               int64_t capacity) {
  if (n < 0 || n > INT32_MAX || !valid_segments(n, seg, T) || num < 0 || den <= 0 || num > den)
    return kBadArg;
  std::vector<float> v(n);
  for (int64_t i = 0; i < n; ++i) {
    const float mu = m * u[i];
    v[i] = mu + g[i];
  }
  const int st = orc_residual_topk(v.data(), r, n, seg, T, num, den, out_idx, out_val, out_off,
                                   capacity);
  if (st != kOk) return st;
  for (int64_t i = 0; i < n; ++i) u[i] = v[i];
  for (int64_t j = 0; j < out_off[T]; ++j) u[out_idx[j]] = 0.0f;
  return kOk;
}

// 2-bit quantisation of a kept list ([AH17] Abstract: sparsification "can be combined with
// quantization"). READING of the rule: every positive kept value becomes m+ = mean of the positive
// kept values, every negative one m- = mean of the negative kept values (a negative number), a
// kept +-0 stays +0 and counts in neither mean. Bit j of sign_bits (word j/32, bit j%32) is set iff
// val_j < 0. Means use the fixed-order sum above.
// residual (nullable): r[idx_j] <- fl(val_j - q_j), the error fed back ([SBC] §II Residual
// Accumulation). write_dequantized: val_j <- q_j.
int orc_quantize(const int32_t* idx, float* val, int64_t K, float* residual, int64_t n,
                 uint32_t* sign_bits, float* means, int32_t write_dequantized) {
  if (K < 0) return kBadArg;
  std::vector<double> v(K);
  std::vector<char> pos(K), neg(K);
  for (int64_t j = 0; j < K; ++j) {
    v[j] = (double)val[j];
    pos[j] = val[j] > 0.0f;
    neg[j] = val[j] < 0.0f;
  }
  const float mpos = ordered_mean(v, pos);
  const float mneg = ordered_mean(v, neg);
  means[0] = mpos;
  means[1] = mneg;
  for (int64_t w = 0; w < (K + 31) / 32; ++w) sign_bits[w] = 0u;
  for (int64_t j = 0; j < K; ++j) {
    const float q = pos[j] ? mpos : (neg[j] ? mneg : 0.0f);
    if (neg[j]) sign_bits[j / 32] |= 1u << (j % 32);
    if (residual) {
      if (idx[j] < 0 || idx[j] >= n) return kRange;
      residual[idx[j]] = val[j] - q;
    }
    if (write_dequantized) val[j] = q;
  }
  return kOk;
}

// Sparse binarisation ([SBC] §II Sparse Binarization). READING: per segment, P = the k_s largest
// positive entries of acc = fl(g + r) (by value, ties to the lower index), N = the k_s most
// negative entries (by |value|); each may hold fewer than k_s entries; zeros are in neither.
// mu+ = mean of P, mu- = mean of |N| (fixed-order sums). The set with the larger mean is sent
// (ties to P), every entry of it replaced by the signed mean; both empty => nothing sent.
// Residual: r_i <- fl(acc_i - m_s) for the sent entries, acc_i for all others.
// Outputs: indices ascending per segment, compacted; out_off[T+1]; mean[s] = signed mean
// (+0.0f when nothing is sent); out_val (nullable) = the signed mean per sent entry.
int orc_binarize(const float* g, float* r, int64_t n, const int64_t* seg, int32_t T, int64_t num,
                 int64_t den, int32_t* out_idx, float* out_val, float* mean, int64_t* out_off,
                 int64_t capacity) {
  if (n < 0 || n > INT32_MAX || !valid_segments(n, seg, T) || num < 0 || den <= 0 || num > den)
    return kBadArg;
  std::vector<float> acc(n);
  for (int64_t i = 0; i < n; ++i) acc[i] = g[i] + r[i];
  auto key = [&](int64_t i) { return mag_key(acc[i]); };

  int64_t o = 0;
  out_off[0] = 0;
  for (int64_t i = 0; i < n; ++i) r[i] = acc[i];
  for (int32_t s = 0; s < T; ++s) {
    const int64_t k = kept_count(seg[s + 1] - seg[s], num, den);
    std::vector<int64_t> positives, negatives;
    for (int64_t i = seg[s]; i < seg[s + 1]; ++i) {
      if (acc[i] > 0.0f) positives.push_back(i);
      if (acc[i] < 0.0f) negatives.push_back(i);
    }
    std::vector<int64_t> P = top_k(positives, k, key);
    std::vector<int64_t> N = top_k(negatives, k, key);
    std::vector<double> vp, vn;
    for (int64_t i : P) vp.push_back((double)acc[i]);
    for (int64_t i : N) vn.push_back(-(double)acc[i]);
    const float mu_pos = ordered_mean(vp, std::vector<char>(vp.size(), 1));
    const float mu_neg = ordered_mean(vn, std::vector<char>(vn.size(), 1));
    const bool take_pos = !P.empty() && mu_pos >= mu_neg;
    const bool take_neg = !take_pos && !N.empty();
    const std::vector<int64_t>& chosen = take_pos ? P : N;
    const float m = take_pos ? mu_pos : (take_neg ? -mu_neg : 0.0f);
    mean[s] = m;
    if (take_pos || take_neg) {
      if (o + (int64_t)chosen.size() > capacity) return kCapacity;
      for (int64_t i : chosen) {
        out_idx[o] = (int32_t)i;
        if (out_val) out_val[o] = m;
        r[i] = acc[i] - m;
        ++o;
      }
    }
    out_off[s + 1] = o;
  }
  return kOk;
}

// Sparse binarisation, the magnitude-first reading ([SBC] §II Sparse Binarization: only the
// largest-magnitude fraction p is retained, its nonzero values are represented by one mean, and
// the sign with the larger absolute mean decides which values remain). READING, per segment:
//   S = the k_s entries of largest |acc| (ties to the lower index), ascending;
//   mu+ = mean of the positive members of S, mu- = mean of |acc| over its negative members, both
//   with the fixed-order sum over the positions of S (blocks of 256 positions, members only);
//   send the positive members with +mu+ if mu+ >= mu- (and any exist), else the negative members
//   with -mu-; residual <- fl(acc - m) on the sent entries and acc everywhere else (the unsent
//   members of S keep their value in the residual).
int orc_binarize_magnitude(const float* g, float* r, int64_t n, const int64_t* seg, int32_t T,
                           int64_t num, int64_t den, int32_t* out_idx, float* out_val, float* mean,
                           int64_t* out_off, int64_t capacity) {
  if (n < 0 || n > INT32_MAX || !valid_segments(n, seg, T) || num < 0 || den <= 0 || num > den)
    return kBadArg;
  std::vector<float> acc(n);
  for (int64_t i = 0; i < n; ++i) acc[i] = g[i] + r[i];
  for (int64_t i = 0; i < n; ++i) r[i] = acc[i];
  int64_t o = 0;
  out_off[0] = 0;
  for (int32_t s = 0; s < T; ++s) {
    std::vector<uint64_t> packed(seg[s + 1] - seg[s]);
    for (int64_t i = seg[s]; i < seg[s + 1]; ++i) packed[i - seg[s]] = pack(mag_key(acc[i]), i);
    const std::vector<int64_t> S = top_k_packed(packed, kept_count(seg[s + 1] - seg[s], num, den));
    std::vector<double> vp(S.size()), vn(S.size());
    std::vector<char> isp(S.size()), isn(S.size());
    for (size_t j = 0; j < S.size(); ++j) {
      const float x = acc[S[j]];
      vp[j] = (double)x;
      vn[j] = -(double)x;
      isp[j] = x > 0.0f;
      isn[j] = x < 0.0f;
    }
    const int64_t np = std::count(isp.begin(), isp.end(), 1);
    const int64_t nn = std::count(isn.begin(), isn.end(), 1);
    const float mu_pos = ordered_mean(vp, isp);
    const float mu_neg = ordered_mean(vn, isn);
    const bool take_pos = np > 0 && mu_pos >= mu_neg;
    const bool take_neg = !take_pos && nn > 0;
    const float m = take_pos ? mu_pos : (take_neg ? -mu_neg : 0.0f);
    mean[s] = m;
    for (size_t j = 0; j < S.size(); ++j) {
      if (!((take_pos && isp[j]) || (take_neg && isn[j]))) continue;
      if (o >= capacity) return kCapacity;
      const int64_t i = S[j];
      out_idx[o] = (int32_t)i;
      if (out_val) out_val[o] = m;
      r[i] = acc[i] - m;
      ++o;
    }
    out_off[s + 1] = o;
  }
  return kOk;
}

// Golomb position coding ([SBC] §II Optimal Position Encoding: the distances between nonzero
// positions are Golomb coded; Appendix A: decoding needs no shape information).
// READING of the code: gaps d_0 = i_0 - base, d_j = i_j - i_{j-1} - 1 (>= 0); with M = 2^b,
// q = d >> b and rem = d mod M, the codeword is q one-bits, one zero-bit, then rem in b bits,
// most significant first. Stream bit t lives in word t/32 at bit t%32; unused tail bits are 0.
// chunk_table (nullable): for codeword c*chunk, the pair (bit offset, preceding index), the
// preceding index of codeword 0 being base - 1.
// Returns the status; *nbits receives the stream length in bits.
int orc_golomb_encode(const int32_t* idx, int64_t K, int64_t base, int32_t b, uint32_t* words,
                      int64_t word_capacity, int64_t* chunk_table, int64_t chunk, uint64_t* nbits) {
  if (K < 0 || b < 0 || b > 30 || (chunk_table && chunk <= 0)) return kBadArg;
  std::vector<uint8_t> bits;
  int64_t prev = base - 1;
  for (int64_t j = 0; j < K; ++j) {
    const int64_t d = (int64_t)idx[j] - prev - 1;
    if (d < 0) return kRange;
    if (chunk_table && j % chunk == 0) {
      chunk_table[2 * (j / chunk)] = (int64_t)bits.size();
      chunk_table[2 * (j / chunk) + 1] = prev;
    }
    const int64_t q = d >> b, rem = d & ((int64_t(1) << b) - 1);
    for (int64_t t = 0; t < q; ++t) bits.push_back(1);
    bits.push_back(0);
    for (int32_t t = b - 1; t >= 0; --t) bits.push_back((uint8_t)((rem >> t) & 1));
    prev = idx[j];
  }
  const int64_t nw = ((int64_t)bits.size() + 31) / 32;
  if (nw > word_capacity) return kCapacity;
  for (int64_t w = 0; w < nw; ++w) words[w] = 0u;
  for (size_t t = 0; t < bits.size(); ++t)
    if (bits[t]) words[t / 32] |= 1u << (t % 32);
  *nbits = bits.size();
  return kOk;
}

// Inverse of orc_golomb_encode: reads exactly K codewords from the first nbits bits. A codeword
// that runs past nbits, or bits left over after K codewords, is a corrupt stream; an index at or
// above n_limit is out of range.
int orc_golomb_decode(const uint32_t* words, uint64_t nbits, int64_t K, int64_t base, int32_t b,
                      int64_t n_limit, int32_t* out_idx) {
  if (K < 0 || b < 0 || b > 30) return kBadArg;
  auto bit = [&](uint64_t t) { return (words[t / 32] >> (t % 32)) & 1u; };
  uint64_t t = 0;
  int64_t prev = base - 1;
  for (int64_t j = 0; j < K; ++j) {
    int64_t q = 0;
    for (;;) {
      if (t >= nbits) return kCorrupt;
      if (bit(t++) == 0) break;
      ++q;
    }
    int64_t rem = 0;
    for (int32_t u = 0; u < b; ++u) {
      if (t >= nbits) return kCorrupt;
      rem = (rem << 1) | bit(t++);
    }
    const int64_t i = prev + 1 + ((q << b) | rem);
    if (i >= n_limit) return kRange;
    out_idx[j] = (int32_t)i;
    prev = i;
  }
  return t == nbits ? kOk : kCorrupt;
}

// Sum of W workers' sparse updates ([AHB19] Abstract: the compressed global gradient; [SBC] §I:
// the master model sums the clients' updates). READING of the order: G starts at +0.0 and adds
// worker 0's values, then worker 1's, ..., one fp32 add per entry. Worker w's list: counts[w]
// ascending distinct indices, values vals[w] (or, when vals[w] is null, uniform[w] for every
// entry, the binarised case). dense (nullable) receives G; merged_* (nullable) receive the
// ascending union of the indices with their G values.
int orc_scatter_accumulate(int32_t W, const int32_t* const* idxs, const float* const* vals,
                           const float* uniform, const int64_t* counts, int64_t n, float* dense,
                           int32_t* merged_idx, float* merged_val, int64_t* merged_count,
                           int64_t merged_capacity) {
  if (W < 1 || n < 0) return kBadArg;
  std::vector<float> G(n, 0.0f);
  std::vector<char> touched(n, 0);
  for (int32_t w = 0; w < W; ++w) {
    for (int64_t j = 0; j < counts[w]; ++j) {
      const int64_t i = idxs[w][j];
      if (i < 0 || i >= n || (j > 0 && idxs[w][j - 1] >= i)) return kRange;
      G[i] = G[i] + (vals[w] ? vals[w][j] : uniform[w]);
      touched[i] = 1;
    }
  }
  if (dense)
    for (int64_t i = 0; i < n; ++i) dense[i] = G[i];
  if (merged_count) {
    int64_t u = 0;
    for (int64_t i = 0; i < n; ++i) {
      if (!touched[i]) continue;
      if (u >= merged_capacity) return kCapacity;
      merged_idx[u] = (int32_t)i;
      merged_val[u] = G[i];
      ++u;
    }
    *merged_count = u;
  }
  return kOk;
}

// Combination of the global sparse sum with the local uncompressed gradient ([AHB19] Abstract).
// READING: mode 0 (sum): out_i = fl(fl(alpha*G_i) + fl(beta*L_i)). Mode 1 (partial): on the
// worker's own sent entries G_i is first replaced by fl(G_i - s_i), so its own contribution comes
// only from the local gradient.
int orc_combine_local(const float* G, const float* L, float* out, int64_t n, float alpha,
                      float beta, int32_t mode, const int32_t* own_idx, const float* own_val,
                      int64_t own_count) {
  if (n < 0 || (mode != 0 && mode != 1)) return kBadArg;
  std::vector<float> g(G, G + n);
  if (mode == 1) {
    for (int64_t j = 0; j < own_count; ++j) {
      const int64_t i = own_idx[j];
      if (i < 0 || i >= n) return kRange;
      g[i] = g[i] - own_val[j];
    }
  }
  for (int64_t i = 0; i < n; ++i) {
    const float a = alpha * g[i];
    const float b = beta * L[i];
    out[i] = a + b;
  }
  return kOk;
}

}  // extern "C"
