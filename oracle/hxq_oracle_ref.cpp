// Plain C++ oracle of the HXQ HelixLinear forward -- TEST INFRASTRUCTURE.
//
// A second, independently written CPU oracle beside oracle/hxq_oracle.py
// (numpy): the tests check that the two agree, decode bit for bit and the
// forward to float64 rounding. Only the tests load it; the CUDA library
// never includes, links or calls it, and the two share no code.
//
// What it computes, as plain loops in the definition's order:
//  * scalar mode: W[n][k] = codebook[indices[n*K + k]] (Zamba2-1.2B-HXQ model
//    card, "What is HelixCode?": 256-entry fp32 codebook, one uint8 index per
//    weight);
//  * 2D mode: pair g = n*K/2 + k/2 of the row-major pair stream has a 12-bit
//    index; group g/2 of the index bytes is the little-endian 24-bit word
//    b0 | b1<<8 | b2<<16 whose low 12 bits index the even pair and high 12
//    bits the odd one; W[n][k] = codebook[2*index + (k & 1)] (HXQ whitepaper,
//    method section: 2D VQ paragraph and "12-bit index packing");
//  * sidecar: W[p / K][p % K] = value for every (p, value) (HXQ whitepaper,
//    method section, "Sidecar outlier correction", read as replacement);
//  * y[m][n] = sum over k, in k order, of double(x[m][k]) * double(W[n][k]),
//    x widened exactly from its bf16 bits; s[m][n] the same sum of absolute
//    values (the tolerance scale).
// The encoder functions below follow the same readings as the numpy encoder
// oracle: fp32 distance decisions with ties to the lowest index, the exact
// mean of a cluster's fp32 coordinates rounded once to fp32 (nearest even)
// with empty clusters kept, a strict threshold on |w - w_hat| that stores the
// weight itself.
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <numeric>
#include <thread>
#include <vector>

namespace {

double bf16_to_double(uint16_t bits) {
  const uint32_t u = (uint32_t)bits << 16;
  float f;
  std::memcpy(&f, &u, sizeof f);
  return (double)f;
}

// Decoded weight W[n][k] before the sidecar (fp32).
float decode_one(int mode, const float* codebook, const uint8_t* indices, int K, int n, int k) {
  if (mode == 0) return codebook[indices[(int64_t)n * K + k]];
  const int64_t g = (int64_t)n * (K / 2) + k / 2;  // pair
  const int64_t grp = g / 2;                        // 3-byte group
  const uint32_t word = (uint32_t)indices[3 * grp] | ((uint32_t)indices[3 * grp + 1] << 8) |
                        ((uint32_t)indices[3 * grp + 2] << 16);
  const uint32_t e = (g % 2 == 0) ? (word & 0xFFFu) : (word >> 12);
  return codebook[2 * e + (k % 2)];
}

}  // namespace

extern "C" {

// Decoded weights W [N][K] (fp32). Returns 0, or -1 for an unknown mode, a
// bad shape, or a sidecar position out of range or repeated.
int oracle_decode(int mode, const float* codebook, const uint8_t* indices, const int64_t* sidecar_pos,
                  const float* sidecar_val, int64_t n_sidecar, int N, int K, float* W) {
  if (N < 1 || K < 1) return -1;
  if (mode != 0 && mode != 1) return -1;
  if (mode == 1 && K % 4 != 0) return -1;
  const int64_t NK = (int64_t)N * K;
  for (int n = 0; n < N; ++n)
    for (int k = 0; k < K; ++k) W[(int64_t)n * K + k] = decode_one(mode, codebook, indices, K, n, k);
  std::vector<char> seen(n_sidecar > 0 ? (size_t)NK : 0, 0);
  for (int64_t i = 0; i < n_sidecar; ++i) {
    const int64_t p = sidecar_pos[i];
    if (p < 0 || p >= NK || seen[(size_t)p]) return -1;
    seen[(size_t)p] = 1;
    W[p] = sidecar_val[i];
  }
  return 0;
}

// y[m][n] and s[m][n] (float64) for x [M][K] given as bf16 bits.
void oracle_forward(const uint16_t* x_bits, const float* W, int M, int N, int K, double* y, double* s) {
  for (int m = 0; m < M; ++m) {
    for (int n = 0; n < N; ++n) {
      double acc = 0.0, mag = 0.0;
      for (int k = 0; k < K; ++k) {
        const double xv = bf16_to_double(x_bits[(int64_t)m * K + k]);
        const double wv = (double)W[(int64_t)n * K + k];
        acc += xv * wv;
        mag += (xv < 0 ? -xv : xv) * (wv < 0 ? -wv : wv);
      }
      y[(int64_t)m * N + n] = acc;
      s[(int64_t)m * N + n] = mag;
    }
  }
}

// The whole path for output rows [r0, r1) of a layer, for timing the oracle
// on the host's cores: each row is decoded (sidecar entries of the row
// replace their weights), then y[m][n - r0] = sum over k, in k order, of
// double(x[m][k]) * double(W[n][k]) -- the arithmetic of oracle_decode and
// oracle_forward, row by row. `threads` std::threads split the rows in
// contiguous blocks. Returns 0, or -1 for a bad argument (positions are not
// checked for repeats here).
int oracle_forward_rows(int mode, const float* codebook, const uint8_t* indices, const int64_t* sidecar_pos,
                        const float* sidecar_val, int64_t n_sidecar, int N, int K, const uint16_t* x_bits, int M,
                        int r0, int r1, int threads, double* y) {
  if (N < 1 || K < 1 || M < 1 || r0 < 0 || r1 > N || r0 >= r1 || threads < 1) return -1;
  if (mode != 0 && mode != 1) return -1;
  if (mode == 1 && K % 4 != 0) return -1;
  // sidecar entries in position order, so that a row finds its own
  std::vector<int64_t> order((size_t)n_sidecar);
  std::iota(order.begin(), order.end(), (int64_t)0);
  std::sort(order.begin(), order.end(), [&](int64_t a, int64_t b) { return sidecar_pos[a] < sidecar_pos[b]; });
  const int64_t NK = (int64_t)N * K;
  for (int64_t i = 0; i < n_sidecar; ++i)
    if (sidecar_pos[i] < 0 || sidecar_pos[i] >= NK) return -1;
  const int R = r1 - r0;
  auto work = [&](int a, int b) {
    std::vector<double> w((size_t)K);
    for (int n = a; n < b; ++n) {
      for (int k = 0; k < K; ++k) w[(size_t)k] = (double)decode_one(mode, codebook, indices, K, n, k);
      auto it = std::lower_bound(order.begin(), order.end(), (int64_t)n * K,
                                 [&](int64_t e, int64_t v) { return sidecar_pos[e] < v; });
      for (; it != order.end() && sidecar_pos[*it] < (int64_t)(n + 1) * K; ++it)
        w[(size_t)(sidecar_pos[*it] - (int64_t)n * K)] = (double)sidecar_val[*it];
      for (int m = 0; m < M; ++m) {
        double acc = 0.0;
        for (int k = 0; k < K; ++k) acc += bf16_to_double(x_bits[(int64_t)m * K + k]) * w[(size_t)k];
        y[(int64_t)m * R + (n - r0)] = acc;
      }
    }
  };
  const int T = std::min(threads, R);
  std::vector<std::thread> pool;
  for (int t = 1; t < T; ++t) pool.emplace_back(work, r0 + (int)((int64_t)R * t / T), r0 + (int)((int64_t)R * (t + 1) / T));
  work(r0, r0 + R / T);
  for (auto& th : pool) th.join();
  return 0;
}

// ---- encoder side (HXQ whitepaper, method section: "Per-tensor k-means",
// "Index assignment", "Sidecar outlier correction"), as plain loops.

// Nearest of k centroids [k][dim] for each of n points [n][dim]: fp32
// distance |p - c| (dim 1) or dx*dx + dy*dy (dim 2), every operation rounded
// to fp32 as written (compiled without contraction); a strictly smaller
// distance wins, so ties keep the lowest index.
static void oracle_assign_range(const float* points, int64_t i0, int64_t i1, int dim, const float* centroids, int k,
                         int32_t* labels) {
  for (int64_t i = i0; i < i1; ++i) {
    float best = 0.f;
    int bi = -1;
    for (int e = 0; e < k; ++e) {
      float d;
      if (dim == 1) {
        const float diff = points[i] - centroids[e];
        d = diff < 0.f ? -diff : diff;
      } else {
        const float dx = points[2 * i] - centroids[2 * e];
        const float dy = points[2 * i + 1] - centroids[2 * e + 1];
        const float xx = dx * dx;
        const float yy = dy * dy;
        d = xx + yy;
      }
      if (bi < 0 || d < best) {
        best = d;
        bi = e;
      }
    }
    labels[i] = bi;
  }
}

void oracle_assign(const float* points, int64_t n, int dim, const float* centroids, int k, int32_t* labels) {
  oracle_assign_range(points, 0, n, dim, centroids, k, labels);
}

// oracle_assign on `threads` host threads, each on a contiguous block of
// points (the same decisions; only the work is split).
void oracle_assign_threads(const float* points, int64_t n, int dim, const float* centroids, int k,
                           int32_t* labels, int threads) {
  const int T = (int)std::max<int64_t>(1, std::min<int64_t>(threads, n));
  std::vector<std::thread> pool;
  for (int t = 1; t < T; ++t)
    pool.emplace_back(oracle_assign_range, points, n * t / T, n * (t + 1) / T, dim, centroids, k, labels);
  oracle_assign_range(points, 0, n / T, dim, centroids, k, labels);
  for (auto& th : pool) th.join();
}

}  // extern "C"

namespace {

// The exact sum of fp32 values as a signed integer in units of 2^-149
// (every fp32 value is a multiple of 2^-149; the largest is below 2^128, so
// 277 bits plus the count's bits), kept as base-2^32 digits in int64 words
// that absorb carries until the end.
struct ExactSum {
  static constexpr int kDigits = 11;  // 352 bits
  int64_t d[kDigits] = {};
  void add(float v) {
    uint32_t bits;
    std::memcpy(&bits, &v, sizeof bits);
    const int ef = (int)((bits >> 23) & 0xFF);
    uint64_t m = bits & 0x7FFFFFu;
    int shift = 0;  // position of m's last bit above 2^-149
    if (ef != 0) {
      m |= 0x800000u;
      shift = ef - 1;
    }
    if (m == 0) return;
    const int neg = (int)(bits >> 31);
    const unsigned __int128 wide = (unsigned __int128)m << (shift % 32);  // under 2^56
    const int i = shift / 32;
    const int64_t lo = (int64_t)(uint64_t)(wide & 0xFFFFFFFFu);
    const int64_t hi = (int64_t)(uint64_t)(wide >> 32);
    d[i] += neg ? -lo : lo;
    d[i + 1] += neg ? -hi : hi;
  }
};

// The fp32 value nearest to (sum x 2^-149) / count, ties to even: carries
// resolved, magnitude divided by count digit by digit from the top, then
// 24 significant bits kept with the rest deciding the rounding.
float exact_mean_f32(const ExactSum& s, int64_t count) {
  int64_t w[ExactSum::kDigits];
  for (int i = 0; i < ExactSum::kDigits; ++i) w[i] = s.d[i];
  for (int i = 0; i + 1 < ExactSum::kDigits; ++i) {  // carries: every digit into [0, 2^32)
    const int64_t carry = w[i] >> 32;                  // floor division (arithmetic shift)
    w[i] -= carry * ((int64_t)1 << 32);
    w[i + 1] += carry;
  }
  const bool neg = w[ExactSum::kDigits - 1] < 0;
  uint32_t mag[ExactSum::kDigits];
  if (neg) {  // two's complement negation of the digit string
    uint64_t borrow = 1;
    for (int i = 0; i < ExactSum::kDigits; ++i) {
      const uint64_t inv = (~(uint64_t)w[i]) & 0xFFFFFFFFu;
      const uint64_t t = inv + borrow;
      mag[i] = (uint32_t)t;
      borrow = t >> 32;
    }
  } else {
    for (int i = 0; i < ExactSum::kDigits; ++i) mag[i] = (uint32_t)w[i];
  }
  uint32_t q[ExactSum::kDigits];
  uint64_t rem = 0;
  for (int i = ExactSum::kDigits - 1; i >= 0; --i) {
    const uint64_t cur = (rem << 32) | mag[i];
    q[i] = (uint32_t)(cur / (uint64_t)count);
    rem = cur % (uint64_t)count;
  }
  int top = -1;  // highest set bit of q
  for (int i = ExactSum::kDigits - 1; i >= 0 && top < 0; --i)
    if (q[i])
      for (int b = 31; b >= 0; --b)
        if ((q[i] >> b) & 1u) {
          top = 32 * i + b;
          break;
        }
  auto bit = [&](int j) -> uint32_t { return j < 0 ? 0u : (q[j / 32] >> (j % 32)) & 1u; };
  const int p = top >= 24 ? top - 23 : 0;  // weight 2^(p - 149) of the kept last bit
  uint64_t sig = 0;
  for (int j = top; j >= p; --j) sig = (sig << 1) | bit(j);
  bool up;
  if (p == 0) {
    up = 2 * rem > (uint64_t)count || (2 * rem == (uint64_t)count && (sig & 1));
  } else {
    bool rest = rem != 0;
    for (int j = p - 2; j >= 0 && !rest; --j) rest = bit(j) != 0;
    up = bit(p - 1) && (rest || (sig & 1));
  }
  sig += up ? 1 : 0;
  const double v = std::ldexp((double)sig, p - 149);
  return (float)(neg ? -v : v);
}

}  // namespace

extern "C" {

// One Lloyd update: each centroid with points moves to their mean -- the
// exact sum of their fp32 coordinates over their count, rounded once to fp32
// (nearest even); the others stay.
void oracle_kmeans_update(const float* points, int64_t n, int dim, const int32_t* labels, int k,
                          float* centroids) {
  std::vector<ExactSum> sum((size_t)k * dim);
  std::vector<int64_t> count((size_t)k, 0);
  for (int64_t i = 0; i < n; ++i) {
    const int e = labels[i];
    ++count[(size_t)e];
    for (int d = 0; d < dim; ++d) sum[(size_t)e * dim + d].add(points[i * dim + d]);
  }
  for (int e = 0; e < k; ++e)
    if (count[(size_t)e] > 0)
      for (int d = 0; d < dim; ++d)
        centroids[(size_t)e * dim + d] = exact_mean_f32(sum[(size_t)e * dim + d], count[(size_t)e]);
}

// Flat positions (ascending) where |w - w_hat| > t in fp32, and the weights
// there; returns their number (at most cap are written).
int64_t oracle_sidecar_select(const float* W, const float* W_hat, int64_t nw, float t, int64_t* pos, float* val,
                              int64_t cap) {
  int64_t c = 0;
  for (int64_t p = 0; p < nw; ++p) {
    const float diff = W[p] - W_hat[p];
    const float err = diff < 0.f ? -diff : diff;
    if (err > t) {
      if (c < cap) {
        pos[c] = p;
        val[c] = W[p];
      }
      ++c;
    }
  }
  return c;
}

}  // extern "C"
