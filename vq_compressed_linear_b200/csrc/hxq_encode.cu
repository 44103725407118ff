// The encoder side of the codec on the GPU (HXQ whitepaper, method section:
// the per-tensor pipeline "Per-tensor k-means", "Index assignment",
// "Sidecar outlier correction", "12-bit index packing").
//
// Nearest-centroid assignment. Every point (one weight, or an adjacent pair
// of a row) is compared with every centroid, held in shared memory; each
// thread keeps four points in registers so one centroid load serves four
// comparisons. Distances are formed in fp32 with explicitly rounded
// operations (no contraction into fused multiply-adds): |p - c| for single
// weights, dx*dx + dy*dy for pairs. A strictly smaller distance replaces the
// best, so ties go to the lowest index. The decision is therefore the same
// as any other fp32 evaluation of the same expressions.
//
// k-means rounds (Lloyd): the assignment kernel also adds every point into
// its centroid's sum and count. A centroid moves to the exact mean of its
// points' fp32 coordinates, rounded once to fp32 (nearest even). The sums
// are exact integers: each coordinate becomes q = p * 2^F, with F chosen
// from the tensor's smallest nonzero magnitude so that every q is an integer
// (and from the largest, so that |q| < 2^62), split as q = hi * 2^32 + lo
// (lo in [0, 2^32)), and the two parts are added in separate 64-bit sums --
// first in shared memory, then once per CTA in global memory -- which no
// count of points below 2^31 can overflow. The finalizing kernel joins them
// into a 128-bit integer, divides by the count and rounds the quotient to
// fp32 from its bits and the remainder. Integer sums do not depend on order,
// so the result is bitwise repeatable and equals the correctly rounded mean
// whenever the nonzero magnitudes span at most 2^38 (beyond that the
// smallest values are first rounded to the 2^-F grid). A centroid without
// points stays where it is.
//
// Sidecar selection: a weight goes to the sidecar when |w - w_hat| > t in
// fp32. The entries are written in ascending position without atomics: one
// pass counts them per chunk of 8192 weights, one CTA turns the counts into
// offsets, and a second pass writes each chunk's entries at its offset in
// order (warp ballots and a block-wide prefix).
#include <climits>

#include "hxq_internal.cuh"

namespace hxq {
namespace {

constexpr int kAssignThreads = 256;
constexpr int kPointsPerThread = 4;
constexpr int kAssignTile = kAssignThreads * kPointsPerThread;  // points per CTA pass
constexpr int kSideChunk = 8192;                                // weights per compaction chunk
constexpr int kSideThreads = 256;
constexpr int kScanThreads = 1024;

// Fixed-point shift F of the k-means sums, from the largest magnitude's and
// the smallest nonzero magnitude's fp32 bits (range[0], range[1]): a value
// of exponent field ef >= 1 has its last bit at 2^(ef - 150) (subnormals at
// 2^-149, as ef = 1), so F = 150 - ef_min makes every value an integer
// multiple of 2^-F; it is lowered if needed so that every |q| < 2^62.
__device__ __forceinline__ int fixed_shift(const unsigned* range) {
  const int ef_max = max(1, (int)((range[0] >> 23) & 0xFF));
  const int ef_min = range[1] == 0xFFFFFFFFu ? ef_max : max(1, (int)((range[1] >> 23) & 0xFF));
  return min(150 - ef_min, 62 + 126 - ef_max);
}

template <int DIM>
__device__ __forceinline__ float dist(const float (&p)[2], const float* c) {
  if (DIM == 1) return fabsf(__fsub_rn(p[0], c[0]));
  const float dx = __fsub_rn(p[0], c[0]);
  const float dy = __fsub_rn(p[1], c[1]);
  return __fadd_rn(__fmul_rn(dx, dx), __fmul_rn(dy, dy));
}

// Nearest centroid of each of the n points [n][DIM]; optionally writes the
// index (labels) and, with ACCUM, adds each point into its centroid's
// fixed-point sum and count.
// gsum: [2][k][DIM] (the hi sums, then the lo sums); range: the largest
// and smallest nonzero magnitudes' bits.
template <int DIM, typename OutT, bool ACCUM>
__global__ void __launch_bounds__(kAssignThreads)
assign_kernel(const float* __restrict__ pts, int64_t n, const float* __restrict__ cent, int k,
              OutT* __restrict__ labels, unsigned long long* __restrict__ gsum, unsigned* __restrict__ gcount,
              const unsigned* __restrict__ range) {
  extern __shared__ __align__(16) unsigned char sm[];
  float* c = reinterpret_cast<float*>(sm);  // [k][DIM]
  unsigned long long* ssum =               // [2][k][DIM]: hi, lo
      reinterpret_cast<unsigned long long*>(sm + (((size_t)k * DIM * sizeof(float) + 15) & ~(size_t)15));
  unsigned* scount = reinterpret_cast<unsigned*>(ssum + 2 * (size_t)k * DIM);
  for (int i = threadIdx.x; i < k * DIM; i += blockDim.x) c[i] = cent[i];
  int F = 0;
  if (ACCUM) {
    for (int i = threadIdx.x; i < 2 * k * DIM; i += blockDim.x) ssum[i] = 0ull;
    for (int i = threadIdx.x; i < k; i += blockDim.x) scount[i] = 0u;
    F = fixed_shift(range);
  }
  __syncthreads();

  for (int64_t tile = (int64_t)blockIdx.x * kAssignTile; tile < n; tile += (int64_t)gridDim.x * kAssignTile) {
    float p[kPointsPerThread][2];
    float best[kPointsPerThread];
    int bi[kPointsPerThread];
#pragma unroll
    for (int j = 0; j < kPointsPerThread; ++j) {
      const int64_t i = min(tile + j * kAssignThreads + threadIdx.x, n - 1);  // clamped: every load in bounds
      p[j][0] = pts[i * DIM];
      p[j][1] = DIM == 2 ? pts[i * DIM + 1] : 0.f;
      best[j] = __int_as_float(0x7f800000);  // +inf
      bi[j] = 0;
    }
    for (int e = 0; e < k; ++e) {
      const float* ce = c + e * DIM;
#pragma unroll
      for (int j = 0; j < kPointsPerThread; ++j) {
        const float d = dist<DIM>(p[j], ce);
        if (d < best[j]) {
          best[j] = d;
          bi[j] = e;
        }
      }
    }
#pragma unroll
    for (int j = 0; j < kPointsPerThread; ++j) {
      const int64_t i = tile + j * kAssignThreads + threadIdx.x;
      if (i >= n) continue;
      if (labels) labels[i] = (OutT)bi[j];
      if (ACCUM) {
        atomicAdd(scount + bi[j], 1u);
#pragma unroll
        for (int d = 0; d < DIM; ++d) {
          // exact: q has at most 24 significant bits
          const long long q = llrint(ldexp((double)p[j][d], F));
          atomicAdd(ssum + (size_t)bi[j] * DIM + d, (unsigned long long)(q >> 32));
          atomicAdd(ssum + (size_t)(k + bi[j]) * DIM + d, (unsigned long long)(q & 0xFFFFFFFFll));
        }
      }
    }
  }
  if (ACCUM) {
    __syncthreads();
    for (int i = threadIdx.x; i < k; i += blockDim.x) {
      if (scount[i] == 0) continue;
      atomicAdd(gcount + i, scount[i]);
#pragma unroll
      for (int d = 0; d < DIM; ++d) {
        atomicAdd(gsum + (size_t)i * DIM + d, ssum[(size_t)i * DIM + d]);
        atomicAdd(gsum + (size_t)(k + i) * DIM + d, ssum[(size_t)(k + i) * DIM + d]);
      }
    }
  }
}

// Largest |p| and smallest nonzero |p| as fp32 bits (non-negative floats
// order like their bits): out[0] starts at 0, out[1] at 0xFFFFFFFF.
__global__ void range_kernel(const float* __restrict__ p, int64_t n, unsigned* __restrict__ out) {
  unsigned mx = 0, mn = 0xFFFFFFFFu;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const unsigned a = __float_as_uint(p[i]) & 0x7FFFFFFFu;
    mx = max(mx, a);
    if (a != 0) mn = min(mn, a);
  }
  mx = __reduce_max_sync(0xffffffffu, mx);
  mn = __reduce_min_sync(0xffffffffu, mn);
  if ((threadIdx.x & 31) == 0) {
    atomicMax(out, mx);
    atomicMin(out + 1, mn);
  }
}

__device__ __forceinline__ int bitlen128(unsigned __int128 v) {
  const unsigned long long hi = (unsigned long long)(v >> 64), lo = (unsigned long long)v;
  return hi ? 128 - __clzll((long long)hi) : (lo ? 64 - __clzll((long long)lo) : 0);
}

// The fp32 value nearest to T / (cnt * 2^F), ties to the even significand.
// The numerator is scaled by 2^sh so that Q = |T| 2^sh / cnt has at least
// 25 bits; the kept last bit is at max(2^(E - 23), 2^-149) for the value's
// exponent E, i.e. at Q's bit p = max(len(Q) - 24, F + sh - 149); the bit
// below it and everything further down, the remainder included, decide the
// rounding.
__device__ __forceinline__ float round_mean_f32(__int128 T, unsigned cnt, int F) {
  if (T == 0) return 0.f;
  const bool neg = T < 0;
  const unsigned __int128 a = neg ? (unsigned __int128)(-T) : (unsigned __int128)T;  // below 2^94
  const int cl = 32 - __clz((int)cnt);
  const int sh = max(0, 26 - (bitlen128(a) - cl));  // then |T| 2^sh stays below 2^(26 + 32)
  const unsigned __int128 num = a << sh;
  const unsigned __int128 Q = num / cnt;
  const unsigned long long R = (unsigned long long)(num % cnt);
  const int Fe = F + sh;
  const int p = max(bitlen128(Q) - 24, Fe - 149);  // at least 1: Q has at least 25 bits
  const unsigned long long sig = p < 128 ? (unsigned long long)(Q >> p) : 0ull;
  const bool half = p - 1 < 128 && ((unsigned)(Q >> (p - 1)) & 1u);
  const unsigned __int128 below = p - 1 < 128 ? Q & ((((unsigned __int128)1) << (p - 1)) - 1) : Q;
  const bool up = half && (below != 0 || R != 0 || (sig & 1));
  const double v = ldexp((double)(sig + (up ? 1 : 0)), p - Fe);  // exact
  return (float)(neg ? -v : v);
}

// New centroid = the exact sum over the count, rounded once to fp32; no
// points: unchanged.
__global__ void kmeans_finalize(float* __restrict__ cent, int k, int dim, const unsigned long long* __restrict__ gsum,
                                const unsigned* __restrict__ gcount, const unsigned* __restrict__ range) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= k) return;
  const unsigned cnt = gcount[i];
  if (cnt == 0) return;
  const int F = fixed_shift(range);
  for (int d = 0; d < dim; ++d) {
    const long long hi = (long long)gsum[(size_t)i * dim + d];
    const long long lo = (long long)gsum[(size_t)(k + i) * dim + d];  // a sum of values below 2^32
    const __int128 T = (__int128)hi * ((__int128)1 << 32) + (__int128)lo;
    cent[(size_t)i * dim + d] = round_mean_f32(T, cnt, F);
  }
}

// 12-bit indices, two per 3 bytes: little-endian 24-bit word, the first
// index in the low 12 bits.
__global__ void pack12_kernel(const uint16_t* __restrict__ lab, int64_t n_groups, uint8_t* __restrict__ out) {
  for (int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; g < n_groups;
       g += (int64_t)gridDim.x * blockDim.x) {
    const uint32_t w = ((uint32_t)lab[2 * g] & 0xFFFu) | (((uint32_t)lab[2 * g + 1] & 0xFFFu) << 12);
    out[3 * g] = (uint8_t)(w & 0xFF);
    out[3 * g + 1] = (uint8_t)((w >> 8) & 0xFF);
    out[3 * g + 2] = (uint8_t)(w >> 16);
  }
}

// The decoded value at flat position p from the encoded indices.
template <int MODE>
__device__ __forceinline__ float decoded_at(const uint8_t* __restrict__ idx, const float* __restrict__ cb, int64_t p) {
  if (MODE == HXQ_MODE_SCALAR8) return cb[idx[p]];
  const int64_t g = p >> 1, grp = g >> 1;
  const uint32_t w = (uint32_t)idx[3 * grp] | ((uint32_t)idx[3 * grp + 1] << 8) | ((uint32_t)idx[3 * grp + 2] << 16);
  const uint32_t e = (g & 1) ? (w >> 12) : (w & 0xFFFu);
  return cb[2 * e + (p & 1)];
}

template <int MODE>
__device__ __forceinline__ bool is_outlier(const float* __restrict__ W, const uint8_t* __restrict__ idx,
                                           const float* __restrict__ cb, int64_t p, float t) {
  return fabsf(__fsub_rn(W[p], decoded_at<MODE>(idx, cb, p))) > t;
}

template <int MODE>
__global__ void __launch_bounds__(kSideThreads)
sidecar_count_kernel(const float* __restrict__ W, const uint8_t* __restrict__ idx, const float* __restrict__ cb,
                     int64_t nw, float t, long long* __restrict__ counts) {
  __shared__ int warp_n[kSideThreads / 32];
  const int64_t c0 = (int64_t)blockIdx.x * kSideChunk, c1 = min(nw, c0 + kSideChunk);
  int mine = 0;
  for (int64_t p = c0 + threadIdx.x; p < c1; p += kSideThreads) mine += is_outlier<MODE>(W, idx, cb, p, t);
  mine = __reduce_add_sync(0xffffffffu, mine);
  if ((threadIdx.x & 31) == 0) warp_n[threadIdx.x >> 5] = mine;
  __syncthreads();
  if (threadIdx.x == 0) {
    long long s = 0;
    for (int w = 0; w < kSideThreads / 32; ++w) s += warp_n[w];
    counts[blockIdx.x] = s;
  }
}

// Exclusive prefix of the chunk counts (one CTA); the total goes to *total.
__global__ void __launch_bounds__(kScanThreads)
sidecar_scan_kernel(const long long* __restrict__ counts, int64_t nb, long long* __restrict__ offsets,
                    int64_t* __restrict__ total) {
  __shared__ long long warp_s[kScanThreads / 32];
  __shared__ long long carry_sh;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) carry_sh = 0;
  __syncthreads();
  for (int64_t base = 0; base < nb; base += kScanThreads) {
    const int64_t i = base + threadIdx.x;
    const long long v = i < nb ? counts[i] : 0;
    long long x = v;  // inclusive warp prefix
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const long long y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) warp_s[warp] = x;
    __syncthreads();
    if (warp == 0) {
      long long w = lane < kScanThreads / 32 ? warp_s[lane] : 0;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const long long y = __shfl_up_sync(0xffffffffu, w, o);
        if (lane >= o) w += y;
      }
      if (lane < kScanThreads / 32) warp_s[lane] = w;  // inclusive prefix over warps
    }
    __syncthreads();
    const long long before = carry_sh + (warp > 0 ? warp_s[warp - 1] : 0) + (x - v);
    if (i < nb) offsets[i] = before;
    __syncthreads();
    if (threadIdx.x == 0) carry_sh += warp_s[kScanThreads / 32 - 1];
    __syncthreads();
  }
  if (threadIdx.x == 0) *total = carry_sh;
}

template <int MODE>
__global__ void __launch_bounds__(kSideThreads)
sidecar_write_kernel(const float* __restrict__ W, const uint8_t* __restrict__ idx, const float* __restrict__ cb,
                     int64_t nw, float t, const long long* __restrict__ offsets, int64_t* __restrict__ pos,
                     float* __restrict__ val, int64_t cap) {
  __shared__ int warp_n[kSideThreads / 32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t c0 = (int64_t)blockIdx.x * kSideChunk, c1 = min(nw, c0 + kSideChunk);
  long long next = offsets[blockIdx.x];
  for (int64_t r = c0; r < c1; r += kSideThreads) {
    const int64_t p = r + threadIdx.x;
    const bool hit = p < c1 && is_outlier<MODE>(W, idx, cb, p, t);
    const unsigned m = __ballot_sync(0xffffffffu, hit);
    if (lane == 0) warp_n[warp] = __popc(m);
    __syncthreads();
    long long o = next + __popc(m & ((1u << lane) - 1u));
    int round_n = 0;
#pragma unroll
    for (int w = 0; w < kSideThreads / 32; ++w) {
      if (w < warp) o += warp_n[w];
      round_n += warp_n[w];
    }
    if (hit && o < cap) {
      pos[o] = p;
      val[o] = W[p];
    }
    next += round_n;
    __syncthreads();  // warp_n is rewritten next round
  }
}

int grid_for(int64_t items, int per_cta, int num_sms, int ctas_per_sm) {
  const int64_t need = (items + per_cta - 1) / per_cta;
  return (int)std::max<int64_t>(1, std::min<int64_t>(need, (int64_t)num_sms * ctas_per_sm));
}

int device_sms() {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    cudaGetLastError();
    return 148;
  }
  return sms;
}

size_t assign_smem(int dim, int k, bool accum) {
  size_t s = ((size_t)k * dim * sizeof(float) + 15) & ~(size_t)15;
  if (accum) s += 2 * (size_t)k * dim * sizeof(unsigned long long) + (size_t)k * sizeof(unsigned);
  return s;
}

template <int DIM, typename OutT, bool ACCUM>
cudaError_t launch_assign(const float* pts, int64_t n, const float* cent, int k, OutT* labels,
                          unsigned long long* gsum, unsigned* gcount, const unsigned* range, cudaStream_t s) {
  auto kern = assign_kernel<DIM, OutT, ACCUM>;
  const size_t smem = assign_smem(DIM, k, ACCUM);
  cudaError_t e = allow_max_smem(reinterpret_cast<const void*>(kern));
  if (e != cudaSuccess) return e;
  const int grid = grid_for(n, kAssignTile, device_sms(), 2);
  kern<<<grid, kAssignThreads, smem, s>>>(pts, n, cent, k, labels, gsum, gcount, range);
  return cudaGetLastError();
}

template <int DIM>
cudaError_t kmeans_rounds(const float* pts, int64_t n, int k, int iters, float* cent, uint16_t* labels,
                          cudaStream_t s) {
  cudaError_t e = cudaSuccess;
  if (iters > 0) {
    // scratch: sums [2][k][DIM] int64, counts [k], the magnitude range
    const size_t sums = 2 * (size_t)k * DIM * 8 + (size_t)k * 4;
    const size_t bytes = sums + 16;
    void* scratch = nullptr;
    if ((e = cudaMallocAsync(&scratch, bytes, s)) != cudaSuccess) return e;
    auto* gsum = static_cast<unsigned long long*>(scratch);
    auto* gcount = reinterpret_cast<unsigned*>(gsum + 2 * (size_t)k * DIM);
    auto* range = gcount + k;
    const int sms = device_sms();
    e = cudaMemsetAsync(range, 0, sizeof(unsigned), s);
    if (e == cudaSuccess) e = cudaMemsetAsync(range + 1, 0xFF, sizeof(unsigned), s);
    if (e == cudaSuccess) {
      range_kernel<<<grid_for(n * DIM, 256, sms, 4), 256, 0, s>>>(pts, n * DIM, range);
      e = cudaGetLastError();
    }
    for (int it = 0; it < iters && e == cudaSuccess; ++it) {
      e = cudaMemsetAsync(scratch, 0, sums, s);
      if (e == cudaSuccess)
        e = launch_assign<DIM, uint16_t, true>(pts, n, cent, k, nullptr, gsum, gcount, range, s);
      if (e == cudaSuccess) {
        kmeans_finalize<<<(k + 255) / 256, 256, 0, s>>>(cent, k, DIM, gsum, gcount, range);
        e = cudaGetLastError();
      }
    }
    const cudaError_t ef = cudaFreeAsync(scratch, s);
    if (e == cudaSuccess) e = ef;
  }
  if (e == cudaSuccess && labels)
    e = launch_assign<DIM, uint16_t, false>(pts, n, cent, k, labels, nullptr, nullptr, nullptr, s);
  return e;
}

template <int MODE>
cudaError_t sidecar_select(const float* W, const uint8_t* idx, const float* cb, int64_t nw, float t, int64_t* pos,
                           float* val, int64_t cap, int64_t* n_out, cudaStream_t s) {
  const int64_t nb = (nw + kSideChunk - 1) / kSideChunk;
  void* scratch = nullptr;
  cudaError_t e = cudaMallocAsync(&scratch, (size_t)nb * 2 * sizeof(long long), s);
  if (e != cudaSuccess) return e;
  auto* counts = static_cast<long long*>(scratch);
  long long* offsets = counts + nb;
  sidecar_count_kernel<MODE><<<(unsigned)nb, kSideThreads, 0, s>>>(W, idx, cb, nw, t, counts);
  e = cudaGetLastError();
  if (e == cudaSuccess) {
    sidecar_scan_kernel<<<1, kScanThreads, 0, s>>>(counts, nb, offsets, n_out);
    e = cudaGetLastError();
  }
  if (e == cudaSuccess) {
    sidecar_write_kernel<MODE><<<(unsigned)nb, kSideThreads, 0, s>>>(W, idx, cb, nw, t, offsets, pos, val, cap);
    e = cudaGetLastError();
  }
  const cudaError_t ef = cudaFreeAsync(scratch, s);
  return e == cudaSuccess ? ef : e;
}

int status_of(cudaError_t e) {
  if (e == cudaSuccess) return HXQ_OK;
  cudaGetLastError();
  if (e == cudaErrorMemoryAllocation) return HXQ_ENOMEM;
  if (e == cudaErrorInvalidValue) return HXQ_EINVAL;
  return HXQ_ECUDA;
}

constexpr int64_t kMaxPoints = (int64_t)1 << 31;  // counts are 32-bit

}  // namespace
}  // namespace hxq

extern "C" {

int hxq_assign(const float* points, int64_t n, int dim, const float* centroids, int k, uint16_t* labels,
               void* stream) {
  using namespace hxq;
  if (!points || !centroids || !labels || n < 1 || n >= kMaxPoints || (dim != 1 && dim != 2) || k < 1 ||
      k > 4096)
    return HXQ_EINVAL;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const cudaError_t e = dim == 1
      ? launch_assign<1, uint16_t, false>(points, n, centroids, k, labels, nullptr, nullptr, nullptr, s)
      : launch_assign<2, uint16_t, false>(points, n, centroids, k, labels, nullptr, nullptr, nullptr, s);
  return status_of(e);
}

int hxq_kmeans(const float* points, int64_t n, int dim, int k, int iters, float* centroids, uint16_t* labels,
               void* stream) {
  using namespace hxq;
  if (!points || !centroids || n < 1 || n >= kMaxPoints || (dim != 1 && dim != 2) || k < 1 || k > 4096 ||
      iters < 0)
    return HXQ_EINVAL;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const cudaError_t e = dim == 1 ? kmeans_rounds<1>(points, n, k, iters, centroids, labels, s)
                                 : kmeans_rounds<2>(points, n, k, iters, centroids, labels, s);
  return status_of(e);
}

int hxq_encode(const float* W, int mode, int N, int K, const float* codebook, float threshold, uint8_t* indices,
               int64_t* sidecar_pos, float* sidecar_val, int64_t max_sidecar, int64_t* n_sidecar, void* stream) {
  using namespace hxq;
  if (!W || !codebook || !indices || !n_sidecar) return HXQ_EINVAL;
  if (mode != HXQ_MODE_SCALAR8 && mode != HXQ_MODE_VQ2D12) return HXQ_EINVAL;
  if (N < 1 || K < 1 || (mode == HXQ_MODE_VQ2D12 && (K % 4) != 0) || (int64_t)N * K >= kMaxPoints)
    return HXQ_EINVAL;
  if (!(threshold >= 0.f) || max_sidecar < 0 || (max_sidecar > 0 && (!sidecar_pos || !sidecar_val)))
    return HXQ_EINVAL;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int64_t nw = (int64_t)N * K;
  cudaError_t e;
  if (mode == HXQ_MODE_SCALAR8) {
    e = launch_assign<1, uint8_t, false>(W, nw, codebook, 256, indices, nullptr, nullptr, nullptr, s);
    if (e == cudaSuccess)
      e = sidecar_select<HXQ_MODE_SCALAR8>(W, indices, codebook, nw, threshold, sidecar_pos, sidecar_val,
                                           max_sidecar, n_sidecar, s);
  } else {
    void* lab = nullptr;
    e = cudaMallocAsync(&lab, (size_t)(nw / 2) * sizeof(uint16_t), s);
    if (e != cudaSuccess) return status_of(e);
    e = launch_assign<2, uint16_t, false>(W, nw / 2, codebook, 4096, static_cast<uint16_t*>(lab), nullptr, nullptr,
                                          nullptr, s);
    if (e == cudaSuccess) {
      pack12_kernel<<<grid_for(nw / 4, 256, device_sms(), 4), 256, 0, s>>>(static_cast<uint16_t*>(lab), nw / 4,
                                                                          indices);
      e = cudaGetLastError();
    }
    const cudaError_t ef = cudaFreeAsync(lab, s);
    if (e == cudaSuccess) e = ef;
    if (e == cudaSuccess)
      e = sidecar_select<HXQ_MODE_VQ2D12>(W, indices, codebook, nw, threshold, sidecar_pos, sidecar_val,
                                          max_sidecar, n_sidecar, s);
  }
  return status_of(e);
}

}  // extern "C"
