// Fused decode + GEMV on CUDA cores for few tokens (M <= 32, used by default
// for M <= 4): y[m][n] = sum_k x[m][k] * W[n][k] with W decoded on the fly
// from the codebook and never written anywhere (the pages' buffered path
// instead materialises W and calls cuBLAS: HXQ whitepaper, method section,
// buffered forward path paragraph).
//
// Work decomposition. A unit is one 128-row tile times one contiguous range
// of 64-weight stages along K (split-K). Each CTA is persistent: it builds
// its shared-memory codebook once, then takes units blockIdx.x,
// blockIdx.x + gridDim.x, ... Inside a unit the CTA's G = 4 groups of 128
// threads take the stages round-robin; thread r of a group owns row r of
// the tile and reads its 16-byte index pieces, so a warp reads 512
// contiguous bytes per load.
//
// Scalar codebook in shared memory: replicated once per lane with entry e of
// lane l at byte e*256 + l*4, so the 32 lanes of a lookup always hit 32
// different banks. The byte address is one PRMT away from the index word:
// {0, 0, index byte, l*4}.
//
// 2D codebook: the 4096 fp32 pairs (32 KB) are kept once; lookups of random
// pairs can conflict on banks (the pair table is too large to replicate).
//
// Sidecar: each row keeps a pointer into its column-sorted patch list and
// substitutes the stored value for the decoded one at the patched columns,
// before the multiply (replacement, HXQ whitepaper, method section,
// "Sidecar outlier correction").
//
// Split-K: units of one tile write fp32 partials to the workspace; the last
// unit to arrive (counted with an integer atomic per tile) sums them in split
// order s = 0, 1, ..., so results are bitwise repeatable.
#include <algorithm>
#include <climits>

#include "hxq_internal.cuh"

namespace hxq {
namespace {

constexpr int kGemvThreads = 512;
constexpr int kGroups = kGemvThreads / kTileRows;  // 4

template <int MT>
struct GemvSmem {
  static constexpr size_t table_bytes(int mode) { return mode == HXQ_MODE_SCALAR8 ? 256 * 256 : 4096 * 8; }
  static constexpr size_t red_bytes() { return (size_t)kGroups * MT * kTileRows * sizeof(float); }
};

__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Load 8 activations x[m][k0 .. k0+8) as fp32 (0 beyond row end or m >= M).
__device__ __forceinline__ void load_x8(const uint16_t* __restrict__ x, int K, int M, int m, int k0, float (&f)[8]) {
  uint4 q = make_uint4(0, 0, 0, 0);
  if (m < M && k0 < K) q = __ldg(reinterpret_cast<const uint4*>(x + (size_t)m * K + k0));
  f[0] = bf16lo(q.x); f[1] = bf16hi(q.x); f[2] = bf16lo(q.y); f[3] = bf16hi(q.y);
  f[4] = bf16lo(q.z); f[5] = bf16hi(q.z); f[6] = bf16lo(q.w); f[7] = bf16hi(q.w);
}

struct Unit {
  int t, s, st0, st1;  // tile, split, stage range [st0, st1)
};

__device__ __forceinline__ Unit unit_of(int u, int S, int n_stages) {
  Unit U;
  U.t = u / S;
  U.s = u % S;
  U.st0 = (int)((int64_t)U.s * n_stages / S);
  U.st1 = (int)((int64_t)(U.s + 1) * n_stages / S);
  return U;
}

// Sum the groups' partials of this unit and publish: straight to y when the
// unit covers all of K, else through the workspace with the last-arriver sum.
template <int MT>
__device__ void finish_unit(const Layer& L, const Unit& U, int M, int S, float* red, float* __restrict__ y,
                            float* __restrict__ work, int* __restrict__ counters, int* flag) {
  const int rows = min(kTileRows, L.N - U.t * kTileRows);
  for (int i = threadIdx.x; i < MT * kTileRows; i += blockDim.x) {
    const int m = i / kTileRows, r = i % kTileRows;
    if (m >= M || r >= rows) continue;
    float v = 0.f;
#pragma unroll
    for (int g = 0; g < kGroups; ++g) v += red[(g * MT + m) * kTileRows + r];
    const size_t n = (size_t)U.t * kTileRows + r;
    if (S == 1) y[(size_t)m * L.N + n] = v;
    else work[((size_t)U.s * M + m) * L.N + n] = v;
  }
  if (S == 1) return;
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) *flag = atomicAdd(counters + U.t * 64, 1) == S - 1;
  __syncthreads();
  if (!*flag) return;
  __threadfence();
  for (int i = threadIdx.x; i < M * kTileRows; i += blockDim.x) {
    const int m = i / kTileRows, r = i % kTileRows;
    if (r >= rows) continue;
    const size_t n = (size_t)U.t * kTileRows + r;
    float v = 0.f;
    for (int s = 0; s < S; ++s) v += __ldcg(work + ((size_t)s * M + m) * L.N + n);
    y[(size_t)m * L.N + n] = v;
  }
  if (threadIdx.x == 0) counters[U.t * 64] = 0;
}

template <int MT>
__global__ void __launch_bounds__(kGemvThreads, 1)
gemv_scalar_kernel(Layer L, const uint16_t* __restrict__ x, float* __restrict__ y, int M, int S,
                   float* __restrict__ work, int* __restrict__ counters) {
  extern __shared__ __align__(1024) uint8_t smem[];
  float* table = reinterpret_cast<float*>(smem);                       // 64 KB
  float* red = reinterpret_cast<float*>(smem + 256 * 256);             // G*MT*128 floats
  __shared__ int flag;
  const int lane = threadIdx.x & 31;
  const int g = threadIdx.x / kTileRows, r = threadIdx.x % kTileRows;

  for (int i = threadIdx.x; i < 256 * 32; i += blockDim.x)
    table[(i >> 5) * 64 + (i & 31)] = __ldg(L.codebook + (i >> 5));
  __syncthreads();

  const uint32_t lane4 = (uint32_t)lane * 4u;
  const char* tb = reinterpret_cast<const char*>(table);
  const int n_stages = L.Kp / kStageK;
  const int units = L.n_tiles * S;

  for (int u = blockIdx.x; u < units; u += gridDim.x) {
    const Unit U = unit_of(u, S, n_stages);
    const int rows = min(kTileRows, L.N - U.t * kTileRows);
    const int n = U.t * kTileRows + r;
    float acc[MT];
#pragma unroll
    for (int m = 0; m < MT; ++m) acc[m] = 0.f;
    if (r < rows) {
      int p = 0, pend = 0, pk = INT_MAX;
      {
        // first patch at or after the unit's first column
        int lo = L.row_ptr[n], hi = L.row_ptr[n + 1];
        pend = hi;
        const int k0 = U.st0 * kStageK;
        while (lo < hi) {
          const int mid = (lo + hi) >> 1;
          if (L.patch_k[mid] < k0) lo = mid + 1; else hi = mid;
        }
        p = lo;
        pk = p < pend ? L.patch_k[p] : INT_MAX;
      }
      for (int st = U.st0 + g; st < U.st1; st += kGroups) {
        uint4 q[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) q[c] = ldg_stream16(L.idx + piece_offset(L, U.t, st * 4 + c, 0, r));
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int k0 = st * kStageK + c * 16;
          const uint32_t wd[4] = {q[c].x, q[c].y, q[c].z, q[c].w};
          float wv[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const uint32_t sel = 0x5504u | ((uint32_t)(j & 3) << 4);
            const uint32_t a = prmt(wd[j >> 2], lane4, sel);
            wv[j] = *reinterpret_cast<const float*>(tb + a);
          }
          while (pk < k0 + 16) {                       // rare: sidecar patches
            if (pk >= k0) {
              const float v = L.patch_v[p];
#pragma unroll
              for (int j = 0; j < 16; ++j) wv[j] = sel_eq(pk - k0, j, v, wv[j]);
            }
            ++p;
            pk = p < pend ? L.patch_k[p] : INT_MAX;
          }
#pragma unroll
          for (int m = 0; m < MT; ++m) {
            float xa[8], xb[8];
            load_x8(x, L.K, M, m, k0, xa);
            load_x8(x, L.K, M, m, k0 + 8, xb);
            float a = acc[m];
#pragma unroll
            for (int j = 0; j < 8; ++j) a = fmaf(wv[j], xa[j], a);
#pragma unroll
            for (int j = 0; j < 8; ++j) a = fmaf(wv[8 + j], xb[j], a);
            acc[m] = a;
          }
        }
      }
    }
#pragma unroll
    for (int m = 0; m < MT; ++m) red[(g * MT + m) * kTileRows + r] = acc[m];
    __syncthreads();
    finish_unit<MT>(L, U, M, S, red, y, work, counters, &flag);
    __syncthreads();
  }
}

template <int MT>
__global__ void __launch_bounds__(kGemvThreads, 1)
gemv_vq2d_kernel(Layer L, const uint16_t* __restrict__ x, float* __restrict__ y, int M, int S,
                 float* __restrict__ work, int* __restrict__ counters) {
  extern __shared__ __align__(1024) uint8_t smem[];
  float2* table = reinterpret_cast<float2*>(smem);                     // 32 KB
  float* red = reinterpret_cast<float*>(smem + 4096 * 8);
  __shared__ int flag;
  const int g = threadIdx.x / kTileRows, r = threadIdx.x % kTileRows;

  const float2* cb2 = reinterpret_cast<const float2*>(L.codebook);
  for (int i = threadIdx.x; i < 4096; i += blockDim.x) table[i] = __ldg(cb2 + i);
  __syncthreads();

  const int n_stages = L.Kp / kStageK;
  const int units = L.n_tiles * S;

  for (int u = blockIdx.x; u < units; u += gridDim.x) {
    const Unit U = unit_of(u, S, n_stages);
    const int rows = min(kTileRows, L.N - U.t * kTileRows);
    const int n = U.t * kTileRows + r;
    float acc[MT];
#pragma unroll
    for (int m = 0; m < MT; ++m) acc[m] = 0.f;
    if (r < rows) {
      int p, pend, pk;
      {
        int lo = L.row_ptr[n], hi = L.row_ptr[n + 1];
        pend = hi;
        const int k0 = U.st0 * kStageK;
        while (lo < hi) {
          const int mid = (lo + hi) >> 1;
          if (L.patch_k[mid] < k0) lo = mid + 1; else hi = mid;
        }
        p = lo;
        pk = p < pend ? L.patch_k[p] : INT_MAX;
      }
      for (int st = U.st0 + g; st < U.st1; st += kGroups) {
        uint32_t w[13];
#pragma unroll
        for (int pl = 0; pl < 3; ++pl) {
          const uint4 q = ldg_stream16(L.idx + piece_offset(L, U.t, st, pl, r));
          w[4 * pl] = q.x; w[4 * pl + 1] = q.y; w[4 * pl + 2] = q.z; w[4 * pl + 3] = q.w;
        }
        w[12] = 0;
        const int kbase = st * kStageK;
#pragma unroll
        for (int h = 0; h < 4; ++h) {                 // 4 x 16 weights
          float wv[16];
#pragma unroll
          for (int jj = 0; jj < 8; ++jj) {
            const int j = h * 8 + jj, bit = 12 * j;
            const uint32_t e = __funnelshift_r(w[bit >> 5], w[(bit >> 5) + 1], bit & 31) & 0xFFF;
            const float2 v = table[e];
            wv[2 * jj] = v.x;
            wv[2 * jj + 1] = v.y;
          }
          const int k0 = kbase + h * 16;
          while (pk < k0 + 16) {
            if (pk >= k0) {
              const float v = L.patch_v[p];
#pragma unroll
              for (int j = 0; j < 16; ++j) wv[j] = sel_eq(pk - k0, j, v, wv[j]);
            }
            ++p;
            pk = p < pend ? L.patch_k[p] : INT_MAX;
          }
#pragma unroll
          for (int m = 0; m < MT; ++m) {
            float xa[8], xb[8];
            load_x8(x, L.K, M, m, k0, xa);
            load_x8(x, L.K, M, m, k0 + 8, xb);
            float a = acc[m];
#pragma unroll
            for (int j = 0; j < 8; ++j) a = fmaf(wv[j], xa[j], a);
#pragma unroll
            for (int j = 0; j < 8; ++j) a = fmaf(wv[8 + j], xb[j], a);
            acc[m] = a;
          }
        }
      }
    }
#pragma unroll
    for (int m = 0; m < MT; ++m) red[(g * MT + m) * kTileRows + r] = acc[m];
    __syncthreads();
    finish_unit<MT>(L, U, M, S, red, y, work, counters, &flag);
    __syncthreads();
  }
}

template <int MT>
cudaError_t launch_mt(const hxq_linear& h, const uint16_t* x, float* y, int M, int S, cudaStream_t s) {
  const bool scalar = h.L.mode == HXQ_MODE_SCALAR8;
  const size_t smem = GemvSmem<MT>::table_bytes(h.L.mode) + GemvSmem<MT>::red_bytes();
  auto kern = scalar ? gemv_scalar_kernel<MT> : gemv_vq2d_kernel<MT>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kGemvThreads, smem);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) per_sm = 1;
  const int units = h.L.n_tiles * S;
  const int grid = std::min(units, h.num_sms * per_sm);
  kern<<<grid, kGemvThreads, smem, s>>>(h.L, x, y, M, S, h.d_work, h.d_counters);
  return cudaGetLastError();
}

}  // namespace

// Split count along K: balance units over the persistent CTAs (whole waves),
// keep every group busy (at least kGroups stages per unit) and stay within
// the workspace.
int choose_split_gemv(const hxq_linear& h, int M) {
  const int n_stages = h.L.Kp / kStageK;
  const int slots = h.num_sms;
  int best = 1;
  double best_score = -1.0;
  for (int S = 1; S <= std::min(n_stages, kMaxSplitK); ++S) {
    if (S > 1 && (size_t)S * M * h.L.N > h.work_floats) break;
    const int units = h.L.n_tiles * S;
    const int waves = (units + slots - 1) / slots;
    const double wave_eff = (double)units / ((double)waves * slots);
    const double per_unit = (double)n_stages / S;
    const double group_eff = std::min(1.0, per_unit / kGroups);
    const double score = wave_eff * group_eff / (1.0 + 0.002 * S);
    if (score > best_score + 1e-9) {
      best_score = score;
      best = S;
    }
  }
  return best;
}

cudaError_t launch_gemv(const hxq_linear& h, const uint16_t* x, float* y, int M, int split, cudaStream_t s) {
  const int n_stages = h.L.Kp / kStageK;
  int S = std::max(1, std::min(split, n_stages));
  if (S > 1 && (size_t)S * M * h.L.N > h.work_floats) return cudaErrorInvalidValue;
  if (M <= 1) return launch_mt<1>(h, x, y, M, S, s);
  if (M <= 2) return launch_mt<2>(h, x, y, M, S, s);
  if (M <= 4) return launch_mt<4>(h, x, y, M, S, s);
  if (M <= 8) return launch_mt<8>(h, x, y, M, S, s);
  if (M <= 16) return launch_mt<16>(h, x, y, M, S, s);
  if (M <= 32) return launch_mt<32>(h, x, y, M, S, s);
  return cudaErrorInvalidValue;
}

}  // namespace hxq
