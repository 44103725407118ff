// Fused decode + GEMV on CUDA cores for few tokens (M <= 4 by default; up to
// M = 32 on request): y[m][n] = sum_k x[m][k] * W[n][k] with W decoded on the
// fly from the codebook and never written anywhere (the pages' buffered path
// instead materialises W and calls cuBLAS: HXQ whitepaper, method section,
// buffered forward path paragraph).
//
// Work decomposition (stream-K). The work items are the tile-stages of the
// layer, (tile of 128 rows) x (64 weights along K), numbered tile-major. A
// persistent grid of one 512-thread CTA per SM takes contiguous item ranges
// of equal size, so every CTA streams the same number of index bytes
// whatever the layer shape. Inside a CTA the 4 groups of 128 threads take
// the items round-robin; thread r of a group owns row r of the item's tile
// (a warp reads 512 contiguous bytes per 16-byte load) and keeps the next
// items' loads in flight in a register ring while it decodes the current
// one. At each tile boundary of the CTA's range the groups' sums meet in
// shared memory; a tile covered by one CTA goes straight to y, a tile split
// between CTAs leaves one fp32 partial per CTA in the workspace and the last
// CTA to arrive (integer atomic per tile) adds them in CTA order: results
// are bitwise repeatable.
//
// Scalar codebook in shared memory: replicated once per lane with entry e of
// lane l at byte e*256 + l*4, so the 32 lanes of a lookup always hit 32
// different banks. The byte address is one PRMT away from the index word:
// {0, 0, index byte, l*4}.
//
// 2D codebook: the 4096 fp32 pairs (32 KB) are kept once; random pair
// lookups can conflict on banks (a per-lane replica would need 1 MB).
//
// Activations are staged once per CTA in shared memory (fp32, or bf16 when
// fp32 would not fit), zero-padded to whole 64-weight stages.
//
// Sidecar (replacement of single weights, HXQ whitepaper, method section,
// "Sidecar outlier correction"): replacing w = c by v adds (v - c) x to the
// dot product, so each entry carries delta = v - c (fp32, computed once when
// the handle is built). The main loop decodes with the codebook alone; at the
// end of each tile segment, the row's patch list (bounds loaded when the
// segment starts) adds delta * x[k] for the entries in the segment's columns.
#include <algorithm>
#include <climits>

#include "hxq_internal.cuh"

namespace hxq {
namespace {

constexpr int kGemvThreads = 512;
constexpr int kGroups = kGemvThreads / kTileRows;  // virtual CTAs per CTA
constexpr size_t kSmemLimit = 227 * 1024;          // dynamic shared memory per CTA

// Dynamic shared memory of one CTA: codebook table, activations (fp32 or
// bf16) and the groups' partial sums.
inline size_t gemv_smem(int mode, int MT, int Kp, bool xf32) {
  return (size_t)(mode == HXQ_MODE_SCALAR8 ? 256 * 256 : 4096 * 8) + (size_t)MT * Kp * (xf32 ? 4 : 2) +
         (size_t)kGroups * MT * kTileRows * sizeof(float);
}

template <int MODE>
constexpr int table_bytes() { return MODE == HXQ_MODE_SCALAR8 ? 256 * 256 : 4096 * 8; }

__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// CTA whose item range [b W / G, (b+1) W / G) contains item w (W * G < 2^31).
__device__ __forceinline__ int cta_of(int w, int W, int G) {
  int b = (w * G) / W;
  while (b + 1 < G && ((b + 1) * W) / G <= w) ++b;
  while (b > 0 && (b * W) / G > w) --b;
  return b;
}

// Load the NP 16-byte index pieces of stage `st` of row r in tile t.
template <int NP>
__device__ __forceinline__ void load_stage(const Layer& L, int t, int st, int r, uint4 (&q)[NP]) {
  const int rows = min(kTileRows, L.N - t * kTileRows);
  if (r < rows) {
    const uint8_t* p = L.idx + (size_t)t * kTileRows * L.KC * 16 * L.P + ((size_t)st * NP) * rows * 16 + r * 16;
#pragma unroll
    for (int j = 0; j < NP; ++j) q[j] = ldg_stream16(p + (size_t)j * rows * 16);
  } else {
#pragma unroll
    for (int j = 0; j < NP; ++j) q[j] = make_uint4(0, 0, 0, 0);
  }
}

// 16 activations x[m][k0 .. k0+16) from shared memory as fp32.
template <bool XF32>
__device__ __forceinline__ void x16(const uint8_t* xs, int Kp, int m, int k0, float (&f)[16]) {
  if (XF32) {
    const float4* p = reinterpret_cast<const float4*>(xs + ((size_t)m * Kp + k0) * 4);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float4 v = p[i];
      f[4 * i] = v.x; f[4 * i + 1] = v.y; f[4 * i + 2] = v.z; f[4 * i + 3] = v.w;
    }
  } else {
    const uint4* p = reinterpret_cast<const uint4*>(xs + ((size_t)m * Kp + k0) * 2);
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const uint4 v = p[i];
      const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        f[8 * i + 2 * j] = bf16lo(u[j]);
        f[8 * i + 2 * j + 1] = bf16hi(u[j]);
      }
    }
  }
}

template <int MT, bool XF32>
__device__ __forceinline__ void accumulate16(float2 (&acc)[MT], const float (&w)[16], const uint8_t* xs, int Kp,
                                             int k0) {
#pragma unroll
  for (int m = 0; m < MT; ++m) {
    float xv[16];
    x16<XF32>(xs, Kp, m, k0, xv);
#pragma unroll
    for (int j = 0; j < 16; j += 2)
      acc[m] = __ffma2_rn(make_float2(w[j], w[j + 1]), make_float2(xv[j], xv[j + 1]), acc[m]);
  }
}

template <int MT, bool XF32>
__device__ __forceinline__ void add_patch(float2 (&acc)[MT], float d, const uint8_t* xs, int Kp, int k) {
#pragma unroll
  for (int m = 0; m < MT; ++m) {
    const float xv = XF32 ? *reinterpret_cast<const float*>(xs + ((size_t)m * Kp + k) * 4)
                          : bf16lo(*reinterpret_cast<const uint16_t*>(xs + ((size_t)m * Kp + k) * 2));
    acc[m].x = fmaf(d, xv, acc[m].x);
  }
}

// Byte offset of the first index piece of item w (tile-major order, NP
// pieces per row and stage); the items of any contiguous range occupy one
// contiguous byte range. Item W (one past the last) maps to the end.
template <int NP>
__device__ __forceinline__ size_t item_offset(const Layer& L, int w, int n_st) {
  const int t = w / n_st, st = w % n_st;
  if (t >= L.n_tiles) return (size_t)L.N * L.KC * 16 * L.P;
  const int rows = min(kTileRows, L.N - t * kTileRows);
  return (size_t)t * kTileRows * L.KC * 16 * L.P + (size_t)st * NP * rows * 16;
}

template <int MT, bool XF32, int MODE>
__global__ void __launch_bounds__(kGemvThreads, 1)
gemv_kernel(Layer L, const uint16_t* __restrict__ x, float* __restrict__ y, int M, int W,
            float* __restrict__ work, int* __restrict__ counters) {
  extern __shared__ __align__(16) uint8_t smem[];
  constexpr int TB = table_bytes<MODE>();
  constexpr int NP = MODE == HXQ_MODE_SCALAR8 ? 4 : 3;  // 16-byte pieces per stage
  uint8_t* xs = smem + TB;
  // per-group partial sums [kGroups][MT][kTileRows], after the activations
  float* red = reinterpret_cast<float*>(xs + (size_t)MT * L.Kp * (XF32 ? 4 : 2));
  __shared__ int last_flag;

  const int g = threadIdx.x >> 7, r = threadIdx.x & (kTileRows - 1), lane = threadIdx.x & 31;
  const int n_st = n_stages(L);
  const int G = gridDim.x;
  const int w0 = (blockIdx.x * W) / G, w1 = ((blockIdx.x + 1) * W) / G;

  // 0. the next kernel in the stream may start its own prologue
  pdl_launch_dependents();
  // 1. stream this CTA's whole index range into L2 (TMA bulk prefetch), then
  //    issue this thread's first item load; items of this thread are
  //    w0 + g, w0 + g + 4, ...
  if (threadIdx.x == 0 && w1 > w0) {
    const size_t a = item_offset<NP>(L, w0, n_st), b = item_offset<NP>(L, w1, n_st);
    for (size_t o = a; o < b; o += 65536) prefetch_l2_bulk(L.idx + o, (uint32_t)min((size_t)65536, b - o));
  }
  uint4 cur[NP];
  int nt = (w0 + g) / n_st, nst = (w0 + g) % n_st;  // next item to load
  if (w0 + g < w1) load_stage<NP>(L, nt, nst, r, cur);

  // 2. shared-memory codebook; activations once the previous kernel is done
  // (compile-time trip counts: all of a thread's codebook loads are in
  // flight together)
  if (MODE == HXQ_MODE_SCALAR8) {
    constexpr int PER = 256 * 32 / kGemvThreads;
    float cv[PER];
#pragma unroll
    for (int j = 0; j < PER; ++j) cv[j] = __ldg(L.codebook + ((threadIdx.x + j * kGemvThreads) >> 5));
    float* tw = reinterpret_cast<float*>(smem);
#pragma unroll
    for (int j = 0; j < PER; ++j) {
      const int i = threadIdx.x + j * kGemvThreads;
      tw[(i >> 5) * 64 + (i & 31)] = cv[j];
    }
  } else {
    constexpr int PER = 2048 / kGemvThreads;
    const float4* cb = reinterpret_cast<const float4*>(L.codebook);
    float4 cv[PER];
#pragma unroll
    for (int j = 0; j < PER; ++j) cv[j] = __ldg(cb + threadIdx.x + j * kGemvThreads);
#pragma unroll
    for (int j = 0; j < PER; ++j) reinterpret_cast<float4*>(smem)[threadIdx.x + j * kGemvThreads] = cv[j];
  }
  pdl_wait();
  {
    constexpr int XU = 4;  // activation loads in flight per thread
    const int n8 = MT * (L.Kp / 8);
    for (int i0 = threadIdx.x; i0 < n8; i0 += XU * kGemvThreads) {
      uint4 q[XU];
#pragma unroll
      for (int u = 0; u < XU; ++u) {
        const int i = i0 + u * kGemvThreads;
        const int m = i / (L.Kp / 8), k = (i % (L.Kp / 8)) * 8;
        q[u] = make_uint4(0, 0, 0, 0);
        if (i < n8 && m < M && k < L.K) q[u] = __ldg(reinterpret_cast<const uint4*>(x + (size_t)m * L.K + k));
      }
#pragma unroll
      for (int u = 0; u < XU; ++u) {
        const int i = i0 + u * kGemvThreads;
        if (i >= n8) break;
        const int m = i / (L.Kp / 8), k = (i % (L.Kp / 8)) * 8;
        if (XF32) {
          float4* d = reinterpret_cast<float4*>(xs + ((size_t)m * L.Kp + k) * 4);
          d[0] = make_float4(bf16lo(q[u].x), bf16hi(q[u].x), bf16lo(q[u].y), bf16hi(q[u].y));
          d[1] = make_float4(bf16lo(q[u].z), bf16hi(q[u].z), bf16lo(q[u].w), bf16hi(q[u].w));
        } else {
          *reinterpret_cast<uint4*>(xs + ((size_t)m * L.Kp + k) * 2) = q[u];
        }
      }
    }
  }
  __syncthreads();

  const uint32_t lane4 = (uint32_t)lane * 4u;
  nst += kGroups;  // (nt, nst): item after the current one
  while (nst >= n_st) { nst -= n_st; ++nt; }

  for (int seg0 = w0; seg0 < w1;) {  // segments: the CTA's items of one tile
    const int t = seg0 / n_st;
    const int seg1 = min(w1, (t + 1) * n_st);
    // group 0 adds the sidecar corrections of row n; its list bounds load now
    const int n = t * kTileRows + r;
    int pr0 = 0, pr1 = 0;
    if (g == 0 && n < L.N) {
      pr0 = __ldg(L.row_ptr + n);
      pr1 = __ldg(L.row_ptr + n + 1);
    }
    float2 acc[MT];
#pragma unroll
    for (int m = 0; m < MT; ++m) acc[m] = make_float2(0.f, 0.f);

    // this thread's items of the segment: w == w0 + g (mod 4)
    for (int w = seg0 + ((w0 + g - seg0) % kGroups + kGroups) % kGroups; w < seg1; w += kGroups) {
      // next item's loads go out first; they land while this item computes
      uint4 nxt[NP];
      if (w + kGroups < w1) load_stage<NP>(L, nt, nst, r, nxt);
      nst += kGroups;
      while (nst >= n_st) { nst -= n_st; ++nt; }

      const int kst = (w - t * n_st) * kStageK;
      if (MODE == HXQ_MODE_SCALAR8) {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const uint32_t wd[4] = {cur[c].x, cur[c].y, cur[c].z, cur[c].w};
          float wv[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const uint32_t a = prmt(wd[j >> 2], lane4, 0x5504u | ((uint32_t)(j & 3) << 4));
            wv[j] = *reinterpret_cast<const float*>(smem + a);
          }
          accumulate16<MT, XF32>(acc, wv, xs, L.Kp, kst + c * 16);
        }
      } else {
        uint32_t wd[13];
#pragma unroll
        for (int c = 0; c < 3; ++c) {
          wd[4 * c] = cur[c].x; wd[4 * c + 1] = cur[c].y; wd[4 * c + 2] = cur[c].z; wd[4 * c + 3] = cur[c].w;
        }
        wd[12] = 0;
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          float wv[16];
#pragma unroll
          for (int jj = 0; jj < 8; ++jj) {
            const int j = h * 8 + jj, bit = 12 * j;
            const uint32_t e8 = (bit & 31) >= 3
                ? (__funnelshift_r(wd[bit >> 5], wd[(bit >> 5) + 1], (bit & 31) - 3) & 0x7FF8u)
                : ((wd[bit >> 5] << (3 - (bit & 31))) & 0x7FF8u);
            const float2 pr = *reinterpret_cast<const float2*>(smem + e8);
            wv[2 * jj] = pr.x;
            wv[2 * jj + 1] = pr.y;
          }
          accumulate16<MT, XF32>(acc, wv, xs, L.Kp, kst + h * 16);
        }
      }
#pragma unroll
      for (int j = 0; j < NP; ++j) cur[j] = nxt[j];
    }

    // sidecar corrections of this segment's columns: acc += delta * x[k]
    if (pr1 > pr0) {
      const int ka = (seg0 - t * n_st) * kStageK, kb = (seg1 - t * n_st) * kStageK;
#pragma unroll 1
      for (int p = pr0; p < pr1; ++p) {
        const int k = __ldg(L.pk + p);
        if (k >= ka && k < kb) add_patch<MT, XF32>(acc, __ldg(L.pd + p), xs, L.Kp, k);
      }
    }

    // segment end: the 4 groups' sums meet in shared memory
#pragma unroll
    for (int m = 0; m < MT; ++m) red[(g * MT + m) * kTileRows + r] = acc[m].x + acc[m].y;
    __syncthreads();
    const int rows = min(kTileRows, L.N - t * kTileRows);
    const bool full = seg0 == t * n_st && seg1 == (t + 1) * n_st;
    const int slot = (t == w0 / n_st) ? 0 : 1;
    float* part = work + (size_t)(blockIdx.x * 2 + slot) * MT * kTileRows;
    for (int i = threadIdx.x; i < MT * kTileRows; i += blockDim.x) {
      const int m = i / kTileRows, rr = i % kTileRows;
      const float v = red[(0 * MT + m) * kTileRows + rr] + red[(1 * MT + m) * kTileRows + rr] +
                      red[(2 * MT + m) * kTileRows + rr] + red[(3 * MT + m) * kTileRows + rr];
      if (full) {
        if (m < M && rr < rows) y[(size_t)m * L.N + t * kTileRows + rr] = v;
      } else {
        part[i] = v;
      }
    }
    if (!full) {
      __threadfence();
      __syncthreads();
      const int c_first = cta_of(t * n_st, W, G), c_last = cta_of((t + 1) * n_st - 1, W, G);
      if (threadIdx.x == 0) last_flag = atomicAdd(counters + t, 1) == c_last - c_first;
      __syncthreads();
      if (last_flag) {
        __threadfence();
        for (int i = threadIdx.x; i < MT * kTileRows; i += blockDim.x) {
          const int m = i / kTileRows, rr = i % kTileRows;
          if (m >= M || rr >= rows) continue;
          float v = 0.f;
#pragma unroll 4
          for (int c = c_first; c <= c_last; ++c) {
            const int cs = (t == ((c * W) / G) / n_st) ? 0 : 1;
            v += __ldcg(work + (size_t)(c * 2 + cs) * MT * kTileRows + i);
          }
          y[(size_t)m * L.N + t * kTileRows + rr] = v;
        }
        if (threadIdx.x == 0) counters[t] = 0;
      }
    }
    __syncthreads();
    seg0 = seg1;
  }
}

template <int MT, bool XF32, int MODE>
cudaError_t launch_cfg(const hxq_linear& h, const uint16_t* x, float* y, int M, int grid, cudaStream_t s) {
  const size_t smem = gemv_smem(MODE, MT, h.L.Kp, XF32);
  auto kern = gemv_kernel<MT, XF32, MODE>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int W = h.L.n_tiles * (h.L.Kp / kStageK);
  return launch_pdl(kern, grid, kGemvThreads, smem, s, h.L, x, y, M, W, h.d_work, h.d_counters);
}

template <int MT, int MODE>
cudaError_t launch_mt(const hxq_linear& h, const uint16_t* x, float* y, int M, int grid, cudaStream_t s) {
  if (gemv_smem(MODE, MT, h.L.Kp, true) <= kSmemLimit) return launch_cfg<MT, true, MODE>(h, x, y, M, grid, s);
  return launch_cfg<MT, false, MODE>(h, x, y, M, grid, s);
}

template <int MODE>
cudaError_t launch_mode(const hxq_linear& h, const uint16_t* x, float* y, int M, int grid, cudaStream_t s) {
  if (M <= 1) return launch_mt<1, MODE>(h, x, y, M, grid, s);
  if (M <= 2) return launch_mt<2, MODE>(h, x, y, M, grid, s);
  if (M <= 4) return launch_mt<4, MODE>(h, x, y, M, grid, s);
  if (M <= 8) return launch_mt<8, MODE>(h, x, y, M, grid, s);
  if (M <= 16) return launch_mt<16, MODE>(h, x, y, M, grid, s);
  return launch_mt<32, MODE>(h, x, y, M, grid, s);
}

int mt_of(int M) { return M <= 1 ? 1 : M <= 2 ? 2 : M <= 4 ? 4 : M <= 8 ? 8 : M <= 16 ? 16 : 32; }

}  // namespace

bool gemv_supports(const hxq_linear& h, int M) {
  return M >= 1 && M <= 32 && gemv_smem(h.L.mode, mt_of(M), h.L.Kp, false) <= kSmemLimit;
}

// Persistent grid: one CTA per SM, fewer when the layer has fewer work items.
// `split` (when non-zero) sets the grid so that each tile's K is shared by
// about `split` CTAs.
cudaError_t launch_gemv(const hxq_linear& h, const uint16_t* x, float* y, int M, int split, cudaStream_t s) {
  if (!gemv_supports(h, M)) return cudaErrorInvalidValue;
  const int64_t W = (int64_t)h.L.n_tiles * (h.L.Kp / kStageK);
  int64_t grid = split > 0 ? (int64_t)h.L.n_tiles * split : h.num_sms;
  grid = std::max<int64_t>(1, std::min<int64_t>({grid, (int64_t)h.num_sms, W}));
  if (W * grid >= INT_MAX) return cudaErrorInvalidValue;  // item arithmetic is 32-bit
  // every CTA writes at most two partial tiles of mt_of(M) x 128 floats
  if ((size_t)grid * 2 * mt_of(M) * kTileRows > h.work_floats) return cudaErrorInvalidValue;
  if (h.L.mode == HXQ_MODE_SCALAR8) return launch_mode<HXQ_MODE_SCALAR8>(h, x, y, M, (int)grid, s);
  return launch_mode<HXQ_MODE_VQ2D12>(h, x, y, M, (int)grid, s);
}

}  // namespace hxq
