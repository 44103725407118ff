// Fused decode + GEMV on CUDA cores for few tokens (M <= 4 by default; up to
// M = 16 on request): y[m][n] = sum_k x[m][k] * W[n][k] with W decoded on the
// fly from the codebook and never written anywhere (the pages' buffered path
// instead materialises W and calls cuBLAS: HXQ whitepaper, method section,
// buffered forward path paragraph).
//
// Work decomposition (stream-K). The work items are the tile-stages of the
// layer, (tile of 128 rows) x (64 weights along K), numbered tile-major; an
// item's indices are one contiguous block of the tiled layout. A persistent
// grid of one CTA per SM takes contiguous item ranges of equal size, so every
// CTA streams the same number of index bytes whatever the layer shape.
//
// Inside a CTA a producer warp streams the items' index blocks with TMA bulk
// copies into a ring of shared-memory slots (up to 12 x 8 KB in flight per
// SM; it starts before the previous kernel has finished, since the indices do
// not depend on it), and 4 groups of 128 consumer threads take the items
// round-robin: thread r of a group owns row r of the item's tile, reads its
// 16-byte pieces from the slot, releases the slot and decodes. At each tile
// boundary of the CTA's range the groups' sums meet in shared memory; a tile
// covered by one CTA goes straight to y, a tile split between CTAs leaves one
// fp32 partial per CTA in the workspace and the last CTA to arrive (integer
// atomic per tile) adds them in CTA order: results are bitwise repeatable.
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
// the handle is built). The main loop decodes with the codebook alone; each
// group loads its share of the row's patch entries when a tile segment
// starts (list bounds fetched one segment ahead) and adds delta * x[k] for
// those in the segment's columns at its end -- no dependent memory access on
// the critical path.
#include <algorithm>
#include <climits>

#include "hxq_internal.cuh"

namespace hxq {
namespace {

constexpr int kGemvThreads = 512;                  // consumers; one more warp produces
constexpr int kGroups = kGemvThreads / kTileRows;  // consumer groups (128 rows each)
constexpr int kMaxRing = 12;                       // index slots in flight per CTA
constexpr size_t kSmemLimit = 226 * 1024;          // dynamic shared memory per CTA (static kept apart)

// Dynamic shared memory of one CTA: codebook table, activations (fp32 or
// bf16) and the groups' partial sums, then the index ring.
inline size_t gemv_smem_fixed(int mode, int MT, int Kp, bool xf32) {
  return (size_t)(mode == HXQ_MODE_SCALAR8 ? 256 * 256 : 4096 * 8) + (size_t)MT * Kp * (xf32 ? 4 : 2) +
         (size_t)kGroups * MT * kTileRows * sizeof(float);
}
inline int slot_bytes(int mode) { return (mode == HXQ_MODE_SCALAR8 ? 4 : 3) * kTileRows * 16; }
// Ring slots that fit next to the fixed part (a multiple of the groups; 0 if
// fewer than one per group fit).
inline int ring_slots(int mode, int MT, int Kp, bool xf32) {
  const size_t fixed = gemv_smem_fixed(mode, MT, Kp, xf32);
  if (fixed + 128 > kSmemLimit) return 0;
  const int fit = (int)((kSmemLimit - fixed - 128) / slot_bytes(mode));
  return std::min(kMaxRing, fit / kGroups * kGroups);
}
inline size_t gemv_smem(int mode, int MT, int Kp, bool xf32) {
  return gemv_smem_fixed(mode, MT, Kp, xf32) + 128 + (size_t)ring_slots(mode, MT, Kp, xf32) * slot_bytes(mode);
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

__device__ __forceinline__ void consumer_sync() {
  asm volatile("bar.sync 1, %0;" ::"r"(kGemvThreads) : "memory");
}

template <int MT, bool XF32, int MODE>
__global__ void __launch_bounds__(kGemvThreads + 32, 1)
gemv_kernel(Layer L, const uint16_t* __restrict__ x, float* __restrict__ y, int M, int W, int R,
            float* __restrict__ work, int* __restrict__ counters, int* __restrict__ status) {
  extern __shared__ __align__(16) uint8_t smem[];
  constexpr int TB = table_bytes<MODE>();
  constexpr int NP = MODE == HXQ_MODE_SCALAR8 ? 4 : 3;  // 16-byte pieces per row and stage
  uint8_t* xs = smem + TB;
  // per-group partial sums [kGroups][MT][kTileRows], after the activations
  float* red = reinterpret_cast<float*>(xs + (size_t)MT * L.Kp * (XF32 ? 4 : 2));
  uint8_t* ring = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(red + kGroups * MT * kTileRows) + 127) & ~(uintptr_t)127);
  constexpr int SLOT = NP * kTileRows * 16;
  __shared__ uint64_t bar_full[kMaxRing], bar_empty[kMaxRing];
  __shared__ int last_flag, abort_sh;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_st = n_stages(L);
  const int G = gridDim.x;
  const int w0 = (blockIdx.x * W) / G, w1 = ((blockIdx.x + 1) * W) / G;
  volatile int* abrt = &abort_sh;

  if (threadIdx.x == 0) {
    for (int i = 0; i < R; ++i) {
      mbar_init(&bar_full[i], 1);
      mbar_init(&bar_empty[i], 4);  // the 4 warps of the consuming group
    }
    abort_sh = 0;
    fence_mbar_init();
  }
  __syncthreads();
  pdl_launch_dependents();  // the next kernel in the stream may start its prologue

  if (warp == kGemvThreads / 32) {
    // ---------------- producer: index blocks of the CTA's items, in order
    if (lane == 0) {
      int issued = 0;
      for (int i = 0; i < w1 - w0; ++i) {
        const int s = i % R;
        if (!mbar_wait(&bar_empty[s], ((i / R) & 1) ^ 1, abrt)) break;
        const int w = w0 + i, t = w / n_st, st = w % n_st;
        const int rows = min(kTileRows, L.N - t * kTileRows);
        const uint32_t bytes = (uint32_t)(NP * rows * 16);
        mbar_arrive_expect_tx(&bar_full[s], bytes);
        bulk_load(ring + (size_t)s * SLOT,
                  L.idx + (size_t)t * kTileRows * L.KC * 16 * L.P + (size_t)st * NP * rows * 16, bytes,
                  &bar_full[s]);
        ++issued;
      }
      if (*abrt) {  // let the copies this thread issued land before the CTA ends
        volatile int never = 0;
        for (int i = max(0, issued - R); i < issued; ++i) mbar_wait(&bar_full[i % R], (i / R) & 1, &never);
      }
    }
    __syncthreads();
    return;
  }

  // ---------------- consumers
  const int g = threadIdx.x >> 7, r = threadIdx.x & (kTileRows - 1);
  // shared-memory codebook (compile-time trip counts: a thread's codebook
  // loads are all in flight together)
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
  // activations (zero-padded to Kp) once the previous kernel is done
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
  consumer_sync();

  const uint32_t lane4 = (uint32_t)lane * 4u;
  bool waited_ok = true;  // after a timed-out wait the data is garbage but every barrier is still met

  // Sidecar: bounds of this thread's row list for the first segment (the
  // next segment's bounds are fetched one segment ahead).
  constexpr int kPE = 4;  // entries per group held in registers (16 per row)
  int pr0 = 0, pr1 = 0;
  {
    const int n0 = (w0 / n_st) * kTileRows + r;
    if (w0 < w1 && n0 < L.N) {
      pr0 = __ldg(L.row_ptr + n0);
      pr1 = __ldg(L.row_ptr + n0 + 1);
    }
  }

  for (int seg0 = w0; seg0 < w1;) {  // segments: the CTA's items of one tile
    const int t = seg0 / n_st;
    const int seg1 = min(w1, (t + 1) * n_st);
    const int rows = min(kTileRows, L.N - t * kTileRows);
    const int n = t * kTileRows + r;
    // this group's share of row n's patch entries (p = pr0 + g + 4j), loaded
    // now and applied at the segment end
    int ek[kPE];
    float ed[kPE];
#pragma unroll
    for (int j = 0; j < kPE; ++j) {
      const int p = pr0 + g + kGroups * j;
      ek[j] = p < pr1 ? __ldg(L.pk + p) : INT_MAX;
      ed[j] = p < pr1 ? __ldg(L.pd + p) : 0.f;
    }
    const int cur0 = pr0, cur1 = pr1;
    // next segment's list bounds
    pr0 = pr1 = 0;
    if (seg1 < w1 && n + kTileRows < L.N) {
      pr0 = __ldg(L.row_ptr + n + kTileRows);
      pr1 = __ldg(L.row_ptr + n + kTileRows + 1);
    }
    float2 acc[MT];
#pragma unroll
    for (int m = 0; m < MT; ++m) acc[m] = make_float2(0.f, 0.f);

    // this group's items of the segment: w == w0 + g (mod 4)
    for (int w = seg0 + ((w0 + g - seg0) % kGroups + kGroups) % kGroups; w < seg1; w += kGroups) {
      const int i = w - w0, s = i % R;
      if (waited_ok) waited_ok = mbar_wait(&bar_full[s], (i / R) & 1, abrt);
      uint4 cur[NP];
#pragma unroll
      for (int j = 0; j < NP; ++j)
        cur[j] = r < rows ? *reinterpret_cast<const uint4*>(ring + (size_t)s * SLOT + (j * rows + r) * 16)
                          : make_uint4(0, 0, 0, 0);
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar_empty[s]);

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
    }

    // sidecar corrections of this segment's columns: acc += delta * x[k]
    {
      const int ka = (seg0 - t * n_st) * kStageK, kb = (seg1 - t * n_st) * kStageK;
#pragma unroll
      for (int j = 0; j < kPE; ++j)
        if (ek[j] >= ka && ek[j] < kb) add_patch<MT, XF32>(acc, ed[j], xs, L.Kp, ek[j]);
#pragma unroll 1
      for (int p = cur0 + g + kGroups * kPE; p < cur1; p += kGroups) {  // rows with > 16 entries
        const int k = __ldg(L.pk + p);
        if (k >= ka && k < kb) add_patch<MT, XF32>(acc, __ldg(L.pd + p), xs, L.Kp, k);
      }
    }

    // segment end: the 4 groups' sums meet in shared memory
#pragma unroll
    for (int m = 0; m < MT; ++m) red[(g * MT + m) * kTileRows + r] = acc[m].x + acc[m].y;
    consumer_sync();
    const bool full = seg0 == t * n_st && seg1 == (t + 1) * n_st;
    const int slot = (t == w0 / n_st) ? 0 : 1;
    float* part = work + (size_t)(blockIdx.x * 2 + slot) * MT * kTileRows;
    for (int i = threadIdx.x; i < MT * kTileRows; i += kGemvThreads) {
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
      consumer_sync();
      const int c_first = cta_of(t * n_st, W, G), c_last = cta_of((t + 1) * n_st - 1, W, G);
      if (threadIdx.x == 0) last_flag = atomicAdd(counters + t, 1) == c_last - c_first;
      consumer_sync();
      if (last_flag) {
        __threadfence();
        for (int i = threadIdx.x; i < MT * kTileRows; i += kGemvThreads) {
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
    consumer_sync();
    seg0 = seg1;
  }
  if (!waited_ok && threadIdx.x == 0) atomicOr(status, kStatusWaitTimeout);
  __syncthreads();
}

template <int MT, bool XF32, int MODE>
cudaError_t launch_cfg(const hxq_linear& h, const uint16_t* x, float* y, int M, int grid, float* work, int* counters,
                       cudaStream_t s) {
  const int R = ring_slots(MODE, MT, h.L.Kp, XF32);
  if (R < kGroups) return cudaErrorInvalidValue;
  const size_t smem = gemv_smem(MODE, MT, h.L.Kp, XF32);
  auto kern = gemv_kernel<MT, XF32, MODE>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int W = h.L.n_tiles * (h.L.Kp / kStageK);
  return launch_pdl(kern, grid, kGemvThreads + 32, smem, s, h.L, x, y, M, W, R, work, counters, h.d_status);
}

template <int MT, int MODE>
cudaError_t launch_mt(const hxq_linear& h, const uint16_t* x, float* y, int M, int grid, float* work, int* counters,
                      cudaStream_t s) {
  if (ring_slots(MODE, MT, h.L.Kp, true) >= kGroups)
    return launch_cfg<MT, true, MODE>(h, x, y, M, grid, work, counters, s);
  return launch_cfg<MT, false, MODE>(h, x, y, M, grid, work, counters, s);
}

template <int MODE>
cudaError_t launch_mode(const hxq_linear& h, const uint16_t* x, float* y, int M, int grid, float* work, int* counters,
                        cudaStream_t s) {
  if (M <= 1) return launch_mt<1, MODE>(h, x, y, M, grid, work, counters, s);
  if (M <= 2) return launch_mt<2, MODE>(h, x, y, M, grid, work, counters, s);
  if (M <= 4) return launch_mt<4, MODE>(h, x, y, M, grid, work, counters, s);
  if (M <= 8) return launch_mt<8, MODE>(h, x, y, M, grid, work, counters, s);
  return launch_mt<16, MODE>(h, x, y, M, grid, work, counters, s);
}

int mt_of(int M) { return M <= 1 ? 1 : M <= 2 ? 2 : M <= 4 ? 4 : M <= 8 ? 8 : 16; }

}  // namespace

bool gemv_supports(const hxq_linear& h, int M) {
  return M >= 1 && M <= 16 && ring_slots(h.L.mode, mt_of(M), h.L.Kp, false) >= kGroups;
}

// Persistent grid: one CTA per SM, fewer when the layer has fewer work items.
// `split` (when non-zero) sets the grid so that each tile's K is shared by
// about `split` CTAs.
int gemv_grid(const hxq_linear& h, int split) {
  const int64_t W = (int64_t)h.L.n_tiles * (h.L.Kp / kStageK);
  int64_t grid = split > 0 ? (int64_t)h.L.n_tiles * split : h.num_sms;
  grid = std::max<int64_t>(1, std::min<int64_t>({grid, (int64_t)h.num_sms, W}));
  if (W * grid >= INT_MAX) return 0;  // item arithmetic is 32-bit
  return (int)grid;
}

cudaError_t launch_gemv(const hxq_linear& h, const uint16_t* x, float* y, int M, int split, cudaStream_t s) {
  if (!gemv_supports(h, M)) return cudaErrorInvalidValue;
  const int grid = gemv_grid(h, split);
  if (grid == 0) return cudaErrorInvalidValue;
  // every CTA writes at most two partial tiles of mt_of(M) x 128 floats
  if ((size_t)grid * 2 * mt_of(M) * kTileRows > h.work_floats) return cudaErrorInvalidValue;
  if (h.L.mode == HXQ_MODE_SCALAR8) return launch_mode<HXQ_MODE_SCALAR8>(h, x, y, M, grid, h.d_work, h.d_counters, s);
  return launch_mode<HXQ_MODE_VQ2D12>(h, x, y, M, grid, h.d_work, h.d_counters, s);
}

}  // namespace hxq

// ----------------------------------------------------------------------------
// hxq_linear_forward_noalloc: the CUDA-core GEMV with its scratch -- the
// stream-K arrival counters and partial sums -- in a fixed array compiled
// into this library instead of the handle's workspace. Nothing is allocated
// on this path; the array stays resident on every GPU that loads the library
// until the process exits.
// ----------------------------------------------------------------------------
#include <mutex>

namespace hxq {
namespace {
constexpr int kNoAllocMaxTiles = 4096;                   // N <= 524288 output features
constexpr size_t kNoAllocPartialFloats = 256 * 1024;     // 1 MiB of fp32 partial sums
constexpr size_t kNoAllocScratchBytes = kNoAllocMaxTiles * sizeof(int) + kNoAllocPartialFloats * sizeof(float);
}  // namespace
}  // namespace hxq

// [0, 16 KB): per-tile arrival counters (must start at zero); then partials.
static __device__ __align__(256) unsigned char g_noalloc_scratch[hxq::kNoAllocScratchBytes];

namespace {
std::mutex g_noalloc_mu;
void* g_noalloc_addr[256];  // device address of g_noalloc_scratch, per device ordinal

// Device address of the scratch array on device `dev` (current). In host code
// the array's name is only a host-side stand-in, so the address comes from
// cudaGetSymbolAddress, once per device.
cudaError_t noalloc_scratch(int dev, void** out) {
  if (dev < 0 || dev >= 256) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_addr[dev]) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_noalloc_addr[dev] = p;
  }
  *out = g_noalloc_addr[dev];
  return cudaSuccess;
}
}  // namespace

extern "C" int hxq_linear_forward_noalloc(hxq_linear_t h, const void* x_bf16, float* y, int M, void* stream) {
  using namespace hxq;
  if (!h || !x_bf16 || !y || M < 1 || M > 4) return HXQ_EINVAL;
  if ((reinterpret_cast<uintptr_t>(x_bf16) & 15) != 0) return HXQ_EINVAL;
  if (!gemv_supports(*h, M) || h->L.n_tiles > kNoAllocMaxTiles) return HXQ_EINVAL;
  const int grid = gemv_grid(*h, 0);
  if (grid == 0 || (size_t)grid * 2 * mt_of(M) * kTileRows > kNoAllocPartialFloats) return HXQ_EINVAL;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return HXQ_ECUDA;
  }
  if (dev != h->device) return HXQ_EINVAL;
  void* base = nullptr;
  if (noalloc_scratch(dev, &base) != cudaSuccess) {
    cudaGetLastError();
    return HXQ_ECUDA;
  }
  int* counters = static_cast<int*>(base);
  float* work = reinterpret_cast<float*>(static_cast<unsigned char*>(base) + kNoAllocMaxTiles * sizeof(int));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // a previous call may have been interrupted mid-way: the counters restart at zero
  cudaError_t e = cudaMemsetAsync(counters, 0, (size_t)h->L.n_tiles * sizeof(int), s);
  if (e == cudaSuccess) {
    const uint16_t* x = static_cast<const uint16_t*>(x_bf16);
    e = h->L.mode == HXQ_MODE_SCALAR8 ? launch_mode<HXQ_MODE_SCALAR8>(*h, x, y, M, grid, work, counters, s)
                                      : launch_mode<HXQ_MODE_VQ2D12>(*h, x, y, M, grid, work, counters, s);
  }
  if (e != cudaSuccess) {
    cudaGetLastError();
    return HXQ_ECUDA;
  }
  return HXQ_OK;
}
