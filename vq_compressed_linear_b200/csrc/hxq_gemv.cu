// Fused decode + GEMV on CUDA cores for few tokens (M <= 4 by default; up to
// M = 8 on request): y[m][n] = sum_k x[m][k] * W[n][k] with W decoded on the
// fly from the codebook and never written anywhere (the pages' buffered path
// instead materialises W and calls cuBLAS: HXQ whitepaper, method section,
// buffered forward path paragraph).
//
// Work decomposition. The layer's stages (tile of 128 rows x 64 weights along
// K) are numbered tile-major. Two ways of cutting them, chosen per handle:
// - cluster split: when some cluster size cs in 2..16 gives one cluster per
//   tile that fills at least 70 % of the SMs (any fill for layers of a few
//   tiles), all clusters resident, tile t goes to cluster t and rank r of it
//   takes the r-th of cs equal K ranges;
// - stream-K otherwise: the stages are cut into contiguous ranges of equal
//   length, one per CTA of a persistent grid (one CTA per SM), so every CTA
//   streams the same number of index bytes whatever the layer shape.
//
// Two launches share an SM. A CTA keeps its shared memory to about half of
// the SM's (a 32 KB codebook table, the activations, a ring of 16 KB slots)
// and its registers to half of the register file, so that while one launch
// drains, the next launch in the stream (programmatic dependent launch)
// already has a CTA on every SM: it builds its table, asks the TMA engine to
// bring its whole index range into L2 (bulk prefetch) and fills its ring,
// and only its activation load waits for the previous launch to finish. HBM
// therefore keeps streaming across launch boundaries.
//
// Inside a CTA a producer warp streams the range in chunks of up to 2 stages
// of one tile (16 KB of scalar indices, contiguous in the tiled layout) with
// TMA bulk copies into the ring; the bulk L2 prefetch runs ahead of it. The
// 8 consumer warps share every chunk: warp q takes the q-th 16-weight piece
// of the chunk (stage q / 4, quarter q % 4) for all 128 rows, lane l for rows
// l, l + 32, l + 64, l + 96. So each activation a warp loads from shared
// memory serves four rows: per 32 weights the decode costs one conflict-free
// table lookup wavefront plus a quarter wavefront of index bytes plus the
// activations (with 8 warps per CTA it runs below that bound, on the
// latency of its lookup chain).
//
// At each tile boundary of the CTA's range the warps' sums meet in shared
// memory. Under the cluster split every rank writes its sums into rank 0's
// shared memory (distributed shared memory) and, after a cluster barrier,
// rank 0 adds them in rank order. Under stream-K a tile covered by one CTA
// goes straight to y; a tile split between CTAs leaves one fp32 partial per
// CTA in the workspace and the last CTA to arrive (integer atomic per tile)
// adds them in CTA order. Either way results are bitwise repeatable.
//
// Scalar codebook in shared memory: replicated once per lane with entry e of
// lane l at byte e*256 + l*4, so the 32 lanes of a lookup always hit 32
// different banks. The byte address is one PRMT away from the index word:
// {0, 0, index byte, l*4}. The table uses the first half of each 256-byte
// row; the other halves hold the activations and the reduction buffers.
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
// the handle is built). The main loop decodes with the codebook alone. When a
// segment starts, the two threads that finish row n load up to four each of
// the row's entries in the segment's columns (found through a per-stage
// lower-bound table, the bounds fetched one segment ahead); at the segment
// end they add delta * x[m][k] to the row's sum.
#include <algorithm>
#include <climits>
#include <type_traits>

#include "hxq_internal.cuh"
#include "hxq_plan.h"

namespace hxq {
namespace {

constexpr int kGemvThreads = 256;                  // consumers; then a producer and a fixup warp
constexpr int kConsumerWarps = kGemvThreads / 32;  // 8: one 16-weight piece of a chunk each
constexpr int kProducerWarp = kConsumerWarps;
constexpr int kFixupWarp = kConsumerWarps + 1;
constexpr int kGemvBlock = kGemvThreads + 64;
constexpr int kBarConsumers = 1;                   // named barrier of the consumers
constexpr int kChunkStages = 2;                    // stages per ring slot (8 pieces per row)
constexpr int kMaxRing = 8;                        // ring slots
constexpr int kGemvMaxM = 8;                       // tokens
constexpr int kSideGroups = kGemvThreads / kTileRows;  // 2 threads per row share its patch entries
constexpr int kPE = 4;                             // patch entries per thread and segment in registers
constexpr size_t kSmemLimit = 226 * 1024;          // dynamic shared memory per CTA (static kept apart)
// At most this much dynamic shared memory per CTA lets two CTAs share an SM:
// 2 x (dynamic + static (under 512 bytes) + 1 KB reserved) <= 228 KB.
constexpr size_t kSmemShared = 113 * 1024 - 512;
constexpr uint32_t kPrefetchAhead = 256 * 1024;    // bulk L2 prefetch distance ahead of the ring
constexpr int kScalarTable = 256 * 256;            // bytes: 256 rows of 32 lanes x fp32, then a 128-byte hole
constexpr uint32_t kHoleBytes = 256 * 128;         // the rows' second halves, used as scratch
constexpr int kPairTable = 4096 * 8;               // bytes: 4096 fp32 pairs

// Scratch of one CTA (bytes): activations (fp32 or bf16), the warps'
// partial sums, the split-tile sums handed to the fixup warp, the sidecar
// corrections and, for a cluster, the cluster's sums of its tile.
inline size_t gemv_scratch(int MT, int Kp, bool xf32, int cs) {
  return (size_t)MT * Kp * (xf32 ? 4 : 2) + (size_t)(kConsumerWarps + 2 + kSideGroups + cs) * MT * kTileRows * sizeof(float);
}
// Dynamic shared memory before the index ring: the codebook table and the
// scratch (in scalar mode partly inside the table's holes).
inline size_t gemv_smem_fixed(int mode, int MT, int Kp, bool xf32, int cs = 0) {
  const size_t sc = gemv_scratch(MT, Kp, xf32, cs);
  if (mode == HXQ_MODE_SCALAR8) return (size_t)kScalarTable + (sc > kHoleBytes ? sc - kHoleBytes : 0);
  return (size_t)kPairTable + sc;
}
inline int slot_bytes(int mode) { return kChunkStages * (mode == HXQ_MODE_SCALAR8 ? 4 : 3) * kTileRows * 16; }
// Ring slots: as many as fit (up to kMaxRing) while two CTAs still share an
// SM; failing that, as many as fit in one CTA per SM; 0 if not even
// kMinRing fit.
constexpr int kMinRing = 2;
constexpr int kMaxCluster = 16;                    // CTAs sharing one tile's K in the cluster split
inline int ring_slots(int mode, int MT, int Kp, bool xf32, int cs = 0) {
  const size_t fixed = gemv_smem_fixed(mode, MT, Kp, xf32, cs) + 128;
  for (size_t cap : {kSmemShared, kSmemLimit}) {
    if (fixed + (size_t)kMinRing * slot_bytes(mode) > cap) continue;
    return std::min(kMaxRing, (int)((cap - fixed) / slot_bytes(mode)));
  }
  return 0;
}
inline size_t gemv_smem(int mode, int MT, int Kp, bool xf32, int cs = 0) {
  return gemv_smem_fixed(mode, MT, Kp, xf32, cs) + 128 + (size_t)ring_slots(mode, MT, Kp, xf32, cs) * slot_bytes(mode);
}
// Activations staged as fp32 (no conversion in the inner loop) unless only
// bf16 staging lets two CTAs share an SM, or fp32 does not fit at all.
inline bool stage_x_f32(int mode, int MT, int Kp) {
  auto shared = [&](bool f32) {
    return gemv_smem_fixed(mode, MT, Kp, f32) + 128 + (size_t)kMinRing * slot_bytes(mode) <= kSmemShared;
  };
  if (shared(true)) return true;
  if (shared(false)) return false;
  return ring_slots(mode, MT, Kp, true) >= kMinRing;
}

template <int MODE>
constexpr int table_bytes() { return MODE == HXQ_MODE_SCALAR8 ? kScalarTable : kPairTable; }

// The CTA's scratch in shared memory, addressed by a logical byte offset: in
// scalar mode the first kHoleBytes lie in the table's holes (the second
// half of each 256-byte row) and the rest follows the table; in 2D mode the
// scratch follows the pair table.
template <int MODE>
struct Scratch {
  uint8_t* smem;
  __device__ __forceinline__ uint8_t* at(uint32_t o) const {
    if (MODE == HXQ_MODE_SCALAR8)
      return smem + (o < kHoleBytes ? ((o >> 7) << 8) + 128 + (o & 127) : kScalarTable + (o - kHoleBytes));
    return smem + kPairTable + o;
  }
  __device__ __forceinline__ float& f(uint32_t o) const { return *reinterpret_cast<float*>(at(o)); }
};

__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// CTA whose stage range [b W / G, (b+1) W / G) contains stage w (W * G < 2^31).
__device__ __forceinline__ int cta_of(int w, int W, int G) {
  int b = (w * G) / W;
  while (b + 1 < G && ((b + 1) * W) / G <= w) ++b;
  while (b > 0 && (b * W) / G > w) --b;
  return b;
}

// 16 activations x[m][k0 .. k0+16) from shared memory as fp32 (the staged
// activations start at scratch offset 0; k0 is a multiple of 16, so the 64
// or 32 bytes never cross a hole).
template <bool XF32, int MODE>
__device__ __forceinline__ void x16(const Scratch<MODE>& sc, int Kp, int m, int k0, float (&f)[16]) {
  if (XF32) {
    const float4* p = reinterpret_cast<const float4*>(sc.at((uint32_t)(m * Kp + k0) * 4));
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float4 v = p[i];
      f[4 * i] = v.x; f[4 * i + 1] = v.y; f[4 * i + 2] = v.z; f[4 * i + 3] = v.w;
    }
  } else {
    const uint4* p = reinterpret_cast<const uint4*>(sc.at((uint32_t)(m * Kp + k0) * 2));
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

__device__ __forceinline__ void fma16(float2& acc, const float (&w)[16], const float (&xv)[16]) {
#pragma unroll
  for (int j = 0; j < 16; j += 2) acc = __ffma2_rn(make_float2(w[j], w[j + 1]), make_float2(xv[j], xv[j + 1]), acc);
}
// One register per sum (scalar FMAs) where paired sums would not fit.
__device__ __forceinline__ void fma16(float& acc, const float (&w)[16], const float (&xv)[16]) {
#pragma unroll
  for (int j = 0; j < 16; ++j) acc = fmaf(w[j], xv[j], acc);
}
__device__ __forceinline__ float acc_sum(float2 a) { return a.x + a.y; }
__device__ __forceinline__ float acc_sum(float a) { return a; }
__device__ __forceinline__ void acc_zero(float2& a) { a = make_float2(0.f, 0.f); }
__device__ __forceinline__ void acc_zero(float& a) { a = 0.f; }

template <int MODE>
__device__ __forceinline__ float x_at(const Scratch<MODE>& sc, int Kp, int m, int k, bool xf32) {
  return xf32 ? *reinterpret_cast<const float*>(sc.at((uint32_t)(m * Kp + k) * 4))
              : bf16lo(*reinterpret_cast<const uint16_t*>(sc.at((uint32_t)(m * Kp + k) * 2)));
}

// The 16 weights of one row's piece: scalar indices (one 16-byte piece).
// lane4 = 4 * lane (scalar table addressing).
template <int MODE>
__device__ __forceinline__ void decode16(const uint8_t* smem, const uint8_t* piece, int rows, int quarter,
                                         uint32_t lane4, float (&wv)[16]) {
  if (MODE == HXQ_MODE_SCALAR8) {
    const uint4 cur = *reinterpret_cast<const uint4*>(piece);
    const uint32_t wd[4] = {cur.x, cur.y, cur.z, cur.w};
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const uint32_t a = prmt(wd[j >> 2], lane4, 0x5504u | ((uint32_t)(j & 3) << 4));
      wv[j] = *reinterpret_cast<const float*>(smem + a);
    }
  } else {
    // the quarter's 8 pairs are bytes [12 q, 12 q + 12) of the row's 48 in
    // the stage's three 16-byte planes (`piece` points at plane 0)
    uint32_t wd[4] = {0, 0, 0, 0};
    const uint8_t* p1 = piece + rows * 16;
    const uint8_t* p2 = p1 + rows * 16;
    if (quarter == 0) {
      const uint4 v = *reinterpret_cast<const uint4*>(piece);
      wd[0] = v.x; wd[1] = v.y; wd[2] = v.z;
    } else if (quarter == 1) {
      const uint2 v = *reinterpret_cast<const uint2*>(p1);
      wd[0] = *reinterpret_cast<const uint32_t*>(piece + 12); wd[1] = v.x; wd[2] = v.y;
    } else if (quarter == 2) {
      const uint2 v = *reinterpret_cast<const uint2*>(p1 + 8);
      wd[0] = v.x; wd[1] = v.y; wd[2] = *reinterpret_cast<const uint32_t*>(p2);
    } else {
      const uint4 v = *reinterpret_cast<const uint4*>(p2);
      wd[0] = v.y; wd[1] = v.z; wd[2] = v.w;
    }
#pragma unroll
    for (int jj = 0; jj < 8; ++jj) {
      const int bit = 12 * jj;
      const uint32_t e8 = (bit & 31) >= 3
          ? (__funnelshift_r(wd[bit >> 5], wd[(bit >> 5) + 1], (bit & 31) - 3) & 0x7FF8u)
          : ((wd[bit >> 5] << (3 - (bit & 31))) & 0x7FF8u);
      const float2 pr = *reinterpret_cast<const float2*>(smem + e8);
      wv[2 * jj] = pr.x;
      wv[2 * jj + 1] = pr.y;
    }
  }
}

__device__ __forceinline__ void consumer_sync() { named_bar_sync(kBarConsumers, kGemvThreads); }

// The CTA's stage range [w0, w1) as segments (its stages of one tile each),
// in processing order. A range that ends inside a tile shared with the next
// CTA processes that split tile first: the next CTA reaches its own part of
// the tile at the end of its range, so by then this CTA's sum has long been
// counted, and the CTA that finishes a split tile last finds the other sums
// ready. Split segments take partial-sum slot 0 (the range's first tile) or
// 1 (its last tile).
struct Segments {
  int w0, w1, n_st, tf, tl, n;
  bool reorder;
  __device__ Segments(int w0_, int w1_, int n_st_) : w0(w0_), w1(w1_), n_st(n_st_) {
    tf = w0 / n_st;
    tl = (w1 - 1) / n_st;
    n = tl - tf + 1;
    reorder = n >= 2 && w1 != (tl + 1) * n_st;
  }
  __device__ int tile(int k) const { return reorder ? (k == 0 ? tl : tf + k - 1) : tf + k; }
  __device__ int begin(int k) const { return max(w0, tile(k) * n_st); }
  __device__ int end(int k) const { return min(w1, (tile(k) + 1) * n_st); }
  __device__ bool split(int k) const {
    const int t = tile(k);
    return begin(k) != t * n_st || end(k) != (t + 1) * n_st;
  }
  __device__ int slot(int k) const { return tile(k) == tf ? 0 : 1; }
};

// y rows of tile t from the sums of its contributors c_first..c_last, added
// in CTA order: this CTA's own sum from the scratch at offset `own`, the
// others' from the workspace (a batch of contributors' loads in flight per
// sum).
template <int MT, int MODE>
__device__ __forceinline__ void finish_tile(const Layer& L, const Out& out, const float* __restrict__ work,
                                            const Scratch<MODE>& sc, uint32_t own, int M, int t, int c_first,
                                            int c_last, int b, int W, int G, int n_st, int tid, int nthreads) {
  const int rows = min(kTileRows, L.N - t * kTileRows);
  for (int i = tid; i < MT * kTileRows; i += nthreads) {
    const int m = i / kTileRows, r = i % kTileRows;
    if (m >= M || r >= rows) continue;
    float v = 0.f;
    for (int c0 = c_first; c0 <= c_last; c0 += 16) {
      float q[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const int c = min(c0 + e, c_last);
        const int cs = (t == ((c * W) / G) / n_st) ? 0 : 1;
        q[e] = __ldcg(work + (size_t)(c * 2 + cs) * MT * kTileRows + i);
      }
#pragma unroll
      for (int e = 0; e < 16; ++e)
        if (c0 + e <= c_last) v += c0 + e == b ? sc.f(own + 4 * i) : q[e];
    }
    store_out(out, (size_t)m * L.N + t * kTileRows + r, t * kTileRows + r, v);
  }
}

// One CTA's work on layer L: CTA b of the G that share the layer's W stages
// (stream-K, cs == 0), or of its tiles' clusters of cs CTAs.
template <int MT, bool XF32, int MODE>
__device__ __forceinline__ void gemv_body(const Layer& L, const uint16_t* __restrict__ x, const Out& out, int M,
                                          int W, int R, int cs, float* __restrict__ work,
                                          int* __restrict__ counters, int* __restrict__ status, const int b,
                                          const int G) {
  extern __shared__ __align__(16) uint8_t smem[];
  constexpr int TB = table_bytes<MODE>();
  constexpr int NP = MODE == HXQ_MODE_SCALAR8 ? 4 : 3;  // 16-byte pieces per row and stage
  constexpr int TS = MT * kTileRows;                    // sums per tile
  const Scratch<MODE> sc{smem};
  // scratch offsets (bytes): activations at 0, then the per-warp partial
  // sums [kConsumerWarps][MT][kTileRows], this CTA's sums of its split tiles
  // [2][TS] (by slot), the sidecar corrections [kSideGroups][TS] and the
  // cluster's sums of its tile [cs][TS] (rank 0's copy)
  const uint32_t red = (uint32_t)MT * L.Kp * (XF32 ? 4 : 2);
  const uint32_t pbuf = red + kConsumerWarps * TS * 4;
  const uint32_t side = pbuf + 2 * TS * 4;
  const uint32_t cbuf = side + kSideGroups * TS * 4;
  const uint32_t sc_end = cbuf + cs * TS * 4;
  const uint32_t fixed =
      MODE == HXQ_MODE_SCALAR8 ? TB + (sc_end > kHoleBytes ? sc_end - kHoleBytes : 0) : TB + sc_end;
  uint8_t* ring = smem + ((fixed + 127) & ~127u);
  constexpr int SLOT = kChunkStages * NP * kTileRows * 16;
  __shared__ uint64_t bar_full[kMaxRing], bar_empty[kMaxRing];
  __shared__ uint64_t bar_handoff[2];  // a split tile's sums (by slot) are in pbuf: consumers -> fixup warp
  __shared__ int abort_sh, flag_sh;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_st = n_stages(L);
  // Stage range: stream-K (cs == 0), or with cs > 0 rank r of cluster t
  // takes stages [r n_st / cs, (r + 1) n_st / cs) of tile t.
  int rw0, rw1;
  if (cs > 0) {
    const int t = b / cs, r = b - t * cs;
    rw0 = t * n_st + (r * n_st) / cs;
    rw1 = t * n_st + ((r + 1) * n_st) / cs;
  } else {
    rw0 = (b * W) / G;
    rw1 = ((b + 1) * W) / G;
  }
  const Segments S(rw0, rw1, n_st);
  volatile int* abrt = &abort_sh;

  if (threadIdx.x == 0) {
    for (int i = 0; i < R; ++i) {
      mbar_init(&bar_full[i], 1);
      mbar_init(&bar_empty[i], kConsumerWarps);  // every consumer warp reads every slot
    }
    mbar_init(&bar_handoff[0], kConsumerWarps);
    mbar_init(&bar_handoff[1], kConsumerWarps);
    abort_sh = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (cs > 0) cluster_arrive_relaxed();  // (its wait precedes the first access to another CTA's memory)
  pdl_launch_dependents();  // the next kernel in the stream may start its prologue

  if (warp == kProducerWarp) {
    // ---------------- producer: the segments' chunks, in processing order,
    // with a bulk L2 prefetch of the range running kPrefetchAhead bytes
    // ahead of the ring (the indices do not depend on the previous kernel)
    if (lane == 0) {
      const size_t tile_bytes = (size_t)kTileRows * L.KC * 16 * L.P;
      int pf_k = 0, pf_w = S.n > 0 ? S.begin(0) : 0;  // prefetch cursor: segment, stage
      size_t pf_bytes = 0, ring_bytes = 0;
      auto prefetch_to = [&](size_t limit) {
        while (pf_k < S.n && pf_bytes < limit) {
          const int t = S.tile(pf_k), seg1 = S.end(pf_k);
          const int rows = min(kTileRows, L.N - t * kTileRows);
          const int we = min(pf_w + 4, seg1);
          const uint32_t bytes = (uint32_t)((we - pf_w) * NP * rows * 16);
          prefetch_l2_bulk(L.idx + (size_t)t * tile_bytes + (size_t)(pf_w - t * n_st) * NP * rows * 16, bytes);
          pf_bytes += bytes;
          pf_w = we;
          if (pf_w >= seg1 && ++pf_k < S.n) pf_w = S.begin(pf_k);
        }
      };
      int issued = 0, s = 0;
      uint32_t ph = 0;
      for (int k = 0; k < S.n && !*abrt; ++k) {
        const int t = S.tile(k), seg1 = S.end(k);
        const int rows = min(kTileRows, L.N - t * kTileRows);
        for (int w = S.begin(k); w < seg1;) {
          const int st = w - t * n_st;
          const int we = min(w + kChunkStages, seg1);
          if (!mbar_wait(&bar_empty[s], ph ^ 1, abrt)) break;
          const uint32_t bytes = (uint32_t)((we - w) * NP * rows * 16);
          mbar_arrive_expect_tx(&bar_full[s], bytes);
          bulk_load(ring + (size_t)s * SLOT, L.idx + (size_t)t * tile_bytes + (size_t)st * NP * rows * 16, bytes,
                    &bar_full[s]);
          ++issued;
          ring_bytes += bytes;
          prefetch_to(ring_bytes + kPrefetchAhead);
          if (++s == R) s = 0, ph ^= 1;
          w = we;
        }
      }
      if (*abrt) {  // let the copies this thread issued land before the CTA ends
        volatile int never = 0;
        for (int i = max(0, issued - R); i < issued; ++i) mbar_wait(&bar_full[i % R], (i / R) & 1, &never);
      }
    }
    if (cs > 0) {  // the cluster barrier's two phases (see the consumers' segment end)
      cluster_wait();
      cluster_arrive_release();
      cluster_wait();
    }
    __syncthreads();
    return;
  }

  if (warp == kFixupWarp) {
    // ---------------- fixup: split tiles processed before the range's last
    // segment, handed over by the consumers so that they never wait on
    // global memory: store this CTA's sum in the workspace and count it on
    // the tile's counter; the last to count (rarely this CTA) adds all sums
    // in CTA order and writes y.
    pdl_wait();  // y, the workspace and the counters may be in use by the previous kernel
    volatile int never = 0;  // the consumers meet every handoff, even after a timed-out wait
    for (int k = 0; k + 1 < S.n; ++k) {
      if (!S.split(k)) continue;
      const int t = S.tile(k), slot = S.slot(k);
      mbar_wait(&bar_handoff[slot], 0, &never, 64);
      const int c_first = cta_of(t * n_st, W, G), c_last = cta_of((t + 1) * n_st - 1, W, G);
      float* part = work + (size_t)(b * 2 + slot) * TS;
      for (int i = lane; i < TS; i += 32) part[i] = sc.f(pbuf + 4 * (slot * TS + i));
      __threadfence();
      __syncwarp();
      int prev = lane == 0 ? atomicAdd(counters + t, 1) : 0;
      prev = __shfl_sync(0xffffffffu, prev, 0);
      if (prev == c_last - c_first) {
        __threadfence();  // the other contributors' sums are visible past their count
        finish_tile<MT>(L, out, work, sc, pbuf + 4 * slot * TS, M, t, c_first, c_last, b, W, G, n_st, lane, 32);
        if (lane == 0) counters[t] = 0;
      }
    }
    if (cs > 0) {  // the cluster barrier's two phases (see the consumers' segment end)
      cluster_wait();
      cluster_arrive_release();
      cluster_wait();
    }
    __syncthreads();
    return;
  }

  // ---------------- consumers
  const int rr = threadIdx.x & (kTileRows - 1);  // row this thread finishes at segment ends
  const int sg = threadIdx.x / kTileRows;         // its share of the row's patch entries
  // Sidecar: the bounds of row rr's entries in the first segment's columns,
  // requested before anything else (those of the next segment are fetched
  // one segment ahead). Thread sg of the row takes entries
  // [lo + kPE sg, lo + kPE (sg + 1)).
  auto seg_bounds = [&](int k, int& lo, int& hi) {
    const int t = S.tile(k), n = t * kTileRows + rr;
    lo = hi = 0;
    if (n < L.N) {
      lo = __ldg(L.seg_ptr + (size_t)(S.begin(k) - t * n_st) * L.N + n);
      hi = __ldg(L.seg_ptr + (size_t)(S.end(k) - t * n_st) * L.N + n);
    }
  };
  int pr0, pr1;
  seg_bounds(0, pr0, pr1);
  // shared-memory codebook (compile-time trip counts: a thread's codebook
  // loads are all in flight together)
  if (MODE == HXQ_MODE_SCALAR8) {
    // lane (i % 32)'s copy of entry i / 32 at word (i / 32) * 64 + i % 32
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
  if (L.K & 7) {
    // rows of x are not 16-byte aligned: one element per load
    const int n = MT * L.Kp;
    for (int i = threadIdx.x; i < n; i += kGemvThreads) {
      const int m = i / L.Kp, k = i % L.Kp;
      const uint16_t v = (m < M && k < L.K) ? __ldg(x + (size_t)m * L.K + k) : (uint16_t)0;
      if (XF32)
        *reinterpret_cast<float*>(sc.at((uint32_t)i * 4)) = bf16lo(v);
      else
        *reinterpret_cast<uint16_t*>(sc.at((uint32_t)i * 2)) = v;
    }
  } else {
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
          float4* d = reinterpret_cast<float4*>(sc.at((uint32_t)(m * L.Kp + k) * 4));
          d[0] = make_float4(bf16lo(q[u].x), bf16hi(q[u].x), bf16lo(q[u].y), bf16hi(q[u].y));
          d[1] = make_float4(bf16lo(q[u].z), bf16hi(q[u].z), bf16lo(q[u].w), bf16hi(q[u].w));
        } else {
          *reinterpret_cast<uint4*>(sc.at((uint32_t)(m * L.Kp + k) * 2)) = q[u];
        }
      }
    }
  }
  consumer_sync();

  const uint32_t lane4 = (uint32_t)lane * 4u;
  const int q = warp;  // piece of the chunk this warp decodes
  const int q_stage = q >> 2, q_quarter = q & 3;
  int rs = 0;        // ring slot of the next chunk
  uint32_t rph = 0;  // its phase parity
  bool waited_ok = true;  // after a timed-out wait the data is garbage but every barrier is still met

  for (int k = 0; k < S.n; ++k) {
    const int t = S.tile(k), seg0 = S.begin(k), seg1 = S.end(k);
    const int rows = min(kTileRows, L.N - t * kTileRows);
    const bool split = S.split(k), last_seg = k + 1 == S.n;
    // this thread's share of row rr's patch entries in the segment's
    // columns, applied at the segment end
    // (loaded from a valid index whatever the bounds, so that nothing waits
    // for the loads before the segment end)
    int ek[kPE];
    float ed[kPE];
    const int pbase = pr0 + kPE * sg, n_mine = min(kPE, pr1 - pbase);
    if (L.n_side > 0) {
#pragma unroll
      for (int j = 0; j < kPE; ++j) {
        const int p = min(pbase + j, L.n_side - 1);
        ek[j] = __ldg(L.pk + p);
        ed[j] = __ldg(L.pd + p);
      }
    }
    const int cur0 = pr0, cur1 = pr1;
    if (!last_seg) seg_bounds(k + 1, pr0, pr1);  // the next segment's bounds
    // sums of 4 rows x MT tokens: even/odd column pairs (paired FMAs) for
    // up to 2 tokens, one register each beyond
    typename std::conditional<(MT >= 4), float, float2>::type acc[4][MT];
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int m = 0; m < MT; ++m) acc_zero(acc[j][m]);

    for (int w = seg0; w < seg1;) {  // chunks
      const int we = min(w + kChunkStages, seg1);
      if (waited_ok) waited_ok = mbar_wait(&bar_full[rs], rph, abrt);
      if (q < (we - w) * 4) {
        const uint8_t* base = ring + (size_t)rs * SLOT + (size_t)q_stage * NP * rows * 16 +
                              (MODE == HXQ_MODE_SCALAR8 ? q_quarter * rows * 16 : 0) + lane * 16;
        const int k0 = (w - t * n_st + q_stage) * kStageK + q_quarter * 16;
        // All four rows are decoded without a per-row test: in a tile of
        // fewer than 128 rows the reads past the last row stay inside the
        // slot (the pieces of a stage are packed at `rows` x 16 bytes) and
        // their sums are never stored.
        if (MT == 1) {
          float xv[16];
          x16<XF32>(sc, L.Kp, 0, k0, xv);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            float wv[16];
            decode16<MODE>(smem, base + j * 512, rows, q_quarter, lane4, wv);
            fma16(acc[j][0], wv, xv);
          }
        } else if (MODE == HXQ_MODE_VQ2D12 && MT >= 4) {
          // 2D, four or more tokens: one row at a time (the pair unpack
          // needs more registers than the scalar lookups), each token's
          // activations loaded per row
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            asm volatile("" ::: "memory");
            float wv[16];
            decode16<MODE>(smem, base + j * 512, rows, q_quarter, lane4, wv);
#pragma unroll
            for (int m = 0; m < MT; ++m) {
              float xv[16];
              x16<XF32>(sc, L.Kp, m, k0, xv);
              fma16(acc[j][m], wv, xv);
            }
          }
        } else {
          // several tokens: rows two at a time, so that two rows' weights,
          // one token's activations and all the sums fit in registers
#pragma unroll
          for (int jp = 0; jp < 2; ++jp) {
            asm volatile("" ::: "memory");
            float wv0[16], wv1[16];
            decode16<MODE>(smem, base + (2 * jp) * 512, rows, q_quarter, lane4, wv0);
            decode16<MODE>(smem, base + (2 * jp + 1) * 512, rows, q_quarter, lane4, wv1);
#pragma unroll
            for (int m = 0; m < MT; ++m) {
              if (MT >= 4) asm volatile("" ::: "memory");  // one token's activations live at a time
              float xv[16];
              x16<XF32>(sc, L.Kp, m, k0, xv);
              fma16(acc[2 * jp][m], wv0, xv);
              fma16(acc[2 * jp + 1][m], wv1, xv);
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar_empty[rs]);
      if (++rs == R) rs = 0, rph ^= 1;
      w = we;
    }

    // segment end: sidecar corrections delta * x[m][k] of this thread's
    // entries (rows with more than kSideGroups * kPE entries in the segment
    // are rare: the last share walks the rest), then the warps' sums meet in
    // shared memory
    {
      float sp[MT];
#pragma unroll
      for (int m = 0; m < MT; ++m) sp[m] = 0.f;
#pragma unroll
      for (int j = 0; j < kPE; ++j)
        if (j < n_mine) {
#pragma unroll
          for (int m = 0; m < MT; ++m) sp[m] = fmaf(ed[j], x_at(sc, L.Kp, m, ek[j], XF32), sp[m]);
        }
      if (sg == kSideGroups - 1) {
#pragma unroll 1
        for (int p = cur0 + kSideGroups * kPE; p < cur1; ++p) {
          const int kk = __ldg(L.pk + p);
          const float d = __ldg(L.pd + p);
#pragma unroll
          for (int m = 0; m < MT; ++m) sp[m] = fmaf(d, x_at(sc, L.Kp, m, kk, XF32), sp[m]);
        }
      }
#pragma unroll
      for (int m = 0; m < MT; ++m) sc.f(side + 4 * ((sg * MT + m) * kTileRows + rr)) = sp[m];
    }
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int m = 0; m < MT; ++m) sc.f(red + 4 * ((q * MT + m) * kTileRows + lane + 32 * j)) = acc_sum(acc[j][m]);
    consumer_sync();
    const int slot = S.slot(k);
    if (cs > 0) cluster_wait();  // every CTA of the cluster has started: rank 0's memory may be written
    for (int i = threadIdx.x; i < TS; i += kGemvThreads) {  // i % kTileRows == rr
      const int m = i / kTileRows;
      float v = 0.f;
#pragma unroll
      for (int qq = 0; qq < kConsumerWarps; ++qq) v += sc.f(red + 4 * ((qq * MT + m) * kTileRows + rr));
#pragma unroll
      for (int g = 0; g < kSideGroups; ++g) v += sc.f(side + 4 * ((g * MT + m) * kTileRows + rr));
      if (!split) {
        if (m < M && rr < rows) store_out(out, (size_t)m * L.N + t * kTileRows + rr, t * kTileRows + rr, v);
      } else if (cs > 0) {
        st_cluster_f32(map_to_rank(smem_u32(sc.at(cbuf + 4 * ((b % cs) * TS + i))), 0), v);
      } else {
        sc.f(pbuf + 4 * (slot * TS + i)) = v;
      }
    }
    if (cs > 0) {
      // Cluster split: the ranks' sums of the tile are in rank 0's shared
      // memory once every thread of the cluster has passed the barrier;
      // rank 0 adds them in rank order and writes y.
      cluster_arrive_release();
      cluster_wait();
      if (b % cs == 0) {
        for (int i = threadIdx.x; i < TS; i += kGemvThreads) {
          const int m = i / kTileRows;
          float v = 0.f;
          for (int r = 0; r < cs; ++r) v += sc.f(cbuf + 4 * (r * TS + i));
          if (m < M && rr < rows) store_out(out, (size_t)m * L.N + t * kTileRows + rr, t * kTileRows + rr, v);
        }
      }
    }
    if (split && !last_seg && cs == 0) {  // to the fixup warp
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar_handoff[slot]);
    }
    if (split && last_seg && cs == 0) {
      // The range's last segment is a split tile. If every other contributor
      // has already counted, add all sums now; otherwise store this CTA's sum
      // and count, and the last to count adds them. Either way the tile's
      // sums are added in CTA order.
      const int c_first = cta_of(t * n_st, W, G), c_last = cta_of((t + 1) * n_st - 1, W, G);
      const int others = c_last - c_first;
      if (threadIdx.x == 0) flag_sh = ld_acquire_gpu(counters + t) == others;
      consumer_sync();
      bool last = flag_sh;
      const uint32_t own = pbuf + 4 * slot * TS;
      if (!last) {
        float* part = work + (size_t)(b * 2 + slot) * TS;
        for (int i = threadIdx.x; i < TS; i += kGemvThreads) part[i] = sc.f(own + 4 * i);
        __threadfence();
        consumer_sync();
        if (threadIdx.x == 0) flag_sh = atomicAdd(counters + t, 1) == others;
        consumer_sync();
        last = flag_sh;
      }
      if (last) {
        __threadfence();  // the other contributors' sums are visible past their count
        finish_tile<MT>(L, out, work, sc, own, M, t, c_first, c_last, b, W, G, n_st, threadIdx.x, kGemvThreads);
        if (threadIdx.x == 0) counters[t] = 0;
      }
    }
    consumer_sync();
  }
  if (!waited_ok && threadIdx.x == 0) atomicOr(status, kStatusWaitTimeout);
  __syncthreads();
}

template <int MT, bool XF32, int MODE>
__global__ void __launch_bounds__(kGemvBlock, 2)
gemv_kernel(Layer L, const uint16_t* __restrict__ x, Out out, int M, int W, int R, int cs,
            float* __restrict__ work, int* __restrict__ counters, int* __restrict__ status) {
  gemv_body<MT, XF32, MODE>(L, x, out, M, W, R, cs, work, counters, status, (int)blockIdx.x, (int)gridDim.x);
}

// Several layers that read the same activations (same K and mode), in one
// launch: layer i owns CTAs [first[i], first[i + 1]) of the grid and runs on
// them exactly as a launch of its own would (its own codebook, sidecar,
// output, workspace and counters). Under the cluster split every first[i] is
// a multiple of the cluster size, so no cluster spans two layers.
struct GemvGroup {
  Layer L[kMaxGroup];
  Out out[kMaxGroup];
  float* work[kMaxGroup];
  int* counters[kMaxGroup];
  int* status[kMaxGroup];
  int W[kMaxGroup];             // stages of each layer
  int first[kMaxGroup + 1];     // first CTA of each layer; first[n] = grid size
  int n;
};

template <int MT, bool XF32, int MODE>
__global__ void __launch_bounds__(kGemvBlock, 2)
gemv_group_kernel(const __grid_constant__ GemvGroup g, const uint16_t* __restrict__ x, int M, int R, int cs) {
  int li = 0;
#pragma unroll
  for (int i = 1; i < kMaxGroup; ++i)
    if (i < g.n && (int)blockIdx.x >= g.first[i]) li = i;
  gemv_body<MT, XF32, MODE>(g.L[li], x, g.out[li], M, g.W[li], R, cs, g.work[li], g.counters[li], g.status[li],
                            (int)blockIdx.x - g.first[li], g.first[li + 1] - g.first[li]);
}

// Launch shapes and SM sharing. Every launch may share an SM with the next
// one (both at most kSmemShared bytes), so that the next layer's prologue
// overlaps this one's tail. The block scheduler may then also put two CTAs of
// ONE launch on an SM (when a CTA slot frees up next to a CTA of the same
// launch): those two run at half speed and the whole launch waits for them.
// Launches in clusters of 2 therefore take `exclusive_smem` bytes: two CTAs
// of that size do not fit on one SM, one still fits next to a CTA of the
// neighbouring launch. (Measured on the Mamba2 in_proj / out_proj pair: 15 %
// less time per pair. Given the exclusive size, launches in larger clusters
// got slower -- their clusters wait for whole groups of SMs to clear -- and
// stream-K launches gained nothing, so they keep the shared size.)
inline bool want_exclusive(int cs) { return cs == 2; }

template <int MT, bool XF32, int MODE, bool GROUP>
size_t exclusive_smem() {
  static const size_t bytes = [] {
    const void* kern = GROUP ? reinterpret_cast<const void*>(gemv_group_kernel<MT, XF32, MODE>)
                             : reinterpret_cast<const void*>(gemv_kernel<MT, XF32, MODE>);
    int dev = 0, per_sm = 0, reserved = 0;
    cudaFuncAttributes fa;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&per_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev) != cudaSuccess ||
        cudaFuncGetAttributes(&fa, kern) != cudaSuccess) {
      cudaGetLastError();
      return (size_t)0;
    }
    const size_t st = (fa.sharedSizeBytes + 127) / 128 * 128;
    // smallest multiple of 128 with 2 x (dynamic + static + reserved) > per_sm
    const size_t half = (size_t)per_sm / 2;
    if (half < (size_t)reserved + st) return (size_t)0;
    const size_t dyn = ((half - reserved - st) / 128 + 1) * 128;
    // room left beside it for a CTA of kSmemShared dynamic bytes
    if (dyn > kSmemLimit || 2 * (st + (size_t)reserved) + dyn + kSmemShared > (size_t)per_sm) return (size_t)0;
    // the occupancy calculator agrees: one CTA per SM
    int nb = 0;
    if (allow_max_smem(kern) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, kern, kGemvBlock, dyn) != cudaSuccess || nb != 1) {
      cudaGetLastError();
      return (size_t)0;
    }
    return dyn;
  }();
  return bytes;
}

// Lets the kernel take `smem` bytes of dynamic shared memory, with the
// largest shared-memory carveout, so that two CTAs of up to kSmemShared bytes
// each (this launch's and the next one's) can be resident on one SM.
template <typename Kern>
cudaError_t set_smem(Kern kern, size_t smem) {
  (void)smem;  // the limit is the device's maximum; the launch passes its own size
  return allow_max_smem(reinterpret_cast<const void*>(kern));
}

// Cluster split (no global-memory reduction): each tile gets a cluster of
// cs CTAs (2..16; above 8 where the device allows such clusters) that split
// its K, for the largest cs whose grid (tiles x cs) fills at least 70 % of
// the SMs without exceeding them (any fill for layers of at most a few
// tiles) and whose clusters all fit on the GPU at once. 0 = the stream-K
// decomposition. `cached` keeps the answer for the next launch of the same
// shape.
template <int MT, bool XF32, int MODE, bool GROUP, typename Kern>
int pick_cluster_for(Kern kern, int n_tiles, int Kp, int num_sms, int& cached) {
  if (cached >= 0) return cached;
  cached = 0;
  if (MT > 4) return 0;
  const int n_st = Kp / kStageK;
  // a layer too small to fill 70 % of the SMs at any cluster size takes the
  // largest that fits: under stream-K its CTAs would hold a stage or two
  // each, and the split-tile fixup chain would outlast the decode
  const bool small = 100 * n_tiles * kMaxCluster < 70 * num_sms;
  for (int cs = kMaxCluster; cs >= 2; --cs) {
    const int g = n_tiles * cs;
    if (g > num_sms || (!small && 100 * g < 70 * num_sms) || n_st < cs) continue;
    if (ring_slots(MODE, MT, Kp, XF32, cs) < kMinRing) continue;
    size_t smem = gemv_smem(MODE, MT, Kp, XF32, cs);
    if (want_exclusive(cs)) smem = std::max(smem, exclusive_smem<MT, XF32, MODE, GROUP>());
    if (set_smem(kern, smem) != cudaSuccess ||
        (cs > 8 && cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess)) {
      cudaGetLastError();
      continue;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(g);
    cfg.blockDim = dim3(kGemvBlock);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = cs;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n_clusters = 0;
    if (cudaOccupancyMaxActiveClusters(&n_clusters, kern, &cfg) == cudaSuccess && n_clusters >= n_tiles) {
      cached = cs;
      return cs;
    }
    cudaGetLastError();
  }
  return 0;
}

// Index of a launch shape's cached cluster size: (activation staging, token
// count class).
template <int MT, bool XF32>
constexpr int cluster_slot() { return (XF32 ? 4 : 0) + (MT <= 1 ? 0 : MT <= 2 ? 1 : MT <= 4 ? 2 : 3); }

template <int MT, bool XF32, int MODE>
int pick_cluster(const hxq_linear& h) {
  return pick_cluster_for<MT, XF32, MODE, false>(gemv_kernel<MT, XF32, MODE>, h.L.n_tiles, h.L.Kp, h.num_sms,
                                          h.gemv_cluster[cluster_slot<MT, XF32>()]);
}

template <int MT, bool XF32, int MODE>
cudaError_t launch_cfg(const hxq_linear& h, const uint16_t* x, const Out& out, int M, int grid, float* work, int* counters,
                       bool allow_cluster, cudaStream_t s) {
  auto kern = gemv_kernel<MT, XF32, MODE>;
  const int W = h.L.n_tiles * (h.L.Kp / kStageK);
  const int cs = allow_cluster ? pick_cluster<MT, XF32, MODE>(h) : 0;
  if (cs > 0) {
    const int Rc = ring_slots(MODE, MT, h.L.Kp, XF32, cs);
    size_t smem = gemv_smem(MODE, MT, h.L.Kp, XF32, cs);
    if (want_exclusive(cs)) smem = std::max(smem, exclusive_smem<MT, XF32, MODE, false>());
    cudaError_t e = set_smem(kern, smem);
    if (e != cudaSuccess) return e;
    return launch_pdl_cluster(kern, h.L.n_tiles * cs, kGemvBlock, smem, cs, s, h.L, x, out, M, W, Rc, cs, work, counters,
                              h.d_status);
  }
  const int R = ring_slots(MODE, MT, h.L.Kp, XF32);
  if (R < kMinRing) return cudaErrorInvalidValue;
  const size_t smem = gemv_smem(MODE, MT, h.L.Kp, XF32);
  cudaError_t e = set_smem(kern, smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(kern, grid, kGemvBlock, smem, s, h.L, x, out, M, W, R, 0, work, counters, h.d_status);
}

template <int MT, int MODE>
cudaError_t launch_mt(const hxq_linear& h, const uint16_t* x, const Out& out, int M, int grid, float* work, int* counters,
                      bool allow_cluster, cudaStream_t s) {
  if (stage_x_f32(MODE, MT, h.L.Kp))
    return launch_cfg<MT, true, MODE>(h, x, out, M, grid, work, counters, allow_cluster, s);
  return launch_cfg<MT, false, MODE>(h, x, out, M, grid, work, counters, allow_cluster, s);
}

template <int MODE>
cudaError_t launch_mode(const hxq_linear& h, const uint16_t* x, const Out& out, int M, int grid, float* work, int* counters,
                        bool allow_cluster, cudaStream_t s) {
  if (M <= 1) return launch_mt<1, MODE>(h, x, out, M, grid, work, counters, allow_cluster, s);
  if (M <= 2) return launch_mt<2, MODE>(h, x, out, M, grid, work, counters, allow_cluster, s);
  if (M <= 4) return launch_mt<4, MODE>(h, x, out, M, grid, work, counters, allow_cluster, s);
  return launch_mt<8, MODE>(h, x, out, M, grid, work, counters, allow_cluster, s);
}

int mt_of(int M) { return M <= 1 ? 1 : M <= 2 ? 2 : M <= 4 ? 4 : 8; }

template <int MT, bool XF32, int MODE>
cudaError_t launch_group_cfg(const hxq_group& g, const uint16_t* x, const Out* outs, int M, cudaStream_t s) {
  auto kern = gemv_group_kernel<MT, XF32, MODE>;
  const int Kp = g.h[0]->L.Kp, n_st = Kp / kStageK;
  GemvGroup p = {};
  p.n = g.n;
  int n_tiles = 0;
  int64_t W[kMaxGroup];
  for (int i = 0; i < g.n; ++i) {
    const hxq_linear& h = *g.h[i];
    p.L[i] = h.L;
    p.out[i] = outs[i];
    p.work[i] = h.d_work;
    p.counters[i] = h.d_counters;
    p.status[i] = h.d_status;
    W[i] = (int64_t)h.L.n_tiles * n_st;
    p.W[i] = (int)W[i];
    n_tiles += h.L.n_tiles;
  }
  const int cs = pick_cluster_for<MT, XF32, MODE, true>(kern, n_tiles, Kp, g.num_sms,
                                                  g.gemv_cluster[cluster_slot<MT, XF32>()]);
  p.first[0] = 0;
  if (cs > 0) {
    for (int i = 0; i < g.n; ++i) p.first[i + 1] = p.first[i] + g.h[i]->L.n_tiles * cs;
  } else {
    int64_t Wt = 0;
    for (int i = 0; i < g.n; ++i) Wt += W[i];
    const int G = (int)std::max<int64_t>(g.n, std::min<int64_t>(g.num_sms, Wt));
    int Gl[kMaxGroup];
    group_shares(W, g.n, G, Gl);
    for (int i = 0; i < g.n; ++i) {
      if (W[i] * Gl[i] >= INT_MAX) return cudaErrorInvalidValue;  // item arithmetic is 32-bit
      // every CTA writes at most two partial tiles of MT x 128 floats
      if ((size_t)Gl[i] * 2 * MT * kTileRows > g.h[i]->work_floats) return cudaErrorInvalidValue;
      p.first[i + 1] = p.first[i] + Gl[i];
    }
  }
  for (int i = g.n + 1; i <= kMaxGroup; ++i) p.first[i] = p.first[g.n];
  const int grid = p.first[g.n];
  const int R = ring_slots(MODE, MT, Kp, XF32, cs);
  if (R < kMinRing) return cudaErrorInvalidValue;
  size_t smem = gemv_smem(MODE, MT, Kp, XF32, cs);
  if (want_exclusive(cs)) smem = std::max(smem, exclusive_smem<MT, XF32, MODE, true>());
  cudaError_t e = set_smem(kern, smem);
  if (e != cudaSuccess) return e;
  if (cs > 0) return launch_pdl_cluster(kern, grid, kGemvBlock, smem, cs, s, p, x, M, R, cs);
  return launch_pdl(kern, grid, kGemvBlock, smem, s, p, x, M, R, 0);
}

template <int MT, int MODE>
cudaError_t launch_group_mt(const hxq_group& g, const uint16_t* x, const Out* outs, int M, cudaStream_t s) {
  if (stage_x_f32(MODE, MT, g.h[0]->L.Kp)) return launch_group_cfg<MT, true, MODE>(g, x, outs, M, s);
  return launch_group_cfg<MT, false, MODE>(g, x, outs, M, s);
}

template <int MODE>
cudaError_t launch_group_mode(const hxq_group& g, const uint16_t* x, const Out* outs, int M, cudaStream_t s) {
  if (M <= 1) return launch_group_mt<1, MODE>(g, x, outs, M, s);
  if (M <= 2) return launch_group_mt<2, MODE>(g, x, outs, M, s);
  return launch_group_mt<4, MODE>(g, x, outs, M, s);
}

}  // namespace

bool gemv_supports(const hxq_linear& h, int M) {
  return M >= 1 && M <= kGemvMaxM && ring_slots(h.L.mode, mt_of(M), h.L.Kp, false) >= kMinRing;
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

cudaError_t launch_gemv_group(const hxq_group& g, const uint16_t* x, const Out* outs, int M, cudaStream_t s) {
  if (g.n < 1 || g.n > kMaxGroup || M < 1 || M > 4) return cudaErrorInvalidValue;
  for (int i = 0; i < g.n; ++i)
    if (!gemv_supports(*g.h[i], M)) return cudaErrorInvalidValue;
  if (g.h[0]->L.mode == HXQ_MODE_SCALAR8) return launch_group_mode<HXQ_MODE_SCALAR8>(g, x, outs, M, s);
  return launch_group_mode<HXQ_MODE_VQ2D12>(g, x, outs, M, s);
}

cudaError_t launch_gemv(const hxq_linear& h, const uint16_t* x, const Out& out, int M, int split, cudaStream_t s) {
  if (!gemv_supports(h, M)) return cudaErrorInvalidValue;
  const int grid = gemv_grid(h, split);
  if (grid == 0) return cudaErrorInvalidValue;
  // every CTA writes at most two partial tiles of mt_of(M) x 128 floats
  if ((size_t)grid * 2 * mt_of(M) * kTileRows > h.work_floats) return cudaErrorInvalidValue;
  if (h.L.mode == HXQ_MODE_SCALAR8)
    return launch_mode<HXQ_MODE_SCALAR8>(h, x, out, M, grid, h.d_work, h.d_counters, split == 0, s);
  return launch_mode<HXQ_MODE_VQ2D12>(h, x, out, M, grid, h.d_work, h.d_counters, split == 0, s);
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

namespace hxq {
// Looks up the scratch array's device address on device `dev` (current) and
// caches it; called when a handle is created, so that the no-alloc entry
// point itself only reads the cache.
cudaError_t noalloc_prepare(int dev) {
  void* p = nullptr;
  return noalloc_scratch(dev, &p);
}
}  // namespace hxq

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
    const Out out{y, nullptr, 0};
    e = h->L.mode == HXQ_MODE_SCALAR8 ? launch_mode<HXQ_MODE_SCALAR8>(*h, x, out, M, grid, work, counters, true, s)
                                      : launch_mode<HXQ_MODE_VQ2D12>(*h, x, out, M, grid, work, counters, true, s);
  }
  if (e != cudaSuccess) {
    cudaGetLastError();
    return HXQ_ECUDA;
  }
  return HXQ_OK;
}
