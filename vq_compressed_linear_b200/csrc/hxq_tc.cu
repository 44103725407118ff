// Fused decode + GEMM on the sm_100a tensor cores (tcgen05), for M > 4:
//   y[m][n] = sum_k x[m][k] * W[n][k],  W decoded on the fly, never stored.
//
// The MMA computes D = A . B^T with A = a 128-row tile of W (output features)
// and B = a tile of BN tokens of x, so D = y^T for that tile and lives in
// tensor memory (TMEM): lane = output feature, column = token.
//
//  * A is written by 8 decoding warps straight from registers into TMEM
//    with tcgen05.st (the "A from tensor memory" form of tcgen05.mma): the
//    decoded weights never touch shared or global memory. Thread r of a
//    decoding warp (one per TMEM lane quadrant and pair of column groups)
//    owns TMEM lane r = row r of the tile and the columns [16 g, 16 g + 16)
//    of its two groups g of every stage. A
//    producer warp streams each item's index block (contiguous in the tiled
//    layout) with TMA bulk copies into a ring of shared-memory slots; the
//    thread reads its 2 x 16 indices from the slot, looks them up in a
//    shared-memory table, substitutes sidecar values, packs two bf16 per
//    32-bit TMEM cell and stores them. All decoding warps work on the same
//    item, so the MMA receives items at an even pace.
//  * B (x) arrives by TMA into 128-byte-swizzled shared memory, 64 columns of
//    K per stage; rows past M and columns past K read as zero.
//  * One thread issues tcgen05.mma (kind::f16, bf16 x bf16 -> fp32 in TMEM)
//    and signals stage release and segment completion with tcgen05.commit.
//  * Four epilogue warps read D back with tcgen05.ld and store y.
//
// Work decomposition (stream-K): the items are (token block, tile, stage)
// triples numbered stage-fastest; a persistent grid of one CTA per SM takes
// contiguous item ranges of equal size. A run of items of one (token block,
// tile) is a segment; a segment that covers all of K is written to y
// directly, the others leave fp32 partials in the workspace and the last
// contributor to arrive sums them in CTA order (bitwise repeatable). With
// BN <= 128 the accumulator is double-buffered so the next segment's MMAs
// overlap the previous segment's epilogue.
//
// Weight precision (TERMS):
//  * TERMS = 1 (M > 32, the prefill): each weight is rounded to bf16 (round
//    to nearest even) -- the pages' decode kernel also writes BF16 weights for
//    the matmul (HXQ whitepaper, method section, fused gather paragraph).
//  * TERMS = 2 (M <= 32): each fp32 weight w is split as hi = bf16(w),
//    mid = bf16(w - hi) and both are multiplied, so the weight carries 16
//    significand bits: |w - hi - mid| <= 2^-17 |w|, inside the fp32-codebook
//    tolerance 1e-5 * sum |x||w| that applies to the decode GEMV.
//
// Sidecar (HXQ whitepaper, method section, "Sidecar outlier correction"):
// each decoding thread keeps a cursor into its row's column-sorted patch list
// (placed at a tile's first stage through a per-stage lower-bound table) with
// the next two entries already requested, and substitutes the stored value
// (as bf16, or as its hi+mid split) before the store.
//
// Every mbarrier wait is bounded (2 s unless a test lowers it): on timeout the
// CTA sets a status bit, drains what it issued, frees TMEM and returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <climits>

#include "hxq_internal.cuh"

namespace hxq {
namespace {

constexpr int kEpiWarp0 = 4;                            // warps 4..7: epilogue
constexpr int kDecWarp0 = 8;                            // warps 8..: decoders
constexpr int kTmemCols = 512;
constexpr int kMaxTokBlocks = 64;                       // token blocks per launch (counter space)
constexpr int kMaxContrib = 8;                          // CTAs sharing one tile's K at most
constexpr int kPrefetchItems = 16;                      // index bytes streamed into L2 this far ahead

// Decoding warps: one per TMEM lane quadrant and pair of 16-column groups.
// Every decoding warp takes part in every item: warp (h, q) decodes the
// column groups h and h + 2 ([16 g, 16 g + 16) of the stage) for the 32
// rows of quadrant q. (Measured: 8 such warps beat 16 warps of one group --
// fewer warps contend with the MMA thread for issue -- and 4 warps of four
// groups; Qwen2.5-3B layers at M=32 155 -> 140 us, prefill M=2048 466 -> 490
// TFLOP/s.)
constexpr int kDecWarps = 8;
constexpr int kGroupsPerWarp = 16 / kDecWarps;  // 16-column groups x quadrants per warp
constexpr int kTcThreads = 32 * (kDecWarp0 + kDecWarps);
constexpr size_t kTcSmemLimit = 226 * 1024;  // dynamic shared memory (the barriers are static)

// x / A pipeline slots, as many as TMEM (accumulators + A slots of 32 columns
// per term) and shared memory (x slots of BN x 128 bytes) allow.
template <int BN, int TERMS>
constexpr int num_slots() {
  return TERMS == 2 ? 7 : (BN <= 64 ? 12 : BN <= 128 ? 6 : 4);
}

__device__ __forceinline__ uint32_t bf16_bits(float f) {
  return (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(f));
}
// hi = bf16(w), mid = bf16(w - hi) packed as one word: hi in the top half.
__device__ __forceinline__ uint32_t split_word(float w) {
  const uint32_t hi = bf16_bits(w);
  const uint32_t mid = bf16_bits(w - __uint_as_float(hi << 16));
  return (hi << 16) | mid;
}

// UMMA shared-memory descriptor, K-major operand in the 128-byte swizzle
// layout: rows of 128 bytes, 8-row atoms 1024 bytes apart.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t addr) {
  return (uint64_t)((addr >> 4) & 0x3FFF) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// Instruction descriptor, kind::f16: D fp32, A and B bf16, both K-major,
// M = 128, N = BN.
template <int BN>
__device__ __forceinline__ uint32_t idesc_bf16() {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
}

template <int MODE, int TERMS>
constexpr size_t table_bytes() {
  return MODE == HXQ_MODE_SCALAR8 ? 256 * 256 : (TERMS == 1 ? 4096 * 4 : 4096 * 8);
}

template <int BN>
constexpr int num_acc() { return BN <= 128 ? 2 : 1; }

// Index ring: one slot holds one item's index block (all rows of the tile).
template <int MODE>
constexpr int idx_slot_bytes() { return (MODE == HXQ_MODE_SCALAR8 ? 4 : 3) * kTileRows * 16; }

template <int BN, int TERMS, int MODE>
constexpr size_t tc_fixed_bytes() {
  return table_bytes<MODE, TERMS>() + 1024 /* alignment slack */ + (size_t)num_slots<BN, TERMS>() * BN * 128;
}
template <int BN, int TERMS, int MODE>
constexpr int idx_slots() {
  return (int)std::min<size_t>(16, (kTcSmemLimit - tc_fixed_bytes<BN, TERMS, MODE>()) / idx_slot_bytes<MODE>());
}
template <int BN, int TERMS, int MODE>
constexpr size_t tc_smem_bytes() {
  return tc_fixed_bytes<BN, TERMS, MODE>() + (size_t)idx_slots<BN, TERMS, MODE>() * idx_slot_bytes<MODE>();
}

// Replace the word at offset j (0..15) of a 16-weight chunk by pw.
__device__ __forceinline__ void patch16(uint32_t (&v)[16], int j, uint32_t pw) {
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = sel_eq(i, j, pw, v[i]);
}
// Replace half h of pair word j (0..7) by the 16-bit value hv.
__device__ __forceinline__ void patch8_half(uint32_t (&v)[8], int j, int h, uint32_t hv) {
#pragma unroll
  for (int i = 0; i < 8; ++i)
    v[i] = sel_eq(i, j, h ? ((v[i] & 0xFFFFu) | (hv << 16)) : ((v[i] & 0xFFFF0000u) | hv), v[i]);
}

// CTA whose item range [b W / G, (b+1) W / G) contains item w.
// (W * G < 2^31, checked at launch)
__device__ __forceinline__ int cta_of(int w, int W, int G) {
  int b = (w * G) / W;
  while (b + 1 < G && ((b + 1) * W) / G <= w) ++b;
  while (b > 0 && (b * W) / G > w) --b;
  return b;
}

// The 12 index bytes [12 g, 12 g + 12) of a row's 48-byte stage (8 pairs),
// from the three 16-byte planes of the row in an index slot.
__device__ __forceinline__ void quarter_words_2d(const uint8_t* p0, int rows, int g, uint32_t (&wd)[4]) {
  const uint8_t* p1 = p0 + rows * 16;
  const uint8_t* p2 = p1 + rows * 16;
  wd[3] = 0;
  if (g == 0) {
    const uint4 v = *reinterpret_cast<const uint4*>(p0);
    wd[0] = v.x; wd[1] = v.y; wd[2] = v.z;
  } else if (g == 1) {
    const uint2 v = *reinterpret_cast<const uint2*>(p1);
    wd[0] = *reinterpret_cast<const uint32_t*>(p0 + 12); wd[1] = v.x; wd[2] = v.y;
  } else if (g == 2) {
    const uint2 v = *reinterpret_cast<const uint2*>(p1 + 8);
    wd[0] = v.x; wd[1] = v.y; wd[2] = *reinterpret_cast<const uint32_t*>(p2);
  } else {
    const uint4 v = *reinterpret_cast<const uint4*>(p2);
    wd[0] = v.y; wd[1] = v.z; wd[2] = v.w;
  }
}

// Test hook of the tensor-core kernel: the limit of every pipeline wait, and
// an item of each CTA's range whose activations are never requested (-1 =
// none), so that a test can make a wait run out without a GPU fault.
struct TestHook {
  uint64_t wait_limit_ns;
  int withhold_item;
};

template <int BN, int TERMS, int MODE>
__global__ void __launch_bounds__(kTcThreads, 1)
tc_kernel(const __grid_constant__ CUtensorMap tmx, Layer L, Out out, int M, int tok0, int n_tb,
          float* __restrict__ work, int* __restrict__ counters, int* __restrict__ status, TestHook hook) {
  constexpr int XSLOT = BN * 128;
  constexpr int kSlots = num_slots<BN, TERMS>();
  constexpr int kIS = idx_slots<BN, TERMS, MODE>();
  constexpr int ISLOT = idx_slot_bytes<MODE>();
  static_assert(kIS >= 2, "index ring");
  constexpr int TB = (int)table_bytes<MODE, TERMS>();
  constexpr int NACC = num_acc<BN>();
  constexpr int ACOL0 = NACC * BN < 64 ? 64 : NACC * BN;  // first TMEM column of the A slots
  static_assert(ACOL0 + kSlots * 32 * TERMS <= kTmemCols, "TMEM budget");
  constexpr int NPC = MODE == HXQ_MODE_SCALAR8 ? 4 : 3;  // 16-byte pieces per row and stage
  // The decode table sits at the start of dynamic shared memory so lookups
  // address it from the array symbol (plain LDS); the x slots follow,
  // aligned to 1024 bytes for the 128-byte swizzle, then the index ring.
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t xs_pad = (1024u - ((smem_u32(smem) + TB) & 1023u)) & 1023u;
  uint8_t* xs = smem + TB + xs_pad;
  uint8_t* ring = xs + kSlots * XSLOT;
  __shared__ uint64_t bar_x[kSlots], bar_a[kSlots], bar_empty[kSlots], bar_acc[NACC], bar_dfree[NACC], bar_drain;
  __shared__ uint64_t bar_ifull[kIS], bar_ifree[kIS];
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint64_t lim = hook.wait_limit_ns;
  const int n_st = n_stages(L);
  const int W = n_tb * L.n_tiles * n_st;
  const int G = gridDim.x;
  const int w0 = (blockIdx.x * W) / G, w1 = ((blockIdx.x + 1) * W) / G;
  const int n_items = w1 - w0;

  pdl_launch_dependents();
  if (threadIdx.x == 0) {
    for (int i = 0; i < kSlots; ++i) {
      mbar_init(&bar_x[i], 1);
      mbar_init(&bar_a[i], kDecWarps);
      mbar_init(&bar_empty[i], 1);
    }
    for (int i = 0; i < kIS; ++i) {
      mbar_init(&bar_ifull[i], 1);
      mbar_init(&bar_ifree[i], kDecWarps);
    }
    for (int i = 0; i < NACC; ++i) {
      mbar_init(&bar_acc[i], 1);
      mbar_init(&bar_dfree[i], 4);
    }
    mbar_init(&bar_drain, 1);
    abort_sh = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) prefetch_tmap(&tmx);
  if (warp == 1) {
    tmem_alloc(&tmem_base_sh, kTmemCols);
    tmem_relinquish();
  }
  // shared-memory decode table (compile-time trip counts: a thread's
  // codebook loads are all in flight together)
  constexpr int NT = kTcThreads;
  if (MODE == HXQ_MODE_SCALAR8) {
    constexpr int PER = (256 * 32 + NT - 1) / NT;
    float cv[PER];
#pragma unroll
    for (int j = 0; j < PER; ++j) {
      const int i = threadIdx.x + j * NT;
      cv[j] = i < 256 * 32 ? __ldg(L.codebook + (i >> 5)) : 0.f;
    }
    uint32_t* tw = reinterpret_cast<uint32_t*>(smem);
#pragma unroll
    for (int j = 0; j < PER; ++j) {
      const int i = threadIdx.x + j * NT;
      if (i < 256 * 32) tw[(i >> 5) * 64 + (i & 31)] = TERMS == 1 ? (bf16_bits(cv[j]) << 16) : split_word(cv[j]);
    }
  } else {
    constexpr int PER = (4096 + NT - 1) / NT;
    const float2* cb2 = reinterpret_cast<const float2*>(L.codebook);
    float2 cv[PER];
#pragma unroll
    for (int j = 0; j < PER; ++j) {
      const int i = threadIdx.x + j * NT;
      cv[j] = i < 4096 ? __ldg(cb2 + i) : make_float2(0.f, 0.f);
    }
#pragma unroll
    for (int j = 0; j < PER; ++j) {
      const int i = threadIdx.x + j * NT;
      if (i >= 4096) break;
      if (TERMS == 1) {
        reinterpret_cast<uint32_t*>(smem)[i] = bf16_bits(cv[j].x) | (bf16_bits(cv[j].y) << 16);
      } else {
        const uint32_t a = split_word(cv[j].x), b = split_word(cv[j].y);
        reinterpret_cast<uint2*>(smem)[i] = make_uint2(prmt(a, b, 0x7632), prmt(a, b, 0x5410));
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  volatile int* abrt = &abort_sh;

  if (warp == 0) {
    // ---------------- TMA producer: x tiles
    if (lane == 0) {
      // index bytes of later items: streamed into L2 ahead of the index ring
      auto prefetch_item = [&](int i) {
        const int w = w0 + i, t = (w / n_st) % L.n_tiles, st = w % n_st;
        const int rows = min(kTileRows, L.N - t * kTileRows);
        prefetch_l2_bulk(L.idx + piece_offset(L, t, MODE == HXQ_MODE_SCALAR8 ? st * 4 : st, 0, 0),
                         (uint32_t)(NPC * rows * 16));
      };
      for (int i = kIS; i < min(n_items, kIS + kPrefetchItems); ++i) prefetch_item(i);
      pdl_wait();  // x may be the previous kernel's output
      int issued = 0, b = 0;
      uint32_t ph = 0;
      for (int i = 0; i < n_items; ++i) {
        const int w = w0 + i;
        const int T = w / n_st, st = w - T * n_st;
        const int tb = T / L.n_tiles;
        if (i + kIS + kPrefetchItems < n_items) prefetch_item(i + kIS + kPrefetchItems);
        if (i == hook.withhold_item) {
          // test hook: this item's activations are never requested; wait for
          // the copies already issued and stop (the MMA thread's wait for
          // them runs out and the CTA aborts)
          volatile int never = 0;
          for (int j = max(0, issued - kSlots); j < issued; ++j)
            mbar_wait(&bar_x[j % kSlots], (j / kSlots) & 1, &never);
          break;
        }
        // (the producers run slots ahead: they poll with short sleeps, so that
        // their warps leave issue slots to the decoders)
        if (!mbar_wait(&bar_empty[b], ph ^ 1, abrt, 64, lim)) break;
        mbar_arrive_expect_tx(&bar_x[b], XSLOT);
        tma_load_2d(xs + b * XSLOT, &tmx, &bar_x[b], st * kStageK, tok0 + tb * BN);
        ++issued;
        if (++b == kSlots) b = 0, ph ^= 1;
      }
      if (*abrt) {  // drain the loads this thread issued before leaving
        volatile int never = 0;
        for (int i = max(0, issued - kSlots); i < issued; ++i)
          mbar_wait(&bar_x[i % kSlots], (i / kSlots) & 1, &never);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16<BN>();
      int seg = -1, b = 0;
      uint32_t par = 0;
      for (int i = 0; i < n_items; ++i) {
        const int w = w0 + i;
        const bool first = (i == 0) || (w % n_st == 0);
        const bool last = (i == n_items - 1) || ((w + 1) % n_st == 0);
        if (first) {
          ++seg;
          const int u = seg / NACC;
          if (u >= 1 && !mbar_wait(&bar_dfree[seg % NACC], (u - 1) & 1, abrt, 0, lim)) break;
        }
        if (!mbar_wait(&bar_x[b], par, abrt, 0, lim) || !mbar_wait(&bar_a[b], par, abrt, 0, lim)) break;
        tc_fence_after();
        const uint32_t xaddr = smem_u32(xs + b * XSLOT);
        const uint32_t dcol = tmem + (seg % NACC) * BN;
#pragma unroll
        for (int kk = 0; kk < kStageK / 16; ++kk) {
          const uint64_t bdesc = smem_desc_sw128(xaddr + kk * 32);
#pragma unroll
          for (int term = 0; term < TERMS; ++term) {
            const uint32_t acol = tmem + ACOL0 + b * 32 * TERMS + term * 32 + kk * 8;
            tc_mma_ts(dcol, acol, bdesc, idesc, (!first || kk || term) ? 1u : 0u);
          }
        }
        tc_commit(&bar_empty[b]);
        if (last) tc_commit(&bar_acc[seg % NACC]);
        if (++b == kSlots) b = 0, par ^= 1;
      }
      if (*abrt) {  // let issued MMAs finish before TMEM is freed
        volatile int never = 0;
        tc_commit(&bar_drain);
        mbar_wait(&bar_drain, 0, &never);
      }
    }
  } else if (warp == 2) {
    // ---------------- index producer: the items' index blocks into the ring
    // (they do not depend on the previous kernel: no wait for it)
    if (lane == 0) {
      int issued = 0, s = 0;
      uint32_t ph = 0;
      for (int i = 0; i < n_items; ++i) {
        if (!mbar_wait(&bar_ifree[s], ph ^ 1, abrt, 64, lim)) break;
        const int w = w0 + i, T = w / n_st, st = w - T * n_st, t = T % L.n_tiles;
        const int rows = min(kTileRows, L.N - t * kTileRows);
        const uint32_t bytes = (uint32_t)(NPC * rows * 16);
        mbar_arrive_expect_tx(&bar_ifull[s], bytes);
        bulk_load(ring + (size_t)s * ISLOT,
                  L.idx + piece_offset(L, t, MODE == HXQ_MODE_SCALAR8 ? st * 4 : st, 0, 0), bytes, &bar_ifull[s]);
        ++issued;
        if (++s == kIS) s = 0, ph ^= 1;
      }
      if (*abrt) {  // let the copies this thread issued land before the CTA ends
        volatile int never = 0;
        for (int i = max(0, issued - kIS); i < issued; ++i) mbar_wait(&bar_ifull[i % kIS], (i / kIS) & 1, &never);
      }
    }
  } else if (warp >= kEpiWarp0 && warp < kDecWarp0) {
    // ---------------- epilogue: D (y^T tile) from TMEM to y / workspace
    const int q = warp & 3, r = q * 32 + lane;
    const uint32_t lane_base = tmem + ((uint32_t)(q * 32) << 16);
    pdl_wait();  // y, the workspace and the counters may be in use by the previous kernel
    int seg = -1;
    for (int i = 0; i < n_items; ++i) {
      const int w = w0 + i;
      if (!((i == n_items - 1) || ((w + 1) % n_st == 0))) continue;  // not a segment end
      ++seg;
      const int T = w / n_st, tb = T / L.n_tiles, t = T % L.n_tiles;
      const int seg_start = max(w0, T * n_st);
      const bool full = seg_start == T * n_st && w == T * n_st + n_st - 1;
      const int rows = min(kTileRows, L.N - t * kTileRows);
      const int n = t * kTileRows + r;
      const int tok_b = tok0 + tb * BN;           // first token of this block
      const int ntok = min(BN, M - tok_b);
      // a whole segment of MMAs away: sleep between polls
      if (!mbar_wait(&bar_acc[seg % NACC], (seg / NACC) & 1, abrt, 200, lim)) break;
      tc_fence_after();
      const int slot = (T == w0 / n_st) ? 0 : 1;
      float* part = work + ((size_t)(blockIdx.x * 2 + slot) * BN) * kTileRows + r;
      const uint32_t dcol = lane_base + (seg % NACC) * BN;
      // 32 columns per wait: two loads in flight before their stores
#pragma unroll 1
      for (int cc = 0; cc < BN; cc += 32) {
        uint32_t v[32];
        tmem_ld16(dcol + cc, *reinterpret_cast<uint32_t(*)[16]>(v));
        if (BN > 16) tmem_ld16(dcol + cc + 16, *reinterpret_cast<uint32_t(*)[16]>(v + 16));
        tmem_wait_ld();
        constexpr int CW = BN > 16 ? 32 : 16;
        if (full) {
          if (r < rows) {
#pragma unroll
            for (int j = 0; j < CW; ++j)
              if (cc + j < ntok) store_out(out, (size_t)(tok_b + cc + j) * L.N + n, n, __uint_as_float(v[j]));
          }
        } else {
#pragma unroll
          for (int j = 0; j < CW; ++j)
            if (cc + j < BN) part[(size_t)(cc + j) * kTileRows] = __uint_as_float(v[j]);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar_dfree[seg % NACC]);
      if (!full) {
        // Split tile: each epilogue warp counts its own 32 rows, so no
        // barrier spans warps (a warp that gave up a wait cannot strand the
        // others). The last contributor's warp sums the partials in CTA order.
        __threadfence();
        __syncwarp();
        const int c_first = cta_of(T * n_st, W, G), c_last = cta_of(T * n_st + n_st - 1, W, G);
        int last = 0;
        if (lane == 0) last = atomicAdd(counters + T * kQuads + q, 1) == c_last - c_first;
        last = __shfl_sync(0xffffffffu, last, 0);
        if (last) {
          __threadfence();
          if (r < rows && BN <= 32) {
            // all tokens of one contributor in flight at a time, added in
            // contributor order
            float acc[BN];
#pragma unroll
            for (int j = 0; j < BN; ++j) acc[j] = 0.f;
            for (int c = c_first; c <= c_last; ++c) {
              const int cs = (T == ((c * W) / G) / n_st) ? 0 : 1;
              const float* src = work + ((size_t)(c * 2 + cs) * BN) * kTileRows + r;
              float pv[BN];
#pragma unroll
              for (int j = 0; j < BN; ++j) pv[j] = j < ntok ? __ldcg(src + j * kTileRows) : 0.f;
#pragma unroll
              for (int j = 0; j < BN; ++j) acc[j] += pv[j];
            }
#pragma unroll
            for (int j = 0; j < BN; ++j)
              if (j < ntok) store_out(out, (size_t)(tok_b + j) * L.N + n, n, acc[j]);
          } else if (r < rows) {
            // 4 tokens x 8 contributors of loads in flight, then added in
            // contributor order
            for (int j0 = 0; j0 < ntok; j0 += 4) {
              float s4[4] = {0.f, 0.f, 0.f, 0.f};
              for (int c0 = c_first; c0 <= c_last; c0 += 8) {
                float pv[8][4];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                  const int c = min(c0 + e, c_last);
                  const int cs = (T == ((c * W) / G) / n_st) ? 0 : 1;
                  const float* src = work + ((size_t)(c * 2 + cs) * BN + j0) * kTileRows + r;
#pragma unroll
                  for (int u = 0; u < 4; ++u) pv[e][u] = j0 + u < ntok ? __ldcg(src + u * kTileRows) : 0.f;
                }
#pragma unroll
                for (int e = 0; e < 8; ++e)
                  if (c0 + e <= c_last) {
#pragma unroll
                    for (int u = 0; u < 4; ++u) s4[u] += pv[e][u];
                  }
              }
#pragma unroll
              for (int u = 0; u < 4; ++u)
                if (j0 + u < ntok) store_out(out, (size_t)(tok_b + j0 + u) * L.N + n, n, s4[u]);
            }
          }
          if (lane == 0) counters[T * kQuads + q] = 0;
        }
      }
    }
  } else if (warp >= kDecWarp0) {
    // ---------------- decoders: groups g0 + u kGStride, columns [16 g, 16 g + 16) of every stage
    const int g0 = (warp - kDecWarp0) >> 2;  // this warp's groups: g0, g0 + 4 / kGroupsPerWarp, ...
    constexpr int kGStride = 4 / kGroupsPerWarp;
    const int q = warp & 3;                  // TMEM lane quadrant
    const int r = q * 32 + lane;             // row of the tile
    const uint32_t lane_base = tmem + ((uint32_t)(q * 32) << 16);
    const uint32_t lane4 = (uint32_t)lane * 4u;
    // Sidecar cursor over this row's patch list (ascending columns): the
    // next two entries are always already requested, so an item without a
    // patch in this quarter costs two compares and stepping past an entry
    // of another quarter does not wait on memory.
    int cur_T = -1, pp = 0, pe = 0, pkn = INT_MAX, pk2 = INT_MAX;
    float pvn = 0.f, pv2 = 0.f;
    // entry p's column and value, loaded from a valid index whatever p
    auto fetch = [&](int p, int& k, float& v) {
      const int pc = min(p, L.n_side - 1);
      k = __ldg(L.pk + pc);
      v = __ldg(L.pv + pc);
    };
    auto step = [&]() {  // the cursor moves to the next entry
      ++pp;
      pkn = pp < pe ? pk2 : INT_MAX;
      pvn = pv2;
      if (pp + 1 < pe) fetch(pp + 1, pk2, pv2);
    };
    int b = 0, is = 0;         // A / x slot and index slot of the next item
    uint32_t bph = 0, iph = 0;  // their phase parities

    // Item i's index words (the index slot goes back to the producer), the
    // sidecar cursor moved to it, and its decoded words: hi (and mid), two
    // weights per 32-bit TMEM cell. false if a wait gave up.
    auto fetch_decode = [&](int i, uint32_t (&hi)[kGroupsPerWarp][8], uint32_t (&mid)[kGroupsPerWarp][8]) -> bool {
      const int w = w0 + i, T = w / n_st, st = w - T * n_st, t = T % L.n_tiles;
      const int rows = min(kTileRows, L.N - t * kTileRows);
      if (!mbar_wait(&bar_ifull[is], iph, abrt, 0, lim)) return false;
      const uint8_t* src = ring + (size_t)is * ISLOT + r * 16;
      uint32_t wd[kGroupsPerWarp][4];
#pragma unroll
      for (int u = 0; u < kGroupsPerWarp; ++u) {
        const int g = g0 + u * kGStride;
        wd[u][0] = wd[u][1] = wd[u][2] = wd[u][3] = 0;
        if (r < rows) {
          if (MODE == HXQ_MODE_SCALAR8) {
            const uint4 v = *reinterpret_cast<const uint4*>(src + g * rows * 16);
            wd[u][0] = v.x; wd[u][1] = v.y; wd[u][2] = v.z; wd[u][3] = v.w;
          } else {
            quarter_words_2d(src, rows, g, wd[u]);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar_ifree[is]);
      if (++is == kIS) is = 0, iph ^= 1;

      if (T != cur_T) {  // new tile: position the cursor at this stage (per-stage table)
        cur_T = T;
        const int n = t * kTileRows + r;
        pkn = INT_MAX;
        pp = pe = 0;
        if (n < L.N) {
          pp = __ldg(L.seg_ptr + (size_t)st * L.N + n);
          pe = __ldg(L.row_ptr + n + 1);
          if (pp < pe) {
            fetch(pp, pkn, pvn);
            if (pp + 1 < pe) fetch(pp + 1, pk2, pv2);
          }
        }
      }
#pragma unroll
      for (int u = 0; u < kGroupsPerWarp; ++u) {  // groups in ascending columns
        const int k0 = st * kStageK + (g0 + u * kGStride) * 16;
        while (pkn < k0) step();  // entries in other quarters
        if (MODE == HXQ_MODE_SCALAR8) {
          uint32_t v[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const uint32_t a = prmt(wd[u][j >> 2], lane4, 0x5504u | ((uint32_t)(j & 3) << 4));
            v[j] = *reinterpret_cast<const uint32_t*>(smem + a);
          }
          while (pkn < k0 + 16) {  // sidecar: substitute the stored value
            patch16(v, pkn - k0, TERMS == 1 ? (bf16_bits(pvn) << 16) : split_word(pvn));
            step();
          }
#pragma unroll
          for (int j = 0; j < 8; ++j) hi[u][j] = prmt(v[2 * j], v[2 * j + 1], 0x7632);
          if (TERMS == 2) {
#pragma unroll
            for (int j = 0; j < 8; ++j) mid[u][j] = prmt(v[2 * j], v[2 * j + 1], 0x5410);
          }
        } else {
#pragma unroll
          for (int jj = 0; jj < 8; ++jj) {  // 8 pairs = 16 weights
            const int bit = 12 * jj;
            const uint32_t e = __funnelshift_r(wd[u][bit >> 5], wd[u][(bit >> 5) + 1], bit & 31) & 0xFFF;
            if (TERMS == 1) {
              hi[u][jj] = *reinterpret_cast<const uint32_t*>(smem + e * 4);
            } else {
              const uint2 hm = *reinterpret_cast<const uint2*>(smem + e * 8);
              hi[u][jj] = hm.x;
              mid[u][jj] = hm.y;
            }
          }
          while (pkn < k0 + 16) {  // sidecar: substitute the stored value
            const int o = pkn - k0;
            if (TERMS == 1) {
              patch8_half(hi[u], o >> 1, o & 1, bf16_bits(pvn));
            } else {
              const uint32_t sw = split_word(pvn);
              patch8_half(hi[u], o >> 1, o & 1, sw >> 16);
              patch8_half(mid[u], o >> 1, o & 1, sw & 0xFFFFu);
            }
            step();
          }
        }
      }
      return true;
    };

    // Software pipeline: item i's TMEM stores drain while item i + 1 is
    // fetched and decoded; then the stores are waited for and the MMA
    // thread is told that slot b holds item i.
    uint32_t hi[kGroupsPerWarp][8], mid[kGroupsPerWarp][8], nhi[kGroupsPerWarp][8], nmid[kGroupsPerWarp][8];
    bool ok = n_items > 0 && fetch_decode(0, hi, mid);
    for (int i = 0; ok && i < n_items; ++i) {
      if (!mbar_wait(&bar_empty[b], bph ^ 1, abrt, 0, lim)) break;
      tc_fence_after();
#pragma unroll
      for (int u = 0; u < kGroupsPerWarp; ++u) {
        const uint32_t acol = lane_base + ACOL0 + b * 32 * TERMS + (g0 + u * kGStride) * 8;
        tmem_st8(acol, hi[u]);
        if (TERMS == 2) tmem_st8(acol + 32, mid[u]);
      }
      if (i + 1 < n_items) ok = fetch_decode(i + 1, nhi, nmid);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar_a[b]);
      if (++b == kSlots) b = 0, bph ^= 1;
#pragma unroll
      for (int u = 0; u < kGroupsPerWarp; ++u)
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          hi[u][j] = nhi[u][j];
          mid[u][j] = nmid[u][j];
        }
    }
  }

  // ---------------- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
  if (*abrt && threadIdx.x == 0) atomicOr(status, kStatusWaitTimeout);
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// x [M][K] into rows of ld elements (ld = K rounded up to 8), so that every
// row starts on the 16-byte boundary the activation tensor map needs.
__global__ void __launch_bounds__(256) restride_kernel(const uint16_t* __restrict__ x, uint16_t* __restrict__ xp,
                                                      int M, int K, int ld) {
  const int64_t n = (int64_t)M * K;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t m = i / K;
    xp[m * ld + (i - m * K)] = x[i];
  }
}

template <int BN, int TERMS, int MODE>
cudaError_t launch_cfg(const hxq_linear& h, const uint16_t* x, int ld, const Out& out, int M, int grid_req,
                       float* work, size_t work_floats, TestHook hook, cudaStream_t st) {
  auto fn = encode_fn();
  if (!fn) return cudaErrorNotSupported;
  CUtensorMap tm;
  cuuint64_t dims[2] = {(cuuint64_t)h.L.K, (cuuint64_t)M};
  cuuint64_t strides[1] = {(cuuint64_t)ld * 2};
  cuuint32_t box[2] = {(cuuint32_t)kStageK, (cuuint32_t)BN};
  cuuint32_t estr[2] = {1, 1};
  CUresult cr = fn(&tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(x), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (cr != CUDA_SUCCESS) return cudaErrorInvalidValue;
  // at least 116 KB of shared memory keeps one CTA per SM (each CTA takes all
  // 512 TMEM columns)
  static_assert(tc_smem_bytes<BN, TERMS, MODE>() <= kTcSmemLimit, "shared memory budget");
  const size_t smem = std::max<size_t>(tc_smem_bytes<BN, TERMS, MODE>(), 116 * 1024);
  auto kern = tc_kernel<BN, TERMS, MODE>;
  cudaError_t e = allow_max_smem(reinterpret_cast<const void*>(kern));
  if (e != cudaSuccess) return e;
  const int n_tb_all = (M + BN - 1) / BN;
  const int n_st = n_stages(h.L);
  for (int tb0 = 0; tb0 < n_tb_all; tb0 += kMaxTokBlocks) {
    const int n_tb = std::min(kMaxTokBlocks, n_tb_all - tb0);
    const int64_t U = (int64_t)n_tb * h.L.n_tiles;  // (token block, tile) pairs
    const int64_t W = U * n_st;
    // one CTA per SM, but no tile's K shared by more than kMaxContrib CTAs
    int64_t grid = grid_req > 0 ? grid_req : std::min<int64_t>(h.num_sms, U * kMaxContrib);
    grid = std::max<int64_t>(1, std::min<int64_t>({grid, (int64_t)h.num_sms, W}));
    if (W * grid >= INT_MAX) return cudaErrorInvalidValue;  // item arithmetic is 32-bit
    if ((size_t)grid * 2 * BN * kTileRows > work_floats) return cudaErrorInvalidValue;
    e = launch_pdl(kern, (unsigned)grid, kTcThreads, smem, st, tm, h.L, out, M, tb0 * BN, n_tb, work,
                   h.d_counters, h.d_status, hook);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

template <int MODE>
cudaError_t launch_mode(const hxq_linear& h, const uint16_t* x, int ld, const Out& out, int M, int grid,
                        float* work, size_t work_floats, TestHook hook, cudaStream_t st) {
  if (M <= 16) return launch_cfg<16, 2, MODE>(h, x, ld, out, M, grid, work, work_floats, hook, st);
  if (M <= 32) return launch_cfg<32, 2, MODE>(h, x, ld, out, M, grid, work, work_floats, hook, st);
  if (M <= 64) return launch_cfg<64, 1, MODE>(h, x, ld, out, M, grid, work, work_floats, hook, st);
  if (M <= 128) return launch_cfg<128, 1, MODE>(h, x, ld, out, M, grid, work, work_floats, hook, st);
  return launch_cfg<256, 1, MODE>(h, x, ld, out, M, grid, work, work_floats, hook, st);
}

}  // namespace

// Split partials of the tensor-core kernel: two slots of up to 256 tokens x
// 128 rows per CTA.
size_t tc_workspace_floats(int num_sms) { return (size_t)num_sms * 2 * 256 * kTileRows; }

// `split` (when non-zero) sets the persistent grid so that each tile's K is
// shared by about `split` CTAs; 0 = one CTA per SM.
cudaError_t launch_tc(const hxq_linear& h, const uint16_t* x, const Out& out, int M, int split, cudaStream_t st,
                      uint64_t wait_limit_ns, int withhold_item) {
  const TestHook hook{wait_limit_ns, withhold_item};
  int grid = 0;
  if (split > 0) {
    const int bn = M <= 16 ? 16 : M <= 32 ? 32 : M <= 64 ? 64 : M <= 128 ? 128 : 256;
    const int n_tb = std::min(kMaxTokBlocks, (M + bn - 1) / bn);
    grid = std::max(1, n_tb * h.L.n_tiles * split);
    grid = std::min(grid, n_tb * h.L.n_tiles * kMaxContrib * 4);
  }
  float* work = nullptr;
  size_t work_floats = 0;
  cudaError_t e = tc_workspace(h.device, st, h.num_sms, &work, &work_floats);
  if (e != cudaSuccess) return e;
  int ld = h.L.K;
  if (h.L.K % 8 != 0) {
    // the tensor map's row stride must be a multiple of 16 bytes
    ld = (h.L.K + 7) / 8 * 8;
    uint16_t* xp = nullptr;
    e = tc_xpad(h.device, st, (size_t)M * ld * sizeof(uint16_t), &xp);
    if (e != cudaSuccess) return e;
    const int64_t n = (int64_t)M * h.L.K;
    const unsigned blocks = (unsigned)std::min<int64_t>((n + 255) / 256, (int64_t)h.num_sms * 8);
    restride_kernel<<<blocks, 256, 0, st>>>(x, xp, M, h.L.K, ld);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    x = xp;
  }
  if (h.L.mode == HXQ_MODE_SCALAR8)
    return launch_mode<HXQ_MODE_SCALAR8>(h, x, ld, out, M, grid, work, work_floats, hook, st);
  return launch_mode<HXQ_MODE_VQ2D12>(h, x, ld, out, M, grid, work, work_floats, hook, st);
}

}  // namespace hxq
