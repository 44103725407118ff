// Fused decode + GEMM on the sm_100a tensor cores (tcgen05), for M > 4:
//   y[m][n] = sum_k x[m][k] * W[n][k],  W decoded on the fly, never stored.
//
// The MMA computes D = A . B^T with A = a 128-row tile of W (output features)
// and B = a tile of BN tokens of x, so D = y^T for that tile and lives in
// tensor memory (TMEM): lane = output feature, column = token.
//
//  * A is written by the decoding warps straight from registers into TMEM
//    with tcgen05.st (the "A from tensor memory" form of tcgen05.mma): the
//    decoded weights never touch shared or global memory. Thread r of a
//    decoding warp group owns TMEM lane r = row r of the tile; it reads its
//    16-byte index pieces (a warp reads 512 contiguous bytes), looks the
//    indices up in a shared-memory table, patches sidecar columns, packs two
//    bf16 per 32-bit TMEM cell and stores 64 weights (one pipeline stage) at
//    a time.
//  * B (x) arrives by TMA into 128-byte-swizzled shared memory, 64 tokens'
//    worth of K per stage; rows past M and columns past K read as zero.
//  * One thread issues tcgen05.mma (kind::f16, bf16 x bf16 -> fp32 in TMEM)
//    and signals stage release and completion with tcgen05.commit.
//  * The decoding warps then read D back with tcgen05.ld and store y (or a
//    split-K partial; the last of the S partials of a tile sums them in order).
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
// Pipeline: kStages slots, each with an x buffer (TMA) and an A region in
// TMEM; mbarriers full_x / full_a / empty per slot and one for the
// accumulator. Every wait is bounded (2 s): on timeout the CTA sets a status
// bit, drains what it issued, frees TMEM and returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <climits>

#include "hxq_internal.cuh"

namespace hxq {
namespace {

constexpr int kStages = 4;
constexpr int kDecodeGroups = 4;                       // groups of 4 warps (128 rows)
constexpr int kTcThreads = 128 + kDecodeGroups * 128;  // warps 0..3 control, 4.. decode
constexpr int kAColBase = 256;                         // A regions live in TMEM columns 256..511
constexpr int kTmemCols = 512;

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

template <int BN, int TERMS, int MODE>
constexpr size_t tc_smem_bytes() {
  return 1024 /* alignment slack */ + (size_t)kStages * BN * 128 + table_bytes<MODE, TERMS>();
}

// Replace the weight at column offset j (0..15) of a 16-weight chunk by the
// word `pw` (scalar tables: one word per weight).
__device__ __forceinline__ void patch16(uint32_t (&v)[16], int j, uint32_t pw) {
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = sel_eq(i, j, pw, v[i]);
}
// Replace half `h` of pair word j (0..7) by the 16-bit value hv.
__device__ __forceinline__ void patch8_half(uint32_t (&v)[8], int j, int h, uint32_t hv) {
#pragma unroll
  for (int i = 0; i < 8; ++i)
    v[i] = sel_eq(i, j, h ? ((v[i] & 0xFFFFu) | (hv << 16)) : ((v[i] & 0xFFFF0000u) | hv), v[i]);
}

template <int BN, int TERMS, int MODE>
__global__ void __launch_bounds__(kTcThreads, 1)
tc_kernel(const __grid_constant__ CUtensorMap tmx, Layer L, float* __restrict__ y, int M, int S,
          float* __restrict__ work, int* __restrict__ counters, int* __restrict__ status) {
  constexpr int XSLOT = BN * 128;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint8_t* xs = smem;
  uint8_t* table = smem + kStages * XSLOT;
  __shared__ uint64_t bar_x[kStages], bar_a[kStages], bar_empty[kStages], bar_acc;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh, last_sh;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_tb = (M + BN - 1) / BN;
  int u = blockIdx.x;
  const int s = u % S;
  u /= S;
  const int tb = u % n_tb, t = u / n_tb;
  const int n_stages_all = L.Kp / kStageK;
  const int st0 = (int)((int64_t)s * n_stages_all / S);
  const int st1 = (int)((int64_t)(s + 1) * n_stages_all / S);
  const int nst = st1 - st0;
  const int rows = min(kTileRows, L.N - t * kTileRows);

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&bar_x[i], 1);
      mbar_init(&bar_a[i], 4);
      mbar_init(&bar_empty[i], 1);
    }
    mbar_init(&bar_acc, 1);
    abort_sh = 0;
    last_sh = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) prefetch_tmap(&tmx);
  if (warp == 1) {
    tmem_alloc(&tmem_base_sh, kTmemCols);
    tmem_relinquish();
  }
  // shared-memory decode table
  if (MODE == HXQ_MODE_SCALAR8) {
    uint32_t* tw = reinterpret_cast<uint32_t*>(table);
    for (int i = threadIdx.x; i < 256 * 32; i += blockDim.x) {
      const float c = __ldg(L.codebook + (i >> 5));
      tw[(i >> 5) * 64 + (i & 31)] = TERMS == 1 ? (bf16_bits(c) << 16) : split_word(c);
    }
  } else {
    const float2* cb2 = reinterpret_cast<const float2*>(L.codebook);
    for (int i = threadIdx.x; i < 4096; i += blockDim.x) {
      const float2 c = __ldg(cb2 + i);
      if (TERMS == 1) {
        reinterpret_cast<uint32_t*>(table)[i] = bf16_bits(c.x) | (bf16_bits(c.y) << 16);
      } else {
        const uint32_t a = split_word(c.x), b = split_word(c.y);
        reinterpret_cast<uint2*>(table)[i] = make_uint2(prmt(a, b, 0x7632), prmt(a, b, 0x5410));
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
      int issued = 0;
      for (int i = 0; i < nst; ++i) {
        const int b = i % kStages;
        if (!mbar_wait(&bar_empty[b], ((i / kStages) & 1) ^ 1, abrt)) break;
        mbar_arrive_expect_tx(&bar_x[b], XSLOT);
        tma_load_2d(xs + b * XSLOT, &tmx, &bar_x[b], (st0 + i) * kStageK, tb * BN);
        ++issued;
      }
      if (*abrt) {  // drain the loads this thread issued before leaving
        for (int i = max(0, issued - kStages); i < issued; ++i) {
          volatile int never = 0;
          mbar_wait(&bar_x[i % kStages], (i / kStages) & 1, &never);
        }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16<BN>();
      for (int i = 0; i < nst; ++i) {
        const int b = i % kStages;
        const uint32_t par = (i / kStages) & 1;
        if (!mbar_wait(&bar_x[b], par, abrt)) break;
        if (!mbar_wait(&bar_a[b], par, abrt)) break;
        tc_fence_after();
        const uint32_t xaddr = smem_u32(xs + b * XSLOT);
#pragma unroll
        for (int kk = 0; kk < kStageK / 16; ++kk) {
          const uint64_t bdesc = smem_desc_sw128(xaddr + kk * 32);
#pragma unroll
          for (int term = 0; term < TERMS; ++term) {
            const uint32_t acol = tmem + kAColBase + b * 32 * TERMS + term * 32 + kk * 8;
            tc_mma_ts(tmem, acol, bdesc, idesc, (i | kk | term) ? 1u : 0u);
          }
        }
        tc_commit(&bar_empty[b]);
      }
      tc_commit(&bar_acc);
      if (*abrt) {  // let issued MMAs finish before TMEM is freed
        volatile int never = 0;
        mbar_wait(&bar_acc, 0, &never);
      }
    }
  } else if (warp >= 4) {
    // ---------------- decoders, then epilogue
    const int dg = (warp - 4) >> 2;  // decode group
    const int q = warp & 3;          // TMEM lane quadrant
    const int r = q * 32 + lane;     // row of the tile
    const int n = t * kTileRows + r;
    const bool valid = r < rows;
    const uint32_t lane_base = tmem + ((uint32_t)(q * 32) << 16);
    const uint32_t lane4 = (uint32_t)lane * 4u;
    const char* tb8 = reinterpret_cast<const char*>(table);

    int p = 0, pend = 0, pk = INT_MAX;
    if (valid) {
      int lo = L.row_ptr[n], hi = L.row_ptr[n + 1];
      pend = hi;
      const int k0 = st0 * kStageK;
      while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (L.patch_k[mid] < k0) lo = mid + 1; else hi = mid;
      }
      p = lo;
      pk = p < pend ? L.patch_k[p] : INT_MAX;
    }
    constexpr int NPC = MODE == HXQ_MODE_SCALAR8 ? 4 : 3;  // 16-byte pieces per stage
    uint4 qn[NPC];
    auto load_stage = [&](int st, uint4 (&dst)[NPC]) {
#pragma unroll
      for (int c = 0; c < NPC; ++c) {
        if (valid) {
          const int chunk = MODE == HXQ_MODE_SCALAR8 ? st * 4 + c : st;
          const int plane = MODE == HXQ_MODE_SCALAR8 ? 0 : c;
          dst[c] = ldg_stream16(L.idx + piece_offset(L, t, chunk, plane, r));
        } else {
          dst[c] = make_uint4(0, 0, 0, 0);
        }
      }
    };
    if (dg < nst) load_stage(st0 + dg, qn);

    for (int i = dg; i < nst; i += kDecodeGroups) {
      const int b = i % kStages;
      uint4 qc[NPC];
#pragma unroll
      for (int c = 0; c < NPC; ++c) qc[c] = qn[c];
      if (i + kDecodeGroups < nst) load_stage(st0 + i + kDecodeGroups, qn);
      if (!mbar_wait(&bar_empty[b], ((i / kStages) & 1) ^ 1, abrt)) break;
      tc_fence_after();
      const uint32_t acol = lane_base + kAColBase + b * 32 * TERMS;
      const int kst = (st0 + i) * kStageK;
      if (MODE == HXQ_MODE_SCALAR8) {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const uint32_t wd[4] = {qc[c].x, qc[c].y, qc[c].z, qc[c].w};
          uint32_t v[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const uint32_t a = prmt(wd[j >> 2], lane4, 0x5504u | ((uint32_t)(j & 3) << 4));
            v[j] = *reinterpret_cast<const uint32_t*>(tb8 + a);
          }
          const int k0 = kst + c * 16;
          while (pk < k0 + 16) {
            const float pv = L.patch_v[p];
            patch16(v, pk - k0, TERMS == 1 ? (bf16_bits(pv) << 16) : split_word(pv));
            ++p;
            pk = p < pend ? L.patch_k[p] : INT_MAX;
          }
          uint32_t hi[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) hi[j] = prmt(v[2 * j], v[2 * j + 1], 0x7632);
          tmem_st8(acol + c * 8, hi);
          if (TERMS == 2) {
            uint32_t mid[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) mid[j] = prmt(v[2 * j], v[2 * j + 1], 0x5410);
            tmem_st8(acol + 32 + c * 8, mid);
          }
        }
      } else {
        uint32_t w[13];
#pragma unroll
        for (int c = 0; c < 3; ++c) {
          w[4 * c] = qc[c].x; w[4 * c + 1] = qc[c].y; w[4 * c + 2] = qc[c].z; w[4 * c + 3] = qc[c].w;
        }
        w[12] = 0;
#pragma unroll
        for (int h = 0; h < 4; ++h) {  // 8 pairs = 16 weights per step
          uint32_t hi[8], mid[8];
#pragma unroll
          for (int jj = 0; jj < 8; ++jj) {
            const int j = h * 8 + jj, bit = 12 * j;
            const uint32_t e = __funnelshift_r(w[bit >> 5], w[(bit >> 5) + 1], bit & 31) & 0xFFF;
            if (TERMS == 1) {
              hi[jj] = reinterpret_cast<const uint32_t*>(table)[e];
            } else {
              const uint2 hm = reinterpret_cast<const uint2*>(table)[e];
              hi[jj] = hm.x;
              mid[jj] = hm.y;
            }
          }
          const int k0 = kst + h * 16;
          while (pk < k0 + 16) {
            const float pv = L.patch_v[p];
            const int o = pk - k0;
            if (TERMS == 1) {
              patch8_half(hi, o >> 1, o & 1, bf16_bits(pv));
            } else {
              const uint32_t sw = split_word(pv);
              patch8_half(hi, o >> 1, o & 1, sw >> 16);
              patch8_half(mid, o >> 1, o & 1, sw & 0xFFFFu);
            }
            ++p;
            pk = p < pend ? L.patch_k[p] : INT_MAX;
          }
          tmem_st8(acol + h * 8, hi);
          if (TERMS == 2) tmem_st8(acol + 32 + h * 8, mid);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar_a[b]);
    }

    // ---------------- epilogue: D (y^T tile) from TMEM to y / workspace
    if (!*abrt && mbar_wait(&bar_acc, 0, abrt)) {
      tc_fence_after();
      for (int cc = dg * 16; cc < BN; cc += kDecodeGroups * 16) {
        uint32_t v[16];
        tmem_ld16(lane_base + cc, v);
        tmem_wait_ld();
        if (valid) {
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int tok = tb * BN + cc + j;
            if (tok < M) {
              if (S == 1) y[(size_t)tok * L.N + n] = __uint_as_float(v[j]);
              else work[((size_t)s * M + tok) * L.N + n] = __uint_as_float(v[j]);
            }
          }
        }
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
  if (*abrt) {
    if (threadIdx.x == 0) atomicOr(status, kStatusWaitTimeout);
    return;
  }
  if (S == 1) return;
  __threadfence();
  __syncthreads();
  int* ctr = counters + t * 64 + tb;
  if (threadIdx.x == 0) last_sh = atomicAdd(ctr, 1) == S - 1;
  __syncthreads();
  if (!last_sh) return;
  __threadfence();
  const int ntok = min(BN, M - tb * BN);
  for (int i = threadIdx.x; i < ntok * rows; i += blockDim.x) {
    const int j = i / rows, rr = i % rows;
    const int tok = tb * BN + j;
    const size_t nn = (size_t)t * kTileRows + rr;
    float v = 0.f;
    for (int ss = 0; ss < S; ++ss) v += __ldcg(work + ((size_t)ss * M + tok) * L.N + nn);
    y[(size_t)tok * L.N + nn] = v;
  }
  if (threadIdx.x == 0) *ctr = 0;
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

template <int BN, int TERMS, int MODE>
cudaError_t launch_cfg(const hxq_linear& h, const uint16_t* x, float* y, int M, int S, cudaStream_t st) {
  auto fn = encode_fn();
  if (!fn) return cudaErrorNotSupported;
  CUtensorMap tm;
  cuuint64_t dims[2] = {(cuuint64_t)h.L.K, (cuuint64_t)M};
  cuuint64_t strides[1] = {(cuuint64_t)h.L.K * 2};
  cuuint32_t box[2] = {(cuuint32_t)kStageK, (cuuint32_t)BN};
  cuuint32_t estr[2] = {1, 1};
  CUresult cr = fn(&tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(x), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (cr != CUDA_SUCCESS) return cudaErrorInvalidValue;
  // at least 116 KB of shared memory keeps one CTA per SM (each CTA takes all
  // 512 TMEM columns)
  const size_t smem = std::max<size_t>(tc_smem_bytes<BN, TERMS, MODE>(), 116 * 1024);
  auto kern = tc_kernel<BN, TERMS, MODE>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int n_tb = (M + BN - 1) / BN;
  const int64_t units = (int64_t)h.L.n_tiles * n_tb * S;
  kern<<<(unsigned)units, kTcThreads, smem, st>>>(tm, h.L, y, M, S, h.d_work, h.d_counters, h.d_status);
  return cudaGetLastError();
}

template <int MODE>
cudaError_t launch_mode(const hxq_linear& h, const uint16_t* x, float* y, int M, int S, cudaStream_t st) {
  if (M <= 16) return launch_cfg<16, 2, MODE>(h, x, y, M, S, st);
  if (M <= 32) return launch_cfg<32, 2, MODE>(h, x, y, M, S, st);
  if (M <= 64) return launch_cfg<64, 1, MODE>(h, x, y, M, S, st);
  if (M <= 128) return launch_cfg<128, 1, MODE>(h, x, y, M, S, st);
  return launch_cfg<256, 1, MODE>(h, x, y, M, S, st);
}

int tc_bn(int M) { return M <= 16 ? 16 : M <= 32 ? 32 : M <= 64 ? 64 : M <= 128 ? 128 : 256; }

}  // namespace

int choose_split_tc(const hxq_linear& h, int M) {
  const int n_stages = h.L.Kp / kStageK;
  const int n_tb = (M + tc_bn(M) - 1) / tc_bn(M);
  if (n_tb > 64) return 1;  // split-K counters cover 64 token blocks per tile
  const int slots = h.num_sms;
  int best = 1;
  double best_score = -1.0;
  for (int S = 1; S <= std::min(n_stages, kMaxSplitK); ++S) {
    if (S > 1 && (size_t)S * M * h.L.N > h.work_floats) break;
    const int64_t units = (int64_t)h.L.n_tiles * n_tb * S;
    const int64_t waves = (units + slots - 1) / slots;
    const double wave_eff = (double)units / ((double)waves * slots);
    const double per_unit = (double)n_stages / S;
    const double pipe_eff = std::min(1.0, per_unit / (2.0 * kStages));
    const double score = wave_eff * pipe_eff / (1.0 + 0.002 * S);
    if (score > best_score + 1e-9) {
      best_score = score;
      best = S;
    }
  }
  return best;
}

cudaError_t launch_tc(const hxq_linear& h, const uint16_t* x, float* y, int M, int split, cudaStream_t st) {
  const int n_stages = h.L.Kp / kStageK;
  const int S = std::max(1, std::min(split, n_stages));
  const int n_tb = (M + tc_bn(M) - 1) / tc_bn(M);
  if (S > 1 && ((size_t)S * M * h.L.N > h.work_floats || n_tb > 64)) return cudaErrorInvalidValue;
  if (h.L.mode == HXQ_MODE_SCALAR8) return launch_mode<HXQ_MODE_SCALAR8>(h, x, y, M, S, st);
  return launch_mode<HXQ_MODE_VQ2D12>(h, x, y, M, S, st);
}

}  // namespace hxq
