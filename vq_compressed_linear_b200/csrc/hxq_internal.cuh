// Internal definitions shared by the libhxq translation units: the handle,
// the tiled index layout, the per-row sidecar patch lists and thin inline-PTX
// wrappers for mbarriers, TMA and tcgen05 (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "hxq.h"  // include/ (on the include path)

namespace hxq {

// ----------------------------------------------------------------------------
// Index layout owned by a handle.
//
// Rows are grouped in tiles of kTileRows = 128 output features (one per TMEM
// lane / one per thread of a 128-thread group). Within a row the weights are
// cut into chunks: 16 weights = 16 bytes in scalar mode, 64 weights = 32
// pairs = 48 bytes = 3 planes of 16 bytes in 2D mode. The tile stores, for
// every chunk and plane, the 16-byte pieces of all its rows back to back, so
// that 32 consecutive rows read 512 consecutive bytes:
//
//   piece(tile t, chunk c, plane p, row r) at byte
//     t*128*KC*CB + (c*P + p)*R_t*16 + r*16
//
// with KC chunks per row, P planes per chunk, CB = 16*P bytes per chunk and
// R_t = min(128, N - 128 t) rows in tile t. K is padded to a multiple of 64
// (kStageK) with index 0; the kernels pair padded weights only with zero
// activations, so a finite codebook entry 0 contributes nothing.
// ----------------------------------------------------------------------------
constexpr int kTileRows = 128;
constexpr int kStageK = 64;           // weights per row per pipeline stage
constexpr int kMaxSplitK = 64;
constexpr int kMaxGroup = HXQ_MAX_GROUP;  // layers in one grouped launch

struct Layer {
  int mode;          // HXQ_MODE_*
  int N, K;
  int Kp;            // K rounded up to kStageK
  int KC;            // chunks per row: Kp/16 (scalar) or Kp/64 (2D)
  int P;             // planes per chunk: 1 (scalar) or 3 (2D)
  int n_tiles;       // ceil(N / 128)
  const float* codebook;     // 256 or 4096*2 floats
  const uint8_t* idx;        // tiled layout above
  // Sidecar as per-row patch lists: the entries of row n are
  // [row_ptr[n], row_ptr[n+1]), in ascending column order.
  const int* row_ptr;        // [N+1]
  // seg_ptr[s * N + n]: the first of row n's entries whose column is at
  // least s * kStageK (s = 0 .. Kp / kStageK), so that a run of stages
  // finds its entries without a search.
  const int* seg_ptr;
  const int* pk;             // column k
  const float* pv;           // the replacement value v
  const float* pd;           // v - (codebook value it replaces), rounded to fp32
  int n_side;                // number of entries
};

constexpr int kQuads = kTileRows / 32;

// Where a forward writes: y[m][n] (+ bias[n]) as fp32, or rounded to bf16
// (round to nearest even).
struct Out {
  void* y;
  const float* bias;  // [N] fp32, or null
  int bf16;           // 0: fp32 y, 1: bf16 y
};

__host__ __device__ inline int n_stages(const Layer& L) { return L.Kp / kStageK; }

__host__ __device__ inline size_t piece_offset(const Layer& L, int t, int c, int p, int r) {
  const int rows = min(kTileRows, L.N - t * kTileRows);
  return (size_t)t * kTileRows * L.KC * (16 * L.P) + ((size_t)c * L.P + p) * rows * 16 + (size_t)r * 16;
}

}  // namespace hxq

struct hxq_linear {
  hxq::Layer L;
  int64_t n_sidecar;
  int device;
  int num_sms;
  float* d_codebook;
  uint8_t* d_idx;
  int* d_row_ptr;
  int* d_seg_ptr;
  int* d_pk;
  float* d_pv;
  float* d_pd;
  float* d_work;        // split-K partial sums
  size_t work_floats;
  int* d_counters;      // per output tile: arrivals of split-K partials
  int n_counters;
  int* d_status;        // device-side error word (bounded waits that gave up)
  // GEMV cluster size chosen per (token count class, activation staging):
  // -1 = not yet chosen, 0 = stream-K
  mutable int gemv_cluster[8];
};

// Layers that share their activations (same mode and K, one device); the
// handles are borrowed.
struct hxq_group {
  int n;
  hxq_linear* h[hxq::kMaxGroup];
  int device;
  int num_sms;
  // cluster size of the grouped GEMV, as hxq_linear::gemv_cluster
  mutable int gemv_cluster[8];
};

namespace hxq {

// Launchers (each returns a cudaError_t from the launch).
cudaError_t launch_decode(const hxq_linear& h, float* W, cudaStream_t s);
cudaError_t launch_gemv(const hxq_linear& h, const uint16_t* x, const Out& out, int M, int split,
                        cudaStream_t s);
// wait_limit_ns bounds every pipeline wait; withhold_item >= 0 is a test
// hook (that item of each CTA never gets its activations).
cudaError_t launch_tc(const hxq_linear& h, const uint16_t* x, const Out& out, int M, int split,
                      cudaStream_t s, uint64_t wait_limit_ns = 2000000000ull, int withhold_item = -1);
// One launch of the GEMV over every layer of g (outs[i] for layer i).
cudaError_t launch_gemv_group(const hxq_group& g, const uint16_t* x, const Out* outs, int M, cudaStream_t s);
bool gemv_supports(const hxq_linear& h, int M);
// Resolves (and caches) the device address of the no-alloc entry point's
// scratch array on the current device `dev`.
cudaError_t noalloc_prepare(int dev);
int gemv_grid(const hxq_linear& h, int split);
size_t tc_workspace_floats(int num_sms);
// The tensor-core kernels' split-partial workspace for (device, stream):
// allocated by the first tensor-core forward on that stream of that device
// and kept until the process exits, so that forwards on different streams
// never share one. cudaErrorMemoryAllocation if it cannot be allocated.
cudaError_t tc_workspace(int device, cudaStream_t s, int num_sms, float** work, size_t* floats);
// Lets `kern` launch with up to the device's opt-in maximum of dynamic shared
// memory and asks for the largest shared-memory carveout, once per (device,
// kernel): the launch's own size then sets its occupancy, and launches do not
// repeat the driver calls.
cudaError_t allow_max_smem(const void* kern);
// A buffer of at least `bytes` for activations re-strided to 16-byte rows on
// (device, stream), which tc_workspace must have created; grown (after a
// synchronize of `s`) when a larger one is asked for.
cudaError_t tc_xpad(int device, cudaStream_t s, size_t bytes, uint16_t** xpad);
// GEMV split partials per handle: two partial tiles of up to kGemvMaxTokens x
// 128 floats per CTA.
constexpr int kGemvMaxTokens = 8;

// Launch `kern` with programmatic stream serialization: it may start while
// the previous kernel in the stream drains, and waits for it (griddepcontrol
// .wait) only where it reads that kernel's results.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), unsigned grid, unsigned block, size_t smem, cudaStream_t s,
                       Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(block);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

// As launch_pdl, with the grid in clusters of `cluster` CTAs (1 = none),
// each cluster's CTAs spread over distinct SMs.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl_cluster(void (*kern)(KArgs...), unsigned grid, unsigned block, size_t smem, unsigned cluster,
                               cudaStream_t s, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(block);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[3];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = cluster;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  attr[2].id = cudaLaunchAttributeClusterSchedulingPolicyPreference;
  attr[2].val.clusterSchedulingPolicyPreference = cudaClusterSchedulingPolicySpread;
  cfg.attrs = attr;
  cfg.numAttrs = 3;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

// Device status bits.
constexpr int kStatusWaitTimeout = 1;

// ----------------------------------------------------------------------------
// Inline PTX helpers (sm_100a).
// ----------------------------------------------------------------------------
#if defined(__CUDACC__)

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;"
               ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait for the phase with the given parity to complete. Gives up after
// kWaitLimitNs of wall time or as soon as another thread of the CTA has set
// *abort; on giving up it sets *abort and returns false. A normal launch never
// comes near the limit (kernels here run for microseconds). A waiter off the
// critical path passes sleep_ns > 0 to sleep between polls, so that its warp
// does not take issue slots from the warps doing the work.
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s

__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort,
                                          uint32_t sleep_ns = 0, uint64_t limit_ns = kWaitLimitNs) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t i = 1;; ++i) {
    if (sleep_ns) __nanosleep(sleep_ns);
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 63) == 0) {  // the abort flag and the clock are read now and then, not on every poll
      if (*abort) return false;
      if (globaltimer_ns() - t0 > limit_ns) {
        *abort = 1;
        return false;
      }
    }
  }
}

// 2D tiled TMA load global -> shared, completion counted on `bar` in bytes.
__device__ __forceinline__ void tma_load_2d(void* dst, const void* tmap, uint64_t* bar, int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
      ::"r"(smem_u32(dst)), "l"(tmap), "r"(c0), "r"(c1), "r"(smem_u32(bar))
      : "memory");
}

// 1D bulk copy global -> shared (TMA engine), completion counted on `bar` in
// bytes. Addresses 16-byte aligned, size a multiple of 16.
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
               ::"r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void prefetch_tmap(const void* tmap) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(tmap) : "memory");
}

// ---- tcgen05 ---------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
               ::"r"(smem_u32(dst_smem)), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// D[tmem] (+)= A[tmem] * B[smem]^T, kind::f16 (bf16 inputs, fp32 accumulate).
__device__ __forceinline__ void tc_mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}"
      ::"r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive once on `bar` when all previously issued tcgen05.mma of this thread finish.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
               ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&v)[8]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};"
               ::"r"(taddr), "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]),
                 "r"(v[6]), "r"(v[7])
               : "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
      "%12, %13, %14, %15}, [%16];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
        "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]),
        "=r"(v[14]), "=r"(v[15])
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// (a == b) ? x : y as one predicated select; written in PTX so that an
// unrolled chain of these over a register array stays in registers instead
// of being turned into a dynamically indexed local-memory store.
__device__ __forceinline__ uint32_t sel_eq(int a, int b, uint32_t x, uint32_t y) {
  uint32_t r;
  asm("{\n\t.reg .pred p;\n\tsetp.eq.s32 p, %1, %2;\n\tselp.b32 %0, %3, %4, p;\n\t}"
      : "=r"(r) : "r"(a), "r"(b), "r"(x), "r"(y));
  return r;
}
__device__ __forceinline__ float sel_eq(int a, int b, float x, float y) {
  return __uint_as_float(sel_eq(a, b, __float_as_uint(x), __float_as_uint(y)));
}

// First entry of row n's patch list with column >= k0 (binary search).
__device__ __forceinline__ int row_lower_bound(const Layer& L, int n, int k0) {
  int lo = L.row_ptr[n], hi = L.row_ptr[n + 1];
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (__ldg(L.pk + mid) < k0) lo = mid + 1; else hi = mid;
  }
  return lo;
}

// Byte permute: result byte i = byte sel_i of the 8-byte value {b:a}.
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
  return r;
}

// Asynchronous bulk prefetch of [p, p + bytes) from global memory into L2
// (TMA engine; no registers, completes on its own). p and bytes: multiples of 16.
__device__ __forceinline__ void prefetch_l2_bulk(const void* p, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

// Programmatic dependent launch: let the next kernel in the stream start its
// prologue now / wait until the previous kernel's results are visible.
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Stores output element idx (feature n) of a forward.
__device__ __forceinline__ void store_out(const Out& o, size_t idx, int n, float v) {
  if (o.bias) v += __ldg(o.bias + n);
  if (o.bf16) {
    reinterpret_cast<__nv_bfloat16*>(o.y)[idx] = __float2bfloat16_rn(v);
  } else {
    reinterpret_cast<float*>(o.y)[idx] = v;
  }
}

// Load with acquire semantics at GPU scope (pairs with a writer's fence +
// atomic, e.g. the stream-K arrival counters).
__device__ __forceinline__ int ld_acquire_gpu(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void named_bar_sync(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}
// Named barrier that also returns whether `v` held in every participating thread.
__device__ __forceinline__ bool named_bar_and(int id, int threads, bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 q, %3, 0;\n\t"
      "barrier.cta.red.and.pred p, %1, %2, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(r)
      : "r"(id), "r"(threads), "r"((uint32_t)v)
      : "memory");
  return r != 0;
}
__device__ __forceinline__ void named_bar_arrive(int id, int threads) {
  asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// Thread-block clusters: the CTA's rank, a shared-memory address mapped to
// another CTA of the cluster, a store there, and the cluster barrier (all
// threads of every CTA in the cluster take part; arrive does not wait).
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t map_to_rank(uint32_t smem_addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_addr), "r"(rank));
  return r;
}
__device__ __forceinline__ void st_cluster_f32(uint32_t addr, float v) {
  asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(addr), "f"(v) : "memory");
}
__device__ __forceinline__ void cluster_arrive_relaxed() {
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_arrive_release() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory"); }

__device__ __forceinline__ uint4 ldg_stream16(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

#endif  // __CUDACC__

}  // namespace hxq
