// C ABI of libhxq: argument checks, the handle's device buffers, the tiled
// index re-layout, the per-row sidecar patch lists and kernel dispatch.
#include <algorithm>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <new>
#include <numeric>
#include <vector>

#include "hxq_internal.cuh"

using hxq::Layer;

namespace {

// One thread per 16-byte piece of the tiled layout (see hxq_internal.cuh).
// Source bytes beyond the end of a row are index 0.
__global__ void relayout_kernel(Layer L, const uint8_t* __restrict__ src, uint8_t* __restrict__ dst,
                                int64_t n_pieces) {
  const int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (i >= n_pieces) return;
  // pieces are enumerated row-fastest inside (tile, chunk, plane)
  const int64_t per_row_pieces = (int64_t)L.KC * L.P;
  const int64_t n = i / per_row_pieces;            // output row
  const int64_t q = i % per_row_pieces;            // (chunk, plane) of this row
  const int c = (int)(q / L.P), p = (int)(q % L.P);
  const int t = (int)(n / hxq::kTileRows), r = (int)(n % hxq::kTileRows);
  const int64_t row_bytes = (L.mode == HXQ_MODE_SCALAR8) ? L.K : 3LL * L.K / 4;
  const int64_t first = (int64_t)c * 16 * L.P + (int64_t)p * 16;   // byte within the row stream
  uint32_t w[4];
  for (int j = 0; j < 4; ++j) {
    uint32_t v = 0;
    for (int b = 0; b < 4; ++b) {
      const int64_t col = first + 4 * j + b;
      const uint32_t byte = col < row_bytes ? src[n * row_bytes + col] : 0u;
      v |= byte << (8 * b);
    }
    w[j] = v;
  }
  *reinterpret_cast<uint4*>(dst + hxq::piece_offset(L, t, c, p, r)) = make_uint4(w[0], w[1], w[2], w[3]);
}

// delta[i] = v_i - (the codebook value the sidecar entry replaces), fp32.
// `pos` holds the flat positions in patch-list order.
__global__ void sidecar_delta_kernel(Layer L, const int64_t* __restrict__ pos, int64_t n,
                                     float* __restrict__ delta) {
  const int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (i >= n) return;
  const int64_t p = pos[i];
  const int row = (int)(p / L.K), k = (int)(p % L.K);
  const int t = row / hxq::kTileRows, r = row % hxq::kTileRows;
  float c;
  if (L.mode == HXQ_MODE_SCALAR8) {
    c = L.codebook[L.idx[hxq::piece_offset(L, t, k / 16, 0, r) + k % 16]];
  } else {
    const int st = k / hxq::kStageK, bit = 12 * ((k % hxq::kStageK) / 2);
    const int b0 = bit / 8, b1 = b0 + 1;
    const uint32_t lo = L.idx[hxq::piece_offset(L, t, st, b0 / 16, r) + b0 % 16];
    const uint32_t hi = L.idx[hxq::piece_offset(L, t, st, b1 / 16, r) + b1 % 16];
    const uint32_t e = ((lo | (hi << 8)) >> (bit & 7)) & 0xFFF;
    c = L.codebook[2 * e + (k & 1)];
  }
  delta[i] = L.pv[i] - c;
}

// x (bf16 bits) from host memory the GPU reads directly (pinned and mapped)
// into a device buffer: a kernel instead of a copy-engine transfer, whose
// fixed cost is several times that of a launch for a few kilobytes. Launched
// with programmatic serialization: the host reads (the first kFetchVec
// 16-byte words of each thread) are in flight while the previous kernel,
// which may still read dst, finishes.
constexpr int kFetchVec = 4;
__global__ void __launch_bounds__(256) fetch_x_kernel(const uint16_t* __restrict__ src, uint16_t* __restrict__ dst,
                                                      int64_t n) {
  hxq::pdl_launch_dependents();
  const bool vec = ((reinterpret_cast<uintptr_t>(src) | reinterpret_cast<uintptr_t>(dst)) & 15) == 0;
  const int64_t n8 = vec ? n / 8 : 0;  // 16-byte words
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  const int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  const uint4* s4 = reinterpret_cast<const uint4*>(src);
  uint4* d4 = reinterpret_cast<uint4*>(dst);
  uint4 v[kFetchVec];
#pragma unroll
  for (int u = 0; u < kFetchVec; ++u)
    if (t + u * stride < n8) v[u] = s4[t + u * stride];
  hxq::pdl_wait();
#pragma unroll
  for (int u = 0; u < kFetchVec; ++u)
    if (t + u * stride < n8) d4[t + u * stride] = v[u];
  for (int64_t i = t + kFetchVec * stride; i < n8; i += stride) d4[i] = s4[i];
  for (int64_t i = n8 * 8 + t; i < n; i += stride) dst[i] = src[i];
}

}  // namespace

namespace hxq {
namespace {
struct StreamWorkspace {
  int device;
  cudaStream_t stream;
  float* work;
  size_t floats;
  uint16_t* xpad;  // activations re-strided to 16-byte rows (K % 8 != 0)
  size_t xpad_bytes;
};
std::mutex g_ws_mu;
std::vector<StreamWorkspace> g_ws;  // lives until the process exits
}  // namespace

cudaError_t tc_workspace(int device, cudaStream_t s, int num_sms, float** work, size_t* floats) {
  std::lock_guard<std::mutex> lock(g_ws_mu);
  for (const StreamWorkspace& w : g_ws)
    if (w.device == device && w.stream == s) {
      *work = w.work;
      *floats = w.floats;
      return cudaSuccess;
    }
  const size_t n = tc_workspace_floats(num_sms);
  float* p = nullptr;
  const cudaError_t e = cudaMalloc(reinterpret_cast<void**>(&p), n * sizeof(float));
  if (e != cudaSuccess) return e;
  try {
    g_ws.push_back({device, s, p, n, nullptr, 0});
  } catch (const std::bad_alloc&) {
    cudaFree(p);
    return cudaErrorMemoryAllocation;
  }
  *work = p;
  *floats = n;
  return cudaSuccess;
}

namespace {
std::mutex g_attr_mu;
std::vector<std::pair<int, const void*>> g_attr_done;  // (device, kernel) pairs already set up
}  // namespace

cudaError_t allow_max_smem(const void* kern) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(g_attr_mu);
  for (const auto& d : g_attr_done)
    if (d.first == dev && d.second == kern) return cudaSuccess;
  int optin = 0;
  cudaFuncAttributes fa;
  if ((e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev)) != cudaSuccess ||
      (e = cudaFuncGetAttributes(&fa, kern)) != cudaSuccess)
    return e;
  // the opt-in maximum covers static and dynamic shared memory together
  const int dyn_max = optin - (int)fa.sharedSizeBytes;
  if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, dyn_max)) != cudaSuccess ||
      (e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                                cudaSharedmemCarveoutMaxShared)) != cudaSuccess)
    return e;
  try {
    g_attr_done.emplace_back(dev, kern);
  } catch (const std::bad_alloc&) {
  }
  return cudaSuccess;
}

cudaError_t tc_xpad(int device, cudaStream_t s, size_t bytes, uint16_t** xpad) {
  std::lock_guard<std::mutex> lock(g_ws_mu);
  for (StreamWorkspace& w : g_ws) {
    if (w.device != device || w.stream != s) continue;
    if (w.xpad_bytes < bytes) {
      if (w.xpad) {
        // kernels queued on this stream may still read the old buffer
        cudaError_t e = cudaStreamSynchronize(s);
        if (e != cudaSuccess) return e;
        cudaFree(w.xpad);
        w.xpad = nullptr;
        w.xpad_bytes = 0;
      }
      const size_t grown = std::max(bytes, (size_t)1 << 20);
      cudaError_t e = cudaMalloc(reinterpret_cast<void**>(&w.xpad), grown);
      if (e != cudaSuccess) {
        w.xpad = nullptr;
        return e;
      }
      w.xpad_bytes = grown;
    }
    *xpad = w.xpad;
    return cudaSuccess;
  }
  return cudaErrorInvalidResourceHandle;  // tc_workspace creates the entry first
}
}  // namespace hxq

namespace {

int cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return HXQ_OK;
  if (e == cudaErrorMemoryAllocation) return HXQ_ENOMEM;
  return HXQ_ECUDA;
}

void free_handle(hxq_linear* h) {
  if (!h) return;
  cudaFree(h->d_codebook);
  cudaFree(h->d_idx);
  cudaFree(h->d_row_ptr);
  cudaFree(h->d_seg_ptr);
  cudaFree(h->d_pk);
  cudaFree(h->d_pv);
  cudaFree(h->d_pd);
  cudaFree(h->d_work);
  cudaFree(h->d_counters);
  cudaFree(h->d_status);
  delete h;
}

template <class T>
cudaError_t dalloc(T** p, size_t count) {
  *p = nullptr;
  if (count == 0) count = 1;
  return cudaMalloc(reinterpret_cast<void**>(p), count * sizeof(T));
}

}  // namespace

extern "C" {

const char* hxq_strerror(int code) {
  switch (code) {
    case HXQ_OK: return "ok";
    case HXQ_EINVAL: return "invalid argument";
    case HXQ_ENOMEM: return "device allocation failed";
    case HXQ_ECUDA: return "CUDA runtime or driver error";
    case HXQ_EUNSUPPORTED: return "device is not an sm_100 (B200-class) GPU";
    case HXQ_ETIMEOUT: return "a device-side wait gave up (kernel aborted)";
    default: return "unknown status";
  }
}

static int create_impl(const float* codebook, const uint8_t* indices, int mode, const int64_t* sidecar_pos,
                       const float* sidecar_val, int64_t n_sidecar, int N, int K, hxq_linear_t* out) {
  // ---- pure argument checks: no CUDA call before these pass
  if (!out) return HXQ_EINVAL;
  *out = nullptr;
  if (!codebook || !indices) return HXQ_EINVAL;
  if (mode != HXQ_MODE_SCALAR8 && mode != HXQ_MODE_VQ2D12) return HXQ_EINVAL;
  if (N < 1 || K < 1 || (mode == HXQ_MODE_VQ2D12 && (K % 4) != 0)) return HXQ_EINVAL;
  if (n_sidecar < 0 || n_sidecar > (int64_t)N * K) return HXQ_EINVAL;
  if (n_sidecar > 0 && (!sidecar_pos || !sidecar_val)) return HXQ_EINVAL;
  if (n_sidecar >= (int64_t)1 << 31) return HXQ_EINVAL;  // patch offsets are int32

  // ---- device check
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return HXQ_EUNSUPPORTED;
  }
  cudaDeviceProp prop;
  if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return HXQ_ECUDA;
  if (prop.major != 10 || prop.minor != 0) return HXQ_EUNSUPPORTED;

  // ---- sidecar: copy to the host, check it, sort it into per-row patch lists
  std::vector<int64_t> pos((size_t)n_sidecar);
  std::vector<float> val((size_t)n_sidecar);
  if (n_sidecar > 0) {
    if (cudaMemcpy(pos.data(), sidecar_pos, n_sidecar * sizeof(int64_t), cudaMemcpyDefault) != cudaSuccess ||
        cudaMemcpy(val.data(), sidecar_val, n_sidecar * sizeof(float), cudaMemcpyDefault) != cudaSuccess) {
      cudaGetLastError();
      return HXQ_ECUDA;
    }
  }
  const int64_t NK = (int64_t)N * K;
  for (int64_t i = 0; i < n_sidecar; ++i)
    if (pos[i] < 0 || pos[i] >= NK) return HXQ_EINVAL;
  std::vector<int> order((size_t)n_sidecar);
  std::iota(order.begin(), order.end(), 0);
  std::sort(order.begin(), order.end(), [&](int a, int b) { return pos[a] < pos[b]; });
  for (int64_t i = 1; i < n_sidecar; ++i)
    if (pos[order[i]] == pos[order[i - 1]]) return HXQ_EINVAL;

  // ---- handle and device buffers
  hxq_linear* h = new hxq_linear();
  std::memset(h, 0, sizeof(*h));
  Layer& L = h->L;
  L.mode = mode;
  L.N = N;
  L.K = K;
  L.Kp = (K + hxq::kStageK - 1) / hxq::kStageK * hxq::kStageK;
  L.P = mode == HXQ_MODE_SCALAR8 ? 1 : 3;
  L.KC = mode == HXQ_MODE_SCALAR8 ? L.Kp / 16 : L.Kp / 64;
  L.n_tiles = (N + hxq::kTileRows - 1) / hxq::kTileRows;
  h->n_sidecar = n_sidecar;
  h->device = dev;
  h->num_sms = prop.multiProcessorCount;
  for (int& c : h->gemv_cluster) c = -1;

  // position order = row-major order: rows, then ascending columns
  std::vector<int> row_ptr((size_t)N + 1, 0), pk((size_t)n_sidecar);
  std::vector<float> pv((size_t)n_sidecar);
  std::vector<int64_t> ppos((size_t)n_sidecar);
  for (int64_t i = 0; i < n_sidecar; ++i) {
    const int64_t p = pos[order[i]];
    row_ptr[(size_t)(p / K) + 1]++;
    pk[i] = (int)(p % K);
    pv[i] = val[order[i]];
    ppos[i] = p;
  }
  for (int n = 0; n < N; ++n) row_ptr[n + 1] += row_ptr[n];
  const int n_st = L.Kp / hxq::kStageK;
  std::vector<int> seg_ptr((size_t)(n_st + 1) * N);
  for (int n = 0; n < N; ++n) {
    int p = row_ptr[n];
    for (int st = 0; st <= n_st; ++st) {
      while (p < row_ptr[n + 1] && pk[p] < st * hxq::kStageK) ++p;
      seg_ptr[(size_t)st * N + n] = p;
    }
  }

  const size_t cb_floats = mode == HXQ_MODE_SCALAR8 ? 256 : 8192;
  const size_t idx_bytes = (size_t)N * L.KC * 16 * L.P;
  const size_t src_bytes = mode == HXQ_MODE_SCALAR8 ? (size_t)NK : (size_t)(3 * NK / 4);
  // GEMV stream-K workspace: two partial tiles of up to 8 tokens per CTA (the
  // tensor-core kernels use a workspace per device and stream, tc_workspace)
  h->work_floats = (size_t)h->num_sms * 2 * hxq::kGemvMaxTokens * hxq::kTileRows;
  h->n_counters = L.n_tiles * 64 * hxq::kQuads;  // (token block, tile, quadrant)

  cudaError_t e = cudaSuccess;
  uint8_t* d_src = nullptr;
  int64_t* d_bpos = nullptr;
  if ((e = dalloc(&h->d_codebook, cb_floats)) != cudaSuccess ||
      (e = dalloc(&h->d_idx, idx_bytes)) != cudaSuccess ||
      (e = dalloc(&h->d_row_ptr, (size_t)N + 1)) != cudaSuccess ||
      (e = dalloc(&h->d_seg_ptr, seg_ptr.size())) != cudaSuccess ||
      (e = dalloc(&h->d_pk, (size_t)n_sidecar)) != cudaSuccess ||
      (e = dalloc(&h->d_pv, (size_t)n_sidecar)) != cudaSuccess ||
      (e = dalloc(&h->d_pd, (size_t)n_sidecar)) != cudaSuccess ||
      (e = dalloc(&d_bpos, (size_t)n_sidecar)) != cudaSuccess ||
      (e = dalloc(&h->d_work, h->work_floats)) != cudaSuccess ||
      (e = dalloc(&h->d_counters, (size_t)h->n_counters)) != cudaSuccess ||
      (e = dalloc(&h->d_status, 1)) != cudaSuccess ||
      (e = dalloc(&d_src, src_bytes)) != cudaSuccess) {
    cudaFree(d_src);
    cudaFree(d_bpos);
    free_handle(h);
    cudaGetLastError();
    return cuda_status(e);
  }
  L.codebook = h->d_codebook;
  L.idx = h->d_idx;
  L.n_side = (int)n_sidecar;
  L.row_ptr = h->d_row_ptr;
  L.seg_ptr = h->d_seg_ptr;
  L.pk = h->d_pk;
  L.pv = h->d_pv;
  L.pd = h->d_pd;

  if ((e = cudaMemcpy(h->d_codebook, codebook, cb_floats * sizeof(float), cudaMemcpyDefault)) != cudaSuccess ||
      (e = cudaMemcpy(d_src, indices, src_bytes, cudaMemcpyDefault)) != cudaSuccess ||
      (e = cudaMemcpy(h->d_row_ptr, row_ptr.data(), row_ptr.size() * sizeof(int), cudaMemcpyHostToDevice)) !=
          cudaSuccess ||
      (e = cudaMemcpy(h->d_seg_ptr, seg_ptr.data(), seg_ptr.size() * sizeof(int), cudaMemcpyHostToDevice)) !=
          cudaSuccess ||
      (n_sidecar > 0 &&
       ((e = cudaMemcpy(h->d_pk, pk.data(), n_sidecar * sizeof(int), cudaMemcpyHostToDevice)) != cudaSuccess ||
        (e = cudaMemcpy(h->d_pv, pv.data(), n_sidecar * sizeof(float), cudaMemcpyHostToDevice)) != cudaSuccess ||
        (e = cudaMemcpy(d_bpos, ppos.data(), n_sidecar * sizeof(int64_t), cudaMemcpyHostToDevice)) !=
            cudaSuccess)) ||
      (e = cudaMemset(h->d_counters, 0, h->n_counters * sizeof(int))) != cudaSuccess ||
      (e = cudaMemset(h->d_status, 0, sizeof(int))) != cudaSuccess) {
    cudaFree(d_src);
    cudaFree(d_bpos);
    free_handle(h);
    cudaGetLastError();
    return cuda_status(e);
  }
  const int64_t n_pieces = (int64_t)N * L.KC * L.P;
  relayout_kernel<<<(unsigned)((n_pieces + 255) / 256), 256>>>(L, d_src, h->d_idx, n_pieces);
  e = cudaGetLastError();
  if (e == cudaSuccess && n_sidecar > 0) {
    sidecar_delta_kernel<<<(unsigned)((n_sidecar + 255) / 256), 256>>>(L, d_bpos, n_sidecar, h->d_pd);
    e = cudaGetLastError();
  }
  if (e == cudaSuccess) e = cudaDeviceSynchronize();
  cudaFree(d_src);
  cudaFree(d_bpos);
  if (e != cudaSuccess) {
    free_handle(h);
    cudaGetLastError();
    return cuda_status(e);
  }
  // the no-alloc forward's scratch address is looked up here, where
  // allocating is allowed (a failure here is reported by that entry point)
  if (hxq::noalloc_prepare(dev) != cudaSuccess) cudaGetLastError();
  *out = h;
  return HXQ_OK;
}

// No C++ exception may cross the C boundary: a host allocation that fails
// (sidecar lists of absurd size) reports HXQ_ENOMEM instead.
int hxq_linear_create(const float* codebook, const uint8_t* indices, int mode, const int64_t* sidecar_pos,
                      const float* sidecar_val, int64_t n_sidecar, int N, int K, hxq_linear_t* out) {
  try {
    return create_impl(codebook, indices, mode, sidecar_pos, sidecar_val, n_sidecar, N, K, out);
  } catch (const std::bad_alloc&) {
    cudaGetLastError();
    return HXQ_ENOMEM;
  }
}

namespace {
// The handle's device must be current: a launch on another device would
// hand its kernels pointers they cannot use. 0 if it is, else a status.
int check_device(int device) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return HXQ_ECUDA;
  }
  return dev == device ? HXQ_OK : HXQ_EINVAL;
}

int forward_impl(hxq_linear_t h, const void* x_bf16, const hxq::Out& out, int M, int kernel, int split_k,
                 void* stream) {
  if (!h || !x_bf16 || !out.y || M < 1) return HXQ_EINVAL;
  if ((reinterpret_cast<uintptr_t>(x_bf16) & 15) != 0) return HXQ_EINVAL;
  if (kernel < HXQ_KERNEL_AUTO || kernel > HXQ_KERNEL_TC) return HXQ_EINVAL;
  if (split_k < 0 || split_k > hxq::kMaxSplitK) return HXQ_EINVAL;
  if (const int rc = check_device(h->device)) return rc;
  if (kernel == HXQ_KERNEL_AUTO) kernel = (M <= 4 && hxq::gemv_supports(*h, M)) ? HXQ_KERNEL_GEMV : HXQ_KERNEL_TC;
  if (kernel == HXQ_KERNEL_GEMV && !hxq::gemv_supports(*h, M)) return HXQ_EINVAL;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const uint16_t* x = static_cast<const uint16_t*>(x_bf16);
  cudaError_t e;
  if (kernel == HXQ_KERNEL_GEMV) {
    e = hxq::launch_gemv(*h, x, out, M, split_k, s);
  } else {
    e = hxq::launch_tc(*h, x, out, M, split_k, s);
  }
  if (e != cudaSuccess) {
    cudaGetLastError();
    return e == cudaErrorInvalidValue ? HXQ_EINVAL : e == cudaErrorMemoryAllocation ? HXQ_ENOMEM : HXQ_ECUDA;
  }
  return HXQ_OK;
}
}  // namespace

int hxq_linear_forward_ex(hxq_linear_t h, const void* x_bf16, float* y, int M, int kernel, int split_k,
                          void* stream) {
  return forward_impl(h, x_bf16, hxq::Out{y, nullptr, 0}, M, kernel, split_k, stream);
}

int hxq_linear_forward(hxq_linear_t h, const void* x_bf16, float* y, int M, void* stream) {
  return forward_impl(h, x_bf16, hxq::Out{y, nullptr, 0}, M, HXQ_KERNEL_AUTO, 0, stream);
}

namespace {
// The address under which the GPU reads or writes host memory `p` directly
// (pinned memory, mapped into the device's address space), or nullptr
// (pageable memory, or not host memory at all).
void* mapped_host(const void* p) {
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  return a.type == cudaMemoryTypeHost ? a.devicePointer : nullptr;
}
}  // namespace

int hxq_linear_forward_host(hxq_linear_t h, const void* x_host, void* x_dev, float* y_dev, float* y_host, int M,
                            void* stream) {
  if (!h || !x_host || !x_dev || !y_dev || !y_host || M < 1) return HXQ_EINVAL;
  if ((reinterpret_cast<uintptr_t>(x_dev) & 15) != 0) return HXQ_EINVAL;
  if (const int rc = check_device(h->device)) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int64_t nx = (int64_t)M * h->L.K;
  cudaError_t e = cudaSuccess;
  if (const void* xm = mapped_host(x_host)) {
    const int64_t per_block = 256LL * kFetchVec * 8;  // elements a block holds across the wait
    const unsigned blocks = (unsigned)std::max<int64_t>(1, std::min<int64_t>((nx + per_block - 1) / per_block,
                                                                           (int64_t)h->num_sms));
    e = hxq::launch_pdl(fetch_x_kernel, blocks, 256, 0, s, static_cast<const uint16_t*>(xm),
                        static_cast<uint16_t*>(x_dev), nx);
  } else {
    e = cudaMemcpyAsync(x_dev, x_host, (size_t)nx * sizeof(uint16_t), cudaMemcpyHostToDevice, s);
  }
  if (e != cudaSuccess) {
    cudaGetLastError();
    return HXQ_ECUDA;
  }
  // y straight into mapped host memory: every output is written once
  float* ym = static_cast<float*>(mapped_host(y_host));
  const int rc = forward_impl(h, x_dev, hxq::Out{ym ? ym : y_dev, nullptr, 0}, M, HXQ_KERNEL_AUTO, 0, stream);
  if (rc != HXQ_OK || ym) return rc;
  if (cudaMemcpyAsync(y_host, y_dev, (size_t)M * h->L.N * sizeof(float), cudaMemcpyDeviceToHost, s) !=
      cudaSuccess) {
    cudaGetLastError();
    return HXQ_ECUDA;
  }
  return HXQ_OK;
}

int hxq_linear_forward_out(hxq_linear_t h, const void* x_bf16, const float* bias, void* y, int out_dtype, int M,
                           void* stream) {
  if (out_dtype != HXQ_OUT_F32 && out_dtype != HXQ_OUT_BF16) return HXQ_EINVAL;
  return forward_impl(h, x_bf16, hxq::Out{y, bias, out_dtype == HXQ_OUT_BF16 ? 1 : 0}, M, HXQ_KERNEL_AUTO, 0,
                      stream);
}

int hxq_group_create(const hxq_linear_t* layers, int n_layers, hxq_group_t* out) {
  if (!out) return HXQ_EINVAL;
  *out = nullptr;
  if (!layers || n_layers < 1 || n_layers > hxq::kMaxGroup) return HXQ_EINVAL;
  for (int i = 0; i < n_layers; ++i) {
    const hxq_linear* h = layers[i];
    if (!h) return HXQ_EINVAL;
    for (int j = 0; j < i; ++j)
      if (layers[j] == h) return HXQ_EINVAL;  // one workspace cannot serve two layers of a launch
    if (h->L.mode != layers[0]->L.mode || h->L.K != layers[0]->L.K || h->device != layers[0]->device)
      return HXQ_EINVAL;
  }
  hxq_group* g = new (std::nothrow) hxq_group();
  if (!g) return HXQ_ENOMEM;
  g->n = n_layers;
  for (int i = 0; i < n_layers; ++i) g->h[i] = layers[i];
  g->device = layers[0]->device;
  g->num_sms = layers[0]->num_sms;
  for (int& c : g->gemv_cluster) c = -1;
  *out = g;
  return HXQ_OK;
}

int hxq_group_forward(hxq_group_t g, const void* x_bf16, const float* const* bias, void* const* y, int out_dtype,
                      int M, void* stream) {
  if (!g || !x_bf16 || !y || M < 1) return HXQ_EINVAL;
  if ((reinterpret_cast<uintptr_t>(x_bf16) & 15) != 0) return HXQ_EINVAL;
  if (out_dtype != HXQ_OUT_F32 && out_dtype != HXQ_OUT_BF16) return HXQ_EINVAL;
  if (const int rc = check_device(g->device)) return rc;
  hxq::Out outs[hxq::kMaxGroup];
  for (int i = 0; i < g->n; ++i) {
    if (!y[i]) return HXQ_EINVAL;
    outs[i] = hxq::Out{y[i], bias ? bias[i] : nullptr, out_dtype == HXQ_OUT_BF16 ? 1 : 0};
  }
  if (M <= 4 && hxq::gemv_supports(*g->h[0], M)) {
    const cudaError_t e = hxq::launch_gemv_group(*g, static_cast<const uint16_t*>(x_bf16), outs, M,
                                                 static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) {
      cudaGetLastError();
      return e == cudaErrorInvalidValue ? HXQ_EINVAL : HXQ_ECUDA;
    }
    return HXQ_OK;
  }
  for (int i = 0; i < g->n; ++i) {
    const int rc = forward_impl(g->h[i], x_bf16, outs[i], M, HXQ_KERNEL_AUTO, 0, stream);
    if (rc != HXQ_OK) return rc;
  }
  return HXQ_OK;
}

void hxq_group_destroy(hxq_group_t g) { delete g; }

int hxq_decode(hxq_linear_t h, float* W_out, void* stream) {
  if (!h || !W_out) return HXQ_EINVAL;
  if (const int rc = check_device(h->device)) return rc;
  cudaError_t e = hxq::launch_decode(*h, W_out, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) {
    cudaGetLastError();
    return HXQ_ECUDA;
  }
  return HXQ_OK;
}

int hxq_linear_info(hxq_linear_t h, int* mode, int* N, int* K, int64_t* n_sidecar) {
  if (!h) return HXQ_EINVAL;
  if (mode) *mode = h->L.mode;
  if (N) *N = h->L.N;
  if (K) *K = h->L.K;
  if (n_sidecar) *n_sidecar = h->n_sidecar;
  return HXQ_OK;
}

int hxq_linear_check(hxq_linear_t h) {
  if (!h) return HXQ_EINVAL;
  int status = 0;
  if (cudaDeviceSynchronize() != cudaSuccess ||
      cudaMemcpy(&status, h->d_status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) {
    cudaGetLastError();
    return HXQ_ECUDA;
  }
  if (status != 0) {
    // an aborted launch may have left split-tile arrivals half counted
    cudaMemset(h->d_status, 0, sizeof(int));
    cudaMemset(h->d_counters, 0, (size_t)h->n_counters * sizeof(int));
    cudaDeviceSynchronize();
    return HXQ_ETIMEOUT;
  }
  return HXQ_OK;
}

int hxq_test_forward_withheld(hxq_linear_t h, const void* x_bf16, float* y, int M, int withhold_item,
                              unsigned wait_limit_us, void* stream) {
  if (!h || !x_bf16 || !y || M < 5 || withhold_item < 0 || wait_limit_us < 1 || wait_limit_us > 2000000u)
    return HXQ_EINVAL;
  if ((reinterpret_cast<uintptr_t>(x_bf16) & 15) != 0) return HXQ_EINVAL;
  if (const int rc = check_device(h->device)) return rc;
  const cudaError_t e = hxq::launch_tc(*h, static_cast<const uint16_t*>(x_bf16), hxq::Out{y, nullptr, 0}, M, 0,
                                       static_cast<cudaStream_t>(stream), (uint64_t)wait_limit_us * 1000ull,
                                       withhold_item);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return e == cudaErrorInvalidValue ? HXQ_EINVAL : HXQ_ECUDA;
  }
  return HXQ_OK;
}

void hxq_linear_destroy(hxq_linear_t h) {
  if (!h) return;
  cudaDeviceSynchronize();
  free_handle(h);
}

}  // extern "C"
