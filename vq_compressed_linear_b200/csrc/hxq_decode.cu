// hxq_decode: write the decoded fp32 weights W[N][K] with the sidecar
// applied. Test helper for bit-exact checks of the index layout, the 12-bit
// unpacking and the patch lists that the fused kernels share.
//
// Decode rule (scalar): W[n][k] = codebook[index], one uint8 index per
// weight (Zamba2-1.2B-HXQ model card, "What is HelixCode?"). 2D: the 12-bit
// index of pair (k, k+1) selects (c0, c1) from the 4096-pair codebook; the
// indices of one row form a little-endian bit stream, index j at bits
// [12j, 12j+12) (HXQ whitepaper, method section, 2D VQ paragraph and
// "12-bit index packing"). Sidecar entries replace single weights (HXQ
// whitepaper, method section, "Sidecar outlier correction").
#include "hxq_internal.cuh"

namespace hxq {
namespace {

// One thread per (row, chunk); consecutive threads walk along a row so the
// fp32 stores are contiguous.
__global__ void __launch_bounds__(256) decode_scalar_kernel(Layer L, float* __restrict__ W) {
  const int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (i >= (int64_t)L.N * L.KC) return;
  const int n = (int)(i / L.KC), c = (int)(i % L.KC);
  const int t = n / kTileRows, r = n % kTileRows;
  const uint4 q = *reinterpret_cast<const uint4*>(L.idx + piece_offset(L, t, c, 0, r));
  const uint32_t w[4] = {q.x, q.y, q.z, q.w};
  float v[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) v[j] = __ldg(L.codebook + ((w[j >> 2] >> (8 * (j & 3))) & 0xFF));
  const int k0 = c * 16;
  // sidecar entries of this row in this chunk (patch list sorted by column)
  for (int p = row_lower_bound(L, n, k0); p < L.row_ptr[n + 1] && L.pk[p] < k0 + 16; ++p) {
#pragma unroll
    for (int jj = 0; jj < 16; ++jj) v[jj] = sel_eq(jj, L.pk[p] - k0, L.pv[p], v[jj]);
  }
  float* out = W + (int64_t)n * L.K + k0;
  const int cnt = min(16, L.K - k0);
  if (cnt == 16 && (reinterpret_cast<uintptr_t>(out) & 15) == 0) {
#pragma unroll
    for (int j = 0; j < 16; j += 4) *reinterpret_cast<float4*>(out + j) = make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]);
  } else {
#pragma unroll
    for (int j = 0; j < 16; ++j)
      if (j < cnt) out[j] = v[j];
  }
}

__global__ void __launch_bounds__(256) decode_vq2d_kernel(Layer L, float* __restrict__ W) {
  const int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (i >= (int64_t)L.N * L.KC) return;
  const int n = (int)(i / L.KC), c = (int)(i % L.KC);
  const int t = n / kTileRows, r = n % kTileRows;
  uint32_t w[13];
#pragma unroll
  for (int p = 0; p < 3; ++p) {
    const uint4 q = *reinterpret_cast<const uint4*>(L.idx + piece_offset(L, t, c, p, r));
    w[4 * p + 0] = q.x; w[4 * p + 1] = q.y; w[4 * p + 2] = q.z; w[4 * p + 3] = q.w;
  }
  w[12] = 0;
  const float2* cb2 = reinterpret_cast<const float2*>(L.codebook);
  const int k0 = c * 64;
  float* out = W + (int64_t)n * L.K + k0;
  const int cnt = min(64, L.K - k0);
  const bool v2 = (reinterpret_cast<uintptr_t>(out) & 7) == 0;
  int p = row_lower_bound(L, n, k0);
  const int pe = L.row_ptr[n + 1];
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    const int bit = 12 * j;
    const uint32_t e = __funnelshift_r(w[bit >> 5], w[(bit >> 5) + 1], bit & 31) & 0xFFF;
    float2 v = __ldg(cb2 + e);
    for (; p < pe && L.pk[p] < k0 + 2 * j + 2; ++p) {
      if (L.pk[p] == k0 + 2 * j) v.x = L.pv[p]; else v.y = L.pv[p];
    }
    if (2 * j + 1 < cnt && v2) {
      *reinterpret_cast<float2*>(out + 2 * j) = v;
    } else if (2 * j + 1 < cnt) {
      out[2 * j] = v.x;
      out[2 * j + 1] = v.y;
    } else if (2 * j < cnt) {
      out[2 * j] = v.x;
    }
  }
}

}  // namespace

cudaError_t launch_decode(const hxq_linear& h, float* W, cudaStream_t s) {
  const int64_t threads = (int64_t)h.L.N * h.L.KC;
  const unsigned blocks = (unsigned)((threads + 255) / 256);
  if (h.L.mode == HXQ_MODE_SCALAR8)
    decode_scalar_kernel<<<blocks, 256, 0, s>>>(h.L, W);
  else
    decode_vq2d_kernel<<<blocks, 256, 0, s>>>(h.L, W);
  return cudaGetLastError();
}

}  // namespace hxq
