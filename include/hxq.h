/*
 * hxq.h -- C ABI of libhxq: the HXQ / HelixCode HelixLinear forward
 *          y = x . W^T on NVIDIA B200 (sm_100a), W never stored dense.
 *
 * What is computed (sources are the pages this library follows):
 *  - Scalar mode: W[n][k] = codebook[indices[n*K + k]], a 256-entry fp32
 *    codebook addressed by one uint8 per weight (Zamba2-1.2B-HXQ model card,
 *    "What is HelixCode?").
 *  - 2D mode: weights (k, k+1), k even, of row n are one entry of a
 *    4096-entry codebook of fp32 pairs, addressed by a 12-bit index; the
 *    indices are packed two per 3 bytes (HXQ whitepaper, method section:
 *    2D VQ paragraph and the "12-bit index packing" pipeline step).
 *  - Sidecar: each (flat position p = n*K + k, fp32 value v) replaces W[n][k]
 *    by v (HXQ whitepaper, method section, "Sidecar outlier correction").
 *  - Forward: y[m][n] = sum_k x[m][k] * W[n][k] for bf16 x and fp32 y, the
 *    product that the pages' HelixLinear runs in place of nn.Linear
 *    (HXQ whitepaper, method section, buffered forward path paragraph).
 *
 * Layouts (all row-major, no padding, no strides):
 *  codebook   scalar: float[256];  2D: float[4096][2] (component 0 -> even k)
 *  indices    scalar: uint8[N][K]; 2D: uint8[3*N*K/4], a flat stream of 3-byte
 *             groups over the pairs in row-major order g = n*K/2 + k/2; the
 *             group's 24-bit little-endian word b0 | b1<<8 | b2<<16 holds the
 *             even pair's index in bits 0..11 and the odd pair's in 12..23
 *  sidecar    int64 positions (unique, in [0, N*K)) and float values
 *  x          bf16 [M][K] (raw bits, 2 bytes per element)
 *  y          float [M][N]
 *
 * Numerics: M <= 32 computes with the fp32 codebook values (error within
 * 1e-5 * sum_k |x||w| per output); M > 32 runs the tensor-core prefill on the
 * weights rounded to bf16 (round to nearest even) with fp32 accumulation
 * (within 8e-3 * sum_k |x||w|). Results are bitwise repeatable run to run.
 *
 * Errors: every entry point validates its arguments on the host and returns
 * a negative status without launching anything when they are wrong. Device
 * faults surface on the stream, as usual for CUDA.
 */
#ifndef HXQ_H
#define HXQ_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct hxq_linear* hxq_linear_t;
typedef struct hxq_group* hxq_group_t;

enum {
    HXQ_MODE_SCALAR8 = 0, /* 256 x fp32 codebook, one uint8 index per weight */
    HXQ_MODE_VQ2D12 = 1   /* 4096 x fp32-pair codebook, 12-bit index per pair */
};

enum {
    HXQ_OK = 0,
    HXQ_EINVAL = -1,       /* a bad argument; nothing was launched           */
    HXQ_ENOMEM = -2,       /* a device allocation failed                     */
    HXQ_ECUDA = -3,        /* a CUDA runtime or driver call failed           */
    HXQ_EUNSUPPORTED = -4, /* the current device is not an sm_100 GPU       */
    HXQ_ETIMEOUT = -5      /* a device-side wait gave up; see hxq_linear_check */
};

/* Kernel choice for hxq_linear_forward_ex. */
enum {
    HXQ_KERNEL_AUTO = 0,   /* CUDA-core GEMV for M <= 4, tensor cores above  */
    HXQ_KERNEL_GEMV = 1,   /* CUDA-core fused-decode GEMV, fp32 weights; M <= 8 
                              and the activations must fit in shared memory */
    HXQ_KERNEL_TC = 2      /* tcgen05 fused-decode GEMM; fp32-exact split
                              weights (hi+mid bf16) for M <= 32, bf16 weights
                              above                                          */
};

/*
 * Build a HelixLinear handle on the current CUDA device.
 *
 *  codebook     scalar: 256 floats; 2D: 8192 floats (4096 pairs)
 *  indices      scalar: N*K bytes; 2D: 3*N*K/4 bytes (layout above)
 *  mode         HXQ_MODE_SCALAR8 or HXQ_MODE_VQ2D12
 *  sidecar_pos  n_sidecar int64 flat positions n*K + k (may be NULL if 0)
 *  sidecar_val  n_sidecar float replacement values (may be NULL if 0)
 *  N, K         output and input features, N >= 1, K >= 1; 2D mode needs
 *               K % 4 == 0 (each row's 12-bit index stream is whole bytes)
 *  out          receives the handle
 *
 * Pointers may be device or host memory (copies use cudaMemcpyDefault).
 * The call copies everything it needs into memory it owns, re-lays the
 * indices out into 128-row tiles for coalesced loads (same information, rows
 * padded to whole 16- or 64-weight chunks), sorts the sidecar into per-row
 * patch lists, and synchronises the device before returning: the caller may
 * free its buffers afterwards. Device memory of a handle: the re-laid-out
 * indices, 12 bytes per sidecar entry plus the per-row and per-stage patch
 * offsets, the codebook, and a small split-K workspace of the CUDA-core
 * GEMV (2 x 8 x 128 floats per SM). The tensor-core kernels (M > 4) use a
 * workspace per device and stream instead (2 x 256 x 128 floats per SM,
 * 39 MB on a 148-SM B200), allocated by the first such forward issued on that
 * stream and kept until the process exits: make that first forward before
 * capturing the stream into a CUDA graph. When K % 8 != 0 the rows of x are
 * not 16-byte aligned for the tensor-core kernels' activation loads: such a
 * forward first copies x into rows of K rounded up to 8 in a buffer of that
 * stream (one more kernel launch; the buffer grows, after a synchronize of
 * the stream, when a forward needs more than it holds, so run the largest M
 * once before capturing). The handle is immutable; forwards
 * on ONE handle must not overlap in time on the GPU (different streams
 * racing on it give wrong results); forwards of different handles may run
 * concurrently on different streams.
 *
 * Returns HXQ_EINVAL for: NULL codebook/indices/out, NULL sidecar arrays with
 * n_sidecar > 0, n_sidecar < 0, > N*K or >= 2^31, N < 1, K < 1, 2D mode with
 * K % 4 != 0, unknown mode, a sidecar position outside [0, N*K) or repeated. HXQ_EUNSUPPORTED if
 * the current device is not compute capability 10.0. HXQ_ENOMEM / HXQ_ECUDA
 * on allocation / copy failures (nothing is leaked).
 */
int hxq_linear_create(const float* codebook, const uint8_t* indices, int mode,
                      const int64_t* sidecar_pos, const float* sidecar_val,
                      int64_t n_sidecar, int N, int K, hxq_linear_t* out);

/*
 * y[M][N] = x[M][K] . W^T on `stream` (a cudaStream_t; NULL = legacy default
 * stream). x (bf16 bits) and y (float) are device pointers; x must be 16-byte
 * aligned. Asynchronous: returns after the launch. M >= 1. The handle's
 * device must be the current one (as for every call that takes a handle).
 * Returns HXQ_EINVAL for a NULL handle/x/y, M < 1, a misaligned x or
 * another device current; HXQ_ENOMEM if the stream's tensor-core workspace
 * cannot be allocated (first forward with M > 4 on a stream); HXQ_ECUDA if a
 * launch fails.
 */
int hxq_linear_forward(hxq_linear_t h, const void* x_bf16, float* y, int M,
                       void* stream);

/*
 * hxq_linear_forward on host buffers, as one call on `stream`: x from host
 * memory x_host (bf16 bits [M][K]) into the caller's device buffer x_dev
 * (M*K bf16, 16-byte aligned), the forward, and y into host memory y_host
 * (M*N floats). Pinned host buffers are read and written by the kernels
 * themselves (a small copy kernel for x; the forward stores y straight into
 * y_host), which costs far less than copy-engine transfers of a few
 * kilobytes; pageable buffers go through cudaMemcpyAsync, y by way of the
 * caller's device buffer y_dev (M*N floats, unused otherwise). Asynchronous:
 * synchronise the stream before reading y_host. The x copy may read x_host
 * before earlier work on the stream has finished (it overlaps the previous
 * kernel), so x_host must hold its final contents when this call is made and
 * must not be a buffer that earlier work on the stream writes; the four
 * buffers must not overlap. Nothing is allocated beyond what
 * hxq_linear_forward allocates. Returns HXQ_EINVAL for a NULL argument,
 * M < 1, a misaligned x_dev or another device current; otherwise as
 * hxq_linear_forward (HXQ_ECUDA also for a failed copy).
 */
int hxq_linear_forward_host(hxq_linear_t h, const void* x_host, void* x_dev, float* y_dev,
                            float* y_host, int M, void* stream);

/*
 * hxq_linear_forward with an explicit kernel choice (HXQ_KERNEL_*) and split
 * count along K (0 = automatic, else 1..64), for tests and benchmarks. The
 * numerics of each kernel are those stated above for its M range.
 * HXQ_EINVAL additionally for an unknown kernel, split_k outside 0..64, or
 * HXQ_KERNEL_GEMV where it does not apply (M > 8, or M * K too large for its
 * shared-memory staging of x; HXQ_KERNEL_AUTO then picks the tensor cores).
 */
int hxq_linear_forward_ex(hxq_linear_t h, const void* x_bf16, float* y, int M,
                          int kernel, int split_k, void* stream);

/* Output element type for hxq_linear_forward_out. */
enum {
    HXQ_OUT_F32 = 0,       /* float                                          */
    HXQ_OUT_BF16 = 1       /* bfloat16 bits, rounded to nearest even         */
};

/*
 * The layer as a drop-in linear module: y[M][N] = x[M][K] . W^T + bias[N]
 * (HelixLinear replaces nn.Linear, Zamba2-1.2B-HXQ model card, "What is
 * HelixCode?"; the bias is kept uncompressed). `bias` is a device pointer
 * to N floats or NULL (no bias); `y` is a device pointer to M*N floats
 * (HXQ_OUT_F32) or M*N bf16 values (HXQ_OUT_BF16). The sum x . W^T + bias
 * is formed in fp32 with the numerics of hxq_linear_forward and, for
 * HXQ_OUT_BF16, rounded to bf16 (round to nearest even) as it is stored.
 * Kernel choice as hxq_linear_forward. Asynchronous on `stream`.
 * Returns HXQ_EINVAL for a NULL handle/x/y, M < 1, a misaligned x or an
 * unknown out_dtype; HXQ_ECUDA if a launch fails.
 */
int hxq_linear_forward_out(hxq_linear_t h, const void* x_bf16, const float* bias,
                           void* y, int out_dtype, int M, void* stream);

/* Most layers in one group (hxq_group_create). */
enum { HXQ_MAX_GROUP = 4 };

/*
 * A group of layers that read the same activations -- the query, key and
 * value projections of an attention block, the gate and up projections of an
 * MLP -- so that one launch runs them all. Every compressed weight tensor is
 * its own layer with its own codebook and sidecar (HXQ whitepaper, method
 * section: the pipeline runs independently on each tensor, "Per-tensor
 * k-means"); the pages' forward decompresses and multiplies one module at a
 * time and pays a fixed cost for each (HXQ whitepaper, the profiling
 * paragraph after the buffered forward path: 0.93 ms per module against
 * 0.39 ms for the matmul alone). At decode sizes a small projection (a key
 * or value projection of 256 x 2048 with 2 KV heads, Qwen2.5-3B-Instruct-HXQ
 * model card, "Compression Benchmark") reads half a megabyte, under 0.1 us
 * at full HBM bandwidth, against the microseconds a launch of its own takes
 * to start, stage its codebook and drain; in a group it shares one grid with
 * its neighbours.
 *
 *  layers    n_layers handles, 1 <= n_layers <= HXQ_MAX_GROUP, pairwise
 *            distinct, all of one mode and one K, created on one device
 *  out       receives the group
 *
 * The group refers to the handles without owning or copying them: they must
 * outlive it. Returns HXQ_EINVAL for a NULL array, handle or out, n_layers
 * outside 1..HXQ_MAX_GROUP, a repeated handle, mixed modes, mixed K or mixed
 * devices; HXQ_ENOMEM if the small host object cannot be allocated.
 */
int hxq_group_create(const hxq_linear_t* layers, int n_layers, hxq_group_t* out);

/*
 * For every layer i of the group: y[i] = x . W_i^T + bias[i], [M][N_i], with
 * the output types and numerics of hxq_linear_forward_out.
 *
 *  x       device pointer, bf16 [M][K], 16-byte aligned, read by all layers
 *  bias    host array of n_layers device pointers (N_i floats each, or NULL
 *          for none), or NULL for no bias on any layer
 *  y       host array of n_layers device pointers (M*N_i floats or bf16
 *          values, by out_dtype); the outputs must not overlap
 *
 * For M <= 4 (the CUDA-core GEMV) the layers run in one launch, each on a
 * share of the grid in proportion to its weights; above, each layer runs its
 * own kernel in turn on `stream`, as hxq_linear_forward_out would. A group
 * forward uses its layers' workspaces: it must not overlap in time on the GPU
 * with another forward of any of them. Asynchronous on `stream`.
 * Returns HXQ_EINVAL for a NULL group, x, y or y[i], M < 1, a misaligned x or
 * an unknown out_dtype; HXQ_ECUDA if a launch fails.
 */
int hxq_group_forward(hxq_group_t g, const void* x_bf16, const float* const* bias,
                      void* const* y, int out_dtype, int M, void* stream);

/* Free a group (NULL is ignored); its layers are untouched. */
void hxq_group_destroy(hxq_group_t g);

/*
 * ---- Encoder: the codec's other side (HXQ whitepaper, method section, the
 * per-tensor pipeline: "Per-tensor k-means", "Index assignment", "Sidecar
 * outlier correction", "12-bit index packing"). All pointers are device
 * pointers; every call is asynchronous on `stream` and writes only its
 * outputs (scratch comes from the stream-ordered allocator).
 *
 * Points are fp32 [n][dim]: dim 1 for scalar VQ (one weight per point, the
 * weight matrix read flat), dim 2 for 2D VQ (adjacent pairs (k, k+1), k
 * even, of a row: the row-major [N][K] weight matrix read as [N*K/2][2]).
 * Points and centroids must be finite. Distances are decided in fp32 with
 * each operation rounded (no fused multiply-add): |p - c| for dim 1,
 * dx*dx + dy*dy for dim 2; equal distances go to the lowest index.
 */

/*
 * Index assignment: labels[i] = index of the nearest of the k centroids
 * ([k][dim] fp32) to point i. 1 <= k <= 4096, 1 <= n < 2^31, dim 1 or 2.
 * Returns HXQ_EINVAL for NULL pointers or sizes out of range; HXQ_ECUDA if
 * a launch fails.
 */
int hxq_assign(const float* points, int64_t n, int dim, const float* centroids, int k,
               uint16_t* labels, void* stream);

/*
 * Per-tensor k-means: `iters` rounds of Lloyd's algorithm on the n points,
 * starting from the k centroids in `centroids` ([k][dim] fp32, overwritten
 * with the result). The pages name no initialisation and no stopping rule:
 * the caller supplies the start (for instance a seeded random sample of the
 * points) and the number of rounds. Each round assigns every point as
 * hxq_assign does and moves every centroid with points to their mean: the
 * exact sum of their fp32 coordinates over their count, rounded once to fp32
 * (nearest even); a centroid without points stays. The sums are exact
 * integers on a fixed-point grid as fine as the smallest nonzero |coordinate|
 * of the points, so every mean is correctly rounded whenever the nonzero
 * magnitudes span at most 2^38 (e.g. 1e-12 .. 0.1); beyond that span the
 * smallest coordinates are first rounded to that grid. Integer sums do not
 * depend on order: results are bitwise repeatable. labels (NULL allowed)
 * receives the assignment to the final centroids. iters >= 0; other limits
 * and errors as hxq_assign, plus HXQ_ENOMEM if scratch cannot be allocated.
 */
int hxq_kmeans(const float* points, int64_t n, int dim, int k, int iters, float* centroids,
               uint16_t* labels, void* stream);

/*
 * Encode a weight matrix W (fp32 [N][K], row-major) with a trained codebook
 * into what hxq_linear_create reads: `indices` in the layout above (scalar:
 * N*K bytes; 2D: 3*N*K/4 bytes) from the nearest entry of each weight or
 * pair, and the sidecar: every weight with |w - w_hat| > threshold (fp32,
 * strict), as flat position n*K + k (ascending) and the weight itself, which
 * replaces the decoded value. `codebook` holds 256 floats (scalar) or 4096
 * fp32 pairs (2D). *n_sidecar (device int64) receives the number of such
 * weights; only the first min(*n_sidecar, max_sidecar) are written, so a
 * caller that finds *n_sidecar > max_sidecar can retry with more room.
 * Shape limits as hxq_linear_create (K >= 1; 2D: K % 4 == 0), N*K < 2^31.
 * Returns HXQ_EINVAL for NULL W/codebook/indices/n_sidecar, NULL sidecar
 * arrays with max_sidecar > 0, max_sidecar < 0, a negative or NaN
 * threshold, an unknown mode or a bad shape; HXQ_ENOMEM / HXQ_ECUDA on
 * scratch or launch failures.
 */
int hxq_encode(const float* W, int mode, int N, int K, const float* codebook, float threshold,
               uint8_t* indices, int64_t* sidecar_pos, float* sidecar_val, int64_t max_sidecar,
               int64_t* n_sidecar, void* stream);

/*
 * Test helper: write the decoded fp32 weights W[N][K] (sidecar applied) to
 * the device buffer W_out on `stream`. Bit-exact with the definition above.
 * Returns HXQ_EINVAL for a NULL handle or W_out, HXQ_ECUDA on launch failure.
 */
int hxq_decode(hxq_linear_t h, float* W_out, void* stream);

/*
 * Synchronise the device and report whether any kernel of this handle gave up
 * a bounded device-side wait since the last check (HXQ_ETIMEOUT, then the
 * flag and the handle's split-tile arrival counters are cleared, so that
 * the next forward starts clean) -- the kernels bound every pipeline wait
 * at 2 s and return early instead of hanging. HXQ_OK otherwise, HXQ_EINVAL
 * for a NULL handle, HXQ_ECUDA if the device reports an error.
 */
int hxq_linear_check(hxq_linear_t h);

/*
 * Test hook, not for production use: the tensor-core forward (M >= 5) with
 * every pipeline wait bounded at wait_limit_us microseconds (1 .. 2e6) and
 * the activations of item `withhold_item` (>= 0) of each CTA's range never
 * requested, so that the MMA's wait for them runs out: the CTAs drain the
 * copies they issued, free their tensor memory and return, and the next
 * hxq_linear_check reports HXQ_ETIMEOUT. y is not written meaningfully.
 * Nothing faults or hangs: every wait is bounded and nothing is left in
 * flight. Returns HXQ_EINVAL for bad arguments, HXQ_ECUDA if a launch fails.
 */
int hxq_test_forward_withheld(hxq_linear_t h, const void* x_bf16, float* y, int M,
                              int withhold_item, unsigned wait_limit_us, void* stream);

/*
 * The CUDA-core GEMV (M <= 4) for callers that cannot call cudaMalloc at the
 * point where they run the layer: code under an allocation-free policy after
 * start-up (a real-time or latency-critical loop, where an allocation would
 * synchronise the device), or code that runs handles created elsewhere and
 * may not assume their workspace is free to use. The paper has no
 * counterpart: its layers allocate and share a materialisation buffer.
 *
 * Same arguments and result as hxq_linear_forward, computed by the same
 * kernel, but its scratch (per-tile arrival counters and the fp32 partial
 * sums of tiles split between CTAs) lives in one fixed array of 1 MiB + 16 KiB
 * compiled into this library, resident on every GPU that loads it until the
 * process exits; the call itself allocates nothing. hxq_linear_create looks
 * up that array's device address (cudaGetSymbolAddress) on its device, so
 * the no-alloc call only reads a cached pointer; the pointer is kept for the
 * life of the process and is not valid across cudaDeviceReset (create the
 * handles again after a reset). The CUDA runtime may still load the
 * kernel's code at its first launch in the process (lazy module loading);
 * callers that must not allocate at all can set CUDA_MODULE_LOADING=EAGER
 * or make one call during set-up. Each call clears the counters on `stream`
 * before the kernel runs. All calls share the one array, which keeps
 * the last call's contents: calls that overlap in time on the GPU (other
 * streams, other threads) race and give wrong results -- serialise them.
 *
 * Limits: 1 <= M <= 4, N <= 524288 (4096 tiles of 128 rows), the handle's
 * device current. Returns HXQ_EINVAL beyond them (nothing is launched), for
 * the argument errors of hxq_linear_forward, or when another device is
 * current; HXQ_ECUDA if the symbol lookup, the clear or the launch fails.
 */
int hxq_linear_forward_noalloc(hxq_linear_t h, const void* x_bf16, float* y, int M,
                               void* stream);

/* Shape of a handle: any output pointer may be NULL. HXQ_EINVAL if h is NULL. */
int hxq_linear_info(hxq_linear_t h, int* mode, int* N, int* K, int64_t* n_sidecar);

/* Free a handle (NULL is ignored). Synchronises the device first. */
void hxq_linear_destroy(hxq_linear_t h);

/* Static description of a status code. */
const char* hxq_strerror(int code);

#ifdef __cplusplus
}
#endif

#endif /* HXQ_H */
