/*
 * int8mm -- the LLM.int8() matrix multiplication Y = X W on NVIDIA B200 (sm_100a).
 *
 * Method: "LLM.int8(): 8-bit Matrix Multiplication for Transformers at Scale"
 * (Dettmers, Lewis, Belkada, Zettlemoyer, 2022), abstract: Int8 matmul for the
 * feed-forward and attention-projection layers of a transformer, as a
 * two-part procedure --
 *   1. vector-wise quantisation: one normalisation constant per row of X and
 *      one per output column of W (each inner product gets its own pair of
 *      constants);
 *   2. mixed-precision decomposition: the outlier feature dimensions of X go
 *      to a 16-bit matmul, everything else is multiplied in 8 bit.
 * Outliers are feature columns of the input batch (axolotl
 * "llama3-model-quantization", "Understanding Outliers in Transformer
 * Models"); quantisation normalises by the absolute maximum ("Key Points") and
 * rounds to the nearest level (scite report for nuQmm, which quotes LLM.int8()
 * as RTN); a 16- or 32-bit checkpoint is turned into int8 once, when it is
 * loaded (abstract) -- int8mm_prepare_weight.
 *
 * What one int8mm_forward computes (X: M x K, W: K x N, both fp16 row-major):
 *   (a) O = ascending list of columns k with |X[m,k]| >= threshold for any m;
 *   (b) ra[m] = max_{k not in O} |X[m,k]|,  Xq[m,k] = k in O ? 0 :
 *       round_half_even(X[m,k] * (127.0f / ra[m])) clamped to [-127, 127]
 *       (fp32 arithmetic, ra = 0 gives Xq = 0);
 *   (c) (at prepare time) ca[n] = max_k |W[k,n]| over all k and
 *       Wq[n,k] = round_half_even(W[k,n] * (127.0f / ca[n]));
 *   (d) Y[m,n] = fp16( sum_k Xq[m,k] Wq[n,k] * ra[m] * ca[n] / 127^2
 *                      + sum_{j} X[m,O[j]] * Wo[j,n] ),
 *       the first sum exact in int32, the second in fp32; Wo[j,:] is the fp16
 *       row W[O[j],:] when O[j] was kept at prepare time, else the dequantised
 *       row fp16(Wq[n,O[j]] * ca[n] / 127).
 *
 * Conventions for every call:
 *   - fp16 tensors are passed as pointers to IEEE binary16 bit patterns
 *     (uint16_t); all matrices are row-major and densely packed.
 *   - "device" pointers point to memory of the current CUDA device; the
 *     caller allocates and owns all memory.  The library calls no device
 *     allocator.  Between calls it keeps only a per-device cache of device
 *     properties on the host, the copy stream and events of
 *     int8mm_forward_host and, for int8mm_forward_decode_noalloc alone, the
 *     static scratch array described with that function.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Calls are stream-ordered and do not synchronise the host,
 *     except where a function says so.
 *   - Shape rules: M >= 1; K, N >= 16 and multiples of 16; K <= 131072
 *     (so that K * 127^2 fits int32); M, N < 2^31.
 *   - Alignment rules: X, W, Y 16-byte aligned; weight and workspace buffers
 *     256-byte aligned.
 *   - Argument errors are returned synchronously and leave every buffer
 *     untouched.  Errors found on the device (a wait that ran out, more
 *     outliers than the workspace holds) are recorded in the workspace and
 *     read back with int8mm_get_device_status.
 */
#ifndef INT8MM_H
#define INT8MM_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    INT8MM_OK = 0,
    INT8MM_ERR_INVALID_ARGUMENT = 1,   /* a shape, count or pointer breaks the rules above */
    INT8MM_ERR_MISALIGNED = 2,         /* a pointer breaks the alignment rules */
    INT8MM_ERR_WORKSPACE_TOO_SMALL = 3,/* buffer smaller than the matching *_bytes() */
    INT8MM_ERR_UNSUPPORTED_DEVICE = 4, /* current device is not compute capability 10.0 */
    INT8MM_ERR_CUDA = 5,               /* a CUDA runtime / driver call failed */
    INT8MM_ERR_TIMEOUT = 6,            /* (device) an in-kernel wait ran out; outputs invalid */
    INT8MM_ERR_OUTLIER_OVERFLOW = 7    /* (device) more outlier columns than max_outliers; outputs invalid */
} int8mm_status;

/* Human-readable name of a status code (static string, never NULL). */
const char* int8mm_status_string(int8mm_status s);

/* Library version as major * 10000 + minor * 100 + patch. */
int int8mm_version(void);

/* ------------------------------------------------------------------------ */
/* Prepared (int8) weight: the 16-bit checkpoint is converted to int8 once, at */
/* load, and then used as it is (LLM.int8() page, abstract).                  */
/* ------------------------------------------------------------------------ */

/* Views into one caller-owned device buffer, filled by int8mm_prepare_weight.
 * The buffer outlives every forward that uses the weight; W itself may be
 * freed once int8mm_prepare_weight returns. */
typedef struct {
    int32_t K, N, n_keep;
    int8_t* wq;          /* device, N x K int8: row n = output channel n, K contiguous */
    float* col_absmax;   /* device, N: ca[n] = max_k |W[k,n]| */
    uint16_t* w_keep;    /* device, n_keep x N fp16: row i = W[keep_idx[i], :] */
    int32_t* keep_idx;   /* device, n_keep, strictly ascending column indices */
    int32_t* keep_slot;  /* device, K: i if k == keep_idx[i], else -1 */
} int8mm_weight;

/* Bytes of the device buffer int8mm_prepare_weight needs. */
size_t int8mm_weight_bytes(int K, int N, int n_keep);

/* Convert W (device, K x N fp16) into the int8 weight.
 *   keep_idx_host: host array of n_keep strictly ascending feature indices in
 *     [0, K) whose fp16 rows W[k, :] are kept for the 16-bit outlier product
 *     (the feature dimensions expected to carry outliers; NULL iff n_keep == 0).
 *   buf / buf_bytes: device buffer of at least int8mm_weight_bytes(K, N, n_keep).
 *   out: host struct receiving the views into buf.
 * Synchronises `stream` before returning (it copies from host memory). */
int8mm_status int8mm_prepare_weight(const uint16_t* W, int K, int N, const int32_t* keep_idx_host,
                                    int n_keep, void* buf, size_t buf_bytes, int8mm_weight* out,
                                    void* stream);

/* ------------------------------------------------------------------------ */
/* Forward  Y = X W                                                           */
/* ------------------------------------------------------------------------ */

/* Bytes of device workspace a forward with these sizes needs.  max_outliers
 * (0 <= max_outliers <= K) bounds how many outlier columns one call may
 * detect; K is always safe. */
size_t int8mm_workspace_bytes(int M, int K, int N, int max_outliers);

/* Zero-fill a workspace (stream-ordered).  Needed once before its first
 * forward, and again after a forward that reported a device error; every
 * successful forward leaves the workspace ready for the next one. */
int8mm_status int8mm_workspace_init(void* ws, size_t ws_bytes, void* stream);

/* Y (device, M x N fp16) = the LLM.int8() product of X (device, M x K fp16)
 * and the prepared weight w, with outlier threshold `threshold` (> 0, may be
 * +inf to disable the decomposition).  ws is a zero-initialised workspace of
 * at least int8mm_workspace_bytes(M, w->K, w->N, max_outliers) bytes; it
 * must not be used by two forwards that overlap on the GPU. */
int8mm_status int8mm_forward(const uint16_t* X, int M, const int8mm_weight* w, float threshold,
                             int max_outliers, uint16_t* Y, void* ws, size_t ws_bytes,
                             void* stream);

enum {
    INT8MM_PATH_AUTO = 0,    /* decode kernel for M <= 16 when it fits (K <= 20480 and its
                                shared-memory plan), tiled GEMM otherwise */
    INT8MM_PATH_GEMM = 1,    /* detect -> quantise -> gather -> tcgen05 GEMM, any M (SM-pair
                                256 x 256 tiles when M > 128) */
    INT8MM_PATH_DECODE = 2,  /* single fused weight-streaming kernel (clusters of CTAs split K),
                                M <= 16, K <= 20480 and its shared-memory plan fits;
                                INT8MM_ERR_INVALID_ARGUMENT otherwise */
    INT8MM_PATH_GEMM_1SM = 3 /* the tiled path with single-SM 128 x 256 GEMM tiles (for tests) */
};

typedef struct {
    int path;                /* INT8MM_PATH_* */
    int32_t* acc_out;        /* optional device M x N int32: the exact int8 sums (for tests) */
    uint64_t wait_limit_ns;  /* bound on every in-kernel wait; 0 = 2 s */
    void* main_start_event;  /* optional cudaEvent_t recorded on `stream` just before the main
                                kernel (the tcgen05 GEMM or the fused decode kernel) ... */
    void* main_stop_event;   /* ... and just after it; both or neither (for timing). */
    uint32_t test_flags;     /* 0 in normal use.  INT8MM_TEST_WITHHOLD_SIGNAL: the main kernel never
                                sends one internal "data ready" signal, so the wait for it runs
                                out after wait_limit_ns and the call reports INT8MM_ERR_TIMEOUT
                                (exercises the timeout path without faulting the GPU). */
} int8mm_forward_opts;

enum { INT8MM_TEST_WITHHOLD_SIGNAL = 1 };

/* int8mm_forward with options (opts may be NULL = defaults). */
int8mm_status int8mm_forward_ex(const uint16_t* X, int M, const int8mm_weight* w, float threshold,
                                int max_outliers, uint16_t* Y, void* ws, size_t ws_bytes,
                                const int8mm_forward_opts* opts, void* stream);

/* int8mm_forward from and to host memory (same method, LLM.int8() abstract).
 *   x_host  HOST, M x K fp16, read by a host-to-device copy into x_dev;
 *   y_host  HOST, M x N fp16, written by device-to-host copies from y_dev;
 *   x_dev   DEVICE, M x K fp16 staging buffer (16-byte aligned), caller-owned;
 *   y_dev   DEVICE, M x N fp16 staging buffer (16-byte aligned), caller-owned;
 *   other arguments as for int8mm_forward.
 * Page-locked (pinned) host buffers let the copies run asynchronously; with
 * pageable ones the driver stages them and the call may block the host.
 * On the tiled path (M > 16) the product is computed in bands of whole
 * 256-row tiles (at most 8 bands) and each band's rows are copied back on a
 * second stream, owned by the library (one per device, created at the first
 * call on that device together with its events), while the next band is
 * computed; the decode path copies Y back after its one kernel.  All the
 * call's work is ordered on `stream`: once the stream has reached the end of
 * the call (e.g. cudaStreamSynchronize returns), y_host holds Y.  The host
 * buffers must not be changed or freed before that.  Device-side errors are
 * read with int8mm_get_device_status, as for int8mm_forward. */
int8mm_status int8mm_forward_host(const uint16_t* x_host, int M, const int8mm_weight* w, float threshold,
                                  int max_outliers, uint16_t* y_host, uint16_t* x_dev, uint16_t* y_dev,
                                  void* ws, size_t ws_bytes, void* stream);

/* Device pointers to the intermediates a forward leaves in its workspace. */
typedef struct {
    int32_t* status;       /* 1 word: bit 0 timeout, bit 1 outlier overflow */
    int32_t* n_outliers;   /* 1 word: number of outlier columns detected (may exceed capacity) */
    int32_t* outlier_idx;  /* K words: ascending outlier columns (first min(n, capacity) valid) */
    float* row_absmax;     /* M: ra */
    int8_t* xq;            /* M x K int8: Xq */
    uint16_t* xo;          /* M x kp fp16: X[:, O] (GEMM path only), zero-padded */
    int32_t kp;            /* row length of xo (max_outliers rounded up to 64) */
} int8mm_workspace_view;

int8mm_status int8mm_workspace_view_get(void* ws, size_t ws_bytes, int M, int K, int N,
                                        int max_outliers, int8mm_workspace_view* out);

/* Wait for `stream`, then report the device-side status of the last forward
 * that used ws: INT8MM_OK, INT8MM_ERR_TIMEOUT or INT8MM_ERR_OUTLIER_OVERFLOW.
 * If n_outliers is not NULL it receives the detected outlier count.
 * Synchronises the host with `stream`. */
int8mm_status int8mm_get_device_status(const void* ws, void* stream, int32_t* n_outliers);

/* ------------------------------------------------------------------------ */
/* Block-wise linear 8-bit codec (axolotl "llama3-model-quantization",      */
/* "8-Bit Optimizers": blocks normalised by their own maximum, an 8-bit     */
/* index per value).                                                         */
/* ------------------------------------------------------------------------ */

/* q (device, n int8) and absmax (device, ceil(n/B) fp32) of x (device, n
 * fp32, finite): block b covers [b*B, min(n, (b+1)*B)), absmax[b] = max |x|
 * over it, q = round_half_even(x * (127.0f / absmax[b])) (fp32 arithmetic;
 * absmax 0 gives 0).  B % 4 == 0, B >= 4; x 16-byte, q and absmax 4-byte
 * aligned. */
int8mm_status int8mm_block_quantize(const float* x, int64_t n, int B, int8_t* q, float* absmax, void* stream);

/* out (device, n fp32) = (q * absmax[block]) / 127 in fp32, the inverse of
 * int8mm_block_quantize up to half a quantisation step.  out 16-byte
 * aligned, q and absmax 4-byte aligned. */
int8mm_status int8mm_block_dequantize(const int8_t* q, const float* absmax, int64_t n, int B, float* out,
                                      void* stream);

/* ------------------------------------------------------------------------ */
/* Group-wise variant: one normalisation constant per row of X and group of */
/* G consecutive k, and per output column and group (the granularity of     */
/* nuQmm and ZeroQuant, finer than vector-wise: scite report for nuQmm,     */
/* citing snippets).  The outlier decomposition is unchanged.              */
/* ------------------------------------------------------------------------ */

/* As int8mm_weight, with col_absmax holding (K/G) x N constants:
 * col_absmax[g*N + n] = max |W[k,n]| over the group g of G consecutive k, and
 * Wq[n,k] quantised with the constant of its group. */
typedef struct {
    int32_t K, N, G, n_keep;
    int8_t* wq;          /* device, N x K int8 */
    float* col_absmax;   /* device, (K/G) x N */
    uint16_t* w_keep;    /* device, n_keep x N fp16 */
    int32_t* keep_idx;   /* device, n_keep */
    int32_t* keep_slot;  /* device, K */
} int8mm_grouped_weight;

/* Bytes of the weight buffer (0 when a rule is broken: the int8mm_weight
 * rules, plus G a multiple of 128 that divides K). */
size_t int8mm_grouped_weight_bytes(int K, int N, int G, int n_keep);

/* As int8mm_prepare_weight, with one constant per column and group. */
int8mm_status int8mm_prepare_weight_grouped(const uint16_t* W, int K, int N, int G, const int32_t* keep_idx_host,
                                            int n_keep, void* buf, size_t buf_bytes, int8mm_grouped_weight* out,
                                            void* stream);

/* Bytes of the workspace of a group-wise forward (its row constants are
 * M x K/G). */
size_t int8mm_grouped_workspace_bytes(int M, int K, int N, int G, int max_outliers);

/* Views into a group-wise workspace; row_absmax holds M x (K/G) constants,
 * row_absmax[m*(K/G) + g]. */
int8mm_status int8mm_grouped_workspace_view_get(void* ws, size_t ws_bytes, int M, int K, int N, int G,
                                                int max_outliers, int8mm_workspace_view* out);

/* Y = X W by the group-wise method, any M >= 1:
 *   ra[m,g] = max |X[m,k]| over the non-outlier k of group g, codes with the
 *   group's scale RN32(127/ra[m,g]) (half-even, outlier columns 0),
 *   acc_g = exact int32 sum over the group, and
 *   y = fp16( sum_g ((float(acc_g) * ra[m,g]) * ca[g,n]) / 16129  (fp32, ascending g)
 *             + sum_j X[m,O[j]] * Wo[j,n] ),
 * where a non-kept outlier row is dequantised with its own group's constant.
 * opts: path is ignored (SM-pair tcgen05 kernel); acc_out, if set, receives
 * the per-group int32 sums, M x N x (K/G), acc_out[(m*N + n)*(K/G) + g];
 * events, wait limit and test flags as for int8mm_forward_ex.  Device-side
 * errors are read with int8mm_get_device_status. */
int8mm_status int8mm_forward_grouped(const uint16_t* X, int M, const int8mm_grouped_weight* w, float threshold,
                                     int max_outliers, uint16_t* Y, void* ws, size_t ws_bytes,
                                     const int8mm_forward_opts* opts, void* stream);

/* ------------------------------------------------------------------------ */
/* 4-bit weight-only product for decode-sized X ("4-Bit Inference" on the   */
/* video page "8-bit Methods for Efficient Deep Learning with Tim Dettmers"; */
/* axolotl "llama3-model-quantization", "Impact of Precision and Parameter  */
/* Count on Model Efficiency": at small batch the weight bytes set the time). */
/* ------------------------------------------------------------------------ */

/* Views into one caller-owned device buffer, filled by
 * int8mm_prepare_weight_int4.  codes: N rows of K/2 bytes; every 32-bit word
 * holds 8 consecutive k of one output column as nibbles u = q + 8 (q in
 * [-7, 7]) in the order k0 -> bits 0-3, k0+1 -> 16-19, k0+2 -> 4-7,
 * k0+3 -> 20-23, k0+4 -> 8-11, k0+5 -> 24-27, k0+6 -> 12-15, k0+7 -> 28-31.
 * absmax: N x (K/G) fp32, absmax[n*(K/G) + g] = max |W[k,n]| over the group
 * g of G consecutive k. */
typedef struct {
    int32_t K, N, G;
    uint8_t* codes;      /* device, N x K/2 bytes */
    float* absmax;       /* device, N x K/G */
} int8mm_int4_weight;

/* Bytes of the buffer for a K x N weight with groups of G (0 when the shape
 * breaks the rules: K, N >= 16, K % 128 == 0, N % 16 == 0, G % 128 == 0,
 * G divides K, K <= 131072). */
size_t int8mm_int4_weight_bytes(int K, int N, int G);

/* Convert W (device, K x N fp16) to 4-bit codes once: per output column n and
 * group g, absmax = max |W[k,n]|, q = round_half_even(W[k,n] * (7.0f /
 * absmax)) (fp32) clamped to +-7, 0 when absmax is 0.  buf: 256-byte aligned
 * device buffer of int8mm_int4_weight_bytes(K, N, G) bytes.  Stream-ordered;
 * W must stay valid until the work on `stream` is done. */
int8mm_status int8mm_prepare_weight_int4(const uint16_t* W, int K, int N, int G, void* buf, size_t buf_bytes,
                                         int8mm_int4_weight* out, void* stream);

/* Y (device, M x N fp16) = X (device, M x K fp16) times the 4-bit weight,
 * 1 <= M <= 16:  y[m,n] = sum_k x[m,k] * (q[n,k] * absmax[n,g(k)] / 7), the
 * products on the tensor cores with fp32 sums, rounded to fp16 once.
 * The kernel keeps its share of X in shared memory, which bounds K: K <=
 * 73728 for M <= 8 and K <= 28672 for 9 <= M <= 16; longer K returns
 * INT8MM_ERR_INVALID_ARGUMENT.
 * status: device int32 word, zero before the call; a wait in the kernel that
 * runs out sets bit 0 (INT8MM_ERR_TIMEOUT: outputs invalid).  Stream-ordered
 * (programmatic dependent launch: the weight stream of a call starts while
 * the previous kernel on the stream finishes). */
int8mm_status int8mm_forward_int4(const uint16_t* X, int M, const int8mm_int4_weight* w, uint16_t* Y,
                                  int32_t* status, void* stream);

/* ------------------------------------------------------------------------ */
/* Decode-sized forward that allocates nothing                               */
/* ------------------------------------------------------------------------ */

/* The paper has no counterpart to this call; it exists for callers that
 * cannot allocate device memory: code that only receives input and output
 * buffers from a host framework which owns all device memory (a plugin
 * interface, say), and latency-critical paths where the cost and the
 * device-wide synchronisation of cudaMalloc are not acceptable.
 *
 * Same result as int8mm_forward on the fused decode kernel, but the scratch
 * memory (outlier list and count, status word, row absmax, int8 codes)
 * lives in one file-scope device array of INT8MM_NOALLOC_SCRATCH_BYTES
 * inside the library, which every GPU that loads the library holds until the
 * process exits.  The caller still passes X, the prepared weight and Y.
 *   Limits: 1 <= M <= 16, K <= 16384, N <= 65536.  Larger sizes return
 *   INT8MM_ERR_INVALID_ARGUMENT and touch nothing.
 *   max_outliers is K: every detected outlier column is handled.
 * It calls no cudaMalloc, cudaFree or other allocating routine.  The first
 * call on a device looks up the array's device address (once per device,
 * with that device current); make that first call before any stream
 * capture.  Each call clears the parts of the array that must start at zero
 * (stream-ordered memset) and then launches the kernel.  All calls share the
 * one array, which keeps the last call's contents: two calls that overlap on
 * the GPU (on different streams, or from different host threads) race and
 * give wrong results.  Device-side errors are read back with
 * int8mm_noalloc_device_status. */
#define INT8MM_NOALLOC_SCRATCH_BYTES (524288u)

int8mm_status int8mm_forward_decode_noalloc(const uint16_t* X, int M, const int8mm_weight* w,
                                            float threshold, uint16_t* Y, void* stream);

/* Wait for `stream`, then report the device-side status of the last
 * int8mm_forward_decode_noalloc on the current device (as
 * int8mm_get_device_status does for a workspace). */
int8mm_status int8mm_noalloc_device_status(void* stream, int32_t* n_outliers);

#ifdef __cplusplus
}
#endif

#endif /* INT8MM_H */
