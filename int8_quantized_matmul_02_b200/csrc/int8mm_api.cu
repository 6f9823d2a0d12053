// C-ABI of libint8mm: argument checks, buffer layouts, TMA descriptors and
// kernel launches for the LLM.int8() matmul ("LLM.int8(): 8-bit Matrix
// Multiplication for Transformers at Scale", abstract).  The declarations and
// their contracts are in include/int8mm.h.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <cmath>
#include <cstring>
#include <mutex>
#include <vector>

#include "int8mm.h"
#include "codec_kernels.cuh"
#include "decode_sm100.cuh"
#include "gemm2sm_sm100.cuh"
#include "gemm_grouped_sm100.cuh"
#include "gemm_sm100.cuh"
#include "int4_sm100.cuh"
#include "quant_kernels.cuh"

namespace {

using namespace i8mm;

constexpr int kVersion = 100;  // 0.1.0
constexpr uint64_t kDefaultWaitNs = 2000ull * 1000 * 1000;
constexpr int kMaxK = 131072;
constexpr int kMaxSmemOptin = 232448;  // 227 KB per block on sm_100
constexpr int kMaxDecodeRows = 16;

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }
inline bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }
inline int cdiv(long long a, long long b) { return (int)((a + b - 1) / b); }

// ------------------------------------------------------------------ device facts

struct DeviceInfo {
    int sm_count = 0;
    bool ok = false;
    bool attrs_set = false;
    int cluster_cap[9] = {};  // clusters of n CTAs that fit at once with one CTA per SM (0: not asked yet)
};
std::mutex g_dev_mu;
DeviceInfo g_dev[64];

int8mm_status current_device(int* dev_out, DeviceInfo** info_out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return INT8MM_ERR_CUDA;
    }
    if (dev < 0 || dev >= 64) return INT8MM_ERR_UNSUPPORTED_DEVICE;
    std::lock_guard<std::mutex> lk(g_dev_mu);
    DeviceInfo& d = g_dev[dev];
    if (!d.ok) {
        int major = 0, minor = 0, sms = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
            cudaGetLastError();
            return INT8MM_ERR_CUDA;
        }
        if (major != 10 || minor != 0) return INT8MM_ERR_UNSUPPORTED_DEVICE;
        d.sm_count = sms;
        d.ok = true;
    }
    if (!d.attrs_set) {
        if (cudaFuncSetAttribute(k_gemm_int8_sm100<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kGemmSmemBytes) != cudaSuccess ||
            cudaFuncSetAttribute(k_gemm_int8_sm100<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kGemmSmemBytes) != cudaSuccess ||
            cudaFuncSetAttribute(k_decode_int8_sm100<8, 8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kMaxSmemOptin) != cudaSuccess ||
            cudaFuncSetAttribute(k_decode_int8_sm100<16, 16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kMaxSmemOptin) != cudaSuccess ||
            cudaFuncSetAttribute(k_gemm_int8_grouped<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kGGSmemBytes) != cudaSuccess ||
            cudaFuncSetAttribute(k_gemm_int8_grouped<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kGGSmemBytes) != cudaSuccess ||
            cudaFuncSetAttribute(k_int4_decode_sm100, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kMaxSmemOptin) != cudaSuccess ||
            cudaFuncSetAttribute(k_gemm_int8_2sm<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kG2SmemBytes) != cudaSuccess ||
            cudaFuncSetAttribute(k_gemm_int8_2sm<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kG2SmemBytes) != cudaSuccess) {
            cudaGetLastError();
            return INT8MM_ERR_CUDA;
        }
        d.attrs_set = true;
    }
    *dev_out = dev;
    *info_out = &d;
    return INT8MM_OK;
}

// Clusters of `cl` CTAs (1..8) that the device runs at once when every CTA
// takes a whole SM: fewer than sm_count / cl when the GPCs' SM counts are not
// multiples of cl.  Asked once per device and size, with the largest
// shared-memory request (so one CTA per SM); sm_count / cl if the query fails.
std::mutex g_cap_mu;

int cluster_capacity(DeviceInfo* d, int cl) {
    if (cl <= 1) return d->sm_count;
    std::lock_guard<std::mutex> lk(g_cap_mu);
    if (d->cluster_cap[cl] == 0) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)(cl * 64));
        cfg.blockDim = dim3(384);
        cfg.dynamicSmemBytes = kMaxSmemOptin - 2048;
        cudaLaunchAttribute a[1];
        a[0].id = cudaLaunchAttributeClusterDimension;
        a[0].val.clusterDim.x = (unsigned)cl;
        a[0].val.clusterDim.y = 1;
        a[0].val.clusterDim.z = 1;
        cfg.attrs = a;
        cfg.numAttrs = 1;
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, k_decode_int8_sm100<8, 8>, &cfg) != cudaSuccess || n <= 0) {
            cudaGetLastError();
            n = std::max(1, d->sm_count / cl);
        }
        d->cluster_cap[cl] = n;
    }
    return d->cluster_cap[cl];
}

// ------------------------------------------------------------------ TMA descriptors

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static std::once_flag once;
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
        else
            cudaGetLastError();
    });
    return fn;
}

// Row-major 2-D tensor of `outer` rows x `inner` elements with a 128-byte
// swizzled box of box_outer rows x box_inner elements (box_inner * elem = 128).
bool make_map(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t inner, uint64_t outer,
              uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {inner, outer};
    cuuint64_t strides[1] = {row_bytes};
    cuuint32_t box[2] = {box_inner, box_outer};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// ------------------------------------------------------------------ layouts

struct WeightLayout {
    size_t wq, ca, w_keep, keep_idx, keep_slot, total;
};

WeightLayout weight_layout(int K, int N, int n_keep) {
    WeightLayout L{};
    size_t o = 0;
    L.wq = o;
    o = align_up(o + (size_t)N * K, 256);
    L.ca = o;
    o = align_up(o + (size_t)N * 4, 256);
    L.w_keep = o;
    o = align_up(o + (size_t)n_keep * N * 2, 256);
    L.keep_idx = o;
    o = align_up(o + (size_t)n_keep * 4, 256);
    L.keep_slot = o;
    o = align_up(o + (size_t)K * 4, 256);
    L.total = o;
    return L;
}

bool grouped_ok(int K, int G) { return G >= 128 && G % 128 == 0 && K % G == 0; }

// The group-wise weight: the vector-wise layout with (K/G) x N constants.
WeightLayout grouped_weight_layout(int K, int N, int G, int n_keep) {
    WeightLayout L{};
    size_t o = 0;
    L.wq = o;
    o = align_up(o + (size_t)N * K, 256);
    L.ca = o;
    o = align_up(o + (size_t)N * (K / G) * 4, 256);
    L.w_keep = o;
    o = align_up(o + (size_t)n_keep * N * 2, 256);
    L.keep_idx = o;
    o = align_up(o + (size_t)n_keep * 4, 256);
    L.keep_slot = o;
    o = align_up(o + (size_t)K * 4, 256);
    L.total = o;
    return L;
}

struct WsLayout {
    size_t status, n_out, ticket, part, mask, spre, idx, ra, xq, xo, wo, total;
    int kp;
};

// Grid of k_detect: gx blocks of 256 columns by gy row splits of `rows` rows
// (a multiple of 8), about kDetectBlocks blocks in all; a fixed budget (not
// the device's SM count) so that the workspace size depends on the shape only.
constexpr int kDetectBlocks = 592;
struct DetectGrid {
    int gx, gy, rows;
};
DetectGrid detect_grid(int M, int K) {
    DetectGrid d;
    d.gx = cdiv(K, 256);
    d.gy = std::max(1, std::min(cdiv(M, 8), cdiv(kDetectBlocks, d.gx)));
    d.rows = (cdiv(M, d.gy) + 7) / 8 * 8;
    d.gy = cdiv(M, d.rows);
    return d;
}

// ng: constants per row of X (1 vector-wise, K / G group-wise)
WsLayout ws_layout(int M, int K, int N, int max_outliers, int ng = 1) {
    WsLayout L{};
    L.kp = (max_outliers + 63) / 64 * 64;
    const size_t nw = (size_t)cdiv(K, 32);
    size_t o = 0;
    L.status = 0;
    L.n_out = 4;
    L.ticket = 8;
    o = 256;
    L.part = o;
    o = align_up(o + (size_t)detect_grid(M, K).gy * nw * 4, 256);
    L.mask = o;
    o = align_up(o + nw * 4, 256);
    L.spre = o;
    o = align_up(o + nw * 4, 256);
    L.idx = o;
    o = align_up(o + (size_t)K * 4, 256);
    L.ra = o;
    o = align_up(o + (size_t)M * ng * 4, 256);
    L.xq = o;
    o = align_up(o + (size_t)M * K, 256);
    L.xo = o;
    o = align_up(o + (size_t)M * L.kp * 2, 256);
    L.wo = o;
    o = align_up(o + (size_t)N * L.kp * 2, 256);
    L.total = o;
    return L;
}

// Outlier detection of the tiled paths (k_detect, finalised by its last block).
cudaError_t launch_detect(const uint16_t* X, int M, int K, float threshold, const WsLayout& L, uint8_t* b, int cap,
                          cudaStream_t s);

bool shape_ok(int M, int K, int N) {
    return M >= 1 && K >= 16 && N >= 16 && K % 16 == 0 && N % 16 == 0 && K <= kMaxK;
}

// Launch with optional programmatic dependent launch (PDL) and an optional
// thread-block cluster size along x (0: launched without a cluster).
template <typename Kern, typename... Args>
cudaError_t launch_ex(Kern kern, dim3 grid, dim3 block, size_t smem, cudaStream_t st, bool pdl, int cluster,
                      Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    int n = 0;
    if (pdl) {
        attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[n].val.programmaticStreamSerializationAllowed = 1;
        ++n;
    }
    if (cluster > 0) {
        attr[n].id = cudaLaunchAttributeClusterDimension;
        attr[n].val.clusterDim.x = (unsigned)cluster;
        attr[n].val.clusterDim.y = 1;
        attr[n].val.clusterDim.z = 1;
        ++n;
    }
    cfg.attrs = n ? attr : nullptr;
    cfg.numAttrs = n;
    return cudaLaunchKernelEx(&cfg, kern, args...);
}

template <typename Kern, typename... Args>
cudaError_t launch(Kern kern, dim3 grid, dim3 block, size_t smem, cudaStream_t st, bool pdl, Args... args) {
    return launch_ex(kern, grid, block, smem, st, pdl, 0, args...);
}

// Launched without PDL: its per-split words and ticket are reused from the
// previous call, whose kernels must have finished.
cudaError_t launch_detect(const uint16_t* X, int M, int K, float threshold, const WsLayout& L, uint8_t* b, int cap,
                          cudaStream_t s) {
    const DetectGrid d = detect_grid(M, K);
    return launch(k_detect, dim3(d.gx, d.gy), dim3(256), 0, s, false, X, M, K, threshold, d.rows,
                  reinterpret_cast<uint32_t*>(b + L.part), reinterpret_cast<uint32_t*>(b + L.mask),
                  reinterpret_cast<int32_t*>(b + L.spre), reinterpret_cast<int32_t*>(b + L.idx),
                  reinterpret_cast<int32_t*>(b + L.n_out), cap, reinterpret_cast<int*>(b + L.status),
                  reinterpret_cast<unsigned*>(b + L.ticket));
}

int8mm_status cuda_status(cudaError_t e) {
    if (e == cudaSuccess) return INT8MM_OK;
    cudaGetLastError();
    return INT8MM_ERR_CUDA;
}

// Value of a non-negative fp16 bit pattern h <= 0x7C00 (+inf).
float fp16_value(uint32_t h) {
    if (h == 0x7C00u) return INFINITY;
    const int e = (int)(h >> 10), m = (int)(h & 0x3FFu);
    return e == 0 ? std::ldexp((float)m, -24) : std::ldexp((float)(1024 + m), e - 25);
}

// Bits of the smallest fp16 value >= thr (thr > 0), replicated in both 16-bit
// lanes; 0x7C01 (above +inf, below any NaN after masking) when none reaches it.
// Non-negative fp16 bit patterns are ordered like their values, so a binary
// search over [0, 0x7C00] finds it.
uint32_t fp16_threshold_bits2(float thr) {
    if (!(fp16_value(0x7C00u) >= thr)) return 0x7C017C01u;
    uint32_t lo = 0, hi = 0x7C00u;  // fp16_value(hi) >= thr
    while (lo < hi) {
        const uint32_t mid = (lo + hi) / 2;
        if (fp16_value(mid) >= thr)
            hi = mid;
        else
            lo = mid + 1;
    }
    return lo | (lo << 16);
}

// Plan of the decode kernel: clusters of `cluster` CTAs split K (each CTA
// one K range of the cluster's `tiles` 128-channel tiles), a TMA ring of
// `stages` 16 KB boxes, and the shared-memory offsets.
struct DecodePlan {
    int cluster, tiles, stages, groups, grid, mr;  // mr: rows per chunk group (8 or 16)
    uint32_t off_xq, off_mask, off_pre, off_list, off_xo, off_oslot, off_red, off_bars, bytes;
};

// False when (M, K, cap) does not fit the kernel: M > 16, a CTA's K range
// wider than its X-side threads hold in registers, or shared memory.
bool decode_plan(int M, int K, int N, int cap, int sms, DecodePlan* P) {
    if (M < 1 || M > kMaxDecodeRows) return false;
    const int kbt = cdiv(K, 128);
    // a CTA's K range holds at most kDecPro 8-column chunks (kP * kDecPro / kR)
    int cl = 0;
    for (int c : {4, 8}) {
        const int cc = std::min(c, kbt);
        if (cdiv(kbt, cc) * 16 <= kDecPro) {
            cl = cc;
            break;
        }
    }
    if (cl == 0) return false;
    const int tiles = cdiv(N, kDecTileN);
    // fewest tiles per cluster that keep the grid within one wave
    int t = cl;
    for (int c = 1; c <= cl; ++c) {
        if ((long long)cl * cdiv(tiles, c) <= sms) {
            t = c;
            break;
        }
    }
    const int groups = (M + 7) / 8;
    const int nw = cdiv(K, 32);
    const size_t xq = (size_t)(cdiv(kbt, cl) * groups + 1) * 1024;
    const size_t mask = align_up((size_t)nw * 4, 16);
    const size_t pre = align_up((size_t)nw * 4, 16);
    const size_t list = align_up((size_t)std::min(K, std::max(cap, 1)) * 2, 16);
    const size_t xo = (size_t)kDecSmemOutliers * 16 * 2;
    const size_t oslot = (size_t)kDecSmemOutliers * 4;
    const size_t red = (size_t)cl * kDecTileN * 8 * groups * 4;  // one partial-sum slot per CTA of the cluster
    const size_t fixed = xq + mask + pre + list + xo + oslot + red;
    for (int s = 16; s >= 4; --s) {
        const size_t bars = (size_t)(2 * s + 5) * 8 + 256;
        const size_t total = 1024 + (size_t)s * kDecStageBytes + fixed + bars;
        if (total <= (size_t)kMaxSmemOptin) {
            P->cluster = cl;
            P->tiles = t;
            P->stages = s;
            P->groups = groups;
            P->grid = cl * cdiv(tiles, t);
            P->mr = M <= 8 ? 8 : 16;
            size_t o = (size_t)s * kDecStageBytes;
            P->off_xq = (uint32_t)o;
            o += xq;
            P->off_mask = (uint32_t)o;
            o += mask;
            P->off_pre = (uint32_t)o;
            o += pre;
            P->off_list = (uint32_t)o;
            o += list;
            P->off_xo = (uint32_t)o;
            o += xo;
            P->off_oslot = (uint32_t)o;
            o += oslot;
            P->off_red = (uint32_t)o;
            o += red;
            P->off_bars = (uint32_t)align_up(o, 8);
            P->bytes = (uint32_t)total;
            return true;
        }
    }
    return false;
}

// Parameters of one decode launch (the workspace pointers are the caller's).
DecodeParams decode_params(const uint16_t* X, int M, const int8mm_weight* w, float threshold, int cap, uint16_t* Y,
                           const DecodePlan& dp) {
    DecodeParams p{};
    p.X = X;
    p.M = M;
    p.K = w->K;
    p.N = w->N;
    p.thr_bits2 = fp16_threshold_bits2(threshold);
    p.cap = cap;
    p.wq = w->wq;
    p.ca = w->col_absmax;
    p.w_keep = w->w_keep;
    p.keep_slot = w->keep_slot;
    p.Y = Y;
    p.num_tiles = cdiv(w->N, kDecTileN);
    p.kb_total = cdiv(w->K, 128);
    p.cluster = dp.cluster;
    p.tiles_per_cluster = dp.tiles;
    p.stages = dp.stages;
    p.groups = dp.groups;
    p.off_xq = dp.off_xq;
    p.off_mask = dp.off_mask;
    p.off_pre = dp.off_pre;
    p.off_list = dp.off_list;
    p.off_xo = dp.off_xo;
    p.off_oslot = dp.off_oslot;
    p.off_red = dp.off_red;
    p.off_bars = dp.off_bars;
    return p;
}

cudaError_t launch_decode(const DecodePlan& dp, const CUtensorMap& tm_w, const DecodeParams& p, cudaStream_t s,
                          bool pdl) {
    if (dp.mr == 8)
        return launch_ex(k_decode_int8_sm100<8, 8>, dim3(dp.grid), dim3(kDecThreads), dp.bytes, s, pdl, dp.cluster, tm_w, p);
    return launch_ex(k_decode_int8_sm100<16, 16>, dim3(dp.grid), dim3(kDecThreads), dp.bytes, s, pdl, dp.cluster, tm_w, p);
}

// ------------------------------------------------------------------ 4-bit weight-only decode

constexpr int kInt4MaxRows = 16;

struct Int4Layout {
    size_t codes, absmax, total;
};

Int4Layout int4_layout(int K, int N, int G) {
    Int4Layout L{};
    L.codes = 0;
    size_t o = align_up((size_t)N * (K / 2), 256);
    L.absmax = o;
    o = align_up(o + (size_t)N * (K / G) * 4, 256);
    L.total = o;
    return L;
}

bool int4_shape_ok(int K, int N, int G) {
    return K >= 128 && N >= 16 && K % 128 == 0 && N % 16 == 0 && K <= kMaxK && G >= 128 && G % 128 == 0 && K % G == 0;
}

// Plan of the 4-bit kernel: clusters of `cluster` CTAs split K in 256-k
// boxes, tiles shared out evenly (at most `cluster` per cluster), one CTA per
// SM (the kernel takes the whole TMEM), one wave when the tiles allow.
struct Int4Plan {
    int cluster, clusters, stages, xrows, grid;
    uint32_t tmem_cols, off_x, off_red, off_bars, bytes;
};

bool int4_plan(int M, int K, int N, DeviceInfo* dev, Int4Plan* P) {
    if (M < 1 || M > kInt4MaxRows) return false;
    const int kbt = cdiv(K, kI4BoxK);
    const int tiles = cdiv(N, kI4TileN);
    const int xrows = M <= 8 ? 8 : 16;
    // one CTA per SM (the kernel takes the whole TMEM)
    for (size_t cap : {(size_t)kMaxSmemOptin}) {
        for (int c : {4, 8}) {
            const int cl = std::min(c, kbt);
            int ncl = std::max(1, std::min(tiles, cluster_capacity(dev, cl)));
            if (cdiv(tiles, ncl) > cl) ncl = cdiv(tiles, cl);
            const size_t xb = (size_t)cdiv(kbt, cl) * (kI4BoxK / 64) * xrows * 128 + 1024;  // + the row-8 overhang
            const size_t red = (size_t)cl * kI4TileN * xrows * 4;  // a slot per peer and one for its own sums
            for (int s = 12; s >= 3; --s) {
                const size_t bars = (size_t)(2 * s + 2 * kI4ASlots + 2 * kI4DSlots + 3) * 8 + 64;
                const size_t total = 1024 + (size_t)s * kI4StageBytes + xb + red + bars;
                if (total > cap) continue;
                P->cluster = cl;
                P->clusters = ncl;
                P->stages = s;
                P->xrows = xrows;
                P->grid = cl * ncl;
                P->tmem_cols = kI4TmemCols;
                size_t o = (size_t)s * kI4StageBytes;
                P->off_x = (uint32_t)o;
                o += xb;
                P->off_red = (uint32_t)o;
                o += red;
                P->off_bars = (uint32_t)align_up(o, 8);
                P->bytes = (uint32_t)total;
                return true;
            }
        }
    }
    return false;
}

// ------------------------------------------------------------------ no-allocation decode forward

// Scratch of int8mm_forward_decode_noalloc: one array per GPU that loads the
// library, zero at load, shared by every call of that entry point.
constexpr size_t kNoAllocBytes = INT8MM_NOALLOC_SCRATCH_BYTES;
constexpr int kNoAllocMaxK = 16384;
constexpr int kNoAllocMaxN = 65536;
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocBytes];

// Layout inside the array: [status, count] (the part cleared before every
// call), then the outlier list, ra and Xq.
struct NoAllocLayout {
    size_t clear_bytes, idx, ra, xq, total;
};

NoAllocLayout noalloc_layout(int M, int K) {
    NoAllocLayout L{};
    size_t o = 256;
    L.clear_bytes = o;
    L.idx = o;
    o = align_up(o + (size_t)K * 4, 256);
    L.ra = o;
    o = align_up(o + (size_t)kMaxDecodeRows * 4, 256);
    L.xq = o;
    o = align_up(o + (size_t)M * K, 256);
    L.total = o;
    return L;
}

// Device address of the array on the current device, looked up once per
// device (with that device current) by cudaGetSymbolAddress.
std::mutex g_noalloc_mu;
uint8_t* g_noalloc_ptr[64] = {};

int8mm_status noalloc_scratch(int dev, uint8_t** out) {
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
            cudaGetLastError();
            return INT8MM_ERR_CUDA;
        }
        g_noalloc_ptr[dev] = static_cast<uint8_t*>(p);
    }
    *out = g_noalloc_ptr[dev];
    return INT8MM_OK;
}

}  // namespace

// ====================================================================== C-ABI

extern "C" {

const char* int8mm_status_string(int8mm_status s) {
    switch (s) {
        case INT8MM_OK: return "INT8MM_OK";
        case INT8MM_ERR_INVALID_ARGUMENT: return "INT8MM_ERR_INVALID_ARGUMENT";
        case INT8MM_ERR_MISALIGNED: return "INT8MM_ERR_MISALIGNED";
        case INT8MM_ERR_WORKSPACE_TOO_SMALL: return "INT8MM_ERR_WORKSPACE_TOO_SMALL";
        case INT8MM_ERR_UNSUPPORTED_DEVICE: return "INT8MM_ERR_UNSUPPORTED_DEVICE";
        case INT8MM_ERR_CUDA: return "INT8MM_ERR_CUDA";
        case INT8MM_ERR_TIMEOUT: return "INT8MM_ERR_TIMEOUT";
        case INT8MM_ERR_OUTLIER_OVERFLOW: return "INT8MM_ERR_OUTLIER_OVERFLOW";
    }
    return "INT8MM_UNKNOWN_STATUS";
}

int int8mm_version(void) { return kVersion; }

size_t int8mm_weight_bytes(int K, int N, int n_keep) {
    if (!shape_ok(1, K, N) || n_keep < 0 || n_keep > K) return 0;
    return weight_layout(K, N, n_keep).total;
}

int8mm_status int8mm_prepare_weight(const uint16_t* W, int K, int N, const int32_t* keep_idx_host, int n_keep,
                                    void* buf, size_t buf_bytes, int8mm_weight* out, void* stream) {
    if (!W || !buf || !out || !shape_ok(1, K, N) || n_keep < 0 || n_keep > K || (n_keep > 0 && !keep_idx_host))
        return INT8MM_ERR_INVALID_ARGUMENT;
    for (int i = 0; i < n_keep; ++i) {
        const int k = keep_idx_host[i];
        if (k < 0 || k >= K || (i > 0 && k <= keep_idx_host[i - 1])) return INT8MM_ERR_INVALID_ARGUMENT;
    }
    if (!aligned(W, 16) || !aligned(buf, 256)) return INT8MM_ERR_MISALIGNED;
    const WeightLayout L = weight_layout(K, N, n_keep);
    if (buf_bytes < L.total) return INT8MM_ERR_WORKSPACE_TOO_SMALL;
    int dev;
    DeviceInfo* info;
    int8mm_status st = current_device(&dev, &info);
    if (st != INT8MM_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    uint8_t* b = static_cast<uint8_t*>(buf);

    int8mm_weight w{};
    w.K = K;
    w.N = N;
    w.n_keep = n_keep;
    w.wq = reinterpret_cast<int8_t*>(b + L.wq);
    w.col_absmax = reinterpret_cast<float*>(b + L.ca);
    w.w_keep = reinterpret_cast<uint16_t*>(b + L.w_keep);
    w.keep_idx = reinterpret_cast<int32_t*>(b + L.keep_idx);
    w.keep_slot = reinterpret_cast<int32_t*>(b + L.keep_slot);

    std::vector<int32_t> slot(K, -1);
    for (int i = 0; i < n_keep; ++i) slot[keep_idx_host[i]] = i;

    cudaError_t e = cudaMemsetAsync(w.col_absmax, 0, (size_t)N * 4, s);
    if (e == cudaSuccess) {
        const int ksplit = std::min(cdiv(K, 64), 128);
        const int rows = cdiv(K, ksplit);
        e = launch(k_col_absmax, dim3(cdiv(N, 2048), ksplit), dim3(256), 0, s, false, W, K, N, rows,
                   reinterpret_cast<unsigned*>(w.col_absmax));
    }
    if (e == cudaSuccess)
        e = launch(k_quant_weight, dim3(cdiv(N, 64), cdiv(K, 64)), dim3(256), 0, s, false, W, K, N, K,
                   (const float*)w.col_absmax, w.wq);
    if (e == cudaSuccess && n_keep > 0)
        e = cudaMemcpyAsync(w.keep_idx, keep_idx_host, (size_t)n_keep * 4, cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess) e = cudaMemcpyAsync(w.keep_slot, slot.data(), (size_t)K * 4, cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess && n_keep > 0)
        e = launch(k_copy_keep_rows, dim3(n_keep), dim3(256), 0, s, false, W, N, (const int32_t*)w.keep_idx,
                   w.w_keep);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);  // the host arrays above go out of scope
    if (e != cudaSuccess) return cuda_status(e);
    *out = w;
    return INT8MM_OK;
}

size_t int8mm_workspace_bytes(int M, int K, int N, int max_outliers) {
    if (!shape_ok(M, K, N) || max_outliers < 0 || max_outliers > K) return 0;
    return ws_layout(M, K, N, max_outliers).total;
}

int8mm_status int8mm_workspace_init(void* ws, size_t ws_bytes, void* stream) {
    if (!ws || ws_bytes == 0) return INT8MM_ERR_INVALID_ARGUMENT;
    if (!aligned(ws, 256)) return INT8MM_ERR_MISALIGNED;
    return cuda_status(cudaMemsetAsync(ws, 0, ws_bytes, reinterpret_cast<cudaStream_t>(stream)));
}

int8mm_status int8mm_workspace_view_get(void* ws, size_t ws_bytes, int M, int K, int N, int max_outliers,
                                        int8mm_workspace_view* out) {
    if (!ws || !out || !shape_ok(M, K, N) || max_outliers < 0 || max_outliers > K)
        return INT8MM_ERR_INVALID_ARGUMENT;
    const WsLayout L = ws_layout(M, K, N, max_outliers);
    if (ws_bytes < L.total) return INT8MM_ERR_WORKSPACE_TOO_SMALL;
    uint8_t* b = static_cast<uint8_t*>(ws);
    out->status = reinterpret_cast<int32_t*>(b + L.status);
    out->n_outliers = reinterpret_cast<int32_t*>(b + L.n_out);
    out->outlier_idx = reinterpret_cast<int32_t*>(b + L.idx);
    out->row_absmax = reinterpret_cast<float*>(b + L.ra);
    out->xq = reinterpret_cast<int8_t*>(b + L.xq);
    out->xo = reinterpret_cast<uint16_t*>(b + L.xo);
    out->kp = L.kp;
    return INT8MM_OK;
}

int8mm_status int8mm_get_device_status(const void* ws, void* stream, int32_t* n_outliers) {
    if (!ws) return INT8MM_ERR_INVALID_ARGUMENT;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    int32_t h[2] = {0, 0};
    cudaError_t e = cudaStreamSynchronize(s);
    if (e == cudaSuccess) e = cudaMemcpy(h, ws, sizeof(h), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_status(e);
    if (n_outliers) *n_outliers = h[1];
    if (h[0] & kStatusTimeout) return INT8MM_ERR_TIMEOUT;
    if (h[0] & kStatusOverflow) return INT8MM_ERR_OUTLIER_OVERFLOW;
    return INT8MM_OK;
}

}  // extern "C"

namespace {

// Per-device copy stream and events of int8mm_forward_host.
constexpr int kHostBands = 8;
struct HostPipe {
    bool ready = false;
    cudaStream_t copy = nullptr;
    cudaEvent_t band_done[kHostBands] = {};
    cudaEvent_t copies_done = nullptr;
};
std::mutex g_host_mu;
HostPipe g_host_pipe[64];

// Copy-back of Y to host memory in row bands (int8mm_forward_host): the tiled
// path runs its GEMM one band at a time and queues each band's copy on a
// second stream as soon as that band is written.
struct HostCopy {
    uint16_t* y_host;
    cudaStream_t copy;
    cudaEvent_t* band_done;  // one per band, recorded on the compute stream
    cudaEvent_t copies_done; // recorded on the copy stream after the last band
    int bands;
};

// The argument checks of a forward that need no options.
int8mm_status forward_check(const uint16_t* X, int M, const int8mm_weight* w, float threshold, int max_outliers,
                            const uint16_t* Y, const void* ws, size_t ws_bytes) {
    if (!X || !w || !Y || !ws || !w->wq || !w->col_absmax || !w->keep_slot) return INT8MM_ERR_INVALID_ARGUMENT;
    const int K = w->K, N = w->N;
    if (!shape_ok(M, K, N) || max_outliers < 0 || max_outliers > K) return INT8MM_ERR_INVALID_ARGUMENT;
    if (!(threshold > 0.0f)) return INT8MM_ERR_INVALID_ARGUMENT;  // also rejects NaN
    if (!aligned(X, 16) || !aligned(Y, 16) || !aligned(ws, 256) || !aligned(w->wq, 256))
        return INT8MM_ERR_MISALIGNED;
    if (ws_bytes < ws_layout(M, K, N, max_outliers).total) return INT8MM_ERR_WORKSPACE_TOO_SMALL;
    return INT8MM_OK;
}

int8mm_status forward_core(const uint16_t* X, int M, const int8mm_weight* w, float threshold, int max_outliers,
                           uint16_t* Y, void* ws, size_t ws_bytes, const int8mm_forward_opts* opts, void* stream,
                           const HostCopy* hc) {
    {
        const int8mm_status chk = forward_check(X, M, w, threshold, max_outliers, Y, ws, ws_bytes);
        if (chk != INT8MM_OK) return chk;
    }
    const int K = w->K, N = w->N;
    const int path = opts ? opts->path : INT8MM_PATH_AUTO;
    if (path < INT8MM_PATH_AUTO || path > INT8MM_PATH_GEMM_1SM) return INT8MM_ERR_INVALID_ARGUMENT;
    int32_t* acc_out = opts ? opts->acc_out : nullptr;
    cudaEvent_t ev0 = opts ? reinterpret_cast<cudaEvent_t>(opts->main_start_event) : nullptr;
    cudaEvent_t ev1 = opts ? reinterpret_cast<cudaEvent_t>(opts->main_stop_event) : nullptr;
    if ((ev0 == nullptr) != (ev1 == nullptr)) return INT8MM_ERR_INVALID_ARGUMENT;
    const bool timed = ev0 != nullptr;
    const uint32_t test_flags = opts ? opts->test_flags : 0u;
    const uint64_t wait_ns = (opts && opts->wait_limit_ns) ? opts->wait_limit_ns : kDefaultWaitNs;
    if (acc_out && !aligned(acc_out, 16)) return INT8MM_ERR_MISALIGNED;
    const WsLayout L = ws_layout(M, K, N, max_outliers);

    // whether the decode kernel fits does not depend on the device; its grid does
    DecodePlan dp{};
    const bool decode_fits = decode_plan(M, K, N, max_outliers, 1 << 20, &dp);
    bool use_decode;
    if (path == INT8MM_PATH_DECODE) {
        if (!decode_fits) return INT8MM_ERR_INVALID_ARGUMENT;
        use_decode = true;
    } else if (path == INT8MM_PATH_GEMM || path == INT8MM_PATH_GEMM_1SM) {
        use_decode = false;
    } else {
        use_decode = decode_fits;
    }
    int dev;
    DeviceInfo* info;
    int8mm_status st = current_device(&dev, &info);
    if (st != INT8MM_OK) return st;
    if (use_decode && !decode_plan(M, K, N, max_outliers, info->sm_count, &dp)) return INT8MM_ERR_INVALID_ARGUMENT;

    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    uint8_t* b = static_cast<uint8_t*>(ws);
    int* status = reinterpret_cast<int*>(b + L.status);
    int32_t* n_out = reinterpret_cast<int32_t*>(b + L.n_out);
    uint32_t* mask = reinterpret_cast<uint32_t*>(b + L.mask);
    int32_t* idx = reinterpret_cast<int32_t*>(b + L.idx);
    float* ra = reinterpret_cast<float*>(b + L.ra);
    int8_t* xq = reinterpret_cast<int8_t*>(b + L.xq);
    uint16_t* xo = reinterpret_cast<uint16_t*>(b + L.xo);
    uint16_t* wo = reinterpret_cast<uint16_t*>(b + L.wo);

    if (use_decode) {
        CUtensorMap tm_w;
        if (!make_map(&tm_w, CU_TENSOR_MAP_DATA_TYPE_UINT8, w->wq, K, N, K, 128, kDecTileN))
            return INT8MM_ERR_CUDA;
        DecodeParams p = decode_params(X, M, w, threshold, max_outliers, Y, dp);
        p.acc_out = acc_out;
        p.idx_out = idx;
        p.n_out = n_out;
        p.ra_out = ra;
        p.xq_out = xq;
        p.status = status;
        p.wait_limit_ns = wait_ns;
        p.test_flags = test_flags;
        cudaError_t e = timed ? cudaEventRecord(ev0, s) : cudaSuccess;
        if (e == cudaSuccess) e = launch_decode(dp, tm_w, p, s, !timed);
        if (e == cudaSuccess && timed) e = cudaEventRecord(ev1, s);
        if (e == cudaSuccess && hc)
            e = cudaMemcpyAsync(hc->y_host, Y, (size_t)M * N * 2, cudaMemcpyDeviceToHost, s);
        return cuda_status(e);
    }

    // ---- tiled path: detect -> quantise -> gather -> tcgen05 GEMM, PDL-chained
    CUtensorMap tm_b, tm_wo;
    const int kp = L.kp;
    if (!make_map(&tm_b, CU_TENSOR_MAP_DATA_TYPE_UINT8, w->wq, K, N, K, 128, kGemmBN)) return INT8MM_ERR_CUDA;
    if (kp > 0) {
        if (!make_map(&tm_wo, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, wo, kp, N, (uint64_t)kp * 2, 64, kGemmBN))
            return INT8MM_ERR_CUDA;
    } else {
        tm_wo = tm_b;  // never dereferenced: no outlier slices without capacity
    }

    const int sms = info->sm_count;
    cudaError_t e = launch_detect(X, M, K, threshold, L, b, max_outliers, s);
    if (e == cudaSuccess) {
        const int kc = cdiv(K / 8, 256);  // 8-column chunks per thread
        if (kc <= 8) {
            // one row per block, held in registers (X read once), with the
            // outlier weight rows gathered by extra blocks in front of the rows
            GatherArgs ga{(const int8_t*)w->wq, (const float*)w->col_absmax, (const uint16_t*)w->w_keep,
                          (const int32_t*)w->keep_slot, N, K, kp > 0 ? cdiv(N, 64) : 0, wo};
            auto kern = kc <= 2 ? k_quant_rows_reg<2> : kc <= 4 ? k_quant_rows_reg<4>
                      : kc <= 6 ? k_quant_rows_reg<6> : k_quant_rows_reg<8>;
            e = launch(kern, dim3(ga.blocks + M), dim3(256), 0, s, true, X, M, K, (const uint32_t*)mask,
                       (const int32_t*)n_out, max_outliers, kp, xq, ra, xo, (const int32_t*)idx, ga);
        } else {
            // mask words, their prefix counts, and one flag word per 2048-column window
            const size_t smem = ((size_t)cdiv(K, 32) * 2 + (size_t)cdiv(K, 2048)) * 4;
            const int grid = std::max(1, std::min(cdiv(M, 8), sms * 4));
            e = launch(k_quant_rows, dim3(grid), dim3(256), smem, s, true, X, M, K, (const uint32_t*)mask,
                       max_outliers, kp, xq, ra, xo);
            if (e == cudaSuccess && kp > 0)
                e = launch(k_gather_wo, dim3(cdiv(N, 64)), dim3(256), 0, s, true, (const int8_t*)w->wq,
                           (const float*)w->col_absmax, (const uint16_t*)w->w_keep, (const int32_t*)w->keep_slot,
                           K, N, K, (const int32_t*)idx, (const int32_t*)n_out, max_outliers, kp, wo);
        }
    }
    // the GEMM over rows [r0, r0 + rows) of Xq / Xo / Y
    auto gemm_rows = [&](int r0, int rows, bool first) -> cudaError_t {
        const bool pair = (path != INT8MM_PATH_GEMM_1SM) && rows > kGemmBM;
        CUtensorMap tm_a, tm_xo, tm_y;
        int8_t* xq_r = xq + (size_t)r0 * K;
        uint16_t* y_r = Y + (size_t)r0 * N;
        if (!make_map(&tm_a, CU_TENSOR_MAP_DATA_TYPE_UINT8, xq_r, K, rows, K, 128, kGemmBM) ||
            !make_map(&tm_y, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, y_r, N, rows, (uint64_t)N * 2, 64, 32))
            return cudaErrorInvalidValue;
        if (kp > 0) {
            if (!make_map(&tm_xo, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, xo + (size_t)r0 * kp, kp, rows, (uint64_t)kp * 2,
                          64, kGemmBM))
                return cudaErrorInvalidValue;
        } else {
            tm_xo = tm_a;
        }
        GemmParams p{};
        p.M = rows;
        p.N = N;
        p.K = K;
        p.num_m_blocks = cdiv(rows, pair ? kG2BM : kGemmBM);
        p.num_n_blocks = cdiv(N, pair ? kG2BN : kGemmBN);
        p.num_tiles = p.num_m_blocks * p.num_n_blocks;
        // Raster: a group of row blocks sweeps all column tiles before the next
        // group starts; the group's band of Xq (group x tile rows x K bytes)
        // stays in L2 while each W column tile is read once per group.  Use
        // the largest group whose band fits in 48 MB (at least 8 row blocks).
        {
            const uint64_t band = (uint64_t)(pair ? kG2BM : kGemmBM) * (uint64_t)K;
            const int fit = (int)std::min<uint64_t>(1u << 20, (48ull << 20) / band);
            p.group_m = std::min(std::max(8, fit), p.num_m_blocks);
        }
        p.kb_int8 = cdiv(K, 128);
        p.n_outliers = n_out;
        p.cap = max_outliers;
        p.ra = ra + r0;
        p.ca = w->col_absmax;
        p.acc_out = acc_out ? acc_out + (size_t)r0 * N : nullptr;
        p.status = status;
        p.wait_limit_ns = wait_ns;
        p.test_flags = test_flags;
        const bool pdl = !timed;
        cudaError_t le = cudaSuccess;
        if (pair) {
            // each CTA of the pair loads 128 rows of B / Wo per slice
            CUtensorMap tm_b2, tm_wo2;
            if (!make_map(&tm_b2, CU_TENSOR_MAP_DATA_TYPE_UINT8, w->wq, K, N, K, 128, 128))
                return cudaErrorInvalidValue;
            if (kp > 0) {
                if (!make_map(&tm_wo2, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, wo, kp, N, (uint64_t)kp * 2, 64, 128))
                    return cudaErrorInvalidValue;
            } else {
                tm_wo2 = tm_b2;
            }
            const int clusters = std::min(p.num_tiles, sms / 2);
            const int grid = 2 * clusters;
            if (timed && first) le = cudaEventRecord(ev0, s);
            if (le == cudaSuccess)
                le = acc_out ? launch_ex(k_gemm_int8_2sm<true>, dim3(grid), dim3(kGemmThreads), kG2SmemBytes, s, pdl,
                                         2, tm_a, tm_b2, tm_xo, tm_wo2, tm_y, p)
                             : launch_ex(k_gemm_int8_2sm<false>, dim3(grid), dim3(kGemmThreads), kG2SmemBytes, s,
                                         pdl, 2, tm_a, tm_b2, tm_xo, tm_wo2, tm_y, p);
        } else {
            const int grid = std::min(p.num_tiles, sms);
            if (timed && first) le = cudaEventRecord(ev0, s);
            if (le == cudaSuccess)
                le = acc_out ? launch(k_gemm_int8_sm100<true>, dim3(grid), dim3(kGemmThreads), kGemmSmemBytes, s,
                                      pdl, tm_a, tm_b, tm_xo, tm_wo, tm_y, p)
                             : launch(k_gemm_int8_sm100<false>, dim3(grid), dim3(kGemmThreads), kGemmSmemBytes, s,
                                      pdl, tm_a, tm_b, tm_xo, tm_wo, tm_y, p);
        }
        return le;
    };

    if (!hc) {
        if (e == cudaSuccess) e = gemm_rows(0, M, true);
        if (e == cudaSuccess && timed) e = cudaEventRecord(ev1, s);
        return cuda_status(e);
    }
    // host copy-back: bands of whole 256-row tiles; each band's copy waits for
    // that band's GEMM only, and the compute stream waits for the last copy
    const int band_rows = std::max(256, cdiv(cdiv(M, hc->bands), 256) * 256);
    for (int r0 = 0, i = 0; e == cudaSuccess && r0 < M; r0 += band_rows, ++i) {
        const int rows = std::min(band_rows, M - r0);
        e = gemm_rows(r0, rows, r0 == 0);
        if (e == cudaSuccess) e = cudaEventRecord(hc->band_done[i], s);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(hc->copy, hc->band_done[i], 0);
        if (e == cudaSuccess)
            e = cudaMemcpyAsync(hc->y_host + (size_t)r0 * N, Y + (size_t)r0 * N, (size_t)rows * N * 2,
                                cudaMemcpyDeviceToHost, hc->copy);
    }
    if (e == cudaSuccess && timed) e = cudaEventRecord(ev1, s);
    if (e == cudaSuccess) e = cudaEventRecord(hc->copies_done, hc->copy);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(s, hc->copies_done, 0);
    return cuda_status(e);
}

}  // namespace

extern "C" {

int8mm_status int8mm_forward_ex(const uint16_t* X, int M, const int8mm_weight* w, float threshold,
                                int max_outliers, uint16_t* Y, void* ws, size_t ws_bytes,
                                const int8mm_forward_opts* opts, void* stream) {
    return forward_core(X, M, w, threshold, max_outliers, Y, ws, ws_bytes, opts, stream, nullptr);
}

int8mm_status int8mm_forward_host(const uint16_t* x_host, int M, const int8mm_weight* w, float threshold,
                                  int max_outliers, uint16_t* y_host, uint16_t* x_dev, uint16_t* y_dev,
                                  void* ws, size_t ws_bytes, void* stream) {
    if (!x_host || !y_host || !x_dev || !y_dev || !w) return INT8MM_ERR_INVALID_ARGUMENT;
    const int K = w->K;
    // argument errors first, before the device is touched or anything is queued
    {
        const int8mm_status chk = forward_check(x_dev, M, w, threshold, max_outliers, y_dev, ws, ws_bytes);
        if (chk != INT8MM_OK) return chk;
    }
    int dev;
    DeviceInfo* info;
    int8mm_status st = current_device(&dev, &info);
    if (st != INT8MM_OK) return st;
    std::lock_guard<std::mutex> lk(g_host_mu);
    HostPipe& hp = g_host_pipe[dev];
    if (!hp.ready) {
        bool ok = cudaStreamCreateWithFlags(&hp.copy, cudaStreamNonBlocking) == cudaSuccess;
        for (int i = 0; ok && i < kHostBands; ++i)
            ok = cudaEventCreateWithFlags(&hp.band_done[i], cudaEventDisableTiming) == cudaSuccess;
        if (ok) ok = cudaEventCreateWithFlags(&hp.copies_done, cudaEventDisableTiming) == cudaSuccess;
        if (!ok) {
            cudaGetLastError();
            return INT8MM_ERR_CUDA;
        }
        hp.ready = true;
    }
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemcpyAsync(x_dev, x_host, (size_t)M * K * 2, cudaMemcpyHostToDevice, s);
    if (e != cudaSuccess) return cuda_status(e);
    HostCopy hc{y_host, hp.copy, hp.band_done, hp.copies_done, kHostBands};
    return forward_core(x_dev, M, w, threshold, max_outliers, y_dev, ws, ws_bytes, nullptr, stream, &hc);
}

int8mm_status int8mm_forward(const uint16_t* X, int M, const int8mm_weight* w, float threshold, int max_outliers,
                             uint16_t* Y, void* ws, size_t ws_bytes, void* stream) {
    return int8mm_forward_ex(X, M, w, threshold, max_outliers, Y, ws, ws_bytes, nullptr, stream);
}

int8mm_status int8mm_forward_decode_noalloc(const uint16_t* X, int M, const int8mm_weight* w, float threshold,
                                            uint16_t* Y, void* stream) {
    if (!X || !w || !Y || !w->wq || !w->col_absmax || !w->keep_slot) return INT8MM_ERR_INVALID_ARGUMENT;
    const int K = w->K, N = w->N;
    if (!shape_ok(M, K, N) || M > kMaxDecodeRows || K > kNoAllocMaxK || N > kNoAllocMaxN)
        return INT8MM_ERR_INVALID_ARGUMENT;
    if (!(threshold > 0.0f)) return INT8MM_ERR_INVALID_ARGUMENT;
    if (!aligned(X, 16) || !aligned(Y, 16) || !aligned(w->wq, 256)) return INT8MM_ERR_MISALIGNED;
    const int cap = K;
    const NoAllocLayout L = noalloc_layout(M, K);
    if (L.total > kNoAllocBytes) return INT8MM_ERR_INVALID_ARGUMENT;
    DecodePlan dp{};
    if (!decode_plan(M, K, N, cap, 1 << 20, &dp)) return INT8MM_ERR_INVALID_ARGUMENT;

    int dev;
    DeviceInfo* info;
    int8mm_status st = current_device(&dev, &info);
    if (st != INT8MM_OK) return st;
    if (!decode_plan(M, K, N, cap, info->sm_count, &dp)) return INT8MM_ERR_INVALID_ARGUMENT;
    uint8_t* b = nullptr;
    st = noalloc_scratch(dev, &b);
    if (st != INT8MM_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);

    CUtensorMap tm_w;
    if (!make_map(&tm_w, CU_TENSOR_MAP_DATA_TYPE_UINT8, w->wq, K, N, K, 128, kDecTileN)) return INT8MM_ERR_CUDA;
    DecodeParams p = decode_params(X, M, w, threshold, cap, Y, dp);
    p.acc_out = nullptr;
    p.idx_out = reinterpret_cast<int32_t*>(b + L.idx);
    p.n_out = reinterpret_cast<int32_t*>(b + 4);
    p.ra_out = reinterpret_cast<float*>(b + L.ra);
    p.xq_out = reinterpret_cast<int8_t*>(b + L.xq);
    p.status = reinterpret_cast<int*>(b);
    p.wait_limit_ns = kDefaultWaitNs;
    p.test_flags = 0;
    // the status word and the outlier count start at zero
    cudaError_t e = cudaMemsetAsync(b, 0, L.clear_bytes, s);
    if (e == cudaSuccess) e = launch_decode(dp, tm_w, p, s, false);
    return cuda_status(e);
}

int8mm_status int8mm_noalloc_device_status(void* stream, int32_t* n_outliers) {
    int dev;
    DeviceInfo* info;
    int8mm_status st = current_device(&dev, &info);
    if (st != INT8MM_OK) return st;
    uint8_t* b = nullptr;
    st = noalloc_scratch(dev, &b);
    if (st != INT8MM_OK) return st;
    return int8mm_get_device_status(b, stream, n_outliers);
}

int8mm_status int8mm_block_quantize(const float* x, int64_t n, int B, int8_t* q, float* absmax, void* stream) {
    if (!x || !q || !absmax || n < 1 || B < 4 || B % 4 != 0) return INT8MM_ERR_INVALID_ARGUMENT;
    if (!aligned(x, 16) || !aligned(q, 4) || !aligned(absmax, 4)) return INT8MM_ERR_MISALIGNED;
    int dev;
    DeviceInfo* info;
    int8mm_status st = current_device(&dev, &info);
    if (st != INT8MM_OK) return st;
    const long long nblocks = (n + B - 1) / B;
    const int grid = (int)std::max<long long>(1, std::min<long long>((nblocks + 7) / 8, (long long)info->sm_count * 16));
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const int kv = (B + 127) / 128;  // float4 chunks per lane for the whole block
    cudaError_t e;
    if (kv <= 1) e = launch(k_block_quant<1>, dim3(grid), dim3(256), 0, s, false, x, (long long)n, B, nblocks, q, absmax);
    else if (kv <= 2) e = launch(k_block_quant<2>, dim3(grid), dim3(256), 0, s, false, x, (long long)n, B, nblocks, q, absmax);
    else if (kv <= 4) e = launch(k_block_quant<4>, dim3(grid), dim3(256), 0, s, false, x, (long long)n, B, nblocks, q, absmax);
    else if (kv <= 8) e = launch(k_block_quant<8>, dim3(grid), dim3(256), 0, s, false, x, (long long)n, B, nblocks, q, absmax);
    else if (kv <= 16) e = launch(k_block_quant<16>, dim3(grid), dim3(256), 0, s, false, x, (long long)n, B, nblocks, q, absmax);
    else e = launch(k_block_quant<0>, dim3(grid), dim3(256), 0, s, false, x, (long long)n, B, nblocks, q, absmax);
    return cuda_status(e);
}

int8mm_status int8mm_block_dequantize(const int8_t* q, const float* absmax, int64_t n, int B, float* out,
                                      void* stream) {
    if (!q || !absmax || !out || n < 1 || B < 4 || B % 4 != 0) return INT8MM_ERR_INVALID_ARGUMENT;
    if (!aligned(q, 4) || !aligned(absmax, 4) || !aligned(out, 16)) return INT8MM_ERR_MISALIGNED;
    int dev;
    DeviceInfo* info;
    int8mm_status st = current_device(&dev, &info);
    if (st != INT8MM_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (B >= 256) {
        // a table of the block's 129 values per block, then look-ups
        const long long nblocks = (n + B - 1) / B;
        const int grid = (int)std::max<long long>(1, std::min<long long>(nblocks, (long long)info->sm_count * 8));
        return cuda_status(launch(k_block_dequant_table, dim3(grid), dim3(256), 0, s, false, q, absmax, (long long)n, B,
                                  out));
    }
    const long long nq = (n + 3) / 4;
    const int grid = (int)std::max<long long>(1, std::min<long long>((nq + 255) / 256, (long long)info->sm_count * 16));
    return cuda_status(launch(k_block_dequant, dim3(grid), dim3(256), 0, s, false, q, absmax, (long long)n, B, out));
}

size_t int8mm_int4_weight_bytes(int K, int N, int G) {
    if (!int4_shape_ok(K, N, G)) return 0;
    return int4_layout(K, N, G).total;
}

int8mm_status int8mm_prepare_weight_int4(const uint16_t* W, int K, int N, int G, void* buf, size_t buf_bytes,
                                         int8mm_int4_weight* out, void* stream) {
    if (!W || !buf || !out || !int4_shape_ok(K, N, G)) return INT8MM_ERR_INVALID_ARGUMENT;
    if (!aligned(W, 16) || !aligned(buf, 256)) return INT8MM_ERR_MISALIGNED;
    const Int4Layout L = int4_layout(K, N, G);
    if (buf_bytes < L.total) return INT8MM_ERR_WORKSPACE_TOO_SMALL;
    int dev;
    DeviceInfo* info;
    int8mm_status st = current_device(&dev, &info);
    if (st != INT8MM_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    uint8_t* b = static_cast<uint8_t*>(buf);
    int8mm_int4_weight w{};
    w.K = K;
    w.N = N;
    w.G = G;
    w.codes = b + L.codes;
    w.absmax = reinterpret_cast<float*>(b + L.absmax);
    const long long na = (long long)(K / G) * N, nc = (long long)(K / 8) * N;
    cudaError_t e = launch(k_int4_absmax, dim3((unsigned)cdiv(na, 256)), dim3(256), 0, s, false, W, K, N, G, w.absmax);
    if (e == cudaSuccess)
        e = launch(k_int4_pack, dim3((unsigned)cdiv(nc, 256)), dim3(256), 0, s, false, W, K, N, G,
                   (const float*)w.absmax, reinterpret_cast<uint32_t*>(w.codes));
    if (e != cudaSuccess) return cuda_status(e);
    *out = w;
    return INT8MM_OK;
}

int8mm_status int8mm_forward_int4(const uint16_t* X, int M, const int8mm_int4_weight* w, uint16_t* Y,
                                  int32_t* status, void* stream) {
    if (!X || !w || !Y || !status || !w->codes || !w->absmax) return INT8MM_ERR_INVALID_ARGUMENT;
    const int K = w->K, N = w->N;
    if (!int4_shape_ok(K, N, w->G) || M < 1 || M > kInt4MaxRows) return INT8MM_ERR_INVALID_ARGUMENT;
    if (!aligned(X, 16) || !aligned(Y, 16) || !aligned(w->codes, 256) || !aligned(status, 4))
        return INT8MM_ERR_MISALIGNED;
    int dev;
    DeviceInfo* info;
    int8mm_status st = current_device(&dev, &info);
    if (st != INT8MM_OK) return st;
    Int4Plan pl{};
    if (!int4_plan(M, K, N, info, &pl)) return INT8MM_ERR_INVALID_ARGUMENT;
    CUtensorMap tm_w, tm_x;
    if (!make_map(&tm_w, CU_TENSOR_MAP_DATA_TYPE_UINT8, w->codes, (uint64_t)K / 2, N, (uint64_t)K / 2, 128, kI4TileN) ||
        !make_map(&tm_x, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, X, K, M, (uint64_t)K * 2, 64, pl.xrows))
        return INT8MM_ERR_CUDA;
    Int4Params p{};
    p.absmax = w->absmax;
    p.Y = Y;
    p.status = status;
    p.wait_limit_ns = kDefaultWaitNs;
    p.test_flags = 0;
    p.M = M;
    p.K = K;
    p.N = N;
    p.G = w->G;
    p.num_tiles = cdiv(N, kI4TileN);
    p.kb_total = cdiv(K, kI4BoxK);
    p.num_clusters = pl.clusters;
    p.cluster = pl.cluster;
    p.stages = pl.stages;
    p.xrows = pl.xrows;
    p.tmem_cols = pl.tmem_cols;
    p.off_x = pl.off_x;
    p.off_red = pl.off_red;
    p.off_bars = pl.off_bars;
    return cuda_status(launch_ex(k_int4_decode_sm100, dim3(pl.grid), dim3(kI4Threads), pl.bytes,
                                 reinterpret_cast<cudaStream_t>(stream), true, pl.cluster, tm_w, tm_x, p));
}

size_t int8mm_grouped_weight_bytes(int K, int N, int G, int n_keep) {
    if (!shape_ok(1, K, N) || !grouped_ok(K, G) || n_keep < 0 || n_keep > K) return 0;
    return grouped_weight_layout(K, N, G, n_keep).total;
}

int8mm_status int8mm_prepare_weight_grouped(const uint16_t* W, int K, int N, int G, const int32_t* keep_idx_host,
                                            int n_keep, void* buf, size_t buf_bytes, int8mm_grouped_weight* out,
                                            void* stream) {
    if (!W || !buf || !out || !shape_ok(1, K, N) || !grouped_ok(K, G) || n_keep < 0 || n_keep > K ||
        (n_keep > 0 && !keep_idx_host))
        return INT8MM_ERR_INVALID_ARGUMENT;
    for (int i = 0; i < n_keep; ++i) {
        const int k = keep_idx_host[i];
        if (k < 0 || k >= K || (i > 0 && k <= keep_idx_host[i - 1])) return INT8MM_ERR_INVALID_ARGUMENT;
    }
    if (!aligned(W, 16) || !aligned(buf, 256)) return INT8MM_ERR_MISALIGNED;
    const WeightLayout L = grouped_weight_layout(K, N, G, n_keep);
    if (buf_bytes < L.total) return INT8MM_ERR_WORKSPACE_TOO_SMALL;
    int dev;
    DeviceInfo* info;
    int8mm_status st = current_device(&dev, &info);
    if (st != INT8MM_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    uint8_t* b = static_cast<uint8_t*>(buf);
    int8mm_grouped_weight w{};
    w.K = K;
    w.N = N;
    w.G = G;
    w.n_keep = n_keep;
    w.wq = reinterpret_cast<int8_t*>(b + L.wq);
    w.col_absmax = reinterpret_cast<float*>(b + L.ca);
    w.w_keep = reinterpret_cast<uint16_t*>(b + L.w_keep);
    w.keep_idx = reinterpret_cast<int32_t*>(b + L.keep_idx);
    w.keep_slot = reinterpret_cast<int32_t*>(b + L.keep_slot);
    std::vector<int32_t> slot(K, -1);
    for (int i = 0; i < n_keep; ++i) slot[keep_idx_host[i]] = i;
    cudaError_t e = launch(k_col_absmax_grouped, dim3(cdiv(N, 2048), K / G), dim3(256), 0, s, false, W, K, N, G,
                           w.col_absmax);
    if (e == cudaSuccess)
        e = launch(k_quant_weight, dim3(cdiv(N, 64), cdiv(K, 64)), dim3(256), 0, s, false, W, K, N, G,
                   (const float*)w.col_absmax, w.wq);
    if (e == cudaSuccess && n_keep > 0)
        e = cudaMemcpyAsync(w.keep_idx, keep_idx_host, (size_t)n_keep * 4, cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess) e = cudaMemcpyAsync(w.keep_slot, slot.data(), (size_t)K * 4, cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess && n_keep > 0)
        e = launch(k_copy_keep_rows, dim3(n_keep), dim3(256), 0, s, false, W, N, (const int32_t*)w.keep_idx,
                   w.w_keep);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);  // the host arrays above go out of scope
    if (e != cudaSuccess) return cuda_status(e);
    *out = w;
    return INT8MM_OK;
}

size_t int8mm_grouped_workspace_bytes(int M, int K, int N, int G, int max_outliers) {
    if (!shape_ok(M, K, N) || !grouped_ok(K, G) || max_outliers < 0 || max_outliers > K) return 0;
    return ws_layout(M, K, N, max_outliers, K / G).total;
}

int8mm_status int8mm_grouped_workspace_view_get(void* ws, size_t ws_bytes, int M, int K, int N, int G,
                                                int max_outliers, int8mm_workspace_view* out) {
    if (!ws || !out || !shape_ok(M, K, N) || !grouped_ok(K, G) || max_outliers < 0 || max_outliers > K)
        return INT8MM_ERR_INVALID_ARGUMENT;
    const WsLayout L = ws_layout(M, K, N, max_outliers, K / G);
    if (ws_bytes < L.total) return INT8MM_ERR_WORKSPACE_TOO_SMALL;
    uint8_t* b = static_cast<uint8_t*>(ws);
    out->status = reinterpret_cast<int32_t*>(b + L.status);
    out->n_outliers = reinterpret_cast<int32_t*>(b + L.n_out);
    out->outlier_idx = reinterpret_cast<int32_t*>(b + L.idx);
    out->row_absmax = reinterpret_cast<float*>(b + L.ra);
    out->xq = reinterpret_cast<int8_t*>(b + L.xq);
    out->xo = reinterpret_cast<uint16_t*>(b + L.xo);
    out->kp = L.kp;
    return INT8MM_OK;
}

int8mm_status int8mm_forward_grouped(const uint16_t* X, int M, const int8mm_grouped_weight* w, float threshold,
                                     int max_outliers, uint16_t* Y, void* ws, size_t ws_bytes,
                                     const int8mm_forward_opts* opts, void* stream) {
    if (!X || !w || !Y || !ws || !w->wq || !w->col_absmax || !w->keep_slot) return INT8MM_ERR_INVALID_ARGUMENT;
    const int K = w->K, N = w->N, G = w->G;
    if (!shape_ok(M, K, N) || !grouped_ok(K, G) || max_outliers < 0 || max_outliers > K)
        return INT8MM_ERR_INVALID_ARGUMENT;
    if (!(threshold > 0.0f)) return INT8MM_ERR_INVALID_ARGUMENT;
    int32_t* acc_out = opts ? opts->acc_out : nullptr;
    cudaEvent_t ev0 = opts ? reinterpret_cast<cudaEvent_t>(opts->main_start_event) : nullptr;
    cudaEvent_t ev1 = opts ? reinterpret_cast<cudaEvent_t>(opts->main_stop_event) : nullptr;
    if ((ev0 == nullptr) != (ev1 == nullptr)) return INT8MM_ERR_INVALID_ARGUMENT;
    const bool timed = ev0 != nullptr;
    const uint32_t test_flags = opts ? opts->test_flags : 0u;
    const uint64_t wait_ns = (opts && opts->wait_limit_ns) ? opts->wait_limit_ns : kDefaultWaitNs;
    if (!aligned(X, 16) || !aligned(Y, 16) || !aligned(ws, 256) || !aligned(w->wq, 256) ||
        (acc_out && !aligned(acc_out, 16)))
        return INT8MM_ERR_MISALIGNED;
    const int ng = K / G;
    const WsLayout L = ws_layout(M, K, N, max_outliers, ng);
    if (ws_bytes < L.total) return INT8MM_ERR_WORKSPACE_TOO_SMALL;
    int dev;
    DeviceInfo* info;
    int8mm_status st = current_device(&dev, &info);
    if (st != INT8MM_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    uint8_t* b = static_cast<uint8_t*>(ws);
    int* status = reinterpret_cast<int*>(b + L.status);
    int32_t* n_out = reinterpret_cast<int32_t*>(b + L.n_out);
    uint32_t* mask = reinterpret_cast<uint32_t*>(b + L.mask);
    int32_t* idx = reinterpret_cast<int32_t*>(b + L.idx);
    float* ra = reinterpret_cast<float*>(b + L.ra);
    int8_t* xq = reinterpret_cast<int8_t*>(b + L.xq);
    uint16_t* xo = reinterpret_cast<uint16_t*>(b + L.xo);
    uint16_t* wo = reinterpret_cast<uint16_t*>(b + L.wo);
    const int kp = L.kp;

    CUtensorMap tm_a, tm_b, tm_xo, tm_wo, tm_y;
    if (!make_map(&tm_a, CU_TENSOR_MAP_DATA_TYPE_UINT8, xq, K, M, K, 128, 128) ||
        !make_map(&tm_b, CU_TENSOR_MAP_DATA_TYPE_UINT8, w->wq, K, N, K, 128, 64) ||
        !make_map(&tm_y, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, Y, N, M, (uint64_t)N * 2, 64, 32))
        return INT8MM_ERR_CUDA;
    if (kp > 0) {
        if (!make_map(&tm_xo, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, xo, kp, M, (uint64_t)kp * 2, 64, 128) ||
            !make_map(&tm_wo, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, wo, kp, N, (uint64_t)kp * 2, 64, 64))
            return INT8MM_ERR_CUDA;
    } else {
        tm_xo = tm_a;  // never dereferenced: no outlier slices without capacity
        tm_wo = tm_b;
    }
    const int sms = info->sm_count;
    cudaError_t e = launch_detect(X, M, K, threshold, L, b, max_outliers, s);
    if (e == cudaSuccess) {
        const size_t smem = (size_t)cdiv(K, 32) * 2 * 4;
        const long long items = (long long)M * ng;
        const int grid = (int)std::max<long long>(1, std::min<long long>(cdiv(items, 8), (long long)sms * 4));
        e = launch(k_quant_rows_grouped, dim3(grid), dim3(256), smem, s, true, X, M, K, G, (const uint32_t*)mask,
                   max_outliers, kp, xq, ra, xo);
    }
    if (e == cudaSuccess && kp > 0)
        e = launch(k_gather_wo, dim3(cdiv(N, 64)), dim3(256), 0, s, true, (const int8_t*)w->wq,
                   (const float*)w->col_absmax, (const uint16_t*)w->w_keep, (const int32_t*)w->keep_slot, K, N, G,
                   (const int32_t*)idx, (const int32_t*)n_out, max_outliers, kp, wo);
    if (e == cudaSuccess) {
        GroupedParams gp{};
        GemmParams& p = gp.g;
        p.M = M;
        p.N = N;
        p.K = K;
        p.num_m_blocks = cdiv(M, kGGBM);
        p.num_n_blocks = cdiv(N, kGGBN);
        p.num_tiles = p.num_m_blocks * p.num_n_blocks;
        {
            const uint64_t band = (uint64_t)kGGBM * (uint64_t)K;
            const int fit = (int)std::min<uint64_t>(1u << 20, (48ull << 20) / band);
            p.group_m = std::min(std::max(8, fit), p.num_m_blocks);
        }
        p.kb_int8 = K / 128;
        p.n_outliers = n_out;
        p.cap = max_outliers;
        p.status = status;
        p.wait_limit_ns = wait_ns;
        p.test_flags = test_flags;
        gp.G = G;
        gp.ng = ng;
        gp.ra = ra;
        gp.ca = w->col_absmax;
        gp.acc_out = acc_out;
        const int clusters = std::min(p.num_tiles, sms / 2);
        if (timed) e = cudaEventRecord(ev0, s);
        if (e == cudaSuccess)
            e = acc_out ? launch_ex(k_gemm_int8_grouped<true>, dim3(2 * clusters), dim3(kGGThreads), kGGSmemBytes, s,
                                    !timed, 2, tm_a, tm_b, tm_xo, tm_wo, tm_y, gp)
                        : launch_ex(k_gemm_int8_grouped<false>, dim3(2 * clusters), dim3(kGGThreads), kGGSmemBytes, s,
                                    !timed, 2, tm_a, tm_b, tm_xo, tm_wo, tm_y, gp);
        if (e == cudaSuccess && timed) e = cudaEventRecord(ev1, s);
    }
    return cuda_status(e);
}

}  // extern "C"
