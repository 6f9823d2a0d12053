// Decode-shaped LLM.int8() forward (M <= 16 rows of X) in one kernel.
//
// At small M the product is bound by reading the int8 weight once ("memory
// loading is significantly more costly than computation", axolotl
// "llama3-model-quantization", "Impact of Precision and Parameter Count on
// Model Efficiency").  Each CTA owns one 128-channel tile of W (split along K
// only when there are too few tiles to occupy the GPU) and streams it through
// a deep TMA ring from the moment it starts, while it redoes the cheap X-side
// steps itself:
//   warps 2-11: outlier columns of X (a) and the row absmax in one pass over X
//     (the M rows of an 8-column chunk are loaded together, so the chunk's
//     flags are final at once), then the int8 codes (b) of the CTA's K range,
//     written straight into shared memory in the tensor-core operand layout
//     (128-byte rows, 128-byte swizzle, 8-row groups);
//   warp 0: TMA producer of 128 (channels) x 128 (K) int8 weight tiles;
//   warp 1: tcgen05.mma kind::i8 with the weight as the 128-row A operand and
//     the (padded) activation rows as the 16-column B operand ("swap AB"),
//     s32 accumulator in TMEM;
//   warps 4-7: the fp16 outlier product (d) while the weights stream, then the
//     accumulator: Y = fp16(acc * ra * ca / 127^2 + o).  With a K split the
//     int32 partial sums meet in a workspace buffer (exact in any order) and
//     the CTA that completes a tile's K range writes Y, leaving the partial
//     sums and counters at zero for the next call.
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "quant_kernels.cuh"
#include "sm100_ptx.cuh"

namespace i8mm {

struct DecodeParams {
    const uint16_t* X;
    int M, K, N;
    float thr;
    uint32_t thr_bits2;         // smallest fp16 >= thr, in both 16-bit lanes
    int cap;                    // outlier capacity (list + overflow flag)
    const int8_t* wq;           // N x K (dequantised outlier rows that were not kept)
    const float* ca;
    const uint16_t* w_keep;
    const int32_t* keep_slot;
    uint16_t* Y;
    int32_t* partial;           // 16 x N int32, zero on entry and on exit (K split only)
    int32_t* counters;          // 4 per tile (one per 32-column quadrant), zero on entry and on exit
    int32_t* acc_out;           // optional M x N
    int32_t* idx_out;           // workspace: outlier list
    int32_t* n_out;             // workspace: outlier count
    float* ra_out;              // workspace: M
    int8_t* xq_out;             // workspace: M x K
    int* status;
    uint64_t wait_limit_ns;
    uint32_t test_flags;        // bit 0: never signal that Xq is ready (timeout test)
    int num_tiles, kb_per_tile, splits, stages, groups;  // groups = ceil(M / 8)
    uint32_t off_xq, off_mask, off_pre, off_list, off_xo, off_oslot, off_bars;  // shared-memory offsets
    uint32_t off_xstage;        // this CTA's quarter of X staged in shared memory (cluster path)
    int cluster;                // CTAs per cluster sharing the X-side work (1 = each CTA alone)
};

constexpr int kDecThreads = 384;             // warp 0 TMA, warp 1 MMA, warps 2..11 X-side, 4..7 epilogue
constexpr int kDecPro = kDecThreads - 64;    // threads of the X-side steps
constexpr int kDecSmemOutliers = 128;        // outlier columns whose x values are staged in shared memory
constexpr int kDecTileN = 128;
constexpr int kDecStageBytes = kDecTileN * 128;  // 16 KB
constexpr int kDecRegChunks = 2;             // 8-column chunks a thread keeps in registers (M <= 8)

// Byte offset of Xq[m, k] inside the shared B operand: local K-block kb =
// k/128 holds `groups` 8-row atoms of 1024 bytes; in an atom row r = m%8 is a
// 128-byte line whose 16-byte chunks are XOR-swizzled with r.
__device__ __forceinline__ uint32_t dec_xq_off(int m, int k, int groups) {
    const int kb = k >> 7, g = m >> 3, r = m & 7, c = (k & 127) >> 4;
    return (uint32_t)(((kb * groups + g) << 10) + (r << 7) + ((c ^ r) << 4) + (k & 15));
}

// int8 codes of one 8-column chunk of a row whose outlier flags are fl
// (scale = 0 when the row absmax is 0, which gives codes 0).  Codes are packed
// with byte permutes: __byte_perm(a, b, 0x0040) puts the low bytes of a and b
// in bytes 0 and 1, and 0x5410 joins two such halves.
__device__ __forceinline__ uint2 quant8_flags(uint4 v, uint32_t fl, float scale) {
    const uint32_t h[4] = {v.x, v.y, v.z, v.w};
    int q[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const float x = __half2float(__ushort_as_half((unsigned short)((h[j >> 1] >> ((j & 1) * 16)) & 0xFFFFu)));
        q[j] = quant1(x, scale);
    }
    uint32_t lo = __byte_perm(__byte_perm((uint32_t)q[0], (uint32_t)q[1], 0x0040),
                              __byte_perm((uint32_t)q[2], (uint32_t)q[3], 0x0040), 0x5410);
    uint32_t hi = __byte_perm(__byte_perm((uint32_t)q[4], (uint32_t)q[5], 0x0040),
                              __byte_perm((uint32_t)q[6], (uint32_t)q[7], 0x0040), 0x5410);
    if (fl) {  // outlier columns are zero in the 8-bit product
        const uint32_t mlo = ((fl & 1u) ? 0u : 0xFFu) | ((fl & 2u) ? 0u : 0xFF00u) | ((fl & 4u) ? 0u : 0xFF0000u) |
                             ((fl & 8u) ? 0u : 0xFF000000u);
        const uint32_t mhi = ((fl & 16u) ? 0u : 0xFFu) | ((fl & 32u) ? 0u : 0xFF00u) |
                             ((fl & 64u) ? 0u : 0xFF0000u) | ((fl & 128u) ? 0u : 0xFF000000u);
        lo &= mlo;
        hi &= mhi;
    }
    return make_uint2(lo, hi);
}

// Max |x| (fp16 bits) over the columns of an 8-column chunk whose flag in fl
// is clear: lanes of flagged columns are masked out, then a SIMD max tree.
__device__ __forceinline__ uint32_t inlier_absmax_simd(uint4 v, uint32_t fl) {
    uint32_t a0 = abs_bits2(v.x), a1 = abs_bits2(v.y), a2 = abs_bits2(v.z), a3 = abs_bits2(v.w);
    if (fl) {
        const uint32_t m0 = ((fl & 1u) ? 0u : 0xFFFFu) | ((fl & 2u) ? 0u : 0xFFFF0000u);
        const uint32_t m1 = ((fl & 4u) ? 0u : 0xFFFFu) | ((fl & 8u) ? 0u : 0xFFFF0000u);
        const uint32_t m2 = ((fl & 16u) ? 0u : 0xFFFFu) | ((fl & 32u) ? 0u : 0xFFFF0000u);
        const uint32_t m3 = ((fl & 64u) ? 0u : 0xFFFFu) | ((fl & 128u) ? 0u : 0xFFFF0000u);
        a0 &= m0;
        a1 &= m1;
        a2 &= m2;
        a3 &= m3;
    }
    const uint32_t m = __vmaxu2(__vmaxu2(a0, a1), __vmaxu2(a2, a3));
    return max(m & 0xFFFFu, m >> 16);
}

// Column flags (8 bits) of one chunk from its rows' |x| maxima (fp16 bits,
// NaN already mapped to 0).  thr_bits2 holds, in both 16-bit lanes, the bits of
// the smallest fp16 value >= the threshold (0x7C01 when no finite value and not
// +inf reaches it), so |x| >= thr  <=>  bits(|x|) >= thr_bits as integers.
__device__ __forceinline__ uint32_t chunk_flags(const uint32_t (&mx)[4], uint32_t thr_bits2) {
    uint32_t fl = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t ge = __vcmpgeu2(mx[i], thr_bits2);  // 0xFFFF per lane where mx >= thr
        fl |= ((ge & 1u) << (2 * i)) | (((ge >> 16) & 1u) << (2 * i + 1));
    }
    return fl;
}

__global__ void __launch_bounds__(kDecThreads, 1)
    k_decode_int8_sm100(const __grid_constant__ CUtensorMap tm_w, const DecodeParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* ring = smem;
    uint8_t* sxq = smem + p.off_xq;
    uint32_t* smask = reinterpret_cast<uint32_t*>(smem + p.off_mask);
    int* spre = reinterpret_cast<int*>(smem + p.off_pre);
    uint16_t* slist = reinterpret_cast<uint16_t*>(smem + p.off_list);
    uint16_t* sxo = reinterpret_cast<uint16_t*>(smem + p.off_xo);  // [kDecSmemOutliers][16] fp16 x values
    int* soslot = reinterpret_cast<int*>(smem + p.off_oslot);      // [kDecSmemOutliers] kept-row slot
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + p.off_bars);
    uint64_t* full = bars;
    uint64_t* empty = bars + p.stages;
    uint64_t* tfull = bars + 2 * p.stages;
    uint64_t* xq_ready = tfull + 1;
    uint64_t* drain = tfull + 2;
    uint64_t* x_full = tfull + 3;
    uint64_t* xchg1 = tfull + 4;  // cluster: outlier flags and row maxima exchanged
    uint64_t* xchg2 = tfull + 5;  // cluster: int8 codes exchanged
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tfull + 6);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    unsigned* sra_bits = reinterpret_cast<unsigned*>(tmem_slot + 2);  // [16] row absmax (fp16 bits)
    int* sflag = reinterpret_cast<int*>(tmem_slot + 18);              // [1] total outliers
    float* sscale = reinterpret_cast<float*>(tmem_slot + 20);         // [16] 127 / ra
    float* srs = reinterpret_cast<float*>(tmem_slot + 36);            // [16] ra / 127^2
    const uint16_t* __restrict__ Xg = p.X;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int M = p.M, K = p.K, N = p.N;
    const int nw = (K + 31) / 32;
    const int nchunk = K / 8;
    WaitCtx wctx{abort_flag, p.status, p.wait_limit_ns};

    // this CTA: tile t (128 output channels), K-blocks [kb_lo, kb_hi); CTAs past
    // the last tile only help their cluster with the X-side steps
    const int KB = p.kb_per_tile;
    const int t = blockIdx.x / p.splits, sp = blockIdx.x - t * p.splits;
    const bool has_tile = t < p.num_tiles;
    const int kb_lo = has_tile ? (int)((long long)KB * sp / p.splits) : 0;
    const int kb_hi = has_tile ? (int)((long long)KB * (sp + 1) / p.splits) : 0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < p.stages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(tfull, 1);
        mbar_init(xq_ready, 1);
        mbar_init(drain, 1);
        mbar_init(x_full, 1);
        mbar_init(xchg1, p.cluster);
        mbar_init(xchg2, p.cluster);
        *abort_flag = 0;
        fence_mbar_init();
        prefetch_tmap(&tm_w);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, 32);
        tmem_relinquish();
    }
    if (threadIdx.x >= 64 && threadIdx.x < 64 + 16) sra_bits[threadIdx.x - 64] = 0u;
    for (int w = threadIdx.x; w < nw; w += kDecThreads) smask[w] = 0u;
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (p.cluster > 1) cluster_sync_all();  // every barrier of the cluster is initialised
    const uint32_t tmem_base = *tmem_slot;
    pdl_launch_dependents();

    if (warp == 0) {
        // ------------------------------------------------ weight stream (needs nothing from earlier kernels)
        if (elect_one()) {
            const uint64_t pol = policy_evict_first();
            int stage = 0;
            uint32_t phase = 0, armed = 0, armed_par = 0;
            for (int kb = kb_lo; kb < kb_hi; ++kb) {
                if (!wait_bounded(&empty[stage], phase ^ 1, wctx)) break;
                mbar_arrive_expect_tx(&full[stage], kDecStageBytes);
                tma_load_2d(ring + stage * kDecStageBytes, &tm_w, &full[stage], kb * 128, t * kDecTileN, pol);
                armed |= 1u << stage;
                armed_par = (armed_par & ~(1u << stage)) | (phase << stage);
                if (++stage == p.stages) {
                    stage = 0;
                    phase ^= 1;
                }
            }
            for (int s = 0; s < p.stages; ++s)
                if (armed & (1u << s)) wait_drain(&full[s], (armed_par >> s) & 1u, 50ull * 1000 * 1000);
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (elect_one()) {
            const uint32_t idesc = idesc_s8_s32(128, 16);
            const uint32_t sxq_addr = smem_u32(sxq);
            int stage = 0;
            uint32_t phase = 0;
            bool issued = false, ok = wait_bounded(xq_ready, 0, wctx);
            tc_fence_after();
            for (int kb = kb_lo; ok && kb < kb_hi; ++kb) {
                if (!wait_bounded(&full[stage], phase, wctx)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t sa = smem_u32(ring + stage * kDecStageBytes);
                const uint32_t sb = sxq_addr + (uint32_t)(kb * p.groups * 1024);
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    mma_s8(tmem_base, sdesc_k128sw(sa + 32 * j), sdesc_k128sw(sb + 32 * j), idesc,
                           (kb != kb_lo || j != 0) ? 1u : 0u);
                issued = true;
                tc_commit(&empty[stage]);
                if (++stage == p.stages) {
                    stage = 0;
                    phase ^= 1;
                }
            }
            if (ok) tc_commit(tfull);
            if (issued) {
                tc_commit(drain);
                wait_drain(drain, 0, 50ull * 1000 * 1000);
            }
        }
    } else {
        // ------------------------------------------------ X-side steps (warps 2..11)
        const int pt = threadIdx.x - 64;  // 0 .. kDecPro-1
        pdl_wait();  // X and the workspace belong to earlier work on the stream
        if (p.cluster > 1) {
            // The CTAs of a cluster split X's columns: each stages its share of
            // the 8-column chunks (a multiple of 4 chunks, one mask word), finds
            // their outlier flags and row maxima, pushes those to every peer,
            // then quantises its share and writes the codes into every peer's
            // operand buffer through distributed shared memory.
            const int CL = p.cluster;
            const uint32_t rank = cluster_ctarank();
            const int nq = ((nchunk + 3) / 4 + CL - 1) / CL * 4;  // chunks per rank, whole mask words
            const int c0 = min(nchunk, (int)rank * nq), c1 = min(nchunk, c0 + nq);
            const int nown = c1 - c0;
            uint8_t* xs = smem + p.off_xstage;  // M rows x nq chunks x 16 bytes
            if (pt == 0 && nown > 0) {
                mbar_arrive_expect_tx(x_full, (uint32_t)(M * nown * 16));
                for (int m = 0; m < M; ++m)
                    bulk_load(xs + (size_t)m * nq * 16, Xg + (size_t)m * K + (size_t)c0 * 8, (uint32_t)(nown * 16), x_full);
            }
            if (nown > 0) wait_bounded(x_full, 0, wctx);
            uint32_t rmax[16];
#pragma unroll
            for (int m = 0; m < 16; ++m) rmax[m] = 0;
#pragma unroll 1
            for (int cl = pt; cl < nown; cl += kDecPro) {
                const int c = c0 + cl;
                uint4 v[16];
                uint32_t mx[4] = {0, 0, 0, 0};
#pragma unroll
                for (int m = 0; m < 16; ++m) {
                    if (m < M) {
                        v[m] = *reinterpret_cast<const uint4*>(xs + (size_t)m * nq * 16 + (size_t)cl * 16);
                        mx[0] = __vmaxu2(mx[0], abs_bits2(v[m].x));
                        mx[1] = __vmaxu2(mx[1], abs_bits2(v[m].y));
                        mx[2] = __vmaxu2(mx[2], abs_bits2(v[m].z));
                        mx[3] = __vmaxu2(mx[3], abs_bits2(v[m].w));
                    }
                }
                const uint32_t fl = chunk_flags(mx, p.thr_bits2);
                if (fl) atomicOr(&smask[c >> 2], fl << ((c & 3) * 8));
#pragma unroll
                for (int m = 0; m < 16; ++m)
                    if (m < M) rmax[m] = max(rmax[m], inlier_absmax_simd(v[m], fl));
            }
#pragma unroll
            for (int m = 0; m < 16; ++m) {
                if (m < M) {
                    const uint32_t r = __reduce_max_sync(0xffffffffu, rmax[m]);
                    if (lane == 0 && r) atomicMax(&sra_bits[m], r);
                }
            }
            named_bar_sync(1, kDecPro);
            // push this CTA's mask words and row maxima to the peers
            for (int w = c0 / 4 + pt; w < (c1 + 3) / 4; w += kDecPro) {
                const uint32_t val = smask[w];
                if (val)
                    for (int r = 0; r < CL; ++r)
                        if (r != (int)rank) st_cluster_u32(map_to_rank(&smask[w], r), val);
            }
            if (pt < M && sra_bits[pt])
                for (int r = 0; r < CL; ++r)
                    if (r != (int)rank) atom_max_cluster_u32(map_to_rank(&sra_bits[pt], r), sra_bits[pt]);
            fence_acq_rel_cluster();
            named_bar_sync(1, kDecPro);
            if (pt == 0)
                for (int r = 0; r < CL; ++r) mbar_arrive_cluster(map_to_rank(xchg1, r));
            wait_bounded_cluster(xchg1, 0, wctx);
            // the whole mask and the row maxima are here now
            if (warp == 2) {
                int carry = 0;
                for (int base = 0; base < nw; base += 32) {
                    const int w = base + lane;
                    const uint32_t word = w < nw ? smask[w] : 0u;
                    const int cnt = __popc(word);
                    int incl = cnt;
#pragma unroll
                    for (int o = 1; o < 32; o <<= 1) {
                        const int v = __shfl_up_sync(0xffffffffu, incl, o);
                        if (lane >= o) incl += v;
                    }
                    if (w < nw) spre[w] = carry + incl - cnt;
                    carry += __shfl_sync(0xffffffffu, incl, 31);
                }
                if (lane == 0) sflag[0] = carry;
            } else if (warp == 3 && lane < 16) {
                const float rmax = half_bits_to_float(sra_bits[lane]);
                sscale[lane] = rmax > 0.0f ? __fdiv_rn(127.0f, rmax) : 0.0f;
                srs[lane] = __fdiv_rn(rmax, 16129.0f);
                if (blockIdx.x == 0 && lane < M) p.ra_out[lane] = rmax;
            }
            named_bar_sync(1, kDecPro);
            // (b) int8 codes of this CTA's chunks, all rows, into every CTA's
            // operand buffer; the first cluster also writes them to the workspace
            for (int e = pt; e < M * nown; e += kDecPro) {
                const int m = e / nown, cl = e - m * nown;
                const int c = c0 + cl;
                const uint4 v = *reinterpret_cast<const uint4*>(xs + (size_t)m * nq * 16 + (size_t)cl * 16);
                const uint32_t fl = (smask[c >> 2] >> ((c & 3) * 8)) & 0xFFu;
                const uint2 q = quant8_flags(v, fl, sscale[m]);
                uint8_t* dst = sxq + dec_xq_off(m, c * 8, p.groups);
                *reinterpret_cast<uint2*>(dst) = q;
                for (int r = 0; r < CL; ++r)
                    if (r != (int)rank) st_cluster_v2(map_to_rank(dst, r), q);
                if ((int)blockIdx.x < CL) *reinterpret_cast<uint2*>(p.xq_out + (size_t)m * K + (size_t)c * 8) = q;
            }
            fence_proxy_async_cluster();
            fence_acq_rel_cluster();
            named_bar_sync(1, kDecPro);
            if (pt == 0)
                for (int r = 0; r < CL; ++r) mbar_arrive_cluster(map_to_rank(xchg2, r));
            wait_bounded_cluster(xchg2, 0, wctx);
        } else {
            // Fast path: every chunk of this thread, all M <= 8 rows, in registers;
            // X is read once and the codes come from the same registers.
            const bool fast = (M <= 8) && (nchunk <= kDecRegChunks * kDecPro);
            uint4 xv[kDecRegChunks][8];
            uint32_t cfl[kDecRegChunks] = {0u, 0u};
            {
                uint32_t rmax[16];
    #pragma unroll
                for (int m = 0; m < 16; ++m) rmax[m] = 0;
                if (fast) {
    #pragma unroll
                    for (int i = 0; i < kDecRegChunks; ++i) {
                        const int c = pt + i * kDecPro;
    #pragma unroll
                        for (int m = 0; m < 8; ++m)
                            if (c < nchunk && m < M) xv[i][m] = __ldg(reinterpret_cast<const uint4*>(Xg + (size_t)m * K) + c);
                    }
    #pragma unroll
                    for (int i = 0; i < kDecRegChunks; ++i) {
                        const int c = pt + i * kDecPro;
                        if (c < nchunk) {
                            uint32_t mx[4] = {0, 0, 0, 0};
    #pragma unroll
                            for (int m = 0; m < 8; ++m) {
                                if (m < M) {
                                    mx[0] = __vmaxu2(mx[0], abs_bits2(xv[i][m].x));
                                    mx[1] = __vmaxu2(mx[1], abs_bits2(xv[i][m].y));
                                    mx[2] = __vmaxu2(mx[2], abs_bits2(xv[i][m].z));
                                    mx[3] = __vmaxu2(mx[3], abs_bits2(xv[i][m].w));
                                }
                            }
                            const uint32_t fl = chunk_flags(mx, p.thr_bits2);
                            cfl[i] = fl;
                            if (fl) atomicOr(&smask[c >> 2], fl << ((c & 3) * 8));
    #pragma unroll
                            for (int m = 0; m < 8; ++m)
                                if (m < M) rmax[m] = max(rmax[m], inlier_absmax_simd(xv[i][m], fl));
                        }
                    }
                } else {
                    for (int c = pt; c < nchunk; c += kDecPro) {
                        uint4 v[16];
    #pragma unroll
                        for (int m = 0; m < 16; ++m)
                            if (m < M) v[m] = __ldg(reinterpret_cast<const uint4*>(Xg + (size_t)m * K) + c);
                        uint32_t mx[4] = {0, 0, 0, 0};
    #pragma unroll
                        for (int m = 0; m < 16; ++m) {
                            if (m < M) {
                                mx[0] = __vmaxu2(mx[0], abs_bits2(v[m].x));
                                mx[1] = __vmaxu2(mx[1], abs_bits2(v[m].y));
                                mx[2] = __vmaxu2(mx[2], abs_bits2(v[m].z));
                                mx[3] = __vmaxu2(mx[3], abs_bits2(v[m].w));
                            }
                        }
                        const uint32_t fl = chunk_flags(mx, p.thr_bits2);
                        if (fl) atomicOr(&smask[c >> 2], fl << ((c & 3) * 8));
    #pragma unroll
                        for (int m = 0; m < 16; ++m)
                            if (m < M) rmax[m] = max(rmax[m], inlier_absmax_simd(v[m], fl));
                    }
                }
    #pragma unroll
                for (int m = 0; m < 16; ++m) {
                    if (m < M) {
                        const uint32_t r = __reduce_max_sync(0xffffffffu, rmax[m]);
                        if (lane == 0 && r) atomicMax(&sra_bits[m], r);
                    }
                }
            }
            named_bar_sync(1, kDecPro);
            // slot prefix of the outlier list (warp 2, off the critical path of
            // the codes); CTA 0 publishes the row absmax
            if (warp == 2) {
                int carry = 0;
                for (int base = 0; base < nw; base += 32) {
                    const int w = base + lane;
                    const uint32_t word = w < nw ? smask[w] : 0u;
                    const int c = __popc(word);
                    int incl = c;
    #pragma unroll
                    for (int o = 1; o < 32; o <<= 1) {
                        const int v = __shfl_up_sync(0xffffffffu, incl, o);
                        if (lane >= o) incl += v;
                    }
                    if (w < nw) spre[w] = carry + incl - c;
                    carry += __shfl_sync(0xffffffffu, incl, 31);
                }
                if (lane == 0) sflag[0] = carry;
            } else if (warp == 3 && lane < 16) {
                const float rmax = half_bits_to_float(sra_bits[lane]);
                srs[lane] = __fdiv_rn(rmax, 16129.0f);
                if (blockIdx.x == 0 && lane < M) p.ra_out[lane] = rmax;
            }
            // (b) int8 codes of this CTA's K-blocks into the shared B operand; the
            // CTAs of tile 0 also write their K-blocks of Xq to the workspace.
            if (fast) {
                float scl[8];
    #pragma unroll
                for (int m = 0; m < 8; ++m) {
                    const float rmax = half_bits_to_float(sra_bits[m]);
                    scl[m] = rmax > 0.0f ? __fdiv_rn(127.0f, rmax) : 0.0f;
                }
    #pragma unroll
                for (int i = 0; i < kDecRegChunks; ++i) {
                    const int c = pt + i * kDecPro;
                    const int kb = c >> 4;
                    if (c < nchunk && kb >= kb_lo && kb < kb_hi) {
    #pragma unroll
                        for (int m = 0; m < 8; ++m) {
                            if (m < M) {
                                const uint2 q = quant8_flags(xv[i][m], cfl[i], scl[m]);
                                *reinterpret_cast<uint2*>(sxq + dec_xq_off(m, c * 8, p.groups)) = q;
                                if (t == 0) *reinterpret_cast<uint2*>(p.xq_out + (size_t)m * K + c * 8) = q;
                            }
                        }
                    }
                }
            } else {
                if (warp == 3 && lane < 16) {
                    const float rmax = half_bits_to_float(sra_bits[lane]);
                    sscale[lane] = rmax > 0.0f ? __fdiv_rn(127.0f, rmax) : 0.0f;
                }
                named_bar_sync(1, kDecPro);  // the general path reads the flags' slot prefix and scales
                const int per_kb = M * 8;    // (row, 16-column chunk) pairs per K-block
                for (int e = pt; e < (kb_hi - kb_lo) * per_kb; e += kDecPro) {
                    const int i = e / per_kb, rem = e - i * per_kb;
                    const int kb = kb_lo + i;
                    const int m = rem >> 3, c16 = kb * 8 + (rem & 7);
                    if (c16 * 16 >= K) continue;
                    const uint4* src = reinterpret_cast<const uint4*>(Xg + (size_t)m * K) + 2 * c16;
                    const uint4 x0 = __ldg(src), x1 = __ldg(src + 1);
                    const float rmax = half_bits_to_float(sra_bits[m]);
                    const uint2 q0 = quant_chunk(x0, smask, spre, 2 * c16, rmax, sscale[m], 0, nullptr);
                    const uint2 q1 = quant_chunk(x1, smask, spre, 2 * c16 + 1, rmax, sscale[m], 0, nullptr);
                    const uint4 q = make_uint4(q0.x, q0.y, q1.x, q1.y);
                    *reinterpret_cast<uint4*>(sxq + dec_xq_off(m, c16 * 16, p.groups)) = q;
                    if (t == 0) *reinterpret_cast<uint4*>(p.xq_out + (size_t)m * K + c16 * 16) = q;
                }
            }
        }
        fence_proxy_async_smem();
        named_bar_sync(1, kDecPro);
        if (pt == 0 && !(p.test_flags & 1u)) mbar_arrive(xq_ready);
        const int total = sflag[0];
        const int n_eff = min(total, p.cap);
        // outlier list (ascending) into shared memory with the x values and
        // kept-row slots of the first kDecSmemOutliers; CTA 0 publishes it
        for (int w = pt; w < nw; w += kDecPro) {
            uint32_t word = smask[w];
            int s = spre[w];
            while (word) {
                const int b = __ffs(word) - 1;
                const int k = w * 32 + b;
                if (s < n_eff) {
                    slist[s] = (uint16_t)k;
                    if (blockIdx.x == 0) p.idx_out[s] = k;
                    if (s < kDecSmemOutliers) {
                        soslot[s] = p.keep_slot[k];
#pragma unroll
                        for (int m = 0; m < 16; ++m) sxo[s * 16 + m] = m < M ? Xg[(size_t)m * K + k] : (uint16_t)0;
                    }
                }
                ++s;
                word &= word - 1;
            }
        }
        if (blockIdx.x == 0 && pt == 0) {
            *p.n_out = total;
            if (total > p.cap) atomicOr(p.status, kStatusOverflow);
        }
        named_bar_sync(1, kDecPro);

        if (warp >= 4 && warp < 8 && has_tile) {
            // ------------------------------------------------ epilogue (warps 4..7)
            const int quad = warp & 3;
            const int n = t * kDecTileN + quad * 32 + lane;
            // (d) fp16 outlier product, ascending j, while the weights stream:
            // the weight value of outlier j is the kept fp16 row or the
            // dequantised int8 row
            float o[16];
#pragma unroll
            for (int m = 0; m < 16; ++m) o[m] = 0.0f;
            const float cav = n < N ? p.ca[n] : 0.0f;
            if (n < N) {
                const int n_fast = min(n_eff, kDecSmemOutliers);
#pragma unroll 4
                for (int j = 0; j < n_fast; ++j) {
                    const int slot = soslot[j];
                    float w;
                    if (slot >= 0) {
                        w = half_bits_to_float(p.w_keep[(size_t)slot * N + n]);
                    } else {
                        const float tq = __fmul_rn((float)p.wq[(size_t)n * K + slist[j]], cav);
                        w = __half2float(__float2half_rn(__fdiv_rn(tq, 127.0f)));
                    }
#pragma unroll
                    for (int m = 0; m < 16; ++m)
                        if (m < M) o[m] = fmaf(half_bits_to_float(sxo[j * 16 + m]), w, o[m]);
                }
                for (int j = n_fast; j < n_eff; ++j) {
                    const int k = slist[j];
                    const int slot = p.keep_slot[k];
                    float w;
                    if (slot >= 0) {
                        w = half_bits_to_float(p.w_keep[(size_t)slot * N + n]);
                    } else {
                        const float tq = __fmul_rn((float)p.wq[(size_t)n * K + k], cav);
                        w = __half2float(__float2half_rn(__fdiv_rn(tq, 127.0f)));
                    }
#pragma unroll
                    for (int m = 0; m < 16; ++m)
                        if (m < M) o[m] = fmaf(half_bits_to_float(Xg[(size_t)m * K + k]), w, o[m]);
                }
            }
            if (__all_sync(0xffffffffu, wait_bounded(tfull, 0, wctx))) {
                tc_fence_after();
                uint32_t r[16];
                tmem_ld16(tmem_base + ((uint32_t)(quad * 32) << 16), r);
                tmem_wait_ld();
                // K split: the partial sums of the tile meet in the workspace;
                // completion is counted per (tile, 32-column quadrant), so each
                // warp decides on its own columns with no block barrier.
                bool last = true;
                if (p.splits > 1) {
                    const int nunits = kb_hi - kb_lo;
                    if (n < N) {
#pragma unroll
                        for (int m = 0; m < 16; ++m)
                            if (m < M) atomicAdd(&p.partial[(size_t)m * N + n], (int)r[m]);
                    }
                    __threadfence();
                    __syncwarp();
                    int old = 0;
                    if (lane == 0) old = atomicAdd(&p.counters[t * 4 + quad], nunits);
                    old = __shfl_sync(0xffffffffu, old, 0);
                    last = (old + nunits == KB);
                    if (last) {
                        __threadfence();
                        if (n < N) {
#pragma unroll
                            for (int m = 0; m < 16; ++m)
                                if (m < M) r[m] = (uint32_t)atomicExch(&p.partial[(size_t)m * N + n], 0);
                        }
                        if (lane == 0) p.counters[t * 4 + quad] = 0;
                    }
                }
                if (last && n < N) {
#pragma unroll
                    for (int m = 0; m < 16; ++m) {
                        if (m < M) {
                            const float y = (float)(int32_t)r[m] * srs[m] * cav + o[m];
                            p.Y[(size_t)m * N + n] = __half_as_ushort(__float2half_rn(y));
                            if (p.acc_out) p.acc_out[(size_t)m * N + n] = (int32_t)r[m];
                        }
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, 32);
    }
    if (p.cluster > 1) cluster_sync_all();  // no CTA leaves while a peer may still write to it
}

}  // namespace i8mm
