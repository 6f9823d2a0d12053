// Decode-shaped LLM.int8() forward (M <= 16 rows of X) in one kernel.
//
// At small M the product is bound by reading the int8 weight once: loading
// weights from memory costs far more than the arithmetic on them (axolotl
// "llama3-model-quantization", "Impact of Precision and Parameter Count on
// Model Efficiency").  The kernel streams the weight through every CTA's TMA
// ring from the moment the CTA starts and keeps the X-side steps that gate
// the first tensor-core instruction short:
//
// Clusters of CL CTAs (4, or 8 for long K; as many as K has 128-column blocks
// when that is fewer) split K: CTA r of a cluster owns the
// r-th K range of the cluster's T (<= CL) 128-channel weight tiles.  It reads
// only its K range of X, so the outlier flags of those columns are final at
// once (all M rows of a column are in the same CTA), quantises only those
// columns, and shares with its peers just the flag words and the row maxima
// (one exchange of asynchronous stores into the peers' shared memory, which
// complete on the receiver's mbarrier).  The int32 partial sums of a tile go
// the same way to the tile's owner (CTA j owns tile j), one slot per source
// CTA, and the owner adds the slots (exact in any order).
//
// Warp roles (384 threads):
//   warp 0: TMA producer of 128 (channels) x 128 (K) int8 weight boxes;
//   warp 1: tcgen05.mma kind::i8 with the weight as the 128-row A operand and
//     the (padded) activation rows as the 16-column B operand ("swap AB"),
//     one s32 TMEM accumulator per tile;
//   warps 2-11: (a) outlier columns and row absmax of the CTA's K range, then
//     (b) the int8 codes straight into shared memory in the tensor-core
//     operand layout (128-byte rows, 128-byte swizzle, 8-row groups);
//   warps 4-7 (after the X-side steps): the fp16 outlier product (d) of the
//     owned tile while the weights stream, then the reduction of the partial
//     sums and Y = fp16(acc * ra * ca / 127^2 + o).
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "sm100_ptx.cuh"

namespace i8mm {

struct DecodeParams {
    const uint16_t* X;
    int M, K, N;
    uint32_t thr_bits2;         // smallest fp16 >= thr, in both 16-bit lanes
    int cap;                    // outlier capacity (list + overflow flag)
    const int8_t* wq;           // N x K (dequantised outlier rows that were not kept)
    const float* ca;
    const uint16_t* w_keep;
    const int32_t* keep_slot;
    uint16_t* Y;
    int32_t* acc_out;           // optional M x N
    int32_t* idx_out;           // workspace: outlier list
    int32_t* n_out;             // workspace: outlier count
    float* ra_out;              // workspace: M
    int8_t* xq_out;             // workspace: M x K
    int* status;
    uint64_t wait_limit_ns;
    uint32_t test_flags;        // bit 0: never signal that Xq is ready (timeout test)
    int num_tiles, kb_total;    // 128-channel tiles, 128-column K blocks
    int cluster, tiles_per_cluster, stages, groups;  // groups = ceil(M / 8)
    uint32_t off_xq, off_mask, off_pre, off_list, off_xo, off_oslot, off_red, off_bars;  // shared-memory offsets
};

constexpr int kDecThreads = 384;             // warp 0 TMA, warp 1 MMA, warps 2..11 X-side, 4..7 epilogue
constexpr int kDecPro = kDecThreads - 64;    // threads of the X-side steps
constexpr int kDecSmemOutliers = 128;        // outlier columns whose x values are staged in shared memory
constexpr int kDecTileN = 128;
constexpr int kDecStageBytes = kDecTileN * 128;  // 16 KB
constexpr int kDecMaxCluster = 8;

__device__ __forceinline__ float dec_half_to_float(uint32_t bits16) {
    return __half2float(__ushort_as_half((unsigned short)bits16));
}

// Byte offset of Xq[m, k] inside the shared B operand (k relative to the
// CTA's K range): K-block kb = k/128 holds `groups` 8-row atoms of 1024 bytes;
// in an atom row r = m%8 is a 128-byte line whose 16-byte chunks are
// XOR-swizzled with r.
__device__ __forceinline__ uint32_t dec_xq_off(int m, int k, int groups) {
    const int kb = k >> 7, g = m >> 3, r = m & 7, c = (k & 127) >> 4;
    return (uint32_t)(((kb * groups + g) << 10) + (r << 7) + ((c ^ r) << 4) + (k & 15));
}

// int8 codes of one 8-column chunk of a row whose outlier flags are fl.
// code = round_half_even(RN32(x * scale)) comes from the low byte of
// RN32(RN32(x * scale) + 1.5 * 2^23): for |v| < 2^22 that sum keeps
// round_half_even(v) in its low mantissa bits, and here |x * scale| is at most
// 127 * (1 + 2^-24) for every non-outlier column, so no clamp is needed.  The
// product and the sum are two separately rounded operations (__fmul_rn and
// __fadd_rn are never contracted into a fused multiply-add, which would round
// only once and move ties such as x * scale = 63.5 - 2e-6).  Outlier columns
// give 0.
__device__ __forceinline__ uint2 dec_quant8(uint4 v, uint32_t fl, float scale) {
    const uint32_t h[4] = {v.x, v.y, v.z, v.w};
    uint32_t b[8];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&h[j]));
        b[2 * j] = __float_as_uint(__fadd_rn(__fmul_rn(f.x, scale), 12582912.0f));
        b[2 * j + 1] = __float_as_uint(__fadd_rn(__fmul_rn(f.y, scale), 12582912.0f));
    }
    // __byte_perm(a, b, 0x0040) puts the low bytes of a and b in bytes 0 and
    // 1; 0x5410 joins two such halves
    uint32_t lo = __byte_perm(__byte_perm(b[0], b[1], 0x0040), __byte_perm(b[2], b[3], 0x0040), 0x5410);
    uint32_t hi = __byte_perm(__byte_perm(b[4], b[5], 0x0040), __byte_perm(b[6], b[7], 0x0040), 0x5410);
    if (fl) {
        uint32_t mlo = 0u, mhi = 0u;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            mlo |= ((fl >> j) & 1u) ? 0u : (0xFFu << (8 * j));
            mhi |= ((fl >> (j + 4)) & 1u) ? 0u : (0xFFu << (8 * j));
        }
        lo &= mlo;
        hi &= mhi;
    }
    return make_uint2(lo, hi);
}

// Pass (a) works on packed fp16 pairs with the native half2 compare and max:
// |x| is the bit pattern with the sign cleared, __hge2_mask gives false for
// NaN (so NaN is never an outlier) and __hmax2 returns the other operand when
// one is NaN (so NaN never enters a row maximum).  thr2 holds, in both
// halves, the smallest fp16 value >= the threshold (a NaN pattern when none
// is, so nothing is flagged), so |x| >= thr  <=>  __hge2(|x|, thr2).
__device__ __forceinline__ __half2 as_h2(uint32_t b) {
    __half2 h;
    memcpy(&h, &b, 4);
    return h;
}

__device__ __forceinline__ uint32_t as_u32(__half2 h) {
    uint32_t b;
    memcpy(&b, &h, 4);
    return b;
}

__device__ __forceinline__ uint4 abs8(uint4 v) {
    return make_uint4(v.x & 0x7FFF7FFFu, v.y & 0x7FFF7FFFu, v.z & 0x7FFF7FFFu, v.w & 0x7FFF7FFFu);
}

// Outlier flags (bit j = column j) of one row's 8 columns from their |x|.
__device__ __forceinline__ uint32_t flags8(uint4 a, __half2 thr2) {
    const uint32_t m0 = __hge2_mask(as_h2(a.x), thr2), m1 = __hge2_mask(as_h2(a.y), thr2);
    const uint32_t m2 = __hge2_mask(as_h2(a.z), thr2), m3 = __hge2_mask(as_h2(a.w), thr2);
    return (m0 & 1u) | ((m0 >> 15) & 2u) | ((m1 & 1u) << 2) | ((m1 >> 13) & 8u) | ((m2 & 1u) << 4) |
           ((m2 >> 11) & 32u) | ((m3 & 1u) << 6) | ((m3 >> 9) & 128u);
}

// Per-lane max of |x| over the columns whose flag in fl is clear (flagged
// lanes count as +0).
__device__ __forceinline__ __half2 inlier_max8(uint4 a, uint32_t fl) {
    if (fl) {
        uint32_t k[4];
#pragma unroll
        for (int w = 0; w < 4; ++w)
            k[w] = (((fl >> (2 * w)) & 1u) ? 0u : 0xFFFFu) | (((fl >> (2 * w + 1)) & 1u) ? 0u : 0xFFFF0000u);
        a.x &= k[0];
        a.y &= k[1];
        a.z &= k[2];
        a.w &= k[3];
    }
    return __hmax2(__hmax2(as_h2(a.x), as_h2(a.y)), __hmax2(as_h2(a.z), as_h2(a.w)));
}

// kR: rows per 8-column chunk group (8 or 16, >= M); kP: (chunk, row) pairs
// per X-side thread (the CTA's K range has at most kP * kDecPro / kR chunks).
template <int kR, int kP>
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
    uint32_t* sred = reinterpret_cast<uint32_t*>(smem + p.off_red);  // [CL][128][RS] partial sums of the owned tile
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + p.off_bars);
    uint64_t* full = bars;
    uint64_t* empty = bars + p.stages;
    uint64_t* tfull = bars + 2 * p.stages;
    uint64_t* xq_ready = tfull + 1;
    uint64_t* drain = tfull + 2;
    uint64_t* xchg = tfull + 3;      // flag words and row maxima of every peer have arrived (tx bytes)
    uint64_t* red_done = tfull + 4;  // every peer's partial sums have arrived (tx bytes)
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tfull + 5);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    unsigned* sra_bits = reinterpret_cast<unsigned*>(tmem_slot + 2);  // [16] row absmax (fp16 bits)
    int* sflag = reinterpret_cast<int*>(tmem_slot + 18);              // [1] total outliers
    float* srs = reinterpret_cast<float*>(tmem_slot + 20);            // [16] ra / 127^2
    const uint16_t* __restrict__ Xg = p.X;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int M = p.M, K = p.K, N = p.N;
    const int nw = (K + 31) / 32;
    const int nchunk = K / 8;
    const int CL = p.cluster;
    const int RS = 8 * p.groups;  // rows of one partial-sum slot
    WaitCtx wctx{abort_flag, p.status, p.wait_limit_ns};

    // this CTA: K blocks [kb_lo, kb_hi) of tiles [tile0, tile0 + nt); it owns
    // tile tile0 + rank when rank < nt
    const int rank = (int)cluster_ctarank();
    const int cid = blockIdx.x / CL;
    const int tile0 = cid * p.tiles_per_cluster;
    const int nt = max(0, min(p.tiles_per_cluster, p.num_tiles - tile0));
    const int kb_lo = p.kb_total * rank / CL;  // kb_total <= 1024, CL <= 8: no overflow
    const int kb_hi = p.kb_total * (rank + 1) / CL;
    const int c0 = kb_lo * 16, c1 = min(nchunk, kb_hi * 16);
    const bool owner = rank < nt;
    const bool has_acc = nt > 0 && kb_hi > kb_lo;
    const uint32_t tmem_cols = p.tiles_per_cluster <= 1 ? 32u : (p.tiles_per_cluster <= 2 ? 64u : (p.tiles_per_cluster <= 4 ? 128u : 256u));

    // Set-up is split by role so that the X-side steps, which gate the first
    // MMA, start at once: warp 0 initialises the mbarriers and starts the
    // weight stream, warp 1 allocates TMEM, the X-side warps clear their
    // buffers and load X.  Named barrier 2 ("mbarriers initialised, TMEM
    // allocated"): warp 0 arrives, everyone else waits on it before the
    // first use.  Peers write into this CTA only after the cluster barrier
    // completes; every thread arrives once its part of the set-up is done and
    // waits just before its first access to a peer (the weight stream needs
    // no peer).
    uint32_t tmem_base = 0;
    if (warp == 0) {
        if (lane == 0) {
            for (int s = 0; s < p.stages; ++s) {
                mbar_init(&full[s], 1);
                mbar_init(&empty[s], 1);
            }
            mbar_init(tfull, 1);
            mbar_init(xq_ready, 1);
            mbar_init(drain, 1);
            mbar_init(xchg, 1);
            mbar_init(red_done, 1);
            *abort_flag = 0;
            fence_mbar_init();
            prefetch_tmap(&tm_w);
            // bytes the peers will store: their flag words and M row maxima
            // each, and (owner) one partial-sum slot per CTA of the cluster
            uint32_t xb = 0;
            for (int q = 0; q < CL; ++q) {
                if (q == rank) continue;
                const int qlo = p.kb_total * q / CL, qhi = p.kb_total * (q + 1) / CL;
                xb += (uint32_t)(((min(nchunk, qhi * 16) + 3) / 4 - qlo * 4) * 4 + M * 4);
            }
            if (xb) mbar_arrive_expect_tx(xchg, xb);
            else mbar_arrive(xchg);
            if (owner && has_acc) mbar_arrive_expect_tx(red_done, (uint32_t)(CL * kDecTileN * RS * 4));
        }
        __syncwarp();
        cluster_arrive();
        named_bar_arrive(2, kDecThreads);
    } else if (warp == 1) {
        tmem_alloc(tmem_slot, tmem_cols);
        tmem_relinquish();
        tc_fence_before();
        cluster_arrive();
        named_bar_sync(2, kDecThreads);
        tc_fence_after();
        tmem_base = *tmem_slot;
    }
    pdl_launch_dependents();

    if (warp == 0) {
        // ------------------------------------------------ weight stream (needs nothing from earlier kernels)
        if (elect_one()) {
            const uint64_t pol = policy_evict_first();
            int stage = 0;
            uint32_t phase = 0, armed = 0, armed_par = 0;
            bool ok = true;
            for (int j = 0; ok && j < nt; ++j) {
                for (int kb = kb_lo; kb < kb_hi; ++kb) {
                    if (!wait_bounded_sleep(&empty[stage], phase ^ 1, wctx)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&full[stage], kDecStageBytes);
                    tma_load_2d(ring + stage * kDecStageBytes, &tm_w, &full[stage], kb * 128, (tile0 + j) * kDecTileN, pol);
                    armed |= 1u << stage;
                    armed_par = (armed_par & ~(1u << stage)) | (phase << stage);
                    if (++stage == p.stages) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
            }
            for (int s = 0; s < p.stages; ++s)
                if (armed & (1u << s)) wait_drain(&full[s], (armed_par >> s) & 1u, 50ull * 1000 * 1000);
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (elect_one() && has_acc) {
            // One thread issues every MMA, so the loop keeps its per-stage work
            // small: descriptors are the base descriptors plus the operand
            // offset >> 4 (the start-address field holds address >> 4 in 14
            // bits, and shared-memory addresses stay below 2^18, so the sum
            // never carries out of the field); 32 bytes of K are +2.
            const uint32_t idesc = idesc_s8_s32(128, 16);
            const uint64_t da0 = sdesc_k128sw(smem_u32(ring));
            const uint64_t db0 = sdesc_k128sw(smem_u32(sxq));
            const uint64_t db_step = (uint64_t)((p.groups * 1024) >> 4);
            int stage = 0;
            uint32_t phase = 0;
            bool issued = false, ok = wait_bounded_sleep(xq_ready, 0, wctx);
            tc_fence_after();
            uint64_t da = da0;  // descriptor of the current ring stage
            for (int j = 0; ok && j < nt; ++j) {
                const uint32_t dtm = tmem_base + (uint32_t)(32 * j);
                uint64_t db = db0;
                for (int kb = kb_lo; kb < kb_hi; ++kb) {
                    if (!mbar_try_wait(&full[stage], phase) && !wait_bounded_sleep(&full[stage], phase, wctx)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    mma_s8_k128_commit(dtm, da, db, idesc, kb != kb_lo ? 1u : 0u, &empty[stage]);
                    db += db_step;
                    issued = true;
                    da += (uint64_t)(kDecStageBytes >> 4);
                    if (++stage == p.stages) {
                        stage = 0;
                        phase ^= 1;
                        da = da0;
                    }
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
        if (pt < 16) sra_bits[pt] = 0u;
        for (int w = pt; w < nw; w += kDecPro) smask[w] = 0u;
        named_bar_sync(1, kDecPro);
        cluster_arrive();
        pdl_wait();  // X belongs to earlier work on the stream
        // (a) Thread pairs (8-column chunk, row): the kR rows of a chunk sit in
        // kR consecutive lanes, so a chunk's outlier flags are the OR of its
        // lanes' flags (shuffles), and a thread's row is the same for all its
        // pairs (kDecPro is a multiple of 32 and of kR), so one running max
        // and one scale per thread.  The values stay in registers for (b).
        const int prow = lane % kR;
        const bool row_ok = prow < M;
        // iterations that hold any pair of this CTA (the same for every thread)
        const int nit = ((c1 - c0) * kR + kDecPro - 1) / kDecPro;
        uint4 xv[kP];
        uint32_t cfl[kP];
#pragma unroll
        for (int i = 0; i < kP; ++i) {
            const int c = c0 + (pt + i * kDecPro) / kR;
            if (i < nit && row_ok && c < c1) xv[i] = __ldg(reinterpret_cast<const uint4*>(Xg + (size_t)prow * K) + c);
        }
        {
            // in phases over the iterations, so that their dependency chains
            // (compare, shuffles, mask, max) overlap
            const __half2 thr2 = as_h2(p.thr_bits2);
            __half2 rmax2 = as_h2(0u);
#pragma unroll
            for (int i = 0; i < kP; ++i) {
                const int c = c0 + (pt + i * kDecPro) / kR;
                cfl[i] = (i < nit && row_ok && c < c1) ? flags8(abs8(xv[i]), thr2) : 0u;
            }
#pragma unroll
            for (int off = 1; off < kR; off <<= 1) {
#pragma unroll
                for (int i = 0; i < kP; ++i)
                    if (i < nit) cfl[i] |= __shfl_xor_sync(0xffffffffu, cfl[i], off);
            }
#pragma unroll
            for (int i = 0; i < kP; ++i) {
                const int c = c0 + (pt + i * kDecPro) / kR;
                if (i < nit && c < c1) {
                    if (prow == 0 && cfl[i]) atomicOr(&smask[c >> 2], cfl[i] << ((c & 3) * 8));
                    if (row_ok) rmax2 = __hmax2(rmax2, inlier_max8(abs8(xv[i]), cfl[i]));
                }
            }
            // non-negative fp16 bit patterns order like their values
            const uint32_t rb = as_u32(rmax2);
            uint32_t rmax = max(rb & 0xFFFFu, rb >> 16);
#pragma unroll
            for (int off = kR; off < 32; off <<= 1) rmax = max(rmax, __shfl_xor_sync(0xffffffffu, rmax, off));
            if (lane < kR && row_ok && rmax) atomicMax(&sra_bits[prow], rmax);
        }
        // every X-side thread's flags and maxima are in; the mbarriers are
        // initialised and TMEM is allocated
        named_bar_sync(2, kDecThreads);
        tc_fence_after();
        tmem_base = *tmem_slot;
        // this CTA's flag words (its K range covers whole words) and row
        // maxima to every peer; the peers' arrive the same way
        if (CL > 1) {
            cluster_wait();  // every peer's barriers and buffers are initialised
            for (int w = c0 / 4 + pt; w < (c1 + 3) / 4; w += kDecPro) {
                const uint32_t val = smask[w];
                for (int q = 0; q < CL; ++q)
                    if (q != rank) st_async_u32(map_to_rank(&smask[w], (uint32_t)q), val, map_to_rank(xchg, (uint32_t)q));
            }
            if (pt >= kDecPro - 16 && pt - (kDecPro - 16) < M) {
                const int m = pt - (kDecPro - 16);
                const uint32_t val = sra_bits[m];
                for (int q = 0; q < CL; ++q)
                    if (q != rank)
                        red_async_max_u32(map_to_rank(&sra_bits[m], (uint32_t)q), val, map_to_rank(xchg, (uint32_t)q));
            }
        } else {
            cluster_wait();
        }
        wait_bounded_sleep(xchg, 0, wctx);
        // the whole mask and the row maxima are here: this thread's scale,
        // then (b) the int8 codes of its pairs into the shared B operand; the
        // first cluster also writes them to the workspace
        {
            const float rmax = row_ok ? dec_half_to_float(sra_bits[prow]) : 0.0f;
            const float scl = rmax > 0.0f ? __fdiv_rn(127.0f, rmax) : 0.0f;
#pragma unroll
            for (int i = 0; i < kP; ++i) {
                const int c = c0 + (pt + i * kDecPro) / kR;
                if (i < nit && row_ok && c < c1) {
                    const uint2 q = dec_quant8(xv[i], cfl[i], scl);
                    *reinterpret_cast<uint2*>(sxq + dec_xq_off(prow, (c - c0) * 8, p.groups)) = q;
                    if ((int)blockIdx.x < CL) *reinterpret_cast<uint2*>(p.xq_out + (size_t)prow * K + (size_t)c * 8) = q;
                }
            }
        }
        if (warp == 3 && lane < 16) {
            const float rmax = dec_half_to_float(sra_bits[lane]);
            srs[lane] = __fdiv_rn(rmax, 16129.0f);
            if (blockIdx.x == 0 && lane < M) p.ra_out[lane] = rmax;
        }
        fence_proxy_async_smem();
        named_bar_sync(1, kDecPro);
        if (pt == 0 && !(p.test_flags & 1u)) mbar_arrive(xq_ready);
        // slot prefix of the outlier flags (off the critical path of the codes)
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
        }
        named_bar_sync(1, kDecPro);
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

        if (warp >= 4 && warp < 8) {
            // ------------------------------------------------ epilogue (warps 4..7)
            const int quad = warp & 3;
            const int ch = quad * 32 + lane;  // channel within a tile (TMEM lane)
            const int n = (tile0 + rank) * kDecTileN + ch;
            // (d) fp16 outlier product of the owned tile, ascending j, while the
            // weights stream: the weight value of outlier j is the kept fp16 row
            // or the dequantised int8 row
            float o[16];
#pragma unroll
            for (int m = 0; m < 16; ++m) o[m] = 0.0f;
            const float cav = (owner && n < N) ? p.ca[n] : 0.0f;
            if (owner && n < N) {
                const int n_fast = min(n_eff, kDecSmemOutliers);
#pragma unroll 4
                for (int j = 0; j < n_fast; ++j) {
                    const int slot = soslot[j];
                    float w;
                    if (slot >= 0) {
                        w = dec_half_to_float(p.w_keep[(size_t)slot * N + n]);
                    } else {
                        const float tq = __fmul_rn((float)p.wq[(size_t)n * K + slist[j]], cav);
                        w = __half2float(__float2half_rn(__fdiv_rn(tq, 127.0f)));
                    }
#pragma unroll
                    for (int m = 0; m < 16; ++m)
                        if (m < M) o[m] = fmaf(dec_half_to_float(sxo[j * 16 + m]), w, o[m]);
                }
                for (int j = n_fast; j < n_eff; ++j) {
                    const int k = slist[j];
                    const int slot = p.keep_slot[k];
                    float w;
                    if (slot >= 0) {
                        w = dec_half_to_float(p.w_keep[(size_t)slot * N + n]);
                    } else {
                        const float tq = __fmul_rn((float)p.wq[(size_t)n * K + k], cav);
                        w = __half2float(__float2half_rn(__fdiv_rn(tq, 127.0f)));
                    }
#pragma unroll
                    for (int m = 0; m < 16; ++m)
                        if (m < M) o[m] = fmaf(dec_half_to_float(Xg[(size_t)m * K + k]), w, o[m]);
                }
            }
            // partial sums of every tile of this CTA into this CTA's slot of the
            // tile owner's buffer (16-byte asynchronous stores, rows of one
            // channel together), completing on the owner's barrier
            if (has_acc && __all_sync(0xffffffffu, wait_bounded_sleep(tfull, 0, wctx))) {
                tc_fence_after();
                for (int j = 0; j < nt; ++j) {
                    uint32_t r[16];
                    tmem_ld16(tmem_base + ((uint32_t)(quad * 32) << 16) + (uint32_t)(32 * j), r);
                    tmem_wait_ld();
                    const uint32_t dst = map_to_rank(&sred[(size_t)(rank * kDecTileN + ch) * RS], (uint32_t)j);
                    const uint32_t mb = map_to_rank(red_done, (uint32_t)j);
                    st_async_v4(dst, r[0], r[1], r[2], r[3], mb);
                    st_async_v4(dst + 16, r[4], r[5], r[6], r[7], mb);
                    if (RS == 16) {
                        st_async_v4(dst + 32, r[8], r[9], r[10], r[11], mb);
                        st_async_v4(dst + 48, r[12], r[13], r[14], r[15], mb);
                    }
                }
            }
            if (owner && has_acc && __all_sync(0xffffffffu, wait_bounded_sleep(red_done, 0, wctx)) && n < N) {
                uint32_t sum[16];
#pragma unroll
                for (int m = 0; m < 16; ++m) sum[m] = 0u;
                for (int q = 0; q < CL; ++q) {
                    const uint4* src = reinterpret_cast<const uint4*>(&sred[(size_t)(q * kDecTileN + ch) * RS]);
#pragma unroll
                    for (int v = 0; v < 4; ++v) {
                        if (4 * v < RS) {
                            const uint4 t = src[v];
                            sum[4 * v] += t.x;
                            sum[4 * v + 1] += t.y;
                            sum[4 * v + 2] += t.z;
                            sum[4 * v + 3] += t.w;
                        }
                    }
                }
#pragma unroll
                for (int m = 0; m < 16; ++m) {
                    if (m < M) {
                        const int32_t acc = (int32_t)sum[m];
                        const float y = (float)acc * srs[m] * cav + o[m];
                        p.Y[(size_t)m * N + n] = __half_as_ushort(__float2half_rn(y));
                        if (p.acc_out) p.acc_out[(size_t)m * N + n] = acc;
                    }
                }
            }
        }
    }

    if (warp < 2) cluster_wait();  // the X-side warps waited before their first peer access
    // Every write into this CTA's shared memory (the peers' flag words, row
    // maxima and partial sums) completes on a barrier this CTA has waited for,
    // so it may leave without a closing cluster barrier; after a timeout a
    // peer's store may still be on its way here: let it land first.
    if (*abort_flag) settle_after_abort();
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, tmem_cols);
    }
}

}  // namespace i8mm
