// Group-wise int8 GEMM on SM pairs (cta_group::2): the vector-wise product
// with one normalisation constant per row and group of G consecutive k on
// the X side and per column and group on the W side, the granularity of nuQmm
// and ZeroQuant (scite report for nuQmm, citing snippets: group-wise is finer
// than LLM.int8()'s vector-wise; its GPTQ snippet quantises groups of G
// consecutive weights independently).  The outlier decomposition stays as it
// is: outlier columns are zero in the int8 operand and go through the fp16
// product.
//
//   acc_g[m, n] = sum_{k in group g} Xq[m, k] * Wq[n, k]    tcgen05 kind::i8, s32 in TMEM
//   v[m, n]     = sum_g ((float(acc_g) * ra[m,g]) * ca[g,n]) / 127^2   fp32, ascending g
//   v[m, n]    += sum_j Xo[m, j] * Wo[n, j]                 tcgen05 kind::f16 onto v in TMEM
//   Y[m, n]     = fp16(v)
//
// The accumulation of a group ends in one of two s32 TMEM accumulators; while
// the tensor cores fill the other with the next group, the epilogue drains
// it, applies the group's constants and adds the result to the running fp32
// sum, which also lives in TMEM (columns 256-383).  The running sum uses the
// same operations in the same order as the definition, so before the outlier
// product it is exact to the bit.  The pair tile is 256 x 128 (each CTA 128
// rows; each CTA stages its 128 rows of A and 64 rows of B per 128-byte K
// slice), persistent CTA pairs walk the tiles in M-grouped order.
//   warp 0     TMA producer (completion counted on the even CTA's barrier);
//   warp 1     TMEM allocation (pair-wide, 512 columns) and, in the even CTA,
//              the MMA issuer;
//   warps 2-9  epilogue: warp w takes TMEM lane quadrant w % 4 (32 rows) and
//              column half (w - 2) / 4 (64 columns).
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "gemm_sm100.cuh"
#include "sm100_ptx.cuh"

namespace i8mm {

struct GroupedParams {
    GemmParams g;          // M, N, K, raster, kb_int8, outlier count, status, waits (g.ra / g.ca unused)
    int G, ng;             // group size (a multiple of 128 dividing K), groups
    const float* ra;       // M x ng: ra[m * ng + g]
    const float* ca;       // ng x N: ca[g * N + n]
    int32_t* acc_out;      // optional M x N x ng: acc_out[(m * N + n) * ng + g]
};

constexpr int kGGBM = 256;                         // rows of the pair tile (128 per CTA)
constexpr int kGGBN = 128;
constexpr int kGGStages = 6;
constexpr int kGGABytes = 128 * 128;               // this CTA's A rows, one 128-byte K slice
constexpr int kGGBBytes = 64 * 128;                // this CTA's B rows
constexpr int kGGStageBytes = kGGABytes + kGGBBytes;  // 24 KB
constexpr int kGGEpiWarps = 8;
constexpr int kGGThreads = 64 + 32 * kGGEpiWarps;  // 320
constexpr int kGGSmemBytes = 1024 + kGGStages * kGGStageBytes + kGGEpiWarps * 2 * kGemmEpiBufBytes + 256;
constexpr uint32_t kGGSumCol = 256;                // running fp32 sums; accumulators at 0 and 128

template <bool kWriteAcc>
__global__ void __launch_bounds__(kGGThreads, 1)
    k_gemm_int8_grouped(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                        const __grid_constant__ CUtensorMap tm_xo, const __grid_constant__ CUtensorMap tm_wo,
                        const __grid_constant__ CUtensorMap tm_y, const GroupedParams gp) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* ring = smem;
    uint8_t* epi = smem + kGGStages * kGGStageBytes;
    uint64_t* bars = reinterpret_cast<uint64_t*>(epi + kGGEpiWarps * 2 * kGemmEpiBufBytes);
    uint64_t* full = bars;                    // [stages] even CTA: both CTAs' bytes
    uint64_t* empty = bars + kGGStages;       // [stages] each CTA: its stage is free
    uint64_t* tfull = bars + 2 * kGGStages;   // [2] each CTA: a group's int8 sums are ready
    uint64_t* tempty = tfull + 2;             // [2] even CTA: both epilogues drained the accumulator
    uint64_t* tscaled = tfull + 4;            // [1] even CTA: both epilogues wrote the tile's fp32 sums
    uint64_t* tfull2 = tfull + 5;             // [1] each CTA: the outlier product is added
    uint64_t* drain = tfull + 6;              // [1]
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const GemmParams& p = gp.g;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();  // 0 = the CTA that issues the MMAs
    const int cid = blockIdx.x >> 1, ncl = gridDim.x >> 1;
    const int ng = gp.ng, kbg = gp.G / 128;   // K slices per group
    WaitCtx wctx{abort_flag, p.status, p.wait_limit_ns};

    if (threadIdx.x == 0) {
        for (int s = 0; s < kGGStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&tfull[a], 1);
            mbar_init(&tempty[a], 2 * kGGEpiWarps);
        }
        mbar_init(tscaled, 2 * kGGEpiWarps);
        mbar_init(tfull2, 1);
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
        prefetch_tmap(&tm_a);
        prefetch_tmap(&tm_b);
        prefetch_tmap(&tm_xo);
        prefetch_tmap(&tm_wo);
        prefetch_tmap(&tm_y);
    }
    if (warp == 1) {
        tmem_alloc_pair(tmem_slot, 512);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync_all();  // both CTAs' barriers and TMEM are ready
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    pdl_wait();  // Xq, Xo, Wo, ra and the outlier count come from earlier kernels
    const int n_eff = min(*p.n_outliers, p.cap);
    const int n_ob = (n_eff + 63) / 64;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer (both CTAs)
        if (elect_one()) {
            const uint64_t pol_a = policy_evict_last();
            const uint64_t pol_b = policy_evict_first();
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (int tile = cid; tile < p.num_tiles && ok; tile += ncl) {
                int mb, nb;
                gemm_tile_coords(p, tile, mb, nb);
                const int row_a = mb * kGGBM + (int)rank * 128;
                const int row_b = nb * kGGBN + (int)rank * 64;
                const int nsl = p.kb_int8 + n_ob;
                for (int sl = 0; sl < nsl; ++sl) {
                    if (!wait_bounded_cluster(&empty[stage], phase ^ 1, wctx)) {
                        ok = false;
                        break;
                    }
                    uint8_t* sa = ring + stage * kGGStageBytes;
                    uint8_t* sb = sa + kGGABytes;
                    if (rank == 0) mbar_arrive_expect_tx(&full[stage], 2 * kGGStageBytes);
                    const uint32_t fbar = map_to_rank(&full[stage], 0);
                    if (sl < p.kb_int8) {
                        tma_load_2d_pair(sa, &tm_a, fbar, sl * 128, row_a, pol_a);
                        tma_load_2d_pair(sb, &tm_b, fbar, sl * 128, row_b, pol_b);
                    } else {
                        const int ob = sl - p.kb_int8;
                        tma_load_2d_pair(sa, &tm_xo, fbar, ob * 64, row_a, pol_a);
                        tma_load_2d_pair(sb, &tm_wo, fbar, ob * 64, row_b, pol_b);
                    }
                    if (++stage == kGGStages) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer (even CTA)
        if (rank == 0 && elect_one()) {
            const uint32_t id_i8 = idesc_s8_s32(kGGBM, kGGBN);
            const uint32_t id_f16 = idesc_f16_f32(kGGBM, kGGBN);
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0, tile_phase = 0;
            bool ok = true, issued = false;
            for (int tile = cid; tile < p.num_tiles && ok; tile += ncl) {
                for (int g = 0; g < ng && ok; ++g) {
                    if (!wait_bounded_cluster(&tempty[acc], acc_phase ^ 1, wctx)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t d = tmem_base + (uint32_t)(acc * kGGBN);
                    for (int kb = g * kbg; kb < (g + 1) * kbg; ++kb) {
                        if (!wait_bounded(&full[stage], phase, wctx)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t sa = smem_u32(ring + stage * kGGStageBytes);
                        const uint32_t sb = sa + kGGABytes;
#pragma unroll
                        for (int k = 0; k < 4; ++k)
                            mma_s8_2sm(d, sdesc_k128sw(sa + 32 * k), sdesc_k128sw(sb + 32 * k), id_i8,
                                       (kb != g * kbg || k != 0) ? 1u : 0u);
                        issued = true;
                        tc_commit_pair(&empty[stage]);
                        if (++stage == kGGStages) {
                            stage = 0;
                            phase ^= 1;
                        }
                    }
                    if (!ok) break;
                    if (!((p.test_flags & 1u) && tile == cid && g == 0)) tc_commit_pair(&tfull[acc]);
                    if (++acc == 2) {
                        acc = 0;
                        acc_phase ^= 1;
                    }
                }
                if (!ok) break;
                if (n_ob > 0) {
                    // the outlier product accumulates onto the tile's fp32 sums
                    if (!wait_bounded_cluster(tscaled, tile_phase, wctx)) break;
                    tc_fence_after();
                    const uint32_t d = tmem_base + kGGSumCol;
                    for (int ob = 0; ob < n_ob; ++ob) {
                        if (!wait_bounded(&full[stage], phase, wctx)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t sa = smem_u32(ring + stage * kGGStageBytes);
                        const uint32_t sb = sa + kGGABytes;
#pragma unroll
                        for (int k = 0; k < 4; ++k)
                            mma_f16_2sm(d, sdesc_k128sw(sa + 32 * k), sdesc_k128sw(sb + 32 * k), id_f16, 1u);
                        tc_commit_pair(&empty[stage]);
                        if (++stage == kGGStages) {
                            stage = 0;
                            phase ^= 1;
                        }
                    }
                    if (!ok) break;
                    tc_commit_pair(tfull2);
                    tile_phase ^= 1;
                }
            }
            if (issued) {  // every pair MMA has retired before TMEM is freed
                tc_commit_pair(drain);
                wait_drain(drain, 0, kDrainLimitNs);
            }
        }
    } else {
        // ------------------------------------------------ epilogue (warps 2..9, both CTAs)
        const int ew = warp - 2;
        const int quad = warp & 3, half = ew >> 2;  // lane quadrant, 64-column half
        uint8_t* bufs = epi + ew * 2 * kGemmEpiBufBytes;
        const uint32_t tempty_even[2] = {map_to_rank(&tempty[0], 0), map_to_rank(&tempty[1], 0)};
        const uint32_t tscaled_even = map_to_rank(tscaled, 0);
        int buf_i = 0;
        int acc = 0;
        uint32_t acc_phase = 0, tile_phase = 0;
        bool ok = true;
        for (int tile = cid; tile < p.num_tiles && ok; tile += ncl) {
            int mb, nb;
            gemm_tile_coords(p, tile, mb, nb);
            const int row0 = mb * kGGBM + (int)rank * 128 + quad * 32;
            const int row = row0 + lane;
            const int colw = nb * kGGBN + half * 64;  // this warp's first column
            const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
            const uint32_t tsum = tmem_base + lane_off + kGGSumCol + (uint32_t)(half * 64);
            for (int g = 0; g < ng; ++g) {
                if (!__all_sync(0xffffffffu, wait_bounded_cluster(&tfull[acc], acc_phase, wctx))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t tacc = tmem_base + lane_off + (uint32_t)(acc * kGGBN + half * 64);
                const float rg = row < p.M ? gp.ra[(size_t)row * ng + g] : 0.0f;
                const bool last = g == ng - 1;
#pragma unroll 1
                for (int c = 0; c < 2; ++c) {
                    uint32_t r[32], sv[32];
                    tmem_ld32(tacc + 32 * c, r);
                    if (g > 0) tmem_ld32(tsum + 32 * c, sv);
                    tmem_wait_ld();
                    const int col = colw + 32 * c;
                    if (kWriteAcc && row < p.M) {
#pragma unroll 4
                        for (int i = 0; i < 32; ++i)
                            if (col + i < p.N) gp.acc_out[((size_t)row * p.N + col + i) * ng + g] = (int32_t)r[i];
                    }
                    float cav[32];
                    load_ca32(gp.ca + (size_t)g * p.N, col, p.N, cav);
                    float v[32];
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        float t = __fmul_rn(__fmul_rn((float)(int32_t)r[i], rg), cav[i]);
                        t = __fdiv_rn(t, 16129.0f);
                        v[i] = __fadd_rn(g > 0 ? __uint_as_float(sv[i]) : 0.0f, t);
                    }
                    if (last && n_ob == 0) {
                        // no outlier product: this is Y (v + 0 in the definition)
                        uint8_t* buf = bufs + buf_i * kGemmEpiBufBytes;
                        if (lane == 0) bulk_wait_read<1>();
                        __syncwarp();
                        float lo[32];
#pragma unroll
                        for (int i = 0; i < 32; ++i) lo[i] = __fadd_rn(v[i], 0.0f);
                        stage_row32(buf, lane, c & 1, lo);
                        if (c == 1) {
                            fence_proxy_async_smem();
                            __syncwarp();
                            if (lane == 0) {
                                if (colw < p.N && row0 < p.M) tma_store_2d(&tm_y, buf, colw, row0);
                                bulk_commit();
                            }
                            buf_i ^= 1;
                        }
                    } else {
                        uint32_t w[32];
#pragma unroll
                        for (int i = 0; i < 32; ++i) w[i] = __float_as_uint(v[i]);
                        tmem_st32(tsum + 32 * c, w);
                    }
                }
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive_cluster(tempty_even[acc]);                   // the accumulator is free
                    if (last && n_ob > 0) mbar_arrive_cluster(tscaled_even);  // the sums are in TMEM
                }
                if (++acc == 2) {
                    acc = 0;
                    acc_phase ^= 1;
                }
            }
            if (!ok) break;
            if (n_ob > 0) {
                if (!__all_sync(0xffffffffu, wait_bounded_cluster(tfull2, tile_phase, wctx))) break;
                tc_fence_after();
                tile_phase ^= 1;
                uint32_t r0[32], r1[32];
                tmem_ld32(tsum, r0);
                tmem_ld32(tsum + 32, r1);
                tmem_wait_ld();
                float v0[32], v1[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    v0[i] = __uint_as_float(r0[i]);
                    v1[i] = __uint_as_float(r1[i]);
                }
                uint8_t* buf = bufs + buf_i * kGemmEpiBufBytes;
                if (lane == 0) bulk_wait_read<1>();
                __syncwarp();
                stage_row32(buf, lane, 0, v0);
                stage_row32(buf, lane, 1, v1);
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    if (colw < p.N && row0 < p.M) tma_store_2d(&tm_y, buf, colw, row0);
                    bulk_commit();
                }
                buf_i ^= 1;
            }
        }
        if (lane == 0) bulk_wait_all<0>();
        __syncwarp();
    }

    if (threadIdx.x == 0 && *abort_flag) settle_after_abort();  // copies issued before the abort land first
    tc_fence_before();
    __syncthreads();
    cluster_sync_all();  // the even CTA's MMAs no longer read this CTA's shared memory or TMEM
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, 512);
    }
}

}  // namespace i8mm
