// The int8 GEMM of the LLM.int8() forward pass on SM pairs (cta_group::2).
//
// Same arithmetic as k_gemm_int8_sm100 (gemm_sm100.cuh): acc = Xq Wq^T on
// tcgen05 kind::i8 in TMEM, the scaled fp32 written back to TMEM, the fp16
// outlier slices accumulated onto it with kind::f16, fp16 Y stored by TMA.
// The tile is 256 x 256 and belongs to a cluster of two CTAs on two SMs:
// each CTA loads its 128 rows of A and its 128 rows of B per 128-byte K slice
// (32 KB per stage, 6 stages), the even CTA issues the pair-wide MMAs, and
// each CTA's TMEM holds its 128 output rows x 256 columns (two accumulator
// buffers of 256 columns).  Per SM this halves the B bytes staged and read
// per MMA compared with the single-SM 128 x 256 tile.
//   warp 0     TMA producer (both CTAs; completion counted on the even CTA's
//              "full" barrier);
//   warp 1     TMEM allocation (pair-wide) and, in the even CTA, the MMA issuer;
//   warps 2-5  epilogue of this CTA's rows.
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "gemm_sm100.cuh"
#include "sm100_ptx.cuh"

namespace i8mm {

constexpr int kG2BM = 256;                         // rows of the pair tile (128 per CTA)
constexpr int kG2BN = 256;
constexpr int kG2Stages = 6;
constexpr int kG2ABytes = 128 * 128;               // this CTA's A rows, one 128-byte K slice
constexpr int kG2BBytes = 128 * 128;               // this CTA's B rows
constexpr int kG2StageBytes = kG2ABytes + kG2BBytes;  // 32 KB
constexpr int kG2SmemBytes = 1024 + kG2Stages * kG2StageBytes + 4 * 2 * kGemmEpiBufBytes + 256;

__device__ __forceinline__ void g2_tile_coords(const GemmParams& p, int tile, int& mb, int& nb) {
    // p.num_m_blocks counts 256-row blocks here
    gemm_tile_coords(p, tile, mb, nb);
}

template <bool kWriteAcc>
__global__ void __launch_bounds__(kGemmThreads, 1)
    k_gemm_int8_2sm(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                    const __grid_constant__ CUtensorMap tm_xo, const __grid_constant__ CUtensorMap tm_wo,
                    const __grid_constant__ CUtensorMap tm_y, const GemmParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* ring = smem;
    uint8_t* epi = smem + kG2Stages * kG2StageBytes;
    uint64_t* bars = reinterpret_cast<uint64_t*>(epi + 4 * 2 * kGemmEpiBufBytes);
    uint64_t* full = bars;                    // [stages] even CTA: both CTAs' bytes
    uint64_t* empty = bars + kG2Stages;       // [stages] each CTA: its stage is free
    uint64_t* tfull = bars + 2 * kG2Stages;   // [2] each CTA: int8 sums ready
    uint64_t* tscaled = tfull + 2;            // [2] even CTA: both epilogues wrote fp32 back
    uint64_t* tfull2 = tfull + 4;             // [2] each CTA: outlier sums ready
    uint64_t* tempty = tfull + 6;             // [2] even CTA: both epilogues drained TMEM
    uint64_t* drain = tfull + 8;              // [1]
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();  // 0 = the CTA that issues the MMAs
    const int cid = blockIdx.x >> 1, ncl = gridDim.x >> 1;
    WaitCtx wctx{abort_flag, p.status, p.wait_limit_ns};

    if (threadIdx.x == 0) {
        for (int s = 0; s < kG2Stages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&tfull[a], 1);
            mbar_init(&tscaled[a], 8);
            mbar_init(&tfull2[a], 1);
            mbar_init(&tempty[a], 8);
        }
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
                g2_tile_coords(p, tile, mb, nb);
                const int row_a = mb * kG2BM + (int)rank * 128;
                const int row_b = nb * kG2BN + (int)rank * 128;
                const int nsl = p.kb_int8 + n_ob;
                for (int sl = 0; sl < nsl; ++sl) {
                    if (!wait_bounded_cluster(&empty[stage], phase ^ 1, wctx)) {
                        ok = false;
                        break;
                    }
                    uint8_t* sa = ring + stage * kG2StageBytes;
                    uint8_t* sb = sa + kG2ABytes;
                    if (rank == 0) mbar_arrive_expect_tx(&full[stage], 2 * kG2StageBytes);
                    const uint32_t fbar = map_to_rank(&full[stage], 0);
                    if (sl < p.kb_int8) {
                        tma_load_2d_pair(sa, &tm_a, fbar, sl * 128, row_a, pol_a);
                        tma_load_2d_pair(sb, &tm_b, fbar, sl * 128, row_b, pol_b);
                    } else {
                        const int ob = sl - p.kb_int8;
                        tma_load_2d_pair(sa, &tm_xo, fbar, ob * 64, row_a, pol_a);
                        tma_load_2d_pair(sb, &tm_wo, fbar, ob * 64, row_b, pol_b);
                    }
                    if (++stage == kG2Stages) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer (even CTA)
        if (rank == 0 && elect_one()) {
            const uint32_t id_i8 = idesc_s8_s32(kG2BM, kG2BN);
            const uint32_t id_f16 = idesc_f16_f32(kG2BM, kG2BN);
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            bool ok = true, issued = false;
            for (int tile = cid; tile < p.num_tiles && ok; tile += ncl) {
                if (!wait_bounded_cluster(&tempty[acc], acc_phase ^ 1, wctx)) break;
                tc_fence_after();
                const uint32_t d = tmem_base + (uint32_t)(acc * kG2BN);
                for (int kb = 0; kb < p.kb_int8; ++kb) {
                    if (!wait_bounded(&full[stage], phase, wctx)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sa = smem_u32(ring + stage * kG2StageBytes);
                    const uint32_t sb = sa + kG2ABytes;
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        mma_s8_2sm(d, sdesc_k128sw(sa + 32 * k), sdesc_k128sw(sb + 32 * k), id_i8, (kb | k) != 0);
                    issued = true;
                    tc_commit_pair(&empty[stage]);
                    if (++stage == kG2Stages) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
                if (!ok) break;
                if (!((p.test_flags & 1u) && tile == cid)) tc_commit_pair(&tfull[acc]);
                if (n_ob > 0) {
                    if (!wait_bounded_cluster(&tscaled[acc], acc_phase, wctx)) break;
                    tc_fence_after();
                    for (int ob = 0; ob < n_ob; ++ob) {
                        if (!wait_bounded(&full[stage], phase, wctx)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t sa = smem_u32(ring + stage * kG2StageBytes);
                        const uint32_t sb = sa + kG2ABytes;
#pragma unroll
                        for (int k = 0; k < 4; ++k)
                            mma_f16_2sm(d, sdesc_k128sw(sa + 32 * k), sdesc_k128sw(sb + 32 * k), id_f16, 1u);
                        tc_commit_pair(&empty[stage]);
                        if (++stage == kG2Stages) {
                            stage = 0;
                            phase ^= 1;
                        }
                    }
                    if (!ok) break;
                    tc_commit_pair(&tfull2[acc]);
                }
                if (++acc == 2) {
                    acc = 0;
                    acc_phase ^= 1;
                }
            }
            if (issued) {  // every pair MMA has retired before TMEM is freed
                tc_commit_pair(drain);
                wait_drain(drain, 0, kDrainLimitNs);
            }
        }
    } else {
        // ------------------------------------------------ epilogue (warps 2..5, both CTAs)
        const int quad = warp & 3;
        uint8_t* bufs = epi + quad * 2 * kGemmEpiBufBytes;
        const uint32_t tempty_even[2] = {map_to_rank(&tempty[0], 0), map_to_rank(&tempty[1], 0)};
        const uint32_t tscaled_even[2] = {map_to_rank(&tscaled[0], 0), map_to_rank(&tscaled[1], 0)};
        int buf_i = 0;
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int tile = cid; tile < p.num_tiles; tile += ncl) {
            int mb, nb;
            g2_tile_coords(p, tile, mb, nb);
            const int row0 = mb * kG2BM + (int)rank * 128 + quad * 32;
            const int row = row0 + lane;
            const float rs = row < p.M ? __fdiv_rn(p.ra[row], 16129.0f) : 0.0f;
            const int col0 = nb * kG2BN;
            if (!__all_sync(0xffffffffu, wait_bounded_cluster(&tfull[acc], acc_phase, wctx))) break;
            tc_fence_after();
            const uint32_t tacc = tmem_base + ((uint32_t)(quad * 32) << 16) + (uint32_t)(acc * kG2BN);
            if (n_ob > 0) {
#pragma unroll 1
                for (int c = 0; c < kG2BN / 32; ++c) {
                    uint32_t r[32];
                    tmem_ld32(tacc + c * 32, r);
                    tmem_wait_ld();
                    if (kWriteAcc && row < p.M) {
                        int32_t* dst = p.acc_out + (size_t)row * p.N + col0 + c * 32;
#pragma unroll
                        for (int i = 0; i < 32; i += 4)
                            if (col0 + c * 32 + i < p.N)
                                *reinterpret_cast<int4*>(dst + i) = make_int4(r[i], r[i + 1], r[i + 2], r[i + 3]);
                    }
                    float cav[32];
                    load_ca32(p.ca, col0 + c * 32, p.N, cav);
#pragma unroll
                    for (int i = 0; i < 32; ++i) r[i] = __float_as_uint((float)(int32_t)r[i] * rs * cav[i]);
                    tmem_st32(tacc + c * 32, r);
                }
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster(tscaled_even[acc]);
                if (!__all_sync(0xffffffffu, wait_bounded_cluster(&tfull2[acc], acc_phase, wctx))) break;
                tc_fence_after();
            }
#pragma unroll 1
            for (int c = 0; c < kG2BN / 64; ++c) {
                uint32_t r0[32], r1[32];
                tmem_ld32(tacc + c * 64, r0);
                tmem_ld32(tacc + c * 64 + 32, r1);
                tmem_wait_ld();
                if (c == kG2BN / 64 - 1) {  // accumulator free for the next tile
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive_cluster(tempty_even[acc]);
                }
                float v0[32], v1[32];
                if (n_ob > 0) {
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        v0[i] = __uint_as_float(r0[i]);
                        v1[i] = __uint_as_float(r1[i]);
                    }
                } else {
                    if (kWriteAcc && row < p.M) {
                        int32_t* dst = p.acc_out + (size_t)row * p.N + col0 + c * 64;
#pragma unroll
                        for (int i = 0; i < 32; i += 4) {
                            if (col0 + c * 64 + i < p.N)
                                *reinterpret_cast<int4*>(dst + i) = make_int4(r0[i], r0[i + 1], r0[i + 2], r0[i + 3]);
                            if (col0 + c * 64 + 32 + i < p.N)
                                *reinterpret_cast<int4*>(dst + 32 + i) =
                                    make_int4(r1[i], r1[i + 1], r1[i + 2], r1[i + 3]);
                        }
                    }
                    float c0v[32], c1v[32];
                    load_ca32(p.ca, col0 + c * 64, p.N, c0v);
                    load_ca32(p.ca, col0 + c * 64 + 32, p.N, c1v);
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        v0[i] = (float)(int32_t)r0[i] * rs * c0v[i];
                        v1[i] = (float)(int32_t)r1[i] * rs * c1v[i];
                    }
                }
                uint8_t* buf = bufs + buf_i * kGemmEpiBufBytes;
                if (lane == 0) bulk_wait_read<1>();
                __syncwarp();
                stage_row32(buf, lane, 0, v0);
                stage_row32(buf, lane, 1, v1);
                fence_proxy_async_smem();
                __syncwarp();
                const int sx = col0 + c * 64, sy = row0;
                if (lane == 0) {
                    if (sx < p.N && sy < p.M) tma_store_2d(&tm_y, buf, sx, sy);
                    bulk_commit();
                }
                buf_i ^= 1;
            }
            if (++acc == 2) {
                acc = 0;
                acc_phase ^= 1;
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
