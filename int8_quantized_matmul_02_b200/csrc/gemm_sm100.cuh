// The int8 GEMM of the LLM.int8() forward pass with its fused epilogue, on the
// fifth-generation tensor cores ("LLM.int8(): 8-bit Matrix Multiplication for
// Transformers at Scale", abstract: the 8-bit vector-wise product plus the
// 16-bit matmul over the outlier feature dimensions).
//
//   acc[m, n] = sum_k Xq[m, k] * Wq[n, k]            tcgen05.mma kind::i8, s32 in TMEM
//   v[m, n]   = acc * ra[m] * ca[n] / 127^2          epilogue pass 1, fp32 written back to TMEM
//   v[m, n]  += sum_j Xo[m, j] * Wo[n, j]            tcgen05.mma kind::f16 accumulating onto v
//   Y[m, n]   = fp16(v)                              epilogue pass 2, TMA store
//
// With no outlier column the epilogue is one pass straight from the s32
// accumulator.  Persistent CTAs (one per SM) walk 128 x 256 output tiles in
// M-grouped order; each CTA runs
//   warp 0     TMA producer: 128-byte-wide K slices of A (128 rows) and B (256
//              rows) into a 4-stage shared-memory ring (128-byte swizzle);
//              the outlier slices (64 fp16 = 128 bytes) use the same ring;
//   warp 1     TMEM allocation (512 columns = two 256-column accumulators) and
//              the single issuing thread of the MMAs;
//   warps 2-5  epilogue, one TMEM lane quadrant (32 rows) each, staging fp16
//              rows in a swizzled per-warp buffer stored by TMA.
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "sm100_ptx.cuh"

namespace i8mm {

struct GemmParams {
    int M, N, K;
    int num_m_blocks, num_n_blocks, num_tiles, group_m;
    int kb_int8;                   // ceil(K / 128)
    const int32_t* n_outliers;     // device count from the quantiser
    int cap;                       // outlier capacity of the workspace
    const float* ra;               // M
    const float* ca;               // N
    int32_t* acc_out;              // optional M x N
    int* status;
    uint64_t wait_limit_ns;
    uint32_t test_flags;           // bit 0: never signal the first tile's accumulator (timeout test)
};

constexpr int kGemmBM = 128;
constexpr int kGemmBN = 256;
constexpr int kGemmStages = 4;
constexpr int kGemmABytes = kGemmBM * 128;                  // 16 KB
constexpr int kGemmBBytes = kGemmBN * 128;                  // 32 KB
constexpr int kGemmStageBytes = kGemmABytes + kGemmBBytes;  // 48 KB
constexpr int kGemmEpiBufBytes = 32 * 128;                  // 32 rows x 64 fp16
constexpr int kGemmThreads = 192;
constexpr int kGemmSmemBytes =
    1024 /*align slack*/ + kGemmStages * kGemmStageBytes + 4 * 2 * kGemmEpiBufBytes + 256 /*barriers*/;
constexpr uint64_t kDrainLimitNs = 50ull * 1000 * 1000;

__device__ __forceinline__ void gemm_tile_coords(const GemmParams& p, int tile, int& mb, int& nb) {
    const int group_size = p.group_m * p.num_n_blocks;
    const int g = tile / group_size;
    const int first_m = g * p.group_m;
    const int gm = min(p.group_m, p.num_m_blocks - first_m);
    const int local = tile - g * group_size;
    mb = first_m + local % gm;
    nb = local / gm;
}

__device__ __forceinline__ uint32_t pack_half2(float a, float b) {
    return (uint32_t)__half_as_ushort(__float2half_rn(a)) | ((uint32_t)__half_as_ushort(__float2half_rn(b)) << 16);
}

// ca[col .. col+32) (zero past N; N is a multiple of 16) as 8 vector loads
// that every lane of the warp shares.
__device__ __forceinline__ void load_ca32(const float* __restrict__ ca, int col, int N, float (&out)[32]) {
#pragma unroll
    for (int i = 0; i < 32; i += 4) {
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        if (col + i < N) v = __ldg(reinterpret_cast<const float4*>(ca + col + i));
        out[i] = v.x;
        out[i + 1] = v.y;
        out[i + 2] = v.z;
        out[i + 3] = v.w;
    }
}

// Convert 32 fp32 values (one row, 32 consecutive columns) to fp16 and put
// them in the row's 128-byte line of the swizzled staging buffer (chunks
// 4*half32 .. 4*half32+3 of the line).
__device__ __forceinline__ void stage_row32(uint8_t* buf, int row, int half32, const float (&v)[32]) {
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        uint4 w;
        w.x = pack_half2(v[8 * c + 0], v[8 * c + 1]);
        w.y = pack_half2(v[8 * c + 2], v[8 * c + 3]);
        w.z = pack_half2(v[8 * c + 4], v[8 * c + 5]);
        w.w = pack_half2(v[8 * c + 6], v[8 * c + 7]);
        const int chunk = half32 * 4 + c;
        *reinterpret_cast<uint4*>(buf + row * 128 + ((chunk ^ (row & 7)) << 4)) = w;
    }
}

template <bool kWriteAcc>
__global__ void __launch_bounds__(kGemmThreads, 1)
    k_gemm_int8_sm100(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                      const __grid_constant__ CUtensorMap tm_xo, const __grid_constant__ CUtensorMap tm_wo,
                      const __grid_constant__ CUtensorMap tm_y, const GemmParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* ring = smem;
    uint8_t* epi = smem + kGemmStages * kGemmStageBytes;
    uint64_t* bars = reinterpret_cast<uint64_t*>(epi + 4 * 2 * kGemmEpiBufBytes);
    uint64_t* full = bars;                       // [stages]
    uint64_t* empty = bars + kGemmStages;        // [stages]
    uint64_t* tfull = bars + 2 * kGemmStages;    // [2] int8 accumulation done
    uint64_t* tscaled = tfull + 2;               // [2] epilogue wrote fp32 back
    uint64_t* tfull2 = tfull + 4;                // [2] outlier accumulation done
    uint64_t* tempty = tfull + 6;                // [2] epilogue drained the accumulator
    uint64_t* drain = tfull + 8;                 // [1]
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    WaitCtx wctx{abort_flag, p.status, p.wait_limit_ns};

    if (threadIdx.x == 0) {
        for (int s = 0; s < kGemmStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&tfull[a], 1);
            mbar_init(&tscaled[a], 4);
            mbar_init(&tfull2[a], 1);
            mbar_init(&tempty[a], 4);
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
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    pdl_wait();  // Xq, Xo, Wo, ra and the outlier count come from earlier kernels
    const int n_eff = min(*p.n_outliers, p.cap);
    const int n_ob = (n_eff + 63) / 64;  // outlier K slices of 64 fp16

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (elect_one()) {
            const uint64_t pol_a = policy_evict_last();
            const uint64_t pol_b = policy_evict_first();
            int stage = 0;
            uint32_t phase = 0;
            uint32_t armed = 0, armed_par = 0;  // per stage: a load was issued / its parity
            bool ok = true;
            for (int tile = blockIdx.x; tile < p.num_tiles && ok; tile += gridDim.x) {
                int mb, nb;
                gemm_tile_coords(p, tile, mb, nb);
                const int nsl = p.kb_int8 + n_ob;
                for (int sl = 0; sl < nsl; ++sl) {
                    if (!wait_bounded(&empty[stage], phase ^ 1, wctx)) {
                        ok = false;
                        break;
                    }
                    uint8_t* sa = ring + stage * kGemmStageBytes;
                    uint8_t* sb = sa + kGemmABytes;
                    mbar_arrive_expect_tx(&full[stage], kGemmStageBytes);
                    if (sl < p.kb_int8) {
                        tma_load_2d(sa, &tm_a, &full[stage], sl * 128, mb * kGemmBM, pol_a);
                        tma_load_2d(sb, &tm_b, &full[stage], sl * 128, nb * kGemmBN, pol_b);
                    } else {
                        const int ob = sl - p.kb_int8;
                        tma_load_2d(sa, &tm_xo, &full[stage], ob * 64, mb * kGemmBM, pol_a);
                        tma_load_2d(sb, &tm_wo, &full[stage], ob * 64, nb * kGemmBN, pol_b);
                    }
                    armed |= 1u << stage;
                    armed_par = (armed_par & ~(1u << stage)) | (phase << stage);
                    if (++stage == kGemmStages) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
            }
            // never leave with a copy in flight into this CTA's shared memory
            for (int s = 0; s < kGemmStages; ++s)
                if (armed & (1u << s)) wait_drain(&full[s], (armed_par >> s) & 1u, kDrainLimitNs);
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (elect_one()) {
            const uint32_t id_i8 = idesc_s8_s32(kGemmBM, kGemmBN);
            const uint32_t id_f16 = idesc_f16_f32(kGemmBM, kGemmBN);
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            bool ok = true, issued = false;
            for (int tile = blockIdx.x; tile < p.num_tiles && ok; tile += gridDim.x) {
                if (!wait_bounded(&tempty[acc], acc_phase ^ 1, wctx)) break;
                tc_fence_after();
                const uint32_t d = tmem_base + (uint32_t)(acc * kGemmBN);
                for (int kb = 0; kb < p.kb_int8; ++kb) {
                    if (!wait_bounded(&full[stage], phase, wctx)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sa = smem_u32(ring + stage * kGemmStageBytes);
                    const uint32_t sb = sa + kGemmABytes;
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        mma_s8(d, sdesc_k128sw(sa + 32 * k), sdesc_k128sw(sb + 32 * k), id_i8, (kb | k) != 0);
                    issued = true;
                    tc_commit(&empty[stage]);
                    if (++stage == kGemmStages) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
                if (!ok) break;
                if (!((p.test_flags & 1u) && tile == (int)blockIdx.x)) tc_commit(&tfull[acc]);
                if (n_ob > 0) {
                    // the epilogue turns the s32 sums into scaled fp32 in place
                    if (!wait_bounded(&tscaled[acc], acc_phase, wctx)) break;
                    tc_fence_after();
                    for (int ob = 0; ob < n_ob; ++ob) {
                        if (!wait_bounded(&full[stage], phase, wctx)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t sa = smem_u32(ring + stage * kGemmStageBytes);
                        const uint32_t sb = sa + kGemmABytes;
#pragma unroll
                        for (int k = 0; k < 4; ++k)
                            mma_f16(d, sdesc_k128sw(sa + 32 * k), sdesc_k128sw(sb + 32 * k), id_f16, 1u);
                        tc_commit(&empty[stage]);
                        if (++stage == kGemmStages) {
                            stage = 0;
                            phase ^= 1;
                        }
                    }
                    if (!ok) break;
                    tc_commit(&tfull2[acc]);
                }
                if (++acc == 2) {
                    acc = 0;
                    acc_phase ^= 1;
                }
            }
            if (issued) {  // every MMA of this CTA has retired before TMEM is freed
                tc_commit(drain);
                wait_drain(drain, 0, kDrainLimitNs);
            }
        }
    } else {
        // ------------------------------------------------ epilogue (warps 2..5)
        const int quad = warp & 3;  // TMEM lanes 32*quad .. 32*quad+31
        uint8_t* bufs = epi + quad * 2 * kGemmEpiBufBytes;
        int buf_i = 0;
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x) {
            int mb, nb;
            gemm_tile_coords(p, tile, mb, nb);
            const int row = mb * kGemmBM + quad * 32 + lane;
            const float rs = row < p.M ? __fdiv_rn(p.ra[row], 16129.0f) : 0.0f;
            const int col0 = nb * kGemmBN;
            if (!__all_sync(0xffffffffu, wait_bounded(&tfull[acc], acc_phase, wctx))) break;
            tc_fence_after();
            const uint32_t tacc = tmem_base + ((uint32_t)(quad * 32) << 16) + (uint32_t)(acc * kGemmBN);
            if (n_ob > 0) {
                // pass 1: s32 -> scaled fp32, written back for the outlier MMAs
#pragma unroll 1
                for (int c = 0; c < kGemmBN / 32; ++c) {
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
                if (lane == 0) mbar_arrive(&tscaled[acc]);
                if (!__all_sync(0xffffffffu, wait_bounded(&tfull2[acc], acc_phase, wctx))) break;
                tc_fence_after();
            }
            // final pass: 64 columns per TMA store
#pragma unroll 1
            for (int c = 0; c < kGemmBN / 64; ++c) {
                uint32_t r0[32], r1[32];
                tmem_ld32(tacc + c * 64, r0);
                tmem_ld32(tacc + c * 64 + 32, r1);
                tmem_wait_ld();
                if (c == kGemmBN / 64 - 1) {  // accumulator free for the next tile
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&tempty[acc]);
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
                    float c0[32], c1[32];
                    load_ca32(p.ca, col0 + c * 64, p.N, c0);
                    load_ca32(p.ca, col0 + c * 64 + 32, p.N, c1);
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        v0[i] = (float)(int32_t)r0[i] * rs * c0[i];
                        v1[i] = (float)(int32_t)r1[i] * rs * c1[i];
                    }
                }
                uint8_t* buf = bufs + buf_i * kGemmEpiBufBytes;
                if (lane == 0) bulk_wait_read<1>();  // the store that last used this buffer has read it
                __syncwarp();
                stage_row32(buf, lane, 0, v0);
                stage_row32(buf, lane, 1, v1);
                fence_proxy_async_smem();
                __syncwarp();
                const int sx = col0 + c * 64, sy = mb * kGemmBM + quad * 32;
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
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, 512);
    }
}

}  // namespace i8mm
