// Decode-shaped LLM.int8() forward (M <= 16 rows of X) in one kernel.
//
// At small M the product is bound by reading the int8 weight once ("memory
// loading is significantly more costly than computation", axolotl
// "llama3-model-quantization", "Impact of Precision and Parameter Count on
// Model Efficiency").  So every CTA streams its share of Wq through a deep TMA
// ring while it redoes the cheap X-side steps itself:
//   prologue (warps 2-7): outlier columns of X (a), row absmax and int8 codes
//     (b), written straight into shared memory in the tensor-core operand
//     layout (128-byte rows, 128-byte swizzle, 8-row groups);
//   warp 0: TMA producer of 128 (output channels) x 128 (K) int8 weight tiles;
//   warp 1: tcgen05.mma kind::i8 with the weight as the 128-row A operand and
//     the (padded) activation rows as the 16-column B operand ("swap AB"),
//     s32 accumulators in TMEM;
//   warps 4-7: read the accumulators and add them into an int32 partial-sum
//     buffer (exact in any order).  The work is split stream-K style: the
//     (tile, K-block) units are cut evenly over the persistent CTAs; the CTA
//     that completes a tile's K range applies ra * ca / 127^2, adds the fp16
//     outlier product (d) and writes fp16 Y, leaving the partial sums and the
//     tile counter at zero for the next call.
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
    int cap;                    // outlier capacity (list + overflow flag)
    const int8_t* wq;           // N x K (dequantised outlier rows that were not kept)
    const float* ca;
    const uint16_t* w_keep;
    const int32_t* keep_slot;
    uint16_t* Y;
    int32_t* partial;           // 16 x N int32, zero on entry and on exit
    int32_t* counters;          // 4 per tile (one per 32-column quadrant), zero on entry and on exit
    int32_t* acc_out;           // optional M x N
    int32_t* idx_out;           // workspace: outlier list
    int32_t* n_out;             // workspace: outlier count
    float* ra_out;              // workspace: M
    int8_t* xq_out;             // workspace: M x K
    int* status;
    uint64_t wait_limit_ns;
    uint32_t test_flags;        // bit 0: never signal that Xq is ready (timeout test)
    int num_tiles, kb_per_tile, stages, groups;  // groups = ceil(M / 8)
    uint32_t off_xq, off_mask, off_pre, off_list, off_bars;  // shared-memory offsets
};

constexpr int kDecThreads = 256;
constexpr int kDecTileN = 128;
constexpr int kDecStageBytes = kDecTileN * 128;  // 16 KB

// Byte offset of Xq[m, k] inside the shared B operand: K-block kb = k/128 holds
// `groups` 8-row atoms of 1024 bytes; in an atom row r = m%8 is a 128-byte
// line whose 16-byte chunks are XOR-swizzled with r.
__device__ __forceinline__ uint32_t dec_xq_off(int m, int k, int groups) {
    const int kb = k >> 7, g = m >> 3, r = m & 7, c = (k & 127) >> 4;
    return (uint32_t)(((kb * groups + g) << 10) + (r << 7) + ((c ^ r) << 4) + (k & 15));
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
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + p.off_bars);
    uint64_t* full = bars;
    uint64_t* empty = bars + p.stages;
    uint64_t* tfull = bars + 2 * p.stages;  // [2]
    uint64_t* tempty = tfull + 2;           // [2]
    uint64_t* xq_ready = tfull + 4;
    uint64_t* drain = tfull + 5;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tfull + 6);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    unsigned* sra_bits = reinterpret_cast<unsigned*>(tmem_slot + 2);  // [16]
    int* sflag = reinterpret_cast<int*>(tmem_slot + 18);              // [1]: total outliers

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int M = p.M, K = p.K, N = p.N;
    const int nw = (K + 31) / 32;
    WaitCtx wctx{abort_flag, p.status, p.wait_limit_ns};

    // stream-K share of this CTA over the (tile, K-block) units
    const long long U = (long long)p.num_tiles * p.kb_per_tile;
    const int u0 = (int)(U * blockIdx.x / gridDim.x);
    const int u1 = (int)(U * (blockIdx.x + 1) / gridDim.x);

    if (threadIdx.x == 0) {
        for (int s = 0; s < p.stages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&tfull[a], 1);
            mbar_init(&tempty[a], 4);
        }
        mbar_init(xq_ready, 1);
        mbar_init(drain, 1);
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
    const uint32_t tmem_base = *tmem_slot;
    pdl_launch_dependents();

    if (warp == 0) {
        // ------------------------------------------------ weight stream (needs nothing from earlier kernels)
        if (elect_one()) {
            const uint64_t pol = policy_evict_first();
            int stage = 0;
            uint32_t phase = 0, armed = 0, armed_par = 0;
            for (int u = u0; u < u1; ++u) {
                if (!wait_bounded(&empty[stage], phase ^ 1, wctx)) break;
                const int t = u / p.kb_per_tile, kb = u - t * p.kb_per_tile;
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
            int stage = 0, acc = 0;
            uint32_t phase = 0, acc_phase = 0;
            bool issued = false, ok = wait_bounded(xq_ready, 0, wctx);
            tc_fence_after();
            int u = u0;
            while (ok && u < u1) {
                const int t = u / p.kb_per_tile;
                const int seg_end = min(u1, (t + 1) * p.kb_per_tile);
                if (!wait_bounded(&tempty[acc], acc_phase ^ 1, wctx)) break;
                tc_fence_after();
                const uint32_t d = tmem_base + (uint32_t)(acc * 16);
                for (int v = u; v < seg_end; ++v) {
                    if (!wait_bounded(&full[stage], phase, wctx)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const int kb = v - t * p.kb_per_tile;
                    const uint32_t sa = smem_u32(ring + stage * kDecStageBytes);
                    const uint32_t sb = sxq_addr + (uint32_t)(kb * p.groups * 1024);
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        mma_s8(d, sdesc_k128sw(sa + 32 * j), sdesc_k128sw(sb + 32 * j), idesc,
                               (v != u || j != 0) ? 1u : 0u);
                    issued = true;
                    tc_commit(&empty[stage]);
                    if (++stage == p.stages) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
                if (!ok) break;
                tc_commit(&tfull[acc]);
                if (++acc == 2) {
                    acc = 0;
                    acc_phase ^= 1;
                }
                u = seg_end;
            }
            if (issued) {
                tc_commit(drain);
                wait_drain(drain, 0, 50ull * 1000 * 1000);
            }
        }
    } else {
        // ------------------------------------------------ X-side steps (warps 2..7)
        const int pt = threadIdx.x - 64;  // 0..191
        constexpr int kPro = kDecThreads - 64;
        pdl_wait();  // X and the workspace belong to earlier work on the stream
        const int nchunk = K / 8;
        // (a) outlier columns: max over the rows of |x| >= thr
        for (int c = pt; c < nchunk; c += kPro) {
            uint32_t mx[4] = {0, 0, 0, 0};
            for (int m = 0; m < M; ++m) {
                uint4 v = __ldg(reinterpret_cast<const uint4*>(p.X + (size_t)m * K) + c);
                mx[0] = __vmaxu2(mx[0], abs_bits2(v.x));
                mx[1] = __vmaxu2(mx[1], abs_bits2(v.y));
                mx[2] = __vmaxu2(mx[2], abs_bits2(v.z));
                mx[3] = __vmaxu2(mx[3], abs_bits2(v.w));
            }
            uint32_t fl = 0;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                if (half_bits_to_float(mx[i] & 0xFFFF) >= p.thr) fl |= 1u << (2 * i);
                if (half_bits_to_float(mx[i] >> 16) >= p.thr) fl |= 1u << (2 * i + 1);
            }
            if (fl) atomicOr(&smask[c >> 2], fl << ((c & 3) * 8));
        }
        named_bar_sync(1, kPro);
        // row absmax over the non-outlier columns (all prologue warps) and the
        // slot prefix of the outlier list (warp 2, after its share)
        {
            uint32_t rmax[16];
#pragma unroll
            for (int m = 0; m < 16; ++m) rmax[m] = 0;
            for (int c = pt; c < nchunk; c += kPro) {
#pragma unroll
                for (int m = 0; m < 16; ++m)
                    if (m < M)
                        rmax[m] = max(rmax[m], chunk_inlier_absmax(
                                                   __ldg(reinterpret_cast<const uint4*>(p.X + (size_t)m * K) + c),
                                                   smask, c));
            }
#pragma unroll
            for (int m = 0; m < 16; ++m) {
                if (m < M) {
                    const uint32_t r = __reduce_max_sync(0xffffffffu, rmax[m]);
                    if (lane == 0 && r) atomicMax(&sra_bits[m], r);
                }
            }
        }
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
        }
        named_bar_sync(1, kPro);
        const int total = sflag[0];
        const int n_eff = min(total, p.cap);
        // outlier list (ascending) into shared memory; CTA 0 also publishes it
        for (int w = pt; w < nw; w += kPro) {
            uint32_t word = smask[w];
            int s = spre[w];
            while (word) {
                const int b = __ffs(word) - 1;
                if (s < n_eff) {
                    slist[s] = (uint16_t)(w * 32 + b);
                    if (blockIdx.x == 0) p.idx_out[s] = w * 32 + b;
                }
                ++s;
                word &= word - 1;
            }
        }
        if (blockIdx.x == 0 && pt == 0) {
            *p.n_out = total;
            if (total > p.cap) atomicOr(p.status, kStatusOverflow);
        }
        // (b) int8 codes into the shared B operand: one 16-column chunk per step
        const int n16 = K / 16;
        for (int e = pt; e < M * n16; e += kPro) {
            const int m = e / n16, c16 = e - m * n16;
            const float rmax = half_bits_to_float(sra_bits[m]);
            const float scale = rmax > 0.0f ? __fdiv_rn(127.0f, rmax) : 0.0f;
            const uint4* src = reinterpret_cast<const uint4*>(p.X + (size_t)m * K) + 2 * c16;
            const uint2 q0 = quant_chunk(__ldg(src), smask, spre, 2 * c16, rmax, scale, 0, nullptr);
            const uint2 q1 = quant_chunk(__ldg(src + 1), smask, spre, 2 * c16 + 1, rmax, scale, 0, nullptr);
            const uint4 q = make_uint4(q0.x, q0.y, q1.x, q1.y);
            *reinterpret_cast<uint4*>(sxq + dec_xq_off(m, c16 * 16, p.groups)) = q;
            if (blockIdx.x == 0) *reinterpret_cast<uint4*>(p.xq_out + (size_t)m * K + c16 * 16) = q;
        }
        if (blockIdx.x == 0 && pt < M) p.ra_out[pt] = half_bits_to_float(sra_bits[pt]);
        fence_proxy_async_smem();
        named_bar_sync(1, kPro);
        if (pt == 0 && !(p.test_flags & 1u)) mbar_arrive(xq_ready);

        if (warp >= 4) {
            // ------------------------------------------------ epilogue (warps 4..7)
            const int quad = warp & 3;
            int acc = 0;
            uint32_t acc_phase = 0;
            int u = u0;
            while (u < u1) {
                const int t = u / p.kb_per_tile;
                const int seg_end = min(u1, (t + 1) * p.kb_per_tile);
                const int nunits = seg_end - u;
                if (!__all_sync(0xffffffffu, wait_bounded(&tfull[acc], acc_phase, wctx))) break;
                tc_fence_after();
                uint32_t r[16];
                tmem_ld16(tmem_base + ((uint32_t)(quad * 32) << 16) + (uint32_t)(acc * 16), r);
                tmem_wait_ld();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&tempty[acc]);
                if (++acc == 2) {
                    acc = 0;
                    acc_phase ^= 1;
                }
                const int n = t * kDecTileN + quad * 32 + lane;
                // Split-K completion is tracked per (tile, 32-column quadrant),
                // so each warp decides on its own columns with no block barrier.
                bool last = true;  // this CTA owns the whole K range of the tile
                if (nunits != p.kb_per_tile) {
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
                    last = (old + nunits == p.kb_per_tile);
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
                    float o[16];
#pragma unroll
                    for (int m = 0; m < 16; ++m) o[m] = 0.0f;
                    for (int j = 0; j < n_eff; ++j) {  // (d) fp16 outlier product, ascending j
                        const int k = slist[j];
                        const int slot = p.keep_slot[k];
                        float w;
                        if (slot >= 0) {
                            w = half_bits_to_float(p.w_keep[(size_t)slot * N + n]);
                        } else {
                            const float tq = __fmul_rn((float)p.wq[(size_t)n * K + k], p.ca[n]);
                            w = __half2float(__float2half_rn(__fdiv_rn(tq, 127.0f)));
                        }
#pragma unroll
                        for (int m = 0; m < 16; ++m)
                            if (m < M) o[m] = fmaf(half_bits_to_float(p.X[(size_t)m * K + k]), w, o[m]);
                    }
                    const float cav = p.ca[n];
#pragma unroll
                    for (int m = 0; m < 16; ++m) {
                        if (m < M) {
                            const float rs = __fdiv_rn(half_bits_to_float(sra_bits[m]), 16129.0f);
                            const float y = (float)(int32_t)r[m] * rs * cav + o[m];
                            p.Y[(size_t)m * N + n] = __half_as_ushort(__float2half_rn(y));
                            if (p.acc_out) p.acc_out[(size_t)m * N + n] = (int32_t)r[m];
                        }
                    }
                }
                u = seg_end;
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, 32);
    }
}

}  // namespace i8mm
