// 4-bit weight-only product Y = X W' for decode-sized X (M <= 16 rows), and
// the one-time conversion of an fp16 weight to 4-bit codes.
//
// Method: weights get linear 4-bit codes q in [-7, 7] with one normalisation
// constant per output column and group of G consecutive k (the rule of the
// 8-bit codes with 7 in place of 127: absmax, scale = RN32(7/absmax),
// round half to even); X stays fp16.  Inference at small batch is bound by
// loading the weights, so half the bits per weight halve the bytes that set
// its time (video page "8-bit Methods for Efficient Deep Learning with Tim
// Dettmers", "4-Bit Inference"; axolotl "llama3-model-quantization", "Impact
// of Precision and Parameter Count on Model Efficiency").  Grouping G
// consecutive weights under one constant is the granularity the scite report
// for nuQmm quotes from GPTQ (group size 1024 there).
//
// What the kernel sums: y[m,n] = sum_g (absmax[n,g] / 7) * sum_{k in g}
// x[m,k] * q[n,k].  The inner sums run on the tensor cores (fp16 x fp16 with
// fp32 accumulation; q is a small integer, exact in fp16), one accumulator per
// 128 consecutive k, and each is scaled by its group's constant in fp32.  The
// weight w' = (q * absmax) / 7 is never formed, so the result differs from
// sum_k x * fp32(w') only by fp32 rounding.
//
// Packed layout of the codes (N rows of K/2 bytes, K contiguous): every
// 32-bit word holds the codes of 8 consecutive k as unsigned nibbles u = q + 8,
// in the order k0 -> bits 0-3, k0+1 -> 16-19, k0+2 -> 4-7, k0+3 -> 20-23,
// k0+4 -> 8-11, k0+5 -> 24-27, k0+6 -> 12-15, k0+7 -> 28-31, so that
// (word >> 4i) & 0x000F000F holds the pair (k0+2i, k0+2i+1) in its two 16-bit
// halves; OR-ing 0x6400 into a half gives the fp16 value 1024 + u, and
// subtracting 1032 leaves q exactly.
//
// Forward kernel: clusters of CL CTAs split K (CTA r owns the r-th K range of
// the cluster's tiles of 128 output columns) as the 8-bit decode kernel
// does; warp 0 streams 128 (columns) x 256 (k) boxes of packed codes through a
// TMA ring from launch on, warps 2-9 widen each half box (128 k) to fp16 and
// write it to tensor memory as the A operand (thread = output column =
// TMEM lane, two warps per lane quarter, one per 64 k; four such operands in
// flight), warp 1 issues tcgen05.mma kind::f16 with A from tensor memory
// and X (loaded once by TMA, 128-byte swizzled, K-major) as the 16-column B
// operand into one of sixteen fp32 accumulators, and warps 10-13 drain them
// four at a time (one wait and one 64-column load per four 128-k blocks, so
// that the drain's latency is paid once per four blocks), scale each by its
// group's constant and add them up per column; the partial sums of a
// tile then go to the tile's owner in the cluster (asynchronous stores into
// its shared memory), which adds them in a fixed order and writes fp16 Y.
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "sm100_ptx.cuh"

namespace i8mm {

// ------------------------------------------------------------------ conversion (one-time)

// absmax[n * ng + g] = max_{k in group g} |W[k, n]|; one thread per (g, n),
// n fastest (coalesced rows of W).
__global__ void __launch_bounds__(256) k_int4_absmax(const uint16_t* __restrict__ W, int K, int N, int G,
                                                     float* __restrict__ absmax) {
    const int ng = K / G;
    const long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (t >= (long long)ng * N) return;
    const int n = (int)(t % N), g = (int)(t / N);
    uint32_t m = 0u;  // non-negative fp16 bit patterns order like their values
    for (int k = g * G; k < (g + 1) * G; ++k) m = max(m, (uint32_t)(W[(size_t)k * N + n] & 0x7FFFu));
    absmax[(size_t)n * ng + g] = __half2float(__ushort_as_half((unsigned short)m));
}

// One 32-bit word of packed codes (8 consecutive k of column n) per thread,
// n fastest.  q = round_half_even(RN32(w * RN32(7 / absmax))) clamped to
// +-7 (0 when absmax is 0); nibble u = q + 8.
__global__ void __launch_bounds__(256) k_int4_pack(const uint16_t* __restrict__ W, int K, int N, int G,
                                                   const float* __restrict__ absmax, uint32_t* __restrict__ codes) {
    const int ng = K / G, k8n = K / 8;
    const long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (t >= (long long)k8n * N) return;
    const int n = (int)(t % N), k0 = (int)(t / N) * 8;
    const float a = absmax[(size_t)n * ng + k0 / G];
    const float s = a > 0.0f ? __fdiv_rn(7.0f, a) : 0.0f;
    // nibble position of k0 + i: low halfword for even i, high for odd, at 4 * (i / 2)
    uint32_t word = 0u;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const float w = __half2float(__ushort_as_half(W[(size_t)(k0 + i) * N + n]));
        float r = a > 0.0f ? rintf(__fmul_rn(w, s)) : 0.0f;
        r = fminf(fmaxf(r, -7.0f), 7.0f);
        const uint32_t u = (uint32_t)((int)r + 8);
        word |= u << ((i & 1) * 16 + (i >> 1) * 4);
    }
    codes[(size_t)n * k8n + k0 / 8] = word;
}

// ------------------------------------------------------------------ forward

struct Int4Params {
    const float* absmax;        // N x (K / G)
    uint16_t* Y;                // M x N
    int* status;                // device word (bit 0: timeout)
    uint64_t wait_limit_ns;
    uint32_t test_flags;        // bit 0: never signal that X is loaded (timeout test)
    int M, K, N, G;
    int num_tiles, kb_total;    // 128-column tiles, 256-k boxes
    int num_clusters, cluster, stages, xrows;  // xrows: rows of one X box (8 or 16)
    uint32_t tmem_cols;
    uint32_t off_x, off_red, off_bars;  // shared-memory offsets
};

constexpr int kI4Threads = 448;          // warp 0 TMA, 1 MMA, 2-9 widen, 10-13 accumulate
constexpr int kI4WidenWarps = 8;
constexpr int kI4TileN = 128;
constexpr int kI4BoxK = 256;             // k per packed box (128 bytes per row)
constexpr int kI4StageBytes = kI4TileN * 128;  // 16 KB
constexpr int kI4DSlots = 16;            // fp32 accumulators in TMEM (16 columns each)
constexpr int kI4DBatch = 4;             // accumulators drained per wait (64 columns, one load pair)
constexpr int kI4ASlots = 4;             // fp16 A operands in TMEM (64 columns = 128 k each)
constexpr uint32_t kI4AColBase = 0;
constexpr uint32_t kI4DColBase = 64 * kI4ASlots;
constexpr uint32_t kI4TmemCols = 512;    // the whole TMEM of the SM: one CTA per SM

__device__ __forceinline__ void i4_mma_f16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                              uint32_t accumulate) {
    const uint32_t z = 0;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, {%5, %5, %5, %5}, p;\n\t}\n" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(z)
        : "memory");
}

// fp16 pairs of the 8 codes in one packed word (see the layout above)
__device__ __forceinline__ void i4_widen(uint32_t w, uint32_t* out) {
    const __half2 off = __halves2half2(__ushort_as_half(0x6408u), __ushort_as_half(0x6408u));  // 1032
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t b = ((w >> (4 * i)) & 0x000F000Fu) | 0x64006400u;
        __half2 h;
        memcpy(&h, &b, 4);
        const __half2 q = __hsub2(h, off);
        memcpy(&out[i], &q, 4);
    }
}

__global__ void __launch_bounds__(kI4Threads, 1)
    k_int4_decode_sm100(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_x,
                        const Int4Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* ring = smem;
    uint8_t* sx = smem + p.off_x;
    float* sred = reinterpret_cast<float*>(smem + p.off_red);  // [CL][128][RS] peers' partial sums, then its own
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + p.off_bars);
    uint64_t* full = bars;
    uint64_t* empty = bars + p.stages;
    uint64_t* afull = bars + 2 * p.stages;  // [kI4ASlots]
    uint64_t* afree = afull + kI4ASlots;    // [kI4ASlots]
    uint64_t* dfull = afree + kI4ASlots;    // [kI4DSlots]
    uint64_t* dfree = dfull + kI4DSlots;    // [kI4DSlots]
    uint64_t* xfull = dfree + kI4DSlots;
    uint64_t* red_done = xfull + 1;
    uint64_t* drain = xfull + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(xfull + 3);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int M = p.M, K = p.K, N = p.N, G = p.G;
    const int CL = p.cluster;
    const int RS = p.xrows;  // rows of one partial-sum slot
    WaitCtx wctx{abort_flag, p.status, p.wait_limit_ns};

    const int rank = (int)cluster_ctarank();
    const int cid = blockIdx.x / CL;
    const int tile0 = (int)((long long)cid * p.num_tiles / p.num_clusters);
    const int nt = (int)((long long)(cid + 1) * p.num_tiles / p.num_clusters) - tile0;
    const int kb_lo = p.kb_total * rank / CL;
    const int kb_hi = p.kb_total * (rank + 1) / CL;
    const int nblk = 2 * (kb_hi - kb_lo);  // 128-k blocks per tile in this CTA's K range
    const int nb = nt * nblk;               // 128-k blocks of this CTA
    const bool owner = rank < nt;
    const int nxb = (kb_hi - kb_lo) * (kI4BoxK / 64);  // X boxes of 64 k
    const uint32_t xbox_bytes = (uint32_t)p.xrows * 128;

    uint32_t tmem_base = 0;
    if (warp == 0) {
        if (lane == 0) {
            for (int s = 0; s < p.stages; ++s) {
                mbar_init(&full[s], 1);
                mbar_init(&empty[s], kI4WidenWarps);
            }
            for (int a = 0; a < kI4ASlots; ++a) {
                mbar_init(&afull[a], kI4WidenWarps);
                mbar_init(&afree[a], 1);
            }
            for (int d = 0; d < kI4DSlots; ++d) {
                mbar_init(&dfull[d], 1);
                mbar_init(&dfree[d], 4);
            }
            mbar_init(xfull, 1);
            mbar_init(red_done, 1);
            mbar_init(drain, 1);
            *abort_flag = 0;
            fence_mbar_init();
            prefetch_tmap(&tm_w);
            prefetch_tmap(&tm_x);
            const uint32_t rb = (uint32_t)((CL - 1) * kI4TileN * RS * 4);
            if (owner && nb > 0 && rb) mbar_arrive_expect_tx(red_done, rb);
            else mbar_arrive(red_done);
        }
        __syncwarp();
        cluster_arrive();
        named_bar_arrive(2, kI4Threads);
    } else if (warp == 1) {
        tmem_alloc(tmem_slot, p.tmem_cols);
        tmem_relinquish();
        tc_fence_before();
        cluster_arrive();
        named_bar_sync(2, kI4Threads);
        tc_fence_after();
        tmem_base = *tmem_slot;
    } else {
        cluster_arrive();
        named_bar_sync(2, kI4Threads);
        tc_fence_after();
        tmem_base = *tmem_slot;
    }
    pdl_launch_dependents();

    if (warp == 0) {
        // ------------------------------------------------ packed-code stream (needs nothing from earlier kernels)
        if (elect_one()) {
            const uint64_t pol = policy_evict_first();
            uint32_t armed = 0, armed_par = 0;
            bool ok = true;
            for (int t = 0; ok && t < nb / 2; ++t) {
                const int stage = t % p.stages;
                const uint32_t ph = (uint32_t)((t / p.stages) & 1);
                if (!wait_bounded_sleep(&empty[stage], ph ^ 1u, wctx)) {
                    ok = false;
                    break;
                }
                const int j = t / (nblk / 2), kb = kb_lo + t % (nblk / 2);
                mbar_arrive_expect_tx(&full[stage], kI4StageBytes);
                tma_load_2d(ring + stage * kI4StageBytes, &tm_w, &full[stage], kb * 128, (tile0 + j) * kI4TileN, pol);
                armed |= 1u << stage;
                armed_par = (armed_par & ~(1u << stage)) | (ph << stage);
            }
            for (int s = 0; s < p.stages; ++s)
                if (armed & (1u << s)) wait_drain(&full[s], (armed_par >> s) & 1u, 50ull * 1000 * 1000);
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (elect_one() && nb > 0) {
            const uint32_t idesc = idesc_f16_f32(128, 16);
            const uint64_t db0 = sdesc_k128sw(smem_u32(sx));
            bool ok = wait_bounded_sleep(xfull, 0, wctx), issued = false;
            tc_fence_after();
            for (int i = 0; ok && i < nb; ++i) {
                const int a = i % kI4ASlots, d = i % kI4DSlots;
                if (!wait_bounded_sleep(&afull[a], (uint32_t)((i / kI4ASlots) & 1), wctx) ||
                    !wait_bounded_sleep(&dfree[d], (uint32_t)(((i / kI4DSlots) & 1) ^ 1), wctx)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const int b = i % nblk;  // 128-k block within the K range
                const uint32_t dt = tmem_base + kI4DColBase + 16u * (uint32_t)d;
                const uint32_t at = tmem_base + kI4AColBase + 64u * (uint32_t)a;
#pragma unroll
                for (int st = 0; st < 8; ++st) {
                    // B: k = b * 128 + 16 st within the range -> X box (k / 64), 32-byte step inside it
                    const int kk = b * 128 + 16 * st;
                    const uint64_t db = db0 + (uint64_t)(((uint32_t)(kk >> 6) * xbox_bytes + (uint32_t)((kk & 63) * 2)) >> 4);
                    i4_mma_f16_ts(dt, at + 8u * (uint32_t)st, db, idesc, st > 0 ? 1u : 0u);
                }
                tc_commit(&afree[a]);
                tc_commit(&dfull[d]);
                issued = true;
            }
            if (issued) {
                tc_commit(drain);
                wait_drain(drain, 0, 50ull * 1000 * 1000);
            }
        }
    } else if (warp < 2 + kI4WidenWarps) {
        // ------------------------------------------------ widen codes to fp16 A operands in TMEM
        const int quad = warp & 3;
        const int part = (warp - 2) >> 2;  // this warp's 64 k of each 128-k block
        const int row = quad * 32 + lane;  // output column within the tile = TMEM lane
        const uint32_t lane_addr = (uint32_t)(quad * 32) << 16;
        bool ok = true;
        for (int i = 0; ok && i < nb; ++i) {
            const int t = i >> 1, h = i & 1, a = i % kI4ASlots;
            const int stage = t % p.stages;
            const uint32_t ph = (uint32_t)((t / p.stages) & 1);
            ok = __all_sync(0xffffffffu, wait_bounded_sleep(&full[stage], ph, wctx)) &&
                 __all_sync(0xffffffffu, wait_bounded_sleep(&afree[a], (uint32_t)(((i / kI4ASlots) & 1) ^ 1), wctx));
            if (!ok) break;
            tc_fence_after();
            const uint8_t* src = ring + stage * kI4StageBytes + row * 128;
            uint32_t v[32];
#pragma unroll
            for (int c2 = 0; c2 < 2; ++c2) {
                const int c = 4 * h + 2 * part + c2;  // 16-byte chunk of the row (128-byte swizzle)
                const uint4 w = *reinterpret_cast<const uint4*>(src + ((c ^ (row & 7)) << 4));
                i4_widen(w.x, &v[16 * c2 + 0]);
                i4_widen(w.y, &v[16 * c2 + 4]);
                i4_widen(w.z, &v[16 * c2 + 8]);
                i4_widen(w.w, &v[16 * c2 + 12]);
            }
            tmem_st32(tmem_base + lane_addr + kI4AColBase + 64u * (uint32_t)a + 32u * (uint32_t)part, v);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&afull[a]);
                if (h == 1) mbar_arrive(&empty[stage]);
            }
        }
    } else {
        // ------------------------------------------------ accumulate (warps 10-13)
        pdl_wait();      // X and Y belong to earlier work on the stream
        cluster_wait();  // every peer's barriers are initialised before the first store into it
        if (warp == 2 + kI4WidenWarps && elect_one()) {
            // X (this CTA's K range, all M rows; rows past M and k past K read as 0)
            const int kx0 = kb_lo * kI4BoxK;
            mbar_arrive_expect_tx(xfull, (uint32_t)nxb * xbox_bytes);
            if (!(p.test_flags & 1u))
                for (int xb = 0; xb < nxb; ++xb)
                    tma_load_2d(sx + (size_t)xb * xbox_bytes, &tm_x, xfull, kx0 + 64 * xb, 0, 0ull);
        }
        const int quad = warp & 3;
        const int ch = quad * 32 + lane;
        const uint32_t lane_addr = (uint32_t)(quad * 32) << 16;
        const int ng = K / G;
        float y[16];
#pragma unroll
        for (int m = 0; m < 16; ++m) y[m] = 0.0f;
        float* own = sred + (size_t)((CL - 1) * kI4TileN + ch) * RS;  // this CTA's sums of its own tile
        // group constant (absmax) of block i for this thread's column; a half
        // box past K (K % 256 == 128) multiplies X's zero fill, so any finite
        // constant will do there
        auto absmax_of = [&](int i) -> float {
            if (i >= nb) return 0.0f;
            const int n = (tile0 + i / nblk) * kI4TileN + ch;
            const int g = min((kb_lo * kI4BoxK + (i % nblk) * 128) / G, ng - 1);
            return n < N ? __ldg(p.absmax + (size_t)n * ng + g) : 0.0f;
        };
        // constants of the next batch load while the current one is drained
        constexpr int kAhead = kI4DBatch;
        float a_next[kAhead];
#pragma unroll
        for (int u = 0; u < kAhead; ++u) a_next[u] = absmax_of(u);
        bool ok = nb > 0;
        for (int i0 = 0; ok && i0 < nb; i0 += kI4DBatch) {
            float a_cur[kAhead];
#pragma unroll
            for (int u = 0; u < kAhead; ++u) a_cur[u] = a_next[u];
            if (i0 + kAhead < nb) {
#pragma unroll
                for (int u = 0; u < kAhead; ++u) a_next[u] = absmax_of(i0 + kAhead + u);
            }
            // the commit of the batch's last block completes after every
            // earlier MMA of the issuing thread, so one wait covers the batch;
            // the batch's slots are consecutive (i0 is a multiple of 4)
            const int last = min(i0 + kI4DBatch, nb) - 1;
            ok = __all_sync(0xffffffffu,
                            wait_bounded_sleep(&dfull[last % kI4DSlots], (uint32_t)((last / kI4DSlots) & 1), wctx));
            if (!ok) break;
            tc_fence_after();
            const uint32_t d0 = (uint32_t)(i0 % kI4DSlots);
            uint32_t r[2][32];
            tmem_ld32(tmem_base + lane_addr + kI4DColBase + 16u * d0, r[0]);
            tmem_ld32(tmem_base + lane_addr + kI4DColBase + 16u * d0 + 32u, r[1]);
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                for (int i = i0; i <= last; ++i) mbar_arrive(&dfree[i % kI4DSlots]);
#pragma unroll
            for (int u = 0; u < kI4DBatch; ++u) {
                const int i = i0 + u;
                if (i > last) break;
                const int j = i / nblk, b = i % nblk;
                const float sc = __fdiv_rn(a_cur[u], 7.0f);
#pragma unroll
                for (int m = 0; m < 16; ++m) y[m] = fmaf(__uint_as_float(r[u >> 1][16 * (u & 1) + m]), sc, y[m]);
                if (b == nblk - 1) {
                    // tile j is complete in this K range: keep it (owner) or send it to its owner
                    if (j == rank) {
#pragma unroll
                        for (int m = 0; m < 16; ++m)
                            if (m < RS) own[m] = y[m];
                    } else {
                        const int slot = rank < j ? rank : rank - 1;
                        const uint32_t dst = map_to_rank(&sred[(size_t)(slot * kI4TileN + ch) * RS], (uint32_t)j);
                        const uint32_t mb = map_to_rank(red_done, (uint32_t)j);
                        st_async_v4(dst, __float_as_uint(y[0]), __float_as_uint(y[1]), __float_as_uint(y[2]),
                                    __float_as_uint(y[3]), mb);
                        st_async_v4(dst + 16, __float_as_uint(y[4]), __float_as_uint(y[5]), __float_as_uint(y[6]),
                                    __float_as_uint(y[7]), mb);
                        if (RS == 16) {
                            st_async_v4(dst + 32, __float_as_uint(y[8]), __float_as_uint(y[9]),
                                        __float_as_uint(y[10]), __float_as_uint(y[11]), mb);
                            st_async_v4(dst + 48, __float_as_uint(y[12]), __float_as_uint(y[13]),
                                        __float_as_uint(y[14]), __float_as_uint(y[15]), mb);
                        }
                    }
#pragma unroll
                    for (int m = 0; m < 16; ++m) y[m] = 0.0f;
                }
            }
        }
        const int n = (tile0 + rank) * kI4TileN + ch;
        if (owner && ok && __all_sync(0xffffffffu, wait_bounded_sleep(red_done, 0, wctx)) && n < N) {
#pragma unroll
            for (int m = 0; m < 16; ++m) {
                if (m < M) {
                    float v = own[m];
                    for (int q = 0; q < CL - 1; ++q) v += sred[(size_t)(q * kI4TileN + ch) * RS + m];
                    p.Y[(size_t)m * N + n] = __half_as_ushort(__float2half_rn(v));
                }
            }
        }
    }

    if (warp < 2 + kI4WidenWarps) cluster_wait();  // warps 10-13 waited before their first peer access
    // every store into this CTA's shared memory completes on a barrier it has
    // waited for; after a timeout a peer's store may still be on its way
    if (*abort_flag) settle_after_abort();
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, p.tmem_cols);
    }
}

}  // namespace i8mm
