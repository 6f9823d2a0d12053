// Bandwidth-bound steps of the LLM.int8() forward pass and the one-time weight
// conversion ("LLM.int8(): 8-bit Matrix Multiplication for Transformers at
// Scale", abstract):
//   k_col_absmax / k_quant_weight   -- per-output-channel absmax int8 weight (c)
//   k_detect                        -- outlier feature columns of X, their
//                                      list and count (a)
//   k_quant_rows_reg (K <= 16384) /
//   k_quant_rows (longer K)         -- row absmax int8 X without the outlier
//                                      columns, plus the fp16 outlier columns (b);
//                                      the first also gathers the outlier
//                                      weight rows in the same grid
//   k_col_absmax_grouped /
//   k_quant_rows_grouped            -- the same with one constant per group of G
//                                      consecutive k (group-wise variant)
//   k_gather_wo                     -- fp16 weight rows of the outlier dims (d),
//                                      for the paths without k_quant_rows_reg
// All loads of X / W are 16-byte vectors along the contiguous dimension.
#pragma once

#include <cuda_fp16.h>
#include <stdint.h>

#include "sm100_ptx.cuh"

namespace i8mm {

// |x| as a comparable integer: the fp16 sign bit cleared, NaN mapped to 0 so
// that a NaN never wins a max and never counts as an outlier.
__device__ __forceinline__ uint32_t abs_bits2(uint32_t two_halves) {
    uint32_t a = two_halves & 0x7FFF7FFFu;
    uint32_t not_nan = __vcmpleu2(a, 0x7C007C00u);  // 0xFFFF per lane where a <= +inf
    return a & not_nan;
}

__device__ __forceinline__ float half_bits_to_float(uint32_t bits16) {
    return __half2float(__ushort_as_half((unsigned short)bits16));
}

// round-half-even(x * scale) clamped to [-127, 127]; fp32 product as in the method.
__device__ __forceinline__ int quant1(float x, float scale) {
    int q = __float2int_rn(__fmul_rn(x, scale));
    return max(-127, min(127, q));
}

// ------------------------------------------------------------------ weight

// ca[n] = max_k |W[k, n]| as float bits via atomicMax (ca pre-zeroed).
// Block: 256 threads, each 8 consecutive columns; grid (ceil(N/2048), ksplit).
__global__ void k_col_absmax(const uint16_t* __restrict__ W, int K, int N, int rows_per_block,
                             unsigned* __restrict__ ca_bits) {
    const int col0 = (blockIdx.x * 256 + threadIdx.x) * 8;
    if (col0 >= N) return;
    const int k0 = blockIdx.y * rows_per_block;
    const int k1 = min(K, k0 + rows_per_block);
    uint32_t m[4] = {0, 0, 0, 0};
    for (int k = k0; k < k1; ++k) {
        uint4 v = __ldg(reinterpret_cast<const uint4*>(W + (size_t)k * N + col0));
        m[0] = __vmaxu2(m[0], abs_bits2(v.x));
        m[1] = __vmaxu2(m[1], abs_bits2(v.y));
        m[2] = __vmaxu2(m[2], abs_bits2(v.z));
        m[3] = __vmaxu2(m[3], abs_bits2(v.w));
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        atomicMax(&ca_bits[col0 + 2 * i], __float_as_uint(half_bits_to_float(m[i] & 0xFFFF)));
        atomicMax(&ca_bits[col0 + 2 * i + 1], __float_as_uint(half_bits_to_float(m[i] >> 16)));
    }
}

// ca[g * N + n] = max over the group g of G consecutive k of |W[k, n]|.
// Block 256 threads, each 8 consecutive columns; grid (ceil(N/2048), K/G).
__global__ void k_col_absmax_grouped(const uint16_t* __restrict__ W, int K, int N, int G, float* __restrict__ ca) {
    const int col0 = (blockIdx.x * 256 + threadIdx.x) * 8;
    if (col0 >= N) return;
    const int g = blockIdx.y;
    uint32_t m[4] = {0, 0, 0, 0};
    for (int k = g * G; k < (g + 1) * G; ++k) {
        uint4 v = __ldg(reinterpret_cast<const uint4*>(W + (size_t)k * N + col0));
        m[0] = __vmaxu2(m[0], abs_bits2(v.x));
        m[1] = __vmaxu2(m[1], abs_bits2(v.y));
        m[2] = __vmaxu2(m[2], abs_bits2(v.z));
        m[3] = __vmaxu2(m[3], abs_bits2(v.w));
    }
    float* dst = ca + (size_t)g * N + col0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        dst[2 * i] = half_bits_to_float(m[i] & 0xFFFF);
        dst[2 * i + 1] = half_bits_to_float(m[i] >> 16);
    }
}

// Wq[n, k] = round_half_even(W[k, n] * (127 / ca)), transposed through a
// 64 x 64 shared tile; ca is the constant of column n and of the group of G
// consecutive k that holds k (ca[(k / G) * N + n]; G = K: one constant per
// column).  G is a multiple of 64, so a tile lies in one group.  Block 256
// threads, grid (ceil(N/64), ceil(K/64)).
__global__ void k_quant_weight(const uint16_t* __restrict__ W, int K, int N, int G, const float* __restrict__ ca,
                               int8_t* __restrict__ Wq) {
    __shared__ uint16_t tile[64][64 + 8];
    const int n0 = blockIdx.x * 64, k0 = blockIdx.y * 64;
    const int t = threadIdx.x;
    // load 64 rows (k) x 64 cols (n): 512 chunks of 8 halves
    for (int c = t; c < 512; c += 256) {
        int r = c >> 3, cc = (c & 7) * 8;
        int k = k0 + r, n = n0 + cc;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (k < K && n < N) v = __ldg(reinterpret_cast<const uint4*>(W + (size_t)k * N + n));
        *reinterpret_cast<uint4*>(&tile[r][cc]) = v;
    }
    __syncthreads();
    // write 64 rows (n) x 64 bytes (k): thread -> (n = t/4, 16 k's)
    const int nl = t >> 2, kl = (t & 3) * 16;
    const int n = n0 + nl;
    if (n >= N) return;
    const float a = ca[(size_t)(k0 / G) * N + n];
    const float scale = a > 0.0f ? __fdiv_rn(127.0f, a) : 0.0f;
    uint32_t packed[4];
#pragma unroll
    for (int w = 0; w < 4; ++w) {
        uint32_t word = 0;
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            int q = a > 0.0f ? quant1(half_bits_to_float(tile[kl + 4 * w + b][nl]), scale) : 0;
            word |= ((uint32_t)(q & 0xFF)) << (8 * b);
        }
        packed[w] = word;
    }
    const int k = k0 + kl;
    if (k < K)  // K % 16 == 0, so the 16-byte group is entirely in or out
        *reinterpret_cast<uint4*>(Wq + (size_t)n * K + k) = make_uint4(packed[0], packed[1], packed[2], packed[3]);
}

// w_keep[i, :] = W[keep_idx[i], :]; one block per kept row.
__global__ void k_copy_keep_rows(const uint16_t* __restrict__ W, int N, const int32_t* __restrict__ keep_idx,
                                 uint16_t* __restrict__ w_keep) {
    const int i = blockIdx.x;
    const uint4* src = reinterpret_cast<const uint4*>(W + (size_t)keep_idx[i] * N);
    uint4* dst = reinterpret_cast<uint4*>(w_keep + (size_t)i * N);
    for (int c = threadIdx.x; c < N / 8; c += blockDim.x) dst[c] = __ldg(src + c);
}

// ------------------------------------------------------------------ (a) detect

// The last block of k_detect: the bitmask as the OR of the row splits' words,
// the exclusive prefix counts, the ascending outlier list, the count and the
// overflow flag; resets the ticket.  All 256 threads of the block.
__device__ __noinline__ void detect_finalise(const uint32_t* __restrict__ part, int ny, int nw,
                                             uint32_t* __restrict__ mask, int32_t* __restrict__ spre,
                                             int32_t* __restrict__ idx, int32_t* __restrict__ n_out, int cap,
                                             int* __restrict__ status, unsigned* __restrict__ ticket) {
    __shared__ int wtot[8];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    int carry = 0;
    for (int base = 0; base < nw; base += 256) {
        const int w = base + tid;
        uint32_t word = 0u;
        if (w < nw) {
            // up to 16 independent loads in flight per step (all of them for
            // up to 16 row splits): this block's latency is on the critical path
            for (int y0 = 0; y0 < ny; y0 += 16) {
                uint32_t t[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) t[i] = y0 + i < ny ? __ldcg(part + (size_t)(y0 + i) * nw + w) : 0u;
#pragma unroll
                for (int i = 0; i < 16; ++i) word |= t[i];
            }
        }
        const int c = __popc(word);
        int incl = c;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
        }
        if (lane == 31) wtot[warp] = incl;
        __syncthreads();
        int before = 0, blk = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            before += i < warp ? wtot[i] : 0;
            blk += wtot[i];
        }
        if (w < nw) {
            int s = carry + before + incl - c;
            mask[w] = word;
            spre[w] = s;
            while (word) {
                idx[s++] = w * 32 + (__ffs(word) - 1);
                word &= word - 1;
            }
        }
        carry += blk;
        __syncthreads();
    }
    if (tid == 0) {
        *n_out = carry;
        if (carry > cap) atomicOr(status, kStatusOverflow);
        *ticket = 0u;
    }
}

// One pass over X: column k is an outlier when max_m |X[m, k]| >= thr.
// Block 256 threads = 8 warps over 256 columns (8 per lane); warps stride over
// rows [row0, row1) of the block's row split blockIdx.y.  Each block stores
// the 8 flag words of its columns for its row split (part[y * nw + w], bit k
// of word k / 32; every word is written on every call, so nothing needs
// clearing).  The last block to finish (a ticket counted in *ticket) OR-s the
// row splits into the bitmask mask[w], forms the exclusive prefix counts
// spre[w] (outlier columns before word w) and writes the ascending outlier
// list idx, the count *n_out and the overflow flag, then resets the ticket.
__global__ void __launch_bounds__(256, 6) k_detect(const uint16_t* __restrict__ X, int M, int K, float thr,
                                                int rows_per_block, uint32_t* __restrict__ part,
                                                uint32_t* __restrict__ mask, int32_t* __restrict__ spre,
                                                int32_t* __restrict__ idx, int32_t* __restrict__ n_out, int cap,
                                                int* __restrict__ status, unsigned* __restrict__ ticket) {
    pdl_launch_dependents();
    __shared__ uint32_t red[8][32][4];
    __shared__ unsigned last_sh;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nw = (K + 31) / 32;
    const int col0 = blockIdx.x * 256 + lane * 8;
    const int row0 = blockIdx.y * rows_per_block;
    const int row1 = min(M, row0 + rows_per_block);
    // running |x| maxima as packed fp16 pairs: __hmax2 returns the other operand
    // when one is NaN, so from the +0 start a NaN never enters a maximum
    __half2 h[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) h[i] = __floats2half2_rn(0.0f, 0.0f);
    if (col0 < K) {
        for (int r = row0 + warp; r < row1; r += 8) {
            const uint4 v = __ldg(reinterpret_cast<const uint4*>(X + (size_t)r * K + col0));
            const uint32_t a[4] = {v.x & 0x7FFF7FFFu, v.y & 0x7FFF7FFFu, v.z & 0x7FFF7FFFu, v.w & 0x7FFF7FFFu};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                __half2 t;
                memcpy(&t, &a[i], 4);
                h[i] = __hmax2(h[i], t);
            }
        }
    }
    uint32_t m[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) memcpy(&m[i], &h[i], 4);
#pragma unroll
    for (int i = 0; i < 4; ++i) red[warp][lane][i] = m[i];
    __syncthreads();
    if (warp == 0) {
#pragma unroll
        for (int w = 1; w < 8; ++w)
#pragma unroll
            for (int i = 0; i < 4; ++i) m[i] = __vmaxu2(m[i], red[w][lane][i]);
        uint32_t flags = 0;  // 8 bits, one per column of this lane
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            if (half_bits_to_float(m[i] & 0xFFFF) >= thr) flags |= 1u << (2 * i);
            if (half_bits_to_float(m[i] >> 16) >= thr) flags |= 1u << (2 * i + 1);
        }
        if (col0 >= K) flags = 0;
        // word j of this block = lanes 4j..4j+3
        const uint32_t f1 = __shfl_down_sync(0xffffffffu, flags, 1);
        const uint32_t f2 = __shfl_down_sync(0xffffffffu, flags, 2);
        const uint32_t f3 = __shfl_down_sync(0xffffffffu, flags, 3);
        const int wi = (blockIdx.x * 256 + lane * 8) >> 5;
        if ((lane & 3) == 0 && wi < nw)
            part[(size_t)blockIdx.y * nw + wi] = flags | (f1 << 8) | (f2 << 16) | (f3 << 24);
        __threadfence();  // the words before the ticket
    }
    __syncthreads();
    if (tid == 0) {
        const unsigned nblk = gridDim.x * gridDim.y;
        last_sh = (atomicAdd(ticket, 1u) == nblk - 1) ? 1u : 0u;
    }
    __syncthreads();
    if (!last_sh) return;
    __threadfence();  // every block's words are visible from here on

    detect_finalise(part, gridDim.y, nw, mask, spre, idx, n_out, cap, status, ticket);
}

// ------------------------------------------------------------------ (b) quantise rows

// Max |x| over the non-outlier columns of one 8-column chunk (as fp16 bits);
// fl = the chunk's 8 outlier flags (bit j: column j of the chunk).  Taken only
// by chunks that hold an outlier column, so it is kept out of line.
__device__ __noinline__ uint32_t chunk_inlier_absmax(uint4 v, uint32_t fl) {
    const uint32_t h[4] = {v.x, v.y, v.z, v.w};
    uint32_t amax = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const uint32_t a = abs_bits2(h[j]);
        const uint32_t lo = ((fl >> (2 * j)) & 1u) ? 0u : (a & 0xFFFFu);
        const uint32_t hi = ((fl >> (2 * j + 1)) & 1u) ? 0u : (a >> 16);
        amax = max(amax, max(lo, hi));
    }
    return amax;
}

// Codes of an 8-column chunk with no outlier column (the common case).  Every
// value is a non-outlier of its row, so |x| <= ra and |x * scale| <= 127 * (1
// + 2^-24): RN32(RN32(x * scale) + 1.5 * 2^23) holds the code in its low
// byte (no clamp can trigger), and the bytes are packed straight from the
// float bit patterns.  (A NaN in X, outside the method's inputs, gets an
// unspecified code.)
__device__ __forceinline__ uint2 quant8_plain(uint4 v, float scale) {
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
    const uint32_t lo = __byte_perm(__byte_perm(b[0], b[1], 0x0040), __byte_perm(b[2], b[3], 0x0040), 0x5410);
    const uint32_t hi = __byte_perm(__byte_perm(b[4], b[5], 0x0040), __byte_perm(b[6], b[7], 0x0040), 0x5410);
    return make_uint2(lo, hi);
}
// Max |x| (fp16 bits) of an 8-column chunk with no outlier column, on packed
// fp16 pairs with the native half2 max: |x| is the bit pattern with the sign
// cleared, and __hmax2 returns the other operand when one is NaN, so a NaN
// never wins (a lane whose 8 values are all NaN gives the +0 of the start).
__device__ __forceinline__ uint32_t chunk_absmax_h2(uint4 v) {
    __half2 a0, a1, a2, a3;
    const uint32_t b0 = v.x & 0x7FFF7FFFu, b1 = v.y & 0x7FFF7FFFu, b2 = v.z & 0x7FFF7FFFu, b3 = v.w & 0x7FFF7FFFu;
    memcpy(&a0, &b0, 4);
    memcpy(&a1, &b1, 4);
    memcpy(&a2, &b2, 4);
    memcpy(&a3, &b3, 4);
    const __half2 zero = __floats2half2_rn(0.0f, 0.0f);
    const __half2 m = __hmax2(zero, __hmax2(__hmax2(a0, a1), __hmax2(a2, a3)));
    uint32_t mb;
    memcpy(&mb, &m, 4);
    return max(mb & 0xFFFFu, mb >> 16);
}


// Quantise one 8-column chunk c of a row; outlier columns give 0 and are
// copied to their slot of the row's fp16 outlier vector.  word = the mask word
// holding the chunk (columns 32 * (c / 4) ...), pre = the outlier columns
// before that word.  Taken only by chunks that hold an outlier column.
__device__ __noinline__ uint2 quant_chunk(uint4 v, uint32_t word, int pre, int c, float rmax, float scale,
                                          int n_eff, uint16_t* xo_row) {
    const uint32_t fl = (word >> ((c & 3) * 8)) & 0xFFu;
    const uint32_t h[4] = {v.x, v.y, v.z, v.w};
    uint32_t out[2] = {0u, 0u};
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const uint32_t bits = (h[j >> 1] >> ((j & 1) * 16)) & 0xFFFFu;
        int q = 0;
        if (!((fl >> j) & 1u)) {
            if (rmax > 0.0f) q = quant1(half_bits_to_float(bits), scale);
        } else {
            const int k = c * 8 + j;
            const int slot = pre + __popc(word & ((1u << (k & 31)) - 1u));
            if (slot < n_eff) xo_row[slot] = (uint16_t)bits;
        }
        out[j >> 2] |= ((uint32_t)(q & 0xFF)) << ((j & 3) * 8);
    }
    return make_uint2(out[0], out[1]);
}

// The outlier bitmask into shared memory with the exclusive prefix counts of
// its words (spre[w] = outlier columns before word w); returns the total.
// Every thread of the 256-thread block calls it (it has block barriers).
__device__ __forceinline__ int load_mask_prefix(const uint32_t* __restrict__ mask, int nw, uint32_t* smask, int* spre,
                                                int* red) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    int carry = 0;
    for (int base = 0; base < nw; base += 256) {
        const int w = base + tid;
        const uint32_t word = w < nw ? mask[w] : 0u;
        if (w < nw) smask[w] = word;
        const int c = __popc(word);
        int incl = c;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
        }
        if (lane == 31) red[warp] = incl;
        __syncthreads();
        int wsum = 0, blk_total = 0;
        for (int i = 0; i < 8; ++i) {
            if (i < warp) wsum += red[i];
            blk_total += red[i];
        }
        if (w < nw) spre[w] = carry + wsum + incl - c;
        carry += blk_total;
        __syncthreads();
    }
    return carry;
}

// Per row m: ra[m] = max over non-outlier columns of |X[m,k]|,
// Xq[m,k] = outlier ? 0 : q(X[m,k]), Xo[m, slot(k)] = X[m,k] for outlier k,
// with Xo zero-padded to a multiple of 64 columns (the outlier list, count
// and overflow flag come from k_detect).
// One warp per row (no block barrier inside the row loop): a first pass over
// the row takes the absmax with 8 independent 16-byte loads in flight per
// lane, a second pass (served by L1/L2) writes the codes.  Block: 256 threads
// = 8 rows at a time; the grid strides over rows.
__global__ void __launch_bounds__(256) k_quant_rows(const uint16_t* __restrict__ X, int M, int K,
                                                    const uint32_t* __restrict__ mask, int cap, int kp,
                                                    int8_t* __restrict__ Xq, float* __restrict__ ra,
                                                    uint16_t* __restrict__ Xo) {
    extern __shared__ uint32_t qsm[];
    const int nw = (K + 31) / 32;
    uint32_t* smask = qsm;                          // nw words
    int* spre = reinterpret_cast<int*>(qsm + nw);   // nw exclusive prefix counts
    __shared__ int red[8];
    __shared__ int total_sh;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    pdl_wait();  // the outlier bitmask comes from k_detect
    pdl_launch_dependents();

    const int carry = load_mask_prefix(mask, nw, smask, spre, red);
    // A warp's iteration covers 256 chunks (2048 columns, 64 mask words); a
    // window with no outlier column (the common case) skips the per-chunk
    // flag lookups.
    const int nchunk = K / 8;
    const int nwin = (nchunk + 255) / 256;
    uint32_t* swin = qsm + 2 * nw;
    for (int t = tid; t < nwin; t += 256) {
        uint32_t o = 0u;
        for (int w = t * 64; w < min(nw, t * 64 + 64); ++w) o |= smask[w];
        swin[t] = o;
    }
    if (tid == 0) total_sh = carry;
    __syncthreads();
    const int total = total_sh;
    const int n_eff = min(total, cap);
    const int n_pad = min(kp, (n_eff + 63) / 64 * 64);

    for (int m = blockIdx.x * 8 + warp; m < M; m += gridDim.x * 8) {
        const uint4* xr = reinterpret_cast<const uint4*>(X + (size_t)m * K);
        uint32_t amax = 0;
        for (int c0 = lane, it = 0; c0 < nchunk; c0 += 32 * 8, ++it) {
            uint4 v[8];
            if (swin[it] == 0u && (it + 1) * 256 <= nchunk) {  // whole window, no outlier column
#pragma unroll
                for (int i = 0; i < 8; ++i) v[i] = __ldg(xr + c0 + 32 * i);
#pragma unroll
                for (int i = 0; i < 8; ++i) amax = max(amax, chunk_absmax_h2(v[i]));
                continue;
            }
#pragma unroll
            for (int i = 0; i < 8; ++i)
                if (c0 + 32 * i < nchunk) v[i] = __ldg(xr + c0 + 32 * i);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int c = c0 + 32 * i;
                if (c < nchunk) {
                    const uint32_t fl = (smask[c >> 2] >> ((c & 3) * 8)) & 0xFFu;
                    amax = max(amax, fl ? chunk_inlier_absmax(v[i], fl) : chunk_absmax_h2(v[i]));
                }
            }
        }
        amax = __reduce_max_sync(0xffffffffu, amax);
        const float rmax = half_bits_to_float(amax);
        const float scale = rmax > 0.0f ? __fdiv_rn(127.0f, rmax) : 0.0f;
        if (lane == 0) ra[m] = rmax;
        uint2* qr = reinterpret_cast<uint2*>(Xq + (size_t)m * K);
        uint16_t* xo_row = Xo + (size_t)m * kp;
        for (int c0 = lane, it = 0; c0 < nchunk; c0 += 32 * 8, ++it) {
            uint4 v[8];
            if (swin[it] == 0u && (it + 1) * 256 <= nchunk) {
#pragma unroll
                for (int i = 0; i < 8; ++i) v[i] = __ldg(xr + c0 + 32 * i);
#pragma unroll
                for (int i = 0; i < 8; ++i) qr[c0 + 32 * i] = quant8_plain(v[i], scale);
                continue;
            }
#pragma unroll
            for (int i = 0; i < 8; ++i)
                if (c0 + 32 * i < nchunk) v[i] = __ldg(xr + c0 + 32 * i);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int c = c0 + 32 * i;
                if (c < nchunk) {
                    const uint32_t fl = (smask[c >> 2] >> ((c & 3) * 8)) & 0xFFu;
                    qr[c] = fl ? quant_chunk(v[i], smask[c >> 2], spre[c >> 2], c, rmax, scale, n_eff, xo_row)
                               : quant8_plain(v[i], scale);
                }
            }
        }
        for (int j = n_eff + lane; j < n_pad; j += 32) xo_row[j] = 0;
    }
}

// Group-wise variant of k_quant_rows: one constant per row and group of G
// consecutive columns (G a multiple of 128), ra[m * (K/G) + g] = max |X[m,k]|
// over the non-outlier columns of the group, and the codes of the group
// with its own scale.  One warp per (row, group) item, lanes strided over the
// group's 8-column chunks: a first pass takes the maximum, a second (served
// by L1/L2) writes the codes and the outlier values.  Block 256 threads.
__global__ void __launch_bounds__(256) k_quant_rows_grouped(const uint16_t* __restrict__ X, int M, int K, int G,
                                                            const uint32_t* __restrict__ mask, int cap, int kp,
                                                            int8_t* __restrict__ Xq, float* __restrict__ ra,
                                                            uint16_t* __restrict__ Xo) {
    extern __shared__ uint32_t qsm[];
    const int nw = (K + 31) / 32;
    uint32_t* smask = qsm;
    int* spre = reinterpret_cast<int*>(qsm + nw);
    __shared__ int red[8];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    pdl_wait();  // the outlier bitmask comes from k_detect
    pdl_launch_dependents();
    const int total = load_mask_prefix(mask, nw, smask, spre, red);
    const int n_eff = min(total, cap);
    const int n_pad = min(kp, (n_eff + 63) / 64 * 64);
    const int ng = K / G, cpg = G / 8;  // chunks per group
    const long long items = (long long)M * ng;
    for (long long it = (long long)blockIdx.x * 8 + warp; it < items; it += (long long)gridDim.x * 8) {
        const int m = (int)(it / ng), g = (int)(it % ng);
        const uint4* xr = reinterpret_cast<const uint4*>(X + (size_t)m * K);
        const int c0 = g * cpg, c1 = c0 + cpg;
        uint32_t amax = 0;
        for (int c = c0 + lane; c < c1; c += 32) {
            const uint4 v = __ldg(xr + c);
            const uint32_t fl = (smask[c >> 2] >> ((c & 3) * 8)) & 0xFFu;
            amax = max(amax, fl ? chunk_inlier_absmax(v, fl) : chunk_absmax_h2(v));
        }
        amax = __reduce_max_sync(0xffffffffu, amax);
        const float rmax = half_bits_to_float(amax);
        const float scale = rmax > 0.0f ? __fdiv_rn(127.0f, rmax) : 0.0f;
        if (lane == 0) ra[(size_t)m * ng + g] = rmax;
        uint2* qr = reinterpret_cast<uint2*>(Xq + (size_t)m * K);
        uint16_t* xo_row = Xo + (size_t)m * kp;
        for (int c = c0 + lane; c < c1; c += 32) {
            const uint4 v = __ldg(xr + c);
            const uint32_t fl = (smask[c >> 2] >> ((c & 3) * 8)) & 0xFFu;
            qr[c] = fl ? quant_chunk(v, smask[c >> 2], spre[c >> 2], c, rmax, scale, n_eff, xo_row)
                       : quant8_plain(v, scale);
        }
        if (g == 0)
            for (int j = n_eff + lane; j < n_pad; j += 32) xo_row[j] = 0;
    }
}

// ------------------------------------------------------------------ (d) outlier weight rows

// Wo[n, j] (N x kp fp16, K-major) = the fp16 weight row of outlier j: the kept
// row W[idx[j], n] when idx[j] was kept at preparation, else the dequantised
// value fp16(Wq[n, idx[j]] * ca / 127) with the constant of column n and of
// the group of idx[j] (ca[(k / G) * N + n]; G = K: one per column); zero for
// n_eff <= j < pad64(n_eff).  One 256-thread block builds the 64 output
// channels from n0: a 64 x 64 tile per 64 outliers, filled along n and
// written along j (row stride 66 halves, so the column reads of the write-out
// meet at most two to a bank).
__device__ __forceinline__ void gather_wo_tile(int n0, const int8_t* __restrict__ Wq, const float* __restrict__ ca,
                                               const uint16_t* __restrict__ w_keep,
                                               const int32_t* __restrict__ keep_slot, int K, int N, int G,
                                               const int32_t* __restrict__ idx, const int32_t* __restrict__ n_out,
                                               int cap, int kp, uint16_t* __restrict__ Wo) {
    __shared__ uint16_t tile[64][66];
    __shared__ int sidx[64];
    __shared__ int sslot[64];
    const int tid = threadIdx.x;
    const int n_eff = min(__ldg(n_out), cap);
    const int n_pad = min(kp, (n_eff + 63) / 64 * 64);
    for (int j0 = 0; j0 < n_pad; j0 += 64) {
        __syncthreads();
        if (tid < 64) {
            const int j = j0 + tid;
            const int k = j < n_eff ? __ldg(idx + j) : -1;
            sidx[tid] = k;
            sslot[tid] = k >= 0 ? __ldg(keep_slot + k) : -1;
        }
        __syncthreads();
        // fill tile[j][n]: coalesced along n
        for (int e = tid; e < 64 * 64; e += 256) {
            const int jl = e >> 6, nl = e & 63;
            const int n = n0 + nl, k = sidx[jl], slot = sslot[jl];
            uint16_t v = 0;
            if (k >= 0 && n < N) {
                if (slot >= 0) {
                    v = __ldg(w_keep + (size_t)slot * N + n);
                } else {
                    const float t = __fmul_rn((float)Wq[(size_t)n * K + k], ca[(size_t)(k / G) * N + n]);
                    v = __half_as_ushort(__float2half_rn(__fdiv_rn(t, 127.0f)));
                }
            }
            tile[jl][nl] = v;
        }
        __syncthreads();
        // write Wo[n][j0 .. j0+64): 64 rows x 128 bytes, 8 threads per row
        for (int e = tid; e < 64 * 8; e += 256) {
            const int nl = e >> 3, c = (e & 7) * 8;
            const int n = n0 + nl;
            if (n >= N) continue;
            uint32_t w4[4];
#pragma unroll
            for (int i = 0; i < 4; ++i)
                w4[i] = (uint32_t)tile[c + 2 * i][nl] | ((uint32_t)tile[c + 2 * i + 1][nl] << 16);
            *reinterpret_cast<uint4*>(Wo + (size_t)n * kp + j0 + c) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
        }
    }
}

// The gather as a kernel of its own (the paths whose row quantiser is not
// k_quant_rows_reg): block b builds channels [64 b, 64 b + 64).
__global__ void __launch_bounds__(256) k_gather_wo(const int8_t* __restrict__ Wq, const float* __restrict__ ca,
                                                   const uint16_t* __restrict__ w_keep,
                                                   const int32_t* __restrict__ keep_slot, int K, int N, int G,
                                                   const int32_t* __restrict__ idx,
                                                   const int32_t* __restrict__ n_out, int cap, int kp,
                                                   uint16_t* __restrict__ Wo) {
    pdl_wait();
    pdl_launch_dependents();
    gather_wo_tile(blockIdx.x * 64, Wq, ca, w_keep, keep_slot, K, N, G, idx, n_out, cap, kp, Wo);
}

// Max |x| (fp16 bits) of an 8-column chunk over its non-outlier columns, fl
// = the chunk's 8 outlier flags; branch-free (the outlier halves are cleared
// before the native half2 max, which, as in chunk_absmax_h2, ignores NaN).
__device__ __forceinline__ uint32_t chunk_absmax_masked(uint4 v, uint32_t fl) {
    const uint32_t h[4] = {v.x, v.y, v.z, v.w};
    __half2 a[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const uint32_t keep = (((fl >> (2 * j)) & 1u) ? 0u : 0x0000FFFFu) | (((fl >> (2 * j + 1)) & 1u) ? 0u : 0xFFFF0000u);
        const uint32_t b = h[j] & 0x7FFF7FFFu & keep;
        memcpy(&a[j], &b, 4);
    }
    const __half2 zero = __floats2half2_rn(0.0f, 0.0f);
    const __half2 m = __hmax2(zero, __hmax2(__hmax2(a[0], a[1]), __hmax2(a[2], a[3])));
    uint32_t mb;
    memcpy(&mb, &m, 4);
    return max(mb & 0xFFFFu, mb >> 16);
}

// 0xFF in byte j of the result for every set bit j < 4 of f.
__device__ __forceinline__ uint32_t spread_bits_to_bytes(uint32_t f) {
    return ((f & 0xFu) * 0x00204081u & 0x01010101u) * 0xFFu;
}

// Gather arguments of the fused register quantiser (see gather_wo_tile).
struct GatherArgs {
    const int8_t* Wq;
    const float* ca;
    const uint16_t* w_keep;
    const int32_t* keep_slot;
    int N, G, blocks;  // blocks = ceil(N / 64) gather tiles in front of the rows
    uint16_t* Wo;
};

// k_quant_rows with one row per 256-thread block, the row held in registers
// (kC 8-column chunks per thread, K <= 2048 * kC), so X is read from memory
// once: the row's 16-byte loads and its outlier flag words (the bitmask that
// k_detect finalised, read through L1) go out together, every warp takes its
// part of the row maximum over the non-outlier columns, one barrier joins the
// warps' maxima, and the codes follow in the same pass (each warp stores 256
// contiguous bytes per step); the row's fp16 outlier values are then copied
// by the outlier list.  The first ga.blocks blocks of the grid instead build
// 64-channel tiles of the outlier weight rows (gather_wo_tile), which need
// only k_detect's list, so that work runs beside the rows rather than after
// them.  Same results as k_quant_rows.
template <int kC>
__global__ void __launch_bounds__(256) k_quant_rows_reg(const uint16_t* __restrict__ X, int M, int K,
                                                        const uint32_t* __restrict__ mask,
                                                        const int32_t* __restrict__ n_out, int cap, int kp,
                                                        int8_t* __restrict__ Xq, float* __restrict__ ra,
                                                        uint16_t* __restrict__ Xo, const int32_t* __restrict__ idx,
                                                        GatherArgs ga) {
    __shared__ uint32_t bmax[8];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int nchunk = K / 8;

    pdl_wait();  // mask, prefix counts, list and count come from k_detect
    pdl_launch_dependents();
    if ((int)blockIdx.x < ga.blocks) {
        gather_wo_tile(blockIdx.x * 64, ga.Wq, ga.ca, ga.w_keep, ga.keep_slot, K, ga.N, ga.G, idx, n_out, cap, kp,
                       ga.Wo);
        return;
    }
    const int m = blockIdx.x - ga.blocks;
    const uint4* xr = reinterpret_cast<const uint4*>(X + (size_t)m * K);
    uint4 v[kC];
    uint32_t fl[kC];  // the outlier flags of each chunk's 8 columns
#pragma unroll
    for (int i = 0; i < kC; ++i) {
        const int c = tid + 256 * i;
        fl[i] = 0u;
        if (c < nchunk) {
            v[i] = __ldg(xr + c);
            fl[i] = (__ldg(mask + (c >> 2)) >> ((c & 3) * 8)) & 0xFFu;
        }
    }
    const int n_eff = min(__ldg(n_out), cap);
    // Chunks with an outlier column are rare (a few per row); a warp that
    // holds one takes the masked forms for that step, all lanes together.
    // The votes are taken by every lane of the warp (fl is 0 past the row).
    uint32_t any_fl = 0u;  // bit i: some lane of the warp has an outlier column in step i
#pragma unroll
    for (int i = 0; i < kC; ++i) any_fl |= (__any_sync(0xffffffffu, fl[i] != 0u) ? 1u : 0u) << i;
    uint32_t amax = 0;
#pragma unroll
    for (int i = 0; i < kC; ++i) {
        const int c = tid + 256 * i;
        if (c < nchunk)
            amax = max(amax, ((any_fl >> i) & 1u) ? chunk_absmax_masked(v[i], fl[i]) : chunk_absmax_h2(v[i]));
    }
    amax = __reduce_max_sync(0xffffffffu, amax);
    if (lane == 0) bmax[warp] = amax;
    __syncthreads();  // the warps' maxima
    amax = 0;
#pragma unroll
    for (int w = 0; w < 8; ++w) amax = max(amax, bmax[w]);
    const float rmax = half_bits_to_float(amax);
    const float scale = rmax > 0.0f ? __fdiv_rn(127.0f, rmax) : 0.0f;
    if (tid == 0) ra[m] = rmax;
    uint2* qr = reinterpret_cast<uint2*>(Xq + (size_t)m * K);
#pragma unroll
    for (int i = 0; i < kC; ++i) {
        const int c = tid + 256 * i;
        if (c < nchunk) {
            uint2 q = quant8_plain(v[i], scale);
            // outlier columns get code 0 (their products go through fp16); the
            // other codes of the chunk are exact as they stand, since those
            // columns are bounded by the row maximum
            if ((any_fl >> i) & 1u) {
                q.x &= ~spread_bits_to_bytes(fl[i]);
                q.y &= ~spread_bits_to_bytes(fl[i] >> 4);
            }
            qr[c] = q;
        }
    }
    // the row's fp16 outlier values by the list (the row is in L1), zero-padded
    uint16_t* xo_row = Xo + (size_t)m * kp;
    const int n_pad = min(kp, (n_eff + 63) / 64 * 64);
    for (int j = tid; j < n_pad; j += 256)
        xo_row[j] = j < n_eff ? __ldg(X + (size_t)m * K + __ldg(idx + j)) : (uint16_t)0;
}

}  // namespace i8mm
