// Block-wise linear 8-bit codec of an fp32 vector on B200 (HBM-bound): the
// chunked quantisation the axolotl page "llama3-model-quantization" applies to
// 32-bit optimizer state ("8-Bit Optimizers" paragraphs): each block is
// normalised by its own absolute maximum, so an outlier costs precision only
// in its own block, and every value keeps an 8-bit index.
//
// Block b covers [b*B, min(n, (b+1)*B)); absmax[b] = max |x| over the block,
// scale = RN32(127/absmax), code = round-half-even(RN32(x*scale)) (no clamp
// is needed: every |x| in a block is at most its absmax), absmax 0 gives
// codes 0.  Dequantised value = RN32(RN32(code*absmax)/127).
//
// Quantise: one warp per block, the block's values held in registers as
// float4 chunks (lane l holds chunks l, l+32, ...), one warp max, one divide,
// codes packed four to a 32-bit store (each warp store is 128 contiguous
// bytes).  Blocks longer than the register budget take a second read (L2).
// Dequantise: four codes per thread, one float4 store.
#pragma once

#include <stdint.h>

namespace i8mm {

__device__ __forceinline__ uint32_t codec_pack4(float4 v, float scale) {
    const uint32_t b0 = __float_as_uint(__fadd_rn(__fmul_rn(v.x, scale), 12582912.0f));
    const uint32_t b1 = __float_as_uint(__fadd_rn(__fmul_rn(v.y, scale), 12582912.0f));
    const uint32_t b2 = __float_as_uint(__fadd_rn(__fmul_rn(v.z, scale), 12582912.0f));
    const uint32_t b3 = __float_as_uint(__fadd_rn(__fmul_rn(v.w, scale), 12582912.0f));
    return __byte_perm(__byte_perm(b0, b1, 0x0040), __byte_perm(b2, b3, 0x0040), 0x5410);
}

// chunk c of a block of `len` values at xb (xb 16-byte aligned); values past
// len read as 0
__device__ __forceinline__ float4 codec_load(const float* __restrict__ xb, int c, int len) {
    if (4 * c + 3 < len) return __ldg(reinterpret_cast<const float4*>(xb) + c);
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (4 * c < len) v.x = __ldg(xb + 4 * c);
    if (4 * c + 1 < len) v.y = __ldg(xb + 4 * c + 1);
    if (4 * c + 2 < len) v.z = __ldg(xb + 4 * c + 2);
    return v;
}

__device__ __forceinline__ void codec_store(int8_t* __restrict__ qb, int c, int len, uint32_t w) {
    if (4 * c + 3 < len) {
        reinterpret_cast<uint32_t*>(qb)[c] = w;
    } else {
        for (int j = 0; j < 4 && 4 * c + j < len; ++j) qb[4 * c + j] = (int8_t)(w >> (8 * j));
    }
}

__device__ __forceinline__ uint32_t abs_bits_max(float4 v, uint32_t m) {
    m = max(m, __float_as_uint(fabsf(v.x)));
    m = max(m, __float_as_uint(fabsf(v.y)));
    m = max(m, __float_as_uint(fabsf(v.z)));
    return max(m, __float_as_uint(fabsf(v.w)));
}

// kV: float4 chunks per lane held in registers (B <= 128 * kV); kV == 0: any
// B, the codes pass reads the block again.
template <int kV>
__global__ void __launch_bounds__(256) k_block_quant(const float* __restrict__ x, long long n, int B,
                                                     long long nblocks, int8_t* __restrict__ q,
                                                     float* __restrict__ absmax) {
    const int lane = threadIdx.x & 31;
    const long long nwarps = (long long)gridDim.x * 8;
    const int nch = (B + 3) / 4;
    for (long long b = (long long)blockIdx.x * 8 + (threadIdx.x >> 5); b < nblocks; b += nwarps) {
        const long long lo = b * (long long)B;
        const int len = (int)min((long long)B, n - lo);
        const float* xb = x + lo;
        uint32_t m = 0u;  // non-negative fp32 bit patterns order like their values
        float4 v[kV > 0 ? kV : 1];
        if constexpr (kV > 0) {
#pragma unroll
            for (int i = 0; i < kV; ++i) {
                const int c = lane + 32 * i;
                v[i] = c < nch ? codec_load(xb, c, len) : make_float4(0.f, 0.f, 0.f, 0.f);
            }
#pragma unroll
            for (int i = 0; i < kV; ++i) m = abs_bits_max(v[i], m);
        } else {
            for (int c = lane; c < nch; c += 32) m = abs_bits_max(codec_load(xb, c, len), m);
        }
        m = __reduce_max_sync(0xffffffffu, m);
        const float amax = __uint_as_float(m);
        const float scale = amax > 0.0f ? __fdiv_rn(127.0f, amax) : 0.0f;
        if (lane == 0) absmax[b] = amax;
        int8_t* qb = q + lo;
        if constexpr (kV > 0) {
#pragma unroll
            for (int i = 0; i < kV; ++i) {
                const int c = lane + 32 * i;
                if (c < nch) codec_store(qb, c, len, codec_pack4(v[i], scale));
            }
        } else {
            for (int c = lane; c < nch; c += 32) codec_store(qb, c, len, codec_pack4(codec_load(xb, c, len), scale));
        }
    }
}

// out[i] = RN32(RN32(q[i] * absmax[i / B]) / 127); thread t handles codes
// [4t, 4t + 4) (B % 4 == 0, so one block constant per thread).
__global__ void __launch_bounds__(256) k_block_dequant(const int8_t* __restrict__ q, const float* __restrict__ absmax,
                                                       long long n, int B, float* __restrict__ out) {
    const long long nq = (n + 3) / 4;
    for (long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x; t < nq; t += (long long)gridDim.x * blockDim.x) {
        const long long i0 = 4 * t;
        const float a = __ldg(absmax + i0 / B);
        if (i0 + 3 < n) {
            const uint32_t w = __ldg(reinterpret_cast<const uint32_t*>(q) + t);
            float4 r;
            r.x = __fdiv_rn(__fmul_rn((float)(int8_t)(w & 0xFFu), a), 127.0f);
            r.y = __fdiv_rn(__fmul_rn((float)(int8_t)((w >> 8) & 0xFFu), a), 127.0f);
            r.z = __fdiv_rn(__fmul_rn((float)(int8_t)((w >> 16) & 0xFFu), a), 127.0f);
            r.w = __fdiv_rn(__fmul_rn((float)(int8_t)(w >> 24), a), 127.0f);
            reinterpret_cast<float4*>(out)[t] = r;
        } else {
            for (long long i = i0; i < n; ++i) out[i] = __fdiv_rn(__fmul_rn((float)q[i], a), 127.0f);
        }
    }
}

// Dequantisation for blocks of at least 256 values: a persistent 256-thread
// CTA takes one block at a time, first the 129 values RN32(RN32(q * absmax) /
// 127) for q = 0..128 into shared memory (one division each; -q gives the
// negated value, since both roundings are symmetric), then the block's codes,
// four per thread per step (one 32-bit load, one 16-byte store), by table
// look-up.  Two tables alternate, so one barrier per block suffices.
// B % 4 == 0, so a block's codes start on a 4-byte boundary.
__global__ void __launch_bounds__(256) k_block_dequant_table(const int8_t* __restrict__ q, const float* __restrict__ absmax,
                                                             long long n, int B, float* __restrict__ out) {
    __shared__ float tbl[2][129];
    const long long nblocks = (n + B - 1) / B;
    int par = 0;
    for (long long b = blockIdx.x; b < nblocks; b += gridDim.x) {
        const float a = __ldg(absmax + b);
        if (threadIdx.x < 129) tbl[par][threadIdx.x] = __fdiv_rn(__fmul_rn((float)threadIdx.x, a), 127.0f);
        __syncthreads();  // (the other table was last read before the previous barrier)
        const long long lo = b * (long long)B;
        const int len = (int)min((long long)B, n - lo);
        const float* t = tbl[par];
        for (int e = 4 * threadIdx.x; e < len; e += 1024) {
            if (e + 3 < len) {
                const uint32_t w = __ldg(reinterpret_cast<const uint32_t*>(q + lo) + e / 4);
                float4 r;
                const int c0 = (int8_t)(w & 0xFFu), c1 = (int8_t)((w >> 8) & 0xFFu);
                const int c2 = (int8_t)((w >> 16) & 0xFFu), c3 = (int8_t)(w >> 24);
                r.x = c0 < 0 ? -t[-c0] : t[c0];
                r.y = c1 < 0 ? -t[-c1] : t[c1];
                r.z = c2 < 0 ? -t[-c2] : t[c2];
                r.w = c3 < 0 ? -t[-c3] : t[c3];
                *reinterpret_cast<float4*>(out + lo + e) = r;
            } else {
                for (int j = e; j < len; ++j) {
                    const int c = q[lo + j];
                    out[lo + j] = c < 0 ? -t[-c] : t[c];
                }
            }
        }
        par ^= 1;
    }
}

}  // namespace i8mm
