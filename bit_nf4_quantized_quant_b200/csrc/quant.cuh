// quant.cuh -- NF4 quantize + double-quantize and dense dequantize kernels.
//
// Both are HBM-bound streaming kernels (2 B read + 0.516 B written per weight,
// and the reverse).  Layout of the quantized weight: see nf4dq_weight in
// include/qlora_nf4.h.
#pragma once
#include "common.cuh"

namespace qnf4 {

// Nearest NF4 level of a normalised value x in [-1, 1]: the number of decision
// thresholds that x lies strictly above, found by a 4-step binary search over
// the sorted thresholds (the result equals the count exactly; a value on a
// threshold takes the lower level).  Thresholds 3, 7 and 11 come from the
// parameter bank, the last two steps index a 15-entry shared-memory copy
// (16 distinct words in 16 banks: no bank conflicts).
__device__ __forceinline__ uint32_t nf4_encode(float x, const NF4Tables& tab, const float* s_m) {
    uint32_t q = (x > tab.m[7]) ? 8u : 0u;
    float t = q ? tab.m[11] : tab.m[3];
    q += (x > t) ? 4u : 0u;
    q += (x > s_m[q + 1]) ? 2u : 0u;
    q += (x > s_m[q]) ? 1u : 0u;
    return q;
}

// The exact level of w in a block with absmax c (the slow path of the encoder
// below): x = fl32(w / c) by IEEE division, then the 4-step search; c = 0
// gives rank 7, the zero level of both codebooks.  Kept out of line: it runs for about one weight in 10^5.
__device__ __noinline__ uint32_t nf4_encode_exact(float w, float c, float m3, float m7, float m11,
                                                  const float* s_m) {
    if (c == 0.f) return 7u;
    const float x = __fdiv_rn(w, c);
    uint32_t q = (x > m7) ? 8u : 0u;
    const float t = q ? m11 : m3;
    q += (x > t) ? 4u : 0u;
    q += (x > s_m[q + 1]) ? 2u : 0u;
    q += (x > s_m[q]) ? 1u : 0u;
    return q;
}

// One CTA (8 warps) per double-quant group of 256 blocks (16384 weights),
// grid-stride over groups.  Warp w owns blocks [32w, 32w+32) of the group; a
// block is handled by 8 lanes of 8 weights each (16-byte loads, coalesced
// 512 B per warp instruction).  Warp 0 then runs the group's second-level
// quantization with the fp64 pairwise tree held in registers: lane l keeps
// slots l, l+32, ..., l+224, so strides 128, 64, 32 are in-register adds and
// strides 16..1 are shuffles -- the same association order as the definition.
//
// FP4 (kFP4): the same search yields the level's rank among the 15 distinct
// FP4 levels in ascending order (threshold 14 is +inf); its nibble is the
// E2M1 bit pattern of that level: ranks 0..6 are -1 .. -1/12 (codes 15..9),
// rank 7 is +0 (code 0), ranks 8..14 are 1/12 .. 1 (codes 1..7).
template <bool kFP4>
__device__ __forceinline__ uint32_t rank_to_nibble(uint32_t q) {
    if (!kFP4) return q;
    return q < 7u ? 15u - q : q - 7u;
}

template <bool kFP4>
__global__ void __launch_bounds__(256, 4) k_quantize_dq(const uint16_t* __restrict__ W, int64_t nblocks,
                                                     uint8_t* __restrict__ packed, int8_t* __restrict__ codes,
                                                     float* __restrict__ scale, float* __restrict__ mean,
                                                     NF4Tables tab, const __grid_constant__ EncTables enc) {
    __shared__ float s_c[kGroup];
    __shared__ float s_m[16];
    __shared__ float2 s_enc[kEncBuckets];          // (threshold, levels below) per bucket
    // constant indices (a thread-dependent index into the by-value table would make every
    // thread copy the whole parameter to local memory first)
#pragma unroll
    for (int q = 0; q < 15; ++q)
        if (threadIdx.x == q) s_m[q] = tab.m[q];
    if (threadIdx.x == 15) s_m[15] = INFINITY;
    for (int b = threadIdx.x; b < kEncBuckets; b += blockDim.x)
        s_enc[b] = make_float2(enc.thr[b], __uint_as_float(enc.qb[b]));
    __syncthreads();

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int part = lane & 7, sub = lane >> 3;
    const int64_t ngroups = cdiv(nblocks, kGroup);

    for (int64_t g = blockIdx.x; g < ngroups; g += gridDim.x) {
        const int64_t b0 = g * kGroup;
        const int nb = (int)((nblocks - b0) < kGroup ? (nblocks - b0) : kGroup);

        uint4 v[8];
#pragma unroll
        for (int it = 0; it < 8; ++it) {
            const int bl = warp * 32 + it * 4 + sub;
            if (bl < nb) v[it] = ldg_nc_v4(W + (b0 + bl) * kBlock + part * 8);
            else v[it] = make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int it = 0; it < 8; ++it) {
            const int bl = warp * 32 + it * 4 + sub;
            const uint32_t wv[4] = {v[it].x, v[it].y, v[it].z, v[it].w};
            float w[8];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                w[2 * j] = bf16lo_to_f32(wv[j]);
                w[2 * j + 1] = bf16hi_to_f32(wv[j]);
            }
            float c = 0.f;
#pragma unroll
            for (int j = 0; j < 8; ++j) c = fmaxf(c, fabsf(w[j]));
            c = fmaxf(c, __shfl_xor_sync(0xffffffffu, c, 1));
            c = fmaxf(c, __shfl_xor_sync(0xffffffffu, c, 2));
            c = fmaxf(c, __shfl_xor_sync(0xffffffffu, c, 4));
            if (bl < nb) {
                // Fast path: x' = w * (1/c) is within 1.5 * 2^-23 of x = fl32(w / c) (|x| <= 1),
                // so when x' is more than 2^-20 from its bucket's threshold, x and x' sit on the
                // same side of it and the level is qb + (x' > thr).  Otherwise (or c = 0, a
                // reciprocal that is not finite, NaN) the exact quotient takes the 4-step search.
                const float rcp = __frcp_rn(c);
                const bool fast_blk = c > 0.f && rcp < INFINITY;
                uint32_t word = 0, slow = fast_blk ? 0u : 0xffu;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const float x = __fmul_rn(w[j], rcp);
                    // round(64 x + 64) from the low bits of 64 x + 64 + 1.5 * 2^23
                    const uint32_t b = min(__float_as_uint(__fmaf_rn(x, 64.f, 12582976.f)) - 0x4B400000u, 128u);
                    const float2 e = s_enc[b];
                    const float d = __fsub_rn(x, e.x);
                    if (!(fabsf(d) > 9.5367431640625e-07f)) slow |= 1u << j;     // 2^-20 (also NaN)
                    const uint32_t q = rank_to_nibble<kFP4>(__float_as_uint(e.y) + (d > 0.f ? 1u : 0u));
                    // element 2i -> high nibble of byte i (little-endian word)
                    word |= q << ((j >> 1) * 8 + ((j & 1) ? 0 : 4));
                }
                // rare: weights near a threshold (or a block the fast path cannot take)
                if (slow) {
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        if ((slow >> j) & 1u) {
                            const int sh = (j >> 1) * 8 + ((j & 1) ? 0 : 4);
                            const uint32_t q =
                                rank_to_nibble<kFP4>(nf4_encode_exact(w[j], c, tab.m[3], tab.m[7], tab.m[11], s_m));
                            word = (word & ~(15u << sh)) | (q << sh);
                        }
                    }
                }
                *reinterpret_cast<uint32_t*>(packed + ((b0 + bl) * kBlock + part * 8) / 2) = word;
                if (part == 0) s_c[bl] = c;
            }
        }
        __syncthreads();

        if (warp == 0) {
            double s[8];
            float cv[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int idx = j * 32 + lane;
                cv[j] = (idx < nb) ? s_c[idx] : 0.f;
                s[j] = (double)cv[j];
            }
#pragma unroll
            for (int j = 0; j < 4; ++j) s[j] = __dadd_rn(s[j], s[j + 4]);   // stride 128
#pragma unroll
            for (int j = 0; j < 2; ++j) s[j] = __dadd_rn(s[j], s[j + 2]);   // stride 64
            double acc = __dadd_rn(s[0], s[1]);                              // stride 32
#pragma unroll
            for (int off = 16; off >= 1; off >>= 1)                          // strides 16..1
                acc = __dadd_rn(acc, __shfl_down_sync(0xffffffffu, acc, off));
            acc = __shfl_sync(0xffffffffu, acc, 0);
            const float mu = __double2float_rn(__ddiv_rn(acc, (double)nb));
            float d[8], dmax = 0.f;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                d[j] = __fsub_rn(cv[j], mu);
                if (j * 32 + lane < nb) dmax = fmaxf(dmax, fabsf(d[j]));
            }
#pragma unroll
            for (int off = 16; off >= 1; off >>= 1) dmax = fmaxf(dmax, __shfl_xor_sync(0xffffffffu, dmax, off));
            const float sc = __fdiv_rn(dmax, 127.0f);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int idx = j * 32 + lane;
                if (idx < nb) {
                    int code = 0;
                    if (sc != 0.f) {
                        float t = rintf(__fdiv_rn(d[j], sc));
                        t = fminf(fmaxf(t, -127.f), 127.f);
                        code = (int)t;
                    }
                    codes[b0 + idx] = (int8_t)code;
                }
            }
            if (lane == 0) {
                scale[g] = sc;
                mean[g] = mu;
            }
        }
        __syncthreads();
    }
}

// Dense dequantization, coalesced on both sides: a warp takes a segment of
// 256 packed 32-bit words (2048 weights) per iteration, lane l the words
// l + 32 k (k = 0..7), so each of its eight 4-byte loads and eight 16-byte
// stores (8 weights of word w go to bytes [16 w, 16 w + 16) of the output)
// covers one contiguous stretch across the warp; all loads of a segment are
// issued before the first store.  W' = bf16_rne(L[q] * c'_b),
// c'_b = fmaf(code_b, scale_g, mean_g).
constexpr int kDqWarpWords = 256;

__global__ void __launch_bounds__(256) k_dequant(const uint8_t* __restrict__ packed,
                                                 const int8_t* __restrict__ codes,
                                                 const float* __restrict__ scale, const float* __restrict__ mean,
                                                 int64_t nwords, uint16_t* __restrict__ out, NF4Tables tab) {
    __shared__ float s_L[16];
    if (threadIdx.x < 16) s_L[threadIdx.x] = tab.L[threadIdx.x];
    __syncthreads();
    const int lane = threadIdx.x & 31;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    const uint32_t* pw = reinterpret_cast<const uint32_t*>(packed);
    for (int64_t seg = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; seg * kDqWarpWords < nwords;
         seg += nwarps) {
        const int64_t w0 = seg * kDqWarpWords + lane;
        uint32_t v[8];
        int cd[8];
        float sc[8], mn[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const int64_t wi = w0 + 32 * k;                 // 8 weights: block wi / 8, group wi / 2048
            v[k] = 0u; cd[k] = 0; sc[k] = 0.f; mn[k] = 0.f;
            if (wi < nwords) {
                v[k] = ldg_nc_u32(pw + wi);
                cd[k] = __ldg(codes + (wi >> 3));
                sc[k] = __ldg(scale + (wi >> 11));
                mn[k] = __ldg(mean + (wi >> 11));
            }
        }
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const int64_t wi = w0 + 32 * k;
            if (wi < nwords) {
                const float cp = __fmaf_rn((float)cd[k], sc[k], mn[k]);
                uint32_t o[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const uint32_t byte = (v[k] >> (8 * j)) & 0xffu;
                    const float hi = __fmul_rn(s_L[byte >> 4], cp);     // element 2j
                    const float lo = __fmul_rn(s_L[byte & 15u], cp);    // element 2j+1
                    o[j] = pack_bf16x2(hi, lo);
                }
                *reinterpret_cast<uint4*>(out + wi * 8) = make_uint4(o[0], o[1], o[2], o[3]);
            }
        }
    }
}

}  // namespace qnf4
