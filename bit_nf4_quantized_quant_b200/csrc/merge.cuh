// merge.cuh -- dequantize-and-merge: the dense bf16 weight of a trained
// QLoRA layer, W_merged = bf16_rne(fmaf(s, d, w')), d = sum_j B[n, j] A[j, k]
// (fp32, one fma per term in increasing j from 0), w' = bf16_rne(L[q] c').
//
// The LoRA product is r fused multiply-adds per output in a fixed order, so
// the kernel runs them on the fp32 pipe (the tensor cores' internal summation
// order is not specified, and the result must be reproducible bit for bit).
// A CTA computes a 64-row x 256-column tile; thread (warp w, lane l) owns
// rows 8w..8w+7 and columns 8l..8l+7 (one packed 32-bit word per row, one
// 16-byte store per row).  Chunks of 64 LoRA terms are staged in shared
// memory as fp32: A[j, tile columns] (read as two 16-byte vectors per lane:
// 512 contiguous bytes per warp) and B[tile rows, j] transposed to [j][row]
// (a broadcast read).  Per term a thread issues 4 shared loads and 64 fmas.
#pragma once
#include "common.cuh"

namespace qnf4 {
namespace merge {

constexpr int TM = 64;          // rows of W per CTA
constexpr int TK = 256;         // columns of W per CTA
constexpr int JC = 64;          // LoRA terms per shared-memory chunk
constexpr int kThreads = 256;
constexpr int SMEM_BYTES = (JC * TK + JC * TM + 16) * 4;

struct Args {
    const uint8_t* packed;
    const int8_t* codes;
    const float* scale;
    const float* mean;
    const uint16_t* A;          // [r, K]
    const uint16_t* B;          // [N, r]
    uint16_t* out;              // [N, K]
    int64_t N, K;
    int r;
    float s;
};

__global__ void __launch_bounds__(kThreads, 2) k_dequant_merge(const Args a, NF4Tables tab) {
    extern __shared__ __align__(16) float smem[];
    float* sA = smem;                       // [JC][TK]
    float* sB = sA + JC * TK;               // [JC][TM]
    float* sL = sB + JC * TM;               // [16]
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid < 16) sL[tid] = tab.L[tid];
    const int64_t n0 = (int64_t)blockIdx.x * TM, k0 = (int64_t)blockIdx.y * TK;

    float acc[8][8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[i][c] = 0.f;

    for (int j0 = 0; j0 < a.r; j0 += JC) {
        const int jc = min(JC, a.r - j0);
        __syncthreads();                    // the previous chunk has been consumed
        // A[j0 + jj, k0 + 8 v .. +8] -> sA[jj][8 v ..]: 32 vectors of 8 per row
        for (int i = tid; i < jc * (TK / 8); i += kThreads) {
            const int jj = i / (TK / 8), v = i % (TK / 8);
            const int64_t k = k0 + 8 * v;
            uint4 x = make_uint4(0, 0, 0, 0);
            if (k < a.K) x = ldg_nc_v4(a.A + (int64_t)(j0 + jj) * a.K + k);
            float4* d = reinterpret_cast<float4*>(sA + jj * TK + 8 * v);
            d[0] = make_float4(bf16lo_to_f32(x.x), bf16hi_to_f32(x.x), bf16lo_to_f32(x.y), bf16hi_to_f32(x.y));
            d[1] = make_float4(bf16lo_to_f32(x.z), bf16hi_to_f32(x.z), bf16lo_to_f32(x.w), bf16hi_to_f32(x.w));
        }
        // B[n0 + row, j0 + jj] -> sB[jj][row] (consecutive threads: consecutive rows, no bank conflicts)
        for (int i = tid; i < jc * TM; i += kThreads) {
            const int jj = i / TM, row = i % TM;
            const int64_t n = n0 + row;
            float v = 0.f;
            if (n < a.N) v = bf16lo_to_f32(__ldg(a.B + n * a.r + j0 + jj));
            sB[jj * TM + row] = v;
        }
        __syncthreads();
        for (int jj = 0; jj < jc; ++jj) {
            const float4 a0 = *reinterpret_cast<const float4*>(sA + jj * TK + 8 * lane);
            const float4 a1 = *reinterpret_cast<const float4*>(sA + jj * TK + 8 * lane + 4);
            const float4 b0 = *reinterpret_cast<const float4*>(sB + jj * TM + 8 * warp);
            const float4 b1 = *reinterpret_cast<const float4*>(sB + jj * TM + 8 * warp + 4);
            const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
            const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
            for (int i = 0; i < 8; ++i)
#pragma unroll
                for (int c = 0; c < 8; ++c) acc[i][c] = __fmaf_rn(bv[i], av[c], acc[i][c]);
        }
    }

    // epilogue: w' of the 8 x 8 outputs, then one fma with the scaled LoRA sum
    const int64_t k = k0 + 8 * lane;
    if (k >= a.K) return;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int64_t n = n0 + 8 * warp + i;
        if (n >= a.N) break;
        const int64_t e = n * a.K + k;                       // flat index of the first of 8 weights
        const uint32_t word = ldg_nc_u32(a.packed + e / 2);
        const int64_t b = e / kBlock;
        const float cp = __fmaf_rn((float)__ldg(a.codes + b), __ldg(a.scale + b / kGroup), __ldg(a.mean + b / kGroup));
        uint32_t o[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const uint32_t byte = (word >> (8 * j)) & 0xffu;
            // element 2j is the high nibble of byte j
            const float w0 = __bfloat162float(__float2bfloat16_rn(__fmul_rn(sL[byte >> 4], cp)));
            const float w1 = __bfloat162float(__float2bfloat16_rn(__fmul_rn(sL[byte & 15u], cp)));
            o[j] = pack_bf16x2(__fmaf_rn(a.s, acc[i][2 * j], w0), __fmaf_rn(a.s, acc[i][2 * j + 1], w1));
        }
        *reinterpret_cast<uint4*>(a.out + e) = make_uint4(o[0], o[1], o[2], o[3]);
    }
}

}  // namespace merge
}  // namespace qnf4
