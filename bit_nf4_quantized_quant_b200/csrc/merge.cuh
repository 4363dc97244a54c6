// merge.cuh -- dequantize-and-merge: the dense bf16 weight of a trained
// QLoRA layer, W_merged = bf16_rne(fmaf(s, d, w')), d = sum_j B[n, j] A[j, k]
// (fp32, one fma per term in increasing j from 0), w' = bf16_rne(L[q] c').
//
// The LoRA product is r fused multiply-adds per output in a fixed order, so
// the kernel runs them on the fp32 pipe (the tensor cores' internal summation
// order is not specified, and the result must be reproducible bit for bit).
// A CTA computes a 32-row x 256-column tile; thread (warp w, lane l) owns
// rows 4w..4w+3 and columns 8l..8l+7 (one packed 32-bit word per row, one
// 16-byte store per row); 32 accumulators per thread leave room for four
// CTAs per SM, whose memory waits then overlap each other's arithmetic.
//   - Every global read of a chunk is in flight at once, so a CTA waits for
//     one memory round trip: the tile's packed nibbles (32 x 128 B) and the
//     chunk's rows of A (bf16) are copied to shared memory with cp.async,
//     while each thread loads the constant inputs of one (row, block) of the
//     tile and its share of B's chunk into registers.
//   - Chunks of 64 LoRA terms: A[j, tile columns] stays bf16 in shared memory
//     (one 16-byte vector per lane, widened in registers), B[tile rows, j] is
//     stored transposed as fp32 [j][row] (a broadcast read).  Per term a
//     thread issues 2 shared loads, 8 widening ops and 32 fmas.
// Measured bound: instruction issue (80 % of issue slots busy at r = 16),
// about 46 instructions per output against the 16 fmas the fixed-order sum
// needs; the per-weight decode and bf16 rounding of w' are most of the rest.
// Staging A as fp32 once per CTA measured slower.
//   - Epilogue: decode from shared memory, one fma per output, 16-byte stores.
#pragma once
#include "common.cuh"

namespace qnf4 {
namespace merge {

constexpr int TM = 32;          // rows of W per CTA
constexpr int RT = TM / 8;      // rows per thread (8 warps)
constexpr int TK = 256;         // columns of W per CTA
constexpr int JC = 64;          // LoRA terms per shared-memory chunk
constexpr int kThreads = 256;
constexpr int OFF_A = 0;                              // bf16 [JC][TK]
constexpr int OFF_B = OFF_A + JC * TK * 2;            // fp32 [JC][TM]
constexpr int OFF_P = OFF_B + JC * TM * 4;            // packed [TM][TK / 2]
constexpr int OFF_C = OFF_P + TM * TK / 2;            // c' [TM][TK / 64]
constexpr int OFF_L = OFF_C + TM * (TK / 64) * 4;     // L [16]
constexpr int SMEM_BYTES = OFF_L + 16 * 4;

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

__global__ void __launch_bounds__(kThreads, 4) k_dequant_merge(const Args a, NF4Tables tab) {
    extern __shared__ __align__(16) uint8_t smem[];
    float* sB = reinterpret_cast<float*>(smem + OFF_B);
    float* sC = reinterpret_cast<float*>(smem + OFF_C);
    float* sL = reinterpret_cast<float*>(smem + OFF_L);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t n0 = (int64_t)blockIdx.x * TM, k0 = (int64_t)blockIdx.y * TK;
    const int64_t nblk = a.K / kBlock;

    // ---- packed tile by cp.async (zero-filled beyond N or K)
    for (int i = tid; i < TM * (TK / 32); i += kThreads) {      // 16-byte chunks: 8 per row
        const int row = i >> 3, ch = i & 7;
        const int64_t n = n0 + row, k = k0 + 32 * ch;
        const bool v = n < a.N && k < a.K;
        const uint8_t* src = v ? a.packed + (n * a.K + k) / 2 : a.packed;
        const uint32_t dst = smem_u32(smem + OFF_P + row * (TK / 2) + 16 * ch);
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(v ? 16 : 0)
                     : "memory");
    }
    // ---- block-constant inputs of (row tid / 4, block tid % 4), in registers until used
    const int crow = tid >> 2, cbl = tid & 3;
    int ccode = 0;
    float cscale = 0.f, cmean = 0.f;
    if (crow < TM) {
        const int64_t n = n0 + crow, kb = k0 / kBlock + cbl;
        if (n < a.N && kb < nblk) {
            const int64_t b = n * nblk + kb;
            ccode = __ldg(a.codes + b);
            cscale = __ldg(a.scale + b / kGroup);
            cmean = __ldg(a.mean + b / kGroup);
        }
    }
    // constant indices: a thread-dependent index into the by-value table would make every
    // thread copy the whole parameter to local memory first
    if (warp == 0) {
#pragma unroll
        for (int q = 0; q < 16; ++q)
            if (lane == q) sL[q] = tab.L[q];
    }

    float acc[RT][8];
#pragma unroll
    for (int i = 0; i < RT; ++i)
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[i][c] = 0.f;

    for (int j0 = 0; j0 < a.r; j0 += JC) {
        const int jc = min(JC, a.r - j0);
        if (j0 > 0) __syncthreads();        // the previous chunk has been consumed
        // A[j0 + jj, k0 + 8 v .. +8] -> sA[jj][8 v ..] (bf16) by cp.async: 32 vectors per row
        for (int i = tid; i < jc * (TK / 8); i += kThreads) {
            const int jj = i / (TK / 8), v = i % (TK / 8);
            const int64_t k = k0 + 8 * v;
            const bool ok = k < a.K;
            const uint16_t* src = ok ? a.A + (int64_t)(j0 + jj) * a.K + k : a.A;
            const uint32_t dst = smem_u32(smem + OFF_A + (jj * TK + 8 * v) * 2);
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(ok ? 16 : 0)
                         : "memory");
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
        // B[n0 + row, j0 + jj]: loaded into registers (all in flight), then -> sB[jj][row]
        float bl[JC * TM / kThreads];
#pragma unroll
        for (int u = 0; u < JC * TM / kThreads; ++u) {
            const int i = tid + u * kThreads, jj = i / TM, row = i % TM;
            const int64_t n = n0 + row;
            bl[u] = (jj < jc && n < a.N) ? bf16lo_to_f32(__ldg(a.B + n * a.r + j0 + jj)) : 0.f;
        }
#pragma unroll
        for (int u = 0; u < JC * TM / kThreads; ++u) {
            const int i = tid + u * kThreads, jj = i / TM, row = i % TM;
            if (jj < jc) sB[jj * TM + row] = bl[u];
        }
        if (j0 == 0 && crow < TM) sC[crow * (TK / 64) + cbl] = __fmaf_rn((float)ccode, cscale, cmean);
        asm volatile("cp.async.wait_all;" ::: "memory");
        __syncthreads();
        const uint8_t* sArow = smem + OFF_A + 16 * lane;
        for (int jj = 0; jj < jc; ++jj) {
            const uint4 x = *reinterpret_cast<const uint4*>(sArow + jj * TK * 2);
            const float4 b0 = *reinterpret_cast<const float4*>(sB + jj * TM + RT * warp);
            const float av[8] = {bf16lo_to_f32(x.x), bf16hi_to_f32(x.x), bf16lo_to_f32(x.y), bf16hi_to_f32(x.y),
                                 bf16lo_to_f32(x.z), bf16hi_to_f32(x.z), bf16lo_to_f32(x.w), bf16hi_to_f32(x.w)};
            const float bv[RT] = {b0.x, b0.y, b0.z, b0.w};
#pragma unroll
            for (int i = 0; i < RT; ++i)
#pragma unroll
                for (int c = 0; c < 8; ++c) acc[i][c] = __fmaf_rn(bv[i], av[c], acc[i][c]);
        }
    }
    // the packed tile and every c' landed before the last chunk's barrier

    // ---- epilogue: w' of the RT x 8 outputs, then one fma with the scaled LoRA sum
    const int64_t k = k0 + 8 * lane;
    if (k >= a.K) return;
#pragma unroll
    for (int i = 0; i < RT; ++i) {
        const int row = RT * warp + i;
        const int64_t n = n0 + row;
        if (n < a.N) {
            const uint32_t word = lds_u32(smem_u32(smem + OFF_P + row * (TK / 2) + 4 * lane));
            const float cp = sC[row * (TK / 64) + (lane >> 3)];
            uint32_t o[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const uint32_t byte = (word >> (8 * j)) & 0xffu;
                // element 2j is the high nibble of byte j
                const float w0 = __bfloat162float(__float2bfloat16_rn(__fmul_rn(sL[byte >> 4], cp)));
                const float w1 = __bfloat162float(__float2bfloat16_rn(__fmul_rn(sL[byte & 15u], cp)));
                o[j] = pack_bf16x2(__fmaf_rn(a.s, acc[i][2 * j], w0), __fmaf_rn(a.s, acc[i][2 * j + 1], w1));
            }
            *reinterpret_cast<uint4*>(a.out + n * a.K + k) = make_uint4(o[0], o[1], o[2], o[3]);
        }
    }
}

}  // namespace merge
}  // namespace qnf4
