// dropout.cuh -- LoRA dropout on the branch input X (the base path is left
// unchanged): the keep mask, the dropped copy X * keep (exact in bf16; the
// scale c of kept values is applied in fp32 where T, dA and the LoRA term of
// dX are formed), and the masked LoRA term of dX.
//
// Element e = m K + k of X is kept iff field >= t, t = llrint(p 2^16), where
// field is 16-bit field (e mod 16) of the Philox4x64-10 output for counter
// (e div 16, offset, 0, 0) and key (seed, 0) (Salmon, Moraes, Dror and Shaw,
// SC 2011: per round (hi0, lo0) = M0 c0, (hi1, lo1) = M1 c2 as 128-bit
// products, c = (hi1 ^ c1 ^ k0, lo1, hi0 ^ c3 ^ k1, lo0), and the key adds
// the Weyl increments between rounds); field 4i + j is bits 16j..16j+15 of
// output i.  Kept values are scaled by c = fl32(1 / (1 - p)).  One generator
// call serves 16 consecutive elements (K % 64 == 0 keeps every group in one
// row); the backward generates the mask once, as a bitmask (bit e % 16 of
// 16-bit word e / 16) that its later kernels read.
#pragma once
#include "common.cuh"

namespace qnf4 {
namespace drop {

struct Params {
    uint64_t seed, offset;
    uint32_t t;        // keep iff field >= t
    float c;           // scale of kept values
};

__device__ __forceinline__ void philox4x64(uint64_t c0, uint64_t c1, uint64_t k0, uint64_t out[4]) {
    constexpr uint64_t M0 = 0xD2E7470EE14C6C93ull, M1 = 0xCA5A826395121157ull;
    constexpr uint64_t W0 = 0x9E3779B97F4A7C15ull, W1 = 0xBB67AE8584CAA73Bull;
    uint64_t c2 = 0, c3 = 0, k1 = 0;
#pragma unroll
    for (int round = 0; round < 10; ++round) {
        if (round > 0) { k0 += W0; k1 += W1; }
        const uint64_t hi0 = __umul64hi(M0, c0), lo0 = M0 * c0;
        const uint64_t hi1 = __umul64hi(M1, c2), lo1 = M1 * c2;
        const uint64_t n0 = hi1 ^ c1 ^ k0, n2 = hi0 ^ c3 ^ k1;
        c0 = n0; c1 = lo1; c2 = n2; c3 = lo0;
    }
    out[0] = c0; out[1] = c1; out[2] = c2; out[3] = c3;
}

// keep bits of elements 16 e16 .. 16 e16 + 15 (bit j = element 16 e16 + j)
__device__ __forceinline__ uint32_t keep16(const Params& d, uint64_t e16) {
    uint64_t o[4];
    philox4x64(e16, d.offset, d.seed, o);
    uint32_t bits = 0;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
        const uint32_t field = (uint32_t)(o[j >> 2] >> (16 * (j & 3))) & 0xffffu;
        bits |= (field >= d.t ? 1u : 0u) << j;
    }
    return bits;
}

// Xd [M, K] = X where kept, 0 where dropped; when mask is given, also its
// keep bits (one 16-bit word per 16 elements).  One thread per 16 elements.
__global__ void __launch_bounds__(256) k_dropout_x(const uint16_t* __restrict__ X, int64_t total16,
                                                   uint16_t* __restrict__ Xd, uint16_t* __restrict__ mask,
                                                   Params d) {
    for (int64_t e16 = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e16 < total16;
         e16 += (int64_t)gridDim.x * blockDim.x) {
        const uint32_t keep = keep16(d, (uint64_t)e16);
        const uint4 x0 = ldg_nc_v4(X + 16 * e16), x1 = ldg_nc_v4(X + 16 * e16 + 8);
        const uint32_t xw[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
        uint32_t o[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const uint32_t lo = (keep >> (2 * j)) & 1u ? (xw[j] & 0xffffu) : 0u;
            const uint32_t hi = (keep >> (2 * j + 1)) & 1u ? (xw[j] & 0xffff0000u) : 0u;
            o[j] = lo | hi;
        }
        uint4* dst = reinterpret_cast<uint4*>(Xd + 16 * e16);
        dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
        dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
        if (mask) mask[e16] = (uint16_t)keep;
    }
}

// keep bit of element e from the bitmask
__device__ __forceinline__ uint32_t mask_bit(const uint16_t* mask, uint64_t e) {
    return ((uint32_t)__ldg(mask + (e >> 4)) >> (e & 15)) & 1u;
}

// dX [M, K] += masked LoRA term, in place on the bf16 base dY W' (written by
// the fused kernel with its LoRA steps switched off):
//   l  = sum_j U[m, j] A[j, k]   (fp32, increasing j)
//   dX = bf16_rne(fmaf(sc, l, fl32(dX)))  where kept, dX unchanged where dropped,
//   sc = fl32(s c).
// A CTA takes 32 rows x 256 columns; thread (warp w, lane l) owns rows
// 4w..4w+3 and columns 8l..8l+7.  Chunks of 64 LoRA terms are staged in
// shared memory: A[j, tile columns] as bf16 by cp.async (read as one 16-byte
// vector per lane), U[tile rows, j] transposed to fp32 [j][row] (a broadcast
// read), so each A element is read from L2 once per 32 rows.
struct DxArgs {
    uint16_t* dX;          // [M, K]
    const float* U;        // [M, ldu] fp32
    int64_t ldu;
    const uint16_t* A;     // [r, K]
    const uint16_t* mask;  // keep bits of [M, K] (k_dropout_x)
    int64_t M, K;
    int r;
    float sc;
};

constexpr int DX_TM = 32, DX_TK = 256, DX_JC = 64, DX_THREADS = 256;
constexpr int DX_SMEM = DX_JC * DX_TK * 2 + DX_JC * DX_TM * 4;

__global__ void __launch_bounds__(DX_THREADS) k_dx_lora_dropout(const DxArgs a) {
    extern __shared__ __align__(16) uint8_t smem[];
    float* sU = reinterpret_cast<float*>(smem + DX_JC * DX_TK * 2);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t m0 = (int64_t)blockIdx.x * DX_TM, k0 = (int64_t)blockIdx.y * DX_TK;
    float acc[4][8];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[i][c] = 0.f;
    for (int j0 = 0; j0 < a.r; j0 += DX_JC) {
        const int jc = min(DX_JC, a.r - j0);
        if (j0 > 0) __syncthreads();
        for (int i = tid; i < jc * (DX_TK / 8); i += DX_THREADS) {
            const int jj = i / (DX_TK / 8), v = i % (DX_TK / 8);
            const int64_t k = k0 + 8 * v;
            const bool ok = k < a.K;
            const uint16_t* src = ok ? a.A + (int64_t)(j0 + jj) * a.K + k : a.A;
            const uint32_t dst = smem_u32(smem + (jj * DX_TK + 8 * v) * 2);
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(ok ? 16 : 0)
                         : "memory");
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
        for (int i = tid; i < jc * DX_TM; i += DX_THREADS) {
            const int jj = i / DX_TM, row = i % DX_TM;
            const int64_t m = m0 + row;
            sU[jj * DX_TM + row] = m < a.M ? __ldg(a.U + m * a.ldu + j0 + jj) : 0.f;
        }
        asm volatile("cp.async.wait_all;" ::: "memory");
        __syncthreads();
        for (int jj = 0; jj < jc; ++jj) {
            const uint4 x = *reinterpret_cast<const uint4*>(smem + (jj * DX_TK + 8 * lane) * 2);
            const float4 u = *reinterpret_cast<const float4*>(sU + jj * DX_TM + 4 * warp);
            const float av[8] = {bf16lo_to_f32(x.x), bf16hi_to_f32(x.x), bf16lo_to_f32(x.y), bf16hi_to_f32(x.y),
                                 bf16lo_to_f32(x.z), bf16hi_to_f32(x.z), bf16lo_to_f32(x.w), bf16hi_to_f32(x.w)};
            const float uv[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int c = 0; c < 8; ++c) acc[i][c] = __fmaf_rn(uv[i], av[c], acc[i][c]);
        }
    }
    const int64_t k = k0 + 8 * lane;
    if (k >= a.K) return;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int64_t m = m0 + 4 * warp + i;
        if (m >= a.M) break;
        const uint64_t e = (uint64_t)(m * a.K + k);     // a multiple of 8: bits e % 16 .. e % 16 + 7
        const uint32_t keep = ((uint32_t)__ldg(a.mask + (e >> 4)) >> (e & 15)) & 0xffu;
        uint4* p = reinterpret_cast<uint4*>(a.dX + m * a.K + k);
        const uint4 b = *p;
        const uint32_t bw[4] = {b.x, b.y, b.z, b.w};
        uint32_t o[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            float lo = bf16lo_to_f32(bw[q]), hi = bf16hi_to_f32(bw[q]);
            if ((keep >> (2 * q)) & 1u) lo = __fmaf_rn(a.sc, acc[i][2 * q], lo);
            if ((keep >> (2 * q + 1)) & 1u) hi = __fmaf_rn(a.sc, acc[i][2 * q + 1], hi);
            o[q] = pack_bf16x2(lo, hi);
        }
        *p = make_uint4(o[0], o[1], o[2], o[3]);
    }
}

}  // namespace drop
}  // namespace qnf4
