// small.cuh -- small-M (decode / GEMV-shaped) forward and backward-dX kernels.
//
// For a few tokens the layer is bound by streaming the 4.13-bit weight from
// HBM, so the kernels are built around the cost of turning nibbles into bf16
// MMA operands:
//   * a shared-memory "pair table" maps a packed byte (two nibbles) straight to
//     a bf16x2 register holding the two *unscaled* NF4 levels; it is replicated
//     once per lane (entry v of lane l at word 32 v + l), so a warp-wide lookup
//     never has a bank conflict;
//   * the per-block constant c'_b is folded out of the inner product: each
//     64-wide block is reduced on the tensor cores (mma.sync m16n8k16, fp32)
//     into a fresh accumulator that is then added with one FMA per output,
//     y += c'_b * sum_{k in b} L[q_k] x_k   (forward), or applied to the other
//     operand (backward: dY[m, n] * c'_{n, b} rounded to bf16).
// The k order inside one m16n8k16 MMA is permuted so that each lane's
// fragment comes from contiguous packed bytes; the activation fragment is
// loaded with the same permutation, so the sum is unchanged.
#pragma once
#include "common.cuh"

namespace qnf4 {

constexpr int kPairTableWords = 256 * 32;
constexpr int kSmallThreads = 512;
constexpr int kSmallWarps = kSmallThreads / 32;

__device__ __forceinline__ void build_pair_table(uint32_t* s_tab, float* s_L, const NF4Tables& tab) {
    if (threadIdx.x < 16) s_L[threadIdx.x] = tab.L[threadIdx.x];
    __syncthreads();
    for (int i = threadIdx.x; i < kPairTableWords; i += blockDim.x) {
        const int v = i >> 5;
        s_tab[i] = pack_bf16x2(s_L[v >> 4], s_L[v & 15]);
    }
    __syncthreads();
}

// bf16x2 (L[hi nibble], L[lo nibble]) of byte `j` of `w`; lane_base = smem
// address of this lane's column of the pair table.
__device__ __forceinline__ uint32_t pair_lookup(uint32_t lane_base, uint32_t w, int j) {
    const uint32_t v = prmt(w, 0u, 0x4440u + (uint32_t)j);
    return lds_u32(lane_base + v * 128u);
}

__device__ __forceinline__ float block_constant(const int8_t* codes, const float* scale, const float* mean,
                                                int64_t b) {
    const int64_t g = b >> 8;
    return __fmaf_rn((float)__ldg(codes + b), __ldg(scale + g), __ldg(mean + g));
}

struct SmallFwdArgs {
    const uint16_t* X;        // [M, K]
    const uint8_t* packed;    // [N, K/2]
    const int8_t* codes;
    const float* scale;
    const float* mean;
    const float* T32;         // [M, rp] fp32 LoRA down-projection, or null
    const uint16_t* B;        // [N, r]
    uint16_t* Y;              // [M, N]
    int64_t M, N, K;
    int rp, r;
    float s;
};

template <int MT>
constexpr int fwd_small_smem_bytes() { return kPairTableWords * 4 + kSmallWarps * 16 * (8 * MT + 4) * 4; }

// Forward.  One CTA per 16-row tile of W (persistent, grid-stride over
// tiles); its 16 warps split the K blocks.  Per warp and 64-wide block:
//   lane (g, t) holds 8 packed bytes of rows g and g+8 (k in [16t, 16t+16)),
//   MMA i uses bytes 2i, 2i+1: logical k {2t, 2t+1} <-> physical
//   16t + 4i + {0, 1} and logical {2t+8, 2t+9} <-> 16t + 4i + {2, 3}.
// Partial tiles are summed across warps in shared memory in a fixed order,
// then s * T[m,:] . B[n,:] is added and Y is written once in bf16.
template <int MT>
__global__ void __launch_bounds__(kSmallThreads) k_fwd_small(SmallFwdArgs a, NF4Tables tab) {
    constexpr int MC = 8 * MT;
    constexpr int RS = MC + 4;                       // padded row stride of the reduction buffer
    extern __shared__ __align__(16) uint8_t smem[];
    uint32_t* s_tab = reinterpret_cast<uint32_t*>(smem);
    float* s_red = reinterpret_cast<float*>(smem + kPairTableWords * 4);   // [warps][16][RS]
    __shared__ float s_L[16];
    build_pair_table(s_tab, s_L, tab);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const uint32_t lane_base = smem_u32(s_tab) + lane * 4;
    const int64_t nblk = a.K / kBlock;
    const int64_t ntiles = cdiv(a.N, 16);
    const int64_t rowbytes = a.K / 2;

    for (int64_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
        const int64_t n0 = tile * 16;
        const int64_t row0 = min(n0 + g, a.N - 1), row1 = min(n0 + g + 8, a.N - 1);
        const uint8_t* p0 = a.packed + row0 * rowbytes + 8 * t;
        const uint8_t* p1 = a.packed + row1 * rowbytes + 8 * t;
        for (int64_t mc = 0; mc < a.M; mc += MC) {
            float acc[MT][4];
#pragma unroll
            for (int nt = 0; nt < MT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
            for (int64_t b = warp; b < nblk; b += kSmallWarps) {
                const uint2 w0 = ldg_nc_v2(p0 + 32 * b);
                const uint2 w1 = ldg_nc_v2(p1 + 32 * b);
                uint32_t xf[MT][8];
#pragma unroll
                for (int nt = 0; nt < MT; ++nt) {
                    const int64_t m = mc + nt * 8 + g;
                    if (m < a.M) {
                        const uint4* xp = reinterpret_cast<const uint4*>(a.X + m * a.K + 64 * b + 16 * t);
                        const uint4 u0 = __ldg(xp), u1 = __ldg(xp + 1);
                        xf[nt][0] = u0.x; xf[nt][1] = u0.y; xf[nt][2] = u0.z; xf[nt][3] = u0.w;
                        xf[nt][4] = u1.x; xf[nt][5] = u1.y; xf[nt][6] = u1.z; xf[nt][7] = u1.w;
                    } else {
#pragma unroll
                        for (int j = 0; j < 8; ++j) xf[nt][j] = 0u;
                    }
                }
                const float c0 = block_constant(a.codes, a.scale, a.mean, row0 * nblk + b);
                const float c1 = block_constant(a.codes, a.scale, a.mean, row1 * nblk + b);
                float tmp[MT][4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const uint32_t u0 = (i < 2) ? w0.x : w0.y;
                    const uint32_t u1 = (i < 2) ? w1.x : w1.y;
                    const int j0 = (2 * i) & 3, j1 = (2 * i + 1) & 3;
                    const uint32_t a0 = pair_lookup(lane_base, u0, j0);
                    const uint32_t a1 = pair_lookup(lane_base, u1, j0);
                    const uint32_t a2 = pair_lookup(lane_base, u0, j1);
                    const uint32_t a3 = pair_lookup(lane_base, u1, j1);
#pragma unroll
                    for (int nt = 0; nt < MT; ++nt) {
                        if (i == 0) mma_bf16_16816_zero(tmp[nt], a0, a1, a2, a3, xf[nt][0], xf[nt][1]);
                        else mma_bf16_16816(tmp[nt], a0, a1, a2, a3, xf[nt][2 * i], xf[nt][2 * i + 1]);
                    }
                }
#pragma unroll
                for (int nt = 0; nt < MT; ++nt) {
                    acc[nt][0] = __fmaf_rn(c0, tmp[nt][0], acc[nt][0]);
                    acc[nt][1] = __fmaf_rn(c0, tmp[nt][1], acc[nt][1]);
                    acc[nt][2] = __fmaf_rn(c1, tmp[nt][2], acc[nt][2]);
                    acc[nt][3] = __fmaf_rn(c1, tmp[nt][3], acc[nt][3]);
                }
            }
            float* red = s_red + warp * 16 * RS;
#pragma unroll
            for (int nt = 0; nt < MT; ++nt) {
                red[g * RS + nt * 8 + 2 * t] = acc[nt][0];
                red[g * RS + nt * 8 + 2 * t + 1] = acc[nt][1];
                red[(g + 8) * RS + nt * 8 + 2 * t] = acc[nt][2];
                red[(g + 8) * RS + nt * 8 + 2 * t + 1] = acc[nt][3];
            }
            __syncthreads();
            for (int idx = threadIdx.x; idx < 16 * MC; idx += blockDim.x) {
                const int row = idx & 15, ml = idx >> 4;
                const int64_t m = mc + ml, n = n0 + row;
                if (m < a.M && n < a.N) {
                    float v = 0.f;
                    for (int w = 0; w < kSmallWarps; ++w) v += s_red[w * 16 * RS + row * RS + ml];
                    if (a.T32 != nullptr) {
                        const float* tr = a.T32 + m * a.rp;
                        const uint16_t* br = a.B + n * a.r;
                        float l = 0.f;
                        for (int i = 0; i < a.r; ++i) l = __fmaf_rn(tr[i], bf16lo_to_f32(br[i]), l);
                        v = __fmaf_rn(a.s, l, v);
                    }
                    a.Y[m * a.N + n] = (uint16_t)(pack_bf16x2(v, 0.f) & 0xffffu);
                }
            }
            __syncthreads();
        }
    }
}

struct SmallBwdArgs {
    const uint16_t* dY;       // [M, N]
    const uint8_t* packed;    // [N, K/2]
    const int8_t* codes;
    const float* scale;
    const float* mean;
    float* part;              // [S][M][K] fp32 partial dY W' (no LoRA term)
    int64_t M, N, K;
    int64_t rows_per_split;   // multiple of 64
    int S;
};

constexpr int kBwdKW = 4;     // k-blocks per CTA
constexpr int kBwdNSUB = 4;   // n sub-ranges per CTA (kBwdKW * kBwdNSUB = 16 warps)

template <int MT>
constexpr int bwd_small_smem_bytes() { return kPairTableWords * 4 + kSmallWarps * 64 * (8 * MT + 4) * 4; }

// Backward dX = dY W' without the LoRA term.  Work unit = (4 consecutive
// 64-wide k-blocks, one split of the N rows); warp w takes k-block w % 4 and
// every 4th 16-row step of the split.  Per step, lane (g, t) reads 4 packed
// bytes (k in [8g, 8g+8) of its block) of rows n0 + {2t, 2t+1, 2t+8, 2t+9};
// MMA j (0..3) maps logical row g <-> k = 8g + 2j, row g+8 <-> 8g + 2j + 1,
// and logical reduction index {2t, 2t+1, 2t+8, 2t+9} <-> those rows.  The
// pair lookups give (k even, k odd) of one row; two byte-permutes transpose
// them into (row n, row n+1) operand pairs.  The per-(row, block) constant
// multiplies dY before it is rounded to bf16.
template <int MT>
__global__ void __launch_bounds__(kSmallThreads) k_bwd_small(SmallBwdArgs a, NF4Tables tab) {
    constexpr int MC = 8 * MT;
    constexpr int RS = MC + 4;
    extern __shared__ __align__(16) uint8_t smem[];
    uint32_t* s_tab = reinterpret_cast<uint32_t*>(smem);
    float* s_red = reinterpret_cast<float*>(smem + kPairTableWords * 4);   // [warps][64][RS]
    __shared__ float s_L[16];
    build_pair_table(s_tab, s_L, tab);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int kw = warp % kBwdKW, sub = warp / kBwdKW;
    const uint32_t lane_base = smem_u32(s_tab) + lane * 4;
    const int64_t nblk = a.K / kBlock;
    const int64_t nkg = cdiv(nblk, kBwdKW);
    const int64_t units = nkg * a.S;
    const int64_t rowbytes = a.K / 2;

    for (int64_t u = blockIdx.x; u < units; u += gridDim.x) {
        const int64_t kg = u / a.S, split = u % a.S;
        const int64_t kb = kg * kBwdKW + kw;
        const bool kvalid = kb < nblk;
        const int64_t n_lo = split * a.rows_per_split;
        const int64_t n_hi = min(a.N, n_lo + a.rows_per_split);
        for (int64_t mc = 0; mc < a.M; mc += MC) {
            float acc[4][MT][4];
#pragma unroll
            for (int j = 0; j < 4; ++j)
#pragma unroll
                for (int nt = 0; nt < MT; ++nt) acc[j][nt][0] = acc[j][nt][1] = acc[j][nt][2] = acc[j][nt][3] = 0.f;
            if (kvalid) {
                for (int64_t n0 = n_lo + sub * 16; n0 < n_hi; n0 += 16 * kBwdNSUB) {
                    // block constants of rows n0 .. n0+15, one per lane, then shuffled
                    float cl = 0.f;
                    if (lane < 16 && n0 + lane < n_hi)
                        cl = block_constant(a.codes, a.scale, a.mean, (n0 + lane) * nblk + kb);
                    const int64_t nA = n0 + 2 * t, nC = nA + 8;
                    const float cA = __shfl_sync(0xffffffffu, cl, 2 * t);
                    const float cB = __shfl_sync(0xffffffffu, cl, 2 * t + 1);
                    const float cC = __shfl_sync(0xffffffffu, cl, 2 * t + 8);
                    const float cD = __shfl_sync(0xffffffffu, cl, 2 * t + 9);
                    const bool vA = nA < n_hi, vC = nC < n_hi;   // nA even and N % 8 == 0: nA+1 valid too
                    const uint8_t* pk = a.packed + 32 * kb + 4 * g;
                    const uint32_t wA = vA ? ldg_nc_u32(pk + nA * rowbytes) : 0u;
                    const uint32_t wB = vA ? ldg_nc_u32(pk + (nA + 1) * rowbytes) : 0u;
                    const uint32_t wC = vC ? ldg_nc_u32(pk + nC * rowbytes) : 0u;
                    const uint32_t wD = vC ? ldg_nc_u32(pk + (nC + 1) * rowbytes) : 0u;
                    uint32_t b0[MT], b1[MT];
#pragma unroll
                    for (int nt = 0; nt < MT; ++nt) {
                        const int64_t m = mc + nt * 8 + g;
                        uint32_t d01 = 0u, d89 = 0u;
                        if (m < a.M) {
                            const uint16_t* dyr = a.dY + m * a.N;
                            if (vA) d01 = __ldg(reinterpret_cast<const unsigned int*>(dyr + nA));
                            if (vC) d89 = __ldg(reinterpret_cast<const unsigned int*>(dyr + nC));
                        }
                        b0[nt] = pack_bf16x2(bf16lo_to_f32(d01) * cA, bf16hi_to_f32(d01) * cB);
                        b1[nt] = pack_bf16x2(bf16lo_to_f32(d89) * cC, bf16hi_to_f32(d89) * cD);
                    }
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const uint32_t PA = pair_lookup(lane_base, wA, j);
                        const uint32_t PB = pair_lookup(lane_base, wB, j);
                        const uint32_t PC = pair_lookup(lane_base, wC, j);
                        const uint32_t PD = pair_lookup(lane_base, wD, j);
                        const uint32_t a0 = prmt(PA, PB, 0x5410u);
                        const uint32_t a1 = prmt(PA, PB, 0x7632u);
                        const uint32_t a2 = prmt(PC, PD, 0x5410u);
                        const uint32_t a3 = prmt(PC, PD, 0x7632u);
#pragma unroll
                        for (int nt = 0; nt < MT; ++nt) mma_bf16_16816(acc[j][nt], a0, a1, a2, a3, b0[nt], b1[nt]);
                    }
                }
            }
            float* red = s_red + warp * 64 * RS;
#pragma unroll
            for (int j = 0; j < 4; ++j)
#pragma unroll
                for (int nt = 0; nt < MT; ++nt) {
                    const int ke = 8 * g + 2 * j;
                    red[ke * RS + nt * 8 + 2 * t] = acc[j][nt][0];
                    red[ke * RS + nt * 8 + 2 * t + 1] = acc[j][nt][1];
                    red[(ke + 1) * RS + nt * 8 + 2 * t] = acc[j][nt][2];
                    red[(ke + 1) * RS + nt * 8 + 2 * t + 1] = acc[j][nt][3];
                }
            __syncthreads();
            for (int idx = threadIdx.x; idx < kBwdKW * 64 * MC; idx += blockDim.x) {
                const int kl = idx % (kBwdKW * 64), ml = idx / (kBwdKW * 64);
                const int kwi = kl / 64, ke = kl % 64;
                const int64_t k = (kg * kBwdKW + kwi) * 64 + ke, m = mc + ml;
                if (k < a.K && m < a.M) {
                    float v = 0.f;
#pragma unroll
                    for (int s = 0; s < kBwdNSUB; ++s) v += s_red[(s * kBwdKW + kwi) * 64 * RS + ke * RS + ml];
                    a.part[(split * a.M + m) * a.K + k] = v;
                }
            }
            __syncthreads();
        }
    }
}

// dX[m, k] = sum_s part[s, m, k] + s_lora * sum_i U[m, i] A[i, k], in bf16.
__global__ void __launch_bounds__(256) k_bwd_small_finish(const float* __restrict__ part, int S, int64_t M, int64_t K,
                                                          const float* __restrict__ U32, int rp,
                                                          const uint16_t* __restrict__ A, int r, float s_lora,
                                                          uint16_t* __restrict__ dX) {
    const int64_t total = M * K;
    for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total; e += (int64_t)gridDim.x * blockDim.x) {
        const int64_t m = e / K, k = e % K;
        float v = 0.f;
        for (int s = 0; s < S; ++s) v += part[s * total + e];
        if (U32 != nullptr) {
            float l = 0.f;
            for (int i = 0; i < r; ++i) l = __fmaf_rn(U32[m * rp + i], bf16lo_to_f32(A[(int64_t)i * K + k]), l);
            v = __fmaf_rn(s_lora, l, v);
        }
        dX[e] = (uint16_t)(pack_bf16x2(v, 0.f) & 0xffffu);
    }
}

}  // namespace qnf4
