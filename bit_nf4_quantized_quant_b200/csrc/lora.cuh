// lora.cuh -- the rank-r adapter products of the layer:
//   T = X A^T [M, r], U = dY B [M, r], dA = s U^T X [r, K], dB = s dY^T T [N, r].
// Each is a skinny bf16 GEMM with one side of size r (<= 256); they run on a
// split-K tensor-core kernel (mma.sync m16n8k16, fp32 accumulation, operands
// staged through shared memory with cp.async and fed with ldmatrix, .trans
// where the stored operand is not K-contiguous), whose fp32 partials are
// summed in a fixed order by a small finishing kernel that also applies the
// scaling and writes the fp32 / bf16 copies the layer needs.
#pragma once
#include "common.cuh"

namespace qnf4 {

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
    const int sz = valid ? 16 : 0;
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(sz));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N)); }

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}

// C[z][i][j] = sum_{k in split z} Aop(i, k) Bop(k, j)  (fp32)
//   Aop(i, k) = A_KMAJ ? A[i * lda + k] : A[k * lda + i]
//   Bop(k, j) = B_KMAJ ? B[j * ldb + k] : B[k * ldb + j]
// Loads outside i < Ilim, j < Jlim, k < Kd read as zero (whole 16-byte
// chunks: every contiguous extent used here is a multiple of 8 elements).
struct GemmArgs {
    const uint16_t* A;
    const uint16_t* B;
    float* C;
    int64_t lda, ldb;
    int64_t I, J, Kd;        // tile extents (I, J multiples of the tile)
    int64_t Ilim, Jlim;      // load limits
    int64_t k_per_split;     // multiple of 32
};

template <bool A_KMAJ, bool B_KMAJ, int BI, int BJ, int WI, int WJ>
// The adapter kernels run as a chain on one stream with programmatic launch:
// each lets the next one start launching at once, then waits for the one
// before it (whose outputs it may read, or whose inputs it may overwrite)
// before touching global memory.
__global__ void __launch_bounds__(128) k_gemm_mma(GemmArgs p) {
    grid_dep_launch();
    grid_dep_wait();
    constexpr int BK = 32;
    constexpr int ST = 4;                              // cp.async stages: 3 tiles in flight per CTA
    constexpr int TI = BI / WI, TJ = BJ / WJ;          // warp tile
    static_assert(WI * WJ == 4 && TI % 16 == 0 && TJ % 16 == 0, "tile");
    constexpr int A_ROWS = A_KMAJ ? BI : BK, A_COLS = A_KMAJ ? BK : BI;
    constexpr int B_ROWS = B_KMAJ ? BJ : BK, B_COLS = B_KMAJ ? BK : BJ;
    constexpr int A_LD = A_COLS + 8, B_LD = B_COLS + 8;  // +16 bytes: ldmatrix rows hit distinct banks
    __shared__ __align__(16) uint16_t sA[ST][A_ROWS * A_LD];
    __shared__ __align__(16) uint16_t sB[ST][B_ROWS * B_LD];

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int wi = warp / WJ, wj = warp % WJ;
    const int64_t i0 = (int64_t)blockIdx.x * BI, j0 = (int64_t)blockIdx.y * BJ;
    const int64_t kbeg = (int64_t)blockIdx.z * p.k_per_split;
    const int64_t kend = min(p.Kd, kbeg + p.k_per_split);

    auto load_tile = [&](int stage, int64_t k0) {
        // A
        constexpr int A_CH = A_ROWS * A_COLS / 8;
        for (int c = tid; c < A_CH; c += 128) {
            const int row = c / (A_COLS / 8), col = (c % (A_COLS / 8)) * 8;
            int64_t gi, gk;
            if (A_KMAJ) { gi = i0 + row; gk = k0 + col; } else { gk = k0 + row; gi = i0 + col; }
            const bool v = gi < p.Ilim && gk < kend;
            const uint16_t* src = p.A + (v ? (A_KMAJ ? gi * p.lda + gk : gk * p.lda + gi) : 0);
            cp_async16(smem_u32(&sA[stage][row * A_LD + col]), src, v);
        }
        constexpr int B_CH = B_ROWS * B_COLS / 8;
        for (int c = tid; c < B_CH; c += 128) {
            const int row = c / (B_COLS / 8), col = (c % (B_COLS / 8)) * 8;
            int64_t gj, gk;
            if (B_KMAJ) { gj = j0 + row; gk = k0 + col; } else { gk = k0 + row; gj = j0 + col; }
            const bool v = gj < p.Jlim && gk < kend;
            const uint16_t* src = p.B + (v ? (B_KMAJ ? gj * p.ldb + gk : gk * p.ldb + gj) : 0);
            cp_async16(smem_u32(&sB[stage][row * B_LD + col]), src, v);
        }
        cp_async_commit();
    };

    float acc[TI / 16][TJ / 8][4];
#pragma unroll
    for (int a = 0; a < TI / 16; ++a)
#pragma unroll
        for (int b = 0; b < TJ / 8; ++b) acc[a][b][0] = acc[a][b][1] = acc[a][b][2] = acc[a][b][3] = 0.f;

    const int nk = (int)cdiv(kend - kbeg, BK);
    // multistage pipeline: tiles kt+1 .. kt+ST-1 are in flight while tile kt is multiplied
#pragma unroll
    for (int s2 = 0; s2 < ST - 1; ++s2) {
        if (s2 < nk) load_tile(s2, kbeg + (int64_t)s2 * BK);
        else cp_async_commit();
    }
    for (int kt = 0; kt < nk; ++kt) {
        const int st = kt % ST;
        cp_async_wait<ST - 2>();
        __syncthreads();                               // tile kt landed; stage (kt-1) % ST is free
        {
            const int nt = kt + ST - 1;
            if (nt < nk) load_tile(nt % ST, kbeg + (int64_t)nt * BK);
            else cp_async_commit();
        }
#pragma unroll
        for (int kk = 0; kk < BK; kk += 16) {
            uint32_t af[TI / 16][4], bfr[TJ / 8][2];
#pragma unroll
            for (int a = 0; a < TI / 16; ++a) {
                const int ib = wi * TI + a * 16;
                uint32_t addr;
                if (A_KMAJ) addr = smem_u32(&sA[st][(ib + (lane & 15)) * A_LD + kk + (lane >> 4) * 8]);
                else {
                    const int mi = lane >> 3, rr = lane & 7;
                    addr = smem_u32(&sA[st][(kk + rr + (mi >> 1) * 8) * A_LD + ib + (mi & 1) * 8]);
                }
                if (A_KMAJ) ldsm_x4(addr, af[a][0], af[a][1], af[a][2], af[a][3]);
                else ldsm_x4_t(addr, af[a][0], af[a][1], af[a][2], af[a][3]);
            }
#pragma unroll
            for (int b = 0; b < TJ / 16; ++b) {
                const int jb = wj * TJ + b * 16;
                uint32_t addr;
                if (B_KMAJ) addr = smem_u32(&sB[st][(jb + (lane & 7) + ((lane >> 4) << 3)) * B_LD + kk + ((lane >> 3) & 1) * 8]);
                else {
                    const int mi = lane >> 3, rr = lane & 7;
                    addr = smem_u32(&sB[st][(kk + rr + (mi & 1) * 8) * B_LD + jb + (mi >> 1) * 8]);
                }
                if (B_KMAJ) ldsm_x4(addr, bfr[2 * b][0], bfr[2 * b][1], bfr[2 * b + 1][0], bfr[2 * b + 1][1]);
                else ldsm_x4_t(addr, bfr[2 * b][0], bfr[2 * b][1], bfr[2 * b + 1][0], bfr[2 * b + 1][1]);
            }
#pragma unroll
            for (int a = 0; a < TI / 16; ++a)
#pragma unroll
                for (int b = 0; b < TJ / 8; ++b)
                    mma_bf16_16816(acc[a][b], af[a][0], af[a][1], af[a][2], af[a][3], bfr[b][0], bfr[b][1]);
        }
    }
    cp_async_wait<0>();

    float* C = p.C + (int64_t)blockIdx.z * p.I * p.J;
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int a = 0; a < TI / 16; ++a)
#pragma unroll
        for (int b = 0; b < TJ / 8; ++b) {
            const int64_t ii = i0 + wi * TI + a * 16 + g;
            const int64_t jj = j0 + wj * TJ + b * 8 + 2 * t;
            if (ii < p.I) *reinterpret_cast<float2*>(C + ii * p.J + jj) = make_float2(acc[a][b][0], acc[a][b][1]);
            if (ii + 8 < p.I) *reinterpret_cast<float2*>(C + (ii + 8) * p.J + jj) = make_float2(acc[a][b][2], acc[a][b][3]);
        }
}

// Sum of the split-K partials in split order, then up to three outputs, for
// i < Iout and j < Jiter (columns at or beyond the partial extent J read as 0):
//   f32 [i * ld_f32 + j]            = v                            (j < Jf)
//   o1  [i * s1i + j * s1j]  (bf16) = alpha1 * v for j < J1, 0 for J1 <= j < J1pad
//   o2  likewise with alpha2, J2, J2pad.
//   hl  [i * hl_ld + j] = bf16(v), hl[i * hl_ld + hl_off + j] = bf16(v - bf16(v))
//       for j < J1 (zero for J1 <= j < hl_off): a hi + lo pair that carries
//       v to about 16 significant bits into a later bf16 product.
// With row_pair (col_pair) > 0 the value is the sum of partial rows i and
// i + row_pair (columns j and j + col_pair): the hi and lo halves of a
// product computed with a hi + lo operand.
struct FinishArgs {
    const float* C;
    int splits;
    int64_t I, J;            // partial layout [splits][I][J]
    int64_t row_pair, col_pair;
    uint16_t* hl;
    int64_t hl_ld, hl_off;
    int64_t Iout, Jiter;
    float* f32;
    int64_t ld_f32, Jf;
    uint16_t* o1;
    int64_t s1i, s1j, J1, J1pad;
    float alpha1;
    uint16_t* o2;
    int64_t s2i, s2j, J2, J2pad;
    float alpha2;
    // o2_lo > 0: o2 holds alpha2 * v as a bf16 hi + lo pair, hi in column j and
    // lo in column o2_lo + j for j < o2_lo, zero in columns [2 o2_lo, J2pad)
    int64_t o2_lo;
    float pre;               // every output is of pre * (the split sum); 1 except under LoRA dropout
};

// v + p[0] + p[stride] + ... + p[(n - 1) stride], added in that order; four
// loads are issued before they are added, so a thread waits for memory about
// n / 4 times instead of n.
__device__ __forceinline__ float split_sum(const float* p, int64_t stride, int n, float v) {
    int z = 0;
    for (; z + 4 <= n; z += 4) {
        const float a0 = p[z * stride], a1 = p[(z + 1) * stride], a2 = p[(z + 2) * stride], a3 = p[(z + 3) * stride];
        v += a0; v += a1; v += a2; v += a3;
    }
    for (; z < n; ++z) v += p[z * stride];
    return v;
}

// The outputs of element (i, j) whose reduced value is v (the stores of the
// finish, shared with the cluster-reduced adapter kernels).
__device__ __forceinline__ void finish_store(const FinishArgs& f, int64_t i, int64_t j, float v) {
    if (f.f32 && j < f.Jf) f.f32[i * f.ld_f32 + j] = v;
    if (f.hl && j < f.hl_off) {
        uint16_t hi = 0, lo = 0;
        if (j < f.J1) {
            hi = (uint16_t)(pack_bf16x2(v, 0.f) & 0xffffu);
            lo = (uint16_t)(pack_bf16x2(v - bf16lo_to_f32(hi), 0.f) & 0xffffu);
        }
        f.hl[i * f.hl_ld + j] = hi;
        f.hl[i * f.hl_ld + f.hl_off + j] = lo;
    }
    if (f.o1 && j < f.J1pad) f.o1[i * f.s1i + j * f.s1j] = (j < f.J1) ? (uint16_t)(pack_bf16x2(f.alpha1 * v, 0.f) & 0xffffu) : (uint16_t)0;
    if (f.o2 && j < f.J2pad) {
        if (f.o2_lo == 0) {
            f.o2[i * f.s2i + j * f.s2j] = (j < f.J2) ? (uint16_t)(pack_bf16x2(f.alpha2 * v, 0.f) & 0xffffu) : (uint16_t)0;
        } else if (j < f.o2_lo) {
            uint16_t hi = 0, lo = 0;
            if (j < f.J2) {
                const float sv = f.alpha2 * v;
                hi = (uint16_t)(pack_bf16x2(sv, 0.f) & 0xffffu);
                lo = (uint16_t)(pack_bf16x2(sv - bf16lo_to_f32(hi), 0.f) & 0xffffu);
            }
            f.o2[i * f.s2i + j * f.s2j] = hi;
            f.o2[i * f.s2i + (f.o2_lo + j) * f.s2j] = lo;
        } else if (j >= 2 * f.o2_lo) {
            f.o2[i * f.s2i + j * f.s2j] = 0;
        }
    }
}

__global__ void __launch_bounds__(256) k_gemm_finish(FinishArgs f) {
    grid_dep_launch();
    grid_dep_wait();
    const int64_t total = f.Iout * f.Jiter;
    for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total; e += (int64_t)gridDim.x * blockDim.x) {
        const int64_t i = e / f.Jiter, j = e % f.Jiter;
        float v = 0.f;
        if (j < f.J) {
            v = split_sum(f.C + i * f.J + j, f.I * f.J, f.splits, v);
            if (f.row_pair > 0) v = split_sum(f.C + (i + f.row_pair) * f.J + j, f.I * f.J, f.splits, v);
            if (f.col_pair > 0) v = split_sum(f.C + i * f.J + j + f.col_pair, f.I * f.J, f.splits, v);
            v = __fmul_rn(v, f.pre);
        }
        finish_store(f, i, j, v);
    }
}

// dst [rows, dcols] bf16 = src [rows, scols] zero-padded (dcols >= scols).
__global__ void k_pad_cols(const uint16_t* __restrict__ src, int64_t rows, int64_t scols, uint16_t* __restrict__ dst,
                           int64_t dcols) {
    grid_dep_launch();
    grid_dep_wait();
    const int64_t total = rows * dcols;
    for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total; e += (int64_t)gridDim.x * blockDim.x) {
        const int64_t i = e / dcols, j = e % dcols;
        dst[e] = (j < scols) ? src[i * scols + j] : (uint16_t)0;
    }
}

}  // namespace qnf4
