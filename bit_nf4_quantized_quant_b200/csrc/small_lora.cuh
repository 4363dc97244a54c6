// small_lora.cuh -- the LoRA adapter products of the small-M path (M <= 32
// tokens).  A decode-sized forward is three launches (fused GEMV, T, finish)
// and the backward three (four when T is recomputed):
//
//   k_lora_down_small  T = X A^T over the whole K (one CTA per rank column
//                      and token group; no cross-CTA reduction)
//   k_lora_bwd_small   U = dY B as per-split partials, and dB = s dY^T T, in
//                      one launch (the first CTAs take U, the rest dB)
//   k_bwd_small_end    dX = (sum of k_tcs_gemm's partial tiles) + s U A and
//                      dA = s U^T X, each CTA first summing the U partials it
//                      needs in a fixed order
//
// The QLoRA paper (Dettmers et al., "QLoRA: Efficient Finetuning of Quantized
// LLMs", section 3, eq. 5-6) defines these products: Y = X W' + s X L1 L2 with
// L1 = A^T, L2 = B^T, and the adapters get gradients while W' gets none.
// At these token counts every product is a short dot product or a sum of
// at most 32 outer products, so plain fp32 FMAs on the CUDA cores with
// 16-byte loads suffice; U and T stay in fp32 end to end.
#pragma once
#include "common.cuh"
#include "dropout.cuh"

namespace qnf4 {

constexpr int kLoraThreads = 256;

// ---------------------------------------------------------------------------
// T = X A^T
// ---------------------------------------------------------------------------
struct LoraDownArgs {
    const uint16_t* X;       // [M, K] bf16, 16-byte aligned
    const uint16_t* A;       // [r, K] bf16, 16-byte aligned
    int64_t M, K;            // K % 64 == 0
    int r, rp;
    int kc;                  // K splits: split z sums the 8-wide chunks [z nch / kc, (z + 1) nch / kc)
    float* T32;              // [kc][M, rp] fp32 partial sums (columns >= r not written)
    uint16_t* T_out;         // [M, r] bf16 copy for the caller (kc == 1 only), or null
};

// K splits of the forward's T: about two 8-wide chunks per thread and split.
inline int64_t down_splits(int64_t K) { return (K / 8 + 255) / 256; }

__device__ __forceinline__ float dot8_bf16(const uint4& x, const uint4& y, float v) {
    const uint32_t xw[4] = {x.x, x.y, x.z, x.w}, yw[4] = {y.x, y.y, y.z, y.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        v = __fmaf_rn(bf16lo_to_f32(xw[j]), bf16lo_to_f32(yw[j]), v);
        v = __fmaf_rn(bf16hi_to_f32(xw[j]), bf16hi_to_f32(yw[j]), v);
    }
    return v;
}

// CTA (i, z, mg) computes split z of T[mg MG .. mg MG + MG, i]; thread t takes
// the split's 8-wide K chunks t, t + 128, ...; fixed-order warp and block
// reductions.  Small enough (128 threads, at most 32 registers) to run beside
// a fused GEMV CTA on its SM.  In the forward it is launched programmatically
// right behind the GEMV, which releases it only once the kernel ahead of the
// GEMV (the writer of X) has completed, so X is read at once, through L2; it
// lets the finish kernel launch at once, and its first CTA waits for the
// GEMV before it ends, so that this grid's completion implies the GEMV's
// (the other CTAs exit as soon as their sums are written).  Launched plainly
// (the backward's recompute, one split) the wait returns at once.
constexpr int kDownThreads = 128;

template <int MG>
__global__ void __launch_bounds__(kDownThreads, 16) k_lora_down_small(LoraDownArgs a) {
    grid_dep_launch();
    __shared__ float s_red[kDownThreads / 32][MG];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int i = blockIdx.x, z = blockIdx.y;
    const int64_t m0 = (int64_t)blockIdx.z * MG;
    const int64_t nch = a.K / 8;
    const int64_t c0 = z * nch / a.kc, c1 = (z + 1) * nch / a.kc;
    const uint4* ar = reinterpret_cast<const uint4*>(a.A + (int64_t)i * a.K);
    const uint4* xr = reinterpret_cast<const uint4*>(a.X + m0 * a.K);
    const int mn = a.M - m0 < MG ? (int)(a.M - m0) : MG;
    float acc[MG];
#pragma unroll
    for (int mm = 0; mm < MG; ++mm) acc[mm] = 0.f;
    for (int64_t c = c0 + tid; c < c1; c += kDownThreads) {
        const uint4 av = ldg_cg_v4(ar + c);
#pragma unroll
        for (int mm = 0; mm < MG; ++mm)
            if (mm < mn) acc[mm] = dot8_bf16(ldg_cg_v4(xr + mm * nch + c), av, acc[mm]);
    }
#pragma unroll
    for (int mm = 0; mm < MG; ++mm) {
        float v = acc[mm];
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
        if (lane == 0) s_red[warp][mm] = v;
    }
    __syncthreads();
    if (tid < mn) {
        float v = 0.f;
#pragma unroll
        for (int w = 0; w < kDownThreads / 32; ++w) v += s_red[w][tid];
        const int64_t m = m0 + tid;
        a.T32[((int64_t)z * a.M + m) * a.rp + i] = v;
        if (a.T_out != nullptr) a.T_out[m * a.r + i] = (uint16_t)(pack_bf16x2(v, 0.f) & 0xffffu);
    }
    if (blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0) grid_dep_wait();
}

// ---------------------------------------------------------------------------
// U = dY B (split partials) and dB = s dY^T T
// ---------------------------------------------------------------------------
struct LoraBwdArgs {
    const uint16_t* dY;      // [M, N] bf16
    const uint16_t* B;       // [N, r] bf16
    const float* T32;        // [M, rp] fp32 T, or null
    const uint16_t* Tb;      // [M, r] bf16 T from the caller (read when T32 is null)
    int64_t M, N;
    int r, rp;
    float s;
    float tscale;            // scale of the T32 values (1 except under LoRA dropout; Tb is taken as is)
    int b_vec;               // B rows are 16-byte loadable (r % 8 == 0, B 16-byte aligned)
    float* Upart;            // [US][M][rp] fp32 partial U (columns >= r not written)
    int US;                  // N splits of U; CTAs [0, US) compute U
    int64_t rows_u;          // rows of B per split
    uint16_t* dB;            // [N, r] bf16
};

constexpr int kUTok = 4;     // tokens per pass of a U split
constexpr int kDbCols = 64;  // rank columns per pass of a dB CTA
constexpr int kSmemLoraBwd = (kLoraThreads / 32) * kUTok * 256 > 32 * kDbCols + kLoraThreads * 33
                                 ? (kLoraThreads / 32) * kUTok * 256
                                 : 32 * kDbCols + kLoraThreads * 33;

__device__ __forceinline__ void load_b8(const LoraBwdArgs& a, int64_t n, int c, float (&bv)[8]) {
    const int col0 = c * 8;
    if (a.b_vec) {
        if (col0 < a.r) {
            const uint4 v = ldg_nc_v4(a.B + n * a.r + col0);
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                bv[2 * j] = bf16lo_to_f32(w[j]);
                bv[2 * j + 1] = bf16hi_to_f32(w[j]);
            }
        } else {
#pragma unroll
            for (int j = 0; j < 8; ++j) bv[j] = 0.f;
        }
        return;
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) bv[j] = col0 + j < a.r ? bf16lo_to_f32(a.B[n * a.r + col0 + j]) : 0.f;
}

__global__ void __launch_bounds__(kLoraThreads) k_lora_bwd_small(LoraBwdArgs a) {
    grid_dep_launch();
    __shared__ __align__(16) float smem[kSmemLoraBwd];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    if ((int)blockIdx.x < a.US) {
        // ---- U split b: rows n in [n0, n1); lane group c owns rank columns 8c .. 8c + 7
        float(*s_red)[kUTok][256] = reinterpret_cast<float(*)[kUTok][256]>(smem);
        const int b = blockIdx.x;
        const int CH = a.rp / 8;
        int CHP = 1;
        while (CHP < CH) CHP <<= 1;
        const int c = tid % CHP, G = kLoraThreads / CHP;
        const int64_t n0 = (int64_t)b * a.rows_u;
        const int64_t n1 = n0 + a.rows_u < a.N ? n0 + a.rows_u : a.N;
        for (int64_t m0 = 0; m0 < a.M; m0 += kUTok) {
            float acc[kUTok][8];
#pragma unroll
            for (int mm = 0; mm < kUTok; ++mm)
#pragma unroll
                for (int j = 0; j < 8; ++j) acc[mm][j] = 0.f;
            if (c < CH) {
                for (int64_t n = n0 + tid / CHP; n < n1; n += G) {
                    float bv[8];
                    load_b8(a, n, c, bv);
#pragma unroll
                    for (int mm = 0; mm < kUTok; ++mm) {
                        const float y = m0 + mm < a.M ? bf16lo_to_f32(a.dY[(m0 + mm) * a.N + n]) : 0.f;
#pragma unroll
                        for (int j = 0; j < 8; ++j) acc[mm][j] = __fmaf_rn(y, bv[j], acc[mm][j]);
                    }
                }
            }
            for (int off = CHP; off < 32; off <<= 1)
#pragma unroll
                for (int mm = 0; mm < kUTok; ++mm)
#pragma unroll
                    for (int j = 0; j < 8; ++j) acc[mm][j] += __shfl_xor_sync(0xffffffffu, acc[mm][j], off);
            if (lane < CHP && c < CH)
#pragma unroll
                for (int mm = 0; mm < kUTok; ++mm)
#pragma unroll
                    for (int j = 0; j < 8; ++j) s_red[warp][mm][c * 8 + j] = acc[mm][j];
            __syncthreads();
            for (int e = tid; e < kUTok * a.rp; e += kLoraThreads) {
                const int mm = e / a.rp, i = e % a.rp;
                if (m0 + mm < a.M && i < a.r) {
                    float v = 0.f;
#pragma unroll
                    for (int w = 0; w < kLoraThreads / 32; ++w) v += s_red[w][mm][i];
                    a.Upart[((int64_t)b * a.M + m0 + mm) * a.rp + i] = v;
                }
            }
            __syncthreads();
        }
        return;
    }

    // ---- dB rows [nb, nb + 256): thread tid owns row nb + tid
    float* s_T = smem;                                   // [M <= 32][kDbCols]
    uint32_t* s_out = reinterpret_cast<uint32_t*>(smem + 32 * kDbCols);   // [256][33] bf16 pairs
    const int64_t nb = (int64_t)(blockIdx.x - a.US) * kLoraThreads;
    const int64_t n = nb + tid;
    for (int i0 = 0; i0 < a.r; i0 += kDbCols) {
        const int ic = a.r - i0 < kDbCols ? a.r - i0 : kDbCols;
        __syncthreads();
        for (int e = tid; e < (int)a.M * kDbCols; e += kLoraThreads) {
            const int mm = e / kDbCols, j = e % kDbCols;
            float tv = 0.f;
            if (j < ic)
                tv = a.T32 != nullptr ? __fmul_rn(a.T32[(int64_t)mm * a.rp + i0 + j], a.tscale)
                                      : bf16lo_to_f32(a.Tb[(int64_t)mm * a.r + i0 + j]);
            s_T[e] = tv;
        }
        __syncthreads();
        float acc[kDbCols];
#pragma unroll
        for (int j = 0; j < kDbCols; ++j) acc[j] = 0.f;
        if (n < a.N) {
            for (int64_t mm = 0; mm < a.M; ++mm) {
                const float y = bf16lo_to_f32(a.dY[mm * a.N + n]);
#pragma unroll
                for (int j = 0; j < kDbCols; ++j) acc[j] = __fmaf_rn(y, s_T[mm * kDbCols + j], acc[j]);
            }
        }
        // stage through shared memory so that each warp stores whole rows
#pragma unroll
        for (int jj = 0; jj < kDbCols / 2; ++jj)
            s_out[tid * 33 + jj] = pack_bf16x2(a.s * acc[2 * jj], a.s * acc[2 * jj + 1]);
        __syncwarp();
        for (int rr = 0; rr < 32; ++rr) {
            const int row = warp * 32 + rr;
            const int64_t nn = nb + row;
            if (nn >= a.N) break;
            const uint32_t w = s_out[row * 33 + lane];
            const int col = 2 * lane;
            uint16_t* dst = a.dB + nn * a.r + i0 + col;
            if (col < ic) dst[0] = (uint16_t)(w & 0xffffu);
            if (col + 1 < ic) dst[1] = (uint16_t)(w >> 16);
        }
        __syncwarp();
    }
}

// ---------------------------------------------------------------------------
// dX = sum_s part_s + s U A,   dA = s U^T X
// ---------------------------------------------------------------------------
struct BwdEndArgs {
    const float* slots;      // [ctas + tiles][NT][128] partial dY W' tiles of k_tcs_gemm
    int NT, nks, ctas;       // that kernel's token width, steps per tile and grid
    int64_t units;
    const float* Upart;      // [US][M][rp] fp32 partial U
    int US;
    const uint16_t* A;       // [r, K]
    const uint16_t* X;       // [M, K]
    int64_t M, K;
    int r, rp;
    float s;
    float s_da;              // scale of dA: s, or fl32(s c) under LoRA dropout
    uint16_t* dX;            // [M, K]
    uint16_t* dA;            // [r, K]
    const uint16_t* mask;    // LoRA dropout: keep bits of [M, K] (the LoRA term of dX is masked, keep * c,
                             // and X above is then X * keep); null without dropout
    float c;                 // scale of kept values
};

// The CTA that owns unit u under k_tcs_gemm's even split of U units over C
// CTAs (U < 2^23 and C <= 148, so the products fit 32 bits).
__device__ __forceinline__ uint32_t end_unit_owner(uint32_t u, uint32_t U, uint32_t C) {
    return ((u + 1) * C + U - 1) / U - 1;
}

// grid (ceil(K / 256), M + r): row y < M writes dX[y, :], row M + i writes dA[i, :].
// Launched programmatically after k_tcs_gemm: it lets the next kernel on the
// stream launch, then waits for that kernel (and so for the U / dB kernel
// before it).
__global__ void __launch_bounds__(kLoraThreads) k_bwd_small_end(BwdEndArgs a) {
    __shared__ float s_q[kLoraThreads];
    __shared__ float s_u[kLoraThreads];
    grid_dep_launch();
    grid_dep_wait();
    const int tid = threadIdx.x;
    const int y = blockIdx.y;
    const bool is_dx = y < a.M;
    // U entries this row needs: U[y, 0..r) for dX, U[0..M, i] for dA
    const int E = is_dx ? a.r : (int)a.M;
    int EP = 1;
    while (EP < E) EP <<= 1;
    const int Q = kLoraThreads / EP;
    {
        const int e = tid % EP, q = tid / EP;
        float v = 0.f;
        if (e < E) {
            const int64_t m = is_dx ? y : e;
            const int i = is_dx ? e : y - (int)a.M;
            for (int b = q; b < a.US; b += Q) v += a.Upart[((int64_t)b * a.M + m) * a.rp + i];
        }
        s_q[tid] = v;
    }
    __syncthreads();
    if (tid < E) {
        float v = 0.f;
        for (int q = 0; q < Q; ++q) v += s_q[q * EP + tid];
        s_u[tid] = v;
    }
    __syncthreads();
    const int64_t k = (int64_t)blockIdx.x * kLoraThreads + tid;
    if (k >= a.K) return;
    if (is_dx) {
        // dY W': the partial tiles of every CTA that took steps of column tile k / 128, in CTA order
        const int64_t tile = k >> 7, row = k & 127;
        const uint32_t tu0 = (uint32_t)tile * (uint32_t)a.nks;
        const int64_t c_first = end_unit_owner(tu0, (uint32_t)a.units, (uint32_t)a.ctas);
        const int64_t c_last = end_unit_owner(tu0 + (uint32_t)a.nks - 1, (uint32_t)a.units, (uint32_t)a.ctas);
        float v = 0.f;
        for (int64_t c = c_first; c <= c_last; ++c) v += a.slots[(c + tile) * (a.NT * 128) + (int64_t)y * 128 + row];
        float l = 0.f;
        for (int i = 0; i < a.r; ++i) l = __fmaf_rn(s_u[i], bf16lo_to_f32(a.A[(int64_t)i * a.K + k]), l);
        if (a.mask)                         // d Xd / d X = keep * c
            l = drop::mask_bit(a.mask, (uint64_t)y * (uint64_t)a.K + (uint64_t)k) ? __fmul_rn(l, a.c) : 0.f;
        v = __fmaf_rn(a.s, l, v);
        a.dX[(int64_t)y * a.K + k] = (uint16_t)(pack_bf16x2(v, 0.f) & 0xffffu);
    } else {
        const int i = y - (int)a.M;
        float v = 0.f;
        for (int64_t m = 0; m < a.M; ++m) v = __fmaf_rn(s_u[m], bf16lo_to_f32(a.X[m * a.K + k]), v);
        a.dA[(int64_t)i * a.K + k] = (uint16_t)(pack_bf16x2(a.s_da * v, 0.f) & 0xffffu);
    }
}

}  // namespace qnf4
