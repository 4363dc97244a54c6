// skinny.cuh -- the rank-r adapter products of the large-M layer as
// HBM-streaming kernels, for padded ranks rp <= 64:
//   row kernel    out [M, JQ] = P [M, L] . Q         T = X A^T  (Q = A^T, A [r, K])
//                                                    U = dY B   (Q = B [N, r])
//   column kernel out [L, JQ] = P [M, L]^T . Q [M, JQ]   dA^T = X^T U, dB = dY^T T
// Each reads a bf16 activation P once for ~r multiply-adds per element, so
// the bound is HBM; the multiply-adds run on mma.sync m16n8k16 (fp32
// accumulation).
//
//  * Operands come through a 6-deep ring of TMA tiles: a 64 x 64 tile of P
//    (128-byte rows, 128-byte swizzle) and the matching 64 x JQ tile of Q
//    (rows of JQ * 2 bytes with the swizzle of that span), both completing on
//    the stage's mbarrier; one producer lane issues them, four consumer warps
//    read them with ldmatrix (the swizzle keeps the eight rows of every 8 x 8
//    matrix in distinct banks).  A CTA holds ~10-24 KB per stage in flight.
//  * The reduction is split over the z CTAs of a thread-block cluster (z <= 8,
//    the reduction tiles dealt out in contiguous runs).  After the loop each
//    CTA leaves its fp32 partial tile in shared memory; after a cluster
//    barrier, CTA q sums rows [64 q / z, 64 (q + 1) / z) of the tile over the
//    ranks in rank order through distributed shared memory and writes every
//    output of those elements itself (fp32, bf16, hi + lo pairs, scaled
//    copies: finish_store).  The result is deterministic and no partial sums
//    go through HBM or a second kernel.
//  * Programmatic launch: the kernel lets the next one launch at once and
//    waits for the one before it before the producer's first load and before
//    any store -- or, with wait_end, where every input is known complete and
//    the kernel before it touches neither the inputs nor the outputs (dB and
//    dA launched behind the fused backward kernel, which starts only after the
//    kernel computing U has completed), not at all at the start: the kernel
//    then runs beside the one before it on the SMs that one leaves free, and
//    one CTA waits for it before exiting, so this grid completes after it.
//  * Every mbarrier wait is bounded (an expired wait raises the CTA's abort
//    flag and the device status); every thread still takes both cluster
//    barriers, so an aborting CTA never strands its cluster.
#pragma once
#include <cuda.h>
#include "common.cuh"
#include "lora.cuh"
#include "tc_gemm.cuh"

namespace qnf4 {
namespace sk {

constexpr int kCons = 4;                          // consumer warps
constexpr int kThreads = 32 * (kCons + 1);        // + the producer warp
constexpr int TILE = 64;                          // a P tile: 64 rows x 64 bf16
constexpr int kStages = 6;
constexpr int P_BYTES = TILE * TILE * 2;          // 8192
constexpr int kMaxCluster = 8;

template <int JQ>
struct Lay {
    static constexpr int Q_BYTES = JQ * 128;              // 64 x JQ bf16 (or JQ x 64)
    static constexpr int STAGE = P_BYTES + Q_BYTES;       // a multiple of 1024
    static constexpr int RED_LD = JQ + 4;                 // fp32 pitch of the partial tile
    static constexpr int OFF_RED = kStages * STAGE;
    static constexpr int OFF_BAR = OFF_RED + TILE * RED_LD * 4;
    static constexpr int SMEM = OFF_BAR + 2 * kStages * 8 + 16;
    static constexpr int SMEM_ALLOC = SMEM + 1024;        // slack for 1024-byte alignment
};
static_assert(Lay<128>::SMEM_ALLOC <= 232448, "shared memory");

struct Args {
    int64_t M;          // rows of P
    int64_t L;          // columns of P
    int ns;             // reduction tiles per cluster rank
    int64_t nred;       // reduction tiles in all
    int pair;           // column kernel: column offset of a lo half added to its hi half (0: none)
    int jout;           // column kernel: output columns j < jout
    int trans_out;      // column kernel: element (l, j) is output (j, l) (dA) instead of (l, j) (dB)
    int wait_end;       // 1: the inputs are complete before launch (see below): no wait before the
                        // loads; the grid's last CTA waits for the kernel before it before exiting
    FinishArgs f;       // the outputs (f.C, f.splits and the split-sum fields are unused)
};

// Byte offset of 16-byte chunk c of row `row` of a TMA tile with `span`-byte
// rows written with the swizzle of that span (32, 64 or 128 bytes; the tile
// starts on a 1024-byte boundary): chunk bits ^= address bits 7.. .
__device__ __forceinline__ uint32_t swz(int row, int c, int span) {
    const int x = span == 128 ? (row & 7) : span == 64 ? ((row >> 1) & 3) : ((row >> 2) & 1);
    return (uint32_t)(row * span + ((c ^ x) << 4));
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}

__device__ __forceinline__ float4 ld_dsmem_v4(uint32_t addr) {
    float4 v;
    asm volatile("ld.shared::cluster.v4.f32 {%0,%1,%2,%3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(addr) : "memory");
    return v;
}

// The ring, the partial tile and the cluster reduction around a per-stage
// product.  COL selects the column kernel; QT (row kernel) the layout of Q:
// 0 = Q^T stored [j][l] (A), 1 = Q stored [l][j] (B).
template <bool COL, int QT, int JQ>
__device__ __forceinline__ void run(const CUtensorMap* tmP, const CUtensorMap* tmQ, const Args& a) {
    using LY = Lay<JQ>;
    constexpr int QSPAN = JQ >= 64 ? 128 : JQ * 2;        // bytes per row of a [rows][JQ] Q box
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const uint32_t sbase = smem_u32(base);
    const uint32_t bar0 = sbase + LY::OFF_BAR;
    auto full = [&](int i) { return bar0 + 8 * i; };
    auto empty = [&](int i) { return bar0 + 8 * (kStages + i); };
    volatile int* s_abort = reinterpret_cast<volatile int*>(base + LY::OFF_BAR + 2 * kStages * 8);
    float* red = reinterpret_cast<float*>(base + LY::OFF_RED);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t rank = cluster_rank();
    uint32_t zc;
    asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(zc));
    const int z = (int)zc;                                // clusters of z consecutive CTAs along x
    const int64_t t0 = (int64_t)(blockIdx.x / zc) * TILE; // first row (row kernel) / column (column kernel) of P
    const int64_t s_begin = (int64_t)rank * a.ns;
    const int n = (int)(s_begin >= a.nred ? 0 : (a.nred - s_begin < a.ns ? a.nred - s_begin : a.ns));

    grid_dep_launch();
    if (tid == 0) {
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(tmP)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(tmQ)) : "memory");
        for (int i = 0; i < kStages; ++i) {
            tc::mbar_init(full(i), 1);
            tc::mbar_init(empty(i), kCons);
        }
        *s_abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    if (!a.wait_end) grid_dep_wait();

    if (warp == kCons) {
        // ---------------------------------------------------------------- producer
        if (lane == 0) {
            int issued = 0;
            bool ok = true;
            for (int s = 0; s < n; ++s) {
                const int st = s % kStages, ph = (s / kStages) & 1;
                if (!tc::mbar_wait(empty(st), ph ^ 1, s_abort)) { ok = false; break; }
                const uint32_t dst = sbase + st * LY::STAGE;
                const int rpos = (int)((s_begin + s) * TILE);     // position along the reduction
                tc::mbar_expect_tx(full(st), LY::STAGE);
                if (!COL) {
                    tc::tma_load_2d(dst, tmP, full(st), rpos, (int)t0);
                    if (QT == 0) tc::tma_load_2d(dst + P_BYTES, tmQ, full(st), rpos, 0);
                    else tc::tma_load_2d(dst + P_BYTES, tmQ, full(st), 0, rpos);
                } else {
                    tc::tma_load_2d(dst, tmP, full(st), (int)t0, rpos);
                    tc::tma_load_2d(dst + P_BYTES, tmQ, full(st), 0, rpos);
                    if (JQ == 128) tc::tma_load_2d(dst + P_BYTES + 8192, tmQ, full(st), 64, rpos);
                }
                ++issued;
            }
            // on abort: the copies in flight land before the CTA leaves
            if (!ok)
                for (int k = 1; k <= kStages && k <= issued; ++k)
                    tc::mbar_drain(full((issued - k) % kStages), ((issued - k) / kStages) & 1);
        }
    } else {
        // ---------------------------------------------------------------- consumers
        float acc[JQ / 8][4];
#pragma unroll
        for (int t = 0; t < JQ / 8; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.f;
        const int mi = lane >> 3, rr = lane & 7;
        for (int s = 0; s < n; ++s) {
            const int st = s % kStages, ph = (s / kStages) & 1;
            if (!tc::mbar_wait(full(st), ph, s_abort)) break;
            const uint32_t pb = sbase + st * LY::STAGE, qb = pb + P_BYTES;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                uint32_t a0, a1, a2, a3;
                uint32_t b[JQ / 8][2];
                if (!COL) {
                    // A: P rows 16 warp .. +15 (tokens), k = columns 16 kk .. +15 of the tile
                    const int row = 16 * warp + (lane & 15);
                    ldsm_x4(pb + swz(row, 2 * kk + (lane >> 4), 128), a0, a1, a2, a3);
#pragma unroll
                    for (int bb = 0; bb < JQ / 16; ++bb) {
                        if (QT == 0) {
                            const int qrow = 16 * bb + (lane & 7) + ((lane >> 4) << 3);
                            ldsm_x4(qb + swz(qrow, 2 * kk + ((lane >> 3) & 1), 128), b[2 * bb][0], b[2 * bb][1],
                                    b[2 * bb + 1][0], b[2 * bb + 1][1]);
                        } else {
                            const int qrow = 16 * kk + rr + (mi & 1) * 8;
                            ldsm_x4_t(qb + swz(qrow, 2 * bb + (mi >> 1), QSPAN), b[2 * bb][0], b[2 * bb][1],
                                      b[2 * bb + 1][0], b[2 * bb + 1][1]);
                        }
                    }
                } else {
                    // A: (l, m) = P^T, l = columns 16 warp .. +15 of the tile, k = rows 16 kk .. +15
                    const int prow = 16 * kk + rr + (mi >> 1) * 8;
                    ldsm_x4_t(pb + swz(prow, 2 * warp + (mi & 1), 128), a0, a1, a2, a3);
                    const int qrow = 16 * kk + rr + (mi & 1) * 8;
#pragma unroll
                    for (int bb = 0; bb < JQ / 16; ++bb) {
                        const int cj = 2 * bb + (mi >> 1);
                        const uint32_t addr = JQ == 128 ? qb + (uint32_t)((cj >> 3) * 8192) + swz(qrow, cj & 7, 128)
                                                        : qb + swz(qrow, cj, QSPAN);
                        ldsm_x4_t(addr, b[2 * bb][0], b[2 * bb][1], b[2 * bb + 1][0], b[2 * bb + 1][1]);
                    }
                }
#pragma unroll
                for (int t = 0; t < JQ / 8; ++t) mma_bf16_16816(acc[t], a0, a1, a2, a3, b[t][0], b[t][1]);
            }
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(empty(st));
        }
        // partial tile: rows 16 warp + g (+ 8), columns 8 t + 2 q (+ 1)
        const int g = lane >> 2, q = lane & 3;
#pragma unroll
        for (int t = 0; t < JQ / 8; ++t) {
            float* r0 = red + (16 * warp + g) * LY::RED_LD + 8 * t + 2 * q;
            *reinterpret_cast<float2*>(r0) = make_float2(acc[t][0], acc[t][1]);
            *reinterpret_cast<float2*>(r0 + 8 * LY::RED_LD) = make_float2(acc[t][2], acc[t][3]);
        }
    }
    __syncthreads();
    cluster_sync();                       // every partial tile of the cluster is in place

    // ---------------------------------------------------------------- reduction + outputs
    const int r_lo = (int)(TILE * rank / z), r_hi = (int)(TILE * (rank + 1) / z);
    const uint32_t red_s = smem_u32(red);
    const FinishArgs& f = a.f;
    if (!COL) {
        // rows of the output = tokens t0 + row; columns j < f.Jiter (JQ and beyond read as 0)
        const int jq4 = (int)(f.Jiter / 4);
        for (int e = tid; e < (r_hi - r_lo) * jq4; e += kThreads) {
            const int row = r_lo + e / jq4, j = 4 * (e % jq4);
            const int64_t i = t0 + row;
            if (i >= a.M) continue;
            float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
            if (j < JQ) {
                const uint32_t off = red_s + (uint32_t)((row * LY::RED_LD + j) * 4);
                float4 pv[kMaxCluster];
#pragma unroll
                for (int p = 0; p < kMaxCluster; ++p)
                    if (p < z) pv[p] = ld_dsmem_v4(mapa(off, (uint32_t)p));
#pragma unroll
                for (int p = 0; p < kMaxCluster; ++p)
                    if (p < z) { v.x += pv[p].x; v.y += pv[p].y; v.z += pv[p].z; v.w += pv[p].w; }
            }
            const float vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const int64_t jj = j + c;
                finish_store(f, i, jj, jj < f.J ? __fmul_rn(vv[c], f.pre) : 0.f);
            }
        }
    } else {
        // rows of the tile = columns l = t0 + row of P; output columns j < a.jout
        const int jo4 = (a.jout + 3) / 4;
        for (int e = tid; e < (r_hi - r_lo) * jo4; e += kThreads) {
            const int row = r_lo + e / jo4, j = 4 * (e % jo4);
            const int64_t l = t0 + row;
            if (l >= a.L) continue;
            float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
            for (int h = 0; h < (a.pair > 0 ? 2 : 1); ++h) {
                const uint32_t off = red_s + (uint32_t)((row * LY::RED_LD + j + h * a.pair) * 4);
                float4 pv[kMaxCluster];
#pragma unroll
                for (int p = 0; p < kMaxCluster; ++p)
                    if (p < z) pv[p] = ld_dsmem_v4(mapa(off, (uint32_t)p));
#pragma unroll
                for (int p = 0; p < kMaxCluster; ++p)
                    if (p < z) { v.x += pv[p].x; v.y += pv[p].y; v.z += pv[p].z; v.w += pv[p].w; }
            }
            const float vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const int jj = j + c;
                if (jj >= a.jout) break;
                const float w = __fmul_rn(vv[c], f.pre);
                if (a.trans_out) finish_store(f, jj, l, w);
                else finish_store(f, l, jj, w);
            }
        }
    }
    cluster_sync();                       // no CTA leaves while its partial tile may still be read
    if (a.wait_end && blockIdx.x == gridDim.x - 1 && tid == 0) grid_dep_wait();
}

template <int QT, int JQ>
__global__ void __launch_bounds__(kThreads) k_rowk(const __grid_constant__ CUtensorMap tmP,
                                                   const __grid_constant__ CUtensorMap tmQ, const Args a) {
    run<false, QT, JQ>(&tmP, &tmQ, a);
}

template <int JQ>
__global__ void __launch_bounds__(kThreads) k_colk(const __grid_constant__ CUtensorMap tmP,
                                                   const __grid_constant__ CUtensorMap tmQ, const Args a) {
    run<true, 0, JQ>(&tmP, &tmQ, a);
}

}  // namespace sk
}  // namespace qnf4
