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
//    barrier, CTA q sums the q-th of z equal runs of the tile's outputs over the
//    ranks in rank order through distributed shared memory and writes every
//    output of those elements itself (fp32, bf16, hi + lo pairs, scaled
//    copies), 8 consecutive elements per thread: two 16-byte loads per rank
//    and one 16-byte store per output array (dA's partial tile is stored
//    transposed so that its 8 elements are contiguous too).  One store per
//    element and array cost more than the rest of the kernel.  The result is
//    deterministic and no partial sums go through HBM or a second kernel.
//  * Programmatic launch: the kernel waits for the one before it before the
//    producer's first load and any store, then lets the next one launch -- or,
//    with wait_end, where every input is known complete and
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
    static constexpr int RED_LD = JQ + 4;                 // fp32 pitch of the partial tile [64][JQ]
    static constexpr int RT_LD = TILE + 4;                // ... stored transposed [JQ][64] (dA)
    static constexpr int RED_FLOATS = TILE * RED_LD > JQ * RT_LD ? TILE * RED_LD : JQ * RT_LD;
    static constexpr int OFF_RED = kStages * STAGE;
    static constexpr int OFF_BAR = OFF_RED + RED_FLOATS * 4;
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
    int* zero;          // row kernel: nzero ints set to 0 (the stream-K counters of the fused
    int64_t nzero;      // kernel launched next, which starts after this one has completed)
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

    if (a.wait_end) grid_dep_launch();
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
    if (!a.wait_end) {
        // the next kernel (the fused one, itself launched programmatically) may start once
        // everything before this one has completed: it then reads only inputs that are ready,
        // except this kernel's outputs, for which it waits
        grid_dep_wait();
        grid_dep_launch();
    }

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
        // partial tile: rows 16 warp + g (+ 8), columns 8 t + 2 q (+ 1); transposed for dA
        const int g = lane >> 2, q = lane & 3;
        if (COL && a.trans_out) {
#pragma unroll
            for (int t = 0; t < JQ / 8; ++t) {
                float* r0 = red + (8 * t + 2 * q) * LY::RT_LD + 16 * warp + g;
                r0[0] = acc[t][0];
                r0[LY::RT_LD] = acc[t][1];
                r0[8] = acc[t][2];
                r0[LY::RT_LD + 8] = acc[t][3];
            }
        } else {
#pragma unroll
            for (int t = 0; t < JQ / 8; ++t) {
                float* r0 = red + (16 * warp + g) * LY::RED_LD + 8 * t + 2 * q;
                *reinterpret_cast<float2*>(r0) = make_float2(acc[t][0], acc[t][1]);
                *reinterpret_cast<float2*>(r0 + 8 * LY::RED_LD) = make_float2(acc[t][2], acc[t][3]);
            }
        }
    }
    __syncthreads();
    cluster_sync();                       // every partial tile of the cluster is in place

    // ---------------------------------------------------------------- reduction + outputs
    // Output groups of 8 consecutive elements, dealt out to the ranks in contiguous runs;
    // a group is 8 partial values of every rank (two 16-byte loads each) summed in rank
    // order, then 16-byte stores.
    const uint32_t red_s = smem_u32(red);
    const FinishArgs& f = a.f;
    auto sum8 = [&](uint32_t off, float (&v)[8]) {
        float4 lo[kMaxCluster], hi[kMaxCluster];
#pragma unroll
        for (int p = 0; p < kMaxCluster; ++p)
            if (p < z) {
                const uint32_t ad = mapa(off, (uint32_t)p);
                lo[p] = ld_dsmem_v4(ad);
                hi[p] = ld_dsmem_v4(ad + 16);
            }
#pragma unroll
        for (int p = 0; p < kMaxCluster; ++p)
            if (p < z) {
                v[0] += lo[p].x; v[1] += lo[p].y; v[2] += lo[p].z; v[3] += lo[p].w;
                v[4] += hi[p].x; v[5] += hi[p].y; v[6] += hi[p].z; v[7] += hi[p].w;
            }
    };
    if (!COL) {
        // row i = t0 + row; value groups j0 = 8 gi < rp (f.J), then the zero columns
        // [2 rp, J2pad) of the s-scaled hi | lo copy
        const int vg = (int)(f.J / 8);
        const int zg = f.o2 ? (int)((f.J2pad - 2 * f.o2_lo) / 8) : 0;
        const int gpr = vg + zg;
        const int G = TILE * gpr;
        const int g_lo = (int)((int64_t)G * rank / z), g_hi = (int)((int64_t)G * (rank + 1) / z);
        const bool o1vec = f.o1 && f.s1i % 8 == 0 && (reinterpret_cast<uintptr_t>(f.o1) & 15) == 0;
        for (int e = g_lo + tid; e < g_hi; e += kThreads) {
            const int row = e / gpr, gi = e - row * gpr;
            const int64_t i = t0 + row;
            if (i >= a.M) continue;
            if (gi >= vg) {
                *reinterpret_cast<uint4*>(f.o2 + i * f.s2i + 2 * f.o2_lo + 8 * (gi - vg)) = make_uint4(0, 0, 0, 0);
                continue;
            }
            const int j0 = 8 * gi;
            float v[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            sum8(red_s + (uint32_t)((row * LY::RED_LD + j0) * 4), v);
#pragma unroll
            for (int c = 0; c < 8; ++c) v[c] = __fmul_rn(v[c], f.pre);
            if (f.f32) {
                float4* d = reinterpret_cast<float4*>(f.f32 + i * f.ld_f32 + j0);
                d[0] = make_float4(v[0], v[1], v[2], v[3]);
                d[1] = make_float4(v[4], v[5], v[6], v[7]);
            }
            uint32_t h[4], l[4], sh[4], sl[4], b[4];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const bool in0 = j0 + 2 * c < f.J1, in1 = j0 + 2 * c + 1 < f.J1;
                const float x0 = in0 ? v[2 * c] : 0.f, x1 = in1 ? v[2 * c + 1] : 0.f;
                h[c] = pack_bf16x2(x0, x1);
                l[c] = pack_bf16x2(x0 - bf16lo_to_f32(h[c]), x1 - bf16hi_to_f32(h[c]));
                const float s0 = in0 ? __fmul_rn(f.alpha2, v[2 * c]) : 0.f;
                const float s1 = in1 ? __fmul_rn(f.alpha2, v[2 * c + 1]) : 0.f;
                sh[c] = pack_bf16x2(s0, s1);
                sl[c] = pack_bf16x2(s0 - bf16lo_to_f32(sh[c]), s1 - bf16hi_to_f32(sh[c]));
                b[c] = pack_bf16x2(in0 ? __fmul_rn(f.alpha1, v[2 * c]) : 0.f, in1 ? __fmul_rn(f.alpha1, v[2 * c + 1]) : 0.f);
            }
            if (f.hl) {
                *reinterpret_cast<uint4*>(f.hl + i * f.hl_ld + j0) = make_uint4(h[0], h[1], h[2], h[3]);
                *reinterpret_cast<uint4*>(f.hl + i * f.hl_ld + f.hl_off + j0) = make_uint4(l[0], l[1], l[2], l[3]);
            }
            if (f.o2) {
                *reinterpret_cast<uint4*>(f.o2 + i * f.s2i + j0) = make_uint4(sh[0], sh[1], sh[2], sh[3]);
                *reinterpret_cast<uint4*>(f.o2 + i * f.s2i + f.o2_lo + j0) = make_uint4(sl[0], sl[1], sl[2], sl[3]);
            }
            if (f.o1 && j0 < f.J1pad) {
                if (o1vec && j0 + 8 <= f.J1pad) {
                    *reinterpret_cast<uint4*>(f.o1 + i * f.s1i + j0) = make_uint4(b[0], b[1], b[2], b[3]);
                } else {
#pragma unroll
                    for (int c = 0; c < 8; ++c)
                        if (j0 + c < f.J1pad)
                            f.o1[i * f.s1i + (j0 + c) * f.s1j] =
                                (uint16_t)((c & 1) ? (b[c >> 1] >> 16) : (b[c >> 1] & 0xffffu));
                }
            }
        }
    } else {
        // out (l, j) = alpha1 * pre * (sum over ranks of the partial at (l, j) [+ at (l, j + pair)]),
        // stored at o1[l * s1i + j] (dB) or o1[j * s1i + l] (dA, from the transposed tile)
        const bool tr = a.trans_out != 0;
        const int jg = (a.jout + 7) / 8;
        const int G = tr ? a.jout * (TILE / 8) : TILE * jg;
        const int g_lo = (int)((int64_t)G * rank / z), g_hi = (int)((int64_t)G * (rank + 1) / z);
        const bool vec = f.s1i % 8 == 0 && (reinterpret_cast<uintptr_t>(f.o1) & 15) == 0;
        for (int e = g_lo + tid; e < g_hi; e += kThreads) {
            int j, l_loc;
            uint32_t off, off2;
            if (tr) {
                j = e / (TILE / 8);
                l_loc = 8 * (e - j * (TILE / 8));
                off = red_s + (uint32_t)((j * LY::RT_LD + l_loc) * 4);
                off2 = off + (uint32_t)(a.pair * LY::RT_LD * 4);
            } else {
                l_loc = e / jg;
                j = 8 * (e - l_loc * jg);
                off = red_s + (uint32_t)((l_loc * LY::RED_LD + j) * 4);
                off2 = off + (uint32_t)(a.pair * 4);
            }
            float v[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            sum8(off, v);
            if (a.pair > 0) sum8(off2, v);
            uint32_t b[4];
#pragma unroll
            for (int c = 0; c < 4; ++c)
                b[c] = pack_bf16x2(__fmul_rn(f.alpha1, __fmul_rn(v[2 * c], f.pre)),
                                   __fmul_rn(f.alpha1, __fmul_rn(v[2 * c + 1], f.pre)));
            if (tr) {
                const int64_t l0 = t0 + l_loc;
                uint16_t* d = f.o1 + (int64_t)j * f.s1i + l0;
                if (vec && l0 + 8 <= a.L) {
                    *reinterpret_cast<uint4*>(d) = make_uint4(b[0], b[1], b[2], b[3]);
                } else {
#pragma unroll
                    for (int c = 0; c < 8; ++c)
                        if (l0 + c < a.L) d[c] = (uint16_t)((c & 1) ? (b[c >> 1] >> 16) : (b[c >> 1] & 0xffffu));
                }
            } else {
                const int64_t l = t0 + l_loc;
                if (l >= a.L) continue;
                uint16_t* d = f.o1 + l * f.s1i + j;
                if (vec && j + 8 <= a.jout) {
                    *reinterpret_cast<uint4*>(d) = make_uint4(b[0], b[1], b[2], b[3]);
                } else {
#pragma unroll
                    for (int c = 0; c < 8; ++c)
                        if (j + c < a.jout) d[c] = (uint16_t)((c & 1) ? (b[c >> 1] >> 16) : (b[c >> 1] & 0xffffu));
                }
            }
        }
    }
    if (!COL)
        for (int64_t i = (int64_t)blockIdx.x * kThreads + tid; i < a.nzero; i += (int64_t)gridDim.x * kThreads)
            a.zero[i] = 0;
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
