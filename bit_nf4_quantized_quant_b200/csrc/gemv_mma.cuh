// gemv_mma.cuh -- small-M forward (M <= 32 tokens): fused exact NF4 decode +
// mma.sync, with the packed weight staged by TMA and the work split evenly
// over one CTA per SM.
//
//   Y [M, N] = X [M, K] . W'^T + s T B^T,   W' = bf16_rne(L[q] c')
//
// At a few tokens the layer is bound by the integer-pipe work of the exact
// decode (a 16-entry bf16 table per 64-weight block and byte permutes, see
// nf4_decode.cuh), so the kernel is built around keeping that pipe busy:
//
//  * The decoded bf16 pairs are the A operand of mma.sync m16n8k16 straight
//    from registers (W rows are the MMA rows, tokens its 8-wide columns), so
//    the weight never goes back to shared memory.  A lane (g, t) of the MMA
//    holds rows g and g + 8 and, in MMA s, the logical k {2t, 2t+1, 2t+8,
//    2t+9}; these are mapped to elements 4s .. 4s+3 of 64-weight block t of a
//    256-wide step, so over the 16 MMAs of a step every lane decodes exactly
//    two whole blocks (rows g and g + 8) and builds two tables.
//  * Work unit = (128 rows, 256 reduction) = 8 warps x 16 rows.  The units
//    are split evenly over the CTAs in (tile, step) order; in a CTA two
//    groups of 8 warps take alternate units, each group with its own producer
//    warp and its own half of the stage ring.  Every (CTA, group) pair writes
//    its partial sum of each tile it touched to its own slot; the small
//    k_nf4_gemv_finish kernel sums the slots of a tile in (CTA, group) order
//    -- deterministic -- and adds s T B^T (no atomics or counters, so the
//    fused kernel ends as soon as its last unit is done).
//  * A producer warp's lane 0 loads each unit's packed tile (128 rows x 128 B,
//    128-byte swizzle) with TMA; its 32 lanes copy the unit's activation slice
//    with cp.async into a fragment-native layout ([j][token][t] 16-byte
//    chunks: the 16 bytes lane (g, t) feeds to MMAs 2j and 2j+1), so the
//    consumers' shared loads are conflict-free; both complete on the stage's
//    mbarrier.  Rows of the slice beyond M are zeroed once and never copied.
//  * Three programmatic launches make the forward: this kernel, then the
//    small T = X A^T kernel (which runs beside it on the SMs' spare registers
//    and ends only after it), then the finish kernel.  Before it waits for
//    the kernel ahead of it on the stream, the GEMV only sets up its barriers
//    and warms L2 with each group's first packed tile (an L2 prefetch cannot
//    return stale data: L2 is the point of coherence); everything it reads is
//    read after the wait, and it releases the T kernel right after it.
#pragma once
#include <cuda.h>
#include "common.cuh"
#include "nf4_decode.cuh"
#include "tc_gemm.cuh"

namespace qnf4 {
namespace gmv {

constexpr int TR = 128;                          // rows of a unit
constexpr int KSTEP = 256;                       // reduction of a unit
constexpr int P_BYTES = TR * KSTEP / 2;          // 16384
constexpr int kGroupWarps = 8;
constexpr int kFirstMath = 2;                    // warps 0, 1: producers of groups 0, 1; 2 .. 17: decode + MMA
constexpr int kThreads = 32 * (kFirstMath + 2 * kGroupWarps);   // 576

template <int NTT>
struct Cfg {
    static constexpr int NT = 8 * NTT;                  // token columns (zero beyond M)
    static constexpr int X_BYTES = NT * KSTEP * 2;      // 4096 * NTT
    static constexpr int STAGE = P_BYTES + X_BYTES;     // a multiple of 1024
    static constexpr int SP = NTT == 4 ? 4 : 8;         // stages, a power of 2
    static constexpr int SPG = SP / 2;                  // stages of each group's ring
    static constexpr int OFF_BAR = SP * STAGE;
    static constexpr int SMEM_ALLOC = OFF_BAR + 2 * SP * 8 + 16 + 1024;
};

struct Args {
    const uint16_t* X;         // [M, K] bf16
    const int8_t* codes;
    const float* scale;
    const float* mean;
    int64_t M, N, K;
    int tiles, nks;            // ceil(N / 128), ceil(K / 256)
    int64_t units;             // tiles * nks
    int ctas;
    float* slots;              // [(ctas + tiles) * 2][NT][128] fp32 partial tiles
};

__host__ __device__ __forceinline__ int64_t unit_begin(int64_t c, int64_t U, int64_t C) { return c * U / C; }
__device__ __forceinline__ void unit_advance(int& tile, int& ks, int n, int nks) {
    ks += n;
    while (ks >= nks) { ks -= nks; ++tile; }
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, int src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}

__device__ __forceinline__ void tma_prefetch_l2(const CUtensorMap* map, int x, int y) {
    asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];"
                 ::"l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y) : "memory");
}

template <int NTT>
__global__ void __launch_bounds__(kThreads, 1) k_nf4_gemv(const __grid_constant__ CUtensorMap tmP, Args a,
                                                        NF4Tables tab) {
    using C = Cfg<NTT>;
    constexpr int NT = C::NT;
    constexpr int SP = C::SP;
    constexpr int SPG = C::SPG;
    extern __shared__ __align__(1024) uint8_t smem[];
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem) + 1023) & ~(uintptr_t)1023);
    const uint32_t sbase = smem_u32(base);
    const uint32_t bar0 = sbase + C::OFF_BAR;
    auto full = [&](int i) { return bar0 + 8 * i; };
    auto empty = [&](int i) { return bar0 + 8 * (SP + i); };
    volatile int* s_abort = reinterpret_cast<volatile int*>(base + C::OFF_BAR + 2 * SP * 8);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t U = a.units;
    const int u0 = (int)unit_begin(blockIdx.x, U, a.ctas), u1 = (int)unit_begin(blockIdx.x + 1, U, a.ctas);
    const int nu = u1 - u0;
    const int nks = a.nks;
    const int tile0 = u0 / nks, ks0 = u0 - tile0 * nks;
    const uint32_t nblk32 = (uint32_t)(a.K / kBlock), N32 = (uint32_t)a.N;

    // token rows >= M of every stage's activation slice stay zero
    for (int e = tid; e < SP * NT * 32; e += kThreads) {
        const int st = e / (NT * 32), c = e % (NT * 32);
        if ((c / 4) % NT >= a.M) {
            const uint32_t dst = sbase + st * C::STAGE + P_BYTES + c * 16;
            asm volatile("st.shared.v4.u32 [%0], {%1,%1,%1,%1};" ::"r"(dst), "r"(0u) : "memory");
        }
    }
    if (tid == 0) {
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmP)) : "memory");
        for (int i = 0; i < SP; ++i) {
            tc::mbar_init(full(i), 1 + 32);              // TMA expect-tx arrival + 32 cp.async arrivals
            tc::mbar_init(empty(i), kGroupWarps);
        }
        *s_abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();

    // CTA-local unit i belongs to group i & 1; its group-local index q = i >> 1
    // selects stage (group, q mod SPG) with parity (q / SPG) & 1.
    if (warp < kFirstMath) {
        // ------------------------------------------------------------ producer of group `warp`
        const int grp = warp;
        const int nq = nu > grp ? (nu - grp + 1) / 2 : 0;
        int tile = tile0, ks = ks0;
        unit_advance(tile, ks, grp, nks);
        // warm L2 with the group's first packed tile only: every CTA's first tile is then
        // at the front of the memory queue (the rest streams through the stage ring)
        if (lane == 0 && nq > 0) tma_prefetch_l2(&tmP, ks * (KSTEP / 2), tile * TR);
        grid_dep_wait();
        // X is complete: the T kernel launched behind this one may start (and read it)
        if (grp == 0 && lane == 0) grid_dep_launch();
        int issued = 0;
        bool ok = true;
        const int64_t mrows = a.M < NT ? a.M : NT;
        for (int q = 0; q < nq; ++q) {
            const int st = grp * SPG + q % SPG, ph = (q / SPG) & 1;
            int w_ok = 1;
            if (lane == 0) w_ok = tc::mbar_wait(empty(st), ph ^ 1, s_abort) ? 1 : 0;
            ok = __shfl_sync(0xffffffffu, w_ok, 0) != 0;
            if (!ok) break;
            const uint32_t sdst = sbase + st * C::STAGE;
            if (lane == 0) {
                tc::mbar_expect_tx(full(st), P_BYTES);
                tc::tma_load_2d(sdst, &tmP, full(st), ks * (KSTEP / 2), tile * TR);
            }
            // activation chunks (m, t, j): 16 bytes of row m at k = 256 ks + 64 t + 8 j,
            // stored at chunk (j * NT + m) * 4 + t of the slice; zero beyond K
            for (int c = lane; c < mrows * 32; c += 32) {
                const int m = c >> 5, t = (c >> 3) & 3, j = c & 7;
                const int64_t k = (int64_t)ks * KSTEP + 64 * t + 8 * j;
                const bool in = k < a.K;
                const uint16_t* src = a.X + (in ? (int64_t)m * a.K + k : 0);
                cp_async16(sdst + P_BYTES + ((j * NT + m) * 4 + t) * 16, src, in ? 16 : 0);
            }
            asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(full(st)) : "memory");
            ++issued;
            unit_advance(tile, ks, 2, nks);
        }
        // on abort: let the copies in flight land before the CTA exits
        asm volatile("cp.async.wait_all;" ::: "memory");
        if (!ok && lane == 0)
            for (int k = 1; k <= SPG && k <= issued; ++k)
                tc::mbar_drain(full(grp * SPG + (issued - k) % SPG), ((issued - k) / SPG) & 1);
    } else {
        // ------------------------------------------------------------ decode + MMA warps
        const int grp = (warp - kFirstMath) / kGroupWarps;    // units i = grp, grp + 2, ...
        const int w8 = (warp - kFirstMath) % kGroupWarps;     // rows 16 w8 .. 16 w8 + 15 of a unit
        const int g = lane >> 2, t = lane & 3;
        const int r0 = 16 * w8 + g;                      // rows r0 and r0 + 8 of the tile
        bool ok = true;
        grid_dep_wait();

        // block-constant inputs of rows r0, r0 + 8, block 4 ks + t of the next unit to
        // fetch (zero beyond the weight); fetches run two group-units ahead
        int fi = grp, ft = tile0, fk = ks0;
        unit_advance(ft, fk, grp, nks);
        struct BC { int c0, c1; float s0, s1, m0, m1; };
        auto fetch = [&](BC& b) {
            b.c0 = b.c1 = 0; b.s0 = b.s1 = b.m0 = b.m1 = 0.f;
            const int tile = ft, ks = fk;
            const bool in = fi < nu;
            fi += 2;
            unit_advance(ft, fk, 2, nks);
            // block indices fit 32 bits (the weight has fewer than 2^38 elements)
            const uint32_t kb = (uint32_t)ks * 4u + (uint32_t)t;
            if (!in || kb >= nblk32) return;
            const uint32_t n0 = (uint32_t)tile * TR + (uint32_t)r0, n1 = n0 + 8u;
            if (n0 < N32) {
                const uint32_t bb = n0 * nblk32 + kb;
                b.c0 = __ldg(a.codes + bb); b.s0 = __ldg(a.scale + (bb >> 8)); b.m0 = __ldg(a.mean + (bb >> 8));
            }
            if (n1 < N32) {
                const uint32_t bb = n1 * nblk32 + kb;
                b.c1 = __ldg(a.codes + bb); b.s1 = __ldg(a.scale + (bb >> 8)); b.m1 = __ldg(a.mean + (bb >> 8));
            }
        };

        float acc[NTT][4];
#pragma unroll
        for (int nt = 0; nt < NTT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;

        // publish this warp's 16 rows x NT tokens of `tile` after the group's last unit of
        // it: partial slot ((CTA + tile) * 2 + group), summed later by k_nf4_gemv_finish
        auto publish = [&](int tile) {
            float* sp = a.slots + (((int64_t)blockIdx.x + tile) * 2 + grp) * (NT * TR);
#pragma unroll
            for (int nt = 0; nt < NTT; ++nt) {
                const int m = 8 * nt + 2 * t;
                sp[m * TR + r0] = acc[nt][0];
                sp[(m + 1) * TR + r0] = acc[nt][1];
                sp[m * TR + r0 + 8] = acc[nt][2];
                sp[(m + 1) * TR + r0 + 8] = acc[nt][3];
                acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
            }
        };

        BC bA, bB;
        fetch(bA);
        fetch(bB);
        int tile = tile0, ks = ks0;
        unit_advance(tile, ks, grp, nks);
        // swizzled offsets of this lane's packed chunks (row r0; row r0 + 8 has the same swizzle)
        const uint32_t pch0 = (uint32_t)(r0 * 128 + (((2 * t) ^ (r0 & 7)) << 4));
        const uint32_t pch1 = (uint32_t)(r0 * 128 + (((2 * t + 1) ^ (r0 & 7)) << 4));
        auto do_unit = [&](int q, BC& b) {
            const float c0 = __fmaf_rn((float)b.c0, b.s0, b.m0), c1 = __fmaf_rn((float)b.c1, b.s1, b.m1);
            fetch(b);
            const int st = grp * SPG + q % SPG, ph = (q / SPG) & 1;
            if (!(ok = tc::mbar_wait(full(st), ph, s_abort))) return;
            const uint32_t sst = sbase + st * C::STAGE;
            uint32_t pa[8], pb[8];
            asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(pa[0]), "=r"(pa[1]), "=r"(pa[2]), "=r"(pa[3]) : "r"(sst + pch0));
            asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(pa[4]), "=r"(pa[5]), "=r"(pa[6]), "=r"(pa[7]) : "r"(sst + pch1));
            asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(pb[0]), "=r"(pb[1]), "=r"(pb[2]), "=r"(pb[3]) : "r"(sst + pch0 + 1024));
            asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(pb[4]), "=r"(pb[5]), "=r"(pb[6]), "=r"(pb[7]) : "r"(sst + pch1 + 1024));
            const BlockTable ta = make_block_table(tab, c0), tb = make_block_table(tab, c1);
            const uint32_t xb = sst + P_BYTES + (uint32_t)(lane * 16);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                uint32_t oa[4], ob[4];
                decode8(ta, pa[j], oa);
                decode8(tb, pb[j], ob);
#pragma unroll
                for (int nt = 0; nt < NTT; ++nt) {
                    uint32_t x0, x1, x2, x3;
                    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                                 : "=r"(x0), "=r"(x1), "=r"(x2), "=r"(x3)
                                 : "r"(xb + (uint32_t)((j * NT + 8 * nt) * 64)));
                    mma_bf16_16816(acc[nt], oa[0], ob[0], oa[1], ob[1], x0, x1);
                    mma_bf16_16816(acc[nt], oa[2], ob[2], oa[3], ob[3], x2, x3);
                }
            }
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(empty(st));
        };
        for (int i = grp, q = 0; i < nu && ok; i += 2, ++q) {
            do_unit(q, (q & 1) ? bB : bA);
            if (!ok) break;
            // the group's next unit is i + 2: finish this tile's segment when it leaves the tile
            const int cur = tile;
            unit_advance(tile, ks, 2, nks);
            if (tile != cur || i + 2 >= nu) publish(cur);
        }
    }
}

// Sum of the partial tiles of every (CTA, group) pair that took units of
// `tile`, in (CTA, group) order, plus s T B^T; CTA = (one 128-row tile, MT
// tokens), thread = one row n.  T is summed over its K splits, in split
// order, into shared memory (tile 0 also hands the caller its bf16 copy).
// Launched programmatically after the T kernel: it lets the next kernel on the
// stream launch, then waits for the T kernel, which completes only after the
// GEMV has.  After the wait, the partial-tile, B-row and T loads are all
// issued before the first of them is used (one round trip to L2).
struct FinishArgs {
    const float* slots;
    int64_t M, N;
    int nks, ctas, NT;
    int64_t units;
    const float* Tpart;        // [kc][M, rp] fp32 split sums of T = X A^T
    int kc, rp, r;
    const uint16_t* lora_B;
    int b_vec;
    float s;
    float tscale;              // T = tscale * (sum of the splits); 1 except under LoRA dropout
    uint16_t* Y;
    uint16_t* T_out;           // [M, r] bf16 copy of T for the caller, or null
};

constexpr int kFinSlots = 4;   // partial tiles loaded per batch
constexpr int kFinB = 4;       // 8-wide chunks of the B row held in registers (r <= 32)

template <int MT>
__global__ void __launch_bounds__(TR, 8) k_nf4_gemv_finish(FinishArgs a) {
    __shared__ float s_T[MT * 256];     // [MT][r], r <= 256
    __shared__ int s_mask[148];         // groups of CTA c_first + j that took units of this tile
    __shared__ int s_slot[2 * 148];     // their slots, in (CTA, group) order
    __shared__ int s_n;
    grid_dep_launch();
    const int tile = blockIdx.x, row = threadIdx.x;
    const int r = a.r;
    const int m0 = blockIdx.y * MT;
    const int mn = a.M - m0 < MT ? (int)a.M - m0 : MT;
    const int64_t n = (int64_t)tile * TR + row;
    const bool live = n < a.N;
    // Before the wait: what depends on the split only (integer arithmetic), and an
    // L2 prefetch of this row of B.
    // unit counts fit 32 bits and CTA * units < 2^32 (units < 2^24, at most 148 CTAs)
    const uint32_t U = (uint32_t)a.units, C = (uint32_t)a.ctas;
    const uint32_t tu0 = (uint32_t)tile * (uint32_t)a.nks, tu1 = tu0 + (uint32_t)a.nks;
    const uint32_t c_first = ((tu0 + 1) * C + U - 1) / U - 1, c_last = (tu1 * C + U - 1) / U - 1;
    const int ncta = (int)(c_last - c_first + 1);
    for (int j = row; j < ncta; j += TR) {
        const uint32_t c = c_first + (uint32_t)j;
        const uint32_t b0 = c * U / C, b1 = (c + 1) * U / C;
        const uint32_t lo = b0 > tu0 ? b0 : tu0, hi = b1 < tu1 ? b1 : tu1;
        s_mask[j] = hi - lo >= 2 ? 3 : (hi - lo == 1 ? 1 << ((lo - b0) & 1) : 0);
    }
    const uint16_t* br = a.lora_B + (live ? n : 0) * r;
    if (live) asm volatile("prefetch.global.L2 [%0];" ::"l"(br));
    __syncthreads();
    if (row == 0) {
        int k = 0;
        for (int j = 0; j < ncta; ++j)
            for (int g2 = 0; g2 < 2; ++g2)
                if ((s_mask[j] >> g2) & 1) s_slot[k++] = (int)(((int64_t)c_first + j + tile) * 2 + g2);
        s_n = k;
    }
    __syncthreads();
    const int ns = s_n;
    grid_dep_wait();

    // partial tiles, kFinSlots at a time, summed in slot order
    float v[MT];
#pragma unroll
    for (int mm = 0; mm < MT; ++mm) v[mm] = 0.f;
    const bool bregs = live && a.b_vec && r <= 8 * kFinB;
    uint4 bq[kFinB];
    if (live) {
        for (int k0 = 0; k0 < ns; k0 += kFinSlots) {
            float t[kFinSlots][MT];
#pragma unroll
            for (int k = 0; k < kFinSlots; ++k) {
                const float* sp = a.slots + (int64_t)s_slot[k0 + k < ns ? k0 + k : k0] * (a.NT * TR) +
                                  (int64_t)m0 * TR + row;
#pragma unroll
                for (int mm = 0; mm < MT; ++mm) t[k][mm] = (k0 + k < ns && mm < mn) ? sp[mm * TR] : 0.f;
            }
            if (k0 == 0 && bregs) {
#pragma unroll
                for (int c = 0; c < kFinB; ++c) bq[c] = 8 * c < r ? ldg_cg_v4(br + 8 * c) : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int k = 0; k < kFinSlots; ++k)
#pragma unroll
                for (int mm = 0; mm < MT; ++mm)
                    if (k0 + k < ns) v[mm] += t[k][mm];
        }
    }
    // T over its K splits, in split order
    for (int e = row; e < mn * r; e += TR) {
        const int mm = e / r, i = e - mm * r;
        const float* tp = a.Tpart + ((int64_t)m0 + mm) * a.rp + i;
        const int64_t zs = a.M * a.rp;
        float t = 0.f;
        int z = 0;
        for (; z + 4 <= a.kc; z += 4) {
            const float t0 = tp[z * zs], t1 = tp[(z + 1) * zs], t2 = tp[(z + 2) * zs], t3 = tp[(z + 3) * zs];
            t += t0; t += t1; t += t2; t += t3;
        }
        for (; z < a.kc; ++z) t += tp[z * zs];
        t = __fmul_rn(t, a.tscale);
        s_T[e] = t;
        if (tile == 0 && a.T_out != nullptr)
            a.T_out[(int64_t)(m0 + mm) * r + i] = (uint16_t)(pack_bf16x2(t, 0.f) & 0xffffu);
    }
    __syncthreads();
    if (!live) return;
    // s T B^T
    float l[MT];
#pragma unroll
    for (int mm = 0; mm < MT; ++mm) l[mm] = 0.f;
    auto chunk = [&](const uint4& bv, int i) {
        const uint32_t bw[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
        for (int mm = 0; mm < MT; ++mm) {
            if (mm < mn) {
                const float* tm = s_T + mm * r + i;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    l[mm] = __fmaf_rn(tm[2 * j], bf16lo_to_f32(bw[j]), l[mm]);
                    l[mm] = __fmaf_rn(tm[2 * j + 1], bf16hi_to_f32(bw[j]), l[mm]);
                }
            }
        }
    };
    if (bregs) {
#pragma unroll
        for (int c = 0; c < kFinB; ++c)
            if (8 * c < r) chunk(bq[c], 8 * c);
    } else if (a.b_vec) {
        for (int i = 0; i < r; i += 8) chunk(ldg_cg_v4(br + i), i);
    } else {
        for (int i = 0; i < r; ++i) {
            const float b = bf16lo_to_f32(br[i]);
#pragma unroll
            for (int mm = 0; mm < MT; ++mm)
                if (mm < mn) l[mm] = __fmaf_rn(s_T[mm * r + i], b, l[mm]);
        }
    }
#pragma unroll
    for (int mm = 0; mm < MT; ++mm)
        if (mm < mn)
            a.Y[(int64_t)(m0 + mm) * a.N + n] = (uint16_t)(pack_bf16x2(__fmaf_rn(a.s, l[mm], v[mm]), 0.f) & 0xffffu);
}

}  // namespace gmv
}  // namespace qnf4
