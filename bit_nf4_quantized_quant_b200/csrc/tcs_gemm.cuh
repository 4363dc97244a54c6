// tcs_gemm.cuh -- backward dX = dY W' for a few tokens (M <= 32) on tcgen05:
// the fused exact NF4 dequant feeds the MMA's A operand, the tokens are its
// N dimension.
//
//   dX^T [K, M] = W'^T [K, N] . dY^T [N, M]      (s A^T U^T is added by k_bwd_small_end)
//
// The weight is the MMA's A operand (M_mma = 128 columns of W; W's rows are
// the reduction, so the dequantized tile is stored MN-major) and the tokens
// are its N dimension (NT = 16 or 32, zero rows beyond M from the TMA's
// out-of-bound fill).  Work unit = (128 output columns, 128 reduction rows).
// The units are split evenly over one CTA per SM in (tile, step) order
// ("stream-K"); every CTA writes its partial sum of each tile it touched to
// its own slot (slot = CTA + tile, unique along the split), and
// k_bwd_small_end sums the slots of a tile in CTA order (deterministic) when
// it forms dX.
//
// Warp roles (768 threads, one CTA per SM):
//   warp 0      TMA producer of the dY tiles (NT x 128 bf16, two
//               128-byte-swizzled boxes of 64 columns);
//   warp 1      TMEM allocator and MMA issuer of decoder group 0's units, warp 3
//               the issuer of group 1's units: 8 MMAs of 128 x NT x 16 per unit,
//               each issuer into its own accumulator (two issuers double the
//               rate: issuing one such MMA costs the issuing thread ~77 cycles);
//   warp 2      TMA producer of the packed NF4 tiles (128 rows x 64 B, 64-byte
//               swizzle), 8 units ahead;
//   warps 4-7   epilogue: TMEM -> registers -> partial slot;
//   warps 8-23  dequantizers, two groups of 8 warps taking alternate units (16
//               warps keep the integer pipe busy while others wait): thread d
//               of a group owns one 64-weight row-block per unit (row
//               8 (d / 16) + d % 8, block (d / 8) % 2), exact bf16_rne(L[q] c')
//               from the per-block register table, written into the swizzled
//               MN-major A-operand layout.
#pragma once
#include "tc_gemm.cuh"

namespace qnf4 {
namespace tcs {

// L2 cache policies.  The block constants of a row are 2 bytes per column tile
// in 32-byte sectors shared by 16 tiles, which different CTAs reach at
// different times: kept in L2 (evict_last) they are read from DRAM once,
// instead of once per tile after the streamed weight has pushed them out.
// The packed weight itself is read once (evict_first).
__device__ __forceinline__ uint64_t l2_policy_evict_last() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}
__device__ __forceinline__ uint64_t l2_policy_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}
__device__ __forceinline__ int ldg_s8_keep(const int8_t* ptr, uint64_t pol) {
    int v;
    asm volatile("ld.global.nc.L2::cache_hint.s8 %0, [%1], %2;" : "=r"(v) : "l"(ptr), "l"(pol));
    return v;
}
__device__ __forceinline__ float ldg_f32_keep(const float* ptr, uint64_t pol) {
    float v;
    asm volatile("ld.global.nc.L2::cache_hint.f32 %0, [%1], %2;" : "=f"(v) : "l"(ptr), "l"(pol));
    return v;
}
__device__ __forceinline__ void tma_load_2d_hint(uint32_t dst, const CUtensorMap* map, uint32_t bar, int x, int y,
                                                 uint64_t pol) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%2, %3}], [%4], %5;"
        ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar), "l"(pol)
        : "memory");
}

constexpr int TR = 128;                    // output rows of a tile (MMA M)
constexpr int KSTEP = 128;                 // reduction per step
constexpr int SX = 3;                      // activation ring stages
constexpr int SW = 4;                      // dequantized weight ring stages (2 per decoder group)
constexpr int SP = 8;                      // packed weight ring stages (4 per decoder group)
constexpr int X_BYTES_MAX = 32 * KSTEP * 2;        // 8192 (NT = 32)
constexpr int W_BYTES = TR * KSTEP * 2;            // 32768
constexpr int P_BYTES = TR * KSTEP / 2;            // 8192
constexpr int kThreads = 768;
constexpr int kGroupThreads = 256;         // one decoder group
constexpr int kEpiThreads = 128;

constexpr int OFF_X = 0;
constexpr int OFF_W = OFF_X + SX * X_BYTES_MAX;
constexpr int OFF_P = OFF_W + SW * W_BYTES;
constexpr int OFF_BAR = OFF_P + SP * P_BYTES;
// fullX[SX] emptyX[SX] fullW[SW] emptyW[SW] fullP[SP] emptyP[SP] tfull[2] tempty[2] drain
constexpr int NBAR = 2 * SX + 2 * SW + 2 * SP + 4 + 1;
constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
constexpr int SMEM_BYTES = OFF_MISC + 16;
constexpr int SMEM_ALLOC = SMEM_BYTES + 1024;

struct Args {
    const int8_t* codes;
    const float* scale;
    const float* mean;
    int64_t M, N, K;           // W is [N, K]; the output has K columns, the reduction N rows
    int tiles, nks;            // ceil(K / 128), ceil(N / 128)
    int64_t units;             // tiles * nks
    int ctas;                  // grid size
    float* slots;              // [ctas + tiles][NT][128] fp32 partial tiles
};

// First unit of CTA c, and the CTA that owns unit u, for an even split of U units over C CTAs.
__host__ __device__ __forceinline__ int64_t unit_begin(int64_t c, int64_t U, int64_t C) { return c * U / C; }

// Instruction descriptor: kind::f16, A = B = bf16, D = f32, M = 128, N = NT, A K- or MN-major.
__host__ __device__ constexpr uint32_t make_idesc(bool a_mn_major, int nt) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn_major ? 1u : 0u) << 15) | ((uint32_t)(nt >> 3) << 17) |
           ((uint32_t)(TR >> 4) << 24);
}

#define TCS_LD16(taddr, r)                                                                                         \
    asm volatile(                                                                                                  \
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"   \
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),        \
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])   \
        : "r"(taddr))

// Row-block of dequantizer thread d in a step: row 0..127 of the step and block 0..1.
// A quarter-warp holds 8 consecutive rows of one block, so its packed reads
// (64-byte swizzle) and its stores into the operand tile are conflict-free.
__device__ __forceinline__ int deq_row(int d) { return 8 * (d >> 4) + (d & 7); }
__device__ __forceinline__ int deq_blk(int d) { return (d >> 3) & 1; }

// Byte offset of 16-byte chunk ch (8 weights) of thread d's row-block in the
// MN-major operand tile (the tile's 128 rows are the reduction, its 2 x 64
// columns the MMA's M): atom column j 16 KB apart, 8-row group n / 8 1 KB
// apart, row n % 8, chunk ch ^ (n % 8).
__device__ __forceinline__ uint32_t w_chunk_offset(int d, int ch) {
    const int n = deq_row(d), j = deq_blk(d);
    return (uint32_t)(j * 16384 + (n >> 3) * 1024 + (n & 7) * 128 + ((ch ^ (n & 7)) << 4));
}

// Packed tile: 128 rows x 64 B (two blocks), 64-byte swizzle (chunk ^= (row / 2) % 4).
__device__ __forceinline__ uint32_t p_chunk_offset(int d, int c) {
    const int n = deq_row(d), j = deq_blk(d);
    return (uint32_t)(n * 64 + (((2 * j + c) ^ ((n >> 1) & 3)) << 4));
}

// Advance a (tile, step) position by n units.
__device__ __forceinline__ void unit_advance(int& tile, int& ks, int n, int nks) {
    ks += n;
    while (ks >= nks) { ks -= nks; ++tile; }
}

// ----------------------------------------------------------------------------
template <int NT>
__global__ void __launch_bounds__(kThreads, 1)
k_tcs_gemm(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmP, Args a,
           NF4Tables tab) {
    constexpr int X_BYTES = NT * KSTEP * 2;
    constexpr uint32_t kCols = NT == 16 ? 64 : 128;     // 2 buffers x 2 issuers x NT columns
    extern __shared__ __align__(1024) uint8_t smem[];
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem) + 1023) & ~(uintptr_t)1023);
    const uint32_t sbase = smem_u32(base);
    const uint32_t bar0 = sbase + OFF_BAR;
    auto fullX = [&](int i) { return bar0 + 8 * i; };
    auto emptyX = [&](int i) { return bar0 + 8 * (SX + i); };
    auto fullW = [&](int i) { return bar0 + 8 * (2 * SX + i); };
    auto emptyW = [&](int i) { return bar0 + 8 * (2 * SX + SW + i); };
    auto fullP = [&](int i) { return bar0 + 8 * (2 * SX + 2 * SW + i); };
    auto emptyP = [&](int i) { return bar0 + 8 * (2 * SX + 2 * SW + SP + i); };
    auto tfull = [&](int i) { return bar0 + 8 * (2 * SX + 2 * SW + 2 * SP + i); };
    auto tempty = [&](int i) { return bar0 + 8 * (2 * SX + 2 * SW + 2 * SP + 2 + i); };
    const uint32_t drain = bar0 + 8 * (2 * SX + 2 * SW + 2 * SP + 4);
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(base + OFF_MISC);
    volatile int* s_abort = reinterpret_cast<volatile int*>(base + OFF_MISC + 4);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t U = a.units;
    // this CTA's units [u0, u1) (fewer than 2^31: the weight has fewer than 2^38
    // elements); unit i of the CTA is u0 + i, and loops walk (tile, step) incrementally
    const int u0 = (int)unit_begin(blockIdx.x, U, a.ctas), u1 = (int)unit_begin(blockIdx.x + 1, U, a.ctas);
    const int nu = u1 - u0;
    const int nks = a.nks;
    const int tile0 = u0 / nks, ks0 = u0 - tile0 * nks;
    const int64_t nblk = a.K / kBlock;

    if (tid == 0) {
        for (int i = 0; i < SX; ++i) { tc::mbar_init(fullX(i), 1); tc::mbar_init(emptyX(i), 1); }
        for (int i = 0; i < SW; ++i) { tc::mbar_init(fullW(i), kGroupThreads / 32); tc::mbar_init(emptyW(i), 1); }
        for (int i = 0; i < SP; ++i) { tc::mbar_init(fullP(i), 1); tc::mbar_init(emptyP(i), kGroupThreads / 32); }
        // tfull: one commit from each MMA issuer per segment; drain: one from each at the end
        for (int i = 0; i < 2; ++i) { tc::mbar_init(tfull(i), 2); tc::mbar_init(tempty(i), kEpiThreads / 32); }
        tc::mbar_init(drain, 2);
        *s_abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(s_tmem)),
                     "r"(kCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
        tc::tc_fence_before();
    }
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem_base = *s_tmem;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer: activations
        if (lane == 0) {
            int sx = 0, px = 0, issued = 0;
            bool ok = true;
            for (int i = 0, ks = ks0; i < nu && ok; ++i, ks = (ks + 1 == nks) ? 0 : ks + 1) {
                if (!(ok = tc::mbar_wait(emptyX(sx), px ^ 1, s_abort))) break;
                tc::mbar_expect_tx(fullX(sx), X_BYTES);
                const uint32_t dst = sbase + OFF_X + sx * X_BYTES_MAX;
                tc::tma_load_2d(dst, &tmX, fullX(sx), ks * KSTEP, 0);
                tc::tma_load_2d(dst + NT * 128, &tmX, fullX(sx), ks * KSTEP + 64, 0);
                ++issued;
                if (++sx == SX) { sx = 0; px ^= 1; }
            }
            if (!ok)
                for (int k = 1; k <= SX && k <= issued; ++k)
                    tc::mbar_drain(fullX((issued - k) % SX), ((issued - k) / SX) & 1);
        }
    } else if (warp == 2) {
        // ------------------------------------------------------------ TMA producer: packed weights
        if (lane == 0) {
            int issued = 0, tile = tile0, ks = ks0;
            bool ok = true;
            const uint64_t stream_pol = l2_policy_evict_first();
            for (int i = 0; i < nu && ok; ++i) {
                const int sp = i & (SP - 1), pp = (i / SP) & 1;
                if (!(ok = tc::mbar_wait(emptyP(sp), pp ^ 1, s_abort))) break;
                tc::mbar_expect_tx(fullP(sp), P_BYTES);
                const uint32_t dst = sbase + OFF_P + sp * P_BYTES;
                tma_load_2d_hint(dst, &tmP, fullP(sp), tile * (TR / 2), ks * KSTEP, stream_pol);
                ++issued;
                unit_advance(tile, ks, 1, nks);
            }
            if (!ok)
                for (int k = 1; k <= SP && k <= issued; ++k)
                    tc::mbar_drain(fullP((issued - k) & (SP - 1)), ((issued - k) / SP) & 1);
        }
    } else if (warp == 1 || warp == 3) {
        // ------------------------------------------------------------ MMA issuers
        // Issuer iss = 0 (warp 1) takes the units of decoder group 0 (even i), issuer 1
        // (warp 3) those of group 1, each into its own accumulator (buffer buf, columns
        // (2 buf + iss) NT): one thread issuing a 128 x NT x 16 MMA spends ~77 cycles on it,
        // so two issuers double the rate.  Both walk every unit so that they agree on the
        // segments (a segment = this CTA's units of one tile): each waits for the
        // segment's buffer to be free and commits the segment's "full" barrier once (the
        // epilogue waits for both commits and adds the accumulators of the issuers that
        // had units in the segment).
        const int iss = warp == 1 ? 0 : 1;
        if (lane == 0) {
            constexpr uint32_t idesc = make_idesc(true, NT);
            int seg = 0, buf = 0;
            bool ok = true, started = false;
            uint32_t d_tmem = tmem_base;
            for (int i = 0, ks = ks0; i < nu && ok; ++i, ks = (ks + 1 == nks) ? 0 : ks + 1) {
                const bool first = (i == 0) || ks == 0;
                const bool last = (i == nu - 1) || ks == nks - 1;
                if (first) {
                    buf = seg & 1;
                    if (!(ok = tc::mbar_wait(tempty(buf), ((seg >> 1) & 1) ^ 1, s_abort))) break;
                    tc::tc_fence_after();
                    d_tmem = tmem_base + (uint32_t)((2 * buf + iss) * NT);
                    started = false;
                }
                if ((i & 1) == iss) {
                    const int sx = i % SX, px = (i / SX) & 1;
                    const int sw = i & (SW - 1), pw = (i / SW) & 1;
                    if (!(ok = tc::mbar_wait(fullX(sx), px, s_abort))) break;
                    if (!(ok = tc::mbar_wait(fullW(sw), pw, s_abort))) break;
                    tc::tc_fence_after();
                    const uint32_t x_addr = sbase + OFF_X + sx * X_BYTES_MAX;
                    const uint32_t w_addr = sbase + OFF_W + sw * W_BYTES;
                    // the 16 descriptors of a unit differ only in their start-address field
                    // (address / 16, 14 bits; every offset keeps it below 2^14): each is the
                    // stage's base descriptor plus a constant
                    const uint64_t a0 = tc::smem_desc_sw128(w_addr, 16384, 1024);
                    const uint64_t b0 = tc::smem_desc_sw128(x_addr, 16, 1024);
#pragma unroll
                    for (int q = 0; q < KSTEP / 16; ++q) {
                        const int h = q >> 2, kk = q & 3;
                        const uint64_t adesc = a0 + (uint64_t)((q * 2048) >> 4);
                        const uint64_t bdesc = b0 + (uint64_t)((h * (NT * 128) + kk * 32) >> 4);
                        tc::tc_mma(d_tmem, adesc, bdesc, idesc, (started || q > 0) ? 1u : 0u);
                    }
                    started = true;
                    tc::tc_commit(emptyX(sx));
                    tc::tc_commit(emptyW(sw));
                }
                if (last) {
                    tc::tc_commit(tfull(buf));
                    ++seg;
                }
            }
            tc::tc_commit(drain);
            tc::mbar_drain(drain, 0);
        }
    } else if (warp >= 8) {
        // ------------------------------------------------------------ dequantizers
        const int grp = (warp - 8) >> 3;                 // group: units i = grp, grp + 2, ...
        const int d = tid - 256 - kGroupThreads * grp;   // thread within the group
        const int drow = deq_row(d), dblk = deq_blk(d);
        bool ok = true;
        // fetch position: the unit whose block-constant inputs are loaded next
        int fi = grp, ft = tile0, fk = ks0;
        unit_advance(ft, fk, grp, nks);
        const uint64_t keep_pol = l2_policy_evict_last();
        auto fetch = [&](int& code, float& sc, float& mu) {
            code = 0; sc = 0.f; mu = 0.f;
            const int tile = ft, ks = fk;
            const bool in = fi < nu;
            fi += 2;
            unit_advance(ft, fk, 2, nks);
            if (!in) return;
            const int64_t n = (int64_t)ks * KSTEP + drow, kb = (int64_t)tile * 2 + dblk;
            if (n < a.N && kb < nblk) {
                const int64_t b = n * nblk + kb;
                code = ldg_s8_keep(a.codes + b, keep_pol);
                sc = ldg_f32_keep(a.scale + (b >> 8), keep_pol);
                mu = ldg_f32_keep(a.mean + (b >> 8), keep_pol);
            }
        };
        // unit i of this group; (code, sc, mu) hold its block-constant inputs and are
        // refilled with those of unit i + 4 (two register slots alternate)
        auto do_unit = [&](int i, int& code, float& sc, float& mu) {
            const float c = __fmaf_rn((float)code, sc, mu);
            fetch(code, sc, mu);
            const int sp = i & (SP - 1), pp = (i / SP) & 1;
            if (!(ok = tc::mbar_wait(fullP(sp), pp, s_abort))) return;
            uint4 p0, p1;
            const uint32_t pst = sbase + OFF_P + sp * P_BYTES;
            const uint32_t src0 = pst + p_chunk_offset(d, 0), src1 = pst + p_chunk_offset(d, 1);
            asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(p0.x), "=r"(p0.y), "=r"(p0.z), "=r"(p0.w) : "r"(src0));
            asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(p1.x), "=r"(p1.y), "=r"(p1.z), "=r"(p1.w) : "r"(src1));
            const BlockTable tb = make_block_table(tab, c);
            const uint32_t pwd[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
            const int sw = i & (SW - 1), pw = (i / SW) & 1;
            if (!(ok = tc::mbar_wait(emptyW(sw), pw ^ 1, s_abort))) return;
            const uint32_t wbase = sbase + OFF_W + sw * W_BYTES;
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) {
                uint32_t o[4];
                decode8(tb, pwd[ch], o);
                tc::st_shared_v4(wbase + w_chunk_offset(d, ch), o[0], o[1], o[2], o[3]);
            }
            tc::fence_proxy_async();
            __syncwarp();
            // the packed stage is released only after the stores above, which consume the
            // values decoded from it (a release right after the shared loads were issued let
            // the next TMA copy overwrite the stage under loads still in flight)
            if (lane == 0) {
                tc::mbar_arrive(fullW(sw));
                tc::mbar_arrive(emptyP(sp));
            }
        };
        int codeA, codeB;
        float scA, scB, muA, muB;
        fetch(codeA, scA, muA);
        fetch(codeB, scB, muB);
        for (int i = grp; i < nu && ok; i += 4) {
            do_unit(i, codeA, scA, muA);
            if (ok && i + 2 < nu) do_unit(i + 2, codeB, scB, muB);
        }
    } else if (warp >= 4) {
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3;                 // TMEM lane quarter of this warp
        const int row = q * 32 + lane;
        bool ok = true;
        int seg = 0;
        for (int u = u0, tile = tile0; u < u1 && ok; ++tile) {
            const int tile_u1 = (tile + 1) * nks;
            const int seg_u0 = u;
            u = tile_u1 < u1 ? tile_u1 : u1;
            const int buf = seg & 1;
            if (!(ok = tc::mbar_wait(tfull(buf), (seg >> 1) & 1, s_abort))) break;
            ++seg;
            tc::tc_fence_after();
            // the segment's units are CTA-local indices [seg_i0, seg_i1): issuer 0 took the even
            // ones, issuer 1 the odd ones; the sum is issuer 0's accumulator plus issuer 1's
            const int seg_i1 = u - u0, seg_i0 = (seg_u0 - u0);
            const bool has0 = seg_i1 - seg_i0 >= 2 || (seg_i0 & 1) == 0;
            const bool has1 = seg_i1 - seg_i0 >= 2 || (seg_i0 & 1) == 1;
            float acc[NT];
#pragma unroll
            for (int m = 0; m < NT; ++m) acc[m] = 0.f;
#pragma unroll
            for (int is = 0; is < 2; ++is) {
                if (is == 0 ? !has0 : !has1) continue;
                uint32_t rr[16];
                const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)((2 * buf + is) * NT);
#pragma unroll
                for (int h = 0; h < NT / 16; ++h) {
                    TCS_LD16(taddr + h * 16, rr);
                    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
                    for (int j = 0; j < 16; ++j) acc[h * 16 + j] += __uint_as_float(rr[j]);
                }
            }
            tc::tc_fence_before();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(tempty(buf));
            float* sp = a.slots + ((int64_t)blockIdx.x + tile) * (NT * TR);
#pragma unroll
            for (int m = 0; m < NT; ++m) sp[m * TR + row] = acc[m];
        }
    }

    __syncthreads();
    if (warp == 1) {
        tc::tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(kCols));
    }
    // launched programmatically after the U / dB kernel, which it does not read: it
    // only may not complete before that kernel has (k_bwd_small_end reads both)
    if (tid == 0) grid_dep_wait();
}

}  // namespace tcs
}  // namespace qnf4
