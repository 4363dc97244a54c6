// tc2_gemm.cuh -- the fused NF4 dequant + GEMM on a pair of SMs
// (tcgen05.mma.cta_group::2), for M > 128 tokens.
//
// Same computation as tc_gemm.cuh (forward Y = X W'^T + s T B^T, backward
// dX = dY W' + s U A), but a cluster of two CTAs computes one 256-token x
// 256-output tile with 256 x 256 x 16 MMAs issued by two threads of the leader
// CTA (rank 0; one thread's issue cost is about one MMA's tensor time):
//   - each CTA holds its 128 tokens of the activation tile (A operand) and
//     its 128 output features of the weight tile (B operand) in its own
//     shared memory, at the same offsets;
//   - each CTA's TMEM holds the accumulator rows of its own 128 tokens;
//   - each CTA dequantizes only its half of W' per reduction step, so the
//     decode work per MMA flop is half that of the single-SM kernel, which is
//     what bounds the single-SM kernel (its ALU pipe runs ~60% busy at ~32%
//     tensor activity).
// Synchronisation across the pair:
//   - activation tiles of both CTAs are loaded with cta_group::2 TMA whose
//     transaction bytes complete on the leader's barrier (the leader arms it
//     for both halves);
//   - the dequantizers and the epilogue of both CTAs arrive on the leader's
//     barriers: the peer's with release at cluster scope (mapa), the leader's
//     own at CTA scope; the leader's waits acquire at cluster scope;
//   - MMA completion is multicast to the "empty" and "accumulator full"
//     barriers of both CTAs (tcgen05.commit ... multicast::cluster, mask 0b11).
// No TMA load uses multicast.  All waits are bounded as in tc_gemm.cuh; a
// cluster barrier before TMEM is freed keeps either CTA from leaving while
// the other may still touch its shared memory.
#pragma once
#include <cuda.h>
#include "common.cuh"
#include "nf4_decode.cuh"
#include "tc_gemm.cuh"

namespace qnf4 {
namespace tc2 {

using tc::Args;

constexpr int BM = 256, BN = 256, BK = 64;       // pair tile
constexpr int HM = 128, HN = 128;                // per-CTA halves
constexpr int A_BYTES = HM * BK * 2;             // 16 KB
constexpr int W_BYTES = HN * BK * 2;             // 16 KB
constexpr int P_BYTES = HN * BK / 2;             // 4 KB
constexpr int kThreads = 512;
constexpr int kGroupThreads = 128;               // dequantizers per step (one group of two)
constexpr int kGroupWarps = kGroupThreads / 32;
constexpr int kEpiWarps = 4;
constexpr int kTmemCols = 512;

// Shared-memory layout for MT token tiles of 256 per pair tile.  Two threads of
// the leader issue the MMAs (one thread spends ~77 cycles issuing one, about as
// long as a 256 x 256 x 16 MMA takes the pair's tensor cores to run, so one
// thread cannot keep them busy).  MT = 2: each decoded W' stage feeds the MMAs of
// two token tiles, one per issuer (two accumulators, all of TMEM), which halves
// the decode work per flop.  MT = 1: issuer g takes the steps of parity g into its
// own accumulator (all of TMEM again) and the epilogue adds the two.  Either way
// the epilogue drains TMEM before the next tile starts.
//   SA: activation slots (one token tile's 128 x 64 half each; a step takes MT);
//   MT = 1 splits them into one sub-ring per step parity, so that each stage is
//   only ever waited on by the issuer of that parity
//   SW / SP: W' and packed stages, split into one sub-ring per dequantizer
//   group (SW / 2 and SP / 2 stages), each filled and drained in that group's
//   step order, so every waiter is at most one phase ahead of the barrier it
//   waits on (a parity wait cannot tell phase k from phase k - 2).
template <int MT>
struct Lay {
    static constexpr int SA = MT == 1 ? 4 : 6, SW = 6, SP = MT == 1 ? 8 : 4;
    static constexpr int SWH = SW / 2, SPH = SP / 2;
    static constexpr int SAS = SA / MT;          // activation stages (MT slots each)
    static constexpr int SAH = SA / 2;           // MT = 1: stages per step-parity sub-ring
    static constexpr int NACC = 1;               // accumulator sets (TMEM holds 2 x 256 columns)
    static constexpr int OFF_A = 0;
    static constexpr int OFF_W = OFF_A + SA * A_BYTES;
    static constexpr int OFF_P = OFF_W + SW * W_BYTES;
    static constexpr int OFF_BAR = OFF_P + SP * P_BYTES;
    static constexpr int NBAR = 2 * SA + 2 * SW + 2 * SP + 4 + 1 + SW;   // + peer-local fullWl[SW]
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
    // per dequantizer thread, 2 slots x (code word, scale, mean) of prefetched block-constant inputs
    static constexpr int OFF_C = OFF_MISC + 16;
    static constexpr int SMEM_BYTES = OFF_C + 2 * 3 * 2 * kGroupThreads * 4;
    static constexpr int SMEM_ALLOC = SMEM_BYTES + 1024;
};
static_assert(Lay<1>::SMEM_ALLOC <= 232448 && Lay<2>::SMEM_ALLOC <= 232448, "shared memory");

// Stream-K partial tiles: per (pair, CTA rank) MT x 8 chunks of 32 columns, each as
// 8 pieces of 4 columns x 128 rows x 16 bytes (row-fastest), so that a warp's 32 rows
// of one piece are 512 contiguous bytes for the contributor's stores and the owner's
// copies.  The owner streams them through kFixD 4 KB buffers per epilogue warp in the
// activation and weight rings, idle by then (the span that adds partials is always
// the pair's last).
constexpr int kFixD = 8;
static_assert((BN / 32) % 2 == 0, "epilogue chunk pairs");
static_assert(4 * kFixD * 4096 <= Lay<1>::OFF_P && 4 * kFixD * 4096 <= Lay<2>::OFF_P, "fix-up staging");
__host__ __device__ constexpr int64_t part_off(int64_t slot, int nchunks, int ucc, int j, int row) {
    return (((slot * nchunks + ucc) * 8 + j) * 128 + row) * 4;
}

__device__ __forceinline__ bool mbar_try_cl(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok) : "r"(bar), "r"(parity) : "memory");
    return ok != 0;
}

// bounded wait, cluster-scope acquire
__device__ __forceinline__ bool mbar_wait_cl(uint32_t bar, uint32_t parity, volatile int* abort_flag) {
    if (mbar_try_cl(bar, parity)) return true;
    const uint64_t t0 = tc::globaltimer();
    while (true) {
        if (mbar_try_cl(bar, parity)) return true;
        if (*abort_flag) return false;
        if (tc::globaltimer() - t0 > tc::kWaitTimeoutNs) {
            *abort_flag = 1;
            report_timeout();
            return false;
        }
    }
}

__device__ __forceinline__ void mbar_drain_cl(uint32_t bar, uint32_t parity) {
    const uint64_t t0 = tc::globaltimer();
    while (!mbar_try_cl(bar, parity)) {
        if (tc::globaltimer() - t0 > tc::kWaitTimeoutNs) { report_timeout(); return; }
    }
}

// arrive on a barrier given by its shared::cluster address (own CTA or the peer)
__device__ __forceinline__ void mbar_arrive_cl(uint32_t cl_addr) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cl_addr) : "memory");
}

__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap* map, uint32_t cl_bar, int x, int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
        ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(cl_bar)
        : "memory");
}

__device__ __forceinline__ void tc2_commit_both(uint32_t bar) {
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;"
        ::"r"(bar), "h"((unsigned short)0x3) : "memory");
}

__device__ __forceinline__ void tc2_commit_local(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void tc2_mma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                        uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

__host__ __device__ constexpr uint32_t make_idesc2(bool b_mn_major) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((b_mn_major ? 1u : 0u) << 16) | ((uint32_t)(BN >> 3) << 17) |
           ((uint32_t)(BM >> 4) << 24);
}

// Row-block of dequantizer thread t (0..127 within its group) in one step:
//   forward : row t of this CTA's 128 W rows, the step's k-block;
//   backward: reduction row n = 16 (t / 32) + 8 ((t / 16) % 2) + t % 8 of the
//             step's 64 W rows, output block j = (t / 8) % 2 of this CTA's
//             128 columns (8 distinct n % 8 per quarter-warp, one j).
template <bool BWD>
__device__ __forceinline__ int deq_row(int t) {
    return BWD ? 16 * (t >> 5) + 8 * ((t >> 4) & 1) + (t & 7) : t;
}
template <bool BWD>
__device__ __forceinline__ int deq_blk(int t) { return BWD ? (t >> 3) & 1 : 0; }

template <bool BWD>
__device__ __forceinline__ uint32_t w_chunk_offset(int t, int ch) {
    if (!BWD) return (uint32_t)(t * 128 + ((ch ^ (t & 7)) << 4));
    const int n = deq_row<true>(t), j = deq_blk<true>(t);
    return (uint32_t)(j * 8192 + (n >> 3) * 1024 + (n & 7) * 128 + ((ch ^ (n & 7)) << 4));
}

// packed tile: forward 128 rows x 32 B (32-byte swizzle), backward 64 rows x
// 64 B (64-byte swizzle: chunk ^= (address / 128) % 4 = (row / 2) % 4)
template <bool BWD>
__device__ __forceinline__ uint32_t p_chunk_offset(int t, int c) {
    if (!BWD) return (uint32_t)(t * 32 + ((c ^ ((t >> 2) & 1)) << 4));
    const int n = deq_row<true>(t), j = deq_blk<true>(t);
    return (uint32_t)(n * 64 + (((2 * j + c) ^ ((n >> 1) & 3)) << 4));
}

// The spans (tile, reduction steps [s0, s1)) a pair takes, in the order it takes them.
// Round-robin: whole tiles pair, pair + npairs, ...  Stream-K: the pair's run
// [u0, u1) of the ntiles x nsteps units (tile-major), walked from its END back, so
// its first span is the head of a tile that a later pair finishes and its last span
// the tail of a tile it finishes itself.  The pair that takes a tile's last step owns
// the tile: it adds the partial sums of the lower pairs that took the tile's head,
// which they computed first, so an owner waits only for lower pairs, and for little.
struct Spans {
    int64_t u0, u, nsteps, next_tile, ntiles, npairs;
    bool sk;
    __host__ __device__ Spans(bool sk_, int64_t pair, int64_t npairs_, int64_t ntiles_, int nsteps_)
        : nsteps(nsteps_), next_tile(pair), ntiles(ntiles_), npairs(npairs_), sk(sk_) {
        const int64_t U = ntiles_ * nsteps_;
        u0 = pair * U / npairs_;
        u = (pair + 1) * U / npairs_;
    }
    __host__ __device__ bool next(int64_t& tile, int& s0, int& s1) {
        if (!sk) {
            if (next_tile >= ntiles) return false;
            tile = next_tile;
            s0 = 0;
            s1 = (int)nsteps;
            next_tile += npairs;
            return true;
        }
        if (u <= u0) return false;
        tile = (u - 1) / nsteps;
        const int64_t tb = tile * nsteps;
        s1 = (int)(u - tb);
        s0 = (int)((u0 > tb ? u0 : tb) - tb);
        u = tb + s0;
        return true;
    }
};

// Steps s in [a, b) with s % 2 == g (a <= b).
__device__ __forceinline__ int count_par(int a, int b, int g) { return ((b + 1 - g) >> 1) - ((a + 1 - g) >> 1); }

__device__ __forceinline__ int ld_acquire_gpu(const int* p) {
    int v;
    asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

template <bool BWD, int MT>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
k_tc2_gemm(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmL,
           const __grid_constant__ CUtensorMap tmP, Args a, NF4Tables tab) {
    using L = Lay<MT>;
    constexpr int SA = L::SA, SW = L::SW, SP = L::SP, SWH = L::SWH, SPH = L::SPH, NACC = L::NACC, SAS = L::SAS;
    constexpr int SAH = L::SAH;
    static_assert(SA % MT == 0 && SA % 2 == 0, "activation stages");
    // MMA-issuing threads of the leader: warp 1 (issuer 0) and warp 15 (issuer 1).  Each
    // commits its own MMAs.  MT = 2: both read every stage, so the stage releases count
    // two arrivals; MT = 1: a stage is read by one issuer (NREL = 1).  Accumulator full
    // and the final drain count one arrival per issuer.
    constexpr int NISS = 2, NREL = MT;
    constexpr int OFF_A = L::OFF_A, OFF_W = L::OFF_W, OFF_P = L::OFF_P, OFF_BAR = L::OFF_BAR;
    constexpr int OFF_MISC = L::OFF_MISC, OFF_C = L::OFF_C;
    extern __shared__ __align__(1024) uint8_t smem[];
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem) + 1023) & ~(uintptr_t)1023);
    const uint32_t sbase = smem_u32(base);
    const uint32_t bar0 = sbase + OFF_BAR;
    auto fullA = [&](int i) { return bar0 + 8 * i; };
    auto emptyA = [&](int i) { return bar0 + 8 * (SA + i); };
    auto fullW = [&](int i) { return bar0 + 8 * (2 * SA + i); };
    auto emptyW = [&](int i) { return bar0 + 8 * (2 * SA + SW + i); };
    auto fullP = [&](int i) { return bar0 + 8 * (2 * SA + 2 * SW + i); };
    auto emptyP = [&](int i) { return bar0 + 8 * (2 * SA + 2 * SW + SP + i); };
    auto tfull = [&](int i) { return bar0 + 8 * (2 * SA + 2 * SW + 2 * SP + i); };
    auto tempty = [&](int i) { return bar0 + 8 * (2 * SA + 2 * SW + 2 * SP + 2 + i); };
    const uint32_t drain = bar0 + 8 * (2 * SA + 2 * SW + 2 * SP + 4);
    auto fullWl = [&](int i) { return bar0 + 8 * (2 * SA + 2 * SW + 2 * SP + 5 + i); };
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(base + OFF_MISC);
    volatile int* s_abort = reinterpret_cast<volatile int*>(base + OFF_MISC + 4);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // Programmatic launch.  This kernel is launched behind the T or U product,
    // which lets it start once everything before that product has completed: the
    // activations, the weight and the LoRA weights of the caller are ready, the
    // product's own outputs (the scaled LoRA activation, the padded LoRA weight,
    // the zeroed stream-K counters) are not, and every role waits before its
    // first use of them.  The kernels behind this one (dB and dA, which read U
    // and nothing this kernel writes) start once every CTA has let them: the
    // peer CTA at once, the leader's first epilogue warp (idle until its first
    // accumulator is full) after waiting for the product.
    if (cluster_rank() != 0 && tid == 0) grid_dep_launch();
    const uint32_t crank = cluster_rank();
    const bool leader = crank == 0;
    const int64_t pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
    const int64_t mtiles = cdiv(a.M, (int64_t)BM * MT), ntiles_n = cdiv(a.n_out, BN);   // token groups
    const int64_t ntiles = mtiles * ntiles_n;
    const int nks = (int)cdiv(a.n_red, BK);
    const int nsteps = nks + a.nlora;
    const int64_t nblk = a.K / kBlock;

    if (tid == 0) {
        for (int i = 0; i < SA; ++i) { tc::mbar_init(fullA(i), 1); tc::mbar_init(emptyA(i), NREL); }
        // leader: its own group's warps + one forwarded arrival from the peer; peer: its group's warps
        for (int i = 0; i < SW; ++i) {
            tc::mbar_init(fullW(i), kGroupWarps + 1);
            tc::mbar_init(emptyW(i), NREL);
            tc::mbar_init(fullWl(i), kGroupWarps);
        }
        for (int i = 0; i < SP; ++i) { tc::mbar_init(fullP(i), 1); tc::mbar_init(emptyP(i), kGroupWarps); }
        for (int i = 0; i < 2; ++i) { tc::mbar_init(tfull(i), NISS); tc::mbar_init(tempty(i), 2 * kEpiWarps); }
        tc::mbar_init(drain, NISS);
        *s_abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    cluster_sync();                      // the leader's barriers exist before anyone signals them
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(s_tmem)),
                     "r"(kTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;");
        tc::tc_fence_before();
    }
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem_base = *s_tmem;

    // Ring position of the j-th step (counted over this CTA's spans so far) of
    // dequantizer group g = step % 2: the group uses stages g * half .. g * half +
    // half - 1 in its own step order.
    auto wpos = [&](int j, int g, int& st, int& ph) {
        st = g * SWH + j % SWH;
        ph = (j / SWH) & 1;
    };
    auto ppos = [&](int j, int g, int& st, int& ph) {
        st = g * SPH + j % SPH;
        ph = (j / SPH) & 1;
    };
    // Activation stage of a step: MT = 2, one ring in step order (jall = this CTA's steps
    // so far); MT = 1, the sub-ring of the step's parity g (jg = its steps of parity g).
    auto apos = [&](int jall, int jg, int g, int& st, int& ph) {
        if (MT == 2) {
            st = jall % SAS;
            ph = (jall / SAS) & 1;
        } else {
            st = g * SAH + jg % SAH;
            ph = (jg / SAH) & 1;
        }
    };
    const bool skm = a.sk != 0;

    // Peer CTA: pass the completion of each stage of the dequantized-weight ring on to
    // the leader's barrier, for the steps of dequantizer group grp: one cluster-scope
    // fence and one relaxed remote arrive per stage.
    auto forward = [&](int grp) {
        bool ok = true;
        int jw = 0;
        Spans spn(skm, pair, npairs, ntiles, nsteps);
        int64_t tile;
        int s0, s1;
        while (ok && spn.next(tile, s0, s1)) {
            for (int step = s0 + ((s0 & 1) != grp ? 1 : 0), k = 0; step < s1 && ok; step += 2, ++k) {
                int sw, pw;
                wpos(jw + k, grp, sw, pw);
                if (!(ok = tc::mbar_wait(fullWl(sw), pw, s_abort))) break;
                asm volatile("fence.acq_rel.cluster;" ::: "memory");
                asm volatile("mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [%0];" ::"r"(mapa(fullW(sw), 0))
                             : "memory");
            }
            jw += count_par(s0, s1, grp);
        }
    };

    // MMA issuer iss (leader only).  MT = 2: token tile u = iss of every step into its
    // accumulator columns; both issuers wait on the same stage barriers (a wait does not
    // consume a phase).  MT = 1: the steps of parity iss into accumulator iss.
    auto issue = [&](const int iss) {
        constexpr uint32_t idesc = make_idesc2(BWD);
        constexpr int sstep = MT == 2 ? 1 : 2;
        const int u = MT == 2 ? iss : 0;
        bool ok = true;
        int it = 0, jw0 = 0, jw1 = 0, ja = 0;
        Spans spn(skm, pair, npairs, ntiles, nsteps);
        int64_t tile;
        int s0, s1;
        while (ok && spn.next(tile, s0, s1)) {
            const int acc = it % NACC, aph = (it / NACC) & 1;
            if (!(ok = mbar_wait_cl(tempty(acc), aph ^ 1, s_abort))) break;
            tc::tc_fence_after();
            const uint32_t d_tmem = tmem_base + (uint32_t)(iss * BN);
            const int first = (MT == 1 && (s0 & 1) != iss) ? s0 + 1 : s0;
            for (int step = first; step < s1 && ok; step += sstep) {
                const int g = step & 1;
                int sw, pw, sa, pa;
                wpos((g ? jw1 : jw0) + count_par(s0, step, g), g, sw, pw);
                apos(ja + (step - s0), (g ? jw1 : jw0) + count_par(s0, step, g), g, sa, pa);
                if (!(ok = mbar_wait_cl(fullW(sw), pw, s_abort))) break;
                const uint32_t w_addr = sbase + OFF_W + sw * W_BYTES;
                // descriptors of the stage's k-slices differ only in their start-address
                // field (address / 16, 14 bits, no carry for these offsets): one is built,
                // the others are it plus a constant (the issuing thread's instructions are
                // on the tensor pipe's critical path)
                const uint64_t bd0 = BWD ? tc::smem_desc_sw128(w_addr, 8192, 1024)
                                         : tc::smem_desc_sw128(w_addr, 16, 1024);
                if (!(ok = mbar_wait_cl(fullA(sa), pa, s_abort))) break;
                tc::tc_fence_after();
                const uint32_t a_addr = sbase + OFF_A + (sa * MT + u) * A_BYTES;
                const uint64_t ad0 = tc::smem_desc_sw128(a_addr, 16, 1024);
#pragma unroll
                for (int kk = 0; kk < BK / 16; ++kk) {
                    const uint64_t adesc = ad0 + (uint64_t)((kk * 32) >> 4);
                    const uint64_t bdesc = bd0 + (uint64_t)((BWD ? kk * 2048 : kk * 32) >> 4);
                    tc2_mma(d_tmem, adesc, bdesc, idesc, (step > first || kk > 0) ? 1u : 0u);
                }
                tc2_commit_both(emptyA(sa));
                tc2_commit_both(emptyW(sw));
            }
            // both issuers commit every span (an MT = 1 issuer with no step in a one-step
            // span commits nothing new: its arrival comes at once); the epilogue adds only
            // the accumulators that received a step
            if (ok) tc2_commit_both(tfull(acc));
            jw0 += count_par(s0, s1, 0);
            jw1 += count_par(s0, s1, 1);
            ja += s1 - s0;
            ++it;
        }
        tc2_commit_local(drain);
        mbar_drain_cl(drain, 0);
    };

    if (warp == 0) {
        // ------------------------------------------------------------ activations (both CTAs)
        if (lane == 0) {
            int last_ph[SA];                             // phase of each stage's last issued copy
#pragma unroll
            for (int i = 0; i < SA; ++i) last_ph[i] = -1;
            int ja = 0, ja0 = 0, ja1 = 0;
            bool ok = true;
            Spans spn(skm, pair, npairs, ntiles, nsteps);
            int64_t tile;
            int s0, s1;
            while (ok && spn.next(tile, s0, s1)) {
                const int m0 = (int)((tile % mtiles) * BM * MT + crank * HM);
                for (int step = s0; step < s1 && ok; ++step) {
                    // one stage = the step's MT token tiles (slots MT sa .. MT sa + MT - 1), one
                    // barrier pair: an issuing thread tests and commits once per step
                    const int g = step & 1;
                    int sa, pa;
                    apos(ja + (step - s0), (g ? ja1 : ja0) + count_par(s0, step, g), g, sa, pa);
                    if (!(ok = tc::mbar_wait(emptyA(sa), pa ^ 1, s_abort))) break;
                    if (leader) tc::mbar_expect_tx(fullA(sa), MT * 2 * A_BYTES);    // both halves land here
                    const uint32_t bar = mapa(fullA(sa), 0);
                    if (step >= nks) grid_dep_wait();              // the scaled LoRA activation is complete
#pragma unroll
                    for (int u = 0; u < MT; ++u) {                 // token tile u of the group
                        const uint32_t dst = sbase + OFF_A + (sa * MT + u) * A_BYTES;
                        if (step < nks) tma_load_2d_pair(dst, &tmA, bar, step * BK, m0 + u * BM);
                        else tma_load_2d_pair(dst, &tmL, bar, (step - nks) * BK, m0 + u * BM);
                    }
                    last_ph[sa] = pa;
                }
                ja += s1 - s0;
                ja0 += count_par(s0, s1, 0);
                ja1 += count_par(s0, s1, 1);
            }
            if (!ok && leader)                           // wait for the copies in flight
                for (int i = 0; i < SA; ++i)
                    if (last_ph[i] >= 0) mbar_drain_cl(fullA(i), last_ph[i]);
        }
    } else if (warp == 14) {
        // ------------------------------------------------------------ packed weights (own half)
        if (lane == 0) {
            int last_ph[SP];                             // phase of each stage's last issued copy
#pragma unroll
            for (int i = 0; i < SP; ++i) last_ph[i] = -1;
            bool ok = true;
            int jp0 = 0, jp1 = 0;
            Spans spn(skm, pair, npairs, ntiles, nsteps);
            int64_t tile;
            int s0, s1;
            while (ok && spn.next(tile, s0, s1)) {
                const int c0 = (int)((tile / mtiles) * BN + crank * HN);
                const int e = s1 < nks ? s1 : nks;
                for (int step = s0; step < e && ok; ++step) {
                    const int g = step & 1;
                    int sp, pp;
                    ppos((g ? jp1 : jp0) + count_par(s0, step, g), g, sp, pp);
                    if (!(ok = tc::mbar_wait(emptyP(sp), pp ^ 1, s_abort))) break;
                    tc::mbar_expect_tx(fullP(sp), P_BYTES);
                    if (!BWD) tc::tma_load_2d(sbase + OFF_P + sp * P_BYTES, &tmP, fullP(sp), step * (BK / 2), c0);
                    else tc::tma_load_2d(sbase + OFF_P + sp * P_BYTES, &tmP, fullP(sp), c0 / 2, step * BK);
                    last_ph[sp] = pp;
                }
                if (s0 < e) {
                    jp0 += count_par(s0, e, 0);
                    jp1 += count_par(s0, e, 1);
                }
            }
            if (!ok)                                     // wait for the copies in flight
                for (int i = 0; i < SP; ++i)
                    if (last_ph[i] >= 0) tc::mbar_drain(fullP(i), last_ph[i]);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer 0 (leader)
        if (leader && lane == 0) issue(0);
        else if (!leader && lane == 0) forward(0);
    } else if (warp == 15) {
        // ------------------------------------------------------------ MMA issuer 1 (leader)
        if (!leader && lane == 0) forward(1);
        if (NISS > 1 && leader && lane == 0) issue(1);
    } else if (warp < 10) {
        // ------------------------------------------------------------ dequantizers: two groups, alternate steps
        const int grp = (warp - 2) >> 2;               // 0: even steps, 1: odd steps
        const int t = ((warp - 2) & 3) * 32 + lane;    // 0..127
        const int drow = deq_row<BWD>(t), dblk = deq_blk<BWD>(t);
        bool ok = true;
        // Block-constant inputs (the code's aligned 32-bit word, scale, mean) of a step are
        // copied with cp.async into this thread's slot two group-steps ahead.  Async
        // copies are not waited for by the release arrives of the stage barriers, so
        // their memory latency stays off the step; the thread waits for its own copies
        // (cp.async.wait_group) just before it needs them.
        const int dthr = (warp - 2) * 32 + lane;                     // 0..255
        const uint32_t cbase = sbase + OFF_C + (uint32_t)dthr * 4;
        auto cslot = [&](int slot, int wd) { return cbase + (uint32_t)((slot * 3 + wd) * 2 * kGroupThreads * 4); };
        int shift0 = 0, shift1 = 0;                                  // byte of the code in its word
        // A step past the tile's last dequantization step (a LoRA step, or beyond the
        // tile) reads no constants: it copies nothing and commits an empty group.  Such
        // steps are the last fetches of a tile, and the next tile's first fetches write
        // the same slots before anyone waits for these; two copies in flight to one
        // address may land in either order, so none of them may be a copy.
        auto fetch = [&](int64_t c0, int st, int slot, int lim) {
            if (st >= lim) {
                asm volatile("cp.async.commit_group;" ::: "memory");
                return;
            }
            int64_t n, kb;
            if (!BWD) { n = c0 + drow; kb = st; }
            else { n = (int64_t)st * BK + drow; kb = c0 / kBlock + dblk; }
            const bool v = n < a.N && kb < nblk;
            const int64_t b = v ? n * nblk + kb : 0;
            const int sz = v ? 4 : 0;                                   // 0: zero-fill (constant 0)
            if (slot) shift1 = (int)(b & 3) * 8;
            else shift0 = (int)(b & 3) * 8;
            asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(cslot(slot, 0)),
                         "l"(a.codes + (b & ~(int64_t)3)), "r"(sz) : "memory");
            asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(cslot(slot, 1)), "l"(a.scale + (b >> 8)),
                         "r"(sz) : "memory");
            asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(cslot(slot, 2)), "l"(a.mean + (b >> 8)),
                         "r"(sz) : "memory");
            asm volatile("cp.async.commit_group;" ::: "memory");
        };
        auto block_const = [&](int slot) {
            asm volatile("cp.async.wait_group 1;" ::: "memory");       // this slot's copies have landed
            const uint32_t wd = lds_u32(cslot(slot, 0));
            const float sc = __uint_as_float(lds_u32(cslot(slot, 1))), mu = __uint_as_float(lds_u32(cslot(slot, 2)));
            const int code = (int)(int8_t)(uint8_t)(wd >> (slot ? shift1 : shift0));
            return __fmaf_rn((float)code, sc, mu);
        };
        int jw = 0, jp = 0;
        Spans spn(skm, pair, npairs, ntiles, nsteps);
        int64_t tile;
        int s0, s1;
        while (ok && spn.next(tile, s0, s1)) {
            const int64_t c0 = (tile / mtiles) * BN + crank * HN;   // this CTA's first output column
            const int lim = s1 < nks ? s1 : nks;                     // dequantization steps of the span end here
            const int f0 = s0 + ((s0 & 1) != grp ? 1 : 0);           // the group's first step of the span
            fetch(c0, f0, 0, lim);
            fetch(c0, f0 + 2, 1, lim);
            for (int step = f0, k = 0; step < s1 && ok; step += 2, ++k) {
                int sw, pw;
                wpos(jw + k, grp, sw, pw);
                const int slot = k & 1;
                uint32_t o[8][4];
                int rel = -1;               // packed stage to release once its data is consumed
                if (step < nks) {
                    const float c = block_const(slot);
                    int sp, pp;
                    ppos(jp + k, grp, sp, pp);
                    rel = sp;
                    if (!(ok = tc::mbar_wait(fullP(sp), pp, s_abort))) break;
                    uint4 p0, p1;
                    const uint32_t pst = sbase + OFF_P + sp * P_BYTES;
                    const uint32_t src0 = pst + p_chunk_offset<BWD>(t, 0), src1 = pst + p_chunk_offset<BWD>(t, 1);
                    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(p0.x), "=r"(p0.y), "=r"(p0.z), "=r"(p0.w) : "r"(src0));
                    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(p1.x), "=r"(p1.y), "=r"(p1.z), "=r"(p1.w) : "r"(src1));
                    const BlockTable tb = make_block_table(tab, c);
                    const uint32_t pwd[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
#pragma unroll
                    for (int ch = 0; ch < 8; ++ch) decode8(tb, pwd[ch], o[ch]);
                } else {
                    grid_dep_wait();                           // the LoRA weight rows (maybe padded) are complete
                    const int lc = step - nks;
                    const uint16_t* src;
                    int64_t col0;
                    bool rowok;
                    if (!BWD) {
                        const int64_t n = c0 + drow;
                        rowok = n < a.N;
                        src = a.lora_w + n * a.ldl;
                        col0 = (int64_t)lc * BK;
                    } else {
                        const int64_t ip = (int64_t)lc * BK + drow, i = ip >= a.lper ? ip - a.lper : ip;
                        rowok = ip < 2 * a.lper && i < a.r;
                        src = a.lora_w + i * a.ldl;
                        col0 = c0 + dblk * 64;
                    }
#pragma unroll
                    for (int ch = 0; ch < 8; ++ch) {
                        int64_t col = col0 + ch * 8;
                        bool v;
                        if (BWD) {
                            v = rowok && col < a.K;
                        } else {                    // rank index: the same B columns for hi and lo
                            v = rowok && col < 2 * a.lper;
                            if (col >= a.lper) col -= a.lper;
                            v = v && col < a.r;
                        }
                        uint4 q = make_uint4(0, 0, 0, 0);
                        if (v) q = __ldg(reinterpret_cast<const uint4*>(src + col));
                        o[ch][0] = q.x; o[ch][1] = q.y; o[ch][2] = q.z; o[ch][3] = q.w;
                    }
                }
                if (!(ok = tc::mbar_wait(emptyW(sw), pw ^ 1, s_abort))) break;
                const uint32_t wbase = sbase + OFF_W + sw * W_BYTES;
#pragma unroll
                for (int ch = 0; ch < 8; ++ch)
                    tc::st_shared_v4(wbase + w_chunk_offset<BWD>(t, ch), o[ch][0], o[ch][1], o[ch][2], o[ch][3]);
                tc::fence_proxy_async();                  // this thread's tile writes -> async proxy
                __syncwarp();
                // the leader's own warps release at CTA scope (same CTA as the MMA issuer);
                // the peer's warps release at cluster scope on the leader's barrier
                // the leader's warps arrive on its own barrier; the peer's on a local one whose
                // completion a forwarder passes on (a cluster-scope release per warp and step
                // would cost each dequantizer a cluster fence, ~1000 cycles)
                // the packed stage is released only after the stores above, which consume
                // the values decoded from it: a release right after the shared loads were
                // issued let the next TMA copy overwrite the stage under loads in flight
                if (lane == 0) {
                    tc::mbar_arrive(leader ? fullW(sw) : fullWl(sw));
                    if (rel >= 0) tc::mbar_arrive(emptyP(rel));
                }
                fetch(c0, step + 4, slot, lim);                // refill: the group's step after next
            }
            jw += count_par(s0, s1, grp);
            jp += count_par(s0, s0 > lim ? s0 : lim, grp);
        }
        asm volatile("cp.async.wait_all;" ::: "memory");
    } else {
        // ------------------------------------------------------------ epilogue (own 128 tokens)
        // Stream-K: a span that does not end its tile leaves its fp32 partial sums in this
        // pair's slot of a.part, then (per warp, after its lanes' stores) counts itself in
        // a.flags[tile][rank][warp]; the span that ends the tile waits, per warp, for the
        // counts of the lower pairs pf .. pair - 1 that took the tile's head and adds their
        // partials to its accumulator in pair order.  No barrier across warps: every wait
        // is a bounded poll.
        const int q = warp & 3;
        const int row = q * 32 + lane;
        if (leader && warp == 10) {
            if (lane == 0) {
                grid_dep_wait();
                grid_dep_launch();
            }
            __syncwarp();
        }
        bool ok = true;
        int it = 0;
        const int64_t U = ntiles * (int64_t)nsteps;
        Spans spn(skm, pair, npairs, ntiles, nsteps);
        int64_t tile;
        int s0, s1;
        while (ok && spn.next(tile, s0, s1)) {
            const int acc = it % NACC, aph = (it / NACC) & 1;
            ++it;
            const int64_t c0 = (tile / mtiles) * BN;
            const bool contrib = skm && s1 < nsteps;
            int64_t pf = pair;                               // first pair whose partials this span adds
            if (skm && s1 == nsteps && s0 > 0) {
                const int64_t tb = tile * (int64_t)nsteps;
                pf = pair - 1;
                while (pf > 0 && pf * U / npairs > tb) --pf;
            }
            int* fq = skm ? a.flags + ((tile * 2 + crank) * 4 + q) : nullptr;
            if (!(ok = tc::mbar_wait(tfull(acc), aph, s_abort))) break;
            tc::tc_fence_after();
            if (skm) grid_dep_wait();                          // the counters are zeroed
            if (pf < pair) {
                const int want = (int)(pair - pf);
                if (ld_acquire_gpu(fq) < want) {
                    const uint64_t t0 = tc::globaltimer();
                    while (ld_acquire_gpu(fq) < want) {
                        if (*s_abort) { ok = false; break; }
                        if (tc::globaltimer() - t0 > tc::kWaitTimeoutNs) {
                            *s_abort = 1;
                            report_timeout();
                            ok = false;
                            break;
                        }
                    }
                }
                ok = __all_sync(0xffffffffu, ok);
                if (!ok) break;
            }
            // owner: item i = (chunk i / nc, lower pair pf + i % nc) of the partials, copied by
            // each lane for its own row (pieces j = 0..7) into buffer i % kFixD of its warp
            const int nc = (int)(pair - pf);
            const int nitems = nc * MT * (BN / 32);
            const uint32_t fbase = sbase + OFF_A + (uint32_t)(q * kFixD * 4096);
            auto fix_buf = [&](int i) { return fbase + (uint32_t)((i % kFixD) * 4096); };
            auto fix_issue = [&](int i) {
                if (i < nitems) {
                    const int ucc = i / nc, c = i - ucc * nc;
                    const float* src = a.part + part_off((pf + c) * 2 + crank, MT * (BN / 32), ucc, 0, row);
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;"
                                     ::"r"(fix_buf(i) + (uint32_t)((j * 32 + lane) * 16)), "l"(src + j * 128 * 4)
                                     : "memory");
                }
                asm volatile("cp.async.commit_group;" ::: "memory");
            };
            int fi = 0;
            if (nc > 0)
                for (int i = 0; i < kFixD; ++i) fix_issue(i);
            // one 32-column chunk of this warp's 32 rows, its accumulator values in r
            auto emit = [&](int ucc, uint32_t (&r)[32]) {
                const int u = ucc / (BN / 32), cc = ucc % (BN / 32);
                const int64_t m = (tile % mtiles) * BM * MT + u * BM + crank * HM + row;
                if (contrib) {
                    float* dst = a.part + part_off(pair * 2 + crank, MT * (BN / 32), ucc, 0, row);
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        *reinterpret_cast<float4*>(dst + j * 128 * 4) =
                            make_float4(__uint_as_float(r[4 * j]), __uint_as_float(r[4 * j + 1]),
                                        __uint_as_float(r[4 * j + 2]), __uint_as_float(r[4 * j + 3]));
                    return;
                }
                for (int c = 0; c < nc; ++c, ++fi) {
                    asm volatile("cp.async.wait_group %0;" ::"n"(kFixD - 1) : "memory");
                    const uint32_t buf = fix_buf(fi);
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        uint32_t v0, v1, v2, v3;
                        asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                                     : "=r"(v0), "=r"(v1), "=r"(v2), "=r"(v3) : "r"(buf + (uint32_t)((j * 32 + lane) * 16)));
                        r[4 * j] = __float_as_uint(__uint_as_float(r[4 * j]) + __uint_as_float(v0));
                        r[4 * j + 1] = __float_as_uint(__uint_as_float(r[4 * j + 1]) + __uint_as_float(v1));
                        r[4 * j + 2] = __float_as_uint(__uint_as_float(r[4 * j + 2]) + __uint_as_float(v2));
                        r[4 * j + 3] = __float_as_uint(__uint_as_float(r[4 * j + 3]) + __uint_as_float(v3));
                    }
                    fix_issue(fi + kFixD);               // this lane's buffer is read: refill it
                }
                if (m < a.M) {
                    uint16_t* dst = a.out + m * a.n_out + c0 + cc * 32;
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        if (c0 + cc * 32 + j * 8 < a.n_out) {
                            uint4 v;
                            v.x = pack_bf16x2(__uint_as_float(r[8 * j + 0]), __uint_as_float(r[8 * j + 1]));
                            v.y = pack_bf16x2(__uint_as_float(r[8 * j + 2]), __uint_as_float(r[8 * j + 3]));
                            v.z = pack_bf16x2(__uint_as_float(r[8 * j + 4]), __uint_as_float(r[8 * j + 5]));
                            v.w = pack_bf16x2(__uint_as_float(r[8 * j + 6]), __uint_as_float(r[8 * j + 7]));
                            *reinterpret_cast<uint4*>(dst + j * 8) = v;
                        }
                    }
                }
            };
            // MT = 1: issuer g's accumulator (columns g BN) holds the span's steps of parity
            // g; the tile's sum is issuer 0's plus issuer 1's (a one-step span fills one)
            const bool has0 = MT == 2 || count_par(s0, s1, 0) > 0;
            const bool has1 = MT == 2 || count_par(s0, s1, 1) > 0;
            const uint32_t trow = tmem_base + ((uint32_t)(q * 32) << 16);
            if (MT == 2 || !(has0 && has1)) {
                // two chunks per wait for the tensor-memory loads (one wait per chunk left
                // the epilogue bound by their latency)
                const uint32_t cb = (MT == 1 && !has0) ? (uint32_t)BN : 0u;
#pragma unroll 1
                for (int ucc = 0; ucc < MT * (BN / 32); ucc += 2) {
                    uint32_t r0[32], r1[32];
                    const uint32_t t0 = trow + cb + (uint32_t)((ucc / (BN / 32)) * BN + (ucc % (BN / 32)) * 32);
                    TC_LD32(t0, r0);
                    TC_LD32(t0 + 32, r1);                // chunk ucc + 1: the next 32 columns (BN / 32 is even)
                    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
                    emit(ucc, r0);
                    emit(ucc + 1, r1);
                }
            } else {
#pragma unroll 1
                for (int ucc = 0; ucc < BN / 32; ++ucc) {
                    uint32_t r0[32], r1[32];
                    const uint32_t t0 = trow + (uint32_t)(ucc * 32);
                    TC_LD32(t0, r0);
                    TC_LD32(t0 + BN, r1);                // the same 32 columns of issuer 1's accumulator
                    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
                    for (int j = 0; j < 32; ++j) r0[j] = __float_as_uint(__uint_as_float(r0[j]) + __uint_as_float(r1[j]));
                    emit(ucc, r0);
                }
            }
            if (nc > 0) asm volatile("cp.async.wait_all;" ::: "memory");
            tc::tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                if (leader) tc::mbar_arrive(tempty(acc));
                else mbar_arrive_cl(mapa(tempty(acc), 0));
                if (contrib) {                   // this warp's partial rows are written: count them
                    __threadfence();
                    atomicAdd(fq, 1);
                }
            }
        }
    }

    __syncthreads();
    cluster_sync();                      // neither CTA leaves while the pair may still use its memory
    if (warp == 1) {
        tc::tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(kTmemCols));
    }
}

}  // namespace tc2
}  // namespace qnf4
