// tc_gemm.cuh -- fused NF4 dequant + GEMM on the 5th-generation tensor cores
// (tcgen05, accumulators in TMEM), for the large-M forward and backward-dX.
//
//   forward : Y [M, N]  = X [M, K]  . W'^T      + (s T)[M, r] . B^T   (B [N, r])
//   backward: dX [M, K] = dY [M, N] . W'        + (s U)[M, r] . A     (A [r, K])
//
// One persistent CTA per SM walks 128 x 256 output tiles (128 tokens x 256
// output features), tokens fastest so that the CTAs running at the same time
// share the same weight tile in L2.  Warp roles (480 threads):
//   warp 0      TMA producer of the activation tiles (128 x 64 bf16, 128-byte
//               swizzle);
//   warp 14     TMA producer of the packed NF4 tiles, on its own 8-deep ring
//               so that the HBM latency of the weight stream stays off the
//               MMA's critical path;
//   warp 1      TMEM allocator and MMA issuer (one thread): 4 MMAs of
//               128 x 256 x 16 per 64-wide reduction step;
//   warps 2-9   dequantizers: one thread per 64-weight row-block per step;
//               exact bf16_rne(L[q] * c') from a per-block register table
//               (nf4_decode.cuh), written straight into the swizzled operand
//               layout the MMA reads (K-major for the forward, MN-major for
//               the backward, where the reduction runs over the rows of W);
//   warps 10-13 epilogue: TMEM -> registers -> bf16 -> global.
// The accumulator is double-buffered in TMEM (2 x 256 columns), so the
// epilogue of one tile overlaps the main loop of the next.  The LoRA term is
// ceil(r / 64) extra reduction steps whose activation side (s T or s U,
// zero-padded to 64 columns by the TMA box) comes through the same ring and
// whose weight side (rows of B, or rows of A) is copied by the dequantizers.
//
// Every mbarrier wait is bounded: after kWaitTimeoutNs the waiting thread
// raises a CTA-wide abort flag and the device status word, every role leaves
// its loop, in-flight TMA copies are waited for (bounded again), the MMA
// thread drains its MMAs, and TMEM is freed before the CTA exits.
#pragma once
#include <cuda.h>
#include "common.cuh"
#include "nf4_decode.cuh"

namespace qnf4 {
namespace tc {

constexpr int BM = 128, BN = 256, BK = 64;
constexpr int SA = 3;                         // activation ring stages (16 KB)
constexpr int SW = 3;                         // dequantized weight ring stages (32 KB)
constexpr int SP = 8;                         // packed weight ring stages (8 KB)
constexpr int A_BYTES = BM * BK * 2;          // 16384
constexpr int W_BYTES = BN * BK * 2;          // 32768
constexpr int P_BYTES = BN * BK / 2;          // 8192
constexpr int kThreads = 480;
constexpr int kDeqThreads = 256;
constexpr int kEpiThreads = 128;
constexpr int kTmemCols = 512;
constexpr unsigned long long kWaitTimeoutNs = 4000000000ull;   // 4 s

constexpr int OFF_A = 0;
constexpr int OFF_W = OFF_A + SA * A_BYTES;
constexpr int OFF_P = OFF_W + SW * W_BYTES;
constexpr int OFF_BAR = OFF_P + SP * P_BYTES;
// barriers: fullA[SA] emptyA[SA] fullW[SW] emptyW[SW] fullP[SP] emptyP[SP] tfull[2] tempty[2] drain
constexpr int NBAR = 2 * SA + 2 * SW + 2 * SP + 4 + 1;
constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
constexpr int SMEM_BYTES = OFF_MISC + 16;
constexpr int SMEM_ALLOC = SMEM_BYTES + 1024;      // slack for 1024-byte alignment

struct Args {
    const int8_t* codes;
    const float* scale;
    const float* mean;
    const uint16_t* lora_w;   // forward: B [N, ldl]; backward: A [r, ldl]
    int64_t ldl;              // row stride of lora_w in elements (multiple of 8)
    int r;                    // LoRA rank
    // The LoRA term enters as extra reduction steps over a scaled activation
    // (s T forward, s U backward) held as a bf16 hi + lo pair, [hi | lo] with
    // each half `lper` columns wide (r rounded up to 16, zero beyond r): LoRA
    // reduction index j' pairs with rank index j' mod lper, for j' < 2 lper.
    int lper;
    int nlora;                // ceil(2 lper / 64) extra reduction steps
    uint16_t* out;            // Y [M, N] or dX [M, K]
    int64_t M, N, K;          // W is [N, K]
    int64_t n_out;            // N (forward) or K (backward)
    int64_t n_red;            // K (forward) or N (backward)
    // stream-K (SM-pair kernel only): the (tile, reduction step) units are dealt to the
    // pairs in equal contiguous runs instead of whole tiles round-robin
    int sk;
    float* part;              // fp32 partial tiles, one slot per pair: [pairs][2 CTAs][MT x 128 rows][256]
    int* flags;               // per (tile, CTA rank): partial tiles written so far; zero at launch
};

// ----------------------------------------------------------------------------
// PTX wrappers
// ----------------------------------------------------------------------------
__device__ __forceinline__ uint64_t globaltimer() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}

__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok) : "r"(bar), "r"(parity) : "memory");
    return ok != 0;
}

// Bounded wait; false if the CTA is aborting or the wait timed out (which
// raises the abort flag and the device status).
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag) {
    if (mbar_try(bar, parity)) return true;
    const uint64_t t0 = globaltimer();
    while (true) {
        if (mbar_try(bar, parity)) return true;
        if (*abort_flag) return false;
        if (globaltimer() - t0 > kWaitTimeoutNs) {
            *abort_flag = 1;
            report_timeout();
            return false;
        }
    }
}

// Bounded wait without the abort shortcut (teardown: waiting for copies already in flight).
__device__ __forceinline__ void mbar_drain(uint32_t bar, uint32_t parity) {
    const uint64_t t0 = globaltimer();
    while (!mbar_try(bar, parity)) {
        if (globaltimer() - t0 > kWaitTimeoutNs) { report_timeout(); return; }
    }
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, uint32_t bar, int x, int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
        ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
        : "memory");
}

__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tc_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}

__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                       uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Shared-memory matrix descriptor, 128-byte swizzle, sm_100 version field.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)2 << 61;
    return d;
}

// Instruction descriptor: kind::f16, A = B = bf16, D = f32, M = 128, N = 256.
__host__ __device__ constexpr uint32_t make_idesc(bool b_mn_major) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((b_mn_major ? 1u : 0u) << 16) | ((uint32_t)(BN >> 3) << 17) |
           ((uint32_t)(BM >> 4) << 24);
}

#define TC_LD32(taddr, r)                                                                                           \
    asm volatile(                                                                                                   \
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18," \
        "%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"                                              \
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),         \
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),   \
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), \
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])  \
        : "r"(taddr))

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

// Which row-block dequantizer thread d (0..255) owns in one reduction step:
//   forward : tile row d (output feature c0 + d), the step's 64-wide k-block;
//   backward: reduction row n = 8 (d / 32) + d % 8 of the step's 64 W rows,
//             output block j = (d / 8) % 4 of the tile's 256 columns.
// In the backward the 8 lanes of a quarter-warp hold 8 different rows, so
// their 16-byte stores land in 8 different bank groups of the swizzled tile.
template <bool BWD>
__device__ __forceinline__ int deq_row(int d) { return BWD ? 8 * (d >> 5) + (d & 7) : d; }
template <bool BWD>
__device__ __forceinline__ int deq_blk(int d) { return BWD ? (d >> 3) & 3 : 0; }

// Byte offset, inside one stage of the weight ring, of 16-byte chunk `ch`
// (8 consecutive weights) of the row-block of thread d:
//   forward  (K-major, 128-byte rows): row d, chunk ch at position ch ^ (d & 7);
//   backward (MN-major): atom j = block (8 KB apart), 8-row group n / 8
//     (1 KB apart), row n % 8 (128 B apart), chunk ch ^ (n % 8).
template <bool BWD>
__device__ __forceinline__ uint32_t w_chunk_offset(int d, int ch) {
    if (!BWD) return (uint32_t)(d * 128 + ((ch ^ (d & 7)) << 4));
    const int n = deq_row<true>(d), j = deq_blk<true>(d);
    return (uint32_t)(j * 8192 + (n >> 3) * 1024 + (n & 7) * 128 + ((ch ^ (n & 7)) << 4));
}

// Byte offsets of the two 16-byte packed chunks of thread d's row-block in a
// stage of the packed ring.  The forward tile (256 rows x 32 B) is written by
// TMA with 32-byte swizzle (chunk ^= address bit 7), the backward tile
// (64 rows x 128 B) with 128-byte swizzle (chunk ^= row % 8).
template <bool BWD>
__device__ __forceinline__ uint32_t p_chunk_offset(int d, int c) {
    if (!BWD) return (uint32_t)(d * 32 + ((c ^ ((d >> 2) & 1)) << 4));
    const int n = deq_row<true>(d), j = deq_blk<true>(d);
    return (uint32_t)(n * 128 + (((2 * j + c) ^ (n & 7)) << 4));
}

// ----------------------------------------------------------------------------
template <bool BWD>
__global__ void __launch_bounds__(kThreads, 1)
k_tc_gemm(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmL,
          const __grid_constant__ CUtensorMap tmP, Args a, NF4Tables tab) {
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
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(base + OFF_MISC);
    volatile int* s_abort = reinterpret_cast<volatile int*>(base + OFF_MISC + 4);

    // kernels launched behind this one with programmatic serialization (the
    // adapter products dB and dA, which read nothing this kernel writes) may start
    grid_dep_launch();
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t mtiles = cdiv(a.M, BM), ntiles_n = cdiv(a.n_out, BN);
    const int64_t ntiles = mtiles * ntiles_n;
    const int nks = (int)cdiv(a.n_red, BK);
    const int nsteps = nks + a.nlora;
    const int64_t nblk = a.K / kBlock;

    if (tid == 0) {
        for (int i = 0; i < SA; ++i) { mbar_init(fullA(i), 1); mbar_init(emptyA(i), 1); }
        for (int i = 0; i < SW; ++i) { mbar_init(fullW(i), kDeqThreads / 32); mbar_init(emptyW(i), 1); }
        for (int i = 0; i < SP; ++i) { mbar_init(fullP(i), 1); mbar_init(emptyP(i), kDeqThreads / 32); }
        for (int i = 0; i < 2; ++i) { mbar_init(tfull(i), 1); mbar_init(tempty(i), kEpiThreads / 32); }
        mbar_init(drain, 1);
        *s_abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(s_tmem)),
                     "r"(kTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
        tc_fence_before();
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *s_tmem;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer: activations
        if (lane == 0) {
            int sa = 0, pa = 0, issued = 0;
            bool ok = true;
            for (int64_t tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x) {
                const int m0 = (int)((tile % mtiles) * BM);
                for (int step = 0; step < nsteps && ok; ++step) {
                    if (!(ok = mbar_wait(emptyA(sa), pa ^ 1, s_abort))) break;
                    mbar_expect_tx(fullA(sa), A_BYTES);
                    if (step < nks) tma_load_2d(sbase + OFF_A + sa * A_BYTES, &tmA, fullA(sa), step * BK, m0);
                    else tma_load_2d(sbase + OFF_A + sa * A_BYTES, &tmL, fullA(sa), (step - nks) * BK, m0);
                    ++issued;
                    if (++sa == SA) { sa = 0; pa ^= 1; }
                }
            }
            if (!ok)   // wait for the copies this thread put in flight (the last SA of them)
                for (int i = 1; i <= SA && i <= issued; ++i) mbar_drain(fullA((issued - i) % SA), ((issued - i) / SA) & 1);
        }
    } else if (warp == 14) {
        // ------------------------------------------------------------ TMA producer: packed weights
        if (lane == 0) {
            int sp = 0, pp = 0, issued = 0;
            bool ok = true;
            for (int64_t tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x) {
                const int c0 = (int)((tile / mtiles) * BN);
                for (int step = 0; step < nks && ok; ++step) {
                    if (!(ok = mbar_wait(emptyP(sp), pp ^ 1, s_abort))) break;
                    mbar_expect_tx(fullP(sp), P_BYTES);
                    if (!BWD) tma_load_2d(sbase + OFF_P + sp * P_BYTES, &tmP, fullP(sp), step * (BK / 2), c0);
                    else tma_load_2d(sbase + OFF_P + sp * P_BYTES, &tmP, fullP(sp), c0 / 2, step * BK);
                    ++issued;
                    if (++sp == SP) { sp = 0; pp ^= 1; }
                }
            }
            if (!ok)
                for (int i = 1; i <= SP && i <= issued; ++i) mbar_drain(fullP((issued - i) % SP), ((issued - i) / SP) & 1);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = make_idesc(BWD);
            int sa = 0, pa = 0, sw = 0, pw = 0;
            bool ok = true;
            int it = 0;
            for (int64_t tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x, ++it) {
                const int acc = it & 1, aph = (it >> 1) & 1;
                if (!(ok = mbar_wait(tempty(acc), aph ^ 1, s_abort))) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + acc * BN;
                for (int step = 0; step < nsteps && ok; ++step) {
                    if (!(ok = mbar_wait(fullA(sa), pa, s_abort))) break;
                    if (!(ok = mbar_wait(fullW(sw), pw, s_abort))) break;
                    tc_fence_after();
                    const uint32_t a_addr = sbase + OFF_A + sa * A_BYTES;
                    const uint32_t w_addr = sbase + OFF_W + sw * W_BYTES;
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk) {
                        const uint64_t adesc = smem_desc_sw128(a_addr + kk * 32, 16, 1024);
                        const uint64_t bdesc = BWD ? smem_desc_sw128(w_addr + kk * 2048, 8192, 1024)
                                                   : smem_desc_sw128(w_addr + kk * 32, 16, 1024);
                        tc_mma(d_tmem, adesc, bdesc, idesc, (step > 0 || kk > 0) ? 1u : 0u);
                    }
                    tc_commit(emptyA(sa));
                    tc_commit(emptyW(sw));
                    if (++sa == SA) { sa = 0; pa ^= 1; }
                    if (++sw == SW) { sw = 0; pw ^= 1; }
                }
                if (ok) tc_commit(tfull(acc));
            }
            // all MMAs issued by this thread have completed once this arrives
            tc_commit(drain);
            mbar_drain(drain, 0);
        }
    } else if (warp < 10) {
        // ------------------------------------------------------------ dequantizers
        const int d = tid - 64;
        const int drow = deq_row<BWD>(d), dblk = deq_blk<BWD>(d);
        int sw = 0, pw = 0, sp = 0, pp = 0;
        bool ok = true;
        // block constant inputs of reduction step `st` for this thread, fetched two steps ahead
        auto fetch = [&](int64_t c0, int st, int& code, float& sc, float& mu) {
            int64_t n, kb;
            if (!BWD) { n = c0 + drow; kb = st; }
            else { n = (int64_t)st * BK + drow; kb = c0 / kBlock + dblk; }
            code = 0; sc = 0.f; mu = 0.f;
            if (st < nks && n < a.N && kb < nblk) {
                const int64_t b = n * nblk + kb;
                const int64_t g = b >> 8;
                code = __ldg(a.codes + b);
                sc = __ldg(a.scale + g);
                mu = __ldg(a.mean + g);
            }
        };
        // one reduction step; (code, sc, mu) hold this step's block-constant inputs on
        // entry and are refilled with those of step + 2 (two slots alternate, so the
        // loads have two steps to land before anything reads the registers)
        auto do_step = [&](int64_t c0, int step, int& code, float& sc, float& mu) {
            uint32_t o[8][4];
            int rel = -1;                   // packed stage to release once its data is consumed
            if (step < nks) {
                const float c = __fmaf_rn((float)code, sc, mu);
                fetch(c0, step + 2, code, sc, mu);
                if (!(ok = mbar_wait(fullP(sp), pp, s_abort))) return;
                uint4 p0, p1;
                const uint32_t pst = sbase + OFF_P + sp * P_BYTES;
                const uint32_t src0 = pst + p_chunk_offset<BWD>(d, 0), src1 = pst + p_chunk_offset<BWD>(d, 1);
                asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(p0.x), "=r"(p0.y), "=r"(p0.z), "=r"(p0.w) : "r"(src0));
                asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(p1.x), "=r"(p1.y), "=r"(p1.z), "=r"(p1.w) : "r"(src1));
                rel = sp;
                if (++sp == SP) { sp = 0; pp ^= 1; }
                const BlockTable tb = make_block_table(tab, c);
                const uint32_t pwd[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
#pragma unroll
                for (int ch = 0; ch < 8; ++ch) decode8(tb, pwd[ch], o[ch]);
            } else {
                // LoRA step: rows of B (forward) or A (backward), zero beyond r / the output edge
                const int lc = step - nks;
                const uint16_t* src;
                int64_t col0;
                bool rowok;
                if (!BWD) {
                    const int64_t n = c0 + drow;
                    rowok = n < a.N;
                    src = a.lora_w + n * a.ldl;
                    col0 = (int64_t)lc * BK;        // LoRA reduction index of chunk 0
                } else {
                    const int64_t ip = (int64_t)lc * BK + drow, i = ip >= a.lper ? ip - a.lper : ip;
                    rowok = ip < 2 * a.lper && i < a.r;
                    src = a.lora_w + i * a.ldl;
                    col0 = c0 + dblk * 64;          // output column of chunk 0
                }
#pragma unroll
                for (int ch = 0; ch < 8; ++ch) {
                    int64_t col = col0 + ch * 8;
                    bool v;
                    if (BWD) {
                        v = rowok && col < a.K;
                    } else {                        // rank index: the same B columns for hi and lo
                        v = rowok && col < 2 * a.lper;
                        if (col >= a.lper) col -= a.lper;
                        v = v && col < a.r;
                    }
                    uint4 q = make_uint4(0, 0, 0, 0);
                    if (v) q = __ldg(reinterpret_cast<const uint4*>(src + col));
                    o[ch][0] = q.x; o[ch][1] = q.y; o[ch][2] = q.z; o[ch][3] = q.w;
                }
            }
            if (!(ok = mbar_wait(emptyW(sw), pw ^ 1, s_abort))) return;
            const uint32_t wbase = sbase + OFF_W + sw * W_BYTES;
#pragma unroll
            for (int ch = 0; ch < 8; ++ch)
                st_shared_v4(wbase + w_chunk_offset<BWD>(d, ch), o[ch][0], o[ch][1], o[ch][2], o[ch][3]);
            fence_proxy_async();
            __syncwarp();
            // The packed stage is released only now: the stores above consume the values
            // decoded from it, so every lane's shared loads of it have returned.  A release
            // right after the loads were issued let the next TMA copy overwrite the stage
            // while some lanes' loads were still in flight.
            if (lane == 0) {
                mbar_arrive(fullW(sw));
                if (rel >= 0) mbar_arrive(emptyP(rel));
            }
            if (++sw == SW) { sw = 0; pw ^= 1; }
        };
        for (int64_t tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x) {
            const int64_t c0 = (tile / mtiles) * BN;
            int codeA, codeB;
            float scA, scB, muA, muB;
            fetch(c0, 0, codeA, scA, muA);
            fetch(c0, 1, codeB, scB, muB);
            for (int step = 0; step < nsteps && ok; step += 2) {
                do_step(c0, step, codeA, scA, muA);
                if (ok && step + 1 < nsteps) do_step(c0, step + 1, codeB, scB, muB);
            }
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3;                    // TMEM lane quarter of this warp
        const int row = q * 32 + lane;
        bool ok = true;
        int it = 0;
        for (int64_t tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x, ++it) {
            const int acc = it & 1, aph = (it >> 1) & 1;
            const int64_t m = (tile % mtiles) * BM + row;
            const int64_t c0 = (tile / mtiles) * BN;
            if (!(ok = mbar_wait(tfull(acc), aph, s_abort))) break;
            tc_fence_after();
#pragma unroll 1
            for (int cc = 0; cc < BN / 32; ++cc) {
                uint32_t r[32];
                const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * BN + cc * 32);
                TC_LD32(taddr, r);
                asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
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
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(tempty(acc));
        }
    }

    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(kTmemCols));
    }
}

}  // namespace tc
}  // namespace qnf4
