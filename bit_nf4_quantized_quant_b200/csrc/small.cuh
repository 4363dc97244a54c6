// small.cuh -- small-M (decode / GEMV-shaped) forward and backward-dX kernels.
//
// For a few tokens the layer is bound by streaming the 4.13-bit weight from
// HBM, and the work per weight is the exact dequantization itself (see
// nf4_decode.cuh: one 16-entry table per 64-weight block, byte-permute
// lookups).  Both kernels let one thread own one row-block (64 consecutive
// weights of a row), so the table is built once per 64 weights.
//
// Forward: Y^T = W' X^T on mma.sync m16n8k16 with the tokens as the MMA rows
// and W' as the B operand.  The B fragment of lane (g, t) is two pairs of one
// row (g) of W, so lane (g, t) can own row n0+g, block 4*ms + t, and feed the
// 16 MMAs of a macro-step (4 blocks, 256 k) straight from registers: in MMA s
// its logical k {2t, 2t+1} are elements 4s, 4s+1 of its block and {2t+8,
// 2t+9} are 4s+2, 4s+3.  The activation fragment is loaded with the same k
// permutation.  No shared memory is touched by the weights.
//
// Backward: dX = dY W' reduces over the rows of W, so the MMA B operand needs
// pairs along n; each thread dequantizes its row-block into a swizzled
// shared-memory tile and the MMA warps read it with ldmatrix.trans.
#pragma once
#include "common.cuh"
#include "nf4_decode.cuh"

namespace qnf4 {

constexpr int kSmallThreads = 512;
constexpr int kSmallWarps = kSmallThreads / 32;
constexpr int kFwdRowGroups = 2;                          // 8-row groups per CTA
constexpr int kFwdKSplits = kSmallWarps / kFwdRowGroups;  // warps sharing a row group

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
    float* part;              // [KS][M][N] fp32 partial sums (KS > 1)
    int* counters;            // [ceil(N/8)] arrival counters, zero on entry, left zero
    int64_t M, N, K;
    int rp, r;
    float s;
    int KS;                   // K splits
    int J;                    // macro-steps (4 blocks, 256 k) per split
};

constexpr int kGemvThreads = 256;
constexpr int kGemvDepth = 4;      // macro-steps whose weight loads are in flight per warp

// One macro-step's weight operands of lane (g, t): 32 packed bytes of row g,
// block 4 ms + t, and the inputs of that block's constant.
struct GemvStage {
    uint4 p0, p1;
    int code;
    float sc, mu;
};

__device__ __forceinline__ void gemv_load(GemvStage& st, const SmallFwdArgs& a, int64_t n, int64_t ms, int64_t ms_end,
                                          int t, int64_t nblk, int64_t rowbytes) {
    const int64_t b = ms * 4 + t;
    if (n < a.N && ms < ms_end && b < nblk) {
        const uint8_t* pp = a.packed + n * rowbytes + 32 * b;
        st.p0 = ldg_nc_v4(pp);
        st.p1 = ldg_nc_v4(pp + 16);
        const int64_t blk = n * nblk + b;
        st.code = __ldg(a.codes + blk);
        st.sc = __ldg(a.scale + (blk >> 8));
        st.mu = __ldg(a.mean + (blk >> 8));
    } else {
        st.p0 = make_uint4(0, 0, 0, 0);
        st.p1 = st.p0;
        st.code = 0;
        st.sc = 0.f;
        st.mu = 0.f;
    }
}

template <int MT>
__device__ __forceinline__ void gemv_compute(float (&acc)[MT][4], const GemvStage& st, const SmallFwdArgs& a,
                                             const NF4Tables& tab, int64_t b, int64_t nblk, int g) {
    const BlockTable tb = make_block_table(tab, __fmaf_rn((float)st.code, st.sc, st.mu));
    const uint32_t pw[8] = {st.p0.x, st.p0.y, st.p0.z, st.p0.w, st.p1.x, st.p1.y, st.p1.z, st.p1.w};
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        uint32_t wa[4], wb[4];
        decode8(tb, pw[2 * u], wa);
        decode8(tb, pw[2 * u + 1], wb);
        const uint32_t wv[8] = {wa[0], wa[1], wa[2], wa[3], wb[0], wb[1], wb[2], wb[3]};
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
            const int64_t m0 = mt * 16 + g, m1 = m0 + 8;
            uint4 x00 = make_uint4(0, 0, 0, 0), x01 = x00, x10 = x00, x11 = x00;
            if (b < nblk) {
                if (m0 < a.M) {
                    const uint4* xp = reinterpret_cast<const uint4*>(a.X + m0 * a.K + 64 * b + 16 * u);
                    x00 = __ldg(xp);
                    x01 = __ldg(xp + 1);
                }
                if (m1 < a.M) {
                    const uint4* xp = reinterpret_cast<const uint4*>(a.X + m1 * a.K + 64 * b + 16 * u);
                    x10 = __ldg(xp);
                    x11 = __ldg(xp + 1);
                }
            }
            const uint32_t xa[8] = {x00.x, x00.y, x00.z, x00.w, x01.x, x01.y, x01.z, x01.w};
            const uint32_t xb[8] = {x10.x, x10.y, x10.z, x10.w, x11.x, x11.y, x11.z, x11.w};
#pragma unroll
            for (int s4 = 0; s4 < 4; ++s4)
                mma_bf16_16816(acc[mt], xa[2 * s4], xb[2 * s4], xa[2 * s4 + 1], xb[2 * s4 + 1], wv[2 * s4],
                               wv[2 * s4 + 1]);
        }
    }
}

// Forward for M <= 16 * MT tokens.  Every warp is independent: work item =
// (8-row group rg, K split ks) covering macro-steps [ks J, ks J + J); its
// weight loads run kGemvDepth macro-steps ahead of the MMAs (a ring of
// register stages indexed at compile time).  The K splits of a row group are
// summed by the warp that arrives last on the group's counter, in split
// order (deterministic), which also adds s * T . B and writes Y in bf16.
template <int MT>
__global__ void __launch_bounds__(kGemvThreads) k_fwd_gemv(SmallFwdArgs a, NF4Tables tab) {
    const int lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int64_t nblk = a.K / kBlock;
    const int64_t nms = cdiv(nblk, 4);
    const int64_t rowbytes = a.K / 2;
    const int64_t nrg = cdiv(a.N, 8);
    const int64_t items = nrg * a.KS;
    const int64_t wid = ((int64_t)blockIdx.x * kGemvThreads + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * kGemvThreads) >> 5;

    for (int64_t item = wid; item < items; item += nwarps) {
        const int64_t rg = item / a.KS, ks = item % a.KS;
        const int64_t n = rg * 8 + g;
        const int64_t ms0 = ks * a.J;
        const int64_t ms_end = min(nms, ms0 + a.J);
        float acc[MT][4];
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) acc[mt][0] = acc[mt][1] = acc[mt][2] = acc[mt][3] = 0.f;
        GemvStage st[kGemvDepth];
#pragma unroll
        for (int u = 0; u < kGemvDepth; ++u) gemv_load(st[u], a, n, ms0 + u, ms_end, t, nblk, rowbytes);
        for (int64_t ms = ms0; ms < ms_end; ms += kGemvDepth) {
#pragma unroll
            for (int u = 0; u < kGemvDepth; ++u) {
                if (ms + u < ms_end) {
                    gemv_compute<MT>(acc, st[u], a, tab, (ms + u) * 4 + t, nblk, g);
                    gemv_load(st[u], a, n, ms + u + kGemvDepth, ms_end, t, nblk, rowbytes);
                }
            }
        }
        // acc[mt]: c0,c1 -> (token mt*16+g, row rg*8 + 2t, +1), c2,c3 -> (token +8)
        const int64_t r0 = rg * 8 + 2 * t;
        if (a.KS == 1) {
#pragma unroll
            for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int64_t m = mt * 16 + g + (e >> 1) * 8, nn = r0 + (e & 1);
                    if (m < a.M && nn < a.N) {
                        float v = acc[mt][e];
                        if (a.T32 != nullptr) {
                            const float* tr = a.T32 + m * a.rp;
                            const uint16_t* br = a.B + nn * a.r;
                            float l = 0.f;
                            for (int i = 0; i < a.r; ++i) l = __fmaf_rn(tr[i], bf16lo_to_f32(br[i]), l);
                            v = __fmaf_rn(a.s, l, v);
                        }
                        a.Y[m * a.N + nn] = (uint16_t)(pack_bf16x2(v, 0.f) & 0xffffu);
                    }
                }
            continue;
        }
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int64_t m = mt * 16 + g + (e >> 1) * 8, nn = r0 + (e & 1);
                if (m < a.M && nn < a.N) a.part[(ks * a.M + m) * a.N + nn] = acc[mt][e];
            }
        __threadfence();
        __syncwarp();
        int last = 0;
        if (lane == 0) last = (atomicAdd(a.counters + rg, 1) == a.KS - 1);
        last = __shfl_sync(0xffffffffu, last, 0);
        if (!last) continue;
        __threadfence();
        // the last warp of the group: sum the splits in order, add the LoRA term, write Y
        for (int idx = lane; idx < 8 * a.M; idx += 32) {
            const int64_t m = idx >> 3, nn = rg * 8 + (idx & 7);
            if (nn >= a.N) continue;
            float v = 0.f;
            for (int k2 = 0; k2 < a.KS; ++k2) v += __ldcg(a.part + (k2 * a.M + m) * a.N + nn);
            if (a.T32 != nullptr) {
                const float* tr = a.T32 + m * a.rp;
                const uint16_t* br = a.B + nn * a.r;
                float l = 0.f;
                for (int i = 0; i < a.r; ++i) l = __fmaf_rn(tr[i], bf16lo_to_f32(br[i]), l);
                v = __fmaf_rn(a.s, l, v);
            }
            a.Y[m * a.N + nn] = (uint16_t)(pack_bf16x2(v, 0.f) & 0xffffu);
        }
        if (lane == 0) a.counters[rg] = 0;           // ready for the next call
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
    int64_t rows_per_split;   // multiple of 256
    int S;
};

constexpr int kBwdThreads = 256;
constexpr int kBwdWarps = kBwdThreads / 32;
constexpr int kBwdChunk = 256;        // W rows dequantized per pass (one per thread)
constexpr int kBwdDepth = 4;          // passes whose packed bytes are in flight

// cp.async of the 32 packed bytes of row n, block kb into staging slot `slot`
// of thread tid (zero-filled beyond the split).
__device__ __forceinline__ void bwd_stage(const struct SmallBwdArgs& a, uint8_t* s_stage, int slot, int64_t n,
                                          int64_t n_hi, int64_t kb, int64_t rowbytes, int tid);

__device__ __forceinline__ void bwd_stage(const SmallBwdArgs& a, uint8_t* s_stage, int slot, int64_t n, int64_t n_hi,
                                          int64_t kb, int64_t rowbytes, int tid) {
    const bool v = n < n_hi;
    const uint8_t* src = a.packed + (v ? n * rowbytes + 32 * kb : 0);
    const uint32_t dst = smem_u32(s_stage) + (uint32_t)((slot * kBwdThreads + tid) * 32);
    const int sz = v ? 16 : 0;
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(sz) : "memory");
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst + 16), "l"(src + 16), "r"(sz) : "memory");
}

template <int MT>
constexpr int bwd_small_smem_bytes() {
    // the cross-warp reduction buffer reuses the tile and staging space after the last pass
    return (kBwdChunk * 128 + kBwdDepth * kBwdThreads * 32) > (kBwdWarps * 64 * (16 * MT + 1) * 4)
               ? (kBwdChunk * 128 + kBwdDepth * kBwdThreads * 32)
               : (kBwdWarps * 64 * (16 * MT + 1) * 4);
}

// Backward dX = dY W' (the LoRA term is added by k_bwd_small_finish).  The
// packed bytes are prefetched kBwdDepth passes ahead with cp.async.  Work
// unit = (one 64-wide k-block kb, one split of the N rows).  Per pass of 256
// rows: thread d dequantizes row nc + d, block kb into the swizzled tile
// (16-byte chunk c of tile row r stored at chunk c ^ (r & 7)); then warp w
// multiplies tile rows [32w, 32w+32): dY fragments from global memory, W'
// fragments with ldmatrix.trans, 8 n8-tiles covering the 64 k of the block.
template <int MT>
__global__ void __launch_bounds__(kBwdThreads) k_bwd_small(SmallBwdArgs a, NF4Tables tab) {
    constexpr int MC = 16 * MT;
    constexpr int RS = MC + 1;
    extern __shared__ __align__(1024) uint8_t smem[];
    uint8_t* s_tile = smem;                                               // [256][128 B]
    uint8_t* s_stage = smem + kBwdChunk * 128;                            // [depth][256][32 B]
    float* s_red = reinterpret_cast<float*>(smem);                        // [warps][64][RS], after the passes

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, t = lane & 3;
    const int64_t nblk = a.K / kBlock;
    const int64_t units = nblk * a.S;
    const int64_t rowbytes = a.K / 2;
    const uint32_t tile_base = smem_u32(s_tile);

    for (int64_t u = blockIdx.x; u < units; u += gridDim.x) {
        const int64_t kb = u / a.S, split = u % a.S;
        const int64_t n_lo = split * a.rows_per_split;
        const int64_t n_hi = min(a.N, n_lo + a.rows_per_split);
        for (int64_t mc = 0; mc < a.M; mc += MC) {
            float acc[MT][8][4];
#pragma unroll
            for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                for (int j = 0; j < 8; ++j) acc[mt][j][0] = acc[mt][j][1] = acc[mt][j][2] = acc[mt][j][3] = 0.f;
            // the packed bytes of pass i are copied (cp.async, 32 B per thread into the
            // thread's own staging slot) kBwdDepth passes before pass i is dequantized
            const int64_t npass = cdiv(n_hi - n_lo, kBwdChunk);
#pragma unroll
            for (int u = 0; u < kBwdDepth; ++u) {
                bwd_stage(a, s_stage, u, n_lo + (int64_t)u * kBwdChunk + tid, n_hi, kb, rowbytes, tid);
                asm volatile("cp.async.commit_group;" ::: "memory");
            }
            for (int64_t ip = 0; ip < npass; ++ip) {
                const int64_t nc = n_lo + ip * kBwdChunk;
                const int slot = (int)(ip % kBwdDepth);
                // ---- dequantize row nc + tid, block kb, into the tile
                {
                    const int64_t n = nc + tid;
                    float c = 0.f;
                    if (n < n_hi) c = block_constant(a.codes, a.scale, a.mean, n * nblk + kb);
                    asm volatile("cp.async.wait_group %0;" ::"n"(kBwdDepth - 1) : "memory");
                    uint4 p0, p1;
                    const uint32_t src = smem_u32(s_stage) + (uint32_t)((slot * kBwdThreads + tid) * 32);
                    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(p0.x), "=r"(p0.y), "=r"(p0.z), "=r"(p0.w) : "r"(src));
                    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(p1.x), "=r"(p1.y), "=r"(p1.z), "=r"(p1.w) : "r"(src + 16));
                    // refill this slot with pass ip + kBwdDepth
                    bwd_stage(a, s_stage, slot, nc + (int64_t)kBwdDepth * kBwdChunk + tid, n_hi, kb, rowbytes, tid);
                    asm volatile("cp.async.commit_group;" ::: "memory");
                    const BlockTable tb = make_block_table(tab, c);
                    const uint32_t pw[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
                    const uint32_t row_addr = tile_base + tid * 128;
#pragma unroll
                    for (int ch = 0; ch < 8; ++ch) {
                        uint32_t o[4];
                        decode8(tb, pw[ch], o);
                        const uint32_t addr = row_addr + ((ch ^ (tid & 7)) << 4);
                        asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(addr), "r"(o[0]), "r"(o[1]),
                                     "r"(o[2]), "r"(o[3]));
                    }
                }
                __syncthreads();
                // ---- multiply: warp w takes tile rows [32w, 32w+32)
#pragma unroll
                for (int s2 = 0; s2 < 2; ++s2) {
                    const int rbase = warp * 32 + s2 * 16;
                    const int64_t nA = nc + rbase + 2 * t;          // reduction index of a0 / a1
                    uint32_t af[MT][4];
#pragma unroll
                    for (int mt = 0; mt < MT; ++mt) {
                        const int64_t m0 = mc + mt * 16 + g, m1 = m0 + 8;
                        af[mt][0] = af[mt][1] = af[mt][2] = af[mt][3] = 0u;
                        if (nA < n_hi) {
                            if (m0 < a.M) af[mt][0] = __ldg(reinterpret_cast<const unsigned int*>(a.dY + m0 * a.N + nA));
                            if (m1 < a.M) af[mt][1] = __ldg(reinterpret_cast<const unsigned int*>(a.dY + m1 * a.N + nA));
                        }
                        if (nA + 8 < n_hi) {
                            if (m0 < a.M) af[mt][2] = __ldg(reinterpret_cast<const unsigned int*>(a.dY + m0 * a.N + nA + 8));
                            if (m1 < a.M) af[mt][3] = __ldg(reinterpret_cast<const unsigned int*>(a.dY + m1 * a.N + nA + 8));
                        }
                    }
                    const int mi = lane >> 3, rr = lane & 7;
                    const int row = rbase + (mi & 1) * 8 + rr;
#pragma unroll
                    for (int jp = 0; jp < 4; ++jp) {
                        const int ch = 2 * jp + (mi >> 1);
                        const uint32_t addr = tile_base + row * 128 + ((ch ^ (row & 7)) << 4);
                        uint32_t b00, b01, b10, b11;
                        asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                                     : "=r"(b00), "=r"(b01), "=r"(b10), "=r"(b11) : "r"(addr));
#pragma unroll
                        for (int mt = 0; mt < MT; ++mt) {
                            mma_bf16_16816(acc[mt][2 * jp], af[mt][0], af[mt][1], af[mt][2], af[mt][3], b00, b01);
                            mma_bf16_16816(acc[mt][2 * jp + 1], af[mt][0], af[mt][1], af[mt][2], af[mt][3], b10, b11);
                        }
                    }
                }
                __syncthreads();
            }
            asm volatile("cp.async.wait_group 0;" ::: "memory");
            __syncthreads();
            // acc[mt][j]: c0,c1 -> (token mt*16+g, k 8j+2t, +1), c2,c3 -> (token +8)
            float* red = s_red + warp * 64 * RS;
#pragma unroll
            for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int k0 = 8 * j + 2 * t;
                    red[k0 * RS + mt * 16 + g] = acc[mt][j][0];
                    red[(k0 + 1) * RS + mt * 16 + g] = acc[mt][j][1];
                    red[k0 * RS + mt * 16 + g + 8] = acc[mt][j][2];
                    red[(k0 + 1) * RS + mt * 16 + g + 8] = acc[mt][j][3];
                }
            __syncthreads();
            for (int idx = tid; idx < 64 * MC; idx += kBwdThreads) {
                const int kl = idx & 63, ml = idx >> 6;
                const int64_t m = mc + ml;
                if (m < a.M) {
                    float v = 0.f;
#pragma unroll
                    for (int w = 0; w < kBwdWarps; ++w) v += s_red[w * 64 * RS + kl * RS + ml];
                    a.part[(split * a.M + m) * a.K + kb * 64 + kl] = v;
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
