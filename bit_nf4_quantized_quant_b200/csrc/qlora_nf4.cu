// qlora_nf4.cu -- the extern "C" entry points of libqlora_nf4.so (single
// translation unit: the kernels are pulled in from the .cuh files).
//
// The ABI is documented in include/qlora_nf4.h.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "quant.cuh"
#include "small_lora.cuh"
#include "tcs_gemm.cuh"
#include "gemv_mma.cuh"
#include "lora.cuh"
#include "tc_gemm.cuh"
#include "tc2_gemm.cuh"
#include "merge.cuh"
#include "adamw8.cuh"
#include "skinny.cuh"

using namespace qnf4;

namespace {

// ---------------------------------------------------------------------------
// Codebook on the host: inverse normal CDF by bisection on libm's erfc,
// Phi(x) = erfc(-x / sqrt 2) / 2, to the resolution of a double.  The
// construction of the 16 levels is the one documented at nf4_codebook().
// ---------------------------------------------------------------------------
double phi(double x) { return 0.5 * std::erfc(-x / std::sqrt(2.0)); }

double inv_phi_bisect(double p) {
    double lo = -40.0, hi = 40.0;
    for (int it = 0; it < 2000; ++it) {
        const double mid = 0.5 * (lo + hi);
        if (mid <= lo || mid >= hi) break;
        if (phi(mid) < p) lo = mid; else hi = mid;
    }
    return 0.5 * (lo + hi);
}

// Tables of the two quant types: [0] NF4, [1] FP4 (E2M1).
NF4Tables g_tables[2];
EncTables g_enc[2];
std::once_flag g_tables_once;

// Decision thresholds of a codebook and the encoder buckets over them.
// `sorted` lists the n distinct levels in ascending order; thresholds beyond
// the n - 1 real ones are +inf (the encoder then returns the level's rank,
// which the quantize kernel maps to its nibble).
void build_encoder(NF4Tables& t, EncTables& e, const float* sorted, int n) {
    for (int i = 0; i < 15; ++i) t.m[i] = (i + 1 < n) ? (sorted[i] + sorted[i + 1]) * 0.5f : INFINITY;
    t.pad = 0.f;
    // encoder buckets: bucket b holds x with round(64 x + 64) = b, i.e. x in
    // [(b - 64.5) / 64, (b - 63.5) / 64], widened by eps against rounding
    const double eps = 1.0 / 512.0;
    for (int b = 0; b < kEncBuckets; ++b) {
        const double lo = (b - 64.5) / 64.0 - eps, hi = (b - 63.5) / 64.0 + eps;
        uint32_t below = 0;
        float thr = INFINITY;
        for (int i = 0; i + 1 < n; ++i) {
            const double mi = t.m[i];
            if (mi < lo) ++below;
            else if (mi <= hi) thr = t.m[i];    // at most one (thresholds are >= 0.08 apart)
        }
        e.thr[b] = thr;
        e.qb[b] = below;
    }
}

void init_tables() {
    // NF4: the nibble is the level's rank
    const double delta = 0.5 * ((1.0 - 1.0 / 32.0) + (1.0 - 1.0 / 30.0));
    double pos[8], neg[7];
    for (int i = 0; i < 8; ++i) pos[i] = inv_phi_bisect(delta - (delta - 0.5) * i / 8.0);   // descending
    for (int i = 0; i < 7; ++i) neg[i] = -inv_phi_bisect(delta - (delta - 0.5) * i / 7.0);  // ascending
    double v[16];
    for (int i = 0; i < 7; ++i) v[i] = neg[i];
    v[7] = 0.0;
    for (int i = 0; i < 8; ++i) v[8 + i] = pos[7 - i];
    const double top = v[15];
    for (int i = 0; i < 16; ++i) g_tables[QLORA_QUANT_NF4].L[i] = (float)(v[i] / top);
    build_encoder(g_tables[QLORA_QUANT_NF4], g_enc[QLORA_QUANT_NF4], g_tables[QLORA_QUANT_NF4].L, 16);
    // FP4: nibble = E2M1 bit pattern (bit 3 sign, bits 2..1 exponent with bias 1, bit 0
    // mantissa; exponent 0 is subnormal), divided by the largest magnitude, 6
    float* L = g_tables[QLORA_QUANT_FP4].L;
    for (int code = 0; code < 16; ++code) {
        const int e = (code >> 1) & 3, m = code & 1;
        const double mag = e == 0 ? 0.5 * m : std::ldexp(1.0 + 0.5 * m, e - 1);
        L[code] = (float)((code & 8 ? -mag : mag) / 6.0);
    }
    float sorted[15];
    int n = 0;
    for (int code = 15; code >= 9; --code) sorted[n++] = L[code];    // -1 .. -1/12
    for (int code = 0; code <= 7; ++code) sorted[n++] = L[code];     // 0 .. 1
    build_encoder(g_tables[QLORA_QUANT_FP4], g_enc[QLORA_QUANT_FP4], sorted, n);
}

const NF4Tables& tables(int qt = QLORA_QUANT_NF4) {
    std::call_once(g_tables_once, init_tables);
    return g_tables[qt == QLORA_QUANT_FP4 ? 1 : 0];
}

const EncTables& enc_tables(int qt) {
    std::call_once(g_tables_once, init_tables);
    return g_enc[qt == QLORA_QUANT_FP4 ? 1 : 0];
}

thread_local int t_last_path = 0;

// Kernel launches made by this library (all threads), for benchmarks.
std::atomic<long long> g_launches{0};
inline void note_launch(int n = 1) { g_launches.fetch_add(n, std::memory_order_relaxed); }

// One-shot events recorded around the next fused dequant-GEMM launch.
thread_local cudaEvent_t t_ev_before = nullptr;
thread_local cudaEvent_t t_ev_after = nullptr;

// Under stream capture the record becomes an event-record node of the graph
// (external record), so each replay of the graph re-records it.
inline void record_hook(cudaEvent_t ev, cudaStream_t st) {
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(st, &cs) == cudaSuccess && cs == cudaStreamCaptureStatusActive)
        cudaEventRecordWithFlags(ev, st, cudaEventRecordExternal);
    else
        cudaEventRecord(ev, st);
}
inline void hook_before(cudaStream_t st) {
    if (t_ev_before) record_hook(t_ev_before, st);
}
inline void hook_after(cudaStream_t st) {
    if (t_ev_after) record_hook(t_ev_after, st);
    t_ev_before = nullptr;
    t_ev_after = nullptr;
}

int g_sm_count[64];
std::atomic<int> g_dev_ok[64];   // 0 unknown, 1 sm_100, -1 other

int check_device(int* sm_count) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return QLORA_ERR_DEVICE;
    if (dev < 0 || dev >= 64) return QLORA_ERR_DEVICE;
    int st = g_dev_ok[dev].load();
    if (st == 0) {
        int major = 0, minor = 0, sms = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return QLORA_ERR_DEVICE;
        g_sm_count[dev] = sms;
        st = (major == 10 && minor == 0) ? 1 : -1;
        if (st == 1) {
            // opt in to more than 48 KB of dynamic shared memory, once per device
            const cudaError_t e = [&] {
                cudaError_t r = cudaSuccess;
                // the small adapter kernels run next to (or just before) the fused kernels,
                // which need most of shared memory: keep the SM in its shared-memory-heavy
                // configuration so that the next kernel's CTAs need no reconfiguration
                const void* smalls[] = {(const void*)k_lora_down_small<1>, (const void*)k_lora_down_small<2>,
                                        (const void*)k_lora_down_small<4>, (const void*)gmv::k_nf4_gemv_finish<1>,
                                        (const void*)gmv::k_nf4_gemv_finish<2>, (const void*)gmv::k_nf4_gemv_finish<4>,
                                        (const void*)gmv::k_nf4_gemv_finish<8>,
                                        (const void*)k_lora_bwd_small, (const void*)k_bwd_small_end};
                for (const void* f : smalls)
                    if (r == cudaSuccess)
                        r = cudaFuncSetAttribute(f, cudaFuncAttributePreferredSharedMemoryCarveout,
                                                 (int)cudaSharedmemCarveoutMaxShared);
                return r;
            }();
            if (e != cudaSuccess) return QLORA_ERR_LAUNCH;
        }
        g_dev_ok[dev].store(st);
    }
    if (st != 1) return QLORA_ERR_DEVICE;
    if (sm_count) *sm_count = g_sm_count[dev];
    return QLORA_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int launch_status() {
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? QLORA_OK : QLORA_ERR_LAUNCH;
}

// Launch with programmatic stream serialization: the kernel may start while
// the kernel before it on the stream is still running (that kernel calls
// grid_dep_launch() first; this one calls grid_dep_wait() before it reads
// anything the other writes).
template <typename... KArgs, typename... Args>
int launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, Args... args) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, args...);
    note_launch();
    return e == cudaSuccess ? QLORA_OK : QLORA_ERR_LAUNCH;
}

// ---------------------------------------------------------------------------
// Workspace plan: every region 256-byte aligned; regions used one after the
// other on a stream may share the "partials" region.
// ---------------------------------------------------------------------------
struct Plan {
    int64_t M, N, K;
    int r, rp, lw;                  // lw: columns of the scaled hi | lo LoRA activation
    // split-K choices
    int zT, zU, zA, zB;
    int64_t kT, kU, kA, kB;         // k per split
    int US;                         // small-path U = dY B: N splits
    int64_t rows_u;                 //   rows of B per split
    int NT;                         // small-path token tile (16 or 32; 8 more for the forward GEMV)
    int TKC;                        // small-path forward: K splits of T = X A^T
    // byte offsets
    size_t off_slots, off_Upart, off_part, off_T32, off_U32, off_Tp, off_Ubf, off_sT, off_sU, off_Bp, total;
    // stream-K SM-pair kernel: partial tiles and per-(tile, CTA, warp) counters
    size_t off_skpart, sk_part_bytes, off_skflags, sk_flag_bytes;
};

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// Tile of the skinny GEMM for an I x J output: (BI, BJ).
void gemm_tile(int64_t I, int64_t J, int64_t* bi, int64_t* bj) {
    if (J <= 16) { *bi = 64; *bj = 16; }
    else if (I <= 16) { *bi = 16; *bj = 64; }
    else { *bi = 64; *bj = 64; }
}

// Bytes of fp32 split-K partials for an I x J output with z splits.
size_t gemm_part_bytes(int64_t I, int64_t J, int z) {
    int64_t bi, bj;
    gemm_tile(I, J, &bi, &bj);
    return (size_t)z * rup(I, bi) * rup(J, bj) * 4;
}

int choose_splits(int64_t tiles, int64_t kd, int64_t target) {
    int64_t z = cdiv(target, tiles > 0 ? tiles : 1);
    const int64_t zmax = cdiv(kd, 256);
    if (z > zmax) z = zmax;
    if (z < 1) z = 1;
    return (int)z;
}

// Token tiles of 256 per SM-pair tile: 2 when a decoded W' stage can feed two
// of them (halving the decode work per flop) without losing more to wave
// quantization than that gains.  Measured on the 7B block at M = 2048: a
// two-tile tile runs 1.2x the flop rate of a one-tile tile, so a wave of them
// costs about 5/3 of a one-tile wave.
int tc2_token_tiles(int64_t M, int64_t n_out, int pairs) {
    const int64_t m1 = cdiv(M, tc2::BM), m2 = cdiv(M, 2 * tc2::BM), nt = cdiv(n_out, tc2::BN);
    if (m1 < 2 || pairs <= 0) return 1;
    const int64_t w1 = cdiv(m1 * nt, pairs), w2 = cdiv(m2 * nt, pairs);
    return 5 * w2 <= 3 * w1 ? 2 : 1;
}

// SM pairs of a B200; the stream-K workspace is sized for this many.
constexpr int kSkMaxPairs = 74;

// Padded ranks the cluster-reduced adapter kernels take (larger ones: split-K + finish).
constexpr int kSkMaxRp = 64;

// Schedule of the SM-pair kernel for an n_out-wide output on `pairs` pairs: token
// tiles per W' stage (mt) and whether the (tile, step) units are dealt stream-K.
// Stream-K when whole tiles would leave a partial wave and there are at least a
// third as many tiles as pairs (fewer: tiles split more than three ways, whose
// owner adds more partial sums than the split gains), but whole tiles are kept
// where they fill at least three quarters of the pairs without covering them: the
// drain of a split tile's partial sums and the owner's fix-up cost more than the
// idle pairs (7B block at 2048 tokens, 64 tiles of its 4096-wide forwards on 74
// pairs: 1.477 -> 1.430 ms a step on one box), and in the backward the pairs left
// free run dB and dA beside it.
// A product that the wave rule leaves at one token tile takes two, and stream-K
// over all pairs, where two-token-tile tiles still number at least a third of the
// pairs: a one-token-tile step is bound by its decode (each decoded stage feeds one
// token tile; 0.49 of the burst peak against 0.75 with two, measured), which costs
// more than the partial sums of tiles split two or three ways and, in the backward,
// than running dB and dA after the fused kernel instead of beside it (70B
// projections at 512 tokens on one box: 1040 -> 1091 TFLOP/s with the forward
// promoted, 1091 -> 1180 with the backward too).
struct Tc2Sched {
    int mt;
    bool sk;
    int64_t ntiles;
};

Tc2Sched tc2_schedule(int64_t M, int64_t n_out, int pairs, bool bwd) {
    Tc2Sched sc{};
    sc.mt = tc2_token_tiles(M, n_out, pairs);
    const int64_t nt = cdiv(n_out, tc2::BN);
    const bool promote = pairs > 0 && sc.mt == 1 && cdiv(M, (int64_t)tc2::BM) >= 2 &&
                         3 * cdiv(M, 2 * (int64_t)tc2::BM) * nt >= pairs;
    if (promote) sc.mt = 2;
    sc.ntiles = cdiv(M, (int64_t)tc2::BM * sc.mt) * nt;
    sc.sk = pairs > 0 && pairs <= kSkMaxPairs && sc.ntiles % pairs != 0 && 3 * sc.ntiles >= pairs &&
            (promote || sc.ntiles > pairs || 4 * sc.ntiles < 3 * (int64_t)pairs);
    return sc;
}

// Stream-K workspace of one schedule: partial tiles (one slot per pair, 2 CTAs x
// mt x 128 rows x 256 fp32) and counters (tile x 2 CTAs x 4 epilogue warps).
size_t sk_part_bytes(const Tc2Sched& sc, int pairs) {
    return sc.sk ? (size_t)pairs * 2 * sc.mt * tc2::HM * tc2::BN * 4 : 0;
}
size_t sk_flag_bytes(const Tc2Sched& sc) { return sc.sk ? (size_t)sc.ntiles * 8 * 4 : 0; }

// CTAs of the small-M tcgen05 kernel: at most one per SM of a B200.
constexpr int64_t kMaxCtas = 148;

Plan make_plan(int64_t M, int64_t N, int64_t K, int r, int sms) {
    Plan p{};
    p.M = M; p.N = N; p.K = K; p.r = r;
    p.rp = (int)rup(r, 16);
    p.lw = (int)rup(2 * p.rp, 64);
    const int64_t target = 4 * (int64_t)sms;      // split-K: ~4 CTAs of the memory-bound adapter GEMMs per SM
    const int64_t bj = p.rp == 16 ? 16 : 64;
    // T = X A^T: I = M (BI 64), J = rp, Kd = K
    p.zT = choose_splits(cdiv(M, 64) * cdiv(p.rp, bj), K, target);
    p.kT = rup(cdiv(K, p.zT), 32);
    p.zT = (int)cdiv(K, p.kT);
    // U = dY B: Kd = N
    p.zU = choose_splits(cdiv(M, 64) * cdiv(p.rp, bj), N, target);
    p.kU = rup(cdiv(N, p.zU), 32);
    p.zU = (int)cdiv(N, p.kU);
    // dA = U^T X: I = rp, J = K (BJ 64), Kd = M
    const int64_t bi = p.rp == 16 ? 16 : 64;
    p.zA = choose_splits(cdiv(p.rp, bi) * cdiv(K, 64), M, target);
    p.kA = rup(cdiv(M, p.zA), 32);
    p.zA = (int)cdiv(M, p.kA);
    // dB = dY^T T: I = N (BI 64), J = rp, Kd = M
    p.zB = choose_splits(cdiv(N, 64) * cdiv(p.rp, bj), M, target);
    p.kB = rup(cdiv(M, p.zB), 32);
    p.zB = (int)cdiv(M, p.kB);
    // small-path U partials: up to 64 splits of at least 128 rows
    {
        int64_t us = cdiv(N, 128);
        if (us > 64) us = 64;
        p.rows_u = rup(cdiv(N, us), 8);
        p.US = (int)cdiv(N, p.rows_u);
    }
    // regions of the path this M takes (the other path's are left empty)
    const bool small = M <= 32;
    size_t part = 0;
    auto upd = [&](size_t b) { if (b > part) part = b; };
    if (small) {
    } else {
        upd(gemm_part_bytes(M, p.rp, p.zT));
        upd(gemm_part_bytes(M, p.rp, p.zU));
        upd(gemm_part_bytes(2 * p.rp, K, p.zA));
        upd(gemm_part_bytes(N, 2 * p.rp, p.zB));
    }
    // small path: partial tiles of the stream-K kernels, 128 x NT fp32 each, one per
    // (CTA + tile) for the backward and per (CTA + tile, group) for the forward GEMV
    size_t slots = 0;
    p.NT = M <= 16 ? 16 : 32;
    if (small) {
        {
            const int64_t tiles = cdiv(K, tcs::TR), units = tiles * cdiv(N, tcs::KSTEP);
            const int64_t ctas = units < kMaxCtas ? units : kMaxCtas;
            slots = (size_t)(ctas + tiles) * p.NT * tcs::TR * 4;
        }
        {
            const int64_t tiles = cdiv(N, gmv::TR), units = tiles * cdiv(K, gmv::KSTEP);
            const int64_t ctas = units < kMaxCtas ? units : kMaxCtas;
            const size_t b = (size_t)(ctas + tiles) * 2 * p.NT * gmv::TR * 4;
            if (b > slots) slots = b;
        }
    }
    const size_t big = small ? 0 : 1;
    size_t off = 0;
    auto take = [&](size_t b) { const size_t o = off; off = align256(off + b); return o; };
    p.off_slots = take(slots);
    p.off_Upart = take(small ? (size_t)p.US * M * p.rp * 4 : 0);
    p.off_part = take(part);
    p.TKC = small ? (int)down_splits(K) : 1;
    p.off_T32 = take((size_t)p.TKC * M * p.rp * 4);
    p.off_U32 = take(big * M * p.rp * 4);
    p.off_Tp = take(big * M * 2 * p.rp * 2);     // T hi | lo
    p.off_Ubf = take(big * M * 2 * p.rp * 2);    // U hi | lo
    p.off_sT = take(big * M * p.lw * 2);
    p.off_sU = take(big * M * p.lw * 2);
    p.off_Bp = take(big * N * p.rp * 2);
    p.sk_part_bytes = p.sk_flag_bytes = 0;
    if (M > 128) {                      // the SM-pair kernel's path (kPairMinM)
        for (const Tc2Sched& sc : {tc2_schedule(M, N, kSkMaxPairs, false), tc2_schedule(M, K, kSkMaxPairs, true)}) {
            if (sk_part_bytes(sc, kSkMaxPairs) > p.sk_part_bytes) p.sk_part_bytes = sk_part_bytes(sc, kSkMaxPairs);
            if (sk_flag_bytes(sc) > p.sk_flag_bytes) p.sk_flag_bytes = sk_flag_bytes(sc);
        }
    }
    p.off_skpart = take(p.sk_part_bytes);
    p.off_skflags = take(p.sk_flag_bytes);
    p.total = off;
    return p;
}

int grid_for(int64_t work, int per, int sms, int64_t cap_mult = 8) {
    int64_t g = cdiv(work, per);
    if (g > (int64_t)sms * cap_mult) g = (int64_t)sms * cap_mult;
    if (g < 1) g = 1;
    return (int)g;
}

// Split-K skinny GEMM + finish.
template <bool AK, bool BK>
int run_gemm(const uint16_t* A, int64_t lda, const uint16_t* B, int64_t ldb, int64_t I, int64_t J, int64_t Kd,
             int64_t Ilim, int64_t Jlim, int z, int64_t kps, float* part, const FinishArgs& fin_in, int sms,
             cudaStream_t st) {
    GemmArgs g{};
    g.A = A; g.B = B; g.C = part; g.lda = lda; g.ldb = ldb;
    g.Kd = Kd; g.Ilim = Ilim; g.Jlim = Jlim; g.k_per_split = kps;
    FinishArgs f = fin_in;
    f.C = part; f.splits = z;
    int64_t bi, bj;
    gemm_tile(I, J, &bi, &bj);
    g.I = rup(I, bi); g.J = rup(J, bj);
    dim3 grid((unsigned)(g.I / bi), (unsigned)(g.J / bj), (unsigned)z);
    int rc;
    if (bj == 16) rc = launch_pdl(k_gemm_mma<AK, BK, 64, 16, 4, 1>, grid, dim3(128), 0, st, g);
    else if (bi == 16) rc = launch_pdl(k_gemm_mma<AK, BK, 16, 64, 1, 4>, grid, dim3(128), 0, st, g);
    else rc = launch_pdl(k_gemm_mma<AK, BK, 64, 64, 2, 2>, grid, dim3(128), 0, st, g);
    if (rc != QLORA_OK) return rc;
    f.I = g.I; f.J = g.J;
    if (f.Iout > I) f.Iout = I;
    return launch_pdl(k_gemm_finish, dim3((unsigned)grid_for(f.Iout * f.Jiter, 256, sms)), dim3(256), 0, st, f);
}

FinishArgs fin_none() {
    FinishArgs f{};
    f.pre = 1.f;
    return f;
}

int validate_weight(const nf4dq_weight* w) {
    if (!w || !w->packed || !w->codes || !w->scale || !w->mean) return QLORA_ERR_NULL;
    if (w->quant_type != QLORA_QUANT_NF4 && w->quant_type != QLORA_QUANT_FP4) return QLORA_ERR_VALUE;
    if (w->N <= 0 || w->K <= 0 || (w->K % kBlock) != 0 || (w->N % 8) != 0) return QLORA_ERR_SHAPE;
    if (w->K > QLORA_MAX_K) return QLORA_ERR_SHAPE;      // grid y of the K-wide adapter products
    if (w->N > (int64_t)1 << 31 || w->K > (int64_t)1 << 31 || w->N * w->K >= ((int64_t)1 << 38)) return QLORA_ERR_SHAPE;
    if (!aligned16(w->packed)) return QLORA_ERR_ALIGN;
    const uintptr_t lo = reinterpret_cast<uintptr_t>(w->codes) | reinterpret_cast<uintptr_t>(w->scale) |
                         reinterpret_cast<uintptr_t>(w->mean);
    if ((lo & 3u) != 0) return QLORA_ERR_ALIGN;
    return QLORA_OK;
}

// ---------------------------------------------------------------------------
// TMA tensor maps (driver entry point fetched through the runtime, so the
// library does not link libcuda directly)
// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    });
    return fn;
}

// 2-D row-major tensor [outer, inner] with the given row pitch; box [box_outer, box_inner].
bool make_map_2d(CUtensorMap* m, CUtensorMapDataType dt, const void* ptr, uint64_t inner, uint64_t outer,
                 uint64_t pitch_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle sw) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {inner, outer};
    const cuuint64_t strides[1] = {pitch_bytes};
    const cuuint32_t box[2] = {box_inner, box_outer};
    const cuuint32_t estr[2] = {1, 1};
    return fn(m, dt, 2, const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool g_tc_attr_set[64];
int g_pairs[64];            // co-resident SM pairs for the cta_group::2 kernel (0: not available)
std::mutex g_tc_mu;

int ensure_tc_attrs() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return QLORA_ERR_DEVICE;
    std::lock_guard<std::mutex> lk(g_tc_mu);
    if (!g_tc_attr_set[dev]) {
        if (cudaFuncSetAttribute(tc::k_tc_gemm<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, tc::SMEM_ALLOC) !=
                cudaSuccess ||
            cudaFuncSetAttribute(tc::k_tc_gemm<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, tc::SMEM_ALLOC) !=
                cudaSuccess ||
            cudaFuncSetAttribute(tc2::k_tc2_gemm<false, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 tc2::Lay<1>::SMEM_ALLOC) != cudaSuccess ||
            cudaFuncSetAttribute(tc2::k_tc2_gemm<true, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 tc2::Lay<1>::SMEM_ALLOC) != cudaSuccess ||
            cudaFuncSetAttribute(tc2::k_tc2_gemm<false, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 tc2::Lay<2>::SMEM_ALLOC) != cudaSuccess ||
            cudaFuncSetAttribute(tc2::k_tc2_gemm<true, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 tc2::Lay<2>::SMEM_ALLOC) != cudaSuccess ||
            cudaFuncSetAttribute(tcs::k_tcs_gemm<16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 tcs::SMEM_ALLOC) != cudaSuccess ||
            cudaFuncSetAttribute(tcs::k_tcs_gemm<32>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 tcs::SMEM_ALLOC) != cudaSuccess)
            return QLORA_ERR_LAUNCH;
        // pairs of SMs that can hold one cluster each at the same time
        cudaLaunchConfig_t cfg = {};
        cudaLaunchAttribute attr;
        attr.id = cudaLaunchAttributeClusterDimension;
        attr.val.clusterDim.x = 2; attr.val.clusterDim.y = 1; attr.val.clusterDim.z = 1;
        cfg.gridDim = dim3(2 * 74, 1, 1);
        cfg.blockDim = dim3(tc2::kThreads, 1, 1);
        cfg.dynamicSmemBytes = tc2::Lay<1>::SMEM_ALLOC;
        cfg.attrs = nullptr;
        cfg.numAttrs = 0;               // the kernel carries its cluster shape (__cluster_dims__)
        int nclusters = 0;
        if (cudaOccupancyMaxActiveClusters(&nclusters, tc2::k_tc2_gemm<false, 1>, &cfg) != cudaSuccess) {
            cudaGetLastError();
            cfg.attrs = &attr;
            cfg.numAttrs = 1;
            if (cudaOccupancyMaxActiveClusters(&nclusters, tc2::k_tc2_gemm<false, 1>, &cfg) != cudaSuccess) {
                cudaGetLastError();
                nclusters = 0;
            }
        }
        g_pairs[dev] = nclusters;
        g_tc_attr_set[dev] = true;
    }
    return QLORA_OK;
}

// Fused dequant-GEMM on the tcgen05 path.  act [M, n_red] bf16 activations,
// lact [M, lw] bf16 scaled LoRA activations as hi | lo halves of rp = rup(r, 16)
// columns each (lw = rup(2 rp, 64)), lora_w / ldl the LoRA weight
// rows (B for the forward, A for the backward).
template <bool BWD>
int launch_tc(const nf4dq_weight* w, const uint16_t* act, int64_t M, const uint16_t* lact, int lw,
              const uint16_t* lora_w, int64_t ldl, int r, uint16_t* out, int sms, cudaStream_t st,
              bool lora = true) {
    int rc = ensure_tc_attrs();
    if (rc != QLORA_OK) return rc;
    const int64_t N = w->N, K = w->K;
    const int64_t n_red = BWD ? N : K, n_out = BWD ? K : N;
    CUtensorMap tmA, tmL, tmP;
    if (!make_map_2d(&tmA, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, act, n_red, M, n_red * 2, 64, 128,
                     CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map_2d(&tmL, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, lact, lw, M, (uint64_t)lw * 2, 64, 128,
                     CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map_2d(&tmP, CU_TENSOR_MAP_DATA_TYPE_UINT8, w->packed, K / 2, N, K / 2, BWD ? 128 : 32,
                     BWD ? 64 : 256, BWD ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_32B))
        return QLORA_ERR_LAUNCH;
    tc::Args a{};
    a.codes = w->codes; a.scale = w->scale; a.mean = w->mean;
    a.lora_w = lora_w; a.ldl = ldl; a.r = r; a.lper = (int)rup(r, 16); a.nlora = lora ? (int)cdiv(lw, 64) : 0;
    a.out = out; a.M = M; a.N = N; a.K = K; a.n_out = n_out; a.n_red = n_red;
    const int64_t ntiles = cdiv(M, tc::BM) * cdiv(n_out, tc::BN);
    const int grid = (int)(ntiles < sms ? ntiles : sms);
    hook_before(st);
    tc::k_tc_gemm<BWD><<<grid, tc::kThreads, tc::SMEM_ALLOC, st>>>(tmA, tmL, tmP, a, tables(w->quant_type));
    hook_after(st);
    note_launch();
    return launch_status();
}


// The same on SM pairs (cta_group::2), 256 x 256 tiles.
template <bool BWD>
int launch_tc2(const nf4dq_weight* w, const uint16_t* act, int64_t M, const uint16_t* lact, int lw,
               const uint16_t* lora_w, int64_t ldl, int r, uint16_t* out, int pairs, cudaStream_t st,
               bool lora, const Plan& p, uint8_t* wsb) {
    const int64_t N = w->N, K = w->K;
    const int64_t n_red = BWD ? N : K, n_out = BWD ? K : N;
    CUtensorMap tmA, tmL, tmP;
    if (!make_map_2d(&tmA, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, act, n_red, M, n_red * 2, 64, 128,
                     CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map_2d(&tmL, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, lact, lw, M, (uint64_t)lw * 2, 64, 128,
                     CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map_2d(&tmP, CU_TENSOR_MAP_DATA_TYPE_UINT8, w->packed, K / 2, N, K / 2, BWD ? 64 : 32,
                     BWD ? 64 : 128, BWD ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B))
        return QLORA_ERR_LAUNCH;
    tc::Args a{};
    a.codes = w->codes; a.scale = w->scale; a.mean = w->mean;
    a.lora_w = lora_w; a.ldl = ldl; a.r = r; a.lper = (int)rup(r, 16); a.nlora = lora ? (int)cdiv(lw, 64) : 0;
    a.out = out; a.M = M; a.N = N; a.K = K; a.n_out = n_out; a.n_red = n_red;
    Tc2Sched sc = tc2_schedule(M, n_out, pairs, BWD);
    // the counters were zeroed by the kernel before this one (the T or U product), or below
    if (sc.sk && (sk_part_bytes(sc, pairs) > p.sk_part_bytes || sk_flag_bytes(sc) > p.sk_flag_bytes)) sc.sk = false;
    a.sk = sc.sk ? 1 : 0;
    a.part = reinterpret_cast<float*>(wsb + p.off_skpart);
    a.flags = reinterpret_cast<int*>(wsb + p.off_skflags);
    if (sc.sk && p.rp > kSkMaxRp &&         // the split-K adapter kernels do not zero the counters
        cudaMemsetAsync(a.flags, 0, sk_flag_bytes(sc), st) != cudaSuccess)
        return QLORA_ERR_LAUNCH;
    const int mt = sc.mt;
    const int np = sc.sk ? pairs : (int)(sc.ntiles < pairs ? sc.ntiles : pairs);
    // launched with programmatic serialization behind the T or U row kernel (see the
    // kernel), which lets it start only after its own wait; the split-K adapter kernels
    // of larger ranks let the next kernel start before theirs, so there it is a plain launch
    const bool pdl = p.rp <= kSkMaxRp;
    hook_before(st);
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)(2 * np));
    cfg.blockDim = dim3(tc2::kThreads);
    cfg.dynamicSmemBytes = mt == 2 ? tc2::Lay<2>::SMEM_ALLOC : tc2::Lay<1>::SMEM_ALLOC;
    cfg.stream = st;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = pdl ? 1 : 0;
    const NF4Tables tb = tables(w->quant_type);
    const cudaError_t e = mt == 2 ? cudaLaunchKernelEx(&cfg, tc2::k_tc2_gemm<BWD, 2>, tmA, tmL, tmP, a, tb)
                                  : cudaLaunchKernelEx(&cfg, tc2::k_tc2_gemm<BWD, 1>, tmA, tmL, tmP, a, tb);
    hook_after(st);
    note_launch();
    return e == cudaSuccess ? QLORA_OK : QLORA_ERR_LAUNCH;
}

// Tokens above this count use the SM-pair kernel.
constexpr int64_t kPairMinM = 128;

int current_pairs() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
    return g_pairs[dev];
}

// ---------------------------------------------------------------------------
// Cluster-reduced adapter products (sk::k_rowk / sk::k_colk, padded rank <= 64)
// ---------------------------------------------------------------------------
bool g_sk_attr_set[64];

int ensure_sk_attrs() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return QLORA_ERR_DEVICE;
    std::lock_guard<std::mutex> lk(g_tc_mu);
    if (!g_sk_attr_set[dev]) {
        const cudaFuncAttribute at = cudaFuncAttributeMaxDynamicSharedMemorySize;
        if (cudaFuncSetAttribute(sk::k_rowk<0, 16>, at, sk::Lay<16>::SMEM_ALLOC) != cudaSuccess ||
            cudaFuncSetAttribute(sk::k_rowk<0, 32>, at, sk::Lay<32>::SMEM_ALLOC) != cudaSuccess ||
            cudaFuncSetAttribute(sk::k_rowk<0, 64>, at, sk::Lay<64>::SMEM_ALLOC) != cudaSuccess ||
            cudaFuncSetAttribute(sk::k_rowk<1, 16>, at, sk::Lay<16>::SMEM_ALLOC) != cudaSuccess ||
            cudaFuncSetAttribute(sk::k_rowk<1, 32>, at, sk::Lay<32>::SMEM_ALLOC) != cudaSuccess ||
            cudaFuncSetAttribute(sk::k_rowk<1, 64>, at, sk::Lay<64>::SMEM_ALLOC) != cudaSuccess ||
            cudaFuncSetAttribute(sk::k_colk<16>, at, sk::Lay<16>::SMEM_ALLOC) != cudaSuccess ||
            cudaFuncSetAttribute(sk::k_colk<32>, at, sk::Lay<32>::SMEM_ALLOC) != cudaSuccess ||
            cudaFuncSetAttribute(sk::k_colk<64>, at, sk::Lay<64>::SMEM_ALLOC) != cudaSuccess ||
            cudaFuncSetAttribute(sk::k_colk<128>, at, sk::Lay<128>::SMEM_ALLOC) != cudaSuccess)
            return QLORA_ERR_LAUNCH;
        g_sk_attr_set[dev] = true;
    }
    return QLORA_OK;
}


int sk_jq(int64_t cols) { return cols <= 16 ? 16 : cols <= 32 ? 32 : cols <= 64 ? 64 : 128; }

CUtensorMapSwizzle sk_swizzle(int span) {
    return span >= 128 ? CU_TENSOR_MAP_SWIZZLE_128B : span == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                                                 : CU_TENSOR_MAP_SWIZZLE_32B;
}

// Cluster size: at most one wave of CTAs (smem_per_cta decides how many an SM
// holds, at most 3), and at least 4 reduction tiles per rank.
int sk_cluster(int64_t tiles, int64_t nred, int smem_per_cta, int sms) {
    int per_sm = 232448 / smem_per_cta;
    if (per_sm > 3) per_sm = 3;
    if (per_sm < 1) per_sm = 1;
    const int64_t slots = (int64_t)sms * per_sm;
    int z = sk::kMaxCluster;
    while (z > 1 && (tiles * z > slots || cdiv(nred, z) < 4)) z >>= 1;
    return z;
}

template <typename... KArgs>
int launch_sk(void (*kern)(KArgs...), int z, int64_t tiles, int smem, cudaStream_t st, const CUtensorMap& tmP,
              const CUtensorMap& tmQ, const sk::Args& a) {
    const int64_t ctas = tiles * z;
    if (ctas > 0x7fffffffLL) return QLORA_ERR_SHAPE;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)ctas, 1, 1);
    cfg.blockDim = dim3(sk::kThreads, 1, 1);
    cfg.dynamicSmemBytes = (size_t)smem;
    cfg.stream = st;
    cudaLaunchAttribute at[2];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = (unsigned)z; at[0].val.clusterDim.y = 1; at[0].val.clusterDim.z = 1;
    at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 2;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, tmP, tmQ, a);
    note_launch();
    return e == cudaSuccess ? QLORA_OK : QLORA_ERR_LAUNCH;
}

// out [M, rp] = P [M, L] . Q with the outputs of f (rows i < M, columns
// j < f.Jiter; f.J = rp).  qt 0: Q^T = A [qn, L] (A's rows, pitch ldq);
// qt 1: Q = B [L, qn] (qn columns, pitch ldq).
int run_rowk(const uint16_t* P, int64_t M, int64_t L, const uint16_t* Q, int qt, int64_t qn, int64_t ldq, int rp,
             FinishArgs f, int sms, cudaStream_t st, int* zero = nullptr, int64_t nzero = 0) {
    int rc = ensure_sk_attrs();
    if (rc != QLORA_OK) return rc;
    const int jq = sk_jq(rp);
    CUtensorMap tmP, tmQ;
    bool ok = make_map_2d(&tmP, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, P, L, M, L * 2, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B);
    if (qt == 0)
        ok = ok && make_map_2d(&tmQ, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, Q, L, qn, ldq * 2, 64, jq,
                               CU_TENSOR_MAP_SWIZZLE_128B);
    else
        ok = ok && make_map_2d(&tmQ, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, Q, qn, L, ldq * 2, jq, 64,
                               sk_swizzle(jq * 2));
    if (!ok) return QLORA_ERR_LAUNCH;
    f.J = rp;
    sk::Args a{};
    a.M = M; a.L = L; a.nred = cdiv(L, sk::TILE); a.f = f;
    a.zero = zero; a.nzero = zero ? nzero : 0;
    const int64_t tiles = cdiv(M, sk::TILE);
    const int smem = jq == 16 ? sk::Lay<16>::SMEM_ALLOC : jq == 32 ? sk::Lay<32>::SMEM_ALLOC : sk::Lay<64>::SMEM_ALLOC;
    const int z = sk_cluster(tiles, a.nred, smem, sms);
    a.ns = (int)cdiv(a.nred, z);
    if (qt == 0) {
        if (jq == 16) return launch_sk(sk::k_rowk<0, 16>, z, tiles, smem, st, tmP, tmQ, a);
        if (jq == 32) return launch_sk(sk::k_rowk<0, 32>, z, tiles, smem, st, tmP, tmQ, a);
        return launch_sk(sk::k_rowk<0, 64>, z, tiles, smem, st, tmP, tmQ, a);
    }
    if (jq == 16) return launch_sk(sk::k_rowk<1, 16>, z, tiles, smem, st, tmP, tmQ, a);
    if (jq == 32) return launch_sk(sk::k_rowk<1, 32>, z, tiles, smem, st, tmP, tmQ, a);
    return launch_sk(sk::k_rowk<1, 64>, z, tiles, smem, st, tmP, tmQ, a);
}

// out (l, j) = sum_m P [m, l] Q [m, j] (+ the same at column j + pair) for
// j < jout, written by finish_store as element (l, j), or (j, l) with trans_out.
// Q [M, qn] with pitch ldq; qn <= 128.
int run_colk(const uint16_t* P, int64_t M, int64_t L, const uint16_t* Q, int64_t qn, int64_t ldq, int pair,
             int jout, bool trans_out, FinishArgs f, int sms, cudaStream_t st, bool wait_end = false) {
    int rc = ensure_sk_attrs();
    if (rc != QLORA_OK) return rc;
    const int jq = sk_jq(qn);
    const int box = jq > 64 ? 64 : jq;
    CUtensorMap tmP, tmQ;
    if (!make_map_2d(&tmP, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, P, L, M, L * 2, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map_2d(&tmQ, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, Q, qn, M, ldq * 2, box, 64, sk_swizzle(box * 2)))
        return QLORA_ERR_LAUNCH;
    sk::Args a{};
    a.M = M; a.L = L; a.nred = cdiv(M, sk::TILE); a.pair = pair; a.jout = jout; a.trans_out = trans_out ? 1 : 0;
    a.wait_end = wait_end ? 1 : 0;
    a.f = f;
    const int64_t tiles = cdiv(L, sk::TILE);
    const int smem = jq == 16 ? sk::Lay<16>::SMEM_ALLOC : jq == 32 ? sk::Lay<32>::SMEM_ALLOC
                   : jq == 64 ? sk::Lay<64>::SMEM_ALLOC : sk::Lay<128>::SMEM_ALLOC;
    const int z = sk_cluster(tiles, a.nred, smem, sms);
    a.ns = (int)cdiv(a.nred, z);
    if (jq == 16) return launch_sk(sk::k_colk<16>, z, tiles, smem, st, tmP, tmQ, a);
    if (jq == 32) return launch_sk(sk::k_colk<32>, z, tiles, smem, st, tmP, tmQ, a);
    if (jq == 64) return launch_sk(sk::k_colk<64>, z, tiles, smem, st, tmP, tmQ, a);
    return launch_sk(sk::k_colk<128>, z, tiles, smem, st, tmP, tmQ, a);
}

// Tokens at or below this count take the small-M (GEMV-shaped) kernels.
constexpr int64_t kSmallMaxM = 32;

// T = X A^T: T32 (fp32 [M, rp]), Thl (bf16 hi|lo [M, 2 rp]), sT (bf16 s*T as hi | lo, [M, lw]),
// and the caller's T_out (bf16 [M, r]) when given.
int compute_T(const Plan& p, const uint16_t* X, const uint16_t* A, float s, uint16_t* T_out, uint8_t* ws, int sms,
              cudaStream_t st, float tscale = 1.f) {
    FinishArgs f = fin_none();
    f.pre = tscale;
    f.Iout = p.M; f.Jiter = p.lw;
    f.f32 = reinterpret_cast<float*>(ws + p.off_T32); f.ld_f32 = p.rp; f.Jf = p.rp;
    f.J1 = p.r;
    f.hl = reinterpret_cast<uint16_t*>(ws + p.off_Tp); f.hl_ld = 2 * p.rp; f.hl_off = p.rp;
    f.o2 = reinterpret_cast<uint16_t*>(ws + p.off_sT); f.s2i = p.lw; f.s2j = 1; f.J2 = p.r; f.J2pad = p.lw; f.alpha2 = s;
    f.o2_lo = p.rp;
    if (T_out) {   // the caller's bf16 T [M, r]: the same rounding as the hi half of Thl
        f.o1 = T_out; f.s1i = p.r; f.s1j = 1; f.J1pad = p.r; f.alpha1 = 1.f;
    }
    if (p.rp <= kSkMaxRp)
        return run_rowk(X, p.M, p.K, A, 0, p.r, p.K, p.rp, f, sms, st, reinterpret_cast<int*>(ws + p.off_skflags),
                        (int64_t)(p.sk_flag_bytes / 4));
    return run_gemm<true, true>(X, p.K, A, p.K, p.M, p.rp, p.K, p.M, p.r, p.zT, p.kT,
                                reinterpret_cast<float*>(ws + p.off_part), f, sms, st);
}


// Small-M T = X A^T into T32 (and the caller's bf16 T_out): programmatic
// launch behind the forward GEMV, plain launch in the backward's recompute.
int small_T(const Plan& p, const uint16_t* X, const uint16_t* A, uint16_t* T_out, uint8_t* ws, cudaStream_t st,
            bool pdl) {
    LoraDownArgs d{};
    d.X = X; d.A = A; d.M = p.M; d.K = p.K; d.r = p.r; d.rp = p.rp;
    d.kc = pdl ? p.TKC : 1;             // the forward's split sums are added by the finish kernel
    d.T32 = reinterpret_cast<float*>(ws + p.off_T32);
    d.T_out = pdl ? nullptr : T_out;
    const int mg = p.M <= 1 ? 1 : p.M <= 2 ? 2 : 4;
    const dim3 grid((unsigned)p.r, (unsigned)d.kc, (unsigned)cdiv(p.M, mg)), block(kDownThreads);
    void (*kern)(LoraDownArgs) = mg == 1 ? k_lora_down_small<1> : mg == 2 ? k_lora_down_small<2>
                                : k_lora_down_small<4>;
    if (pdl) return launch_pdl(kern, grid, block, 0, st, d);
    kern<<<grid, block, 0, st>>>(d);
    note_launch();
    return launch_status();
}

// Small-M backward dY W' on tcgen05 (stream-K over one CTA per SM), launched
// programmatically after the U / dB kernel; it leaves partial tiles in the
// workspace for k_bwd_small_end.
int launch_tcs_bwd(const Plan& p, const nf4dq_weight* w, const uint16_t* dY, uint8_t* wsb, int sms, cudaStream_t st,
                   tcs::Args* out) {
    int rc = ensure_tc_attrs();
    if (rc != QLORA_OK) return rc;
    const int64_t M = p.M, N = p.N, K = p.K;
    CUtensorMap tmX, tmP;
    if (!make_map_2d(&tmX, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, dY, N, M, N * 2, 64, p.NT, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map_2d(&tmP, CU_TENSOR_MAP_DATA_TYPE_UINT8, w->packed, K / 2, N, K / 2, 64, tcs::TR,
                     CU_TENSOR_MAP_SWIZZLE_64B))
        return QLORA_ERR_LAUNCH;
    tcs::Args a{};
    a.codes = w->codes; a.scale = w->scale; a.mean = w->mean;
    a.M = M; a.N = N; a.K = K;
    a.tiles = (int)cdiv(K, tcs::TR);
    a.nks = (int)cdiv(N, tcs::KSTEP);
    a.units = (int64_t)a.tiles * a.nks;
    int64_t ctas = sms < kMaxCtas ? sms : kMaxCtas;
    if (ctas > a.units) ctas = a.units;
    a.ctas = (int)ctas;
    a.slots = reinterpret_cast<float*>(wsb + p.off_slots);
    *out = a;
    const dim3 grid((unsigned)ctas), block(tcs::kThreads);
    const NF4Tables& tab = tables(w->quant_type);
    if (p.NT == 16) return launch_pdl(tcs::k_tcs_gemm<16>, grid, block, tcs::SMEM_ALLOC, st, tmX, tmP, a, tab);
    return launch_pdl(tcs::k_tcs_gemm<32>, grid, block, tcs::SMEM_ALLOC, st, tmX, tmP, a, tab);
}

// Small-M forward: the GEMV (mma.sync, stream-K over one CTA per SM), the
// T = X A^T kernel and the finish kernel, all launched programmatically.
template <int NTT>
int launch_gemv_ntt(const Plan& p, const nf4dq_weight* w, const uint16_t* X, const uint16_t* Xl, const uint16_t* A,
                    const uint16_t* B, float s, uint16_t* Y, uint16_t* T_out, uint8_t* wsb, int sms, cudaStream_t st,
                    float tscale) {
    using C = gmv::Cfg<NTT>;
    static bool attr_set[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return QLORA_ERR_DEVICE;
    if (!attr_set[dev]) {
        std::lock_guard<std::mutex> lk(g_tc_mu);
        // the same (shared-memory-heavy) carveout as the small kernels launched beside it,
        // so that their CTAs can share its SMs
        if (cudaFuncSetAttribute(gmv::k_nf4_gemv<NTT>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_ALLOC) !=
                cudaSuccess ||
            cudaFuncSetAttribute(gmv::k_nf4_gemv<NTT>, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 (int)cudaSharedmemCarveoutMaxShared) != cudaSuccess)
            return QLORA_ERR_LAUNCH;
        attr_set[dev] = true;
    }
    const int64_t N = p.N, K = p.K;
    CUtensorMap tmP;
    if (!make_map_2d(&tmP, CU_TENSOR_MAP_DATA_TYPE_UINT8, w->packed, K / 2, N, K / 2, gmv::KSTEP / 2, gmv::TR,
                     CU_TENSOR_MAP_SWIZZLE_128B))
        return QLORA_ERR_LAUNCH;
    gmv::Args a{};
    a.X = X; a.codes = w->codes; a.scale = w->scale; a.mean = w->mean;
    a.M = p.M; a.N = N; a.K = K;
    a.tiles = (int)cdiv(N, gmv::TR);
    a.nks = (int)cdiv(K, gmv::KSTEP);
    a.units = (int64_t)a.tiles * a.nks;
    int64_t ctas = sms < kMaxCtas ? sms : kMaxCtas;
    if (ctas > a.units) ctas = a.units;
    a.ctas = (int)ctas;
    a.slots = reinterpret_cast<float*>(wsb + p.off_slots);
    int rc = launch_pdl(gmv::k_nf4_gemv<NTT>, dim3((unsigned)ctas), dim3(gmv::kThreads), (size_t)C::SMEM_ALLOC, st,
                        tmP, a, tables(w->quant_type));
    if (rc != QLORA_OK) return rc;
    rc = small_T(p, Xl, A, nullptr, wsb, st, true);
    if (rc != QLORA_OK) return rc;
    gmv::FinishArgs f{};
    f.slots = a.slots; f.M = p.M; f.N = N; f.nks = a.nks; f.ctas = a.ctas; f.NT = C::NT; f.units = a.units;
    f.Tpart = reinterpret_cast<const float*>(wsb + p.off_T32); f.kc = p.TKC; f.rp = p.rp; f.r = p.r;
    f.lora_B = B; f.b_vec = (p.r % 8 == 0 && aligned16(B)) ? 1 : 0; f.s = s; f.tscale = tscale; f.Y = Y;
    f.T_out = T_out;
    const int mt = p.M <= 1 ? 1 : p.M <= 2 ? 2 : p.M <= 4 ? 4 : 8;
    void (*fin)(gmv::FinishArgs) = mt == 1 ? gmv::k_nf4_gemv_finish<1> : mt == 2 ? gmv::k_nf4_gemv_finish<2>
                                 : mt == 4 ? gmv::k_nf4_gemv_finish<4> : gmv::k_nf4_gemv_finish<8>;
    return launch_pdl(fin, dim3((unsigned)a.tiles, (unsigned)cdiv(p.M, mt)), dim3(gmv::TR), 0, st, f);
}

// Small-M forward: fused GEMV, T = X A^T beside it, then the finish kernel
// (partial tiles summed, s T B^T added).
int small_fwd(const Plan& p, const uint16_t* X, const uint16_t* Xl, const nf4dq_weight* w, const uint16_t* A,
              const uint16_t* B, float scaling, uint16_t* Y, uint16_t* T_out, uint8_t* wsb, int sms, cudaStream_t st,
              float tscale) {
    hook_before(st);
    int rc;
    if (p.M <= 8) rc = launch_gemv_ntt<1>(p, w, X, Xl, A, B, scaling, Y, T_out, wsb, sms, st, tscale);
    else if (p.M <= 16) rc = launch_gemv_ntt<2>(p, w, X, Xl, A, B, scaling, Y, T_out, wsb, sms, st, tscale);
    else rc = launch_gemv_ntt<4>(p, w, X, Xl, A, B, scaling, Y, T_out, wsb, sms, st, tscale);
    hook_after(st);
    return rc;
}

// Small-M backward: [T], U partials + dB, the fused dY W' kernel (overlapping
// the U / dB kernel), then dX = dY W' + s U A and dA.
int small_bwd(const Plan& p, const uint16_t* Xl, const uint16_t* dY, const nf4dq_weight* w, const uint16_t* A,
              const uint16_t* B, float scaling, const uint16_t* T, uint16_t* dX, uint16_t* dA, uint16_t* dB,
              uint8_t* wsb, int sms, cudaStream_t st, const drop::Params* dp, const uint16_t* mask) {
    int rc = QLORA_OK;
    const float* T32 = nullptr;
    if (T == nullptr) {
        rc = small_T(p, Xl, A, nullptr, wsb, st, false);
        if (rc != QLORA_OK) return rc;
        T32 = reinterpret_cast<const float*>(wsb + p.off_T32);
    }
    hook_before(st);
    LoraBwdArgs b{};
    b.dY = dY; b.B = B; b.T32 = T32; b.Tb = T; b.M = p.M; b.N = p.N; b.r = p.r; b.rp = p.rp; b.s = scaling;
    b.tscale = dp ? dp->c : 1.f;
    b.b_vec = (p.r % 8 == 0 && aligned16(B)) ? 1 : 0;
    b.Upart = reinterpret_cast<float*>(wsb + p.off_Upart); b.US = p.US; b.rows_u = p.rows_u; b.dB = dB;
    k_lora_bwd_small<<<(unsigned)(p.US + cdiv(p.N, kLoraThreads)), kLoraThreads, 0, st>>>(b);
    note_launch();
    rc = launch_status();
    if (rc != QLORA_OK) return rc;
    tcs::Args ta{};
    rc = launch_tcs_bwd(p, w, dY, wsb, sms, st, &ta);
    hook_after(st);
    if (rc != QLORA_OK) return rc;
    BwdEndArgs e{};
    e.slots = ta.slots; e.NT = p.NT; e.nks = ta.nks; e.ctas = ta.ctas; e.units = ta.units;
    e.Upart = b.Upart; e.US = p.US; e.A = A; e.X = Xl;
    if (dp) { e.mask = mask; e.c = dp->c; }
    e.M = p.M; e.K = p.K; e.r = p.r; e.rp = p.rp; e.s = scaling; e.dX = dX; e.dA = dA;
    e.s_da = dp ? (float)((double)scaling * (double)dp->c) : scaling;
    return launch_pdl(k_bwd_small_end, dim3((unsigned)cdiv(p.K, kLoraThreads), (unsigned)(p.M + p.r)),
                      dim3(kLoraThreads), 0, st, e);
}

// Bytes of the dropped copy of X that the dropout entry points need past the
// regular workspace plan.
size_t dropout_bytes(int64_t M, int64_t K) {
    return align256((size_t)M * (size_t)K * 2) + align256((size_t)M * (size_t)K / 8);
}

int dropout_params(float p, uint64_t seed, uint64_t offset, drop::Params* d) {
    if (!(p >= 0.f && p < 1.f)) return QLORA_ERR_VALUE;
    d->seed = seed;
    d->offset = offset;
    d->t = (uint32_t)std::llrint((double)p * 65536.0);
    d->c = (float)(1.0 / (1.0 - (double)p));
    return QLORA_OK;
}

// Xd = X * keep [M, K] into the workspace, and (mask non-null) its keep bits.
int launch_dropout_x(const uint16_t* X, int64_t M, int64_t K, uint8_t* dst, uint16_t* mask, const drop::Params& d,
                     int sms, cudaStream_t st) {
    const int64_t total16 = M * K / 16;
    drop::k_dropout_x<<<grid_for(total16, 256, sms), 256, 0, st>>>(X, total16, reinterpret_cast<uint16_t*>(dst),
                                                                   mask, d);
    note_launch();
    return launch_status();
}

}  // namespace

// ===========================================================================
// extern "C" entry points
// ===========================================================================
extern "C" {

int nf4_codebook(float out16[16]) {
    if (!out16) return QLORA_ERR_NULL;
    const NF4Tables& t = tables();
    for (int i = 0; i < 16; ++i) out16[i] = t.L[i];
    return QLORA_OK;
}

int nf4dq_sizes(int64_t N, int64_t K, int64_t* packed_bytes, int64_t* n_blocks, int64_t* n_groups) {
    if (N <= 0 || K <= 0 || (K % kBlock) != 0) return QLORA_ERR_SHAPE;
    if (N > ((int64_t)1 << 40) / K) return QLORA_ERR_SHAPE;
    const int64_t nb = N * K / kBlock;
    if (packed_bytes) *packed_bytes = N * K / 2;
    if (n_blocks) *n_blocks = nb;
    if (n_groups) *n_groups = cdiv(nb, kGroup);
    return QLORA_OK;
}

int quant4_codebook(int quant_type, float out16[16]) {
    if (!out16) return QLORA_ERR_NULL;
    if (quant_type != QLORA_QUANT_NF4 && quant_type != QLORA_QUANT_FP4) return QLORA_ERR_VALUE;
    const NF4Tables& t = tables(quant_type);
    for (int i = 0; i < 16; ++i) out16[i] = t.L[i];
    return QLORA_OK;
}

int quant4_quantize_dq(const qlora_bf16* W, int64_t N, int64_t K, int quant_type, uint8_t* packed, int8_t* codes,
                       float* scale, float* mean, qlora_stream_t stream) {
    if (!W || !packed || !codes || !scale || !mean) return QLORA_ERR_NULL;
    if (quant_type != QLORA_QUANT_NF4 && quant_type != QLORA_QUANT_FP4) return QLORA_ERR_VALUE;
    int64_t nb = 0, ng = 0;
    if (nf4dq_sizes(N, K, nullptr, &nb, &ng) != QLORA_OK) return QLORA_ERR_SHAPE;
    if (!aligned16(W) || !aligned16(packed)) return QLORA_ERR_ALIGN;
    int sms = 0;
    int rc = check_device(&sms);
    if (rc != QLORA_OK) return rc;
    const NF4Tables& tab = tables(quant_type);
    const EncTables& enc = enc_tables(quant_type);
    int grid = (int)(ng < (int64_t)sms * 8 ? ng : (int64_t)sms * 8);
    if (quant_type == QLORA_QUANT_FP4)
        k_quantize_dq<true><<<grid, 256, 0, (cudaStream_t)stream>>>(W, nb, packed, codes, scale, mean, tab, enc);
    else
        k_quantize_dq<false><<<grid, 256, 0, (cudaStream_t)stream>>>(W, nb, packed, codes, scale, mean, tab, enc);
    note_launch();
    return launch_status();
}

int nf4_quantize_dq(const qlora_bf16* W, int64_t N, int64_t K, uint8_t* packed, int8_t* codes, float* scale,
                    float* mean, qlora_stream_t stream) {
    return quant4_quantize_dq(W, N, K, QLORA_QUANT_NF4, packed, codes, scale, mean, stream);
}

int nf4_dequant(const nf4dq_weight* w, qlora_bf16* W_out, qlora_stream_t stream) {
    int rc = (!w || !W_out) ? QLORA_ERR_NULL : QLORA_OK;
    if (rc != QLORA_OK) return rc;
    if (!w->packed || !w->codes || !w->scale || !w->mean) return QLORA_ERR_NULL;
    if (w->quant_type != QLORA_QUANT_NF4 && w->quant_type != QLORA_QUANT_FP4) return QLORA_ERR_VALUE;
    if (nf4dq_sizes(w->N, w->K, nullptr, nullptr, nullptr) != QLORA_OK) return QLORA_ERR_SHAPE;
    if (!aligned16(w->packed) || !aligned16(W_out)) return QLORA_ERR_ALIGN;
    int sms = 0;
    rc = check_device(&sms);
    if (rc != QLORA_OK) return rc;
    const int64_t nwords = w->N * w->K / 8;                    // 8 weights per packed 32-bit word
    k_dequant<<<grid_for(nwords, 8 * kDqWarpWords, sms, 4), 256, 0, (cudaStream_t)stream>>>(
        w->packed, w->codes, w->scale, w->mean, nwords, W_out, tables(w->quant_type));
    note_launch();
    return launch_status();
}

int nf4_dequant_merge(const nf4dq_weight* w, const qlora_bf16* A, const qlora_bf16* B, int r, float scaling,
                      qlora_bf16* W_out, qlora_stream_t stream) {
    if (!w || !A || !B || !W_out) return QLORA_ERR_NULL;
    if (!w->packed || !w->codes || !w->scale || !w->mean) return QLORA_ERR_NULL;
    if (w->quant_type != QLORA_QUANT_NF4 && w->quant_type != QLORA_QUANT_FP4) return QLORA_ERR_VALUE;
    if (nf4dq_sizes(w->N, w->K, nullptr, nullptr, nullptr) != QLORA_OK || w->K > QLORA_MAX_K) return QLORA_ERR_SHAPE;
    if (r < 1 || r > QLORA_MAX_RANK) return QLORA_ERR_RANK;
    if (!std::isfinite(scaling)) return QLORA_ERR_VALUE;
    if (!aligned16(w->packed) || !aligned16(A) || !aligned16(W_out)) return QLORA_ERR_ALIGN;
    int sms = 0;
    int rc = check_device(&sms);
    if (rc != QLORA_OK) return rc;
    static bool attr_set[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return QLORA_ERR_DEVICE;
    if (!attr_set[dev]) {
        std::lock_guard<std::mutex> lk(g_tc_mu);
        if (cudaFuncSetAttribute(merge::k_dequant_merge, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 merge::SMEM_BYTES) != cudaSuccess)
            return QLORA_ERR_LAUNCH;
        attr_set[dev] = true;
    }
    merge::Args a{};
    a.packed = w->packed; a.codes = w->codes; a.scale = w->scale; a.mean = w->mean;
    a.A = A; a.B = B; a.out = W_out; a.N = w->N; a.K = w->K; a.r = r; a.s = scaling;
    const dim3 grid((unsigned)cdiv(w->N, merge::TM), (unsigned)cdiv(w->K, merge::TK));
    merge::k_dequant_merge<<<grid, merge::kThreads, merge::SMEM_BYTES, (cudaStream_t)stream>>>(a, tables(w->quant_type));
    note_launch();
    return launch_status();
}

int adamw_8bit_step(qlora_bf16* p, const qlora_bf16* g, int64_t n, uint8_t* m_code, float* m_scale,
                    uint8_t* v_code, float* v_scale, int64_t step, float lr, float beta1, float beta2, float eps,
                    float weight_decay, qlora_stream_t stream) {
    if (!p || !g || !m_code || !m_scale || !v_code || !v_scale) return QLORA_ERR_NULL;
    if (n <= 0 || n > ((int64_t)1 << 40)) return QLORA_ERR_SHAPE;
    if (step < 1 || !std::isfinite(lr) || !std::isfinite(eps) || !std::isfinite(weight_decay) ||
        !(beta1 >= 0.f && beta1 < 1.f) || !(beta2 >= 0.f && beta2 < 1.f))
        return QLORA_ERR_VALUE;
    if (!aligned16(p) || !aligned16(g) || (reinterpret_cast<uintptr_t>(m_code) & 7u) != 0 ||
        (reinterpret_cast<uintptr_t>(v_code) & 7u) != 0 || (reinterpret_cast<uintptr_t>(m_scale) & 3u) != 0 ||
        (reinterpret_cast<uintptr_t>(v_scale) & 3u) != 0)
        return QLORA_ERR_ALIGN;
    int sms = 0;
    int rc = check_device(&sms);
    if (rc != QLORA_OK) return rc;
    adam::Args a{};
    a.p = p; a.g = g; a.n = n; a.m_code = m_code; a.m_scale = m_scale; a.v_code = v_code; a.v_scale = v_scale;
    a.lr = lr; a.b1 = beta1; a.b2 = beta2; a.eps = eps; a.wd = weight_decay;
    // host constants, each rounded once to fp32 from a double computation
    a.omb1 = (float)(1.0 - (double)beta1);
    a.omb2 = (float)(1.0 - (double)beta2);
    a.rbc1 = (float)(1.0 / (1.0 - std::pow((double)beta1, (double)step)));
    a.rbc2 = (float)(1.0 / (1.0 - std::pow((double)beta2, (double)step)));
    if (!std::isfinite(a.rbc1) || !std::isfinite(a.rbc2)) return QLORA_ERR_VALUE;
    const int64_t nblocks = cdiv(n, adam::kBlockParams);
    const int grid = grid_for(nblocks, adam::kThreads / 32, sms, 8);
    adam::k_adamw8<<<grid, adam::kThreads, 0, (cudaStream_t)stream>>>(a);
    note_launch();
    return launch_status();
}

size_t qlora_workspace_bytes(int64_t M, int64_t N, int64_t K, int r) {
    if (M <= 0 || N <= 0 || K <= 0 || (K % kBlock) != 0 || (N % 8) != 0 || K > QLORA_MAX_K) return 0;
    if (r < 1 || r > QLORA_MAX_RANK) return 0;
    return make_plan(M, N, K, r, 148).total;
}

// The forward with the LoRA branch reading Xl (X, or its dropped copy in the
// workspace past the regular plan when dp is given).
static int fwd_impl(const qlora_bf16* X, int64_t M, const nf4dq_weight* w, const qlora_bf16* A,
                    const qlora_bf16* B, int r, float scaling, qlora_bf16* Y, qlora_bf16* T_out, void* ws,
                    size_t ws_bytes, qlora_stream_t stream, const drop::Params* dp) {
    if (!X || !A || !B || !Y) return QLORA_ERR_NULL;
    int rc = validate_weight(w);
    if (rc != QLORA_OK) return rc;
    if (M <= 0 || M > ((int64_t)1 << 31)) return QLORA_ERR_SHAPE;
    if (r < 1 || r > QLORA_MAX_RANK) return QLORA_ERR_RANK;
    if (!std::isfinite(scaling)) return QLORA_ERR_VALUE;
    if (!aligned16(X) || !aligned16(Y) || !aligned16(A)) return QLORA_ERR_ALIGN;
    if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return ws ? QLORA_ERR_ALIGN : QLORA_ERR_WORKSPACE;
    int sms = 0;
    rc = check_device(&sms);
    if (rc != QLORA_OK) return rc;
    const Plan p = make_plan(M, w->N, w->K, r, 148);
    if (ws_bytes < p.total + (dp ? dropout_bytes(M, w->K) : 0)) return QLORA_ERR_WORKSPACE;
    cudaStream_t st = (cudaStream_t)stream;
    uint8_t* wsb = static_cast<uint8_t*>(ws);
    const uint16_t* Xl = X;
    if (dp) {
        rc = launch_dropout_x(X, M, w->K, wsb + p.total, nullptr, *dp, sms, st);
        if (rc != QLORA_OK) return rc;
        Xl = reinterpret_cast<const uint16_t*>(wsb + p.total);
    }

    if (M <= kSmallMaxM) {
        rc = small_fwd(p, X, Xl, w, A, B, scaling, Y, T_out, wsb, sms, st, dp ? dp->c : 1.f);
        if (rc == QLORA_OK) t_last_path = 1;
        return rc;
    }
    rc = compute_T(p, Xl, A, scaling, T_out, wsb, sms, st, dp ? dp->c : 1.f);
    if (rc != QLORA_OK) return rc;

    // tcgen05 path: LoRA weight rows must be 16-byte granular (r % 8 == 0) or padded
    const uint16_t* lw = B;
    int64_t ldl = r;
    if (r % 8 != 0) {
        uint16_t* Bp = reinterpret_cast<uint16_t*>(wsb + p.off_Bp);
        rc = launch_pdl(k_pad_cols, dim3((unsigned)grid_for(w->N * p.rp, 256, sms)), dim3(256), 0, st, B, w->N,
                        (int64_t)r, Bp, (int64_t)p.rp);
        if (rc != QLORA_OK) return rc;
        lw = Bp;
        ldl = p.rp;
    } else if (!aligned16(B)) {
        return QLORA_ERR_ALIGN;
    }
    rc = ensure_tc_attrs();
    if (rc != QLORA_OK) return rc;
    const int pairs = current_pairs();
    if (M > kPairMinM && pairs > 0) {
        rc = launch_tc2<false>(w, X, M, reinterpret_cast<const uint16_t*>(wsb + p.off_sT), p.lw, lw, ldl, r, Y,
                               pairs, st, true, p, wsb);
        if (rc == QLORA_OK) t_last_path = 3;
        return rc;
    }
    rc = launch_tc<false>(w, X, M, reinterpret_cast<const uint16_t*>(wsb + p.off_sT), p.lw, lw, ldl, r, Y, sms, st);
    if (rc == QLORA_OK) t_last_path = 2;
    return rc;
}

// The backward; with dp the LoRA branch reads the dropped copy of X and the
// LoRA term of dX is masked (keep * c).
static int bwd_impl(const qlora_bf16* X, const qlora_bf16* dY, int64_t M, const nf4dq_weight* w,
                    const qlora_bf16* A, const qlora_bf16* B, int r, float scaling, const qlora_bf16* T,
                    qlora_bf16* dX, qlora_bf16* dA, qlora_bf16* dB, void* ws, size_t ws_bytes,
                    qlora_stream_t stream, const drop::Params* dp) {
    if (!X || !dY || !A || !B || !dX || !dA || !dB) return QLORA_ERR_NULL;
    int rc = validate_weight(w);
    if (rc != QLORA_OK) return rc;
    if (M <= 0 || M > ((int64_t)1 << 31)) return QLORA_ERR_SHAPE;
    if (r < 1 || r > QLORA_MAX_RANK) return QLORA_ERR_RANK;
    if (!std::isfinite(scaling)) return QLORA_ERR_VALUE;
    if (!aligned16(X) || !aligned16(dY) || !aligned16(A) || !aligned16(dX)) return QLORA_ERR_ALIGN;
    if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return ws ? QLORA_ERR_ALIGN : QLORA_ERR_WORKSPACE;
    int sms = 0;
    rc = check_device(&sms);
    if (rc != QLORA_OK) return rc;
    const int64_t N = w->N, K = w->K;
    const Plan p = make_plan(M, N, K, r, 148);
    if (ws_bytes < p.total + (dp ? dropout_bytes(M, K) : 0)) return QLORA_ERR_WORKSPACE;
    cudaStream_t st = (cudaStream_t)stream;
    uint8_t* wsb = static_cast<uint8_t*>(ws);
    const uint16_t* Xl = X;
    uint16_t* mask = nullptr;
    if (dp) {
        mask = reinterpret_cast<uint16_t*>(wsb + p.total + align256((size_t)M * (size_t)K * 2));
        rc = launch_dropout_x(X, M, K, wsb + p.total, mask, *dp, sms, st);
        if (rc != QLORA_OK) return rc;
        Xl = reinterpret_cast<const uint16_t*>(wsb + p.total);
    }
    if (M <= kSmallMaxM) {
        rc = small_bwd(p, Xl, dY, w, A, B, scaling, T, dX, dA, dB, wsb, sms, st, dp, mask);
        if (rc == QLORA_OK) t_last_path = 1;
        return rc;
    }
    float* part = reinterpret_cast<float*>(wsb + p.off_part);
    uint16_t* Thl = reinterpret_cast<uint16_t*>(wsb + p.off_Tp);
    uint16_t* Uhl = reinterpret_cast<uint16_t*>(wsb + p.off_Ubf);
    uint16_t* Bp = reinterpret_cast<uint16_t*>(wsb + p.off_Bp);

    // T: recompute (hi + lo pair), or take the caller's bf16 copy as it is -- read in
    // place by the dB product when its rows are 16-byte granular, else padded to [M, 2 rp]
    // with a zero lo half
    const bool t_direct = T != nullptr && r % 8 == 0 && aligned16(T);
    if (T == nullptr) {
        rc = compute_T(p, Xl, A, scaling, nullptr, wsb, sms, st, dp ? dp->c : 1.f);
    } else if (!t_direct) {
        rc = launch_pdl(k_pad_cols, dim3((unsigned)grid_for(M * 2 * p.rp, 256, sms)), dim3(256), 0, st, T, M,
                        (int64_t)r, Thl, (int64_t)(2 * p.rp));
    }
    if (rc != QLORA_OK) return rc;

    // U = dY B  ->  U32 (fp32), Uhl (bf16 hi | lo), sU (bf16 s*U as hi | lo, [M, lw])
    const uint16_t* Bop = B;
    int64_t ldb = r;
    if (r % 8 != 0 || !aligned16(B)) {
        rc = launch_pdl(k_pad_cols, dim3((unsigned)grid_for(N * p.rp, 256, sms)), dim3(256), 0, st, B, N, (int64_t)r,
                        Bp, (int64_t)p.rp);
        if (rc != QLORA_OK) return rc;
        Bop = Bp; ldb = p.rp;
    }
    {
        FinishArgs f = fin_none();
        f.Iout = M; f.Jiter = p.lw;
        f.f32 = reinterpret_cast<float*>(wsb + p.off_U32); f.ld_f32 = p.rp; f.Jf = p.rp;
        f.J1 = r;
        f.hl = Uhl; f.hl_ld = 2 * p.rp; f.hl_off = p.rp;
        f.o2 = reinterpret_cast<uint16_t*>(wsb + p.off_sU); f.s2i = p.lw; f.s2j = 1; f.J2 = r; f.J2pad = p.lw;
        f.o2_lo = p.rp;
        f.alpha2 = scaling;
        if (p.rp <= kSkMaxRp)
            rc = run_rowk(dY, M, N, Bop, 1, ldb, ldb, p.rp, f, sms, st, reinterpret_cast<int*>(wsb + p.off_skflags),
                          (int64_t)(p.sk_flag_bytes / 4));
        else rc = run_gemm<true, false>(dY, N, Bop, ldb, M, p.rp, N, M, r, p.zU, p.kU, part, f, sms, st);
        if (rc != QLORA_OK) return rc;
    }
    // dX = dY W' + s U A (with dropout: the fused kernel computes dY W' alone, then the
    // masked LoRA term is added in place)
    rc = ensure_tc_attrs();
    if (rc != QLORA_OK) return rc;
    const int pairs = current_pairs();
    const bool fused_lora = dp == nullptr;
    const uint16_t* sU = reinterpret_cast<const uint16_t*>(wsb + p.off_sU);
    int path;
    if (M > kPairMinM && pairs > 0) {
        rc = launch_tc2<true>(w, dY, M, sU, p.lw, A, K, r, dX, pairs, st, fused_lora, p, wsb);
        path = 3;
    } else {
        rc = launch_tc<true>(w, dY, M, sU, p.lw, A, K, r, dX, sms, st, fused_lora);
        path = 2;
    }
    if (rc != QLORA_OK) return rc;
    // dB and dA read dY, X, T and U (complete: the fused kernel starts after the
    // kernel computing U has completed) and nothing the fused kernel writes, so
    // they run beside it (wait_end) on the SMs it leaves free
    const bool beside = p.rp <= kSkMaxRp;
    // dB = s dY^T T  [N, r]   (T as hi | lo columns, summed in the finish, or the caller's T)
    {
        FinishArgs f = fin_none();
        f.Iout = N; f.Jiter = r; f.col_pair = t_direct ? 0 : p.rp;
        f.o1 = dB; f.s1i = r; f.s1j = 1; f.J1 = r; f.J1pad = r; f.alpha1 = scaling;
        if (p.rp <= kSkMaxRp && t_direct)
            rc = run_colk(dY, M, N, T, r, r, 0, r, false, f, sms, st, beside);
        else if (p.rp <= kSkMaxRp)
            rc = run_colk(dY, M, N, Thl, 2 * p.rp, 2 * p.rp, p.rp, r, false, f, sms, st, beside);
        else if (t_direct)
            rc = run_gemm<false, false>(dY, N, T, r, N, p.rp, M, N, r, p.zB, p.kB, part, f, sms, st);
        else
            rc = run_gemm<false, false>(dY, N, Thl, 2 * p.rp, N, 2 * p.rp, M, N, 2 * p.rp, p.zB, p.kB, part, f, sms,
                                        st);
        if (rc != QLORA_OK) return rc;
    }
    // dA = s U^T X  [r, K]   (U as hi | lo rows, summed in the finish)
    {
        FinishArgs f = fin_none();
        f.Iout = r; f.Jiter = K; f.row_pair = p.rp;
        f.o1 = dA; f.s1i = K; f.s1j = 1; f.J1 = K; f.J1pad = K;
        f.alpha1 = dp ? (float)((double)scaling * (double)dp->c) : scaling;
        if (p.rp <= kSkMaxRp)
            rc = run_colk(Xl, M, K, Uhl, 2 * p.rp, 2 * p.rp, p.rp, r, true, f, sms, st, beside);
        else
            rc = run_gemm<false, false>(Uhl, 2 * p.rp, Xl, K, 2 * p.rp, K, M, 2 * p.rp, K, p.zA, p.kA, part, f, sms,
                                        st);
        if (rc != QLORA_OK) return rc;
    }
    // with dropout, the masked LoRA term of dX (a plain launch: it starts after dA has
    // completed, and so after the fused kernel)
    if (rc == QLORA_OK && dp) {
        drop::DxArgs d{};
        d.dX = dX; d.U = reinterpret_cast<const float*>(wsb + p.off_U32); d.ldu = p.rp; d.A = A; d.mask = mask;
        d.M = M; d.K = K; d.r = r; d.sc = (float)((double)scaling * (double)dp->c);
        static bool dx_attr[64];
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return QLORA_ERR_DEVICE;
        if (!dx_attr[dev]) {
            std::lock_guard<std::mutex> lk(g_tc_mu);
            if (cudaFuncSetAttribute(drop::k_dx_lora_dropout, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     drop::DX_SMEM) != cudaSuccess)
                return QLORA_ERR_LAUNCH;
            dx_attr[dev] = true;
        }
        const dim3 grid((unsigned)cdiv(M, drop::DX_TM), (unsigned)cdiv(K, drop::DX_TK));
        drop::k_dx_lora_dropout<<<grid, drop::DX_THREADS, drop::DX_SMEM, st>>>(d);
        note_launch();
        rc = launch_status();
    }
    if (rc == QLORA_OK) t_last_path = path;
    return rc;
}

int qlora_linear_fwd(const qlora_bf16* X, int64_t M, const nf4dq_weight* w, const qlora_bf16* A,
                     const qlora_bf16* B, int r, float scaling, qlora_bf16* Y, qlora_bf16* T_out, void* ws,
                     size_t ws_bytes, qlora_stream_t stream) {
    return fwd_impl(X, M, w, A, B, r, scaling, Y, T_out, ws, ws_bytes, stream, nullptr);
}

int qlora_linear_bwd(const qlora_bf16* X, const qlora_bf16* dY, int64_t M, const nf4dq_weight* w,
                     const qlora_bf16* A, const qlora_bf16* B, int r, float scaling, const qlora_bf16* T,
                     qlora_bf16* dX, qlora_bf16* dA, qlora_bf16* dB, void* ws, size_t ws_bytes,
                     qlora_stream_t stream) {
    return bwd_impl(X, dY, M, w, A, B, r, scaling, T, dX, dA, dB, ws, ws_bytes, stream, nullptr);
}

size_t qlora_dropout_workspace_bytes(int64_t M, int64_t N, int64_t K, int r) {
    const size_t b = qlora_workspace_bytes(M, N, K, r);
    return b == 0 ? 0 : b + dropout_bytes(M, K);
}

int qlora_linear_fwd_dropout(const qlora_bf16* X, int64_t M, const nf4dq_weight* w, const qlora_bf16* A,
                             const qlora_bf16* B, int r, float scaling, float dropout_p, uint64_t seed,
                             uint64_t offset, qlora_bf16* Y, qlora_bf16* T_out, void* ws, size_t ws_bytes,
                             qlora_stream_t stream) {
    drop::Params d{};
    const int rc = dropout_params(dropout_p, seed, offset, &d);
    if (rc != QLORA_OK) return rc;
    return fwd_impl(X, M, w, A, B, r, scaling, Y, T_out, ws, ws_bytes, stream, &d);
}

int qlora_linear_bwd_dropout(const qlora_bf16* X, const qlora_bf16* dY, int64_t M, const nf4dq_weight* w,
                             const qlora_bf16* A, const qlora_bf16* B, int r, float scaling, float dropout_p,
                             uint64_t seed, uint64_t offset, const qlora_bf16* T, qlora_bf16* dX, qlora_bf16* dA,
                             qlora_bf16* dB, void* ws, size_t ws_bytes, qlora_stream_t stream) {
    drop::Params d{};
    const int rc = dropout_params(dropout_p, seed, offset, &d);
    if (rc != QLORA_OK) return rc;
    return bwd_impl(X, dY, M, w, A, B, r, scaling, T, dX, dA, dB, ws, ws_bytes, stream, &d);
}


const char* qlora_status_string(int status) {
    switch (status) {
        case QLORA_OK: return "ok";
        case QLORA_ERR_NULL: return "a required pointer is NULL";
        case QLORA_ERR_SHAPE: return "invalid shape (M, N, K must be > 0, K % 64 == 0, N % 8 == 0)";
        case QLORA_ERR_RANK: return "LoRA rank r outside [1, 256]";
        case QLORA_ERR_ALIGN: return "pointer not 16-byte aligned (workspace: 256-byte)";
        case QLORA_ERR_WORKSPACE: return "workspace missing or smaller than qlora_workspace_bytes()";
        case QLORA_ERR_DEVICE: return "current CUDA device is not compute capability 10.0 (B200)";
        case QLORA_ERR_LAUNCH: return "CUDA launch or runtime call failed";
        case QLORA_ERR_TIMEOUT: return "a device-side bounded wait gave up";
        case QLORA_ERR_VALUE: return "a scalar argument is not finite";
        case QLORA_ERR_SCRATCH: return "needs more scratch than the fixed no-alloc scratch (QLORA_NOALLOC_SCRATCH_BYTES)";
        default: return "unknown status";
    }
}

int qlora_device_status(int reset) {
    if (cudaDeviceSynchronize() != cudaSuccess) return QLORA_ERR_LAUNCH;
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_status, sizeof(int)) != cudaSuccess) return QLORA_ERR_LAUNCH;
    if (reset) {
        const int z = 0;
        if (cudaMemcpyToSymbol(g_status, &z, sizeof(int)) != cudaSuccess) return QLORA_ERR_LAUNCH;
    }
    return v;
}

int qlora_last_path(void) { return t_last_path; }

int qlora_pair_schedule(int64_t M, int64_t n_out, int pairs, int bwd, int* mt, int64_t* ntiles, int* stream_k) {
    if (!mt || !ntiles || !stream_k) return QLORA_ERR_NULL;
    if (M <= 0 || n_out <= 0 || pairs <= 0) return QLORA_ERR_VALUE;
    const Tc2Sched sc = tc2_schedule(M, n_out, pairs, bwd != 0);
    *mt = sc.mt;
    *ntiles = sc.ntiles;
    *stream_k = sc.sk ? 1 : 0;
    return QLORA_OK;
}

int qlora_pair_spans(int64_t ntiles, int nsteps, int pair, int npairs, int64_t* out, int max_spans) {
    if (!out) return QLORA_ERR_NULL;
    if (ntiles <= 0 || nsteps <= 0 || npairs <= 0 || pair < 0 || pair >= npairs || max_spans < 0)
        return QLORA_ERR_VALUE;
    tc2::Spans spn(true, pair, npairs, ntiles, nsteps);
    int64_t tile;
    int s0, s1, n = 0;
    while (spn.next(tile, s0, s1)) {
        if (n < max_spans) {
            out[3 * n] = tile;
            out[3 * n + 1] = s0;
            out[3 * n + 2] = s1;
        }
        ++n;
    }
    return n;
}

long long qlora_launch_count(void) { return g_launches.load(); }

int qlora_set_kernel_events(void* before, void* after) {
    if ((before == nullptr) != (after == nullptr)) return QLORA_ERR_NULL;
    t_ev_before = static_cast<cudaEvent_t>(before);
    t_ev_after = static_cast<cudaEvent_t>(after);
    return QLORA_OK;
}

}  // extern "C"

// ===========================================================================
// Allocation-free forward: the workspace is a fixed static device array.
// ===========================================================================
namespace {

// Scratch of qlora_linear_fwd_noalloc; every device that loads the library
// holds it until the process exits.
static __device__ __align__(256) uint8_t g_noalloc_scratch[QLORA_NOALLOC_SCRATCH_BYTES];

void* g_noalloc_ptr[64];
std::mutex g_noalloc_mu;

// Device address of the scratch on the current device, looked up once per
// device with that device current (the host-side symbol is not a device
// address and must never be handed to a kernel).
int noalloc_scratch(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return QLORA_ERR_DEVICE;
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    if (g_noalloc_ptr[dev] == nullptr) {
        void* ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || ptr == nullptr) return QLORA_ERR_LAUNCH;
        g_noalloc_ptr[dev] = ptr;
    }
    *out = g_noalloc_ptr[dev];
    return QLORA_OK;
}

}  // namespace

extern "C" int qlora_linear_fwd_noalloc(const qlora_bf16* X, int64_t M, const nf4dq_weight* w, const qlora_bf16* A,
                                        const qlora_bf16* B, int r, float scaling, qlora_bf16* Y, qlora_bf16* T_out,
                                        qlora_stream_t stream) {
    if (w != nullptr) {
        const size_t need = qlora_workspace_bytes(M, w->N, w->K, r);
        if (need > (size_t)QLORA_NOALLOC_SCRATCH_BYTES) return QLORA_ERR_SCRATCH;
    }
    void* ws = nullptr;
    if (w != nullptr && qlora_workspace_bytes(M, w->N, w->K, r) != 0) {
        const int rc = noalloc_scratch(&ws);
        if (rc != QLORA_OK) return rc;
    }
    // invalid arguments are reported by the regular forward before anything is launched
    return qlora_linear_fwd(X, M, w, A, B, r, scaling, Y, T_out, ws, QLORA_NOALLOC_SCRATCH_BYTES, stream);
}
