// adamw8.cuh -- one AdamW step of the LoRA adapters with 8-bit moment states.
//
// States: per block of 256 consecutive parameters one fp32 scale and one
// FP8 E4M3 code per parameter, value = fl32(e4m3(code) * scale),
// scale = fl32(absmax / 448), code = e4m3_rn_satfinite(fl32(x * inv)),
// inv = fl32(448 / absmax) (code 0 when absmax = 0).
// Update (every operation one IEEE fp32 rounding, in this order):
//   m = b1 m + omb1 g;  v = b2 v + omb2 (g g);  mh = m rbc1;  vh = v rbc2
//   u = mh / (sqrt(vh) + eps) + wd p;  p = bf16_rne(p - lr u)
// then the block's new m and v are requantized with the block's new absmax.
// One division and one square root per parameter; the bias corrections are
// host-computed reciprocals and the block scale's reciprocal is one division
// per block.
//
// HBM-bound streaming kernel (read 2 + 2 + 1 + 1 B, write 2 + 1 + 1 B per
// parameter, plus 16 B of scales per block): one warp per block, lane l takes
// parameters 8l..8l+7 (16-byte loads of p and g, 8-byte loads of the codes),
// the block absmax is a warp shuffle reduction, the E4M3 conversions are the
// hardware cvt instructions (round to nearest even, saturating at 448).
#pragma once
#include <cuda_fp16.h>
#include "common.cuh"

namespace qnf4 {
namespace adam {

constexpr int kBlockParams = 256;
constexpr int kThreads = 256;
constexpr float kE4M3Max = 448.f;

struct Args {
    uint16_t* p;
    const uint16_t* g;
    int64_t n;
    uint8_t* m_code;
    float* m_scale;
    uint8_t* v_code;
    float* v_scale;
    float lr, b1, b2, eps, wd, omb1, omb2, rbc1, rbc2;
};

// two E4M3 codes (low byte first) -> two fp32 values, exact
__device__ __forceinline__ float2 e4m3x2_to_f32(uint32_t two) {
    uint32_t h2;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"((unsigned short)(two & 0xffffu)));
    __half2 h = *reinterpret_cast<__half2*>(&h2);
    return __half22float2(h);
}

// two fp32 -> two E4M3 codes, lo in the low byte
__device__ __forceinline__ uint32_t f32x2_to_e4m3(float lo, float hi) {
    unsigned short d;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(d) : "f"(hi), "f"(lo));
    return (uint32_t)d;
}

__global__ void __launch_bounds__(kThreads) k_adamw8(const Args a) {
    const int lane = threadIdx.x & 31;
    const int64_t nblocks = cdiv(a.n, kBlockParams);
    const int64_t warps = ((int64_t)gridDim.x * kThreads) >> 5;
    for (int64_t blk = ((int64_t)blockIdx.x * kThreads + threadIdx.x) >> 5; blk < nblocks; blk += warps) {
        const int64_t e0 = blk * kBlockParams + 8 * lane;
        const bool full = e0 + 8 <= a.n;
        uint16_t pv[8], gv[8];
        uint8_t mc[8], vc[8];
        if (full) {
            const uint4 p4 = *reinterpret_cast<const uint4*>(a.p + e0);
            const uint4 g4 = ldg_nc_v4(a.g + e0);
            const uint2 m2 = *reinterpret_cast<const uint2*>(a.m_code + e0);
            const uint2 v2 = *reinterpret_cast<const uint2*>(a.v_code + e0);
            const uint32_t pw[4] = {p4.x, p4.y, p4.z, p4.w}, gw[4] = {g4.x, g4.y, g4.z, g4.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                pv[2 * j] = (uint16_t)(pw[j] & 0xffffu); pv[2 * j + 1] = (uint16_t)(pw[j] >> 16);
                gv[2 * j] = (uint16_t)(gw[j] & 0xffffu); gv[2 * j + 1] = (uint16_t)(gw[j] >> 16);
            }
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                mc[j] = (uint8_t)(m2.x >> (8 * j)); mc[4 + j] = (uint8_t)(m2.y >> (8 * j));
                vc[j] = (uint8_t)(v2.x >> (8 * j)); vc[4 + j] = (uint8_t)(v2.y >> (8 * j));
            }
        } else {
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const bool in = e0 + j < a.n;
                pv[j] = in ? a.p[e0 + j] : (uint16_t)0;
                gv[j] = in ? a.g[e0 + j] : (uint16_t)0;
                mc[j] = in ? a.m_code[e0 + j] : (uint8_t)0;
                vc[j] = in ? a.v_code[e0 + j] : (uint8_t)0;
            }
        }
        const float msc = a.m_scale[blk], vsc = a.v_scale[blk];
        float mn[8], vn[8];
        uint16_t po[8];
        float mmax = 0.f, vmax = 0.f;
#pragma unroll
        for (int j = 0; j < 8; j += 2) {
            const float2 mo = e4m3x2_to_f32((uint32_t)mc[j] | ((uint32_t)mc[j + 1] << 8));
            const float2 vo = e4m3x2_to_f32((uint32_t)vc[j] | ((uint32_t)vc[j + 1] << 8));
            const float mov[2] = {__fmul_rn(mo.x, msc), __fmul_rn(mo.y, msc)};
            const float vov[2] = {__fmul_rn(vo.x, vsc), __fmul_rn(vo.y, vsc)};
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int i = j + h;
                const float gf = bf16lo_to_f32(gv[i]), pf = bf16lo_to_f32(pv[i]);
                const float m = __fadd_rn(__fmul_rn(a.b1, mov[h]), __fmul_rn(a.omb1, gf));
                const float v = __fadd_rn(__fmul_rn(a.b2, vov[h]), __fmul_rn(a.omb2, __fmul_rn(gf, gf)));
                const float mh = __fmul_rn(m, a.rbc1), vh = __fmul_rn(v, a.rbc2);
                const float den = __fadd_rn(__fsqrt_rn(vh), a.eps);
                const float u = __fadd_rn(__fdiv_rn(mh, den), __fmul_rn(a.wd, pf));
                po[i] = __bfloat16_as_ushort(__float2bfloat16_rn(__fsub_rn(pf, __fmul_rn(a.lr, u))));
                const bool in = e0 + i < a.n;
                mn[i] = in ? m : 0.f;
                vn[i] = in ? v : 0.f;
                mmax = fmaxf(mmax, fabsf(mn[i]));
                vmax = fmaxf(vmax, fabsf(vn[i]));
            }
        }
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) {
            mmax = fmaxf(mmax, __shfl_xor_sync(0xffffffffu, mmax, off));
            vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, off));
        }
        const float ms = __fdiv_rn(mmax, kE4M3Max), vs = __fdiv_rn(vmax, kE4M3Max);
        const float mi = mmax == 0.f ? 0.f : __fdiv_rn(kE4M3Max, mmax);
        const float vi = vmax == 0.f ? 0.f : __fdiv_rn(kE4M3Max, vmax);
        uint32_t mq[4], vq[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            mq[j] = mmax == 0.f ? 0u : f32x2_to_e4m3(__fmul_rn(mn[2 * j], mi), __fmul_rn(mn[2 * j + 1], mi));
            vq[j] = vmax == 0.f ? 0u : f32x2_to_e4m3(__fmul_rn(vn[2 * j], vi), __fmul_rn(vn[2 * j + 1], vi));
        }
        if (full) {
            *reinterpret_cast<uint4*>(a.p + e0) =
                make_uint4((uint32_t)po[0] | ((uint32_t)po[1] << 16), (uint32_t)po[2] | ((uint32_t)po[3] << 16),
                           (uint32_t)po[4] | ((uint32_t)po[5] << 16), (uint32_t)po[6] | ((uint32_t)po[7] << 16));
            *reinterpret_cast<uint2*>(a.m_code + e0) = make_uint2(mq[0] | (mq[1] << 16), mq[2] | (mq[3] << 16));
            *reinterpret_cast<uint2*>(a.v_code + e0) = make_uint2(vq[0] | (vq[1] << 16), vq[2] | (vq[3] << 16));
        } else {
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                if (e0 + j < a.n) {
                    a.p[e0 + j] = po[j];
                    a.m_code[e0 + j] = (uint8_t)(mq[j >> 1] >> (8 * (j & 1)));
                    a.v_code[e0 + j] = (uint8_t)(vq[j >> 1] >> (8 * (j & 1)));
                }
            }
        }
        if (lane == 0) {
            a.m_scale[blk] = ms;
            a.v_scale[blk] = vs;
        }
    }
}

}  // namespace adam
}  // namespace qnf4
