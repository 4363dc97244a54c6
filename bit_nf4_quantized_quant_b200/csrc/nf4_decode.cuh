// nf4_decode.cuh -- exact NF4 decode of one 64-weight block in registers.
//
// The dequantized weight of a block with constant c' is one of 16 values,
// v[q] = bf16_rne(L[q] * c').  They are computed once per block (16 fp32
// multiplies, 8 packs) and kept as two byte planes (low and high byte of each
// bf16), four registers each.  A packed word of 8 nibbles is then decoded
// with byte permutes: prmt picks bytes from an 8-entry half-table with a
// 3-bit index, a second prmt in sign-replicate mode turns bit 3 of each
// nibble into a byte mask that selects between the two halves, and two more
// permutes interleave the planes into bf16x2 words.  The result is bit for
// bit the dense dequantization, for 21 integer instructions per 8 weights.
#pragma once
#include "common.cuh"

namespace qnf4 {

struct BlockTable {
    uint32_t lo[4];   // low bytes of v[0..15], 4 per register
    uint32_t hi[4];   // high bytes
};

__device__ __forceinline__ uint32_t lop3_sel(uint32_t a, uint32_t b, uint32_t m) {
    // (a & ~m) | (b & m)
    uint32_t d;
    asm("lop3.b32 %0, %1, %2, %3, 0xD8;" : "=r"(d) : "r"(a), "r"(b), "r"(m));
    return d;
}

__device__ __forceinline__ BlockTable make_block_table(const NF4Tables& tab, float c) {
    uint32_t p[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) p[j] = pack_bf16x2(__fmul_rn(tab.L[2 * j], c), __fmul_rn(tab.L[2 * j + 1], c));
    BlockTable t;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        t.lo[i] = prmt(p[2 * i], p[2 * i + 1], 0x6420u);
        t.hi[i] = prmt(p[2 * i], p[2 * i + 1], 0x7531u);
    }
    return t;
}

// w: 4 packed bytes = elements 0..7 of a run (byte j: element 2j in the high
// nibble, 2j+1 in the low nibble).  out[k] = bf16x2(v[elem 2k], v[elem 2k+1]).
__device__ __forceinline__ void decode8(const BlockTable& t, uint32_t w, uint32_t (&out)[4]) {
    const uint32_t s = w & 0x77777777u;
    const uint32_t w4 = w << 4;
    const uint32_t m_lo = prmt(w4, w, 0xD9C8u);     // bit 3 of nibbles 0..3 -> byte masks
    const uint32_t m_hi = prmt(w4, w, 0xFBEAu);     // bit 3 of nibbles 4..7
    const uint32_t s_hi = s >> 16;
    {
        const uint32_t LO = lop3_sel(prmt(t.lo[0], t.lo[1], s), prmt(t.lo[2], t.lo[3], s), m_lo);
        const uint32_t HI = lop3_sel(prmt(t.hi[0], t.hi[1], s), prmt(t.hi[2], t.hi[3], s), m_lo);
        out[0] = prmt(LO, HI, 0x4051u);
        out[1] = prmt(LO, HI, 0x6273u);
    }
    {
        const uint32_t LO = lop3_sel(prmt(t.lo[0], t.lo[1], s_hi), prmt(t.lo[2], t.lo[3], s_hi), m_hi);
        const uint32_t HI = lop3_sel(prmt(t.hi[0], t.hi[1], s_hi), prmt(t.hi[2], t.hi[3], s_hi), m_hi);
        out[2] = prmt(LO, HI, 0x4051u);
        out[3] = prmt(LO, HI, 0x6273u);
    }
}

}  // namespace qnf4
