// lut.cuh -- device helpers for the lookup-table decode of 3:4 ternary blocks.
//
// One table of 32 fp32 entries per block of 4 activations x0..x3 holds every
// value a packed block can take ("Sherry: Hardware-Efficient 1.25-Bit Ternary
// Quantization via Fine-grained Sparsification", digest paragraph on the 5-bit
// code: 1 sign bit + 4 lookup bits; inference builds lookup tables from the
// activations):  entry[16 G + 4 z + 2 d1 + d2] = (-1)^G (x_p0 + (-1)^d1 x_p1 +
// (-1)^d2 x_p2), p0 < p1 < p2 the positions other than z.  Tables are 144 bytes
// apart (128 + 16 pad) so that 16-byte stores of consecutive tables rotate over
// the shared-memory banks; a lookup by all lanes of a warp into one table is a
// single conflict-free access.
#pragma once

#include <stdint.h>

namespace sherry {

constexpr int kTab = 144;  // bytes per table

__device__ __forceinline__ float lds_f32(uint32_t addr) {
    float v;
    asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(addr));
    return v;
}

__device__ __forceinline__ void sts_v4(uint32_t addr, float a, float b, float c, float d) {
    asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "f"(a), "f"(b), "f"(c), "f"(d));
}

__device__ __forceinline__ float bf16lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf16hi(uint32_t u) { return __uint_as_float(u & 0xffff0000u); }

// Build the 32-entry table of one block of 4 activations at `tab` (shared address).
__device__ __forceinline__ void build_table(uint32_t tab, uint2 xb) {
    const float x0 = bf16lo(xb.x), x1 = bf16hi(xb.x), x2 = bf16lo(xb.y), x3 = bf16hi(xb.y);
    float e[16];
#pragma unroll
    for (int z = 0; z < 4; ++z) {
        const float a = z == 0 ? x1 : x0;
        const float b = z <= 1 ? x2 : x1;
        const float c = z == 3 ? x2 : x3;
        const float s = a + b, d = a - b;
        e[4 * z + 0] = s + c;
        e[4 * z + 1] = s - c;
        e[4 * z + 2] = d + c;
        e[4 * z + 3] = d - c;
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) sts_v4(tab + 16 * q, e[4 * q], e[4 * q + 1], e[4 * q + 2], e[4 * q + 3]);
#pragma unroll
    for (int q = 0; q < 4; ++q)
        sts_v4(tab + 64 + 16 * q, -e[4 * q], -e[4 * q + 1], -e[4 * q + 2], -e[4 * q + 3]);
}

// Even/odd byte-vectors of one packed word: byte i of `ev` is 4*code of block 2i,
// byte i of `od` is 4*code of block 2i+1 (code = nibble + 16*G).
__device__ __forceinline__ void spread_word(uint32_t w, uint32_t s, uint32_t& ev, uint32_t& od) {
    ev = ((w << 2) & 0x3c3c3c3cu) | (((s & 0x55u) * 0x01041040u) & 0x40404040u);
    od = ((w >> 2) & 0x3c3c3c3cu) | (((s & 0xaau) * 0x00820820u) & 0x40404040u);
}

// Sum of the 8 lookups of one word for MT tokens; tables of block j of this
// word sit at base + (boff + j)*kTab, token m at + m*tstride.
template <int MT>
__device__ __forceinline__ void word_lookups(uint32_t w, uint32_t s, uint32_t base, int boff, int tstride,
                                             float (&ws)[MT]) {
    uint32_t ev, od;
    spread_word(w, s, ev, od);
    float v[MT][8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const uint32_t src = (j & 1) ? od : ev;
        const uint32_t a = __byte_perm(src, base, (uint32_t)(j >> 1) | 0x7650u);
#pragma unroll
        for (int m = 0; m < MT; ++m) v[m][j] = lds_f32(a + (uint32_t)((boff + j) * kTab + m * tstride));
    }
#pragma unroll
    for (int m = 0; m < MT; ++m)
        ws[m] = ((v[m][0] + v[m][1]) + (v[m][2] + v[m][3])) + ((v[m][4] + v[m][5]) + (v[m][6] + v[m][7]));
}

// shared-memory load at a compile-time byte offset from `a`
template <int OFF>
__device__ __forceinline__ float lds_imm(uint32_t a) {
    float v;
    asm volatile("ld.shared.f32 %0, [%1+%2];" : "=f"(v) : "r"(a), "n"(OFF));
    return v;
}

// (x, y) = (a0 + b0, a1 + b1) with one packed fp32x2 add (sm_100)
__device__ __forceinline__ void add2(float& x, float& y, float a0, float a1, float b0, float b1) {
    asm("{\n\t.reg .b64 ra, rb, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(x), "=f"(y)
        : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}

// bf16 {+1, 0, -1} of the 4 weights of a block: two packed halves
__device__ __forceinline__ uint2 decode_block_bf16(uint32_t nib, uint32_t g) {
    const uint32_t z = nib >> 2;
    const uint32_t d1 = (nib >> 1) & 1u, d2 = nib & 1u;
    const uint32_t k3 = g | ((g ^ d1) << 1) | ((g ^ d2) << 2);
    const uint32_t negs = (k3 & ((1u << z) - 1u)) | ((k3 >> z) << (z + 1));
    uint32_t h[4];
#pragma unroll
    for (uint32_t i = 0; i < 4; ++i) h[i] = (i == z) ? 0u : (0x3f80u | (((negs >> i) & 1u) << 15));
    return make_uint2(h[0] | (h[1] << 16), h[2] | (h[3] << 16));
}

}  // namespace sherry
