// df11_symtab.h -- the derived 12-bit symbol table of the decoders, as one
// definition for the device (each CTA's set-up when a stream carries no
// table) and the host (df11_build_format stores the table with the stream).
//
// "Decoding berbasis LUT hierarkis": a code is decoded through the page's
// hierarchical LUTs: LUT 0 on the first 8 bits of a 32-bit window, a pointer
// value 256 - j continues in LUT j on the next 8 bits, CodeLengths gives the
// length of the symbol found.  The derived table answers, for each 12-bit
// window, the first up to three whole codes that lie inside it: entry =
// exponents (rotated right by one bit) in bytes 0..2, their total length in
// bits 24..28, their count in bits 29..30.
#pragma once

#include <cstdint>

#if defined(__CUDACC__)
#define DF11_HD __host__ __device__ __forceinline__
#else
#define DF11_HD inline
#endif

namespace df11_symtab {

constexpr int kIdxBits = 12;
constexpr int kIdxEntries = 1 << kIdxBits;
constexpr uint32_t kPointerBase = 240;

DF11_HD uint32_t ror8(uint32_t s) { return ((s >> 1) | (s << 7)) & 0xFFu; }

// The page's hierarchical lookup of the code at the top of win: symbol |
// length << 8; *bad on a dangling pointer.  Bytes: anything indexable by a
// byte offset (a pointer, or a device accessor of shared memory).
template <class Bytes>
DF11_HD uint32_t lut_decode(uint32_t win, const Bytes &luts, const Bytes &cl, uint32_t num_luts, bool *bad)
{
    uint32_t e = luts[win >> 24];
#if defined(__CUDA_ARCH__)
#pragma unroll
#endif
    for (int lvl = 1; lvl <= 3; lvl++) {
        if (e < kPointerBase)
            break;
        const uint32_t j = 256u - e;
        if (j >= num_luts) {
            *bad = true;
            return 32u << 8;
        }
        e = luts[j * 256u + ((win >> (24 - 8 * lvl)) & 0xFFu)];
    }
    if (e >= kPointerBase) {
        *bad = true;
        return 32u << 8;
    }
    return e | ((uint32_t)cl[e] << 8);
}

// The first code of 12-bit window i (bits past 12 read as zeros): symbol |
// length << 8, or 0 when that code is longer than 12 bits (a code found in a
// zero-filled window is genuine when it ends inside the window: prefix
// property).
DF11_HD uint16_t first_code(uint32_t i, const uint8_t *luts, const uint8_t *cl, uint32_t num_luts)
{
    bool bad = false;
    const uint32_t e = lut_decode(i << (32 - kIdxBits), luts, cl, num_luts, &bad);
    const uint32_t len = e >> 8;
    return (!bad && len >= 1 && len <= (uint32_t)kIdxBits) ? (uint16_t)e : (uint16_t)0;
}

// Entry i of the derived table from the first codes of all windows: the
// first three codes of window i, by three dependent lookups.
DF11_HD uint32_t table_entry(uint32_t i, const uint16_t *fc)
{
    uint32_t syms = 0, bits = 0, n = 0;
#if defined(__CUDA_ARCH__)
#pragma unroll
#endif
    for (int j = 0; j < 3; j++) {
        const uint32_t f = fc[(i << bits) & (kIdxEntries - 1)];
        const uint32_t len = f >> 8;
        if (len != 0 && len + bits <= (uint32_t)kIdxBits && n == (uint32_t)j) {
            syms |= ror8(f & 0xFFu) << (8 * j);
            bits += len;
            n++;
        }
    }
    return syms | (bits << 24) | (n << 29);
}

}  // namespace df11_symtab
