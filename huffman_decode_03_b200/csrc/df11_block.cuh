// df11_block.cuh -- the per-block decode of DF11 shared by the sm_100a
// kernels (rebuild to memory, fused matrix-vector product, fused GEMM).
//
// "DFloat11: Kompresi inferensi GPU lossless ..." (id.news.hada.io/topic?id=20542),
// "Decoding berbasis LUT hierarkis" and "Kernel GPU 2 tahap dan metadata
// bantu": one warp decodes one format block of T = 32 C segments (lane l owns
// segments l and l + 32 as two chains), prefix-sums the chains' code counts
// and places the block's exponents, rotated right by one bit, contiguously in
// the warp's write buffer.  What the exponents are then merged into (global
// memory, a dot product, a tensor-core operand tile) is up to the kernel.
//
// A kernel's parameter struct P provides: stream, sm, gaps (uint32 halves of
// the Gaps words), offs, luts, cl, sym_table (optional stored symbol table),
// status, n, total_bits, nseg, nblocks, num_luts, min_code_len and cap
// (bytes of one warp's exponent buffer).
#pragma once

#include "df11.h"
#include "df11_symtab.h"

#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>

namespace {

constexpr int kIdxBits = 12;  // index width of the derived table
constexpr int kIdxEntries = 1 << kIdxBits;
constexpr int kLutBytes = DF11_MAX_LUTS * 256;
constexpr uint32_t kPointerBase = 240;
// bytes per lane's staging slot: codes start at most every lmin bits of a
// 64-bit segment, plus two zero-fill codes, stored as whole words (the last
// word may hold up to three bytes past the codes): 36 when the shortest code
// has >= 2 bits, 68 otherwise (both odd word counts, so the 32 lanes' slots
// start in 32 distinct banks)
constexpr uint32_t kSlotShort = 36, kSlotLong = 68;
// per warp: two chains x 32 lanes, plus 32 bytes so that a chain of
// inconsistent data stays inside the warp's own slots (such a block is
// reported and writes nothing): a chain reads at most 95 bits before its last
// lookup, each code of >= 2 bits (short slots) or >= 1 bit (long slots, and
// long codes >= 13), so it holds at most 47 + 3 or 94 + 3 codes, whose words
// end by byte 52 or 100 of its slot
__host__ __device__ constexpr uint32_t slot_bytes(uint32_t stride) { return 2 * 32 * stride + 32; }

__host__ __device__ constexpr uint32_t align16(uint32_t x) { return (x + 15u) & ~15u; }

// Shared memory: tables at fixed offsets, then per warp: the exponent write
// buffer and the chains' staging slots.  R copies of the symbol table,
// interleaved word by word (entry i of copy c at word R i + c): lane l reads
// copy l mod R, so a lookup's 32 lanes spread over R groups of banks and
// fewer of them meet in one bank.
template <uint32_t R>
struct SmemR {
    static constexpr uint32_t sym = 0;                           // uint32[4096 R]
    static constexpr uint32_t luts = sym + kIdxEntries * 4 * R;  // 17 * 256
    static constexpr uint32_t cl = luts + kLutBytes;         // 256
    static constexpr uint32_t zq = cl + 256;                 // uint8[16]
    static constexpr uint32_t ctr = zq + 16;                 // uint32 block counter (decoder), 16 B
    static constexpr uint32_t bufs = ctr + 16;
    __host__ __device__ static constexpr uint32_t per_warp(uint32_t cap, uint32_t stride)
    {
        return cap + slot_bytes(stride);
    }
    __host__ __device__ static constexpr uint32_t bytes(uint32_t cap, uint32_t warps, uint32_t stride)
    {
        return bufs + warps * per_warp(cap, stride);
    }
};
using Smem = SmemR<1>;
static_assert(SmemR<1>::bufs % 16 == 0 && SmemR<2>::bufs % 16 == 0 && SmemR<4>::bufs % 16 == 0,
              "buffers must be 16-byte aligned");
static_assert(slot_bytes(kSlotShort) % 16 == 0 && slot_bytes(kSlotLong) % 16 == 0,
              "slots keep the buffers 16-byte aligned");

__device__ __forceinline__ uint32_t bswap32(uint32_t x) { return __byte_perm(x, 0, 0x0123); }

// ror8 (exponents stored rotated right by one bit) and the page's
// hierarchical LUT lookup, shared with the host's copy of the derived table
using df11_symtab::lut_decode;
using df11_symtab::ror8;
static_assert(df11_symtab::kIdxBits == kIdxBits && df11_symtab::kPointerBase == kPointerBase, "one definition");

// 96-bit window h:m:l shifted left by c bits (0 <= c <= 32).
__device__ __forceinline__ void shift_window(uint32_t &h, uint32_t &m, uint32_t &l, uint32_t c)
{
    h = __funnelshift_lc(m, h, c);
    m = __funnelshift_lc(l, m, c);
    l = __funnelshift_lc(0u, l, c);
}

// Four BF16 values from four sign/mantissa bytes S and four rotated exponent
// bytes E (ror8(e) = e >> 1 | (e & 1) << 7):
//   high byte = sign | e >> 1,  low byte = (e & 1) << 7 | mantissa.
__device__ __forceinline__ void merge4(uint32_t S, uint32_t E, uint32_t &lo2, uint32_t &hi2)
{
    const uint32_t HB = (S & 0x80808080u) | (E & 0x7F7F7F7Fu);
    const uint32_t LB = (E & 0x80808080u) | (S & 0x7F7F7F7Fu);
    lo2 = __byte_perm(LB, HB, 0x5140);
    hi2 = __byte_perm(LB, HB, 0x7362);
}

__device__ __forceinline__ uint16_t merge1(uint32_t s, uint32_t e_rot)
{
    return (uint16_t)((((s & 0x80u) | (e_rot & 0x7Fu)) << 8) | (e_rot & 0x80u) | (s & 0x7Fu));
}

// Shared-memory accesses by 32-bit address.  They are volatile (kept in
// program order with each other and with the PTX loops); the staging slots
// and write buffers they touch are not accessed through C++ pointers.
__device__ __forceinline__ void st_u8(uint32_t addr, uint32_t v)
{
    asm volatile("st.shared.u8 [%0], %1;" ::"r"(addr), "r"(v));
}

__device__ __forceinline__ uint32_t ld_u8(uint32_t addr)
{
    uint32_t v;
    asm volatile("ld.shared.u8 %0, [%1];" : "=r"(v) : "r"(addr));
    return v;
}

__device__ __forceinline__ uint32_t ld_u32(uint32_t addr)
{
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
    return v;
}

__device__ __forceinline__ void st_u32(uint32_t addr, uint32_t v)
{
    asm volatile("st.shared.u32 [%0], %1;" ::"r"(addr), "r"(v));
}

// Bytes of shared memory by 32-bit address, for lut_decode: keeps the
// tables' addresses in one register each instead of generic pointers.
struct SharedBytes {
    uint32_t base;
    __device__ __forceinline__ uint32_t operator[](uint32_t i) const { return ld_u8(base + i); }
};

// Decode loop for two chains (A, B) of one lane, in PTX.  Shared-memory
// table entry (table_word): number of codes in bits 0..1, their total length
// in bits 2..6, their rotated exponents in bits 7..30 (bytes past the count
// zero); 2^31 = a code longer than 12 bits.  A chain is active while rem
// (its bits left before pend) is > 0; the bits of its window past pend are
// zeros.  Per lookup the window advances and rem drops by the length
// ((entry >> 2) serves as the funnel-shift amount directly: wrap mode reads
// only its low five bits; masked with its sign bits kept, the long-code
// entry takes 2^31 or 2^30 from rem, which ends the chain) and the exponents
// are added to the chain's pending word w at byte n, where mul = 2^(8 n); mul
// rotates left by 8 x count bits.  When the pending word fills (the rotation
// wraps, mul decreases) it is stored at the slot address qa, qa advances one
// word and w keeps the bytes that spilled past it.  The long-code entry moves
// nothing but adds 2^24 x mul to w; chain_roles undoes both, and the caller
// resolves that code and calls again.
struct Chain {
    uint32_t h, m, l;  // 96-bit window, next bit at the top of h
    int rem;           // pend - bits consumed
    uint32_t qa;       // slot word that w goes to
    uint32_t w;        // pending exponents, bytes 0..n-1
    uint32_t mul;      // 2^(8 n)
};

// One pass of the loop for both chains.  The pending word and mul trade
// registers every pass: a pass reads mul from MA (MB) and w from WA (WB) and
// leaves the new mul in WA (WB) and the new w in MA (MB), so no value is
// moved; the next pass is written with the roles exchanged.
#define DF11_DB_CHAIN(P, E, H, M, L, REM, QA, MUL, W, MASK)        \
    "@" P " shr.s32 ca, " E ", 2;\n\t"                            \
    "@" P " and.b32 t, ca, " MASK ";\n\t"                         \
    "@" P " sub.s32 " REM ", " REM ", t;\n\t"                      \
    "@" P " shf.l.wrap.b32 " H ", " M ", " H ", ca;\n\t"          \
    "@" P " shf.l.wrap.b32 " M ", " L ", " M ", ca;\n\t"          \
    "@" P " shf.l.wrap.b32 " L ", 0, " L ", ca;\n\t"              \
    "@" P " shr.u32 t, " E ", 7;\n\t"                             \
    "@" P " mul.hi.u32 ca, t, " MUL ";\n\t"                       \
    "@" P " mad.lo.u32 t, t, " MUL ", " W ";\n\t"                 \
    "@" P " shl.b32 " W ", " E ", 3;\n\t"                         \
    "@" P " shf.l.wrap.b32 " W ", " MUL ", " MUL ", " W ";\n\t"   \
    "setp.lt.and.u32 po, " W ", " MUL ", " P ";\n\t"              \
    "@po st.shared.u32 [" QA "], t;\n\t"                          \
    "@po add.u32 " QA ", " QA ", 4;\n\t"                          \
    "@" P " selp.b32 " MUL ", ca, t, po;\n\t"
#define DF11_DB_PASS(MA, WA, MB, WB, MASK)                                         \
    "@pa shr.u32 ea, %0, 20;\n\t"                                                 \
    "@pb shr.u32 eb, %7, 20;\n\t"                                                 \
    "@pa mad.lo.u32 ea, ea, %15, %14;\n\t"                                        \
    "@pb mad.lo.u32 eb, eb, %15, %14;\n\t"                                        \
    "@pa ld.shared.u32 ea, [ea];\n\t"                                             \
    "@pb ld.shared.u32 eb, [eb];\n\t"                                             \
    DF11_DB_CHAIN("pa", "ea", "%0", "%1", "%2", "%3", "%4", MA, WA, MASK)          \
    DF11_DB_CHAIN("pb", "eb", "%7", "%8", "%9", "%10", "%11", MB, WB, MASK)        \
    /* a chain stays active while bits are left (a long-code entry took */        \
    /* 2^31 or 2^30 from them) */                                                  \
    "setp.gt.s32 pa, %3, 0;\n\t"                                                  \
    "setp.gt.s32 pb, %10, 0;\n\t"                                                 \
    "or.pred pz, pa, pb;\n\t"

// A chain's mul and w after decode_bulk2 (w and mul name its two registers):
// a chain that ran out of bits has them in either order, the larger being
// mul (w holds only the n bytes below mul = 2^(8 n)).  A chain stopped on a
// code longer than 12 bits took 2^31 from rem in a first pass of the loop,
// 2^30 in a second, which also tells the order, and its pending word holds
// 2^24 x mul more: both are undone, leaving rem > 0 for the caller.
__device__ __forceinline__ void chain_roles(Chain &c)
{
    const uint32_t r0 = c.w, r1 = c.mul;
    if (c.rem < -(1 << 29)) {
        const bool first = c.rem < -(3 << 29);  // 2^31 taken: a first pass
        c.mul = first ? r0 : r1;
        c.w = (first ? r1 : r0) - 0x01000000u * c.mul;
        c.rem = (int)((uint32_t)c.rem + (first ? 0x80000000u : 0x40000000u));
    } else {
        c.mul = r0 > r1 ? r0 : r1;
        c.w = r0 > r1 ? r1 : r0;
    }
}

// The loop, two passes per trip (mul and w exchanged between them); each
// chain's values are sorted out afterwards by chain_roles.
template <uint32_t R>
__device__ __forceinline__ void decode_bulk2(Chain &A, Chain &B, uint32_t sym_base)
{
    asm volatile(
        "{\n\t"
        ".reg .pred pa, pb, pz, po;\n\t"
        ".reg .u32 ea, eb, ca, t;\n\t"
        "setp.gt.s32 pa, %3, 0;\n\t"
        "setp.gt.s32 pb, %10, 0;\n\t"
        "or.pred pz, pa, pb;\n\t"
        "@!pz bra DB_END;\n\t"
        "DB_TOP:\n\t"
        DF11_DB_PASS("%6", "%5", "%13", "%12", "0x8000001F")
        "@!pz bra DB_END;\n\t"
        DF11_DB_PASS("%5", "%6", "%12", "%13", "0x4000001F")
        "@pz bra DB_TOP;\n\t"
        "DB_END:\n\t"
        "}"
        : "+r"(A.h), "+r"(A.m), "+r"(A.l), "+r"(A.rem), "+r"(A.qa), "+r"(A.w), "+r"(A.mul), "+r"(B.h), "+r"(B.m),
          "+r"(B.l), "+r"(B.rem), "+r"(B.qa), "+r"(B.w), "+r"(B.mul)
        : "r"(sym_base), "n"(4 * R)
        : "memory");
    chain_roles(A);
    chain_roles(B);
}
#undef DF11_DB_PASS
#undef DF11_DB_CHAIN

// The byte-store form of the decode loop (the fused GEMM's decode warps, for
// which the pending-word form measured no faster): symbol-table
// entry as stored (table_entry): up to three rotated exponents in bytes
// 0..2, their total length in bits 24..28, their number in bits 29..30
// (0 = a code longer than 12 bits).
// A chain is active while pos < pend and its last entry was not 0; the bits
// of its window past pend are zeros.  Per lookup: the three exponent bytes go
// to the chain's staging slot at q unconditionally (bytes past the codes
// found are overwritten by the next lookup or never read), q advances by the
// count, the window and pos by the length.  (entry >> 24) serves as the
// funnel-shift amount directly: wrap mode reads only its low five bits.  An
// entry of 0 changes nothing and stops its chain: the caller resolves that
// long code, resets the chain's entry to non-zero and calls again.
__device__ __forceinline__ void decode_bulk2_bytes(uint32_t &hA, uint32_t &mA, uint32_t &lA, uint32_t &qA, int &posA,
                                             uint32_t &eA, uint32_t &hB, uint32_t &mB, uint32_t &lB, uint32_t &qB,
                                             int &posB, uint32_t &eB, int pendA, int pendB, uint32_t sym_base)
{
    asm volatile(
        "{\n\t"
        ".reg .pred pa, pb, pz;\n\t"
        ".reg .u32 ca, cb, t;\n\t"
        "DC_TOP:\n\t"
        "setp.lt.s32 pa, %4, %12;\n\t"
        "setp.lt.s32 pb, %10, %13;\n\t"
        "setp.ne.and.u32 pa, %5, 0, pa;\n\t"
        "setp.ne.and.u32 pb, %11, 0, pb;\n\t"
        "or.pred pz, pa, pb;\n\t"
        "@!pz bra DC_END;\n\t"
        "@pa shr.u32 %5, %0, 20;\n\t"
        "@pb shr.u32 %11, %6, 20;\n\t"
        "@pa mad.lo.u32 %5, %5, 4, %14;\n\t"
        "@pb mad.lo.u32 %11, %11, 4, %14;\n\t"
        "@pa ld.shared.u32 %5, [%5];\n\t"
        "@pb ld.shared.u32 %11, [%11];\n\t"
        // chain A
        "@pa st.shared.u8 [%3], %5;\n\t"
        "@pa mul.hi.u32 t, %5, 16777216;\n\t"
        "@pa st.shared.u8 [%3+1], t;\n\t"
        "@pa mul.hi.u32 t, %5, 65536;\n\t"
        "@pa st.shared.u8 [%3+2], t;\n\t"
        "@pa shr.u32 ca, %5, 24;\n\t"
        "@pa mul.hi.u32 t, %5, 8;\n\t"
        "@pa add.u32 %3, %3, t;\n\t"
        "@pa and.b32 t, ca, 31;\n\t"
        "@pa add.s32 %4, %4, t;\n\t"
        "@pa shf.l.wrap.b32 %0, %1, %0, ca;\n\t"
        "@pa shf.l.wrap.b32 %1, %2, %1, ca;\n\t"
        "@pa shf.l.wrap.b32 %2, 0, %2, ca;\n\t"
        // chain B
        "@pb st.shared.u8 [%9], %11;\n\t"
        "@pb mul.hi.u32 t, %11, 16777216;\n\t"
        "@pb st.shared.u8 [%9+1], t;\n\t"
        "@pb mul.hi.u32 t, %11, 65536;\n\t"
        "@pb st.shared.u8 [%9+2], t;\n\t"
        "@pb shr.u32 cb, %11, 24;\n\t"
        "@pb mul.hi.u32 t, %11, 8;\n\t"
        "@pb add.u32 %9, %9, t;\n\t"
        "@pb and.b32 t, cb, 31;\n\t"
        "@pb add.s32 %10, %10, t;\n\t"
        "@pb shf.l.wrap.b32 %6, %7, %6, cb;\n\t"
        "@pb shf.l.wrap.b32 %7, %8, %7, cb;\n\t"
        "@pb shf.l.wrap.b32 %8, 0, %8, cb;\n\t"
        "bra DC_TOP;\n\t"
        "DC_END:\n\t"
        "}"
        : "+r"(hA), "+r"(mA), "+r"(lA), "+r"(qA), "+r"(posA), "+r"(eA), "+r"(hB), "+r"(mB), "+r"(lB), "+r"(qB),
          "+r"(posB), "+r"(eB)
        : "r"(pendA), "r"(pendB), "r"(sym_base)
        : "memory");
}

// Adds one exponent (rotated) to a chain's pending word; the long-code path.
__device__ __forceinline__ void chain_put1(Chain &c, uint32_t sym)
{
    const uint32_t lo = sym * c.mul + c.w;
    const uint32_t nm = __funnelshift_l(c.mul, c.mul, 8);
    if (nm < c.mul) {
        st_u32(c.qa, lo);
        c.qa += 4;
        c.w = 0;
    } else {
        c.w = lo;
    }
    c.mul = nm;
}

// Registers one lane holds for one block: per chain its 12 stream bytes and
// the Gaps words holding its field and the next one; the block's offsets.
template <int C>
struct BlockRegs {
    uint2 s01[C];
    uint32_t s2[C];
    uint32_t g0[C], g1[C];
    uint32_t o0, o1;
};

template <int C, class P>
__device__ __forceinline__ void load_block(const P &p, uint32_t b, int lane, BlockRegs<C> &r)
{
    // segment seg = 32 (C b + k) + lane: its 12 stream bytes at 8 seg; its
    // Gap field and the next one are Gaps bits [5 seg, 5 seg + 10), which
    // start in 32-bit word 5 (C b + k) + (5 lane >> 5), at bit 5 lane mod 32
    const uint8_t *s = p.stream + 8ull * ((uint64_t)b * (32 * C) + (uint32_t)lane);
    const uint32_t *g = p.gaps + (uint64_t)(5 * C) * b + ((5u * (uint32_t)lane) >> 5);
#pragma unroll
    for (int k = 0; k < C; k++) {
        r.s01[k] = __ldg(reinterpret_cast<const uint2 *>(s + 256 * k));
        r.s2[k] = __ldg(reinterpret_cast<const uint32_t *>(s + 256 * k + 8));
        r.g0[k] = __ldg(g + 5 * k);
        r.g1[k] = __ldg(g + 5 * k + 1);
    }
    r.o0 = __ldg(p.offs + b);
    r.o1 = __ldg(p.offs + b + 1);
}

// Copies each of two chains' staging slots (shared address src[k], 4-byte
// aligned, len[k] bytes) to the write buffer at shared address dst[k]: the up
// to three bytes before dst's first word boundary and after its last one
// singly (those words are shared with neighbouring chains), the words in
// between as 32-bit stores assembled by funnel shifts.  The path of blocks
// with a chain of fewer than 3 codes, so the chains go one after the other
// (few registers) rather than fast.
__device__ __noinline__ void copy_slots2(uint32_t dA, uint32_t dB, uint32_t sA, uint32_t sB, uint32_t nA, uint32_t nB)
{
    // scalar arguments: arrays would be passed through local memory
    const uint32_t dst0[2] = {dA, dB}, src0[2] = {sA, sB}, len0[2] = {nA, nB};
#pragma unroll
    for (int k = 0; k < 2; k++) {
        uint32_t head = (4u - (dst0[k] & 3u)) & 3u;
        head = head < len0[k] ? head : len0[k];
        for (uint32_t i = 0; i < head; i++)
            st_u8(dst0[k] + i, ld_u8(src0[k] + i));
        const uint32_t dst = dst0[k] + head, src = src0[k] + head, len = len0[k] - head;
        const uint32_t nw = len >> 2, sh = 8u * (src & 3u), sa = src & ~3u;
        uint32_t cur = ld_u32(sa);
        for (uint32_t w = 0; w < nw; w++) {
            const uint32_t nxt = ld_u32(sa + 4 * w + 4);
            st_u32(dst + 4 * w, __funnelshift_r(cur, nxt, sh));
            cur = nxt;
        }
        for (uint32_t i = 4 * nw; i < len; i++)
            st_u8(dst + i, ld_u8(src + i));
    }
}

// Places every chain's staging slot in the write buffer with 32-bit stores
// only; valid when every chain of the block holds >= 3 codes.  Chain B's slot
// must lie 32 slots after chain A's.  Chain c covers
// bytes [s_c, s_c + cnt_c) of the buffer.  It writes the words from the one
// holding s_c up to, not including, the word that holds its own last byte
// (the next chain writes that one); the block's last chain also writes its
// final partial word.  The bytes of a chain's first word that precede s_c are
// the previous chain's last bytes: each chain reads its last four slot bytes
// as one word and passes it on by shuffle.  src[k]: the chain's slot (4-byte
// aligned shared address); s[k]: its byte offset in the buffer at shared
// address exp_base.
template <int C, uint32_t SLOT>
__device__ __forceinline__ void place_words(uint32_t exp_base, const uint32_t s[2], const uint32_t src[2],
                                            const uint32_t cnt[2], int lane)
{
    uint32_t last[2] = {0u, 0u}, prev[2] = {0u, 0u};
#pragma unroll
    for (int k = 0; k < C; k++) {
        const uint32_t t = src[k] + cnt[k] - 4u;  // >= src[k] - 1: inside the shared buffers
        const uint32_t a = t & ~3u;
        last[k] = __funnelshift_r(ld_u32(a), ld_u32(a + 4), 8u * (t & 3u));
        prev[k] = __shfl_up_sync(0xffffffffu, last[k], 1);
    }
    if (C == 2) {
        // chain (lane 0, B) follows chain (lane 31, A)
        const uint32_t x = __shfl_sync(0xffffffffu, last[0], 31);
        if (lane == 0)
            prev[1] = x;
    }
    uint32_t dst[2] = {0u, 0u}, nw[2] = {0u, 0u}, sh[2] = {0u, 0u};
#pragma unroll
    for (int k = 0; k < C; k++) {
        const uint32_t e = s[k] + cnt[k];
        const bool final_chain = lane == 31 && k == C - 1;
        dst[k] = exp_base + (s[k] & ~3u);
        nw[k] = (final_chain ? (e + 3u) >> 2 : e >> 2) - (s[k] >> 2);
        sh[k] = 8u * (s[k] & 3u);
    }
    // words i and i + 1 of each chain per pass: slot word i (chain B's slot
    // lies 32 slots after chain A's) funnel-shifted with the word before it,
    // predicated per chain and word, no divergent branch inside
    const int nw1m[2] = {(int)nw[0] - 1, (int)nw[1] - 1};
    uint32_t sa = src[0], i = 0;
    // Two passes per loop trip, the second with the roles of the previous
    // and last words' registers exchanged, so no word is moved between
    // passes; the trip count is tested after each pass.
#define DF11_PW_PASS(PA, PB, DA, DB)                      \
    "setp.lt.s32 r0, %5, %11;\n\t"                      \
    "setp.lt.s32 r1, %5, %12;\n\t"                      \
    "@p0 ld.shared.u32 c0, [%4];\n\t"                   \
    "@p1 ld.shared.u32 c1, [%4+%10];\n\t"               \
    "@r0 ld.shared.u32 " DA ", [%4+4];\n\t"             \
    "@r1 ld.shared.u32 " DB ", [%4+%10+4];\n\t"         \
    "@p0 shf.l.clamp.b32 w0, " PA ", c0, %8;\n\t"       \
    "@p1 shf.l.clamp.b32 w1, " PB ", c1, %9;\n\t"       \
    "@p0 st.shared.u32 [%2], w0;\n\t"                   \
    "@p1 st.shared.u32 [%3], w1;\n\t"                   \
    "@r0 shf.l.clamp.b32 w0, c0, " DA ", %8;\n\t"       \
    "@r1 shf.l.clamp.b32 w1, c1, " DB ", %9;\n\t"       \
    "@r0 st.shared.u32 [%2+4], w0;\n\t"                 \
    "@r1 st.shared.u32 [%3+4], w1;\n\t"                 \
    "add.u32 %4, %4, 8;\n\t"                            \
    "add.u32 %2, %2, 8;\n\t"                            \
    "add.u32 %3, %3, 8;\n\t"                            \
    "add.u32 %5, %5, 2;\n\t"                            \
    "setp.lt.u32 p0, %5, %6;\n\t"                       \
    "setp.lt.u32 p1, %5, %7;\n\t"                       \
    "or.pred pz, p0, p1;\n\t"
    asm volatile(
        "{\n\t"
        ".reg .pred p0, p1, r0, r1, pz;\n\t"
        ".reg .u32 c0, c1, d0, d1, w0, w1;\n\t"
        "setp.lt.u32 p0, %5, %6;\n\t"
        "setp.lt.u32 p1, %5, %7;\n\t"
        "or.pred pz, p0, p1;\n\t"
        "@!pz bra PW_END;\n\t"
        "PW_TOP:\n\t"
        DF11_PW_PASS("%0", "%1", "d0", "d1")
        "@!pz bra PW_END;\n\t"
        DF11_PW_PASS("d0", "d1", "%0", "%1")
        "@pz bra PW_TOP;\n\t"
        "PW_END:\n\t"
        "}"
        : "+r"(prev[0]), "+r"(prev[1]), "+r"(dst[0]), "+r"(dst[1]), "+r"(sa), "+r"(i)
        : "r"(nw[0]), "r"(nw[1]), "r"(sh[0]), "r"(sh[1]), "n"(32 * SLOT), "r"(nw1m[0]), "r"(nw1m[1])
        : "memory");
#undef DF11_PW_PASS
}

// A symbol-table entry (df11_symtab::table_entry: exponents in bytes 0..2,
// total length in bits 24..28, count in bits 29..30) in the decode loop's
// shared-memory form, the bytes past the count's exponents zero: with WORDS
// (the pending-word loop) count in bits 0..1, length in bits 2..6, the
// exponents in bits 7..30, and 2^31 for a code longer than 12 bits; else as
// stored.  *bad when no code set
// with codes of >= min_bits bits each produces the entry (more than 3
// codes, more than 12 bits, fewer than min_bits x count bits, or a length
// without codes).
template <bool WORDS>
__device__ __forceinline__ uint32_t table_word(uint32_t e, uint32_t min_bits, bool &bad)
{
    const uint32_t n = e >> 29, bits = (e >> 24) & 31u;
    bad |= n > 3u || bits > (uint32_t)kIdxBits || bits < n * min_bits || (n == 0 && bits != 0);
    const uint32_t syms = n >= 3u ? e & 0xFFFFFFu : e & ((1u << (8u * n)) - 1u);
    if (!WORDS)
        return syms | (bits << 24) | (n << 29);
    return n == 0 ? 0x80000000u : (n & 3u) | ((bits & 31u) << 2) | (syms << 7);
}

// Once per CTA, called by all its nthreads threads (tid = thread index): the
// page's LUTs and CodeLengths into shared memory and the tables derived from
// them.  Uses the first 8 KB after Smem::bufs as scratch.  min_bits: the
// shortest code the staging slots allow (2 for short slots, else 1).
// Returns false (every thread alike) when the symbol table, stored or
// derived, has an entry no such code set produces (table_word): the decode
// loop's slot bound relies on every code taking at least min_bits bits.
template <bool WORDS, uint32_t R = 1>
__device__ __forceinline__ bool build_tables(const uint8_t *luts_g, const uint8_t *cl_g, uint32_t num_luts,
                                             const uint32_t *sym_g, uint8_t *smem, uint32_t tid, uint32_t nthreads,
                                             uint32_t min_bits)
{
    using S = SmemR<R>;
    uint32_t *sym_tab = reinterpret_cast<uint32_t *>(smem + S::sym);
    uint8_t *luts = smem + S::luts;
    uint8_t *cl = smem + S::cl;
    uint8_t *zq = smem + S::zq;
    const uint32_t lut_bytes = num_luts * 256u;
    for (uint32_t i = tid; i < lut_bytes; i += nthreads)
        luts[i] = luts_g[i];
    for (uint32_t i = tid; i < 256; i += nthreads)
        cl[i] = cl_g[i];
    bool bad = false;
    if (sym_g) {
        // the stream carries the derived table (df11_build_format): copied
        // and checked
        for (uint32_t i = tid; i < kIdxEntries / 4; i += nthreads) {
            const uint4 v = __ldg(reinterpret_cast<const uint4 *>(sym_g) + i);
            const uint32_t t[4] = {table_word<WORDS>(v.x, min_bits, bad), table_word<WORDS>(v.y, min_bits, bad),
                                   table_word<WORDS>(v.z, min_bits, bad), table_word<WORDS>(v.w, min_bits, bad)};
            if (R == 1) {
                reinterpret_cast<uint4 *>(sym_tab)[i] = make_uint4(t[0], t[1], t[2], t[3]);
            } else {
#pragma unroll
                for (int k = 0; k < 4; k++)
#pragma unroll
                    for (uint32_t c = 0; c < R; c++)
                        sym_tab[R * (4 * i + k) + c] = t[k];
            }
        }
    } else {
        __syncthreads();
        // the first code of each 12-bit window (df11_symtab::first_code), in
        // scratch in the per-warp buffers, which are free until the blocks start
        uint16_t *first_code = reinterpret_cast<uint16_t *>(smem + S::bufs);
        for (uint32_t i = tid; i < kIdxEntries; i += nthreads)
            first_code[i] = df11_symtab::first_code(i, luts, cl, num_luts);
        __syncthreads();
        for (uint32_t i = tid; i < kIdxEntries; i += nthreads)
        {
            const uint32_t t = table_word<WORDS>(df11_symtab::table_entry(i, first_code), min_bits, bad);
#pragma unroll
            for (uint32_t c = 0; c < R; c++)
                sym_tab[R * i + c] = t;
        }
    }
    if (__syncthreads_or(bad))
        return false;
    if (tid < 16) {
        // codes formed by d trailing zero bits, d = 0..15: the all-zero code
        // (the canonical first code, of length lmin) repeated d / lmin times;
        // bit 7 flags d as a multiple of lmin
        bool bad = false;
        const uint32_t lmin = lut_decode(0u, luts, cl, num_luts, &bad) >> 8;
        const uint32_t d = (uint32_t)tid;
        zq[tid] = (lmin >= 1 && !bad) ? (uint8_t)((d / lmin) | ((d % lmin == 0) << 7)) : (uint8_t)0;
    }
    __syncthreads();
    return true;
}

// Outputs of one decoded block: stream elements [g0 + lo_off, g0 + hi) have
// their rotated exponents at bytes [lo_off, hi) of the warp's write buffer
// (g0 is a multiple of 16).
struct BlockOut {
    uint64_t g0;
    uint32_t lo_off;
    uint32_t hi;
};

// Decodes format block b (its registers in cur, loaded by load_block) into
// the warp's write buffer at shared address exp_base, through the lane's
// staging slots at slot_base; sym_base: the shared address of the symbol
// table (and of the tables after it), in the form build_tables<WORDS> made.
// WORDS: the pending-word loop (decode_bulk2), else the byte-store loop
// (decode_bulk2_bytes).  Asks L2 for the block's
// sign/mantissa bytes first.  Returns false, after setting DF11_ERR_CORRUPT
// in *p.status, when the block is inconsistent (nothing placed).  Called by
// all 32 lanes of the warp.
template <int C, uint32_t SLOT, bool WORDS, uint32_t R, class P>
__device__ __forceinline__ bool decode_block(const P &p, uint32_t b, int lane, const BlockRegs<C> &cur,
                                             uint32_t sym_base, uint32_t exp_base, uint32_t slot_base, BlockOut &out)
{
    // the LUTs, CodeLengths and zero-code table lie at fixed offsets from the
    // symbol table (SmemR)
    using S = SmemR<R>;
    const SharedBytes luts{sym_base + (S::luts - S::sym)}, cl{sym_base + (S::cl - S::sym)};
    const uint32_t zq = sym_base + (S::zq - S::sym);
    constexpr uint32_t T = 32 * C;
    const uint32_t o0 = cur.o0, o1 = cur.o1;
    const uint32_t lo_off = o0 & 15u;
    const uint64_t g0 = (uint64_t)o0 - lo_off;  // multiple of 16
    const bool offs_ok = o1 >= o0 && (uint64_t)o1 <= p.n && (uint64_t)lo_off + (o1 - o0) + 16u <= p.cap;

    // ---- the block's sign/mantissa bytes: into L2 now, read by the merge
    const uint32_t nbytes = offs_ok ? align16(lo_off + (o1 - o0)) : 0u;
    if (nbytes && lane == 0)
        asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p.sm + g0), "r"(nbytes) : "memory");

    // ---- locate: chain k's codes start in [pos0, pend) of its window.  In
    // every block but the stream's last, every segment has a successor, so
    // pend = 64 + the next Gap and only the window's third word holds bits
    // past it; the last block checks segments against the stream's end.
    bool bad = false;
    int pos0[2] = {0, 0}, pend[2] = {0, 0};
    uint32_t h[2] = {0u, 0u}, m[2] = {0u, 0u}, l[2] = {0u, 0u};
    const uint32_t goff = (5u * (uint32_t)lane) & 31u;
    const bool last_block = b + 1 >= p.nblocks;  // warp-uniform
#pragma unroll
    for (int k = 0; k < C; k++) {
        const uint32_t v = __funnelshift_r(cur.g0[k], cur.g1[k], goff);
        const uint32_t gap = v & 31u, gap_next = (v >> 5) & 31u;
        h[k] = bswap32(cur.s01[k].x);
        m[k] = bswap32(cur.s01[k].y);
        l[k] = bswap32(cur.s2[k]);
        if (!last_block) {
            pos0[k] = (int)gap;
            pend[k] = 64 + (int)gap_next;
            l[k] &= ~(0xFFFFFFFFu >> gap_next);
        } else {
            const uint32_t seg = b * T + (uint32_t)lane + 32u * k;
            const uint32_t nseg = (uint32_t)p.nseg;
            if (seg < nseg) {
                pos0[k] = (int)gap;
                pend[k] = seg + 1 < nseg ? 64 + (int)gap_next : (int)((uint32_t)p.total_bits - 64u * seg);
            }
            // bits from pend on belong to the next chain: zeros instead
            const uint32_t pe = (uint32_t)pend[k];
            h[k] &= ~__funnelshift_rc(0xFFFFFFFFu, 0u, pe);
            m[k] &= ~__funnelshift_rc(0xFFFFFFFFu, 0u, pe > 32u ? pe - 32u : 0u);
            l[k] &= ~__funnelshift_rc(0xFFFFFFFFu, 0u, pe > 64u ? pe - 64u : 0u);
        }
        shift_window(h[k], m[k], l[k], (uint32_t)pos0[k]);
    }

    // ---- decode each chain once into its staging slot.  Past pend the
    // window reads zeros, which decode as the all-zero code (the
    // canonical first code, of length lmin); the last lookup of a chain
    // starts on one of its own codes, so at most its two further codes
    // are such zero codes: pos overshoots pend by a multiple of lmin
    // (< 12) and the count by overshoot / lmin.
    uint32_t cnt[2];
    if constexpr (WORDS) {
        Chain ch[2];
#pragma unroll
        for (int k = 0; k < 2; k++) {
            ch[k].h = h[k];
            ch[k].m = m[k];
            ch[k].l = l[k];
            ch[k].rem = pend[k] - pos0[k];
            ch[k].qa = slot_base + k * (32 * SLOT);
            ch[k].w = 0u;
            ch[k].mul = 1u;
        }
        for (;;) {  // each pass resolves >= 1 code or ends both chains
            decode_bulk2<R>(ch[0], ch[1], sym_base + 4u * ((uint32_t)lane % R));
            bool any_long = false;
#pragma unroll
            for (int k = 0; k < 2; k++) {
                if (ch[k].rem > 0) {
                    // stopped on a code longer than 12 bits: the page's LUTs
                    // (a code the table leaves to them has >= 13 bits)
                    const uint32_t d = lut_decode(ch[k].h, luts, cl, p.num_luts, &bad);
                    uint32_t len = d >> 8;
                    bad |= len <= (uint32_t)kIdxBits;
                    len = len > (uint32_t)kIdxBits ? len : (uint32_t)kIdxBits + 1u;
                    chain_put1(ch[k], ror8(d & 0xFFu));
                    ch[k].rem -= (int)len;
                    shift_window(ch[k].h, ch[k].m, ch[k].l, len);
                    any_long = true;
                }
            }
            if (!any_long)
                break;
        }
#pragma unroll
        for (int k = 0; k < 2; k++) {
            st_u32(ch[k].qa, ch[k].w);  // the pending bytes
            const uint32_t q0 = slot_base + k * (32 * SLOT);
            const uint32_t bytes = ch[k].qa - q0 + ((uint32_t)(__ffs((int)ch[k].mul) - 1) >> 3);
            const uint32_t d = (uint32_t)(-ch[k].rem);  // overshoot past pend, >= 0
            const uint32_t z = ld_u8(zq + (d & 15u));
            bad |= d > 15u || !(z & 0x80u);
            cnt[k] = bytes - (z & 0x7Fu);
        }
    } else {
        uint32_t q[2], q0[2], e[2] = {1u, 1u};
        int pos[2];
#pragma unroll
        for (int k = 0; k < 2; k++) {
            q0[k] = slot_base + k * (32 * SLOT);
            q[k] = q0[k];
            pos[k] = pos0[k];
        }
        for (;;) {  // each pass resolves >= 1 code or ends both chains
            decode_bulk2_bytes(h[0], m[0], l[0], q[0], pos[0], e[0], h[1], m[1], l[1], q[1], pos[1], e[1], pend[0],
                               pend[1], sym_base);
            bool any_long = false;
#pragma unroll
            for (int k = 0; k < 2; k++) {
                if (pos[k] < pend[k]) {
                    const uint32_t d = lut_decode(h[k], luts, cl, p.num_luts, &bad);
                    uint32_t len = d >> 8;
                    bad |= len <= (uint32_t)kIdxBits;
                    len = len > (uint32_t)kIdxBits ? len : (uint32_t)kIdxBits + 1u;
                    st_u8(q[k], ror8(d & 0xFFu));
                    q[k] += 1;
                    pos[k] += (int)len;
                    shift_window(h[k], m[k], l[k], len);
                    e[k] = 1u;
                    any_long = true;
                }
            }
            if (!any_long)
                break;
        }
#pragma unroll
        for (int k = 0; k < 2; k++) {
            const uint32_t d = (uint32_t)(pos[k] - pend[k]);  // >= 0
            const uint32_t z = ld_u8(zq + (d & 15u));
            bad |= d > 15u || !(z & 0x80u);
            cnt[k] = q[k] - q0[k] - (z & 0x7Fu);
        }
    }

    // ---- warp prefix sum of the counts; both chains in one packed scan
    // (a chain holds at most 64 codes, a block at most 2048 per chain)
    uint32_t packed = 0;
#pragma unroll
    for (int k = 0; k < C; k++)
        packed |= (cnt[k] & 0xFFFFu) << (16 * k);
    // (the shuffle's own predicate says whether the source lane exists)
    uint32_t incl = packed;
    asm("{\n\t.reg .pred q;\n\t.reg .u32 y;\n\t"
        "shfl.sync.up.b32 y|q, %0, 1, 0, -1;\n\t"
        "@q add.u32 %0, %0, y;\n\t"
        "shfl.sync.up.b32 y|q, %0, 2, 0, -1;\n\t"
        "@q add.u32 %0, %0, y;\n\t"
        "shfl.sync.up.b32 y|q, %0, 4, 0, -1;\n\t"
        "@q add.u32 %0, %0, y;\n\t"
        "shfl.sync.up.b32 y|q, %0, 8, 0, -1;\n\t"
        "@q add.u32 %0, %0, y;\n\t"
        "shfl.sync.up.b32 y|q, %0, 16, 0, -1;\n\t"
        "@q add.u32 %0, %0, y;\n\t}"
        : "+r"(incl));
    const uint32_t tot = __shfl_sync(0xffffffffu, incl, 31);
    uint32_t first[2] = {0u, 0u};
    uint32_t total = 0;
#pragma unroll
    for (int k = 0; k < C; k++) {
        first[k] = total + ((incl >> (16 * k)) & 0xFFFFu) - cnt[k];
        total += (tot >> (16 * k)) & 0xFFFFu;
        bad |= cnt[k] > 64u;
    }
    const bool block_bad = __any_sync(0xffffffffu, bad) || !offs_ok || total != o1 - o0;
    if (block_bad) {
        if (lane == 0)
            atomicOr(p.status, (uint32_t)DF11_ERR_CORRUPT);
        __syncwarp();
        return false;
    }
    // ---- place: each chain's slot into the write buffer; whole words
    // when every chain holds >= 3 codes (the normal case), else
    // with single bytes at the chains' edges
    {
        const uint32_t srcs[2] = {slot_base, slot_base + 32 * SLOT};
        bool short_chain = cnt[0] < 3u;
        if (C == 2)
            short_chain |= cnt[1] < 3u;
        if (!__any_sync(0xffffffffu, short_chain)) {
            const uint32_t offs2[2] = {lo_off + first[0], lo_off + first[1]};
            place_words<C, SLOT>(exp_base, offs2, srcs, cnt, lane);
        } else {
            copy_slots2(exp_base + lo_off + first[0], exp_base + lo_off + first[1], srcs[0], srcs[1], cnt[0], cnt[1]);
        }
    }
    __syncwarp();
    out.g0 = g0;
    out.lo_off = lo_off;
    out.hi = lo_off + total;
    return true;
}

// ------------------------------------------------------------- host side
inline bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

// Checks a stream's arrays (device pointers) and fills the launch fields they
// determine.
template <class P>
df11_status stream_params(const df11_arrays *a, uint32_t *status_dev, P &prm)
{
    if (!a || !status_dev)
        return DF11_ERR_INVALID_ARG;
    const uint32_t T = a->threads_per_block;
    if (T != 32 && T != 64)
        return DF11_ERR_INVALID_ARG;
    if (!a->encoded_exponent || !a->packed_sign_mantissa || !a->gaps || !a->block_offset || !a->luts ||
        !a->code_lengths)
        return DF11_ERR_INVALID_ARG;
    if (!aligned(a->encoded_exponent, 16) || !aligned(a->packed_sign_mantissa, 16) || !aligned(a->gaps, 8) ||
        !aligned(a->block_offset, 4) || !aligned(a->symbol_table, 16))
        return DF11_ERR_INVALID_ARG;
    if (a->num_luts < 1 || a->num_luts > DF11_MAX_LUTS || a->n >= (1ull << 32))
        return DF11_ERR_INVALID_ARG;
    const uint64_t nseg = (a->total_bits + 63) / 64;
    if (nseg != a->num_segments || (nseg + T - 1) / T != a->num_blocks || a->num_blocks == 0)
        return DF11_ERR_INVALID_ARG;
    // every load stays inside its array
    if (a->encoded_exponent_bytes < (uint64_t)a->num_blocks * T * 8 + 16 ||
        a->packed_sign_mantissa_bytes < ((a->n + 15) / 16) * 16 ||
        a->gaps_words < (5ull * a->num_blocks * T + 63) / 64 + 2 || a->max_block_elems > 64u * T)
        return DF11_ERR_INVALID_ARG;
    std::memset(&prm, 0, sizeof(prm));
    prm.stream = a->encoded_exponent;
    prm.sm = a->packed_sign_mantissa;
    prm.gaps = reinterpret_cast<const uint32_t *>(a->gaps);
    prm.offs = a->block_offset;
    prm.luts = a->luts;
    prm.cl = a->code_lengths;
    prm.sym_table = a->symbol_table;  // optional: null derives it in each CTA
    prm.status = status_dev;
    prm.n = a->n;
    prm.total_bits = a->total_bits;
    prm.nseg = nseg;
    prm.nblocks = a->num_blocks;
    prm.num_luts = a->num_luts;
    prm.min_code_len = a->min_code_len <= 32 ? a->min_code_len : 0u;
    // the per-warp buffers of 8 warps hold the 8 KB set-up scratch table
    prm.cap = align16(a->max_block_elems + 32);
    return DF11_OK;
}

}  // namespace
