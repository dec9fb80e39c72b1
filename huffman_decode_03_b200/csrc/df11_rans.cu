// df11_rans.cu -- sm_100a decoder of the rANS variant of the exponent coder.
//
// The DFloat11 page's discussion proposes rANS (range asymmetric numeral
// systems) as the entropy coder for the exponents that suits SIMD hardware
// better than Huffman coding.  The layout (include/df11.h, df11_rans_arrays)
// is made for a warp: 32 lanes each hold one 32-bit state and step together
// through a block of 512 * chunks elements; lane l's elements are 16
// consecutive ones out of every 512, so a lane's 16 decoded exponents are
// merged with 16 consecutive sign/mantissa bytes and leave in one 32-byte
// store, and a warp's stores cover 1 KB contiguous -- no prefix sum, no
// placement through shared memory, unlike the Huffman decoder.
//
// Per step and lane: one lookup in a 4096-entry table (the slot's exponent,
// rotated right by one bit for the merge, slot - cum and freq - 1), one
// multiply-add for the new state, and, when the state falls below 2^16, the
// next 16-bit word of the lane's own stream (a predicated load and a pointer
// increment: the lanes do not coordinate).  A block's streams follow one
// another; each lane finds its start from the 32 lane counts by one warp
// scan per block.  A block's words are read from shared memory: each warp
// has two buffers, and the next block's words are copied into the other one
// (cp.async) and its sign/mantissa bytes prefetched into L2 while the
// current block decodes.  The buffers are sized for the stream's largest
// block while 32 warps per CTA still fit (blocks of up to about 1,500 words);
// the few blocks of a stream that exceed that read their words straight from
// global memory (asked into L2 one block ahead), each load clamped to the
// word array.  Every lane must end the block
// at x = 2^16 with its stream used up, and the lane counts must add up to
// the block's words; otherwise DF11_ERR_CORRUPT is set.  Copies are clamped
// to the padded array and to the buffer; a lane's start is clamped to the
// copied words, and a block reads at most 16 words per chunk and lane beyond
// it, inside the buffer's slack of 16 chunks + 8 words.  So inconsistent
// data never reads out of bounds; nothing traps and every loop has a fixed
// trip count.  Blocks go to warps by striding over the stream when its last
// round is nearly full, else as contiguous ranges per CTA handed to its
// warps by a shared-memory counter.
#include "df11.h"

#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

namespace {

constexpr uint32_t kProbBits = 12;
constexpr uint32_t kSlots = 1u << kProbBits;
constexpr uint32_t kLow = 1u << 16;
constexpr int kMaxWarps = 32;

struct RansParams {
    const uint16_t *words;
    const uint32_t *states;
    const uint32_t *block_word;
    const uint16_t *freq;
    const uint8_t *sm;
    uint16_t *dst;
    uint32_t *status;
    uint64_t n;
    uint32_t num_blocks;
    uint32_t chunks;
    uint32_t wide;  // dst is 32-byte aligned: 32-byte stores
    uint32_t cap;        // words a block may copy into its buffer (multiple of 8); a block spanning more
                         // reads its words from global memory
    uint32_t bufw;       // words of one buffer: cap plus the slack a block's reads need past a clamped start
    uint32_t words_end;  // copies end at or below this word: num_words rounded down to 8, plus the 8 padding words
    const uint8_t *lane_words;
};

__device__ __forceinline__ uint32_t ror8(uint32_t s) { return ((s >> 1) | (s << 7)) & 0xFFu; }

// BF16 from sign/mantissa bytes S and rotated exponent bytes E (4 each):
// high byte = sign | e >> 1, low byte = (e & 1) << 7 | mantissa.
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

// The lane's next word: from its block's buffer in shared memory (a 32-bit
// shared address) or, for a block too large for the buffer, from global
// memory (a 64-bit address); the address advances past it.
__device__ __forceinline__ uint32_t next_word(uint32_t &wp)
{
    uint32_t w;
    asm volatile("ld.shared.u16 %0, [%1];" : "=r"(w) : "r"(wp) : "memory");
    wp += 2u;
    return w;
}
struct GlobalWords {
    uint64_t p;     // address of the lane's next word
    uint64_t last;  // the word array's last word: loads are clamped to it
};
__device__ __forceinline__ uint32_t next_word(GlobalWords &g)
{
    uint32_t w;
    const uint64_t a = g.p < g.last ? g.p : g.last;
    asm volatile("ld.global.nc.u16 %0, [%1];" : "=r"(w) : "l"(a) : "memory");
    g.p += 2u;
    return w;
}

// One decode step of one lane.  valid: the lane's element exists; acc
// receives the exponent byte at byte position Q; wp: the address of the
// lane's next word (next_word).
template <int Q, class W>
__device__ __forceinline__ void step(uint32_t &x, uint32_t &acc, W &wp, bool valid, const uint32_t *table)
{
    if (valid) {
        const uint32_t e = table[x & (kSlots - 1)];
        const uint32_t xh = x >> kProbBits;
        x = (e >> 20) * xh + xh + ((e >> 8) & 0xFFFu);
        acc = __byte_perm(acc, e, (0x3210 & ~(0xF << (4 * Q))) | (4 << (4 * Q)));
        if (x < kLow)
            x = (x << 16) | next_word(wp);
    }
}

// 16 steps of the last, partial block: elements past n are skipped.
template <class W>
__device__ __forceinline__ void decode_chunk_tail(uint32_t &x, W &wp, uint64_t pos0, const uint32_t *table,
                                                  const RansParams &p, uint32_t acc[4])
{
#define DF11_STEP(I) step<(I) & 3, W>(x, acc[(I) >> 2], wp, pos0 + (I) < p.n, table)
    DF11_STEP(0); DF11_STEP(1); DF11_STEP(2); DF11_STEP(3);
    DF11_STEP(4); DF11_STEP(5); DF11_STEP(6); DF11_STEP(7);
    DF11_STEP(8); DF11_STEP(9); DF11_STEP(10); DF11_STEP(11);
    DF11_STEP(12); DF11_STEP(13); DF11_STEP(14); DF11_STEP(15);
#undef DF11_STEP
}

// One step of a full block in PTX, the same arithmetic as step() with the
// word read predicated.  Operands: %0 the state, %1 the shared address of
// the lane's next word, A the accumulator that takes the exponent byte at
// the position SEL selects, %6 the table's shared address.  No clamp: a lane
// starts at most cap words into its buffer and reads at most one word per
// step, 16 per chunk, and the buffer has that much slack.
#define DF11_RSTEP(A, SEL)                       \
    "and.b32 ts, %0, 4095;\n\t"                  \
    "shl.b32 ts, ts, 2;\n\t"                     \
    "add.u32 ts, ts, %6;\n\t"                    \
    "ld.shared.u32 te, [ts];\n\t"                \
    "shr.u32 th, %0, 12;\n\t"                    \
    "shr.u32 tf, te, 20;\n\t"                    \
    "bfe.u32 to, te, 8, 12;\n\t"                 \
    "mad.lo.u32 %0, tf, th, th;\n\t"             \
    "add.u32 %0, %0, to;\n\t"                    \
    "prmt.b32 " A ", " A ", te, " SEL ";\n\t"    \
    "setp.lt.u32 tp, %0, 65536;\n\t"             \
    "@tp ld.shared.u16 tw, [%1];\n\t"            \
    "@tp prmt.b32 %0, tw, %0, 0x5410;\n\t"       \
    "@tp add.u32 %1, %1, 2;\n\t"
#define DF11_RSTEP4(A) \
    DF11_RSTEP(A, "0x3214") DF11_RSTEP(A, "0x3240") DF11_RSTEP(A, "0x3410") DF11_RSTEP(A, "0x4210")

// 16 steps of a full block (all lanes valid).
__device__ __forceinline__ void decode_chunk_full(uint32_t &x, uint32_t &wp, uint32_t tbl, uint32_t acc[4])
{
    asm volatile("{\n\t.reg .b32 ts, te, th, tf, to, tw;\n\t.reg .pred tp;\n\t"
                 DF11_RSTEP4("%2") DF11_RSTEP4("%3") DF11_RSTEP4("%4") DF11_RSTEP4("%5")
                 "}"
                 : "+r"(x), "+r"(wp), "+r"(acc[0]), "+r"(acc[1]), "+r"(acc[2]), "+r"(acc[3])
                 : "r"(tbl)
                 : "memory");
}
// The same 16 steps for a block whose words stay in global memory (the word
// load through the read-only path, its address clamped to the array's last
// word: a lane of inconsistent data may read up to 16 words per chunk past
// its stream, and global memory has no slack).
#define DF11_RSTEP_G(A, SEL)                     \
    "and.b32 ts, %0, 4095;\n\t"                  \
    "shl.b32 ts, ts, 2;\n\t"                     \
    "add.u32 ts, ts, %6;\n\t"                    \
    "ld.shared.u32 te, [ts];\n\t"                \
    "shr.u32 th, %0, 12;\n\t"                    \
    "shr.u32 tf, te, 20;\n\t"                    \
    "bfe.u32 to, te, 8, 12;\n\t"                 \
    "mad.lo.u32 %0, tf, th, th;\n\t"             \
    "add.u32 %0, %0, to;\n\t"                    \
    "prmt.b32 " A ", " A ", te, " SEL ";\n\t"    \
    "setp.lt.u32 tp, %0, 65536;\n\t"             \
    "@tp min.u64 ta, %1, %7;\n\t"                \
    "@tp ld.global.nc.u16 tw, [ta];\n\t"         \
    "@tp prmt.b32 %0, tw, %0, 0x5410;\n\t"       \
    "@tp add.u64 %1, %1, 2;\n\t"
#define DF11_RSTEP4_G(A) \
    DF11_RSTEP_G(A, "0x3214") DF11_RSTEP_G(A, "0x3240") DF11_RSTEP_G(A, "0x3410") DF11_RSTEP_G(A, "0x4210")

__device__ __forceinline__ void decode_chunk_full(uint32_t &x, GlobalWords &g, uint32_t tbl, uint32_t acc[4])
{
    asm volatile("{\n\t.reg .b32 ts, te, th, tf, to, tw;\n\t.reg .b64 ta;\n\t.reg .pred tp;\n\t"
                 DF11_RSTEP4_G("%2") DF11_RSTEP4_G("%3") DF11_RSTEP4_G("%4") DF11_RSTEP4_G("%5")
                 "}"
                 : "+r"(x), "+l"(g.p), "+r"(acc[0]), "+r"(acc[1]), "+r"(acc[2]), "+r"(acc[3])
                 : "r"(tbl), "l"(g.last)
                 : "memory");
}
#undef DF11_RSTEP4_G
#undef DF11_RSTEP_G
#undef DF11_RSTEP4
#undef DF11_RSTEP

// Asynchronous copy (cp.async) of a block's words [bw0, bw1) into a warp
// buffer at shared address buf: from the 16-byte boundary at or below bw0 to
// the one at or above bw1 (inside the array's 8-word padding), one commit
// group.  A block spanning more than cap words from that boundary (big(), and
// inconsistent offsets) is not copied: its words are asked into L2 and read
// from global memory.  Returns the index of the buffer's first word.
__device__ __forceinline__ bool big_block(const RansParams &p, uint32_t bw1, uint32_t w0) { return bw1 - w0 > p.cap; }

template <bool BIG>
__device__ __forceinline__ uint32_t copy_words(const RansParams &p, uint32_t bw0, uint32_t bw1, int lane,
                                               uint32_t buf)
{
    const uint32_t w0 = bw0 & ~7u;
    uint32_t w1 = (bw1 + 7u) & ~7u;
    w1 = w1 < p.words_end ? w1 : p.words_end;
    if (!BIG || !big_block(p, bw1, w0)) {
        // (without BIG, inconsistent offsets: what fits the buffer)
        const uint32_t w1c = w1 <= w0 ? w0 : (w1 - w0 <= p.cap ? w1 : w0 + p.cap);
        for (uint32_t o = 8u * (uint32_t)lane; w0 + o < w1c; o += 256u)
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(buf + 2u * o), "l"(p.words + w0 + o)
                         : "memory");
    } else if (lane == 0 && w1 > w0) {
        const uint32_t bytes = w1 - w0 < 32768u ? 2u * (w1 - w0) : 65536u;
        asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p.words + w0), "r"(bytes) : "memory");
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
    return w0;
}

// The 16 sign/mantissa bytes at pos (a multiple of 16), or zeros past the end.
__device__ __forceinline__ uint4 load_sm(const RansParams &p, uint64_t pos)
{
    return pos < p.n ? __ldg(reinterpret_cast<const uint4 *>(p.sm + pos)) : make_uint4(0u, 0u, 0u, 0u);
}

// DYN: blocks as contiguous ranges per CTA handed out by a shared-memory
// counter; otherwise strided over the stream (balanced when the last round
// is nearly full).  BIG: the stream has blocks larger than the warp buffers
// (they read their words from global memory); without it such a block is
// inconsistent data.
template <bool DYN, bool BIG>
__global__ void __launch_bounds__(kMaxWarps * 32, 1) rans_decode_kernel(const RansParams p)
{
    __shared__ uint32_t table[kSlots];
    __shared__ uint32_t cum[257];
    __shared__ uint32_t next_block;
    extern __shared__ __align__(16) uint16_t wbufs[];  // per warp: two buffers of cap words
    const uint32_t tid = threadIdx.x, warp = tid >> 5;
    const int lane = (int)(tid & 31u);

    if (DYN && tid == 0)  // published by the barriers below
        next_block = (uint32_t)(((uint64_t)p.num_blocks * blockIdx.x) / gridDim.x) + (blockDim.x >> 5);
    // cumulative frequencies (one warp: 8 per lane, shuffle scan)
    if (warp == 0) {
        uint32_t f[8], s = 0;
#pragma unroll
        for (int k = 0; k < 8; k++) {
            f[k] = p.freq[8 * lane + k];
            s += f[k];
        }
        uint32_t incl = s;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const uint32_t y = __shfl_up_sync(0xffffffffu, incl, d);
            if (lane >= d)
                incl += y;
        }
        uint32_t c = incl - s;
#pragma unroll
        for (int k = 0; k < 8; k++) {
            cum[8 * lane + k] = c;
            c += f[k];
        }
        if (lane == 31)
            cum[256] = c;
    }
    __syncthreads();
    // slot -> entry: the exponent whose range holds the slot (binary search)
    for (uint32_t slot = tid; slot < kSlots; slot += blockDim.x) {
        uint32_t lo = 0, hi = 256;  // cum[lo] <= slot < cum[hi]
#pragma unroll
        for (int k = 0; k < 8; k++) {
            const uint32_t mid = (lo + hi) >> 1;
            if (cum[mid] <= slot)
                lo = mid;
            else
                hi = mid;
        }
        const uint32_t f = cum[lo + 1] - cum[lo];
        table[slot] = ror8(lo) | ((slot - cum[lo]) << 8) | (((f - 1u) & 0xFFFu) << 20);
    }
    __syncthreads();
    if (cum[256] != kSlots) {  // the model does not sum to 2^12
        if (tid == 0)
            atomicOr(p.status, (uint32_t)DF11_ERR_CORRUPT);
        return;
    }

    const uint64_t B = 512ull * p.chunks;
    const uint32_t warps = blockDim.x >> 5;
    uint16_t *wbuf = wbufs + 2u * p.bufw * warp;
    const uint32_t wbuf_s = static_cast<uint32_t>(__cvta_generic_to_shared(wbuf));
    const uint32_t tbl = static_cast<uint32_t>(__cvta_generic_to_shared(table));
    // with DYN the CTA's blocks are a contiguous range, and each warp takes
    // its first one here and every next one from a counter in shared memory;
    // otherwise the warps stride over the whole stream (when that leaves the
    // last round nearly full it is as balanced, and neighbouring warps read
    // neighbouring blocks)
    const uint32_t stride = gridDim.x * warps;
    const uint32_t b_end = DYN ? (uint32_t)(((uint64_t)p.num_blocks * (blockIdx.x + 1)) / gridDim.x) : p.num_blocks;
    uint32_t b = (DYN ? (uint32_t)(((uint64_t)p.num_blocks * blockIdx.x) / gridDim.x) : blockIdx.x * warps) + warp,
             k = 0;
    auto take_next = [&]() -> uint32_t {
        if (!DYN)
            return b + stride;
        uint32_t v = 0;
        if (lane == 0)
            v = atomicAdd(&next_block, 1u);
        return __shfl_sync(0xffffffffu, v, 0);
    };
    // software pipeline: the next block's state, lane count and word
    // offsets, and the next chunk's sign/mantissa bytes, are loaded one step
    // ahead
    uint32_t x_n = 0, c_n = 0, bw0_n = 0, bw1_n = 0, wfirst = 0;
    uint4 s_n = make_uint4(0u, 0u, 0u, 0u);
    if (b < b_end) {
        x_n = __ldg(p.states + 32ull * b + lane);
        c_n = __ldg(p.lane_words + 32ull * b + lane);
        bw0_n = __ldg(p.block_word + b);
        bw1_n = __ldg(p.block_word + b + 1);
        wfirst = copy_words<BIG>(p, bw0_n, bw1_n, lane, wbuf_s);
        s_n = load_sm(p, b * B + 16u * (uint32_t)lane);
    }
    uint32_t nb = 0;
    for (; b < b_end; b = nb, k ^= 1u) {
        // this block's words have landed; the next block's go to the other buffer
        asm volatile("cp.async.wait_group 0;" ::: "memory");
        __syncwarp();
        const uint32_t wb_s = wbuf_s + 2u * p.bufw * k;
        uint32_t x = x_n;
        // the lane's stream: after the streams of the lanes below it
        uint32_t incl = c_n;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const uint32_t y = __shfl_up_sync(0xffffffffu, incl, d);
            if (lane >= d)
                incl += y;
        }
        const uint32_t total = __shfl_sync(0xffffffffu, incl, 31);
        const uint32_t first = (bw0_n - wfirst) + (incl - c_n);  // bw0 - wfirst = bw0 mod 8
        const uint32_t end = first + c_n;                          // words, from the buffer's start
        const bool big = BIG && big_block(p, bw1_n, wfirst);  // warp-uniform: words in global memory
        bool bad = total != bw1_n - bw0_n || (!BIG && big_block(p, bw1_n, wfirst));
        uint32_t wp = wb_s + 2u * (first < p.cap ? first : p.cap);  // clamped: inconsistent counts
        // big block: the lane's stream in global memory (every load clamped
        // to the array, next_word)
        const uint64_t gfirst = (uint64_t)wfirst + first, wbase = reinterpret_cast<uint64_t>(p.words);
        GlobalWords wg{wbase + 2u * (gfirst < p.words_end ? gfirst : p.words_end), wbase + 2u * (p.words_end - 1u)};
        const uint64_t wg_end = wbase + 2u * ((uint64_t)wfirst + end);
        const bool full = (b + 1) * B <= p.n;  // warp-uniform
        nb = take_next();
        if (nb < b_end) {
            x_n = __ldg(p.states + 32ull * nb + lane);
            c_n = __ldg(p.lane_words + 32ull * nb + lane);
            bw0_n = __ldg(p.block_word + nb);
            bw1_n = __ldg(p.block_word + nb + 1);
            wfirst = copy_words<BIG>(p, bw0_n, bw1_n, lane, wbuf_s + 2u * p.bufw * (k ^ 1u));
            const uint64_t s0 = nb * B, s1 = s0 + B < p.n ? s0 + B : p.n;
            if (lane == 0)
                asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p.sm + s0),
                             "r"((uint32_t)(((s1 - s0) + 15) & ~15ull))
                             : "memory");
        }
        for (uint32_t j = 0; j < p.chunks; j++) {
            const uint64_t pos0 = b * B + 512ull * j + 16u * (uint32_t)lane;
            const uint4 s4 = s_n;
            s_n = load_sm(p, j + 1 < p.chunks ? pos0 + 512
                                              : (!DYN || nb < b_end ? (uint64_t)nb * B + 16u * (uint32_t)lane : p.n));
            uint32_t acc[4] = {0u, 0u, 0u, 0u};
            if (!BIG || !big) {
                if (full)
                    decode_chunk_full(x, wp, tbl, acc);
                else
                    decode_chunk_tail(x, wp, pos0, table, p, acc);
            } else {
                if (full)
                    decode_chunk_full(x, wg, tbl, acc);
                else
                    decode_chunk_tail(x, wg, pos0, table, p, acc);
            }
            // merge with the 16 sign/mantissa bytes and store
            if (pos0 + 16 <= p.n) {
                uint32_t r[8];
                merge4(s4.x, acc[0], r[0], r[1]);
                merge4(s4.y, acc[1], r[2], r[3]);
                merge4(s4.z, acc[2], r[4], r[5]);
                merge4(s4.w, acc[3], r[6], r[7]);
                if (p.wide) {
                    asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p.dst + pos0),
                                 "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]),
                                 "r"(r[7])
                                 : "memory");
                } else {
                    uint4 *d = reinterpret_cast<uint4 *>(p.dst + pos0);
                    d[0] = make_uint4(r[0], r[1], r[2], r[3]);
                    d[1] = make_uint4(r[4], r[5], r[6], r[7]);
                }
            } else {
#pragma unroll
                for (int i = 0; i < 16; i++)
                    if (pos0 + i < p.n)
                        p.dst[pos0 + i] = merge1(p.sm[pos0 + i], (acc[i >> 2] >> (8 * (i & 3))) & 0xFFu);
            }
        }
        bad = bad || x != kLow || (big ? wg.p != wg_end : wp != wb_s + 2u * end);
        if (__any_sync(0xffffffffu, bad) && lane == 0)
            atomicOr(p.status, (uint32_t)DF11_ERR_CORRUPT);
        __syncwarp();  // every lane is done with this buffer before it is refilled
    }
}

std::mutex g_rans_mu;
int g_rans_sms[64] = {0};
int g_rans_optin[64] = {0};
uint32_t g_rans_granted[4][64] = {};  // [DYN + 2 BIG][device]

}  // namespace

extern "C" df11_status df11_rans_decompress(const df11_rans_arrays *a, uint16_t *dst, uint32_t *status_dev,
                                            void *stream)
{
    if (!a || !status_dev)
        return DF11_ERR_INVALID_ARG;
    if (a->n == 0)
        return DF11_OK;
    if (!dst || (reinterpret_cast<uintptr_t>(dst) & 15) || !a->words || (reinterpret_cast<uintptr_t>(a->words) & 15) ||
        !a->states || !a->block_word || !a->lane_words || !a->freq ||
        !a->packed_sign_mantissa || (reinterpret_cast<uintptr_t>(a->packed_sign_mantissa) & 15))
        return DF11_ERR_INVALID_ARG;
    if (a->prob_bits != kProbBits || a->chunks < 1 || a->chunks > 15 || a->n >= (1ull << 32))
        return DF11_ERR_INVALID_ARG;
    const uint64_t B = 512ull * a->chunks;
    if (a->num_blocks != (a->n + B - 1) / B || a->num_words + 8 >= (1ull << 32) ||
        a->packed_sign_mantissa_bytes < ((a->n + 15) / 16) * 16)
        return DF11_ERR_INVALID_ARG;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        return DF11_ERR_CUDA;
    int sms = 0, optin = 0;
    {
        std::lock_guard<std::mutex> lock(g_rans_mu);
        if (!g_rans_sms[dev] &&
            (cudaDeviceGetAttribute(&g_rans_sms[dev], cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
             cudaDeviceGetAttribute(&g_rans_optin[dev], cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess))
            return DF11_ERR_CUDA;
        sms = g_rans_sms[dev];
        optin = g_rans_optin[dev];
    }
    RansParams p;
    p.words = a->words;
    p.states = a->states;
    p.block_word = a->block_word;
    p.lane_words = a->lane_words;
    p.freq = a->freq;
    p.sm = a->packed_sign_mantissa;
    p.dst = dst;
    p.status = status_dev;
    p.n = a->n;
    p.num_blocks = a->num_blocks;
    p.chunks = a->chunks;
    p.wide = (reinterpret_cast<uintptr_t>(dst) & 31) == 0;
    p.words_end = (uint32_t)((a->num_words & ~7ull) + 8);
    // two buffers per warp of cap words plus the slack a lane's reads past
    // its clamped start need (16 words per chunk); cap holds the largest
    // block unless that leaves room for fewer than 32 warps: then the few
    // larger blocks read their words from global memory
    const uint32_t slack = 16u * p.chunks + 8u;
    const uint64_t room = (uint64_t)optin - sizeof(uint32_t) * (kSlots + 257) - 1024;
    const uint64_t cap_all = ((uint64_t)a->max_block_words + 16u + 7u) & ~7ull;
    const uint64_t cap_32 = room / (4ull * kMaxWarps) > slack + 256u ? (room / (4ull * kMaxWarps) - slack) & ~7ull : 256u;
    p.cap = (uint32_t)(cap_all < cap_32 ? cap_all : cap_32);
    p.bufw = p.cap + slack;
    const uint64_t per_warp = 4ull * p.bufw;
    const uint64_t warps = room / per_warp < (uint64_t)kMaxWarps ? room / per_warp : (uint64_t)kMaxWarps;
    if (warps == 0)
        return DF11_ERR_INVALID_ARG;  // cannot happen for chunks <= 64 (at most 24,576 words per block)
    const uint64_t dyn = per_warp * warps;
    uint32_t grid = (uint32_t)((a->num_blocks + warps - 1) / warps);
    if (grid > (uint32_t)sms)
        grid = (uint32_t)sms;
    // striding when its last round is at least 85 % full, else ranges per CTA
    const uint64_t W = (uint64_t)grid * warps, rem = a->num_blocks % W;
    const int di = (rem != 0 && rem * 100 < W * 85) ? 1 : 0;
    const bool big = cap_all > p.cap;
    static void (*const kernels[4])(RansParams) = {rans_decode_kernel<false, false>, rans_decode_kernel<true, false>,
                                                   rans_decode_kernel<false, true>, rans_decode_kernel<true, true>};
    const int ki = di + (big ? 2 : 0);
    auto kern = kernels[ki];
    {
        std::lock_guard<std::mutex> lock(g_rans_mu);
        if (dyn > g_rans_granted[ki][dev]) {
            if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dyn) != cudaSuccess)
                return DF11_ERR_CUDA;
            g_rans_granted[ki][dev] = (uint32_t)dyn;
        }
    }
    kern<<<grid, (uint32_t)(warps * 32), (size_t)dyn, reinterpret_cast<cudaStream_t>(stream)>>>(p);
    return cudaGetLastError() == cudaSuccess ? DF11_OK : DF11_ERR_CUDA;
}
