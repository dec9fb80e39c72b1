// df11_decode.cu -- sm_100a kernel that rebuilds BF16 weights from DF11.
//
// "DFloat11: Kompresi inferensi GPU lossless ..." (id.news.hada.io/topic?id=20542):
//   "Decoding berbasis LUT hierarkis"  -- codes are resolved by table lookup
//        instead of a bit-by-bit tree walk; the tree is cut into height-8
//        subtrees stored as 256-entry LUTs whose values 240..255 are pointers;
//   "Kernel GPU 2 tahap dan metadata bantu" -- one thread per 8-byte segment
//        of EncodedExponent, starting at the segment's Gap; the number of codes
//        of each thread, prefix-summed over the thread block and added to the
//        block's stored output position, gives each thread its first output
//        index; exponents are placed in an on-chip write buffer and the block's
//        outputs leave in one coalesced write;
//   "Format DFloat11" -- sign and mantissa come verbatim from
//        PackedSignMantissa.
//
// B200 design (what differs from the page's kernel):
//   * the format's thread block is one warp (T = 64 segments by default; lane
//     l decodes segments l and l + 32 as two independent chains, which keeps
//     two lookups in flight per thread): a block's prefix sum is five warp
//     shuffles and its buffers are private to the warp, so warps never wait
//     for one another -- no block-wide barrier after set-up.  One persistent
//     CTA per SM takes a contiguous range of blocks, and its warps take them
//     one at a time from a counter in shared memory, so that they finish
//     within about one block of each other;
//   * decode once, not twice: the page counts the codes of every segment in
//     a first pass and decodes them again in a second.  Here every chain
//     decodes once into a private staging slot in shared memory (slots 68
//     bytes apart, so the 32 lanes of a warp store to distinct banks), its
//     code count falls out of that pass, and after the warp prefix sum each
//     chain copies its slot into the block's write buffer a 32-bit word at a
//     time;
//   * the CTA stages the page's LUTs and CodeLengths once and derives from
//     them a symbol table over the next 12 bits of the stream: up to 3 whole
//     codes, their total length and their exponents (~3 exponents per shared
//     memory lookup).  Exponents are stored rotated right by one bit, which
//     turns the final BF16 merge into two bit-selects and two byte permutes
//     per 4 elements.  Codes longer than 12 bits fall back to the page's
//     pointer-chasing LUTs;
//   * a chain ends exactly at its last code: the next segment's Gap gives the
//     bit where the next chain starts; the chain's window reads zeros past
//     that bit, the decode loop runs until the position passes it, and the
//     codes the zeros form (the all-zero code is the canonical first code;
//     at most two per chain) are discounted;
//   * each chain's 64 + 32 bits live in a three-register shift window: the
//     table index is the top 12 bits, a step is three funnel shifts;
//   * the decode loop is hand-written PTX: both chains of a lane step in one
//     predicated loop; right shifts by constants that are off the loop's
//     dependency chain are written as mul.hi (x >> k == mul.hi(x, 2^(32-k))),
//     which runs on the FMA pipe and leaves the integer ALU pipe to the
//     funnel shifts and compares;
//   * the next block's stream words, Gaps words and offsets are loaded into
//     registers while the current block is decoded; the current block's
//     sign/mantissa bytes are prefetched into L2 (one bulk prefetch by the
//     TMA unit) when its decoding starts and read from there by the merge,
//     which keeps shared memory for 32 warps per SM: their number, not a
//     staging copy, hides the load latency;
//   * the merge writes 16 outputs per lane with one 32-byte store when the
//     output is 32-byte aligned (a warp's stores then cover 1 KB contiguous);
//   * df11_decompress_sms caps the persistent grid below one CTA per SM, so
//     that kernels on other streams (the use of the previous transformer
//     block) can run beside the decode.
// Every loop is bounded; inconsistent data sets a status word, never traps.
#include "df11.h"
#include "df11_block.cuh"

#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <vector>

namespace {

// One matrix of a fused decode + matrix-vector product: rows x cols,
// row-major, elements [off, end) of the stream; its rows are numbered
// rowbase.. across the launch's matrices.
struct GemvMat {
    uint32_t end, off, cols, rowbase;
    const uint16_t *x;  // cols BF16 activations
    float *y;           // rows outputs, accumulated
};
constexpr uint32_t kMaxGemvMats = 16;

struct Params {
    const uint8_t *stream;
    const uint8_t *sm;
    const uint32_t *gaps;  // the uint64 Gaps words read as little-endian halves
    const uint32_t *offs;
    const uint8_t *luts;
    const uint8_t *cl;
    const uint32_t *sym_table;  // optional stored symbol table (null: derived per CTA)
    uint16_t *dst;
    uint32_t *status;
    uint64_t n;
    uint64_t total_bits;
    uint64_t nseg;
    uint32_t nblocks;
    uint32_t num_luts;
    uint32_t cap;  // bytes of one warp's exponent (and sign/mantissa) buffer
    uint32_t wide;  // dst is 32-byte aligned: the merge uses 32-byte stores
    uint32_t max_ctas;  // 0 = one CTA on every SM
    uint32_t min_code_len;  // from the stream's arrays: 0 when not known
    uint32_t num_mats;  // fused matrix-vector product (MODE 1) only
    GemvMat mats[kMaxGemvMats];
};

// Matrix of the fused product holding stream element g (matrices in order).
__device__ __forceinline__ uint32_t gemv_matrix(const Params &p, uint32_t g)
{
    uint32_t m = 0;
    while (m + 1 < p.num_mats && g >= p.mats[m].end)
        m++;
    return m;
}

__device__ __forceinline__ float bf16_lo(uint32_t two) { return __uint_as_float(two << 16); }

// Sums v over each run of lanes that hold the same key (a run's key is not
// used by any other lane) and adds the sum to *y from the run's first lane
// (y may be null: nothing to add).  When every lane holds the same key, a
// plain butterfly sum and one atomic add.
__device__ __forceinline__ void add_runs(float v, uint32_t key, float *y, int lane)
{
    if (__all_sync(0xffffffffu, key == __shfl_sync(0xffffffffu, key, 0))) {
#pragma unroll
        for (int d = 16; d >= 1; d >>= 1)
            v += __shfl_xor_sync(0xffffffffu, v, d);
        if (lane == 0 && y)
            atomicAdd(y, v);
        return;
    }
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const float o = __shfl_down_sync(0xffffffffu, v, d);
        const uint32_t k = __shfl_down_sync(0xffffffffu, key, d);
        if (lane + d < 32 && k == key)
            v += o;
    }
    const uint32_t before = __shfl_up_sync(0xffffffffu, key, 1);
    if ((lane == 0 || before != key) && y)
        atomicAdd(y, v);
}

// v += the dot product of 8 BF16 pairs (w[j], x[j]) held two per word, by
// the mixed-precision FMA (BF16 operands, fp32 addend and result; the BF16
// product is exact in fp32, so each step rounds once, as an fp32 FMA of the
// widened operands does).
__device__ __forceinline__ float dot16_bf16(float v, const uint32_t w[8], const uint32_t x[8])
{
#pragma unroll
    for (int j = 0; j < 8; j++)
        asm("{\n\t.reg .b16 wl, wh, xl, xh;\n\t"
            "mov.b32 {wl, wh}, %1;\n\t"
            "mov.b32 {xl, xh}, %2;\n\t"
            "fma.rn.f32.bf16 %0, wl, xl, %0;\n\t"
            "fma.rn.f32.bf16 %0, wh, xh, %0;\n\t}"
            : "+f"(v)
            : "r"(w[j]), "r"(x[j]));
    return v;
}

// Fused use of one decoded block (MODE 1): y += W x for the block's outputs
// [g0 + lo_off, g0 + hi), instead of storing them.  16 elements per lane and
// step (a 16-element chunk never crosses a row: columns and matrix sizes are
// multiples of 16); products in fp32, summed per row over the warp, one
// atomic add per row and step.  The ragged first and last chunks: one element
// per lane.
__device__ __forceinline__ void gemv_block(const Params &p, uint64_t g0, uint32_t lo_off, uint32_t hi,
                                           const uint8_t *exp_s, int lane)
{
    const uint8_t *smg = p.sm + g0;
    const uint32_t c_first = lo_off ? 1u : 0u, c_end = hi >> 4;  // full chunks [c_first, c_end)
    // the lane's chunks are 512 elements apart: its matrix, row and column
    // from one division, then advanced step by step
    uint32_t m = 0, row = 0, col = 0;
    {
        const uint32_t g = (uint32_t)(g0 + 16 * (c_first + lane));
        m = gemv_matrix(p, g);
        const uint32_t rel = g - p.mats[m].off;
        row = rel / p.mats[m].cols;
        col = rel - row * p.mats[m].cols;
    }
    for (uint32_t base = c_first; base < c_end; base += 32) {
        const uint32_t c = base + lane;
        float v = 0.f;
        uint32_t key = 0xFFFFFFFFu - lane;  // lanes without a chunk: runs of one, nothing to add
        float *y = nullptr;
        if (c < c_end) {
            const uint32_t l0 = 16 * c;
            const GemvMat &M = p.mats[m];
            const uint4 s4 = __ldg(reinterpret_cast<const uint4 *>(smg + l0));
            const uint4 e4 = *reinterpret_cast<const uint4 *>(exp_s + l0);
            uint32_t w[8];
            merge4(s4.x, e4.x, w[0], w[1]);
            merge4(s4.y, e4.y, w[2], w[3]);
            merge4(s4.z, e4.z, w[4], w[5]);
            merge4(s4.w, e4.w, w[6], w[7]);
            const uint4 *xp = reinterpret_cast<const uint4 *>(M.x + col);
            const uint4 xa = __ldg(xp), xb = __ldg(xp + 1);
            const uint32_t xw[8] = {xa.x, xa.y, xa.z, xa.w, xb.x, xb.y, xb.z, xb.w};
            v = dot16_bf16(v, w, xw);
            key = 2 * (M.rowbase + row);
            y = M.y + row;
            // next chunk of this lane: 512 elements on
            const uint32_t g = (uint32_t)(g0 + l0) + 512u;
            if (g < M.end) {
                col += 512u;
                while (col >= M.cols) {  // at most 512 / cols + 1 steps
                    col -= M.cols;
                    row++;
                }
            } else if (c + 32 < c_end) {
                m = gemv_matrix(p, g);
                const uint32_t rel = g - p.mats[m].off;
                row = rel / p.mats[m].cols;
                col = rel - row * p.mats[m].cols;
            }
        }
        add_runs(v, key, y, lane);
    }
    // ragged chunks: lanes 0..15 the first, lanes 16..31 the last; the two
    // halves get distinct keys even for the same row (runs must be unique)
    {
        const bool head = lane < 16;
        const uint32_t l = head ? lane : 16 * c_end + (lane - 16);
        const bool want = head ? (lo_off != 0 || hi < 16) : (c_end > 0 && (hi & 15u) != 0);
        float v = 0.f;
        uint32_t key = 0xFFFFFFFFu - lane;
        float *y = nullptr;
        if (want && l >= lo_off && l < hi) {
            const uint32_t g = (uint32_t)(g0 + l);
            const GemvMat &M = p.mats[gemv_matrix(p, g)];
            const uint32_t rel = g - M.off, row = rel / M.cols, col = rel - row * M.cols;
            const uint32_t wbits = merge1(smg[l], exp_s[l]);
            v = bf16_lo(wbits) * bf16_lo(M.x[col]);
            key = 2 * (M.rowbase + row) + (head ? 0u : 1u);
            y = M.y + row;
        }
        add_runs(v, key, y, lane);
    }
}

// A warp's copy of one format block's metadata in shared memory (byte
// offsets): the stream bytes of its 32 C segments plus the 16 the last chain
// reads beyond, the 5 C + 1 Gaps words holding its fields and the next
// block's first, and its two BlockOffset entries.
template <int C>
struct NextBuf {
    static constexpr uint32_t stream = 0;
    static constexpr uint32_t gaps = 256 * C + 16;
    static constexpr uint32_t offs = (gaps + 4 * (5 * C + 1) + 7) & ~7u;  // read as one 8-byte word
    static constexpr uint32_t bytes = (offs + 8 + 15) & ~15u;
    // 16-byte cp.async targets at multiples of 16, the 8-byte load at a multiple of 8
    static_assert(stream % 16 == 0 && gaps % 16 == 0 && offs % 8 == 0 && bytes % 16 == 0, "alignment");
};

// Asynchronous copy (cp.async, no registers held) of format block b's
// metadata into the warp's buffer at shared address buf; every lane of the
// warp takes part, one commit group per block.  The stream bytes go in
// 16-byte pieces (the stream array is 16-byte aligned and padded by 16
// bytes), Gaps and BlockOffset words in 4-byte pieces: every source lies
// inside its array (checked by stream_params on the host).
template <int C>
__device__ __forceinline__ void prefetch_block(const Params &p, uint32_t b, int lane, uint32_t buf)
{
    const uint8_t *st = p.stream + (uint64_t)(256 * C) * b;
    if (lane < 16 * C)
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(buf + 16u * lane), "l"(st + 16 * lane)
                     : "memory");
    if (lane == 31)
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(buf + 256u * C), "l"(st + 256 * C)
                     : "memory");
    const uint32_t *g = p.gaps + (uint64_t)(5 * C) * b;
    if (lane <= 5 * C)
        asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(buf + NextBuf<C>::gaps + 4u * lane),
                     "l"(g + lane)
                     : "memory");
    if (lane >= 30)
        asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(buf + NextBuf<C>::offs + 4u * (lane - 30)),
                     "l"(p.offs + b + (lane - 30))
                     : "memory");
    asm volatile("cp.async.commit_group;" ::: "memory");
}

// The registers of one block (what load_block would load) from the warp's
// buffer, once its copy has landed; the buffer is free again on return.
template <int C>
__device__ __forceinline__ void read_block(uint32_t buf, int lane, BlockRegs<C> &r)
{
    asm volatile("cp.async.wait_group 0;" ::: "memory");
    __syncwarp();
    const uint32_t L = (5u * (uint32_t)lane) >> 5;
#pragma unroll
    for (int k = 0; k < C; k++) {
        const uint32_t a = buf + 8u * (lane + 32 * k);
        asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(r.s01[k].x), "=r"(r.s01[k].y) : "r"(a));
        asm volatile("ld.shared.u32 %0, [%1];" : "=r"(r.s2[k]) : "r"(a + 8));
        const uint32_t ga = buf + NextBuf<C>::gaps + 4u * (5 * k + L);
        asm volatile("ld.shared.u32 %0, [%1];" : "=r"(r.g0[k]) : "r"(ga));
        asm volatile("ld.shared.u32 %0, [%1];" : "=r"(r.g1[k]) : "r"(ga + 4));
    }
    asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(r.o0), "=r"(r.o1) : "r"(buf + NextBuf<C>::offs));
    __syncwarp();
}

// The merge of up to four 16-element chunks of one lane, in PTX: chunk k
// (k < nit) has its 16 sign/mantissa bytes at sp + 512 k (global), its
// rotated exponents at ea + 512 k (shared) and its 16 outputs at dp + 1024 k
// (32-byte aligned).  Two sign/mantissa loads are in flight: chunks 0 and 1
// first, chunk 2 into chunk 0's registers once that is merged, chunk 3 into
// chunk 1's.  Per 4 elements two bit-selects and two byte permutes (as
// merge4); the merged words overwrite their inputs.
#define DF11_MERGE4(S, E)                                  \
    "lop3.b32 h, " S ", " E ", 0x80808080, 0xE4;\n\t"    \
    "lop3.b32 l, " E ", " S ", 0x80808080, 0xE4;\n\t"    \
    "prmt.b32 " S ", l, h, 0x5140;\n\t"                  \
    "prmt.b32 " E ", l, h, 0x7362;\n\t"
#define DF11_CHUNK(Q, A, OFFE, OFFD)                                                                        \
    "@" Q " ld.shared.v4.b32 {e0, e1, e2, e3}, [%2+" OFFE "];\n\t"                                      \
    DF11_MERGE4(A "0", "e0") DF11_MERGE4(A "1", "e1") DF11_MERGE4(A "2", "e2") DF11_MERGE4(A "3", "e3")   \
    "@" Q " st.global.v8.b32 [%1+" OFFD "], {" A "0, e0, " A "1, e1, " A "2, e2, " A "3, e3};\n\t"
__device__ __forceinline__ void merge_chunks4(const uint8_t *sp, uint16_t *dp, uint32_t ea, uint32_t nit)
{
    asm volatile(
        "{\n\t"
        ".reg .pred q0, q1, q2, q3;\n\t"
        ".reg .b32 a0, a1, a2, a3, b0, b1, b2, b3, e0, e1, e2, e3, h, l;\n\t"
        "setp.gt.u32 q0, %3, 0;\n\t"
        "setp.gt.u32 q1, %3, 1;\n\t"
        "setp.gt.u32 q2, %3, 2;\n\t"
        "setp.gt.u32 q3, %3, 3;\n\t"
        "@q0 ld.global.nc.v4.b32 {a0, a1, a2, a3}, [%0];\n\t"
        "@q1 ld.global.nc.v4.b32 {b0, b1, b2, b3}, [%0+512];\n\t"
        DF11_CHUNK("q0", "a", "0", "0")
        "@q2 ld.global.nc.v4.b32 {a0, a1, a2, a3}, [%0+1024];\n\t"
        DF11_CHUNK("q1", "b", "512", "1024")
        "@q3 ld.global.nc.v4.b32 {b0, b1, b2, b3}, [%0+1536];\n\t"
        DF11_CHUNK("q2", "a", "1024", "2048")
        DF11_CHUNK("q3", "b", "1536", "3072")
        "}"
        ::"l"(sp), "l"(dp), "r"(ea), "r"(nit)
        : "memory");
}
#undef DF11_CHUNK
#undef DF11_MERGE4

// Per-warp shared memory of a launch: the write buffer, the staging slots
// and, with short slots, the metadata buffer of the next block.
template <int C, uint32_t SLOT>
__host__ __device__ constexpr uint32_t warp_bytes(uint32_t cap)
{
    return Smem::per_warp(cap, SLOT) + (SLOT == kSlotShort ? NextBuf<C>::bytes : 0u);
}

// C = segments per lane: the format block is 32 * C segments, one warp; lane
// l decodes segments l, l + 32, ... as C independent chains.  WARPS warps per
// CTA, one CTA per SM.  SLOT: bytes of a chain's staging slot (kSlotShort
// when no code is 1 bit long; the kernel checks that and reports
// DF11_ERR_CORRUPT otherwise); with short slots the next block's metadata is
// copied into shared memory by cp.async, with long slots it is loaded into
// registers.
// MODE 0: store the BF16 outputs; MODE 1: fused matrix-vector product.
template <int C, int WARPS, int MODE, uint32_t SLOT, uint32_t R>
__global__ void __launch_bounds__(WARPS * 32, 1) df11_decode_kernel(const Params p)
{
    static_assert(C == 1 || C == 2, "one or two chains per lane");
    constexpr int kWarps = WARPS, kThreads = WARPS * 32;
    constexpr bool kCopy = SLOT == kSlotShort;  // metadata by cp.async
    // the pending-word decode loop in both modes (the fused GEMM's decode
    // warps keep the byte-store loop)
    constexpr bool kWords = true;
    constexpr uint32_t kR = R;  // symbol-table copies (SmemR)
    using S = SmemR<kR>;
    extern __shared__ __align__(128) uint8_t smem[];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    uint8_t *exp_s = smem + S::bufs + warp * warp_bytes<C, SLOT>(p.cap);
    uint8_t *slots = exp_s + p.cap;
    const uint32_t nbuf = static_cast<uint32_t>(__cvta_generic_to_shared(slots + slot_bytes(SLOT)));

    // the CTA's blocks are a contiguous range; each warp takes its first one
    // here and every next one from a counter in shared memory, so that the
    // CTA's warps all finish within about one block of each other
    uint32_t &next_block = *reinterpret_cast<uint32_t *>(smem + S::ctr);
    const uint32_t b_end = (uint32_t)(((uint64_t)p.nblocks * (blockIdx.x + 1)) / gridDim.x);
    uint32_t b = (uint32_t)(((uint64_t)p.nblocks * blockIdx.x) / gridDim.x) + (uint32_t)warp;
    if (tid == 0)
        next_block = b + kWarps;  // published by the barriers in build_tables
    auto take_next = [&]() -> uint32_t {
        uint32_t v = 0;
        if (lane == 0)
            v = atomicAdd(&next_block, 1u);
        return __shfl_sync(0xffffffffu, v, 0);
    };
    // the first block's metadata arrives while the tables are set up: with
    // long slots into registers; with short slots copied into the warp's
    // buffer, unless the table is derived (its scratch overlaps the buffers)
    BlockRegs<C> cur, nxt;
    if (!kCopy && b < b_end)
        load_block<C>(p, b, lane, cur);
    const bool early = kCopy && p.sym_table != nullptr;  // uniform
    if (early && b < b_end)
        prefetch_block<C>(p, b, lane, nbuf);

    if (!build_tables<kWords, kR>(p.luts, p.cl, p.num_luts, p.sym_table, smem, (uint32_t)tid, (uint32_t)kThreads,
                      SLOT < kSlotLong ? 2u : 1u)) {
        if (tid == 0)
            atomicOr(p.status, (uint32_t)DF11_ERR_CORRUPT);
        asm volatile("cp.async.wait_all;" ::: "memory");  // no copy outlives the CTA
        return;
    }
    if (SLOT < kSlotLong) {
        // short slots hold a segment's codes only when no code is 1 bit long
        // (the all-zero code is the shortest: canonical codes)
        bool bad = false;
        const uint32_t lmin = lut_decode(0u, smem + S::luts, smem + S::cl, p.num_luts, &bad) >> 8;
        if (bad || lmin < 2) {
            if (tid == 0)
                atomicOr(p.status, (uint32_t)DF11_ERR_CORRUPT);
            asm volatile("cp.async.wait_all;" ::: "memory");
            return;
        }
    }
    // a derived table used the start of the per-warp buffers as scratch:
    // the first block's metadata is copied only now
    if (kCopy && !early && b < b_end)
        prefetch_block<C>(p, b, lane, nbuf);

    const uint32_t sym_base = static_cast<uint32_t>(__cvta_generic_to_shared(smem + S::sym));
    const uint32_t exp_base = static_cast<uint32_t>(__cvta_generic_to_shared(exp_s));
    const uint32_t slot_base = static_cast<uint32_t>(__cvta_generic_to_shared(slots)) + lane * SLOT;

    // ---- each warp decodes the blocks it takes; no block-wide barrier from here on
    for (uint32_t nb; b < b_end; b = nb) {
        nb = take_next();
        if (kCopy) {
            read_block<C>(nbuf, lane, cur);
            if (nb < b_end)
                prefetch_block<C>(p, nb, lane, nbuf);
        } else if (nb < b_end) {
            load_block<C>(p, nb, lane, nxt);
        }
        BlockOut bo;
        if (decode_block<C, SLOT, kWords, kR>(p, b, lane, cur, sym_base, exp_base, slot_base, bo)) {
            // ---- merge with sign/mantissa (from L2)
            const uint64_t g0 = bo.g0;
            const uint32_t lo_off = bo.lo_off, hi = bo.hi;
            const uint8_t *smg = p.sm + g0;
            if (MODE == 1) {
                gemv_block(p, g0, lo_off, hi, exp_s, lane);
            } else if (p.wide) {
                // 16 elements per lane and step, one 32-byte store: a warp's
                // stores cover 1 KB contiguous
                const uint32_t c_first = lo_off ? 1u : 0u, c_end = hi >> 4;  // full chunks [c_first, c_end)
                if (kCopy) {
                    // (registers free of the next block's metadata) up to
                    // four chunks of a lane per call
                    for (uint32_t c0 = c_first + (uint32_t)lane; c0 < c_end; c0 += 128u)
                        merge_chunks4(smg + 16u * c0, p.dst + g0 + 16u * c0, exp_base + 16u * c0,
                                      (c_end - c0 + 31u) >> 5);
                } else
#pragma unroll 2
                for (uint32_t c = c_first + lane; c < c_end; c += 32) {
                    const uint32_t l0 = 16 * c;
                    const uint4 s4 = __ldg(reinterpret_cast<const uint4 *>(smg + l0));
                    const uint4 e4 = *reinterpret_cast<const uint4 *>(exp_s + l0);
                    uint32_t r[8];
                    merge4(s4.x, e4.x, r[0], r[1]);
                    merge4(s4.y, e4.y, r[2], r[3]);
                    merge4(s4.z, e4.z, r[4], r[5]);
                    merge4(s4.w, e4.w, r[6], r[7]);
                    asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p.dst + g0 + l0),
                                 "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]),
                                 "r"(r[7])
                                 : "memory");
                }
                // partial first chunk (lanes 0..15) and partial last chunk
                // (lanes 16..31): one element per lane
                const bool head = lane < 16;
                const uint32_t l = head ? lane : 16 * c_end + (lane - 16);
                const bool want = head ? (lo_off != 0 || hi < 16) : (c_end > 0 && (hi & 15u) != 0);
                if (want && l >= lo_off && l < hi)
                    p.dst[g0 + l] = merge1(__ldg(smg + l), ld_u8(exp_base + l));
            } else {
                // 8 elements per lane and step, one 16-byte store: a warp's
                // stores cover 512 contiguous bytes
                const uint32_t u_first = (lo_off + 7u) >> 3, u_end = hi >> 3;  // full units [u_first, u_end)
#pragma unroll 4
                for (uint32_t u = u_first + lane; u < u_end; u += 32) {
                    const uint32_t l0 = 8 * u;
                    const uint2 s2 = __ldg(reinterpret_cast<const uint2 *>(smg + l0));
                    const uint2 e2 = *reinterpret_cast<const uint2 *>(exp_s + l0);
                    uint4 r;
                    merge4(s2.x, e2.x, r.x, r.y);
                    merge4(s2.y, e2.y, r.z, r.w);
                    *reinterpret_cast<uint4 *>(p.dst + g0 + l0) = r;
                }
                // the partial units before u_first (lanes 0..15) and from
                // u_end on (lanes 16..31): one element per lane
                const uint32_t head_end = 8 * u_first < hi ? 8 * u_first : hi;
                const uint32_t tail0 = 8 * (u_end > u_first ? u_end : u_first);
                const uint32_t l = lane < 16 ? (uint32_t)lane : tail0 + (lane - 16);
                const bool want = lane < 16 ? (l >= lo_off && l < head_end) : (lane < 24 && l < hi);
                if (want)
                    p.dst[g0 + l] = merge1(__ldg(smg + l), ld_u8(exp_base + l));
            }
            __syncwarp();
        }
        if (!kCopy)
            cur = nxt;
    }
}

// ------------------------------------------------------------- host side
// Per-device launch facts, looked up once: SM count and the opt-in shared
// memory limit; per kernel instantiation, the largest dynamic shared memory
// size already granted.
struct DeviceFacts {
    int sms = 0;
    int smem_optin = 0;
    uint32_t granted[2][2][2][5] = {};  // [MODE][C - 1][short slots][warps 32 / 24 / 16 / 8, 32 with 2 tables]
    cudaStream_t up = nullptr, down = nullptr;  // copy streams of the host path, made on first use
};
std::mutex g_mu;
DeviceFacts g_dev[64];

df11_status device_facts(DeviceFacts **out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        return DF11_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mu);
    DeviceFacts &f = g_dev[dev];
    if (!f.sms) {
        int sms = 0, optin = 0;
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
            return DF11_ERR_CUDA;
        f.smem_optin = optin;
        f.sms = sms;
    }
    *out = &f;
    return DF11_OK;
}

template <int C, int WARPS, int MODE, uint32_t SLOT, uint32_t R = 1>
df11_status launch_warps(const Params &prm, cudaStream_t stream, uint32_t smem, DeviceFacts *f, uint32_t &granted)
{
    auto kern = df11_decode_kernel<C, WARPS, MODE, SLOT, R>;
    if (smem > granted) {
        std::lock_guard<std::mutex> lock(g_mu);
        if (smem > granted) {
            if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
                return DF11_ERR_CUDA;
            granted = smem;
        }
    }
    // one persistent CTA per SM: __launch_bounds__(WARPS * 32, 1) and the
    // shared-memory footprint allow no second one
    uint64_t grid = (uint64_t)f->sms;
    if (prm.max_ctas && prm.max_ctas < grid)
        grid = prm.max_ctas;
    const uint64_t need = (prm.nblocks + WARPS - 1) / WARPS;
    if (grid > need)
        grid = need;
    kern<<<(unsigned)grid, WARPS * 32, smem, stream>>>(prm);
    return cudaGetLastError() == cudaSuccess ? DF11_OK : DF11_ERR_CUDA;
}

// As many warps per CTA (32, 24, 16 or 8) as the per-warp buffers allow in
// shared memory; blocks of very short codes hold up to 64 outputs per segment.
// Short staging slots when the stream states that no code is 1 bit long.
template <int C, int MODE, uint32_t SLOT>
df11_status launch_slots(const Params &prm, cudaStream_t stream, DeviceFacts *f)
{
    const uint32_t optin = (uint32_t)f->smem_optin;
    auto &g = f->granted[MODE][C - 1][SLOT == kSlotShort ? 1 : 0];
    const uint32_t wb = warp_bytes<C, SLOT>(prm.cap);
    // the rebuild to memory takes two copies of the symbol table (fewer bank
    // conflicts in its lookups) when 32 warps still fit beside them
    if (MODE == 0 && SmemR<2>::bufs + 32 * wb <= optin)
        return launch_warps<C, 32, MODE, SLOT, 2>(prm, stream, SmemR<2>::bufs + 32 * wb, f, g[4]);
    const uint32_t base = Smem::bufs;
    if (base + 32 * wb <= optin)
        return launch_warps<C, 32, MODE, SLOT>(prm, stream, base + 32 * wb, f, g[0]);
    if (base + 24 * wb <= optin)
        return launch_warps<C, 24, MODE, SLOT>(prm, stream, base + 24 * wb, f, g[1]);
    if (base + 16 * wb <= optin)
        return launch_warps<C, 16, MODE, SLOT>(prm, stream, base + 16 * wb, f, g[2]);
    if (base + 8 * wb <= optin)
        return launch_warps<C, 8, MODE, SLOT>(prm, stream, base + 8 * wb, f, g[3]);
    return DF11_ERR_INVALID_ARG;
}

template <int C, int MODE>
df11_status launch(const Params &prm, cudaStream_t stream)
{
    DeviceFacts *f = nullptr;
    df11_status st = device_facts(&f);
    if (st != DF11_OK)
        return st;
    return prm.min_code_len >= 2 ? launch_slots<C, MODE, kSlotShort>(prm, stream, f)
                                 : launch_slots<C, MODE, kSlotLong>(prm, stream, f);
}

}  // namespace

namespace {
df11_status decompress_impl(const df11_arrays *a, uint16_t *dst, uint32_t *status_dev, void *stream,
                            uint32_t max_sms)
{
    if (!a || !status_dev)
        return DF11_ERR_INVALID_ARG;
    if (a->n == 0)
        return DF11_OK;
    if (!dst || !aligned(dst, 16))
        return DF11_ERR_INVALID_ARG;
    Params prm;
    const df11_status st = stream_params(a, status_dev, prm);
    if (st != DF11_OK)
        return st;
    prm.dst = dst;
    prm.wide = aligned(dst, 32) ? 1u : 0u;
    prm.max_ctas = max_sms;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    return a->threads_per_block == 32 ? launch<1, 0>(prm, s) : launch<2, 0>(prm, s);
}

// Decodes format blocks [b0, b1) only: the stream, Gaps and BlockOffset
// pointers move to block b0 (its Gap fields start on a 32-bit boundary: 5 * 32
// and 5 * 64 bits per block); BlockOffset values, output and sign/mantissa
// stay absolute.  A range that ends before the stream's last block counts one
// segment more, so that its last chain ends at the next block's first Gap.
df11_status decompress_blocks(const df11_arrays *a, uint32_t b0, uint32_t b1, uint16_t *dst, uint32_t *status_dev,
                              cudaStream_t s)
{
    Params prm;
    const df11_status st = stream_params(a, status_dev, prm);
    if (st != DF11_OK)
        return st;
    if (b0 >= b1 || b1 > a->num_blocks)
        return DF11_ERR_INVALID_ARG;
    const uint64_t T = a->threads_per_block;
    prm.stream += b0 * T * 8;
    prm.gaps += (5 * T * b0) / 32;
    prm.offs += b0;
    prm.nblocks = b1 - b0;
    if (b1 < a->num_blocks) {
        prm.nseg = (uint64_t)(b1 - b0) * T + 1;
    } else {
        prm.nseg -= b0 * T;
        prm.total_bits -= 64 * b0 * T;
    }
    prm.dst = dst;
    prm.wide = aligned(dst, 32) ? 1u : 0u;
    return T == 32 ? launch<1, 0>(prm, s) : launch<2, 0>(prm, s);
}
}  // namespace

extern "C" df11_status df11_decompress(const df11_arrays *a, uint16_t *dst, uint32_t *status_dev, void *stream)
{
    return decompress_impl(a, dst, status_dev, stream, 0);
}

extern "C" df11_status df11_decompress_sms(const df11_arrays *a, uint16_t *dst, uint32_t *status_dev, void *stream,
                                           uint32_t max_sms)
{
    return decompress_impl(a, dst, status_dev, stream, max_sms);
}

extern "C" df11_status df11_decompress_host(const df11_arrays *h, const df11_arrays *d, uint16_t *dst_dev,
                                            uint16_t *dst_host, uint32_t *status_dev, void *stream)
{
    if (!h || !d || !dst_dev || !dst_host)
        return DF11_ERR_INVALID_ARG;
    if (d->encoded_exponent_bytes < h->encoded_exponent_bytes ||
        d->packed_sign_mantissa_bytes < h->packed_sign_mantissa_bytes || d->gaps_words < h->gaps_words)
        return DF11_ERR_INVALID_ARG;
    if (!h->encoded_exponent || !h->packed_sign_mantissa || !h->gaps || !h->block_offset || !h->luts ||
        !h->code_lengths || !d->encoded_exponent || !d->packed_sign_mantissa || !d->gaps || !d->block_offset ||
        !d->luts || !d->code_lengths)
        return DF11_ERR_INVALID_ARG;
    if (h->n == 0)
        return DF11_OK;
    df11_arrays dev = *h;  // same sizes, device pointers
    dev.encoded_exponent = d->encoded_exponent;
    dev.packed_sign_mantissa = d->packed_sign_mantissa;
    dev.gaps = d->gaps;
    dev.block_offset = d->block_offset;
    dev.luts = d->luts;
    dev.code_lengths = d->code_lengths;
    // the derived table travels with the other small arrays when both sides
    // have one; otherwise every CTA derives it
    dev.symbol_table = h->symbol_table && d->symbol_table ? d->symbol_table : nullptr;
    {
        Params check;  // the whole stream's arguments, before anything is queued
        const df11_status st = stream_params(&dev, status_dev, check);
        if (st != DF11_OK)
            return st;
        if (!aligned(dst_dev, 16))
            return DF11_ERR_INVALID_ARG;
    }
    DeviceFacts *f = nullptr;
    if (device_facts(&f) != DF11_OK)
        return DF11_ERR_CUDA;
    {
        std::lock_guard<std::mutex> lock(g_mu);
        if (!f->up && cudaStreamCreateWithFlags(&f->up, cudaStreamNonBlocking) != cudaSuccess)
            return DF11_ERR_CUDA;
        if (!f->down && cudaStreamCreateWithFlags(&f->down, cudaStreamNonBlocking) != cudaSuccess)
            return DF11_ERR_CUDA;
    }
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream), up = f->up, down = f->down;

    // Pieces of whole format blocks, ~8 Mi outputs each: piece k's arrays go
    // up on `up`, it decodes on `s`, its outputs come down on `down`, so the
    // copies of one piece overlap the decode of its neighbours.  A piece's
    // decode reads a few bytes past its last block (the stream's 16-byte
    // tail, the sign/mantissa bytes up to the next 16-byte boundary); the
    // next piece's uploads start where the previous ones ended, so no copy
    // rewrites bytes that a running decode reads.
    const uint32_t nb = h->num_blocks;
    const uint64_t per_piece = 8ull << 20;
    uint32_t pieces = (uint32_t)((h->n + per_piece - 1) / per_piece);
    pieces = pieces < 1 ? 1 : pieces;
    pieces = pieces > nb ? nb : pieces;
    const uint32_t *offs = h->block_offset;
    const uint64_t T = h->threads_per_block;
    cudaEvent_t start, done;
    std::vector<cudaEvent_t> evs;
    auto event = [&](cudaEvent_t *e) {
        if (cudaEventCreateWithFlags(e, cudaEventDisableTiming) != cudaSuccess)
            return false;
        evs.push_back(*e);
        return true;
    };
    auto cleanup = [&](df11_status st) {
        for (cudaEvent_t e : evs)
            cudaEventDestroy(e);  // released once their work completes
        return st;
    };
    if (!event(&start) || !event(&done))
        return cleanup(DF11_ERR_CUDA);
    uint64_t stream_done = 0, sm_done = 0;  // bytes uploaded so far, from 0
    bool ok = cudaEventRecord(start, s) == cudaSuccess && cudaStreamWaitEvent(up, start, 0) == cudaSuccess &&
              cudaStreamWaitEvent(down, start, 0) == cudaSuccess;
    // the small arrays whole, first
    ok = ok && cudaMemcpyAsync(const_cast<uint64_t *>(d->gaps), h->gaps, h->gaps_words * 8, cudaMemcpyHostToDevice,
                               up) == cudaSuccess;
    ok = ok && cudaMemcpyAsync(const_cast<uint32_t *>(d->block_offset), offs, (nb + 1) * 4ull,
                               cudaMemcpyHostToDevice, up) == cudaSuccess;
    ok = ok && cudaMemcpyAsync(const_cast<uint8_t *>(d->luts), h->luts, h->num_luts * 256ull, cudaMemcpyHostToDevice,
                               up) == cudaSuccess;
    ok = ok && cudaMemcpyAsync(const_cast<uint8_t *>(d->code_lengths), h->code_lengths, 256, cudaMemcpyHostToDevice,
                               up) == cudaSuccess;
    ok = ok && (!dev.symbol_table ||
                cudaMemcpyAsync(const_cast<uint32_t *>(d->symbol_table), h->symbol_table, 4096 * 4,
                                cudaMemcpyHostToDevice, up) == cudaSuccess);
    if (!ok)
        return cleanup(DF11_ERR_CUDA);
    for (uint32_t k = 0; k < pieces; k++) {
        uint32_t b0 = (uint32_t)((uint64_t)nb * k / pieces), b1 = (uint32_t)((uint64_t)nb * (k + 1) / pieces);
        if (b0 == b1)
            continue;
        // stream bytes of the blocks plus the 16 the last chain reads beyond,
        // from where the previous piece's upload ended
        const uint64_t s0 = std::max<uint64_t>(b0 * T * 8, stream_done);
        const uint64_t s1 = std::min<uint64_t>(b1 * T * 8 + 16, h->encoded_exponent_bytes);
        // the piece's outputs: BlockOffset entries clamped to n, so that a
        // corrupt host copy (which the kernel reports) cannot move a copy
        // outside the arrays
        const uint64_t e0 = std::min<uint64_t>(offs[b0], h->n), e1 = std::min<uint64_t>(offs[b1], h->n);
        // their sign/mantissa bytes, in whole 16-byte units, from where the
        // previous piece's upload ended
        const uint64_t m0 = std::max<uint64_t>(e0 & ~15ull, sm_done);
        const uint64_t m1 = std::min<uint64_t>((e1 + 15ull) & ~15ull, h->packed_sign_mantissa_bytes);
        cudaEvent_t in, dec;
        if (!event(&in) || !event(&dec))
            return cleanup(DF11_ERR_CUDA);
        ok = s1 <= s0 || cudaMemcpyAsync(const_cast<uint8_t *>(d->encoded_exponent) + s0, h->encoded_exponent + s0,
                                         s1 - s0, cudaMemcpyHostToDevice, up) == cudaSuccess;
        stream_done = std::max(stream_done, s1);
        sm_done = std::max(sm_done, m1);
        ok = ok && (m1 <= m0 || cudaMemcpyAsync(const_cast<uint8_t *>(d->packed_sign_mantissa) + m0,
                                                h->packed_sign_mantissa + m0, m1 - m0, cudaMemcpyHostToDevice,
                                                up) == cudaSuccess);
        ok = ok && cudaEventRecord(in, up) == cudaSuccess && cudaStreamWaitEvent(s, in, 0) == cudaSuccess;
        if (!ok)
            return cleanup(DF11_ERR_CUDA);
        const df11_status st = decompress_blocks(&dev, b0, b1, dst_dev, status_dev, s);
        if (st != DF11_OK)
            return cleanup(st);
        ok = cudaEventRecord(dec, s) == cudaSuccess && cudaStreamWaitEvent(down, dec, 0) == cudaSuccess;
        ok = ok && (e1 <= e0 || cudaMemcpyAsync(dst_host + e0, dst_dev + e0, (e1 - e0) * 2, cudaMemcpyDeviceToHost,
                                                down) == cudaSuccess);
        if (!ok)
            return cleanup(DF11_ERR_CUDA);
    }
    // the caller's stream resumes after the last outputs have come down
    ok = cudaEventRecord(done, down) == cudaSuccess && cudaStreamWaitEvent(s, done, 0) == cudaSuccess;
    return cleanup(ok ? DF11_OK : DF11_ERR_CUDA);
}

extern "C" df11_status df11_read_status(const uint32_t *status_dev, void *stream)
{
    if (!status_dev)
        return DF11_ERR_INVALID_ARG;
    uint32_t v = 0;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (cudaMemcpyAsync(&v, status_dev, 4, cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
        return DF11_ERR_CUDA;
    return v ? DF11_ERR_CORRUPT : DF11_OK;
}

extern "C" df11_status df11_decompress_gemv(const df11_arrays *a, const df11_gemv_matrix *mats, uint32_t num_mats,
                                            uint32_t *status_dev, void *stream)
{
    if (!a || !status_dev || !mats || num_mats < 1 || num_mats > kMaxGemvMats)
        return DF11_ERR_INVALID_ARG;
    Params prm;
    if (a->n == 0)
        return DF11_ERR_INVALID_ARG;  // no matrix has zero elements
    const df11_status st = stream_params(a, status_dev, prm);
    if (st != DF11_OK)
        return st;
    uint64_t off = 0, rows = 0;
    for (uint32_t m = 0; m < num_mats; m++) {
        const df11_gemv_matrix &M = mats[m];
        if (M.rows == 0 || M.cols == 0 || M.cols % 16 || !M.x || !M.y || !aligned(M.x, 16) || !aligned(M.y, 4))
            return DF11_ERR_INVALID_ARG;
        const uint64_t size = (uint64_t)M.rows * M.cols;
        prm.mats[m].off = (uint32_t)off;
        off += size;
        if (off > a->n)
            return DF11_ERR_INVALID_ARG;
        prm.mats[m].end = (uint32_t)off;
        prm.mats[m].cols = M.cols;
        prm.mats[m].rowbase = (uint32_t)rows;
        rows += M.rows;
        if (rows >= (1ull << 30))
            return DF11_ERR_INVALID_ARG;
        prm.mats[m].x = M.x;
        prm.mats[m].y = M.y;
    }
    if (off != a->n)
        return DF11_ERR_INVALID_ARG;  // the matrices must cover the stream exactly
    prm.num_mats = num_mats;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    return a->threads_per_block == 32 ? launch<1, 1>(prm, s) : launch<2, 1>(prm, s);
}
