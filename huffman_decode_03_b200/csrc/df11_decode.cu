// df11_decode.cu -- sm_100a kernel that rebuilds BF16 weights from DF11.
//
// "DFloat11: Kompresi inferensi GPU lossless ..." (id.news.hada.io/topic?id=20542):
//   "Decoding berbasis LUT hierarkis"  -- codes are resolved by table lookup
//        instead of a bit-by-bit tree walk; the tree is cut into height-8
//        subtrees stored as 256-entry LUTs whose values 240..255 are pointers;
//   "Kernel GPU 2 tahap dan metadata bantu" -- one thread per 8-byte segment
//        of EncodedExponent, starting at the segment's Gap; stage 1 counts the
//        codes of each segment, a prefix sum over the thread block plus the
//        block's stored output position gives each thread its first output
//        index, stage 2 decodes again and places the exponents in an on-chip
//        write buffer, and the block's outputs leave in one coalesced write;
//   "Format DFloat11" -- sign and mantissa come verbatim from
//        PackedSignMantissa.
//
// B200 design (what differs from the page's kernel):
//   * the format's thread block is one warp (T = 32 segments): a block's
//     prefix sum is five warp shuffles and its write buffer is private to
//     the warp, so warps never wait for one another -- no block-wide barrier
//     after set-up.  One persistent CTA of 32 warps runs per SM and every
//     warp walks its own sequence of blocks;
//   * the CTA stages the page's LUTs and CodeLengths once and derives two
//     wider tables from them in shared memory, shared by its 32 warps:
//       - a count table over the next 12 bits: how many whole codes they
//         hold and how many bits those codes use (stage 1 advances about 10
//         bits per lookup);
//       - a symbol table over the next 12 bits: up to 3 whole codes, their
//         total length and their exponents (stage 2 places ~3 exponents per
//         lookup).  Exponents are stored rotated right by one bit, which
//         turns the final BF16 merge into two bit-selects and two byte
//         permutes per 4 elements.
//     Codes longer than 12 bits fall back to the page's pointer-chasing LUTs;
//   * stage 1 stops exactly at the thread's last code: the next segment's
//     Gap gives the bit where the next thread starts; the final lookup masks
//     the bits past that point to zeros, and the codes the zeros form (the
//     all-zero code is the canonical first code) are subtracted;
//   * stage 2 runs until the thread has placed as many exponents as stage 1
//     counted;
//   * each thread's 64 + 32 bits live in a three-register shift window: the
//     table index is the top 12 bits, a step is three funnel shifts;
//   * the next block's stream words, Gaps words and offsets are loaded into
//     registers while the current block is decoded.
// Every loop is bounded; inconsistent data sets a status word, never traps.
#include "df11.h"

#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

namespace {

constexpr int kIdxBits = 12;  // index width of both derived tables
constexpr int kIdxEntries = 1 << kIdxBits;
constexpr int kLutBytes = DF11_MAX_LUTS * 256;
constexpr uint32_t kPointerBase = 240;
constexpr int kBlockSegs = 32;  // segments per format block = lanes per warp
constexpr int kWarps = 32;      // warps per CTA
constexpr int kThreads = kWarps * 32;

struct Params {
    const uint8_t *stream;
    const uint8_t *sm;
    const uint64_t *gaps;
    const uint32_t *offs;
    const uint8_t *luts;
    const uint8_t *cl;
    uint16_t *dst;
    uint32_t *status;
    uint64_t n;
    uint64_t total_bits;
    uint64_t nseg;
    uint32_t nblocks;
    uint32_t num_luts;
    uint32_t cap;  // bytes of one warp's exponent buffer
};

__host__ __device__ constexpr uint32_t align16(uint32_t x) { return (x + 15u) & ~15u; }

// Shared memory: tables at fixed offsets (lookups need no base register),
// then one exponent buffer per warp.
struct Smem {
    static constexpr uint32_t sym = 0;                       // uint32[4096]
    static constexpr uint32_t cnt = sym + kIdxEntries * 4;   // uint8[4096]
    static constexpr uint32_t luts = cnt + kIdxEntries;      // 17 * 256
    static constexpr uint32_t cl = luts + kLutBytes;         // 256
    static constexpr uint32_t ztab = cl + 256;               // uint16[16]
    static constexpr uint32_t bufs = ztab + 32;
    static constexpr uint32_t bytes(uint32_t cap) { return bufs + kWarps * cap; }
};
static_assert(Smem::bufs % 16 == 0, "buffers must be 16-byte aligned");

__device__ __forceinline__ uint32_t bswap32(uint32_t x) { return __byte_perm(x, 0, 0x0123); }

__device__ __forceinline__ uint32_t ror8(uint32_t s) { return ((s >> 1) | (s << 7)) & 0xFFu; }

// The page's hierarchical lookup: LUT 0 on the first 8 bits of the window,
// pointer value 256 - j continues in LUT j on the next 8 bits.  Returns
// symbol | length << 8; *bad on a dangling pointer.
__device__ __forceinline__ uint32_t lut_decode(uint32_t win, const uint8_t *luts, const uint8_t *cl,
                                               uint32_t num_luts, bool *bad)
{
    uint32_t e = luts[win >> 24];
#pragma unroll
    for (int lvl = 1; lvl <= 3; lvl++) {
        if (e < kPointerBase)
            break;
        uint32_t j = 256u - e;
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

// Registers one lane holds for one block: its stream words (raw), the Gaps
// word pair holding its field and the next one, and the block's offsets.
struct BlockRegs {
    uint2 s01;
    uint32_t s2;
    uint64_t g0, g1;
    uint32_t o0, o1;
};

__device__ __forceinline__ void load_block(const Params &p, uint32_t b, int lane, BlockRegs &r)
{
    const uint8_t *s = p.stream + (uint64_t)b * (kBlockSegs * 8) + 8 * lane;
    r.s01 = __ldg(reinterpret_cast<const uint2 *>(s));
    r.s2 = __ldg(reinterpret_cast<const uint32_t *>(s + 8));
    const uint64_t bit = 5ull * ((uint64_t)b * kBlockSegs + lane);
    const uint64_t w = bit >> 6;
    r.g0 = __ldg(p.gaps + w);
    r.g1 = __ldg(p.gaps + w + 1);
    r.o0 = __ldg(p.offs + b);
    r.o1 = __ldg(p.offs + b + 1);
}

__global__ void __launch_bounds__(kThreads, 1) df11_decode_kernel(const Params p)
{
    extern __shared__ __align__(128) uint8_t smem[];
    uint32_t *sym_tab = reinterpret_cast<uint32_t *>(smem + Smem::sym);
    uint8_t *cnt_tab = smem + Smem::cnt;
    uint8_t *luts = smem + Smem::luts;
    uint8_t *cl = smem + Smem::cl;
    uint16_t *ztab = reinterpret_cast<uint16_t *>(smem + Smem::ztab);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    uint8_t *exp_s = smem + Smem::bufs + warp * p.cap;

    // ---- once per CTA: the page's LUTs and CodeLengths, derived tables
    const uint32_t lut_bytes = p.num_luts * 256u;
    for (uint32_t i = tid; i < lut_bytes; i += kThreads)
        luts[i] = p.luts[i];
    for (uint32_t i = tid; i < 256; i += kThreads)
        cl[i] = p.cl[i];
    __syncthreads();
    for (uint32_t i = tid; i < kIdxEntries; i += kThreads) {
        const uint32_t w = i << (32 - kIdxBits);
        uint32_t pos = 0, ncodes = 0, syms = 0, sym_bits = 0, sym_n = 0;
        for (int it = 0; it < kIdxBits; it++) {
            bool bad = false;
            const uint32_t e = lut_decode(w << pos, luts, cl, p.num_luts, &bad);
            const uint32_t len = e >> 8;
            if (bad || len < 1 || pos + len > kIdxBits)
                break;
            if (ncodes < 3) {
                syms |= ror8(e & 0xFFu) << (8 * ncodes);
                sym_bits = pos + len;
                sym_n = ncodes + 1;
            }
            ncodes++;
            pos += len;
        }
        cnt_tab[i] = (uint8_t)(ncodes | (pos << 4));
        // exponents in bytes 0..2, count in bits 24..25, total length in 28..31
        sym_tab[i] = syms | (sym_n << 24) | (sym_bits << 28);
    }
    if (tid <= kIdxBits) {
        // codes formed by the zero bits r..11 after a code boundary: the
        // all-zero code (the canonical first code) repeated; count | bits << 8
        bool bad = false;
        const uint32_t lmin = lut_decode(0u, luts, cl, p.num_luts, &bad) >> 8;
        const uint32_t z = (lmin >= 1 && !bad) ? (kIdxBits - tid) / lmin : 0u;
        ztab[tid] = (uint16_t)(z | ((z * lmin) << 8));
    }
    __syncthreads();

    // ---- each warp walks its own blocks; no block-wide barrier from here on
    const uint32_t stride = gridDim.x * kWarps;
    uint32_t b = blockIdx.x * kWarps + warp;
    BlockRegs cur, nxt;
    if (b < p.nblocks)
        load_block(p, b, lane, cur);
    for (; b < p.nblocks; b += stride) {
        if (b + stride < p.nblocks)
            load_block(p, b + stride, lane, nxt);
        const uint32_t o0 = cur.o0, o1 = cur.o1;
        const uint32_t lo_off = o0 & 15u;

        // ---- locate: this lane's codes start in [pos0, pend) of its window
        const uint64_t seg = (uint64_t)b * kBlockSegs + lane;
        int pos0 = 0, pend = 0;
        {
            const uint32_t off = (uint32_t)((5ull * seg) & 63);
            uint64_t v = cur.g0 >> off;
            if (off > 54)  // this field and the next reach into the second word
                v |= cur.g1 << (64 - off);
            const uint32_t gap = (uint32_t)v & 31u, gap_next = (uint32_t)(v >> 5) & 31u;
            if (seg < p.nseg) {
                pos0 = (int)gap;
                pend = seg + 1 < p.nseg ? 64 + (int)gap_next : (int)(p.total_bits - 64 * seg);
            }
        }
        const uint32_t w0 = bswap32(cur.s01.x), w1 = bswap32(cur.s01.y), w2 = bswap32(cur.s2);

        // ---- stage 1: count the codes starting in [pos0, pend)
        bool bad = false;
        uint32_t cnt = 0;
        {
            uint32_t h = w0, m = w1, l = w2;
            shift_window(h, m, l, (uint32_t)pos0);
            int pos = pos0;
            const int bulk_end = pend - kIdxBits;
            while (pos < bulk_end) {  // pos strictly increases: at most 95 steps
                uint32_t e = cnt_tab[h >> (32 - kIdxBits)];
                uint32_t c = e >> 4;
                if (c == 0) {  // a code longer than 12 bits
                    c = lut_decode(h, luts, cl, p.num_luts, &bad) >> 8;
                    c = c ? c : 1u;
                    e = 1;
                }
                cnt += e & 15u;
                pos += (int)c;
                shift_window(h, m, l, c);
            }
            const int r = pend - pos;
            if (r > 0) {
                // the last r <= 12 bits hold whole codes; mask the rest to zeros
                const uint32_t idx = (h >> (32 - kIdxBits)) & ((0xFFFu << (kIdxBits - r)) & 0xFFFu);
                const uint32_t e = cnt_tab[idx];
                const uint32_t z = ztab[r];
                cnt += (e & 15u) - (z & 0xFFu);
                bad |= (e >> 4) - (z >> 8) != (uint32_t)r;
            } else if (r < 0) {
                bad = true;
            }
        }

        // ---- warp prefix sum of the counts
        uint32_t incl = cnt;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const uint32_t y = __shfl_up_sync(0xffffffffu, incl, d);
            if (lane >= d)
                incl += y;
        }
        const uint32_t total = __shfl_sync(0xffffffffu, incl, 31);
        const uint32_t first = incl - cnt;
        const bool block_bad = __any_sync(0xffffffffu, bad) || o1 < o0 || (uint64_t)o1 > p.n ||
                               total != o1 - o0 || lo_off + total + 16u > p.cap;
        if (block_bad) {
            if (lane == 0)
                atomicOr(p.status, (uint32_t)DF11_ERR_CORRUPT);
        } else {
            // ---- stage 2: decode again, place rotated exponents
            {
                uint32_t h = w0, m = w1, l = w2;
                shift_window(h, m, l, (uint32_t)pos0);
                uint32_t q = lo_off + first;
                const uint32_t qend = q + cnt;
                while (q < qend) {  // q strictly increases
                    uint32_t e = sym_tab[h >> (32 - kIdxBits)];
                    uint32_t c = e >> 28, nsym = (e >> 24) & 3u;
                    if (nsym == 0) {  // a code longer than 12 bits
                        const uint32_t d = lut_decode(h, luts, cl, p.num_luts, &bad);
                        e = ror8(d & 0xFFu);
                        c = d >> 8;
                        nsym = 1;
                    }
                    exp_s[q] = (uint8_t)e;
                    if (q + 1 < qend)
                        exp_s[q + 1] = (uint8_t)(e >> 8);
                    if (q + 2 < qend)
                        exp_s[q + 2] = (uint8_t)(e >> 16);
                    q += nsym;
                    shift_window(h, m, l, c);
                }
            }
            __syncwarp();

            // ---- merge with sign/mantissa, coalesced 16-byte stores
            const uint32_t hi = lo_off + total;
            const uint64_t g0 = (uint64_t)o0 - lo_off;  // multiple of 16
            const uint32_t nchunks = (hi + 15) / 16;
            for (uint32_t c = lane; c < nchunks; c += 32) {
                const uint32_t l0 = 16 * c;
                if (l0 >= lo_off && l0 + 16 <= hi) {
                    const uint4 s = __ldg(reinterpret_cast<const uint4 *>(p.sm + g0 + l0));
                    const uint4 e = *reinterpret_cast<const uint4 *>(exp_s + l0);
                    uint4 r0, r1;
                    merge4(s.x, e.x, r0.x, r0.y);
                    merge4(s.y, e.y, r0.z, r0.w);
                    merge4(s.z, e.z, r1.x, r1.y);
                    merge4(s.w, e.w, r1.z, r1.w);
                    uint4 *d = reinterpret_cast<uint4 *>(p.dst + g0 + l0);
                    d[0] = r0;
                    d[1] = r1;
                }
            }
            // partial first / last chunk: one element per lane
            {
                const uint32_t chunk = lane < 16 ? 0u : nchunks - 1;
                const uint32_t l = 16 * chunk + (lane & 15);
                const bool partial = lo_off > 16 * chunk || 16 * chunk + 16 > hi;
                if ((lane < 16 || nchunks > 1) && partial && l >= lo_off && l < hi)
                    p.dst[g0 + l] = merge1(__ldg(p.sm + g0 + l), exp_s[l]);
            }
            __syncwarp();
        }
        cur = nxt;
    }
}

// ------------------------------------------------------------- host side
std::mutex g_mu;
int g_sms[64];

df11_status device_sms(int *sms)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        return DF11_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_sms[dev]) {
        int v = 0;
        if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return DF11_ERR_CUDA;
        g_sms[dev] = v;
    }
    *sms = g_sms[dev];
    return DF11_OK;
}

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

}  // namespace

extern "C" df11_status df11_decompress(const df11_arrays *a, uint16_t *dst, uint32_t *status_dev, void *stream)
{
    if (!a || !status_dev)
        return DF11_ERR_INVALID_ARG;
    if (a->n == 0)
        return DF11_OK;
    if (a->threads_per_block != kBlockSegs)
        return DF11_ERR_INVALID_ARG;
    if (!dst || !a->encoded_exponent || !a->packed_sign_mantissa || !a->gaps || !a->block_offset || !a->luts ||
        !a->code_lengths)
        return DF11_ERR_INVALID_ARG;
    if (!aligned(dst, 16) || !aligned(a->encoded_exponent, 16) || !aligned(a->packed_sign_mantissa, 16) ||
        !aligned(a->gaps, 8) || !aligned(a->block_offset, 4))
        return DF11_ERR_INVALID_ARG;
    if (a->num_luts < 1 || a->num_luts > DF11_MAX_LUTS || a->n >= (1ull << 32))
        return DF11_ERR_INVALID_ARG;
    const uint64_t nseg = (a->total_bits + 63) / 64;
    if (nseg != a->num_segments || (nseg + kBlockSegs - 1) / kBlockSegs != a->num_blocks || a->num_blocks == 0)
        return DF11_ERR_INVALID_ARG;
    // every load stays inside its array
    if (a->encoded_exponent_bytes < (uint64_t)a->num_blocks * kBlockSegs * 8 + 16 ||
        a->packed_sign_mantissa_bytes < ((a->n + 15) / 16) * 16 ||
        a->gaps_words < (5ull * a->num_blocks * kBlockSegs + 63) / 64 + 2 ||
        a->max_block_elems > 64u * kBlockSegs)
        return DF11_ERR_INVALID_ARG;

    Params prm;
    prm.stream = a->encoded_exponent;
    prm.sm = a->packed_sign_mantissa;
    prm.gaps = a->gaps;
    prm.offs = a->block_offset;
    prm.luts = a->luts;
    prm.cl = a->code_lengths;
    prm.dst = dst;
    prm.status = status_dev;
    prm.n = a->n;
    prm.total_bits = a->total_bits;
    prm.nseg = nseg;
    prm.nblocks = a->num_blocks;
    prm.num_luts = a->num_luts;
    prm.cap = align16(a->max_block_elems + 32);

    const uint32_t smem = Smem::bytes(prm.cap);
    if (cudaFuncSetAttribute(df11_decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess)
        return DF11_ERR_CUDA;
    int sms = 0;
    df11_status st = device_sms(&sms);
    if (st != DF11_OK)
        return st;
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, df11_decode_kernel, kThreads, smem) != cudaSuccess ||
        per_sm < 1)
        return DF11_ERR_CUDA;
    uint64_t grid = (uint64_t)sms * (uint64_t)per_sm;
    const uint64_t need = (a->num_blocks + kWarps - 1) / kWarps;
    if (grid > need)
        grid = need;
    df11_decode_kernel<<<(unsigned)grid, kThreads, smem, reinterpret_cast<cudaStream_t>(stream)>>>(prm);
    return cudaGetLastError() == cudaSuccess ? DF11_OK : DF11_ERR_CUDA;
}

extern "C" df11_status df11_decompress_host(const df11_arrays *h, const df11_arrays *d, uint16_t *dst_dev,
                                            uint16_t *dst_host, uint32_t *status_dev, void *stream)
{
    if (!h || !d || !dst_dev || !dst_host)
        return DF11_ERR_INVALID_ARG;
    if (d->encoded_exponent_bytes < h->encoded_exponent_bytes ||
        d->packed_sign_mantissa_bytes < h->packed_sign_mantissa_bytes || d->gaps_words < h->gaps_words)
        return DF11_ERR_INVALID_ARG;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const cudaMemcpyKind k = cudaMemcpyHostToDevice;
    struct Copy {
        const void *src;
        const void *dst;
        size_t bytes;
    } copies[] = {
        {h->encoded_exponent, d->encoded_exponent, h->encoded_exponent_bytes},
        {h->packed_sign_mantissa, d->packed_sign_mantissa, h->packed_sign_mantissa_bytes},
        {h->gaps, d->gaps, h->gaps_words * 8},
        {h->block_offset, d->block_offset, (h->num_blocks + 1) * 4ull},
        {h->luts, d->luts, h->num_luts * 256ull},
        {h->code_lengths, d->code_lengths, 256},
    };
    for (const Copy &c : copies) {
        if (!c.src || !c.dst)
            return DF11_ERR_INVALID_ARG;
        if (cudaMemcpyAsync(const_cast<void *>(c.dst), c.src, c.bytes, k, s) != cudaSuccess)
            return DF11_ERR_CUDA;
    }
    df11_arrays dev = *h;  // same sizes, device pointers
    dev.encoded_exponent = d->encoded_exponent;
    dev.packed_sign_mantissa = d->packed_sign_mantissa;
    dev.gaps = d->gaps;
    dev.block_offset = d->block_offset;
    dev.luts = d->luts;
    dev.code_lengths = d->code_lengths;
    df11_status st = df11_decompress(&dev, dst_dev, status_dev, stream);
    if (st != DF11_OK)
        return st;
    if (h->n && cudaMemcpyAsync(dst_host, dst_dev, h->n * 2, cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return DF11_ERR_CUDA;
    return DF11_OK;
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
