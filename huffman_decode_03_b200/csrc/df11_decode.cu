// df11_decode.cu -- sm_100a kernel that rebuilds BF16 weights from DF11.
//
// "DFloat11: Kompresi inferensi GPU lossless ..." (id.news.hada.io/topic?id=20542):
//   "Decoding berbasis LUT hierarkis"  -- codes are resolved by table lookup
//        instead of a bit-by-bit tree walk; the tree is cut into height-8
//        subtrees stored as 256-entry LUTs whose values 240..255 are pointers;
//   "Kernel GPU 2 tahap dan metadata bantu" -- one thread per 8-byte segment
//        of EncodedExponent, starting at the segment's Gap; per-thread counts
//        are prefix-summed inside the block and added to the block's stored
//        output position; exponents are placed in an on-chip buffer and the
//        block's outputs leave in one coalesced write;
//   "Format DFloat11" -- sign and mantissa come verbatim from
//        PackedSignMantissa.
//
// B200 design (what differs from the page's kernel):
//   * persistent CTAs (a multiple of the SM count) walk the blocks, so the
//     per-CTA set-up -- LUTs and CodeLengths into shared memory plus a
//     2^K-entry first-level table derived from them -- is paid once per CTA,
//     not once per block;
//   * the derived table resolves every code of length <= K with ONE shared
//     memory lookup (symbol and length in 16 bits); longer codes fall back to
//     the page's pointer-chasing LUTs (at most 4 levels for 32-bit codes);
//   * the thread's 64 + 31 bits live in three registers; the 32-bit window
//     is one funnel shift;
//   * the block prefix sum is a warp-shuffle scan plus a scan of warp totals
//     (the page uses Blelloch's tree scan);
//   * the merge reads 16 sign/mantissa bytes and 16 exponent bytes per
//     thread and writes 32 bytes of BF16 with two 16-byte stores.
// Every loop is bounded; inconsistent data sets a status word, never traps.
#include "df11.h"

#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

namespace {

constexpr int kFastBits = 12;                // K: first-level table index bits
constexpr int kFastEntries = 1 << kFastBits;
constexpr int kLutBytes = DF11_MAX_LUTS * 256;
constexpr uint32_t kPointerBase = 240;

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
    uint32_t exp_cap;  // bytes of the shared exponent buffer
};

__host__ __device__ constexpr uint32_t align16(uint32_t x) { return (x + 15u) & ~15u; }

// Shared-memory layout, in bytes, for T threads and an exponent buffer of
// exp_cap bytes.
struct SmemLayout {
    uint32_t fast, luts, cl, warp, stream, exps, total;
    __host__ __device__ SmemLayout(uint32_t T, uint32_t exp_cap)
    {
        fast = 0;
        luts = fast + kFastEntries * 2;
        cl = luts + kLutBytes;
        warp = cl + 256;
        stream = warp + 32 * 4;
        exps = stream + align16(T * 8 + 16);
        total = exps + exp_cap;
    }
};

__device__ __forceinline__ uint32_t load_be32(const uint8_t *p)
{
    return __byte_perm(*reinterpret_cast<const uint32_t *>(p), 0, 0x0123);
}

// 5-bit Gap of segment s (fields packed LSB-first in uint64 words).
__device__ __forceinline__ uint32_t read_gap(const uint64_t *gaps, uint64_t s)
{
    uint64_t bit = 5 * s;
    uint64_t w = bit >> 6;
    uint32_t off = (uint32_t)(bit & 63);
    uint64_t v = __ldg(gaps + w) >> off;
    if (off > 59)
        v |= __ldg(gaps + w + 1) << (64 - off);
    return (uint32_t)v & 31u;
}

// The page's hierarchical lookup: LUT 0 on the first 8 bits of the window,
// pointer value 256 - j continues in LUT j on the next 8 bits.  Returns
// symbol | length << 8; sets *bad on a dangling pointer.
__device__ __forceinline__ uint32_t lut_decode(uint32_t win, const uint8_t *luts,
                                               const uint8_t *cl, uint32_t num_luts, bool *bad)
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

// One code at bit position pos (0..63) of the thread's 96-bit window
// (w0 w1 w2, big-endian words).  Returns symbol | length << 8.
__device__ __forceinline__ uint32_t decode_one(uint32_t w0, uint32_t w1, uint32_t w2, int pos,
                                               const uint16_t *fast, const uint8_t *luts,
                                               const uint8_t *cl, uint32_t num_luts, bool *bad)
{
    uint32_t hi = pos < 32 ? w0 : w1;
    uint32_t lo = pos < 32 ? w1 : w2;
    uint32_t win = __funnelshift_l(lo, hi, (uint32_t)pos);
    uint32_t e = fast[win >> (32 - kFastBits)];
    if (e >> 8)
        return e;
    return lut_decode(win, luts, cl, num_luts, bad);
}

// Exclusive prefix sum over the block; *total receives the block sum.
template <int T>
__device__ __forceinline__ uint32_t block_exclusive_scan(uint32_t v, uint32_t *warp_sums,
                                                         uint32_t *total)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t x = v;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        uint32_t y = __shfl_up_sync(0xffffffffu, x, d);
        if (lane >= d)
            x += y;
    }
    if (lane == 31)
        warp_sums[warp] = x;
    __syncthreads();
    if (warp == 0) {
        uint32_t s = lane < T / 32 ? warp_sums[lane] : 0;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            uint32_t y = __shfl_up_sync(0xffffffffu, s, d);
            if (lane >= d)
                s += y;
        }
        if (lane < T / 32)
            warp_sums[lane] = s;  // inclusive warp prefix
    }
    __syncthreads();
    uint32_t before = warp ? warp_sums[warp - 1] : 0;
    *total = warp_sums[T / 32 - 1];
    return before + x - v;
}

// BF16 from exponent and sign/mantissa bytes, two elements per 32-bit word:
// lanes hold s (sign<<7 | mantissa) and e; (e << 7) + s puts the sign bit on
// top of the exponent's lowest bit, adding 255 * (s & 0x80) moves it to bit 15.
__device__ __forceinline__ uint32_t merge2(uint32_t s_lanes, uint32_t e_lanes)
{
    return (e_lanes << 7) + s_lanes + (s_lanes & 0x00800080u) * 255u;
}

__device__ __forceinline__ void merge16(const uint4 &s, const uint4 &e, uint4 &out_lo, uint4 &out_hi)
{
    out_lo.x = merge2(__byte_perm(s.x, 0, 0x4140), __byte_perm(e.x, 0, 0x4140));
    out_lo.y = merge2(__byte_perm(s.x, 0, 0x4342), __byte_perm(e.x, 0, 0x4342));
    out_lo.z = merge2(__byte_perm(s.y, 0, 0x4140), __byte_perm(e.y, 0, 0x4140));
    out_lo.w = merge2(__byte_perm(s.y, 0, 0x4342), __byte_perm(e.y, 0, 0x4342));
    out_hi.x = merge2(__byte_perm(s.z, 0, 0x4140), __byte_perm(e.z, 0, 0x4140));
    out_hi.y = merge2(__byte_perm(s.z, 0, 0x4342), __byte_perm(e.z, 0, 0x4342));
    out_hi.z = merge2(__byte_perm(s.w, 0, 0x4140), __byte_perm(e.w, 0, 0x4140));
    out_hi.w = merge2(__byte_perm(s.w, 0, 0x4342), __byte_perm(e.w, 0, 0x4342));
}

__device__ __forceinline__ uint16_t merge1(uint32_t s, uint32_t e)
{
    return (uint16_t)(((s & 0x80u) << 8) | (e << 7) | (s & 0x7Fu));
}

template <int T>
__global__ void __launch_bounds__(T) df11_decode_kernel(const Params p)
{
    extern __shared__ __align__(16) uint8_t smem[];
    const SmemLayout L(T, p.exp_cap);
    uint16_t *fast = reinterpret_cast<uint16_t *>(smem + L.fast);
    uint8_t *luts = smem + L.luts;
    uint8_t *cl = smem + L.cl;
    uint32_t *warp_sums = reinterpret_cast<uint32_t *>(smem + L.warp);
    uint8_t *stream_s = smem + L.stream;
    uint8_t *exp_s = smem + L.exps;
    const int tid = threadIdx.x;

    // ---- once per CTA: page LUTs + CodeLengths, then the derived table
    const uint32_t lut_bytes = p.num_luts * 256u;
    for (uint32_t i = tid; i < lut_bytes; i += T)
        luts[i] = p.luts[i];
    for (uint32_t i = tid; i < 256; i += T)
        cl[i] = p.cl[i];
    __syncthreads();
    for (uint32_t i = tid; i < kFastEntries; i += T) {
        bool bad = false;
        uint32_t e = lut_decode(i << (32 - kFastBits), luts, cl, p.num_luts, &bad);
        uint32_t len = e >> 8;
        fast[i] = (!bad && len >= 1 && len <= kFastBits) ? (uint16_t)e : (uint16_t)0;
    }
    __syncthreads();

    for (uint32_t b = blockIdx.x; b < p.nblocks; b += gridDim.x) {
        const uint32_t o0 = __ldg(p.offs + b), o1 = __ldg(p.offs + b + 1);
        const uint32_t lo = o0 & 15u;
        const bool offs_ok = o1 >= o0 && (uint64_t)o1 <= p.n && lo + (o1 - o0) + 16u <= p.exp_cap;

        // ---- stage this block's 8*T bytes (+16 bytes of look-ahead)
        {
            const uint4 *src = reinterpret_cast<const uint4 *>(p.stream + (uint64_t)b * T * 8);
            uint4 *dstv = reinterpret_cast<uint4 *>(stream_s);
            for (int i = tid; i < (T * 8 + 16) / 16; i += T)
                dstv[i] = __ldg(src + i);
        }
        __syncthreads();

        // ---- locate: this thread decodes codes starting in [pos0, pend)
        const uint64_t seg = (uint64_t)b * T + tid;
        int pos0 = 0, pend = 0;
        if (seg < p.nseg) {
            pos0 = (int)read_gap(p.gaps, seg);
            uint64_t endbit = seg + 1 < p.nseg ? 64 * (seg + 1) + read_gap(p.gaps, seg + 1) : p.total_bits;
            pend = (int)(endbit - 64 * seg);
        }
        const uint32_t w0 = load_be32(stream_s + 8 * tid);
        const uint32_t w1 = load_be32(stream_s + 8 * tid + 4);
        const uint32_t w2 = load_be32(stream_s + 8 * tid + 8);

        // ---- pass 1: count
        bool bad = false;
        int pos = pos0;
        uint32_t cnt = 0;
        for (int it = 0; it < 64 && pos < pend; it++) {
            uint32_t e = decode_one(w0, w1, w2, pos, fast, luts, cl, p.num_luts, &bad);
            pos += (int)(e >> 8);
            cnt++;
        }
        bad |= pos != pend;

        uint32_t total;
        const uint32_t first = block_exclusive_scan<T>(cnt, warp_sums, &total);
        const bool block_bad = __syncthreads_or(bad) || !offs_ok || total != o1 - o0;
        if (block_bad) {
            if (tid == 0)
                atomicOr(p.status, (uint32_t)DF11_ERR_CORRUPT);
            __syncthreads();
            continue;
        }

        // ---- pass 2: decode again, place exponents in shared memory
        {
            uint8_t *out = exp_s + lo + first;
            int q = pos0;
            for (uint32_t j = 0; j < cnt; j++) {
                uint32_t e = decode_one(w0, w1, w2, q, fast, luts, cl, p.num_luts, &bad);
                out[j] = (uint8_t)e;
                q += (int)(e >> 8);
            }
        }
        __syncthreads();

        // ---- merge with sign/mantissa, coalesced 16-byte stores
        {
            const uint32_t hi = lo + (o1 - o0);
            const uint64_t g0 = (uint64_t)o0 - lo;  // multiple of 16
            const uint32_t nchunks = (hi + 15) / 16;
            for (uint32_t c = tid; c < nchunks; c += T) {
                const uint32_t l0 = 16 * c;
                const uint64_t g = g0 + l0;
                if (l0 >= lo && l0 + 16 <= hi) {
                    uint4 s = __ldg(reinterpret_cast<const uint4 *>(p.sm + g));
                    uint4 e = *reinterpret_cast<const uint4 *>(exp_s + l0);
                    uint4 r0, r1;
                    merge16(s, e, r0, r1);
                    uint4 *d = reinterpret_cast<uint4 *>(p.dst + g);
                    d[0] = r0;
                    d[1] = r1;
                } else {
                    for (uint32_t i = 0; i < 16; i++) {
                        uint32_t l = l0 + i;
                        if (l >= lo && l < hi)
                            p.dst[g + i] = merge1(p.sm[g + i], exp_s[l]);
                    }
                }
            }
        }
        __syncthreads();
    }
}

// ------------------------------------------------------------- host side
struct DeviceInfo {
    int sms = 0;
};

std::mutex g_mu;
DeviceInfo g_dev[64];

df11_status device_sms(int *sms)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        return DF11_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_dev[dev].sms) {
        int v = 0;
        if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return DF11_ERR_CUDA;
        g_dev[dev].sms = v;
    }
    *sms = g_dev[dev].sms;
    return DF11_OK;
}

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

template <int T>
df11_status launch(const Params &prm, cudaStream_t stream)
{
    const SmemLayout L(T, prm.exp_cap);
    auto kern = df11_decode_kernel<T>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L.total) != cudaSuccess)
        return DF11_ERR_CUDA;
    int sms = 0;
    df11_status st = device_sms(&sms);
    if (st != DF11_OK)
        return st;
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, T, L.total) != cudaSuccess || per_sm < 1)
        return DF11_ERR_CUDA;
    uint64_t grid = (uint64_t)sms * (uint64_t)per_sm;
    if (grid > prm.nblocks)
        grid = prm.nblocks;
    kern<<<(unsigned)grid, T, L.total, stream>>>(prm);
    return cudaGetLastError() == cudaSuccess ? DF11_OK : DF11_ERR_CUDA;
}

}  // namespace

extern "C" df11_status df11_decompress(const df11_arrays *a, uint16_t *dst, uint32_t *status_dev,
                                       void *stream)
{
    if (!a || !status_dev)
        return DF11_ERR_INVALID_ARG;
    if (a->n == 0)
        return DF11_OK;
    const uint32_t T = a->threads_per_block;
    if (!dst || !a->encoded_exponent || !a->packed_sign_mantissa || !a->gaps || !a->block_offset ||
        !a->luts || !a->code_lengths)
        return DF11_ERR_INVALID_ARG;
    if (!aligned(dst, 16) || !aligned(a->encoded_exponent, 16) || !aligned(a->packed_sign_mantissa, 16) ||
        !aligned(a->gaps, 8) || !aligned(a->block_offset, 4))
        return DF11_ERR_INVALID_ARG;
    if (a->num_luts < 1 || a->num_luts > DF11_MAX_LUTS || a->n >= (1ull << 32))
        return DF11_ERR_INVALID_ARG;
    const uint64_t nseg = (a->total_bits + 63) / 64;
    if (nseg != a->num_segments || (nseg + T - 1) / T != a->num_blocks)
        return DF11_ERR_INVALID_ARG;
    if (a->encoded_exponent_bytes < (uint64_t)a->num_blocks * T * 8 + 16 ||
        a->packed_sign_mantissa_bytes < ((a->n + 15) / 16) * 16 ||
        a->gaps_words < (5ull * a->num_blocks * T + 63) / 64 + 1 ||
        a->max_block_elems > 64u * T)
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
    prm.exp_cap = align16(a->max_block_elems + 32);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    switch (T) {
    case 128: return launch<128>(prm, s);
    case 256: return launch<256>(prm, s);
    case 512: return launch<512>(prm, s);
    default: return DF11_ERR_INVALID_ARG;
    }
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
