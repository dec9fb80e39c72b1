// df11_encode.cu -- DF11 compression of BF16 weights already in device memory.
//
// "DFloat11: Kompresi inferensi GPU lossless ..." (id.news.hada.io/topic?id=20542)
// compresses offline: "Format DFloat11" splits each BF16 weight into its
// exponent and its sign+mantissa byte, Huffman-codes the exponents and
// bit-packs the codes into EncodedExponent; "Kernel GPU 2 tahap dan metadata
// bantu" adds one 5-bit Gap per 8-byte segment and one output position per
// thread block.  This file runs those steps on the GPU for weights that are
// already resident there, producing exactly the arrays df11_build_format
// builds on the host (same code, same bytes):
//   1. df11_device_histogram: exponent histogram (per-warp shared-memory
//      counters, then one 64-bit atomic add per bin and CTA);
//   2. the host turns the 256 counts into the code (df11_plan_from_histogram:
//      Huffman or package-merge lengths, canonical codes, LUTs) -- microseconds
//      of work on 256 numbers;
//   3. df11_device_encode: the code length of every element summed per
//      8192-element chunk, one exclusive scan over the chunks, then one CTA per
//      chunk: a block scan of its threads' bit counts gives every code's start
//      bit; codes are OR-ed into a shared-memory copy of the chunk's bits and
//      its segments' Gap fields, which leave in whole words (the two words at
//      each end, shared with the neighbouring chunks, by atomic OR); the code
//      start that first reaches a segment boundary writes that segment's Gap
//      and, every T segments, the block's BlockOffset; sign/mantissa bytes
//      leave in 16-byte stores.
// Every loop is bounded; an element whose exponent has no code (input changed
// since its histogram) sets the status word and is skipped.
#include "df11.h"

#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>
#include <mutex>

df11_status df11_internal_plan_codes(const df11_format *f, uint32_t *codes256);  // df11_format.cpp

namespace {

constexpr uint32_t kChunk = 8192;                      // elements per CTA
constexpr uint32_t kThreads = 256;                     // threads per CTA
constexpr uint32_t kPerThread = kChunk / kThreads;     // 32 consecutive elements each
constexpr uint32_t kMaxChunkBits = kChunk * 32;        // codes are <= 32 bits
constexpr uint32_t kBitWords = kMaxChunkBits / 32 + 2;  // + partial words at both ends
constexpr uint32_t kMaxSegs = kMaxChunkBits / 64 + 3;
constexpr uint32_t kGapWords = (5 * kMaxSegs) / 32 + 3;  // 32-bit staging words
static_assert(kPerThread == 32, "one warp-sized run of elements per thread");

struct EncParams {
    const uint16_t *w;
    uint8_t *stream;  // EncodedExponent
    uint8_t *sm;      // PackedSignMantissa
    uint64_t *gaps;
    uint32_t *offs;
    uint64_t *chunk_bits;  // scratch: nchunks + 1 words
    uint32_t *status;
    uint32_t *max_block;
    uint64_t n;
    uint64_t total_bits;
    uint64_t nseg;
    uint32_t T;
    uint32_t t32_magic;  // ceil(2^32 / (T / 32)): umulhi(x, magic) = x / (T / 32) exactly for x < 2^26
    uint32_t nblocks;
    uint32_t nchunks;
    uint32_t code[256];  // canonical code, right-aligned
    uint8_t len[256];    // code length, 0 = no code
};

__device__ __forceinline__ uint32_t exponent(uint32_t w) { return (w >> 7) & 0xFFu; }

__device__ __forceinline__ uint32_t sign_mantissa(uint32_t w) { return ((w >> 8) & 0x80u) | (w & 0x7Fu); }

// The 32 elements [i0, i0 + 32) of a thread (fewer at the end of the stream).
__device__ __forceinline__ uint32_t load_run(const uint16_t *w, uint64_t i0, uint64_t n, uint32_t v[16])
{
    const uint64_t cnt64 = i0 < n ? n - i0 : 0;
    const uint32_t cnt = cnt64 < 32 ? (uint32_t)cnt64 : 32u;
    if (cnt == 32) {
        const uint4 *src = reinterpret_cast<const uint4 *>(w + i0);
#pragma unroll
        for (int k = 0; k < 4; k++) {
            const uint4 q = __ldg(src + k);
            v[4 * k] = q.x;
            v[4 * k + 1] = q.y;
            v[4 * k + 2] = q.z;
            v[4 * k + 3] = q.w;
        }
    } else {
#pragma unroll
        for (int k = 0; k < 16; k++) {
            const uint32_t a = 2 * k < (int)cnt ? w[i0 + 2 * k] : 0u;
            const uint32_t b = 2 * k + 1 < (int)cnt ? w[i0 + 2 * k + 1] : 0u;
            v[k] = a | (b << 16);
        }
    }
    return cnt;
}

__device__ __forceinline__ uint32_t element(const uint32_t v[16], uint32_t k)
{
    return (k & 1u) ? (v[k >> 1] >> 16) : (v[k >> 1] & 0xFFFFu);
}

// Exclusive sum over the CTA's threads (kThreads); *total gets the sum.
__device__ __forceinline__ uint32_t block_exclusive_sum(uint32_t x, uint32_t *warp_tot, uint32_t *total)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t incl = x;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, incl, d);
        if (lane >= d)
            incl += y;
    }
    if (lane == 31)
        warp_tot[warp] = incl;
    __syncthreads();
    uint32_t before = 0, all = 0;
#pragma unroll
    for (int k = 0; k < (int)(kThreads / 32); k++) {
        const uint32_t t = warp_tot[k];
        before += k < warp ? t : 0u;
        all += t;
    }
    __syncthreads();
    *total = all;
    return before + incl - x;
}

// ---------------------------------------------------------------- kernels
// Per-warp exponent counters in shared memory, one 64-bit atomic per bin and
// CTA into the histogram.
__global__ void __launch_bounds__(kThreads) histogram_kernel(const uint16_t *w, uint64_t n,
                                                             unsigned long long *hist)
{
    __shared__ uint32_t h[kThreads / 32][256];
    for (uint32_t i = threadIdx.x; i < (kThreads / 32) * 256; i += kThreads)
        (&h[0][0])[i] = 0;
    __syncthreads();
    uint32_t *mine = h[threadIdx.x >> 5];
    const uint64_t groups = n / 8;  // 8 elements per 16-byte load
    const uint4 *src = reinterpret_cast<const uint4 *>(w);
    for (uint64_t g = (uint64_t)blockIdx.x * kThreads + threadIdx.x; g < groups; g += (uint64_t)gridDim.x * kThreads) {
        const uint4 q = __ldg(src + g);
        const uint32_t words[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
        for (int k = 0; k < 4; k++) {
            atomicAdd(&mine[exponent(words[k])], 1u);
            atomicAdd(&mine[exponent(words[k] >> 16)], 1u);
        }
    }
    if (blockIdx.x == 0)
        for (uint64_t i = groups * 8 + threadIdx.x; i < n; i += kThreads)
            atomicAdd(&mine[exponent(w[i])], 1u);
    __syncthreads();
    for (uint32_t b = threadIdx.x; b < 256; b += kThreads) {
        uint32_t s = 0;
#pragma unroll
        for (int k = 0; k < (int)(kThreads / 32); k++)
            s += h[k][b];
        if (s)
            atomicAdd(&hist[b], (unsigned long long)s);
    }
}

// chunk_bits[c] = bits of chunk c's codes.
__global__ void __launch_bounds__(kThreads) chunk_bits_kernel(const EncParams p)
{
    __shared__ uint32_t warp_tot[kThreads / 32];
    __shared__ uint8_t s_len[256];
    for (uint32_t i = threadIdx.x; i < 256; i += kThreads)
        s_len[i] = p.len[i];
    const uint64_t i0 = (uint64_t)blockIdx.x * kChunk + (uint64_t)threadIdx.x * kPerThread;
    uint32_t v[16];
    const uint32_t cnt = load_run(p.w, i0, p.n, v);
    __syncthreads();
    uint32_t bits = 0;
    bool missing = false;
#pragma unroll
    for (uint32_t k = 0; k < 32; k++) {
        if (k < cnt) {
            const uint32_t l = s_len[exponent(element(v, k))];
            bits += l;
            missing |= l == 0;
        }
    }
    if (missing)
        atomicOr(p.status, (uint32_t)DF11_ERR_CORRUPT);
    uint32_t total;
    block_exclusive_sum(bits, warp_tot, &total);
    if (threadIdx.x == 0)
        p.chunk_bits[blockIdx.x] = total;
}

// chunk_bits -> exclusive prefix (chunk c's first bit); chunk_bits[nchunks] =
// total, checked against the plan's total.  One CTA of 1024 threads.
__global__ void __launch_bounds__(1024) chunk_scan_kernel(const EncParams p)
{
    __shared__ unsigned long long part[1024];
    const uint32_t nc = p.nchunks, per = (nc + 1023) / 1024;
    const uint32_t c0 = threadIdx.x * per, c1 = min(nc, c0 + per);
    unsigned long long s = 0;
    for (uint32_t c = c0; c < c1; c++)
        s += p.chunk_bits[c];
    part[threadIdx.x] = s;
    __syncthreads();
    // Hillis-Steele inclusive scan over the 1024 partial sums
    for (uint32_t d = 1; d < 1024; d <<= 1) {
        const unsigned long long y = threadIdx.x >= d ? part[threadIdx.x - d] : 0ull;
        __syncthreads();
        part[threadIdx.x] += y;
        __syncthreads();
    }
    unsigned long long run = part[threadIdx.x] - s;
    for (uint32_t c = c0; c < c1; c++) {
        const unsigned long long b = p.chunk_bits[c];
        p.chunk_bits[c] = run;
        run += b;
    }
    if (threadIdx.x == 1023) {
        p.chunk_bits[nc] = part[1023];
        if (part[1023] != p.total_bits)
            atomicOr(p.status, (uint32_t)DF11_ERR_CORRUPT);
    }
}

// Gap field of segment s (5 bits at bit 5 s of the packed words, LSB first)
// into the chunk's 32-bit staging words, which start at global 32-bit word
// gw0 (the uint64 Gaps words read as little-endian halves).
__device__ __forceinline__ void put_gap(uint32_t *gbuf, uint64_t gw0, uint64_t s, uint32_t g)
{
    const uint64_t bit = 5 * s;
    const uint32_t w = (uint32_t)(bit / 32 - gw0);
    const uint32_t sh = (uint32_t)(bit % 32);
    atomicOr(&gbuf[w], (g & 31u) << sh);
    if (sh > 27)
        atomicOr(&gbuf[w + 1], (g & 31u) >> (32 - sh));
}

// Segment s (< 2^31) starts a format block: s % T == 0, with T a multiple of
// 32; *b gets s / T.
__device__ __forceinline__ bool block_start(const EncParams &p, uint64_t s, uint32_t *b)
{
    const uint32_t s32 = (uint32_t)s;
    if (s32 & 31u)
        return false;
    const uint32_t x = s32 >> 5, t32 = p.T >> 5;
    const uint32_t q = t32 == 1 ? x : __umulhi(x, p.t32_magic);
    *b = q;
    return x - q * t32 == 0;
}

__global__ void __launch_bounds__(kThreads) encode_kernel(const EncParams p)
{
    extern __shared__ __align__(16) uint8_t smem[];
    uint32_t *bits = reinterpret_cast<uint32_t *>(smem);                                  // kBitWords
    uint32_t *gbuf = reinterpret_cast<uint32_t *>(smem + kBitWords * 4);  // kGapWords
    __shared__ uint32_t s_code[256];
    __shared__ uint8_t s_len[256];
    __shared__ uint32_t warp_tot[kThreads / 32];
    for (uint32_t i = threadIdx.x; i < 256; i += kThreads) {
        s_code[i] = p.code[i];
        s_len[i] = p.len[i];
    }
    const uint32_t c = blockIdx.x;
    const uint64_t lo = (uint64_t)c * kChunk;
    const uint64_t hi = p.n - lo < kChunk ? p.n : lo + kChunk;
    const uint64_t B = p.chunk_bits[c], E = p.chunk_bits[c + 1];
    if (E < B || E - B > kMaxChunkBits || E > p.total_bits) {  // inconsistent scratch or input
        if (threadIdx.x == 0)
            atomicOr(p.status, (uint32_t)DF11_ERR_CORRUPT);
        return;
    }
    const uint64_t wb0 = B / 32;
    const uint32_t nbw = (uint32_t)((E + 31) / 32 - wb0);
    // segments whose first code start lies in this chunk: boundaries 64 s in
    // (start of element lo - 1, start of element hi - 1]; the last chunk also
    // takes the segments after the last start
    __syncthreads();  // s_len ready
    const uint64_t prev_start = lo ? B - s_len[exponent(p.w[lo - 1])] : 0;
    const uint64_t s_lo = lo ? prev_start / 64 + 1 : 0;
    const uint64_t last_start = E - s_len[exponent(p.w[hi - 1])];
    const uint64_t s_hi1 = hi == p.n ? p.nseg : last_start / 64 + 1;  // exclusive
    const uint64_t gw0 = 5 * s_lo / 32;
    const uint32_t ngw = s_hi1 > s_lo ? (uint32_t)((5 * (s_hi1 - 1) + 4) / 32 + 1 - gw0) : 0u;
    if (ngw > kGapWords) {
        if (threadIdx.x == 0)
            atomicOr(p.status, (uint32_t)DF11_ERR_CORRUPT);
        return;
    }
    for (uint32_t j = threadIdx.x; j < nbw; j += kThreads)
        bits[j] = 0;
    for (uint32_t j = threadIdx.x; j < ngw; j += kThreads)
        gbuf[j] = 0;

    // this thread's elements, their bit offset in the chunk
    const uint64_t i0 = lo + (uint64_t)threadIdx.x * kPerThread;
    uint32_t v[16];
    const uint32_t cnt = load_run(p.w, i0, p.n, v);
    uint32_t tbits = 0;
#pragma unroll
    for (uint32_t k = 0; k < 32; k++)
        if (k < cnt)
            tbits += s_len[exponent(element(v, k))];
    uint32_t chunk_total;
    const uint32_t toff = block_exclusive_sum(tbits, warp_tot, &chunk_total);  // also orders the zeroing

    uint64_t pos = B + toff;
    uint64_t prev = i0 ? pos - s_len[exponent(p.w[i0 - 1])] : 0;
    bool have_prev = i0 != 0;
    // four passes over 8 elements each (reloaded from L1): a loop body of 8
    // elements, not 32, keeps the code within the instruction cache
    for (uint32_t grp = 0; grp < 4; grp++) {
        if (8 * grp >= cnt)
            break;
        uint32_t g4[4];
        if (8 * grp + 8 <= cnt) {
            const uint4 q4 = __ldg(reinterpret_cast<const uint4 *>(p.w + i0) + grp);
            g4[0] = q4.x;
            g4[1] = q4.y;
            g4[2] = q4.z;
            g4[3] = q4.w;
        } else {
#pragma unroll
            for (uint32_t j = 0; j < 4; j++) {
                const uint32_t k0 = 8 * grp + 2 * j;
                const uint32_t a = k0 < cnt ? (uint32_t)p.w[i0 + k0] : 0u;
                const uint32_t b = k0 + 1 < cnt ? (uint32_t)p.w[i0 + k0 + 1] : 0u;
                g4[j] = a | (b << 16);
            }
        }
#pragma unroll
        for (uint32_t j = 0; j < 8; j++) {
            const uint32_t k = 8 * grp + j;
            if (k >= cnt)
                break;
            const uint32_t e = exponent((j & 1u) ? (g4[j >> 1] >> 16) : (g4[j >> 1] & 0xFFFFu));
            const uint32_t l = s_len[e];
            if (l == 0)
                continue;  // reported by chunk_bits_kernel
            // a code of <= 32 bits after the previous start: at most one segment
            // boundary lies in (prev, pos], and then this code is the first to
            // start in segment pos / 64, at Gap pos % 64
            const uint64_t seg = pos >> 6;
            if (!have_prev || (prev >> 6) != seg) {
                put_gap(gbuf, gw0, seg, (uint32_t)(pos & 63));
                uint32_t blk;
                if (block_start(p, seg, &blk))
                    p.offs[blk] = (uint32_t)(i0 + k);
            }
            // the code, MSB first, into the chunk's big-endian bit words
            const uint64_t q = pos - 32 * wb0;
            const uint32_t o = (uint32_t)(q & 31);
            const unsigned long long val = (unsigned long long)s_code[e] << (64 - o - l);
            atomicOr(&bits[q >> 5], (uint32_t)(val >> 32));
            if ((uint32_t)val)
                atomicOr(&bits[(q >> 5) + 1], (uint32_t)val);
            prev = pos;
            have_prev = true;
            pos += l;
        }
    }
    if (cnt && i0 + cnt == p.n) {
        // the stream's last code: the segments after it end at total_bits
        for (uint64_t s = prev / 64 + 1; s < p.nseg; s++) {  // at most one
            put_gap(gbuf, gw0, s, (uint32_t)(p.total_bits - 64 * s));
            uint32_t blk;
            if (block_start(p, s, &blk))
                p.offs[blk] = (uint32_t)p.n;
        }
        p.offs[p.nblocks] = (uint32_t)p.n;
    }
    // sign/mantissa bytes
    if (cnt == 32) {
        uint32_t b[8];
#pragma unroll
        for (int j = 0; j < 8; j++)
            b[j] = sign_mantissa(element(v, 4 * j)) | (sign_mantissa(element(v, 4 * j + 1)) << 8) |
                   (sign_mantissa(element(v, 4 * j + 2)) << 16) | (sign_mantissa(element(v, 4 * j + 3)) << 24);
        uint4 *dst = reinterpret_cast<uint4 *>(p.sm + i0);
        dst[0] = make_uint4(b[0], b[1], b[2], b[3]);
        dst[1] = make_uint4(b[4], b[5], b[6], b[7]);
    } else {
#pragma unroll
        for (uint32_t k = 0; k < 32; k++)
            if (k < cnt)
                p.sm[i0 + k] = (uint8_t)sign_mantissa(element(v, k));
    }
    __syncthreads();

    // the chunk's words; the first and last may hold a neighbour's bits too
    uint32_t *stream32 = reinterpret_cast<uint32_t *>(p.stream);
    for (uint32_t j = threadIdx.x; j < nbw; j += kThreads) {
        const uint32_t val = __byte_perm(bits[j], 0, 0x0123);
        if (j == 0 || j + 1 == nbw)
            atomicOr(&stream32[wb0 + j], val);
        else
            stream32[wb0 + j] = val;
    }
    uint32_t *gaps32 = reinterpret_cast<uint32_t *>(p.gaps);
    for (uint32_t j = threadIdx.x; j < ngw; j += kThreads) {
        if (j == 0 || j + 1 == ngw)
            atomicOr(&gaps32[gw0 + j], gbuf[j]);
        else
            gaps32[gw0 + j] = gbuf[j];
    }
}

__global__ void max_block_kernel(const uint32_t *offs, uint32_t nblocks, uint32_t *max_block)
{
    uint32_t m = 0;
    for (uint32_t b = blockIdx.x * blockDim.x + threadIdx.x; b < nblocks; b += gridDim.x * blockDim.x)
        m = max(m, offs[b + 1] - offs[b]);
    if (m)
        atomicMax(max_block, m);
}

bool aligned(const void *q, uintptr_t a) { return (reinterpret_cast<uintptr_t>(q) & (a - 1)) == 0; }

int sm_count()
{
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) !=
                                                  cudaSuccess)
        return 0;
    return sms;
}

// Scratch of df11_device_encode_static: one word per 8192-element chunk plus
// one, for streams of up to 2^16 chunks = 2^29 elements (512 KiB).  Every
// call writes each entry it reads before reading it, so nothing in it has to
// start at zero.  One array per device, shared by every call.
constexpr uint64_t kStaticMaxChunks = 1ull << 16;
static __device__ __align__(256) uint64_t g_static_scratch[kStaticMaxChunks + 1];

std::mutex g_static_mu;
uint64_t *g_static_addr[64] = {};  // per device, the last address looked up

// The array's device address on the current device.  It is looked up again
// on every call made while `s` is not being captured, so that a device reset
// (which reloads the module and may move the array) is picked up; a call
// made during a capture reuses the device's last looked-up address and fails
// with DF11_ERR_CUDA if there is none yet.
df11_status static_scratch(cudaStream_t s, uint64_t **out)
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        return DF11_ERR_CUDA;
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(s, &cap) != cudaSuccess)
        return DF11_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_static_mu);
    if (cap == cudaStreamCaptureStatusNone) {
        void *addr = nullptr;
        if (cudaGetSymbolAddress(&addr, g_static_scratch) != cudaSuccess || !addr)
            return DF11_ERR_CUDA;
        g_static_addr[dev] = static_cast<uint64_t *>(addr);
    }
    if (!g_static_addr[dev])
        return DF11_ERR_CUDA;
    *out = g_static_addr[dev];
    return DF11_OK;
}

}  // namespace

extern "C" df11_status df11_device_histogram(const uint16_t *w_dev, uint64_t n, uint64_t *hist_dev, void *stream)
{
    if (!hist_dev || (n && !w_dev) || !aligned(w_dev, 16))
        return DF11_ERR_INVALID_ARG;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(hist_dev, 0, 256 * sizeof(uint64_t), s) != cudaSuccess)
        return DF11_ERR_CUDA;
    if (!n)
        return DF11_OK;
    const int sms = sm_count();
    if (!sms)
        return DF11_ERR_CUDA;
    uint64_t grid = (n / 8 + kThreads - 1) / kThreads;
    if (grid > 4ull * sms)
        grid = 4ull * sms;
    if (grid == 0)
        grid = 1;
    histogram_kernel<<<(unsigned)grid, kThreads, 0, s>>>(w_dev, n, reinterpret_cast<unsigned long long *>(hist_dev));
    return cudaGetLastError() == cudaSuccess ? DF11_OK : DF11_ERR_CUDA;
}

extern "C" uint64_t df11_device_encode_scratch_words(uint64_t n)
{
    return (n + kChunk - 1) / kChunk + 1;
}

extern "C" df11_status df11_device_encode(const df11_format *plan, const uint16_t *w_dev, const df11_arrays *dst,
                                          uint64_t *scratch_dev, uint64_t scratch_words, uint32_t *max_block_dev,
                                          uint32_t *status_dev, void *stream)
{
    if (!plan || !dst || !max_block_dev || !status_dev)
        return DF11_ERR_INVALID_ARG;
    df11_arrays a;
    df11_status st = df11_format_arrays(plan, &a);
    if (st != DF11_OK)
        return st;
    const uint64_t n = a.n;
    if (n && (!w_dev || !aligned(w_dev, 16)))
        return DF11_ERR_INVALID_ARG;
    if (!dst->encoded_exponent || !dst->packed_sign_mantissa || !dst->gaps || !dst->block_offset || !dst->luts ||
        !dst->code_lengths)
        return DF11_ERR_INVALID_ARG;
    if (!aligned(dst->encoded_exponent, 16) || !aligned(dst->packed_sign_mantissa, 16) || !aligned(dst->gaps, 8) ||
        !aligned(dst->block_offset, 4))
        return DF11_ERR_INVALID_ARG;
    if (dst->encoded_exponent_bytes < a.encoded_exponent_bytes ||
        dst->packed_sign_mantissa_bytes < a.packed_sign_mantissa_bytes || dst->gaps_words < a.gaps_words)
        return DF11_ERR_INVALID_ARG;
    const uint64_t nchunks = (n + kChunk - 1) / kChunk;
    if (n && (!scratch_dev || scratch_words < nchunks + 1))
        return DF11_ERR_INVALID_ARG;

    EncParams prm;
    std::memset(&prm, 0, sizeof(prm));
    if (df11_internal_plan_codes(plan, prm.code) != DF11_OK)
        return DF11_ERR_INVALID_ARG;
    std::memcpy(prm.len, a.code_lengths, 256);
    prm.w = w_dev;
    prm.stream = const_cast<uint8_t *>(dst->encoded_exponent);
    prm.sm = const_cast<uint8_t *>(dst->packed_sign_mantissa);
    prm.gaps = const_cast<uint64_t *>(dst->gaps);
    prm.offs = const_cast<uint32_t *>(dst->block_offset);
    prm.chunk_bits = scratch_dev;
    prm.status = status_dev;
    prm.max_block = max_block_dev;
    prm.n = n;
    prm.total_bits = a.total_bits;
    prm.nseg = a.num_segments;
    prm.T = a.threads_per_block;
    // T / 32 in 1..32; unused for 1 (its reciprocal does not fit 32 bits)
    prm.t32_magic = prm.T == 32 ? 0u : (uint32_t)(((1ull << 32) + (prm.T / 32) - 1) / (prm.T / 32));
    prm.nblocks = a.num_blocks;
    prm.nchunks = (uint32_t)nchunks;

    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    uint8_t *luts_dev = const_cast<uint8_t *>(dst->luts);
    uint8_t *cl_dev = const_cast<uint8_t *>(dst->code_lengths);
    // the tables, and zeros wherever the kernels OR bits in or leave padding
    if (cudaMemcpyAsync(luts_dev, a.luts, 256ull * a.num_luts, cudaMemcpyHostToDevice, s) != cudaSuccess ||
        cudaMemcpyAsync(cl_dev, a.code_lengths, 256, cudaMemcpyHostToDevice, s) != cudaSuccess ||
        cudaMemsetAsync(prm.stream, 0, a.encoded_exponent_bytes, s) != cudaSuccess ||
        cudaMemsetAsync(prm.gaps, 0, a.gaps_words * 8, s) != cudaSuccess ||
        cudaMemsetAsync(prm.sm + n, 0, a.packed_sign_mantissa_bytes - n, s) != cudaSuccess ||
        cudaMemsetAsync(max_block_dev, 0, 4, s) != cudaSuccess)
        return DF11_ERR_CUDA;
    if (!n)
        return cudaMemsetAsync(prm.offs, 0, 4, s) == cudaSuccess ? DF11_OK : DF11_ERR_CUDA;

    const size_t smem = kBitWords * 4 + kGapWords * 4;
    chunk_bits_kernel<<<(unsigned)nchunks, kThreads, 0, s>>>(prm);
    chunk_scan_kernel<<<1, 1024, 0, s>>>(prm);
    encode_kernel<<<(unsigned)nchunks, kThreads, smem, s>>>(prm);
    const uint32_t mgrid = (a.num_blocks + 255) / 256;
    max_block_kernel<<<mgrid ? (mgrid < 1024 ? mgrid : 1024) : 1, 256, 0, s>>>(prm.offs, a.num_blocks, max_block_dev);
    return cudaGetLastError() == cudaSuccess ? DF11_OK : DF11_ERR_CUDA;
}

extern "C" df11_status df11_device_encode_static(const df11_format *plan, const uint16_t *w_dev,
                                                 const df11_arrays *dst, uint32_t *max_block_dev,
                                                 uint32_t *status_dev, void *stream)
{
    df11_arrays a;
    if (!plan || df11_format_arrays(plan, &a) != DF11_OK)
        return DF11_ERR_INVALID_ARG;
    if (df11_device_encode_scratch_words(a.n) > kStaticMaxChunks + 1)
        return DF11_ERR_TOO_LARGE;  // more than 2^29 elements
    uint64_t *scratch = nullptr;
    const df11_status st = static_scratch(reinterpret_cast<cudaStream_t>(stream), &scratch);
    if (st != DF11_OK)
        return st;
    return df11_device_encode(plan, w_dev, dst, scratch, kStaticMaxChunks + 1, max_block_dev, status_dev, stream);
}
