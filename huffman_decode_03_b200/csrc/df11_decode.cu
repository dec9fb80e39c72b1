// df11_decode.cu -- sm_100a kernel that rebuilds BF16 weights from DF11.
//
// "DFloat11: Kompresi inferensi GPU lossless ..." (id.news.hada.io/topic?id=20542):
//   "Decoding berbasis LUT hierarkis"  -- codes are resolved by table lookup
//        instead of a bit-by-bit tree walk; the tree is cut into height-8
//        subtrees stored as 256-entry LUTs whose values 240..255 are pointers;
//   "Kernel GPU 2 tahap dan metadata bantu" -- one thread per 8-byte segment
//        of EncodedExponent, starting at the segment's Gap; stage 1 counts the
//        codes of each segment, a block-wide prefix sum plus the block's stored
//        output position gives each thread its first output index, stage 2
//        decodes again and places the exponents in an on-chip write buffer,
//        and the block's outputs leave in one coalesced write; the encoded
//        stream is in shared memory before stage 1;
//   "Format DFloat11" -- sign and mantissa come verbatim from
//        PackedSignMantissa.
//
// B200 design (what differs from the page's kernel):
//   * persistent CTAs (a multiple of the SM count) walk the blocks; each
//     CTA stages the page's LUTs and CodeLengths once and derives two wider
//     tables from them in shared memory:
//       - a count table over the next 12 bits: how many whole codes they
//         hold and how many bits those codes use (stage 1 advances about 10
//         bits per lookup);
//       - a symbol table over the next 12 bits: up to 3 whole codes, their
//         total length and their exponents (stage 2 places ~3 exponents per
//         lookup).  Exponents are stored rotated right by one bit, which
//         turns the final BF16 merge into two bit-selects and two byte
//         permutes per 4 elements.
//     Codes longer than 12 bits fall back to the page's pointer-chasing LUTs.
//   * stage 1 stops exactly at the thread's last code: the next segment's
//     Gap gives the bit where the next thread starts; the final lookup masks
//     the bits past that point to zeros, and the codes the zeros form (the
//     all-zero code is the canonical first code) are subtracted.
//   * stage 2 runs until the thread has placed as many exponents as stage 1
//     counted; no second end test is needed.
//   * each thread's 64 + 32 bits live in a three-register shift window: the
//     table index is the top 12 bits, a step is three funnel shifts.
//   * the next block's EncodedExponent slice, Gaps words and
//     PackedSignMantissa slice are fetched by bulk asynchronous copies
//     (cp.async.bulk, completion on an mbarrier) while the current block is
//     decoded: two buffers per CTA.
//   * the block prefix sum is a warp-shuffle scan plus a scan of warp totals
//     (the page uses Blelloch's tree scan).
// Every loop and every wait is bounded; inconsistent data sets a status word
// and never traps.
#include "df11.h"

#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

namespace {

constexpr int kIdxBits = 12;                // index width of both derived tables
constexpr int kIdxEntries = 1 << kIdxBits;
constexpr int kLutBytes = DF11_MAX_LUTS * 256;
constexpr uint32_t kPointerBase = 240;
constexpr uint32_t kWaitTries = 1u << 22;   // bounded mbarrier polling

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
    uint32_t sm_cap;  // bytes of one PackedSignMantissa / exponent buffer
};

__host__ __device__ constexpr uint32_t align16(uint32_t x) { return (x + 15u) & ~15u; }

// Per-block bytes of the Gaps slice: fields T b .. T b + T (the extra field
// is the next block's first gap), whole 64-bit words, rounded to 16 bytes.
__host__ __device__ constexpr uint32_t gaps_slice_bytes(uint32_t T) { return align16((5 * T) / 8 + 16); }
__host__ __device__ constexpr uint32_t stream_slice_bytes(uint32_t T) { return T * 8 + 16; }

// Shared-memory layout in bytes.  The derived tables sit at fixed offsets so
// lookups need no base register.
struct SmemLayout {
    static constexpr uint32_t sym = 0;                              // uint32[4096]
    static constexpr uint32_t cnt = sym + kIdxEntries * 4;          // uint8[4096]
    static constexpr uint32_t luts = cnt + kIdxEntries;             // 17 * 256
    static constexpr uint32_t cl = luts + kLutBytes;                // 256
    static constexpr uint32_t ztab = cl + 256;                      // uint16[16]
    static constexpr uint32_t warp = ztab + 32;                     // uint32[32]
    static constexpr uint32_t bar = warp + 128;                     // 2 mbarriers
    static constexpr uint32_t scal = bar + 16;                      // 2 x {o0, o1, bad, pad}
    static constexpr uint32_t bufs = scal + 32;
    uint32_t buf_stride, stream_off, gaps_off, sm_off, exps, total;
    __host__ __device__ SmemLayout(uint32_t T, uint32_t sm_cap)
    {
        stream_off = 0;
        gaps_off = stream_off + align16(stream_slice_bytes(T));
        sm_off = gaps_off + gaps_slice_bytes(T);
        buf_stride = sm_off + sm_cap;
        exps = bufs + 2 * buf_stride;
        total = exps + sm_cap;
    }
};
static_assert(SmemLayout::bufs % 16 == 0, "buffers must be 16-byte aligned");

__device__ __forceinline__ uint32_t smem_addr(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

// Bounded wait for the phase with the given parity; false on timeout.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity)
{
    for (uint32_t i = 0; i < kWaitTries; i++) {
        uint32_t done;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(done)
            : "r"(bar), "r"(parity)
            : "memory");
        if (done)
            return true;
    }
    return false;
}

// Bulk global -> shared copy (no multicast), completion counted in bytes on
// the mbarrier.  Addresses 16-byte aligned, size a multiple of 16.
__device__ __forceinline__ void bulk_copy(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
        "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}

__device__ __forceinline__ void fence_proxy_async()
{
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ uint32_t load_be32(const uint8_t *p)
{
    return __byte_perm(*reinterpret_cast<const uint32_t *>(p), 0, 0x0123);
}

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

// Exclusive prefix sum over the block; *total receives the block sum.
template <int T>
__device__ __forceinline__ uint32_t block_exclusive_scan(uint32_t v, uint32_t *warp_sums, uint32_t *total)
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
            warp_sums[lane] = s;
    }
    __syncthreads();
    uint32_t before = warp ? warp_sums[warp - 1] : 0;
    *total = warp_sums[T / 32 - 1];
    return before + x - v;
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

template <int T>
__global__ void __launch_bounds__(T) df11_decode_kernel(const Params p)
{
    extern __shared__ __align__(128) uint8_t smem[];
    const SmemLayout L(T, p.sm_cap);
    uint32_t *sym_tab = reinterpret_cast<uint32_t *>(smem + SmemLayout::sym);
    uint8_t *cnt_tab = smem + SmemLayout::cnt;
    uint8_t *luts = smem + SmemLayout::luts;
    uint8_t *cl = smem + SmemLayout::cl;
    uint16_t *ztab = reinterpret_cast<uint16_t *>(smem + SmemLayout::ztab);
    uint32_t *warp_sums = reinterpret_cast<uint32_t *>(smem + SmemLayout::warp);
    uint32_t *scal = reinterpret_cast<uint32_t *>(smem + SmemLayout::scal);
    uint8_t *exp_s = smem + L.exps;
    const uint32_t bar0 = smem_addr(smem + SmemLayout::bar);
    const int tid = threadIdx.x;
    const uint32_t G = gridDim.x;

    // thread 0: fetch block b into buffer k (offsets from registers o0, o1)
    auto issue = [&](uint32_t b, int k, uint32_t o0, uint32_t o1) {
        uint8_t *buf = smem + SmemLayout::bufs + k * L.buf_stride;
        const uint32_t bar = bar0 + 8 * k;
        const uint32_t base = o0 & ~15u;
        const uint64_t end16 = ((uint64_t)o1 + 15u) & ~(uint64_t)15u;
        const bool ok = o1 >= o0 && (uint64_t)o1 <= p.n && end16 - base <= p.sm_cap;
        const uint32_t sm_bytes = ok ? (uint32_t)(end16 - base) : 0u;
        scal[4 * k + 0] = o0;
        scal[4 * k + 1] = o1;
        scal[4 * k + 2] = ok ? 0u : 1u;
        fence_proxy_async();
        mbar_arrive_expect_tx(bar, stream_slice_bytes(T) + gaps_slice_bytes(T) + sm_bytes);
        bulk_copy(smem_addr(buf + L.stream_off), p.stream + (uint64_t)b * T * 8, stream_slice_bytes(T), bar);
        bulk_copy(smem_addr(buf + L.gaps_off), reinterpret_cast<const uint8_t *>(p.gaps) + (uint64_t)b * (5 * T / 8),
                  gaps_slice_bytes(T), bar);
        if (sm_bytes)
            bulk_copy(smem_addr(buf + L.sm_off), p.sm + base, sm_bytes, bar);
    };

    // ---- once per CTA: barriers, the page's LUTs, derived tables
    uint32_t next_o0 = 0, next_o1 = 0;
    if (tid == 0) {
        mbar_init(bar0, 1);
        mbar_init(bar0 + 8, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        fence_proxy_async();
        const uint32_t b = blockIdx.x;
        issue(b, 0, __ldg(p.offs + b), __ldg(p.offs + b + 1));
        if (b + G < p.nblocks) {
            next_o0 = __ldg(p.offs + b + G);
            next_o1 = __ldg(p.offs + b + G + 1);
        }
    }
    const uint32_t lut_bytes = p.num_luts * 256u;
    for (uint32_t i = tid; i < lut_bytes; i += T)
        luts[i] = p.luts[i];
    for (uint32_t i = tid; i < 256; i += T)
        cl[i] = p.cl[i];
    __syncthreads();
    for (uint32_t i = tid; i < kIdxEntries; i += T) {
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
        sym_tab[i] = syms | (sym_bits << 24) | (sym_n << 28);
    }
    if (tid <= kIdxBits) {
        // codes formed by r..11 zero bits after a code boundary: the all-zero
        // code (the canonical first code) repeated; count | bits << 8
        bool bad = false;
        const uint32_t lmin = lut_decode(0u, luts, cl, p.num_luts, &bad) >> 8;
        const uint32_t z = (lmin >= 1 && !bad) ? (kIdxBits - tid) / lmin : 0u;
        ztab[tid] = (uint16_t)(z | ((z * lmin) << 8));
    }
    __syncthreads();

    uint32_t i = 0;
    for (uint32_t b = blockIdx.x; b < p.nblocks; b += G, i++) {
        const int k = i & 1;
        if (tid == 0 && b + G < p.nblocks) {
            issue(b + G, k ^ 1, next_o0, next_o1);
            if (b + 2 * G < p.nblocks) {
                next_o0 = __ldg(p.offs + b + 2 * G);
                next_o1 = __ldg(p.offs + b + 2 * G + 1);
            }
        }
        const bool timed_out = !mbar_wait(bar0 + 8 * k, (i >> 1) & 1);
        if (__syncthreads_or(timed_out)) {
            if (tid == 0)
                atomicOr(p.status, (uint32_t)DF11_ERR_CORRUPT);
            mbar_wait(bar0 + 8 * (k ^ 1), ((i + 1) >> 1) & 1);  // bounded: copies still in flight
            return;
        }
        const uint8_t *buf = smem + SmemLayout::bufs + k * L.buf_stride;
        const uint8_t *stream_s = buf + L.stream_off;
        const uint64_t *gaps_s = reinterpret_cast<const uint64_t *>(buf + L.gaps_off);
        const uint8_t *sm_s = buf + L.sm_off;
        const uint32_t o0 = scal[4 * k + 0], o1 = scal[4 * k + 1];
        const bool offs_bad = scal[4 * k + 2] != 0;
        const uint32_t lo_off = o0 & 15u;

        // ---- locate: this thread's codes start in [pos0, pend) of its window
        const uint64_t seg = (uint64_t)b * T + tid;
        int pos0 = 0, pend = 0;
        {
            const uint32_t bit = 5u * tid;
            const uint32_t w = bit >> 6, off = bit & 63u;
            uint64_t v = gaps_s[w] >> off;
            if (off > 54)  // fields tid and tid + 1 reach into the next word
                v |= gaps_s[w + 1] << (64 - off);
            const uint32_t g0 = (uint32_t)v & 31u, g1 = (uint32_t)(v >> 5) & 31u;
            if (seg < p.nseg) {
                pos0 = (int)g0;
                pend = seg + 1 < p.nseg ? 64 + (int)g1 : (int)(p.total_bits - 64 * seg);
            }
        }
        const uint32_t w0 = load_be32(stream_s + 8 * tid);
        const uint32_t w1 = load_be32(stream_s + 8 * tid + 4);
        const uint32_t w2 = load_be32(stream_s + 8 * tid + 8);

        // ---- stage 1: count the codes starting in [pos0, pend)
        bool bad = false;
        uint32_t cnt = 0;
        {
            uint32_t h = w0, m = w1, l = w2;
            shift_window(h, m, l, (uint32_t)pos0);
            int pos = pos0;
            for (int it = 0; it < 64 && pend - pos > kIdxBits; it++) {
                uint32_t e = cnt_tab[h >> (32 - kIdxBits)];
                uint32_t c = e >> 4;
                if (c == 0) {  // a code longer than 12 bits
                    c = lut_decode(h, luts, cl, p.num_luts, &bad) >> 8;
                    e = 1;
                }
                cnt += e & 15u;
                pos += (int)c;
                shift_window(h, m, l, c);
            }
            const int r = pend - pos;
            if (r > kIdxBits) {
                bad = true;  // the loop bound ran out: not a valid segment
            } else if (r > 0) {
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

        uint32_t total;
        const uint32_t first = block_exclusive_scan<T>(cnt, warp_sums, &total);
        const bool block_bad = __syncthreads_or(bad) || offs_bad || total != o1 - o0 ||
                               lo_off + total + 16u > p.sm_cap;
        if (block_bad) {
            if (tid == 0)
                atomicOr(p.status, (uint32_t)DF11_ERR_CORRUPT);
            __syncthreads();
            continue;
        }

        // ---- stage 2: decode again, place rotated exponents
        {
            uint32_t h = w0, m = w1, l = w2;
            shift_window(h, m, l, (uint32_t)pos0);
            uint32_t q = lo_off + first;
            const uint32_t qend = q + cnt;
            for (int it = 0; it < 64 && q < qend; it++) {
                uint32_t e = sym_tab[h >> (32 - kIdxBits)];
                uint32_t c = (e >> 24) & 15u, nsym = e >> 28;
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
        __syncthreads();

        // ---- merge with sign/mantissa, coalesced 16-byte stores
        {
            const uint32_t hi = lo_off + total;
            const uint64_t g0 = (uint64_t)o0 - lo_off;  // multiple of 16
            const uint32_t nchunks = (hi + 15) / 16;
            for (uint32_t c = tid; c < nchunks; c += T) {
                const uint32_t l0 = 16 * c;
                if (l0 >= lo_off && l0 + 16 <= hi) {
                    const uint4 s = *reinterpret_cast<const uint4 *>(sm_s + l0);
                    const uint4 e = *reinterpret_cast<const uint4 *>(exp_s + l0);
                    uint4 r0, r1;
                    merge4(s.x, e.x, r0.x, r0.y);
                    merge4(s.y, e.y, r0.z, r0.w);
                    merge4(s.z, e.z, r1.x, r1.y);
                    merge4(s.w, e.w, r1.z, r1.w);
                    uint4 *d = reinterpret_cast<uint4 *>(p.dst + g0 + l0);
                    d[0] = r0;
                    d[1] = r1;
                } else {
                    for (uint32_t j = 0; j < 16; j++) {
                        const uint32_t l = l0 + j;
                        if (l >= lo_off && l < hi)
                            p.dst[g0 + l] = merge1(sm_s[l], exp_s[l]);
                    }
                }
            }
        }
        __syncthreads();
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

template <int T>
df11_status launch(const Params &prm, cudaStream_t stream)
{
    const SmemLayout L(T, prm.sm_cap);
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

extern "C" df11_status df11_decompress(const df11_arrays *a, uint16_t *dst, uint32_t *status_dev, void *stream)
{
    if (!a || !status_dev)
        return DF11_ERR_INVALID_ARG;
    if (a->n == 0)
        return DF11_OK;
    const uint32_t T = a->threads_per_block;
    if (T != 128 && T != 256 && T != 512)
        return DF11_ERR_INVALID_ARG;
    if (!dst || !a->encoded_exponent || !a->packed_sign_mantissa || !a->gaps || !a->block_offset || !a->luts ||
        !a->code_lengths)
        return DF11_ERR_INVALID_ARG;
    if (!aligned(dst, 16) || !aligned(a->encoded_exponent, 16) || !aligned(a->packed_sign_mantissa, 16) ||
        !aligned(a->gaps, 16) || !aligned(a->block_offset, 4))
        return DF11_ERR_INVALID_ARG;
    if (a->num_luts < 1 || a->num_luts > DF11_MAX_LUTS || a->n >= (1ull << 32))
        return DF11_ERR_INVALID_ARG;
    const uint64_t nseg = (a->total_bits + 63) / 64;
    if (nseg != a->num_segments || (nseg + T - 1) / T != a->num_blocks || a->num_blocks == 0)
        return DF11_ERR_INVALID_ARG;
    // every bulk copy must stay inside its array
    if (a->encoded_exponent_bytes < (uint64_t)a->num_blocks * T * 8 + 16 ||
        a->packed_sign_mantissa_bytes < ((a->n + 15) / 16) * 16 ||
        a->gaps_words * 8 < (uint64_t)(a->num_blocks - 1) * (5 * T / 8) + gaps_slice_bytes(T) ||
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
    prm.sm_cap = align16(a->max_block_elems + 32);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    switch (T) {
    case 128: return launch<128>(prm, s);
    case 256: return launch<256>(prm, s);
    default: return launch<512>(prm, s);
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
