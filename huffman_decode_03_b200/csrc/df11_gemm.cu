// df11_gemm.cu -- sm_100a: DF11 weights decoded straight into tensor-core
// operand tiles and multiplied by a batch of activation vectors
// (tcgen05.mma, float32 accumulators in tensor memory).  The BF16 weights
// never exist in global memory.
//
// "DFloat11: Kompresi inferensi GPU lossless ..." (id.news.hada.io/topic?id=20542),
// "Dekompresi yang disesuaikan untuk inferensi GPU": weights are decompressed
// right before the matrix multiplication that uses them and discarded after
// it; the page's discussion proposes a GEMM that decompresses each tile just
// before its arithmetic.  This is that GEMM: Y_m += X_m W_m^T for every matrix
// m of a stream, X_m holding `batch` activation vectors of cols_m elements.
//
// Element order.  A DF11 stream is one run of elements whose order the page
// leaves to the compressor.  Here each matrix is stored in 128 x 64 tiles:
// its row tiles (128 rows) in order, within a row tile its column tiles (64
// columns) in order, within a tile its 128 rows of 64 elements
// (df11_tile_major writes this order).  So 8192 consecutive stream elements
// are one A operand tile of the MMA (M = 128 rows, K = 64), and the K chunks
// of a row tile follow one another.
//
// Work unit: up to 16 consecutive K chunks of one row tile of one matrix.  A
// prep kernel packs every 64-column chunk of X into the shared-memory image
// the tensor core reads and finds each unit's first and last format block.
// Then one persistent CTA per SM takes units blockIdx.x, + gridDim.x, ...:
//   * DW decode warps (27, the most a 1024-thread CTA seats beside the
//     control and epilogue warps, when at least 3 ring stages fit beside
//     them; else 20; else 16): warp w decodes the unit's format blocks w,
//     w + DW, ... with the per-block decode shared with the other kernels,
//     merges each exponent with its sign/mantissa byte and stores the BF16 weight at its
//     place in a ring of S operand tiles in shared memory (K-major, 128-byte
//     swizzle).  A warp arrives on a tile's "full" barrier as soon as none
//     of its remaining blocks reaches into that tile: on the tiles before a
//     block's first output BEFORE it waits for that block's ring slots (a
//     slot frees only after the MMA of an earlier tile, which needs every
//     warp's arrival), and on those before its next block right after;
//   * 1 control warp: allocates tensor memory; one of its threads copies each
//     K chunk of X into the ring by a bulk copy (cp.async.bulk, no tensor
//     map), waits for the tile to be full, issues four tcgen05.mma (K = 16
//     each) into the unit's accumulator and frees the ring slot with
//     tcgen05.commit;
//   * 4 epilogue warps: read the 128 x batch float32 accumulator with
//     tcgen05.ld and add it into Y by atomic adds (the units of one row tile
//     share its rows).  Two accumulators let the next unit's MMAs start while
//     the last one is read out.
// Every wait on a barrier is bounded.  When one runs out, the kernel sets bit
// 31 of the status word and an abort flag on which every role stops, waits
// (bounded) for its own copies and MMAs in flight, frees its tensor memory and
// ends.  Inconsistent data sets DF11_ERR_CORRUPT as in the other kernels; a
// unit whose tiles did not receive exactly their elements is reported too.
#include "df11.h"
#include "df11_block.cuh"

#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>
#include <mutex>

namespace {

constexpr uint32_t kTileRows = 128, kTileCols = 64;
constexpr uint32_t kTileElems = kTileRows * kTileCols;  // 8192
constexpr uint32_t kTileShift = 13;
constexpr uint32_t kTileBytes = kTileElems * 2;          // 16 KB
// DW decode warps, then the control warp (warp DW), then 4 epilogue warps.
// 27, 20 or 16 decode warps, the most that leave room for enough exponent
// tiles (more warps hide more of the decode loop's latency).
__host__ __device__ constexpr uint32_t gemm_threads(uint32_t dw) { return (dw + 1 + 4) * 32; }
constexpr uint32_t kStages = 2;     // operand tiles in the ring (the MMA is short)
constexpr uint32_t kMaxETiles = 16;  // exponent tiles, at most
constexpr uint32_t kUnitChunks = 16;  // K chunks per work unit, at most
constexpr uint32_t kMaxGemmMats = 16;
constexpr uint32_t kSpinLimit = 1u << 22;         // polls of one wait, at most
constexpr uint64_t kWaitLimitNs = 1000000000ull;  // and 1 s of waiting
constexpr uint32_t kSuspendNs = 20000;            // a poll sleeps up to 20 us unless the phase completes
constexpr uint32_t kTimeoutFlag = 0x80000000u;

// Barrier and flag area after the decode warps' buffers: full[8], empty[8],
// xfull[8], accf[2], tfree[2], drain (8 bytes each), then the tensor-memory
// address, the abort flag, the count of MMAs known complete, and per
// exponent tile its element count and its count of merges (both over all
// its uses).  Counters, not barriers, for the waits of the decode warps: a
// warp may run two or more uses ahead of a tile, and an mbarrier's phase
// parity cannot tell those uses apart.
constexpr uint32_t kBarFull = 0, kBarEmpty = 8, kBarX = 16, kBarAcc = 24, kBarFree = 26, kBarDrain = 28;
constexpr uint32_t kNumBars = 29;
constexpr uint32_t kCtrlBytes = 1024;
static_assert(kNumBars * 8 + 12 + 8 * kMaxETiles <= kCtrlBytes, "control area");

struct GemmMat {
    uint32_t off;           // first stream element
    uint32_t rows, cols;    // multiples of 128 and 64
    uint32_t unit0;         // its first work unit
    uint32_t units_per_rt;  // work units per row tile
    uint32_t piece0;        // its first 16-byte piece of X (packing)
    uint64_t xoff;          // byte offset of its packed X
    const uint16_t *x;      // batch x cols BF16, row-major
    float *y;               // batch x rows float32, row-major
};

struct GemmParams {
    // the stream: the fields the shared per-block decode reads
    const uint8_t *stream;
    const uint8_t *sm;
    const uint32_t *gaps;
    const uint32_t *offs;
    const uint8_t *luts;
    const uint8_t *cl;
    const uint32_t *sym_table;  // optional stored symbol table (null: derived per CTA)
    uint32_t *status;
    uint64_t n;
    uint64_t total_bits;
    uint64_t nseg;
    uint32_t nblocks;
    uint32_t num_luts;
    uint32_t cap;
    uint32_t min_code_len;  // from the stream's arrays: 0 when not known
    // the product
    uint32_t batch;      // N of the MMA
    uint32_t stages;     // S, operand tiles in the ring
    uint32_t etiles;     // E, exponent tiles
    uint32_t tmem_cols;  // power of two >= 2 * batch
    uint32_t num_mats;
    uint32_t num_units;
    uint32_t num_pieces;
    uint8_t *xpack;           // packed X of every matrix
    uint32_t *unit_blocks;    // per unit: first block, end block (exclusive)
    GemmMat mats[kMaxGemmMats];
};

__host__ __device__ constexpr uint32_t ctrl_offset(uint32_t cap, uint32_t dw, uint32_t slot)
{
    return align16(Smem::bufs + dw * Smem::per_warp(cap, slot));
}

// Dynamic shared memory of a launch: tables, decode buffers, control area,
// 1 KB to align the ring, the operand ring (weight and activation tiles),
// the exponent tiles.
__host__ __device__ constexpr uint32_t gemm_smem_bytes(uint32_t cap, uint32_t batch, uint32_t stages, uint32_t etiles,
                                                      uint32_t dw, uint32_t slot)
{
    return ctrl_offset(cap, dw, slot) + kCtrlBytes + 1024 + stages * (kTileBytes + batch * 128) + etiles * kTileElems;
}

// Instruction descriptor of tcgen05.mma kind::f16: BF16 A and B, both
// K-major, float32 accumulator, M x N.
__host__ __device__ constexpr uint32_t idesc_bf16(uint32_t m, uint32_t n)
{
    return (1u << 4) | (1u << 7) | (1u << 10) | ((n >> 3) << 17) | ((m >> 4) << 24);
}

// Shared-memory matrix descriptor of a K-major operand in the 128-byte
// swizzled layout: rows of 64 BF16 (128 bytes) at a 128-byte pitch, groups of
// 8 rows 1024 bytes apart; saddr 1024-byte aligned (K step k adds 32 k bytes).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr)
{
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | (1ull << 16) | ((uint64_t)(1024 >> 4) << 32) | (1ull << 46) |
           (2ull << 61);
}

// Byte offset of element i (row-major 128 x 64) of an operand tile in that
// layout: the 16-byte group of 8 columns is XORed with the row mod 8.
__device__ __forceinline__ uint32_t tile_offset(uint32_t i)
{
    const uint32_t r = i >> 6, c = i & 63u;
    return (r << 7) + ((((c >> 3) ^ r) & 7u) << 4) + ((c & 7u) << 1);
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_arrive_tx(uint32_t bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// The same test, but a thread whose phase is not complete is suspended in
// hardware until it completes or kSuspendNs pass: a waiting warp takes no
// issue slots from the decode warps while it waits.
__device__ __forceinline__ bool mbar_try_sleep(uint32_t bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity), "r"(kSuspendNs)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ uint64_t global_ns()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Waits until the barrier's phase of the given parity has completed.  Gives
// up (false) when the kernel is aborting (checked every 8 polls), or after
// kWaitLimitNs or kSpinLimit polls, which starts the abort.  With
// honour_abort false it keeps waiting during an abort (used to drain the
// kernel's own copies and MMAs).
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile uint32_t *abort_flag,
                                          uint32_t *status, bool honour_abort = true)
{
    if (mbar_try(bar, parity))
        return true;
    const uint64_t t0 = global_ns();
    for (uint32_t i = 1; i < kSpinLimit; i++) {
        if (mbar_try_sleep(bar, parity))
            return true;
        if ((i & 7u) == 0) {
            if (honour_abort && *abort_flag)
                return false;
            if (global_ns() - t0 > kWaitLimitNs)
                break;
        }
    }
    *abort_flag = 1u;
    atomicOr(status, kTimeoutFlag);
    return false;
}

__device__ __forceinline__ void bulk_copy_g2s(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar)
{
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
                 "l"(src), "r"(bytes), "r"(bar)
                 : "memory");
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint4 v)
{
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}

__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void umma_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrives on the barrier once every tcgen05 operation this thread issued
// before has completed.
__device__ __forceinline__ void umma_commit(uint32_t bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}

// 32 lanes x 16 consecutive float32 columns of tensor memory.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16])
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
          "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Work unit u: its matrix, first row, first K chunk, number of K chunks and
// first stream element.
struct Unit {
    uint32_t m, row0, kc0, ntiles, e0;
};

__device__ __forceinline__ Unit unit_of(const GemmParams &p, uint32_t u)
{
    uint32_t m = 0;
    while (m + 1 < p.num_mats && u >= p.mats[m + 1].unit0)
        m++;
    const GemmMat &M = p.mats[m];
    const uint32_t rel = u - M.unit0, rt = rel / M.units_per_rt, ku = rel - rt * M.units_per_rt;
    const uint32_t kchunks = M.cols / kTileCols, kc0 = ku * kUnitChunks;
    Unit U;
    U.m = m;
    U.row0 = rt * kTileRows;
    U.kc0 = kc0;
    U.ntiles = kchunks - kc0 < kUnitChunks ? kchunks - kc0 : kUnitChunks;
    U.e0 = M.off + (rt * kchunks + kc0) * kTileElems;
    return U;
}

// Largest block b < nblocks with offs[b] <= x (offs[0] = 0).
__device__ __forceinline__ uint32_t block_of(const uint32_t *offs, uint32_t nblocks, uint32_t x)
{
    uint32_t lo = 0, hi = nblocks - 1;
    while (lo < hi) {
        const uint32_t mid = (lo + hi + 1) >> 1;
        if (__ldg(offs + mid) <= x)
            lo = mid;
        else
            hi = mid - 1;
    }
    return lo;
}

// Packs X (one thread per 16-byte piece: 8 activations of one vector) into
// the operand image of each K chunk, and finds each unit's blocks.
__global__ void gemm_prep_kernel(const GemmParams p)
{
    // the GEMM kernel may launch now and do its set-up beside this one; it
    // waits (griddepcontrol.wait) before it reads what this kernel writes
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const uint32_t g = blockIdx.x * blockDim.x + threadIdx.x;
    if (g < p.num_pieces) {
        uint32_t m = 0;
        while (m + 1 < p.num_mats && g >= p.mats[m + 1].piece0)
            m++;
        const GemmMat &M = p.mats[m];
        const uint32_t per_vec = M.cols / 8, idx = g - M.piece0;
        const uint32_t v = idx / per_vec, j8 = idx - v * per_vec, kc = j8 >> 3, j = j8 & 7u;
        const uint4 d = __ldg(reinterpret_cast<const uint4 *>(M.x + (uint64_t)v * M.cols + 8 * j8));
        uint8_t *dst = p.xpack + M.xoff + (uint64_t)kc * p.batch * 128 + v * 128 + (((j ^ v) & 7u) << 4);
        *reinterpret_cast<uint4 *>(dst) = d;
    }
    if (g < p.num_units) {
        const Unit U = unit_of(p, g);
        const uint32_t e1 = U.e0 + U.ntiles * kTileElems;
        p.unit_blocks[2 * g] = block_of(p.offs, p.nblocks, U.e0);
        p.unit_blocks[2 * g + 1] = block_of(p.offs, p.nblocks, e1 - 1) + 1;
    }
}

struct Roles {
    uint32_t ring_a, ring_b, ring_e, bars;  // shared addresses
    volatile uint32_t *abort_flag;
    volatile uint32_t *mma_done;  // the MMAs of tiles 0 .. mma_done - 1 have completed
    uint32_t *ecount;             // per exponent tile: elements received, over all its uses
    volatile uint32_t *emerged;   // per exponent tile: uses merged
    uint32_t tmem;
};

// Waits until *c >= target (a counter that only grows).  Gives up like
// mbar_wait: when the kernel is aborting, or after kWaitLimitNs or
// kSpinLimit polls, which starts the abort.
__device__ __forceinline__ bool count_wait(const volatile uint32_t *c, uint32_t target, const Roles &R,
                                           uint32_t *status)
{
    if (*c >= target)
        return true;
    const uint64_t t0 = global_ns();
    for (uint32_t i = 1; i < kSpinLimit; i++) {
        __nanosleep(1000);
        if (*c >= target)
            return true;
        if ((i & 7u) == 0) {
            if (*R.abort_flag)
                return false;
            if (global_ns() - t0 > kWaitLimitNs)
                break;
        }
    }
    *R.abort_flag = 1u;
    atomicOr(status, kTimeoutFlag);
    return false;
}

__device__ __forceinline__ uint32_t bar(const Roles &R, uint32_t i) { return R.bars + 8 * i; }

__device__ __forceinline__ uint4 ld_shared_v4(uint32_t addr)
{
    uint4 v;
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(addr)
                 : "memory");
    return v;
}

__device__ __forceinline__ void st_shared_u8(uint32_t addr, uint32_t v)
{
    asm volatile("st.shared.u8 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

// The sign/mantissa bytes of this lane in one quarter (2048 elements) of
// the tile whose first stream element is tile0 (four 16-byte loads, from L2).
__device__ __forceinline__ void load_quarter(const GemmParams &p, uint64_t tile0, uint32_t quarter, int lane,
                                             uint4 (&s4)[4])
{
    const uint8_t *smt = p.sm + tile0 + 2048u * quarter + 16u * (uint32_t)lane;
#pragma unroll
    for (uint32_t j = 0; j < 4; j++)
        s4[j] = __ldg(reinterpret_cast<const uint4 *>(smt + 512u * j));
}

// One quarter of tile q, whose 8192 exponents are all in its exponent tile:
// merged with the sign/mantissa bytes s4 (load_quarter) into operand slot
// q mod S, at the swizzled positions the tensor core reads.  The caller has
// waited until the slot is free.  One warp.
__device__ __forceinline__ void merge_quarter(const GemmParams &p, const Roles &R, uint32_t q, uint32_t quarter,
                                              int lane, const uint4 (&s4)[4])
{
    const uint32_t ea = R.ring_e + (q % p.etiles) * kTileElems, sa = R.ring_a + (q % p.stages) * kTileBytes;
#pragma unroll
    for (uint32_t j = 0; j < 4; j++) {
        const uint32_t l = 2048u * quarter + 512u * j + 16u * (uint32_t)lane;
        const uint4 e4 = ld_shared_v4(ea + l);
        uint4 r0, r1;
        merge4(s4[j].x, e4.x, r0.x, r0.y);
        merge4(s4[j].y, e4.y, r0.z, r0.w);
        merge4(s4[j].z, e4.z, r1.x, r1.y);
        merge4(s4[j].w, e4.w, r1.z, r1.w);
        const uint32_t a0 = sa + tile_offset(l);
        st_shared_v4(a0, r0);
        st_shared_v4(a0 ^ 16u, r1);  // the next 8 columns: group index + 1, XOR row
    }
}

// Decode warp: every unit of the CTA, blocks warp, warp + DW, ... of it.
// Each block is decoded into the warp's own buffer; its exponents are then
// copied to their places in the exponent tiles of the tiles it covers (once
// those are free: tile q - E merged), and the tiles' element counters are
// advanced.  A decode warp waits only for exponent tiles, and the decode
// itself never waits.
template <int C, int DW, uint32_t SLOT>
__device__ __forceinline__ void decode_role(const GemmParams &p, const Roles &R, uint8_t *smem, uint32_t warp,
                                            int lane)
{
    const uint32_t E = p.etiles;
    uint8_t *exp_s = smem + Smem::bufs + warp * Smem::per_warp(p.cap, SLOT);
    const uint32_t sym_base = static_cast<uint32_t>(__cvta_generic_to_shared(smem + Smem::sym));
    const uint32_t exp_base = static_cast<uint32_t>(__cvta_generic_to_shared(exp_s));
    const uint32_t slot_base =
        static_cast<uint32_t>(__cvta_generic_to_shared(exp_s + p.cap)) + (uint32_t)lane * SLOT;

    uint32_t q0 = 0;  // tile sequence number of the unit's first tile
    // waits until exponent tile q may be written (the four quarters of tile
    // q - E have been merged)
    auto etile_free = [&](uint32_t q) -> bool {
        if (q < E)
            return true;
        const bool ok = __all_sync(0xffffffffu, count_wait(R.emerged + q % E, 4 * (q / E), R, p.status));
        __threadfence_block();
        return ok;
    };
    for (uint32_t u = blockIdx.x; u < p.num_units; u += gridDim.x) {
        if (*R.abort_flag)
            return;
        const Unit U = unit_of(p, u);
        const uint64_t e0 = U.e0, e1 = e0 + (uint64_t)U.ntiles * kTileElems;
        const uint32_t bb = p.unit_blocks[2 * u], be = p.unit_blocks[2 * u + 1];
        BlockRegs<C> cur, nxt;
        uint32_t b = bb + warp;
        if (b < be)
            load_block<C>(p, b, lane, cur);
        for (; b < be; b += DW) {
            if (b + DW < be)
                load_block<C>(p, b + DW, lane, nxt);
            // the block's share of the unit, by its offsets: [r0, r1)
            const uint64_t o0 = cur.o0, o1 = cur.o1 > cur.o0 ? cur.o1 : cur.o0;
            const uint64_t r0 = o0 > e0 ? o0 : e0, r1 = o1 < e1 ? o1 : e1;
            BlockOut bo;
            const bool dok = decode_block<C, SLOT, false, 1>(p, b, lane, cur, sym_base, exp_base, slot_base, bo);
            if (r0 < r1) {
                const uint32_t t_first = (uint32_t)((r0 - e0) >> kTileShift);
                const uint32_t t_last = (uint32_t)((r1 - 1 - e0) >> kTileShift);
                for (uint32_t t = t_first; t <= t_last; t++)
                    if (!etile_free(q0 + t))
                        return;
                if (dok) {
                    // exponents [lo, hi) of the block (relative to g0) to their exponent tiles
                    const uint64_t g0 = bo.g0;
                    const uint32_t lo = (uint32_t)(r0 - g0), hi = (uint32_t)(r1 - g0);
                    const uint32_t ea0 = R.ring_e + ((q0 + t_first) % E) * kTileElems;
                    const uint32_t ea1 = R.ring_e + ((q0 + t_first + 1) % E) * kTileElems;
                    auto eaddr = [&](uint32_t l) {
                        const uint32_t v = (uint32_t)(g0 + l - e0);
                        return ((v >> kTileShift) == t_first ? ea0 : ea1) + (v & (kTileElems - 1));
                    };
                    // whole groups of 16 (a group never crosses a tile) ...
                    const uint32_t c_lo = (lo + 15u) & ~15u, c_hi = hi & ~15u;
                    for (uint32_t l0 = c_lo + 16u * lane; l0 < c_hi; l0 += 512u)
                        st_shared_v4(eaddr(l0), *reinterpret_cast<const uint4 *>(exp_s + l0));
                    // ... and up to 15 single bytes at each end
                    const uint32_t head_end = c_lo < hi ? c_lo : hi, tail0 = c_hi > c_lo ? c_hi : c_lo;
                    const uint32_t l = lane < 16 ? lo + lane : tail0 + (lane - 16);
                    if (lane < 16 ? l < head_end : l < hi)
                        st_shared_u8(eaddr(l), exp_s[l]);
                }
                // counted after every lane's copies (a corrupt block still
                // counts its elements, so no tile waits for ever)
                __syncwarp();
                if (lane == 0) {
                    __threadfence_block();
                    for (uint32_t t = t_first; t <= t_last; t++) {
                        const uint64_t a = e0 + ((uint64_t)t << kTileShift), z = a + kTileElems;
                        const uint32_t cnt = (uint32_t)((r1 < z ? r1 : z) - (r0 > a ? r0 : a));
                        const uint32_t q = q0 + t, full = (q / E + 1) * kTileElems;
                        if (atomicAdd(R.ecount + q % E, cnt) + cnt > full)
                            atomicOr(p.status, (uint32_t)DF11_ERR_CORRUPT);
                    }
                }
            }
            cur = nxt;
        }
        q0 += U.ntiles;
    }
}

// Control thread: X copies, MMAs, commits.
__device__ __forceinline__ void control_role(const GemmParams &p, const Roles &R)
{
    const uint32_t S = p.stages, N = p.batch, xbytes = N * 128;
    const uint32_t idesc = idesc_bf16(kTileRows, N);
    uint32_t q0 = 0, k = 0, x_issued = 0, x_used = 0, committed = 0;
    bool ok = true;
    for (uint32_t u = blockIdx.x; u < p.num_units && ok; u += gridDim.x, k++) {
        const Unit U = unit_of(p, u);
        const GemmMat &M = p.mats[U.m];
        const uint8_t *xsrc = p.xpack + M.xoff + (uint64_t)U.kc0 * xbytes;
        const uint32_t d = k & 1u;
        // X chunk of tile t of the unit into its slot, once the slot is free
        auto issue_x = [&](uint32_t t) -> bool {
            const uint32_t q = q0 + t, s = q % S;
            if (q >= S && !mbar_wait(bar(R, kBarEmpty + s), (q / S - 1) & 1u, R.abort_flag, p.status))
                return false;
            mbar_arrive_tx(bar(R, kBarX + s), xbytes);
            bulk_copy_g2s(R.ring_b + s * xbytes, xsrc + (uint64_t)t * xbytes, xbytes, bar(R, kBarX + s));
            x_issued = q + 1;
            return true;
        };
        const uint32_t ahead = S - 1 < U.ntiles ? S - 1 : U.ntiles;
        for (uint32_t t = 0; t < ahead && ok; t++)
            ok = issue_x(t);
        // the accumulator is free once the epilogue has read unit k - 2
        if (ok && k >= 2)
            ok = mbar_wait(bar(R, kBarFree + d), ((k >> 1) - 1) & 1u, R.abort_flag, p.status);
        for (uint32_t t = 0; t < U.ntiles && ok; t++) {
            const uint32_t q = q0 + t, s = q % S, ph = (q / S) & 1u;
            ok = mbar_wait(bar(R, kBarFull + s), ph, R.abort_flag, p.status) &&
                 mbar_wait(bar(R, kBarX + s), ph, R.abort_flag, p.status);
            if (!ok)
                break;
            x_used = q + 1;
            tc_fence_after();
            const uint64_t ad = sw128_desc(R.ring_a + s * kTileBytes), bd = sw128_desc(R.ring_b + s * xbytes);
#pragma unroll
            for (uint32_t kk = 0; kk < 4; kk++)
                umma_bf16(R.tmem + d * N, ad + 2 * kk, bd + 2 * kk, idesc, (t | kk) != 0);
            umma_commit(bar(R, kBarEmpty + s));
            committed = 1;
            // the MMA's completion, published at once: the decode warp that
            // merges tile q + S waits for it
            ok = mbar_wait(bar(R, kBarEmpty + s), (q / S) & 1u, R.abort_flag, p.status);
            if (!ok)
                break;
            *R.mma_done = q + 1;
            if (t + S - 1 < U.ntiles)
                ok = issue_x(t + S - 1);
        }
        if (!ok)
            break;
        umma_commit(bar(R, kBarAcc + d));
        q0 += U.ntiles;
    }
    // drain: copies issued but never waited for, and every MMA
    for (uint32_t q = x_used; q < x_issued; q++)
        mbar_wait(bar(R, kBarX + q % S), (q / S) & 1u, R.abort_flag, p.status, false);
    if (committed) {
        umma_commit(bar(R, kBarDrain));
        mbar_wait(bar(R, kBarDrain), 0u, R.abort_flag, p.status, false);
    }
}

// Merge and epilogue warp (four of them, warp mod 4 = quarter).  In tile
// order: wait until the tile's exponents are all in (its counter), and its
// operand slot free (the MMA of tile q - S complete, as the control thread
// publishes), merge this warp's quarter, arrive on the tile's full barrier
// and count the quarter merged (the exponent tile is free after all four).
// After a unit's tiles, the epilogue of the unit before: add the rows 32
// quarter .. 32 quarter + 31 of its accumulator (the tensor-memory lanes
// this warp may read) into Y; the last unit's epilogue at the end.
__device__ __forceinline__ void merge_epilogue_role(const GemmParams &p, const Roles &R, uint32_t warp, int lane)
{
    const uint32_t quarter = warp & 3u, N = p.batch, S = p.stages, E = p.etiles;
    auto epilogue = [&](uint32_t u, uint32_t k) -> bool {
        const uint32_t d = k & 1u;
        if (!__all_sync(0xffffffffu, mbar_wait(bar(R, kBarAcc + d), (k >> 1) & 1u, R.abort_flag, p.status)))
            return false;
        tc_fence_after();
        const Unit U = unit_of(p, u);
        const GemmMat &M = p.mats[U.m];
        const uint32_t row = U.row0 + 32 * quarter + (uint32_t)lane;
        const uint32_t taddr = R.tmem + ((32 * quarter) << 16) + d * N;
        for (uint32_t c0 = 0; c0 < N; c0 += 16) {
            uint32_t r[16];
            tmem_ld16(taddr + c0, r);
#pragma unroll
            for (uint32_t j = 0; j < 16; j++)
                atomicAdd(M.y + (uint64_t)(c0 + j) * M.rows + row, __uint_as_float(r[j]));
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0)
            mbar_arrive(bar(R, kBarFree + d));
        return true;
    };
    uint32_t q0 = 0, k = 0;
    uint4 s4[4];  // the next tile's sign/mantissa bytes, loaded before its exponents are all in
    for (uint32_t u = blockIdx.x; u < p.num_units; u += gridDim.x, k++) {
        const Unit U = unit_of(p, u);
        load_quarter(p, U.e0, quarter, lane, s4);
        for (uint32_t t = 0; t < U.ntiles; t++) {
            const uint32_t q = q0 + t;
            if (!__all_sync(0xffffffffu, count_wait(R.ecount + q % E, (q / E + 1) * kTileElems, R, p.status)))
                return;
            if (q >= S && !__all_sync(0xffffffffu, count_wait(R.mma_done, q - S + 1, R, p.status)))
                return;
            __threadfence_block();
            merge_quarter(p, R, q, quarter, lane, s4);
            if (t + 1 < U.ntiles)
                load_quarter(p, U.e0 + ((uint64_t)(t + 1) << kTileShift), quarter, lane, s4);
            fence_proxy_async();  // the operand tile is read by the tensor core (async proxy)
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(bar(R, kBarFull + q % S));
                __threadfence_block();
                atomicAdd(const_cast<uint32_t *>(R.emerged + q % E), 1u);
            }
        }
        q0 += U.ntiles;
        if (k >= 1 && !epilogue(u - gridDim.x, k - 1))
            return;
    }
    if (k >= 1)
        epilogue(blockIdx.x + (k - 1) * gridDim.x, k - 1);
}

template <int C, int DW, uint32_t SLOT>
__global__ void __launch_bounds__(gemm_threads(DW), 1) df11_gemm_kernel(const GemmParams p)
{
    extern __shared__ __align__(1024) uint8_t smem[];
    const uint32_t tid = threadIdx.x, warp = tid >> 5;
    const int lane = (int)(tid & 31u);
    const uint32_t S = p.stages;
    uint8_t *ctrl = smem + ctrl_offset(p.cap, DW, SLOT);
    Roles R;
    const uint32_t base = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
    R.bars = static_cast<uint32_t>(__cvta_generic_to_shared(ctrl));
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(ctrl + kNumBars * 8);
    R.abort_flag = tmem_slot + 1;
    R.mma_done = tmem_slot + 2;
    R.ecount = tmem_slot + 3;
    R.emerged = tmem_slot + 3 + kMaxETiles;
    R.ring_a = (base + ctrl_offset(p.cap, DW, SLOT) + kCtrlBytes + 1023u) & ~1023u;
    R.ring_b = R.ring_a + S * kTileBytes;
    R.ring_e = R.ring_b + S * p.batch * 128;

    if (tid == 0) {
        for (uint32_t s = 0; s < S; s++) {
            mbar_init(bar(R, kBarFull + s), 4);  // the four merge warps
            mbar_init(bar(R, kBarEmpty + s), 1);
            mbar_init(bar(R, kBarX + s), 1);
        }
        for (uint32_t d = 0; d < 2; d++) {
            mbar_init(bar(R, kBarAcc + d), 1);
            mbar_init(bar(R, kBarFree + d), 4);
        }
        mbar_init(bar(R, kBarDrain), 1);
        for (uint32_t i = 0; i < kMaxETiles; i++) {
            R.ecount[i] = 0u;
            R.emerged[i] = 0u;
        }
        *R.mma_done = 0u;
        *R.abort_flag = 0u;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        fence_proxy_async();
    }
    if (warp == DW) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         static_cast<uint32_t>(__cvta_generic_to_shared(tmem_slot))),
                     "r"(p.tmem_cols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
        tc_fence_before();
    }
    // the tables (the barriers, flags and tensor-memory address above are
    // published by its __syncthreads)
    const bool tables_ok = build_tables<false>(p.luts, p.cl, p.num_luts, p.sym_table, smem, tid, gemm_threads(DW),
                                        SLOT < kSlotLong ? 2u : 1u);
    tc_fence_after();
    R.tmem = *reinterpret_cast<volatile uint32_t *>(tmem_slot);
    // the prep kernel's packed activations and unit ranges are complete and
    // visible from here on (a launch without a programmatic dependency
    // passes at once)
    asm volatile("griddepcontrol.wait;" ::: "memory");

    // short staging slots hold a segment's codes only when no code is 1 bit
    // long (the all-zero code is the shortest): otherwise no role runs, the
    // stream is reported and the tensor memory is released below
    bool slots_ok = tables_ok;  // a stored table with an impossible entry: reported below
    if (!tables_ok && tid == 0)
        atomicOr(p.status, (uint32_t)DF11_ERR_CORRUPT);
    if (tables_ok && SLOT < kSlotLong) {
        bool bad = false;
        const uint32_t lmin = lut_decode(0u, smem + Smem::luts, smem + Smem::cl, p.num_luts, &bad) >> 8;
        slots_ok = !bad && lmin >= 2;
        if (!slots_ok && tid == 0)
            atomicOr(p.status, (uint32_t)DF11_ERR_CORRUPT);
    }
    if (!slots_ok) {
    } else if (warp < DW) {
        decode_role<C, DW, SLOT>(p, R, smem, warp, lane);
    } else if (warp == DW) {
        if (lane == 0)
            control_role(p, R);
        __syncwarp();
    } else {
        merge_epilogue_role(p, R, warp, lane);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == DW) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(R.tmem), "r"(p.tmem_cols)
                     : "memory");
    }
}

// SM count and opt-in shared memory per device, and the dynamic shared
// memory already granted to each kernel.
struct GemmFacts {
    int sms = 0;
    int smem_optin = 0;
    uint32_t granted[2][3][2] = {};  // [C - 1][16, 20 or 27 decode warps][short slots]
};
std::mutex g_gemm_mu;
GemmFacts g_gemm[64];

// Work units and packed-X bytes of a matrix list; false if it is invalid.
bool plan_units(const df11_gemm_matrix *mats, uint32_t num_mats, uint32_t batch, uint64_t *units, uint64_t *xbytes)
{
    if (!mats || num_mats < 1 || num_mats > kMaxGemmMats || batch < 16 || batch > 256 || batch % 16)
        return false;
    uint64_t nu = 0, xb = 0;
    for (uint32_t m = 0; m < num_mats; m++) {
        const df11_gemm_matrix &M = mats[m];
        if (M.rows == 0 || M.cols == 0 || M.rows % kTileRows || M.cols % kTileCols)
            return false;
        const uint64_t kchunks = M.cols / kTileCols;
        nu += (uint64_t)(M.rows / kTileRows) * ((kchunks + kUnitChunks - 1) / kUnitChunks);
        xb += (uint64_t)M.cols * batch * 2;
    }
    if (nu >= (1ull << 31))
        return false;
    *units = nu;
    *xbytes = xb;
    return true;
}

}  // namespace

extern "C" uint64_t df11_gemm_scratch_bytes(const df11_gemm_matrix *mats, uint32_t num_mats, uint32_t batch)
{
    uint64_t units = 0, xbytes = 0;
    if (!plan_units(mats, num_mats, batch, &units, &xbytes))
        return 0;
    return xbytes + 8 * units;
}

extern "C" df11_status df11_decompress_gemm(const df11_arrays *a, const df11_gemm_matrix *mats, uint32_t num_mats,
                                            uint32_t batch, void *scratch, uint64_t scratch_bytes,
                                            uint32_t *status_dev, void *stream)
{
    uint64_t units = 0, xbytes = 0;
    if (!a || !status_dev || !plan_units(mats, num_mats, batch, &units, &xbytes) || a->n == 0)
        return DF11_ERR_INVALID_ARG;
    if (!scratch || !aligned(scratch, 16) || scratch_bytes < xbytes + 8 * units)
        return DF11_ERR_INVALID_ARG;
    GemmParams prm;
    const df11_status st = stream_params(a, status_dev, prm);
    if (st != DF11_OK)
        return st;
    uint64_t off = 0, unit0 = 0, piece0 = 0, xoff = 0;
    for (uint32_t m = 0; m < num_mats; m++) {
        const df11_gemm_matrix &M = mats[m];
        if (!M.x || !M.y || !aligned(M.x, 16) || !aligned(M.y, 4))
            return DF11_ERR_INVALID_ARG;
        GemmMat &G = prm.mats[m];
        G.off = (uint32_t)off;
        G.rows = M.rows;
        G.cols = M.cols;
        G.unit0 = (uint32_t)unit0;
        G.units_per_rt = (M.cols / kTileCols + kUnitChunks - 1) / kUnitChunks;
        G.piece0 = (uint32_t)piece0;
        G.xoff = xoff;
        G.x = M.x;
        G.y = M.y;
        off += (uint64_t)M.rows * M.cols;
        if (off > a->n)
            return DF11_ERR_INVALID_ARG;
        unit0 += (uint64_t)(M.rows / kTileRows) * G.units_per_rt;
        piece0 += (uint64_t)M.cols / 8 * batch;
        xoff += (uint64_t)M.cols * batch * 2;
    }
    if (off != a->n || piece0 >= (1ull << 31))
        return DF11_ERR_INVALID_ARG;  // the matrices must cover the stream exactly
    prm.batch = batch;
    prm.num_mats = num_mats;
    prm.num_units = (uint32_t)units;
    prm.num_pieces = (uint32_t)piece0;
    prm.xpack = static_cast<uint8_t *>(scratch);
    prm.unit_blocks = reinterpret_cast<uint32_t *>(static_cast<uint8_t *>(scratch) + xbytes);
    uint32_t cols = 32;
    while (cols < 2 * batch)
        cols <<= 1;
    prm.tmem_cols = cols;

    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        return DF11_ERR_CUDA;
    GemmFacts *f = &g_gemm[dev];
    {
        std::lock_guard<std::mutex> lock(g_gemm_mu);
        if (!f->sms) {
            int sms = 0, optin = 0;
            if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
                cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
                return DF11_ERR_CUDA;
            f->smem_optin = optin;
            f->sms = sms;
        }
    }
    // two operand stages; as many exponent tiles as fit (up to 16) beside
    // the most decode warps that leave at least 4 of them (27 warps), else 3
    // (20 warps), else 2 (16 warps; a block covers at most two tiles); short
    // staging slots when the stream states that no code is 1 bit long
    const uint32_t optin = (uint32_t)f->smem_optin;
    const uint32_t slot = prm.min_code_len >= 2 ? kSlotShort : kSlotLong;
    auto max_etiles = [&](uint32_t dw) {
        uint32_t e = kMaxETiles;
        while (e >= 1 && gemm_smem_bytes(prm.cap, batch, kStages, e, dw, slot) > optin)
            e--;
        return e;
    };
    uint32_t dw = 27, etiles = max_etiles(27);
    if (etiles < 4) {
        dw = 20;
        etiles = max_etiles(20);
    }
    if (etiles < 3) {
        dw = 16;
        etiles = max_etiles(16);
    }
    if (etiles < 2)
        return DF11_ERR_INVALID_ARG;
    prm.stages = kStages;
    prm.etiles = etiles;
    const uint32_t smem = gemm_smem_bytes(prm.cap, batch, kStages, etiles, dw, slot);
    const int ci = a->threads_per_block == 32 ? 0 : 1, wi = dw == 27 ? 2 : (dw == 20 ? 1 : 0),
              si = slot == kSlotShort ? 1 : 0;
    using Kernel = void (*)(const GemmParams);
    static const Kernel kernels[2][3][2] = {
        {{df11_gemm_kernel<1, 16, kSlotLong>, df11_gemm_kernel<1, 16, kSlotShort>},
         {df11_gemm_kernel<1, 20, kSlotLong>, df11_gemm_kernel<1, 20, kSlotShort>},
         {df11_gemm_kernel<1, 27, kSlotLong>, df11_gemm_kernel<1, 27, kSlotShort>}},
        {{df11_gemm_kernel<2, 16, kSlotLong>, df11_gemm_kernel<2, 16, kSlotShort>},
         {df11_gemm_kernel<2, 20, kSlotLong>, df11_gemm_kernel<2, 20, kSlotShort>},
         {df11_gemm_kernel<2, 27, kSlotLong>, df11_gemm_kernel<2, 27, kSlotShort>}}};
    const Kernel kern = kernels[ci][wi][si];
    {
        std::lock_guard<std::mutex> lock(g_gemm_mu);
        if (smem > f->granted[ci][wi][si]) {
            if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
                return DF11_ERR_CUDA;
            f->granted[ci][wi][si] = smem;
        }
    }
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const uint64_t prep = prm.num_pieces > prm.num_units ? prm.num_pieces : prm.num_units;
    gemm_prep_kernel<<<(unsigned)((prep + 255) / 256), 256, 0, s>>>(prm);
    if (cudaGetLastError() != cudaSuccess)
        return DF11_ERR_CUDA;
    const uint32_t grid = (uint32_t)f->sms < prm.num_units ? (uint32_t)f->sms : prm.num_units;
    // programmatic dependent launch: the GEMM kernel's set-up (tensor memory,
    // barriers, tables) overlaps the prep kernel's tail
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(gemm_threads(dw));
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kern, prm) != cudaSuccess)
        return DF11_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? DF11_OK : DF11_ERR_CUDA;
}

extern "C" df11_status df11_tile_major(const uint16_t *src, uint32_t rows, uint32_t cols, uint16_t *dst)
{
    if (!src || !dst || rows % kTileRows || cols % kTileCols)
        return DF11_ERR_INVALID_ARG;
    uint64_t o = 0;
    for (uint32_t r0 = 0; r0 < rows; r0 += kTileRows)
        for (uint32_t c0 = 0; c0 < cols; c0 += kTileCols)
            for (uint32_t r = r0; r < r0 + kTileRows; r++) {
                std::memcpy(dst + o, src + (uint64_t)r * cols + c0, kTileCols * 2);
                o += kTileCols;
            }
    return DF11_OK;
}
