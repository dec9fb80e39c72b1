// df11_format.cpp -- host side of the DF11 library: builds the compressed
// stream that the GPU kernel decodes.
//
// Steps, in the order of "DFloat11: Kompresi inferensi GPU lossless ..."
// (id.news.hada.io/topic?id=20542):
//   1. split BF16 into exponent / sign+mantissa bytes   ("Ruang kompresi",
//      "Format DFloat11")
//   2. exponent histogram and Huffman code lengths      ("Format DFloat11"),
//      capped at 32 bits ("Kernel GPU 2 tahap": Gaps are 5 bits because the
//      longest code is 32) with package-merge when plain Huffman is deeper
//   3. canonical codes and the MSB-first EncodedExponent bit stream
//   4. Gaps (5 bits per 8-byte segment) and BlockOffset (one output position
//      per thread block)                                 ("Kernel GPU 2 tahap")
//   5. hierarchical 256-entry LUTs with pointer values 240..255 and the
//      CodeLengths table                                 ("Decoding berbasis
//      LUT hierarkis")
// The byte layout is specified in include/df11.h.  Steps 1, 3 and 4 run in
// parallel over element chunks; everything is exact integer work.
#include "df11.h"
#include "df11_symtab.h"

#include <algorithm>
#include <array>
#include <atomic>
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <map>
#include <new>
#include <queue>
#include <thread>
#include <vector>

namespace {

constexpr int kSymbols = 256;
constexpr int kFirstPointer = 240;
constexpr uint64_t kChunk = 1ull << 22;  // elements per host work item

template <class F>
void parallel_for(uint64_t count, F &&fn)
{
    unsigned hw = std::thread::hardware_concurrency();
    unsigned nt = (unsigned)std::min<uint64_t>(count, hw ? hw : 1);
    if (nt <= 1) {
        for (uint64_t i = 0; i < count; i++)
            fn(i);
        return;
    }
    std::atomic<uint64_t> next{0};
    std::vector<std::thread> pool;
    pool.reserve(nt);
    for (unsigned t = 0; t < nt; t++)
        pool.emplace_back([&] {
            for (uint64_t i = next.fetch_add(1); i < count; i = next.fetch_add(1))
                fn(i);
        });
    for (auto &th : pool)
        th.join();
}

// ---------------------------------------------------------------- lengths
// Huffman with the format's tie-break: the two live nodes with the smallest
// (weight, smallest symbol in subtree) are merged first.
int huffman_lengths(const uint64_t *hist, uint8_t *len)
{
    struct Node {
        uint64_t w;
        int minsym;
        int id;
    };
    auto later = [](const Node &a, const Node &b) {
        return a.w != b.w ? a.w > b.w : a.minsym > b.minsym;
    };
    std::priority_queue<Node, std::vector<Node>, decltype(later)> pq(later);
    std::vector<int> parent;
    int leaf_id[kSymbols];
    int k = 0;
    for (int s = 0; s < kSymbols; s++) {
        len[s] = 0;
        leaf_id[s] = -1;
        if (hist[s]) {
            leaf_id[s] = (int)parent.size();
            parent.push_back(-1);
            pq.push({hist[s], s, leaf_id[s]});
            k++;
        }
    }
    if (k == 0)
        return 0;
    if (k == 1) {
        for (int s = 0; s < kSymbols; s++)
            if (leaf_id[s] >= 0)
                len[s] = 1;
        return 1;
    }
    while (pq.size() > 1) {
        Node a = pq.top();
        pq.pop();
        Node b = pq.top();
        pq.pop();
        int id = (int)parent.size();
        parent.push_back(-1);
        parent[a.id] = id;
        parent[b.id] = id;
        pq.push({a.w + b.w, std::min(a.minsym, b.minsym), id});
    }
    // depth = distance to the root; parents always have larger ids
    std::vector<int> depth(parent.size(), 0);
    for (int v = (int)parent.size() - 2; v >= 0; v--)
        depth[v] = depth[parent[v]] + 1;
    int longest = 0;
    for (int s = 0; s < kSymbols; s++)
        if (leaf_id[s] >= 0) {
            len[s] = (uint8_t)depth[leaf_id[s]];
            longest = std::max(longest, (int)len[s]);
        }
    return longest;
}

// Package-merge (Larmore & Hirschberg 1990), optimal lengths <= cap.  Items
// of a level are leaves or pairs of items of the level below; at equal
// weight leaves precede pairs (the format's tie rule).  The first 2(k-1)
// items of the top level are expanded and every leaf met adds one to its
// symbol's length.
bool package_merge(const uint64_t *hist, int cap, uint8_t *len)
{
    std::vector<int> syms;
    for (int s = 0; s < kSymbols; s++) {
        len[s] = 0;
        if (hist[s])
            syms.push_back(s);
    }
    int k = (int)syms.size();
    if (k == 0)
        return true;
    if (k == 1) {
        len[syms[0]] = 1;
        return true;
    }
    if (cap < 31 && (1 << cap) < k)
        return false;
    std::stable_sort(syms.begin(), syms.end(), [&](int a, int b) {
        return hist[a] != hist[b] ? hist[a] < hist[b] : a < b;
    });
    struct Item {
        uint64_t w;
        int sym;         // >= 0: a leaf
        int left, right; // pair: indices into the level below
    };
    std::vector<std::vector<Item>> level(cap);  // level[0] = deepest (2^-cap)
    for (int s : syms)
        level[0].push_back({hist[s], s, -1, -1});
    for (int d = 1; d < cap; d++) {
        const auto &prev = level[d - 1];
        std::vector<Item> pairs;
        for (size_t i = 0; i + 1 < prev.size(); i += 2)
            pairs.push_back({prev[i].w + prev[i + 1].w, -1, (int)i, (int)i + 1});
        auto &cur = level[d];
        size_t i = 0, j = 0;
        while (i < syms.size() || j < pairs.size()) {
            if (j >= pairs.size() || (i < syms.size() && hist[syms[i]] <= pairs[j].w)) {
                cur.push_back({hist[syms[i]], syms[i], -1, -1});
                i++;
            } else {
                cur.push_back(pairs[j++]);
            }
        }
    }
    // expand the selection level by level: `take` marks items to count
    std::vector<char> take(level[cap - 1].size(), 0);
    for (int i = 0; i < 2 * (k - 1); i++)
        take[i] = 1;
    for (int d = cap - 1; d >= 0; d--) {
        std::vector<char> below(d > 0 ? level[d - 1].size() : 0, 0);
        for (size_t i = 0; i < level[d].size(); i++) {
            if (!take[i])
                continue;
            const Item &it = level[d][i];
            if (it.sym >= 0)
                len[it.sym]++;
            else {
                below[it.left] = 1;
                below[it.right] = 1;
            }
        }
        take.swap(below);
    }
    return true;
}

// RFC 1951 section 3.2.2 construction: count codes per length, first code
// of each length, then hand out consecutive values in symbol order.
void canonical_codes(const uint8_t *len, uint32_t *code)
{
    uint32_t bl_count[DF11_MAX_CODE_LEN + 2] = {0};
    for (int s = 0; s < kSymbols; s++)
        if (len[s])
            bl_count[len[s]]++;
    uint64_t next[DF11_MAX_CODE_LEN + 2] = {0};
    uint64_t c = 0;
    for (int l = 1; l <= DF11_MAX_CODE_LEN; l++) {
        c = (c + bl_count[l - 1]) << 1;
        next[l] = c;
    }
    for (int s = 0; s < kSymbols; s++) {
        code[s] = 0;
        if (len[s])
            code[s] = (uint32_t)next[len[s]]++;
    }
}

// Length of the shortest code (0 when no symbol has a code).
uint32_t shortest_code(const uint8_t *len)
{
    uint32_t m = 0;
    for (int s = 0; s < kSymbols; s++)
        if (len[s] && (m == 0 || len[s] < m))
            m = len[s];
    return m;
}

// ------------------------------------------------------------------- LUTs
// Height-8 subtrees as 256-entry tables, built from the code values: a code
// of length l with 8m < l <= 8(m+1) fills 2^(8(m+1)-l) entries of the table
// of its 8m-bit prefix; a longer code puts a pointer to the table of its
// 8(m+1)-bit prefix.  Tables are numbered level by level, prefix ascending.
df11_status build_luts(const uint8_t *len, const uint32_t *code, std::vector<uint8_t> &luts,
                       uint32_t *num_luts)
{
    int longest = 0, nsym = 0, only = 0;
    for (int s = 0; s < kSymbols; s++)
        if (len[s]) {
            longest = std::max(longest, (int)len[s]);
            nsym++;
            only = s;
        }
    // table ids: key = (level, prefix value)
    std::vector<std::map<uint32_t, int>> ids((longest + 7) / 8 + 1);
    ids[0][0] = 0;
    int count = 1;
    for (int m = 1; 8 * m < longest; m++) {
        for (int s = 0; s < kSymbols; s++)
            if (len[s] > 8 * m)
                ids[m].emplace(code[s] >> (len[s] - 8 * m), 0);
        for (auto &kv : ids[m])
            kv.second = count++;
    }
    if (count > DF11_MAX_LUTS)
        return DF11_ERR_TOO_MANY_LUTS;
    luts.assign((size_t)count * 256, nsym == 1 ? (uint8_t)only : 0);
    for (int s = 0; s < kSymbols; s++) {
        int l = len[s];
        if (!l)
            continue;
        for (int m = 0; 8 * m < l; m++) {
            uint32_t prefix = m ? code[s] >> (l - 8 * m) : 0;
            int table = ids[m].at(prefix);
            if (l <= 8 * (m + 1)) {
                uint32_t low = code[s] & ((1u << (l - 8 * m)) - 1);  // bits after the prefix
                uint32_t first = low << (8 * (m + 1) - l);
                uint32_t span = 1u << (8 * (m + 1) - l);
                std::memset(&luts[(size_t)table * 256 + first], s, span);
            } else {
                uint32_t idx = (code[s] >> (l - 8 * (m + 1))) & 0xFF;
                uint32_t child_prefix = code[s] >> (l - 8 * (m + 1));
                int child = ids[m + 1].at(child_prefix);
                luts[(size_t)table * 256 + idx] = (uint8_t)(256 - child);
            }
        }
    }
    *num_luts = (uint32_t)count;
    return DF11_OK;
}

// The decoders' derived 12-bit table (df11_symtab.h) from a code's LUTs and
// CodeLengths: the same functions the kernels run when a stream has none.
void derive_symbol_table(const uint8_t *luts, const uint8_t *cl, uint32_t num_luts, uint32_t *out)
{
    std::vector<uint16_t> fc(df11_symtab::kIdxEntries);
    for (uint32_t i = 0; i < (uint32_t)df11_symtab::kIdxEntries; i++)
        fc[i] = df11_symtab::first_code(i, luts, cl, num_luts);
    for (uint32_t i = 0; i < (uint32_t)df11_symtab::kIdxEntries; i++)
        out[i] = df11_symtab::table_entry(i, fc.data());
}

}  // namespace

extern "C" df11_status df11_symbol_table(const uint8_t *luts, const uint8_t *code_lengths, uint32_t num_luts,
                                         uint32_t *out)
{
    if (!luts || !code_lengths || !out || num_luts < 1 || num_luts > DF11_MAX_LUTS)
        return DF11_ERR_INVALID_ARG;
    derive_symbol_table(luts, code_lengths, num_luts, out);
    return DF11_OK;
}

// ------------------------------------------------------------------ handle
struct df11_format {
    df11_arrays a;  // host pointers into the vectors below
    std::vector<uint8_t> stream, sm, luts;
    std::vector<uint64_t> gaps;
    std::vector<uint32_t> offsets;
    std::vector<uint32_t> symbol_table;  // the decoders' derived table (df11_symtab.h)
    uint8_t code_lengths[kSymbols];
    uint32_t codes[kSymbols];
    uint64_t hist[kSymbols];
    bool plan_only = false;  // made by df11_plan_from_histogram: no host arrays
};

extern "C" df11_status df11_build_format(const uint16_t *const *mats, const uint64_t *counts,
                                         int num_mats, uint32_t T, df11_format **out)
{
    if (!out)
        return DF11_ERR_INVALID_ARG;
    *out = nullptr;
    if (num_mats < 0 || (num_mats > 0 && (!mats || !counts)))
        return DF11_ERR_INVALID_ARG;
    if (T == 0)
        T = DF11_DEFAULT_THREADS;
    if (T < 32 || T > 1024 || T % 32)
        return DF11_ERR_INVALID_ARG;
    uint64_t n = 0;
    std::vector<uint64_t> first(num_mats + 1, 0);
    for (int i = 0; i < num_mats; i++) {
        if (counts[i] && !mats[i])
            return DF11_ERR_INVALID_ARG;
        first[i] = n;
        n += counts[i];
        if (n >= (1ull << 32))
            return DF11_ERR_TOO_LARGE;
    }
    first[num_mats] = n;

    df11_format *f = new (std::nothrow) df11_format();
    if (!f)
        return DF11_ERR_NO_MEMORY;
    try {
        // ---- 1. split + histogram (parallel over chunks of each matrix)
        std::vector<uint8_t> exps(n);
        f->sm.assign(((n + 15) / 16) * 16 + 16, 0);
        struct Work {
            int mat;
            uint64_t lo, hi;
        };
        std::vector<Work> work;
        for (int i = 0; i < num_mats; i++)
            for (uint64_t lo = 0; lo < counts[i]; lo += kChunk)
                work.push_back({i, lo, std::min(counts[i], lo + kChunk)});
        std::vector<std::array<uint64_t, kSymbols>> part(work.size());
        std::atomic<bool> bad{false};
        parallel_for(work.size(), [&](uint64_t wi) {
            const Work &wk = work[wi];
            auto &h = part[wi];
            h.fill(0);
            const uint16_t *src = mats[wk.mat];
            uint64_t base = first[wk.mat];
            for (uint64_t i = wk.lo; i < wk.hi; i++) {
                uint16_t v = src[i];
                uint8_t e = (uint8_t)(v >> 7);
                exps[base + i] = e;
                f->sm[base + i] = (uint8_t)(((v >> 8) & 0x80) | (v & 0x7F));
                h[e]++;
            }
        });
        std::memset(f->hist, 0, sizeof(f->hist));
        for (auto &h : part)
            for (int s = 0; s < kSymbols; s++)
                f->hist[s] += h[s];
        for (int s = kFirstPointer; s < kSymbols; s++)
            if (f->hist[s])
                bad = true;
        if (bad) {
            delete f;
            return DF11_ERR_UNSUPPORTED_EXPONENT;
        }

        // ---- 2. code lengths, 3a. canonical codes
        int longest = huffman_lengths(f->hist, f->code_lengths);
        if (longest > DF11_MAX_CODE_LEN) {
            if (!package_merge(f->hist, DF11_MAX_CODE_LEN, f->code_lengths)) {
                delete f;
                return DF11_ERR_INVALID_ARG;
            }
            longest = 0;
            for (int s = 0; s < kSymbols; s++)
                longest = std::max(longest, (int)f->code_lengths[s]);
        }
        canonical_codes(f->code_lengths, f->codes);

        // ---- 3b. bit lengths per chunk, prefix sums
        uint64_t nchunks = (n + kChunk - 1) / kChunk;
        std::vector<uint64_t> chunk_bits(nchunks + 1, 0);
        parallel_for(nchunks, [&](uint64_t c) {
            uint64_t lo = c * kChunk, hi = std::min(n, lo + kChunk);
            uint64_t bits = 0;
            for (uint64_t i = lo; i < hi; i++)
                bits += f->code_lengths[exps[i]];
            chunk_bits[c + 1] = bits;
        });
        for (uint64_t c = 0; c < nchunks; c++)
            chunk_bits[c + 1] += chunk_bits[c];
        uint64_t total_bits = chunk_bits[nchunks];
        uint64_t nseg = (total_bits + 63) / 64;
        uint64_t nblocks = (nseg + T - 1) / T;
        if (nblocks >= (1ull << 31)) {
            delete f;
            return DF11_ERR_TOO_LARGE;
        }
        f->stream.assign(nblocks * T * 8 + 16, 0);
        std::vector<uint8_t> gap8(nblocks * T, 0);
        f->offsets.assign(nblocks + 1, 0);

        // ---- 3c + 4. encode chunks; each code start fills the gaps of the
        // segment boundaries in (previous start, this start]
        std::vector<uint8_t> head(nchunks, 0), tail(nchunks, 0);
        parallel_for(nchunks, [&](uint64_t c) {
            uint64_t lo = c * kChunk, hi = std::min(n, lo + kChunk);
            uint64_t pos = chunk_bits[c];
            uint64_t prev = lo ? pos - f->code_lengths[exps[lo - 1]] : 0;
            bool have_prev = lo != 0;
            uint64_t acc = 0;   // pending bits, left aligned in the low `nacc` bits
            int nacc = (int)(pos & 7);
            uint64_t byte = pos >> 3;
            bool first_out = true;
            for (uint64_t i = lo; i < hi; i++) {
                // metadata for this start
                uint64_t s_lo = have_prev ? prev / 64 + 1 : 0;
                uint64_t s_hi = pos / 64;
                for (uint64_t s = s_lo; s <= s_hi && s < nseg; s++) {
                    gap8[s] = (uint8_t)(pos - 64 * s);
                    if (s % T == 0)
                        f->offsets[s / T] = (uint32_t)i;
                }
                int l = f->code_lengths[exps[i]];
                acc = (acc << l) | f->codes[exps[i]];
                nacc += l;
                while (nacc >= 8) {
                    uint8_t v = (uint8_t)(acc >> (nacc - 8));
                    if (first_out)
                        head[c] = v;  // byte shared with the previous chunk
                    else
                        f->stream[byte] = v;
                    first_out = false;
                    byte++;
                    nacc -= 8;
                }
                acc &= (nacc ? ((1ull << nacc) - 1) : 0);
                prev = pos;
                have_prev = true;
                pos += l;
            }
            tail[c] = nacc ? (uint8_t)(acc << (8 - nacc)) : 0;  // partial last byte
        });
        // boundary bytes: OR in chunk order
        for (uint64_t c = 0; c < nchunks; c++) {
            uint64_t s = chunk_bits[c], e = chunk_bits[c + 1];
            // head[c] is the first whole byte the chunk completed (if any)
            bool completed_any = ((s & 7) + (e - s)) >= 8;
            if (completed_any)
                f->stream[s >> 3] |= head[c];
            if (e & 7)
                f->stream[e >> 3] |= tail[c];
        }
        // segments after the last code start
        uint64_t last_start = n ? total_bits - f->code_lengths[exps[n - 1]] : 0;
        for (uint64_t s = n ? last_start / 64 + 1 : 0; s < nseg; s++) {
            gap8[s] = (uint8_t)(total_bits - 64 * s);
            if (s % T == 0)
                f->offsets[s / T] = (uint32_t)n;
        }
        f->offsets[nblocks] = (uint32_t)n;

        // ---- 4b. pack gaps: word w holds fields overlapping bits [64w, 64w+64)
        uint64_t nwords = (5 * nblocks * T + 63) / 64 + 2;
        f->gaps.assign(nwords, 0);
        parallel_for((nwords + 4095) / 4096, [&](uint64_t blk) {
            for (uint64_t w = blk * 4096; w < std::min(nwords, (blk + 1) * 4096); w++) {
                uint64_t word = 0;
                uint64_t s0 = (64 * w) / 5, s1 = (64 * w + 63) / 5;
                for (uint64_t s = s0; s <= s1 && s < gap8.size(); s++) {
                    int64_t shift = (int64_t)(5 * s) - (int64_t)(64 * w);
                    uint64_t g = gap8[s] & 31u;
                    word |= shift >= 0 ? (g << shift) : (g >> -shift);
                }
                f->gaps[w] = word;
            }
        });

        // ---- 5. LUTs
        df11_status st = build_luts(f->code_lengths, f->codes, f->luts, &f->a.num_luts);
        if (st != DF11_OK) {
            delete f;
            return st;
        }

        uint32_t max_block = 0;
        for (uint64_t b = 0; b < nblocks; b++)
            max_block = std::max(max_block, f->offsets[b + 1] - f->offsets[b]);

        df11_arrays &a = f->a;
        a.n = n;
        a.total_bits = total_bits;
        a.num_segments = nseg;
        a.threads_per_block = T;
        a.num_blocks = (uint32_t)nblocks;
        a.max_code_len = (uint32_t)longest;
        a.max_block_elems = max_block;
        a.min_code_len = shortest_code(f->code_lengths);
        a.encoded_exponent = f->stream.data();
        a.encoded_exponent_bytes = f->stream.size();
        a.packed_sign_mantissa = f->sm.data();
        a.packed_sign_mantissa_bytes = f->sm.size();
        a.gaps = f->gaps.data();
        a.gaps_words = f->gaps.size();
        a.block_offset = f->offsets.data();
        a.luts = f->luts.data();
        a.code_lengths = f->code_lengths;
        f->symbol_table.assign(df11_symtab::kIdxEntries, 0);
        derive_symbol_table(f->luts.data(), f->code_lengths, a.num_luts, f->symbol_table.data());
        a.symbol_table = f->symbol_table.data();
    } catch (const std::bad_alloc &) {
        delete f;
        return DF11_ERR_NO_MEMORY;
    }
    *out = f;
    return DF11_OK;
}

// A code without its arrays: the output of df11_plan_from_histogram.  Same
// steps 2, 3a and 5 as df11_build_format, from a histogram instead of the
// elements; the array sizes follow from sum(hist * length).
extern "C" df11_status df11_plan_from_histogram(const uint64_t *hist, uint32_t T, df11_format **out)
{
    if (!out || !hist)
        return DF11_ERR_INVALID_ARG;
    *out = nullptr;
    if (T == 0)
        T = DF11_DEFAULT_THREADS;
    if (T < 32 || T > 1024 || T % 32)
        return DF11_ERR_INVALID_ARG;
    uint64_t n = 0;
    for (int s = 0; s < kSymbols; s++) {
        if (hist[s] && s >= kFirstPointer)
            return DF11_ERR_UNSUPPORTED_EXPONENT;
        n += hist[s];
        if (n >= (1ull << 32))
            return DF11_ERR_TOO_LARGE;
    }
    df11_format *f = new (std::nothrow) df11_format();
    if (!f)
        return DF11_ERR_NO_MEMORY;
    try {
        std::memcpy(f->hist, hist, sizeof(f->hist));
        int longest = huffman_lengths(f->hist, f->code_lengths);
        if (longest > DF11_MAX_CODE_LEN) {
            if (!package_merge(f->hist, DF11_MAX_CODE_LEN, f->code_lengths)) {
                delete f;
                return DF11_ERR_INVALID_ARG;
            }
            longest = 0;
            for (int s = 0; s < kSymbols; s++)
                longest = std::max(longest, (int)f->code_lengths[s]);
        }
        canonical_codes(f->code_lengths, f->codes);
        uint64_t total_bits = 0;
        for (int s = 0; s < kSymbols; s++)
            total_bits += f->hist[s] * f->code_lengths[s];
        const uint64_t nseg = (total_bits + 63) / 64;
        const uint64_t nblocks = (nseg + T - 1) / T;
        if (nblocks >= (1ull << 31)) {
            delete f;
            return DF11_ERR_TOO_LARGE;
        }
        df11_status st = build_luts(f->code_lengths, f->codes, f->luts, &f->a.num_luts);
        if (st != DF11_OK) {
            delete f;
            return st;
        }
        df11_arrays &a = f->a;
        a.n = n;
        a.total_bits = total_bits;
        a.num_segments = nseg;
        a.threads_per_block = T;
        a.num_blocks = (uint32_t)nblocks;
        a.max_code_len = (uint32_t)longest;
        a.max_block_elems = 0;  // known once the elements are encoded
        a.min_code_len = shortest_code(f->code_lengths);
        a.encoded_exponent = nullptr;
        a.encoded_exponent_bytes = nblocks * T * 8 + 16;
        a.packed_sign_mantissa = nullptr;
        a.packed_sign_mantissa_bytes = ((n + 15) / 16) * 16 + 16;
        a.gaps = nullptr;
        a.gaps_words = (5 * nblocks * T + 63) / 64 + 2;
        a.block_offset = nullptr;
        a.luts = f->luts.data();
        a.code_lengths = f->code_lengths;
        f->symbol_table.assign(df11_symtab::kIdxEntries, 0);
        derive_symbol_table(f->luts.data(), f->code_lengths, a.num_luts, f->symbol_table.data());
        a.symbol_table = f->symbol_table.data();
        f->plan_only = true;
    } catch (const std::bad_alloc &) {
        delete f;
        return DF11_ERR_NO_MEMORY;
    }
    *out = f;
    return DF11_OK;
}

// Read by the device encoder (df11_encode.cu): a plan's canonical codes.
// Library-internal: not exported.
__attribute__((visibility("hidden"))) df11_status df11_internal_plan_codes(const df11_format *f,
                                                                           uint32_t *codes256)
{
    if (!f || !codes256)
        return DF11_ERR_INVALID_ARG;
    std::memcpy(codes256, f->codes, sizeof(f->codes));
    return DF11_OK;
}

extern "C" df11_status df11_format_arrays(const df11_format *f, df11_arrays *out)
{
    if (!f || !out)
        return DF11_ERR_INVALID_ARG;
    *out = f->a;
    return DF11_OK;
}

extern "C" df11_status df11_format_info(const df11_format *f, df11_info *out)
{
    if (!f || !out)
        return DF11_ERR_INVALID_ARG;
    std::memset(out, 0, sizeof(*out));
    const df11_arrays &a = f->a;
    out->n = a.n;
    out->total_bits = a.total_bits;
    out->compressed_bytes = (a.total_bits + 7) / 8 + a.n + (5 * a.num_segments + 7) / 8 +
                            4ull * (a.num_blocks + 1) + 256ull * a.num_luts + 256;
    double h = 0;
    uint32_t distinct = 0;
    for (int s = 0; s < kSymbols; s++) {
        out->histogram[s] = f->hist[s];
        if (f->hist[s]) {
            distinct++;
            double p = (double)f->hist[s] / (double)a.n;
            h -= p * std::log2(p);
        }
    }
    out->entropy_bits = h;
    out->avg_code_len = a.n ? (double)a.total_bits / (double)a.n : 0.0;
    out->distinct_exponents = distinct;
    out->max_code_len = a.max_code_len;
    out->num_luts = a.num_luts;
    out->threads_per_block = a.threads_per_block;
    return DF11_OK;
}

extern "C" void df11_free(df11_format *f)
{
    delete f;
}

extern "C" const char *df11_strerror(df11_status s)
{
    switch (s) {
    case DF11_OK: return "ok";
    case DF11_ERR_INVALID_ARG: return "invalid argument";
    case DF11_ERR_UNSUPPORTED_EXPONENT: return "exponent 240..255 (reserved for LUT pointers)";
    case DF11_ERR_TOO_LARGE: return "stream has 2^32 or more elements";
    case DF11_ERR_TOO_MANY_LUTS: return "code needs more than 16 child LUTs";
    case DF11_ERR_CUDA: return "CUDA runtime error";
    case DF11_ERR_CORRUPT: return "inconsistent compressed data";
    case DF11_ERR_NO_MEMORY: return "out of host memory";
    }
    return "unknown status";
}
