// df11_rans_format.cpp -- host side of the rANS variant of the exponent coder.
//
// The DFloat11 page's discussion proposes rANS (range asymmetric numeral
// systems) instead of Huffman coding for the exponents, as the coder that
// suits SIMD-style hardware; the pages fix none of its parameters.  The model
// and layout are stated in include/df11.h (df11_rans_arrays): frequencies
// quantised to 2^12, one 32-bit state per lane in [2^16, 2^32), 16-bit
// renormalisation words, blocks of 512 * chunks elements decoded by 32 lanes
// in step.  Sign and mantissa stay verbatim, as in DF11 ("Format DFloat11").
//
// Encoding runs each block's steps backwards (step descending) from x = 2^16
// in every lane; the final states are the decoder's start states and each
// lane's words, reversed, its stream in the order the decoder takes them.
// A block's words are lane 0's stream, then lane 1's, ...  Blocks are
// independent and encoded in parallel.
#include "df11.h"

#include <algorithm>
#include <atomic>
#include <cstring>
#include <new>
#include <thread>
#include <vector>

struct df11_rans_format {
    df11_rans_arrays a;
    std::vector<uint16_t> words;
    std::vector<uint32_t> states, block_word;
    std::vector<uint8_t> lane_words;
    std::vector<uint16_t> freq;
    std::vector<uint8_t> sm;
};

namespace {

constexpr uint32_t kProbBits = 12;
constexpr uint64_t kLow = 1ull << 16;  // lower bound of the state

template <class F>
void for_each_index(uint64_t count, F &&fn)
{
    const unsigned hw = std::max(1u, std::thread::hardware_concurrency());
    const unsigned nt = (unsigned)std::min<uint64_t>(count, hw);
    if (nt <= 1) {
        for (uint64_t i = 0; i < count; i++)
            fn(i);
        return;
    }
    std::atomic<uint64_t> next{0};
    std::vector<std::thread> pool;
    for (unsigned t = 0; t < nt; t++)
        pool.emplace_back([&] {
            for (uint64_t i; (i = next.fetch_add(1)) < count;)
                fn(i);
        });
    for (auto &th : pool)
        th.join();
}

// Quantised frequencies (rule in df11.h).  The shortfall always goes to the
// same exponent (the one with the largest count), so it is added at once.
bool quantise(const uint64_t *hist, uint16_t *freq)
{
    const uint64_t M = 1ull << kProbBits;
    uint64_t n = 0;
    for (int s = 0; s < 256; s++)
        n += hist[s];
    if (n == 0)
        return false;
    uint64_t total = 0;
    int top = -1;  // largest count, smallest exponent on ties
    for (int s = 0; s < 256; s++) {
        const uint64_t f = hist[s] ? std::max<uint64_t>(1, hist[s] * M / n) : 0;
        freq[s] = (uint16_t)f;
        total += f;
        if (hist[s] && (top < 0 || hist[s] > hist[top]))
            top = s;
    }
    while (total > M) {  // the largest frequency (smallest exponent on ties) gives one up
        int big = 0;
        for (int s = 1; s < 256; s++)
            if (freq[s] > freq[big])
                big = s;
        freq[big]--;
        total--;
    }
    freq[top] = (uint16_t)(freq[top] + (M - total));
    return true;
}

}  // namespace

extern "C" df11_status df11_rans_build(const uint16_t *const *mats, const uint64_t *counts, int num_mats,
                                       uint32_t chunks, df11_rans_format **out)
{
    if (!out)
        return DF11_ERR_INVALID_ARG;
    *out = nullptr;
    if (num_mats < 0 || (num_mats > 0 && (!mats || !counts)))
        return DF11_ERR_INVALID_ARG;
    if (chunks == 0)
        chunks = 10;
    if (chunks > 15)  // a lane's words per block (at most one per step) are counted in a byte
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
    df11_rans_format *f = new (std::nothrow) df11_rans_format();
    if (!f)
        return DF11_ERR_NO_MEMORY;
    try {
        // fields: exponent = bits 7..14, sign/mantissa byte = sign << 7 | mantissa
        std::vector<uint8_t> exps(n);
        f->sm.assign(((n + 15) / 16) * 16 + 16, 0);
        for (int m = 0; m < num_mats; m++) {
            const uint16_t *src = mats[m];
            const uint64_t base = first[m], cnt = counts[m];
            for_each_index((cnt + (1u << 20) - 1) >> 20, [&](uint64_t c) {
                const uint64_t lo = c << 20, hi = std::min<uint64_t>(cnt, lo + (1u << 20));
                for (uint64_t i = lo; i < hi; i++) {
                    const uint16_t w = src[i];
                    exps[base + i] = (uint8_t)(w >> 7);
                    f->sm[base + i] = (uint8_t)(((w >> 8) & 0x80) | (w & 0x7F));
                }
            });
        }
        uint64_t hist[256] = {0};
        for (uint64_t i = 0; i < n; i++)
            hist[exps[i]]++;
        f->freq.assign(256, 0);
        if (n)
            quantise(hist, f->freq.data());
        uint32_t cum[257] = {0};
        for (int s = 0; s < 256; s++)
            cum[s + 1] = cum[s] + f->freq[s];

        const uint64_t B = 512ull * chunks;
        const uint64_t nblocks = (n + B - 1) / B;
        if (nblocks >= (1ull << 32))
            throw std::bad_alloc();
        std::vector<std::vector<uint16_t>> blk(nblocks);
        f->states.assign(32 * nblocks, 0);
        f->lane_words.assign(32 * nblocks, 0);
        for_each_index(nblocks, [&](uint64_t b) {
            uint64_t x[32];
            std::fill(x, x + 32, kLow);
            std::vector<uint16_t> lane[32];
            const uint64_t b0 = b * B;
            for (int t = (int)(16 * chunks) - 1; t >= 0; t--) {
                const uint64_t row = b0 + 512ull * (uint64_t)(t >> 4) + (uint64_t)(t & 15);
                for (int l = 0; l < 32; l++) {
                    const uint64_t pos = row + 16ull * (uint64_t)l;
                    if (pos >= n)
                        continue;
                    const uint32_t s = exps[pos];
                    const uint64_t fs = f->freq[s];
                    if (x[l] >= (fs << (32 - kProbBits))) {
                        lane[l].push_back((uint16_t)x[l]);
                        x[l] >>= 16;
                    }
                    const uint64_t q = x[l] / fs;
                    x[l] = (q << kProbBits) + (x[l] - q * fs) + cum[s];
                }
            }
            std::vector<uint16_t> &st = blk[b];
            for (int l = 0; l < 32; l++) {
                st.insert(st.end(), lane[l].rbegin(), lane[l].rend());
                f->lane_words[32 * b + l] = (uint8_t)lane[l].size();
                f->states[32 * b + l] = (uint32_t)x[l];
            }
        });
        f->block_word.assign(nblocks + 1, 0);
        uint64_t total = 0;
        uint32_t most = 0;
        for (uint64_t b = 0; b < nblocks; b++) {
            f->block_word[b] = (uint32_t)total;
            total += blk[b].size();
            most = std::max<uint32_t>(most, (uint32_t)blk[b].size());
        }
        f->block_word[nblocks] = (uint32_t)total;
        f->words.assign(total + 8, 0);
        for_each_index(nblocks, [&](uint64_t b) {
            std::copy(blk[b].begin(), blk[b].end(), f->words.begin() + f->block_word[b]);
        });

        df11_rans_arrays &a = f->a;
        std::memset(&a, 0, sizeof(a));
        a.n = n;
        a.num_words = total;
        a.prob_bits = kProbBits;
        a.chunks = chunks;
        a.num_blocks = (uint32_t)nblocks;
        a.max_block_words = most;
        a.words = f->words.data();
        a.states = f->states.data();
        a.block_word = f->block_word.data();
        a.lane_words = f->lane_words.data();
        a.freq = f->freq.data();
        a.packed_sign_mantissa = f->sm.data();
        a.packed_sign_mantissa_bytes = f->sm.size();
    } catch (const std::bad_alloc &) {
        delete f;
        return DF11_ERR_NO_MEMORY;
    }
    *out = f;
    return DF11_OK;
}

extern "C" df11_status df11_rans_format_arrays(const df11_rans_format *f, df11_rans_arrays *out)
{
    if (!f || !out)
        return DF11_ERR_INVALID_ARG;
    *out = f->a;
    return DF11_OK;
}

extern "C" void df11_rans_free(df11_rans_format *f) { delete f; }
