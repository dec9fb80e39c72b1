/*
 * df11_oracle.c -- plain, slow CPU oracle for DFloat11 (DF11) compression.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call this file:
 * only the test suite, the package's smoke check and the benchmark's CPU
 * baseline leg load it.  It shares no code, header, table or constant with
 * the CUDA library; both sides read the same seeded inputs and nothing else.
 *
 * Source: "DFloat11: Kompresi inferensi GPU lossless yang mengecilkan LLM
 * menjadi 70% ukurannya" (id.news.hada.io/topic?id=20542), sections
 *   "Ruang kompresi yang tersisa pada exponent BFloat16"  (BF16 fields),
 *   "Format DFloat11"                                     (Huffman on the
 *        exponent, EncodedExponent, PackedSignMantissa),
 *   "Dekompresi yang disesuaikan untuk inferensi GPU"     (the sequential,
 *        bit-by-bit tree walk that the GPU kernel replaces -- this oracle uses
 *        exactly that walk because it is the obviously correct decoder),
 *   "Decoding berbasis LUT hierarkis"                     (height-8 subtrees
 *        as 256-entry LUTs, pointer values 240..255, CodeLengths),
 *   "Kernel GPU 2 tahap dan metadata bantu"               (8-byte segments
 *        per thread, 5-bit Gaps, per-thread-block output positions).
 *
 * Readings where the page is silent (each one is a choice, listed in the
 * design notes with its reason):
 *   - PackedSignMantissa byte = (sign << 7) | mantissa7.
 *   - Huffman ties: merge the two live nodes with the smallest
 *     (weight, smallest symbol in the subtree).
 *   - Codes longer than 32 bits are impossible in the format (Gaps are 5 bits
 *     because the longest code is 32): if plain Huffman exceeds the cap, the
 *     lengths come from package-merge (Larmore & Hirschberg 1990) instead.
 *   - Codes are canonical: symbols sorted by (length, symbol) get increasing
 *     code values (the DEFLATE construction, RFC 1951 section 3.2.2).
 *   - Bits are packed MSB-first within each byte, bytes in stream order.
 *   - One distinct symbol gets a 1-bit code "0".
 *   - Gap of segment s = (first code start >= 64 s, or the stream's end if no
 *     code starts there) - 64 s; 5-bit fields packed LSB-first into uint64
 *     words (field s at bits 5s .. 5s+4 of the word sequence).
 *   - BlockOffset[b] = number of codes that start before bit 64*T*b, plus a
 *     final entry equal to n.
 *   - LUT pointers: value 256 - j refers to child LUT j (j = 1..16); children
 *     are numbered breadth first, in increasing order of their bit prefix.
 *     Entries no code reaches (only with a single symbol) repeat that symbol.
 *
 * Every step is written the plain way: O(k^2) node scans, explicit trees,
 * one bit at a time.  Speed is not a goal.
 */
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_NSYM 256

/* ---------------------------------------------------------------------------
 * BF16 field split ("Ruang kompresi": 1 sign + 8 exponent + 7 mantissa bits;
 * "Format DFloat11": sign and mantissa kept verbatim).
 * Returns -1 when every exponent is < 240, else the index of the first element
 * whose exponent is in 240..255 (those values are reserved as LUT pointers,
 * "Decoding berbasis LUT hierarkis").
 * ------------------------------------------------------------------------- */
int64_t df11o_split(const uint16_t *w, uint64_t n, uint8_t *exps, uint8_t *sm)
{
    for (uint64_t i = 0; i < n; i++) {
        unsigned sign = (w[i] >> 15) & 1u;
        unsigned exponent = (w[i] >> 7) & 0xFFu;
        unsigned mantissa = w[i] & 0x7Fu;
        if (exponent >= 240u)
            return (int64_t)i;
        exps[i] = (uint8_t)exponent;
        sm[i] = (uint8_t)((sign << 7) | mantissa);
    }
    return -1;
}

/* Exponent histogram ("Ruang kompresi": the exponent distribution). */
void df11o_histogram(const uint8_t *exps, uint64_t n, uint64_t *hist)
{
    for (int s = 0; s < ORACLE_NSYM; s++)
        hist[s] = 0;
    for (uint64_t i = 0; i < n; i++)
        hist[exps[i]]++;
}

/* ---------------------------------------------------------------------------
 * Plain Huffman code lengths ("Format DFloat11": frequent exponents get short
 * codes, rare ones long codes).  Textbook construction: repeatedly merge the
 * two live nodes of smallest weight; a symbol's length is its leaf depth.
 * Returns the longest length (0 when no symbol occurs).
 * ------------------------------------------------------------------------- */
int df11o_huffman_lengths(const uint64_t *hist, uint8_t *len)
{
    uint64_t weight[2 * ORACLE_NSYM];
    int minsym[2 * ORACLE_NSYM];
    int parent[2 * ORACLE_NSYM];
    int live[2 * ORACLE_NSYM];
    int leaf_of[ORACLE_NSYM];
    int nodes = 0;

    for (int s = 0; s < ORACLE_NSYM; s++) {
        len[s] = 0;
        leaf_of[s] = -1;
        if (hist[s] > 0) {
            weight[nodes] = hist[s];
            minsym[nodes] = s;
            parent[nodes] = -1;
            live[nodes] = 1;
            leaf_of[s] = nodes;
            nodes++;
        }
    }
    int leaves = nodes;
    if (leaves == 0)
        return 0;
    if (leaves == 1) {
        for (int s = 0; s < ORACLE_NSYM; s++)
            if (leaf_of[s] >= 0)
                len[s] = 1;
        return 1;
    }
    for (int merges = 0; merges < leaves - 1; merges++) {
        int a = -1, b = -1;
        for (int i = 0; i < nodes; i++) {
            if (!live[i])
                continue;
            if (a < 0 || weight[i] < weight[a] ||
                (weight[i] == weight[a] && minsym[i] < minsym[a])) {
                b = a;
                a = i;
            } else if (b < 0 || weight[i] < weight[b] ||
                       (weight[i] == weight[b] && minsym[i] < minsym[b])) {
                b = i;
            }
        }
        live[a] = 0;
        live[b] = 0;
        weight[nodes] = weight[a] + weight[b];
        minsym[nodes] = minsym[a] < minsym[b] ? minsym[a] : minsym[b];
        parent[nodes] = -1;
        live[nodes] = 1;
        parent[a] = nodes;
        parent[b] = nodes;
        nodes++;
    }
    int longest = 0;
    for (int s = 0; s < ORACLE_NSYM; s++) {
        if (leaf_of[s] < 0)
            continue;
        int depth = 0;
        for (int v = leaf_of[s]; parent[v] >= 0; v = parent[v])
            depth++;
        len[s] = (uint8_t)depth;
        if (depth > longest)
            longest = depth;
    }
    return longest;
}

/* ---------------------------------------------------------------------------
 * Package-merge (Larmore & Hirschberg 1990): optimal prefix-code lengths with
 * every length <= max_len.  Coin-collector form, written out literally: every
 * item carries a vector counting how often each symbol occurs inside it.
 *   list(max_len) = leaves sorted by (weight, symbol)
 *   list(d)       = merge of the leaves with the pairs of list(d+1)
 *                   (pairs taken in order, an odd last item dropped);
 *                   at equal weight leaves come first, then pairs in order.
 *   take the first 2(k-1) items of list(1); length(s) = occurrences of s.
 * Returns 0, or -1 when 2^max_len < k (no such code exists).
 * ------------------------------------------------------------------------- */
typedef struct {
    uint64_t weight;
    uint16_t count[ORACLE_NSYM];
} oracle_item;

int df11o_package_merge(const uint64_t *hist, int max_len, uint8_t *len)
{
    int syms[ORACLE_NSYM];
    int k = 0;
    for (int s = 0; s < ORACLE_NSYM; s++) {
        len[s] = 0;
        if (hist[s] > 0)
            syms[k++] = s;
    }
    if (k == 0)
        return 0;
    if (k == 1) {
        len[syms[0]] = 1;
        return 0;
    }
    if (max_len < 1 || (max_len < 31 && (1 << max_len) < k))
        return -1;
    /* leaves sorted by (weight, symbol): insertion sort, k <= 256 */
    for (int i = 1; i < k; i++) {
        int v = syms[i], j = i - 1;
        while (j >= 0 && (hist[syms[j]] > hist[v] ||
                          (hist[syms[j]] == hist[v] && syms[j] > v))) {
            syms[j + 1] = syms[j];
            j--;
        }
        syms[j + 1] = v;
    }
    oracle_item *leaves = (oracle_item *)calloc((size_t)k, sizeof(oracle_item));
    oracle_item *cur = (oracle_item *)calloc((size_t)2 * k, sizeof(oracle_item));
    oracle_item *pairs = (oracle_item *)calloc((size_t)k, sizeof(oracle_item));
    oracle_item *next = (oracle_item *)calloc((size_t)2 * k, sizeof(oracle_item));
    if (!leaves || !cur || !pairs || !next) {
        free(leaves); free(cur); free(pairs); free(next);
        return -1;
    }
    for (int i = 0; i < k; i++) {
        leaves[i].weight = hist[syms[i]];
        leaves[i].count[syms[i]] = 1;
    }
    int ncur = k;
    for (int i = 0; i < k; i++)
        cur[i] = leaves[i];
    for (int d = max_len - 1; d >= 1; d--) {
        int npairs = ncur / 2;
        for (int p = 0; p < npairs; p++) {
            pairs[p].weight = cur[2 * p].weight + cur[2 * p + 1].weight;
            for (int s = 0; s < ORACLE_NSYM; s++)
                pairs[p].count[s] = (uint16_t)(cur[2 * p].count[s] + cur[2 * p + 1].count[s]);
        }
        int i = 0, j = 0, m = 0;
        while (i < k || j < npairs) {
            if (j >= npairs || (i < k && leaves[i].weight <= pairs[j].weight))
                next[m++] = leaves[i++];
            else
                next[m++] = pairs[j++];
        }
        ncur = m;
        oracle_item *t = cur; cur = next; next = t;
    }
    for (int i = 0; i < 2 * (k - 1); i++)
        for (int s = 0; s < ORACLE_NSYM; s++)
            len[s] = (uint8_t)(len[s] + cur[i].count[s]);
    free(leaves); free(cur); free(pairs); free(next);
    return 0;
}

/* Code lengths of the format: Huffman, or package-merge when Huffman's
 * longest code exceeds max_len ("Kernel GPU 2 tahap": the longest code is
 * 32 bits).  Returns the longest length, or -1 if no code fits. */
int df11o_code_lengths(const uint64_t *hist, int max_len, uint8_t *len)
{
    int longest = df11o_huffman_lengths(hist, len);
    if (longest <= max_len)
        return longest;
    if (df11o_package_merge(hist, max_len, len) != 0)
        return -1;
    longest = 0;
    for (int s = 0; s < ORACLE_NSYM; s++)
        if (len[s] > longest)
            longest = len[s];
    return longest;
}

/* Canonical code values from lengths (RFC 1951 section 3.2.2 construction):
 * walk symbols in (length, symbol) order; each next code is the previous one
 * plus one, shifted left by the growth in length. */
void df11o_canonical_codes(const uint8_t *len, uint32_t *code)
{
    uint64_t next_code = 0;
    int prev_len = 0;
    for (int s = 0; s < ORACLE_NSYM; s++)
        code[s] = 0;
    for (int l = 1; l <= 64; l++) {
        for (int s = 0; s < ORACLE_NSYM; s++) {
            if (len[s] != l)
                continue;
            next_code <<= (l - prev_len);
            prev_len = l;
            code[s] = (uint32_t)next_code;
            next_code++;
        }
    }
}

/* ---------------------------------------------------------------------------
 * EncodedExponent ("Format DFloat11": the exponents bit-packed in a byte
 * array).  Appends each element's code MSB-first, one bit at a time.
 * stream must hold ceil(total/8) bytes and be zeroed by the caller.
 * Returns the number of bits written.
 * ------------------------------------------------------------------------- */
uint64_t df11o_encode(const uint8_t *exps, uint64_t n, const uint8_t *len,
                      const uint32_t *code, uint8_t *stream)
{
    uint64_t pos = 0;
    for (uint64_t i = 0; i < n; i++) {
        int l = len[exps[i]];
        uint32_t c = code[exps[i]];
        for (int b = l - 1; b >= 0; b--) {
            unsigned bit = (c >> b) & 1u;
            if (bit)
                stream[pos >> 3] |= (uint8_t)(0x80u >> (pos & 7));
            pos++;
        }
    }
    return pos;
}

/* ---------------------------------------------------------------------------
 * Decoder metadata ("Kernel GPU 2 tahap dan metadata bantu").
 *   gaps[s]          one byte per 8-byte segment, in [0, 31]
 *   block_offset[b]  codes starting before bit 64*T*b; block_offset[nblocks]=n
 * with nsegments = ceil(total_bits / 64) and nblocks = ceil(nsegments / T).
 * Every code start is visited in order; each segment boundary 64 s gets the
 * first start at or after it.  Returns 0, or -1 if a gap exceeds 31.
 * ------------------------------------------------------------------------- */
int df11o_metadata(const uint8_t *exps, uint64_t n, const uint8_t *len,
                   uint64_t total_bits, uint32_t T,
                   uint8_t *gaps, uint32_t *block_offset)
{
    uint64_t nseg = (total_bits + 63) / 64;
    uint64_t nblocks = (nseg + T - 1) / T;
    uint64_t s = 0;   /* next segment boundary not yet assigned */
    uint64_t pos = 0; /* start bit of element i's code */
    for (uint64_t i = 0; i < n; i++) {
        while (s < nseg && 64 * s <= pos) {
            uint64_t gap = pos - 64 * s;
            if (gap > 31)
                return -1;
            gaps[s] = (uint8_t)gap;
            if (s % T == 0)
                block_offset[s / T] = (uint32_t)i;
            s++;
        }
        pos += len[exps[i]];
    }
    for (; s < nseg; s++) {
        uint64_t gap = total_bits - 64 * s;
        if (gap > 31)
            return -1;
        gaps[s] = (uint8_t)gap;
        if (s % T == 0)
            block_offset[s / T] = (uint32_t)n;
    }
    block_offset[nblocks] = (uint32_t)n;
    return 0;
}

/* 5-bit Gaps fields packed LSB-first: field s sits at bits 5s..5s+4 of the
 * little-endian concatenation of the uint64 words (zeroed by the caller). */
void df11o_pack_gaps(const uint8_t *gaps, uint64_t nseg, uint64_t *words)
{
    for (uint64_t s = 0; s < nseg; s++) {
        for (int b = 0; b < 5; b++) {
            uint64_t bitpos = 5 * s + (uint64_t)b;
            if ((gaps[s] >> b) & 1u)
                words[bitpos / 64] |= (uint64_t)1 << (bitpos % 64);
        }
    }
}

/* ---------------------------------------------------------------------------
 * Explicit code tree, shared by the LUT builder and the decoder below.
 * ------------------------------------------------------------------------- */
typedef struct {
    int child[2];
    int sym; /* -1 for an internal node */
} oracle_node;

/* Builds the binary tree of the canonical code.  Returns the node count, or
 * -1 when two codes collide (not a prefix code). */
static int oracle_build_tree(const uint8_t *len, const uint32_t *code,
                             oracle_node *tree, int cap)
{
    int nodes = 1;
    tree[0].child[0] = tree[0].child[1] = -1;
    tree[0].sym = -1;
    for (int s = 0; s < ORACLE_NSYM; s++) {
        if (len[s] == 0)
            continue;
        int v = 0;
        for (int b = len[s] - 1; b >= 0; b--) {
            if (tree[v].sym >= 0)
                return -1;
            int bit = (int)((code[s] >> b) & 1u);
            if (tree[v].child[bit] < 0) {
                if (nodes >= cap)
                    return -1;
                tree[nodes].child[0] = tree[nodes].child[1] = -1;
                tree[nodes].sym = -1;
                tree[v].child[bit] = nodes++;
            }
            v = tree[v].child[bit];
        }
        if (tree[v].sym >= 0 || tree[v].child[0] >= 0 || tree[v].child[1] >= 0)
            return -1;
        tree[v].sym = s;
    }
    return nodes;
}

/* ---------------------------------------------------------------------------
 * Hierarchical LUTs ("Decoding berbasis LUT hierarkis"): the tree is cut into
 * height-8 subtrees; each becomes a 256-entry table indexed by the next 8
 * bits.  An entry holds the symbol whose code ends inside this subtree, or the
 * pointer value 256 - j naming child LUT j (pointer values 240..255).
 * Each table is filled by walking the explicit tree from the subtree root,
 * one bit at a time, for each of the 256 indices.
 * luts must hold 17*256 bytes.  Returns 0, -1 (tree error) or -2 (more than
 * 16 child LUTs).
 * ------------------------------------------------------------------------- */
int df11o_build_luts(const uint8_t *len, const uint32_t *code, uint8_t *luts,
                     int *num_luts)
{
    int cap = 2 * 64 * ORACLE_NSYM + 1;
    oracle_node *tree = (oracle_node *)malloc(sizeof(oracle_node) * (size_t)cap);
    if (!tree)
        return -1;
    if (oracle_build_tree(len, code, tree, cap) < 0) {
        free(tree);
        return -1;
    }
    int only_sym = -1, nsym = 0;
    for (int s = 0; s < ORACLE_NSYM; s++)
        if (len[s] > 0) {
            nsym++;
            only_sym = s;
        }
    int root_of[17];
    int count = 1;
    root_of[0] = 0;
    memset(luts, 0, 17 * 256);
    for (int t = 0; t < count; t++) {
        for (int idx = 0; idx < 256; idx++) {
            int v = root_of[t];
            int entry = -1;
            for (int d = 0; d < 8; d++) {
                int bit = (idx >> (7 - d)) & 1;
                int c = tree[v].child[bit];
                if (c < 0) {
                    /* no code goes here: only possible with one symbol */
                    entry = nsym == 1 ? only_sym : 0;
                    break;
                }
                v = c;
                if (tree[v].sym >= 0) {
                    entry = tree[v].sym;
                    break;
                }
            }
            if (entry < 0) {
                /* eight bits consumed, still inside the tree: new child LUT */
                if (count >= 17) {
                    free(tree);
                    return -2;
                }
                root_of[count] = v;
                entry = 256 - count;
                count++;
            }
            luts[t * 256 + idx] = (uint8_t)entry;
        }
    }
    *num_luts = count;
    free(tree);
    return 0;
}

/* ---------------------------------------------------------------------------
 * Decoder: the sequential Huffman tree walk, one bit at a time ("Dekompresi
 * yang disesuaikan untuk inferensi GPU"), then BF16 reassembly from the
 * exponent and the verbatim sign/mantissa byte.
 * Returns 0, or -1 if the stream is inconsistent with the code.
 * ------------------------------------------------------------------------- */
int df11o_decode(const uint8_t *stream, uint64_t total_bits, const uint8_t *len,
                 const uint32_t *code, const uint8_t *sm, uint64_t n,
                 uint16_t *out)
{
    int cap = 2 * 64 * ORACLE_NSYM + 1;
    oracle_node *tree = (oracle_node *)malloc(sizeof(oracle_node) * (size_t)cap);
    if (!tree)
        return -1;
    if (oracle_build_tree(len, code, tree, cap) < 0) {
        free(tree);
        return -1;
    }
    uint64_t pos = 0;
    for (uint64_t i = 0; i < n; i++) {
        int v = 0;
        while (tree[v].sym < 0) {
            if (pos >= total_bits) {
                free(tree);
                return -1;
            }
            int bit = (stream[pos >> 3] >> (7 - (pos & 7))) & 1;
            pos++;
            v = tree[v].child[bit];
            if (v < 0) {
                free(tree);
                return -1;
            }
        }
        unsigned exponent = (unsigned)tree[v].sym;
        unsigned sign = (sm[i] >> 7) & 1u;
        unsigned mantissa = sm[i] & 0x7Fu;
        out[i] = (uint16_t)((sign << 15) | (exponent << 7) | mantissa);
    }
    free(tree);
    return pos == total_bits ? 0 : -1;
}

/* Decodes only the exponents of the codes that start in bit range
 * [start_bit, end_bit), with the same tree walk; used to check what one GPU
 * thread or one thread block must produce.  Returns the number of symbols,
 * or -1 on an inconsistent stream. */
int64_t df11o_decode_range(const uint8_t *stream, uint64_t stream_bits,
                           uint64_t start_bit, uint64_t end_bit,
                           const uint8_t *len, const uint32_t *code,
                           uint8_t *exps_out, uint64_t cap)
{
    int tcap = 2 * 64 * ORACLE_NSYM + 1;
    oracle_node *tree = (oracle_node *)malloc(sizeof(oracle_node) * (size_t)tcap);
    if (!tree)
        return -1;
    if (oracle_build_tree(len, code, tree, tcap) < 0) {
        free(tree);
        return -1;
    }
    uint64_t pos = start_bit;
    int64_t count = 0;
    while (pos < end_bit) {
        int v = 0;
        while (tree[v].sym < 0) {
            if (pos >= stream_bits) {
                free(tree);
                return -1;
            }
            int bit = (stream[pos >> 3] >> (7 - (pos & 7))) & 1;
            pos++;
            v = tree[v].child[bit];
            if (v < 0) {
                free(tree);
                return -1;
            }
        }
        if ((uint64_t)count >= cap) {
            free(tree);
            return -1;
        }
        exps_out[count++] = (uint8_t)tree[v].sym;
    }
    free(tree);
    return count;
}

/* ===========================================================================
 * rANS variant of the exponent coder (the page's discussion proposes rANS
 * as an entropy coder that suits SIMD-style hardware better than Huffman
 * coding).  The pages give no parameters; this restates the range variant
 * of asymmetric numeral systems from its published definition (J. Duda,
 * "Asymmetric numeral systems", 2013, range variant; one 32-bit state,
 * 16-bit renormalisation words, as in F. Giesen's description), with the
 * readings below.  TEST INFRASTRUCTURE: plain loops, no fusion.
 *
 *   model    : exponent counts h[s] quantised to frequencies f[s] summing to
 *              M = 2^prob_bits; cumulative c[s] = sum of f[t] for t < s.
 *   state    : x in [L, 2^32), L = 2^16.
 *   encode s : if x >= 2^(32 - prob_bits) * f[s]: emit x mod 2^16 (one
 *              16-bit word), x = floor(x / 2^16); then
 *              x = floor(x / f[s]) * M + (x mod f[s]) + c[s].
 *   decode   : slot = x mod M; s = the symbol with c[s] <= slot < c[s] + f[s];
 *              x = f[s] * floor(x / M) + slot - c[s]; if x < L: x = x * 2^16 +
 *              the next 16-bit word.
 *   layout   : blocks of B = 32 * 16 * J elements; lane l (0..31) of block b
 *              owns elements b B + 512 j + 16 l + i (j = 0..J-1, i = 0..15),
 *              decoded in the order (j, i); all lanes step together, step
 *              t = 16 j + i; a lane whose element lies at or past n skips the
 *              step.  Each lane has its own word stream: a renormalising lane
 *              reads the next word of it.  A block's words are lane 0's
 *              stream, then lane 1's, ..., lane 31's; lane_words[32 b + l]
 *              counts lane l's words (at most one per step: 16 J <= 240
 *              words, so J <= 15).  The encoder runs the same steps backwards
 *              (t descending), starting every lane at x = L; its final states
 *              are the decoder's start states, and each lane's words,
 *              reversed, that lane's stream.
 * ======================================================================== */

/* Frequencies: f[s] = max(1, floor(h[s] M / n)) for every symbol present,
 * 0 otherwise; then, while the sum exceeds M, the largest frequency (ties:
 * smallest symbol) drops by one, and while it is short of M the symbol with
 * the largest count (ties: smallest symbol) gains one.  Returns 0, or -1 when
 * no symbol is present or more symbols are present than M allows. */
int df11o_rans_freqs(const uint64_t *hist, int prob_bits, uint32_t *freq)
{
    uint64_t n = 0;
    int present = 0;
    for (int s = 0; s < ORACLE_NSYM; s++) {
        n += hist[s];
        present += hist[s] > 0;
    }
    const uint32_t M = 1u << prob_bits;
    if (n == 0 || (uint32_t)present > M)
        return -1;
    uint64_t sum = 0;
    for (int s = 0; s < ORACLE_NSYM; s++) {
        freq[s] = 0;
        if (hist[s]) {
            uint64_t f = hist[s] * (uint64_t)M / n;
            freq[s] = f < 1 ? 1u : (uint32_t)f;
        }
        sum += freq[s];
    }
    while (sum > M) {
        int best = -1;
        for (int s = 0; s < ORACLE_NSYM; s++)
            if (freq[s] > 1 && (best < 0 || freq[s] > freq[best]))
                best = s;
        freq[best]--;
        sum--;
    }
    while (sum < M) {
        int best = -1;
        for (int s = 0; s < ORACLE_NSYM; s++)
            if (hist[s] && (best < 0 || hist[s] > hist[best]))
                best = s;
        freq[best]++;
        sum++;
    }
    return 0;
}

/* Element of block b owned by lane l at step t (J chunks per lane). */
static uint64_t oracle_rans_pos(uint64_t b, int J, int l, int t)
{
    return b * (uint64_t)(512 * J) + 512u * (uint64_t)(t / 16) + 16u * (uint64_t)l + (uint64_t)(t % 16);
}

/* rANS encode of n exponents, blocks of 512 J elements (J <= 15).  words
 * receives the words of block 0 (lane 0's stream, then lane 1's, ...), then
 * block 1, ...; offsets[b] (nblocks + 1 entries) the index of block b's
 * first word; lane_words[32 b + l] the length of lane l's stream in block b;
 * states[32 b + l] the start state of lane l of block b.  Returns the number
 * of words, or -1 (J out of range, capacity, a symbol with frequency 0, or a
 * state outside [L, 2^32)). */
int64_t df11o_rans_encode(const uint8_t *exps, uint64_t n, const uint32_t *freq, int prob_bits, int J,
                          uint16_t *words, uint64_t cap, uint32_t *states, uint64_t *offsets, uint8_t *lane_words)
{
    const uint64_t L = 1ull << 16, M = 1ull << prob_bits;
    if (J < 1 || J > 15)
        return -1;
    const uint64_t B = 512ull * (uint64_t)J;
    const uint64_t nblocks = (n + B - 1) / B;
    uint64_t cum[ORACLE_NSYM];
    uint64_t c = 0;
    for (int s = 0; s < ORACLE_NSYM; s++) {
        cum[s] = c;
        c += freq[s];
    }
    if (c != M)
        return -1;
    /* one stack per lane: at most one word per step */
    uint16_t *stack = (uint16_t *)malloc(sizeof(uint16_t) * 32 * 16 * (size_t)J);
    if (!stack)
        return -1;
    uint64_t total = 0;
    for (uint64_t b = 0; b < nblocks; b++) {
        uint64_t x[32];
        int depth[32];
        for (int l = 0; l < 32; l++) {
            x[l] = L;
            depth[l] = 0;
        }
        for (int t = 16 * J - 1; t >= 0; t--) {
            for (int l = 0; l < 32; l++) {
                const uint64_t pos = oracle_rans_pos(b, J, l, t);
                if (pos >= n)
                    continue;
                const int s = exps[pos];
                const uint64_t f = freq[s];
                if (f == 0) {
                    free(stack);
                    return -1;
                }
                if (x[l] >= (1ull << (32 - prob_bits)) * f) {
                    stack[16 * J * l + depth[l]++] = (uint16_t)(x[l] & 0xFFFFu);
                    x[l] >>= 16;
                }
                x[l] = (x[l] / f) * M + (x[l] % f) + cum[s];
                if (x[l] < L || x[l] >= (1ull << 32)) {
                    free(stack);
                    return -1;
                }
            }
        }
        offsets[b] = total;
        for (int l = 0; l < 32; l++) {
            if (total + (uint64_t)depth[l] > cap) {
                free(stack);
                return -1;
            }
            for (int k = 0; k < depth[l]; k++)
                words[total + k] = stack[16 * J * l + depth[l] - 1 - k];
            total += (uint64_t)depth[l];
            lane_words[32 * b + l] = (uint8_t)depth[l];
            states[32 * b + l] = (uint32_t)x[l];
        }
    }
    offsets[nblocks] = total;
    free(stack);
    return (int64_t)total;
}

/* rANS decode back to BF16 bits (exponent from the words, sign and mantissa
 * from sm).  Returns 0, or -1 when the words, states, offsets or lane counts
 * are inconsistent (the lane counts do not add up to the block's words, a
 * lane reads past its stream or does not use all of it, or does not end at
 * x = L). */
int df11o_rans_decode(const uint16_t *words, const uint32_t *states, const uint64_t *offsets,
                      const uint8_t *lane_words, const uint32_t *freq, int prob_bits, int J, uint64_t n,
                      const uint8_t *sm, uint16_t *out)
{
    const uint64_t L = 1ull << 16, M = 1ull << prob_bits;
    if (J < 1 || J > 15)
        return -1;
    const uint64_t B = 512ull * (uint64_t)J;
    const uint64_t nblocks = (n + B - 1) / B;
    uint64_t cum[ORACLE_NSYM];
    uint64_t c = 0;
    for (int s = 0; s < ORACLE_NSYM; s++) {
        cum[s] = c;
        c += freq[s];
    }
    if (c != M)
        return -1;
    for (uint64_t b = 0; b < nblocks; b++) {
        uint64_t x[32], ptr[32], end[32];
        uint64_t start = offsets[b];
        for (int l = 0; l < 32; l++) {
            x[l] = states[32 * b + l];
            ptr[l] = start;
            end[l] = start + lane_words[32 * b + l];
            start = end[l];
        }
        if (start != offsets[b + 1])
            return -1;
        for (int t = 0; t < 16 * J; t++) {
            for (int l = 0; l < 32; l++) {
                const uint64_t pos = oracle_rans_pos(b, J, l, t);
                if (pos >= n)
                    continue;
                const uint64_t slot = x[l] % M;
                int s = -1;
                for (int k = 0; k < ORACLE_NSYM; k++)
                    if (freq[k] && cum[k] <= slot && slot < cum[k] + freq[k])
                        s = k;
                if (s < 0)
                    return -1;
                x[l] = freq[s] * (x[l] / M) + slot - cum[s];
                const unsigned sign = (sm[pos] >> 7) & 1u, mantissa = sm[pos] & 0x7Fu;
                out[pos] = (uint16_t)((sign << 15) | ((unsigned)s << 7) | mantissa);
                if (x[l] < L) {
                    if (ptr[l] >= end[l])
                        return -1;
                    x[l] = (x[l] << 16) | words[ptr[l]++];
                }
            }
        }
        for (int l = 0; l < 32; l++)
            if (ptr[l] != end[l] || x[l] != L)
                return -1;
    }
    return 0;
}

/* One rANS step on a single state, for exhaustive checks: encodes s into
 * x (x in [L, 2^32)) and returns the new state; *word / *emitted receive the
 * renormalisation word, if any. */
uint64_t df11o_rans_step_encode(uint64_t x, int s, const uint32_t *freq, int prob_bits, uint32_t *word,
                                int *emitted)
{
    uint64_t cum = 0;
    for (int k = 0; k < s; k++)
        cum += freq[k];
    const uint64_t f = freq[s], M = 1ull << prob_bits;
    *emitted = 0;
    if (x >= (1ull << (32 - prob_bits)) * f) {
        *word = (uint32_t)(x & 0xFFFFu);
        *emitted = 1;
        x >>= 16;
    }
    return (x / f) * M + (x % f) + cum;
}

/* BF16 field split for the rANS variant: as df11o_split, but every exponent
 * 0..255 is allowed (rANS needs no pointer values). */
void df11o_split_all(const uint16_t *w, uint64_t n, uint8_t *exps, uint8_t *sm)
{
    for (uint64_t i = 0; i < n; i++) {
        unsigned sign = (w[i] >> 15) & 1u;
        unsigned exponent = (w[i] >> 7) & 0xFFu;
        unsigned mantissa = w[i] & 0x7Fu;
        exps[i] = (uint8_t)exponent;
        sm[i] = (uint8_t)((sign << 7) | mantissa);
    }
}
