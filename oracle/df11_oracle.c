/*
 * df11_oracle.c -- plain, slow, single-threaded CPU reference of the
 * Dynamic-Length Float (DFloat11) exponent code.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product (the entropy_decoding_b200
 * package, its C-ABI library or its kernels) includes, links or calls this
 * file; only tests/, the smoke check and the CPU baseline of bench.py do.  It
 * shares no code, header, table or constant with the product: every step is
 * written out here again from the method's definition, in the order the
 * sources state it, with no blocking, fusion or reordering.
 *
 * Sources (cited by page title and section):
 *  [DF11]  "70% Size, 100% Accuracy: Lossless LLM Compression for Efficient
 *          GPU Inference via Dynamic-Length Float (DFloat11)", Abstract:
 *          entropy-code the low-entropy part of BF16 with frequency-based
 *          dynamic-length codes; lossless (bit-for-bit identical outputs);
 *          per-thread read/write positions coordinated by auxiliary variables.
 *  [BLOG]  "Compressing LLMs without Compromise" summary page, section
 *          "Where the redundancy lives": BF16 = 1 sign + 8 exponent + 7
 *          mantissa bits; only the exponent is low-entropy.  Section "Three
 *          ways to spend the savings": DFloat11 Huffman-codes the exponents
 *          offline and replaces the 8 bits by shorter lookup keys.
 *  [ECF8]  "To Compress or Not? ... Exponent Concentration", Abstract: the same
 *          exponent coding applied to FP8 weights.
 *  [SHANNON] "Approaching Shannon Bound with Lossless LLM Weight
 *          Compression", Abstract: tile-level decoding with Asymmetric
 *          Numeral Systems, within 0.01-0.1 bits of the Shannon limit
 *          (section 9, the rANS variant).
 *
 * Where the sources are silent the oracle takes these readings (all listed
 * in the repository's design notes):
 *  - Huffman tie-break: a min-heap keyed (count, order) with order = symbol
 *    value for leaves and 256 + creation index for merged nodes.  Exactly one
 *    distinct symbol gets length 1.  Zero-count symbols get no code.
 *  - Length limit: when the Huffman depth exceeds max_len, the lengths are
 *    replaced by the package-merge solution (optimal among length-limited
 *    prefix codes); equal weights keep leaves before packages, leaves in
 *    (count, symbol) order, packages in creation order.
 *  - Canonical code assignment: symbols sorted by (length, symbol), first
 *    code 0, next = (previous + 1) << (length increase).
 *  - Bit order: code bits are appended most-significant first; stream bit k
 *    is bit (7 - k % 8) of byte k / 8.
 *  - Auxiliary variables: the stream is cut into chunks of chunk_bits bits,
 *    one per decoding thread; gap[c] = (first code start >= c*chunk_bits, or
 *    total_bits) - c*chunk_bits.  Threads are grouped into tiles of
 *    tile_threads chunks; out_off[b] = number of codes starting before bit
 *    b*tile_threads*chunk_bits, for b = 0..n_tiles (out_off[n_tiles] = n).
 *  - Chunk counts (this implementation's optional container section):
 *    counts[c] = number of codes whose first bit lies in chunk c.
 *  - Raw fields: BF16 keeps one byte (sign << 7 | 7-bit mantissa) per weight;
 *    E4M3 keeps one nibble (sign << 3 | 3-bit mantissa) per weight, element
 *    2i in the low nibble of byte i.
 *
 * Parity status: every function here is pinned by tests that do not reuse
 * it (round-trip identity, Kraft equality, entropy bounds, brute-force
 * optimality, closed forms, hand-derived golden streams, an independent
 * dynamic program for length-limited optimality, independent aux walks, a
 * tally of code starts for the chunk counts; for section 9 hand-derived
 * frequencies, states and words, closed forms, the information bound and
 * the distance to the Shannon limit).
 */
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_OK 0
#define ORACLE_EINVAL 1
#define ORACLE_ENOMEM 2
#define ORACLE_ECORRUPT 4

/* ------------------------------------------------------------------ */
/* 1. Field split  ([BLOG] "Where the redundancy lives"; [ECF8])        */
/* ------------------------------------------------------------------ */

/* BF16 word w: sign = bit 15, exponent = bits 14..7, mantissa = bits 6..0. */
void oracle_split_bf16(const uint16_t *w, uint64_t n, uint8_t *exps, uint8_t *plane)
{
    for (uint64_t i = 0; i < n; i++) {
        uint16_t v = w[i];
        uint8_t sign = (uint8_t)((v >> 15) & 1u);
        uint8_t expo = (uint8_t)((v >> 7) & 0xFFu);
        uint8_t mant = (uint8_t)(v & 0x7Fu);
        exps[i] = expo;
        plane[i] = (uint8_t)((sign << 7) | mant);
    }
}

/* E4M3 byte b: sign = bit 7, exponent = bits 6..3, mantissa = bits 2..0.
 * plane must hold (n + 1) / 2 bytes and is fully written. */
void oracle_split_e4m3(const uint8_t *b, uint64_t n, uint8_t *exps, uint8_t *plane)
{
    for (uint64_t i = 0; i < (n + 1) / 2; i++) plane[i] = 0;
    for (uint64_t i = 0; i < n; i++) {
        uint8_t v = b[i];
        uint8_t sign = (uint8_t)((v >> 7) & 1u);
        uint8_t expo = (uint8_t)((v >> 3) & 0xFu);
        uint8_t mant = (uint8_t)(v & 0x7u);
        uint8_t nib = (uint8_t)((sign << 3) | mant);
        exps[i] = expo;
        if (i % 2 == 0)
            plane[i / 2] = (uint8_t)(plane[i / 2] | nib);
        else
            plane[i / 2] = (uint8_t)(plane[i / 2] | (nib << 4));
    }
}

/* Inverse of the split: rebuild each weight from its exponent and raw field. */
void oracle_merge_bf16(const uint8_t *exps, const uint8_t *plane, uint64_t n, uint16_t *out)
{
    for (uint64_t i = 0; i < n; i++) {
        uint16_t sign = (uint16_t)((plane[i] >> 7) & 1u);
        uint16_t mant = (uint16_t)(plane[i] & 0x7Fu);
        uint16_t expo = exps[i];
        out[i] = (uint16_t)((sign << 15) | (expo << 7) | mant);
    }
}

void oracle_merge_e4m3(const uint8_t *exps, const uint8_t *plane, uint64_t n, uint8_t *out)
{
    for (uint64_t i = 0; i < n; i++) {
        uint8_t nib = (i % 2 == 0) ? (uint8_t)(plane[i / 2] & 0xFu) : (uint8_t)(plane[i / 2] >> 4);
        uint8_t sign = (uint8_t)((nib >> 3) & 1u);
        uint8_t mant = (uint8_t)(nib & 0x7u);
        out[i] = (uint8_t)((sign << 7) | ((exps[i] & 0xFu) << 3) | mant);
    }
}

/* ------------------------------------------------------------------ */
/* 2. Histogram  ([DF11] "based on frequency")                          */
/* ------------------------------------------------------------------ */

/* Adds the symbol counts of exps[0..n) into counts[] (not cleared). */
void oracle_histogram(const uint8_t *exps, uint64_t n, uint64_t *counts)
{
    for (uint64_t i = 0; i < n; i++) counts[exps[i]] += 1;
}

/* ------------------------------------------------------------------ */
/* 3. Huffman code lengths  ([BLOG] "Huffman-codes the exponents")      */
/* ------------------------------------------------------------------ */

typedef struct {
    uint64_t count;
    int order;   /* symbol for leaves, 256 + creation index for merged nodes */
    int parent;  /* -1 for the root */
} hnode;

static int key_less(const hnode *a, const hnode *b)
{
    if (a->count != b->count) return a->count < b->count;
    return a->order < b->order;
}

static void heap_push(int *heap, int *size, const hnode *nodes, int id)
{
    int i = (*size)++;
    heap[i] = id;
    while (i > 0) {
        int p = (i - 1) / 2;
        if (key_less(&nodes[heap[i]], &nodes[heap[p]])) {
            int t = heap[i]; heap[i] = heap[p]; heap[p] = t;
            i = p;
        } else {
            break;
        }
    }
}

static int heap_pop(int *heap, int *size, const hnode *nodes)
{
    int top = heap[0];
    (*size)--;
    heap[0] = heap[*size];
    int i = 0;
    for (;;) {
        int l = 2 * i + 1, r = 2 * i + 2, m = i;
        if (l < *size && key_less(&nodes[heap[l]], &nodes[heap[m]])) m = l;
        if (r < *size && key_less(&nodes[heap[r]], &nodes[heap[m]])) m = r;
        if (m == i) break;
        int t = heap[i]; heap[i] = heap[m]; heap[m] = t;
        i = m;
    }
    return top;
}

/* Unconstrained Huffman lengths; returns the maximum depth. */
static int huffman_unlimited(const uint64_t *counts, int nsym, uint8_t *lengths)
{
    hnode nodes[2 * 256];
    int heap[2 * 256];
    int leaf_of_sym[256];
    int nn = 0, hs = 0, distinct = 0;
    for (int s = 0; s < nsym; s++) {
        lengths[s] = 0;
        leaf_of_sym[s] = -1;
        if (counts[s] > 0) {
            nodes[nn].count = counts[s];
            nodes[nn].order = s;
            nodes[nn].parent = -1;
            leaf_of_sym[s] = nn;
            heap_push(heap, &hs, nodes, nn);
            nn++;
            distinct++;
        }
    }
    if (distinct == 0) return 0;
    if (distinct == 1) {
        for (int s = 0; s < nsym; s++)
            if (counts[s] > 0) lengths[s] = 1;
        return 1;
    }
    int created = 0;
    while (hs > 1) {
        int a = heap_pop(heap, &hs, nodes);
        int b = heap_pop(heap, &hs, nodes);
        nodes[nn].count = nodes[a].count + nodes[b].count;
        nodes[nn].order = 256 + created;
        nodes[nn].parent = -1;
        nodes[a].parent = nn;
        nodes[b].parent = nn;
        heap_push(heap, &hs, nodes, nn);
        nn++;
        created++;
    }
    int maxd = 0;
    for (int s = 0; s < nsym; s++) {
        if (leaf_of_sym[s] < 0) continue;
        int d = 0;
        for (int v = leaf_of_sym[s]; nodes[v].parent >= 0; v = nodes[v].parent) d++;
        lengths[s] = (uint8_t)(d > 255 ? 255 : d);
        if (d > maxd) maxd = d;
    }
    return maxd;
}

/* Package-merge (Larmore & Hirschberg): optimal prefix code lengths with every
 * length <= max_len.  Items are leaves (one per used symbol) or packages (a
 * pair of items from the list one level deeper).  The list for the top level
 * is built from max_len levels; its first 2(m-1) items are selected and each
 * symbol's length is the number of times its leaf occurs inside them. */
typedef struct {
    uint64_t w;
    int sym;  /* >= 0 for a leaf, -1 for a package */
    int a, b; /* children (item ids) of a package */
} pm_item;

static void pm_count(const pm_item *items, int id, uint8_t *lengths)
{
    if (items[id].sym >= 0) {
        lengths[items[id].sym]++;
        return;
    }
    pm_count(items, items[id].a, lengths);
    pm_count(items, items[id].b, lengths);
}

static int package_merge(const uint64_t *counts, int nsym, int max_len, uint8_t *lengths)
{
    int syms[256];
    int m = 0;
    for (int s = 0; s < nsym; s++) {
        lengths[s] = 0;
        if (counts[s] > 0) syms[m++] = s;
    }
    /* leaves sorted by (count, symbol): insertion sort, m <= 256 */
    for (int i = 1; i < m; i++) {
        int v = syms[i], j = i - 1;
        while (j >= 0 && (counts[syms[j]] > counts[v] ||
                          (counts[syms[j]] == counts[v] && syms[j] > v))) {
            syms[j + 1] = syms[j];
            j--;
        }
        syms[j + 1] = v;
    }
    if (m <= 1) {
        if (m == 1) lengths[syms[0]] = 1;
        return ORACLE_OK;
    }
    if (max_len < 32 && ((uint64_t)1 << max_len) < (uint64_t)m) return ORACLE_EINVAL;

    size_t cap = (size_t)max_len * (size_t)(2 * m) + 16;
    pm_item *items = (pm_item *)malloc(cap * sizeof(pm_item));
    int *prev = (int *)malloc((size_t)(2 * m) * sizeof(int));
    int *cur = (int *)malloc((size_t)(2 * m) * sizeof(int));
    int *pk = (int *)malloc((size_t)m * sizeof(int));
    if (!items || !prev || !cur || !pk) {
        free(items); free(prev); free(cur); free(pk);
        return ORACLE_ENOMEM;
    }
    int ni = 0, nprev = 0;
    for (int level = max_len; level >= 1; level--) {
        /* packages from the deeper list: consecutive pairs, odd one dropped */
        int np = 0;
        for (int i = 0; i + 1 < nprev; i += 2) {
            items[ni].w = items[prev[i]].w + items[prev[i + 1]].w;
            items[ni].sym = -1;
            items[ni].a = prev[i];
            items[ni].b = prev[i + 1];
            pk[np++] = ni++;
        }
        /* fresh leaves for this level */
        int leaf0 = ni;
        for (int i = 0; i < m; i++) {
            items[ni].w = counts[syms[i]];
            items[ni].sym = syms[i];
            items[ni].a = items[ni].b = -1;
            ni++;
        }
        /* merge by weight; equal weight: leaf first */
        int i = 0, j = 0, nc = 0;
        while (i < m || j < np) {
            if (j >= np || (i < m && items[leaf0 + i].w <= items[pk[j]].w))
                cur[nc++] = leaf0 + i++;
            else
                cur[nc++] = pk[j++];
        }
        int *t = prev; prev = cur; cur = t;
        nprev = nc;
    }
    for (int i = 0; i < 2 * (m - 1); i++) pm_count(items, prev[i], lengths);
    free(items); free(prev); free(cur); free(pk);
    return ORACLE_OK;
}

/* Code lengths for counts[0..nsym): Huffman, replaced by package-merge when
 * the Huffman depth exceeds max_len.  Returns ORACLE_OK or ORACLE_EINVAL. */
int oracle_code_lengths(const uint64_t *counts, int nsym, int max_len, uint8_t *lengths)
{
    if (nsym < 1 || nsym > 256 || max_len < 1 || max_len > 32) return ORACLE_EINVAL;
    int d = huffman_unlimited(counts, nsym, lengths);
    if (d <= max_len) return ORACLE_OK;
    return package_merge(counts, nsym, max_len, lengths);
}

/* Unconstrained Huffman lengths only (exposed so tests can check the
 * textbook bound and the depth that triggers the limiter). */
int oracle_huffman_depth(const uint64_t *counts, int nsym, uint8_t *lengths)
{
    return huffman_unlimited(counts, nsym, lengths);
}

/* ------------------------------------------------------------------ */
/* 4. Canonical codes                                                   */
/* ------------------------------------------------------------------ */

void oracle_canonical_codes(const uint8_t *lengths, int nsym, uint32_t *codes)
{
    int order[256];
    int m = 0;
    for (int s = 0; s < nsym; s++) {
        codes[s] = 0;
        if (lengths[s] > 0) order[m++] = s;
    }
    for (int i = 1; i < m; i++) {
        int v = order[i], j = i - 1;
        while (j >= 0 && (lengths[order[j]] > lengths[v] ||
                          (lengths[order[j]] == lengths[v] && order[j] > v))) {
            order[j + 1] = order[j];
            j--;
        }
        order[j + 1] = v;
    }
    uint64_t code = 0;
    for (int i = 0; i < m; i++) {
        if (i > 0) code = (code + 1) << (lengths[order[i]] - lengths[order[i - 1]]);
        codes[order[i]] = (uint32_t)code;
    }
}

/* ------------------------------------------------------------------ */
/* 5. Bitstream  ([DF11] dynamic-length encodings; MSB-first reading)   */
/* ------------------------------------------------------------------ */

uint64_t oracle_total_bits(const uint8_t *exps, uint64_t n, const uint8_t *lengths)
{
    uint64_t t = 0;
    for (uint64_t i = 0; i < n; i++) t += lengths[exps[i]];
    return t;
}

/* stream must hold at least ceil(total_bits / 8) zeroed bytes. */
int oracle_pack(const uint8_t *exps, uint64_t n, const uint8_t *lengths, const uint32_t *codes,
                uint8_t *stream, uint64_t stream_bytes)
{
    uint64_t k = 0;
    for (uint64_t i = 0; i < n; i++) {
        int len = lengths[exps[i]];
        if (len == 0) return ORACLE_EINVAL; /* symbol without a code */
        uint32_t code = codes[exps[i]];
        for (int j = len - 1; j >= 0; j--) {
            uint32_t bit = (code >> j) & 1u;
            if ((k >> 3) >= stream_bytes) return ORACLE_EINVAL;
            if (bit) stream[k >> 3] = (uint8_t)(stream[k >> 3] | (0x80u >> (k & 7)));
            k++;
        }
    }
    return ORACLE_OK;
}

/* ------------------------------------------------------------------ */
/* 6. Auxiliary variables  ([DF11] two-phase kernel coordinating thread  */
/*    read/write positions with lightweight auxiliary variables)        */
/* ------------------------------------------------------------------ */

/* Number of chunks and tiles for a stream of total_bits bits. */
void oracle_layout(uint64_t total_bits, int chunk_bits, int tile_threads,
                   uint64_t *n_chunks, uint64_t *n_tiles)
{
    uint64_t c = (total_bits + (uint64_t)chunk_bits - 1) / (uint64_t)chunk_bits;
    *n_chunks = c;
    *n_tiles = (c + (uint64_t)tile_threads - 1) / (uint64_t)tile_threads;
}

/* gaps: n_tiles * tile_threads bytes (entries past the last chunk are 0).
 * out_off: n_tiles + 1 entries.  Walks the code start positions once. */
int oracle_aux(const uint8_t *exps, uint64_t n, const uint8_t *lengths,
               int chunk_bits, int tile_threads,
               uint8_t *gaps, uint64_t *out_off, uint64_t *max_span)
{
    uint64_t total = oracle_total_bits(exps, n, lengths);
    uint64_t n_chunks, n_tiles;
    oracle_layout(total, chunk_bits, tile_threads, &n_chunks, &n_tiles);
    uint64_t tile_bits = (uint64_t)chunk_bits * (uint64_t)tile_threads;
    for (uint64_t c = 0; c < n_tiles * (uint64_t)tile_threads; c++) gaps[c] = 0;

    /* gap: for each chunk, the first code start at or after its first bit */
    uint64_t i = 0, start = 0;
    for (uint64_t c = 0; c < n_chunks; c++) {
        uint64_t c0 = c * (uint64_t)chunk_bits;
        while (i < n && start < c0) {
            start += lengths[exps[i]];
            i++;
        }
        uint64_t first = (i < n) ? start : total;
        uint64_t g = first - c0;
        if (g > 255) return ORACLE_EINVAL;
        gaps[c] = (uint8_t)g;
    }
    /* out_off: codes starting before each tile's first bit */
    i = 0;
    start = 0;
    for (uint64_t b = 0; b <= n_tiles; b++) {
        uint64_t b0 = b * tile_bits;
        while (i < n && start < b0) {
            start += lengths[exps[i]];
            i++;
        }
        out_off[b] = i;
    }
    uint64_t ms = 0;
    for (uint64_t b = 0; b < n_tiles; b++)
        if (out_off[b + 1] - out_off[b] > ms) ms = out_off[b + 1] - out_off[b];
    *max_span = ms;
    return ORACLE_OK;
}

/* Chunk counts (a container section of this implementation, not of the
 * pages' format; it stores what the first of the two phases computes, the
 * number of codes each thread's chunk holds, so that the decoder needs only
 * the second): counts[c] = the number of codes whose first bit lies in
 * [c * chunk_bits, (c + 1) * chunk_bits).  n_tiles * tile_threads entries,
 * 0 past the last chunk.  Fails when a count does not fit a byte. */
int oracle_chunk_counts(const uint8_t *exps, uint64_t n, const uint8_t *lengths,
                        int chunk_bits, int tile_threads, uint8_t *counts)
{
    uint64_t total = oracle_total_bits(exps, n, lengths);
    uint64_t n_chunks, n_tiles;
    oracle_layout(total, chunk_bits, tile_threads, &n_chunks, &n_tiles);
    uint64_t *tally = (uint64_t *)calloc(n_chunks ? n_chunks : 1, sizeof(uint64_t));
    if (!tally) return ORACLE_ENOMEM;
    uint64_t start = 0;
    for (uint64_t i = 0; i < n; i++) {
        tally[start / (uint64_t)chunk_bits]++;
        start += lengths[exps[i]];
    }
    int rc = ORACLE_OK;
    for (uint64_t c = 0; c < n_tiles * (uint64_t)tile_threads; c++) {
        uint64_t v = c < n_chunks ? tally[c] : 0;
        if (v > 255) rc = ORACLE_EINVAL;
        counts[c] = (uint8_t)v;
    }
    free(tally);
    return rc;
}

/* ------------------------------------------------------------------ */
/* 7. Decoding: bit-by-bit walk of the explicit code tree               */
/* ------------------------------------------------------------------ */

typedef struct {
    int child[2]; /* node ids, -1 when absent */
    int sym;      /* >= 0 at a leaf */
} tnode;

/* Builds the binary code tree.  Returns the node count or -1 when two codes
 * collide (not a prefix code). */
static int build_tree(const uint8_t *lengths, const uint32_t *codes, int nsym, tnode *t, int cap)
{
    int nn = 1;
    t[0].child[0] = t[0].child[1] = -1;
    t[0].sym = -1;
    for (int s = 0; s < nsym; s++) {
        int len = lengths[s];
        if (len == 0) continue;
        int v = 0;
        for (int j = len - 1; j >= 0; j--) {
            if (t[v].sym >= 0) return -1;
            int bit = (int)((codes[s] >> j) & 1u);
            if (t[v].child[bit] < 0) {
                if (nn >= cap) return -1;
                t[nn].child[0] = t[nn].child[1] = -1;
                t[nn].sym = -1;
                t[v].child[bit] = nn++;
            }
            v = t[v].child[bit];
        }
        if (t[v].sym >= 0 || t[v].child[0] >= 0 || t[v].child[1] >= 0) return -1;
        t[v].sym = s;
    }
    return nn;
}

/* Decodes `count` symbols starting at stream bit start_bit; every bit read
 * must lie below total_bits.  Returns ORACLE_ECORRUPT on a bit path that
 * leaves the tree or runs past total_bits. */
int oracle_decode(const uint8_t *stream, uint64_t total_bits,
                  const uint8_t *lengths, int nsym,
                  uint64_t start_bit, uint64_t count, uint8_t *exps_out)
{
    uint32_t codes[256];
    oracle_canonical_codes(lengths, nsym, codes);
    int cap = 32 * 256 + 2;
    tnode *t = (tnode *)malloc((size_t)cap * sizeof(tnode));
    if (!t) return ORACLE_ENOMEM;
    if (build_tree(lengths, codes, nsym, t, cap) < 0) {
        free(t);
        return ORACLE_EINVAL;
    }
    uint64_t k = start_bit;
    for (uint64_t i = 0; i < count; i++) {
        int v = 0;
        while (t[v].sym < 0) {
            if (k >= total_bits) { free(t); return ORACLE_ECORRUPT; }
            int bit = (stream[k >> 3] >> (7 - (k & 7))) & 1;
            k++;
            v = t[v].child[bit];
            if (v < 0) { free(t); return ORACLE_ECORRUPT; }
        }
        exps_out[i] = (uint8_t)t[v].sym;
    }
    free(t);
    return ORACLE_OK;
}

/* ------------------------------------------------------------------ */
/* 9. rANS variant of the exponent coder.                               */
/*    [SHANNON] "Approaching Shannon Bound with Lossless LLM Weight     */
/*    Compression", Abstract: tile-level decoding with Asymmetric       */
/*    Numeral Systems, within 0.01-0.1 bits of the Shannon limit.       */
/*    The page gives no coder details.  This is the range variant of    */
/*    ANS (rANS, Duda) in its textbook form: a state x; a symbol s      */
/*    with quantized frequency f_s and cumulative frequency c_s over a  */
/*    total M = 2^12 is coded as                                        */
/*        x' = floor(x / f_s) * M + (x mod f_s) + c_s                   */
/*    and decoded from x' as the s with c_s <= x' mod M < c_s + f_s,    */
/*        x = f_s * floor(x' / M) + (x' mod M) - c_s,                   */
/*    the state kept in [2^16, 2^32) by moving 16-bit words.            */
/*    Readings (the page is silent; all listed in the design notes):   */
/*    frequencies by the rule of oracle_rans_freqs; 32 interleaved      */
/*    coders per tile in the order of oracle_rans_encode; tiles of      */
/*    tile_symbols symbols.                                             */
/* ------------------------------------------------------------------ */

#define ORACLE_RANS_BITS 12
#define ORACLE_RANS_M (1u << ORACLE_RANS_BITS)
#define ORACLE_RANS_L 65536u
#define ORACLE_RANS_LANES 32

/* Quantized frequencies summing to M = 2^12: a present symbol s gets
 * max(1, floor(count_s * M / total)); the shortfall is then given one unit
 * at a time to the present symbols in order of decreasing count (smaller
 * symbol first on ties), cycling, and an excess taken one unit at a time in
 * the same order from symbols above 1.  Absent symbols get 0. */
int oracle_rans_freqs(const uint64_t *counts, int nsym, uint32_t *freqs)
{
    uint64_t total = 0;
    int order[256], present = 0;
    for (int s = 0; s < nsym; s++) {
        freqs[s] = 0;
        total += counts[s];
        if (counts[s]) order[present++] = s;
    }
    if (present == 0) return ORACLE_OK;
    /* order: count descending, symbol ascending (insertion sort) */
    for (int i = 1; i < present; i++) {
        int s = order[i], j = i - 1;
        while (j >= 0 && (counts[order[j]] < counts[s] ||
                          (counts[order[j]] == counts[s] && order[j] > s))) {
            order[j + 1] = order[j];
            j--;
        }
        order[j + 1] = s;
    }
    long long sum = 0;
    for (int i = 0; i < present; i++) {
        int s = order[i];
        uint64_t f = counts[s] * (uint64_t)ORACLE_RANS_M / total;
        if (f < 1) f = 1;
        freqs[s] = (uint32_t)f;
        sum += (long long)f;
    }
    long long d = (long long)ORACLE_RANS_M - sum;
    for (int i = 0; d > 0; i++, d--) freqs[order[i % present]]++;
    for (int i = 0; d < 0; i++) {
        int s = order[i % present];
        if (freqs[s] > 1) {
            freqs[s]--;
            d++;
        }
    }
    return ORACLE_OK;
}

/* Tiles of tile_symbols symbols (the last one shorter), each coded by 32
 * interleaved coders: coder j takes the tile's symbols j, j + 32, j + 64, ...
 * Decoding runs steps k = 0, 1, ... and in each step coders j = 0..31 in
 * turn: coder j decodes symbol 32k + j (when the tile has it), then, if its
 * state fell below 2^16, appends the tile's next 16-bit word below it.  The
 * encoder runs that order backwards from states 2^16, moving a word out
 * before a symbol whenever the state would leave [2^16, 2^32), and reverses
 * the words it wrote.  Each tile's words start at a multiple of 8 words
 * (zero padding between tiles).  Outputs: words; states[t * 32 + j] =
 * coder j's final encoder state (its initial decoder state); tile_words
 * (n_tiles + 1 offsets in words, the last one the padded total). */
int oracle_rans_encode(const uint8_t *exps, uint64_t n, const uint32_t *freqs, int nsym,
                       uint32_t tile_symbols, uint16_t *words, uint64_t words_cap,
                       uint32_t *states, uint64_t *tile_words)
{
    uint32_t cum[257];
    if (n == 0) { /* no symbol: no table needed */
        tile_words[0] = 0;
        return ORACLE_OK;
    }
    cum[0] = 0;
    for (int s = 0; s < nsym; s++) cum[s + 1] = cum[s] + freqs[s];
    if (nsym < 1 || cum[nsym] != ORACLE_RANS_M || tile_symbols == 0 || tile_symbols % ORACLE_RANS_LANES)
        return ORACLE_EINVAL;
    uint64_t n_tiles = (n + tile_symbols - 1) / tile_symbols;
    uint16_t *tmp = (uint16_t *)malloc((size_t)tile_symbols * sizeof(uint16_t));
    if (!tmp) return ORACLE_ENOMEM;
    uint64_t pos = 0;
    for (uint64_t t = 0; t < n_tiles; t++) {
        uint64_t base = t * tile_symbols;
        uint64_t m = n - base < tile_symbols ? n - base : tile_symbols;
        uint32_t x[ORACLE_RANS_LANES];
        for (int j = 0; j < ORACLE_RANS_LANES; j++) x[j] = ORACLE_RANS_L;
        uint64_t nw = 0;
        uint64_t steps = (m + ORACLE_RANS_LANES - 1) / ORACLE_RANS_LANES;
        for (uint64_t k = steps; k-- > 0;) {
            for (int j = ORACLE_RANS_LANES - 1; j >= 0; j--) {
                uint64_t p = k * ORACLE_RANS_LANES + (uint64_t)j;
                if (p >= m) continue;
                int s = exps[base + p];
                if (s >= nsym || freqs[s] == 0) { free(tmp); return ORACLE_EINVAL; }
                uint32_t f = freqs[s];
                /* after coding, x' < 2^32 needs x < f * 2^20 */
                if ((uint64_t)x[j] >= ((uint64_t)f << (32 - ORACLE_RANS_BITS))) {
                    tmp[nw++] = (uint16_t)(x[j] & 0xFFFFu);
                    x[j] >>= 16;
                }
                x[j] = (x[j] / f) * ORACLE_RANS_M + (x[j] % f) + cum[s];
            }
        }
        tile_words[t] = pos;
        if (pos + nw + 8 > words_cap) { free(tmp); return ORACLE_EINVAL; }
        for (uint64_t i = 0; i < nw; i++) words[pos + i] = tmp[nw - 1 - i];
        pos += nw;
        while (pos % 8) words[pos++] = 0;
        for (int j = 0; j < ORACLE_RANS_LANES; j++) states[t * ORACLE_RANS_LANES + (uint64_t)j] = x[j];
    }
    tile_words[n_tiles] = pos;
    free(tmp);
    return ORACLE_OK;
}

/* Words a tile of tile_symbols symbols can need at most: one per symbol,
 * plus the padding. */
uint64_t oracle_rans_words_bound(uint64_t n, uint32_t tile_symbols)
{
    uint64_t n_tiles = (n + tile_symbols - 1) / tile_symbols;
    return n + 8 * n_tiles + 8;
}

/* The decoder in the order the encoder defines (steps, then coders).  Every
 * coder must end in state 2^16 having read only its tile's words (the rest
 * of the tile's range being padding): ORACLE_ECORRUPT otherwise. */
int oracle_rans_decode(const uint16_t *words, const uint32_t *states, const uint64_t *tile_words,
                       uint64_t n, const uint32_t *freqs, int nsym, uint32_t tile_symbols,
                       uint8_t *exps_out)
{
    uint32_t cum[257];
    uint8_t sym[ORACLE_RANS_M];
    if (n == 0) return ORACLE_OK;
    cum[0] = 0;
    for (int s = 0; s < nsym; s++) cum[s + 1] = cum[s] + freqs[s];
    if (nsym < 1 || cum[nsym] != ORACLE_RANS_M || tile_symbols == 0 || tile_symbols % ORACLE_RANS_LANES)
        return ORACLE_EINVAL;
    for (int s = 0; s < nsym; s++)
        for (uint32_t v = cum[s]; v < cum[s + 1]; v++) sym[v] = (uint8_t)s;
    uint64_t n_tiles = (n + tile_symbols - 1) / tile_symbols;
    for (uint64_t t = 0; t < n_tiles; t++) {
        uint64_t base = t * tile_symbols;
        uint64_t m = n - base < tile_symbols ? n - base : tile_symbols;
        uint32_t x[ORACLE_RANS_LANES];
        for (int j = 0; j < ORACLE_RANS_LANES; j++) x[j] = states[t * ORACLE_RANS_LANES + (uint64_t)j];
        uint64_t ptr = tile_words[t], end = tile_words[t + 1];
        uint64_t steps = (m + ORACLE_RANS_LANES - 1) / ORACLE_RANS_LANES;
        for (uint64_t k = 0; k < steps; k++) {
            for (int j = 0; j < ORACLE_RANS_LANES; j++) {
                uint64_t p = k * ORACLE_RANS_LANES + (uint64_t)j;
                if (p >= m) continue;
                uint32_t slot = x[j] & (ORACLE_RANS_M - 1);
                int s = sym[slot];
                x[j] = freqs[s] * (x[j] >> ORACLE_RANS_BITS) + slot - cum[s];
                if (x[j] < ORACLE_RANS_L) {
                    if (ptr >= end) return ORACLE_ECORRUPT;
                    x[j] = (x[j] << 16) | words[ptr++];
                }
                exps_out[base + p] = (uint8_t)s;
            }
        }
        for (int j = 0; j < ORACLE_RANS_LANES; j++)
            if (x[j] != ORACLE_RANS_L) return ORACLE_ECORRUPT;
        if (end - ptr >= 8) return ORACLE_ECORRUPT;
    }
    return ORACLE_OK;
}
