/*
 * CPU oracle for exponent-Huffman BF16 weight compression.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing in the product library calls, links or
 * includes this file; only the tests, the smoke check and the benchmark's CPU
 * baseline use it. It shares no source with the CUDA library: it is a plain,
 * slow, single-threaded restatement of what the method computes, written so a
 * reader can check each step against the pages by eye.
 *
 * What the pages fix, and where:
 *   - mlx-dfloat (PyPI page), intro and its bit diagram: a BF16 weight is
 *     s | eeeeeeee | mmmmmmm; the 8 exponent bits are replaced by a
 *     variable-length code and the sign and fraction are kept as one raw byte;
 *     the result is bit for bit the original.
 *   - df11pack (GitHub page), intro and "Licence": the codebook is built
 *     deterministically from the exponent frequencies.
 *   - mlx-dfloat, "Try it": codes have a maximum length (the "max-code" group).
 *   - df11pack, "What is checked" (--luts=correct, --index idx8) and "Use"
 *     (chunks, units): lookup tables, a block index and independently
 *     decodable chunks exist.
 * What the pages leave open (the Huffman variant, the length limit, the bit
 * order, the chunk size, the gap and index encodings) is fixed by this
 * library's own container layout; each reading is stated where it is used.
 *
 * Steps, in order:
 *   1 split, 2 histogram, 3 code lengths by package-merge, 4 canonical codes,
 *   5 MSB-first bitstream, 6 chunk gaps, 7 block offsets, 8 bit-serial decode,
 *   9 size accounting.
 *
 * Parity pins (tests): Kraft equality, the length limit, brute-force
 * optimality on tiny alphabets, equality with a heap Huffman when the limit
 * does not bind, dyadic and uniform closed forms, the entropy bound, round
 * trips over all 65,536 BF16 patterns, and gap/offset re-derivation from the
 * decoder's own code positions. Parity unpinned: the compression ratio on
 * real model weights (no real weights are available).
 */
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_OK 0
#define ORACLE_EINVAL (-1)
#define ORACLE_ECORRUPT (-2)
#define ORACLE_ENOMEM (-3)

#define HEADER_BYTES 64u /* fixed per-tensor header of the container */

/* ---- 1. split (mlx-dfloat, intro bit diagram) --------------------------- */

static uint8_t exponent_of(uint16_t w) { return (uint8_t)((w >> 7) & 0xFFu); }
static uint8_t sign_mantissa_of(uint16_t w) { return (uint8_t)(((w >> 8) & 0x80u) | (w & 0x7Fu)); }
static uint16_t join(uint8_t e, uint8_t sm) {
    return (uint16_t)(((uint32_t)(sm & 0x80u) << 8) | ((uint32_t)e << 7) | (sm & 0x7Fu));
}

void oracle_split(const uint16_t* w, uint64_t n, uint8_t* e, uint8_t* sm) {
    for (uint64_t i = 0; i < n; ++i) {
        e[i] = exponent_of(w[i]);
        sm[i] = sign_mantissa_of(w[i]);
    }
}

void oracle_join(const uint8_t* e, const uint8_t* sm, uint64_t n, uint16_t* w) {
    for (uint64_t i = 0; i < n; ++i) w[i] = join(e[i], sm[i]);
}

/* ---- 2. histogram ----------------------------------------------------------
 * Counts of each exponent value: the frequencies the codebook is built from
 * (df11pack, GitHub page, intro and "Licence").
 */

void oracle_histogram(const uint16_t* w, uint64_t n, uint64_t hist[256]) {
    for (int s = 0; s < 256; ++s) hist[s] = 0;
    for (uint64_t i = 0; i < n; ++i) hist[exponent_of(w[i])]++;
}

/* ---- 3. code lengths: package-merge (Larmore and Hirschberg, 1990) -------
 *
 * Optimal prefix code with no length above max_len. Each list entry carries,
 * for every symbol, how many of that symbol's coins it holds; an original item
 * holds one coin of its own symbol, a package the coins of the two entries it
 * joins. A symbol's code length is the number of its coins among the 2k-2
 * cheapest entries of the final list.
 *
 * Tie rules (this library's reading, the pages give none): items are sorted by
 * (frequency, symbol); a merge is stable and puts an item before a package of
 * equal weight. Special cases: no symbol -> no code; one symbol -> length 1
 * (code "0").
 */
typedef struct {
    uint64_t weight;
    uint8_t coins[256];
} pm_entry;

static void sort_items(const uint64_t hist[256], int* sym, int* k_out) {
    int k = 0;
    for (int s = 0; s < 256; ++s)
        if (hist[s] > 0) sym[k++] = s;
    /* insertion sort by (frequency, symbol): plain and stable */
    for (int i = 1; i < k; ++i) {
        int v = sym[i], j = i - 1;
        while (j >= 0 && (hist[sym[j]] > hist[v] || (hist[sym[j]] == hist[v] && sym[j] > v))) {
            sym[j + 1] = sym[j];
            --j;
        }
        sym[j + 1] = v;
    }
    *k_out = k;
}

int oracle_package_merge(const uint64_t hist[256], int max_len, uint8_t lengths[256]) {
    int sym[256], k;
    for (int s = 0; s < 256; ++s) lengths[s] = 0;
    if (max_len < 1 || max_len > 32) return ORACLE_EINVAL;
    sort_items(hist, sym, &k);
    if (k == 0) return ORACLE_OK;
    if (k == 1) {
        lengths[sym[0]] = 1;
        return ORACLE_OK;
    }
    if ((uint64_t)k > (1ull << max_len)) return ORACLE_EINVAL;

    pm_entry* items = (pm_entry*)calloc((size_t)k, sizeof(pm_entry));
    pm_entry* prev = (pm_entry*)calloc((size_t)(2 * k), sizeof(pm_entry));
    pm_entry* cur = (pm_entry*)calloc((size_t)(2 * k), sizeof(pm_entry));
    if (!items || !prev || !cur) {
        free(items), free(prev), free(cur);
        return ORACLE_ENOMEM;
    }
    for (int i = 0; i < k; ++i) {
        items[i].weight = hist[sym[i]];
        items[i].coins[sym[i]] = 1;
    }
    /* list at level max_len: the items */
    int prev_len = k;
    memcpy(prev, items, (size_t)k * sizeof(pm_entry));

    for (int level = max_len - 1; level >= 1; --level) {
        /* packages from pairs of consecutive entries of the previous list */
        int n_pkg = prev_len / 2;
        pm_entry* pkg = (pm_entry*)calloc((size_t)(n_pkg > 0 ? n_pkg : 1), sizeof(pm_entry));
        if (!pkg) {
            free(items), free(prev), free(cur);
            return ORACLE_ENOMEM;
        }
        for (int p = 0; p < n_pkg; ++p) {
            pkg[p].weight = prev[2 * p].weight + prev[2 * p + 1].weight;
            for (int s = 0; s < 256; ++s)
                pkg[p].coins[s] = (uint8_t)(prev[2 * p].coins[s] + prev[2 * p + 1].coins[s]);
        }
        /* stable merge with the items; an item goes first on equal weight */
        int i = 0, p = 0, o = 0;
        while (i < k || p < n_pkg) {
            if (p >= n_pkg || (i < k && items[i].weight <= pkg[p].weight))
                cur[o++] = items[i++];
            else
                cur[o++] = pkg[p++];
        }
        free(pkg);
        pm_entry* t = prev;
        prev = cur;
        cur = t;
        prev_len = o;
    }
    /* the 2k-2 cheapest entries of the final list */
    for (int e = 0; e < 2 * k - 2; ++e)
        for (int s = 0; s < 256; ++s) lengths[s] = (uint8_t)(lengths[s] + prev[e].coins[s]);
    free(items), free(prev), free(cur);
    return ORACLE_OK;
}

/* ---- 4. canonical codes ---------------------------------------------------
 * Symbols sorted by (length, symbol); the first gets code 0, each next one
 * code = (previous code + 1) << (its length - previous length). The pages
 * require a deterministic codebook (df11pack, intro and "Licence") but do not
 * say how codes are assigned to lengths; canonical order is this library's
 * reading.
 */
void oracle_canonical_codes(const uint8_t lengths[256], uint32_t codes[256]) {
    int order[256], k = 0;
    for (int s = 0; s < 256; ++s) {
        codes[s] = 0;
        if (lengths[s] > 0) order[k++] = s;
    }
    for (int i = 1; i < k; ++i) { /* insertion sort by (length, symbol) */
        int v = order[i], j = i - 1;
        while (j >= 0 && (lengths[order[j]] > lengths[v] || (lengths[order[j]] == lengths[v] && order[j] > v))) {
            order[j + 1] = order[j];
            --j;
        }
        order[j + 1] = v;
    }
    uint64_t code = 0;
    for (int i = 0; i < k; ++i) {
        if (i > 0) code = (code + 1) << (lengths[order[i]] - lengths[order[i - 1]]);
        codes[order[i]] = (uint32_t)code;
    }
}

/* ---- 9. size accounting ----------------------------------------------------
 * The pages give only the outcome, about 70% of the BF16 size (mlx-dfloat,
 * PyPI page, intro; df11pack, intro). Container layout (this library's own;
 * the pages do not give one):
 *   stream   n_chunks * C bytes of MSB-first code bits, then 16 zero bytes
 *   gaps     5 bits per chunk, MSB-first, then zero padding: at least one
 *            byte, up to a multiple of 16
 *   offsets  (n_blocks + 1) little-endian uint64
 *   sm       n bytes, one sign|fraction byte per weight
 *   lengths  256 bytes; header 64 bytes
 * with n_chunks = max(1, ceil(total_bits / 8C)) and n_blocks = ceil(n_chunks / T).
 */
typedef struct {
    uint64_t total_bits, n_chunks, stream_bytes, gap_bytes, n_blocks, offsets_bytes, sm_bytes, container_bytes;
} oracle_sizes_t;

int oracle_sizes(uint64_t n, uint64_t total_bits, uint32_t chunk_bytes, uint32_t threads_per_block,
                 oracle_sizes_t* out) {
    if (chunk_bytes == 0 || threads_per_block == 0) return ORACLE_EINVAL;
    uint64_t chunk_bits = 8ull * chunk_bytes;
    out->total_bits = total_bits;
    out->n_chunks = total_bits == 0 ? 1 : (total_bits + chunk_bits - 1) / chunk_bits;
    out->stream_bytes = out->n_chunks * chunk_bytes + 16;
    out->gap_bytes = ((5 * out->n_chunks + 7) / 8 + 1 + 15) / 16 * 16;
    out->n_blocks = (out->n_chunks + threads_per_block - 1) / threads_per_block;
    out->offsets_bytes = 8 * (out->n_blocks + 1);
    out->sm_bytes = n;
    out->container_bytes =
        out->stream_bytes + out->gap_bytes + out->offsets_bytes + out->sm_bytes + 256 + HEADER_BYTES;
    return ORACLE_OK;
}

uint64_t oracle_total_bits(const uint64_t hist[256], const uint8_t lengths[256]) {
    uint64_t t = 0;
    for (int s = 0; s < 256; ++s) t += hist[s] * lengths[s];
    return t;
}

/* ---- 6/7. chunk gaps and block offsets from code start positions ----------
 * The pages name independently decodable chunks / units (df11pack, "Use") and
 * a block index (df11pack, "What is checked", --index idx8) without their
 * encoding. A code belongs to the chunk that holds its first bit. gap[j] is the distance
 * from the chunk's first bit 8Cj to the first code start at or after it; when
 * no code starts in the chunk (possible only in the last one), the end of the
 * stream, total_bits, counts as that start (this library's reading: it lets a
 * decoder begin at chunk start + gap and stop at once). offsets[b] is the
 * number of codes that start before bit 8C*T*b, and offsets[n_blocks] = n.
 */
typedef struct {
    uint64_t chunk_bits, n_chunks, next_chunk, T;
    uint8_t* gaps;      /* packed 5-bit fields (nullable) */
    uint64_t* offsets;  /* nullable */
} index_walk;

static void put_bits_msb(uint8_t* buf, uint64_t pos, uint32_t value, int nbits) {
    for (int b = nbits - 1; b >= 0; --b, ++pos)
        if ((value >> b) & 1u) buf[pos >> 3] |= (uint8_t)(0x80u >> (pos & 7));
}

static int get_bit_msb(const uint8_t* buf, uint64_t pos) { return (buf[pos >> 3] >> (7 - (pos & 7))) & 1; }

/* Called with every code start in increasing order (index i), then once with
 * the end of the stream (index n). */
static void index_visit(index_walk* wk, uint64_t start, uint64_t index) {
    while (wk->next_chunk < wk->n_chunks && wk->chunk_bits * wk->next_chunk <= start) {
        uint64_t j = wk->next_chunk;
        uint64_t gap = start - wk->chunk_bits * j;
        if (wk->gaps) put_bits_msb(wk->gaps, 5 * j, (uint32_t)gap, 5);
        if (wk->offsets && j % wk->T == 0) wk->offsets[j / wk->T] = index;
        wk->next_chunk++;
    }
}

/* ---- 5. encode --------------------------------------------------------------
 * The exponent byte of each weight is replaced by its variable-length code and
 * the sign|fraction byte is kept raw (mlx-dfloat, PyPI page, intro and its bit
 * diagram). For i = 0..n-1 append code[e_i] in len[e_i] bits, most
 * significant bit first; the first stream bit is bit 7 of byte 0 (the bit
 * order is this library's reading). Buffers are sized by
 * oracle_sizes and are zeroed here.
 */
int oracle_encode(const uint16_t* w, uint64_t n, const uint8_t lengths[256], const uint32_t codes[256],
                  uint32_t chunk_bytes, uint32_t threads_per_block, uint8_t* stream, uint8_t* gaps,
                  uint64_t* offsets, uint8_t* sm) {
    uint64_t hist[256];
    oracle_histogram(w, n, hist);
    for (int s = 0; s < 256; ++s)
        if (hist[s] > 0 && lengths[s] == 0) return ORACLE_EINVAL;
    oracle_sizes_t z;
    if (oracle_sizes(n, oracle_total_bits(hist, lengths), chunk_bytes, threads_per_block, &z) != ORACLE_OK)
        return ORACLE_EINVAL;
    memset(stream, 0, z.stream_bytes);
    memset(gaps, 0, z.gap_bytes);
    index_walk wk = {8ull * chunk_bytes, z.n_chunks, 0, threads_per_block, gaps, offsets};
    uint64_t pos = 0;
    for (uint64_t i = 0; i < n; ++i) {
        uint8_t e = exponent_of(w[i]);
        index_visit(&wk, pos, i);
        put_bits_msb(stream, pos, codes[e], lengths[e]);
        pos += lengths[e];
        sm[i] = sign_mantissa_of(w[i]);
    }
    index_visit(&wk, pos, n);
    offsets[z.n_blocks] = n;
    return ORACLE_OK;
}

/* ---- 8. bit-serial canonical decode ------------------------------------------
 * Decoding gives back the original bits exactly (mlx-dfloat, PyPI page, intro
 * and "Status"). One bit at a time from bit 0: code = code << 1 | bit; at length l the code is
 * complete when first[l] <= code < first[l] + count[l], and names symbol
 * sorted[base[l] + code - first[l]] (canonical decoding; no lookup tables).
 * Every code must end at or before total_bits, exactly n codes must be read
 * and they must use all total_bits bits; otherwise ORACLE_ECORRUPT. When gaps
 * or offsets are given, they are re-derived from the decoded code positions.
 */
int oracle_decode(const uint8_t* stream, uint64_t total_bits, const uint8_t* sm, uint64_t n,
                  const uint8_t lengths[256], uint32_t chunk_bytes, uint32_t threads_per_block, uint16_t* out,
                  uint8_t* gaps, uint64_t* offsets) {
    uint64_t count[34] = {0}, first[34] = {0}, base[34] = {0};
    int sorted[256], k = 0, max_l = 0;
    for (int l = 1; l <= 32; ++l)
        for (int s = 0; s < 256; ++s)
            if (lengths[s] == l) {
                sorted[k++] = s;
                count[l]++;
                if (l > max_l) max_l = l;
            }
    for (int s = 0; s < 256; ++s)
        if (lengths[s] > 32) return ORACLE_EINVAL;
    uint64_t idx = 0;
    for (int l = 1; l <= 32; ++l) {
        base[l] = idx;
        idx += count[l];
        first[l + 1] = (first[l] + count[l]) << 1;
    }
    oracle_sizes_t z;
    if (oracle_sizes(n, total_bits, chunk_bytes ? chunk_bytes : 32, threads_per_block ? threads_per_block : 256,
                     &z) != ORACLE_OK)
        return ORACLE_EINVAL;
    if (gaps) memset(gaps, 0, z.gap_bytes);
    index_walk wk = {8ull * (chunk_bytes ? chunk_bytes : 32), z.n_chunks, 0,
                     threads_per_block ? threads_per_block : 256, gaps, offsets};
    uint64_t pos = 0;
    for (uint64_t i = 0; i < n; ++i) {
        index_visit(&wk, pos, i);
        uint64_t code = 0;
        int sym = -1;
        for (int l = 1; l <= max_l; ++l) {
            if (pos >= total_bits) return ORACLE_ECORRUPT;
            code = (code << 1) | (uint64_t)get_bit_msb(stream, pos++);
            if (count[l] > 0 && code >= first[l] && code - first[l] < count[l]) {
                sym = sorted[base[l] + (code - first[l])];
                break;
            }
        }
        if (sym < 0) return ORACLE_ECORRUPT;
        out[i] = join((uint8_t)sym, sm[i]);
    }
    if (pos != total_bits) return ORACLE_ECORRUPT;
    index_visit(&wk, pos, n);
    if (offsets) offsets[z.n_blocks] = n;
    return ORACLE_OK;
}
