// Host half of the library: code construction, decode-table derivation,
// container size planning, status strings.
//
// The code is an optimal length-limited prefix code over the exponents
// (package-merge, Larmore and Hirschberg 1990), made canonical. The pages fix
// only that the codebook is built deterministically from the exponent
// frequencies (df11pack, GitHub page: intro and "Licence") and that codes have
// a maximum length (mlx-dfloat, PyPI page: "Try it", the "max-code" group);
// the tie rule below makes the build deterministic.
#include <algorithm>
#include <cstring>
#include <vector>

#include "df_internal.h"

namespace df {

static thread_local int g_last_cuda_error = 0;

df_status cuda_fail(cudaError_t e) {
    g_last_cuda_error = static_cast<int>(e);
    return DF_ERR_CUDA;
}

namespace {

// Package-merge in its array form. Level j (1..L) keeps one weight per entry
// and whether the entry is a package. The 2k-2 cheapest entries of level 1 are
// selected; going down the levels, a selected prefix holds the first `items`
// original items (each gains one bit of length) and the first `pk` packages,
// which stand for the first 2*pk entries of the level below.
// Ties: items sorted by (frequency, symbol); an item precedes a package of
// equal weight.
bool package_merge(const uint64_t hist[256], uint32_t max_len, uint8_t lengths[256]) {
    std::memset(lengths, 0, 256);
    std::vector<int> sym;
    for (int s = 0; s < 256; ++s)
        if (hist[s]) sym.push_back(s);
    std::stable_sort(sym.begin(), sym.end(), [&](int a, int b) { return hist[a] < hist[b]; });
    const size_t k = sym.size();
    if (k == 0) return true;
    if (k == 1) {
        lengths[sym[0]] = 1;
        return true;
    }
    if (max_len < 1 || max_len > 32 || k > (1ull << max_len)) return false;

    std::vector<uint64_t> item_w(k);
    for (size_t i = 0; i < k; ++i) item_w[i] = hist[sym[i]];

    // level L is the items alone; build levels L-1 .. 1
    std::vector<std::vector<uint64_t>> w(max_len + 1);
    std::vector<std::vector<uint8_t>> is_pkg(max_len + 1);
    w[max_len] = item_w;
    is_pkg[max_len].assign(k, 0);
    for (uint32_t lvl = max_len - 1; lvl >= 1; --lvl) {
        const std::vector<uint64_t>& below = w[lvl + 1];
        const size_t npk = below.size() / 2;
        std::vector<uint64_t>& cw = w[lvl];
        std::vector<uint8_t>& cp = is_pkg[lvl];
        cw.reserve(k + npk);
        cp.reserve(k + npk);
        size_t i = 0, p = 0;
        while (i < k || p < npk) {
            const uint64_t pw = p < npk ? below[2 * p] + below[2 * p + 1] : 0;
            if (p >= npk || (i < k && item_w[i] <= pw)) {
                cw.push_back(item_w[i++]);
                cp.push_back(0);
            } else {
                cw.push_back(pw);
                cp.push_back(1);
                ++p;
            }
        }
        if (lvl == 1) break;
    }
    // walk the selection down the levels
    std::vector<uint32_t> len(k, 0);
    size_t take = 2 * k - 2;
    for (uint32_t lvl = 1; lvl <= max_len && take > 0; ++lvl) {
        size_t items = 0, pk = 0;
        for (size_t e = 0; e < take; ++e) (is_pkg[lvl][e] ? pk : items)++;
        for (size_t i = 0; i < items; ++i) len[i]++;
        take = 2 * pk;
    }
    for (size_t i = 0; i < k; ++i) lengths[sym[i]] = static_cast<uint8_t>(len[i]);
    return true;
}

// Canonical codes: in (length, symbol) order, each code is the previous one
// plus one, shifted left by the growth in length. Computed per length: the
// first code of length l is (first code of length l-1 + codes of length l-1)
// shifted left once, and codes of one length go to symbols in increasing order.
void canonical(const uint8_t lengths[256], uint32_t codes[256]) {
    std::memset(codes, 0, 256 * sizeof(uint32_t));
    uint32_t bl_count[34] = {0};
    for (int s = 0; s < 256; ++s)
        if (lengths[s]) bl_count[lengths[s]]++;
    uint64_t next[34] = {0};
    for (int l = 2; l <= 32; ++l) next[l] = (next[l - 1] + bl_count[l - 1]) << 1;
    for (int s = 0; s < 256; ++s)
        if (lengths[s]) codes[s] = static_cast<uint32_t>(next[lengths[s]]++);
}

bool valid_format(uint32_t chunk_bytes, uint32_t tpb) {
    return chunk_bytes >= 16 && chunk_bytes <= 4096 && chunk_bytes % 16 == 0 && tpb >= 32 && tpb <= 1024 &&
           tpb % 32 == 0;
}

}  // namespace
}  // namespace df

using namespace df;

extern "C" {

const char* df_status_string(df_status s) {
    switch (s) {
    case DF_OK: return "DF_OK";
    case DF_ERR_INVALID_ARG: return "DF_ERR_INVALID_ARG";
    case DF_ERR_CUDA: return "DF_ERR_CUDA";
    case DF_ERR_CORRUPT: return "DF_ERR_CORRUPT";
    case DF_ERR_UNSUPPORTED: return "DF_ERR_UNSUPPORTED";
    case DF_ERR_WORKSPACE: return "DF_ERR_WORKSPACE";
    default: return "DF_ERR_UNKNOWN";
    }
}

int df_last_cuda_error(void) { return g_last_cuda_error; }

df_status df_code_from_lengths(const uint8_t lengths[256], uint32_t max_len, df_code* out) {
    if (!lengths || !out) return DF_ERR_INVALID_ARG;
    if (max_len < 1 || max_len > 32) return DF_ERR_UNSUPPORTED;
    df_code c;
    std::memset(&c, 0, sizeof(c));
    c.max_len = max_len;
    uint64_t kraft = 0;  // sum of 2^(32-l): at most 2^32 for a prefix code
    for (int s = 0; s < 256; ++s) {
        const uint32_t l = lengths[s];
        if (l > max_len) return DF_ERR_INVALID_ARG;
        c.lengths[s] = static_cast<uint8_t>(l);
        if (!l) continue;
        kraft += 1ull << (32 - l);
        c.n_symbols++;
        if (!c.min_len || l < c.min_len) c.min_len = l;
    }
    if (kraft > (1ull << 32)) return DF_ERR_INVALID_ARG;
    canonical(c.lengths, c.codes);
    // decode tables: one root plus one per distinct prefix of 8, 16 and 24
    // bits shared by codes longer than that prefix
    std::vector<uint64_t> prefixes;
    for (int s = 0; s < 256; ++s)
        for (uint32_t lvl = 1; lvl <= 3; ++lvl)
            if (c.lengths[s] > 8 * lvl) {
                const uint32_t l = c.lengths[s];
                prefixes.push_back((static_cast<uint64_t>(lvl) << 40) | (c.codes[s] >> (l - 8 * lvl)));
            }
    std::sort(prefixes.begin(), prefixes.end());
    c.n_tables = 1 + static_cast<uint32_t>(std::unique(prefixes.begin(), prefixes.end()) - prefixes.begin());
    *out = c;
    return DF_OK;
}

df_status df_build_code(const uint64_t hist[256], uint32_t max_len, df_code* out) {
    if (!hist || !out) return DF_ERR_INVALID_ARG;
    if (max_len < 1 || max_len > 32) return DF_ERR_UNSUPPORTED;
    uint8_t lengths[256];
    if (!package_merge(hist, max_len, lengths)) return DF_ERR_UNSUPPORTED;
    return df_code_from_lengths(lengths, max_len, out);
}

size_t df_lut_words(const df_code* code) {
    return code ? kWideWords + static_cast<size_t>(code->n_tables) * 256 + 64 + 4 : 0;
}

df_status df_build_lut(const df_code* code, uint32_t* lut, size_t lut_words) {
    if (!code || !lut || code->n_tables < 1 || lut_words < df_lut_words(code)) return DF_ERR_INVALID_ARG;
    const size_t words = df_lut_words(code);
    std::memset(lut, 0, words * sizeof(uint32_t));

    // 1. the 8-bit-indexed tables, one code per entry (the long-code path)
    std::vector<uint32_t> tables(static_cast<size_t>(code->n_tables) * 256, 0);
    uint32_t next_table = 1;
    for (int s = 0; s < 256; ++s) {
        const uint32_t l = code->lengths[s];
        if (!l) continue;
        if (l > 32) return DF_ERR_INVALID_ARG;
        const uint32_t c = code->codes[s];
        uint32_t t = 0, rem = l;
        while (rem > 8) {
            const uint32_t idx = (c >> (rem - 8)) & 0xFFu;
            uint32_t& e = tables[static_cast<size_t>(t) * 256 + idx];
            if (e == 0) {
                if (next_table >= code->n_tables) return DF_ERR_INVALID_ARG;
                e = next_table;  // count 0: a link to the next level
                ++next_table;
            } else if ((e >> kNsymShift) & 3u) {
                return DF_ERR_INVALID_ARG;  // a shorter code is a prefix of this one
            }
            t = e & 0xFFFFu;
            rem -= 8;
        }
        const uint32_t low = c & ((1u << rem) - 1u);
        const uint32_t lo = low << (8 - rem), hi = (low + 1) << (8 - rem);
        for (uint32_t x = lo; x < hi; ++x) {
            uint32_t& e = tables[static_cast<size_t>(t) * 256 + x];
            if (e != 0) return DF_ERR_INVALID_ARG;
            e = sub_leaf(static_cast<uint32_t>(s), l);
        }
    }
    uint32_t* hier = lut + kWideWords;
    std::memcpy(hier, tables.data(), tables.size() * sizeof(uint32_t));
    uint32_t* tail = lut + kWideWords + static_cast<size_t>(code->n_tables) * 256;
    std::memcpy(tail, code->lengths, 256);
    uint32_t min_len = 0;
    for (int s = 0; s < 256; ++s)
        if (code->lengths[s] && (!min_len || code->lengths[s] < min_len)) min_len = code->lengths[s];
    tail[64] = min_len;  // header: the shortest code, which bounds the codes per chunk
    tail[65] = code->max_len;
    tail[66] = code->n_tables;
    tail[67] = kLutMagic;

    // 2. the wide table: for every kWideBits-bit window, the codes that lie
    // wholly inside it from its first bit on (at most kWideMaxCodes)
    const uint32_t W = kWideBits, N = 1u << W;
    std::vector<uint32_t> first(N, 0);  // (len << 8) | symbol of the code at bit 0, if len <= W
    for (int s = 0; s < 256; ++s) {
        const uint32_t l = code->lengths[s];
        if (!l || l > W) continue;
        const uint32_t c = code->codes[s];
        for (uint32_t x = c << (W - l); x < ((c + 1) << (W - l)); ++x) first[x] = (l << 8) | static_cast<uint32_t>(s);
    }
    uint64_t* wide = reinterpret_cast<uint64_t*>(lut);
    uint16_t* wide_mask = reinterpret_cast<uint16_t*>(lut + kWideEntryWords);
    for (uint32_t x = 0; x < N; ++x) {
        uint32_t used = 0, n = 0, mask = 0, syms = 0;
        while (n < kWideMaxCodes && used < W) {
            const uint32_t e = first[(x << used) & (N - 1)];  // the unknown low bits read as 0
            const uint32_t l = e >> 8;
            if (!l || l > W - used) break;  // this code needs bits beyond the window
            mask |= 1u << used;
            syms |= (e & 0xFFu) << (8 * n);
            used += l;
            ++n;
        }
        const uint32_t step = used ? (used << kStepShift) | (n << kStepCountShift) : 0u;
        wide[x] = syms | (static_cast<uint64_t>(step) << 32);
        wide_mask[x] = static_cast<uint16_t>(mask);
    }
    return DF_OK;
}

df_status df_container_sizes(uint64_t n, uint64_t total_bits, uint32_t chunk_bytes, uint32_t tpb,
                             df_sizes* out) {
    if (!out || !valid_format(chunk_bytes, tpb)) return DF_ERR_INVALID_ARG;
    if (n > DF_MAX_WEIGHTS) return DF_ERR_UNSUPPORTED;
    // every code is at least one bit and at most 32 bits long
    if (total_bits > 32 * n || (n && total_bits < n)) return DF_ERR_INVALID_ARG;
    df_sizes z;
    std::memset(&z, 0, sizeof(z));
    const uint64_t cbits = 8ull * chunk_bytes;
    z.total_bits = total_bits;
    z.n_chunks = total_bits ? (total_bits + cbits - 1) / cbits : 1;
    z.stream_bytes = z.n_chunks * chunk_bytes + 16;
    const uint64_t field_bytes = (5 * z.n_chunks + 7) / 8;
    z.gap_bytes = (field_bytes + 1 + 15) & ~15ull;
    z.n_blocks = (z.n_chunks + tpb - 1) / tpb;
    z.offsets_bytes = 8 * (z.n_blocks + 1);
    z.sm_bytes = n;
    z.container_bytes = z.stream_bytes + z.gap_bytes + z.offsets_bytes + z.sm_bytes + 256 + 64;
    // encode workspace: per-tile bit counts and bases (tiles of 4096 weights)
    const uint64_t tiles = (n + 4095) / 4096;
    z.encode_ws_bytes = 16 * (tiles + 2) + 256;
    *out = z;
    return DF_OK;
}

df_status df_plan(const df_code* code, const uint64_t hist[256], uint64_t n, uint32_t chunk_bytes,
                  uint32_t tpb, df_sizes* out) {
    if (!code || !hist || !out || !valid_format(chunk_bytes, tpb)) return DF_ERR_INVALID_ARG;
    if (n > DF_MAX_WEIGHTS) return DF_ERR_UNSUPPORTED;
    uint64_t total = 0, bits = 0;
    for (int s = 0; s < 256; ++s) {
        if (hist[s] && !code->lengths[s]) return DF_ERR_INVALID_ARG;
        total += hist[s];
        bits += hist[s] * code->lengths[s];
    }
    if (total != n) return DF_ERR_INVALID_ARG;
    return df_container_sizes(n, bits, chunk_bytes, tpb, out);
}

}  // extern "C"
