// Decode kernel: compressed exponent stream + sign|fraction bytes -> BF16.
//
// The pages fix what decoding restores (mlx-dfloat, PyPI page, intro: the
// exponent code is undone and the raw sign|fraction byte put back, bit for bit)
// and that it runs blockwise on the GPU (mlx-dfloat, "Status"; df11pack, intro).
// The layout of the work below is this library's own, written for sm_100a.
//
// A CUDA block is 8 independent warps that share one staged copy of the
// current tensor's wide table (10-bit multi-code table: the codes that lie
// wholly inside a 10-bit window, their start mask, bits used and exponents).
// Each warp decodes a whole format block (T chunks of C stream bytes) on its
// own, T/32 sub-rounds of 32 chunks, one chunk per lane:
//   1. the lane's chunk is staged in the warp's shared memory as big-endian
//      words at an odd word stride (no bank conflicts between lanes)
//   2. one decode pass over the chunk, from chunk start + gap to the chunk end:
//      the window comes from a 64-bit register bit buffer refilled a word at a
//      time; each table step yields up to 4 codes whose exponents go to the
//      lane's own word-aligned region with 32-bit stores; codes longer than
//      10 bits walk the 8-bit-indexed tables
//   3. a warp scan of the code counts gives each lane's output position
//   4. an owner map names, for every group of 16 outputs, the lane whose region
//      holds its first exponent
//   5. merge: per group, 16 exponents gathered from one or two regions, one
//      16-byte load of sign|fraction bytes, two 16-byte BF16 stores; the last,
//      incomplete group of a sub-round is carried (in registers) into the next
// No block-wide barrier is taken except when the CTA's warps move to another
// tensor and the shared table is restaged; a warp whose block belongs to a
// tensor other than the staged one reads that tensor's table from global
// memory instead.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstring>
#include <vector>

#include "df_internal.h"

namespace df {
namespace {

constexpr uint32_t kWideN = 1u << kWideBits;
constexpr uint32_t kWarpsPerCta = 8;
constexpr uint32_t kCtaThreads = 32 * kWarpsPerCta;
constexpr uint32_t kFull = 0xFFFFFFFFu;
constexpr uint32_t kPosBytes = 176;  // scan positions (33 words) and two carry slots (8 words)

struct SingleSrc {
    DevTensor t;
    // the tensor holding global block g, and its block range [lo, hi)
    __device__ __forceinline__ const DevTensor* find(uint64_t g, uint64_t* lo, uint64_t* hi) const {
        *lo = 0;
        *hi = t.n_blocks;
        return &t;
    }
};

struct BatchSrc {
    const DevTensor* tensors;
    const uint64_t* block_start;  // count+1 prefix sums of n_blocks
    uint32_t count;
    __device__ __forceinline__ const DevTensor* find(uint64_t g, uint64_t* lo, uint64_t* hi) const {
        uint32_t a = 0, z = count;  // block_start[a] <= g < block_start[z]
        while (z - a > 1) {
            const uint32_t mid = (a + z) >> 1;
            if (block_start[mid] <= g)
                a = mid;
            else
                z = mid;
        }
        *lo = block_start[a];
        *hi = block_start[a + 1];
        return tensors + a;
    }
};

struct LaunchCfg {
    uint32_t words_per_chunk;  // shared-memory words of a chunk slot (odd)
    uint32_t region_bytes;     // exponent region of a lane (4 * odd)
    uint32_t owner_bytes;      // owner map of a warp (one byte per 16-output group)
    uint32_t warp_bytes;       // shared memory of one warp
    uint64_t total_blocks;
};

// Per-warp shared memory: chunk slots, scan positions, owner map, regions.
struct WarpArea {
    uint32_t* words;
    uint32_t* pos;  // 33 entries: each lane's first stage position, then the end;
                    // entries 36-43: two slots for a carried group's exponents
    uint8_t* owner;
    uint8_t* priv;  // 32 regions of region_bytes, then slack for over-reads
};

__device__ __forceinline__ uint32_t bswap32(uint32_t x) { return __byte_perm(x, 0, 0x0123); }

// Codes longer than the wide window: walk the 8-bit-indexed tables (global
// memory, cached). Returns the leaf (exponent bits 0-7, length bits 8-13,
// count 1 in bits 24-25) or 0 for a bit pattern no code starts with.
__device__ __noinline__ uint32_t long_code(uint32_t win, const uint32_t* __restrict__ hier) {
    uint32_t e = __ldg(hier + (win >> 24));
#pragma unroll 1
    for (int lvl = 1; lvl <= 3; ++lvl) {
        if ((e >> kNsymShift) & 3u) return e;
        const uint32_t t = e & 0xFFFFu;
        if (t == 0) return 0;
        e = __ldg(hier + static_cast<size_t>(t) * 256 + ((win >> (24 - 8 * lvl)) & 0xFFu));
    }
    return ((e >> kNsymShift) & 3u) ? e : 0;
}

__device__ __forceinline__ uint32_t warp_incl_scan(uint32_t v, uint32_t lane) {
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const uint32_t u = __shfl_up_sync(kFull, v, d);
        if (lane >= static_cast<uint32_t>(d)) v += u;
    }
    return v;
}

// 16 bytes of shared memory from byte address base + a (any alignment).
__device__ __forceinline__ void gather16(const uint8_t* base, int a, uint32_t e[4]) {
    const uint32_t* w = reinterpret_cast<const uint32_t*>(base + (a & ~3));
    const uint32_t sh = 8 * (a & 3);
    const uint32_t w0 = w[0], w1 = w[1], w2 = w[2], w3 = w[3], w4 = w[4];
    e[0] = __funnelshift_r(w0, w1, sh);
    e[1] = __funnelshift_r(w1, w2, sh);
    e[2] = __funnelshift_r(w2, w3, sh);
    e[3] = __funnelshift_r(w3, w4, sh);
}

// e := the first k bytes of lo, then the rest of hi (k = 0..16)
__device__ __forceinline__ void take_bytes(uint32_t e[4], const uint32_t lo[4], const uint32_t hi[4], uint32_t k) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int sbits = 8 * static_cast<int>(k) - 32 * i;
        const uint32_t m = sbits >= 32 ? 0xFFFFFFFFu : (sbits <= 0 ? 0u : (1u << sbits) - 1u);
        e[i] = (lo[i] & m) | (hi[i] & ~m);
    }
}

// 4 BF16 weights from 4 sign|fraction bytes and 4 exponent bytes: the high
// byte of weight k is s | e >> 1, the low byte (e & 1) << 7 | fraction.
__device__ __forceinline__ void merge4(uint32_t s, uint32_t e, uint32_t* o0, uint32_t* o1) {
    const uint32_t hi = (s & 0x80808080u) | ((e >> 1) & 0x7F7F7F7Fu);
    const uint32_t lo = ((e << 7) & 0x80808080u) | (s & 0x7F7F7F7Fu);
    *o0 = __byte_perm(lo, hi, 0x5140);
    *o1 = __byte_perm(lo, hi, 0x7362);
}

struct SmemTable {
    const uint64_t* w;
    __device__ __forceinline__ uint64_t operator()(uint32_t i) const { return w[i]; }
};
struct GlobalTable {
    const uint64_t* w;
    __device__ __forceinline__ uint64_t operator()(uint32_t i) const { return __ldg(w + i); }
};

// Decoder of one lane's chunk.
struct Lane {
    uint64_t buf;   // the next stream bits, left-aligned
    uint32_t nb;    // valid bits in buf (>= 32 before every step)
    uint32_t nw;    // the next word to append
    uint32_t wi;    // index of nw in the chunk slot
    uint32_t p;     // bit position in the chunk
    uint32_t end;   // codes must start before this bit
    uint32_t cnt;   // codes counted
    uint32_t app;   // exponents appended to the region (cnt, plus up to 3 past the end)
    uint64_t acc;   // exponents not yet stored, app & 3 of them
    bool bad;
};

// One wide-table step. kTail: the window may reach past the chunk end, so
// only the codes that start before it are counted.
template <bool kTail, class Tab>
__device__ __forceinline__ void decode_step(Lane& L, const uint32_t* words, const Tab& wide,
                                            const uint32_t* hier, uint32_t* region) {
    const uint32_t win = static_cast<uint32_t>(L.buf >> 32);
    const uint64_t e = wide(win >> (32 - kWideBits));
    uint32_t used = static_cast<uint32_t>(e >> kWideUsedShift) & 15u;
    uint32_t sy, ns, counted;
    if (used == 0) {  // a code longer than the window (or corrupt data)
        const uint32_t l = long_code(win, hier);
        ns = counted = (l >> kNsymShift) & 3u;
        used = (l >> 8) & 63u;
        sy = l & 0xFFu;
        if (ns == 0) {
            L.bad = true;
            L.end = L.p;
        }
    } else {
        sy = static_cast<uint32_t>(e);
        ns = static_cast<uint32_t>(e >> kWideCountShift) & 7u;
        counted = ns;
        if (kTail) {
            const uint32_t mask = static_cast<uint32_t>(e >> kWideMaskShift) & ((1u << kWideBits) - 1u);
            counted = __popc(mask & ((1u << (L.end - L.p)) - 1u));
        }
    }
    L.acc |= static_cast<uint64_t>(sy) << (8 * (L.app & 3u));
    const uint32_t na = L.app + ns;
    if ((na ^ L.app) & ~3u) {
        region[L.app >> 2] = static_cast<uint32_t>(L.acc);
        L.acc >>= 32;
    }
    L.app = na;
    L.cnt += counted;
    L.p += used;
    L.buf <<= used;
    L.nb -= used;
    if (L.nb < 32) {  // append the next word; fetch the one after
        L.buf |= static_cast<uint64_t>(L.nw) << (32 - L.nb);
        L.nb += 32;
        L.nw = words[++L.wi];
    }
}

// Decode format block b of tensor td with this warp.
template <class Tab>
__device__ __forceinline__ uint32_t decode_block(const DevTensor* __restrict__ td, uint64_t b, const Tab& wide,
                                                 const WarpArea& wa, uint32_t lane, const LaunchCfg& cfg) {
    const uint64_t out0 = td->offs[b];
    const uint64_t out1 = td->offs[b + 1];
    if (out1 < out0 || out1 > td->n || (b + 1 == td->n_blocks && out1 != td->n)) return DF_EFLAG_OFFSETS;
    const uint32_t C = td->chunk_bytes;
    const uint32_t wpc = C / 4 + 1;
    const uint32_t nsub = td->tpb / 32;
    const uint32_t RB = cfg.region_bytes;
    const uint32_t* hier = td->lut + kWideWords;
    const uint8_t* __restrict__ sm = td->sm;
    uint16_t* __restrict__ out = td->out;
    const bool vec = td->vec_ok != 0;
    uint32_t* my_words = wa.words + lane * wpc;
    uint32_t* my_region = reinterpret_cast<uint32_t*>(wa.priv + lane * RB);

    uint64_t rs = out0;  // first output of the sub-round
    bool have_carry = false;
    for (uint32_t k = 0; k < nsub; ++k) {
        const uint64_t first = b * td->tpb + 32ull * k;
        if (first >= td->n_chunks) break;
        const bool last_sub = k + 1 == nsub || first + 32 >= td->n_chunks;
        // 1. the lane's chunk
        const uint64_t chunk = first + lane;
        Lane L;
        L.p = L.end = L.cnt = L.app = 0;
        L.acc = 0;
        L.bad = false;
        if (chunk < td->n_chunks) {
            const uint4* c4 = reinterpret_cast<const uint4*>(td->stream + chunk * C);
            for (uint32_t q = 0; q < C / 16; ++q) {
                const uint4 v = __ldg(c4 + q);
                my_words[4 * q + 0] = bswap32(v.x);
                my_words[4 * q + 1] = bswap32(v.y);
                my_words[4 * q + 2] = bswap32(v.z);
                my_words[4 * q + 3] = bswap32(v.w);
            }
            my_words[C / 4] = bswap32(__ldg(reinterpret_cast<const uint32_t*>(td->stream + (chunk + 1) * C)));
            const uint64_t q = 5 * chunk;
            const uint32_t two = (static_cast<uint32_t>(__ldg(td->gaps + (q >> 3))) << 8) |
                                 __ldg(td->gaps + (q >> 3) + 1);
            const uint32_t cbits = 8 * C;
            const uint64_t bit0 = chunk * cbits;
            const uint64_t rem = td->total_bits > bit0 ? td->total_bits - bit0 : 0;
            L.p = (two >> (11 - (q & 7))) & 31u;
            L.end = static_cast<uint32_t>(rem < cbits ? rem : cbits);
        }
        __syncwarp();
        // 2. decode into the region: the bit buffer starts at bit p of word 0
        L.buf = ((static_cast<uint64_t>(my_words[0]) << 32) | my_words[1]) << L.p;
        L.nb = 64 - L.p;
        L.wi = 2;
        L.nw = my_words[2];
        for (;;) {  // two whole windows per vote
            const bool act = L.p + 2 * kWideBits <= L.end;
            if (!__any_sync(kFull, act)) break;
            if (act) {
                decode_step<false>(L, my_words, wide, hier, my_region);
                // a long code may have moved p past the second window
                if (L.p + kWideBits <= L.end) decode_step<false>(L, my_words, wide, hier, my_region);
            }
        }
        for (;;) {  // whole windows
            const bool act = L.p + kWideBits <= L.end;
            if (!__any_sync(kFull, act)) break;
            if (act) decode_step<false>(L, my_words, wide, hier, my_region);
        }
        for (;;) {  // windows reaching past the end
            const bool act = L.p < L.end;
            if (!__any_sync(kFull, act)) break;
            if (act) decode_step<true>(L, my_words, wide, hier, my_region);
        }
        my_region[L.app >> 2] = static_cast<uint32_t>(L.acc);
        my_region[(L.app >> 2) + 1] = static_cast<uint32_t>(L.acc >> 32);
        const uint32_t cnt = L.cnt;

        // 3. warp scan
        const uint32_t incl = warp_incl_scan(cnt, lane);
        const uint32_t total = __shfl_sync(kFull, incl, 31);
        if (__any_sync(kFull, L.bad)) return DF_EFLAG_BAD_CODE;
        const uint64_t re = rs + total;
        if (re > out1) return DF_EFLAG_COUNT;
        const uint32_t align = static_cast<uint32_t>(rs & 15);
        const uint32_t pos = align + incl - cnt;
        wa.pos[lane] = pos;
        if (lane == 31) wa.pos[32] = pos + cnt;
        const uint32_t ngroups = (align + total + 15) >> 4;
        if (ngroups * 1u > cfg.owner_bytes) return DF_EFLAG_COUNT;

        // 4. owner map: group gi (stage positions [16gi, 16gi+16)) belongs to
        // the lane whose range holds max(16gi, align)
        if (cnt) {
            const uint32_t hi = pos + cnt;
            if (pos <= align && align < hi) wa.owner[0] = static_cast<uint8_t>(lane);
            for (uint32_t gi = max((pos + 15) >> 4, 1u); 16 * gi < hi; ++gi) wa.owner[gi] = static_cast<uint8_t>(lane);
        }
        if (total == 0 && lane == 0) wa.owner[0] = 0;
        __syncwarp();

        // 5. merge and store
        const uint64_t gbase = rs & ~15ull;
        const uint32_t vend = align + total;  // decoded stage positions are [align, vend)
        const uint64_t g_last = gbase + 16ull * (ngroups - 1);
        const bool carry_out = ngroups > 0 && !last_sub && g_last + 16 > re;
        for (uint32_t gi = lane; gi < ngroups; gi += 32) {
            const uint64_t G = gbase + 16ull * gi;
            const uint32_t c0 = 16 * gi;
            uint32_t t = wa.owner[gi];
            const uint32_t vlo = max(c0, align), vhi = min(c0 + 16, vend);
            uint32_t e[4];
            const uint32_t b1 = wa.pos[t + 1];
            if (vhi <= b1) {  // one region
                gather16(wa.priv, static_cast<int>(t * RB + c0) - static_cast<int>(wa.pos[t]), e);
            } else if (t + 1 < 32 && vhi <= wa.pos[t + 2]) {  // two regions
                uint32_t x[4], y[4];
                gather16(wa.priv, static_cast<int>(t * RB + c0) - static_cast<int>(wa.pos[t]), x);
                gather16(wa.priv, static_cast<int>((t + 1) * RB) - static_cast<int>(b1 - c0), y);
                take_bytes(e, x, y, b1 - c0);
            } else {  // three or more: one exponent at a time
                e[0] = e[1] = e[2] = e[3] = 0;
                for (uint32_t c = vlo; c < vhi; ++c) {
                    while (c >= wa.pos[t + 1]) ++t;
                    const uint32_t byte = wa.priv[t * RB + (c - wa.pos[t])];
                    e[(c - c0) >> 2] |= byte << (8 * ((c - c0) & 3));
                }
            }
            if (gi == 0 && have_carry) {  // the slot the previous sub-round wrote
                const uint32_t* cin = wa.pos + 36 + 4 * (k & 1);
                const uint32_t cw[4] = {cin[0], cin[1], cin[2], cin[3]};
                take_bytes(e, cw, e, align);
            }
            if (carry_out && G == g_last) {  // completed by the next sub-round
                uint32_t* cout = wa.pos + 36 + 4 * ((k + 1) & 1);
                cout[0] = e[0];
                cout[1] = e[1];
                cout[2] = e[2];
                cout[3] = e[3];
                continue;
            }
            const uint64_t slo = max(G, out0), shi = min(G + 16, re);
            uint4 s16 = make_uint4(0, 0, 0, 0);
            const bool whole_sm = vec && G + 16 <= td->n;
            if (whole_sm) {
                s16 = __ldg(reinterpret_cast<const uint4*>(sm + G));
            } else {
                uint32_t sw[4] = {0, 0, 0, 0};
                for (uint64_t i = slo; i < shi; ++i) sw[(i - G) >> 2] |= static_cast<uint32_t>(sm[i]) << (8 * ((i - G) & 3));
                s16 = make_uint4(sw[0], sw[1], sw[2], sw[3]);
            }
            uint32_t o[8];
            merge4(s16.x, e[0], &o[0], &o[1]);
            merge4(s16.y, e[1], &o[2], &o[3]);
            merge4(s16.z, e[2], &o[4], &o[5]);
            merge4(s16.w, e[3], &o[6], &o[7]);
            if (vec && slo == G && shi == G + 16) {
                uint4* dst = reinterpret_cast<uint4*>(out + G);
                dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
                dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
            } else {
#pragma unroll
                for (uint32_t q = 0; q < 16; ++q)
                    if (G + q >= slo && G + q < shi) out[G + q] = static_cast<uint16_t>(o[q >> 1] >> (16 * (q & 1)));
            }
        }
        have_carry = carry_out;
        __syncwarp();  // the next sub-round overwrites the slots, regions and map
        rs = re;
    }
    return rs == out1 ? 0u : DF_EFLAG_COUNT;
}

// The staged table's header check: 1 if `lut` was built for this descriptor
// and its codes fit the launch's regions.
__device__ __forceinline__ uint32_t tables_ok(const DevTensor* td, const LaunchCfg& cfg) {
    const uint32_t* hdr = td->lut + kWideWords + static_cast<size_t>(td->n_tables) * 256 + 64;
    const uint32_t minl = __ldg(hdr);
    return __ldg(hdr + 3) == kLutMagic && __ldg(hdr + 2) == td->n_tables && minl >= 1 &&
           (8 * td->chunk_bytes + minl - 1) / minl + 12 <= cfg.region_bytes;
}

template <class Src>
__global__ void __launch_bounds__(kCtaThreads, 4) decode_kernel(const __grid_constant__ Src src, const LaunchCfg cfg,
                                                               uint32_t* d_err) {
    extern __shared__ __align__(16) uint8_t smem[];
    const uint32_t lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint64_t* s_wide = reinterpret_cast<uint64_t*>(smem);
    uint32_t* s_hdr = reinterpret_cast<uint32_t*>(smem + 8 * kWideN);
    uint8_t* area = smem + 8 * kWideN + 16 + warp * cfg.warp_bytes;
    WarpArea wa;
    wa.words = reinterpret_cast<uint32_t*>(area);
    const uint32_t slot_bytes = (32 * cfg.words_per_chunk + 4) * 4;
    wa.pos = reinterpret_cast<uint32_t*>(area + slot_bytes);
    wa.owner = area + slot_bytes + kPosBytes;
    wa.priv = area + slot_bytes + kPosBytes + cfg.owner_bytes;

    const DevTensor* staged = nullptr;
    const DevTensor* rtd = nullptr;  // tensor of the round's first block
    const DevTensor* td = nullptr;   // tensor of this warp's block
    uint64_t rlo = 0, rhi = 0, lo = 0, hi = 0;
    uint32_t flags = 0;
    const uint64_t stride = static_cast<uint64_t>(gridDim.x) * kWarpsPerCta;
    for (uint64_t r0 = static_cast<uint64_t>(blockIdx.x) * kWarpsPerCta; r0 < cfg.total_blocks; r0 += stride) {
        if (r0 < rlo || r0 >= rhi) rtd = src.find(r0, &rlo, &rhi);
        if (rtd != staged) {  // restage the shared table (all warps take this branch together)
            __syncthreads();
            const uint4* t4 = reinterpret_cast<const uint4*>(rtd->lut);
            uint4* d4 = reinterpret_cast<uint4*>(smem);
            for (uint32_t i = threadIdx.x; i < kWideWords / 4; i += kCtaThreads) d4[i] = __ldg(t4 + i);
            if (threadIdx.x == 0) s_hdr[0] = tables_ok(rtd, cfg);
            __syncthreads();
            staged = rtd;
        }
        const uint64_t g = r0 + warp;
        if (g >= cfg.total_blocks) continue;
        if (g < lo || g >= hi) td = src.find(g, &lo, &hi);
        if (td == staged) {
            if (s_hdr[0])
                flags |= decode_block(td, g - lo, SmemTable{s_wide}, wa, lane, cfg);
            else
                flags |= DF_EFLAG_TABLES;
        } else {
            if (tables_ok(td, cfg))
                flags |= decode_block(td, g - lo, GlobalTable{reinterpret_cast<const uint64_t*>(td->lut)}, wa, lane,
                                      cfg);
            else
                flags |= DF_EFLAG_TABLES;
        }
        __syncwarp();
    }
    if (flags && lane == 0 && d_err) atomicOr(d_err, flags);
}

struct Prepared {
    DevTensor dev;
    uint32_t words_per_chunk, region_bytes, owner_bytes;
};

uint32_t min_len_of(const uint8_t* lengths) {
    uint32_t m = 0;
    for (int s = 0; s < 256; ++s)
        if (lengths[s] && (!m || lengths[s] < m)) m = lengths[s];
    return m;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

// Validate a descriptor and fill the device-side copy and the shared-memory
// needs of its blocks.
df_status prepare(const df_tensor* t, uint16_t* out, Prepared* pr) {
    if (!t || !out) return DF_ERR_INVALID_ARG;
    const uint32_t C = t->chunk_bytes, T = t->threads_per_block;
    if (C < 16 || C > 4096 || C % 16 || T < 32 || T > 1024 || T % 32) return DF_ERR_INVALID_ARG;
    if (t->max_len < 1 || t->max_len > 32 || t->n_tables < 1) return DF_ERR_INVALID_ARG;
    if (t->n > DF_MAX_WEIGHTS) return DF_ERR_UNSUPPORTED;
    if (!t->stream || !t->gaps || !t->block_offsets || !t->sm || !t->lut) return DF_ERR_INVALID_ARG;
    if (!aligned(t->stream, 16) || !aligned(t->lut, 16) || !aligned(t->block_offsets, 8) || !aligned(out, 2))
        return DF_ERR_INVALID_ARG;
    const uint32_t minl = min_len_of(t->lengths);
    if (t->n > 0 && minl == 0) return DF_ERR_INVALID_ARG;
    for (int s = 0; s < 256; ++s)
        if (t->lengths[s] > t->max_len) return DF_ERR_INVALID_ARG;
    const uint64_t cbits = 8ull * C;
    const uint64_t n_chunks = t->total_bits ? (t->total_bits + cbits - 1) / cbits : 1;
    const uint64_t n_blocks = (n_chunks + T - 1) / T;
    if (n_blocks > 0xFFFFFFFFull) return DF_ERR_UNSUPPORTED;
    DevTensor d;
    std::memset(&d, 0, sizeof(d));
    d.stream = t->stream;
    d.gaps = t->gaps;
    d.offs = t->block_offsets;
    d.sm = t->sm;
    d.lut = t->lut;
    d.out = out;
    d.n = t->n;
    d.total_bits = t->total_bits;
    d.n_chunks = n_chunks;
    d.n_blocks = static_cast<uint32_t>(n_blocks);
    d.n_tables = t->n_tables;
    d.chunk_bytes = C;
    d.tpb = T;
    d.vec_ok = aligned(t->sm, 16) && aligned(out, 16);
    pr->dev = d;
    pr->words_per_chunk = C / 4 + 1;  // odd: C is a multiple of 16
    // a chunk holds at most 8C/min_len code starts; its region also takes up
    // to 3 exponents past the last counted code and the final two-word flush
    const uint64_t per_chunk = (cbits + minl - 1) / (minl ? minl : 1);
    uint64_t rb = (per_chunk + 12 + 3) & ~3ull;
    if (((rb / 4) & 1) == 0) rb += 4;  // odd word stride: regions start in distinct banks
    // one owner entry per 16 outputs of a sub-round (32 chunks), plus the
    // partial groups at both ends
    const uint64_t groups = (32 * per_chunk + 15 + 15) / 16 + 1;
    if (rb > (1u << 16) || groups > (1u << 16)) return DF_ERR_UNSUPPORTED;
    pr->region_bytes = static_cast<uint32_t>(rb);
    pr->owner_bytes = static_cast<uint32_t>((groups + 15) & ~15ull);
    return DF_OK;
}

uint32_t warp_bytes(const LaunchCfg& c) {
    // chunk slots (+4 words read ahead by the last lane), scan positions,
    // owner map, regions, slack for 16-byte reads past the last region
    return ((32 * c.words_per_chunk + 4) * 4 + kPosBytes + c.owner_bytes + 32 * c.region_bytes + 32 + 15) & ~15u;
}

size_t smem_bytes(const LaunchCfg& c) { return 8u * kWideN + 16 + static_cast<size_t>(kWarpsPerCta) * c.warp_bytes; }

df_status device_limits(int* sms, int* max_smem) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e);
    e = cudaDeviceGetAttribute(sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return cuda_fail(e);
    e = cudaDeviceGetAttribute(max_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    if (e != cudaSuccess) return cuda_fail(e);
    return DF_OK;
}

template <class Src>
df_status launch(const Src& src, const LaunchCfg& cfg, size_t smem, uint32_t* d_err, cudaStream_t stream) {
    if (cfg.total_blocks == 0) return DF_OK;
    int sms = 0, max_smem = 0;
    df_status st = device_limits(&sms, &max_smem);
    if (st != DF_OK) return st;
    if (smem > static_cast<size_t>(max_smem)) return DF_ERR_UNSUPPORTED;
    auto kern = decode_kernel<Src>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return cuda_fail(e);
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, static_cast<int>(kCtaThreads), smem);
    if (e != cudaSuccess) return cuda_fail(e);
    if (per_sm < 1) return DF_ERR_UNSUPPORTED;
    // persistent blocks: every resident slot loops over rounds of 8 format blocks
    const uint64_t rounds = (cfg.total_blocks + kWarpsPerCta - 1) / kWarpsPerCta;
    const uint64_t slots = static_cast<uint64_t>(sms) * per_sm;
    const uint64_t grid = rounds < slots ? rounds : slots;
    kern<<<static_cast<unsigned>(grid), kCtaThreads, smem, stream>>>(src, cfg, d_err);
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e);
    return DF_OK;
}

void widen(LaunchCfg* c, const Prepared& p) {
    c->words_per_chunk = std::max(c->words_per_chunk, p.words_per_chunk);
    c->region_bytes = std::max(c->region_bytes, p.region_bytes);
    c->owner_bytes = std::max(c->owner_bytes, p.owner_bytes);
    c->warp_bytes = warp_bytes(*c);
}

}  // namespace
}  // namespace df

using namespace df;

extern "C" {

df_status df_decode(const df_tensor* t, uint16_t* d_out, uint32_t* d_err, void* stream) {
    if (!t) return DF_ERR_INVALID_ARG;
    if (t->n == 0) return DF_OK;
    Prepared pr;
    df_status st = prepare(t, d_out, &pr);
    if (st != DF_OK) return st;
    SingleSrc src{pr.dev};
    LaunchCfg cfg;
    std::memset(&cfg, 0, sizeof(cfg));
    widen(&cfg, pr);
    cfg.total_blocks = pr.dev.n_blocks;
    return launch(src, cfg, smem_bytes(cfg), d_err, static_cast<cudaStream_t>(stream));
}

size_t df_decode_batch_workspace(uint32_t count) {
    return (static_cast<size_t>(count) * sizeof(DevTensor) + 255) / 256 * 256 + (static_cast<size_t>(count) + 1) * 8;
}

df_status df_decode_batch_prepare(const df_tensor* tensors, uint16_t* const* d_outs, uint32_t count, void* d_ws,
                                  size_t ws_bytes, df_batch_plan* plan, void* stream) {
    if (!plan || (count && (!tensors || !d_outs))) return DF_ERR_INVALID_ARG;
    std::memset(plan, 0, sizeof(*plan));
    if (count && !d_ws) return DF_ERR_INVALID_ARG;
    if (ws_bytes < df_decode_batch_workspace(count)) return DF_ERR_WORKSPACE;
    if (!aligned(d_ws, 16)) return DF_ERR_INVALID_ARG;
    std::vector<DevTensor> dev;
    std::vector<uint64_t> start(1, 0);
    dev.reserve(count);
    LaunchCfg cfg;
    std::memset(&cfg, 0, sizeof(cfg));
    for (uint32_t i = 0; i < count; ++i) {
        const df_tensor* t = tensors + i;
        if (t->n == 0) continue;
        Prepared pr;
        df_status st = prepare(t, d_outs[i], &pr);
        if (st != DF_OK) return st;
        widen(&cfg, pr);
        dev.push_back(pr.dev);
        start.push_back(start.back() + pr.dev.n_blocks);
    }
    plan->d_ws = d_ws;
    plan->count = static_cast<uint32_t>(dev.size());
    plan->threads_per_block = kCtaThreads;
    plan->words_per_chunk = cfg.words_per_chunk;
    plan->region_bytes = cfg.region_bytes;
    plan->max_groups = cfg.owner_bytes;
    plan->total_blocks = start.back();
    if (plan->count == 0) return DF_OK;
    const size_t sm = smem_bytes(cfg);
    int sms = 0, max_smem = 0;
    df_status st = device_limits(&sms, &max_smem);
    if (st != DF_OK) return st;
    if (sm > static_cast<size_t>(max_smem)) return DF_ERR_UNSUPPORTED;
    plan->smem_bytes = static_cast<uint32_t>(sm);
    // layout: the live descriptors (rounded up to 256 bytes), then the block
    // prefix sums. Copies from pageable host memory return once the source has
    // been staged, so the host vectors may die on return.
    const size_t table_bytes = (dev.size() * sizeof(DevTensor) + 255) / 256 * 256;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemcpyAsync(d_ws, dev.data(), dev.size() * sizeof(DevTensor), cudaMemcpyHostToDevice, s);
    if (e != cudaSuccess) return cuda_fail(e);
    e = cudaMemcpyAsync(static_cast<uint8_t*>(d_ws) + table_bytes, start.data(), start.size() * 8,
                        cudaMemcpyHostToDevice, s);
    if (e != cudaSuccess) return cuda_fail(e);
    return DF_OK;
}

df_status df_decode_batch_run(const df_batch_plan* plan, uint32_t* d_err, void* stream) {
    if (!plan) return DF_ERR_INVALID_ARG;
    if (plan->count == 0) return DF_OK;
    if (!plan->d_ws) return DF_ERR_INVALID_ARG;
    BatchSrc src;  // same layout as df_decode_batch_prepare writes
    src.tensors = static_cast<const DevTensor*>(plan->d_ws);
    src.count = plan->count;
    const size_t table_bytes = (static_cast<size_t>(plan->count) * sizeof(DevTensor) + 255) / 256 * 256;
    src.block_start = reinterpret_cast<const uint64_t*>(static_cast<const uint8_t*>(plan->d_ws) + table_bytes);
    LaunchCfg cfg;
    std::memset(&cfg, 0, sizeof(cfg));
    cfg.words_per_chunk = plan->words_per_chunk;
    cfg.region_bytes = plan->region_bytes;
    cfg.owner_bytes = plan->max_groups;
    cfg.warp_bytes = warp_bytes(cfg);
    cfg.total_blocks = plan->total_blocks;
    if (smem_bytes(cfg) != plan->smem_bytes) return DF_ERR_INVALID_ARG;
    return launch(src, cfg, plan->smem_bytes, d_err, static_cast<cudaStream_t>(stream));
}

df_status df_decode_batch(const df_tensor* tensors, uint16_t* const* d_outs, uint32_t count, void* d_ws,
                          size_t ws_bytes, uint32_t* d_err, void* stream) {
    df_batch_plan plan;
    df_status st = df_decode_batch_prepare(tensors, d_outs, count, d_ws, ws_bytes, &plan, stream);
    if (st != DF_OK) return st;
    return df_decode_batch_run(&plan, d_err, stream);
}

df_status df_read_error(const uint32_t* d_err, void* stream, uint32_t* flags) {
    if (!d_err) return DF_ERR_INVALID_ARG;
    uint32_t h = 0;
    cudaError_t e = cudaMemcpyAsync(&h, d_err, 4, cudaMemcpyDeviceToHost, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e);
    e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e);
    if (flags) *flags = h;
    return h ? DF_ERR_CORRUPT : DF_OK;
}

}  // extern "C"
