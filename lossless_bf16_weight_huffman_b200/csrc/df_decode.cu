// Decode kernel: compressed exponent stream + sign|fraction bytes -> BF16.
//
// The pages fix what decoding restores (mlx-dfloat, PyPI page, intro: the
// exponent code is undone and the raw sign|fraction byte put back, bit for bit)
// and that it runs blockwise on the GPU (mlx-dfloat, "Status"; df11pack, intro).
// The layout of the work below is this library's own, written for sm_100a.
//
// Every warp is an independent decoder: it owns a contiguous run of whole
// format blocks (T chunks of C stream bytes, one block index entry each:
// a uint64 offset, or the compact index's anchor, base and delta) of one
// tensor and streams through it in rounds of 32 chunks, one chunk per lane.
// Nothing a warp does waits for another warp, so a CUDA block only
// synchronises when its tensor changes (to restage the decode tables). A CUDA
// block loops over a contiguous range of the format blocks of all tensors of
// the launch (persistent blocks, one range each) and splits each tensor's part
// of it into one run per warp. Per round:
//   1. each lane's chunk (plus the next chunk's first word) sits byte-swapped
//      to big-endian words in the warp's slot area, word i of lane l at
//      i * 32 + l (the 32 lanes read 32 different banks wherever their windows
//      are); it was loaded into registers during the previous round
//   2. one decode pass per lane from chunk start + gap until the bit position
//      reaches the chunk end: a state word (bit position << 18) | (exponents
//      so far << 3) advances by one add per lookup of the wide table (the
//      exponents of up to 4 codes and their step word); the 32-bit window
//      comes from three stream words held in registers (one slot load per 32
//      bits consumed, off the lookup's critical path); the exponents go to
//      the lane's own shared-memory region, one 32-bit store per lookup; codes
//      longer than the window walk the 8-bit tables. The last lookup may take
//      codes that start past the chunk end (they belong to the next chunk):
//      the window's start mask says how many, and they are not counted.
//      Lane 0's region first holds the exponents of the 16-output group the
//      previous round left open, so every round starts on a group boundary
//   3. warp scan of the region sizes: every lane's first stage position
//   4. an owner map: for every group of 16 outputs, the lane whose region
//      holds its first exponent; then each lane completes the group its range
//      ends inside by copying the next lane's first 16 exponents into its
//      region's slack, so nearly every group lies in one region
//   5. merge: every group takes its 16 exponents from its owner's region;
//      one 16-byte load of sign|fraction bytes, two 16-byte stores. Groups
//      that could not be completed (short or full regions) gather from
//      several regions in a separate, rarely taken path. The round's last
//      group, if the round ends inside it, stays open for the next round;
//      only a run's first and last groups take element stores.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstring>
#include <vector>

#include "df_internal.h"

namespace df {
namespace {

constexpr uint32_t kWideN = 1u << kWideBits;
constexpr uint32_t kFull = 0xFFFFFFFFu;
constexpr uint32_t kLanes = 32;
constexpr uint32_t kMaxWarps = 32;   // CUDA blocks of up to 1024 threads
constexpr uint32_t kPosWords = 72;   // 33 stage positions, 3 spare, the 4-word carry, 32 region bases
constexpr uint32_t kCarryWord = 36;  // the carry's first word within them
constexpr uint32_t kBaseWord = 40;   // the first region base
constexpr uint32_t kRegionSlack = 12;  // up to 3 uncounted exponents and the word they end in
constexpr uint32_t kSmemSlack = 32;  // gathers may read a few bytes past the last region
// shared memory before the per-warp areas: the wide table, the current
// tensor's descriptor and the tables-valid flag
constexpr uint32_t kFixedBytes = 8u * kWideN + sizeof(DevTensor) + 16;

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
    uint32_t words_per_chunk;  // slot words of a lane (C / 4 + 1 for the widest C)
    uint32_t region_bytes;     // exponent region of a lane (4 * odd)
    uint32_t max_groups;       // owner-map entries of a round
    uint32_t warp_bytes;       // shared memory of one warp
    uint64_t total_blocks;
};

__device__ __forceinline__ uint32_t bswap32(uint32_t x) { return __byte_perm(x, 0, 0x0123); }

// Byte offset of lane t's exponent region from the start of the regions; lane
// 0's starts 16 bytes early, in the pad before them, because it also holds the
// exponents a round carries over to the next.
__device__ __forceinline__ int region_off(uint32_t t, uint32_t RB) {
    return static_cast<int>(t * RB) - (t == 0 ? 16 : 0);
}

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

// Compact block index (superblocks of 64 format blocks): codes in block b.
// A wide superblock's overflow slot past the wide count marks *bad.
__device__ __forceinline__ uint32_t idx8_count(const DevTensor* td, uint64_t b, bool* bad) {
    const uint64_t S = (static_cast<uint64_t>(td->n_blocks) + 63) >> 6;
    const uint8_t* ix = reinterpret_cast<const uint8_t*>(td->offs);
    const uint32_t w = __ldg(reinterpret_cast<const uint32_t*>(ix + 8 * S) + (b >> 6));
    if (!(w & 0x80000000u)) return w + __ldg(ix + 12 * S + b);
    const uint32_t slot = w & 0x7FFFFFFFu;
    if (slot + 1 >= td->idx8) {
        *bad = true;
        return 0;
    }
    return __ldg(reinterpret_cast<const uint32_t*>(ix + 76 * S) + 64ull * slot + (b & 63));
}

// Output index of block b's first code from the compact index: its
// superblock's anchor plus the counts of the blocks before it there (each
// lane adds two of them). Called by the whole warp.
__device__ __noinline__ uint64_t idx8_start(const DevTensor* td, uint64_t b, uint32_t lane, bool* bad) {
    const uint64_t s0 = b & ~63ull;
    bool bd = false;
    uint32_t c = 0;
    if (s0 + lane < b) c += idx8_count(td, s0 + lane, &bd);
    if (s0 + lane + 32 < b) c += idx8_count(td, s0 + lane + 32, &bd);
    const uint32_t sum = __reduce_add_sync(0xffffffffu, c);  // a valid superblock's counts sum below 2^29
    if (__any_sync(0xffffffffu, bd)) *bad = true;
    return __ldg(reinterpret_cast<const uint64_t*>(td->offs) + (b >> 6)) + sum;
}

__device__ __forceinline__ uint32_t warp_incl_scan(uint32_t v, uint32_t lane) {
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const uint32_t u = __shfl_up_sync(kFull, v, d);
        if (lane >= static_cast<uint32_t>(d)) v += u;
    }
    return v;
}

__device__ __forceinline__ uint16_t merge1(uint8_t sm, uint8_t e) {
    return static_cast<uint16_t>((static_cast<uint32_t>(sm & 0x80u) << 8) | (static_cast<uint32_t>(e) << 7) |
                                 (sm & 0x7Fu));
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

// 4 BF16 weights from 4 sign|fraction bytes and 4 exponent bytes: the high
// byte of weight k is s | e >> 1, the low byte (e & 1) << 7 | fraction.
// Bit select: the bits of a where m is set, the bits of b elsewhere (one
// three-input logic instruction).
__device__ __forceinline__ uint32_t bitsel(uint32_t a, uint32_t b, uint32_t m) {
    uint32_t d;
    asm("lop3.b32 %0, %1, %2, %3, 0xE4;" : "=r"(d) : "r"(a), "r"(b), "r"(m));
    return d;
}

__device__ __forceinline__ void merge4(uint32_t s, uint32_t e, uint32_t* o0, uint32_t* o1) {
    const uint32_t hi = bitsel(s, e >> 1, 0x80808080u);
    const uint32_t lo = bitsel(e << 7, s, 0x80808080u);
    *o0 = __byte_perm(lo, hi, 0x5140);
    *o1 = __byte_perm(lo, hi, 0x7362);
}

// 16 outputs from their 16 sign|fraction bytes and 16 exponents: two 16-byte
// stores, marked evict-first (the outputs are not read again by this kernel and
// should not push the stream and sign|fraction lines out of L2).
__device__ __forceinline__ void merge16(const uint4 s16, const uint32_t e[4], uint16_t* __restrict__ dst16) {
    uint32_t o[8];
    merge4(s16.x, e[0], &o[0], &o[1]);
    merge4(s16.y, e[1], &o[2], &o[3]);
    merge4(s16.z, e[2], &o[4], &o[5]);
    merge4(s16.w, e[3], &o[6], &o[7]);
    uint4* dst = reinterpret_cast<uint4*>(dst16);
    __stcs(dst, make_uint4(o[0], o[1], o[2], o[3]));
    __stcs(dst + 1, make_uint4(o[4], o[5], o[6], o[7]));
}

// Shared-memory accesses by 32-bit shared-window address.
__device__ __forceinline__ uint32_t lds32(uint32_t a) {
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a));
    return v;
}
__device__ __forceinline__ uint2 lds64(uint32_t a) {
    uint2 v;
    asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(a));
    return v;
}
__device__ __forceinline__ void sts32(uint32_t a, uint32_t v) {
    asm volatile("st.shared.u32 [%0], %1;" ::"r"(a), "r"(v) : "memory");
}
__device__ __forceinline__ uint32_t shared_addr(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// The 32 stream bits from bit p of a lane's chunk, whose big-endian words
// start at shared address wb, one word every 32 * 4 bytes.
__device__ __forceinline__ uint32_t window_at(uint32_t wb, uint32_t p) {
    const uint32_t a = wb + (p >> 5) * (kLanes * 4);
    return __funnelshift_l(lds32(a + kLanes * 4), lds32(a), p);
}

// Decoder state of one lane: st = (bit position << 18) | (exponents appended
// to the region << 3); acc holds the region word being filled (its
// (st & 24) / 8 low bytes are exponents) and wp is that word's address.
struct Lane {
    uint32_t st;
    uint32_t endst;  // codes must start before bit endst >> 18: st < endst
    uint32_t acc;
    uint32_t wp;
    uint32_t kw;          // c0, c1, c2: stream words kw, kw + 1, kw + 2 of the chunk
    uint32_t c0, c1, c2;  // (big-endian), so the window needs no shared load
    bool bad;
};

// Append the exponents of one lookup (step word w, exponents sy) to the
// lane's region. The region word being filled is stored on every lookup (a
// later store of the same word supersedes it), and the exponents that spill
// into the next word start the new accumulator. (st & 31) is the byte shift
// of the next exponent in its word, so the two funnel shifts place the new
// exponents without masking the state.
__device__ __forceinline__ void append(Lane& L, uint32_t w, uint32_t sy) {
    const uint32_t lo = L.acc | __funnelshift_l(0u, sy, L.st);
    const uint32_t hi = __funnelshift_l(sy, 0u, L.st);
    const uint32_t nst = L.st + w;
    sts32(L.wp, lo);
    // bit 5 of the state flips when the count enters the next region word
    const uint32_t d = (nst ^ L.st) & 32u;
    L.acc = __funnelshift_rc(lo, hi, d);
    L.wp += d >> 3;
    L.st = nst;
}

// One lookup at the lane's bit position: up to 4 codes from the wide table
// (at shared address tb), or one longer code from the 8-bit tables.
__device__ __forceinline__ void step(Lane& L, uint32_t wb, uint32_t tb, const uint32_t* hier) {
    const uint32_t p = L.st >> kStepShift;
    if ((p >> 5) != L.kw) {  // a lookup moves at most 32 bits: one word on
        L.c0 = L.c1;
        L.c1 = L.c2;
        L.kw += 1;
        // used two words from now; past the chunk's words this reads the
        // warp's position words, whose bits no lookup uses
        L.c2 = lds32(wb + (L.kw + 2) * (kLanes * 4));
    }
    const uint32_t win = __funnelshift_l(L.c1, L.c0, p);
    const uint2 e = lds64(tb + (win >> (32 - kWideBits)) * 8u);
    uint32_t sy = e.x, w = e.y;
    if (w == 0) {
        const uint32_t l = long_code(win, hier);
        sy = l & 0xFFu;
        w = l ? (((l >> 8) & 63u) << kStepShift) | (1u << kStepCountShift) : 0u;
        if (w == 0) {  // a bit pattern no code starts with
            L.bad = true;
            L.endst = 0;
        }
    }
    append(L, w, sy);
}

// Decode one lane's chunk (words at shared address wb) into its region
// (shared address region), appending to what the region already holds: st
// starts at (gap << 18) | (exponents already there << 3) and acc holds the
// bytes of the region's last, unfinished word. Returns the region's byte
// count with only the codes that start before the chunk end (bits
// endst >> 18; the exponents of codes past it are in the region too, after
// the counted ones), plus 1 << 31 for a bit pattern no code starts with.
// Kept out of line: the lookup loop then runs in a register set of its own
// instead of sharing one with the caller's bookkeeping.
__device__ __noinline__ uint32_t decode_chunk(uint32_t st, uint32_t endst, uint32_t acc, uint32_t wb,
                                              uint32_t region, uint32_t tb, const uint32_t* __restrict__ lut) {
    const uint32_t* hier = lut + kWideWords;
    Lane L;
    L.st = st;
    L.endst = endst;
    L.acc = acc;
    L.wp = region + ((st & kStepCountMask) >> 3 & ~3u);
    L.kw = st >> (kStepShift + 5);
    L.c0 = lds32(wb + L.kw * (kLanes * 4));
    L.c1 = lds32(wb + (L.kw + 1) * (kLanes * 4));
    L.c2 = lds32(wb + (L.kw + 2) * (kLanes * 4));
    L.bad = false;
    uint32_t prev = st;  // the state before the last lookup
    for (;;) {  // two lookups per vote
        const bool act = L.st < L.endst;
        if (!__any_sync(kFull, act)) break;
        if (act) {
            prev = L.st;
            step(L, wb, tb, hier);
            if (L.st < L.endst) {
                prev = L.st;
                step(L, wb, tb, hier);
            }
        }
    }
    sts32(L.wp, L.acc);  // the word being filled
    uint32_t cnt = (L.st & kStepCountMask) >> kStepCountShift;
    if (L.bad) return cnt | 0x80000000u;
    if (L.st != st) {  // every lookup advances the bit position
        // codes of the last lookup that start at or after the chunk end
        const uint32_t p = prev >> kStepShift;
        const uint32_t rel = (L.endst >> kStepShift) - p;
        if (rel < kWideBits) {
            const uint32_t x = window_at(wb, p) >> (32 - kWideBits);
            if (lds64(tb + x * 8u).y) {  // a wide-table lookup (a long code starts at p, before the end)
                const uint16_t* mask = reinterpret_cast<const uint16_t*>(lut + kWideEntryWords);
                cnt -= __popc(static_cast<uint32_t>(__ldg(mask + x)) >> rel);
            }
        }
    }
    return cnt;
}

template <class Src>
__global__ void __launch_bounds__(kMaxWarps * kLanes, 1)
    decode_kernel(const __grid_constant__ Src src, const LaunchCfg cfg, uint32_t* d_err) {
    extern __shared__ __align__(16) uint8_t smem[];
    const uint32_t tid = threadIdx.x;
    const uint32_t lane = tid & 31, warp = tid >> 5;
    const uint32_t nwarps = blockDim.x >> 5;

    // shared memory carve-up (sizes in warp_area_bytes())
    uint64_t* s_wide = reinterpret_cast<uint64_t*>(smem);
    DevTensor* s_td = reinterpret_cast<DevTensor*>(smem + 8u * kWideN);
    volatile uint32_t* s_ok = reinterpret_cast<uint32_t*>(s_td + 1);  // 1 when the tables fit the tensor
    uint8_t* wb = smem + kFixedBytes + static_cast<size_t>(warp) * cfg.warp_bytes;
    uint32_t* s_words = reinterpret_cast<uint32_t*>(wb);
    uint32_t* s_pos = s_words + kLanes * cfg.words_per_chunk;  // 33 stage positions
    uint32_t* s_carry = s_pos + kCarryWord;                     // 16 bytes: the group a round leaves open
    int* s_base = reinterpret_cast<int*>(s_pos + kBaseWord);    // per lane: region byte of stage position 0
    uint8_t* s_owner = reinterpret_cast<uint8_t*>(s_pos + kPosWords);
    // lane 0's region starts 16 bytes early: it holds up to 15 carried
    // exponents before its own
    uint8_t* s_priv = s_owner + ((cfg.max_groups + 15) & ~15u) + 16;
    const uint32_t RB = cfg.region_bytes;
    const int my_off = region_off(lane, RB);  // this lane's region, from s_priv
    uint32_t* my_words = s_words + lane;  // word i of this lane's chunk at my_words[i * 32]
    uint32_t* my_region = reinterpret_cast<uint32_t*>(s_priv + my_off);
    const DevTensor* const td = s_td;

    // each CUDA block takes a contiguous range of format blocks, so that it
    // changes tensors (and restages tables) as rarely as possible
    const uint64_t per = cfg.total_blocks / gridDim.x, extra = cfg.total_blocks % gridDim.x;
    const uint64_t g_begin = blockIdx.x * per + min(static_cast<uint64_t>(blockIdx.x), extra);
    const uint64_t g_end = g_begin + per + (blockIdx.x < extra ? 1 : 0);
    for (uint64_t g = g_begin; g < g_end;) {
        uint64_t t_lo, t_hi;
        const DevTensor* tg = src.find(g, &t_lo, &t_hi);
        const uint64_t seg_end = min(g_end, t_hi);
        // restage: every warp is done with the previous tensor's tables
        __syncthreads();
        if (tid < sizeof(DevTensor) / 4)
            reinterpret_cast<uint32_t*>(s_td)[tid] = reinterpret_cast<const uint32_t*>(tg)[tid];
        {
            const uint32_t* lut = tg->lut;
            const uint4* t4 = reinterpret_cast<const uint4*>(lut);
            uint4* d4 = reinterpret_cast<uint4*>(s_wide);
            for (uint32_t i = tid; i < kWideEntryWords / 4; i += blockDim.x) d4[i] = __ldg(t4 + i);
            if (tid == 0) {
                const uint32_t nt = tg->n_tables, C = tg->chunk_bytes;
                const uint32_t* hdr = lut + kWideWords + static_cast<size_t>(nt) * 256 + 64;
                const uint32_t minl = __ldg(hdr);
                // the region must hold every code the tables can yield in one chunk
                *s_ok = __ldg(hdr + 3) == kLutMagic && __ldg(hdr + 2) == nt && minl >= 1 &&
                        (8 * C + minl - 1) / minl + kRegionSlack <= RB && C / 4 + 1 <= cfg.words_per_chunk;
            }
        }
        __syncthreads();
        if (!*s_ok) {
            if (tid == 0 && d_err) atomicOr(d_err, DF_EFLAG_TABLES);
            g = seg_end;
            continue;
        }
        // this warp's run: a contiguous range of the segment's format blocks
        const uint64_t nb = seg_end - g;
        const uint64_t wb0 = g + nb * warp / nwarps, wb1 = g + nb * (warp + 1) / nwarps;
        g = seg_end;
        if (wb0 >= wb1) continue;
        const uint32_t T = td->tpb, C = td->chunk_bytes;
        const uint64_t n_chunks = td->n_chunks;
        const uint8_t* __restrict__ sm = td->sm;
        uint16_t* __restrict__ out = td->out;
        const bool vec = td->vec_ok != 0;
        uint64_t b = wb0 - t_lo;  // local index of the current block
        const uint64_t c_end = min((wb1 - t_lo) * T, n_chunks);
        uint64_t c = b * T;                 // first chunk of the current round
        bool bad_index = false;
        uint64_t outr = td->idx8 ? idx8_start(td, b, lane, &bad_index)  // output index of the round's first code
                                 : td->offs[b];
        const uint64_t vstart = outr;       // outputs before it belong to the previous run
        bool pre = false;      // this lane's chunk of the round is already in its slot
        uint32_t pre_two = 0;  // and its two gap bytes
        bool ok = outr <= td->n && !bad_index;
        if (!ok && lane == 0 && d_err) atomicOr(d_err, DF_EFLAG_OFFSETS);
        while (ok && c < c_end) {  // the run's blocks
            // a block starts where the one before ended (checked at its end)
            uint64_t out1;
            if (td->idx8) {
                bool bad = false;
                const uint32_t cnt = idx8_count(td, b, &bad);
                out1 = bad ? ~0ull : outr + cnt;
            } else {
                out1 = td->offs[b + 1];
            }
            if (out1 < outr || out1 > td->n || (b + 1 == td->n_blocks && out1 != td->n)) {
                if (lane == 0 && d_err) atomicOr(d_err, DF_EFLAG_OFFSETS);
                break;
            }
            // warm L2 with the block's sign|fraction bytes
            if (lane == 0) {
                const uintptr_t lo = (reinterpret_cast<uintptr_t>(sm + outr) + 15) & ~static_cast<uintptr_t>(15);
                const uintptr_t hi = reinterpret_cast<uintptr_t>(sm + out1) & ~static_cast<uintptr_t>(15);
                if (hi > lo)
                    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(lo),
                                 "r"(static_cast<uint32_t>(hi - lo)) : "memory");
            }
            const uint64_t c_blk = min((b + 1) * T, n_chunks);
            for (; c < c_blk; c += 32) {  // the block's rounds of 32 chunks
                const bool block_last = c + 32 >= c_blk;
                const bool run_last = c + 32 >= c_end;
                const uint32_t align = static_cast<uint32_t>(outr & 15);
                // 1. lane 0 starts from the exponents the previous round left
                // open (stage positions [0, align)); at the start of a run they
                // are placeholders for outputs of the previous run
                uint32_t st = 0, endst = 0, acc = 0;
                if (lane == 0) {
                    *reinterpret_cast<uint4*>(my_region) = *reinterpret_cast<const uint4*>(s_carry);
                    acc = s_carry[align >> 2] & ((1u << (8 * (align & 3))) - 1u);
                    st = align << kStepCountShift;
                }
                // this lane's chunk and gap
                const uint64_t chunk = c + lane;
                if (chunk < n_chunks) {
                    const uint64_t q = 5 * chunk;
                    uint32_t two;
                    if (pre) {
                        two = pre_two;
                    } else {
                        const uint4* c4 = reinterpret_cast<const uint4*>(td->stream + chunk * C);
                        for (uint32_t k = 0; k < C / 16; ++k) {
                            const uint4 v = __ldg(c4 + k);
                            my_words[(4 * k + 0) * kLanes] = bswap32(v.x);
                            my_words[(4 * k + 1) * kLanes] = bswap32(v.y);
                            my_words[(4 * k + 2) * kLanes] = bswap32(v.z);
                            my_words[(4 * k + 3) * kLanes] = bswap32(v.w);
                        }
                        my_words[(C / 4) * kLanes] =
                            bswap32(__ldg(reinterpret_cast<const uint32_t*>(td->stream + (chunk + 1) * C)));
                        two = (static_cast<uint32_t>(__ldg(td->gaps + (q >> 3))) << 8) | __ldg(td->gaps + (q >> 3) + 1);
                    }
                    const uint32_t cbits = 8 * C;
                    const uint64_t bit0 = chunk * cbits;
                    const uint64_t rem = td->total_bits > bit0 ? td->total_bits - bit0 : 0;
                    st += ((two >> (11 - (q & 7))) & 31u) << kStepShift;
                    endst = static_cast<uint32_t>(rem < cbits ? rem : cbits) << kStepShift;
                }
                pre = false;

                // 2. decode: ext = the exponents in this lane's region
                const uint32_t dec = decode_chunk(st, endst, acc, shared_addr(my_words), shared_addr(my_region),
                                                  shared_addr(s_wide), td->lut);
                const uint32_t ext = dec & 0x7FFFFFFFu;

                // the chunk of the next round into registers now; it goes into
                // the slot after the scan
                const uint64_t nchunk = chunk + 32;
                const bool nx = C <= 32 && !run_last && nchunk < n_chunks;
                uint4 na = make_uint4(0, 0, 0, 0), nb4 = make_uint4(0, 0, 0, 0);
                uint32_t ntail = 0, ntwo = 0;
                if (nx) {
                    const uint4* c4 = reinterpret_cast<const uint4*>(td->stream + nchunk * C);
                    na = __ldg(c4);
                    if (C == 32) nb4 = __ldg(c4 + 1);
                    ntail = __ldg(reinterpret_cast<const uint32_t*>(td->stream + (nchunk + 1) * C));
                    const uint64_t qn = 5 * nchunk;
                    ntwo = (static_cast<uint32_t>(__ldg(td->gaps + (qn >> 3))) << 8) | __ldg(td->gaps + (qn >> 3) + 1);
                }

                // 3. warp scan: stage positions; checks against the block index
                const uint32_t incl = warp_incl_scan(ext, lane);
                const uint32_t vend = __shfl_sync(kFull, incl, 31);  // positions [0, vend) hold exponents
                const uint32_t total = vend - align;                  // codes of this round
                const bool any_bad = __any_sync(kFull, dec >> 31);
                uint32_t flags = 0;
                if (any_bad)
                    flags = DF_EFLAG_BAD_CODE;
                else if (outr + total > out1 || (block_last && outr + total != out1))
                    flags = DF_EFLAG_COUNT;
                else if ((vend + 15) / 16 > cfg.max_groups)
                    flags = DF_EFLAG_OFFSETS;
                if (flags) {  // uniform over the warp: the run stops here
                    if (lane == 0 && d_err) atomicOr(d_err, flags);
                    ok = false;
                    break;
                }
                const uint32_t pos = incl - ext;
                const int my_base = my_off - static_cast<int>(pos);  // stage position p is byte my_base + p
                s_pos[lane] = pos;
                s_base[lane] = my_base;
                if (lane == 31) s_pos[32] = vend;

                // 4. owner map: group gi (stage positions [16gi, 16gi+16))
                // belongs to the lane whose range holds 16gi; bit 7 marks a
                // group that runs past that range (completed in 4b, else merged in 5b)
                if (ext) {
                    const uint32_t hi = pos + ext;
                    for (uint32_t gi = (pos + 15) >> 4; 16 * gi < hi; ++gi)
                        s_owner[gi] = static_cast<uint8_t>(lane | (16 * gi + 16 > hi ? 0x80u : 0u));
                }
                if (nx) {  // only this lane reads its slot, and its decode is done
                    my_words[0 * kLanes] = bswap32(na.x);
                    my_words[1 * kLanes] = bswap32(na.y);
                    my_words[2 * kLanes] = bswap32(na.z);
                    my_words[3 * kLanes] = bswap32(na.w);
                    if (C == 32) {
                        my_words[4 * kLanes] = bswap32(nb4.x);
                        my_words[5 * kLanes] = bswap32(nb4.y);
                        my_words[6 * kLanes] = bswap32(nb4.z);
                        my_words[7 * kLanes] = bswap32(nb4.w);
                    }
                    my_words[(C / 4) * kLanes] = bswap32(ntail);
                    pre_two = ntwo;
                    pre = true;
                }
                __syncwarp();

                // 4b. complete the group this lane's range ends inside: the
                // round's last group has all its exponents here already; any
                // other takes the next lane's first 16 exponents into the slack
                // after this lane's own, so that 5a finds all 16 in one region.
                // Both regions must hold at least 20 exponents (this lane's
                // writes start past the bytes the lane before reads, and the
                // next lane's writes past the bytes read here) and this region
                // must have 20 bytes to spare; the rest stay for 5b.
                const uint32_t bend = pos + ext;
                const uint32_t ext_next = __shfl_down_sync(kFull, ext, 1);
                if (ext && (bend & 15) && (bend & ~15u) >= pos) {  // this lane owns that group
                    const uint32_t gi = bend >> 4;
                    if (bend == vend) {
                        s_owner[gi] = static_cast<uint8_t>(lane);
                    } else if (lane + 1 < kLanes && ext >= 20 && ext_next >= 20 && ext + 20 <= RB) {
                        const uint32_t sa = shared_addr(s_priv + region_off(lane + 1, RB));
                        const uint32_t w0 = lds32(sa), w1 = lds32(sa + 4), w2 = lds32(sa + 8), w3 = lds32(sa + 12);
                        const uint32_t da = shared_addr(s_priv + my_off) + (ext & ~3u);
                        const uint32_t r8 = 8 * (ext & 3);
                        const uint32_t keep = r8 ? lds32(da) & ((1u << r8) - 1u) : 0u;
                        sts32(da, keep | (w0 << r8));
                        sts32(da + 4, __funnelshift_l(w0, w1, r8));
                        sts32(da + 8, __funnelshift_l(w1, w2, r8));
                        sts32(da + 12, __funnelshift_l(w2, w3, r8));
                        if (r8) sts32(da + 16, w3 >> (32 - r8));
                        s_owner[gi] = static_cast<uint8_t>(lane);
                    }
                }
                __syncwarp();

                // 5. merge and store; stage position p <-> output gbase + p,
                // group gi <-> the 16 sign|fraction bytes at smg + 16gi
                const uint64_t gbase = outr - align;
                const uint64_t rend = outr + total;  // this round's outputs end here
                const uint32_t ngroups = (vend + 15) >> 4;
                const uint32_t gv0 = gbase < vstart ? 1u : 0u;      // group 0 may start before the run
                const uint32_t glast = (vend & 15) ? ngroups - 1 : ngroups;  // a last group the round ends inside
                const uint8_t* __restrict__ smg = sm + gbase;
                uint16_t* __restrict__ outg = out + gbase;
                // 5a. groups inside their owner's range (bit 7 of the owner byte
                // clear); the others are merged in 5b. Two groups per lane and
                // iteration: both sign|fraction loads are in flight first. A
                // run's first group and a round's unfinished last group are
                // merged below.
                if (vec) {
                    for (uint32_t g0 = lane; g0 < ngroups; g0 += 2 * kLanes) {
                        const uint32_t g1 = g0 + kLanes;
                        const uint32_t o0 = s_owner[g0];
                        const uint32_t o1 = g1 < ngroups ? s_owner[g1] : 0x80u;
                        const bool v0 = !(o0 & 0x80u) && g0 >= gv0 && g0 != glast;
                        const bool v1 = !(o1 & 0x80u) && g1 != glast;
                        uint4 s0 = make_uint4(0, 0, 0, 0), s1 = make_uint4(0, 0, 0, 0);
                        if (v0) s0 = __ldg(reinterpret_cast<const uint4*>(smg) + g0);
                        if (v1) s1 = __ldg(reinterpret_cast<const uint4*>(smg) + g1);
                        uint32_t e[4];
                        if (v0) {
                            gather16(s_priv, s_base[o0 & 31u] + static_cast<int>(16 * g0), e);
                            merge16(s0, e, outg + 16 * g0);
                        }
                        if (v1) {
                            gather16(s_priv, s_base[o1 & 31u] + static_cast<int>(16 * g1), e);
                            merge16(s1, e, outg + 16 * g1);
                        }
                    }
                }
                // edge groups, element stores: a run's first group (it starts
                // before the run's outputs), the round's unfinished last group
                // (carried into the next round unless the run ends here), and
                // every group of buffers without 16-byte alignment
                auto edge = [&](uint32_t gi) {
                    const uint32_t o = s_owner[gi];
                    if (o & 0x80u) return;  // 5b takes it
                    uint32_t e[4];
                    gather16(s_priv, s_base[o & 31u] + static_cast<int>(16 * gi), e);
                    if (gi == glast && !run_last) {
                        *reinterpret_cast<uint4*>(s_carry) = make_uint4(e[0], e[1], e[2], e[3]);
                        return;
                    }
                    const uint64_t G = gbase + 16 * gi;
                    const uint64_t lo_i = max(G, vstart), hi_i = min(G + 16, rend);
                    for (uint64_t i = lo_i; i < hi_i; ++i)
                        out[i] = merge1(sm[i], static_cast<uint8_t>(e[(i - G) >> 2] >> (8 * ((i - G) & 3))));
                };
                if (!vec) {
                    for (uint32_t gi = lane; gi < ngroups; gi += kLanes) edge(gi);
                } else {
                    if (lane == 0 && gv0) edge(0);
                    if (lane == 1 && glast < ngroups && !(gv0 && glast == 0)) edge(glast);
                }
                // 5b. a group that spans regions and was not completed in 4b:
                // the lane whose range it starts in gathers it from the regions
                // (rare: short or full regions, three or more regions)
                const bool span = ext && (bend & 15) && s_owner[bend >> 4] == (lane | 0x80u);
                if (__any_sync(kFull, span) && span) {
                    const uint32_t c0 = bend & ~15u;
                    const uint64_t G = gbase + c0;
                    const uint32_t hi = min(c0 + 16, vend);
                    uint32_t e[4];
                    if (hi <= bend) {  // the round ends in this region
                        gather16(s_priv, my_base + static_cast<int>(c0), e);
                    } else if (lane + 1 < kLanes && hi <= s_pos[lane + 2]) {  // this region and the next
                        uint32_t x[4], y[4];
                        gather16(s_priv, my_base + static_cast<int>(c0), x);
                        gather16(s_priv, static_cast<int>((lane + 1) * RB) - static_cast<int>(bend - c0), y);
#pragma unroll
                        for (int i = 0; i < 4; ++i) {  // bytes before bend from x, the rest from y
                            const int sbits = 8 * static_cast<int>(bend - c0) - 32 * i;
                            const uint32_t m = sbits >= 32 ? 0xFFFFFFFFu : (sbits <= 0 ? 0u : (1u << sbits) - 1u);
                            e[i] = (x[i] & m) | (y[i] & ~m);
                        }
                    } else {  // three or more regions
                        e[0] = e[1] = e[2] = e[3] = 0;
                        uint32_t t = lane;
                        for (uint32_t p = c0; p < hi; ++p) {
                            while (p >= s_pos[t + 1]) ++t;
                            e[(p - c0) >> 2] |= static_cast<uint32_t>(s_priv[s_base[t] + static_cast<int>(p)])
                                                << (8 * ((p - c0) & 3));
                        }
                    }
                    if (c0 + 16 > vend && !run_last) {
                        *reinterpret_cast<uint4*>(s_carry) = make_uint4(e[0], e[1], e[2], e[3]);
                    } else {
                        const uint64_t lo_i = max(G, vstart), hi_i = min(G + 16, rend);
                        if (vec && lo_i == G && hi_i == G + 16) {
                            merge16(__ldg(reinterpret_cast<const uint4*>(sm + G)), e, out + G);
                        } else {
                            for (uint64_t i = lo_i; i < hi_i; ++i)
                                out[i] = merge1(sm[i], static_cast<uint8_t>(e[(i - G) >> 2] >> (8 * ((i - G) & 3))));
                        }
                    }
                }
                __syncwarp();  // the next round overwrites the regions, positions, owner map and carry
                outr = rend;
            }
            ++b;
        }
    }
}

struct Prepared {
    DevTensor dev;
    uint32_t words_per_chunk, region_bytes, max_groups;
};

uint32_t min_len_of(const uint8_t* lengths) {
    uint32_t m = 0;
    for (int s = 0; s < 256; ++s)
        if (lengths[s] && (!m || lengths[s] < m)) m = lengths[s];
    return m;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

// Validate a descriptor and fill the device-side copy and the shared-memory
// needs of its rounds.
df_status prepare(const df_tensor* t, uint16_t* out, Prepared* pr) {
    if (!t || !out) return DF_ERR_INVALID_ARG;
    const uint32_t C = t->chunk_bytes, T = t->threads_per_block;
    if (C < 16 || C > 4096 || C % 16 || T < 32 || T > 1024 || T % 32) return DF_ERR_INVALID_ARG;
    // the state word keeps a bit position below 2^14 (C <= 1024 bytes)
    if (C > 1024) return DF_ERR_UNSUPPORTED;
    if (t->max_len < 1 || t->max_len > 32 || t->n_tables < 1) return DF_ERR_INVALID_ARG;
    if (t->n > DF_MAX_WEIGHTS) return DF_ERR_UNSUPPORTED;
    if (!t->stream || !t->gaps || !t->sm || !t->lut) return DF_ERR_INVALID_ARG;
    if (!t->block_offsets == !t->index8) return DF_ERR_INVALID_ARG;  // exactly one block index
    if (!aligned(t->stream, 16) || !aligned(t->lut, 16) || !aligned(t->block_offsets, 8) ||
        !aligned(t->index8, 8) || !aligned(out, 2))
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
    if (t->index8) {
        if (t->index8_wide > (n_blocks + 63) / 64) return DF_ERR_INVALID_ARG;
        d.offs = reinterpret_cast<const uint64_t*>(t->index8);
        d.idx8 = static_cast<uint32_t>(t->index8_wide + 1);
    } else {
        d.offs = t->block_offsets;
    }
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
    pr->words_per_chunk = C / 4 + 1;  // the chunk and the next chunk's first word
    // a chunk holds at most 8C/min_len code starts; its region also takes up
    // to 3 exponents past the last counted code and the word they end in
    const uint64_t per_chunk = (cbits + minl - 1) / (minl ? minl : 1);
    uint64_t rb = (per_chunk + kRegionSlack + 3) & ~3ull;
    if (((rb / 4) & 1) == 0) rb += 4;  // odd word stride: regions start in distinct banks
    // a round holds at most 32 * 8C/min_len codes and never more than n
    uint64_t per_round = per_chunk * kLanes;
    if (per_round > t->n) per_round = t->n;
    const uint64_t groups = (per_round + 15 + 15) / 16 + 1;
    if (rb > (1u << 20) || groups > 0xFFFFu) return DF_ERR_UNSUPPORTED;
    pr->region_bytes = static_cast<uint32_t>(rb);
    pr->max_groups = static_cast<uint32_t>(groups);
    return DF_OK;
}

// Shared memory of one warp: chunk slots, stage positions and carry, owner
// map, the 16-byte pad before the regions, regions.
uint32_t warp_area_bytes(const LaunchCfg& c) {
    const uint64_t b = static_cast<uint64_t>(kLanes) * c.words_per_chunk * 4 + kPosWords * 4 +
                       ((c.max_groups + 15) & ~15u) + 16 + static_cast<uint64_t>(kLanes) * c.region_bytes;
    return static_cast<uint32_t>(std::min<uint64_t>((b + 15) & ~15ull, 0xFFFFFFFFull));
}

size_t smem_bytes(const LaunchCfg& c, uint32_t warps) {
    return kFixedBytes + static_cast<size_t>(warps) * c.warp_bytes + kSmemSlack;
}

df_status device_limits(int* sms, int* max_smem, int* smem_per_sm) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e);
    e = cudaDeviceGetAttribute(sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return cuda_fail(e);
    e = cudaDeviceGetAttribute(max_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    if (e != cudaSuccess) return cuda_fail(e);
    e = cudaDeviceGetAttribute(smem_per_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev);
    if (e != cudaSuccess) return cuda_fail(e);
    return DF_OK;
}

// Warps per CUDA block. For large launches: as many resident warps per SM as
// shared memory allows (at most 32, the register file's limit at 64
// registers), with the most warps per block among equals (one copy of the
// wide table serves them all). Smaller CUDA blocks when that would leave SMs
// idle or warps waiting: a launch of fewer format blocks than one per warp of
// the whole GPU spreads its blocks over every SM, and a launch over more
// tensors than SMs that average fewer than 128 format blocks each (every
// tensor change synchronises the CUDA block, and a small tensor keeps most of
// a wide block's warps waiting) uses blocks of 8 warps, two per SM.
df_status choose_warps(const LaunchCfg& c, uint64_t total_blocks, uint64_t tensors, uint32_t* warps) {
    int sms = 0, max_smem = 0, per_sm = 0;
    df_status st = device_limits(&sms, &max_smem, &per_sm);
    if (st != DF_OK) return st;
    uint32_t best = 0, best_resident = 0;
    for (uint32_t w = 1; w <= kMaxWarps; ++w) {
        const size_t s = smem_bytes(c, w);
        if (s > static_cast<size_t>(max_smem)) break;
        const uint32_t ctas = static_cast<uint32_t>(per_sm / (s + 1024));  // 1 KB reserved per block
        const uint32_t resident = std::min(ctas * w, kMaxWarps);
        if (resident >= best_resident && resident > 0) {
            best = w;
            best_resident = resident;
        }
    }
    if (!best) return DF_ERR_UNSUPPORTED;
    uint64_t w = best;
    const uint64_t per_sm_blocks = (total_blocks + sms - 1) / static_cast<uint64_t>(sms);
    if (per_sm_blocks < w) w = per_sm_blocks;
    // many tensors of few format blocks each: 8 measured best on 2000 tensors
    // of log-uniform sizes (mean 25 blocks); large tensors keep wide blocks
    if (tensors > static_cast<uint64_t>(sms) && total_blocks < 128 * tensors && w > 8) w = 8;
    *warps = static_cast<uint32_t>(w < 1 ? 1 : (w > best ? best : w));
    return DF_OK;
}

template <class Src>
df_status launch(const Src& src, const LaunchCfg& cfg, uint32_t warps, uint32_t max_ctas, uint32_t* d_err,
                 cudaStream_t stream) {
    if (cfg.total_blocks == 0) return DF_OK;
    int sms = 0, max_smem = 0, per_sm = 0;
    df_status st = device_limits(&sms, &max_smem, &per_sm);
    if (st != DF_OK) return st;
    const size_t smem = smem_bytes(cfg, warps);
    if (warps < 1 || warps > kMaxWarps || smem > static_cast<size_t>(max_smem)) return DF_ERR_UNSUPPORTED;
    auto kern = decode_kernel<Src>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return cuda_fail(e);
    int resident = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&resident, kern, static_cast<int>(warps * kLanes), smem);
    if (e != cudaSuccess) return cuda_fail(e);
    if (resident < 1) return DF_ERR_UNSUPPORTED;
    // persistent blocks: every resident slot loops over a range of format
    // blocks; a range is never shorter than one format block per warp
    const uint64_t slots = static_cast<uint64_t>(sms) * resident;
    const uint64_t want = (cfg.total_blocks + warps - 1) / warps;
    uint64_t grid = want < slots ? want : slots;
    if (max_ctas && grid > max_ctas) grid = max_ctas;
    kern<<<static_cast<unsigned>(grid), warps * kLanes, smem, stream>>>(src, cfg, d_err);
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e);
    return DF_OK;
}

void widen(LaunchCfg* c, const Prepared& p) {
    c->words_per_chunk = std::max(c->words_per_chunk, p.words_per_chunk);
    c->region_bytes = std::max(c->region_bytes, p.region_bytes);
    c->max_groups = std::max(c->max_groups, p.max_groups);
    c->warp_bytes = warp_area_bytes(*c);
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
    uint32_t warps = 0;
    st = choose_warps(cfg, cfg.total_blocks, 1, &warps);
    if (st != DF_OK) return st;
    return launch(src, cfg, warps, 0, d_err, static_cast<cudaStream_t>(stream));
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
    plan->words_per_chunk = cfg.words_per_chunk;
    plan->region_bytes = cfg.region_bytes;
    plan->max_groups = cfg.max_groups;
    plan->total_blocks = start.back();
    if (plan->count == 0) return DF_OK;
    uint32_t warps = 0;
    df_status st = choose_warps(cfg, plan->total_blocks, plan->count, &warps);
    if (st != DF_OK) return st;
    plan->cta_threads = warps * kLanes;
    plan->smem_bytes = static_cast<uint32_t>(smem_bytes(cfg, warps));
    // A CUDA block decodes a contiguous range of format blocks, restaging the
    // tables (and waiting for all its warps) at every tensor; a tensor of
    // fewer format blocks than warps leaves most warps idle until the next
    // restage. When such small tensors outnumber the resident CUDA blocks,
    // spread them evenly between the large ones, so every range holds its
    // share instead of a few ranges holding clusters of them (the descriptors
    // carry their own outputs, so their order is free). A few small tensors
    // stay where they are: moving one only adds a restage.
    int sms = 0, max_smem = 0, per_sm = 0;
    st = device_limits(&sms, &max_smem, &per_sm);
    if (st != DF_OK) return st;
    const uint64_t resident = static_cast<uint64_t>(sms) *
                              std::max<uint64_t>(1, static_cast<uint64_t>(per_sm) / (plan->smem_bytes + 1024));
    {
        std::vector<uint32_t> small, large;
        uint64_t large_blocks = 0;
        for (uint32_t i = 0; i < dev.size(); ++i) {
            if (dev[i].n_blocks < warps) {
                small.push_back(i);
            } else {
                large.push_back(i);
                large_blocks += dev[i].n_blocks;
            }
        }
        if (small.size() >= resident && !large.empty()) {
            std::vector<DevTensor> order;
            order.reserve(dev.size());
            uint64_t done = 0;  // large blocks placed so far
            size_t si = 0;
            for (uint32_t li : large) {
                order.push_back(dev[li]);
                done += dev[li].n_blocks;
                // small tensor k belongs after (k + 1/2) / small.size() of the large blocks
                while (si < small.size() && static_cast<unsigned __int128>(2 * si + 1) * large_blocks <=
                                                static_cast<unsigned __int128>(2 * done) * small.size())
                    order.push_back(dev[small[si++]]);
            }
            while (si < small.size()) order.push_back(dev[small[si++]]);
            dev.swap(order);
            for (size_t i = 0; i < dev.size(); ++i) start[i + 1] = start[i] + dev[i].n_blocks;
        }
    }
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
    if (!plan->d_ws || plan->cta_threads % kLanes) return DF_ERR_INVALID_ARG;
    BatchSrc src;  // same layout as df_decode_batch_prepare writes
    src.tensors = static_cast<const DevTensor*>(plan->d_ws);
    src.count = plan->count;
    const size_t table_bytes = (static_cast<size_t>(plan->count) * sizeof(DevTensor) + 255) / 256 * 256;
    src.block_start = reinterpret_cast<const uint64_t*>(static_cast<const uint8_t*>(plan->d_ws) + table_bytes);
    LaunchCfg cfg;
    std::memset(&cfg, 0, sizeof(cfg));
    cfg.words_per_chunk = plan->words_per_chunk;
    cfg.region_bytes = plan->region_bytes;
    cfg.max_groups = plan->max_groups;
    cfg.warp_bytes = warp_area_bytes(cfg);
    cfg.total_blocks = plan->total_blocks;
    const uint32_t warps = plan->cta_threads / kLanes;
    if (smem_bytes(cfg, warps) != plan->smem_bytes) return DF_ERR_INVALID_ARG;
    return launch(src, cfg, warps, plan->max_ctas, d_err, static_cast<cudaStream_t>(stream));
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
