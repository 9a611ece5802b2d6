// Decode kernel: compressed exponent stream + sign|fraction bytes -> BF16.
//
// The pages fix what decoding restores (mlx-dfloat, PyPI page, intro: the
// exponent code is undone and the raw sign|fraction byte put back, bit for bit)
// and that it runs blockwise on the GPU (mlx-dfloat, "Status"; df11pack, intro).
// The layout of the work below is this library's own, written for sm_100a.
//
// One CUDA block of T threads handles one format block (T chunks of C stream
// bytes) at a time and loops over a contiguous range of the format blocks of
// all tensors of the launch (persistent blocks, one range each):
//   1. when the tensor changes, copy its descriptor and stage its wide table
//      in shared memory (1024 entries indexed by 10 stream bits: the exponents
//      of the codes that lie wholly inside the window and one step word,
//      (bits used << 18) | (count << 3)); warm L2 with the next block's stream
//      slice (bulk prefetch);
//      stage the block's stream slice, one chunk per thread, byte-swapped to
//      big-endian words, word i of thread t at i * T + t (the 32 lanes of a
//      warp read 32 different banks wherever their windows are)
//   2. one decode pass per thread over its chunk, from chunk start + gap to
//      the chunk end: the state word (bit position << 18) | (exponents so
//      far << 3) advances by one add per table step (up to 4 codes); the
//      exponents go to the thread's own word-aligned shared-memory region
//      with 32-bit stores; codes longer than 10 bits walk the 8-bit tables
//      then warm L2 with this block's sign|fraction bytes, and load this
//      thread's chunk of the next block into registers (it goes into the idle
//      slot just before the merge, so the next block starts without a load)
//   3. block scan of the code counts (warp shuffles + one shared array): the
//      first output position of every thread; checked against the block index
//   4. an owner map: for every group of 16 outputs, the thread whose region
//      holds its first exponent
//   5. merge, in two loops: groups that lie in one region take their 16
//      exponents from it; then each thread takes the one group, if any, that
//      its range ends inside, gathering from its region and the next one(s).
//      Per group: one 16-byte load of sign|fraction bytes, two 16-byte stores.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstring>
#include <vector>

#include "df_internal.h"

namespace df {
namespace {

constexpr uint32_t kWideN = 1u << kWideBits;
constexpr uint32_t kMaxThreads = 1024;
constexpr uint32_t kFull = 0xFFFFFFFFu;

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
    uint32_t words_per_chunk;  // shared-memory words of a chunk (C / 4 + 1 for the widest C)
    uint32_t region_bytes;     // exponent region of a thread (4 * odd)
    uint32_t max_groups;       // owner-map entries
    uint32_t pad;
    uint64_t total_blocks;
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

// The 32 stream bits from bit p of a chunk whose big-endian words are at
// w[0], w[S], w[2S], ... (S = the block size).
template <uint32_t kT>
__device__ __forceinline__ uint32_t window(const uint32_t* w, uint32_t p) {
    const uint32_t S = kT ? kT : blockDim.x;  // word i of the chunk at w[i * S]
    const uint32_t* a = w + (p >> 5) * S;
    return __funnelshift_l(a[S], a[0], p);
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
__device__ __forceinline__ void merge4(uint32_t s, uint32_t e, uint32_t* o0, uint32_t* o1) {
    const uint32_t hi = (s & 0x80808080u) | ((e >> 1) & 0x7F7F7F7Fu);
    const uint32_t lo = ((e << 7) & 0x80808080u) | (s & 0x7F7F7F7Fu);
    *o0 = __byte_perm(lo, hi, 0x5140);
    *o1 = __byte_perm(lo, hi, 0x7362);
}

// 16 outputs from their 16 sign|fraction bytes and 16 exponents: two 16-byte
// stores, marked evict-first (the outputs are not read again by this kernel and
// should not push the prefetched stream and sign|fraction lines out of L2).
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

// A code longer than the wide window, as a step word ((length << 18) | 1 << 3,
// or 0 for a bit pattern no code starts with) and its exponent.
__device__ __forceinline__ uint32_t long_step(uint32_t win, const uint32_t* hier, uint32_t* sym) {
    const uint32_t l = long_code(win, hier);
    *sym = l & 0xFFu;
    return l ? (((l >> 8) & 63u) << kStepShift) | (1u << kStepCountShift) : 0u;
}

// Decoder of one thread's chunk: state word (bit position << 18) |
// (exponents appended to the region << 3); the exponents of the region word
// not yet stored sit in the low bytes of acc ((state & 24) / 8 of them).
struct Lane {
    uint32_t st;
    uint32_t end;  // codes must start before this bit
    uint32_t acc;
    bool bad;
};

// Append the exponents of one step word to the region.
__device__ __forceinline__ void append(Lane& L, uint32_t w, uint32_t sy, uint32_t* region) {
    const uint32_t sh = L.st & 24u;
    const uint32_t lo = L.acc | (sy << sh);
    const uint32_t nst = L.st + w;
    if ((nst ^ L.st) & (kStepCountMask & ~31u)) {  // a region word is complete
        region[(L.st & kStepCountMask) >> 5] = lo;
        L.acc = __funnelshift_rc(sy, 0u, 32u - sh);  // the bytes past it (none when sh = 0)
    } else {
        L.acc = lo;
    }
    L.st = nst;
}

// One table step whose window lies before the chunk end.
template <uint32_t kT>
__device__ __forceinline__ void full_step(Lane& L, const uint32_t* words, const uint64_t* wide, const uint32_t* hier,
                                          uint32_t* region) {
    const uint32_t win = window<kT>(words, L.st >> kStepShift);
    const uint64_t e = wide[win >> (32 - kWideBits)];
    uint32_t sy = static_cast<uint32_t>(e);
    uint32_t w = static_cast<uint32_t>(e >> 32);
    if (w == 0) {
        w = long_step(win, hier, &sy);
        if (w == 0) {
            L.bad = true;
            L.end = 0;
        }
    }
    append(L, w, sy, region);
}

// kT: the block size when fixed at compile time (256, the default format),
// else 0 and the block size is read at run time.
template <class Src, class OwnerT, uint32_t kT>
__global__ void __launch_bounds__(kT ? kT : kMaxThreads, kMaxThreads / (kT ? kT : kMaxThreads))
    decode_kernel(const __grid_constant__ Src src, const LaunchCfg cfg,
                                                             uint32_t* d_err) {
    extern __shared__ __align__(16) uint8_t smem[];
    const uint32_t T = kT ? kT : blockDim.x;  // a compile-time block size folds the address arithmetic
    const uint32_t tid = threadIdx.x;
    const uint32_t lane = tid & 31, warp = tid >> 5;
    const uint32_t nwarps = T >> 5;

    // shared memory carve-up (sizes in smem_bytes())
    const uint64_t* s_wide = reinterpret_cast<const uint64_t*>(smem);
    uint32_t* s_words = reinterpret_cast<uint32_t*>(smem + 8 * kWideN);
    uint32_t* s_pos = s_words + ((T * cfg.words_per_chunk + 3) & ~3u);
    uint32_t* s_warp = s_pos + ((T + 1 + 3) & ~3u);
    uint32_t* s_hdr = s_warp + 32;  // 1 when the staged tables belong to the staged tensor
    // the current tensor's descriptor: copied here on a tensor switch, because
    // the merge's streaming loads keep evicting it from L1
    DevTensor* s_td = reinterpret_cast<DevTensor*>(s_hdr + 4);
    OwnerT* s_owner = reinterpret_cast<OwnerT*>(reinterpret_cast<uint8_t*>(s_td) + sizeof(DevTensor));
    uint8_t* s_priv = reinterpret_cast<uint8_t*>(s_owner) + ((cfg.max_groups * sizeof(OwnerT) + 15) & ~15u);
    const uint32_t RB = cfg.region_bytes;
    uint32_t* my_region = reinterpret_cast<uint32_t*>(s_priv + tid * RB);

    const DevTensor* tg = nullptr;      // the current tensor's descriptor in global memory
    const DevTensor* staged = nullptr;
    const DevTensor* const td = s_td;  // read through its shared-memory copy
    uint64_t t_lo = 0, t_hi = 0;
    bool pre = false;      // this thread's chunk of block g is already in its slot
    uint32_t pre_two = 0;  // and its two gap bytes
    // each CUDA block takes a contiguous range of format blocks, so that it
    // changes tensors (and restages tables) as rarely as possible
    const uint64_t per = cfg.total_blocks / gridDim.x, extra = cfg.total_blocks % gridDim.x;
    const uint64_t g_begin = blockIdx.x * per + min(static_cast<uint64_t>(blockIdx.x), extra);
    const uint64_t g_end = g_begin + per + (blockIdx.x < extra ? 1 : 0);
    for (uint64_t g = g_begin; g < g_end; ++g) {
        if (g < t_lo || g >= t_hi) tg = src.find(g, &t_lo, &t_hi);
        const uint64_t b = g - t_lo;
        // 1. descriptor and tables (when the tensor changes) and the stream slice
        const bool restage = tg != staged;
        if (restage) {
            if (tid < sizeof(DevTensor) / 4)
                reinterpret_cast<uint32_t*>(s_td)[tid] = reinterpret_cast<const uint32_t*>(tg)[tid];
            __syncthreads();
            const uint4* t4 = reinterpret_cast<const uint4*>(td->lut);
            uint4* d4 = reinterpret_cast<uint4*>(smem);
            for (uint32_t i = tid; i < kWideEntryWords / 4; i += T) d4[i] = __ldg(t4 + i);
            if (tid == 0) {
                const uint32_t* hdr = td->lut + kWideWords + static_cast<size_t>(td->n_tables) * 256 + 64;
                const uint32_t minl = __ldg(hdr);
                // the region must hold every code the tables can yield in one chunk
                s_hdr[0] = __ldg(hdr + 3) == kLutMagic && __ldg(hdr + 2) == td->n_tables && minl >= 1 &&
                           (8 * td->chunk_bytes + minl - 1) / minl + 12 <= RB;
            }
            staged = tg;
        }
        const uint32_t C = td->chunk_bytes;
        // warm L2 with the stream slice of the next block of the same tensor
        const uint64_t g_next = g + 1;
        if (tid == 0 && g_next < t_hi && g_next < g_end) {
            const uint64_t s0 = (g_next - t_lo) * T * C;
            const uint64_t s_bytes = min(static_cast<uint64_t>(T) * C + 16, td->n_chunks * C + 16 - s0);
            asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(td->stream + s0),
                         "r"(static_cast<uint32_t>(s_bytes)) : "memory");
        }
        uint32_t* my_words = s_words + tid;  // word i of this chunk at my_words[i * T]
        const uint64_t chunk = b * T + tid;
        Lane L;
        L.st = 0;
        L.end = 0;
        L.acc = 0;
        L.bad = false;
        if (chunk < td->n_chunks) {
            const uint64_t q = 5 * chunk;
            uint32_t two;
            if (pre) {
                two = pre_two;
            } else {
                const uint4* c4 = reinterpret_cast<const uint4*>(td->stream + chunk * C);
                for (uint32_t k = 0; k < C / 16; ++k) {
                    const uint4 v = __ldg(c4 + k);
                    my_words[(4 * k + 0) * T] = bswap32(v.x);
                    my_words[(4 * k + 1) * T] = bswap32(v.y);
                    my_words[(4 * k + 2) * T] = bswap32(v.z);
                    my_words[(4 * k + 3) * T] = bswap32(v.w);
                }
                my_words[(C / 4) * T] = bswap32(__ldg(reinterpret_cast<const uint32_t*>(td->stream + (chunk + 1) * C)));
                two = (static_cast<uint32_t>(__ldg(td->gaps + (q >> 3))) << 8) | __ldg(td->gaps + (q >> 3) + 1);
            }
            const uint32_t cbits = 8 * C;
            const uint64_t bit0 = chunk * cbits;
            const uint64_t rem = td->total_bits > bit0 ? td->total_bits - bit0 : 0;
            L.st = ((two >> (11 - (q & 7))) & 31u) << kStepShift;
            L.end = static_cast<uint32_t>(rem < cbits ? rem : cbits);
        }
        pre = false;
        const uint64_t out0 = td->offs[b];
        const uint64_t out1 = td->offs[b + 1];
        // only the staged tables and their check are shared here: every thread
        // reads only its own chunk slot before the scan
        if (restage) __syncthreads();
        if (!s_hdr[0]) {  // tables that do not belong to this descriptor
            if (tid == 0 && d_err) atomicOr(d_err, DF_EFLAG_TABLES);
            __syncthreads();
            continue;
        }

        // 2. decode this thread's chunk into its region
        const uint32_t* hier = td->lut + kWideWords;
        for (;;) {  // two whole windows per vote
            const bool act = (L.st >> kStepShift) + 2 * kWideBits <= L.end;
            if (!__any_sync(kFull, act)) break;
            if (act) {
                full_step<kT>(L, my_words, s_wide, hier, my_region);
                // a long code may have moved p past the second window
                if ((L.st >> kStepShift) + kWideBits <= L.end) full_step<kT>(L, my_words, s_wide, hier, my_region);
            }
        }
        uint32_t cnt = (L.st & kStepCountMask) >> kStepCountShift;  // codes of whole windows start before the end
        for (;;) {  // windows that may reach past the end: count the codes starting before it
            const uint32_t p = L.st >> kStepShift;
            const bool act = p < L.end;
            if (!__any_sync(kFull, act)) break;
            if (act) {
                const uint32_t win = window<kT>(my_words, p);
                const uint32_t x = win >> (32 - kWideBits);
                const uint64_t e = s_wide[x];
                uint32_t sy = static_cast<uint32_t>(e);
                uint32_t w = static_cast<uint32_t>(e >> 32);
                uint32_t counted;
                if (w == 0) {
                    w = long_step(win, hier, &sy);
                    counted = (w & kStepCountMask) >> kStepCountShift;
                    if (w == 0) {
                        L.bad = true;
                        L.end = 0;
                    }
                } else if (L.end - p < kWideBits) {
                    const uint16_t* mask = reinterpret_cast<const uint16_t*>(td->lut + kWideEntryWords);
                    counted = __popc(__ldg(mask + x) & ((1u << (L.end - p)) - 1u));
                } else {
                    counted = (w & kStepCountMask) >> kStepCountShift;
                }
                append(L, w, sy, my_region);  // exponents past the end land in the region, uncounted
                cnt += counted;
            }
        }
        // the pending exponents (at most 3) complete the region
        my_region[(L.st & kStepCountMask) >> 5] = L.acc;
        // load this thread's chunk of the next block (same tensor, C <= 32) now;
        // it goes into the (idle) slot after the owner map, before the merge
        const uint64_t nchunk = chunk + T;
        const bool nx = C <= 32 && g + 1 < g_end && g + 1 < t_hi && nchunk < td->n_chunks;
        uint4 na = make_uint4(0, 0, 0, 0), nb = make_uint4(0, 0, 0, 0);
        uint32_t ntail = 0, ntwo = 0;
        if (nx) {
            const uint4* c4 = reinterpret_cast<const uint4*>(td->stream + nchunk * C);
            na = __ldg(c4);
            if (C == 32) nb = __ldg(c4 + 1);
            ntail = __ldg(reinterpret_cast<const uint32_t*>(td->stream + (nchunk + 1) * C));
            const uint64_t qn = 5 * nchunk;
            ntwo = (static_cast<uint32_t>(__ldg(td->gaps + (qn >> 3))) << 8) | __ldg(td->gaps + (qn >> 3) + 1);
        }
        // warm L2 with the block's sign|fraction bytes (the offsets have arrived by now)
        if (tid == 0 && out0 <= out1 && out1 <= td->n) {
            const uintptr_t lo = (reinterpret_cast<uintptr_t>(td->sm + out0) + 15) & ~static_cast<uintptr_t>(15);
            const uintptr_t hi = reinterpret_cast<uintptr_t>(td->sm + out1) & ~static_cast<uintptr_t>(15);
            if (hi > lo)
                asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(lo),
                             "r"(static_cast<uint32_t>(hi - lo)) : "memory");
        }

        // 3. block scan of the counts: warp totals (with a corrupt-data bit)
        // in shared memory, then every warp scans them again on its own
        const uint32_t incl = warp_incl_scan(cnt, lane);
        const bool warp_bad = __any_sync(kFull, L.bad);
        if (lane == 31) s_warp[warp] = incl | (warp_bad ? 0x80000000u : 0u);
        __syncthreads();
        const uint32_t wv = lane < nwarps ? s_warp[lane] : 0u;
        const bool any_bad = __any_sync(kFull, wv >> 31);
        const uint32_t wincl = warp_incl_scan(wv & 0x7FFFFFFFu, lane);
        const uint32_t wprefix = __shfl_sync(kFull, wincl - (wv & 0x7FFFFFFFu), warp);
        const uint32_t total = __shfl_sync(kFull, wincl, nwarps - 1);
        const uint32_t align = static_cast<uint32_t>(out0 & 15);
        const uint32_t pos = align + wprefix + incl - cnt;
        s_pos[tid] = pos;
        if (tid == T - 1) s_pos[T] = pos + cnt;

        // consistency with the block index (uniform over the block)
        uint32_t flags = 0;
        if (out1 < out0 || out1 > td->n || (out1 - out0 + align + 15) / 16 > cfg.max_groups ||
            (b + 1 == td->n_blocks && out1 != td->n))
            flags |= DF_EFLAG_OFFSETS;
        else if (static_cast<uint64_t>(total) != out1 - out0)
            flags |= DF_EFLAG_COUNT;
        if (any_bad) flags |= DF_EFLAG_BAD_CODE;
        if (flags) {
            if (tid == 0 && d_err) atomicOr(d_err, flags);
            __syncthreads();
            continue;
        }

        // 4. owner map: group gi (stage positions [16gi, 16gi+16)) belongs to
        // the thread whose range holds max(16gi, align)
        if (cnt) {
            const uint32_t hi = pos + cnt;
            if (pos <= align && align < hi) s_owner[0] = static_cast<OwnerT>(tid);
            for (uint32_t gi = max((pos + 15) >> 4, 1u); 16 * gi < hi; ++gi) s_owner[gi] = static_cast<OwnerT>(tid);
        }
        __syncthreads();
        if (nx) {  // only this thread reads its slot, and not before the next block's decode
            my_words[0 * T] = bswap32(na.x);
            my_words[1 * T] = bswap32(na.y);
            my_words[2 * T] = bswap32(na.z);
            my_words[3 * T] = bswap32(na.w);
            if (C == 32) {
                my_words[4 * T] = bswap32(nb.x);
                my_words[5 * T] = bswap32(nb.y);
                my_words[6 * T] = bswap32(nb.z);
                my_words[7 * T] = bswap32(nb.w);
            }
            my_words[(C / 4) * T] = bswap32(ntail);
            pre_two = ntwo;
            pre = true;
        }

        // 5. merge and store; stage position c <-> output gbase + c
        const uint8_t* __restrict__ sm = td->sm;
        uint16_t* __restrict__ out = td->out;
        const uint64_t gbase = out0 & ~15ull;
        const uint32_t vend = align + total;  // decoded stage positions are [align, vend)
        const uint32_t ngroups = total ? (vend + 15) >> 4 : 0;  // a block may hold no code start
        const bool vec = td->vec_ok != 0;
        // 5a. groups inside their owner's range; the others are left to 5b.
        // Two groups per thread and iteration: both sign|fraction loads are
        // in flight before the first merge.
        for (uint32_t g0 = tid; g0 < ngroups; g0 += 2 * T) {
            uint4 sv[2];
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                const uint32_t gi = g0 + k * T;
                const uint64_t G = gbase + 16 * gi;
                sv[k] = make_uint4(0, 0, 0, 0);
                if (vec && gi < ngroups && G >= out0 && 16 * gi + 16 <= vend)
                    sv[k] = __ldg(reinterpret_cast<const uint4*>(sm + G));
            }
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                const uint32_t gi = g0 + k * T;
                if (gi >= ngroups) break;
                const uint32_t c0 = 16 * gi;
                const uint32_t t = s_owner[gi];
                if (c0 + 16 > s_pos[t + 1]) continue;
                const uint64_t G = gbase + c0;
                uint32_t e[4];
                gather16(s_priv, static_cast<int>(t * RB + c0) - static_cast<int>(s_pos[t]), e);
                if (vec && G >= out0) {
                    merge16(sv[k], e, out + G);
                } else {  // the block's first group, or buffers without 16-byte alignment
                    for (uint32_t q = 0; q < 16; ++q) {
                        const uint64_t i = G + q;
                        if (i >= out0) out[i] = merge1(sm[i], static_cast<uint8_t>(e[q >> 2] >> (8 * (q & 3))));
                    }
                }
            }
        }
        // 5b. the group this thread's range ends inside, when it owns that
        // group (then the group runs past the range, into later regions)
        const uint32_t bend = pos + cnt;
        if (cnt && (bend & 15) && s_owner[bend >> 4] == tid) {
            const uint32_t c0 = bend & ~15u;
            const uint64_t G = gbase + c0;
            const uint32_t hi = min(c0 + 16, vend);
            uint32_t e[4];
            if (tid + 1 < T && hi <= s_pos[tid + 2]) {  // two regions: this one and the next
                uint32_t x[4], y[4];
                gather16(s_priv, static_cast<int>(tid * RB + c0) - static_cast<int>(pos), x);
                gather16(s_priv, static_cast<int>((tid + 1) * RB) - static_cast<int>(bend - c0), y);
#pragma unroll
                for (int i = 0; i < 4; ++i) {  // bytes before bend from x, the rest from y
                    const int sbits = 8 * static_cast<int>(bend - c0) - 32 * i;
                    const uint32_t m = sbits >= 32 ? 0xFFFFFFFFu : (sbits <= 0 ? 0u : (1u << sbits) - 1u);
                    e[i] = (x[i] & m) | (y[i] & ~m);
                }
            } else {  // three or more regions, or the last thread
                e[0] = e[1] = e[2] = e[3] = 0;
                uint32_t t = tid;
                for (uint32_t c = max(c0, pos); c < hi; ++c) {
                    while (c >= s_pos[t + 1]) ++t;
                    e[(c - c0) >> 2] |= static_cast<uint32_t>(s_priv[t * RB + (c - s_pos[t])]) << (8 * ((c - c0) & 3));
                }
            }
            const uint64_t lo_i = max(G, out0), hi_i = min(G + 16, out1);
            if (vec && lo_i == G && hi_i == G + 16) {
                merge16(__ldg(reinterpret_cast<const uint4*>(sm + G)), e, out + G);
            } else {
                for (uint64_t i = lo_i; i < hi_i; ++i)
                    out[i] = merge1(sm[i], static_cast<uint8_t>(e[(i - G) >> 2] >> (8 * ((i - G) & 3))));
            }
        }
        __syncthreads();  // the next block overwrites shared memory
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
// needs of its blocks.
df_status prepare(const df_tensor* t, uint16_t* out, Prepared* pr) {
    if (!t || !out) return DF_ERR_INVALID_ARG;
    const uint32_t C = t->chunk_bytes, T = t->threads_per_block;
    if (C < 16 || C > 4096 || C % 16 || T < 32 || T > kMaxThreads || T % 32) return DF_ERR_INVALID_ARG;
    // the state word keeps a bit position below 2^14 (C <= 1024 bytes)
    if (C > 1024) return DF_ERR_UNSUPPORTED;
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
    pr->words_per_chunk = C / 4 + 1;  // the chunk and the next chunk's first word
    // a chunk holds at most 8C/min_len code starts; its region also takes up
    // to 3 exponents past the last counted code and the word they end in
    const uint64_t per_chunk = (cbits + minl - 1) / (minl ? minl : 1);
    uint64_t rb = (per_chunk + 12 + 3) & ~3ull;
    if (((rb / 4) & 1) == 0) rb += 4;  // odd word stride: regions start in distinct banks
    // a block holds at most 8CT/min_len codes and never more than n
    uint64_t per_block = per_chunk * T;
    if (per_block > t->n) per_block = t->n;
    const uint64_t groups = (per_block + 15 + 15) / 16 + 1;
    if (rb > (1u << 20) || groups > 0xFFFFu) return DF_ERR_UNSUPPORTED;
    pr->region_bytes = static_cast<uint32_t>(rb);
    pr->max_groups = static_cast<uint32_t>(groups);
    return DF_OK;
}

// owner-map entries are bytes when a block has at most 256 threads
size_t owner_size(uint32_t T) { return T <= 256 ? 1 : 2; }

size_t smem_bytes(const LaunchCfg& c, uint32_t T) {
    return 8u * kWideN + ((static_cast<size_t>(T) * c.words_per_chunk + 3) & ~static_cast<size_t>(3)) * 4 +
           ((T + 1 + 3) & ~3u) * 4 + 32 * 4 + 16 + sizeof(DevTensor) + ((c.max_groups * owner_size(T) + 15) & ~static_cast<size_t>(15)) +
           static_cast<size_t>(T) * c.region_bytes;
}

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

template <class Src, class OwnerT>
df_status launch_as(const Src& src, const LaunchCfg& cfg, uint32_t T, size_t smem, uint32_t* d_err,
                    cudaStream_t stream) {
    int sms = 0, max_smem = 0;
    df_status st = device_limits(&sms, &max_smem);
    if (st != DF_OK) return st;
    if (smem > static_cast<size_t>(max_smem)) return DF_ERR_UNSUPPORTED;
    auto kern = T == 256 ? decode_kernel<Src, OwnerT, 256> : decode_kernel<Src, OwnerT, 0>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return cuda_fail(e);
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, static_cast<int>(T), smem);
    if (e != cudaSuccess) return cuda_fail(e);
    if (per_sm < 1) return DF_ERR_UNSUPPORTED;
    // persistent blocks: every resident slot loops over the format blocks
    const uint64_t slots = static_cast<uint64_t>(sms) * per_sm;
    const uint64_t grid = cfg.total_blocks < slots ? cfg.total_blocks : slots;
    kern<<<static_cast<unsigned>(grid), T, smem, stream>>>(src, cfg, d_err);
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e);
    return DF_OK;
}

template <class Src>
df_status launch(const Src& src, const LaunchCfg& cfg, uint32_t T, size_t smem, uint32_t* d_err,
                 cudaStream_t stream) {
    if (cfg.total_blocks == 0) return DF_OK;
    return T <= 256 ? launch_as<Src, uint8_t>(src, cfg, T, smem, d_err, stream)
                    : launch_as<Src, uint16_t>(src, cfg, T, smem, d_err, stream);
}

void widen(LaunchCfg* c, const Prepared& p) {
    c->words_per_chunk = std::max(c->words_per_chunk, p.words_per_chunk);
    c->region_bytes = std::max(c->region_bytes, p.region_bytes);
    c->max_groups = std::max(c->max_groups, p.max_groups);
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
    return launch(src, cfg, t->threads_per_block, smem_bytes(cfg, t->threads_per_block), d_err,
                  static_cast<cudaStream_t>(stream));
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
    uint32_t T = 0;
    LaunchCfg cfg;
    std::memset(&cfg, 0, sizeof(cfg));
    for (uint32_t i = 0; i < count; ++i) {
        const df_tensor* t = tensors + i;
        if (t->n == 0) continue;
        Prepared pr;
        df_status st = prepare(t, d_outs[i], &pr);
        if (st != DF_OK) return st;
        if (!T)
            T = t->threads_per_block;
        else if (T != t->threads_per_block)
            return DF_ERR_INVALID_ARG;
        widen(&cfg, pr);
        dev.push_back(pr.dev);
        start.push_back(start.back() + pr.dev.n_blocks);
    }
    plan->d_ws = d_ws;
    plan->count = static_cast<uint32_t>(dev.size());
    plan->threads_per_block = T;
    plan->words_per_chunk = cfg.words_per_chunk;
    plan->region_bytes = cfg.region_bytes;
    plan->max_groups = cfg.max_groups;
    plan->total_blocks = start.back();
    if (plan->count == 0) return DF_OK;
    const size_t sm = smem_bytes(cfg, T);
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
    cfg.max_groups = plan->max_groups;
    cfg.total_blocks = plan->total_blocks;
    if (smem_bytes(cfg, plan->threads_per_block) != plan->smem_bytes) return DF_ERR_INVALID_ARG;
    return launch(src, cfg, plan->threads_per_block, plan->smem_bytes, d_err, static_cast<cudaStream_t>(stream));
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
