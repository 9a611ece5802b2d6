// Encode path: exponent histogram, then one pass that writes the container.
//
// What is coded (mlx-dfloat, PyPI page, intro bit diagram): the 8 exponent
// bits of each BF16 weight become a variable-length code; the sign and the 7
// fraction bits become one raw byte. The codebook comes from the exponent
// frequencies (df11pack, GitHub page, intro). The stream layout (MSB-first
// bits, C-byte chunks with 5-bit start gaps, per-block output offsets) is the
// one df11.h defines.
//
// One encode kernel after the histogram: persistent CUDA blocks of 8 warps,
// each over a contiguous range of 512-weight warp tiles (16 consecutive
// weights per lane), taken in launch order from a counter. Pass 1 writes the
// sign|fraction bytes of the range and sums its code lengths; the range's
// first stream bit comes from a decoupled look-back over the ranges before it
// (warp 0, 128 predecessors per poll, bounded waits). Pass 2 packs warp tile
// by warp tile: a warp scan of the lanes' bit counts places every lane's
// codes (at most 64 bits in one register in the common case) in the tile's
// stream words in shared memory; a lane's code-end mask gives the code that
// crosses a chunk boundary, hence that chunk's gap and, at a format-block
// boundary, the block offset. Whole words go out with plain stores, the
// words a tile shares with its neighbours with atomic ORs into the zeroed
// buffers. The input is read three times in all: by the histogram and by
// both passes; each pass asks for its input two warp tiles ahead (an L2
// prefetch hint).
//
// The grouped encode does the same for many tensors with one launch per
// step: a histogram kernel over fixed tiles of every tensor, a kernel that
// zeroes every tensor's outputs, and an encode kernel whose persistent CUDA
// blocks take ranges of every tensor from one counter and run the same range
// code (encode_range) on each, the range's tensor found by binary search.
#include <cuda_runtime.h>

#include <cstddef>
#include <cstring>
#include <mutex>
#include <vector>

#include "df_internal.h"

namespace df {
namespace {

constexpr uint32_t kTile = 4096;
constexpr uint32_t kEncThreads = 256;
constexpr uint32_t kPerThread = kTile / kEncThreads;  // 16 consecutive weights per thread

__device__ __forceinline__ uint32_t bswap32(uint32_t x) { return __byte_perm(x, 0, 0x0123); }

__global__ void __launch_bounds__(256) hist_kernel(const uint16_t* __restrict__ in, uint64_t n, int vec,
                                                   unsigned long long* __restrict__ hist) {
    __shared__ uint32_t sh[8][256];
    const uint32_t warp = threadIdx.x >> 5;
    for (uint32_t i = threadIdx.x; i < 8 * 256; i += blockDim.x) (&sh[0][0])[i] = 0;
    __syncthreads();
    const uint64_t stride = static_cast<uint64_t>(gridDim.x) * blockDim.x;
    uint64_t done = 0;
    if (vec) {
        const uint64_t n8 = n / 8;
        const uint4* in4 = reinterpret_cast<const uint4*>(in);
        for (uint64_t i = static_cast<uint64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n8; i += stride) {
            const uint4 v = __ldg(in4 + i);
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                atomicAdd(&sh[warp][(w[k] >> 7) & 0xFFu], 1u);
                atomicAdd(&sh[warp][(w[k] >> 23) & 0xFFu], 1u);
            }
        }
        done = n8 * 8;
    }
    for (uint64_t i = done + static_cast<uint64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n; i += stride)
        atomicAdd(&sh[warp][(__ldg(in + i) >> 7) & 0xFFu], 1u);
    __syncthreads();
    for (uint32_t s = threadIdx.x; s < 256; s += blockDim.x) {
        uint32_t c = 0;
#pragma unroll
        for (int w = 0; w < 8; ++w) c += sh[w][s];
        if (c) atomicAdd(hist + s, static_cast<unsigned long long>(c));
    }
}

struct EncTables {
    uint32_t codes[256];
    uint8_t lengths[256];
};

// The 16 consecutive weights of a thread from weight i0 on, two per 32-bit
// word (weight i0 + k in bits 16 * (k & 1) of word k / 2); weights at or past n
// read as 0. Returns how many of the 16 are below n.
__device__ __forceinline__ uint32_t load16(const uint16_t* __restrict__ in, uint64_t n, uint64_t i0, bool vec,
                                           uint32_t wv[kPerThread / 2]) {
    const bool full = i0 + kPerThread <= n;
    if (full && vec) {
        const uint4* p4 = reinterpret_cast<const uint4*>(in + i0);
        const uint4 v0 = __ldg(p4), v1 = __ldg(p4 + 1);
        wv[0] = v0.x; wv[1] = v0.y; wv[2] = v0.z; wv[3] = v0.w;
        wv[4] = v1.x; wv[5] = v1.y; wv[6] = v1.z; wv[7] = v1.w;
    } else {
#pragma unroll
        for (uint32_t k = 0; k < kPerThread / 2; ++k) {
            const uint64_t i = i0 + 2 * k;
            const uint32_t lo = i < n ? __ldg(in + i) : 0u;
            const uint32_t hi = i + 1 < n ? __ldg(in + i + 1) : 0u;
            wv[k] = lo | (hi << 16);
        }
    }
    return full ? kPerThread : (i0 < n ? static_cast<uint32_t>(n - i0) : 0u);
}

// Hint that weight i (below n) of `in` will be read soon: its line is
// fetched into L2 now. No effect on results.
__device__ __forceinline__ void prefetch_l2(const uint16_t* in, uint64_t n, uint64_t i) {
    if (i < n) asm volatile("prefetch.global.L2 [%0];" ::"l"(in + i));
}

struct alignas(16) EncArgs {
    const uint16_t* in;
    uint64_t n;
    uint32_t* stream32;     // the stream as 32-bit words (zeroed)
    uint32_t* gaps32;       // the gap fields as 32-bit words (zeroed)
    uint64_t* offsets;      // block offsets (zeroed)
    uint8_t* sm;
    unsigned long long* state;  // per tile: (kAggregate | bits) or (kPrefix | bits up to its end); zeroed
    uint32_t* ticket;           // tile counter (zeroed)
    uint64_t total_bits;        // the planned stream length
    uint64_t n_chunks;
    uint64_t stream_words;      // words the stream buffer holds: writes beyond are refused
    uint64_t gap_words;         // words the gap buffer holds
    uint64_t n_blocks;
    uint32_t chunk_bits;
    uint32_t threads_per_block;  // T: chunks per format block
    uint32_t tiles;
    uint32_t* err;
    uint32_t in_vec;    // input 16-byte aligned
    uint32_t sm_vec;    // sign|fraction output 16-byte aligned
    uint32_t cb_shift;  // log2(chunk_bits) when it is a power of two, else 32
    uint32_t t_shift;   // log2(threads_per_block) when it is a power of two, else 32
};

// x / d and x % d, by a shift and a mask when d = 2^sh (sh < 32)
__device__ __forceinline__ uint32_t div_by(uint32_t x, uint32_t d, uint32_t sh) { return sh < 32 ? x >> sh : x / d; }
__device__ __forceinline__ uint32_t mod_by(uint32_t x, uint32_t d, uint32_t sh) {
    return sh < 32 ? x & (d - 1) : x % d;
}

constexpr unsigned long long kAggregate = 1ull << 62;  // a tile's own bit count is published
constexpr unsigned long long kPrefix = 2ull << 62;     // ... and the bits of all tiles up to its end
constexpr unsigned long long kValue = (1ull << 62) - 1;
constexpr uint32_t kSpinLimit = 1u << 20;  // polls of a predecessor before giving up (DF_EFLAG_ENC_WAIT)

__device__ __forceinline__ unsigned long long ld_acquire(const unsigned long long* p) {
    unsigned long long v;
    asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void st_release(unsigned long long* p, unsigned long long v) {
    asm volatile("st.release.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

__device__ __forceinline__ uint64_t warp_sum64(uint64_t x) {
#pragma unroll
    for (int d = 16; d > 0; d >>= 1) x += __shfl_xor_sync(0xFFFFFFFFu, x, d);
    return x;
}

// The stream bits before range `tile` (warp 0): decoupled look-back over the
// ranges before it, 128 at a time (4 per lane, polled together). Every range
// publishes its own bit count as soon as it has it and its prefix once it
// knows it; ranges take their index from a counter in launch order, so a range
// only waits on ranges whose CUDA blocks are already running. Each wait is
// bounded: when a predecessor stays silent for kSpinLimit polls, the error
// word gets DF_EFLAG_ENC_WAIT and the range goes on with what it has (its
// output is then wrong, and flagged).
constexpr uint32_t kLookPerLane = 4;

__device__ uint64_t look_back(const EncArgs& a, uint32_t tile, uint64_t total, uint32_t lane) {
    if (tile == 0) {
        if (lane == 0) st_release(a.state, kPrefix | total);
        return 0;
    }
    if (lane == 0) st_release(a.state + tile, kAggregate | total);
    uint64_t acc = 0;
    int64_t top = static_cast<int64_t>(tile) - 1;  // the nearest predecessor not yet accounted for
    uint32_t spins = 0;
    for (;;) {
        // entry q of this lane: predecessor top - (4 lane + q), at distance 4 lane + q
        unsigned long long v[kLookPerLane];
#pragma unroll
        for (uint32_t q = 0; q < kLookPerLane; ++q) {
            const int64_t i = top - static_cast<int64_t>(kLookPerLane * lane + q);
            v[q] = i >= 0 ? ld_acquire(a.state + i) : kPrefix;  // before tile 0: prefix 0
        }
        for (;;) {
            bool wait = false;
#pragma unroll
            for (uint32_t q = 0; q < kLookPerLane; ++q) wait |= (v[q] >> 62) == 0;
            if (!__any_sync(0xFFFFFFFFu, wait)) break;
            const bool give_up = ++spins > kSpinLimit;
            if (give_up && lane == 0 && a.err) atomicOr(a.err, DF_EFLAG_ENC_WAIT);
#pragma unroll
            for (uint32_t q = 0; q < kLookPerLane; ++q) {
                if ((v[q] >> 62) == 0) {
                    const int64_t i = top - static_cast<int64_t>(kLookPerLane * lane + q);
                    v[q] = give_up ? kPrefix : ld_acquire(a.state + i);
                }
            }
        }
        // the nearest tile with a prefix ends the walk
        uint32_t qpre = kLookPerLane;
#pragma unroll
        for (int q = kLookPerLane - 1; q >= 0; --q)
            if ((v[q] >> 62) == 2) qpre = q;
        const uint32_t pre = __ballot_sync(0xFFFFFFFFu, qpre < kLookPerLane);
        const uint32_t lp = pre ? __ffs(pre) - 1 : 32u;  // the nearest lane with one
        const uint32_t qlim = lane < lp ? kLookPerLane : (lane == lp ? qpre + 1 : 0u);
        uint64_t x = 0;
#pragma unroll
        for (uint32_t q = 0; q < kLookPerLane; ++q) x += q < qlim ? (v[q] & kValue) : 0;
        acc += warp_sum64(x);
        if (pre) break;
        top -= 32 * kLookPerLane;
    }
    if (lane == 0) st_release(a.state + tile, kPrefix | (acc + total));
    return acc;
}

// Code lengths of a thread's weights, their sum, and whether an exponent
// without a code occurs (kFull: all 16 weights are below n).
template <bool kFull>
__device__ __forceinline__ uint32_t length_sum(const uint2* s_cl, const uint32_t wv[kPerThread / 2], uint32_t cnt,
                                               bool* missing) {
    uint32_t sum = 0;
#pragma unroll
    for (uint32_t k = 0; k < kPerThread; ++k) {
        const uint32_t l = (kFull || k < cnt) ? s_cl[(wv[k >> 1] >> (16 * (k & 1) + 7)) & 0xFFu].y : 1u;
        *missing |= l == 0;
        sum += (kFull || k < cnt) ? l : 0u;
    }
    return sum;
}

// The code lengths' sum and, when it is at most 64, the codes packed into
// one register MSB-first (the first code in the highest bits of the sum),
// with a mask of the same layout that marks the last bit of every code: a
// code that ends `d` bits after the lane's first bit has its mark at bit
// sum - d.
template <bool kFull>
__device__ __forceinline__ uint32_t pack64(const uint2* s_cl, const uint32_t wv[kPerThread / 2], uint32_t cnt,
                                           unsigned long long* v, unsigned long long* ends) {
    uint32_t sum = 0;
    unsigned long long x = 0, e = 0;
#pragma unroll
    for (uint32_t k = 0; k < kPerThread; ++k) {
        if (kFull || k < cnt) {
            const uint2 cl = s_cl[(wv[k >> 1] >> (16 * (k & 1) + 7)) & 0xFFu];
            x = (x << cl.y) | cl.x;
            e = (e << cl.y) | 1ull;
            sum += cl.y;
        }
    }
    *v = x;
    *ends = e;
    return sum;
}

constexpr uint32_t kWarpTile = 32 * kPerThread;      // 512 weights: a warp, 16 consecutive weights per lane
constexpr uint32_t kPrefetchTiles = 2;  // both passes ask for the input this many warp tiles ahead
constexpr uint32_t kEncWarps = kEncThreads / 32;
constexpr uint32_t kWarpWords = kWarpTile + 2;       // a warp tile holds at most 512 codes of at most 32 bits
// gap fields a warp tile can hold (every code 32 bits, 16-byte chunks) as
// words, plus the partial words at both ends
constexpr uint32_t kWarpGapWords = (5 * (kWarpTile * 32 / 128 + 2) + 31) / 32 + 4;

// Persistent CUDA blocks, each over a contiguous range of the tensor's warp
// tiles (512 weights, 16 consecutive weights per lane), split into one
// sub-range per warp, in two passes:
//   1. every warp writes the sign|fraction bytes of its sub-range and sums
//      its code lengths; the CUDA block's range gets its stream offset from a
//      look-back over the ranges before it (once per CUDA block), and every
//      warp its own from the sums of the warps before it
//   2. every warp packs its tiles on its own, with no block-wide barrier: a
//      warp scan of the lanes' code-length sums gives every code its bit
//      offset; each lane packs its codes MSB-first into a 64-bit register and
//      writes the tile's words in the warp's shared memory, whole words with
//      plain stores and the two partial words it shares with its neighbours
//      with shared OR. The code that crosses or ends on a chunk boundary
//      writes that chunk's gap into the warp's gap words (and, at a
//      format-block boundary, the block offset). The tile's stream and gap
//      words go out with coalesced stores, except the end words shared with
//      the neighbouring tiles, which are OR-ed into the zeroed buffers.
//
// encode_range does one range with the whole CUDA block: range `range` of
// the R into which the tensor `a` describes is split, sh.cl holding its code.
// It has two block-wide barriers of its own (after pass 1 and after the
// look-back) and none at its start or end: the caller fills sh.cl and a
// before a barrier and synchronises again before it overwrites them.
struct EncShared {
    uint2 cl[256];  // per exponent: (code right-aligned, length)
    unsigned long long sum[kEncWarps];
    unsigned long long pre[kEncWarps];
    uint32_t words[kEncWarps][kWarpWords];
    uint32_t gaps[kEncWarps][kWarpGapWords];
};

__device__ __forceinline__ void encode_range(const EncArgs& a, EncShared& sh, uint64_t range, uint64_t R) {
    const uint32_t tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const uint2* s_cl = sh.cl;
    unsigned long long* s_sum = sh.sum;
    unsigned long long* s_pre = sh.pre;
    const uint64_t wtiles = (a.n + kWarpTile - 1) / kWarpTile;
    // balanced contiguous splits (no products that could overflow)
    const uint64_t r_begin = (wtiles / R) * range + min(range, wtiles % R);
    const uint64_t r_len = wtiles / R + (range < wtiles % R ? 1 : 0);
    const uint64_t t_begin = r_begin + (r_len / kEncWarps) * warp + min(static_cast<uint64_t>(warp), r_len % kEncWarps);
    const uint64_t t_end = t_begin + r_len / kEncWarps + (warp < r_len % kEncWarps ? 1 : 0);

    // 1. sign|fraction bytes and the bit count of this warp's sub-range
    uint64_t lsum = 0;
    bool missing = false;
    for (uint32_t d = 1; d < kPrefetchTiles; ++d)
        if (t_begin + d < t_end) prefetch_l2(a.in, a.n, (t_begin + d) * kWarpTile + lane * kPerThread);
    for (uint64_t t = t_begin; t < t_end; ++t) {
        const uint64_t i0 = t * kWarpTile + lane * kPerThread;
        if (t + kPrefetchTiles < t_end) prefetch_l2(a.in, a.n, i0 + kPrefetchTiles * kWarpTile);
        uint32_t wv[kPerThread / 2];
        const uint32_t cnt = load16(a.in, a.n, i0, a.in_vec != 0, wv);
        uint32_t smw[kPerThread / 4];
#pragma unroll
        for (uint32_t k = 0; k < kPerThread / 4; ++k) {
            const uint32_t x = wv[2 * k], y = wv[2 * k + 1];
            // byte j of the word: (w >> 8 & 0x80) | (w & 0x7F) of weight 4k + j
            const uint32_t hi = __byte_perm(x, y, 0x7531) & 0x80808080u;
            const uint32_t lo = __byte_perm(x, y, 0x6420) & 0x7F7F7F7Fu;
            smw[k] = hi | lo;
        }
        if (cnt == kPerThread && a.sm_vec) {
            *reinterpret_cast<uint4*>(a.sm + i0) = make_uint4(smw[0], smw[1], smw[2], smw[3]);
        } else {
            for (uint32_t k = 0; k < cnt; ++k) a.sm[i0 + k] = static_cast<uint8_t>(smw[k >> 2] >> (8 * (k & 3)));
        }
        lsum += cnt == kPerThread ? length_sum<true>(s_cl, wv, cnt, &missing) : length_sum<false>(s_cl, wv, cnt, &missing);
    }
    const uint64_t wsum = warp_sum64(lsum);
    if (lane == 0) s_sum[warp] = wsum;
    if (__syncthreads_or(missing) && tid == 0 && a.err) atomicOr(a.err, DF_EFLAG_ENC_SYMBOL);
    if (warp == 0) {
        uint64_t total = 0, before = 0;
#pragma unroll
        for (uint32_t w = 0; w < kEncWarps; ++w) {
            const uint64_t v = s_sum[w];
            before += w < lane ? v : 0;
            total += v;
        }
        const uint64_t pre = look_back(a, static_cast<uint32_t>(range), total, lane);
        if (lane < kEncWarps) s_pre[lane] = pre + before;
    }
    __syncthreads();

    // 2. pack, warp tile by warp tile
    uint32_t* words = sh.words[warp];
    uint32_t* gapw = sh.gaps[warp];
    const uint32_t cbits = a.chunk_bits, T = a.threads_per_block, csh = a.cb_shift, tsh = a.t_shift;
    uint64_t bit0 = s_pre[warp];              // the first stream bit of the next tile
    uint32_t rr = static_cast<uint32_t>(bit0 % cbits);  // bit0 = jc * cbits + rr
    uint64_t jc = bit0 / cbits;
    uint32_t jcT = static_cast<uint32_t>(jc % T);
    for (uint32_t d = 1; d < kPrefetchTiles; ++d)
        if (t_begin + d < t_end) prefetch_l2(a.in, a.n, (t_begin + d) * kWarpTile + lane * kPerThread);
    for (uint64_t t = t_begin; t < t_end; ++t) {
        const uint64_t i0 = t * kWarpTile + lane * kPerThread;
        if (t + kPrefetchTiles < t_end) prefetch_l2(a.in, a.n, i0 + kPrefetchTiles * kWarpTile);
        uint32_t wv[kPerThread / 2];
        const uint32_t cnt = load16(a.in, a.n, i0, a.in_vec != 0, wv);
        unsigned long long v, ends;
        const uint32_t sum =
            cnt == kPerThread ? pack64<true>(s_cl, wv, cnt, &v, &ends) : pack64<false>(s_cl, wv, cnt, &v, &ends);
        uint32_t incl = sum;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const uint32_t u = __shfl_up_sync(0xFFFFFFFFu, incl, d);
            if (lane >= static_cast<uint32_t>(d)) incl += u;
        }
        const uint32_t total = __shfl_sync(0xFFFFFFFFu, incl, 31);
        const uint32_t head = static_cast<uint32_t>(bit0 & 31);  // bits of the first word before the tile
        const uint32_t nw = (head + total + 31) >> 5;          // words the tile touches
        for (uint32_t k = lane; k < nw; k += 32) words[k] = 0;
        if (lane < kWarpGapWords) gapw[lane] = 0;
        // chunk boundaries in tile-relative bits: B0 + m * cbits is the start of
        // chunk jt0 + m. This tile writes the gaps of the boundaries B with
        // 0 < B <= total (the code that crosses or ends on B starts before it);
        // a boundary at 0 belongs to the previous tile's last code.
        const uint32_t B0 = rr ? cbits - rr : 0u;
        const uint64_t jt0 = jc + (rr ? 1u : 0u);
        const uint64_t j_first = jt0 + (B0 == 0 ? 1u : 0u);
        const uint32_t gw0 = static_cast<uint32_t>((5 * j_first) >> 5);  // the tile's first gap word
        const uint32_t jt0_mod_T = mod_by(jcT + (rr ? 1u : 0u), T, tsh);
        __syncwarp();  // zeroed

        // this lane's codes into the tile's words
        const uint32_t off = incl - sum;  // this lane's first bit within the tile
        const uint32_t q = head + off;
        uint32_t* wp = words + (q >> 5);
        const uint32_t sh = q & 31;  // bits of the first word before this lane's
        if (sum <= 64) {
            // the packed codes placed at bit sh of a three-word window (only
            // the first and last words are shared with the neighbours)
            if (sum) {
                const unsigned long long x = v << (64 - sum);  // left-aligned
                const uint32_t xh = static_cast<uint32_t>(x >> 32), xl = static_cast<uint32_t>(x);
                const uint32_t n = (sh + sum + 31) >> 5;  // words touched: 1..3
                atomicOr(wp, xh >> sh);
                if (n == 2) atomicOr(wp + 1, __funnelshift_r(xl, xh, sh));
                if (n == 3) {
                    wp[1] = __funnelshift_r(xl, xh, sh);
                    atomicOr(wp + 2, xl << (32 - sh));
                }
            }
        } else {  // longer codes: a running 64-bit register, whole words as they fill
            uint32_t nbits = sh;
            unsigned long long acc = 0;  // pending bits, left-aligned
            bool first = true;
#pragma unroll
            for (uint32_t k = 0; k < kPerThread; ++k) {
                const uint2 cl = k < cnt ? s_cl[(wv[k >> 1] >> (16 * (k & 1) + 7)) & 0xFFu] : make_uint2(0u, 0u);
                if (cl.y) {
                    acc |= (static_cast<unsigned long long>(cl.x << (32 - cl.y)) << 32) >> nbits;
                    nbits += cl.y;
                    if (nbits >= 32) {
                        const uint32_t word = static_cast<uint32_t>(acc >> 32);
                        if (first)
                            atomicOr(wp, word);
                        else
                            *wp = word;
                        first = false;
                        ++wp;
                        acc <<= 32;
                        nbits -= 32;
                    }
                }
            }
            if (nbits) atomicOr(wp, static_cast<uint32_t>(acc >> 32));
        }
        // chunk boundaries in (off, off + sum]: the code that crosses or ends on
        // one writes its chunk's gap (the next code start - the boundary) and,
        // at a format-block boundary, the block offset
        uint32_t m = off < B0 ? 0u : div_by(off - B0, cbits, csh) + 1;
        uint32_t nb = B0 + m * cbits;  // the first boundary after this lane's start
        if (nb <= off + sum && sum <= 64) {
            // a chunk (at least 128 bits) holds this lane's codes at most once:
            // one boundary; the code that crosses or ends on it is the first
            // whose end is at or past it, i.e. the highest end mark at or
            // below bit sum - (nb - off) (the last code's mark, bit 0, always is)
            const uint32_t jmax = sum - (nb - off);
            const unsigned long long cand = jmax >= 63 ? ends : (ends & ((2ull << jmax) - 1ull));
            const uint32_t jb = 63u - static_cast<uint32_t>(__clzll(cand));
            const uint32_t end = off + sum - jb;
            const uint32_t codes = static_cast<uint32_t>(__popcll(ends >> jb));  // up to and with that code
            const uint64_t j = jt0 + m;
            if (j < a.n_chunks) {
                const uint64_t gq = 5 * j;
                const uint32_t gw = static_cast<uint32_t>(gq >> 5) - gw0;
                const uint32_t o = static_cast<uint32_t>(gq & 31);
                const uint32_t g = end - nb;
                if (o <= 27) {
                    atomicOr(gapw + gw, g << (27 - o));
                } else {
                    atomicOr(gapw + gw, g >> (o - 27));
                    atomicOr(gapw + gw + 1, g << (59 - o));
                }
                if (mod_by(jt0_mod_T + m, T, tsh) == 0) a.offsets[tsh < 32 ? j >> tsh : j / T] = i0 + codes;
            }
        } else if (nb <= off + sum) {  // longer codes: walk them
            uint32_t end = off;
#pragma unroll
            for (uint32_t k = 0; k < kPerThread; ++k) {
                const uint32_t l = k < cnt ? s_cl[(wv[k >> 1] >> (16 * (k & 1) + 7)) & 0xFFu].y : 0u;
                end += l;
                if (l && end >= nb) {
                    const uint64_t j = jt0 + m;
                    if (j < a.n_chunks) {
                        const uint64_t gq = 5 * j;
                        const uint32_t gw = static_cast<uint32_t>(gq >> 5) - gw0;
                        const uint32_t o = static_cast<uint32_t>(gq & 31);
                        const uint32_t g = end - nb;
                        if (o <= 27) {
                            atomicOr(gapw + gw, g << (27 - o));
                        } else {
                            atomicOr(gapw + gw, g >> (o - 27));
                            atomicOr(gapw + gw + 1, g << (59 - o));
                        }
                        if (mod_by(jt0_mod_T + m, T, tsh) == 0) a.offsets[tsh < 32 ? j >> tsh : j / T] = i0 + k + 1;
                    }
                    ++m;
                    nb += cbits;
                }
            }
        }
        if (t + 1 == wtiles && lane == 0) {  // the last tile closes the stream
            if (bit0 + total != a.total_bits && a.err) atomicOr(a.err, DF_EFLAG_ENC_TOTAL);
            a.offsets[a.n_blocks] = a.n;
        }
        __syncwarp();
        // out: whole words inside the tile are stored, the two edge words OR-ed in
        const uint64_t w0 = bit0 >> 5;
        for (uint32_t k = lane; k < nw; k += 32) {
            const uint64_t W = w0 + k;
            const uint32_t val = bswap32(words[k]);
            if (W >= a.stream_words) {
                if (a.err) atomicOr(a.err, DF_EFLAG_ENC_TOTAL);
            } else if (k == 0 || k + 1 == nw) {
                if (val) atomicOr(a.stream32 + W, val);
            } else {
                a.stream32[W] = val;
            }
        }
        // the tile's gap fields: chunks j_first .. j_last; the words at both
        // ends may hold fields of the neighbouring tiles
        if (total >= B0) {
            uint64_t j_last = jt0 + div_by(total - B0, cbits, csh);
            if (j_last >= a.n_chunks) j_last = a.n_chunks - 1;
            if (j_last >= j_first) {
                const uint32_t gwn = static_cast<uint32_t>((5 * j_last + 4) >> 5) - gw0 + 1;
                for (uint32_t k = lane; k < gwn; k += 32) {
                    const uint64_t W = gw0 + k;
                    const uint32_t val = bswap32(gapw[k]);
                    if (W >= a.gap_words) continue;
                    if (k == 0 || k + 1 == gwn) {
                        if (val) atomicOr(a.gaps32 + W, val);
                    } else {
                        a.gaps32[W] = val;
                    }
                }
            }
        }
        __syncwarp();  // the next tile zeroes the words
        bit0 += total;
        const uint32_t rn = rr + total;
        const uint32_t qn = div_by(rn, cbits, csh);
        jc += qn;
        jcT = mod_by(jcT + qn, T, tsh);
        rr = rn - qn * cbits;
    }
}

// One tensor: one range per CUDA block, taken in launch order.
__global__ void __launch_bounds__(kEncThreads) encode_kernel(EncArgs a, EncTables tab) {
    __shared__ EncShared sh;
    __shared__ uint32_t s_range;
    const uint32_t tid = threadIdx.x;
    if (tid == 0) s_range = atomicAdd(a.ticket, 1u);  // ranges start in index order
    for (uint32_t i = tid; i < 256; i += kEncThreads) sh.cl[i] = make_uint2(tab.codes[i], tab.lengths[i]);
    __syncthreads();
    encode_range(a, sh, s_range, gridDim.x);
}

// The index t of the entry with starts[t] <= g < starts[t + 1] (starts
// non-decreasing, starts[0] = 0 <= g < starts[count]): the tensor that holds
// unit g of a grouped launch; tensors without units are skipped.
__device__ __forceinline__ uint32_t tensor_at(const uint64_t* __restrict__ starts, uint32_t count, uint64_t g) {
    uint32_t lo = 0, hi = count;
    while (hi - lo > 1) {
        const uint32_t mid = (lo + hi) >> 1;
        if (__ldg(starts + mid) <= g)
            lo = mid;
        else
            hi = mid;
    }
    return lo;
}

// Grouped encode of many tensors in one launch: persistent CUDA blocks take
// ranges from one counter in index order (a tensor's ranges are consecutive,
// rstart[t] .. rstart[t + 1]); a range's tensor comes from a binary search,
// its descriptor and code are copied to shared memory, and the range is
// encoded as encode_kernel does it. Each descriptor's look-back state is its
// own, so a tensor's first range publishes its prefix at once and no range
// waits on another tensor's.
__global__ void __launch_bounds__(kEncThreads)
    encode_batch_kernel(const EncArgs* __restrict__ descs, const uint2* __restrict__ codes,
                        const uint64_t* __restrict__ rstart, uint32_t count, uint32_t* ticket, uint32_t* err) {
    __shared__ EncShared sh;
    __shared__ EncArgs s_a;
    __shared__ unsigned long long s_g, s_range, s_R;
    __shared__ uint32_t s_t;
    constexpr uint32_t kArgWords = sizeof(EncArgs) / 4;
    constexpr uint32_t kErrWord = offsetof(EncArgs, err) / 4;
    const uint32_t tid = threadIdx.x;
    const uint64_t total = __ldg(rstart + count);
    for (;;) {
        if (tid == 0) {
            const uint64_t g = atomicAdd(ticket, 1u);  // ranges start in index order
            s_g = g;
            if (g < total) {
                const uint32_t t = tensor_at(rstart, count, g);
                s_t = t;
                s_range = g - __ldg(rstart + t);
                s_R = __ldg(rstart + t + 1) - __ldg(rstart + t);
            }
        }
        __syncthreads();  // the last range is done with s_a and sh
        if (s_g >= total) break;
        const uint32_t t = s_t;
        const uint32_t* src = reinterpret_cast<const uint32_t*>(descs + t);
        uint32_t* dst = reinterpret_cast<uint32_t*>(&s_a);
        for (uint32_t i = tid; i < kArgWords; i += kEncThreads)
            if (i != kErrWord && i != kErrWord + 1) dst[i] = __ldg(src + i);
        if (tid == 0) s_a.err = err;
        for (uint32_t i = tid; i < 256; i += kEncThreads) sh.cl[i] = __ldg(codes + 256ull * t + i);
        const uint64_t range = s_range, R = s_R;
        __syncthreads();
        encode_range(s_a, sh, range, R);
    }
}

// Zeroes the stream, gap and block-offset words of every tensor of a grouped
// encode (the encoder ORs the words that neighbouring warp tiles share): one
// CUDA block per kZeroTileWords words of one tensor, zstart[t] .. zstart[t+1]
// being tensor t's tiles.
constexpr uint32_t kZeroTileWords = 4096;

__global__ void __launch_bounds__(256)
    zero_batch_kernel(const EncArgs* __restrict__ descs, const uint64_t* __restrict__ zstart, uint32_t count) {
    const uint32_t t = tensor_at(zstart, count, blockIdx.x);
    const EncArgs& d = descs[t];
    const uint64_t zs = d.stream_words, zg = d.gap_words, zo = 2 * (d.n_blocks + 1);
    const uint64_t w0 = (blockIdx.x - __ldg(zstart + t)) * kZeroTileWords;
    const uint64_t w1 = min(w0 + kZeroTileWords, zs + zg + zo);
    uint32_t* stream32 = d.stream32;
    uint32_t* gaps32 = d.gaps32;
    uint32_t* offs32 = reinterpret_cast<uint32_t*>(d.offsets);
    for (uint64_t w = w0 + threadIdx.x; w < w1; w += blockDim.x) {
        if (w < zs)
            stream32[w] = 0;
        else if (w < zs + zg)
            gaps32[w - zs] = 0;
        else
            offs32[w - zs - zg] = 0;
    }
}

// Exponent histograms of every tensor of a grouped encode: one CUDA block per
// `tile` weights of one tensor (hstart[t] .. hstart[t+1] being tensor t's
// tiles), per-warp shared counters as in hist_kernel, the block's nonzero
// counts added to hist[256 t ..]. tile is a multiple of 8, so a 16-byte
// aligned input stays aligned at every tile start.
__global__ void __launch_bounds__(256)
    hist_batch_kernel(const EncArgs* __restrict__ descs, const uint64_t* __restrict__ hstart, uint32_t count,
                      uint64_t tile, unsigned long long* __restrict__ hist) {
    __shared__ uint32_t sh[8][256];
    const uint32_t warp = threadIdx.x >> 5;
    for (uint32_t i = threadIdx.x; i < 8 * 256; i += blockDim.x) (&sh[0][0])[i] = 0;
    const uint32_t t = tensor_at(hstart, count, blockIdx.x);
    const uint16_t* in = descs[t].in;
    const uint64_t n = descs[t].n;
    const uint64_t b = (blockIdx.x - __ldg(hstart + t)) * tile;
    const uint64_t e = min(n, b + tile);
    __syncthreads();
    uint64_t done = b;
    if (descs[t].in_vec) {
        const uint4* in4 = reinterpret_cast<const uint4*>(in);
        for (uint64_t i = b / 8 + threadIdx.x; i < e / 8; i += blockDim.x) {
            const uint4 v = __ldg(in4 + i);
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                atomicAdd(&sh[warp][(w[k] >> 7) & 0xFFu], 1u);
                atomicAdd(&sh[warp][(w[k] >> 23) & 0xFFu], 1u);
            }
        }
        done = e / 8 * 8;
    }
    for (uint64_t i = done + threadIdx.x; i < e; i += blockDim.x)
        atomicAdd(&sh[warp][(__ldg(in + i) >> 7) & 0xFFu], 1u);
    __syncthreads();
    for (uint32_t s = threadIdx.x; s < 256; s += blockDim.x) {
        uint32_t c = 0;
#pragma unroll
        for (int w = 0; w < 8; ++w) c += sh[w][s];
        if (c) atomicAdd(hist + 256ull * t + s, static_cast<unsigned long long>(c));
    }
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

df_status sm_count(int* sms) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e);
    e = cudaDeviceGetAttribute(sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return cuda_fail(e);
    return DF_OK;
}

// The descriptor of one tensor's encode for a container of total_bits code
// bits under chunk_bytes and tpb (the sizes df_container_sizes gives); the
// look-back state, the range counter and the error word are left to the caller.
EncArgs make_args(const uint16_t* in, uint64_t n, uint64_t total_bits, uint32_t chunk_bytes, uint32_t tpb,
                  uint8_t* stream, uint8_t* gaps, uint64_t* offsets, uint8_t* sm) {
    const uint64_t cbits = 8ull * chunk_bytes;
    const uint64_t n_chunks = total_bits ? (total_bits + cbits - 1) / cbits : 1;
    EncArgs a;
    std::memset(&a, 0, sizeof(a));
    a.in = in;
    a.n = n;
    a.stream32 = reinterpret_cast<uint32_t*>(stream);
    a.gaps32 = reinterpret_cast<uint32_t*>(gaps);
    a.offsets = offsets;
    a.sm = sm;
    a.state = nullptr;
    a.ticket = nullptr;
    a.total_bits = total_bits;
    a.n_chunks = n_chunks;
    a.stream_words = (n_chunks * chunk_bytes + 16) / 4;
    a.gap_words = ((((5 * n_chunks + 7) / 8) + 1 + 15) & ~15ull) / 4;
    a.n_blocks = (n_chunks + tpb - 1) / tpb;
    a.chunk_bits = static_cast<uint32_t>(cbits);
    a.threads_per_block = tpb;
    a.tiles = static_cast<uint32_t>((n + kTile - 1) / kTile);
    a.err = nullptr;
    a.in_vec = aligned(in, 16) ? 1u : 0u;
    a.sm_vec = aligned(sm, 16) ? 1u : 0u;
    a.cb_shift = a.t_shift = 32;
    for (uint32_t k = 0; k < 32; ++k) {
        if ((1ull << k) == cbits) a.cb_shift = k;
        if ((1u << k) == tpb) a.t_shift = k;
    }
    return a;
}

bool format_ok(uint32_t chunk_bytes, uint32_t tpb) {
    return chunk_bytes >= 16 && chunk_bytes <= 4096 && chunk_bytes % 16 == 0 && tpb >= 32 && tpb <= 1024 &&
           tpb % 32 == 0;
}

// Workspace of a grouped encode: descriptors, codes as (code, length) pairs,
// the unit prefix sums of the histogram, range and zeroing launches, the
// range counter and the look-back states (one per range, at most one per 4096
// weights), each part 16-byte aligned.
struct EncBatchLayout {
    size_t descs, codes, hstart, rstart, zstart, ticket, state, bytes;
};

size_t round16(size_t x) { return (x + 15) & ~static_cast<size_t>(15); }

EncBatchLayout enc_batch_layout(uint32_t count, uint64_t sum_tiles) {
    EncBatchLayout l;
    const size_t c = count;
    size_t o = 0;
    l.descs = o;
    o += round16(sizeof(EncArgs) * c);
    l.codes = o;
    o += sizeof(uint2) * 256 * c;
    l.hstart = o;
    o += round16(8 * (c + 1));
    l.rstart = o;
    o += round16(8 * (c + 1));
    l.zstart = o;
    o += round16(8 * (c + 1));
    l.ticket = o;
    o += 16;
    l.state = o;
    o += 8 * static_cast<size_t>(sum_tiles);
    l.bytes = round16(o);
    return l;
}

// Ranges of one tensor in a grouped encode: at most kBatchRangeTiles warp
// tiles each (several per large tensor, so that CUDA blocks interleave over
// tensors), at most one per 4096 weights (the look-back state's size).
constexpr uint64_t kBatchRangeTiles = 64;

uint64_t ranges_of(uint64_t n) {
    if (n == 0) return 0;
    const uint64_t wtiles = (n + kWarpTile - 1) / kWarpTile;
    const uint64_t tiles = (n + kTile - 1) / kTile;
    const uint64_t r = (wtiles + kBatchRangeTiles - 1) / kBatchRangeTiles;
    return r < tiles ? r : tiles;
}

// Scratch of df_encode_noalloc: per-tile bit counts and bases for at most
// DF_ENCODE_NOALLOC_MAX_WEIGHTS weights, in a file-scope device array of
// 16 * (tiles + 2) + 256 bytes (tiles = 2^29 / 4096): 2 MiB + 288 bytes, the
// workspace df_encode asks for at that size. Host code must not use the
// array's name as a device address; noalloc_scratch() looks the address up.
constexpr uint64_t kNoAllocTiles = DF_ENCODE_NOALLOC_MAX_WEIGHTS / kTile;
static __device__ __align__(256) uint64_t g_noalloc_scratch[2 * (kNoAllocTiles + 2) + 32];
constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mutex;
void* g_noalloc_address[kMaxDevices] = {};

// The device address of the static scratch on the current device. Outside a
// stream capture it is looked up on every call, so a device reset (after
// which the module, and the array, may load elsewhere) never leaves a stale
// address behind; during a capture the address of the last call on this
// device is used (a lookup is not made while the stream captures).
df_status noalloc_scratch(cudaStream_t s, void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e);
    if (dev < 0 || dev >= kMaxDevices) return DF_ERR_UNSUPPORTED;
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    e = cudaStreamIsCapturing(s, &cs);
    if (e != cudaSuccess) return cuda_fail(e);
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    if (cs == cudaStreamCaptureStatusNone || !g_noalloc_address[dev]) {
        if (cs != cudaStreamCaptureStatusNone) return DF_ERR_UNSUPPORTED;  // first call inside a capture
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return cuda_fail(e);
        g_noalloc_address[dev] = p;
    }
    *out = g_noalloc_address[dev];
    return DF_OK;
}

}  // namespace
}  // namespace df

using namespace df;

extern "C" {

df_status df_histogram(const uint16_t* d_in, uint64_t n, uint64_t* d_hist256, void* stream) {
    if (!d_hist256 || (n && !d_in) || !aligned(d_in, 2) || !aligned(d_hist256, 8)) return DF_ERR_INVALID_ARG;
    if (n > DF_MAX_WEIGHTS) return DF_ERR_UNSUPPORTED;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemsetAsync(d_hist256, 0, 256 * sizeof(uint64_t), s);
    if (e != cudaSuccess) return cuda_fail(e);
    if (n == 0) return DF_OK;
    int sms = 0;
    df_status st = sm_count(&sms);
    if (st != DF_OK) return st;
    // at most 2^30 weights per block keeps the 32-bit shared counters exact
    uint64_t grid = (n + 256ull * 8 * 4 - 1) / (256ull * 8 * 4);
    const uint64_t cap = static_cast<uint64_t>(sms) * 8;
    if (grid > cap) grid = cap;
    const uint64_t floor_blocks = (n >> 30) + 1;
    if (grid < floor_blocks) grid = floor_blocks;
    hist_kernel<<<static_cast<unsigned>(grid), 256, 0, s>>>(d_in, n, aligned(d_in, 16) ? 1 : 0,
                                                          reinterpret_cast<unsigned long long*>(d_hist256));
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e);
    return DF_OK;
}

df_status df_encode(const df_code* code, const uint16_t* d_in, uint64_t n, uint64_t total_bits,
                    uint32_t chunk_bytes, uint32_t tpb, uint8_t* d_stream, uint8_t* d_gaps,
                    uint64_t* d_block_offsets, uint8_t* d_sm, void* d_ws, size_t ws_bytes, uint32_t* d_err,
                    void* stream) {
    if (!code || !d_stream || !d_gaps || !d_block_offsets || (n && (!d_in || !d_sm))) return DF_ERR_INVALID_ARG;
    if (chunk_bytes < 16 || chunk_bytes > 4096 || chunk_bytes % 16 || tpb < 32 || tpb > 1024 || tpb % 32)
        return DF_ERR_INVALID_ARG;
    if (!aligned(d_stream, 16) || !aligned(d_gaps, 4) || !aligned(d_block_offsets, 8) || !aligned(d_in, 2))
        return DF_ERR_INVALID_ARG;
    if (n > DF_MAX_WEIGHTS) return DF_ERR_UNSUPPORTED;
    const uint64_t tiles = (n + kTile - 1) / kTile;
    const uint64_t need_ws = 16 * (tiles + 2) + 256;
    if (n && (ws_bytes < need_ws || !d_ws)) return DF_ERR_WORKSPACE;
    if (n && !aligned(d_ws, 16)) return DF_ERR_INVALID_ARG;
    if (tiles > 0x7FFFFFFFull) return DF_ERR_UNSUPPORTED;
    EncArgs a = make_args(d_in, n, total_bits, chunk_bytes, tpb, d_stream, d_gaps, d_block_offsets, d_sm);

    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemsetAsync(d_stream, 0, 4 * a.stream_words, s);
    if (e == cudaSuccess) e = cudaMemsetAsync(d_gaps, 0, 4 * a.gap_words, s);
    if (e == cudaSuccess) e = cudaMemsetAsync(d_block_offsets, 0, 8 * (a.n_blocks + 1), s);
    if (e != cudaSuccess) return cuda_fail(e);
    if (n == 0) return DF_OK;  // empty stream, zero gap, offsets {0, 0}

    EncTables tab;
    std::memcpy(tab.codes, code->codes, sizeof(tab.codes));
    std::memcpy(tab.lengths, code->lengths, sizeof(tab.lengths));
    // workspace: per-tile look-back state, then the tile counter; both zeroed
    e = cudaMemsetAsync(d_ws, 0, 8 * tiles + 16, s);
    if (e != cudaSuccess) return cuda_fail(e);
    a.state = static_cast<unsigned long long*>(d_ws);
    a.ticket = reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(d_ws) + 8 * tiles);
    a.err = d_err;
    // persistent CUDA blocks: as many as are resident at once, at most one per tile
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, encode_kernel, kEncThreads, 0);
    if (e != cudaSuccess) return cuda_fail(e);
    int sms = 0;
    const df_status st = sm_count(&sms);
    if (st != DF_OK) return st;
    const uint64_t slots = static_cast<uint64_t>(sms) * static_cast<uint64_t>(per_sm < 1 ? 1 : per_sm);
    const uint64_t grid = tiles < slots ? tiles : slots;  // at least one warp tile per warp (8 per block)
    encode_kernel<<<static_cast<unsigned>(grid), kEncThreads, 0, s>>>(a, tab);
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e);
    return DF_OK;
}

df_status df_encode_noalloc(const df_code* code, const uint16_t* d_in, uint64_t n, uint64_t total_bits,
                            uint32_t chunk_bytes, uint32_t tpb, uint8_t* d_stream, uint8_t* d_gaps,
                            uint64_t* d_block_offsets, uint8_t* d_sm, uint32_t* d_err, void* stream) {
    if (n > DF_ENCODE_NOALLOC_MAX_WEIGHTS) return DF_ERR_UNSUPPORTED;
    void* ws = nullptr;
    const df_status st = noalloc_scratch(static_cast<cudaStream_t>(stream), &ws);
    if (st != DF_OK) return st;
    return df_encode(code, d_in, n, total_bits, chunk_bytes, tpb, d_stream, d_gaps, d_block_offsets, d_sm, ws,
                     sizeof(g_noalloc_scratch), d_err, stream);
}

size_t df_encode_batch_workspace(const df_encode_tensor* h_tensors, uint32_t count) {
    if (count && !h_tensors) return 0;
    uint64_t sum_tiles = 0;
    for (uint32_t i = 0; i < count; ++i) sum_tiles += (h_tensors[i].n + kTile - 1) / kTile;
    return enc_batch_layout(count, sum_tiles).bytes;
}

df_status df_encode_batch_prepare(const df_encode_tensor* h_tensors, uint32_t count, void* d_ws, size_t ws_bytes,
                                  df_encode_plan* plan, void* stream) {
    if (!plan || (count && (!h_tensors || !d_ws)) || !aligned(d_ws, 16)) return DF_ERR_INVALID_ARG;
    uint32_t with_code = 0;
    uint64_t sum_tiles = 0, total_n = 0;
    for (uint32_t i = 0; i < count; ++i) {
        const df_encode_tensor& t = h_tensors[i];
        if (t.n > DF_MAX_WEIGHTS) return DF_ERR_UNSUPPORTED;
        if ((t.n && !t.in) || !aligned(t.in, 2)) return DF_ERR_INVALID_ARG;
        with_code += t.code ? 1u : 0u;
        sum_tiles += (t.n + kTile - 1) / kTile;
        total_n += t.n;
    }
    if (with_code && with_code != count) return DF_ERR_INVALID_ARG;
    const bool has_codes = count && with_code == count;
    for (uint32_t i = 0; has_codes && i < count; ++i) {
        const df_encode_tensor& t = h_tensors[i];
        if (!format_ok(t.chunk_bytes, t.threads_per_block)) return DF_ERR_INVALID_ARG;
        if (!t.stream || !t.gaps || !t.block_offsets || (t.n && !t.sm)) return DF_ERR_INVALID_ARG;
        if (!aligned(t.stream, 16) || !aligned(t.gaps, 4) || !aligned(t.block_offsets, 8)) return DF_ERR_INVALID_ARG;
        for (uint32_t e = 0; e < 256; ++e)
            if (t.code->lengths[e] > 32) return DF_ERR_INVALID_ARG;
    }
    const EncBatchLayout l = enc_batch_layout(count, sum_tiles);
    if (count && ws_bytes < l.bytes) return DF_ERR_WORKSPACE;
    std::memset(plan, 0, sizeof(*plan));
    plan->d_ws = d_ws;
    if (!count) return DF_OK;

    // histogram tiles: about four CUDA blocks per resident slot over the whole
    // set, 2^16 to 2^20 weights each (a power of two, so a multiple of 8)
    int sms = 0;
    df_status st = sm_count(&sms);
    if (st != DF_OK) return st;
    const uint64_t want = total_n / (4ull * 8 * static_cast<uint64_t>(sms)) + 1;
    uint64_t tile = 1ull << 16;
    while (tile < want && tile < (1ull << 20)) tile <<= 1;

    std::vector<EncArgs> descs(count);
    std::vector<uint2> codes(has_codes ? 256 * static_cast<size_t>(count) : 0);
    std::vector<uint64_t> hstart(static_cast<size_t>(count) + 1, 0), rstart(hstart), zstart(hstart);
    uint8_t* ws = static_cast<uint8_t*>(d_ws);
    for (uint32_t i = 0; i < count; ++i) {
        const df_encode_tensor& t = h_tensors[i];
        if (has_codes) {
            for (uint32_t e = 0; e < 256; ++e)
                codes[256 * static_cast<size_t>(i) + e] = make_uint2(t.code->codes[e], t.code->lengths[e]);
            descs[i] = make_args(t.in, t.n, t.total_bits, t.chunk_bytes, t.threads_per_block, t.stream, t.gaps,
                                 t.block_offsets, t.sm);
            descs[i].state = reinterpret_cast<unsigned long long*>(ws + l.state) + rstart[i];
            const uint64_t words = descs[i].stream_words + descs[i].gap_words + 2 * (descs[i].n_blocks + 1);
            zstart[i + 1] = zstart[i] + (words + kZeroTileWords - 1) / kZeroTileWords;
            rstart[i + 1] = rstart[i] + ranges_of(t.n);
        } else {
            std::memset(&descs[i], 0, sizeof(EncArgs));
            descs[i].in = t.in;
            descs[i].n = t.n;
            descs[i].in_vec = aligned(t.in, 16) ? 1u : 0u;
        }
        hstart[i + 1] = hstart[i] + (t.n + tile - 1) / tile;
    }
    if (hstart[count] > 0x7FFFFFFFull || rstart[count] > 0x7FFFFFFFull || zstart[count] > 0x7FFFFFFFull)
        return DF_ERR_UNSUPPORTED;
    plan->count = count;
    plan->has_codes = has_codes ? 1u : 0u;
    plan->sum_tiles = sum_tiles;
    plan->hist_tiles = hstart[count];
    plan->hist_tile_weights = tile;
    plan->ranges = rstart[count];
    plan->zero_tiles = zstart[count];
    // copies from pageable host memory return once the source has been
    // staged, so the host vectors may die on return
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemcpyAsync(ws + l.descs, descs.data(), sizeof(EncArgs) * descs.size(),
                                    cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess && has_codes)
        e = cudaMemcpyAsync(ws + l.codes, codes.data(), sizeof(uint2) * codes.size(), cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(ws + l.hstart, hstart.data(), 8 * hstart.size(), cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(ws + l.rstart, rstart.data(), 8 * rstart.size(), cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(ws + l.zstart, zstart.data(), 8 * zstart.size(), cudaMemcpyHostToDevice, s);
    return e == cudaSuccess ? DF_OK : cuda_fail(e);
}

df_status df_histogram_batch_run(const df_encode_plan* plan, uint64_t* d_hist, void* stream) {
    if (!plan || (plan->count && (!plan->d_ws || !d_hist)) || !aligned(d_hist, 8)) return DF_ERR_INVALID_ARG;
    if (!plan->count) return DF_OK;
    if (plan->hist_tiles > 0x7FFFFFFFull || plan->hist_tile_weights % 8) return DF_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemsetAsync(d_hist, 0, 256 * sizeof(uint64_t) * plan->count, s);
    if (e != cudaSuccess) return cuda_fail(e);
    if (!plan->hist_tiles) return DF_OK;
    const EncBatchLayout l = enc_batch_layout(plan->count, plan->sum_tiles);
    const uint8_t* ws = static_cast<const uint8_t*>(plan->d_ws);
    hist_batch_kernel<<<static_cast<unsigned>(plan->hist_tiles), 256, 0, s>>>(
        reinterpret_cast<const EncArgs*>(ws + l.descs), reinterpret_cast<const uint64_t*>(ws + l.hstart),
        plan->count, plan->hist_tile_weights, reinterpret_cast<unsigned long long*>(d_hist));
    e = cudaGetLastError();
    return e == cudaSuccess ? DF_OK : cuda_fail(e);
}

df_status df_encode_batch_run(const df_encode_plan* plan, uint32_t* d_err, void* stream) {
    if (!plan || (plan->count && !plan->d_ws)) return DF_ERR_INVALID_ARG;
    if (!plan->count) return DF_OK;
    if (!plan->has_codes || plan->ranges > 0x7FFFFFFFull || plan->zero_tiles > 0x7FFFFFFFull)
        return DF_ERR_INVALID_ARG;
    const EncBatchLayout l = enc_batch_layout(plan->count, plan->sum_tiles);
    uint8_t* ws = static_cast<uint8_t*>(plan->d_ws);
    const EncArgs* descs = reinterpret_cast<const EncArgs*>(ws + l.descs);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (plan->zero_tiles) {
        zero_batch_kernel<<<static_cast<unsigned>(plan->zero_tiles), 256, 0, s>>>(
            descs, reinterpret_cast<const uint64_t*>(ws + l.zstart), plan->count);
        const cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return cuda_fail(e);
    }
    if (!plan->ranges) return DF_OK;
    // the range counter and one look-back state per range, zeroed
    cudaError_t e = cudaMemsetAsync(ws + l.ticket, 0, 16 + 8 * plan->ranges, s);
    if (e != cudaSuccess) return cuda_fail(e);
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, encode_batch_kernel, kEncThreads, 0);
    if (e != cudaSuccess) return cuda_fail(e);
    int sms = 0;
    const df_status st = sm_count(&sms);
    if (st != DF_OK) return st;
    const uint64_t slots = static_cast<uint64_t>(sms) * static_cast<uint64_t>(per_sm < 1 ? 1 : per_sm);
    const uint64_t grid = plan->ranges < slots ? plan->ranges : slots;
    encode_batch_kernel<<<static_cast<unsigned>(grid), kEncThreads, 0, s>>>(
        descs, reinterpret_cast<const uint2*>(ws + l.codes), reinterpret_cast<const uint64_t*>(ws + l.rstart),
        plan->count, reinterpret_cast<uint32_t*>(ws + l.ticket), d_err);
    e = cudaGetLastError();
    return e == cudaSuccess ? DF_OK : cuda_fail(e);
}

}  // extern "C"
