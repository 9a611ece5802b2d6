// The fixed 12-bit format (include/nf12.h): encode and decode kernels.
//
// The format leaves out the top four exponent bits, shared by nearly every
// weight, and packs each group of 8 weights into 12 bytes; a group with any
// other top bits is escaped to a side buffer (agihunt.info, "Developer
// open-sources nf12: lossless 12-bit compression for BF16 models",
// "Confirmed").
//
// Both directions are plain streams over HBM. A CUDA block owns a tile of
// 2048 groups: 8 warps x 256 groups, and lane l of a warp handles groups
// 32 j + l, j = 0..7, of its warp's 256. So for each j a warp reads 384
// contiguous slot bytes (three 32-bit loads per lane) and writes 512
// contiguous weight bytes (one 16-byte store per lane), and the 32 escape
// flags of one j are one ballot, i.e. one bitmap word. All loads of a lane
// are issued before the first store, 24 slot words in flight per lane.
//
// Encode writes side entries in group order. The pass over the groups counts
// escapes per tile; a one-block scan turns the counts into tile bases; a
// second pass over the bitmap (a 64-thread CUDA block per tile, which returns
// at once when its tile has no escapes; escapes are usually 1-2% of groups)
// writes side entries and side indices. The caller reads the total between
// the passes to size the side buffer. The grouped encode runs the same three
// steps once for many tensors: tiles of every tensor in one launch (a tile
// finds its tensor by binary search over the tensors' first tiles), one
// CUDA block per tensor for the scans.
#include <cuda_runtime.h>
#include <stdint.h>

#include <vector>

#include "df_internal.h"
#include "nf12.h"

namespace df {
namespace {

constexpr int kNfThreads = 256;
constexpr int kNfWarps = kNfThreads / 32;
constexpr int kNfPerLane = 8;  // groups per lane in a tile
constexpr uint64_t kTile = DF_NF12_TILE_GROUPS;
static_assert(kNfWarps * 32 * kNfPerLane == DF_NF12_TILE_GROUPS, "a tile is one block's groups");
constexpr int kWordsPerTile = DF_NF12_TILE_GROUPS / 32;
constexpr uint64_t kMaxGroups = 1ull << 32;  // side indices are 32-bit
constexpr int kScanThreads = 1024;

struct Nf12Dev {
    const uint32_t* slots;
    const uint32_t* bitmap;
    const uint4* side;
    uint16_t* out;
    uint64_t n;
    uint64_t n_escaped;
    uint32_t top;
    uint32_t out_vec;  // out is 16-byte aligned
    uint64_t pad;
};
static_assert(sizeof(Nf12Dev) == 64, "descriptors are copied in 64-byte units");

// Two BF16 weights from two 12-bit fields, one in the low 12 bits of each
// 16-bit half of x: the field's sign bit (bit 11) goes to bit 15, its low 11
// bits stay, and the shared top exponent bits fill bits 11..14.
__device__ __forceinline__ uint32_t expand_pair(uint32_t x, uint32_t topbits) {
    return (x & 0x07FF07FFu) | ((x & 0x08000800u) << 4) | topbits;
}

// The 8 weights of a normal group from its 96-bit slot a0 | a1 << 32 | a2 << 64,
// in which field k sits at bit 12 k. Word k of the result holds weights 2k, 2k+1.
__device__ __forceinline__ uint4 unpack_slot(uint32_t a0, uint32_t a1, uint32_t a2, uint32_t topbits) {
    uint4 r;
    r.x = expand_pair((a0 & 0xFFFu) | ((a0 << 4) & 0x0FFF0000u), topbits);
    r.y = expand_pair((__funnelshift_r(a0, a1, 24) & 0xFFFu) | ((a1 << 12) & 0x0FFF0000u), topbits);
    r.z = expand_pair(((a1 >> 16) & 0xFFFu) | ((__funnelshift_r(a1, a2, 28) << 16) & 0x0FFF0000u), topbits);
    r.w = expand_pair(((a2 >> 8) & 0xFFFu) | ((a2 >> 4) & 0x0FFF0000u), topbits);
    return r;
}

// Two weights' 12-bit fields, each in its 16-bit half, from a pair of BF16
// weights: sign to bit 11, low exponent bits and fraction kept.
__device__ __forceinline__ uint32_t field_pair(uint32_t w) { return ((w >> 4) & 0x08000800u) | (w & 0x07FF07FFu); }

// Does a pair of weights have top exponent bits other than topcmp's halves?
__device__ __forceinline__ bool pair_escapes(uint32_t w, uint32_t topcmp) { return ((w >> 11) & 0x000F000Fu) != topcmp; }

// Group g's 8 weights; weights at or past n read as the padding value.
template <bool kVec>
__device__ __forceinline__ uint4 load_group(const uint16_t* __restrict__ in, uint64_t n, uint64_t g, uint16_t pad) {
    if (kVec && 8 * g + 8 <= n) return __ldg(reinterpret_cast<const uint4*>(in) + g);
    uint32_t h[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) h[k] = 8 * g + k < n ? __ldg(in + 8 * g + k) : pad;
    return make_uint4(h[0] | h[1] << 16, h[2] | h[3] << 16, h[4] | h[5] << 16, h[6] | h[7] << 16);
}

template <bool kVec>
__device__ __forceinline__ void store_group(uint16_t* __restrict__ out, uint64_t n, uint64_t g, uint4 v) {
    if (8 * g + 8 <= n) {
        if (kVec) {
            reinterpret_cast<uint4*>(out)[g] = v;
            return;
        }
    }
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int k = 0; k < 8; ++k)
        if (8 * g + k < n) out[8 * g + k] = static_cast<uint16_t>(w[k >> 1] >> (16 * (k & 1)));
}

// ---------------------------------------------------------------- decode

template <bool kVec>
__device__ __forceinline__ void decode_tile(const Nf12Dev& d, uint64_t tile, uint32_t* err) {
    const int lane = threadIdx.x & 31;
    const uint64_t G = (d.n + 7) >> 3;
    const uint64_t g0 = tile * kTile + static_cast<uint64_t>(threadIdx.x >> 5) * (32 * kNfPerLane);
    if (g0 >= G) return;
    const uint32_t topbits = (d.top << 11) * 0x00010001u;
    const uint64_t w0 = g0 >> 5;
    uint32_t escw = 0;  // lane j < 8 holds the escape word of groups g0 + 32 j ..
    if (lane < kNfPerLane && w0 + lane < ((G + 31) >> 5)) escw = __ldg(d.bitmap + w0 + lane);
    uint32_t a[kNfPerLane][3];
#pragma unroll
    for (int j = 0; j < kNfPerLane; ++j) {
        const uint64_t g = g0 + 32 * j + lane;
        if (g < G) {
            const uint32_t* s = d.slots + 3 * g;
            a[j][0] = __ldg(s);
            a[j][1] = __ldg(s + 1);
            a[j][2] = __ldg(s + 2);
        } else {
            a[j][0] = a[j][1] = a[j][2] = 0;
        }
    }
#pragma unroll
    for (int j = 0; j < kNfPerLane; ++j) {
        const uint32_t e = __shfl_sync(0xffffffffu, escw, j);
        const uint64_t g = g0 + 32 * j + lane;
        if (g >= G) continue;
        uint4 v = unpack_slot(a[j][0], a[j][1], a[j][2], topbits);
        if ((e >> lane) & 1u) {
            const uint32_t idx = a[j][0];
            if (idx < d.n_escaped) {
                v = __ldg(d.side + idx);
            } else if (err) {
                atomicOr(err, DF_EFLAG_NF12_SIDE);
            }
        }
        store_group<kVec>(d.out, d.n, g, v);
    }
}

__global__ void __launch_bounds__(kNfThreads) decode_kernel(Nf12Dev d, uint32_t* err) {
    if (d.out_vec)
        decode_tile<true>(d, blockIdx.x, err);
    else
        decode_tile<false>(d, blockIdx.x, err);
}

// starts[t] = first tile of tensor t (starts[count] = total tiles); the block's
// tensor is the last t with starts[t] <= its tile.
__global__ void __launch_bounds__(kNfThreads)
    decode_batch_kernel(const Nf12Dev* __restrict__ descs, const uint64_t* __restrict__ starts, uint32_t count,
                        uint32_t* err) {
    const uint64_t tile = blockIdx.x;
    uint32_t lo = 0, hi = count;  // starts[lo] <= tile < starts[hi]
    while (hi - lo > 1) {
        const uint32_t mid = (lo + hi) >> 1;
        if (__ldg(starts + mid) <= tile)
            lo = mid;
        else
            hi = mid;
    }
    const Nf12Dev d = descs[lo];
    const uint64_t t = tile - __ldg(starts + lo);
    if (d.out_vec)
        decode_tile<true>(d, t, err);
    else
        decode_tile<false>(d, t, err);
}

// ---------------------------------------------------------------- encode

template <bool kVec>
__device__ __forceinline__ void pack_tile(const uint16_t* __restrict__ in, uint64_t n, uint32_t top,
                                          uint32_t* __restrict__ slots, uint32_t* __restrict__ bitmap,
                                          uint64_t* __restrict__ count_out, uint64_t tile) {
    __shared__ uint32_t warp_count[kNfWarps];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const uint64_t G = (n + 7) >> 3;
    const uint64_t g0 = tile * kTile + static_cast<uint64_t>(warp) * (32 * kNfPerLane);
    uint32_t cnt = 0;
    if (g0 < G) {
        const uint16_t pad = static_cast<uint16_t>(top << 11);
        const uint32_t topcmp = top * 0x00010001u;
        uint4 v[kNfPerLane];
#pragma unroll
        for (int j = 0; j < kNfPerLane; ++j) {
            const uint64_t g = g0 + 32 * j + lane;
            v[j] = g < G ? load_group<kVec>(in, n, g, pad) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int j = 0; j < kNfPerLane; ++j) {
            const uint64_t g = g0 + 32 * j + lane;
            const bool esc = g < G && (pair_escapes(v[j].x, topcmp) | pair_escapes(v[j].y, topcmp) |
                                       pair_escapes(v[j].z, topcmp) | pair_escapes(v[j].w, topcmp));
            const uint32_t ballot = __ballot_sync(0xffffffffu, esc);
            if (g0 + 32 * j >= G) continue;  // warp-uniform: no group of this j exists
            if (lane == 0) bitmap[(g0 >> 5) + j] = ballot;
            cnt += __popc(ballot);
            if (g >= G) continue;
            uint32_t a0 = 0, a1 = 0, a2 = 0;  // an escaped slot stays zero until its side index is written
            if (!esc) {
                const uint32_t y0 = field_pair(v[j].x), y1 = field_pair(v[j].y), y2 = field_pair(v[j].z),
                               y3 = field_pair(v[j].w);
                // 24 bits per pair: field 2k at bit 0, field 2k+1 at bit 12
                const uint32_t p0 = (y0 & 0xFFFu) | ((y0 >> 4) & 0xFFF000u);
                const uint32_t p1 = (y1 & 0xFFFu) | ((y1 >> 4) & 0xFFF000u);
                const uint32_t p2 = (y2 & 0xFFFu) | ((y2 >> 4) & 0xFFF000u);
                const uint32_t p3 = (y3 & 0xFFFu) | ((y3 >> 4) & 0xFFF000u);
                a0 = p0 | (p1 << 24);
                a1 = (p1 >> 8) | (p2 << 16);
                a2 = (p2 >> 16) | (p3 << 8);
            }
            uint32_t* s = slots + 3 * g;
            s[0] = a0;
            s[1] = a1;
            s[2] = a2;
        }
    }
    if (lane == 0) warp_count[warp] = cnt;
    __syncthreads();
    if (threadIdx.x == 0) {
        uint32_t t = 0;
#pragma unroll
        for (int w = 0; w < kNfWarps; ++w) t += warp_count[w];
        *count_out = t;
    }
}

__global__ void __launch_bounds__(kNfThreads)
    pack_kernel(const uint16_t* __restrict__ in, uint64_t n, uint32_t top, uint32_t* __restrict__ slots,
                uint32_t* __restrict__ bitmap, uint64_t* __restrict__ counts, int vec) {
    if (vec)
        pack_tile<true>(in, n, top, slots, bitmap, counts + blockIdx.x, blockIdx.x);
    else
        pack_tile<false>(in, n, top, slots, bitmap, counts + blockIdx.x, blockIdx.x);
}

// Exclusive prefix of counts[0 .. tiles) in place; counts[tiles] and
// *escaped get the total. One block: thread i scans a contiguous run.
__global__ void __launch_bounds__(kScanThreads) scan_kernel(uint64_t* counts, uint64_t tiles, uint64_t* escaped) {
    __shared__ uint64_t warp_sum[kScanThreads / 32];
    const uint64_t per = (tiles + kScanThreads - 1) / kScanThreads;
    const uint64_t b = threadIdx.x * per, e = b + per < tiles ? b + per : tiles;
    uint64_t s = 0;
    for (uint64_t i = b; i < e; ++i) s += counts[i];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint64_t incl = s;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint64_t y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) warp_sum[warp] = incl;
    __syncthreads();
    uint64_t before = 0;
    for (int w = 0; w < warp; ++w) before += warp_sum[w];
    uint64_t run = before + incl - s;
    for (uint64_t i = b; i < e; ++i) {
        const uint64_t c = counts[i];
        counts[i] = run;
        run += c;
    }
    if (threadIdx.x == kScanThreads - 1) {
        counts[tiles] = run;
        *escaped = run;
    }
}

// One block of 64 threads per tile; thread i owns the tile's bitmap word i
// (32 groups) and writes the side entries of its escaped groups in order,
// from side index `base` (the escapes of the tensor's tiles before this one).
template <bool kVec>
__device__ __forceinline__ void escape_tile(const uint16_t* __restrict__ in, uint64_t n, uint32_t top,
                                            uint32_t* __restrict__ slots, const uint32_t* __restrict__ bitmap,
                                            uint64_t tile, uint64_t base, uint4* __restrict__ side, uint64_t cap,
                                            uint32_t* err) {
    __shared__ uint32_t warp_total[kWordsPerTile / 32];
    const uint64_t G = (n + 7) >> 3;
    const uint64_t wi = tile * kWordsPerTile + threadIdx.x;
    uint32_t word = wi < ((G + 31) >> 5) ? bitmap[wi] : 0;
    const uint32_t c = __popc(word);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) warp_total[warp] = incl;
    __syncthreads();
    uint64_t idx = base + incl - c + (warp ? warp_total[0] : 0);
    const uint16_t pad = static_cast<uint16_t>(top << 11);
    while (word) {
        const int bit = __ffs(word) - 1;
        word &= word - 1;
        const uint64_t g = wi * 32 + bit;
        if (idx < cap) {
            side[idx] = load_group<kVec>(in, n, g, pad);
            slots[3 * g] = static_cast<uint32_t>(idx);
        } else if (err) {
            atomicOr(err, DF_EFLAG_NF12_SIDE);
        }
        ++idx;
    }
}

static_assert(kWordsPerTile == 64, "escape_tile combines two warps");

__global__ void __launch_bounds__(kWordsPerTile)
    escape_kernel(const uint16_t* __restrict__ in, uint64_t n, uint32_t top, uint32_t* __restrict__ slots,
                  const uint32_t* __restrict__ bitmap, const uint64_t* __restrict__ prefix, uint4* __restrict__ side,
                  uint64_t cap, uint32_t* err, int vec) {
    const uint64_t tile = blockIdx.x, base = prefix[tile];
    if (prefix[tile + 1] == base) return;  // no escapes in this tile
    if (vec)
        escape_tile<true>(in, n, top, slots, bitmap, tile, base, side, cap, err);
    else
        escape_tile<false>(in, n, top, slots, bitmap, tile, base, side, cap, err);
}

// ---------------------------------------------------------------- grouped encode

struct Nf12EncDev {
    const uint16_t* in;
    uint32_t* slots;
    uint32_t* bitmap;
    uint4* side;
    uint64_t n;
    uint64_t cap;
    uint32_t top;
    uint32_t in_vec;  // in is 16-byte aligned
    uint64_t pad;
};
static_assert(sizeof(Nf12EncDev) == 64, "descriptors are copied in 64-byte units");

// The tensor of global tile `tile` (starts[t] <= tile < starts[t + 1]).
__device__ __forceinline__ uint32_t tensor_of(const uint64_t* __restrict__ starts, uint32_t count, uint64_t tile) {
    uint32_t lo = 0, hi = count;
    while (hi - lo > 1) {
        const uint32_t mid = (lo + hi) >> 1;
        if (__ldg(starts + mid) <= tile)
            lo = mid;
        else
            hi = mid;
    }
    return lo;
}

__global__ void __launch_bounds__(kNfThreads)
    pack_batch_kernel(const Nf12EncDev* __restrict__ descs, const uint64_t* __restrict__ starts, uint32_t count,
                      uint64_t* __restrict__ counts) {
    const uint64_t tile = blockIdx.x;
    const uint32_t ti = tensor_of(starts, count, tile);
    const Nf12EncDev d = descs[ti];
    const uint64_t t = tile - __ldg(starts + ti);
    if (d.in_vec)
        pack_tile<true>(d.in, d.n, d.top, d.slots, d.bitmap, counts + tile, t);
    else
        pack_tile<false>(d.in, d.n, d.top, d.slots, d.bitmap, counts + tile, t);
}

// Per tensor (one CUDA block each): the exclusive prefix of its tiles' escape
// counts in place, and its total.
constexpr int kBatchScanThreads = 256;
__global__ void __launch_bounds__(kBatchScanThreads)
    scan_batch_kernel(const uint64_t* __restrict__ starts, uint64_t* __restrict__ counts, uint64_t* __restrict__ totals) {
    __shared__ uint64_t warp_sum[kBatchScanThreads / 32];
    const uint32_t ti = blockIdx.x;
    const uint64_t t0 = starts[ti], tiles = starts[ti + 1] - t0;
    uint64_t* c = counts + t0;
    const uint64_t per = (tiles + kBatchScanThreads - 1) / kBatchScanThreads;
    const uint64_t b = threadIdx.x * per, e = b + per < tiles ? b + per : tiles;
    uint64_t s = 0;
    for (uint64_t i = b; i < e; ++i) s += c[i];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint64_t incl = s;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint64_t y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) warp_sum[warp] = incl;
    __syncthreads();
    uint64_t run = incl - s;
    for (int w = 0; w < warp; ++w) run += warp_sum[w];
    for (uint64_t i = b; i < e; ++i) {
        const uint64_t x = c[i];
        c[i] = run;
        run += x;
    }
    if (threadIdx.x == kBatchScanThreads - 1) totals[ti] = run;
}

__global__ void __launch_bounds__(kWordsPerTile)
    escape_batch_kernel(const Nf12EncDev* __restrict__ descs, const uint64_t* __restrict__ starts, uint32_t count,
                        const uint64_t* __restrict__ prefix, const uint64_t* __restrict__ totals, uint32_t* err) {
    const uint64_t tile = blockIdx.x;
    const uint32_t ti = tensor_of(starts, count, tile);
    const uint64_t base = prefix[tile];
    const uint64_t next = tile + 1 < __ldg(starts + ti + 1) ? prefix[tile + 1] : totals[ti];
    if (next == base) return;  // no escapes in this tile
    const Nf12EncDev d = descs[ti];
    const uint64_t t = tile - __ldg(starts + ti);
    if (d.in_vec)
        escape_tile<true>(d.in, d.n, d.top, d.slots, d.bitmap, t, base, d.side, d.cap, err);
    else
        escape_tile<false>(d.in, d.n, d.top, d.slots, d.bitmap, t, base, d.side, d.cap, err);
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

df_status launched() {
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? DF_OK : cuda_fail(e);
}

df_status to_dev(const df_nf12_tensor& t, Nf12Dev* d) {
    if (t.top > 15 || t.reserved) return DF_ERR_INVALID_ARG;
    if (t.n > DF_MAX_WEIGHTS) return DF_ERR_UNSUPPORTED;
    if (t.n && (!t.slots || !t.bitmap || !t.out || (t.n_escaped && !t.side))) return DF_ERR_INVALID_ARG;
    if (!aligned(t.slots, 4) || !aligned(t.bitmap, 4) || !aligned(t.side, 16) || !aligned(t.out, 2))
        return DF_ERR_INVALID_ARG;
    const uint64_t G = (t.n + 7) / 8;
    if (G > kMaxGroups || t.n_escaped > G) return DF_ERR_INVALID_ARG;
    d->slots = static_cast<const uint32_t*>(t.slots);
    d->bitmap = static_cast<const uint32_t*>(t.bitmap);
    d->side = static_cast<const uint4*>(t.side);
    d->out = static_cast<uint16_t*>(t.out);
    d->n = t.n;
    d->n_escaped = t.n_escaped;
    d->top = t.top;
    d->out_vec = aligned(t.out, 16);
    d->pad = 0;
    return DF_OK;
}

uint64_t tiles_of(uint64_t n) { return ((n + 7) / 8 + kTile - 1) / kTile; }

}  // namespace
}  // namespace df

using namespace df;

extern "C" {

df_status df_nf12_sizes_for(uint64_t n, df_nf12_sizes* out) {
    if (!out) return DF_ERR_INVALID_ARG;
    if (n > DF_MAX_WEIGHTS) return DF_ERR_UNSUPPORTED;
    const uint64_t G = (n + 7) / 8;
    out->groups = G;
    out->slots_bytes = 12 * G;
    out->bitmap_bytes = 4 * ((G + 31) / 32);
    out->tiles = tiles_of(n);
    out->encode_ws_bytes = 8 * (out->tiles + 1);
    return DF_OK;
}

df_status df_nf12_encode_groups(const uint16_t* d_in, uint64_t n, uint32_t top, void* d_slots, void* d_bitmap,
                                void* d_ws, size_t ws_bytes, uint64_t* d_escaped, void* stream) {
    if (top > 15 || !d_ws || !d_escaped || (n && (!d_in || !d_slots || !d_bitmap))) return DF_ERR_INVALID_ARG;
    if (!aligned(d_in, 2) || !aligned(d_slots, 4) || !aligned(d_bitmap, 4) || !aligned(d_ws, 8) ||
        !aligned(d_escaped, 8))
        return DF_ERR_INVALID_ARG;
    df_nf12_sizes z;
    df_status st = df_nf12_sizes_for(n, &z);
    if (st != DF_OK) return st;
    if (z.groups > kMaxGroups) return DF_ERR_UNSUPPORTED;
    if (ws_bytes < z.encode_ws_bytes) return DF_ERR_WORKSPACE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint64_t* counts = static_cast<uint64_t*>(d_ws);
    if (z.tiles) {
        pack_kernel<<<static_cast<unsigned>(z.tiles), kNfThreads, 0, s>>>(
            d_in, n, top, static_cast<uint32_t*>(d_slots), static_cast<uint32_t*>(d_bitmap), counts,
            aligned(d_in, 16) ? 1 : 0);
        if ((st = launched()) != DF_OK) return st;
    }
    scan_kernel<<<1, kScanThreads, 0, s>>>(counts, z.tiles, d_escaped);
    return launched();
}

df_status df_nf12_encode_escapes(const uint16_t* d_in, uint64_t n, uint32_t top, void* d_slots,
                                 const void* d_bitmap, const void* d_ws, size_t ws_bytes, void* d_side,
                                 uint64_t side_capacity, uint32_t* d_err, void* stream) {
    if (top > 15 || !d_ws || (n && (!d_in || !d_slots || !d_bitmap)) || (side_capacity && !d_side))
        return DF_ERR_INVALID_ARG;
    if (!aligned(d_in, 2) || !aligned(d_slots, 4) || !aligned(d_bitmap, 4) || !aligned(d_ws, 8) ||
        !aligned(d_side, 16))
        return DF_ERR_INVALID_ARG;
    df_nf12_sizes z;
    df_status st = df_nf12_sizes_for(n, &z);
    if (st != DF_OK) return st;
    if (z.groups > kMaxGroups) return DF_ERR_UNSUPPORTED;
    if (ws_bytes < z.encode_ws_bytes) return DF_ERR_WORKSPACE;
    if (!z.tiles) return DF_OK;
    escape_kernel<<<static_cast<unsigned>(z.tiles), kWordsPerTile, 0, static_cast<cudaStream_t>(stream)>>>(
        d_in, n, top, static_cast<uint32_t*>(d_slots), static_cast<const uint32_t*>(d_bitmap),
        static_cast<const uint64_t*>(d_ws), static_cast<uint4*>(d_side), side_capacity, d_err,
        aligned(d_in, 16) ? 1 : 0);
    return launched();
}

df_status df_nf12_decode(const df_nf12_tensor* t, uint32_t* d_err, void* stream) {
    if (!t) return DF_ERR_INVALID_ARG;
    Nf12Dev d;
    const df_status st = to_dev(*t, &d);
    if (st != DF_OK) return st;
    const uint64_t tiles = tiles_of(t->n);
    if (!tiles) return DF_OK;
    if (tiles > 0x7FFFFFFFull) return DF_ERR_UNSUPPORTED;
    decode_kernel<<<static_cast<unsigned>(tiles), kNfThreads, 0, static_cast<cudaStream_t>(stream)>>>(d, d_err);
    return launched();
}

size_t df_nf12_decode_batch_workspace(uint32_t count) {
    return static_cast<size_t>(count) * sizeof(Nf12Dev) + 8 * (static_cast<size_t>(count) + 1);
}

df_status df_nf12_decode_batch_prepare(const df_nf12_tensor* h_tensors, uint32_t count, void* d_ws,
                                       size_t ws_bytes, df_nf12_plan* plan, void* stream) {
    if (!plan || (count && (!h_tensors || !d_ws)) || !aligned(d_ws, 16)) return DF_ERR_INVALID_ARG;
    if (ws_bytes < df_nf12_decode_batch_workspace(count)) return DF_ERR_WORKSPACE;
    std::vector<Nf12Dev> dev(count);
    std::vector<uint64_t> start(count + 1, 0);
    for (uint32_t i = 0; i < count; ++i) {
        const df_status st = to_dev(h_tensors[i], &dev[i]);
        if (st != DF_OK) return st;
        start[i + 1] = start[i] + tiles_of(h_tensors[i].n);
    }
    if (start[count] > 0x7FFFFFFFull) return DF_ERR_UNSUPPORTED;
    plan->d_ws = d_ws;
    plan->count = count;
    plan->reserved = 0;
    plan->total_tiles = start[count];
    if (!count) return DF_OK;
    // copies from pageable host memory return once the source has been
    // staged, so the host vectors may die on return
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemcpyAsync(d_ws, dev.data(), dev.size() * sizeof(Nf12Dev), cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(static_cast<uint8_t*>(d_ws) + dev.size() * sizeof(Nf12Dev), start.data(),
                            start.size() * 8, cudaMemcpyHostToDevice, s);
    return e == cudaSuccess ? DF_OK : cuda_fail(e);
}

df_status df_nf12_decode_batch_run(const df_nf12_plan* plan, uint32_t* d_err, void* stream) {
    if (!plan || (plan->count && !plan->d_ws)) return DF_ERR_INVALID_ARG;
    if (!plan->total_tiles) return DF_OK;
    if (plan->total_tiles > 0x7FFFFFFFull) return DF_ERR_UNSUPPORTED;
    const Nf12Dev* descs = static_cast<const Nf12Dev*>(plan->d_ws);
    const uint64_t* starts = reinterpret_cast<const uint64_t*>(descs + plan->count);
    decode_batch_kernel<<<static_cast<unsigned>(plan->total_tiles), kNfThreads, 0,
                          static_cast<cudaStream_t>(stream)>>>(descs, starts, plan->count, d_err);
    return launched();
}

}  // extern "C"

// ---------------------------------------------------------------- grouped encode, host side

namespace {

struct EncLayout {
    size_t descs, starts, counts, totals, bytes;
};

EncLayout enc_layout(uint32_t count, uint64_t total_tiles) {
    EncLayout l;
    l.descs = 0;
    l.starts = static_cast<size_t>(count) * sizeof(df::Nf12EncDev);
    l.counts = l.starts + 8 * (static_cast<size_t>(count) + 1);
    l.totals = l.counts + 8 * static_cast<size_t>(total_tiles);
    l.bytes = l.totals + 8 * static_cast<size_t>(count);
    return l;
}

uint64_t enc_tiles(const df_nf12_encode_tensor* h, uint32_t count) {
    uint64_t t = 0;
    for (uint32_t i = 0; i < count; ++i) t += df::tiles_of(h[i].n);
    return t;
}

}  // namespace

extern "C" {

size_t df_nf12_encode_batch_workspace(const df_nf12_encode_tensor* h_tensors, uint32_t count) {
    if (count && !h_tensors) return 0;
    return enc_layout(count, enc_tiles(h_tensors, count)).bytes;
}

df_status df_nf12_encode_batch_prepare(const df_nf12_encode_tensor* h_tensors, uint32_t count, void* d_ws,
                                       size_t ws_bytes, df_nf12_plan* plan, void* stream) {
    if (!plan || (count && (!h_tensors || !d_ws)) || !df::aligned(d_ws, 16)) return DF_ERR_INVALID_ARG;
    std::vector<df::Nf12EncDev> dev(count);
    std::vector<uint64_t> start(static_cast<size_t>(count) + 1, 0);
    for (uint32_t i = 0; i < count; ++i) {
        const df_nf12_encode_tensor& t = h_tensors[i];
        if (t.top > 15 || t.reserved || t.reserved2) return DF_ERR_INVALID_ARG;
        if (t.n > DF_MAX_WEIGHTS) return DF_ERR_UNSUPPORTED;
        if (t.n && (!t.in || !t.slots || !t.bitmap)) return DF_ERR_INVALID_ARG;
        if (t.side_capacity && !t.side) return DF_ERR_INVALID_ARG;
        if (!df::aligned(t.in, 2) || !df::aligned(t.slots, 4) || !df::aligned(t.bitmap, 4) ||
            !df::aligned(t.side, 16))
            return DF_ERR_INVALID_ARG;
        if ((t.n + 7) / 8 > df::kMaxGroups) return DF_ERR_UNSUPPORTED;
        df::Nf12EncDev& d = dev[i];
        d.in = t.in;
        d.slots = static_cast<uint32_t*>(t.slots);
        d.bitmap = static_cast<uint32_t*>(t.bitmap);
        d.side = static_cast<uint4*>(t.side);
        d.n = t.n;
        d.cap = t.side_capacity;
        d.top = t.top;
        d.in_vec = df::aligned(t.in, 16) ? 1u : 0u;
        d.pad = 0;
        start[i + 1] = start[i] + df::tiles_of(t.n);
    }
    const uint64_t total = start[count];
    if (total > 0x7FFFFFFFull) return DF_ERR_UNSUPPORTED;
    const EncLayout l = enc_layout(count, total);
    if (ws_bytes < l.bytes) return DF_ERR_WORKSPACE;
    plan->d_ws = d_ws;
    plan->count = count;
    plan->reserved = 0;
    plan->total_tiles = total;
    if (!count) return DF_OK;
    // copies from pageable host memory return once the source has been
    // staged, so the host vectors may die on return
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint8_t* ws = static_cast<uint8_t*>(d_ws);
    cudaError_t e = cudaMemcpyAsync(ws + l.descs, dev.data(), dev.size() * sizeof(df::Nf12EncDev),
                                    cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(ws + l.starts, start.data(), start.size() * 8, cudaMemcpyHostToDevice, s);
    return e == cudaSuccess ? DF_OK : cuda_fail(e);
}

df_status df_nf12_encode_batch_groups(const df_nf12_plan* plan, uint64_t* d_escaped, void* stream) {
    if (!plan || !d_escaped || (plan->count && !plan->d_ws) || !df::aligned(d_escaped, 8)) return DF_ERR_INVALID_ARG;
    if (!plan->count) return DF_OK;
    if (plan->total_tiles > 0x7FFFFFFFull) return DF_ERR_UNSUPPORTED;
    const EncLayout l = enc_layout(plan->count, plan->total_tiles);
    uint8_t* ws = static_cast<uint8_t*>(plan->d_ws);
    const df::Nf12EncDev* descs = reinterpret_cast<const df::Nf12EncDev*>(ws + l.descs);
    const uint64_t* starts = reinterpret_cast<const uint64_t*>(ws + l.starts);
    uint64_t* counts = reinterpret_cast<uint64_t*>(ws + l.counts);
    uint64_t* totals = reinterpret_cast<uint64_t*>(ws + l.totals);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    df_status st;
    if (plan->total_tiles) {
        df::pack_batch_kernel<<<static_cast<unsigned>(plan->total_tiles), df::kNfThreads, 0, s>>>(descs, starts,
                                                                                                 plan->count, counts);
        if ((st = df::launched()) != DF_OK) return st;
    }
    df::scan_batch_kernel<<<plan->count, df::kBatchScanThreads, 0, s>>>(starts, counts, totals);
    if ((st = df::launched()) != DF_OK) return st;
    const cudaError_t e = cudaMemcpyAsync(d_escaped, totals, 8 * static_cast<size_t>(plan->count),
                                          cudaMemcpyDeviceToDevice, s);
    return e == cudaSuccess ? DF_OK : cuda_fail(e);
}

df_status df_nf12_encode_batch_escapes(const df_nf12_plan* plan, uint32_t* d_err, void* stream) {
    if (!plan || (plan->count && !plan->d_ws)) return DF_ERR_INVALID_ARG;
    if (!plan->count || !plan->total_tiles) return DF_OK;
    if (plan->total_tiles > 0x7FFFFFFFull) return DF_ERR_UNSUPPORTED;
    const EncLayout l = enc_layout(plan->count, plan->total_tiles);
    const uint8_t* ws = static_cast<const uint8_t*>(plan->d_ws);
    df::escape_batch_kernel<<<static_cast<unsigned>(plan->total_tiles), df::kWordsPerTile, 0,
                              static_cast<cudaStream_t>(stream)>>>(
        reinterpret_cast<const df::Nf12EncDev*>(ws + l.descs), reinterpret_cast<const uint64_t*>(ws + l.starts),
        plan->count, reinterpret_cast<const uint64_t*>(ws + l.counts), reinterpret_cast<const uint64_t*>(ws + l.totals),
        d_err);
    return df::launched();
}

}  // extern "C"
