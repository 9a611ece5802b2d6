// Encode path: exponent histogram, per-tile code-length sums, a scan of the
// tile sums into bit offsets, and a warp-level bit packer.
//
// What is coded (mlx-dfloat, PyPI page, intro bit diagram): the 8 exponent
// bits of each BF16 weight become a variable-length code; the sign and the 7
// fraction bits become one raw byte. The codebook comes from the exponent
// frequencies (df11pack, GitHub page, intro). The stream layout (MSB-first
// bits, C-byte chunks with 5-bit start gaps, per-block output offsets) is the
// one df11.h defines.
//
// Tiles of 4096 weights, 256 threads x 16 consecutive weights: a block scan of
// the threads' code-length sums gives every code its bit offset; the tile's
// stream words are assembled in shared memory and stored whole, except the two
// edge words a tile shares with its neighbours, which are OR-ed atomically into
// the zeroed stream.
#include <cuda_runtime.h>

#include <cstring>
#include <mutex>

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

// Sum of code lengths of each tile of 4096 weights (16 consecutive weights per
// thread, as the packer reads them).
__global__ void __launch_bounds__(kEncThreads) tile_bits_kernel(const uint16_t* __restrict__ in, uint64_t n,
                                                                int vec, EncTables tab,
                                                                uint64_t* __restrict__ tile_bits, uint32_t* d_err) {
    __shared__ uint8_t s_len[256];
    __shared__ uint32_t s_red[kEncThreads / 32];
    for (uint32_t i = threadIdx.x; i < 256; i += blockDim.x) s_len[i] = tab.lengths[i];
    const uint64_t i0 = static_cast<uint64_t>(blockIdx.x) * kTile + threadIdx.x * kPerThread;
    uint32_t wv[kPerThread / 2];
    const uint32_t cnt = load16(in, n, i0, vec != 0, wv);
    __syncthreads();  // the length table
    uint32_t sum = 0;
    bool missing = false;
#pragma unroll
    for (uint32_t k = 0; k < kPerThread; ++k) {
        if (k < cnt) {
            const uint32_t l = s_len[(wv[k >> 1] >> (16 * (k & 1) + 7)) & 0xFFu];
            missing |= (l == 0);
            sum += l;
        }
    }
    if (__syncthreads_or(missing) && threadIdx.x == 0 && d_err) atomicOr(d_err, DF_EFLAG_ENC_SYMBOL);
#pragma unroll
    for (int d = 16; d > 0; d >>= 1) sum += __shfl_xor_sync(0xFFFFFFFFu, sum, d);
    if ((threadIdx.x & 31) == 0) s_red[threadIdx.x >> 5] = sum;
    __syncthreads();
    if (threadIdx.x == 0) {
        uint32_t t = 0;
        for (uint32_t w = 0; w < kEncThreads / 32; ++w) t += s_red[w];
        tile_bits[blockIdx.x] = t;
    }
}

// Exclusive scan of the tile sums (one block): tile_base[0..tiles].
__global__ void __launch_bounds__(1024) tile_scan_kernel(const uint64_t* __restrict__ tile_bits, uint64_t tiles,
                                                         uint64_t* __restrict__ tile_base, uint64_t want_total,
                                                         uint64_t* __restrict__ offsets, uint64_t n_blocks,
                                                         uint64_t n, uint32_t* d_err) {
    __shared__ uint64_t s_w[32];
    __shared__ uint64_t s_carry;
    if (threadIdx.x == 0) s_carry = 0;
    __syncthreads();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (uint64_t start = 0; start < tiles; start += blockDim.x) {
        const uint64_t i = start + threadIdx.x;
        const uint64_t v = i < tiles ? tile_bits[i] : 0;
        uint64_t x = v;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const uint64_t u = __shfl_up_sync(0xFFFFFFFFu, x, d);
            if (lane >= d) x += u;
        }
        if (lane == 31) s_w[warp] = x;
        __syncthreads();
        if (warp == 0) {
            uint64_t y = lane < static_cast<int>(blockDim.x >> 5) ? s_w[lane] : 0;
#pragma unroll
            for (int d = 1; d < 32; d <<= 1) {
                const uint64_t u = __shfl_up_sync(0xFFFFFFFFu, y, d);
                if (lane >= d) y += u;
            }
            s_w[lane] = y;
        }
        __syncthreads();
        const uint64_t carry = s_carry;
        const uint64_t incl = x + (warp > 0 ? s_w[warp - 1] : 0);
        if (i < tiles) tile_base[i] = carry + incl - v;
        __syncthreads();
        if (threadIdx.x == 0) s_carry = carry + s_w[(blockDim.x >> 5) - 1];
        __syncthreads();
    }
    if (threadIdx.x == 0) {
        tile_base[tiles] = s_carry;
        if (s_carry != want_total && d_err) atomicOr(d_err, DF_EFLAG_ENC_TOTAL);
        offsets[0] = 0;
        offsets[n_blocks] = n;
    }
}

struct PackArgs {
    const uint16_t* in;
    uint64_t n;
    const uint64_t* tile_base;
    uint32_t* stream32;   // the stream as 32-bit words (zeroed)
    uint32_t* gaps32;     // the gap fields as 32-bit words (zeroed)
    uint64_t* offsets;
    uint8_t* sm;
    uint64_t total_bits;
    uint64_t n_chunks;
    uint64_t stream_words;  // words the stream buffer holds: writes beyond are refused
    uint32_t chunk_bits;
    uint32_t threads_per_block;
    uint32_t* err;
    uint32_t in_vec;  // input 16-byte aligned
    uint32_t sm_vec;  // sign|fraction output 16-byte aligned
};

__device__ __forceinline__ void or_gap(uint32_t* gaps32, uint64_t j, uint32_t g) {
    const uint64_t q = 5 * j;
    const uint32_t o = static_cast<uint32_t>(q & 31);
    uint32_t* w = gaps32 + (q >> 5);
    if (o <= 27) {
        atomicOr(w, bswap32(g << (27 - o)));
    } else {
        atomicOr(w, bswap32(g >> (o - 27)));
        atomicOr(w + 1, bswap32(g << (59 - o)));
    }
}

// One tile of 4096 weights per CUDA block, 16 consecutive weights per thread.
// A block scan of the threads' code-length sums gives every code its bit
// offset; the codes are OR-ed into the tile's words in shared memory (shared
// atomics: neighbouring threads may share a word), then the words go out with
// coalesced stores, byte-swapped to MSB-first order. The first and last word
// of a tile may hold bits of the neighbouring tiles: those are OR-ed into the
// zeroed stream atomically. The code that crosses or ends on a chunk boundary
// writes that chunk's gap (and, at a block boundary, the block offset).

__global__ void __launch_bounds__(kEncThreads) pack_kernel(PackArgs a, EncTables tab) {
    __shared__ uint32_t s_code[256];
    __shared__ uint8_t s_len[256];
    __shared__ uint32_t s_warp[kEncThreads / 32];
    __shared__ uint32_t s_words[kTile + 2];  // a tile holds at most 4096 codes of at most 32 bits
    const uint32_t tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    for (uint32_t i = tid; i < 256; i += kEncThreads) {
        s_code[i] = tab.codes[i];
        s_len[i] = tab.lengths[i];
    }
    const uint64_t i0 = static_cast<uint64_t>(blockIdx.x) * kTile + tid * kPerThread;
    uint32_t wv[kPerThread / 2];  // this thread's 16 weights
    const uint32_t cnt = load16(a.in, a.n, i0, a.in_vec != 0, wv);
    const bool full = cnt == kPerThread;
    // sign|fraction bytes
    uint32_t smw[kPerThread / 4];
#pragma unroll
    for (uint32_t k = 0; k < kPerThread / 4; ++k) {
        const uint32_t x = wv[2 * k], y = wv[2 * k + 1];
        // byte j of the word: (w >> 8 & 0x80) | (w & 0x7F) of weight 4k + j
        const uint32_t hi = __byte_perm(x, y, 0x7531) & 0x80808080u;
        const uint32_t lo = __byte_perm(x, y, 0x6420) & 0x7F7F7F7Fu;
        smw[k] = hi | lo;
    }
    if (full && a.sm_vec) {
        *reinterpret_cast<uint4*>(a.sm + i0) = make_uint4(smw[0], smw[1], smw[2], smw[3]);
    } else {
        for (uint32_t k = 0; k < cnt; ++k) a.sm[i0 + k] = static_cast<uint8_t>(smw[k >> 2] >> (8 * (k & 3)));
    }
    __syncthreads();  // the code tables
    uint32_t sum = 0;
#pragma unroll
    for (uint32_t k = 0; k < kPerThread; ++k) {
        const uint32_t e = (wv[k >> 1] >> (16 * (k & 1) + 7)) & 0xFFu;
        sum += k < cnt ? s_len[e] : 0u;
    }
    // block scan of the sums
    uint32_t incl = sum;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const uint32_t u = __shfl_up_sync(0xFFFFFFFFu, incl, d);
        if (lane >= static_cast<uint32_t>(d)) incl += u;
    }
    if (lane == 31) s_warp[warp] = incl;
    const uint64_t tile_bit0 = a.tile_base[blockIdx.x];
    const uint32_t head = static_cast<uint32_t>(tile_bit0 & 31);  // bits of the first word before the tile
    __syncthreads();
    uint32_t wprefix = 0, total = 0;
#pragma unroll
    for (uint32_t w = 0; w < kEncThreads / 32; ++w) {
        const uint32_t t = s_warp[w];
        wprefix += w < warp ? t : 0u;
        total += t;
    }
    const uint32_t nw = (head + total + 31) >> 5;  // words the tile touches
    for (uint32_t k = tid; k < nw; k += kEncThreads) s_words[k] = 0;
    __syncthreads();
    // OR the codes into the tile's words (bit q of the tile -> bit 31 - q % 32 of word q / 32)
    const uint32_t off = wprefix + incl - sum;  // this thread's first bit within the tile
    uint32_t lp = head + off;
    uint64_t gb = tile_bit0 + off;  // ... and in the stream
    // the first chunk boundary after gb, and its chunk index
    uint64_t jn = gb / a.chunk_bits + 1;
    uint64_t nb = jn * a.chunk_bits;
#pragma unroll
    for (uint32_t k = 0; k < kPerThread; ++k) {
        if (k >= cnt) break;
        const uint32_t e = (wv[k >> 1] >> (16 * (k & 1) + 7)) & 0xFFu;
        const uint32_t l = s_len[e];
        if (l == 0) continue;
        const uint32_t v = s_code[e] << (32 - l);  // the code, left-aligned
        const uint32_t sh = lp & 31;
        atomicOr(&s_words[lp >> 5], v >> sh);
        if (sh + l > 32) atomicOr(&s_words[(lp >> 5) + 1], v << (32 - sh));
        lp += l;
        gb += l;
        if (gb >= nb) {  // this code crosses or ends on chunk boundary nb: the next start is gb
            if (jn < a.n_chunks) {
                or_gap(a.gaps32, jn, static_cast<uint32_t>(gb - nb));
                if (jn % a.threads_per_block == 0) a.offsets[jn / a.threads_per_block] = i0 + k + 1;
            }
            ++jn;
            nb += a.chunk_bits;
        }
    }
    __syncthreads();
    // out: whole words inside the tile are stored, the two edge words OR-ed in
    const uint64_t w0 = tile_bit0 >> 5;
    for (uint32_t k = tid; k < nw; k += kEncThreads) {
        const uint64_t W = w0 + k;
        const uint32_t val = bswap32(s_words[k]);
        if (W >= a.stream_words) {
            if (a.err) atomicOr(a.err, DF_EFLAG_ENC_TOTAL);
        } else if (k == 0 || k + 1 == nw) {
            if (val) atomicOr(a.stream32 + W, val);
        } else {
            a.stream32[W] = val;
        }
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
    const uint64_t cbits = 8ull * chunk_bytes;
    const uint64_t n_chunks = total_bits ? (total_bits + cbits - 1) / cbits : 1;
    const uint64_t stream_bytes = n_chunks * chunk_bytes + 16;
    const uint64_t gap_bytes = (((5 * n_chunks + 7) / 8) + 1 + 15) & ~15ull;
    const uint64_t n_blocks = (n_chunks + tpb - 1) / tpb;
    const uint64_t tiles = (n + kTile - 1) / kTile;
    const uint64_t need_ws = 16 * (tiles + 2) + 256;
    if (n && (ws_bytes < need_ws || !d_ws)) return DF_ERR_WORKSPACE;
    if (n && !aligned(d_ws, 16)) return DF_ERR_INVALID_ARG;
    if (tiles > 0x7FFFFFFFull) return DF_ERR_UNSUPPORTED;

    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemsetAsync(d_stream, 0, stream_bytes, s);
    if (e == cudaSuccess) e = cudaMemsetAsync(d_gaps, 0, gap_bytes, s);
    if (e == cudaSuccess) e = cudaMemsetAsync(d_block_offsets, 0, 8 * (n_blocks + 1), s);
    if (e != cudaSuccess) return cuda_fail(e);
    if (n == 0) return DF_OK;  // empty stream, zero gap, offsets {0, 0}

    EncTables tab;
    std::memcpy(tab.codes, code->codes, sizeof(tab.codes));
    std::memcpy(tab.lengths, code->lengths, sizeof(tab.lengths));
    uint64_t* tile_bits = static_cast<uint64_t*>(d_ws);
    uint64_t* tile_base = tile_bits + tiles;
    tile_bits_kernel<<<static_cast<unsigned>(tiles), kEncThreads, 0, s>>>(d_in, n, aligned(d_in, 16) ? 1 : 0, tab,
                                                                         tile_bits, d_err);
    tile_scan_kernel<<<1, 1024, 0, s>>>(tile_bits, tiles, tile_base, total_bits, d_block_offsets, n_blocks, n,
                                         d_err);
    PackArgs a;
    a.in = d_in;
    a.n = n;
    a.tile_base = tile_base;
    a.stream32 = reinterpret_cast<uint32_t*>(d_stream);
    a.gaps32 = reinterpret_cast<uint32_t*>(d_gaps);
    a.offsets = d_block_offsets;
    a.sm = d_sm;
    a.total_bits = total_bits;
    a.n_chunks = n_chunks;
    a.stream_words = stream_bytes / 4;
    a.err = d_err;
    a.chunk_bits = static_cast<uint32_t>(cbits);
    a.threads_per_block = tpb;
    a.in_vec = aligned(d_in, 16) ? 1u : 0u;
    a.sm_vec = aligned(d_sm, 16) ? 1u : 0u;
    pack_kernel<<<static_cast<unsigned>(tiles), kEncThreads, 0, s>>>(a, tab);
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

}  // extern "C"
