// Compact block index (df11.h, "compact block index"): build it from the
// uint64 block offsets, and expand it back.
//
// df11pack (GitHub page), "What is checked, and what is not": the opt-in
// --index idx8 is an 8-bit block index that makes the file smaller. The
// layout here is this library's: superblocks of 64 format blocks, each with a
// 64-bit anchor and a 32-bit base, one delta byte per block, and full 32-bit
// counts for the rare superblock whose counts spread over more than 255.
//
// Build: one 64-thread CUDA block per superblock writes its anchor, base (or
// a wide mark) and deltas; then one CUDA block numbers the wide superblocks
// in order and writes their overflow counts. Expand: one 64-thread CUDA block
// per superblock scans its counts.
#include <cuda_runtime.h>
#include <stdint.h>

#include "df_internal.h"

namespace df {
namespace {

constexpr uint32_t kSuper = 64;
constexpr uint32_t kWide = 0x80000000u;
constexpr int kNumberThreads = 1024;

struct Index8View {
    uint64_t* anchor;
    uint32_t* base;
    uint8_t* delta;
    uint32_t* overflow;
};

__host__ __device__ inline Index8View view_of(void* p, uint64_t S) {
    uint8_t* b = static_cast<uint8_t*>(p);
    return {reinterpret_cast<uint64_t*>(b), reinterpret_cast<uint32_t*>(b + 8 * S), b + 12 * S,
            reinterpret_cast<uint32_t*>(b + 76 * S)};
}

// Counts of a superblock's blocks (0 past the last block) and their range.
__global__ void __launch_bounds__(kSuper)
    superblock_kernel(const uint64_t* __restrict__ offs, uint64_t n_blocks, Index8View ix, uint32_t* err) {
    __shared__ uint32_t s_lo[2], s_hi[2];
    const uint64_t s = blockIdx.x;
    const uint64_t b = s * kSuper + threadIdx.x;
    const bool real = b < n_blocks;
    uint64_t c64 = real ? offs[b + 1] - offs[b] : 0;
    if (real && c64 >= kWide) {  // offsets going backwards wrap to huge counts too
        if (err) atomicOr(err, DF_EFLAG_INDEX8);
        c64 = 0;
    }
    const uint32_t c = static_cast<uint32_t>(c64);
    const uint32_t lo_w = __reduce_min_sync(0xffffffffu, real ? c : 0xFFFFFFFFu);
    const uint32_t hi_w = __reduce_max_sync(0xffffffffu, real ? c : 0u);
    const int warp = threadIdx.x >> 5;
    if ((threadIdx.x & 31) == 0) {
        s_lo[warp] = lo_w;
        s_hi[warp] = hi_w;
    }
    __syncthreads();
    const uint32_t lo = min(s_lo[0], s_lo[1]), hi = max(s_hi[0], s_hi[1]);
    const bool wide = hi - lo > 255u;  // block 0 of s is always real, so lo <= hi
    ix.delta[b] = (!wide && real) ? static_cast<uint8_t>(c - lo) : 0;
    if (threadIdx.x == 0) {
        ix.anchor[s] = offs[s * kSuper];
        ix.base[s] = wide ? kWide : lo;
    }
}

// Numbers the wide superblocks in order (thread i: a contiguous run of
// superblocks) and writes their overflow counts while there is room.
__global__ void __launch_bounds__(kNumberThreads)
    number_wide_kernel(const uint64_t* __restrict__ offs, uint64_t n_blocks, uint64_t S, Index8View ix,
                       uint64_t room, uint64_t* n_wide, uint32_t* err) {
    __shared__ uint32_t warp_sum[kNumberThreads / 32];
    const uint64_t per = (S + kNumberThreads - 1) / kNumberThreads;
    const uint64_t s0 = threadIdx.x * per, s1 = s0 + per < S ? s0 + per : S;
    uint32_t mine = 0;
    for (uint64_t s = s0; s < s1; ++s) mine += (ix.base[s] & kWide) ? 1u : 0u;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t incl = mine;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) warp_sum[warp] = incl;
    __syncthreads();
    uint64_t k = incl - mine;
    for (int w = 0; w < warp; ++w) k += warp_sum[w];
    for (uint64_t s = s0; s < s1; ++s) {
        if (!(ix.base[s] & kWide)) continue;
        ix.base[s] = kWide | static_cast<uint32_t>(k);
        if (k < room) {
            for (uint32_t j = 0; j < kSuper; ++j) {
                const uint64_t b = s * kSuper + j;
                const uint64_t c = b < n_blocks ? offs[b + 1] - offs[b] : 0;
                ix.overflow[k * kSuper + j] = c < kWide ? static_cast<uint32_t>(c) : 0u;
            }
        } else if (err) {
            atomicOr(err, DF_EFLAG_INDEX8);
        }
        ++k;
    }
    if (threadIdx.x == kNumberThreads - 1) *n_wide = k;
}

__global__ void __launch_bounds__(kSuper)
    expand_kernel(Index8View ix, uint64_t n_blocks, uint64_t n_wide, uint64_t* __restrict__ offs, uint32_t* err) {
    __shared__ uint32_t s_sum;
    const uint64_t s = blockIdx.x;
    const uint64_t b = s * kSuper + threadIdx.x;
    const uint32_t w = ix.base[s];
    uint32_t c = 0;
    if (b < n_blocks) {
        if (!(w & kWide)) {
            c = w + ix.delta[b];
        } else if ((w & ~kWide) < n_wide) {
            c = ix.overflow[static_cast<uint64_t>(w & ~kWide) * kSuper + threadIdx.x];
        } else if (err) {
            atomicOr(err, DF_EFLAG_INDEX8);
        }
    }
    const int lane = threadIdx.x & 31;
    uint32_t incl = c;  // counts of a superblock sum below 2^32: each is below 2^23 in a valid index
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    if (threadIdx.x == 31) s_sum = incl;
    __syncthreads();
    const uint64_t before = (threadIdx.x >= 32 ? static_cast<uint64_t>(s_sum) : 0) + incl - c;
    const uint64_t a = ix.anchor[s];
    if (b < n_blocks) offs[b] = a + before;
    if (b + 1 == n_blocks) offs[n_blocks] = a + before + c;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

df_status launched() {
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? DF_OK : cuda_fail(e);
}

}  // namespace
}  // namespace df

using namespace df;

extern "C" {

uint64_t df_index8_bytes(uint64_t n_blocks, uint64_t n_wide) {
    return 76 * ((n_blocks + kSuper - 1) / kSuper) + 4ull * kSuper * n_wide;
}

df_status df_index8_build(const uint64_t* d_offsets, uint64_t n_blocks, void* d_index8, size_t index8_bytes,
                          uint64_t* d_n_wide, uint32_t* d_err, void* stream) {
    if (!d_offsets || !d_n_wide || (n_blocks && !d_index8) || !aligned(d_index8, 8) || !aligned(d_offsets, 8) ||
        !aligned(d_n_wide, 8))
        return DF_ERR_INVALID_ARG;
    if (n_blocks >= (1ull << 32)) return DF_ERR_UNSUPPORTED;
    const uint64_t S = (n_blocks + kSuper - 1) / kSuper;
    const uint64_t fixed = df_index8_bytes(n_blocks, 0);
    if (index8_bytes < fixed) return DF_ERR_INVALID_ARG;
    const uint64_t room = (index8_bytes - fixed) / (4ull * kSuper);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const Index8View ix = view_of(d_index8, S);
    if (S) {
        superblock_kernel<<<static_cast<unsigned>(S), kSuper, 0, s>>>(d_offsets, n_blocks, ix, d_err);
        const df_status st = launched();
        if (st != DF_OK) return st;
    }
    number_wide_kernel<<<1, kNumberThreads, 0, s>>>(d_offsets, n_blocks, S, ix, room, d_n_wide, d_err);
    return launched();
}

df_status df_index8_expand(const void* d_index8, uint64_t n_blocks, uint64_t n_wide, uint64_t* d_offsets,
                           uint32_t* d_err, void* stream) {
    if (!d_offsets || (n_blocks && !d_index8) || !aligned(d_index8, 8) || !aligned(d_offsets, 8))
        return DF_ERR_INVALID_ARG;
    if (n_blocks >= (1ull << 32)) return DF_ERR_UNSUPPORTED;
    const uint64_t S = (n_blocks + kSuper - 1) / kSuper;
    if (n_wide > S) return DF_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (!S) {  // no blocks: O[0] = 0
        const cudaError_t e = cudaMemsetAsync(d_offsets, 0, 8, s);
        return e == cudaSuccess ? DF_OK : cuda_fail(e);
    }
    expand_kernel<<<static_cast<unsigned>(S), kSuper, 0, s>>>(view_of(const_cast<void*>(d_index8), S), n_blocks,
                                                              n_wide, d_offsets, d_err);
    return launched();
}

}  // extern "C"
