// Checks of a container without or with its source: the structure check
// (block offsets and sizes, no decode), an element-wise compare of a decode
// with its source, and a SHA-256 digest of device data.
//
// df11pack (GitHub page), "Use": verify checks a container's structure with
// no source, decodes sampled chunks (or all of them) and compares them with the
// source, and exits 0 on pass, 1 when a check fails, 2 when it could not
// check; "What is checked" (--hashes): a per-tensor SHA-256 in the header lets
// verify catch corruption without the source.
//
// The digest of n bytes is this library's own tree over SHA-256 (FIPS 180-4):
// the data is cut into leaves of 64 KiB (the last one shorter), each leaf is
// hashed on the GPU by its own thread, and the digest is the SHA-256 of the
// concatenated leaf digests, computed on the host. Every step is plain
// SHA-256, so any SHA-256 implementation reproduces it.
#include <cuda_runtime.h>

#include <cstring>
#include <vector>

#include "df_internal.h"

namespace df {
namespace {

// SHA-256 round constants and initial hash value (FIPS 180-4, 4.2.2 and 5.3.3),
// once for the device (constant memory) and once for the host.
#define DF_SHA256_K                                                                                             \
    {0x428a2f98u, 0x71374491u, 0xb5c0fbcfu, 0xe9b5dba5u, 0x3956c25bu, 0x59f111f1u, 0x923f82a4u, 0xab1c5ed5u,     \
     0xd807aa98u, 0x12835b01u, 0x243185beu, 0x550c7dc3u, 0x72be5d74u, 0x80deb1feu, 0x9bdc06a7u, 0xc19bf174u,     \
     0xe49b69c1u, 0xefbe4786u, 0x0fc19dc6u, 0x240ca1ccu, 0x2de92c6fu, 0x4a7484aau, 0x5cb0a9dcu, 0x76f988dau,     \
     0x983e5152u, 0xa831c66du, 0xb00327c8u, 0xbf597fc7u, 0xc6e00bf3u, 0xd5a79147u, 0x06ca6351u, 0x14292967u,     \
     0x27b70a85u, 0x2e1b2138u, 0x4d2c6dfcu, 0x53380d13u, 0x650a7354u, 0x766a0abbu, 0x81c2c92eu, 0x92722c85u,     \
     0xa2bfe8a1u, 0xa81a664bu, 0xc24b8b70u, 0xc76c51a3u, 0xd192e819u, 0xd6990624u, 0xf40e3585u, 0x106aa070u,     \
     0x19a4c116u, 0x1e376c08u, 0x2748774cu, 0x34b0bcb5u, 0x391c0cb3u, 0x4ed8aa4au, 0x5b9cca4fu, 0x682e6ff3u,     \
     0x748f82eeu, 0x78a5636fu, 0x84c87814u, 0x8cc70208u, 0x90befffau, 0xa4506cebu, 0xbef9a3f7u, 0xc67178f2u}
#define DF_SHA256_H0 {0x6a09e667u, 0xbb67ae85u, 0x3c6ef372u, 0xa54ff53au, 0x510e527fu, 0x9b05688cu, 0x1f83d9abu, 0x5be0cd19u}
__constant__ uint32_t kSha256Kd[64] = DF_SHA256_K;
__constant__ uint32_t kSha256H0d[8] = DF_SHA256_H0;
[[maybe_unused]] const uint32_t kSha256Kh[64] = DF_SHA256_K;
[[maybe_unused]] const uint32_t kSha256H0h[8] = DF_SHA256_H0;
#undef DF_SHA256_K
#undef DF_SHA256_H0

__host__ __device__ __forceinline__ uint32_t sha_k(int t) {
#ifdef __CUDA_ARCH__
    return kSha256Kd[t];
#else
    return kSha256Kh[t];
#endif
}

__host__ __device__ __forceinline__ uint32_t sha_h0(int i) {
#ifdef __CUDA_ARCH__
    return kSha256H0d[i];
#else
    return kSha256H0h[i];
#endif
}
constexpr uint64_t kLeafBytes = 64 * 1024;

__host__ __device__ __forceinline__ uint32_t rotr(uint32_t x, uint32_t n) { return (x >> n) | (x << (32 - n)); }

// One 512-bit block (16 big-endian words) into the state (FIPS 180-4, 6.2.2).
// Loop unrolling for the device pass (the host compiler does not know the pragma).
#ifdef __CUDA_ARCH__
#define DF_UNROLL _Pragma("unroll")
#else
#define DF_UNROLL
#endif

__host__ __device__ inline void sha256_block(uint32_t h[8], const uint32_t w_in[16]) {
    uint32_t w[16];
    DF_UNROLL
    for (int i = 0; i < 16; ++i) w[i] = w_in[i];
    uint32_t a = h[0], b = h[1], c = h[2], d = h[3], e = h[4], f = h[5], g = h[6], k = h[7];
    // unrolled on the device: the schedule's indices are constants, so w stays in registers
    DF_UNROLL
    for (int t = 0; t < 64; ++t) {
        uint32_t wt;
        if (t < 16) {
            wt = w[t];
        } else {
            const uint32_t w15 = w[(t - 15) & 15], w2 = w[(t - 2) & 15];
            const uint32_t s0 = rotr(w15, 7) ^ rotr(w15, 18) ^ (w15 >> 3);
            const uint32_t s1 = rotr(w2, 17) ^ rotr(w2, 19) ^ (w2 >> 10);
            wt = w[t & 15] = w[t & 15] + s0 + w[(t - 7) & 15] + s1;
        }
        const uint32_t S1 = rotr(e, 6) ^ rotr(e, 11) ^ rotr(e, 25);
        const uint32_t ch = (e & f) ^ (~e & g);
        const uint32_t t1 = k + S1 + ch + sha_k(t) + wt;
        const uint32_t S0 = rotr(a, 2) ^ rotr(a, 13) ^ rotr(a, 22);
        const uint32_t maj = (a & b) ^ (a & c) ^ (b & c);
        const uint32_t t2 = S0 + maj;
        k = g;
        g = f;
        f = e;
        e = d + t1;
        d = c;
        c = b;
        b = a;
        a = t1 + t2;
    }
    h[0] += a;
    h[1] += b;
    h[2] += c;
    h[3] += d;
    h[4] += e;
    h[5] += f;
    h[6] += g;
    h[7] += k;
}

__host__ __device__ inline uint32_t load_be32(const uint8_t* p) {
    return (static_cast<uint32_t>(p[0]) << 24) | (static_cast<uint32_t>(p[1]) << 16) |
           (static_cast<uint32_t>(p[2]) << 8) | p[3];
}

// SHA-256 of len bytes (the message padding of FIPS 180-4, 5.1.1).
__host__ __device__ inline void sha256(const uint8_t* data, uint64_t len, uint8_t out[32]) {
    uint32_t h[8];
    for (int i = 0; i < 8; ++i) h[i] = sha_h0(i);
    uint32_t w[16];
    uint64_t i = 0;
    for (; i + 64 <= len; i += 64) {
        for (int j = 0; j < 16; ++j) w[j] = load_be32(data + i + 4 * j);
        sha256_block(h, w);
    }
    uint8_t tail[128];
    const uint32_t rem = static_cast<uint32_t>(len - i);
    for (uint32_t j = 0; j < rem; ++j) tail[j] = data[i + j];
    tail[rem] = 0x80;
    const uint32_t tlen = rem + 9 <= 64 ? 64 : 128;
    for (uint32_t j = rem + 1; j < tlen - 8; ++j) tail[j] = 0;
    const uint64_t bits = len * 8;
    for (int j = 0; j < 8; ++j) tail[tlen - 1 - j] = static_cast<uint8_t>(bits >> (8 * j));
    for (uint32_t o = 0; o < tlen; o += 64) {
        for (int j = 0; j < 16; ++j) w[j] = load_be32(tail + o + 4 * j);
        sha256_block(h, w);
    }
    for (int j = 0; j < 8; ++j) {
        out[4 * j] = static_cast<uint8_t>(h[j] >> 24);
        out[4 * j + 1] = static_cast<uint8_t>(h[j] >> 16);
        out[4 * j + 2] = static_cast<uint8_t>(h[j] >> 8);
        out[4 * j + 3] = static_cast<uint8_t>(h[j]);
    }
}

// One thread per 64 KiB leaf.
__global__ void __launch_bounds__(128) sha256_leaves_kernel(const uint8_t* __restrict__ data, uint64_t nbytes,
                                                            uint64_t leaves, uint8_t* __restrict__ digests) {
    const uint64_t i = static_cast<uint64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (i >= leaves) return;
    const uint64_t off = i * kLeafBytes;
    const uint64_t len = nbytes - off < kLeafBytes ? nbytes - off : kLeafBytes;
    const uint8_t* p = data + off;
    if (len != kLeafBytes || (reinterpret_cast<uintptr_t>(p) & 15)) {
        sha256(p, len, digests + 32 * i);  // the last, shorter leaf or unaligned data: byte loads
        return;
    }
    // a whole aligned leaf: 16-byte loads, then the padding block of FIPS 180-4, 5.1.1
    uint32_t h[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) h[j] = sha_h0(j);
    const uint4* q = reinterpret_cast<const uint4*>(p);
    for (uint64_t blk = 0; blk < kLeafBytes / 64; ++blk) {
        uint32_t w[16];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const uint4 v = __ldg(q + 4 * blk + j);
            w[4 * j] = __byte_perm(v.x, 0, 0x0123);
            w[4 * j + 1] = __byte_perm(v.y, 0, 0x0123);
            w[4 * j + 2] = __byte_perm(v.z, 0, 0x0123);
            w[4 * j + 3] = __byte_perm(v.w, 0, 0x0123);
        }
        sha256_block(h, w);
    }
    uint32_t w[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) w[j] = 0;
    w[0] = 0x80000000u;
    const uint64_t bits = static_cast<uint64_t>(kLeafBytes) * 8;
    w[14] = static_cast<uint32_t>(bits >> 32);
    w[15] = static_cast<uint32_t>(bits);
    sha256_block(h, w);
    uint8_t* out = digests + 32 * i;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        out[4 * j] = static_cast<uint8_t>(h[j] >> 24);
        out[4 * j + 1] = static_cast<uint8_t>(h[j] >> 16);
        out[4 * j + 2] = static_cast<uint8_t>(h[j] >> 8);
        out[4 * j + 3] = static_cast<uint8_t>(h[j]);
    }
}

// Structure of one container, no decode: block offsets start at 0, never
// decrease, end at n, and no block holds more codes than its chunks can.
__global__ void __launch_bounds__(256) structure_kernel(const uint64_t* __restrict__ offs, uint64_t n_blocks,
                                                        uint64_t n, uint64_t max_per_block,
                                                        uint32_t* __restrict__ d_flags) {
    const uint64_t stride = static_cast<uint64_t>(gridDim.x) * blockDim.x;
    bool bad = false;
    for (uint64_t b = static_cast<uint64_t>(blockIdx.x) * blockDim.x + threadIdx.x; b < n_blocks; b += stride) {
        const uint64_t lo = offs[b], hi = offs[b + 1];
        bad |= hi < lo || hi - lo > max_per_block || hi > n;
        if (b == 0) bad |= lo != 0;
        if (b + 1 == n_blocks) bad |= hi != n;
    }
    if (__any_sync(0xFFFFFFFFu, bad) && (threadIdx.x & 31) == 0) atomicOr(d_flags, DF_EFLAG_OFFSETS);
}

// The first index where a and b differ (atomicMin into *first).
__global__ void __launch_bounds__(256) compare_kernel(const uint16_t* __restrict__ a, const uint16_t* __restrict__ b,
                                                      uint64_t n, unsigned long long* __restrict__ first) {
    const uint64_t stride = static_cast<uint64_t>(gridDim.x) * blockDim.x;
    const uint64_t t0 = static_cast<uint64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    unsigned long long mine = ~0ull;
    uint64_t done = 0;
    if (!((reinterpret_cast<uintptr_t>(a) | reinterpret_cast<uintptr_t>(b)) & 15)) {
        // both 16-byte aligned: 8 weights per load, two loads of each in flight
        const uint4* a4 = reinterpret_cast<const uint4*>(a);
        const uint4* b4 = reinterpret_cast<const uint4*>(b);
        const uint64_t n8 = n / 8;
        for (uint64_t i = t0; i < n8; i += 2 * stride) {
            const bool two = i + stride < n8;
            const uint4 x0 = __ldg(a4 + i), y0 = __ldg(b4 + i);
            uint4 x1 = x0, y1 = y0;
            if (two) {
                x1 = __ldg(a4 + i + stride);
                y1 = __ldg(b4 + i + stride);
            }
            const uint32_t d0[4] = {x0.x ^ y0.x, x0.y ^ y0.y, x0.z ^ y0.z, x0.w ^ y0.w};
            const uint32_t d1[4] = {x1.x ^ y1.x, x1.y ^ y1.y, x1.z ^ y1.z, x1.w ^ y1.w};
            for (int k = 0; k < 8 && mine == ~0ull; ++k)
                if ((d0[k >> 1] >> (16 * (k & 1))) & 0xFFFFu) mine = 8 * i + k;
            for (int k = 0; k < 8 && two && mine == ~0ull; ++k)
                if ((d1[k >> 1] >> (16 * (k & 1))) & 0xFFFFu) mine = 8 * (i + stride) + k;
            if (mine != ~0ull) break;  // later indices of this thread are larger
        }
        done = 8 * n8;
    }
    for (uint64_t i = done + t0; i < n; i += stride)
        if (a[i] != b[i] && i < mine) mine = i;
    for (int d = 16; d > 0; d >>= 1) {
        const unsigned long long o = __shfl_xor_sync(0xFFFFFFFFu, mine, d);
        mine = o < mine ? o : mine;
    }
    if ((threadIdx.x & 31) == 0 && mine != ~0ull) atomicMin(first, mine);
}

df_status grid_for(uint64_t items, uint32_t threads, unsigned* grid) {
    int dev = 0, sms = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return cuda_fail(e);
    uint64_t g = (items + threads - 1) / threads;
    const uint64_t cap = static_cast<uint64_t>(sms) * 16;
    if (g > cap) g = cap;
    *grid = static_cast<unsigned>(g < 1 ? 1 : g);
    return DF_OK;
}

}  // namespace
}  // namespace df

using namespace df;

extern "C" {

df_status df_check_structure(const df_tensor* t, uint32_t* d_flags, void* stream) {
    if (!t || !d_flags || (t->n && !t->block_offsets)) return DF_ERR_INVALID_ARG;
    if (t->n == 0) return DF_OK;
    df_sizes z;
    df_status st = df_container_sizes(t->n, t->total_bits, t->chunk_bytes, t->threads_per_block, &z);
    if (st == DF_ERR_INVALID_ARG) {  // sizes no valid container has: a structure failure, not a bad call
        const uint32_t f = DF_EFLAG_OFFSETS;
        cudaError_t e = cudaMemcpyAsync(d_flags, &f, 4, cudaMemcpyHostToDevice, static_cast<cudaStream_t>(stream));
        if (e != cudaSuccess) return cuda_fail(e);
        e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
        return e == cudaSuccess ? DF_OK : cuda_fail(e);
    }
    if (st != DF_OK) return st;
    uint32_t minl = 0;
    for (int s = 0; s < 256; ++s)
        if (t->lengths[s] && (!minl || t->lengths[s] < minl)) minl = t->lengths[s];
    if (!minl) minl = 1;
    const uint64_t max_per_block = static_cast<uint64_t>(t->threads_per_block) * ((8ull * t->chunk_bytes + minl - 1) / minl);
    unsigned grid = 1;
    st = grid_for(z.n_blocks, 256, &grid);
    if (st != DF_OK) return st;
    structure_kernel<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(t->block_offsets, z.n_blocks, t->n,
                                                                          max_per_block, d_flags);
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? DF_OK : cuda_fail(e);
}

df_status df_compare(const uint16_t* d_a, const uint16_t* d_b, uint64_t n, uint64_t* d_first_diff, void* stream) {
    if ((n && (!d_a || !d_b)) || !d_first_diff) return DF_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemsetAsync(d_first_diff, 0xFF, 8, s);
    if (e != cudaSuccess) return cuda_fail(e);
    if (n == 0) return DF_OK;
    unsigned grid = 1;
    const df_status st = grid_for(n, 256, &grid);
    if (st != DF_OK) return st;
    compare_kernel<<<grid, 256, 0, s>>>(d_a, d_b, n, reinterpret_cast<unsigned long long*>(d_first_diff));
    e = cudaGetLastError();
    return e == cudaSuccess ? DF_OK : cuda_fail(e);
}

size_t df_sha256_workspace(uint64_t nbytes) {
    const uint64_t leaves = nbytes ? (nbytes + kLeafBytes - 1) / kLeafBytes : 1;
    return static_cast<size_t>(32 * leaves);
}

df_status df_sha256_device(const void* d_data, uint64_t nbytes, void* d_ws, size_t ws_bytes, uint8_t digest[32],
                           void* stream) {
    if (!digest || (nbytes && !d_data) || !d_ws) return DF_ERR_INVALID_ARG;
    if (ws_bytes < df_sha256_workspace(nbytes)) return DF_ERR_WORKSPACE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const uint64_t leaves = nbytes ? (nbytes + kLeafBytes - 1) / kLeafBytes : 0;
    std::vector<uint8_t> dig(32 * leaves);
    if (leaves) {
        sha256_leaves_kernel<<<static_cast<unsigned>((leaves + 127) / 128), 128, 0, s>>>(
            static_cast<const uint8_t*>(d_data), nbytes, leaves, static_cast<uint8_t*>(d_ws));
        cudaError_t e = cudaGetLastError();
        if (e == cudaSuccess) e = cudaMemcpyAsync(dig.data(), d_ws, dig.size(), cudaMemcpyDeviceToHost, s);
        if (e == cudaSuccess) e = cudaStreamSynchronize(s);
        if (e != cudaSuccess) return cuda_fail(e);
    }
    sha256(dig.data(), dig.size(), digest);
    return DF_OK;
}

df_status df_sha256(const void* data, uint64_t nbytes, uint8_t digest[32]) {
    if (!digest || (nbytes && !data)) return DF_ERR_INVALID_ARG;
    sha256(static_cast<const uint8_t*>(data), nbytes, digest);
    return DF_OK;
}

}  // extern "C"
