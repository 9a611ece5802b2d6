// Decode kernel: compressed exponent stream + sign|fraction bytes -> BF16.
//
// The pages fix what decoding restores (mlx-dfloat, PyPI page, intro: the
// exponent code is undone and the raw sign|fraction byte put back, bit for bit)
// and that it runs blockwise on the GPU (mlx-dfloat, "Status"; df11pack, intro).
// The layout of the work below is this library's own, written for sm_100a:
//
//   one CUDA block = one format block = T chunks of C bytes of stream
//   1. stage the decode tables and the block's stream slice
//      (byte-swapped to big-endian words) in shared memory
//   2. count pass: thread t decodes the codes that start in chunk t
//      (from chunk start + gap, up to the chunk end or the end of the stream)
//      through the 8-bit multi-code root table and counts them
//   3. block scan of the counts: each thread's first output position
//   4. check the block total against the block offsets (corrupt -> error bit)
//   5. write pass: decode again, exponent bytes into a shared-memory stage
//      placed so that stage index == output index mod 16
//   6. merge with the sign|fraction bytes: 16 weights per pair of 16-byte stores
#include <cuda_runtime.h>

#include <algorithm>
#include <cstring>
#include <vector>

#include "df_internal.h"

namespace df {
namespace {

constexpr int kMaxThreads = 1024;
constexpr uint32_t kSmemTableCap = 16;  // decode tables staged in shared memory

struct SingleSrc {
    DevTensor t;
    __device__ __forceinline__ const DevTensor* lookup(uint64_t g, uint64_t* local) const {
        *local = g;
        return &t;
    }
};

struct BatchSrc {
    const DevTensor* tensors;
    const uint64_t* block_start;  // count+1 prefix sums of n_blocks
    uint32_t count;
    __device__ __forceinline__ const DevTensor* lookup(uint64_t g, uint64_t* local) const {
        uint32_t lo = 0, hi = count;  // block_start[lo] <= g < block_start[hi]
        while (hi - lo > 1) {
            const uint32_t mid = (lo + hi) >> 1;
            if (block_start[mid] <= g)
                lo = mid;
            else
                hi = mid;
        }
        *local = g - block_start[lo];
        return tensors + lo;
    }
};

struct LaunchCfg {
    uint32_t chunk_bytes;
    uint32_t smem_tables;
    uint32_t stage_bytes;
    uint64_t total_blocks;
};

__device__ __forceinline__ uint32_t bswap32(uint32_t x) { return __byte_perm(x, 0, 0x0123); }

// Next-level lookup for codes longer than 8 bits. `win` holds the 32 bits
// starting at the code; returns the next-level leaf (exponent in bits 0-7,
// length in bits 8-13, count 1), or 0 for a path no code takes.
__device__ __forceinline__ uint32_t descend(uint32_t win, uint32_t e, const uint32_t* s_lut, const uint32_t* g_lut,
                                            uint32_t smem_tables) {
#pragma unroll
    for (int lvl = 1; lvl <= 3; ++lvl) {
        const uint32_t t = e & 0xFFFFu;
        if (t == 0) return 0;
        const uint32_t idx = (win >> (24 - 8 * lvl)) & 0xFFu;
        e = t < smem_tables ? s_lut[t * 256 + idx] : __ldg(g_lut + static_cast<size_t>(t) * 256 + idx);
        if ((e >> kNsymShift) & 3u) return e;
    }
    return 0;
}

struct BitWindow {
    const uint32_t* words;
    uint32_t wi, sh, cur, nxt;
    __device__ __forceinline__ void init(const uint32_t* w, uint32_t p) {
        words = w;
        wi = p >> 5;
        sh = p & 31;
        cur = w[wi];
        nxt = w[wi + 1];
    }
    // the 32 stream bits starting at the current position
    __device__ __forceinline__ uint32_t peek() const { return __funnelshift_l(nxt, cur, sh); }
    __device__ __forceinline__ void skip(uint32_t nb) {
        sh += nb;
        if (sh >= 32) {
            sh -= 32;
            cur = nxt;
            ++wi;
            nxt = words[wi + 1];
        }
    }
};

// Decode the codes that start in [p, end). kWrite=false counts them,
// kWrite=true also stores their exponents at stage[pos...]. Returns the
// count; an unreachable table entry sets *bad and ends the chunk.
// The loop runs in step across the warp (one vote per step) so that lanes
// that took the long-code path rejoin the others at once.
template <bool kWrite>
__device__ __forceinline__ uint32_t decode_chunk(const uint32_t* s_words, uint32_t p, uint32_t end,
                                                 const uint32_t* s_lut, const uint32_t* g_lut, uint32_t smem_tables,
                                                 uint8_t* stage, uint32_t pos, bool* bad) {
    BitWindow bw;
    bw.init(s_words, p);
    uint32_t cnt = 0;
    for (;;) {
        const bool act = p < end;
        if (!__any_sync(0xFFFFFFFFu, act)) break;
        if (act) {
            const uint32_t win = bw.peek();
            uint32_t e = s_lut[win >> 24];
            uint32_t ns = (e >> kNsymShift) & 3u;
            uint32_t nb;
            if (ns == 0) {  // a code longer than 8 bits (or corrupt data)
                e = descend(win, e, s_lut, g_lut, smem_tables);
                ns = (e >> kNsymShift) & 3u;
                nb = (e >> 8) & 63u;
                if (ns == 0) {
                    *bad = true;
                    end = p;
                }
            } else if (p + 8 > end) {  // near the end: only the first code surely starts before it
                ns = 1;
                nb = (e >> 29) + 1;
            } else {
                nb = ((e >> 26) & 7u) + 1;
            }
            if (kWrite) {
                if (ns > 0) stage[pos + cnt] = static_cast<uint8_t>(e);
                if (ns > 1) stage[pos + cnt + 1] = static_cast<uint8_t>(e >> 8);
                if (ns > 2) stage[pos + cnt + 2] = static_cast<uint8_t>(e >> 16);
            }
            cnt += ns;
            p += nb;
            bw.skip(nb);
        }
    }
    return cnt;
}

__device__ __forceinline__ uint32_t warp_incl_scan(uint32_t v, int lane) {
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const uint32_t u = __shfl_up_sync(0xFFFFFFFFu, v, d);
        if (lane >= d) v += u;
    }
    return v;
}

__device__ __forceinline__ uint16_t merge1(uint8_t sm, uint8_t e) {
    return static_cast<uint16_t>((static_cast<uint32_t>(sm & 0x80u) << 8) | (static_cast<uint32_t>(e) << 7) |
                                 (sm & 0x7Fu));
}

template <class Src>
__global__ void __launch_bounds__(kMaxThreads) decode_kernel(Src src, LaunchCfg cfg, uint32_t* d_err) {
    extern __shared__ __align__(16) uint8_t smem[];
    const uint32_t T = blockDim.x;
    const uint32_t tid = threadIdx.x;
    const uint32_t C = cfg.chunk_bytes;

    for (uint64_t g = blockIdx.x; g < cfg.total_blocks; g += gridDim.x) {
        uint64_t b;
        const DevTensor* td = src.lookup(g, &b);
        const uint32_t n_tables = td->n_tables;
        const uint32_t stab = n_tables < cfg.smem_tables ? n_tables : cfg.smem_tables;

        // shared memory carve-up
        uint32_t* s_lut = reinterpret_cast<uint32_t*>(smem);
        uint32_t* s_words = reinterpret_cast<uint32_t*>(smem + static_cast<size_t>(cfg.smem_tables) * 1024);
        const uint32_t slice_words = T * C / 4 + 4;
        uint32_t* s_warp = s_words + slice_words;
        uint8_t* s_stage = reinterpret_cast<uint8_t*>(s_warp + 32);

        // 1. tables, stream slice
        {
            const uint4* src4 = reinterpret_cast<const uint4*>(td->lut);
            uint4* dst4 = reinterpret_cast<uint4*>(s_lut);
            for (uint32_t i = tid; i < stab * 64; i += T) dst4[i] = __ldg(src4 + i);
            const uint64_t slice_byte0 = b * static_cast<uint64_t>(T) * C;
            const uint64_t stream_bytes = td->n_chunks * C + 16;
            const uint64_t avail = stream_bytes - slice_byte0;
            const uint32_t want16 = slice_words / 4;  // uint4 units
            const uint32_t have16 = avail / 16 < want16 ? static_cast<uint32_t>(avail / 16) : want16;
            const uint4* s4 = reinterpret_cast<const uint4*>(td->stream + slice_byte0);
            uint4* d4 = reinterpret_cast<uint4*>(s_words);
            for (uint32_t i = tid; i < want16; i += T) {
                uint4 v = make_uint4(0, 0, 0, 0);
                if (i < have16) v = __ldg(s4 + i);
                v.x = bswap32(v.x);
                v.y = bswap32(v.y);
                v.z = bswap32(v.z);
                v.w = bswap32(v.w);
                d4[i] = v;
            }
        }
        const uint64_t out0 = td->offs[b];
        const uint64_t out1 = td->offs[b + 1];
        __syncthreads();

        // this thread's chunk
        const uint64_t chunk = b * T + tid;
        const uint32_t cbits = 8 * C;
        uint32_t p0 = 0, end = 0;
        if (chunk < td->n_chunks) {
            const uint64_t q = 5 * chunk;
            const uint32_t two = (static_cast<uint32_t>(__ldg(td->gaps + (q >> 3))) << 8) |
                                 __ldg(td->gaps + (q >> 3) + 1);
            const uint32_t gap = (two >> (11 - (q & 7))) & 31u;
            const uint64_t chunk_bit0 = chunk * cbits;
            const uint64_t rem = td->total_bits > chunk_bit0 ? td->total_bits - chunk_bit0 : 0;
            p0 = tid * cbits + gap;
            end = tid * cbits + static_cast<uint32_t>(rem < cbits ? rem : cbits);
        }

        // 2. count pass
        bool bad = false;
        const uint32_t cnt = decode_chunk<false>(s_words, p0, end, s_lut, td->lut, stab, nullptr, 0, &bad);

        // 3. block scan
        const int lane = tid & 31, warp = tid >> 5;
        const uint32_t incl = warp_incl_scan(cnt, lane);
        if (lane == 31) s_warp[warp] = incl;
        __syncthreads();
        const uint32_t nwarps = T >> 5;
        if (warp == 0) {
            uint32_t v = lane < static_cast<int>(nwarps) ? s_warp[lane] : 0;
            v = warp_incl_scan(v, lane);
            if (lane < static_cast<int>(nwarps)) s_warp[lane] = v;
        }
        __syncthreads();
        const uint32_t excl = incl - cnt + (warp > 0 ? s_warp[warp - 1] : 0);
        const uint32_t total = s_warp[nwarps - 1];

        // 4. consistency with the block index
        const uint32_t align = static_cast<uint32_t>(out0 & 15);
        uint32_t flags = 0;
        if (out1 < out0 || out1 > td->n || out1 - out0 + align > cfg.stage_bytes ||
            (b + 1 == td->n_blocks && out1 != td->n))
            flags |= DF_EFLAG_OFFSETS;
        else if (static_cast<uint64_t>(total) != out1 - out0) flags |= DF_EFLAG_COUNT;
        const bool any_bad = __syncthreads_or(bad) != 0;
        if (any_bad) flags |= DF_EFLAG_BAD_CODE;
        if (flags) {
            if (tid == 0 && d_err) atomicOr(d_err, flags);
            __syncthreads();  // s_warp and the stage are reused by the next block
            continue;
        }

        // 5. write pass into the stage
        decode_chunk<true>(s_words, p0, end, s_lut, td->lut, stab, s_stage, align + excl, &bad);
        __syncthreads();

        // 6. merge and store: 16 weights per group (one 16-byte load of
        // sign|fraction bytes, one of staged exponents, two 16-byte stores);
        // two groups per thread per step keep two loads in flight
        const uint8_t* sm = td->sm;
        uint16_t* out = td->out;
        const uint64_t gbase = out0 & ~15ull;  // stage index 0 <-> output gbase
        const uint64_t ngroups = (out1 - gbase + 15) >> 4;
        const bool vec = td->vec_ok != 0;
        for (uint64_t g0 = tid; g0 < ngroups; g0 += 2 * static_cast<uint64_t>(T)) {
            uint4 s16[2];
            bool full[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const uint64_t gi = g0 + static_cast<uint64_t>(u) * T;
                const uint64_t G = gbase + 16 * gi;
                full[u] = vec && gi < ngroups && G >= out0 && G + 16 <= out1;
                if (full[u]) s16[u] = __ldg(reinterpret_cast<const uint4*>(sm + G));
            }
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const uint64_t gi = g0 + static_cast<uint64_t>(u) * T;
                if (gi >= ngroups) continue;
                const uint64_t G = gbase + 16 * gi;
                const uint32_t si = static_cast<uint32_t>(16 * gi);
                if (full[u]) {
                    const uint4 e16 = *reinterpret_cast<const uint4*>(s_stage + si);
                    const uint32_t sw[4] = {s16[u].x, s16[u].y, s16[u].z, s16[u].w};
                    const uint32_t ew[4] = {e16.x, e16.y, e16.z, e16.w};
                    uint32_t o[8];
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const uint32_t hi = (sw[k] & 0x80808080u) | ((ew[k] >> 1) & 0x7F7F7F7Fu);
                        const uint32_t lo = ((ew[k] << 7) & 0x80808080u) | (sw[k] & 0x7F7F7F7Fu);
                        o[2 * k] = __byte_perm(lo, hi, 0x5140);
                        o[2 * k + 1] = __byte_perm(lo, hi, 0x7362);
                    }
                    uint4* dst = reinterpret_cast<uint4*>(out + G);
                    dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
                    dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
                } else {
                    for (uint32_t k = 0; k < 16; ++k) {
                        const uint64_t i = G + k;
                        if (i >= out0 && i < out1) out[i] = merge1(sm[i], s_stage[si + k]);
                    }
                }
            }
        }
        __syncthreads();  // the next block overwrites shared memory
    }
}

struct Prepared {
    DevTensor dev;
    uint32_t stage_need;
};

uint32_t min_len_of(const uint8_t* lengths) {
    uint32_t m = 0;
    for (int s = 0; s < 256; ++s)
        if (lengths[s] && (!m || lengths[s] < m)) m = lengths[s];
    return m;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

// Validate a descriptor and fill the device-side copy.
df_status prepare(const df_tensor* t, uint16_t* out, Prepared* pr) {
    if (!t || !out) return DF_ERR_INVALID_ARG;
    const uint32_t C = t->chunk_bytes, T = t->threads_per_block;
    if (C < 16 || C > 4096 || C % 16 || T < 32 || T > kMaxThreads || T % 32) return DF_ERR_INVALID_ARG;
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
    d.vec_ok = aligned(t->sm, 16) && aligned(out, 16);
    pr->dev = d;
    // a block holds at most 8CT/min_len codes, and never more than n
    uint64_t need = minl ? (cbits * T + minl - 1) / minl : 0;
    if (need > t->n) need = t->n;
    need = (need + 16 + 15) & ~15ull;  // + alignment slack
    if (need > (1u << 30)) return DF_ERR_UNSUPPORTED;
    pr->stage_need = static_cast<uint32_t>(need);
    return DF_OK;
}

size_t smem_bytes(uint32_t tables, uint32_t C, uint32_t T, uint32_t stage) {
    return static_cast<size_t>(tables) * 1024 + (static_cast<size_t>(T) * C / 4 + 4) * 4 + 32 * 4 + stage;
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

template <class Src>
df_status launch(const Src& src, const LaunchCfg& cfg, uint32_t T, size_t smem, uint32_t* d_err,
                 cudaStream_t stream) {
    int sms = 0, max_smem = 0;
    df_status st = device_limits(&sms, &max_smem);
    if (st != DF_OK) return st;
    if (smem > static_cast<size_t>(max_smem)) return DF_ERR_UNSUPPORTED;
    cudaError_t e = cudaFuncSetAttribute(decode_kernel<Src>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return cuda_fail(e);
    const uint64_t grid = cfg.total_blocks < 0x7FFFFFFFull ? cfg.total_blocks : 0x7FFFFFFFull;
    if (grid == 0) return DF_OK;
    decode_kernel<Src><<<static_cast<unsigned>(grid), T, smem, stream>>>(src, cfg, d_err);
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e);
    return DF_OK;
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
    cfg.chunk_bytes = t->chunk_bytes;
    cfg.smem_tables = std::min<uint32_t>(t->n_tables, kSmemTableCap);
    cfg.stage_bytes = pr.stage_need;
    cfg.total_blocks = pr.dev.n_blocks;
    const size_t smem = smem_bytes(cfg.smem_tables, t->chunk_bytes, t->threads_per_block, cfg.stage_bytes);
    return launch(src, cfg, t->threads_per_block, smem, d_err, static_cast<cudaStream_t>(stream));
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
    uint32_t C = 0, T = 0, stage = 16, tables = 1;
    for (uint32_t i = 0; i < count; ++i) {
        const df_tensor* t = tensors + i;
        if (t->n == 0) continue;
        Prepared pr;
        df_status st = prepare(t, d_outs[i], &pr);
        if (st != DF_OK) return st;
        if (!C) {
            C = t->chunk_bytes;
            T = t->threads_per_block;
        } else if (C != t->chunk_bytes || T != t->threads_per_block) {
            return DF_ERR_INVALID_ARG;
        }
        stage = std::max(stage, pr.stage_need);
        tables = std::max(tables, std::min<uint32_t>(t->n_tables, kSmemTableCap));
        dev.push_back(pr.dev);
        start.push_back(start.back() + pr.dev.n_blocks);
    }
    plan->d_ws = d_ws;
    plan->count = static_cast<uint32_t>(dev.size());
    plan->threads_per_block = T;
    plan->chunk_bytes = C;
    plan->smem_tables = tables;
    plan->stage_bytes = stage;
    plan->total_blocks = start.back();
    if (plan->count == 0) return DF_OK;
    const size_t sm = smem_bytes(tables, C, T, stage);
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
    // same layout as df_decode_batch_prepare writes
    BatchSrc src;
    src.tensors = static_cast<const DevTensor*>(plan->d_ws);
    src.count = plan->count;
    src.block_start = nullptr;
    const size_t table_bytes = (static_cast<size_t>(plan->count) * sizeof(DevTensor) + 255) / 256 * 256;
    src.block_start = reinterpret_cast<const uint64_t*>(static_cast<const uint8_t*>(plan->d_ws) + table_bytes);
    LaunchCfg cfg;
    cfg.chunk_bytes = plan->chunk_bytes;
    cfg.smem_tables = plan->smem_tables;
    cfg.stage_bytes = plan->stage_bytes;
    cfg.total_blocks = plan->total_blocks;
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
