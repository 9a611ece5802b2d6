// Internal declarations shared by the library's host and device sources.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "df11.h"

namespace df {

// Device-side descriptor of one tensor (one per tensor in a grouped decode).
struct DevTensor {
    const uint8_t* stream;
    const uint8_t* gaps;
    const uint64_t* offs;
    const uint8_t* sm;
    const uint32_t* lut;   // n_tables*256 table words, then 64 words of lengths
    uint16_t* out;
    uint64_t n;
    uint64_t total_bits;
    uint64_t n_chunks;
    uint32_t n_blocks;
    uint32_t n_tables;
    uint32_t vec_ok;       // sm 8-byte and out 16-byte aligned
    uint32_t pad;
};

// Decode-table entries (uint32).
//   root table, leaf:  bits 0-23 up to three exponents (first in bits 0-7),
//                      24-25 how many (1..3), 26-28 bits they use - 1,
//                      29-31 length of the first code - 1
//   next-level leaf:   bits 0-7 the exponent, 8-13 its full code length,
//                      24-25 = 1
//   link (any table):  bits 0-15 index of the next-level table (>= 1), 24-25 = 0
//   unreachable:       0
constexpr uint32_t kNsymShift = 24;
constexpr uint32_t kNbitsShift = 26;  // build-time single-code form: full length in bits 26-31

inline __host__ __device__ uint32_t lut_leaf(uint32_t syms, uint32_t nsym, uint32_t nbits) {
    return syms | (nsym << kNsymShift) | (nbits << kNbitsShift);
}
inline __host__ __device__ uint32_t root_entry(uint32_t syms, uint32_t nsym, uint32_t used, uint32_t len0) {
    return syms | (nsym << 24) | ((used - 1) << 26) | ((len0 - 1) << 29);
}
inline __host__ __device__ uint32_t sub_leaf(uint32_t sym, uint32_t len) { return sym | (len << 8) | (1u << 24); }

// Records the CUDA error for df_last_cuda_error and maps it to DF_ERR_CUDA.
df_status cuda_fail(cudaError_t e);

}  // namespace df
