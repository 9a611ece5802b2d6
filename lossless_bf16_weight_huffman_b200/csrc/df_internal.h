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

// LUT entry fields.
constexpr uint32_t kNsymShift = 24;
constexpr uint32_t kNbitsShift = 26;

inline __host__ __device__ uint32_t lut_leaf(uint32_t syms, uint32_t nsym, uint32_t nbits) {
    return syms | (nsym << kNsymShift) | (nbits << kNbitsShift);
}

// Records the CUDA error for df_last_cuda_error and maps it to DF_ERR_CUDA.
df_status cuda_fail(cudaError_t e);

}  // namespace df
