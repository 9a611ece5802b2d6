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
    uint32_t chunk_bytes;
    uint32_t vec_ok;       // sm and out 16-byte aligned
};

// Decode tables (the words df_build_lut writes), in order:
//   wide table, kWideBits = 10 bits of window per entry:
//     meta[1024] uint16: bit i (i < 10) set if a code starts at window bit i
//                        and lies wholly inside the window (at most 4 codes,
//                        taken from bit 0 on); bits 10-13: the bits those
//                        codes use (0: the first code is longer than 10 bits)
//     sym[1024]  uint32: their exponents, first in bits 0-7
//   8-bit-indexed tables for codes of any length (root + next levels):
//     leaf:  bits 0-7 the exponent, 8-13 its full code length, 24-25 = 1
//     link:  bits 0-15 index of the next-level table (>= 1), 24-25 = 0
//     unreachable: 0
//   code lengths: 256 bytes
constexpr uint32_t kWideBits = 10;
constexpr uint32_t kWideMaxCodes = 4;
constexpr uint32_t kWideMetaWords = (1u << kWideBits) / 2;
constexpr uint32_t kWideWords = kWideMetaWords + (1u << kWideBits);
constexpr uint32_t kNsymShift = 24;

inline __host__ __device__ uint32_t sub_leaf(uint32_t sym, uint32_t len) { return sym | (len << 8) | (1u << 24); }

// Records the CUDA error for df_last_cuda_error and maps it to DF_ERR_CUDA.
df_status cuda_fail(cudaError_t e);

}  // namespace df
