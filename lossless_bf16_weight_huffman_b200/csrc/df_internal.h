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
    const uint64_t* offs;  // block offsets, or the compact index when idx8 != 0
    const uint8_t* sm;
    const uint32_t* lut;   // n_tables*256 table words, then 64 words of lengths
    uint16_t* out;
    uint64_t n;
    uint64_t total_bits;
    uint64_t n_chunks;
    uint32_t n_blocks;
    uint32_t n_tables;
    uint32_t chunk_bytes;  // C
    uint32_t tpb;          // T: chunks per format block
    uint32_t vec_ok;       // sm and out 16-byte aligned
    uint32_t idx8;         // 0: offs holds uint64 block offsets; else the compact
                           // index with idx8 - 1 wide superblocks
};
static_assert(sizeof(DevTensor) % 16 == 0, "descriptors are copied and placed in 16-byte units");

// Decode tables (the words df_build_lut writes), in order:
//   wide table, 4096 uint64 indexed by the next kWideBits = 12 stream bits:
//     bits 0-31  the exponents of the codes that lie wholly inside the window,
//                taken from its first bit on (at most 4; first in bits 0-7)
//     bits 32-63 (bits used << 18) | (how many codes << 3); 0 when the first
//                code is longer than the window. A decoder whose state word is
//                (bit position << 18) | (codes so far << 3) advances by one
//                add, and (state & 24) is the byte shift of the next exponent
//                within a 32-bit word.
//   wide start masks, 4096 uint16: bit i set when one of those codes starts
//     at window bit i
//   8-bit-indexed tables for codes of any length (root + next levels):
//     leaf:  bits 0-7 the exponent, 8-13 its full code length, 24-25 = 1
//     link:  bits 0-15 index of the next-level table (>= 1), 24-25 = 0
//     unreachable: 0
//   code lengths: 256 bytes
//   header, 4 words: shortest code length, max_len, n_tables, kLutMagic
constexpr uint32_t kWideBits = 12;
constexpr uint32_t kWideMaxCodes = 4;
constexpr uint32_t kStepShift = 18;                     // bits-used field of a step word
constexpr uint32_t kStepCountMask = (1u << kStepShift) - 1;
constexpr uint32_t kStepCountShift = 3;                 // the count field holds count << 3
constexpr uint32_t kWideEntryWords = 2u << kWideBits;   // the uint64 entries
constexpr uint32_t kWideMaskWords = (1u << kWideBits) / 2;
constexpr uint32_t kWideWords = kWideEntryWords + kWideMaskWords;
constexpr uint32_t kNsymShift = 24;
constexpr uint32_t kLutMagic = 0xDF11DF12u;

inline __host__ __device__ uint32_t sub_leaf(uint32_t sym, uint32_t len) { return sym | (len << 8) | (1u << 24); }

// Records the CUDA error for df_last_cuda_error and maps it to DF_ERR_CUDA.
df_status cuda_fail(cudaError_t e);

}  // namespace df
