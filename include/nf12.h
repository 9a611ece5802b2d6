/* nf12.h - the fixed 12-bit lossless BF16 format on the GPU (sm_100a).
 *
 * A second codec beside the Huffman one of df11.h: every weight keeps its
 * sign, its 7 fraction bits and the low 4 of its 8 exponent bits; the top 4
 * exponent bits, the same for nearly all weights of a trained model, are left
 * out. Source: agihunt.info, "Developer open-sources nf12: lossless 12-bit
 * compression for BF16 models", section "Confirmed" (the top exponent bits
 * 0111 are shared and elided; groups of 8 weights pack from 16 bytes to 12;
 * a group that cannot be packed is escaped, 28 bytes in all; decode is
 * bit-exact).
 *
 * Layout (the page gives none; these are this library's readings), for n
 * weights in G = ceil(n / 8) groups of 8, the last group padded with weights
 * whose top exponent bits are `top` and whose other bits are 0:
 *   slots   12 G bytes. Normal group g: field k of weight k is
 *           f = sign << 11 | (exponent & 15) << 7 | fraction, and the 96-bit
 *           little-endian value of bytes 12g .. 12g+11 is sum f_k << 12k.
 *           Escaped group: uint32 LE side index, then 8 zero bytes.
 *   bitmap  4 ceil(G / 32) bytes, uint32 words: bit g & 31 of word g >> 5 is
 *           set when group g is escaped; bits past G are 0.
 *   side    16 bytes per escaped group, in group order: the 8 raw weights
 *           (padded as above for the last group).
 * A group is escaped when one of its weights has top exponent bits other
 * than `top` (4 bits; the page's 0111 = 7 is the usual value).
 *
 * Conventions as in df11.h: d_ pointers are device memory, the library
 * allocates nothing and never synchronizes; every call enqueues on `stream`
 * (a cudaStream_t; NULL = the legacy default stream). Device error words are
 * uint32, OR-ed with DF_EFLAG_* bits; the caller zeroes them.
 * Alignment: weights (d_in, d_out, tensor.out) 2 bytes, slots and bitmap 4,
 * side 16; the kernels use 16-byte accesses where weights are 16-aligned.
 */
#ifndef NF12_H
#define NF12_H

#include <stddef.h>
#include <stdint.h>

#include "df11.h"

#ifdef __cplusplus
extern "C" {
#endif

#define DF_NF12_TOP 7u                 /* the page's shared top exponent bits 0111 */
#define DF_NF12_TILE_GROUPS 2048u      /* groups per CUDA block in the kernels     */
#define DF_EFLAG_NF12_SIDE 128u        /* a side index past the escaped groups     */

typedef struct df_nf12_sizes {
    uint64_t groups;          /* G = ceil(n / 8)                        */
    uint64_t slots_bytes;     /* 12 G                                   */
    uint64_t bitmap_bytes;    /* 4 ceil(G / 32)                         */
    uint64_t tiles;           /* ceil(G / DF_NF12_TILE_GROUPS)          */
    uint64_t encode_ws_bytes; /* per-tile escape counts: 8 (tiles + 1)  */
} df_nf12_sizes;

/* One tensor of a grouped decode (host array; copied by the prepare call). */
typedef struct df_nf12_tensor {
    uint64_t n;               /* weights                                */
    uint64_t n_escaped;       /* escaped groups (side entries)          */
    const void* slots;        /* device, 12 G bytes, 4-byte aligned     */
    const void* bitmap;       /* device, 4 ceil(G / 32) bytes           */
    const void* side;         /* device, 16 n_escaped bytes, 16-aligned; may be NULL when n_escaped = 0 */
    void* out;                /* device, n uint16 (BF16 bits)           */
    uint32_t top;             /* shared top exponent bits, 0..15        */
    uint32_t reserved;        /* 0                                      */
} df_nf12_tensor;

typedef struct df_nf12_plan {
    void* d_ws;               /* descriptors + tile starts, set by prepare */
    uint32_t count;
    uint32_t reserved;
    uint64_t total_tiles;
} df_nf12_plan;

/* Sizes of the parts for n weights. Source: agihunt.info nf12 item,
 * "Confirmed" (16 -> 12 bytes per group of 8; 28 bytes per escaped group, of
 * which 16 sit in the side buffer). Errors: DF_ERR_INVALID_ARG (out NULL),
 * DF_ERR_UNSUPPORTED (n > DF_MAX_WEIGHTS). */
df_status df_nf12_sizes_for(uint64_t n, df_nf12_sizes* out);

/* Encode, first half: writes the slots of every group (an escaped group's
 * slot gets zeros for now), the bitmap, and per-tile escape counts with their
 * exclusive prefix in d_ws (sizes.encode_ws_bytes); writes the number of
 * escaped groups to *d_escaped (device uint64). Read it to size the side
 * buffer, then call df_nf12_encode_escapes. Source: agihunt.info nf12 item,
 * "Confirmed" (groups of 8 packed to 12 bytes; groups that cannot be packed
 * flagged as outliers). Errors: DF_ERR_INVALID_ARG (null pointers, top > 15,
 * misalignment), DF_ERR_WORKSPACE, DF_ERR_UNSUPPORTED, DF_ERR_CUDA. */
df_status df_nf12_encode_groups(const uint16_t* d_in, uint64_t n, uint32_t top, void* d_slots, void* d_bitmap,
                                void* d_ws, size_t ws_bytes, uint64_t* d_escaped, void* stream);

/* Encode, second half: for every escaped group, in group order, copies its 8
 * raw weights to the side buffer and writes the side index into its slot.
 * side_capacity is the side buffer's size in groups; an index at or past it
 * is not written and sets DF_EFLAG_NF12_SIDE in d_err (nullable). Same
 * d_in, n, top, d_slots, d_bitmap and d_ws as the first half. Source:
 * agihunt.info nf12 item, "Confirmed" (original BF16 values of an outlier
 * group go to an escape buffer). Errors: DF_ERR_INVALID_ARG, DF_ERR_WORKSPACE,
 * DF_ERR_CUDA. */
df_status df_nf12_encode_escapes(const uint16_t* d_in, uint64_t n, uint32_t top, void* d_slots,
                                 const void* d_bitmap, const void* d_ws, size_t ws_bytes, void* d_side,
                                 uint64_t side_capacity, uint32_t* d_err, void* stream);

/* Decode one tensor: the n BF16 weights to d_out. A side index at or past
 * n_escaped sets DF_EFLAG_NF12_SIDE in d_err (nullable) and leaves that
 * group's 8 outputs as decoded from its slot. Source: agihunt.info nf12 item,
 * "Confirmed" (the elided bits are restored at decode; decoded weights are
 * bit-identical). Errors: DF_ERR_INVALID_ARG, DF_ERR_UNSUPPORTED, DF_ERR_CUDA. */
df_status df_nf12_decode(const df_nf12_tensor* t, uint32_t* d_err, void* stream);

/* Bytes of device workspace a grouped decode of `count` tensors needs. Source:
 * no counterpart in the pages (a launch detail). */
size_t df_nf12_decode_batch_workspace(uint32_t count);

/* Grouped decode, set-up: copies the descriptors and each tensor's first
 * tile into d_ws (enqueued on `stream`; h_tensors is read before the call
 * returns and may be freed then) and fills *plan. Source: agihunt.info nf12 item, "Confirmed" (decode of a whole
 * model's weights). Errors: DF_ERR_INVALID_ARG, DF_ERR_WORKSPACE,
 * DF_ERR_UNSUPPORTED, DF_ERR_CUDA. */
df_status df_nf12_decode_batch_prepare(const df_nf12_tensor* h_tensors, uint32_t count, void* d_ws,
                                       size_t ws_bytes, df_nf12_plan* plan, void* stream);

/* Grouped decode, launch: one kernel over every tile of every prepared
 * tensor (safe to capture in a CUDA graph). Errors as df_nf12_decode. Source:
 * agihunt.info nf12 item, "Confirmed". */
df_status df_nf12_decode_batch_run(const df_nf12_plan* plan, uint32_t* d_err, void* stream);

/* One tensor of a grouped encode (host array; copied by the prepare call). */
typedef struct df_nf12_encode_tensor {
    const uint16_t* in;       /* device, n weights (BF16 bits), 2-byte aligned   */
    uint64_t n;
    void* slots;              /* device, 12 G bytes, 4-byte aligned             */
    void* bitmap;             /* device, 4 ceil(G / 32) bytes, 4-byte aligned    */
    void* side;               /* device, 16 side_capacity bytes, 16-byte aligned;
                                 NULL before the escape counts are known        */
    uint64_t side_capacity;   /* side entries (groups) the buffer holds         */
    uint32_t top;             /* shared top exponent bits, 0..15                */
    uint32_t reserved;        /* 0                                              */
    uint64_t reserved2;       /* 0                                              */
} df_nf12_encode_tensor;

/* Bytes of device workspace a grouped encode of these tensors needs
 * (descriptors, tile starts, per-tile escape counts and per-tensor totals).
 * Source: no counterpart in the pages (a launch detail). */
size_t df_nf12_encode_batch_workspace(const df_nf12_encode_tensor* h_tensors, uint32_t count);

/* Grouped encode, set-up: copies the descriptors into d_ws (enqueued on
 * `stream`; h_tensors is read before the call returns) and fills *plan. Call
 * it again with the side buffers filled in before the escapes (the escape
 * counts in d_ws are kept). Source: agihunt.info nf12 item, "Confirmed".
 * Errors: DF_ERR_INVALID_ARG, DF_ERR_WORKSPACE, DF_ERR_UNSUPPORTED,
 * DF_ERR_CUDA. */
df_status df_nf12_encode_batch_prepare(const df_nf12_encode_tensor* h_tensors, uint32_t count, void* d_ws,
                                       size_t ws_bytes, df_nf12_plan* plan, void* stream);

/* Grouped encode, first half: the slots and bitmap of every tensor (one
 * launch over all their tiles) and each tensor's escape count, written to
 * d_escaped[0 .. count) (device uint64). Source: as df_nf12_encode_groups.
 * Errors: DF_ERR_INVALID_ARG, DF_ERR_CUDA. */
df_status df_nf12_encode_batch_groups(const df_nf12_plan* plan, uint64_t* d_escaped, void* stream);

/* Grouped encode, second half: every tensor's side buffer and side indices,
 * as df_nf12_encode_escapes does for one (a tensor whose escapes exceed its
 * side_capacity sets DF_EFLAG_NF12_SIDE in d_err). Source: as
 * df_nf12_encode_escapes. Errors: DF_ERR_INVALID_ARG, DF_ERR_CUDA. */
df_status df_nf12_encode_batch_escapes(const df_nf12_plan* plan, uint32_t* d_err, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* NF12_H */
