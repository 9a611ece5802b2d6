/*
 * df11.h - C ABI of the B200 (sm_100a) exponent-Huffman BF16 weight codec.
 *
 * What the codec does (mlx-dfloat, PyPI page, intro and its bit diagram): a
 * BF16 weight is s | eeeeeeee | mmmmmmm; the 8 exponent bits are replaced by
 * a variable-length prefix code and the sign and 7 fraction bits are kept as
 * one raw byte, so that decoding gives back the original bits exactly. The
 * codebook is built deterministically from the exponent frequencies
 * (df11pack, GitHub page, intro and "Licence"), codes have a maximum length
 * (mlx-dfloat, "Try it": the "max-code" group), the decoder uses lookup tables
 * and a block index (df11pack, "What is checked": --luts=correct,
 * --index idx8) and the stream is cut into independently decodable chunks
 * (df11pack, "Use": --safe and verify decode units and chunks). The pages do
 * not give a container layout; this header defines it.
 *
 * Container of one tensor of n weights (all sizes from df_plan):
 *   stream  n_chunks*C bytes of code bits, most significant bit first (the
 *           first code bit is bit 7 of byte 0), zero after the last code,
 *           then 16 zero bytes. n_chunks = max(1, ceil(total_bits / 8C)).
 *   gaps    one 5-bit field per chunk, MSB first, zero padded (at least one
 *           byte, to a multiple of 16 bytes). gap[j] = (first code start at
 *           or after bit 8Cj) - 8Cj, where the end of the stream counts as a
 *           code start; a code belongs to the chunk that holds its first bit.
 *   block_offsets  n_blocks+1 uint64: offsets[b] = number of codes that start
 *           before bit 8*C*T*b; offsets[n_blocks] = n. n_blocks = ceil(n_chunks/T).
 *   sm      n bytes: sm[i] = (w >> 8 & 0x80) | (w & 0x7F).
 *   lengths 256 code lengths (0 = symbol absent), canonical codes: symbols in
 *           (length, symbol) order, code = (previous + 1) << (length step).
 * C (chunk_bytes, a multiple of 16) and T (threads_per_block: chunks per
 * format block, a multiple of 32) are per-tensor parameters; the defaults are
 * C = 32 and T = 32 (a block of T chunks is the unit one warp starts on, so
 * small T spreads small tensors over more warps; each block costs 8 bytes).
 *
 * Conventions for every function:
 *   - returns a df_status; nothing is thrown across the ABI;
 *   - device pointers are owned by the caller; the library allocates no device
 *     memory and frees nothing; workspaces are passed in;
 *   - kernels are launched asynchronously on `stream`, a cudaStream_t passed
 *     as void* (NULL = the legacy default stream); a DF_OK return means the
 *     launch was accepted, not that the data was valid: decode-time data
 *     errors are reported through the optional device error word `d_err`
 *     (DF_EFLAG_* bits OR-ed in; the caller zeroes it) and df_read_error;
 *   - no function keeps global mutable state except the per-thread last CUDA
 *     error returned by df_last_cuda_error and df_encode_noalloc's static
 *     device scratch (with its per-device address, looked up once).
 */
#ifndef DF11_H
#define DF11_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef int df_status;
#define DF_OK 0
#define DF_ERR_INVALID_ARG 1 /* a null, misaligned or inconsistent argument     */
#define DF_ERR_CUDA 2        /* a CUDA call failed; see df_last_cuda_error()   */
#define DF_ERR_CORRUPT 3     /* the device error word reported corrupt data     */
#define DF_ERR_UNSUPPORTED 4 /* valid but outside this library's limits         */
#define DF_ERR_WORKSPACE 5   /* workspace too small                             */

/* bits of the device error word */
#define DF_EFLAG_BAD_CODE 1u      /* decode: a bit pattern no code starts with        */
#define DF_EFLAG_COUNT 2u         /* decode: codes in a block != its offset difference */
#define DF_EFLAG_OFFSETS 4u       /* decode: block offsets out of range               */
#define DF_EFLAG_TABLES 8u        /* decode: tables not built for this descriptor      */
#define DF_EFLAG_ENC_TOTAL 16u    /* encode: stream length != the planned total_bits   */
#define DF_EFLAG_ENC_SYMBOL 32u   /* encode: an exponent without a code                */
#define DF_EFLAG_ENC_WAIT 64u     /* encode: a tile waited too long for the one before */
#define DF_EFLAG_INDEX8 256u      /* compact index: wide superblocks past the room given,
                                     or an overflow slot past the wide count          */

#define DF_DEFAULT_CHUNK_BYTES 32u
#define DF_DEFAULT_THREADS_PER_BLOCK 32u
#define DF_DEFAULT_MAX_LEN 32u
#define DF_MAX_WEIGHTS (1ull << 48) /* n above this is DF_ERR_UNSUPPORTED */

/* A code table. Built by df_build_code from an exponent histogram. */
typedef struct df_code {
    uint32_t max_len;    /* the length limit the code was built with (1..32) */
    uint32_t n_symbols;  /* exponents with a code                            */
    uint32_t min_len;    /* shortest code length (0 when n_symbols == 0)     */
    uint32_t n_tables;   /* 256-entry decode tables (see df_build_lut)       */
    uint8_t lengths[256];
    uint32_t codes[256]; /* canonical code of each exponent, right-aligned   */
} df_code;

/* Exact sizes of one tensor's container and of the encode workspace. */
typedef struct df_sizes {
    uint64_t total_bits, n_chunks, stream_bytes, gap_bytes, n_blocks, offsets_bytes, sm_bytes;
    uint64_t container_bytes; /* stream + gaps + offsets + sm + 256 lengths + 64-byte header */
    uint64_t encode_ws_bytes; /* device workspace df_encode needs                           */
} df_sizes;

/* Descriptor of one compressed tensor for decoding. Device pointers are
 * read only; lut is the device copy of df_build_lut's output. */
typedef struct df_tensor {
    uint64_t n;
    uint64_t total_bits;
    uint32_t chunk_bytes;
    uint32_t threads_per_block;
    uint32_t max_len;
    uint32_t n_tables;
    const uint8_t* stream;         /* 16-byte aligned                 */
    const uint8_t* gaps;
    const uint64_t* block_offsets; /* 8-byte aligned; NULL when the compact
                                      index below is given instead     */
    const uint8_t* sm;             /* 8-byte aligned for vector loads  */
    const uint32_t* lut;           /* 16-byte aligned                 */
    uint8_t lengths[256];          /* host copy of the code lengths   */
    const uint8_t* index8;         /* compact block index (df_index8_build),
                                      8-byte aligned; used when
                                      block_offsets is NULL, else NULL */
    uint64_t index8_wide;          /* its wide superblocks (df_index8_build) */
} df_tensor;

/* Host plan of a grouped decode, filled by df_decode_batch_prepare. */
typedef struct df_batch_plan {
    void* d_ws;                /* the workspace holding the device table        */
    uint32_t count;            /* tensors with n > 0                            */
    uint32_t cta_threads;      /* threads per CUDA block of the launch          */
    uint32_t words_per_chunk;  /* shared-memory words per chunk (widest C)      */
    uint32_t region_bytes;     /* shared-memory exponent region of a lane       */
    uint32_t max_groups;       /* 16-output groups a round of 32 chunks spans   */
    uint32_t smem_bytes;       /* dynamic shared memory per CUDA block          */
    uint32_t max_ctas;         /* 0: as many CUDA blocks as fit on the GPU; else
                                  at most this many (the caller may set it
                                  between prepare and run, e.g. to leave SMs to
                                  a kernel running beside the decode)          */
    uint32_t reserved;         /* 0                                             */
    uint64_t total_blocks;     /* format blocks over all tensors                */
} df_batch_plan;

/* One tensor of a grouped encode (host array; read by
 * df_encode_batch_prepare before it returns). Inputs and outputs as
 * df_encode's arguments of the same names. A table whose `code` entries are
 * all NULL plans the histograms only; a table with every code set (and its
 * outputs) plans the encode as well. */
typedef struct df_encode_tensor {
    const uint16_t* in;        /* device, n BF16 bit patterns, 2-byte aligned   */
    uint64_t n;
    const df_code* code;       /* host; NULL until the histogram is known      */
    uint64_t total_bits;       /* df_plan's value for this tensor and code     */
    uint32_t chunk_bytes;      /* C: multiple of 16 in 16..4096                */
    uint32_t threads_per_block; /* T: multiple of 32 in 32..1024               */
    uint8_t* stream;           /* device, sizes.stream_bytes, 16-byte aligned  */
    uint8_t* gaps;             /* device, sizes.gap_bytes, 4-byte aligned      */
    uint64_t* block_offsets;   /* device, n_blocks + 1, 8-byte aligned         */
    uint8_t* sm;               /* device, n bytes                              */
} df_encode_tensor;

/* Host plan of a grouped encode, filled by df_encode_batch_prepare. */
typedef struct df_encode_plan {
    void* d_ws;                /* the workspace holding the device tables       */
    uint32_t count;            /* tensors                                       */
    uint32_t has_codes;        /* 1: every tensor has its code and outputs      */
    uint64_t sum_tiles;        /* sum of ceil(n / 4096) (sizes the workspace)   */
    uint64_t hist_tiles;       /* CUDA blocks of the grouped histogram          */
    uint64_t hist_tile_weights; /* weights per histogram CUDA block             */
    uint64_t ranges;           /* encode ranges over all tensors               */
    uint64_t zero_tiles;       /* CUDA blocks that zero the outputs             */
} df_encode_plan;

/* Human-readable name of a status. Static string; never NULL.
 * Source: none on the pages (an error-reporting helper of this ABI). */
const char* df_status_string(df_status s);

/* The cudaError_t of the last failing CUDA call made by this thread inside
 * the library (0 if none). Source: none on the pages (an error-reporting
 * helper of this ABI). */
int df_last_cuda_error(void);

/* ---- code construction (host only) ---------------------------------------
 * df_build_code: optimal prefix code over the exponents with hist[e] > 0 and
 * no code longer than max_len (1..32), by package-merge (Larmore and
 * Hirschberg 1990) with ties resolved as: items sorted by (count, exponent), an
 * item before a package of equal weight. One exponent gets length 1 (code 0);
 * an empty histogram gives an empty code. Then canonical codes.
 * Source: df11pack (GitHub page), intro and "Licence" (deterministic codebook
 * from frequencies); mlx-dfloat (PyPI page), "Try it" (a maximum code length).
 * Errors: DF_ERR_INVALID_ARG for null pointers; DF_ERR_UNSUPPORTED when
 * max_len is outside 1..32 or 2^max_len is below the number of exponents.
 */
df_status df_build_code(const uint64_t hist[256], uint32_t max_len, df_code* out);

/* df_code_from_lengths: the canonical code for given code lengths (0 = no
 * code), e.g. the lengths stored in a container. Source: df11pack, intro
 * (the codebook is a function of the stored frequencies/lengths, so a reader
 * rebuilds the same code). Errors: DF_ERR_INVALID_ARG
 * (null, a length above max_len, or lengths that break Kraft's inequality
 * sum 2^-l <= 1); DF_ERR_UNSUPPORTED (max_len outside 1..32). */
df_status df_code_from_lengths(const uint8_t lengths[256], uint32_t max_len, df_code* out);

/* Number of uint32 words df_build_lut writes: the wide table (5 words per
 * window value), 256 per 8-bit-indexed table, 64 for the code lengths and a
 * 4-word header. 0 for a NULL code. Source: df11pack, "What is checked"
 * (decode lookup tables). */
size_t df_lut_words(const df_code* code);

/* df_build_lut: derive the decode tables of a code into host memory `lut`
 * (lut_words >= df_lut_words(code)); the caller copies the words to the
 * device and passes them as df_tensor.lut. Layout, in order:
 *   - the wide table: 4096 uint64 indexed by the next 12 stream bits; an
 *     entry holds the exponents of the codes that lie wholly inside the
 *     window from its first bit on (up to 4, bits 0-31, the first in bits
 *     0-7) and, in bits 32-63, (bits they use << 18) | (their count << 3),
 *     or 0 when the first code is longer than 12 bits;
 *   - 4096 uint16: for each window, the mask of the window bits where those
 *     codes start;
 *   - n_tables tables of 256 uint32 indexed by 8 stream bits, for codes of
 *     any length: a leaf holds the exponent (bits 0-7), the full code length
 *     (bits 8-13) and a 1 in bits 24-25; a link holds the index of the
 *     next-level table (bits 0-15, >= 1) and 0 in bits 24-25; table 0 is the
 *     root, at most four levels for 32-bit codes;
 *   - the 256 code lengths as bytes;
 *   - a header: the shortest code length, max_len, n_tables, 0xDF11DF12.
 * Entries no code reaches are zero. Source: df11pack, "What is checked"
 * (--luts=correct zero-fills unreachable table entries).
 * Errors: DF_ERR_INVALID_ARG (null, too small, or a code that is not prefix free).
 */
df_status df_build_lut(const df_code* code, uint32_t* lut, size_t lut_words);

/* df_plan: exact sizes of the container for n weights with exponent
 * histogram hist under `code`, and of df_encode's workspace. Source:
 * mlx-dfloat, intro (the container is the exponent code plus one raw byte per
 * weight); the byte counts follow the layout at the top of this header.
 * Errors: DF_ERR_INVALID_ARG (null; hist total != n; an exponent present in
 * hist without a code; chunk_bytes not a multiple of 16 in 16..4096;
 * threads_per_block not a multiple of 32 in 32..1024); DF_ERR_UNSUPPORTED
 * (n > DF_MAX_WEIGHTS). */
df_status df_plan(const df_code* code, const uint64_t hist[256], uint64_t n, uint32_t chunk_bytes,
                  uint32_t threads_per_block, df_sizes* out);

/* df_container_sizes: the same sizes for a container whose histogram is not
 * at hand (one read from a file, one to be filled by df_encode): n weights
 * and total_bits code bits under chunk_bytes and threads_per_block. The
 * buffer sizes depend on nothing else. Source: the container layout at the
 * top of this header (the pages give none). Errors: DF_ERR_INVALID_ARG (null;
 * the format checks of df_plan; total_bits outside [n, 32n]);
 * DF_ERR_UNSUPPORTED (n > DF_MAX_WEIGHTS). */
df_status df_container_sizes(uint64_t n, uint64_t total_bits, uint32_t chunk_bytes, uint32_t threads_per_block,
                             df_sizes* out);

/* ---- encode (device) ---------------------------------------------------------
 * df_histogram: d_hist256[e] = number of weights of d_in[0..n) whose exponent
 * bits (w >> 7 & 0xFF) equal e. Overwrites d_hist256 (256 uint64, device,
 * 8-byte aligned). d_in: n uint16 BF16 bit patterns on the device, 2-byte
 * aligned (16-byte alignment takes the vector path). Source: df11pack, intro
 * (codebook from exponent frequencies). Errors: DF_ERR_INVALID_ARG,
 * DF_ERR_CUDA.
 */
df_status df_histogram(const uint16_t* d_in, uint64_t n, uint64_t* d_hist256, void* stream);

/* df_encode: write the container of d_in[0..n) under `code`: d_stream
 * (sizes.stream_bytes, 16-byte aligned), d_gaps (sizes.gap_bytes, 4-byte
 * aligned), d_block_offsets (n_blocks+1 uint64), d_sm (n bytes). The bytes
 * equal those of the layout above for the same code. d_ws: device workspace
 * of at least sizes.encode_ws_bytes (16-byte aligned). total_bits is the
 * value df_plan returned for the same input; a mismatch, or an exponent
 * without a code, sets DF_EFLAG_ENC_* in d_err (nullable). Source:
 * mlx-dfloat, intro bit diagram (what is coded and what is kept raw).
 * Errors: DF_ERR_INVALID_ARG, DF_ERR_WORKSPACE, DF_ERR_CUDA.
 */
df_status df_encode(const df_code* code, const uint16_t* d_in, uint64_t n, uint64_t total_bits,
                    uint32_t chunk_bytes, uint32_t threads_per_block, uint8_t* d_stream, uint8_t* d_gaps,
                    uint64_t* d_block_offsets, uint8_t* d_sm, void* d_ws, size_t ws_bytes, uint32_t* d_err,
                    void* stream);

/* df_encode_noalloc: df_encode without a workspace argument, for callers
 * that cannot allocate device memory when they encode (for example a
 * runtime that owns all device memory up front in a fixed arena, or a plug-in
 * that may only use the buffers its host hands it). Its scratch (per-tile bit
 * counts and bases) lives in a static device array of the library, 2 MiB per
 * GPU that loads the library, held until the process exits; n is limited to
 * DF_ENCODE_NOALLOC_MAX_WEIGHTS. A call looks up the array's device address
 * (cudaGetSymbolAddress) on its device, except while `stream` is capturing,
 * when the address found by the last call on that device is used; so make
 * the first call on a device before any stream capture (a first call inside
 * a capture returns DF_ERR_UNSUPPORTED), and after a device reset call it
 * once outside a capture before capturing it again. Every call on a device shares the
 * array, so calls that overlap on the GPU (other streams, other host threads)
 * race: serialize them. Allocates nothing: no cudaMalloc, cudaFree or
 * allocating library routine. The pages have no counterpart of this entry
 * point. Arguments, outputs and errors as df_encode, plus DF_ERR_UNSUPPORTED
 * when n > DF_ENCODE_NOALLOC_MAX_WEIGHTS.
 */
#define DF_ENCODE_NOALLOC_MAX_WEIGHTS (1ull << 29) /* 536,870,912 weights */
df_status df_encode_noalloc(const df_code* code, const uint16_t* d_in, uint64_t n, uint64_t total_bits,
                            uint32_t chunk_bytes, uint32_t threads_per_block, uint8_t* d_stream, uint8_t* d_gaps,
                            uint64_t* d_block_offsets, uint8_t* d_sm, uint32_t* d_err, void* stream);

/* ---- grouped encode (device) ---------------------------------------------------
 * df_histogram and df_encode over many tensors with one launch per step for
 * all of them, so that many small tensors (biases, norms, small linears) cost
 * a few launches instead of several each. Every tensor's histogram and
 * container bytes equal those of df_histogram and df_encode on it alone.
 * Source: df11pack, intro (the codebook from each tensor's exponent
 * frequencies; the compressor's speed over a whole model's tensors is the
 * page's headline, "Measured"); grouping them into one launch is this
 * library's own.
 *
 * df_encode_batch_workspace: device workspace bytes for these tensors (only
 * their n is read, so one workspace serves both prepare calls). */
size_t df_encode_batch_workspace(const df_encode_tensor* h_tensors, uint32_t count);

/* df_encode_batch_prepare: validate the table, copy the device descriptors
 * (and the codes, when every tensor has one) into d_ws (16-byte aligned)
 * asynchronously on `stream`, and fill *plan. Call it once with the codes
 * NULL to run the histograms, then again with every code and output set
 * (after df_build_code and df_plan on the host) to run the encode. Errors:
 * DF_ERR_INVALID_ARG (a bad pointer, alignment or format, a code length over
 * 32, codes set for some tensors only), DF_ERR_WORKSPACE, DF_ERR_UNSUPPORTED
 * (n > DF_MAX_WEIGHTS; more than 2^31 - 1 CUDA blocks or ranges), DF_ERR_CUDA.
 * Source: as the section above. */
df_status df_encode_batch_prepare(const df_encode_tensor* h_tensors, uint32_t count, void* d_ws, size_t ws_bytes,
                                  df_encode_plan* plan, void* stream);

/* df_histogram_batch_run: d_hist[256 t + e] = the number of weights of tensor
 * t whose exponent bits equal e, for every tensor of the plan (d_hist: count
 * x 256 uint64, device, 8-byte aligned; overwritten). One launch over fixed
 * tiles of every tensor. Source: as df_histogram. Errors: DF_ERR_INVALID_ARG,
 * DF_ERR_CUDA. */
df_status df_histogram_batch_run(const df_encode_plan* plan, uint64_t* d_hist, void* stream);

/* df_encode_batch_run: write every tensor's container, as df_encode does for
 * one: a launch that zeroes all outputs, then one over ranges of every tensor
 * (a tensor's look-back stays within its own ranges). Needs a plan prepared
 * with every code. A wrong total_bits or an exponent without a code sets
 * DF_EFLAG_ENC_* in d_err (nullable), as in df_encode. Source: as df_encode.
 * Errors: DF_ERR_INVALID_ARG, DF_ERR_CUDA. */
df_status df_encode_batch_run(const df_encode_plan* plan, uint32_t* d_err, void* stream);

/* ---- decode (device) ---------------------------------------------------------
 * df_decode: d_out[0..t->n) = the original BF16 bit patterns (uint16, device;
 * 16-byte alignment of d_out and t->sm takes the vector path). Every warp
 * decodes whole format blocks on its own, 32 chunks at a time: each lane
 * decodes one chunk into a shared-memory region of exponents (multi-code
 * table lookups), a warp scan turns the counts into output positions, and
 * the warp merges the exponents with the sign|fraction bytes in groups of 16
 * outputs (16-byte loads and stores). Chunks of up to 1024 bytes. Source:
 * mlx-dfloat, intro and "Status" (blockwise GPU decode back to identical
 * bits); df11pack, "Use" (independently decodable chunks).
 * Data errors set DF_EFLAG_* in d_err (nullable); the affected block stops
 * at the round (32 chunks) where the error shows, so its outputs may be
 * partly written, never outside d_out[0..n). Errors: DF_ERR_INVALID_ARG,
 * DF_ERR_UNSUPPORTED (a layout whose warp needs more shared memory than the
 * device has), DF_ERR_CUDA.
 */
df_status df_decode(const df_tensor* t, uint16_t* d_out, uint32_t* d_err, void* stream);

/* Device workspace bytes df_decode_batch needs for `count` tensors.
 * Source: none on the pages (the grouped launch is this library's own). */
size_t df_decode_batch_workspace(uint32_t count);

/* df_decode_batch_prepare: validate `count` descriptors (host array) and
 * their outputs (host array of device pointers), write the device table into
 * d_ws (asynchronously on `stream`; the host arrays may be reused on return)
 * and fill *plan. chunk_bytes and threads_per_block may differ between
 * tensors (shared memory is sized for the widest chunk). Source: none on the
 * pages: one launch over many tensors (biases, norms, small linears) is this
 * library's own entry point; each tensor decodes as in df_decode.
 * Errors: DF_ERR_INVALID_ARG, DF_ERR_WORKSPACE, DF_ERR_UNSUPPORTED, DF_ERR_CUDA. */
df_status df_decode_batch_prepare(const df_tensor* tensors, uint16_t* const* d_outs, uint32_t count, void* d_ws,
                                  size_t ws_bytes, df_batch_plan* plan, void* stream);

/* df_decode_batch_run: decode every tensor of a prepared table in one launch
 * (persistent CUDA blocks over the format blocks of all tensors; block ->
 * tensor by a binary search of the prefix sum of block counts). The
 * workspace must hold the prepared table until the launch has run.
 * Source: none on the pages (see df_decode_batch_prepare); per tensor as
 * df_decode. Errors: DF_ERR_INVALID_ARG, DF_ERR_CUDA. */
df_status df_decode_batch_run(const df_batch_plan* plan, uint32_t* d_err, void* stream);

/* df_decode_batch: prepare + run. Source: none on the pages (see
 * df_decode_batch_prepare). */
df_status df_decode_batch(const df_tensor* tensors, uint16_t* const* d_outs, uint32_t count, void* d_ws,
                          size_t ws_bytes, uint32_t* d_err, void* stream);

/* df_read_error: wait for `stream`, copy the device error word to *flags
 * (nullable) and return DF_ERR_CORRUPT if any bit is set, else DF_OK.
 * Source: df11pack, "Use" (a check reports pass, mismatch or could-not-check:
 * here DF_OK, DF_ERR_CORRUPT, or another status).
 * Errors: DF_ERR_INVALID_ARG, DF_ERR_CUDA. */
df_status df_read_error(const uint32_t* d_err, void* stream, uint32_t* flags);

/* ---- checks (df11pack, GitHub page, "Use": verify checks a container's
 * structure with no source, decodes sampled chunks, or all of them, and
 * compares them with the source, exiting 0 on pass, 1 when a check fails, 2
 * when it could not check; "What is checked": --hashes, a per-tensor SHA-256
 * that lets verify catch corruption without the source) ------------------- */

/* df_check_structure: the container's block offsets, without decoding:
 * offsets[0] = 0, offsets never decrease, offsets[n_blocks] = n, and no block
 * holds more codes than its chunks can (T * ceil(8C / shortest code length)).
 * Sizes no container can have (total_bits outside [n, 32n], a bad format) also
 * fail. A failure ORs DF_EFLAG_OFFSETS into *d_flags (device word, caller
 * zeroes it; read it with df_read_error). Source: df11pack, "Use" (verify:
 * structure, no source needed). Errors: DF_ERR_INVALID_ARG, DF_ERR_CUDA. */
df_status df_check_structure(const df_tensor* t, uint32_t* d_flags, void* stream);

/* df_compare: *d_first_diff (device uint64) = the first i < n with
 * d_a[i] != d_b[i], or UINT64_MAX when they are equal (both device arrays of n
 * uint16). Source: df11pack, "Use" (decoded chunks compared with the source).
 * Errors: DF_ERR_INVALID_ARG, DF_ERR_CUDA. */
df_status df_compare(const uint16_t* d_a, const uint16_t* d_b, uint64_t n, uint64_t* d_first_diff, void* stream);

/* Device workspace bytes df_sha256_device needs for nbytes of data (32 per
 * leaf). Source: as df_sha256_device. */
size_t df_sha256_workspace(uint64_t nbytes);

/* df_sha256_device: the digest of nbytes of device data, a tree over SHA-256
 * (FIPS 180-4): the data is cut into leaves of 65,536 bytes (the last one
 * shorter; none for nbytes = 0), each leaf is hashed on the GPU, and digest =
 * SHA-256 of the leaf digests in order (computed on the host after waiting
 * for `stream`). Source: df11pack, "What is checked" (--hashes: a per-tensor
 * SHA-256); the leaf tree is this library's own, so that a large tensor hashes
 * in parallel. Errors: DF_ERR_INVALID_ARG, DF_ERR_WORKSPACE, DF_ERR_CUDA. */
df_status df_sha256_device(const void* d_data, uint64_t nbytes, void* d_ws, size_t ws_bytes, uint8_t digest[32],
                           void* stream);

/* df_sha256: plain SHA-256 (FIPS 180-4) of nbytes of host data. Source: as
 * df_sha256_device. Errors: DF_ERR_INVALID_ARG. */
df_status df_sha256(const void* data, uint64_t nbytes, uint8_t digest[32]);

/* ---- compact block index ----------------------------------------------
 * In place of one uint64 output offset per format block (block_offsets,
 * O[0] = 0 .. O[B] = n; block b holds c_b = O[b+1] - O[b] codes), blocks are
 * grouped in superblocks of 64, S = ceil(B / 64), and one buffer holds:
 *   [0, 8S)          anchor[s], uint64: O[64 s]
 *   [8S, 12S)        base[s], uint32: the smallest count of superblock s when
 *                    all its counts lie within 255 of it; else 2^31 | k, k =
 *                    how many wide superblocks come before s
 *   [12S, 76S)       delta[b], uint8: c_b - base[s] (0 in a wide superblock
 *                    and past the last block)
 *   [76S, 76S+256W)  overflow: the 64 counts (uint32) of each of the W wide
 *                    superblocks, in order (0 past the last block)
 * So O[64 s + j] = anchor[s] + c_{64 s} + ... + c_{64 s + j - 1}. Source:
 * df11pack (GitHub page), "What is checked, and what is not", opt-in
 * --index idx8: an experimental 8-bit block index that makes the file
 * smaller; the page gives no layout, this one is the library's own. */

/* Bytes of a compact index of n_blocks blocks with n_wide wide superblocks:
 * 76 ceil(n_blocks / 64) + 256 n_wide. Source: as above. */
uint64_t df_index8_bytes(uint64_t n_blocks, uint64_t n_wide);

/* Build the compact index of d_offsets (n_blocks + 1 device uint64 offsets)
 * into d_index8 (index8_bytes bytes, 8-byte aligned). Wide superblocks past
 * the room that index8_bytes leaves for the overflow are not written and set
 * DF_EFLAG_INDEX8 in d_err (nullable); *d_n_wide (device uint64) gets the
 * number of wide superblocks, so a caller that gave room for none reads it
 * and builds again. A count of 2^31 or more also sets DF_EFLAG_INDEX8.
 * Source: as above. Errors: DF_ERR_INVALID_ARG (null, misaligned, index8_bytes
 * below df_index8_bytes(n_blocks, 0)), DF_ERR_UNSUPPORTED (n_blocks >= 2^32),
 * DF_ERR_CUDA. */
df_status df_index8_build(const uint64_t* d_offsets, uint64_t n_blocks, void* d_index8, size_t index8_bytes,
                          uint64_t* d_n_wide, uint32_t* d_err, void* stream);

/* The block offsets (n_blocks + 1 device uint64, O[0] from anchor[0]) back
 * from a compact index with n_wide wide superblocks. An overflow slot at or
 * past n_wide sets DF_EFLAG_INDEX8 in d_err (nullable) and counts as 0.
 * Source: as above. Errors: DF_ERR_INVALID_ARG, DF_ERR_UNSUPPORTED, DF_ERR_CUDA. */
df_status df_index8_expand(const void* d_index8, uint64_t n_blocks, uint64_t n_wide, uint64_t* d_offsets,
                           uint32_t* d_err, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* DF11_H */
