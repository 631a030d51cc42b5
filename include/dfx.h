/*
 * dfx.h -- C ABI of libdfx, a lossless BF16 weight codec for NVIDIA B200 (sm_100a).
 *
 * The problem the calls solve: store BF16 network weights smaller, losslessly,
 * and restore them bit for bit on the GPU before use.  The weight distribution
 * of trained networks has low entropy, so an entropy code that gives frequent
 * values short codes removes the redundancy of the 16-bit format without
 * changing a single bit of the decoded weights ("DFloat11: lossless LLM
 * compression for GPU", aikraft.ru blog, section 02; a ~1.5:1 ratio on
 * Llama 2 7B weights is reported in "From a Lossless (~1.5:1) Compression
 * Algorithm for Llama2 7B Weights to Variable Precision, Variable Range,
 * Compressed Numeric Data Types for CNNs and LLMs", abstract).  The GPU decoder
 * uses lookup tables in on-chip shared memory and per-thread auxiliary
 * position variables (the same blog, section 03, items 1 and 2).
 *
 * Coding scheme (this library's reading; the pages leave it open):
 *   - every BF16 word w[x] is split into its exponent e = (w[x] >> 7) & 0xFF and
 *     the mantissa+sign byte m[x] = ((w[x] & 0x7F) << 1) | (w[p] >> 15): its
 *     mantissa above the sign of its partner p = x ^ 1 (p = x when x ^ 1 >= n).
 *     For a pair (2i, 2i+1) the 32-bit word m[2i] | e[2i] << 8 | m[2i+1] << 16 |
 *     e[2i+1] << 24 rotated right by one bit is the two BF16 words;
 *   - the exponents are coded with a per-tensor canonical Huffman code whose
 *     lengths come from package-merge with a length limit (24 by default),
 *     leaves ordered by (count, symbol value), a leaf ahead of a package of
 *     equal weight, codes assigned in (length, symbol) order; a tensor with a
 *     single exponent value gets a second, never-used phantom symbol (1 if the
 *     value is 0, else 0) so both codes are 1 bit long;
 *   - or (coder 1, DFX_CODER_TANS) the exponents are coded with tabled asymmetric
 *     numeral systems (tANS; one page names ANS as the coder of its compressed
 *     number formats: the "From a Lossless (~1.5:1) ..." abstract) over a table of
 *     M = 2^table_log states: every used exponent gets f[s] = count * M / n rounded
 *     half up (at least 1), the largest f (smallest symbol among equal ones) taking a
 *     shortfall or giving up an excess one unit at a time; occurrence i of the
 *     symbol-ordered list of f[s] copies per symbol takes slot (i * step) mod M,
 *     step = M/2 + M/8 + 3; each symbol's slots, ascending, are states f[s] ..
 *     2 f[s] - 1; a chunk is encoded from its last symbol to its first from state M
 *     (for symbol s, nb bits with f[s] <= X >> nb < 2 f[s] are emitted, low bits of
 *     X, and X becomes M + the slot of state X >> nb) and stored as the final state
 *     minus M (table_log bits) followed by the fields in symbol order (a chunk of the
 *     last group with no element has no bits);
 *   - or (coder 2, DFX_CODER_TANS2) the same tANS code with two interleaved states
 *     per chunk: the symbols at even positions of a chunk are coded by state A, those
 *     at odd positions by state B, each as above from state M on its own, and the
 *     chunk is stored as A's final state minus M, B's final state minus M, then every
 *     symbol's field in symbol order (a decoder's two table lookups per symbol pair
 *     are independent; a chunk costs table_log bits more);
 *   - the m bytes are stored raw, in element order;
 *   - the exponent codes are cut into chunks of K codes, 32 chunks to a group:
 *     a group covers 32*K consecutive elements in 8-element blocks, block b of
 *     the group belongs to chunk b mod 32, and a chunk's codes follow its
 *     blocks in order; the chunks of the last group hold only elements below n
 *     (possibly none).
 *
 * Container ("DFX1", all integers little-endian, every section starts on a
 * 16-byte boundary, every padding byte zero):
 *   off  0  char[4] "DFX1"; u16 version = 1; u16 header_bytes = 64
 *   off  8  u64 n                 BF16 elements
 *   off 16  u64 total_bits        code stream length in bits
 *   off 24  u64 total_bytes       container size
 *   off 32  u32 K                 symbols per chunk (one decoding thread), a multiple of 8
 *   off 36  u32 G                 chunks per group (one warp)
 *   off 40  u32 n_chunk = G * n_group;  off 44  u32 n_group = ceil(n / (G * K))
 *   off 48  u64 off_m             offset of the sign+mantissa plane
 *   off 56  u32 max_len;          off 60  u32 coder = 0
 *   off 64  u8  len[256]          code length per exponent value, 0 = unused
 *   off 320 u64 gbase[n_group+1]  start bit of each group; last = total_bits
 *   then    u16 clen[n_chunk]     bit length of each chunk (0 for an empty chunk)
 *   then    u8  m[n]              mantissa+sign bytes in element order (above)
 *   then    u32 stream[]          codes MSB-first: bit k of the stream is bit
 *                                 31 - (k mod 32) of word k / 32; the section
 *                                 is 4*ceil(total_bits/32) bytes rounded up
 *                                 to 16, plus 16 zero bytes
 * Coder 1 changes three things: off 56 holds table_log (4..12), off 60 holds
 * coder = 1, and u16 freq[256] (summing to 2^table_log, all 0 when n = 0) sits at
 * off 64 with gbase following at off 576; the other sections are as above.
 * Two conforming encoders produce identical bytes for the same input and
 * parameters.
 *
 * Memory and streams.  The caller owns every device buffer and the stream.
 * The library allocates device memory only inside dfx_plan (one small status
 * buffer per plan) and frees it in dfx_free.  Every call is asynchronous and
 * stream-ordered unless stated otherwise.  Input and output buffers must not
 * overlap.  A plan may be used by one host thread at a time.
 *
 * Errors.  Every call returns DFX_OK or one of the DFX_ERR_* codes below.
 * Argument errors are detected on the host before anything is launched.  A
 * corrupt container is detected by the decode kernel, which never traps and
 * never reads outside [d_comp, d_comp + comp_bytes): it records a flag in the
 * plan's sticky device status word, read with dfx_device_status.
 */
#ifndef DFX_H_
#define DFX_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* The CUDA runtime's stream handle (identical to the CUDA headers' typedef). */
typedef struct CUstream_st *cudaStream_t;

#define DFX_OK 0
#define DFX_ERR_ARG 1          /* bad pointer, size, alignment or parameter */
#define DFX_ERR_CAPACITY 2     /* output or workspace buffer too small */
#define DFX_ERR_CORRUPT 3      /* container malformed (host check or device status) */
#define DFX_ERR_TOO_LARGE 4    /* n >= 2^32 */
#define DFX_ERR_CUDA 5         /* a CUDA runtime call failed */
#define DFX_ERR_UNSUPPORTED 6  /* valid parameters this GPU path does not implement */

/* Bits of the device status word (dfx_device_status). */
#define DFX_STATUS_HEADER 0x1u  /* header disagrees with the plan or the buffer size */
#define DFX_STATUS_TABLE 0x2u   /* code lengths above 24 or Kraft sum not exactly 1
                                   (coder 1: frequencies not summing to 2^table_log) */
#define DFX_STATUS_INDEX 0x4u   /* group start bits or chunk lengths inconsistent */
#define DFX_STATUS_STREAM 0x8u  /* a bit pattern that is no code, or a chunk that
                                   did not consume exactly its stated length */
#define DFX_STATUS_TIMEOUT 0x10u /* a copy into shared memory did not complete within the
                                   kernel's bounded wait; the output is not valid */

typedef struct dfx_plan_s *dfx_plan_t; /* opaque, host-owned */

/* Exponent coders. */
#define DFX_CODER_HUFFMAN 0u /* canonical length-limited Huffman (the default) */
#define DFX_CODER_TANS 1u    /* tabled asymmetric numeral systems */
#define DFX_CODER_TANS2 2u   /* tANS with two interleaved states per chunk */

typedef struct {
    uint32_t chunk_symbols; /* K: a multiple of 8; 32, 64 or 128 on the GPU path (0 -> 128) */
    uint32_t group_chunks;  /* G: 32 on the GPU path (0 -> 32) */
    uint32_t max_len;       /* coder 0: code-length limit, 8..24 (0 -> 24) */
    uint32_t coder;         /* DFX_CODER_HUFFMAN, DFX_CODER_TANS or DFX_CODER_TANS2 */
    uint32_t table_log;     /* coders 1, 2: log2 of the state table, 4..12 (0 -> 12); dfx_encode
                               needs 8..12 (room for all 256 exponent values), every value
                               decodes */
    uint32_t decode_flags;  /* 0 or DFX_DECODE_EARLY_READ */
} dfx_params;

/* Decode flag: the kernel that precedes a decode of this plan in its stream never writes
 * that decode's container (for instance the containers of a model's weights, written
 * once before layer-by-layer decoding starts).  The decode kernels are launched as
 * programmatic dependents of the work before them, so their CTAs can start while the
 * preceding kernel finishes; with this flag a CTA also reads the container's header,
 * builds its tables and starts copying its first group during that time, and waits for
 * the preceding kernel only before its first output write.  Without it (the default)
 * the CTA waits before it reads anything, which is always safe.  Applies to dfx_decode,
 * dfx_decode_range, dfx_decode_batch, dfx_decode_host and dfx_decode_gemm (which, with
 * the flag, reads X and writes Y and W only after the wait). */
#define DFX_DECODE_EARLY_READ 0x1u

/* Byte offsets of the container sections for given n, params and stream length. */
typedef struct {
    uint64_t n, n_chunk, n_group;
    uint64_t off_len, off_gbase, off_clen, off_m, off_stream;  /* off_len: the code section */
    uint64_t stream_bytes, total_bytes;
} dfx_layout;

/* Library version, (major << 16) | minor. */
uint32_t dfx_version(void);

/* Static description of an error code; never NULL. */
const char *dfx_strerror(int code);

/* Host-only: container layout for n elements, params (NULL = defaults) and a
 * stream of total_bits bits.  Pure arithmetic, no CUDA call. */
int dfx_container_layout(uint64_t n, const dfx_params *params, uint64_t total_bits, dfx_layout *out);

/* Create a plan for tensors of n BF16 elements on the current CUDA device.
 *   params                NULL or parameters (see dfx_params; zero fields take defaults)
 *   max_compressed_bytes  out (may be NULL): capacity an encode output buffer needs;
 *                         an optimal code never costs more than 8 bits per exponent
 *   workspace_bytes       out (may be NULL): device scratch size dfx_encode needs
 * Allocates the plan's device status word.  Argument errors are returned before
 * any CUDA call.  Synchronous. */
int dfx_plan(dfx_plan_t *plan, uint64_t n, const dfx_params *params,
             size_t *max_compressed_bytes, size_t *workspace_bytes);

/* Encode n BF16 elements (d_bf16, device, 16-byte aligned) into a DFX1
 * container at d_out (device, 16-byte aligned, out_capacity >=
 * max_compressed_bytes).  d_workspace: device scratch of workspace_bytes
 * (16-byte aligned), contents on entry ignored.  The bytes of d_out past the
 * container's end (up to max_compressed_bytes) are not part of the result: the
 * Huffman coder leaves them as they were, the tANS coders zero them.
 * h_compressed_bytes: NULL keeps the call asynchronous; otherwise the call
 * synchronises the stream and stores the container size.  The size is also
 * in the header at byte offset 24 (u64). */
int dfx_encode(dfx_plan_t plan, const void *d_bf16, void *d_out, size_t out_capacity,
               void *d_workspace, size_t workspace_bytes, size_t *h_compressed_bytes,
               cudaStream_t stream);

/* Decode a DFX1 container (d_comp, device, 16-byte aligned, comp_bytes long,
 * produced with this plan's n and parameters) into n BF16 elements at d_bf16
 * (device, 16-byte aligned).  One kernel launch.  A malformed container sets
 * bits of the plan's device status word and leaves d_bf16 partly unwritten;
 * the call itself only reports host-side errors. */
int dfx_decode(dfx_plan_t plan, const void *d_comp, size_t comp_bytes, void *d_bf16,
               cudaStream_t stream);

/* Decode part of a container: the elements of groups [first_group, first_group +
 * group_count) (a group is 32 chunks of chunk_symbols elements, so rows of a
 * weight matrix whose length is a multiple of 32 * chunk_symbols are whole
 * groups) into d_bf16, which receives element first_group * 32 *
 * chunk_symbols at d_bf16[0] and ends at element n at the latest.  This lets a
 * caller restore a weight matrix slice by slice into a small (L2-sized) buffer
 * just before the computation that reads it, instead of writing the whole BF16
 * tensor to HBM (the pages decode weights on the GPU ahead of the computation
 * that uses them: "DFloat11: lossless LLM compression for GPU", section 02).
 * d_comp, comp_bytes: the whole container, as for dfx_decode (its header and
 * index are checked every call).  A range past the last group returns
 * DFX_ERR_ARG; group_count = 0 is a no-op.  Asynchronous; one kernel launch with
 * a CTA per 32 groups up to one per SM. */
int dfx_decode_range(dfx_plan_t plan, const void *d_comp, size_t comp_bytes, uint64_t first_group,
                     uint64_t group_count, void *d_bf16, cudaStream_t stream);

/* Decode a container that sits in host memory, streaming it to the device while
 * it decodes: the weights of a model kept in host memory and brought to the GPU
 * compressed, so the host link carries the container instead of the BF16 tensor.
 * The pages name the slow host-to-GPU link as what limits offloaded weights
 * ("DFloat11: lossless LLM compression for GPU", section 01) and shorten that
 * transfer by sending the weights compressed (the Endor abstract, for pruned
 * weights).  The header and index are copied first, then the groups in
 * `slices` runs (0 -> 8, at most 64): each run's sign+mantissa bytes and stream
 * words are copied with cudaMemcpyAsync on copy_stream and decoded with
 * dfx_decode_range on decode_stream once they have landed, so copies and decoding
 * overlap.
 *   h_comp: the container in host memory (pinned, for the copies to run
 *   asynchronously), comp_bytes long; d_staging: device buffer of staging_bytes
 *   >= the container's size (16-byte aligned), which receives the container;
 *   d_bf16: the n BF16 outputs.  The host reads the container's size and group
 *   index directly from h_comp.  Errors as for dfx_decode; staging too small ->
 *   DFX_ERR_CAPACITY.  The copies into d_staging wait for the work already
 *   queued on decode_stream when the call starts, so a call may reuse the
 *   staging buffer of an earlier call on that stream (work queued on other
 *   streams that reads d_staging is the caller's to order).  The plan's slice
 *   events order copies and decoding, so calls on the same plan must be issued
 *   from one host thread at a time.  Returns after queueing the work; h_comp
 *   must stay valid until copy_stream has finished it. */
int dfx_decode_host(dfx_plan_t plan, const void *h_comp, size_t comp_bytes, void *d_staging,
                    size_t staging_bytes, void *d_bf16, uint32_t slices, cudaStream_t copy_stream,
                    cudaStream_t decode_stream);

/* Y = X W^T with the weight matrix W restored from its container inside the kernel
 * that multiplies it: the decoded BF16 weights go from the decoding threads into
 * shared-memory tiles read by the tensor cores (tcgen05.mma, FP32 accumulation in
 * tensor memory) and are never written to HBM.  The pages decompress weights on
 * the GPU just before the computation that uses them, rebuilding them in a form
 * ready for that computation ("DFloat11: lossless LLM compression for GPU",
 * aikraft.ru blog, section 02 and section 03, item 2).
 *   plan, d_comp, comp_bytes: as for dfx_decode; coder 0 (Huffman) only, else
 *     DFX_ERR_UNSUPPORTED.
 *   rows, cols: W's shape, row-major in the container's element order (rows * cols
 *     must equal the plan's n, else DFX_ERR_ARG); cols must be a multiple of
 *     32 * chunk_symbols (every group inside one row), else DFX_ERR_UNSUPPORTED.
 *   d_x: X, tokens x cols BF16, row-major, device, 16-byte aligned; 1 <= tokens <= 32,
 *     else DFX_ERR_ARG.
 *   d_y: Y, tokens x rows FP32, row-major, device, 16-byte aligned; written whole.
 *   d_w_out: NULL, or a device buffer (16-byte aligned) of rows * cols BF16 that also
 *     receives the decoded W (for checking the decode; costs the 2n-byte write the
 *     fused path otherwise avoids).
 * Y is the exact product rounded by FP32 accumulation in an order of the hardware's
 * choosing.  A corrupt container sets the plan's status word as dfx_decode does (Y
 * is then not valid).  Asynchronous; one kernel launch of one CTA per SM, each
 * decoding a tile of at most 100 rows once and feeding it to the tensor cores. */
int dfx_decode_gemm(dfx_plan_t plan, const void *d_comp, size_t comp_bytes, uint64_t rows, uint64_t cols,
                    const void *d_x, uint32_t tokens, float *d_y, void *d_w_out, cudaStream_t stream);

/* Decode `count` containers (1..32; 0 is a no-op) with one kernel launch: a
 * whole layer's weights restored before use in one go (the pages decode a
 * model's compressed weights on the GPU ahead of the computation that reads
 * them: "DFloat11: lossless LLM compression for GPU", title and section 02).
 * plans[i], d_comps[i], comp_bytes[i], d_bf16s[i]: as for dfx_decode, one per
 * tensor (host arrays of count entries; the buffers are device memory).  All
 * plans must belong to the current device and share chunk_symbols, else
 * DFX_ERR_UNSUPPORTED; host argument errors of any tensor return before any
 * launch.  The device's CTAs are split among the tensors in proportion to their
 * groups, each CTA decoding part of one tensor.  Corruption is reported in each
 * tensor's own plan status word.  Outputs must not overlap each other or the
 * containers.  Asynchronous. */
int dfx_decode_batch(const dfx_plan_t *plans, const void *const *d_comps, const size_t *comp_bytes,
                     void *const *d_bf16s, uint32_t count, cudaStream_t stream);

/* Synchronise `stream`, return the plan's sticky device status word in
 * *h_status (0 = no corruption seen since the last read) and clear it. */
int dfx_device_status(dfx_plan_t plan, cudaStream_t stream, uint32_t *h_status);

/* Test hook for the decoder's failure detection, with no GPU fault: with
 * DFX_INJECT_SKIP_SLICE_COPY set, every later decode leaves out the copy of the
 * stream slice of its first group, so the warp that waits for it runs out its
 * bounded wait (about a second) and the plan's status word gets
 * DFX_STATUS_TIMEOUT (that group's output is then not valid).  No copy is left
 * in flight.  flags = 0 restores normal decoding.  Process-wide, not for
 * concurrent use; unknown flags return DFX_ERR_ARG. */
#define DFX_INJECT_SKIP_SLICE_COPY 0x1u
int dfx_debug_inject(uint32_t flags);

/* Release the plan and its device status word.  NULL is accepted. */
int dfx_free(dfx_plan_t plan);

/* dfx_encode for callers that cannot allocate device memory.  No page has a
 * counterpart: it exists for processes whose device memory belongs to another
 * allocator (a serving pool that reserves nearly all HBM up front) or that must
 * never risk the implicit synchronisation of cudaFree.  It needs no plan and no
 * workspace; its scratch is a fixed array in the library's device memory
 * (1 MiB + 4.25 KiB per GPU that loads the library, held until exit).
 *   d_bf16, n, params, d_out, out_capacity, h_compressed_bytes, stream: as in
 *   dfx_plan + dfx_encode (out_capacity >= the plan's max_compressed_bytes).
 * Limit: at most 262144 groups of 32 chunks (n <= 2^28 with K = 32, 2^29 with
 * K = 64, 2^30 with K = 128); larger n returns DFX_ERR_CAPACITY before any work.
 * Coder 0 only (coder 1 returns DFX_ERR_UNSUPPORTED).
 * All calls on a device share the scratch array and it keeps the last call's
 * contents; calls whose GPU work overlaps race and corrupt each other, so order
 * them on one stream.  Every call looks up the array's address in the current
 * context, so calls after a cudaDeviceReset or from another context on the same
 * device find the array that context holds; the first call in a context loads
 * the library's module there, so make it before any stream capture.  Produces
 * the same bytes as dfx_encode. */
int dfx_encode_static(const void *d_bf16, uint64_t n, const dfx_params *params, void *d_out,
                      size_t out_capacity, size_t *h_compressed_bytes, cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* DFX_H_ */
