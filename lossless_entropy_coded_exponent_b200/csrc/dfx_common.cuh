// dfx_common.cuh -- definitions shared by the libdfx CUDA sources (encode,
// decode, C ABI).  The container rules are stated in include/dfx.h.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "dfx.h"

namespace dfx {

constexpr uint32_t kHeaderBytes = 64;
constexpr uint32_t kOffLen = 64;        // coder 0: u8 len[256]
constexpr uint32_t kOffGbase = 320;     // coder 0: group start bits
constexpr uint32_t kOffFreq = 64;       // coder 1: u16 freq[256]
constexpr uint32_t kOffGbaseTans = 576; // coder 1: group start bits
constexpr uint32_t kMaxLenLimit = 24;   // longest code the decoder tables support
constexpr uint32_t kTansMinLog = 4, kTansMaxLog = 12;  // tANS table sizes 2^4 .. 2^12
constexpr uint32_t kWarp = 32;
constexpr unsigned kFull = 0xffffffffu;  // all lanes of a warp

// coders 1 and 2 are the tANS code with one or two states per chunk: same container layout
__host__ __device__ constexpr bool is_tans(uint32_t coder) { return coder == DFX_CODER_TANS || coder == DFX_CODER_TANS2; }
__host__ __device__ constexpr uint32_t tans_states(uint32_t coder) { return coder == DFX_CODER_TANS2 ? 2u : 1u; }
__host__ __device__ inline uint32_t gbase_offset(uint32_t coder) { return is_tans(coder) ? kOffGbaseTans : kOffGbase; }

__host__ __device__ constexpr uint64_t align16(uint64_t x) { return (x + 15u) & ~uint64_t(15); }

struct Layout {
    uint64_t n, n_chunk, n_group;
    uint64_t off_gbase, off_clen, off_m, off_stream;
    uint32_t K, G, coder;
};

__host__ __device__ inline Layout make_layout(uint64_t n, uint32_t K, uint32_t G, uint32_t coder = DFX_CODER_HUFFMAN) {
    Layout L;
    L.n = n;
    L.K = K;
    L.G = G;
    L.coder = coder;
    L.off_gbase = gbase_offset(coder);
    // a group holds G * K elements in 8-element blocks; block b belongs to chunk b mod G
    L.n_group = (n + (uint64_t)G * K - 1) / ((uint64_t)G * K);
    L.n_chunk = L.n_group * G;
    L.off_clen = align16(L.off_gbase + 8 * (L.n_group + 1));
    L.off_m = align16(L.off_clen + 2 * L.n_chunk);
    L.off_stream = align16(L.off_m + n);
    return L;
}

// Element of the first entry of block k of chunk `lane` in group g (G = 32 chunks).
__host__ __device__ inline uint64_t block_element(uint64_t g, uint32_t K, uint32_t k, uint32_t lane) {
    return g * 32ull * K + (32ull * k + lane) * 8;
}

__host__ __device__ inline uint64_t stream_bytes(uint64_t total_bits) {
    return align16(4 * ((total_bits + 31) / 32)) + 16;
}

// Every piece of state a decode launch needs, passed by value.
struct DecodeArgs {
    const uint8_t* comp;
    uint64_t comp_bytes;
    uint16_t* out;
    uint64_t n;
    uint32_t K, G;
    uint32_t n_chunk, n_group;
    uint64_t off_clen, off_m, off_stream;
    uint32_t* status;
    uint32_t g_begin, g_end;  // groups to decode (all: 0, n_group)
    uint64_t out_first;       // element index stored at out[0] (g_begin * G * K)
    uint32_t inject;          // test hook flags (dfx_debug_inject), normally 0
    uint32_t early;           // 1: read the container before the preceding kernel completes
};

struct EncodeArgs {
    const uint16_t* in;
    uint8_t* out;
    uint64_t n;
    uint32_t K, G, max_len;
    uint32_t coder, table_log;      // DFX_CODER_*; tANS table log (coder 1)
    uint32_t n_chunk, n_group;
    uint64_t off_gbase, off_clen, off_m, off_stream;
    unsigned long long* ws_counts;  // [256]
    uint32_t* ws_code;              // [256]
    uint8_t* ws_len;                // [256]
    uint32_t* ws_group_bits;        // coder 0: [n_group] u64 look-back words; tANS: [n_group] u32 group sums
    unsigned long long* ws_edge;    // coder 0: [n_group + 1] arrivals and bits at each group boundary
    uint32_t* ws_tans;              // coder 1: [kWsTansWords] encode tables
    uint32_t* status;
    uint64_t max_bytes;             // the container's capacity (tANS: zeroed past the m plane)
};

// Several tensors decoded by one launch: tensor i gets CTAs [cta_begin[i], cta_begin[i+1]).
constexpr uint32_t kMaxBatch = 32;
struct BatchArgs {
    uint32_t count;
    uint32_t cta_begin[kMaxBatch + 1];
    DecodeArgs t[kMaxBatch];
};

// Workspace layout for encode.
constexpr uint64_t kWsCounts = 0;
constexpr uint64_t kWsCode = 2048;
constexpr uint64_t kWsLen = 3072;
constexpr uint64_t kWsTicket = 3328;     // coder 0: the pack's CTA ticket counter
constexpr uint64_t kWsTotalBits = 3336;  // coder 0: the stream's bit count, from the code book
constexpr uint64_t kWsGroupBits = 4096;
// coder 0: per group boundary b = 0 .. n_group (the start of group b), the bits that groups
// b - 1 and b put in the stream word the boundary falls in (low half) and how many of the
// two have done so (high half)
__host__ __device__ constexpr uint64_t ws_edge_offset(uint64_t n_group) { return align16(kWsGroupBits + 8 * n_group); }
// coder 1: per symbol (threshold << 16 | nb_hi, cs << 16 | f) and the slot of every
// (symbol, state number) pair, after the group sums
constexpr uint64_t kWsTansWords = 2 * 256 + (1u << kTansMaxLog);
inline uint64_t ws_tans_offset(uint64_t n_group) { return (kWsGroupBits + 4 * n_group + 255) & ~uint64_t(255); }
inline uint64_t workspace_bytes_for(uint64_t n_group, uint32_t coder = DFX_CODER_HUFFMAN) {
    return is_tans(coder) ? ws_tans_offset(n_group) + 4 * kWsTansWords
                                   : ws_edge_offset(n_group) + 8 * (n_group + 1);
}

// Launchers (encode.cu, encode_tans.cu / decode.cu, decode_tans.cu); `coder` selects the
// exponent coder's kernels.
cudaError_t launch_encode(const EncodeArgs& a, uint64_t max_bytes, cudaStream_t s);
cudaError_t launch_encode_tans(const EncodeArgs& a, int phase, cudaStream_t s);  // 0: before the group scan, 1: after
cudaError_t launch_decode(const DecodeArgs& a, uint32_t coder, int grid, cudaStream_t s);
cudaError_t launch_decode_batch(const BatchArgs& b, uint32_t K, uint32_t coder, cudaStream_t s);
int decode_blocks_per_sm(uint32_t K, uint32_t coder);
int decode_warps_per_block(uint32_t K);
bool decode_supports(uint32_t K, uint32_t G);
cudaError_t launch_decode_huffman(const DecodeArgs& a, int grid, cudaStream_t s);
cudaError_t launch_decode_batch_huffman(const BatchArgs& b, uint32_t K, cudaStream_t s);
int decode_blocks_per_sm_huffman(uint32_t K);
cudaError_t launch_decode_tans(const DecodeArgs& a, uint32_t states, int grid, cudaStream_t s);
cudaError_t launch_decode_batch_tans(const BatchArgs& b, uint32_t K, uint32_t states, cudaStream_t s);
int decode_blocks_per_sm_tans(uint32_t K, uint32_t states);
// Y = X W^T from W's container (decode_gemm.cu): at most kGemmMaxTokens tokens, at most
// kGemmMaxRows rows of W per CTA
constexpr uint32_t kGemmMaxTokens = 32;
constexpr uint32_t kGemmMaxRows = 100;
cudaError_t launch_decode_gemm(const DecodeArgs& d, const uint16_t* x, float* y, uint16_t* w_out, uint32_t rows,
                               uint32_t cols, uint32_t tokens, int grid, cudaStream_t s);

}  // namespace dfx
