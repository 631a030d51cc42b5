// decode.cu -- the DFX1 decode kernel for sm_100a with the canonical Huffman exponent coder
// (coder 0): compressed container -> BF16 in HBM.
//
// The memory pipeline and group loop are shared with the tANS coder (decode_pipeline.cuh);
// this file holds what is particular to the Huffman code (the pages' GPU decoder is prior
// art, "DFloat11: lossless LLM compression for GPU", aikraft.ru blog, section 03):
//   * one CTA per SM first builds its tables in shared memory from len[256]: a pair table
//     on the next 14 bits that resolves two codes at once when both fit, a one-code view
//     of it, and, for codes longer than 14 bits, the canonical per-length limits (the
//     levels of the hierarchical table of section 03, item 1);
//   * each lane keeps its bit position and a 32-bit peek of the stream; the peek is
//     reloaded from the warp's shared-memory copy of the group's stream slice once per
//     two pair lookups, so the common path has no per-code branch besides the rare
//     unresolved-pair test;
//   * each pair lookup is merged at once: one byte permute of the table entry with the m
//     word and one 32-bit rotate give two BF16 (the m bytes of a pair carry each other's
//     sign).
#include <cuda_runtime.h>
#include <stdint.h>

#include "decode_pipeline.cuh"
#include "huffman_reader.cuh"
#include "huffman_tables.cuh"

namespace dfx {
namespace {

struct HuffmanCoder {
    using Tables = HuffTables;
    template <class Words>
    using Reader = BitReader<Words>;
    static constexpr uint32_t kGbaseOffset = kOffGbase;
    static constexpr size_t kTableBytes = sizeof(uint32_t) << kLutBits;  // the pair table
    static constexpr size_t kScratchBytes = 0;
    // codes of at most 24 bits: a chunk spans at most 3K/4 words
    __host__ __device__ static constexpr uint32_t chunk_words(uint32_t K) { return (3u * K) / 4u; }
    __device__ static bool prepare(const DecodeArgs& a, Tables& T) { return build_canonical(a, T); }
    __device__ static void build(const Tables& T, uint32_t* table, uint8_t*) { build_pair_table(T, table); }
    template <class Words>
    __device__ static void init(Reader<Words>& br, const Tables&, const uint32_t* table, const Words& w, uint32_t start) {
        br.init(table, w, start);
    }
    template <class Words>
    __device__ static uint4 block(Reader<Words>& br, const Tables& T, uint2 m, uint32_t& err) {
        return decode_block(br, T, m, err);
    }
    template <class Words>
    __device__ static uint32_t one(Reader<Words>& br, const Tables& T, uint32_t& err) {
        return br.one(T, err);
    }
    // (an empty chunk consumes nothing, so it needs no separate rule)
    template <class Words>
    __device__ static bool done(const Reader<Words>& br, uint32_t clen, bool) {
        return br.consumed() == clen;
    }
};

static_assert(sizeof(WarpBuffers<128>::munit) >= 4 * (3 * 128 / 4 + 8) && sizeof(WarpBuffers<32>::munit) >= 4 * (3 * 32 / 4 + 8),
              "the m units after the slices cover the longest run past a slice");
static_assert(DecodeShape<32>::kThreads >= 256 && DecodeShape<64>::kThreads >= 256 && DecodeShape<128>::kThreads >= 256,
              "the table build gives each of the 256 symbols its own thread");
static_assert(dyn_smem_bytes<HuffmanCoder, 64>() + 1024 <= 227 * 1024 &&
                  dyn_smem_bytes<HuffmanCoder, 128>() + 1024 <= 227 * 1024,
              "shared memory");

}  // namespace

bool decode_supports(uint32_t K, uint32_t G) { return G == 32 && (K == 32 || K == 64 || K == 128); }

int decode_warps_per_block(uint32_t K) {
    return K == 32 ? DecodeShape<32>::kWarps : K == 64 ? DecodeShape<64>::kWarps : DecodeShape<128>::kWarps;
}

int decode_blocks_per_sm_huffman(uint32_t K) { return blocks_per_sm_coder<HuffmanCoder>(K); }

cudaError_t launch_decode_huffman(const DecodeArgs& a, int grid, cudaStream_t s) {
    return launch_coder<HuffmanCoder>(a, grid, s);
}

cudaError_t launch_decode_batch_huffman(const BatchArgs& b, uint32_t K, cudaStream_t s) {
    return launch_batch_coder<HuffmanCoder>(b, K, s);
}

int decode_blocks_per_sm(uint32_t K, uint32_t coder) {
    return is_tans(coder) ? decode_blocks_per_sm_tans(K, tans_states(coder)) : decode_blocks_per_sm_huffman(K);
}

cudaError_t launch_decode(const DecodeArgs& a, uint32_t coder, int grid, cudaStream_t s) {
    return is_tans(coder) ? launch_decode_tans(a, tans_states(coder), grid, s) : launch_decode_huffman(a, grid, s);
}

cudaError_t launch_decode_batch(const BatchArgs& b, uint32_t K, uint32_t coder, cudaStream_t s) {
    return is_tans(coder) ? launch_decode_batch_tans(b, K, tans_states(coder), s) : launch_decode_batch_huffman(b, K, s);
}

}  // namespace dfx
