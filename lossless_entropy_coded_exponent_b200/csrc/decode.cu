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

namespace dfx {
namespace {

constexpr int kLutBits = 14;

// Pair table entry (u32), indexed by the next kLutBits stream bits:
//   bits 0-7   first symbol        bits 8-15  second symbol
//   bits 16-20 length of the first code (0: the first code is longer than kLutBits)
//   bits 26-30 bits the fast path consumes: both codes' lengths when both fit in the
//              index bits, else the first code's length (0 for a long first code)
//   bit  31    set when the entry does not hold two complete codes
constexpr uint32_t kNotPair = 0x80000000u;

struct HuffTables {
    uint32_t limit[kMaxLenLimit + 1];         // left-justified 24-bit end of the codes of length l
    uint32_t first[kMaxLenLimit + 1];         // first canonical code of length l
    uint32_t index[kMaxLenLimit + 1];         // rank in `sorted` of the first symbol of length l
    uint8_t sorted[256];                      // used symbols in (length, symbol) order
    uint8_t slen[256];                        // their code lengths
    uint8_t lens[256];
    uint8_t wcount[8][kMaxLenLimit + 1];      // symbols of each length among 32-symbol slices
    unsigned long long total_bits;
    uint32_t n_words;                         // 32-bit words of the stream section
    uint32_t bad;
};

// Checks the header and builds the per-length canonical tables in T.  The header, the
// group index ends and len[256] are read in one round of loads (the host has checked that
// the buffer holds at least the index and the m plane).  Every thread of the block calls
// it; false means the container was rejected and its status bits are set.
__device__ bool build_canonical(const DecodeArgs& a, HuffTables& T) {
    const int t = threadIdx.x;
    const unsigned warp = t >> 5, lane = t & 31;
    if (t < 8 * (int)(kMaxLenLimit + 1)) (&T.wcount[0][0])[t] = 0;
    if (t == 0) T.bad = 0;
    __syncthreads();
    uint32_t l_t = 0, within = 0;
    if (t < 256) l_t = a.comp[kOffLen + t];
    if (t == 0) {
        const uint8_t* h = a.comp;
        const unsigned long long* gbase = reinterpret_cast<const unsigned long long*>(h + kOffGbase);
        const unsigned long long gb_first = gbase[0], gb_last = gbase[a.n_group];
        uint32_t bad = 0;
        const unsigned long long n = *reinterpret_cast<const unsigned long long*>(h + 8);
        const unsigned long long total_bits = *reinterpret_cast<const unsigned long long*>(h + 16);
        const unsigned long long total_bytes = *reinterpret_cast<const unsigned long long*>(h + 24);
        const uint32_t max_len = *reinterpret_cast<const uint32_t*>(h + 56);
        if (*reinterpret_cast<const uint32_t*>(h) != 0x31584644u) bad = DFX_STATUS_HEADER;
        if (*reinterpret_cast<const uint16_t*>(h + 4) != 1 || *reinterpret_cast<const uint16_t*>(h + 6) != kHeaderBytes)
            bad = DFX_STATUS_HEADER;
        if (n != a.n || *reinterpret_cast<const uint32_t*>(h + 32) != a.K || *reinterpret_cast<const uint32_t*>(h + 36) != a.G ||
            *reinterpret_cast<const uint32_t*>(h + 40) != a.n_chunk || *reinterpret_cast<const uint32_t*>(h + 44) != a.n_group ||
            *reinterpret_cast<const unsigned long long*>(h + 48) != a.off_m || *reinterpret_cast<const uint32_t*>(h + 60) != 0)
            bad = DFX_STATUS_HEADER;
        if (max_len < 1 || max_len > kMaxLenLimit || total_bits > (unsigned long long)max_len * a.n) bad = DFX_STATUS_HEADER;
        if (total_bytes != a.off_stream + stream_bytes(total_bits) || total_bytes > a.comp_bytes) bad = DFX_STATUS_HEADER;
        // the group index must start at bit 0 and end at total_bits
        if (!bad && (gb_first != 0 || gb_last != total_bits)) bad = DFX_STATUS_INDEX;
        T.total_bits = total_bits;
        T.n_words = bad ? 0u : (uint32_t)((total_bytes - a.off_stream) / 4);
        if (bad) atomicOr(&T.bad, bad);
    }
    // rank of each used symbol among the symbols of its length (warps 0-7 hold symbols
    // 0-255, one per lane): lower lanes of the same warp now, the counts of lower warps
    // once every warp has written them
    if (t < 256) {
        T.lens[t] = (uint8_t)l_t;
        if (l_t > kMaxLenLimit) atomicOr(&T.bad, DFX_STATUS_TABLE);
        const unsigned peers = __match_any_sync(kFull, l_t);
        const unsigned below = peers & ((1u << lane) - 1u);
        within = __popc(below);
        if (l_t && l_t <= kMaxLenLimit && below == 0) T.wcount[warp][l_t] = (uint8_t)__popc(peers);
    }
    __syncthreads();
    if (T.bad) {
        if (t == 0) atomicOr(a.status, T.bad);
        return false;
    }
    if (warp == 0) {
        // canonical tables by a warp scan over the lengths (lane l holds length l):
        // F = sum over shorter lengths j of nlen[j] << (24 - j) is the left-justified
        // first code of length l; the Kraft sum is F past the longest length
        uint32_t nl = 0;
        if (lane >= 1 && lane <= kMaxLenLimit)
            for (int w = 0; w < 8; w++) nl += T.wcount[w][lane];
        const uint32_t weight = (lane >= 1 && lane <= kMaxLenLimit) ? nl << (kMaxLenLimit - lane) : 0u;
        uint32_t f = weight, c = nl;  // inclusive scans
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const uint32_t fy = __shfl_up_sync(kFull, f, d), cy = __shfl_up_sync(kFull, c, d);
            if (lane >= (unsigned)d) {
                f += fy;
                c += cy;
            }
        }
        const uint32_t kraft = __shfl_sync(kFull, f, 31);
        if (lane >= 1 && lane <= kMaxLenLimit) {
            T.first[lane] = (f - weight) >> (kMaxLenLimit - lane);
            T.index[lane] = c - nl;
            T.limit[lane] = f;
        }
        if (lane == 0 && (a.n > 0 ? kraft != (1u << kMaxLenLimit) : kraft != 0)) T.bad = DFX_STATUS_TABLE;
    }
    __syncthreads();
    if (T.bad) {
        if (t == 0) atomicOr(a.status, T.bad);
        return false;
    }
    if (t < 256 && l_t) {
        uint32_t r = within;
        for (unsigned w = 0; w < warp; w++) r += T.wcount[w][l_t];
        T.sorted[T.index[l_t] + r] = (uint8_t)t;
        T.slen[T.index[l_t] + r] = (uint8_t)l_t;
    }
    __syncthreads();
    return true;
}

// Fill `cnt` entries from `p` with v (cnt a power of two and p aligned to it), the warp's
// lanes sharing the stores.
__device__ __forceinline__ void fill_run(uint32_t* p, uint32_t cnt, uint32_t v, unsigned lane) {
    if (cnt >= 4) {
        uint4* q = reinterpret_cast<uint4*>(p);
        for (uint32_t j = lane; j < cnt / 4; j += 32) q[j] = make_uint4(v, v, v, v);
    } else if (lane < cnt) {
        p[lane] = v;
    }
}

// The pair table `lut` (1 << kLutBits entries) from the canonical tables.  The entries
// whose index bits start with the code c0 of a first symbol s0 of length l0 <= kLutBits
// are [c0, c0 + 1) << (kLutBits - l0); one warp per first symbol marks that run "first
// code only" and then overwrites, for every second symbol whose code c1 fits the
// remaining r = kLutBits - l0 bits, the sub-run that continues with c1.  Entries no short
// code starts keep the "long first code" mark.  Every thread of the block calls it.
__device__ void build_pair_table(const HuffTables& T, uint32_t* lut) {
    const int t = threadIdx.x;
    const unsigned warp = t >> 5, lane = t & 31;
    for (int i = t; i < (1 << kLutBits) / 4; i += blockDim.x)
        reinterpret_cast<uint4*>(lut)[i] = make_uint4(kNotPair, kNotPair, kNotPair, kNotPair);
    __syncthreads();
    const uint32_t n_short = T.index[kLutBits + 1];  // symbols with codes of at most kLutBits bits
    for (uint32_t i0 = warp; i0 < n_short; i0 += blockDim.x >> 5) {
        const uint32_t l0 = T.slen[i0], s0 = T.sorted[i0];
        const uint32_t r = kLutBits - l0;
        const uint32_t lo = (T.first[l0] + i0 - T.index[l0]) << r;
        fill_run(lut + lo, 1u << r, kNotPair | s0 | (l0 << 16) | (l0 << 26), lane);
        __syncwarp();
        const uint32_t n1 = T.index[r + 1];  // second symbols with codes of at most r bits
        for (uint32_t i1 = 0; i1 < n1; i1++) {
            const uint32_t l1 = T.slen[i1];
            const uint32_t sh = r - l1;
            fill_run(lut + lo + ((T.first[l1] + i1 - T.index[l1]) << sh), 1u << sh,
                     s0 | ((uint32_t)T.sorted[i1] << 8) | (l0 << 16) | ((l0 + l1) << 26), lane);
        }
    }
    __syncthreads();
}


// A code longer than kLutBits: find its length from the canonical limits.  Returns
// (len << 8) | symbol; bit 16 flags a bit pattern that is no code (Kraft-complete
// tables make that impossible for a well-formed stream).
__device__ __noinline__ uint32_t decode_long(uint32_t peek, const HuffTables& T) {
    const uint32_t v = peek >> (32 - kMaxLenLimit);
    int l = kLutBits + 1;
    while (l <= (int)kMaxLenLimit && v >= T.limit[l]) l++;
    if (l > (int)kMaxLenLimit) return (1u << 16) | (kMaxLenLimit << 8);
    return ((uint32_t)l << 8) | T.sorted[T.index[l] + (v >> (kMaxLenLimit - l)) - T.first[l]];
}


// ---------------------------------------------------------------- bit reader
//
// A lane's state is its bit position p, relative to the first word of its word source,
// `peek`, the 32 stream bits starting at p, and the two words cur, nxt that hold them
// (word cw and cw + 1).  Once per round of two pairs, peek is rebuilt from cur and nxt
// with one funnel shift; only when p has moved into the next word does the lane shift
// its words along and load one new word.  No reload follows more than 32 consumed bits
// (two table pairs take at most 28, a single code at most 24), so p moves at most one
// word between reloads, and about one lane in three loads a word per round.  Every
// pair the table resolves consumes at most kLutBits = 14 bits, so after the first pair
// of a round at least 18 valid bits remain for the second.  Pairs the table cannot
// resolve (the second code does not fit the index bits, or the first code is longer)
// take a rare branch: it reloads after the first code and, when both codes are at most
// kLutBits long, reads the second from the table entry at the new position; otherwise
// it decodes code by code with the canonical limits.
//
// Word sources: the global stream (with or without a bound clamp) or a warp's
template <class Words>
struct BitReader {
    const uint32_t* lut;  // pair table in shared memory
    Words words;
    uint32_t p, p0, peek;
    uint32_t cw, cur, nxt;  // cur = word cw, nxt = word cw + 1

    __device__ __forceinline__ void init(const uint32_t* table, const Words& w, uint32_t start) {
        lut = table;
        words = w;
        p = p0 = start;
        cw = start >> 5;
        cur = words.load(cw);
        nxt = words.load(cw + 1);
    }
    __device__ __forceinline__ void reload() {
        const uint32_t wi = p >> 5;
        if (wi != cw) {  // wi == cw + 1
            cw = wi;
            cur = nxt;
            nxt = words.load(wi + 1);
        }
        peek = __funnelshift_l(nxt, cur, p);  // shift uses p & 31
    }
    // One code, the general way (peek must be current): returns its symbol.
    __device__ __forceinline__ uint32_t one(const HuffTables& T, uint32_t& err) {
        const uint32_t e = lut[peek >> (32 - kLutBits)];
        uint32_t len, sym;
        if ((e & 0x001F0000u) == 0) {
            uint32_t ent = decode_long(peek, T);
            if (ent >> 16) {
                err |= DFX_STATUS_STREAM;
                ent &= 0xFFFFu;
            }
            len = ent >> 8;
            sym = ent & 0xFFu;
        } else {
            len = (e >> 16) & 31u;
            sym = e & 0xFFu;
        }
        p += len;
        reload();
        return sym;
    }
    // Two codes, merged with their m bytes (bytes 2j and 2j+1 of mw): two BF16.
    template <int j>
    __device__ __forceinline__ uint32_t pair(uint32_t mw, const HuffTables& T, uint32_t& err) {
        constexpr uint32_t sel = j == 0 ? 0x5140u : 0x5342u;  // [mw.2j, sym0, mw.2j+1, sym1]
        const uint32_t e = lut[peek >> (32 - kLutBits)];
        const uint32_t len = e >> 26;           // bit 5 is set when the entry is not a pair
        peek = __funnelshift_l(0u, peek, len);  // shifts by len & 31
        p += len;
        uint32_t syms = e;
        if ((int32_t)e < 0) {
            p -= 32;  // undo bit 5 of `len`
            reload();
            // usually both codes fit the table on their own: the second one is the first
            // code of the entry at the new position, and peek keeps at least 18 valid bits
            const uint32_t e2 = lut[peek >> (32 - kLutBits)];
            if ((e & 0x001F0000u) && (e2 & 0x001F0000u)) {
                const uint32_t l1 = (e2 >> 16) & 31u;
                p += l1;
                peek = __funnelshift_l(0u, peek, l1);
                syms = (e & 0xFFu) | ((e2 & 0xFFu) << 8);
            } else {
                uint32_t s0 = e & 0xFFu;
                if ((e & 0x001F0000u) == 0) s0 = one(T, err);
                syms = s0 | (one(T, err) << 8);
            }
        }
        return bf16_pair(__byte_perm(mw, syms, sel));
    }
    __device__ __forceinline__ uint32_t consumed() const { return p - p0; }
};

// Decode the 8 codes of one block and merge them with the block's m bytes: 8 BF16.
template <class Words>
__device__ __forceinline__ uint4 decode_block(BitReader<Words>& br, const HuffTables& T, uint2 m, uint32_t& err) {
    uint4 o;
    br.reload();
    o.x = br.template pair<0>(m.x, T, err);
    o.y = br.template pair<1>(m.x, T, err);
    br.reload();
    o.z = br.template pair<0>(m.y, T, err);
    o.w = br.template pair<1>(m.y, T, err);
    return o;
}

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
    return coder == DFX_CODER_TANS ? decode_blocks_per_sm_tans(K) : decode_blocks_per_sm_huffman(K);
}

cudaError_t launch_decode(const DecodeArgs& a, uint32_t coder, int grid, cudaStream_t s) {
    return coder == DFX_CODER_TANS ? launch_decode_tans(a, grid, s) : launch_decode_huffman(a, grid, s);
}

cudaError_t launch_decode_batch(const BatchArgs& b, uint32_t K, uint32_t coder, cudaStream_t s) {
    return coder == DFX_CODER_TANS ? launch_decode_batch_tans(b, K, s) : launch_decode_batch_huffman(b, K, s);
}

}  // namespace dfx
