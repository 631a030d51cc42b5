// decode_tans.cu -- the DFX1 decode kernels for sm_100a with the tANS exponent coder,
// one state per chunk (coder 1) or two interleaved states (coder 2): compressed container
// -> BF16 in HBM.
//
// The memory pipeline and group loop are those of the Huffman decoder
// (decode_pipeline.cuh); this file holds what is particular to tabled asymmetric numeral
// systems (J. Duda, "Asymmetric numeral systems", 2013; one page names ANS as the
// coder of its compressed number formats: "From a Lossless (~1.5:1) Compression
// Algorithm for Llama2 7B Weights to Variable Precision, Variable Range, Compressed
// Numeric Data Types for CNNs and LLMs", abstract):
//   * one CTA per SM builds the decoding table from freq[256] (tans_tables.cuh: the
//     stride spread of the symbols over the M = 2^R slots, then every slot's state
//     number k = f[s] + the slots of s below it);
//   * a table entry is nb | symbol << 8 | (4 * base) << 16 with nb = R - floor(log2 k)
//     and base = k 2^nb - M: a decoding step is one shared load, two funnel shifts (the
//     next nb bits of the peek, and the peek moved past them; both take the shift
//     amount from the entry's low 5 bits) and one add, with no per-symbol branch;
//   * a lane's state is kept as 4 x (its table index), the byte offset of its next
//     entry; its first R bits are the chunk's start state and the chunk ends in state 0;
//     with two states (coder 2) the chunk starts with state A's R bits, then B's, A
//     decodes the even positions and B the odd ones, so the two table loads of a symbol
//     pair do not wait on each other and only the field extraction stays in order;
//   * two symbols per peek reload (a field is at most R <= 12 bits), merged with their m
//     bytes by two byte permutes and one rotate into two BF16.
#include <cuda_runtime.h>
#include <stdint.h>

#include "decode_pipeline.cuh"
#include "tans_tables.cuh"

namespace dfx {
namespace {

struct TansTables {
    unsigned long long total_bits;
    uint32_t n_words;      // 32-bit words of the stream section
    uint32_t R;            // table log
    uint32_t bad;
    uint32_t wsum[8];      // scan of the frequencies, one sum per warp
    uint32_t f[256];       // frequencies
    uint32_t cs[256];      // their exclusive prefix sums
};


// Checks the header (coder 1 or 2, as `states` says) and loads the frequency table and
// its prefix sums into T.  Every thread of the block calls it; false means the container
// was rejected and its status bits are set.
template <uint32_t States>
__device__ bool tans_prepare(const DecodeArgs& a, TansTables& T) {
    const int t = threadIdx.x;
    const unsigned warp = t >> 5, lane = t & 31;
    if (t == 0) T.bad = 0;
    __syncthreads();
    uint32_t f = 0, incl = 0;
    if (t < 256) f = reinterpret_cast<const uint16_t*>(a.comp + kOffFreq)[t];
    if (t == 0) {
        const uint8_t* h = a.comp;
        const unsigned long long* gbase = reinterpret_cast<const unsigned long long*>(h + kOffGbaseTans);
        const unsigned long long gb_first = gbase[0], gb_last = gbase[a.n_group];
        uint32_t bad = 0;
        const unsigned long long n = *reinterpret_cast<const unsigned long long*>(h + 8);
        const unsigned long long total_bits = *reinterpret_cast<const unsigned long long*>(h + 16);
        const unsigned long long total_bytes = *reinterpret_cast<const unsigned long long*>(h + 24);
        const uint32_t R = *reinterpret_cast<const uint32_t*>(h + 56);
        if (*reinterpret_cast<const uint32_t*>(h) != 0x31584644u) bad = DFX_STATUS_HEADER;
        if (*reinterpret_cast<const uint16_t*>(h + 4) != 1 || *reinterpret_cast<const uint16_t*>(h + 6) != kHeaderBytes)
            bad = DFX_STATUS_HEADER;
        if (n != a.n || *reinterpret_cast<const uint32_t*>(h + 32) != a.K || *reinterpret_cast<const uint32_t*>(h + 36) != a.G ||
            *reinterpret_cast<const uint32_t*>(h + 40) != a.n_chunk || *reinterpret_cast<const uint32_t*>(h + 44) != a.n_group ||
            *reinterpret_cast<const unsigned long long*>(h + 48) != a.off_m ||
            *reinterpret_cast<const uint32_t*>(h + 60) != (States == 2 ? DFX_CODER_TANS2 : DFX_CODER_TANS))
            bad = DFX_STATUS_HEADER;
        if (R < kTansMinLog || R > kTansMaxLog || total_bits > (unsigned long long)R * (a.n + States * a.n_chunk))
            bad = DFX_STATUS_HEADER;
        if (total_bytes != a.off_stream + stream_bytes(total_bits) || total_bytes > a.comp_bytes) bad = DFX_STATUS_HEADER;
        // the group index must start at bit 0 and end at total_bits
        if (!bad && (gb_first != 0 || gb_last != total_bits)) bad = DFX_STATUS_INDEX;
        T.total_bits = total_bits;
        T.R = bad ? kTansMinLog : R;
        T.n_words = bad ? 0u : (uint32_t)((total_bytes - a.off_stream) / 4);
        if (bad) atomicOr(&T.bad, bad);
    }
    // exclusive prefix sums of the frequencies (warps 0-7 hold symbols 0-255)
    if (t < 256) {
        incl = f;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const uint32_t y = __shfl_up_sync(kFull, incl, d);
            if (lane >= (unsigned)d) incl += y;
        }
        if (lane == 31) T.wsum[warp] = incl;
    }
    __syncthreads();
    if (t < 256) {
        uint32_t base = 0;
        for (unsigned w = 0; w < warp; w++) base += T.wsum[w];
        T.f[t] = f;
        T.cs[t] = base + incl - f;
        if (t == 255 && !T.bad && base + incl != (a.n > 0 ? (1u << T.R) : 0u)) atomicOr(&T.bad, DFX_STATUS_TABLE);
    }
    __syncthreads();
    if (T.bad) {
        if (t == 0) atomicOr(a.status, T.bad);
        return false;
    }
    return true;
}

// The decoding table (2^R entries) from the frequencies.  Every thread of the block calls
// it.  A tensor with n = 0 has no used symbol and no state to decode; the table is then
// left unwritten.
__device__ void tans_build(const TansTables& T, uint32_t* table, uint8_t* scratch) {
    const uint32_t R = T.R, M = 1u << R;
    if (T.cs[255] + T.f[255] != M) return;  // n = 0 (prepare checked the sum otherwise)
    tans_number_states(T.f, T.cs, R, scratch, [&](uint32_t j, uint32_t s, uint32_t k) {
        const uint32_t nb = R - (31u - __clz(k));
        const uint32_t base = (k << nb) - M;
        table[j] = nb | (s << 8) | ((4u * base) << 16);
    });
}

// ---------------------------------------------------------------- reader
//
// The bit position p, the 32-bit peek and the two cached words are kept as in the
// Huffman reader; reloads come once per two symbols (at most 2R <= 24 bits), so p moves
// at most one word between them.
template <class Words, uint32_t States>
struct TansReader {
    const uint8_t* tbl;  // decoding table (shared memory)
    Words words;
    uint32_t p, p0, peek;
    uint32_t cw, cur, nxt;  // cur = word cw, nxt = word cw + 1
    uint32_t x4[States];    // the states times 4: byte offsets of their table entries
    uint32_t next;          // the state of the next single symbol (the tail's one())

    __device__ __forceinline__ void reload() {
        const uint32_t wi = p >> 5;
        if (wi != cw) {  // wi == cw + 1
            cw = wi;
            cur = nxt;
            nxt = words.load(wi + 1);
        }
        peek = __funnelshift_l(nxt, cur, p);  // shift uses p & 31
    }
    __device__ __forceinline__ void init(const uint32_t* table, uint32_t R, const Words& w, uint32_t start) {
        tbl = reinterpret_cast<const uint8_t*>(table);
        words = w;
        p = p0 = start;
        cw = start >> 5;
        cur = words.load(cw);
        nxt = words.load(cw + 1);
        reload();
        // the chunk's first R bits per state: the start states (2R <= 24 bits of the peek)
#pragma unroll
        for (uint32_t s = 0; s < States; s++) x4[s] = ((peek << (s * R)) >> (32 - R)) << 2;
        p += States * R;
        next = 0;
    }
    // One decoding step of state x: its entry; the state becomes base + the next nb bits.
    // The caller advances p.
    __device__ __forceinline__ uint32_t step(uint32_t& x) {
        const uint32_t e = *reinterpret_cast<const uint32_t*>(tbl + x);
        const uint32_t v = __funnelshift_l(peek, 0u, e);  // peek >> (32 - nb); 0 when nb = 0
        peek = __funnelshift_l(0u, peek, e);               // peek << nb
        x = (e >> 16) + (v << 2);
        return e;
    }
    // Two symbols (peek current), merged with their m bytes (bytes 2j and 2j+1 of mw).
    // With two states the pair's first symbol is A's and its second B's.
    template <int j>
    __device__ __forceinline__ uint32_t pair(uint32_t mw) {
        constexpr uint32_t sel = j == 0 ? 0x5140u : 0x5342u;  // [mw.2j, sym0, mw.2j+1, sym1]
        const uint32_t e0 = step(x4[0]);
        const uint32_t e1 = step(x4[States - 1]);
        p += (e0 + e1) & 63u;  // nb0 + nb1 (each below 32, in the entries' low bits)
        return bf16_pair(__byte_perm(mw, __byte_perm(e0, e1, 0x0051u), sel));
    }
    // One symbol (peek current); reloads after it.
    __device__ __forceinline__ uint32_t one() {
        uint32_t e;
        if (States == 2 && next) e = step(x4[States - 1]);
        else e = step(x4[0]);
        next ^= States - 1;
        p += e & 31u;
        reload();
        return (e >> 8) & 0xFFu;
    }
    __device__ __forceinline__ bool done(uint32_t clen) const {
        bool zero = true;
#pragma unroll
        for (uint32_t s = 0; s < States; s++) zero = zero && x4[s] == 0;
        return p - p0 == clen && zero;
    }
};

template <uint32_t States>
struct TansCoder {
    using Tables = TansTables;
    template <class Words>
    using Reader = TansReader<Words, States>;
    static constexpr uint32_t kGbaseOffset = kOffGbaseTans;
    static constexpr size_t kTableBytes = 4u * kTansSlotsMax;
    static constexpr size_t kScratchBytes = (kTansScratchBytes + 15) & ~size_t(15);
    // fields of at most 12 bits and 12-bit states: a chunk spans at most 3K/8 + 2 words
    // (3K/8 + 3 with two states)
    __host__ __device__ static constexpr uint32_t chunk_words(uint32_t K) { return (3u * K) / 8u + 1u + States; }
    __device__ static bool prepare(const DecodeArgs& a, Tables& T) { return tans_prepare<States>(a, T); }
    __device__ static void build(const Tables& T, uint32_t* table, uint8_t* scratch) { tans_build(T, table, scratch); }
    template <class Words>
    __device__ static void init(Reader<Words>& br, const Tables& T, const uint32_t* table, const Words& w, uint32_t start) {
        br.init(table, T.R, w, start);
    }
    template <class Words>
    __device__ static uint4 block(Reader<Words>& br, const Tables&, uint2 m, uint32_t&) {
        uint4 o;
        br.reload();
        o.x = br.template pair<0>(m.x);
        br.reload();
        o.y = br.template pair<1>(m.x);
        br.reload();
        o.z = br.template pair<0>(m.y);
        br.reload();
        o.w = br.template pair<1>(m.y);
        return o;
    }
    template <class Words>
    __device__ static uint32_t one(Reader<Words>& br, const Tables&, uint32_t&) {
        return br.one();
    }
    // An empty chunk has no bits (its reader's start-state read looked past it); a chunk
    // with elements ends in state 0 after exactly its bits.
    template <class Words>
    __device__ static bool done(const Reader<Words>& br, uint32_t clen, bool has_elements) {
        return has_elements ? br.done(clen) : clen == 0;
    }
};

static_assert(dyn_smem_bytes<TansCoder<2>, 64>() + sizeof(TansTables) + 1024 <= 227 * 1024 &&
                  dyn_smem_bytes<TansCoder<2>, 128>() + sizeof(TansTables) + 1024 <= 227 * 1024,
              "shared memory");
static_assert(DecodeShape<128>::kThreads == 1024 && DecodeShape<128>::kWarps <= 32,
              "the state-number rounds hold one slot per thread and one count per warp");

}  // namespace

int decode_blocks_per_sm_tans(uint32_t K, uint32_t states) {
    return states == 2 ? blocks_per_sm_coder<TansCoder<2>>(K) : blocks_per_sm_coder<TansCoder<1>>(K);
}

cudaError_t launch_decode_tans(const DecodeArgs& a, uint32_t states, int grid, cudaStream_t s) {
    return states == 2 ? launch_coder<TansCoder<2>>(a, grid, s) : launch_coder<TansCoder<1>>(a, grid, s);
}

cudaError_t launch_decode_batch_tans(const BatchArgs& b, uint32_t K, uint32_t states, cudaStream_t s) {
    return states == 2 ? launch_batch_coder<TansCoder<2>>(b, K, s) : launch_batch_coder<TansCoder<1>>(b, K, s);
}

}  // namespace dfx
