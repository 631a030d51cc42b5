// decode.cu -- the DFX1 decode kernel for sm_100a: compressed container -> BF16 in HBM.
//
// Design (B200-first; the pages' GPU decoder is prior art, "DFloat11: lossless LLM
// compression for GPU", aikraft.ru blog, section 03):
//   * persistent grid, 8 warps per CTA; each CTA first builds its decoding tables in
//     shared memory from len[256]: a direct lookup table on the next 11 bits for every
//     code of length <= 11 and, for longer codes, the canonical per-length limits (the
//     two levels of the hierarchical table of section 03, item 1);
//   * one warp decodes one group of 32 chunks; lane i owns chunk i of the group and
//     decodes exactly K codes.  Its read position is the group's start bit plus the
//     warp's exclusive scan of the chunk bit lengths (the "lightweight auxiliary
//     variables" that coordinate read positions, section 03, item 2).  Output positions
//     need no scan: chunk i writes elements [i*K, i*K + K) of the group;
//   * decoded exponents go to a per-warp shared-memory stash laid out so that both the
//     lane-per-chunk writes and the coalesced reads of the merge step are free of bank
//     conflicts; the merge joins them with the sign+mantissa bytes (8-byte loads, issued
//     before decoding starts so they are in flight while the warp decodes) and writes
//     BF16 with 16-byte stores, 512 contiguous bytes per warp instruction.
// Every read of the container is bounded by the header-checked section sizes; a bad
// container sets bits of the status word and the kernel finishes normally.
#include <cuda_runtime.h>
#include <stdint.h>

#include "dfx_common.cuh"

namespace dfx {
namespace {

constexpr int kLutBits = 11;
constexpr int kDecodeWarps = 8;
constexpr int kDecodeThreads = kDecodeWarps * 32;
constexpr unsigned kFull = 0xffffffffu;

// Stash row stride (words): row q holds symbols 4q..4q+3 of every lane.  32 + 128/K
// makes the merge step's reads (lane l reads rows 2a, 2a+1 of lane l/(K/8) ...) hit
// 32 distinct banks for K = 32, 64, 128.
template <int K>
struct StashShape {
    static constexpr int kStride = 32 + 128 / K;
    static constexpr int kWords = (K / 4) * kStride;
};

struct Tables {
    uint16_t lut[1 << kLutBits];              // (len << 8) | symbol, or 0 for codes longer than kLutBits
    uint32_t limit[kMaxLenLimit + 1];         // left-justified 24-bit end of the codes of length l
    uint32_t first[kMaxLenLimit + 1];         // first canonical code of length l
    uint32_t index[kMaxLenLimit + 1];         // rank in `sorted` of the first symbol of length l
    uint32_t nlen[kMaxLenLimit + 1];
    uint8_t sorted[256];                      // used symbols in (length, symbol) order
    uint8_t lens[256];
    unsigned long long total_bits;
    uint32_t n_words;                         // 32-bit words of the stream section
    uint32_t bad;
};

__device__ bool build_tables(const DecodeArgs& a, Tables& T) {
    const int t = threadIdx.x;
    if (t == 0) {
        const uint8_t* h = a.comp;
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
        if (!bad) {
            // the group index must start at bit 0 and end at total_bits
            const unsigned long long* gbase = reinterpret_cast<const unsigned long long*>(h + kOffGbase);
            if (gbase[0] != 0 || gbase[a.n_group] != total_bits) bad = DFX_STATUS_INDEX;
        }
        T.total_bits = total_bits;
        T.n_words = bad ? 0u : (uint32_t)((total_bytes - a.off_stream) / 4);
        T.bad = bad;
    }
    if (t <= (int)kMaxLenLimit) T.nlen[t] = 0;
    __syncthreads();
    if (T.bad) {
        if (t == 0) atomicOr(a.status, T.bad);
        return false;
    }
    for (int s = t; s < 256; s += blockDim.x) {
        const uint32_t l = a.comp[kOffLen + s];
        T.lens[s] = (uint8_t)l;
        if (l > kMaxLenLimit) atomicOr(&T.bad, DFX_STATUS_TABLE);
        else if (l) atomicAdd(&T.nlen[l], 1u);
    }
    __syncthreads();
    if (t == 0 && !T.bad) {
        unsigned long long kraft = 0;
        for (int l = 1; l <= (int)kMaxLenLimit; l++) kraft += (unsigned long long)T.nlen[l] << (kMaxLenLimit - l);
        if (a.n > 0 ? kraft != (1ull << kMaxLenLimit) : kraft != 0) T.bad = DFX_STATUS_TABLE;
        uint32_t code = 0, idx = 0;
        for (int l = 1; l <= (int)kMaxLenLimit; l++) {
            T.first[l] = code;
            T.index[l] = idx;
            T.limit[l] = (code + T.nlen[l]) << (kMaxLenLimit - l);
            idx += T.nlen[l];
            code = (code + T.nlen[l]) << 1;
        }
    }
    __syncthreads();
    if (T.bad) {
        if (t == 0) atomicOr(a.status, T.bad);
        return false;
    }
    for (int s = t; s < 256; s += blockDim.x) {
        const uint32_t l = T.lens[s];
        if (l) {
            uint32_t r = 0;
            for (int s2 = 0; s2 < s; s2++) r += (T.lens[s2] == l);
            T.sorted[T.index[l] + r] = (uint8_t)s;
        }
    }
    __syncthreads();
    for (int e = t; e < (1 << kLutBits); e += blockDim.x) {
        const uint32_t v = (uint32_t)e << (kMaxLenLimit - kLutBits);
        int l = 1;
        while (l <= kLutBits && v >= T.limit[l]) l++;
        uint16_t ent = 0;
        if (l <= kLutBits) ent = (uint16_t)((l << 8) | T.sorted[T.index[l] + (v >> (kMaxLenLimit - l)) - T.first[l]]);
        T.lut[e] = ent;
    }
    __syncthreads();
    return true;
}

// A code longer than kLutBits: find its length from the canonical limits.  Returns
// (len << 8) | symbol; bit 16 flags a bit pattern that is no code (Kraft-complete
// tables make that impossible for a well-formed stream).
__device__ __noinline__ uint32_t decode_long(uint32_t peek, const Tables& T) {
    const uint32_t v = peek >> (32 - kMaxLenLimit);
    int l = kLutBits + 1;
    while (l <= (int)kMaxLenLimit && v >= T.limit[l]) l++;
    if (l > (int)kMaxLenLimit) return (1u << 16) | (kMaxLenLimit << 8);
    return ((uint32_t)l << 8) | T.sorted[T.index[l] + (v >> (kMaxLenLimit - l)) - T.first[l]];
}

__device__ __forceinline__ uint32_t ld_word(const uint32_t* sw, uint32_t i, uint32_t maxw) {
    return __ldg(sw + min(i, maxw));
}

// Two BF16 from x = [m0, e0, m1, e1] (bytes, low to high).
__device__ __forceinline__ uint32_t bf16_pair(uint32_t x) {
    return ((x >> 1) & 0x7F807F80u) | ((x << 8) & 0x80008000u) | (x & 0x007F007Fu);
}

__device__ __forceinline__ uint4 merge8(uint2 m, uint32_t e0, uint32_t e1) {
    uint4 o;
    o.x = bf16_pair(__byte_perm(m.x, e0, 0x5140));
    o.y = bf16_pair(__byte_perm(m.x, e0, 0x7362));
    o.z = bf16_pair(__byte_perm(m.y, e1, 0x5140));
    o.w = bf16_pair(__byte_perm(m.y, e1, 0x7362));
    return o;
}

struct GroupStart {
    uint64_t start;  // first bit of this lane's chunk
    uint32_t clen;
    bool ok;
};

__device__ __forceinline__ GroupStart group_start(const DecodeArgs& a, const Tables& T, uint64_t g, unsigned lane,
                                                  bool has_chunk) {
    const unsigned long long* gbase = reinterpret_cast<const unsigned long long*>(a.comp + kOffGbase);
    const uint16_t* clen = reinterpret_cast<const uint16_t*>(a.comp + a.off_clen);
    const uint64_t c = g * 32 + lane;
    const unsigned long long gb0 = __ldg(gbase + g), gb1 = __ldg(gbase + g + 1);
    const uint32_t cl = has_chunk ? (uint32_t)__ldg(clen + c) : 0u;
    uint32_t incl = cl;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const uint32_t y = __shfl_up_sync(kFull, incl, d);
        if (lane >= (unsigned)d) incl += y;
    }
    const uint32_t sum = __shfl_sync(kFull, incl, 31);
    GroupStart r;
    r.ok = gb0 <= gb1 && gb1 - gb0 == sum && gb1 <= T.total_bits;
    r.start = gb0 + (incl - cl);
    r.clen = cl;
    return r;
}

struct BitReader {
    const uint32_t* sw;
    uint32_t maxw, wi, wi0, off0, off;
    uint32_t w0, w1, w2;

    __device__ __forceinline__ void init(const uint32_t* s, uint32_t mw, uint64_t start) {
        sw = s;
        maxw = mw;
        wi = (uint32_t)(start >> 5);
        wi0 = wi;
        off0 = off = (uint32_t)start & 31u;
        w0 = ld_word(sw, wi, maxw);
        w1 = ld_word(sw, wi + 1, maxw);
        w2 = ld_word(sw, wi + 2, maxw);
        wi += 3;
    }
    // Decode one code: returns (len << 8) | symbol and advances.
    __device__ __forceinline__ uint32_t next(const Tables& T, uint32_t& err) {
        const uint32_t peek = __funnelshift_l(w1, w0, off);
        uint32_t ent = T.lut[peek >> (32 - kLutBits)];
        if (ent == 0) {
            ent = decode_long(peek, T);
            if (ent >> 16) {
                err |= DFX_STATUS_STREAM;
                ent &= 0xFFFFu;
            }
        }
        off += ent >> 8;
        if (off >= 32) {
            off -= 32;
            w0 = w1;
            w1 = w2;
            w2 = ld_word(sw, wi, maxw);
            wi++;
        }
        return ent;
    }
    __device__ __forceinline__ uint32_t consumed() const { return (wi - 3 - wi0) * 32 + off - off0; }
};

// A group whose 32 chunks all hold K codes.
template <int K>
__device__ __forceinline__ void decode_full_group(const DecodeArgs& a, const Tables& T, uint32_t* stash, uint64_t g,
                                                  unsigned lane, uint32_t& err) {
    constexpr int S = StashShape<K>::kStride;
    constexpr int R = K / 8;              // 8-element output slots per lane
    constexpr bool kPrefetchM = K <= 64;  // keeps the register budget for K = 128

    const GroupStart gs = group_start(a, T, g, lane, true);
    if (!gs.ok) {
        err |= DFX_STATUS_INDEX;
        return;
    }
    const uint2* mp = reinterpret_cast<const uint2*>(a.comp + a.off_m) + g * (32 * K / 8) + lane;
    uint2 mreg[kPrefetchM ? R : 1];
    if (kPrefetchM) {
#pragma unroll
        for (int r = 0; r < R; r++) mreg[r] = __ldg(mp + 32 * r);
    }

    BitReader br;
    br.init(reinterpret_cast<const uint32_t*>(a.comp + a.off_stream), T.n_words - 1, gs.start);
#pragma unroll 2
    for (int q = 0; q < K / 4; q++) {
        uint32_t acc = 0;
#pragma unroll
        for (int j = 0; j < 4; j++) acc |= (br.next(T, err) & 0xFFu) << (8 * j);
        stash[q * S + lane] = acc;
    }
    if (br.consumed() != gs.clen) err |= DFX_STATUS_STREAM;
    __syncwarp();

    uint4* out4 = reinterpret_cast<uint4*>(a.out) + g * (32 * K / 8) + lane;
#pragma unroll
    for (int r = 0; r < R; r++) {
        const int j0 = 8 * (int)lane + 256 * r;
        const int t = j0 / K, q0 = (j0 % K) / 4;
        const uint32_t e0 = stash[q0 * S + t], e1 = stash[(q0 + 1) * S + t];
        const uint2 m = kPrefetchM ? mreg[kPrefetchM ? r : 0] : __ldg(mp + 32 * r);
        out4[32 * r] = merge8(m, e0, e1);
    }
    __syncwarp();
}

// The last group when it is ragged: chunks may be short or absent, outputs stop at n.
template <int K>
__device__ void decode_tail_group(const DecodeArgs& a, const Tables& T, uint32_t* stash, uint64_t g, unsigned lane,
                                  uint32_t& err) {
    constexpr int S = StashShape<K>::kStride;
    const uint64_t c = g * 32 + lane;
    const bool has = c < a.n_chunk;
    const uint32_t cnt = has ? (uint32_t)min((uint64_t)K, a.n - c * K) : 0u;
    const GroupStart gs = group_start(a, T, g, lane, has);
    if (!gs.ok) {
        err |= DFX_STATUS_INDEX;
        return;
    }
    if (has) {
        BitReader br;
        br.init(reinterpret_cast<const uint32_t*>(a.comp + a.off_stream), T.n_words - 1, gs.start);
        for (int q = 0; q < K / 4; q++) {
            uint32_t acc = 0;
            for (int j = 0; j < 4; j++)
                if ((uint32_t)(4 * q + j) < cnt) acc |= (br.next(T, err) & 0xFFu) << (8 * j);
            stash[q * S + lane] = acc;
        }
        if (br.consumed() != gs.clen) err |= DFX_STATUS_STREAM;
    }
    __syncwarp();
    const uint64_t gbase_elem = g * 32 * K;
    const uint8_t* mplane = a.comp + a.off_m;
    for (int r = 0; r < K / 8; r++) {
        const int j0 = 8 * (int)lane + 256 * r;
        const uint64_t elem = gbase_elem + j0;
        const int t = j0 / K, q0 = (j0 % K) / 4;
        if (elem + 8 <= a.n) {
            const uint2 m = __ldg(reinterpret_cast<const uint2*>(mplane + elem));
            reinterpret_cast<uint4*>(a.out)[elem / 8] = merge8(m, stash[q0 * S + t], stash[(q0 + 1) * S + t]);
        } else {
            for (int i = 0; i < 8; i++) {
                if (elem + i >= a.n) break;
                const int k = (j0 + i) % K;
                const uint32_t e = (stash[(k / 4) * S + t] >> (8 * (k % 4))) & 0xFFu;
                const uint32_t m = mplane[elem + i];
                a.out[elem + i] = (uint16_t)(((m & 0x80u) << 8) | (e << 7) | (m & 0x7Fu));
            }
        }
    }
    __syncwarp();
}

template <int K>
__global__ void __launch_bounds__(kDecodeThreads) k_decode(DecodeArgs a) {
    __shared__ Tables T;
    __shared__ uint32_t stash_all[kDecodeWarps][StashShape<K>::kWords];
    if (!build_tables(a, T)) return;
    const unsigned warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint32_t* stash = stash_all[warp];
    uint32_t err = 0;
    const uint64_t n_full = (a.n % (32ull * K) == 0) ? a.n_group : a.n_group - 1;
    const uint64_t step = (uint64_t)gridDim.x * kDecodeWarps;
    for (uint64_t g = (uint64_t)blockIdx.x * kDecodeWarps + warp; g < a.n_group; g += step) {
        if (g < n_full) decode_full_group<K>(a, T, stash, g, lane, err);
        else decode_tail_group<K>(a, T, stash, g, lane, err);
    }
    if (err) atomicOr(a.status, err);
}

template <int K>
int blocks_per_sm() {
    int b = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, k_decode<K>, kDecodeThreads, 0) != cudaSuccess) return 1;
    return b > 0 ? b : 1;
}

}  // namespace

bool decode_supports(uint32_t K, uint32_t G) { return G == 32 && (K == 32 || K == 64 || K == 128); }

int decode_blocks_per_sm(uint32_t K) {
    switch (K) {
        case 32: return blocks_per_sm<32>();
        case 64: return blocks_per_sm<64>();
        case 128: return blocks_per_sm<128>();
        default: return 1;
    }
}

int decode_warps_per_block() { return kDecodeWarps; }

cudaError_t launch_decode(const DecodeArgs& a, int grid, cudaStream_t s) {
    switch (a.K) {
        case 32: k_decode<32><<<grid, kDecodeThreads, 0, s>>>(a); break;
        case 64: k_decode<64><<<grid, kDecodeThreads, 0, s>>>(a); break;
        case 128: k_decode<128><<<grid, kDecodeThreads, 0, s>>>(a); break;
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

}  // namespace dfx
