// huffman_tables.cuh -- the per-CTA tables of the canonical Huffman exponent code, built
// in shared memory from the container's len[256]: the canonical per-length limits and a
// pair table on the next 14 stream bits that resolves two codes at once when both fit
// (the levels of the hierarchical lookup tables of "DFloat11: lossless LLM compression
// for GPU", aikraft.ru blog, section 03, item 1).  Shared by the decode kernel (decode.cu)
// and the decode-into-GEMM kernel (decode_gemm.cu).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "dfx_common.cuh"

namespace dfx {
namespace {

constexpr int kLutBits = 14;  // the decode kernel's pair table: 2^14 entries (64 KiB)

// Pair table entry (u32), indexed by the next LB stream bits (LB = kLutBits for the decode
// kernel; the table has 2^LB entries):
//   bits 0-7   first symbol        bits 8-15  second symbol
//   bits 16-20 length of the first code (0: the first code is longer than LB)
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

// The pair table `lut` (1 << LB entries) from the canonical tables.  The entries whose
// index bits start with the code c0 of a first symbol s0 of length l0 <= LB are
// [c0, c0 + 1) << (LB - l0); one warp per first symbol marks that run "first
// code only" and then overwrites, for every second symbol whose code c1 fits the
// remaining r = LB - l0 bits, the sub-run that continues with c1.  Entries no short
// code starts keep the "long first code" mark.  Every thread of the block calls it.
template <int LB = kLutBits>
__device__ void build_pair_table(const HuffTables& T, uint32_t* lut) {
    const int t = threadIdx.x;
    const unsigned warp = t >> 5, lane = t & 31;
    for (int i = t; i < (1 << LB) / 4; i += blockDim.x)
        reinterpret_cast<uint4*>(lut)[i] = make_uint4(kNotPair, kNotPair, kNotPair, kNotPair);
    __syncthreads();
    const uint32_t n_short = T.index[LB + 1];  // symbols with codes of at most LB bits
    for (uint32_t i0 = warp; i0 < n_short; i0 += blockDim.x >> 5) {
        const uint32_t l0 = T.slen[i0], s0 = T.sorted[i0];
        const uint32_t r = LB - l0;
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
template <int LB = kLutBits>
__device__ __noinline__ uint32_t decode_long(uint32_t peek, const HuffTables& T) {
    const uint32_t v = peek >> (32 - kMaxLenLimit);
    int l = LB + 1;
    while (l <= (int)kMaxLenLimit && v >= T.limit[l]) l++;
    if (l > (int)kMaxLenLimit) return (1u << 16) | (kMaxLenLimit << 8);
    return ((uint32_t)l << 8) | T.sorted[T.index[l] + (v >> (kMaxLenLimit - l)) - T.first[l]];
}


}  // namespace
}  // namespace dfx
