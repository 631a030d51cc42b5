// huffman_reader.cuh -- a lane's reader of the canonical Huffman code stream (the pair
// table and per-length limits of huffman_tables.cuh) over a word source of
// decode_pipeline.cuh, and the 8-code block decode that merges the exponents with their
// sign+mantissa bytes.  Used by the decode kernel (decode.cu) and the decode-into-GEMM
// kernel (decode_gemm.cu).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "decode_pipeline.cuh"
#include "huffman_tables.cuh"

namespace dfx {
namespace {

// ---------------------------------------------------------------- bit reader
//
// A lane's state is its bit position p, relative to the first word of its word source,
// `peek`, the 32 stream bits starting at p, and the two words cur, nxt that hold them
// (word cw and cw + 1).  Once per round of two pairs, peek is rebuilt from cur and nxt
// with one funnel shift; only when p has moved into the next word does the lane shift
// its words along and load one new word.  No reload follows more than 32 consumed bits
// (two table pairs take at most 28, a single code at most 24), so p moves at most one
// word between reloads, and about one lane in three loads a word per round.  Every
// pair the table resolves consumes at most LB (<= 14) bits, so after the first pair
// of a round at least 18 valid bits remain for the second.  Pairs the table cannot
// resolve (the second code does not fit the index bits, or the first code is longer)
// take a rare branch: it reloads after the first code and, when both codes are at most
// LB long, reads the second from the table entry at the new position; otherwise
// it decodes code by code with the canonical limits.
//
// Word sources: the global stream (with or without a bound clamp) or a warp's
// shared-memory copy of a stream slice (decode_pipeline.cuh).
template <class Words, int LB = kLutBits>  // LB: index bits of the pair table
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
        const uint32_t e = lut[peek >> (32 - LB)];
        uint32_t len, sym;
        if ((e & 0x001F0000u) == 0) {
            uint32_t ent = decode_long<LB>(peek, T);
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
        const uint32_t e = lut[peek >> (32 - LB)];
        const uint32_t len = e >> 26;           // bit 5 is set when the entry is not a pair
        peek = __funnelshift_l(0u, peek, len);  // shifts by len & 31
        p += len;
        uint32_t syms = e;
        if ((int32_t)e < 0) {
            p -= 32;  // undo bit 5 of `len`
            reload();
            // usually both codes fit the table on their own: the second one is the first
            // code of the entry at the new position, and peek keeps at least 18 valid bits
            const uint32_t e2 = lut[peek >> (32 - LB)];
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
template <class Words, int LB>
__device__ __forceinline__ uint4 decode_block(BitReader<Words, LB>& br, const HuffTables& T, uint2 m, uint32_t& err) {
    uint4 o;
    br.reload();
    o.x = br.template pair<0>(m.x, T, err);
    o.y = br.template pair<1>(m.x, T, err);
    br.reload();
    o.z = br.template pair<0>(m.y, T, err);
    o.w = br.template pair<1>(m.y, T, err);
    return o;
}

}  // namespace
}  // namespace dfx
