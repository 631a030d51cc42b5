// decode.cu -- the DFX1 decode kernel for sm_100a: compressed container -> BF16 in HBM.
//
// Design (B200-first; the pages' GPU decoder is prior art, "DFloat11: lossless LLM
// compression for GPU", aikraft.ru blog, section 03):
//   * persistent grid, one CTA of 32 warps per SM that first builds its tables in shared
//     memory from len[256]: a pair table on the next 14 bits that resolves two
//     codes at once when both fit, a one-code view of it, and, for codes longer than 14
//     bits, the canonical per-length limits (the levels of the hierarchical table of
//     section 03, item 1);
//   * one warp decodes one group of 32 chunks; lane i owns chunk i of the group: the
//     group's 8-element blocks i, i+32, ...  Its read position is the group's start bit
//     plus the warp's exclusive scan of the chunk bit lengths (the "lightweight
//     auxiliary variables" that coordinate read positions, section 03, item 2).  Write
//     positions need no scan: after every 8 codes the lane holds 8 consecutive outputs
//     and the warp's 16-byte stores cover 512 contiguous bytes;
//   * each lane keeps its bit position and a 32-bit peek of the stream; the peek is
//     reloaded from the warp's shared-memory copy of the group's stream slice once per
//     two pair lookups, so the common path has no per-code branch besides the rare
//     unresolved-pair test;
//   * the next group's stream slice is copied into shared memory (cp.async) and its
//     index loaded while the current group decodes; the group's sign+mantissa bytes are
//     prefetched into L2 when it starts and each block's are loaded a block ahead; each pair
//     lookup is merged at once: one byte permute of the table entry with the m word and
//     one 32-bit rotate give two BF16 (the m bytes of a pair carry each other's sign).
// Every read of the container is bounded by the header-checked section sizes; a bad
// container sets bits of the status word and the kernel finishes normally.
#include <cuda_runtime.h>
#include <stdint.h>

#include "dfx_common.cuh"

namespace dfx {
namespace {

constexpr int kLutBits = 14;
// Warps per CTA: one CTA per SM holds the 64 KiB pair table once.
template <int K>
struct DecodeShape {
    static constexpr int kWarps = 32;
    static constexpr int kThreads = kWarps * 32;
};
constexpr unsigned kFull = 0xffffffffu;

// Pair table entry (u32), indexed by the next kLutBits stream bits:
//   bits 0-7   first symbol        bits 8-15  second symbol
//   bits 16-20 length of the first code (0: the first code is longer than kLutBits)
//   bits 26-30 bits the fast path consumes: both codes' lengths when both fit in the
//              index bits, else the first code's length (0 for a long first code)
//   bit  31    set when the entry does not hold two complete codes
constexpr uint32_t kNotPair = 0x80000000u;

struct Tables {
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
__device__ bool build_canonical(const DecodeArgs& a, Tables& T) {
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
__device__ void build_pair_table(const Tables& T, uint32_t* lut) {
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
__device__ __noinline__ uint32_t decode_long(uint32_t peek, const Tables& T) {
    const uint32_t v = peek >> (32 - kMaxLenLimit);
    int l = kLutBits + 1;
    while (l <= (int)kMaxLenLimit && v >= T.limit[l]) l++;
    if (l > (int)kMaxLenLimit) return (1u << 16) | (kMaxLenLimit << 8);
    return ((uint32_t)l << 8) | T.sorted[T.index[l] + (v >> (kMaxLenLimit - l)) - T.first[l]];
}


// Two BF16 from x = [m0, e0, m1, e1] (bytes, low to high), where the m byte of each
// element is its mantissa above its partner's sign: rotating x right by one bit puts
// both mantissas and exponents in place and moves each partner's sign bit to the top
// of the other half.
__device__ __forceinline__ uint32_t bf16_pair(uint32_t x) { return __funnelshift_r(x, x, 1); }



// ---------------------------------------------------------------- group index

struct GroupIndex {
    unsigned long long gb0;  // start bit of the group
    uint32_t span;           // group bits, or 0xFFFFFFFF if the group's entries are inconsistent
    uint32_t clen;           // this lane's chunk bits
};

__device__ __forceinline__ GroupIndex load_index(const DecodeArgs& a, const Tables& T, uint64_t g, unsigned lane,
                                                 bool has_chunk) {
    const unsigned long long* gbase = reinterpret_cast<const unsigned long long*>(a.comp + kOffGbase);
    const uint16_t* clen = reinterpret_cast<const uint16_t*>(a.comp + a.off_clen);
    GroupIndex r;
    r.gb0 = __ldg(gbase + g);
    const unsigned long long gb1 = __ldg(gbase + g + 1);
    const bool bad = gb1 < r.gb0 || gb1 > T.total_bits || gb1 - r.gb0 >= 0xFFFFFFFFull;
    r.span = bad ? 0xFFFFFFFFu : (uint32_t)(gb1 - r.gb0);
    r.clen = has_chunk ? (uint32_t)__ldg(clen + g * 32 + lane) : 0u;
    return r;
}

struct GroupStart {
    unsigned long long start;  // first bit of this lane's chunk
    unsigned long long gb0;    // first bit of the group
    uint32_t span;             // bits of the group
    uint32_t clen;
    bool ok;
};

// Warp exclusive scan of the chunk lengths: the lane's read position.
__device__ __forceinline__ GroupStart scan_index(const GroupIndex& x, unsigned lane) {
    uint32_t incl = x.clen;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const uint32_t y = __shfl_up_sync(kFull, incl, d);
        if (lane >= (unsigned)d) incl += y;
    }
    const uint32_t sum = __shfl_sync(kFull, incl, 31);
    GroupStart r;
    r.ok = x.span == sum;
    r.start = x.gb0 + (incl - x.clen);
    r.gb0 = x.gb0;
    r.span = x.span;
    r.clen = x.clen;
    return r;
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
// shared-memory copy of its group's slice of the stream.
struct GlobalWords {
    const uint32_t* p;  // first word of the source
    __device__ __forceinline__ uint32_t load(uint32_t i) const { return __ldg(p + i); }
};
struct ClampedGlobalWords {
    const uint32_t* p;
    uint32_t maxw;  // last readable index
    __device__ __forceinline__ uint32_t load(uint32_t i) const { return __ldg(p + min(i, maxw)); }
};
struct SharedWords {
    uint32_t s;  // shared-memory address of the slice buffer
    // Well-formed groups read inside the slice.  A corrupt one reads at most 3K/4 + 2
    // words past a chunk start, into the other slice buffer or the warp's m units that
    // follow them: never outside the warp's own buffers.
    __device__ __forceinline__ uint32_t load(uint32_t i) const {
        uint32_t v;
        asm volatile("ld.shared.u32 %0, [%1];\n" : "=r"(v) : "r"(s + 4u * i));
        return v;
    }
};

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
    __device__ __forceinline__ uint32_t one(const Tables& T, uint32_t& err) {
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
    __device__ __forceinline__ uint32_t pair(uint32_t mw, const Tables& T, uint32_t& err) {
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
__device__ __forceinline__ uint4 decode_block(BitReader<Words>& br, const Tables& T, uint2 m, uint32_t& err) {
    uint4 o;
    br.reload();
    o.x = br.template pair<0>(m.x, T, err);
    o.y = br.template pair<1>(m.x, T, err);
    br.reload();
    o.z = br.template pair<0>(m.y, T, err);
    o.w = br.template pair<1>(m.y, T, err);
    return o;
}

// ---------------------------------------------------------------- per-warp buffers
//
// Everything a warp reads in bulk is copied into its shared-memory buffers ahead of use by
// one lane with cp.async.bulk (the 1-D bulk copy engine), each buffer completing on its own
// mbarrier: the stream slice of the next group (double-buffered) and the sign+mantissa
// bytes in units of 4 blocks (1 KiB), kMUnits units ahead.  Without that a warp keeps only
// a few hundred bytes of loads in flight and, at one CTA of 32 warps per SM, the memory
// system stalls on latency well below its bandwidth.

// Stream words staged per group: the slice of a K = 64 group averages ~0.7 KiB on
// Gaussian weights; groups that do not fit decode from global memory.
template <int K>
struct SliceShape {
    static constexpr uint32_t kWords = K <= 64 ? 4u * K : 3u * K;  // 1 KiB at K = 64, 1.5 KiB at K = 128
};

constexpr uint32_t kMUnitBlocks = 4;                      // blocks of one m unit
constexpr uint32_t kMUnitBytes = kMUnitBlocks * 32 * 8;   // 1 KiB
constexpr uint32_t kMUnits = 2;                           // m units in flight per warp

template <int K>
struct WarpBuffers {
    __align__(16) uint32_t slice[2][SliceShape<K>::kWords];  // this group's stream words and the next's
    uint2 munit[kMUnits][kMUnitBlocks * 32];                  // m bytes, [block][lane]
    unsigned long long mbar[2 + kMUnits];                     // slice 0, slice 1, m units
};

template <int K>
__host__ __device__ constexpr size_t warp_buffer_bytes() {
    return (sizeof(WarpBuffers<K>) + 15) & ~size_t(15);
}

__device__ __forceinline__ uint32_t smem_addr(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }
__device__ __forceinline__ void mbar_init(unsigned long long* bar) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;\n" ::"r"(smem_addr(bar)) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() { asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory"); }
// orders this thread's (and, after a warp barrier, the warp's) earlier generic accesses to
// shared memory before the bulk copies it issues next
__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory"); }
// arm `bar` for `bytes` and copy them from global `src` to shared `dst` (both 16-byte
// aligned, bytes a multiple of 16)
__device__ __forceinline__ void bulk_copy(void* dst, const void* src, uint32_t bytes, unsigned long long* bar) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(smem_addr(bar)), "r"(bytes) : "memory");
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::"r"(
                     smem_addr(dst)),
                 "l"(src), "r"(bytes), "r"(smem_addr(bar))
                 : "memory");
}
// Wait for the phase with the given parity of `bar` to complete.  One blocking poll first
// (try_wait, which suspends the warp for at most the 100 us time hint: staged data
// normally lands within it), then non-blocking polls (test_wait) with a sleep of at most
// 128 ns between them (__nanosleep(64) lasts at most twice its argument); a wait that
// never completes gives up after ~0.1 ms + ~0.35 s and the caller reports
// DFX_STATUS_TIMEOUT.
constexpr uint32_t kWaitPolls = 1u << 21;
__device__ __forceinline__ bool mbar_wait(unsigned long long* bar, uint32_t parity) {
    const uint32_t addr = smem_addr(bar);
    uint32_t done;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, 100000;\n selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(done)
        : "r"(addr), "r"(parity)
        : "memory");
    if (done) return true;
    for (uint32_t i = 0; i < kWaitPolls; i++) {
        asm volatile(
            "{\n .reg .pred p;\n mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
            : "=r"(done)
            : "r"(addr), "r"(parity)
            : "memory");
        if (done) return true;
        __nanosleep(64);
    }
    return false;
}
__device__ __forceinline__ void prefetch_l2(const void* p, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;\n" ::"l"(p), "r"(bytes) : "memory");
}
__device__ __forceinline__ void prefetch_line_l2(const void* p) {
    asm volatile("prefetch.global.L2 [%0];\n" ::"l"(p) : "memory");
}
__device__ __forceinline__ uint2 ld_shared_u2(const void* p) {
    uint2 v;
    asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];\n" : "=r"(v.x), "=r"(v.y) : "r"(smem_addr(p)));
    return v;
}

// The stream words of one group, [gb0 >> 5, ((gb0 + span) >> 5) + 4), in 16-byte units:
// staged when the group is consistent and they fit the slice buffer, else the group is
// decoded straight from global memory.
struct Slice {
    uint32_t base;   // stream word index of the first staged word
    uint32_t bytes;  // bytes to copy
    bool staged;
};

template <uint32_t kWords>
__device__ __forceinline__ Slice plan_slice(const Tables& T, unsigned long long gb0, uint32_t span, bool ok) {
    Slice r;
    const uint32_t beg = ((uint32_t)(gb0 >> 5) * 4u) & ~15u;  // bytes into the stream section
    const uint32_t end = min((((uint32_t)((gb0 + span) >> 5) + 4u) * 4u + 15u) & ~15u, T.n_words * 4u);
    r.base = beg / 4u;
    r.staged = ok && end > beg && end - beg <= kWords * 4u;
    r.bytes = r.staged ? end - beg : 0u;
    return r;
}

// The m pipeline of one warp: unit j of the warp's sequence (group j / U of the warp,
// blocks 4 (j % U) .. 4 (j % U) + 3, U = K / 32 units per group) is copied into slot
// j % kMUnits when unit j - kMUnits has been decoded.
template <int K>
struct MPipe {
    static constexpr uint32_t U = K / 32;
    uint32_t j;       // next unit to decode
    uint32_t g0;      // the warp's first group
    uint32_t step;    // groups between the warp's consecutive groups
    uint32_t groups;  // full groups of this warp

    // lane 0 only; the slot's previous contents have been read by the whole warp
    __device__ __forceinline__ void issue(const DecodeArgs& a, WarpBuffers<K>& wb, uint32_t unit) const {
        if (unit / U < groups) {
            const uint32_t g = g0 + (unit / U) * step;
            const uint32_t slot = unit % kMUnits;
            bulk_copy(wb.munit[slot], a.comp + a.off_m + (uint64_t)g * (32u * K) + (unit % U) * kMUnitBytes,
                      kMUnitBytes, &wb.mbar[2 + slot]);
        }
    }
};

// Decode one full group's 32 chunks (lane i: blocks i, i+32, ... of the group) and write
// its BF16 output.  Each lane decodes 8 codes, then stores 8 outputs (16 bytes; 512
// contiguous bytes per warp store).  The m bytes come from the staged units; once a unit
// has been decoded, lane 0 refills its slot with the unit kMUnits further on.
template <int K, class Words>
__device__ __forceinline__ void decode_group_blocks(const DecodeArgs& a, const Tables& T, BitReader<Words>* br,
                                                    WarpBuffers<K>& wb, MPipe<K>& mp, uint32_t g, unsigned lane,
                                                    uint32_t& err) {
    uint4* op = reinterpret_cast<uint4*>(a.out) + ((uint64_t)g * (32u * K) - a.out_first) / 8u + lane;
    for (uint32_t u = 0; u < MPipe<K>::U; u++) {
        const uint32_t slot = mp.j % kMUnits;
        if (!mbar_wait(&wb.mbar[2 + slot], (mp.j / kMUnits) & 1u)) err |= DFX_STATUS_TIMEOUT;
        if (br) {
            const uint2* mu = wb.munit[slot] + lane;
#pragma unroll 2
            for (uint32_t kk = 0; kk < kMUnitBlocks; kk++)
                op[32u * (kMUnitBlocks * u + kk)] = decode_block(*br, T, ld_shared_u2(mu + 32u * kk), err);
        }
        __syncwarp();
        if (lane == 0) {
            fence_proxy_async();
            mp.issue(a, wb, mp.j + kMUnits);
        }
        mp.j++;
    }
}

// A warp's position in its sequence of full groups g0, g0 + step, ...
template <int K>
struct GroupState {
    MPipe<K> mp;
    GroupStart st;      // the group to decode next
    Slice sl;           // its stream slice
    GroupIndex idx_n;   // the index entries of the group after it
    uint32_t g, gn;     // those two groups
    uint32_t b;         // slice buffer of group g
    uint32_t sphase;    // parity of each slice buffer's next phase
};

// Start the copies of the warp's first group (stream slice, first kMUnits m units) and
// load the index of its second group; needs only the canonical tables, so it runs while
// the block builds the pair table.  The warp has at least one full group.
template <int K>
__device__ __forceinline__ void group_prologue(const DecodeArgs& a, const Tables& T, WarpBuffers<K>& wb, uint32_t g,
                                               uint32_t step, uint32_t n_full, unsigned lane, GroupState<K>& s) {
    if (lane == 0) {
        for (int i = 0; i < 2 + (int)kMUnits; i++) mbar_init(&wb.mbar[i]);
        fence_mbar_init();
        fence_proxy_async();
    }
    __syncwarp();
    s.mp = MPipe<K>{0u, g, step, (n_full - g + step - 1) / step};
    s.st = scan_index(load_index(a, T, g, lane, true), lane);
    s.sl = plan_slice<SliceShape<K>::kWords>(T, s.st.gb0, s.st.span, s.st.ok);
    if (lane == 0) {
        // (the test hook leaves one copy out, so that its bounded wait runs out)
        const bool skip = (a.inject & DFX_INJECT_SKIP_SLICE_COPY) && g == a.g_begin;
        if (s.sl.staged && !skip) bulk_copy(wb.slice[0], a.comp + a.off_stream + 4u * s.sl.base, s.sl.bytes, &wb.mbar[0]);
        for (uint32_t u = 0; u < kMUnits; u++) s.mp.issue(a, wb, u);
    }
    s.g = g;
    s.gn = g + step;
    if (s.gn < n_full) s.idx_n = load_index(a, T, s.gn, lane, true);
    s.b = 0;
    s.sphase = 0;
}

// Full groups, one warp at a time, from the state the prologue left.  While group g
// decodes, the stream slice of the warp's next group is copied into the other slice
// buffer, the index of the group after that is loaded, and the m units run kMUnits units
// (4 blocks each) ahead of the decode.
template <int K>
__device__ void decode_full_groups(const DecodeArgs& a, const Tables& T, const uint32_t* lut, WarpBuffers<K>& wb,
                                   GroupState<K>& s0, uint32_t step, uint32_t n_full, unsigned lane, uint32_t& err) {
    constexpr uint32_t kWords = SliceShape<K>::kWords;
    const uint32_t* sw = reinterpret_cast<const uint32_t*>(a.comp + a.off_stream);
    const uint8_t* sbytes = a.comp + a.off_stream;
    const uint32_t maxw = T.n_words - 1;
    MPipe<K> mp = s0.mp;
    GroupStart st = s0.st;
    Slice sl = s0.sl;
    GroupIndex idx_n = s0.idx_n;
    uint32_t g = s0.g, gn = s0.gn, b = s0.b, sphase = s0.sphase;

    while (true) {
        const bool has_next = gn < n_full;
        const uint32_t gnn = gn + step;
        GroupStart st_n;
        Slice sl_n;
        GroupIndex idx_nn;
        if (has_next) {
            st_n = scan_index(idx_n, lane);
            sl_n = plan_slice<kWords>(T, st_n.gb0, st_n.span, st_n.ok);
            if (lane == 0 && sl_n.staged)  // buffer b ^ 1 was released at the end of the previous group
                bulk_copy(wb.slice[b ^ 1], sbytes + 4u * sl_n.base, sl_n.bytes, &wb.mbar[b ^ 1]);
            if (gnn < n_full) idx_nn = load_index(a, T, gnn, lane, true);
        }
        if (sl.staged) {
            if (!mbar_wait(&wb.mbar[b], (sphase >> b) & 1u)) err |= DFX_STATUS_TIMEOUT;
            sphase ^= 1u << b;
        }

        if (st.ok) {
            uint32_t used;
            if (sl.staged) {
                BitReader<SharedWords> br;
                br.init(lut, SharedWords{smem_addr(wb.slice[b])}, (uint32_t)(st.start - 32ull * sl.base));
                decode_group_blocks<K>(a, T, &br, wb, mp, g, lane, err);
                used = br.consumed();
            } else {
                // A chunk reads at most 3K/4 + 2 words past its start (24-bit codes); lane 31
                // starts last.  When that stays inside the stream the loads need no clamp.
                const uint32_t first = (uint32_t)(st.gb0 >> 5);
                const uint32_t last = __shfl_sync(kFull, (uint32_t)(st.start >> 5), 31);
                const uint32_t rel = (uint32_t)(st.start - 32ull * first);
                if (last + (3u * K) / 4u + 8u <= maxw) {
                    BitReader<GlobalWords> br;
                    br.init(lut, GlobalWords{sw + first}, rel);
                    decode_group_blocks<K>(a, T, &br, wb, mp, g, lane, err);
                    used = br.consumed();
                } else {
                    BitReader<ClampedGlobalWords> br;
                    br.init(lut, ClampedGlobalWords{sw + first, maxw - first}, rel);
                    decode_group_blocks<K>(a, T, &br, wb, mp, g, lane, err);
                    used = br.consumed();
                }
            }
            if (used != st.clen) err |= DFX_STATUS_STREAM;
        } else {
            err |= DFX_STATUS_INDEX;
            decode_group_blocks<K, SharedWords>(a, T, nullptr, wb, mp, g, lane, err);  // keeps the m pipeline in step
        }
        __syncwarp();  // the slice buffer is refilled by the copy issued next iteration
        if (lane == 0) fence_proxy_async();
        if (!has_next) break;
        g = gn;
        gn = gnn;
        st = st_n;
        sl = sl_n;
        idx_n = idx_nn;
        b ^= 1;
    }
}

// The blocks of the ragged last group: a lane's chunk holds the elements of its blocks
// that are below n (a prefix of the chunk, possibly empty).  Whole blocks take the pair
// path; the lane's last, partial block is decoded code by code and stored element-wise.
template <int K, class Words>
__device__ __forceinline__ void decode_tail_blocks(const DecodeArgs& a, const Tables& T, BitReader<Words>& br,
                                                   uint32_t g, unsigned lane, uint32_t& err) {
    const uint8_t* mplane = a.comp + a.off_m;
    for (uint32_t k = 0; k < K / 8; k++) {
        const uint64_t x0 = block_element(g, K, k, lane);
        if (x0 + 8 <= a.n) {
            reinterpret_cast<uint4*>(a.out)[(x0 - a.out_first) / 8] =
                decode_block(br, T, __ldg(reinterpret_cast<const uint2*>(mplane + x0)), err);
            continue;
        }
        if (x0 < a.n) {
            const uint32_t cnt = (uint32_t)(a.n - x0);
            br.reload();
            for (uint32_t j = 0; j < cnt; j++) {  // decode and store one element at a time
                const uint32_t ex = br.one(T, err);
                const uint64_t x = x0 + j, partner = (x ^ 1u) < a.n ? (x ^ 1u) : x;
                a.out[x - a.out_first] = (uint16_t)(((mplane[partner] & 1u) << 15) | (ex << 7) | (mplane[x] >> 1u));
            }
        }
        break;
    }
}

// The last group when it is ragged, by one warp after its full groups: its stream slice
// is copied into the warp's (now idle) slice buffer when it fits, else read from global
// memory with clamped loads.
template <int K>
__device__ void decode_tail_group(const DecodeArgs& a, const Tables& T, const uint32_t* lut, WarpBuffers<K>& wb,
                                  uint32_t g, unsigned lane, uint32_t& err) {
    const GroupStart gs = scan_index(load_index(a, T, g, lane, true), lane);
    if (!gs.ok) {
        err |= DFX_STATUS_INDEX;
        return;
    }
    const Slice sl = plan_slice<SliceShape<K>::kWords>(T, gs.gb0, gs.span, gs.ok);
    uint32_t used;
    if (sl.staged) {
        const uint4* src = reinterpret_cast<const uint4*>(a.comp + a.off_stream + 4u * sl.base);
        uint4* dst = reinterpret_cast<uint4*>(wb.slice[0]);
        for (uint32_t c = lane; c < sl.bytes / 16u; c += 32) dst[c] = __ldg(src + c);
        __syncwarp();
        BitReader<SharedWords> br;
        br.init(lut, SharedWords{smem_addr(wb.slice[0])}, (uint32_t)(gs.start - 32ull * sl.base));
        decode_tail_blocks<K>(a, T, br, g, lane, err);
        used = br.consumed();
    } else {
        const uint32_t* sw = reinterpret_cast<const uint32_t*>(a.comp + a.off_stream);
        const uint32_t maxw = T.n_words - 1;
        const uint32_t first = (uint32_t)(gs.gb0 >> 5);
        BitReader<ClampedGlobalWords> br;
        br.init(lut, ClampedGlobalWords{sw + first, maxw - first}, (uint32_t)(gs.start - 32ull * first));
        decode_tail_blocks<K>(a, T, br, g, lane, err);
        used = br.consumed();
    }
    if (used != gs.clen) err |= DFX_STATUS_STREAM;
}

constexpr size_t kLutBytes = sizeof(uint32_t) << kLutBits;

// One tensor's decode by `ctas` CTAs of which this is number `cta`: the body of both
// kernels below.
template <int K>
__device__ __forceinline__ void decode_tensor(const DecodeArgs& a, uint32_t cta, uint32_t ctas) {
    constexpr int kDecodeWarps = DecodeShape<K>::kWarps;
    __shared__ Tables T;
    // dynamic shared memory: the pair table, then one buffer per warp
    extern __shared__ __align__(16) uint8_t dyn_smem[];
    uint32_t* lut = reinterpret_cast<uint32_t*>(dyn_smem);
    uint8_t* warp_area = dyn_smem + kLutBytes;
    const uint32_t n_full = (a.n % (32ull * K) == 0) ? a.n_group : a.n_group - 1;
    const uint32_t full_end = min(n_full, a.g_end);  // full groups to decode: [g_begin, full_end)
    {
        // start fetching each warp's first group (index entries, m plane) into L2 while
        // the tables are built
        const uint32_t g0 = a.g_begin + cta + ctas * (threadIdx.x >> 5);
        if ((threadIdx.x & 31) == 0 && g0 < full_end) {
            prefetch_line_l2(a.comp + kOffGbase + 8ull * g0);
            prefetch_line_l2(a.comp + a.off_clen + 64ull * g0);
            prefetch_line_l2(a.comp + a.off_clen + 64ull * g0 + 63);
            prefetch_l2(a.comp + a.off_m + (uint64_t)g0 * (32u * K), 32u * K);
        }
    }
    if (!build_canonical(a, T)) return;
    const unsigned warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    WarpBuffers<K>& wb = *reinterpret_cast<WarpBuffers<K>*>(warp_area + warp * warp_buffer_bytes<K>());
    uint32_t err = 0;
    const uint32_t step = ctas * kDecodeWarps;
    // groups are dealt to the CTAs (one per SM) in turn and each CTA's to its warps in
    // turn, so that every SM gets the same number of groups within one
    const uint32_t gw = a.g_begin + cta + ctas * warp;
    GroupState<K> gs;
    if (gw < full_end) group_prologue<K>(a, T, wb, gw, step, full_end, lane, gs);
    build_pair_table(T, lut);
    if (gw < full_end) decode_full_groups<K>(a, T, lut, wb, gs, step, full_end, lane, err);
    // the ragged last group, by the warp whose sequence it would continue
    if (n_full < a.n_group && n_full >= a.g_begin && n_full < a.g_end && gw == a.g_begin + (n_full - a.g_begin) % step)
        decode_tail_group<K>(a, T, lut, wb, n_full, lane, err);
    if (err) atomicOr(a.status, err);
}

template <int K>
__global__ void __launch_bounds__(DecodeShape<K>::kThreads, 1) k_decode(DecodeArgs a) {
    decode_tensor<K>(a, blockIdx.x, gridDim.x);
}

// Several tensors in one launch (all with the same K): each CTA decodes its share of one
// tensor, so it builds that tensor's tables once.
template <int K>
__global__ void __launch_bounds__(DecodeShape<K>::kThreads, 1) k_decode_batch(const __grid_constant__ BatchArgs b) {
    uint32_t i = 0;
    while (i + 1 < b.count && blockIdx.x >= b.cta_begin[i + 1]) i++;
    decode_tensor<K>(b.t[i], blockIdx.x - b.cta_begin[i], b.cta_begin[i + 1] - b.cta_begin[i]);
}

constexpr size_t kGuardBytes = 0;  // reads past a warp's slices stay in its m units, see SharedWords

template <int K>
constexpr size_t dyn_smem_bytes() {
    return kLutBytes + DecodeShape<K>::kWarps * warp_buffer_bytes<K>() + kGuardBytes;
}
static_assert(sizeof(WarpBuffers<128>::munit) >= 4 * (3 * 128 / 4 + 8) && sizeof(WarpBuffers<32>::munit) >= 4 * (3 * 32 / 4 + 8),
              "the m units after the slices cover the longest run past a slice");
static_assert(DecodeShape<32>::kThreads >= 256 && DecodeShape<64>::kThreads >= 256 && DecodeShape<128>::kThreads >= 256,
              "the table build gives each of the 256 symbols its own thread");
static_assert(dyn_smem_bytes<64>() + 1024 <= 227 * 1024 && dyn_smem_bytes<128>() + 1024 <= 227 * 1024, "shared memory");

template <int K>
int blocks_per_sm() {
    int b = 0;
    if (cudaFuncSetAttribute(k_decode<K>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dyn_smem_bytes<K>()) !=
        cudaSuccess)
        return 1;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, k_decode<K>, DecodeShape<K>::kThreads, dyn_smem_bytes<K>()) !=
        cudaSuccess)
        return 1;
    return b > 0 ? b : 1;
}

// The dynamic shared-memory limit of a kernel is raised once per device (needed above
// 48 KiB).
template <class F>
cudaError_t allow_smem(F* kernel, size_t bytes, bool* done) {
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 64 && done[dev]) return cudaSuccess;
    const cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e == cudaSuccess && dev >= 0 && dev < 64) done[dev] = true;
    return e;
}

template <int K>
cudaError_t launch_k(const DecodeArgs& a, int grid, cudaStream_t s) {
    static bool attr_set[64] = {};
    const cudaError_t e = allow_smem(k_decode<K>, dyn_smem_bytes<K>(), attr_set);
    if (e != cudaSuccess) return e;
    k_decode<K><<<grid, DecodeShape<K>::kThreads, dyn_smem_bytes<K>(), s>>>(a);
    return cudaGetLastError();
}

template <int K>
cudaError_t launch_batch_k(const BatchArgs& b, cudaStream_t s) {
    static bool attr_set[64] = {};
    const cudaError_t e = allow_smem(k_decode_batch<K>, dyn_smem_bytes<K>(), attr_set);
    if (e != cudaSuccess) return e;
    k_decode_batch<K><<<b.cta_begin[b.count], DecodeShape<K>::kThreads, dyn_smem_bytes<K>(), s>>>(b);
    return cudaGetLastError();
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

int decode_warps_per_block(uint32_t K) {
    return K == 32 ? DecodeShape<32>::kWarps : K == 64 ? DecodeShape<64>::kWarps : DecodeShape<128>::kWarps;
}

cudaError_t launch_decode_batch(const BatchArgs& b, uint32_t K, cudaStream_t s) {
    if (b.count == 0 || b.count > kMaxBatch || b.cta_begin[b.count] == 0) return cudaErrorInvalidValue;
    switch (K) {
        case 32: return launch_batch_k<32>(b, s);
        case 64: return launch_batch_k<64>(b, s);
        case 128: return launch_batch_k<128>(b, s);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_decode(const DecodeArgs& a, int grid, cudaStream_t s) {
    switch (a.K) {
        case 32: return launch_k<32>(a, grid, s);
        case 64: return launch_k<64>(a, grid, s);
        case 128: return launch_k<128>(a, grid, s);
        default: return cudaErrorInvalidValue;
    }
}


}  // namespace dfx
