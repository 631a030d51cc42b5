// decode_pipeline.cuh -- the memory pipeline and group loop shared by the decode kernels of
// both exponent coders (decode.cu: canonical Huffman, decode_tans.cu: tANS).
//
// Everything here is independent of how the exponents are coded:
//   * persistent grid, one CTA of 32 warps per SM; the coder builds its tables in shared
//     memory first (while the first group's copies are already in flight);
//   * one warp decodes one group of 32 chunks; lane i owns chunk i of the group: the
//     group's 8-element blocks i, i+32, ...  Its read position is the group's start bit
//     plus the warp's exclusive scan of the chunk bit lengths: the per-group start bits
//     and per-chunk bit lengths are the small position records with which each thread
//     finds where to read ("DFloat11: lossless LLM compression for GPU", aikraft.ru
//     blog, section 03, item 2).  Write positions need
//     no scan: after every 8 codes the lane holds 8 consecutive outputs and the warp's
//     16-byte stores cover 512 contiguous bytes;
//   * the next group's stream slice and the sign+mantissa bytes are copied into the warp's
//     shared-memory buffers by the bulk copy engine, each buffer completing on its own
//     mbarrier, while the current group decodes; the index of the group after next is
//     loaded meanwhile;
//   * the ragged last group, and ranges of groups (a slice of the tensor into a buffer
//     holding just that slice), take the same path.
// Every read of the container is bounded by the header-checked section sizes; a bad
// container sets bits of the status word and the kernel finishes normally.
//
// A coder C supplies (all static):
//   Tables                 its per-CTA tables (static shared memory), with members
//                          total_bits and n_words (32-bit words of the stream section)
//   Reader<Words>          a lane's reader over a word source, with reload()
//   kGbaseOffset           container offset of the group start bits
//   kTableBytes, kScratchBytes  dynamic shared memory of its lookup table and of the
//                          scratch its table build uses
//   chunk_words(K)         most stream words a well-formed chunk spans past its start
//   prepare(a, T)          check the header and fill T (every thread; false: rejected)
//   build(T, table, scratch)    fill the lookup table (every thread)
//   init(br, T, table, words, start), block(br, T, m, err) -> 8 BF16,
//   one(br, T, err) -> one exponent (peek current; reloads after),
//   done(br, clen, has_elements) -> whether the lane read exactly its chunk (a chunk of
//                          the ragged last group may hold no element)
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "bulk.cuh"
#include "dfx_common.cuh"

namespace dfx {
namespace {

// One CTA of 32 warps per SM.
template <int K>
struct DecodeShape {
    static constexpr int kWarps = 32;
    static constexpr int kThreads = kWarps * 32;
};

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

template <class C>
__device__ __forceinline__ GroupIndex load_index(const DecodeArgs& a, const typename C::Tables& T, uint64_t g,
                                                 unsigned lane, bool has_chunk) {
    const unsigned long long* gbase = reinterpret_cast<const unsigned long long*>(a.comp + C::kGbaseOffset);
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

// ---------------------------------------------------------------- word sources
//
// The global stream (with or without a bound clamp) or a warp's shared-memory copy of its
// group's slice of the stream.
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
    // Well-formed groups read inside the slice.  A corrupt one reads at most
    // chunk_words(K) + 2 words past a chunk start, into the other slice buffer or the
    // warp's m units that follow them: never outside the warp's own buffers.
    __device__ __forceinline__ uint32_t load(uint32_t i) const {
        uint32_t v;
        asm volatile("ld.shared.u32 %0, [%1];\n" : "=r"(v) : "r"(s + 4u * i));
        return v;
    }
};

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
__device__ __forceinline__ Slice plan_slice(uint32_t n_words, unsigned long long gb0, uint32_t span, bool ok) {
    Slice r;
    const uint32_t beg = ((uint32_t)(gb0 >> 5) * 4u) & ~15u;  // bytes into the stream section
    const uint32_t end = min((((uint32_t)((gb0 + span) >> 5) + 4u) * 4u + 15u) & ~15u, n_words * 4u);
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
template <class C, int K, class Reader>
__device__ __forceinline__ void decode_group_blocks(const DecodeArgs& a, const typename C::Tables& T, Reader* br,
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
                op[32u * (kMUnitBlocks * u + kk)] = C::block(*br, T, ld_shared_u2(mu + 32u * kk), err);
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
// load the index of its second group; needs only the coder's header tables, so it runs
// while the block builds its lookup table.  The warp has at least one full group.
template <class C, int K>
__device__ __forceinline__ void group_prologue(const DecodeArgs& a, const typename C::Tables& T, WarpBuffers<K>& wb,
                                               uint32_t g, uint32_t step, uint32_t n_full, unsigned lane,
                                               GroupState<K>& s) {
    if (lane == 0) {
        for (int i = 0; i < 2 + (int)kMUnits; i++) mbar_init(&wb.mbar[i]);
        fence_mbar_init();
        fence_proxy_async();
    }
    __syncwarp();
    s.mp = MPipe<K>{0u, g, step, (n_full - g + step - 1) / step};
    s.st = scan_index(load_index<C>(a, T, g, lane, true), lane);
    s.sl = plan_slice<SliceShape<K>::kWords>(T.n_words, s.st.gb0, s.st.span, s.st.ok);
    if (lane == 0) {
        // (the test hook leaves one copy out, so that its bounded wait runs out)
        const bool skip = (a.inject & DFX_INJECT_SKIP_SLICE_COPY) && g == a.g_begin;
        if (s.sl.staged && !skip) bulk_copy(wb.slice[0], a.comp + a.off_stream + 4u * s.sl.base, s.sl.bytes, &wb.mbar[0]);
        for (uint32_t u = 0; u < kMUnits; u++) s.mp.issue(a, wb, u);
    }
    s.g = g;
    s.gn = g + step;
    if (s.gn < n_full) s.idx_n = load_index<C>(a, T, s.gn, lane, true);
    s.b = 0;
    s.sphase = 0;
}

// Full groups, one warp at a time, from the state the prologue left.  While group g
// decodes, the stream slice of the warp's next group is copied into the other slice
// buffer, the index of the group after that is loaded, and the m units run kMUnits units
// (4 blocks each) ahead of the decode.
template <class C, int K>
__device__ void decode_full_groups(const DecodeArgs& a, const typename C::Tables& T, const uint32_t* table,
                                   WarpBuffers<K>& wb, GroupState<K>& s0, uint32_t step, uint32_t n_full,
                                   unsigned lane, uint32_t& err) {
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
            sl_n = plan_slice<kWords>(T.n_words, st_n.gb0, st_n.span, st_n.ok);
            if (lane == 0 && sl_n.staged)  // buffer b ^ 1 was released at the end of the previous group
                bulk_copy(wb.slice[b ^ 1], sbytes + 4u * sl_n.base, sl_n.bytes, &wb.mbar[b ^ 1]);
            if (gnn < n_full) idx_nn = load_index<C>(a, T, gnn, lane, true);
        }
        if (sl.staged) {
            if (!mbar_wait(&wb.mbar[b], (sphase >> b) & 1u)) err |= DFX_STATUS_TIMEOUT;
            sphase ^= 1u << b;
        }

        if (st.ok) {
            bool ok;
            if (sl.staged) {
                typename C::template Reader<SharedWords> br;
                C::init(br, T, table, SharedWords{smem_addr(wb.slice[b])}, (uint32_t)(st.start - 32ull * sl.base));
                decode_group_blocks<C, K>(a, T, &br, wb, mp, g, lane, err);
                ok = C::done(br, st.clen, true);
            } else {
                // A chunk reads at most chunk_words(K) + 2 words past its start; lane 31
                // starts last.  When that stays inside the stream the loads need no clamp.
                const uint32_t first = (uint32_t)(st.gb0 >> 5);
                const uint32_t last = __shfl_sync(kFull, (uint32_t)(st.start >> 5), 31);
                const uint32_t rel = (uint32_t)(st.start - 32ull * first);
                if (last + C::chunk_words(K) + 8u <= maxw) {
                    typename C::template Reader<GlobalWords> br;
                    C::init(br, T, table, GlobalWords{sw + first}, rel);
                    decode_group_blocks<C, K>(a, T, &br, wb, mp, g, lane, err);
                    ok = C::done(br, st.clen, true);
                } else {
                    typename C::template Reader<ClampedGlobalWords> br;
                    C::init(br, T, table, ClampedGlobalWords{sw + first, maxw - first}, rel);
                    decode_group_blocks<C, K>(a, T, &br, wb, mp, g, lane, err);
                    ok = C::done(br, st.clen, true);
                }
            }
            if (!ok) err |= DFX_STATUS_STREAM;
        } else {
            err |= DFX_STATUS_INDEX;
            // keeps the m pipeline in step
            decode_group_blocks<C, K>(a, T, (typename C::template Reader<SharedWords>*)nullptr, wb, mp, g, lane, err);
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
// that are below n (a prefix of the chunk, possibly empty).  Whole blocks take the block
// path; the lane's last, partial block is decoded code by code and stored element-wise.
template <class C, int K, class Reader>
__device__ __forceinline__ void decode_tail_blocks(const DecodeArgs& a, const typename C::Tables& T, Reader& br,
                                                   uint32_t g, unsigned lane, uint32_t& err) {
    const uint8_t* mplane = a.comp + a.off_m;
    for (uint32_t k = 0; k < K / 8; k++) {
        const uint64_t x0 = block_element(g, K, k, lane);
        if (x0 + 8 <= a.n) {
            reinterpret_cast<uint4*>(a.out)[(x0 - a.out_first) / 8] =
                C::block(br, T, __ldg(reinterpret_cast<const uint2*>(mplane + x0)), err);
            continue;
        }
        if (x0 < a.n) {
            const uint32_t cnt = (uint32_t)(a.n - x0);
            br.reload();
            for (uint32_t j = 0; j < cnt; j++) {  // decode and store one element at a time
                const uint32_t ex = C::one(br, T, err);
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
template <class C, int K>
__device__ void decode_tail_group(const DecodeArgs& a, const typename C::Tables& T, const uint32_t* table,
                                  WarpBuffers<K>& wb, uint32_t g, unsigned lane, uint32_t& err) {
    const GroupStart gs = scan_index(load_index<C>(a, T, g, lane, true), lane);
    if (!gs.ok) {
        err |= DFX_STATUS_INDEX;
        return;
    }
    const Slice sl = plan_slice<SliceShape<K>::kWords>(T.n_words, gs.gb0, gs.span, gs.ok);
    const bool has_elements = block_element(g, K, 0, lane) < a.n;
    bool ok;
    if (sl.staged) {
        const uint4* src = reinterpret_cast<const uint4*>(a.comp + a.off_stream + 4u * sl.base);
        uint4* dst = reinterpret_cast<uint4*>(wb.slice[0]);
        for (uint32_t c = lane; c < sl.bytes / 16u; c += 32) dst[c] = __ldg(src + c);
        __syncwarp();
        typename C::template Reader<SharedWords> br;
        C::init(br, T, table, SharedWords{smem_addr(wb.slice[0])}, (uint32_t)(gs.start - 32ull * sl.base));
        decode_tail_blocks<C, K>(a, T, br, g, lane, err);
        ok = C::done(br, gs.clen, has_elements);
    } else {
        const uint32_t* sw = reinterpret_cast<const uint32_t*>(a.comp + a.off_stream);
        const uint32_t maxw = T.n_words - 1;
        const uint32_t first = (uint32_t)(gs.gb0 >> 5);
        typename C::template Reader<ClampedGlobalWords> br;
        C::init(br, T, table, ClampedGlobalWords{sw + first, maxw - first}, (uint32_t)(gs.start - 32ull * first));
        decode_tail_blocks<C, K>(a, T, br, g, lane, err);
        ok = C::done(br, gs.clen, has_elements);
    }
    if (!ok) err |= DFX_STATUS_STREAM;
}

// The decode kernels are launched as programmatic dependents of the work before them in
// the stream: a CTA may be scheduled while the previous kernel is still finishing (back-to-
// back decodes then lose no time between launches).  It waits for that work to complete,
// memory included, before it reads anything in global memory, or, when the plan says the
// preceding kernel does not write the container (DFX_DECODE_EARLY_READ), only before its
// first output write: its header checks, table build and first copies then overlap the
// preceding kernel's last groups.
__device__ __forceinline__ void wait_prior_grid() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }
__device__ __forceinline__ void enter_dependent(const DecodeArgs& a) {
    asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
    if (!a.early) wait_prior_grid();
}

// One tensor's decode by `ctas` CTAs of which this is number `cta`: the body of both
// kernels below.
template <class C, int K>
__device__ __forceinline__ void decode_tensor(const DecodeArgs& a, uint32_t cta, uint32_t ctas) {
    constexpr int kDecodeWarps = DecodeShape<K>::kWarps;
    __shared__ typename C::Tables T;
    // dynamic shared memory: the coder's lookup table, its build scratch, then one buffer
    // per warp
    extern __shared__ __align__(16) uint8_t dyn_smem[];
    uint32_t* table = reinterpret_cast<uint32_t*>(dyn_smem);
    uint8_t* scratch = dyn_smem + C::kTableBytes;
    uint8_t* warp_area = dyn_smem + C::kTableBytes + C::kScratchBytes;
    const uint32_t n_full = (a.n % (32ull * K) == 0) ? a.n_group : a.n_group - 1;
    const uint32_t full_end = min(n_full, a.g_end);  // full groups to decode: [g_begin, full_end)
    {
        // start fetching each warp's first group (index entries, m plane) into L2 while
        // the tables are built
        const uint32_t g0 = a.g_begin + cta + ctas * (threadIdx.x >> 5);
        if ((threadIdx.x & 31) == 0 && g0 < full_end) {
            prefetch_line_l2(a.comp + C::kGbaseOffset + 8ull * g0);
            prefetch_line_l2(a.comp + a.off_clen + 64ull * g0);
            prefetch_line_l2(a.comp + a.off_clen + 64ull * g0 + 63);
            prefetch_l2(a.comp + a.off_m + (uint64_t)g0 * (32u * K), 32u * K);
        }
    }
    if (!C::prepare(a, T)) return;
    const unsigned warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    WarpBuffers<K>& wb = *reinterpret_cast<WarpBuffers<K>*>(warp_area + warp * warp_buffer_bytes<K>());
    uint32_t err = 0;
    const uint32_t step = ctas * kDecodeWarps;
    // groups are dealt to the CTAs (one per SM) in turn and each CTA's to its warps in
    // turn, highest warp first, so that every SM gets the same number of groups within
    // one; the warps that get one group more than the rest are the highest-numbered ones,
    // which the schedulers favour (they finish their groups first)
    const uint32_t gw = a.g_begin + cta + ctas * (kDecodeWarps - 1 - warp);
    GroupState<K> gs;
    if (gw < full_end) group_prologue<C, K>(a, T, wb, gw, step, full_end, lane, gs);
    C::build(T, table, scratch);
    if (a.early) wait_prior_grid();  // before the first output write
    if (gw < full_end) decode_full_groups<C, K>(a, T, table, wb, gs, step, full_end, lane, err);
    // the ragged last group, by the warp whose sequence it would continue
    if (n_full < a.n_group && n_full >= a.g_begin && n_full < a.g_end && gw == a.g_begin + (n_full - a.g_begin) % step)
        decode_tail_group<C, K>(a, T, table, wb, n_full, lane, err);
    if (err) atomicOr(a.status, err);
}

template <class C, int K>
__global__ void __launch_bounds__(DecodeShape<K>::kThreads, 1) k_decode(DecodeArgs a) {
    enter_dependent(a);
    decode_tensor<C, K>(a, blockIdx.x, gridDim.x);
}

// Several tensors in one launch (all with the same K and coder): each CTA decodes its
// share of one tensor, so it builds that tensor's tables once.
template <class C, int K>
__global__ void __launch_bounds__(DecodeShape<K>::kThreads, 1) k_decode_batch(const __grid_constant__ BatchArgs b) {
    uint32_t i = 0;
    while (i + 1 < b.count && blockIdx.x >= b.cta_begin[i + 1]) i++;
    enter_dependent(b.t[i]);
    decode_tensor<C, K>(b.t[i], blockIdx.x - b.cta_begin[i], b.cta_begin[i + 1] - b.cta_begin[i]);
}

template <class C, int K>
constexpr size_t dyn_smem_bytes() {
    return C::kTableBytes + C::kScratchBytes + DecodeShape<K>::kWarps * warp_buffer_bytes<K>();
}

template <class C, int K>
int blocks_per_sm() {
    int b = 0;
    if (cudaFuncSetAttribute(k_decode<C, K>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dyn_smem_bytes<C, K>()) !=
        cudaSuccess)
        return 1;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, k_decode<C, K>, DecodeShape<K>::kThreads,
                                                      dyn_smem_bytes<C, K>()) != cudaSuccess)
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

// Launch with programmatic stream serialisation (the kernel starts with enter_dependent).
template <class Kern, class Arg>
cudaError_t launch_programmatic(Kern* kernel, int grid, int threads, size_t smem, cudaStream_t s, const Arg& arg) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3((unsigned)threads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, arg);
}

template <class C, int K>
cudaError_t launch_k(const DecodeArgs& a, int grid, cudaStream_t s) {
    static bool attr_set[64] = {};
    const cudaError_t e = allow_smem(k_decode<C, K>, dyn_smem_bytes<C, K>(), attr_set);
    if (e != cudaSuccess) return e;
    return launch_programmatic(k_decode<C, K>, grid, DecodeShape<K>::kThreads, dyn_smem_bytes<C, K>(), s, a);
}

template <class C, int K>
cudaError_t launch_batch_k(const BatchArgs& b, cudaStream_t s) {
    static bool attr_set[64] = {};
    const cudaError_t e = allow_smem(k_decode_batch<C, K>, dyn_smem_bytes<C, K>(), attr_set);
    if (e != cudaSuccess) return e;
    return launch_programmatic(k_decode_batch<C, K>, (int)b.cta_begin[b.count], DecodeShape<K>::kThreads,
                               dyn_smem_bytes<C, K>(), s, b);
}

// The launchers of one coder for K = 32, 64, 128.
template <class C>
cudaError_t launch_coder(const DecodeArgs& a, int grid, cudaStream_t s) {
    switch (a.K) {
        case 32: return launch_k<C, 32>(a, grid, s);
        case 64: return launch_k<C, 64>(a, grid, s);
        case 128: return launch_k<C, 128>(a, grid, s);
        default: return cudaErrorInvalidValue;
    }
}
template <class C>
cudaError_t launch_batch_coder(const BatchArgs& b, uint32_t K, cudaStream_t s) {
    if (b.count == 0 || b.count > kMaxBatch || b.cta_begin[b.count] == 0) return cudaErrorInvalidValue;
    switch (K) {
        case 32: return launch_batch_k<C, 32>(b, s);
        case 64: return launch_batch_k<C, 64>(b, s);
        case 128: return launch_batch_k<C, 128>(b, s);
        default: return cudaErrorInvalidValue;
    }
}
template <class C>
int blocks_per_sm_coder(uint32_t K) {
    switch (K) {
        case 32: return blocks_per_sm<C, 32>();
        case 64: return blocks_per_sm<C, 64>();
        case 128: return blocks_per_sm<C, 128>();
        default: return 1;
    }
}

}  // namespace
}  // namespace dfx
