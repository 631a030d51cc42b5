// encode.cu -- GPU encoder for DFX1 containers (sm_100a).
//
// Passes, all stream-ordered on the caller's stream:
//   0. zero the container's index region and the workspace words the pack counts in;
//   1. k_histogram      exponent histogram: input streamed by the bulk-copy engine, counts
//                       of the 16 most frequent neighbouring values in registers;
//   2. k_build_codebook one CTA: package-merge code lengths (limit max_len), canonical codes,
//                       len[256], the constant header fields and the stream's bit count;
//   3. k_pack_fused     one warp per group, groups in ticket order: the group's input read
//                       once (a group's elements come in 8-element blocks, block b belongs
//                       to chunk b mod 32, so lane i reads blocks i, i+32, ...: 16-byte
//                       loads, 512 contiguous bytes per warp instruction), per block its 8
//                       codes joined into one word and its mantissa+sign bytes (mantissa * 2
//                       + the sign of the pair partner, element x ^ 1) written in element
//                       order, per chunk its code bits (clen), the group's start bit by a
//                       decoupled look-back over the groups before it (gbase, total_bits,
//                       total_bytes), and the joined codes packed MSB-first into 32-bit
//                       words; every stream word is written once (the word two groups share
//                       by the second of them to finish), then the container's zero
//                       padding; the bytes past the container are not written.
// The tANS coder shares pass 1 and k_group_scan (a one-CTA scan of per-group sums); its
// passes 2, 3 and 5 are in encode_tans.cu.
// The method: frequent exponent values get short codes ("DFloat11: lossless LLM
// compression for GPU", aikraft.ru blog, section 02); the exact code and layout rules
// are the ones stated in include/dfx.h.
#include <cuda_runtime.h>
#include <stdint.h>

#include "bulk.cuh"
#include "dfx_common.cuh"

namespace dfx {
namespace {

__device__ __forceinline__ uint32_t warp_incl_scan(uint32_t v, unsigned lane) {
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        uint32_t y = __shfl_up_sync(kFull, v, d);
        if (lane >= (unsigned)d) v += y;
    }
    return v;
}

// Programmatic dependent launch within the encode: the code book and the pack are launched
// while the kernel before them runs and wait for its completion (and memory) here.
__device__ __forceinline__ void wait_for_previous_kernel() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }
__device__ __forceinline__ void allow_next_kernel() { asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory"); }
template <class Kern, class... Args>
cudaError_t launch_dependent(Kern* kernel, unsigned grid, unsigned threads, size_t smem, cudaStream_t s, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(threads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}

__device__ __forceinline__ unsigned long long warp_incl_scan64(unsigned long long v, unsigned lane) {
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        unsigned long long y = __shfl_up_sync(kFull, v, d);
        if (lane >= (unsigned)d) v += y;
    }
    return v;
}

// ---------------------------------------------------------------- 1. histogram
//
// One CTA of 32 warps per SM.  The input's 16-byte units (8 exponents each) are cut into
// chunks of 192 units (3 KiB); each warp takes a contiguous run of chunks and streams them
// into its shared-memory buffers with the bulk-copy engine, kHistBufs chunks in flight,
// so the bytes in flight do not depend on registers.  The exponents of a weight tensor
// crowd into a few neighbouring values: each CTA counts its warps' first chunks into a
// shared histogram and picks the 16 consecutive exponents [b, b + 16) with the most of
// that sample.  From then on a lane counts the values in that window in registers:
// 4-bit counters, eight per 32-bit word (value b + d adds 1 << 4d to the first word for
// d < 8 and 1 << 4(d - 8) to the second for 8 <= d < 16).  The two values of a 32-bit
// input word take one shared-memory load of the increments of the pair (a 17 x 17 table,
// offset 16 standing for "outside") instead of shifts.  The loop leans on the integer
// (ALU) pipe, so its field extractions are multiplications by powers of two, which run on
// the FMA pipe: x * 2^k is x << k and the high word of x * 2^(32 - k) is x >> k.  After
// every unit (at most 8 per counter) the nibbles are spread
// into 8-bit counters, after kHistFold chunks those into 16-bit counters, and these into
// the shared histogram at the end.  Values outside the window are rare: the warp checks
// once per unit whether any lane met one, and only then takes shared-memory atomics.
constexpr int kHistWarps = 32;
constexpr uint32_t kHistChunkUnits = 192;  // 16-byte units per chunk (3 KiB)
constexpr uint32_t kHistBufs = 2;          // chunks in flight per warp
constexpr uint32_t kHistFold = 5;          // chunks between byte folds (5 x 48 < 256)
constexpr uint32_t kHistHalfFolds = 256;   // byte folds between half-word flushes (256 x 240 < 65536)

struct HistWarpBuffers {
    uint4 chunk[kHistBufs][kHistChunkUnits];
    unsigned long long bar[kHistBufs];
};
constexpr size_t kHistSmem = kHistWarps * sizeof(HistWarpBuffers);

// Spread two words of 4-bit counters (values b .. b + 15) into four words of 8-bit counters:
// c8[0] takes values b + {0, 2, 4, 6}, c8[1] b + {1, 3, 5, 7}, c8[2] and c8[3] the same for
// b + 8 ..
// x16 = 2^28: the high nibbles move down by the high word of a multiplication.
__device__ __forceinline__ void fold_nibbles(uint32_t& n0, uint32_t& n1, uint32_t (&c8)[4], uint32_t x16) {
    c8[0] += n0 & 0x0F0F0F0Fu;
    c8[1] = __umulhi(n0 & 0xF0F0F0F0u, x16) + c8[1];
    c8[2] += n1 & 0x0F0F0F0Fu;
    c8[3] = __umulhi(n1 & 0xF0F0F0F0u, x16) + c8[3];
    n0 = n1 = 0u;
}
// Spread the 8-bit counters into 16-bit ones: c16[2 w + h] holds byte h and byte h + 2 of
// c8[w] (values b + {0, 4}, {2, 6}, {1, 5}, {3, 7}, {8, 12}, ...).
__device__ __forceinline__ void fold_bytes(uint32_t (&c8)[4], uint32_t (&c16)[8]) {
#pragma unroll
    for (int w = 0; w < 4; w++) {
        c16[2 * w] += c8[w] & 0x00FF00FFu;
        c16[2 * w + 1] += (c8[w] >> 8) & 0x00FF00FFu;
        c8[w] = 0u;
    }
}
// The value b + d that half h (0: low, 1: high) of c16[i] counts.
__host__ __device__ constexpr uint32_t c16_value(int i, int h) {
    return 8u * ((i >> 2) & 1) + 2u * (i & 1) + ((i >> 1) & 1) + 4u * h;
}

__global__ void __launch_bounds__(kHistWarps * 32, 1) k_histogram(const uint16_t* __restrict__ in, uint64_t n,
                                                                  unsigned long long* __restrict__ counts,
                                                                  uint32_t* status) {
    __shared__ uint32_t h[256];
    __shared__ uint32_t window;
    __shared__ uint32_t pow2[4];         // 2^17, 2, 2^8, 2^28, read back so they stay multiplications
    __shared__ uint2 pair_add[17 * 17];  // (d0, d1) -> the two counter words' increments
    extern __shared__ __align__(16) uint8_t hist_smem[];
    allow_next_kernel();  // the code book may be scheduled; it waits for this kernel to end
    const unsigned warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    HistWarpBuffers& wb = reinterpret_cast<HistWarpBuffers*>(hist_smem)[warp];
    for (int i = threadIdx.x; i < 256; i += blockDim.x) h[i] = 0;
    const uint64_t units = n / 8;
    const uint64_t chunks = (units + kHistChunkUnits - 1) / kHistChunkUnits;
    const uint64_t nw = (uint64_t)gridDim.x * kHistWarps, wg = (uint64_t)blockIdx.x * kHistWarps + warp;
    const uint64_t c0 = chunks * wg / nw;
    const uint32_t nc = (uint32_t)(chunks * (wg + 1) / nw - c0);  // this warp's chunks c0 .. c0 + nc - 1
    const uint4* in4 = reinterpret_cast<const uint4*>(in);
    auto chunk_units = [&](uint32_t k) -> uint32_t {
        const uint64_t left = units - (c0 + k) * kHistChunkUnits;
        return left < kHistChunkUnits ? (uint32_t)left : kHistChunkUnits;
    };
    auto issue = [&](uint32_t k) {  // lane 0: chunk k of the warp into buffer k % kHistBufs
        bulk_copy(wb.chunk[k % kHistBufs], in4 + (c0 + k) * kHistChunkUnits, 16u * chunk_units(k),
                  &wb.bar[k % kHistBufs]);
    };
    if (lane == 0) {
        for (uint32_t i = 0; i < kHistBufs; i++) mbar_init(&wb.bar[i]);
        fence_mbar_init();
        for (uint32_t k = 0; k < kHistBufs && k < nc; k++) issue(k);
    }
    __syncthreads();  // h zeroed
    uint32_t err = 0;
    if (nc > 0) {  // the sample: every warp's first chunk (its counts are kept)
        if (!mbar_wait(&wb.bar[0], 0)) err |= DFX_STATUS_TIMEOUT;
        const uint32_t nu = chunk_units(0);
        for (uint32_t u = lane; u < nu; u += 32) {
            const uint4 v = wb.chunk[0][u];
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int k = 0; k < 8; k++) atomicAdd(&h[(w[k >> 1] >> (16 * (k & 1) + 7)) & 0xFFu], 1u);
        }
        __syncwarp();
        if (lane == 0 && kHistBufs < nc) {
            fence_proxy_async();
            issue(kHistBufs);
        }
    }
    __syncthreads();
    if (threadIdx.x < 32) {  // the window with the largest sample mass: lane l tries b = l + 32 j
        uint32_t best = 0, best_b = 0;
        for (uint32_t b = threadIdx.x; b <= 240; b += 32) {
            uint32_t m = 0;
            for (uint32_t k = 0; k < 16; k++) m += h[b + k];
            if (m > best) {
                best = m;
                best_b = b;
            }
        }
#pragma unroll
        for (int d = 16; d >= 1; d >>= 1) {
            const uint32_t ob = __shfl_xor_sync(kFull, best, d), obb = __shfl_xor_sync(kFull, best_b, d);
            if (ob > best || (ob == best && obb < best_b)) {
                best = ob;
                best_b = obb;
            }
        }
        if (threadIdx.x == 0) window = best_b;
    }
    // one value at window offset d < 16 adds 1 << 4d to counter word 0 (d < 8) or
    // 1 << 4 (d - 8) to word 1; offset 16 stands for any value outside the window
    for (uint32_t i = threadIdx.x; i < 17 * 17; i += blockDim.x) {
        uint2 v = make_uint2(0u, 0u);
        for (uint32_t d : {i / 17, i % 17}) {
            if (d < 8) v.x += 1u << (4 * d);
            else if (d < 16) v.y += 1u << (4 * (d - 8));
        }
        pair_add[i] = v;
    }
    if (threadIdx.x == 0) {
        pow2[0] = 1u << 17;
        pow2[1] = 2u;
        pow2[2] = 1u << 8;
        pow2[3] = 1u << 28;
    }
    __syncthreads();
    const uint32_t b = window;
    // a word's two window offsets (e - b) mod 256, which is 16 or more for every e outside
    // [b, b + 16) since b <= 240: the low exponent field (bits 7..14) is moved to the top
    // byte by * 2^17, the high one (bits 23..30) by * 2, b is subtracted from the top byte
    // alone (cb has no lower bits) and the top byte taken by the high word of * 2^8
    const uint32_t x17 = pow2[0], x1 = pow2[1], x8 = pow2[2], x28 = pow2[3];
    const uint32_t cb = 0u - (b << 24);
    uint32_t n0 = 0u, n1 = 0u, c8[4] = {0u, 0u, 0u, 0u}, c16[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
    uint32_t since = 0, folds = 0;
    for (uint32_t k = 1; k < nc; k++) {
        const uint32_t slot = k % kHistBufs;
        if (!mbar_wait(&wb.bar[slot], (k / kHistBufs) & 1u)) err |= DFX_STATUS_TIMEOUT;
        const uint32_t nu = chunk_units(k);
        uint4 v[kHistChunkUnits / 32];
#pragma unroll
        for (uint32_t j = 0; j < kHistChunkUnits / 32; j++)
            v[j] = (lane + 32 * j < nu) ? wb.chunk[slot][lane + 32 * j] : make_uint4(0, 0, 0, 0);
        __syncwarp();
        if (lane == 0 && k + kHistBufs < nc) {
            fence_proxy_async();
            issue(k + kHistBufs);
        }
        if (nu == kHistChunkUnits) {
#pragma unroll
            for (uint32_t j = 0; j < kHistChunkUnits / 32; j++) {
                const uint32_t w[4] = {v[j].x, v[j].y, v[j].z, v[j].w};
                uint32_t outside = 0;
#pragma unroll
                for (int q = 0; q < 4; q++) {
                    const uint32_t d0 = __umulhi(w[q] * x17 + cb, x8), d1 = __umulhi(w[q] * x1 + cb, x8);
                    const uint2 t = pair_add[17u * min(d0, 16u) + min(d1, 16u)];  // 16: outside
                    n0 += t.x;
                    n1 += t.y;
                    outside |= d0 | d1;
                }
                fold_nibbles(n0, n1, c8, x28);
                if (__any_sync(kFull, outside >= 16u) && outside >= 16u) {
#pragma unroll
                    for (int q = 0; q < 8; q++) {
                        const uint32_t e = (w[q >> 1] >> (16 * (q & 1) + 7)) & 0xFFu;
                        if (e - b >= 16u) atomicAdd(&h[e], 1u);
                    }
                }
            }
            if (++since == kHistFold) {
                fold_bytes(c8, c16);
                since = 0;
                if (++folds == kHistHalfFolds) {
#pragma unroll
                    for (int i = 0; i < 8; i++) {
                        if (c16[i] & 0xFFFFu) atomicAdd(&h[b + c16_value(i, 0)], c16[i] & 0xFFFFu);
                        if (c16[i] >> 16) atomicAdd(&h[b + c16_value(i, 1)], c16[i] >> 16);
                        c16[i] = 0u;
                    }
                    folds = 0;
                }
            }
        } else {  // the last chunk of the input, partial: shared-memory atomics
            for (uint32_t j = 0; j < kHistChunkUnits / 32; j++) {
                if (lane + 32 * j >= nu) continue;
                const uint32_t w[4] = {v[j].x, v[j].y, v[j].z, v[j].w};
                for (int q = 0; q < 8; q++) atomicAdd(&h[(w[q >> 1] >> (16 * (q & 1) + 7)) & 0xFFu], 1u);
            }
        }
    }
    fold_bytes(c8, c16);
#pragma unroll
    for (int i = 0; i < 8; i++) {
        if (c16[i] & 0xFFFFu) atomicAdd(&h[b + c16_value(i, 0)], c16[i] & 0xFFFFu);
        if (c16[i] >> 16) atomicAdd(&h[b + c16_value(i, 1)], c16[i] >> 16);
    }
    if (blockIdx.x == 0 && threadIdx.x < (n & 7)) atomicAdd(&h[(in[units * 8 + threadIdx.x] >> 7) & 0xFFu], 1u);
    if (err) atomicOr(status, err);
    __syncthreads();
    wait_for_previous_kernel();  // the counts are zeroed by the kernel before this one
    for (int k = threadIdx.x; k < 256; k += blockDim.x)
        if (h[k]) atomicAdd(&counts[k], (unsigned long long)h[k]);
}

// ---------------------------------------------------------------- 2. code book
//
// Package-merge, computed level by level with merge ranks instead of explicit
// package trees.  List 0 is the leaves sorted by (count, symbol).  List j merges
// the leaves with the packages of list j-1 (pairs of consecutive items, a trailing
// odd item dropped), a leaf ahead of a package of equal weight.  A leaf's rank in
// list j is its index plus the number of packages lighter than it; a package's
// rank is its index plus the number of leaves not heavier than it.  The first
// 2m-2 items of the last list are selected.  Selected items of every list form a
// prefix, and the packages inside the prefix of list j are its first p_j packages,
// which expand to the first 2 p_j items of list j-1.  So walking back from the
// last list, q_j = number of leaves in the selected prefix of list j, and the
// length of the leaf of sorted rank i is the number of lists with i < q_j.
//
// The kernel is one CTA and a chain of short dependent steps, so it is written for
// latency: the used symbols are compacted first (the sort compares m counts, not 256);
// a package's weight is summed from list j-1 where it is needed, so a level takes one
// barrier; with m <= 128 the leaves' ranks and the packages' ranks are computed by
// different warps; and a rank search probes 8 x 8 entries when the list has at most 64.

// The number of the first n (<= 256) entries of the ascending sequence v(0), v(1), ...
// that are below w (or, with Le, not above it), in two dependent rounds of probes instead
// of a binary search's eight: the last entries of B blocks of B first, then the B entries
// of the one block that straddles w (B * B >= n).
template <int B, bool Le, class V>
__device__ __forceinline__ int count_sorted_in(V v, int n, unsigned long long w) {
    auto in = [&](unsigned long long x) { return Le ? x <= w : x < w; };
    int blocks = 0;  // whole B-entry blocks below w (their last entry is)
#pragma unroll
    for (int i = 0; i < B; i++) blocks += (B * i + B - 1 < n && in(v(B * i + B - 1))) ? 1 : 0;
    int r = B * blocks;
#pragma unroll
    for (int k = 0; k < B; k++) {
        const int i = B * blocks + k;
        r += (i < n && in(v(i))) ? 1 : 0;
    }
    return r;
}
template <bool Le, class V>
__device__ __forceinline__ int count_sorted(V v, int n, unsigned long long w) {
    return n <= 64 ? count_sorted_in<8, Le>(v, n, w) : count_sorted_in<16, Le>(v, n, w);
}

__global__ void __launch_bounds__(256) k_build_codebook(EncodeArgs a) {
    __shared__ unsigned long long ucnt[256];  // the used symbols' counts, in symbol order
    __shared__ unsigned long long leafw[256];
    __shared__ uint8_t leafsym[256];
    __shared__ unsigned long long lw[2][512];
    __shared__ uint16_t leafpos[kMaxLenLimit][256];
    __shared__ int qsel[kMaxLenLimit];
    __shared__ uint8_t lens[256];
    __shared__ uint32_t nlen[kMaxLenLimit + 1];
    __shared__ uint32_t firstc[kMaxLenLimit + 1];
    __shared__ uint8_t wlen[8][kMaxLenLimit + 1];  // symbols of each length per 32-symbol slice
    __shared__ uint32_t wused[8];                  // used symbols per 32-symbol slice

    allow_next_kernel();
    wait_for_previous_kernel();  // the histogram's counts
    const int t = threadIdx.x;
    const unsigned lane = t & 31, warp = t >> 5;
    const int L = (int)a.max_len;
    const unsigned long long c = a.ws_counts[t];
    lens[t] = 0;
    if (t <= (int)kMaxLenLimit) nlen[t] = 0;
    if (t < 8 * (int)(kMaxLenLimit + 1)) (&wlen[0][0])[t] = 0;
    const bool used = c > 0;
    const unsigned used_bits = __ballot_sync(kFull, used);
    if (lane == 0) wused[warp] = __popc(used_bits);
    __syncthreads();
    int m = 0, idx = __popc(used_bits & ((1u << lane) - 1u));  // idx: the symbol's place among the used
#pragma unroll
    for (int w = 0; w < 8; w++) {
        m += wused[w];
        idx += (w < (int)warp) ? wused[w] : 0;
    }
    if (used) ucnt[idx] = c;
    __syncthreads();

    if (m == 1) {
        // one exponent value: it and a phantom partner both get 1-bit codes
        if (used) {
            lens[t] = 1;
            lens[t == 0 ? 1 : 0] = 1;
        }
    } else if (m >= 2) {
        if (used) {  // the rank by (count, symbol); the used symbols are in symbol order
            int r = 0;
#pragma unroll 4
            for (int k = 0; k < m; k++) {
                const unsigned long long ck = ucnt[k];
                r += (ck < c || (ck == c && k < idx)) ? 1 : 0;
            }
            leafw[r] = c;
            lw[0][r] = c;
            leafsym[r] = (uint8_t)t;
        }
        __syncthreads();
        // leaf t and package pk of each list; pk = t - 128 puts the packages on other warps
        const int pk = m <= 128 ? t - 128 : t;
        const unsigned long long leaf = t < m ? leafw[t] : 0ull;
        int size = m;
        for (int j = 1; j < L; j++) {
            const unsigned long long* prev = lw[(j - 1) & 1];
            unsigned long long* cur = lw[j & 1];
            const int np = size / 2;
            if (t < m) {
                const int lo = count_sorted<false>([&](int i) { return prev[2 * i] + prev[2 * i + 1]; }, np, leaf);
                cur[t + lo] = leaf;  // after the packages lighter than the leaf
                leafpos[j][t] = (uint16_t)(t + lo);
            }
            if (pk >= 0 && pk < np) {
                const unsigned long long w = prev[2 * pk] + prev[2 * pk + 1];
                cur[pk + count_sorted<true>([&](int i) { return leafw[i]; }, m, w)] = w;  // after the leaves not heavier
            }
            size = m + np;
            __syncthreads();
        }
        if (t < 32) {  // one warp: the leaves among the first s items of each list, last list first
            int s = 2 * m - 2;
            const int slices = (m + 31) / 32;
            for (int j = L - 1; j >= 1; j--) {
                int lo = 0;
                for (int k = 0; k < slices; k++) {
                    const int i = t + 32 * k;
                    lo += __popc(__ballot_sync(kFull, i < m && leafpos[j][i] < s));
                }
                if (t == 0) qsel[j] = lo;
                s = 2 * (s - lo);
            }
            if (t == 0) qsel[0] = s;
        }
        __syncthreads();
        if (t < m) {
            int l = 0;
            for (int j = 0; j < L; j++) l += (t < qsel[j]);
            lens[leafsym[t]] = (uint8_t)l;
        }
    }
    __syncthreads();

    // canonical codes: first code per length, then rank among equal lengths by symbol
    const uint32_t l = lens[t];
    if (l) atomicAdd(&nlen[l], 1u);
    // rank of the symbol among those of its length: lower lanes of its warp now, the
    // counts of lower warps after the barrier
    const unsigned peers = __match_any_sync(kFull, l), below = peers & ((1u << lane) - 1u);
    if (l && below == 0) wlen[warp][l] = (uint8_t)__popc(peers);
    __syncthreads();
    if (t == 0) {
        uint32_t code = 0;
        for (int k = 1; k <= (int)kMaxLenLimit; k++) {
            firstc[k] = code;
            code = (code + nlen[k]) << 1;
        }
    }
    __syncthreads();
    uint32_t code = 0;
    if (l) {
        uint32_t r = __popc(below);
        for (unsigned w = 0; w < warp; w++) r += wlen[w][l];
        code = firstc[l] + r;
    }
    a.ws_code[t] = code;
    a.ws_len[t] = (uint8_t)l;
    a.out[kOffLen + t] = (uint8_t)l;
    // the stream's bit count (for the container's zero padding after the stream): a sum
    // per warp, then over the warps
    __shared__ unsigned long long wbits[8];
    unsigned long long tb = l ? c * l : 0ull;
#pragma unroll
    for (int d = 16; d >= 1; d >>= 1) tb += __shfl_xor_sync(kFull, tb, d);
    if (lane == 0) wbits[warp] = tb;
    __syncthreads();
    if (t == 0) {
        unsigned long long total_bits = 0;
        for (int w = 0; w < 8; w++) total_bits += wbits[w];
        *reinterpret_cast<unsigned long long*>(reinterpret_cast<uint8_t*>(a.ws_counts) + kWsTotalBits) = total_bits;
    }

    if (t == 0) {
        uint8_t* h = a.out;
        *reinterpret_cast<uint32_t*>(h + 0) = 0x31584644u;  // "DFX1"
        *reinterpret_cast<uint16_t*>(h + 4) = 1;
        *reinterpret_cast<uint16_t*>(h + 6) = (uint16_t)kHeaderBytes;
        *reinterpret_cast<unsigned long long*>(h + 8) = a.n;
        *reinterpret_cast<uint32_t*>(h + 32) = a.K;
        *reinterpret_cast<uint32_t*>(h + 36) = a.G;
        *reinterpret_cast<uint32_t*>(h + 40) = a.n_chunk;
        *reinterpret_cast<uint32_t*>(h + 44) = a.n_group;
        *reinterpret_cast<unsigned long long*>(h + 48) = a.off_m;
        *reinterpret_cast<uint32_t*>(h + 56) = a.max_len;
        *reinterpret_cast<uint32_t*>(h + 60) = 0;
    }
}

// ---------------------------------------------------------------- group scan (tANS; empty tensors)

constexpr int kScanThreads = 1024;
constexpr int kScanItems = 16;  // four 16-byte loads per thread per round

__global__ void __launch_bounds__(kScanThreads) k_group_scan(EncodeArgs a) {
    __shared__ unsigned long long wsum[32];
    const unsigned t = threadIdx.x, lane = t & 31, warp = t >> 5;
    unsigned long long* gbase = reinterpret_cast<unsigned long long*>(a.out + a.off_gbase);
    unsigned long long carry = 0;
    for (uint64_t base = 0; base < a.n_group; base += (uint64_t)kScanThreads * kScanItems) {
        const uint64_t i = base + (uint64_t)t * kScanItems;
        uint32_t v[kScanItems];
        unsigned long long local = 0;
        if (i + kScanItems <= a.n_group) {  // the group sums start 16-byte aligned in the workspace
            const uint4* q = reinterpret_cast<const uint4*>(a.ws_group_bits + i);
#pragma unroll
            for (int k = 0; k < kScanItems / 4; k++) {
                const uint4 x = q[k];
                v[4 * k] = x.x;
                v[4 * k + 1] = x.y;
                v[4 * k + 2] = x.z;
                v[4 * k + 3] = x.w;
            }
        } else {
#pragma unroll
            for (int k = 0; k < kScanItems; k++) v[k] = (i + k < a.n_group) ? a.ws_group_bits[i + k] : 0u;
        }
#pragma unroll
        for (int k = 0; k < kScanItems; k++) local += v[k];
        const unsigned long long incl = warp_incl_scan64(local, lane);
        if (lane == 31) wsum[warp] = incl;
        __syncthreads();
        if (warp == 0) wsum[lane] = warp_incl_scan64(wsum[lane], lane);
        __syncthreads();
        unsigned long long run = carry + (warp ? wsum[warp - 1] : 0ull) + incl - local;
#pragma unroll
        for (int k = 0; k < kScanItems; k++)
            if (i + k < a.n_group) {
                gbase[i + k] = run;
                run += v[k];
            }
        carry += wsum[31];
        __syncthreads();
    }
    if (t == 0) {
        gbase[a.n_group] = carry;
        *reinterpret_cast<unsigned long long*>(a.out + 16) = carry;
        *reinterpret_cast<unsigned long long*>(a.out + 24) = a.off_stream + stream_bytes(carry);
    }
}

// ---------------------------------------------------------------- bit writers

// Where a chunk's packed words go when pack_chunk writes them straight to the stream in
// global memory: the first word of a chunk and its last, partial word may hold bits of
// the neighbouring chunks and are OR-ed in; the words between belong to the chunk alone.
struct GlobalSink {
    uint32_t* stream;
    __device__ __forceinline__ void shared_word(uint64_t wi, uint32_t v) const { atomicOr(stream + wi, v); }
    __device__ __forceinline__ void own_word(uint64_t wi, uint32_t v) const { stream[wi] = v; }
};

template <class Sink>
struct BitWriter {
    Sink sink;
    uint64_t wi;     // index of the word being assembled
    uint32_t fill;   // bits already in `cur`
    uint32_t cur;
    bool first;      // the first emitted word may hold bits of the previous chunk

    __device__ __forceinline__ void emit() {
        if (first) {
            sink.shared_word(wi, cur);
            first = false;
        } else {
            sink.own_word(wi, cur);
        }
        wi++;
    }
    __device__ __forceinline__ void put(uint32_t code, uint32_t l) {
        const uint32_t total = fill + l;
        if (total < 32) {
            cur |= code << (32 - total);
            fill = total;
        } else {
            const uint32_t over = total - 32;
            cur |= code >> over;
            emit();
            cur = over ? (code << (32 - over)) : 0u;
            fill = over;
        }
    }
    __device__ __forceinline__ void finish() {
        if (fill) sink.shared_word(wi, cur);  // shared with the next chunk
    }
};

__device__ __forceinline__ BitWriter<GlobalSink> make_writer(GlobalSink sink, uint64_t start) {
    BitWriter<GlobalSink> bw;
    bw.sink = sink;
    bw.wi = start >> 5;
    bw.fill = (uint32_t)(start & 31);
    bw.cur = 0;
    bw.first = true;
    return bw;
}

// A chunk's writer into the warp's shared copy of its group's words: the codes go into a
// 64-bit accumulator and every completed word is OR-ed in (the copy starts zeroed, and a
// chunk's first and last words may hold bits of its neighbours).  A put takes at most 32
// bits, so the accumulator never holds more than 63.
struct SliceWriter {
    uint32_t* words;          // the group's first stream word is words[0]
    uint32_t wo;              // offset of the word being completed
    unsigned long long acc;   // the low `nbits` bits are the pending bits
    uint32_t nbits;

    __device__ __forceinline__ void put(uint32_t code, uint32_t l) {
        acc = (acc << l) | code;
        nbits += l;
        if (nbits >= 32) {
            nbits -= 32;
            atomicOr(words + wo, (uint32_t)(acc >> nbits));
            wo++;
        }
    }
    __device__ __forceinline__ void finish() {
        if (nbits) atomicOr(words + wo, (uint32_t)(acc << (32 - nbits)));
    }
};

// Pack chunk c (lane `lane` of group c / 32), whose codes start at stream bit `start`,
// and write its elements' mantissa+sign bytes.  cl2[e] = (code, length).
template <int K, class Sink>
__device__ __forceinline__ void pack_chunk(const EncodeArgs& a, const uint2* cl2, uint64_t c, unsigned lane,
                                           uint64_t start, Sink sink) {
    auto bw = make_writer(sink, start);
    uint8_t* mpl = a.out + a.off_m;

    // the chunk's whole blocks (a prefix of its K/8 blocks), their loads one block ahead
    const uint64_t g = c / 32;
    uint32_t full = K / 8;
    if ((g + 1) * 32ull * K > a.n) {
        full = 0;
        while (full < K / 8 && block_element(g, K, full, lane) + 8 <= a.n) full++;
    }
    uint4 v_next = make_uint4(0u, 0u, 0u, 0u);
    if (full) v_next = __ldg(reinterpret_cast<const uint4*>(a.in + block_element(g, K, 0, lane)));
    for (uint32_t k = 0; k <= full && k < K / 8; k++) {
        const uint64_t x0 = block_element(g, K, k, lane);
        if (k < full) {
            const uint4 v = v_next;
            if (k + 1 < full) v_next = __ldg(reinterpret_cast<const uint4*>(a.in + block_element(g, K, k + 1, lane)));
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
            uint32_t mw[4];
#pragma unroll
            for (int j = 0; j < 4; j++) {
                // the pair (2j, 2j + 1): its two codes, as one put when they fit 32 bits
                const uint2 c0 = cl2[(w[j] >> 7) & 0xFFu], c1 = cl2[(w[j] >> 23) & 0xFFu];
                if (c0.y + c1.y <= 32u) {
                    bw.put((c0.x << c1.y) | c1.x, c0.y + c1.y);
                } else {
                    bw.put(c0.x, c0.y);
                    bw.put(c1.x, c1.y);
                }
                // their m bytes in bytes 0 and 2: each mantissa above the other's sign
                mw[j] = ((w[j] & 0x007F007Fu) << 1) | (w[j] >> 31) | ((w[j] << 1) & 0x00010000u);
            }
            *reinterpret_cast<uint2*>(mpl + x0) = make_uint2(__byte_perm(mw[0], mw[1], 0x6420), __byte_perm(mw[2], mw[3], 0x6420));
        } else {  // the partial block, if any
            for (uint64_t x = x0; x < a.n; x++) {
                const uint32_t h = a.in[x];
                const uint32_t partner = a.in[(x ^ 1u) < a.n ? (x ^ 1u) : x];
                const uint32_t e = (h >> 7) & 0xFFu;
                bw.put(cl2[e].x, cl2[e].y);
                mpl[x] = (uint8_t)(((h & 0x7Fu) << 1) | (partner >> 15));
            }
            break;
        }
    }
    bw.finish();
}

// ---------------------------------------------------------------- 3. lengths, scan and pack
//
// Chunk lengths, the scan of the group lengths and the pack in one kernel, reading the
// input once.  A CTA of 8 warps takes the next 8 groups from a ticket counter (so the
// CTAs holding earlier groups are always running and the scan below always makes
// progress); a warp reads its group (lane i: the 16-byte blocks i, i + 32, ... of the
// group) and, per block, looks up its 8 codes, joins them two by two, the pairs into two
// 32-bit halves and those into one 64-bit word (kept in shared memory with its length),
// writes the block's sign+mantissa bytes and adds the length to its chunk's count.  A
// group publishes its bit count as soon as it is known (flag kGroupCount) and, once it has
// its own start, its inclusive end (flag kGroupEnd), each as one 64-bit word written by an
// atomic exchange.  Before it looks for its own start, a warp puts its blocks' joined
// codes into the warp's shared copy of its words, counted from the group's bit 0 (one or
// two puts per block), so that its predecessors' counts have arrived by the time it needs
// them.  It finds the group's start bit by a decoupled look-back over the group words of
// the workspace, adding up its predecessors' counts, 32 at a time, back to the nearest
// group whose end is published; then it writes its words out, each shifted by the start
// bit mod 32.  A block whose half does not fit 32 bits is looked up again, code by code,
// at the put; the last, partial group and a group whose words do not fit the shared copy
// are packed straight into the stream (pack_chunk) after the look-back.

constexpr int kFusedWarps = 8;

// x << n for any n (0 from 32 on, as the PTX shift defines it)
__device__ __forceinline__ uint32_t shl32(uint32_t x, uint32_t n) {
    uint32_t r;
    asm("shl.b32 %0, %1, %2;" : "=r"(r) : "r"(x), "r"(n));
    return r;
}
constexpr uint32_t kPackSliceWords = 512;  // a group's stream words staged per warp (2 KiB)
constexpr uint8_t kSlowBlock = 255;        // a block whose codes are not joined (lengths are <= 192)

template <int K>
struct PackWarp {
    unsigned long long code[K / 8][32];  // block k of lane i: its codes joined, in the low len bits
    uint8_t len[K / 8][32];              // their length, or kSlowBlock
    uint32_t slice[kPackSliceWords];     // the group's stream words
};
template <int K>
constexpr size_t pack_smem_bytes() {
    return kFusedWarps * sizeof(PackWarp<K>);
}
// A group's look-back word (u64, in the workspace): kGroupCount with its bit count, then
// kGroupEnd | kGroupCount with its inclusive end bit.  Each is written whole by one atomic
// exchange and read whole, so no other memory access needs ordering around it.
constexpr unsigned long long kGroupCount = 1ull << 62;
constexpr unsigned long long kGroupEnd = 1ull << 63;
constexpr unsigned long long kGroupValue = kGroupCount - 1;
constexpr uint32_t kLookbackPolls = 1u << 20;

__device__ __forceinline__ unsigned long long ld_relaxed64(const unsigned long long* p) {
    unsigned long long v;
    asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ uint32_t ld_volatile(const uint32_t* p) { return *reinterpret_cast<const volatile uint32_t*>(p); }

// The stream word at the start of group b holds bits of groups b - 1 and b.  Each adds its
// bits (disjoint from the other's, so the sum is their union) and one arrival to the
// boundary's workspace word in one atomic; the group that arrives second writes the word.
__device__ __forceinline__ void boundary_word(const EncodeArgs& a, uint32_t b, uint32_t* word, uint32_t bits) {
    const unsigned long long old = atomicAdd(a.ws_edge + b, (1ull << 32) | bits);
    if ((old >> 32) == 1u) *word = (uint32_t)old | bits;
}

// The exclusive start bit of group g: predecessors' published counts back to the nearest
// published end.  Every wait is bounded (a word that never comes sets DFX_STATUS_TIMEOUT
// and counts as 0).
__device__ uint64_t lookback(const EncodeArgs& a, uint32_t g, unsigned lane, uint32_t& err) {
    const unsigned long long* gw = reinterpret_cast<const unsigned long long*>(a.ws_group_bits);
    uint64_t excl = 0;
    int64_t pos = (int64_t)g - 1;
    while (pos >= 0) {
        const int64_t i = pos - (int64_t)lane;
        unsigned long long v = kGroupCount | kGroupEnd;  // before group 0: an end at bit 0
        for (uint32_t it = 0;; it++) {
            if (i >= 0) v = ld_relaxed64(gw + i);
            if (__all_sync(kFull, (v & kGroupCount) != 0)) break;
            if (it == kLookbackPolls) {
                err |= DFX_STATUS_TIMEOUT;
                v = kGroupCount | kGroupEnd;
                break;
            }
            __nanosleep(32);
        }
        const uint32_t ends = __ballot_sync(kFull, (v & kGroupEnd) != 0);
        // the nearest predecessor with its end published gives that end, the ones after it
        // their counts
        const unsigned first = ends ? __ffs(ends) - 1 : 32u;
        uint64_t c = lane <= first ? (v & kGroupValue) : 0ull;
#pragma unroll
        for (int d = 16; d >= 1; d >>= 1) c += __shfl_xor_sync(kFull, c, d);
        excl += c;
        if (ends) break;
        pos -= 32;
    }
    return excl;
}

template <int K>
__global__ void __launch_bounds__(kFusedWarps * 32, 4) k_pack_fused(EncodeArgs a) {
    __shared__ uint2 cl2[256];  // (code, length)
    __shared__ uint32_t cta_ticket;
    extern __shared__ __align__(16) uint8_t pack_smem[];
    {
        // the input of the group this warp will most likely get (tickets follow the order in
        // which the CTAs start), sent to L2 while the code book is still being built
        const uint64_t gp = (uint64_t)blockIdx.x * kFusedWarps + (threadIdx.x >> 5);
        if ((threadIdx.x & 31) == 0 && (gp + 1) * 32u * K <= a.n) prefetch_l2(a.in + gp * 32u * K, 64u * K);
    }
    wait_for_previous_kernel();  // the code book
    cl2[threadIdx.x] = make_uint2(a.ws_code[threadIdx.x], a.ws_len[threadIdx.x]);
    if (threadIdx.x == 0) cta_ticket = atomicAdd(reinterpret_cast<uint32_t*>(reinterpret_cast<uint8_t*>(a.ws_counts) + kWsTicket), 1u);
    __syncthreads();
    if (blockIdx.x == 0) {
        // the container's zero bytes after the last stream word (the stream's length is
        // known from the code book): up to the 16-byte boundary, then 16 more
        const unsigned long long total =
            *reinterpret_cast<const unsigned long long*>(reinterpret_cast<const uint8_t*>(a.ws_counts) + kWsTotalBits);
        const uint64_t z0 = a.off_stream + 4 * ((total + 31) / 32), z1 = a.off_stream + stream_bytes(total);
        if (z1 <= a.max_bytes && threadIdx.x < (z1 - z0) / 4) reinterpret_cast<uint32_t*>(a.out + z0)[threadIdx.x] = 0u;
    }
    const unsigned warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t g = cta_ticket * kFusedWarps + warp;
    if (g >= a.n_group) return;
    PackWarp<K>& pw = reinterpret_cast<PackWarp<K>*>(pack_smem)[warp];
    const uint64_t c = (uint64_t)g * 32 + lane;
    const bool ragged = (uint64_t)(g + 1) * 32u * K > a.n;
    uint32_t err = 0;

    // the lane's chunk: its blocks' joined codes, their m bytes and the chunk's code bits
    constexpr uint32_t NB = K / 8;
    uint32_t bits = 0;
    if (!ragged) {
        uint8_t* mpl = a.out + a.off_m;
        if (lane == 0) prefetch_l2(a.in + (uint64_t)g * 32u * K, 64u * K);  // the whole group, while its first blocks load
#pragma unroll 4
        for (uint32_t k = 0; k < NB; k++) {
            const uint64_t x0 = block_element(g, K, k, lane);
            const uint4 v = __ldg(reinterpret_cast<const uint4*>(a.in + x0));
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
            uint32_t p[4], pl[4], mw[4];
#pragma unroll
            for (int q = 0; q < 4; q++) {
                const uint2 c0 = cl2[(w[q] >> 7) & 0xFFu], c1 = cl2[(w[q] >> 23) & 0xFFu];
                pl[q] = c0.y + c1.y;
                p[q] = (c0.x << c1.y) | c1.x;  // exact when pl[q] <= 32
                // the m bytes in bytes 0 and 2: each mantissa above the other's sign
                mw[q] = ((w[q] << 1) & 0x00FF00FEu) | (w[q] >> 31);
            }
            // the pairs joined into two 32-bit halves, then one 64-bit shift
            const uint32_t la = pl[0] + pl[1], lb = pl[2] + pl[3], L = la + lb;
            const bool slow = max(la, lb) > 32u;
            const uint32_t qa = shl32(p[0], pl[1]) | p[1], qb = shl32(p[2], pl[3]) | p[3];  // exact unless slow
            const unsigned long long x = ((unsigned long long)qa << lb) | qb;
            pw.code[k][lane] = x;
            pw.len[k][lane] = slow ? kSlowBlock : (uint8_t)L;
            bits += L;
            *reinterpret_cast<uint2*>(mpl + x0) = make_uint2(__byte_perm(mw[0], mw[1], 0x6420), __byte_perm(mw[2], mw[3], 0x6420));
        }
    } else {
        for (uint32_t k = 0; k < NB; k++) {
            const uint64_t x0 = block_element(g, K, k, lane);
            for (uint64_t x = x0; x < x0 + 8 && x < a.n; x++) bits += cl2[(a.in[x] >> 7) & 0xFFu].y;
            if (x0 + 8 > a.n) break;
        }
    }
    reinterpret_cast<uint16_t*>(a.out + a.off_clen)[c] = (uint16_t)bits;
    const uint32_t incl = warp_incl_scan(bits, lane);
    const uint32_t group_bits = __shfl_sync(kFull, incl, 31);

    // publish the group's bit count, then assemble its words from the group's bit 0 while
    // the predecessors' counts arrive; they are shifted into place once the start bit is known
    unsigned long long* gw = reinterpret_cast<unsigned long long*>(a.ws_group_bits);
    if (lane == 0) atomicExch(gw + g, kGroupCount | group_bits);
    uint32_t* sm = pw.slice;
    const uint32_t staged_words = (group_bits + 31) / 32 + 1;  // the group's words, at any start bit
    const bool staged = !ragged && staged_words <= kPackSliceWords;
    if (staged) {
        for (uint32_t i = lane; i < staged_words; i += 32) sm[i] = 0u;
        __syncwarp();
        // the bits of the previous chunk in the first word count as already placed zeros
        const uint32_t rel = incl - bits;  // the chunk's first bit within the group
        SliceWriter bw{sm, rel >> 5, 0ull, rel & 31u};
        for (uint32_t k = 0; k < NB; k++) {
            const uint32_t L = pw.len[k][lane];
            const unsigned long long x = pw.code[k][lane];
            if (L <= 32u) {
                bw.put((uint32_t)x, L);
            } else if (L != kSlowBlock) {
                bw.put((uint32_t)(x >> 32), L - 32u);
                bw.put((uint32_t)x, 32u);
            } else {  // code by code
                const uint4 v = __ldg(reinterpret_cast<const uint4*>(a.in + block_element(g, K, k, lane)));
                const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int q = 0; q < 8; q++) {
                    const uint2 cl = cl2[(w[q >> 1] >> (16 * (q & 1) + 7)) & 0xFFu];
                    bw.put(cl.x, cl.y);
                }
            }
        }
        bw.finish();
        __syncwarp();
    }

    // the group's start bit
    const uint64_t gb0 = lookback(a, g, lane, err);
    if (lane == 0) {
        unsigned long long* gbase = reinterpret_cast<unsigned long long*>(a.out + kOffGbase);
        gbase[g + 1] = gb0 + group_bits;
        atomicExch(gw + g, kGroupEnd | kGroupCount | (gb0 + group_bits));
        if (g + 1 == a.n_group) {
            *reinterpret_cast<unsigned long long*>(a.out + 16) = gb0 + group_bits;
            *reinterpret_cast<unsigned long long*>(a.out + 24) = a.off_stream + stream_bytes(gb0 + group_bits);
        }
    }

    // the group's words
    uint32_t* stream = reinterpret_cast<uint32_t*>(a.out + a.off_stream);
    const uint64_t wf = gb0 >> 5, wl = (gb0 + group_bits + 31) >> 5;  // the group's words [wf, wl)
    const uint32_t count = (uint32_t)(wl - wf);
    // a word shared with the previous or the next group (a whole group holds at least 32 K
    // bits, so only the last group can end in the word it starts in, and it has no next)
    const bool shared_first = (gb0 & 31u) != 0;
    const bool shared_last = ((gb0 + group_bits) & 31u) != 0 && g + 1 < a.n_group;
    if (staged) {
        // stream word wf + i holds the group's bits from 32 i - sh on (sh = gb0 mod 32): the
        // low sh bits of staged word i - 1 above the high 32 - sh bits of staged word i
        const uint32_t sh = (uint32_t)(gb0 & 31u);
        for (uint32_t i = lane; i < count; i += 32) {
            if ((i == 0 && shared_first) || (i + 1 == count && shared_last)) continue;
            stream[wf + i] = __funnelshift_r(sm[i], i ? sm[i - 1] : 0u, sh);
        }
        if (lane == 0 && shared_first) boundary_word(a, g, stream + wf, sm[0] >> sh);
        if (lane == 0 && shared_last)
            boundary_word(a, g + 1, stream + wl - 1, __funnelshift_r(sm[count - 1], count > 1 ? sm[count - 2] : 0u, sh));
    } else {
        // straight into the stream: the group's words start at zero, the codes are OR-ed in
        for (uint32_t i = lane; i < count; i += 32) stream[wf + i] = 0u;
        __syncwarp();
        __threadfence();
        pack_chunk<K>(a, cl2, c, lane, gb0 + (incl - bits), GlobalSink{stream});
        __syncwarp();
        __threadfence();
        if (lane == 0 && shared_first) boundary_word(a, g, stream + wf, ld_volatile(stream + wf));
        if (lane == 0 && shared_last) boundary_word(a, g + 1, stream + wl - 1, ld_volatile(stream + wl - 1));
    }
    if (err) atomicOr(a.status, err);
}

// The zeroing a Huffman encode needs before its passes: the container's index region
// [0, off_m) and the padding [off_m + n, off_stream), the workspace's histogram counts
// [0, 2048) and [kWsTicket, ws_end) (the pack's ticket, look-back and boundary words).
// Every region but the padding is a whole number of 8-byte words.
__global__ void __launch_bounds__(256) k_zero_regions(EncodeArgs a, uint64_t ws_end) {
    allow_next_kernel();  // the histogram waits for this kernel only before its final counts
    const uint64_t w_out = a.off_m / 8, w_cnt = 2048 / 8, w_ws = (ws_end - kWsTicket) / 8;
    unsigned long long* out = reinterpret_cast<unsigned long long*>(a.out);
    unsigned long long* ws = reinterpret_cast<unsigned long long*>(a.ws_counts);
    const uint64_t stride = (uint64_t)gridDim.x * blockDim.x;
    for (uint64_t i = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; i < w_out + w_cnt + w_ws; i += stride) {
        if (i < w_out) out[i] = 0ull;
        else if (i < w_out + w_cnt) ws[i - w_out] = 0ull;
        else ws[kWsTicket / 8 + (i - w_out - w_cnt)] = 0ull;
    }
    if (blockIdx.x == 0 && a.off_m + a.n + threadIdx.x < a.off_stream) a.out[a.off_m + a.n + threadIdx.x] = 0;
}

template <int K>
cudaError_t launch_pack(const EncodeArgs& a, unsigned ctas, int dev, cudaStream_t s) {
    static bool attr_set[64] = {};
    if (dev >= 0 && dev < 64 && !attr_set[dev]) {
        const cudaError_t e =
            cudaFuncSetAttribute(k_pack_fused<K>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)pack_smem_bytes<K>());
        if (e != cudaSuccess) return e;
        attr_set[dev] = true;
    }
    return launch_dependent(k_pack_fused<K>, ctas, kFusedWarps * 32, pack_smem_bytes<K>(), s, a);
}

}  // namespace

cudaError_t launch_encode(const EncodeArgs& a, uint64_t max_bytes, cudaStream_t s) {
    cudaError_t err;
    // the index region (header .. clen padding) starts at zero; so does everything after the
    // m plane for the tANS coders (their packs OR codes into the stream), while the Huffman
    // pack writes every stream word and the container's zero padding itself
    const bool packs = !is_tans(a.coder) && a.n_group > 0;
    if (packs) {
        // one kernel: the index region, the m plane's padding, the histogram counts and the
        // pack's ticket, look-back and boundary words
        const uint64_t ws_end = ws_edge_offset(a.n_group) + 8 * (a.n_group + 1);
        const uint64_t words = (a.off_m + 2048 + ws_end - kWsTicket) / 8;
        const unsigned blocks = (unsigned)((words + 4095) / 4096 < 148 ? (words + 4095) / 4096 : 148);
        k_zero_regions<<<blocks, 256, 0, s>>>(a, ws_end);
        if ((err = cudaGetLastError()) != cudaSuccess) return err;
    } else {
        if ((err = cudaMemsetAsync(a.out, 0, a.off_m, s)) != cudaSuccess) return err;
        if (max_bytes > a.off_m + a.n &&
            (err = cudaMemsetAsync(a.out + a.off_m + a.n, 0, max_bytes - (a.off_m + a.n), s)) != cudaSuccess)
            return err;
        if ((err = cudaMemsetAsync(a.ws_counts, 0, 256 * sizeof(unsigned long long), s)) != cudaSuccess) return err;
    }

    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    {
        static bool attr_set[64] = {};
        if (dev >= 0 && dev < 64 && !attr_set[dev]) {
            if ((err = cudaFuncSetAttribute(k_histogram, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kHistSmem)) !=
                cudaSuccess)
                return err;
            attr_set[dev] = true;
        }
        // one CTA per SM, fewer for small inputs (at least one chunk per warp)
        const uint64_t chunks = (a.n / 8 + kHistChunkUnits - 1) / kHistChunkUnits;
        const uint64_t ctas = (chunks + kHistWarps - 1) / kHistWarps;
        const unsigned hist_blocks = (unsigned)(ctas == 0 ? 1 : (ctas < (uint64_t)sms ? ctas : (uint64_t)sms));
        if ((err = launch_dependent(k_histogram, hist_blocks, kHistWarps * 32, kHistSmem, s, a.in, a.n, a.ws_counts,
                                    a.status)) != cudaSuccess)
            return err;
    }
    if (is_tans(a.coder)) {  // the tANS passes around the same group scan
        if ((err = launch_encode_tans(a, 0, s)) != cudaSuccess) return err;
        k_group_scan<<<1, kScanThreads, 0, s>>>(a);
        if ((err = cudaGetLastError()) != cudaSuccess) return err;
        return launch_encode_tans(a, 1, s);
    }
    if ((err = launch_dependent(k_build_codebook, 1, 256, 0, s, a)) != cudaSuccess) return err;
    if (a.n_group == 0) {  // an empty tensor: the group scan writes the header totals
        k_group_scan<<<1, kScanThreads, 0, s>>>(a);
        return cudaGetLastError();
    }
    const unsigned ctas = (a.n_group + kFusedWarps - 1) / kFusedWarps;
    switch (a.K) {
        case 32: return launch_pack<32>(a, ctas, dev, s);
        case 64: return launch_pack<64>(a, ctas, dev, s);
        case 128: return launch_pack<128>(a, ctas, dev, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace dfx
