// tans_tables.cuh -- the tANS state table of one tensor, built by one CTA in shared
// memory; used by the encoder's table kernel and by every decoding CTA.
//
// Rules (stated in include/dfx.h): the M = 2^R slots are dealt to the symbols with an
// odd stride (occurrence i of the list holding every symbol s f[s] times, in symbol
// order, goes to slot i * step mod M, step = M/2 + M/8 + 3), and the slots of each
// symbol, in ascending order, are its states f[s], f[s] + 1, ..., 2 f[s] - 1.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "dfx_common.cuh"

namespace dfx {
namespace {

// Shared-memory scratch of tans_number_states.
constexpr uint32_t kTansSlotsMax = 1u << kTansMaxLog;
constexpr size_t kTansScratchSym = 0;                                   // u8 [M]
constexpr size_t kTansScratchWc = kTansSlotsMax;                        // u16 [256][32]
constexpr size_t kTansScratchRun = kTansScratchWc + 256 * 32 * 2;       // u32 [256]
constexpr size_t kTansScratchBytes = kTansScratchRun + 256 * 4;

// Every thread of the block (at most 32 warps) calls it with the frequencies f[256]
// (summing to M = 2^R) and their exclusive prefix sums cs[256] in shared memory;
// emit(j, s, k) is called once for every slot j with its symbol s and state number k.
// The slot of occurrence i is found from the other side: the symbol of slot j = i * step
// is the last s with cs[s] <= i.  State numbers come in rounds of one slot per thread in
// ascending slot order: __match_any_sync ranks a slot among the warp's slots of its
// symbol, and a per-symbol prefix over the warps (one warp per symbol, one lane per
// warp's count) adds the slots of lower warps and of earlier rounds.
template <class Emit>
__device__ void tans_number_states(const uint32_t* f, const uint32_t* cs, uint32_t R, uint8_t* scratch, Emit emit) {
    const uint32_t t = threadIdx.x, warp = t >> 5, lane = t & 31, nwarps = blockDim.x >> 5;
    const uint32_t M = 1u << R;
    uint8_t* sym = scratch + kTansScratchSym;
    uint16_t* wc = reinterpret_cast<uint16_t*>(scratch + kTansScratchWc);  // [symbol][warp]
    uint32_t* run = reinterpret_cast<uint32_t*>(scratch + kTansScratchRun);
    const uint32_t step = (M >> 1) + (M >> 3) + 3;
    for (uint32_t i = t; i < M; i += blockDim.x) {
        uint32_t lo = 0, hi = 256;  // cs[lo] <= i < cs[hi], with cs[256] = M
        while (hi - lo > 1) {
            const uint32_t mid = (lo + hi) >> 1;
            if (cs[mid] <= i) lo = mid;
            else hi = mid;
        }
        sym[(i * step) & (M - 1)] = (uint8_t)lo;
    }
    if (t < 256) run[t] = 0;
    __syncthreads();
    for (uint32_t r0 = 0; r0 < M; r0 += blockDim.x) {
        for (uint32_t i = t; i < 256 * 32 * 2 / 16; i += blockDim.x) reinterpret_cast<uint4*>(wc)[i] = make_uint4(0, 0, 0, 0);
        __syncthreads();
        const uint32_t j = r0 + t;
        const bool valid = j < M;
        const uint32_t s = valid ? sym[j] : 256u;
        const unsigned peers = __match_any_sync(0xffffffffu, s);
        const unsigned below = peers & ((1u << lane) - 1u);
        if (valid && below == 0) wc[s * 32 + warp] = (uint16_t)__popc(peers);
        __syncthreads();
        for (uint32_t sy = warp; sy < 256; sy += nwarps) {
            if (f[sy] == 0) continue;
            const uint32_t c = lane < nwarps ? wc[sy * 32 + lane] : 0u;
            const uint32_t before = run[sy];
            uint32_t incl = c;
#pragma unroll
            for (int d = 1; d < 32; d <<= 1) {
                const uint32_t y = __shfl_up_sync(0xffffffffu, incl, d);
                if (lane >= (unsigned)d) incl += y;
            }
            if (lane < nwarps) wc[sy * 32 + lane] = (uint16_t)(before + incl - c);
            if (lane == 31) run[sy] = before + incl;
        }
        __syncthreads();
        if (valid) emit(j, s, f[s] + wc[s * 32 + warp] + __popc(below));
        __syncthreads();
    }
}

}  // namespace
}  // namespace dfx
