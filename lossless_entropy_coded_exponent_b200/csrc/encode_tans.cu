// encode_tans.cu -- GPU encoder passes of the tANS exponent coder, one state per chunk
// (coder 1) or two interleaved states (coder 2: even positions on state A, odd on B),
// sm_100a.
//
// After the exponent histogram (encode.cu), on the caller's stream:
//   phase 0  k_tans_tables      one CTA: the frequencies (counts * M / n rounded half up,
//                               at least 1, the largest absorbing the difference), their
//                               prefix sums, the state table (tans_tables.cuh), the
//                               encoder's per-symbol parameters and slot table, freq[256]
//                               and the constant header fields;
//            k_tans_chunk_bits  per chunk its bit length: the encoder run over the chunk
//                               from its last symbol to its first, counting the field bits,
//                               plus the state; per group of 32 chunks the sum;
//   (the group scan of encode.cu then writes gbase, total_bits and total_bytes)
//   phase 1  k_tans_pack        per group (one warp): every lane runs its chunk's encoder
//                               again and writes the fields backward from the chunk's end,
//                               the last one emitted (the chunk's first symbol) right after
//                               the final state(s), which go first (A's, then B's); the
//                               mantissa+sign bytes.
// The encoding step for symbol s in state X (M <= X < 2M): nb = the bits with
// f <= X >> nb < 2f, which for h = floor(log2 f) is R - h, one less when X < f << (R - h);
// emit the low nb bits of X; X becomes M + the slot of s numbered X >> nb.  The rules are
// stated in include/dfx.h; tabled ANS is J. Duda's ("Asymmetric numeral systems", 2013).
#include <cuda_runtime.h>
#include <stdint.h>

#include "dfx_common.cuh"
#include "tans_tables.cuh"

namespace dfx {
namespace {

constexpr unsigned kFullMask = 0xffffffffu;

// Workspace words (a.ws_tans): per symbol sp = threshold << 16 | (R - h), sc = cs << 16 | f,
// then enc[cs[s] + k - f[s]] = M + the slot of s numbered k.
constexpr uint32_t kWsSp = 0, kWsSc = 256, kWsEnc = 512;

__device__ __forceinline__ uint32_t warp_incl_scan_u32(uint32_t v, unsigned lane) {
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const uint32_t y = __shfl_up_sync(kFullMask, v, d);
        if (lane >= (unsigned)d) v += y;
    }
    return v;
}

// ---------------------------------------------------------------- tables

constexpr int kTablesThreads = 1024;

__global__ void __launch_bounds__(kTablesThreads) k_tans_tables(EncodeArgs a) {
    __shared__ uint32_t f[256], cs[256], wsum[8];
    __shared__ __align__(16) uint8_t scratch[kTansScratchBytes];
    const uint32_t t = threadIdx.x, warp = t >> 5, lane = t & 31;
    const uint32_t R = a.table_log, M = 1u << R;
    const unsigned long long n = a.n;
    if (t < 256) {
        const unsigned long long c = a.ws_counts[t];
        uint32_t q = 0;
        if (c) {
            const unsigned long long r = (2ull * c * M + n) / (2ull * n);  // counts * M / n, rounded half up
            q = r ? (uint32_t)r : 1u;
        }
        f[t] = q;
    }
    __syncthreads();
    if (warp == 0 && n > 0) {
        // the largest frequency (the smallest symbol among equal ones) takes the whole
        // shortfall, or gives up an excess one unit at a time; lane l holds symbols
        // l, l + 32, ..., l + 224
        uint32_t sum = 0;
        for (uint32_t s = lane; s < 256; s += 32) sum += f[s];
#pragma unroll
        for (int d = 16; d > 0; d >>= 1) sum += __shfl_xor_sync(kFullMask, sum, d);
        while (sum != M) {
            uint32_t bf = 0, bs = 256;
            for (uint32_t s = lane; s < 256; s += 32)
                if (f[s] > bf) bf = f[s], bs = s;
#pragma unroll
            for (int d = 16; d > 0; d >>= 1) {
                const uint32_t of = __shfl_xor_sync(kFullMask, bf, d), os = __shfl_xor_sync(kFullMask, bs, d);
                if (of > bf || (of == bf && os < bs)) bf = of, bs = os;
            }
            if (lane == 0) f[bs] = sum < M ? bf + (M - sum) : bf - 1;
            __syncwarp();
            sum = sum < M ? M : sum - 1;
        }
    }
    __syncthreads();
    uint32_t incl = 0, fv = 0;
    if (t < 256) {
        fv = f[t];
        incl = warp_incl_scan_u32(fv, lane);
        if (lane == 31) wsum[warp] = incl;
    }
    __syncthreads();
    if (t < 256) {
        uint32_t base = 0;
        for (uint32_t w = 0; w < warp; w++) base += wsum[w];
        const uint32_t c0 = base + incl - fv;
        cs[t] = c0;
        uint32_t sp = 0;
        if (fv) {
            const uint32_t nb_hi = R - (31u - __clz(fv));
            sp = ((fv << nb_hi) << 16) | nb_hi;
        }
        a.ws_tans[kWsSp + t] = sp;
        a.ws_tans[kWsSc + t] = (c0 << 16) | fv;
        reinterpret_cast<uint16_t*>(a.out + kOffFreq)[t] = (uint16_t)fv;
    }
    __syncthreads();
    if (n > 0) {
        uint32_t* enc = a.ws_tans + kWsEnc;
        tans_number_states(f, cs, R, scratch, [&](uint32_t j, uint32_t s, uint32_t k) { enc[cs[s] + k - f[s]] = M + j; });
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
        *reinterpret_cast<uint32_t*>(h + 56) = R;
        *reinterpret_cast<uint32_t*>(h + 60) = a.coder;
    }
}

// ---------------------------------------------------------------- the encoder of one chunk

// The encoder tables in shared memory: per symbol (sp, sc) and the slot table.
struct EncTables {
    uint2 spc[256];
    uint32_t enc[kTansSlotsMax];
};

__device__ __forceinline__ void load_enc_tables(const EncodeArgs& a, EncTables& E) {
    const uint32_t M = 1u << a.table_log;
    for (uint32_t i = threadIdx.x; i < 256; i += blockDim.x)
        E.spc[i] = make_uint2(a.ws_tans[kWsSp + i], a.ws_tans[kWsSc + i]);
    for (uint32_t i = threadIdx.x; i < M; i += blockDim.x) E.enc[i] = a.ws_tans[kWsEnc + i];
    __syncthreads();
}

// One encoding step of exponent e from state X: calls put(v, nb) with the emitted field.
template <class Put>
__device__ __forceinline__ uint32_t enc_step(const EncTables& E, uint32_t X, uint32_t e, Put& put) {
    const uint2 q = E.spc[e];
    const uint32_t nb = (q.x & 0xFFFFu) - (X < (q.x >> 16) ? 1u : 0u);
    put(X & ((1u << nb) - 1u), nb);
    return E.enc[(q.y >> 16) + (X >> nb) - (q.y & 0xFFFFu)];
}

// Runs the encoder over chunk `lane` of group g from its last element to its first,
// starting in state M (each state, with two: the element at chunk position i on state
// i mod 2); put(v, nb) receives the fields in that order.  With WriteM the chunk's
// mantissa+sign bytes are written too.  Returns the final states (M when the chunk is
// empty, which has no bits).
template <int K, uint32_t States, bool WriteM, class Put>
__device__ __forceinline__ uint2 encode_chunk(const EncodeArgs& a, const EncTables& E, uint64_t g, unsigned lane,
                                              Put& put) {
    const uint32_t M = 1u << a.table_log;
    uint32_t X[2] = {M, M};
    uint8_t* mpl = a.out + a.off_m;
    // the chunk's whole blocks (a prefix of its K/8 blocks) and a partial one after them
    uint32_t full = K / 8;
    if ((g + 1) * 32ull * K > a.n) {
        full = 0;
        while (full < K / 8 && block_element(g, K, full, lane) + 8 <= a.n) full++;
    }
    if (full < K / 8) {
        const uint64_t x0 = block_element(g, K, full, lane);
        for (uint64_t x = a.n; x-- > x0;) {  // nothing when x0 >= n
            const uint32_t h = a.in[x];
            uint32_t& Xs = X[States == 2 ? (uint32_t)(x - x0) & 1u : 0u];  // blocks before hold 8 k elements
            Xs = enc_step(E, Xs, (h >> 7) & 0xFFu, put);
            if (WriteM) {
                const uint32_t partner = a.in[(x ^ 1u) < a.n ? (x ^ 1u) : x];
                mpl[x] = (uint8_t)(((h & 0x7Fu) << 1) | (partner >> 15));
            }
        }
    }
    uint4 v_next = make_uint4(0u, 0u, 0u, 0u);
    if (full) v_next = __ldg(reinterpret_cast<const uint4*>(a.in + block_element(g, K, full - 1, lane)));
    for (uint32_t k = full; k-- > 0;) {
        const uint4 v = v_next;
        if (k > 0) v_next = __ldg(reinterpret_cast<const uint4*>(a.in + block_element(g, K, k - 1, lane)));
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int j = 7; j >= 0; j--) {
            const uint32_t h = (w[j >> 1] >> (16 * (j & 1))) & 0xFFFFu;
            uint32_t& Xs = X[States == 2 ? (uint32_t)j & 1u : 0u];
            Xs = enc_step(E, Xs, (h >> 7) & 0xFFu, put);
        }
        if (WriteM) {
            uint32_t mb[2] = {0u, 0u};
#pragma unroll
            for (int j = 0; j < 8; j++) {
                const uint32_t h = (w[j >> 1] >> (16 * (j & 1))) & 0xFFFFu;
                const uint32_t partner = (w[j >> 1] >> (16 * ((j & 1) ^ 1))) & 0xFFFFu;  // element j ^ 1
                mb[j >> 2] |= (((h & 0x7Fu) << 1) | (partner >> 15)) << (8 * (j & 3));
            }
            *reinterpret_cast<uint2*>(mpl + block_element(g, K, k, lane)) = make_uint2(mb[0], mb[1]);
        }
    }
    return make_uint2(X[0], X[1]);
}

// ---------------------------------------------------------------- chunk bit lengths

constexpr int kTansChunkThreads = 256;

struct CountBits {
    uint32_t bits;
    __device__ __forceinline__ void operator()(uint32_t, uint32_t nb) { bits += nb; }
};

template <int K, uint32_t States>
__global__ void __launch_bounds__(kTansChunkThreads) k_tans_chunk_bits(EncodeArgs a) {
    __shared__ EncTables E;
    load_enc_tables(a, E);
    const uint64_t c = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const unsigned lane = threadIdx.x & 31;
    uint32_t bits = 0;
    if (c < a.n_chunk) {
        const uint64_t g = c / 32;
        CountBits cb{0u};
        encode_chunk<K, States, false>(a, E, g, lane, cb);
        const bool empty = block_element(g, K, 0, lane) >= a.n;
        bits = empty ? 0u : cb.bits + States * a.table_log;
        reinterpret_cast<uint16_t*>(a.out + a.off_clen)[c] = (uint16_t)bits;
    }
    const uint32_t incl = warp_incl_scan_u32(bits, lane);
    const uint64_t g = c / 32;
    if (lane == 31 && g < a.n_group) a.ws_group_bits[g] = incl;
}

// ---------------------------------------------------------------- pack

constexpr int kTansPackThreads = 256;
constexpr uint32_t kTansPackSliceWords = 512;  // a group's stream words staged per warp (2 KiB)

// Writes fields backward: each one ends where the previous began.  `acc` holds the
// pending bits of word wi (low half) and of word wi - 1 (high half); r = pos - 32 wi is
// the number of bit positions of word wi below the current position (1..32).  A completed
// word is OR-ed in (the destination starts zeroed, and a chunk's first and last words may
// hold bits of its neighbours).
struct BackWriter {
    uint32_t* words;  // stream word `base` is words[0]
    uint64_t base;
    uint64_t wi;
    unsigned long long acc;
    uint32_t r;

    __device__ __forceinline__ void operator()(uint32_t v, uint32_t nb) {
        acc |= (unsigned long long)v << (32u - r);
        const int32_t rr = (int32_t)r - (int32_t)nb;
        if (rr <= 0) {
            atomicOr(words + (wi - base), (uint32_t)acc);
            acc >>= 32;
            wi--;
            r = (uint32_t)(rr + 32);
        } else {
            r = (uint32_t)rr;
        }
    }
    __device__ __forceinline__ void finish() {
        if (r < 32u) atomicOr(words + (wi - base), (uint32_t)acc);
    }
};

template <int K, uint32_t States>
__global__ void __launch_bounds__(kTansPackThreads) k_tans_pack(EncodeArgs a) {
    __shared__ EncTables E;
    __shared__ uint32_t slice[kTansPackThreads / 32][kTansPackSliceWords];
    load_enc_tables(a, E);
    const uint64_t c = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const unsigned lane = threadIdx.x & 31;
    if (c >= a.n_chunk) return;  // n_chunk is a multiple of 32: whole warps leave
    const uint64_t g = c / 32;
    const uint16_t* clen = reinterpret_cast<const uint16_t*>(a.out + a.off_clen);
    const uint32_t cl = clen[c];
    const uint32_t incl = warp_incl_scan_u32(cl, lane);
    const uint64_t gb0 = reinterpret_cast<const unsigned long long*>(a.out + a.off_gbase)[g];
    const uint64_t start = gb0 + (incl - cl), end = start + cl;
    uint32_t* stream = reinterpret_cast<uint32_t*>(a.out + a.off_stream);
    const uint32_t group_bits = __shfl_sync(kFullMask, incl, 31);
    const uint64_t wf = gb0 >> 5, wl = (gb0 + group_bits + 31) >> 5;  // the group's words [wf, wl)
    const uint32_t count = (uint32_t)(wl - wf);
    const bool staged = count <= kTansPackSliceWords;
    uint32_t* sm = slice[threadIdx.x >> 5];
    if (staged) {
        for (uint32_t i = lane; i < count; i += 32) sm[i] = 0u;
        __syncwarp();
    }
    if (cl) {  // a chunk with elements (an empty one has no bits and no m bytes)
        BackWriter bw{staged ? sm : stream, staged ? wf : 0ull, (end - 1) >> 5, 0ull, 0u};
        bw.r = (uint32_t)(end - 32ull * bw.wi);
        const uint2 X = encode_chunk<K, States, true>(a, E, g, lane, bw);
        // the states: the chunk's first bits, A's before B's
        if (States == 2) bw(X.y - (1u << a.table_log), a.table_log);
        bw(X.x - (1u << a.table_log), a.table_log);
        bw.finish();
    }
    if (staged) {
        __syncwarp();
        for (uint32_t i = lane; i < count; i += 32) {
            const uint32_t v = sm[i];
            if (i == 0 || i + 1 == count) {
                if (v) atomicOr(stream + wf + i, v);
            } else {
                stream[wf + i] = v;
            }
        }
    }
}

template <uint32_t States>
cudaError_t launch_tans_passes(const EncodeArgs& a, int phase, unsigned blocks, cudaStream_t s) {
    if (phase == 0) {
        switch (a.K) {
            case 32: k_tans_chunk_bits<32, States><<<blocks, kTansChunkThreads, 0, s>>>(a); break;
            case 64: k_tans_chunk_bits<64, States><<<blocks, kTansChunkThreads, 0, s>>>(a); break;
            case 128: k_tans_chunk_bits<128, States><<<blocks, kTansChunkThreads, 0, s>>>(a); break;
            default: return cudaErrorInvalidValue;
        }
    } else {
        switch (a.K) {
            case 32: k_tans_pack<32, States><<<blocks, kTansPackThreads, 0, s>>>(a); break;
            case 64: k_tans_pack<64, States><<<blocks, kTansPackThreads, 0, s>>>(a); break;
            case 128: k_tans_pack<128, States><<<blocks, kTansPackThreads, 0, s>>>(a); break;
            default: return cudaErrorInvalidValue;
        }
    }
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_encode_tans(const EncodeArgs& a, int phase, cudaStream_t s) {
    if (a.n_chunk == 0 && phase == 1) return cudaSuccess;
    const unsigned blocks = (unsigned)((a.n_chunk + kTansChunkThreads - 1) / kTansChunkThreads);
    if (phase == 0) {
        k_tans_tables<<<1, kTablesThreads, 0, s>>>(a);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess || a.n_chunk == 0) return e;
    }
    return tans_states(a.coder) == 2 ? launch_tans_passes<2>(a, phase, blocks, s)
                                     : launch_tans_passes<1>(a, phase, blocks, s);
}

}  // namespace dfx
