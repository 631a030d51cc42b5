// decode_gemm.cu -- Y = X W^T with the weight matrix W restored from its DFX1 container
// inside the kernel that multiplies it, on the 5th-generation tensor cores of sm_100a.
//
// The pages decompress the weights on the GPU just before the computation that uses them
// ("DFloat11: lossless LLM compression for GPU", aikraft.ru blog, section 02, and section
// 03 item 2, where the decoded values are rebuilt in a form ready for computation).  Here
// the decoded BF16 weights never reach HBM: they go from the decoding threads' registers
// into shared-memory tiles that tcgen05.mma reads, with the accumulator in tensor memory.
//
// Shapes: W is rows x cols BF16 (row-major, the container's element order), cols a whole
// number of groups (32 chunks of K codes), so every group lies inside one row.  X is
// tokens x cols BF16 (row-major), tokens <= 32; Y is tokens x rows FP32 (row-major).
//
// One CTA (one per SM) takes a tile of at most 128 rows of W:
//   * every thread first helps build the Huffman tables in shared memory (the canonical
//     per-length limits and the 14-bit pair table of huffman_tables.cuh);
//   * 15 decoding warps hold up to 8 rows each (row slot i of warp w is tile row w + 15 i;
//     a tile has at most 120 rows, the MMA's M = 128 rows past them unused).
//     A warp decodes its rows side by side, one step at a time: in a step each lane
//     decodes the next 8 codes of its chunk in every row, which are the row's 256
//     consecutive weights [256 t, 256 t + 256), lane i holding weights 8 i .. 8 i + 7;
//   * the 8 weights are merged with their sign+mantissa bytes and written as one 16-byte
//     store into the A tile of the step: 128 rows x 256 K in the canonical K-major layout
//     with the 128-byte swizzle (four 64-wide K atoms; in each 8-row group of an atom, row
//     r's 16-byte chunk c sits at chunk c ^ (r mod 8)).  The same threads copy the step's
//     slice of X into the B tile in the same layout;
//   * one MMA warp waits for the step's tiles, issues 16 tcgen05.mma (M = 128, N = tokens
//     rounded up to 16, K = 16 each) accumulating in tensor memory, and commits them to
//     the stage's "free" barrier, which the decoding warps wait on before reusing the
//     stage two steps later (two stages of A and B);
//   * after the last step, decoding warps 0-3 read the accumulator (tensor memory lanes
//     32 w .. 32 w + 31 are tile rows) and write Y.
// Each lane's stream words come from global memory with one word of read-ahead (a step's
// worth of decoding hides its latency); the sign+mantissa bytes and the slice of X of the
// next step are loaded into registers while the current step decodes.
// Every wait is bounded: a wait that runs out sets DFX_STATUS_TIMEOUT and the kernel
// carries on (with a wrong Y) and releases its tensor memory.  A corrupt container sets
// the same status bits as dfx_decode and never makes the kernel read outside it.
#include <cuda_runtime.h>
#include <stdint.h>

#include "decode_pipeline.cuh"
#include "huffman_tables.cuh"

namespace dfx {
namespace {

// 15 decoding warps and the MMA warp: 16 warps, 4 per SM sub-partition, so that each thread
// may hold up to 128 registers (a 17th warp would cut that to 96).
constexpr int kGemmDecodeWarps = 15;
constexpr int kGemmRowSlots = 8;                                     // rows per decoding warp
static_assert(kGemmMaxRows == kGemmDecodeWarps * kGemmRowSlots, "rows per tile at most");
constexpr int kGemmTileRows = 128;                                   // MMA M (rows past the tile's are unused)
constexpr int kGemmThreads = (kGemmDecodeWarps + 1) * 32;
constexpr int kGemmDecodeThreads = kGemmDecodeWarps * 32;
constexpr uint32_t kStepK = 256;                                   // K per step
constexpr uint32_t kAtomBytes = 128;                               // one swizzle row: 64 BF16
constexpr uint32_t kAStageBytes = kGemmTileRows * kStepK * 2;      // 64 KiB
constexpr uint32_t kTmemCols = 32;                                 // FP32 accumulator columns
static_assert(kGemmMaxRows <= kGemmTileRows, "the rows of a tile fit the MMA's M = 128");

// ---------------------------------------------------------------- tcgen05 helpers

// Shared-memory matrix descriptor of a K-major tile with the 128-byte swizzle: 8-row
// groups 1024 bytes apart (stride byte offset), leading byte offset 16 (unused by this
// layout), descriptor version 1 (sm_100), layout type 2 (128-byte swizzle).  The tile
// base is 1024-byte aligned, so the base-offset field stays 0.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t addr) {
    return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
           ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// Instruction descriptor of kind::f16: FP32 accumulator, BF16 A and B, both K-major,
// N = n (multiple of 16), M = 128.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(uint32_t n) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((n >> 3) << 17) | ((128u >> 4) << 24);
}

__device__ __forceinline__ void mma_bf16(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(tmem_d),
        "l"(a), "l"(b), "r"(idesc), "r"(acc)
        : "memory");
}
// arrives on `bar` once every tcgen05 operation this thread issued before has completed
__device__ __forceinline__ void mma_commit(unsigned long long* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(smem_addr(bar))
                 : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory"); }
__device__ __forceinline__ void mbar_init_count(unsigned long long* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive(unsigned long long* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(smem_addr(bar)) : "memory");
}
// 16 FP32 accumulator columns of this warp's 32 tensor-memory lanes
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&v)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15}, [%16];\n"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]), "=r"(v[8]),
          "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory");
}
__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint4 v) {
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};\n" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}

// Byte offset of (row r, 16-byte chunk c of K atom a) in a K-major 128-byte-swizzled tile
// of `rows` rows: atoms one after another, 8-row groups 1024 bytes apart, row r of its
// group at 128 (r mod 8), its chunk c at chunk c ^ (r mod 8).
__device__ __forceinline__ uint32_t sw128_offset(uint32_t rows, uint32_t r, uint32_t a, uint32_t c) {
    return a * rows * kAtomBytes + (r >> 3) * 1024u + (r & 7u) * kAtomBytes + ((c ^ (r & 7u)) << 4);
}

// ---------------------------------------------------------------- stream reader
//
// The bit reader of decode.cu over global memory, with one word of read-ahead: a lane
// holds its bit position p (relative to word `bw` of the stream), the 32-bit peek at p, the
// words cur, nxt under it (cw and cw + 1) and `ahead` (cw + 2), loaded when the position
// moves into a new word and first needed when it moves again, about 12 codes later.  No
// reload follows more than 32 consumed bits, so p moves at most one word between reloads.
// Loads are clamped to the stream section.
struct GemmReader {
    uint32_t bw, p, cw, peek, cur, nxt, ahead;

    __device__ __forceinline__ static uint32_t word(const uint32_t* s, uint32_t i, uint32_t maxw) {
        return __ldg(s + min(i, maxw));
    }
    __device__ __forceinline__ void init(const uint32_t* s, uint32_t maxw, uint32_t base_word, uint32_t start) {
        bw = base_word;
        p = start;
        cw = start >> 5;
        cur = word(s, bw + cw, maxw);
        nxt = word(s, bw + cw + 1, maxw);
        ahead = word(s, bw + cw + 2, maxw);
    }
    __device__ __forceinline__ void reload(const uint32_t* s, uint32_t maxw) {
        const uint32_t wi = p >> 5;
        if (wi != cw) {  // wi == cw + 1
            cw = wi;
            cur = nxt;
            nxt = ahead;
            ahead = word(s, bw + cw + 2, maxw);
        }
        peek = __funnelshift_l(nxt, cur, p);
    }
    __device__ __forceinline__ uint32_t one(const uint32_t* lut, const HuffTables& T, const uint32_t* s, uint32_t maxw,
                                            uint32_t& err) {
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
        reload(s, maxw);
        return sym;
    }
    // two codes merged with their m bytes (bytes 2j, 2j+1 of mw): two BF16
    template <int j>
    __device__ __forceinline__ uint32_t pair(uint32_t mw, const uint32_t* lut, const HuffTables& T, const uint32_t* s,
                                             uint32_t maxw, uint32_t& err) {
        constexpr uint32_t sel = j == 0 ? 0x5140u : 0x5342u;
        const uint32_t e = lut[peek >> (32 - kLutBits)];
        const uint32_t len = e >> 26;
        peek = __funnelshift_l(0u, peek, len);
        p += len;
        uint32_t syms = e;
        if ((int32_t)e < 0) {
            p -= 32;
            reload(s, maxw);
            const uint32_t e2 = lut[peek >> (32 - kLutBits)];
            if ((e & 0x001F0000u) && (e2 & 0x001F0000u)) {
                const uint32_t l1 = (e2 >> 16) & 31u;
                p += l1;
                peek = __funnelshift_l(0u, peek, l1);
                syms = (e & 0xFFu) | ((e2 & 0xFFu) << 8);
            } else {
                uint32_t s0 = e & 0xFFu;
                if ((e & 0x001F0000u) == 0) s0 = one(lut, T, s, maxw, err);
                syms = s0 | (one(lut, T, s, maxw, err) << 8);
            }
        }
        return bf16_pair(__byte_perm(mw, syms, sel));
    }
    __device__ __forceinline__ uint4 block(uint2 m, const uint32_t* lut, const HuffTables& T, const uint32_t* s,
                                           uint32_t maxw, uint32_t& err) {
        uint4 o;
        reload(s, maxw);
        o.x = pair<0>(m.x, lut, T, s, maxw, err);
        o.y = pair<1>(m.x, lut, T, s, maxw, err);
        reload(s, maxw);
        o.z = pair<0>(m.y, lut, T, s, maxw, err);
        o.w = pair<1>(m.y, lut, T, s, maxw, err);
        return o;
    }
};

// ---------------------------------------------------------------- the kernel

struct GemmArgs {
    DecodeArgs d;      // the container (whole tensor: g_begin = 0, g_end = n_group)
    const uint16_t* x; // tokens x cols BF16
    float* y;          // tokens x rows FP32
    uint16_t* w_out;   // optional: the decoded W (rows x cols BF16), for checking
    uint32_t rows, cols, tokens;
    uint32_t gpr;      // groups per row
};

template <int NT>  // N = 16 NT accumulator columns (tokens rounded up to 16)
__host__ __device__ constexpr uint32_t gemm_b_stage_bytes() {
    return 16u * NT * kStepK * 2u;
}
template <int NT>
constexpr size_t gemm_dyn_smem_bytes() {
    // 1 KiB of alignment slack, two A stages, two B stages, the pair table
    return 1024 + 2 * (size_t)kAStageBytes + 2 * (size_t)gemm_b_stage_bytes<NT>() + (sizeof(uint32_t) << kLutBits);
}

template <int NT>
__global__ void __launch_bounds__(kGemmThreads, 1) k_decode_gemm(const __grid_constant__ GemmArgs ga) {
    constexpr uint32_t N = 16u * NT;
    constexpr int NX = (int)((N * 32 + kGemmDecodeThreads - 1) / kGemmDecodeThreads);  // B chunks per thread
    constexpr uint32_t kBStage = gemm_b_stage_bytes<NT>();
    __shared__ HuffTables T;
    __shared__ __align__(8) unsigned long long bar_full[2], bar_free[2], bar_done;
    __shared__ uint32_t tmem_slot;
    extern __shared__ __align__(16) uint8_t dyn_smem[];
    const DecodeArgs& a = ga.d;

    // 1024-byte aligned tiles (the swizzle pattern follows address bits 4-9)
    const uint32_t dyn0 = smem_addr(dyn_smem);
    const uint32_t pad = (1024u - (dyn0 & 1023u)) & 1023u;
    const uint32_t sA = dyn0 + pad;                 // two A stages
    const uint32_t sB = sA + 2 * kAStageBytes;      // two B stages
    const uint32_t* lut = reinterpret_cast<const uint32_t*>(dyn_smem + pad + 2 * kAStageBytes + 2 * kBStage);

    const unsigned warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t lo = (uint32_t)((uint64_t)blockIdx.x * ga.rows / gridDim.x);
    const uint32_t hi = (uint32_t)((uint64_t)(blockIdx.x + 1) * ga.rows / gridDim.x);
    const uint32_t rows_t = hi - lo;  // <= 128 (the host sizes the grid)

    if (!build_canonical(a, T)) return;
    build_pair_table(T, const_cast<uint32_t*>(lut));

    if (warp == kGemmDecodeWarps) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(smem_addr(&tmem_slot)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
        if (lane == 0) {
            for (int i = 0; i < 2; i++) {
                mbar_init_count(&bar_full[i], kGemmDecodeWarps);
                mbar_init_count(&bar_free[i], 1);
            }
            mbar_init_count(&bar_done, 1);
            fence_mbar_init();
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_slot;

    const uint32_t S = ga.cols / kStepK;  // steps per row
    const uint32_t spg = a.K / 8;         // steps per group
    uint32_t err = 0;

    if (warp == kGemmDecodeWarps) {
        // ------------------------------------------------------------ MMA warp
        constexpr uint32_t idesc = idesc_bf16_f32(N);
        for (uint32_t t = 0; t < S; t++) {
            const uint32_t st = t & 1u;
            if (!mbar_wait(&bar_full[st], (t >> 1) & 1u)) err |= DFX_STATUS_TIMEOUT;
            tc_fence_after();
            if (lane == 0) {
#pragma unroll
                for (uint32_t at = 0; at < kStepK / 64; at++)
#pragma unroll
                    for (uint32_t kk = 0; kk < 4; kk++) {
                        const uint32_t aa = sA + st * kAStageBytes + at * kGemmTileRows * kAtomBytes + kk * 32u;
                        const uint32_t bb = sB + st * kBStage + at * N * kAtomBytes + kk * 32u;
                        mma_bf16(tmem, smem_desc_sw128(aa), smem_desc_sw128(bb), idesc, (t | at | kk) != 0);
                    }
                mma_commit(&bar_free[st]);
                if (t + 1 == S) mma_commit(&bar_done);
            }
            __syncwarp();
        }
    } else {
        // ------------------------------------------------------------ decoding warps
        const uint32_t* sw = reinterpret_cast<const uint32_t*>(a.comp + a.off_stream);
        const uint32_t maxw = T.n_words - 1;
        const uint8_t* mplane = a.comp + a.off_m;
        const unsigned long long* gbase = reinterpret_cast<const unsigned long long*>(a.comp + kOffGbase);
        const uint16_t* clen = reinterpret_cast<const uint16_t*>(a.comp + a.off_clen);
        const uint32_t nr = rows_t > warp ? (rows_t - warp + kGemmDecodeWarps - 1) / kGemmDecodeWarps : 0u;

        GemmReader rd[kGemmRowSlots];
        uint32_t end[kGemmRowSlots];
        uint2 mcur[kGemmRowSlots], mnext[kGemmRowSlots];
        uint4 xnext[NX];

        // the B tile entries of this thread: token q / 32, 16-byte chunk q mod 32 of the step
        auto load_x = [&](uint32_t t) {
#pragma unroll
            for (int j = 0; j < NX; j++) {
                const uint32_t q = threadIdx.x + kGemmDecodeThreads * j;
                const uint32_t tk = q >> 5, c = q & 31u;
                xnext[j] = q < N * 32 && tk < ga.tokens
                               ? __ldg(reinterpret_cast<const uint4*>(ga.x + (uint64_t)tk * ga.cols + kStepK * t) + c)
                               : make_uint4(0, 0, 0, 0);
            }
        };
        auto load_m = [&](uint32_t t, uint2 (&mm)[kGemmRowSlots]) {
#pragma unroll
            for (int i = 0; i < kGemmRowSlots; i++)
                if ((uint32_t)i < nr) {
                    const uint64_t row = lo + warp + kGemmDecodeWarps * i;
                    mm[i] = __ldg(reinterpret_cast<const uint2*>(mplane + row * ga.cols + kStepK * t) + lane);
                }
        };
        load_x(0);
        load_m(0, mnext);

        for (uint32_t t = 0; t < S; t++) {
            const uint32_t st = t & 1u;
            const uint32_t kstep = t % spg;
#pragma unroll
            for (int i = 0; i < kGemmRowSlots; i++) mcur[i] = mnext[i];
            if (kstep == 0) {
                // a new group in every row: its start bits and this lane's chunk
#pragma unroll
                for (int i = 0; i < kGemmRowSlots; i++)
                    if ((uint32_t)i < nr) {
                        const uint64_t g = (uint64_t)(lo + warp + kGemmDecodeWarps * i) * ga.gpr + t / spg;
                        const unsigned long long gb0 = __ldg(gbase + g), gb1 = __ldg(gbase + g + 1);
                        const uint32_t cl = __ldg(clen + g * 32 + lane);
                        uint32_t incl = cl;
#pragma unroll
                        for (int d = 1; d < 32; d <<= 1) {
                            const uint32_t yv = __shfl_up_sync(kFull, incl, d);
                            if (lane >= (unsigned)d) incl += yv;
                        }
                        const uint32_t sum = __shfl_sync(kFull, incl, 31);
                        const bool ok = gb1 >= gb0 && gb1 <= T.total_bits && gb1 - gb0 == (unsigned long long)sum;
                        if (!ok) err |= DFX_STATUS_INDEX;
                        const uint32_t start = ok ? (uint32_t)(gb0 & 31u) + incl - cl : 0u;
                        rd[i].init(sw, maxw, ok ? (uint32_t)(gb0 >> 5) : 0u, start);
                        end[i] = start + (ok ? cl : 0u);
                    }
            }
            // next step's operands, loaded while this step decodes
            if (t + 1 < S) {
                load_m(t + 1, mnext);
            }
            uint4 xv[NX];
#pragma unroll
            for (int j = 0; j < NX; j++) xv[j] = xnext[j];
            if (t + 1 < S) load_x(t + 1);

            // stage st was last read by the MMAs of step t - 2
            if (t >= 2 && !mbar_wait(&bar_free[st], ((t >> 1) - 1) & 1u)) err |= DFX_STATUS_TIMEOUT;
#pragma unroll
            for (int j = 0; j < NX; j++) {
                const uint32_t q = threadIdx.x + kGemmDecodeThreads * j;
                if (q < N * 32) st_shared_v4(sB + st * kBStage + sw128_offset(N, q >> 5, (q & 31u) >> 3, q & 7u), xv[j]);
            }
#pragma unroll
            for (int i = 0; i < kGemmRowSlots; i++)
                if ((uint32_t)i < nr) {
                    const uint32_t r = warp + kGemmDecodeWarps * i;  // tile row
                    const uint4 o = rd[i].block(mcur[i], lut, T, sw, maxw, err);
                    st_shared_v4(sA + st * kAStageBytes + sw128_offset(kGemmTileRows, r, lane >> 3, lane & 7u), o);
                    if (ga.w_out)
                        reinterpret_cast<uint4*>(ga.w_out + (uint64_t)(lo + r) * ga.cols + kStepK * t)[lane] = o;
                }
            if (kstep + 1 == spg) {
#pragma unroll
                for (int i = 0; i < kGemmRowSlots; i++)
                    if ((uint32_t)i < nr && rd[i].p != end[i]) err |= DFX_STATUS_STREAM;
            }
            fence_proxy_async();  // the tiles are read by the tensor cores (async proxy)
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar_full[st]);
        }

        // ------------------------------------------------------------ epilogue
        if (warp < 4) {
            if (!mbar_wait(&bar_done, 0)) err |= DFX_STATUS_TIMEOUT;
            tc_fence_after();
            const uint32_t r = 32u * warp + lane;  // tile row = tensor-memory lane
#pragma unroll
            for (int j = 0; j < NT; j++) {
                uint32_t v[16];
                tmem_ld16(tmem + ((32u * warp) << 16) + 16u * j, v);
                if (r < rows_t)
#pragma unroll
                    for (int c = 0; c < 16; c++) {
                        const uint32_t tk = 16u * j + c;
                        if (tk < ga.tokens) ga.y[(uint64_t)tk * ga.rows + lo + r] = __uint_as_float(v[c]);
                    }
            }
        }
    }
    if (err) atomicOr(a.status, err);
    tc_fence_before();
    __syncthreads();
    if (warp == kGemmDecodeWarps) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "r"(kTmemCols) : "memory");
    }
}

template <int NT>
cudaError_t launch_gemm_nt(const GemmArgs& g, int grid, cudaStream_t s) {
    static bool attr_set[64] = {};
    const cudaError_t e = allow_smem(k_decode_gemm<NT>, gemm_dyn_smem_bytes<NT>(), attr_set);
    if (e != cudaSuccess) return e;
    k_decode_gemm<NT><<<grid, kGemmThreads, gemm_dyn_smem_bytes<NT>(), s>>>(g);
    return cudaGetLastError();
}

}  // namespace

// Y = X W^T from W's container (Huffman coder); `grid` CTAs, each at most 128 rows.
cudaError_t launch_decode_gemm(const DecodeArgs& d, const uint16_t* x, float* y, uint16_t* w_out, uint32_t rows,
                               uint32_t cols, uint32_t tokens, int grid, cudaStream_t s) {
    GemmArgs g;
    g.d = d;
    g.x = x;
    g.y = y;
    g.w_out = w_out;
    g.rows = rows;
    g.cols = cols;
    g.tokens = tokens;
    g.gpr = cols / (32u * d.K);
    if (tokens == 0 || tokens > kGemmMaxTokens || g.gpr == 0 || cols % (32u * d.K) != 0 ||
        (uint64_t)rows > (uint64_t)grid * kGemmMaxRows)
        return cudaErrorInvalidValue;
    return tokens <= 16 ? launch_gemm_nt<1>(g, grid, s) : launch_gemm_nt<2>(g, grid, s);
}

}  // namespace dfx
