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
// One CTA of 26 warps (one per SM) takes a tile of at most 100 rows of W (the MMA's
// M = 128 covers them):
//   * every thread first helps build the Huffman tables in shared memory: the canonical
//     per-length limits and a pair table on the next 13 stream bits (huffman_tables.cuh;
//     32 KiB, half the decode kernel's);
//   * 25 decoding warps hold up to 4 rows each, tile row R in warp R mod 25 (a warp without
//     a row sits out); eight lanes share a row, so a tile of 97 rows (14336 rows on 148
//     SMs) leaves 3 of 100 lane groups idle.  A group's 32 chunks are decoded in 4 rounds
//     of 8: in round j lane q of
//     a row decodes chunk 8 (j mod 4) + q from its first code to its last, 8 codes (one
//     block) at a time, with the decode kernel's reader, from a shared-memory copy of the
//     round's stream slice that the bulk-copy engine brought in during the previous round;
//   * the sum over K of X W^T does not depend on the order of K, so the kernel takes K in
//     the order it decodes it: one block of the eight chunks of a round, 64 weights per
//     row, makes one K atom of A, 128 rows x 128 bytes (the canonical K-major layout with
//     the 128-byte swizzle: in each 8-row group, row r's 16-byte chunk c sits at chunk
//     c ^ (r mod 8)); two consecutive blocks make one pipeline stage.  The MMA warp copies
//     the same columns of X into the stage's B tile with 16-byte asynchronous copies
//     (cp.async), one stage ahead;
//   * the MMA warp waits for a stage's A (every decoding warp arrives on its barrier),
//     issues 8 tcgen05.mma (M = 128, N = tokens rounded up to 16, K = 16) accumulating in
//     tensor memory and commits them to the stage's "free" barrier, which the decoding
//     warps (and the next B copy) wait on before they write the stage again, kStages
//     stages later;
//   * after the last stage, decoding warps 0-3 read the accumulator (tensor-memory lanes
//     32 w .. 32 w + 31 are tile rows) and write Y.
// Every wait is bounded: a wait that runs out sets DFX_STATUS_TIMEOUT and the kernel
// carries on (with a wrong Y) and releases its tensor memory.  A corrupt container sets
// the same status bits as dfx_decode and never makes the kernel read outside it or
// outside its own shared memory.
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include "decode_pipeline.cuh"
#include "huffman_reader.cuh"
#include "huffman_tables.cuh"

namespace dfx {
namespace {

constexpr int kGemmLutBits = 13;      // pair table index bits
constexpr int kGemmDecodeWarps = 25;  // + the MMA warp: 26 warps of up to 72 registers
constexpr int kGemmLanesPerRow = 8;
constexpr int kGemmRowSlots = 32 / kGemmLanesPerRow;  // rows per decoding warp
static_assert(kGemmMaxRows <= kGemmDecodeWarps * kGemmRowSlots, "rows per tile at most");
constexpr int kGemmTileRows = 128;    // MMA M (tile rows past the tile's own are never stored)
static_assert(kGemmMaxRows <= kGemmTileRows, "the rows of a tile fit the MMA's M = 128");
constexpr int kGemmThreads = (kGemmDecodeWarps + 1) * 32;
constexpr uint32_t kRoundsPerGroup = 32 / kGemmLanesPerRow;
constexpr uint32_t kAtomBytes = 128;                           // one swizzle row: 64 BF16
constexpr uint32_t kStageAtoms = 2;                            // K atoms (blocks of the round) per stage
constexpr uint32_t kAAtomBytes = kGemmTileRows * kAtomBytes;    // 16 KiB: 128 rows x 64 K
constexpr uint32_t kAStageBytes = kStageAtoms * kAAtomBytes;    // 32 KiB
constexpr uint32_t kStages = 2;
constexpr uint32_t kTmemCols = 32;                             // FP32 accumulator columns
constexpr uint32_t kSliceBytes = 416;                          // a row's stream slice for one round
constexpr uint32_t kSliceWords = kSliceBytes / 4;
static_assert(kSliceBytes % 16 == 0, "bulk copies move 16-byte units");

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
// 16 bytes from global src to shared dst without a register stage; zeros when !valid
__device__ __forceinline__ void cp_async16_zfill(uint32_t dst, const void* src, bool valid) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(valid ? 16u : 0u)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
// waits until at most the newest committed group of this thread's copies is in flight
__device__ __forceinline__ void cp_async_wait_prior() { asm volatile("cp.async.wait_group 1;\n" ::: "memory"); }
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

// ---------------------------------------------------------------- the kernel

// A row's staged stream slice: loads clamped to the slot's buffer, so a corrupt stream
// never reads outside the warp's own buffers.
struct SlotWords {
    uint32_t s;  // shared-memory address of the slice
    __device__ __forceinline__ uint32_t load(uint32_t i) const {
        uint32_t v;
        asm volatile("ld.shared.u32 %0, [%1];\n" : "=r"(v) : "r"(s + 4u * min(i, kSliceWords - 1)));
        return v;
    }
};

struct GemmArgs {
    DecodeArgs d;      // the container (whole tensor: g_begin = 0, g_end = n_group)
    const uint16_t* x; // tokens x cols BF16
    float* y;          // tokens x rows FP32
    uint16_t* w_out;   // optional: the decoded W (rows x cols BF16), for checking
    uint32_t rows, cols, tokens;
    uint32_t gpr;      // groups per row
};

// Per decoding warp: the index of its rows' current group and two buffers of round slices.
struct GemmWarp {
    uint32_t incl[kGemmRowSlots][32];  // inclusive chunk-bit prefix of each row's group
    unsigned long long gb0[kGemmRowSlots];
    uint32_t base[2][kGemmRowSlots];   // per buffer and row: stream word of the first staged word
    uint32_t staged[2];                // per buffer: bit r set when row r's slice is staged
    unsigned long long bar[2];
    __align__(16) uint32_t slice[2][kGemmRowSlots][kSliceWords];
};

template <int NT>  // N = 16 NT accumulator columns (tokens rounded up to 16)
__host__ __device__ constexpr uint32_t gemm_b_stage_bytes() {
    return kStageAtoms * 16u * NT * kAtomBytes;
}
template <int NT>
constexpr size_t gemm_dyn_smem_bytes() {
    // 1 KiB of alignment slack, the A and B stages, the pair table, the warps' buffers
    return 1024 + kStages * (size_t)(kAStageBytes + gemm_b_stage_bytes<NT>()) + (sizeof(uint32_t) << kGemmLutBits) +
           kGemmDecodeWarps * sizeof(GemmWarp);
}
static_assert(gemm_dyn_smem_bytes<2>() + 1536 <= 227 * 1024, "shared memory");

template <int NT>
__global__ void __launch_bounds__(kGemmThreads, 1) k_decode_gemm(const __grid_constant__ GemmArgs ga) {
    constexpr uint32_t N = 16u * NT;
    constexpr uint32_t kBStage = gemm_b_stage_bytes<NT>();
    __shared__ HuffTables T;
    __shared__ __align__(8) unsigned long long bar_full[kStages], bar_free[kStages], bar_done;
    __shared__ uint32_t tmem_slot;
    extern __shared__ __align__(16) uint8_t dyn_smem[];
    const DecodeArgs& a = ga.d;

    // 1024-byte aligned tiles (the swizzle pattern follows address bits 4-9)
    const uint32_t dyn0 = smem_addr(dyn_smem);
    const uint32_t pad = (1024u - (dyn0 & 1023u)) & 1023u;
    const uint32_t sA = dyn0 + pad;                   // kStages A stages
    const uint32_t sB = sA + kStages * kAStageBytes;  // kStages B stages
    uint8_t* after_b = dyn_smem + pad + kStages * (kAStageBytes + kBStage);
    uint32_t* lut = reinterpret_cast<uint32_t*>(after_b);
    GemmWarp* warps = reinterpret_cast<GemmWarp*>(after_b + (sizeof(uint32_t) << kGemmLutBits));

    const unsigned warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t lo = (uint32_t)((uint64_t)blockIdx.x * ga.rows / gridDim.x);
    const uint32_t hi = (uint32_t)((uint64_t)(blockIdx.x + 1) * ga.rows / gridDim.x);
    const uint32_t rows_t = hi - lo;  // <= 120 (the host sizes the grid)
    const uint32_t busy = min(rows_t, (uint32_t)kGemmDecodeWarps);  // decoding warps with rows

    // launched as a programmatic dependent: without DFX_DECODE_EARLY_READ wait for the
    // preceding kernel here; with it, only before reading X and before writing Y or W
    enter_dependent(a);
    if (!build_canonical(a, T)) return;
    const uint32_t bpr = a.K / 8;                       // blocks per chunk: stages per round
    const uint32_t rounds = ga.gpr * kRoundsPerGroup;  // rounds per row
    const uint32_t spr = bpr / kStageAtoms;              // stages per round (bpr is even)
    const uint32_t n_stages = rounds * spr;             // stages per tile
    uint32_t err = 0;

    // the MMA warp's state
    constexpr uint32_t idesc = idesc_bf16_f32(N);
    constexpr uint32_t NX = kStageAtoms * N * 8 / 32;  // 16-byte pieces per lane and stage
    // B of stage i into stage buffer sb with 16-byte asynchronous copies (tokens past
    // `tokens` read as zeros).  Piece q: atom q / 8N, token t, 16-byte column chunk c; the
    // atom holds block k0 + atom of chunks 8 jj .. 8 jj + 7 of group grp (round j = i / spr)
    auto copy_x = [&](uint32_t i, uint32_t sb) {
        const uint32_t j = i / spr, k0 = kStageAtoms * (i % spr), grp = j / kRoundsPerGroup, jj = j % kRoundsPerGroup;
#pragma unroll
        for (uint32_t u = 0; u < NX; u++) {
            const uint32_t q = lane + 32u * u, at = q / (8u * N), t = (q % (8u * N)) / 8, c = q % 8;
            const uint32_t pos = grp * 32u * a.K + (32u * (k0 + at) + kGemmLanesPerRow * jj + c) * 8u;
            const bool valid = t < ga.tokens;
            cp_async16_zfill(sB + sb * kBStage + at * (N * kAtomBytes) + sw128_offset(N, t, 0, c),
                             ga.x + (valid ? (uint64_t)t * ga.cols + pos : 0u), valid);
        }
    };

    // the decoding warps' state (warp < busy)
    GemmWarp& W = warps[warp < kGemmDecodeWarps ? warp : 0];
    const uint32_t* sw = reinterpret_cast<const uint32_t*>(a.comp + a.off_stream);
    const uint32_t maxw = T.n_words - 1;
    const uint8_t* mplane = a.comp + a.off_m;
    const unsigned long long* gbase = reinterpret_cast<const unsigned long long*>(a.comp + kOffGbase);
    const uint16_t* clen = reinterpret_cast<const uint16_t*>(a.comp + a.off_clen);
    const uint32_t slot = lane / kGemmLanesPerRow, q = lane % kGemmLanesPerRow;
    const uint32_t R = warp + kGemmDecodeWarps * slot;  // this lane's tile row
    const bool live = R < rows_t;
    const uint64_t row = lo + R;

    // group grp's index for every row of the warp (lane = chunk)
    auto load_group = [&](uint32_t grp) {
        unsigned long long g0[kGemmRowSlots], g1[kGemmRowSlots];
        uint32_t cl[kGemmRowSlots];
#pragma unroll
        for (int r = 0; r < kGemmRowSlots; r++) {
            if (warp + kGemmDecodeWarps * r < rows_t) {
                const uint64_t g = (uint64_t)(lo + warp + kGemmDecodeWarps * r) * ga.gpr + grp;
                g0[r] = __ldg(gbase + g);
                g1[r] = __ldg(gbase + g + 1);
                cl[r] = __ldg(clen + g * 32 + lane);
            }
        }
#pragma unroll
        for (int r = 0; r < kGemmRowSlots; r++) {
            if (warp + kGemmDecodeWarps * r >= rows_t) continue;  // the same for every lane
            uint32_t incl = cl[r];
#pragma unroll
            for (int d = 1; d < 32; d <<= 1) {
                const uint32_t yv = __shfl_up_sync(kFull, incl, d);
                if (lane >= (unsigned)d) incl += yv;
            }
            const uint32_t sum = __shfl_sync(kFull, incl, 31);
            const bool ok = g1[r] >= g0[r] && g1[r] <= T.total_bits && g1[r] - g0[r] == (unsigned long long)sum;
            if (!ok) err |= DFX_STATUS_INDEX;
            W.incl[r][lane] = ok ? incl : 0u;
            if (lane == 0) W.gb0[r] = ok ? g0[r] : 0ull;
        }
        __syncwarp();
    };
    // lanes 0 .. kGemmRowSlots - 1: copy round j's slice of row slot `lane` into buffer
    // b (or arrive without a copy when the row is empty or its slice does not fit)
    auto stage_round = [&](uint32_t j, uint32_t b) {
        if (lane < kGemmRowSlots) {
            const uint32_t r = lane, c0 = kGemmLanesPerRow * (j % kRoundsPerGroup);
            uint32_t bytes = 0;
            if (warp + kGemmDecodeWarps * r < rows_t) {
                const unsigned long long s0 = W.gb0[r] + (c0 ? W.incl[r][c0 - 1] : 0u);
                const unsigned long long s1 = W.gb0[r] + W.incl[r][c0 + kGemmLanesPerRow - 1];
                const uint32_t beg = ((uint32_t)(s0 >> 5) * 4u) & ~15u;
                const uint32_t end = min((((uint32_t)(s1 >> 5) + 4u) * 4u + 15u) & ~15u, T.n_words * 4u);
                W.base[b][r] = beg / 4u;
                if (end > beg && end - beg <= kSliceBytes) bytes = end - beg;
            }
            const uint32_t mask = __ballot_sync((1u << kGemmRowSlots) - 1u, bytes != 0);
            if (lane == 0) W.staged[b] = mask;
            __syncwarp((1u << kGemmRowSlots) - 1u);
            fence_proxy_async();  // the buffer's previous contents were read (generic proxy)
            if (bytes) bulk_copy(W.slice[b][r], a.comp + a.off_stream + 4ull * W.base[b][r], bytes, &W.bar[b]);
            else mbar_arrive(&W.bar[b]);
        }
        __syncwarp();
    };
    // the m bytes of this lane's chunk in round j: block k at m_base(j) + 32 k (uint2)
    auto m_base = [&](uint32_t j) -> const uint2* {
        const uint32_t grp = j / kRoundsPerGroup, c = kGemmLanesPerRow * (j % kRoundsPerGroup) + q;
        return reinterpret_cast<const uint2*>(mplane + row * ga.cols + grp * 32u * a.K) + c;
    };
    const uint32_t a_off = sA + sw128_offset(kGemmTileRows, R, 0, q);  // this lane's 16 bytes of an A stage

    uint32_t sphase = 0;  // parity of each round buffer's next phase
    // the m bytes of the next two blocks (block k in mq[k % 2]); at a round's end the ring
    // runs on into the next round's first blocks
    uint2 mq[2] = {make_uint2(0, 0), make_uint2(0, 0)};
    const uint2* mp = nullptr;

    // Start-up: the MMA warp allocates the accumulator, sets up the stage barriers and
    // loads the first B stage; each decoding warp loads its rows' first group index and
    // starts its first round's copies and m loads; all of them in flight while every
    // thread then builds the pair table.
    if (warp == kGemmDecodeWarps) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(smem_addr(&tmem_slot)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
        if (lane == 0) {
            for (uint32_t i = 0; i < kStages; i++) {
                mbar_init_count(&bar_full[i], busy);
                mbar_init_count(&bar_free[i], 1);
            }
            mbar_init_count(&bar_done, 1);
            fence_mbar_init();
        }
        if (a.early) wait_prior_grid();
        copy_x(0, 0);
        cp_async_commit();
    } else {
        // slices start zeroed: a lane without a row decodes zeros from its never-staged slot
        uint4* z = reinterpret_cast<uint4*>(&W.slice[0][0][0]);
        for (uint32_t k = lane; k < sizeof(W.slice) / 16; k += 32) z[k] = make_uint4(0, 0, 0, 0);
        fence_proxy_async();  // before the bulk copies into the same buffers
        if (lane == 0) {
            for (int b = 0; b < 2; b++) mbar_init_count(&W.bar[b], kGemmRowSlots);
            fence_mbar_init();
        }
        __syncwarp();
        if (warp < busy) {
            if (a.early && ga.w_out) wait_prior_grid();
            load_group(0);
            stage_round(0, 0);
            mp = m_base(0);
            mq[0] = live ? __ldg(mp) : make_uint2(0, 0);
            mq[1] = live ? __ldg(mp + 32) : make_uint2(0, 0);
        }
    }
    build_pair_table<kGemmLutBits>(T, lut);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_slot;

    if (warp == kGemmDecodeWarps) {
        // ------------------------------------------------------------ MMA warp: B tiles, MMAs
        // Stage i's B tile is X's 64 columns that hold block k of chunks 8 jj .. 8 jj + 7 of
        // group grp (round j = kRoundsPerGroup grp + jj = i / bpr, k = i mod bpr), all tokens
        // (rows past `tokens` zero): the warp loads the next stage's 16-byte pieces while the
        // decoding warps fill the current stage's A, and stores them swizzled once the MMAs
        // that last read the buffer have completed.
        uint32_t st = 0, ph = 0;
        for (uint32_t i = 0; i < n_stages; i++) {
            // the next stage's B, into the buffer the MMAs of stage i + 1 - kStages read
            if (i + 1 < n_stages) {
                const uint32_t nb = st + 1 == kStages ? 0u : st + 1;
                if (i + 1 >= kStages && !mbar_wait(&bar_free[nb], ((i + 1 - kStages) / kStages) & 1u))
                    err |= DFX_STATUS_TIMEOUT;
                copy_x(i + 1, nb);
            }
            cp_async_commit();
            cp_async_wait_prior();  // every group but the newest: stage i's B has landed
            fence_proxy_async();    // B is read by the tensor cores
            __syncwarp();
            if (!mbar_wait(&bar_full[st], ph)) err |= DFX_STATUS_TIMEOUT;
            tc_fence_after();
            if (lane == 0) {
#pragma unroll
                for (uint32_t at = 0; at < kStageAtoms; at++)
#pragma unroll
                    for (uint32_t kk = 0; kk < 4; kk++)
                        mma_bf16(tmem, smem_desc_sw128(sA + st * kAStageBytes + at * kAAtomBytes + kk * 32u),
                                 smem_desc_sw128(sB + st * kBStage + at * (N * kAtomBytes) + kk * 32u), idesc,
                                 (i | at | kk) != 0);
                mma_commit(&bar_free[st]);
                if (i + 1 == n_stages) mma_commit(&bar_done);
            }
            __syncwarp();
            if (++st == kStages) {
                st = 0;
                ph ^= 1u;
            }
        }
    } else if (warp < busy) {
        // ------------------------------------------------------------ decoding warps
        uint32_t st = 0, ph = 0;  // stage buffer of the current stage and the parity of its use
        bool reuse = false;       // the stage buffers have been used once (their frees are awaited)
        for (uint32_t j = 0; j < rounds; j++) {
            const uint32_t b = j & 1u, c = kGemmLanesPerRow * (j % kRoundsPerGroup) + q;
            // this lane's chunk: start (relative to the group) and bits, read before the
            // next group's index replaces them
            uint32_t c_start = 0, c_bits = 0;
            unsigned long long g_start = 0;
            if (live) {
                const uint32_t e = W.incl[slot][c];
                c_start = c ? W.incl[slot][c - 1] : 0u;
                c_bits = e - c_start;
                g_start = W.gb0[slot];
            }
            __syncwarp();
            // the next round's slice (a new group's index first)
            if (j + 1 < rounds) {
                if ((j + 1) % kRoundsPerGroup == 0) load_group((j + 1) / kRoundsPerGroup);
                stage_round(j + 1, b ^ 1u);
            }
            if (!mbar_wait(&W.bar[b], (sphase >> b) & 1u)) err |= DFX_STATUS_TIMEOUT;
            sphase ^= 1u << b;
            const bool staged = (W.staged[b] >> slot) & 1u;
            const unsigned long long p0 = g_start + c_start;  // the chunk's first stream bit
            const uint2* mnext = j + 1 < rounds ? m_base(j + 1) : mp;  // the next round's m bytes
            // decode the round: every lane runs the same steps; a lane without a row stores
            // nothing and its reader reads the slot's zeroed buffer (or word 0 of the stream)
            auto run = [&](auto& br) {
                for (uint32_t k0 = 0; k0 < bpr; k0 += 2) {  // bpr is even
#pragma unroll
                    for (uint32_t h = 0; h < 2; h++) {
                        const uint32_t k = k0 + h;
                        const uint2 m = mq[h];
                        // the m bytes two blocks on (in the next round at a round's end)
                        if (live) mq[h] = k + 2 < bpr ? __ldg(mp + 32u * (k + 2)) : __ldg(mnext + 32u * (k + 2 - bpr));
                        const uint4 o = decode_block(br, T, m, err);
                        if (h == 0 && reuse && !mbar_wait(&bar_free[st], ph ^ 1u)) err |= DFX_STATUS_TIMEOUT;
                        if (live) {
                            st_shared_v4(a_off + st * kAStageBytes + h * kAAtomBytes, o);
                            if (ga.w_out)
                                *reinterpret_cast<uint4*>(ga.w_out + row * ga.cols + ga.cols / ga.gpr * (j / kRoundsPerGroup) +
                                                          (32u * k + c) * 8u) = o;
                        }
                        if (h + 1 == kStageAtoms) {  // the stage is complete
                            fence_proxy_async();  // A is read by the tensor cores
                            __syncwarp();
                            if (lane == 0) mbar_arrive(&bar_full[st]);
                            if (++st == kStages) {
                                st = 0;
                                ph ^= 1u;
                                reuse = true;
                            }
                        }
                    }
                }
                if (live && br.consumed() != c_bits) err |= DFX_STATUS_STREAM;
            };
            if (__all_sync(kFull, staged || !live)) {
                BitReader<SlotWords, kGemmLutBits> br;
                const uint32_t rel = live ? (uint32_t)(p0 - 32ull * W.base[b][slot]) : 0u;
                br.init(lut, SlotWords{smem_addr(W.slice[b][slot])}, rel);
                run(br);
            } else {
                // a slice that did not fit: the whole warp reads this round from global memory
                const uint32_t first = live ? (uint32_t)(p0 >> 5) : 0u;
                BitReader<ClampedGlobalWords, kGemmLutBits> br;
                br.init(lut, ClampedGlobalWords{sw + first, maxw - first}, live ? (uint32_t)(p0 & 31u) : 0u);
                run(br);
            }
            mp = mnext;
        }

        // ------------------------------------------------------------ epilogue
        if (warp < 4) {
            if (a.early) wait_prior_grid();
            if (!mbar_wait(&bar_done, 0)) err |= DFX_STATUS_TIMEOUT;
            tc_fence_after();
            const uint32_t r = 32u * warp + lane;  // tile row = tensor-memory lane
#pragma unroll
            for (int jn = 0; jn < NT; jn++) {
                uint32_t v[16];
                tmem_ld16(tmem + ((32u * warp) << 16) + 16u * jn, v);
                if (r < rows_t)
#pragma unroll
                    for (int cc = 0; cc < 16; cc++) {
                        const uint32_t tk = 16u * jn + cc;
                        if (tk < ga.tokens) ga.y[(uint64_t)tk * ga.rows + lo + r] = __uint_as_float(v[cc]);
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
    return launch_programmatic(k_decode_gemm<NT>, grid, kGemmThreads, gemm_dyn_smem_bytes<NT>(), s, g);
}

}  // namespace

// Y = X W^T from W's container (Huffman coder); `grid` CTAs, each at most 128 rows.
cudaError_t launch_decode_gemm(const DecodeArgs& d, const uint16_t* x, float* y, uint16_t* w_out, uint32_t rows,
                               uint32_t cols, uint32_t tokens, int grid, cudaStream_t s) {
    GemmArgs g;
    memset(&g, 0, sizeof(g));
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
