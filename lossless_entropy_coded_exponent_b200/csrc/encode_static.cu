// encode_static.cu -- dfx_encode_static: the encoder for callers that cannot allocate
// device memory.
//
// Some callers of a weight codec may not call cudaMalloc or cudaFree at all: a serving
// process whose device memory belongs to its own pool allocator (it reserves nearly all
// of HBM at start-up, so a raw cudaMalloc either fails or carves memory out from under
// the pool), or a component that must never trigger the implicit device-wide
// synchronisation cudaFree can cause.  dfx_plan allocates a status word and dfx_encode
// needs a workspace from the caller; this entry point needs neither.  Its scratch (the
// exponent histogram, the code tables and the per-group bit counts) lives in a
// fixed-size array in the library's own device memory, created with the module.
//
// Limits and sharing:
//   * at most kStaticMaxGroups = 262144 groups of 32 chunks, i.e. n <= 2^28 with K = 32,
//     2^29 with K = 64 and 2^30 with K = 128; larger tensors get DFX_ERR_CAPACITY;
//   * the array costs 1 MiB + 4.25 KiB on every GPU that loads the library, until the
//     process exits;
//   * every call on a device uses the same array, and the array keeps the previous call's
//     contents (the histogram is cleared by each call; everything else is overwritten
//     before it is read).  Two calls whose GPU work overlaps (different streams, or host
//     threads without ordering between them) race on it and corrupt each other's output:
//     order them on one stream or with events;
//   * every call looks up the array's device address in the current context
//     (cudaGetSymbolAddress) instead of keeping it from an earlier call: after a
//     cudaDeviceReset, or in another context on the same device, the module and its array
//     are loaded again at another address.  The first call in a context loads the module
//     there; make that first call before any stream capture.
#include <cuda_runtime.h>
#include <stdint.h>

#include "dfx.h"
#include "dfx_common.cuh"

namespace {

constexpr uint64_t kStaticMaxGroups = 262144;
constexpr uint64_t kStaticWorkspace = dfx::ws_edge_offset(kStaticMaxGroups) + 8 * (kStaticMaxGroups + 1);
constexpr uint64_t kStaticStatus = kStaticWorkspace;          // one u32, unused by encode kernels
constexpr uint64_t kStaticBytes = kStaticWorkspace + 256;

static __device__ __align__(256) uint8_t g_static_scratch[kStaticBytes];

}  // namespace

extern "C" int dfx_encode_static(const void* d_bf16, uint64_t n, const dfx_params* params, void* d_out,
                                 size_t out_capacity, size_t* h_compressed_bytes, cudaStream_t stream) {
    if (n >= (1ull << 32)) return DFX_ERR_TOO_LARGE;
    const uint32_t K = (params && params->chunk_symbols) ? params->chunk_symbols : 128u;
    const uint32_t G = (params && params->group_chunks) ? params->group_chunks : 32u;
    const uint32_t L = (params && params->max_len) ? params->max_len : 24u;
    if (L < 8 || L > dfx::kMaxLenLimit || K < 8 || K % 8 != 0) return DFX_ERR_ARG;
    if (params && dfx::is_tans(params->coder)) return DFX_ERR_UNSUPPORTED;
    if (params && params->coder != DFX_CODER_HUFFMAN) return DFX_ERR_ARG;
    if (!dfx::decode_supports(K, G)) return DFX_ERR_UNSUPPORTED;
    if (!d_out || (!d_bf16 && n)) return DFX_ERR_ARG;
    if (((uintptr_t)d_bf16 & 15u) || ((uintptr_t)d_out & 15u)) return DFX_ERR_ARG;
    const dfx::Layout lay = dfx::make_layout(n, K, G);
    if (lay.n_group > kStaticMaxGroups) return DFX_ERR_CAPACITY;
    const uint64_t max_bytes = lay.off_stream + dfx::stream_bytes(8 * n);
    if (out_capacity < max_bytes) return DFX_ERR_CAPACITY;

    // In host code g_static_scratch names a host-side stand-in, not device memory: the
    // kernels get the array's address in the current context, looked up on every call.
    uint8_t* scratch = nullptr;
    {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || !p) {
            cudaGetLastError();
            return DFX_ERR_CUDA;
        }
        scratch = (uint8_t*)p;
    }

    dfx::EncodeArgs a;
    a.in = (const uint16_t*)d_bf16;
    a.out = (uint8_t*)d_out;
    a.n = n;
    a.K = K;
    a.G = G;
    a.max_len = L;
    a.coder = DFX_CODER_HUFFMAN;
    a.table_log = 0;
    a.n_chunk = (uint32_t)lay.n_chunk;
    a.n_group = (uint32_t)lay.n_group;
    a.off_gbase = lay.off_gbase;
    a.off_clen = lay.off_clen;
    a.off_m = lay.off_m;
    a.off_stream = lay.off_stream;
    a.ws_counts = (unsigned long long*)(scratch + dfx::kWsCounts);
    a.ws_code = (uint32_t*)(scratch + dfx::kWsCode);
    a.ws_len = scratch + dfx::kWsLen;
    a.ws_group_bits = (uint32_t*)(scratch + dfx::kWsGroupBits);
    a.ws_edge = (unsigned long long*)(scratch + dfx::ws_edge_offset(lay.n_group));
    a.ws_tans = nullptr;
    a.status = (uint32_t*)(scratch + kStaticStatus);
    a.max_bytes = max_bytes;
    if (dfx::launch_encode(a, max_bytes, stream) != cudaSuccess) {
        cudaGetLastError();
        return DFX_ERR_CUDA;
    }
    if (h_compressed_bytes) {
        unsigned long long total = 0;
        if (cudaMemcpyAsync(&total, a.out + 24, 8, cudaMemcpyDeviceToHost, stream) != cudaSuccess ||
            cudaStreamSynchronize(stream) != cudaSuccess) {
            cudaGetLastError();
            return DFX_ERR_CUDA;
        }
        *h_compressed_bytes = (size_t)total;
    }
    return DFX_OK;
}
