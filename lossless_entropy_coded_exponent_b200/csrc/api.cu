// api.cu -- the C ABI declared in include/dfx.h: argument checks, plans, launches.
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include "dfx.h"
#include "dfx_common.cuh"

struct dfx_plan_s {
    uint64_t n;
    uint32_t K, G, max_len;
    uint32_t coder, table_log;  // exponent coder; tANS table log (coder 1)
    uint32_t decode_flags;      // DFX_DECODE_*
    dfx::Layout L;
    uint64_t max_bytes;
    uint64_t ws_bytes;
    uint32_t* d_status;
    int device;
    int sms;  // streaming multiprocessors of the device
    int decode_grid;
    int resident_ctas;  // decode CTAs that fit on the device at once
    // events ordering dfx_decode_host's copies before the decode of their slices,
    // created on first use
    static constexpr uint32_t kHostSlicesMax = 64;
    cudaEvent_t slice_done[kHostSlicesMax];
    // recorded on the decode stream when dfx_decode_host starts: its copies into the
    // staging buffer wait for the decoding already queued there (an earlier call's
    // slices may still be reading the buffer)
    cudaEvent_t decode_idle;
    bool events_made;
};

namespace {

struct Params {
    uint32_t K, G, L, coder, R, flags;
};

// Defaults and checks of dfx_params.  Only the fields of the chosen coder are checked:
// max_len for coder 0, table_log for coders 1 and 2.
int resolve_params(const dfx_params* p, Params* r) {
    r->K = (p && p->chunk_symbols) ? p->chunk_symbols : 128u;
    r->G = (p && p->group_chunks) ? p->group_chunks : 32u;
    r->L = (p && p->max_len) ? p->max_len : 24u;
    r->coder = p ? p->coder : DFX_CODER_HUFFMAN;
    r->R = (p && p->table_log) ? p->table_log : dfx::kTansMaxLog;
    r->flags = p ? p->decode_flags : 0u;
    if (r->flags & ~(uint32_t)DFX_DECODE_EARLY_READ) return DFX_ERR_ARG;
    if (r->K < 8 || r->K % 8 != 0) return DFX_ERR_ARG;  // chunks are made of 8-element blocks
    if (r->coder == DFX_CODER_HUFFMAN) {
        if (r->L < 8 || r->L > dfx::kMaxLenLimit) return DFX_ERR_ARG;
        if ((uint64_t)r->K * r->L > 65535u) return DFX_ERR_ARG;  // a chunk's bit length must fit u16
        r->R = 0;
    } else if (dfx::is_tans(r->coder)) {
        if (r->R < dfx::kTansMinLog || r->R > dfx::kTansMaxLog) return DFX_ERR_ARG;
        // fields and states fit u16
        if ((uint64_t)(r->K + dfx::tans_states(r->coder)) * r->R > 65535u) return DFX_ERR_ARG;
        r->L = 0;
    } else {
        return DFX_ERR_ARG;
    }
    return DFX_OK;
}

// Longest stream a coder may produce: at most 8 bits per exponent for an optimal prefix
// code, at most table_log bits per exponent and per chunk state for tANS.
uint64_t max_stream_bits(const Params& q, uint64_t n, uint64_t n_chunk) {
    return dfx::is_tans(q.coder) ? (uint64_t)q.R * (n + dfx::tans_states(q.coder) * n_chunk) : 8 * n;
}

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

uint32_t g_inject = 0;  // dfx_debug_inject

// Host checks of one decode and its kernel arguments.
int make_decode_args(const dfx_plan_s* plan, const void* d_comp, size_t comp_bytes, void* d_bf16, dfx::DecodeArgs* a);

int check_device(const dfx_plan_s* plan) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return DFX_ERR_CUDA;
    return dev == plan->device ? DFX_OK : DFX_ERR_ARG;
}

}  // namespace

extern "C" {

uint32_t dfx_version(void) { return (1u << 16) | 0u; }

int dfx_debug_inject(uint32_t flags) {
    if (flags & ~(uint32_t)DFX_INJECT_SKIP_SLICE_COPY) return DFX_ERR_ARG;
    g_inject = flags;
    return DFX_OK;
}

const char* dfx_strerror(int code) {
    switch (code) {
        case DFX_OK: return "ok";
        case DFX_ERR_ARG: return "invalid argument (pointer, size, alignment or parameter)";
        case DFX_ERR_CAPACITY: return "output or workspace buffer too small";
        case DFX_ERR_CORRUPT: return "container is malformed";
        case DFX_ERR_TOO_LARGE: return "tensor too large (n must be below 2^32)";
        case DFX_ERR_CUDA: return "CUDA runtime error";
        case DFX_ERR_UNSUPPORTED: return "parameters not implemented by the GPU path";
        default: return "unknown error code";
    }
}

int dfx_container_layout(uint64_t n, const dfx_params* params, uint64_t total_bits, dfx_layout* out) {
    if (!out) return DFX_ERR_ARG;
    if (n >= (1ull << 32)) return DFX_ERR_TOO_LARGE;
    Params q;
    int rc = resolve_params(params, &q);
    if (rc) return rc;
    if (q.G < 1) return DFX_ERR_ARG;
    const dfx::Layout lay = dfx::make_layout(n, q.K, q.G, q.coder);
    out->n = n;
    out->n_chunk = lay.n_chunk;
    out->n_group = lay.n_group;
    out->off_len = dfx::is_tans(q.coder) ? dfx::kOffFreq : dfx::kOffLen;
    out->off_gbase = lay.off_gbase;
    out->off_clen = lay.off_clen;
    out->off_m = lay.off_m;
    out->off_stream = lay.off_stream;
    out->stream_bytes = dfx::stream_bytes(total_bits);
    out->total_bytes = lay.off_stream + out->stream_bytes;
    return DFX_OK;
}

int dfx_plan(dfx_plan_t* plan, uint64_t n, const dfx_params* params, size_t* max_compressed_bytes,
             size_t* workspace_bytes) {
    if (!plan) return DFX_ERR_ARG;
    *plan = nullptr;
    if (n >= (1ull << 32)) return DFX_ERR_TOO_LARGE;
    Params q;
    int rc = resolve_params(params, &q);
    if (rc) return rc;
    const uint32_t K = q.K, G = q.G;
    if (!dfx::decode_supports(K, G)) return DFX_ERR_UNSUPPORTED;

    dfx_plan_s* p = (dfx_plan_s*)calloc(1, sizeof(dfx_plan_s));
    if (!p) return DFX_ERR_ARG;
    p->n = n;
    p->K = K;
    p->G = G;
    p->max_len = q.L;
    p->coder = q.coder;
    p->table_log = q.R;
    p->decode_flags = q.flags;
    p->L = dfx::make_layout(n, K, G, q.coder);
    p->max_bytes = p->L.off_stream + dfx::stream_bytes(max_stream_bits(q, n, p->L.n_chunk));
    p->ws_bytes = dfx::workspace_bytes_for(p->L.n_group, q.coder);
    int sms = 0;
    if (cudaGetDevice(&p->device) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, p->device) != cudaSuccess ||
        cudaMalloc((void**)&p->d_status, 256) != cudaSuccess || cudaMemset(p->d_status, 0, 256) != cudaSuccess) {
        cudaGetLastError();
        if (p->d_status) cudaFree(p->d_status);
        free(p);
        return DFX_ERR_CUDA;
    }
    p->sms = sms;
    const uint64_t resident = dfx::decode_blocks_per_sm(K, q.coder) * (uint64_t)sms;  // CTAs that fit at once
    p->resident_ctas = (int)resident;
    const uint64_t wpb = (uint64_t)dfx::decode_warps_per_block(K);
    const uint64_t need = (p->L.n_group + wpb - 1) / wpb;                    // CTAs with work (a warp per group)
    p->decode_grid = (int)(need == 0 ? 1 : (need < resident ? need : resident));
    if (max_compressed_bytes) *max_compressed_bytes = (size_t)p->max_bytes;
    if (workspace_bytes) *workspace_bytes = (size_t)p->ws_bytes;
    *plan = p;
    return DFX_OK;
}

int dfx_encode(dfx_plan_t plan, const void* d_bf16, void* d_out, size_t out_capacity, void* d_workspace,
               size_t workspace_bytes, size_t* h_compressed_bytes, cudaStream_t stream) {
    if (!plan) return DFX_ERR_ARG;
    if (!d_out || !d_workspace || (!d_bf16 && plan->n)) return DFX_ERR_ARG;
    if (!aligned16(d_bf16) || !aligned16(d_out) || !aligned16(d_workspace)) return DFX_ERR_ARG;
    if (out_capacity < plan->max_bytes || workspace_bytes < plan->ws_bytes) return DFX_ERR_CAPACITY;
    // all 256 exponent values must fit a tANS table
    if (dfx::is_tans(plan->coder) && plan->table_log < 8) return DFX_ERR_UNSUPPORTED;
    int rc = check_device(plan);
    if (rc) return rc;
    dfx::EncodeArgs a;
    a.in = (const uint16_t*)d_bf16;
    a.out = (uint8_t*)d_out;
    a.n = plan->n;
    a.K = plan->K;
    a.G = plan->G;
    a.max_len = plan->max_len;
    a.coder = plan->coder;
    a.table_log = plan->table_log;
    a.n_chunk = (uint32_t)plan->L.n_chunk;
    a.n_group = (uint32_t)plan->L.n_group;
    a.off_gbase = plan->L.off_gbase;
    a.off_clen = plan->L.off_clen;
    a.off_m = plan->L.off_m;
    a.off_stream = plan->L.off_stream;
    uint8_t* ws = (uint8_t*)d_workspace;
    a.ws_counts = (unsigned long long*)(ws + dfx::kWsCounts);
    a.ws_code = (uint32_t*)(ws + dfx::kWsCode);
    a.ws_len = ws + dfx::kWsLen;
    a.ws_group_bits = (uint32_t*)(ws + dfx::kWsGroupBits);
    a.ws_edge = (unsigned long long*)(ws + dfx::ws_edge_offset(plan->L.n_group));
    a.ws_tans = (uint32_t*)(ws + dfx::ws_tans_offset(plan->L.n_group));
    a.status = plan->d_status;
    a.max_bytes = plan->max_bytes;
    if (dfx::launch_encode(a, plan->max_bytes, stream) != cudaSuccess) {
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

int dfx_decode(dfx_plan_t plan, const void* d_comp, size_t comp_bytes, void* d_bf16, cudaStream_t stream) {
    dfx::DecodeArgs a;
    const int rc = make_decode_args(plan, d_comp, comp_bytes, d_bf16, &a);
    if (rc) return rc;
    if (dfx::launch_decode(a, plan->coder, plan->decode_grid, stream) != cudaSuccess) {
        cudaGetLastError();
        return DFX_ERR_CUDA;
    }
    return DFX_OK;
}

int dfx_decode_range(dfx_plan_t plan, const void* d_comp, size_t comp_bytes, uint64_t first_group,
                     uint64_t group_count, void* d_bf16, cudaStream_t stream) {
    if (!plan) return DFX_ERR_ARG;
    if (first_group > plan->L.n_group || group_count > plan->L.n_group - first_group) return DFX_ERR_ARG;
    if (group_count == 0) return DFX_OK;
    dfx::DecodeArgs a;
    const int rc = make_decode_args(plan, d_comp, comp_bytes, d_bf16, &a);
    if (rc) return rc;
    a.g_begin = (uint32_t)first_group;
    a.g_end = (uint32_t)(first_group + group_count);
    a.out_first = first_group * (uint64_t)plan->G * plan->K;
    const uint64_t need = (group_count + 31) / 32;  // a warp per group
    const int grid = (int)(need < (uint64_t)plan->resident_ctas ? need : (uint64_t)plan->resident_ctas);
    if (dfx::launch_decode(a, plan->coder, grid, stream) != cudaSuccess) {
        cudaGetLastError();
        return DFX_ERR_CUDA;
    }
    return DFX_OK;
}

int dfx_decode_host(dfx_plan_t plan, const void* h_comp, size_t comp_bytes, void* d_staging, size_t staging_bytes,
                    void* d_bf16, uint32_t slices, cudaStream_t copy_stream, cudaStream_t decode_stream) {
    if (!plan || !h_comp || !d_staging) return DFX_ERR_ARG;
    if (!aligned16(d_staging)) return DFX_ERR_ARG;
    const dfx::Layout& L = plan->L;
    if (comp_bytes < L.off_stream + dfx::stream_bytes(0)) return DFX_ERR_CORRUPT;
    uint64_t total = 0;  // the container's size from its header
    memcpy(&total, (const uint8_t*)h_comp + 24, 8);
    if (total > comp_bytes || total < L.off_stream + dfx::stream_bytes(0)) return DFX_ERR_CORRUPT;
    if (staging_bytes < total) return DFX_ERR_CAPACITY;
    dfx::DecodeArgs probe;
    int rc = make_decode_args(plan, d_staging, total, d_bf16, &probe);
    if (rc) return rc;
    if (!plan->events_made) {
        if (cudaEventCreateWithFlags(&plan->decode_idle, cudaEventDisableTiming) != cudaSuccess) {
            cudaGetLastError();
            return DFX_ERR_CUDA;
        }
        for (uint32_t i = 0; i < dfx_plan_s::kHostSlicesMax; i++)
            if (cudaEventCreateWithFlags(&plan->slice_done[i], cudaEventDisableTiming) != cudaSuccess) {
                cudaGetLastError();
                for (uint32_t j = 0; j < i; j++) cudaEventDestroy(plan->slice_done[j]);
                cudaEventDestroy(plan->decode_idle);
                return DFX_ERR_CUDA;
            }
        plan->events_made = true;
    }
    const uint64_t ng = L.n_group;
    uint64_t ns = slices ? slices : 8;
    if (ns > dfx_plan_s::kHostSlicesMax) ns = dfx_plan_s::kHostSlicesMax;
    if (ns > ng) ns = ng ? ng : 1;
    const uint8_t* h = (const uint8_t*)h_comp;
    uint8_t* d = (uint8_t*)d_staging;
    const uint64_t ge = (uint64_t)L.G * L.K;
    const uint64_t* gbase = (const uint64_t*)(h + L.off_gbase);
    auto fail = [] {
        cudaGetLastError();
        return DFX_ERR_CUDA;
    };
    // the staging buffer is overwritten only once the decoding queued before this call
    // (which may read it) has finished
    if (cudaEventRecord(plan->decode_idle, decode_stream) != cudaSuccess ||
        cudaStreamWaitEvent(copy_stream, plan->decode_idle, 0) != cudaSuccess)
        return fail();
    // header, code section and the group index: every slice's decode reads them
    if (cudaMemcpyAsync(d, h, L.off_m, cudaMemcpyHostToDevice, copy_stream) != cudaSuccess) return fail();
    for (uint64_t s = 0; s < ns; s++) {
        const uint64_t g0 = ng * s / ns, g1 = ng * (s + 1) / ns;
        // the slice's sign+mantissa bytes
        const uint64_t m0 = L.off_m + g0 * ge, m1 = L.off_m + (g1 * ge < L.n ? g1 * ge : L.n);
        if (m1 > m0 && cudaMemcpyAsync(d + m0, h + m0, m1 - m0, cudaMemcpyHostToDevice, copy_stream) != cudaSuccess)
            return fail();
        // its stream words, from the word of its first bit to a few words past its last
        // (what the decoder stages), clamped to the container
        uint64_t b0 = gbase[g0], b1 = gbase[g1];
        if (b1 < b0 || b1 > total * 8) b0 = 0, b1 = (total - L.off_stream) * 8;  // a bad index: copy everything
        uint64_t s0 = L.off_stream + ((b0 >> 5) * 4 & ~uint64_t(15));
        uint64_t s1 = L.off_stream + dfx::align16(((b1 >> 5) + 8) * 4);
        if (s1 > total) s1 = total;
        if (s1 > s0 && cudaMemcpyAsync(d + s0, h + s0, s1 - s0, cudaMemcpyHostToDevice, copy_stream) != cudaSuccess)
            return fail();
        if (cudaEventRecord(plan->slice_done[s], copy_stream) != cudaSuccess ||
            cudaStreamWaitEvent(decode_stream, plan->slice_done[s], 0) != cudaSuccess)
            return fail();
        rc = dfx_decode_range(plan, d_staging, total, g0, g1 - g0, (uint16_t*)d_bf16 + g0 * ge, decode_stream);
        if (rc) return rc;
    }
    return DFX_OK;
}

int dfx_decode_gemm(dfx_plan_t plan, const void* d_comp, size_t comp_bytes, uint64_t rows, uint64_t cols,
                    const void* d_x, uint32_t tokens, float* d_y, void* d_w_out, cudaStream_t stream) {
    if (!plan) return DFX_ERR_ARG;
    if (plan->coder != DFX_CODER_HUFFMAN) return DFX_ERR_UNSUPPORTED;
    if (rows == 0 || cols == 0 || rows * cols != plan->n || rows >= (1ull << 31) || cols >= (1ull << 31))
        return DFX_ERR_ARG;
    if (tokens == 0 || tokens > dfx::kGemmMaxTokens) return DFX_ERR_ARG;
    if (cols % (32ull * plan->K) != 0) return DFX_ERR_UNSUPPORTED;  // every group inside one row
    if (!d_x || !d_y || !aligned16(d_x) || !aligned16(d_y) || !aligned16(d_w_out)) return DFX_ERR_ARG;
    dfx::DecodeArgs a;
    const int rc = make_decode_args(plan, d_comp, comp_bytes, d_w_out ? d_w_out : d_y, &a);
    if (rc) return rc;
    // one CTA per SM, each a tile of at most kGemmMaxRows rows; more CTAs (several waves)
    // only when the rows need them
    uint64_t grid = rows < (uint64_t)plan->sms ? rows : (uint64_t)plan->sms;
    const uint64_t need = (rows + dfx::kGemmMaxRows - 1) / dfx::kGemmMaxRows;
    if (need > grid) grid = need;
    if (dfx::launch_decode_gemm(a, (const uint16_t*)d_x, d_y, (uint16_t*)d_w_out, (uint32_t)rows, (uint32_t)cols, tokens,
                                (int)grid, stream) != cudaSuccess) {
        cudaGetLastError();
        return DFX_ERR_CUDA;
    }
    return DFX_OK;
}

int dfx_decode_batch(const dfx_plan_t* plans, const void* const* d_comps, const size_t* comp_bytes,
                     void* const* d_bf16s, uint32_t count, cudaStream_t stream) {
    if (count == 0) return DFX_OK;
    if (!plans || !d_comps || !comp_bytes || !d_bf16s || count > dfx::kMaxBatch) return DFX_ERR_ARG;
    static_assert(sizeof(dfx::BatchArgs) <= 4000, "the batch descriptor is passed as a kernel parameter");
    dfx::BatchArgs b;
    b.count = count;
    uint64_t groups[dfx::kMaxBatch];
    for (uint32_t i = 0; i < count; i++) {
        if (!plans[i]) return DFX_ERR_ARG;
        if (plans[i]->K != plans[0]->K || plans[i]->coder != plans[0]->coder || plans[i]->device != plans[0]->device)
            return DFX_ERR_UNSUPPORTED;
        const int rc = make_decode_args(plans[i], d_comps[i], comp_bytes[i], d_bf16s[i], &b.t[i]);
        if (rc) return rc;
        groups[i] = plans[i]->L.n_group;
    }
    // CTAs in proportion to the groups: every tensor gets one (an empty one only checks its
    // header), then each further CTA goes to the tensor with the most groups per CTA.
    const uint32_t total = (uint32_t)plans[0]->resident_ctas;
    if (total < count) return DFX_ERR_UNSUPPORTED;
    uint32_t ctas[dfx::kMaxBatch];
    for (uint32_t i = 0; i < count; i++) ctas[i] = 1;
    for (uint32_t left = total - count; left > 0; left--) {
        int best = -1;
        for (uint32_t i = 0; i < count; i++) {
            if (ctas[i] >= (groups[i] + 31) / 32) continue;  // every warp already has a group
            if (best < 0 || groups[i] * ctas[best] > groups[best] * ctas[i]) best = (int)i;
        }
        if (best < 0) break;
        ctas[best]++;
    }
    b.cta_begin[0] = 0;
    for (uint32_t i = 0; i < count; i++) b.cta_begin[i + 1] = b.cta_begin[i] + ctas[i];
    if (dfx::launch_decode_batch(b, plans[0]->K, plans[0]->coder, stream) != cudaSuccess) {
        cudaGetLastError();
        return DFX_ERR_CUDA;
    }
    return DFX_OK;
}

int dfx_device_status(dfx_plan_t plan, cudaStream_t stream, uint32_t* h_status) {
    if (!plan || !h_status) return DFX_ERR_ARG;
    uint32_t v = 0;
    if (cudaMemcpyAsync(&v, plan->d_status, 4, cudaMemcpyDeviceToHost, stream) != cudaSuccess ||
        cudaMemsetAsync(plan->d_status, 0, 4, stream) != cudaSuccess || cudaStreamSynchronize(stream) != cudaSuccess) {
        cudaGetLastError();
        return DFX_ERR_CUDA;
    }
    *h_status = v;
    return DFX_OK;
}

int dfx_free(dfx_plan_t plan) {
    if (!plan) return DFX_OK;
    int rc = DFX_OK;
    if (plan->d_status && cudaFree(plan->d_status) != cudaSuccess) {
        cudaGetLastError();
        rc = DFX_ERR_CUDA;
    }
    if (plan->events_made) {
        for (uint32_t i = 0; i < dfx_plan_s::kHostSlicesMax; i++) cudaEventDestroy(plan->slice_done[i]);
        cudaEventDestroy(plan->decode_idle);
    }
    free(plan);
    return rc;
}

}  // extern "C"

namespace {

int make_decode_args(const dfx_plan_s* plan, const void* d_comp, size_t comp_bytes, void* d_bf16, dfx::DecodeArgs* a) {
    if (!plan) return DFX_ERR_ARG;
    if (!d_comp || (!d_bf16 && plan->n)) return DFX_ERR_ARG;
    if (!aligned16(d_comp) || !aligned16(d_bf16)) return DFX_ERR_ARG;
    if (comp_bytes < plan->L.off_stream + dfx::stream_bytes(0)) return DFX_ERR_CORRUPT;
    const int rc = check_device(plan);
    if (rc) return rc;
    a->comp = (const uint8_t*)d_comp;
    a->comp_bytes = comp_bytes;
    a->out = (uint16_t*)d_bf16;
    a->n = plan->n;
    a->K = plan->K;
    a->G = plan->G;
    a->n_chunk = (uint32_t)plan->L.n_chunk;
    a->n_group = (uint32_t)plan->L.n_group;
    a->off_clen = plan->L.off_clen;
    a->off_m = plan->L.off_m;
    a->off_stream = plan->L.off_stream;
    a->status = plan->d_status;
    a->g_begin = 0;
    a->g_end = (uint32_t)plan->L.n_group;
    a->out_first = 0;
    a->inject = g_inject;
    a->early = (plan->decode_flags & DFX_DECODE_EARLY_READ) ? 1u : 0u;
    return DFX_OK;
}

}  // namespace
