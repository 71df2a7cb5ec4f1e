// kda_fwd_no_alloc: the prefill for callers that cannot allocate device memory.
//
// kda_fwd takes its scratch (the longest-first order of packed documents, one int32 per
// document) from a caller-provided workspace. This entry point takes it from a static device
// array instead. It does nothing else: it validates the one extra limit, finds the array's device
// address and hands it to kda_fwd as the workspace. It allocates nothing.

#include <cuda_runtime.h>

#include <mutex>

#include "kda.h"
#include "kda_internal.cuh"

static_assert(KDA_NO_ALLOC_MAX_DOCS == kda::kMaxOrderedDocs,
              "the static scratch holds every document the chunked path orders");

namespace {

// The scratch: one slot per packed document, shared by every call on a device. Each call's
// scheduling kernel writes slots [0, N) before the chunked kernel reads them, so the array
// never needs clearing. Overlapping calls on one device race on it.
static __device__ __align__(256) int32_t g_no_alloc_order[KDA_NO_ALLOC_MAX_DOCS];

constexpr int kMaxDevices = 64;
int32_t* g_scratch[kMaxDevices] = {};
std::mutex g_mu;

// Device address of the scratch on the current device: looked up once per device, with that
// device current (in host code the array's name is only a host-side stand-in).
kda_status_t scratch_for_current_device(int32_t** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) {
        kda::set_last_error("kda_fwd_no_alloc: cudaGetDevice failed");
        return KDA_ERR_CUDA;
    }
    if (dev < 0 || dev >= kMaxDevices) {
        kda::set_last_error("kda_fwd_no_alloc: device index out of range");
        return KDA_ERR_UNSUPPORTED;
    }
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_no_alloc_order);
        if (e != cudaSuccess || !p) {
            kda::set_last_error("kda_fwd_no_alloc: cudaGetSymbolAddress of the scratch failed");
            return KDA_ERR_CUDA;
        }
        g_scratch[dev] = static_cast<int32_t*>(p);
    }
    *out = g_scratch[dev];
    return KDA_OK;
}

}  // namespace

extern "C" kda_status_t kda_fwd_no_alloc(const kda_fwd_desc_t* desc, const void* q,
                                         const void* k, const void* v, const float* log_g,
                                         const void* beta, const float* h0,
                                         const int32_t* cu_seqlens, void* o, float* hT,
                                         kda_stream_t stream) {
    if (desc && cu_seqlens && desc->num_seqs > KDA_NO_ALLOC_MAX_DOCS) {
        kda::set_last_error(
            "kda_fwd_no_alloc: more packed documents than the static scratch holds "
            "(KDA_NO_ALLOC_MAX_DOCS = 2048); use kda_fwd with a workspace");
        return KDA_ERR_INVALID_ARG;
    }
    int32_t* scratch = nullptr;
    const kda_status_t st = scratch_for_current_device(&scratch);
    if (st != KDA_OK) return st;
    return kda_fwd(desc, q, k, v, log_g, beta, h0, cu_seqlens, o, hT, scratch,
                   sizeof(int32_t) * KDA_NO_ALLOC_MAX_DOCS, stream);
}
