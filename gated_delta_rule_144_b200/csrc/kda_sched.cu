// Scheduling of packed documents for the chunked prefill.
//
// A chunked CTA walks one (document, head) chain from its first chunk to its last, so the
// launch's makespan is at least the longest document's chain. CTAs start in grid order; when the
// long documents come last they start last and set the makespan. This kernel ranks the documents
// by length (longest first, ties by index) so that the chunked kernel can hand the longest
// chains to the first CTAs: the classic longest-processing-time-first rule.

#include "kda_internal.cuh"

namespace kda {
namespace {

constexpr int kThreads = 1024;

__global__ void __launch_bounds__(kThreads)
doc_order_kernel(const int32_t* __restrict__ cu_seqlens, int N, int32_t* __restrict__ order) {
    extern __shared__ int32_t len_s[];
    for (int i = threadIdx.x; i < N; i += kThreads) len_s[i] = cu_seqlens[i + 1] - cu_seqlens[i];
    __syncthreads();
    // rank of d = number of documents that go before it; ranks form a permutation because
    // (length descending, index ascending) is a strict total order
    for (int d = threadIdx.x; d < N; d += kThreads) {
        const int ld = len_s[d];
        int rank = 0;
        for (int e = 0; e < N; ++e) {
            const int le = len_s[e];
            rank += (le > ld) | ((le == ld) & (e < d));
        }
        order[rank] = d;
    }
}

}  // namespace

cudaError_t launch_doc_order(const int32_t* cu_seqlens, int N, int32_t* order,
                             cudaStream_t stream) {
    if (N <= 0 || N > kMaxOrderedDocs) return cudaErrorInvalidValue;
    doc_order_kernel<<<1, kThreads, N * sizeof(int32_t), stream>>>(cu_seqlens, N, order);
    return cudaGetLastError();
}

}  // namespace kda
