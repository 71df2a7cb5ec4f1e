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

// map[g] = d for the chunk records g of document d: g runs over [lo_d, lo_{d+1}) with
// lo_d = floor(t0_d / 64) + d; the records past the document's last chunk (at most one) get -1.
// Every write stays inside [0, G) whatever cu_seqlens holds; a malformed cu_seqlens is reported.
__global__ void chunk_map_kernel(const int32_t* __restrict__ cu, int N, int T, long long G,
                                 int32_t* __restrict__ map, unsigned* err) {
    for (int d = blockIdx.x * blockDim.x + threadIdx.x; d < N; d += gridDim.x * blockDim.x) {
        const long long a = cu[d], b = cu[d + 1];
        const bool bad = b < a || a < 0 || b > T || (d == 0 && a != 0) || (d == N - 1 && b != T);
        if (bad) {
            set_device_error(err, DEV_BAD_SEQLENS);
            continue;
        }
        const long long lo = a / 64 + d;
        const long long hi = b > a ? (b - 1) / 64 + d : lo - 1;   // last record with a chunk
        long long lo_next = G;
        if (d + 1 < N) {
            const long long a2 = cu[d + 1];
            lo_next = (a2 >= 0 && a2 <= T) ? a2 / 64 + d + 1 : G;
        }
        for (long long g = lo < 0 ? 0 : lo; g < lo_next && g < G; ++g)
            map[g] = g <= hi ? d : -1;
    }
}

}  // namespace

cudaError_t launch_chunk_map(const int32_t* cu_seqlens, int N, int T, long long G, int32_t* map,
                             unsigned* err, cudaStream_t stream) {
    if (N <= 0 || G <= 0) return cudaSuccess;
    const int threads = 256;
    const int blocks = (N + threads - 1) / threads;
    chunk_map_kernel<<<blocks, threads, 0, stream>>>(cu_seqlens, N, T, G, map, err);
    return cudaGetLastError();
}

cudaError_t launch_doc_order(const int32_t* cu_seqlens, int N, int32_t* order,
                             cudaStream_t stream) {
    if (N <= 0 || N > kMaxOrderedDocs) return cudaErrorInvalidValue;
    doc_order_kernel<<<1, kThreads, N * sizeof(int32_t), stream>>>(cu_seqlens, N, order);
    return cudaGetLastError();
}

}  // namespace kda
