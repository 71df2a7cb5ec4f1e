// Private declarations shared by the translation units of libkda.so.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

namespace kda {

// Codes the kernels store into the sticky device error word (same values as kda_status_t).
enum DeviceError : unsigned {
    DEV_OK = 0,
    DEV_TIMEOUT = 4,
    DEV_BAD_SEQLENS = 5,
    DEV_RANGE = 6,   // reserved: steep decays take the chunked kernels' direct path instead
};

// The first error sticks; later ones are dropped.
__device__ __forceinline__ void set_device_error(unsigned* err, unsigned code) {
    atomicCAS(err, 0u, code);
}

// Workspace of the split chunked prefill: the WY factors of every (chunk record, head), written
// by the intra-chunk kernel and read by the state pass. Record index = g * H + head, where g is
// sequence * ncT + chunk (ncT = ceil(T / 64)), or, for packed documents, floor(t0 / 64) +
// document + chunk (strictly increasing over (document, chunk), so records never collide and
// g < ncT + N).
struct SplitWorkspace {
    __nv_bfloat16* wq;   // [R * 128][128]: rows 0-63 W, 64-127 Q+
    __nv_bfloat16* ke;   // [R * 64][128]: K_end
    __nv_bfloat16* ut;   // [R * 128][64]: U~^T (value column, token)
    __nv_bfloat16* aq;   // [R * 64][64]: A_qk (row r, column i; zero above the diagonal)
    float* decay;        // [R][128]: e^{Gamma_end}
    int32_t* map;        // [G]: document of chunk record g, -1 if unused (packed only)
    float* state;        // [N][H][128][128]: state between segments (equal-length sequences only)
    unsigned long long* counters;   // [kMaxSegments]: record counters of the intra-chunk launches
    long long G;         // chunk records per head; R = G * H
    int ncT;
};

// The split path may run in up to this many chunk segments (equal-length sequences): the state
// pass of segment s overlaps the intra-chunk kernel of segment s + 1.
constexpr int kMaxSegments = 16;

// One launch of the state pass: chunks [c_begin, c_end) of every chain, from the state h0 to the
// state hT (the caller's, or the workspace's scratch state between segments; either nullable).
struct ScanSegment {
    int c_begin, c_end;
    const float* h0;
    float* hT;
};

struct FwdParams {
    const void* q;
    const void* k;
    const void* v;
    const float* log_g;
    const void* beta;
    const float* h0;          // nullable
    const int32_t* cu_seqlens;  // nullable (device)
    void* o;
    float* hT;                // nullable
    int B, T, H, dk, dv, N;
    bool bf16;
    unsigned* err;            // device error word
    const int32_t* doc_order;   // nullable: packed documents in the order CTAs should take them
    const SplitWorkspace* split;  // nullable: run the fused kernel instead
};

struct DecodeParams {
    const void* q;
    const void* k;
    const void* v;
    const float* log_g;
    const void* beta;
    float* S;
    void* o;
    int N, H, dk, dv;
    bool bf16;
    unsigned* err;
};

// Largest number of packed documents the chunked path schedules longest first (above it, CTAs
// take documents in their packed order).
constexpr int kMaxOrderedDocs = 2048;

// Record the text kda_last_error() returns on this host thread.
void set_last_error(const char* msg);

// Launchers (host). Each returns the launch status of its kernel(s).
// Writes order[0..N) = document indices by decreasing length (ties: lower index first).
cudaError_t launch_doc_order(const int32_t* cu_seqlens, int N, int32_t* order,
                             cudaStream_t stream);
cudaError_t launch_recurrent(const FwdParams& p, cudaStream_t stream);
cudaError_t launch_decode_d128(const DecodeParams& p, cudaStream_t stream);
// T tokens per sequence ([N, T, H, d] inputs), state read once and written once (d = 128).
cudaError_t launch_decode_tokens_d128(const DecodeParams& p, int T, cudaStream_t stream);
cudaError_t launch_chunk64(const FwdParams& p, cudaStream_t stream);
// Split chunked prefill: map[g] for packed documents (sets DEV_BAD_SEQLENS on a malformed
// cu_seqlens), the intra-chunk kernel over all records, then the state pass over all chains.
cudaError_t launch_chunk_map(const int32_t* cu_seqlens, int N, int T, long long G, int32_t* map,
                             unsigned* err, cudaStream_t stream);
// Intra-chunk kernel over the records of chunks [c_begin, c_begin + c_span) of every sequence (all
// records for packed documents, which are not segmented); CTAs claim records from *counter,
// which must be zero at launch.
cudaError_t launch_chunk64_intra(const FwdParams& p, int c_begin, int c_span,
                                 unsigned long long* counter, cudaStream_t stream);
// Gated RMSNorm applied by the state pass to its output (y = o / sqrt(mean(o^2) + eps) * weight *
// sigmoid(gate) per (token, head)), instead of a separate pass over o.
struct ScanNorm {
    const void* gate;      // shaped and typed like o
    const float* weight;   // [128]
    float eps;
};
cudaError_t launch_chunk_scan(const FwdParams& p, const ScanSegment& seg, cudaStream_t stream,
                              const ScanNorm* norm = nullptr);
// y = x / sqrt(mean(x^2) + eps) * w * sigmoid(gate) per vector of dv elements (dv <= 256);
// y may alias x.
cudaError_t launch_out_norm_gated(const void* x, const void* gate, const float* w, float eps,
                                  void* y, long long vectors, int dv, bool bf16,
                                  cudaStream_t stream);
// Short causal convolution with document resets, optional SiLU (act = 1) and L2 norm per group
// of `group` channels (0: none); x, y [B, T, C]; w [C][W], 1 <= W <= 8.
cudaError_t launch_short_conv(const void* x, const float* w, const int32_t* cu, int N, void* y,
                              int B, int T, int C, int W, bool bf16, int act, int group, float eps,
                              unsigned* err, cudaStream_t stream);
bool chunk64_available();
// Value columns one chunked-kernel CTA owns for N sequences x H heads (64 or 128).
int chunk64_value_width(int N, int H);

// One-time set-up per device (kernel attributes, occupancy queries): `fn(device)` runs once for
// each device index, with that device current, and its status is kept for later calls. Kernel
// attributes such as the dynamic shared-memory limit belong to a device's context, so a process
// that launches on several devices needs them set on each.
class PerDevice {
  public:
    static constexpr int kMax = 64;
    template <class F>
    cudaError_t run(F&& fn, int* dev_out = nullptr) {
        int dev = 0;
        cudaError_t e = cudaGetDevice(&dev);
        if (e != cudaSuccess) return e;
        if (dev < 0 || dev >= kMax) return cudaErrorInvalidDevice;
        if (dev_out) *dev_out = dev;
        std::lock_guard<std::mutex> lock(mu_);
        if (!done_[dev]) {
            err_[dev] = fn(dev);
            done_[dev] = true;
        }
        return err_[dev];
    }

  private:
    std::mutex mu_;
    bool done_[kMax] = {};
    cudaError_t err_[kMax] = {};
};

// Element loads shared by the CUDA-core kernels.
__device__ __forceinline__ float load_elem(const float* p, int64_t i) { return p[i]; }
__device__ __forceinline__ float load_elem(const __nv_bfloat16* p, int64_t i) {
    return __bfloat162float(p[i]);
}
__device__ __forceinline__ void store_elem(float* p, int64_t i, float x) { p[i] = x; }
__device__ __forceinline__ void store_elem(__nv_bfloat16* p, int64_t i, float x) {
    p[i] = __float2bfloat16_rn(x);
}

}  // namespace kda
