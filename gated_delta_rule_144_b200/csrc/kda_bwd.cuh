// Private declarations of the gradient kernel (kda_bwd), shared by kda_bwd.cu and kda_api.cu.
#pragma once

#include <cstddef>
#include <cstdint>

#include "kda_internal.cuh"

namespace kda {

// Gradients of the recurrence (kda_bwd): dk = dv = 128, outputs fp32.
struct BwdParams {
    const void* q;
    const void* k;
    const void* v;
    const void* beta;
    const void* dout;
    const float* log_g;
    const float* h0;            // nullable
    const float* dhT;           // nullable
    const int32_t* cu_seqlens;  // nullable (device)
    float* dq;
    float* dk;
    float* dv;
    float* dlog_g;
    float* dbeta;
    float* dh0;                 // nullable
    void* workspace;            // bwd_workspace_bytes(N * H, T)
    int T, H, N;
    bool bf16;
    unsigned* err;
};

// Checkpoints of every chain (one 128 x 128 fp32 state per 64 tokens, plus one) and one chunk's
// states and read-outs per chain.
size_t bwd_workspace_bytes(long long chains, int T);
cudaError_t launch_bwd(const BwdParams& p, cudaStream_t stream);

}  // namespace kda
