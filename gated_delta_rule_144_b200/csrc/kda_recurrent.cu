// Per-token walk: the exact fp32 evaluation of the KDA recurrence on CUDA cores.
//
// This is the path for fp32 inputs, for head sizes other than 128, and the general decode path.
// It follows the recurrence token by token (GLM-5.3-Flash model card, Kimi Delta Attention
// snippet), which the metrale glm5next_layer page calls the "per-token walk" of prefill.
//
// Work split. The dv columns of S evolve independently (column j of S only meets column j of v),
// so one warp owns NC = 4 value columns of one (sequence, head) for the whole sequence, with the
// dk rows spread over the 32 lanes (lane l holds rows l, l + 32, ...). Per token, the warp
//   1. decays its rows by g = exp(log_g),
//   2. reduces k^T S, q^T S (for its 4 columns) and q.k over the rows with one butterfly,
//   3. forms delta = beta (v - k^T S) and o = q^T S + (q.k) delta (= q^T of the written state),
//   4. writes S += k delta^T.
// Everything is fp32. Inputs of token t + 1 are fetched while token t is computed.
// h0 and hT may alias (decode updates a state in place): each warp reads its own block of the
// state before the walk and writes the same block after it, and no other warp touches it.

#include "kda_internal.cuh"

namespace kda {
namespace {

constexpr int kNC = 4;           // value columns per warp
constexpr int kWarpsPerBlock = 4;

template <typename Tin, int RPL>
__global__ void __launch_bounds__(kWarpsPerBlock * 32)
recurrent_kernel(const Tin* __restrict__ q, const Tin* __restrict__ k, const Tin* __restrict__ v,
                 const float* __restrict__ log_g, const Tin* __restrict__ beta,
                 const float* h0, const int32_t* __restrict__ cu_seqlens,
                 Tin* __restrict__ o, float* hT, int T, int H, int dk, int dv,
                 int N, int col_groups, unsigned* err) {
    const int lane = threadIdx.x & 31;
    const int64_t warp = (int64_t)blockIdx.x * kWarpsPerBlock + (threadIdx.x >> 5);
    const int64_t units = (int64_t)N * H;
    if (warp >= units * col_groups) return;
    const int unit = (int)(warp / col_groups);
    const int cg = (int)(warp % col_groups);
    const int n = unit / H, h = unit % H;

    int64_t t0, t1;
    if (cu_seqlens) {
        t0 = cu_seqlens[n];
        t1 = cu_seqlens[n + 1];
        const bool bad_ends = (n == 0 && t0 != 0) || (n == N - 1 && t1 != T);
        if (t1 < t0 || t0 < 0 || t1 > T || bad_ends) {
            if (lane == 0) set_device_error(err, DEV_BAD_SEQLENS);
            return;
        }
    } else {
        t0 = (int64_t)n * T;
        t1 = t0 + T;
    }

    const int j0 = cg * kNC;
    float S[RPL][kNC];
    const size_t state_off = ((size_t)n * H + h) * (size_t)dk * dv;
#pragma unroll
    for (int r = 0; r < RPL; ++r) {
        const int c = lane + 32 * r;
#pragma unroll
        for (int i = 0; i < kNC; ++i) {
            const int j = j0 + i;
            S[r][i] = (h0 && c < dk && j < dv) ? h0[state_off + (size_t)c * dv + j] : 0.f;
        }
    }

    // register double buffer for the per-token inputs
    float kr[RPL], qr[RPL], lg[RPL], vr[kNC], b = 0.f;
    auto fetch = [&](int64_t t, float* kk, float* qq, float* ll, float* vv, float& bb) {
        const int64_t qk = (t * H + h) * (int64_t)dk;
        const int64_t vo = (t * H + h) * (int64_t)dv;
#pragma unroll
        for (int r = 0; r < RPL; ++r) {
            const int c = lane + 32 * r;
            const bool ok = c < dk;
            kk[r] = ok ? load_elem(k, qk + c) : 0.f;
            qq[r] = ok ? load_elem(q, qk + c) : 0.f;
            ll[r] = ok ? log_g[qk + c] : 0.f;
        }
#pragma unroll
        for (int i = 0; i < kNC; ++i) vv[i] = (j0 + i < dv) ? load_elem(v, vo + j0 + i) : 0.f;
        bb = load_elem(beta, t * H + h);
    };
    if (t0 < t1) fetch(t0, kr, qr, lg, vr, b);

    for (int64_t t = t0; t < t1; ++t) {
        float kn[RPL], qn[RPL], ln[RPL], vn[kNC], bn = 0.f;
        if (t + 1 < t1) fetch(t + 1, kn, qn, ln, vn, bn);

        float red[2 * kNC + 1];
#pragma unroll
        for (int i = 0; i < 2 * kNC + 1; ++i) red[i] = 0.f;
#pragma unroll
        for (int r = 0; r < RPL; ++r) {
            const float g = expf(lg[r]);
#pragma unroll
            for (int i = 0; i < kNC; ++i) {
                S[r][i] *= g;
                red[i] = fmaf(kr[r], S[r][i], red[i]);
                red[kNC + i] = fmaf(qr[r], S[r][i], red[kNC + i]);
            }
            red[2 * kNC] = fmaf(qr[r], kr[r], red[2 * kNC]);
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1)
#pragma unroll
            for (int i = 0; i < 2 * kNC + 1; ++i)
                red[i] += __shfl_xor_sync(0xffffffffu, red[i], off);

        float delta[kNC];
#pragma unroll
        for (int i = 0; i < kNC; ++i) delta[i] = b * (vr[i] - red[i]);
        if (lane < kNC && j0 + lane < dv) {
            float oi = 0.f;
#pragma unroll
            for (int i = 0; i < kNC; ++i)
                if (i == lane) oi = fmaf(red[2 * kNC], delta[i], red[kNC + i]);
            store_elem(o, (t * H + h) * (int64_t)dv + j0 + lane, oi);
        }
#pragma unroll
        for (int r = 0; r < RPL; ++r)
#pragma unroll
            for (int i = 0; i < kNC; ++i) S[r][i] = fmaf(kr[r], delta[i], S[r][i]);

#pragma unroll
        for (int r = 0; r < RPL; ++r) {
            kr[r] = kn[r];
            qr[r] = qn[r];
            lg[r] = ln[r];
        }
#pragma unroll
        for (int i = 0; i < kNC; ++i) vr[i] = vn[i];
        b = bn;
    }

    if (hT) {
#pragma unroll
        for (int r = 0; r < RPL; ++r) {
            const int c = lane + 32 * r;
            if (c >= dk) continue;
#pragma unroll
            for (int i = 0; i < kNC; ++i)
                if (j0 + i < dv) hT[state_off + (size_t)c * dv + j0 + i] = S[r][i];
        }
    }
}

template <typename Tin, int RPL>
cudaError_t launch_typed(const FwdParams& p, cudaStream_t stream) {
    const int col_groups = (p.dv + kNC - 1) / kNC;
    const int64_t warps = (int64_t)p.N * p.H * col_groups;
    const int64_t blocks = (warps + kWarpsPerBlock - 1) / kWarpsPerBlock;
    if (blocks > 0x7fffffff) return cudaErrorInvalidConfiguration;
    recurrent_kernel<Tin, RPL><<<(unsigned)blocks, kWarpsPerBlock * 32, 0, stream>>>(
        static_cast<const Tin*>(p.q), static_cast<const Tin*>(p.k),
        static_cast<const Tin*>(p.v), p.log_g, static_cast<const Tin*>(p.beta), p.h0,
        p.cu_seqlens, static_cast<Tin*>(p.o), p.hT, p.T, p.H, p.dk, p.dv, p.N, col_groups,
        p.err);
    return cudaGetLastError();
}

template <typename Tin>
cudaError_t launch_rpl(const FwdParams& p, cudaStream_t stream) {
    if (p.dk <= 32) return launch_typed<Tin, 1>(p, stream);
    if (p.dk <= 64) return launch_typed<Tin, 2>(p, stream);
    if (p.dk <= 128) return launch_typed<Tin, 4>(p, stream);
    return launch_typed<Tin, 8>(p, stream);
}

}  // namespace

cudaError_t launch_recurrent(const FwdParams& p, cudaStream_t stream) {
    if ((int64_t)p.N * p.H == 0) return cudaSuccess;
    return p.bf16 ? launch_rpl<__nv_bfloat16>(p, stream) : launch_rpl<float>(p, stream);
}

}  // namespace kda
