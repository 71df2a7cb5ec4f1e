// Short causal convolution of the KDA inputs (the prologue of the recurrence), with packed-document
// resets, an optional SiLU and an optional per-group L2 normalisation, in one bandwidth-bound pass.
//
// NeMo glm5_next layers, _TorchShortConvolution: a depthwise causal Conv1d over
// [batch, sequence, channels] that resets at packed boundaries (q_conv1d, k_conv1d and v_conv1d of
// Glm5NextLinearAttention, linear_conv_kernel_dim taps). Per channel c and token t of a document
// that starts at s:
//   y[t, c] = sum_{j < W} w[c, j] x[t - (W - 1) + j, c]   (positions before s contribute zero),
// then optionally y <- y sigmoid(y) (SiLU) and y <- y / sqrt(sum over its group of y^2 + eps) for
// each group of g consecutive channels (g = head_dim normalises each head vector, as the
// recurrence's q and k arrive).
//
// Work split: a warp owns 128 consecutive channels (4 per lane: 8-byte bf16 / 16-byte fp32
// accesses, a warp row access is 256 or 512 contiguous bytes) and a run of kRun consecutive tokens
// of one batch row; it keeps the last W - 1 input rows of its channels in registers, so each input
// row is read once per run (plus W - 1 rows of halo at the run's start), the run's rows all
// loaded before the first is used. A group norm of g channels is a shuffle reduction over g / 4
// lanes.

#include <cstdint>
#include <type_traits>

#include "kda_internal.cuh"

namespace kda {
namespace {

// tokens per warp: the run's rows are held in registers (16 bf16 rows, 8 fp32 rows)
template <typename T>
constexpr int run_of() { return sizeof(T) == 2 ? 16 : 8; }
constexpr int kWarps = 8;     // warps per block

__device__ __forceinline__ void load4(const float* p, float (&v)[4]) {
    const float4 x = *reinterpret_cast<const float4*>(p);
    v[0] = x.x; v[1] = x.y; v[2] = x.z; v[3] = x.w;
}
__device__ __forceinline__ void load4(const __nv_bfloat16* p, float (&v)[4]) {
    const uint2 u = *reinterpret_cast<const uint2*>(p);
    v[0] = __uint_as_float(u.x << 16);
    v[1] = __uint_as_float(u.x & 0xffff0000u);
    v[2] = __uint_as_float(u.y << 16);
    v[3] = __uint_as_float(u.y & 0xffff0000u);
}
__device__ __forceinline__ void unpack4(const uint2& u, float (&v)[4]) {
    v[0] = __uint_as_float(u.x << 16);
    v[1] = __uint_as_float(u.x & 0xffff0000u);
    v[2] = __uint_as_float(u.y << 16);
    v[3] = __uint_as_float(u.y & 0xffff0000u);
}
__device__ __forceinline__ void unpack4(const uint4& u, float (&v)[4]) {
    v[0] = __uint_as_float(u.x);
    v[1] = __uint_as_float(u.y);
    v[2] = __uint_as_float(u.z);
    v[3] = __uint_as_float(u.w);
}
__device__ __forceinline__ void store4(float* p, const float (&v)[4]) {
    *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
}
__device__ __forceinline__ void store4(__nv_bfloat16* p, const float (&v)[4]) {
    __nv_bfloat162 a = __floats2bfloat162_rn(v[0], v[1]);
    __nv_bfloat162 b = __floats2bfloat162_rn(v[2], v[3]);
    *reinterpret_cast<uint2*>(p) =
        make_uint2(*reinterpret_cast<uint32_t*>(&a), *reinterpret_cast<uint32_t*>(&b));
}

struct ConvArgs {
    const void* x;
    const float* w;          // [C][W]
    const int32_t* cu;       // nullable: document offsets of the one packed row
    int N;                   // documents (with cu)
    void* y;
    int B, T, C;
    int act;                 // 0: none, 1: SiLU
    int group;               // 0 or the channels of one norm group (divides 128 and C)
    float eps;
    unsigned* err;
};

template <typename T, int W>
__global__ void __launch_bounds__(32 * kWarps)
short_conv_kernel(const ConvArgs a) {
    constexpr int kRun = run_of<T>();
    const int lane = threadIdx.x & 31;
    const long long warp_id = (long long)blockIdx.x * kWarps + (threadIdx.x >> 5);
    const int cgroups = (a.C + 127) / 128;
    const int runs = (a.T + kRun - 1) / kRun;
    const long long items = (long long)a.B * runs * cgroups;
    if (warp_id >= items) return;
    const int cg = (int)(warp_id % cgroups);
    const long long rr = warp_id / cgroups;
    const int b = (int)(rr / runs);
    const int t_begin = (int)(rr % runs) * kRun;
    const int t_end = min(a.T, t_begin + kRun);
    const int c0 = 128 * cg + 4 * lane;
    const bool active = c0 < a.C;   // C % 4 == 0: a lane is wholly in or out
    const T* x = static_cast<const T*>(a.x);
    T* y = static_cast<T*>(a.y);

    float w[4][W];
#pragma unroll
    for (int e = 0; e < 4; ++e)
#pragma unroll
        for (int j = 0; j < W; ++j) w[e][j] = active ? a.w[(size_t)(c0 + e) * W + j] : 0.f;

    // every input row of the run and its W - 1 rows of halo are loaded first, before the
    // document lookup below (a few dependent loads of cu_seqlens), so that all of them are in
    // flight together
    const size_t row = (size_t)a.C;
    const size_t base = (size_t)b * a.T * row + c0;
    using Raw = typename std::conditional<sizeof(T) == 2, uint2, uint4>::type;
    Raw raw[kRun], halo[W > 1 ? W - 1 : 1];
#pragma unroll
    for (int i = 0; i < W - 1; ++i) {
        const int p = t_begin - (W - 1) + i;
        halo[i] = Raw{};
        if (active && p >= 0)
            halo[i] = *reinterpret_cast<const Raw*>(x + base + (size_t)p * row);
    }
#pragma unroll
    for (int r = 0; r < kRun; ++r) {
        raw[r] = Raw{};
        if (active && t_begin + r < t_end)
            raw[r] = *reinterpret_cast<const Raw*>(x + base + (size_t)(t_begin + r) * row);
    }

    // document of the run's first token (packed row), and where the next one starts
    int doc_start = 0, next_start = a.T;
    int d = 0;
    if (a.cu) {
        // last d with cu[d] <= t_begin (binary search over the N + 1 offsets)
        int lo = 0, hi = a.N;   // cu[lo] <= t_begin < cu[hi] (cu[N] == T > t_begin)
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (a.cu[mid] <= t_begin) lo = mid;
            else hi = mid;
        }
        d = lo;
        doc_start = a.cu[d];
        next_start = a.cu[d + 1];
        if (doc_start < 0 || next_start > a.T || doc_start > next_start) {
            if (lane == 0) set_device_error(a.err, DEV_BAD_SEQLENS);
            return;
        }
    }
    // window: xw[i] holds the input at position t - (W - 1) + i, zero before the document start
    float xw[W > 1 ? W - 1 : 1][4];
#pragma unroll
    for (int i = 0; i < W - 1; ++i) {
        unpack4(halo[i], xw[i]);
        if (t_begin - (W - 1) + i < doc_start) {
#pragma unroll
            for (int e = 0; e < 4; ++e) xw[i][e] = 0.f;
        }
    }
    // pass 1: the convolution of every token of the run (outputs depend on inputs only), SiLU
    float v[kRun][4];
#pragma unroll
    for (int r = 0; r < kRun; ++r) {
        const int t = t_begin + r;
        if (t >= next_start && t < t_end) {   // a new document starts at t: restart the window
            while (d + 1 < a.N && a.cu[d + 1] <= t) ++d;
            doc_start = a.cu[d];
            next_start = a.cu[d + 1];
#pragma unroll
            for (int i = 0; i < W - 1; ++i)
#pragma unroll
                for (int e = 0; e < 4; ++e) xw[i][e] = 0.f;
        }
        float xt[4];
        unpack4(raw[r], xt);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            float s = 0.f;
#pragma unroll
            for (int i = 0; i < W - 1; ++i) s = fmaf(w[e][i], xw[i][e], s);
            v[r][e] = fmaf(w[e][W - 1], xt[e], s);
        }
        if (a.act == 1) {
#pragma unroll
            for (int e = 0; e < 4; ++e) v[r][e] = __fdividef(v[r][e], 1.f + __expf(-v[r][e]));
        }
#pragma unroll
        for (int i = 0; i + 1 < W - 1; ++i)
#pragma unroll
            for (int e = 0; e < 4; ++e) xw[i][e] = xw[i + 1][e];
        if (W > 1) {
#pragma unroll
            for (int e = 0; e < 4; ++e) xw[W > 1 ? W - 2 : 0][e] = xt[e];
        }
    }
    // pass 2: the group norms of all the run's tokens at once (independent shuffle chains)
    if (a.group > 0) {
        float ss[kRun];
#pragma unroll
        for (int r = 0; r < kRun; ++r) {
            ss[r] = 0.f;
#pragma unroll
            for (int e = 0; e < 4; ++e) ss[r] = fmaf(v[r][e], v[r][e], ss[r]);
        }
        for (int off = 1; off < a.group / 4; off <<= 1) {
#pragma unroll
            for (int r = 0; r < kRun; ++r) ss[r] += __shfl_xor_sync(0xffffffffu, ss[r], off);
        }
#pragma unroll
        for (int r = 0; r < kRun; ++r) {
            const float inv = rsqrtf(ss[r] + a.eps);
#pragma unroll
            for (int e = 0; e < 4; ++e) v[r][e] *= inv;
        }
    }
    // pass 3: stores
#pragma unroll
    for (int r = 0; r < kRun; ++r)
        if (active && t_begin + r < t_end) store4(y + base + (size_t)(t_begin + r) * row, v[r]);
}

template <typename T>
cudaError_t launch_typed(const ConvArgs& a, int W, unsigned blocks, cudaStream_t s) {
    const unsigned th = 32 * kWarps;
    switch (W) {
        case 1: short_conv_kernel<T, 1><<<blocks, th, 0, s>>>(a); break;
        case 2: short_conv_kernel<T, 2><<<blocks, th, 0, s>>>(a); break;
        case 3: short_conv_kernel<T, 3><<<blocks, th, 0, s>>>(a); break;
        case 4: short_conv_kernel<T, 4><<<blocks, th, 0, s>>>(a); break;
        case 5: short_conv_kernel<T, 5><<<blocks, th, 0, s>>>(a); break;
        case 6: short_conv_kernel<T, 6><<<blocks, th, 0, s>>>(a); break;
        case 7: short_conv_kernel<T, 7><<<blocks, th, 0, s>>>(a); break;
        case 8: short_conv_kernel<T, 8><<<blocks, th, 0, s>>>(a); break;
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_short_conv(const void* x, const float* w, const int32_t* cu, int N, void* y,
                              int B, int T, int C, int W, bool bf16, int act, int group, float eps,
                              unsigned* err, cudaStream_t stream) {
    const int run = bf16 ? run_of<__nv_bfloat16>() : run_of<float>();
    const long long items = (long long)B * ((T + run - 1) / run) * ((C + 127) / 128);
    if (items <= 0) return cudaSuccess;
    const long long blocks = (items + kWarps - 1) / kWarps;
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    ConvArgs a{x, w, cu, N, y, B, T, C, act, group, eps, err};
    return bf16 ? launch_typed<__nv_bfloat16>(a, W, (unsigned)blocks, stream)
                : launch_typed<float>(a, W, (unsigned)blocks, stream);
}

}  // namespace kda
