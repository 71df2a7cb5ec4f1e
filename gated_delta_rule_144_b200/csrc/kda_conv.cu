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
// Work split: a warp owns 32 * CH consecutive channels (CH = 4 per lane) and a segment of 64
// consecutive tokens of one batch row, which it streams through in blocks of rows: the next
// block's rows are in flight while the current one is computed, and the last W - 1 input rows of
// its channels stay in registers, so each input row is read once (plus W - 1 rows of halo at the
// segment's start). A block inside one document is computed without branches, so that its rows'
// conv, SiLU and norm chains interleave; a block with a document start or the segment's end goes
// row by row. A group norm of g channels is a shuffle reduction over g / CH lanes.

#include <cstdint>

#include "kda_internal.cuh"

namespace kda {
namespace {

constexpr int kWarps = 4;     // warps per block
// channels per lane: 8-byte bf16 / 16-byte fp32 accesses, a warp row is 256 or 512 contiguous
// bytes (eight per lane measured 5 % slower: its registers allow fewer warps per SM)
constexpr int kCh = 4;

// A lane's CH consecutive channels of one row, as raw words (CH * sizeof(T) bytes: 8, 16 or 32).
template <typename T, int CH>
struct Row {
    static constexpr int kWords = CH * (int)sizeof(T) / 4;
    uint32_t u[kWords];
    __device__ __forceinline__ void zero() {
#pragma unroll
        for (int i = 0; i < kWords; ++i) u[i] = 0u;
    }
    __device__ __forceinline__ void load(const T* p) {
        if constexpr (kWords == 2) {
            const uint2 x = *reinterpret_cast<const uint2*>(p);
            u[0] = x.x; u[1] = x.y;
        } else {
#pragma unroll
            for (int i = 0; i < kWords; i += 4) {
                const uint4 x = *reinterpret_cast<const uint4*>(reinterpret_cast<const uint32_t*>(p) + i);
                u[i] = x.x; u[i + 1] = x.y; u[i + 2] = x.z; u[i + 3] = x.w;
            }
        }
    }
    __device__ __forceinline__ void unpack(float (&v)[CH]) const {
        if constexpr (sizeof(T) == 2) {
#pragma unroll
            for (int i = 0; i < kWords; ++i) {
                v[2 * i] = __uint_as_float(u[i] << 16);
                v[2 * i + 1] = __uint_as_float(u[i] & 0xffff0000u);
            }
        } else {
#pragma unroll
            for (int i = 0; i < CH; ++i) v[i] = __uint_as_float(u[i]);
        }
    }
};

template <typename T, int CH>
__device__ __forceinline__ void store_row(T* p, const float (&v)[CH]) {
    if constexpr (sizeof(T) == 2) {
        uint32_t w[CH / 2];
#pragma unroll
        for (int i = 0; i < CH / 2; ++i) {
            __nv_bfloat162 b = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
            w[i] = *reinterpret_cast<uint32_t*>(&b);
        }
        if constexpr (CH == 4) {
            *reinterpret_cast<uint2*>(p) = make_uint2(w[0], w[1]);
        } else {
            *reinterpret_cast<uint4*>(p) = make_uint4(w[0], w[1], w[2], w[3]);
        }
    } else {
#pragma unroll
        for (int i = 0; i < CH; i += 4)
            *reinterpret_cast<float4*>(p + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
    }
}

// x sigmoid(x), with the fast exponential and division (subnormals flushed in this file)
__device__ __forceinline__ float silu(float x) { return __fdividef(x, 1.f + __expf(-x)); }

// tokens per warp item, and input rows in flight per lane (64 bytes of loads per lane)
constexpr int kSeg = 64;
template <typename T, int CH>
constexpr int ahead_of() {
    return 64 / (CH * (int)sizeof(T)) < 2 ? 2 : 64 / (CH * (int)sizeof(T));
}

struct ConvArgs {
    const void* x;
    const float* w;          // [C][W]
    const int32_t* cu;       // nullable: document offsets of the one packed row
    int N;                   // documents (with cu)
    void* y;
    int B, T, C;
    int act;                 // 0: none, 1: SiLU
    int group;               // 0 or the channels of one norm group (>= CH; divides C)
    float eps;
    unsigned* err;
};

template <typename T, int W, int CH>
__global__ void __launch_bounds__(32 * kWarps)
short_conv_kernel(const ConvArgs a) {
    constexpr int kAhead = ahead_of<T, CH>();
    constexpr int kSpan = 32 * CH;   // channels per warp
    constexpr int kHalo = W > 1 ? W - 1 : 1;
    const int lane = threadIdx.x & 31;
    const long long warp_id = (long long)blockIdx.x * kWarps + (threadIdx.x >> 5);
    const int cgroups = (a.C + kSpan - 1) / kSpan;
    const int segs = (a.T + kSeg - 1) / kSeg;
    const long long items = (long long)a.B * segs * cgroups;
    if (warp_id >= items) return;
    const int cg = (int)(warp_id % cgroups);
    const long long rr = warp_id / cgroups;
    const int b = (int)(rr / segs);
    const int t_begin = (int)(rr % segs) * kSeg;
    const int t_end = min(a.T, t_begin + kSeg);
    const int c0 = kSpan * cg + CH * lane;
    const bool active = c0 < a.C;   // C % CH == 0: a lane is wholly in or out
    const size_t row = (size_t)a.C;
    const T* xb = static_cast<const T*>(a.x) + (size_t)b * a.T * row + c0;
    T* yb = static_cast<T*>(a.y) + (size_t)b * a.T * row + c0;

    // the W - 1 halo rows and the first kAhead rows go out before anything waits on memory
    Row<T, CH> halo[kHalo], raw[kAhead];
#pragma unroll
    for (int i = 0; i < W - 1; ++i) {
        const int p = t_begin - (W - 1) + i;
        halo[i].zero();
        if (active && p >= 0) halo[i].load(xb + (size_t)p * row);
    }
#pragma unroll
    for (int j = 0; j < kAhead; ++j) {
        raw[j].zero();
        if (active && t_begin + j < t_end) raw[j].load(xb + (size_t)(t_begin + j) * row);
    }
    float w[CH][W];
#pragma unroll
    for (int e = 0; e < CH; ++e)
#pragma unroll
        for (int j = 0; j < W; ++j) w[e][j] = active ? a.w[(size_t)(c0 + e) * W + j] : 0.f;

    // document of the segment's first token (packed row), and where the next one starts
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
    float xw[kHalo][CH];
#pragma unroll
    for (int i = 0; i < W - 1; ++i) {
        halo[i].unpack(xw[i]);
        if (t_begin - (W - 1) + i < doc_start) {
#pragma unroll
            for (int e = 0; e < CH; ++e) xw[i][e] = 0.f;
        }
    }
    const int lanes_per_group = a.group / CH;
    for (int t0 = t_begin; t0 < t_end; t0 += kAhead) {
        if (t0 + kAhead <= t_end && t0 + kAhead <= next_start) {
            // the common case: kAhead whole rows inside one document, computed branch-free so
            // that their conv, SiLU and norm chains interleave
            float v[kAhead][CH];
#pragma unroll
            for (int j = 0; j < kAhead; ++j) {
                float xt[CH];
                raw[j].unpack(xt);
                if (active && t0 + j + kAhead < t_end)
                    raw[j].load(xb + (size_t)(t0 + j + kAhead) * row);
#pragma unroll
                for (int e = 0; e < CH; ++e) {
                    float s = 0.f;
#pragma unroll
                    for (int i = 0; i < W - 1; ++i) s = fmaf(w[e][i], xw[i][e], s);
                    v[j][e] = fmaf(w[e][W - 1], xt[e], s);
                }
#pragma unroll
                for (int i = 0; i + 1 < W - 1; ++i)
#pragma unroll
                    for (int e = 0; e < CH; ++e) xw[i][e] = xw[i + 1][e];
                if (W > 1) {
#pragma unroll
                    for (int e = 0; e < CH; ++e) xw[kHalo - 1][e] = xt[e];
                }
            }
            if (a.act == 1) {
#pragma unroll
                for (int j = 0; j < kAhead; ++j)
#pragma unroll
                    for (int e = 0; e < CH; ++e) v[j][e] = silu(v[j][e]);
            }
            if (lanes_per_group > 0) {
                float ss[kAhead];
#pragma unroll
                for (int j = 0; j < kAhead; ++j) {
                    ss[j] = 0.f;
#pragma unroll
                    for (int e = 0; e < CH; ++e) ss[j] = fmaf(v[j][e], v[j][e], ss[j]);
                }
#pragma unroll
                for (int off = 1; off < 32; off <<= 1) {
                    if (off < lanes_per_group) {
#pragma unroll
                        for (int j = 0; j < kAhead; ++j)
                            ss[j] += __shfl_xor_sync(0xffffffffu, ss[j], off);
                    }
                }
#pragma unroll
                for (int j = 0; j < kAhead; ++j) {
                    const float inv = rsqrtf(ss[j] + a.eps);
#pragma unroll
                    for (int e = 0; e < CH; ++e) v[j][e] *= inv;
                }
            }
            if (active) {
#pragma unroll
                for (int j = 0; j < kAhead; ++j)
                    store_row<T, CH>(yb + (size_t)(t0 + j) * row, v[j]);
            }
            continue;
        }
        // a document boundary or the segment's end falls in this block: row by row
#pragma unroll
        for (int j = 0; j < kAhead; ++j) {
            const int t = t0 + j;
            if (t >= t_end) break;
            float xt[CH];
            raw[j].unpack(xt);
            // the row kAhead further on takes this row's registers
            if (active && t + kAhead < t_end) raw[j].load(xb + (size_t)(t + kAhead) * row);
            if (t >= next_start) {   // a new document starts at t: restart the window
                while (d + 1 < a.N && a.cu[d + 1] <= t) ++d;
                next_start = a.cu[d + 1];
#pragma unroll
                for (int i = 0; i < W - 1; ++i)
#pragma unroll
                    for (int e = 0; e < CH; ++e) xw[i][e] = 0.f;
            }
            float v[CH];
#pragma unroll
            for (int e = 0; e < CH; ++e) {
                float s = 0.f;
#pragma unroll
                for (int i = 0; i < W - 1; ++i) s = fmaf(w[e][i], xw[i][e], s);
                v[e] = fmaf(w[e][W - 1], xt[e], s);
            }
            if (a.act == 1) {
#pragma unroll
                for (int e = 0; e < CH; ++e) v[e] = silu(v[e]);
            }
            if (lanes_per_group > 0) {
                float ss = 0.f;
#pragma unroll
                for (int e = 0; e < CH; ++e) ss = fmaf(v[e], v[e], ss);
#pragma unroll
                for (int off = 1; off < 32; off <<= 1)
                    if (off < lanes_per_group) ss += __shfl_xor_sync(0xffffffffu, ss, off);
                const float inv = rsqrtf(ss + a.eps);
#pragma unroll
                for (int e = 0; e < CH; ++e) v[e] *= inv;
            }
            if (active) store_row<T, CH>(yb + (size_t)t * row, v);
#pragma unroll
            for (int i = 0; i + 1 < W - 1; ++i)
#pragma unroll
                for (int e = 0; e < CH; ++e) xw[i][e] = xw[i + 1][e];
            if (W > 1) {
#pragma unroll
                for (int e = 0; e < CH; ++e) xw[kHalo - 1][e] = xt[e];
            }
        }
    }
}

template <typename T, int CH>
cudaError_t launch_typed(const ConvArgs& a, int W, unsigned blocks, cudaStream_t s) {
    const unsigned th = 32 * kWarps;
    switch (W) {
        case 1: short_conv_kernel<T, 1, CH><<<blocks, th, 0, s>>>(a); break;
        case 2: short_conv_kernel<T, 2, CH><<<blocks, th, 0, s>>>(a); break;
        case 3: short_conv_kernel<T, 3, CH><<<blocks, th, 0, s>>>(a); break;
        case 4: short_conv_kernel<T, 4, CH><<<blocks, th, 0, s>>>(a); break;
        case 5: short_conv_kernel<T, 5, CH><<<blocks, th, 0, s>>>(a); break;
        case 6: short_conv_kernel<T, 6, CH><<<blocks, th, 0, s>>>(a); break;
        case 7: short_conv_kernel<T, 7, CH><<<blocks, th, 0, s>>>(a); break;
        case 8: short_conv_kernel<T, 8, CH><<<blocks, th, 0, s>>>(a); break;
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

template <typename T, int CH>
cudaError_t launch_ch(const ConvArgs& a, int W, cudaStream_t stream) {
    const long long items =
        (long long)a.B * ((a.T + kSeg - 1) / kSeg) * ((a.C + 32 * CH - 1) / (32 * CH));
    if (items <= 0) return cudaSuccess;
    const long long blocks = (items + kWarps - 1) / kWarps;
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    return launch_typed<T, CH>(a, W, (unsigned)blocks, stream);
}

}  // namespace

cudaError_t launch_short_conv(const void* x, const float* w, const int32_t* cu, int N, void* y,
                              int B, int T, int C, int W, bool bf16, int act, int group, float eps,
                              unsigned* err, cudaStream_t stream) {
    ConvArgs a{x, w, cu, N, y, B, T, C, act, group, eps, err};
    return bf16 ? launch_ch<__nv_bfloat16, kCh>(a, W, stream) : launch_ch<float, kCh>(a, W, stream);
}

}  // namespace kda
