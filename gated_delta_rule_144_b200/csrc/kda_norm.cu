// Gated per-head RMSNorm of the KDA output, as a vectorised pass over o after the recurrence (a
// version folded into the state pass's output store was slower: it lengthened the per-chunk chain).
//
// Per (token, head): y = x / sqrt(mean over head_dim of x^2 + eps) * w * sigmoid(gate), with the
// variance accumulated in fp32 (NeMo glm5_next layers, _TorchRMSNormGated: normalise, then gate
// with a sigmoid; Glm5NextRMSNorm: fp32 variance, a weight of head_dim entries; metrale
// glm5next_layer: every norm is x * w / rms). One warp per (token, head) vector; y may alias x.

#include "kda_internal.cuh"

namespace kda {
namespace {

constexpr int kWarps = 8;

// sigmoid(g) = 1 / (1 + e^{-g}) with the fast exponential and reciprocal intrinsics (about 2 ulp
// each); exactly the arithmetic of the state pass's fused epilogue (kda_scan.cu), so that both
// give the same bits.
__device__ __forceinline__ float sigmoid_fast(float g) { return __fdividef(1.f, 1.f + __expf(-g)); }

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
__device__ __forceinline__ void store4(float* p, const float (&v)[4]) {
    *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
}
__device__ __forceinline__ void store4(__nv_bfloat16* p, const float (&v)[4]) {
    __nv_bfloat162 a = __floats2bfloat162_rn(v[0], v[1]);
    __nv_bfloat162 b = __floats2bfloat162_rn(v[2], v[3]);
    *reinterpret_cast<uint2*>(p) =
        make_uint2(*reinterpret_cast<uint32_t*>(&a), *reinterpret_cast<uint32_t*>(&b));
}

// kVec: dv is a multiple of 4 and lane l takes elements 4 (l + 32 i) .. + 3 (16- or 8-byte
// accesses); otherwise lane l takes elements l + 32 i one at a time.
template <typename T, bool kVec>
__global__ void __launch_bounds__(32 * kWarps)
out_norm_gated_kernel(const T* x, const T* __restrict__ gate, const float* __restrict__ w,
                      float eps, T* y, long long vectors, int dv) {
    const long long vec = (long long)blockIdx.x * kWarps + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (vec >= vectors) return;
    const size_t base = (size_t)vec * dv;
    constexpr int kGroups = kVec ? 2 : 8;   // dv <= 256
    constexpr int kPer = kVec ? 4 : 1;
    float xv[kGroups][kPer];
    float ss = 0.f;
#pragma unroll
    for (int i = 0; i < kGroups; ++i) {
        const int c = kVec ? 4 * (lane + 32 * i) : lane + 32 * i;
        if (c < dv) {
            if constexpr (kVec) {
                load4(x + base + c, xv[i]);
            } else {
                xv[i][0] = load_elem(x, base + c);
            }
        } else {
#pragma unroll
            for (int e = 0; e < kPer; ++e) xv[i][e] = 0.f;
        }
#pragma unroll
        for (int e = 0; e < kPer; ++e) ss = fmaf(xv[i][e], xv[i][e], ss);
    }
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
    const float inv = rsqrtf(ss / (float)dv + eps);
#pragma unroll
    for (int i = 0; i < kGroups; ++i) {
        const int c = kVec ? 4 * (lane + 32 * i) : lane + 32 * i;
        if (c >= dv) continue;
        if constexpr (kVec) {
            float g[4], out[4];
            load4(gate + base + c, g);
            const float4 wv = *reinterpret_cast<const float4*>(w + c);
            const float ws[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) out[e] = xv[i][e] * inv * ws[e] * sigmoid_fast(g[e]);
            store4(y + base + c, out);
        } else {
            const float g = load_elem(gate, base + c);
            store_elem(y, base + c, xv[i][0] * inv * w[c] * sigmoid_fast(g));
        }
    }
}

}  // namespace

cudaError_t launch_out_norm_gated(const void* x, const void* gate, const float* w, float eps,
                                  void* y, long long vectors, int dv, bool bf16,
                                  cudaStream_t stream) {
    if (vectors <= 0) return cudaSuccess;
    const long long blocks = (vectors + kWarps - 1) / kWarps;
    if (blocks > 0x7fffffffLL || dv > 256) return cudaErrorInvalidConfiguration;
    // 16-byte (fp32) / 8-byte (bf16) accesses need dv % 4 == 0 and aligned bases (the ABI
    // requires 16-byte aligned buffers; every vector then starts 8-byte aligned for bf16)
    const bool vec4 = dv % 4 == 0 && (reinterpret_cast<uintptr_t>(w) & 15) == 0;
    const unsigned g = (unsigned)blocks, t = 32 * kWarps;
    if (bf16) {
        auto* xb = static_cast<const __nv_bfloat16*>(x);
        auto* gb = static_cast<const __nv_bfloat16*>(gate);
        auto* yb = static_cast<__nv_bfloat16*>(y);
        if (vec4)
            out_norm_gated_kernel<__nv_bfloat16, true>
                <<<g, t, 0, stream>>>(xb, gb, w, eps, yb, vectors, dv);
        else
            out_norm_gated_kernel<__nv_bfloat16, false>
                <<<g, t, 0, stream>>>(xb, gb, w, eps, yb, vectors, dv);
    } else {
        auto* xf = static_cast<const float*>(x);
        auto* gf = static_cast<const float*>(gate);
        auto* yf = static_cast<float*>(y);
        if (vec4)
            out_norm_gated_kernel<float, true><<<g, t, 0, stream>>>(xf, gf, w, eps, yf, vectors, dv);
        else
            out_norm_gated_kernel<float, false><<<g, t, 0, stream>>>(xf, gf, w, eps, yf, vectors,
                                                                     dv);
    }
    return cudaGetLastError();
}

}  // namespace kda
