// Single-token decode for dk = dv = 128: the bandwidth-bound state update, in place.
//
// One token per sequence (metrale glm5next_layer page: KDA decode with a per-sequence
// KdaSeqState), recurrence from the GLM-5.3-Flash model card's Kimi Delta Attention snippet.
// The fp32 state (64 KiB per sequence-head) is read once and written once; every other byte is
// small. With S' = diag(g) S,
//     m = k^T S',  p = q^T S',  delta = beta (v - m),  o = p + (q.k) delta,  S <- S' + k delta^T
// (o equals q^T of the written state because q^T (S' + k delta^T) = p + (q.k) delta^T).
//
// Layout of the work: a 128-thread block owns one (sequence, head); warp w owns value columns
// [32w, 32w + 32). Lane l covers row phase l / 8 (rows r = l/8 + 4i, i < 32) and the four
// columns 32w + 4 (l % 8) .. + 3, so each warp load instruction reads four 128-byte row segments
// (fully coalesced 16-byte loads) and every lane keeps its 32 float4 of S in registers between
// the read and the write. The key-axis reduction is 32 rows in-thread, then a butterfly over the
// four row phases (shuffle xor 8, 16). Loads and stores of S use the streaming cache hint: the
// state is touched once per step.

#include "kda_internal.cuh"

namespace kda {
namespace {

constexpr int kD = 128;
constexpr int kRowsPerLane = 32;

__device__ __forceinline__ float4 load_v4(const __nv_bfloat16* p) {
    const uint2 u = *reinterpret_cast<const uint2*>(p);
    float4 r;
    r.x = __uint_as_float(u.x << 16);
    r.y = __uint_as_float(u.x & 0xffff0000u);
    r.z = __uint_as_float(u.y << 16);
    r.w = __uint_as_float(u.y & 0xffff0000u);
    return r;
}
__device__ __forceinline__ float4 load_v4(const float* p) {
    return *reinterpret_cast<const float4*>(p);
}
__device__ __forceinline__ void store_v4(__nv_bfloat16* p, float4 x) {
    __nv_bfloat162 a = __floats2bfloat162_rn(x.x, x.y);
    __nv_bfloat162 b = __floats2bfloat162_rn(x.z, x.w);
    uint2 u;
    u.x = *reinterpret_cast<uint32_t*>(&a);
    u.y = *reinterpret_cast<uint32_t*>(&b);
    *reinterpret_cast<uint2*>(p) = u;
}
__device__ __forceinline__ void store_v4(float* p, float4 x) {
    *reinterpret_cast<float4*>(p) = x;
}

template <typename Tin>
__global__ void __launch_bounds__(128)
decode_d128_kernel(const Tin* __restrict__ q, const Tin* __restrict__ k,
                   const Tin* __restrict__ v, const float* __restrict__ log_g,
                   const Tin* __restrict__ beta, float* __restrict__ S, Tin* __restrict__ o) {
    __shared__ float s_q[kD], s_k[kD], s_g[kD];
    const int unit = blockIdx.x;  // n * H + h
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int phase = lane >> 3;                  // row phase 0..3
    const int col = warp * 32 + (lane & 7) * 4;   // first of this lane's four columns

    float4* Sp = reinterpret_cast<float4*>(S + (size_t)unit * kD * kD);
    float4 s[kRowsPerLane];
#pragma unroll
    for (int i = 0; i < kRowsPerLane; ++i) {
        const int r = phase + 4 * i;
        s[i] = __ldcs(Sp + (r * kD + col) / 4);
    }

    const size_t vec = (size_t)unit * kD;
    s_q[tid] = load_elem(q, vec + tid);
    s_k[tid] = load_elem(k, vec + tid);
    s_g[tid] = expf(log_g[vec + tid]);
    const float4 vv = load_v4(v + vec + col);
    const float b = load_elem(beta, unit);
    __syncthreads();

    float4 m = make_float4(0.f, 0.f, 0.f, 0.f), p = m;
    float qk = 0.f;
#pragma unroll
    for (int i = 0; i < kRowsPerLane; ++i) {
        const int r = phase + 4 * i;
        const float g = s_g[r], kr = s_k[r], qr = s_q[r];
        s[i].x *= g; s[i].y *= g; s[i].z *= g; s[i].w *= g;
        m.x = fmaf(kr, s[i].x, m.x); m.y = fmaf(kr, s[i].y, m.y);
        m.z = fmaf(kr, s[i].z, m.z); m.w = fmaf(kr, s[i].w, m.w);
        p.x = fmaf(qr, s[i].x, p.x); p.y = fmaf(qr, s[i].y, p.y);
        p.z = fmaf(qr, s[i].z, p.z); p.w = fmaf(qr, s[i].w, p.w);
        qk = fmaf(qr, kr, qk);
    }
#pragma unroll
    for (int off = 8; off <= 16; off <<= 1) {
        m.x += __shfl_xor_sync(0xffffffffu, m.x, off);
        m.y += __shfl_xor_sync(0xffffffffu, m.y, off);
        m.z += __shfl_xor_sync(0xffffffffu, m.z, off);
        m.w += __shfl_xor_sync(0xffffffffu, m.w, off);
        p.x += __shfl_xor_sync(0xffffffffu, p.x, off);
        p.y += __shfl_xor_sync(0xffffffffu, p.y, off);
        p.z += __shfl_xor_sync(0xffffffffu, p.z, off);
        p.w += __shfl_xor_sync(0xffffffffu, p.w, off);
        qk += __shfl_xor_sync(0xffffffffu, qk, off);
    }
    float4 d;
    d.x = b * (vv.x - m.x); d.y = b * (vv.y - m.y);
    d.z = b * (vv.z - m.z); d.w = b * (vv.w - m.w);
    if (phase == 0) {
        float4 out;
        out.x = fmaf(qk, d.x, p.x); out.y = fmaf(qk, d.y, p.y);
        out.z = fmaf(qk, d.z, p.z); out.w = fmaf(qk, d.w, p.w);
        store_v4(o + vec + col, out);
    }
#pragma unroll
    for (int i = 0; i < kRowsPerLane; ++i) {
        const int r = phase + 4 * i;
        const float kr = s_k[r];
        s[i].x = fmaf(kr, d.x, s[i].x); s[i].y = fmaf(kr, d.y, s[i].y);
        s[i].z = fmaf(kr, d.z, s[i].z); s[i].w = fmaf(kr, d.w, s[i].w);
        __stcs(Sp + (r * kD + col) / 4, s[i]);
    }
}

// T tokens per (sequence, head) against the same state layout (speculative "verify rows", or a
// short prefill continuing a decode state): the state is read once, updated T times in
// registers and written once, so the HBM cost stays one state round trip per call. Token t of
// sequence n reads row (n * T + t) of the [N, T, H, d] inputs. The arithmetic of each token is
// that of decode_d128_kernel, in the same order.
//
// The kernel is persistent (two 128-thread blocks per SM walking the (sequence, head) units):
// while a block updates one unit's state in registers, the next unit's 64 KiB state streams into
// shared memory by bulk copy, so the reads stay in flight through the token loop instead of
// alternating with it. The inputs of up to kRowGroup tokens are staged in shared memory at once.
constexpr int kRowGroup = 8;
constexpr uint32_t kStateBytes = kD * kD * 4;

__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes,
                                         uint32_t bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        ::"r"(dst), "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
        : "memory");
}
__device__ __forceinline__ bool bar_try(uint32_t bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(bar), "r"(parity)
        : "memory");
    return done != 0;
}
// bounded wait (about a second of SM clock): false on expiry; the clock (a slow read) only once
// the first test has failed
__device__ __forceinline__ bool bar_wait(uint32_t bar, uint32_t parity) {
    if (bar_try(bar, parity)) return true;
    const long long t0 = clock64();
    for (;;) {
        if (bar_try(bar, parity)) return true;
        if (clock64() - t0 > (1ll << 31)) return false;
    }
}

template <typename Tin>
__global__ void __launch_bounds__(128, 2)
decode_d128_tokens_kernel(const Tin* __restrict__ q, const Tin* __restrict__ k,
                          const Tin* __restrict__ v, const float* __restrict__ log_g,
                          const Tin* __restrict__ beta, float* __restrict__ S,
                          Tin* __restrict__ o, int H, int T, long long units, unsigned* err) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    float* sbuf = reinterpret_cast<float*>(smem_raw);             // next unit's state
    // token rows staged per lane's access order: element r of q, k, g at [r % 4][r / 4], so that a
    // lane (row phase r % 4) reads its 32 rows as 8 float4; the phases 36 floats apart, so that
    // a warp's four phases fall in different banks (32 apart they would share them, four ways);
    // v in natural order; q.k per row
    constexpr int kPh = 36;
    __shared__ __align__(16) float s_q[kRowGroup][4][kPh], s_k[kRowGroup][4][kPh],
        s_g[kRowGroup][4][kPh], s_v[kRowGroup][kD];
    __shared__ float s_b[kRowGroup], s_qk[kRowGroup];
    __shared__ __align__(8) unsigned long long s_bar;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int phase = lane >> 3;
    const int col = warp * 32 + (lane & 7) * 4;
    const uint32_t bar = static_cast<uint32_t>(__cvta_generic_to_shared(&s_bar));
    const uint32_t dst = static_cast<uint32_t>(__cvta_generic_to_shared(sbuf));
    auto fetch = [&](long long u) {   // one thread: unit u's state into sbuf
        asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar),
                     "r"(kStateBytes)
                     : "memory");
        const uint8_t* src = reinterpret_cast<const uint8_t*>(S + (size_t)u * kD * kD);
#pragma unroll
        for (int i = 0; i < 4; ++i)
            bulk_g2s(dst + i * (kStateBytes / 4), src + i * (kStateBytes / 4), kStateBytes / 4,
                     bar);
    };
    if (tid == 0) {
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(bar) : "memory");
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        if ((long long)blockIdx.x < units) fetch(blockIdx.x);
    }
    __syncthreads();

    uint32_t parity = 0;
    bool pending = (long long)blockIdx.x < units;   // a fetch issued and not yet waited for
    for (long long unit = blockIdx.x; unit < units; unit += gridDim.x, parity ^= 1) {
        const int n = (int)(unit / H), h = (int)(unit - (long long)n * H);
        // this unit's state, from shared memory into registers
        const bool ok = bar_wait(bar, parity);
        if (__syncthreads_or(!ok)) {
            if (tid == 0) set_device_error(err, DEV_TIMEOUT);
            break;
        }
        pending = false;
        float4 s[kRowsPerLane];
#pragma unroll
        for (int i = 0; i < kRowsPerLane; ++i) {
            const int r = phase + 4 * i;
            s[i] = *reinterpret_cast<const float4*>(sbuf + r * kD + col);
        }
        __syncthreads();   // every thread has its state: the buffer takes the next unit's
        if (unit + gridDim.x < units) {
            if (tid == 0) fetch(unit + gridDim.x);
            pending = true;
        }
        float4* Sp = reinterpret_cast<float4*>(S + (size_t)unit * kD * kD);

        auto row = [&](int t) { return ((size_t)n * T + t) * H + h; };   // token row index
        for (int t0 = 0; t0 < T; t0 += kRowGroup) {
            const int nt = min(kRowGroup, T - t0);
            if (t0 > 0) __syncthreads();   // the previous group's rows are no longer read
            for (int u = 0; u < nt; ++u) {
                const size_t r = row(t0 + u);
                const float qv = load_elem(q, r * kD + tid), kv = load_elem(k, r * kD + tid);
                s_q[u][tid & 3][tid >> 2] = qv;
                s_k[u][tid & 3][tid >> 2] = kv;
                s_g[u][tid & 3][tid >> 2] = expf(log_g[r * kD + tid]);
                s_v[u][tid] = load_elem(v, r * kD + tid);
            }
            if (tid < nt) s_b[tid] = load_elem(beta, row(t0 + tid));
            __syncthreads();
            // q.k per row, once (warp u % 4 for row u), in the single step's order: lane l sums
            // rows l / 8 + 4 i over i, then a butterfly over the four row phases
            if ((lane & 7) == 0) {
                for (int u = warp; u < nt; u += 4) {
                    float qk = 0.f;
#pragma unroll
                    for (int i = 0; i < kRowsPerLane; ++i)
                        qk = fmaf(s_q[u][phase][i], s_k[u][phase][i], qk);
                    // combine the four phases as xor 8, then 16 would: (0 + 1) + (2 + 3)
                    const unsigned lanes = 0x01010101u;
                    const float a0 = __shfl_sync(lanes, qk, 0), a1 = __shfl_sync(lanes, qk, 8);
                    const float a2 = __shfl_sync(lanes, qk, 16), a3 = __shfl_sync(lanes, qk, 24);
                    if (lane == 0) s_qk[u] = (a0 + a1) + (a2 + a3);
                }
            }
            __syncthreads();
            for (int u = 0; u < nt; ++u) {
                const float4 vv = *reinterpret_cast<const float4*>(&s_v[u][col]);
                const float b = s_b[u];
                const float qk = s_qk[u];
                float4 m = make_float4(0.f, 0.f, 0.f, 0.f), p = m;
                const float4* g4 = reinterpret_cast<const float4*>(s_g[u][phase]);
                const float4* k4 = reinterpret_cast<const float4*>(s_k[u][phase]);
                const float4* q4 = reinterpret_cast<const float4*>(s_q[u][phase]);
#pragma unroll
                for (int i4 = 0; i4 < kRowsPerLane / 4; ++i4) {
                    const float4 gg = g4[i4], kk = k4[i4], qq = q4[i4];
                    const float ga[4] = {gg.x, gg.y, gg.z, gg.w}, ka[4] = {kk.x, kk.y, kk.z, kk.w},
                                qa[4] = {qq.x, qq.y, qq.z, qq.w};
#pragma unroll
                    for (int jj = 0; jj < 4; ++jj) {
                        const int i = 4 * i4 + jj;
                        const float g = ga[jj], kr = ka[jj], qr = qa[jj];
                        s[i].x *= g; s[i].y *= g; s[i].z *= g; s[i].w *= g;
                        m.x = fmaf(kr, s[i].x, m.x); m.y = fmaf(kr, s[i].y, m.y);
                        m.z = fmaf(kr, s[i].z, m.z); m.w = fmaf(kr, s[i].w, m.w);
                        p.x = fmaf(qr, s[i].x, p.x); p.y = fmaf(qr, s[i].y, p.y);
                        p.z = fmaf(qr, s[i].z, p.z); p.w = fmaf(qr, s[i].w, p.w);
                    }
                }
#pragma unroll
                for (int off = 8; off <= 16; off <<= 1) {
                    m.x += __shfl_xor_sync(0xffffffffu, m.x, off);
                    m.y += __shfl_xor_sync(0xffffffffu, m.y, off);
                    m.z += __shfl_xor_sync(0xffffffffu, m.z, off);
                    m.w += __shfl_xor_sync(0xffffffffu, m.w, off);
                    p.x += __shfl_xor_sync(0xffffffffu, p.x, off);
                    p.y += __shfl_xor_sync(0xffffffffu, p.y, off);
                    p.z += __shfl_xor_sync(0xffffffffu, p.z, off);
                    p.w += __shfl_xor_sync(0xffffffffu, p.w, off);
                }
                float4 d;
                d.x = b * (vv.x - m.x); d.y = b * (vv.y - m.y);
                d.z = b * (vv.z - m.z); d.w = b * (vv.w - m.w);
                if (phase == 0) {
                    float4 out;
                    out.x = fmaf(qk, d.x, p.x); out.y = fmaf(qk, d.y, p.y);
                    out.z = fmaf(qk, d.z, p.z); out.w = fmaf(qk, d.w, p.w);
                    store_v4(o + row(t0 + u) * kD + col, out);
                }
#pragma unroll
                for (int i4 = 0; i4 < kRowsPerLane / 4; ++i4) {
                    const float4 kk = k4[i4];
                    const float ka[4] = {kk.x, kk.y, kk.z, kk.w};
#pragma unroll
                    for (int jj = 0; jj < 4; ++jj) {
                        const int i = 4 * i4 + jj;
                        const float kr = ka[jj];
                        s[i].x = fmaf(kr, d.x, s[i].x); s[i].y = fmaf(kr, d.y, s[i].y);
                        s[i].z = fmaf(kr, d.z, s[i].z); s[i].w = fmaf(kr, d.w, s[i].w);
                    }
                }
            }
        }
#pragma unroll
        for (int i = 0; i < kRowsPerLane; ++i) {
            const int r = phase + 4 * i;
            __stcs(Sp + (r * kD + col) / 4, s[i]);
        }
        __syncthreads();   // the token rows of this unit are no longer read
    }
    // a copy still in flight (after an expired wait) lands before the shared memory goes away
    if (tid == 0 && pending) bar_wait(bar, parity);
    __syncthreads();
}

}  // namespace

cudaError_t launch_decode_tokens_d128(const DecodeParams& p, int T, cudaStream_t stream) {
    const int64_t units = (int64_t)p.N * p.H;
    if (units == 0 || T <= 0) return cudaSuccess;
    static PerDevice setup;
    static int sms[PerDevice::kMax];
    int dev = 0;
    cudaError_t e = setup.run(
        [](int d) {
            cudaError_t r = cudaFuncSetAttribute(decode_d128_tokens_kernel<__nv_bfloat16>,
                                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 (int)kStateBytes);
            if (r == cudaSuccess)
                r = cudaFuncSetAttribute(decode_d128_tokens_kernel<float>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kStateBytes);
            if (r == cudaSuccess) r = cudaDeviceGetAttribute(&sms[d], cudaDevAttrMultiProcessorCount, d);
            return r;
        },
        &dev);
    if (e != cudaSuccess) return e;
    // persistent: two blocks per SM (registers and shared memory allow two)
    const int64_t grid = units < 2LL * sms[dev] ? units : 2LL * sms[dev];
    if (p.bf16)
        decode_d128_tokens_kernel<__nv_bfloat16><<<(unsigned)grid, 128, kStateBytes, stream>>>(
            static_cast<const __nv_bfloat16*>(p.q), static_cast<const __nv_bfloat16*>(p.k),
            static_cast<const __nv_bfloat16*>(p.v), p.log_g,
            static_cast<const __nv_bfloat16*>(p.beta), p.S, static_cast<__nv_bfloat16*>(p.o),
            p.H, T, units, p.err);
    else
        decode_d128_tokens_kernel<float><<<(unsigned)grid, 128, kStateBytes, stream>>>(
            static_cast<const float*>(p.q), static_cast<const float*>(p.k),
            static_cast<const float*>(p.v), p.log_g, static_cast<const float*>(p.beta), p.S,
            static_cast<float*>(p.o), p.H, T, units, p.err);
    return cudaGetLastError();
}

cudaError_t launch_decode_d128(const DecodeParams& p, cudaStream_t stream) {
    const int64_t units = (int64_t)p.N * p.H;
    if (units == 0) return cudaSuccess;
    if (units > 0x7fffffff) return cudaErrorInvalidConfiguration;
    if (p.bf16)
        decode_d128_kernel<__nv_bfloat16><<<(unsigned)units, 128, 0, stream>>>(
            static_cast<const __nv_bfloat16*>(p.q), static_cast<const __nv_bfloat16*>(p.k),
            static_cast<const __nv_bfloat16*>(p.v), p.log_g,
            static_cast<const __nv_bfloat16*>(p.beta), p.S, static_cast<__nv_bfloat16*>(p.o));
    else
        decode_d128_kernel<float><<<(unsigned)units, 128, 0, stream>>>(
            static_cast<const float*>(p.q), static_cast<const float*>(p.k),
            static_cast<const float*>(p.v), p.log_g, static_cast<const float*>(p.beta), p.S,
            static_cast<float*>(p.o));
    return cudaGetLastError();
}

}  // namespace kda
