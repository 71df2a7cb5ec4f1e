// Gradients of the KDA recurrence (the training direction) on CUDA cores, fp32, dk = dv = 128.
//
// The reverse-mode derivative of the per-token steps (NeMo glm5_next layers, `_torch_recurrent_kda`
// is a differentiable reference KDA; the forward is the GLM-5.3-Flash model card's Kimi Delta
// Attention snippet). Per (sequence or document, head), with g_t = exp(log_g_t),
//   S'_t = diag(g_t) S_{t-1},  m_t = S'_t^T k_t,  d_t = beta_t (v_t - m_t),  S_t = S'_t + k_t d_t^T,
//   o_t = S_t^T q_t,
// and upstream gradients do_t (of o) and dhT (of the final state), tokens are taken from the last
// to the first:
//   dq_t = S_t do_t;   dS += q_t do_t^T;   dd = dS^T k_t;   dbeta_t = <dd, v_t - m_t>;
//   dv_t = beta_t dd;  dm = -beta_t dd;    dk_t = dS d_t + S'_t dm;   dS' = dS + k_t dm^T;
//   dlog_g_t = g_t * rowsum(dS' * S_{t-1});   dS = diag(g_t) dS'   (dh0 = dS after the first).
// The backward needs S_{t-1} at every token in reverse order. Each CTA first runs the forward and
// stores the state at the start of every 64-token chunk (checkpoints, in the workspace); then,
// chunk by chunk from the last, it re-runs the chunk's forward from its checkpoint, keeping the
// chunk's states and m_t, d_t in the workspace, and walks the chunk backwards.
//
// Value columns are independent in both directions: column j of S, m, d, dS and dd depends on
// column j alone. So a chain is split over 16 slices of 8 value columns, one warp each, which
// walk their columns with no exchange; only dq, dk, dlog_g (sums over columns) and dbeta are
// summed over the 16 slices, by fp32 atomic adds into outputs the launch zeroes first (the order
// of those adds is not fixed, so the last bits of dq, dk, dlog_g and dbeta may differ between
// runs; dv and dh0 are written once).
//
// Threads: one warp per slice, four independent warps per CTA; lane l owns rows 4 l .. 4 l + 3
// of the slice's S and dS (all 8 columns), so sums over columns are in-lane and sums over rows
// (m, dd) stay inside the warp: a transposing reduce-scatter on lane bits 16, 8, 4 (each lane
// keeps half of its remaining columns and adds its partner's other half), exchanges on bits 2
// and 1, then every column's total gathered to all lanes; no shared memory, no barrier. The
// token's inputs are read straight into registers (a lane's 4 rows of k, q and log g are 8 or
// 16 contiguous bytes), fetched a step ahead. The kernel's own copies of the state interleave
// the lanes' elements (every warp access is one contiguous 128-byte line), and each lane adds its
// 4 rows of dq, dk and dlog_g with one 16-byte vector reduction each. The lines of the token a
// few steps ahead are prefetched into L1. Plain fp32 arithmetic and __expf (a few ulp, far inside
// the gradients' tolerance), no tensor cores: a per-token kernel, not the chunked one. With one
// warp per scheduler it is bound by each warp's own instruction stream (about 1500 instructions
// per token over its three passes, a few cycles each).

#include <cstdint>

#include "kda_bwd.cuh"

namespace kda {
namespace {

constexpr int kD = 128;
constexpr int kCk = 64;                 // tokens per checkpointed chunk
constexpr int kCols = 8;                // value columns per slice (one warp)
constexpr int kSlices = kD / kCols;     // slices per chain
constexpr int kRows = kD / 32;          // rows per lane
constexpr int kSmat = kD * kCols;       // floats of one slice of the state
constexpr int kWarpsPerCta = 4;
static_assert(kCols == 8 && kRows == 4, "the reductions below assume 8 columns, 4 rows per lane");

struct BwdArgs {
    const void* q;
    const void* k;
    const void* v;
    const void* beta;
    const void* dout;
    const float* log_g;
    const float* h0;     // nullable
    const float* dhT;    // nullable
    const int32_t* cu;   // nullable
    float* dq;           // zeroed by the launch: the slices of a chain add into dq, dk, dlog_g, dbeta
    float* dk;
    float* dv;
    float* dlog_g;
    float* dbeta;
    float* dh0;          // nullable
    float* ckpt;         // [chains][slices][nck][kSmat]
    float* chunk_s;      // [chains][slices][kCk][kSmat]
    float* chunk_md;     // [chains][slices][kCk][2][kCols]
    int T, H, N, nck;
    long long units;     // chains x slices
    unsigned* err;
};

// 4 consecutive elements from row-major data: bf16 (8 bytes) or fp32 (16 bytes), 8- or
// 16-byte aligned (the index is a multiple of 4)
__device__ __forceinline__ void load4(const __nv_bfloat16* p, size_t i, float (&x)[4]) {
    const uint2 u = *reinterpret_cast<const uint2*>(p + i);
    x[0] = __uint_as_float(u.x << 16);
    x[1] = __uint_as_float(u.x & 0xffff0000u);
    x[2] = __uint_as_float(u.y << 16);
    x[3] = __uint_as_float(u.y & 0xffff0000u);
}
__device__ __forceinline__ void load4(const float* p, size_t i, float (&x)[4]) {
    const float4 u = *reinterpret_cast<const float4*>(p + i);
    x[0] = u.x; x[1] = u.y; x[2] = u.z; x[3] = u.w;
}
// 8 consecutive elements (the slice's columns of v or do), 16- or 32-byte aligned
__device__ __forceinline__ void load8(const __nv_bfloat16* p, size_t i, float (&x)[8]) {
    const uint4 u = *reinterpret_cast<const uint4*>(p + i);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        x[2 * e] = __uint_as_float(w[e] << 16);
        x[2 * e + 1] = __uint_as_float(w[e] & 0xffff0000u);
    }
}
__device__ __forceinline__ void load8(const float* p, size_t i, float (&x)[8]) {
    const float4 u = *reinterpret_cast<const float4*>(p + i);
    const float4 w = *reinterpret_cast<const float4*>(p + i + 4);
    x[0] = u.x; x[1] = u.y; x[2] = u.z; x[3] = u.w;
    x[4] = w.x; x[5] = w.y; x[6] = w.z; x[7] = w.w;
}
// the line holding p into this SM's L1 (p must lie inside an allocation)
__device__ __forceinline__ void prefetch_l1(const void* p) {
    asm volatile("prefetch.global.L1 [%0];" ::"l"(p));
}
// [p .. p + 3] += x, one 16-byte vector reduction (p 16-byte aligned)
__device__ __forceinline__ void red_add4(float* p, float x0, float x1, float x2, float x3) {
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(x0), "f"(x1),
                 "f"(x2), "f"(x3)
                 : "memory");
}

// Sums over the warp's 32 lanes of c[0..7] (one partial per lane and column), returned to
// every lane in c. Reduce-scatter on lane bits 16, 8, 4: a lane keeps the upper or lower half of
// its remaining columns and adds its partner's copy of that half; after three levels lane l
// holds column 4 [l & 16] + 2 [l & 8] + [l & 4] summed over 8 lanes, exchanges on bits 2 and 1
// finish it, and the 8 totals are gathered from lanes 0, 4, 8, .. 28.
__device__ __forceinline__ void warp_colsum8(float (&c)[kCols], int lane) {
    float x[4];
    {
        const bool up = lane & 16;
#pragma unroll
        for (int i = 0; i < 4; ++i)
            x[i] = (up ? c[4 + i] : c[i]) + __shfl_xor_sync(0xffffffffu, up ? c[i] : c[4 + i], 16);
    }
    float y[2];
    {
        const bool up = lane & 8;
#pragma unroll
        for (int i = 0; i < 2; ++i)
            y[i] = (up ? x[2 + i] : x[i]) + __shfl_xor_sync(0xffffffffu, up ? x[i] : x[2 + i], 8);
    }
    float z;
    {
        const bool up = lane & 4;
        z = (up ? y[1] : y[0]) + __shfl_xor_sync(0xffffffffu, up ? y[0] : y[1], 4);
    }
    z += __shfl_xor_sync(0xffffffffu, z, 2);
    z += __shfl_xor_sync(0xffffffffu, z, 1);
#pragma unroll
    for (int col = 0; col < kCols; ++col)
        c[col] = __shfl_sync(0xffffffffu, z, ((col & 4) << 2) | ((col & 2) << 2) | ((col & 1) << 2));
}

template <typename E>
__global__ void __launch_bounds__(32 * kWarpsPerCta) bwd_kernel(const BwdArgs a) {
    const int lane = threadIdx.x & 31;
    const long long unit = (long long)blockIdx.x * kWarpsPerCta + (threadIdx.x >> 5);
    if (unit >= a.units) return;
    const int chain = (int)(unit / kSlices), slice = (int)(unit % kSlices);
    const int cs0 = kCols * slice;          // first value column of the slice
    const int r0 = kRows * lane;            // first row of this lane
    const int n = chain / a.H, h = chain % a.H;
    const E* q = static_cast<const E*>(a.q);
    const E* k = static_cast<const E*>(a.k);
    const E* v = static_cast<const E*>(a.v);
    const E* beta = static_cast<const E*>(a.beta);
    const E* dout = static_cast<const E*>(a.dout);

    long long t0, L;
    if (a.cu) {
        const long long lo = a.cu[n], hi = a.cu[n + 1];
        const bool bad = hi < lo || lo < 0 || hi > a.T || (n == 0 && lo != 0) ||
                         (n == a.N - 1 && hi != a.T);
        if (bad) {
            if (lane == 0) set_device_error(a.err, DEV_BAD_SEQLENS);
            return;
        }
        t0 = lo;
        L = hi - lo;
    } else {
        t0 = (long long)n * a.T;
        L = a.T;
    }
    const int nck = (int)((L + kCk - 1) / kCk);
    if (nck > a.nck) {   // only a malformed cu_seqlens gets here
        if (lane == 0) set_device_error(a.err, DEV_BAD_SEQLENS);
        return;
    }
    const size_t mat = (size_t)kD * kD;
    float* ckpt = a.ckpt + (size_t)unit * a.nck * kSmat;
    float* cs = a.chunk_s + (size_t)unit * kCk * kSmat;
    float* cmd = a.chunk_md + (size_t)unit * kCk * 2 * kCols;
    // element (ri, c) of this lane in a caller's 128 x 128 matrix (h0, dhT, dh0), and in the
    // kernel's own copies (element e of every lane side by side)
    auto my = [&](int ri, int c) { return (size_t)(r0 + ri) * kD + cs0 + c; };
    auto ti = [&](int e) { return (size_t)e * 32 + lane; };

    // the token's inputs, fetched a step ahead: this lane's rows of k, log g (and q), the slice's
    // columns of v (and do), beta
    struct In {
        float k[kRows], lg[kRows], q[kRows], v[kCols], dout[kCols], b;
    };
    In nx;
    long long n_row = -1;
    bool n_bwd = false;
    auto fetch = [&](long long row, bool backward) {
        const size_t e = ((size_t)row * a.H + h) * kD;
        load4(k, e + r0, nx.k);
        load4(a.log_g, e + r0, nx.lg);
        load8(v, e + cs0, nx.v);
        if (backward) {
            load4(q, e + r0, nx.q);
            load8(dout, e + cs0, nx.dout);
        }
        nx.b = load_elem(beta, (size_t)row * a.H + h);
        n_row = row;
        n_bwd = backward;
    };
    // the inputs of `row` (fetched now unless they were fetched ahead), then the next row's fetch
    auto take = [&](long long row, bool backward, long long next_row, bool next_bwd) -> In {
        if (n_row != row || n_bwd != backward) fetch(row, backward);
        In cur = nx;
        if (next_row >= 0) fetch(next_row, next_bwd);
        else n_row = -1;
        return cur;
    };

    // Loads of a step wait on the previous step's fetch, so every token would take a global
    // round trip; the lines of the token kPre steps ahead are pulled into L1 instead (k, log g
    // and v in the forward passes; q and do for the reverse walk while its chunk is re-run).
    constexpr int kPre = 4;
    auto prefetch_row = [&](long long row, bool fwd_part, bool bwd_part) {
        const size_t e = ((size_t)row * a.H + h) * kD;
        if (fwd_part) {
            prefetch_l1(k + e + r0);
            prefetch_l1(a.log_g + e + r0);
            if (lane == 0) {
                prefetch_l1(v + e + cs0);
                prefetch_l1(beta + (size_t)row * a.H + h);
            }
        }
        if (bwd_part) {
            prefetch_l1(q + e + r0);
            if (lane == 0) prefetch_l1(dout + e + cs0);
        }
    };

    float S[kRows][kCols], dS[kRows][kCols];
    float gr[kRows], m[kCols], d[kCols];
    // forward step on token inputs `x`: S <- diag(g) S, m = S^T k, d = beta (v - m), S += k d^T
    auto forward_step = [&](const In& x) {
#pragma unroll
        for (int ri = 0; ri < kRows; ++ri) gr[ri] = __expf(x.lg[ri]);
#pragma unroll
        for (int c = 0; c < kCols; ++c) {
            float p = 0.f;
#pragma unroll
            for (int ri = 0; ri < kRows; ++ri) {
                S[ri][c] *= gr[ri];
                p = fmaf(x.k[ri], S[ri][c], p);
            }
            m[c] = p;
        }
        warp_colsum8(m, lane);
#pragma unroll
        for (int c = 0; c < kCols; ++c) {
            d[c] = x.b * (x.v[c] - m[c]);
#pragma unroll
            for (int ri = 0; ri < kRows; ++ri) S[ri][c] = fmaf(x.k[ri], d[c], S[ri][c]);
        }
    };

    // ---------------------------------------------------------------- forward, checkpoints
#pragma unroll
    for (int ri = 0; ri < kRows; ++ri)
#pragma unroll
        for (int c = 0; c < kCols; ++c)
            S[ri][c] = a.h0 ? a.h0[(size_t)chain * mat + my(ri, c)] : 0.f;
    for (long long s = 0; s < L; ++s) {
        if (s % kCk == 0) {
#pragma unroll
            for (int ri = 0; ri < kRows; ++ri)
#pragma unroll
                for (int c = 0; c < kCols; ++c)
                    ckpt[(size_t)(s / kCk) * kSmat + ti(ri * kCols + c)] = S[ri][c];
        }
        if (s + kPre < L) prefetch_row(t0 + s + kPre, true, false);
        // next: the token after, or the first token of the last chunk's re-run
        const In x = take(t0 + s, false, s + 1 < L ? t0 + s + 1 : t0 + (long long)(nck - 1) * kCk,
                          false);
        forward_step(x);
    }

    // ---------------------------------------------------------------- backward, chunk by chunk
#pragma unroll
    for (int ri = 0; ri < kRows; ++ri)
#pragma unroll
        for (int c = 0; c < kCols; ++c)
            dS[ri][c] = a.dhT ? a.dhT[(size_t)chain * mat + my(ri, c)] : 0.f;
    for (int ci = nck - 1; ci >= 0; --ci) {
        const long long s0 = (long long)ci * kCk;
        const long long s1 = min(L, s0 + kCk);
        // the chunk's forward again, keeping S_{s-1}, m_s and d_s of every token
#pragma unroll
        for (int ri = 0; ri < kRows; ++ri)
#pragma unroll
            for (int c = 0; c < kCols; ++c)
                S[ri][c] = ckpt[(size_t)ci * kSmat + ti(ri * kCols + c)];
        for (long long s = s0; s < s1; ++s) {
            const size_t j = (size_t)(s - s0);
#pragma unroll
            for (int ri = 0; ri < kRows; ++ri)
#pragma unroll
                for (int c = 0; c < kCols; ++c) cs[j * kSmat + ti(ri * kCols + c)] = S[ri][c];
            if (s + kPre < s1) prefetch_row(t0 + s + kPre, true, false);
            prefetch_row(t0 + s, false, true);   // q and do of this row, for the reverse walk
            // next: the token after, or the chunk's last token for the backward walk
            const In x = s + 1 < s1 ? take(t0 + s, false, t0 + s + 1, false)
                                    : take(t0 + s, false, t0 + s1 - 1, true);
            forward_step(x);
            if (lane < kCols) {   // every lane holds all of m and d; lane c stores column c
                float mv = m[0], dv = d[0];
#pragma unroll
                for (int c = 1; c < kCols; ++c)
                    if (lane == c) mv = m[c], dv = d[c];
                cmd[j * 2 * kCols + lane] = mv;
                cmd[j * 2 * kCols + kCols + lane] = dv;
            }
        }
        // the chunk's tokens from the last to the first. S_{s-1}, m_s and d_s (stored by this
        // warp in the pass above; lanes 0-7 wrote m and d) are read a step ahead.
        __syncwarp();
        float Sn[kRows][kCols], mn[kCols], dn[kCols];
        auto load_sd = [&](size_t j) {
#pragma unroll
            for (int c = 0; c < kCols; ++c) {
                mn[c] = cmd[j * 2 * kCols + c];
                dn[c] = cmd[j * 2 * kCols + kCols + c];
            }
#pragma unroll
            for (int ri = 0; ri < kRows; ++ri)
#pragma unroll
                for (int c = 0; c < kCols; ++c) Sn[ri][c] = cs[j * kSmat + ti(ri * kCols + c)];
        };
        load_sd((size_t)(s1 - 1 - s0));
        for (long long s = s1 - 1; s >= s0; --s) {
            const size_t j = (size_t)(s - s0);
            const long long row = t0 + s;
            // next: the token before, or the first token of the previous chunk's re-run
            const In x = s > s0 ? take(row, true, row - 1, true)
                                : take(row, true, ci > 0 ? t0 + (long long)(ci - 1) * kCk : -1,
                                       false);
#pragma unroll
            for (int c = 0; c < kCols; ++c) {
                m[c] = mn[c];
                d[c] = dn[c];
            }
#pragma unroll
            for (int ri = 0; ri < kRows; ++ri)
#pragma unroll
                for (int c = 0; c < kCols; ++c) S[ri][c] = Sn[ri][c];   // S_{s-1}
            if (s > s0) load_sd(j - 1);
            if (s - kPre >= s0) {   // the stored state and read-outs kPre tokens back
                const size_t jp = j - kPre;
                prefetch_l1(cs + jp * kSmat + (size_t)lane * 32);   // its 32 lines, one per lane
                if (lane == 0) prefetch_l1(cmd + jp * 2 * kCols);
            }
#pragma unroll
            for (int ri = 0; ri < kRows; ++ri) gr[ri] = __expf(x.lg[ri]);
            float pq[kRows], pk[kRows], dd[kCols];
#pragma unroll
            for (int ri = 0; ri < kRows; ++ri) {
                pq[ri] = 0.f;
                pk[ri] = 0.f;
            }
#pragma unroll
            for (int c = 0; c < kCols; ++c) {
                float p = 0.f;
#pragma unroll
                for (int ri = 0; ri < kRows; ++ri) {
                    const float st = fmaf(gr[ri], S[ri][c], x.k[ri] * d[c]);   // S_s
                    pq[ri] = fmaf(st, x.dout[c], pq[ri]);
                    dS[ri][c] = fmaf(x.q[ri], x.dout[c], dS[ri][c]);
                    pk[ri] = fmaf(dS[ri][c], d[c], pk[ri]);
                    p = fmaf(x.k[ri], dS[ri][c], p);
                }
                dd[c] = p;
            }
            warp_colsum8(dd, lane);   // dd = dS^T k
            const float bt = x.b;
            float pb = 0.f;
#pragma unroll
            for (int c = 0; c < kCols; ++c) pb = fmaf(dd[c], x.v[c] - m[c], pb);
            if (lane < kCols) {
                float ddv = dd[0];
#pragma unroll
                for (int c = 1; c < kCols; ++c)
                    if (lane == c) ddv = dd[c];
                a.dv[((size_t)row * a.H + h) * kD + cs0 + lane] = bt * ddv;
            }
            if (lane == 0) atomicAdd(a.dbeta + (size_t)row * a.H + h, pb);
            float pg[kRows];
#pragma unroll
            for (int ri = 0; ri < kRows; ++ri) pg[ri] = 0.f;
#pragma unroll
            for (int c = 0; c < kCols; ++c) {
                const float dm = -bt * dd[c];
#pragma unroll
                for (int ri = 0; ri < kRows; ++ri) {
                    const float sp = gr[ri] * S[ri][c];   // S'_s
                    pk[ri] = fmaf(sp, dm, pk[ri]);
                    const float dsp = fmaf(x.k[ri], dm, dS[ri][c]);
                    pg[ri] = fmaf(dsp, S[ri][c], pg[ri]);
                    dS[ri][c] = gr[ri] * dsp;
                }
            }
            {   // this lane's rows' sums over the slice's columns
                const size_t e = ((size_t)row * a.H + h) * kD + r0;
                red_add4(a.dq + e, pq[0], pq[1], pq[2], pq[3]);
                red_add4(a.dk + e, pk[0], pk[1], pk[2], pk[3]);
                red_add4(a.dlog_g + e, gr[0] * pg[0], gr[1] * pg[1], gr[2] * pg[2],
                         gr[3] * pg[3]);
            }
        }
    }
    if (a.dh0) {
#pragma unroll
        for (int ri = 0; ri < kRows; ++ri)
#pragma unroll
            for (int c = 0; c < kCols; ++c) a.dh0[(size_t)chain * mat + my(ri, c)] = dS[ri][c];
    }
}

}  // namespace

size_t bwd_workspace_bytes(long long chains, int T) {
    const long long nck = (T + kCk - 1) / kCk + 1;
    return (size_t)chains * ((size_t)(nck + kCk) * kD * kD + (size_t)kCk * 2 * kD) * sizeof(float);
}

cudaError_t launch_bwd(const BwdParams& p, cudaStream_t stream) {
    const long long chains = (long long)p.N * p.H;
    if (chains == 0) return cudaSuccess;
    if (chains * kSlices / kWarpsPerCta + 1 > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    // the CTAs of a chain add their slices' parts of dq, dk, dlog_g and dbeta
    const size_t rows = (size_t)(p.cu_seqlens ? 1 : p.N) * p.T * p.H;
    cudaError_t e;
    if ((e = cudaMemsetAsync(p.dq, 0, rows * kD * sizeof(float), stream)) != cudaSuccess ||
        (e = cudaMemsetAsync(p.dk, 0, rows * kD * sizeof(float), stream)) != cudaSuccess ||
        (e = cudaMemsetAsync(p.dlog_g, 0, rows * kD * sizeof(float), stream)) != cudaSuccess ||
        (e = cudaMemsetAsync(p.dbeta, 0, rows * sizeof(float), stream)) != cudaSuccess)
        return e;
    BwdArgs a;
    a.q = p.q;
    a.k = p.k;
    a.v = p.v;
    a.beta = p.beta;
    a.dout = p.dout;
    a.log_g = p.log_g;
    a.h0 = p.h0;
    a.dhT = p.dhT;
    a.cu = p.cu_seqlens;
    a.dq = p.dq;
    a.dk = p.dk;
    a.dv = p.dv;
    a.dlog_g = p.dlog_g;
    a.dbeta = p.dbeta;
    a.dh0 = p.dh0;
    const long long nck = (p.T + kCk - 1) / kCk + 1;
    float* w = static_cast<float*>(p.workspace);
    a.ckpt = w;
    a.chunk_s = a.ckpt + (size_t)chains * nck * kD * kD;
    a.chunk_md = a.chunk_s + (size_t)chains * kCk * kD * kD;
    a.T = p.T;
    a.H = p.H;
    a.N = p.N;
    a.nck = (int)nck;
    a.units = chains * kSlices;
    a.err = p.err;
    const unsigned grid = (unsigned)((a.units + kWarpsPerCta - 1) / kWarpsPerCta);
    if (p.bf16)
        bwd_kernel<__nv_bfloat16><<<grid, 32 * kWarpsPerCta, 0, stream>>>(a);
    else
        bwd_kernel<float><<<grid, 32 * kWarpsPerCta, 0, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace kda
