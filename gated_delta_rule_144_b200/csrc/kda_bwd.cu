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
// column j alone. So a chain is split over 32 CTAs of 4 value columns each, which walk their
// columns with no exchange; only dq, dk, dlog_g (sums over columns) and dbeta are summed over the
// 32 CTAs, by fp32 atomic adds into outputs the launch zeroes first (the order of those adds is
// not fixed, so the last bits of dq, dk, dlog_g and dbeta may differ between runs; dv and dh0 are
// written once).
//
// Threads: 128 per CTA; thread r owns row r of the slice's S and dS (4 columns). Sums over
// columns are in-thread; sums over rows (m, dd) are a reduce-scatter over the 32 rows of a warp
// (6 shuffles) and a sum over the 4 warps in shared memory. The kernel's own copies of the state interleave the threads' elements, so that every
// warp access to them is one contiguous 128-byte line; the next token's inputs are fetched into
// registers a step ahead. Plain fp32 arithmetic and expf, no tensor cores: a per-token kernel,
// not the chunked one.

#include <cstdint>

#include "kda_bwd.cuh"

namespace kda {
namespace {

constexpr int kD = 128;
constexpr int kCk = 64;                 // tokens per checkpointed chunk
// CTAs per chain (prefill-t4096 on one B200: 8, 16, 32 slices take 19.8, 13.1, 12.1 ms)
constexpr int kSlices = 32;
constexpr int kCols = kD / kSlices;     // value columns per CTA, all held by each thread
constexpr int kThreads = kD;            // one row of the slice per thread
constexpr int kWarps = kThreads / 32;
constexpr int kSmat = kD * kCols;       // floats of one slice of the state
static_assert(kCols == 4 || kCols == 8, "4 or 8 value columns per CTA");

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
    float* dq;           // zeroed by the launch: the CTAs of a chain add into dq, dk, dlog_g, dbeta
    float* dk;
    float* dv;
    float* dlog_g;
    float* dbeta;
    float* dh0;          // nullable
    float* ckpt;         // [chains][slices][nck][kSmat]
    float* chunk_s;      // [chains][slices][kCk][kSmat]
    float* chunk_md;     // [chains][slices][kCk][2][kCols]
    int T, H, N, nck;
    unsigned* err;
};

template <typename E>
__global__ void __launch_bounds__(kThreads, 512 / kThreads) bwd_kernel(const BwdArgs a) {
    __shared__ float q_s[kD], k_s[kD], g_s[kD];
    __shared__ float v_s[kCols], do_s[kCols], m_s[kCols], d_s[kCols], x_s[kCols];
    __shared__ float part[kWarps][kCols];
    __shared__ float beta_s;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int r = tid;                      // row of S
    const int chain = blockIdx.x / kSlices, slice = blockIdx.x % kSlices;
    const int cs0 = kCols * slice;          // first value column of the slice
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
            if (tid == 0) set_device_error(a.err, DEV_BAD_SEQLENS);
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
        if (tid == 0) set_device_error(a.err, DEV_BAD_SEQLENS);
        return;
    }
    const size_t mat = (size_t)kD * kD;
    const size_t unit = (size_t)chain * kSlices + slice;
    float* ckpt = a.ckpt + unit * a.nck * kSmat;
    float* cs = a.chunk_s + unit * kCk * kSmat;
    float* cmd = a.chunk_md + unit * kCk * 2 * kCols;
    // this thread's 8 elements in a caller's 128 x 128 matrix (h0, dhT, dh0)
    const size_t my = (size_t)r * kD + cs0;
    // the same elements in the kernel's own copies: element i of every thread side by side
    auto ti = [&](int i) { return (size_t)i * kThreads + tid; };

    // Inputs of token row `row` into shared memory: threads < 128 one key channel each (k, log g,
    // q), threads < 16 one of the slice's value columns (v, do). The next row staged is fetched
    // into registers right after, so its loads are in flight during this step; a row that was
    // not fetched ahead is loaded on the spot.
    float nk = 0.f, nlg = 0.f, nq = 0.f, nv = 0.f, ndo = 0.f, nb = 0.f;
    long long n_row = -1;
    bool n_bwd = false;
    auto fetch = [&](long long row, bool backward) {
        if (tid < kD) {
            const size_t e = ((size_t)row * a.H + h) * kD;
            nk = load_elem(k, e + tid);
            nlg = a.log_g[e + tid];
            if (backward) nq = load_elem(q, e + tid);
            if (tid < kCols) {
                nv = load_elem(v, e + cs0 + tid);
                if (backward) ndo = load_elem(dout, e + cs0 + tid);
            }
            if (tid == 0) nb = load_elem(beta, (size_t)row * a.H + h);
        }
        n_row = row;
        n_bwd = backward;
    };
    auto stage = [&](long long row, bool backward, long long next_row, bool next_bwd) {
        __syncthreads();   // the previous step has finished reading the staged values
        if (n_row != row || n_bwd != backward) fetch(row, backward);
        if (tid < kD) {
            k_s[tid] = nk;
            g_s[tid] = expf(nlg);
            if (backward) q_s[tid] = nq;
            if (tid < kCols) {
                v_s[tid] = nv;
                if (backward) do_s[tid] = ndo;
            }
            if (tid == 0) beta_s = nb;
        }
        __syncthreads();
        if (next_row >= 0) fetch(next_row, next_bwd);
        else n_row = -1;
    };
    // out[c] = sum over the 128 rows of f(c); the result lands in shared memory for every thread
    // after the call. Within a warp (32 rows) each lane first keeps one column summed over a group
    // of rows (halving exchanges on lane bits 16, 8 (, 4): a lane keeps the upper or lower half of
    // its columns and adds its partner's), plain exchanges then finish the warp's 32 rows, and the
    // 4 warps' partials are added in shared memory.
    auto colsum = [&](auto f, float* out) {
        float c[kCols];
#pragma unroll
        for (int i = 0; i < kCols; ++i) c[i] = f(i);
        int col = 0;
#pragma unroll
        for (int half = kCols / 2, bit = 16; half >= 1; half >>= 1, bit >>= 1) {
            const bool up = lane & bit;
#pragma unroll
            for (int i = 0; i < half; ++i)
                c[i] = (up ? c[half + i] : c[i]) +
                       __shfl_xor_sync(0xffffffffu, up ? c[i] : c[half + i], bit);
            if (up) col += half;
        }
#pragma unroll
        for (int bit = 16 / kCols; bit >= 1; bit >>= 1) c[0] += __shfl_xor_sync(0xffffffffu, c[0], bit);
        if ((lane & (2 * (16 / kCols) - 1)) == 0) part[warp][col] = c[0];
        __syncthreads();
        if (tid < kCols) {
            float s = 0.f;
#pragma unroll
            for (int w = 0; w < kWarps; ++w) s += part[w][tid];
            out[tid] = s;
        }
        __syncthreads();
    };

    float S[kCols], dS[kCols];
    // forward step on the staged token: S <- S' + k d^T; m and d land in m_s, d_s
    auto forward_step = [&]() {
        const float gr = g_s[r], kr = k_s[r];
#pragma unroll
        for (int i = 0; i < kCols; ++i) S[i] *= gr;
        colsum([&](int i) { return kr * S[i]; }, m_s);
        if (tid < kCols) d_s[tid] = beta_s * (v_s[tid] - m_s[tid]);
        __syncthreads();
#pragma unroll
        for (int i = 0; i < kCols; ++i) S[i] += kr * d_s[i];
    };

    // ---------------------------------------------------------------- forward, checkpoints
#pragma unroll
    for (int i = 0; i < kCols; ++i) S[i] = a.h0 ? a.h0[(size_t)chain * mat + my + i] : 0.f;
    for (long long s = 0; s < L; ++s) {
        if (s % kCk == 0) {
#pragma unroll
            for (int i = 0; i < kCols; ++i) ckpt[(size_t)(s / kCk) * kSmat + ti(i)] = S[i];
        }
        // next: the token after, or the first token of the last chunk's re-run
        stage(t0 + s, false, s + 1 < L ? t0 + s + 1 : t0 + (long long)(nck - 1) * kCk, false);
        forward_step();
    }

    // ---------------------------------------------------------------- backward, chunk by chunk
#pragma unroll
    for (int i = 0; i < kCols; ++i) dS[i] = a.dhT ? a.dhT[(size_t)chain * mat + my + i] : 0.f;
    for (int ci = nck - 1; ci >= 0; --ci) {
        const long long s0 = (long long)ci * kCk;
        const long long s1 = min(L, s0 + kCk);
        // the chunk's forward again, keeping S_{s-1}, m_s and d_s of every token
#pragma unroll
        for (int i = 0; i < kCols; ++i) S[i] = ckpt[(size_t)ci * kSmat + ti(i)];
        for (long long s = s0; s < s1; ++s) {
            const size_t j = (size_t)(s - s0);
#pragma unroll
            for (int i = 0; i < kCols; ++i) cs[j * kSmat + ti(i)] = S[i];
            // next: the token after, or the chunk's last token for the backward walk
            if (s + 1 < s1) stage(t0 + s, false, t0 + s + 1, false);
            else stage(t0 + s, false, t0 + s1 - 1, true);
            forward_step();
            if (tid < kCols) {
                cmd[j * 2 * kCols + tid] = m_s[tid];
                cmd[j * 2 * kCols + kCols + tid] = d_s[tid];
            }
        }
        // the chunk's tokens from the last to the first
        for (long long s = s1 - 1; s >= s0; --s) {
            const size_t j = (size_t)(s - s0);
            const long long row = t0 + s;
            // next: the token before, or the first token of the previous chunk's re-run
            if (s > s0) stage(row, true, row - 1, true);
            else stage(row, true, ci > 0 ? t0 + (long long)(ci - 1) * kCk : -1, false);
            if (tid < kCols) {   // written by this same thread in the pass above
                m_s[tid] = cmd[j * 2 * kCols + tid];
                d_s[tid] = cmd[j * 2 * kCols + kCols + tid];
            }
#pragma unroll
            for (int i = 0; i < kCols; ++i) S[i] = cs[j * kSmat + ti(i)];   // S_{s-1}
            __syncthreads();
            const float gr = g_s[r], kr = k_s[r], qr = q_s[r];
            float pq = 0.f, pk = 0.f;
#pragma unroll
            for (int i = 0; i < kCols; ++i) {
                const float dl = d_s[i], dov = do_s[i];
                const float st = gr * S[i] + kr * dl;   // S_s
                pq = fmaf(st, dov, pq);
                dS[i] = fmaf(qr, dov, dS[i]);
                pk = fmaf(dS[i], dl, pk);
            }
            colsum([&](int i) { return kr * dS[i]; }, x_s);   // dd
            const float bt = beta_s;
            if (tid < kCols) {   // the first lanes of warp 0
                const float dd = x_s[tid];
                a.dv[((size_t)row * a.H + h) * kD + cs0 + tid] = bt * dd;
                float p = dd * (v_s[tid] - m_s[tid]);
#pragma unroll
                for (int off = kCols / 2; off >= 1; off >>= 1)
                    p += __shfl_xor_sync((1u << kCols) - 1u, p, off);
                if (tid == 0) atomicAdd(a.dbeta + (size_t)row * a.H + h, p);
            }
            float pg = 0.f;
#pragma unroll
            for (int i = 0; i < kCols; ++i) {
                const float dm = -bt * x_s[i];
                const float sp = gr * S[i];   // S'_s
                pk = fmaf(sp, dm, pk);
                const float dsp = fmaf(kr, dm, dS[i]);
                pg = fmaf(dsp, S[i], pg);
                dS[i] = gr * dsp;
            }
            {   // this row's sums over the slice's columns
                const size_t e = ((size_t)row * a.H + h) * kD + r;
                atomicAdd(a.dq + e, pq);
                atomicAdd(a.dk + e, pk);
                atomicAdd(a.dlog_g + e, gr * pg);
            }
        }
    }
    if (a.dh0) {
#pragma unroll
        for (int i = 0; i < kCols; ++i) a.dh0[(size_t)chain * mat + my + i] = dS[i];
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
    if (chains * kSlices > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
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
    a.err = p.err;
    const unsigned grid = (unsigned)(chains * kSlices);
    if (p.bf16)
        bwd_kernel<__nv_bfloat16><<<grid, kThreads, 0, stream>>>(a);
    else
        bwd_kernel<float><<<grid, kThreads, 0, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace kda
