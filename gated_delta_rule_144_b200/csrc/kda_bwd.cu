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
// The backward needs S_{t-1} at every token in reverse order. One CTA per chain first runs the
// forward and stores the state at the start of every 64-token chunk (checkpoints, in the
// workspace); then, chunk by chunk from the last, it re-runs the chunk's forward from its
// checkpoint, keeping the chunk's states and m_t, d_t in the workspace, and walks the chunk
// backwards.
//
// Threads: 512 per chain; thread (r, q) owns row r of S and of dS, columns 32 q .. 32 q + 31.
// Sums over columns (dq, dk, dlog_g) are two shuffles among the four threads of a row; sums over
// rows (m, dd) are a reduce-scatter over the 8 rows of a warp (each lane keeps 4 columns) and a
// sum over the 16 warps in shared memory. The kernel's own copies of the state (checkpoints, the
// chunk's per-token states) interleave the threads' elements, so that every warp access to them
// is one contiguous 128-byte line (a thread's 32 consecutive floats would touch 32 lines per warp
// instruction: measured 14 K of a token's 26 K cycles); the staged per-column vectors are padded
// so that the four column groups of a warp read different banks; the next token's inputs are
// fetched into registers a step ahead. Plain fp32 arithmetic and expf, no tensor cores: this
// kernel is the correct first version of the training direction, not yet its fast one.

#include <cstdint>

#include "kda_bwd.cuh"

namespace kda {
namespace {

constexpr int kD = 128;
constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kCk = 64;   // tokens per checkpointed chunk
constexpr int kDp = kD + kD / 32;   // padded per-column vectors: entry c at c + c / 32

// Entry c of a per-column vector in shared memory. Thread (r, q) reads entries 32 q + i of its
// column group; one word of padding per 32 puts the four groups of a warp in different banks.
__device__ __forceinline__ int pc(int c) { return c + (c >> 5); }

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
    float* dq;
    float* dk;
    float* dv;
    float* dlog_g;
    float* dbeta;
    float* dh0;          // nullable
    float* ckpt;         // [chains][nck][128][128]
    float* chunk_s;      // [chains][kCk][128][128]
    float* chunk_md;     // [chains][kCk][2][128]
    int T, H, N, nck;
    unsigned* err;
};

template <typename E>
__global__ void __launch_bounds__(kThreads, 1) bwd_kernel(const BwdArgs a) {
    __shared__ float q_s[kD], k_s[kD], g_s[kD], v_s[kD], do_s[kDp], m_s[kDp], d_s[kDp], x_s[kDp];
    __shared__ float part[kWarps * kD];
    __shared__ float beta_s, db_s[4];

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int r = tid >> 2, qq = tid & 3;   // row of S, column group
    const int c0 = 32 * qq;
    const int chain = blockIdx.x;
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
    float* ckpt = a.ckpt + (size_t)chain * a.nck * mat;
    float* cs = a.chunk_s + (size_t)chain * kCk * mat;
    float* cmd = a.chunk_md + (size_t)chain * kCk * 2 * kD;
    const size_t my = (size_t)r * kD + c0;   // this thread's 32 elements in a 128 x 128 matrix
    // the same 32 elements in the kernel's own copies (checkpoints, the chunk's states): element i
    // of every thread side by side, so that a warp's access is 128 contiguous bytes
    auto ti = [&](int i) { return (size_t)i * kThreads + tid; };

    // Inputs of token row `row` into shared memory (threads < 128, one channel each). The next
    // row staged (forward, re-run and backward walks included) is fetched into registers right
    // after, so its loads are in flight during this step; a row that was not fetched ahead is
    // loaded on the spot.
    float nk = 0.f, nlg = 0.f, nv = 0.f, nq = 0.f, ndo = 0.f, nb = 0.f;
    long long n_row = -1;
    bool n_bwd = false;
    auto fetch = [&](long long row, bool backward) {
        if (tid < kD) {
            const size_t e = ((size_t)row * a.H + h) * kD + tid;
            nk = load_elem(k, e);
            nlg = a.log_g[e];
            nv = load_elem(v, e);
            if (backward) {
                nq = load_elem(q, e);
                ndo = load_elem(dout, e);
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
            v_s[tid] = nv;
            if (backward) {
                q_s[tid] = nq;
                do_s[pc(tid)] = ndo;
            }
            if (tid == 0) beta_s = nb;
        }
        __syncthreads();
        if (next_row >= 0) fetch(next_row, next_bwd);
        else n_row = -1;
    };
    // out[c] = sum over rows of f(i) (i: this thread's column 32 qq + i); the result lands in
    // shared memory for every thread after the call
    auto colsum = [&](auto f, float* out) {
        float s16[16], s8[8], s4[4];
        const bool b4 = lane & 16, b3 = lane & 8, b2 = lane & 4;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const float lo = f(i), hi = f(16 + i);
            s16[i] = (b4 ? hi : lo) + __shfl_xor_sync(0xffffffffu, b4 ? lo : hi, 16);
        }
#pragma unroll
        for (int i = 0; i < 8; ++i)
            s8[i] = (b3 ? s16[8 + i] : s16[i]) +
                    __shfl_xor_sync(0xffffffffu, b3 ? s16[i] : s16[8 + i], 8);
#pragma unroll
        for (int i = 0; i < 4; ++i)
            s4[i] = (b2 ? s8[4 + i] : s8[i]) +
                    __shfl_xor_sync(0xffffffffu, b2 ? s8[i] : s8[4 + i], 4);
        const int base = c0 + (b4 ? 16 : 0) + (b3 ? 8 : 0) + (b2 ? 4 : 0);
#pragma unroll
        for (int i = 0; i < 4; ++i) part[warp * kD + base + i] = s4[i];
        __syncthreads();
        if (tid < kD) {
            float s = 0.f;
#pragma unroll 4
            for (int w = 0; w < kWarps; ++w) s += part[w * kD + tid];
            out[pc(tid)] = s;
        }
        __syncthreads();
    };
    // sum over this row's four threads
    auto rowsum = [&](float x) {
        x += __shfl_xor_sync(0xffffffffu, x, 1);
        x += __shfl_xor_sync(0xffffffffu, x, 2);
        return x;
    };

    float S[32], dS[32];
    // forward step on the staged token: S <- S' + k d^T; m and d land in m_s, d_s
    auto forward_step = [&]() {
        const float gr = g_s[r], kr = k_s[r];
#pragma unroll
        for (int i = 0; i < 32; ++i) S[i] *= gr;
        colsum([&](int i) { return kr * S[i]; }, m_s);
        if (tid < kD) d_s[pc(tid)] = beta_s * (v_s[tid] - m_s[pc(tid)]);
        __syncthreads();
#pragma unroll
        for (int i = 0; i < 32; ++i) S[i] += kr * d_s[pc(c0 + i)];
    };

    // ---------------------------------------------------------------- forward, checkpoints
#pragma unroll
    for (int i = 0; i < 32; ++i) S[i] = a.h0 ? a.h0[(size_t)chain * mat + my + i] : 0.f;
    for (long long s = 0; s < L; ++s) {
        if (s % kCk == 0) {
#pragma unroll
            for (int i = 0; i < 32; ++i) ckpt[(size_t)(s / kCk) * mat + ti(i)] = S[i];
        }
        // next: the token after, or the first token of the last chunk's re-run
        stage(t0 + s, false, s + 1 < L ? t0 + s + 1 : t0 + (long long)(nck - 1) * kCk, false);
        forward_step();
    }

    // ---------------------------------------------------------------- backward, chunk by chunk
#pragma unroll
    for (int i = 0; i < 32; ++i) dS[i] = a.dhT ? a.dhT[(size_t)chain * mat + my + i] : 0.f;
    for (int ci = nck - 1; ci >= 0; --ci) {
        const long long s0 = (long long)ci * kCk;
        const long long s1 = min(L, s0 + kCk);
        // the chunk's forward again, keeping S_{s-1}, m_s and d_s of every token
#pragma unroll
        for (int i = 0; i < 32; ++i) S[i] = ckpt[(size_t)ci * mat + ti(i)];
        for (long long s = s0; s < s1; ++s) {
            const size_t j = (size_t)(s - s0);
#pragma unroll
            for (int i = 0; i < 32; ++i) cs[j * mat + ti(i)] = S[i];
            // next: the token after, or the chunk's last token for the backward walk
            if (s + 1 < s1) stage(t0 + s, false, t0 + s + 1, false);
            else stage(t0 + s, false, t0 + s1 - 1, true);
            forward_step();
            if (tid < kD) {
                cmd[j * 2 * kD + tid] = m_s[pc(tid)];
                cmd[j * 2 * kD + kD + tid] = d_s[pc(tid)];
            }
        }
        // the chunk's tokens from the last to the first
        for (long long s = s1 - 1; s >= s0; --s) {
            const size_t j = (size_t)(s - s0);
            const long long row = t0 + s;
            // next: the token before, or the first token of the previous chunk's re-run
            if (s > s0) stage(row, true, row - 1, true);
            else stage(row, true, ci > 0 ? t0 + (long long)(ci - 1) * kCk : -1, false);
            if (tid < kD) {   // written by this same thread in the pass above
                m_s[pc(tid)] = cmd[j * 2 * kD + tid];
                d_s[pc(tid)] = cmd[j * 2 * kD + kD + tid];
            }
#pragma unroll
            for (int i = 0; i < 32; ++i) S[i] = cs[j * mat + ti(i)];   // S_{s-1}
            __syncthreads();
            const float gr = g_s[r], kr = k_s[r], qr = q_s[r];
            float pq = 0.f, pk = 0.f;
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                const float dl = d_s[pc(c0 + i)], dov = do_s[pc(c0 + i)];
                const float st = gr * S[i] + kr * dl;   // S_s
                pq = fmaf(st, dov, pq);
                dS[i] = fmaf(qr, dov, dS[i]);
                pk = fmaf(dS[i], dl, pk);
            }
            colsum([&](int i) { return kr * dS[i]; }, x_s);   // dd
            const float bt = beta_s;
            if (tid < kD) {
                const float dd = x_s[pc(tid)];
                a.dv[((size_t)row * a.H + h) * kD + tid] = bt * dd;
                float p = dd * (v_s[tid] - m_s[pc(tid)]);
#pragma unroll
                for (int off = 16; off >= 1; off >>= 1) p += __shfl_xor_sync(0xffffffffu, p, off);
                if (lane == 0) db_s[warp] = p;
            }
            __syncthreads();
            if (tid == 0) a.dbeta[(size_t)row * a.H + h] = (db_s[0] + db_s[1]) + (db_s[2] + db_s[3]);
            float pg = 0.f;
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                const float dm = -bt * x_s[pc(c0 + i)];
                const float sp = gr * S[i];   // S'_s
                pk = fmaf(sp, dm, pk);
                const float dsp = fmaf(kr, dm, dS[i]);
                pg = fmaf(dsp, S[i], pg);
                dS[i] = gr * dsp;
            }
            pq = rowsum(pq);
            pk = rowsum(pk);
            pg = rowsum(pg);
            if (qq == 0) {
                const size_t e = ((size_t)row * a.H + h) * kD + r;
                a.dq[e] = pq;
                a.dk[e] = pk;
                a.dlog_g[e] = gr * pg;
            }
        }
    }
    if (a.dh0) {
#pragma unroll
        for (int i = 0; i < 32; ++i) a.dh0[(size_t)chain * mat + my + i] = dS[i];
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
    if (chains > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
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
    if (p.bf16)
        bwd_kernel<__nv_bfloat16><<<(unsigned)chains, kThreads, 0, stream>>>(a);
    else
        bwd_kernel<float><<<(unsigned)chains, kThreads, 0, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace kda
