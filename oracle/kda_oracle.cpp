// KDA gated delta-rule oracle: plain float64 CPU implementation of the per-token recurrence.
//
// TEST INFRASTRUCTURE ONLY. This file is the independent checker for the GPU library. Only the
// test suite, the smoke check and the benchmark's CPU-baseline leg may load it. It shares no
// code, header, table or helper with the CUDA path, and the product never calls it.
//
// What it computes (GLM-5.3-Flash model card, the Kimi Delta Attention snippet of
// Glm5NextTextLinearAttention; NeMo AutoModel glm5_next layers page, `_torch_recurrent_kda`):
// for every (sequence, head) the state S is a dk x dv matrix, and for each token t in order
//
//     S      <- diag(g_t) S            (the snippet scales the state by the gate, key axis)
//     m      <- k_t^T S                (the snippet reads the state through k, summing keys)
//     delta  <- beta_t (v_t - m)       (the snippet's error term: value minus read, times beta)
//     S      <- S + k_t delta^T        (the snippet's rank-one write of k and delta)
//     o_t    <- S^T q_t                (read-out after the write, no 1/sqrt(dk) scale)
//
// with g_t = exp(log_g_t) per key channel. Packed variable-length input (cu_seqlens) restarts
// the state at every document boundary (the NeMo `_torch_recurrent_kda` docstring: the state
// resets at packed boundaries). The state starts from h0 (or zero) and the final state of each
// sequence or document is returned.
//
// All arithmetic is float64; exp is std::exp. Inputs arrive as float32 arrays that hold exactly
// the values the GPU sees (bf16 and fp32 values are both exactly representable in fp32).
// Parallelism: OpenMP over independent (sequence, head) pairs, nothing else.
//
// Pins (tests/test_oracle_pins.py): a brute-force unrolled matrix-product evaluation on T <= 8,
// the beta = 0 closed form, exact recall under orthonormal keys, linearity, column permutation,
// document separation, and a hand-worked example under tests/golden/.

#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>
#ifdef _OPENMP
#include <omp.h>
#endif

// Planted mistakes for the pin tests (tests/test_oracle_mutants.py builds one library per value).
// The default build defines none of them and compiles the recurrence exactly as stated above.
#ifndef KDA_ORACLE_MUTANT
#define KDA_ORACLE_MUTANT 0
#endif

namespace {

// One (sequence, head) chain over tokens [t0, t1) of a token-major [rows, H, d] layout (rows is
// B * T for a batch, the packed length for cu_seqlens, N for a decode batch).
void run_chain(int dk, int dv, int64_t t0, int64_t t1, int h, int H,
               const float* q, const float* k, const float* v, const float* log_g,
               const float* beta, const float* s_in, double* o, double* s_out) {
    std::vector<double> S((size_t)dk * dv, 0.0), m(dv), g(dk), kk(dk), qq(dk);
#if KDA_ORACLE_MUTANT == 7  // ignores the initial state
    s_in = nullptr;
#endif
    if (s_in)
        for (size_t i = 0; i < S.size(); ++i) S[i] = (double)s_in[i];
    for (int64_t t = t0; t < t1; ++t) {
        const int64_t qk_off = (t * H + h) * (int64_t)dk;
        const int64_t v_off = (t * H + h) * (int64_t)dv;
        const double b = (double)beta[t * H + h];
        for (int c = 0; c < dk; ++c) {
#if KDA_ORACLE_MUTANT == 6  // sign error in the gate
            g[c] = std::exp(-(double)log_g[qk_off + c]);
#else
            g[c] = std::exp((double)log_g[qk_off + c]);
#endif
            kk[c] = (double)k[qk_off + c];
            qq[c] = (double)q[qk_off + c];
        }
        // decay rows (key axis)
        for (int c = 0; c < dk; ++c)
            for (int j = 0; j < dv; ++j)
#if KDA_ORACLE_MUTANT == 1  // decays the value axis instead
                S[(size_t)c * dv + j] *= g[j % dk];
#else
                S[(size_t)c * dv + j] *= g[c];
#endif
#if KDA_ORACLE_MUTANT == 2  // reads out before the write
        for (int j = 0; j < dv; ++j) {
            double acc = 0.0;
            for (int c = 0; c < dk; ++c) acc += qq[c] * S[(size_t)c * dv + j];
            o[v_off + j] = acc;
        }
#endif
        // m = k^T S
        for (int j = 0; j < dv; ++j) m[j] = 0.0;
        for (int c = 0; c < dk; ++c)
            for (int j = 0; j < dv; ++j) m[j] += kk[c] * S[(size_t)c * dv + j];
        // delta = beta (v - m);  S += k delta^T
#if KDA_ORACLE_MUTANT == 3  // drops beta
        for (int j = 0; j < dv; ++j) m[j] = ((double)v[v_off + j] - m[j]);
#else
        for (int j = 0; j < dv; ++j) m[j] = b * ((double)v[v_off + j] - m[j]);
#endif
        for (int c = 0; c < dk; ++c)
            for (int j = 0; j < dv; ++j)
#if KDA_ORACLE_MUTANT == 4  // writes with k and delta swapped between the axes
                S[(size_t)c * dv + j] += kk[j % dk] * m[c % dv];
#else
                S[(size_t)c * dv + j] += kk[c] * m[j];
#endif
#if KDA_ORACLE_MUTANT != 2
        // o = S^T q
        for (int j = 0; j < dv; ++j) {
            double acc = 0.0;
            for (int c = 0; c < dk; ++c) acc += qq[c] * S[(size_t)c * dv + j];
            o[v_off + j] = acc;
        }
#endif
    }
    if (s_out)
        for (size_t i = 0; i < S.size(); ++i) s_out[i] = S[i];
}

}  // namespace

extern "C" {

// Prefill over a [B, T, H, *] batch, or over one packed row (B == 1) split by cu_seqlens.
//   q, k, log_g : [B, T, H, dk] float32      v : [B, T, H, dv] float32    beta : [B, T, H]
//   h0          : [N, H, dk, dv] float32 or NULL (zero state), N = B or len(cu_seqlens) - 1
//   cu_seqlens  : int32 [N + 1] offsets into the packed token axis, or NULL
//   o           : [B, T, H, dv] float64 (written)      hT : [N, H, dk, dv] float64 or NULL
// Returns 0 on success, 1 on malformed arguments.
int kda_oracle_fwd(int B, int T, int H, int dk, int dv, const float* q, const float* k,
                   const float* v, const float* log_g, const float* beta, const float* h0,
                   const int32_t* cu_seqlens, int num_seqs, double* o, double* hT,
                   int num_threads) {
    if (B < 1 || T < 0 || H < 1 || dk < 1 || dv < 1) return 1;
    if (cu_seqlens) {
        if (B != 1 || num_seqs < 1 || cu_seqlens[0] != 0 || cu_seqlens[num_seqs] != T) return 1;
        for (int n = 0; n < num_seqs; ++n)
            if (cu_seqlens[n + 1] < cu_seqlens[n]) return 1;
    } else if (num_seqs != B) {
        return 1;
    }
#ifdef _OPENMP
    if (num_threads > 0) omp_set_num_threads(num_threads);
#else
    (void)num_threads;
#endif
    const int64_t units = (int64_t)num_seqs * H;
    const size_t state = (size_t)dk * dv;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t u = 0; u < units; ++u) {
        const int n = (int)(u / H), h = (int)(u % H);
        int64_t t0, t1;
        if (cu_seqlens) {
#if KDA_ORACLE_MUTANT == 5  // carries the state across document boundaries
            t0 = 0;
#else
            t0 = cu_seqlens[n];
#endif
            t1 = cu_seqlens[n + 1];
        } else {
            t0 = (int64_t)n * T;
            t1 = t0 + T;
        }
        run_chain(dk, dv, t0, t1, h, H, q, k, v, log_g, beta,
                  h0 ? h0 + ((size_t)n * H + h) * state : nullptr, o,
                  hT ? hT + ((size_t)n * H + h) * state : nullptr);
    }
    return 0;
}

// One decode token for N independent sequences. The state is read from S_in and the updated
// state written to S_out (both [N, H, dk, dv]); o is [N, H, dv]. Same recurrence as above with
// T = 1 (Rust engine page, KDA decode with a per-sequence KdaSeqState).
int kda_oracle_decode(int N, int H, int dk, int dv, const float* q, const float* k,
                      const float* v, const float* log_g, const float* beta, const float* S_in,
                      double* S_out, double* o, int num_threads) {
    if (N < 1 || H < 1 || dk < 1 || dv < 1 || !S_in || !S_out) return 1;
#ifdef _OPENMP
    if (num_threads > 0) omp_set_num_threads(num_threads);
#else
    (void)num_threads;
#endif
    const int64_t units = (int64_t)N * H;
    const size_t state = (size_t)dk * dv;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t u = 0; u < units; ++u) {
        const int n = (int)(u / H), h = (int)(u % H);
        // A decode batch is N sequences of length one: token index n in a [N, 1, H, d] layout.
        run_chain(dk, dv, n, n + 1, h, H, q, k, v, log_g, beta, S_in + u * state, o,
                  S_out + u * state);
    }
    return 0;
}

int kda_oracle_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

}  // extern "C"
