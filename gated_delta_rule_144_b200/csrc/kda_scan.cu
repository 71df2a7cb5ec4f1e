// State pass of the split chunked prefill: the only part of the chunked form that is sequential
// over chunks.
//
// The intra-chunk kernel (intra_kernel, kda_intra.cu) has already written, for every chunk
// of 64 tokens and every head, the chunk's WY factors to the workspace:
//   [W; Q+] (128 x 128 bf16), K_end (64 x 128 bf16), U~^T (128 value columns x 64 tokens, bf16),
//   A_qk (64 x 64 bf16) and the chunk's total decay e^{Gamma_end} (128 fp32).
// Per (sequence or document, head) this kernel then walks the chunks in order (the WY form of the
// gated delta rule; GLM-5.3-Flash model card, Kimi Delta Attention snippet, and the state-passing
// identity it implies):
//   U = U~ - W S,   o = Q+ S + A_qk U,   S <- diag(e^{Gamma_end}) S + K_end^T U.
//
// Layout: the state is kept transposed, S^T [value column j][key channel c], in TMEM lane j, so
// every product takes its state-side operand from TMEM and no shared-memory write sits on the
// critical path:
//   D = S^T [W; Q+]^T     (A = bf16 copy of S^T in TMEM, B = [W; Q+] K-major in shared memory)
//   S^T += U^T K_end      (A = bf16 U^T in TMEM, B = K_end MN-major in shared memory)
//   o^T = (Q+ S)^T + U^T A_qk^T   (accumulated into D's second half; A = U^T, B = A_qk K-major)
// Eight data warps: warps w and w + 4 share TMEM lane quarter w mod 4 (lane j = value column j)
// and split the columns of every TMEM row between them. A ninth warp only issues the MMAs, so that
// no MMA issue waits behind a data warp's work. Per chunk c the critical chain is
//   bf16(S^T) -> D (8 K steps) -> U^T -> S^T += U^T K_end (4 K steps);
// the o product follows the update in the tensor pipe, off the chain. The decay of S^T, the load of
// U~^T and the output of chunk c-1 (read from the other of two D buffers, staged in shared memory
// and written by a TMA store) run while the D product of chunk c is in flight. The MMA-issuing
// thread also issues the TMA loads, while the D product runs (two stages: chunk c+1 arrives while
// chunk c runs), and lane 0 of warp 2 the output stores. Every mbarrier wait is bounded; on expiry the CTA records KDA_ERR_TIMEOUT, drains
// its own copies and MMAs, frees TMEM and exits.

#include <cuda.h>
#include <cudaTypedefs.h>

#include <cstdlib>
#include <cstring>
#include <mutex>

#include "kda_internal.cuh"
#include "kda_sm100.cuh"
#include "kda_tma.cuh"

namespace kda {
namespace {

using namespace sm100;

constexpr int kC = 64;
constexpr int kD = 128;
constexpr int kDataWarps = 8;
constexpr int kThreads = 32 * kDataWarps + 32;   // + one warp that only issues MMAs

// one pipeline stage (bytes from a 1024-aligned stage base)
constexpr uint32_t ST_WQ = 0;        // [W; Q~] 128 x 128 bf16, K-major SW128: 2 panels of 16 KB
constexpr uint32_t ST_KE = 32768;    // K_end 64 x 128 bf16, MN-major SW128: 2 panels of 8 KB
constexpr uint32_t ST_UT = 49152;    // U~^T [128 j][64 tokens] bf16, SW128
constexpr uint32_t ST_AQ = 65536;    // A_qk [64 r][64 i] bf16, K-major SW128
constexpr uint32_t ST_DEC = 73728;   // e^{Gamma_end} [128] f32
constexpr uint32_t kStage = 74752;   // 73 KB, a multiple of 1024
constexpr uint32_t kTxStage = 32768 + 2 * 16384 + 8192 + 512;
constexpr uint32_t OFF_O = 2 * kStage;       // two output tiles o [64 tokens][128] bf16
constexpr uint32_t OFF_BAR = OFF_O + 32768;  // full[2], mma1, mma2, never, mma3
constexpr uint32_t OFF_TMEM = OFF_BAR + 64;
constexpr uint32_t kSmemBytes = OFF_TMEM + 16 + 1024;
static_assert(kSmemBytes <= 232448, "shared memory budget");

// TMEM columns (128 lanes = value columns)
constexpr uint32_t TS = 0;     // S^T fp32 [128 x 128]
constexpr uint32_t TB = 128;   // bf16 S^T, A operand: 64 columns
constexpr uint32_t TU = 192;   // bf16 U^T, A operand: 32 columns
constexpr uint32_t TD = 256;   // two buffers of S^T [W; Q+]^T fp32 (128 columns each):
                               //   columns 0-63 (W S)^T, 64-127 (Q+ S)^T, then o^T
constexpr uint32_t kTmemCols = 512;

struct ScanArgs {
    const int32_t* order;   // nullable: document taken by the k-th (document, head) group
    const int32_t* cu;      // nullable
    const float* h0;        // state at chunk c_begin (nullable: zero)
    float* hT;              // state after chunk c_end - 1 (nullable: not written)
    int c_begin, c_end;     // chunks of every chain this launch walks
    __nv_bfloat16* o;
    const float* decay;     // [R][128]
    int T, H, N, ncT;       // ncT: chunk records per sequence when cu is null
    long long G;            // chunk records per head
    long long budget;
    int debug_stall;
    unsigned* err;
};

struct ScanMaps {
    CUtensorMap wq, ke, ut, aq, o;
};

__device__ __forceinline__ uint32_t pack2(float x, float y) {
    __nv_bfloat162 v = __floats2bfloat162_rn(x, y);
    return *reinterpret_cast<uint32_t*>(&v);
}
__device__ __forceinline__ float lo_bf(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float hi_bf(uint32_t u) { return __uint_as_float(u & 0xffff0000u); }

__global__ void __launch_bounds__(kThreads, 1)
chunk_scan_kernel(const __grid_constant__ ScanMaps maps, const ScanArgs args) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
    const uint32_t sb = smem_u32(sm);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int qd = warp & 3, hs = warp >> 2;   // TMEM lane quarter, column half
    const int j = 32 * qd + lane;              // value column = TMEM lane
    constexpr int kStorer = 64;                // thread that issues the output stores
    constexpr int kMma = 32 * kDataWarps;      // thread that issues the MMAs and the TMA loads
    const bool data = warp < kDataWarps;
    const int unit = blockIdx.x;
    const int h = unit % args.H;
    const int n = args.order ? args.order[unit / args.H] : unit / args.H;

    long long t0, t1, g0;
    if (args.cu) {
        t0 = args.cu[n];
        t1 = args.cu[n + 1];
        const bool bad_ends = (n == 0 && t0 != 0) || (n == args.N - 1 && t1 != args.T);
        if (t1 < t0 || t0 < 0 || t1 > args.T || bad_ends) {
            if (tid == 0) set_device_error(args.err, DEV_BAD_SEQLENS);
            return;
        }
        g0 = t0 / kC + n;
    } else {
        t0 = (long long)n * args.T;
        t1 = t0 + args.T;
        g0 = (long long)n * args.ncT;
    }
    if (g0 + (t1 - t0 + kC - 1) / kC > args.G) {   // only a malformed cu_seqlens gets here
        if (tid == 0) set_device_error(args.err, DEV_BAD_SEQLENS);
        return;
    }
    {   // this launch's segment of the chain: chunks [c_begin, c_end), possibly empty
        const long long sb0 = min(t1, t0 + (long long)kC * args.c_begin);
        const long long sb1 = min(t1, t0 + (long long)kC * args.c_end);
        g0 += (sb0 - t0 + kC - 1) / kC;
        t0 = sb0;
        t1 = max(sb0, sb1);
    }
    const int nchunks = (int)((t1 - t0 + kC - 1) / kC);

    uint32_t* tmem_s = reinterpret_cast<uint32_t*>(sm + OFF_TMEM);
    const uint32_t bar_full0 = sb + OFF_BAR, bar_mma1 = bar_full0 + 16, bar_mma2 = bar_full0 + 24;
    const uint32_t bar_never = bar_full0 + 32, bar_mma3 = bar_full0 + 40;
    if (tid == 0) {
        mbar_init(bar_full0, 1);
        mbar_init(bar_full0 + 8, 1);
        mbar_init(bar_mma1, 1);
        mbar_init(bar_mma2, 1);
        mbar_init(bar_never, 1);
        mbar_init(bar_mma3, 1);
        fence_mbar_init();
        prefetch_tmap(&maps.wq);
        prefetch_tmap(&maps.ke);
        prefetch_tmap(&maps.ut);
        prefetch_tmap(&maps.aq);
        prefetch_tmap(&maps.o);
    }
    if (warp == 0) {
        tmem_alloc(smem_u32(tmem_s), kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_s;
    const uint32_t lq = (uint32_t)(32 * qd) << 16;   // this warp's TMEM lane quarter
    const size_t state_base = ((size_t)n * args.H + h) * kD * kD;

    // initial state, transposed: lane j, column c holds S[c][j]; this thread: c in [64 hs, +64)
#pragma unroll 1
    for (int p = 0; p < (data ? 2 : 0); ++p) {
        float v[32];
        const int c0 = 64 * hs + 32 * p;
#pragma unroll
        for (int i = 0; i < 32; ++i)
            v[i] = args.h0 ? args.h0[state_base + (size_t)(c0 + i) * kD + j] : 0.f;
        tmem_st32(tbase + lq + TS + c0, v);
    }
    tmem_st_wait();

    auto issue = [&](int c) {
        const uint32_t st = sb + (uint32_t)(c & 1) * kStage;
        const uint32_t bar = bar_full0 + 8 * (c & 1);
        const long long rec = (g0 + c) * args.H + h;
        mbar_arrive_expect_tx(bar, kTxStage);
        tma_load_2d(st + ST_WQ, &maps.wq, bar, 0, (int)(rec * 128));
        tma_load_2d(st + ST_WQ + 16384, &maps.wq, bar, 64, (int)(rec * 128));
        tma_load_2d(st + ST_KE, &maps.ke, bar, 0, (int)(rec * 64));
        tma_load_2d(st + ST_KE + 8192, &maps.ke, bar, 64, (int)(rec * 64));
        tma_load_2d(st + ST_UT, &maps.ut, bar, 0, (int)(rec * 128));
        tma_load_2d(st + ST_AQ, &maps.aq, bar, 0, (int)(rec * 64));
        bulk_load(st + ST_DEC, args.decay + rec * kD, 512, bar);
    };

    const uint64_t dK = sw128_desc(0, 16, 1024);     // K-major, 128B swizzle
    const uint64_t dM8 = sw128_desc(0, 8192, 1024);  // MN-major, 64-row panels
    const uint32_t id1 = idesc_bf16(128, 128, 0, 0);
    const uint32_t id2 = idesc_bf16(128, 128, 0, 1);
    const uint32_t id3 = idesc_bf16(128, 64, 0, 0);

    // outstanding asynchronous work, drained before exit if a wait expires
    int issued = 0;          // chunks whose copies were issued
    int landed = 0;          // chunks whose copies were waited for
    bool mma1_pending = false, mma2_pending = false, mma3_pending = false;
    int mma1_chunk = 0, mma2_chunk = 0, mma3_chunk = 0;   // chunk of the last commit (parity)
    bool aborted = false;
    // One thread polls; the rest of the CTA waits at the barrier that publishes the outcome (and
    // any failure a thread has recorded in `also_bad` since the last barrier).
    auto wait_all = [&](uint32_t bar, uint32_t parity, bool also_bad = false) -> bool {
        const bool ok = tid != 0 || mbar_wait(bar, parity, args.budget);
        return __syncthreads_or(!ok || also_bad) == 0;
    };

    // o of chunk cc (rows < L): o^T = (Q+ S)^T + U^T A_qk^T from D buffer cc & 1 (this thread's
    // 32 tokens), staged row-major in output tile cc & 1. Waits (every data thread, bounded) for
    // the o product of chunk cc; returns false if that wait expired.
    auto stage_o = [&](int cc) -> bool {
        const bool ok = mbar_wait(bar_mma3, (uint32_t)(cc & 1), args.budget);
        tc_fence_after();
        float w[32];
        tmem_ld32(tbase + lq + TD + 128 * (cc & 1) + 64 + 32 * hs, w);
        tmem_ld_wait();
        __nv_bfloat16* tile = reinterpret_cast<__nv_bfloat16*>(sm + OFF_O + 16384 * (cc & 1));
#pragma unroll
        for (int i = 0; i < 32; ++i) tile[(32 * hs + i) * kD + j] = __float2bfloat16_rn(w[i]);
        return ok;
    };
    // write staged tile cc to o: one TMA store for a full chunk, row copies for a partial one
    // (a TMA box would run into the next document's rows). Call after a CTA barrier that
    // follows fence_proxy_async by the writers.
    auto flush_o = [&](int cc) {
        const long long r0 = t0 + (long long)kC * cc;
        const int L = (int)min((long long)kC, t1 - r0);
        if (L == kC) {
            if (tid == kStorer) {
                tma_store_3d(&maps.o, sb + OFF_O + 16384 * (cc & 1), 0, h, (int)r0);
                bulk_commit();
            }
        } else {
            const uint4* src = reinterpret_cast<const uint4*>(sm + OFF_O + 16384 * (cc & 1));
            for (int i = tid; i < L * 16; i += kThreads) {
                const int r = i >> 4, q = i & 15;
                *reinterpret_cast<uint4*>(args.o + ((size_t)(r0 + r) * args.H + h) * kD + 8 * q) =
                    src[r * 16 + q];
            }
        }
    };

    if (tid == kMma) {
        if (nchunks > 0) issue(0);
        if (nchunks > 1) issue(1);
    }
    issued = min(nchunks, 2);
    if (args.debug_stall && !wait_all(bar_never, 0)) aborted = true;

    for (int c = 0; c < nchunks && !aborted; ++c) {
        const uint32_t st = sb + (uint32_t)(c & 1) * kStage;
        const uint8_t* stp = sm + (size_t)(c & 1) * kStage;

        if (!wait_all(bar_full0 + 8 * (c & 1), (uint32_t)((c >> 1) & 1))) { aborted = true; break; }
        landed = c + 1;
        if (mma2_pending) {   // S of chunk c is complete once the previous update has landed
            if (!wait_all(bar_mma2, (uint32_t)(mma2_chunk & 1))) { aborted = true; break; }
            mma2_pending = false;
        }
        tc_fence_after();

        // ---------------------------------------------------------------- bf16 S^T -> TB
        float va[32], vb[32];
        if (data) {
            tmem_ld32(tbase + lq + TS + 64 * hs, va);
            tmem_ld32(tbase + lq + TS + 64 * hs + 32, vb);
            tmem_ld_wait();
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) pk[i] = pack2(va[2 * i], va[2 * i + 1]);
            tmem_st16u(tbase + lq + TB + 32 * hs, pk);
#pragma unroll
            for (int i = 0; i < 16; ++i) pk[i] = pack2(vb[2 * i], vb[2 * i + 1]);
            tmem_st16u(tbase + lq + TB + 32 * hs + 16, pk);
            tmem_st_wait();
        }
        // output tile (c-1)&1 is rewritten below; its previous store (chunk c-3) must be done
        if (tid == kStorer && c >= 3) bulk_wait_read_le1();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();

        // ---------------------------------------------------------------- D = S^T [W; Q+]^T
        bool o_bad = false;
        if (tid == kMma) {
            tc_fence_after();
#pragma unroll
            for (int s = 0; s < kD / 16; ++s)
                umma_f16_ts(tbase + TD + 128 * (c & 1), tbase + TB + 8 * s,
                            desc_at(dK, st + ST_WQ + (s >> 2) * 16384 + (s & 3) * 32), id1, s > 0);
            umma_commit(bar_mma1);
            // Stage (c+1)&1 held chunk c-1, read by its update (waited for at this chunk's start)
            // and its o product: once that is done, fetch chunk c+1 into it. This thread issues
            // nothing else until the D product is waited for, so the copies (about 100 cycles to
            // issue each) cost the chain nothing.
            if (c >= 1 && c + 1 < nchunks) {
                if (mbar_wait(bar_mma3, (uint32_t)((c - 1) & 1), args.budget)) issue(c + 1);
                else o_bad = true;
            }
        }
        if (c >= 1 && c + 1 < nchunks) issued = c + 2;   // (an expired wait aborts below; the
                                                         //  drain's waits are bounded)
        mma1_pending = true;
        mma1_chunk = c;

        // ---------------------------------------------------------------- while D runs
        // decay: TS = S^T diag(e^{Gamma_end}) (the update accumulates into it)
        uint32_t ub[16];
        if (data) {
            const float* dec = reinterpret_cast<const float*>(stp + ST_DEC) + 64 * hs;
#pragma unroll
            for (int i = 0; i < 32; i += 4) {
                const float4 d0 = *reinterpret_cast<const float4*>(dec + i);
                const float4 d1 = *reinterpret_cast<const float4*>(dec + 32 + i);
                va[i] *= d0.x; va[i + 1] *= d0.y; va[i + 2] *= d0.z; va[i + 3] *= d0.w;
                vb[i] *= d1.x; vb[i + 1] *= d1.y; vb[i + 2] *= d1.z; vb[i + 3] *= d1.w;
            }
            tmem_st32(tbase + lq + TS + 64 * hs, va);
            tmem_st32(tbase + lq + TS + 64 * hs + 32, vb);
            // U~^T of this chunk: row j, tokens [32 hs, +32)
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const uint4 x = *reinterpret_cast<const uint4*>(
                    stp + ST_UT + sw128_off(128, j, 32 * hs + 8 * m));
                ub[4 * m] = x.x; ub[4 * m + 1] = x.y; ub[4 * m + 2] = x.z; ub[4 * m + 3] = x.w;
            }
            if (c >= 1) o_bad = !stage_o(c - 1);
            tmem_st_wait();
        }
        if (c >= 1) mma3_pending = false;   // (waited for above, or the CTA aborts below)

        if (!wait_all(bar_mma1, (uint32_t)(c & 1), o_bad)) { aborted = true; break; }
        mma1_pending = false;
        tc_fence_after();

        // ---------------------------------------------------------------- U^T = U~^T - (W S)^T
        if (data) {
            float w[32];
            tmem_ld32(tbase + lq + TD + 128 * (c & 1) + 32 * hs, w);
            tmem_ld_wait();
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
                pk[i] = pack2(lo_bf(ub[i]) - w[2 * i], hi_bf(ub[i]) - w[2 * i + 1]);
            tmem_st16u(tbase + lq + TU + 16 * hs, pk);
        }
        if (data) tmem_st_wait();
        fence_proxy_async();   // output tile c-1 -> TMA store
        tc_fence_before();
        __syncthreads();
        tc_fence_after();

        // ---------------------------------------------------------------- S^T += U^T K_end
        if (tid == kMma) {
            tc_fence_after();
#pragma unroll
            for (int s = 0; s < kC / 16; ++s)
                umma_f16_ts(tbase + TS, tbase + TU + 8 * s, desc_at(dM8, st + ST_KE + 2048 * s),
                            id2, 1);
            umma_commit(bar_mma2);
            // o^T = (Q+ S)^T + U^T A_qk^T, behind the update in the pipe (off the chain)
#pragma unroll
            for (int s = 0; s < kC / 16; ++s)
                umma_f16_ts(tbase + TD + 128 * (c & 1) + 64, tbase + TU + 8 * s,
                            desc_at(dK, st + ST_AQ + 32 * s), id3, 1);
            umma_commit(bar_mma3);
        }
        mma2_pending = mma3_pending = true;
        mma2_chunk = mma3_chunk = c;
        if (c >= 1) flush_o(c - 1);
    }

    if (aborted) {
        if (tid == 0) set_device_error(args.err, DEV_TIMEOUT);
        // wind down: this CTA's own copies and MMAs finish before TMEM and smem go away
        const long long drain = 1ll << 31;
        for (int c = landed; c < issued; ++c)
            mbar_wait(bar_full0 + 8 * (c & 1), (uint32_t)((c >> 1) & 1), drain);
        if (mma1_pending) mbar_wait(bar_mma1, (uint32_t)(mma1_chunk & 1), drain);
        if (mma2_pending) mbar_wait(bar_mma2, (uint32_t)(mma2_chunk & 1), drain);
        if (mma3_pending) mbar_wait(bar_mma3, (uint32_t)(mma3_chunk & 1), drain);
        __syncthreads();
    } else {
        if (mma2_pending && !wait_all(bar_mma2, (uint32_t)(mma2_chunk & 1))) {
            if (tid == 0) set_device_error(args.err, DEV_TIMEOUT);
            mbar_wait(bar_mma2, (uint32_t)(mma2_chunk & 1), 1ll << 31);
        }
        tc_fence_after();
        if (nchunks > 0) {   // output of the last chunk
            if (tid == kStorer && nchunks >= 3) bulk_wait_read_le1();
            __syncthreads();
            bool bad = false;
            if (data) bad = !stage_o(nchunks - 1);
            fence_proxy_async();
            if (__syncthreads_or(bad)) {
                if (tid == 0) set_device_error(args.err, DEV_TIMEOUT);
                mbar_wait(bar_mma3, (uint32_t)((nchunks - 1) & 1), 1ll << 31);
            } else {
                flush_o(nchunks - 1);
            }
        }
        if (args.hT && data) {
#pragma unroll 1
            for (int p = 0; p < 2; ++p) {
                float v[32];
                const int c0 = 64 * hs + 32 * p;
                tmem_ld32(tbase + lq + TS + c0, v);
                tmem_ld_wait();
#pragma unroll
                for (int i = 0; i < 32; ++i) args.hT[state_base + (size_t)(c0 + i) * kD + j] = v[i];
            }
        }
    }
    if (tid == kStorer) bulk_wait_all();   // output stores complete before the smem goes away
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tbase, kTmemCols);
}

long long scan_wait_budget() {
    static long long budget = [] {
        const char* s = std::getenv("KDA_DEBUG_WAIT_CYCLES");
        if (s && *s) {
            const long long v = std::atoll(s);
            if (v > 0) return v;
        }
        return 1ll << 31;   // about one second of SM clock
    }();
    return budget;
}

int scan_debug_stall() {
    static int v = [] {
        const char* s = std::getenv("KDA_DEBUG_STALL_WAIT");
        return (s && *s && *s != '0') ? 1 : 0;
    }();
    return v;
}

}  // namespace

// One CTA (4 warps) per (sequence or document, head); packed documents are taken longest first
// when an order is given.
cudaError_t launch_chunk_scan(const FwdParams& p, const ScanSegment& seg, cudaStream_t stream) {
    const SplitWorkspace& ws = *p.split;
    const long long units = (long long)p.N * p.H;
    if (units == 0) return cudaSuccess;
    if (units > 0x7fffffffLL || ws.G * p.H * 128 > 0x7fffffffLL)
        return cudaErrorInvalidConfiguration;
    const unsigned long long R = (unsigned long long)(ws.G * p.H);
    const auto BF = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    ScanMaps m;
    cudaError_t e;
    if ((e = make_map_2d(&m.wq, ws.wq, BF, 2, R * 128, kD, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B)) !=
            cudaSuccess ||
        (e = make_map_2d(&m.ke, ws.ke, BF, 2, R * 64, kD, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B)) !=
            cudaSuccess ||
        (e = make_map_2d(&m.ut, ws.ut, BF, 2, R * 128, kC, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B)) !=
            cudaSuccess ||
        (e = make_map_2d(&m.aq, ws.aq, BF, 2, R * 64, kC, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B)) !=
            cudaSuccess ||
        (e = make_map_3d_rows(&m.o, p.o, BF, 2, (unsigned long long)p.B * p.T, p.H, kD, kC)) !=
            cudaSuccess)
        return e;
    static PerDevice attr;
    const cudaError_t attr_err = attr.run([](int) {
        return cudaFuncSetAttribute(chunk_scan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    (int)kSmemBytes);
    });
    if (attr_err != cudaSuccess) return attr_err;
    ScanArgs a;
    memset(&a, 0, sizeof(a));
    a.order = p.doc_order;
    a.cu = p.cu_seqlens;
    a.h0 = seg.h0;
    a.hT = seg.hT;
    a.c_begin = seg.c_begin;
    a.c_end = seg.c_end;
    a.o = static_cast<__nv_bfloat16*>(p.o);
    a.decay = ws.decay;
    a.T = p.T;
    a.H = p.H;
    a.N = p.N;
    a.ncT = ws.ncT;
    a.G = ws.G;
    a.budget = scan_wait_budget();
    a.debug_stall = scan_debug_stall();
    a.err = p.err;
    chunk_scan_kernel<<<(unsigned)units, kThreads, kSmemBytes, stream>>>(m, a);
    return cudaGetLastError();
}

}  // namespace kda
