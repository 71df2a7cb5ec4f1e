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
// With a gated RMSNorm epilogue (NeMo glm5_next layers, _TorchRMSNormGated) the kernel writes
// y = o / sqrt(mean over the head's value columns of o^2 + eps) * w * sigmoid(gate) instead of o,
// from o rounded to bf16, in the same arithmetic as the separate pass (kda_norm.cu).
//
// Layout: the state is kept transposed, S^T [value column j][key channel c], in TMEM lane j, so
// every product takes its state-side operand from TMEM and no shared-memory write sits on the
// critical path:
//   D = S^T [W; Q+]^T     (A = bf16 copy of S^T in TMEM, B = [W; Q+] K-major in shared memory)
//   S^T += U^T K_end      (A = bf16 U^T in TMEM, B = K_end MN-major in shared memory)
//   o^T = (Q+ S)^T + U^T A_qk^T   (accumulated into D's second half; A = U^T, B = A_qk K-major)
//
// Roles (14 warps):
//   - 8 chain warps walk the chunks: warps w and w + 4 share TMEM lane quarter w mod 4 (lane j =
//     value column j) and split the columns of every TMEM row between them. Per chunk c the chain
//     is bf16(S^T) -> (W S)^T (8 K steps; the (Q+ S)^T half of D follows it in the pipe, off the
//     chain) -> U^T = U~^T - (W S)^T -> S^T += U^T K_end (4 K steps); the
//     decay of S^T and the load of U~^T run while D is in flight.
//   - 1 MMA warp: issues every tcgen05.mma (the whole warp runs the issue code, one elected lane
//     issues, so that the operands stay warp-uniform).
//   - 4 epilogue warps (one per lane quarter) take o of chunk c out of TMEM once its product is
//     done, stage it row-major in shared memory (applying the norm when asked, with the gate
//     tile of chunk c fetched by TMA a chunk ahead) and store it, so that none of the output's
//     work sits on the chain. The D buffers are double-buffered: the MMA thread issues chunk c's
//     D product once the epilogue has read chunk c-2's.
//   - 1 loader warp: one thread issues the TMA copies of the records (two stages): chunk c+2's
//     as soon as chunk c's o product is done, which frees chunk c's stage (its update precedes
//     it), a whole chunk before they are needed (a record takes about 2.5 K cycles to land,
//     and issuing its copies about 650).
// The chain warps and the MMA warp synchronise with named barrier 1, the epilogue warps with named
// barrier 2, and the two groups only through mbarriers. Every mbarrier wait is bounded; on expiry
// the CTA records KDA_ERR_TIMEOUT, drains its own copies and MMAs, frees TMEM and exits.
//
// The same kernel serves the two-level state pass (kda_scan.cuh): a segmented launch gives each
// CTA one (segment, chain) unit with its own initial and final state, a transition-map unit
// starts from S = I with U~ taken as 0 (its final state is the segment's map A), and a launch
// without outputs skips the epilogue's stores. scan_combine_kernel, below, chains the segments'
// initial states between the launches.

#include <cuda.h>
#include <cudaTypedefs.h>

#include <cstdlib>
#include <cstring>
#include <mutex>

#include "kda_internal.cuh"
#include "kda_scan.cuh"
#include "kda_sm100.cuh"
#include "kda_tma.cuh"

namespace kda {
namespace {

using namespace sm100;

constexpr int kC = 64;
constexpr int kD = 128;
constexpr int kDataWarps = 8;
constexpr int kEpiWarps = 4;
constexpr int kChainThreads = 32 * kDataWarps + 32;          // chain warps + the MMA warp
constexpr int kEpiThreads = 32 * kEpiWarps;
constexpr int kThreads = kChainThreads + kEpiThreads + 32;     // + the loader warp
constexpr int kMma = 32 * kDataWarps;    // first thread of the warp that issues the MMAs
constexpr int kMmaWarp = kDataWarps;
constexpr int kEpi0 = kChainThreads;     // first epilogue thread (issues the output stores)
constexpr int kLoader = kChainThreads + kEpiThreads;   // thread that issues the record copies
constexpr uint32_t kBarChain = 1, kBarEpi = 2;   // named barriers (0 is __syncthreads)

// one pipeline stage (bytes from a 1024-aligned stage base)
constexpr uint32_t ST_WQ = 0;        // [W; Q+] 128 x 128 bf16, K-major SW128: 2 panels of 16 KB
constexpr uint32_t ST_KE = 32768;    // K_end 64 x 128 bf16, MN-major SW128: 2 panels of 8 KB
constexpr uint32_t ST_UT = 49152;    // U~^T [128 j][64 tokens] bf16, SW128
constexpr uint32_t ST_AQ = 65536;    // A_qk [64 r][64 i] bf16, K-major SW128
constexpr uint32_t ST_DEC = 73728;   // e^{Gamma_end} [128] f32
constexpr uint32_t kStage = 74752;   // 73 KB, a multiple of 1024
constexpr uint32_t kTxStage = 32768 + 2 * 16384 + 8192 + 512;
constexpr uint32_t OFF_G = 2 * kStage;       // two norm gate tiles [64 tokens][128] bf16
constexpr uint32_t OFF_Y = OFF_G + 32768;    // two output tiles [64 tokens][128] bf16
constexpr uint32_t OFF_BAR = OFF_Y + 32768;  // mbarriers
constexpr uint32_t OFF_FLAG = OFF_BAR + 128; // set when the chain aborts
constexpr uint32_t OFF_TMEM = OFF_FLAG + 16;
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
    __nv_bfloat16* o;       // o, or y with the norm
    const float* decay;     // [R][128]
    const __nv_bfloat16* gate;   // norm gate, shaped like o (nullable: no norm)
    const float* nw;             // norm weight [128]
    float eps;
    int T, H, N, ncT;       // ncT: chunk records per sequence when cu is null
    // segmented launch (seg_m > 0; equal-length sequences): unit u = (group, segment, chain),
    // as ScanSplit describes; ident: group 0 starts from S = I with U~ = 0
    int seg_m, seg_p0, seg_count, nseg;
    int ident, no_out, hT_last;
    long long G;            // chunk records per head
    long long budget;
    int debug_stall;
    unsigned* err;
};

struct ScanMaps {
    CUtensorMap wq, ke, ut, aq, o, g;   // g: the norm gate, shaped like o (unused without it)
};

__device__ __forceinline__ uint32_t pack2(float x, float y) {
    __nv_bfloat162 v = __floats2bfloat162_rn(x, y);
    return *reinterpret_cast<uint32_t*>(&v);
}
__device__ __forceinline__ float lo_bf(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float hi_bf(uint32_t u) { return __uint_as_float(u & 0xffff0000u); }

// Named barrier over `count` threads (a multiple of 32), and the same with an OR of `pred`.
__device__ __forceinline__ void bar_sync(uint32_t id, uint32_t count) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}
__device__ __forceinline__ bool bar_or(uint32_t id, uint32_t count, bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 q, %1, 0;\n\t"
        "bar.red.or.pred p, %2, %3, q;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)pred), "r"(id), "r"(count)
        : "memory");
    return r != 0;
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__global__ void __launch_bounds__(kThreads, 1)
chunk_scan_kernel(const __grid_constant__ ScanMaps maps, const ScanArgs args) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
    const uint32_t sb = smem_u32(sm);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int qd = warp & 3;                   // TMEM lane quarter (every role)
    const int hs = (warp >> 2) & 1;            // chain warps: column half
    const int j = 32 * qd + lane;              // value column = TMEM lane
    const bool data = warp < kDataWarps;
    const bool epi = tid >= kEpi0 && tid < kLoader;
    const bool loader = tid >= kLoader;
    const int unit = blockIdx.x;
    int chain = unit, seg = 0, c_begin = args.c_begin, c_end = args.c_end;
    bool ident = false;
    if (args.seg_m > 0) {
        const int chains = args.N * args.H;
        chain = unit % chains;
        const int rest = unit / chains;
        seg = args.seg_p0 + rest % args.seg_count;
        ident = args.ident && rest < args.seg_count;
        c_begin = seg * args.seg_m;
        c_end = c_begin + args.seg_m;
    }
    const int h = chain % args.H;
    const int n = args.order ? args.order[chain / args.H] : chain / args.H;

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
        const long long sb0 = min(t1, t0 + (long long)kC * c_begin);
        const long long sb1 = min(t1, t0 + (long long)kC * c_end);
        g0 += (sb0 - t0 + kC - 1) / kC;
        t0 = sb0;
        t1 = max(sb0, sb1);
    }
    const int nchunks = (int)((t1 - t0 + kC - 1) / kC);

    uint32_t* tmem_s = reinterpret_cast<uint32_t*>(sm + OFF_TMEM);
    volatile int* abort_s = reinterpret_cast<volatile int*>(sm + OFF_FLAG);
    const uint32_t bar_full0 = sb + OFF_BAR;                       // + 8 (c & 1)
    const uint32_t bar_mma1 = bar_full0 + 16, bar_mma2 = bar_full0 + 24;
    const uint32_t bar_never = bar_full0 + 32;
    const uint32_t bar_o0 = bar_full0 + 40;      // + 8 (c & 1): o product of chunk c done
    const uint32_t bar_dfree0 = bar_full0 + 56;  // + 8 (c & 1): epilogue has read D buffer c & 1
    const uint32_t bar_gate0 = bar_full0 + 72;   // + 8 (c & 1): gate tile of chunk c landed
    if (tid == 0) {
        mbar_init(bar_full0, 1);
        mbar_init(bar_full0 + 8, 1);
        mbar_init(bar_mma1, 1);
        mbar_init(bar_mma2, 1);
        mbar_init(bar_never, 1);
        mbar_init(bar_o0, 1);
        mbar_init(bar_o0 + 8, 1);
        mbar_init(bar_dfree0, kEpiThreads);
        mbar_init(bar_dfree0 + 8, kEpiThreads);
        mbar_init(bar_gate0, 1);
        mbar_init(bar_gate0 + 8, 1);
        *abort_s = 0;
        fence_mbar_init();
        prefetch_tmap(&maps.wq);
        prefetch_tmap(&maps.ke);
        prefetch_tmap(&maps.ut);
        prefetch_tmap(&maps.aq);
        prefetch_tmap(&maps.o);
        if (args.gate) prefetch_tmap(&maps.g);
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
    // a segmented launch keeps its states per unit (the last segment's hT per chain)
    const size_t h0_base = args.seg_m > 0 ? (size_t)unit * kD * kD : state_base;
    float* const hT = args.seg_m > 0 && args.hT_last && seg != args.nseg - 1 ? nullptr : args.hT;
    const size_t hT_base = args.seg_m > 0 && !args.hT_last ? (size_t)unit * kD * kD : state_base;

    // initial state, transposed: lane j, column c holds S[c][j]; this thread: c in [64 hs, +64)
    // (the identity for a transition-map unit)
#pragma unroll 1
    for (int p = 0; p < (data ? 2 : 0); ++p) {
        float v[32];
        const int c0 = 64 * hs + 32 * p;
#pragma unroll
        for (int i = 0; i < 32; ++i)
            v[i] = ident ? (c0 + i == j ? 1.f : 0.f)
                         : (args.h0 ? args.h0[h0_base + (size_t)(c0 + i) * kD + j] : 0.f);
        tmem_st32(tbase + lq + TS + c0, v);
    }
    tmem_st_wait();

    // records of chunk c into stage c & 1 (issued by the loader thread)
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

    if (loader) {
        // ============================================================ loader warp
        // chunk c's stage is free once its o product is done (its update precedes it): chunk
        // c+2's records go there. After a chain abort the wait expires and the loader stops.
        if (tid == kLoader) {
            int last0 = -1, last1 = -1;   // the chunk whose records went last into each stage
            if (nchunks > 0) issue(0), last0 = 0;
            if (nchunks > 1) issue(1), last1 = 1;
            for (int c = 0; c + 2 < nchunks; ++c) {
                if (!mbar_wait(bar_o0 + 8 * (c & 1), (uint32_t)((c >> 1) & 1), args.budget)) break;
                issue(c + 2);
                if (c & 1) last1 = c + 2;
                else last0 = c + 2;
            }
            // copies still in flight land before the smem goes away (bounded; earlier copies
            // were waited for by the chain, and a completed phase returns at once)
            if (last0 >= 0) mbar_wait(bar_full0, (uint32_t)((last0 >> 1) & 1), 1ll << 31);
            if (last1 >= 0) mbar_wait(bar_full0 + 8, (uint32_t)((last1 >> 1) & 1), 1ll << 31);
        }
    } else if (!epi) {
        // ============================================================ chain warps and MMA warp
        const uint64_t dK = sw128_desc(0, 16, 1024);     // K-major, 128B swizzle
        const uint64_t dM8 = sw128_desc(0, 8192, 1024);  // MN-major, 64-row panels
        const uint32_t id_half = idesc_bf16(128, 64, 0, 0);   // D halves and the o product
        const uint32_t id2 = idesc_bf16(128, 128, 0, 1);

        // outstanding MMAs, drained before exit if a wait expires (the record copies are the
        // epilogue's to drain)
        bool mma1_pending = false, mma2_pending = false, o_pending = false;
        int mma1_chunk = 0, mma2_chunk = 0, o_chunk = 0;   // chunk of the last commit
        bool aborted = false;
        // thread 0 polls; the chain waits at the barrier that publishes the outcome (and any
        // failure a thread has recorded in `also_bad` since the last barrier)
        auto wait_chain = [&](uint32_t bar, uint32_t parity, bool also_bad) -> bool {
            const bool ok = tid != 0 || mbar_wait(bar, parity, args.budget);
            return !bar_or(kBarChain, kChainThreads, !ok || also_bad);
        };

        if (args.debug_stall && !wait_chain(bar_never, 0, false)) aborted = true;

        for (int c = 0; c < nchunks && !aborted; ++c) {
            const uint32_t st = sb + (uint32_t)(c & 1) * kStage;
            const uint8_t* stp = sm + (size_t)(c & 1) * kStage;

            // records of chunk c landed; S of chunk c complete once the previous update has.
            // Every chain thread waits itself (bounded) and the outcome is agreed on at the
            // barrier after the conversion, so no barrier of its own sits on the chain.
            bool ok = true;
            if (data) {
                ok = mbar_wait(bar_full0 + 8 * (c & 1), (uint32_t)((c >> 1) & 1), args.budget);
                if (ok && mma2_pending)
                    ok = mbar_wait(bar_mma2, (uint32_t)(mma2_chunk & 1), args.budget);
                tc_fence_after();
            }

            // ------------------------------------------------------------ bf16 S^T -> TB
            if (data && ok) {
                float va[32], vb[32];
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
            tc_fence_before();
            if (bar_or(kBarChain, kChainThreads, !ok)) { aborted = true; break; }
            mma2_pending = false;
            tc_fence_after();

            // ------------------------------------------------------------ D = S^T [W; Q+]^T
            bool mma_bad = false;
            if (warp == kMmaWarp) {
                // D buffer c & 1 last held chunk c-2's product: wait until the epilogue has
                // read its o (long done in steady state)
                if (c >= 2 && lane == 0)
                    mma_bad = !mbar_wait(bar_dfree0 + 8 * (c & 1), (uint32_t)(((c - 2) >> 1) & 1),
                                         args.budget);
                mma_bad = __shfl_sync(0xffffffffu, mma_bad, 0);
                if (!mma_bad) {
                    tc_fence_after();
                    // (W S)^T first, committed on its own: the chain needs only this half; the
                    // (Q+ S)^T half follows in the pipe while the chain forms U
#pragma unroll
                    for (int s = 0; s < kD / 16; ++s)
                        umma_f16_ts_warp(tbase + TD + 128 * (c & 1), tbase + TB + 8 * s,
                                         desc_at(dK, st + ST_WQ + (s >> 2) * 16384 + (s & 3) * 32),
                                         id_half, s > 0);
                    umma_commit_warp(bar_mma1);
#pragma unroll
                    for (int s = 0; s < kD / 16; ++s)
                        umma_f16_ts_warp(
                            tbase + TD + 128 * (c & 1) + 64, tbase + TB + 8 * s,
                            desc_at(dK, st + ST_WQ + 8192 + (s >> 2) * 16384 + (s & 3) * 32),
                            id_half, s > 0);
                }
            }
            mma1_pending = true;
            mma1_chunk = c;

            // ------------------------------------------------------------ while D runs
            // decay: S^T diag(e^{Gamma_end}) in registers (stored into TS, where the update
            // accumulates, with U^T below); U~^T rows
            uint32_t ub[16];
            if (data) {
                float va[32], vb[32];
                tmem_ld32(tbase + lq + TS + 64 * hs, va);
                tmem_ld32(tbase + lq + TS + 64 * hs + 32, vb);
                const float* dec = reinterpret_cast<const float*>(stp + ST_DEC) + 64 * hs;
#pragma unroll
                for (int m = 0; m < 4; ++m) {   // (zero for a transition-map unit)
                    const uint4 x = ident ? make_uint4(0u, 0u, 0u, 0u)
                                          : *reinterpret_cast<const uint4*>(
                                                stp + ST_UT + sw128_off(128, j, 32 * hs + 8 * m));
                    ub[4 * m] = x.x; ub[4 * m + 1] = x.y; ub[4 * m + 2] = x.z; ub[4 * m + 3] = x.w;
                }
                tmem_ld_wait();
#pragma unroll
                for (int i = 0; i < 32; i += 4) {
                    const float4 d0 = *reinterpret_cast<const float4*>(dec + i);
                    const float4 d1 = *reinterpret_cast<const float4*>(dec + 32 + i);
                    va[i] *= d0.x; va[i + 1] *= d0.y; va[i + 2] *= d0.z; va[i + 3] *= d0.w;
                    vb[i] *= d1.x; vb[i + 1] *= d1.y; vb[i + 2] *= d1.z; vb[i + 3] *= d1.w;
                }
                tmem_st32(tbase + lq + TS + 64 * hs, va);
                tmem_st32(tbase + lq + TS + 64 * hs + 32, vb);
                tmem_st_wait();
            }

            // (W S)^T done: again each chain thread waits itself, agreed on at the next barrier
            bool ok1 = true;
            if (data) {
                ok1 = mbar_wait(bar_mma1, (uint32_t)(c & 1), args.budget);
                tc_fence_after();
            }

            // ------------------------------------------------------------ U^T = U~^T - (W S)^T
            if (data && ok1) {
                float w[32];
                tmem_ld32(tbase + lq + TD + 128 * (c & 1) + 32 * hs, w);
                tmem_ld_wait();
                uint32_t pk[16];
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    pk[i] = pack2(lo_bf(ub[i]) - w[2 * i], hi_bf(ub[i]) - w[2 * i + 1]);
                tmem_st16u(tbase + lq + TU + 16 * hs, pk);
                tmem_st_wait();
            }
            tc_fence_before();
            if (bar_or(kBarChain, kChainThreads, !ok1 || mma_bad)) { aborted = true; break; }
            mma1_pending = false;
            tc_fence_after();

            // ------------------------------------------------------------ S^T += U^T K_end
            if (warp == kMmaWarp) {
                tc_fence_after();
#pragma unroll
                for (int s = 0; s < kC / 16; ++s)
                    umma_f16_ts_warp(tbase + TS, tbase + TU + 8 * s,
                                     desc_at(dM8, st + ST_KE + 2048 * s), id2, 1);
                umma_commit_warp(bar_mma2);
                // o^T = (Q+ S)^T + U^T A_qk^T, behind the update in the pipe (off the chain)
#pragma unroll
                for (int s = 0; s < kC / 16; ++s)
                    umma_f16_ts_warp(tbase + TD + 128 * (c & 1) + 64, tbase + TU + 8 * s,
                                     desc_at(dK, st + ST_AQ + 32 * s), id_half, 1);
                umma_commit_warp(bar_o0 + 8 * (c & 1));
            }
            mma2_pending = o_pending = true;
            mma2_chunk = o_chunk = c;
        }

        if (aborted) {
            if (tid == 0) set_device_error(args.err, DEV_TIMEOUT);
            *abort_s = 1;
            // wind down: this CTA's own copies and MMAs finish before TMEM and smem go away
            const long long drain = 1ll << 31;
            if (tid == kMma) {
                if (mma1_pending) mbar_wait(bar_mma1, (uint32_t)(mma1_chunk & 1), drain);
                if (mma2_pending) mbar_wait(bar_mma2, (uint32_t)(mma2_chunk & 1), drain);
                if (o_pending)
                    mbar_wait(bar_o0 + 8 * (o_chunk & 1), (uint32_t)((o_chunk >> 1) & 1), drain);
            }
        } else {
            bool ok = true;
            if (tid == 0 && mma2_pending)
                ok = mbar_wait(bar_mma2, (uint32_t)(mma2_chunk & 1), args.budget);
            if (bar_or(kBarChain, kChainThreads, !ok)) {
                if (tid == 0) set_device_error(args.err, DEV_TIMEOUT);
                *abort_s = 1;
                if (tid == kMma) mbar_wait(bar_mma2, (uint32_t)(mma2_chunk & 1), 1ll << 31);
            } else {
                tc_fence_after();
                if (hT && data) {
#pragma unroll 1
                    for (int p = 0; p < 2; ++p) {
                        float v[32];
                        const int c0 = 64 * hs + 32 * p;
                        tmem_ld32(tbase + lq + TS + c0, v);
                        tmem_ld_wait();
#pragma unroll
                        for (int i = 0; i < 32; ++i)
                            hT[hT_base + (size_t)(c0 + i) * kD + j] = v[i];
                    }
                }
            }
        }
    } else {
        // ============================================================ epilogue warps
        const int et = tid - kEpi0;   // 0..127
        const int ew = et >> 5;       // 0..3: rows 16 ew .. 16 ew + 15 of the norm pass
        const bool norm = args.gate != nullptr;
        float wv[4] = {0.f, 0.f, 0.f, 0.f};
        if (norm) {
            const float4 x = *reinterpret_cast<const float4*>(args.nw + 4 * lane);
            wv[0] = x.x; wv[1] = x.y; wv[2] = x.z; wv[3] = x.w;
        }
        // gate tile of chunk cc (one 64-row box of this head; rows past the document are read
        // but not used) into gate buffer cc & 1
        auto issue_gate = [&](int cc) {
            const uint32_t bar = bar_gate0 + 8 * (cc & 1);
            mbar_arrive_expect_tx(bar, 16384);
            tma_load_3d(sb + OFF_G + 16384 * (cc & 1), &maps.g, bar, 0, h,
                        (int)(t0 + (long long)kC * cc));
        };
        int gate_issued = 0, gate_landed = 0;
        if (norm && et == 0 && nchunks > 0) issue_gate(0);
        if (norm) gate_issued = min(nchunks, 1);

        for (int c = 0; c < nchunks; ++c) {
            // o product of chunk c done (every epilogue thread polls, bounded; after a chain
            // abort the wait expires and the epilogue stops)
            const bool ok =
                mbar_wait(bar_o0 + 8 * (c & 1), (uint32_t)((c >> 1) & 1), args.budget);
            if (bar_or(kBarEpi, kEpiThreads, !ok)) {
                if (et == 0 && !*abort_s) set_device_error(args.err, DEV_TIMEOUT);
                break;
            }
            // the gate of chunk c+1 goes into the buffer chunk c-1's norm finished reading
            if (norm && c + 1 < nchunks) {
                if (et == 0) issue_gate(c + 1);
                gate_issued = c + 2;
            }
            tc_fence_after();
            float v[64];   // o^T row j: tokens 0..63 of value column j
            {
                float a[32], b[32];
                tmem_ld32(tbase + lq + TD + 128 * (c & 1) + 64, a);
                tmem_ld32(tbase + lq + TD + 128 * (c & 1) + 96, b);
                tmem_ld_wait();
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    v[i] = a[i];
                    v[32 + i] = b[i];
                }
            }
            tc_fence_before();
            mbar_arrive(bar_dfree0 + 8 * (c & 1));   // D buffer c & 1 may be overwritten now
            if (args.no_out) continue;
            // output tile c & 1 was last stored for chunk c-2: that store must have read it
            if (et == 0 && c >= 2) bulk_wait_read_le1();
            bar_sync(kBarEpi, kEpiThreads);
            __nv_bfloat16* tile = reinterpret_cast<__nv_bfloat16*>(sm + OFF_Y + 16384 * (c & 1));
            const long long r0 = t0 + (long long)kC * c;
            const int L = (int)min((long long)kC, t1 - r0);
#pragma unroll
            for (int t = 0; t < kC; ++t) tile[t * kD + j] = __float2bfloat16_rn(v[t]);
            if (norm) {
                const bool gok =
                    mbar_wait(bar_gate0 + 8 * (c & 1), (uint32_t)((c >> 1) & 1), args.budget);
                gate_landed = c + 1;
                if (bar_or(kBarEpi, kEpiThreads, !gok)) {   // also: the tile is complete
                    if (et == 0) set_device_error(args.err, DEV_TIMEOUT);
                    break;
                }
                const __nv_bfloat16* gt =
                    reinterpret_cast<const __nv_bfloat16*>(sm + OFF_G + 16384 * (c & 1));
                // one warp per 16 rows, lane l on columns 4 l .. 4 l + 3, in place; the same
                // arithmetic as the separate pass (kda_norm.cu)
#pragma unroll 8
                for (int rr = 0; rr < 16; ++rr) {
                    const int t = 16 * ew + rr;
                    const uint2 u = *reinterpret_cast<const uint2*>(tile + t * kD + 4 * lane);
                    const float x[4] = {lo_bf(u.x), hi_bf(u.x), lo_bf(u.y), hi_bf(u.y)};
                    float ss = 0.f;
#pragma unroll
                    for (int e = 0; e < 4; ++e) ss = fmaf(x[e], x[e], ss);
#pragma unroll
                    for (int off = 16; off >= 1; off >>= 1)
                        ss += __shfl_xor_sync(0xffffffffu, ss, off);
                    const float inv = rsqrtf(ss / (float)kD + args.eps);
                    const uint2 gu = *reinterpret_cast<const uint2*>(gt + t * kD + 4 * lane);
                    const float g[4] = {lo_bf(gu.x), hi_bf(gu.x), lo_bf(gu.y), hi_bf(gu.y)};
                    float y[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        y[e] = x[e] * inv * wv[e] * __fdividef(1.f, 1.f + __expf(-g[e]));
                    *reinterpret_cast<uint2*>(tile + t * kD + 4 * lane) =
                        make_uint2(pack2(y[0], y[1]), pack2(y[2], y[3]));
                }
            }
            fence_proxy_async();   // tile -> TMA store
            bar_sync(kBarEpi, kEpiThreads);
            // one TMA store for a full chunk, row copies for a partial one (a TMA box would run
            // into the next document's rows)
            if (L == kC) {
                if (et == 0) {
                    tma_store_3d(&maps.o, smem_u32(tile), 0, h, (int)r0);
                    bulk_commit();
                }
            } else {
                const uint4* src = reinterpret_cast<const uint4*>(tile);
                for (int i = et; i < L * 16; i += kEpiThreads) {
                    const int r = i >> 4, q = i & 15;
                    *reinterpret_cast<uint4*>(args.o + ((size_t)(r0 + r) * args.H + h) * kD +
                                              8 * q) = src[r * 16 + q];
                }
            }
        }
        if (et == 0) {
            // gate copies still in flight land before the smem goes away (bounded)
            for (int cc = gate_landed; cc < gate_issued; ++cc)
                mbar_wait(bar_gate0 + 8 * (cc & 1), (uint32_t)((cc >> 1) & 1), 1ll << 31);
            bulk_wait_all();   // output stores complete before the smem goes away
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tbase, kTmemCols);
}

// Initial states of the two-level state pass's segments, S_p = A_{p-1} S_{p-1} + B_{p-1} for
// p = 1 .. steps (a few 128 x 128 x 128 products per chain, on the critical path once per
// segment). Block (jb, chain) owns value columns 16 jb .. 16 jb + 15 of one chain (the columns
// are independent); warp w computes rows 16 w .. 16 w + 15 of them with tensor-core products in
// 3xTF32: each fp32 operand x = hi + lo with hi = x rounded to tf32 and lo = the rest rounded
// to tf32, and a b is taken as hi_a hi_b + (lo_a hi_b + hi_a lo_b) (the lo lo term, about 2^-22 of
// the product, is dropped), each of the three in its own fp32 accumulator (short dependency
// chains), summed at the end with B_{p-1}. The maps are staged in shared memory by 16-byte
// asynchronous copies, double-buffered: A_p lands while step p computes, and B_p is read into
// registers a step ahead. The row strides (132 floats for A, 24 for S) put every fragment read
// of a warp in distinct banks.
constexpr int kCombCols = 16;
constexpr int kCombLdA = 132;
constexpr int kCombLdS = 24;
constexpr uint32_t kCombSmem = (uint32_t)(2 * kD * kCombLdA + kD * kCombLdS) * 4;

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
    asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ uint32_t to_tf32(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}
__device__ __forceinline__ void split_tf32(float x, uint32_t& hi, uint32_t& lo) {
    hi = to_tf32(x);
    lo = to_tf32(x - __uint_as_float(hi));
}

__global__ void __launch_bounds__(256)
scan_combine_kernel(const float* __restrict__ amap, const float* __restrict__ bmap,
                    float* __restrict__ sinit, int chains, int steps) {
    extern __shared__ float4 comb_raw[];
    float* As0 = reinterpret_cast<float*>(comb_raw);   // 2 x [128][kCombLdA]: A_{p-1}, A_p
    float* Ss = As0 + 2 * kD * kCombLdA;                // [128][kCombLdS]: S_{p-1}'s columns
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, t = lane & 3, r0 = 16 * warp;
    const int jb = blockIdx.x, chain = blockIdx.y;
    const size_t mat = (size_t)kD * kD;
    const size_t col0 = (size_t)kCombCols * jb;
    // A_{p-1} into buffer (p - 1) & 1: 16 copies of 16 bytes per thread, one commit group
    auto stage = [&](int p) {
        const float* A = amap + ((size_t)(p - 1) * chains + chain) * mat;
        float* As = As0 + ((p - 1) & 1) * kD * kCombLdA;
#pragma unroll
        for (int u = 0; u < kD * kD / 4 / 256; ++u) {
            const int i = tid + 256 * u, r = i >> 5, q = i & 31;
            cp_async16(smem_u32(As + r * kCombLdA + 4 * q), A + (size_t)r * kD + 4 * q);
        }
        cp_async_commit();
    };
    // B_{p-1} of this thread's fragment into bnext
    float bnext[2][4];
    auto load_b = [&](int p) {
        const float* B = bmap + ((size_t)(p - 1) * chains + chain) * mat + col0;
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            const int col = 8 * nt + 2 * t;
            const float2 u = *reinterpret_cast<const float2*>(B + (size_t)(r0 + g) * kD + col);
            const float2 v = *reinterpret_cast<const float2*>(B + (size_t)(r0 + g + 8) * kD + col);
            bnext[nt][0] = u.x; bnext[nt][1] = u.y; bnext[nt][2] = v.x; bnext[nt][3] = v.y;
        }
    };
    stage(1);
    load_b(1);
    for (int i = tid; i < kD * kCombCols / 4; i += 256) {
        const int r = i >> 2, q = i & 3;
        *reinterpret_cast<float4*>(Ss + r * kCombLdS + 4 * q) =
            *reinterpret_cast<const float4*>(sinit + chain * mat + (size_t)r * kD + col0 + 4 * q);
    }
    for (int p = 1; p <= steps; ++p) {
        // the next map goes into the buffer step p - 1 read (released by its closing barrier)
        if (p < steps) stage(p + 1);
        const float* As = As0 + ((p - 1) & 1) * kD * kCombLdA;
        // B_{p-1} (read a step ahead) and the next step's, in the m16n8 fragment layout: rows
        // r0 + g (+ 8), columns 8 nt + 2 t (+ 1)
        float bias[2][4];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) bias[nt][e] = bnext[nt][e];
        if (p < steps) load_b(p + 1);
        float acc[2][4] = {}, acc_x[2][4] = {}, acc_y[2][4] = {};
        if (p < steps)
            cp_async_wait<1>();   // this step's map landed (the next one may still be in flight)
        else
            cp_async_wait<0>();
        __syncthreads();   // A_{p-1} staged by every thread, S_{p-1} complete
#pragma unroll 4
        for (int kk = 0; kk < kD; kk += 8) {
            const float* la = As + (r0 + g) * kCombLdA + kk + t;
            uint32_t ah[4], al[4];
            split_tf32(la[0], ah[0], al[0]);
            split_tf32(la[8 * kCombLdA], ah[1], al[1]);
            split_tf32(la[4], ah[2], al[2]);
            split_tf32(la[8 * kCombLdA + 4], ah[3], al[3]);
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                const float* lb = Ss + (kk + t) * kCombLdS + 8 * nt + g;
                uint32_t bh[2], bl[2];
                split_tf32(lb[0], bh[0], bl[0]);
                split_tf32(lb[4 * kCombLdS], bh[1], bl[1]);
                mma_tf32_16x8x8(acc_x[nt], al, bh);
                mma_tf32_16x8x8(acc_y[nt], ah, bl);
                mma_tf32_16x8x8(acc[nt], ah, bh);
            }
        }
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e)
                acc[nt][e] = bias[nt][e] + (acc[nt][e] + (acc_x[nt][e] + acc_y[nt][e]));
        __syncthreads();   // every warp has read A_{p-1} and S_{p-1}
        float* out = sinit + ((size_t)p * chains + chain) * mat + col0;
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            const int col = 8 * nt + 2 * t;
            *reinterpret_cast<float2*>(Ss + (r0 + g) * kCombLdS + col) =
                make_float2(acc[nt][0], acc[nt][1]);
            *reinterpret_cast<float2*>(Ss + (r0 + g + 8) * kCombLdS + col) =
                make_float2(acc[nt][2], acc[nt][3]);
            *reinterpret_cast<float2*>(out + (size_t)(r0 + g) * kD + col) =
                make_float2(acc[nt][0], acc[nt][1]);
            *reinterpret_cast<float2*>(out + (size_t)(r0 + g + 8) * kD + col) =
                make_float2(acc[nt][2], acc[nt][3]);
        }
    }
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

// One CTA (14 warps) per (sequence or document, head); packed documents are taken longest first
// when an order is given.
cudaError_t launch_chunk_scan(const FwdParams& p, const ScanSegment& seg, cudaStream_t stream,
                              const ScanNorm* norm) {
    return launch_chunk_scan_split(p, seg, ScanSplit{}, stream, norm);
}

cudaError_t launch_chunk_scan_split(const FwdParams& p, const ScanSegment& seg,
                                    const ScanSplit& split, cudaStream_t stream,
                                    const ScanNorm* norm) {
    const SplitWorkspace& ws = *p.split;
    const long long chains = (long long)p.N * p.H;
    const long long units = split.seg_m > 0 ? chains * split.seg_count * split.groups : chains;
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
    if (norm) {
        if ((e = make_map_3d_rows(&m.g, norm->gate, BF, 2, (unsigned long long)p.B * p.T, p.H, kD,
                                  kC)) != cudaSuccess)
            return e;
    } else {
        memset(&m.g, 0, sizeof(m.g));
    }
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
    a.seg_m = split.seg_m;
    a.seg_p0 = split.seg_p0;
    a.seg_count = split.seg_count;
    a.nseg = split.nseg;
    a.ident = split.ident ? 1 : 0;
    a.no_out = split.no_out ? 1 : 0;
    a.hT_last = split.hT_last ? 1 : 0;
    a.o = static_cast<__nv_bfloat16*>(p.o);
    a.decay = ws.decay;
    if (norm) {
        a.gate = static_cast<const __nv_bfloat16*>(norm->gate);
        a.nw = norm->weight;
        a.eps = norm->eps;
    }
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

cudaError_t launch_scan_combine(const float* amap, const float* bmap, float* sinit, int chains,
                                int steps, cudaStream_t stream) {
    if (steps <= 0 || chains <= 0) return cudaSuccess;
    if (chains > 65535) return cudaErrorInvalidConfiguration;
    static PerDevice attr;
    const cudaError_t attr_err = attr.run([](int) {
        return cudaFuncSetAttribute(scan_combine_kernel,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kCombSmem);
    });
    if (attr_err != cudaSuccess) return attr_err;
    scan_combine_kernel<<<dim3(kD / kCombCols, (unsigned)chains), 256, kCombSmem, stream>>>(
        amap, bmap, sinit, chains, steps);
    return cudaGetLastError();
}

}  // namespace kda
