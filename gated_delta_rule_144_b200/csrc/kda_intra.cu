// Intra-chunk kernel of the split chunked prefill: the WY factors of every (chunk, head) record,
// independent of the state, so all records of all sequences run at once.
//
// Per chunk of 64 rows r of one head (WY / UT form of the gated delta rule; GLM-5.3-Flash model
// card, Kimi Delta Attention snippet), with Gamma the within-chunk cumulative log decay per key
// channel:
//   A_kk[r,i] = sum_c k_rc k_ic e^{Gamma_rc - Gamma_ic}  (i < r)    A_qk: same with q_r, i <= r
//   T  = (I + diag(beta) A_kk)^-1 diag(beta)                          (UT transform, fp32)
//   W  = T (k e^{Gamma}),  U~ = T v,  Q+ = q e^{Gamma},
//   K_end = k e^{Gamma_end - Gamma},  decay = e^{Gamma_end}
// and the state pass later applies U = U~ - W S, o = Q+ S + A_qk U, S <- diag(decay) S + K_end^T U.
// A_kk and A_qk come from one tensor-core product R C^T of separable factors anchored at the
// middle of each 16-row block (rows of R at their own block's middle, diagonal-block columns at
// theirs, the columns a later block needs at that later block's middle), so no factor leaves the
// float32 range while the summed decay of 8 consecutive rows stays above about -69 nats; a chunk
// with a steeper decay is evaluated directly (steep_chunk).
//
// Occupancy: two CTAs share each SM, so that one CTA's tensor-core waits, barriers and memory
// latency are covered by the other's CUDA-core work. To fit two CTAs (about 110 KB of shared memory
// and 256 TMEM columns each) the tiles share space: k and q arrive by TMA where R's rows go and are
// overwritten in place by k rho and q rho, log g arrives in the K+ / V region and is consumed before
// K+ and V are written there, the R/C region then holds the UT solve and finally the store staging.
// Q+ and K_end go from registers straight to the workspace. The next record's input tiles are
// prefetched into L2 while this one runs.
//
// Per record (256 threads; warp 0 issues the MMAs, lane 0 of warp 7 the copies):
//   TMA k, q, log g -> decay products -> TMA V; R, C, K+ (shared), Q+, K_end (global) ->
//   MMA R C^T -> A_kk, A_qk (TMA store of A_qk) -> UT solve -> MMA [T; -] K+ and V^T T^T ->
//   W, U~^T staged in shared memory -> TMA stores.
// Every mbarrier wait is bounded; on expiry the CTA records KDA_ERR_TIMEOUT, drains its own
// copies and MMAs, frees TMEM and exits.

#include <cuda.h>
#include <cudaTypedefs.h>

#include <cstdlib>
#include <cstring>
#include <mutex>
#include <type_traits>

#include "kda_internal.cuh"
#include "kda_sm100.cuh"
#include "kda_tma.cuh"

namespace kda {
namespace {

using namespace sm100;

constexpr int kC = 64;    // tokens per chunk
constexpr int kD = 128;   // dk = dv
constexpr int kThreads = 256;

// shared memory (bytes from a 1024-aligned base)
constexpr uint32_t OFF_KP = 0;               // K+ [64 tokens][128] bf16, MN-major B (2 x 8 KB)
constexpr uint32_t OFF_V = 16384;            // V  [64 tokens][128] bf16, MN-major (TMA, SW128)
constexpr uint32_t OFF_R = 32768;            // R  [128][128] bf16, K-major A (2 x 16 KB)
constexpr uint32_t OFF_C = OFF_R + 32768;    // C  [160][128] bf16, K-major B (2 x 20 KB)
//   after R C^T the R/C region holds the solve buffers:
constexpr uint32_t OFF_LB = OFF_R;           // L = diag(beta) A_kk, f32 [64][kLdl]
constexpr uint32_t OFF_MB = OFF_R + 17408;   // (I + L)^-1, f32 [64][kLdm]
constexpr uint32_t OFF_YS = OFF_R + 35840;   // four 16x17 f32 scratch blocks of the solve
constexpr uint32_t OFF_TT = OFF_R + 40960;   // [T; -] [128][64] bf16 (K-major A of the first WY
                                             //   product, rows 64-127 unused; rows 0-63 also the
                                             //   K-major B of the second)
constexpr uint32_t OFF_ZA = OFF_R + 57344;   // [0; A_qk] [128][64] bf16: rows 64-127 are the
                                             //   record's A_qk tile, stored from here by TMA
//   and, once the UT solve is done with them, the staging tiles of the stores:
constexpr uint32_t OFF_SW = OFF_R;           // W [64][128] (2 panels x 8 KB)
constexpr uint32_t OFF_SUT = OFF_R + 16384;  // U~^T [128 value columns][64 tokens]
constexpr uint32_t OFF_MISC = OFF_C + 40960;
// (steep-decay path only: half-block sums at OFF_C and K+ staged at OFF_C + 4096, both below
// OFF_ZA, which that path writes at the same time)
static_assert(OFF_C + 4096 + 16384 <= OFF_ZA, "steep-path scratch overlaps [0; A_qk]");
constexpr uint32_t OFF_BETA = OFF_MISC;           // f32 [64]
constexpr uint32_t OFF_LOUP = OFF_MISC + 256;     // f32 [4 blocks][2 halves][128]
constexpr uint32_t OFF_BAR = OFF_LOUP + 4096;     // mbarriers
constexpr uint32_t OFF_TMEM = OFF_BAR + 64;       // TMEM base address
constexpr uint32_t OFF_CLAIM = OFF_TMEM + 16;     // two claimed record indices (by parity)
constexpr uint32_t kSmemBytes = OFF_CLAIM + 16 + 1024;   // + alignment slack
static_assert(OFF_ZA + 16384 == OFF_C + 40960, "solve buffers fill the R/C region exactly");
static_assert(OFF_YS + 4 * 16 * 17 * 4 <= OFF_TT, "solve scratch overlaps [T; T']");
static_assert(OFF_SUT + 16384 <= OFF_TT, "staging must not touch [T; -] (read by the second WY "
                                        "product while W is staged) or A_qk (stored meanwhile)");
static_assert(2 * (kSmemBytes + 1024) <= 233472, "two CTAs per SM");
// TMEM columns (fp32, 128 lanes; row m of an M = 128 product sits in lane m)
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t TM_A = 0;     // R C^T [128 x 160]; later [T; -] K+ (0-127, W in lanes
                                 //   0-63) and V^T T^T (128-191: U~^T)
constexpr int kLdl = 68;         // row stride (floats) of L: conflict-free A-fragment loads
constexpr int kLdm = 72;         // row stride (floats) of M: conflict-free B-fragment loads
constexpr uint32_t kTxV = 16384;
constexpr uint32_t kTxIn = 16384 + 16384 + 32768;   // k, q (bf16) and log g (fp32) tiles
constexpr uint32_t OFF_G = 0;   // log g [64][128] f32 row-major, in the K+ / V region until the
                                //   decay products have read it

// row offset, inside C[64:], of the columns row block a needs from earlier blocks
__host__ __device__ constexpr int cross_off(int a) { return a == 1 ? 0 : (a == 2 ? 16 : 48); }

struct IntraArgs {
    const __nv_bfloat16* q;
    const __nv_bfloat16* k;
    const float* g;
    const __nv_bfloat16* beta;
    const int32_t* cu;       // nullable: packed documents
    const int32_t* map;      // packed: document of chunk record g (-1: unused)
    __nv_bfloat16* wq;       // [R * 128][128]: W (rows 0-63, TMA), Q+ (rows 64-127, stores)
    __nv_bfloat16* ke;       // [R * 64][128]: K_end
    float* decay;            // [R][128]
    long long G;             // chunk records per head
    int ncT, T, H, N;
    int c_begin, c_span;     // equal-length sequences: chunks [c_begin, c_begin + c_span) of each
    unsigned long long* counter;   // records claimed so far by this launch (zero at launch)
    long long budget;
    int debug_stall;         // failure-injection hook: wait on a barrier nothing ever signals
    int force_direct;        // test hook: every record takes the steep-decay (direct) path
    unsigned* err;
};

// q, k, v: [rows, H, 128] maps of one head's 64-row tile in 64-column boxes (128-byte swizzle);
// log g: the same with whole 128-column rows, no swizzle; w (the W rows of the [W; Q+] record
// tile), ut, aq: record stores (128-byte swizzle).
struct IntraMaps {
    CUtensorMap q, k, g, v, w, ut, aq;
};

struct Unit {
    int h;
    int L;            // valid rows
    long long row0;   // first token row
    long long rec;    // workspace record
};

__device__ __forceinline__ uint32_t pack_bf16(float x, float y) {
    __nv_bfloat162 v = __floats2bfloat162_rn(x, y);
    return *reinterpret_cast<uint32_t*>(&v);
}
__device__ __forceinline__ float2 unpack_bf16(uint32_t u) {
    return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xffff0000u));
}
__device__ __forceinline__ void st_bf16x4(uint8_t* p, float a, float b, float c, float d) {
    *reinterpret_cast<uint2*>(p) = make_uint2(pack_bf16(a, b), pack_bf16(c, d));
}
__device__ __forceinline__ void st_bf16x8(uint8_t* p, const float* v) {
    *reinterpret_cast<uint4*>(p) = make_uint4(pack_bf16(v[0], v[1]), pack_bf16(v[2], v[3]),
                                              pack_bf16(v[4], v[5]), pack_bf16(v[6], v[7]));
}
__device__ __forceinline__ uint32_t f2tf(float x) { return __float_as_uint(x); }
__device__ __forceinline__ float4 ld4(const float* p) { return *reinterpret_cast<const float4*>(p); }
__device__ __forceinline__ float4 mul4(float4 a, float4 b) {
    return make_float4(a.x * b.x, a.y * b.y, a.z * b.z, a.w * b.w);
}
// Two bf16 products (round to nearest) of the bf16 pair packed in u with the pair f.
__device__ __forceinline__ uint32_t hmul2_u32(uint32_t u, __nv_bfloat162 f) {
    __nv_bfloat162 x = __hmul2(*reinterpret_cast<const __nv_bfloat162*>(&u), f);
    return *reinterpret_cast<uint32_t*>(&x);
}

__device__ __forceinline__ void tma_prefetch_3d(const void* tmap, int c0, int c1, int c2) {
    asm volatile("cp.async.bulk.prefetch.tensor.3d.L2.global.tile [%0, {%1, %2, %3}];" ::"l"(
                     reinterpret_cast<uint64_t>(tmap)),
                 "r"(c0), "r"(c1), "r"(c2)
                 : "memory");
}

// Steep-decay path of one record (all 256 threads; called in place of the operand pass, the
// R C^T product and the assembly when some product of 8 consecutive decays falls below 1e-30).
// On entry: k, q (bf16) in R's rows, log g (f32) in its tile, beta in shared memory. On return
// (after a CTA barrier): L = diag(beta) A_kk, [0; A_qk] and K+ in their buffers, Q+ and K_end in
// the workspace, exactly as the fast path leaves them. Not inlined, so that its registers do not
// weigh on the fast path.
__device__ __noinline__ void steep_chunk(uint8_t* sm, int L, long long rec, __nv_bfloat16* wq,
                                         __nv_bfloat16* ke) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int pb = warp >> 1, hh = warp & 1;
    const int ch0 = 4 * lane;
    const int rbase = 16 * pb + 8 * hh;
    const int rb8 = 2 * pb + hh;
    const uint32_t lh4 = (uint32_t)(((lane & 15) >> 1) << 4);
    const uint32_t lo8 = (uint32_t)((lane & 1) * 8);
    auto toff = [&](int R, int rb, int j) -> uint32_t {
        return (uint32_t)((lane >> 4) * R * 128 + rb * 1024 + j * 128) + (lh4 ^ (uint32_t)(j << 4)) +
               lo8;
    };
    const float* gs = reinterpret_cast<const float*>(sm + OFF_G);
    const float* beta_s = reinterpret_cast<const float*>(sm + OFF_BETA);
    // A chunk whose decay over some 8 rows exceeds the anchored factors' range. Gamma is
    // formed in log space, A_kk and A_qk are summed directly as
    //   sum_c k_rc k_ic e^{Gamma_rc - Gamma_ic}   (exponent <= 0 for i <= r),
    // and K+, Q+, K_end from e^{Gamma} and e^{Gamma_end - Gamma} (both <= 1), so nothing
    // overflows; factors below the float range become zero, as their true values are
    // negligible. The buffers then look as after the fast path's assembly, and the UT
    // transform and the WY products run unchanged.
    float* gsw = reinterpret_cast<float*>(sm + OFF_G);     // log g -> Gamma, in place
    float* hsum = reinterpret_cast<float*>(sm + OFF_C);    // [8 half blocks][128]
    float cg[8][4];
    {
        float run[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const float4 x = *reinterpret_cast<const float4*>(gs + (rbase + j) * kD + ch0);
            const bool ok = rbase + j < L;   // rows past the document do not decay
            run[0] += ok ? x.x : 0.f;
            run[1] += ok ? x.y : 0.f;
            run[2] += ok ? x.z : 0.f;
            run[3] += ok ? x.w : 0.f;
#pragma unroll
            for (int i = 0; i < 4; ++i) cg[j][i] = run[i];
        }
        *reinterpret_cast<float4*>(hsum + rb8 * kD + ch0) =
            make_float4(run[0], run[1], run[2], run[3]);
    }
    __syncthreads();
    float gend[4] = {0.f, 0.f, 0.f, 0.f}, goff[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int hb = 0; hb < 8; ++hb) {
        const float4 x = *reinterpret_cast<const float4*>(hsum + hb * kD + ch0);
        const float xs[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            gend[i] += xs[i];
            if (hb < rb8) goff[i] += xs[i];
        }
    }
    // this thread's Gamma rows back into the tile; its K+, Q+ and K_end elements (K+
    // staged in the free part of C until the log g tile under K+'s tile is read)
    uint8_t* kp_stage = sm + OFF_C + 4096;
    {
        __nv_bfloat16* qplus = wq + ((size_t)rec * 128 + 64) * kD + ch0;
        __nv_bfloat16* kend = ke + (size_t)rec * kC * kD + ch0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int r = rbase + j;
            const bool ok = r < L;
            float G4[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) G4[i] = goff[i] + cg[j][i];
            *reinterpret_cast<float4*>(gsw + r * kD + ch0) =
                make_float4(G4[0], G4[1], G4[2], G4[3]);
            const uint2 kv = ok ? *reinterpret_cast<const uint2*>(sm + OFF_R + toff(128, rb8, j))
                                : make_uint2(0u, 0u);
            const uint2 qv = ok ? *reinterpret_cast<const uint2*>(sm + OFF_R + toff(128, rb8 + 8, j))
                                : make_uint2(0u, 0u);
            const float2 k01 = unpack_bf16(kv.x), k23 = unpack_bf16(kv.y);
            const float2 q01 = unpack_bf16(qv.x), q23 = unpack_bf16(qv.y);
            const float kk[4] = {k01.x, k01.y, k23.x, k23.y};
            const float qq[4] = {q01.x, q01.y, q23.x, q23.y};
            float e[4], eb[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                e[i] = __expf(G4[i]);
                eb[i] = __expf(gend[i] - G4[i]);
            }
            *reinterpret_cast<uint2*>(kp_stage + toff(64, rb8, j)) =
                make_uint2(pack_bf16(kk[0] * e[0], kk[1] * e[1]),
                           pack_bf16(kk[2] * e[2], kk[3] * e[3]));
            *reinterpret_cast<uint2*>(qplus + (size_t)r * kD) =
                make_uint2(pack_bf16(qq[0] * e[0], qq[1] * e[1]),
                           pack_bf16(qq[2] * e[2], qq[3] * e[3]));
            *reinterpret_cast<uint2*>(kend + (size_t)r * kD) =
                make_uint2(pack_bf16(kk[0] * eb[0], kk[1] * eb[1]),
                           pack_bf16(kk[2] * eb[2], kk[3] * eb[3]));
        }
    }
    __syncthreads();
    // A_kk, A_qk: thread (R4, I4) sums the 4 x 4 block of rows 4 R4.., columns 4 I4..
    // over the key channels (each thread starts at its own channel offset, so that the
    // Gamma and k loads of a warp spread over the banks)
    const int R4 = tid >> 4, I4 = tid & 15;
    float akk[4][4], aqk[4][4];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) akk[a][b] = aqk[a][b] = 0.f;
    if (I4 <= R4) {
#pragma unroll 1
        for (int cc = 0; cc < kD; ++cc) {
            const int c = (cc + 2 * I4) & (kD - 1);
            float Gr[4], Gi[4], kr[4], qr[4], ki[4];
#pragma unroll
            for (int a = 0; a < 4; ++a) {
                const int r = 4 * R4 + a, i = 4 * I4 + a;
                Gr[a] = gsw[r * kD + c];
                Gi[a] = gsw[i * kD + c];
                kr[a] = __bfloat162float(
                    *reinterpret_cast<const __nv_bfloat16*>(sm + OFF_R + sw128_off(128, r, c)));
                qr[a] = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(
                    sm + OFF_R + sw128_off(128, 64 + r, c)));
                ki[a] = __bfloat162float(
                    *reinterpret_cast<const __nv_bfloat16*>(sm + OFF_R + sw128_off(128, i, c)));
            }
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int b = 0; b < 4; ++b) {
                    const float e = __expf(fminf(Gr[a] - Gi[b], 0.f)) * ki[b];
                    akk[a][b] = fmaf(kr[a], e, akk[a][b]);
                    aqk[a][b] = fmaf(qr[a], e, aqk[a][b]);
                }
        }
    }
    // A_qk (i <= r) in rows 64 + r of [0; A_qk], zeros above the diagonal
#pragma unroll
    for (int a = 0; a < 4; ++a) {
        const int r = 4 * R4 + a;
        float x[4];
#pragma unroll
        for (int b = 0; b < 4; ++b) x[b] = 4 * I4 + b <= r ? aqk[a][b] : 0.f;
        st_bf16x4(sm + OFF_ZA + sw128_off(128, 64 + r, 4 * I4), x[0], x[1], x[2], x[3]);
    }
    __syncthreads();   // k, q and Gamma fully read: R and the log g tile may be reused
    {
        float* Lb = reinterpret_cast<float*>(sm + OFF_LB);
#pragma unroll
        for (int a = 0; a < 4; ++a) {
            const int r = 4 * R4 + a;
            const float br = beta_s[r];
            float x[4];
#pragma unroll
            for (int b = 0; b < 4; ++b) x[b] = 4 * I4 + b < r ? br * akk[a][b] : 0.f;
            *reinterpret_cast<float4*>(Lb + r * kLdl + 4 * I4) =
                make_float4(x[0], x[1], x[2], x[3]);
        }
#pragma unroll
        for (int j = 0; j < 8; ++j)
            *reinterpret_cast<uint2*>(sm + OFF_KP + toff(64, rb8, j)) =
                *reinterpret_cast<const uint2*>(kp_stage + toff(64, rb8, j));
    }
}

__global__ void __launch_bounds__(kThreads, 2)
intra_kernel(const __grid_constant__ IntraMaps maps, const IntraArgs args) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
    const uint32_t sb = smem_u32(sm);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int qd = warp & 3, hf = warp >> 2;          // TMEM lane quarter, column half
    const int H = args.H;

    // Records are claimed one at a time from a counter shared by the launch's CTAs, so that a CTA
    // that starts late (its SM busy with another kernel) takes fewer records instead of
    // finishing last. Index idx < total names record (g, head): for packed documents g = idx / H;
    // for equal-length sequences idx runs over (sequence, chunk in this launch's span, head).
    const long long total = args.cu ? args.G * H : (long long)args.N * args.c_span * H;
    auto decode = [&](long long idx, Unit& u) -> bool {
        // q = idx / H, and for equal-length sequences sequence sq, chunk-in-span cr = q / c_span,
        // q % c_span: 32-bit divisions whenever the launch's indices fit (a 64-bit division is a
        // long software sequence, and every thread decodes each record)
        long long q, sq = 0, cr = 0;
        if (total <= 0x7fffffffLL) {
            const uint32_t i32 = (uint32_t)idx, h32 = (uint32_t)H, q32 = i32 / h32;
            u.h = (int)(i32 - q32 * h32);
            q = q32;
            if (!args.cu) {
                const uint32_t cs = (uint32_t)args.c_span, s32 = q32 / cs;
                sq = s32;
                cr = q32 - s32 * cs;
            }
        } else {
            u.h = (int)(idx % H);
            q = idx / H;
            if (!args.cu) {
                sq = q / args.c_span;
                cr = q % args.c_span;
            }
        }
        if (args.cu) {
            const long long g = q;
            u.rec = idx;
            const int d = args.map[g];
            if (d < 0 || d >= args.N) return false;
            const long long a = args.cu[d], b = args.cu[d + 1];
            if (b <= a || a < 0 || b > args.T) return false;   // reported by the map kernel
            const long long cc = g - d - a / kC;
            if (cc < 0 || a + kC * cc >= b) return false;
            u.row0 = a + kC * cc;
            u.L = (int)min((long long)kC, b - u.row0);
        } else {
            const long long cc = args.c_begin + cr;
            u.rec = (sq * args.ncT + cc) * H + u.h;
            u.row0 = sq * args.T + kC * cc;
            u.L = (int)min((long long)kC, (long long)args.T - kC * cc);
        }
        return true;
    };
    // next valid record of the launch, or -1 (called by one thread)
    auto claim = [&]() -> long long {
        for (;;) {
            const long long idx = (long long)atomicAdd(args.counter, 1ull);
            if (idx >= total) return -1;
            Unit u;
            if (decode(idx, u)) return idx;
        }
    };
    long long* claim_s = reinterpret_cast<long long*>(sm + OFF_CLAIM);
    Unit cur;

    float* beta_s = reinterpret_cast<float*>(sm + OFF_BETA);
    float* loup_s = reinterpret_cast<float*>(sm + OFF_LOUP);
    uint32_t* tmem_s = reinterpret_cast<uint32_t*>(sm + OFF_TMEM);
    const uint32_t bar_v = sb + OFF_BAR, bar_mma = bar_v + 8, bar_wy2 = bar_v + 16;
    const uint32_t bar_never = bar_v + 24, bar_in = bar_v + 32;
    // lane 0 of the last warp issues copies and the [W; Q~] stores; warps 5 and 6 the others
    const int copier = kThreads - 32;

    if (tid == 0) {
        mbar_init(bar_v, 1);
        mbar_init(bar_mma, 1);
        mbar_init(bar_wy2, 1);
        mbar_init(bar_never, 1);
        mbar_init(bar_in, 1);
        fence_mbar_init();
    }
    if (tid == copier) {
        claim_s[0] = claim();
        prefetch_tmap(&maps.q);
        prefetch_tmap(&maps.k);
        prefetch_tmap(&maps.g);
        prefetch_tmap(&maps.v);
        prefetch_tmap(&maps.w);
        prefetch_tmap(&maps.ut);
        prefetch_tmap(&maps.aq);
    }
    if (warp == 0) {
        tmem_alloc(smem_u32(tmem_s), kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_s;
    const uint32_t lane_q = (uint32_t)(32 * qd) << 16;   // this warp's TMEM lane quarter
    bool has_cur = claim_s[0] >= 0 && decode(claim_s[0], cur);

    auto issue_v = [&](const Unit& u) {
        mbar_arrive_expect_tx(bar_v, kTxV);
        tma_load_3d(sb + OFF_V, &maps.v, bar_v, 0, u.h, (int)u.row0);
        tma_load_3d(sb + OFF_V + 8192, &maps.v, bar_v, 64, u.h, (int)u.row0);
    };
    // q and k land where R's k rows (0-63) and q rows (64-127) go, one 64-column panel per box,
    // so that each thread overwrites its own elements with k rho and q rho; log g lands in the
    // K+ / V region, which it leaves before K+ and V are written
    auto issue_in = [&](const Unit& u) {
        const int row0 = (int)u.row0;
        mbar_arrive_expect_tx(bar_in, kTxIn);
        tma_load_3d(sb + OFF_R, &maps.k, bar_in, 0, u.h, row0);
        tma_load_3d(sb + OFF_R + 16384, &maps.k, bar_in, 64, u.h, row0);
        tma_load_3d(sb + OFF_R + 8192, &maps.q, bar_in, 0, u.h, row0);
        tma_load_3d(sb + OFF_R + 16384 + 8192, &maps.q, bar_in, 64, u.h, row0);
        tma_load_3d(sb + OFF_G, &maps.g, bar_in, 0, u.h, row0);
    };
    auto prefetch_inputs = [&](const Unit& u) {
        const int row0 = (int)u.row0;
        tma_prefetch_3d(&maps.q, 0, u.h, row0);
        tma_prefetch_3d(&maps.q, 64, u.h, row0);
        tma_prefetch_3d(&maps.k, 0, u.h, row0);
        tma_prefetch_3d(&maps.k, 64, u.h, row0);
        tma_prefetch_3d(&maps.g, 0, u.h, row0);
        tma_prefetch_3d(&maps.v, 0, u.h, row0);
        tma_prefetch_3d(&maps.v, 64, u.h, row0);
    };

    // constant parts of the shared-memory descriptors (the start address is added per MMA)
    const uint64_t dK = sw128_desc(0, 16, 1024);     // K-major, 128B swizzle
    const uint64_t dM8 = sw128_desc(0, 8192, 1024);  // MN-major, 128B swizzle, 64-row panels

    bool v_pending = false, mma_pending = false, wy2_pending = false, stores_pending = false;
    bool in_pending = false;
    int v_count = 0, wy2_count = 0, in_count = 0;
    uint32_t mma_phase = 0;
    bool aborted = false;
    // One thread polls; the rest of the CTA waits at the barrier that publishes the outcome.
    auto wait_all = [&](uint32_t bar, uint32_t parity) -> bool {
        const bool ok = tid != 0 || mbar_wait_sleep(bar, parity, args.budget);
        return __syncthreads_or(!ok) == 0;
    };

    if (has_cur && tid == copier) prefetch_inputs(cur);
    // Failure injection (KDA_DEBUG_STALL_WAIT): a wait on a barrier that nothing signals must
    // expire, report KDA_ERR_TIMEOUT and wind down cleanly.
    if (args.debug_stall && !wait_all(bar_never, 0)) aborted = true;

    // elementwise thread mapping: 16-row block pb, half hh (rows 0-7 / 8-15), channels ch0..+3
    const int pb = warp >> 1, hh = warp & 1;
    const int ch0 = 4 * lane;
    const int rbase = 16 * pb + 8 * hh;
    const int rb8 = 2 * pb + hh;
    const uint32_t lh4 = (uint32_t)(((lane & 15) >> 1) << 4);   // 16-byte chunk within a row
    const uint32_t lo8 = (uint32_t)((lane & 1) * 8);
    // byte offset of (row 8*rb + j, channels ch0..ch0+3) in a 128-column tile of R rows
    auto toff = [&](int R, int rb, int j) -> uint32_t {
        return (uint32_t)((lane >> 4) * R * 128 + rb * 1024 + j * 128) + (lh4 ^ (uint32_t)(j << 4)) +
               lo8;
    };
    const float* gs = reinterpret_cast<const float*>(sm + OFF_G);

    for (int c = 0; has_cur && !aborted; ++c) {
        const long long row0 = cur.row0;
        const int L = cur.L;
        const int h = cur.h;
        const long long rec = cur.rec;

        // inputs of this record: the previous record's products have completed (K+ / V region
        // free) and, after the wait below, its stores have read the staging tiles (R/C region)
        if (stores_pending) {
            if (tid == copier || tid == kThreads - 64 || tid == kThreads - 96) bulk_wait_read_all();
            __syncthreads();
            stores_pending = false;
        }
        if (tid == copier) {
            issue_in(cur);
            const long long nx = claim();   // the record after this one, published by parity
            claim_s[(c + 1) & 1] = nx;
            Unit ahead;
            if (nx >= 0 && decode(nx, ahead)) prefetch_inputs(ahead);
        }
        in_pending = true;
        if (tid < kC)
            beta_s[tid] = tid < L ? __bfloat162float(args.beta[(row0 + tid) * H + h]) : 0.f;
        if (!wait_all(bar_in, in_count & 1)) { aborted = true; break; }
        ++in_count;
        in_pending = false;

        // ---------------------------------------------------------------- decay products
        // With a_t = e^{log g_t} over this thread's 8 rows: the lower half (hh = 0) keeps the
        // suffix products y_j = prod_{t > j} a_t, the upper half the prefix products
        // y_j = prod_{t <= j} a_t; tot = prod over all 8 rows. The other product of each row is
        // tot / y_j, formed below from the reciprocal that the operands need anyway.
        // (This kernel is bound partly by instruction fetch: one copy of each phase, with
        // selects where the half or the row mask differs, runs faster than copies specialised
        // per half or for full chunks.)
        float y[8][4], tot[4];
        bool range_bad = false;
        {
            float a[8][4];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const float4 g = *reinterpret_cast<const float4*>(gs + (rbase + j) * kD + ch0);
                const bool ok = rbase + j < L;   // rows past the document: a = 1
                a[j][0] = ok ? __expf(g.x) : 1.f;
                a[j][1] = ok ? __expf(g.y) : 1.f;
                a[j][2] = ok ? __expf(g.z) : 1.f;
                a[j][3] = ok ? __expf(g.w) : 1.f;
            }
            // The anchored factors invert these running products; they stay finite while every
            // product is >= 1e-30. The products only shrink, so the first suffix (lower half) or
            // the last prefix (upper half) is the smallest. A chunk with a steeper decay anywhere
            // takes the direct path (steep_chunk) instead.
            if (hh == 0) {
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    float run = 1.f;
#pragma unroll
                    for (int j = 7; j >= 0; --j) {
                        y[j][i] = run;
                        run *= a[j][i];
                    }
                    tot[i] = run;
                    range_bad |= y[0][i] < 1e-30f;
                }
            } else {
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    float run = 1.f;
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        run *= a[j][i];
                        y[j][i] = run;
                    }
                    tot[i] = run;
                    range_bad |= y[7][i] < 1e-30f;
                }
            }
        }
        *reinterpret_cast<float4*>(loup_s + rb8 * kD + ch0) =
            make_float4(tot[0], tot[1], tot[2], tot[3]);
        const bool steep = __syncthreads_or(range_bad || args.force_direct) != 0;
        // log g consumed (unless steep): the K+ / V region is free for V and K+
        if (!steep) {
            if (tid == copier) issue_v(cur);
            v_pending = true;
        }
        // half totals of every block: Lo_b (rows 0-7), Up_b (rows 8-15), P_b = Lo_b Up_b.
        // F = prod_{b < pb} P_b, G = prod_{b > pb} P_b; XA[a] = Lo_a prod_{pb < b < a} P_b carries
        // a column of this block to the middle of a later block a; own = Up_pb (lower half) or
        // Lo_pb (upper half). pb is the same for a whole warp: each warp runs only its block's
        // case, with no per-block predication.
        float4 F, G, XA[3];
        const float4 own = ld4(loup_s + (rb8 ^ 1) * kD + ch0);
        {
            float4 P[4];
#pragma unroll
            for (int bb = 0; bb < 4; ++bb)
                P[bb] = mul4(ld4(loup_s + (2 * bb) * kD + ch0), ld4(loup_s + (2 * bb + 1) * kD + ch0));
            auto setup = [&](auto pb_c) {
                constexpr int PB = decltype(pb_c)::value;
                F = G = make_float4(1.f, 1.f, 1.f, 1.f);
#pragma unroll
                for (int bb = 0; bb < PB; ++bb) F = mul4(F, P[bb]);
#pragma unroll
                for (int bb = PB + 1; bb < 4; ++bb) G = mul4(G, P[bb]);
                float4 between = make_float4(1.f, 1.f, 1.f, 1.f);
#pragma unroll
                for (int aa = PB + 1; aa < 4; ++aa) {
                    XA[aa - 1] = mul4(ld4(loup_s + (2 * aa) * kD + ch0), between);
                    between = mul4(between, P[aa]);
                }
            };
            switch (pb) {
                case 0: setup(std::integral_constant<int, 0>{}); break;
                case 1: setup(std::integral_constant<int, 1>{}); break;
                case 2: setup(std::integral_constant<int, 2>{}); break;
                default: setup(std::integral_constant<int, 3>{}); break;
            }
            if (warp == 0)
                *reinterpret_cast<float4*>(args.decay + rec * kD + ch0) =
                    mul4(mul4(P[0], P[1]), mul4(P[2], P[3]));
        }

        // ---------------------------------------------------------------- operands
        //   R: k rho, q rho (rho_r = e^{Gamma_r - Gamma_m}, m the middle of r's block)
        //   C: k kappa (kappa = e^{Gamma_m - Gamma_r}), cross columns k sigma X_a, X_a <= 1
        //   K+ = k e^{Gamma} (shared), Q+ = q e^{Gamma} and K_end = k e^{Gamma_end - Gamma} =
        //   k G sigma (workspace)
        // Per row, with yi = 1 / y_j:
        //   lower half: rho = yi, kappa = y_j, sigma = y_j own, e^{Gamma} = F tot yi
        //   upper half: rho = y_j, kappa = yi, sigma = tot yi, e^{Gamma} = F own y_j
        // so that sigma = kappa sf and e^{Gamma} = cE rho, with sf = own (lower) or tot (upper)
        // and cE = F tot (lower) or F own (upper). R, C and K_end take fp32 products of k rho,
        // q rho, k kappa; K+ and Q+ are the bf16 products of the rounded k rho, q rho with cE
        // (one bf16x2 multiply per two elements: the extra rounding does not move the result
        // measurably, where rounding the factors of R, C or K_end would).
        if (!steep) {
            __nv_bfloat16* qplus = args.wq + ((size_t)rec * 128 + 64) * kD + ch0;
            __nv_bfloat16* kend = args.ke + (size_t)rec * kC * kD + ch0;
            {
                const bool kUpper = hh != 0;
                const float totv[4] = {tot[0], tot[1], tot[2], tot[3]};
                const float4 sf4 = kUpper ? make_float4(totv[0], totv[1], totv[2], totv[3]) : own;
                const float4 cE4 = kUpper ? mul4(F, own) : mul4(F, make_float4(totv[0], totv[1],
                                                                                totv[2], totv[3]));
                const float4 gf4 = mul4(G, sf4);
                const float gf[4] = {gf4.x, gf4.y, gf4.z, gf4.w};
                float xa[3][4];
#pragma unroll
                for (int aa = 0; aa < 3; ++aa) {
                    const float4 x = mul4(XA[aa], sf4);
                    xa[aa][0] = x.x; xa[aa][1] = x.y; xa[aa][2] = x.z; xa[aa][3] = x.w;
                }
                const __nv_bfloat162 cE01 = __floats2bfloat162_rn(cE4.x, cE4.y);
                const __nv_bfloat162 cE23 = __floats2bfloat162_rn(cE4.z, cE4.w);
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int r = rbase + j;
                    const bool ok = r < L;   // rows past the document read as k = q = 0
                    const uint2 kv = ok ? *reinterpret_cast<const uint2*>(sm + OFF_R + toff(128, rb8, j))
                                        : make_uint2(0u, 0u);
                    const uint2 qv = ok ? *reinterpret_cast<const uint2*>(sm + OFF_R + toff(128, rb8 + 8, j))
                                        : make_uint2(0u, 0u);
                    const float2 k01 = unpack_bf16(kv.x), k23 = unpack_bf16(kv.y);
                    const float2 q01 = unpack_bf16(qv.x), q23 = unpack_bf16(qv.y);
                    const float kk[4] = {k01.x, k01.y, k23.x, k23.y};
                    const float qq[4] = {q01.x, q01.y, q23.x, q23.y};
                    float kr[4], qr[4], kc[4];   // k rho, q rho, k kappa
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const float yv = y[j][i];
                        const float yi = __fdividef(1.f, yv);
                        const float rho = kUpper ? yv : yi;
                        const float kap = kUpper ? yi : yv;
                        kr[i] = kk[i] * rho;
                        qr[i] = qq[i] * rho;
                        kc[i] = kk[i] * kap;
                    }
                    const uint2 krb = make_uint2(pack_bf16(kr[0], kr[1]), pack_bf16(kr[2], kr[3]));
                    const uint2 qrb = make_uint2(pack_bf16(qr[0], qr[1]), pack_bf16(qr[2], qr[3]));
                    *reinterpret_cast<uint2*>(sm + OFF_R + toff(128, rb8, j)) = krb;
                    *reinterpret_cast<uint2*>(sm + OFF_R + toff(128, rb8 + 8, j)) = qrb;
                    st_bf16x4(sm + OFF_C + toff(160, rb8, j), kc[0], kc[1], kc[2], kc[3]);
#pragma unroll
                    for (int aa = 1; aa < 4; ++aa) {
                        if (aa <= pb) continue;
                        const float* x = xa[aa - 1];   // sf X_a
                        st_bf16x4(sm + OFF_C + toff(160, rb8 + 8 + cross_off(aa) / 8, j),
                                  kc[0] * x[0], kc[1] * x[1], kc[2] * x[2], kc[3] * x[3]);
                    }
                    *reinterpret_cast<uint2*>(sm + OFF_KP + toff(64, rb8, j)) =
                        make_uint2(hmul2_u32(krb.x, cE01), hmul2_u32(krb.y, cE23));
                    *reinterpret_cast<uint2*>(qplus + (size_t)r * kD) =
                        make_uint2(hmul2_u32(qrb.x, cE01), hmul2_u32(qrb.y, cE23));
                    *reinterpret_cast<uint2*>(kend + (size_t)r * kD) =
                        make_uint2(pack_bf16(kc[0] * gf[0], kc[1] * gf[1]),
                                   pack_bf16(kc[2] * gf[2], kc[3] * gf[3]));
                }
            }
        }
        if (!steep) {
        fence_proxy_async();
        __syncthreads();

        // ---------------------------------------------------------------- MMA: R C^T
        if (warp == 0) {   // the whole warp runs the issue code; one elected lane issues
            tc_fence_after();
            const uint32_t id = idesc_bf16(128, 160, 0, 0);
#pragma unroll
            for (int s = 0; s < kD / 16; ++s) {
                const int k0 = 16 * s;
                const uint64_t ad = desc_at(dK, sb + OFF_R + (k0 >> 6) * 16384 + (k0 & 63) * 2);
                const uint64_t bd = desc_at(dK, sb + OFF_C + (k0 >> 6) * 20480 + (k0 & 63) * 2);
                umma_f16_warp(tbase + TM_A, ad, bd, id, s > 0);
            }
            umma_commit_warp(bar_mma);
        }
        mma_pending = true;

        // ---------------------------------------------------------------- assemble A_kk, A_qk
        if (!wait_all(bar_mma, mma_phase & 1)) { aborted = true; break; }
        ++mma_phase;
        mma_pending = false;
        tc_fence_after();
        {
            float* Lb = reinterpret_cast<float*>(sm + OFF_LB);
            const bool is_q = qd >= 2;
            const int r = 32 * (qd & 1) + lane;
            const int a = r >> 4;
            const float br = beta_s[r];
            // write 16 consecutive entries (i0 .. i0+15) of row r
            auto put16 = [&](int i0, const float* x) {
                if (is_q) {
                    st_bf16x8(sm + OFF_ZA + sw128_off(128, 64 + r, i0), x);
                    st_bf16x8(sm + OFF_ZA + sw128_off(128, 64 + r, i0 + 8), x + 8);
                } else {
                    float4* dst = reinterpret_cast<float4*>(Lb + r * kLdl + i0);
#pragma unroll
                    for (int m = 0; m < 4; ++m)
                        dst[m] = make_float4(br * x[4 * m], br * x[4 * m + 1], br * x[4 * m + 2],
                                             br * x[4 * m + 3]);
                }
            };
            if (hf == 0) {
                // this row's diagonal block, masked to i < r (A_kk) or i <= r (A_qk)
                float v[32];
                tmem_ld32(tbase + lane_q + TM_A + 32 * (qd & 1), v);
                tmem_ld_wait();
                float x[16];
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const int i = 16 * a + j;
                    const float val = (a & 1) ? v[16 + j] : v[j];
                    x[j] = (is_q ? i <= r : i < r) ? val : 0.f;
                }
                put16(16 * a, x);
                if (is_q) {   // A_qk is lower triangular: zero the blocks after the diagonal one
                    const uint4 z = make_uint4(0, 0, 0, 0);
                    for (int i = 16 * (a + 1); i < kC; i += 8)
                        *reinterpret_cast<uint4*>(sm + OFF_ZA + sw128_off(128, 64 + r, i)) = z;
                }
            } else if ((qd & 1) == 0) {
                float w[16];
                tmem_ld16(tbase + lane_q + TM_A + 64 + cross_off(1), w);   // block 1: i in 0..15
                tmem_ld_wait();
                if (a == 1) put16(0, w);
            } else {
                // rows of blocks 2 and 3: all three loads in flight before one wait
                float v2[32], v3[32], w[16];
                tmem_ld32(tbase + lane_q + TM_A + 64 + cross_off(2), v2);        // block 2: i 0..31
                tmem_ld32(tbase + lane_q + TM_A + 64 + cross_off(3), v3);        // block 3: i 0..31
                tmem_ld16(tbase + lane_q + TM_A + 64 + cross_off(3) + 32, w);   // i in 32..47
                tmem_ld_wait();
                if (a == 2) {
                    put16(0, v2);
                    put16(16, v2 + 16);
                } else {
                    put16(0, v3);
                    put16(16, v3 + 16);
                    put16(32, w);
                }
            }
        }
        } else {
            // ------------------------------------------------------------ steep decay: direct
            steep_chunk(sm, L, rec, args.wq, args.ke);
            if (tid == copier) issue_v(cur);
            v_pending = true;
        }
        fence_proxy_async();
        tc_fence_before();
        __syncthreads();
        // A_qk (rows 64-127 of [0; A_qk]) is final: store it while the UT transform runs
        if (tid == kThreads - 96) {
            tma_store_2d(&maps.aq, sb + OFF_ZA + 8192, 0, (int)(rec * 64));
            bulk_commit();
        }
        stores_pending = true;

        // ---------------------------------------------------------------- UT transform
        {
            const float* Lb = reinterpret_cast<const float*>(sm + OFF_LB);
            float* Mb = reinterpret_cast<float*>(sm + OFF_MB);
            // diagonal 16x16 blocks of (I + L)^-1: forward substitution for column j of block bk,
            // x_k = [k = j] - sum_{m<k} L[k][m] x_m, by four threads: part t keeps the running
            // sums of rows t, t + 4, t + 8, t + 12 and the owner of row k broadcasts x_k to the
            // other three. L is zero on and above the diagonal of its diagonal blocks, so every
            // row takes every update.
            {
                const int bk = tid >> 6, j = (tid >> 2) & 15, t = tid & 3;
                const int base = 16 * bk;
                const int src0 = lane & ~3;
                float lr[4][16];
#pragma unroll
                for (int ii = 0; ii < 4; ++ii)
#pragma unroll
                    for (int m = 0; m < 4; ++m) {
                        const float4 x = *reinterpret_cast<const float4*>(
                            Lb + (base + t + 4 * ii) * kLdl + base + 4 * m);
                        lr[ii][4 * m] = x.x;
                        lr[ii][4 * m + 1] = x.y;
                        lr[ii][4 * m + 2] = x.z;
                        lr[ii][4 * m + 3] = x.w;
                    }
                float acc[4] = {0.f, 0.f, 0.f, 0.f}, xo[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int k = 0; k < 16; ++k) {
                    const int own = k & 3, kk = k >> 2;
                    float xk = (k == j ? 1.f : 0.f) - acc[kk];   // meaningful on the owner only
                    xk = __shfl_sync(0xffffffffu, xk, src0 + own);
                    if (t == own) xo[kk] = xk;
#pragma unroll
                    for (int ii = 0; ii < 4; ++ii) acc[ii] = fmaf(lr[ii][k], xk, acc[ii]);
                }
#pragma unroll
                for (int ii = 0; ii < 4; ++ii) Mb[(base + t + 4 * ii) * kLdm + base + j] = xo[ii];
            }
            __syncthreads();
            // off-diagonal blocks of M = (I + L)^-1 (tf32 mma.sync, one warp per 16x16 block).
            //   level 1:  M_{b+1,b} = -M_{b+1,b+1} L_{b+1,b} M_bb
            //   level 2:  the lower-left 32x32 block, M[32:, :32] = -M[32:, 32:] L[32:, :32] M[:32, :32],
            //             as Y = L[32:, :32] M[:32, :32] (four blocks) and then -M[32:, 32:] Y
            //             (blocks (2,0), (3,0), (3,1); (2,1) is known from level 1)
            const int g = lane >> 2, t = lane & 3;
            float* ysb = reinterpret_cast<float*>(sm + OFF_YS);
            // acc += A[0:16, 0:K] B[0:K, 0:16] for fp32 row-major sources
            auto mm16 = [&](float (&acc)[2][4], const float* A, int lda, const float* B, int ldb,
                            int K) {
                for (int kk = 0; kk < K; kk += 8) {
                    const float* la = A + g * lda + kk + t;
                    const uint32_t a[4] = {f2tf(la[0]), f2tf(la[8 * lda]), f2tf(la[4]),
                                           f2tf(la[8 * lda + 4])};
#pragma unroll
                    for (int nt = 0; nt < 2; ++nt) {
                        const float* lb = B + (kk + t) * ldb + 8 * nt + g;
                        const uint32_t b[2] = {f2tf(lb[0]), f2tf(lb[4 * ldb])};
                        mma_tf32_16x8x8(acc[nt], a, b);
                    }
                }
            };
            auto st16 = [&](float* dst, int ld, const float (&z)[2][4], float sign) {
#pragma unroll
                for (int nt = 0; nt < 2; ++nt) {
                    dst[g * ld + 8 * nt + 2 * t] = sign * z[nt][0];
                    dst[g * ld + 8 * nt + 2 * t + 1] = sign * z[nt][1];
                    dst[(g + 8) * ld + 8 * nt + 2 * t] = sign * z[nt][2];
                    dst[(g + 8) * ld + 8 * nt + 2 * t + 1] = sign * z[nt][3];
                }
            };
            if (warp < 3) {
                const int bb = warp, aa = warp + 1;
                float* ys = ysb + warp * 16 * 17;
                float yy[2][4] = {}, z[2][4] = {};
                mm16(yy, Lb + 16 * aa * kLdl + 16 * bb, kLdl, Mb + 16 * bb * kLdm + 16 * bb, kLdm, 16);
                st16(ys, 17, yy, 1.f);
                __syncwarp();
                mm16(z, Mb + 16 * aa * kLdm + 16 * aa, kLdm, ys, 17, 16);
                st16(Mb + 16 * aa * kLdm + 16 * bb, kLdm, z, -1.f);
            }
            __syncthreads();
            if (warp < 4) {   // Y_{ra,cb} = sum over k-blocks cb..1 of L_{ra,k} M_{k,cb}
                const int ra = 2 + (warp >> 1), cb = warp & 1;
                float yy[2][4] = {};
                mm16(yy, Lb + 16 * ra * kLdl + 16 * cb, kLdl, Mb + 16 * cb * kLdm + 16 * cb, kLdm,
                     32 - 16 * cb);
                st16(ysb + warp * 16 * 17, 17, yy, 1.f);   // Y_{2,cb} in slot cb, Y_{3,cb} in 2 + cb
            }
            __syncthreads();
            if (warp < 3) {   // warp 0: M_20 = -M_22 Y_20;  warps 1, 2: M_3c = -(M_32 Y_2c + M_33 Y_3c)
                const int cb = warp == 2 ? 1 : 0;
                float z[2][4] = {};
                if (warp == 0) {
                    mm16(z, Mb + 32 * kLdm + 32, kLdm, ysb, 17, 16);
                    st16(Mb + 32 * kLdm, kLdm, z, -1.f);
                } else {
                    mm16(z, Mb + 48 * kLdm + 32, kLdm, ysb + cb * 16 * 17, 17, 16);
                    mm16(z, Mb + 48 * kLdm + 48, kLdm, ysb + (2 + cb) * 16 * 17, 17, 16);
                    st16(Mb + 48 * kLdm + 16 * cb, kLdm, z, -1.f);
                }
            }
            __syncthreads();
            // T = (I + L)^-1 diag(beta): lower triangle, bf16 K-major
            {
                const int i = 2 * lane;
                const float b0 = beta_s[i], b1 = beta_s[i + 1];
#pragma unroll
                for (int rr8 = 0; rr8 < 8; ++rr8) {
                    const int r = 8 * warp + rr8;
                    const float2 m = *reinterpret_cast<const float2*>(Mb + r * kLdm + i);
                    const float x0 = (i <= r) ? m.x * b0 : 0.f;
                    const float x1 = (i + 1 <= r) ? m.y * b1 : 0.f;
                    *reinterpret_cast<uint32_t*>(sm + OFF_TT + sw128_off(128, r, i)) =
                        pack_bf16(x0, x1);
                }
            }
        }
        fence_proxy_async();
        __syncthreads();

        // ---------------------------------------------------------------- MMA: WY products
        // [T; -] K+ (lanes 0-63: W; rows 64-127 of the A operand are never read out) and,
        // transposed for the state pass, V^T T^T (lane j = value column: U~^T in columns
        // 128-191)
        if (!wait_all(bar_v, v_count & 1)) { aborted = true; break; }
        ++v_count;
        v_pending = false;
        if (warp == 0) {
            tc_fence_after();
            const uint32_t id = idesc_bf16(128, 128, 0, 1);
            const uint32_t idt = idesc_bf16(128, 64, 1, 0);
#pragma unroll
            for (int s = 0; s < kC / 16; ++s)
                umma_f16_warp(tbase + TM_A, desc_at(dK, sb + OFF_TT + 32 * s),
                              desc_at(dM8, sb + OFF_KP + 2048 * s), id, s > 0);
            umma_commit_warp(bar_mma);   // W: read out while the next product runs
#pragma unroll
            for (int s = 0; s < kC / 16; ++s)
                umma_f16_warp(tbase + TM_A + 128, desc_at(dM8, sb + OFF_V + 2048 * s),
                              desc_at(dK, sb + OFF_TT + 32 * s), idt, s > 0);
            umma_commit_warp(bar_wy2);
        }
        mma_pending = wy2_pending = true;
        if (!wait_all(bar_mma, mma_phase & 1)) { aborted = true; break; }
        ++mma_phase;
        mma_pending = false;
        tc_fence_after();
        if (qd < 2) {
            // W rows r = 32 qd + lane (TMEM lanes 0-63); each warp takes 64 of the 128 columns
            const int r = 32 * qd + lane;
#pragma unroll
            for (int part = 0; part < 2; ++part) {
                const int c0 = 64 * hf + 32 * part;
                float v[32];
                tmem_ld32(tbase + lane_q + TM_A + c0, v);
                tmem_ld_wait();
#pragma unroll
                for (int m = 0; m < 4; ++m)
                    st_bf16x8(sm + OFF_SW + sw128_off(64, r, c0 + 8 * m), v + 8 * m);
            }
        }
        if (!wait_all(bar_wy2, wy2_count & 1)) { aborted = true; break; }
        ++wy2_count;
        wy2_pending = false;
        tc_fence_after();
        {
            // U~^T (TMEM columns 128-191), lane j = value column, into the bf16 staging tile
            // [128 j][64 tokens] (128-byte swizzle); each warp takes 32 of the 64 tokens
            const int jrow = 32 * qd + lane;
            float v[32];
            tmem_ld32(tbase + lane_q + TM_A + 128 + 32 * hf, v);
            tmem_ld_wait();
#pragma unroll
            for (int m = 0; m < 4; ++m)
                st_bf16x8(sm + OFF_SUT + sw128_off(128, jrow, 32 * hf + 8 * m), v + 8 * m);
        }
        // shared staging tiles before the async-proxy stores
        fence_proxy_async();
        tc_fence_before();
        __syncthreads();
        {
            if (tid == copier) {
                tma_store_2d(&maps.w, sb + OFF_SW, 0, (int)(rec * 128));
                tma_store_2d(&maps.w, sb + OFF_SW + 8192, 64, (int)(rec * 128));
                bulk_commit();
            } else if (tid == kThreads - 64) {
                tma_store_2d(&maps.ut, sb + OFF_SUT, 0, (int)(rec * 128));
                bulk_commit();
            }
            stores_pending = true;
        }
        {
            const long long nx = claim_s[(c + 1) & 1];   // written at this record's start
            has_cur = nx >= 0 && decode(nx, cur);
        }
    }

    if (aborted) {
        if (tid == 0) set_device_error(args.err, DEV_TIMEOUT);
        // wind down: let this CTA's own copies and MMAs finish before TMEM and smem go away
        const long long drain = 1ll << 31;
        if (in_pending && tid == 0) mbar_wait(bar_in, in_count & 1, drain);
        if (v_pending && tid == 0) mbar_wait(bar_v, v_count & 1, drain);
        if (mma_pending && tid == 0) mbar_wait(bar_mma, mma_phase & 1, drain);
        if (wy2_pending && tid == 0) mbar_wait(bar_wy2, wy2_count & 1, drain);
    }
    if (tid == copier || tid == kThreads - 64 || tid == kThreads - 96)
        bulk_wait_all();   // stores complete before the smem goes away
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tbase, kTmemCols);
}

// ------------------------------------------------------------------ host side

// [rows, H, 128] row-major tensor, one head's 64-row tile per box of box_inner columns
cudaError_t make_rows_map(CUtensorMap* m, const void* base, CUtensorMapDataType dt,
                          int elem_bytes, long long rows, int H, int box_inner,
                          CUtensorMapSwizzle sw) {
    return make_map_3d_box(m, base, dt, elem_bytes, (unsigned long long)rows, H, kD, box_inner,
                           kC, sw);
}

long long wait_budget() {
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

int debug_stall() {
    static int v = [] {
        const char* s = std::getenv("KDA_DEBUG_STALL_WAIT");
        return (s && *s && *s != '0') ? 1 : 0;
    }();
    return v;
}

// KDA_DEBUG_FORCE_DIRECT=1 (read once per process): every chunk takes the steep-decay path, so
// that tests can check that path against the oracle on ordinary inputs.
int force_direct() {
    static int v = [] {
        const char* s = std::getenv("KDA_DEBUG_FORCE_DIRECT");
        return (s && *s && *s != '0') ? 1 : 0;
    }();
    return v;
}

// resident CTAs of intra_kernel across the GPU: as many per SM as its registers and shared
// memory allow (two on B200), by the SM's own limits and by the runtime's occupancy query,
// whichever is larger. A CTA beyond the resident count would only start later, never wait on
// another, so an overestimate costs time, not correctness.
cudaError_t intra_grid_cap(int* cap) {
    static PerDevice once;
    static int value[PerDevice::kMax];
    int dev = 0;
    const cudaError_t err = once.run(
        [](int d) {
            cudaError_t e = cudaFuncSetAttribute(
                intra_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
            if (e != cudaSuccess) return e;
            e = cudaFuncSetAttribute(intra_kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                                     (int)cudaSharedmemCarveoutMaxShared);
            if (e != cudaSuccess) return e;
            int sms = 0, smem_sm = 0, smem_rsv = 0, regs_sm = 0, per_sm = 0;
            cudaFuncAttributes fa;
            if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, d)) !=
                    cudaSuccess ||
                (e = cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor,
                                            d)) != cudaSuccess ||
                (e = cudaDeviceGetAttribute(&smem_rsv, cudaDevAttrReservedSharedMemoryPerBlock,
                                            d)) != cudaSuccess ||
                (e = cudaDeviceGetAttribute(&regs_sm, cudaDevAttrMaxRegistersPerMultiprocessor,
                                            d)) != cudaSuccess ||
                (e = cudaFuncGetAttributes(&fa, intra_kernel)) != cudaSuccess ||
                (e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, intra_kernel, kThreads,
                                                                   kSmemBytes)) != cudaSuccess)
                return e;
            const int by_smem = smem_sm / ((int)kSmemBytes + fa.sharedSizeBytes + smem_rsv);
            const int by_regs = fa.numRegs > 0 ? regs_sm / (fa.numRegs * kThreads) : 1;
            int fit = by_smem < by_regs ? by_smem : by_regs;
            if (fit > 2) fit = 2;   // __launch_bounds__ sizes the kernel for two
            if (per_sm < fit) per_sm = fit;
            value[d] = sms * (per_sm > 0 ? per_sm : 1);
            return cudaSuccess;
        },
        &dev);
    *cap = err == cudaSuccess ? value[dev] : 0;
    return err;
}

}  // namespace

cudaError_t launch_chunk64_intra(const FwdParams& p, int c_begin, int c_span,
                                 unsigned long long* counter, cudaStream_t stream) {
    const SplitWorkspace& ws = *p.split;
    cudaError_t e = tma_encoder_ready();
    if (e != cudaSuccess) return e;
    const long long rows = (long long)p.B * p.T;
    const long long items = p.cu_seqlens ? ws.G * p.H : (long long)p.N * c_span * p.H;
    if (items == 0 || rows <= 0) return cudaSuccess;
    if (ws.G * p.H * 128 > 0x7fffffffLL || rows > 0x7fffffffLL)
        return cudaErrorInvalidConfiguration;
    const auto BF = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    const auto F32 = CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
    const auto SWN = CU_TENSOR_MAP_SWIZZLE_NONE;
    const auto SW = CU_TENSOR_MAP_SWIZZLE_128B;
    IntraMaps m;
    const unsigned long long R = (unsigned long long)(ws.G * p.H);
    if ((e = make_rows_map(&m.q, p.q, BF, 2, rows, p.H, 64, SW)) != cudaSuccess ||
        (e = make_rows_map(&m.k, p.k, BF, 2, rows, p.H, 64, SW)) != cudaSuccess ||
        (e = make_rows_map(&m.g, p.log_g, F32, 4, rows, p.H, kD, SWN)) != cudaSuccess ||
        (e = make_rows_map(&m.v, p.v, BF, 2, rows, p.H, 64, SW)) != cudaSuccess ||
        (e = make_map_2d(&m.w, ws.wq, BF, 2, R * 128, kD, 64, 64, SW)) != cudaSuccess ||
        (e = make_map_2d(&m.ut, ws.ut, BF, 2, R * 128, kC, 64, 128, SW)) != cudaSuccess ||
        (e = make_map_2d(&m.aq, ws.aq, BF, 2, R * 64, kC, 64, 64, SW)) != cudaSuccess)
        return e;
    int cap = 0;
    if ((e = intra_grid_cap(&cap)) != cudaSuccess) return e;
    IntraArgs a;
    memset(&a, 0, sizeof(a));
    a.q = static_cast<const __nv_bfloat16*>(p.q);
    a.k = static_cast<const __nv_bfloat16*>(p.k);
    a.g = p.log_g;
    a.beta = static_cast<const __nv_bfloat16*>(p.beta);
    a.cu = p.cu_seqlens;
    a.map = ws.map;
    a.wq = ws.wq;
    a.ke = ws.ke;
    a.decay = ws.decay;
    a.G = ws.G;
    a.ncT = ws.ncT;
    a.c_begin = c_begin;
    a.c_span = c_span;
    a.counter = counter;
    a.T = p.T;
    a.H = p.H;
    a.N = p.N;
    a.budget = wait_budget();
    a.debug_stall = debug_stall();
    a.force_direct = force_direct();
    a.err = p.err;
    const long long grid = items < cap ? items : cap;
    intra_kernel<<<(unsigned)grid, kThreads, kSmemBytes, stream>>>(m, a);
    return cudaGetLastError();
}

}  // namespace kda
