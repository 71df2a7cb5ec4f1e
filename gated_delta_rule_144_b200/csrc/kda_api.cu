// C ABI of libkda.so: argument validation, path selection and the device error word.
// Declarations and the contract of every entry point are in include/kda.h.

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "kda.h"

#include "kda_bwd.cuh"
#include "kda_internal.cuh"
#include "kda_scan.cuh"

namespace {

// Sticky device error word (one per device context; see kda_get_device_error).
__device__ unsigned g_device_error = 0;

thread_local char t_last_error[512] = "";

kda_status_t fail(kda_status_t st, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(t_last_error, sizeof(t_last_error), fmt, ap);
    va_end(ap);
    return st;
}

kda_status_t cuda_fail(cudaError_t e, const char* what) {
    return fail(KDA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

constexpr int kMaxDevices = 64;
unsigned* g_err_addr[kMaxDevices] = {};
std::mutex g_err_mu;

// Device address of the error word on the current device (looked up once per device).
kda_status_t device_error_word(unsigned** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= kMaxDevices) return fail(KDA_ERR_UNSUPPORTED, "device %d", dev);
    std::lock_guard<std::mutex> lock(g_err_mu);
    if (!g_err_addr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_device_error);
        if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(error word)");
        g_err_addr[dev] = static_cast<unsigned*>(p);
    }
    *out = g_err_addr[dev];
    return KDA_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

kda_status_t check_ptr(const void* p, const char* name, bool required) {
    if (!p) return required ? fail(KDA_ERR_INVALID_ARG, "%s is NULL", name) : KDA_OK;
    if (!aligned16(p)) return fail(KDA_ERR_INVALID_ARG, "%s is not 16-byte aligned", name);
    return KDA_OK;
}

enum class Path { kPerToken, kChunk64 };

kda_status_t check_fwd_desc(const kda_fwd_desc_t* d, bool has_cu, Path* path) {
    if (!d) return fail(KDA_ERR_INVALID_ARG, "desc is NULL");
    if (d->B < 1 || d->T < 0 || d->H < 1 || d->dk < 1 || d->dv < 1 || d->num_seqs < 0)
        return fail(KDA_ERR_INVALID_ARG, "bad sizes B=%d T=%d H=%d dk=%d dv=%d N=%d", d->B, d->T,
                    d->H, d->dk, d->dv, d->num_seqs);
    if (d->dtype != KDA_F32 && d->dtype != KDA_BF16)
        return fail(KDA_ERR_INVALID_ARG, "unknown dtype %d", (int)d->dtype);
    if (has_cu) {
        if (d->B != 1) return fail(KDA_ERR_INVALID_ARG, "cu_seqlens requires B == 1");
    } else if (d->num_seqs != d->B) {
        return fail(KDA_ERR_INVALID_ARG, "num_seqs (%d) must equal B (%d) without cu_seqlens",
                    d->num_seqs, d->B);
    }
    if ((int64_t)d->B * d->T * d->H > (int64_t)1 << 40)
        return fail(KDA_ERR_INVALID_ARG, "problem too large");
    const bool tc_shape =
        d->dtype == KDA_BF16 && d->dk == 128 && d->dv == 128 && kda::chunk64_available();
    switch (d->chunk_size) {
        case KDA_CHUNK_AUTO:
            *path = tc_shape ? Path::kChunk64 : Path::kPerToken;
            break;
        case KDA_CHUNK_PER_TOKEN:
            *path = Path::kPerToken;
            break;
        case KDA_CHUNK_64:
            if (d->dtype == KDA_F32) {
                *path = Path::kPerToken;  // fp32 inputs always take the exact path
                break;
            }
            if (!tc_shape)
                return fail(KDA_ERR_UNSUPPORTED,
                            "chunk_size 64 needs bf16 with dk = dv = 128 (and the chunked kernel)");
            *path = Path::kChunk64;
            break;
        default:
            if (d->dtype == KDA_F32 && d->chunk_size > 0) {
                *path = Path::kPerToken;
                break;
            }
            return fail(KDA_ERR_UNSUPPORTED, "chunk_size %d", d->chunk_size);
    }
    if (*path == Path::kPerToken && (d->dk > 256 || d->dv > 256))
        return fail(KDA_ERR_UNSUPPORTED, "per-token path supports dk, dv <= 256");
    return KDA_OK;
}

}  // namespace

namespace kda {
void set_last_error(const char* msg) {
    snprintf(t_last_error, sizeof(t_last_error), "%s", msg);
}
}  // namespace kda

extern "C" {

int kda_version(void) { return 100; }

const char* kda_last_error(void) { return t_last_error; }

const char* kda_status_string(kda_status_t s) {
    switch (s) {
        case KDA_OK: return "ok";
        case KDA_ERR_INVALID_ARG: return "invalid argument";
        case KDA_ERR_UNSUPPORTED: return "unsupported configuration";
        case KDA_ERR_CUDA: return "CUDA runtime error";
        case KDA_ERR_TIMEOUT: return "device pipeline wait timed out";
        case KDA_ERR_BAD_SEQLENS: return "malformed cu_seqlens";
        case KDA_ERR_RANGE: return "decay out of range (reserved; no longer raised)";
    }
    return "unknown status";
}

// Segments of at least 32 chunks, at most 12, and one segment up to 64 chunks. Measured on one
// B200 (L2 flushed before each call): the long-context workload (1024 chunks per sequence, 64
// chains) takes 3.84, 3.89, 3.63, 3.71, 3.65 ms at 1, 4, 8, 12, 16 segments; the single-sequence
// one (64 chunks, 16 chains) 0.154, 0.178, 0.170, 0.168 ms at 1, 2, 3, 4: the next segment's
// intra-chunk launch takes the SMs before a short state pass can start, so a short chain gains no
// overlap and pays the side stream's joins.
// KDA_SPLIT_SEGMENTS (1-16, read per call) overrides the count, capped at the chunk count; the
// result is the same whatever the count (the state crosses segments in fp32).
static int split_segments(int ncT) {
    int s = ncT <= 64 ? 1 : ncT / 32;
    if (s > 12) s = 12;
    if (const char* env = std::getenv("KDA_SPLIT_SEGMENTS")) {
        const int v = std::atoi(env);
        if (v >= 1) s = v;
    }
    if (s > kda::kMaxSegments) s = kda::kMaxSegments;
    return s > ncT ? (ncT > 0 ? ncT : 1) : s;
}

// Two-level state pass for equal-length sequences with few chains (the sequential chunk chain,
// one SM per chain, would leave most SMs idle): P segments of m chunks, P >= 3, or 1 for the
// plain pass. Phases (one SM per unit): the state pass of segment 0 from h0 (with its outputs),
// beside the transition maps A_p and zero-start states B_p of segments 1 .. P-2 (2 (P-2) units per
// chain, no outputs); then S_{p+1} = A_p S_p + B_p in fp32 (P - 2 steps of a 128 x 128 x 128
// product per chain); then segments 1 .. P-1 at once from their initial states. P minimises a
// cost model in units of one chunk of the state pass (about 1.6 us on B200): the intra-chunk
// kernel (about 3.7 units of SM time per record, all SMs), then the phases, each ceil(units /
// 148) waves of m chunks, plus 2.5 units per combine step and 4 for the launches; the plain pass is
// intra-chunk kernel + chain (one segment) or the larger of the two (chunk segments overlapping).
// The two-level pass is used when it models at least 15 % faster. Measured on one B200 (L2
// flushed, ms per call at P = plain, 3, 4, 5, 6, 7, 8, 10): 1 x 4096 tokens x 16 heads 0.158,
// 0.147, 0.133, 0.129, 0.127, 0.144, 0.139, 0.141 (the model picks 6); 1 x 16384 x 16 0.543,
// 0.440, 0.381, 0.354, 0.336, 0.373, 0.359, 0.354 (picks 6); 1 x 8192 x 8 0.260, 0.205, 0.176,
// 0.162, 0.155, 0.150, 0.145, 0.143 (picks 10). KDA_SCAN_SEGMENTS (read per
// call) overrides: 0 or 1 = the plain pass, 3 .. 32 = that many segments (capped by the chunks).
static int scan_segments(int ncT, long long chains) {
    if (ncT < 3 || chains <= 0 || chains > 148) return 1;
    auto effective = [&](int P) {   // segments of ceil(ncT / P) chunks, none empty
        const int m = (ncT + P - 1) / P;
        return (ncT + m - 1) / m;
    };
    if (const char* env = std::getenv("KDA_SCAN_SEGMENTS")) {
        int v = std::atoi(env);
        if (v < 3) return 1;
        if (v > kda::kMaxScanSegments) v = kda::kMaxScanSegments;
        if (v > ncT) v = ncT;
        v = effective(v);
        return v >= 3 ? v : 1;
    }
    const double sms = 148.0, ch = (double)chains;
    const double intra = (double)ncT * ch * 3.7 / sms;
    const int S = split_segments(ncT);
    const double plain = S == 1 ? intra + ncT
                                : std::max(intra * sms / (sms - std::min(ch, 74.0)), (double)ncT);
    double best = 0.85 * plain;
    int bestP = 1;
    for (int P = 3; P <= std::min(ncT, kda::kMaxScanSegments); ++P) {
        if (effective(P) != P) continue;
        const int m = (ncT + P - 1) / P;
        const double w1 = std::ceil((2.0 * (P - 2) + 1.0) * ch / sms);
        const double w3 = std::ceil((P - 1.0) * ch / sms);
        const double cost = intra + (w1 + w3) * m + 2.5 * (P - 2) + 4.0;
        if (cost < best) best = cost, bestP = P;
    }
    return bestP;
}

int kda_fwd_algorithm(const kda_fwd_desc_t* desc, int has_cu_seqlens) {
    Path path;
    const kda_status_t st = check_fwd_desc(desc, has_cu_seqlens != 0, &path);
    if (st != KDA_OK) return -(int)st;
    return path == Path::kChunk64 ? KDA_CHUNK_64 : KDA_CHUNK_PER_TOKEN;
}

int kda_fwd_split_segments(const kda_fwd_desc_t* desc, int has_cu_seqlens) {
    Path path;
    const kda_status_t st = check_fwd_desc(desc, has_cu_seqlens != 0, &path);
    if (st != KDA_OK) return -(int)st;
    if (path != Path::kChunk64 || has_cu_seqlens || desc->T <= 0) return 1;
    const int ncT = (desc->T + 63) / 64;
    if (scan_segments(ncT, (long long)desc->num_seqs * desc->H) >= 3) return 1;
    return split_segments(ncT);
}

int kda_fwd_scan_segments(const kda_fwd_desc_t* desc, int has_cu_seqlens) {
    Path path;
    const kda_status_t st = check_fwd_desc(desc, has_cu_seqlens != 0, &path);
    if (st != KDA_OK) return -(int)st;
    if (path != Path::kChunk64 || has_cu_seqlens || desc->T <= 0) return 1;
    return scan_segments((desc->T + 63) / 64, (long long)desc->num_seqs * desc->H);
}

// Packed documents on the chunked path are scheduled longest first; the permutation lives in the
// caller's workspace (one int32 per document). Nothing else needs scratch.
static size_t order_bytes(const kda_fwd_desc_t* d, Path path) {
    const bool packed = d->B == 1 && d->num_seqs >= 2;  // without cu_seqlens num_seqs == B
    if (path != Path::kChunk64 || !packed || d->num_seqs > kda::kMaxOrderedDocs) return 0;
    return ((size_t)d->num_seqs * sizeof(int32_t) + 255) / 256 * 256;
}

// Workspace of the split chunked path (intra-chunk kernel + state pass), 256-byte aligned parts.
struct SplitLayout {
    size_t order, map, counters, state, decay, wq, ke, ut, aq, total;
    size_t maps, total_pscan;   // two-level state pass: its states, and the workspace it needs
    long long G;
    int ncT;
    int P;                      // segments of the two-level state pass (1: the plain pass)
    bool has_order;
};

static size_t up256(size_t x) { return (x + 255) / 256 * 256; }

// packed: the call passes cu_seqlens (records are indexed floor(t0 / 64) + document + chunk).
static bool split_layout(const kda_fwd_desc_t* d, Path path, bool packed, SplitLayout* L) {
    if (path != Path::kChunk64 || d->T <= 0 || d->num_seqs <= 0) return false;
    L->ncT = (d->T + 63) / 64;
    L->G = packed ? (long long)L->ncT + d->num_seqs : (long long)d->B * L->ncT;
    const long long R = L->G * d->H;
    if (R * 128 > 0x7fffffffLL) return false;   // TMA row coordinates are 32-bit
    L->has_order = packed && d->num_seqs >= 2 && d->num_seqs <= kda::kMaxOrderedDocs;
    size_t off = 0;
    L->order = off; off += L->has_order ? up256((size_t)d->num_seqs * 4) : 0;
    L->map = off;   off += packed ? up256((size_t)L->G * 4) : 0;
    L->counters = off; off += up256((size_t)kda::kMaxSegments * 8);
    // state between chunk segments (equal-length sequences): N x H fp32 128 x 128
    L->state = off; off += packed ? 0 : (size_t)d->num_seqs * d->H * 65536;
    L->decay = off; off += up256((size_t)R * 512);
    L->wq = off;    off += (size_t)R * 32768;
    L->ke = off;    off += (size_t)R * 16384;
    L->ut = off;    off += (size_t)R * 16384;
    L->aq = off;    off += (size_t)R * 8192;
    L->total = off;
    // two-level state pass: A_p and B_p of segments 1 .. P-2, then the initial states of
    // segments 1 .. P-1, each N x H fp32 128 x 128
    L->P = packed ? 1 : scan_segments(L->ncT, (long long)d->num_seqs * d->H);
    L->maps = off;
    if (L->P >= 3) off += (size_t)(3 * L->P - 5) * d->num_seqs * d->H * 65536;
    L->total_pscan = off;
    return true;
}

size_t kda_fwd_workspace_size(const kda_fwd_desc_t* desc) {
    Path path;
    const bool maybe_packed = desc && desc->B == 1;
    if (!desc || check_fwd_desc(desc, maybe_packed && desc->num_seqs >= 2, &path) != KDA_OK)
        return 0;
    t_last_error[0] = 0;
    SplitLayout L;
    // B == 1 may come with cu_seqlens: size for the packed record numbering (one record more
    // per document than a single sequence needs), or for the two-level state pass without them
    if (split_layout(desc, path, maybe_packed, &L)) {
        size_t t = L.total_pscan;
        SplitLayout U;
        if (maybe_packed && split_layout(desc, path, false, &U)) t = std::max(t, U.total_pscan);
        return t;
    }
    return order_bytes(desc, path);
}

size_t kda_fwd_workspace_size_min(const kda_fwd_desc_t* desc) {
    Path path;
    if (!desc || check_fwd_desc(desc, desc->B == 1 && desc->num_seqs >= 2, &path) != KDA_OK)
        return 0;
    t_last_error[0] = 0;
    return order_bytes(desc, path);
}

// Chunk segments of the split path for equal-length sequences with ncT chunks each: the state
// pass of segment s (one CTA per chain, so at most N x H SMs) runs on a side stream while the
// intra-chunk kernel works on segment s + 1 with the other SMs. Short sequences run in one.
// Side stream (highest priority, so that its state-pass CTAs take SMs first when both kernels are
// ready) and events, one set per host thread and device: concurrent calls from several host
// threads never share events.
struct SideStream {
    cudaStream_t aux = nullptr;
    cudaEvent_t join = nullptr;
    cudaEvent_t seg[kda::kMaxSegments] = {};
};
static thread_local SideStream t_side[kMaxDevices];

static cudaError_t side_stream(SideStream** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    SideStream& ss = t_side[dev];
    if (!ss.aux) {
        int least = 0, greatest = 0;
        if ((e = cudaDeviceGetStreamPriorityRange(&least, &greatest)) != cudaSuccess) return e;
        cudaStream_t aux;
        if ((e = cudaStreamCreateWithPriority(&aux, cudaStreamNonBlocking, greatest)) !=
            cudaSuccess)
            return e;
        if ((e = cudaEventCreateWithFlags(&ss.join, cudaEventDisableTiming)) != cudaSuccess)
            return e;
        for (int i = 0; i < kda::kMaxSegments; ++i)
            if ((e = cudaEventCreateWithFlags(&ss.seg[i], cudaEventDisableTiming)) != cudaSuccess)
                return e;
        ss.aux = aux;
    }
    *out = &ss;
    return cudaSuccess;
}

// kda_fwd with an optional gated RMSNorm epilogue (norm == nullptr: none).
static kda_status_t fwd_impl(const kda_fwd_desc_t* d, const void* q, const void* k,
                             const void* v, const float* log_g, const void* beta,
                             const float* h0, const int32_t* cu_seqlens, void* o, float* hT,
                             void* workspace, size_t workspace_bytes,
                             const kda_out_norm_t* norm, kda_stream_t stream) {
    t_last_error[0] = 0;
    Path path;
    kda_status_t st = check_fwd_desc(d, cu_seqlens != nullptr, &path);
    if (st != KDA_OK) return st;
    const bool tokens = (int64_t)d->B * d->T > 0;
    const bool has_units = d->num_seqs > 0;
    if ((st = check_ptr(q, "q", tokens)) || (st = check_ptr(k, "k", tokens)) ||
        (st = check_ptr(v, "v", tokens)) || (st = check_ptr(log_g, "log_g", tokens)) ||
        (st = check_ptr(beta, "beta", false)) || (st = check_ptr(o, "o", tokens)) ||
        (st = check_ptr(h0, "h0", false)) || (st = check_ptr(hT, "hT", false)) ||
        (st = check_ptr(cu_seqlens, "cu_seqlens", false)))
        return st;
    if (tokens && !beta) return fail(KDA_ERR_INVALID_ARG, "beta is NULL");
    if (norm) {
        if ((st = check_ptr(norm->gate, "norm gate", tokens)) ||
            (st = check_ptr(norm->weight, "norm weight", tokens)))
            return st;
        if (!(norm->eps >= 0.f)) return fail(KDA_ERR_INVALID_ARG, "norm eps must be >= 0");
    }
    SplitLayout L;
    const bool split = tokens && split_layout(d, path, cu_seqlens != nullptr, &L) && workspace &&
                       aligned16(workspace) && workspace_bytes >= L.total;
    // the two-level state pass when the plan has one and the workspace holds its states
    const bool pscan = split && !cu_seqlens && L.P >= 3 && workspace_bytes >= L.total_pscan;
    const size_t need_ws = (cu_seqlens && !split) ? order_bytes(d, path) : 0;
    if (need_ws > 0 && (workspace_bytes < need_ws || !workspace || !aligned16(workspace)))
        return fail(KDA_ERR_INVALID_ARG,
                    "workspace must be a 16-byte aligned device buffer of %zu bytes "
                    "(kda_fwd_workspace_size)", need_ws);
    if (!has_units) return KDA_OK;

    kda::FwdParams p{};
    p.q = q; p.k = k; p.v = v; p.log_g = log_g; p.beta = beta; p.h0 = h0;
    p.cu_seqlens = cu_seqlens; p.o = o; p.hT = hT;
    p.B = d->B; p.T = d->T; p.H = d->H; p.dk = d->dk; p.dv = d->dv; p.N = d->num_seqs;
    p.bf16 = d->dtype == KDA_BF16;
    p.doc_order = nullptr;
    if ((st = device_error_word(&p.err)) != KDA_OK) return st;
    // the epilogue: on the split path the state pass's epilogue warps apply it to the fp32 o as
    // they store it; the other paths run it as one bandwidth-bound pass over o afterwards
    auto norm_after = [&]() -> cudaError_t {
        if (!norm || !tokens) return cudaSuccess;
        return kda::launch_out_norm_gated(o, norm->gate, norm->weight, norm->eps, o,
                                          (long long)d->B * d->T * d->H, d->dv, p.bf16,
                                          reinterpret_cast<cudaStream_t>(stream));
    };
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = cudaSuccess;
    if (split) {
        uint8_t* w = static_cast<uint8_t*>(workspace);
        kda::SplitWorkspace ws;
        ws.wq = reinterpret_cast<__nv_bfloat16*>(w + L.wq);
        ws.ke = reinterpret_cast<__nv_bfloat16*>(w + L.ke);
        ws.ut = reinterpret_cast<__nv_bfloat16*>(w + L.ut);
        ws.aq = reinterpret_cast<__nv_bfloat16*>(w + L.aq);
        ws.decay = reinterpret_cast<float*>(w + L.decay);
        ws.map = cu_seqlens ? reinterpret_cast<int32_t*>(w + L.map) : nullptr;
        ws.counters = reinterpret_cast<unsigned long long*>(w + L.counters);
        ws.state = cu_seqlens ? nullptr : reinterpret_cast<float*>(w + L.state);
        ws.G = L.G;
        ws.ncT = L.ncT;
        p.split = &ws;
        if (L.has_order) {
            int32_t* order = reinterpret_cast<int32_t*>(w + L.order);
            e = kda::launch_doc_order(cu_seqlens, d->num_seqs, order, s);
            if (e != cudaSuccess) return cuda_fail(e, "kda_fwd document scheduling");
            p.doc_order = order;
        }
        if (cu_seqlens) {
            e = kda::launch_chunk_map(cu_seqlens, d->num_seqs, d->T, L.G, ws.map, p.err, s);
            if (e != cudaSuccess) return cuda_fail(e, "kda_fwd chunk map");
        }
        kda::ScanNorm sn{};
        const kda::ScanNorm* snp = nullptr;
        if (norm) {
            sn.gate = norm->gate;
            sn.weight = norm->weight;
            sn.eps = norm->eps;
            snp = &sn;
        }
        const int S = cu_seqlens || pscan ? 1 : split_segments(L.ncT);
        e = cudaMemsetAsync(ws.counters, 0, sizeof(unsigned long long) * S, s);
        if (e != cudaSuccess) return cuda_fail(e, "kda_fwd workspace counters");
        if (pscan) {
            // intra-chunk kernel over every chunk; then segment 0 (side stream) beside the maps
            // of segments 1 .. P-2 (caller's stream); the segments' initial states; then
            // segments 1 .. P-1 at once
            const int P = L.P, m = (L.ncT + P - 1) / P;
            const size_t states = (size_t)d->num_seqs * d->H * 16384;   // floats per state set
            float* maps = reinterpret_cast<float*>(w + L.maps);         // A: [P-2], B: [P-2]
            float* sinit = maps + 2 * (size_t)(P - 2) * states;          // [P-1]
            SideStream* ss = nullptr;
            if ((e = side_stream(&ss)) != cudaSuccess) return cuda_fail(e, "kda_fwd side stream");
            e = kda::launch_chunk64_intra(p, 0, L.ncT, ws.counters, s);
            if (e != cudaSuccess) return cuda_fail(e, "kda_fwd intra-chunk launch");
            const kda::ScanSegment seg0{0, m, h0, sinit};
            const kda::ScanSegment mid{0, 0, nullptr, maps};
            kda::ScanSplit mid_split;
            mid_split.seg_m = m;
            mid_split.seg_p0 = 1;
            mid_split.seg_count = P - 2;
            mid_split.groups = 2;
            mid_split.nseg = P;
            mid_split.ident = true;
            mid_split.no_out = true;
            const kda::ScanSegment rest{0, 0, sinit, hT};
            kda::ScanSplit rest_split;
            rest_split.seg_m = m;
            rest_split.seg_p0 = 1;
            rest_split.seg_count = P - 1;
            rest_split.nseg = P;
            rest_split.hT_last = true;
            cudaError_t first = cudaSuccess;
            if ((first = cudaEventRecord(ss->seg[0], s)) == cudaSuccess &&
                (first = cudaStreamWaitEvent(ss->aux, ss->seg[0], 0)) == cudaSuccess &&
                (first = kda::launch_chunk_scan(p, seg0, ss->aux, snp)) == cudaSuccess)
                first = kda::launch_chunk_scan_split(p, mid, mid_split, s);
            // join even after a failed launch, so that nothing is left pending on the side stream
            e = cudaEventRecord(ss->join, ss->aux);
            if (e == cudaSuccess) e = cudaStreamWaitEvent(s, ss->join, 0);
            if (first != cudaSuccess) return cuda_fail(first, "kda_fwd state-pass launch");
            if (e != cudaSuccess) return cuda_fail(e, "kda_fwd side stream join");
            e = kda::launch_scan_combine(maps, maps + (size_t)(P - 2) * states, sinit,
                                         d->num_seqs * d->H, P - 2, s);
            if (e != cudaSuccess) return cuda_fail(e, "kda_fwd segment-state launch");
            e = kda::launch_chunk_scan_split(p, rest, rest_split, s, snp);
            if (e != cudaSuccess) return cuda_fail(e, "kda_fwd state-pass launch");
        } else if (S == 1) {
            e = kda::launch_chunk64_intra(p, 0, L.ncT, ws.counters, s);
            if (e != cudaSuccess) return cuda_fail(e, "kda_fwd intra-chunk launch");
            e = kda::launch_chunk_scan(p, kda::ScanSegment{0, L.ncT, h0, hT}, s, snp);
            if (e != cudaSuccess) return cuda_fail(e, "kda_fwd state-pass launch");
        } else {
            // intra(0) intra(1) ... on the caller's stream; state(i) on the side stream after
            // intra(i) and state(i - 1); the caller's stream then waits for the last state pass
            SideStream* ss = nullptr;
            if ((e = side_stream(&ss)) != cudaSuccess) return cuda_fail(e, "kda_fwd side stream");
            cudaError_t first = cudaSuccess;
            for (int i = 0; i < S && first == cudaSuccess; ++i) {
                const int cb = (int)((long long)L.ncT * i / S);
                const int ce = (int)((long long)L.ncT * (i + 1) / S);
                const kda::ScanSegment seg{cb, ce, i == 0 ? h0 : ws.state,
                                           i == S - 1 ? hT : ws.state};
                if ((e = kda::launch_chunk64_intra(p, cb, ce - cb, ws.counters + i, s)) !=
                        cudaSuccess ||
                    (e = cudaEventRecord(ss->seg[i], s)) != cudaSuccess ||
                    (e = cudaStreamWaitEvent(ss->aux, ss->seg[i], 0)) != cudaSuccess ||
                    (e = kda::launch_chunk_scan(p, seg, ss->aux, snp)) != cudaSuccess)
                    first = e;
            }
            // join even after a failed launch, so that nothing is left pending on the side stream
            e = cudaEventRecord(ss->join, ss->aux);
            if (e == cudaSuccess) e = cudaStreamWaitEvent(s, ss->join, 0);
            if (first != cudaSuccess) return cuda_fail(first, "kda_fwd split launch");
            if (e != cudaSuccess) return cuda_fail(e, "kda_fwd side stream join");
        }
        return KDA_OK;
    }
    if (need_ws > 0 && tokens) {
        int32_t* order = static_cast<int32_t*>(workspace);
        e = kda::launch_doc_order(cu_seqlens, d->num_seqs, order, s);
        if (e != cudaSuccess) return cuda_fail(e, "kda_fwd document scheduling");
        p.doc_order = order;
    }
    e = path == Path::kChunk64 ? kda::launch_chunk64(p, s) : kda::launch_recurrent(p, s);
    if (e != cudaSuccess) return cuda_fail(e, "kda_fwd launch");
    e = norm_after();
    if (e != cudaSuccess) return cuda_fail(e, "kda_fwd output norm launch");
    return KDA_OK;
}

kda_status_t kda_fwd(const kda_fwd_desc_t* d, const void* q, const void* k, const void* v,
                     const float* log_g, const void* beta, const float* h0,
                     const int32_t* cu_seqlens, void* o, float* hT, void* workspace,
                     size_t workspace_bytes, kda_stream_t stream) {
    return fwd_impl(d, q, k, v, log_g, beta, h0, cu_seqlens, o, hT, workspace, workspace_bytes,
                    nullptr, stream);
}

kda_status_t kda_fwd_normed(const kda_fwd_desc_t* d, const void* q, const void* k,
                            const void* v, const float* log_g, const void* beta,
                            const float* h0, const int32_t* cu_seqlens,
                            const kda_out_norm_t* norm, void* y, float* hT, void* workspace,
                            size_t workspace_bytes, kda_stream_t stream) {
    if (!norm) {
        t_last_error[0] = 0;
        return fail(KDA_ERR_INVALID_ARG, "norm is NULL");
    }
    if (d && d->dv > 256) {
        t_last_error[0] = 0;
        return fail(KDA_ERR_UNSUPPORTED, "the output norm supports dv <= 256");
    }
    return fwd_impl(d, q, k, v, log_g, beta, h0, cu_seqlens, y, hT, workspace, workspace_bytes,
                    norm, stream);
}

static kda_status_t check_bwd_desc(const kda_fwd_desc_t* d, bool has_cu) {
    Path path;
    kda_status_t st = check_fwd_desc(d, has_cu, &path);
    if (st != KDA_OK) return st;
    if (d->dk != 128 || d->dv != 128)
        return fail(KDA_ERR_UNSUPPORTED, "kda_bwd supports dk = dv = 128 (got %d, %d)", d->dk,
                    d->dv);
    return KDA_OK;
}

size_t kda_bwd_workspace_size(const kda_fwd_desc_t* desc) {
    if (!desc || check_bwd_desc(desc, desc->B == 1 && desc->num_seqs >= 2) != KDA_OK) return 0;
    t_last_error[0] = 0;
    if (desc->T <= 0 || desc->num_seqs <= 0) return 0;
    return kda::bwd_workspace_bytes((long long)desc->num_seqs * desc->H, desc->T);
}

kda_status_t kda_bwd(const kda_fwd_desc_t* d, const void* q, const void* k, const void* v,
                     const float* log_g, const void* beta, const float* h0,
                     const int32_t* cu_seqlens, const void* dout, const float* dhT, float* dq,
                     float* dk, float* dv, float* dlog_g, float* dbeta, float* dh0,
                     void* workspace, size_t workspace_bytes, kda_stream_t stream) {
    t_last_error[0] = 0;
    kda_status_t st = check_bwd_desc(d, cu_seqlens != nullptr);
    if (st != KDA_OK) return st;
    const bool tokens = (int64_t)d->B * d->T > 0;
    if ((st = check_ptr(q, "q", tokens)) || (st = check_ptr(k, "k", tokens)) ||
        (st = check_ptr(v, "v", tokens)) || (st = check_ptr(log_g, "log_g", tokens)) ||
        (st = check_ptr(beta, "beta", false)) || (st = check_ptr(dout, "do", tokens)) ||
        (st = check_ptr(dq, "dq", tokens)) || (st = check_ptr(dk, "dk", tokens)) ||
        (st = check_ptr(dv, "dv", tokens)) || (st = check_ptr(dlog_g, "dlog_g", tokens)) ||
        (st = check_ptr(dbeta, "dbeta", false)) || (st = check_ptr(h0, "h0", false)) ||
        (st = check_ptr(dhT, "dhT", false)) || (st = check_ptr(dh0, "dh0", false)) ||
        (st = check_ptr(cu_seqlens, "cu_seqlens", false)))
        return st;
    if (tokens && (!beta || !dbeta)) return fail(KDA_ERR_INVALID_ARG, "beta or dbeta is NULL");
    const long long chains = (long long)d->num_seqs * d->H;
    const size_t need = (tokens && chains > 0) ? kda::bwd_workspace_bytes(chains, d->T) : 0;
    if (need > 0 && (!workspace || !aligned16(workspace) || workspace_bytes < need))
        return fail(KDA_ERR_INVALID_ARG,
                    "workspace must be a 16-byte aligned device buffer of %zu bytes "
                    "(kda_bwd_workspace_size)", need);
    if (chains == 0) return KDA_OK;
    if (!tokens) {   // no tokens: dh0 = dhT (or zero)
        if (!dh0) return KDA_OK;
        cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
        const size_t bytes = (size_t)chains * 128 * 128 * sizeof(float);
        cudaError_t e = dhT ? cudaMemcpyAsync(dh0, dhT, bytes, cudaMemcpyDeviceToDevice, s)
                            : cudaMemsetAsync(dh0, 0, bytes, s);
        return e == cudaSuccess ? KDA_OK : cuda_fail(e, "kda_bwd dh0");
    }
    kda::BwdParams p{};
    p.q = q; p.k = k; p.v = v; p.beta = beta; p.dout = dout; p.log_g = log_g; p.h0 = h0;
    p.dhT = dhT; p.cu_seqlens = cu_seqlens; p.dq = dq; p.dk = dk; p.dv = dv; p.dlog_g = dlog_g;
    p.dbeta = dbeta; p.dh0 = dh0; p.workspace = workspace;
    p.T = d->T; p.H = d->H; p.N = d->num_seqs;
    p.bf16 = d->dtype == KDA_BF16;
    if ((st = device_error_word(&p.err)) != KDA_OK) return st;
    cudaError_t e = kda::launch_bwd(p, reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "kda_bwd launch");
    return KDA_OK;
}

kda_status_t kda_out_norm_gated(long long vectors, int dv, kda_dtype_t dtype, const void* x,
                                const void* gate, const float* weight, float eps, void* y,
                                kda_stream_t stream) {
    t_last_error[0] = 0;
    if (vectors < 0 || dv < 1) return fail(KDA_ERR_INVALID_ARG, "bad sizes vectors=%lld dv=%d",
                                           vectors, dv);
    if (dv > 256) return fail(KDA_ERR_UNSUPPORTED, "the output norm supports dv <= 256");
    if (dtype != KDA_F32 && dtype != KDA_BF16)
        return fail(KDA_ERR_INVALID_ARG, "unknown dtype %d", (int)dtype);
    if (!(eps >= 0.f)) return fail(KDA_ERR_INVALID_ARG, "eps must be >= 0");
    kda_status_t st;
    const bool any = vectors > 0;
    if ((st = check_ptr(x, "x", any)) || (st = check_ptr(gate, "gate", any)) ||
        (st = check_ptr(weight, "weight", any)) || (st = check_ptr(y, "y", any)))
        return st;
    if (!any) return KDA_OK;
    cudaError_t e = kda::launch_out_norm_gated(x, gate, weight, eps, y, vectors, dv,
                                               dtype == KDA_BF16,
                                               reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "kda_out_norm_gated launch");
    return KDA_OK;
}

kda_status_t kda_short_conv(int B, int T, int C, int W, kda_dtype_t dtype, const void* x,
                            const float* weight, const int32_t* cu_seqlens, int num_seqs,
                            kda_activation_t act, int norm_group, float eps, void* y,
                            kda_stream_t stream) {
    t_last_error[0] = 0;
    if (B < 1 || T < 0 || C < 1 || num_seqs < 0)
        return fail(KDA_ERR_INVALID_ARG, "bad sizes B=%d T=%d C=%d N=%d", B, T, C, num_seqs);
    if (W < 1 || W > 8) return fail(KDA_ERR_UNSUPPORTED, "kernel width %d (1..8)", W);
    if (C % 4) return fail(KDA_ERR_UNSUPPORTED, "C = %d is not a multiple of 4", C);
    if (dtype != KDA_F32 && dtype != KDA_BF16)
        return fail(KDA_ERR_INVALID_ARG, "unknown dtype %d", (int)dtype);
    if (act != KDA_ACT_NONE && act != KDA_ACT_SILU)
        return fail(KDA_ERR_INVALID_ARG, "unknown activation %d", (int)act);
    if (norm_group != 0 && (norm_group < 4 || norm_group > 128 ||
                            (norm_group & (norm_group - 1)) || C % norm_group))
        return fail(KDA_ERR_UNSUPPORTED,
                    "norm_group %d (0, or a power of two from 4 to 128 dividing C)", norm_group);
    if (!(eps >= 0.f)) return fail(KDA_ERR_INVALID_ARG, "eps must be >= 0");
    if (cu_seqlens && B != 1) return fail(KDA_ERR_INVALID_ARG, "cu_seqlens requires B == 1");
    if (cu_seqlens && num_seqs < 1)
        return fail(KDA_ERR_INVALID_ARG, "cu_seqlens needs num_seqs >= 1");
    if ((int64_t)B * T * C > (int64_t)1 << 40) return fail(KDA_ERR_INVALID_ARG, "problem too large");
    kda_status_t st;
    const bool any = (int64_t)B * T > 0;
    if ((st = check_ptr(x, "x", any)) || (st = check_ptr(weight, "weight", any)) ||
        (st = check_ptr(y, "y", any)) || (st = check_ptr(cu_seqlens, "cu_seqlens", false)))
        return st;
    if (!any) return KDA_OK;
    const size_t esz = dtype == KDA_BF16 ? 2 : 4;
    const uintptr_t xb = reinterpret_cast<uintptr_t>(x), yb = reinterpret_cast<uintptr_t>(y);
    const size_t bytes = (size_t)B * T * C * esz;
    if (xb < yb + bytes && yb < xb + bytes)
        return fail(KDA_ERR_INVALID_ARG, "y overlaps x (the window reads earlier rows of x)");
    unsigned* err = nullptr;
    if ((st = device_error_word(&err)) != KDA_OK) return st;
    cudaError_t e = kda::launch_short_conv(x, weight, cu_seqlens, num_seqs, y, B, T, C, W,
                                           dtype == KDA_BF16, (int)act, norm_group, eps, err,
                                           reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "kda_short_conv launch");
    return KDA_OK;
}

kda_status_t kda_decode_step(int N, int H, int dk, int dv, kda_dtype_t dtype, const void* q,
                             const void* k, const void* v, const float* log_g, const void* beta,
                             float* S_inout, void* o, kda_stream_t stream) {
    t_last_error[0] = 0;
    if (N < 0 || H < 1 || dk < 1 || dv < 1)
        return fail(KDA_ERR_INVALID_ARG, "bad sizes N=%d H=%d dk=%d dv=%d", N, H, dk, dv);
    if (dtype != KDA_F32 && dtype != KDA_BF16)
        return fail(KDA_ERR_INVALID_ARG, "unknown dtype %d", (int)dtype);
    if (dk > 256 || dv > 256) return fail(KDA_ERR_UNSUPPORTED, "decode supports dk, dv <= 256");
    kda_status_t st;
    const bool any = N > 0;
    if ((st = check_ptr(q, "q", any)) || (st = check_ptr(k, "k", any)) ||
        (st = check_ptr(v, "v", any)) || (st = check_ptr(log_g, "log_g", any)) ||
        (st = check_ptr(beta, "beta", any)) || (st = check_ptr(S_inout, "S_inout", any)) ||
        (st = check_ptr(o, "o", any)))
        return st;
    if (!any) return KDA_OK;
    unsigned* err = nullptr;
    if ((st = device_error_word(&err)) != KDA_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e;
    if (dk == 128 && dv == 128) {
        kda::DecodeParams p{q, k, v, log_g, beta, S_inout, o, N, H, dk, dv,
                            dtype == KDA_BF16, err};
        e = kda::launch_decode_d128(p, s);
    } else {
        // general sizes: the per-token walk over one token, state read from and written to S
        kda::FwdParams p{};
        p.q = q; p.k = k; p.v = v; p.log_g = log_g; p.beta = beta; p.h0 = S_inout;
        p.cu_seqlens = nullptr; p.o = o; p.hT = S_inout;
        p.B = N; p.T = 1; p.H = H; p.dk = dk; p.dv = dv; p.N = N;
        p.bf16 = dtype == KDA_BF16;
        p.err = err;
        e = kda::launch_recurrent(p, s);
    }
    if (e != cudaSuccess) return cuda_fail(e, "kda_decode_step launch");
    return KDA_OK;
}

kda_status_t kda_decode_tokens(int N, int H, int T, int dk, int dv, kda_dtype_t dtype,
                               const void* q, const void* k, const void* v, const float* log_g,
                               const void* beta, float* S_inout, void* o, kda_stream_t stream) {
    t_last_error[0] = 0;
    if (N < 0 || H < 1 || T < 0 || dk < 1 || dv < 1)
        return fail(KDA_ERR_INVALID_ARG, "bad sizes N=%d H=%d T=%d dk=%d dv=%d", N, H, T, dk,
                    dv);
    if (dtype != KDA_F32 && dtype != KDA_BF16)
        return fail(KDA_ERR_INVALID_ARG, "unknown dtype %d", (int)dtype);
    if (dk > 256 || dv > 256) return fail(KDA_ERR_UNSUPPORTED, "decode supports dk, dv <= 256");
    if ((int64_t)N * T * H > (int64_t)1 << 40) return fail(KDA_ERR_INVALID_ARG, "problem too large");
    kda_status_t st;
    const bool any = N > 0 && T > 0;
    if ((st = check_ptr(q, "q", any)) || (st = check_ptr(k, "k", any)) ||
        (st = check_ptr(v, "v", any)) || (st = check_ptr(log_g, "log_g", any)) ||
        (st = check_ptr(beta, "beta", any)) || (st = check_ptr(S_inout, "S_inout", any)) ||
        (st = check_ptr(o, "o", any)))
        return st;
    if (!any) return KDA_OK;
    unsigned* err = nullptr;
    if ((st = device_error_word(&err)) != KDA_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e;
    if (dk == 128 && dv == 128) {
        kda::DecodeParams p{q, k, v, log_g, beta, S_inout, o, N, H, dk, dv,
                            dtype == KDA_BF16, err};
        e = kda::launch_decode_tokens_d128(p, T, s);
    } else {
        // general sizes: the per-token walk over N sequences of T tokens, state in place
        kda::FwdParams p{};
        p.q = q; p.k = k; p.v = v; p.log_g = log_g; p.beta = beta; p.h0 = S_inout;
        p.cu_seqlens = nullptr; p.o = o; p.hT = S_inout;
        p.B = N; p.T = T; p.H = H; p.dk = dk; p.dv = dv; p.N = N;
        p.bf16 = dtype == KDA_BF16;
        p.err = err;
        e = kda::launch_recurrent(p, s);
    }
    if (e != cudaSuccess) return cuda_fail(e, "kda_decode_tokens launch");
    return KDA_OK;
}

kda_status_t kda_get_device_error(kda_stream_t stream) {
    t_last_error[0] = 0;
    unsigned* err = nullptr;
    kda_status_t st = device_error_word(&err);
    if (st != KDA_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    unsigned host = 0;
    cudaError_t e = cudaMemcpyAsync(&host, err, sizeof(host), cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_fail(e, "reading the device error word");
    if (host != 0) {
        const unsigned zero = 0;
        e = cudaMemcpyAsync(err, &zero, sizeof(zero), cudaMemcpyHostToDevice, s);
        if (e == cudaSuccess) e = cudaStreamSynchronize(s);
        if (e != cudaSuccess) return cuda_fail(e, "clearing the device error word");
        return fail(static_cast<kda_status_t>(host), "device reported: %s",
                    kda_status_string(static_cast<kda_status_t>(host)));
    }
    return KDA_OK;
}

}  // extern "C"
