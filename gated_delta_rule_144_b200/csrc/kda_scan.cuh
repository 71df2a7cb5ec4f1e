// Two-level state pass of the split chunked prefill (equal-length sequences with few chains).
//
// The chunks of every chain are cut into segments of seg_m chunks. The map from a segment's
// initial state to its final state is affine, S -> A_p S + B_p (each chunk's map is
// S -> (diag(e^{Gamma_end}) - K_end^T W) S + K_end^T U~), so the segments' initial states follow
// from a short product chain over the segments, after which every segment runs at once.
#pragma once

#include "kda_internal.cuh"

namespace kda {

constexpr int kMaxScanSegments = 32;

// A segmented launch of the state pass (seg_m > 0): unit u = (group, segment, chain), chain =
// u % (N H), segment = seg_p0 + (u / (N H)) % seg_count, group = u / (N H seg_count), chunks
// [segment seg_m, (segment + 1) seg_m); h0 and hT are indexed by u (hT_last: only segment
// nseg - 1 writes hT, at the chain's index). With ident, group 0 starts from S = I with U~ = 0
// (it computes A_p); no_out suppresses the output stores. seg_m = 0: the plain launch.
struct ScanSplit {
    int seg_m = 0, seg_p0 = 0, seg_count = 0, groups = 1, nseg = 0;
    bool ident = false, no_out = false, hT_last = false;
};
cudaError_t launch_chunk_scan_split(const FwdParams& p, const ScanSegment& seg,
                                    const ScanSplit& split, cudaStream_t stream,
                                    const ScanNorm* norm = nullptr);

// The segments' initial states of the two-level state pass, in fp32:
//   sinit[p] = amap[p - 1] sinit[p - 1] + bmap[p - 1],  p = 1 .. steps,
// every array [.][chains][128][128] (row = key channel, column = value column), sinit[0] given.
cudaError_t launch_scan_combine(const float* amap, const float* bmap, float* sinit, int chains,
                                int steps, cudaStream_t stream);

}  // namespace kda
