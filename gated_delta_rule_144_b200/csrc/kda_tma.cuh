// Host-side tensor-map encoding shared by the TMA kernels (driver entry point resolved once).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

namespace kda {

// The driver's cuTensorMapEncodeTiled, resolved on first use.
cudaError_t tma_encoder_ready();

// Row-major [rows][cols] tensor, box of box_rows x box_cols elements.
cudaError_t make_map_2d(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int elem_bytes,
                        unsigned long long rows, int cols, int box_cols, int box_rows,
                        CUtensorMapSwizzle sw);

// Token-major [rows][H][cols] tensor (one head's rows), box of box_rows rows x box_cols columns.
cudaError_t make_map_3d_box(CUtensorMap* m, const void* base, CUtensorMapDataType dt,
                            int elem_bytes, unsigned long long rows, int H, int cols, int box_cols,
                            int box_rows, CUtensorMapSwizzle sw);

// The same with whole rows per box (box_cols = cols) and no swizzle.
cudaError_t make_map_3d_rows(CUtensorMap* m, const void* base, CUtensorMapDataType dt,
                             int elem_bytes, unsigned long long rows, int H, int cols,
                             int box_rows);

}  // namespace kda
