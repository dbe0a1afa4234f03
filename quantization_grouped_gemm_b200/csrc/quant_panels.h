// Host interface of the panel kernel (quant_panels.cu): the jagged
// column-wise quantisation into the padded transposed layout, and its
// dual-output form with the rowwise quantisation of the same rows.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "device_common.cuh"

namespace fp8qgg {

// Scratch layout: [0, 256) the task counter; one arrival counter per unit
// (num_groups x panels, rounded up to 256 bytes); the column absmax words
// [num_groups, cols]; dual form: the row absmax words [rows_total].
struct PanelScratch {
  size_t arrive_off, amax_off, rowmax_off, bytes;
};

PanelScratch panel_scratch(int64_t rows_total, int64_t cols, int32_t num_groups, bool dual);

// Enqueues the panel kernel.  q_row == nullptr selects the column-wise form.
// The first panel_scratch(...).bytes of `scratch` must be zero on `stream`.
int panel_launch(const void *x, int64_t rows_total, int64_t cols, int64_t ld_x,
                 const int32_t *offsets, int32_t num_groups, uint8_t *q_col, int64_t ld_qc,
                 float *scales_col, uint8_t *q_row, int64_t ld_qr, float *scales_row, int fmt,
                 float scale_max, uint64_t *sat_count, int32_t *dev_status, void *scratch,
                 UnitWait uw, cudaStream_t stream);

// The wait settings set by fp8qgg_test_unit_wait (normal ones otherwise).
UnitWait current_unit_wait();

// Argument checks of a jagged column-wise call (quant_colwise_jagged.cu).
int colwise_check(const void *x, int64_t rows_total, int64_t cols, int64_t ld_x,
                  const int32_t *offsets, int32_t num_groups, uint8_t *q, int64_t ld_q,
                  int layout, float *scales, int fmt, float scale_max, uint64_t *sat_count,
                  int32_t *dev_status);

}  // namespace fp8qgg
