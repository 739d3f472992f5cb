// Tensor-core (tcgen05) path for the dense hot prefix at token batches
// (host interface, internal).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "pi.h"
#include "pi_common.cuh"

namespace pi {

// True when the hot prefix's gate/up products and down projection of this
// layer at this batch run on tensor cores: fp16 weights, 16 <= batch <= 64,
// hot % 128 == 0 and hot >= 128, d_model % 128 == 0 (and PI_DISABLE_TC unset).
bool hot_tc_supported(const pi_layer& L, int batch);

// Workspace bytes the path needs for a layer of this shape (0 if unused).
size_t hot_tc_scratch_bytes(int d_model, int hot, int batch);

// h[n * batch + b] for every hot row n < hot and token b < batch: the
// activation of the hot neurons' gate/up products with xh [batch][d_model]
// (fp32, rounded to fp16 for the tensor cores; fp32 accumulation).
// `scratch`: hot_tc_scratch_bytes(...) bytes, 256-byte aligned.
cudaError_t launch_hot_up_tc(const pi_layer& L, const float* xh, int batch, float* h,
                             void* scratch, WsHeader* hdr, cudaStream_t s);

// Split-K slices the hot down projection writes (part[0 .. splits)).
int hot_tc_down_splits(const pi_layer& L);

// part[k][b][:] for k < hot_tc_down_splits(L): the hot rows' contribution
// sum_{j < hot} h[j][b] * w_down_t[j] (from the fp16 h that
// launch_hot_up_tc left in `scratch`), split over the hot rows in a fixed
// order; adds hot to the workspace's down-row counter.
cudaError_t launch_hot_down_tc(const pi_layer& L, int batch, float* part, void* scratch,
                               WsHeader* hdr, cudaStream_t s);

}  // namespace pi
