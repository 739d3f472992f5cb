// Tensor-core (tcgen05) path for the FFN at token batches (host interface,
// internal).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "pi.h"
#include "pi_common.cuh"

namespace pi {

// True when this layer's listed rows (hot prefix, then the cold list) run
// on the tensor cores at this batch: fp16 weights, 16 <= batch <= 64,
// d_model % 128 == 0, 16-byte row strides (and PI_DISABLE_TC unset).
bool ffn_tc_supported(const pi_layer& L, int batch);

// Workspace bytes the tensor-core paths (FFN and predictor) need for a layer
// shape at this batch (0: none).
size_t tc_scratch_bytes(int d_model, int d_ff, int rank, int batch);

// True when this layer's predictor runs on the tensor cores at this batch:
// fp16 predictor, 16 <= batch <= 64, rank % 128 == 0, d_model % 128 == 0.
bool pred_tc_supported(const pi_layer& L, int batch);

// mask [batch][words] of xh [batch][d_model]: u = P1 xh and z = P2[j] u + c
// on the tensor cores with each fp32 vector split into two fp16 parts
// (fp32 accumulation); bit j = j < hot or z_j > theta.  `uni` (optional,
// [words]): the OR of the tokens' words, written for the words from the
// one holding `hot` on (the words below are not written).
// split_ready: the fp16 hi / lo split of xh in `scratch` (tc_split_buffers)
// is already current (the stack's RMSNorm wrote it), so it is not rebuilt.
cudaError_t launch_predict_tc(const pi_layer& L, const float* xh, int batch, float theta,
                              uint32_t* mask, void* scratch, WsHeader* hdr, cudaStream_t s,
                              uint32_t* uni = nullptr, bool split_ready = false);

// The predictor's fp16 operands of xh in `scratch`: hi and lo, [nt][d_model]
// each, nt = batch rounded up to 16.
void tc_split_buffers(const pi_layer& L, void* scratch, void** hi, void** lo);

// Up/gate products of list positions [0, hot + count) (row p for p < hot,
// idx[p - hot] after) with xh [batch][d_model] (fp32, rounded to fp16 for
// the tensor cores; fp32 accumulation), bias, ReLU / ReGLU, each token's own
// mask bit for cold rows when `mask` ([batch][words]) is given; leaves the
// fp16 activations in `scratch` for launch_ffn_down_tc.  xh16_ready: the
// fp16 copy of xh in `scratch` is already current (launch_predict_tc wrote
// it from the same xh and batch), so it is not rebuilt.
// cold_stage (at least tc_cold_stage_bytes(L)): a Q4_0 layer with a
// host-memory cold tier copies its listed cold rows there first, once.
cudaError_t launch_ffn_up_tc(const pi_layer& L, const float* xh, int batch, const uint32_t* mask,
                             const int32_t* idx, const int32_t* count, void* scratch,
                             WsHeader* hdr, cudaStream_t s, bool xh16_ready = false,
                             char* cold_stage = nullptr);

// Device bytes the tensor-core kernels stage a Q4_0 cold tier's listed rows
// in (0: no cold tier).
size_t tc_cold_stage_bytes(const pi_layer& L);

// Split-K slices the down projection writes (part[0 .. splits)).
int ffn_tc_down_splits(const pi_layer& L);

// part[k][b][:] for k < ffn_tc_down_splits(L): sum over the k-th share of
// the list positions of h[p][b] * w_down_t[row(p)].
cudaError_t launch_ffn_down_tc(const pi_layer& L, int batch, const int32_t* idx,
                               const int32_t* count, float* part, void* scratch, WsHeader* hdr,
                               cudaStream_t s, char* cold_stage = nullptr);

}  // namespace pi
