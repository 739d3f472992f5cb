// Launchers of the libpi kernels (host side, internal to the library).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

#include "pi.h"
#include "pi_common.cuh"

namespace pi {

int device_sms();                 // SM count of the current device (cached)
void note_launch();               // counts one kernel launch (pi_kernel_launches)
unsigned long long launches_so_far();

// Raises a kernel's dynamic shared-memory limit on the current device once.
cudaError_t allow_smem_fn(const void* fn, size_t bytes);

// Whether launch_dep sets programmatic stream serialization (on unless the
// environment variable PI_NO_PDL is set to a value other than 0).
bool pdl_enabled();

// Launches kernel k like k<<<grid, block, smem, s>>>(args...) and counts
// the launch; with dep, and when pdl_enabled(), with programmatic stream
// serialization (the kernel must call pdl_wait() before touching global
// memory another kernel uses).  The CUDA-core kernels of small token
// batches, whose grids are sized to the SM count, are launched without it
// (and do not trigger their dependents early): CTAs scheduled while the
// previous kernel still holds SMs would be placed unevenly.
template <typename... KArgs, typename... Args>
cudaError_t launch_k(bool dep, void (*k)(KArgs...), dim3 grid, dim3 block, size_t smem,
                     cudaStream_t s, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = dep && pdl_enabled() ? 1 : 0;
  note_launch();
  return cudaLaunchKernelEx(&cfg, k, std::forward<Args>(args)...);
}

template <typename... KArgs, typename... Args>
cudaError_t launch_dep(void (*k)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                       Args&&... args) {
  return launch_k(true, k, grid, block, smem, s, std::forward<Args>(args)...);
}

template <typename... KArgs, typename... Args>
cudaError_t launch_plain(void (*k)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                         Args&&... args) {
  return launch_k(false, k, grid, block, smem, s, std::forward<Args>(args)...);
}
int pick_tb(int batch, int d);    // tokens per pass of the x-staged kernels
int down_tb(int batch);           // tokens per pass of the down projection
int down_splits(int batch, int d);// split-K slices of the down projection

// xh[b] = x[b] / sqrt(mean(x[b]^2) + 1e-6), b < batch.
// xh = rmsnorm(x) per token; with hi / lo ([nt][d] fp16, nt >= batch) also
// the split hi = fp16(xh), lo = fp16(xh - hi), zero rows past the batch.
cudaError_t launch_rmsnorm(const float* x, int batch, int d, float* xh, cudaStream_t s,
                           void* hi = nullptr, void* lo = nullptr, int nt = 0);

// u[b][k] = p1[k] . xh[b]
cudaError_t launch_pred_u(const pi_layer& L, const float* xh, int batch, float* u,
                          cudaStream_t s);

// mask[b] from z = p2 u + p_bias (rows >= hot), bits < hot set.
cudaError_t launch_pred_z(const pi_layer& L, const float* u, int batch, float theta,
                          uint32_t* mask, cudaStream_t s);

// out[w] = OR over b < batch of mask[b][w], w < words (many CTAs).
cudaError_t launch_mask_union(const uint32_t* mask, int batch, int words, uint32_t* out,
                              cudaStream_t s);

// ascending set-bit lists (see pi_compact)
cudaError_t launch_compact(const uint32_t* mask, int batch, int d_ff, int begin, int mode,
                           int32_t* idx, int32_t* count, cudaStream_t s);

// h[n][b] for rows n of [0,hot) U idx[0..count).  `stage` (optional, at
// least cold_stage_bytes(L, batch)): a layer with a host-memory cold tier
// first copies its listed cold rows there, so that every token chunk reads
// them from device memory.
cudaError_t launch_ffn_up(const pi_layer& L, const float* xh, int batch, const uint32_t* mask,
                          int per_token, const int32_t* idx, const int32_t* count, float* h,
                          WsHeader* hdr, cudaStream_t s, int n0 = 0, char* stage = nullptr);

// Device bytes launch_ffn_up and launch_ffn_down stage a host-memory cold
// tier's listed rows in (0: the layer has none, or its tokens fit one chunk
// of each kernel and read each row once).
size_t cold_stage_bytes(const pi_layer& L, int batch);

// Copies the first matrix's (and ReGLU's W_up) rows of a host-memory cold
// tier's listed neurons to stage[r][p] (row bytes stage_row_bytes, r the
// matrix, p the list position; zeros for an id outside [hot, d_ff)).
cudaError_t launch_stage_cold(const pi_layer& L, const int32_t* idx, const int32_t* count,
                              char* stage, WsHeader* hdr, cudaStream_t s);
// Copies their w_down_t rows to stage[p]: with h ([n][batch] fp32), only the
// rows whose h is nonzero for some token; without, every listed row.
cudaError_t launch_stage_cold_down(const pi_layer& L, int batch, const int32_t* idx,
                                   const int32_t* count, const float* h, char* stage,
                                   WsHeader* hdr, cudaStream_t s);

// part[s][b][:] = sum over the slice's rows of h[n][b] * w_down_t[row n],
// the list positions [nb, H + count) split into `splits` slices
// `stage`: as for launch_ffn_up (the same buffer); a cold-tier layer's down
// rows that some token needs are staged there first when the tokens take
// four chunks or more.
cudaError_t launch_ffn_down(const pi_layer& L, int batch, const int32_t* idx,
                            const int32_t* count, const float* h, float* part, int splits,
                            WsHeader* hdr, cudaStream_t s, int nb = 0, char* stage = nullptr);

// out[b][i] = (resid ? resid[b][i] : 0) + sum_s part[s][b][i], s ascending.
cudaError_t launch_reduce(const float* part, int splits, int batch, int d, const float* resid,
                          float* out, cudaStream_t s);

// A kernel that waits about `ns` nanoseconds of device time and exits
// (lets the host enqueue a timed sequence before the device reaches it).
cudaError_t launch_delay(unsigned long long ns, cudaStream_t s);

}  // namespace pi
