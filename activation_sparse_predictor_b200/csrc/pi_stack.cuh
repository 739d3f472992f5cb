// Persistent single-token stack kernel (host interface, internal).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "pi.h"
#include "pi_common.cuh"

namespace pi {

// True when the fused single-token path handles these layers: batch 1, all
// layers sharing shape and dtypes, d_model <= 12288, rank <= 2048, and a
// shared-memory plan that fits.
bool stack1_supported(const pi_layer* layers, int n_layers, int batch);

// Layers per launch of the persistent kernel.
int stack1_chunk();

// Runs n_layers (<= stack1_chunk()) layers on x [d] (batch 1) with one
// cooperative launch.  mask_trace: nullable [n_layers][words].  `ws`/`lay`:
// the caller's workspace; counters and status live in its header.  trace:
// nullable device [n_layers][SMs][16] timeline (globaltimer ns).
cudaError_t launch_stack1(const pi_layer* layers, int n_layers, float* x, uint32_t* mask_trace,
                          void* ws, const WsLayout& lay, float theta, cudaStream_t s,
                          unsigned long long* trace = nullptr,
                          unsigned long long* utrace = nullptr);

// Units per layer recorded by the unit trace (first CTA only).
int stack1_unit_trace_len();

// Runs the fused kernel's bounded-wait code on a wait nothing completes
// (kind 0: mbarrier, kind 1: grid barrier), limited to limit_ns.
cudaError_t launch_wait_selftest(void* ws, int kind, unsigned long long limit_ns, cudaStream_t s);

}  // namespace pi
