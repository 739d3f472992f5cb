// Device helpers shared by the libpi kernels: streaming loads, weight-row
// decoding for fp32 / fp16 / Q4_0, warp reductions, status bits and the
// workspace layout.
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "pi.h"

namespace pi {

// ------------------------------------------------------------ status bits
// Sticky bits OR-ed into the workspace status word by device-side checks.
enum : uint32_t {
  DEV_BAD_INDEX = 1u,   // a listed neuron id outside [hot, d_ff): skipped
  DEV_BAD_COUNT = 2u,   // a list length outside [0, d_ff - hot]: clamped
  DEV_TIMEOUT = 4u,     // a bounded inter-CTA wait gave up
};

// Workspace header (first 256 bytes of every workspace).
struct WsHeader {
  uint32_t status;                   // sticky DEV_* bits
  uint32_t pad0[15];
  unsigned long long rows_listed;    // first-matrix neuron rows processed (x token passes)
  unsigned long long rows_down;      // down-projection rows read
  unsigned long long rows_second;    // ReGLU W_up rows read
  unsigned long long cold_listed;    // the three counts above, for rows read
  unsigned long long cold_down;      //   from a host-memory cold tier
  unsigned long long cold_second;
  unsigned long long stats_pad[2];
  uint32_t counters[32];             // grid-barrier / arrival counters
};
static_assert(sizeof(WsHeader) == 256, "workspace header is 256 bytes");

// ------------------------------------------------ dependent launches
// The per-step kernels are launched with programmatic stream serialization
// (launch_dep): a kernel's CTAs may be scheduled while the previous kernel
// on the stream drains.  Each such kernel calls pdl_wait() before its first
// access to global memory that another kernel writes or reads (it returns
// once the previous kernel has completed and its writes are visible; a
// no-op when the kernel was launched without the attribute), and then
// pdl_trigger(), which lets the next kernel's CTAs be scheduled once every
// CTA of this one has started.  Since each kernel waits for the one before
// it, every earlier kernel has completed by then too.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---------------------------------------------------------------- loads
// 16-byte streaming load of data read once per kernel (weights): no L1
// allocation, so the reused vectors in L1/shared memory are not evicted.
__device__ __forceinline__ uint4 ld_stream16(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ uint16_t ld_stream_u16(const void* p) {
  uint16_t v;
  asm volatile("ld.global.nc.L1::no_allocate.u16 %0, [%1];" : "=h"(v) : "l"(p));
  return v;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ float h2f(uint16_t bits) {
  return __half2float(__ushort_as_half(bits));
}

// Decode the 8 binary16 values of a 16-byte chunk.
__device__ __forceinline__ void f16x8_to_f32(const uint4& v, float* o) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[i]));
    o[2 * i] = f.x;
    o[2 * i + 1] = f.y;
  }
}

// Exact (q - 8) of the 4-bit code q in the low bits of `nib` (0..15), as a
// float: the bit pattern 0x4B000000 | q is the float 2^23 + q.
__device__ __forceinline__ float q4_centered(uint32_t nib) {
  return __int_as_float(0x4B000000 | nib) - 8388616.0f;
}

// ------------------------------------------------------------ dtype traits
// A "chunk" is 16 bytes of a weight row; CHUNK_COLS columns per chunk.
template <int DT> struct WTraits;
template <> struct WTraits<PI_F32> { static constexpr int CHUNK_COLS = 4; };
template <> struct WTraits<PI_F16> { static constexpr int CHUNK_COLS = 8; };
template <> struct WTraits<PI_Q4_0> { static constexpr int CHUNK_COLS = 32; };

// Bytes of one weight row of d columns (codes only for Q4_0).
__host__ __device__ __forceinline__ int64_t row_bytes(int dt, int d) {
  return dt == PI_F32 ? 4LL * d : (dt == PI_F16 ? 2LL * d : (int64_t)d / 2);
}

// Bytes of one staged row: its codes, then (Q4_0) its scales, padded to 16.
__host__ __device__ __forceinline__ int64_t stage_row_bytes(int dt, int d) {
  const int64_t b = row_bytes(dt, d) + (dt == PI_Q4_0 ? d / 16 : 0);
  return (b + 15) & ~(int64_t)15;
}

// Row-to-row distance of a weight matrix's codes, and of its Q4_0 scales.
__host__ __device__ __forceinline__ int64_t code_stride(int dt, int d, int64_t stride) {
  return stride ? stride : row_bytes(dt, d);
}
__host__ __device__ __forceinline__ int64_t scale_stride(int d, int64_t stride) {
  return stride ? stride : (int64_t)(d / 32) * 2;
}

// ----------------------------------------------------------- workspace
// Offsets (bytes from the workspace base) of the buffers a call uses.
struct WsLayout {
  size_t xh;        // fp32 [B][d]        normalised stack input
  size_t u;         // fp32 [B][r]        predictor hidden vector
  size_t mask;      // u32  [B][words]    stack-internal masks
  size_t idx;       // i32  [F]           compacted list
  size_t count;     // i32  [4]           list length
  size_t h;         // fp32 [F][B]        activations of listed rows
  size_t part;      // fp32 [S][B][d]     split-K partials
  size_t y;         // fp32 [B][d]        FFN output (stack)
  size_t tc;        // tensor-core scratch (fp16 layers at 2-64 tokens)
  size_t cta;       // u32  [SMs]         per-CTA list lengths (single-token kernel)
  size_t stage;     // listed cold rows of a host-memory cold tier, staged (token batches)
  size_t stage_bytes;
  size_t total;
  int splits;       // S
};

__host__ __forceinline__ size_t align256(size_t v) { return (v + 255) & ~(size_t)255; }

}  // namespace pi
