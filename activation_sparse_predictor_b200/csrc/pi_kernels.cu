// libpi kernels, sm_100a.
//
// The hot path of one FFN layer (see pi.h for the operation definitions):
//   rmsnorm -> predictor u = p1 xh -> predictor logits + threshold -> mask
//   -> compaction -> gathered up/gate rows + activation -> gathered split-K
//   down projection -> fixed-order reduction (+ residual).
//
// All weight traffic is 16-byte streaming loads of whole neuron rows (a row
// per warp for the dot products, a row per CTA for the down projection),
// with the reused vectors (xh, u) staged in shared memory.  Accumulation is
// fp32 throughout.
#include <algorithm>
#include <cstdlib>
#include <atomic>
#include <mutex>
#include <unordered_map>

#include "pi_kernels.cuh"

namespace pi {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
// Kernels that stage the inputs of a token chunk in shared memory (up to
// 200 KB, one CTA per SM) run wider CTAs, so more warps share one staged copy
// and more weight rows stream at once.
constexpr int kWideThreads = 512;
constexpr int kWideWarps = kWideThreads / 32;
// (Q4_0 rows keep the narrow CTA: their decode needs the registers)
template <int WT> constexpr int up_threads() { return WT == PI_Q4_0 ? kThreads : kWideThreads; }

__device__ __forceinline__ void flag(uint32_t* status, uint32_t bit) {
  if (status) atomicOr(status, bit);
}

// Stage xh[t0 .. t0+TB) (fp32 [B][d]) into shared memory, zero past B.
template <int TB>
__device__ __forceinline__ void stage_x(float* sx, const float* xh, int B, int d, int t0) {
  const int n4 = d / 4;
  for (int e = threadIdx.x; e < TB * n4; e += blockDim.x) {
    const int b = e / n4, i = e % n4;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (t0 + b < B) v = reinterpret_cast<const float4*>(xh + (size_t)(t0 + b) * d)[i];
    reinterpret_cast<float4*>(sx + (size_t)b * d)[i] = v;
  }
}

// ---------------------------------------------------------------------------
// Dot products of NR weight rows against TB staged vectors, one 16-byte chunk
// (chunk c covers columns [c*CC, (c+1)*CC)) at a time.
template <int WT, int NR, int TB>
struct RowDot {
  __device__ __forceinline__ static void chunk(const char* const* rows,
                                               const uint16_t* const* scales, int c,
                                               const float* sx, int d,
                                               float (&acc)[NR][TB]) {
    if constexpr (WT == PI_F32) {
      uint4 v[NR];
#pragma unroll
      for (int r = 0; r < NR; ++r) v[r] = ld_stream16(rows[r] + (size_t)c * 16);
#pragma unroll
      for (int b = 0; b < TB; ++b) {
        const float4 x = *reinterpret_cast<const float4*>(sx + (size_t)b * d + c * 4);
#pragma unroll
        for (int r = 0; r < NR; ++r) {
          float a = acc[r][b];
          a = fmaf(__uint_as_float(v[r].x), x.x, a);
          a = fmaf(__uint_as_float(v[r].y), x.y, a);
          a = fmaf(__uint_as_float(v[r].z), x.z, a);
          a = fmaf(__uint_as_float(v[r].w), x.w, a);
          acc[r][b] = a;
        }
      }
    } else if constexpr (WT == PI_F16) {
      float w[NR][8];
#pragma unroll
      for (int r = 0; r < NR; ++r) f16x8_to_f32(ld_stream16(rows[r] + (size_t)c * 16), w[r]);
#pragma unroll
      for (int b = 0; b < TB; ++b) {
        const float4 x0 = *reinterpret_cast<const float4*>(sx + (size_t)b * d + c * 8);
        const float4 x1 = *reinterpret_cast<const float4*>(sx + (size_t)b * d + c * 8 + 4);
        const float xv[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
#pragma unroll
        for (int r = 0; r < NR; ++r) {
          float a = acc[r][b];
#pragma unroll
          for (int e = 0; e < 8; ++e) a = fmaf(w[r][e], xv[e], a);
          acc[r][b] = a;
        }
      }
    } else {  // Q4_0: chunk c = block c of the row
      uint4 v[NR];
      float s[NR];
#pragma unroll
      for (int r = 0; r < NR; ++r) {
        v[r] = ld_stream16(rows[r] + (size_t)c * 16);
        s[r] = h2f(ld_stream_u16(scales[r] + c));
      }
#pragma unroll
      for (int b = 0; b < TB; ++b) {
        const float* xp = sx + (size_t)b * d + c * 32;
        float xv[32];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const float4 t = reinterpret_cast<const float4*>(xp)[q];
          xv[4 * q] = t.x; xv[4 * q + 1] = t.y; xv[4 * q + 2] = t.z; xv[4 * q + 3] = t.w;
        }
#pragma unroll
        for (int r = 0; r < NR; ++r) {
          const uint32_t wd[4] = {v[r].x, v[r].y, v[r].z, v[r].w};
          float a = 0.f;
#pragma unroll
          for (int k = 0; k < 16; ++k) {
            const uint32_t byte = (wd[k >> 2] >> (8 * (k & 3))) & 0xFFu;
            a = fmaf(q4_centered(byte & 0xFu), xv[k], a);
            a = fmaf(q4_centered(byte >> 4), xv[k + 16], a);
          }
          acc[r][b] = fmaf(a, s[r], acc[r][b]);
        }
      }
    }
  }
};

// ---------------------------------------------------------------------------
// One CTA per row (d <= 16384, d % 4 == 0): the row is read once into
// registers (up to four float4 per thread), its mean square reduced across
// the CTA, and the scaled row written from the registers.
// xh = x / sqrt(mean(x^2) + 1e-6), one CTA per token.  With hi / lo (the
// tensor-core predictor's operands, [nt][d] fp16), also hi = fp16(xh) and
// lo = fp16(xh - hi), and zero rows for the padding tokens batch .. nt-1
// (CTAs past the batch), which the predictor would otherwise build in a
// kernel of its own.
__global__ void __launch_bounds__(1024) k_rmsnorm(const float* __restrict__ x, int d,
                                                  float* __restrict__ xh, int batch,
                                                  __half* __restrict__ hi, __half* __restrict__ lo) {
  pdl_wait();
  pdl_trigger();
  if ((int)blockIdx.x >= batch) {  // a padding token of the fp16 operands
    for (int i = threadIdx.x; i < d / 4; i += blockDim.x) {
      reinterpret_cast<uint2*>(hi + (size_t)blockIdx.x * d)[i] = make_uint2(0u, 0u);
      reinterpret_cast<uint2*>(lo + (size_t)blockIdx.x * d)[i] = make_uint2(0u, 0u);
    }
    return;
  }
  const float4* xr = reinterpret_cast<const float4*>(x + (size_t)blockIdx.x * d);
  float4* yr = reinterpret_cast<float4*>(xh + (size_t)blockIdx.x * d);
  const int n4 = d >> 2;
  float4 v[4];
  float ss = 0.f;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int i = threadIdx.x + k * blockDim.x;
    v[k] = i < n4 ? xr[i] : make_float4(0.f, 0.f, 0.f, 0.f);
    ss = fmaf(v[k].x, v[k].x, ss);
    ss = fmaf(v[k].y, v[k].y, ss);
    ss = fmaf(v[k].z, v[k].z, ss);
    ss = fmaf(v[k].w, v[k].w, ss);
  }
  ss = warp_sum(ss);
  __shared__ float red[32];
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  if (threadIdx.x < 32) {
    float t = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.f;
    t = warp_sum(t);
    if (threadIdx.x == 0) red[0] = t;
  }
  __syncthreads();
  const float inv = 1.0f / sqrtf(red[0] / (float)d + 1e-6f);
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int i = threadIdx.x + k * blockDim.x;
    if (i >= n4) continue;
    const float4 y = make_float4(v[k].x * inv, v[k].y * inv, v[k].z * inv, v[k].w * inv);
    yr[i] = y;
    if (hi) {
      const float e[4] = {y.x, y.y, y.z, y.w};
      __align__(8) __half h[4], l[4];
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        h[m] = __float2half_rn(e[m]);
        l[m] = __float2half_rn(e[m] - __half2float(h[m]));
      }
      reinterpret_cast<uint2*>(hi + (size_t)blockIdx.x * d)[i] = *reinterpret_cast<const uint2*>(h);
      reinterpret_cast<uint2*>(lo + (size_t)blockIdx.x * d)[i] = *reinterpret_cast<const uint2*>(l);
    }
  }
}

// u[b][k] = p1[k] . xh[b]; one warp per predictor row.
template <int PT, int TB>
__global__ void __launch_bounds__(kWideThreads) k_pred_u(const char* __restrict__ p1,
                                                     const float* __restrict__ xh, int B,
                                                     int d, int r, float* __restrict__ u) {
  pdl_wait();
  extern __shared__ __align__(16) float sx[];
  const int t0 = blockIdx.y * TB;
  stage_x<TB>(sx, xh, B, d, t0);
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int CC = WTraits<PT>::CHUNK_COLS;
  const int nch = d / CC;
  const int64_t rb = row_bytes(PT, d);
  for (int k = blockIdx.x * kWideWarps + warp; k < r; k += gridDim.x * kWideWarps) {
    float acc[1][TB];
#pragma unroll
    for (int b = 0; b < TB; ++b) acc[0][b] = 0.f;
    const char* rows[1] = {p1 + (size_t)k * rb};
    const uint16_t* sc[1] = {nullptr};
#pragma unroll 8
    for (int c = lane; c < nch; c += 32) RowDot<PT, 1, TB>::chunk(rows, sc, c, sx, d, acc);
#pragma unroll
    for (int b = 0; b < TB; ++b) {
      const float v = warp_sum(acc[0][b]);
      if (lane == 0 && t0 + b < B) u[(size_t)(t0 + b) * r + k] = v;
    }
  }
}

// Predictor logits and threshold: one warp per mask word (32 neurons).
template <int PT, int TB>
__global__ void __launch_bounds__(kThreads) k_pred_z(const char* __restrict__ p2,
                                                     const float* __restrict__ pbias,
                                                     const float* __restrict__ u, int B, int r,
                                                     int F, int H, float theta,
                                                     uint32_t* __restrict__ mask, int words) {
  pdl_wait();
  extern __shared__ __align__(16) float su[];
  const int t0 = blockIdx.y * TB;
  stage_x<TB>(su, u, B, r, t0);
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int CC = WTraits<PT>::CHUNK_COLS;
  const int nch = r / CC;
  const int64_t rb = row_bytes(PT, r);
  for (int w = blockIdx.x * kWarps + warp; w < words; w += gridDim.x * kWarps) {
    const int j0 = w * 32;
    float zl[TB];
#pragma unroll
    for (int b = 0; b < TB; ++b) zl[b] = 0.f;
    if (j0 + 32 > H) {
      for (int jj = 0; jj < 32; jj += 2) {
        // two neurons per pass for more loads in flight
        const int ja = j0 + jj, jb = j0 + jj + 1;
        const bool va = ja >= H && ja < F, vb = jb >= H && jb < F;
        if (!va && !vb) continue;
        float acc[2][TB];
#pragma unroll
        for (int b = 0; b < TB; ++b) acc[0][b] = acc[1][b] = 0.f;
        const char* rows[2] = {p2 + (size_t)(va ? ja : jb) * rb, p2 + (size_t)(vb ? jb : ja) * rb};
        const uint16_t* sc[2] = {nullptr, nullptr};
#pragma unroll 4
        for (int c = lane; c < nch; c += 32) RowDot<PT, 2, TB>::chunk(rows, sc, c, su, r, acc);
#pragma unroll
        for (int b = 0; b < TB; ++b) {
          const float za = warp_sum(acc[0][b]);
          const float zb = warp_sum(acc[1][b]);
          if (lane == jj && va) zl[b] = za + (pbias ? pbias[ja] : 0.f);
          if (lane == jj + 1 && vb) zl[b] = zb + (pbias ? pbias[jb] : 0.f);
        }
      }
    }
    const int j = j0 + lane;
#pragma unroll
    for (int b = 0; b < TB; ++b) {
      const bool on = j < F && (j < H || zl[b] > theta);
      const uint32_t bits = __ballot_sync(0xffffffffu, on);
      if (lane == 0 && t0 + b < B) mask[(size_t)(t0 + b) * words + w] = bits;
    }
  }
}

// Compaction.  Grid (chunks, lists): CTA x of list l takes the
// kCompactWords mask words [x * kCompactWords, ...) of the list, one word
// per thread.  Its first output position is the number of set bits in the
// list's words before the chunk, which the CTA counts itself (a few KB of
// mask words at most); then a scan of its words' popcounts places every
// word's bits, and each warp writes its 32 words' entries in order, lane t
// taking bit t of each word (the entries of one word go to consecutive
// positions).  The last chunk's CTA writes the count.  Bits below `begin`
// and from F on are cleared; `unite` ORs the B tokens' words first.
constexpr int kCompactWords = 256;

__device__ __forceinline__ uint32_t compact_word(const uint32_t* __restrict__ mask, int B,
                                                 int words, int F, int begin, int unite, int list,
                                                 int w) {
  uint32_t m = 0u;
  if (unite) {
#pragma unroll 8
    for (int b = 0; b < B; ++b) m |= mask[(size_t)b * words + w];
  } else {
    m = mask[(size_t)list * words + w];
  }
  const int lo = w * 32;
  if (begin > lo) m = (begin - lo >= 32) ? 0u : (m & (~0u << (begin - lo)));
  if (F < lo + 32) m = (F <= lo) ? 0u : (m & ((1u << (F - lo)) - 1u));
  return m;
}

__global__ void __launch_bounds__(kCompactWords) k_compact(const uint32_t* __restrict__ mask, int B,
                                                           int words, int F, int begin, int unite,
                                                           int32_t* __restrict__ idx, int idx_stride,
                                                           int32_t* __restrict__ count) {
  pdl_wait();
  pdl_trigger();
  constexpr int NW = kCompactWords / 32;
  __shared__ int wsum[NW + 1];
  __shared__ int s_base;
  const int list = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int w_lo = blockIdx.x * kCompactWords;
  // set bits of the list's words before this chunk (words below `begin`
  // are empty and skipped)
  int before = 0;
  for (int w = max(begin >> 5, 0) + tid; w < w_lo; w += kCompactWords)
    before += __popc(compact_word(mask, B, words, F, begin, unite, list, w));
  before = __reduce_add_sync(0xffffffffu, before);
  if (lane == 0) wsum[warp] = before;
  __syncthreads();
  if (tid == 0) {
    int t = 0;
    for (int k = 0; k < NW; ++k) t += wsum[k];
    s_base = t;
  }
  __syncthreads();
  const int w = w_lo + tid;
  const uint32_t m = w < words ? compact_word(mask, B, words, F, begin, unite, list, w) : 0u;
  const int c = __popc(m);
  int incl = c;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  if (tid == 0) {
    int run = 0;
    for (int k = 0; k < NW; ++k) {
      const int t = wsum[k];
      wsum[k] = run;
      run += t;
    }
    wsum[NW] = run;
  }
  __syncthreads();
  int32_t* out = idx + (size_t)list * idx_stride;
  int run = s_base + wsum[warp];
  const int wfirst = w_lo + warp * 32;
  for (int i = 0; i < 32; ++i) {
    const uint32_t mi = __shfl_sync(0xffffffffu, m, i);
    if ((mi >> lane) & 1u) out[run + __popc(mi & ((1u << lane) - 1u))] = (wfirst + i) * 32 + lane;
    run += __popc(mi);
  }
  if (blockIdx.x == gridDim.x - 1 && tid == 0) count[list] = s_base + wsum[NW];
}

// out[w] = OR over tokens b < B of mask[b][w].  Block: 32 words x 8 token
// groups (token b goes to group b % 8, eight loads in flight per thread),
// the groups combined in shared memory.
__global__ void __launch_bounds__(256) k_mask_union(const uint32_t* __restrict__ mask, int B,
                                                    int words, uint32_t* __restrict__ out) {
  pdl_wait();
  __shared__ uint32_t sm[8][32];
  const int wl = threadIdx.x & 31, tg = threadIdx.x >> 5;
  const int w = blockIdx.x * 32 + wl;
  uint32_t m = 0u;
  if (w < words) {
    uint32_t a[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) a[k] = 0u;
    for (int b0 = tg; b0 < B; b0 += 64) {
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int b = b0 + 8 * k;
        if (b < B) a[k] |= mask[(size_t)b * words + w];
      }
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) m |= a[k];
  }
  sm[tg][wl] = m;
  __syncthreads();
  if (tg == 0 && w < words) {
    uint32_t u = 0u;
#pragma unroll
    for (int g = 0; g < 8; ++g) u |= sm[g][wl];
    out[w] = u;
  }
}

// Row j of a weight matrix whose rows [H, F) may live in a host-memory cold
// tier (`cold` != null): those rows are read over the host link from there.
__device__ __forceinline__ const char* wrow(const void* hot, const void* cold, int j, int H,
                                            int64_t stride) {
  return cold && j >= H ? (const char*)cold + (size_t)(j - H) * stride
                        : (const char*)hot + (size_t)j * stride;
}

// Gathered up/gate rows + activation: one warp per listed row.
template <int WT, int ACT, int TB>
__global__ void __launch_bounds__(up_threads<WT>()) k_ffn_up(pi_layer L, const float* __restrict__ xh,
                                                     int B, const uint32_t* __restrict__ mask,
                                                     int per_token, int words,
                                                     const int32_t* __restrict__ idx,
                                                     const int32_t* __restrict__ count,
                                                     float* __restrict__ h, WsHeader* hdr,
                                                     int n0, const char* __restrict__ stg) {
  pdl_wait();
  extern __shared__ __align__(16) float sx[];
  uint32_t* status = hdr ? &hdr->status : nullptr;
  const int d = L.d_model, F = L.d_ff, H = L.hot;
  const int t0 = blockIdx.y * TB;
  stage_x<TB>(sx, xh, B, d, t0);
  __syncthreads();
  int cnt = *count;
  if (cnt < 0 || cnt > F - H) {
    if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) flag(status, DEV_BAD_COUNT);
    cnt = cnt < 0 ? 0 : F - H;
  }
  const int N = H + cnt;
  if (hdr && blockIdx.x == 0 && threadIdx.x == 0) {
    atomicAdd(&hdr->rows_listed, (unsigned long long)(N - n0));
    if (ACT == PI_REGLU) atomicAdd(&hdr->rows_second, (unsigned long long)(N - n0));
    const int nc = N - (n0 > H ? n0 : H);  // list positions >= H hold the cold rows
    if (L.w_up_cold && !stg && nc > 0) {  // (staged rows were counted when staged)
      atomicAdd(&hdr->cold_listed, (unsigned long long)nc);
      if (ACT == PI_REGLU) atomicAdd(&hdr->cold_second, (unsigned long long)nc);
    }
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool sq = L.act == PI_RELU2;
  constexpr int NR = (ACT == PI_REGLU) ? 2 : 1;
  constexpr int CC = WTraits<WT>::CHUNK_COLS;
  const int nch = d / CC;
  const int64_t rb = code_stride(WT, d, L.w_row_stride);
  const int64_t sbs = scale_stride(d, L.w_row_stride);
  const int64_t up_rs = (ACT == PI_REGLU && L.w_up_row_stride) ? L.w_up_row_stride : L.w_row_stride;
  const int64_t rb2 = code_stride(WT, d, up_rs);
  const int64_t sbs2 = scale_stride(d, up_rs);
  // list positions n0 .. N-1 (n0 = H when the hot rows are computed elsewhere)
  constexpr int UPW = up_threads<WT>() / 32;
  for (int n = n0 + blockIdx.x * UPW + warp; n < N; n += gridDim.x * UPW) {
    const int j = n < H ? n : idx[n - H];
    if (j < H && n >= H || j >= F || j < 0) {
      if (lane == 0) {
        flag(status, DEV_BAD_INDEX);
        for (int b = 0; b < TB; ++b)
          if (t0 + b < B) h[(size_t)n * B + t0 + b] = 0.f;
      }
      continue;
    }
    const char* rows[NR];
    const uint16_t* sc[NR];
    if (stg && n >= H) {  // a cold row staged in device memory at its list position
      const int64_t srb = stage_row_bytes(WT, d), cb = row_bytes(WT, d);
#pragma unroll
      for (int r = 0; r < NR; ++r) {
        rows[r] = stg + ((size_t)r * (F - H) + (n - H)) * srb;
        sc[r] = (const uint16_t*)(rows[r] + cb);
      }
    } else if constexpr (ACT == PI_REGLU) {
      rows[0] = wrow(L.w_gate, L.w_gate_cold, j, H, rb);
      rows[1] = wrow(L.w_up, L.w_up_cold, j, H, rb2);
      sc[0] = (const uint16_t*)wrow(L.w_gate_scales, L.w_gate_cold_scales, j, H, sbs);
      sc[1] = (const uint16_t*)wrow(L.w_up_scales, L.w_up_cold_scales, j, H, sbs2);
    } else {
      rows[0] = wrow(L.w_up, L.w_up_cold, j, H, rb);
      sc[0] = (const uint16_t*)wrow(L.w_up_scales, L.w_up_cold_scales, j, H, sbs);
    }
    float acc[NR][TB];
#pragma unroll
    for (int r = 0; r < NR; ++r)
#pragma unroll
      for (int b = 0; b < TB; ++b) acc[r][b] = 0.f;
    // several 16-byte loads per lane in flight: one row per warp, so the
    // warp's memory parallelism comes from unrolling along the row
#pragma unroll (8 / NR)
    for (int c = lane; c < nch; c += 32) RowDot<WT, NR, TB>::chunk(rows, sc, c, sx, d, acc);
    const float bj = L.bias ? L.bias[j] : 0.f;
#pragma unroll
    for (int b = 0; b < TB; ++b) {
      float g = warp_sum(acc[0][b]) + bj;
      float hv = g > 0.f ? g : 0.f;
      if constexpr (ACT == PI_REGLU) hv *= warp_sum(acc[NR - 1][b]);
      else if (sq) hv *= hv;  // squared ReLU
      if (per_token && n >= H && mask && t0 + b < B) {
        const uint32_t bit = (mask[(size_t)(t0 + b) * words + (j >> 5)] >> (j & 31)) & 1u;
        if (!bit) hv = 0.f;
      }
      if (lane == 0 && t0 + b < B) h[(size_t)n * B + t0 + b] = hv;
    }
  }
}

// Copies the listed cold rows of the first matrix (and ReGLU's W_up) from a
// host-memory cold tier into device memory, at their list positions
// (stage_row_bytes each: codes, then Q4_0 scales), so that the up kernel's
// token chunks read them from HBM and each row crosses the host link once.
// One warp per list position; a position holding an id outside [H, F) gets
// a zero row (the up kernels flag such ids; the tensor-core kernels read
// every staged position, so none may hold stale bytes).
template <int WT, int NR>
__global__ void __launch_bounds__(kThreads) k_stage_cold(pi_layer L, const int32_t* __restrict__ idx,
                                                         const int32_t* __restrict__ count,
                                                         char* __restrict__ stg, WsHeader* hdr) {
  pdl_wait();
  const int d = L.d_model, F = L.d_ff, H = L.hot;
  int cnt = *count;
  cnt = cnt < 0 ? 0 : (cnt > F - H ? F - H : cnt);
  if (hdr && blockIdx.x == 0 && threadIdx.x == 0 && cnt > 0) {
    atomicAdd(&hdr->cold_listed, (unsigned long long)cnt);
    if (NR == 2) atomicAdd(&hdr->cold_second, (unsigned long long)cnt);
  }
  const int64_t srb = stage_row_bytes(WT, d), cb = row_bytes(WT, d);
  const int nsc = WT == PI_Q4_0 ? d / 32 : 0;
  const int64_t up_rs = (NR == 2 && L.w_up_row_stride) ? L.w_up_row_stride : L.w_row_stride;
  const int64_t rs[2] = {code_stride(WT, d, L.w_row_stride), code_stride(WT, d, up_rs)};
  const int64_t ss[2] = {scale_stride(d, L.w_row_stride), scale_stride(d, up_rs)};
  const void* hot[2] = {NR == 2 ? L.w_gate : L.w_up, L.w_up};
  const void* cold[2] = {NR == 2 ? L.w_gate_cold : L.w_up_cold, L.w_up_cold};
  const void* shot[2] = {NR == 2 ? L.w_gate_scales : L.w_up_scales, L.w_up_scales};
  const void* scold[2] = {NR == 2 ? L.w_gate_cold_scales : L.w_up_cold_scales, L.w_up_cold_scales};
  const int lane = threadIdx.x & 31;
  const int wpb = blockDim.x >> 5;
  for (int p = blockIdx.x * wpb + (threadIdx.x >> 5); p < cnt; p += gridDim.x * wpb) {
    const int j = idx[p];
    const bool ok = j >= H && j < F;
#pragma unroll
    for (int r = 0; r < NR; ++r) {
      const char* src = ok ? wrow(hot[r], cold[r], j, H, rs[r]) : nullptr;
      char* dst = stg + ((size_t)r * (F - H) + p) * srb;
      for (int64_t c = lane; c < cb / 16; c += 32)
        *reinterpret_cast<uint4*>(dst + 16 * c) = ok ? ld_stream16(src + 16 * c) : make_uint4(0, 0, 0, 0);
      if (nsc) {
        const uint16_t* ssrc = ok ? (const uint16_t*)wrow(shot[r], scold[r], j, H, ss[r]) : nullptr;
        for (int e = lane; e < nsc; e += 32)
          reinterpret_cast<uint16_t*>(dst + cb)[e] = ok ? ld_stream_u16(ssrc + e) : (uint16_t)0;
      }
    }
  }
}

// Copies w_down_t rows of listed cold neurons from the host-memory cold tier
// into device memory at their list positions (one warp per position), so
// that the down kernel reads them from HBM.  With h (the CUDA-core path:
// h[n][b]) only rows whose h is nonzero for some token are copied, the rows
// the down kernel reads; ids outside [H, F) are skipped (it reads those, if
// in range, from the device rows).  Without h (the tensor-core path, which
// reads every listed position) every row is copied, and a bad id gets a
// zero row.
template <int WT>
__global__ void __launch_bounds__(kThreads) k_stage_cold_down(pi_layer L,
                                                              const int32_t* __restrict__ idx,
                                                              const int32_t* __restrict__ count,
                                                              const float* __restrict__ h, int B,
                                                              char* __restrict__ stg,
                                                              WsHeader* hdr) {
  pdl_wait();
  const int d = L.d_model, F = L.d_ff, H = L.hot;
  int cnt = *count;
  cnt = cnt < 0 ? 0 : (cnt > F - H ? F - H : cnt);
  const int64_t srb = stage_row_bytes(WT, d), cb = row_bytes(WT, d);
  const int nsc = WT == PI_Q4_0 ? d / 32 : 0;
  const int64_t rs = code_stride(WT, d, L.w_down_row_stride), ss = scale_stride(d, L.w_down_row_stride);
  const int lane = threadIdx.x & 31;
  const int wpb = blockDim.x >> 5;
  unsigned long long copied = 0;
  for (int p = blockIdx.x * wpb + (threadIdx.x >> 5); p < cnt; p += gridDim.x * wpb) {
    const int j = idx[p];
    const bool ok = j >= H && j < F;
    if (h) {
      if (!ok) continue;
      bool nz = false;
      for (int b = lane; b < B; b += 32) nz |= h[(size_t)(H + p) * B + b] != 0.f;
      if (!__any_sync(0xffffffffu, nz)) continue;
    }
    copied += ok;
    const char* src = ok ? wrow(L.w_down_t, L.w_down_t_cold, j, H, rs) : nullptr;
    char* dst = stg + (size_t)p * srb;
    for (int64_t c = lane; c < cb / 16; c += 32)
      *reinterpret_cast<uint4*>(dst + 16 * c) = ok ? ld_stream16(src + 16 * c) : make_uint4(0, 0, 0, 0);
    if (nsc) {
      const uint16_t* ssrc =
          ok ? (const uint16_t*)wrow(L.w_down_t_scales, L.w_down_t_cold_scales, j, H, ss) : nullptr;
      for (int e = lane; e < nsc; e += 32)
        reinterpret_cast<uint16_t*>(dst + cb)[e] = ok ? ld_stream_u16(ssrc + e) : (uint16_t)0;
    }
  }
  if (hdr && lane == 0 && copied) atomicAdd(&hdr->cold_down, copied);
}

// Split-K gathered down projection.  Grid (column tiles, S, token chunks):
// CTA (x, s, z) accumulates its slice s of the list positions [nb, N) for 8
// columns per thread and TB tokens, skipping rows whose h is 0 for all of
// its tokens, and writes its partial sums.  The slice is taken in passes of
// kDownStage positions: the CTA first lists the pass's rows with a nonzero
// h (row id and the tokens' h, in position order) in shared memory, then
// streams just those rows, several loads in flight per thread.  Rows j >= H
// come from `wdc` / `wscc` when those are set (a host-memory cold tier).
constexpr int kDownStage = 512;

template <int WT, int TB>
__global__ void __launch_bounds__(kThreads) k_ffn_down(const char* __restrict__ wd,
                                                       const uint16_t* __restrict__ wsc,
                                                       const char* __restrict__ wdc,
                                                       const uint16_t* __restrict__ wscc, int d,
                                                       int F, int H,
                                                       const int32_t* __restrict__ idx,
                                                       const int32_t* __restrict__ count,
                                                       const float* __restrict__ h, int B,
                                                       int S, float* __restrict__ part,
                                                       WsHeader* hdr, int64_t stride, int nb,
                                                       const char* __restrict__ stg) {
  pdl_wait();
  __shared__ int srow[kDownStage];  // row id, or -1 - (list position) for a staged cold row
  __shared__ float sh[kDownStage][TB];
  __shared__ int swarp[kWarps + 1];
  const int s = blockIdx.y, t0 = blockIdx.z * TB;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int col0 = (blockIdx.x * blockDim.x + tid) * 8;
  int cnt = *count;
  cnt = cnt < 0 ? 0 : (cnt > F - H ? F - H : cnt);
  const int N = H + cnt, M = N - nb;
  const int n0 = nb + (int)((int64_t)s * M / S), n1 = nb + (int)((int64_t)(s + 1) * M / S);
  float acc[TB][8];
#pragma unroll
  for (int b = 0; b < TB; ++b)
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[b][e] = 0.f;
  const int64_t rb = code_stride(WT, d, stride);
  const int64_t sbs = scale_stride(d, stride);
  unsigned long long nread = 0, ncold = 0;
  for (int p0 = n0; p0 < n1; p0 += kDownStage) {
    const int pn = min(kDownStage, n1 - p0);
    // the pass's rows with a nonzero h for some token of the chunk, in order
    int base = 0;
    for (int r0 = 0; r0 < pn; r0 += kThreads) {
      const int q = r0 + tid;
      const int n = p0 + q;
      float hv[TB];
      bool keep = false;
      int j = 0;
      if (q < pn) {
#pragma unroll
        for (int b = 0; b < TB; ++b) {
          hv[b] = (t0 + b < B) ? h[(size_t)n * B + t0 + b] : 0.f;
          keep |= hv[b] != 0.f;
        }
        j = n < H ? n : idx[n - H];
        keep = keep && j >= 0 && j < F;
      }
      const uint32_t bal = __ballot_sync(0xffffffffu, keep);
      const uint32_t cbal = __ballot_sync(0xffffffffu, keep && j >= H);
      if (lane == 0 && !stg) ncold += __popc(cbal);  // this warp's cold rows (staged: counted there)
      if (lane == 0) swarp[warp] = __popc(bal);
      __syncthreads();
      if (tid == 0) {
        int t = base;
        for (int w = 0; w < kWarps; ++w) {
          const int c = swarp[w];
          swarp[w] = t;
          t += c;
        }
        swarp[kWarps] = t;
      }
      __syncthreads();
      if (keep) {
        const int pos = swarp[warp] + __popc(bal & ((1u << lane) - 1u));
        srow[pos] = (stg && j >= H) ? -1 - (n - H) : j;
#pragma unroll
        for (int b = 0; b < TB; ++b) sh[pos][b] = hv[b];
      }
      base = swarp[kWarps];
      __syncthreads();
    }
    nread += (unsigned long long)base;
    if (col0 < d) {
#pragma unroll (WT == PI_Q4_0 ? 4 : 8)
      for (int q = 0; q < base; ++q) {
        const int j = srow[q];
        float w[8];
        const char* row = j < 0 ? stg + (size_t)(-1 - j) * stage_row_bytes(WT, d)
                                : wrow(wd, wdc, j, H, rb);
        if constexpr (WT == PI_F32) {
          const uint4 a = ld_stream16(row + (size_t)col0 * 4);
          const uint4 c = ld_stream16(row + (size_t)col0 * 4 + 16);
          w[0] = __uint_as_float(a.x); w[1] = __uint_as_float(a.y);
          w[2] = __uint_as_float(a.z); w[3] = __uint_as_float(a.w);
          w[4] = __uint_as_float(c.x); w[5] = __uint_as_float(c.y);
          w[6] = __uint_as_float(c.z); w[7] = __uint_as_float(c.w);
        } else if constexpr (WT == PI_F16) {
          f16x8_to_f32(ld_stream16(row + (size_t)col0 * 2), w);
        } else {
          const int blk = col0 >> 5, k0 = col0 & 31;
          const uint2 qv = *reinterpret_cast<const uint2*>(row + (size_t)blk * 16 + (k0 & 15));
          const uint16_t* scp =
              j < 0 ? reinterpret_cast<const uint16_t*>(row + row_bytes(WT, d))
                    : reinterpret_cast<const uint16_t*>(wrow(wsc, wscc, j, H, sbs));
          const float sc = h2f(scp[blk]);
          const int sh4 = k0 >= 16 ? 4 : 0;
          const uint32_t qq[2] = {qv.x, qv.y};
#pragma unroll
          for (int e = 0; e < 8; ++e)
            w[e] = q4_centered((qq[e >> 2] >> (8 * (e & 3) + sh4)) & 0xFu) * sc;
        }
#pragma unroll
        for (int b = 0; b < TB; ++b) {
          const float hb = sh[q][b];
#pragma unroll
          for (int e = 0; e < 8; ++e) acc[b][e] = fmaf(hb, w[e], acc[b][e]);
        }
      }
    }
  }
  if (col0 < d) {
#pragma unroll
    for (int b = 0; b < TB; ++b) {
      if (t0 + b >= B) continue;
      float* o = part + ((size_t)s * B + t0 + b) * d + col0;
      reinterpret_cast<float4*>(o)[0] = make_float4(acc[b][0], acc[b][1], acc[b][2], acc[b][3]);
      reinterpret_cast<float4*>(o)[1] = make_float4(acc[b][4], acc[b][5], acc[b][6], acc[b][7]);
    }
  }
  if (hdr && blockIdx.x == 0 && tid == 0 && nread) atomicAdd(&hdr->rows_down, nread);
  if (hdr && wdc && blockIdx.x == 0 && lane == 0 && ncold) atomicAdd(&hdr->cold_down, ncold);
}

// out = resid + (sum over the S slices in order), four floats per thread
// (n % 4 == 0; part, resid and out 16-byte aligned); the slices' loads are
// unrolled so that several are in flight at once.
__global__ void __launch_bounds__(kThreads) k_reduce(const float* __restrict__ part, int S,
                                                     int64_t n, const float* resid,
                                                     float* out) {
  pdl_wait();
  pdl_trigger();
  const int64_t n4 = n >> 2;
  const float4* p4 = reinterpret_cast<const float4*>(part);
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < n4;
       e += (int64_t)gridDim.x * blockDim.x) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 8
    for (int s = 0; s < S; ++s) {
      const float4 v = __ldcg(p4 + (size_t)s * n4 + e);
      acc.x += v.x;
      acc.y += v.y;
      acc.z += v.z;
      acc.w += v.w;
    }
    if (resid) {
      const float4 r = reinterpret_cast<const float4*>(resid)[e];
      acc = make_float4(r.x + acc.x, r.y + acc.y, r.z + acc.z, r.w + acc.w);
    }
    reinterpret_cast<float4*>(out)[e] = acc;
  }
}

__global__ void k_delay(unsigned long long ns) {
  unsigned long long t0, t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t0));
  do {
    __nanosleep(1000);
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  } while (t - t0 < ns && t >= t0);
}

template <typename K>
cudaError_t allow_smem(K kernel, size_t bytes) {
  return allow_smem_fn(reinterpret_cast<const void*>(kernel), bytes);
}

}  // namespace

// ------------------------------------------------------------------ policy

// Shared-memory opt-in: raises a kernel's dynamic shared-memory limit on the
// current device the first time a launch needs more than 48 KB (keyed by the
// kernel's address), so a warm-up call leaves nothing but launches for a
// later graph capture.
cudaError_t allow_smem_fn(const void* fn, size_t bytes) {
  if (bytes <= 48 * 1024) return cudaSuccess;
  static std::mutex mu;
  static std::unordered_map<uint64_t, size_t> granted;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) dev = 0;
  const uint64_t key = (uint64_t)(uintptr_t)fn * 131u + (uint64_t)dev;
  std::lock_guard<std::mutex> lock(mu);
  auto it = granted.find(key);
  if (it != granted.end() && it->second >= bytes) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e == cudaSuccess) granted[key] = bytes;
  return e;
}


namespace {
std::atomic<unsigned long long> g_launches{0};  // kernels launched by this library
}  // namespace

void note_launch() { g_launches.fetch_add(1ull, std::memory_order_relaxed); }
unsigned long long launches_so_far() { return g_launches.load(std::memory_order_relaxed); }

bool pdl_enabled() {
  static const bool on = [] {
    const char* e = getenv("PI_NO_PDL");
    return !(e && e[0] && e[0] != '0');
  }();
  return on;
}

int device_sms() {
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (!cache[dev]) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0)
      v = 148;
    cache[dev] = v;
  }
  return cache[dev];
}

int pick_tb(int batch, int d) {
  int tb = batch <= 1 ? 1 : (batch <= 2 ? 2 : (batch <= 4 ? 4 : 8));
  while (tb > 1 && (size_t)tb * d * 4 > 200 * 1024) tb >>= 1;
  return tb;
}

int down_tb(int batch) { return batch <= 1 ? 1 : (batch <= 2 ? 2 : (batch <= 4 ? 4 : 8)); }

// Stage sizes of a cold-tier layer: the first matrix (and ReGLU's W_up)
// when the up kernel takes more than one token chunk (a single chunk reads
// each row once anyway); the down rows when the down kernel takes four
// chunks or more: staging copies every row some token needs and the chunks
// then read it from HBM, which pays where the chunks share most of their
// rows (measured: 1.24x at 64 tokens with union masks, 0.93x at 16 tokens
// with per-token masks, whose two chunks hardly overlap).
static size_t stage_up_bytes(const pi_layer& L, int batch) {
  const int tb = pick_tb(batch, L.d_model);
  if (!L.w_up_cold || (batch + tb - 1) / tb <= 1) return 0;
  return (size_t)(L.d_ff - L.hot) * (size_t)stage_row_bytes(L.w_dtype, L.d_model) *
         (L.act == PI_REGLU ? 2u : 1u);
}
static size_t stage_down_bytes(const pi_layer& L, int batch) {
  const int tb = down_tb(batch);
  if (!L.w_up_cold || (batch + tb - 1) / tb < 4) return 0;
  return (size_t)(L.d_ff - L.hot) * (size_t)stage_row_bytes(L.w_dtype, L.d_model);
}
size_t cold_stage_bytes(const pi_layer& L, int batch) {
  return stage_up_bytes(L, batch) + stage_down_bytes(L, batch);
}

cudaError_t launch_stage_cold(const pi_layer& L, const int32_t* idx, const int32_t* count,
                              char* stage, WsHeader* hdr, cudaStream_t s) {
  const int grid = std::max(1, std::min((L.d_ff - L.hot + kWarps - 1) / kWarps, device_sms() * 4));
  const bool two = L.act == PI_REGLU;
  if (L.w_dtype == PI_F32)
    (void)launch_plain(two ? k_stage_cold<PI_F32, 2> : k_stage_cold<PI_F32, 1>, grid, kThreads, 0,
                       s, L, idx, count, stage, hdr);
  else if (L.w_dtype == PI_F16)
    (void)launch_plain(two ? k_stage_cold<PI_F16, 2> : k_stage_cold<PI_F16, 1>, grid, kThreads, 0,
                       s, L, idx, count, stage, hdr);
  else
    (void)launch_plain(two ? k_stage_cold<PI_Q4_0, 2> : k_stage_cold<PI_Q4_0, 1>, grid, kThreads, 0,
                       s, L, idx, count, stage, hdr);
  return cudaGetLastError();
}

cudaError_t launch_stage_cold_down(const pi_layer& L, int batch, const int32_t* idx,
                                   const int32_t* count, const float* h, char* stage,
                                   WsHeader* hdr, cudaStream_t s) {
  const int grid = std::max(1, std::min((L.d_ff - L.hot + kWarps - 1) / kWarps, device_sms() * 4));
  auto kern = L.w_dtype == PI_F32 ? k_stage_cold_down<PI_F32>
              : L.w_dtype == PI_F16 ? k_stage_cold_down<PI_F16> : k_stage_cold_down<PI_Q4_0>;
  (void)launch_plain(kern, grid, kThreads, 0, s, L, idx, count, h, batch, stage, hdr);
  return cudaGetLastError();
}


int down_splits(int batch, int d) {
  const int sms = device_sms();
  const int tiles = (d + 8 * kThreads - 1) / (8 * kThreads);
  const int chunks = (batch + down_tb(batch) - 1) / down_tb(batch);
  int s = (2 * sms + tiles * chunks - 1) / (tiles * chunks);
  return std::max(1, std::min(s, sms));
}

// ---------------------------------------------------------------- launches

cudaError_t launch_rmsnorm(const float* x, int batch, int d, float* xh, cudaStream_t s,
                           void* hi, void* lo, int nt) {
  // one float4 per thread up to d = 4096, then 1024 threads with up to four
  const int n4 = d / 4, threads = std::min(1024, (n4 + 31) / 32 * 32);
  (void)launch_dep(k_rmsnorm, hi ? nt : batch, threads, 0, s, x, d, xh, batch,
                   static_cast<__half*>(hi), static_cast<__half*>(lo));
  return cudaGetLastError();
}

template <int PT, int TB>
static cudaError_t pred_u_t(const pi_layer& L, const float* xh, int batch, float* u,
                            cudaStream_t s) {
  const size_t smem = (size_t)TB * L.d_model * 4;
  auto kern = k_pred_u<PT, TB>;
  cudaError_t e = allow_smem(kern, smem);
  if (e != cudaSuccess) return e;
  dim3 grid(std::min((L.rank + kWideWarps - 1) / kWideWarps, device_sms() * 2), (batch + TB - 1) / TB);
  (void)launch_plain(kern, grid, kWideThreads, smem, s, (const char*)L.p1, xh, batch, L.d_model,
                     L.rank, u);
  return cudaGetLastError();
}

cudaError_t launch_pred_u(const pi_layer& L, const float* xh, int batch, float* u,
                          cudaStream_t s) {
  const int tb = pick_tb(batch, L.d_model);
#define PI_PU(PT)                                                         \
  switch (tb) {                                                           \
    case 1: return pred_u_t<PT, 1>(L, xh, batch, u, s);                   \
    case 2: return pred_u_t<PT, 2>(L, xh, batch, u, s);                   \
    case 4: return pred_u_t<PT, 4>(L, xh, batch, u, s);                   \
    default: return pred_u_t<PT, 8>(L, xh, batch, u, s);                  \
  }
  if (L.p_dtype == PI_F32) { PI_PU(PI_F32) } else { PI_PU(PI_F16) }
#undef PI_PU
}

template <int PT, int TB>
static cudaError_t pred_z_t(const pi_layer& L, const float* u, int batch, float theta,
                            uint32_t* mask, cudaStream_t s) {
  const size_t smem = (size_t)TB * L.rank * 4;
  auto kern = k_pred_z<PT, TB>;
  cudaError_t e = allow_smem(kern, smem);
  if (e != cudaSuccess) return e;
  const int words = (L.d_ff + 31) / 32;
  dim3 grid(std::min((words + kWarps - 1) / kWarps, device_sms() * 4), (batch + TB - 1) / TB);
  (void)launch_plain(kern, grid, kThreads, smem, s, (const char*)L.p2, L.p_bias, u, batch, L.rank,
                     L.d_ff, L.hot, theta, mask, words);
  return cudaGetLastError();
}

cudaError_t launch_pred_z(const pi_layer& L, const float* u, int batch, float theta,
                          uint32_t* mask, cudaStream_t s) {
  const int tb = pick_tb(batch, L.rank);
#define PI_PZ(PT)                                                         \
  switch (tb) {                                                           \
    case 1: return pred_z_t<PT, 1>(L, u, batch, theta, mask, s);          \
    case 2: return pred_z_t<PT, 2>(L, u, batch, theta, mask, s);          \
    case 4: return pred_z_t<PT, 4>(L, u, batch, theta, mask, s);          \
    default: return pred_z_t<PT, 8>(L, u, batch, theta, mask, s);         \
  }
  if (L.p_dtype == PI_F32) { PI_PZ(PI_F32) } else { PI_PZ(PI_F16) }
#undef PI_PZ
}

cudaError_t launch_mask_union(const uint32_t* mask, int batch, int words, uint32_t* out,
                              cudaStream_t s) {
  (void)launch_plain(k_mask_union, (words + 31) / 32, 256, 0, s, mask, batch, words, out);
  return cudaGetLastError();
}

cudaError_t launch_compact(const uint32_t* mask, int batch, int d_ff, int begin, int mode,
                           int32_t* idx, int32_t* count, cudaStream_t s) {
  const int words = (d_ff + 31) / 32;
  const int unite = (mode == PI_MASK_UNION);
  const int lists = unite ? 1 : batch;
  const dim3 grid((words + kCompactWords - 1) / kCompactWords, lists);
  (void)launch_dep(k_compact, grid, kCompactWords, 0, s, mask, batch, words, d_ff, begin, unite,
                   idx, d_ff, count);
  return cudaGetLastError();
}

template <int WT, int ACT, int TB>
static cudaError_t ffn_up_t(const pi_layer& L, const float* xh, int batch, const uint32_t* mask,
                            int per_token, const int32_t* idx, const int32_t* count, float* h,
                            WsHeader* status, cudaStream_t s, int n0, const char* stg) {
  const size_t smem = (size_t)TB * L.d_model * 4;
  auto kern = k_ffn_up<WT, ACT, TB>;
  cudaError_t e = allow_smem(kern, smem);
  if (e != cudaSuccess) return e;
  constexpr int T = up_threads<WT>();
  dim3 grid(std::min((L.d_ff + T / 32 - 1) / (T / 32), device_sms() * (1024 / T)), (batch + TB - 1) / TB);
  (void)launch_plain(kern, grid, T, smem, s, L, xh, batch, mask, per_token, (L.d_ff + 31) / 32, idx,
                     count, h, status, n0, stg);
  return cudaGetLastError();
}

template <int WT, int ACT>
static cudaError_t ffn_up_a(const pi_layer& L, const float* xh, int batch, const uint32_t* mask,
                            int per_token, const int32_t* idx, const int32_t* count, float* h,
                            WsHeader* status, cudaStream_t s, int n0, char* stage) {
  const char* stg = nullptr;
  if (stage && stage_up_bytes(L, batch)) {
    const cudaError_t e = launch_stage_cold(L, idx, count, stage, status, s);
    if (e != cudaSuccess) return e;
    stg = stage;
  }
  switch (pick_tb(batch, L.d_model)) {
    case 1: return ffn_up_t<WT, ACT, 1>(L, xh, batch, mask, per_token, idx, count, h, status, s, n0, stg);
    case 2: return ffn_up_t<WT, ACT, 2>(L, xh, batch, mask, per_token, idx, count, h, status, s, n0, stg);
    case 4: return ffn_up_t<WT, ACT, 4>(L, xh, batch, mask, per_token, idx, count, h, status, s, n0, stg);
    default: return ffn_up_t<WT, ACT, 8>(L, xh, batch, mask, per_token, idx, count, h, status, s, n0, stg);
  }
}

cudaError_t launch_ffn_up(const pi_layer& L, const float* xh, int batch, const uint32_t* mask,
                          int per_token, const int32_t* idx, const int32_t* count, float* h,
                          WsHeader* status, cudaStream_t s, int n0, char* stage) {
#define PI_UP(WT)                                                                          \
  return L.act == PI_REGLU ? ffn_up_a<WT, PI_REGLU>(L, xh, batch, mask, per_token, idx,   \
                                                    count, h, status, s, n0, stage)       \
                           : ffn_up_a<WT, PI_RELU>(L, xh, batch, mask, per_token, idx,    \
                                                   count, h, status, s, n0, stage);
  if (L.w_dtype == PI_F32) { PI_UP(PI_F32) }
  if (L.w_dtype == PI_F16) { PI_UP(PI_F16) }
  PI_UP(PI_Q4_0)
#undef PI_UP
}

template <int WT, int TB>
static cudaError_t ffn_down_t(const pi_layer& L, int batch, const int32_t* idx,
                              const int32_t* count, const float* h, float* part, int S,
                              WsHeader* hdr, cudaStream_t s, int nb, const char* stg) {
  const int tiles = (L.d_model + 8 * kThreads - 1) / (8 * kThreads);
  dim3 grid(tiles, S, (batch + TB - 1) / TB);
  (void)launch_plain(k_ffn_down<WT, TB>, grid, kThreads, 0, s, (const char*)L.w_down_t,
                     (const uint16_t*)L.w_down_t_scales, (const char*)L.w_down_t_cold,
                     (const uint16_t*)L.w_down_t_cold_scales, L.d_model, L.d_ff, L.hot, idx, count, h,
                     batch, S, part, hdr, L.w_down_row_stride, nb, stg);
  return cudaGetLastError();
}

template <int WT>
static cudaError_t ffn_down_w(const pi_layer& L, int batch, const int32_t* idx,
                              const int32_t* count, const float* h, float* part, int S,
                              WsHeader* hdr, cudaStream_t s, int nb, char* stage) {
  const char* stg = nullptr;
  if (stage && stage_down_bytes(L, batch)) {
    char* dst = stage + stage_up_bytes(L, batch);
    const cudaError_t e = launch_stage_cold_down(L, batch, idx, count, h, dst, hdr, s);
    if (e != cudaSuccess) return e;
    stg = dst;
  }
  switch (down_tb(batch)) {
    case 1: return ffn_down_t<WT, 1>(L, batch, idx, count, h, part, S, hdr, s, nb, stg);
    case 2: return ffn_down_t<WT, 2>(L, batch, idx, count, h, part, S, hdr, s, nb, stg);
    case 4: return ffn_down_t<WT, 4>(L, batch, idx, count, h, part, S, hdr, s, nb, stg);
    default: return ffn_down_t<WT, 8>(L, batch, idx, count, h, part, S, hdr, s, nb, stg);
  }
}

cudaError_t launch_ffn_down(const pi_layer& L, int batch, const int32_t* idx,
                            const int32_t* count, const float* h, float* part, int splits,
                            WsHeader* hdr, cudaStream_t s, int nb, char* stage) {
  if (L.w_dtype == PI_F32)
    return ffn_down_w<PI_F32>(L, batch, idx, count, h, part, splits, hdr, s, nb, stage);
  if (L.w_dtype == PI_F16)
    return ffn_down_w<PI_F16>(L, batch, idx, count, h, part, splits, hdr, s, nb, stage);
  return ffn_down_w<PI_Q4_0>(L, batch, idx, count, h, part, splits, hdr, s, nb, stage);
}

cudaError_t launch_delay(unsigned long long ns, cudaStream_t s) {
  k_delay<<<1, 32, 0, s>>>(ns);
  note_launch();
  return cudaGetLastError();
}

cudaError_t launch_reduce(const float* part, int splits, int batch, int d, const float* resid,
                          float* out, cudaStream_t s) {
  const int64_t n = (int64_t)batch * d;  // d % 4 == 0
  const int grid = (int)std::min<int64_t>((n / 4 + kThreads - 1) / kThreads, device_sms() * 8);
  (void)launch_dep(k_reduce, grid, kThreads, 0, s, part, splits, n, resid, out);
  return cudaGetLastError();
}

}  // namespace pi
