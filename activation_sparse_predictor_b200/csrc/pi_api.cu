// C ABI of libpi (declared in include/pi.h): argument validation, workspace
// layout and the stream-ordered launch sequences of each entry point.
#include <cmath>
#include <cstddef>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <vector>

#include "pi.h"
#include "pi_common.cuh"
#include "pi_kernels.cuh"
#include "pi_stack.cuh"
#include "pi_tc.cuh"

namespace pi {
namespace {

thread_local char g_err[512] = "";

pi_status fail(pi_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof g_err, fmt, ap);
  va_end(ap);
  return st;
}

pi_status cuda_fail(cudaError_t e, const char* what) {
  return fail(PI_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }

int words_of(int F) { return (F + 31) / 32; }

bool has_cold(const pi_layer& L) {
  return L.w_gate_cold || L.w_up_cold || L.w_down_t_cold || L.w_gate_cold_scales ||
         L.w_up_cold_scales || L.w_down_t_cold_scales;
}

// Validates one layer descriptor.
pi_status check_layer(const pi_layer* L, int i) {
  if (!L) return fail(PI_ERR_INVALID, "layer %d: null descriptor", i);
  const int d = L->d_model, F = L->d_ff, r = L->rank, H = L->hot;
  if (d < 1 || d > PI_MAX_D_MODEL) return fail(PI_ERR_INVALID, "layer %d: d_model %d out of range", i, d);
  if (F < 1 || F > PI_MAX_D_FF) return fail(PI_ERR_INVALID, "layer %d: d_ff %d out of range", i, F);
  if (r < 1 || r > PI_MAX_RANK) return fail(PI_ERR_INVALID, "layer %d: rank %d out of range", i, r);
  if (H < 0 || H > F) return fail(PI_ERR_INVALID, "layer %d: hot %d not in [0, d_ff]", i, H);
  if (L->act != PI_RELU && L->act != PI_REGLU && L->act != PI_RELU2)
    return fail(PI_ERR_INVALID, "layer %d: unknown activation %d", i, L->act);
  if (L->w_dtype != PI_F32 && L->w_dtype != PI_F16 && L->w_dtype != PI_Q4_0)
    return fail(PI_ERR_INVALID, "layer %d: unknown weight dtype %d", i, L->w_dtype);
  if (L->p_dtype == PI_Q4_0)
    return fail(PI_ERR_UNSUPPORTED, "layer %d: Q4_0 predictor weights are not supported", i);
  if (L->p_dtype != PI_F32 && L->p_dtype != PI_F16)
    return fail(PI_ERR_INVALID, "layer %d: unknown predictor dtype %d", i, L->p_dtype);
  const int dmul = L->w_dtype == PI_Q4_0 ? 32 : 8;
  if (d % dmul) return fail(PI_ERR_INVALID, "layer %d: d_model %d not a multiple of %d", i, d, dmul);
  if (L->p_dtype == PI_F32 ? (d % 4) : (d % 8))
    return fail(PI_ERR_INVALID, "layer %d: d_model %d not a multiple of the predictor chunk", i, d);
  if (L->p_dtype == PI_F32 ? (r % 4) : (r % 8))
    return fail(PI_ERR_INVALID, "layer %d: rank %d not a multiple of %d", i, r,
                L->p_dtype == PI_F32 ? 4 : 8);
  const bool reglu = L->act == PI_REGLU, q4 = L->w_dtype == PI_Q4_0;
  if (!L->w_up || !L->w_down_t || !L->p1 || !L->p2 || (reglu && !L->w_gate))
    return fail(PI_ERR_INVALID, "layer %d: null weight pointer", i);
  if (q4 && (!L->w_up_scales || !L->w_down_t_scales || (reglu && !L->w_gate_scales)))
    return fail(PI_ERR_INVALID, "layer %d: Q4_0 weights need scale arrays", i);
  const void* w16[] = {L->w_up, L->w_down_t, L->p1, L->p2, reglu ? L->w_gate : L->w_up};
  for (const void* p : w16)
    if (!aligned(p, 16)) return fail(PI_ERR_INVALID, "layer %d: weight pointer not 16-byte aligned", i);
  if (q4) {
    const void* s2[] = {L->w_up_scales, L->w_down_t_scales, reglu ? L->w_gate_scales : L->w_up_scales};
    for (const void* p : s2)
      if (!aligned(p, 2)) return fail(PI_ERR_INVALID, "layer %d: scale pointer not 2-byte aligned", i);
  }
  if ((L->bias && !aligned(L->bias, 4)) || (L->p_bias && !aligned(L->p_bias, 4)))
    return fail(PI_ERR_INVALID, "layer %d: bias pointer not 4-byte aligned", i);
  const int64_t codes = row_bytes(L->w_dtype, d);
  if (!reglu && L->w_up_row_stride)
    return fail(PI_ERR_INVALID, "layer %d: w_up_row_stride is for ReGLU layers only", i);
  const int64_t strides[3] = {L->w_row_stride, L->w_down_row_stride, L->w_up_row_stride};
  for (int64_t st : strides)
    if (st != 0 && (st < codes || st % 16 != 0))
      return fail(PI_ERR_INVALID, "layer %d: row stride %lld must be 0 or a multiple of 16 >= %lld",
                  i, (long long)st, (long long)codes);
  if (has_cold(*L)) {
    if (!L->w_up_cold || !L->w_down_t_cold || (reglu && !L->w_gate_cold))
      return fail(PI_ERR_INVALID, "layer %d: cold tier needs w_up_cold, w_down_t_cold%s", i,
                  reglu ? " and w_gate_cold" : "");
    if (q4 && (!L->w_up_cold_scales || !L->w_down_t_cold_scales || (reglu && !L->w_gate_cold_scales)))
      return fail(PI_ERR_INVALID, "layer %d: Q4_0 cold tier needs its scale arrays", i);
    if (!aligned(L->w_up_cold, 16) || !aligned(L->w_down_t_cold, 16) || !aligned(L->w_gate_cold, 16))
      return fail(PI_ERR_INVALID, "layer %d: cold-tier pointer not 16-byte aligned", i);
    if (!aligned(L->w_up_cold_scales, 2) || !aligned(L->w_down_t_cold_scales, 2) ||
        !aligned(L->w_gate_cold_scales, 2))
      return fail(PI_ERR_INVALID, "layer %d: cold-tier scale pointer not 2-byte aligned", i);
  }
  return PI_OK;
}

// The layers as the kernels read them: a layer with a host-memory cold tier
// gets the device addresses of its cold rows (cudaPointerGetAttributes;
// page-locked memory the current device can address, else PI_ERR_INVALID).
// Layers without one are passed through untouched (*out = in, no copy).
pi_status cold_resolve(const pi_layer* in, int n, std::vector<pi_layer>& store,
                       const pi_layer** out) {
  *out = in;
  bool any = false;
  for (int l = 0; l < n; ++l) any = any || has_cold(in[l]);
  if (!any) return PI_OK;
  store.assign(in, in + n);
  for (int l = 0; l < n; ++l) {
    pi_layer& L = store[l];
    const void** ptrs[6] = {&L.w_gate_cold, &L.w_up_cold, &L.w_down_t_cold,
                            &L.w_gate_cold_scales, &L.w_up_cold_scales, &L.w_down_t_cold_scales};
    for (const void** p : ptrs) {
      if (!*p) continue;
      cudaPointerAttributes a{};
      const cudaError_t e = cudaPointerGetAttributes(&a, *p);
      if (e != cudaSuccess) {
        (void)cudaGetLastError();
        return fail(PI_ERR_INVALID, "layer %d: cold-tier pointer %p: %s", l, *p, cudaGetErrorString(e));
      }
      if (a.type != cudaMemoryTypeHost || !a.devicePointer)
        return fail(PI_ERR_INVALID,
                    "layer %d: cold-tier pointer %p is not page-locked host memory mapped for "
                    "this device", l, *p);
      *p = a.devicePointer;
    }
  }
  *out = store.data();
  return PI_OK;
}

WsLayout layout_for(int d, int F, int r, int batch, int H, size_t stage_bytes = 0) {
  WsLayout w{};
  size_t off = sizeof(WsHeader);
  auto take = [&](size_t bytes) { size_t o = off; off = align256(off + bytes); return o; };
  w.splits = down_splits(batch, d);
  w.xh = take((size_t)batch * d * 4);
  w.u = take((size_t)batch * r * 4);
  w.mask = take((size_t)(batch > 2 ? batch : 2) * words_of(F) * 4);
  w.idx = take((size_t)F * 4);
  w.count = take(16);
  w.h = take((size_t)F * batch * 4);
  // split-K partials: the multi-kernel split, or one row per SM for the
  // fused single-token stack
  // (+ up to 8 slices of the tensor-core down projection at token batches)
  const size_t tcp = tc_scratch_bytes(d, F, r, batch) ? (size_t)8 * batch : 0;
  const size_t parts = (size_t)w.splits * batch + tcp > (size_t)device_sms()
                           ? (size_t)w.splits * batch + tcp
                           : (size_t)device_sms();
  w.part = take(parts * d * 4);
  w.y = take((size_t)batch * d * 4);
  w.tc = take(tc_scratch_bytes(d, F, r, batch));
  w.cta = take(4 * (size_t)device_sms());
  w.stage_bytes = stage_bytes;
  w.stage = take(stage_bytes);
  w.total = off;
  return w;
}

WsLayout layout_for_layers(const pi_layer* layers, int n, int batch) {
  int d = 0, F = 0, r = 0, H = 0;
  size_t stage = 0;
  for (int l = 0; l < n; ++l) {
    const size_t sb = ffn_tc_supported(layers[l], batch) ? tc_cold_stage_bytes(layers[l])
                                                         : cold_stage_bytes(layers[l], batch);
    stage = stage > sb ? stage : sb;
    d = d > layers[l].d_model ? d : layers[l].d_model;
    F = F > layers[l].d_ff ? F : layers[l].d_ff;
    r = r > layers[l].rank ? r : layers[l].rank;
    H = H > layers[l].hot ? H : layers[l].hot;
  }
  return layout_for(d, F, r, batch, H, stage);
}

pi_status check_ws(void* ws, size_t ws_bytes, const WsLayout& lay) {
  if (!ws) return fail(PI_ERR_INVALID, "null workspace");
  if (!aligned(ws, 256)) return fail(PI_ERR_INVALID, "workspace not 256-byte aligned");
  if (ws_bytes < lay.total)
    return fail(PI_ERR_INVALID, "workspace too small: %zu < %zu bytes", ws_bytes, lay.total);
  return PI_OK;
}

template <typename T>
T* at(void* ws, size_t off) { return reinterpret_cast<T*>((char*)ws + off); }

WsHeader* header(void* ws) { return reinterpret_cast<WsHeader*>(ws); }
uint32_t* status_word(void* ws) { return &header(ws)->status; }

float logit32(float tau) { return (float)std::log((double)tau / (1.0 - (double)tau)); }

// Optional per-launch event recorder used by pi_ffn_stack_profile.
struct Prof {
  cudaEvent_t* ev = nullptr;  // 2 per launch
  int* kind = nullptr;
  int cap = 0, n = 0;
  cudaStream_t s = nullptr;
  void before(int k) {
    if (!ev || n >= cap) return;
    kind[n] = k;
    cudaEventRecord(ev[2 * n], s);
  }
  void after() {
    if (!ev || n >= cap) return;
    cudaEventRecord(ev[2 * n + 1], s);
    ++n;
  }
};

pi_status ffn_body(const pi_layer& L, const float* xh, int batch, const uint32_t* mask,
                   int per_token, const int32_t* idx, const int32_t* count, const float* resid,
                   float* out, void* ws, const WsLayout& lay, cudaStream_t s,
                   Prof* prof = nullptr, bool xh16_ready = false) {
  Prof none;
  Prof& P = prof ? *prof : none;
  const int S = down_splits(batch, L.d_model);
  float* part = at<float>(ws, lay.part);
  int St = S;  // split-K slices to reduce
  cudaError_t e = cudaSuccess;
  // a host-memory cold tier's rows are staged in the workspace when it has
  // room for them (it does when sized by pi_workspace_bytes for these layers)
  char* stage = lay.stage_bytes ? at<char>(ws, lay.stage) : nullptr;
  if (ffn_tc_supported(L, batch) && lay.stage_bytes >= tc_cold_stage_bytes(L)) {
    // token batches: both contractions over the listed rows on the tensor cores
    P.before(PI_KIND_FFN_UP);
    e = launch_ffn_up_tc(L, xh, batch, mask, idx, count, at<void>(ws, lay.tc), header(ws), s,
                         xh16_ready, stage);
    P.after();
    if (e != cudaSuccess) return cuda_fail(e, "ffn up (tensor cores) launch");
    P.before(PI_KIND_FFN_DOWN);
    St = ffn_tc_down_splits(L);
    e = launch_ffn_down_tc(L, batch, idx, count, part, at<void>(ws, lay.tc), header(ws), s, stage);
    P.after();
    if (e != cudaSuccess) return cuda_fail(e, "ffn down (tensor cores) launch");
  } else {
    P.before(PI_KIND_FFN_UP);
    if (lay.stage_bytes < cold_stage_bytes(L, batch)) stage = nullptr;  // read the host rows directly
    e = launch_ffn_up(L, xh, batch, mask, per_token, idx, count, at<float>(ws, lay.h), header(ws), s,
                      0, stage);
    P.after();
    if (e != cudaSuccess) return cuda_fail(e, "ffn_up launch");
    P.before(PI_KIND_FFN_DOWN);
    e = launch_ffn_down(L, batch, idx, count, at<float>(ws, lay.h), part, S, header(ws), s, 0,
                        stage);
    P.after();
    if (e != cudaSuccess) return cuda_fail(e, "ffn_down launch");
  }
  P.before(PI_KIND_REDUCE);
  e = launch_reduce(part, St, batch, L.d_model, resid, out, s);
  P.after();
  if (e != cudaSuccess) return cuda_fail(e, "reduce launch");
  return PI_OK;
}

// mask [batch][words] of xh: the predictor (tensor cores at token batches).
// `uni` (optional): the tensor-core predictor also writes there the OR of
// the tokens' words from the word holding `hot` on; *uni_done says whether
// it did.
pi_status predict_body(const pi_layer& L, const float* xh, int batch, float theta, uint32_t* mask,
                       void* ws, const WsLayout& lay, cudaStream_t s, Prof* prof = nullptr,
                       uint32_t* uni = nullptr, bool* uni_done = nullptr, bool split_ready = false) {
  Prof none;
  Prof& P = prof ? *prof : none;
  cudaError_t e;
  if (uni_done) *uni_done = false;
  if (pred_tc_supported(L, batch)) {
    P.before(PI_KIND_PRED_U);
    e = launch_predict_tc(L, xh, batch, theta, mask, at<void>(ws, lay.tc), header(ws), s, uni,
                          split_ready);
    if (uni_done) *uni_done = uni != nullptr;
    P.after();
    return e == cudaSuccess ? PI_OK : cuda_fail(e, "predictor (tensor cores) launch");
  }
  P.before(PI_KIND_PRED_U);
  e = launch_pred_u(L, xh, batch, at<float>(ws, lay.u), s);
  P.after();
  if (e != cudaSuccess) return cuda_fail(e, "pred_u launch");
  P.before(PI_KIND_PRED_Z);
  e = launch_pred_z(L, at<float>(ws, lay.u), batch, theta, mask, s);
  P.after();
  return e == cudaSuccess ? PI_OK : cuda_fail(e, "pred_z launch");
}

pi_status stack_check(const pi_layer* layers, int n_layers, float* x, int batch, float tau,
                      int mode, uint32_t* mask_trace, void* ws, size_t ws_bytes, WsLayout* lay) {
  if (!layers || n_layers < 1) return fail(PI_ERR_INVALID, "need at least one layer");
  pi_status st;
  for (int l = 0; l < n_layers; ++l) {
    if ((st = check_layer(&layers[l], l)) != PI_OK) return st;
    if (layers[l].d_model != layers[0].d_model || layers[l].d_ff != layers[0].d_ff)
      return fail(PI_ERR_INVALID, "layer %d: all layers must share d_model and d_ff", l);
  }
  if (batch < 1 || batch > PI_MAX_BATCH) return fail(PI_ERR_INVALID, "batch %d not in [1, 64]", batch);
  if (!(tau > 0.f && tau < 1.f)) return fail(PI_ERR_INVALID, "tau must lie in (0, 1)");
  if (mode != PI_MASK_PER_TOKEN && mode != PI_MASK_UNION) return fail(PI_ERR_INVALID, "unknown mask mode %d", mode);
  if (!x || !aligned(x, 16)) return fail(PI_ERR_INVALID, "x null or not 16-byte aligned");
  if (mask_trace && !aligned(mask_trace, 4)) return fail(PI_ERR_INVALID, "mask_trace misaligned");
  *lay = layout_for_layers(layers, n_layers, batch);
  return check_ws(ws, ws_bytes, *lay);
}

pi_status stack_run(const pi_layer* layers, int n_layers, float* x, int batch, float tau,
                    int mode, uint32_t* mask_trace, void* ws, const WsLayout& lay,
                    cudaStream_t s, Prof* prof, unsigned long long* trace = nullptr,
                    unsigned long long* utrace = nullptr) {
  Prof none;
  Prof& P = prof ? *prof : none;
  pi_status st;
  const float theta = logit32(tau);
  // the fused single-token kernel over the stack for the token at xt
  auto fused = [&](float* xt, uint32_t* trace_l0) -> pi_status {
    const int words = words_of(layers[0].d_ff), chunk = stack1_chunk();
    for (int l0 = 0; l0 < n_layers; l0 += chunk) {
      const int n = n_layers - l0 < chunk ? n_layers - l0 : chunk;
      P.before(PI_KIND_FUSED);
      cudaError_t e = launch_stack1(layers + l0, n, xt,
                                    trace_l0 ? trace_l0 + (size_t)l0 * words : nullptr, ws,
                                    lay, theta, s, trace ? trace + (size_t)l0 * device_sms() * 16 : nullptr,
                                    utrace ? utrace + (size_t)l0 * stack1_unit_trace_len() * 4 : nullptr);
      P.after();
      if (e != cudaSuccess) return cuda_fail(e, "fused stack launch");
      note_launch();
    }
    return PI_OK;
  };
  if (stack1_supported(layers, n_layers, batch)) return fused(x, mask_trace);
  // Q4_0 stacks with per-token masks below 5 tokens (or where the layers
  // do not qualify for the tensor cores): each token's per-token FFN is the
  // single-token computation on that token, and one fused pass per token
  // (Llama2-70B shape: 3.5 ms, 286 tokens/s) costs less than a batched step
  // there (262 tokens/s at 4 tokens on the tensor cores, 377 at 6; 97 at 4
  // on the CUDA-core kernels, which dequantize every weight block to fp32
  // for every token).  A mask trace
  // keeps the batched path, whose trace layout is [layer][token][word].
  if (batch > 1 && mode == PI_MASK_PER_TOKEN && !mask_trace && !trace &&
      layers[0].w_dtype == PI_Q4_0 && stack1_supported(layers, n_layers, 1) &&
      (batch < 5 || !ffn_tc_supported(layers[0], batch))) {
    const int d = layers[0].d_model;
    for (int b = 0; b < batch; ++b) {
      if ((st = fused(x + (size_t)b * d, nullptr)) != PI_OK) return st;
    }
    return PI_OK;
  }
  const int d = layers[0].d_model, words = words_of(layers[0].d_ff);
  const int per_token = (mode == PI_MASK_PER_TOKEN && batch > 1);
  float* xh = at<float>(ws, lay.xh);
  int32_t* idx = at<int32_t>(ws, lay.idx);
  int32_t* cnt = at<int32_t>(ws, lay.count);
  for (int l = 0; l < n_layers; ++l) {
    const pi_layer& L = layers[l];
    uint32_t* mask = mask_trace ? mask_trace + (size_t)l * batch * words : at<uint32_t>(ws, lay.mask);
    // with the tensor-core predictor, the RMSNorm also writes its fp16 operands
    const bool ptc = pred_tc_supported(L, batch);
    void *hi = nullptr, *lo = nullptr;
    if (ptc) tc_split_buffers(L, at<void>(ws, lay.tc), &hi, &lo);
    P.before(PI_KIND_RMSNORM);
    cudaError_t e = launch_rmsnorm(x, batch, d, xh, s, hi, lo, (batch + 15) / 16 * 16);
    P.after();
    if (e != cudaSuccess) return cuda_fail(e, "rmsnorm launch");
    // at token batches the tokens' union goes into the activation buffer
    // (free until the up projection): from the tensor-core predictor's
    // epilogue, else from a union kernel; then one list from it
    uint32_t* uni = batch > 1 ? at<uint32_t>(ws, lay.h) : nullptr;
    bool uni_done = false;
    if ((st = predict_body(L, xh, batch, theta, mask, ws, lay, s, prof, uni, &uni_done, ptc)) != PI_OK)
      return st;
    P.before(PI_KIND_COMPACT);
    if (batch > 1) {
      e = uni_done ? cudaSuccess : launch_mask_union(mask, batch, words, uni, s);
      if (e == cudaSuccess) e = launch_compact(uni, 1, L.d_ff, L.hot, PI_MASK_UNION, idx, cnt, s);
    } else {
      e = launch_compact(mask, batch, L.d_ff, L.hot, PI_MASK_UNION, idx, cnt, s);
    }
    P.after();
    if (e != cudaSuccess) return cuda_fail(e, "compact launch");
    // the tensor-core predictor leaves the fp16 copy of xh the FFN reads
    if ((st = ffn_body(L, xh, batch, per_token ? mask : nullptr, per_token, idx, cnt, x, x, ws,
                       lay, s, prof, pred_tc_supported(L, batch))) != PI_OK)
      return st;
  }
  return PI_OK;
}

}  // namespace
}  // namespace pi

// Scratch of pi_predict_noalloc: the predictor's hidden vector u for
// batch * rank <= PI_PREDICT_NOALLOC_MAX_FLOATS, one copy per device (part of
// the module image, so it takes no allocation at run time).
static __device__ __align__(256) float g_predict_u[PI_PREDICT_NOALLOC_MAX_FLOATS];

namespace pi {
namespace {

// Device address of g_predict_u on the current device.  Looked up once per
// device, by the first pi_predict_noalloc call made with that device current,
// and kept for the life of the process (a cudaDeviceReset would make it stale;
// the header tells callers not to use this entry point across one).
pi_status predict_scratch(float** out) {
  static std::mutex mu;
  static float* addr[64] = {};
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= 64) return fail(PI_ERR_UNSUPPORTED, "device %d: at most 64 devices", dev);
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_predict_u);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress of the predictor scratch");
    addr[dev] = static_cast<float*>(p);
  }
  *out = addr[dev];
  return PI_OK;
}

}  // namespace
}  // namespace pi

using namespace pi;

extern "C" {

int pi_version(void) { return PI_VERSION; }

const char* pi_last_error(void) { return g_err; }

const char* pi_status_string(int status) {
  switch (status) {
    case PI_OK: return "PI_OK";
    case PI_ERR_INVALID: return "PI_ERR_INVALID";
    case PI_ERR_UNSUPPORTED: return "PI_ERR_UNSUPPORTED";
    case PI_ERR_CUDA: return "PI_ERR_CUDA";
    case PI_ERR_TIMEOUT: return "PI_ERR_TIMEOUT";
    case PI_ERR_DEVICE_CHECK: return "PI_ERR_DEVICE_CHECK";
    default: return "PI_ERR_UNKNOWN";
  }
}

size_t pi_workspace_bytes(const pi_layer* layers, int n_layers, int batch) {
  if (!layers || n_layers < 1 || batch < 1 || batch > PI_MAX_BATCH) return 0;
  for (int l = 0; l < n_layers; ++l)
    if (check_layer(&layers[l], l) != PI_OK) return 0;
  return layout_for_layers(layers, n_layers, batch).total;
}

pi_status pi_workspace_init(void* ws, size_t ws_bytes, void* stream) {
  if (!ws || !aligned(ws, 256) || ws_bytes < sizeof(WsHeader))
    return fail(PI_ERR_INVALID, "workspace must be 256-byte aligned and >= 256 bytes");
  cudaError_t e = cudaMemsetAsync(ws, 0, sizeof(WsHeader), (cudaStream_t)stream);
  return e == cudaSuccess ? PI_OK : cuda_fail(e, "workspace init");
}

pi_status pi_predict(const pi_layer* layer, const float* xh, int batch, float tau,
                     uint32_t* mask, void* ws, size_t ws_bytes, void* stream) {
  pi_status st = check_layer(layer, 0);
  if (st != PI_OK) return st;
  if (batch < 1 || batch > PI_MAX_BATCH) return fail(PI_ERR_INVALID, "batch %d not in [1, 64]", batch);
  if (!(tau > 0.f && tau < 1.f)) return fail(PI_ERR_INVALID, "tau must lie in (0, 1)");
  if (!xh || !aligned(xh, 16)) return fail(PI_ERR_INVALID, "xh null or not 16-byte aligned");
  if (!mask || !aligned(mask, 4)) return fail(PI_ERR_INVALID, "mask null or misaligned");
  const WsLayout lay = layout_for_layers(layer, 1, batch);
  if ((st = check_ws(ws, ws_bytes, lay)) != PI_OK) return st;
  return predict_body(*layer, xh, batch, logit32(tau), mask, ws, lay, (cudaStream_t)stream);
}

pi_status pi_predict_noalloc(const pi_layer* layer, const float* xh, int batch, float tau,
                             uint32_t* mask, void* stream) {
  pi_status st = check_layer(layer, 0);
  if (st != PI_OK) return st;
  if (batch < 1 || batch > PI_MAX_BATCH) return fail(PI_ERR_INVALID, "batch %d not in [1, 64]", batch);
  if (!(tau > 0.f && tau < 1.f)) return fail(PI_ERR_INVALID, "tau must lie in (0, 1)");
  if (!xh || !aligned(xh, 16)) return fail(PI_ERR_INVALID, "xh null or not 16-byte aligned");
  if (!mask || !aligned(mask, 4)) return fail(PI_ERR_INVALID, "mask null or misaligned");
  const long long need = (long long)batch * layer->rank;
  if (need > PI_PREDICT_NOALLOC_MAX_FLOATS)
    return fail(PI_ERR_INVALID,
                "pi_predict_noalloc: batch * rank = %lld exceeds its static scratch of %d floats; "
                "use pi_predict with a workspace",
                need, PI_PREDICT_NOALLOC_MAX_FLOATS);
  float* u = nullptr;
  if ((st = predict_scratch(&u)) != PI_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e = launch_pred_u(*layer, xh, batch, u, s);
  if (e != cudaSuccess) return cuda_fail(e, "pred_u launch");
  e = launch_pred_z(*layer, u, batch, logit32(tau), mask, s);
  if (e != cudaSuccess) return cuda_fail(e, "pred_z launch");
  return PI_OK;
}

pi_status pi_compact(const uint32_t* mask, int batch, int d_ff, int begin, int mode,
                     int32_t* idx, int32_t* count, void* stream) {
  if (batch < 1 || batch > PI_MAX_BATCH) return fail(PI_ERR_INVALID, "batch %d not in [1, 64]", batch);
  if (d_ff < 1 || d_ff > PI_MAX_D_FF) return fail(PI_ERR_INVALID, "d_ff %d out of range", d_ff);
  if (begin < 0 || begin > d_ff) return fail(PI_ERR_INVALID, "begin %d not in [0, d_ff]", begin);
  if (mode != PI_MASK_PER_TOKEN && mode != PI_MASK_UNION) return fail(PI_ERR_INVALID, "unknown mask mode %d", mode);
  if (!mask || !idx || !count || !aligned(mask, 4) || !aligned(idx, 4) || !aligned(count, 4))
    return fail(PI_ERR_INVALID, "null or misaligned mask/idx/count");
  cudaError_t e = launch_compact(mask, batch, d_ff, begin, mode, idx, count, (cudaStream_t)stream);
  return e == cudaSuccess ? PI_OK : cuda_fail(e, "compact launch");
}

pi_status pi_sparse_ffn(const pi_layer* layer, const float* xh, int batch, const uint32_t* mask,
                        const int32_t* idx, const int32_t* count, int mode, float* y, void* ws,
                        size_t ws_bytes, void* stream) {
  pi_status st = check_layer(layer, 0);
  if (st != PI_OK) return st;
  if (batch < 1 || batch > PI_MAX_BATCH) return fail(PI_ERR_INVALID, "batch %d not in [1, 64]", batch);
  if (mode != PI_MASK_PER_TOKEN && mode != PI_MASK_UNION) return fail(PI_ERR_INVALID, "unknown mask mode %d", mode);
  if (!xh || !aligned(xh, 16)) return fail(PI_ERR_INVALID, "xh null or not 16-byte aligned");
  if (!y || !aligned(y, 16)) return fail(PI_ERR_INVALID, "y null or not 16-byte aligned");
  if (!idx || !count || !aligned(idx, 4) || !aligned(count, 4))
    return fail(PI_ERR_INVALID, "null or misaligned idx/count");
  const int per_token = (mode == PI_MASK_PER_TOKEN && batch > 1);
  if (per_token && (!mask || !aligned(mask, 4)))
    return fail(PI_ERR_INVALID, "per-token mode with batch > 1 needs the mask");
  const WsLayout lay = layout_for_layers(layer, 1, batch);
  if ((st = check_ws(ws, ws_bytes, lay)) != PI_OK) return st;
  std::vector<pi_layer> store;
  const pi_layer* kl;
  if ((st = cold_resolve(layer, 1, store, &kl)) != PI_OK) return st;
  return ffn_body(*kl, xh, batch, per_token ? mask : nullptr, per_token, idx, count, nullptr, y,
                  ws, lay, (cudaStream_t)stream);
}

pi_status pi_ffn_stack(const pi_layer* layers, int n_layers, float* x, int batch, float tau,
                       int mode, uint32_t* mask_trace, void* ws, size_t ws_bytes, void* stream) {
  WsLayout lay;
  pi_status st = stack_check(layers, n_layers, x, batch, tau, mode, mask_trace, ws, ws_bytes, &lay);
  if (st != PI_OK) return st;
  std::vector<pi_layer> store;
  const pi_layer* kl;
  if ((st = cold_resolve(layers, n_layers, store, &kl)) != PI_OK) return st;
  return stack_run(kl, n_layers, x, batch, tau, mode, mask_trace, ws, lay, (cudaStream_t)stream,
                   nullptr);
}

const char* pi_kind_name(int kind) {
  static const char* names[PI_KINDS] = {"rmsnorm", "pred_u",   "pred_z", "compact",
                                        "ffn_up",  "ffn_down", "reduce", "fused_stack"};
  return (kind >= 0 && kind < PI_KINDS) ? names[kind] : "unknown";
}

pi_status pi_ffn_stack_profile(const pi_layer* layers, int n_layers, float* x, int batch,
                               float tau, int mode, uint32_t* mask_trace, void* ws,
                               size_t ws_bytes, void* stream, float* kind_ms,
                               int* kind_launches) {
  WsLayout lay;
  pi_status st = stack_check(layers, n_layers, x, batch, tau, mode, mask_trace, ws, ws_bytes, &lay);
  if (st != PI_OK) return st;
  std::vector<pi_layer> store;
  const pi_layer* kl;
  if ((st = cold_resolve(layers, n_layers, store, &kl)) != PI_OK) return st;
  layers = kl;
  cudaStream_t s = (cudaStream_t)stream;
  Prof P;
  P.cap = n_layers * 8;
  P.s = s;
  P.ev = new cudaEvent_t[2 * P.cap];
  P.kind = new int[P.cap];
  int made = 0;
  cudaError_t e = cudaSuccess;
  for (; made < 2 * P.cap && e == cudaSuccess; ++made) e = cudaEventCreate(&P.ev[made]);
  if (e == cudaSuccess) e = launch_delay(2000000ull, s);
  if (e != cudaSuccess) st = cuda_fail(e, "profile setup");
  if (st == PI_OK) st = stack_run(layers, n_layers, x, batch, tau, mode, mask_trace, ws, lay, s, &P);
  if (st == PI_OK && (e = cudaStreamSynchronize(s)) != cudaSuccess) st = cuda_fail(e, "profile sync");
  if (st == PI_OK) {
    float ms[PI_KINDS] = {0};
    int cnt[PI_KINDS] = {0};
    for (int i = 0; i < P.n; ++i) {
      float t = 0.f;
      if (cudaEventElapsedTime(&t, P.ev[2 * i], P.ev[2 * i + 1]) == cudaSuccess) {
        ms[P.kind[i]] += t;
        cnt[P.kind[i]] += 1;
      }
    }
    for (int k = 0; k < PI_KINDS; ++k) {
      if (kind_ms) kind_ms[k] = ms[k];
      if (kind_launches) kind_launches[k] = cnt[k];
    }
  }
  for (int i = 0; i < made; ++i) cudaEventDestroy(P.ev[i]);
  delete[] P.ev;
  delete[] P.kind;
  return st;
}

pi_status pi_ffn_stack_timeline(const pi_layer* layers, int n_layers, float* x, float tau,
                                void* ws, size_t ws_bytes, void* stream,
                                unsigned long long* timeline, unsigned long long* unit_timeline) {
  WsLayout lay;
  pi_status st = stack_check(layers, n_layers, x, 1, tau, PI_MASK_UNION, nullptr, ws, ws_bytes, &lay);
  if (st != PI_OK) return st;
  if (!timeline || !aligned(timeline, 8)) return fail(PI_ERR_INVALID, "timeline null or misaligned");
  if (!stack1_supported(layers, n_layers, 1))
    return fail(PI_ERR_UNSUPPORTED, "these layers do not run on the persistent kernel");
  return stack_run(layers, n_layers, x, 1, tau, PI_MASK_UNION, nullptr, ws, lay,
                   (cudaStream_t)stream, nullptr, timeline, unit_timeline);
}

int pi_device_sms(void) { return device_sms(); }

unsigned long long pi_kernel_launches(void) { return launches_so_far(); }

pi_status pi_wait_selftest(void* ws, size_t ws_bytes, int kind, unsigned timeout_us, void* stream) {
  if (!ws || !aligned(ws, 256) || ws_bytes < sizeof(WsHeader))
    return fail(PI_ERR_INVALID, "workspace null, misaligned or smaller than its header");
  if (kind != 0 && kind != 1) return fail(PI_ERR_INVALID, "kind %d not 0 (mbarrier) or 1 (grid)", kind);
  if (timeout_us < 1 || timeout_us > 10000000u)
    return fail(PI_ERR_INVALID, "timeout %u us not in [1, 1e7]", timeout_us);
  cudaError_t e = launch_wait_selftest(ws, kind, 1000ull * timeout_us, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "wait self-test launch");
  note_launch();
  return PI_OK;
}

pi_status pi_read_counters(void* ws, void* stream, int clear, uint64_t* out) {
  if (!ws || !aligned(ws, 256) || !out) return fail(PI_ERR_INVALID, "workspace or output null");
  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "stream synchronize");
  unsigned long long v[3];
  static_assert(offsetof(WsHeader, rows_second) == offsetof(WsHeader, rows_listed) + 16,
                "counters are adjacent");
  e = cudaMemcpy(v, &header(ws)->rows_listed, sizeof v, cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "counter read");
  if (clear && (e = cudaMemset(&header(ws)->rows_listed, 0, sizeof v)) != cudaSuccess)
    return cuda_fail(e, "counter clear");
  out[0] = v[0];
  out[1] = v[1];
  out[2] = v[2];
  return PI_OK;
}

pi_status pi_read_cold_counters(void* ws, void* stream, int clear, uint64_t* out) {
  if (!ws || !aligned(ws, 256) || !out) return fail(PI_ERR_INVALID, "workspace or output null");
  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "stream synchronize");
  unsigned long long v[3];
  static_assert(offsetof(WsHeader, cold_second) == offsetof(WsHeader, cold_listed) + 16,
                "counters are adjacent");
  e = cudaMemcpy(v, &header(ws)->cold_listed, sizeof v, cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "counter read");
  if (clear && (e = cudaMemset(&header(ws)->cold_listed, 0, sizeof v)) != cudaSuccess)
    return cuda_fail(e, "counter clear");
  for (int k = 0; k < 3; ++k) out[k] = v[k];
  return PI_OK;
}

pi_status pi_read_list(const pi_layer* layers, int n_layers, int batch, void* ws,
                       size_t ws_bytes, void* stream, int32_t* idx_out, int cap,
                       int32_t* count_out) {
  if (!layers || n_layers < 1) return fail(PI_ERR_INVALID, "need at least one layer");
  if (batch < 1 || batch > PI_MAX_BATCH) return fail(PI_ERR_INVALID, "batch %d not in [1, 64]", batch);
  pi_status st;
  for (int l = 0; l < n_layers; ++l)
    if ((st = check_layer(&layers[l], l)) != PI_OK) return st;
  if (!count_out || cap < 0 || (cap > 0 && !idx_out))
    return fail(PI_ERR_INVALID, "null count_out, negative cap or null idx_out");
  const WsLayout lay = layout_for_layers(layers, n_layers, batch);
  if ((st = check_ws(ws, ws_bytes, lay)) != PI_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "stream synchronize");
  int32_t n = 0;
  e = cudaMemcpy(&n, at<int32_t>(ws, lay.count), sizeof n, cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "list length read");
  int maxn = 0;
  for (int l = 0; l < n_layers; ++l)
    maxn = maxn > layers[l].d_ff - layers[l].hot ? maxn : layers[l].d_ff - layers[l].hot;
  if (n < 0 || n > maxn) return fail(PI_ERR_DEVICE_CHECK, "list length %d out of range", n);
  *count_out = n;
  const int k = n < cap ? n : cap;
  if (k > 0 && (e = cudaMemcpy(idx_out, at<int32_t>(ws, lay.idx), sizeof(int32_t) * (size_t)k,
                               cudaMemcpyDeviceToHost)) != cudaSuccess)
    return cuda_fail(e, "list read");
  return PI_OK;
}

pi_status pi_get_device_status(void* ws, void* stream, int clear, uint32_t* detail) {
  if (!ws || !aligned(ws, 256)) return fail(PI_ERR_INVALID, "workspace null or misaligned");
  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "stream synchronize");
  uint32_t word = 0;
  e = cudaMemcpy(&word, status_word(ws), sizeof word, cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "status read");
  if (clear) {
    e = cudaMemset(status_word(ws), 0, sizeof word);
    if (e != cudaSuccess) return cuda_fail(e, "status clear");
  }
  if (detail) *detail = word;
  if (word & DEV_TIMEOUT) return fail(PI_ERR_TIMEOUT, "a bounded device wait gave up (status 0x%x)", word);
  if (word) return fail(PI_ERR_DEVICE_CHECK, "device-side range check failed (status 0x%x)", word);
  return PI_OK;
}

}  // extern "C"
