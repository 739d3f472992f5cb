/*
 * pi.h — C ABI of the predictor-gated, neuron-aware sparse FFN decode step
 * (libpi.so, CUDA kernels for sm_100a).
 *
 * What the operations are, from the PowerInfer write-ups:
 *  - Before a layer's FFN runs, a small per-layer predictor decides which
 *    neurons the input activates, and only those neurons are computed
 *    (QbitAI article, r-manual.ru, §"Что такое «разреженная активация»?").
 *  - Neurons split into a small always-active ("hot") group and a large
 *    input-dependent ("cold") group; each group's partial result is summed
 *    into the layer output (same article, §"Гибридный дизайн вывода
 *    CPU/GPU", the example in which an input activates neurons 3, 4 and 5;
 *    aibars.net "SJTU-IPADS/PowerInfer", §"Mecanismo de Neurônios Quentes e
 *    Frios").  Here the hot group is a frequency-sorted prefix [0, hot) of
 *    the neuron order and both groups run on the same GPU.
 *  - Activations ReLU and ReGLU (hada.io summary, §"Hạn chế và FAQ"),
 *    weights optionally INT4 Q4_0 (same page, §"Lượng tử hóa và tương
 *    thích").
 *
 * Conventions shared by every call
 *  - Every data pointer is a DEVICE pointer owned by the caller; the library
 *    never allocates, frees or synchronises (except pi_get_device_status).
 *    Work is enqueued on `stream` (a cudaStream_t passed as void*; NULL = the
 *    legacy default stream) and runs asynchronously.
 *  - Matrices are row-major.  FFN weights are NEURON-MAJOR: row j of
 *    w_gate, w_up and w_down_t is neuron j's d_model weights, so every
 *    active neuron is one contiguous row per matrix.
 *  - Q4_0 weights: a [d_ff][d_model/32][16]-byte array of 4-bit codes and a
 *    [d_ff][d_model/32] array of binary16 scales.  Weight (j, c) is
 *    (q - 8) * s with s the scale of block c/32 of row j and q the nibble for
 *    element k = c % 32: the low nibble of byte k for k < 16, the high nibble
 *    of byte k - 16 otherwise.
 *  - Masks: bit j of a token's mask is bit (j % 32) of 32-bit word j / 32;
 *    a token's mask has ceil(d_ff / 32) words; bits at or beyond d_ff are 0.
 *  - Synchronous argument errors return PI_ERR_INVALID (null or misaligned
 *    pointer, bad size, workspace too small) or PI_ERR_UNSUPPORTED (a dtype /
 *    activation / size combination the library does not implement) before
 *    anything is enqueued.  A failed launch returns PI_ERR_CUDA.  Problems
 *    only the device can see (an index out of range, a bounded wait that ran
 *    out) set sticky bits in the workspace's status word and skip the bad
 *    access; read them with pi_get_device_status.
 *  - pi_last_error() describes the last failure of the calling thread.
 */
#ifndef PI_H
#define PI_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define PI_VERSION 3
#define PI_MAX_BATCH 64        /* tokens per call                           */
#define PI_MAX_D_MODEL 16384   /* d_model upper bound                       */
#define PI_MAX_RANK 8192       /* predictor rank upper bound                */
#define PI_MAX_D_FF (1 << 20)  /* d_ff upper bound                          */

typedef enum pi_status {
  PI_OK = 0,
  PI_ERR_INVALID = 1,      /* bad argument, nothing enqueued                */
  PI_ERR_UNSUPPORTED = 2,  /* valid but not implemented, nothing enqueued   */
  PI_ERR_CUDA = 3,         /* a CUDA call or launch failed                  */
  PI_ERR_TIMEOUT = 4,      /* a bounded device-side wait ran out            */
  PI_ERR_DEVICE_CHECK = 5  /* a device-side range check failed              */
} pi_status;

typedef enum pi_dtype { PI_F32 = 0, PI_F16 = 1, PI_Q4_0 = 2 } pi_dtype;
typedef enum pi_act { PI_RELU = 0, PI_REGLU = 1, PI_RELU2 = 2 } pi_act;

/* How a batch's tokens share the predicted neuron set.
 *  PER_TOKEN: each token's FFN runs over its own predicted set; rows
 *             listed for any token are read once and a token whose own
 *             mask bit is 0 gets h = 0 for that neuron.
 *  UNION:     every token's FFN runs over the union of the batch's
 *             predicted sets (prefill). */
typedef enum pi_mask_mode { PI_MASK_PER_TOKEN = 0, PI_MASK_UNION = 1 } pi_mask_mode;

/* One FFN layer and its predictor.  All pointers are device pointers, except
 * the optional cold-tier pointers at the end (page-locked host memory).
 *  d_model, d_ff, rank : sizes d, F, r.  hot : H, 0 <= H <= F, the
 *                        always-active prefix [0, H) of the neuron order.
 *  act        : PI_RELU  h_j = max(0, w_up[j].xh + bias[j])
 *               PI_REGLU h_j = max(0, w_gate[j].xh + bias[j]) * (w_up[j].xh)
 *               PI_RELU2 h_j = max(0, w_up[j].xh + bias[j])^2  (squared ReLU)
 *               A neuron is active when its first matrix's pre-activation
 *               (w_gate for ReGLU, w_up otherwise) plus bias is > 0; an
 *               inactive neuron's h is 0 and its down row, and (ReGLU) its
 *               w_up row, contribute nothing and need not be read.
 *  w_dtype    : PI_F32, PI_F16 or PI_Q4_0 for w_gate / w_up / w_down_t.
 *  p_dtype    : PI_F32 or PI_F16 for p1 / p2.
 *  w_gate     : [F][d] (ReGLU only; NULL otherwise).   w_up : [F][d].
 *  w_down_t   : [F][d], row j = column j of W_down, so y = sum_j h_j w_down_t[j].
 *  *_scales   : Q4_0 only, [F][d/32] binary16; NULL otherwise.
 *  bias       : [F] fp32 on the first matrix (gate for ReGLU, up for ReLU); NULL = 0.
 *  p1         : [r][d], p2 : [F][r]; predictor logits z = p2 (p1 xh) + p_bias.
 *  p_bias     : [F] fp32; NULL = 0.
 *  w_row_stride     : bytes from row j to row j+1 of w_gate and w_up, and (Q4_0)
 *                     of their scale arrays; 0 = dense rows (codes d/2 bytes,
 *                     scales d/16 bytes apart for Q4_0).
 *  w_down_row_stride: the same for w_down_t and its scales.
 *  w_up_row_stride  : ReGLU only: the same for w_up, when it differs from
 *                     w_row_stride (0 = w_row_stride).
 *  Strides let neuron records share buffers so that what is read together
 *  is one contiguous span.  The single-token kernel reads fastest from:
 *    ReGLU: gate records [codes | scales] one after another (w_row_stride =
 *           record size), and per neuron [up record | down record]
 *           (w_up_row_stride = w_down_row_stride = 2 records, w_down_t =
 *           w_up + one record), so an active neuron's up and down rows are
 *           one read;
 *    ReLU / squared ReLU: up records one after another, down records one
 *           after another (Q4_0: each row's scales right behind its codes).
 * Alignment: every weight pointer 16-byte aligned; d % 8 (F32, F16),
 * d % 32 (Q4_0) == 0; r % 4 (F32 predictor) / r % 8 (F16 predictor) == 0;
 * strides multiples of 16 and at least one row's codes.
 *
 * Hybrid cold tier (optional; the QbitAI article, §"Гибридный дизайн вывода
 * CPU/GPU": hot neurons stay in GPU memory, cold ones in host memory, and
 * the partial results are merged on the GPU).  When w_up_cold is not NULL,
 * rows [hot, d_ff) of w_gate, w_up and w_down_t, and of their Q4_0 scale
 * arrays, are read from the *_cold pointers instead: row j >= hot of w_up
 * is at w_up_cold + (j - hot) * stride, with the same strides as the device
 * rows (so packed records keep their layout), and rows [hot, d_ff) of the
 * device pointers are never read (they may be left unallocated past row
 * hot - 1).  The cold pointers must point into page-locked host memory
 * that the current device can address (cudaHostAlloc / cudaMallocHost, or
 * cudaHostRegister with cudaHostRegisterMapped); anything else returns
 * PI_ERR_INVALID.  All cold pointers a layer needs must be set together
 * (w_gate_cold for ReGLU, the scale arrays for Q4_0), with the alignment of
 * their device counterparts.  The GPU reads the cold rows over the host
 * link (PCIe or C2C) and merges them in the same kernels as the hot rows:
 * the result is the same as with every row in device memory on those
 * kernels.  Such layers take the multi-kernel path (batch 1 included): the
 * CUDA-core kernels, or for Q4_0 layers at 2-64 tokens the tensor-core
 * kernels.  Where those kernels would read a row more than once (several
 * token chunks, or the tensor cores' tiles), each call first copies the
 * listed cold rows into the workspace once (pi_workspace_bytes counts that
 * stage).  Each call looks the cold pointers up (cudaPointerGetAttributes,
 * a few microseconds per layer on the host; also legal inside a stream
 * capture in cudaStreamCaptureModeRelaxed).  The host memory must stay
 * allocated and unchanged until the stream has run the call. */
typedef struct pi_layer {
  int32_t d_model, d_ff, rank, hot;
  int32_t act, w_dtype, p_dtype;
  const void* w_gate;
  const void* w_up;
  const void* w_down_t;
  const void* w_gate_scales;
  const void* w_up_scales;
  const void* w_down_t_scales;
  const float* bias;
  const void* p1;
  const void* p2;
  const float* p_bias;
  int64_t w_row_stride;
  int64_t w_down_row_stride;
  int64_t w_up_row_stride;
  const void* w_gate_cold;
  const void* w_up_cold;
  const void* w_down_t_cold;
  const void* w_gate_cold_scales;
  const void* w_up_cold_scales;
  const void* w_down_t_cold_scales;
} pi_layer;

/* Bytes of workspace the calls below need for these layers at this batch
 * size, on the current CUDA device (the split of the down projection
 * follows the device's SM count; layers with a host-memory cold tier add
 * the stage of their listed cold rows where the kernels use one).  Returns
 * 0 on invalid arguments. */
size_t pi_workspace_bytes(const pi_layer* layers, int n_layers, int batch);

/* Clears the workspace's status word and wait counters; call once after
 * allocating a workspace (256-byte aligned) and before its first use. */
pi_status pi_workspace_init(void* ws, size_t ws_bytes, void* stream);

/* The activation predictor (QbitAI article, §"Что такое «разреженная
 * активация»?": a small per-layer model predicts the neurons the input
 * activates).  For each token b of xh [batch][d] (the FFN input, fp32):
 *   u = p1 xh_b (fp32 accumulation),  z_j = p2[j] . u + p_bias[j],
 *   bit j of mask[b] = 1  if j < hot, or if sigmoid(z_j) > tau, i.e.
 *                         z_j > logit(tau) (logit taken in double, rounded
 *                         to fp32); 0 otherwise.  Rows j < hot of p2 are not read.
 * mask: [batch][ceil(d_ff/32)] uint32.  tau in (0, 1).  batch in [1, 64].
 * Workspace: pi_workspace_bytes(layer, 1, batch). */
pi_status pi_predict(const pi_layer* layer, const float* xh, int batch, float tau,
                     uint32_t* mask, void* ws, size_t ws_bytes, void* stream);

/* pi_predict without a workspace, for callers that cannot allocate device
 * memory: cudaMalloc and cudaFree synchronise the whole device (stalling
 * every stream, which latency-bound serving loops avoid), and a process
 * whose device memory is reserved up front by its own allocator has none
 * left to give to a workspace.  The method itself has no counterpart to
 * this entry point.  The hidden vector u lives in a static buffer of the
 * library, one per device, of PI_PREDICT_NOALLOC_MAX_FLOATS floats (1 MiB).
 *   Kernels: always the CUDA-core predictor pair (u = p1 xh, then logits,
 *          threshold and mask), at every batch.  pi_predict takes the
 *          tensor-core predictor for fp16 predictors at 2-64 tokens, so at
 *          those batches the two calls may set different bits for neurons
 *          whose logit lies within about 1e-4 of logit(tau); elsewhere they
 *          agree.  At other batches and dtypes the kernels, and so the
 *          masks, are the same as pi_predict's.
 *   Limit: batch * rank <= PI_PREDICT_NOALLOC_MAX_FLOATS; larger calls
 *          return PI_ERR_INVALID (use pi_predict with a workspace).
 *   Set-up: the first call on each device, with that device current, looks
 *          up the buffer's device address (cudaGetSymbolAddress) and keeps
 *          it for the life of the process; make that first call before any
 *          stream capture, and do not call this entry point again on a
 *          device after cudaDeviceReset (the kept address would be stale).
 *   Zeroing: nothing; every element of u is written before it is read.
 *   Concurrency: the buffer is shared by all calls on a device, so calls
 *          whose GPU work overlaps (e.g. on two streams with no ordering
 *          between them) race on it and produce wrong masks; issue them on
 *          one stream, or use pi_predict with a workspace per stream.
 * Allocates nothing. */
#define PI_PREDICT_NOALLOC_MAX_FLOATS 262144
pi_status pi_predict_noalloc(const pi_layer* layer, const float* xh, int batch, float tau,
                             uint32_t* mask, void* stream);

/* Mask compaction: neuron ids j in [begin, d_ff) whose bit is set, in
 * ascending order, int32.  mask: [batch][ceil(d_ff/32)].
 *   PI_MASK_UNION    : one list over the OR of the batch's masks;
 *                      idx [d_ff] (first count[0] entries valid), count [1].
 *   PI_MASK_PER_TOKEN: one list per token; token b's list at idx + b*d_ff,
 *                      its length in count[b]; idx [batch][d_ff], count [batch].
 * count stays on the device.  0 <= begin <= d_ff. */
pi_status pi_compact(const uint32_t* mask, int batch, int d_ff, int begin, int mode,
                     int32_t* idx, int32_t* count, void* stream);

/* The FFN over the neuron set S = [0, hot) U idx[0 .. *count) for a batch of
 * FFN inputs xh [batch][d]:
 *   y[b] = sum over j in S, of h_bj * w_down_t[j]   (fp32, [batch][d])
 * with h_bj the activation of `act`.  idx: ascending neuron ids in
 * [hot, d_ff) (e.g. pi_compact with begin = hot and PI_MASK_UNION); count: a
 * device int32.  mode PI_MASK_PER_TOKEN with batch > 1 also needs `mask`
 * ([batch][ceil(d_ff/32)]) and sets h_bj = 0 when token b's bit j is 0 for
 * a cold neuron j; otherwise mask may be NULL.  Rows whose h is 0 for every
 * token of the batch are not read from w_down_t.  The down projection is a
 * split-K sum whose split and order are fixed for a given device, batch
 * and count, so results are bitwise reproducible.  Out-of-range ids or
 * count are skipped and flagged in the status word.
 * Workspace: pi_workspace_bytes(layer, 1, batch). */
pi_status pi_sparse_ffn(const pi_layer* layer, const float* xh, int batch,
                        const uint32_t* mask, const int32_t* idx, const int32_t* count,
                        int mode, float* y, void* ws, size_t ws_bytes, void* stream);

/* A stack of n_layers sparse FFN layers on the residual stream
 * x [batch][d] (fp32, updated in place), each layer l being
 *   xh = x / sqrt(mean(x^2) + 1e-6);  mask = pi_predict(layer l, xh, tau);
 *   S  = [0, hot) U (compaction of the mask over [hot, d_ff));
 *   x  = x + FFN_S(xh)
 * (the pre-norm residual chaining is this library's reading; the pages do
 * not describe how layers chain).  With batch 1 and layers of one shape
 * (d_model <= 12288, rank <= 1024 for an fp16 predictor and <= 512 for an
 * fp32 one; Q4_0 also d_model <= 8192, d_model % 256 == 0 and 16-byte
 * aligned scale arrays) the whole stack runs in one persistent cooperative
 * kernel per 40 layers; otherwise as a sequence of per-step kernels (fp16
 * and Q4_0 layers at 2-64 tokens on the tensor cores).  Q4_0 stacks that
 * meet the single-token conditions run below 5 tokens with
 * PI_MASK_PER_TOKEN and no mask_trace as one persistent pass per token,
 * which gives each token its per-token FFN exactly.  Setting the
 * environment variable PI_DISABLE_FUSED=1 forces the sequence.  All layers
 * must share d_model and d_ff; `layers` is a HOST array of n_layers
 * descriptors.  mode: PI_MASK_PER_TOKEN or
 * PI_MASK_UNION as in pi_sparse_ffn.  mask_trace: NULL, or device
 * [n_layers][batch][ceil(d_ff/32)] receiving every layer's predicted masks
 * (d_ff of the largest layer).  No host synchronisation; capturable in a
 * CUDA graph.  Workspace: pi_workspace_bytes(layers, n_layers, batch). */
pi_status pi_ffn_stack(const pi_layer* layers, int n_layers, float* x, int batch, float tau,
                       int mode, uint32_t* mask_trace, void* ws, size_t ws_bytes,
                       void* stream);

/* Kernel kinds timed by pi_ffn_stack_profile, in launch order per layer. */
enum {
  PI_KIND_RMSNORM = 0,
  PI_KIND_PRED_U = 1,    /* u = p1 xh                                     */
  PI_KIND_PRED_Z = 2,    /* logits, threshold, mask                        */
  PI_KIND_COMPACT = 3,   /* mask -> ascending list                          */
  PI_KIND_FFN_UP = 4,    /* gathered gate/up rows + activation              */
  PI_KIND_FFN_DOWN = 5,  /* gathered split-K down projection                */
  PI_KIND_REDUCE = 6,    /* fixed-order partial sum + residual              */
  PI_KIND_FUSED = 7,     /* persistent single-token stack kernel (all steps) */
  PI_KINDS = 8
};

/* Measurement variant of pi_ffn_stack (same arguments, same launches and
 * results) that records a CUDA event on `stream` before and after every
 * launch.  A short delay kernel (about 2 ms, ends on its own) runs first so
 * the host has enqueued the whole sequence before the device reaches it,
 * and event intervals hold device time only.  Synchronises `stream` at the
 * end.  kind_ms[PI_KINDS] receives each kind's total milliseconds,
 * kind_launches[PI_KINDS] its number of launches (both nullable). */
pi_status pi_ffn_stack_profile(const pi_layer* layers, int n_layers, float* x, int batch,
                               float tau, int mode, uint32_t* mask_trace, void* ws,
                               size_t ws_bytes, void* stream, float* kind_ms,
                               int* kind_launches);

const char* pi_kind_name(int kind);

/* Measurement variant of pi_ffn_stack for the persistent single-token
 * kernel (batch 1; PI_ERR_UNSUPPORTED otherwise): the same launches and
 * results, plus a timeline.  timeline: device [n_layers][pi_device_sms()][16]
 * of unsigned 64-bit values per layer and CTA: slots 0-11 are %globaltimer
 * stamps (ns) taken by the CTA's first consumer thread at the layer's phase
 * boundaries: 0 layer start, 1 input normalised, 2 predictor rows of P1
 * done, 3 grid barrier 1 passed, 4 mask words done, 5 hot items done,
 * 6 grid barrier 2 passed, 7 compaction and cold items done, 8 down rows
 * done, 9 grid barrier 3 passed, 10 column slice reduced, 11 grid barrier 4
 * passed; slots 12-14 are the producer warp's stall times in ns (waiting for
 * a free stage, for the cold list, for activations) and slot 15
 * the producer's end-of-layer stamp.  unit_timeline: NULL, or device
 * [n_layers][512][4] receiving, for the first CTA's first 512 streamed units
 * of each layer, the times the unit's copy was armed, its data seen by the
 * first consumer warp and its stage released, and its byte count.
 * Asynchronous like pi_ffn_stack. */
pi_status pi_ffn_stack_timeline(const pi_layer* layers, int n_layers, float* x, float tau,
                                void* ws, size_t ws_bytes, void* stream,
                                unsigned long long* timeline, unsigned long long* unit_timeline);

/* Number of SMs of the current device (the persistent kernel's grid). */
int pi_device_sms(void);

/* Number of kernels this library has launched in this process so far, over
 * every entry point (a host-side count taken at each launch; a launch made
 * while a stream is being captured into a CUDA graph counts once, at capture,
 * so the difference across one captured call is the graph's kernel count).
 * Never fails. */
unsigned long long pi_kernel_launches(void);

/* Synchronises `stream` and reads the workspace's three row counters, which
 * every FFN launch advances on the device: out[0] = neuron rows whose first
 * matrix (w_gate for ReGLU, w_up otherwise) was read, out[1] = rows of
 * w_down_t read, out[2] = rows of w_up read for ReGLU (0 otherwise).  The
 * single-token kernel reads w_up (ReGLU) and w_down_t rows only for neurons
 * whose first pre-activation is positive; the batch kernels read w_up for
 * every listed neuron and w_down_t rows whose h is nonzero for some token.
 * Each pass over a row by a token chunk of at most 8 tokens counts once.
 * Together with the predictor's fixed size they give the bytes the path
 * actually read.  out: uint64_t[3].  `clear` != 0 resets all three. */
pi_status pi_read_counters(void* ws, void* stream, int clear, uint64_t* out);

/* The same three counts restricted to rows read from a hybrid cold tier
 * (host memory, see pi_layer): out[0] first-matrix rows, out[1] w_down_t
 * rows, out[2] ReGLU w_up rows.  Multiplied by the row bytes they give the
 * bytes that crossed the host link.  out: uint64_t[3].  `clear` != 0 resets
 * all three. */
pi_status pi_read_cold_counters(void* ws, void* stream, int clear, uint64_t* out);

/* Synchronises `stream` and copies to the host the ascending list of cold
 * neurons (ids in [hot, d_ff)) that the LAST layer of the last
 * pi_ffn_stack / pi_ffn_stack_profile / pi_ffn_stack_timeline call on this
 * workspace ran over (batch > 1: the list of the batch's union mask):
 * *count_out receives the list's length and idx_out (host, int32) its first
 * min(length, cap) ids.  layers, n_layers and batch are that call's (they
 * fix the workspace layout).  Inspection of the compaction step
 * (QbitAI article, §"Что такое «разреженная активация»?": only the predicted
 * neurons are computed; the list is that set), used by tests. */
pi_status pi_read_list(const pi_layer* layers, int n_layers, int batch, void* ws,
                       size_t ws_bytes, void* stream, int32_t* idx_out, int cap,
                       int32_t* count_out);

/* Synchronises `stream`, reads the workspace's status word and returns
 * PI_OK, PI_ERR_DEVICE_CHECK or PI_ERR_TIMEOUT (timeout wins).  `detail`
 * (nullable) receives the raw word; `clear` != 0 resets it. */
pi_status pi_get_device_status(void* ws, void* stream, int clear, uint32_t* detail);

/* Failure-detection self-test: runs, in one thread of a tiny kernel, the
 * bounded waits the fused kernel uses, on a wait nothing can satisfy
 * (kind 0: an mbarrier phase with no arrival; kind 1: the workspace's grid
 * barrier counter against a target no CTA reaches), limited to timeout_us
 * (1 .. 1e7) instead of the kernel's 1 s.  The wait runs out, records the
 * timeout in the workspace status word (pi_get_device_status then returns
 * PI_ERR_TIMEOUT) and the kernel returns normally: the context stays usable.
 * Resets the workspace's grid-barrier counters.  Not part of the method. */
pi_status pi_wait_selftest(void* ws, size_t ws_bytes, int kind, unsigned timeout_us, void* stream);

const char* pi_status_string(int status);
const char* pi_last_error(void);
int pi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* PI_H */
