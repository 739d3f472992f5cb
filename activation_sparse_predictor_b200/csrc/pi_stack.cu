// Persistent single-token decode kernel for the whole FFN stack (sm_100a).
//
// One cooperative launch runs a chunk of layers with one CTA per SM.  Each
// CTA has three producer warps (one thread each) that stream every weight
// row the CTA will use through a ring of shared-memory stages with 1-D bulk
// copies (cp.async.bulk, completion counted on an mbarrier per stage; each
// copy costs its thread a few hundred ns to issue, so the copies of
// consecutive stages are issued by different threads), a list warp, and
// sixteen consumer warps in groups: a unit (stage) goes to one group, whose
// threads each take a slice of its columns, so a stage is held only briefly
// and the ring keeps many rows in flight.  Per layer:
//
//   x^  : every CTA normalises the full residual vector (rmsnorm) itself
//   A   : predictor rows of P1 (a static share per CTA)   -> u      | grid barrier 1
//   B   : predictor rows of P2 for the CTA's mask words (words s, s + SMs, ...
//         of the cold range) -> mask words; the CTA lists the predicted cold
//         neurons of its own words at once (no grid barrier)
//   C   : first matrix (W_gate for ReGLU, W_up otherwise) of the CTA's hot
//         neurons (j = s, s + SMs, ... in groups of adjacent neurons), then
//         of its cold neurons; each unit is finalised as soon as it is
//         consumed: the neuron's first pre-activation + bias and its flag
//   D   : ReLU / squared ReLU: down rows of the neurons whose h != 0.
//         ReGLU (second-level sparsity): [W_up | W_down^T] of the neurons
//         whose gate fired, read only for those; two up groups of consumer
//         warps form the W_up dots and h = gate * up of alternate units while
//         a down group accumulates h times the down rows of the unit before
//                                                          -> partial y | grid barrier 3
//   E   : fixed-order reduction of the CTA's column slice, residual add | grid barrier 4
//
// The producers run ahead across phases for every row whose address does
// not depend on this layer's data (P1, P2, hot rows, the next layer's rows);
// cold rows wait for the CTA's list and the rows of phase D for their
// neuron's flag.  (L2 prefetching of the static rows ahead of the ring, by
// bulk or per-line prefetches, measured slower at every distance tried,
// 256 KB to 1 MB per CTA, and is not used.)  The kernel is bound by latency
// more than by issue: its instruction footprint counts (instruction-fetch
// stalls), so the timeline instrumentation is a separate instantiation and
// the per-unit loops are unrolled only as far as a unit's records go.
// Every wait (mbarrier, grid barrier, flag) is bounded by %globaltimer; a
// wait that runs out sets DEV_TIMEOUT and an abort flag, after which every
// thread runs the rest of its loops without waiting or computing and the
// producer waits (bounded) for its own copies in flight before exiting.
//
// Q4_0 gate/up dot products are exact integer sums: the normalised input is
// rounded once per layer to int16 on a per-vector scale, each block's
// sum_k (q_k - 8) x_k is formed with dp2a in int32 (no rounding), then
// scaled in fp32.  Everything else accumulates in fp32.
#include <cstdlib>
#include <cstring>

#include "pi_kernels.cuh"
#include "pi_stack.cuh"

namespace pi {
namespace {

constexpr int NCW = 16;             // consumer warps
constexpr int NCT = NCW * 32;       // consumer threads
constexpr int NPMAX = 3;            // producer warps (after the consumers)
constexpr int NTHR = NCT + 32 * (NPMAX + 1);  // + the compaction warp
constexpr int NSMAX = 24;           // ring stages at most
constexpr int MAXL = 40;            // layers per launch (the parameter block stays under 4 KB)
constexpr int MAXA = 16;            // P1 rows per CTA at most
constexpr unsigned long long kTimeoutNs = 1000000000ull;  // 1 s per wait
constexpr int UTR = 512;            // units per layer recorded by the unit trace
constexpr int DRMAX = 16;           // D records per unit at most
constexpr int HQ = 32;              // ReGLU down-phase unit flags (a ring, >= ring depth)
constexpr int kMaxRec = 4;          // first records per C unit at most
constexpr int DR2MAX = 4;           // D records per unit at most, ReGLU (W_up dot partials)
constexpr int kQ4Blocks = 1;        // Q4_0 blocks per thread in phase D

struct LayerPtrs {
  const char* first;            // W_gate (ReGLU) or W_up (ReLU): codes / rows
  const char* second;           // W_up (ReGLU only)
  const char* down;             // W_down^T
  const char* first_scales;     // Q4_0 scales
  const char* second_scales;
  const char* down_scales;
  const float* bias;
  const char* p1;
  const char* p2;
  const float* pbias;
};
static_assert(sizeof(LayerPtrs) == 80, "compact layer pointers");

// Shape and shared-memory plan, identical for every CTA.
//
// Phase C streams "first" records (the matrix whose ReLU decides activity:
// W_gate for ReGLU, W_up for ReLU): [codes | scales (Q4_0)], padded to 16
// bytes.  Phase D streams, for the neurons whose first pre-activation is
// positive, "D records": ReGLU [up codes | up scales | pad | down codes |
// down scales | pad], ReLU [down codes | down scales | pad].
struct Plan {
  int d, F, r, H;
  int ns, G, maxc, maxi, nsms;
  int np;                           // producer warps
  int gw, gd;                       // consumer warp groups: phases A-C / phase D
  int hp;                           // first records per hot unit (adjacent neurons)
  int cp;                           // first records per cold unit
  int dr;                           // D records per unit (the last one of a layer: fewer)
  int sq;                           // squared ReLU: h = max(0, g)^2
  int first_packed, d2_packed;      // records contiguous in memory at their own size
  int first_contig, second_contig, down_contig;  // a row's Q4_0 scales right behind its codes
  long long first_stride, first_sstride;    // bytes between neurons: codes / Q4_0 scales
  long long second_stride, second_sstride;  // ReGLU W_up
  long long down_stride, down_sstride;
  uint32_t sb;                      // stage bytes
  uint32_t rowb, scb;               // weight row bytes (codes), Q4_0 scale row bytes
  uint32_t p1_bytes, p2_row;        // predictor row bytes
  uint32_t first_b;                 // a first record in a stage
  uint32_t d2_bytes, o_d2_down;     // a D record in a stage; offset of its down row
  uint32_t o_misc, o_xf, o_xi, o_bsum, o_u, o_bw, o_scan, o_items, o_hval, o_flag,
      o_dlist, o_pbs, o_hbs, o_redA, o_redC, o_redD, o_hflag, o_redE, o_ring, total;
};

struct StackParams {
  Plan pl;
  int n_layers;
  float theta;
  float* x;              // [d] residual stream, in/out
  uint32_t* mask;        // this chunk's first layer's mask words
  long long mask_stride; // words between consecutive layers' masks (0: two alternating slots)
  long long mask_words;  // words per mask
  float* u;              // [r]
  float* part;           // [nsms][d]
  int32_t* count;        // cold-list length of the last layer
  int32_t* idx;          // [d_ff] the layer's ascending cold list (last layer's stays)
  uint32_t* cta_counts;  // [SMs] per-CTA cold-list lengths of the current layer (tagged)
  WsHeader* hdr;
  unsigned long long* trace;  // nullable [n_layers][nsms][16] timeline
  unsigned long long* utrace; // nullable [n_layers][UTR][4]: CTA 0's units
  LayerPtrs L[MAXL];
};
static_assert(sizeof(StackParams) < 4000, "kernel parameter block under 4 KB");

// -------------------------------------------------------------- primitives

__device__ __forceinline__ uint32_t sa(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ uint64_t gtime() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(uint64_t* b, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(sa(b)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive_tx(uint64_t* b, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(sa(b)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* b, uint32_t count) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0], %1;" ::"r"(sa(b)), "r"(count)
               : "memory");
}

__device__ __forceinline__ bool mbar_try(uint64_t* b, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(sa(b)), "r"(parity)
      : "memory");
  return ok != 0;
}

// try_wait that lets the hardware suspend the warp until the phase completes
// or `hint_ns` passes, so waiting warps do not take issue slots from working ones.
__device__ __forceinline__ bool mbar_try_sleep(uint64_t* b, uint32_t parity, uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(sa(b)), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}

// 1-D bulk copy global -> shared, completion counted on `bar` (bytes % 16 == 0,
// both addresses 16-byte aligned).
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes,
                                         uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(sa(dst)),
      "l"(src), "r"(bytes), "r"(sa(bar))
      : "memory");
}

__device__ __forceinline__ uint4 lds128(const void* p) { return *reinterpret_cast<const uint4*>(p); }

__device__ __forceinline__ void csync() { asm volatile("bar.sync 1, 512;" ::: "memory"); }

__device__ __forceinline__ uint32_t ld_acquire(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Grid-barrier arrival (after a CTA-wide bar.sync): release at gpu scope,
// cumulative over the writes the CTA's threads made before the bar.sync.
__device__ __forceinline__ void grid_arrive(uint32_t* ctr) {
  asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(ctr) : "memory");
}

__device__ __forceinline__ float4 f4add(float4 a, float4 b) {
  return make_float4(a.x + b.x, a.y + b.y, a.z + b.z, a.w + b.w);
}

// ------------------------------------------------------ vector layouts
// Vectors dotted with fp16 rows (x^ and u when the predictor is fp16) are
// staged "split-half": element i at ((i & 7) >> 2) * n/2 + (i >> 3) * 4 + (i & 3),
// so the two float4 halves of 16-byte chunk c are float4 number c and
// n/8 + c, and consecutive threads read consecutive 16-byte words (no bank
// conflicts).  fp32 rows use the natural order.  The int16 copy of x^ for
// Q4_0 rows is sub-chunk-major: element 32k + 8q + o at (q * nb + k) * 8 + o
// (nb = d / 32 blocks).
template <int DT>
__device__ __forceinline__ int vpos(int i, int n) {
  if constexpr (DT == PI_F16) return ((i & 7) >> 2) * (n >> 1) + ((i >> 3) << 2) + (i & 3);
  return i;
}


// The staged-vector elements that chunk c of a DT row multiplies.
struct VFrag {
  float4 lo, hi;  // hi only for fp16 rows
};

template <int DT>
__device__ __forceinline__ VFrag vfrag(const float* v, int c, int n) {
  const float4* v4 = reinterpret_cast<const float4*>(v);
  VFrag f;
  f.lo = v4[c];
  if constexpr (DT == PI_F16) f.hi = v4[(n >> 3) + c];
  else f.hi = f.lo;
  return f;
}

// Dot product of a 16-byte chunk of a DT row with its vector fragment.
template <int DT>
__device__ __forceinline__ float frag_dot(const uint4 w, const VFrag& x) {
  if constexpr (DT == PI_F32) {
    float a = __uint_as_float(w.x) * x.lo.x;
    a = fmaf(__uint_as_float(w.y), x.lo.y, a);
    a = fmaf(__uint_as_float(w.z), x.lo.z, a);
    return fmaf(__uint_as_float(w.w), x.lo.w, a);
  } else {
    float f[8];
    f16x8_to_f32(w, f);
    const float4 lo = x.lo, hi = x.hi;
    float a = f[0] * lo.x, b = f[4] * hi.x;
    a = fmaf(f[1], lo.y, a);
    b = fmaf(f[5], hi.y, b);
    a = fmaf(f[2], lo.z, a);
    b = fmaf(f[6], hi.z, b);
    a = fmaf(f[3], lo.w, a);
    b = fmaf(f[7], hi.w, b);
    return a + b;
  }
}

// Dot product of 16-byte chunk c of a DT row with the staged vector v (length n).
template <int DT>
__device__ __forceinline__ float chunk_dot(const uint4 w, const float* v, int c, int n) {
  return frag_dot<DT>(w, vfrag<DT>(v, c, n));
}

// Two nibbles of a Q4_0 word as floats 1 + q/16: x holds 0x80 | q << 3 in
// each byte (q = the nibble), and the byte permute places byte b (and b+1)
// as bits 16..23 under the exponent byte 0x3F.
__device__ __forceinline__ float2 nib_pair(uint32_t x, int b) {
  return make_float2(__uint_as_float(__byte_perm(x, 0x3F00u, 0x5044u | ((uint32_t)b << 8))),
                     __uint_as_float(__byte_perm(x, 0x3F00u, 0x5044u | ((uint32_t)(b + 1) << 8))));
}

// sum_k (q_k - 8) * x_k over one Q4_0 block in exact int32 arithmetic:
// xw[m] holds the int16 pair (x[2m], x[2m+1]); `base` = -8 * sum_k x_k.
__device__ __forceinline__ int q4_block_dot(const uint4 v, const int (&xw)[16], int base) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  int lo_acc = base, hi_acc = 0;
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    const int lo = (int)(w[m] & 0x0F0F0F0Fu);         // elements 4m .. 4m+3
    const int hi = (int)((w[m] >> 4) & 0x0F0F0F0Fu);  // elements 4m+16 .. 4m+19
    lo_acc = __dp2a_lo(xw[2 * m], lo, lo_acc);
    lo_acc = __dp2a_hi(xw[2 * m + 1], lo, lo_acc);
    hi_acc = __dp2a_lo(xw[8 + 2 * m], hi, hi_acc);
    hi_acc = __dp2a_hi(xw[9 + 2 * m], hi, hi_acc);
  }
  return lo_acc + hi_acc;
}

// -------------------------------------------------------- shared carving

struct Smem {
  uint64_t* full;
  uint64_t* empty;
  uint64_t* listbar;          // the CTA's cold list of the layer is ready
  uint64_t* listdone;         // the list warp is done with it
  volatile int* abort;        // CTA-wide: stop waiting and computing
  volatile int* nc;           // this CTA's cold items (current layer)
  float* xscale;              // int16 scale of xh (Q4_0)
  float* xf;
  int16_t* xi;
  int* bsum;
  float* us;
  uint32_t* bw;
  int* scan;
  int* items;                 // neuron of each item: hot items, then this layer's cold list
  float* hval;
  volatile int* flag;
  volatile int* hflag;        // [HQ] ReGLU down phase: unit q's h is ready (tag | q + 1)
  int* dlist;
  float* pbs;                 // predictor biases of the CTA's mask words
  float* hbs;                 // activation biases of the CTA's items
  float* redA;
  float* redC;                // [GW][2][8][WPG] first-record dot partials
  float* redD;                // [GD][2][DR2MAX][WPD] W_up dot partials (ReGLU)
  float4* redE;
  char* ring;
};

__device__ __forceinline__ Smem carve(unsigned char* base, const Plan& pl) {
  Smem S;
  S.full = reinterpret_cast<uint64_t*>(base);
  S.empty = S.full + NSMAX;
  S.listbar = S.empty + NSMAX;
  S.listdone = S.listbar + 1;
  int* misc = reinterpret_cast<int*>(base + pl.o_misc);
  S.abort = misc;
  S.nc = misc + 1;
  S.xscale = reinterpret_cast<float*>(misc + 2);
  S.xf = reinterpret_cast<float*>(base + pl.o_xf);
  S.xi = reinterpret_cast<int16_t*>(base + pl.o_xi);
  S.bsum = reinterpret_cast<int*>(base + pl.o_bsum);
  S.us = reinterpret_cast<float*>(base + pl.o_u);
  S.bw = reinterpret_cast<uint32_t*>(base + pl.o_bw);
  S.scan = reinterpret_cast<int*>(base + pl.o_scan);
  S.items = reinterpret_cast<int*>(base + pl.o_items);
  S.hval = reinterpret_cast<float*>(base + pl.o_hval);
  S.flag = reinterpret_cast<volatile int*>(base + pl.o_flag);
  S.hflag = reinterpret_cast<volatile int*>(base + pl.o_hflag);
  S.dlist = reinterpret_cast<int*>(base + pl.o_dlist);
  S.pbs = reinterpret_cast<float*>(base + pl.o_pbs);
  S.hbs = reinterpret_cast<float*>(base + pl.o_hbs);
  S.redA = reinterpret_cast<float*>(base + pl.o_redA);
  S.redC = reinterpret_cast<float*>(base + pl.o_redC);
  S.redD = reinterpret_cast<float*>(base + pl.o_redD);
  S.redE = reinterpret_cast<float4*>(base + pl.o_redE);
  S.ring = reinterpret_cast<char*>(base + pl.o_ring);
  return S;
}

// Marks this CTA (and the grid) as aborted after a wait ran out.
__device__ void raise_abort(const Smem& S, WsHeader* hdr) {
  *S.abort = 1;
  atomicOr(&hdr->status, DEV_TIMEOUT);
  atomicExch(&hdr->counters[1], 1u);
}

// Bounded mbarrier wait; false on abort or timeout (timeout raises abort).
// The first try usually succeeds; the warp sleeps in the hardware wait
// between later checks.
__device__ __forceinline__ bool wait_mbar(uint64_t* bar, uint32_t parity, const Smem& S,
                                          WsHeader* hdr,
                                          unsigned long long limit_ns = kTimeoutNs) {
  if (mbar_try(bar, parity)) return true;
  if (*S.abort) return false;
  const uint64_t t0 = gtime();
  while (true) {
    if (mbar_try_sleep(bar, parity, 50000u)) return true;
    if (*S.abort) return false;
    if (gtime() - t0 > limit_ns) {
      raise_abort(S, hdr);
      return false;
    }
  }
}

// Bounded grid-barrier wait by one thread: counter >= target.
__device__ bool grid_wait(WsHeader* hdr, uint32_t target, const Smem& S,
                          unsigned long long limit_ns = kTimeoutNs) {
  if (*S.abort) return false;
  if (ld_acquire(&hdr->counters[0]) >= target) return true;
  const uint64_t t0 = gtime();
  while (true) {
    __nanosleep(64);
    if (ld_acquire(&hdr->counters[0]) >= target) return true;
    if (ld_acquire(&hdr->counters[1]) != 0u) {
      *S.abort = 1;
      return false;
    }
    if (gtime() - t0 > limit_ns) {
      raise_abort(S, hdr);
      return false;
    }
  }
}

// The mask words of layer l: its slot of the caller's trace, or one of two
// alternating workspace slots.
__device__ __forceinline__ uint32_t* layer_mask(const StackParams& P, int l) {
  return P.mask + (P.mask_stride ? (size_t)l * P.mask_stride : (size_t)(l & 1) * P.mask_words);
}

// Timeline stamp, when a trace buffer is given.
template <bool TR>
__device__ __forceinline__ void tstamp(const StackParams& P, int l, int slot,
                                       unsigned long long v) {
  if constexpr (TR) {
    if (TR && P.trace) P.trace[((size_t)l * gridDim.x + blockIdx.x) * 16 + slot] = v;
  }
}

// Unit trace of CTA 0 (slot 0 armed, 1 data seen by consumer warp 0,
// 2 released by consumer warp 0, 3 bytes).
template <bool TR>
__device__ __forceinline__ void utstamp(const StackParams& P, int l, uint32_t u, int slot,
                                        unsigned long long v) {
  if constexpr (TR) {
    if (P.utrace && blockIdx.x == 0 && u < (uint32_t)UTR)
      P.utrace[((size_t)l * UTR + u) * 4 + slot] = v;
  }
}

// ------------------------------------------------------------ per-CTA shares

struct Ranges {
  int kA0, kA1;   // P1 rows
  int nw;         // mask words evaluated here: Wlo + s + k * SMs, k < nw
  int Wlo, W;     // first word holding a cold neuron, words per mask
  int ngh;        // hot groups g = s, s + SMs, ... of hp adjacent neurons
  int nh;         // hot neurons in them
};

// The k-th of CTA s's items dealt round by round over S CTAs, every other
// round in reverse ("snake"): where the items' expected work falls along
// the order (the frequency-sorted neurons), every CTA gets the same share.
__device__ __forceinline__ int snake(int k, int s, int S) {
  return k * S + ((k & 1) ? S - 1 - s : s);
}

// The CTA that owns item i of a snake deal over S CTAs.
__device__ __forceinline__ int snake_owner(int i, int S) {
  const int k = i / S, p = i - k * S;
  return (k & 1) ? S - 1 - p : p;
}

// Items of a snake deal of n items that CTA s owns.
__device__ __forceinline__ int snake_count(int n, int s, int S) {
  const int full = n / S, rem = n - full * S;
  const int pos = (full & 1) ? S - 1 - s : s;
  return full + (rem > 0 && pos < rem ? 1 : 0);
}

__device__ __forceinline__ Ranges ranges(const Plan& pl) {
  Ranges R;
  const int S = gridDim.x, s = blockIdx.x;
  R.kA0 = (int)((long long)s * pl.r / S);
  R.kA1 = (int)((long long)(s + 1) * pl.r / S);
  R.W = (pl.F + 31) / 32;
  R.Wlo = pl.H / 32;
  const int Wc = R.W - R.Wlo;
  // the cold mask words Wlo + snake(k): every CTA's words sample the whole
  // cold range (the predicted density falls along the order)
  R.nw = snake_count(Wc, s, S);
  // the hot groups snake(gi) of hp adjacent neurons (the last one shorter)
  const int G = (pl.H + pl.hp - 1) / pl.hp;
  R.ngh = snake_count(G, s, S);
  R.nh = R.ngh * pl.hp;
  if (R.ngh > 0 && snake(R.ngh - 1, s, S) == G - 1) R.nh -= G * pl.hp - pl.H;
  return R;
}

// First neuron of this CTA's hot group gi.
__device__ __forceinline__ int hot_group_first(int gi, const Plan& pl) {
  return snake(gi, (int)blockIdx.x, (int)gridDim.x) * pl.hp;
}

// This CTA's k-th cold mask word.
__device__ __forceinline__ int cold_word(int k, const Ranges& R) {
  return R.Wlo + snake(k, (int)blockIdx.x, (int)gridDim.x);
}

// Position in the unit sequence: unit number, its stage (uc % ns) and the
// stage's use count (uc / ns), advanced without divisions.
struct Cursor {
  uint32_t uc = 0;
  int st = 0;
  uint32_t gen = 0;
  __device__ __forceinline__ void next(int ns) {
    ++uc;
    if (++st == ns) {
      st = 0;
      ++gen;
    }
  }
};

// Down-row units: the rows of consecutive nonzero items in item order, pl.dr
// per unit (the last unit of a layer holds the rest).  The producers and the
// consumers apply this rule to the same sequence.

// ---------------------------------------------------------------- producer

template <int WT, int ACT, int PT, bool TR>
__device__ void producer(const StackParams& P, const Smem& S, const int p) {
  const Plan& pl = P.pl;
  WsHeader* hdr = P.hdr;
  const Ranges R = ranges(pl);
  Cursor cu;  // unit sequence, identical on every producer and consumer
  uint32_t last[NSMAX];  // use count of each stage's last copy issued here
#pragma unroll
  for (int i = 0; i < NSMAX; ++i) last[i] = 0xFFFFFFFFu;
  bool ok = true;
  unsigned long long w_empty = 0, w_list = 0, w_flag = 0;  // stall time (ns)
  int cur_l = 0;
  uint32_t l_uc0 = 0;  // first unit of the current layer

  // Stage st belongs to producer st % NPMAX.
  auto mine = [&]() { return cu.st % NPMAX == p; };
  // Claims the current unit's stage (one of ours) and arms its full barrier for `bytes`.
  auto claim = [&](uint32_t bytes) -> char* {
    const int st = cu.st;
    const uint32_t k = cu.gen;
    if (k > 0 && !mbar_try(&S.empty[st], (k - 1) & 1u)) {
      const unsigned long long t0 = (TR && P.trace) ? gtime() : 0ull;
      if (!wait_mbar(&S.empty[st], (k - 1) & 1u, S, hdr)) {
        ok = false;
        return nullptr;
      }
      if (TR && P.trace) w_empty += gtime() - t0;
    }
    mbar_arrive_tx(&S.full[st], bytes);
    last[st] = k;
    if (TR && P.utrace) {
      utstamp<TR>(P, cur_l, cu.uc - l_uc0, 0, gtime());
      utstamp<TR>(P, cur_l, cu.uc - l_uc0, 3, bytes);
    }
    return S.ring + (size_t)st * pl.sb;
  };
  auto bar_of = [&]() { return &S.full[cu.st]; };

  // One row part (codes, then Q4_0 scales right behind them) of neuron j.
  auto part = [&](char* o, const char* codes, const char* scales, size_t j, long long cs,
                  long long ss, bool contig, uint64_t* b) {
    if (contig) {
      bulk_g2s(o, codes + j * cs, pl.rowb + pl.scb, b);
    } else {
      bulk_g2s(o, codes + j * cs, pl.rowb, b);
      if constexpr (WT == PI_Q4_0) bulk_g2s(o + pl.rowb, scales + j * ss, pl.scb, b);
    }
  };
  // First records of n neurons into one stage, record r at r * first_b:
  // the adjacent neurons j0 .. j0+n-1 (one copy when packed) or jl[0 .. n).
  auto firsts = [&](const LayerPtrs& L, const int* jl, int j0, int n) {
    if (mine()) {
      char* dst = claim(pl.first_b * (uint32_t)n);
      if (dst) {
        uint64_t* b = bar_of();
        if (!jl && pl.first_packed) {
          bulk_g2s(dst, L.first + (size_t)j0 * pl.first_stride, pl.first_b * (uint32_t)n, b);
        } else {
          for (int r = 0; r < n; ++r)
            part(dst + (size_t)r * pl.first_b, L.first, L.first_scales,
                 (size_t)(jl ? jl[r] : j0 + r), pl.first_stride, pl.first_sstride,
                 pl.first_contig, b);
        }
      }
    }
    cu.next(pl.ns);
  };
  // D records of the neurons uj[0 .. n) into one stage, record k at
  // k * d2_bytes (ReGLU: W_up part, then the down part at o_d2_down);
  // adjacent packed records share one copy.
  auto d2s = [&](const LayerPtrs& L, const int* uj, int n) {
    if (mine()) {
      char* dst = claim(pl.d2_bytes * (uint32_t)n);
      if (dst) {
        uint64_t* b = bar_of();
        for (int k = 0; k < n;) {
          int m = 1;
          if (pl.d2_packed)
            while (k + m < n && uj[k + m] == uj[k] + m) ++m;
          char* o = dst + (size_t)k * pl.d2_bytes;
          const size_t j = (size_t)uj[k];
          if (pl.d2_packed) {
            const char* src = ACT == PI_REGLU ? L.second + j * pl.second_stride
                                              : L.down + j * pl.down_stride;
            bulk_g2s(o, src, pl.d2_bytes * (uint32_t)m, b);
          } else {
            if constexpr (ACT == PI_REGLU)
              part(o, L.second, L.second_scales, j, pl.second_stride, pl.second_sstride,
                   pl.second_contig, b);
            part(o + pl.o_d2_down, L.down, L.down_scales, j, pl.down_stride, pl.down_sstride,
                 pl.down_contig, b);
          }
          k += m;
        }
      }
    }
    cu.next(pl.ns);
  };

  for (int l = 0; l < P.n_layers && ok; ++l) {
    const LayerPtrs& L = P.L[l];
    cur_l = l;
    l_uc0 = cu.uc;
    // A: predictor rows of P1
    for (int k = R.kA0; k < R.kA1 && ok; ++k, cu.next(pl.ns)) {
      if (mine()) {
        char* dst = claim(pl.p1_bytes);
        if (!dst) break;
        bulk_g2s(dst, L.p1 + (size_t)k * pl.p1_bytes, pl.p1_bytes, bar_of());
      }
    }
    // B: predictor rows of P2, G per unit
    for (int k = 0; k < R.nw && ok; ++k) {
      const int w = cold_word(k, R);
      for (int ja = 32 * w; ja < 32 * w + 32 && ja < pl.F && ok; ja += pl.G, cu.next(pl.ns)) {
        const int jb = min(ja + pl.G, pl.F);
        const uint32_t bytes = (uint32_t)(jb - ja) * pl.p2_row;
        if (mine()) {
          char* dst = claim(bytes);
          if (!dst) break;
          bulk_g2s(dst, L.p2 + (size_t)ja * pl.p2_row, bytes, bar_of());
        }
      }
    }
    // C: first records of the hot groups, then (once the consumers have
    // listed the cold neurons of the CTA's own mask words) of the cold
    // neurons, pl.cp per unit
    for (int gi = 0; gi < R.ngh && ok; ++gi) {
      const int j0 = hot_group_first(gi, pl);
      firsts(L, nullptr, j0, min(pl.hp, pl.H - j0));
    }
    {
      const unsigned long long t0 = (TR && P.trace) ? gtime() : 0ull;
      if (!ok || !wait_mbar(S.listbar, (uint32_t)l & 1u, S, hdr)) break;
      if (TR && P.trace) w_list += gtime() - t0;
    }
    const int nc = *S.nc;
    for (int i = 0; i < nc && ok; i += pl.cp) firsts(L, S.items + R.nh + i, 0, min(pl.cp, nc - i));
    // D: D records of items whose first pre-activation is positive, in item
    // order, pl.dr per unit
    const int tag = (l + 1) << 2;
    int uj[DRMAX], un = 0;  // the open unit's neurons
    for (int i = 0; i < R.nh + nc && ok; ++i) {
      int f = S.flag[i];
      if ((f & ~3) != tag) {
        const uint64_t t0 = gtime();
        while (((f = S.flag[i]) & ~3) != tag) {
          if (*S.abort) { ok = false; break; }
          if (gtime() - t0 > kTimeoutNs) { raise_abort(S, hdr); ok = false; break; }
          __nanosleep(128);
        }
        if (TR && P.trace) w_flag += gtime() - t0;
        if (!ok) break;
      }
      if ((f & 3) != 2) continue;
      uj[un++] = S.items[i];
      if (un == pl.dr) {
        d2s(L, uj, un);
        un = 0;
      }
    }
    if (ok && un > 0) d2s(L, uj, un);
    if (TR && P.trace && p == 0) {
      tstamp<TR>(P, l, 12, w_empty);
      tstamp<TR>(P, l, 13, w_list);
      tstamp<TR>(P, l, 14, w_flag);
      tstamp<TR>(P, l, 15, gtime());
      w_empty = w_list = w_flag = 0;
    }
  }
  // Drain: wait (bounded) until every copy this thread issued has landed.
  for (int st = 0; st < pl.ns; ++st) {
    if (last[st] == 0xFFFFFFFFu) continue;
    const uint32_t par = last[st] & 1u;
    const uint64_t t0 = gtime();
    while (!mbar_try(&S.full[st], par)) {
      if (gtime() - t0 > kTimeoutNs) {
        atomicOr(&hdr->status, DEV_TIMEOUT);
        break;
      }
    }
  }
}

// --------------------------------------------------------------- list warp

// One warp, off the critical path: once the CTA's mask words of a layer are
// out (right after its phase B), it tags its slot of the per-CTA array,
// waits (bounded) until every CTA has, then walks the layer's cold mask
// words in order with a running count and writes the neurons of the CTA's
// own words at their positions of the global ascending list (CTA 0 also
// writes its length).  The computation never reads this list; it is there
// for inspection (pi_read_list).  A wait that gives up leaves the list
// incomplete and records the timeout.
template <int WT, int ACT, int PT, bool TR>
__device__ void list_writer(const StackParams& P, const Smem& S) {
  const Plan& pl = P.pl;
  WsHeader* hdr = P.hdr;
  const Ranges R = ranges(pl);
  const int lane = threadIdx.x & 31, nS = gridDim.x, s = blockIdx.x;
  for (int l = 0; l < P.n_layers; ++l) {
    int ok = 1;
    if (lane == 0) ok = wait_mbar(S.listbar, (uint32_t)l & 1u, S, hdr) ? 1 : 0;
    if (!__shfl_sync(0xffffffffu, ok, 0)) return;
    const uint32_t tag = (uint32_t)(l + 1);  // the array is zeroed before each launch
    if (lane == 0)
      asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(P.cta_counts + s), "r"(tag) : "memory");
    const uint64_t t0 = gtime();
    for (int c = lane; c < nS && ok; c += 32) {
      while (ld_acquire(P.cta_counts + c) != tag) {
        if (*S.abort || gtime() - t0 > kTimeoutNs) { ok = 0; break; }
        __nanosleep(256);
      }
    }
    if (!__all_sync(0xffffffffu, ok)) {
      if (lane == 0) atomicOr(&hdr->status, DEV_TIMEOUT);
      return;
    }
    const uint32_t* mask = layer_mask(P, l);
    int base = 0;
    for (int w0 = R.Wlo; w0 < R.W; w0 += 32) {
      const int w = w0 + lane;
      uint32_t m = w < R.W ? __ldcg(mask + w) : 0u;
      const int lo = 32 * w;
      if (pl.H > lo) m = pl.H - lo >= 32 ? 0u : m & (~0u << (pl.H - lo));  // hot bits
      const int c = __popc(m);
      int incl = c;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
      }
      if (w < R.W && snake_owner(w - R.Wlo, nS) == s) {
        int pos = base + incl - c;
        for (; m; m &= m - 1u, ++pos) __stcg(P.idx + pos, lo + __ffs(m) - 1);
      }
      base += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0 && s == 0) __stcg(P.count, base);
    __syncwarp();
    if (lane == 0) mbar_arrive(S.listdone, 1u);  // done with this layer's mask
  }
}

// ---------------------------------------------------------------- consumers

template <int WT, int ACT, int PT, bool TR>
__device__ void consumers(const StackParams& P, const Smem& S) {
  constexpr bool two = (ACT == PI_REGLU);
  const Plan& pl = P.pl;
  WsHeader* hdr = P.hdr;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nS = gridDim.x, s = blockIdx.x;
  const Ranges R = ranges(pl);
  const int d = pl.d, nb = d / 32;
  // Units of the predictor and up-projection phases are shared by groups of
  // WPG warps; unit uc goes to group uc % GW.  GW divides the ring depth, so
  // a stage is always consumed by the same group and every warp has seen the
  // previous phase of each stage it waits on (exact parity test).
  const int GW = pl.gw, WPG = NCW / GW, grp = warp / WPG, wg = warp % WPG;
  const int gtid = wg * 32 + lane, GT = WPG * 32;
  // The down-projection phase uses GD groups of NCW / GD warps.
  const int GD = pl.gd, WPD = NCW / GD, dgrp = warp / WPD;
  const int dtid = (warp % WPD) * 32 + lane, DT = WPD * 32;
  Cursor cu;  // the unit sequence (every warp walks all of it)
  uint32_t nbar = 0;
  int cur_l = 0;
  uint32_t l_uc0 = 0;
  const uint32_t gwm = (uint32_t)GW - 1u, gdm = (uint32_t)GD - 1u;  // GW, GD: powers of 2

  // the current unit's data has landed (false on abort / timeout)
  auto ready = [&]() -> bool {
    const bool ok = wait_mbar(&S.full[cu.st], cu.gen & 1u, S, hdr);
    if (TR && P.utrace && tid == 0) utstamp<TR>(P, cur_l, cu.uc - l_uc0, 1, gtime());
    return __all_sync(0xffffffffu, ok);
  };
  auto stage = [&]() { return S.ring + (size_t)cu.st * pl.sb; };
  // each of the `warps` warps that shared the current unit releases its part of it
  auto release = [&](int warps) {
    __syncwarp();
    if (lane == 0) mbar_arrive(&S.empty[cu.st], (uint32_t)(NCW / warps));
    if (TR && P.utrace && tid == 0) utstamp<TR>(P, cur_l, cu.uc - l_uc0, 2, gtime());
  };
  auto gsync_arrive = [&]() {
    csync();
    ++nbar;
    if (tid == 0 && !*S.abort) grid_arrive(&hdr->counters[0]);
  };
  auto gsync_wait = [&]() {
    if (tid == 0) grid_wait(hdr, nbar * (uint32_t)nS, S);
    csync();
  };

  for (int l = 0; l < P.n_layers; ++l) {
    const LayerPtrs& L = P.L[l];
    uint32_t* mask = layer_mask(P, l);
    const int tag = (l + 1) << 2;
    cur_l = l;
    l_uc0 = cu.uc;

    // ---- x^ = x / sqrt(mean(x^2) + 1e-6): each thread takes 8-element
    // chunks c = tid, tid + NCT, ... (all loads issued at once); one CTA-wide
    // reduction gives sum(x^2) and max|x|; 16-byte stores of x^ (and of its
    // int16 copy) are conflict-free
    if (tid == 0) tstamp<TR>(P, l, 0, gtime());
    {
      constexpr int MC = 3;  // chunks per thread, d <= 12288
      const int nc8 = d / 8;
      const float4* x4 = reinterpret_cast<const float4*>(P.x);
      float4 xa[MC], xb[MC];
#pragma unroll
      for (int m = 0; m < MC; ++m) {
        const int c = tid + m * NCT;
        const bool in = c < nc8;
        xa[m] = in ? __ldcg(x4 + 2 * c) : make_float4(0.f, 0.f, 0.f, 0.f);
        xb[m] = in ? __ldcg(x4 + 2 * c + 1) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
      float ss = 0.f, mx = 0.f;
#pragma unroll
      for (int m = 0; m < MC; ++m) {
        const float e[8] = {xa[m].x, xa[m].y, xa[m].z, xa[m].w, xb[m].x, xb[m].y, xb[m].z, xb[m].w};
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          ss = fmaf(e[k], e[k], ss);
          mx = fmaxf(mx, fabsf(e[k]));
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        ss += __shfl_xor_sync(0xffffffffu, ss, o);
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      }
      if (lane == 0) {
        S.redA[warp] = ss;
        S.redA[NCW + warp] = mx;
      }
      csync();
      float tot = 0.f, amax = 0.f;
#pragma unroll
      for (int w = 0; w < NCW; ++w) {
        tot += S.redA[w];
        amax = fmaxf(amax, S.redA[NCW + w]);
      }
      const float inv = 1.0f / sqrtf(tot / (float)d + 1e-6f);
      float ixs = 1.f;
      if constexpr (WT == PI_Q4_0) {
        const float xm = amax * inv;  // max |x^|: scaling by inv > 0 keeps the order
        const float xs = xm > 0.f ? xm / 32767.0f : 1.0f;
        ixs = 1.0f / xs;
        if (tid == 0) *S.xscale = xs;
      }
      float4* xf4 = reinterpret_cast<float4*>(S.xf);
#pragma unroll
      for (int m = 0; m < MC; ++m) {
        const int c = tid + m * NCT;
        if (c >= nc8) break;  // warp-uniform for Q4_0 (d % 256 == 0)
        const float4 lo = make_float4(xa[m].x * inv, xa[m].y * inv, xa[m].z * inv, xa[m].w * inv);
        const float4 hi = make_float4(xb[m].x * inv, xb[m].y * inv, xb[m].z * inv, xb[m].w * inv);
        if constexpr (PT == PI_F16) {
          xf4[c] = lo;  // split-half layout
          xf4[nc8 + c] = hi;
        } else {
          xf4[2 * c] = lo;
          xf4[2 * c + 1] = hi;
        }
        if constexpr (WT == PI_Q4_0) {
          const float e[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
          int v[8], t = 0;
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            int q = __float2int_rn(e[k] * ixs);
            q = q > 32767 ? 32767 : (q < -32767 ? -32767 : q);
            v[k] = q;
            t += q;
          }
          // chunk c = 4 * block + sub-chunk: sub-chunk-major int16 layout
          reinterpret_cast<int4*>(S.xi)[(c & 3) * nb + (c >> 2)] =
              make_int4((v[0] & 0xFFFF) | (v[1] << 16), (v[2] & 0xFFFF) | (v[3] << 16),
                        (v[4] & 0xFFFF) | (v[5] << 16), (v[6] & 0xFFFF) | (v[7] << 16));
          // block sum over the block's 4 chunks (4 adjacent lanes)
          t += __shfl_xor_sync(0xffffffffu, t, 1);
          t += __shfl_xor_sync(0xffffffffu, t, 2);
          if ((lane & 3) == 0) S.bsum[c >> 2] = t;
        }
      }
      csync();
    }
    if (tid == 0) tstamp<TR>(P, l, 1, gtime());

    // ---- A: u = P1 xh; each row shared by one warp group
    const int nA = R.kA1 - R.kA0;
    {
      constexpr int CCP = WTraits<PT>::CHUNK_COLS;
      const int nch = d / CCP;
      for (int a = 0; a < nA; ++a, cu.next(pl.ns)) {
        if ((int)(cu.uc & gwm) != grp) continue;
        if (!ready()) continue;
        const char* row = stage();
        float v0 = 0.f, v1 = 0.f, v2 = 0.f, v3 = 0.f;
        int c = gtid;
        for (; c + 3 * GT < nch; c += 4 * GT) {
          v0 += chunk_dot<PT>(lds128(row + (size_t)c * 16), S.xf, c, d);
          v1 += chunk_dot<PT>(lds128(row + (size_t)(c + GT) * 16), S.xf, c + GT, d);
          v2 += chunk_dot<PT>(lds128(row + (size_t)(c + 2 * GT) * 16), S.xf, c + 2 * GT, d);
          v3 += chunk_dot<PT>(lds128(row + (size_t)(c + 3 * GT) * 16), S.xf, c + 3 * GT, d);
        }
        for (; c < nch; c += GT) v0 += chunk_dot<PT>(lds128(row + (size_t)c * 16), S.xf, c, d);
        release(WPG);
        float v = warp_sum((v0 + v1) + (v2 + v3));
        if (lane == 0) S.redA[MAXA + a * NCW + wg] = v;
      }
      csync();
      for (int a = tid; a < nA; a += NCT) {
        const int wpg = NCW / (int)(pl.gw);
        float v = 0.f;
        for (int w = 0; w < wpg; ++w) v += S.redA[MAXA + a * NCW + w];
        __stcg(P.u + R.kA0 + a, v);
      }
    }
    if (tid == 0) tstamp<TR>(P, l, 2, gtime());
    gsync_arrive();  // 1: u complete
    // biases used later in this layer: their load latency overlaps the barrier
    for (int k = tid; k < R.nw * 32; k += NCT) {
      const int j = 32 * cold_word(k >> 5, R) + (k & 31);
      S.pbs[k] = (L.pbias && j < pl.F) ? L.pbias[j] : 0.f;
    }
    for (int i = tid; i < R.nh; i += NCT) S.hbs[i] = L.bias ? L.bias[S.items[i]] : 0.f;
    gsync_wait();
    if (tid == 0) tstamp<TR>(P, l, 3, gtime());

    // ---- B: logits of the CTA's mask words; the group's warps take the rows
    for (int k = tid; k < pl.r; k += NCT) S.us[vpos<PT>(k, pl.r)] = __ldcg(P.u + k);
    for (int k = tid; k < R.nw; k += NCT) S.bw[k] = 0u;
    csync();
    {
      constexpr int CCP = WTraits<PT>::CHUNK_COLS;
      const int nch = pl.r / CCP;  // <= 32 * MU (plan)
      // the lane's u chunks, kept in registers for the whole phase
      constexpr int MU = 4;
      VFrag ur[MU];
#pragma unroll
      for (int m = 0; m < MU; ++m) {
        const int c = lane + 32 * m;
        if (c < nch) {
          ur[m] = vfrag<PT>(S.us, c, pl.r);
        } else {
          ur[m].lo = ur[m].hi = make_float4(0.f, 0.f, 0.f, 0.f);
        }
      }
      for (int kw = 0; kw < R.nw; ++kw) {
        const int w = cold_word(kw, R);
        for (int ja = 32 * w; ja < 32 * w + 32 && ja < pl.F; ja += pl.G, cu.next(pl.ns)) {
          if ((int)(cu.uc & gwm) != grp) continue;
          if (!ready()) continue;
          const char* buf = stage();
          const int jb = min(ja + pl.G, pl.F);
          uint32_t bits = 0u;
          // a warp takes rows j and j + WPG together (one u load for both)
          for (int j = ja + wg; j < jb; j += 2 * WPG) {
            const int j2 = j + WPG;
            const bool pair = j2 < jb;  // warp-uniform
            const char* row = buf + (size_t)(j - ja) * pl.p2_row;
            const char* row2 = row + (size_t)WPG * pl.p2_row;
            float z0 = 0.f, z1 = 0.f;
#pragma unroll
            for (int m = 0; m < MU; ++m) {
              const int c = lane + 32 * m;
              if (c >= nch) break;
              z0 += frag_dot<PT>(lds128(row + (size_t)c * 16), ur[m]);
              if (pair) z1 += frag_dot<PT>(lds128(row2 + (size_t)c * 16), ur[m]);
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
              z0 += __shfl_xor_sync(0xffffffffu, z0, o);
              z1 += __shfl_xor_sync(0xffffffffu, z1, o);
            }
            const float za = z0 + S.pbs[32 * kw + (j & 31)];
            if (j >= pl.H && za > P.theta) bits |= 1u << (j & 31);
            if (pair) {
              const float zb = z1 + S.pbs[32 * kw + (j2 & 31)];
              if (j2 >= pl.H && zb > P.theta) bits |= 1u << (j2 & 31);
            }
          }
          release(WPG);
          if (lane == 0 && bits) atomicOr(&S.bw[kw], bits);
        }
      }
    }
    csync();
    for (int k = tid; k < R.nw; k += NCT) {
      const int w = cold_word(k, R);
      uint32_t word = S.bw[k];
      const int lo = 32 * w;
      if (pl.H > lo) word |= (pl.H - lo >= 32) ? 0xFFFFFFFFu : ((1u << (pl.H - lo)) - 1u);
      __stcg(mask + w, word);
    }
    for (int w = (int)((long long)s * R.Wlo / nS) + tid; w < (int)((long long)(s + 1) * R.Wlo / nS);
         w += NCT)
      __stcg(mask + w, 0xFFFFFFFFu);
    // the CTA's cold list: the predicted cold neurons of its own mask words,
    // ascending (one lane per word), published to the producers at once; no
    // grid barrier is needed, the CTAs' word shares being disjoint
    if (warp == 0) {
      if (l > 0 && lane == 0) (void)wait_mbar(S.listdone, (uint32_t)(l - 1) & 1u, S, hdr);
      __syncwarp();
      const int nw = R.nw;  // <= 32 (plan)
      const uint32_t word = lane < nw ? S.bw[lane] : 0u;
      const int cnt = __popc(word);
      int incl = cnt;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
      }
      const int total = __shfl_sync(0xffffffffu, incl, 31);
      int pos = R.nh + incl - cnt;
      for (uint32_t m = word; m; m &= m - 1u, ++pos) {
        const int j = 32 * cold_word(lane, R) + __ffs(m) - 1;
        S.items[pos] = j;
        S.hbs[pos] = L.bias ? L.bias[j] : 0.f;
      }
      if (lane == 0) *S.nc = total;
      __syncwarp();
      if (lane == 0) mbar_arrive(S.listbar, 1u);  // releases the list to the producers
    }
    if (tid == 0) tstamp<TR>(P, l, 4, gtime());
    csync();
    const int nc = *S.nc;

    // ---- C: first records (hot units, then cold units); each unit shared
    // by one warp group.  Right after a unit the group's per-warp partial
    // sums are combined in fixed order (a named barrier per group, partial
    // buffers alternating by the group's unit parity) and the items' flags
    // are set, so the producers can fetch the D records at once.
    int gk = 0;  // units this group has taken in this layer
    // Q4_0: the thread's int16 x^ blocks (k = gtid + GT m) in registers for
    // phase C and the ReGLU up groups of phase D (same thread-to-block map)
    constexpr int MQ = 2;  // d / 32 <= MQ * GT (plan)
    int xq[MQ][16], bq[MQ];
#pragma unroll
    for (int m = 0; m < MQ; ++m) {
      bq[m] = 0;
#pragma unroll
      for (int e = 0; e < 16; ++e) xq[m][e] = 0;
    }
    if constexpr (WT == PI_Q4_0) {
      const int4* xb = reinterpret_cast<const int4*>(S.xi);
#pragma unroll
      for (int m = 0; m < MQ; ++m) {
        const int k = gtid + GT * m;
        if (k < nb) {
          const int4 x0 = xb[k], x1 = xb[nb + k], x2 = xb[2 * nb + k], x3 = xb[3 * nb + k];
          const int v[16] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w,
                             x2.x, x2.y, x2.z, x2.w, x3.x, x3.y, x3.z, x3.w};
#pragma unroll
          for (int e = 0; e < 16; ++e) xq[m][e] = v[e];
          bq[m] = -8 * S.bsum[k];
        }
      }
    }
    auto unit_items = [&](int i0, int n) {
      if ((int)(cu.uc & gwm) == grp) {
        const bool ok = ready();
        float a[kMaxRec];
#pragma unroll
        for (int r = 0; r < kMaxRec; ++r) a[r] = 0.f;
        if (ok) {
          const char* base = stage();
          if constexpr (WT == PI_Q4_0) {
#pragma unroll
            for (int m = 0; m < MQ; ++m) {
              const int k = gtid + GT * m;
              if (k >= nb) break;
#pragma unroll
              for (int r = 0; r < kMaxRec; ++r) {
                if (r >= n) break;
                const char* buf = base + (size_t)r * pl.first_b;
                const uint4 cf = lds128(buf + (size_t)k * 16);
                const float sf = h2f(reinterpret_cast<const uint16_t*>(buf + pl.rowb)[k]);
                a[r] = fmaf((float)q4_block_dot(cf, xq[m], bq[m]), sf, a[r]);
              }
            }
          } else {
            constexpr int CCW = WTraits<WT>::CHUNK_COLS;
            const int nch = d / CCW;
            for (int c = gtid; c < nch; c += GT) {
#pragma unroll
              for (int r = 0; r < kMaxRec; ++r) {
                if (r >= n) break;
                a[r] += chunk_dot<WT>(lds128(base + (size_t)r * pl.first_b + (size_t)c * 16), S.xf,
                                      c, d);
              }
            }
          }
          release(WPG);
        }
#pragma unroll
        for (int r = 0; r < kMaxRec; ++r) {
          if (r >= n) break;
          a[r] = warp_sum(a[r]);
        }
        float* rc = S.redC + (size_t)((grp * 2 + (gk & 1)) * kMaxRec) * WPG;
        if (lane == 0) {
#pragma unroll
          for (int r = 0; r < kMaxRec; ++r) {
            if (r >= n) break;
            rc[r * WPG + wg] = a[r];
          }
        }
        // every warp of the group reaches this barrier for every unit the
        // group owns, whether or not its wait succeeded
        asm volatile("bar.sync %0, %1;" ::"r"(2 + grp), "r"(GT) : "memory");
        if (wg == 0 && lane < n) {
          const float* q = rc + lane * WPG;
          float g = 0.f;
          for (int w = 0; w < WPG; ++w) g += q[w];
          if constexpr (WT == PI_Q4_0) g *= *S.xscale;
          g += S.hbs[i0 + lane];
          float h = g > 0.f ? g : 0.f;  // ReGLU: the gate's ReLU; W_up comes in phase D
          if constexpr (!two) {
            if (pl.sq) h *= h;  // squared ReLU
          }
          S.hval[i0 + lane] = h;
          __threadfence_block();
          S.flag[i0 + lane] = tag | (h != 0.f ? 2 : 1);
        }
        ++gk;
      }
      cu.next(pl.ns);
    };
    for (int gi = 0; gi < R.ngh; ++gi) {
      const int j0 = hot_group_first(gi, pl);
      unit_items(gi * pl.hp, min(pl.hp, pl.H - j0));
    }
    if (tid == 0) tstamp<TR>(P, l, 5, gtime());

    // ---- then the CTA's cold neurons (nc was read after the barrier that
    // follows the list, so every warp of a group walks the same units and
    // reaches its group barrier the same number of times)
    if (tid == 0) tstamp<TR>(P, l, 6, gtime());
    for (int i = 0; i < nc; i += pl.cp) unit_items(R.nh + i, min(pl.cp, nc - i));
    csync();
    if (tid == 0) tstamp<TR>(P, l, 7, gtime());

    // ---- D: D records of the items whose first pre-activation is positive
    // (hval != 0), pl.dr per unit, each unit shared by one of GD warp
    // groups, each group covering every column with its own accumulators.
    // ReGLU: the group first forms each record's W_up dot (per-warp partials
    // combined in fixed order after a named barrier), h = gate * up, then
    // accumulates h times the down row.
    const int ni = R.nh + nc;
    if (warp == 0) {
      int base = 0;
      for (int i0 = 0; i0 < ni; i0 += 32) {
        const int i = i0 + lane;
        const bool nz = i < ni && S.hval[i] != 0.f;
        const uint32_t bal = __ballot_sync(0xffffffffu, nz);
        if (nz) S.dlist[base + __popc(bal & ((1u << lane) - 1u))] = i;
        base += __popc(bal);
      }
      if (lane == 0) S.scan[NCW] = base;
    }
    csync();
    const int nd = S.scan[NCW];
    const int nruns = (nd + pl.dr - 1) / pl.dr;  // units of pl.dr records
    const int wd = warp % WPD;
    int dk = 0;  // D units this group has taken in this layer
    // h of the unit's record rr (ReGLU: after the group's W_up dot)
    auto unit_h = [&](int q0, int len, const float* part_up, int rr) -> float {
      const float g = S.hval[S.dlist[q0 + rr]];
      if constexpr (!two) return g;
      float u = 0.f;
      for (int w = 0; w < WPD; ++w) u += part_up[rr * WPD + w];
      if constexpr (WT == PI_Q4_0) u *= *S.xscale;
      return g * u;
    };
    if constexpr (!two) {
      if constexpr (WT == PI_Q4_0) {
        // QB Q4_0 blocks (32 columns each) per thread (the plan keeps d / 32
        // within a group's QB * DT).  sum_j hs_j (q - 8), hs_j = h_j * scale,
        // is accumulated as sum_j 16 hs_j (1 + q/16) with packed fp32x2 FMAs on
        // floats built from the nibbles by byte permutes, minus 24 sum_j hs_j
        // at the end.
        constexpr int QB = kQ4Blocks;
        const int nch = d / 32;
        float2 acc[QB][16];
        float corr[QB];
  #pragma unroll
        for (int kb = 0; kb < QB; ++kb) {
          corr[kb] = 0.f;
  #pragma unroll
          for (int e = 0; e < 16; ++e) acc[kb][e] = make_float2(0.f, 0.f);
        }
        for (int q = 0; q < nruns; ++q, cu.next(pl.ns)) {
          if ((int)(cu.uc & gdm) != dgrp) continue;
          const bool ok = ready();
          const int q0 = q * pl.dr, len = min(pl.dr, nd - q0);
          float* pu = S.redD + (size_t)((dgrp * 2 + (dk & 1)) * DR2MAX) * WPD;
          if constexpr (two) {
            // W_up dots of the unit's records
            for (int rr = 0; rr < len; ++rr) {
              float a = 0.f;
              if (ok) {
                const char* row = stage() + (size_t)rr * pl.d2_bytes;
                const int4* xb = reinterpret_cast<const int4*>(S.xi);
                for (int c = dtid; c < nch; c += DT) {
                  const int4 x0 = xb[c], x1 = xb[nch + c], x2 = xb[2 * nch + c], x3 = xb[3 * nch + c];
                  const int xw[16] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w,
                                      x2.x, x2.y, x2.z, x2.w, x3.x, x3.y, x3.z, x3.w};
                  a = fmaf((float)q4_block_dot(lds128(row + (size_t)c * 16), xw, -8 * S.bsum[c]),
                           h2f(reinterpret_cast<const uint16_t*>(row + pl.rowb)[c]), a);
                }
              }
              a = warp_sum(a);
              if (lane == 0) pu[rr * WPD + wd] = a;
            }
            asm volatile("bar.sync %0, %1;" ::"r"(6 + dgrp), "r"(DT) : "memory");
          }
          if (ok) {
  #pragma unroll 1
            for (int rr = 0; rr < len; ++rr) {
              const char* row = stage() + (size_t)rr * pl.d2_bytes + pl.o_d2_down;
              const float hv = unit_h(q0, len, pu, rr);
  #pragma unroll
              for (int kb = 0; kb < QB; ++kb) {
                const int c = dtid + kb * DT;
                if (c >= nch) break;
                const uint4 v = lds128(row + (size_t)c * 16);
                const float hs = hv * h2f(reinterpret_cast<const uint16_t*>(row + pl.rowb)[c]);
                corr[kb] += hs;
                const float2 h2 = make_float2(16.f * hs, 16.f * hs);
                const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
  #pragma unroll
                for (int m = 0; m < 4; ++m) {
                  // byte b: 0x80 | q << 3 for element 4m + b (low nibbles) / 16 + 4m + b (high)
                  const uint32_t lo = ((wv[m] << 3) & 0x78787878u) | 0x80808080u;
                  const uint32_t hi = ((wv[m] >> 1) & 0x78787878u) | 0x80808080u;
  #pragma unroll
                  for (int b = 0; b < 4; b += 2) {
                    acc[kb][(4 * m + b) >> 1] =
                        __ffma2_rn(nib_pair(lo, b), h2, acc[kb][(4 * m + b) >> 1]);
                    acc[kb][(16 + 4 * m + b) >> 1] =
                        __ffma2_rn(nib_pair(hi, b), h2, acc[kb][(16 + 4 * m + b) >> 1]);
                  }
                }
              }
            }
            release(WPD);
          }
          ++dk;
        }
        // the CTA's partial row s: group GD-1 leaves its sums in shared memory
        // (the fp32 copy of x^, free until the next layer), group 0 adds them
        // to its own in a fixed order and writes the row
        float4* xs4 = reinterpret_cast<float4*>(S.xf);
        csync();
        if (GD > 1 && dgrp == GD - 1) {
  #pragma unroll
          for (int kb = 0; kb < QB; ++kb) {
            const int c = dtid + kb * DT;
            if (c >= nch) break;
            const float k24 = 24.f * corr[kb];
  #pragma unroll
            for (int e = 0; e < 16; e += 2)
              xs4[c * 8 + e / 2] = make_float4(acc[kb][e].x - k24, acc[kb][e].y - k24,
                                               acc[kb][e + 1].x - k24, acc[kb][e + 1].y - k24);
          }
        }
        csync();
        if (dgrp == 0) {
  #pragma unroll
          for (int kb = 0; kb < QB; ++kb) {
            const int c = dtid + kb * DT;
            if (c >= nch) break;
            float* part = P.part + (size_t)s * d + (size_t)c * 32;
            const float k24 = 24.f * corr[kb];
  #pragma unroll
            for (int e = 0; e < 16; e += 2) {
              float4 v = make_float4(acc[kb][e].x - k24, acc[kb][e].y - k24, acc[kb][e + 1].x - k24,
                                     acc[kb][e + 1].y - k24);
              if (GD > 1) v = f4add(v, xs4[c * 8 + e / 2]);
              __stcg(reinterpret_cast<float4*>(part + 2 * e), v);
            }
          }
        }
      } else {
        // fp16 / fp32 rows: up to 48 columns per thread (32 for ReGLU, whose
        // D phase also forms the W_up dots)
        constexpr int CC = WTraits<WT>::CHUNK_COLS;
        constexpr int MAXK = (two ? 32 : 48) / CC;  // chunks per thread of a D group
        const int nch = d / CC;
        float acc[MAXK][CC];
  #pragma unroll
        for (int k = 0; k < MAXK; ++k)
  #pragma unroll
          for (int e = 0; e < CC; ++e) acc[k][e] = 0.f;
        for (int q = 0; q < nruns; ++q, cu.next(pl.ns)) {
          if ((int)(cu.uc & gdm) != dgrp) continue;
          const bool ok = ready();
          const int q0 = q * pl.dr, len = min(pl.dr, nd - q0);
          float* pu = S.redD + (size_t)((dgrp * 2 + (dk & 1)) * DR2MAX) * WPD;
          if constexpr (two) {
            for (int rr = 0; rr < len; ++rr) {
              float a = 0.f;
              if (ok) {
                const char* row = stage() + (size_t)rr * pl.d2_bytes;
                for (int c = dtid; c < nch; c += DT)
                  a += chunk_dot<WT>(lds128(row + (size_t)c * 16), S.xf, c, d);
              }
              a = warp_sum(a);
              if (lane == 0) pu[rr * WPD + wd] = a;
            }
            asm volatile("bar.sync %0, %1;" ::"r"(6 + dgrp), "r"(DT) : "memory");
          }
          if (ok) {
            for (int rr = 0; rr < len; ++rr) {
              const char* row = stage() + (size_t)rr * pl.d2_bytes + pl.o_d2_down;
              const float hv = unit_h(q0, len, pu, rr);
  #pragma unroll
              for (int k = 0; k < MAXK; ++k) {
                const int c = dtid + k * DT;
                if (c >= nch) break;
                const uint4 v = lds128(row + (size_t)c * 16);
                if constexpr (WT == PI_F16) {
                  float f[8];
                  f16x8_to_f32(v, f);
  #pragma unroll
                  for (int e = 0; e < 8; ++e) acc[k][e] = fmaf(hv, f[e], acc[k][e]);
                } else {
                  acc[k][0] = fmaf(hv, __uint_as_float(v.x), acc[k][0]);
                  acc[k][1] = fmaf(hv, __uint_as_float(v.y), acc[k][1]);
                  acc[k][2] = fmaf(hv, __uint_as_float(v.z), acc[k][2]);
                  acc[k][3] = fmaf(hv, __uint_as_float(v.w), acc[k][3]);
                }
              }
            }
            release(WPD);
          }
          ++dk;
        }
        // the CTA's partial row s: group GD-1 leaves its sums in shared memory
        // (the fp32 copy of x^, free until the next layer), group 0 adds them
        // to its own in a fixed order and writes the row
        float4* xs4 = reinterpret_cast<float4*>(S.xf);
        csync();
        if (GD > 1 && dgrp == GD - 1) {
  #pragma unroll
          for (int k = 0; k < MAXK; ++k) {
            const int c = dtid + k * DT;
            if (c >= nch) break;
  #pragma unroll
            for (int e = 0; e < CC; e += 4)
              xs4[(c * CC + e) / 4] = make_float4(acc[k][e], acc[k][e + 1], acc[k][e + 2], acc[k][e + 3]);
          }
        }
        csync();
        if (dgrp == 0) {
          float* part = P.part + (size_t)s * d;
  #pragma unroll
          for (int k = 0; k < MAXK; ++k) {
            const int c = dtid + k * DT;
            if (c >= nch) break;
  #pragma unroll
            for (int e = 0; e < CC; e += 4) {
              float4 v = make_float4(acc[k][e], acc[k][e + 1], acc[k][e + 2], acc[k][e + 3]);
              if (GD > 1) v = f4add(v, xs4[(c * CC + e) / 4]);
              __stcg(reinterpret_cast<float4*>(part + c * CC + e), v);
            }
          }
        }
      }
    } else {
      // ReGLU: a two-role pipeline over the D units ([W_up | W_down^T]
      // records of the items whose gate fired, pl.dr per unit).  Warps
      // 0 .. NCW/2-1 form two up groups; group q & 1 forms unit q's W_up dots
      // (per-warp partials combined in fixed order after a named barrier),
      // h = gate * up for its records, and raises the unit's flag.  Warps
      // NCW/2 .. NCW-1 take every unit in order once its flag is up and
      // accumulate h times the down rows over all columns (one partial row
      // per CTA).  The two roles work on consecutive units at once.
      constexpr int UW = NCW / 4;              // warps per up group
      constexpr int UT = UW * 32, VT = NCT / 2;
      const bool vrole = warp >= NCW / 2;
      const int ug = warp / UW;                // up group (up role)
      const int uw = warp % UW, ut = uw * 32 + lane;
      const int vt = tid - NCT / 2;            // thread of the down role
      const int ntag = (l + 1) << 16;
      if (!vrole) {
        int uk = 0;  // units this up group has taken in this layer
        for (int q = 0; q < nruns; ++q, cu.next(pl.ns)) {
          if ((q & 1) != ug) continue;
          const bool ok = ready();
          const int q0 = q * pl.dr, len = min(pl.dr, nd - q0);
          float* pu = S.redD + (size_t)((ug * 2 + (uk & 1)) * DR2MAX) * UW;
          for (int rr = 0; rr < len; ++rr) {
            float a = 0.f;
            if (ok) {
              const char* row = stage() + (size_t)rr * pl.d2_bytes;
              if constexpr (WT == PI_Q4_0) {
                static_assert(UT == NCT / 4, "up-group threads map to the phase-C blocks");
#pragma unroll
                for (int m = 0; m < MQ; ++m) {
                  const int c = ut + UT * m;
                  if (c >= nb) break;
                  a = fmaf((float)q4_block_dot(lds128(row + (size_t)c * 16), xq[m], bq[m]),
                           h2f(reinterpret_cast<const uint16_t*>(row + pl.rowb)[c]), a);
                }
              } else {
                constexpr int CCW = WTraits<WT>::CHUNK_COLS;
                for (int c = ut; c < d / CCW; c += UT)
                  a += chunk_dot<WT>(lds128(row + (size_t)c * 16), S.xf, c, d);
              }
            }
            a = warp_sum(a);
            if (lane == 0) pu[rr * UW + uw] = a;
          }
          // every warp of the up group reaches this barrier for every unit it owns
          asm volatile("bar.sync %0, %1;" ::"r"(2 + ug), "r"(UT) : "memory");
          if (uw == 0) {
            if (lane < len) {
              float u = 0.f;
              for (int w = 0; w < UW; ++w) u += pu[lane * UW + w];
              if constexpr (WT == PI_Q4_0) u *= *S.xscale;
              const int i = S.dlist[q0 + lane];
              S.hval[i] = S.hval[i] * u;  // gate (after its ReLU) * up
            }
            __syncwarp();
            __threadfence_block();
            if (lane == 0) S.hflag[q & (HQ - 1)] = ntag | (q + 1);
          }
          if (ok) release(NCW / 2);
          ++uk;
        }
      } else {
        // the unit's flag, by one lane per warp (bounded)
        auto hready = [&](int q) -> bool {
          int okf = 1;
          if (lane == 0) {
            const int want = ntag | (q + 1);
            if (S.hflag[q & (HQ - 1)] != want) {
              const uint64_t t0 = gtime();
              while (S.hflag[q & (HQ - 1)] != want) {
                if (*S.abort) { okf = 0; break; }
                if (gtime() - t0 > kTimeoutNs) { raise_abort(S, hdr); okf = 0; break; }
                __nanosleep(32);
              }
            }
          }
          __syncwarp();
          return __shfl_sync(0xffffffffu, okf, 0) != 0;
        };
        float* part = P.part + (size_t)s * d;
        if constexpr (WT == PI_Q4_0) {
          // one Q4_0 block (32 columns) per thread, accumulated as in the
          // ReLU branch above
          const int nch = d / 32, c = vt;
          float2 acc[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) acc[e] = make_float2(0.f, 0.f);
          float corr = 0.f;
          for (int q = 0; q < nruns; ++q, cu.next(pl.ns)) {
            const bool ok = ready();
            const bool hk = hready(q);
            const int q0 = q * pl.dr, len = min(pl.dr, nd - q0);
            if (ok && hk && c < nch) {
#pragma unroll 1
              for (int rr = 0; rr < len; ++rr) {
                const char* row = stage() + (size_t)rr * pl.d2_bytes + pl.o_d2_down;
                const uint4 v = lds128(row + (size_t)c * 16);
                const float hs = S.hval[S.dlist[q0 + rr]] *
                                 h2f(reinterpret_cast<const uint16_t*>(row + pl.rowb)[c]);
                corr += hs;
                const float2 h2 = make_float2(16.f * hs, 16.f * hs);
                const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                  const uint32_t lo = ((wv[m] << 3) & 0x78787878u) | 0x80808080u;
                  const uint32_t hi = ((wv[m] >> 1) & 0x78787878u) | 0x80808080u;
#pragma unroll
                  for (int b2 = 0; b2 < 4; b2 += 2) {
                    acc[(4 * m + b2) >> 1] = __ffma2_rn(nib_pair(lo, b2), h2, acc[(4 * m + b2) >> 1]);
                    acc[(16 + 4 * m + b2) >> 1] =
                        __ffma2_rn(nib_pair(hi, b2), h2, acc[(16 + 4 * m + b2) >> 1]);
                  }
                }
              }
            }
            if (ok) release(NCW);
          }
          if (c < nch) {
            const float k24 = 24.f * corr;
#pragma unroll
            for (int e = 0; e < 16; e += 2)
              __stcg(reinterpret_cast<float4*>(part + (size_t)c * 32 + 2 * e),
                     make_float4(acc[e].x - k24, acc[e].y - k24, acc[e + 1].x - k24,
                                 acc[e + 1].y - k24));
          }
        } else {
          constexpr int CC = WTraits<WT>::CHUNK_COLS;
          constexpr int MAXK = 48 / CC;
          const int nch = d / CC;
          float acc[MAXK][CC];
#pragma unroll
          for (int k = 0; k < MAXK; ++k)
#pragma unroll
            for (int e = 0; e < CC; ++e) acc[k][e] = 0.f;
          for (int q = 0; q < nruns; ++q, cu.next(pl.ns)) {
            const bool ok = ready();
            const bool hk = hready(q);
            const int q0 = q * pl.dr, len = min(pl.dr, nd - q0);
            if (ok && hk) {
              for (int rr = 0; rr < len; ++rr) {
                const char* row = stage() + (size_t)rr * pl.d2_bytes + pl.o_d2_down;
                const float hv = S.hval[S.dlist[q0 + rr]];
#pragma unroll
                for (int k = 0; k < MAXK; ++k) {
                  const int c = vt + k * VT;
                  if (c >= nch) break;
                  const uint4 v = lds128(row + (size_t)c * 16);
                  if constexpr (WT == PI_F16) {
                    float f[8];
                    f16x8_to_f32(v, f);
#pragma unroll
                    for (int e = 0; e < 8; ++e) acc[k][e] = fmaf(hv, f[e], acc[k][e]);
                  } else {
                    acc[k][0] = fmaf(hv, __uint_as_float(v.x), acc[k][0]);
                    acc[k][1] = fmaf(hv, __uint_as_float(v.y), acc[k][1]);
                    acc[k][2] = fmaf(hv, __uint_as_float(v.z), acc[k][2]);
                    acc[k][3] = fmaf(hv, __uint_as_float(v.w), acc[k][3]);
                  }
                }
              }
            }
            if (ok) release(NCW);
          }
#pragma unroll
          for (int k = 0; k < MAXK; ++k) {
            const int c = vt + k * VT;
            if (c >= nch) break;
#pragma unroll
            for (int e = 0; e < CC; e += 4)
              __stcg(reinterpret_cast<float4*>(part + c * CC + e),
                     make_float4(acc[k][e], acc[k][e + 1], acc[k][e + 2], acc[k][e + 3]));
          }
        }
      }
      csync();
    }
    if (tid == 0) {
      atomicAdd(&hdr->rows_listed, (unsigned long long)ni);
      if constexpr (two) atomicAdd(&hdr->rows_second, (unsigned long long)nd);
      atomicAdd(&hdr->rows_down, (unsigned long long)nd);
      tstamp<TR>(P, l, 8, gtime());
    }
    gsync_arrive();  // 3: partials complete
    gsync_wait();
    if (tid == 0) tstamp<TR>(P, l, 9, gtime());

    // ---- E: reduce this CTA's float4 column slice over the nS partial rows
    // in a fixed order (rows in interleaved groups, then the groups in
    // order), residual add.
    {
      const int q4n = d / 4, nP = nS;
      const int cq0 = (int)((long long)s * q4n / nS), cq1 = (int)((long long)(s + 1) * q4n / nS);
      const int nq = cq1 - cq0;  // <= 32
      const int g = nq > 0 ? NCT / nq : 0;
      const float4* pp = reinterpret_cast<const float4*>(P.part);
      float4* x4 = reinterpret_cast<float4*>(P.x) + cq0 + tid;
      const float4 xo = tid < nq ? __ldcg(x4) : make_float4(0.f, 0.f, 0.f, 0.f);
      if (nq > 0 && tid < nq * g) {
        // rows gi, gi + g, ... summed in that order; 12 loads in flight
        constexpr int ER = 8;
        const int q = tid % nq, gi = tid / nq;
        float4 t = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int sp0 = gi; sp0 < nP; sp0 += ER * g) {
          float4 v[ER];
#pragma unroll
          for (int m = 0; m < ER; ++m) {
            const int sp = sp0 + m * g;
            v[m] = sp < nP ? __ldcg(pp + (size_t)sp * q4n + cq0 + q) : make_float4(0.f, 0.f, 0.f, 0.f);
          }
#pragma unroll
          for (int m = 0; m < ER; ++m) t = f4add(t, v[m]);
        }
        S.redE[gi * nq + q] = t;
      }
      csync();
      if (tid < nq) {
        float4 y = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int gi = 0; gi < g; ++gi) y = f4add(y, S.redE[gi * nq + tid]);
        __stcg(x4, f4add(xo, y));
      }
    }
    csync();
    if (tid == 0) tstamp<TR>(P, l, 10, gtime());
    if (l + 1 < P.n_layers) {
      gsync_arrive();  // 4: x complete
      gsync_wait();
    }
    if (tid == 0) tstamp<TR>(P, l, 11, gtime());
  }
}

template <int WT, int ACT, int PT, bool TR>
__global__ void __launch_bounds__(NTHR, 1) k_stack1(const __grid_constant__ StackParams P) {
  extern __shared__ __align__(128) unsigned char smem[];
  const Smem S = carve(smem, P.pl);
  if (threadIdx.x == 0) {
    for (int i = 0; i < P.pl.ns; ++i) {
      mbar_init(&S.full[i], 1u);
      mbar_init(&S.empty[i], (uint32_t)NCW);
    }
    mbar_init(S.listbar, 1u);
    mbar_init(S.listdone, 1u);
    *S.abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  for (int i = threadIdx.x; i < P.pl.maxi; i += NTHR) S.flag[i] = 0;
  for (int i = threadIdx.x; i < HQ; i += NTHR) S.hflag[i] = 0;
  {
    // the CTA's hot items: groups g = s, s + SMs, ... of hp adjacent neurons
    const Ranges R = ranges(P.pl);
    for (int i = threadIdx.x; i < R.nh; i += NTHR)
      S.items[i] = hot_group_first(i / P.pl.hp, P.pl) + i % P.pl.hp;
  }
  __syncthreads();
  if (threadIdx.x >= NCT) {
    const int p = (threadIdx.x - NCT) >> 5;
    if (p < P.pl.np) {
      if ((threadIdx.x & 31) == 0) producer<WT, ACT, PT, TR>(P, S, p);
    } else if (p == NPMAX) {
      list_writer<WT, ACT, PT, TR>(P, S);
    }
    return;
  }
  consumers<WT, ACT, PT, TR>(P, S);
}

// ------------------------------------------------------------------- host

int smem_optin() {
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  if (!cache[dev]) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess) v = 0;
    cache[dev] = v;
  }
  return cache[dev];
}

uint32_t up16(uint32_t v) { return (v + 15u) & ~15u; }
uint32_t up128(uint32_t v) { return (v + 127u) & ~127u; }

// Layout flags of the layers' weights (all layers must agree): whether a
// row's Q4_0 scales sit right behind its codes ("contig"), and whether whole
// records are contiguous at their own size, so adjacent neurons are one copy
// ("packed").  First records: [codes | scales] of W_gate (ReGLU) / W_up
// (ReLU).  D records: ReGLU [W_up codes | scales | W_down^T codes | scales],
// ReLU [W_down^T codes | scales].
void packing(const pi_layer* layers, int n, uint32_t rowb, uint32_t scb, Plan* pl) {
  pl->first_packed = pl->d2_packed = pl->first_contig = pl->second_contig = pl->down_contig = 1;
  const uintptr_t rec = (uintptr_t)rowb + scb;
  for (int l = 0; l < n; ++l) {
    const pi_layer& L = layers[l];
    const bool two = L.act == PI_REGLU, q4 = L.w_dtype == PI_Q4_0;
    const uintptr_t first = (uintptr_t)(two ? L.w_gate : L.w_up);
    const uintptr_t first_s = (uintptr_t)(two ? L.w_gate_scales : L.w_up_scales);
    const int64_t up_rs = two && L.w_up_row_stride ? L.w_up_row_stride : L.w_row_stride;
    if (q4 && first_s != first + rowb) pl->first_contig = 0;
    if (q4 && two && (uintptr_t)L.w_up_scales != (uintptr_t)L.w_up + rowb) pl->second_contig = 0;
    if (q4 && (uintptr_t)L.w_down_t_scales != (uintptr_t)L.w_down_t + rowb) pl->down_contig = 0;
    if (!(pl->first_contig && code_stride(L.w_dtype, L.d_model, L.w_row_stride) == (int64_t)rec))
      pl->first_packed = 0;
    bool dk;
    if (two)
      dk = pl->second_contig && pl->down_contig &&
           (uintptr_t)L.w_down_t == (uintptr_t)L.w_up + rec &&
           code_stride(L.w_dtype, L.d_model, up_rs) == 2 * (int64_t)rec &&
           code_stride(L.w_dtype, L.d_model, L.w_down_row_stride) == 2 * (int64_t)rec;
    else
      dk = pl->down_contig &&
           code_stride(L.w_dtype, L.d_model, L.w_down_row_stride) == (int64_t)rec;
    if (!dk) pl->d2_packed = 0;
  }
}

bool make_plan(const pi_layer* layers, int n_layers, int nsms, Plan* out) {
  const pi_layer& L0 = layers[0];
  Plan pl{};
  pl.d = L0.d_model;
  pl.F = L0.d_ff;
  pl.r = L0.rank;
  pl.H = L0.hot;
  pl.nsms = nsms;
  pl.sq = L0.act == PI_RELU2;
  const int d = pl.d, F = pl.F, r = pl.r, H = pl.H;
  const bool q4 = L0.w_dtype == PI_Q4_0, two = L0.act == PI_REGLU;
  const uint32_t pb = L0.p_dtype == PI_F32 ? 4u : 2u;
  pl.rowb = (uint32_t)row_bytes(L0.w_dtype, d);
  pl.scb = q4 ? (uint32_t)(d / 32) * 2u : 0u;
  pl.p1_bytes = (uint32_t)d * pb;
  pl.p2_row = (uint32_t)r * pb;
  const uint32_t rec = pl.rowb + pl.scb;
  if (rec % 16 || pl.rowb % 16 || pl.scb % 16) return false;  // 16-byte bulk copies
  pl.first_b = rec;
  pl.o_d2_down = two ? rec : 0u;
  pl.d2_bytes = two ? 2u * rec : rec;
  packing(layers, n_layers, pl.rowb, pl.scb, &pl);
  const int64_t up_rs = L0.w_up_row_stride ? L0.w_up_row_stride : L0.w_row_stride;
  pl.first_stride = code_stride(L0.w_dtype, d, L0.w_row_stride);
  pl.first_sstride = scale_stride(d, L0.w_row_stride);
  pl.second_stride = code_stride(L0.w_dtype, d, up_rs);
  pl.second_sstride = scale_stride(d, up_rs);
  pl.down_stride = code_stride(L0.w_dtype, d, L0.w_down_row_stride);
  pl.down_sstride = scale_stride(d, L0.w_down_row_stride);
  for (int l = 1; l < n_layers; ++l)
    if (layers[l].w_row_stride != L0.w_row_stride || layers[l].w_down_row_stride != L0.w_down_row_stride ||
        layers[l].w_up_row_stride != L0.w_up_row_stride)
      return false;
  // first records per hot unit (adjacent neurons): units of at least 16 KB,
  // at most kMaxRec records
  pl.hp = 1;
  while (pl.hp < kMaxRec && (uint32_t)pl.hp * rec < 16384u) ++pl.hp;
  pl.cp = pl.hp;
  uint32_t sb = pl.p1_bytes;
  sb = sb > (uint32_t)pl.hp * rec ? sb : (uint32_t)pl.hp * rec;
  sb = sb > pl.d2_bytes ? sb : pl.d2_bytes;
  sb = sb > pl.p2_row ? sb : pl.p2_row;
  sb = up128(sb);
  pl.sb = sb;
  pl.dr = (int)(sb / pl.d2_bytes);
  const int drmax = two ? DR2MAX : DRMAX;
  if (pl.dr > drmax) pl.dr = drmax;
  if (pl.dr < 1) pl.dr = 1;
  int G = 32;
  while (G > 1 && (uint32_t)G * pl.p2_row > sb) G >>= 1;
  pl.G = G;
  const int W = (F + 31) / 32, Wlo = H / 32, Wc = W - Wlo;
  // a CTA's cold neurons come from its own share of the mask words (one
  // warp lane per word): up to 32 per word
  const int wpc = (Wc + nsms - 1) / nsms;  // mask words per CTA at most
  if (wpc > 32) return false;
  pl.maxc = 32 * wpc;
  pl.maxi = (H + nsms - 1) / nsms + pl.hp + pl.maxc + 1;
  const int bw = wpc + 2;
  uint32_t o = 8 * (2 * NSMAX + 2);  // mbarriers
  o = up16(o);
  pl.o_misc = o;       o = up16(o + 16);
  pl.o_xf = o;         o = up16(o + 4u * d);
  pl.o_xi = o;         o = up16(o + (q4 ? 2u * d : 0u));
  pl.o_bsum = o;       o = up16(o + (q4 ? 4u * (d / 32) : 0u));
  pl.o_u = o;          o = up16(o + 4u * r);
  pl.o_bw = o;         o = up16(o + 4u * bw);
  pl.o_scan = o;       o = up16(o + 4u * (NCW + 4));
  pl.o_items = o;      o = up16(o + 4u * pl.maxi);
  pl.o_hval = o;       o = up16(o + 4u * pl.maxi);
  pl.o_flag = o;       o = up16(o + 4u * pl.maxi);
  pl.o_dlist = o;      o = up16(o + 4u * pl.maxi);
  pl.o_pbs = o;        o = up16(o + 4u * 32u * bw);
  pl.o_hbs = o;        o = up16(o + 4u * pl.maxi);
  pl.o_redA = o;       o = up16(o + 4u * (MAXA + MAXA * NCW));
  pl.o_redC = o;       o = up16(o + 4u * (2 * 8 * NCW));
  pl.o_redD = o;       o = up16(o + 4u * (2 * DR2MAX * NCW));
  pl.o_hflag = o;      o = up16(o + 4u * HQ);
  pl.o_redE = o;       o = up16(o + 16u * NCT);
  pl.o_ring = up128(o);
  const int avail = smem_optin() - (int)pl.o_ring;
  if (avail <= 0) return false;
  int ns = avail / (int)sb;
  if (ns > NSMAX) ns = NSMAX;
  if (ns < 3) return false;
  // an even ring (a multiple of 4 when deep) lets the consumer groups divide it
  if (ns >= 8) ns -= ns % 4;
  else if (ns >= 4) ns -= ns % 2;
  pl.ns = ns;
  pl.np = NPMAX;  // producer warp p owns the stages st with st % NPMAX == p
  // consumer groups must divide the ring depth (a stage is always consumed
  // by the same group); the down phase also needs every column to fit one
  // group's accumulators (64 floats per thread)
  pl.gw = ns % 4 == 0 ? 4 : (ns % 2 == 0 ? 2 : 1);
  {
    // chunks per consumer thread in the down phase must fit its accumulators
    // (one Q4_0 block, or 48 fp16 / fp32 values)
    const int cc = L0.w_dtype == PI_Q4_0 ? 32 : (L0.w_dtype == PI_F16 ? 8 : 4);
    const int cap = cc == 32 ? kQ4Blocks : (two ? 32 : 48) / cc;
    const int per2 = (d / cc + NCT / 2 - 1) / (NCT / 2);
    const int per1 = (d / cc + NCT - 1) / NCT;
    if (ns % 2 == 0 && per2 <= cap) pl.gd = 2;
    else if (per1 <= cap) pl.gd = 1;
    else return false;
  }
  if (two) {
    // the ReGLU down phase: its up groups alternate units (an even ring keeps
    // each stage with one group) and its down group covers every column
    // with one Q4_0 block or at most 48 fp16 / fp32 values per thread; its
    // up groups reuse the phase-C threads' x^ blocks (four groups in C)
    if (ns % 2 || pl.gw != 4) return false;
    const int cc = L0.w_dtype == PI_Q4_0 ? 32 : (L0.w_dtype == PI_F16 ? 8 : 4);
    const int per = (d / cc + NCT / 2 - 1) / (NCT / 2);
    if (per > (cc == 32 ? 1 : 48 / cc)) return false;
  }
  pl.total = pl.o_ring + (uint32_t)ns * sb;
  *out = pl;
  return true;
}

bool fused_disabled() {
  static int v = -1;
  if (v < 0) {
    const char* e = getenv("PI_DISABLE_FUSED");
    v = (e && e[0] && e[0] != '0') ? 1 : 0;
  }
  return v == 1;
}

template <int WT, int ACT, int PT>
cudaError_t launch_t(const StackParams& P, cudaStream_t s) {
  // the timeline instrumentation lives in its own instantiation, so the
  // kernel that normally runs carries none of it
  auto kern = (P.trace || P.utrace) ? k_stack1<WT, ACT, PT, true> : k_stack1<WT, ACT, PT, false>;
  cudaError_t e = allow_smem_fn(reinterpret_cast<const void*>(kern), P.pl.total);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(P.pl.nsms);
  cfg.blockDim = dim3(NTHR);
  cfg.dynamicSmemBytes = P.pl.total;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, P);
}

cudaError_t launch_any(const StackParams& P, int wt, int act, int pt, cudaStream_t s) {
  // weight / predictor dtype pairs that share one staged-vector layout
  if (wt == PI_Q4_0) {
    if (act == PI_REGLU)
      return pt == PI_F32 ? launch_t<PI_Q4_0, PI_REGLU, PI_F32>(P, s)
                          : launch_t<PI_Q4_0, PI_REGLU, PI_F16>(P, s);
    return pt == PI_F32 ? launch_t<PI_Q4_0, PI_RELU, PI_F32>(P, s)
                        : launch_t<PI_Q4_0, PI_RELU, PI_F16>(P, s);
  }
  if (wt == PI_F16)
    return act == PI_REGLU ? launch_t<PI_F16, PI_REGLU, PI_F16>(P, s)
                           : launch_t<PI_F16, PI_RELU, PI_F16>(P, s);
  return act == PI_REGLU ? launch_t<PI_F32, PI_REGLU, PI_F32>(P, s)
                         : launch_t<PI_F32, PI_RELU, PI_F32>(P, s);
}

// One CTA, one thread: the kernel's own bounded waits on state nothing
// completes (kind 0: an mbarrier phase with no arrival; kind 1: a grid
// barrier target no CTA reaches), ended by `limit_ns`.
__global__ void k_wait_selftest(WsHeader* hdr, int kind, unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  Smem S{};
  S.abort = &abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1u);
    abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    if (kind == 0)
      (void)wait_mbar(&bar, 0u, S, hdr, limit_ns);
    else
      (void)grid_wait(hdr, 0xFFFFFFFFu, S, limit_ns);
  }
}

}  // namespace

cudaError_t launch_wait_selftest(void* ws, int kind, unsigned long long limit_ns, cudaStream_t s) {
  WsHeader* hdr = reinterpret_cast<WsHeader*>(ws);
  cudaError_t e = cudaMemsetAsync(hdr->counters, 0, 2 * sizeof(uint32_t), s);
  if (e != cudaSuccess) return e;
  k_wait_selftest<<<1, 32, 0, s>>>(hdr, kind, limit_ns);
  return cudaGetLastError();
}

int stack1_chunk() { return MAXL; }
int stack1_unit_trace_len() { return UTR; }

bool stack1_supported(const pi_layer* layers, int n_layers, int batch) {
  if (batch != 1 || n_layers < 1 || fused_disabled()) return false;
  // rows in a host-memory cold tier are read by the CUDA-core kernels only
  for (int l = 0; l < n_layers; ++l)
    if (layers[l].w_up_cold) return false;
  const pi_layer& a = layers[0];
  for (int l = 1; l < n_layers; ++l) {
    const pi_layer& b = layers[l];
    if (b.d_model != a.d_model || b.d_ff != a.d_ff || b.rank != a.rank || b.hot != a.hot ||
        b.act != a.act || b.w_dtype != a.w_dtype || b.p_dtype != a.p_dtype)
      return false;
  }
  // fp16 weights go with an fp16 predictor, fp32 with fp32 (one staged layout)
  if ((a.w_dtype == PI_F16 && a.p_dtype != PI_F16) || (a.w_dtype == PI_F32 && a.p_dtype != PI_F32))
    return false;
  // the predictor's u and (Q4_0) x^ stay in consumer registers
  if (a.d_model > 12288 || a.rank > (a.p_dtype == PI_F16 ? 1024 : 512)) return false;
  if (a.w_dtype == PI_Q4_0 && a.d_model > 8192) return false;
  if (a.w_dtype == PI_Q4_0) {
    if (a.d_model % 256) return false;
    for (int l = 0; l < n_layers; ++l) {
      const pi_layer& b = layers[l];
      if (((uintptr_t)b.w_up_scales | (uintptr_t)b.w_down_t_scales |
           (uintptr_t)(b.act == PI_REGLU ? b.w_gate_scales : b.w_up_scales)) & 15u)
        return false;
    }
  }
  const int nsms = device_sms();
  if (nsms < 128) return false;                                // slice bounds below
  if ((a.d_model / 4 + nsms - 1) / nsms > 32) return false;    // reduce slice <= 32 float4
  if ((a.rank + nsms - 1) / nsms > MAXA) return false;         // P1 rows per CTA
  Plan pl;
  return make_plan(layers, n_layers, nsms, &pl);
}

cudaError_t launch_stack1(const pi_layer* layers, int n_layers, float* x, uint32_t* mask_trace,
                          void* ws, const WsLayout& lay, float theta, cudaStream_t s,
                          unsigned long long* trace, unsigned long long* utrace) {
  const int nsms = device_sms();
  if (n_layers < 1 || n_layers > MAXL) return cudaErrorInvalidValue;
  StackParams P;
  memset(&P, 0, sizeof P);
  if (!make_plan(layers, n_layers, nsms, &P.pl)) return cudaErrorInvalidConfiguration;
  const pi_layer& a = layers[0];
  const int words = (a.d_ff + 31) / 32;
  WsHeader* hdr = reinterpret_cast<WsHeader*>(ws);
  P.theta = theta;
  P.x = x;
  P.u = reinterpret_cast<float*>((char*)ws + lay.u);
  P.part = reinterpret_cast<float*>((char*)ws + lay.part);
  P.count = reinterpret_cast<int32_t*>((char*)ws + lay.count);
  P.idx = reinterpret_cast<int32_t*>((char*)ws + lay.idx);
  P.cta_counts = reinterpret_cast<uint32_t*>((char*)ws + lay.cta);
  P.hdr = hdr;
  P.trace = trace;
  P.utrace = utrace;
  P.n_layers = n_layers;
  P.mask_words = words;
  if (mask_trace) {
    P.mask = mask_trace;
    P.mask_stride = words;
  } else {
    P.mask = reinterpret_cast<uint32_t*>((char*)ws + lay.mask);
    P.mask_stride = 0;
  }
  for (int i = 0; i < n_layers; ++i) {
    const pi_layer& L = layers[i];
    const bool two = L.act == PI_REGLU;
    LayerPtrs& p = P.L[i];
    p.first = (const char*)(two ? L.w_gate : L.w_up);
    p.first_scales = (const char*)(two ? L.w_gate_scales : L.w_up_scales);
    p.second = (const char*)(two ? L.w_up : nullptr);
    p.second_scales = (const char*)(two ? L.w_up_scales : nullptr);
    p.down = (const char*)L.w_down_t;
    p.down_scales = (const char*)L.w_down_t_scales;
    p.bias = L.bias;
    p.p1 = (const char*)L.p1;
    p.p2 = (const char*)L.p2;
    p.pbias = L.p_bias;
  }
  cudaError_t e = cudaMemsetAsync(hdr->counters, 0, 2 * sizeof(uint32_t), s);
  if (e == cudaSuccess) e = cudaMemsetAsync(P.cta_counts, 0, sizeof(uint32_t) * (size_t)nsms, s);
  if (e != cudaSuccess) return e;
  return launch_any(P, a.w_dtype, a.act, a.p_dtype, s);
}

}  // namespace pi
