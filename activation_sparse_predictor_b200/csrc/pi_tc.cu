// The FFN of a layer at token batches on the tensor cores (sm_100a).
//
// At 2-64 tokens the listed rows (the hot prefix [0, hot), then the cold
// list idx) of every token batch form real contractions, both run as tcgen05
// GEMMs over list positions p (row(p) = p for p < hot, idx[p - hot] after):
//
//   up   : D[p][t] = sum_k W[row(p)][k] xh[t][k] for 128 list positions per
//          tile (the MMA's A operand, K-major) and all tokens t (B: an fp16
//          copy of the normalised inputs, tokens padded to 16, shared with
//          the predictor); the tiles that hold list positions, and the
//          share of d each CTA takes, are sized on the device from the list
//          length so that the CTAs fill the SMs; a second
//          kernel sums the splits in a fixed
//          order, adds the bias, applies ReLU / ReGLU and the per-token bits
//          and writes an fp16 copy h16 of h, tile-major: the 64 positions
//          of k tile kt for token t at h16[(kt * nt + t) * 64 ..];
//   down : D[c][t] = sum_p W_down^T[row(p)][c] h[t][p] for 128 output
//          columns per tile; W_down^T (columns contiguous) is an MN-major A
//          operand; the k tiles that hold list positions split evenly over
//          up to 8 CTAs; the partial rows go to the fixed-order split-K
//          reduction.
//
// The predictor at token batches is two more contractions: u = P1 xh and
// z = P2[H:] u.  Their results decide mask bits, so the fp32 vector operand
// is split into two fp16 parts (hi + lo, ~22 bits) and both products
// accumulate into the same fp32 accumulator; z's epilogue adds the bias,
// compares with logit(tau) and turns each warp's 32 consecutive rows into
// one mask word per token with a ballot.
//
// A tile whose rows all lie in the hot prefix is one TMA box per operand
// and stage; any other tile is gathered with TMA tile::gather4 loads (four
// rows, a one-row-high box).  A gather costs its issuing lane a while, so
// the FFN kernels run 8 warps: warp 1 issues the MMAs, the other seven deal
// out a stage's gathers round-robin and each arms its own bytes on the
// stage's mbarrier; warps 0-3 then drain the accumulators.  Two CTAs
// (about 100 KB of shared memory each) fit per SM, and the K splits are
// sized to fill them.  128-byte swizzle throughout, a 4-stage ring for the
// FFN (2 for the ReGLU up kernel, whose stage carries two operands) and a
// 3-stage one for the predictor, fp32 accumulators in tensor
// memory, one thread issuing the MMAs.  Every
// mbarrier wait is bounded by %globaltimer (1 s): a wait that runs out sets
// DEV_TIMEOUT in the workspace status word and a CTA abort flag; the
// producer waits (bounded) for its copies in flight and the tensor memory
// is always freed after the MMAs have completed.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_fp16.h>

#include <algorithm>
#include <cstdlib>
#include <mutex>

#include "pi_kernels.cuh"
#include "pi_tc.cuh"

namespace pi {
namespace {

constexpr int TC_M = 128;        // list positions (up) / output columns (down) per tile
constexpr int TC_BK = 64;        // k per stage: one 128-byte swizzle atom of fp16
constexpr int TC_STAGES = 4;
constexpr int TC_THREADS = 128;
constexpr int TC_FFN_WARPS = 8;  // warps of the FFN kernels: warp 1 issues the MMAs, the rest
constexpr int TC_PW = TC_FFN_WARPS - 1;  // load (warps 0-3 also drain the accumulators)
constexpr int TC_KSMAX_D = 8;    // CTAs sharing one down tile's list positions at most
constexpr int TC_TMAX = 64;      // tokens at most (MMA N)
// Tokens at least: from two tokens on, one pass over the listed rows on the
// tensor cores (the token tile padded to 16 with zero rows) costs less than
// the CUDA-core kernels' passes; one token takes the CUDA-core kernels.
constexpr int TC_MIN_BATCH = 2;
constexpr unsigned long long kTcTimeoutNs = 1000000000ull;

__device__ __forceinline__ uint32_t tc_sa(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ uint64_t tc_time() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ bool tc_try(uint64_t* b, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(tc_sa(b)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait for phase `parity` of `bar`; false after an abort or a
// timeout (which raises the abort and the status bit).
__device__ bool tc_wait(uint64_t* bar, uint32_t parity, volatile int* abort, WsHeader* hdr) {
  if (tc_try(bar, parity)) return true;
  const uint64_t t0 = tc_time();
  while (!tc_try(bar, parity)) {
    if (*abort) return false;
    if (tc_time() - t0 > kTcTimeoutNs) {
      *abort = 1;
      if (hdr) atomicOr(&hdr->status, DEV_TIMEOUT);
      return false;
    }
  }
  return true;
}

// try_wait with a suspend-time hint: the thread may sleep in hardware
// until the phase completes (or the hint elapses) instead of spinning.
__device__ __forceinline__ bool tc_try_sleep(uint64_t* b, uint32_t parity, uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(tc_sa(b)), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}

// Bounded wait that ignores the abort flag (used before freeing resources,
// and by warps with nothing else to do until a kernel's products are
// final): it sleeps between tries, so waiting warps take no issue slots
// from the working ones.
__device__ bool tc_wait_quiet(uint64_t* bar, uint32_t parity, WsHeader* hdr) {
  if (tc_try(bar, parity)) return true;
  const uint64_t t0 = tc_time();
  while (!tc_try_sleep(bar, parity, 100000u)) {
    if (tc_time() - t0 > kTcTimeoutNs) {
      if (hdr) atomicOr(&hdr->status, DEV_TIMEOUT);
      return false;
    }
  }
  return true;
}

// Shared-memory matrix descriptor of a K-major tile with 128-byte swizzle:
// rows of 128 bytes, 8-row atoms 1024 bytes apart (stride byte offset),
// leading byte offset unused (1), descriptor version 1, layout 2 (128B).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)1 << 16) |
         ((uint64_t)(1024u >> 4) << 32) | ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// Descriptor of an MN-major tile with 128-byte swizzle: 8 K-rows of 128
// bytes (64 MN elements) per 1024-byte atom, K atoms 1024 bytes apart
// (stride byte offset), MN atoms `mn_stride` bytes apart (leading byte offset).
__device__ __forceinline__ uint64_t sw128_mn_desc(uint32_t saddr, uint32_t mn_stride) {
  return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)((mn_stride >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)(1024u >> 4) << 32) | ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// D (tensor memory) [+]= A * B^T for one K = 16 slice, issued by one thread.
__device__ __forceinline__ void mma_f16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                        uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n}\n" ::"r"(
          tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(0), "r"(0), "r"(0), "r"(0));
}

// Arrives on `bar` once every tcgen05.mma this thread issued has completed.
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   tc_sa(bar))
               : "memory");
}

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, "
      "%3}], [%4];" ::"r"(tc_sa(dst)),
      "l"(map), "r"(x), "r"(y), "r"(tc_sa(bar))
      : "memory");
}

// Four rows y0..y3 (columns x .. x+63) of a map whose box is one row high,
// to 4 consecutive 128-byte rows at dst.
__device__ __forceinline__ void tma_gather4(void* dst, const CUtensorMap* map, int x, int y0,
                                            int y1, int y2, int y3, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile::gather4.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4, %5, %6}], [%7];" ::"r"(tc_sa(dst)),
      "l"(map), "r"(x), "r"(y0), "r"(y1), "r"(y2), "r"(y3), "r"(tc_sa(bar))
      : "memory");
}

__device__ __forceinline__ void tc_init(uint64_t* full, uint64_t* empty, uint64_t* done,
                                        volatile int* abort, int stages = TC_STAGES,
                                        uint32_t full_arrivals = 1u) {
  for (int i = 0; i < stages; ++i) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(tc_sa(&full[i])), "r"(full_arrivals)
                 : "memory");
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(tc_sa(&empty[i])) : "memory");
  }
  asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(tc_sa(done)) : "memory");
  *abort = 0;
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void tmem_alloc(uint32_t* slot, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(tc_sa(slot)),
               "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

// 16 consecutive accumulator columns of this warp's 32 lanes.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
      "%12, %13, %14, %15}, [%16];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
        "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]),
        "=r"(v[14]), "=r"(v[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// List length hot + count with count clamped to [0, F - hot].
__device__ __forceinline__ int list_len(const int32_t* count, int H, int F, WsHeader* hdr) {
  int c = *count;
  if (c < 0 || c > F - H) {
    if (hdr && blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0)
      atomicOr(&hdr->status, DEV_BAD_COUNT);
    c = c < 0 ? 0 : F - H;
  }
  return H + c;
}

// Weight row of list position p (a valid row for every p: positions beyond
// the list and bad indices read row 0; their h is 0).
__device__ __forceinline__ int list_row(int p, int H, int N, int F, const int32_t* idx) {
  if (p < H) return p;
  if (p >= N) return 0;
  const int j = idx[p - H];
  return (j >= H && j < F) ? j : 0;
}

// Ring stages of the up kernel by operand count and token tile, as many as
// keep two CTAs (under 113 KB of shared memory each) on an SM: a stage is
// NR 16 KB weight tiles and the activation tile (nt x 128 bytes, rounded to
// the 1 KB swizzle atom).
__host__ __device__ constexpr int up_stages(int nr, int nt) {
  return nr == 1 ? (nt <= 32 ? 5 : 4) : (nt <= 32 ? 3 : 2);
}

// Work of the up kernel for a list of N positions: nT = ceil(N / 128) row
// tiles, each split over ks shares of d (nk k tiles) so that nT * ks CTAs
// fill the g CTA slots of the grid.  A split costs a 32 KB fp32 partial
// tile per operand, written here and read back by the finish kernel, about
// 4 ks / nk of the tile's weight bytes; ks <= nk / 32 keeps that near 1/8.
// Partial sums are laid out [ks][NR][nT * 128][nt].  The same function
// sizes the work on both sides of the finish kernel.
//
// fit (the Q4_0 kernel, bound by its loaders rather than by HBM, two CTAs
// per SM): g is the number of resident CTA slots and ks the split, up to
// the cap, that fills the last wave of nT * ks CTAs best (the largest
// split within 2 % of the best fill: more, shorter CTAs balance the SMs
// better), so that few SMs run one CTA while others run two.  (Llama2-70B
// shape, tokens/s: 8 tokens 402 -> 472, 16 tokens 578 -> 759, 64 tokens
// 1892 -> 2167 against ks = g / nT.)
struct UpShare {
  int nT, ks;
};
__host__ __device__ inline UpShare up_share(int N, int g, int nk, bool fit = false) {
  UpShare u;
  u.nT = (N + TC_M - 1) / TC_M;
  const int cap = nk / 32 > 1 ? nk / 32 : 1;
  if (fit && u.nT > 0) {
    auto fill = [&](int k) {
      const int c = u.nT * k, w = (c + g - 1) / g;
      return (float)c / (float)(w * g);
    };
    float be = 0.f;
    for (int k = 1; k <= cap; ++k) be = fmaxf(be, fill(k));
    u.ks = 1;
    for (int k = cap; k >= 1; --k)
      if (fill(k) >= be - 0.02f) {
        u.ks = k;
        break;
      }
    return u;
  }
  int ks = u.nT > 0 ? g / u.nT : 1;
  u.ks = ks < 1 ? 1 : (ks > cap ? cap : ks);
  return u;
}

// up: NR = 1 ReLU (W_up), NR = 2 ReGLU (W_gate, W_up).  One-dimensional
// grid of at least g CTAs; CTA b takes tile b / ks, share b % ks of
// up_share(N, g, nk) and exits past nT * ks.  part: [ks][NR][nT * 128][nt] fp32.
template <int NR, int NS>
__global__ void __launch_bounds__(32 * TC_FFN_WARPS, 1)
    k_ffn_up_tc(const __grid_constant__ CUtensorMap mw0, const __grid_constant__ CUtensorMap mw1,
                const __grid_constant__ CUtensorMap mg0, const __grid_constant__ CUtensorMap mg1,
                const __grid_constant__ CUtensorMap mx, int nt, int nk, int g, int H, int F,
                const int32_t* __restrict__ idx, const int32_t* __restrict__ count,
                float* __restrict__ part, WsHeader* hdr, const float* __restrict__ bias,
                const uint32_t* __restrict__ mask, int words, __half* __restrict__ h16,
                int batch, int sq) {
  pdl_wait();
  pdl_trigger();
  constexpr uint32_t A_BYTES = TC_M * TC_BK * 2;     // 16 KB
  const uint32_t STAGE = NR * A_BYTES + (((uint32_t)nt * TC_BK * 2 + 1023u) & ~1023u);
  constexpr uint32_t NCOLS = NR == 1 ? 64u : 128u;   // >= NR * nt, a power of two
  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw = tc_sa(smem_raw);
  unsigned char* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);  // swizzle atoms: 1 KB aligned
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + NS * STAGE);
  uint64_t* empty = full + NS;
  uint64_t* done = empty + NS;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort = reinterpret_cast<volatile int*>(tslot + 1);
  int* rows = reinterpret_cast<int*>(tslot + 4);  // [128], 16-byte aligned

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int N = list_len(count, H, F, hdr);
  const UpShare us = up_share(N, g, nk);
  const int ks = us.ks, Np = us.nT * TC_M;
  if ((int)blockIdx.x >= us.nT * ks) return;  // no share of the list for this CTA
  const int tile = blockIdx.x / ks, split = blockIdx.x % ks;
  const int p0 = tile * TC_M;
  const bool dense = p0 + TC_M <= H;
  const int kt0 = (int)((long long)split * nk / ks), kt1 = (int)((long long)(split + 1) * nk / ks);
  const int nkt = kt1 - kt0;

  if (threadIdx.x < TC_M) rows[threadIdx.x] = list_row(p0 + threadIdx.x, H, N, F, idx);
  if (threadIdx.x == 0) tc_init(full, empty, done, abort, NS, (uint32_t)TC_PW);
  if (warp == 0) tmem_alloc(tslot, NCOLS);
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem = *tslot;

  if (warp != 1) {
    // TC_PW producer warps, each arming its own bytes on the stage's full
    // barrier (TC_PW arrivals per phase).  A dense tile is one TMA box per
    // operand (warp 0).  A gathered tile's NR * 32 four-row gathers (rows
    // 4g .. 4g+3 of operand o / 32, g = o % 32) are dealt out round-robin,
    // gather o = TC_PW * lane + pw, so a stage issues from every producer warp.
    const int pw = warp == 0 ? 0 : warp - 1;
    const int o = TC_PW * lane + pw;
    const int opnd = o >> 5, g = o & 31;
    const bool gl = !dense && o < NR * 32;
    const int r = 4 * g;
    const int y0 = rows[r], y1 = rows[r + 1], y2 = rows[r + 2], y3 = rows[r + 3];
    const uint32_t bx = (uint32_t)nt * TC_BK * 2;  // the activation tile
    const uint32_t mine = (uint32_t)((NR * 32 - pw + TC_PW - 1) / TC_PW);  // gathers of this warp
    const uint32_t tx = dense ? (pw == 0 ? NR * A_BYTES + bx : 0u) : 512u * mine + (pw == 0 ? bx : 0u);
    int last[NS];
    for (int i = 0; i < NS; ++i) last[i] = -1;
    for (int i = 0; i < nkt; ++i) {
      const int st = i % NS;
      int ok = 1;
      if (lane == 0 && i >= NS) ok = tc_wait(&empty[st], ((i / NS) - 1) & 1, abort, hdr);
      if (!__shfl_sync(0xffffffffu, ok, 0)) break;
      unsigned char* a = smem + st * STAGE;
      if (lane == 0)
        asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(tc_sa(&full[st])),
                     "r"(tx)
                     : "memory");
      __syncwarp();
      const int k = (kt0 + i) * TC_BK;
      if (dense) {
        if (pw == 0 && lane == 0) {
          tma_load_2d(a, &mw0, k, p0, &full[st]);
          if constexpr (NR == 2) tma_load_2d(a + A_BYTES, &mw1, k, p0, &full[st]);
        }
      } else if (gl) {
        tma_gather4(a + opnd * A_BYTES + 512u * g, opnd == 0 ? &mg0 : &mg1, k, y0, y1, y2, y3,
                    &full[st]);
      }
      if (pw == 0 && lane == 0) tma_load_2d(a + NR * A_BYTES, &mx, k, 0, &full[st]);
      if (lane == 0) last[st] = i;
    }
    if (lane == 0) {  // every copy of this CTA has landed before it may exit (bounded)
      for (int st = 0; st < NS; ++st)
        if (last[st] >= 0) (void)tc_wait_quiet(&full[st], (uint32_t)(last[st] / NS) & 1u, hdr);
    }
  } else if (warp == 1 && lane == 0) {
    // MMA issuer: kind::f16, fp16 A and B, fp32 D, both K-major, M = 128, N = nt
    const uint32_t idesc = (1u << 4) | ((uint32_t)(nt >> 3) << 17) | ((uint32_t)(TC_M >> 4) << 24);
    for (int i = 0; i < nkt; ++i) {
      const int st = i % NS;
      if (!tc_wait(&full[st], (uint32_t)(i / NS) & 1u, abort, hdr)) break;
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      const uint32_t a = tc_sa(smem + st * STAGE), b = a + NR * A_BYTES;
#pragma unroll
      for (int kk = 0; kk < TC_BK / 16; ++kk) {  // 32 bytes of K per MMA inside the atom
        const uint64_t bd = sw128_desc(b + 32u * kk);
        const uint32_t acc = (i | kk) != 0 ? 1u : 0u;
        mma_f16(tmem, sw128_desc(a + 32u * kk), bd, idesc, acc);
        if constexpr (NR == 2)
          mma_f16(tmem + (uint32_t)nt, sw128_desc(a + A_BYTES + 32u * kk), bd, idesc, acc);
      }
      mma_commit(&empty[st]);  // the stage is free once these products have read it
    }
    mma_commit(done);  // the accumulators are final (after an abort: quiescent)
  }
  __syncwarp();

  // epilogue: warp w holds accumulator lanes [32w, 32w + 32) = list
  // positions p0 + 32w + lane, one column per token.  `done` is awaited even
  // after an abort, so no product still writes tensor memory when it is freed.
  bool ok = tc_wait_quiet(done, 0u, hdr);
  ok = __all_sync(0xffffffffu, ok && !*abort && nkt > 0);
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  if (ok && warp < 4 && ks == 1) {
    // one share of d per row tile: the accumulators are the pre-activations,
    // so the activation is applied here, with the arithmetic of k_ffn_finish
    // for one split (which then skips this layer), and h16 written directly
    const int p = p0 + warp * 32 + lane;
    int j = 0;
    bool valid = false;
    float bb = 0.f;
    if (p < N) {
      j = p < H ? p : idx[p - H];
      if (p >= H && (j < H || j >= F)) {
        if (hdr) atomicOr(&hdr->status, DEV_BAD_INDEX);
      } else {
        valid = true;
        bb = bias ? bias[j] : 0.f;
      }
    }
    __half* hrow = h16 + (size_t)(p / 64) * nt * 64 + (p % 64);
    for (int c0 = 0; c0 < nt; c0 += 16) {
      uint32_t gv16[16], uv16[16];
      tmem_ld16(tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)c0, gv16);
      if constexpr (NR == 2) tmem_ld16(tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)(nt + c0), uv16);
#pragma unroll
      for (int q = 0; q < 16; ++q) {
        const int b = c0 + q;
        float hv = 0.f;
        if (valid && b < batch) {
          const float gv = (0.f + __uint_as_float(gv16[q])) + bb;
          hv = gv > 0.f ? gv : 0.f;
          if constexpr (NR == 2) hv *= 0.f + __uint_as_float(uv16[q]);
          else if (sq) hv *= hv;  // squared ReLU
          if (mask && p >= H && !((__ldg(mask + (size_t)b * words + (j >> 5)) >> (j & 31)) & 1u))
            hv = 0.f;
        }
        hrow[(size_t)b * 64] = __float2half_rn(hv);
      }
    }
  } else if (ok && warp < 4) {
    const int p = p0 + warp * 32 + lane;
#pragma unroll
    for (int r = 0; r < NR; ++r) {
      float* dst = part + ((size_t)(split * NR + r) * Np + p) * nt;
      for (int c0 = 0; c0 < nt; c0 += 16) {
        uint32_t v[16];
        tmem_ld16(tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)(r * nt + c0), v);
#pragma unroll
        for (int q = 0; q < 4; ++q)
          __stcg(reinterpret_cast<float4*>(dst + c0) + q,
                 make_float4(__uint_as_float(v[4 * q]), __uint_as_float(v[4 * q + 1]),
                             __uint_as_float(v[4 * q + 2]), __uint_as_float(v[4 * q + 3])));
      }
    }
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  if (warp == 0)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(NCOLS)
                 : "memory");
}

// ------------------------------------------------------------------ Q4_0
// Q4_0 weights on the tensor cores.  The listed rows' codes and scales are
// loaded by 256 threads with vector loads, TC_Q4_PRE stages ahead in
// registers, decoded to fp16 (q - 8) * s and stored into the 128-byte
// swizzled operand tile of the ring; each thread fences its stores for
// the tensor cores' (async) proxy and arrives on the stage's barrier,
// which completes when all 256 have arrived and the activation tile's TMA
// bytes have landed (one arrival per warp after a warp barrier measured
// slower: the warp then waits for its slowest lane).  Warp 8 issues the
// MMAs; warps 8-11 drain the accumulators.
constexpr int TC_Q4_WARPS = 12;
constexpr int TC_Q4_LOADERS = 256;  // threads 0..255 load and decode
constexpr int TC_Q4_PRE = 4;        // stages of codes each loader holds ahead

// Elements 8c .. 8c+7 of a Q4_0 block (16 code bytes: byte k holds element
// k in its low nibble and element k + 16 in its high nibble) as eight fp16
// values (q - 8) * s: c = 0, 1 take the low nibbles of bytes 8c .. 8c+7,
// c = 2, 3 the high nibbles of bytes 8(c-2) ..  A nibble n becomes the
// fp16 number 1024 + n (0x6400 | n) by a byte permute, from which 1032 is
// subtracted exactly; the product with the scale is rounded once.
__device__ __forceinline__ uint4 q4_chunk_f16(uint32_t w0, uint32_t w1, bool high, __half2 s2) {
  if (high) {
    w0 >>= 4;
    w1 >>= 4;
  }
  w0 &= 0x0F0F0F0Fu;
  w1 &= 0x0F0F0F0Fu;
  const uint32_t p[4] = {__byte_perm(w0, 0x64u, 0x4140), __byte_perm(w0, 0x64u, 0x4342),
                         __byte_perm(w1, 0x64u, 0x4140), __byte_perm(w1, 0x64u, 0x4342)};
  const __half2 off = __half2half2(__ushort_as_half((unsigned short)0x6408u));  // 1032
  uint32_t r[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const __half2 v = __hmul2(__hsub2(*reinterpret_cast<const __half2*>(&p[k]), off), s2);
    r[k] = *reinterpret_cast<const uint32_t*>(&v);
  }
  return make_uint4(r[0], r[1], r[2], r[3]);
}

// Read-only loads of Q4_0 codes and scales that ask L2 to fetch the whole
// 256-byte block around them: a row's next stages (and, for the down
// projection, the neighbouring column tiles, which read the same rows at
// the same time) then hit L2, so DRAM sees 256-byte requests instead of
// the 64 bytes one stage takes from a row.
__device__ __forceinline__ uint4 ld_q4_codes(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.L2::256B.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}
__device__ __forceinline__ uint32_t ld_q4_scales2(const void* p) {
  uint32_t v;
  asm volatile("ld.global.nc.L2::256B.u32 %0, [%1];" : "=r"(v) : "l"(p));
  return v;
}
__device__ __forceinline__ uint16_t ld_q4_scale(const void* p) {
  uint16_t v;
  asm volatile("ld.global.nc.L2::256B.u16 %0, [%1];" : "=h"(v) : "l"(p));
  return v;
}

__device__ __forceinline__ void sts128(uint32_t addr, uint4 v) {
  asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z),
               "r"(v.w)
               : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;" ::"r"(tc_sa(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive_release(uint64_t* bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(tc_sa(bar)) : "memory");
}

__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Q4_0 up/gate: as k_ffn_up_tc (grid, work shares, part layout), with
// K = 64 KB per stage (KB 64-column atoms) and NS = 2 ring stages, two CTAs
// per SM (a separate, deeper ring for the activation tiles, loaded ahead
// by an idle warp, measured slower).  Loader thread t
// decodes blocks KB h .. KB h + KB - 1 of the stage in row t / 2 (h = t %
// 2) of each operand: 16 KB contiguous code bytes and KB scales per
// operand and stage.
template <int NR, int KB>
__global__ void __launch_bounds__(32 * TC_Q4_WARPS, 2)
    k_ffn_up_q4tc(const __grid_constant__ CUtensorMap mx, const char* __restrict__ cw0,
                  const char* __restrict__ sw0, int64_t cst0, int64_t sst0,
                  const char* __restrict__ cw1, const char* __restrict__ sw1, int64_t cst1,
                  int64_t sst1, const char* __restrict__ cc0, const char* __restrict__ cc1,
                  int64_t cstr, int cscb, int nt, int nk,
                  int g, int H, int F, const int32_t* __restrict__ idx,
                  const int32_t* __restrict__ count, float* __restrict__ part, WsHeader* hdr) {
  pdl_wait();
  pdl_trigger();
  constexpr int NS = 2;
  constexpr uint32_t AT = TC_M * 128;  // one 64-column atom of a 128-row tile: 16 KB
  constexpr uint32_t NCOLS = NR == 1 ? 64u : 128u;
  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw = tc_sa(smem_raw);
  unsigned char* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  const uint32_t batom = (uint32_t)nt * 128u;  // one 64-column atom of the activation tile
  const uint32_t STAGE = NR * KB * AT + ((KB * batom + 1023u) & ~1023u);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + NS * STAGE);
  uint64_t* empty = full + NS;
  uint64_t* done = empty + NS;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort = reinterpret_cast<volatile int*>(tslot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int N = list_len(count, H, F, hdr);
  const UpShare us = up_share(N, g, nk, true);
  const int ks = us.ks, Np = us.nT * TC_M;
  if ((int)blockIdx.x >= us.nT * ks) return;
  const int tile = blockIdx.x / ks, split = blockIdx.x % ks;
  const int p0 = tile * TC_M;
  const int kt0 = (int)((long long)split * nk / ks), kt1 = (int)((long long)(split + 1) * nk / ks);
  const int nkt = kt1 - kt0;

  if (threadIdx.x == 0) tc_init(full, empty, done, abort, NS, (uint32_t)TC_Q4_LOADERS);
  if (warp == 0) tmem_alloc(tslot, NCOLS);
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem = *tslot;

  if (threadIdx.x < TC_Q4_LOADERS) {
    const int t = threadIdx.x, m = t >> 1, h = t & 1;
    const int p = p0 + m, row = list_row(p, H, N, F, idx);
    // a host-memory cold tier's listed rows were staged in device memory at
    // their list positions (cc0 / cc1: codes, scales cscb bytes behind; a
    // bad id staged as zeros); positions past the list read staged row 0
    // when there is no hot row 0 to read
    const bool cold = cc0 && p >= H && (p < N || H == 0);
    const size_t cq0 = (size_t)(p < N ? p - H : 0) * cstr;
    const char* cp[2] = {cold ? cc0 + cq0 : cw0 + (size_t)row * cst0,
                         NR == 2 ? (cold ? cc1 + cq0 : cw1 + (size_t)row * cst1) : nullptr};
    const char* sp[2] = {cold ? cc0 + cq0 + cscb : sw0 + (size_t)row * sst0,
                         NR == 2 ? (cold ? cc1 + cq0 + cscb : sw1 + (size_t)row * sst1) : nullptr};
    uint4 cq[TC_Q4_PRE][NR][KB];
    uint32_t sq[TC_Q4_PRE][NR];
    // codes and scales of stage i into register slot u
    auto fetch = [&](int i, int u) {
      if (i < nkt) {
        const size_t kb = (size_t)(kt0 + i) * 32 * KB + (size_t)h * 16 * KB;  // code bytes
        const size_t sb = (size_t)(kt0 + i) * 4 * KB + (size_t)h * 2 * KB;    // scale bytes
#pragma unroll
        for (int r = 0; r < NR; ++r) {
#pragma unroll
          for (int q = 0; q < KB; ++q) cq[u][r][q] = ld_q4_codes(cp[r] + kb + 16 * q);
          sq[u][r] = KB == 2 ? ld_q4_scales2(sp[r] + sb) : (uint32_t)ld_q4_scale(sp[r] + sb);
        }
      }
    };
#pragma unroll
    for (int u = 0; u < TC_Q4_PRE; ++u) fetch(u, u);
    const uint32_t sm0 = tc_sa(smem);
    bool stop = false;
    int last = -1;  // thread 0: the last stage whose activation tile it loaded
    for (int i0 = 0; i0 < nkt && !stop; i0 += TC_Q4_PRE) {
#pragma unroll
      for (int u = 0; u < TC_Q4_PRE; ++u) {
        const int i = i0 + u;
        if (i >= nkt) break;
        const int st = u % NS;  // i % NS (TC_Q4_PRE is a multiple of NS)
        int ok = 1;
        if (lane == 0 && i >= NS) ok = tc_wait(&empty[st], ((i / NS) - 1) & 1, abort, hdr);
        if (!__shfl_sync(0xffffffffu, ok, 0)) {
          stop = true;
          break;
        }
        unsigned char* a = smem + st * STAGE;
        if (t == 0) {
          mbar_expect_tx(&full[st], KB * batom);
          const int k = (kt0 + i) * 64 * KB;
#pragma unroll
          for (int at = 0; at < KB; ++at)
            tma_load_2d(a + NR * KB * AT + at * batom, &mx, k + 64 * at, 0, &full[st]);
          last = i;
        }
        // block h KB + q of the stage: atom (h KB + q) / 2, chunks 4 ((h KB + q) % 2) ..
        const uint32_t srow = sm0 + (uint32_t)st * STAGE + (uint32_t)m * 128u;
#pragma unroll
        for (int r = 0; r < NR; ++r) {
#pragma unroll
          for (int q = 0; q < KB; ++q) {
            const int blk = h * KB + q;
            const uint32_t ar = srow + (uint32_t)(r * KB + blk / 2) * AT;
            const uint32_t sbits = q ? (sq[u][r] >> 16) : (sq[u][r] & 0xFFFFu);
            const __half2 s2 = __half2half2(__ushort_as_half((unsigned short)sbits));
            const uint4 v = cq[u][r][q];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              const uint4 o = q4_chunk_f16(c & 1 ? v.z : v.x, c & 1 ? v.w : v.y, c >= 2, s2);
              const uint32_t cc = (uint32_t)(4 * (blk & 1) + c);
              sts128(ar + ((cc ^ (uint32_t)(m & 7)) << 4), o);
            }
          }
        }
        fence_async_smem();
        mbar_arrive_release(&full[st]);
        fetch(i + TC_Q4_PRE, u);
      }
    }
    if (t == 0 && last >= 0) {  // the activation tiles it loaded have landed (bounded)
      for (int i = last; i >= 0 && i > last - NS; --i)
        (void)tc_wait_quiet(&full[i % NS], (uint32_t)(i / NS) & 1u, hdr);
    }
  } else if (warp == 8 && lane == 0) {
    // kind::f16, fp16 A and B, both K-major, M = 128, N = nt
    const uint32_t idesc = (1u << 4) | ((uint32_t)(nt >> 3) << 17) | ((uint32_t)(TC_M >> 4) << 24);
    for (int i = 0; i < nkt; ++i) {
      const int st = i % NS;
      if (!tc_wait(&full[st], (uint32_t)(i / NS) & 1u, abort, hdr)) break;
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      const uint32_t a = tc_sa(smem + st * STAGE), b = a + NR * KB * AT;
#pragma unroll
      for (int at = 0; at < KB; ++at)
#pragma unroll
        for (int kk = 0; kk < TC_BK / 16; ++kk) {
          const uint64_t bd = sw128_desc(b + (uint32_t)at * batom + 32u * kk);
          const uint32_t acc = (i | at | kk) != 0 ? 1u : 0u;
#pragma unroll
          for (int r = 0; r < NR; ++r)
            mma_f16(tmem + (uint32_t)(r * nt), sw128_desc(a + (uint32_t)(r * KB + at) * AT + 32u * kk),
                    bd, idesc, acc);
        }
      mma_commit(&empty[st]);
    }
    mma_commit(done);
  }
  __syncwarp();

  bool ok = tc_wait_quiet(done, 0u, hdr);
  ok = __all_sync(0xffffffffu, ok && !*abort && nkt > 0);
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  if (ok && warp >= 8) {
    const int e = warp - 8;
    const int p = p0 + e * 32 + lane;
#pragma unroll
    for (int r = 0; r < NR; ++r) {
      float* dst = part + ((size_t)(split * NR + r) * Np + p) * nt;
      for (int c0 = 0; c0 < nt; c0 += 16) {
        uint32_t v[16];
        tmem_ld16(tmem + ((uint32_t)(e * 32) << 16) + (uint32_t)(r * nt + c0), v);
#pragma unroll
        for (int q = 0; q < 4; ++q)
          __stcg(reinterpret_cast<float4*>(dst + c0) + q,
                 make_float4(__uint_as_float(v[4 * q]), __uint_as_float(v[4 * q + 1]),
                             __uint_as_float(v[4 * q + 2]), __uint_as_float(v[4 * q + 3])));
      }
    }
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  if (warp == 0)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(NCOLS)
                 : "memory");
}

// Q4_0 down: as k_ffn_down_tc (grid (d / 128, ks), the k tiles that hold
// list positions split evenly over the ks CTAs of a column tile, part rows
// [split][b][c]), with the MN-major operand tile decoded from W_down^T's
// Q4_0 rows: loader t takes list position t / 4 of the stage's 64 and
// columns c0 + 32 (t % 4) .. +31 of it (one block: 16 code bytes and a
// scale).  The list rows are loaded one stage before
// the codes that depend on them, the codes TC_Q4_PRE - 1 stages ahead.
__global__ void __launch_bounds__(32 * TC_Q4_WARPS, 2)
    k_ffn_down_q4tc(const __grid_constant__ CUtensorMap mh, const char* __restrict__ cw,
                    const char* __restrict__ sw, int64_t cst, int64_t sst,
                    const char* __restrict__ cwc, int64_t cstr, int cscb, int nt, int ks, int d,
                    int batch, int H, int F, const int32_t* __restrict__ idx,
                    const int32_t* __restrict__ count, float* __restrict__ part, WsHeader* hdr) {
  pdl_wait();
  pdl_trigger();
  constexpr int NS = 4;
  constexpr uint32_t BOX = 64 * TC_BK * 2;  // 64 columns x 64 positions: 8 KB
  constexpr uint32_t A_BYTES = 2 * BOX;     // 128 columns
  constexpr uint32_t NCOLS = 64u;
  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw = tc_sa(smem_raw);
  unsigned char* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  const uint32_t bx = (uint32_t)nt * TC_BK * 2;  // the activation tile
  const uint32_t STAGE = A_BYTES + ((bx + 1023u) & ~1023u);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + NS * STAGE);
  uint64_t* empty = full + NS;
  uint64_t* done = empty + NS;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort = reinterpret_cast<volatile int*>(tslot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tile = blockIdx.x, split = blockIdx.y;
  const int N = list_len(count, H, F, hdr);
  const int nkN = (N + TC_BK - 1) / TC_BK;  // k tiles holding list positions
  const int kt0 = (int)((long long)split * nkN / ks);
  const int kt1 = (int)((long long)(split + 1) * nkN / ks);
  const int nkt = kt1 > kt0 ? kt1 - kt0 : 0;
  const int c0 = tile * TC_M;

  if (threadIdx.x == 0) {
    tc_init(full, empty, done, abort, NS, (uint32_t)TC_Q4_LOADERS);
    if (hdr && tile == 0 && split == 0) atomicAdd(&hdr->rows_down, (unsigned long long)N);
  }
  if (warp == 0) tmem_alloc(tslot, NCOLS);
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem = *tslot;

  if (threadIdx.x < TC_Q4_LOADERS) {
    const int t = threadIdx.x, k = t >> 2, q = t & 3;  // position in the stage, column block
    const size_t cb = (size_t)(c0 + 32 * q) / 2;       // code bytes of the block in a row
    const size_t sb = (size_t)(c0 + 32 * q) / 32 * 2;  // scale bytes
    int rq[TC_Q4_PRE] = {};  // list rows, one slot per stage
    uint4 cq[TC_Q4_PRE];     // codes
    uint16_t sq[TC_Q4_PRE];  // scales
    auto row_of = [&](int i) { return i < nkt ? list_row((kt0 + i) * TC_BK + k, H, N, F, idx) : 0; };
    auto fetch = [&](int i, int u) {
      if (i < nkt) {
        // a host-memory cold tier's listed rows, staged at their list
        // positions (as in the up kernel)
        const int pos = (kt0 + i) * TC_BK + k;
        const bool cold = cwc && pos >= H && (pos < N || H == 0);
        const size_t cq0 = (size_t)(pos < N ? pos - H : 0) * cstr;
        cq[u] = ld_q4_codes(cold ? cwc + cq0 + cb : cw + (size_t)rq[u] * cst + cb);
        sq[u] = ld_q4_scale(cold ? cwc + cq0 + cscb + sb : sw + (size_t)rq[u] * sst + sb);
      }
    };
#pragma unroll
    for (int u = 0; u < TC_Q4_PRE; ++u) rq[u] = row_of(u);
#pragma unroll
    for (int u = 0; u < TC_Q4_PRE - 1; ++u) fetch(u, u);
    const uint32_t sm0 = tc_sa(smem);
    const uint32_t h = (uint32_t)(q >> 1), cbase = (uint32_t)(4 * (q & 1));
    bool stop = false;
    int last = -1;
    for (int i0 = 0; i0 < nkt && !stop; i0 += TC_Q4_PRE) {
#pragma unroll
      for (int u = 0; u < TC_Q4_PRE; ++u) {
        const int i = i0 + u;
        if (i >= nkt) break;
        // the codes of stage i + PRE - 1 (their row came one stage ago), then
        // the row of stage i + PRE into the slot this stage frees
        const int un = (u + TC_Q4_PRE - 1) % TC_Q4_PRE;
        fetch(i + TC_Q4_PRE - 1, un);
        const int st = u % NS;
        int ok = 1;
        if (lane == 0 && i >= NS) ok = tc_wait(&empty[st], ((i / NS) - 1) & 1, abort, hdr);
        if (!__shfl_sync(0xffffffffu, ok, 0)) {
          stop = true;
          break;
        }
        unsigned char* a = smem + st * STAGE;
        if (t == 0) {
          mbar_expect_tx(&full[st], bx);
          tma_load_2d(a + A_BYTES, &mh, 0, (kt0 + i) * nt, &full[st]);
          last = i;
        }
        const __half2 s2 = __half2half2(__ushort_as_half(sq[u]));
        const uint4 v = cq[u];
        const uint32_t ab = sm0 + (uint32_t)st * STAGE + h * BOX + (uint32_t)k * 128u;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const uint4 o = q4_chunk_f16(c & 1 ? v.z : v.x, c & 1 ? v.w : v.y, c >= 2, s2);
          sts128(ab + (((cbase + (uint32_t)c) ^ (uint32_t)(k & 7)) << 4), o);
        }
        fence_async_smem();
        mbar_arrive_release(&full[st]);
        rq[u] = row_of(i + TC_Q4_PRE);
      }
    }
    if (t == 0 && last >= 0) {
      for (int i = last; i >= 0 && i > last - NS; --i)
        (void)tc_wait_quiet(&full[i % NS], (uint32_t)(i / NS) & 1u, hdr);
    }
  } else if (warp == 8 && lane == 0) {
    // kind::f16, fp16 A (MN-major) and B (K-major), fp32 D, M = 128, N = nt
    const uint32_t idesc = (1u << 4) | (1u << 15) | ((uint32_t)(nt >> 3) << 17) |
                           ((uint32_t)(TC_M >> 4) << 24);
    for (int i = 0; i < nkt; ++i) {
      const int st = i % NS;
      if (!tc_wait(&full[st], (uint32_t)(i / NS) & 1u, abort, hdr)) break;
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      const uint32_t a = tc_sa(smem + st * STAGE), b = a + A_BYTES;
#pragma unroll
      for (int kk = 0; kk < TC_BK / 16; ++kk)
        mma_f16(tmem, sw128_mn_desc(a + 2048u * kk, BOX), sw128_desc(b + 32u * kk), idesc,
                (i | kk) != 0 ? 1u : 0u);
      mma_commit(&empty[st]);
    }
    mma_commit(done);
  }
  __syncwarp();

  bool ok = tc_wait_quiet(done, 0u, hdr);
  ok = __all_sync(0xffffffffu, ok && !*abort);
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  // accumulator lane = output column, accumulator column = token; a split
  // with no list positions writes zeros (the reduction sums every slice)
  if (warp >= 8) {
    const int e = warp - 8;
    const int c = c0 + e * 32 + lane;
    for (int t0 = 0; t0 < nt; t0 += 16) {
      uint32_t v[16];
      if (ok && nkt > 0) {
        tmem_ld16(tmem + ((uint32_t)(e * 32) << 16) + (uint32_t)t0, v);
      } else {
#pragma unroll
        for (int tt = 0; tt < 16; ++tt) v[tt] = 0u;
      }
#pragma unroll
      for (int tt = 0; tt < 16; ++tt)
        if (t0 + tt < batch) __stcg(part + ((size_t)split * batch + t0 + tt) * d + c, __uint_as_float(v[tt]));
    }
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  if (warp == 0)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(NCOLS)
                 : "memory");
}

// xh (fp32 [batch][d]) -> xh16 (fp16 [nt][d], rows >= batch zero); 8 per thread.
__global__ void k_xh16(const float* __restrict__ xh, int batch, int d, int nt,
                       __half* __restrict__ xh16) {
  pdl_wait();
  pdl_trigger();
  const int n8 = d / 8;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < nt * n8; i += gridDim.x * blockDim.x) {
    const int t = i / n8, c = i % n8;
    uint4 o = make_uint4(0u, 0u, 0u, 0u);
    if (t < batch) {
      const float4 a = __ldg(reinterpret_cast<const float4*>(xh + (size_t)t * d) + 2 * c);
      const float4 b = __ldg(reinterpret_cast<const float4*>(xh + (size_t)t * d) + 2 * c + 1);
      const __half2 h0 = __floats2half2_rn(a.x, a.y), h1 = __floats2half2_rn(a.z, a.w);
      const __half2 h2 = __floats2half2_rn(b.x, b.y), h3 = __floats2half2_rn(b.z, b.w);
      o = make_uint4(*reinterpret_cast<const uint32_t*>(&h0), *reinterpret_cast<const uint32_t*>(&h1),
                     *reinterpret_cast<const uint32_t*>(&h2), *reinterpret_cast<const uint32_t*>(&h3));
    }
    reinterpret_cast<uint4*>(xh16 + (size_t)t * d)[c] = o;
  }
}

// For list positions p of this block's 64: h = act(sum over splits (fixed
// order) + bias), zero for a token whose own bit is 0 (per-token masks, cold
// positions), for positions past the list and for bad list entries (which
// also set DEV_BAD_INDEX); written to h16 tile-major, [Fp / 64][nt][64]
// (tokens t >= batch: 0), so that the down kernel's activation tile of a
// stage is one contiguous 8 KB block: every column tile loads the same
// tile at about the same time, and 64 rows a whole d_ff apart would
// gather those loads on a few L2 slices.
// Blocks wholly past the list write nothing: the down kernel reads h16 only
// in 64-position tiles that hold list positions.
// Partial sums read and h16 written coalesced through shared memory.
template <int NR>
__global__ void __launch_bounds__(256) k_ffn_finish(const float* __restrict__ part, int g, int nk,
                                                    int fit, int direct, int H, int F, int Fp,
                                                    int nt, int batch,
                                                    const int32_t* __restrict__ idx,
                                                    const int32_t* __restrict__ count,
                                                    const float* __restrict__ bias,
                                                    const uint32_t* __restrict__ mask, int words,
                                                    __half* __restrict__ h16, WsHeader* hdr,
                                                    int sq) {
  pdl_wait();
  pdl_trigger();
  __shared__ float sh[64][TC_TMAX + 1];
  __shared__ int sj[64];    // each row's neuron
  __shared__ float sb[64];  // and bias
  __shared__ int sv[64];    // 1: a listed row with a valid neuron
  const int N = list_len(count, H, F, hdr);
  if (hdr && blockIdx.x == 0 && threadIdx.x == 0) {
    atomicAdd(&hdr->rows_listed, (unsigned long long)N);
    if (NR == 2) atomicAdd(&hdr->rows_second, (unsigned long long)N);
  }
  const int n0 = blockIdx.x * 64;
  if (n0 >= N) return;
  const UpShare us = up_share(N, g, nk, fit != 0);
  if (direct && us.ks == 1) return;  // the up kernel applied the activation itself
  const int ks = us.ks, Np = us.nT * TC_M;
  const int m = 64 * nt;
  // per row once: neuron, index check, bias
  if (threadIdx.x < 64) {
    const int p = n0 + threadIdx.x;
    int j = 0, v = 0;
    float bb = 0.f;
    if (p < N) {
      j = p < H ? p : idx[p - H];
      if (p >= H && (j < H || j >= F)) {
        if (hdr) atomicOr(&hdr->status, DEV_BAD_INDEX);
      } else {
        v = 1;
        bb = bias ? bias[j] : 0.f;
      }
    }
    sj[threadIdx.x] = j;
    sb[threadIdx.x] = bb;
    sv[threadIdx.x] = v;
  }
  __syncthreads();
  // this thread's elements i = threadIdx.x + 256 e of the block's 64 x nt:
  // the sums over the splits stay in registers, and each split's loads of
  // all of them are in flight together
  constexpr int EPT = 64 * TC_TMAX / 256;
  float gs[EPT], ua[EPT];
#pragma unroll
  for (int e = 0; e < EPT; ++e) gs[e] = ua[e] = 0.f;
  for (int s = 0; s < ks; ++s) {
    const float* pg = part + ((size_t)(s * NR) * Np + n0) * nt;
    const float* pu = part + ((size_t)(s * NR + 1) * Np + n0) * nt;
#pragma unroll
    for (int e = 0; e < EPT; ++e) {
      const int i = threadIdx.x + 256 * e;
      if (i < m) {
        gs[e] += __ldcg(pg + i);
        if constexpr (NR == 2) ua[e] += __ldcg(pu + i);
      }
    }
  }
#pragma unroll
  for (int e = 0; e < EPT; ++e) {
    const int i = threadIdx.x + 256 * e;
    if (i >= m) break;
    const int nn = i / nt, b = i % nt, p = n0 + nn;
    float hv = 0.f;
    if (sv[nn] && b < batch) {
      const int j = sj[nn];
      const float gv = gs[e] + sb[nn];
      hv = gv > 0.f ? gv : 0.f;
      if constexpr (NR == 2) hv *= ua[e];
      else if (sq) hv *= hv;  // squared ReLU
      if (mask && p >= H && !((__ldg(mask + (size_t)b * words + (j >> 5)) >> (j & 31)) & 1u)) hv = 0.f;
    }
    sh[nn][b] = hv;
  }
  __syncthreads();
  for (int i = threadIdx.x; i < m; i += blockDim.x) {
    const int b = i / 64, nn = i % 64;
    h16[((size_t)(n0 / 64) * nt + b) * 64 + nn] = __float2half_rn(sh[nn][b]);
  }
}

// down: part[split][b][c] = sum over the split's list positions p of
// W_down^T[row(p)][c] h[b][p], for the tile's 128 CH columns c (CH M = 128
// operands and accumulators; CH = 2 reads each listed row in 512-byte
// pieces from half as many CTAs, with a 2-stage ring).  Grid
// (d / (128 CH), ks).
template <int CH>
__global__ void __launch_bounds__(32 * TC_FFN_WARPS, 1)
    k_ffn_down_tc(const __grid_constant__ CUtensorMap mwd, const __grid_constant__ CUtensorMap mwg,
                  const __grid_constant__ CUtensorMap mh, int nt, int nk, int ks, int d, int batch,
                  int H, int F, const int32_t* __restrict__ idx, const int32_t* __restrict__ count,
                  float* __restrict__ part, WsHeader* hdr) {
  pdl_wait();
  pdl_trigger();
  constexpr uint32_t BOX = 64 * TC_BK * 2;             // 64 columns x 64 positions: 8 KB
  constexpr uint32_t A_BYTES = 2 * CH * BOX;           // 128 CH columns
  constexpr uint32_t B_BYTES = TC_TMAX * TC_BK * 2;    // 8 KB
  constexpr uint32_t STAGE = A_BYTES + B_BYTES;
  constexpr uint32_t NCOLS = 64u * CH;
  constexpr int DS = CH == 1 ? TC_STAGES : 2;  // ring stages
  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw = tc_sa(smem_raw);
  unsigned char* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + DS * STAGE);
  uint64_t* empty = full + DS;
  uint64_t* done = empty + DS;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort = reinterpret_cast<volatile int*>(tslot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tile = blockIdx.x, split = blockIdx.y;
  const int N = list_len(count, H, F, hdr);
  const int nkN = (N + TC_BK - 1) / TC_BK;  // k tiles holding list positions
  // the splits share the k tiles that hold list positions, not all of d_ff
  // (the list is usually much shorter), so no split idles
  (void)nk;
  const int kt0 = (int)((long long)split * nkN / ks);
  const int kt1 = (int)((long long)(split + 1) * nkN / ks);
  const int nkt = kt1 > kt0 ? kt1 - kt0 : 0;

  if (threadIdx.x == 0) {
    tc_init(full, empty, done, abort, DS, (uint32_t)TC_PW);
    if (hdr && tile == 0 && split == 0) atomicAdd(&hdr->rows_down, (unsigned long long)N);
  }
  if (warp == 0) tmem_alloc(tslot, NCOLS);
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem = *tslot;
  const int c0 = tile * TC_M * CH;

  if (warp != 1) {
    // TC_PW producer warps, each arming its own bytes on the stage's full
    // barrier (TC_PW arrivals per phase).  A stage inside the hot prefix is
    // two 64-column boxes (warp 0).  Otherwise its 32 four-position gathers
    // (positions pk + 4g .. pk + 4g + 3 of 64-column part o / 16, g = o % 16)
    // are dealt out round-robin, gather o = TC_PW * lane + pw.  Each lane
    // holds the list rows of its gather for as many stages ahead as the ring
    // is deep, so the list loads of a stage are in flight a whole ring ahead
    // of its gathers (the loop runs the ring's slots unrolled, and the row
    // registers are indexed statically).
    const int pw = warp == 0 ? 0 : warp - 1;
    const int o = TC_PW * lane + pw;
    const int part64 = o >> 4, g = o & 15;  // 64-column part, position group
    const bool gl = o < 32 * CH;
    const uint32_t bx = (uint32_t)nt * TC_BK * 2;  // the activation tile
    const uint32_t mine = (uint32_t)((32 * CH - pw + TC_PW - 1) / TC_PW);  // gathers of this warp
    int yr[DS][4];  // list rows of this lane's gather, one set per ring slot
    auto rows_at = [&](int i, int (&v)[4]) {
      const int q = (kt0 + i) * TC_BK + 4 * g;
#pragma unroll
      for (int t = 0; t < 4; ++t) v[t] = gl ? list_row(q + t, H, N, F, idx) : 0;
    };
#pragma unroll
    for (int u = 0; u < DS; ++u)
      if (u < nkt) rows_at(u, yr[u]);
    int last[DS];
#pragma unroll
    for (int u = 0; u < DS; ++u) last[u] = -1;
    bool stop = false;
    for (int i0 = 0; i0 < nkt && !stop; i0 += DS) {
#pragma unroll
      for (int st = 0; st < DS; ++st) {  // ring slot st = i % DS
        const int i = i0 + st;
        if (i >= nkt) break;
        int ok = 1;
        if (lane == 0 && i >= DS) ok = tc_wait(&empty[st], ((i / DS) - 1) & 1, abort, hdr);
        if (!__shfl_sync(0xffffffffu, ok, 0)) {
          stop = true;
          break;
        }
        unsigned char* a = smem + st * STAGE;
        const int pk = (kt0 + i) * TC_BK;  // first list position of the stage
        const bool boxed = pk + TC_BK <= H;
        const uint32_t tx = boxed ? (pw == 0 ? A_BYTES + bx : 0u) : 512u * mine + (pw == 0 ? bx : 0u);
        const int y0 = yr[st][0], y1 = yr[st][1], y2 = yr[st][2], y3 = yr[st][3];
        if (i + DS < nkt) rows_at(i + DS, yr[st]);
        if (lane == 0)
          asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(tc_sa(&full[st])),
                       "r"(tx)
                       : "memory");
        __syncwarp();
        if (boxed) {
          if (pw == 0 && lane == 0) {
#pragma unroll
            for (int q = 0; q < 2 * CH; ++q) tma_load_2d(a + q * BOX, &mwd, c0 + 64 * q, pk, &full[st]);
          }
        } else if (gl) {
          tma_gather4(a + part64 * BOX + 512u * g, &mwg, c0 + 64 * part64, y0, y1, y2, y3,
                      &full[st]);
        }
        if (pw == 0 && lane == 0) tma_load_2d(a + A_BYTES, &mh, 0, (pk / TC_BK) * nt, &full[st]);
        last[st] = i;
      }
    }
    if (lane == 0) {
#pragma unroll
      for (int st = 0; st < DS; ++st)
        if (last[st] >= 0) (void)tc_wait_quiet(&full[st], (uint32_t)(last[st] / DS) & 1u, hdr);
    }
  } else if (warp == 1 && lane == 0) {
    // kind::f16, fp16 A (MN-major) and B (K-major), fp32 D, M = 128, N = nt
    const uint32_t idesc = (1u << 4) | (1u << 15) | ((uint32_t)(nt >> 3) << 17) |
                           ((uint32_t)(TC_M >> 4) << 24);
    for (int i = 0; i < nkt; ++i) {
      const int st = i % DS;
      if (!tc_wait(&full[st], (uint32_t)(i / DS) & 1u, abort, hdr)) break;
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      const uint32_t a = tc_sa(smem + st * STAGE), b = a + A_BYTES;
#pragma unroll
      for (int kk = 0; kk < TC_BK / 16; ++kk) {  // 16 positions = 2 K atoms of the A tile per MMA
        const uint64_t bd = sw128_desc(b + 32u * kk);
#pragma unroll
        for (int hh = 0; hh < CH; ++hh)
          mma_f16(tmem + 64u * hh, sw128_mn_desc(a + 2 * hh * BOX + 2048u * kk, BOX), bd, idesc,
                  (i | kk) != 0 ? 1u : 0u);
      }
      mma_commit(&empty[st]);
    }
    mma_commit(done);
  }
  __syncwarp();

  bool ok = tc_wait_quiet(done, 0u, hdr);
  ok = __all_sync(0xffffffffu, ok && !*abort);
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  // accumulator lane = output column, accumulator column = token; a split
  // with no list positions writes zeros (the reduction sums every slice)
  for (int hh = 0; hh < CH; ++hh)
  for (int t0 = 0; t0 < nt && warp < 4; t0 += 16) {
    const int c = c0 + 128 * hh + warp * 32 + lane;
    uint32_t v[16];
    if (ok && nkt > 0) {
      tmem_ld16(tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)(64 * hh + t0), v);
    } else {
#pragma unroll
      for (int t = 0; t < 16; ++t) v[t] = 0u;
    }
#pragma unroll
    for (int t = 0; t < 16; ++t)
      if (t0 + t < batch) __stcg(part + ((size_t)split * batch + t0 + t) * d + c, __uint_as_float(v[t]));
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  if (warp == 0)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(NCOLS)
                 : "memory");
}

constexpr int TC_KSMAX_U = 16;  // CTAs sharing one tile of P1's d at most
constexpr int TC_PSTAGES = 3;   // predictor ring stages: 97 KB, two CTAs per SM

// x (fp32 [batch][n]) -> hi = fp16(x), lo = fp16(x - hi), [nt][n] each
// (rows >= batch zero); eight elements per thread (n % 8 == 0).
__global__ void k_split16(const float* __restrict__ x, int batch, int n, int nt,
                          __half* __restrict__ hi, __half* __restrict__ lo) {
  pdl_wait();
  pdl_trigger();
  const int n8 = n / 8;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < nt * n8; i += gridDim.x * blockDim.x) {
    const int t = i / n8;
    float v[8];
    if (t < batch) {
      const float4 a = __ldg(reinterpret_cast<const float4*>(x) + 2 * (size_t)i);
      const float4 b = __ldg(reinterpret_cast<const float4*>(x) + 2 * (size_t)i + 1);
      v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
      v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    } else {
#pragma unroll
      for (int k = 0; k < 8; ++k) v[k] = 0.f;
    }
    __align__(16) __half h[8], l[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      h[k] = __float2half_rn(v[k]);
      l[k] = __float2half_rn(v[k] - __half2float(h[k]));
    }
    reinterpret_cast<uint4*>(hi)[i] = *reinterpret_cast<const uint4*>(h);
    reinterpret_cast<uint4*>(lo)[i] = *reinterpret_cast<const uint4*>(l);
  }
}

// MODE 0: D = P1 (x_hi + x_lo)^T for 128 predictor rows per tile, d split
// over ks CTAs -> part[split][token][row] (token-major, so the finish
// kernel reads and writes along the rows).  MODE 1: D = P2 (u_hi + u_lo)^T
// for 128 neuron rows per tile from row0 (a multiple of 32, <= hot) -> mask
// words: bit j of token t = (j < hot) or (z_j + c_j > theta) for j < d_ff;
// the words below row0 (all hot) are written all ones by the CTAs in turn,
// and `uni`, when given, gets each word's OR over the batch's tokens (each
// warp holds one word of every token).  Grid (tiles, ks).
template <int MODE>
__global__ void __launch_bounds__(TC_THREADS, 1)
    k_pred_tc(const __grid_constant__ CUtensorMap ma, const __grid_constant__ CUtensorMap mbh,
              const __grid_constant__ CUtensorMap mbl, int nt, int nk, int ks, int row0, int M,
              float* __restrict__ part, const float* __restrict__ bias, float theta, int H,
              uint32_t* __restrict__ mask, int words, int batch, WsHeader* hdr,
              uint32_t* __restrict__ uni) {
  constexpr uint32_t A_BYTES = TC_M * TC_BK * 2;     // 16 KB
  constexpr uint32_t B_BYTES = TC_TMAX * TC_BK * 2;  // 8 KB per part
  constexpr uint32_t STAGE = A_BYTES + 2 * B_BYTES;
  constexpr uint32_t NCOLS = 64u;
  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw = tc_sa(smem_raw);
  unsigned char* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + TC_PSTAGES * STAGE);
  uint64_t* empty = full + TC_PSTAGES;
  uint64_t* done = empty + TC_PSTAGES;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort = reinterpret_cast<volatile int*>(tslot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tile = blockIdx.x, split = blockIdx.y;
  const int m0 = row0 + tile * TC_M;
  const int kt0 = (int)((long long)split * nk / ks), kt1 = (int)((long long)(split + 1) * nk / ks);
  const int nkt = kt1 - kt0;

  if (threadIdx.x == 0) tc_init(full, empty, done, abort, TC_PSTAGES);
  if (warp == 0) tmem_alloc(tslot, NCOLS);
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem = *tslot;
  pdl_wait();  // the prologue above touches no global memory
  pdl_trigger();

  if (warp == 0 && lane == 0) {
    const uint32_t tx = A_BYTES + 2u * (uint32_t)nt * TC_BK * 2;
    int last[TC_PSTAGES];
    for (int i = 0; i < TC_PSTAGES; ++i) last[i] = -1;
    for (int i = 0; i < nkt; ++i) {
      const int st = i % TC_PSTAGES;
      if (i >= TC_PSTAGES && !tc_wait(&empty[st], ((i / TC_PSTAGES) - 1) & 1, abort, hdr)) break;
      unsigned char* a = smem + st * STAGE;
      asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(tc_sa(&full[st])),
                   "r"(tx)
                   : "memory");
      const int k = (kt0 + i) * TC_BK;
      tma_load_2d(a, &ma, k, m0, &full[st]);  // rows past the matrix read zeros
      tma_load_2d(a + A_BYTES, &mbh, k, 0, &full[st]);
      tma_load_2d(a + A_BYTES + B_BYTES, &mbl, k, 0, &full[st]);
      last[st] = i;
    }
    for (int st = 0; st < TC_PSTAGES; ++st)
      if (last[st] >= 0) (void)tc_wait_quiet(&full[st], (uint32_t)(last[st] / TC_PSTAGES) & 1u, hdr);
  } else if (warp == 1 && lane == 0) {
    const uint32_t idesc = (1u << 4) | ((uint32_t)(nt >> 3) << 17) | ((uint32_t)(TC_M >> 4) << 24);
    for (int i = 0; i < nkt; ++i) {
      const int st = i % TC_PSTAGES;
      if (!tc_wait(&full[st], (uint32_t)(i / TC_PSTAGES) & 1u, abort, hdr)) break;
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      const uint32_t a = tc_sa(smem + st * STAGE), bh = a + A_BYTES, bl = bh + B_BYTES;
#pragma unroll
      for (int kk = 0; kk < TC_BK / 16; ++kk) {
        const uint64_t ad = sw128_desc(a + 32u * kk);
        mma_f16(tmem, ad, sw128_desc(bh + 32u * kk), idesc, (i | kk) != 0 ? 1u : 0u);
        mma_f16(tmem, ad, sw128_desc(bl + 32u * kk), idesc, 1u);
      }
      mma_commit(&empty[st]);
    }
    mma_commit(done);
  }
  __syncwarp();

  bool ok = tc_wait_quiet(done, 0u, hdr);
  ok = __all_sync(0xffffffffu, ok && !*abort && nkt > 0);
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const int m = m0 + warp * 32 + lane;  // this thread's row
  uint32_t any = 0u;                     // MODE 1: OR of this warp's word over the tokens
  for (int c0 = 0; c0 < nt; c0 += 16) {
    uint32_t v[16];
    if (ok) {
      tmem_ld16(tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)c0, v);
    } else {
#pragma unroll
      for (int t = 0; t < 16; ++t) v[t] = 0u;
    }
    if constexpr (MODE == 0) {
      if (m < M) {
        float* dst = part + ((size_t)split * nt + c0) * M + m;
#pragma unroll
        for (int t = 0; t < 16; ++t) __stcg(dst + (size_t)t * M, __uint_as_float(v[t]));
      }
    } else {
      const float cb = (bias && m < M) ? bias[m] : 0.f;
      const int w = (m0 + warp * 32) >> 5;  // this warp's mask word
#pragma unroll
      for (int t = 0; t < 16; ++t) {
        const bool bit = m < H || (m < M && __uint_as_float(v[t]) + cb > theta);
        const uint32_t word = __ballot_sync(0xffffffffu, bit);
        if (c0 + t < batch) any |= word;
        if (lane == 0 && c0 + t < batch && w < words) mask[(size_t)(c0 + t) * words + w] = word;
      }
    }
  }
  if constexpr (MODE == 1) {
    const int w = (m0 + warp * 32) >> 5;
    if (uni && lane == 0 && w < words) uni[w] = any;
    const int w0 = row0 >> 5;  // hot words, all ones
    for (int i = (blockIdx.x * gridDim.y + blockIdx.y) * TC_THREADS + threadIdx.x; i < batch * w0;
         i += gridDim.x * gridDim.y * TC_THREADS)
      mask[(size_t)(i / w0) * words + i % w0] = 0xFFFFFFFFu;
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  if (warp == 0)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(NCOLS)
                 : "memory");
}

// u = sum over the splits (fixed order) of part[split][t][k] -> u_hi,
// u_lo [nt][r] (tokens >= batch: 0); four rows k per thread (r % 4 == 0),
// every split's load issued before the sums (ks <= TC_KSMAX_U).
__global__ void k_pred_u_finish(const float* __restrict__ part, int ks, int r, int nt, int batch,
                                __half* __restrict__ uhi, __half* __restrict__ ulo) {
  pdl_wait();
  pdl_trigger();
  const int r4 = r / 4;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < nt * r4; i += gridDim.x * blockDim.x) {
    const int t = i / r4;
    float4 u = make_float4(0.f, 0.f, 0.f, 0.f);
    if (t < batch) {
      float4 v[TC_KSMAX_U];
#pragma unroll
      for (int s = 0; s < TC_KSMAX_U; ++s)
        if (s < ks) v[s] = __ldcg(reinterpret_cast<const float4*>(part + (size_t)s * nt * r) + i);
#pragma unroll
      for (int s = 0; s < TC_KSMAX_U; ++s)
        if (s < ks) {
          u.x += v[s].x;
          u.y += v[s].y;
          u.z += v[s].z;
          u.w += v[s].w;
        }
    }
    const float uu[4] = {u.x, u.y, u.z, u.w};
    __align__(8) __half h[4], l[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      h[k] = __float2half_rn(uu[k]);
      l[k] = __float2half_rn(uu[k] - __half2float(h[k]));
    }
    reinterpret_cast<uint2*>(uhi)[i] = *reinterpret_cast<const uint2*>(h);
    reinterpret_cast<uint2*>(ulo)[i] = *reinterpret_cast<const uint2*>(l);
  }
}

// Mask words below the first evaluated row: all hot, all ones.
__global__ void k_hot_words(uint32_t* __restrict__ mask, int words, int w0, int batch) {
  pdl_wait();
  pdl_trigger();
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < batch * w0; i += gridDim.x * blockDim.x)
    mask[(size_t)(i / w0) * words + i % w0] = 0xFFFFFFFFu;
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static std::mutex mu;
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// 2-D fp16 tensor [rows][inner] with `row_bytes` between rows; box
// [box_rows][64], 128-byte swizzle (box_rows = 1 for gather4 maps).
bool map_2d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint64_t row_bytes,
            uint32_t box_rows) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  const cuuint64_t dims[2] = {inner, rows};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {(cuuint32_t)TC_BK, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool tc_disabled() {
  const char* e = getenv("PI_DISABLE_TC");
  return e && e[0] && e[0] != '0';
}

size_t up256(size_t v) { return (v + 255) & ~(size_t)255; }

int fpad(int F) { return (F + TC_M - 1) / TC_M * TC_M; }

// CTA slots of the up kernel's grid (two CTAs per SM), and its length:
// every row tile of the longest list (ks = 1) or the slots, whichever is more.
int up_slots() { return 2 * device_sms(); }
int up_grid(int F) { return std::max(up_slots(), fpad(F) / TC_M); }

int pred_u_splits(int d, int r) {
  int ks = device_sms() / (r / TC_M);
  ks = ks < 1 ? 1 : (ks > TC_KSMAX_U ? TC_KSMAX_U : ks);
  return ks > d / TC_BK ? d / TC_BK : ks;
}

// Scratch: xh16 [64][d] fp16 | up partial sums [ks][2][Fp][64] fp32 |
// h16 [Fp / 64][64][64] fp16 | predictor: xs_lo [64][d] fp16 | u partial sums
// [ksu][r][64] fp32 | u_hi, u_lo [64][r] fp16 (xh16 doubles as xs_hi).
struct TcScratch {
  __half* xh16;
  float* part;
  __half* h16;
  __half* xlo;
  float* upart;
  __half* uhi;
  __half* ulo;
  size_t bytes;
};

TcScratch tc_scratch(void* base, int d, int F, int r) {
  char* p0 = static_cast<char*>(base);
  char* p = p0;
  TcScratch t;
  t.xh16 = reinterpret_cast<__half*>(p);
  p += up256((size_t)TC_TMAX * d * 2);
  t.part = reinterpret_cast<float*>(p);
  // nT * ks <= up_grid(F) partial row tiles of two operands (fp16), or
  // (Fp / 128) * (d / 2048) (Q4_0: up to nk / 32 shares per tile, nk <= d / 64)
  const size_t ptiles = std::max((size_t)up_grid(F), (size_t)(fpad(F) / TC_M) * std::max(1, d / 2048));
  p += up256(ptiles * TC_M * 2 * TC_TMAX * 4);
  t.h16 = reinterpret_cast<__half*>(p);
  p += up256((size_t)TC_TMAX * fpad(F) * 2);
  t.xlo = reinterpret_cast<__half*>(p);
  p += up256((size_t)TC_TMAX * d * 2);
  t.upart = reinterpret_cast<float*>(p);
  p += up256(r % TC_M == 0 ? (size_t)pred_u_splits(d, r) * r * TC_TMAX * 4 : 0);
  t.uhi = reinterpret_cast<__half*>(p);
  p += up256((size_t)TC_TMAX * r * 2);
  t.ulo = reinterpret_cast<__half*>(p);
  p += up256((size_t)TC_TMAX * r * 2);
  t.bytes = (size_t)(p - p0);
  return t;
}

template <int NR>
cudaError_t launch_up_nr(const pi_layer& L, const float* xh, int batch, const uint32_t* mask,
                         const int32_t* idx, const int32_t* count, void* scratch, WsHeader* hdr,
                         cudaStream_t s, bool xh16_ready) {
  const int d = L.d_model, H = L.hot, F = L.d_ff, Fp = fpad(F);
  const int nt = (batch + 15) / 16 * 16;
  const TcScratch sc = tc_scratch(scratch, d, F, L.rank);
  const int64_t rs = code_stride(PI_F16, d, L.w_row_stride);
  const int64_t rs2 = code_stride(PI_F16, d, NR == 2 && L.w_up_row_stride ? L.w_up_row_stride
                                                                           : L.w_row_stride);
  const void* w0 = NR == 2 ? L.w_gate : L.w_up;
  CUtensorMap m0, m1, g0, g1, mx;
  if (!map_2d(&m0, w0, (uint64_t)d, (uint64_t)F, (uint64_t)rs, TC_M) ||
      !map_2d(&m1, L.w_up, (uint64_t)d, (uint64_t)F, (uint64_t)rs2, TC_M) ||
      !map_2d(&g0, w0, (uint64_t)d, (uint64_t)F, (uint64_t)rs, 1) ||
      !map_2d(&g1, L.w_up, (uint64_t)d, (uint64_t)F, (uint64_t)rs2, 1) ||
      !map_2d(&mx, sc.xh16, (uint64_t)d, (uint64_t)nt, (uint64_t)d * 2, (uint32_t)nt))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaSuccess;
  if (!xh16_ready) {
    (void)launch_dep(k_xh16, std::min((nt * d / 8 + 255) / 256, device_sms() * 4), 256, 0, s, xh,
                     batch, d, nt, sc.xh16);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  const int nk = d / TC_BK, g = up_slots();
  const int NS = up_stages(NR, nt);
  const uint32_t stage = NR * TC_M * TC_BK * 2 + (((uint32_t)nt * TC_BK * 2 + 1023u) & ~1023u);
  const size_t smem = 1024 + (size_t)NS * stage + 8 * (2 * NS + 1) + 16 + 4 * TC_M;
  auto kern = NS == up_stages(NR, 64) ? k_ffn_up_tc<NR, up_stages(NR, 64)>
                                      : k_ffn_up_tc<NR, up_stages(NR, 16)>;
  e = allow_smem_fn(reinterpret_cast<const void*>(kern), smem);
  if (e != cudaSuccess) return e;
  (void)launch_dep(kern, up_grid(F), 32 * TC_FFN_WARPS, smem, s, m0, m1, g0, g1, mx, nt, nk, g, H,
                   F, idx, count, sc.part, hdr, L.bias, mask, (F + 31) / 32, sc.h16, batch,
                   L.act == PI_RELU2 ? 1 : 0);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  (void)launch_dep(k_ffn_finish<NR>, Fp / 64, 256, 0, s, sc.part, g, nk, 0, 1, H, F, Fp, nt, batch, idx,
                   count, L.bias, mask, (F + 31) / 32, sc.h16, hdr, L.act == PI_RELU2 ? 1 : 0);
  return cudaGetLastError();
}

// Q4_0 up/gate (k_ffn_up_q4tc) and the same finish kernel, two CTAs per
// SM: one operand takes K = 128 per stage (two 48 KB stages at most), two
// operands K = 64 (two 40 KB stages).
template <int NR>
cudaError_t launch_up_q4(const pi_layer& L, const float* xh, int batch, const uint32_t* mask,
                         const int32_t* idx, const int32_t* count, void* scratch, WsHeader* hdr,
                         cudaStream_t s, bool xh16_ready, char* cold_stage) {
  const int d = L.d_model, H = L.hot, F = L.d_ff, Fp = fpad(F);
  const int nt = (batch + 15) / 16 * 16;
  const TcScratch sc = tc_scratch(scratch, d, F, L.rank);
  const int64_t ur = NR == 2 && L.w_up_row_stride ? L.w_up_row_stride : L.w_row_stride;
  const char* cw0 = static_cast<const char*>(NR == 2 ? L.w_gate : L.w_up);
  const char* sw0 = static_cast<const char*>(NR == 2 ? L.w_gate_scales : L.w_up_scales);
  CUtensorMap mx;
  if (!map_2d(&mx, sc.xh16, (uint64_t)d, (uint64_t)nt, (uint64_t)d * 2, (uint32_t)nt))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaSuccess;
  if (!xh16_ready) {
    (void)launch_dep(k_xh16, std::min((nt * d / 8 + 255) / 256, device_sms() * 4), 256, 0, s, xh,
                     batch, d, nt, sc.xh16);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  // a host-memory cold tier: its listed rows first, once, into the stage
  const int64_t srb = stage_row_bytes(PI_Q4_0, d);
  const char *cc0 = nullptr, *cc1 = nullptr;
  if (L.w_up_cold) {
    if (!cold_stage) return cudaErrorInvalidValue;
    if ((e = launch_stage_cold(L, idx, count, cold_stage, hdr, s)) != cudaSuccess) return e;
    cc0 = cold_stage;
    cc1 = cold_stage + (size_t)(F - H) * srb;
  }
  constexpr int KB = NR == 1 ? 2 : 1;
  const int nk = d / (64 * KB), g = 2 * device_sms();
  const uint32_t stage = NR * KB * TC_M * 128 + (((uint32_t)nt * 128 * KB + 1023u) & ~1023u);
  const size_t smem = 1024 + 2 * (size_t)stage + 8 * (2 * 2 + 1) + 16;
  e = allow_smem_fn(reinterpret_cast<const void*>(k_ffn_up_q4tc<NR, KB>), smem);
  if (e != cudaSuccess) return e;
  // up to nk / 32 shares of each of at most Fp / 128 row tiles (up_share, fit)
  const int grid = std::max(g, (Fp / TC_M) * std::max(1, nk / 32));
  (void)launch_dep(k_ffn_up_q4tc<NR, KB>, grid, 32 * TC_Q4_WARPS, smem, s, mx, cw0,
                   sw0, code_stride(PI_Q4_0, d, L.w_row_stride), scale_stride(d, L.w_row_stride),
                   static_cast<const char*>(L.w_up), static_cast<const char*>(L.w_up_scales),
                   code_stride(PI_Q4_0, d, ur), scale_stride(d, ur),
                   cc0, cc1, srb, d / 2, nt, nk, g, H, F, idx, count, sc.part, hdr);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  (void)launch_dep(k_ffn_finish<NR>, Fp / 64, 256, 0, s, sc.part, g, nk, 1, 0, H, F, Fp, nt, batch, idx,
                   count, L.bias, mask, (F + 31) / 32, sc.h16, hdr, L.act == PI_RELU2 ? 1 : 0);
  return cudaGetLastError();
}

}  // namespace

bool ffn_tc_supported(const pi_layer& L, int batch) {
  if (tc_disabled()) return false;
  if ((L.w_dtype != PI_F16 && L.w_dtype != PI_Q4_0) || batch < TC_MIN_BATCH || batch > TC_TMAX)
    return false;
  if (L.d_model % TC_M != 0) return false;
  // a host-memory cold tier: the Q4_0 kernels' loaders read its rows with
  // plain loads; the fp16 kernels' TMA loads read device memory only
  if (L.w_up_cold && L.w_dtype != PI_Q4_0) return false;
  if (L.w_dtype == PI_Q4_0) {
    // 16-byte code loads, 4-byte scale loads (two scales at a time)
    const int d = L.d_model;
    const int64_t ur = L.act == PI_REGLU && L.w_up_row_stride ? L.w_up_row_stride : L.w_row_stride;
    const int64_t cs[3] = {code_stride(PI_Q4_0, d, L.w_row_stride), code_stride(PI_Q4_0, d, ur),
                           code_stride(PI_Q4_0, d, L.w_down_row_stride)};
    const int64_t ss[3] = {scale_stride(d, L.w_row_stride), scale_stride(d, ur),
                           scale_stride(d, L.w_down_row_stride)};
    for (int k = 0; k < 3; ++k)
      if (cs[k] % 16 != 0 || ss[k] % 4 != 0) return false;
    const uintptr_t codes = (uintptr_t)L.w_up | (uintptr_t)L.w_down_t |
                            (uintptr_t)(L.act == PI_REGLU ? L.w_gate : L.w_up);
    const uintptr_t scales = (uintptr_t)L.w_up_scales | (uintptr_t)L.w_down_t_scales |
                             (uintptr_t)(L.act == PI_REGLU ? L.w_gate_scales : L.w_up_scales);
    if ((codes & 15u) || (scales & 3u)) return false;
    const uintptr_t ccodes = (uintptr_t)L.w_up_cold | (uintptr_t)L.w_down_t_cold |
                             (uintptr_t)L.w_gate_cold;
    const uintptr_t cscales = (uintptr_t)L.w_up_cold_scales | (uintptr_t)L.w_down_t_cold_scales |
                              (uintptr_t)L.w_gate_cold_scales;
    if ((ccodes & 15u) || (cscales & 3u)) return false;
    return tensor_map_encoder() != nullptr;
  }
  const int64_t rs = code_stride(PI_F16, L.d_model, L.w_row_stride);
  const int64_t rd = code_stride(PI_F16, L.d_model, L.w_down_row_stride);
  const int64_t ru = code_stride(PI_F16, L.d_model, L.w_up_row_stride ? L.w_up_row_stride
                                                                      : L.w_row_stride);
  if (rs % 16 != 0 || rd % 16 != 0 || ru % 16 != 0) return false;
  const uintptr_t bases = (uintptr_t)L.w_up | (uintptr_t)L.w_down_t |
                          (uintptr_t)(L.act == PI_REGLU ? L.w_gate : L.w_up);
  if (bases & 15u) return false;
  return tensor_map_encoder() != nullptr;
}

size_t tc_scratch_bytes(int d_model, int d_ff, int rank, int batch) {
  if (batch < TC_MIN_BATCH || d_model % TC_M != 0) return 0;
  return tc_scratch(nullptr, d_model, d_ff, rank).bytes;
}

bool pred_tc_supported(const pi_layer& L, int batch) {
  if (tc_disabled()) return false;
  if (L.p_dtype != PI_F16 || batch < TC_MIN_BATCH || batch > TC_TMAX) return false;
  if (L.rank % TC_M != 0 || L.d_model % TC_M != 0) return false;
  if (((uintptr_t)L.p1 | (uintptr_t)L.p2) & 15u) return false;
  return tensor_map_encoder() != nullptr;
}

void tc_split_buffers(const pi_layer& L, void* scratch, void** hi, void** lo) {
  const TcScratch sc = tc_scratch(scratch, L.d_model, L.d_ff, L.rank);
  *hi = sc.xh16;
  *lo = sc.xlo;
}

cudaError_t launch_predict_tc(const pi_layer& L, const float* xh, int batch, float theta,
                              uint32_t* mask, void* scratch, WsHeader* hdr, cudaStream_t s,
                              uint32_t* uni, bool split_ready) {
  const int d = L.d_model, r = L.rank, F = L.d_ff, H = L.hot, words = (F + 31) / 32;
  const int nt = (batch + 15) / 16 * 16;
  const TcScratch sc = tc_scratch(scratch, d, F, r);
  CUtensorMap m1, mxh, mxl, m2, muh, mul;
  if (!map_2d(&m1, L.p1, (uint64_t)d, (uint64_t)r, (uint64_t)d * 2, TC_M) ||
      !map_2d(&mxh, sc.xh16, (uint64_t)d, (uint64_t)nt, (uint64_t)d * 2, (uint32_t)nt) ||
      !map_2d(&mxl, sc.xlo, (uint64_t)d, (uint64_t)nt, (uint64_t)d * 2, (uint32_t)nt) ||
      !map_2d(&m2, L.p2, (uint64_t)r, (uint64_t)F, (uint64_t)r * 2, TC_M) ||
      !map_2d(&muh, sc.uhi, (uint64_t)r, (uint64_t)nt, (uint64_t)r * 2, (uint32_t)nt) ||
      !map_2d(&mul, sc.ulo, (uint64_t)r, (uint64_t)nt, (uint64_t)r * 2, (uint32_t)nt))
    return cudaErrorInvalidValue;
  const int grid = device_sms() * 4;
  cudaError_t e = cudaSuccess;
  if (!split_ready) {
    (void)launch_dep(k_split16, std::min((nt * d / 8 + 255) / 256, grid), 256, 0, s, xh, batch, d,
                     nt, sc.xh16, sc.xlo);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  constexpr uint32_t STAGE = TC_M * TC_BK * 2 + 2 * TC_TMAX * TC_BK * 2;
  const size_t smem = 1024 + (size_t)TC_PSTAGES * STAGE + 8 * (2 * TC_PSTAGES + 1) + 16;
  e = allow_smem_fn(reinterpret_cast<const void*>(k_pred_tc<0>), smem);
  if (e == cudaSuccess) e = allow_smem_fn(reinterpret_cast<const void*>(k_pred_tc<1>), smem);
  if (e != cudaSuccess) return e;
  // u = P1 xh
  const int ksu = pred_u_splits(d, r);
  (void)launch_dep(k_pred_tc<0>, dim3(r / TC_M, ksu), TC_THREADS, smem, s, m1, mxh, mxl, nt,
                   d / TC_BK, ksu, 0, r, sc.upart, nullptr, 0.f, 0, nullptr, 0, batch, hdr,
                   nullptr);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  (void)launch_dep(k_pred_u_finish, std::min((r / 4 * nt + 255) / 256, grid), 256, 0, s, sc.upart,
                   ksu, r, nt, batch, sc.uhi, sc.ulo);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  // z = P2 u + c for rows from the word holding `hot`; the words below it
  // are hot (written by the z kernel, or here when every row is hot)
  const int w0 = H / 32, row0 = 32 * w0;
  if (row0 < F) {
    const int tiles = (F - row0 + TC_M - 1) / TC_M;
    (void)launch_dep(k_pred_tc<1>, dim3(tiles, 1), TC_THREADS, smem, s, m2, muh, mul, nt, r / TC_BK,
                     1, row0, F, nullptr, L.p_bias, theta, H, mask, words, batch, hdr, uni);
    e = cudaGetLastError();
  } else {
    (void)launch_dep(k_hot_words, std::min((batch * w0 + 255) / 256, grid), 256, 0, s, mask, words,
                     w0, batch);
    e = cudaGetLastError();
  }
  return e;
}

// Columns per down tile, in units of 128: 256 where d_model / 256 tiles
// still fill the SMs with up to TC_KSMAX_D splits each (d_model >= 8192).
int down_ch(const pi_layer& L) {
  return (L.w_dtype == PI_F16 && L.d_model >= 8192 && L.d_model % 256 == 0) ? 2 : 1;
}

int ffn_tc_down_splits(const pi_layer& L) {
  // up to TC_KSMAX_D list shares per column tile, to fill two CTAs per SM
  int ks = 2 * device_sms() / (L.d_model / (TC_M * down_ch(L)));
  ks = ks < 1 ? 1 : (ks > TC_KSMAX_D ? TC_KSMAX_D : ks);
  const int nk = fpad(L.d_ff) / TC_BK;
  return ks > nk ? nk : ks;
}

cudaError_t launch_ffn_up_tc(const pi_layer& L, const float* xh, int batch, const uint32_t* mask,
                             const int32_t* idx, const int32_t* count, void* scratch,
                             WsHeader* hdr, cudaStream_t s, bool xh16_ready, char* stage) {
  if (L.w_dtype == PI_Q4_0)
    return L.act == PI_REGLU
               ? launch_up_q4<2>(L, xh, batch, mask, idx, count, scratch, hdr, s, xh16_ready, stage)
               : launch_up_q4<1>(L, xh, batch, mask, idx, count, scratch, hdr, s, xh16_ready, stage);
  return L.act == PI_REGLU
             ? launch_up_nr<2>(L, xh, batch, mask, idx, count, scratch, hdr, s, xh16_ready)
             : launch_up_nr<1>(L, xh, batch, mask, idx, count, scratch, hdr, s, xh16_ready);
}

size_t tc_cold_stage_bytes(const pi_layer& L) {
  if (!L.w_up_cold || L.w_dtype != PI_Q4_0) return 0;
  return (size_t)(L.d_ff - L.hot) * (size_t)stage_row_bytes(PI_Q4_0, L.d_model) *
         (L.act == PI_REGLU ? 3u : 2u);
}

cudaError_t launch_ffn_down_tc(const pi_layer& L, int batch, const int32_t* idx,
                               const int32_t* count, float* part, void* scratch, WsHeader* hdr,
                               cudaStream_t s, char* cold_stage) {
  const int d = L.d_model, H = L.hot, F = L.d_ff, Fp = fpad(F);
  const int nt = (batch + 15) / 16 * 16;
  const TcScratch sc = tc_scratch(scratch, d, F, L.rank);
  if (L.w_dtype == PI_Q4_0) {
    CUtensorMap mh;
    if (!map_2d(&mh, sc.h16, (uint64_t)TC_BK, (uint64_t)(Fp / TC_BK) * nt, (uint64_t)TC_BK * 2,
                (uint32_t)nt))
      return cudaErrorInvalidValue;
    const int tiles = d / TC_M, ks = ffn_tc_down_splits(L);
    const uint32_t stage = 2 * 64 * TC_BK * 2 + (((uint32_t)nt * TC_BK * 2 + 1023u) & ~1023u);
    const size_t smem = 1024 + 4 * (size_t)stage + 8 * (2 * 4 + 1) + 16;
    cudaError_t e = allow_smem_fn(reinterpret_cast<const void*>(k_ffn_down_q4tc), smem);
    if (e != cudaSuccess) return e;
    // a host-memory cold tier: every listed down row, once, into the stage
    // behind the up kernel's (the kernel reads every listed position)
    const int64_t srb = stage_row_bytes(PI_Q4_0, d);
    char* cwc = nullptr;
    if (L.w_up_cold) {
      if (!cold_stage) return cudaErrorInvalidValue;
      cwc = cold_stage + (size_t)(F - H) * srb * (L.act == PI_REGLU ? 2u : 1u);
      if ((e = launch_stage_cold_down(L, batch, idx, count, nullptr, cwc, hdr, s)) != cudaSuccess)
        return e;
    }
    (void)launch_dep(k_ffn_down_q4tc, dim3(tiles, ks), 32 * TC_Q4_WARPS, smem, s, mh,
                     static_cast<const char*>(L.w_down_t),
                     static_cast<const char*>(L.w_down_t_scales),
                     code_stride(PI_Q4_0, d, L.w_down_row_stride),
                     scale_stride(d, L.w_down_row_stride),
                     cwc, srb, d / 2, nt, ks, d, batch, H, F, idx, count, part, hdr);
    return cudaGetLastError();
  }
  const int64_t rd = code_stride(PI_F16, d, L.w_down_row_stride);
  CUtensorMap mwd, mwg, mh;
  if (!map_2d(&mwd, L.w_down_t, (uint64_t)d, (uint64_t)F, (uint64_t)rd, TC_BK) ||
      !map_2d(&mwg, L.w_down_t, (uint64_t)d, (uint64_t)F, (uint64_t)rd, 1) ||
      !map_2d(&mh, sc.h16, (uint64_t)TC_BK, (uint64_t)(Fp / TC_BK) * nt, (uint64_t)TC_BK * 2,
              (uint32_t)nt))
    return cudaErrorInvalidValue;
  const int ch = down_ch(L), ds = ch == 1 ? TC_STAGES : 2;
  const int tiles = d / (TC_M * ch), nk = Fp / TC_BK, ks = ffn_tc_down_splits(L);
  const uint32_t stage = 2 * ch * 64 * TC_BK * 2 + TC_TMAX * TC_BK * 2;
  const size_t smem = 1024 + (size_t)ds * stage + 8 * (2 * ds + 1) + 16;
  auto kern = ch == 2 ? k_ffn_down_tc<2> : k_ffn_down_tc<1>;
  cudaError_t e = allow_smem_fn(reinterpret_cast<const void*>(kern), smem);
  if (e != cudaSuccess) return e;
  (void)launch_dep(kern, dim3(tiles, ks), 32 * TC_FFN_WARPS, smem, s, mwd, mwg, mh, nt, nk, ks, d,
                   batch, H, F, idx, count, part, hdr);
  return cudaGetLastError();
}

}  // namespace pi
