// Decode-batch kernels (T <= 16 tokens, bf16) of the DECO MoE layer.
//
// At a few tokens the layer is bound by HBM: every weight byte is used by at
// most 16 tokens, and only the routed experts that some token activates need
// to be read (the paper's point about sparse activation saving memory access,
// "DECO: Sparse Mixture-of-Experts with Dense-Comparable Performance on
// End-Side Devices", §1 and §5).  The three kernels therefore stream weights:
//
//   kd_route  rows [W_r ; W_bar_up ; W_s_up]  -> r, active, u, SiLU(shared up)
//   kd_up     rows of W_up[e] for the union of active experts -> centred
//             activations c = g - u; the CTA that completes an expert applies
//             NormSiLU's RMS normalisation and SiLU to that expert's tokens
//   kd_down   each CTA owns a block of output rows and walks the shared
//             expert, then the active experts in ascending order, so every
//             output element is summed in one fixed order (no atomics)
//
// Every kernel runs one CTA per SM with 8 consumer warps and 1 producer warp.
// The producer streams the CTA's weight rows into a ring of 32 KB shared-memory
// stages with cp.async.bulk (evict-first in L2), signalled by mbarriers; the
// consumers compute from shared memory.  Rows are split evenly over the CTAs.
// Waits are bounded: after ~1 s a wait gives up, sets bit 2 of the device
// error word and the CTA stops issuing work (no hang, no trap).
// Consecutive kernels use programmatic dependent launch: a kernel starts
// while its predecessor drains and waits (griddepcontrol.wait) only before it
// reads what the predecessor wrote.
#pragma once

#include "common.cuh"

namespace deco {
namespace dec {

constexpr int kConsumerWarps = 8;
constexpr int kThreads = (kConsumerWarps + 1) * 32;
constexpr int kMaxT = 16;                      // decode batches
constexpr uint32_t kStageBytes = 32768;
constexpr int kMaxStages = 8;
constexpr size_t kSmemLimit = 232448;          // 227 KB opt-in per CTA on sm_100
constexpr long long kWaitCycles = 2000000000ll;  // ~1 s at 1.9 GHz
constexpr int kErrTimeout = 2;

// ---------------------------------------------------------------------------
// PTX wrappers

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait for the phase with `parity` to complete.  Returns false (and
// flags the CTA-wide abort word and the device error word) on timeout.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                          int* err) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (*abort_flag) return false;
    if (clock64() - t0 > kWaitCycles) {
      *abort_flag = 1;
      atomicOr(err, kErrTimeout);
      return false;
    }
  }
  return true;
}
__device__ __forceinline__ uint64_t evict_first_policy() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}
// global -> shared bulk copy completing on `bar` (bytes and addresses 16-B multiples)
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar,
                                         uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1], %2, [%3], %4;" ::"r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" :::); }

__device__ __forceinline__ void bf16x8_to_f32(const uint4& q, float (&v)[8]) { unpack16(q, v); }

// ---------------------------------------------------------------------------
// Ring of weight stages shared by the three kernels.

struct Ring {
  uint64_t* full;    // [kMaxStages]
  uint64_t* empty;   // [kMaxStages]
  unsigned char* stage;
  uint32_t stage_bytes;
  int nstages;
};

// dynamic shared memory layout: [barriers 256 B][ring stages][kernel operand];
// kStaticReserve bytes are left for each kernel's static __shared__ arrays.
constexpr uint32_t kHeaderBytes = 256;
constexpr uint32_t kStaticReserve = 1536;

struct SmemPlan {
  uint32_t ring_off, op_off, total, stage_bytes;
  int nstages;
};

__host__ __device__ inline SmemPlan smem_plan(uint32_t operand_bytes, uint32_t stage_bytes) {
  SmemPlan p;
  p.ring_off = kHeaderBytes;
  p.stage_bytes = stage_bytes;
  const uint32_t room = (uint32_t)kSmemLimit - kStaticReserve - kHeaderBytes -
                        ((operand_bytes + 127) & ~127u);
  p.nstages = (int)(room / stage_bytes);
  if (p.nstages > kMaxStages) p.nstages = kMaxStages;
  p.op_off = p.ring_off + p.nstages * stage_bytes;
  p.total = p.op_off + ((operand_bytes + 127) & ~127u);
  return p;
}

// barriers: full[8], empty[8], opbar, abort word (136 B of the 256 B header)
__device__ __forceinline__ void ring_setup(unsigned char* smem, const SmemPlan& sp, Ring& ring,
                                           uint64_t*& opbar, volatile int*& abort_flag) {
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem);
  ring.full = bars;
  ring.empty = bars + kMaxStages;
  opbar = bars + 2 * kMaxStages;
  abort_flag = reinterpret_cast<volatile int*>(bars + 2 * kMaxStages + 1);
  ring.stage = smem + sp.ring_off;
  ring.stage_bytes = sp.stage_bytes;
  ring.nstages = sp.nstages;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kMaxStages; ++s) {
      mbar_init(&ring.full[s], 1);
      mbar_init(&ring.empty[s], kConsumerWarps);
    }
    mbar_init(opbar, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
}

// ---------------------------------------------------------------------------

struct Args {
  int T, D, E, d_e, d_s;
  float eps;
  int residual;
  const bf16* x;
  const bf16* W_r;
  const float* b_r;
  const bf16* W_bar;
  const bf16* W_up;
  const bf16* W_down;
  const float* s;
  const bf16* W_s_up;
  const bf16* W_s_down;
  float* r;         // [T][E]
  uint8_t* act;     // [T][E]
  float* u;         // [T][d_e]
  bf16* hs;         // [T][d_s]   SiLU(x W_s_up^T)
  float* C;         // [T][E][d_e] centred up-projection
  bf16* A;          // [T][E][d_e] NormSiLU output
  int* done;        // [E] rows of each expert finished by kd_up
  int* err;
  bf16* out;
  uint32_t down_stage;   // kd_down ring stage bytes (>= one expert's weights + activations)
};

// per-expert token masks and the ascending list of experts some token uses
__device__ __forceinline__ void build_union(const Args& a, uint16_t* emask, uint8_t* ulist, int* U) {
  for (int e = threadIdx.x; e < a.E; e += blockDim.x) {
    uint16_t m = 0;
    for (int t = 0; t < a.T; ++t)
      if (__ldcg(a.act + (size_t)t * a.E + e)) m |= (uint16_t)(1u << t);
    emask[e] = m;
  }
  __syncthreads();
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    int n = 0;
    for (int base = 0; base < a.E; base += 32) {
      const int e = base + lane;
      const bool f = e < a.E && emask[e] != 0;
      const unsigned bal = __ballot_sync(kFull, f);
      if (f) ulist[n + __popc(bal & ((1u << lane) - 1u))] = (uint8_t)e;
      n += __popc(bal);
    }
    if (lane == 0) *U = n;
  }
  __syncthreads();
}

// Reduce N = 2^m per-lane values across the warp in 31-ish shuffles instead of
// 5 per value: at each of the first m levels a lane keeps one half of its
// values, sends the other half to its partner and adds what it receives;
// the remaining 5 - m levels are plain butterflies.  Afterwards lane l holds
// the warp total of value index (l >> (5 - m)) & (N - 1); every total is a
// fixed-shape tree over the 32 lane partials (depth 5), so it is
// deterministic and its rounding is that of a 5-level pairwise sum.
template <int N>
__device__ __forceinline__ float warp_reduce_scatter(float (&v)[N], int lane) {
  static_assert(N >= 1 && N <= 32 && (N & (N - 1)) == 0, "N must be a power of two <= 32");
  int c = N;
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    if (c > 1) {
      const int h = c >> 1;
      const bool upper = (lane & o) != 0;
#pragma unroll
      for (int i = 0; i < N / 2; ++i) {
        if (i < h) {
          const float send = upper ? v[i] : v[i + h];
          const float keep = upper ? v[i + h] : v[i];
          v[i] = keep + __shfl_xor_sync(kFull, send, o);
        }
      }
      c = h;
    } else {
      v[0] += __shfl_xor_sync(kFull, v[0], o);
    }
  }
  return v[0];
}

constexpr int kMaxChunks = 16;   // D <= 4096 bf16: D/256 chunks of 8 per lane

// load this lane's chunks (lane + 32 i, 8 bf16 each) of a row in shared memory
__device__ __forceinline__ void load_row_chunks(const bf16* row, int nc, int lane, uint4 (&w)[kMaxChunks]) {
#pragma unroll
  for (int i = 0; i < kMaxChunks; ++i)
    if (i < nc) w[i] = *reinterpret_cast<const uint4*>(row + (size_t)(lane + 32 * i) * 8);
}

// Partial dot products of one row (chunks in registers) with the token rows of
// xs[16][D] selected by `tmask`; each lane sums its terms in chunk order.
template <bool ABS>
__device__ __forceinline__ void row_token_partials(const uint4 (&w)[kMaxChunks], int nc, const bf16* xs,
                                                   int D, uint32_t tmask, int lane, float (&acc)[16],
                                                   float (&aacc)[16]) {
#pragma unroll
  for (int t = 0; t < 16; ++t) {
    acc[t] = 0.f;
    aacc[t] = 0.f;
  }
#pragma unroll
  for (int i = 0; i < kMaxChunks; ++i) {
    if (i < nc) {
      float wv[8];
      bf16x8_to_f32(w[i], wv);
#pragma unroll
      for (int t = 0; t < 16; ++t) {
        if ((tmask >> t) & 1u) {
          float xv[8];
          bf16x8_to_f32(*reinterpret_cast<const uint4*>(xs + (size_t)t * D + (size_t)(lane + 32 * i) * 8), xv);
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            acc[t] = fmaf(xv[k], wv[k], acc[t]);
            if (ABS) aacc[t] = fmaf(fabsf(xv[k]), fabsf(wv[k]), aacc[t]);
          }
        }
      }
    }
  }
}

// ---------------------------------------------------------------------------
// kd_route

__global__ void __launch_bounds__(kThreads, 1) kd_route(Args a) {
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ unsigned long long limbs[kConsumerWarps][kLimbs];   // 1280 B <= kStaticReserve
  const uint32_t xbytes = (uint32_t)a.T * a.D * 2;
  const SmemPlan sp = smem_plan(xbytes, kStageBytes);
  Ring ring;
  uint64_t* xbar;
  volatile int* abort_flag;
  ring_setup(smem, sp, ring, xbar, abort_flag);
  const bf16* xs = reinterpret_cast<const bf16*>(smem + sp.op_off);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  pdl_trigger();
  if (blockIdx.x == 0)
    for (int e = threadIdx.x; e < a.E; e += blockDim.x) a.done[e] = 0;

  const int Ntot = a.E + a.d_e + a.d_s;
  const int Q = (Ntot + gridDim.x - 1) / gridDim.x;
  const int g0 = min(Ntot, (int)blockIdx.x * Q), g1 = min(Ntot, g0 + Q);
  const int rowbytes = a.D * 2;
  const int RPS = min(kConsumerWarps, (int)(kStageBytes / rowbytes));
  const int WPR = kConsumerWarps / RPS;
  auto seg_end = [&](int g) { return g < a.E ? a.E : (g < a.E + a.d_e ? a.E + a.d_e : Ntot); };
  auto row_ptr = [&](int g) -> const bf16* {
    if (g < a.E) return a.W_r + (size_t)g * a.D;
    if (g < a.E + a.d_e) return a.W_bar + (size_t)(g - a.E) * a.D;
    return a.W_s_up + (size_t)(g - a.E - a.d_e) * a.D;
  };

  if (warp == kConsumerWarps) {
    if (lane == 0 && g0 < g1) {
      const uint64_t pol = evict_first_policy();
      mbar_expect_tx(xbar, xbytes);
      bulk_g2s(smem + sp.op_off, a.x, xbytes, xbar);
      int k = 0;
      for (int g = g0; g < g1; ++k) {
        const int n = min(RPS, min(g1, seg_end(g)) - g);
        const int s = k % ring.nstages;
        if (!mbar_wait(&ring.empty[s], ((k / ring.nstages) & 1) ^ 1, abort_flag, a.err)) break;
        mbar_expect_tx(&ring.full[s], n * rowbytes);
        bulk_g2s(ring.stage + (size_t)s * ring.stage_bytes, row_ptr(g), n * rowbytes, &ring.full[s], pol);
        g += n;
      }
    }
    return;
  }

  const int nc = a.D / 256;
  const int n_terms = a.D / 32 + 6;
  const float gm = gamma_f32(n_terms);
  const float bscale = 2.f * gm * (1.f + 2.f * gm);
  const float tiny = float(n_terms) * 2.8025969e-45f;
  const uint32_t all_t = (a.T >= 32) ? 0xffffffffu : ((1u << a.T) - 1u);
  bool bad = false;
  // the activation copy is issued iff this CTA has rows; it is always awaited
  const bool x_ok = g0 < g1 && mbar_wait(xbar, 0, abort_flag, a.err);
  int k = 0;
  for (int g = g0; x_ok && g < g1; ++k) {
    const int n = min(RPS, min(g1, seg_end(g)) - g);
    const int s = k % ring.nstages;
    if (!mbar_wait(&ring.full[s], (k / ring.nstages) & 1, abort_flag, a.err)) break;
    const int rs = warp / WPR, sub = warp % WPR;
    if (rs < n) {
      const int row = g + rs;
      const bf16* wrow =
          reinterpret_cast<const bf16*>(ring.stage + (size_t)s * ring.stage_bytes + (size_t)rs * rowbytes);
      uint4 w[kMaxChunks];
      load_row_chunks(wrow, nc, lane, w);
      // with two warps per row each takes every other token
      const uint32_t tm = all_t & (WPR == 1 ? 0xffffffffu : (sub ? 0xaaaaaaaau : 0x55555555u));
      float acc[16], aacc[16];
      if (row < a.E) {
        const int e = row;
        row_token_partials<true>(w, nc, xs, a.D, tm, lane, acc, aacc);
        float v[32];
#pragma unroll
        for (int t = 0; t < 16; ++t) {
          v[t] = acc[t];
          v[16 + t] = aacc[t];
        }
        const float tot = warp_reduce_scatter<32>(v, lane);   // lane l: value l
        const float S = __shfl_sync(kFull, tot, (lane + 16) & 31);
        const float b = a.b_r[e];
        const int t = lane;
        const bool mine = t < 16 && ((tm >> t) & 1u);
        const float z = tot + b;
        const float B = bscale * (S + fabsf(b)) + tiny;
        const bool sure = fabsf(z) > B;
        bool on = sure && z > 0.f;
        // guard band: exact re-evaluation of the sign, one whole warp per score
        unsigned need = __ballot_sync(kFull, mine && !sure);
        while (need) {
          const int tt = __ffs(need) - 1;
          need &= need - 1;
          const int sg = exact_sign_warp(xs + (size_t)tt * a.D, wrow, a.D, b, limbs[warp], &bad);
          if (lane == tt) on = sg > 0;
        }
        if (mine) {
          a.r[(size_t)t * a.E + e] = on ? fmaxf(z, 0.f) : 0.f;
          a.act[(size_t)t * a.E + e] = on ? 1 : 0;
        }
      } else {
        row_token_partials<false>(w, nc, xs, a.D, tm, lane, acc, aacc);
        const float tot = warp_reduce_scatter<16>(acc, lane);   // lane l: token l >> 1
        const int t = lane >> 1;
        if ((lane & 1) == 0 && ((tm >> t) & 1u)) {
          if (row < a.E + a.d_e)
            a.u[(size_t)t * a.d_e + (row - a.E)] = tot;
          else
            a.hs[(size_t)t * a.d_s + (row - a.E - a.d_e)] = __float2bfloat16_rn(silu_f(tot));
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&ring.empty[s]);
    g += n;
  }
  if (bad && lane == 0) atomicOr(a.err, 1);
}

// ---------------------------------------------------------------------------
// kd_up

__global__ void __launch_bounds__(kThreads, 1) kd_up(Args a) {
  extern __shared__ __align__(128) unsigned char smem[];
  // static shared memory stays within kStaticReserve
  __shared__ uint16_t emask[256];
  __shared__ uint8_t ulist[256];
  __shared__ int s_U;
  __shared__ int touched_e[32], touched_n[32];
  __shared__ int n_touched, fin[32], n_fin;
  const uint32_t xbytes = (uint32_t)a.T * a.D * 2;
  const SmemPlan sp = smem_plan(xbytes, kStageBytes);
  Ring ring;
  uint64_t* xbar;
  volatile int* abort_flag;
  ring_setup(smem, sp, ring, xbar, abort_flag);
  const bf16* xs = reinterpret_cast<const bf16*>(smem + sp.op_off);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    n_touched = 0;
    n_fin = 0;
    // x does not depend on the router: stage it before waiting for it
    mbar_expect_tx(xbar, xbytes);
    bulk_g2s(smem + sp.op_off, a.x, xbytes, xbar);
  }
  pdl_wait();          // router outputs (act, u) and the zeroed counters
  pdl_trigger();
  build_union(a, emask, ulist, &s_U);
  const int U = s_U;
  const int Ntot = U * a.d_e;
  const int Q = (Ntot + gridDim.x - 1) / gridDim.x;
  const int g0 = min(Ntot, (int)blockIdx.x * Q), g1 = min(Ntot, g0 + Q);
  const int rowbytes = a.D * 2;
  const int RPS = min(kConsumerWarps, (int)(kStageBytes / rowbytes));
  const int WPR = kConsumerWarps / RPS;

  if (warp == kConsumerWarps) {
    if (lane == 0) {
      const uint64_t pol = evict_first_policy();
      int k = 0;
      for (int g = g0; g < g1; ++k) {
        const int e = ulist[g / a.d_e], j = g % a.d_e;
        const int n = min(RPS, min(g1 - g, a.d_e - j));
        const int s = k % ring.nstages;
        if (!mbar_wait(&ring.empty[s], ((k / ring.nstages) & 1) ^ 1, abort_flag, a.err)) break;
        mbar_expect_tx(&ring.full[s], n * rowbytes);
        bulk_g2s(ring.stage + (size_t)s * ring.stage_bytes, a.W_up + ((size_t)e * a.d_e + j) * a.D,
                 n * rowbytes, &ring.full[s], pol);
        g += n;
      }
    }
  } else {
    const int nc = a.D / 256;
    // the activation copy was issued unconditionally: always await it
    const bool x_ok = mbar_wait(xbar, 0, abort_flag, a.err);
    int k = 0;
    for (int g = g0; x_ok && g < g1; ++k) {
      const int e = ulist[g / a.d_e], j = g % a.d_e;
      const int n = min(RPS, min(g1 - g, a.d_e - j));
      const int s = k % ring.nstages;
      if (threadIdx.x == 0) {
        if (n_touched > 0 && touched_e[n_touched - 1] == e) {
          touched_n[n_touched - 1] += n;
        } else if (n_touched < 32) {
          touched_e[n_touched] = e;
          touched_n[n_touched] = n;
          ++n_touched;
        }
      }
      if (!mbar_wait(&ring.full[s], (k / ring.nstages) & 1, abort_flag, a.err)) break;
      const int rs = warp / WPR, sub = warp % WPR;
      if (rs < n) {
        const int jr = j + rs;
        const bf16* wrow =
            reinterpret_cast<const bf16*>(ring.stage + (size_t)s * ring.stage_bytes + (size_t)rs * rowbytes);
        uint4 w[kMaxChunks];
        load_row_chunks(wrow, nc, lane, w);
        const uint32_t tm =
            (uint32_t)emask[e] & (WPR == 1 ? 0xffffffffu : (sub ? 0xaaaaaaaau : 0x55555555u));
        float acc[16], aacc[16];
        row_token_partials<false>(w, nc, xs, a.D, tm, lane, acc, aacc);
        const float tot = warp_reduce_scatter<16>(acc, lane);   // lane l: token l >> 1
        const int t = lane >> 1;
        if ((lane & 1) == 0 && ((tm >> t) & 1u)) a.C[((size_t)t * a.E + e) * a.d_e + jr] = tot;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&ring.empty[s]);
      g += n;
    }
  }
  // publish this CTA's rows; the CTA completing an expert normalises it
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0 && !*abort_flag) {
    for (int i = 0; i < n_touched; ++i) {
      const int e = touched_e[i];
      const int old = atomicAdd(a.done + e, touched_n[i]);
      if (old + touched_n[i] == a.d_e) fin[n_fin++] = e;
    }
  }
  __syncthreads();
  if (warp >= kConsumerWarps) return;
  __threadfence();
  const float inv_de = 1.f / float(a.d_e);
  int item = 0;
  for (int f = 0; f < n_fin; ++f) {
    const int e = fin[f];
    for (uint32_t m = emask[e]; m; m &= m - 1, ++item) {
      if (item % kConsumerWarps != warp) continue;
      const int t = __ffs(m) - 1;
      const float* gr = a.C + ((size_t)t * a.E + e) * a.d_e;
      const float* ur = a.u + (size_t)t * a.d_e;
      float cv[16];   // d_e <= 512: 16 per lane
      float ss = 0.f;
#pragma unroll
      for (int q = 0; q < 16; ++q) {
        const int jj = lane + 32 * q;
        cv[q] = 0.f;
        if (jj < a.d_e) {
          cv[q] = __ldcg(gr + jj) - __ldcg(ur + jj);   // c = g - u
          ss = fmaf(cv[q], cv[q], ss);
        }
      }
      ss = warp_sum(ss);
      const float rinv = 1.f / sqrtf(ss * inv_de + a.eps);
      bf16* ao = a.A + ((size_t)t * a.E + e) * a.d_e;
#pragma unroll
      for (int q = 0; q < 16; ++q) {
        const int jj = lane + 32 * q;
        if (jj < a.d_e) ao[jj] = __float2bfloat16_rn(silu_f(cv[q] * rinv));
      }
    }
  }
}

// ---------------------------------------------------------------------------
// kd_down
//
// The CTA's work is a sequence of units: pieces of W_s_down[n0:n1][:] (the
// shared expert) and then, for each active expert e in ascending order,
// [W_down[e][n0:n1][:] | A[t][e][:] for its active tokens t, ascending].
// Consecutive units are packed greedily into ring stages of a.down_stage
// bytes; producer and consumers compute the same packing.

struct DownUnits {
  int n0, n1, srows, nshared, nunits;
  uint32_t wbytes, abytes_row;
};

__device__ __forceinline__ uint32_t unit_bytes(const Args& a, const DownUnits& du, const uint16_t* emask,
                                               const uint8_t* ulist, int u) {
  if (u < du.nshared) {
    const int m0 = du.n0 + u * du.srows, m1 = min(du.n1, m0 + du.srows);
    return (uint32_t)(m1 - m0) * a.d_s * 2;
  }
  return du.wbytes + __popc(emask[ulist[u - du.nshared]]) * du.abytes_row;
}

// end of the stage that starts at unit u (at least one unit per stage)
__device__ __forceinline__ int stage_end(const Args& a, const DownUnits& du, const uint16_t* emask,
                                         const uint8_t* ulist, int u, uint32_t cap) {
  uint32_t used = unit_bytes(a, du, emask, ulist, u);
  int v = u + 1;
  while (v < du.nunits) {
    const uint32_t b = unit_bytes(a, du, emask, ulist, v);
    if (used + b > cap) break;
    used += b;
    ++v;
  }
  return v;
}

__global__ void __launch_bounds__(kThreads, 1) kd_down(Args a) {
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ uint16_t emask[256];
  __shared__ uint8_t ulist[256];
  __shared__ int s_U;
  const uint32_t hbytes = (uint32_t)a.T * a.d_s * 2;
  const uint32_t rbytes = (uint32_t)a.T * a.E * 4;     // r staged next to hs
  const uint32_t hpad = (hbytes + 127) & ~127u;
  const SmemPlan sp = smem_plan(hpad + rbytes, a.down_stage);
  Ring ring;
  uint64_t* hbar;
  volatile int* abort_flag;
  ring_setup(smem, sp, ring, hbar, abort_flag);
  const bf16* hsm = reinterpret_cast<const bf16*>(smem + sp.op_off);
  float* r_s = reinterpret_cast<float*>(smem + sp.op_off + hpad);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // The router's outputs are complete: this grid starts only after every CTA
  // of kd_up passed its own wait on the router.
  build_union(a, emask, ulist, &s_U);
  for (int i = threadIdx.x; i < a.T * a.E; i += blockDim.x) r_s[i] = __ldcg(a.r + i);
  __syncthreads();
  DownUnits du;
  du.n0 = (int)(((long long)blockIdx.x * a.D) / gridDim.x);
  du.n1 = (int)(((long long)(blockIdx.x + 1) * a.D) / gridDim.x);
  const int R = du.n1 - du.n0;
  du.srows = max(1, (int)(a.down_stage / (a.d_s * 2)));
  du.nshared = (R + du.srows - 1) / du.srows;
  du.nunits = du.nshared + s_U;
  du.wbytes = (uint32_t)R * a.d_e * 2;
  du.abytes_row = (uint32_t)a.d_e * 2;
  const int n0 = du.n0, n1 = du.n1;

  if (warp == kConsumerWarps) {
    if (lane == 0) {
      const uint64_t pol = evict_first_policy();
      mbar_expect_tx(hbar, hbytes);
      bulk_g2s(smem + sp.op_off, a.hs, hbytes, hbar);
      // weights of stage k; activations are issued separately (after kd_up)
      auto issue_w = [&](int u0, int u1, int s) {
        unsigned char* st = ring.stage + (size_t)s * ring.stage_bytes;
        uint32_t total = 0;
        for (int u = u0; u < u1; ++u) total += unit_bytes(a, du, emask, ulist, u);
        mbar_expect_tx(&ring.full[s], total);
        uint32_t off = 0;
        for (int u = u0; u < u1; ++u) {
          if (u < du.nshared) {
            const int m0 = n0 + u * du.srows, m1 = min(n1, m0 + du.srows);
            const uint32_t bytes = (uint32_t)(m1 - m0) * a.d_s * 2;
            bulk_g2s(st + off, a.W_s_down + (size_t)m0 * a.d_s, bytes, &ring.full[s], pol);
          } else {
            const int e = ulist[u - du.nshared];
            bulk_g2s(st + off, a.W_down + ((size_t)e * a.D + n0) * a.d_e, du.wbytes, &ring.full[s], pol);
          }
          off += unit_bytes(a, du, emask, ulist, u);
        }
      };
      auto issue_a = [&](int u0, int u1, int s) {   // activations written by kd_up
        unsigned char* st = ring.stage + (size_t)s * ring.stage_bytes;
        uint32_t off = 0;
        for (int u = u0; u < u1; ++u) {
          if (u >= du.nshared) {
            const int e = ulist[u - du.nshared];
            int slot = 0;
            for (uint32_t m = emask[e]; m; m &= m - 1, ++slot) {
              const int t = __ffs(m) - 1;
              bulk_g2s(st + off + du.wbytes + (size_t)slot * du.abytes_row,
                       a.A + ((size_t)t * a.E + e) * a.d_e, du.abytes_row, &ring.full[s]);
            }
          }
          off += unit_bytes(a, du, emask, ulist, u);
        }
      };
      // weights of the first stages go out before kd_up has finished ...
      int u = 0, k = 0;
      int first_u[kMaxStages + 1];
      for (; u < du.nunits && k < ring.nstages; ++k) {
        const int v = stage_end(a, du, emask, ulist, u, ring.stage_bytes);
        first_u[k] = u;
        issue_w(u, v, k);
        u = v;
      }
      first_u[k] = u;
      pdl_wait();
      // ... their activations only once it has
      for (int q = 0; q < k; ++q) issue_a(first_u[q], first_u[q + 1], q);
      for (; u < du.nunits; ++k) {
        const int v = stage_end(a, du, emask, ulist, u, ring.stage_bytes);
        const int s = k % ring.nstages;
        if (!mbar_wait(&ring.empty[s], ((k / ring.nstages) & 1) ^ 1, abort_flag, a.err)) break;
        issue_w(u, v, s);
        issue_a(u, v, s);
        u = v;
      }
    }
    return;
  }

  // consumer warp w owns rows n0 + w + 8q, q < 4; a row pair (q, q+1) and the
  // 16 token slots make 32 partial sums reduced together, lane l ending with
  // row (l >> 4) of the pair and token (l & 15)
  float acc[2] = {0.f, 0.f};
  const int my_t = lane & 15;
  const bool ok = mbar_wait(hbar, 0, abort_flag, a.err);
  int k = 0;
  for (int u0 = 0; ok && u0 < du.nunits; ++k) {
    const int u1 = stage_end(a, du, emask, ulist, u0, ring.stage_bytes);
    const int s = k % ring.nstages;
    if (!mbar_wait(&ring.full[s], (k / ring.nstages) & 1, abort_flag, a.err)) break;
    const unsigned char* st = ring.stage + (size_t)s * ring.stage_bytes;
    uint32_t off = 0;
    for (int u = u0; u < u1; ++u) {
      const bool shared = u < du.nshared;
      const int m0 = shared ? n0 + u * du.srows : n0;
      const int m1 = shared ? min(n1, m0 + du.srows) : n1;
      const int K = shared ? a.d_s : a.d_e;
      const int e = shared ? -1 : ulist[u - du.nshared];
      const uint32_t tmask = shared ? ((1u << a.T) - 1u) : (uint32_t)emask[e];
      const bf16* wbase = reinterpret_cast<const bf16*>(st + off);
      const bf16* act_base = shared ? hsm : reinterpret_cast<const bf16*>(st + off + du.wbytes);
#pragma unroll
      for (int qp = 0; qp < 2; ++qp) {
        const int ra = n0 + warp + 16 * qp, rb = ra + 8;   // the pair's two rows
        const bool has_a = ra >= m0 && ra < m1, has_b = rb >= m0 && rb < m1;
        if (!(has_a || has_b)) continue;
        float v[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = 0.f;
        const bf16* wa = wbase + (size_t)(ra - m0) * K;
        const bf16* wb = wbase + (size_t)(rb - m0) * K;
        for (int c = lane; c < K / 8; c += 32) {
          float fa[8], fb[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) fa[i] = fb[i] = 0.f;
          if (has_a) bf16x8_to_f32(*reinterpret_cast<const uint4*>(wa + (size_t)c * 8), fa);
          if (has_b) bf16x8_to_f32(*reinterpret_cast<const uint4*>(wb + (size_t)c * 8), fb);
          int slot = 0;
#pragma unroll
          for (int t = 0; t < 16; ++t) {
            if ((tmask >> t) & 1u) {
              const bf16* av = act_base + (size_t)(shared ? t : slot) * K;
              float hv[8];
              bf16x8_to_f32(*reinterpret_cast<const uint4*>(av + (size_t)c * 8), hv);
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                v[t] = fmaf(fa[i], hv[i], v[t]);
                v[16 + t] = fmaf(fb[i], hv[i], v[16 + t]);
              }
              ++slot;
            }
          }
        }
        const float tot = warp_reduce_scatter<32>(v, lane);   // lane l: value l
        const bool mine_row = (lane < 16) ? has_a : has_b;
        if (mine_row && ((tmask >> my_t) & 1u)) {
          if (shared)
            acc[qp] += tot;
          else
            acc[qp] = fmaf(a.s[e] * r_s[my_t * a.E + e], tot, acc[qp]);
        }
      }
      off += unit_bytes(a, du, emask, ulist, u);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&ring.empty[s]);
    u0 = u1;
  }
  if (my_t < a.T && !*abort_flag) {
#pragma unroll
    for (int qp = 0; qp < 2; ++qp) {
      const int m = n0 + warp + 16 * qp + (lane >= 16 ? 8 : 0);
      if (m >= n1) continue;
      float val = acc[qp];
      if (a.residual) val += __bfloat162float(a.x[(size_t)my_t * a.D + m]);
      a.out[(size_t)my_t * a.D + m] = __float2bfloat16_rn(val);
    }
  }
}

}  // namespace dec
}  // namespace deco
