// Decode-batch kernels (T <= 16 tokens, bf16) of the DECO MoE layer.
//
// At a few tokens the layer is bound by HBM: every weight byte is used by at
// most 16 tokens, and only the routed experts that some token activates need
// to be read (the paper's point about sparse activation saving memory access,
// "DECO: Sparse Mixture-of-Experts with Dense-Comparable Performance on
// End-Side Devices", §1 and §5).  Three kernels stream the weights once and
// a fourth adds the partial results:
//
//   kd_route  router rows W_r (exact activation decisions, CUDA cores), and
//             the mean up-projection W_bar_up and shared up-projection W_s_up
//             (tensor cores) -> r, active, u = x W_bar_up^T, SiLU(x W_s_up^T)
//   kd_up     W_up[e] of the union of active experts (tensor cores) -> g
//   kd_down   units of 128 output rows of one active expert's W_down (or of a
//             256-column part of W_s_down) arrive as TMA boxes; the CTA computes
//             the expert's NormSiLU (subtract u, RMS over d_e, SiLU, times
//             s_e r_e) when the expert changes and writes fp32 partials
//   kd_combine adds the shared-expert parts and the active experts' partials
//             in ascending expert order (+ the residual)
//
// Data movement: one CTA per SM, 8 consumer warps and 1 producer warp.  The
// producer streams contiguous weight rows with bulk copies of >= 4 KB each
// (cp.async.bulk, L2 evict-first) into a ring of shared-memory stages behind
// mbarriers; on B200 a copy engine sustains HBM bandwidth with copies this
// size, while small tensor-map boxes (2 KB) are limited by per-copy cost.
// kd_route / kd_up give each CTA a contiguous range of weight rows at full
// width and copy each row into a 16-byte padded shared-memory row, so that
// ldmatrix reads of 8 rows hit 8 different bank groups; the 8 consumer warps
// split the columns and add their partial sums in warp order.  kd_down loads
// 128-row x 64-column tiles with TMA in the 128-byte swizzle, which ldmatrix
// reads directly; each consumer warp owns 16 of the 128 rows.
// Activations a later kernel consumes are written in a layout its ldmatrix
// reads can use directly (an XOR swizzle of the 16-byte chunks inside each
// row).
//
// Arithmetic: the projections are thin dense contractions (up to 16 tokens
// against 8-row chunks or 128-row units of weights) done with mma.sync
// m16n8k16 (bf16 in, fp32 accumulate) with the weights as A: a tensor-core
// instruction per 16x8x16 tile keeps the instruction count far below the
// memory time, which is the bound at these batch sizes.
// Intermediates fed back into a contraction (the shared expert's hidden
// activations and the scaled NormSiLU outputs) are stored as a bf16 pair
// hi + lo with lo = bf16(v - hi), and both halves are multiplied, so they
// carry ~16 significant bits instead of 8.
//
// Waits are bounded: after ~1 s a wait gives up, sets bit 2 of the device
// error word and the CTA stops issuing work (no hang, no trap).  Consecutive
// kernels use programmatic dependent launch.
#pragma once

#include <cuda.h>

#include "common.cuh"

namespace deco {
namespace dec {

constexpr int kConsumerWarps = 8;
constexpr int kThreads = (kConsumerWarps + 1) * 32;
constexpr int kMaxT = 16;                      // decode batches
constexpr int kTok = 16;                       // token rows of every activation tile
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
// 2-D TMA tile load (coordinates: column, row); columns are a multiple of 64
__device__ __forceinline__ void tma_2d(void* dst, const CUtensorMap* map, int col, int row, uint64_t* bar,
                                       uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(col), "r"(row), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}
__device__ __forceinline__ void tma_2d(void* dst, const CUtensorMap* map, int col, int row, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(col), "r"(row), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" :::); }
__device__ __forceinline__ void consumer_sync() {   // the 8 consumer warps only
  asm volatile("bar.sync 1, %0;" ::"n"(kConsumerWarps * 32) : "memory");
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x2(uint32_t addr, uint32_t& r0, uint32_t& r1) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];" : "=r"(r0), "=r"(r1) : "r"(addr));
}
// D[16 x 8] += A[16 x 16] B[16 x 8], bf16 inputs, fp32 accumulators
__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9},"
      " {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Tiles of R rows x 64 bf16 columns, 128 B per row, at a 1024-B aligned
// base: 16-byte chunk c of row r sits at chunk position c ^ (r & 7).  This is
// the TMA 128-byte swizzle, and ldmatrix reads of 8 rows at one chunk hit 8
// different bank groups.
__device__ __forceinline__ uint32_t swz(uint32_t base, int row, int chunk) {
  return base + (uint32_t)row * 128u + ((uint32_t)(chunk ^ (row & 7)) << 4);
}

// ---------------------------------------------------------------------------
// Ring of weight stages shared by the three streaming kernels.

struct Ring {
  uint64_t* full;    // [kMaxStages]
  uint64_t* empty;   // [kMaxStages]
  unsigned char* stage;
  uint32_t stage_bytes;
  int nstages;
};

// dynamic shared memory: [<=1 KB alignment slack][barriers 1 KB][ring][operand];
// kStaticReserve bytes are left for each kernel's static __shared__ arrays.
constexpr uint32_t kHeaderBytes = 1024;
constexpr uint32_t kStaticReserve = 1536;

struct SmemPlan {
  uint32_t ring_off, op_off, total, stage_bytes;
  int nstages;
};

__host__ __device__ inline SmemPlan smem_plan(uint32_t operand_bytes, uint32_t stage_bytes) {
  SmemPlan p;
  p.ring_off = kHeaderBytes;
  p.stage_bytes = stage_bytes;
  const uint32_t op = (operand_bytes + 1023u) & ~1023u;
  const uint32_t room = (uint32_t)kSmemLimit - kStaticReserve - 1024u - kHeaderBytes - op;
  p.nstages = (int)(room / stage_bytes);
  if (p.nstages > kMaxStages) p.nstages = kMaxStages;
  p.op_off = p.ring_off + p.nstages * stage_bytes;
  p.total = p.op_off + op + 1024u;   // + alignment slack
  return p;
}

// barriers: full[8], empty[8], opbar, abort word; returns the 1024-B aligned base
__device__ __forceinline__ unsigned char* ring_setup(unsigned char* smem_raw, const SmemPlan& sp, Ring& ring,
                                                     uint64_t*& opbar, volatile int*& abort_flag) {
  unsigned char* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
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
  return smem;
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
  float* r;          // [T][E]
  uint8_t* act;      // [T][E]
  float* u;          // [T][d_e]
  bf16* hs;          // [16 tok][hi d_s | lo d_s], chunk-swizzled rows: SiLU(x W_s_up^T)
  float* C;          // [kp <= 8][E][16 tok][d_e] up-projection g = x W_up[e]^T (active experts),
                     // partial sums over K parts
  float* P;          // [E][16 slots][D] routed down-projection partials, slot i = the i-th
                     // active token of expert e (ascending)
  float* Ps;         // [ceil(d_s / 256)][16 tok][D] shared down-projection partials
  int* err;
  bf16* out;
};

// physical 16-byte chunk of logical chunk k in a row with index r: the low 3
// bits are XOR-ed with the row index, so 8 consecutive rows of one logical
// chunk sit in 8 different bank groups
__host__ __device__ __forceinline__ int row_chunk(int r, int k) { return (k & ~7) | ((k ^ r) & 7); }

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

__device__ __forceinline__ void bf16x8_to_f32(const uint4& q, float (&v)[8]) { unpack16(q, v); }

// Reduce N = 2^m per-lane values across the warp: at each of the first m
// levels a lane keeps one half of its values, sends the other half to its
// partner and adds what it receives; the remaining 5 - m levels are plain
// butterflies.  Afterwards lane l holds the warp total of value index
// (l >> (5 - m)) & (N - 1), a fixed 5-level tree over the 32 lane partials.
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

// v as a bf16 pair (hi, lo = v - hi) at element j of a chunk-swizzled row of
// 2L elements (hi part [0, L), lo part [L, 2L)); r is the row index
__device__ __forceinline__ void store_row_hi_lo(bf16* row, int r, int L, int j, float v) {
  const bf16 hi = __float2bfloat16_rn(v);
  const bf16 lo = __float2bfloat16_rn(v - __bfloat162float(hi));
  row[row_chunk(r, j >> 3) * 8 + (j & 7)] = hi;
  row[row_chunk(r, (L + j) >> 3) * 8 + (j & 7)] = lo;
}

// ---------------------------------------------------------------------------
// Row-range streaming (kd_route, kd_up): a CTA's rows are taken in chunks of
// `rc` rows (one stage), each row one bulk copy into a padded smem row of
// pitch D*2 + 16 bytes.  For a chunk, warp w multiplies the 16 token rows of x
// by the chunk's rows over columns [w*D/8, (w+1)*D/8): one m16n8 tile per
// 16-column step.  The 8 warps' 16 x 8 results are then added in warp order.

__host__ __device__ inline uint32_t x_pitch(int D) { return (uint32_t)D * 2u + 16u; }
__host__ __device__ inline int rows_per_chunk(int D) { return D <= 2048 ? 8 : 4; }
__host__ __device__ inline uint32_t row_stage_bytes(int D) {
  return ((uint32_t)rows_per_chunk(D) * x_pitch(D) + 1023u) & ~1023u;
}

__device__ __forceinline__ uint32_t x_addr(uint32_t xs, uint32_t pitch, int lane, int chunk) {
  return xs + (uint32_t)((lane & 7) + ((lane >> 3) & 1) * 8) * pitch + (uint32_t)(chunk + (lane >> 4)) * 16u;
}
// B operand (8 weight rows x 16 columns) from padded rows; rows >= rc (a
// chunk of fewer rows) repeat row 0, and their outputs are discarded
__device__ __forceinline__ uint32_t w_addr(uint32_t ws, uint32_t pitch, int lane, int chunk, int rc) {
  const int r = (lane & 7) < rc ? (lane & 7) : 0;
  return ws + (uint32_t)r * pitch + (uint32_t)(chunk + ((lane >> 3) & 1)) * 16u;
}

// issue the T row copies of x into padded rows (one thread)
__device__ __forceinline__ void stage_x(const Args& a, unsigned char* xs, uint64_t* bar) {
  const uint32_t pitch = x_pitch(a.D);
  mbar_expect_tx(bar, (uint32_t)a.T * a.D * 2);
  for (int t = 0; t < a.T; ++t) bulk_g2s(xs + (size_t)t * pitch, a.x + (size_t)t * a.D, (uint32_t)a.D * 2, bar);
}
// zero the rows T..15 of the 16-row x operand (consumer threads)
__device__ __forceinline__ void zero_x_tail(const Args& a, unsigned char* xs, int tid, int nthreads) {
  const uint32_t pitch = x_pitch(a.D);
  const int words = (int)(pitch / 16);
  for (int i = tid; i < (kTok - a.T) * words; i += nthreads)
    reinterpret_cast<uint4*>(xs + (size_t)(a.T + i / words) * pitch)[i % words] = make_uint4(0u, 0u, 0u, 0u);
}

// y[16 tok][8 rows] for one chunk; returns in `red_out` (thread o < 128 of the
// consumer warps gets output o = tok*8 + row)
__device__ __forceinline__ float chunk_gemv(uint32_t xs, uint32_t ws, uint32_t pitch, int D, int warp, int lane,
                                            float* red, bool math) {
  const int rc = rows_per_chunk(D);
  float d[4] = {0.f, 0.f, 0.f, 0.f};
  if (math) {
    const int c0 = warp * (D / 8) / 8, c1 = c0 + (D / 8) / 8;   // 16-byte chunks of this warp
    for (int ch = c0; ch < c1; ch += 2) {
      uint32_t a0, a1, a2, a3, b0, b1;
      ldsm_x4(x_addr(xs, pitch, lane, ch), a0, a1, a2, a3);
      ldsm_x2(w_addr(ws, pitch, lane, ch, rc), b0, b1);
      mma16816(d, a0, a1, a2, a3, b0, b1);
    }
  }
  // red: [8 warps][16 tok][8 rows]
  const int tok = lane >> 2, col = 2 * (lane & 3);
  *reinterpret_cast<float2*>(red + warp * 128 + tok * 8 + col) = make_float2(d[0], d[1]);
  *reinterpret_cast<float2*>(red + warp * 128 + (tok + 8) * 8 + col) = make_float2(d[2], d[3]);
  consumer_sync();
  float v = 0.f;
  const int o = threadIdx.x;
  if (o < 128) {
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w) v += red[w * 128 + o];
  }
  consumer_sync();
  return v;
}

// ---------------------------------------------------------------------------
// kd_route
//
// CTAs [0, Cr) with Cr = min(E, 64): router rows on CUDA cores with an exact
// sign decision (see common.cuh), the 8 warps of a CTA splitting each row's
// columns.  The remaining CTAs split the rows of [W_bar_up ; W_s_up] evenly
// and write u = x W_bar_up^T and SiLU(x W_s_up^T) (as hi/lo pairs) for them.

// router CTAs of kd_route: one router row each (E <= 64), else several
__host__ __device__ inline int router_ctas(int E) { return E < 64 ? E : 64; }

__global__ void __launch_bounds__(kThreads, 1) kd_route(const __grid_constant__ Args a) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  __shared__ unsigned long long limbs[1][kLimbs];
  const int Cr = router_ctas(a.E);
  const bool router_cta = (int)blockIdx.x < Cr;
  const uint32_t pitch = x_pitch(a.D);
  // operand: x rows, then the 4 KB cross-warp reduction scratch
  const SmemPlan sp = smem_plan(kTok * pitch + 4096, router_cta ? kStageBytes : row_stage_bytes(a.D));
  Ring ring;
  uint64_t* xbar;
  volatile int* abort_flag;
  unsigned char* smem = ring_setup(smem_raw, sp, ring, xbar, abort_flag);
  unsigned char* xsm = smem + sp.op_off;
  float* red = reinterpret_cast<float*>(xsm + kTok * pitch);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  pdl_trigger();

  if (router_cta) {
    // router rows e = blockIdx.x + Cr i; for each row the 8 consumer warps
    // split the D columns (16-byte chunks), and their partial sums are added
    // in warp order
    const int nrow = (a.E - (int)blockIdx.x + Cr - 1) / Cr;
    const uint32_t rowbytes = (uint32_t)a.D * 2;
    const int per = (int)(kStageBytes / rowbytes);   // router rows per stage
    const int nst = (nrow + per - 1) / per;
    if (warp == kConsumerWarps) {
      if (lane == 0) {
        const uint64_t pol = evict_first_policy();
        stage_x(a, xsm, xbar);
        for (int k = 0; k < nst; ++k) {
          const int n = min(per, nrow - k * per);
          mbar_expect_tx(&ring.full[k], n * rowbytes);
          for (int j = 0; j < n; ++j)
            bulk_g2s(ring.stage + (size_t)k * kStageBytes + (size_t)j * rowbytes,
                     a.W_r + (size_t)(blockIdx.x + Cr * (k * per + j)) * a.D, rowbytes, &ring.full[k], pol);
        }
      }
      return;
    }
    // a value goes through <= 8 ceil(D / 2048) products in its lane, 5
    // butterfly levels, 7 cross-warp additions and the bias
    const int n_terms = 8 * ((a.D + 2047) / 2048) + 16;
    const float gm = gamma_f32(n_terms);
    const float bscale = 2.f * gm * (1.f + 2.f * gm);
    const float tiny = float(n_terms) * 2.8025969e-45f;
    bool bad = false;
    // every consumer warp waits for x and for every stage, so every issued
    // copy is awaited before the CTA exits
    bool ok = mbar_wait(xbar, 0, abort_flag, a.err);
    for (int k = 0; k < nst; ++k) ok = ok && mbar_wait(&ring.full[k], 0, abort_flag, a.err);
    for (int i = 0; i < nrow; ++i) {
      const int e = blockIdx.x + Cr * i;
      const bf16* wrow =
          reinterpret_cast<const bf16*>(ring.stage + (size_t)(i / per) * kStageBytes + (size_t)(i % per) * rowbytes);
      float v[32];
#pragma unroll
      for (int q = 0; q < 32; ++q) v[q] = 0.f;
      // z partials in v[t], sum |x w| partials in v[16 + t]
      if (ok) {
#pragma unroll 1
        for (int ch = warp * 32 + lane; ch < a.D / 8; ch += kConsumerWarps * 32) {
          float wv[8];
          bf16x8_to_f32(*reinterpret_cast<const uint4*>(wrow + (size_t)ch * 8), wv);
#pragma unroll
          for (int t = 0; t < kTok; ++t) {
            if (t < a.T) {
              float xv[8];
              bf16x8_to_f32(*reinterpret_cast<const uint4*>(xsm + (size_t)t * pitch + (size_t)ch * 16), xv);
#pragma unroll
              for (int q = 0; q < 8; ++q) {
                v[t] = fmaf(xv[q], wv[q], v[t]);
                v[16 + t] = fmaf(fabsf(xv[q]), fabsf(wv[q]), v[16 + t]);
              }
            }
          }
        }
      }
      red[warp * 32 + lane] = warp_reduce_scatter<32>(v, lane);   // lane l: this warp's value l
      consumer_sync();
      if (warp == 0 && ok) {
        float tot = 0.f;
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w) tot += red[w * 32 + lane];
        const float S = __shfl_sync(kFull, tot, (lane + 16) & 31);
        const float b = a.b_r[e];
        const int t = lane;
        const bool mine = t < a.T;
        const float z = tot + b;
        const float B = bscale * (S + fabsf(b)) + tiny;
        const bool sure = fabsf(z) > B;
        bool on = sure && z > 0.f;
        // guard band: exact re-evaluation of the sign, the whole warp per score
        unsigned need = __ballot_sync(kFull, mine && !sure);
        while (need) {
          const int tt = __ffs(need) - 1;
          need &= need - 1;
          const int sg = exact_sign_warp(reinterpret_cast<const bf16*>(xsm + (size_t)tt * pitch), wrow, a.D, b,
                                         limbs[0], &bad);
          if (lane == tt) on = sg > 0;
        }
        if (mine) {
          a.r[(size_t)t * a.E + e] = on ? fmaxf(z, 0.f) : 0.f;
          a.act[(size_t)t * a.E + e] = on ? 1 : 0;
        }
      }
      consumer_sync();   // red is reused by the next row
    }
    if (bad && lane == 0) atomicOr(a.err, 1);
    return;
  }

  // rows of [W_bar_up ; W_s_up], split evenly over the remaining CTAs
  const int nrows = a.d_e + a.d_s;
  const int G = gridDim.x - Cr, c = blockIdx.x - Cr;
  const int ra = (int)((long long)c * nrows / G), rb = (int)((long long)(c + 1) * nrows / G);
  const int rc = rows_per_chunk(a.D);
  const int nchunks = (rb - ra + rc - 1) / rc;
  auto row_src = [&](int g) -> const bf16* {
    return g < a.d_e ? a.W_bar + (size_t)g * a.D : a.W_s_up + (size_t)(g - a.d_e) * a.D;
  };
  if (warp == kConsumerWarps) {
    if (lane == 0 && nchunks > 0) {
      const uint64_t pol = evict_first_policy();
      stage_x(a, xsm, xbar);
      for (int k = 0; k < nchunks; ++k) {
        const int s = k % ring.nstages;
        if (!mbar_wait(&ring.empty[s], ((k / ring.nstages) & 1) ^ 1, abort_flag, a.err)) break;
        const int g0 = ra + k * rc, n = min(rc, rb - g0);
        mbar_expect_tx(&ring.full[s], (uint32_t)n * a.D * 2);
        for (int i = 0; i < n; ++i)
          bulk_g2s(ring.stage + (size_t)s * ring.stage_bytes + (size_t)i * pitch, row_src(g0 + i),
                   (uint32_t)a.D * 2, &ring.full[s], pol);
      }
    }
    return;
  }
  if (nchunks == 0) return;
  zero_x_tail(a, xsm, threadIdx.x, kConsumerWarps * 32);
  consumer_sync();
  bool ok = mbar_wait(xbar, 0, abort_flag, a.err);
  for (int k = 0; k < nchunks; ++k) {
    const int s = k % ring.nstages;
    ok = ok && mbar_wait(&ring.full[s], (k / ring.nstages) & 1, abort_flag, a.err);
    const float v = chunk_gemv(smem_u32(xsm), smem_u32(ring.stage + (size_t)s * ring.stage_bytes), pitch, a.D,
                               warp, lane, red, ok);
    if (ok && lane == 0) mbar_arrive(&ring.empty[s]);
    const int o = threadIdx.x;
    const int t = o >> 3, i = o & 7;
    const int g = ra + k * rc + i;
    if (ok && o < 128 && i < rc && g < rb) {
      if (g < a.d_e) {
        if (t < a.T) a.u[(size_t)t * a.d_e + g] = v;
      } else {
        const int j = g - a.d_e;   // shared hidden unit
        store_row_hi_lo(a.hs + (size_t)t * 2 * a.d_s, t, a.d_s, j, t < a.T ? silu_f(v) : 0.f);
      }
    }
  }
}

// ---------------------------------------------------------------------------
// kd_up: g = x W_up[e]^T for the experts some token uses, as fp32 partial
// sums over K parts.  Units are (expert e of the union, block of 128 rows of
// W_up[e], K part p of D / kp columns), with kp <= 8 the smallest power of
// two that gives every CTA at least two units; CTA c takes a contiguous range
// of them.  Weights arrive as 128 x 64 TMA boxes (two per 32 KB stage, the
// 128-byte swizzle ldmatrix reads directly), x stays resident in padded
// shared-memory rows, and consumer warp w multiplies rows 16w..16w+15 of the
// unit by the 16 token rows.  Results go to C[p][e][t][j]; kd_down adds the
// K parts in order.  (NormSiLU runs in kd_down.)

constexpr int kDRows = 128;                  // weight rows per unit (kd_up, kd_down)
constexpr uint32_t kBoxBytes = kDRows * 128; // 128 rows x 64 bf16 columns

__host__ __device__ inline int up_kparts(int U, int d_e, int D, int G) {
  const int units = U * ((d_e + kDRows - 1) / kDRows);
  int kp = 1;
  while (kp < 8 && D / (2 * kp) >= 256 && units * kp < 2 * G) kp *= 2;
  return kp;
}

__global__ void __launch_bounds__(kThreads, 1)
    kd_up(const __grid_constant__ CUtensorMap tmU, const __grid_constant__ Args a) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  __shared__ uint16_t emask[256];
  __shared__ uint8_t ulist[256];
  __shared__ int s_U;
  const uint32_t pitch = x_pitch(a.D);
  const SmemPlan sp = smem_plan(kTok * pitch, kStageBytes);
  Ring ring;
  uint64_t* xbar;
  volatile int* abort_flag;
  unsigned char* smem = ring_setup(smem_raw, sp, ring, xbar, abort_flag);
  unsigned char* xsm = smem + sp.op_off;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // x does not depend on the router: stage it before waiting for it
  if (threadIdx.x == 0) stage_x(a, xsm, xbar);
  if (warp < kConsumerWarps) zero_x_tail(a, xsm, threadIdx.x, kConsumerWarps * 32);
  pdl_wait();          // router outputs
  pdl_trigger();
  build_union(a, emask, ulist, &s_U);
  const int nrb = (a.d_e + kDRows - 1) / kDRows;
  const int kp = up_kparts(s_U, a.d_e, a.D, gridDim.x);
  const int Kp = a.D / kp;
  const int NU = s_U * nrb * kp;
  const int u0 = (int)((long long)blockIdx.x * NU / gridDim.x);
  const int u1 = (int)((long long)(blockIdx.x + 1) * NU / gridDim.x);
  if (warp == kConsumerWarps) {
    if (lane == 0) {
      const uint64_t pol = evict_first_policy();
      int k = 0;
      for (int u = u0; u < u1; ++u) {
        const int p = u % kp, rb = (u / kp) % nrb, e = ulist[u / (kp * nrb)];
        const int row = e * a.d_e + rb * kDRows;
        for (int c0 = 0; c0 < Kp; c0 += 128, ++k) {
          const int s = k % ring.nstages;
          if (!mbar_wait(&ring.empty[s], ((k / ring.nstages) & 1) ^ 1, abort_flag, a.err)) break;
          const int nb = min(2, (Kp - c0) / 64);
          mbar_expect_tx(&ring.full[s], (uint32_t)nb * kBoxBytes);
          for (int b = 0; b < nb; ++b)
            tma_2d(ring.stage + (size_t)s * ring.stage_bytes + b * kBoxBytes, &tmU, p * Kp + c0 + 64 * b, row,
                   &ring.full[s], pol);
        }
        if (*abort_flag) break;
      }
    }
    return;
  }
  // the x copies were issued unconditionally: always await them
  bool ok = mbar_wait(xbar, 0, abort_flag, a.err);
  const uint32_t x_u32 = smem_u32(xsm);
  const int ntiles = (a.T + 7) / 8;
  int k = 0;
  for (int u = u0; u < u1; ++u) {
    const int p = u % kp, rb = (u / kp) % nrb, e = ulist[u / (kp * nrb)];
    float acc[2][4] = {};
    for (int c0 = 0; c0 < Kp; c0 += 128, ++k) {
      const int s = k % ring.nstages;
      ok = ok && mbar_wait(&ring.full[s], (k / ring.nstages) & 1, abort_flag, a.err);
      const int nb = min(2, (Kp - c0) / 64);
      if (ok) {
        const uint32_t st = smem_u32(ring.stage + (size_t)s * ring.stage_bytes);
        for (int b = 0; b < nb; ++b) {
          const uint32_t box = st + b * kBoxBytes;
#pragma unroll
          for (int ks = 0; ks < 4; ++ks) {
            uint32_t a0, a1, a2, a3;
            ldsm_x4(swz(box, 16 * warp + (lane & 7) + ((lane >> 3) & 1) * 8, 2 * ks + (lane >> 4)), a0, a1, a2,
                    a3);
            const int kc = (p * Kp + c0 + 64 * b) / 8 + 2 * ks + ((lane >> 3) & 1);
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
              if (nt < ntiles) {
                uint32_t b0, b1;
                ldsm_x2(x_u32 + (uint32_t)(8 * nt + (lane & 7)) * pitch + (uint32_t)kc * 16u, b0, b1);
                mma16816(acc[nt], a0, a1, a2, a3, b0, b1);
              }
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&ring.empty[s]);
    }
    if (!ok) continue;
    // acc[nt][i]: row 16 warp + lane/4 + 8 (i >> 1), token 8 nt + 2 (lane & 3) + (i & 1)
    const int j0 = rb * kDRows + 16 * warp + (lane >> 2);
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int t = 8 * nt + 2 * (lane & 3) + (i & 1);
        const int j = j0 + 8 * (i >> 1);
        if (t < a.T && j < a.d_e) a.C[(((size_t)p * a.E + e) * kTok + t) * a.d_e + j] = acc[nt][i];
      }
    }
  }
}

// ---------------------------------------------------------------------------
// kd_down: the routed and the shared down-projections as fp32 partial sums.
//
// Units are (expert e of the union, block of 128 output rows), with all of d_e
// as K, and (K part q of 256 columns of W_s_down, block of 128 output rows)
// for the shared expert.  CTA c takes a contiguous range of the units (shared
// ones first, then experts ascending), so consecutive units mostly share an
// expert.  A unit's weights arrive as TMA boxes of 128 rows x 64 columns
// (16 KB, 128-byte swizzle, the layout ldmatrix reads without bank
// conflicts), two boxes per 32 KB stage; consumer warp w multiplies the unit's
// rows 16w..16w+15 (m16n8k16, weights as A, tokens as B).  B rows are the
// shared expert's hidden activations (hi/lo, resident in shared memory) or the
// expert's NormSiLU activations, which the CTA computes when the expert
// changes: c = g - u, h = c / sqrt(mean c^2 + eps), a = s_e r_e SiLU(h), stored
// as hi/lo in compact slots (slot i = the i-th active token of e).  Results go
// to P[e][slot][row] and Ps[q][token][row]; kd_combine adds them.

constexpr int kSq = 256;                     // K columns per shared-expert unit

__host__ __device__ inline int down_nsq(int d_s) { return (d_s + kSq - 1) / kSq; }

struct DUnit {
  bool shared;
  int e, q, rb, K, kb0;   // kb0: first K column of the unit within its matrix row
};

__device__ __forceinline__ DUnit down_unit(const Args& a, const uint8_t* ulist, int nrb, int u) {
  DUnit d;
  const int ns = down_nsq(a.d_s) * nrb;
  d.shared = u < ns;
  if (d.shared) {
    d.q = u / nrb;
    d.rb = u - d.q * nrb;
    d.kb0 = d.q * kSq;
    d.K = min(kSq, a.d_s - d.kb0);
    d.e = -1;
  } else {
    const int v = u - ns, ui = v / nrb;
    d.rb = v - ui * nrb;
    d.e = ulist[ui];
    d.q = 0;
    d.kb0 = 0;
    d.K = a.d_e;
  }
  return d;
}

__global__ void __launch_bounds__(kThreads, 1)
    kd_down(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmS,
            const __grid_constant__ Args a) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  __shared__ uint16_t emask[256];
  __shared__ uint8_t ulist[256];
  __shared__ int s_U;
  // operand: hs rows (16 x 4 d_s bytes), the NormSiLU tile (16 x 4 d_e bytes),
  // a zero row for slots past the expert's tokens (4 d_e <= 1 KB)
  const uint32_t hbytes = (uint32_t)kTok * a.d_s * 4;
  const uint32_t tbytes = (uint32_t)kTok * a.d_e * 4;
  const SmemPlan sp = smem_plan(hbytes + tbytes + 1024, kStageBytes);
  Ring ring;
  uint64_t* hbar;
  volatile int* abort_flag;
  unsigned char* smem = ring_setup(smem_raw, sp, ring, hbar, abort_flag);
  unsigned char* hsm = smem + sp.op_off;
  unsigned char* tile = hsm + hbytes;
  unsigned char* zrow = tile + tbytes;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  pdl_trigger();
  for (int i = threadIdx.x; i < 1024 / 16; i += blockDim.x) reinterpret_cast<uint4*>(zrow)[i] = make_uint4(0, 0, 0, 0);
  // The router's outputs are complete: this grid starts only after every CTA
  // of kd_up passed its own wait on the router.
  build_union(a, emask, ulist, &s_U);
  const int nrb = a.D / kDRows;
  const int NU = (down_nsq(a.d_s) + s_U) * nrb;
  const int kp_up = up_kparts(s_U, a.d_e, a.D, gridDim.x);   // kd_up runs on the same grid
  const int u0 = (int)((long long)blockIdx.x * NU / gridDim.x);
  const int u1 = (int)((long long)(blockIdx.x + 1) * NU / gridDim.x);

  if (warp == kConsumerWarps) {
    if (lane == 0) {
      const uint64_t pol = evict_first_policy();
      mbar_expect_tx(hbar, hbytes);
      bulk_g2s(hsm, a.hs, hbytes, hbar);
      // weights do not depend on kd_up: they stream while it finishes
      int k = 0;
      for (int u = u0; u < u1; ++u) {
        const DUnit d = down_unit(a, ulist, nrb, u);
        const int row = d.shared ? d.rb * kDRows : d.e * a.D + d.rb * kDRows;
        for (int c0 = 0; c0 < d.K; c0 += 128, ++k) {
          const int s = k % ring.nstages;
          if (!mbar_wait(&ring.empty[s], ((k / ring.nstages) & 1) ^ 1, abort_flag, a.err)) break;
          const int nb = min(2, (d.K - c0) / 64);
          mbar_expect_tx(&ring.full[s], (uint32_t)nb * kBoxBytes);
          for (int b = 0; b < nb; ++b)
            tma_2d(ring.stage + (size_t)s * ring.stage_bytes + b * kBoxBytes, d.shared ? &tmS : &tmW,
                   d.kb0 + c0 + 64 * b, row, &ring.full[s], pol);
        }
        if (*abort_flag) break;
      }
    }
    return;
  }

  pdl_wait();   // g (kd_up), u, r (kd_route)
  bool ok = mbar_wait(hbar, 0, abort_flag, a.err);
  const uint32_t hs_u32 = smem_u32(hsm), tile_u32 = smem_u32(tile), z_u32 = smem_u32(zrow);
  int cur_e = -1, n_cur = 0, k = 0;
  for (int u = u0; u < u1; ++u) {
    const DUnit d = down_unit(a, ulist, nrb, u);
    if (!d.shared && d.e != cur_e) {
      // NormSiLU rows of expert e, one warp per active token
      consumer_sync();   // every warp is done with the previous tile
      const int e = d.e;
      const uint32_t m_e = emask[e];
      n_cur = __popc(m_e);
      if (ok && !*abort_flag) {
        for (int slot = warp; slot < n_cur; slot += kConsumerWarps) {
          uint32_t m = m_e;
          for (int i = 0; i < slot; ++i) m &= m - 1;
          const int t = __ffs(m) - 1;
          // every load of the token's row is issued before the first is used
          const float rte = __ldcg(a.r + (size_t)t * a.E + e);
          const float se = __ldg(a.s + e);
          float gp[8][8], uq[8];   // [K part][value], d_e <= 256: 8 values per lane
#pragma unroll
          for (int pp = 0; pp < 8; ++pp)
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              const int j = lane + 32 * q;
              gp[pp][q] = (pp < kp_up && j < a.d_e)
                              ? __ldcg(a.C + (((size_t)pp * a.E + e) * kTok + t) * a.d_e + j) : 0.f;
            }
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const int j = lane + 32 * q;
            uq[q] = j < a.d_e ? __ldcg(a.u + (size_t)t * a.d_e + j) : 0.f;
          }
          float cv[8];
          float ss = 0.f;
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            float g = 0.f;   // kd_up's K parts, in order (absent parts add an exact 0)
#pragma unroll
            for (int pp = 0; pp < 8; ++pp) g += gp[pp][q];
            cv[q] = g - uq[q];
            ss = fmaf(cv[q], cv[q], ss);
          }
          ss = warp_sum(ss);
          const float rinv = 1.f / sqrtf(ss / float(a.d_e) + a.eps);
          const float coef = se * rte;
          bf16* row = reinterpret_cast<bf16*>(tile + (size_t)slot * 4 * a.d_e);
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const int j = lane + 32 * q;
            if (j < a.d_e) store_row_hi_lo(row, slot, a.d_e, j, coef * silu_f(cv[q] * rinv));
          }
        }
      }
      consumer_sync();
      cur_e = e;
    }
    // B rows of this unit: tokens (shared) or slots (routed); rows past n read zeros
    const int n = d.shared ? a.T : n_cur;
    const int ntiles = (n + 7) / 8;
    const int L = d.shared ? a.d_s : a.d_e;            // hi half length of a B row
    uint32_t brow[2];
    int bsw[2];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      const int r = 8 * nt + (lane & 7);
      // hidden rows of tokens >= T are zeros (kd_route writes all 16 rows)
      const bool on = d.shared || r < n;
      brow[nt] = on ? (d.shared ? hs_u32 : tile_u32) + (uint32_t)r * 4u * (uint32_t)L : z_u32;
      bsw[nt] = on ? r : 0;
    }
    const int kcb = d.kb0 / 8;                          // first 16-byte chunk of the unit in a B row
    float acc[2][4] = {};
    for (int c0 = 0; c0 < d.K; c0 += 128, ++k) {
      const int s = k % ring.nstages;
      ok = ok && mbar_wait(&ring.full[s], (k / ring.nstages) & 1, abort_flag, a.err);
      const int nb = min(2, (d.K - c0) / 64);
      if (ok) {
        const uint32_t st = smem_u32(ring.stage + (size_t)s * ring.stage_bytes);
        for (int b = 0; b < nb; ++b) {
          const uint32_t box = st + b * kBoxBytes;
#pragma unroll
          for (int ks = 0; ks < 4; ++ks) {
            uint32_t a0, a1, a2, a3;
            ldsm_x4(swz(box, 16 * warp + (lane & 7) + ((lane >> 3) & 1) * 8, 2 * ks + (lane >> 4)), a0, a1, a2,
                    a3);
            const int kc = kcb + (c0 + 64 * b) / 8 + 2 * ks + ((lane >> 3) & 1);
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
              if (nt < ntiles) {
                uint32_t bh0, bh1, bl0, bl1;
                ldsm_x2(brow[nt] + (uint32_t)row_chunk(bsw[nt], kc) * 16u, bh0, bh1);
                ldsm_x2(brow[nt] + (uint32_t)row_chunk(bsw[nt], kc + L / 8) * 16u, bl0, bl1);
                mma16816(acc[nt], a0, a1, a2, a3, bh0, bh1);
                mma16816(acc[nt], a0, a1, a2, a3, bl0, bl1);
              }
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&ring.empty[s]);
    }
    if (!ok) continue;
    // acc[nt][i]: row 16 warp + lane/4 + 8 (i >> 1), column 8 nt + 2 (lane & 3) + (i & 1)
    const int r0 = d.rb * kDRows + 16 * warp + (lane >> 2);
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int col = 8 * nt + 2 * (lane & 3) + (i & 1);
        const int row = r0 + 8 * (i >> 1);
        if (col < n) {
          float* dst = d.shared ? a.Ps + ((size_t)d.q * kTok + col) * a.D
                                : a.P + ((size_t)d.e * kTok + col) * a.D;
          dst[row] = acc[nt][i];
        }
      }
    }
  }
}

// ---------------------------------------------------------------------------
// kd_combine: out[t][row] = sum over the shared-expert K parts q of Ps[q][t][row]
// + sum over t's active experts e, ascending, of P[e][slot][row] (+ x[t][row]);
// a fixed order, so the result is bitwise reproducible.

__global__ void __launch_bounds__(256) kd_combine(const __grid_constant__ Args a) {
  __shared__ int list_e[256], list_s[256], n_list;
  const int t = blockIdx.y, lane = threadIdx.x & 31;
  // The router's outputs are complete: this grid starts only after every CTA
  // of kd_down started, and kd_down starts only after kd_up passed its wait on
  // the router.  The token's expert list is built while kd_down finishes.
  if (threadIdx.x < 32) {
    int n = 0;
    for (int e0 = 0; e0 < a.E; e0 += 32) {
      const int e = e0 + lane;
      uint32_t toks = 0;   // tokens using e (all flags loaded before any is used)
      if (e < a.E) {
        uint8_t fl[kTok];
#pragma unroll
        for (int tp = 0; tp < kTok; ++tp) fl[tp] = tp < a.T ? __ldcg(a.act + (size_t)tp * a.E + e) : 0;
#pragma unroll
        for (int tp = 0; tp < kTok; ++tp) toks |= (fl[tp] ? 1u : 0u) << tp;
      }
      const bool f = (toks >> t) & 1u;
      const int slot = __popc(toks & ((1u << t) - 1u));
      const unsigned m = __ballot_sync(kFull, f);
      if (f) {
        const int i = n + __popc(m & ((1u << lane) - 1u));
        list_e[i] = e;
        list_s[i] = slot;
      }
      n += __popc(m);
    }
    if (lane == 0) n_list = n;
  }
  __syncthreads();
  pdl_wait();   // the partials (kd_down)
  const int row = blockIdx.x * 256 + threadIdx.x;
  if (row >= a.D) return;
  float v = 0.f;
  const int nsq = down_nsq(a.d_s);
  for (int q = 0; q < nsq; ++q) v += __ldcg(a.Ps + ((size_t)q * kTok + t) * a.D + row);
  const int n = n_list;
  for (int i = 0; i < n; ++i) v += __ldcg(a.P + ((size_t)list_e[i] * kTok + list_s[i]) * a.D + row);
  if (a.residual) v += __bfloat162float(a.x[(size_t)t * a.D + row]);
  a.out[(size_t)t * a.D + row] = __float2bfloat16_rn(v);
}

}  // namespace dec
}  // namespace deco
