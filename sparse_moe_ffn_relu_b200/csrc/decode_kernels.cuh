// Decode-batch kernel (T <= 16 tokens, bf16) of the DECO MoE layer.
//
// At a few tokens the layer is bound by HBM: every weight byte is used by at
// most 16 tokens, and only the routed experts that some token activates need
// to be read (the paper's point about sparse activation saving memory access,
// "DECO: Sparse Mixture-of-Experts with Dense-Comparable Performance on
// End-Side Devices", §1 and §5).  The whole layer is one persistent kernel,
// kd_layer, with one CTA per SM (a cooperative launch, so every CTA is
// resident), that streams each needed weight byte once through a shared-memory
// ring and hands data between CTAs through counters in global memory instead
// of kernel boundaries:
//
//   phase R  CTAs [0, Cr): the router rows W_r (exact activation decisions on
//            CUDA cores, see common.cuh) -> r, active, and per expert the mask
//            of tokens using it.  The other CTAs: the rows of [W_bar_up ;
//            W_s_up] -> u = x W_bar_up^T and the shared hidden
//            SiLU(x W_s_up^T), kept as bf16 hi/lo tiles.
//   phase U  once every router CTA is done: the union of the batch's active
//            experts (built by each CTA's producer warp for all its warps).  Its W_up[e] rows are a sequence of 128-column stages
//            (run by run, a run being 128 rows of one expert's matrix), and
//            every CTA takes a contiguous share of it, writing one fp32 piece
//            of g = x W_up[e]^T per run it touches.  At the end of its share
//            a CTA counts its stages of each expert; the CTA that completes an
//            expert computes its NormSiLU for every token using it (the
//            pieces added in CTA order, subtract u, RMS over d_e, SiLU, times
//            s_e r_e) as a bf16 hi/lo tile.
//   phase D  units (128 output rows, then one K part of W_s_down or one active
//            expert's W_down[e] in ascending order); a CTA adds its
//            consecutive units of one row block in its tensor-core
//            accumulators and writes one fp32 partial per row block (at most
//            two).  At the end of its share it counts them; the CTA that
//            completes a row block adds its partials in CTA order (+ the
//            residual) and writes the output rows: a fixed order, so the
//            result is bitwise reproducible.
//
// The same kernel with no routed experts is the equal-parameter dense FFN at
// decode batch sizes.
//
// Data movement: 8 consumer warps, 1 producer warp and 1 loader warp per CTA.
// The producer streams the CTA's weights in one continuous sequence of 33 KB
// stages behind mbarriers: phase R rows as bulk copies into 16-byte padded
// rows, phase U and D tiles as 128-row x 64-column TMA boxes in the 128-byte
// swizzle (ldmatrix reads both without bank conflicts).  It needs only the
// union of active experts, so the W_up and W_down streams run ahead of the
// consumers' dependencies.  x stays resident in shared memory during phases R
// and U; in phase D the loader warp waits for each unit's 16 KB activation
// tile to be ready and brings it in with cp.async into a ring of up to four
// tiles.  (The loader has a warp of its own: spinning lanes in the producer's
// warp would take issue slots from the lane that streams the weights.)
//
// Arithmetic: the projections are thin dense contractions done with mma.sync
// m16n8k16 (bf16 in, fp32 accumulate), weights as A, tokens as B: one
// tensor-core instruction per 16x8x16 tile keeps the instruction count well
// below the memory time.  Intermediates fed back into a contraction (the
// shared hidden activations and the scaled NormSiLU outputs) are bf16 pairs
// hi + lo with lo = bf16(v - hi), and both halves are multiplied, so they
// carry ~16 significant bits instead of 8.
//
// Waits are bounded: after about a second a wait gives up, sets bit 2 of the
// device error word and the CTA stops issuing work; before it exits it waits
// (again bounded) for every copy it issued.  No trap, no assert.
#pragma once

#include <cooperative_groups.h>
#include <cuda.h>

#include "common.cuh"

namespace deco {
namespace dec {

constexpr int kConsumerWarps = 8;
constexpr int kConsumerThreads = kConsumerWarps * 32;
constexpr int kProducerWarp = kConsumerWarps;       // weight ring (lane 0)
constexpr int kLoaderWarp = kConsumerWarps + 1;     // phase-D activation tiles
constexpr int kThreads = kConsumerThreads + 64;
constexpr int kMaxT = 16;                      // decode batches
constexpr int kTok = 16;                       // token rows of every activation tile
constexpr uint32_t kStageBytes = 33792;        // a ring stage: two TMA boxes, or <= 8 padded weight rows
constexpr int kMaxStages = 8;
constexpr size_t kSmemLimit = 232448;          // 227 KB opt-in per CTA on sm_100
constexpr long long kWaitCycles = 2000000000ll;  // ~1 s at 1.9 GHz
constexpr int kErrTimeout = 2;
constexpr int kMaxSms = 160;                  // kd_layer grids (one CTA per SM) up to this size
constexpr int kDRows = 128;                    // weight rows per phase-U run and phase-D unit
constexpr uint32_t kBoxBytes = kDRows * 128;   // 128 rows x 64 bf16 columns
constexpr int kSq = 256;                       // K columns per shared-expert down unit
constexpr int kTileElems = kTok * 2 * kSq;     // activation tile: 16 rows x (256 hi | 256 lo) bf16
constexpr uint32_t kTileBytes = kTileElems * 2;

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
// flags the CTA-wide abort word and the device error word) on timeout, or
// when another thread of the CTA has aborted.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag, int* err,
                                          long long limit = kWaitCycles) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (*abort_flag) return false;
    if (clock64() - t0 > limit) {
      *abort_flag = 1;
      atomicOr(err, kErrTimeout);
      return false;
    }
  }
  return true;
}
// Bounded wait that ignores the abort word: the drain of copies already
// issued, before a CTA that gave up exits.
__device__ __forceinline__ void mbar_drain(uint64_t* bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity) && clock64() - t0 < kWaitCycles) {
  }
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
__device__ __forceinline__ void consumer_sync() {   // the 8 consumer warps only
  asm volatile("bar.sync 1, %0;" ::"n"(kConsumerThreads) : "memory");
}
// 16-byte global -> shared copy through L2 (generic proxy; cp.async.wait_group)
__device__ __forceinline__ void cp_async16_cg(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
// arrive on `bar` once this thread's cp.async copies so far have landed
__device__ __forceinline__ void cp_async_mbar_arrive(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// inter-CTA counters (global memory, gpu scope)
__device__ __forceinline__ unsigned ld_acquire(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ unsigned atom_add_acq_rel(unsigned* p, unsigned v) {
  unsigned old;
  asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}
__device__ __forceinline__ void st_release(unsigned* p, unsigned v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
// Bounded wait (one thread) until *p >= target.  Returns false on timeout
// (setting the abort and error words) or when the CTA has aborted.
__device__ __forceinline__ bool spin_until(const unsigned* p, unsigned target, long long limit,
                                           volatile int* abort_flag, int* err) {
  if (ld_acquire(p) >= target) return true;
  const long long t0 = clock64();
  while (true) {
    __nanosleep(40);
    if (ld_acquire(p) >= target) return true;
    if (*abort_flag) return false;
    if (clock64() - t0 > limit) {
      *abort_flag = 1;
      atomicOr(err, kErrTimeout);
      return false;
    }
  }
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

// physical 16-byte chunk of logical chunk k in a row with index r: the low 3
// bits are XOR-ed with the row index, so 8 consecutive rows of one logical
// chunk sit in 8 different bank groups
__host__ __device__ __forceinline__ int row_chunk(int r, int k) { return (k & ~7) | ((k ^ r) & 7); }

// ---------------------------------------------------------------------------
// Shared-memory plan: [<= 1 KB alignment slack][barriers 1 KB][ring][operand].
// kStaticReserve bytes are left for the kernels' static __shared__ arrays.

constexpr uint32_t kHeaderBytes = 1024;
constexpr uint32_t kStaticReserve = 3072;

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

// Padded token rows of x: row t at t * x_pitch, so that ldmatrix reads of 8
// rows at one 16-byte column hit 8 different bank groups.
__host__ __device__ inline uint32_t x_pitch(int D) { return (uint32_t)D * 2u + 16u; }
// phase R streams <= 8 (D <= 2048) or 4 (D <= 4096) padded weight rows per stage
__host__ __device__ inline int rows_per_chunk(int D) { return D <= 2048 ? 8 : 4; }
// the operand region: 16 padded x rows and the 4 KB cross-warp reduction
// scratch (phases R, U), later two activation tiles (phase D)
__host__ __device__ inline uint32_t operand_bytes(int D) {
  const uint32_t xr = kTok * x_pitch(D) + 4096u;
  return xr > 2u * kTileBytes ? xr : 2u * kTileBytes;
}
__host__ __device__ inline SmemPlan layer_smem(int D) { return smem_plan(operand_bytes(D), kStageBytes); }
// phase-D activation tiles that fit the operand region (2..4)
__host__ __device__ inline int tile_slots(int D) {
  const int n = (int)(operand_bytes(D) / (uint32_t)kTileBytes);
  return n < 4 ? n : 4;
}

// router CTAs of phase R: one router row each (E <= 64), else several
__host__ __device__ inline int router_ctas(int E) { return E < 64 ? E : 64; }

__host__ __device__ inline int down_nsq(int d_s) { return (d_s + kSq - 1) / kSq; }

// CTA c's contiguous share [range_lo(c), range_lo(c + 1)) of n items (rows,
// stages or units) among G CTAs; (c + 1) * n and (i + 1) * G stay below 2^31
// for every count here (n <= 2^17, G <= kMaxSms)
__host__ __device__ inline int range_lo(int c, int n, int G) { return c * n / G; }
// the CTA whose range holds item i < n: the largest c with range_lo(c) <= i
__host__ __device__ inline int range_owner(int i, int n, int G) { return ((i + 1) * G - 1) / n; }

// ---------------------------------------------------------------------------

struct Args {
  int T, D, E, d_e, d_s;
  float eps;
  int residual;
  long long wait_cycles;   // limit of the waits for data (kWaitCycles unless a test lowers it)
  int pre_routed;          // r and act come from earlier kernels (TopK routing): no router CTAs
  int gated;               // gated experts: a = NormSiLU(x W_up^T - u) * (x W_val^T)
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
  unsigned* tmask;   // [E] bit t set iff token t activates expert e (written by the router CTAs)
  float* u;          // [T][d_e]
  bf16* HS;          // [nsq][16 tok][256 hi | 256 lo], chunk-swizzled rows: SiLU(x W_s_up^T)
  bf16* A;           // [E][16 tok][256 hi | 256 lo]: s_e r_e NormSiLU(x W_up[e]^T), 0 for
                     // tokens not using e
  float* Pu;         // [E * nbr * nrb_up + G][16 tok][128]: phase-U pieces, CTA c's sum of
                     // x W^T over its stages of run r in slot r + c
  float* Part;       // [G][2][16 tok][128]: a CTA's down-projection sum per row block
  unsigned* sync;    // inter-CTA counters (layout: SyncIdx); kd_layer clears them itself
  int* err;
  bf16* out;
};

// counters: router CTAs done, CTAs done with the other phase-R rows, up
// stages done per expert, NormSiLU tile ready per expert, CTAs done per
// output row block
struct SyncIdx {
  int route_done, pre_done, g_cnt, a_ready, rb_cnt, total;
};
__host__ __device__ inline SyncIdx sync_idx(int E, int D) {
  SyncIdx s;
  s.route_done = 0;
  s.pre_done = 1;
  s.g_cnt = 2;
  s.a_ready = 2 + E;
  s.rb_cnt = 2 + 2 * E;
  s.total = 2 + 2 * E + D / kDRows;
  return s;
}

// v as a bf16 pair (hi, lo = v - hi) at element j of a chunk-swizzled row of
// 2L elements (hi part [0, L), lo part [L, 2L)); r is the row index
__device__ __forceinline__ void store_row_hi_lo(bf16* row, int r, int L, int j, float v) {
  const bf16 hi = __float2bfloat16_rn(v);
  const bf16 lo = __float2bfloat16_rn(v - __bfloat162float(hi));
  row[row_chunk(r, j >> 3) * 8 + (j & 7)] = hi;
  row[row_chunk(r, (L + j) >> 3) * 8 + (j & 7)] = lo;
}

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

// ---------------------------------------------------------------------------
// Phase R, rows of [W_bar_up ; W_s_up]: a CTA's rows come in chunks of rc
// consecutive rows (one stage), each row one bulk copy into a 16-byte padded
// shared-memory row, the copies of a chunk issued by rc lanes at once (a bulk
// copy takes a while to issue).  For a chunk, warp w multiplies the 16 token
// rows of x (padded the same way) by the chunk's rows over columns
// [w*D/8, (w+1)*D/8): one m16n8 tile per 16-column step.  The 8 warps' 16 x 8
// results are then added in warp order.

__device__ __forceinline__ uint32_t x_addr(uint32_t xs, uint32_t pitch, int lane, int chunk) {
  return xs + (uint32_t)((lane & 7) + ((lane >> 3) & 1) * 8) * pitch + (uint32_t)(chunk + (lane >> 4)) * 16u;
}
// B operand (8 weight rows x 16 columns) from padded rows; rows >= rc (a
// chunk of fewer rows) repeat row 0, and their outputs are discarded
__device__ __forceinline__ uint32_t w_addr(uint32_t ws, uint32_t pitch, int lane, int chunk, int rc) {
  const int r = (lane & 7) < rc ? (lane & 7) : 0;
  return ws + (uint32_t)r * pitch + (uint32_t)(chunk + ((lane >> 3) & 1)) * 16u;
}

// the T row copies of x into padded rows, issued by lanes 0..T-1 of the
// calling warp in parallel (a bulk copy takes a while to issue); every lane
// of the warp calls this
__device__ __forceinline__ void stage_x(const Args& a, unsigned char* xs, uint64_t* bar, int lane) {
  if (lane == 0) mbar_expect_tx(bar, (uint32_t)a.T * a.D * 2);
  __syncwarp();
  if (lane < a.T)
    bulk_g2s(xs + (size_t)lane * x_pitch(a.D), a.x + (size_t)lane * a.D, (uint32_t)a.D * 2, bar);
}
// zero the rows T..15 of the 16-row x operand (consumer threads)
__device__ __forceinline__ void zero_x_tail(const Args& a, unsigned char* xs) {
  const uint32_t pitch = x_pitch(a.D);
  const int words = (int)(pitch / 16);
  for (int i = threadIdx.x; i < (kTok - a.T) * words; i += kConsumerThreads)
    reinterpret_cast<uint4*>(xs + (size_t)(a.T + i / words) * pitch)[i % words] = make_uint4(0u, 0u, 0u, 0u);
}

// y[16 tok][8 rows] for one chunk; thread o < 128 of the consumer warps gets
// output o = tok * 8 + row
__device__ __forceinline__ float chunk_gemv(uint32_t xs, uint32_t ws, uint32_t pitch, uint32_t wpitch, int D,
                                            int warp, int lane, float* red, bool math) {
  const int rc = rows_per_chunk(D);
  float d[4] = {0.f, 0.f, 0.f, 0.f};
  if (math) {
    const int c0 = warp * (D / 8) / 8, c1 = c0 + (D / 8) / 8;   // 16-byte chunks of this warp
    for (int ch = c0; ch < c1; ch += 2) {
      uint32_t a0, a1, a2, a3, b0, b1;
      ldsm_x4(x_addr(xs, pitch, lane, ch), a0, a1, a2, a3);
      ldsm_x2(w_addr(ws, wpitch, lane, ch, rc), b0, b1);
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
// Router rows (phase R of CTAs [0, Cr), and the routing-only kernel): rows
// e = c + Cr i of W_r, packed in one stage; for each row the 8 consumer warps
// split the D columns (16-byte chunks), and their partial sums are added in
// warp order.  The activation decision is exact: the fp32 sum comes with a
// rigorous error bound and, inside it, the sign is settled by exact integer
// accumulation (common.cuh).

__device__ __forceinline__ int router_rows(const Args& a, int c, int Cr) { return (a.E - c + Cr - 1) / Cr; }

// producer side: x and the router rows of CTA c into stage 0, issued by the
// lanes of the calling warp in parallel (every lane calls this)
__device__ __forceinline__ void issue_router(const Args& a, int c, int Cr, unsigned char* xsm, uint64_t* xbar,
                                             unsigned char* stage, uint64_t* full, uint64_t pol, int lane) {
  const int nrow = router_rows(a, c, Cr);   // <= 4
  const uint32_t rowbytes = (uint32_t)a.D * 2;
  if (lane == 0) mbar_expect_tx(full, nrow * rowbytes);
  stage_x(a, xsm, xbar, lane);              // (synchronises the warp first)
  const int j = lane - kTok;
  if (j >= 0 && j < nrow)
    bulk_g2s(stage + (size_t)j * rowbytes, a.W_r + (size_t)(c + Cr * j) * a.D, rowbytes, full, pol);
}

// consumer side: r and active of the CTA's rows for every token (8 warps);
// `ok` says the stage and x are in shared memory
__device__ __forceinline__ void route_rows(const Args& a, int c, int Cr, const unsigned char* xsm,
                                           const unsigned char* stage, float* red, unsigned long long* limbs,
                                           bool ok) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t pitch = x_pitch(a.D);
  const int nrow = router_rows(a, c, Cr);
  // a value goes through <= 8 ceil(D / 2048) products in its lane, 5
  // butterfly levels, 7 cross-warp additions and the bias
  const int n_terms = 8 * ((a.D + 2047) / 2048) + 16;
  const float gm = gamma_f32(n_terms);
  const float bscale = 2.f * gm * (1.f + 2.f * gm);
  const float tiny = float(n_terms) * 2.8025969e-45f;
  bool bad = false;
  for (int i = 0; i < nrow; ++i) {
    const int e = c + Cr * i;
    const bf16* wrow = reinterpret_cast<const bf16*>(stage + (size_t)i * a.D * 2);
    float v[32];
#pragma unroll
    for (int q = 0; q < 32; ++q) v[q] = 0.f;
    // z partials in v[t], sum |x w| partials in v[16 + t]
    if (ok) {
#pragma unroll 1
      for (int ch = warp * 32 + lane; ch < a.D / 8; ch += kConsumerWarps * 32) {
        float wv[8];
        unpack16(*reinterpret_cast<const uint4*>(wrow + (size_t)ch * 8), wv);
#pragma unroll
        for (int t = 0; t < kTok; ++t) {
          if (t < a.T) {
            float xv[8];
            unpack16(*reinterpret_cast<const uint4*>(xsm + (size_t)t * pitch + (size_t)ch * 16), xv);
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
                                       limbs, &bad);
        if (lane == tt) on = sg > 0;
      }
      if (mine) {
        a.r[(size_t)t * a.E + e] = on ? fmaxf(z, 0.f) : 0.f;
        a.act[(size_t)t * a.E + e] = on ? 1 : 0;
      }
      const unsigned m = __ballot_sync(kFull, mine && on);
      if (lane == 0) a.tmask[e] = m;

    }
    consumer_sync();   // red is reused by the next row
  }
  if (bad && (threadIdx.x & 31) == 0) atomicOr(a.err, 1);
}

// Barriers and bookkeeping kept in the 1 KB header: weight ring full/empty,
// x landed, union built, the producer's last word (stages issued), x
// released by the consumers, activation-tile ring full/empty.
constexpr int kTileSlots = 4;                  // phase-D activation tiles in flight (at most)
constexpr int kLoaderLanes = 32;               // the loader warp's lanes load them

struct Ctl {
  uint64_t* full;
  uint64_t* empty;
  uint64_t* xbar;
  uint64_t* ubar;    // the producer warp has built the union of active experts
  uint64_t* pbar;
  uint64_t* xfree;   // consumers are done with x (its region then holds the tile ring)
  uint64_t* tfull;   // [kTileSlots] activation tile landed
  uint64_t* tempty;  // [kTileSlots] consumers done with the tile
  volatile int* abort_flag;
  volatile int* k_issued;
  int* bcast;        // [4] consumer broadcast words
  unsigned char* stage;
  uint32_t stage_bytes;
  int nstages;
};

__device__ __forceinline__ unsigned char* ctl_setup(unsigned char* smem_raw, const SmemPlan& sp, Ctl& c) {
  unsigned char* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem);
  c.full = bars;
  c.empty = bars + kMaxStages;
  c.xbar = bars + 2 * kMaxStages;
  c.ubar = c.xbar + 1;
  c.pbar = c.xbar + 2;
  c.xfree = c.xbar + 3;
  c.tfull = c.xbar + 4;
  c.tempty = c.tfull + kTileSlots;
  int* words = reinterpret_cast<int*>(c.tempty + kTileSlots);
  c.abort_flag = words;
  c.k_issued = words + 1;
  c.bcast = words + 2;
  c.stage = smem + sp.ring_off;
  c.stage_bytes = sp.stage_bytes;
  c.nstages = sp.nstages;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kMaxStages; ++s) {
      mbar_init(&c.full[s], 1);
      mbar_init(&c.empty[s], kConsumerWarps);
    }
    mbar_init(c.xbar, 1);
    mbar_init(c.ubar, 1);
    mbar_init(c.pbar, 1);
    mbar_init(c.xfree, kConsumerWarps);
    for (int s = 0; s < kTileSlots; ++s) {
      mbar_init(&c.tfull[s], kLoaderLanes);
      mbar_init(&c.tempty[s], kConsumerWarps);
    }
    *c.abort_flag = 0;
    *c.k_issued = 0;
    fence_barrier_init();
  }
  __syncthreads();
  return smem;
}

// ---------------------------------------------------------------------------
// Routing alone (deco_moe_routing on decode batches): the router CTAs of
// kd_layer's phase R, with the same code, so the same decisions bit for bit.

__global__ void __launch_bounds__(kThreads, 1) kd_router(const __grid_constant__ Args a) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  __shared__ unsigned long long limbs[kLimbs];
  const int Cr = router_ctas(a.E);
  const SmemPlan sp = layer_smem(a.D);
  Ctl ctl;
  unsigned char* smem = ctl_setup(smem_raw, sp, ctl);
  unsigned char* xsm = smem + sp.op_off;
  float* red = reinterpret_cast<float*>(xsm + kTok * x_pitch(a.D));
  const int warp = threadIdx.x >> 5;
  if (warp == kProducerWarp) {
    issue_router(a, blockIdx.x, Cr, xsm, ctl.xbar, ctl.stage, &ctl.full[0], evict_first_policy(),
                 threadIdx.x & 31);
    return;
  }
  if (warp == kLoaderWarp) return;
  // both waits always run (bounded), so every issued copy lands before exit
  bool ok = mbar_wait(ctl.xbar, 0, ctl.abort_flag, a.err, a.wait_cycles);
  ok = mbar_wait(&ctl.full[0], 0, ctl.abort_flag, a.err, a.wait_cycles) && ok;
  ok = __all_sync(kFull, ok);   // warp-uniform: it guards warp-collective instructions
  if (!ok && (threadIdx.x & 31) == 0) {
    mbar_drain(ctl.xbar, 0);
    mbar_drain(&ctl.full[0], 0);
  }
  route_rows(a, blockIdx.x, Cr, xsm, ctl.stage, red, limbs, ok);
}

// ---------------------------------------------------------------------------
// The layer.

// The schedule of phases U and D.  Phase U is a sequence of stages: run r
// (one block of 128 rows of W_up[e] or W_val[e]) is stages r * nkc ..
// r * nkc + nkc - 1, 128 columns each, an expert's runs consecutive.  Every
// CTA takes a contiguous share of the stages, which may begin or end inside a
// run (shares differ by one stage at most); it writes one piece per run it
// touches.  Phase D: every CTA takes a contiguous share of the units.
struct Sched {
  int U;              // active experts (the union)
  int nbr;            // up-projection matrices per expert: W_up, and W_val when gated
  int nrb_up, nkc;    // runs per matrix, stages per run
  int NS;             // phase-U stages
  int nrb, nsq;
  int J, ND;          // phase-D units per row block, and in all
};

__device__ __forceinline__ Sched make_sched(const Args& a, int U, int G) {
  Sched S;
  S.U = U;
  S.nrb_up = (a.d_e + kDRows - 1) / kDRows;
  S.nkc = a.D / 128;
  S.nrb = a.D / kDRows;
  S.nsq = down_nsq(a.d_s);
  S.nbr = a.gated ? 2 : 1;
  S.NS = U * S.nbr * S.nrb_up * S.nkc;
  S.J = S.nsq + U;
  S.ND = S.nrb * S.J;
  return S;
}

// run r of phase U: index of its expert in the union, the matrix (0 W_up,
// 1 W_val) and the block of 128 rows of it
struct URun {
  int ei, mat, rbu;
};
__device__ __forceinline__ URun up_run(const Sched& S, int r) {
  URun q;
  q.rbu = r % S.nrb_up;
  const int m = r / S.nrb_up;
  q.mat = m % S.nbr;
  q.ei = m / S.nbr;
  return q;
}

// Unit v of phase D: row block rb of the output, then j < nsq a K part of
// W_s_down, the rest the active experts' W_down in ascending order.
struct DUnit {
  int rb, j, e, K, col0;
};
__device__ __forceinline__ DUnit down_unit(const Args& a, const uint8_t* ulist, const Sched& S, int v) {
  DUnit d;
  d.rb = v / S.J;
  d.j = v - d.rb * S.J;
  if (d.j < S.nsq) {
    d.e = -1;
    d.col0 = d.j * kSq;
    d.K = min(kSq, a.d_s - d.col0);
  } else {
    d.e = ulist[d.j - S.nsq];
    d.col0 = 0;
    d.K = a.d_e;
  }
  return d;
}

// The producer's walk over its stages: phase-U stages [sg, s1), then the
// phase-D units [v, v1), unit v from column c0.  pwalk_get gives the tensor
// map and coordinates of the current stage's first box (a second box, when
// nb = 2, is 64 columns on); false once the walk is over.
struct PWalk {
  int sg, s1, v, v1, c0;
};
struct PStage {
  const CUtensorMap* m;
  int col, row, nb;
};
__device__ __forceinline__ bool pwalk_get(const Args& a, const Sched& S, const uint8_t* ulist, const PWalk& w,
                                          const CUtensorMap* tmU, const CUtensorMap* tmV, const CUtensorMap* tmW,
                                          const CUtensorMap* tmS, PStage& st) {
  if (w.sg < w.s1) {
    const int r = w.sg / S.nkc, kc = w.sg - r * S.nkc;
    const URun q = up_run(S, r);
    st.m = q.mat ? tmV : tmU;
    st.col = kc * 128;
    st.row = ulist[q.ei] * a.d_e + q.rbu * kDRows;
    st.nb = 2;
    return true;
  }
  if (w.v < w.v1) {
    const DUnit d = down_unit(a, ulist, S, w.v);
    const bool sh = d.e < 0;
    st.m = sh ? tmS : tmW;
    st.col = d.col0 + w.c0;
    st.row = sh ? d.rb * kDRows : d.e * a.D + d.rb * kDRows;
    st.nb = min(2, (d.K - w.c0) / 64);
    return true;
  }
  return false;
}
__device__ __forceinline__ void pwalk_next(const Args& a, const Sched& S, const uint8_t* ulist, PWalk& w) {
  if (w.sg < w.s1) {
    ++w.sg;
  } else if (w.v < w.v1) {
    w.c0 += 128;
    if (w.c0 >= down_unit(a, ulist, S, w.v).K) {
      w.c0 = 0;
      ++w.v;
    }
  }
}

// The partials of row block rb in the fixed order of the combine: the CTAs
// whose unit range meets rb, ascending (one warp: lane l tests CTAs l,
// l + 32, ...).  Returns the count and fills src[i] = 2 c + (which of the
// CTA's two row blocks).
__device__ __forceinline__ int rb_sources(int rb, const Sched& S, int G, int* src) {
  const int lane = threadIdx.x & 31;
  int n = 0;
  for (int c0 = 0; c0 < G; c0 += 32) {
    const int c = c0 + lane;
    bool hit = false;
    int slot = 0;
    if (c < G) {
      const int v0 = range_lo(c, S.ND, G), v1 = range_lo(c + 1, S.ND, G);
      hit = v0 < v1 && v0 < (rb + 1) * S.J && v1 > rb * S.J;
      slot = rb - v0 / S.J;
    }
    const unsigned m = __ballot_sync(kFull, hit);
    if (hit) src[n + __popc(m & ((1u << lane) - 1u))] = 2 * c + slot;
    n += __popc(m);
  }
  return n;
}

__device__ __forceinline__ void add4(float4& a, const float4& b) {
  a.x += b.x;
  a.y += b.y;
  a.z += b.z;
  a.w += b.w;
}

// Lane's 8 features of run r for token t: the pieces of the CTAs whose stage
// shares meet the run, added in CTA order (up to 4 pieces' loads in flight).
// The next such CTA owns the stage after the current one's share (CTAs with
// an empty share, when there are fewer stages than CTAs, are skipped).
__device__ __forceinline__ void run_sum(const Args& a, const Sched& S, int G, int r, int t, int row0, bool live,
                                        float4& g0, float4& g1) {
  g0 = make_float4(0.f, 0.f, 0.f, 0.f);
  g1 = g0;
  if (!live) return;
  const int end = (r + 1) * S.nkc;   // the stage after the run
  int cc = range_owner(r * S.nkc, S.NS, G);
  while (cc >= 0) {
    float4 v[4][2];
    bool has[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      has[i] = cc >= 0;
      if (has[i]) {
        const float4* src = reinterpret_cast<const float4*>(a.Pu + ((size_t)(r + cc) * kTok + t) * kDRows + row0);
        v[i][0] = __ldcg(src);
        v[i][1] = __ldcg(src + 1);
        const int nxt = range_lo(cc + 1, S.NS, G);
        cc = nxt < end ? range_owner(nxt, S.NS, G) : -1;
      }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      if (has[i]) {
        add4(g0, v[i][0]);
        add4(g1, v[i][1]);
      }
    }
  }
}

// NormSiLU tile of expert e, the ei-th of the union (consumer threads): g =
// x W_up[e]^T from its pieces, c = g - u, h = c / sqrt(mean c^2 + eps), a =
// s_e r_e SiLU(h) (times x W_val[e]^T for gated experts) as hi/lo rows; rows
// of tokens not using e are zero.
__device__ void norm_silu_tile(const Args& a, const Sched& S, int G, int e, int ei, uint32_t m_e) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  bf16* tile = a.A + (size_t)e * kTileElems;
  for (int i = threadIdx.x; i < kTok * 64; i += kConsumerThreads) {   // 64 chunks of 16 B per row
    const int t = i >> 6;
    if (!((m_e >> t) & 1u)) reinterpret_cast<uint4*>(tile)[i] = make_uint4(0u, 0u, 0u, 0u);
  }
  const int n_e = __popc(m_e);
  const bool live = 8 * lane < a.d_e;   // lane l holds features 8 l .. 8 l + 7
  const int rbu = (8 * lane) / kDRows, row0 = (8 * lane) % kDRows;
  const int r_up = (ei * S.nbr) * S.nrb_up + rbu;
  for (int slot = warp; slot < n_e; slot += kConsumerWarps) {
    uint32_t m = m_e;
    for (int i = 0; i < slot; ++i) m &= m - 1;
    const int t = __ffs(m) - 1;
    const float rte = __ldcg(a.r + (size_t)t * a.E + e);
    const float se = __ldg(a.s + e);
    float4 uq[2];
    const float4* usrc = reinterpret_cast<const float4*>(a.u + (size_t)t * a.d_e) + 2 * lane;
    uq[0] = live ? __ldcg(usrc) : make_float4(0.f, 0.f, 0.f, 0.f);
    uq[1] = live ? __ldcg(usrc + 1) : make_float4(0.f, 0.f, 0.f, 0.f);
    float4 g[2];
    run_sum(a, S, G, r_up, t, row0, live, g[0], g[1]);
    float cv[8];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      cv[4 * h + 0] = g[h].x - uq[h].x;
      cv[4 * h + 1] = g[h].y - uq[h].y;
      cv[4 * h + 2] = g[h].z - uq[h].z;
      cv[4 * h + 3] = g[h].w - uq[h].w;
    }
    float ss = 0.f;
#pragma unroll
    for (int q = 0; q < 8; ++q) ss = fmaf(cv[q], cv[q], ss);
    // gated experts: the value branch
    float val[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) val[q] = 1.f;
    if (a.gated) {
      float4 vg[2];
      run_sum(a, S, G, r_up + S.nrb_up, t, row0, live, vg[0], vg[1]);
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        val[4 * h + 0] = vg[h].x;
        val[4 * h + 1] = vg[h].y;
        val[4 * h + 2] = vg[h].z;
        val[4 * h + 3] = vg[h].w;
      }
    }
    ss = warp_sum(ss);
    const float rinv = 1.f / sqrtf(ss / float(a.d_e) + a.eps);
    const float coef = se * rte;
    if (live) {
      uint32_t hi[4], lo[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float v0 = coef * silu_f(cv[2 * q] * rinv) * val[2 * q];
        const float v1 = coef * silu_f(cv[2 * q + 1] * rinv) * val[2 * q + 1];
        const __nv_bfloat162 h2 = __floats2bfloat162_rn(v0, v1);
        const float2 hf = __bfloat1622float2(h2);
        const __nv_bfloat162 l2 = __floats2bfloat162_rn(v0 - hf.x, v1 - hf.y);
        hi[q] = *reinterpret_cast<const uint32_t*>(&h2);
        lo[q] = *reinterpret_cast<const uint32_t*>(&l2);
      }
      bf16* row = tile + (size_t)t * 2 * kSq;
      reinterpret_cast<uint4*>(row)[row_chunk(t, lane)] = make_uint4(hi[0], hi[1], hi[2], hi[3]);
      reinterpret_cast<uint4*>(row)[row_chunk(t, kSq / 8 + lane)] = make_uint4(lo[0], lo[1], lo[2], lo[3]);
    }
  }
}

// out rows of row block rb: the sources' partials in CTA order (+ x).  A
// thread owns output float4s o and o + 256 (T * 32 of them); up to
// kCombineBatch sources' loads for both are in flight before they are added
// in order (a row block has about ten sources).
constexpr int kCombineBatch = 12;

__device__ void combine_rb(const Args& a, int rb, const int* src, int n) {
  constexpr int kQ = kDRows / 4;   // float4s per token row of a block
  const int n4 = a.T * kQ;
  for (int o0 = threadIdx.x; o0 < n4; o0 += 2 * kConsumerThreads) {
    const int o1 = o0 + kConsumerThreads;
    const bool two = o1 < n4;
    const int t0 = o0 / kQ, q0 = o0 - t0 * kQ;
    const int t1 = two ? o1 / kQ : t0, q1 = two ? o1 - t1 * kQ : q0;
    float4 acc0 = make_float4(0.f, 0.f, 0.f, 0.f), acc1 = acc0;
    for (int i = 0; i < n; i += kCombineBatch) {
      float4 v0[kCombineBatch], v1[kCombineBatch];
#pragma unroll
      for (int k = 0; k < kCombineBatch; ++k) {
        if (i + k < n) {
          const float* P = a.Part + (size_t)src[i + k] * kTok * kDRows;
          v0[k] = __ldcg(reinterpret_cast<const float4*>(P + (size_t)t0 * kDRows) + q0);
          v1[k] = __ldcg(reinterpret_cast<const float4*>(P + (size_t)t1 * kDRows) + q1);
        }
      }
#pragma unroll
      for (int k = 0; k < kCombineBatch; ++k) {
        if (i + k < n) {
          add4(acc0, v0[k]);
          add4(acc1, v1[k]);
        }
      }
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      if (h == 1 && !two) break;
      float4 acc = h ? acc1 : acc0;
      const size_t o_idx = (size_t)(h ? t1 : t0) * a.D + (size_t)rb * kDRows + 4 * (h ? q1 : q0);
      if (a.residual) {
        const uint2 xr = *reinterpret_cast<const uint2*>(a.x + o_idx);
        acc.x += __uint_as_float(xr.x << 16);
        acc.y += __uint_as_float(xr.x & 0xffff0000u);
        acc.z += __uint_as_float(xr.y << 16);
        acc.w += __uint_as_float(xr.y & 0xffff0000u);
      }
      const __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x, acc.y), hi = __floats2bfloat162_rn(acc.z, acc.w);
      uint2 w;
      w.x = *reinterpret_cast<const uint32_t*>(&lo);
      w.y = *reinterpret_cast<const uint32_t*>(&hi);
      *reinterpret_cast<uint2*>(a.out + o_idx) = w;
    }
  }
}

__global__ void __launch_bounds__(kThreads, 1)
    kd_layer(const __grid_constant__ CUtensorMap tmU, const __grid_constant__ CUtensorMap tmV,
             const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmS,
             const __grid_constant__ Args a) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  __shared__ unsigned long long limbs[kLimbs];
  __shared__ uint16_t emask[256];   // the union, built by the producer warp: token masks,
  __shared__ uint8_t ulist[256];    // active experts and their count (then read-only)
  __shared__ int s_U;
  __shared__ int s_src[2 * kMaxSms];   // the sources of the (at most two) row blocks of a share
  __shared__ int s_nsrc[2];
  __shared__ int s_done[32];            // (index in the union << 16) | stages, per expert of a share
  const int G = gridDim.x, c = blockIdx.x;
  const int Cr = (a.E > 0 && !a.pre_routed) ? router_ctas(a.E) : 0;
  const bool router_cta = c < Cr;
  const uint32_t pitch = x_pitch(a.D);
  const SmemPlan sp = layer_smem(a.D);
  if (threadIdx.x == 0) s_U = 0;
  Ctl ctl;
  unsigned char* smem = ctl_setup(smem_raw, sp, ctl);
  unsigned char* xsm = smem + sp.op_off;
  float* red = reinterpret_cast<float*>(xsm + kTok * pitch);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const SyncIdx si = sync_idx(a.E, a.D);
  unsigned* sync = a.sync;
  // phase R rows of a non-router CTA
  const int nrows = a.d_e + a.d_s;
  const int Gp = G - Cr, cp = c - Cr;
  const int ra = router_cta ? 0 : range_lo(cp, nrows, Gp), rbr = router_cta ? 0 : range_lo(cp + 1, nrows, Gp);
  const int rc = rows_per_chunk(a.D);
  const int nchunks = (rbr - ra + rc - 1) / rc;

  // x (and a router CTA's rows, into stage 0 of the first round, which is
  // free) are issued by the producer warp's lanes in parallel, and are in
  // flight while the counters are cleared
  const uint64_t pol = evict_first_policy();
  if (warp == kProducerWarp) {
    if (router_cta) issue_router(a, c, Cr, xsm, ctl.xbar, ctl.stage, &ctl.full[0], pol, lane);
    else stage_x(a, xsm, ctl.xbar, lane);
  }
  // Every call starts with its counters at zero: CTA 0 clears them (and the
  // error word, unless earlier kernels of the call may have set it), and the
  // grid-wide barrier of the cooperative launch orders that before any use.
  if (c == 0) {
    for (int i = threadIdx.x; i < si.total; i += blockDim.x) sync[i] = 0u;
    if (!a.pre_routed && threadIdx.x == 0) *a.err = 0;
  }
  cooperative_groups::this_grid().sync();

  if (warp == kProducerWarp) {
    // ---------------- producer warp ----------------
    int k = router_cta ? 1 : 0;
    bool ok = true;
    auto next_stage = [&](int& s) -> bool {   // lane 0: wait for a free stage
      s = k % ctl.nstages;
      return mbar_wait(&ctl.empty[s], ((k / ctl.nstages) & 1) ^ 1, ctl.abort_flag, a.err, a.wait_cycles);
    };
    // phase R rows of a non-router CTA: chunks of consecutive rows of
    // [W_bar_up ; W_s_up], one bulk copy per row, issued by rc lanes at once
    if (!router_cta) {
      const uint32_t rowbytes = (uint32_t)a.D * 2;
      for (int ch = 0; ch < nchunks && ok; ++ch) {
        int s = 0;
        if (lane == 0) {
          ok = next_stage(s);
          if (ok) mbar_expect_tx(&ctl.full[s], (uint32_t)min(rc, rbr - (ra + ch * rc)) * rowbytes);
        }
        ok = __shfl_sync(kFull, ok, 0);
        s = __shfl_sync(kFull, s, 0);
        if (!ok) break;
        const int g = ra + ch * rc + lane;   // lane i copies row i of the chunk into a padded row
        if (lane < rc && g < rbr) {
          const bf16* src = g < a.d_e ? a.W_bar + (size_t)g * a.D : a.W_s_up + (size_t)(g - a.d_e) * a.D;
          bulk_g2s(ctl.stage + (size_t)s * ctl.stage_bytes + (size_t)lane * pitch, src, rowbytes, &ctl.full[s],
                   pol);
        }
        ++k;
      }
    }
    // the union of active experts, for every warp of the CTA (published
    // through ubar): the router rows' token masks, once every router CTA is
    // done (one thread per CTA waits on the count)
    if (lane == 0 && ok && !a.pre_routed)
      ok = spin_until(sync + si.route_done, (unsigned)Cr, a.wait_cycles, ctl.abort_flag, a.err);
    ok = __shfl_sync(kFull, ok, 0);
    if (ok) {
      if (!a.pre_routed) ld_acquire(sync + si.route_done);   // each lane acquires the router CTAs' writes
      for (int e = lane; e < a.E; e += 32) {
        uint32_t m = 0;
        if (a.pre_routed) {   // decisions from earlier kernels: scan act
#pragma unroll
          for (int t = 0; t < kTok; ++t)
            if (t < a.T && __ldcg(a.act + (size_t)t * a.E + e)) m |= 1u << t;
        } else {
          m = __ldcg(a.tmask + e);
        }
        emask[e] = (uint16_t)m;
      }
    }
    __syncwarp();
    if (ok) {
      int n = 0;
      for (int base = 0; base < a.E; base += 32) {
        const int e = base + lane;
        const bool f = e < a.E && emask[e] != 0;
        const unsigned bal = __ballot_sync(kFull, f);
        if (f) ulist[n + __popc(bal & ((1u << lane) - 1u))] = (uint8_t)e;
        n += __popc(bal);
      }
      if (lane == 0) s_U = n;
    } else if (lane == 0) {
      s_U = 0;
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(ctl.ubar);   // the other warps read the union (or see the abort)
    if (lane != 0) return;
    const int U = s_U;
    {
      const Sched S = make_sched(a, U, G);
      // phases U and D: W_up (W_val) boxes, then W_s_down / W_down boxes,
      // one or two per stage
      PWalk w{range_lo(c, S.NS, G), range_lo(c + 1, S.NS, G), range_lo(c, S.ND, G), range_lo(c + 1, S.ND, G), 0};
      PStage ps;
      while (ok && pwalk_get(a, S, ulist, w, &tmU, &tmV, &tmW, &tmS, ps)) {
        int s;
        if (!(ok = next_stage(s))) break;
        mbar_expect_tx(&ctl.full[s], (uint32_t)ps.nb * kBoxBytes);
        for (int b = 0; b < ps.nb; ++b)
          tma_2d(ctl.stage + (size_t)s * ctl.stage_bytes + b * kBoxBytes, ps.m, ps.col + 64 * b, ps.row,
                 &ctl.full[s], pol);
        pwalk_next(a, S, ulist, w);
        ++k;
      }
      *ctl.k_issued = k;
      mbar_arrive(ctl.pbar);
    }
    return;
  }

  if (warp == kLoaderWarp) {
    // ---------------- loader warp ----------------
    // the activation tile of each phase-D unit, in order, into the tile ring
    // (the x region, once the consumers are done with x)
    bool lok = mbar_wait(ctl.ubar, 0, ctl.abort_flag, a.err, a.wait_cycles);
    const Sched S = make_sched(a, lok ? s_U : 0, G);
    const int nslots = tile_slots(a.D);
    const int v0 = range_lo(c, S.ND, G), v1 = range_lo(c + 1, S.ND, G);
    lok = lok && v0 < v1 && mbar_wait(ctl.xfree, 0, ctl.abort_flag, a.err, a.wait_cycles);
    {
      for (int v = v0; v < v1 && lok; ++v) {
        const int i = v - v0;
        const int slot = i % nslots;
        if (!(lok = mbar_wait(&ctl.tempty[slot], ((i / nslots) & 1) ^ 1, ctl.abort_flag, a.err, a.wait_cycles)))
          break;
        const DUnit d = down_unit(a, ulist, S, v);
        const unsigned* f = d.e < 0 ? sync + si.pre_done : sync + si.a_ready + d.e;
        if (!(lok = spin_until(f, d.e < 0 ? (unsigned)Gp : 1u, a.wait_cycles, ctl.abort_flag, a.err))) break;
        const unsigned char* src = reinterpret_cast<const unsigned char*>(
            d.e < 0 ? a.HS + (size_t)d.j * kTileElems : a.A + (size_t)d.e * kTileElems);
        unsigned char* dst = xsm + (size_t)slot * kTileBytes;
        for (int q = lane; q < (int)(kTileBytes / 16); q += kLoaderLanes)
          cp_async16_cg(dst + (size_t)q * 16, src + (size_t)q * 16);
        cp_async_mbar_arrive(&ctl.tfull[slot]);
      }
    }
    cp_async_wait_all();   // every copy lands before the warp exits
    return;
  }

  // ---------------- consumer warps ----------------
  const uint32_t x_u32 = smem_u32(xsm);
  int k = 0;          // ring stages consumed
  int k_ok = 0;       // stages whose data this thread saw arrive
  bool ok = true;
  // `ok` is kept warp-uniform (it guards ldmatrix / mma.sync / ballots); every
  // consumer thread runs the same loops and barriers whatever its value
  auto wait_full = [&]() -> bool {
    const int s = k % ctl.nstages;
    bool w = ok && mbar_wait(&ctl.full[s], (k / ctl.nstages) & 1, ctl.abort_flag, a.err, a.wait_cycles);
    if (w) k_ok = k + 1;
    return __all_sync(kFull, w);
  };
  auto release = [&](int s) {   // the warp is done with stage s
    __syncwarp();
    if (lane == 0) mbar_arrive(&ctl.empty[s]);
  };
  zero_x_tail(a, xsm);
  consumer_sync();
  const bool x_ok = mbar_wait(ctl.xbar, 0, ctl.abort_flag, a.err, a.wait_cycles);
  ok = __all_sync(kFull, x_ok);

  // ---- phase R ----
  if (router_cta) {
    const int s = k % ctl.nstages;
    ok = wait_full();
    route_rows(a, c, Cr, xsm, ctl.stage + (size_t)s * ctl.stage_bytes, red, limbs, ok);
    release(s);
    ++k;
  } else {
    for (int ch = 0; ch < nchunks; ++ch) {
      const int s = k % ctl.nstages;
      ok = wait_full();
      const float v = chunk_gemv(x_u32, smem_u32(ctl.stage + (size_t)s * ctl.stage_bytes), pitch, pitch, a.D,
                                 warp, lane, red, ok);
      release(s);
      ++k;
      const int o = threadIdx.x;
      const int t = o >> 3, i = o & 7;
      const int g = ra + ch * rc + i;
      if (ok && o < 128 && i < rc && g < rbr) {
        if (g < a.d_e) {
          if (t < a.T) a.u[(size_t)t * a.d_e + g] = v;
        } else {
          const int j = g - a.d_e;   // shared hidden unit
          store_row_hi_lo(a.HS + (size_t)(j / kSq) * kTileElems + (size_t)t * 2 * kSq, t, kSq, j % kSq,
                          t < a.T ? silu_f(v) : 0.f);
        }
      }
    }
  }
  consumer_sync();
  if (threadIdx.x == 0)   // releases every consumer thread's phase-R writes (they precede the barrier)
    atom_add_acq_rel(sync + (router_cta ? si.route_done : si.pre_done), 1u);

  // ---- the union of active experts, from the producer warp ----
  ok = __all_sync(kFull, ok && mbar_wait(ctl.ubar, 0, ctl.abort_flag, a.err, a.wait_cycles));
  const int U = ok ? s_U : 0;
  const Sched S = make_sched(a, U, G);
  const int ntiles = (a.T + 7) / 8;
  // this CTA's phase-D row blocks (at most two) and the sources of their
  // partials, found now rather than at the end of the kernel
  const int dv0 = range_lo(c, S.ND, G), dv1 = range_lo(c + 1, S.ND, G);
  const int rb0 = dv0 < dv1 ? dv0 / S.J : 0;
  const int n_rb = dv0 < dv1 ? (dv1 - 1) / S.J - rb0 + 1 : 0;
  if (warp == 0) {
    const int n0 = n_rb > 0 ? rb_sources(rb0, S, G, s_src) : 0;
    const int n1 = n_rb > 1 ? rb_sources(rb0 + 1, S, G, s_src + kMaxSms) : 0;
    if (lane == 0) {
      s_nsrc[0] = n0;
      s_nsrc[1] = n1;
    }
  }

  // ---- phase U ----
  {
    const int s0 = range_lo(c, S.NS, G), s1 = range_lo(c + 1, S.NS, G);
    const int per_e = S.nbr * S.nrb_up * S.nkc;   // stages of one expert
    int n_here = 0;                                 // this CTA's stages of the current expert
    int n_done = 0;                                 // experts this share touched (s_done)
    float acc[2][4] = {};
    for (int sg = s0; sg < s1; ++sg) {
      const int r = sg / S.nkc, kc = sg - r * S.nkc;
      const URun q = up_run(S, r);
      ++n_here;
      {
        const int s = k % ctl.nstages;
        const bool w = wait_full();
        ok = ok && w;
        if (ok) {
          const uint32_t st = smem_u32(ctl.stage + (size_t)s * ctl.stage_bytes);
#pragma unroll
          for (int b = 0; b < 2; ++b) {
            const uint32_t box = st + b * kBoxBytes;
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
              uint32_t a0, a1, a2, a3;
              ldsm_x4(swz(box, 16 * warp + (lane & 7) + ((lane >> 3) & 1) * 8, 2 * ks + (lane >> 4)), a0, a1, a2,
                      a3);
              const int kch = (kc * 128 + 64 * b) / 8 + 2 * ks + ((lane >> 3) & 1);
#pragma unroll
              for (int nt = 0; nt < 2; ++nt) {
                if (nt < ntiles) {
                  uint32_t b0, b1;
                  ldsm_x2(x_u32 + (uint32_t)(8 * nt + (lane & 7)) * pitch + (uint32_t)kch * 16u, b0, b1);
                  mma16816(acc[nt], a0, a1, a2, a3, b0, b1);
                }
              }
            }
          }
        }
        release(s);
        ++k;
      }
      // the end of a run (or of the CTA's share): its piece, slot r + c
      // acc[nt][i]: row 16 warp + lane/4 + 8 (i >> 1), token 8 nt + 2 (lane & 3) + (i & 1)
      if (kc == S.nkc - 1 || sg + 1 == s1) {
        if (ok) {
          float* dst = a.Pu + (size_t)(r + c) * kTok * kDRows;
          const int j0 = 16 * warp + (lane >> 2);
#pragma unroll
          for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int t = 8 * nt + 2 * (lane & 3) + (i & 1);
              if (t < a.T) dst[(size_t)t * kDRows + j0 + 8 * (i >> 1)] = acc[nt][i];
            }
          }
        }
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
          for (int i = 0; i < 4; ++i) acc[nt][i] = 0.f;
      }
      // after the share's last stage of expert e: note its count of stages
      // (counted at the end of the share, so the stream never waits on it)
      const bool e_ends = sg + 1 == s1 || up_run(S, (sg + 1) / S.nkc).ei != q.ei;
      if (e_ends) {
        if (threadIdx.x == 0) s_done[n_done] = (q.ei << 16) | n_here;
        ++n_done;
        n_here = 0;
      }
    }
    // the end of the share: one count per expert it touched (a lane each);
    // the CTA that completes an expert's stages computes its NormSiLU tile
    consumer_sync();   // every warp's pieces precede the counts, which release them
    if (warp == 0) {
      bool last = false;
      if (ok && lane < n_done) {
        const int ei = s_done[lane] >> 16, n = s_done[lane] & 0xffff;
        const unsigned old = atom_add_acq_rel(sync + si.g_cnt + ulist[ei], (unsigned)n);
        last = old + (unsigned)n == (unsigned)per_e;
      }
      unsigned lm = __ballot_sync(kFull, last);
      if (lm) {   // u comes from phase R
        int pre = 0;
        if (lane == 0) pre = spin_until(sync + si.pre_done, (unsigned)Gp, a.wait_cycles, ctl.abort_flag, a.err);
        if (!__shfl_sync(kFull, pre, 0)) lm = 0;
      }
      if (lane == 0) ctl.bcast[0] = (int)lm;
    }
    consumer_sync();
    for (unsigned lm = (unsigned)ctl.bcast[0]; lm; lm &= lm - 1) {
      const int ei = s_done[__ffs(lm) - 1] >> 16, e = ulist[ei];
      norm_silu_tile(a, S, G, e, ei, emask[e]);
      consumer_sync();
      if (threadIdx.x == 0) st_release(sync + si.a_ready + e, 1u);
    }
    ok = __all_sync(kFull, ok && !*ctl.abort_flag);
  }

  // ---- phase D ----
  // x is no longer needed: its region becomes the ring of activation tiles
  // that the loader warp fills
  __syncwarp();
  if (lane == 0) mbar_arrive(ctl.xfree);
  {
    const int nslots = tile_slots(a.D);
    int cur_rb = -1, slot = -1;
    float acc[2][4] = {};
    auto flush = [&]() {      // this CTA's partial of row block cur_rb
      if (ok) {
        const int r0 = 16 * warp + (lane >> 2);
        float* dst = a.Part + (size_t)(2 * c + slot) * kTok * kDRows;
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
          for (int qq = 0; qq < 4; ++qq) {
            const int t = 8 * nt + 2 * (lane & 3) + (qq & 1);
            if (t < a.T) dst[(size_t)t * kDRows + r0 + 8 * (qq >> 1)] = acc[nt][qq];
          }
      }
    };
    {
      const int v0 = range_lo(c, S.ND, G), v1 = range_lo(c + 1, S.ND, G);
      for (int v = v0; v < v1; ++v) {
        const DUnit d = down_unit(a, ulist, S, v);
        const int i = v - v0, ts = i % nslots;
        if (d.rb != cur_rb) {
          if (cur_rb >= 0) flush();
          cur_rb = d.rb;
          slot = cur_rb - v0 / S.J;
#pragma unroll
          for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int qq = 0; qq < 4; ++qq) acc[nt][qq] = 0.f;
        }
        ok = __all_sync(kFull, ok && mbar_wait(&ctl.tfull[ts], (i / nslots) & 1, ctl.abort_flag, a.err,
                                               a.wait_cycles));
        const uint32_t bt = smem_u32(xsm + (size_t)ts * kTileBytes);
        uint32_t brow[2];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) brow[nt] = bt + (uint32_t)(8 * nt + (lane & 7)) * (uint32_t)(4 * kSq);
        const int br = lane & 7;   // B row index for the swizzle (8 nt + br has the same low 3 bits)
        for (int c0 = 0; c0 < d.K; c0 += 128) {
          const int s = k % ctl.nstages;
          const bool w = wait_full();
          ok = ok && w;
          const int nb = min(2, (d.K - c0) / 64);
          if (ok) {
            const uint32_t st = smem_u32(ctl.stage + (size_t)s * ctl.stage_bytes);
            for (int b = 0; b < nb; ++b) {
              const uint32_t box = st + b * kBoxBytes;
#pragma unroll
              for (int ks = 0; ks < 4; ++ks) {
                uint32_t a0, a1, a2, a3;
                ldsm_x4(swz(box, 16 * warp + (lane & 7) + ((lane >> 3) & 1) * 8, 2 * ks + (lane >> 4)), a0, a1,
                        a2, a3);
                const int kc = (c0 + 64 * b) / 8 + 2 * ks + ((lane >> 3) & 1);
#pragma unroll
                for (int nt = 0; nt < 2; ++nt) {
                  if (nt < ntiles) {
                    uint32_t bh0, bh1, bl0, bl1;
                    ldsm_x2(brow[nt] + (uint32_t)row_chunk(br, kc) * 16u, bh0, bh1);
                    ldsm_x2(brow[nt] + (uint32_t)row_chunk(br, kc + kSq / 8) * 16u, bl0, bl1);
                    mma16816(acc[nt], a0, a1, a2, a3, bh0, bh1);
                    mma16816(acc[nt], a0, a1, a2, a3, bl0, bl1);
                  }
                }
              }
            }
          }
          release(s);
          ++k;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctl.tempty[ts]);   // this warp is done with the tile
      }
      if (cur_rb >= 0) flush();
    }
    // the end of the share: one count per row block it touched (counted
    // here, so the stream never waits on it); the CTA that completes a row
    // block's partials combines them
    consumer_sync();   // every warp's partials precede the counts, which release them
    if (warp == 0) {
      bool last = false;
      if (ok && lane < n_rb)
        last = atom_add_acq_rel(sync + si.rb_cnt + rb0 + lane, 1u) + 1u == (unsigned)s_nsrc[lane];
      const unsigned lm = __ballot_sync(kFull, last);
      if (lane == 0) ctl.bcast[0] = (int)lm;
    }
    consumer_sync();
    for (unsigned lm = (unsigned)ctl.bcast[0]; lm; lm &= lm - 1) {
      const int i = __ffs(lm) - 1;
      combine_rb(a, rb0 + i, s_src + i * kMaxSms, s_nsrc[i]);
    }
  }

  // ---- exit: a CTA that gave up waits for every copy it issued ----
  cp_async_wait<0>();
  consumer_sync();
  if (threadIdx.x == 0 && *ctl.abort_flag) {
    if (!x_ok) mbar_drain(ctl.xbar, 0);
    mbar_drain(ctl.pbar, 0);
    const int ki = *ctl.k_issued;
    for (int kk = k_ok; kk < ki; ++kk) mbar_drain(&ctl.full[kk % ctl.nstages], (kk / ctl.nstages) & 1);
  }
}

}  // namespace dec
}  // namespace deco
