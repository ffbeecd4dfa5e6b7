// Prefill kernels (bf16, more than 16 tokens) of the DECO MoE layer on the
// 5th-generation tensor cores (tcgen05, accumulators in tensor memory).
//
// Layer: "DECO: Sparse Mixture-of-Experts with Dense-Comparable Performance on
// End-Side Devices", §2 (Router design, Expert design): a ReLU router picks
// each token's experts, a routed expert computes W_down[e] NormSiLU(W_up[e] x)
// with NormSiLU = SiLU of the RMS-normalised difference between the expert's
// up-projection and the mean up-projection x W_bar_up^T, its output is scaled
// by s_e * r_e, and an always-on shared expert is added.
//
// With thousands of tokens every projection is a dense contraction, so all
// four run as one warp-specialised, persistent tcgen05 GEMM kernel,
// instantiated per stage:
//
//   kProj    [x] x [W_bar_up; W_s_up]^T        -> u (fp32), hs = SiLU(.) (bf16)
//   kUp      gathered x rows of expert e's pairs x W_up[e]^T, epilogue
//            NormSiLU: subtract u, RMS over the d_e columns a thread holds,
//            SiLU, times s_e * r_e            -> a (bf16, one row per pair)
//   kDown    a rows of expert e x W_down[e]^T  -> v (fp16, one row per pair)
//   kShared  hs x W_s_down^T, epilogue adds the token's routed rows v in
//            ascending expert order (fixed order: deterministic) and the
//            residual                          -> out (bf16)
//
// Tiles are 128 rows x 256 columns x 64-element K blocks (128 B: one 128-byte
// swizzle atom).  A 4-stage shared-memory ring feeds the tensor core: warp 5
// loads B (and A, except in kUp) with 2-D TMA tiles; in kUp warps 6-7 gather
// the expert's token rows of x with 16-byte cp.async into the same swizzled
// layout (zero-filling rows past the tile).  Warp 4 allocates 512 TMEM columns
// (two 256-column accumulators) and one lane issues tcgen05.mma, 128x256x16
// per instruction, committing each stage back to its producer and each
// finished accumulator to the epilogue.  Warps 0-3 read the accumulator with
// tcgen05.ld (TMEM lane = tile row = thread), so every thread owns whole rows
// and the RMS of kUp needs no cross-thread reduction; the epilogue of one tile
// overlaps the main loop of the next through the second accumulator.
//
// Waits are bounded (about 1 s), after which the kernel sets bit 2 of the
// device error word, drains the copies it issued, frees tensor memory and
// returns.
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>

#include "common.cuh"
#include "decode_kernels.cuh"   // mbarrier, bulk-copy and TMA wrappers

namespace deco {
namespace pf {

using dec::fence_barrier_init;
using dec::mbar_arrive;
using dec::mbar_expect_tx;
using dec::mbar_init;
using dec::mbar_try_wait;
using dec::mbar_wait;
using dec::smem_u32;
using dec::tma_2d;

constexpr int kBM = 128;                       // tile rows (TMEM lanes)
constexpr int kBN = 256;                       // tile columns (accumulator columns)
constexpr int kBK = 64;                        // K elements per stage (128 B of bf16)
constexpr int kStages = 4;
constexpr uint32_t kABytes = kBM * kBK * 2;    // 16 KB
constexpr uint32_t kBBytes = kBN * kBK * 2;    // 32 KB
constexpr int kThreads = 256;
constexpr int kEpiThreads = 128;               // warps 0-3
constexpr int kMmaWarp = 4;
constexpr int kTmaWarp = 5;
constexpr int kGatherWarp0 = 6;                // warps 6-7 (kUp only)
constexpr int kGatherThreads = 64;
constexpr uint32_t kTmemCols = 2 * kBN;
constexpr uint32_t kBarOffset = kStages * (kABytes + kBBytes);
constexpr size_t kSmemBytes = 1024 + kBarOffset + 256;   // 1 KB alignment slack + ring + barriers

enum : int { kProj = 0, kUp = 1, kDown = 2, kShared = 3 };
constexpr int kErrRange = 4;   // device error bit: a routed expert output outside the fp16 range

struct Args {
  int T, D, E, d_e, d_s;
  float eps;
  int residual;
  int K;            // contraction length (a multiple of 64)
  int n_tiles_n;    // column tiles per row tile
  int m_tiles;      // row tiles of kProj / kShared
  int nu;           // kProj: column tiles over W_bar_up; the rest cover W_s_up
  int bn;           // kUp: MMA N (= d_e)
  const int4* tiles;          // kUp / kDown: {e, first pair, rows, 0} per row tile
  const int* n_row_tiles;     // kUp / kDown: number of row tiles (device)
  const bf16* x;              // [T][D]
  const int* perm;            // pairs sorted by expert: token of each pair
  const float* r;             // [T][E] router weights
  const float* s;             // [E] expert scales
  const int* pair_of;         // [T][E] pair index of (t, e) or -1
  float* u;                   // [T][d_e]
  bf16* hs;                   // [T][d_s]
  bf16* a_pairs;              // [pairs][d_e]
  __half* v_pairs;            // [pairs][D] fp16: 3 more significant bits than bf16
                              // for the only intermediate that is not an MMA operand
  bf16* out;                  // [T][D]
  int* err;
};

// ---------------------------------------------------------------------------
// tcgen05 / cp.async wrappers

// Shared-memory matrix descriptor: K-major operand in 128-byte swizzled rows,
// 8-row groups 1024 B apart (the layout TMA writes with 128-byte swizzle).
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t addr) {
  uint64_t d = (uint64_t)((addr & 0x3FFFFu) >> 4);   // start address
  d |= (uint64_t)1 << 16;                            // leading offset (unused when swizzled)
  d |= (uint64_t)(1024 >> 4) << 32;                  // stride between 8-row groups
  d |= (uint64_t)1 << 46;                            // descriptor version
  d |= (uint64_t)2 << 61;                            // 128-byte swizzle
  return d;
}
// Instruction descriptor: bf16 x bf16 -> fp32, both operands K-major.
__device__ __forceinline__ uint32_t idesc_bf16(int M, int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}
__device__ __forceinline__ void umma_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
}
// arrive on `bar` once every tcgen05.mma this thread issued so far has completed
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tmem_alloc(uint32_t* slot, uint32_t cols) {   // whole warp
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(slot)),
               "r"(cols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t cols) {   // whole warp
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(cols) : "memory");
}
// 32 consecutive fp32 accumulator columns of this thread's TMEM lane
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t q[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(q[0]), "=r"(q[1]), "=r"(q[2]), "=r"(q[3]), "=r"(q[4]), "=r"(q[5]), "=r"(q[6]), "=r"(q[7]),
        "=r"(q[8]), "=r"(q[9]), "=r"(q[10]), "=r"(q[11]), "=r"(q[12]), "=r"(q[13]), "=r"(q[14]),
        "=r"(q[15]), "=r"(q[16]), "=r"(q[17]), "=r"(q[18]), "=r"(q[19]), "=r"(q[20]), "=r"(q[21]),
        "=r"(q[22]), "=r"(q[23]), "=r"(q[24]), "=r"(q[25]), "=r"(q[26]), "=r"(q[27]), "=r"(q[28]),
        "=r"(q[29]), "=r"(q[30]), "=r"(q[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(q[j]);
}
// 16-byte global -> shared copy; src_bytes = 0 writes zeros
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes)
               : "memory");
}
// arrive on `bar` when this thread's cp.async copies so far have landed
__device__ __forceinline__ void cp_async_arrive(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}
// 32 fp32 values -> 32 bf16 (64 B) at a 16-byte aligned address
__device__ __forceinline__ void store_bf16x32(bf16* dst, const float (&v)[32]) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint4 w;
    w.x = pack_bf16x2(v[8 * q + 0], v[8 * q + 1]);
    w.y = pack_bf16x2(v[8 * q + 2], v[8 * q + 3]);
    w.z = pack_bf16x2(v[8 * q + 4], v[8 * q + 5]);
    w.w = pack_bf16x2(v[8 * q + 6], v[8 * q + 7]);
    reinterpret_cast<uint4*>(dst)[q] = w;
  }
}
// 32 fp32 values -> 32 fp16 (64 B) at a 16-byte aligned address; returns
// false if a value is outside the fp16 range (or not finite)
__device__ __forceinline__ bool store_f16x32(__half* dst, const float (&v)[32]) {
  bool fin = true;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint32_t w[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float lo = v[8 * q + 2 * j], hi = v[8 * q + 2 * j + 1];
      fin = fin && fabsf(lo) <= 65504.f && fabsf(hi) <= 65504.f;
      const __half2 h = __floats2half2_rn(lo, hi);
      w[j] = *reinterpret_cast<const uint32_t*>(&h);
    }
    reinterpret_cast<uint4*>(dst)[q] = make_uint4(w[0], w[1], w[2], w[3]);
  }
  return fin;
}
// v += 32 fp16 at a 16-byte aligned address
__device__ __forceinline__ void add_f16x32(float (&v)[32], const __half* src) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint4 w = __ldg(reinterpret_cast<const uint4*>(src) + q);
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&ws[j]));
      v[8 * q + 2 * j] += f.x;
      v[8 * q + 2 * j + 1] += f.y;
    }
  }
}
// v += 32 bf16 at a 16-byte aligned address
__device__ __forceinline__ void add_bf16x32(float (&v)[32], const bf16* src) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    float f[8];
    unpack16(__ldg(reinterpret_cast<const uint4*>(src) + q), f);
#pragma unroll
    for (int j = 0; j < 8; ++j) v[8 * q + j] += f[j];
  }
}

// ---------------------------------------------------------------------------
// tile schedule: tile idx -> operand rows and output columns

struct Tile {
  int arow;   // first A row (token, or pair in kUp / kDown)
  int rows;   // valid rows (<= 128)
  int brow;   // first B row in its tensor map
  int bmap;   // kProj: 0 = W_bar_up, 1 = W_s_up
  int n0;     // first output column
  int e;      // expert (kUp / kDown)
};

template <int MODE>
__device__ __forceinline__ int tile_total(const Args& a) {
  if (MODE == kProj || MODE == kShared) return a.m_tiles * a.n_tiles_n;
  const int n = *a.n_row_tiles;
  return MODE == kUp ? n : n * a.n_tiles_n;
}

template <int MODE>
__device__ __forceinline__ Tile tile_at(const Args& a, int idx) {
  Tile t{};
  if (MODE == kUp) {
    const int4 q = a.tiles[idx];
    t.e = q.x;
    t.arow = q.y;
    t.rows = q.z;
    t.brow = q.x * a.d_e;
    return t;
  }
  const int mt = idx / a.n_tiles_n, nt = idx - mt * a.n_tiles_n;
  if (MODE == kDown) {
    const int4 q = a.tiles[mt];
    t.e = q.x;
    t.arow = q.y;
    t.rows = q.z;
    t.n0 = nt * kBN;
    t.brow = q.x * a.D + t.n0;
    return t;
  }
  t.arow = mt * kBM;
  t.rows = min(kBM, a.T - t.arow);
  if (MODE == kProj && nt >= a.nu) {
    t.bmap = 1;
    t.brow = (nt - a.nu) * kBN;
  } else {
    t.brow = nt * kBN;
  }
  t.n0 = t.brow;
  return t;
}

// ---------------------------------------------------------------------------
// epilogues: thread i (0..127) owns tile row i, TMEM lane i; `trow` is the
// TMEM address of its lane at the accumulator's first column.  tcgen05.ld is
// warp-collective, so every thread loads; only stores are predicated.

template <int MODE>
__device__ __forceinline__ void epilogue(const Args& a, const Tile& t, uint32_t trow, int i) {
  if (MODE == kProj) {
    const int tok = t.arow + i;
    const bool ok = i < t.rows;
    const int lim = t.bmap == 0 ? a.d_e : a.d_s;
    for (int c0 = 0; c0 < kBN; c0 += 32) {
      if (t.n0 + c0 >= lim) break;                       // uniform across the warp
      float v[32];
      tmem_ld32(trow + c0, v);
      if (!ok) continue;
      const int col = t.n0 + c0;                         // lim is a multiple of 64: all 32 valid
      if (t.bmap == 0) {
        float4* dst = reinterpret_cast<float4*>(a.u + (size_t)tok * a.d_e + col);
#pragma unroll
        for (int q = 0; q < 8; ++q) dst[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = silu_f(v[j]);
        store_bf16x32(a.hs + (size_t)tok * a.d_s + col, v);
      }
    }
  } else if (MODE == kUp) {
    const bool ok = i < t.rows;
    const int pair = t.arow + i;
    const int tok = ok ? a.perm[pair] : 0;
    const float coef = ok ? a.s[t.e] * a.r[(size_t)tok * a.E + t.e] : 0.f;
    const float* ur = a.u + (size_t)tok * a.d_e;
    float ss = 0.f;
    for (int c0 = 0; c0 < a.d_e; c0 += 32) {
      float v[32];
      tmem_ld32(trow + c0, v);
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const float4 uq = __ldg(reinterpret_cast<const float4*>(ur + c0) + q);
        const float c_0 = v[4 * q] - uq.x, c_1 = v[4 * q + 1] - uq.y;
        const float c_2 = v[4 * q + 2] - uq.z, c_3 = v[4 * q + 3] - uq.w;
        ss = fmaf(c_0, c_0, ss);
        ss = fmaf(c_1, c_1, ss);
        ss = fmaf(c_2, c_2, ss);
        ss = fmaf(c_3, c_3, ss);
      }
    }
    const float inv = rsqrtf(ss / (float)a.d_e + a.eps);
    bf16* dst = a.a_pairs + (size_t)pair * a.d_e;
    for (int c0 = 0; c0 < a.d_e; c0 += 32) {
      float v[32];
      tmem_ld32(trow + c0, v);
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const float4 uq = __ldg(reinterpret_cast<const float4*>(ur + c0) + q);
        v[4 * q] = silu_f((v[4 * q] - uq.x) * inv) * coef;
        v[4 * q + 1] = silu_f((v[4 * q + 1] - uq.y) * inv) * coef;
        v[4 * q + 2] = silu_f((v[4 * q + 2] - uq.z) * inv) * coef;
        v[4 * q + 3] = silu_f((v[4 * q + 3] - uq.w) * inv) * coef;
      }
      if (ok) store_bf16x32(dst + c0, v);
    }
  } else if (MODE == kDown) {
    const bool ok = i < t.rows;
    __half* dst = a.v_pairs + (size_t)(t.arow + i) * a.D;
    bool fin = true;
    for (int c0 = 0; c0 < kBN; c0 += 32) {
      const int col = t.n0 + c0;
      if (col >= a.D) break;                             // D is a multiple of 64
      float v[32];
      tmem_ld32(trow + c0, v);
      if (ok) fin = store_f16x32(dst + col, v) && fin;
    }
    if (!fin) atomicOr(a.err, kErrRange);
  } else {   // kShared: shared expert + routed rows in ascending expert order + residual
    const int tok = t.arow + i;
    const bool ok = i < t.rows;
    const int* po = a.pair_of + (size_t)(ok ? tok : 0) * a.E;
    for (int c0 = 0; c0 < kBN; c0 += 32) {
      const int col = t.n0 + c0;
      if (col >= a.D) break;
      float v[32];
      tmem_ld32(trow + c0, v);
      if (!ok) continue;
      for (int e = 0; e < a.E; ++e) {
        const int q = __ldg(po + e);
        if (q >= 0) add_f16x32(v, a.v_pairs + (size_t)q * a.D + col);
      }
      if (a.residual) add_bf16x32(v, a.x + (size_t)tok * a.D + col);
      store_bf16x32(a.out + (size_t)tok * a.D + col, v);
    }
  }
}

// ---------------------------------------------------------------------------

template <int MODE>
__global__ void __launch_bounds__(kThreads, 1)
    kp_gemm(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
            const __grid_constant__ CUtensorMap tmB2, const Args a) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;          // 128-byte swizzle needs 1 KB alignment
  uint8_t* sm = smem_raw + (base - raw);
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + kBarOffset);
  uint64_t* empty = full + kStages;
  uint64_t* accf = empty + kStages;
  uint64_t* acce = accf + 2;
  uint64_t* drain = acce + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1 + (MODE == kUp ? kGatherThreads : 0));
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&accf[b], 1);
      mbar_init(&acce[b], kEpiThreads);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kMmaWarp) tmem_alloc(tmem_slot, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const int total = tile_total<MODE>(a);
  const int nk = a.K / kBK;

  if (warp == kTmaWarp) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t armed = 0, armed_parity = 0;               // per-stage bits, for the drain
      const uint32_t bytes = kBBytes + (MODE == kUp ? 0u : kABytes);
      for (int idx = blockIdx.x; idx < total && !*abort_flag; idx += gridDim.x) {
        const Tile t = tile_at<MODE>(a, idx);
        const CUtensorMap* mb = (MODE == kProj && t.bmap) ? &tmB2 : &tmB;
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag, a.err)) break;
          mbar_expect_tx(&full[stage], bytes);
          if (MODE != kUp) tma_2d(sm + stage * kABytes, &tmA, kb * kBK, t.arow, &full[stage]);
          tma_2d(sm + kStages * kABytes + stage * kBBytes, mb, kb * kBK, t.brow, &full[stage]);
          armed |= 1u << stage;
          armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      if (*abort_flag) {   // let every issued copy land before the CTA exits
        for (int s = 0; s < kStages; ++s) {
          if (!(armed >> s & 1)) continue;
          const long long t0 = clock64();
          while (!mbar_try_wait(&full[s], armed_parity >> s & 1) && clock64() - t0 < dec::kWaitCycles) {
          }
        }
      }
    }
  } else if (MODE == kUp && warp >= kGatherWarp0) {
    const int j = threadIdx.x - kGatherWarp0 * 32;       // 0..63
    const int c = j & 7, rsub = j >> 3;                  // 16-byte chunk, row within 8-row group
    int stage = 0;
    uint32_t phase = 0;
    bool stop = false;
    for (int idx = blockIdx.x; idx < total && !stop; idx += gridDim.x) {
      const Tile t = tile_at<MODE>(a, idx);
      int tok[16];
#pragma unroll
      for (int q = 0; q < 16; ++q) {
        const int row = q * 8 + rsub;
        tok[q] = row < t.rows ? a.perm[t.arow + row] : -1;
      }
      for (int kb = 0; kb < nk; ++kb) {
        if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag, a.err)) {
          stop = true;
          break;
        }
        const uint32_t sA = base + stage * kABytes;
#pragma unroll
        for (int q = 0; q < 16; ++q) {
          const int row = q * 8 + rsub;
          const uint32_t dst = sA + row * 128 + ((c ^ rsub) << 4);
          const bf16* src = tok[q] >= 0 ? a.x + (size_t)tok[q] * a.D + kb * kBK + c * 8 : a.x;
          cp_async16(dst, src, tok[q] >= 0 ? 16u : 0u);
        }
        cp_async_arrive(&full[stage]);
        if (++stage == kStages) {
          stage = 0;
          phase ^= 1;
        }
      }
    }
    cp_async_wait_all();
  } else if (warp == kMmaWarp) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16(kBM, MODE == kUp ? a.bn : kBN);
      int stage = 0;
      uint32_t phase = 0;
      int lt = 0;
      bool stop = false;
      for (int idx = blockIdx.x; idx < total && !stop; idx += gridDim.x, ++lt) {
        const int b = lt & 1;
        if (!mbar_wait(&acce[b], ((lt >> 1) & 1) ^ 1, abort_flag, a.err)) break;
        tc_fence_after();
        const uint32_t dt = tmem + b * kBN;
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(&full[stage], phase, abort_flag, a.err)) {
            stop = true;
            break;
          }
          if (MODE == kUp) fence_proxy_async_smem();   // cp.async data -> tensor core (async proxy)
          tc_fence_after();
          const uint32_t sA = base + stage * kABytes;
          const uint32_t sB = base + kStages * kABytes + stage * kBBytes;
#pragma unroll
          for (int k = 0; k < kBK / 16; ++k)
            umma_bf16(dt, sdesc_sw128(sA + k * 32), sdesc_sw128(sB + k * 32), idesc, (kb | k) != 0);
          umma_commit(&empty[stage]);
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!stop) umma_commit(&accf[b]);
      }
      // all issued MMAs complete before tensor memory is freed
      umma_commit(drain);
      const long long t0 = clock64();
      while (!mbar_try_wait(drain, 0) && clock64() - t0 < dec::kWaitCycles) {
      }
    }
  } else if (warp < 4) {
    int lt = 0;
    for (int idx = blockIdx.x; idx < total; idx += gridDim.x, ++lt) {
      const int b = lt & 1;
      if (!mbar_wait(&accf[b], (lt >> 1) & 1, abort_flag, a.err)) break;
      tc_fence_after();
      const Tile t = tile_at<MODE>(a, idx);
      epilogue<MODE>(a, t, tmem + ((uint32_t)(warp * 32) << 16) + b * kBN, threadIdx.x);
      tc_fence_before();
      mbar_arrive(&acce[b]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace pf
}  // namespace deco
