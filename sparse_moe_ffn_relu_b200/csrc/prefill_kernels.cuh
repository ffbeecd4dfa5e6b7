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
//            SiLU                             -> a (bf16, one row per pair),
//                                                s_e * r_e (fp32, per pair)
//   kDown    a rows of expert e x W_down[e]^T  -> v (fp16, one row per pair)
//   kShared  hs x W_s_down^T                   -> S (fp32)
//   kVal     (gated experts) gathered x rows x W_val[e]^T -> value rows (bf16,
//            one per pair), which kUp's epilogue multiplies in
//
// and two CUDA-core kernels around them: k_router (exact ReLU routing) and
// k_combine, out = S + the token's routed rows s_e r_e v in ascending expert
// order (a fixed order: deterministic) + the residual, one CTA per token with
// coalesced row reads.
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
// overlaps the main loop of the next through the second accumulator.  Results
// leave through shared memory: each epilogue warp fills 32-row x 128-byte
// boxes (128-byte swizzle) and stores each with one TMA tensor store, two
// boxes in flight per warp.  kUp stages the u rows of its tokens through the
// same boxes with coalesced loads and keeps c = g - u in TMEM between its two
// passes (sum of squares, then SiLU).
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
constexpr uint32_t kStageOut = 4096;                      // one output box: 32 rows x 128 B
constexpr uint32_t kEpiOffset = kStages * (kABytes + kBBytes);
constexpr uint32_t kBarOffset = kEpiOffset + 4 * 2 * kStageOut;   // two boxes per epilogue warp
constexpr size_t kSmemBytes = 1024 + kBarOffset + 256;   // 1 KB alignment slack + ring + boxes + barriers

enum : int { kProj = 0, kUp = 1, kDown = 2, kShared = 3, kVal = 4 };
// the modes whose A rows are gathered token rows of x (one expert's pairs)
template <int MODE>
__host__ __device__ constexpr bool gathers() { return MODE == kUp || MODE == kVal; }
constexpr int kErrRange = 4;   // device error bit: a routed expert output outside the fp16 range

struct Args {
  int T, D, E, d_e, d_s;
  float eps;
  int residual;
  long long wait_cycles;      // limit of the waits for data (dec::kWaitCycles unless a test lowers it)
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
  bf16* a_pairs;              // [pairs][d_e] NormSiLU outputs, SiLU(h): |a| <= sqrt(d_e)
                              // (times the value branch for gated experts)
  const bf16* val_pairs;      // [pairs][d_e] gated experts' value rows (kVal writes, kUp reads), or null
  float* coef_pairs;          // [pairs] s_e r_e of each pair, applied in the combine
  __half* v_pairs;            // [pairs][D] W_down[e] a in fp16 (3 more significant bits than
                              // bf16); unscaled by s_e r_e, so |v| <= sqrt(d_e) max_j ||W_down[e][j]||_1
                              // is a property of the weights, not of the input
  float* s_out;               // [T][D] shared-expert output (MoE layer; null: kShared writes out)
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
// 32 consecutive fp32 TMEM columns of this thread's lane <- v
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]), "f"(v[8]),
      "f"(v[9]), "f"(v[10]), "f"(v[11]), "f"(v[12]), "f"(v[13]), "f"(v[14]), "f"(v[15]), "f"(v[16]),
      "f"(v[17]), "f"(v[18]), "f"(v[19]), "f"(v[20]), "f"(v[21]), "f"(v[22]), "f"(v[23]), "f"(v[24]),
      "f"(v[25]), "f"(v[26]), "f"(v[27]), "f"(v[28]), "f"(v[29]), "f"(v[30]), "f"(v[31])
      : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
// shared -> global 2-D TMA tensor store of one box at (col, row)
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, uint32_t src, int col, int row) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(src), "r"(col), "r"(row)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// wait until at most N committed store groups may still read shared memory
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
// SiLU with the fast exponential and division intrinsics (bf16 results)
__device__ __forceinline__ float silu_fast(float h) { return __fdividef(h, 1.0f + __expf(-h)); }

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
  return gathers<MODE>() ? n : n * a.n_tiles_n;
}

template <int MODE>
__device__ __forceinline__ Tile tile_at(const Args& a, int idx) {
  Tile t{};
  if (gathers<MODE>()) {
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
// epilogue output boxes: 32 rows x 128 B, 16-byte chunk q of row r at
// r * 128 + (q ^ (r & 7)) * 16 (the 128-byte swizzle of the output tensor maps)

struct Out {
  uint8_t* stg;      // this warp's two boxes
  uint32_t stg_s;    // the same, shared-window address
  int lane;
  int n;             // boxes stored so far by this warp
};

__device__ __forceinline__ uint32_t box_off(int r, int q) {
  return (uint32_t)r * 128u + ((uint32_t)(q ^ (r & 7)) << 4);
}
// the next box to fill, once the store that last read it is done
__device__ __forceinline__ uint8_t* box_begin(Out& o) {
  if (o.lane == 0 && o.n >= 2) bulk_wait_read<1>();
  __syncwarp();
  return o.stg + (o.n & 1) * kStageOut;
}
// hand the filled box to the async proxy and store it at (col, row)
__device__ __forceinline__ void box_store(Out& o, const CUtensorMap* map, int col, int row) {
  fence_proxy_async_smem();
  __syncwarp();
  if (o.lane == 0) {
    tma_store_2d(map, o.stg_s + (o.n & 1) * kStageOut, col, row);
    bulk_commit();
  }
  ++o.n;
}
__device__ __forceinline__ void box_put_f32(uint8_t* box, int r, const float (&v)[32]) {
#pragma unroll
  for (int q = 0; q < 8; ++q)
    *reinterpret_cast<float4*>(box + box_off(r, q)) = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
}
// 32 16-bit values: half h of the row
__device__ __forceinline__ void box_put_16(uint8_t* box, int r, int h, const uint4 (&w)[4]) {
#pragma unroll
  for (int q = 0; q < 4; ++q) *reinterpret_cast<uint4*>(box + box_off(r, 4 * h + q)) = w[q];
}
__device__ __forceinline__ void pack_bf16x32(const float (&v)[32], uint4 (&w)[4]) {
#pragma unroll
  for (int q = 0; q < 4; ++q)
    w[q] = make_uint4(pack_bf16x2(v[8 * q], v[8 * q + 1]), pack_bf16x2(v[8 * q + 2], v[8 * q + 3]),
                      pack_bf16x2(v[8 * q + 4], v[8 * q + 5]), pack_bf16x2(v[8 * q + 6], v[8 * q + 7]));
}
// fp16; returns false if a value is outside the fp16 range (or not finite)
__device__ __forceinline__ bool pack_f16x32(const float (&v)[32], uint4 (&w)[4]) {
  bool fin = true;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint32_t h[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float lo = v[8 * q + 2 * j], hi = v[8 * q + 2 * j + 1];
      fin = fin && fabsf(lo) <= 65504.f && fabsf(hi) <= 65504.f;
      const __half2 x = __floats2half2_rn(lo, hi);
      h[j] = *reinterpret_cast<const uint32_t*>(&x);
    }
    w[q] = make_uint4(h[0], h[1], h[2], h[3]);
  }
  return fin;
}

// ---------------------------------------------------------------------------
// epilogues: epilogue warp w (0..3) owns tile rows 32w..32w+31, lane r row
// 32w + r, which is TMEM lane 32w + r; `trow` is that lane's TMEM address at
// the accumulator's first column.  tcgen05.ld/st are warp-collective, so every
// lane executes them; rows past the tile are dropped by the tensor map's
// bounds (token rows) or written by direct stores of the valid rows only
// (pair rows, whose next rows belong to another expert).

template <int MODE>
__device__ __forceinline__ void epilogue(const Args& a, const Tile& t, uint32_t trow, int warp, Out& o,
                                         const CUtensorMap* tmO, const CUtensorMap* tmO2) {
  const int r = o.lane, i = warp * 32 + r;
  const int row0 = t.arow + warp * 32;
  const bool ok = i < t.rows;
  const bool full_warp = warp * 32 + 32 <= t.rows;
  if ((MODE == kProj || (MODE == kShared && a.s_out)) && row0 >= a.T) return;   // no row of this warp exists
  if (MODE == kProj) {
    if (t.bmap == 0) {   // u, fp32: one box per 32 columns
      for (int c0 = 0; c0 < kBN; c0 += 32) {
        if (t.n0 + c0 >= a.d_e) break;                   // uniform across the warp
        float v[32];
        tmem_ld32(trow + c0, v);
        uint8_t* box = box_begin(o);
        box_put_f32(box, r, v);
        box_store(o, tmO, t.n0 + c0, row0);
      }
    } else {             // SiLU(shared up-projection), bf16: one box per 64 columns
      for (int c0 = 0; c0 < kBN; c0 += 64) {
        if (t.brow + c0 >= a.d_s) break;                 // d_s is a multiple of 64
        uint8_t* box = box_begin(o);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          float v[32];
          tmem_ld32(trow + c0 + 32 * h, v);
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] = silu_fast(v[j]);
          uint4 w[4];
          pack_bf16x32(v, w);
          box_put_16(box, r, h, w);
        }
        box_store(o, tmO2, t.brow + c0, row0);
      }
    }
  } else if (MODE == kUp) {
    const int pair = t.arow + i;
    const int tok = ok ? a.perm[pair] : 0;
    const float coef = ok ? a.s[t.e] * a.r[(size_t)tok * a.E + t.e] : 0.f;
    // pass 1: c = g - u back into TMEM, sum of c^2.  The warp stages its 32
    // rows' u through the two boxes, 32 columns (128 B per row) at a time: lane
    // l loads 16 B of rows 4j + l/8 (j < 8), column chunk l % 8.
    if (o.lane == 0) bulk_wait_read<0>();                // earlier stores done reading the boxes
    __syncwarp();
    int tk[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) tk[j] = __shfl_sync(kFull, tok, 4 * j + (r >> 3));
    const int cq = r & 7;
    float4 q[8];
    auto u_load = [&](int c0) {
#pragma unroll
      for (int j = 0; j < 8; ++j)
        q[j] = __ldg(reinterpret_cast<const float4*>(a.u + (size_t)tk[j] * a.d_e + c0) + cq);
    };
    auto u_put = [&](uint8_t* buf) {
#pragma unroll
      for (int j = 0; j < 8; ++j) *reinterpret_cast<float4*>(buf + box_off(4 * j + (r >> 3), cq)) = q[j];
    };
    const int nc = a.d_e / 32;
    u_load(0);
    u_put(o.stg);
    __syncwarp();
    float ss = 0.f;
    for (int c = 0; c < nc; ++c) {
      if (c + 1 < nc) u_load((c + 1) * 32);
      float v[32];
      tmem_ld32(trow + c * 32, v);
      const uint8_t* ub = o.stg + (c & 1) * kStageOut;
#pragma unroll
      for (int qq = 0; qq < 8; ++qq) {
        const float4 uq = *reinterpret_cast<const float4*>(ub + box_off(r, qq));
        v[4 * qq] -= uq.x;
        v[4 * qq + 1] -= uq.y;
        v[4 * qq + 2] -= uq.z;
        v[4 * qq + 3] -= uq.w;
      }
#pragma unroll
      for (int j = 0; j < 32; ++j) ss = fmaf(v[j], v[j], ss);
      tmem_st32(trow + c * 32, v);
      if (c + 1 < nc) u_put(o.stg + ((c + 1) & 1) * kStageOut);
      __syncwarp();
    }
    tmem_wait_st();
    const float inv = rsqrtf(ss / (float)a.d_e + a.eps);
    if (ok) a.coef_pairs[pair] = coef;
    // pass 2: a = SiLU(c / rms), bf16, 64 columns per box (s_e r_e is applied in the combine)
    bf16* dst = a.a_pairs + (size_t)pair * a.d_e;
    for (int c0 = 0; c0 < a.d_e; c0 += 64) {
      uint8_t* box = full_warp ? box_begin(o) : nullptr;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        float v[32];
        tmem_ld32(trow + c0 + 32 * h, v);
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = silu_fast(v[j] * inv);
        if (a.val_pairs && ok) {   // gated experts: times the value row (bf16, 64 B)
          float vv[32];
#pragma unroll
          for (int q = 0; q < 4; ++q)
            unpack16(__ldg(reinterpret_cast<const uint4*>(a.val_pairs + (size_t)pair * a.d_e + c0 + 32 * h) + q),
                     *reinterpret_cast<float(*)[8]>(vv + 8 * q));
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] *= vv[j];
        }
        uint4 w[4];
        pack_bf16x32(v, w);
        if (full_warp) {
          box_put_16(box, r, h, w);
        } else if (ok) {
#pragma unroll
          for (int qq = 0; qq < 4; ++qq) reinterpret_cast<uint4*>(dst + c0 + 32 * h)[qq] = w[qq];
        }
      }
      if (full_warp) box_store(o, tmO, c0, row0);
    }
  } else if (MODE == kVal) {   // value rows, bf16, 64 columns per box
    const int pair = t.arow + i;
    bf16* dst = const_cast<bf16*>(a.val_pairs) + (size_t)pair * a.d_e;
    for (int c0 = 0; c0 < a.d_e; c0 += 64) {
      uint8_t* box = full_warp ? box_begin(o) : nullptr;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        float v[32];
        tmem_ld32(trow + c0 + 32 * h, v);
        uint4 w[4];
        pack_bf16x32(v, w);
        if (full_warp) {
          box_put_16(box, r, h, w);
        } else if (ok) {
#pragma unroll
          for (int qq = 0; qq < 4; ++qq) reinterpret_cast<uint4*>(dst + c0 + 32 * h)[qq] = w[qq];
        }
      }
      if (full_warp) box_store(o, tmO, c0, row0);
    }
  } else if (MODE == kDown) {
    __half* dst = a.v_pairs + (size_t)(t.arow + i) * a.D;
    bool fin = true;
    for (int c0 = 0; c0 < kBN; c0 += 64) {
      const int col = t.n0 + c0;
      if (col >= a.D) break;                             // D is a multiple of 64
      uint8_t* box = full_warp ? box_begin(o) : nullptr;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        float v[32];
        tmem_ld32(trow + c0 + 32 * h, v);
        uint4 w[4];
        const bool f = pack_f16x32(v, w);
        if (full_warp) {
          box_put_16(box, r, h, w);
          fin = fin && f;
        } else if (ok) {
#pragma unroll
          for (int qq = 0; qq < 4; ++qq) reinterpret_cast<uint4*>(dst + col + 32 * h)[qq] = w[qq];
          fin = fin && f;
        }
      }
      if (full_warp) box_store(o, tmO, col, row0);
    }
    if (!fin) atomicOr(a.err, kErrRange);
  } else {   // kShared: the shared expert's output rows
    const int tok = t.arow + i;
    for (int c0 = 0; c0 < kBN; c0 += 32) {
      const int col = t.n0 + c0;
      if (col >= a.D) break;
      float v[32];
      tmem_ld32(trow + c0, v);
      if (a.s_out) {   // MoE layer: fp32 boxes; the combine kernel adds the routed rows
        uint8_t* box = box_begin(o);
        box_put_f32(box, r, v);
        box_store(o, tmO, col, row0);
      } else if (ok) { // dense FFN: the output itself
        if (a.residual) add_bf16x32(v, a.x + (size_t)tok * a.D + col);
        store_bf16x32(a.out + (size_t)tok * a.D + col, v);
      }
    }
  }
}

// ---------------------------------------------------------------------------

template <int MODE>
__global__ void __launch_bounds__(kThreads, 1)
    kp_gemm(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
            const __grid_constant__ CUtensorMap tmB2, const __grid_constant__ CUtensorMap tmO,
            const __grid_constant__ CUtensorMap tmO2, const Args a) {
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
      mbar_init(&full[s], 1 + (gathers<MODE>() ? kGatherThreads : 0));
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
      const uint32_t bytes = kBBytes + (gathers<MODE>() ? 0u : kABytes);
      for (int idx = blockIdx.x; idx < total && !*abort_flag; idx += gridDim.x) {
        const Tile t = tile_at<MODE>(a, idx);
        const CUtensorMap* mb = (MODE == kProj && t.bmap) ? &tmB2 : &tmB;
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag, a.err, a.wait_cycles)) break;
          mbar_expect_tx(&full[stage], bytes);
          if (!gathers<MODE>()) tma_2d(sm + stage * kABytes, &tmA, kb * kBK, t.arow, &full[stage]);
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
  } else if (gathers<MODE>() && warp >= kGatherWarp0) {
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
        if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag, a.err, a.wait_cycles)) {
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
      const uint32_t idesc = idesc_bf16(kBM, gathers<MODE>() ? a.bn : kBN);
      int stage = 0;
      uint32_t phase = 0;
      int lt = 0;
      bool stop = false;
      for (int idx = blockIdx.x; idx < total && !stop; idx += gridDim.x, ++lt) {
        const int b = lt & 1;
        if (!mbar_wait(&acce[b], ((lt >> 1) & 1) ^ 1, abort_flag, a.err, a.wait_cycles)) break;
        tc_fence_after();
        const uint32_t dt = tmem + b * kBN;
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(&full[stage], phase, abort_flag, a.err, a.wait_cycles)) {
            stop = true;
            break;
          }
          if (gathers<MODE>()) fence_proxy_async_smem();   // cp.async data -> tensor core (async proxy)
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
    Out o;
    o.stg = sm + kEpiOffset + warp * 2 * kStageOut;
    o.stg_s = base + kEpiOffset + warp * 2 * kStageOut;
    o.lane = lane;
    o.n = 0;
    int lt = 0;
    for (int idx = blockIdx.x; idx < total; idx += gridDim.x, ++lt) {
      const int b = lt & 1;
      // warp-uniform: tcgen05.ld below is warp-collective
      if (!__all_sync(kFull, mbar_wait(&accf[b], (lt >> 1) & 1, abort_flag, a.err, a.wait_cycles))) break;
      tc_fence_after();
      const Tile t = tile_at<MODE>(a, idx);
      epilogue<MODE>(a, t, tmem + ((uint32_t)(warp * 32) << 16) + b * kBN, warp, o, &tmO, &tmO2);
      tc_fence_before();
      mbar_arrive(&acce[b]);
    }
    if (lane == 0) bulk_wait_all();   // every output store has landed
    __syncwarp();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// Router: z[t][e] = b_r[e] + x_t . W_r[e] on CUDA cores in fp32, with a
// rigorous bound B on |z - exact| so that the sign, which decides whether e is
// active for t (ReLU routing, "DECO ...", §2 Router design), is exact: pairs
// with |z| <= B go to a list that k_router_exact settles with an exact integer
// accumulation.
//
// A CTA computes 32 tokens x 64 experts with 8 warps; warp g takes the
// 16-element K chunks g, g+8, g+16, ... through its own shared-memory slice
// (no block barrier in the main loop), each lane an 8 x 8 block of (token,
// expert) sums.  Each chunk is summed from zero and added to the warp's running
// total; the 8 warp totals are added in warp order at the end, so every value
// goes through at most kRK + D/(8 kRK) + 8 roundings before the bias.  The
// product-magnitude sum S in the bound is replaced by its Cauchy-Schwarz upper
// bound ||x_t|| ||W_r[e]||, the norms accumulated from the staged tiles.

constexpr int kRT = 32;          // tokens per CTA
constexpr int kRE = 64;          // experts per CTA
constexpr int kRK = 16;          // K chunk
constexpr int kRWarps = 8;
constexpr int kRThreads = kRWarps * 32;
constexpr int kRTL = kRT / 4;    // tokens per lane (4 token groups x 8 expert groups of lanes)
static_assert(kRTL == 8, "the lane tile below reads 8 tokens as two float4");
constexpr size_t kRStage = (size_t)kRWarps * kRK * (kRT + kRE) * 4;   // per-warp staging slices
constexpr size_t kRTotals = (size_t)kRWarps * kRT * kRE * 4;          // warp totals (alias the staging)
constexpr size_t kRouterSmem = (kRStage > kRTotals ? kRStage : kRTotals) + (size_t)kRWarps * (kRT + kRE) * 4;

struct RouterArgs {
  const bf16* x;
  const bf16* W_r;
  const float* b_r;
  int T, D, E;
  float* r;          // [T][E]
  uint8_t* act;      // [T][E]
  int2* fb;          // ambiguous pairs: {t * E + e, bits of z}
  int* n_fb;
  int* err;
};

__device__ __forceinline__ unsigned long long f2pack(float lo, float hi) {
  unsigned long long r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ float2 f2unpack(unsigned long long v) {
  float2 r;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(r.x), "=f"(r.y) : "l"(v));
  return r;
}
// d = a * b + d on both fp32 halves (each an IEEE fma, round to nearest)
__device__ __forceinline__ void ffma2(unsigned long long& d, unsigned long long a, unsigned long long b) {
  asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(d) : "l"(a), "l"(b));
}

__global__ void __launch_bounds__(kRThreads, 1) k_router(const RouterArgs a) {
  extern __shared__ __align__(16) float rsm[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t0 = blockIdx.x * kRT, e0 = blockIdx.y * kRE;
  // this warp's staging slice: xs[kRK][kRT], ws[kRK][kRE]
  float* xs = rsm + (size_t)warp * kRK * (kRT + kRE);
  float* ws = xs + kRK * kRT;
  constexpr size_t kNormOff = (kRStage > kRTotals ? kRStage : kRTotals) / 4;   // floats
  float* nx_w = rsm + kNormOff + warp * (kRT + kRE);   // [kRT] then [kRE]
  float* nw_w = nx_w + kRT;
  // loading: lane = token row lane and expert rows lane, lane + 32; 16 k each
  const bool xok = lane < kRT && t0 + lane < a.T;
  const bool wok0 = e0 + lane < a.E, wok1 = e0 + lane + 32 < a.E;
  const bf16* xrow = a.x + (size_t)(xok ? t0 + lane : 0) * a.D;
  const bf16* wrow0 = a.W_r + (size_t)(wok0 ? e0 + lane : 0) * a.D;
  const bf16* wrow1 = a.W_r + (size_t)(wok1 ? e0 + lane + 32 : 0) * a.D;
  float sx = 0.f, sw0 = 0.f, sw1 = 0.f;
  // computing: tokens ty*kRTL + i, experts tx*4 + {0..3} and 32 + tx*4 + {0..3}
  const int ty = lane >> 3, tx = lane & 7;
  unsigned long long tot[kRTL][4];
#pragma unroll
  for (int i = 0; i < kRTL; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) tot[i][j] = 0ull;
  const int nchunks = a.D / kRK;
  const uint4 zero4 = make_uint4(0, 0, 0, 0);
  uint4 q[6];   // next chunk: x (2), W rows (2 + 2)
  auto fetch = [&](int c) {
    const bool live = c < nchunks;
    const int k0 = c * kRK;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      q[h] = (live && xok) ? *reinterpret_cast<const uint4*>(xrow + k0 + 8 * h) : zero4;
      q[2 + h] = (live && wok0) ? *reinterpret_cast<const uint4*>(wrow0 + k0 + 8 * h) : zero4;
      q[4 + h] = (live && wok1) ? *reinterpret_cast<const uint4*>(wrow1 + k0 + 8 * h) : zero4;
    }
  };
  fetch(warp);
  for (int c = warp; c < nchunks; c += kRWarps) {
    float fx[16], fw0[16], fw1[16];
    unpack16(q[0], *reinterpret_cast<float(*)[8]>(fx));
    unpack16(q[1], *reinterpret_cast<float(*)[8]>(fx + 8));
    unpack16(q[2], *reinterpret_cast<float(*)[8]>(fw0));
    unpack16(q[3], *reinterpret_cast<float(*)[8]>(fw0 + 8));
    unpack16(q[4], *reinterpret_cast<float(*)[8]>(fw1));
    unpack16(q[5], *reinterpret_cast<float(*)[8]>(fw1 + 8));
    __syncwarp();   // the previous chunk's reads are done
#pragma unroll
    for (int k = 0; k < kRK; ++k) {
      if (lane < kRT) xs[k * kRT + lane] = fx[k];
      ws[k * kRE + lane] = fw0[k];
      ws[k * kRE + lane + 32] = fw1[k];
      sx = fmaf(fx[k], fx[k], sx);
      sw0 = fmaf(fw0[k], fw0[k], sw0);
      sw1 = fmaf(fw1[k], fw1[k], sw1);
    }
    __syncwarp();
    fetch(c + kRWarps);
    unsigned long long part[kRTL][4];
#pragma unroll
    for (int i = 0; i < kRTL; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) part[i][j] = 0ull;
#pragma unroll 4
    for (int k = 0; k < kRK; ++k) {
      const float4 xa = *reinterpret_cast<const float4*>(xs + k * kRT + ty * kRTL);
      const float4 xb = *reinterpret_cast<const float4*>(xs + k * kRT + ty * kRTL + 4);
      const ulonglong2 wa = *reinterpret_cast<const ulonglong2*>(ws + k * kRE + tx * 4);
      const ulonglong2 wb = *reinterpret_cast<const ulonglong2*>(ws + k * kRE + 32 + tx * 4);
      const float xv[kRTL] = {xa.x, xa.y, xa.z, xa.w, xb.x, xb.y, xb.z, xb.w};
#pragma unroll
      for (int i = 0; i < kRTL; ++i) {
        const unsigned long long xx = f2pack(xv[i], xv[i]);
        ffma2(part[i][0], xx, wa.x);
        ffma2(part[i][1], xx, wa.y);
        ffma2(part[i][2], xx, wb.x);
        ffma2(part[i][3], xx, wb.y);
      }
    }
#pragma unroll
    for (int i = 0; i < kRTL; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 p = f2unpack(part[i][j]), t = f2unpack(tot[i][j]);
        tot[i][j] = f2pack(t.x + p.x, t.y + p.y);
      }
  }
  if (lane < kRT) nx_w[lane] = sx;
  nw_w[lane] = sw0;
  nw_w[lane + 32] = sw1;
  __syncthreads();   // every warp is past its staging slice
  // warp totals: red[warp][t][e]
  float* red = rsm + (size_t)warp * kRT * kRE;
#pragma unroll
  for (int i = 0; i < kRTL; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 t = f2unpack(tot[i][j]);
      const int e = (j < 2 ? tx * 4 : 32 + tx * 4) + 2 * (j & 1);
      red[(ty * kRTL + i) * kRE + e] = t.x;
      red[(ty * kRTL + i) * kRE + e + 1] = t.y;
    }
  __syncthreads();
  const int n = kRK + a.D / (kRWarps * kRK) + kRWarps + 3;
  const float gm = gamma_f32(n);
  const float scale = 2.f * gm * (1.f + 2.f * gm);
  const float tiny = float(n) * 2.8025969e-45f;                   // n * 2^-148
  const float gD = gamma_f32(a.D);
  const float sub = float(a.D) * 1.4012985e-45f;                  // D * 2^-149
  const float* nrm = rsm + kNormOff;
  for (int p = threadIdx.x; p < kRT * kRE; p += kRThreads) {
    const int tr = p / kRE, er = p - tr * kRE;
    const int t = t0 + tr, e = e0 + er;
    if (t >= a.T || e >= a.E) continue;
    float zt = 0.f, nx = 0.f, nw = 0.f;
#pragma unroll
    for (int w = 0; w < kRWarps; ++w) {
      zt += rsm[(size_t)w * kRT * kRE + p];
      nx += nrm[w * (kRT + kRE) + tr];
      nw += nrm[w * (kRT + kRE) + kRT + er];
    }
    // upper bounds of the squared norms from their fp32 sums (any order: error
    // <= gamma_D), then S <= ||x_t|| ||W_r[e]||
    const float S = sqrtf((nx + sub) * (1.f + 3.f * gD)) * sqrtf((nw + sub) * (1.f + 3.f * gD)) * (1.f + 1e-6f);
    const float b = a.b_r[e];
    const float z = zt + b;
    const float B = scale * (S + fabsf(b)) + tiny;
    const size_t o = (size_t)t * a.E + e;
    if (fabsf(z) > B) {
      a.r[o] = z > 0.f ? z : 0.f;
      a.act[o] = z > 0.f ? 1 : 0;
    } else {
      const int slot = atomicAdd(a.n_fb, 1);
      a.fb[slot] = make_int2((int)o, __float_as_int(z));   // NaN lands here too
    }
  }
}

// exact sign of every listed pair: one warp each, integer accumulation
__global__ void __launch_bounds__(256) k_router_exact(const RouterArgs a) {
  __shared__ unsigned long long limbs[8][kLimbs];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n = *a.n_fb;
  bool bad = false;
  for (int i = blockIdx.x * 8 + warp; i < n; i += gridDim.x * 8) {
    const int2 f = a.fb[i];
    const int t = f.x / a.E, e = f.x - t * a.E;
    const float z = __int_as_float(f.y);
    const int sg = exact_sign_warp(a.x + (size_t)t * a.D, a.W_r + (size_t)e * a.D, a.D, a.b_r[e],
                                   limbs[warp], &bad);
    if (lane == 0) {
      a.r[f.x] = sg > 0 ? fmaxf(z, 0.f) : 0.f;
      a.act[f.x] = sg > 0 ? 1 : 0;
    }
  }
  if (bad && lane == 0) atomicOr(a.err, 1);
}

// ---------------------------------------------------------------------------
// out[t] = S[t] + sum over the token's active experts, ascending, of
// s_e r_e v[pair] (+ x[t]): one CTA per token, 8 columns per thread, 16-byte
// coalesced loads.

constexpr int kCThreads = 256;

__global__ void __launch_bounds__(kCThreads) k_combine(const float* __restrict__ S, const __half* __restrict__ v,
                                                       const float* __restrict__ coef,
                                                       const int* __restrict__ pair_of,
                                                       const bf16* __restrict__ x, bf16* __restrict__ out,
                                                       int D, int E, int residual) {
  __shared__ int list[256];
  __shared__ float list_c[256];
  __shared__ int n_list;
  const int t = blockIdx.x, lane = threadIdx.x & 31;
  if (threadIdx.x < 32) {   // the token's pairs in ascending expert order
    int n = 0;
    for (int e0 = 0; e0 < E; e0 += 32) {
      const int e = e0 + lane;
      const int q = e < E ? pair_of[(size_t)t * E + e] : -1;
      const unsigned m = __ballot_sync(kFull, q >= 0);
      if (q >= 0) list[n + __popc(m & ((1u << lane) - 1u))] = q;
      n += __popc(m);
    }
    if (lane == 0) n_list = n;
  }
  __syncthreads();
  const int n = n_list;
  if (threadIdx.x < n) list_c[threadIdx.x] = coef[list[threadIdx.x]];
  __syncthreads();
  for (int c = threadIdx.x * 8; c < D; c += kCThreads * 8) {
    const float4* sp = reinterpret_cast<const float4*>(S + (size_t)t * D + c);
    const float4 s0 = sp[0], s1 = sp[1];
    float acc[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
    for (int i = 0; i < n; i += 8) {   // up to 8 rows in flight, added in list order
      uint4 w[8];
#pragma unroll
      for (int j = 0; j < 8; ++j)
        w[j] = i + j < n ? __ldg(reinterpret_cast<const uint4*>(v + (size_t)list[i + j] * D + c))
                         : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (i + j >= n) break;
        const uint32_t ws4[4] = {w[j].x, w[j].y, w[j].z, w[j].w};
        const float cf = list_c[i + j];
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&ws4[h]));
          acc[2 * h] = fmaf(cf, f.x, acc[2 * h]);
          acc[2 * h + 1] = fmaf(cf, f.y, acc[2 * h + 1]);
        }
      }
    }
    if (residual) {
      float f[8];
      unpack16(*reinterpret_cast<const uint4*>(x + (size_t)t * D + c), f);
#pragma unroll
      for (int j = 0; j < 8; ++j) acc[j] += f[j];
    }
    uint4 o;
    o.x = pack_bf16x2(acc[0], acc[1]);
    o.y = pack_bf16x2(acc[2], acc[3]);
    o.z = pack_bf16x2(acc[4], acc[5]);
    o.w = pack_bf16x2(acc[6], acc[7]);
    *reinterpret_cast<uint4*>(out + (size_t)t * D + c) = o;
  }
}

// ---------------------------------------------------------------------------
// Token -> expert tables for large batches: a stable counting sort of the
// active (token, expert) pairs by expert, tokens ascending within an expert.
// The tokens are cut into units of 32, one warp each.  k_tab_count counts a
// unit's pairs per expert with one ballot per expert (and every token's pair
// count); k_tab_scatter gives each unit, per expert, the pairs of the experts
// before it plus the pairs of the same expert in earlier units, and places
// the unit's pairs lane by lane.  Unit 0 also writes counts, offsets and the
// list of row tiles (<= tile_rows pairs of one expert each).

constexpr int kTabThreads = 128;                 // 4 units per block
constexpr int kTabWarps = kTabThreads / 32;
constexpr int kTabUnit = 32;                     // tokens per unit

// The active flags of a unit's 32 tokens, [32][E] bytes, into shared memory
// with 16-byte loads where the rows allow it (tokens past T read as 0).
__device__ __forceinline__ void load_unit_flags(const uint8_t* __restrict__ act, int T, int E, int u, uint8_t* fl) {
  const int lane = threadIdx.x & 31;
  const int t0 = u * kTabUnit;
  const int nt = min(kTabUnit, T - t0);
  const uint8_t* src = act + (size_t)t0 * E;
  const int nbytes = nt * E;
  if ((E & 15) == 0 && (reinterpret_cast<uintptr_t>(act) & 15) == 0) {   // 16-byte aligned: vector loads
    for (int i = lane; i < nbytes / 16; i += 32)
      reinterpret_cast<uint4*>(fl)[i] = __ldg(reinterpret_cast<const uint4*>(src) + i);
  } else {
    for (int i = lane; i < nbytes; i += 32) fl[i] = src[i];
  }
  for (int i = nbytes + lane; i < kTabUnit * E; i += 32) fl[i] = 0;
  __syncwarp();
}

__global__ void __launch_bounds__(kTabThreads) k_tab_count(const uint8_t* __restrict__ act, int T, int E,
                                                           int* __restrict__ n_tok, int* __restrict__ unit_counts) {
  __shared__ __align__(16) uint8_t flags[kTabWarps][kTabUnit * 256];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int u = blockIdx.x * kTabWarps + warp;
  if (u * kTabUnit >= T) return;   // whole warps
  uint8_t* fl = flags[warp];
  load_unit_flags(act, T, E, u, fl);
  // the unit's pairs per expert: lane j sums experts j, j + 32, ... over the 32 tokens
  for (int e = lane; e < E; e += 32) {
    int c = 0;
#pragma unroll 8
    for (int t = 0; t < kTabUnit; ++t) c += fl[t * E + e];
    unit_counts[(size_t)u * E + e] = c;
  }
  // each token's pair count: lane = token
  const int t = u * kTabUnit + lane;
  if (t < T) {
    int n = 0;
    for (int e = 0; e < E; ++e) n += fl[lane * E + ((e + lane) % E)];   // rotated start: no bank conflicts
    n_tok[t] = n;
  }
}

// Per expert e, the pairs of e in the units before each unit (exclusive scan
// over units, in place in unit_counts) and e's total: one warp per expert.
__global__ void __launch_bounds__(kTabThreads) k_tab_scan(int E, int nu, int* __restrict__ unit_counts,
                                                          int* __restrict__ totals) {
  const int lane = threadIdx.x & 31;
  const int e = blockIdx.x * kTabWarps + (threadIdx.x >> 5);
  if (e >= E) return;   // whole warps
  int run = 0;
  for (int v0 = 0; v0 < nu; v0 += 32) {
    const int v = v0 + lane;
    const int c = v < nu ? unit_counts[(size_t)v * E + e] : 0;
    int incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(kFull, incl, o);
      if (lane >= o) incl += y;
    }
    if (v < nu) unit_counts[(size_t)v * E + e] = run + incl - c;
    run += __shfl_sync(kFull, incl, 31);
  }
  if (lane == 0) totals[e] = run;
}

__global__ void __launch_bounds__(kTabThreads) k_tab_scatter(const uint8_t* __restrict__ act, int T, int E,
                                                             const int* __restrict__ unit_base,
                                                             const int* __restrict__ totals, int* counts,
                                                             int* offsets, int* perm, int* pair_of, int4* tiles,
                                                             int* n_tiles, int tile_rows) {
  __shared__ __align__(16) uint8_t flags[kTabWarps][kTabUnit * 256];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int u = blockIdx.x * kTabWarps + warp;
  if (u * kTabUnit >= T) return;   // whole warps; no block-wide barrier below
  // per expert (lane j: experts j, j + 32, ...): the total count and the
  // pairs of the expert in earlier units
  int tot[8], before[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int e = lane + 32 * i;
    tot[i] = e < E ? totals[e] : 0;
    before[i] = e < E ? unit_base[(size_t)u * E + e] : 0;
  }
  uint8_t* fl = flags[warp];
  load_unit_flags(act, T, E, u, fl);
  // exclusive scan of tot over experts (ascending e = i * 32 + lane)
  int run = 0, ntl_run = 0;
  int off[8], toff[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int c = (lane + 32 * i < E) ? tot[i] : 0;
    const int nt = (c + tile_rows - 1) / tile_rows;
    int incl = c, incl_t = nt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(kFull, incl, o), yt = __shfl_up_sync(kFull, incl_t, o);
      if (lane >= o) {
        incl += y;
        incl_t += yt;
      }
    }
    off[i] = run + incl - c;
    toff[i] = ntl_run + incl_t - nt;
    run += __shfl_sync(kFull, incl, 31);
    ntl_run += __shfl_sync(kFull, incl_t, 31);
  }
  if (u == 0) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int e = lane + 32 * i;
      if (e >= E) continue;
      counts[e] = tot[i];
      offsets[e] = off[i];
      const int n = (tot[i] + tile_rows - 1) / tile_rows;
      for (int j = 0; j < n; ++j)
        tiles[toff[i] + j] = make_int4(e, off[i] + j * tile_rows, min(tile_rows, tot[i] - j * tile_rows), 0);
    }
    if (lane == 0) {
      offsets[E] = run;
      *n_tiles = ntl_run;
    }
  }
  // the unit's pairs: lane j walks the 32 tokens for experts j, j + 32, ...;
  // the pair_of row of a token is written by the lanes together
  const int t0 = u * kTabUnit;
  const int nt = min(kTabUnit, T - t0);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int e = lane + 32 * i;
    if (i * 32 >= E) break;
    int pos = off[i] + before[i];
    for (int t = 0; t < nt; ++t) {
      const bool f = e < E && fl[t * E + e];
      if (f) perm[pos] = t0 + t;
      if (e < E) pair_of[(size_t)(t0 + t) * E + e] = f ? pos : -1;
      pos += f ? 1 : 0;
    }
  }
}

}  // namespace pf
}  // namespace deco
