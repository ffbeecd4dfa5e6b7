// General-shape CUDA-core kernels of the DECO MoE layer: router with exact
// activation decisions, token->expert tables, grouped up-projection with the
// NormSiLU epilogue (cluster/DSMEM RMS reduction), and the down-projection with
// s_e*r_e scaling, a fixed-order combine and the shared expert.
//
// Layer definition: "DECO: Sparse Mixture-of-Experts with Dense-Comparable
// Performance on End-Side Devices", §1 and §2 (Router design, Expert design);
// NormSiLU's two steps as the qidianchuan.cn summary's core-design part gives
// them.
#pragma once

#include <cooperative_groups.h>

#include "common.cuh"

namespace deco {

constexpr int kThreads = 256;   // 8 warps
constexpr int kWarps = 8;
constexpr int kCluster = 8;     // CTAs sharing one expert's d_e rows in k_up

// ---------------------------------------------------------------------------
// dot products of one weight row with TT token rows staged in shared memory.
// Each lane accumulates its D/32 products sequentially (one FMA per term),
// then a 5-level xor butterfly adds the lanes: every lane ends with the same
// total, and the total has gone through D/32 + 5 roundings.

template <typename T, int TT, bool ABS>
__device__ __forceinline__ void dot_row_tokens(const T* __restrict__ w, const T* xs, int D,
                                               float (&acc)[TT], float (&aacc)[TT]) {
  constexpr int V = VecN<T>::N;
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int tt = 0; tt < TT; ++tt) {
    acc[tt] = 0.f;
    aacc[tt] = 0.f;
  }
#pragma unroll 4
  for (int k = lane * V; k < D; k += 32 * V) {
    float wv[V];
    load_w<T, V>(w + k, wv);
#pragma unroll
    for (int tt = 0; tt < TT; ++tt) {
      float xv[V];
      load_s<T, V>(xs + (size_t)tt * D + k, xv);
#pragma unroll
      for (int i = 0; i < V; ++i) {
        acc[tt] = fmaf(xv[i], wv[i], acc[tt]);
        if (ABS) aacc[tt] = fmaf(fabsf(xv[i]), fabsf(wv[i]), aacc[tt]);
      }
    }
  }
#pragma unroll
  for (int tt = 0; tt < TT; ++tt) {
    acc[tt] = warp_sum(acc[tt]);
    if (ABS) aacc[tt] = warp_sum(aacc[tt]);
  }
}

// stage token rows x[tok[i]] (i < TT; tok < 0 -> zeros) into xs[TT][D]
template <typename T, int TT>
__device__ __forceinline__ void stage_rows(const T* __restrict__ x, int D, const int* tok, T* xs) {
  constexpr int V = VecN<T>::N;
  const int vpr = D / V;
  for (int i = threadIdx.x; i < TT * vpr; i += blockDim.x) {
    const int tt = i / vpr, c = i - tt * vpr;
    const int t = tok[tt];
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (t >= 0) v = *reinterpret_cast<const uint4*>(x + (size_t)t * D + (size_t)c * V);
    reinterpret_cast<uint4*>(xs)[i] = v;
  }
}

// ---------------------------------------------------------------------------
// k_route: one pass over the rows [W_r ; W_bar_up ; W_s_up] for a chunk of TT
// tokens.  Router rows give r = ReLU(z) and the exact active flag; mean rows
// give u = x W_bar_up^T; shared rows give hs = SiLU(x W_s_up^T).

struct RouteArgs {
  const void* x;
  int T, D;
  const void* W_r;
  const float* b_r;
  int E;
  const void* W_bar;
  int d_e;
  const void* W_s_up;
  int d_s;
  float* r;          // [T][E]
  uint8_t* act;      // [T][E]
  float* u;          // [T][d_e]
  float* hs;         // [T][d_s]
  int* err;
  float* zt;         // TopK routing: [T][E] fp32 logits (router rows then decide nothing)
  float* bt;         // TopK routing: [T][E] bound on |fp32 logit - exact logit|
};

template <typename T, int TT>
__global__ void __launch_bounds__(kThreads) k_route(RouteArgs a) {
  extern __shared__ __align__(16) unsigned char smem[];
  T* xs = reinterpret_cast<T*>(smem);
  unsigned long long* limbs =
      reinterpret_cast<unsigned long long*>(smem + (size_t)TT * a.D * sizeof(T));
  __shared__ int tok[TT];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t0 = blockIdx.y * TT;
  const int nt = min(TT, a.T - t0);
  if (threadIdx.x < TT) tok[threadIdx.x] = (int)threadIdx.x < nt ? t0 + (int)threadIdx.x : -1;
  __syncthreads();
  stage_rows<T, TT>(reinterpret_cast<const T*>(a.x), a.D, tok, xs);
  __syncthreads();

  const int R = a.E + a.d_e + a.d_s;
  const int row = blockIdx.x * kWarps + warp;
  if (row >= R) return;
  float acc[TT], aacc[TT];
  if (row < a.E) {
    const int e = row;
    const T* w = reinterpret_cast<const T*>(a.W_r) + (size_t)e * a.D;
    dot_row_tokens<T, TT, true>(w, xs, a.D, acc, aacc);
    const float b = a.b_r[e];
    // rigorous bound on |fp32 value - exact value|: n = D/32 lane terms +
    // 5 butterfly levels + the bias add; factor 2 of margin; gradual
    // underflow adds at most 2^-149 per operation.
    const int n = a.D / 32 + 6;
    const float g = gamma_f32(n);
    const float scale = 2.f * g * (1.f + 2.f * g);
    const float tiny = float(n) * 2.8025969e-45f;  // n * 2^-148
    bool bad = false;
    for (int tt = 0; tt < nt; ++tt) {
      float z = acc[tt] + b;
      const float B = scale * (aacc[tt] + fabsf(b)) + tiny;
      if (a.zt) {                // TopK: k_topk_select ranks the logits
        if (lane == 0) {
          const size_t o = (size_t)(t0 + tt) * a.E + e;
          a.zt[o] = z;
          a.bt[o] = B;
        }
        continue;
      }
      bool on;
      if (fabsf(z) > B) {
        on = z > 0.f;
      } else {
        on = exact_sign_warp(xs + (size_t)tt * a.D, w, a.D, b, limbs + warp * kLimbs, &bad) > 0;
      }
      if (lane == 0) {
        const size_t o = (size_t)(t0 + tt) * a.E + e;
        a.r[o] = on ? fmaxf(z, 0.f) : 0.f;
        a.act[o] = on ? 1 : 0;
      }
    }
    if (bad && lane == 0) atomicOr(a.err, 1);
  } else if (row < a.E + a.d_e) {
    const int j = row - a.E;
    const T* w = reinterpret_cast<const T*>(a.W_bar) + (size_t)j * a.D;
    dot_row_tokens<T, TT, false>(w, xs, a.D, acc, aacc);
    if (lane == 0)
      for (int tt = 0; tt < nt; ++tt) a.u[(size_t)(t0 + tt) * a.d_e + j] = acc[tt];
  } else {
    const int j = row - a.E - a.d_e;
    const T* w = reinterpret_cast<const T*>(a.W_s_up) + (size_t)j * a.D;
    dot_row_tokens<T, TT, false>(w, xs, a.D, acc, aacc);
    if (lane == 0)
      for (int tt = 0; tt < nt; ++tt) a.hs[(size_t)(t0 + tt) * a.d_s + j] = silu_f(acc[tt]);
  }
}

// ---------------------------------------------------------------------------
// token -> expert tables: a stable counting sort of the (token, expert) pairs
// by expert.  k_count: per-expert counts (blocks < E) and per-token counts.
// k_scatter: offsets, perm, pair index of every (t, e), and the list of
// up-projection tiles (<= tile_rows pairs of one expert each).

__global__ void __launch_bounds__(kThreads) k_count(const uint8_t* __restrict__ act, int T, int E,
                                                    int* counts, int* n_tok) {
  __shared__ int red[kWarps];
  if ((int)blockIdx.x < E) {
    const int e = blockIdx.x;
    int c = 0;
    for (int t = threadIdx.x; t < T; t += blockDim.x) c += act[(size_t)t * E + e];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(kFull, c, o);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = c;
    __syncthreads();
    if (threadIdx.x == 0) {
      int s = 0;
      for (int i = 0; i < kWarps; ++i) s += red[i];
      counts[e] = s;
    }
  } else {
    const int t = (blockIdx.x - E) * blockDim.x + threadIdx.x;
    if (t < T && n_tok) {
      int c = 0;
      for (int e = 0; e < E; ++e) c += act[(size_t)t * E + e];
      n_tok[t] = c;
    }
  }
}

__global__ void __launch_bounds__(kThreads) k_scatter(const uint8_t* __restrict__ act, int T, int E,
                                                      const int* __restrict__ counts, int* offsets,
                                                      int* perm, int* pair_of, int4* tiles,
                                                      int* n_tiles, int tile_rows) {
  __shared__ int s_off, s_toff, s_base;
  __shared__ int wsum[kWarps];
  const int e = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    int o = 0, to = 0;
    for (int q = 0; q < e; ++q) {
      o += counts[q];
      to += (counts[q] + tile_rows - 1) / tile_rows;
    }
    s_off = o;
    s_toff = to;
    s_base = 0;
    offsets[e] = o;
    if (e == E - 1) {
      offsets[E] = o + counts[e];
      if (n_tiles) *n_tiles = to + (counts[e] + tile_rows - 1) / tile_rows;
    }
  }
  __syncthreads();
  const int cnt = counts[e];
  if (tiles) {
    const int ntl = (cnt + tile_rows - 1) / tile_rows;
    for (int j = threadIdx.x; j < ntl; j += blockDim.x)
      tiles[s_toff + j] = make_int4(e, s_off + j * tile_rows, min(tile_rows, cnt - j * tile_rows), 0);
  }
  for (int t0 = 0; t0 < T; t0 += blockDim.x) {
    const int t = t0 + threadIdx.x;
    const int f = (t < T) ? act[(size_t)t * E + e] : 0;
    int incl = f;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(kFull, incl, o);
      if (lane >= o) incl += v;
    }
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    int before = 0, total = 0;
    for (int i = 0; i < kWarps; ++i) {
      if (i < warp) before += wsum[i];
      total += wsum[i];
    }
    if (t < T) {
      if (f) {
        const int pos = s_off + s_base + before + incl - 1;
        if (perm) perm[pos] = t;
        if (pair_of) pair_of[(size_t)t * E + e] = pos;
      } else if (pair_of) {
        pair_of[(size_t)t * E + e] = -1;
      }
    }
    __syncthreads();
    if (threadIdx.x == 0) s_base += total;
    __syncthreads();
  }
}

// ---------------------------------------------------------------------------
// k_up: grouped up-projection with the NormSiLU epilogue.  A cluster of 8 CTAs
// owns one tile (<= TT pairs of one expert e); CTA q computes rows
// [q*d_e/8, (q+1)*d_e/8) of g = W_up[e] x_t, centres them (c = g - u_t), and
// publishes its partial sum of c^2 per pair.  After a cluster barrier every
// CTA adds the 8 partials in rank order through distributed shared memory,
// giving the RMS over all d_e features, and writes a = SiLU(c / rms) for its
// rows to H[pair][d_e] (times the value branch W_val[e] x_t for gated experts).

struct UpArgs {
  const void* x;
  int D;
  const void* W_up;
  const void* W_val;   // gated experts' value branch, or null
  int d_e;
  const float* u;
  const int* perm;
  const int4* tiles;
  const int* n_tiles;
  float* H;
  float eps;
};

template <typename T, int TT>
__global__ void __cluster_dims__(kCluster, 1, 1) __launch_bounds__(kThreads) k_up(UpArgs a) {
  namespace cg = cooperative_groups;
  cg::cluster_group cluster = cg::this_cluster();
  extern __shared__ __align__(16) unsigned char smem[];
  const int RPC = a.d_e / kCluster;
  T* xs = reinterpret_cast<T*>(smem);
  float* gs = reinterpret_cast<float*>(smem + (size_t)TT * a.D * sizeof(T));   // [TT][RPC]
  float* vs = gs + TT * RPC;                                                     // [TT][RPC] (gated)
  __shared__ float part[TT];
  __shared__ float rinv[TT];
  __shared__ int tok[TT];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rank = (int)cluster.block_rank();
  const int cid = blockIdx.x / kCluster, ncl = gridDim.x / kCluster;
  const int j0 = rank * RPC;
  const int ntiles = *a.n_tiles;
  for (int ti = cid; ti < ntiles; ti += ncl) {
    const int4 tile = a.tiles[ti];
    const int e = tile.x, p0 = tile.y, np = tile.z;
    if (threadIdx.x < TT) tok[threadIdx.x] = threadIdx.x < np ? a.perm[p0 + threadIdx.x] : -1;
    __syncthreads();
    stage_rows<T, TT>(reinterpret_cast<const T*>(a.x), a.D, tok, xs);
    __syncthreads();
    for (int jr = warp; jr < RPC; jr += kWarps) {
      const T* w = reinterpret_cast<const T*>(a.W_up) + ((size_t)e * a.d_e + j0 + jr) * a.D;
      float acc[TT], dummy[TT];
      dot_row_tokens<T, TT, false>(w, xs, a.D, acc, dummy);
      if (lane == 0)
        for (int tt = 0; tt < np; ++tt)
          gs[tt * RPC + jr] = acc[tt] - a.u[(size_t)tok[tt] * a.d_e + j0 + jr];
      if (a.W_val) {   // gated: the value branch of the same row
        const T* wv = reinterpret_cast<const T*>(a.W_val) + ((size_t)e * a.d_e + j0 + jr) * a.D;
        dot_row_tokens<T, TT, false>(wv, xs, a.D, acc, dummy);
        if (lane == 0)
          for (int tt = 0; tt < np; ++tt) vs[tt * RPC + jr] = acc[tt];
      }
    }
    __syncthreads();
    if (threadIdx.x < TT) {
      float ss = 0.f;
      if ((int)threadIdx.x < np)
        for (int j = 0; j < RPC; ++j) ss = fmaf(gs[threadIdx.x * RPC + j], gs[threadIdx.x * RPC + j], ss);
      part[threadIdx.x] = ss;
    }
    cluster.sync();
    if ((int)threadIdx.x < np) {
      float tot = 0.f;
      for (int q = 0; q < kCluster; ++q) tot += cluster.map_shared_rank(part, q)[threadIdx.x];
      rinv[threadIdx.x] = 1.f / sqrtf(tot / float(a.d_e) + a.eps);
    }
    __syncthreads();
    for (int i = threadIdx.x; i < np * RPC; i += blockDim.x) {
      const int tt = i / RPC, j = i - tt * RPC;
      const float act = silu_f(gs[i] * rinv[tt]);
      a.H[(size_t)(p0 + tt) * a.d_e + j0 + j] = a.W_val ? act * vs[i] : act;
    }
    cluster.sync();   // partial sums stay readable until every rank is done
  }
}

// ---------------------------------------------------------------------------
// k_down: output rows [n0, n0 + 8*RPW) of a chunk of TT tokens.  The CTA walks
// the routed experts in ascending order; for each expert used by a token of
// the chunk it stages those tokens' activations and adds
// s_e * r_{t,e} * (W_down[e][n] . a_{t,e}) to the token's accumulator, then
// adds the shared expert W_s_down[n] . hs_t.  Every output element is thus
// summed in one fixed order: deterministic, with no atomics and no scratch.

struct DownArgs {
  int T, D, E, d_e, d_s;
  const uint8_t* act;
  const float* r;
  const float* s;
  const int* pair_of;
  const float* H;
  const void* W_down;
  const void* W_s_down;
  const float* hs;
  const void* x;
  void* out;
  int residual;
};

constexpr int kDownK = 512;      // staged K chunk (floats per token row)

template <typename T, int TT, int RPW>
__global__ void __launch_bounds__(kThreads) k_down(DownArgs a) {
  constexpr int V = VecN<T>::N;
  extern __shared__ __align__(16) unsigned char smem[];
  float* hbuf = reinterpret_cast<float*>(smem);                          // [TT][kDownK]
  uint32_t* emask = reinterpret_cast<uint32_t*>(smem + sizeof(float) * TT * kDownK);  // [E]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * kWarps * RPW;
  const int t0 = blockIdx.y * TT;
  const int nt = min(TT, a.T - t0);
  for (int e = threadIdx.x; e < a.E; e += blockDim.x) {
    uint32_t m = 0;
    for (int tt = 0; tt < nt; ++tt)
      if (a.act[(size_t)(t0 + tt) * a.E + e]) m |= 1u << tt;
    emask[e] = m;
  }
  __syncthreads();
  float acc[RPW];
#pragma unroll
  for (int q = 0; q < RPW; ++q) acc[q] = 0.f;

  const T* Wd = reinterpret_cast<const T*>(a.W_down);
  for (int e = 0; e < a.E; ++e) {
    const uint32_t m = emask[e];
    if (!m) continue;
    const int q4 = a.d_e / 4;
    for (int i = threadIdx.x; i < TT * q4; i += blockDim.x) {
      const int tt = i / q4, c = i - tt * q4;
      if ((m >> tt) & 1u) {
        const int p = a.pair_of[(size_t)(t0 + tt) * a.E + e];
        reinterpret_cast<float4*>(hbuf + tt * kDownK)[c] =
            reinterpret_cast<const float4*>(a.H + (size_t)p * a.d_e)[c];
      }
    }
    __syncthreads();
    float coef = 0.f;
    if (lane < nt && ((m >> lane) & 1u)) coef = a.s[e] * a.r[(size_t)(t0 + lane) * a.E + e];
#pragma unroll
    for (int q = 0; q < RPW; ++q) {
      const int n = n0 + warp * RPW + q;
      const T* w = Wd + ((size_t)e * a.D + n) * a.d_e;
      float wv[kDownK / 32];   // this lane's share of the row (d_e <= kDownK)
      int nw = 0;
      for (int k = lane * V; k < a.d_e; k += 32 * V) {
        float v[V];
        load_w<T, V>(w + k, v);
#pragma unroll
        for (int i = 0; i < V; ++i) wv[nw + i] = v[i];
        nw += V;
      }
      for (uint32_t mm = m; mm; mm &= mm - 1) {
        const int tt = __ffs(mm) - 1;
        const float* h = hbuf + tt * kDownK;
        float p = 0.f;
        int idx = 0;
        for (int k = lane * V; k < a.d_e; k += 32 * V) {
#pragma unroll
          for (int i = 0; i < V; ++i) p = fmaf(wv[idx + i], h[k + i], p);
          idx += V;
        }
        p = warp_sum(p);
        if (lane == tt) acc[q] = fmaf(coef, p, acc[q]);
      }
    }
    __syncthreads();
  }

  // shared expert, K staged in chunks of kDownK
  float sacc[RPW];
#pragma unroll
  for (int q = 0; q < RPW; ++q) sacc[q] = 0.f;
  const T* Ws = reinterpret_cast<const T*>(a.W_s_down);
  for (int k0 = 0; k0 < a.d_s; k0 += kDownK) {
    const int kc = min(kDownK, a.d_s - k0);
    const int q4 = kc / 4;
    for (int i = threadIdx.x; i < nt * q4; i += blockDim.x) {
      const int tt = i / q4, c = i - tt * q4;
      reinterpret_cast<float4*>(hbuf + tt * kDownK)[c] =
          reinterpret_cast<const float4*>(a.hs + (size_t)(t0 + tt) * a.d_s + k0)[c];
    }
    __syncthreads();
#pragma unroll
    for (int q = 0; q < RPW; ++q) {
      const int n = n0 + warp * RPW + q;
      const T* w = Ws + (size_t)n * a.d_s + k0;
      float wv[kDownK / 32];
      int nw = 0;
      for (int k = lane * V; k < kc; k += 32 * V) {
        float v[V];
        load_w<T, V>(w + k, v);
#pragma unroll
        for (int i = 0; i < V; ++i) wv[nw + i] = v[i];
        nw += V;
      }
      for (int tt = 0; tt < nt; ++tt) {
        const float* h = hbuf + tt * kDownK;
        float p = 0.f;
        int idx = 0;
        for (int k = lane * V; k < kc; k += 32 * V) {
#pragma unroll
          for (int i = 0; i < V; ++i) p = fmaf(wv[idx + i], h[k + i], p);
          idx += V;
        }
        p = warp_sum(p);
        if (lane == tt) sacc[q] += p;
      }
    }
    __syncthreads();
  }
  if (lane < nt) {
    const int t = t0 + lane;
#pragma unroll
    for (int q = 0; q < RPW; ++q) {
      const int n = n0 + warp * RPW + q;
      float v = acc[q] + sacc[q];
      if (a.residual) v += to_f32(reinterpret_cast<const T*>(a.x)[(size_t)t * a.D + n]);
      reinterpret_cast<T*>(a.out)[(size_t)t * a.D + n] = from_f32<T>(v);
    }
  }
}

// ---------------------------------------------------------------------------
// mean up-projection: fp64 sum over experts in ascending order, fp64 divide,
// one round-to-nearest-even to the storage dtype.

template <typename T>
__global__ void k_mean_up(const T* __restrict__ W_up, T* __restrict__ W_bar, int E, size_t n) {
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n;
       i += (size_t)gridDim.x * blockDim.x) {
    double acc = 0.0;
    for (int e = 0; e < E; ++e) acc += (double)to_f32(W_up[(size_t)e * n + i]);
    const double m = acc / (double)E;
    if constexpr (sizeof(T) == 4) {
      W_bar[i] = __double2float_rn(m);
    } else {
      W_bar[i] = __double2bfloat16(m);
    }
  }
}


// ---------------------------------------------------------------------------
// TopK routing (the conventional baseline DECO is compared with at the same
// activation ratio, "DECO: Sparse Mixture-of-Experts with Dense-Comparable
// Performance on End-Side Devices", §5): each token keeps its k largest
// logits, ties to the lower expert index, with weights ReLU(z).  The ranking
// is exact: one warp per token ranks the fp32 logits, and the selection
// stands if the k-th lower bound (logit - B) lies above every unselected
// upper bound (logit + B); otherwise only the experts whose intervals overlap
// that boundary are ranked among themselves by exact comparisons
// (exact_cmp_warp), while the ones above or below it are certain.

struct TopkArgs {
  const void* x;
  const void* W_r;
  const float* b_r;
  int T, D, E, k;
  const float* zt;   // [T][E] fp32 logits
  const float* bt;   // [T][E] their error bounds
  float* r;          // [T][E]
  uint8_t* act;      // [T][E]
  int* err;
};

constexpr int kTopkWarps = 8;

template <typename T>
__global__ void __launch_bounds__(kTopkWarps * 32) k_topk_select(const TopkArgs a) {
  __shared__ float sz[kTopkWarps][256];
  __shared__ int mlist[kTopkWarps][256];
  __shared__ int mrank[kTopkWarps][256];
  __shared__ unsigned long long limbs[kTopkWarps][kLimbs];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * kTopkWarps + warp;
  if (t >= a.T) return;   // whole warps only: no block-wide barrier below
  const float inf = __int_as_float(0x7f800000);
  float z[8], B[8];
  bool bad = false;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int e = lane + 32 * i;
    z[i] = -inf;
    B[i] = 0.f;
    if (e < a.E) {
      z[i] = a.zt[(size_t)t * a.E + e];
      B[i] = a.bt[(size_t)t * a.E + e];
      if (!(fabsf(z[i]) < inf) || !(B[i] < inf)) {   // non-finite operand: rank it last
        bad = true;
        z[i] = -inf;
        B[i] = 0.f;
      }
      sz[warp][e] = z[i];
    }
  }
  __syncwarp();
  // rank by the fp32 logit, ties to the lower index
  bool in[8];
  float lo = inf, hi = -inf;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int e = lane + 32 * i;
    in[i] = false;
    if (e >= a.E) continue;
    int rank = 0;
    for (int f = 0; f < a.E; ++f) {
      const float v = sz[warp][f];
      rank += (v > z[i] || (v == z[i] && f < e)) ? 1 : 0;
    }
    in[i] = rank < a.k;
    if (in[i]) lo = fminf(lo, z[i] - B[i]);
    else hi = fmaxf(hi, z[i] + B[i]);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    lo = fminf(lo, __shfl_xor_sync(kFull, lo, o));
    hi = fmaxf(hi, __shfl_xor_sync(kFull, hi, o));
  }
  bad = __any_sync(kFull, bad);
  if (!(lo > hi) && !bad) {
    // the boundary is not certain: experts above hi are in, below lo are
    // out, the rest (M) are ranked exactly among themselves
    int n_in = 0, n_m = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int e = lane + 32 * i;
      const bool live = e < a.E;
      const bool sure_in = live && z[i] - B[i] > hi;
      const bool sure_out = live && z[i] + B[i] < lo;
      const bool m = live && !sure_in && !sure_out;
      n_in += __popc(__ballot_sync(kFull, sure_in));
      const unsigned bm = __ballot_sync(kFull, m);
      if (m) mlist[warp][n_m + __popc(bm & ((1u << lane) - 1u))] = e;
      n_m += __popc(bm);
      in[i] = sure_in;
    }
    __syncwarp();
    for (int i = lane; i < n_m; i += 32) mrank[warp][i] = 0;
    __syncwarp();
    const T* x = static_cast<const T*>(a.x) + (size_t)t * a.D;
    const T* W = static_cast<const T*>(a.W_r);
    for (int i = 0; i < n_m; ++i)
      for (int j = i + 1; j < n_m; ++j) {   // mlist ascending: on an exact tie i ranks above j
        const int ei = mlist[warp][i], ej = mlist[warp][j];
        const int sg = exact_cmp_warp(x, W + (size_t)ei * a.D, W + (size_t)ej * a.D, a.D, a.b_r[ei], a.b_r[ej],
                                      limbs[warp], &bad);
        if (lane == 0) {
          if (sg >= 0) mrank[warp][j] += 1;
          else mrank[warp][i] += 1;
        }
        __syncwarp();
      }
    const int need = a.k - n_in;
    for (int i = 0; i < n_m; ++i) {
      const int e = mlist[warp][i];
      const bool take = mrank[warp][i] < need;
#pragma unroll
      for (int q = 0; q < 8; ++q)
        if (take && e == lane + 32 * q) in[q] = true;
    }
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int e = lane + 32 * i;
    if (e >= a.E) continue;
    const size_t o = (size_t)t * a.E + e;
    a.act[o] = in[i] ? 1 : 0;
    a.r[o] = in[i] ? fmaxf(z[i], 0.f) : 0.f;
  }
  if (bad && lane == 0) atomicOr(a.err, 1);
}

}  // namespace deco
