// Training side of the DECO MoE layer: the backward pass, the router-entropy
// regulariser and its gradient.
//
// Sources: the layer of "DECO: Sparse Mixture-of-Experts with
// Dense-Comparable Performance on End-Side Devices" (§1, §2 Router and Expert
// design); its training objective, adaptive sparsity regularisation on the
// router entropy, from §2 "Auxiliary training objective" and the
// qidianchuan.cn summary's part 3.
//
// Gradients, per token t and active expert e (z_e > 0, r_e = z_e), with
// c = W_up[e] x - u, rho = (mean c^2 + eps)^-1/2, h = rho c, a = SiLU(h)
// (times q = W_val[e] x when gated), v = W_down[e] a, y += s_e r_e v:
//   w = dy . v = (W_down[e]^T dy) . a        ds_e += r_e w
//   dz_e = s_e w (+ an extra logit gradient) dW_r[e] += dz x, db_r[e] += dz
//   dW_down[e] += (s_e r_e dy) a^T           da = s_e r_e W_down[e]^T dy
//   dh = da SiLU'(h) (times q)               dq = da SiLU(h), dW_val[e] += dq x^T
//   dc = rho dh - (rho^3 / d_e) (dh . c) c  dW_up[e] += dc x^T, du -= dc
// and the shared expert and the mean up-projection, whose gradient
// dW_bar = sum_t du x^T reaches every W_up[e] as dW_bar / E.
//
// The kernels run on CUDA cores in fp32 from the stored operands, one output
// element per thread with its sums in a fixed order (pairs of an expert in
// token order, experts of a token ascending), so the gradients are bitwise
// reproducible.  They favour clarity over speed:
//   kb_token_fwd   per token and 64 rows: u = W_bar x, hs = W_s_up x (pre-activation)
//   kb_pair        per active (token, expert): the pair's a, dc, dq, dz, r w
//   kb_token_mid   per token and 32 shared columns: dhs, SiLU(hs); and du
//   kb_dx          per token and 32 columns: dx
//   kb_sums        dW_bar, dW_s_up, dW_s_down (sums over tokens)
//   kb_expert      dW_up (+ dW_bar / E), dW_val, dW_down, dW_r, db_r, ds
//                  (sums over each expert's pairs)
//   kb_entropy     router entropy per token and its logit gradient
#pragma once

#include "common.cuh"

namespace deco {
namespace bwd {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

struct Args {
  int T, D, E, d_e, d_s;
  float eps;
  int gated;
  int residual;           // the layer's output includes x: dx gets dy as well
  const void* x;          // [T][D]
  const void* dy;         // [T][D]
  const float* dz_extra;  // [T][E] or null
  const void* W_r;
  const void* W_bar;
  const void* W_up;
  const void* W_down;
  const float* s;
  const void* W_s_up;
  const void* W_s_down;
  const void* W_val;
  // routing (exact decisions of the forward pass's router)
  const float* r;         // [T][E]
  const uint8_t* act;     // [T][E]
  const int* offsets;     // [E+1]
  const int* perm;        // pairs: token of each, expert-major then token
  const int* pair_of;     // [T][E] pair index of (t, e)
  // workspace
  float* u;      // [T][d_e]
  float* hs;     // [T][d_s]
  float* as;     // [T][d_s]  SiLU(hs)
  float* du;     // [T][d_e]
  float* dhs;    // [T][d_s]
  float* pa;     // [T*E][d_e] a of each pair
  float* pdc;    // [T*E][d_e]
  float* pdq;    // [T*E][d_e] (gated)
  float* pz;     // [T*E] dz
  float* pw;     // [T*E] r w
  float* pk;     // [T*E] s_e r_e
  float* dWbar;  // [d_e][D]
  // gradients (fp32)
  float* dx;
  float* dW_r;
  float* db_r;
  float* dW_up;
  float* dW_down;
  float* ds;
  float* dW_s_up;
  float* dW_s_down;
  float* dW_val;
};

template <typename T>
__device__ __forceinline__ float ldf(const void* p, size_t i) {
  return to_f32(reinterpret_cast<const T*>(p)[i]);
}

__device__ __forceinline__ float silu_grad_f(float h) {
  const float sg = 1.f / (1.f + expf(-h));
  return sg * (1.f + h * (1.f - sg));
}

// row . v over D (v in shared memory), one warp; lanes stride the row
template <typename T>
__device__ __forceinline__ float warp_dot(const void* W, size_t row_off, const float* v, int D, int lane) {
  float acc = 0.f;
  for (int k = lane; k < D; k += 32) acc = fmaf(ldf<T>(W, row_off + k), v[k], acc);
  return warp_sum(acc);
}

// sum over the block's threads of v, in a fixed order (warp trees, then the
// warps in order); every thread gets the total
__device__ __forceinline__ float block_sum(float v, float* red) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  v = warp_sum(v);
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float t = 0.f;
  for (int w = 0; w < kWarps; ++w) t += red[w];
  return t;
}

// per token and block of kFwdRows rows: u = W_bar x and hs = W_s_up x
// (before the SiLU); grid (T, rows / kFwdRows)
constexpr int kFwdRows = 64;
template <typename T>
__global__ void __launch_bounds__(kThreads) kb_token_fwd(const Args a) {
  extern __shared__ float sm[];
  float* xs = sm;   // [D]
  const int t = blockIdx.x, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int k = threadIdx.x; k < a.D; k += kThreads) xs[k] = ldf<T>(a.x, (size_t)t * a.D + k);
  __syncthreads();
  const int j1 = min(a.d_e + a.d_s, (int)(blockIdx.y + 1) * kFwdRows);
  for (int j = blockIdx.y * kFwdRows + warp; j < j1; j += kWarps) {
    const bool mean = j < a.d_e;
    const float v = mean ? warp_dot<T>(a.W_bar, (size_t)j * a.D, xs, a.D, lane)
                         : warp_dot<T>(a.W_s_up, (size_t)(j - a.d_e) * a.D, xs, a.D, lane);
    if (lane == 0) {
      if (mean) a.u[(size_t)t * a.d_e + j] = v;
      else a.hs[(size_t)t * a.d_s + (j - a.d_e)] = v;
    }
  }
}

// per active pair (t, e): recompute its forward values and the pair's
// gradient terms
template <typename T>
__global__ void __launch_bounds__(kThreads) kb_pair(const Args a) {
  const int t = blockIdx.x, e = blockIdx.y;
  if (!a.act[(size_t)t * a.E + e]) return;
  extern __shared__ float sm[];
  float* xs = sm;               // [D]
  float* dys = xs + a.D;        // [D]
  float* g = dys + a.D;         // [d_e] then c
  float* q = g + a.d_e;         // [d_e] value branch
  float* dyw = q + a.d_e;       // [d_e] W_down[e]^T dy
  float* dpart = dyw + a.d_e;   // [kWarps][d_e] per-warp partial sums of it
  __shared__ float red[kWarps];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int p = a.pair_of[(size_t)t * a.E + e];
  for (int k = threadIdx.x; k < a.D; k += kThreads) {
    xs[k] = ldf<T>(a.x, (size_t)t * a.D + k);
    dys[k] = ldf<T>(a.dy, (size_t)t * a.D + k);
  }
  __syncthreads();
  for (int j = warp; j < a.d_e; j += kWarps) {
    const float gj = warp_dot<T>(a.W_up, ((size_t)e * a.d_e + j) * a.D, xs, a.D, lane);
    const float qj = a.gated ? warp_dot<T>(a.W_val, ((size_t)e * a.d_e + j) * a.D, xs, a.D, lane) : 1.f;
    if (lane == 0) {
      g[j] = gj - a.u[(size_t)t * a.d_e + j];   // c
      q[j] = qj;
    }
  }
  {   // W_down[e]^T dy: warp w sums rows n in [w D/8, (w+1) D/8) for columns
      // j = lane + 32 m (8 independent sums per lane), then the warps' parts
      // are added in warp order
    const int n0 = warp * a.D / kWarps, n1 = (warp + 1) * a.D / kWarps;
    for (int m0 = 0; m0 < a.d_e; m0 += 32 * 8) {
      float acc[8];
#pragma unroll
      for (int m = 0; m < 8; ++m) acc[m] = 0.f;
      for (int n = n0; n < n1; ++n) {
        const float dv = dys[n];
        const size_t row = ((size_t)e * a.D + n) * a.d_e;
#pragma unroll
        for (int m = 0; m < 8; ++m) {
          const int j = m0 + 32 * m + lane;
          if (j < a.d_e) acc[m] = fmaf(ldf<T>(a.W_down, row + j), dv, acc[m]);
        }
      }
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        const int j = m0 + 32 * m + lane;
        if (j < a.d_e) dpart[warp * a.d_e + j] = acc[m];
      }
    }
  }
  __syncthreads();
  for (int j = threadIdx.x; j < a.d_e; j += kThreads) {
    float v = 0.f;
    for (int w = 0; w < kWarps; ++w) v += dpart[w * a.d_e + j];
    dyw[j] = v;
  }
  __syncthreads();
  float ss = 0.f;
  for (int j = threadIdx.x; j < a.d_e; j += kThreads) ss = fmaf(g[j], g[j], ss);
  const float ms = block_sum(ss, red) / float(a.d_e);
  const float rho = 1.f / sqrtf(ms + a.eps);
  float wp = 0.f;
  for (int j = threadIdx.x; j < a.d_e; j += kThreads) {
    const float h = rho * g[j];
    const float aj = silu_f(h) * q[j];
    a.pa[(size_t)p * a.d_e + j] = aj;
    wp = fmaf(dyw[j], aj, wp);
  }
  const float w = block_sum(wp, red);
  const float r = a.r[(size_t)t * a.E + e], se = a.s[e];
  const float kk = se * r;
  float dhc = 0.f;
  for (int j = threadIdx.x; j < a.d_e; j += kThreads) {
    const float h = rho * g[j];
    const float da = kk * dyw[j];
    const float dh = da * q[j] * silu_grad_f(h);
    if (a.gated) a.pdq[(size_t)p * a.d_e + j] = da * silu_f(h);
    dyw[j] = dh;   // (each thread rewrites only its own entries)
    dhc = fmaf(dh, g[j], dhc);
  }
  const float sdc = block_sum(dhc, red);
  const float c3 = rho * rho * rho / float(a.d_e) * sdc;
  for (int j = threadIdx.x; j < a.d_e; j += kThreads) a.pdc[(size_t)p * a.d_e + j] = rho * dyw[j] - c3 * g[j];
  if (threadIdx.x == 0) {
    a.pz[p] = se * w + (a.dz_extra ? a.dz_extra[(size_t)t * a.E + e] : 0.f);
    a.pw[p] = r * w;
    a.pk[p] = kk;
  }
}

// per token and block of 32 shared-expert columns i: dhs = (W_s_down^T dy)
// SiLU'(hs) and SiLU(hs), the 8 warps splitting the sum over D (then added
// in warp order); the CTAs of column block 0 also write du = -sum_e dc
// (experts ascending).  Grid (T, ceil(d_s / 32)).
template <typename T>
__global__ void __launch_bounds__(kThreads) kb_token_mid(const Args a) {
  __shared__ float part[kWarps][32];
  const int t = blockIdx.x, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int i = blockIdx.y * 32 + lane;
  const int n0 = warp * a.D / kWarps, n1 = (warp + 1) * a.D / kWarps;
  float acc = 0.f;
  if (i < a.d_s)
    for (int n = n0; n < n1; ++n)
      acc = fmaf(ldf<T>(a.W_s_down, (size_t)n * a.d_s + i), ldf<T>(a.dy, (size_t)t * a.D + n), acc);
  part[warp][lane] = acc;
  __syncthreads();
  if (warp == 0 && i < a.d_s) {
    float v = 0.f;
    for (int w = 0; w < kWarps; ++w) v += part[w][lane];
    const float h = a.hs[(size_t)t * a.d_s + i];
    a.dhs[(size_t)t * a.d_s + i] = v * silu_grad_f(h);
    a.as[(size_t)t * a.d_s + i] = silu_f(h);
  }
  if (blockIdx.y == 0)
    for (int j = threadIdx.x; j < a.d_e; j += kThreads) {
      float d = 0.f;
      for (int e = 0; e < a.E; ++e)
        if (a.act[(size_t)t * a.E + e]) d -= a.pdc[(size_t)a.pair_of[(size_t)t * a.E + e] * a.d_e + j];
      a.du[(size_t)t * a.d_e + j] = d;
    }
}

// per token and block of 32 columns k of dx: the shared expert, then the
// active experts ascending (W_up, W_val, W_r), then the mean up-projection
// (+ dy for a residual layer).  Warp w sums every eighth row of each term for
// lane l's column; the warps' parts are added in warp order.  Grid
// (T, ceil(D / 32)).
template <typename T>
__global__ void __launch_bounds__(kThreads) kb_dx(const Args a) {
  extern __shared__ float sm[];
  float* dhs = sm;            // [d_s]
  float* du = dhs + a.d_s;    // [d_e]
  float* dc = du + a.d_e;     // [d_e]
  float* dq = dc + a.d_e;     // [d_e]
  __shared__ float part[kWarps][32];
  const int t = blockIdx.x, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int k = blockIdx.y * 32 + lane;
  const bool kin = k < a.D;
  for (int i = threadIdx.x; i < a.d_s; i += kThreads) dhs[i] = a.dhs[(size_t)t * a.d_s + i];
  for (int j = threadIdx.x; j < a.d_e; j += kThreads) du[j] = a.du[(size_t)t * a.d_e + j];
  __syncthreads();
  float acc = 0.f;
  if (kin)
    for (int i = warp; i < a.d_s; i += kWarps) acc = fmaf(ldf<T>(a.W_s_up, (size_t)i * a.D + k), dhs[i], acc);
  for (int e = 0; e < a.E; ++e) {
    if (!a.act[(size_t)t * a.E + e]) continue;
    const int p = a.pair_of[(size_t)t * a.E + e];
    __syncthreads();   // dc / dq of the previous expert are consumed
    for (int j = threadIdx.x; j < a.d_e; j += kThreads) {
      dc[j] = a.pdc[(size_t)p * a.d_e + j];
      if (a.gated) dq[j] = a.pdq[(size_t)p * a.d_e + j];
    }
    __syncthreads();
    if (kin) {
      for (int j = warp; j < a.d_e; j += kWarps)
        acc = fmaf(ldf<T>(a.W_up, ((size_t)e * a.d_e + j) * a.D + k), dc[j], acc);
      if (a.gated)
        for (int j = warp; j < a.d_e; j += kWarps)
          acc = fmaf(ldf<T>(a.W_val, ((size_t)e * a.d_e + j) * a.D + k), dq[j], acc);
      if (warp == 0) acc = fmaf(a.pz[p], ldf<T>(a.W_r, (size_t)e * a.D + k), acc);
    }
  }
  if (kin)
    for (int j = warp; j < a.d_e; j += kWarps) acc = fmaf(ldf<T>(a.W_bar, (size_t)j * a.D + k), du[j], acc);
  part[warp][lane] = acc;
  __syncthreads();
  if (warp == 0 && kin) {
    float v = 0.f;
    for (int w = 0; w < kWarps; ++w) v += part[w][lane];
    if (a.residual) v += ldf<T>(a.dy, (size_t)t * a.D + k);
    a.dx[(size_t)t * a.D + k] = v;
  }
}

// sums over tokens: dW_bar[j][k] = sum_t du[t][j] x[t][k],
// dW_s_up[i][k] = sum_t dhs[t][i] x[t][k], dW_s_down[n][i] = sum_t dy[t][n] SiLU(hs[t][i])
template <typename T>
__global__ void __launch_bounds__(kThreads) kb_sums(const Args a) {
  const size_t n_bar = (size_t)a.d_e * a.D, n_sup = (size_t)a.d_s * a.D, n_sdn = (size_t)a.D * a.d_s;
  const size_t total = n_bar + n_sup + n_sdn;
  for (size_t idx = (size_t)blockIdx.x * kThreads + threadIdx.x; idx < total; idx += (size_t)gridDim.x * kThreads) {
    float acc = 0.f;
    if (idx < n_bar) {
      const int j = (int)(idx / a.D), k = (int)(idx % a.D);
      for (int t = 0; t < a.T; ++t) acc = fmaf(a.du[(size_t)t * a.d_e + j], ldf<T>(a.x, (size_t)t * a.D + k), acc);
      a.dWbar[idx] = acc;
    } else if (idx < n_bar + n_sup) {
      const size_t o = idx - n_bar;
      const int i = (int)(o / a.D), k = (int)(o % a.D);
      for (int t = 0; t < a.T; ++t) acc = fmaf(a.dhs[(size_t)t * a.d_s + i], ldf<T>(a.x, (size_t)t * a.D + k), acc);
      a.dW_s_up[o] = acc;
    } else {
      const size_t o = idx - n_bar - n_sup;
      const int n = (int)(o / a.d_s), i = (int)(o % a.d_s);
      for (int t = 0; t < a.T; ++t) acc = fmaf(ldf<T>(a.dy, (size_t)t * a.D + n), a.as[(size_t)t * a.d_s + i], acc);
      a.dW_s_down[o] = acc;
    }
  }
}

// sums over each expert's pairs (token order): dW_up (+ dW_bar / E), dW_val,
// dW_down, dW_r, db_r, ds; blockIdx.y is the expert
template <typename T>
__global__ void __launch_bounds__(kThreads) kb_expert(const Args a) {
  const int e = blockIdx.y;
  const int p0 = a.offsets[e], p1 = a.offsets[e + 1];
  const size_t n_up = (size_t)a.d_e * a.D, n_val = a.gated ? n_up : 0, n_dn = (size_t)a.D * a.d_e;
  const size_t total = n_up + n_val + n_dn + a.D + 2;
  const float inv_E = 1.f / float(a.E);
  for (size_t idx = (size_t)blockIdx.x * kThreads + threadIdx.x; idx < total; idx += (size_t)gridDim.x * kThreads) {
    float acc = 0.f;
    if (idx < n_up + n_val) {
      const bool val = idx >= n_up;
      const size_t o = val ? idx - n_up : idx;
      const int j = (int)(o / a.D), k = (int)(o % a.D);
      const float* src = val ? a.pdq : a.pdc;
      for (int p = p0; p < p1; ++p)
        acc = fmaf(src[(size_t)p * a.d_e + j], ldf<T>(a.x, (size_t)a.perm[p] * a.D + k), acc);
      if (val) {
        a.dW_val[(size_t)e * n_up + o] = acc;
      } else {
        a.dW_up[(size_t)e * n_up + o] = fmaf(a.dWbar[o], inv_E, acc);
      }
    } else if (idx < n_up + n_val + n_dn) {
      const size_t o = idx - n_up - n_val;
      const int n = (int)(o / a.d_e), j = (int)(o % a.d_e);
      for (int p = p0; p < p1; ++p)
        acc = fmaf(a.pk[p] * ldf<T>(a.dy, (size_t)a.perm[p] * a.D + n), a.pa[(size_t)p * a.d_e + j], acc);
      a.dW_down[(size_t)e * n_dn + o] = acc;
    } else if (idx < n_up + n_val + n_dn + a.D) {
      const int k = (int)(idx - n_up - n_val - n_dn);
      for (int p = p0; p < p1; ++p) acc = fmaf(a.pz[p], ldf<T>(a.x, (size_t)a.perm[p] * a.D + k), acc);
      a.dW_r[(size_t)e * a.D + k] = acc;
    } else if (idx == n_up + n_val + n_dn + a.D) {
      for (int p = p0; p < p1; ++p) acc += a.pz[p];
      a.db_r[e] = acc;
    } else {
      for (int p = p0; p < p1; ++p) acc += a.pw[p];
      a.ds[e] = acc;
    }
  }
}

// Router entropy: per token (one warp) over its active experts, r = ReLU(z),
// R = sum r, p = r / R, H_t = -sum p log p (0 with none active), and
// dz[t][e] = lambda / T * dH_t/dr_e = -lambda (log p_e + H_t) / (R T) where
// active (0 elsewhere); Ht[t] = H_t.  Then kb_entropy_mean: Ht[T] = the mean,
// summed in token order.
__global__ void __launch_bounds__(kThreads) kb_entropy(const float* r, const uint8_t* act, int T, int E,
                                                       float lambda, float* Ht, float* dz) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * kWarps + warp;
  if (t >= T) return;
  float R = 0.f;
  for (int e = lane; e < E; e += 32)
    if (act[(size_t)t * E + e]) R += r[(size_t)t * E + e];
  R = warp_sum(R);
  float H = 0.f;
  if (R > 0.f)
    for (int e = lane; e < E; e += 32)
      if (act[(size_t)t * E + e]) {
        const float pe = r[(size_t)t * E + e] / R;
        H -= pe * logf(pe);
      }
  H = warp_sum(H);
  for (int e = lane; e < E; e += 32) {
    float d = 0.f;
    if (R > 0.f && act[(size_t)t * E + e]) {
      const float pe = r[(size_t)t * E + e] / R;
      d = -lambda * (logf(pe) + H) / (R * float(T));
    }
    dz[(size_t)t * E + e] = d;
  }
  if (lane == 0) Ht[t] = H;
}

__global__ void kb_entropy_mean(float* Ht, int T) {
  if (threadIdx.x != 0 || blockIdx.x != 0) return;
  float acc = 0.f;
  for (int t = 0; t < T; ++t) acc += Ht[t];
  Ht[T] = T > 0 ? acc / float(T) : 0.f;
}

}  // namespace bwd
}  // namespace deco
