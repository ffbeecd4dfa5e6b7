// Device helpers shared by the DECO MoE kernels (sm_100a).
#pragma once

#include <climits>

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace deco {

using bf16 = __nv_bfloat16;

constexpr unsigned kFull = 0xffffffffu;

// ---------------------------------------------------------------------------
// 16-byte vector loads, widened to fp32.  VecN<T>::N elements per 16 bytes.

template <typename T> struct VecN;
template <> struct VecN<float> { static constexpr int N = 4; };
template <> struct VecN<bf16> { static constexpr int N = 8; };

__device__ __forceinline__ void unpack16(const uint4& q, float (&v)[8]) {
  const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    v[2 * i] = __uint_as_float(w[i] << 16);
    v[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}
__device__ __forceinline__ void unpack16(const uint4& q, float (&v)[4]) {
  v[0] = __uint_as_float(q.x);
  v[1] = __uint_as_float(q.y);
  v[2] = __uint_as_float(q.z);
  v[3] = __uint_as_float(q.w);
}

// Streaming load of read-only weights: no L1 allocation.
__device__ __forceinline__ uint4 ld_stream16(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

template <typename T, int N>
__device__ __forceinline__ void load_w(const T* p, float (&v)[N]) {
  static_assert(N == VecN<T>::N, "vector width");
  unpack16(ld_stream16(p), v);
}
template <typename T, int N>
__device__ __forceinline__ void load_s(const T* p, float (&v)[N]) {
  static_assert(N == VecN<T>::N, "vector width");
  unpack16(*reinterpret_cast<const uint4*>(p), v);
}

__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(bf16 v) { return __bfloat162float(v); }

template <typename T> __device__ __forceinline__ T from_f32(float v);
template <> __device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ bf16 from_f32<bf16>(float v) { return __float2bfloat16_rn(v); }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
  return v;  // xor butterfly: every lane holds the identical total
}

// SiLU(h) = h * sigmoid(h) = h / (1 + exp(-h)); expf overflow gives -0 in the limit.
__device__ __forceinline__ float silu_f(float h) { return h / (1.0f + expf(-h)); }

// ---------------------------------------------------------------------------
// Exact sign of b + sum_k x_k w_k over fp32-representable operands.
//
// Every fp32 value is m * 2^e with an integer m < 2^24 and e >= -149, so every
// product x_k w_k is M * 2^f with M < 2^48 and f >= -298.  The sum is
// accumulated exactly in a fixed-point integer with its least significant bit
// at 2^-298, kept as kLimbs signed 64-bit limbs of 32 bits each (the spare
// 32 bits of every limb absorb carries).  Products of finite fp32 values
// reach at most 2^(208+48) and a sum of at most 2^16 of them 2^272, far below
// the top limb.  One warp evaluates one sum; limbs live in shared memory.

constexpr int kLimbs = 20;          // 640 bits with the LSB at 2^-298
constexpr int kLsbExp = -298;

struct FpParts {
  uint32_t m;   // integer significand (0 for zero)
  int e;        // exponent of the significand's LSB
  bool neg;
  bool finite;
};

__device__ __forceinline__ FpParts fp_parts(float f) {
  const uint32_t b = __float_as_uint(f);
  const uint32_t ef = (b >> 23) & 0xffu;
  const uint32_t frac = b & 0x7fffffu;
  FpParts p;
  p.neg = (b >> 31) != 0;
  p.finite = ef != 0xffu;
  if (ef == 0) {
    p.m = frac;
    p.e = -149;
  } else {
    p.m = frac | 0x800000u;
    p.e = int(ef) - 150;
  }
  return p;
}

__device__ __forceinline__ void limb_add(unsigned long long* limbs, int i, unsigned long long v,
                                         bool neg) {
  if (v) atomicAdd(&limbs[i], neg ? (0ull - v) : v);
}

// adds (-1)^neg * M * 2^(o + kLsbExp), M < 2^48, o >= 0
__device__ __forceinline__ void limbs_add_scaled(unsigned long long* limbs, unsigned long long M,
                                                 int o, bool neg) {
  const int i = o >> 5, sh = o & 31;
  const unsigned long long lo = M & 0xffffffffull, hi = M >> 32;
  const unsigned long long a = lo << sh;   // < 2^63
  const unsigned long long c = hi << sh;   // < 2^47
  limb_add(limbs, i, a & 0xffffffffull, neg);
  limb_add(limbs, i + 1, (a >> 32) + (c & 0xffffffffull), neg);
  limb_add(limbs, i + 2, c >> 32, neg);
}

// 8 consecutive elements (16-byte aligned) widened to fp32
__device__ __forceinline__ void load8(const bf16* p, float (&v)[8]) {
  unpack16(*reinterpret_cast<const uint4*>(p), v);
}
__device__ __forceinline__ void load8(const float* p, float (&v)[8]) {
  const float4 a = reinterpret_cast<const float4*>(p)[0], b = reinterpret_cast<const float4*>(p)[1];
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

// Exact sign (-1, 0, +1) of b + sum_{k<D} x[k] w[k] in the full fixed-point
// integer: the general routine, used when the register window below does not
// hold every product.  Called by all 32 lanes of one warp with the same
// arguments; `limbs` is this warp's kLimbs-entry shared buffer.
template <typename Tx, typename Tw>
__device__ int exact_sign_warp_limbs(const Tx* x, const Tw* w, int D, float b,
                                     unsigned long long* limbs) {
  const int lane = threadIdx.x & 31;
  for (int i = lane; i < kLimbs; i += 32) limbs[i] = 0ull;
  __syncwarp();
  for (int k = lane; k < D; k += 32) {
    const FpParts px = fp_parts(to_f32(x[k]));
    const FpParts pw = fp_parts(to_f32(w[k]));
    if (px.m && pw.m)
      limbs_add_scaled(limbs, (unsigned long long)px.m * pw.m, px.e + pw.e - kLsbExp,
                       px.neg != pw.neg);
  }
  if (lane == 0) {
    const FpParts pb = fp_parts(b);
    if (pb.m) limbs_add_scaled(limbs, pb.m, pb.e - kLsbExp, pb.neg);
  }
  __syncwarp();
  int sign = 0;
  if (lane == 0) {
    long long carry = 0;
    bool nz = false;
    for (int i = 0; i < kLimbs; ++i) {
      const long long v = (long long)limbs[i] + carry;
      nz |= (v & 0xffffffffll) != 0;
      carry = v >> 32;   // arithmetic shift: floor division by 2^32
    }
    sign = carry < 0 ? -1 : ((carry > 0 || nz) ? 1 : 0);
  }
  sign = __shfl_sync(kFull, sign, 0);
  __syncwarp();
  return sign;
}

// The same sum in a window of kWin 32-bit limbs held in registers.  The
// window's least significant bit sits at 2^base with base = f_max + 64 -
// 32 kWin, f_max the largest exponent (of the least significant bit) among
// the nonzero products and b: a product M 2^f with f >= base occupies bits
// [f - base, f - base + 47] <= 32 kWin - 17 of the window, and every lane's
// limb sums stay below 2^43 (at most D/32 + 1 terms below 2^33 each).  Each
// lane adds its products to its own limbs (no shared memory, no atomics),
// then the warp adds the limbs lane-wise and propagates carries.  A product
// below the window (f < base: more than 128 bits under the largest one) sends
// the sum to exact_sign_warp_limbs.
constexpr int kWin = 6;

__device__ __forceinline__ void win_add(long long (&L)[kWin], unsigned long long M, int o, bool neg) {
  const int i = o >> 5, sh = o & 31;
  const unsigned long long lo = M & 0xffffffffull, hi = M >> 32;
  const unsigned long long a = lo << sh;   // < 2^63
  const unsigned long long c = hi << sh;   // < 2^47
  long long c0 = (long long)(a & 0xffffffffull);
  long long c1 = (long long)((a >> 32) + (c & 0xffffffffull));
  long long c2 = (long long)(c >> 32);
  if (neg) {
    c0 = -c0;
    c1 = -c1;
    c2 = -c2;
  }
#pragma unroll
  for (int j = 0; j < kWin; ++j) L[j] += j == i ? c0 : (j == i + 1 ? c1 : (j == i + 2 ? c2 : 0ll));
}

// Exact sign (-1, 0, +1) of b + sum_{k<D} x[k] w[k]; called by all 32 lanes of
// one warp with the same arguments.  `limbs` is this warp's kLimbs-entry
// shared buffer (used only by the general routine).  Sets *nonfinite if an
// operand is Inf/NaN (the result is then 0).
template <typename Tx, typename Tw>
__device__ int exact_sign_warp(const Tx* x, const Tw* w, int D, float b,
                               unsigned long long* limbs, bool* nonfinite) {
  const int lane = threadIdx.x & 31;
  // pass 1: finiteness and the largest exponent (8 elements per lane per
  // step, loaded as 16-byte vectors: D is a multiple of 64, rows 16-B aligned)
  bool bad = false;
  int fmax = INT_MIN;
#pragma unroll 2
  for (int k0 = lane * 8; k0 < D; k0 += 256) {
    float xv[8], wv[8];
    load8(x + k0, xv);
    load8(w + k0, wv);
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const FpParts px = fp_parts(xv[q]);
      const FpParts pw = fp_parts(wv[q]);
      bad |= !(px.finite && pw.finite);
      if (px.m && pw.m) fmax = max(fmax, px.e + pw.e);
    }
  }
  const FpParts pb = fp_parts(b);
  bad |= !pb.finite;
  if (pb.m) fmax = max(fmax, pb.e);
  bad = __any_sync(kFull, bad);
  fmax = __reduce_max_sync(kFull, fmax);
  if (bad) {
    *nonfinite = true;
    return 0;
  }
  if (fmax == INT_MIN) return 0;   // every product and b are zero
  // pass 2: the window
  const int base = fmax + 64 - 32 * kWin;
  long long L[kWin];
#pragma unroll
  for (int j = 0; j < kWin; ++j) L[j] = 0;
  bool below = false;
  for (int k0 = lane * 8; k0 < D; k0 += 256) {
    float xv[8], wv[8];
    load8(x + k0, xv);
    load8(w + k0, wv);
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const FpParts px = fp_parts(xv[q]);
      const FpParts pw = fp_parts(wv[q]);
      if (px.m && pw.m) {
        const int o = px.e + pw.e - base;
        if (o < 0) below = true;
        else win_add(L, (unsigned long long)px.m * pw.m, o, px.neg != pw.neg);
      }
    }
  }
  if (lane == 0 && pb.m) {
    const int o = pb.e - base;
    if (o < 0) below = true;
    else win_add(L, pb.m, o, pb.neg);
  }
  if (__any_sync(kFull, below)) return exact_sign_warp_limbs(x, w, D, b, limbs);
#pragma unroll
  for (int j = 0; j < kWin; ++j) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) L[j] += __shfl_xor_sync(kFull, L[j], o);
  }
  long long carry = 0;
  bool nz = false;
#pragma unroll
  for (int j = 0; j < kWin; ++j) {
    const long long v = L[j] + carry;
    nz |= (v & 0xffffffffll) != 0;
    carry = v >> 32;   // arithmetic shift: floor division by 2^32
  }
  return carry < 0 ? -1 : ((carry > 0 || nz) ? 1 : 0);
}

// Exact sign (-1, 0, +1) of (b1 + sum_k x[k] w1[k]) - (b2 + sum_k x[k] w2[k]):
// the exact comparison of two logits of one token (TopK ranking).  The same
// integer accumulation as exact_sign_warp, with the second row's products and
// bias entering negated: a window of kWin limbs in registers anchored at the
// largest product, and the 640-bit fixed point in shared memory when a
// product lies below the window.  Called by all 32 lanes of one warp.
template <typename Tx, typename Tw>
__device__ int exact_cmp_warp_limbs(const Tx* x, const Tw* w1, const Tw* w2, int D, float b1, float b2,
                                    unsigned long long* limbs) {
  const int lane = threadIdx.x & 31;
  for (int i = lane; i < kLimbs; i += 32) limbs[i] = 0ull;
  __syncwarp();
  for (int k = lane; k < D; k += 32) {
    const FpParts px = fp_parts(to_f32(x[k]));
    const FpParts p1 = fp_parts(to_f32(w1[k]));
    const FpParts p2 = fp_parts(to_f32(w2[k]));
    if (px.m && p1.m)
      limbs_add_scaled(limbs, (unsigned long long)px.m * p1.m, px.e + p1.e - kLsbExp, px.neg != p1.neg);
    if (px.m && p2.m)
      limbs_add_scaled(limbs, (unsigned long long)px.m * p2.m, px.e + p2.e - kLsbExp, px.neg == p2.neg);
  }
  if (lane == 0) {
    const FpParts q1 = fp_parts(b1), q2 = fp_parts(b2);
    if (q1.m) limbs_add_scaled(limbs, q1.m, q1.e - kLsbExp, q1.neg);
    if (q2.m) limbs_add_scaled(limbs, q2.m, q2.e - kLsbExp, !q2.neg);
  }
  __syncwarp();
  int sign = 0;
  if (lane == 0) {
    long long carry = 0;
    bool nz = false;
    for (int i = 0; i < kLimbs; ++i) {
      const long long v = (long long)limbs[i] + carry;
      nz |= (v & 0xffffffffll) != 0;
      carry = v >> 32;
    }
    sign = carry < 0 ? -1 : ((carry > 0 || nz) ? 1 : 0);
  }
  sign = __shfl_sync(kFull, sign, 0);
  __syncwarp();
  return sign;
}

template <typename Tx, typename Tw>
__device__ int exact_cmp_warp(const Tx* x, const Tw* w1, const Tw* w2, int D, float b1, float b2,
                              unsigned long long* limbs, bool* nonfinite) {
  const int lane = threadIdx.x & 31;
  bool bad = false;
  int fmax = INT_MIN;
  for (int k0 = lane * 8; k0 < D; k0 += 256) {
    float xv[8], v1[8], v2[8];
    load8(x + k0, xv);
    load8(w1 + k0, v1);
    load8(w2 + k0, v2);
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const FpParts px = fp_parts(xv[q]), p1 = fp_parts(v1[q]), p2 = fp_parts(v2[q]);
      bad |= !(px.finite && p1.finite && p2.finite);
      if (px.m && p1.m) fmax = max(fmax, px.e + p1.e);
      if (px.m && p2.m) fmax = max(fmax, px.e + p2.e);
    }
  }
  const FpParts q1 = fp_parts(b1), q2 = fp_parts(b2);
  bad |= !(q1.finite && q2.finite);
  if (q1.m) fmax = max(fmax, q1.e);
  if (q2.m) fmax = max(fmax, q2.e);
  bad = __any_sync(kFull, bad);
  fmax = __reduce_max_sync(kFull, fmax);
  if (bad) {
    *nonfinite = true;
    return 0;
  }
  if (fmax == INT_MIN) return 0;
  const int base = fmax + 64 - 32 * kWin;
  long long L[kWin];
#pragma unroll
  for (int j = 0; j < kWin; ++j) L[j] = 0;
  bool below = false;
  for (int k0 = lane * 8; k0 < D; k0 += 256) {
    float xv[8], v1[8], v2[8];
    load8(x + k0, xv);
    load8(w1 + k0, v1);
    load8(w2 + k0, v2);
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const FpParts px = fp_parts(xv[q]), p1 = fp_parts(v1[q]), p2 = fp_parts(v2[q]);
      if (px.m && p1.m) {
        const int o = px.e + p1.e - base;
        if (o < 0) below = true;
        else win_add(L, (unsigned long long)px.m * p1.m, o, px.neg != p1.neg);
      }
      if (px.m && p2.m) {
        const int o = px.e + p2.e - base;
        if (o < 0) below = true;
        else win_add(L, (unsigned long long)px.m * p2.m, o, px.neg == p2.neg);
      }
    }
  }
  if (lane == 0) {
    if (q1.m) {
      const int o = q1.e - base;
      if (o < 0) below = true;
      else win_add(L, q1.m, o, q1.neg);
    }
    if (q2.m) {
      const int o = q2.e - base;
      if (o < 0) below = true;
      else win_add(L, q2.m, o, !q2.neg);
    }
  }
  if (__any_sync(kFull, below)) return exact_cmp_warp_limbs(x, w1, w2, D, b1, b2, limbs);
#pragma unroll
  for (int j = 0; j < kWin; ++j) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) L[j] += __shfl_xor_sync(kFull, L[j], o);
  }
  long long carry = 0;
  bool nz = false;
#pragma unroll
  for (int j = 0; j < kWin; ++j) {
    const long long v = L[j] + carry;
    nz |= (v & 0xffffffffll) != 0;
    carry = v >> 32;
  }
  return carry < 0 ? -1 : ((carry > 0 || nz) ? 1 : 0);
}

// gamma_n = n u / (1 - n u) with u = 2^-24: the classical bound on the
// relative error of an n-step fp32 recursive (FMA) summation.
__device__ __forceinline__ float gamma_f32(int n) {
  const double nu = double(n) * 5.9604644775390625e-8;
  return float(nu / (1.0 - nu));
}

}  // namespace deco
