// Host side of the C ABI declared in include/deco_moe.h: argument checks,
// workspace plan and the launch sequence.  No allocation, no synchronisation
// (except deco_moe_device_error), so every call can be graph-captured.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <mutex>

#include "../../include/deco_moe.h"
#include "simt_kernels.cuh"
#include "backward_kernels.cuh"
#include "decode_kernels.cuh"
#include "prefill_kernels.cuh"

namespace deco {
namespace {

inline size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

// Workspace layout of one forward / routing call.
struct Plan {
  size_t err, err_bytes, r, act, u, hs, counts, offsets, n_tok, perm, pair_of, tiles, n_tiles, H, total;
  // decode path (T <= 16): up-projection partials, shared hidden and NormSiLU
  // tiles, per-CTA down-projection partials (the inter-CTA counters follow
  // the error word)
  size_t Pu, HS, A16, Part, tmask;
  // bf16, T > 16: ambiguous router pairs; prefill path: routed expert output
  // rows (one fp16 row per pair) and the shared expert's fp32 output
  size_t fb, blk, etot, v_pairs, coef, s_out, val_pairs;
  // TopK routing: fp32 logits and their error bounds
  size_t zt, bt;
  int tile_rows;
  int sms;
};

inline size_t elem_size(int dtype) { return dtype == DECO_F32 ? 4 : 2; }

int num_sms() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n;
}

// rows of x staged per CTA: 16 when the tile fits in 128 KB of shared memory
inline int token_tile(int D, int dtype) { return (16 * (size_t)D * elem_size(dtype) <= 131072) ? 16 : 8; }

// The tcgen05 prefill kernels (prefill_kernels.cuh) take bf16 batches of more
// than 16 tokens whose routed experts fit one 256-column accumulator.
bool prefill_eligible(const deco_moe_shape_t& s) {
  return s.dtype == DECO_BF16 && s.T > dec::kMaxT && s.d_e <= pf::kBN && !s.experts_on_host;
}

// bf16 batches of more than 16 tokens are routed by the tiled router
// (prefill_kernels.cuh), whatever path computes the experts
bool tiled_router(const deco_moe_shape_t& s) { return s.dtype == DECO_BF16 && s.T > dec::kMaxT; }

Plan make_plan(const deco_moe_shape_t& s) {
  Plan p{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align256(off + bytes);
    return o;
  };
  const size_t T = s.T, E = s.E, P = T * E;
  p.tile_rows = token_tile(s.d_model, s.dtype);
  p.sms = num_sms();
  // error word (+ the prefill router's ambiguous-pair count), then the decode
  // kernel's counters; all cleared by every call
  p.err_bytes = 16;
  if (s.T <= dec::kMaxT) p.err_bytes += 4 * (size_t)dec::sync_idx(s.E, s.d_model).total;
  p.err = take(p.err_bytes);
  p.r = take(T * E * 4);
  p.act = take(T * E);
  p.u = take(T * s.d_e * 4);
  p.hs = take(T * s.d_s * 4);
  p.counts = take(E * 4);
  p.offsets = take((E + 1) * 4);
  p.n_tok = take(T * 4);
  p.perm = take(P * 4);
  p.pair_of = take(P * 4);
  p.tiles = take((P / p.tile_rows + E) * 16);
  p.n_tiles = take(4);
  p.H = take(P * s.d_e * 4);       // NormSiLU activations (fp32; bf16 on the prefill path)
  if (tiled_router(s)) {
    p.fb = take(P * 8);
    p.blk = take((size_t)((s.T + pf::kTabUnit - 1) / pf::kTabUnit) * E * 4);   // [units of 32 tokens][E]
    p.etot = take(E * 4);
  }
  if (s.topk > 0) {
    p.zt = take(P * 4);
    p.bt = take(P * 4);
  }
  if (prefill_eligible(s)) {
    p.v_pairs = take(P * s.d_model * 2);
    p.coef = take(P * 4);
    if (s.gated) p.val_pairs = take(P * s.d_e * 2);   // bf16 value-branch rows per pair
    p.s_out = take(T * s.d_model * 4);
  }
  if (s.T <= dec::kMaxT) {         // decode path buffers (see decode_kernels.cuh)
    const size_t runs = E * (s.gated ? 2 : 1) * ((s.d_e + dec::kDRows - 1) / dec::kDRows);
    p.Pu = take((runs + std::max(p.sms, 1)) * dec::kTok * dec::kDRows * 4);   // phase-U pieces, fp32
    p.HS = take((size_t)dec::down_nsq(s.d_s) * dec::kTileBytes);       // [nsq] 16 KB tiles
    p.A16 = take(E * dec::kTileBytes);                                 // [E] 16 KB tiles
    p.Part = take((size_t)std::max(p.sms, 1) * 2 * dec::kTok * dec::kDRows * 4);   // [G][2][16][128]
    p.tmask = take(E * 4);                                             // [E] token masks
  }
  p.total = off;
  return p;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

deco_status_t check_shape(const deco_moe_shape_t* s) {
  if (!s) return DECO_ERR_INVALID_ARG;
  if (s->T < 0 || s->d_model <= 0 || s->E <= 0 || s->d_e <= 0 || s->d_s <= 0)
    return DECO_ERR_INVALID_ARG;
  if (s->dtype != DECO_F32 && s->dtype != DECO_BF16) return DECO_ERR_INVALID_ARG;
  if (!(s->rms_eps >= 0.f) || !std::isfinite(s->rms_eps)) return DECO_ERR_INVALID_ARG;
  if (s->residual != 0 && s->residual != 1) return DECO_ERR_INVALID_ARG;
  if (s->topk < 0 || s->topk > s->E) return DECO_ERR_INVALID_ARG;
  if (s->gated != 0 && s->gated != 1) return DECO_ERR_INVALID_ARG;
  if (s->experts_on_host != 0 && s->experts_on_host != 1) return DECO_ERR_INVALID_ARG;
  if (s->d_model % 64 || s->d_model > 16384) return DECO_ERR_UNSUPPORTED;
  if (s->E > 256) return DECO_ERR_UNSUPPORTED;
  if (s->d_e % 64 || s->d_e > 512) return DECO_ERR_UNSUPPORTED;
  if (s->d_s % 64 || s->d_s > 16384) return DECO_ERR_UNSUPPORTED;
  if (s->T > (1 << 20)) return DECO_ERR_UNSUPPORTED;
  return DECO_OK;
}

// host memory the device reads through its own address space: pinned and
// mapped, with unified addressing (the device pointer is the host pointer)
bool host_mapped(const void* p) {
  cudaPointerAttributes at{};
  if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  return at.type == cudaMemoryTypeHost && at.devicePointer == p;
}

deco_status_t check_weights(const deco_moe_weights_t* w, bool router_only, bool gated = false,
                            bool experts_on_host = false) {
  if (!w || !w->W_r || !w->b_r) return DECO_ERR_INVALID_ARG;
  if (!aligned16(w->W_r)) return DECO_ERR_INVALID_ARG;
  if (router_only) return DECO_OK;
  if (gated && (!w->W_val || !aligned16(w->W_val))) return DECO_ERR_INVALID_ARG;
  const void* ps[] = {w->W_up, w->W_bar_up, w->W_down, w->s, w->W_s_up, w->W_s_down};
  for (const void* p : ps)
    if (!p || !aligned16(p)) return DECO_ERR_INVALID_ARG;
  if (experts_on_host &&
      (!host_mapped(w->W_up) || !host_mapped(w->W_down) || (gated && !host_mapped(w->W_val))))
    return DECO_ERR_INVALID_ARG;
  return DECO_OK;
}

// Opt every kernel into the dynamic shared memory it may use (once per device).
template <typename K>
cudaError_t allow_smem(K kernel, size_t bytes) {
  if (bytes <= 48 * 1024) return cudaSuccess;
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

thread_local char g_cuda_msg[256] = "";

// maps a CUDA error to DECO_ERR_CUDA and remembers its text for deco_last_cuda_error
deco_status_t cuda_status(cudaError_t e, const char* where) {
  if (e == cudaSuccess) return DECO_OK;
  snprintf(g_cuda_msg, sizeof(g_cuda_msg), "%s: %s (%s)", where, cudaGetErrorName(e),
           cudaGetErrorString(e));
  return DECO_ERR_CUDA;
}

// benchmark timing hook (deco_moe_set_profiling)
cudaEvent_t const* g_prof_events = nullptr;
int g_prof_n = 0;

inline void prof_mark(int idx, cudaStream_t st) {
  if (!g_prof_events || idx >= g_prof_n) return;
  // while the stream is being graph-captured the record must be external to
  // become an event-record node; outside a capture that flag is illegal
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  cudaStreamIsCapturing(st, &cs);
  if (cs == cudaStreamCaptureStatusActive)
    cudaEventRecordWithFlags(g_prof_events[idx], st, cudaEventRecordExternal);
  else
    cudaEventRecord(g_prof_events[idx], st);
}

// The decode kernel (decode_kernels.cuh) takes bf16 batches of up to 16 tokens
// with d_model a multiple of 256 up to 4096 and d_e <= 256, on GPUs of at most
// dec::kMaxSms SMs whose router CTAs leave room for the other phase-R rows.
bool decode_grid_ok(int D, int E, int sms) {
  if (D % 256 || D > 4096 || sms > dec::kMaxSms) return false;
  if (D / dec::kDRows > sms) return false;   // a CTA's share of phase-D units spans <= 2 row blocks
  if (dec::router_ctas(E) + 16 > sms) return false;
  return dec::layer_smem(D).nstages >= 2;
}

bool decode_eligible(const deco_moe_shape_t& s, int sms) {
  if (s.dtype != DECO_BF16 || s.T < 1 || s.T > dec::kMaxT || s.experts_on_host) return false;
  if (s.E > 256 || s.d_e > 256 || s.d_e % 64 || s.d_s % 64) return false;
  return decode_grid_ok(s.d_model, s.E, sms);
}

// limit of the kernels' waits for data (deco_set_wait_limit; the drains of
// copies already issued keep the default)
long long g_wait_cycles = dec::kWaitCycles;

// ---------------------------------------------------------------------------
template <typename T, int TT>
cudaError_t launch_route(const RouteArgs& a, cudaStream_t st) {
  if (a.T == 0) return cudaSuccess;
  const size_t smem = (size_t)TT * a.D * sizeof(T) + kWarps * kLimbs * sizeof(unsigned long long);
  cudaError_t err = allow_smem(k_route<T, TT>, smem);
  if (err != cudaSuccess) return err;
  const int R = a.E + a.d_e + a.d_s;
  dim3 grid((R + kWarps - 1) / kWarps, (a.T + TT - 1) / TT);
  k_route<T, TT><<<grid, kThreads, smem, st>>>(a);
  return cudaGetLastError();
}

template <typename T>
cudaError_t route_any(const RouteArgs& a, int tt, cudaStream_t st) {
  return tt == 16 ? launch_route<T, 16>(a, st) : launch_route<T, 8>(a, st);
}

template <typename T, int TT>
cudaError_t launch_up(const UpArgs& a, int max_tiles, cudaStream_t st) {
  const size_t smem = (size_t)TT * a.D * sizeof(T) + (a.W_val ? 2 : 1) * (size_t)TT * (a.d_e / kCluster) * sizeof(float);
  cudaError_t err = allow_smem(k_up<T, TT>, smem);
  if (err != cudaSuccess) return err;
  int clusters = std::min(max_tiles, std::max(1, 2 * num_sms() / kCluster));
  k_up<T, TT><<<clusters * kCluster, kThreads, smem, st>>>(a);
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_down(const DownArgs& a, cudaStream_t st) {
  if (a.T == 0) return cudaSuccess;
  constexpr int TT = 16, RPW = 2;
  const size_t smem = sizeof(float) * TT * kDownK + sizeof(uint32_t) * (size_t)std::max(a.E, 1);
  cudaError_t err = allow_smem(k_down<T, TT, RPW>, smem);
  if (err != cudaSuccess) return err;
  dim3 grid(a.D / (kWarps * RPW), (a.T + TT - 1) / TT);
  k_down<T, TT, RPW><<<grid, kThreads, smem, st>>>(a);
  return cudaGetLastError();
}

// router + tables (shared by forward and routing)
template <typename T>
cudaError_t run_routing(const deco_moe_shape_t& s, const void* x, const deco_moe_weights_t& w,
                        unsigned char* ws, const Plan& p, bool with_mean_shared, float* r,
                        uint8_t* act, int* counts, int* offsets, int* perm, int* n_tok,
                        cudaStream_t st, int tile_rows, bool decide_only = false) {
  RouteArgs ra{};
  ra.x = x;
  ra.T = s.T;
  ra.D = s.d_model;
  ra.W_r = w.W_r;
  ra.b_r = w.b_r;
  ra.E = s.E;
  ra.W_bar = w.W_bar_up;
  ra.d_e = with_mean_shared ? s.d_e : 0;
  ra.W_s_up = w.W_s_up;
  ra.d_s = with_mean_shared ? s.d_s : 0;
  ra.r = r;
  ra.act = act;
  ra.u = reinterpret_cast<float*>(ws + p.u);
  ra.hs = reinterpret_cast<float*>(ws + p.hs);
  ra.err = reinterpret_cast<int*>(ws + p.err);
  prof_mark(0, st);
  cudaError_t err;
  if (s.topk > 0) {
    // TopK: logits and bounds from the general router, then the exact selection
    ra.zt = reinterpret_cast<float*>(ws + p.zt);
    ra.bt = reinterpret_cast<float*>(ws + p.bt);
    if ((err = route_any<T>(ra, token_tile(s.d_model, s.dtype), st)) != cudaSuccess) return err;
    TopkArgs ta{};
    ta.x = x;
    ta.W_r = w.W_r;
    ta.b_r = w.b_r;
    ta.T = s.T;
    ta.D = s.d_model;
    ta.E = s.E;
    ta.k = s.topk;
    ta.zt = ra.zt;
    ta.bt = ra.bt;
    ta.r = r;
    ta.act = act;
    ta.err = ra.err;
    k_topk_select<T><<<(s.T + kTopkWarps - 1) / kTopkWarps, kTopkWarps * 32, 0, st>>>(ta);
  } else if (!with_mean_shared && s.dtype == DECO_BF16 && decode_eligible(s, p.sms)) {
    // the decode forward's own router: kd_layer's router CTAs alone (the
    // same per-row code and order, so the same decisions bit for bit)
    dec::Args da{};
    da.T = s.T;
    da.D = s.d_model;
    da.E = s.E;
    da.wait_cycles = g_wait_cycles;
    da.x = static_cast<const bf16*>(x);
    da.W_r = static_cast<const bf16*>(w.W_r);
    da.b_r = w.b_r;
    da.r = r;
    da.act = act;
    da.tmask = reinterpret_cast<unsigned*>(ws + p.tmask);
    da.err = reinterpret_cast<int*>(ws + p.err);
    const uint32_t smem = dec::layer_smem(s.d_model).total;
    if ((err = allow_smem(dec::kd_router, smem)) != cudaSuccess) return err;
    dec::kd_router<<<dec::router_ctas(s.E), dec::kThreads, smem, st>>>(da);
  } else if (!with_mean_shared && tiled_router(s)) {
    pf::RouterArgs rt{};
    rt.x = static_cast<const bf16*>(x);
    rt.W_r = static_cast<const bf16*>(w.W_r);
    rt.b_r = w.b_r;
    rt.T = s.T;
    rt.D = s.d_model;
    rt.E = s.E;
    rt.r = r;
    rt.act = act;
    rt.fb = reinterpret_cast<int2*>(ws + p.fb);
    rt.n_fb = reinterpret_cast<int*>(ws + p.err) + 1;   // zeroed with the error word
    rt.err = reinterpret_cast<int*>(ws + p.err);
    if ((err = allow_smem(pf::k_router, pf::kRouterSmem)) != cudaSuccess) return err;
    pf::k_router<<<dim3((s.T + pf::kRT - 1) / pf::kRT, (s.E + pf::kRE - 1) / pf::kRE), pf::kRThreads,
                   pf::kRouterSmem, st>>>(rt);
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
    pf::k_router_exact<<<p.sms, 256, 0, st>>>(rt);
  } else {
    err = route_any<T>(ra, token_tile(s.d_model, s.dtype), st);
  }
  if ((err = cudaGetLastError()) != cudaSuccess) return err;
  prof_mark(1, st);
  if (decide_only) return cudaSuccess;
  if (!with_mean_shared && tiled_router(s)) {   // token-block tables
    const int nu = (s.T + pf::kTabUnit - 1) / pf::kTabUnit;   // units of 32 tokens, one warp each
    const int nb = (nu + pf::kTabWarps - 1) / pf::kTabWarps;
    int* blk = reinterpret_cast<int*>(ws + p.blk);
    prof_mark(2, st);
    pf::k_tab_count<<<nb, pf::kTabThreads, 0, st>>>(act, s.T, s.E, n_tok, blk);
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
    int* etot = reinterpret_cast<int*>(ws + p.etot);
    pf::k_tab_scan<<<(s.E + pf::kTabWarps - 1) / pf::kTabWarps, pf::kTabThreads, 0, st>>>(s.E, nu, blk, etot);
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
    prof_mark(3, st);
    prof_mark(4, st);
    pf::k_tab_scatter<<<nb, pf::kTabThreads, 0, st>>>(act, s.T, s.E, blk, etot, counts, offsets, perm,
                                                      reinterpret_cast<int*>(ws + p.pair_of),
                                                      reinterpret_cast<int4*>(ws + p.tiles),
                                                      reinterpret_cast<int*>(ws + p.n_tiles), tile_rows);
    prof_mark(5, st);
    return cudaGetLastError();
  }
  prof_mark(2, st);
  k_count<<<s.E + (s.T + kThreads - 1) / kThreads, kThreads, 0, st>>>(act, s.T, s.E, counts, n_tok);
  if ((err = cudaGetLastError()) != cudaSuccess) return err;
  prof_mark(3, st);
  prof_mark(4, st);
  k_scatter<<<s.E, kThreads, 0, st>>>(act, s.T, s.E, counts, offsets, perm,
                                       reinterpret_cast<int*>(ws + p.pair_of),
                                       reinterpret_cast<int4*>(ws + p.tiles),
                                       reinterpret_cast<int*>(ws + p.n_tiles), tile_rows);
  prof_mark(5, st);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// decode path: bf16, T <= 16 (weight-streaming kernels, see decode_kernels.cuh)

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* q = nullptr;
    cudaDriverEntryPointQueryResult res;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &q, 12000, cudaEnableDefault, &res) ==
            cudaSuccess &&
        res == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(q);
  });
  return fn;
}

// Tensor map over a row-major matrix [rows][cols] of 2- or 4-byte elements:
// boxes of 128 B of columns (one swizzle atom) x box_rows rows, 128-byte
// swizzle; loads read zeros past the ends, stores are clipped there.
cudaError_t make_map(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, uint32_t box_rows,
                     CUtensorMapDataType type = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16) {
  PFN_cuTensorMapEncodeTiled_v12000 fn = encode_fn();
  if (!fn) return cudaErrorNotSupported;
  const uint64_t esz = type == CU_TENSOR_MAP_DATA_TYPE_FLOAT32 ? 4 : 2;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * esz};
  const cuuint32_t box[2] = {(cuuint32_t)(128 / esz), box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(m, type, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// one CTA per SM, all resident at once (the CTAs wait on one another's
// counters), so the launch is cooperative
cudaError_t launch_layer(const CUtensorMap& tmU, const CUtensorMap& tmV, const CUtensorMap& tmW,
                         const CUtensorMap& tmS, const dec::Args& a, int sms, cudaStream_t st) {
  const uint32_t smem = dec::layer_smem(a.D).total;
  cudaError_t err = cudaFuncSetAttribute(dec::kd_layer, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(sms);
  cfg.blockDim = dim3(dec::kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, dec::kd_layer, tmU, tmV, tmW, tmS, a);
}

// the decode kernel's buffers in a workspace laid out by make_plan
void decode_buffers(dec::Args& a, unsigned char* ws, const Plan& p) {
  a.wait_cycles = g_wait_cycles;
  a.r = reinterpret_cast<float*>(ws + p.r);
  a.act = reinterpret_cast<uint8_t*>(ws + p.act);
  a.tmask = reinterpret_cast<unsigned*>(ws + p.tmask);
  a.u = reinterpret_cast<float*>(ws + p.u);
  a.HS = reinterpret_cast<bf16*>(ws + p.HS);
  a.A = reinterpret_cast<bf16*>(ws + p.A16);
  a.Pu = reinterpret_cast<float*>(ws + p.Pu);
  a.Part = reinterpret_cast<float*>(ws + p.Part);
  a.err = reinterpret_cast<int*>(ws + p.err);
  a.sync = reinterpret_cast<unsigned*>(ws + p.err + 16);
}

cudaError_t run_decode(const deco_moe_shape_t& s, const void* x, const deco_moe_weights_t& w,
                       void* out, unsigned char* ws, const Plan& p, cudaStream_t st) {
  dec::Args a{};
  a.T = s.T;
  a.D = s.d_model;
  a.E = s.E;
  a.d_e = s.d_e;
  a.d_s = s.d_s;
  a.eps = s.rms_eps;
  a.residual = s.residual;
  a.x = static_cast<const bf16*>(x);
  a.W_r = static_cast<const bf16*>(w.W_r);
  a.b_r = w.b_r;
  a.W_bar = static_cast<const bf16*>(w.W_bar_up);
  a.W_up = static_cast<const bf16*>(w.W_up);
  a.W_down = static_cast<const bf16*>(w.W_down);
  a.s = w.s;
  a.W_s_up = static_cast<const bf16*>(w.W_s_up);
  a.W_s_down = static_cast<const bf16*>(w.W_s_down);
  a.out = static_cast<bf16*>(out);
  a.pre_routed = s.topk > 0;
  a.gated = s.gated;
  decode_buffers(a, ws, p);
  // weight tiles of phases U and D: 128 rows x 64 columns
  CUtensorMap tmU, tmV, tmW, tmS;
  cudaError_t err;
  if ((err = make_map(&tmV, s.gated ? w.W_val : w.W_up, s.d_model, (uint64_t)s.E * s.d_e, dec::kDRows)) !=
          cudaSuccess ||
      (err = make_map(&tmU, w.W_up, s.d_model, (uint64_t)s.E * s.d_e, dec::kDRows)) != cudaSuccess ||
      (err = make_map(&tmW, w.W_down, s.d_e, (uint64_t)s.E * s.d_model, dec::kDRows)) != cudaSuccess ||
      (err = make_map(&tmS, w.W_s_down, s.d_s, s.d_model, dec::kDRows)) != cudaSuccess)
    return err;
  prof_mark(16, st);
  err = launch_layer(tmU, tmV, tmW, tmS, a, p.sms, st);
  prof_mark(17, st);
  return err;
}

// dense FFN y = W2 SiLU(W1 x) at decode batch sizes: the same kernel with no
// routed experts (W1 streams as phase-R rows, W2 as phase-D units)
size_t dense_decode_bytes(int D, int d_ff, int sms) {
  return 16 + 4 * (size_t)dec::sync_idx(0, D).total + (size_t)dec::down_nsq(d_ff) * dec::kTileBytes +
         (size_t)sms * 2 * dec::kTok * dec::kDRows * 4 + 3 * 256;
}

cudaError_t run_dense_decode(int T, int D, int d_ff, const void* x, const void* W1, const void* W2, void* out,
                             unsigned char* ws, int sms, cudaStream_t st) {
  dec::Args a{};
  a.T = T;
  a.D = D;
  a.E = 0;
  a.d_e = 0;
  a.d_s = d_ff;
  a.wait_cycles = g_wait_cycles;
  a.x = static_cast<const bf16*>(x);
  a.W_s_up = static_cast<const bf16*>(W1);
  a.W_s_down = static_cast<const bf16*>(W2);
  a.out = static_cast<bf16*>(out);
  const size_t sync_bytes = 16 + 4 * (size_t)dec::sync_idx(0, D).total;
  a.err = reinterpret_cast<int*>(ws);
  a.sync = reinterpret_cast<unsigned*>(ws + 16);
  const size_t hs_off = align256(sync_bytes);
  a.HS = reinterpret_cast<bf16*>(ws + hs_off);
  a.Part = reinterpret_cast<float*>(ws + align256(hs_off + (size_t)dec::down_nsq(d_ff) * dec::kTileBytes));
  cudaError_t err;
  CUtensorMap tmS;
  if ((err = make_map(&tmS, W2, d_ff, D, dec::kDRows)) != cudaSuccess) return err;
  return launch_layer(tmS, tmS, tmS, tmS, a, sms, st);   // no routed experts: the other maps are unused
}

// ---------------------------------------------------------------------------
// prefill path: bf16, T > 16 (tcgen05 GEMMs, see prefill_kernels.cuh)

template <int MODE>
cudaError_t launch_pf(const CUtensorMap& A, const CUtensorMap& B, const CUtensorMap& B2, const CUtensorMap& O,
                      const CUtensorMap& O2, const pf::Args& a, int grid, cudaStream_t st) {
  if (grid <= 0) return cudaSuccess;
  cudaError_t err = allow_smem(pf::kp_gemm<MODE>, pf::kSmemBytes);
  if (err != cudaSuccess) return err;
  pf::kp_gemm<MODE><<<grid, pf::kThreads, pf::kSmemBytes, st>>>(A, B, B2, O, O2, a);
  return cudaGetLastError();
}

inline int cdiv(int a, int b) { return (a + b - 1) / b; }

cudaError_t run_prefill(const deco_moe_shape_t& s, const void* x, const deco_moe_weights_t& w, void* out,
                        unsigned char* ws, const Plan& p, cudaStream_t st) {
  float* r = reinterpret_cast<float*>(ws + p.r);
  uint8_t* act = reinterpret_cast<uint8_t*>(ws + p.act);
  cudaError_t err = run_routing<bf16>(s, x, w, ws, p, false, r, act, reinterpret_cast<int*>(ws + p.counts),
                                      reinterpret_cast<int*>(ws + p.offsets), reinterpret_cast<int*>(ws + p.perm),
                                      reinterpret_cast<int*>(ws + p.n_tok), st, pf::kBM);
  if (err != cudaSuccess) return err;
  const int T = s.T, D = s.d_model, E = s.E, d_e = s.d_e, d_s = s.d_s;
  const uint64_t P = (uint64_t)T * E;
  pf::Args a{};
  a.wait_cycles = g_wait_cycles;
  a.T = T;
  a.D = D;
  a.E = E;
  a.d_e = d_e;
  a.d_s = d_s;
  a.eps = s.rms_eps;
  a.residual = s.residual;
  a.tiles = reinterpret_cast<const int4*>(ws + p.tiles);
  a.n_row_tiles = reinterpret_cast<const int*>(ws + p.n_tiles);
  a.x = static_cast<const bf16*>(x);
  a.perm = reinterpret_cast<const int*>(ws + p.perm);
  a.r = r;
  a.s = w.s;
  a.pair_of = reinterpret_cast<const int*>(ws + p.pair_of);
  a.u = reinterpret_cast<float*>(ws + p.u);
  a.hs = reinterpret_cast<bf16*>(ws + p.hs);
  a.a_pairs = reinterpret_cast<bf16*>(ws + p.H);
  a.v_pairs = reinterpret_cast<__half*>(ws + p.v_pairs);
  a.coef_pairs = reinterpret_cast<float*>(ws + p.coef);
  a.val_pairs = s.gated ? reinterpret_cast<const bf16*>(ws + p.val_pairs) : nullptr;
  a.s_out = reinterpret_cast<float*>(ws + p.s_out);
  a.out = static_cast<bf16*>(out);
  a.err = reinterpret_cast<int*>(ws + p.err);
  // operand maps (tiles of 128 or 256 rows) and output maps (32-row boxes)
  CUtensorMap mx, mbar, msup, mup, mapr, mdown, mhs, msdown, ou, ohs, oapr, ov, os;
  constexpr CUtensorMapDataType F32 = CU_TENSOR_MAP_DATA_TYPE_FLOAT32, F16 = CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  if ((err = make_map(&mx, x, D, T, pf::kBM)) != cudaSuccess ||
      (err = make_map(&mbar, w.W_bar_up, D, d_e, pf::kBN)) != cudaSuccess ||
      (err = make_map(&msup, w.W_s_up, D, d_s, pf::kBN)) != cudaSuccess ||
      (err = make_map(&mup, w.W_up, D, (uint64_t)E * d_e, pf::kBN)) != cudaSuccess ||
      (err = make_map(&mapr, a.a_pairs, d_e, P, pf::kBM)) != cudaSuccess ||
      (err = make_map(&mdown, w.W_down, d_e, (uint64_t)E * D, pf::kBN)) != cudaSuccess ||
      (err = make_map(&mhs, a.hs, d_s, T, pf::kBM)) != cudaSuccess ||
      (err = make_map(&msdown, w.W_s_down, d_s, D, pf::kBN)) != cudaSuccess ||
      (err = make_map(&ou, a.u, d_e, T, 32, F32)) != cudaSuccess ||
      (err = make_map(&ohs, a.hs, d_s, T, 32)) != cudaSuccess ||
      (err = make_map(&oapr, a.a_pairs, d_e, P, 32)) != cudaSuccess ||
      (err = make_map(&ov, a.v_pairs, D, P, 32, F16)) != cudaSuccess ||
      (err = make_map(&os, a.s_out, D, T, 32, F32)) != cudaSuccess)
    return err;
  const int row_tiles_max = (int)std::min<uint64_t>(P / pf::kBM + E, 1u << 30);
  // u and SiLU(x W_s_up^T)
  a.K = D;
  a.nu = cdiv(d_e, pf::kBN);
  a.n_tiles_n = a.nu + cdiv(d_s, pf::kBN);
  a.m_tiles = cdiv(T, pf::kBM);
  prof_mark(10, st);
  err = launch_pf<pf::kProj>(mx, mbar, msup, ou, ohs, a, std::min(a.m_tiles * a.n_tiles_n, p.sms), st);
  if (err != cudaSuccess) return err;
  prof_mark(11, st);
  // routed up-projections with NormSiLU (after the value rows of gated experts)
  a.bn = d_e;
  prof_mark(6, st);
  if (s.gated) {
    CUtensorMap mval, oval;
    if ((err = make_map(&mval, w.W_val, D, (uint64_t)E * d_e, pf::kBN)) != cudaSuccess ||
        (err = make_map(&oval, a.val_pairs, d_e, P, 32)) != cudaSuccess)
      return err;
    err = launch_pf<pf::kVal>(mx, mval, mval, oval, oval, a, std::min(row_tiles_max, p.sms), st);
    if (err != cudaSuccess) return err;
  }
  err = launch_pf<pf::kUp>(mx, mup, mup, oapr, oapr, a, std::min(row_tiles_max, p.sms), st);
  if (err != cudaSuccess) return err;
  prof_mark(7, st);
  // routed down-projections, one output row per pair
  a.K = d_e;
  a.n_tiles_n = cdiv(D, pf::kBN);
  prof_mark(8, st);
  err = launch_pf<pf::kDown>(mapr, mdown, mdown, ov, ov, a, p.sms, st);
  if (err != cudaSuccess) return err;
  prof_mark(9, st);
  // shared expert down-projection + combine + residual
  a.K = d_s;
  prof_mark(12, st);
  err = launch_pf<pf::kShared>(mhs, msdown, msdown, os, os, a, std::min(a.m_tiles * a.n_tiles_n, p.sms), st);
  if (err != cudaSuccess) return err;
  prof_mark(13, st);
  // out = shared + routed rows in ascending expert order (+ x)
  prof_mark(14, st);
  pf::k_combine<<<T, pf::kCThreads, 0, st>>>(a.s_out, a.v_pairs, a.coef_pairs, a.pair_of, a.x, a.out, D, E,
                                             s.residual);
  prof_mark(15, st);
  return cudaGetLastError();
}

// dense FFN y = W2 SiLU(W1 x) on the same kernels (bf16, T > 16)
cudaError_t run_dense_tc(int T, int D, int d_ff, const void* x, const void* W1, const void* W2, void* out,
                         unsigned char* ws, cudaStream_t st) {
  pf::Args a{};
  a.wait_cycles = g_wait_cycles;
  a.T = T;
  a.D = D;
  a.E = 0;
  a.d_e = 0;
  a.d_s = d_ff;
  a.x = static_cast<const bf16*>(x);
  a.hs = reinterpret_cast<bf16*>(ws + 256);
  a.out = static_cast<bf16*>(out);
  a.err = reinterpret_cast<int*>(ws);
  CUtensorMap mx, m1, mh, m2, oh;
  cudaError_t err;
  if ((err = make_map(&mx, x, D, T, pf::kBM)) != cudaSuccess ||
      (err = make_map(&m1, W1, D, d_ff, pf::kBN)) != cudaSuccess ||
      (err = make_map(&mh, a.hs, d_ff, T, pf::kBM)) != cudaSuccess ||
      (err = make_map(&m2, W2, d_ff, D, pf::kBN)) != cudaSuccess ||
      (err = make_map(&oh, a.hs, d_ff, T, 32)) != cudaSuccess)
    return err;
  const int sms = num_sms();
  a.K = D;
  a.nu = 0;
  a.n_tiles_n = cdiv(d_ff, pf::kBN);
  a.m_tiles = cdiv(T, pf::kBM);
  err = launch_pf<pf::kProj>(mx, m1, m1, oh, oh, a, std::min(a.m_tiles * a.n_tiles_n, sms), st);
  if (err != cudaSuccess) return err;
  a.K = d_ff;
  a.n_tiles_n = cdiv(D, pf::kBN);
  return launch_pf<pf::kShared>(mh, m2, m2, oh, oh, a, std::min(a.m_tiles * a.n_tiles_n, sms), st);
}

template <typename T>
cudaError_t run_forward(const deco_moe_shape_t& s, const void* x, const deco_moe_weights_t& w,
                        void* out, unsigned char* ws, const Plan& p, cudaStream_t st) {
  if (s.T <= dec::kMaxT && decode_eligible(s, p.sms)) {
    if (s.topk > 0) {   // TopK decisions first; the layer kernel then has no router CTAs
      cudaError_t err = run_routing<T>(s, x, w, ws, p, false, reinterpret_cast<float*>(ws + p.r),
                                       reinterpret_cast<uint8_t*>(ws + p.act),
                                       reinterpret_cast<int*>(ws + p.counts), reinterpret_cast<int*>(ws + p.offsets),
                                       reinterpret_cast<int*>(ws + p.perm), reinterpret_cast<int*>(ws + p.n_tok), st,
                                       p.tile_rows, /*decide_only=*/true);
      if (err != cudaSuccess) return err;
    }
    return run_decode(s, x, w, out, ws, p, st);
  }
  if (prefill_eligible(s)) return run_prefill(s, x, w, out, ws, p, st);
  float* r = reinterpret_cast<float*>(ws + p.r);
  uint8_t* act = reinterpret_cast<uint8_t*>(ws + p.act);
  int* counts = reinterpret_cast<int*>(ws + p.counts);
  cudaError_t err = run_routing<T>(s, x, w, ws, p, true, r, act, counts,
                                   reinterpret_cast<int*>(ws + p.offsets),
                                   reinterpret_cast<int*>(ws + p.perm),
                                   reinterpret_cast<int*>(ws + p.n_tok), st, p.tile_rows);
  if (err != cudaSuccess) return err;
  UpArgs ua{};
  ua.x = x;
  ua.D = s.d_model;
  ua.W_up = w.W_up;
  ua.W_val = s.gated ? w.W_val : nullptr;
  ua.d_e = s.d_e;
  ua.u = reinterpret_cast<const float*>(ws + p.u);
  ua.perm = reinterpret_cast<const int*>(ws + p.perm);
  ua.tiles = reinterpret_cast<const int4*>(ws + p.tiles);
  ua.n_tiles = reinterpret_cast<const int*>(ws + p.n_tiles);
  ua.H = reinterpret_cast<float*>(ws + p.H);
  ua.eps = s.rms_eps;
  const int max_tiles = (int)((size_t)s.T * s.E / p.tile_rows + s.E);
  prof_mark(6, st);
  err = p.tile_rows == 16 ? launch_up<T, 16>(ua, max_tiles, st) : launch_up<T, 8>(ua, max_tiles, st);
  if (err != cudaSuccess) return err;
  prof_mark(7, st);
  DownArgs da{};
  da.T = s.T;
  da.D = s.d_model;
  da.E = s.E;
  da.d_e = s.d_e;
  da.d_s = s.d_s;
  da.act = act;
  da.r = r;
  da.s = w.s;
  da.pair_of = reinterpret_cast<const int*>(ws + p.pair_of);
  da.H = reinterpret_cast<const float*>(ws + p.H);
  da.W_down = w.W_down;
  da.W_s_down = w.W_s_down;
  da.hs = reinterpret_cast<const float*>(ws + p.hs);
  da.x = x;
  da.out = out;
  da.residual = s.residual;
  prof_mark(8, st);
  err = launch_down<T>(da, st);
  prof_mark(9, st);
  return err;
}

std::mutex g_smem_mutex;   // serialises first-use attribute setting

}  // namespace
}  // namespace deco

using namespace deco;

extern "C" {

const char* deco_last_cuda_error(void) { return g_cuda_msg; }

const char* deco_status_string(deco_status_t s) {
  switch (s) {
    case DECO_OK: return "ok";
    case DECO_ERR_INVALID_ARG: return "invalid argument";
    case DECO_ERR_UNSUPPORTED: return "unsupported shape or dtype";
    case DECO_ERR_WORKSPACE: return "workspace missing or too small";
    case DECO_ERR_CUDA: return "CUDA error";
    case DECO_ERR_DEVICE: return "device-side error";
  }
  return "unknown status";
}

deco_status_t deco_moe_workspace_size(const deco_moe_shape_t* shape, size_t* bytes) {
  if (!bytes) return DECO_ERR_INVALID_ARG;
  const deco_status_t st = check_shape(shape);
  if (st != DECO_OK) return st;
  *bytes = make_plan(*shape).total;
  return DECO_OK;
}

deco_status_t deco_moe_forward(const deco_moe_shape_t* shape, const void* x,
                               const deco_moe_weights_t* w, void* out, void* workspace,
                               size_t workspace_bytes, void* stream) {
  deco_status_t st = check_shape(shape);
  if (st != DECO_OK) return st;
  if ((st = check_weights(w, false, shape->gated, shape->experts_on_host)) != DECO_OK) return st;
  if (shape->T == 0) return DECO_OK;
  if (!x || !out || !aligned16(x) || !aligned16(out) || x == out) return DECO_ERR_INVALID_ARG;
  const Plan p = make_plan(*shape);
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return DECO_ERR_WORKSPACE;
  if (workspace_bytes < p.total) return DECO_ERR_WORKSPACE;
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  cudaStream_t cs = as_stream(stream);
  std::lock_guard<std::mutex> lock(g_smem_mutex);
  cudaError_t err = cudaSuccess;
  // the decode kernel clears its counters and (with ReLU routing, when it is
  // the call's only kernel) the error word itself
  const bool self_clearing = shape->T <= dec::kMaxT && decode_eligible(*shape, p.sms);
  if (!self_clearing || shape->topk > 0) err = cudaMemsetAsync(ws + p.err, 0, 16, cs);
  if (err != cudaSuccess) return cuda_status(err, "forward: clearing the error word");
  err = shape->dtype == DECO_F32 ? run_forward<float>(*shape, x, *w, out, ws, p, cs)
                                 : run_forward<bf16>(*shape, x, *w, out, ws, p, cs);
  return cuda_status(err, "forward");
}

deco_status_t deco_moe_routing(const deco_moe_shape_t* shape, const void* x,
                               const deco_moe_weights_t* w, const deco_routing_t* out,
                               void* workspace, size_t workspace_bytes, void* stream) {
  deco_status_t st = check_shape(shape);
  if (st != DECO_OK) return st;
  if ((st = check_weights(w, true)) != DECO_OK) return st;
  if (!out) return DECO_ERR_INVALID_ARG;
  if (shape->T == 0) return DECO_OK;
  if (!x || !aligned16(x)) return DECO_ERR_INVALID_ARG;
  const Plan p = make_plan(*shape);
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return DECO_ERR_WORKSPACE;
  if (workspace_bytes < p.total) return DECO_ERR_WORKSPACE;
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  cudaStream_t cs = as_stream(stream);
  float* r = out->r ? out->r : reinterpret_cast<float*>(ws + p.r);
  uint8_t* act = out->active ? out->active : reinterpret_cast<uint8_t*>(ws + p.act);
  int* counts = out->counts ? out->counts : reinterpret_cast<int*>(ws + p.counts);
  int* offsets = out->offsets ? out->offsets : reinterpret_cast<int*>(ws + p.offsets);
  int* perm = out->perm ? out->perm : reinterpret_cast<int*>(ws + p.perm);
  int* n_tok = out->n_tok ? out->n_tok : reinterpret_cast<int*>(ws + p.n_tok);
  std::lock_guard<std::mutex> lock(g_smem_mutex);
  cudaError_t err = cudaMemsetAsync(ws + p.err, 0, 16, cs);
  if (err != cudaSuccess) return cuda_status(err, "routing: clearing the error word");
  err = shape->dtype == DECO_F32
            ? run_routing<float>(*shape, x, *w, ws, p, false, r, act, counts, offsets, perm, n_tok, cs,
                                 p.tile_rows)
            : run_routing<bf16>(*shape, x, *w, ws, p, false, r, act, counts, offsets, perm, n_tok, cs,
                                p.tile_rows);
  return cuda_status(err, "routing");
}

deco_status_t deco_moe_mean_up(int E, int d_e, int d_model, int dtype, const void* W_up,
                               void* W_bar_up, void* stream) {
  if (E <= 0 || d_e <= 0 || d_model <= 0 || !W_up || !W_bar_up) return DECO_ERR_INVALID_ARG;
  if (dtype != DECO_F32 && dtype != DECO_BF16) return DECO_ERR_INVALID_ARG;
  if (W_up == W_bar_up) return DECO_ERR_INVALID_ARG;
  const size_t n = (size_t)d_e * d_model;
  const int blocks = (int)std::min<size_t>((n + 255) / 256, 4096);
  cudaStream_t cs = as_stream(stream);
  if (dtype == DECO_F32)
    k_mean_up<float><<<blocks, 256, 0, cs>>>(static_cast<const float*>(W_up),
                                              static_cast<float*>(W_bar_up), E, n);
  else
    k_mean_up<bf16><<<blocks, 256, 0, cs>>>(static_cast<const bf16*>(W_up),
                                             static_cast<bf16*>(W_bar_up), E, n);
  return cuda_status(cudaGetLastError(), "mean_up");
}

// dense FFN: workspace = [err | hs [T][d_ff] fp32]
deco_status_t deco_dense_ffn_workspace_size(int T, int d_model, int d_ff, int dtype, size_t* bytes) {
  if (!bytes || T < 0 || d_model <= 0 || d_ff <= 0) return DECO_ERR_INVALID_ARG;
  if (dtype != DECO_F32 && dtype != DECO_BF16) return DECO_ERR_INVALID_ARG;
  if (d_model % 64 || d_model > 16384 || d_ff % 64 || d_ff > (1 << 20) || T > (1 << 20))
    return DECO_ERR_UNSUPPORTED;
  *bytes = 256 + align256((size_t)T * d_ff * 4);
  if (dtype == DECO_BF16 && T <= dec::kMaxT && decode_grid_ok(d_model, 0, num_sms()))
    *bytes = std::max(*bytes, dense_decode_bytes(d_model, d_ff, num_sms()));
  return DECO_OK;
}

deco_status_t deco_dense_ffn_forward(int T, int d_model, int d_ff, int dtype, const void* x,
                                     const void* W1, const void* W2, void* out, void* workspace,
                                     size_t workspace_bytes, void* stream) {
  size_t need = 0;
  deco_status_t st = deco_dense_ffn_workspace_size(T, d_model, d_ff, dtype, &need);
  if (st != DECO_OK) return st;
  if (T == 0) return DECO_OK;
  if (!x || !W1 || !W2 || !out || x == out) return DECO_ERR_INVALID_ARG;
  const void* ps[] = {x, W1, W2, out};
  for (const void* q : ps)
    if (!aligned16(q)) return DECO_ERR_INVALID_ARG;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) || workspace_bytes < need)
    return DECO_ERR_WORKSPACE;
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  cudaStream_t cs = as_stream(stream);
  std::lock_guard<std::mutex> lock(g_smem_mutex);
  RouteArgs ra{};
  ra.x = x;
  ra.T = T;
  ra.D = d_model;
  ra.E = 0;
  ra.d_e = 0;
  ra.W_s_up = W1;
  ra.d_s = d_ff;
  ra.hs = reinterpret_cast<float*>(ws + 256);
  ra.err = reinterpret_cast<int*>(ws);
  DownArgs da{};
  da.T = T;
  da.D = d_model;
  da.E = 0;
  da.d_e = 64;
  da.d_s = d_ff;
  da.W_s_down = W2;
  da.hs = ra.hs;
  da.x = x;
  da.out = out;
  da.residual = 0;
  cudaError_t err;
  const int sms = num_sms();
  if (dtype == DECO_BF16 && T <= dec::kMaxT && decode_grid_ok(d_model, 0, sms))   // weight streaming
    return cuda_status(run_dense_decode(T, d_model, d_ff, x, W1, W2, out, ws, sms, cs), "dense_ffn");
  if (dtype == DECO_BF16)   // tensor cores (a 128-row tile covers a small batch)
    return cuda_status(run_dense_tc(T, d_model, d_ff, x, W1, W2, out, ws, cs), "dense_ffn");
  const int tt = token_tile(d_model, dtype);
  if (dtype == DECO_F32) {
    err = route_any<float>(ra, tt, cs);
    if (err == cudaSuccess) err = launch_down<float>(da, cs);
  } else {
    err = route_any<bf16>(ra, tt, cs);
    if (err == cudaSuccess) err = launch_down<bf16>(da, cs);
  }
  return cuda_status(err, "dense_ffn");
}

deco_status_t deco_set_wait_limit(long long cycles) {
  if (cycles < 0) return DECO_ERR_INVALID_ARG;
  g_wait_cycles = cycles == 0 ? dec::kWaitCycles : cycles;
  return DECO_OK;
}

deco_status_t deco_moe_set_profiling(void* const* events, int n_events) {
  if (events && n_events < 0) return DECO_ERR_INVALID_ARG;
  g_prof_events = events ? reinterpret_cast<cudaEvent_t const*>(events) : nullptr;
  g_prof_n = events ? n_events : 0;
  return DECO_OK;
}

deco_status_t deco_moe_device_error(void* workspace, int* code, void* stream) {
  if (!workspace || !code) return DECO_ERR_INVALID_ARG;
  cudaStream_t cs = as_stream(stream);
  int v = 0;
  cudaError_t err = cudaMemcpyAsync(&v, workspace, sizeof(int), cudaMemcpyDeviceToHost, cs);
  if (err == cudaSuccess) err = cudaStreamSynchronize(cs);
  if (err != cudaSuccess) return cuda_status(err, "device_error");
  *code = v;
  return cuda_status(cudaMemsetAsync(workspace, 0, sizeof(int), cs), "device_error: clear");
}

}  // extern "C"

// ---------------------------------------------------------------------------
// deco_moe_forward_static: the forward pass on a library-owned static scratch
// array instead of a caller workspace, for callers that cannot allocate.

namespace deco {
namespace {

// The scratch every deco_moe_forward_static call on a device uses.  Host code
// must not pass `g_static_scratch` itself to a kernel: on the host the name is
// only a stand-in for the symbol, so its device address is looked up once per
// device with cudaGetSymbolAddress and cached here.  The cache is not
// invalidated by cudaDeviceReset (the module, and with it the array, may then
// be reloaded elsewhere), so the entry point is not for use after a reset.
static __device__ __align__(256) unsigned char g_static_scratch[DECO_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_static_mutex;
void* g_static_ptr[kMaxDevices] = {};

// address of this device's scratch array (set up on the first call per device)
cudaError_t static_scratch(unsigned char** out) {
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_static_mutex);
  if (!g_static_ptr[dev]) {
    void* p = nullptr;
    err = cudaGetSymbolAddress(&p, g_static_scratch);
    if (err != cudaSuccess) return err;
    g_static_ptr[dev] = p;
  }
  *out = static_cast<unsigned char*>(g_static_ptr[dev]);
  return cudaSuccess;
}

}  // namespace
}  // namespace deco

extern "C" deco_status_t deco_moe_forward_static(const deco_moe_shape_t* shape, const void* x,
                                                 const deco_moe_weights_t* w, void* out,
                                                 void* stream) {
  deco_status_t st = check_shape(shape);
  if (st != DECO_OK) return st;
  if ((st = check_weights(w, false, shape->gated, shape->experts_on_host)) != DECO_OK) return st;
  if (shape->T == 0) return DECO_OK;
  if (!x || !out || !aligned16(x) || !aligned16(out) || x == out) return DECO_ERR_INVALID_ARG;
  if (make_plan(*shape).total > DECO_STATIC_SCRATCH_BYTES) return DECO_ERR_WORKSPACE;
  unsigned char* scratch = nullptr;
  const cudaError_t err = static_scratch(&scratch);
  if (err != cudaSuccess) return cuda_status(err, "forward_static: scratch address");
  // the forward pass clears the error word it keeps at the start of the
  // scratch and overwrites everything else it reads
  return deco_moe_forward(shape, x, w, out, scratch, DECO_STATIC_SCRATCH_BYTES, stream);
}

extern "C" deco_status_t deco_moe_static_device_error(int* code, void* stream) {
  if (!code) return DECO_ERR_INVALID_ARG;
  unsigned char* scratch = nullptr;
  const cudaError_t err = static_scratch(&scratch);
  if (err != cudaSuccess) return cuda_status(err, "static_device_error: scratch address");
  // the error word sits at the start of every workspace plan
  return deco_moe_device_error(scratch, code, stream);
}

// ---------------------------------------------------------------------------
// training side: backward pass, router entropy, sparsity controller
// (backward_kernels.cuh)

namespace deco {
namespace {

struct BwdPlan {
  Plan route;   // the routing buffers of a forward plan (no tensor-core staging)
  size_t u, hs, as, du, dhs, pa, pdc, pdq, pz, pw, pk, dWbar, total;
};

BwdPlan make_bwd_plan(const deco_moe_shape_t& s) {
  deco_moe_shape_t rs = s;
  rs.experts_on_host = 1;   // a plan for the general kernels: routing, tables, no per-pair rows
  BwdPlan b{};
  b.route = make_plan(rs);
  size_t off = b.route.total;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align256(off + bytes);
    return o;
  };
  const size_t T = s.T, P = T * s.E;
  b.u = take(T * s.d_e * 4);
  b.hs = take(T * s.d_s * 4);
  b.as = take(T * s.d_s * 4);
  b.du = take(T * s.d_e * 4);
  b.dhs = take(T * s.d_s * 4);
  b.pa = take(P * s.d_e * 4);
  b.pdc = take(P * s.d_e * 4);
  b.pdq = s.gated ? take(P * s.d_e * 4) : 0;
  b.pz = take(P * 4);
  b.pw = take(P * 4);
  b.pk = take(P * 4);
  b.dWbar = take((size_t)s.d_e * s.d_model * 4);
  b.total = off;
  return b;
}

deco_status_t check_bwd_shape(const deco_moe_shape_t* s) {
  const deco_status_t st = check_shape(s);
  if (st != DECO_OK) return st;
  if (s->topk != 0) return DECO_ERR_UNSUPPORTED;   // the gradient is that of ReLU routing
  return DECO_OK;
}

template <typename T>
cudaError_t run_backward(const deco_moe_shape_t& s, const void* x, const deco_moe_weights_t& w, const void* dy,
                         const float* dz_extra, const deco_moe_grads_t& g, unsigned char* ws, const BwdPlan& b,
                         cudaStream_t st) {
  const Plan& p = b.route;
  float* r = reinterpret_cast<float*>(ws + p.r);
  uint8_t* act = ws + p.act;
  int* counts = reinterpret_cast<int*>(ws + p.counts);
  int* offsets = reinterpret_cast<int*>(ws + p.offsets);
  int* perm = reinterpret_cast<int*>(ws + p.perm);
  int* n_tok = reinterpret_cast<int*>(ws + p.n_tok);
  cudaError_t err = run_routing<T>(s, x, w, ws, p, false, r, act, counts, offsets, perm, n_tok, st, p.tile_rows);
  if (err != cudaSuccess) return err;
  bwd::Args a{};
  a.T = s.T;
  a.D = s.d_model;
  a.E = s.E;
  a.d_e = s.d_e;
  a.d_s = s.d_s;
  a.eps = s.rms_eps;
  a.gated = s.gated;
  a.residual = s.residual;
  a.x = x;
  a.dy = dy;
  a.dz_extra = dz_extra;
  a.W_r = w.W_r;
  a.W_bar = w.W_bar_up;
  a.W_up = w.W_up;
  a.W_down = w.W_down;
  a.s = w.s;
  a.W_s_up = w.W_s_up;
  a.W_s_down = w.W_s_down;
  a.W_val = w.W_val;
  a.r = r;
  a.act = act;
  a.offsets = offsets;
  a.perm = perm;
  a.pair_of = reinterpret_cast<const int*>(ws + p.pair_of);
  a.u = reinterpret_cast<float*>(ws + b.u);
  a.hs = reinterpret_cast<float*>(ws + b.hs);
  a.as = reinterpret_cast<float*>(ws + b.as);
  a.du = reinterpret_cast<float*>(ws + b.du);
  a.dhs = reinterpret_cast<float*>(ws + b.dhs);
  a.pa = reinterpret_cast<float*>(ws + b.pa);
  a.pdc = reinterpret_cast<float*>(ws + b.pdc);
  a.pdq = s.gated ? reinterpret_cast<float*>(ws + b.pdq) : nullptr;
  a.pz = reinterpret_cast<float*>(ws + b.pz);
  a.pw = reinterpret_cast<float*>(ws + b.pw);
  a.pk = reinterpret_cast<float*>(ws + b.pk);
  a.dWbar = reinterpret_cast<float*>(ws + b.dWbar);
  a.dx = g.dx;
  a.dW_r = g.dW_r;
  a.db_r = g.db_r;
  a.dW_up = g.dW_up;
  a.dW_down = g.dW_down;
  a.ds = g.ds;
  a.dW_s_up = g.dW_s_up;
  a.dW_s_down = g.dW_s_down;
  a.dW_val = g.dW_val;
  const size_t sm0 = (size_t)s.d_model * 4;
  const size_t sm1 = (2 * (size_t)s.d_model + (3 + bwd::kWarps) * (size_t)s.d_e) * 4;
  const size_t sm3 = ((size_t)s.d_s + 3 * (size_t)s.d_e) * 4;
  if ((err = allow_smem(bwd::kb_token_fwd<T>, sm0)) != cudaSuccess) return err;
  if ((err = allow_smem(bwd::kb_pair<T>, sm1)) != cudaSuccess) return err;
  if ((err = allow_smem(bwd::kb_dx<T>, sm3)) != cudaSuccess) return err;
  bwd::kb_token_fwd<T><<<dim3(s.T, (s.d_e + s.d_s + bwd::kFwdRows - 1) / bwd::kFwdRows), bwd::kThreads, sm0, st>>>(a);
  bwd::kb_pair<T><<<dim3(s.T, s.E), bwd::kThreads, sm1, st>>>(a);
  bwd::kb_token_mid<T><<<dim3(s.T, (s.d_s + 31) / 32), bwd::kThreads, 0, st>>>(a);
  bwd::kb_dx<T><<<dim3(s.T, (s.d_model + 31) / 32), bwd::kThreads, sm3, st>>>(a);
  const size_t n_sums = ((size_t)s.d_e + 2 * (size_t)s.d_s) * s.d_model;
  bwd::kb_sums<T><<<(unsigned)std::min<size_t>((n_sums + bwd::kThreads - 1) / bwd::kThreads, 4096),
                    bwd::kThreads, 0, st>>>(a);
  const size_t n_exp = (size_t)s.d_e * s.d_model * (s.gated ? 3 : 2) + s.d_model + 2;
  bwd::kb_expert<T><<<dim3((unsigned)std::min<size_t>((n_exp + bwd::kThreads - 1) / bwd::kThreads, 64), s.E),
                      bwd::kThreads, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace
}  // namespace deco

extern "C" deco_status_t deco_moe_backward_workspace_size(const deco_moe_shape_t* shape, size_t* bytes) {
  using namespace deco;
  const deco_status_t st = check_bwd_shape(shape);
  if (st != DECO_OK) return st;
  if (!bytes) return DECO_ERR_INVALID_ARG;
  *bytes = make_bwd_plan(*shape).total;
  return DECO_OK;
}

extern "C" deco_status_t deco_moe_backward(const deco_moe_shape_t* shape, const void* x,
                                           const deco_moe_weights_t* w, const void* dy, const float* dz_extra,
                                           const deco_moe_grads_t* g, void* workspace, size_t workspace_bytes,
                                           void* stream) {
  using namespace deco;
  deco_status_t st = check_bwd_shape(shape);
  if (st != DECO_OK) return st;
  if ((st = check_weights(w, false, shape->gated, shape->experts_on_host)) != DECO_OK) return st;
  if (!g) return DECO_ERR_INVALID_ARG;
  float* gs[] = {g->dx, g->dW_r, g->db_r, g->dW_up, g->dW_down, g->ds, g->dW_s_up, g->dW_s_down};
  for (float* q : gs)
    if (!q || !aligned16(q)) return DECO_ERR_INVALID_ARG;
  if (shape->gated && (!g->dW_val || !aligned16(g->dW_val))) return DECO_ERR_INVALID_ARG;
  if (shape->T == 0) return DECO_OK;
  if (!x || !dy || !aligned16(x) || !aligned16(dy)) return DECO_ERR_INVALID_ARG;
  if (dz_extra && (reinterpret_cast<uintptr_t>(dz_extra) & 3u)) return DECO_ERR_INVALID_ARG;
  const BwdPlan b = make_bwd_plan(*shape);
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return DECO_ERR_WORKSPACE;
  if (workspace_bytes < b.total) return DECO_ERR_WORKSPACE;
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  cudaStream_t cs = as_stream(stream);
  std::lock_guard<std::mutex> lock(g_smem_mutex);
  cudaError_t err = cudaMemsetAsync(ws + b.route.err, 0, 16, cs);
  if (err != cudaSuccess) return cuda_status(err, "backward: clearing the error word");
  err = shape->dtype == DECO_F32 ? run_backward<float>(*shape, x, *w, dy, dz_extra, *g, ws, b, cs)
                                 : run_backward<bf16>(*shape, x, *w, dy, dz_extra, *g, ws, b, cs);
  return cuda_status(err, "backward");
}

extern "C" deco_status_t deco_moe_router_entropy(int T, int E, const float* r, const uint8_t* active,
                                                 float lambda, float* H, float* dz, void* stream) {
  using namespace deco;
  if (T < 0 || E <= 0 || E > 256 || !std::isfinite(lambda)) return DECO_ERR_INVALID_ARG;
  if (T == 0) return DECO_OK;
  if (!r || !active || !H || !dz || (reinterpret_cast<uintptr_t>(r) & 3u) ||
      (reinterpret_cast<uintptr_t>(H) & 3u) || (reinterpret_cast<uintptr_t>(dz) & 3u))
    return DECO_ERR_INVALID_ARG;
  cudaStream_t cs = as_stream(stream);
  bwd::kb_entropy<<<(T + bwd::kWarps - 1) / bwd::kWarps, bwd::kThreads, 0, cs>>>(r, active, T, E, lambda, H, dz);
  bwd::kb_entropy_mean<<<1, 32, 0, cs>>>(H, T);
  return cuda_status(cudaGetLastError(), "router_entropy");
}

extern "C" deco_status_t deco_sparsity_controller(double* lambda, double ratio, double target, double factor) {
  if (!lambda || !(factor > 1.0) || !std::isfinite(factor) || !std::isfinite(ratio) || !std::isfinite(target) ||
      !std::isfinite(*lambda))
    return DECO_ERR_INVALID_ARG;
  if (ratio > target) *lambda *= factor;
  else if (ratio < target) *lambda /= factor;
  return DECO_OK;
}
