// Backward pieces outside the expert GEMMs, for the objective
// <dy, y> + alpha * L_lb + beta * L_z ("OLMoE Guide", "Router Mechanics & Loss
// Formulations"; "OLMoE: Open Mixture-of-Experts Language Models", 4.1.6 and
// 4.1.7 for alpha and beta). No gradient flows through the choice of experts or
// through the counts f_i (a bincount).
//
//   combine backward  dw_tj = <dy_t, o_tj> with the fp32 expert outputs the
//                     forward kept; dO[r] = w_tj dy_t for the row r of pair
//                     (t, j), zero on padding rows.           (row-parallel gather)
//   router backward   dp_ti = sum_j [S_tj = i] dw_tj + alpha E f_i / T
//                     dh_t  = p_t * (dp_t - <dp_t, p_t>) + beta (2 lse_t / T) p_t
//   dx                dx_t = sum_j dX_perm[row(t, j)] + sum_e dh_t,e W_r[e]
//   router weights    dW_r[e] = sum_t dh_t,e x_t   (split over tokens, then a
//                     fixed-order reduction of the partials)
// Every reduction runs in a fixed order, so the gradients are deterministic.
#include "moe_internal.h"
#include "sm100.cuh"

namespace moe {
namespace {

template <typename T_>
__device__ __forceinline__ void load8(const T_* p, float (&v)[8]) {
  if constexpr (sizeof(T_) == 4) {
    const float4 a = reinterpret_cast<const float4*>(p)[0];
    const float4 b = reinterpret_cast<const float4*>(p)[1];
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  } else {
    const uint4 q = reinterpret_cast<const uint4*>(p)[0];
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 f = bf16x2_to_float2(w[j]);
      v[2 * j] = f.x;
      v[2 * j + 1] = f.y;
    }
  }
}

template <typename T_>
__device__ __forceinline__ void store8(T_* p, const float (&v)[8]) {
  if constexpr (sizeof(T_) == 4) {
    reinterpret_cast<float4*>(p)[0] = make_float4(v[0], v[1], v[2], v[3]);
    reinterpret_cast<float4*>(p)[1] = make_float4(v[4], v[5], v[6], v[7]);
  } else {
    uint4 q;
    q.x = pack_bf16x2(v[0], v[1]);
    q.y = pack_bf16x2(v[2], v[3]);
    q.z = pack_bf16x2(v[4], v[5]);
    q.w = pack_bf16x2(v[6], v[7]);
    reinterpret_cast<uint4*>(p)[0] = q;
  }
}

// One warp per padded row; o_perm holds the fp32 expert outputs.
template <typename T_>
__global__ void __launch_bounds__(256)
    combine_bwd_kernel(const T_* __restrict__ dy, const float* __restrict__ o_perm, const int32_t* __restrict__ row_pair,
                       const int32_t* __restrict__ gs, int E, const float* __restrict__ wts, int d, int k,
                       float* __restrict__ dw, T_* __restrict__ dout) {
  pdl_trigger();
  pdl_wait();  // reads and writes buffers an earlier kernel of the layer uses
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t r = static_cast<int64_t>(blockIdx.x) * 8 + warp;
  if (r >= gs[E]) return;
  const int pair = row_pair[r];
  const int nv = d / 8;
  T_* orow = dout + r * d;
  if (pair < 0) {
    const float z[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    for (int v = lane; v < nv; v += 32) store8<T_>(orow + v * 8, z);
    return;
  }
  const int64_t t = pair / k;
  const float w = wts[pair];
  float dot = 0.f;
  for (int v = lane; v < nv; v += 32) {
    float g[8], o[8], out[8];
    load8<T_>(dy + t * d + v * 8, g);
    load8<float>(o_perm + r * d + v * 8, o);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      dot = fmaf(g[i], o[i], dot);
      out[i] = w * g[i];
    }
    store8<T_>(orow + v * 8, out);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
  if (lane == 0) dw[pair] = dot;
}

// One warp per token.
__global__ void __launch_bounds__(256)
    router_bwd_kernel(const float* __restrict__ dw, const int32_t* __restrict__ idx, const float* __restrict__ probs,
                      const float* __restrict__ lse, const int32_t* __restrict__ counts, int64_t T, int E, int k,
                      float alpha, float beta, int renorm, float* __restrict__ dh) {
  pdl_trigger();
  pdl_wait();  // reads and writes buffers an earlier kernel of the layer uses
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t t = static_cast<int64_t>(blockIdx.x) * 8 + warp;
  if (t >= T) return;
  // Renormalised weights w_j = p_j / s (s = sum of the chosen p): the chosen
  // probabilities receive (dw_j - <dw, w>) / s instead of dw_j. Lane j < k holds
  // slot j; the two sums use a fixed butterfly.
  float inv_s = 1.f, shift = 0.f;
  if (renorm) {
    float pj = 0.f, dwj = 0.f;
    if (lane < k) {
      const int e = idx[t * k + lane];
      pj = (e >= 0 && e < E) ? probs[t * E + e] : 0.f;
      dwj = dw[t * k + lane];
    }
    float ssum = pj, wdot = dwj * pj;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      ssum += __shfl_xor_sync(0xffffffffu, ssum, o);
      wdot += __shfl_xor_sync(0xffffffffu, wdot, o);
    }
    inv_s = ssum > 0.f ? 1.f / ssum : 0.f;
    shift = wdot * inv_s;  // <dw, w>
  }
  constexpr int Q = kMaxExperts / 32;
  const float Tf = static_cast<float>(T);
  float dp[Q], p[Q];
  float dot = 0.f;
#pragma unroll
  for (int q = 0; q < Q; ++q) {
    const int e = lane + 32 * q;
    dp[q] = 0.f;
    p[q] = 0.f;
    if (e < E) {
      p[q] = probs[t * E + e];
      float g = alpha * static_cast<float>(E) * (static_cast<float>(counts[e]) / (Tf * k)) / Tf;
      for (int j = 0; j < k; ++j)
        if (idx[t * k + j] == e) g += renorm ? (dw[t * k + j] - shift) * inv_s : dw[t * k + j];
      dp[q] = g;
      dot = fmaf(g, p[q], dot);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
  const float zterm = beta * 2.0f * lse[t] / Tf;
#pragma unroll
  for (int q = 0; q < Q; ++q) {
    const int e = lane + 32 * q;
    if (e < E) dh[t * E + e] = p[q] * (dp[q] - dot) + zterm * p[q];
  }
}

// dx for a 64-token x 128-column tile per CTA: the router term dh W_r from
// shared-memory tiles of dh and W_r (64 experts at a time; thread = 8 tokens x
// 4 columns), then the k expert rows added in slot order.
constexpr int kDxRows = 64;
constexpr int kDxCols = 128;
constexpr int kDxE = 64;

template <typename T_>
__device__ __forceinline__ void load4(const T_* p, float (&v)[4]) {
  if constexpr (sizeof(T_) == 4) {
    const float4 a = *reinterpret_cast<const float4*>(p);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  } else {
    const uint2 q = *reinterpret_cast<const uint2*>(p);
    const float2 f0 = bf16x2_to_float2(q.x);
    const float2 f1 = bf16x2_to_float2(q.y);
    v[0] = f0.x; v[1] = f0.y; v[2] = f1.x; v[3] = f1.y;
  }
}

template <typename T_>
__device__ __forceinline__ void store4(T_* p, const float (&v)[4]) {
  if constexpr (sizeof(T_) == 4) {
    *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
  } else {
    uint2 q;
    q.x = pack_bf16x2(v[0], v[1]);
    q.y = pack_bf16x2(v[2], v[3]);
    *reinterpret_cast<uint2*>(p) = q;
  }
}

template <typename T_>
__global__ void __launch_bounds__(256)
    dx_kernel(const T_* __restrict__ dx_perm, const int32_t* __restrict__ inv_perm, const float* __restrict__ dh,
              const T_* __restrict__ w_router, int64_t T, int d, int E, int k, T_* __restrict__ dx) {
  pdl_trigger();
  pdl_wait();  // reads and writes buffers an earlier kernel of the layer uses
  __shared__ float sdh[kDxRows][kDxE];
  __shared__ __align__(16) float sw[kDxE][kDxCols];
  const int64_t t0 = static_cast<int64_t>(blockIdx.x) * kDxRows;
  const int c0 = blockIdx.y * kDxCols;
  const int tg = threadIdx.x >> 5;        // tokens t0 + 8 tg .. +7
  const int cg = threadIdx.x & 31;        // columns c0 + 4 cg .. +3
  float acc[8][4];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
  for (int e0 = 0; e0 < E; e0 += kDxE) {
    const int ne = min(kDxE, E - e0);
    __syncthreads();
    for (int i = threadIdx.x; i < kDxRows * kDxE; i += blockDim.x) {
      const int r = i / kDxE, e = i - r * kDxE;
      sdh[r][e] = (t0 + r < T && e < ne) ? dh[(t0 + r) * E + e0 + e] : 0.f;
    }
    for (int i = threadIdx.x; i < kDxE * (kDxCols / 4); i += blockDim.x) {
      const int e = i / (kDxCols / 4), c = (i - e * (kDxCols / 4)) * 4;
      float v[4] = {0.f, 0.f, 0.f, 0.f};
      if (e < ne && c0 + c < d) load4<T_>(w_router + static_cast<int64_t>(e0 + e) * d + c0 + c, v);
      *reinterpret_cast<float4*>(&sw[e][c]) = make_float4(v[0], v[1], v[2], v[3]);
    }
    __syncthreads();
    for (int e = 0; e < ne; ++e) {
      const float4 w = *reinterpret_cast<const float4*>(&sw[e][4 * cg]);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float g = sdh[8 * tg + i][e];
        acc[i][0] = fmaf(g, w.x, acc[i][0]);
        acc[i][1] = fmaf(g, w.y, acc[i][1]);
        acc[i][2] = fmaf(g, w.z, acc[i][2]);
        acc[i][3] = fmaf(g, w.w, acc[i][3]);
      }
    }
  }
  const int col = c0 + 4 * cg;
  if (col >= d) return;
  for (int i = 0; i < 8; ++i) {
    const int64_t t = t0 + 8 * tg + i;
    if (t >= T) break;
    float out[4] = {0.f, 0.f, 0.f, 0.f};
    for (int j = 0; j < k; ++j) {
      const int r = inv_perm[t * k + j];
      if (r < 0) continue;
      float g[4];
      load4<T_>(dx_perm + static_cast<int64_t>(r) * d + col, g);
#pragma unroll
      for (int c = 0; c < 4; ++c) out[c] += g[c];
    }
#pragma unroll
    for (int c = 0; c < 4; ++c) out[c] += acc[i][c];
    store4<T_>(dx + t * d + col, out);
  }
}

constexpr int kWrSplit = 32;  // token splits for the router weight gradient
constexpr int kWrTok = 32;    // tokens per shared-memory chunk

// Partial dW_r over a token range for a 64-expert x 128-column tile: chunks of
// 32 tokens of dh and x staged in shared memory; thread = 8 experts x 4 columns.
template <typename T_>
__global__ void __launch_bounds__(256)
    router_wgrad_partial(const float* __restrict__ dh, const T_* __restrict__ x, int64_t T, int d, int E,
                         float* __restrict__ part) {
  pdl_trigger();
  pdl_wait();  // reads and writes buffers an earlier kernel of the layer uses
  __shared__ __align__(16) float sdh[kWrTok][64];
  __shared__ __align__(16) float sx[kWrTok][128];
  const int c0 = blockIdx.x * 128;
  const int split = blockIdx.y;
  const int e0 = blockIdx.z * 64;
  const int eg = threadIdx.x >> 5;  // experts e0 + 8 eg .. +7
  const int cg = threadIdx.x & 31;  // columns c0 + 4 cg .. +3
  const int64_t per = (T + kWrSplit - 1) / kWrSplit;
  const int64_t ta = split * per;
  const int64_t tb = (ta + per) < T ? (ta + per) : T;
  float acc[8][4];
#pragma unroll
  for (int a = 0; a < 8; ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b) acc[a][b] = 0.f;
  for (int64_t tc = ta; tc < tb; tc += kWrTok) {
    const int nt = static_cast<int>((tb - tc) < kWrTok ? (tb - tc) : kWrTok);
    __syncthreads();
    for (int i = threadIdx.x; i < kWrTok * 64; i += blockDim.x) {
      const int r = i >> 6, e = i & 63;
      sdh[r][e] = (r < nt && e0 + e < E) ? dh[(tc + r) * E + e0 + e] : 0.f;
    }
    for (int i = threadIdx.x; i < kWrTok * 32; i += blockDim.x) {
      const int r = i >> 5, c = (i & 31) * 4;
      float v[4] = {0.f, 0.f, 0.f, 0.f};
      if (r < nt && c0 + c < d) load4<T_>(x + (tc + r) * d + c0 + c, v);
      *reinterpret_cast<float4*>(&sx[r][c]) = make_float4(v[0], v[1], v[2], v[3]);
    }
    __syncthreads();
    for (int r = 0; r < nt; ++r) {
      const float4 xv = *reinterpret_cast<const float4*>(&sx[r][4 * cg]);
      const float4 g0 = *reinterpret_cast<const float4*>(&sdh[r][8 * eg]);
      const float4 g1 = *reinterpret_cast<const float4*>(&sdh[r][8 * eg + 4]);
      const float g[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
#pragma unroll
      for (int a = 0; a < 8; ++a) {
        acc[a][0] = fmaf(g[a], xv.x, acc[a][0]);
        acc[a][1] = fmaf(g[a], xv.y, acc[a][1]);
        acc[a][2] = fmaf(g[a], xv.z, acc[a][2]);
        acc[a][3] = fmaf(g[a], xv.w, acc[a][3]);
      }
    }
  }
  const int col = c0 + 4 * cg;
  if (col >= d) return;
  for (int a = 0; a < 8; ++a) {
    const int e = e0 + 8 * eg + a;
    if (e >= E) break;
    *reinterpret_cast<float4*>(part + (static_cast<int64_t>(split) * E + e) * d + col) =
        make_float4(acc[a][0], acc[a][1], acc[a][2], acc[a][3]);
  }
}

template <typename T_>
__global__ void router_wgrad_reduce(const float* __restrict__ part, int64_t n, T_* __restrict__ out) {
  pdl_trigger();
  pdl_wait();  // reads and writes buffers an earlier kernel of the layer uses
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= n) return;
  float s = 0.f;
  for (int sp = 0; sp < kWrSplit; ++sp) s += part[sp * n + i];
  out[i] = from_f32<T_>(s);
}

}  // namespace

size_t router_wgrad_partial_bytes(const Shape& s) {
  return static_cast<size_t>(kWrSplit) * s.E * s.d * sizeof(float);
}

cudaError_t launch_combine_backward(const Shape& s, const void* dy, const void* o_perm, const int32_t* gs,
                                    const int32_t* row_pair, const float* wts, float* dw, void* dout,
                                    cudaStream_t st) {
  const unsigned grid = static_cast<unsigned>((s.P + 7) / 8);
  const float* o32 = static_cast<const float*>(o_perm);
  if (s.fp32)
    launch_dependent(combine_bwd_kernel<float>, dim3(grid), dim3(256), 0, st, nullptr, 0, static_cast<const float*>(dy), o32, row_pair, gs, s.E, wts, s.d,
                                                    s.k, dw, static_cast<float*>(dout));
  else
    launch_dependent(combine_bwd_kernel<__nv_bfloat16>, dim3(grid), dim3(256), 0, st, nullptr, 0, static_cast<const __nv_bfloat16*>(dy), o32, row_pair, gs,
                                                            s.E, wts, s.d, s.k, dw, static_cast<__nv_bfloat16*>(dout));
  return cudaGetLastError();
}

cudaError_t launch_router_backward(const Shape& s, const float* dw, const int32_t* idx, const float* probs,
                                   const float* lse, const int32_t* counts, float alpha, float beta, float* dh,
                                   cudaStream_t st) {
  const unsigned grid = static_cast<unsigned>((s.T + 7) / 8);
  launch_dependent(router_bwd_kernel, dim3(grid), dim3(256), 0, st, nullptr, 0, dw, idx, probs, lse, counts, s.T, s.E, s.k, alpha, beta,
                                          s.renorm ? 1 : 0, dh);
  return cudaGetLastError();
}

cudaError_t launch_dx_combine(const Shape& s, const void* dx_perm, const int32_t* inv_perm, const float* dh,
                              const void* w_router, void* dx, cudaStream_t st) {
  const dim3 grid(static_cast<unsigned>((s.T + kDxRows - 1) / kDxRows), static_cast<unsigned>((s.d + kDxCols - 1) / kDxCols));
  const int threads = 256;
  if (s.fp32)
    launch_dependent(dx_kernel<float>, dim3(grid), dim3(threads), 0, st, nullptr, 0, static_cast<const float*>(dx_perm), inv_perm, dh,
                                               static_cast<const float*>(w_router), s.T, s.d, s.E, s.k,
                                               static_cast<float*>(dx));
  else
    launch_dependent(dx_kernel<__nv_bfloat16>, dim3(grid), dim3(threads), 0, st, nullptr, 0, static_cast<const __nv_bfloat16*>(dx_perm), inv_perm, dh,
                                                       static_cast<const __nv_bfloat16*>(w_router), s.T, s.d, s.E, s.k,
                                                       static_cast<__nv_bfloat16*>(dx));
  return cudaGetLastError();
}

cudaError_t launch_router_weight_grad(const Shape& s, const float* dh, const void* x, void* dw_router, float* part,
                                      cudaStream_t st) {
  dim3 grid((s.d + 127) / 128, kWrSplit, (s.E + 63) / 64);
  if (s.fp32)
    launch_dependent(router_wgrad_partial<float>, dim3(grid), dim3(256), 0, st, nullptr, 0, dh, static_cast<const float*>(x), s.T, s.d, s.E, part);
  else
    launch_dependent(router_wgrad_partial<__nv_bfloat16>, dim3(grid), dim3(256), 0, st, nullptr, 0, dh, static_cast<const __nv_bfloat16*>(x), s.T, s.d,
                                                              s.E, part);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int64_t n = static_cast<int64_t>(s.E) * s.d;
  const unsigned g2 = static_cast<unsigned>((n + 255) / 256);
  if (s.fp32 || s.grad32)
    launch_dependent(router_wgrad_reduce<float>, dim3(g2), dim3(256), 0, st, nullptr, 0, part, n, static_cast<float*>(dw_router));
  else
    launch_dependent(router_wgrad_reduce<__nv_bfloat16>, dim3(g2), dim3(256), 0, st, nullptr, 0, part, n, static_cast<__nv_bfloat16*>(dw_router));
  return cudaGetLastError();
}

}  // namespace moe
