// Combine and RMSNorm.
//
// Combine ("OLMoE Guide", "Top-8 Softmax Routing Formulation": y = sum_i P_i
// Expert_i(x); "Mixture-of-experts LLMs from scratch with OLMoE", section 2,
// `dispatch` adds each expert's weighted rows back to their tokens): a gather,
// not a scatter. Token t reads its k expert rows through inv_perm and sums
// w_tj * o_tj in fp32 in slot order j = 0..k-1, then rounds once, so the result
// is deterministic (no atomics). The residual variant adds the fp32 sum into
// an fp32 residual stream instead (section 3, Block: x + mlp(norm(x)).float()).
//
// RMSNorm (section 3, RMSNorm, eps 1e-5): y = r / sqrt(mean(r^2) + eps) * w on
// the fp32 residual, written in the layer's input dtype. The mean of squares is
// reduced in a fixed order.
#include "moe_internal.h"
#include "sm100.cuh"

namespace moe {
namespace {

template <typename T_>
struct Vec8 {
  float v[8];
  __device__ __forceinline__ void load(const T_* p) {
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
  __device__ __forceinline__ void store(T_* p) const {
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
};

// Eight elements as loaded (16 bytes of bf16 or 32 of fp32), unpacked later.
template <typename T_>
struct Raw8 {
  uint4 a, b;
  __device__ __forceinline__ void load(const T_* p) {
    a = __ldg(reinterpret_cast<const uint4*>(p));
    if constexpr (sizeof(T_) == 4) b = __ldg(reinterpret_cast<const uint4*>(p) + 1);
  }
  __device__ __forceinline__ void unpack(float (&v)[8]) const {
    if constexpr (sizeof(T_) == 4) {
      v[0] = __uint_as_float(a.x); v[1] = __uint_as_float(a.y); v[2] = __uint_as_float(a.z); v[3] = __uint_as_float(a.w);
      v[4] = __uint_as_float(b.x); v[5] = __uint_as_float(b.y); v[6] = __uint_as_float(b.z); v[7] = __uint_as_float(b.w);
    } else {
      const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 f = bf16x2_to_float2(w[j]);
        v[2 * j] = f.x;
        v[2 * j + 1] = f.y;
      }
    }
  }
};

// OT: element type of the expert rows (the layer dtype, or fp32 when the
// forward keeps them for the backward); T_: the output's.
template <typename OT, typename T_, bool RESID>
__global__ void __launch_bounds__(256)
    combine_kernel(const OT* __restrict__ o_perm, const int32_t* __restrict__ inv_perm, const float* __restrict__ wts,
                   int64_t T, int d, int k, T_* __restrict__ y, float* __restrict__ resid) {
  pdl_trigger();
  pdl_wait();  // reads and writes buffers an earlier kernel of the layer uses
  __shared__ int32_t rows[kMaxTopK];
  __shared__ float ws_[kMaxTopK];
  const int64_t t = blockIdx.x;
  if (threadIdx.x < k) {
    rows[threadIdx.x] = inv_perm[t * k + threadIdx.x];
    ws_[threadIdx.x] = wts[t * k + threadIdx.x];
  }
  __syncthreads();
  const int nv = d / 8;
  for (int v = threadIdx.x; v < nv; v += blockDim.x) {
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.f;
    // The k rows' loads go out together (unconditional: a slot without a row
    // re-reads row 0, which always exists, and is then skipped), then the sum
    // runs in slot order.
    for (int j0 = 0; j0 < k; j0 += 8) {
      Raw8<OT> q[8];
#pragma unroll
      for (int jj = 0; jj < 8; ++jj) {
        const int j = j0 + jj;
        const int r = (j < k) ? rows[j] : -1;
        q[jj].load(o_perm + static_cast<int64_t>(r < 0 ? 0 : r) * d + v * 8);
      }
#pragma unroll
      for (int jj = 0; jj < 8; ++jj) {
        const int j = j0 + jj;
        if (j < k && rows[j] >= 0) {
          float o[8];
          q[jj].unpack(o);
          const float w = ws_[j];
#pragma unroll
          for (int i = 0; i < 8; ++i) acc[i] = fmaf(w, o[i], acc[i]);
        }
      }
    }
    if constexpr (RESID) {
      float* rp = resid + t * d + v * 8;
      float4 a = reinterpret_cast<float4*>(rp)[0];
      float4 b = reinterpret_cast<float4*>(rp)[1];
      a.x += acc[0]; a.y += acc[1]; a.z += acc[2]; a.w += acc[3];
      b.x += acc[4]; b.y += acc[5]; b.z += acc[6]; b.w += acc[7];
      reinterpret_cast<float4*>(rp)[0] = a;
      reinterpret_cast<float4*>(rp)[1] = b;
    } else {
      Vec8<T_> out;
#pragma unroll
      for (int i = 0; i < 8; ++i) out.v[i] = acc[i];
      out.store(y + t * d + v * 8);
    }
  }
}

// Expert-choice combine: token t's experts are the e with slot_row[t, e] >= 0,
// taken in ascending e with weight p[t, e]; warp 0 compacts the list with
// ballots first (so the launch has at least 32 threads), then the loads of up
// to eight rows go out together; a token no expert took gets zero.
template <typename T_>
__global__ void __launch_bounds__(256)
    combine_ec_kernel(const T_* __restrict__ o_perm, const int32_t* __restrict__ slot_row,
                      const float* __restrict__ probs, int64_t T, int d, int E, T_* __restrict__ y) {
  pdl_trigger();
  pdl_wait();  // reads and writes buffers an earlier kernel of the layer uses
  __shared__ int32_t rows[kMaxExperts];
  __shared__ float ws_[kMaxExperts];
  __shared__ int s_n;
  const int64_t t = blockIdx.x;
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    int n = 0;
    for (int c = 0; c < E; c += 32) {
      const int e = c + lane;
      // both loads issued before the ballot, so they overlap
      const int r = e < E ? __ldg(slot_row + t * E + e) : -1;
      const float pw = e < E ? __ldg(probs + t * E + e) : 0.f;
      const unsigned b = __ballot_sync(0xffffffffu, r >= 0);
      if (r >= 0) {
        const int p = n + __popc(b & ((1u << lane) - 1u));
        rows[p] = r;
        ws_[p] = pw;
      }
      n += __popc(b);
    }
    if (lane == 0) s_n = n;
  }
  __syncthreads();
  const int n = s_n;
  const int nv = d / 8;
  for (int v = threadIdx.x; v < nv; v += blockDim.x) {
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.f;
    for (int j0 = 0; j0 < n; j0 += 8) {
      Raw8<T_> q[8];
#pragma unroll
      for (int jj = 0; jj < 8; ++jj) {
        const int j = j0 + jj < n ? j0 + jj : n - 1;  // past the list: re-read the last row, skipped below
        q[jj].load(o_perm + static_cast<int64_t>(rows[j]) * d + v * 8);
      }
#pragma unroll
      for (int jj = 0; jj < 8; ++jj) {
        if (j0 + jj < n) {
          float o[8];
          q[jj].unpack(o);
          const float w = ws_[j0 + jj];
#pragma unroll
          for (int i = 0; i < 8; ++i) acc[i] = fmaf(w, o[i], acc[i]);
        }
      }
    }
    Vec8<T_> out;
#pragma unroll
    for (int i = 0; i < 8; ++i) out.v[i] = acc[i];
    out.store(y + t * d + v * 8);
  }
}

// The normalised value is formed in fp64 (sum of squares, square root, one
// reciprocal per row and a product per element), then rounded to fp32 and on
// to the output type: within an ulp of fp64 of an fp64 evaluation of the
// formula, so the layer input's rounding is decided as an exact computation
// decides it (short of values within ~1e-16 of a rounding boundary).
template <typename T_>
__global__ void __launch_bounds__(256)
    rmsnorm_kernel(const float* __restrict__ resid, const float* __restrict__ weight, double eps, int d,
                   T_* __restrict__ out) {
  pdl_trigger();
  pdl_wait();  // reads and writes buffers an earlier kernel of the layer uses
  __shared__ double red[8];
  const int64_t t = blockIdx.x;
  const float* r = resid + t * d;
  double ss = 0.0;
  for (int i = threadIdx.x; i < d; i += blockDim.x) ss = fma(static_cast<double>(r[i]), static_cast<double>(r[i]), ss);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  if (threadIdx.x == 0) {
    double s = 0.0;
    for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) s += red[w];
    red[0] = s;
  }
  __syncthreads();
  const double inv = 1.0 / sqrt(red[0] / static_cast<double>(d) + eps);
  for (int i = threadIdx.x; i < d; i += blockDim.x) {
    double v = static_cast<double>(r[i]) * inv;
    if (weight != nullptr) v *= static_cast<double>(weight[i]);
    out[t * d + i] = from_f32<T_>(static_cast<float>(v));
  }
}

__device__ __forceinline__ void store4(float* p, const float (&o)[4]) {
  *reinterpret_cast<float4*>(p) = make_float4(o[0], o[1], o[2], o[3]);
}
__device__ __forceinline__ void store4(__nv_bfloat16* p, const __nv_bfloat16 (&o)[4]) {
  __nv_bfloat162 lo, hi;
  lo.x = o[0];
  lo.y = o[1];
  hi.x = o[2];
  hi.y = o[3];
  uint2 u;
  u.x = *reinterpret_cast<const uint32_t*>(&lo);
  u.y = *reinterpret_cast<const uint32_t*>(&hi);
  *reinterpret_cast<uint2*>(p) = u;
}

// The same values for rows of up to 2048 elements, 64 threads per row: thread
// p holds elements 4p + 256j (j < 8) in registers, so the row is read once
// with 16-byte loads. The sum of squares runs over each thread's elements in
// order, then a fixed butterfly within each warp, then warp 0's sum plus warp
// 1's.
constexpr int kNormRowsPerCta = 4;

template <typename T_>
__global__ void __launch_bounds__(64 * kNormRowsPerCta)
    rmsnorm_rows_kernel(const float* __restrict__ resid, const float* __restrict__ weight, double eps, int d,
                        int64_t T, T_* __restrict__ out) {
  pdl_trigger();
  pdl_wait();  // reads and writes buffers an earlier kernel of the layer uses
  constexpr int kV = 8;  // float4 per thread: d <= 256 * kV
  __shared__ double part[kNormRowsPerCta][2];
  const int p = threadIdx.x & 63, row = threadIdx.x >> 6;
  const int64_t t = static_cast<int64_t>(blockIdx.x) * kNormRowsPerCta + row;
  const bool live = t < T;
  const float4* r = reinterpret_cast<const float4*>(resid + t * d);
  const int nv = d / 4;
  float4 v[kV];
#pragma unroll
  for (int j = 0; j < kV; ++j)
    if (live && p + 64 * j < nv) v[j] = __ldg(r + p + 64 * j);
  double ss = 0.0;
#pragma unroll
  for (int j = 0; j < kV; ++j) {
    if (live && p + 64 * j < nv) {
      ss = fma(static_cast<double>(v[j].x), static_cast<double>(v[j].x), ss);
      ss = fma(static_cast<double>(v[j].y), static_cast<double>(v[j].y), ss);
      ss = fma(static_cast<double>(v[j].z), static_cast<double>(v[j].z), ss);
      ss = fma(static_cast<double>(v[j].w), static_cast<double>(v[j].w), ss);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if ((p & 31) == 0) part[row][p >> 5] = ss;
  __syncthreads();
  if (!live) return;
  const double inv = 1.0 / sqrt((part[row][0] + part[row][1]) / static_cast<double>(d) + eps);
#pragma unroll
  for (int j = 0; j < kV; ++j) {
    const int i = 4 * (p + 64 * j);
    if (i < d) {
      const float a[4] = {v[j].x, v[j].y, v[j].z, v[j].w};
      T_ o[4];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        double x = static_cast<double>(a[c]) * inv;
        if (weight != nullptr) x *= static_cast<double>(weight[i + c]);
        o[c] = from_f32<T_>(static_cast<float>(x));
      }
      store4(out + t * d + i, o);
    }
  }
}

}  // namespace

cudaError_t launch_combine_ec(const Shape& s, const void* o_perm, const int32_t* slot_row, const float* probs,
                              void* y, cudaStream_t st) {
  if (s.fp32) return cudaErrorInvalidValue;  // expert choice runs on the bf16 tensor-core router
  // at least one whole warp: warp 0 compacts the expert list with ballots
  const int threads = s.d / 8 < 32 ? 32 : (s.d / 8 < 256 ? s.d / 8 : 256);
  combine_ec_kernel<__nv_bfloat16><<<static_cast<unsigned>(s.T), threads, 0, st>>>(
      static_cast<const __nv_bfloat16*>(o_perm), slot_row, probs, s.T, s.d, s.E, static_cast<__nv_bfloat16*>(y));
  return cudaGetLastError();
}

namespace {
template <typename OT, typename T_>
cudaError_t combine_typed(const Shape& s, const void* o_perm, const int32_t* inv_perm, const float* wts, void* y,
                          float* resid, cudaStream_t st) {
  const int threads = s.d / 8 < 256 ? s.d / 8 : 256;
  const unsigned grid = static_cast<unsigned>(s.T);
  const OT* o = static_cast<const OT*>(o_perm);
  if (resid != nullptr)
    launch_dependent(combine_kernel<OT, T_, true>, dim3(grid), dim3(threads), 0, st, nullptr, 0, o, inv_perm, wts, s.T, s.d, s.k, nullptr, resid);
  else
    launch_dependent(combine_kernel<OT, T_, false>, dim3(grid), dim3(threads), 0, st, nullptr, 0, o, inv_perm, wts, s.T, s.d, s.k, static_cast<T_*>(y),
                                                           nullptr);
  return cudaGetLastError();
}
}  // namespace

cudaError_t launch_combine(const Shape& s, const void* o_perm, bool o32, const int32_t* inv_perm, const float* wts,
                           void* y, float* resid, cudaStream_t st) {
  if (s.fp32) return combine_typed<float, float>(s, o_perm, inv_perm, wts, y, resid, st);
  if (o32) return combine_typed<float, __nv_bfloat16>(s, o_perm, inv_perm, wts, y, resid, st);
  return combine_typed<__nv_bfloat16, __nv_bfloat16>(s, o_perm, inv_perm, wts, y, resid, st);
}

cudaError_t launch_rmsnorm(const Shape& s, const float* resid, const float* weight, double eps, void* out,
                           cudaStream_t st) {
  if (s.d <= 2048) {  // 64 threads per row, the row in registers
    const unsigned grid = static_cast<unsigned>((s.T + kNormRowsPerCta - 1) / kNormRowsPerCta);
    if (s.fp32)
      launch_dependent(rmsnorm_rows_kernel<float>, dim3(grid), dim3(64 * kNormRowsPerCta), 0, st, nullptr, 0, resid,
                       weight, eps, s.d, s.T, static_cast<float*>(out));
    else
      launch_dependent(rmsnorm_rows_kernel<__nv_bfloat16>, dim3(grid), dim3(64 * kNormRowsPerCta), 0, st, nullptr, 0,
                       resid, weight, eps, s.d, s.T, static_cast<__nv_bfloat16*>(out));
    return cudaGetLastError();
  }
  const unsigned grid = static_cast<unsigned>(s.T);
  if (s.fp32)
    launch_dependent(rmsnorm_kernel<float>, dim3(grid), dim3(256), 0, st, nullptr, 0, resid, weight, eps, s.d, static_cast<float*>(out));
  else
    launch_dependent(rmsnorm_kernel<__nv_bfloat16>, dim3(grid), dim3(256), 0, st, nullptr, 0, resid, weight, eps, s.d, static_cast<__nv_bfloat16*>(out));
  return cudaGetLastError();
}

}  // namespace moe
