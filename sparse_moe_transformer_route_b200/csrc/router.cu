// Router: logits, softmax over all experts, top-k without renormalisation,
// per-expert counts and the two router losses, in one kernel.
//
// "Mixture-of-experts LLMs from scratch with OLMoE", section 2 (softmax_topk:
// softmax over all experts, then the k largest probabilities, unrenormalised —
// OLMoE's norm_topk_prob is False, section 3) and section 3 MoE.forward (scores
// in fp32, an optional per-expert offset before the softmax). "OLMoE Guide",
// "Router Mechanics & Loss Formulations": f_i = count_i / (T k), P_i = mean_t p,
// L_lb = E sum_i f_i P_i, L_z = mean_t lse_t^2.
//
// Each CTA takes 16 tokens. The dot products h_t,e = <x_t, W_r,e> are formed
// from exact products of the inputs accumulated in fp64 (a warp per expert,
// lanes strided over d, then a fixed shuffle tree), so the top-k order is the
// order of the exact logits except for gaps below ~1e-15 relative; the
// probabilities and the log-normaliser are then taken in fp32. Ties go to the
// lower expert index. Per-CTA partial sums (counts, sum_t p_t,e, sum_t lse_t^2)
// are reduced by the last CTA to finish, in CTA order, so the losses are
// deterministic.
#include <cfloat>
#include <cmath>

#include "moe_internal.h"
#include "sm100.cuh"

namespace moe {
namespace {

constexpr int kThreads = 256;
constexpr int kTok = kRouterTokensPerCta;

template <typename Tin>
__global__ void __launch_bounds__(kThreads) router_kernel(
    const Tin* __restrict__ x, const Tin* __restrict__ w_router, const float* __restrict__ bias, int64_t T, int d,
    int E, int k, int32_t* __restrict__ idx_out, float* __restrict__ w_out, float* __restrict__ probs,
    float* __restrict__ lse_out, int32_t* __restrict__ counts_part, float* __restrict__ psum_part,
    double* __restrict__ zsum_part, int32_t* __restrict__ counts_ws, int32_t* __restrict__ counts_user,
    float* __restrict__ losses_ws, float* __restrict__ losses_user, int32_t* __restrict__ ticket, int renorm) {
  pdl_trigger();
  pdl_wait();  // reads and writes buffers an earlier kernel of the layer uses
  extern __shared__ __align__(16) unsigned char smem[];
  Tin* xs = reinterpret_cast<Tin*>(smem);                                            // [kTok][d]
  double* logit = reinterpret_cast<double*>(smem + static_cast<size_t>(kTok) * d * sizeof(Tin));  // [kTok][E]
  float* ps = reinterpret_cast<float*>(logit + kTok * E);                           // [kTok][E]
  float* lses = ps + kTok * E;                                                       // [kTok]
  int* cnt = reinterpret_cast<int*>(lses + kTok);                                    // [E]
  __shared__ int s_last;
  __shared__ double s_psum[kMaxExperts];

  const int64_t t0 = static_cast<int64_t>(blockIdx.x) * kTok;
  const int ntok = static_cast<int>((T - t0) < kTok ? (T - t0) : kTok);
  {
    constexpr int kVec = 16 / sizeof(Tin);
    const int nv = ntok * d / kVec;
    const uint4* src = reinterpret_cast<const uint4*>(x + t0 * d);
    uint4* dst = reinterpret_cast<uint4*>(xs);
    for (int i = threadIdx.x; i < nv; i += blockDim.x) dst[i] = src[i];
    // rows past the last token read as zero
    for (int i = ntok * d / kVec + threadIdx.x; i < kTok * d / kVec; i += blockDim.x) dst[i] = make_uint4(0, 0, 0, 0);
  }
  for (int e = threadIdx.x; e < E; e += blockDim.x) cnt[e] = 0;
  __syncthreads();

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarps = blockDim.x >> 5;

  // ---- logits: a warp per expert, lanes strided over d, fp64 accumulation
  for (int e = warp; e < E; e += nwarps) {
    double acc[kTok];
#pragma unroll
    for (int t = 0; t < kTok; ++t) acc[t] = 0.0;
    const Tin* wrow = w_router + static_cast<size_t>(e) * d;
    for (int i = lane; i < d; i += 32) {
      const double wv = static_cast<double>(to_f32(wrow[i]));
#pragma unroll
      for (int t = 0; t < kTok; ++t) acc[t] = fma(wv, static_cast<double>(to_f32(xs[t * d + i])), acc[t]);
    }
#pragma unroll
    for (int t = 0; t < kTok; ++t) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc[t] += __shfl_xor_sync(0xffffffffu, acc[t], o);
    }
    if (lane == 0) {
      const double b = (bias != nullptr) ? static_cast<double>(bias[e]) : 0.0;
      for (int t = 0; t < ntok; ++t) logit[t * E + e] = acc[t] + b;
    }
  }
  __syncthreads();

  // ---- softmax (fp32) and top-k (on the fp64 logits): a warp per token
  constexpr int Q = kMaxExperts / 32;
  for (int t = warp; t < ntok; t += nwarps) {
    double hv[Q];
    float m = -FLT_MAX;
#pragma unroll
    for (int q = 0; q < Q; ++q) {
      const int e = lane + 32 * q;
      hv[q] = (e < E) ? logit[t * E + e] : -static_cast<double>(INFINITY);
      if (e < E) m = fmaxf(m, static_cast<float>(hv[q]));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    float ex[Q];
    float s = 0.f;
#pragma unroll
    for (int q = 0; q < Q; ++q) {
      const int e = lane + 32 * q;
      ex[q] = (e < E) ? expf(static_cast<float>(hv[q]) - m) : 0.f;
      s += ex[q];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    float p[Q];
    const int64_t tg = t0 + t;
#pragma unroll
    for (int q = 0; q < Q; ++q) {
      const int e = lane + 32 * q;
      p[q] = ex[q] / s;
      if (e < E) {
        ps[t * E + e] = p[q];
        probs[tg * E + e] = p[q];
      }
    }
    const float lse = m + logf(s);

    uint32_t taken = 0;  // bit q: expert lane+32q already chosen
    float chosen_sum = 0.f;  // renormalised weights: the chosen probabilities' sum, in slot order
    for (int j = 0; j < k; ++j) {
      double bv = -static_cast<double>(INFINITY);
      int bi = 0x7fffffff;
#pragma unroll
      for (int q = 0; q < Q; ++q) {
        const int e = lane + 32 * q;
        if (e < E && !((taken >> q) & 1u) && (hv[q] > bv || (hv[q] == bv && e < bi))) {
          bv = hv[q];
          bi = e;
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const double ov = __shfl_xor_sync(0xffffffffu, bv, o);
        const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
        if (ov > bv || (ov == bv && oi < bi)) {
          bv = ov;
          bi = oi;
        }
      }
      if (bi >= E) bi = -1;  // only NaN logits left: recorded as an invalid choice
      const int qq = bi >> 5;
      float mine = 0.f;
#pragma unroll
      for (int q = 0; q < Q; ++q)
        if (q == qq) mine = p[q];
      const float pw = __shfl_sync(0xffffffffu, mine, bi & 31);
      if (bi >= 0 && lane == (bi & 31)) taken |= 1u << qq;
      if (bi >= 0) chosen_sum += pw;
      if (lane == 0) {
        idx_out[tg * k + j] = bi;
        w_out[tg * k + j] = (bi >= 0) ? pw : 0.f;
        if (bi >= 0) atomicAdd(&cnt[bi], 1);
      }
    }
    if (renorm && lane == 0 && chosen_sum > 0.f)
      for (int j = 0; j < k; ++j) w_out[tg * k + j] = w_out[tg * k + j] / chosen_sum;
    if (lane == 0) {
      lses[t] = lse;
      lse_out[tg] = lse;
    }
  }
  __syncthreads();

  // ---- per-CTA partials, fixed order
  const int cta = blockIdx.x;
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    float acc = 0.f;
    for (int t = 0; t < ntok; ++t) acc += ps[t * E + e];
    psum_part[static_cast<size_t>(cta) * E + e] = acc;
    counts_part[static_cast<size_t>(cta) * E + e] = cnt[e];
  }
  if (threadIdx.x == 0) {
    double z = 0.0;
    for (int t = 0; t < ntok; ++t) z += static_cast<double>(lses[t]) * lses[t];
    zsum_part[cta] = z;
  }
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) s_last = (atomicAdd(ticket, 1) == static_cast<int>(gridDim.x) - 1);
  __syncthreads();
  if (!s_last) return;

  // ---- the last CTA reduces the partials in CTA order
  __threadfence();
  const int nb = gridDim.x;
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int c = 0;
    double pe = 0.0;
    for (int b0 = 0; b0 < nb; b0 += 16) {  // batched so the L2 round trips overlap
      int cv[16];
      float pv[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        cv[i] = (b0 + i < nb) ? __ldcg(&counts_part[static_cast<size_t>(b0 + i) * E + e]) : 0;
        pv[i] = (b0 + i < nb) ? __ldcg(&psum_part[static_cast<size_t>(b0 + i) * E + e]) : 0.f;
      }
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        c += cv[i];
        pe += static_cast<double>(pv[i]);
      }
    }
    counts_ws[e] = c;
    if (counts_user != nullptr) counts_user[e] = c;
    cnt[e] = c;
    s_psum[e] = pe;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    double z = 0.0;
    for (int b0 = 0; b0 < nb; b0 += 16) {
      double zv[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) zv[i] = (b0 + i < nb) ? __ldcg(&zsum_part[b0 + i]) : 0.0;
#pragma unroll
      for (int i = 0; i < 16; ++i) z += zv[i];
    }
    const double Td = static_cast<double>(T);
    double lb = 0.0;
    for (int e = 0; e < E; ++e) lb += (static_cast<double>(cnt[e]) / (Td * k)) * (s_psum[e] / Td);
    lb *= E;
    const float l0 = static_cast<float>(lb), l1 = static_cast<float>(z / Td);
    losses_ws[0] = l0;
    losses_ws[1] = l1;
    if (losses_user != nullptr) {
      losses_user[0] = l0;
      losses_user[1] = l1;
    }
    *ticket = 0;
  }
}

template <typename Tin>
cudaError_t run(const Shape& s, const void* x, const void* w_router, const float* bias, int32_t* idx, float* wts,
                int32_t* counts, float* losses, void* ws, const Workspace& L, cudaStream_t st) {
  const size_t smem = static_cast<size_t>(kTok) * s.d * sizeof(Tin) + static_cast<size_t>(kTok) * s.E * 12 +
                      kTok * 4 + s.E * 4;
  static std::atomic<size_t> smem_set[kMaxDevices];
  if (smem > 48 * 1024) {
    cudaError_t e = raise_smem_limit(reinterpret_cast<const void*>(router_kernel<Tin>), smem, smem_set);
    if (e != cudaSuccess) return e;
  }
  // ctrl[1] is zero between calls (moe_workspace_init, then each launch's last CTA)
  int32_t* ctrl = at<int32_t>(ws, L.ctrl);
  const int grid = static_cast<int>(s.router_ctas());
  launch_dependent(router_kernel<Tin>, dim3(grid), dim3(kThreads), smem, st, nullptr, 0, 
      static_cast<const Tin*>(x), static_cast<const Tin*>(w_router), bias, s.T, s.d, s.E, s.k, idx, wts,
      at<float>(ws, L.probs), at<float>(ws, L.lse), at<int32_t>(ws, L.counts_part), at<float>(ws, L.psum_part),
      at<double>(ws, L.zsum_part), at<int32_t>(ws, L.counts), counts, at<float>(ws, L.losses), losses, ctrl + 1,
      s.renorm ? 1 : 0);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_router(const Shape& s, const void* x, const void* w_router, const float* bias, int32_t* idx,
                          float* wts, int32_t* counts, float* losses, void* ws, const Workspace& L,
                          cudaStream_t st) {
  if (s.fp32) return run<float>(s, x, w_router, bias, idx, wts, counts, losses, ws, L, st);
  return run<__nv_bfloat16>(s, x, w_router, bias, idx, wts, counts, losses, ws, L, st);
}

}  // namespace moe

// ---------------------------------------------------------------------------
// The router on library-owned scratch: moe_route_static.
//
// For callers that cannot hand the library a workspace: code whose device
// memory is owned and planned by a host framework or serving runtime (it may
// not call cudaMalloc itself, and has no arena slot for an extra buffer), or a
// latency-critical loop that must not allocate because cudaMalloc synchronises
// the device. The router's scratch (per-CTA partial sums, the completion
// counter, the saved probabilities) then lives in one file-scope device array
// that every device loading this library holds until the process exits.
//
// Host code must not pass the array's name to a kernel: on the host it is only
// a stand-in symbol, not a device address. Its device address is looked up
// once per device, with that device current, on the first call made on that
// device; make that first call before any stream capture. Every call uses the
// same array and finds the previous call's contents in it: the completion
// counter is cleared on the stream before each launch, and everything else is
// overwritten before it is read. Calls whose executions overlap on the GPU
// (other streams, other host threads) race on the array.
#include <mutex>

namespace moe {
namespace {

constexpr size_t kStaticScratchBytes = static_cast<size_t>(MOE_ROUTE_STATIC_SCRATCH_BYTES);
static __device__ __align__(256) unsigned char g_route_scratch[kStaticScratchBytes];

struct StaticLayout {
  size_t ticket, counts_part, psum_part, zsum_part, counts, losses, probs, lse, total;
};

StaticLayout static_layout(const Shape& s) {
  StaticLayout L{};
  size_t o = 0;
  auto take = [&](size_t bytes) {
    const size_t at_ = o;
    o = (o + bytes + 255) / 256 * 256;
    return at_;
  };
  const size_t ctas = static_cast<size_t>(s.router_ctas());
  const size_t T = static_cast<size_t>(s.T), E = static_cast<size_t>(s.E);
  L.ticket = take(sizeof(int32_t));
  L.counts_part = take(ctas * E * sizeof(int32_t));
  L.psum_part = take(ctas * E * sizeof(float));
  L.zsum_part = take(ctas * sizeof(double));
  L.counts = take(E * sizeof(int32_t));
  L.losses = take(2 * sizeof(float));
  L.probs = take(T * E * sizeof(float));
  L.lse = take(T * sizeof(float));
  L.total = o;
  return L;
}

// The array's device address belongs to the context it was looked up in; a
// device reset (or any new primary context) loads the module afresh, so the
// address is kept together with the context and looked up again when the
// current context is another one.
struct ScratchAddr {
  CUcontext ctx = nullptr;
  unsigned char* addr = nullptr;
};
std::mutex g_scratch_mu;
ScratchAddr g_scratch[kMaxDevices];

using CtxGetCurrent = CUresult (*)(CUcontext*);

CtxGetCurrent ctx_get_current() {
  static CtxGetCurrent fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &p, 12000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<CtxGetCurrent>(p);
    return static_cast<CtxGetCurrent>(nullptr);
  }();
  return fn;
}

// Device address of g_route_scratch in the current device's current context.
cudaError_t static_scratch(unsigned char** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  const CtxGetCurrent get_ctx = ctx_get_current();
  if (get_ctx == nullptr) return cudaErrorNotSupported;
  CUcontext ctx = nullptr;
  if (get_ctx(&ctx) != CUDA_SUCCESS) return cudaErrorUnknown;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  ScratchAddr& c = g_scratch[dev];
  if (c.addr == nullptr || ctx == nullptr || c.ctx != ctx) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_route_scratch);  // makes the primary context current if none was
    if (e != cudaSuccess) return e;
    if (get_ctx(&ctx) != CUDA_SUCCESS) return cudaErrorUnknown;
    c.ctx = ctx;
    c.addr = static_cast<unsigned char*>(p);
  }
  *out = c.addr;
  return cudaSuccess;
}

template <typename Tin>
cudaError_t run_static(const Shape& s, const void* x, const void* w_router, const float* bias, int32_t* idx,
                       float* wts, int32_t* counts, float* losses, unsigned char* scratch, const StaticLayout& L,
                       cudaStream_t st) {
  const size_t smem = static_cast<size_t>(kTok) * s.d * sizeof(Tin) + static_cast<size_t>(kTok) * s.E * 12 +
                      kTok * 4 + s.E * 4;
  static std::atomic<size_t> smem_set[moe::kMaxDevices];
  if (smem > 48 * 1024) {
    cudaError_t e = raise_smem_limit(reinterpret_cast<const void*>(router_kernel<Tin>), smem, smem_set);
    if (e != cudaSuccess) return e;
  }
  int32_t* ticket = reinterpret_cast<int32_t*>(scratch + L.ticket);
  cudaError_t e = cudaMemsetAsync(ticket, 0, sizeof(int32_t), st);
  if (e != cudaSuccess) return e;
  const int grid = static_cast<int>(s.router_ctas());
  launch_dependent(router_kernel<Tin>, dim3(grid), dim3(kThreads), smem, st, nullptr, 0, 
      static_cast<const Tin*>(x), static_cast<const Tin*>(w_router), bias, s.T, s.d, s.E, s.k, idx, wts,
      reinterpret_cast<float*>(scratch + L.probs), reinterpret_cast<float*>(scratch + L.lse),
      reinterpret_cast<int32_t*>(scratch + L.counts_part), reinterpret_cast<float*>(scratch + L.psum_part),
      reinterpret_cast<double*>(scratch + L.zsum_part), reinterpret_cast<int32_t*>(scratch + L.counts), counts,
      reinterpret_cast<float*>(scratch + L.losses), losses, ticket, s.renorm ? 1 : 0);
  return cudaGetLastError();
}

}  // namespace
}  // namespace moe

extern "C" moe_status moe_route_static(const moe_config* cfg, const void* x, const void* w_router,
                                       const float* router_bias, int32_t* topk_idx, float* topk_w, int32_t* counts,
                                       float* losses, cudaStream_t stream) {
  using namespace moe;
  if (cfg == nullptr) return MOE_ERR_INVALID_ARG;
  Shape s;
  if (!make_shape(cfg, &s)) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (x == nullptr || w_router == nullptr || topk_idx == nullptr || topk_w == nullptr ||
      (reinterpret_cast<uintptr_t>(x) & 15u) != 0 || (reinterpret_cast<uintptr_t>(w_router) & 15u) != 0)
    return MOE_ERR_INVALID_ARG;
  const StaticLayout L = static_layout(s);
  if (L.total > kStaticScratchBytes) return MOE_ERR_WORKSPACE_TOO_SMALL;
  int dev = -1, major = 0, minor = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess || major != 10 ||
      minor != 0)
    return MOE_ERR_NO_DEVICE;
  unsigned char* scratch = nullptr;
  if (static_scratch(&scratch) != cudaSuccess) return MOE_ERR_CUDA;
  const cudaError_t e =
      s.fp32 ? run_static<float>(s, x, w_router, router_bias, topk_idx, topk_w, counts, losses, scratch, L, stream)
             : run_static<__nv_bfloat16>(s, x, w_router, router_bias, topk_idx, topk_w, counts, losses, scratch, L,
                                         stream);
  return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
