// The C ABI declared in include/moe.h: argument validation, the workspace
// layout, and the sequence of kernel launches for each entry point. Nothing here
// computes on the host; every step of the layer runs in the kernels of this
// directory.
#include <cstring>

#include "moe_internal.h"

namespace moe {

namespace {
constexpr size_t kAlign = 1024;
size_t up(size_t v, size_t a) { return (v + a - 1) / a * a; }

struct DeviceInfo {
  int id = -1;
  int sms = 0;
  bool sm100 = false;
};

bool current_device(DeviceInfo* out) {
  static DeviceInfo cache[64];
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
  DeviceInfo& c = cache[dev];
  if (c.id != dev) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return false;
    if (cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) return false;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return false;
    c.sms = sms;
    c.sm100 = (major == 10 && minor == 0);
    c.id = dev;
  }
  *out = c;
  return true;
}
}  // namespace

cudaError_t raise_smem_limit(const void* func, size_t bytes, std::atomic<size_t>* cache) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) dev = -1;
  if (dev >= 0 && dev < kMaxDevices && cache[dev].load() >= bytes) return cudaSuccess;
  const cudaError_t e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes));
  if (e == cudaSuccess && dev >= 0 && dev < kMaxDevices) {
    size_t cur = cache[dev].load();
    while (cur < bytes && !cache[dev].compare_exchange_weak(cur, bytes)) {
    }
  }
  return e;
}

int device_sm_count() {
  DeviceInfo d;
  return current_device(&d) ? d.sms : 148;
}

bool make_shape(const moe_config* cfg, Shape* s) {
  if (cfg == nullptr) return false;
  if (cfg->dtype != MOE_BF16 && cfg->dtype != MOE_FP32) return false;
  if (cfg->grad_dtype != MOE_BF16 && cfg->grad_dtype != MOE_FP32) return false;
  if (cfg->router_mode != MOE_ROUTER_SOFTMAX_TOPK && cfg->router_mode != MOE_ROUTER_RENORM) return false;
  const bool fp32 = cfg->dtype == MOE_FP32;
  const int dmax = fp32 ? 2048 : 4096;
  if (cfg->T < 1 || cfg->T > (int64_t(1) << 24)) return false;
  if (cfg->d_model < 128 || cfg->d_model > dmax || cfg->d_model % 128 != 0) return false;
  if (cfg->d_ff < 128 || cfg->d_ff > 4096 || cfg->d_ff % 128 != 0) return false;
  if (cfg->n_experts < 1 || cfg->n_experts > kMaxExperts) return false;
  if (cfg->top_k < 1 || cfg->top_k > kMaxTopK || cfg->top_k > cfg->n_experts) return false;
  s->T = cfg->T;
  s->d = cfg->d_model;
  s->E = cfg->n_experts;
  s->k = cfg->top_k;
  s->f = cfg->d_ff;
  s->fp32 = fp32;
  s->grad32 = fp32 || cfg->grad_dtype == MOE_FP32;
  s->renorm = cfg->router_mode == MOE_ROUTER_RENORM;
  s->esize = fp32 ? 4 : 2;
  s->P = static_cast<int64_t>(up(static_cast<size_t>(cfg->T * cfg->top_k + int64_t(cfg->n_experts) * (kRowAlign - 1)),
                                 kRowAlign));
  return true;
}

Workspace layout(const Shape& s) {
  Workspace L{};
  size_t o = 0;
  auto take = [&](size_t bytes) {
    const size_t at_ = o;
    o = up(o + bytes, kAlign);
    return at_;
  };
  const size_t T = static_cast<size_t>(s.T), E = s.E, k = s.k, P = static_cast<size_t>(s.P);
  const size_t ctas = static_cast<size_t>(s.router_ctas()), chunks = static_cast<size_t>(s.chunks());
  L.ctrl = take(256);
  L.counts_part = take(ctas * E * 4);
  L.psum_part = take(ctas * E * 4);
  L.zsum_part = take(ctas * 8);
  L.counts = take(E * 4);
  L.losses = take(8);
  L.probs = take(T * E * 4);
  L.lse = take(T * 4);
  L.idx = take(T * k * 4);
  L.wts = take(T * k * 4);
  L.local_rank = take(T * k * 4);
  L.chunk_count = take(chunks * E * 4);
  L.chunk_base = take(chunks * E * 4);
  L.offsets = take((E + 1) * 4);
  L.group_start = take((E + 1) * 4);
  L.perm = take(T * k * 4);
  L.inv_perm = take(T * k * 4);
  L.row_pair = take(P * 4);
  L.x_perm = take(P * s.d * s.esize);
  L.h = take(P * s.f * s.esize);
  L.o_perm = take(P * s.d * s.esize);
  L.x_dev = take(T * s.d * s.esize);
  L.y_dev = take(T * s.d * s.esize);
  L.ec_sel = take(P * 4);
  L.ec_gate = take(P * 4);
  L.ec_slot = take(T * E * 4);
  L.fwd_bytes = o;
  L.preact = take(P * 2 * s.f * 4);
  L.o32 = take(P * s.d * 4);
  L.dw = take(T * k * 4);
  L.dh = take(T * E * 4);
  L.dout = take(P * s.d * s.esize);
  L.dab = take(P * 2 * s.f * s.esize);
  L.dx_perm = take(P * s.d * s.esize);
  L.wr_part = take(router_wgrad_partial_bytes(s));
  L.bwd_bytes = o;
  return L;
}

}  // namespace moe

using namespace moe;

namespace {

struct Ctx {
  Shape s;
  Workspace L;
};

moe_status prepare(const moe_config* cfg, void* ws, size_t ws_bytes, bool backward, Ctx* c) {
  if (cfg == nullptr) return MOE_ERR_INVALID_ARG;
  if (!make_shape(cfg, &c->s)) return MOE_ERR_UNSUPPORTED_SHAPE;
  c->L = layout(c->s);
  if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return MOE_ERR_INVALID_ARG;
  if (ws_bytes < (backward ? c->L.bwd_bytes : c->L.fwd_bytes)) return MOE_ERR_WORKSPACE_TOO_SMALL;
  DeviceInfo d;
  if (!current_device(&d) || !d.sm100) return MOE_ERR_NO_DEVICE;
  return MOE_OK;
}

moe_status device_ready() {
  DeviceInfo d;
  if (!current_device(&d) || !d.sm100) return MOE_ERR_NO_DEVICE;
  return MOE_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

#define MOE_TRY(expr)                                 \
  do {                                                \
    if ((expr) != cudaSuccess) return MOE_ERR_CUDA;   \
  } while (0)

thread_local cudaEvent_t g_stage_events[MOE_STAGE_EVENTS];
thread_local bool g_stage_armed = false;

struct StageMarks {
  bool on;
  cudaStream_t st;
  explicit StageMarks(cudaStream_t s) : on(g_stage_armed), st(s) { g_stage_armed = false; }
  cudaError_t mark(int i) const { return on ? cudaEventRecord(g_stage_events[i], st) : cudaSuccess; }
};

moe_status forward_impl(const Ctx& c, const void* x, const void* w_router, const float* bias, const void* w_gate_up,
                        const void* w_down, void* y, float* losses, float* resid, int32_t* topk_idx, float* topk_w,
                        bool save, void* ws, cudaStream_t st, int32_t* counts = nullptr) {
  const Shape& s = c.s;
  const Workspace& L = c.L;
  int32_t* status = at<int32_t>(ws, L.ctrl);
  int32_t* idx = at<int32_t>(ws, L.idx);
  float* wts = at<float>(ws, L.wts);
  int32_t* gs = at<int32_t>(ws, L.group_start);
  int32_t* off = at<int32_t>(ws, L.offsets);
  void* x_perm = at<void>(ws, L.x_perm);
  const StageMarks marks(st);
  MOE_TRY(marks.mark(0));
  if (!save && resid == nullptr && s.T <= kDecodeAutoTokens && decode_supported(s)) {
    // a decode-sized batch: the whole layer in one kernel (every stage mark after it)
    MOE_TRY(launch_decode_layer(s, x, nullptr, 0.0, w_router, bias, w_gate_up, w_down, y, topk_idx, topk_w, counts,
                                losses, ws, L, st));
    for (int i = 1; i <= 5; ++i) MOE_TRY(marks.mark(i));
    return MOE_OK;
  }
  if (router_tc_supported(s)) {
    // the tensor-core router also leaves the dispatch ranking in ws
    MOE_TRY(launch_router_tc(s, x, w_router, bias, idx, wts, counts, losses, ws, L, st));
    MOE_TRY(marks.mark(1));
    MOE_TRY(launch_permute(s, idx, x, at<int32_t>(ws, L.perm), at<int32_t>(ws, L.inv_perm), x_perm, ws, L, save, st));
  } else {
    MOE_TRY(launch_router(s, x, w_router, bias, idx, wts, counts, losses, ws, L, st));
    MOE_TRY(marks.mark(1));
    MOE_TRY(launch_dispatch_impl(s, idx, x, nullptr, at<int32_t>(ws, L.perm), at<int32_t>(ws, L.inv_perm), nullptr,
                                 x_perm, ws, L, save, st));
  }
  MOE_TRY(marks.mark(2));
  MOE_TRY(launch_gate_up(s, x_perm, gs, off, w_gate_up, at<void>(ws, L.h), save ? at<void>(ws, L.preact) : nullptr,
                         status, st));
  MOE_TRY(marks.mark(3));
  // Kept for the backward, the expert outputs stay in fp32: the router's
  // gradient dw = <dy, o> reads them and no contraction does.
  void* o_rows = save ? at<void>(ws, L.o32) : at<void>(ws, L.o_perm);
  MOE_TRY(launch_down(s, at<void>(ws, L.h), gs, off, w_down, o_rows, save, status, st));
  MOE_TRY(marks.mark(4));
  MOE_TRY(launch_combine(s, o_rows, save, at<int32_t>(ws, L.inv_perm), wts, y, resid, st));
  MOE_TRY(marks.mark(5));
  const size_t nk = static_cast<size_t>(s.T) * s.k;
  if (topk_idx != nullptr) MOE_TRY(cudaMemcpyAsync(topk_idx, idx, nk * 4, cudaMemcpyDeviceToDevice, st));
  if (topk_w != nullptr) MOE_TRY(cudaMemcpyAsync(topk_w, wts, nk * 4, cudaMemcpyDeviceToDevice, st));
  return MOE_OK;
}

// Checks shared by the expert-choice entry points; *C receives the capacity.
moe_status ec_prepare(const moe_config* cfg, int64_t capacity, void* ws, size_t ws_bytes, Ctx* c, int64_t* C) {
  const moe_status r = prepare(cfg, ws, ws_bytes, false, c);
  if (r != MOE_OK) return r;
  if (!router_tc_supported(c->s) || c->s.renorm) return MOE_ERR_UNSUPPORTED_SHAPE;
  *C = capacity > 0 ? capacity : ec_default_capacity(c->s);
  if (capacity < 0 || !ec_capacity_ok(c->s, *C)) return MOE_ERR_INVALID_ARG;
  return MOE_OK;
}

}  // namespace

extern "C" {

const char* moe_status_string(int32_t status) {
  switch (status) {
    case MOE_OK: return "MOE_OK";
    case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG: null, misaligned or out-of-range argument";
    case MOE_ERR_UNSUPPORTED_SHAPE: return "MOE_ERR_UNSUPPORTED_SHAPE: shape outside the supported set";
    case MOE_ERR_WORKSPACE_TOO_SMALL: return "MOE_ERR_WORKSPACE_TOO_SMALL: workspace smaller than moe_workspace_bytes";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA: a CUDA call or kernel launch failed";
    case MOE_ERR_DEVICE_CHECK: return "MOE_ERR_DEVICE_CHECK: a kernel recorded a failed invariant";
    case MOE_ERR_NO_DEVICE: return "MOE_ERR_NO_DEVICE: the current device is not an sm_100 GPU";
    default: return "unknown moe_status";
  }
}

int32_t moe_abi_version(void) { return MOE_ABI_VERSION; }

moe_status moe_check_config(const moe_config* cfg) {
  if (cfg == nullptr) return MOE_ERR_INVALID_ARG;
  Shape s;
  return make_shape(cfg, &s) ? MOE_OK : MOE_ERR_UNSUPPORTED_SHAPE;
}

int64_t moe_padded_rows(const moe_config* cfg) {
  Shape s;
  return make_shape(cfg, &s) ? s.P : -1;
}

size_t moe_workspace_bytes(const moe_config* cfg, int32_t for_backward) {
  Shape s;
  if (!make_shape(cfg, &s)) return 0;
  const Workspace L = layout(s);
  return for_backward ? L.bwd_bytes : L.fwd_bytes;
}

moe_status moe_workspace_init(void* ws, cudaStream_t stream) {
  if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return MOE_ERR_INVALID_ARG;
  MOE_TRY(cudaMemsetAsync(ws, 0, 256, stream));
  return MOE_OK;
}

moe_status moe_route(const moe_config* cfg, const void* x, const void* w_router, const float* router_bias,
                     int32_t* topk_idx, float* topk_w, int32_t* counts, float* losses, void* ws, size_t ws_bytes,
                     cudaStream_t stream) {
  Ctx c;
  moe_status r = prepare(cfg, ws, ws_bytes, false, &c);
  if (r != MOE_OK) return r;
  if (x == nullptr || w_router == nullptr || topk_idx == nullptr || topk_w == nullptr || !aligned16(x) ||
      !aligned16(w_router))
    return MOE_ERR_INVALID_ARG;
  if (router_tc_supported(c.s))
    MOE_TRY(launch_router_tc(c.s, x, w_router, router_bias, topk_idx, topk_w, counts, losses, ws, c.L, stream));
  else
    MOE_TRY(launch_router(c.s, x, w_router, router_bias, topk_idx, topk_w, counts, losses, ws, c.L, stream));
  return MOE_OK;
}

moe_status moe_dispatch(const moe_config* cfg, const int32_t* topk_idx, const void* x, int32_t* offsets,
                        int32_t* perm, int32_t* inv_perm, int32_t* group_start, void* x_perm, void* ws,
                        size_t ws_bytes, cudaStream_t stream) {
  Ctx c;
  moe_status r = prepare(cfg, ws, ws_bytes, false, &c);
  if (r != MOE_OK) return r;
  if (topk_idx == nullptr || x == nullptr || offsets == nullptr || perm == nullptr || inv_perm == nullptr ||
      group_start == nullptr || x_perm == nullptr || !aligned16(x) || !aligned16(x_perm))
    return MOE_ERR_INVALID_ARG;
  MOE_TRY(launch_dispatch_impl(c.s, topk_idx, x, offsets, perm, inv_perm, group_start, x_perm, ws, c.L, true,
                               stream));
  return MOE_OK;
}

moe_status moe_expert_gate_up(const moe_config* cfg, const void* x_perm, const int32_t* group_start,
                              const int32_t* offsets, const void* w_gate_up, void* h, void* preact, void* ws,
                              size_t ws_bytes, cudaStream_t stream) {
  Ctx c;
  moe_status r = prepare(cfg, ws, ws_bytes, false, &c);
  if (r != MOE_OK) return r;
  if (x_perm == nullptr || group_start == nullptr || offsets == nullptr || w_gate_up == nullptr || h == nullptr ||
      !aligned16(x_perm) || !aligned16(w_gate_up) || !aligned16(h) || (preact != nullptr && !aligned16(preact)))
    return MOE_ERR_INVALID_ARG;
  MOE_TRY(launch_gate_up(c.s, x_perm, group_start, offsets, w_gate_up, h, preact, at<int32_t>(ws, c.L.ctrl),
                         stream));
  return MOE_OK;
}

moe_status moe_expert_down(const moe_config* cfg, const void* h, const int32_t* group_start, const int32_t* offsets,
                           const void* w_down, void* o_perm, void* ws, size_t ws_bytes, cudaStream_t stream) {
  Ctx c;
  moe_status r = prepare(cfg, ws, ws_bytes, false, &c);
  if (r != MOE_OK) return r;
  if (h == nullptr || group_start == nullptr || offsets == nullptr || w_down == nullptr || o_perm == nullptr ||
      !aligned16(h) || !aligned16(w_down) || !aligned16(o_perm))
    return MOE_ERR_INVALID_ARG;
  MOE_TRY(launch_down(c.s, h, group_start, offsets, w_down, o_perm, false, at<int32_t>(ws, c.L.ctrl), stream));
  return MOE_OK;
}

moe_status moe_expert_ffn(const moe_config* cfg, const void* x_perm, const int32_t* group_start,
                          const int32_t* offsets, const void* w_gate_up, const void* w_down, void* h, void* o_perm,
                          void* ws, size_t ws_bytes, cudaStream_t stream) {
  moe_status r = moe_expert_gate_up(cfg, x_perm, group_start, offsets, w_gate_up, h, nullptr, ws, ws_bytes, stream);
  if (r != MOE_OK) return r;
  return moe_expert_down(cfg, h, group_start, offsets, w_down, o_perm, ws, ws_bytes, stream);
}

moe_status moe_combine(const moe_config* cfg, const void* o_perm, const int32_t* inv_perm, const float* topk_w,
                       void* y, cudaStream_t stream) {
  Shape s;
  if (cfg == nullptr) return MOE_ERR_INVALID_ARG;
  if (!make_shape(cfg, &s)) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (o_perm == nullptr || inv_perm == nullptr || topk_w == nullptr || y == nullptr || !aligned16(o_perm) ||
      !aligned16(y))
    return MOE_ERR_INVALID_ARG;
  moe_status r = device_ready();
  if (r != MOE_OK) return r;
  MOE_TRY(launch_combine(s, o_perm, false, inv_perm, topk_w, y, nullptr, stream));
  return MOE_OK;
}

moe_status moe_combine_residual(const moe_config* cfg, const void* o_perm, const int32_t* inv_perm,
                                const float* topk_w, float* resid, cudaStream_t stream) {
  Shape s;
  if (cfg == nullptr) return MOE_ERR_INVALID_ARG;
  if (!make_shape(cfg, &s)) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (o_perm == nullptr || inv_perm == nullptr || topk_w == nullptr || resid == nullptr || !aligned16(o_perm) ||
      !aligned16(resid))
    return MOE_ERR_INVALID_ARG;
  moe_status r = device_ready();
  if (r != MOE_OK) return r;
  MOE_TRY(launch_combine(s, o_perm, false, inv_perm, topk_w, nullptr, resid, stream));
  return MOE_OK;
}

moe_status moe_forward(const moe_config* cfg, const void* x, const void* w_router, const float* router_bias,
                       const void* w_gate_up, const void* w_down, void* y, float* losses, int32_t* topk_idx,
                       float* topk_w, int32_t save_for_backward, void* ws, size_t ws_bytes, cudaStream_t stream) {
  Ctx c;
  moe_status r = prepare(cfg, ws, ws_bytes, save_for_backward != 0, &c);
  if (r != MOE_OK) return r;
  if (x == nullptr || w_router == nullptr || w_gate_up == nullptr || w_down == nullptr || y == nullptr ||
      !aligned16(x) || !aligned16(w_router) || !aligned16(w_gate_up) || !aligned16(w_down) || !aligned16(y))
    return MOE_ERR_INVALID_ARG;
  return forward_impl(c, x, w_router, router_bias, w_gate_up, w_down, y, losses, nullptr, topk_idx, topk_w,
                      save_for_backward != 0, ws, stream);
}

moe_status moe_forward_decode(const moe_config* cfg, const void* x, const void* w_router, const float* router_bias,
                              const void* w_gate_up, const void* w_down, void* y, float* losses, int32_t* topk_idx,
                              float* topk_w, void* ws, size_t ws_bytes, cudaStream_t stream) {
  Ctx c;
  moe_status r = prepare(cfg, ws, ws_bytes, false, &c);
  if (r != MOE_OK) return r;
  if (!decode_supported(c.s)) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (x == nullptr || w_router == nullptr || w_gate_up == nullptr || w_down == nullptr || y == nullptr ||
      !aligned16(x) || !aligned16(w_router) || !aligned16(w_gate_up) || !aligned16(w_down) || !aligned16(y))
    return MOE_ERR_INVALID_ARG;
  MOE_TRY(launch_decode_layer(c.s, x, nullptr, 0.0, w_router, router_bias, w_gate_up, w_down, y, topk_idx, topk_w,
                              nullptr, losses, ws, c.L, stream));
  return MOE_OK;
}

moe_status moe_forward_host_async(const moe_config* cfg, const void* x_host, const void* w_router,
                                  const float* router_bias, const void* w_gate_up, const void* w_down, void* y_host,
                                  float* losses_host, void* ws, size_t ws_bytes, cudaStream_t stream) {
  Ctx c;
  moe_status r = prepare(cfg, ws, ws_bytes, false, &c);
  if (r != MOE_OK) return r;
  if (x_host == nullptr || y_host == nullptr || w_router == nullptr || w_gate_up == nullptr || w_down == nullptr ||
      !aligned16(w_router) || !aligned16(w_gate_up) || !aligned16(w_down))
    return MOE_ERR_INVALID_ARG;
  const size_t bytes = static_cast<size_t>(c.s.T) * c.s.d * c.s.esize;
  void* xd = at<void>(ws, c.L.x_dev);
  void* yd = at<void>(ws, c.L.y_dev);
  MOE_TRY(cudaMemcpyAsync(xd, x_host, bytes, cudaMemcpyHostToDevice, stream));
  r = forward_impl(c, xd, w_router, router_bias, w_gate_up, w_down, yd, nullptr, nullptr, nullptr, nullptr, false, ws,
                   stream);
  if (r != MOE_OK) return r;
  MOE_TRY(cudaMemcpyAsync(y_host, yd, bytes, cudaMemcpyDeviceToHost, stream));
  if (losses_host != nullptr)
    MOE_TRY(cudaMemcpyAsync(losses_host, at<float>(ws, c.L.losses), 2 * sizeof(float), cudaMemcpyDeviceToHost,
                            stream));
  return MOE_OK;
}

moe_status moe_forward_host(const moe_config* cfg, const void* x_host, const void* w_router,
                            const float* router_bias, const void* w_gate_up, const void* w_down, void* y_host,
                            float* losses_host, void* ws, size_t ws_bytes, cudaStream_t stream) {
  const moe_status r = moe_forward_host_async(cfg, x_host, w_router, router_bias, w_gate_up, w_down, y_host,
                                              losses_host, ws, ws_bytes, stream);
  if (r != MOE_OK) return r;
  MOE_TRY(cudaStreamSynchronize(stream));
  return MOE_OK;
}

moe_status moe_backward(const moe_config* cfg, const void* dy, const void* x, const void* w_router,
                        const void* w_gate_up, const void* w_down, void* dx, void* dw_router, void* dw_gate_up,
                        void* dw_down, void* ws, size_t ws_bytes, cudaStream_t stream) {
  Ctx c;
  moe_status r = prepare(cfg, ws, ws_bytes, true, &c);
  if (r != MOE_OK) return r;
  // The weight- and data-gradient GEMMs read operands MN-major, which the tf32
  // UMMA path does not take in the 128-byte swizzle used here: bf16 only.
  if (c.s.fp32) return MOE_ERR_UNSUPPORTED_SHAPE;
  const void* ptrs[] = {dy, x, w_router, w_gate_up, w_down, dx, dw_router, dw_gate_up, dw_down};
  for (const void* p : ptrs)
    if (p == nullptr || !aligned16(p)) return MOE_ERR_INVALID_ARG;
  const Shape& s = c.s;
  const Workspace& L = c.L;
  int32_t* status = at<int32_t>(ws, L.ctrl);
  int32_t* gs = at<int32_t>(ws, L.group_start);
  int32_t* off = at<int32_t>(ws, L.offsets);
  float* dw = at<float>(ws, L.dw);
  float* dh = at<float>(ws, L.dh);
  MOE_TRY(launch_combine_backward(s, dy, at<void>(ws, L.o32), gs, at<int32_t>(ws, L.row_pair), at<float>(ws, L.wts),
                                  dw, at<void>(ws, L.dout), stream));
  MOE_TRY(launch_router_backward(s, dw, at<int32_t>(ws, L.idx), at<float>(ws, L.probs), at<float>(ws, L.lse),
                                 at<int32_t>(ws, L.counts), cfg->alpha_lb, cfg->beta_z, dh, stream));
  MOE_TRY(launch_down_backward_data(s, at<void>(ws, L.dout), gs, off, w_down, at<void>(ws, L.preact),
                                    at<void>(ws, L.dab), status, stream));
  MOE_TRY(launch_gate_up_backward_data(s, at<void>(ws, L.dab), gs, off, w_gate_up, at<void>(ws, L.dx_perm), status,
                                       stream));
  MOE_TRY(launch_weight_grads(s, at<void>(ws, L.dout), at<void>(ws, L.h), at<void>(ws, L.dab), at<void>(ws, L.x_perm),
                              gs, dw_down, dw_gate_up, status, stream));
  MOE_TRY(launch_dx_combine(s, at<void>(ws, L.dx_perm), at<int32_t>(ws, L.inv_perm), dh, w_router, dx, stream));
  MOE_TRY(launch_router_weight_grad(s, dh, x, dw_router, at<float>(ws, L.wr_part), stream));
  return MOE_OK;
}

int64_t moe_expert_choice_capacity(const moe_config* cfg) {
  Shape s;
  return make_shape(cfg, &s) ? ec_default_capacity(s) : -1;
}


moe_status moe_route_expert_choice(const moe_config* cfg, int64_t capacity, const void* x, const void* w_router,
                                   const float* router_bias, int32_t* sel, float* gates, float* probs,
                                   int32_t* counts, float* losses, void* ws, size_t ws_bytes, cudaStream_t stream) {
  Ctx c;
  int64_t C = 0;
  const moe_status r = ec_prepare(cfg, capacity, ws, ws_bytes, &c, &C);
  if (r != MOE_OK) return r;
  if (x == nullptr || w_router == nullptr || sel == nullptr || gates == nullptr || !aligned16(x) ||
      !aligned16(w_router))
    return MOE_ERR_INVALID_ARG;
  MOE_TRY(launch_router_probs(c.s, x, w_router, router_bias, ws, c.L, stream));
  MOE_TRY(launch_ec_select(c.s, C, x, w_router, router_bias, counts, losses, ws, c.L, stream));
  const size_t n = static_cast<size_t>(c.s.E) * static_cast<size_t>(C);
  MOE_TRY(cudaMemcpyAsync(sel, at<int32_t>(ws, c.L.ec_sel), n * 4, cudaMemcpyDeviceToDevice, stream));
  MOE_TRY(cudaMemcpyAsync(gates, at<float>(ws, c.L.ec_gate), n * 4, cudaMemcpyDeviceToDevice, stream));
  if (probs != nullptr)
    MOE_TRY(cudaMemcpyAsync(probs, at<float>(ws, c.L.probs), static_cast<size_t>(c.s.T) * c.s.E * 4,
                            cudaMemcpyDeviceToDevice, stream));
  return MOE_OK;
}

moe_status moe_forward_expert_choice(const moe_config* cfg, int64_t capacity, const void* x, const void* w_router,
                                     const float* router_bias, const void* w_gate_up, const void* w_down, void* y,
                                     float* losses, int32_t* sel, float* gates, void* ws, size_t ws_bytes,
                                     cudaStream_t stream) {
  Ctx c;
  int64_t C = 0;
  const moe_status r = ec_prepare(cfg, capacity, ws, ws_bytes, &c, &C);
  if (r != MOE_OK) return r;
  if (x == nullptr || w_router == nullptr || w_gate_up == nullptr || w_down == nullptr || y == nullptr ||
      !aligned16(x) || !aligned16(w_router) || !aligned16(w_gate_up) || !aligned16(w_down) || !aligned16(y))
    return MOE_ERR_INVALID_ARG;
  const Shape& s = c.s;
  const Workspace& L = c.L;
  int32_t* status = at<int32_t>(ws, L.ctrl);
  int32_t* gs = at<int32_t>(ws, L.group_start);
  int32_t* off = at<int32_t>(ws, L.offsets);
  void* x_perm = at<void>(ws, L.x_perm);
  const StageMarks marks(stream);
  MOE_TRY(marks.mark(0));
  MOE_TRY(launch_router_probs(s, x, w_router, router_bias, ws, L, stream));
  MOE_TRY(marks.mark(1));
  MOE_TRY(launch_ec_select(s, C, x, w_router, router_bias, nullptr, losses, ws, L, stream));
  MOE_TRY(launch_ec_gather(s, C, x, ws, L, stream));
  MOE_TRY(marks.mark(2));
  MOE_TRY(launch_gate_up(s, x_perm, gs, off, w_gate_up, at<void>(ws, L.h), nullptr, status, stream));
  MOE_TRY(marks.mark(3));
  MOE_TRY(launch_down(s, at<void>(ws, L.h), gs, off, w_down, at<void>(ws, L.o_perm), false, status, stream));
  MOE_TRY(marks.mark(4));
  MOE_TRY(launch_combine_ec(s, at<void>(ws, L.o_perm), at<int32_t>(ws, L.ec_slot), at<float>(ws, L.probs), y, stream));
  MOE_TRY(marks.mark(5));
  const size_t n = static_cast<size_t>(s.E) * static_cast<size_t>(C);
  if (sel != nullptr) MOE_TRY(cudaMemcpyAsync(sel, at<int32_t>(ws, L.ec_sel), n * 4, cudaMemcpyDeviceToDevice, stream));
  if (gates != nullptr)
    MOE_TRY(cudaMemcpyAsync(gates, at<float>(ws, L.ec_gate), n * 4, cudaMemcpyDeviceToDevice, stream));
  return MOE_OK;
}

moe_status moe_rmsnorm(const moe_config* cfg, const float* resid, const float* weight, float eps, void* out,
                       cudaStream_t stream) {
  Shape s;
  if (cfg == nullptr) return MOE_ERR_INVALID_ARG;
  if (!make_shape(cfg, &s)) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (resid == nullptr || out == nullptr || !(eps >= 0.f)) return MOE_ERR_INVALID_ARG;
  moe_status r = device_ready();
  if (r != MOE_OK) return r;
  MOE_TRY(launch_rmsnorm(s, resid, weight, eps, out, stream));
  return MOE_OK;
}

moe_status moe_stack_forward_trace(const moe_config* cfg, int32_t n_layers, const void* const* w_router,
                                   const float* const* router_biases, const void* const* w_gate_up,
                                   const void* const* w_down, float* resid, int32_t* counts, float* losses,
                                   int32_t* topk_idx, void* ws, size_t ws_bytes, cudaStream_t stream) {
  Ctx c;
  moe_status r = prepare(cfg, ws, ws_bytes, false, &c);
  if (r != MOE_OK) return r;
  if (n_layers < 1 || w_router == nullptr || w_gate_up == nullptr || w_down == nullptr || resid == nullptr ||
      !aligned16(resid))
    return MOE_ERR_INVALID_ARG;
  for (int l = 0; l < n_layers; ++l)
    if (w_router[l] == nullptr || w_gate_up[l] == nullptr || w_down[l] == nullptr) return MOE_ERR_INVALID_ARG;
  void* xn = at<void>(ws, c.L.x_dev);
  const int64_t tk = c.s.T * c.s.k;
  if (c.s.T <= kDecodeAutoTokens && decode_supported(c.s)) {
    // the whole stack in one persistent kernel (RMSNorm, layer and residual add of every layer)
    MOE_TRY(launch_decode_stack(c.s, resid, kStackRmsEps, n_layers, w_router, router_biases, w_gate_up, w_down, topk_idx,
                                counts, losses, ws, c.L, stream));
    return MOE_OK;
  }
  for (int l = 0; l < n_layers; ++l) {
    MOE_TRY(launch_rmsnorm(c.s, resid, nullptr, kStackRmsEps, xn, stream));
    const float* bias = (router_biases != nullptr) ? router_biases[l] : nullptr;
    r = forward_impl(c, xn, w_router[l], bias, w_gate_up[l], w_down[l], nullptr,
                     losses != nullptr ? losses + 2 * l : nullptr, resid,
                     topk_idx != nullptr ? topk_idx + l * tk : nullptr, nullptr, false, ws, stream,
                     counts != nullptr ? counts + static_cast<int64_t>(l) * c.s.E : nullptr);
    if (r != MOE_OK) return r;
  }
  return MOE_OK;
}

moe_status moe_stack_forward(const moe_config* cfg, int32_t n_layers, const void* const* w_router,
                             const float* const* router_biases, const void* const* w_gate_up,
                             const void* const* w_down, float* resid, void* ws, size_t ws_bytes,
                             cudaStream_t stream) {
  return moe_stack_forward_trace(cfg, n_layers, w_router, router_biases, w_gate_up, w_down, resid, nullptr, nullptr,
                                 nullptr, ws, ws_bytes, stream);
}

moe_status moe_set_stage_events(void* const* events) {
  if (events == nullptr) {
    g_stage_armed = false;
    return MOE_OK;
  }
  for (int i = 0; i < MOE_STAGE_EVENTS; ++i) {
    if (events[i] == nullptr) return MOE_ERR_INVALID_ARG;
    g_stage_events[i] = static_cast<cudaEvent_t>(events[i]);
  }
  g_stage_armed = true;
  return MOE_OK;
}

moe_status moe_get_device_status(void* ws, int32_t* code, cudaStream_t stream) {
  if (ws == nullptr || code == nullptr) return MOE_ERR_INVALID_ARG;
  int32_t v = 0;
  MOE_TRY(cudaMemcpyAsync(&v, ws, sizeof(int32_t), cudaMemcpyDeviceToHost, stream));
  MOE_TRY(cudaStreamSynchronize(stream));
  // the status word and, with it, the completion counters: a launch that gave
  // up part-way may have left a counter behind
  MOE_TRY(cudaMemsetAsync(ws, 0, 8 * sizeof(int32_t), stream));
  *code = v;
  return v == 0 ? MOE_OK : MOE_ERR_DEVICE_CHECK;
}

}  // extern "C"
