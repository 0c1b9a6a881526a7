// Internal declarations shared by the host-side entry points and the kernel
// launchers: the workspace layout and the launcher signatures.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstddef>
#include <cstdint>

#include "../../include/moe.h"

namespace moe {

constexpr int kRowAlign = MOE_ROW_ALIGN;  // expert groups start on multiples of this
constexpr int kRouterTokensPerCta = 16;   // router kernel token block
constexpr int kDispatchChunk = 32;        // tokens per dispatch ranking chunk (= one router tile)
constexpr int kMaxExperts = 256;
constexpr int kMaxTopK = 16;

struct Shape {
  int64_t T;
  int d, E, k, f;
  bool fp32;
  bool grad32;   // backward writes the weight gradients in fp32
  bool renorm;   // router weights renormalised over the k chosen experts
  size_t esize;  // bytes per activation / weight element
  int64_t P;     // padded row capacity
  int64_t router_ctas() const { return (T + kRouterTokensPerCta - 1) / kRouterTokensPerCta; }
  int64_t chunks() const { return (T + kDispatchChunk - 1) / kDispatchChunk; }
};

// Byte offsets of every region inside the caller's workspace.
struct Workspace {
  // control words: [0] status, [1] router ticket, [2] dispatch ticket,
  // [3] grid-barrier arrivals, [4] CTAs past their last grid barrier
  size_t ctrl;
  size_t counts_part, psum_part, zsum_part;  // router per-CTA partials
  size_t counts, losses;                     // router totals
  size_t probs, lse;                         // saved for backward: p [T,E], lse [T]
  size_t idx, wts;                           // top-k indices and weights
  size_t local_rank, chunk_count, chunk_base;
  size_t offsets, group_start, perm, inv_perm, row_pair;
  size_t x_perm, h, o_perm;
  size_t preact;                              // [P, 2f] fp32 (training)
  size_t o32;                                 // [P, d] fp32 expert outputs (training)
  size_t dw, dh, dout, dab, dx_perm, wr_part; // backward scratch
  size_t x_dev, y_dev;                        // staging for the host-buffer entry point
  size_t ec_sel, ec_gate, ec_slot;            // expert choice: [E, C] tokens and weights, [T, E] rows
  size_t fwd_bytes, bwd_bytes;
};

bool make_shape(const moe_config* cfg, Shape* s);
Workspace layout(const Shape& s);

template <typename T>
inline T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<char*>(ws) + off);
}

// ---- launchers (each returns cudaSuccess or the launch error)
cudaError_t launch_router(const Shape& s, const void* x, const void* w_router, const float* bias, int32_t* idx,
                          float* wts, int32_t* counts, float* losses, void* ws, const Workspace& L,
                          cudaStream_t st);
// Tensor-core router (bf16, E <= 64). Besides launch_router's outputs it leaves
// the dispatch ranking in the workspace (local ranks, per-chunk counts and
// bases, offsets, group starts), so the rank kernel can be skipped.
bool router_tc_supported(const Shape& s);
cudaError_t launch_router_tc(const Shape& s, const void* x, const void* w_router, const float* bias, int32_t* idx,
                             float* wts, int32_t* counts, float* losses, void* ws, const Workspace& L,
                             cudaStream_t st);
cudaError_t launch_permute(const Shape& s, const int32_t* idx, const void* x, int32_t* perm, int32_t* inv_perm,
                           void* x_perm, void* ws, const Workspace& L, bool zero_pads, cudaStream_t st);
cudaError_t launch_dispatch(const Shape& s, const int32_t* idx, const void* x, int32_t* offsets, int32_t* perm,
                            int32_t* inv_perm, int32_t* group_start, void* x_perm, void* ws, const Workspace& L,
                            cudaStream_t st);
cudaError_t launch_gate_up(const Shape& s, const void* x_perm, const int32_t* group_start,
                           const int32_t* offsets, const void* w_gate_up, void* h, void* preact, int32_t* status,
                           cudaStream_t st);
// gate/up: `preact` (or null) receives the pre-activations in fp32.
// down: o_perm in fp32 when `out32` (the expert outputs kept for the backward),
// else in the layer dtype.
cudaError_t launch_down(const Shape& s, const void* h, const int32_t* group_start, const int32_t* offsets,
                        const void* w_down, void* o_perm, bool out32, int32_t* status, cudaStream_t st);
// `o32`: o_perm holds fp32 rows (the saved expert outputs) instead of the layer dtype.
cudaError_t launch_combine(const Shape& s, const void* o_perm, bool o32, const int32_t* inv_perm, const float* wts,
                           void* y, float* resid, cudaStream_t st);
// Expert choice: the router's probabilities and log-normaliser only (no top-k),
// then each expert's top-C tokens, the row gather and the combine.
cudaError_t launch_router_probs(const Shape& s, const void* x, const void* w_router, const float* bias, void* ws,
                                const Workspace& L, cudaStream_t st);
int64_t ec_default_capacity(const Shape& s);
bool ec_capacity_ok(const Shape& s, int64_t C);
// x, w_router, bias: the router's inputs, for the exact re-ranking near the C-th value
cudaError_t launch_ec_select(const Shape& s, int64_t C, const void* x, const void* w_router, const float* bias,
                             int32_t* counts, float* losses, void* ws, const Workspace& L, cudaStream_t st);
cudaError_t launch_ec_gather(const Shape& s, int64_t C, const void* x, void* ws, const Workspace& L,
                             cudaStream_t st);
cudaError_t launch_combine_ec(const Shape& s, const void* o_perm, const int32_t* slot_row, const float* probs,
                              void* y, cudaStream_t st);
// Fused decode layer (T <= 8, bf16, E <= 64, staged rows within shared memory):
// the whole forward in one cooperative kernel. With `resid` non-null the input
// is RMSNorm(resid) (unit weight, eps) and the output is added to resid;
// otherwise x -> y. Forward only (nothing is kept for the backward).
bool decode_supported(const Shape& s);
// Batches the layer forward routes to the one-kernel form by itself: up to 4
// tokens (measured on B200 in CUDA-graph replays, L2 flushed before each: T=1
// 45 us, T=4 102 us; at T=8 the layered tensor-core path is ahead, about 152
// against 197 us).
constexpr int64_t kDecodeAutoTokens = 4;
cudaError_t launch_decode_layer(const Shape& s, const void* x, float* resid, double eps, const void* w_router,
                                const float* bias, const void* w_gate_up, const void* w_down, void* y,
                                int32_t* topk_idx, float* topk_w, int32_t* counts, float* losses, void* ws,
                                const Workspace& L, cudaStream_t st);
// RMSNorm of the fp32 residual, evaluated in fp64 and rounded once to fp32
// and then to the layer dtype.
// A stack of n_layers decode blocks, resid <- resid + MoE_l(RMSNorm(resid)),
// in one launch per 16 layers (per-layer outputs may be null).
cudaError_t launch_decode_stack(const Shape& s, float* resid, double eps, int n_layers, const void* const* w_router,
                                const float* const* biases, const void* const* w_gate_up, const void* const* w_down,
                                int32_t* topk_idx, int32_t* counts, float* losses, void* ws, const Workspace& L,
                                cudaStream_t st);
cudaError_t launch_rmsnorm(const Shape& s, const float* resid, const float* weight, double eps, void* out,
                           cudaStream_t st);
// eps of the stack's pre-norm ("Mixture-of-experts LLMs from scratch with OLMoE",
// section 3: RMSNorm with the library default 1e-5)
constexpr double kStackRmsEps = 1e-5;

// backward pieces (o32: the fp32 expert outputs saved by the forward)
cudaError_t launch_dispatch_impl(const Shape& s, const int32_t* idx, const void* x, int32_t* offsets,
                                 int32_t* perm, int32_t* inv_perm, int32_t* group_start, void* x_perm, void* ws,
                                 const Workspace& L, bool zero_pads, cudaStream_t st);
cudaError_t launch_combine_backward(const Shape& s, const void* dy, const void* o_perm, const int32_t* gs,
                                    const int32_t* row_pair, const float* wts, float* dw, void* dout,
                                    cudaStream_t st);
cudaError_t launch_down_backward_data(const Shape& s, const void* dout, const int32_t* group_start,
                                      const int32_t* offsets, const void* w_down, const void* preact, void* dab,
                                      int32_t* status, cudaStream_t st);
cudaError_t launch_gate_up_backward_data(const Shape& s, const void* dab, const int32_t* group_start,
                                         const int32_t* offsets, const void* w_gate_up, void* dx_perm,
                                         int32_t* status, cudaStream_t st);
cudaError_t launch_weight_grads(const Shape& s, const void* dout, const void* h, const void* dab,
                                const void* x_perm, const int32_t* group_start, void* dw_down, void* dw_gate_up,
                                int32_t* status, cudaStream_t st);
cudaError_t launch_router_backward(const Shape& s, const float* dw, const int32_t* idx, const float* probs,
                                   const float* lse, const int32_t* counts, float alpha, float beta, float* dh,
                                   cudaStream_t st);
cudaError_t launch_dx_combine(const Shape& s, const void* dx_perm, const int32_t* inv_perm, const float* dh,
                              const void* w_router, void* dx, cudaStream_t st);
cudaError_t launch_router_weight_grad(const Shape& s, const float* dh, const void* x, void* dw_router,
                                      float* part, cudaStream_t st);
size_t router_wgrad_partial_bytes(const Shape& s);

int device_sm_count();

// Launches `kern` as a programmatic dependent of the previous kernel in the
// stream: it may be scheduled while that kernel finishes, and calls pdl_wait()
// (sm100.cuh) before touching memory an earlier kernel writes or reads.
// `extra` (or null) are further launch attributes (a cluster shape).
template <typename... KArgs, typename... Args>
cudaError_t launch_dependent(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                             const cudaLaunchAttribute* extra, int n_extra, Args... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[4];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  int n = 1;
  for (int i = 0; i < n_extra && n < 4; ++i) attr[n++] = extra[i];
  cfg.attrs = attr;
  cfg.numAttrs = static_cast<unsigned>(n);
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

// Raises `func`'s dynamic shared-memory limit to at least `bytes` on the current
// device. `cache` (one entry per device id < 64, zero-initialised, owned by the
// call site) remembers the largest limit already set, so each device is
// configured once however many devices a process drives.
constexpr int kMaxDevices = 64;
cudaError_t raise_smem_limit(const void* func, size_t bytes, std::atomic<size_t>* cache);

// 2-D TMA descriptor over a row-major [rows, cols] bf16/fp32 matrix with a
// [box_rows, box_cols] box and 128-byte swizzle (out-of-range boxes read zeros).
bool make_map(CUtensorMap* m, const void* base, bool fp32, uint64_t rows, uint64_t cols, uint32_t box_cols,
              uint32_t box_rows);

}  // namespace moe
