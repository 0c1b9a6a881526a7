// The whole MoE layer for a decode-sized batch (T <= 8 tokens) in one
// persistent cooperative kernel: router, gate/up + SwiGLU, down and combine,
// optionally with the block's RMSNorm in front and the residual add behind;
// and a stack of such blocks (up to 16 per launch) in the same kernel, which
// walks the layers with a grid barrier between one layer's residual update
// and the next layer's RMSNorm.
//
// Method: the layer of "Mixture-of-experts LLMs from scratch with OLMoE",
// section 2 (softmax over all experts, top-k without renormalisation, each
// expert once on its tokens, weighted sum back) and section 3 (the Block:
// r + MoE(RMSNorm(r)) on an fp32 residual), the SwiGLU expert of "OLMoE
// Guide", "Top-8 Softmax Routing Formulation", and its losses ("Router
// Mechanics & Loss Formulations"). Section 6 of the lesson notes that at a
// batch of one token the layer reads only the k chosen experts' weights, so
// decoding is bound by streaming those weights; this kernel exists to stream
// them with nothing else in the way (one launch, one grid barrier).
//
// One CTA per SM (grid = SM count, cooperative launch, 16 warps):
//   prologue  every CTA stages the T input rows in shared memory (with the
//             RMSNorm applied when the input is the fp32 residual).
//   phase 0   every CTA computes the T*E router logits itself (W_r is read
//             from L2 by each CTA; no grid barrier): products of bf16 values
//             are exact in fp32 and are summed in fp32; a token whose k+1
//             largest logits hold near-equal neighbours has its logits
//             recomputed as fp64 sums of the exact products, so the top-k
//             matches an exact computation except for exactly equal logits
//             (lower index wins). Every CTA takes the same decisions.
//   phase 0b  every CTA: each expert's rank among a token's logits gives the
//             top-k at once (no sequential selection); softmax in fp32; the
//             tokens of each expert as a bit mask; CTA 0 writes the losses,
//             counts and the optional top-k outputs.
//   phase 1   one warp per (touched expert, hidden row i): the gate row i and
//             the up row i stream once from HBM (all of the pair's loads in
//             flight before any arithmetic) and meet every token that chose
//             the expert; h = SiLU(g) * u is stored in bf16 (as the grouped
//             GEMM stores it).
//   barrier
//   phase 2   every CTA stages h; one warp per output column c: row c of each
//             touched expert's down matrix streams once, its dot products with
//             the tokens' h rows are summed per token in slot order in fp32,
//             weighted, and written once (bf16 y, or added to the residual).
// The grid barrier is an arrival counter and a generation word in the
// workspace; each wait gives up after about a second, records a status and
// lets the kernel finish. Every single-lane section rejoins its warp
// (__syncwarp) before a block-wide barrier.
#include "moe_internal.h"
#include "sm100.cuh"

namespace moe {
namespace {

constexpr int kDecThreads = 512;
constexpr int kDecWarps = kDecThreads / 32;
constexpr int kDecMaxT = 8;
constexpr int kDecMaxE = 64;
constexpr int kDecSlots = kDecMaxT * kMaxTopK;            // (token, slot) pairs
constexpr size_t kDecActBytes = 160 * 1024;               // staged x, then h
constexpr size_t kDecMiscBytes = 28 * 1024;
constexpr size_t kDecSmem = kDecActBytes + kDecMiscBytes;
constexpr int kDecMaxLayers = 16;                          // layers of a stack per launch

// One layer's weights.
struct DecLayer {
  const __nv_bfloat16* wr;   // [E, d]
  const float* bias;         // [E] or null
  const __nv_bfloat16* wgu;  // [E, 2f, d]
  const __nv_bfloat16* wd;   // [E, d, f]
};

struct DecArgs {
  int T, d, E, k, f;
  int renorm;
  double eps;
  int n_layers;              // 1, or up to kDecMaxLayers blocks of a stack (with `resid`)
  DecLayer layer[kDecMaxLayers];
  const __nv_bfloat16* x;    // [T, d] layer input, or null when `resid` is the input
  float* resid;              // [T, d] fp32 residual (in/out), or null
  __nv_bfloat16* y;          // [T, d] out (null with `resid`)
  __nv_bfloat16* h;          // [T*k, f] workspace
  int32_t* idx_out;          // [n_layers, T, k] or null
  float* w_out;              // [T, k] or null (single layer)
  int32_t* counts;           // [n_layers, E] or null
  float* losses;             // [n_layers, 2] or null
  float* losses_ws;          // [2] workspace copy (of the last layer)
  unsigned* bar;             // [2] arrival count, generation
  int32_t* status;
};

struct DecSmem {
  int sel_e[kDecSlots];
  float sel_w[kDecSlots];
  float ps[kDecWarps][kDecSlots];  // per-warp dot products of one output column
  unsigned tokmask[kDecMaxE];      // bit t: token t chose the expert
  int slot_of[kDecMaxT][kDecMaxE]; // slot of expert e among token t's choices, or -1
  int touched[kDecMaxE];           // experts chosen by some token, ascending
  int n_touched;
  int ok;
  double rms[kDecMaxT];             // 1 / sqrt(mean square + eps) of each input row
  double hd[kDecMaxT][kDecMaxE];   // logits (+ offset)
  float p[kDecMaxT][kDecMaxE];
  float lse[kDecMaxT];
  DecLayer layers[kDecMaxLayers];  // the launch's layer table
};
static_assert(sizeof(DecSmem) <= kDecMiscBytes, "decode bookkeeping fits");

// Grid-wide barrier (all CTAs co-resident: cooperative launch). Returns false
// when the wait gave up; the failure is recorded and every CTA then unwinds.
__device__ bool grid_barrier(unsigned* bar, unsigned n, int32_t* status, int* ok_s) {
  __syncwarp();
  __syncthreads();
  if (threadIdx.x == 0) {
    volatile unsigned* gen = bar + 1;
    const unsigned g = *gen;
    __threadfence();
    int ok = 1;
    if (atomicAdd(bar, 1u) == n - 1) {
      atomicExch(bar, 0u);
      __threadfence();
      atomicAdd(bar + 1, 1u);
    } else {
      const uint64_t t0 = global_timer_ns();
      uint32_t spins = 0;
      while (*gen == g) {
        if (++spins > 1024u) __nanosleep(32);
        if ((spins & 255u) == 0u && global_timer_ns() - t0 > kWaitLimitNs) {
          report(status, DEV_WAIT_TIMEOUT_GRID);
          ok = 0;
          break;
        }
      }
    }
    __threadfence();
    *ok_s = ok;
  }
  __syncwarp();  // warp 0 whole again before the block barrier
  __syncthreads();
  return *ok_s != 0;
}

__device__ __forceinline__ void bf16x8(const uint4& q, float (&v)[8]) {
  const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float2 f2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[j]));
    v[2 * j] = f2.x;
    v[2 * j + 1] = f2.y;
  }
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// NT: tokens the phase-1 accumulators are sized for (1, 2, 4 or 8; T <= NT).
// STACK: walks a.n_layers layers of a stack; otherwise exactly one layer (a
// loop whose trip count the compiler knows keeps the kernel free of register
// spills; the stack's runtime layer loop costs some).
template <int NT, bool STACK>
__global__ void __launch_bounds__(kDecThreads, 1) decode_layer_kernel(const __grid_constant__ DecArgs a) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  __nv_bfloat16* act = reinterpret_cast<__nv_bfloat16*>(smem_raw);  // x [T, d], later h [T*k, f]
  DecSmem& m = *reinterpret_cast<DecSmem*>(smem_raw + kDecActBytes);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int T = a.T, d = a.d, E = a.E, k = a.k, f = a.f;
  const int nvd = d / 8, nvf = f / 8;  // 16-byte vectors per row
  const int gw = blockIdx.x * kDecWarps + warp;
  const int nw = gridDim.x * kDecWarps;
  // the layer table in shared memory (indexed by layer below; kernel parameters
  // are only read at fixed offsets)
#pragma unroll
  for (int l = 0; l < kDecMaxLayers; ++l)
    if (tid == l) m.layers[l] = a.layer[l];
  __syncthreads();

  const int n_layers = STACK ? a.n_layers : 1;
#pragma unroll 1
  for (int l = 0; l < n_layers; ++l) {
  // a layer of a stack reads the residual the previous layer completed
  if (l > 0 && !grid_barrier(a.bar, gridDim.x, a.status, &m.ok)) return;
  const DecLayer Ly = m.layers[l];
  int32_t* const idx_out = a.idx_out != nullptr ? a.idx_out + static_cast<int64_t>(l) * T * k : nullptr;
  int32_t* const counts = a.counts != nullptr ? a.counts + static_cast<int64_t>(l) * E : nullptr;
  float* const losses = a.losses != nullptr ? a.losses + 2 * l : nullptr;

  // ---- prologue: the T input rows, bf16, in shared memory
  if (a.resid != nullptr) {
    if (warp < T) {  // RMSNorm (unit weight) of token `warp` in fp64, mean of squares in a fixed order
      const float* r = a.resid + static_cast<int64_t>(warp) * d;
      double ss = 0.0;
      for (int i = lane; i < d; i += 32) ss = fma(static_cast<double>(r[i]), static_cast<double>(r[i]), ss);
      ss = warp_sum_d(ss);
      if (lane == 0) m.rms[warp] = 1.0 / sqrt(ss / static_cast<double>(d) + a.eps);
      __syncwarp();
    }
    __syncthreads();
    // the fp64 value rounded to fp32, then to bf16 (as the separate RMSNorm kernel does)
    for (int i = tid; i < T * d; i += kDecThreads)
      act[i] = __float2bfloat16_rn(static_cast<float>(static_cast<double>(a.resid[i]) * m.rms[i / d]));
  } else {
    const uint4* src = reinterpret_cast<const uint4*>(a.x);
    uint4* dst = reinterpret_cast<uint4*>(act);
    for (int i = tid; i < T * nvd; i += kDecThreads) dst[i] = __ldg(src + i);
  }
  if (tid < kDecMaxE) m.tokmask[tid] = 0u;
  if (tid < kDecSlots) m.sel_e[tid] = 0;  // defined even if non-finite logits leave a slot unranked
  __syncthreads();

  // ---- phase 0 (every CTA, no grid barrier): the T*E router logits. Warp w
  //      takes experts w, w + 16, ...; each W_r row is read once into registers
  //      and meets every token. bf16 x bf16 products are exact in fp32 and are
  //      summed in fp32 here; every CTA sums in the same order, so every CTA
  //      holds the same values and takes the same decisions.
  for (int e = warp; e < E; e += kDecWarps) {
    const uint4* wrow = reinterpret_cast<const uint4*>(Ly.wr + static_cast<int64_t>(e) * d);
    float acc[NT];
#pragma unroll
    for (int q = 0; q < NT; ++q) acc[q] = 0.f;
    for (int v0 = 0; v0 < nvd; v0 += 32 * 8) {
      uint4 wq[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int v = v0 + j * 32 + lane;
        if (v < nvd) wq[j] = __ldg(wrow + v);
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int v = v0 + j * 32 + lane;
        if (v < nvd) {
          float wv[8];
          bf16x8(wq[j], wv);
#pragma unroll
          for (int q = 0; q < NT; ++q) {
            if (q < T) {
              float xv[8];
              bf16x8(reinterpret_cast<const uint4*>(act + static_cast<int64_t>(q) * d)[v], xv);
#pragma unroll
              for (int i = 0; i < 8; ++i) acc[q] = fmaf(xv[i], wv[i], acc[q]);
            }
          }
        }
      }
    }
#pragma unroll
    for (int q = 0; q < NT; ++q) {
      if (q < T) {
        const float h = warp_sum(acc[q]);
        if (lane == 0) m.hd[q][e] = static_cast<double>(h) + (Ly.bias != nullptr ? static_cast<double>(Ly.bias[e]) : 0.0);
      }
    }
  }
  __syncthreads();
  // The choice must be the exact one: a token whose k+1 largest fp32 logits
  // hold two values closer than 2e-4 * max(1, |h|) (far above the error of a
  // 2048-term fp32 sum of exact products) has all E logits recomputed exactly
  // (fp64 sums of the exact products), lane l taking experts l and l + 32.
  if (warp < T) {
    const int t = warp;
    const int e0 = lane, e1 = lane + 32;
    const double h0 = e0 < E ? m.hd[t][e0] : -INFINITY, h1 = e1 < E ? m.hd[t][e1] : -INFINITY;
    int r0 = 0, r1 = 0;
    for (int e = 0; e < E; ++e) {
      const double v = m.hd[t][e];
      r0 += (v > h0 || (v == h0 && e < e0)) ? 1 : 0;
      r1 += (v > h1 || (v == h1 && e < e1)) ? 1 : 0;
    }
    bool near = false;
    for (int e = 0; e < E; ++e) {
      const double v = m.hd[t][e];
      const double g = 2e-4 * fmax(1.0, fabs(v));
      if (e0 < E && e != e0 && r0 <= k && fabs(v - h0) < g) near = true;
      if (e1 < E && e != e1 && r1 <= k && fabs(v - h1) < g) near = true;
    }
    // (a near value may rank below k + 1 itself: then it is within the gap of
    // a ranked one, which the loop above finds from that ranked lane)
    if (__any_sync(0xffffffffu, near)) {
      const uint4* xrow = reinterpret_cast<const uint4*>(act + static_cast<int64_t>(t) * d);
      double ex[2] = {0.0, 0.0};
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int e = lane + 32 * u;
        if (e < E) {
          const uint4* wrow = reinterpret_cast<const uint4*>(Ly.wr + static_cast<int64_t>(e) * d);
          double acc = 0.0;
          for (int v = 0; v < nvd; ++v) {
            float xv[8], wv[8];
            bf16x8(xrow[v], xv);
            bf16x8(__ldg(wrow + v), wv);
#pragma unroll
            for (int i = 0; i < 8; ++i) acc += static_cast<double>(xv[i] * wv[i]);  // exact product
          }
          ex[u] = acc + (Ly.bias != nullptr ? static_cast<double>(Ly.bias[e]) : 0.0);
        }
      }
      __syncwarp();
      if (e0 < E) m.hd[t][e0] = ex[0];
      if (e1 < E) m.hd[t][e1] = ex[1];
    }
    __syncwarp();
  }
  __syncthreads();

  // ---- phase 0b (every CTA): warp t takes token t; lane l holds experts l, l + 32
  if (warp < T) {
    const int t = warp;
    const int e0 = lane, e1 = lane + 32;
    const double h0 = e0 < E ? m.hd[t][e0] : -INFINITY;
    const double h1 = e1 < E ? m.hd[t][e1] : -INFINITY;
    // rank by (logit descending, index ascending): the experts ranked below k are the choice
    int r0 = 0, r1 = 0;
    for (int e = 0; e < E; ++e) {
      const double v = m.hd[t][e];
      r0 += (v > h0 || (v == h0 && e < e0)) ? 1 : 0;
      r1 += (v > h1 || (v == h1 && e < e1)) ? 1 : 0;
    }
    if (e0 < E) {
      m.slot_of[t][e0] = r0 < k ? r0 : -1;
      if (r0 < k) {
        m.sel_e[t * k + r0] = e0;
        atomicOr(&m.tokmask[e0], 1u << t);
      }
    }
    if (e1 < E) {
      m.slot_of[t][e1] = r1 < k ? r1 : -1;
      if (r1 < k) {
        m.sel_e[t * k + r1] = e1;
        atomicOr(&m.tokmask[e1], 1u << t);
      }
    }
    // softmax over all experts in fp32 from the exact logits
    double mx = fmax(h0, h1);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmax(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    const float x0 = e0 < E ? expf(static_cast<float>(h0 - mx)) : 0.f;
    const float x1 = e1 < E ? expf(static_cast<float>(h1 - mx)) : 0.f;
    const float sum = warp_sum(x0 + x1);
    if (e0 < E) m.p[t][e0] = x0 / sum;
    if (e1 < E) m.p[t][e1] = x1 / sum;
    if (lane == 0) m.lse[t] = static_cast<float>(mx) + logf(sum);
    __syncwarp();
    if (lane == 0) {  // weights in slot order (renormalised: over the k chosen, summed in slot order)
      float den = 0.f;
      for (int j = 0; j < k; ++j) den += m.p[t][m.sel_e[t * k + j]];
      for (int j = 0; j < k; ++j) {
        const int e = m.sel_e[t * k + j];
        const float w = a.renorm ? m.p[t][e] / den : m.p[t][e];
        m.sel_w[t * k + j] = w;
        if (blockIdx.x == 0) {
          if (idx_out != nullptr) idx_out[t * k + j] = e;
          if (a.w_out != nullptr) a.w_out[t * k + j] = w;
        }
      }
    }
    __syncwarp();
  }
  __syncthreads();
  if (warp == 0) {  // the touched experts, ascending; CTA 0: counts and losses
    int base = 0;
    double lb = 0.0;
    for (int c = 0; c < E; c += 32) {
      const int e = c + lane;
      const bool on = e < E && m.tokmask[e] != 0u;
      const unsigned b = __ballot_sync(0xffffffffu, on);
      if (on) m.touched[base + __popc(b & ((1u << lane) - 1u))] = e;
      base += __popc(b);
      if (blockIdx.x == 0 && e < E) {
        const int ce = __popc(m.tokmask[e]);
        double pe = 0.0;
        for (int t = 0; t < T; ++t) pe += m.p[t][e];
        lb += static_cast<double>(ce) * pe;
        if (counts != nullptr) counts[e] = ce;
      }
    }
    if (lane == 0) m.n_touched = base;
    if (blockIdx.x == 0) {  // E * sum_e (c_e / (T k)) (P_e / T), and the mean of lse^2
      lb = warp_sum_d(lb);
      if (lane == 0) {
        double z = 0.0;
        for (int t = 0; t < T; ++t) z += static_cast<double>(m.lse[t]) * m.lse[t];
        const double Td = static_cast<double>(T);
        const float l0 = static_cast<float>(lb * E / (Td * Td * k)), l1 = static_cast<float>(z / Td);
        a.losses_ws[0] = l0;
        a.losses_ws[1] = l1;
        if (losses != nullptr) {
          losses[0] = l0;
          losses[1] = l1;
        }
      }
    }
    __syncwarp();
  }
  __syncthreads();
  const int nt = m.n_touched;

  // ---- phase 1: gate/up rows of the touched experts, a warp per (expert, row);
  //      the whole row pair's loads are in flight before any arithmetic
  for (int item = gw; item < nt * f; item += nw) {
    const int u = item / f, i = item - u * f;
    const int e = m.touched[u];
    const unsigned tmask = m.tokmask[e];
    const uint4* grow = reinterpret_cast<const uint4*>(Ly.wgu + (static_cast<int64_t>(e) * 2 * f + i) * d);
    const uint4* urow = grow + static_cast<int64_t>(f) * nvd;
    float ag[NT], au[NT];
#pragma unroll
    for (int q = 0; q < NT; ++q) ag[q] = au[q] = 0.f;
    for (int v0 = 0; v0 < nvd; v0 += 32 * 8) {
      uint4 gq[8], uq[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int v = v0 + j * 32 + lane;
        if (v < nvd) {
          gq[j] = __ldg(grow + v);
          uq[j] = __ldg(urow + v);
        }
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int v = v0 + j * 32 + lane;
        if (v < nvd) {
          float gv[8], uv[8];
          bf16x8(gq[j], gv);
          bf16x8(uq[j], uv);
#pragma unroll
          for (int q = 0; q < NT; ++q) {
            if ((tmask >> q) & 1u) {
              float xv[8];
              bf16x8(reinterpret_cast<const uint4*>(act + static_cast<int64_t>(q) * d)[v], xv);
#pragma unroll
              for (int c = 0; c < 8; ++c) {
                ag[q] = fmaf(gv[c], xv[c], ag[q]);
                au[q] = fmaf(uv[c], xv[c], au[q]);
              }
            }
          }
        }
      }
    }
#pragma unroll
    for (int q = 0; q < NT; ++q) {
      if ((tmask >> q) & 1u) {
        const float g = warp_sum(ag[q]), uu = warp_sum(au[q]);
        if (lane == 0) {
          const int slot = q * k + m.slot_of[q][e];
          a.h[static_cast<int64_t>(slot) * f + i] = __float2bfloat16_rn(silu_fast(g) * uu);
        }
      }
    }
  }
  if (!grid_barrier(a.bar, gridDim.x, a.status, &m.ok)) return;

  // ---- phase 2: h in shared memory, then a warp per output column
  {
    const uint4* src = reinterpret_cast<const uint4*>(a.h);
    uint4* dst = reinterpret_cast<uint4*>(act);
    for (int i = tid; i < T * k * nvf; i += kDecThreads) dst[i] = __ldcg(src + i);
  }
  __syncthreads();
  for (int c = gw; c < d; c += nw) {
    for (int u0 = 0; u0 < nt; u0 += 4) {
      uint4 wq[4][4];  // four experts' rows, four 16-byte vectors per lane at a time
      for (int v0 = 0; v0 < nvf; v0 += 32 * 4) {
#pragma unroll
        for (int uu = 0; uu < 4; ++uu) {
          if (u0 + uu < nt) {
            const uint4* row =
                reinterpret_cast<const uint4*>(Ly.wd + (static_cast<int64_t>(m.touched[u0 + uu]) * d + c) * f);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const int v = v0 + j * 32 + lane;
              if (v < nvf) wq[uu][j] = __ldg(row + v);
            }
          }
        }
#pragma unroll
        for (int uu = 0; uu < 4; ++uu) {
          if (u0 + uu < nt) {
            const int e = m.touched[u0 + uu];
            unsigned tm = m.tokmask[e];
            while (tm != 0u) {
              const int t = __ffs(tm) - 1;
              tm &= tm - 1u;
              const int slot = t * k + m.slot_of[t][e];
              const uint4* hrow = reinterpret_cast<const uint4*>(act + static_cast<int64_t>(slot) * f);
              float acc = 0.f;
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                const int v = v0 + j * 32 + lane;
                if (v < nvf) {
                  float wv[8], hv[8];
                  bf16x8(wq[uu][j], wv);
                  bf16x8(hrow[v], hv);
#pragma unroll
                  for (int cc = 0; cc < 8; ++cc) acc = fmaf(wv[cc], hv[cc], acc);
                }
              }
              acc = warp_sum(acc);
              if (lane == 0) m.ps[warp][slot] = (v0 == 0 ? 0.f : m.ps[warp][slot]) + acc;
            }
          }
        }
      }
    }
    __syncwarp();
    if (lane < T) {  // token `lane`: weighted sum over its slots, in slot order
      float acc = 0.f;
      for (int j = 0; j < k; ++j) acc = fmaf(m.sel_w[lane * k + j], m.ps[warp][lane * k + j], acc);
      const int64_t o = static_cast<int64_t>(lane) * d + c;
      if (a.resid != nullptr)
        a.resid[o] += acc;
      else
        a.y[o] = __float2bfloat16_rn(acc);
    }
    __syncwarp();
  }
  }  // layers
}

}  // namespace

bool decode_supported(const Shape& s) {
  if (s.fp32 || s.T > kDecMaxT || s.E > kDecMaxE || s.k > kMaxTopK) return false;
  const size_t x_bytes = static_cast<size_t>(s.T) * s.d * 2, h_bytes = static_cast<size_t>(s.T) * s.k * s.f * 2;
  return x_bytes <= kDecActBytes && h_bytes <= kDecActBytes;
}

namespace {
// One cooperative launch over `n` (<= kDecMaxLayers) layers.
cudaError_t launch_decode(const Shape& s, const void* x, float* resid, double eps, int n,
                          const void* const* w_router, const float* const* biases, const void* const* w_gate_up,
                          const void* const* w_down, void* y, int32_t* topk_idx, float* topk_w, int32_t* counts,
                          float* losses, void* ws, const Workspace& L, cudaStream_t st) {
  // the accumulator count follows the batch: fewer live registers for small T
  // keep more of each warp's row loads in flight
  static std::atomic<size_t> set_smem[8][kMaxDevices];
  const bool stack = n > 1;
  void (*kern)(DecArgs) = s.T <= 1 ? (stack ? decode_layer_kernel<1, true> : decode_layer_kernel<1, false>)
                          : s.T <= 2 ? (stack ? decode_layer_kernel<2, true> : decode_layer_kernel<2, false>)
                          : s.T <= 4 ? (stack ? decode_layer_kernel<4, true> : decode_layer_kernel<4, false>)
                                     : (stack ? decode_layer_kernel<8, true> : decode_layer_kernel<8, false>);
  const int which = (s.T <= 1 ? 0 : s.T <= 2 ? 1 : s.T <= 4 ? 2 : 3) + (stack ? 4 : 0);
  cudaError_t e = raise_smem_limit(reinterpret_cast<const void*>(kern), kDecSmem, set_smem[which]);
  if (e != cudaSuccess) return e;
  if (n < 1 || n > kDecMaxLayers) return cudaErrorInvalidValue;
  DecArgs a{};
  a.T = static_cast<int>(s.T);
  a.d = s.d;
  a.E = s.E;
  a.k = s.k;
  a.f = s.f;
  a.renorm = s.renorm ? 1 : 0;
  a.eps = eps;
  a.n_layers = n;
  for (int l = 0; l < n; ++l) {
    a.layer[l].wr = static_cast<const __nv_bfloat16*>(w_router[l]);
    a.layer[l].bias = biases != nullptr ? biases[l] : nullptr;
    a.layer[l].wgu = static_cast<const __nv_bfloat16*>(w_gate_up[l]);
    a.layer[l].wd = static_cast<const __nv_bfloat16*>(w_down[l]);
  }
  a.x = static_cast<const __nv_bfloat16*>(x);
  a.resid = resid;
  a.y = static_cast<__nv_bfloat16*>(y);
  a.h = at<__nv_bfloat16>(ws, L.h);
  a.idx_out = topk_idx;
  a.w_out = topk_w;
  a.counts = counts;
  a.losses = losses;
  a.losses_ws = at<float>(ws, L.losses);
  a.bar = reinterpret_cast<unsigned*>(at<int32_t>(ws, L.ctrl) + 3);
  a.status = at<int32_t>(ws, L.ctrl);
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(device_sm_count()));
  cfg.blockDim = dim3(kDecThreads);
  cfg.dynamicSmemBytes = kDecSmem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, a);
}
}  // namespace

cudaError_t launch_decode_layer(const Shape& s, const void* x, float* resid, double eps, const void* w_router,
                                const float* bias, const void* w_gate_up, const void* w_down, void* y,
                                int32_t* topk_idx, float* topk_w, int32_t* counts, float* losses, void* ws,
                                const Workspace& L, cudaStream_t st) {
  return launch_decode(s, x, resid, eps, 1, &w_router, &bias, &w_gate_up, &w_down, y, topk_idx, topk_w, counts, losses,
                       ws, L, st);
}

cudaError_t launch_decode_stack(const Shape& s, float* resid, double eps, int n_layers, const void* const* w_router,
                                const float* const* biases, const void* const* w_gate_up, const void* const* w_down,
                                int32_t* topk_idx, int32_t* counts, float* losses, void* ws, const Workspace& L,
                                cudaStream_t st) {
  for (int l0 = 0; l0 < n_layers; l0 += kDecMaxLayers) {
    const int n = n_layers - l0 < kDecMaxLayers ? n_layers - l0 : kDecMaxLayers;
    const cudaError_t e = launch_decode(
        s, nullptr, resid, eps, n, w_router + l0, biases != nullptr ? biases + l0 : nullptr, w_gate_up + l0,
        w_down + l0, nullptr, topk_idx != nullptr ? topk_idx + static_cast<int64_t>(l0) * s.T * s.k : nullptr,
        nullptr, counts != nullptr ? counts + static_cast<int64_t>(l0) * s.E : nullptr,
        losses != nullptr ? losses + 2 * l0 : nullptr, ws, L, st);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace moe
