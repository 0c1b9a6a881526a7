// The whole MoE layer for a decode-sized batch (T <= 8 tokens) in one
// persistent cooperative kernel: router, gate/up + SwiGLU, down and combine,
// optionally with the block's RMSNorm in front and the residual add behind;
// and a stack of such blocks (up to 16 per launch) in the same kernel.
//
// Method: the layer of "Mixture-of-experts LLMs from scratch with OLMoE",
// section 2 (softmax over all experts, top-k without renormalisation, each
// expert once on its tokens, weighted sum back) and section 3 (the Block:
// r + MoE(RMSNorm(r)) on an fp32 residual), the SwiGLU expert of "OLMoE
// Guide", "Top-8 Softmax Routing Formulation", and its losses ("Router
// Mechanics & Loss Formulations"). Section 6 of the lesson notes that at a
// batch of one token the layer reads only the k chosen experts' weights, so
// decoding is bound by streaming those weights; this kernel is built to keep
// that stream running.
//
// One CTA per SM (grid = SM count, cooperative launch, 16 warps). Per layer:
//   prologue  every CTA stages the T input rows in shared memory (RMSNorm of
//             the fp32 residual in fp64 when the input is the residual).
//   logits    the T*E router logits are spread over the grid, one warp per
//             (expert, token): fp64 sums of the exact bf16 x bf16 products,
//             written to the workspace. Grid barrier.
//   routing   every CTA reads the T*E logits and takes the same decisions:
//             each expert's rank among a token's logits gives the top-k at
//             once (equal logits: lower index first); softmax in fp32; the
//             tokens of each expert as a bit mask; CTA 0 writes the losses,
//             counts and the optional top-k outputs.
//   phase 1   this CTA's share of the touched experts' (expert, hidden row)
//             list, one gate/up row pair per job: the pair meets every token
//             that chose the expert; h = SiLU(g) * u is stored in bf16 (as the
//             grouped GEMM stores it). Grid barrier; every CTA copies h of all
//             slots into shared memory.
//   phase 2   this CTA's share of the output columns: the down-matrix rows of
//             each column's touched experts, a few rows per job; their dot
//             products with the h rows of the expert's tokens; then each
//             token's slot-ordered weighted sum is written once (bf16 y, or
//             added to the residual, whose columns this CTA owns).
// The streaming warps each own a few job buffers in shared memory, each with
// an mbarrier; lane 0 fetches a job as bulk copies of whole weight rows (the
// copy engine, not the load/store units, moves the bytes), the next jobs'
// bytes in flight while the current one is computed; so no register holds
// data in flight, and the copies of a warp's first phase-2 jobs go out before
// the grid barrier.
// Shares are dealt round-robin by rows (pairs, columns): every SM streams
// within one row of the same number of bytes, and at any moment the grid
// reads one contiguous stretch of each weight matrix (per-CTA contiguous
// ranges, read in lockstep, streamed at about half the rate on B200). The
// grid barrier is an arrival counter that the launch counts up (barrier j
// completes at j * grid) and that the last CTA to finish puts back to zero;
// every wait gives up after about a second, records a status and lets the
// kernel finish; a launch that finds the status word set does nothing
// (moe_get_device_status clears it and the counters).
#include <climits>

#include "moe_internal.h"
#include "sm100.cuh"

namespace moe {
namespace {

constexpr int kDecThreads = 512;
constexpr int kDecWarps = kDecThreads / 32;
constexpr int kDecMaxT = 8;
constexpr int kDecMaxE = 64;
constexpr int kDecSlots = kDecMaxT * kMaxTopK;  // (token, slot) pairs
constexpr int kDecMaxLayers = 16;               // layers of a stack per launch
constexpr size_t kDecSmemCap = 227 * 1024;      // dynamic shared memory of one CTA
constexpr int kMaxStreamWarps = kDecWarps;     // warps that fetch and compute jobs
constexpr int kDecBufsPerWarp = 2;             // job buffers of one streaming warp
constexpr int kDecJobBufs = kMaxStreamWarps * kDecBufsPerWarp;

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
  double* logits;            // [T, E] workspace
  int32_t* idx_out;          // [n_layers, T, k] or null
  float* w_out;              // [T, k] or null (single layer)
  int32_t* counts;           // [n_layers, E] or null
  float* losses;             // [n_layers, 2] or null
  float* losses_ws;          // [2] workspace copy (of the last layer)
  unsigned* bar;             // [0] grid-barrier arrivals, [1] CTAs finished
  int32_t* status;
  // shared-memory plan (byte offsets from the start of dynamic shared memory)
  uint32_t act_off, ps_off, buf_off;
  uint32_t job_bytes;        // one job buffer: a gate/up row pair, or rows_per_job down rows
  int rows_per_job;
  int n_stream;              // streaming warps (0 .. n_stream-1), kDecBufsPerWarp job buffers each
};

struct DecSmem {
  int sel_e[kDecSlots];
  float sel_w[kDecSlots];
  unsigned tokmask[kDecMaxE];      // bit t: token t chose the expert
  int slot_of[kDecMaxT][kDecMaxE]; // slot of expert e among token t's choices, or -1
  int touched[kDecMaxE];           // experts chosen by some token, ascending
  int n_touched;
  int ok;                          // result of the last grid barrier
  int abort;                       // a failure is recorded: do nothing
  unsigned bars;                   // grid barriers passed in this launch
  double wss[kDecWarps];           // each warp's sum of squares (of its input row)
  double rinv[kDecMaxT];           // 1 / sqrt(mean square + eps) of each input row
  double hd[kDecMaxT][kDecMaxE];   // logits (+ offset)
  long long key[kDecMaxT][kDecMaxE];  // the logits as ordered integers (order_key)
  float p[kDecMaxT][kDecMaxE];
  float lse[kDecMaxT];
  DecLayer layers[kDecMaxLayers];  // the launch's layer table
  uint64_t jbar[kDecJobBufs];      // completion of each job buffer (streaming warp w: w * kDecBufsPerWarp ...)
};

// One thread per CTA: grid barrier number `m.bars + 1` (sm100.cuh).
__device__ bool grid_sync_thread(DecSmem& m, unsigned* count, int32_t* status) {
  m.bars += 1;
  return grid_arrive_wait(count, m.bars * gridDim.x, status);  // at most 48 barriers of <= 1024 CTAs
}

// Grid barrier with every thread of the CTA taking part; the result is the
// same in every thread.
__device__ bool grid_barrier(DecSmem& m, const DecArgs& a) {
  __syncwarp();
  __syncthreads();
  if (threadIdx.x == 0) m.ok = grid_sync_thread(m, a.bar, a.status) ? 1 : 0;
  __syncthreads();
  return m.ok != 0;
}

// Eight bf16 values to fp32 (integer widening: the conversion instructions'
// pipe bounded this kernel's inner loops).
__device__ __forceinline__ void bf16x8(const uint4& q, float (&v)[8]) {
  const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float2 f = bf16x2_to_float2(w[j]);
    v[2 * j] = f.x;
    v[2 * j + 1] = f.y;
  }
}

// A double as a signed integer in the same order (-0 taken as +0), so that
// comparisons run on the integer pipe (FP64 runs at a small fraction of the
// FP32 rate on this part). A NaN becomes `nan_key`: the smallest integer for a
// value compared against (it beats nothing), the largest for the value being
// ranked (nothing beats it), as every comparison with NaN is false.
__device__ __forceinline__ long long order_key(double x, long long nan_key) {
  long long b = __double_as_longlong(x);
  if ((b & 0x7FFFFFFFFFFFFFFFll) == 0) b = 0;
  const long long k = b ^ ((b >> 63) & 0x7FFFFFFFFFFFFFFFll);
  return (b & 0x7FFFFFFFFFFFFFFFll) > 0x7FF0000000000000ll ? nan_key : k;
}

// acc + a.lo * x.lo, then + a.hi * x.hi: two fused multiply-adds of bf16
// operands into fp32 (each the exact product, one rounding), in element order.
__device__ __forceinline__ float fma2_bf16(uint32_t a, uint32_t x, float acc) {
  asm("{\n\t.reg .b16 al, ah, xl, xh;\n\t"
      "mov.b32 {al, ah}, %1;\n\t"
      "mov.b32 {xl, xh}, %2;\n\t"
      "fma.rn.f32.bf16 %0, al, xl, %0;\n\t"
      "fma.rn.f32.bf16 %0, ah, xh, %0;\n\t}"
      : "+f"(acc)
      : "r"(a), "r"(x));
  return acc;
}

// The same for two rows (gate and up) against one x pair.
__device__ __forceinline__ void fma2_bf16_pair(uint32_t g, uint32_t u, uint32_t x, float& ag, float& au) {
  asm("{\n\t.reg .b16 gl, gh, ul, uh, xl, xh;\n\t"
      "mov.b32 {gl, gh}, %2;\n\t"
      "mov.b32 {ul, uh}, %3;\n\t"
      "mov.b32 {xl, xh}, %4;\n\t"
      "fma.rn.f32.bf16 %0, gl, xl, %0;\n\t"
      "fma.rn.f32.bf16 %1, ul, xl, %1;\n\t"
      "fma.rn.f32.bf16 %0, gh, xh, %0;\n\t"
      "fma.rn.f32.bf16 %1, uh, xh, %1;\n\t}"
      : "+f"(ag), "+f"(au)
      : "r"(g), "r"(u), "r"(x));
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

// This CTA's share of the output columns, dealt round-robin (its l-th is
// CTA + G l; ncols of them), whose down rows (each column's touched experts in
// turn) form n2 jobs of rows_per_job rows. (The gate/up pairs are dealt by
// pair_index below.)
struct Share {
  int ncols;
  int rows2, n2;
};

__device__ Share cta_share(const DecArgs& a, int nt) {
  Share s;
  const int G = gridDim.x, c = blockIdx.x;
  s.ncols = c < a.d ? (a.d - c + G - 1) / G : 0;
  s.rows2 = s.ncols * nt;
  s.n2 = (s.rows2 + a.rows_per_job - 1) / a.rows_per_job;
  return s;
}

// The gate/up pair of streaming warp w's q-th job.
__device__ __forceinline__ int pair_index(int SW, int w, int q) {
  return static_cast<int>(blockIdx.x) + static_cast<int>(gridDim.x) * (w + SW * q);
}

// How many jobs streaming warp w has in phase 1.
__device__ __forceinline__ int pair_jobs(int SW, int w, int P) {
  const int first = pair_index(SW, w, 0);
  return first < P ? (P - first + static_cast<int>(gridDim.x) * SW - 1) / (static_cast<int>(gridDim.x) * SW) : 0;
}

// Output column of this CTA's l-th column.
__device__ __forceinline__ int cta_col(int l) { return static_cast<int>(blockIdx.x) + static_cast<int>(gridDim.x) * l; }

// A streaming warp's job buffers: job q goes to buffer q % kDecBufsPerWarp, whose
// mbarrier completes once per job. `ph` holds the parity each buffer's next
// wait expects, `pend` the buffers with a copy in flight; both live across
// layers. `live` turns false when a wait gave up (recorded in the status
// word): the warp then issues and computes nothing more.
struct JobPipe {
  uint64_t* bar;       // [kDecBufsPerWarp]
  unsigned char* buf;  // kDecBufsPerWarp buffers of job_bytes
  uint32_t job_bytes;
  uint32_t ph, pend;
  bool live;
  __device__ unsigned char* at(int q) const { return buf + static_cast<size_t>(q % kDecBufsPerWarp) * job_bytes; }
};

// Lane 0: warp w's job q (its phase-1 pairs w, w + SW, ... then its phase-2
// jobs w, w + SW, ...) into `buf` as bulk copies of whole weight rows,
// completing on the buffer's mbarrier; nothing when q is past the warp's last
// job. The caller has made the whole warp's reads of the buffer complete.
__device__ __forceinline__ void fetch_job(const DecArgs& a, const DecSmem& m, const DecLayer& Ly, const Share& sh,
                                          int nt, int w, int c1, int c2, int q, unsigned char* buf, uint64_t* bar) {
  const int SW = a.n_stream;
  if (q < c1) {
    const int p = pair_index(SW, w, q);
    const int u = p / a.f, i = p - u * a.f;
    const __nv_bfloat16* g = Ly.wgu + (static_cast<int64_t>(m.touched[u]) * 2 * a.f + i) * a.d;
    const uint32_t rb = static_cast<uint32_t>(a.d) * 2;
    fence_proxy_async_smem();
    mbar_arrive_expect_tx(bar, 2 * rb);
    bulk_load(buf, g, rb, bar);
    bulk_load(buf + rb, g + static_cast<int64_t>(a.f) * a.d, rb, bar);
  } else if (q < c1 + c2) {
    const int r0 = (w + SW * (q - c1)) * a.rows_per_job;
    const int nr = min(a.rows_per_job, sh.rows2 - r0);
    const uint32_t rb = static_cast<uint32_t>(a.f) * 2;
    int cl = r0 / nt, u = r0 - cl * nt;  // the row's column (of this CTA's) and touched-expert index
    fence_proxy_async_smem();
    mbar_arrive_expect_tx(bar, static_cast<uint32_t>(nr) * rb);
    for (int rr = 0; rr < nr; ++rr) {
      const __nv_bfloat16* row = Ly.wd + (static_cast<int64_t>(m.touched[u]) * a.d + cta_col(cl)) * a.f;
      bulk_load(buf + static_cast<size_t>(rr) * rb, row, rb, bar);
      if (++u == nt) {
        u = 0;
        ++cl;
      }
    }
  }
}

// The whole warp: issue job q (if it exists) into buffer q % kDecBufsPerWarp.
__device__ __forceinline__ void issue_job(const DecArgs& a, const DecSmem& m, const DecLayer& Ly, const Share& sh,
                                          int nt, int w, int lane, int c1, int c2, int q, JobPipe& jp) {
  if (!jp.live || q >= c1 + c2) return;
  const int b = q % kDecBufsPerWarp;
  __syncwarp();
  if (lane == 0) fetch_job(a, m, Ly, sh, nt, w, c1, c2, q, jp.at(q), jp.bar + b);
  jp.pend |= 1u << b;
}

// The whole warp: wait until buffer b's bytes have landed (every lane
// observes the completion itself). False when the warp is no longer live.
__device__ __forceinline__ bool await_buf(JobPipe& jp, int b, int32_t* status) {
  if (!jp.live) return false;
  const bool ok = __all_sync(0xffffffffu, mbar_wait(jp.bar + b, (jp.ph >> b) & 1u));
  jp.ph ^= 1u << b;
  jp.pend &= ~(1u << b);
  if (!ok) {
    report(status, DEV_WAIT_TIMEOUT_PRODUCER);
    jp.live = false;
  }
  return ok;
}

__device__ __forceinline__ bool await_job(JobPipe& jp, int q, int32_t* status) {
  return await_buf(jp, q % kDecBufsPerWarp, status);
}

// The whole warp, before the CTA leaves: no copy in flight into its buffers
// (each wait bounded).
__device__ __forceinline__ void drain_jobs(JobPipe& jp) {
  for (int b = 0; b < kDecBufsPerWarp; ++b)
    if ((jp.pend >> b) & 1u) {
      mbar_wait(jp.bar + b, (jp.ph >> b) & 1u);
      jp.ph ^= 1u << b;
    }
  jp.pend = 0;
  __syncwarp();
}

// Logit task q: expert q / T, token q % T, as an fp64 sum of the exact
// products (a bf16 x bf16 product is exact in fp32), lane l taking elements
// 8l + 256i, then a fixed reduction tree; written to the workspace. One warp.
__device__ __forceinline__ void logit_task(const DecArgs& a, const DecLayer& Ly, const __nv_bfloat16* act, int q,
                                           int lane) {
  const int T = a.T, d = a.d, E = a.E, nvd = d / 8;
  const int e = q / T, t = q - e * T;
  const uint4* wrow = reinterpret_cast<const uint4*>(Ly.wr + static_cast<int64_t>(e) * d);
  const uint4* xrow = reinterpret_cast<const uint4*>(act + static_cast<int64_t>(t) * d);
  double acc = 0.0;
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
        float wv[8], xv[8];
        bf16x8(wq[j], wv);
        bf16x8(xrow[v], xv);
#pragma unroll
        for (int i = 0; i < 8; ++i) acc += static_cast<double>(xv[i] * wv[i]);
      }
    }
  }
  acc = warp_sum_d(acc);
  if (lane == 0) a.logits[t * E + e] = acc + (Ly.bias != nullptr ? static_cast<double>(Ly.bias[e]) : 0.0);
}

// The tokens of a mask in ascending order: tok[j] is its j-th set bit
// (statically indexed, so the list stays in registers).
template <int NT>
__device__ __forceinline__ int mask_tokens(unsigned tm, int (&tok)[NT]) {
  const int n = __popc(tm);
#pragma unroll
  for (int j = 0; j < NT; ++j) {
    tok[j] = tm != 0u ? __ffs(tm) - 1 : 0;
    tm &= tm - 1u;
  }
  return n;
}

// Calls body.template run<n>() for the runtime count n in [1, NT], so the
// per-token accumulators are sized to the tokens present rather than to NT
// (predicated-off tokens would still take issue slots).
template <int N, int NT, class Body>
__device__ __forceinline__ void with_count(int n, Body& body) {
  if constexpr (N <= NT) {
    if (n == N)
      body.template run<N>();
    else
      with_count<N + 1, NT>(n, body);
  }
}

// Phase-1 job: gate/up row pair p (in `buf`) meets the n tokens of the pair's
// expert; h = SiLU(g) * u in bf16.
template <int NT>
struct PairBody {
  const DecArgs& a;
  const DecSmem& m;
  const uint4* g4;
  const uint4* x4;
  const int (&tok)[NT];
  int e, i, lane;
  template <int N>
  __device__ __forceinline__ void run() {
    const int nvd = a.d / 8;
    const uint4* u4 = g4 + nvd;
    float ag[N], au[N];
#pragma unroll
    for (int j = 0; j < N; ++j) ag[j] = au[j] = 0.f;
    for (int v = lane; v < nvd; v += 32) {
      const uint4 gq = g4[v], uq = u4[v];
#pragma unroll
      for (int j = 0; j < N; ++j) {
        const uint4 xq = x4[tok[j] * nvd + v];
        fma2_bf16_pair(gq.x, uq.x, xq.x, ag[j], au[j]);
        fma2_bf16_pair(gq.y, uq.y, xq.y, ag[j], au[j]);
        fma2_bf16_pair(gq.z, uq.z, xq.z, ag[j], au[j]);
        fma2_bf16_pair(gq.w, uq.w, xq.w, ag[j], au[j]);
      }
    }
#pragma unroll
    for (int j = 0; j < N; ++j) {
      const float g = warp_sum(ag[j]), uu = warp_sum(au[j]);
      if (lane == 0) {
        const int t = tok[j];
        a.h[static_cast<int64_t>(t * a.k + m.slot_of[t][e]) * a.f + i] = __float2bfloat16_rn(silu_fast(g) * uu);
      }
    }
  }
};

template <int NT>
__device__ __forceinline__ void pair_job(const DecArgs& a, const DecSmem& m, const __nv_bfloat16* act,
                                         const unsigned char* buf, int p, int lane) {
  const int u = p / a.f, i = p - u * a.f;
  const int e = m.touched[u];
  int tok[NT];
  const int n = mask_tokens<NT>(m.tokmask[e], tok);
  PairBody<NT> body{a, m, reinterpret_cast<const uint4*>(buf), reinterpret_cast<const uint4*>(act), tok, e, i, lane};
  with_count<1, NT>(n, body);
}

// One down row (in shared memory) against the h rows of its expert's n
// tokens (slots slot[j]): the row is widened once for all of them.
template <int NT>
struct DownBody {
  const uint4* w4;
  const uint4* h4;
  const int (&slot)[NT];
  float* ps;  // this row's column: ps[slot]
  int nvf, lane;
  template <int N>
  __device__ __forceinline__ void run() {
    float acc[N];
#pragma unroll
    for (int j = 0; j < N; ++j) acc[j] = 0.f;
    for (int v = lane; v < nvf; v += 32) {
      const uint4 wq = w4[v];
#pragma unroll
      for (int j = 0; j < N; ++j) {
        const uint4 hq = h4[slot[j] * nvf + v];
        acc[j] = fma2_bf16(wq.x, hq.x, acc[j]);
        acc[j] = fma2_bf16(wq.y, hq.y, acc[j]);
        acc[j] = fma2_bf16(wq.z, hq.z, acc[j]);
        acc[j] = fma2_bf16(wq.w, hq.w, acc[j]);
      }
    }
#pragma unroll
    for (int j = 0; j < N; ++j) {
      const float r = warp_sum(acc[j]);
      if (lane == 0) ps[slot[j]] = r;
    }
  }
};

// Phase-2 job g of this CTA (down rows g * rows_per_job ..., in `buf`): each
// row's dot products with the h rows (shared memory) of its expert's tokens.
template <int NT>
__device__ __forceinline__ void down_job(const DecArgs& a, const DecSmem& m, const Share& sh, int nt,
                                         const __nv_bfloat16* act, float* ps, const unsigned char* buf, int g,
                                         int lane) {
  const int k = a.k, nvf = a.f / 8, TK = a.T * k;
  const int r0 = g * a.rows_per_job;
  const int nr = min(a.rows_per_job, sh.rows2 - r0);
  int cl = r0 / nt, u = r0 - cl * nt;  // the row's column (of this CTA's) and touched-expert index
  for (int rr = 0; rr < nr; ++rr) {
    const int e = m.touched[u];
    int slot[NT];
    const int n = mask_tokens<NT>(m.tokmask[e], slot);
#pragma unroll
    for (int j = 0; j < NT; ++j) slot[j] = slot[j] * k + max(m.slot_of[slot[j]][e], 0);
    DownBody<NT> body{reinterpret_cast<const uint4*>(buf) + rr * nvf, reinterpret_cast<const uint4*>(act), slot,
                      ps + cl * TK, nvf, lane};
    with_count<1, NT>(n, body);
    if (++u == nt) {
      u = 0;
      ++cl;
    }
  }
}

// The block's RMSNorm (unit weight) of the fp32 residual rows into the bf16
// layer input `act`, all rows at once: 512 / T (rounded down to a power of
// two, at least 64) threads per row. In fp64: each thread's squares in
// element order, a butterfly within each warp, the row's warps in order; one
// reciprocal root per row and a product per element, rounded to fp32, then to
// bf16 (as the separate RMSNorm kernel rounds). The row is read twice, from
// L2, so that no register holds it across the block barrier.
__device__ __forceinline__ void stage_rmsnorm(const DecArgs& a, DecSmem& m, __nv_bfloat16* act) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int T = a.T, d = a.d, nv = d / 4;
  const int tpr = T <= 1 ? kDecThreads : T <= 2 ? kDecThreads / 2 : T <= 4 ? kDecThreads / 4 : kDecThreads / 8;
  const int row = tid / tpr, p = tid - row * tpr;
  const bool live = row < T;
  const float4* r = reinterpret_cast<const float4*>(a.resid + static_cast<int64_t>(row) * d);
  double ss = 0.0;
  if (live) {
#pragma unroll 4
    for (int i = p; i < nv; i += tpr) {
      const float4 q = __ldcg(r + i);
      ss = fma(static_cast<double>(q.x), static_cast<double>(q.x), ss);
      ss = fma(static_cast<double>(q.y), static_cast<double>(q.y), ss);
      ss = fma(static_cast<double>(q.z), static_cast<double>(q.z), ss);
      ss = fma(static_cast<double>(q.w), static_cast<double>(q.w), ss);
    }
  }
  ss = warp_sum_d(ss);  // a warp lies within one row
  if (lane == 0) m.wss[warp] = ss;
  __syncthreads();
  if (tid < T) {
    const int wpr = tpr / 32;
    double sum = 0.0;
    for (int w = tid * wpr; w < (tid + 1) * wpr; ++w) sum += m.wss[w];
    m.rinv[tid] = 1.0 / sqrt(sum / static_cast<double>(d) + a.eps);
  }
  __syncthreads();
  if (live) {
    const double inv = m.rinv[row];
#pragma unroll 4
    for (int i = p; i < nv; i += tpr) {
      const float4 q = __ldcg(r + i);
      uint2 o;
      o.x = pack_bf16x2(static_cast<float>(static_cast<double>(q.x) * inv), static_cast<float>(static_cast<double>(q.y) * inv));
      o.y = pack_bf16x2(static_cast<float>(static_cast<double>(q.z) * inv), static_cast<float>(static_cast<double>(q.w) * inv));
      *reinterpret_cast<uint2*>(act + static_cast<int64_t>(row) * d + 4 * i) = o;
    }
  }
}

// NT: tokens the phase-1 accumulators are sized for (1, 2, 4 or 8; T <= NT).
template <int NT>
__global__ void __launch_bounds__(kDecThreads, 1) decode_layer_kernel(const __grid_constant__ DecArgs a) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  DecSmem& m = *reinterpret_cast<DecSmem*>(smem_raw);
  __nv_bfloat16* act = reinterpret_cast<__nv_bfloat16*>(smem_raw + a.act_off);  // x [T, d], later h [T*k, f]
  float* ps = reinterpret_cast<float*>(smem_raw + a.ps_off);  // [ncols][T*k] down-row dot products
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int T = a.T, d = a.d, E = a.E, k = a.k;
  const int TK = T * k;
  const int nvd = d / 8, nvf = a.f / 8;  // 16-byte vectors per row
  const int G = gridDim.x;
  const int SW = a.n_stream;

  if (tid == 0) {
    m.abort = *reinterpret_cast<volatile int32_t*>(a.status) != 0 ? 1 : 0;
    m.bars = 0;
  }
  if (tid < kDecMaxLayers) m.layers[tid] = a.layer[tid];
  if (tid < kDecJobBufs) mbar_init(&m.jbar[tid], 1);
  fence_mbar_init();
  __syncthreads();
  if (m.abort != 0) return;  // a failure is recorded: the counters may be stale
  JobPipe jp{m.jbar + warp * kDecBufsPerWarp,
             smem_raw + a.buf_off + static_cast<size_t>(warp) * kDecBufsPerWarp * a.job_bytes, a.job_bytes, 0u, 0u,
             warp < SW};

#pragma unroll 1
  for (int l = 0; l < a.n_layers; ++l) {
    const DecLayer& Ly = m.layers[l];
    // this CTA's logit tasks: task q = warp * G + CTA, expert q / T, token q % T
    const int q = warp * G + blockIdx.x;
    const bool has_task = q < T * E;
    // a layer of a stack reads the residual the previous layer completed
    if (l > 0 && !grid_barrier(m, a)) return;
    int32_t* const idx_out = a.idx_out != nullptr ? a.idx_out + static_cast<int64_t>(l) * TK : nullptr;
    int32_t* const counts = a.counts != nullptr ? a.counts + static_cast<int64_t>(l) * E : nullptr;
    float* const losses = a.losses != nullptr ? a.losses + 2 * l : nullptr;

    // ---- prologue: the T input rows, bf16, in shared memory
    if (a.resid != nullptr) {
      stage_rmsnorm(a, m, act);
    } else {
      const uint4* src = reinterpret_cast<const uint4*>(a.x);
      uint4* dst = reinterpret_cast<uint4*>(act);
      for (int i = tid; i < T * nvd; i += kDecThreads) dst[i] = __ldg(src + i);
    }
    if (tid < kDecMaxE) m.tokmask[tid] = 0u;
    if (tid < kDecSlots) m.sel_e[tid] = 0;  // defined even if non-finite logits leave a slot unranked
    for (int i = tid; i < (d / G + 1) * TK; i += kDecThreads) ps[i] = 0.f;
    __syncthreads();

    // ---- logits: fp64 sums of the exact products (a bf16 x bf16 product is
    //      exact in fp32), lane l taking elements 8l + 256i; fixed reduction tree
    if (has_task) logit_task(a, Ly, act, q, lane);
    if (!grid_barrier(m, a)) return;
    for (int i = tid; i < T * E; i += kDecThreads) {
      const double h = __ldcg(a.logits + i);
      m.hd[i / E][i % E] = h;
      m.key[i / E][i % E] = order_key(h, LLONG_MIN);
    }
    __syncthreads();

    // ---- routing (every CTA): warp t takes token t; lane l holds experts l, l + 32
    if (warp < T) {
      const int t = warp;
      const int e0 = lane, e1 = lane + 32;
      const double h0 = e0 < E ? m.hd[t][e0] : -INFINITY;
      const double h1 = e1 < E ? m.hd[t][e1] : -INFINITY;
      // rank by (logit descending, index ascending): the experts ranked below k
      // are the choice (branch-free integer compares of the keys; a short
      // loop, as once-per-layer code runs from a cold instruction cache)
      const long long k0 = order_key(h0, LLONG_MAX), k1 = order_key(h1, LLONG_MAX);
      int r0 = 0, r1 = 0;
#pragma unroll 4
      for (int e = 0; e < E; ++e) {
        const long long v = m.key[t][e];
        r0 += static_cast<int>(v > k0) | (static_cast<int>(v == k0) & static_cast<int>(e < e0));
        r1 += static_cast<int>(v > k1) | (static_cast<int>(v == k1) & static_cast<int>(e < e1));
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
      // softmax over all experts in fp32 from the logits
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
      // weights, lane j taking slot j (renormalised: over the k chosen, summed in slot order)
      const int ej = lane < k ? m.sel_e[t * k + lane] : 0;
      const float pj = lane < k ? m.p[t][ej] : 0.f;
      float den = 0.f;
      if (a.renorm)
        for (int j = 0; j < k; ++j) den += __shfl_sync(0xffffffffu, pj, j);
      if (lane < k) {
        const float w = a.renorm ? pj / den : pj;
        m.sel_w[t * k + lane] = w;
        if (blockIdx.x == 0) {
          if (idx_out != nullptr) idx_out[t * k + lane] = ej;
          if (a.w_out != nullptr) a.w_out[t * k + lane] = w;
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
    const Share sh = cta_share(a, nt);

    // this warp's jobs: phase-1 pairs warp, warp + SW, ... then phase-2 jobs likewise
    const bool streams = warp < SW;
    const int c1 = streams ? pair_jobs(SW, warp, nt * a.f) : 0;
    const int c2 = streams && warp < sh.n2 ? (sh.n2 - warp + SW - 1) / SW : 0;
    if (streams) {
      for (int qq = 0; qq < kDecBufsPerWarp; ++qq) issue_job(a, m, Ly, sh, nt, warp, lane, c1, c2, qq, jp);
      // ---- phase 1: the next jobs' copies in flight while this one is computed
      for (int qq = 0; qq < c1; ++qq) {
        if (await_job(jp, qq, a.status)) pair_job<NT>(a, m, act, jp.at(qq), pair_index(SW, warp, qq), lane);
        issue_job(a, m, Ly, sh, nt, warp, lane, c1, c2, qq + kDecBufsPerWarp, jp);
      }
    }
    // every CTA's h is written before any CTA reads it
    if (!grid_barrier(m, a)) {
      drain_jobs(jp);  // no copy in flight when the CTA leaves
      return;
    }
    // the next layer's router rows of this warp's logit task, asked into L2
    // now so that its logits do not wait on DRAM
    if (lane == 0 && l + 1 < a.n_layers) {
      const int q1 = warp * G + static_cast<int>(blockIdx.x);
      if (q1 < T * E)
        bulk_prefetch_l2(m.layers[l + 1].wr + static_cast<int64_t>(q1 / T) * d, static_cast<uint32_t>(d) * 2);
    }
    {  // h of all slots into shared memory (x is dead)
      const uint4* src = reinterpret_cast<const uint4*>(a.h);
      uint4* dst = reinterpret_cast<uint4*>(act);
      for (int i = tid; i < TK * nvf; i += kDecThreads) dst[i] = __ldcg(src + i);
    }
    __syncthreads();

    // ---- phase 2
    if (streams) {
      for (int qq = c1; qq < c1 + c2; ++qq) {
        if (await_job(jp, qq, a.status)) down_job<NT>(a, m, sh, nt, act, ps, jp.at(qq), warp + SW * (qq - c1), lane);
        issue_job(a, m, Ly, sh, nt, warp, lane, c1, c2, qq + kDecBufsPerWarp, jp);
      }
      drain_jobs(jp);
    }
    __syncthreads();
    // each (column, token): the weighted sum over the token's slots in slot order
    for (int it = tid; it < sh.ncols * T; it += kDecThreads) {
      const int t = it / sh.ncols, cl = it - t * sh.ncols;
      float acc = 0.f;
      for (int j = 0; j < k; ++j) acc = fmaf(m.sel_w[t * k + j], ps[cl * TK + t * k + j], acc);
      const int64_t o = static_cast<int64_t>(t) * d + cta_col(cl);
      if (a.resid != nullptr)
        a.resid[o] = __ldcg(a.resid + o) + acc;
      else
        a.y[o] = __float2bfloat16_rn(acc);
    }
    __syncthreads();
  }  // layers

  // every CTA has passed its last grid barrier: the last one out puts the counters back to zero
  if (tid == 0) grid_exit(a.bar);
}

// Shared-memory plan for T tokens on a grid of G CTAs: bookkeeping, the
// activation rows (x, later h), the per-column dot products, and
// kDecBufsPerWarp job buffers for as many streaming warps (up to 16) as fit.
struct DecPlan {
  uint32_t act_off, ps_off, buf_off, job_bytes;
  int rows_per_job, n_stream;
  size_t smem;
};

size_t align128(size_t v) { return (v + 127) / 128 * 128; }

bool decode_plan(const Shape& s, int G, DecPlan* p) {
  const size_t misc = align128(sizeof(DecSmem));
  const size_t act = align128(std::max(static_cast<size_t>(s.T) * s.d * 2, static_cast<size_t>(s.T) * s.k * s.f * 2));
  const size_t ps = align128(static_cast<size_t>(s.d / G + 1) * s.T * s.k * 4);
  const size_t jb = align128(std::max(static_cast<size_t>(s.d) * 4, static_cast<size_t>(s.f) * 2));
  const size_t nb = kDecBufsPerWarp;
  if (misc + act + ps + nb * jb > kDecSmemCap) return false;
  const size_t sw = std::min<size_t>(kMaxStreamWarps, (kDecSmemCap - misc - act - ps) / (nb * jb));
  p->act_off = static_cast<uint32_t>(misc);
  p->ps_off = static_cast<uint32_t>(misc + act);
  p->buf_off = static_cast<uint32_t>(misc + act + ps);
  p->job_bytes = static_cast<uint32_t>(jb);
  p->rows_per_job = static_cast<int>(jb / (static_cast<size_t>(s.f) * 2));
  p->n_stream = static_cast<int>(sw);
  p->smem = misc + act + ps + nb * sw * jb;
  return true;
}

}  // namespace

bool decode_supported(const Shape& s) {
  if (s.fp32 || s.T < 1 || s.T > kDecMaxT || s.E > kDecMaxE || s.k > kMaxTopK) return false;
  if (s.d % 8 != 0 || s.f % 8 != 0) return false;  // 16-byte rows
  const size_t rows = std::max(static_cast<size_t>(s.T) * s.d, static_cast<size_t>(s.T) * s.k * s.f) * 2;
  // the staged rows (x, later h) and at least two job buffers in shared memory
  if (rows + static_cast<size_t>(s.d) * 8 > 192 * 1024) return false;
  if (static_cast<size_t>(s.T) * s.E * 8 > static_cast<size_t>(s.P) * s.d * s.esize) return false;  // logits scratch
  DecPlan p;
  return decode_plan(s, device_sm_count(), &p);
}

namespace {
// One cooperative launch over `n` (<= kDecMaxLayers) layers.
cudaError_t launch_decode(const Shape& s, const void* x, float* resid, double eps, int n,
                          const void* const* w_router, const float* const* biases, const void* const* w_gate_up,
                          const void* const* w_down, void* y, int32_t* topk_idx, float* topk_w, int32_t* counts,
                          float* losses, void* ws, const Workspace& L, cudaStream_t st) {
  // the accumulator count follows the batch: fewer live registers for small T
  static std::atomic<size_t> set_smem[4][kMaxDevices];
  void (*kern)(DecArgs) = s.T <= 1   ? decode_layer_kernel<1>
                          : s.T <= 2 ? decode_layer_kernel<2>
                          : s.T <= 4 ? decode_layer_kernel<4>
                                     : decode_layer_kernel<8>;
  const int which = s.T <= 1 ? 0 : s.T <= 2 ? 1 : s.T <= 4 ? 2 : 3;
  if (n < 1 || n > kDecMaxLayers) return cudaErrorInvalidValue;
  const int G = device_sm_count();
  DecPlan plan;
  if (!decode_plan(s, G, &plan)) return cudaErrorInvalidValue;
  cudaError_t e = raise_smem_limit(reinterpret_cast<const void*>(kern), kDecSmemCap, set_smem[which]);
  if (e != cudaSuccess) return e;
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
  a.logits = at<double>(ws, L.x_perm);
  a.idx_out = topk_idx;
  a.w_out = topk_w;
  a.counts = counts;
  a.losses = losses;
  a.losses_ws = at<float>(ws, L.losses);
  a.bar = reinterpret_cast<unsigned*>(at<int32_t>(ws, L.ctrl) + 3);
  a.status = at<int32_t>(ws, L.ctrl);
  a.act_off = plan.act_off;
  a.ps_off = plan.ps_off;
  a.buf_off = plan.buf_off;
  a.job_bytes = plan.job_bytes;
  a.rows_per_job = plan.rows_per_job;
  a.n_stream = plan.n_stream;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(G));
  cfg.blockDim = dim3(kDecThreads);
  cfg.dynamicSmemBytes = plan.smem;
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
