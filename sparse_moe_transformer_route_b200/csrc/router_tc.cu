// Tensor-core router for bf16 layers with up to 64 experts: logits on tcgen05,
// softmax over all experts, top-k without renormalisation, both loss partials
// and the dispatch ranking, in one kernel.
//
// Method: "Mixture-of-experts LLMs from scratch with OLMoE", section 2
// (softmax over all experts, then the k largest probabilities are both the
// choice and the weights; OLMoE does not renormalise, section 3) and section 3
// MoE.forward (fp32 scores, optional per-expert offset); "OLMoE Guide",
// "Router Mechanics & Loss Formulations" (f_i, P_i, L_lb, L_z).
//
// One CTA takes 32 tokens (one dispatch chunk), so a 4096-token layer spreads
// over 128 SMs:
//   warp 0     TMA loads of x [32 x 64] and W_r [E_pad x 64] per K step into a
//              16-deep ring. The MMA reads a 128-row A operand; rows 32..127
//              are whatever lies in shared memory after the 32 loaded rows,
//              and their accumulator rows are never read.
//   warp 1     tcgen05.mma M=128 N=E_pad K=16, fp32 accumulator in TMEM
//   warps 2..5 epilogue. Warp 4 (TMEM lanes 0..31) copies the 32 tokens'
//              logits to shared memory; then a quad of threads takes each
//              token, 16 experts per thread: softmax with quad reductions, the
//              top k+3 in fp32 by quad arg-max, and the top-k decided with
//              exact logits where fp32 cannot: every run of neighbours among
//              the first k+1 whose fp32 gaps are under 2e-4 * max(1, |logit|)
//              (far above the accumulation error of a 2048-long fp32 sum of
//              exact bf16 products) is recomputed exactly (fp64 sums of exact
//              products) and re-ranked; ties in the exact values go to the
//              lower expert index. Probabilities, weights and the log-normaliser
//              come from the fp32 logits.
// A 32-bit mask per expert of the tokens that chose it gives each (token,
// slot) pair its rank inside the chunk. The last CTA to finish scans the
// per-chunk counts (block by block, through shared memory) into chunk bases,
// the bincount offsets and the padded group starts, and reduces the loss
// partials. Every sum runs in a fixed order, so the results are deterministic.
// For expert-choice routing the same kernels stop after the probabilities and
// the log-normaliser (launch_router_probs); the selection runs afterwards.
#include <cfloat>
#include <cmath>

#include "moe_internal.h"
#include "sm100.cuh"

namespace moe {
namespace {

constexpr int kTile = kDispatchChunk;  // 32 tokens
constexpr int kThreads = 192;
constexpr int kMaxE = 64;
constexpr int kMaxSel = kMaxTopK + 3;
constexpr int kAload = kTile * 128;                      // bytes of A loaded per stage
constexpr int kStageMax = kAload + kMaxE * 128;          // 12 KB
// ring bytes for S stages, plus the over-read of the last stage's A
constexpr int ring_bytes(int S) { return S * kStageMax + 16 * 1024; }
constexpr int kLogitStride = kMaxE + 1;
constexpr int kScanBlock = 128;                          // chunks scanned per pass in the last CTA
constexpr size_t kMiscBytes = 4096;
constexpr size_t smem_bytes(int S) { return 1024 + static_cast<size_t>(ring_bytes(S)) + kMiscBytes; }
static_assert(kTile == 32, "one mask word per expert");
static_assert(kScanBlock * kMaxE * 8 <= ring_bytes(7), "scan block fits in the smallest ring");

struct RArgs {
  int64_t T;
  int d, E, k, NP;
  const float* bias;
  const __nv_bfloat16* x;
  const __nv_bfloat16* w;
  int32_t* idx_out;
  float* w_out;
  float* probs;
  float* lse_out;
  int32_t* local_rank;
  int32_t* chunk_count;
  int32_t* chunk_base;
  float* psum_part;
  double* zsum_part;
  int32_t* counts_ws;
  int32_t* counts_user;
  float* losses_ws;
  float* losses_user;
  int32_t* offsets_ws;
  int32_t* gs_ws;
  int32_t* ticket;
  int32_t* status;
  float* logit_part;  // split form: [ksplit][T][E] partial logits
  int ksplit;         // split form: K ranges per 128-token tile
  int renorm;         // weights divided by the sum of the k chosen probabilities
  int probs_only;     // stop after p and lse (expert choice selects from p afterwards)
};

__device__ __forceinline__ void epi_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

__device__ __forceinline__ float near_gap(float v) { return 2e-4f * fmaxf(1.0f, fabsf(v)); }

// Arg-max across the 4 threads of a quad: larger value wins, equal values go to the lower index.
// Quads may diverge (near-ties, the ragged last tile), so every quad shuffle
// names only its own four lanes.
__device__ __forceinline__ unsigned quad_mask() { return 0xFu << ((threadIdx.x & 31) & 28); }

template <typename V>
__device__ __forceinline__ void quad_argmax(V& v, int& i) {
  const unsigned qm = quad_mask();
#pragma unroll
  for (int o = 1; o <= 2; o <<= 1) {
    const V ov = __shfl_xor_sync(qm, v, o);
    const int oi = __shfl_xor_sync(qm, i, o);
    if (ov > v || (ov == v && oi < i)) {
      v = ov;
      i = oi;
    }
  }
}

// <x_t, W_r[e]> from exact products of bf16 inputs, summed in fp64 by a whole
// warp: lane l takes elements 8l + 256i; the loads of up to 16 steps are issued
// before any arithmetic so the row pair costs about one memory round trip. The
// lane sums are combined by a fixed shuffle tree (every lane gets the result).
__device__ __forceinline__ double exact_logit_warp(const __nv_bfloat16* xr, const __nv_bfloat16* wr, int d,
                                                   int lane) {
  constexpr int kBatch = 16;
  double acc = 0.0;
  for (int base = lane * 8; base < d; base += 256 * kBatch) {
    uint4 xv[kBatch], wv[kBatch];
#pragma unroll
    for (int b = 0; b < kBatch; ++b) {
      const int i = base + 256 * b;
      if (i < d) {
        xv[b] = *reinterpret_cast<const uint4*>(xr + i);
        wv[b] = *reinterpret_cast<const uint4*>(wr + i);
      }
    }
#pragma unroll
    for (int b = 0; b < kBatch; ++b) {
      if (base + 256 * b < d) {
        const uint32_t xa[4] = {xv[b].x, xv[b].y, xv[b].z, xv[b].w}, wa[4] = {wv[b].x, wv[b].y, wv[b].z, wv[b].w};
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const float2 xf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&xa[c]));
          const float2 wf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&wa[c]));
          acc = fma(static_cast<double>(xf.x), static_cast<double>(wf.x), acc);
          acc = fma(static_cast<double>(xf.y), static_cast<double>(wf.y), acc);
        }
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  return acc;
}

// The router's work once the tile's 32 logit rows are in shared memory (S),
// shared by the fused kernel and the epilogue-only kernel. 128 threads
// (tid 0..127, lane = tid % 32) synchronise on named barrier 1; the last CTA
// of the grid also scans the per-chunk counts through `ring` (kScanBlock*E*8 bytes).
struct EpiSmem {
  float* S;
  float* P;
  int32_t* chosen;
  uint32_t* queue;
  double* exact;
  int32_t* qn;
  uint32_t* mask;
  float* lse_s;
  int32_t* s_last;
  int32_t* tot;
  double* tot_p;
  double* zred;
  unsigned char* ring;
};

__device__ __forceinline__ void router_epilogue(const RArgs& a, const EpiSmem& sm, int64_t t0, int tid, int lane) {
  float* S = sm.S;
  float* P = sm.P;
  int32_t* chosen = sm.chosen;
  uint32_t* queue = sm.queue;
  double* exact = sm.exact;
  int32_t* qn = sm.qn;
  uint32_t* mask = sm.mask;
  float* lse_s = sm.lse_s;
  int32_t* s_last = sm.s_last;
  int32_t* tot = sm.tot;
  double* tot_p = sm.tot_p;
  double* zred = sm.zred;
  unsigned char* ring = sm.ring;
  const int E = a.E, k = a.k;
  // ---- a quad per token: thread qp holds experts 16*qp .. 16*qp+15
  const int r = tid >> 2, qp = tid & 3;
  const int64_t t = t0 + r;
  const bool valid = t < a.T;  // the whole quad agrees
  const int eb = qp * 16;
  float h[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) h[i] = S[r * kLogitStride + eb + i];
  float m = -INFINITY;
#pragma unroll
  for (int i = 0; i < 16; ++i) m = fmaxf(m, h[i]);
  const unsigned qm = quad_mask();
  m = fmaxf(m, __shfl_xor_sync(qm, m, 1));
  m = fmaxf(m, __shfl_xor_sync(qm, m, 2));
  float ex[16];  // exp(h - m), computed once for the sum and the probabilities
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    ex[i] = (eb + i < E) ? expf(h[i] - m) : 0.f;
    s += ex[i];
  }
  s += __shfl_xor_sync(qm, s, 1);
  s += __shfl_xor_sync(qm, s, 2);
  const float lse = m + logf(s);
  {
    float pv[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) pv[i] = valid ? ex[i] / s : 0.f;
#pragma unroll
    for (int i = 0; i < 16; ++i) P[r * kMaxE + eb + i] = pv[i];
    if (valid && eb < E) {
      float* dst = a.probs + t * E + eb;
      if (eb + 16 <= E) {
#pragma unroll
        for (int i = 0; i < 4; ++i)
          reinterpret_cast<float4*>(dst)[i] = make_float4(pv[4 * i], pv[4 * i + 1], pv[4 * i + 2], pv[4 * i + 3]);
      } else {
        for (int i = 0; i < E - eb; ++i) dst[i] = pv[i];
      }
    }
  }
  if (qp == 0) {
    lse_s[r] = valid ? lse : 0.f;
    if (valid) a.lse_out[t] = lse;
  }
  if (a.probs_only) return;  // uniform over the CTA

  // ---- top (k+3) in fp32 by quad arg-max (uniform within the quad); nearm bit j
  //      marks ranks j and j+1 as closer than the fp32 uncertainty
  const int nsel = min(k + 3, E);
  int ord[kMaxSel];
  float val[kMaxSel];
  uint32_t taken = 0;  // bit i: expert eb + i chosen
  uint32_t nearm = 0;
#pragma unroll
  for (int j = 0; j < kMaxSel; ++j) {
    if (j < nsel) {
      float v = -INFINITY;
      int bi = 0x7fffffff;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        if (eb + i < E && !((taken >> i) & 1u) && (bi == 0x7fffffff || h[i] > v)) {
          v = h[i];
          bi = eb + i;
        }
      }
      quad_argmax(v, bi);
      if (bi - eb >= 0 && bi - eb < 16) taken |= 1u << (bi - eb);
      ord[j] = bi;
      val[j] = v;
      if (j > 0 && val[j - 1] - v < near_gap(val[j - 1])) nearm |= 1u << (j - 1);
    }
  }
  float hv[kMaxSel];  // fp32 logit of ord[j], kept for the weights
#pragma unroll
  for (int j = 0; j < kMaxSel; ++j) hv[j] = val[j];
  // Slow path (rare): some run of near-equal neighbours decides a slot order or
  // the k-th choice. It works on local copies so the common path stays in registers.
  const bool slow = valid && (nearm & ((1u << k) - 1u)) != 0;
  bool fallback = false;
  int run_a[kMaxSel], run_b[kMaxSel];
  int nrun = 0;
  int oloc[kMaxSel];
  float hloc[kMaxSel];
  if (slow) {
#pragma unroll
    for (int j = 0; j < kMaxSel; ++j) {
      oloc[j] = ord[j];
      hloc[j] = hv[j];
    }
    int jj = 0;
    while (jj < nsel - 1) {
      if ((nearm >> jj) & 1u) {
        int b = jj + 1;
        while (b < nsel - 1 && ((nearm >> b) & 1u)) ++b;
        if (jj <= k - 1) {
          if (b == nsel - 1 && nsel < E) {
            fallback = true;
            break;
          }
          run_a[nrun] = jj;
          run_b[nrun] = b;
          ++nrun;
        }
        jj = b;
      } else {
        ++jj;
      }
    }
  }
  // queue the (token, expert) pairs whose exact logits are needed
  int nitems = 0;
  if (fallback) {
    nitems = E;
  } else {
    for (int i = 0; i < nrun; ++i) nitems += run_b[i] - run_a[i] + 1;
  }
  int qbase = 0;
  if (qp == 0 && nitems > 0) qbase = atomicAdd(qn, nitems);
  qbase = __shfl_sync(qm, qbase, lane & ~3);
  if (fallback) {
    for (int e = qp; e < E; e += 4) queue[qbase + e] = (static_cast<uint32_t>(r) << 8) | static_cast<uint32_t>(e);
  } else if (nrun > 0) {
    int p = 0;
    for (int i = 0; i < nrun; ++i)
      for (int y = run_a[i]; y <= run_b[i]; ++y, ++p)
        if ((p & 3) == qp) queue[qbase + p] = (static_cast<uint32_t>(r) << 8) | static_cast<uint32_t>(oloc[y]);
  }
  epi_sync();
  // ---- exact logits of the queued pairs: a warp per pair, all loads in flight together
  {
    const int nq = *qn;
    const int ew = tid >> 5;
    for (int it = ew; it < nq; it += 4) {
      const uint32_t code = queue[it];
      const int rr = static_cast<int>(code >> 8), e = static_cast<int>(code & 255u);
      const double v = exact_logit_warp(a.x + (t0 + rr) * a.d, a.w + static_cast<int64_t>(e) * a.d, a.d, lane);
      if (lane == 0) exact[it] = v + (a.bias != nullptr ? static_cast<double>(a.bias[e]) : 0.0);
    }
  }
  epi_sync();
  if (slow) {
    if (!fallback) {  // re-rank each run by its exact logits (ties: lower expert index)
      int p = qbase;
      for (int i = 0; i < nrun; ++i) {
        const int ra = run_a[i], rb = run_b[i];
        double ex[kMaxSel];
        for (int y = ra; y <= rb; ++y) ex[y] = exact[p++];
        for (int x1 = ra + 1; x1 <= rb; ++x1) {
          const double ve = ex[x1];
          const int oe = oloc[x1];
          const float he = hloc[x1];
          int y = x1 - 1;
          while (y >= ra && (ex[y] < ve || (ex[y] == ve && oloc[y] > oe))) {
            ex[y + 1] = ex[y];
            oloc[y + 1] = oloc[y];
            hloc[y + 1] = hloc[y];
            --y;
          }
          ex[y + 1] = ve;
          oloc[y + 1] = oe;
          hloc[y + 1] = he;
        }
      }
    } else {  // a run reaches past rank k+3: rank every expert by its exact logit
      double xe[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) xe[i] = (eb + i < E) ? exact[qbase + eb + i] : -INFINITY;
      uint32_t tk = 0;
      for (int j = 0; j < k; ++j) {
        double v = -INFINITY;
        int bi = 0x7fffffff;
        float hb = 0.f;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          if (eb + i < E && !((tk >> i) & 1u) && (bi == 0x7fffffff || xe[i] > v)) {
            v = xe[i];
            bi = eb + i;
            hb = h[i];
          }
        }
        quad_argmax(v, bi);
        if (bi - eb >= 0 && bi - eb < 16) tk |= 1u << (bi - eb);
        oloc[j] = bi;
        // the fp32 logit of the winner, from the thread that holds it
        const int owner = (lane & ~3) | ((bi >> 4) & 3);
        hloc[j] = __shfl_sync(qm, (bi >= eb && bi < eb + 16) ? hb : 0.f, owner);
      }
    }
#pragma unroll
    for (int j = 0; j < kMaxSel; ++j) {
      ord[j] = oloc[j];
      hv[j] = hloc[j];
    }
  }
  // ---- outputs: thread qp writes slots qp, qp+4, ...
  if (valid) {
    // the weights' denominator: all experts' exponentials, or (renormalised)
    // the k chosen ones summed in slot order
    float den = s;
    if (a.renorm) {
      den = 0.f;
#pragma unroll
      for (int j = 0; j < kMaxTopK; ++j)
        if (j < k) den += expf(hv[j] - m);
    }
#pragma unroll
    for (int j = 0; j < kMaxTopK; ++j) {
      if (j < k && (j & 3) == qp) {
        const int e = ord[j];
        a.idx_out[t * k + j] = e;
        a.w_out[t * k + j] = expf(hv[j] - m) / den;
        chosen[r * kMaxTopK + j] = e;
        atomicOr(&mask[e], 1u << r);
      }
    }
  }
  epi_sync();
  // ---- ranks inside the chunk and per-CTA partials
  if (valid) {
#pragma unroll
    for (int j = 0; j < kMaxTopK; ++j) {
      if (j < k && (j & 3) == qp) {
        const int e = ord[j];
        a.local_rank[t * k + j] = __popc(mask[e] & ((1u << r) - 1u));
      }
    }
  }
  const int cta = blockIdx.x;
  if (tid < E) {
    a.chunk_count[static_cast<size_t>(cta) * E + tid] = __popc(mask[tid]);
    float ps = 0.f;
    for (int rr = 0; rr < kTile; ++rr) ps += P[rr * kMaxE + tid];
    a.psum_part[static_cast<size_t>(cta) * E + tid] = ps;
  }
  if (tid == 0) {
    double z = 0.0;
    for (int rr = 0; rr < kTile; ++rr) z += static_cast<double>(lse_s[rr]) * lse_s[rr];
    a.zsum_part[cta] = z;
  }
  __threadfence();
  epi_sync();
  if (tid == 0) *s_last = (atomicAdd(a.ticket, 1) == static_cast<int>(gridDim.x) - 1);
  epi_sync();
  if (*s_last) {
    __threadfence();
    const int nb = gridDim.x;
    int32_t* cnt_s = reinterpret_cast<int32_t*>(ring);                     // [kScanBlock][E]
    float* ps_s = reinterpret_cast<float*>(ring + kScanBlock * kMaxE * 4);  // [kScanBlock][E]
    int run = 0;       // thread tid < E: running total of expert tid
    double pe = 0.0;
    for (int c0 = 0; c0 < nb; c0 += kScanBlock) {
      const int nc = min(kScanBlock, nb - c0);
      // the block's counts and probability sums, read with all 128 threads as
      // 16-byte loads, eight in flight per thread (c0 * E is a multiple of 4)
      {
        const int n = nc * E;
        const int32_t* gc = a.chunk_count + static_cast<size_t>(c0) * E;
        const float* gp = a.psum_part + static_cast<size_t>(c0) * E;
        for (int i0 = tid * 4; i0 < (n & ~3); i0 += 128 * 4 * 8) {
          int4 cv[8];
          float4 pv[8];
#pragma unroll
          for (int b = 0; b < 8; ++b) {
            const int i = i0 + b * 512;
            if (i < (n & ~3)) {
              cv[b] = __ldcg(reinterpret_cast<const int4*>(gc + i));
              pv[b] = __ldcg(reinterpret_cast<const float4*>(gp + i));
            }
          }
#pragma unroll
          for (int b = 0; b < 8; ++b) {
            const int i = i0 + b * 512;
            if (i < (n & ~3)) {
              *reinterpret_cast<int4*>(cnt_s + i) = cv[b];
              *reinterpret_cast<float4*>(ps_s + i) = pv[b];
            }
          }
        }
        for (int i = (n & ~3) + tid; i < n; i += 128) {
          cnt_s[i] = __ldcg(gc + i);
          ps_s[i] = __ldcg(gp + i);
        }
      }
      epi_sync();
      if (tid < E) {  // eight chunks' loads in flight, then the running sums in order
        int c = 0;
        for (; c + 8 <= nc; c += 8) {
          int v[8];
          float q[8];
#pragma unroll
          for (int b = 0; b < 8; ++b) {
            v[b] = cnt_s[(c + b) * E + tid];
            q[b] = ps_s[(c + b) * E + tid];
          }
#pragma unroll
          for (int b = 0; b < 8; ++b) {
            cnt_s[(c + b) * E + tid] = run;  // becomes the chunk base
            run += v[b];
            pe += static_cast<double>(q[b]);
          }
        }
        for (; c < nc; ++c) {
          const int v = cnt_s[c * E + tid];
          cnt_s[c * E + tid] = run;
          run += v;
          pe += static_cast<double>(ps_s[c * E + tid]);
        }
      }
      epi_sync();
      for (int i = tid; i < nc * E; i += 128) a.chunk_base[static_cast<size_t>(c0) * E + i] = cnt_s[i];
      epi_sync();
    }
    if (tid < E) {
      tot[tid] = run;
      tot_p[tid] = pe;
      a.counts_ws[tid] = run;
      if (a.counts_user != nullptr) a.counts_user[tid] = run;
    }
    // sum of lse^2 partials: 128 contiguous slices in order, then the slices in order
    {
      const int per = (nb + 127) / 128;
      double z = 0.0;
      for (int c = tid * per; c < min(nb, (tid + 1) * per); ++c) z += __ldcg(&a.zsum_part[c]);
      zred[tid] = z;
    }
    epi_sync();
    if (tid < 32) {
      // warp-wide finalisation (E <= 64): lane holds experts lane and lane + 32.
      // Group starts and offsets are exclusive prefix sums; the two loss sums use a
      // fixed butterfly order, so every lane ends with the same bits on every run.
      const int e0 = lane, e1 = lane + 32;
      const int c0v = e0 < E ? tot[e0] : 0, c1v = e1 < E ? tot[e1] : 0;
      const int g0v = (c0v + kRowAlign - 1) / kRowAlign * kRowAlign;
      const int g1v = (c1v + kRowAlign - 1) / kRowAlign * kRowAlign;
      int ic0 = c0v, ig0 = g0v, ic1 = c1v, ig1 = g1v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int u0 = __shfl_up_sync(0xffffffffu, ic0, o), w0 = __shfl_up_sync(0xffffffffu, ig0, o);
        const int u1 = __shfl_up_sync(0xffffffffu, ic1, o), w1 = __shfl_up_sync(0xffffffffu, ig1, o);
        if (lane >= o) {
          ic0 += u0;
          ig0 += w0;
          ic1 += u1;
          ig1 += w1;
        }
      }
      const int tc0 = __shfl_sync(0xffffffffu, ic0, 31), tg0 = __shfl_sync(0xffffffffu, ig0, 31);
      const int tc1 = __shfl_sync(0xffffffffu, ic1, 31), tg1 = __shfl_sync(0xffffffffu, ig1, 31);
      if (e0 < E) {
        a.offsets_ws[e0] = ic0 - c0v;
        a.gs_ws[e0] = ig0 - g0v;
      }
      if (e1 < E) {
        a.offsets_ws[e1] = tc0 + ic1 - c1v;
        a.gs_ws[e1] = tg0 + ig1 - g1v;
      }
      // load balance: E * sum_e (c_e / (T k)) (P_e / T) = E * sum_e c_e P_e / (T^2 k)
      double lb = (e0 < E ? static_cast<double>(c0v) * tot_p[e0] : 0.0) +
                  (e1 < E ? static_cast<double>(c1v) * tot_p[e1] : 0.0);
      double zt = ((zred[4 * lane] + zred[4 * lane + 1]) + zred[4 * lane + 2]) + zred[4 * lane + 3];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        lb += __shfl_xor_sync(0xffffffffu, lb, o);
        zt += __shfl_xor_sync(0xffffffffu, zt, o);
      }
      if (lane == 0) {
        const int off = tc0 + tc1;
        a.offsets_ws[E] = off;
        a.gs_ws[E] = tg0 + tg1;
        const double Td = static_cast<double>(a.T);
        const float l0 = static_cast<float>(lb * E / (Td * Td * k)), l1 = static_cast<float>(zt / Td);
        a.losses_ws[0] = l0;
        a.losses_ws[1] = l1;
        if (a.losses_user != nullptr) {
          a.losses_user[0] = l0;
          a.losses_user[1] = l1;
        }
        if (static_cast<int64_t>(off) != a.T * k) report(a.status, DEV_COUNT_MISMATCH);
        *a.ticket = 0;
      }
    }
  }
}

// STAGES-deep ring, MINB CTAs per SM: one CTA with a 16-deep ring when the
// tiles fit on the SMs at once, two with 7-deep rings (one's epilogue then
// overlaps the other's loads) when there are more tiles than SMs.
template <int STAGES, int MINB>
__global__ void __launch_bounds__(kThreads, MINB)
    router_tc_kernel(const __grid_constant__ CUtensorMap tmx, const __grid_constant__ CUtensorMap tmw,
                     const RArgs a) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int STAGE = kAload + a.NP * 128;  // A rows 0..31, then B
  unsigned char* ring = smem;
  unsigned char* misc = smem + ring_bytes(STAGES);
  uint64_t* full = reinterpret_cast<uint64_t*>(misc);
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(acc_full + 1);
  uint32_t* mask = tmem_holder + 4;                          // [kMaxE]
  float* lse_s = reinterpret_cast<float*>(mask + kMaxE);      // [kTile]
  int32_t* s_last = reinterpret_cast<int32_t*>(lse_s + kTile);
  int32_t* tot = s_last + 4;                                  // [kMaxE]
  double* tot_p = reinterpret_cast<double*>(tot + kMaxE);     // [kMaxE]
  double* zred = tot_p + kMaxE;                               // [128]
  // once the accumulator is complete the ring is free
  float* S = reinterpret_cast<float*>(ring);                          // [kTile][kLogitStride] logits
  float* P = S + kTile * kLogitStride;                                 // [kTile][kMaxE] probabilities
  int32_t* chosen = reinterpret_cast<int32_t*>(P + kTile * kMaxE);     // [kTile][kMaxTopK]
  uint32_t* queue = reinterpret_cast<uint32_t*>(ring + 20480);         // [kTile * kMaxE] (token << 8) | expert
  double* exact = reinterpret_cast<double*>(ring + 20480 + kTile * kMaxE * 4);  // [kTile * kMaxE]
  int32_t* qn = s_last + 1;                                            // queued pairs

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nk = a.d / 64;
  const int64_t t0 = static_cast<int64_t>(blockIdx.x) * kTile;

  pdl_trigger();
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, a.NP <= 32 ? 32u : 64u);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  pdl_wait();  // x may come from the kernel before (the stack's RMSNorm)

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&tmx);
      tma_prefetch_desc(&tmw);
      int issued = 0;
      // CTAs walk K from different starting points so they do not all read the
      // same router-weight tile of L2 at the same moment
      const int k0 = static_cast<int>(blockIdx.x % static_cast<unsigned>(nk));
      for (int kb = 0; kb < nk; ++kb) {
        const int s = kb % STAGES;
        const uint32_t ph = static_cast<uint32_t>(kb / STAGES) & 1u;
        if (!mbar_wait(&empty[s], ph ^ 1u)) {
          report(a.status, DEV_WAIT_TIMEOUT_PRODUCER);
          break;
        }
        const int kc = (kb + k0) % nk;
        unsigned char* st = ring + static_cast<size_t>(s) * STAGE;
        mbar_arrive_expect_tx(&full[s], STAGE);
        tma_load_2d(&tmx, &full[s], st, kc * 64, static_cast<int32_t>(t0));
        tma_load_2d(&tmw, &full[s], st + kAload, kc * 64, 0);
        ++issued;
      }
      for (int s = 0; s < STAGES && s < issued; ++s) {
        const int last = ((issued - 1 - s) / STAGES) * STAGES + s;
        if (!mbar_wait(&full[s], static_cast<uint32_t>((last / STAGES) & 1))) report(a.status, DEV_WAIT_TIMEOUT_DRAIN);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = make_idesc(false, false, false, 128, a.NP);
      bool ok = true;
      for (int kb = 0; kb < nk; ++kb) {
        const int s = kb % STAGES;
        if (!mbar_wait(&full[s], static_cast<uint32_t>(kb / STAGES) & 1u)) {
          report(a.status, DEV_WAIT_TIMEOUT_MMA);
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t sa = smem_u32(ring + static_cast<size_t>(s) * STAGE);
        const uint32_t sb = sa + kAload;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          umma_bf16(tmem, smem_desc_sw128(sa + kk * 32, 16, 1024), smem_desc_sw128(sb + kk * 32, 16, 1024), idesc,
                    (kb > 0 || kk > 0) ? 1u : 0u);
        umma_commit(&empty[s]);
      }
      if (ok) umma_commit(acc_full);
    }
  } else {
    // ------------------------------------------------------------ epilogue (warps 2..5)
    const int tid = threadIdx.x - 64;  // 0..127
    const int E = a.E, k = a.k;
    if (tid < kMaxE) mask[tid] = 0u;
    if (tid == 0) *qn = 0;
    if (!mbar_wait(acc_full, 0)) report(a.status, DEV_WAIT_TIMEOUT_EPILOGUE);
    tc_fence_after();
    if (warp == 4) {  // TMEM lanes 0..31 hold the 32 tokens' logits
      for (int c = 0; c < a.NP; c += 16) {
        uint32_t v[16];
        tmem_ld16(tmem + c, v);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int e = c + i;
          float h = __uint_as_float(v[i]);
          if (e < E && a.bias != nullptr) h += a.bias[e];
          S[lane * kLogitStride + e] = (e < E) ? h : -INFINITY;
        }
      }
      for (int e = a.NP; e < kMaxE; ++e) S[lane * kLogitStride + e] = -INFINITY;
    }
    tc_fence_before();
    epi_sync();

    const EpiSmem sm{S, P, chosen, queue, exact, qn, mask, lse_s, s_last, tot, tot_p, zred, ring};
    router_epilogue(a, sm, t0, tid, lane);
  }
  __syncwarp();  // single-lane roles rejoin their warp before the block barrier
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, a.NP <= 32 ? 32u : 64u);
  }
}


// ------------------------------------------------------------------ split form
// Two kernels: logits for 128 tokens per CTA (the M=128 MMA then carries 128
// real rows, so the tcgen05 issue cost, which bounds this phase, is spread
// over 4x the tokens), with the K steps divided among `ksplit` CTAs per tile
// when there are fewer tiles than SMs, as fp32 partials in the workspace; then
// the epilogue above on 32-token tiles, two CTAs per SM, which sums the
// partials in a fixed order.
constexpr int kLogitTile = 128;
constexpr int kLogitStages = 8;
constexpr int kLogitStage = kLogitTile * 128 + kMaxE * 128;  // x rows, then W_r rows (per 64-wide K step)
constexpr size_t kLogitSmem = 1024 + static_cast<size_t>(kLogitStages) * kLogitStage + 1024;
constexpr int kEpiRing = 64 * 1024;  // shared-memory scratch of the epilogue (and of the last CTA's scan)
constexpr size_t kEpiSmem = 1024 + kEpiRing + kMiscBytes;
static_assert(kScanBlock * kMaxE * 8 <= kEpiRing, "scan block fits in the epilogue scratch");
static_assert(20480 + kTile * kMaxE * 12 <= kEpiRing, "epilogue tiles fit in the scratch");

__global__ void __launch_bounds__(kThreads, 1)
    router_logits_kernel(const __grid_constant__ CUtensorMap tmx, const __grid_constant__ CUtensorMap tmw,
                         const RArgs a) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* ring = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int STAGE = kLogitTile * 128 + a.NP * 128;
  uint64_t* full = reinterpret_cast<uint64_t*>(ring + static_cast<size_t>(kLogitStages) * kLogitStage);
  uint64_t* empty = full + kLogitStages;
  uint64_t* acc_full = empty + kLogitStages;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(acc_full + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // this CTA's share of the 64-wide K steps
  const int ks = blockIdx.y;
  const int kb_lo = (ks * (a.d / 64)) / a.ksplit;
  const int nk = ((ks + 1) * (a.d / 64)) / a.ksplit - kb_lo;
  const int64_t t0 = static_cast<int64_t>(blockIdx.x) * kLogitTile;
  pdl_trigger();
  if (threadIdx.x == 0) {
    for (int s = 0; s < kLogitStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, a.NP <= 32 ? 32u : 64u);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  pdl_wait();
  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&tmx);
      tma_prefetch_desc(&tmw);
      int issued = 0;
      const int k0 = static_cast<int>(blockIdx.x % static_cast<unsigned>(nk));
      int s = 0;
      uint32_t ph = 0;
      int kc = k0;
      for (int kb = 0; kb < nk; ++kb) {
        if (!mbar_wait(&empty[s], ph ^ 1u)) {
          report(a.status, DEV_WAIT_TIMEOUT_PRODUCER);
          break;
        }
        unsigned char* st = ring + static_cast<size_t>(s) * STAGE;
        mbar_arrive_expect_tx(&full[s], STAGE);
        tma_load_2d(&tmx, &full[s], st, (kb_lo + kc) * 64, static_cast<int32_t>(t0));
        tma_load_2d(&tmw, &full[s], st + kLogitTile * 128, (kb_lo + kc) * 64, 0);
        ++issued;
        if (++s == kLogitStages) {
          s = 0;
          ph ^= 1u;
        }
        if (++kc == nk) kc = 0;
      }
      for (int q = 0; q < kLogitStages && q < issued; ++q) {
        const int last = ((issued - 1 - q) / kLogitStages) * kLogitStages + q;
        if (!mbar_wait(&full[q], static_cast<uint32_t>((last / kLogitStages) & 1)))
          report(a.status, DEV_WAIT_TIMEOUT_DRAIN);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = make_idesc(false, false, false, 128, a.NP);
      bool ok = true;
      int s = 0;
      uint32_t ph = 0;
      for (int kb = 0; kb < nk; ++kb) {
        if (!mbar_wait(&full[s], ph)) {
          report(a.status, DEV_WAIT_TIMEOUT_MMA);
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t sa = smem_u32(ring + static_cast<size_t>(s) * STAGE);
        const uint32_t sb = sa + kLogitTile * 128;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          umma_bf16(tmem, smem_desc_sw128(sa + kk * 32, 16, 1024), smem_desc_sw128(sb + kk * 32, 16, 1024), idesc,
                    (kb > 0 || kk > 0) ? 1u : 0u);
        umma_commit(&empty[s]);
        if (++s == kLogitStages) {
          s = 0;
          ph ^= 1u;
        }
      }
      if (ok) umma_commit(acc_full);
    }
  } else {
    // warps 2..5: TMEM lane quarter (warp % 4) holds tokens 32*(warp % 4) .. +31
    const int q = warp & 3;
    const int64_t t = t0 + q * 32 + lane;
    if (!mbar_wait(acc_full, 0)) report(a.status, DEV_WAIT_TIMEOUT_EPILOGUE);
    tc_fence_after();
    for (int c = 0; c < a.NP; c += 16) {
      uint32_t v[16];
      tmem_ld16(tmem + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(c), v);
      tmem_ld_wait();
      if (t < a.T) {
        float* dst = a.logit_part + (static_cast<int64_t>(ks) * a.T + t) * a.E;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int e = c + i;
          if (e < a.E) dst[e] = __uint_as_float(v[i]);
        }
      }
    }
  }
  __syncwarp();  // single-lane roles rejoin their warp before the block barrier
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, a.NP <= 32 ? 32u : 64u);
  }
}

__global__ void __launch_bounds__(128, 2) router_epi_kernel(const RArgs a) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* ring = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  unsigned char* misc = ring + kEpiRing;
  uint32_t* mask = reinterpret_cast<uint32_t*>(misc);          // [kMaxE]
  float* lse_s = reinterpret_cast<float*>(mask + kMaxE);      // [kTile]
  int32_t* s_last = reinterpret_cast<int32_t*>(lse_s + kTile);
  int32_t* tot = s_last + 4;                                  // [kMaxE]
  double* tot_p = reinterpret_cast<double*>(tot + kMaxE);     // [kMaxE]
  double* zred = tot_p + kMaxE;                               // [128]
  float* S = reinterpret_cast<float*>(ring);
  float* P = S + kTile * kLogitStride;
  int32_t* chosen = reinterpret_cast<int32_t*>(P + kTile * kMaxE);
  uint32_t* queue = reinterpret_cast<uint32_t*>(ring + 20480);
  double* exact = reinterpret_cast<double*>(ring + 20480 + kTile * kMaxE * 4);
  int32_t* qn = s_last + 1;
  const int tid = threadIdx.x, lane = tid & 31;
  const int64_t t0 = static_cast<int64_t>(blockIdx.x) * kTile;
  pdl_trigger();
  if (tid < kMaxE) mask[tid] = 0u;
  if (tid == 0) *qn = 0;
  pdl_wait();
  // this tile's logits: the K-range partials (all loads in flight, then summed
  // in a fixed order), plus the offset
  for (int i = tid; i < kTile * kMaxE; i += 128) {
    const int r = i / kMaxE, e = i - r * kMaxE;
    float h = -INFINITY;
    if (t0 + r < a.T && e < a.E) {
      const float* src = a.logit_part + (t0 + r) * a.E + e;
      const int64_t step = a.T * a.E;
      float v[16];
#pragma unroll
      for (int ks = 0; ks < 16; ++ks) v[ks] = (ks < a.ksplit) ? __ldcg(src + ks * step) : 0.f;
      h = v[0];
#pragma unroll
      for (int ks = 1; ks < 16; ++ks)
        if (ks < a.ksplit) h += v[ks];
      if (a.bias != nullptr) h += a.bias[e];
    }
    S[r * kLogitStride + e] = h;
  }
  epi_sync();
  const EpiSmem sm{S, P, chosen, queue, exact, qn, mask, lse_s, s_last, tot, tot_p, zred, ring};
  router_epilogue(a, sm, t0, tid, lane);
}

}  // namespace

bool router_tc_supported(const Shape& s) { return !s.fp32 && s.E <= kMaxE && s.k + 3 <= kMaxSel; }

namespace {
cudaError_t router_tc_impl(const Shape& s, const void* x, const void* w_router, const float* bias, int32_t* idx,
                           float* wts, int32_t* counts, float* losses, void* ws, const Workspace& L, bool probs_only,
                           cudaStream_t st) {
  {
    static std::atomic<size_t> set_fused[kMaxDevices], set_logits[kMaxDevices], set_epi[kMaxDevices];
    cudaError_t e = raise_smem_limit(reinterpret_cast<const void*>(router_tc_kernel<16, 1>), smem_bytes(16), set_fused);
    if (e == cudaSuccess)
      e = raise_smem_limit(reinterpret_cast<const void*>(router_logits_kernel), kLogitSmem, set_logits);
    if (e == cudaSuccess) e = raise_smem_limit(reinterpret_cast<const void*>(router_epi_kernel), kEpiSmem, set_epi);
    if (e != cudaSuccess) return e;
  }
  const int NP = (s.E + 15) / 16 * 16;
  CUtensorMap tx, tw;
  if (!make_map(&tx, x, false, static_cast<uint64_t>(s.T), s.d, 64, kTile)) return cudaErrorInvalidValue;
  if (!make_map(&tw, w_router, false, static_cast<uint64_t>(s.E), s.d, 64, NP)) return cudaErrorInvalidValue;
  // ctrl[1], the completion counter, is zero between calls: moe_workspace_init
  // clears it and the last CTA of every router launch puts it back to zero
  int32_t* ctrl = at<int32_t>(ws, L.ctrl);
  cudaError_t e = cudaSuccess;
  RArgs a{};
  a.T = s.T;
  a.d = s.d;
  a.E = s.E;
  a.k = s.k;
  a.NP = NP;
  a.bias = bias;
  a.x = static_cast<const __nv_bfloat16*>(x);
  a.w = static_cast<const __nv_bfloat16*>(w_router);
  a.idx_out = idx;
  a.w_out = wts;
  a.probs = at<float>(ws, L.probs);
  a.lse_out = at<float>(ws, L.lse);
  a.local_rank = at<int32_t>(ws, L.local_rank);
  a.chunk_count = at<int32_t>(ws, L.chunk_count);
  a.chunk_base = at<int32_t>(ws, L.chunk_base);
  a.psum_part = at<float>(ws, L.psum_part);
  a.zsum_part = at<double>(ws, L.zsum_part);
  a.counts_ws = at<int32_t>(ws, L.counts);
  a.counts_user = counts;
  a.losses_ws = at<float>(ws, L.losses);
  a.losses_user = losses;
  a.offsets_ws = at<int32_t>(ws, L.offsets);
  a.gs_ws = at<int32_t>(ws, L.group_start);
  a.ticket = ctrl + 1;
  a.status = ctrl;
  a.renorm = s.renorm ? 1 : 0;
  a.probs_only = probs_only ? 1 : 0;
  const unsigned grid = static_cast<unsigned>((s.T + kTile - 1) / kTile);
  // A few tokens: logits split over K among many CTAs, then the epilogue
  // (T=1: 24.5 us against 28.7 us fused, warm; T=32: 32.8 against ~28.7).
  // Up to one wave of 32-token tiles: the fused kernel (T=64: 28.7 us against
  // 41.0 us split; T=4096: 40.9 us against 49.2 us). More tiles than SMs: the
  // split form (T=16384: 87-94 us against 102 us fused).
  if (s.T > 8 && static_cast<int>(grid) <= device_sm_count())
    return launch_dependent(router_tc_kernel<16, 1>, dim3(grid), dim3(kThreads), smem_bytes(16), st, nullptr, 0, tx,
                            tw, a);
  CUtensorMap tx128;
  if (!make_map(&tx128, x, false, static_cast<uint64_t>(s.T), s.d, 64, kLogitTile)) return cudaErrorInvalidValue;
  const unsigned grid_l = static_cast<unsigned>((s.T + kLogitTile - 1) / kLogitTile);
  // K ranges per tile: enough CTAs to cover the SMs, at least two K steps each,
  // and no more partials than the scratch (the permuted-rows region, unused yet) holds
  int ks = device_sm_count() / static_cast<int>(grid_l);
  ks = ks < 1 ? 1 : (ks > 16 ? 16 : ks);
  while (ks > 1 && s.d / 64 / ks < 2) --ks;
  const size_t cap = static_cast<size_t>(s.P) * s.d * s.esize;
  while (ks > 1 && static_cast<size_t>(ks) * s.T * s.E * 4 > cap) --ks;
  if (static_cast<size_t>(ks) * s.T * s.E * 4 > cap)  // tiny layers: the fused kernel
    return launch_dependent(router_tc_kernel<16, 1>, dim3(grid), dim3(kThreads), smem_bytes(16), st, nullptr, 0, tx,
                            tw, a);
  a.logit_part = at<float>(ws, L.x_perm);
  a.ksplit = ks;
  e = launch_dependent(router_logits_kernel, dim3(grid_l, static_cast<unsigned>(ks)), dim3(kThreads), kLogitSmem, st,
                       nullptr, 0, tx128, tw, a);
  if (e != cudaSuccess) return e;
  return launch_dependent(router_epi_kernel, dim3(grid), dim3(128), kEpiSmem, st, nullptr, 0, a);
}
}  // namespace

cudaError_t launch_router_tc(const Shape& s, const void* x, const void* w_router, const float* bias, int32_t* idx,
                             float* wts, int32_t* counts, float* losses, void* ws, const Workspace& L,
                             cudaStream_t st) {
  return router_tc_impl(s, x, w_router, bias, idx, wts, counts, losses, ws, L, false, st);
}

cudaError_t launch_router_probs(const Shape& s, const void* x, const void* w_router, const float* bias, void* ws,
                                const Workspace& L, cudaStream_t st) {
  return router_tc_impl(s, x, w_router, bias, nullptr, nullptr, nullptr, nullptr, ws, L, true, st);
}

}  // namespace moe
