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
constexpr int kThreads = 192;          // logits kernel: TMA warp, MMA warp, 4 epilogue warps
constexpr int kFusedThreads = 512;     // fused kernel: 16 warps; warps 0 and 1 also load and issue the MMAs
constexpr int kMaxE = 64;
constexpr int kMaxSel = kMaxTopK + 3;
constexpr int kAload = kTile * 128;                      // bytes of A loaded per stage
constexpr int kStageMax = kAload + kMaxE * 128;          // 12 KB
// ring bytes for S stages, plus the over-read of the last stage's A
constexpr int ring_bytes(int S) { return S * kStageMax + 16 * 1024; }
constexpr int kLogitStride = kMaxE + 1;
// Independent accumulators the K steps are dealt to (K step kb accumulates into
// chain kb % kChains; the epilogue adds the chains in order). One chain of
// M=128 x N=E x K=16 UMMAs is a dependent sequence whose latency, not the
// tensor pipe, bounds it; four chains let the UMMAs overlap.
constexpr int kChains = 4;
__host__ __device__ constexpr uint32_t tmem_cols(int NP) { return NP <= 32 ? 32u * kChains : 64u * kChains; }
constexpr size_t kMiscBytes = 4096;
constexpr size_t smem_bytes(int S) { return 1024 + static_cast<size_t>(ring_bytes(S)) + kMiscBytes; }
static_assert(kTile == 32, "one mask word per expert");

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

// The router's work once the tile's 32 logit rows are in shared memory (S),
// shared by the fused kernel and the epilogue-only kernel. kEpiThreads
// threads (tid 0..511, 16 warps) synchronise on named barrier 1; a half-warp
// takes a token and each of its 16 threads four experts (e = sub + 16 i).
//   softmax      half-warp max and sum, probabilities and lse in fp32;
//   ranks        each expert's rank among the token's fp32 logits (larger
//                first, equal values to the lower index) and the distance to
//                the nearest other logit, in one pass over the row;
//   exact ranks  a token whose k+1 largest logits hold two values closer than
//                2e-4 * max(1, |h|) (far above the error of a 2048-term fp32
//                sum of exact bf16 products) has every run of such neighbours
//                that reaches its top k recomputed exactly (fp64 sums of the
//                exact products, a warp per logit) and re-ranked; a run that
//                reaches past rank k+3 has all E logits recomputed;
//   outputs      the k best experts in slot order with their weights, a bit
//                mask per expert of the tile's tokens that chose it (each
//                pair's rank inside the chunk), the per-chunk counts and the
//                loss partials.
// The last CTA to finish scans the per-chunk counts into chunk bases (each
// expert's chunks cut into 8 segments, one thread each), the bincount
// offsets and the padded group starts, and reduces the loss partials. Every
// sum runs in a fixed order, so the results are deterministic.
constexpr int kEpiThreads = 512;
constexpr int kEpiWarps = kEpiThreads / 32;
constexpr int kScanSeg = kEpiThreads / kMaxE;   // segments per expert in the scan
constexpr int kScanBlock = 64;                  // chunks per pass of the scan
constexpr int kWin = kMaxSel + 1;               // sorted window of a token: ranks 0 .. k+3
// byte offsets inside the free ring (after the accumulator is complete)
constexpr int kOffS = 0;                                        // float [kTile][kLogitStride]
constexpr int kOffP = kOffS + kTile * kLogitStride * 4;         // float [kTile][kMaxE]
constexpr int kOffRk = kOffP + kTile * kMaxE * 4;               // uint8 [kTile][kMaxE]
constexpr int kOffSv = kOffRk + kTile * kMaxE;                  // float [kTile][kWin]
constexpr int kOffSe = kOffSv + kTile * kWin * 4;               // int   [kTile][kWin]
constexpr int kOffQ = kOffSe + kTile * kWin * 4;                // uint32 [kTile * kMaxE]
constexpr int kOffX = (kOffQ + kTile * kMaxE * 4 + 7) / 8 * 8;  // double [kTile * kMaxE]
constexpr int kOffQb = kOffX + kTile * kMaxE * 8;               // int [kTile] first slot, count, all-E flag
constexpr int kOffSegI = kOffQb + 3 * kTile * 4;                // int [kScanSeg][kMaxE]
constexpr int kOffSegD = kOffSegI + kScanSeg * kMaxE * 4;       // double [kScanSeg][kMaxE]
constexpr int kOffZ = kOffSegD + kScanSeg * kMaxE * 8;          // double [kEpiThreads]
constexpr int kOffScan = kOffZ + kEpiThreads * 8;               // int + float [kScanBlock][kMaxE]
constexpr int kEpiScratch = kOffScan + kScanBlock * kMaxE * 8;
static_assert(kOffX % 8 == 0 && kOffSegD % 8 == 0 && kOffZ % 8 == 0 && kOffScan % 16 == 0, "alignment");

struct EpiSmem {
  unsigned char* ring;  // kEpiScratch bytes
  uint32_t* mask;       // [kMaxE]
  float* lse_s;         // [kTile]
  int32_t* s_last;
  int32_t* qn;
  int32_t* tot;         // [kMaxE]
  double* tot_p;        // [kMaxE]
};

__device__ __forceinline__ void epi_sync() { asm volatile("bar.sync 1, 512;" ::: "memory"); }

__device__ __forceinline__ float near_gap(float v) { return 2e-4f * fmaxf(1.0f, fabsf(v)); }

// <x_t, W_r[e]> from exact products of bf16 inputs, summed in fp64 by a whole
// warp: lane l takes elements 8l + 256i; the loads of 4 steps are issued before
// their arithmetic, so a row pair of d = 2048 costs two memory round trips. The
// lane sums are combined by a fixed shuffle tree (every lane gets the result).
__device__ __forceinline__ double exact_logit_warp(const __nv_bfloat16* xr, const __nv_bfloat16* wr, int d,
                                                   int lane) {
  constexpr int kBatch = 4;
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
          const float2 xf = bf16x2_to_float2(xa[c]);
          const float2 wf = bf16x2_to_float2(wa[c]);
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

// Tile `cta` (tokens cta * 32 ...) of `ntiles`; the last tile to finish scans.
// A tile's per-chunk partials (counts from the chosen-token masks, the
// probability sums from P [kTile][kMaxE], the sum of lse^2), then the ticket:
// the last tile to finish scans the per-chunk counts into chunk bases,
// offsets and group starts and reduces both losses, in a fixed order.
__device__ __forceinline__ void router_finish(const RArgs& a, const EpiSmem& sm, const float* P, int cta, int ntiles,
                                              int tid, int lane) {
  unsigned char* R = sm.ring;
  const int E = a.E, k = a.k;
  if (tid < E) {
    a.chunk_count[static_cast<size_t>(cta) * E + tid] = __popc(sm.mask[tid]);
    float ps = 0.f;
    for (int rr = 0; rr < kTile; ++rr) ps += P[rr * kMaxE + tid];
    a.psum_part[static_cast<size_t>(cta) * E + tid] = ps;
  }
  if (tid == kMaxE) {
    double z = 0.0;
    for (int rr = 0; rr < kTile; ++rr) z += static_cast<double>(sm.lse_s[rr]) * sm.lse_s[rr];
    a.zsum_part[cta] = z;
  }
  __threadfence();
  epi_sync();
  if (tid == 0) *sm.s_last = (atomicAdd(a.ticket, 1) == ntiles - 1);
  epi_sync();
  if (!*sm.s_last) return;

  // ---- the last CTA: scan of the per-chunk counts, losses
  __threadfence();
  const int nb = ntiles;
  int32_t* seg_i = reinterpret_cast<int32_t*>(R + kOffSegI);
  double* seg_d = reinterpret_cast<double*>(R + kOffSegD);
  double* zred = reinterpret_cast<double*>(R + kOffZ);
  int32_t* cnt_s = reinterpret_cast<int32_t*>(R + kOffScan);               // [kScanBlock][E]
  float* ps_s = reinterpret_cast<float*>(R + kOffScan + kScanBlock * kMaxE * 4);  // [kScanBlock][E]
  const int e = tid & (kMaxE - 1), g = tid / kMaxE;  // expert, segment
  constexpr int kSegLen = kScanBlock / kScanSeg;
  int run = 0;
  double pe = 0.0;
  for (int c0 = 0; c0 < nb; c0 += kScanBlock) {
    const int nc = min(kScanBlock, nb - c0);
    {  // the block's counts and probability sums, 16-byte loads (c0 * E is a multiple of 4)
      const int n = nc * E;
      const int32_t* gc = a.chunk_count + static_cast<size_t>(c0) * E;
      const float* gp = a.psum_part + static_cast<size_t>(c0) * E;
      for (int i = tid * 4; i < (n & ~3); i += kEpiThreads * 4) {
        *reinterpret_cast<int4*>(cnt_s + i) = __ldcg(reinterpret_cast<const int4*>(gc + i));
        *reinterpret_cast<float4*>(ps_s + i) = __ldcg(reinterpret_cast<const float4*>(gp + i));
      }
      for (int i = (n & ~3) + tid; i < n; i += kEpiThreads) {
        cnt_s[i] = __ldcg(gc + i);
        ps_s[i] = __ldcg(gp + i);
      }
    }
    epi_sync();
    int sc = 0;
    double sp = 0.0;
    if (e < E) {
      for (int j = 0; j < kSegLen; ++j) {
        const int c = g * kSegLen + j;
        if (c < nc) {
          sc += cnt_s[c * E + e];
          sp += static_cast<double>(ps_s[c * E + e]);
        }
      }
    }
    seg_i[g * kMaxE + e] = sc;
    seg_d[g * kMaxE + e] = sp;
    epi_sync();
    if (e < E) {
      int base = run;
      for (int g2 = 0; g2 < g; ++g2) base += seg_i[g2 * kMaxE + e];
      for (int j = 0; j < kSegLen; ++j) {
        const int c = g * kSegLen + j;
        if (c < nc) {
          a.chunk_base[static_cast<size_t>(c0 + c) * E + e] = base;
          base += cnt_s[c * E + e];
        }
      }
      for (int g2 = 0; g2 < kScanSeg; ++g2) {
        run += seg_i[g2 * kMaxE + e];
        pe += seg_d[g2 * kMaxE + e];
      }
    }
    epi_sync();  // the block's scratch is reused by the next pass
  }
  if (g == 0 && e < E) {
    sm.tot[e] = run;
    sm.tot_p[e] = pe;
    a.counts_ws[e] = run;
    if (a.counts_user != nullptr) a.counts_user[e] = run;
  }
  {  // sum of lse^2 partials: contiguous slices in order, then the slices in order
    const int per = (nb + kEpiThreads - 1) / kEpiThreads;
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
    const int c0v = e0 < E ? sm.tot[e0] : 0, c1v = e1 < E ? sm.tot[e1] : 0;
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
    double lb = (e0 < E ? static_cast<double>(c0v) * sm.tot_p[e0] : 0.0) +
                (e1 < E ? static_cast<double>(c1v) * sm.tot_p[e1] : 0.0);
    double zt = 0.0;
    for (int j = 0; j < kEpiThreads / 32; ++j) zt += zred[lane * (kEpiThreads / 32) + j];
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

__device__ __forceinline__ void router_epilogue(const RArgs& a, const EpiSmem& sm, int cta, int ntiles, int tid,
                                                int lane) {
  const int64_t t0 = static_cast<int64_t>(cta) * kTile;
  unsigned char* R = sm.ring;
  float* S = reinterpret_cast<float*>(R + kOffS);
  float* P = reinterpret_cast<float*>(R + kOffP);
  uint8_t* rk = R + kOffRk;
  float* sv = reinterpret_cast<float*>(R + kOffSv);
  int32_t* se = reinterpret_cast<int32_t*>(R + kOffSe);
  uint32_t* queue = reinterpret_cast<uint32_t*>(R + kOffQ);
  double* exact = reinterpret_cast<double*>(R + kOffX);
  int32_t* qb = reinterpret_cast<int32_t*>(R + kOffQb);  // [kTile] first slot, [kTile] count, [kTile] all-E
  const int E = a.E, k = a.k;
  const int r = tid >> 4, sub = tid & 15;
  const unsigned hm = 0xFFFFu << (lane & 16);
  const int64_t t = t0 + r;
  const bool valid = t < a.T;  // the whole half-warp agrees
  // ---- softmax over the token's E logits
  float h[4], ex[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int e = sub + 16 * i;
    h[i] = e < E ? S[r * kLogitStride + e] : -INFINITY;
  }
  float m = fmaxf(fmaxf(h[0], h[1]), fmaxf(h[2], h[3]));
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(hm, m, o));
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    ex[i] = (sub + 16 * i < E) ? expf(h[i] - m) : 0.f;
    s += ex[i];
  }
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) s += __shfl_xor_sync(hm, s, o);
  const float lse = m + logf(s);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int e = sub + 16 * i;
    const float p = valid ? ex[i] / s : 0.f;
    P[r * kMaxE + e] = p;
    if (valid && e < E) a.probs[t * E + e] = p;
  }
  if (sub == 0) {
    sm.lse_s[r] = valid ? lse : 0.f;
    if (valid) a.lse_out[t] = lse;
  }
  if (a.probs_only) return;  // uniform over the CTA

  // ---- the sorted window: the first min(k + 4, E) ranks by (logit
  //      descending, expert ascending), picked one per round by an arg-max
  //      over the half-warp; every other expert gets rank 255 (not chosen).
  //      A NaN logit counts as -inf here.
  const int win = min(k + 4, E);
  float cv[4];
  bool live[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int e = sub + 16 * i;
    cv[i] = (e < E && !isnan(h[i])) ? h[i] : -INFINITY;
    live[i] = true;
    if (e < E) rk[r * kMaxE + e] = 255;
  }
  for (int p = 0; p < win; ++p) {
    float bv = -INFINITY;
    int be = 0x7fffffff;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int e = sub + 16 * i;
      if (live[i] && (cv[i] > bv || (cv[i] == bv && e < be))) {
        bv = cv[i];
        be = e;
      }
    }
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(hm, bv, o);
      const int oe = __shfl_xor_sync(hm, be, o);
      if (ov > bv || (ov == bv && oe < be)) {
        bv = ov;
        be = oe;
      }
    }
    if ((be & 15) == sub) {  // the owner of the picked expert (be < E: win <= E live experts remain)
      live[be >> 4] = false;
      rk[r * kMaxE + be] = static_cast<uint8_t>(p);
    }
    if (sub == 0) {
      sv[r * kWin + p] = bv;
      se[r * kWin + p] = be;
    }
  }
  __syncwarp(hm);
  // near neighbours among the first k + 1 ranks (both sides lie in the window)
  bool nearv = false;
  for (int p = sub; p <= k && p < win; p += 16) {
    const float v = sv[r * kWin + p];
    const float up = p > 0 ? sv[r * kWin + p - 1] : INFINITY;
    const float dn = p + 1 < win ? sv[r * kWin + p + 1] : -INFINITY;
    if (fminf(up - v, v - dn) < near_gap(v)) nearv = true;
  }
  int rank[4];
  const bool near = valid && __any_sync(hm, nearv);
  if (tid == 0) *sm.qn = 0;
  epi_sync();
  // ---- queue the logits to recompute exactly: runs of near neighbours in the
  //      sorted window that reach into the top k (rare; one thread per token)
  if (sub == 0) {
    int cnt = 0, base = 0;
    bool fallback = false;
    if (near) {
      const int win = min(k + 4, E);
      // run bounds [ra, rb] with consecutive gaps under the bar
      int ra = 0;
      for (int j = 1; j <= win; ++j) {
        const bool link = j < win && (sv[r * kWin + j - 1] - sv[r * kWin + j] < near_gap(sv[r * kWin + j - 1]));
        if (!link) {
          if (j - 1 > ra && ra <= k - 1) {  // a run of length >= 2 reaching into the top k
            if (j == win && win < E) fallback = true;  // it may continue past the window
            cnt += j - ra;
          }
          ra = j;
        }
      }
      if (fallback) cnt = E;
      base = atomicAdd(sm.qn, cnt);
      if (fallback) {
        for (int e = 0; e < E; ++e) queue[base + e] = (static_cast<uint32_t>(r) << 8) | static_cast<uint32_t>(e);
      } else {
        int p = base;
        ra = 0;
        for (int j = 1; j <= win; ++j) {
          const bool link = j < win && (sv[r * kWin + j - 1] - sv[r * kWin + j] < near_gap(sv[r * kWin + j - 1]));
          if (!link) {
            if (j - 1 > ra && ra <= k - 1)
              for (int y = ra; y < j; ++y)
                queue[p++] = (static_cast<uint32_t>(r) << 8) | static_cast<uint32_t>(se[r * kWin + y]);
            ra = j;
          }
        }
      }
    }
    qb[r] = base;
    qb[kTile + r] = cnt;
    qb[2 * kTile + r] = fallback ? 1 : 0;
  }
  epi_sync();
  // ---- exact logits of the queued pairs: a warp per pair
  {
    const int nq = *sm.qn;
    const int w = tid >> 5;
    for (int it = w; it < nq; it += kEpiWarps) {
      const uint32_t code = queue[it];
      const int rr = static_cast<int>(code >> 8), e = static_cast<int>(code & 255u);
      const double v = exact_logit_warp(a.x + (t0 + rr) * a.d, a.w + static_cast<int64_t>(e) * a.d, a.d, lane);
      if (lane == 0) exact[it] = v + (a.bias != nullptr ? static_cast<double>(a.bias[e]) : 0.0);
    }
  }
  epi_sync();
  // ---- re-rank the queued experts of each such token by their exact logits
  if (sub == 0 && qb[kTile + r] > 0) {
    const int base = qb[r], cnt = qb[kTile + r];
    if (qb[2 * kTile + r] != 0) {  // every expert (queued in expert order): ranks from the exact values
      for (int i = 0; i < E; ++i) {
        const double vi = exact[base + i];
        int rr = 0;
        for (int j = 0; j < E; ++j) {
          const double vj = exact[base + j];
          rr += (vj > vi || (vj == vi && j < i)) ? 1 : 0;
        }
        rk[r * kMaxE + i] = static_cast<uint8_t>(rr);  // queue order is expert order
      }
    } else {
      // each queued run occupies consecutive ranks; sort every run by the exact
      // values (equal values: the lower expert) and hand its ranks back in order
      int i0 = 0;
      while (i0 < cnt) {
        const int first_rank = rk[r * kMaxE + (queue[base + i0] & 255u)];
        int i1 = i0 + 1;
        while (i1 < cnt && rk[r * kMaxE + (queue[base + i1] & 255u)] == first_rank + (i1 - i0)) ++i1;
        for (int i = i0; i < i1; ++i) {
          const int ei = static_cast<int>(queue[base + i] & 255u);
          const double vi = exact[base + i];
          int rr = 0;
          for (int j = i0; j < i1; ++j) {
            const int ej = static_cast<int>(queue[base + j] & 255u);
            const double vj = exact[base + j];
            rr += (vj > vi || (vj == vi && ej < ei)) ? 1 : 0;
          }
          rk[r * kMaxE + ei] = static_cast<uint8_t>(first_rank + rr);
        }
        i0 = i1;
      }
    }
  }
  epi_sync();
  // ---- outputs: the experts ranked below k, slot = rank
  float chosen_ex = 0.f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int e = sub + 16 * i;
    rank[i] = e < E ? static_cast<int>(rk[r * kMaxE + e]) : E;
    if (rank[i] < k) chosen_ex += ex[i];
  }
  float den = s;
  if (a.renorm) {  // the weights' denominator: the k chosen exponentials
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) chosen_ex += __shfl_xor_sync(hm, chosen_ex, o);
    den = chosen_ex;
  }
  if (valid) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int e = sub + 16 * i;
      if (rank[i] < k) {
        a.idx_out[t * k + rank[i]] = e;
        a.w_out[t * k + rank[i]] = ex[i] / den;
        atomicOr(&sm.mask[e], 1u << r);
      }
    }
  }
  epi_sync();
  // ---- ranks inside the chunk and the per-CTA partials
  if (valid) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int e = sub + 16 * i;
      if (rank[i] < k) a.local_rank[t * k + rank[i]] = __popc(sm.mask[e] & ((1u << r) - 1u));
    }
  }
  router_finish(a, sm, P, cta, ntiles, tid, lane);
}

// STAGES-deep ring, MINB CTAs per SM: one CTA with a 16-deep ring when the
// tiles fit on the SMs at once, two with 7-deep rings (one's epilogue then
// overlaps the other's loads) when there are more tiles than SMs.
template <int STAGES, int MINB>
__global__ void __launch_bounds__(kFusedThreads, MINB)
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
  int32_t* qn = s_last + 1;                                   // queued pairs
  int32_t* tot = s_last + 4;                                  // [kMaxE]
  double* tot_p = reinterpret_cast<double*>(tot + kMaxE);     // [kMaxE]
  // once the accumulator is complete the ring is free: the logits go to its start
  float* S = reinterpret_cast<float*>(ring + kOffS);          // [kTile][kLogitStride]

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
    tmem_alloc(tmem_holder, tmem_cols(a.NP));
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
        const uint32_t acc = tmem + static_cast<uint32_t>((kb % kChains) * a.NP);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          umma_bf16(acc, smem_desc_sw128(sa + kk * 32, 16, 1024), smem_desc_sw128(sb + kk * 32, 16, 1024), idesc,
                    (kb >= kChains || kk > 0) ? 1u : 0u);
        umma_commit(&empty[s]);
      }
      if (ok) umma_commit(acc_full);
    }
  }
  __syncwarp();  // the single-lane roles rejoin their warps
  {
    // ------------------------------------------------------------ epilogue (all 16 warps)
    const int tid = threadIdx.x;
    const int E = a.E, k = a.k;
    if (tid < kMaxE) mask[tid] = 0u;
    if (tid == 0) *qn = 0;
    if (!mbar_wait(acc_full, 0)) report(a.status, DEV_WAIT_TIMEOUT_EPILOGUE);
    tc_fence_after();
    if (warp == 4) {  // TMEM lanes 0..31 hold the 32 tokens' logits, one partial per chain
      const int nch = nk < kChains ? nk : kChains;
      for (int c = 0; c < a.NP; c += 16) {
        float hs[16];
        for (int j = 0; j < nch; ++j) {
          uint32_t v[16];
          tmem_ld16(tmem + static_cast<uint32_t>(j * a.NP + c), v);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 16; ++i) hs[i] = j == 0 ? __uint_as_float(v[i]) : hs[i] + __uint_as_float(v[i]);
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int e = c + i;
          float h = hs[i];
          if (e < E && a.bias != nullptr) h += a.bias[e];
          S[lane * kLogitStride + e] = (e < E) ? h : -INFINITY;
        }
      }
      for (int e = a.NP; e < kMaxE; ++e) S[lane * kLogitStride + e] = -INFINITY;
    }
    tc_fence_before();
    epi_sync();

    const EpiSmem sm{ring, mask, lse_s, s_last, qn, tot, tot_p};
    router_epilogue(a, sm, static_cast<int>(blockIdx.x), static_cast<int>(gridDim.x), tid, lane);
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, tmem_cols(a.NP));
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
constexpr int kEpiRing = (kEpiScratch + 1023) / 1024 * 1024;  // scratch of the epilogue and the last CTA's scan
constexpr size_t kEpiSmem = 1024 + kEpiRing + kMiscBytes;
static_assert(kEpiScratch <= ring_bytes(16), "the fused kernel's ring holds the epilogue scratch");

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
    tmem_alloc(tmem_holder, tmem_cols(a.NP));
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
        const uint32_t acc = tmem + static_cast<uint32_t>((kb % kChains) * a.NP);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          umma_bf16(acc, smem_desc_sw128(sa + kk * 32, 16, 1024), smem_desc_sw128(sb + kk * 32, 16, 1024), idesc,
                    (kb >= kChains || kk > 0) ? 1u : 0u);
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
    const int nch = nk < kChains ? nk : kChains;
    for (int c = 0; c < a.NP; c += 16) {
      float hs[16];
      for (int j = 0; j < nch; ++j) {
        uint32_t v[16];
        tmem_ld16(tmem + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(j * a.NP + c), v);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 16; ++i) hs[i] = j == 0 ? __uint_as_float(v[i]) : hs[i] + __uint_as_float(v[i]);
      }
      if (t < a.T) {
        float* dst = a.logit_part + (static_cast<int64_t>(ks) * a.T + t) * a.E;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int e = c + i;
          if (e < a.E) dst[e] = hs[i];
        }
      }
    }
  }
  __syncwarp();  // single-lane roles rejoin their warp before the block barrier
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, tmem_cols(a.NP));
  }
}

// The epilogue of tile `tile` of `ntiles` from logits in the workspace (the
// K-range partials, summed in a fixed order, plus the offset). `smem` is
// 1024-aligned with kEpiSmem bytes.
__device__ __forceinline__ void epi_tile(const RArgs& a, unsigned char* ring, int tile, int ntiles) {
  unsigned char* misc = ring + kEpiRing;
  uint32_t* mask = reinterpret_cast<uint32_t*>(misc);          // [kMaxE]
  float* lse_s = reinterpret_cast<float*>(mask + kMaxE);      // [kTile]
  int32_t* s_last = reinterpret_cast<int32_t*>(lse_s + kTile);
  int32_t* qn = s_last + 1;
  int32_t* tot = s_last + 4;                                  // [kMaxE]
  double* tot_p = reinterpret_cast<double*>(tot + kMaxE);     // [kMaxE]
  float* S = reinterpret_cast<float*>(ring + kOffS);
  const int tid = threadIdx.x, lane = tid & 31;
  const int64_t t0 = static_cast<int64_t>(tile) * kTile;
  if (tid < kMaxE) mask[tid] = 0u;
  if (tid == 0) *qn = 0;
  for (int i = tid; i < kTile * kMaxE; i += kEpiThreads) {
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
  const EpiSmem sm{ring, mask, lse_s, s_last, qn, tot, tot_p};
  router_epilogue(a, sm, tile, ntiles, tid, lane);
}

__global__ void __launch_bounds__(kEpiThreads, 2) router_epi_kernel(const RArgs a) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* ring = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  pdl_trigger();
  pdl_wait();
  epi_tile(a, ring, static_cast<int>(blockIdx.x), static_cast<int>(gridDim.x));
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
    return launch_dependent(router_tc_kernel<16, 1>, dim3(grid), dim3(kFusedThreads), smem_bytes(16), st, nullptr, 0, tx,
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
    return launch_dependent(router_tc_kernel<16, 1>, dim3(grid), dim3(kFusedThreads), smem_bytes(16), st, nullptr, 0, tx,
                            tw, a);
  a.logit_part = at<float>(ws, L.x_perm);
  a.ksplit = ks;
  e = launch_dependent(router_logits_kernel, dim3(grid_l, static_cast<unsigned>(ks)), dim3(kThreads), kLogitSmem, st,
                       nullptr, 0, tx128, tw, a);
  if (e != cudaSuccess) return e;
  return launch_dependent(router_epi_kernel, dim3(grid), dim3(kEpiThreads), kEpiSmem, st, nullptr, 0, a);
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
