// Expert-choice routing: each expert takes the C tokens with the highest
// router probability for it, instead of each token taking its top-k experts.
//
// Method: "OLMoE: Open Mixture-of-Experts Language Models" (summary page),
// section 4.1.4 "Expert Choice vs. Token Choice" compares the two routings at
// equal compute. The pages give no formula, so the plain reading is built:
// the router probabilities p = softmax over experts of the logits (the same
// as token choice, computed by the tensor-core router in its
// probabilities-only mode); expert e keeps the C = ceil(T k / E) tokens (at
// most T) with the largest p[t, e], equal values going to the lower token
// index; its rows are those tokens in ascending token order; the weight of
// (t, e) is p[t, e]; a token sums its experts' outputs in ascending expert
// order and is zero when no expert took it.
//
// Kernels:
//   ec_select_kernel   one CTA per expert: a radix select (four 8-bit passes
//                      over the fp32 bit patterns, which order like the values
//                      since p >= 0) finds the C-th largest fp32 p[:, e]. Tokens
//                      whose fp32 p lies within 4e-4 (relative) of it, a band
//                      wider than any error of the fp32 probabilities (the
//                      token-choice router's 2e-4 bound on each logit, twice),
//                      are then ranked by their exact key h[t, e] - lse_t, the
//                      logits summed in fp64 from exact bf16 products (equal
//                      keys: the lower token index), and the ones above the
//                      band are taken outright; so the choice is the one an
//                      exact computation makes. One pass in token order then
//                      writes the chosen tokens, their weights, and for every
//                      token its row in the expert's group (or -1). One more
//                      CTA sums the z-loss and writes the group table.
//   ec_gather_kernel   x_perm[group_start[e] + i] = x[sel[e, i]], a warp per row.
// The expert GEMMs are the token-choice ones (every group holds C rows), and
// the combine is combine_ec_kernel in combine.cu.
#include "moe_internal.h"
#include "sm100.cuh"

namespace moe {
namespace {

constexpr int kEcThreads = 1024;
constexpr int kEcWarps = kEcThreads / 32;
// Columns up to this many tokens are staged in shared memory (160 KB); longer
// ones are read from the probabilities in L2 on every pass.
constexpr int64_t kEcSmemTokens = 40960;

// Tokens near the C-th value that one CTA re-ranks exactly; more (only when
// that many probabilities tie within the band) fall back to the fp32 order.
constexpr int kEcMaxCand = 256;

struct EcArgs {
  const float* probs;  // [T, E]
  const float* lse;    // [T]
  const __nv_bfloat16* x;   // [T, d] tokens (for the exact keys)
  const __nv_bfloat16* wr;  // [E, d] router weight
  const float* bias;        // [E] or null
  int d;
  int64_t T;
  int E, C, Cpad;
  int32_t* sel;          // [E, C] chosen tokens, ascending
  float* gates;          // [E, C] p[sel, e]
  int32_t* slot_row;     // [T, E] row of (t, e) in the grouped rows, or -1
  int32_t* group_start;  // [E + 1] e * Cpad
  int32_t* offsets;      // [E + 1] e * C
  int32_t* counts_ws;    // [E] C
  int32_t* counts_user;  // [E] or null
  float* losses_ws;      // [2] (0, L_z)
  float* losses_user;    // [2] or null
  int32_t* status;
};

__device__ __forceinline__ unsigned lanemask_lt() {
  unsigned m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

// Exclusive prefix over the block's warps of one count per warp (written by each
// warp's lane 0 into cnt[warp]); returns this warp's offset, and the total in *tot.
__device__ __forceinline__ int block_warp_scan(int* cnt, int* tot_s, int warp, int lane, int* tot) {
  __syncthreads();
  if (warp == 0) {
    const int v = cnt[lane];
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += u;
    }
    cnt[lane] = incl - v;
    if (lane == 31) *tot_s = incl;
  }
  __syncthreads();
  *tot = *tot_s;
  return cnt[warp];
}

// The exact logit <x_t, W_r[ee]> (+ bias) by one warp: lane l takes 8-element
// pieces l, l + 32, ... (coalesced), every load in flight before the
// arithmetic, exact bf16 products summed in fp64, then a fixed shuffle tree.
__device__ __forceinline__ double exact_logit(const EcArgs& a, int64_t t, int ee, int lane) {
  constexpr int kPieces = 4;  // 16-byte pieces per lane in flight (a 1024-thread CTA has 64 registers)
  const uint4* xrow = reinterpret_cast<const uint4*>(a.x + t * a.d);
  const uint4* wrow = reinterpret_cast<const uint4*>(a.wr + static_cast<int64_t>(ee) * a.d);
  const int nv = a.d / 8;
  double acc = 0.0;
  for (int v0 = 0; v0 < nv; v0 += 32 * kPieces) {
    uint4 xq[kPieces], wq[kPieces];
#pragma unroll
    for (int j = 0; j < kPieces; ++j) {
      const int v = v0 + lane + 32 * j;
      if (v < nv) {
        xq[j] = __ldg(xrow + v);
        wq[j] = __ldg(wrow + v);
      }
    }
#pragma unroll
    for (int j = 0; j < kPieces; ++j) {
      if (v0 + lane + 32 * j < nv) {
        const uint32_t xa[4] = {xq[j].x, xq[j].y, xq[j].z, xq[j].w}, wa[4] = {wq[j].x, wq[j].y, wq[j].z, wq[j].w};
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const float2 xf = bf16x2_to_float2(xa[c]);
          const float2 wf = bf16x2_to_float2(wa[c]);
          acc += static_cast<double>(xf.x * wf.x);  // exact products
          acc += static_cast<double>(xf.y * wf.y);
        }
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  return acc + (a.bias != nullptr ? static_cast<double>(a.bias[ee]) : 0.0);
}

__global__ void __launch_bounds__(kEcThreads, 1) ec_select_kernel(const EcArgs a) {
  extern __shared__ uint32_t keys_s[];  // [min(T, kEcSmemTokens)]
  __shared__ int hist[256];
  __shared__ int64_t cand_t[kEcMaxCand];
  __shared__ double cand_x[kEcMaxCand];
  __shared__ unsigned char cand_take[kEcMaxCand];
  __shared__ double cand_h[kMaxExperts];
  __shared__ int s_ncand, s_nhi;
  __shared__ int wcnt[kEcWarps];
  __shared__ int s_tot;
  __shared__ int s_digit, s_above;
  __shared__ double zred[kEcThreads];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int E = a.E;
  const int64_t T = a.T;

  if (static_cast<int>(blockIdx.x) == E) {
    // z-loss, (1/T) sum_t lse_t^2: per-thread strided sums, then a fixed tree
    double z = 0.0;
    for (int64_t t = tid; t < T; t += kEcThreads) {
      const double v = a.lse[t];
      z += v * v;
    }
    zred[tid] = z;
    __syncthreads();
    for (int w = kEcThreads / 2; w > 0; w >>= 1) {
      if (tid < w) zred[tid] += zred[tid + w];
      __syncthreads();
    }
    if (tid == 0) {
      const float lz = static_cast<float>(zred[0] / static_cast<double>(T));
      a.losses_ws[0] = 0.f;
      a.losses_ws[1] = lz;
      if (a.losses_user != nullptr) {
        a.losses_user[0] = 0.f;
        a.losses_user[1] = lz;
      }
      a.group_start[E] = E * a.Cpad;
      a.offsets[E] = E * a.C;
    }
    return;
  }

  const int e = blockIdx.x;
  if (tid == 0) {
    a.group_start[e] = e * a.Cpad;
    a.offsets[e] = e * a.C;
    a.counts_ws[e] = a.C;
    if (a.counts_user != nullptr) a.counts_user[e] = a.C;
  }
  const float* col = a.probs + e;
  const bool staged = T <= kEcSmemTokens;
  if (staged) {
    for (int64_t t = tid; t < T; t += kEcThreads) keys_s[t] = __float_as_uint(__ldg(col + t * E));
  }
  auto key = [&](int64_t t) -> uint32_t { return staged ? keys_s[t] : __float_as_uint(__ldg(col + t * E)); };

  // ---- radix select of the C-th largest key, most significant byte first
  uint32_t prefix = 0, pmask = 0;
  int need = a.C;  // keys still to take among those matching the prefix
  for (int shift = 24; shift >= 0; shift -= 8) {
    if (tid < 256) hist[tid] = 0;
    __syncthreads();
    // every lane runs every iteration, so the warp stays whole for the match
    for (int64_t c0 = 0; c0 < T; c0 += kEcThreads) {
      const int64_t t = c0 + tid;
      const uint32_t k = t < T ? key(t) : 0u;
      const bool in = t < T && (k & pmask) == prefix;
      const int dgt = in ? static_cast<int>((k >> shift) & 255u) : -1;
      // one shared-memory atomic per distinct digit in the warp
      const unsigned peers = __match_any_sync(0xffffffffu, dgt);
      if (in && lane == __ffs(peers) - 1) atomicAdd(&hist[dgt], __popc(peers));
    }
    __syncthreads();
    if (warp == 0) {
      // lane l holds digits 255-8l down to 248-8l; counts accumulate from the top
      int c[8], sum = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        c[j] = hist[255 - 8 * lane - j];
        sum += c[j];
      }
      int incl = sum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += u;
      }
      const int excl = incl - sum;
      if (excl < need && need <= incl) {  // exactly one lane
        int run = excl;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (run < need && run + c[j] >= need) {
            s_digit = 255 - 8 * lane - j;
            s_above = run;
          }
          run += c[j];
        }
      }
    }
    __syncthreads();
    need -= s_above;
    prefix |= static_cast<uint32_t>(s_digit) << shift;
    pmask |= 255u << shift;
    __syncthreads();
  }
  const uint32_t kstar = prefix;  // the C-th largest fp32 key; `need` of its equals are taken

  // ---- exact decision inside the band [lo, hi] around the C-th value
  const float vstar = __uint_as_float(kstar);
  const uint32_t lo_key = __float_as_uint(vstar * (1.0f - 4e-4f));
  const uint32_t hi_key = __float_as_uint(vstar * (1.0f + 4e-4f));
  if (tid == 0) {
    s_ncand = 0;
    s_nhi = 0;
  }
  __syncthreads();
  {
    int nhi = 0;
    for (int64_t t = tid; t < T; t += kEcThreads) {
      const uint32_t k = key(t);
      if (k > hi_key) {
        ++nhi;
      } else if (k >= lo_key) {
        const int slot = atomicAdd(&s_ncand, 1);
        if (slot < kEcMaxCand) cand_t[slot] = t;
      }
    }
    atomicAdd(&s_nhi, nhi);
  }
  __syncthreads();
  const int ncand = s_ncand;
  const bool exact = ncand <= kEcMaxCand;  // else: the fp32 order decides (many equal values)
  if (exact) {
    // each candidate's exact key h[t, e] - lse_t: its E exact logits by the
    // CTA's warps, then lse in fp64 (max, sum of exponentials, in expert order)
    for (int i = 0; i < ncand; ++i) {
      for (int ee = warp; ee < E; ee += kEcWarps) {
        const double hv = exact_logit(a, cand_t[i], ee, lane);
        if (lane == 0) cand_h[ee] = hv;
      }
      __syncthreads();
      if (warp == 0) {
        const double h0 = lane < E ? cand_h[lane] : -INFINITY, h1 = lane + 32 < E ? cand_h[lane + 32] : -INFINITY;
        double mx = fmax(h0, h1);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx = fmax(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        double sum = (lane < E ? exp(h0 - mx) : 0.0) + (lane + 32 < E ? exp(h1 - mx) : 0.0);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
        if (lane == 0) cand_x[i] = cand_h[e] - (mx + log(sum));
      }
      __syncthreads();
    }
    const int need_c = a.C - s_nhi;  // taken from the band
    for (int i = tid; i < ncand; i += kEcThreads) {
      int rank = 0;
      for (int j = 0; j < ncand; ++j)
        rank += (cand_x[j] > cand_x[i] || (cand_x[j] == cand_x[i] && cand_t[j] < cand_t[i])) ? 1 : 0;
      cand_take[i] = rank < need_c ? 1 : 0;
    }
    __syncthreads();
  }

  // ---- one pass in token order: ranks among the equals, then positions
  const int gs_e = e * a.Cpad;
  int run_eq = 0, run_sel = 0;
  for (int64_t c0 = 0; c0 < T; c0 += kEcThreads) {
    const int64_t t = c0 + tid;
    const bool valid = t < T;
    const uint32_t k = valid ? key(t) : 0u;
    bool gt = valid && k > kstar;
    bool eq = valid && k == kstar;
    if (exact) {  // above the band: taken; inside it: the exact decision; below: not
      bool tk = valid && k > hi_key;
      if (valid && k >= lo_key && k <= hi_key)
        for (int i = 0; i < ncand; ++i)
          if (cand_t[i] == t) tk = cand_take[i] != 0;
      gt = tk;
      eq = false;
    }
    const unsigned beq = __ballot_sync(0xffffffffu, eq);
    if (lane == 0) wcnt[warp] = __popc(beq);
    int eq_tot;
    const int eq_off = block_warp_scan(wcnt, &s_tot, warp, lane, &eq_tot);
    const int eq_rank = run_eq + eq_off + __popc(beq & lanemask_lt());
    const bool take = gt || (eq && eq_rank < need);
    const unsigned btk = __ballot_sync(0xffffffffu, take);
    __syncthreads();  // everyone has read wcnt
    if (lane == 0) wcnt[warp] = __popc(btk);
    int tk_tot;
    const int tk_off = block_warp_scan(wcnt, &s_tot, warp, lane, &tk_tot);
    const int pos = run_sel + tk_off + __popc(btk & lanemask_lt());
    if (valid) {
      const bool fits = take && pos < a.C;
      a.slot_row[t * E + e] = fits ? gs_e + pos : -1;
      if (fits) {
        a.sel[static_cast<int64_t>(e) * a.C + pos] = static_cast<int32_t>(t);
        a.gates[static_cast<int64_t>(e) * a.C + pos] = __uint_as_float(k);
      }
    }
    run_eq += eq_tot;
    run_sel += tk_tot;
    __syncthreads();  // wcnt and s_tot are reused by the next chunk
  }
  if (tid == 0 && run_sel != a.C) report(a.status, DEV_COUNT_MISMATCH);
}

// x_perm[group_start[e] + i] = x[sel[e, i]] for the E*C chosen rows, a warp per
// row, 16-byte loads all in flight before the stores.
// A token index outside [0, T) (a failed selection) is recorded and its row skipped.
__global__ void __launch_bounds__(256) ec_gather_kernel(const uint4* __restrict__ x, const int32_t* __restrict__ sel,
                                                        int64_t rows, int64_t T, int C, int Cpad, int vec_per_row,
                                                        uint4* __restrict__ x_perm, int32_t* status) {
  const int64_t r = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (r >= rows) return;
  const int e = static_cast<int>(r / C), i = static_cast<int>(r - static_cast<int64_t>(e) * C);
  const int32_t t = sel[r];
  if (t < 0 || t >= T) {
    if (lane == 0) report(status, DEV_COUNT_MISMATCH);
    return;
  }
  const uint4* src = x + static_cast<int64_t>(t) * vec_per_row;
  uint4* dst = x_perm + (static_cast<int64_t>(e) * Cpad + i) * vec_per_row;
  for (int v0 = 0; v0 < vec_per_row; v0 += 32 * 8) {
    uint4 q[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int v = v0 + j * 32 + lane;
      if (v < vec_per_row) q[j] = __ldg(src + v);
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int v = v0 + j * 32 + lane;
      if (v < vec_per_row) dst[v] = q[j];
    }
  }
}

}  // namespace

int64_t ec_default_capacity(const Shape& s) {
  const int64_t c = (s.T * s.k + s.E - 1) / s.E;
  return c < s.T ? c : s.T;
}

bool ec_capacity_ok(const Shape& s, int64_t C) {
  if (C < 1 || C > s.T || C > (int64_t(1) << 30) / s.E) return false;
  const int64_t cpad = (C + kRowAlign - 1) / kRowAlign * kRowAlign;
  return static_cast<int64_t>(s.E) * cpad <= s.P;
}

cudaError_t launch_ec_select(const Shape& s, int64_t C, const void* x, const void* w_router, const float* bias,
                             int32_t* counts, float* losses, void* ws, const Workspace& L, cudaStream_t st) {
  EcArgs a{};
  a.probs = at<float>(ws, L.probs);
  a.lse = at<float>(ws, L.lse);
  a.x = static_cast<const __nv_bfloat16*>(x);
  a.wr = static_cast<const __nv_bfloat16*>(w_router);
  a.bias = bias;
  a.d = s.d;
  a.T = s.T;
  a.E = s.E;
  a.C = static_cast<int>(C);
  a.Cpad = static_cast<int>((C + kRowAlign - 1) / kRowAlign * kRowAlign);
  a.sel = at<int32_t>(ws, L.ec_sel);
  a.gates = at<float>(ws, L.ec_gate);
  a.slot_row = at<int32_t>(ws, L.ec_slot);
  a.group_start = at<int32_t>(ws, L.group_start);
  a.offsets = at<int32_t>(ws, L.offsets);
  a.counts_ws = at<int32_t>(ws, L.counts);
  a.counts_user = counts;
  a.losses_ws = at<float>(ws, L.losses);
  a.losses_user = losses;
  a.status = at<int32_t>(ws, L.ctrl);
  const int64_t staged = s.T <= kEcSmemTokens ? s.T : 0;
  const size_t smem = static_cast<size_t>(staged) * 4;
  static std::atomic<size_t> set_select[kMaxDevices];
  const cudaError_t e = raise_smem_limit(reinterpret_cast<const void*>(ec_select_kernel), smem, set_select);
  if (e != cudaSuccess) return e;
  ec_select_kernel<<<s.E + 1, kEcThreads, smem, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_ec_gather(const Shape& s, int64_t C, const void* x, void* ws, const Workspace& L,
                             cudaStream_t st) {
  const int64_t rows = static_cast<int64_t>(s.E) * C;
  const int Cpad = static_cast<int>((C + kRowAlign - 1) / kRowAlign * kRowAlign);
  const int vec = static_cast<int>(static_cast<size_t>(s.d) * s.esize / 16);
  const int64_t blocks = (rows + 7) / 8;
  ec_gather_kernel<<<static_cast<unsigned>(blocks), 256, 0, st>>>(
      static_cast<const uint4*>(x), at<int32_t>(ws, L.ec_sel), rows, s.T, static_cast<int>(C), Cpad, vec,
      at<uint4>(ws, L.x_perm), at<int32_t>(ws, L.ctrl));
  return cudaGetLastError();
}

}  // namespace moe
