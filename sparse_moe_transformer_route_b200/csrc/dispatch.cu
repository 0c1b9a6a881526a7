// Dispatch: group the (token, slot) pairs by expert, dropless, stable in token
// order, and gather token rows into expert-contiguous order.
//
// "Mixture-of-experts LLMs from scratch with OLMoE", section 2, `dispatch`: the
// flattened choices are argsorted stably by expert, `tokens = order // k`, and
// bincount gives each expert's group. A stable sort by expert of pairs numbered
// t*k+j, where each token names an expert at most once, is the order by
// (expert, token); this is what the kernels build, without a sort:
//
//   1. rank kernel: tokens are cut into chunks of 128. For each chunk and
//      expert, a 128-bit mask marks the tokens that chose the expert; a pair's
//      rank inside its chunk is a popcount of the mask below its token. The last
//      CTA to finish scans the per-chunk counts: the base of every (chunk,
//      expert), the unpadded offsets (the bincount prefix) and the padded group
//      starts (each expert's rows begin on a multiple of 128).
//   2. permute kernel: a warp per token computes its k sorted positions and
//      padded rows, writes perm / inv_perm / row_pair, and copies the token row
//      into its k rows of x_perm (read once, written k times). Optionally the
//      padding rows are zeroed and marked -1 in row_pair.
// Everything is integer work with a fixed result, independent of scheduling.
#include "moe_internal.h"
#include "sm100.cuh"

namespace moe {
namespace {

constexpr int kWords = kDispatchChunk / 32;

__global__ void __launch_bounds__(kDispatchChunk)
    rank_kernel(const int32_t* __restrict__ idx, int64_t T, int E, int k, int32_t* __restrict__ local_rank,
                int32_t* __restrict__ chunk_count, int32_t* __restrict__ chunk_base, int32_t* __restrict__ offsets_ws,
                int32_t* __restrict__ gs_ws, int32_t* __restrict__ offsets_user, int32_t* __restrict__ gs_user,
                int32_t* __restrict__ ticket, int32_t* __restrict__ status) {
  pdl_trigger();
  pdl_wait();  // reads and writes buffers an earlier kernel of the layer uses
  __shared__ uint32_t mask[kMaxExperts * kWords];
  __shared__ int32_t total[kMaxExperts];
  __shared__ int s_last;
  const int c = blockIdx.x;
  const int tl = threadIdx.x;
  const int64_t t = static_cast<int64_t>(c) * kDispatchChunk + tl;
  for (int i = tl; i < E * kWords; i += blockDim.x) mask[i] = 0u;
  __syncthreads();
  int ev[kMaxTopK];
  if (t < T) {
    for (int j = 0; j < k; ++j) {
      int e = idx[t * k + j];
      if (e < 0 || e >= E) {
        report(status, DEV_BAD_EXPERT_INDEX);
        e = -1;
      } else {
        atomicOr(&mask[e * kWords + (tl >> 5)], 1u << (tl & 31));
      }
      ev[j] = e;
    }
  }
  __syncthreads();
  if (t < T) {
    const int w = tl >> 5;
    const uint32_t below = (1u << (tl & 31)) - 1u;
    for (int j = 0; j < k; ++j) {
      const int e = ev[j];
      int r = -1;
      if (e >= 0) {
        r = __popc(mask[e * kWords + w] & below);
        for (int q = 0; q < w; ++q) r += __popc(mask[e * kWords + q]);
      }
      local_rank[t * k + j] = r;
    }
  }
  for (int e = tl; e < E; e += blockDim.x) {
    int n = 0;
    for (int q = 0; q < kWords; ++q) n += __popc(mask[e * kWords + q]);
    chunk_count[static_cast<size_t>(c) * E + e] = n;
  }
  __threadfence();
  __syncthreads();
  if (tl == 0) s_last = (atomicAdd(ticket, 1) == static_cast<int>(gridDim.x) - 1);
  __syncthreads();
  if (!s_last) return;

  __threadfence();
  const int nchunks = gridDim.x;
  for (int e = tl; e < E; e += blockDim.x) {
    int run = 0;
    // loads in batches of 16 so their L2 round trips overlap
    for (int c0 = 0; c0 < nchunks; c0 += 16) {
      int cv[16];
#pragma unroll
      for (int i = 0; i < 16; ++i)
        cv[i] = (c0 + i < nchunks) ? __ldcg(&chunk_count[static_cast<size_t>(c0 + i) * E + e]) : 0;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        if (c0 + i < nchunks) {
          chunk_base[static_cast<size_t>(c0 + i) * E + e] = run;
          run += cv[i];
        }
      }
    }
    total[e] = run;
  }
  __syncthreads();
  if (tl == 0) {
    int off = 0, gsv = 0;
    for (int e = 0; e < E; ++e) {
      offsets_ws[e] = off;
      gs_ws[e] = gsv;
      if (offsets_user != nullptr) offsets_user[e] = off;
      if (gs_user != nullptr) gs_user[e] = gsv;
      off += total[e];
      gsv += (total[e] + kRowAlign - 1) / kRowAlign * kRowAlign;
    }
    offsets_ws[E] = off;
    gs_ws[E] = gsv;
    if (offsets_user != nullptr) offsets_user[E] = off;
    if (gs_user != nullptr) gs_user[E] = gsv;
    if (static_cast<int64_t>(off) != T * k) report(status, DEV_COUNT_MISMATCH);
    *ticket = 0;
  }
}

template <typename T_>
__global__ void __launch_bounds__(256)
    permute_kernel(const int32_t* __restrict__ idx, const T_* __restrict__ x, int64_t T, int d, int E, int k,
                   const int32_t* __restrict__ local_rank, const int32_t* __restrict__ chunk_base,
                   const int32_t* __restrict__ offsets, const int32_t* __restrict__ gs, int32_t* __restrict__ perm,
                   int32_t* __restrict__ inv_perm, int32_t* __restrict__ row_pair, T_* __restrict__ x_perm,
                   int zero_pads) {
  pdl_trigger();
  pdl_wait();  // reads and writes buffers an earlier kernel of the layer uses
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t t = static_cast<int64_t>(blockIdx.x) * 8 + warp;
  const int nvec = d * static_cast<int>(sizeof(T_)) / 16;
  if (t < T) {
    int row = -1;
    if (lane < k) {
      const int e = idx[t * k + lane];
      const int lr = local_rank[t * k + lane];
      const int64_t pair = t * k + lane;
      if (e >= 0 && e < E && lr >= 0) {
        const int rank = chunk_base[(t / kDispatchChunk) * E + e] + lr;
        perm[offsets[e] + rank] = static_cast<int32_t>(pair);
        row = gs[e] + rank;
        row_pair[row] = static_cast<int32_t>(pair);
      }
      inv_perm[pair] = row;
    }
    int rows[kMaxTopK];
#pragma unroll
    for (int j = 0; j < kMaxTopK; ++j) rows[j] = __shfl_sync(0xffffffffu, row, j < k ? j : 0);
    const uint4* src = reinterpret_cast<const uint4*>(x + t * d);
    for (int v = lane; x_perm != nullptr && v < nvec; v += 32) {
      const uint4 val = src[v];
#pragma unroll
      for (int j = 0; j < kMaxTopK; ++j) {
        if (j < k && rows[j] >= 0) reinterpret_cast<uint4*>(x_perm + static_cast<int64_t>(rows[j]) * d)[v] = val;
      }
    }
  }
  if (zero_pads) {
    // padding rows of expert e: [gs[e] + count_e, gs[e+1])
    for (int e = blockIdx.x; e < E; e += gridDim.x) {
      const int r0 = gs[e] + (offsets[e + 1] - offsets[e]);
      const int r1 = gs[e + 1];
      for (int r = r0 + warp; r < r1; r += 8) {
        if (lane == 0) row_pair[r] = -1;
        if (x_perm == nullptr) continue;
        uint4* dst = reinterpret_cast<uint4*>(x_perm + static_cast<int64_t>(r) * d);
        for (int v = lane; v < nvec; v += 32) dst[v] = make_uint4(0, 0, 0, 0);
      }
    }
  }
}

}  // namespace

cudaError_t launch_dispatch_impl(const Shape& s, const int32_t* idx, const void* x, int32_t* offsets,
                                 int32_t* perm, int32_t* inv_perm, int32_t* group_start, void* x_perm, void* ws,
                                 const Workspace& L, bool zero_pads, cudaStream_t st) {
  // ctrl[2] is zero between calls (moe_workspace_init, then each launch's last CTA)
  int32_t* ctrl = at<int32_t>(ws, L.ctrl);
  cudaError_t e = cudaSuccess;
  const int nchunks = static_cast<int>(s.chunks());
  launch_dependent(rank_kernel, dim3(nchunks), dim3(kDispatchChunk), 0, st, nullptr, 0, idx, s.T, s.E, s.k, at<int32_t>(ws, L.local_rank),
                                                  at<int32_t>(ws, L.chunk_count), at<int32_t>(ws, L.chunk_base),
                                                  at<int32_t>(ws, L.offsets), at<int32_t>(ws, L.group_start), offsets,
                                                  group_start, ctrl + 2, ctrl);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_permute(s, idx, x, perm, inv_perm, x_perm, ws, L, zero_pads, st);
}

cudaError_t launch_permute(const Shape& s, const int32_t* idx, const void* x, int32_t* perm, int32_t* inv_perm,
                           void* x_perm, void* ws, const Workspace& L, bool zero_pads, cudaStream_t st) {
  const int grid = static_cast<int>((s.T + 7) / 8);
  const int grid2 = zero_pads ? (grid > s.E ? grid : s.E) : grid;
  if (s.fp32) {
    launch_dependent(permute_kernel<float>, dim3(grid2), dim3(256), 0, st, nullptr, 0, 
        idx, static_cast<const float*>(x), s.T, s.d, s.E, s.k, at<int32_t>(ws, L.local_rank),
        at<int32_t>(ws, L.chunk_base), at<int32_t>(ws, L.offsets), at<int32_t>(ws, L.group_start), perm, inv_perm,
        at<int32_t>(ws, L.row_pair), static_cast<float*>(x_perm), zero_pads ? 1 : 0);
  } else {
    launch_dependent(permute_kernel<__nv_bfloat16>, dim3(grid2), dim3(256), 0, st, nullptr, 0, 
        idx, static_cast<const __nv_bfloat16*>(x), s.T, s.d, s.E, s.k, at<int32_t>(ws, L.local_rank),
        at<int32_t>(ws, L.chunk_base), at<int32_t>(ws, L.offsets), at<int32_t>(ws, L.group_start), perm, inv_perm,
        at<int32_t>(ws, L.row_pair), static_cast<__nv_bfloat16*>(x_perm), zero_pads ? 1 : 0);
  }
  return cudaGetLastError();
}

cudaError_t launch_dispatch(const Shape& s, const int32_t* idx, const void* x, int32_t* offsets, int32_t* perm,
                            int32_t* inv_perm, int32_t* group_start, void* x_perm, void* ws, const Workspace& L,
                            cudaStream_t st) {
  return launch_dispatch_impl(s, idx, x, offsets, perm, inv_perm, group_start, x_perm, ws, L, true, st);
}

}  // namespace moe
