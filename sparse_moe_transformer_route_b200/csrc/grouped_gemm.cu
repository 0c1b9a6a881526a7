// Grouped GEMMs over variable-sized expert groups on tcgen05 tensor cores.
//
// One persistent kernel template serves every expert contraction of the layer
// ("OLMoE Guide", "Top-8 Softmax Routing Formulation": the SwiGLU expert;
// "Mixture-of-experts LLMs from scratch with OLMoE", section 2: each expert
// runs once on the rows that chose it; production kernels run all groups in one
// grouped matrix multiplication):
//
//   forward   gate_up : h = SiLU(X W_gate^T) * (X W_up^T)     M-grouped, SwiGLU epilogue
//             down    : O = H W_down^T                          M-grouped
//   backward  dG      : dG = dO W_down, then the SwiGLU derivative in the epilogue
//             dX      : dX = [dA|dB] W_gate_up                   M-grouped, B MN-major
//             dW      : dW_e = sum over the rows of expert e     K-grouped, A and B MN-major
//
// "M-grouped": the rows (M) of A are the expert-contiguous rows; expert e owns
// rows [group_start[e], group_start[e+1]) (a multiple of 128 rows, zero-padded
// past its count) and multiplies them by its own weight matrix. "K-grouped":
// the reduction runs over an expert's rows; each expert yields its own output
// matrix.
//
// Structure per CTA (one per SM, persistent over a static tile schedule read
// from device memory, so the host never learns the group sizes):
//   warp 0      : one thread issues TMA loads into a STAGES-deep smem ring
//   warp 1      : allocates TMEM; one thread issues tcgen05.mma (M=128, N=BN)
//   warps 2..5  : epilogue; tcgen05.ld the fp32 accumulator, apply the epilogue,
//                 store to global. The accumulator is double-buffered in TMEM so
//                 the epilogue of tile i overlaps the MMAs of tile i+1.
// Every mbarrier wait is bounded (about one second); a timeout is recorded in the
// workspace status word and the CTA unwinds, drains its copies, frees TMEM.
#include <cudaTypedefs.h>

#include <type_traits>

#include "moe_internal.h"
#include "sm100.cuh"

namespace moe {
namespace {

enum class Group { M, K };
enum class Epi { SwigluFwd, Store, SwigluBwd };

template <bool TF32_, bool A_MN_, bool B_MN_, Group G_, Epi EP_, int BN_>
struct Cfg {
  static constexpr bool TF32 = TF32_;
  static constexpr bool A_MN = A_MN_;
  static constexpr bool B_MN = B_MN_;
  static constexpr Group G = G_;
  static constexpr Epi EP = EP_;
  static constexpr int BN = BN_;
  using T = std::conditional_t<TF32, float, __nv_bfloat16>;
  static constexpr int BM = 128;
  static constexpr int ESZ = TF32 ? 4 : 2;
  static constexpr int BK = 128 / ESZ;      // K per stage (one 128-byte swizzle row when K-major)
  static constexpr int UK = 32 / ESZ;       // K per UMMA instruction
  static constexpr int KSTEPS = BK / UK;    // UMMAs per stage
  static constexpr int CH = 128 / ESZ;      // MN elements per 128-byte chunk when MN-major
  static constexpr int A_BYTES = BM * BK * ESZ;
  static constexpr int B_BYTES = BN * BK * ESZ;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int STAGES = (BN == 256) ? 4 : 6;
  static constexpr uint32_t IDESC = make_idesc(TF32, A_MN, B_MN, BM, BN);
  static constexpr uint32_t TMEM_COLS = (2 * BN <= 256) ? 256u : 512u;
  static constexpr int THREADS = 192;
  // N columns of output per tile (SwiGLU forward pairs BN/2 gate with BN/2 up columns)
  static constexpr int OUT_N = (EP == Epi::SwigluFwd) ? BN / 2 : BN;
  static constexpr size_t SMEM_BYTES = 1024 + static_cast<size_t>(STAGES) * STAGE_BYTES + 1024 +
                                       2 * (kMaxExperts + 1) * sizeof(int32_t);
  static_assert(BN == 128 || BN == 256, "tile N");
  static_assert(!(EP == Epi::SwigluFwd && B_MN), "gate/up weights are read K-major");
};

struct Args {
  const int32_t* group_start;  // [E+1] padded row starts
  const int32_t* offsets;      // [E+1] unpadded prefix: valid rows of e = offsets[e+1]-offsets[e]
  int E;
  int M_total;     // K-grouped: output rows per expert
  int N_total;     // output columns of the full product (f for gate_up's h, d for down, ...)
  int K_total;     // M-grouped: reduction length
  int b_rows_per_expert;  // rows of one expert's block in the B tensor map
  int f_half;      // SwiGLU: offset of the up half (rows of W_gate_up / columns of preact)
  void* out;
  int64_t ld_out;
  int64_t out_expert_stride;  // K-grouped: elements between experts' outputs
  void* out2;                 // SwiGLU forward: preact [P, 2f] or null
  int64_t ld_out2;
  const void* aux;            // SwiGLU backward: preact [P, 2f]
  int64_t ld_aux;
  int32_t* status;
};

struct Tile {
  int e;
  int m0;     // M-grouped: first row; K-grouped: first output row inside the expert
  int n0;     // first accumulator-mapped output column (see OUT_N)
  int valid;  // M-grouped: valid rows in this tile (rest are padding)
  int krow0;  // K-grouped: first row of the expert
  int nk;     // K stages
};

template <class C>
__device__ __forceinline__ int num_n_tiles(const Args& a) {
  return a.N_total / C::OUT_N;
}

template <class C>
__device__ __forceinline__ int total_tiles(const Args& a, const int32_t* gs) {
  if constexpr (C::G == Group::M) {
    return (gs[a.E] / C::BM) * num_n_tiles<C>(a);
  } else {
    return a.E * (a.M_total / C::BM) * num_n_tiles<C>(a);
  }
}

template <class C>
__device__ __forceinline__ Tile decode_tile(const Args& a, const int32_t* gs, const int32_t* off, int L) {
  Tile t;
  const int nN = num_n_tiles<C>(a);
  if constexpr (C::G == Group::M) {
    const int mt = L / nN;
    const int nt = L - mt * nN;
    const int row0 = mt * C::BM;
    // largest e with gs[e] <= row0 (groups are non-decreasing; empty groups are skipped)
    int lo = 0, hi = a.E - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (gs[mid] <= row0) lo = mid; else hi = mid - 1;
    }
    t.e = lo;
    t.m0 = row0;
    t.n0 = nt * C::OUT_N;
    const int cnt = off[lo + 1] - off[lo];
    t.valid = min(C::BM, gs[lo] + cnt - row0);
    t.krow0 = 0;
    t.nk = a.K_total / C::BK;
  } else {
    const int mT = a.M_total / C::BM;
    const int per_e = mT * nN;
    t.e = L / per_e;
    const int rem = L - t.e * per_e;
    const int mt = rem / nN;
    const int nt = rem - mt * nN;
    t.m0 = mt * C::BM;
    t.n0 = nt * C::OUT_N;
    t.valid = C::BM;
    t.krow0 = gs[t.e];
    t.nk = (gs[t.e + 1] - gs[t.e]) / C::BK;
  }
  return t;
}

// -------------------------------------------------------------- epilogue stores

template <typename T>
__device__ __forceinline__ void store16(T* dst, const float (&v)[16]) {
  if constexpr (std::is_same_v<T, float>) {
    float4* d4 = reinterpret_cast<float4*>(dst);
#pragma unroll
    for (int i = 0; i < 4; ++i) d4[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
  } else {
    uint4 w0, w1;
    w0.x = pack_bf16x2(v[0], v[1]);
    w0.y = pack_bf16x2(v[2], v[3]);
    w0.z = pack_bf16x2(v[4], v[5]);
    w0.w = pack_bf16x2(v[6], v[7]);
    w1.x = pack_bf16x2(v[8], v[9]);
    w1.y = pack_bf16x2(v[10], v[11]);
    w1.z = pack_bf16x2(v[12], v[13]);
    w1.w = pack_bf16x2(v[14], v[15]);
    uint4* d4 = reinterpret_cast<uint4*>(dst);
    d4[0] = w0;
    d4[1] = w1;
  }
}

template <typename T>
__device__ __forceinline__ void load16(const T* src, float (&v)[16]) {
  if constexpr (std::is_same_v<T, float>) {
    const float4* s4 = reinterpret_cast<const float4*>(src);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float4 q = s4[i];
      v[4 * i] = q.x;
      v[4 * i + 1] = q.y;
      v[4 * i + 2] = q.z;
      v[4 * i + 3] = q.w;
    }
  } else {
    const uint4* s4 = reinterpret_cast<const uint4*>(src);
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const uint4 q = s4[i];
      const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162*>(&w[j]);
        const float2 f = __bfloat1622float2(b);
        v[8 * i + 2 * j] = f.x;
        v[8 * i + 2 * j + 1] = f.y;
      }
    }
  }
}

// -------------------------------------------------------------- the kernel

template <class C>
__global__ void __launch_bounds__(C::THREADS, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                        const Args a) {
  using T = typename C::T;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  // 1024-byte alignment for the swizzle atoms
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  unsigned char* stage_base = smem;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + static_cast<size_t>(C::STAGES) * C::STAGE_BYTES);
  uint64_t* full = bars;
  uint64_t* empty = bars + C::STAGES;
  uint64_t* acc_full = bars + 2 * C::STAGES;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  int32_t* gs = reinterpret_cast<int32_t*>(smem + static_cast<size_t>(C::STAGES) * C::STAGE_BYTES + 1024);
  int32_t* off = gs + (kMaxExperts + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  for (int i = threadIdx.x; i <= a.E; i += blockDim.x) {
    gs[i] = a.group_start[i];
    off[i] = (a.offsets != nullptr) ? a.offsets[i] : 0;
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 128);
    }
    mbar_init(drain, 1);
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  const int n_tiles = total_tiles<C>(a, gs);

  if (warp == 0) {
    // ------------------------------------------------ TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;
      bool ok = true;
      for (int L = blockIdx.x; L < n_tiles && ok; L += gridDim.x) {
        const Tile t = decode_tile<C>(a, gs, off, L);
        for (int kb = 0; kb < t.nk; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u)) {
            report(a.status, DEV_WAIT_TIMEOUT_PRODUCER);
            ok = false;
            break;
          }
          unsigned char* sa = stage_base + static_cast<size_t>(stage) * C::STAGE_BYTES;
          unsigned char* sb = sa + C::A_BYTES;
          mbar_arrive_expect_tx(&full[stage], C::STAGE_BYTES);
          // A operand
          if constexpr (!C::A_MN) {
            tma_load_2d(&tmA, &full[stage], sa, kb * C::BK, t.m0);
          } else {
#pragma unroll
            for (int ch = 0; ch < C::BM / C::CH; ++ch)
              tma_load_2d(&tmA, &full[stage], sa + ch * (C::BK * 128), t.m0 + ch * C::CH,
                          t.krow0 + kb * C::BK);
          }
          // B operand
          if constexpr (C::EP == Epi::SwigluFwd) {
            const int rb = t.e * a.b_rows_per_expert + t.n0;
            tma_load_2d(&tmB, &full[stage], sb, kb * C::BK, rb);
            tma_load_2d(&tmB, &full[stage], sb + (C::BN / 2) * 128, kb * C::BK, rb + a.f_half);
          } else if constexpr (!C::B_MN) {
            tma_load_2d(&tmB, &full[stage], sb, kb * C::BK, t.e * a.b_rows_per_expert + t.n0);
          } else {
            const int kr = (C::G == Group::M) ? (t.e * a.b_rows_per_expert + kb * C::BK)
                                              : (t.krow0 + kb * C::BK);
#pragma unroll
            for (int ch = 0; ch < C::BN / C::CH; ++ch)
              tma_load_2d(&tmB, &full[stage], sb + ch * (C::BK * 128), t.n0 + ch * C::CH, kr);
          }
          ++issued;
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // Drain: wait until every copy this thread issued has landed.
      for (int s = 0; s < C::STAGES; ++s) {
        if (issued <= s) break;
        const int last = ((issued - 1 - s) / C::STAGES) * C::STAGES + s;  // last issue index into stage s
        if (!mbar_wait(&full[s], static_cast<uint32_t>((last / C::STAGES) & 1))) {
          report(a.status, DEV_WAIT_TIMEOUT_DRAIN);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int L = blockIdx.x; L < n_tiles && ok; L += gridDim.x) {
        const Tile t = decode_tile<C>(a, gs, off, L);
        if (t.nk == 0) continue;  // the epilogue writes zeros without TMEM
        if (!mbar_wait(&acc_empty[acc], acc_phase ^ 1u)) {
          report(a.status, DEV_WAIT_TIMEOUT_MMA);
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * C::BN);
        for (int kb = 0; kb < t.nk; ++kb) {
          if (!mbar_wait(&full[stage], phase)) {
            report(a.status, DEV_WAIT_TIMEOUT_MMA);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(stage_base + static_cast<size_t>(stage) * C::STAGE_BYTES);
          const uint32_t sb = sa + C::A_BYTES;
#pragma unroll
          for (int kk = 0; kk < C::KSTEPS; ++kk) {
            const uint64_t ad = C::A_MN ? smem_desc_sw128(sa + kk * C::UK * 128, C::BK * 128, 1024)
                                        : smem_desc_sw128(sa + kk * C::UK * C::ESZ, 16, 1024);
            const uint64_t bd = C::B_MN ? smem_desc_sw128(sb + kk * C::UK * 128, C::BK * 128, 1024)
                                        : smem_desc_sw128(sb + kk * C::UK * C::ESZ, 16, 1024);
            const uint32_t accum = (kb > 0 || kk > 0) ? 1u : 0u;
            if constexpr (C::TF32)
              umma_tf32(d_tmem, ad, bd, C::IDESC, accum);
            else
              umma_bf16(d_tmem, ad, bd, C::IDESC, accum);
          }
          umma_commit(&empty[stage]);  // frees the smem slot once these MMAs finish
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit(&acc_full[acc]);
        if (++acc == 2) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
      // Drain: every MMA this thread issued has completed once `drain` flips.
      umma_commit(drain);
      if (!mbar_wait(drain, 0)) report(a.status, DEV_WAIT_TIMEOUT_DRAIN);
    }
  } else {
    // ------------------------------------------------ epilogue (warps 2..5)
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    const int r_local = q * 32 + lane;
    int acc = 0;
    uint32_t acc_phase = 0;
    T* out = static_cast<T*>(a.out);
    for (int L = blockIdx.x; L < n_tiles; L += gridDim.x) {
      const Tile t = decode_tile<C>(a, gs, off, L);
      const bool row_ok = r_local < t.valid;
      const int64_t row = static_cast<int64_t>(t.m0) + r_local;
      T* orow;
      if constexpr (C::G == Group::M)
        orow = out + row * a.ld_out + t.n0;
      else
        orow = out + static_cast<int64_t>(t.e) * a.out_expert_stride + row * a.ld_out + t.n0;

      if (t.nk == 0) {  // K-grouped expert with no rows: its gradient is zero
        float z[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) z[i] = 0.f;
        for (int c = 0; c < C::OUT_N; c += 16) store16<T>(orow + c, z);
        continue;
      }
      if (!mbar_wait(&acc_full[acc], acc_phase)) {
        report(a.status, DEV_WAIT_TIMEOUT_EPILOGUE);
        break;
      }
      tc_fence_after();
      const uint32_t tbase = tmem_base + static_cast<uint32_t>(acc * C::BN) + (static_cast<uint32_t>(q * 32) << 16);

      if constexpr (C::EP == Epi::Store) {
        for (int c = 0; c < C::BN; c += 16) {
          uint32_t r[16];
          tmem_ld16(tbase + c, r);
          tmem_ld_wait();
          float v[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) v[i] = row_ok ? __uint_as_float(r[i]) : 0.f;
          store16<T>(orow + c, v);
        }
      } else if constexpr (C::EP == Epi::SwigluFwd) {
        T* prow = (a.out2 != nullptr) ? static_cast<T*>(a.out2) + row * a.ld_out2 + t.n0 : nullptr;
        for (int c = 0; c < C::BN / 2; c += 16) {
          uint32_t rg[16], ru[16];
          tmem_ld16(tbase + c, rg);
          tmem_ld16(tbase + C::BN / 2 + c, ru);
          tmem_ld_wait();
          float g[16], u[16], hv[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            g[i] = row_ok ? __uint_as_float(rg[i]) : 0.f;
            u[i] = row_ok ? __uint_as_float(ru[i]) : 0.f;
            hv[i] = silu_f(g[i]) * u[i];
          }
          store16<T>(orow + c, hv);
          if (prow != nullptr) {
            store16<T>(prow + c, g);
            store16<T>(prow + a.f_half + c, u);
          }
        }
      } else {  // SwigluBwd: accumulator holds dG for columns [n0, n0+BN)
        const T* arow = static_cast<const T*>(a.aux) + row * a.ld_aux + t.n0;
        for (int c = 0; c < C::BN; c += 16) {
          uint32_t r[16];
          tmem_ld16(tbase + c, r);
          tmem_ld_wait();
          float da[16], db[16];
          if (row_ok) {
            float av[16], bv[16];
            load16<T>(arow + c, av);
            load16<T>(arow + a.f_half + c, bv);
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const float dg = __uint_as_float(r[i]);
              const float sg = 1.0f / (1.0f + __expf(-av[i]));
              da[i] = dg * bv[i] * (sg * (1.0f + av[i] * (1.0f - sg)));
              db[i] = dg * av[i] * sg;
            }
          } else {
#pragma unroll
            for (int i = 0; i < 16; ++i) da[i] = db[i] = 0.f;
          }
          store16<T>(orow + c, da);
          store16<T>(orow + a.f_half + c, db);
        }
      }
      tc_fence_before();
      mbar_arrive(&acc_empty[acc]);
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

// -------------------------------------------------------------- host side

PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// 2-D tensor map over a row-major [rows, cols] matrix, 128-byte swizzle.
bool make_map(CUtensorMap* m, const void* base, bool fp32, uint64_t rows, uint64_t cols, uint32_t box_cols,
              uint32_t box_rows) {
  auto enc = get_encode();
  if (enc == nullptr) return false;
  const size_t es = fp32 ? 4 : 2;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * es};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, fp32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                   const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <class C>
cudaError_t launch(const CUtensorMap& ta, const CUtensorMap& tb, const Args& a, int max_tiles, cudaStream_t st) {
  static bool configured = false;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(grouped_gemm_kernel<C>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(C::SMEM_BYTES));
    if (e != cudaSuccess) return e;
    configured = true;
  }
  int grid = device_sm_count();
  if (max_tiles < grid) grid = max_tiles;
  if (grid <= 0) return cudaSuccess;
  grouped_gemm_kernel<C><<<grid, C::THREADS, C::SMEM_BYTES, st>>>(ta, tb, a);
  return cudaGetLastError();
}

Args base_args(const Shape& s, const int32_t* gs, const int32_t* off, int32_t* status) {
  Args a{};
  a.group_start = gs;
  a.offsets = off;
  a.E = s.E;
  a.status = status;
  return a;
}

int ch_elems(bool fp32) { return fp32 ? 32 : 64; }

}  // namespace

// Tile N for a forward GEMM whose accumulator covers `n` columns per expert.
static int pick_bn(int n) { return (n % 256 == 0) ? 256 : 128; }

cudaError_t launch_gate_up(const Shape& s, const void* x_perm, const int32_t* group_start,
                           const int32_t* offsets, const void* w_gate_up, void* h, void* preact, int32_t* status,
                           cudaStream_t st) {
  // accumulator: BN/2 gate columns and BN/2 up columns of the same outputs
  const int bn = ((s.f % 128) == 0) ? 256 : 128;
  const int kcols = ch_elems(s.fp32);
  CUtensorMap ta, tb;
  if (!make_map(&ta, x_perm, s.fp32, s.P, s.d, kcols, 128)) return cudaErrorInvalidValue;
  if (!make_map(&tb, w_gate_up, s.fp32, static_cast<uint64_t>(s.E) * 2 * s.f, s.d, kcols, bn / 2))
    return cudaErrorInvalidValue;
  Args a = base_args(s, group_start, offsets, status);
  a.N_total = s.f;
  a.K_total = s.d;
  a.b_rows_per_expert = 2 * s.f;
  a.f_half = s.f;
  a.out = h;
  a.ld_out = s.f;
  a.out2 = preact;
  a.ld_out2 = 2 * s.f;
  const int max_tiles = static_cast<int>((s.P / 128) * (s.f / (bn / 2)));
  if (s.fp32) {
    if (bn == 256) return launch<Cfg<true, false, false, Group::M, Epi::SwigluFwd, 256>>(ta, tb, a, max_tiles, st);
    return launch<Cfg<true, false, false, Group::M, Epi::SwigluFwd, 128>>(ta, tb, a, max_tiles, st);
  }
  if (bn == 256) return launch<Cfg<false, false, false, Group::M, Epi::SwigluFwd, 256>>(ta, tb, a, max_tiles, st);
  return launch<Cfg<false, false, false, Group::M, Epi::SwigluFwd, 128>>(ta, tb, a, max_tiles, st);
}

cudaError_t launch_down(const Shape& s, const void* h, const int32_t* group_start, const int32_t* offsets,
                        const void* w_down, void* o_perm, int32_t* status, cudaStream_t st) {
  const int bn = pick_bn(s.d);
  const int kcols = ch_elems(s.fp32);
  CUtensorMap ta, tb;
  if (!make_map(&ta, h, s.fp32, s.P, s.f, kcols, 128)) return cudaErrorInvalidValue;
  if (!make_map(&tb, w_down, s.fp32, static_cast<uint64_t>(s.E) * s.d, s.f, kcols, bn))
    return cudaErrorInvalidValue;
  Args a = base_args(s, group_start, offsets, status);
  a.N_total = s.d;
  a.K_total = s.f;
  a.b_rows_per_expert = s.d;
  a.out = o_perm;
  a.ld_out = s.d;
  const int max_tiles = static_cast<int>((s.P / 128) * (s.d / bn));
  if (s.fp32) {
    if (bn == 256) return launch<Cfg<true, false, false, Group::M, Epi::Store, 256>>(ta, tb, a, max_tiles, st);
    return launch<Cfg<true, false, false, Group::M, Epi::Store, 128>>(ta, tb, a, max_tiles, st);
  }
  if (bn == 256) return launch<Cfg<false, false, false, Group::M, Epi::Store, 256>>(ta, tb, a, max_tiles, st);
  return launch<Cfg<false, false, false, Group::M, Epi::Store, 128>>(ta, tb, a, max_tiles, st);
}

// dG = dO W_down (K = d, B read MN-major from W_down [E*d, f]); epilogue forms
// dA = dG * b * silu'(a), dB = dG * silu(a) from the saved pre-activations.
cudaError_t launch_down_backward_data(const Shape& s, const void* dout, const int32_t* group_start,
                                      const int32_t* offsets, const void* w_down, const void* preact, void* dab,
                                      int32_t* status, cudaStream_t st) {
  const int bn = pick_bn(s.f);
  const int kc = ch_elems(s.fp32);
  const int bk = s.fp32 ? 32 : 64;
  CUtensorMap ta, tb;
  if (!make_map(&ta, dout, s.fp32, s.P, s.d, kc, 128)) return cudaErrorInvalidValue;
  if (!make_map(&tb, w_down, s.fp32, static_cast<uint64_t>(s.E) * s.d, s.f, kc, bk)) return cudaErrorInvalidValue;
  Args a = base_args(s, group_start, offsets, status);
  a.N_total = s.f;
  a.K_total = s.d;
  a.b_rows_per_expert = s.d;
  a.f_half = s.f;
  a.out = dab;
  a.ld_out = 2 * s.f;
  a.aux = preact;
  a.ld_aux = 2 * s.f;
  const int max_tiles = static_cast<int>((s.P / 128) * (s.f / bn));
  if (s.fp32) {
    if (bn == 256) return launch<Cfg<true, false, true, Group::M, Epi::SwigluBwd, 256>>(ta, tb, a, max_tiles, st);
    return launch<Cfg<true, false, true, Group::M, Epi::SwigluBwd, 128>>(ta, tb, a, max_tiles, st);
  }
  if (bn == 256) return launch<Cfg<false, false, true, Group::M, Epi::SwigluBwd, 256>>(ta, tb, a, max_tiles, st);
  return launch<Cfg<false, false, true, Group::M, Epi::SwigluBwd, 128>>(ta, tb, a, max_tiles, st);
}

// dX_perm = [dA|dB] W_gate_up (K = 2f, B read MN-major from W_gate_up [E*2f, d]).
cudaError_t launch_gate_up_backward_data(const Shape& s, const void* dab, const int32_t* group_start,
                                         const int32_t* offsets, const void* w_gate_up, void* dx_perm,
                                         int32_t* status, cudaStream_t st) {
  const int bn = pick_bn(s.d);
  const int kc = ch_elems(s.fp32);
  const int bk = s.fp32 ? 32 : 64;
  CUtensorMap ta, tb;
  if (!make_map(&ta, dab, s.fp32, s.P, 2 * s.f, kc, 128)) return cudaErrorInvalidValue;
  if (!make_map(&tb, w_gate_up, s.fp32, static_cast<uint64_t>(s.E) * 2 * s.f, s.d, kc, bk))
    return cudaErrorInvalidValue;
  Args a = base_args(s, group_start, offsets, status);
  a.N_total = s.d;
  a.K_total = 2 * s.f;
  a.b_rows_per_expert = 2 * s.f;
  a.out = dx_perm;
  a.ld_out = s.d;
  const int max_tiles = static_cast<int>((s.P / 128) * (s.d / bn));
  if (s.fp32) {
    if (bn == 256) return launch<Cfg<true, false, true, Group::M, Epi::Store, 256>>(ta, tb, a, max_tiles, st);
    return launch<Cfg<true, false, true, Group::M, Epi::Store, 128>>(ta, tb, a, max_tiles, st);
  }
  if (bn == 256) return launch<Cfg<false, false, true, Group::M, Epi::Store, 256>>(ta, tb, a, max_tiles, st);
  return launch<Cfg<false, false, true, Group::M, Epi::Store, 128>>(ta, tb, a, max_tiles, st);
}

namespace {
// C_e[m, n] = sum over rows r of expert e of A[r, m] * B[r, n]  (both MN-major)
cudaError_t launch_kgrouped(const Shape& s, const void* A, int M_total, const void* B, int N_total,
                            const int32_t* gs, const int32_t* off, void* out, int32_t* status, cudaStream_t st) {
  const int bn = pick_bn(N_total);
  const int kc = ch_elems(s.fp32);
  const int bk = s.fp32 ? 32 : 64;
  CUtensorMap ta, tb;
  if (!make_map(&ta, A, s.fp32, s.P, M_total, kc, bk)) return cudaErrorInvalidValue;
  if (!make_map(&tb, B, s.fp32, s.P, N_total, kc, bk)) return cudaErrorInvalidValue;
  Args a = base_args(s, gs, off, status);
  a.M_total = M_total;
  a.N_total = N_total;
  a.out = out;
  a.ld_out = N_total;
  a.out_expert_stride = static_cast<int64_t>(M_total) * N_total;
  const int max_tiles = s.E * (M_total / 128) * (N_total / bn);
  if (s.fp32) {
    if (bn == 256) return launch<Cfg<true, true, true, Group::K, Epi::Store, 256>>(ta, tb, a, max_tiles, st);
    return launch<Cfg<true, true, true, Group::K, Epi::Store, 128>>(ta, tb, a, max_tiles, st);
  }
  if (bn == 256) return launch<Cfg<false, true, true, Group::K, Epi::Store, 256>>(ta, tb, a, max_tiles, st);
  return launch<Cfg<false, true, true, Group::K, Epi::Store, 128>>(ta, tb, a, max_tiles, st);
}
}  // namespace

// dW_down,e = dO_e^T H_e   ([d, f]);   dW_gate_up,e = [dA|dB]_e^T X_perm,e   ([2f, d]).
cudaError_t launch_weight_grads(const Shape& s, const void* dout, const void* h, const void* dab,
                                const void* x_perm, const int32_t* group_start, void* dw_down, void* dw_gate_up,
                                int32_t* status, cudaStream_t st) {
  cudaError_t e = launch_kgrouped(s, dout, s.d, h, s.f, group_start, nullptr, dw_down, status, st);
  if (e != cudaSuccess) return e;
  return launch_kgrouped(s, dab, 2 * s.f, x_perm, s.d, group_start, nullptr, dw_gate_up, status, st);
}

}  // namespace moe
