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

// H = number of 128-row halves per tile. H = 2 (a 256-row tile) issues two
// M=128 UMMAs on every B stage, so each byte of B feeds twice the MMA work:
// 64 B per MMA cycle instead of 96, the difference between starving and not
// on HBM-resident weights. A 256-row tile whose second half lies past its
// expert's rows issues only the first half.
// O32: fp32 output whatever the operand type: the plain store's result (weight
// gradients kept in fp32 for the caller's optimizer), or the SwiGLU forward's
// pre-activations (kept for the backward, which reads no rounded copy of them).
template <bool TF32_, bool A_MN_, bool B_MN_, Group G_, Epi EP_, int BN_, int H_ = 1, bool O32_ = false>
struct Cfg {
  static constexpr bool TF32 = TF32_;
  static constexpr bool A_MN = A_MN_;
  static constexpr bool B_MN = B_MN_;
  static constexpr Group G = G_;
  static constexpr Epi EP = EP_;
  static constexpr int BN = BN_;
  static constexpr int H = H_;
  using T = std::conditional_t<TF32, float, __nv_bfloat16>;
  static constexpr bool O32 = O32_;
  using OutT = std::conditional_t<TF32 || O32, float, __nv_bfloat16>;
  static constexpr int BM = 128 * H;
  static constexpr int ESZ = TF32 ? 4 : 2;
  static constexpr int BK = 128 / ESZ;      // K per stage (one 128-byte swizzle row when K-major)
  static constexpr int UK = 32 / ESZ;       // K per UMMA instruction
  static constexpr int KSTEPS = BK / UK;    // UMMAs per stage and half
  static constexpr int CH = 128 / ESZ;      // MN elements per 128-byte chunk when MN-major
  static constexpr int A_HALF = 128 * BK * ESZ;  // bytes of one 128-row half of A per stage
  static constexpr int A_BYTES = H * A_HALF;
  static constexpr int B_BYTES = BN * BK * ESZ;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int ACC_BUFS = (2 * H * BN <= 512) ? 2 : 1;  // TMEM holds 512 fp32 columns
  static constexpr uint32_t IDESC = make_idesc(TF32, A_MN, B_MN, 128, BN);
  static constexpr uint32_t TMEM_COLS = (ACC_BUFS * H * BN <= 256) ? 256u : 512u;
  // two epilogue warps per TMEM lane quarter and half, each on half of the columns
  static constexpr int EPI_WARPS = 8 * H;
  static constexpr int THREADS = 64 + 32 * EPI_WARPS;
  // Each epilogue warp stages a 32 x 32 output chunk in shared memory (rows
  // padded by 16 bytes against bank conflicts) and writes it back as whole rows.
  // staging rows sized for the operand type (fp32 output of bf16 operands
  // leaves in two passes), so fp32 output costs no ring stage
  static constexpr int STG_PITCH = 32 * static_cast<int>(sizeof(T)) + 16;
  static constexpr int STG_WARP_BYTES = 32 * STG_PITCH;
  static constexpr int STG_BYTES = EPI_WARPS * STG_WARP_BYTES;
  static constexpr int MISC_BYTES = 1024 + 3 * (kMaxExperts + 1) * static_cast<int>(sizeof(int32_t));
  static constexpr int STAGES = (227 * 1024 - 1024 - MISC_BYTES - STG_BYTES) / STAGE_BYTES;
  // N columns of output per tile (SwiGLU forward pairs BN/2 gate with BN/2 up columns)
  static constexpr int OUT_N = (EP == Epi::SwigluFwd) ? BN / 2 : BN;
  static constexpr size_t SMEM_BYTES =
      1024 + static_cast<size_t>(STAGES) * STAGE_BYTES + STG_BYTES + static_cast<size_t>(MISC_BYTES);
  static_assert(STAGES >= 2, "shared memory ring");
  static_assert(BN == 128 || BN == 256, "tile N");
  static_assert(H == 1 || H == 2, "tile M");
  static_assert(!(H == 2 && TF32), "256-row tiles are bf16 only");
  static_assert(!(EP == Epi::SwigluFwd && B_MN), "gate/up weights are read K-major");
  static_assert(!O32 || EP != Epi::SwigluBwd, "fp32 output for plain stores and saved pre-activations");
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
  int m0;      // M-grouped: first row; K-grouped: first output row inside the expert
  int n0;      // first accumulator-mapped output column (see OUT_N)
  int valid;   // M-grouped: valid rows in this tile (rest are padding)
  int halves;  // 128-row halves to compute (1 or 2 for H = 2; always 1 for H = 1)
  int krow0;   // K-grouped: first row of the expert
  int nk;      // K stages
};

template <class C>
__device__ __forceinline__ int num_n_tiles(const Args& a) {
  return a.N_total / C::OUT_N;
}

// ts[e]: first M-tile of expert e (M-grouped); groups are multiples of 128
// rows, so a group of R rows spans ceil(R / BM) tiles.
template <class C>
__device__ __forceinline__ void tile_starts(const Args& a, const int32_t* gs, int32_t* ts) {
  if (threadIdx.x == 0) {
    int acc = 0;
    for (int e = 0; e < a.E; ++e) {
      ts[e] = acc;
      acc += (gs[e + 1] - gs[e] + C::BM - 1) / C::BM;
    }
    ts[a.E] = acc;
  }
}

template <class C>
__device__ __forceinline__ int total_tiles(const Args& a, const int32_t* ts) {
  if constexpr (C::G == Group::M) {
    return ts[a.E] * num_n_tiles<C>(a);
  } else {
    return a.E * (a.M_total / C::BM) * num_n_tiles<C>(a);
  }
}

template <class C>
__device__ __forceinline__ Tile decode_tile(const Args& a, const int32_t* gs, const int32_t* off, const int32_t* ts,
                                            int L) {
  Tile t;
  const int nN = num_n_tiles<C>(a);
  if constexpr (C::G == Group::M) {
    const int mt = L / nN;
    const int nt = L - mt * nN;
    // largest e with ts[e] <= mt (experts without rows own no tiles and are skipped)
    int lo = 0, hi = a.E - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (ts[mid] <= mt) lo = mid; else hi = mid - 1;
    }
    const int row0 = gs[lo] + (mt - ts[lo]) * C::BM;
    t.e = lo;
    t.m0 = row0;
    t.n0 = nt * C::OUT_N;
    const int cnt = off[lo + 1] - off[lo];
    t.valid = min(C::BM, gs[lo] + cnt - row0);
    t.halves = (C::H == 2 && row0 + 128 < gs[lo + 1]) ? 2 : 1;
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
    t.halves = C::H;
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
        const float2 f = bf16x2_to_float2(w[j]);
        v[8 * i + 2 * j] = f.x;
        v[8 * i + 2 * j + 1] = f.y;
      }
    }
  }
}

// One warp writes a 32-row x 32-column chunk whose row `lane` this thread holds
// in v: the rows go to shared memory first, then leave as whole rows (each
// store instruction covers several complete rows), instead of 32 scattered
// 16-byte pieces per instruction. `g` points at (the warp's first row, the
// chunk's first column); `ld` is the row stride in elements. A staging row of
// PITCH bytes holds up to (PITCH - 16) bytes of values; wider rows (fp32 output
// through a buffer sized for bf16) go out in two passes of 16 columns.
template <typename T, int PITCH>
__device__ __forceinline__ void warp_store_chunk(unsigned char* stg, const float (&v)[32], T* g, int64_t ld,
                                                 int lane) {
  constexpr int CPP = ((PITCH - 16) / static_cast<int>(sizeof(T))) < 32 ? 16 : 32;  // columns per pass
  constexpr int RB = CPP * static_cast<int>(sizeof(T));  // bytes of one row of a pass
  constexpr int LPR = RB / 16;                            // lanes per row on the way out
  constexpr int RPI = 32 / LPR;                           // rows per store instruction
  static_assert(RB + 16 <= PITCH || CPP == 16, "staging row");
  unsigned char* mine = stg + lane * PITCH;
#pragma unroll
  for (int p = 0; p < 32 / CPP; ++p) {
    if constexpr (std::is_same_v<T, float>) {
#pragma unroll
      for (int i = 0; i < CPP / 4; ++i)
        *reinterpret_cast<float4*>(mine + 16 * i) =
            make_float4(v[p * CPP + 4 * i], v[p * CPP + 4 * i + 1], v[p * CPP + 4 * i + 2], v[p * CPP + 4 * i + 3]);
    } else {
#pragma unroll
      for (int i = 0; i < CPP / 8; ++i) {
        const int b = p * CPP + 8 * i;
        uint4 w;
        w.x = pack_bf16x2(v[b], v[b + 1]);
        w.y = pack_bf16x2(v[b + 2], v[b + 3]);
        w.z = pack_bf16x2(v[b + 4], v[b + 5]);
        w.w = pack_bf16x2(v[b + 6], v[b + 7]);
        *reinterpret_cast<uint4*>(mine + 16 * i) = w;
      }
    }
    __syncwarp();
#pragma unroll
    for (int it = 0; it < 32 / RPI; ++it) {
      const int r = it * RPI + lane / LPR;
      const int seg = lane % LPR;
      const uint4 val = *reinterpret_cast<const uint4*>(stg + r * PITCH + seg * 16);
      *reinterpret_cast<uint4*>(reinterpret_cast<unsigned char*>(g + r * ld + p * CPP) + seg * 16) = val;
    }
    __syncwarp();
  }
}

// -------------------------------------------------------------- the kernel

template <class C>
__global__ void __launch_bounds__(C::THREADS, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmA32,
                        const __grid_constant__ CUtensorMap tmB,
                        const Args a) {
  using T = typename C::T;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  // 1024-byte alignment for the swizzle atoms
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  unsigned char* stage_base = smem;
  unsigned char* stg_base = smem + static_cast<size_t>(C::STAGES) * C::STAGE_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(stg_base + C::STG_BYTES);
  uint64_t* full = bars;
  uint64_t* empty = bars + C::STAGES;
  uint64_t* acc_full = bars + 2 * C::STAGES;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  int32_t* gs = reinterpret_cast<int32_t*>(stg_base + C::STG_BYTES + 1024);
  int32_t* off = gs + (kMaxExperts + 1);
  int32_t* ts = off + (kMaxExperts + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // prologue that reads nothing an earlier kernel writes, overlapping its tail
  pdl_trigger();
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < C::ACC_BUFS; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 32 * C::EPI_WARPS);
    }
    mbar_init(drain, 1);
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    if constexpr (!C::A_MN) tma_prefetch_desc(&tmA32);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, C::TMEM_COLS);
    tmem_relinquish();
  }
  __syncwarp();  // single-lane roles rejoin their warp before the block barrier
  pdl_wait();
  for (int i = threadIdx.x; i <= a.E; i += blockDim.x) {
    gs[i] = a.group_start[i];
    off[i] = (a.offsets != nullptr) ? a.offsets[i] : 0;
  }
  __syncthreads();
  if constexpr (C::G == Group::M) tile_starts<C>(a, gs, ts);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  const int n_tiles = total_tiles<C>(a, ts);

  if (warp == 0) {
    // ------------------------------------------------ TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;
      bool ok = true;
      for (int L = blockIdx.x; L < n_tiles && ok; L += gridDim.x) {
        const Tile t = decode_tile<C>(a, gs, off, ts, L);
        for (int kb = 0; kb < t.nk; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u)) {
            report(a.status, DEV_WAIT_TIMEOUT_PRODUCER);
            ok = false;
            break;
          }
          unsigned char* sa = stage_base + static_cast<size_t>(stage) * C::STAGE_BYTES;
          unsigned char* sb = sa + C::A_BYTES;
          // A operand, K-major: a 128-row box per half, or, for a half with at
          // most 96 valid rows, 32-row boxes covering only those (the rows past
          // them keep stale data; their accumulator rows are never stored).
          // MN-major: 128-byte column chunks of whole halves.
          if constexpr (!C::A_MN) {
            int a_bytes = 0;
            for (int hh = 0; hh < t.halves; ++hh) {
              const int vr = max(0, min(128, t.valid - hh * 128));
              a_bytes += (vr > 96) ? C::A_HALF : ((vr + 31) / 32) * (32 * 128);
            }
            mbar_arrive_expect_tx(&full[stage], a_bytes + C::B_BYTES);
            for (int hh = 0; hh < t.halves; ++hh) {
              const int vr = max(0, min(128, t.valid - hh * 128));
              if (vr > 96) {
                tma_load_2d(&tmA, &full[stage], sa + hh * C::A_HALF, kb * C::BK, t.m0 + hh * 128);
              } else {
                for (int q = 0; q < (vr + 31) / 32; ++q)
                  tma_load_2d(&tmA32, &full[stage], sa + hh * C::A_HALF + q * (32 * 128), kb * C::BK,
                              t.m0 + hh * 128 + 32 * q);
              }
            }
          } else {
            mbar_arrive_expect_tx(&full[stage], t.halves * C::A_HALF + C::B_BYTES);
            for (int ch = 0; ch < t.halves * (128 / C::CH); ++ch)
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
        const Tile t = decode_tile<C>(a, gs, off, ts, L);
        if (t.nk == 0) continue;  // the epilogue writes zeros without TMEM
        if (!mbar_wait(&acc_empty[acc], acc_phase ^ 1u)) {
          report(a.status, DEV_WAIT_TIMEOUT_MMA);
          break;
        }
        tc_fence_after();
        // accumulator of half hh of buffer acc: TMEM columns [(acc*H + hh) * BN, +BN)
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * C::H * C::BN);
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
            const uint64_t bd = C::B_MN ? smem_desc_sw128(sb + kk * C::UK * 128, C::BK * 128, 1024)
                                        : smem_desc_sw128(sb + kk * C::UK * C::ESZ, 16, 1024);
            const uint32_t accum = (kb > 0 || kk > 0) ? 1u : 0u;
            for (int hh = 0; hh < t.halves; ++hh) {
              const uint32_t sah = sa + hh * C::A_HALF;
              const uint64_t ad = C::A_MN ? smem_desc_sw128(sah + kk * C::UK * 128, C::BK * 128, 1024)
                                          : smem_desc_sw128(sah + kk * C::UK * C::ESZ, 16, 1024);
              if constexpr (C::TF32)
                umma_tf32(d_tmem + hh * C::BN, ad, bd, C::IDESC, accum);
              else
                umma_bf16(d_tmem + hh * C::BN, ad, bd, C::IDESC, accum);
            }
          }
          umma_commit(&empty[stage]);  // frees the smem slot once these MMAs finish
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit(&acc_full[acc]);
        if (++acc == C::ACC_BUFS) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
      // Drain: every MMA this thread issued has completed once `drain` flips.
      umma_commit(drain);
      if (!mbar_wait(drain, 0)) report(a.status, DEV_WAIT_TIMEOUT_DRAIN);
    }
  } else {
    // ------------------------------------------------ epilogue (warps 2 .. 2 + 4H)
    const int q = warp & 3;            // TMEM lane quarter this warp may access
    const int grp = (warp - 2) >> 2;   // 0 .. 2H-1
    const int hsel = grp >> 1;         // which 128-row half of the tile
    const int csel = grp & 1;          // which half of the tile's columns
    const int r_local = q * 32 + lane;
    int acc = 0;
    uint32_t acc_phase = 0;
    using OutT = typename C::OutT;
    OutT* out = static_cast<OutT*>(a.out);
    for (int L = blockIdx.x; L < n_tiles; L += gridDim.x) {
      const Tile t = decode_tile<C>(a, gs, off, ts, L);
      if (hsel >= t.halves) {  // this half lies past the expert's rows: nothing to store
        if (t.nk == 0) continue;
        if (!mbar_wait(&acc_full[acc], acc_phase)) {
          report(a.status, DEV_WAIT_TIMEOUT_EPILOGUE);
          break;
        }
        mbar_arrive(&acc_empty[acc]);
        if (++acc == C::ACC_BUFS) {
          acc = 0;
          acc_phase ^= 1u;
        }
        continue;
      }
      const bool row_ok = hsel * 128 + r_local < t.valid;
      const int64_t wrow0 = static_cast<int64_t>(t.m0) + hsel * 128 + q * 32;  // the warp's first row
      const int64_t row = wrow0 + lane;
      // this warp's share of the tile's output columns
      constexpr int WCOLS = C::OUT_N / 2;
      const int cw = csel * WCOLS;
      OutT* obase;  // (wrow0, n0 + cw)
      if constexpr (C::G == Group::M)
        obase = out + wrow0 * a.ld_out + t.n0 + cw;
      else
        obase = out + static_cast<int64_t>(t.e) * a.out_expert_stride + wrow0 * a.ld_out + t.n0 + cw;
      unsigned char* stg = stg_base + (warp - 2) * C::STG_WARP_BYTES;

      if (t.nk == 0) {  // K-grouped expert with no rows: its gradient is zero
        float z[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) z[i] = 0.f;
        for (int c = 0; c < WCOLS; c += 32) warp_store_chunk<OutT, C::STG_PITCH>(stg, z, obase + c, a.ld_out, lane);
        continue;
      }
      if (!mbar_wait(&acc_full[acc], acc_phase)) {
        report(a.status, DEV_WAIT_TIMEOUT_EPILOGUE);
        break;
      }
      tc_fence_after();
      const uint32_t tbase = tmem_base + static_cast<uint32_t>((acc * C::H + hsel) * C::BN + cw) +
                             (static_cast<uint32_t>(q * 32) << 16);

      if constexpr (C::EP == Epi::Store) {
#pragma unroll 1
        for (int c = 0; c < WCOLS; c += 32) {
          uint32_t r[32];
          tmem_ld32(tbase + c, r);
          tmem_ld_wait();
          float v[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = row_ok ? __uint_as_float(r[i]) : 0.f;
          warp_store_chunk<OutT, C::STG_PITCH>(stg, v, obase + c, a.ld_out, lane);
        }
      } else if constexpr (C::EP == Epi::SwigluFwd) {
        T* hbase = static_cast<T*>(a.out) + wrow0 * a.ld_out + t.n0 + cw;  // h has the operand type
        OutT* pbase = (a.out2 != nullptr) ? static_cast<OutT*>(a.out2) + wrow0 * a.ld_out2 + t.n0 + cw : nullptr;
#pragma unroll 1
        for (int c = 0; c < WCOLS; c += 32) {
          uint32_t rg[32], ru[32];
          tmem_ld32(tbase + c, rg);                // gate columns
          tmem_ld32(tbase + C::BN / 2 + c, ru);    // the matching up columns
          tmem_ld_wait();
          float hv[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float g = row_ok ? __uint_as_float(rg[i]) : 0.f;
            const float u = row_ok ? __uint_as_float(ru[i]) : 0.f;
            hv[i] = silu_fast(g) * u;
          }
          warp_store_chunk<T, C::STG_PITCH>(stg, hv, hbase + c, a.ld_out, lane);
          if (pbase != nullptr) {
            float g[32], u[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              g[i] = row_ok ? __uint_as_float(rg[i]) : 0.f;
              u[i] = row_ok ? __uint_as_float(ru[i]) : 0.f;
            }
            warp_store_chunk<OutT, C::STG_PITCH>(stg, g, pbase + c, a.ld_out2, lane);
            warp_store_chunk<OutT, C::STG_PITCH>(stg, u, pbase + a.f_half + c, a.ld_out2, lane);
          }
        }
      } else {  // SwigluBwd: accumulator holds dG for columns [n0, n0+BN); the
                // saved pre-activations are fp32
        const float* arow = static_cast<const float*>(a.aux) + row * a.ld_aux + t.n0 + cw;
#pragma unroll 1
        for (int c = 0; c < WCOLS; c += 32) {
          uint32_t r[32];
          tmem_ld32(tbase + c, r);
          tmem_ld_wait();
          float da[32], db[32];
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            if (row_ok) {
              float av[16], bv[16];
              load16<float>(arow + c + 16 * hh, av);
              load16<float>(arow + a.f_half + c + 16 * hh, bv);
#pragma unroll
              for (int i = 0; i < 16; ++i) {
                const float dg = __uint_as_float(r[16 * hh + i]);
                const float sg = __fdividef(1.0f, 1.0f + __expf(-av[i]));
                da[16 * hh + i] = dg * bv[i] * (sg * (1.0f + av[i] * (1.0f - sg)));
                db[16 * hh + i] = dg * av[i] * sg;
              }
            } else {
#pragma unroll
              for (int i = 0; i < 16; ++i) da[16 * hh + i] = db[16 * hh + i] = 0.f;
            }
          }
          warp_store_chunk<T, C::STG_PITCH>(stg, da, obase + c, a.ld_out, lane);
          warp_store_chunk<T, C::STG_PITCH>(stg, db, obase + a.f_half + c, a.ld_out, lane);
        }
      }
      tc_fence_before();
      mbar_arrive(&acc_empty[acc]);
      if (++acc == C::ACC_BUFS) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
  }

  __syncwarp();  // single-lane roles rejoin their warp before the block barrier
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}


// -------------------------------------------------------------- CTA-pair kernel
//
// The forward GEMMs (gate/up + SwiGLU, down) on pairs of CTAs (a cluster of
// two on the SMs of one TPC). A tile is 256 rows x 256 accumulator columns:
// each CTA loads its own 128 rows of A and 128 of the 256 B rows (gate/up: the
// leader the gate rows, the peer the matching up rows; down: the two column
// halves), and the leader issues cta_group::2 UMMAs (M = 256) that read both
// CTAs' shared memory and accumulate each CTA's 128 rows in its own TMEM. Per
// SM a 64-wide K step then moves 32 KB for the MMA work that costs 48 KB with
// one CTA per tile, so the same shared-memory ring keeps 1.5x the MMA work in
// flight. Barriers: TMA bytes of both CTAs land on the leader's `full`; the
// leader's commits arrive on `empty` and `acc_full` in both CTAs; both CTAs'
// epilogues arrive on the leader's `acc_empty`.
// O32: the store epilogue writes fp32 (the expert outputs kept for the
// backward), or the SwiGLU epilogue writes fp32 pre-activations.
template <Epi EP_, bool O32_ = false>
struct PairCfg {
  static constexpr Epi EP = EP_;
  static constexpr bool O32 = O32_;
  using OutT = std::conditional_t<O32, float, __nv_bfloat16>;  // store output / pre-activations
  static constexpr int BN = 256;                   // accumulator columns per tile
  static constexpr int BK = 64;                    // K per stage (one 128-byte swizzle row)
  static constexpr int UK = 16;                    // K per UMMA
  static constexpr int KSTEPS = BK / UK;
  static constexpr int A_BYTES = 128 * 128;        // this CTA's 128 rows of A
  static constexpr int A_TAIL_BYTES = 64 * 128;    // its 64 rows of A in a tail tile
  static constexpr int B_BYTES = 128 * 128;        // this CTA's 128 rows of B
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int ACC_BUFS = 2;
  static constexpr uint32_t IDESC = make_idesc(false, false, false, 256, BN);
  static constexpr uint32_t IDESC_TAIL = make_idesc(false, false, false, 128, BN);  // 64 rows per CTA
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr int EPI_WARPS = 8;
  static constexpr int THREADS = 64 + 32 * EPI_WARPS;
  static constexpr int STG_PITCH = 32 * 2 + 16;  // bf16-sized rows; fp32 output leaves in two passes
  static constexpr int STG_WARP_BYTES = 32 * STG_PITCH;
  static constexpr int STG_BYTES = EPI_WARPS * STG_WARP_BYTES;
  static constexpr int MISC_BYTES = 1024 + 3 * (kMaxExperts + 1) * static_cast<int>(sizeof(int32_t));
  static constexpr int STAGES = (227 * 1024 - 1024 - MISC_BYTES - STG_BYTES) / STAGE_BYTES;
  static constexpr int OUT_N = (EP == Epi::SwigluFwd) ? BN / 2 : BN;  // output columns per tile
  static constexpr size_t SMEM_BYTES =
      1024 + static_cast<size_t>(STAGES) * STAGE_BYTES + STG_BYTES + static_cast<size_t>(MISC_BYTES);
  static_assert(STAGES >= 4, "shared memory ring");
  static_assert(EP == Epi::SwigluFwd || EP == Epi::Store, "forward epilogues");
};

// A tile is 256 rows (128 per CTA, M = 256 MMAs), except an expert group's
// last tile when only 128 of its rows remain: that tail tile is 128 rows (64
// per CTA, M = 128 MMAs), so no MMA work is spent on the next group's rows.
// In an M = 128 pair MMA each CTA's accumulator holds its 64 rows twice over:
// TMEM lanes 0..63 carry output columns 0..127 and lanes 64..127 columns
// 128..255, both at TMEM columns 0..127 (lane 64 + r is row r again; checked
// on B200 by passing each row's and column's index through the MMA).
struct PairTile {
  int e, m0, n0;
  int tail;   // 1: a 128-row tail tile
  int valid;  // valid rows of this CTA's share (may be 0)
  int share;  // rows per CTA: 128, or 64 in a tail tile
};

// pts[e]: first pair tile of expert e; a group of R rows (R a multiple of 128)
// spans ceil(R / 256) pair tiles, the last one a tail tile when R / 128 is odd.
__device__ __forceinline__ void pair_tile_starts(int E, const int32_t* gs, int32_t* pts) {
  if (threadIdx.x == 0) {
    int acc = 0;
    for (int e = 0; e < E; ++e) {
      pts[e] = acc;
      acc += (gs[e + 1] - gs[e] + 255) / 256;
    }
    pts[E] = acc;
  }
}

template <class P>
__device__ __forceinline__ PairTile decode_pair_tile(const Args& a, const int32_t* gs, const int32_t* off,
                                                     const int32_t* pts, int L, uint32_t rank) {
  const int nN = a.N_total / P::OUT_N;
  const int mt = L / nN;
  const int nt = L - mt * nN;
  int lo = 0, hi = a.E - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (pts[mid] <= mt) lo = mid; else hi = mid - 1;
  }
  PairTile t;
  t.e = lo;
  t.m0 = gs[lo] + (mt - pts[lo]) * 256;
  t.n0 = nt * P::OUT_N;
  t.tail = (gs[lo + 1] - t.m0 == 128) ? 1 : 0;
  t.share = t.tail ? 64 : 128;
  const int my0 = t.m0 + t.share * static_cast<int>(rank);
  t.valid = max(0, min(t.share, gs[lo] + (off[lo + 1] - off[lo]) - my0));
  return t;
}

template <class P>
__global__ void __launch_bounds__(P::THREADS, 1)
    pair_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmA64,
                     const __grid_constant__ CUtensorMap tmB, const __grid_constant__ CUtensorMap tmB64,
                     const Args a) {
  using OutT = typename P::OutT;
  using HT = __nv_bfloat16;  // h, the SwiGLU output
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  unsigned char* stage_base = smem;
  unsigned char* stg_base = smem + static_cast<size_t>(P::STAGES) * P::STAGE_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(stg_base + P::STG_BYTES);
  uint64_t* full = bars;
  uint64_t* empty = bars + P::STAGES;
  uint64_t* acc_full = bars + 2 * P::STAGES;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  int32_t* gs = reinterpret_cast<int32_t*>(stg_base + P::STG_BYTES + 1024);
  int32_t* off = gs + (kMaxExperts + 1);
  int32_t* pts = off + (kMaxExperts + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int cluster = static_cast<int>(blockIdx.x >> 1);
  const int n_clusters = static_cast<int>(gridDim.x >> 1);

  pdl_trigger();
  if (threadIdx.x == 0) {
    for (int s = 0; s < P::STAGES; ++s) {
      mbar_init(&full[s], 1);   // the leader's expect_tx arrival (its copy is the one used)
      mbar_init(&empty[s], 1);  // one commit from the leader's MMA thread
    }
    for (int b = 0; b < P::ACC_BUFS; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 2 * P::EPI_WARPS);  // both CTAs' epilogue warps (the leader's copy)
    }
    mbar_init(drain, 1);
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmA64);
    tma_prefetch_desc(&tmB);
    tma_prefetch_desc(&tmB64);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_holder, P::TMEM_COLS);
    tmem_relinquish_pair();
  }
  __syncwarp();
  // the group layout comes from an earlier kernel
  pdl_wait();
  for (int i = threadIdx.x; i <= a.E; i += blockDim.x) {
    gs[i] = a.group_start[i];
    off[i] = a.offsets[i];
  }
  __syncthreads();
  pair_tile_starts(a.E, gs, pts);
  tc_fence_before();
  // both CTAs' barriers are initialised before either CTA's copies or commits
  // reach them (and the tile starts are visible to every warp)
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  const int n_tiles = pts[a.E] * (a.N_total / P::OUT_N);

  if (warp == 0) {
    // ------------------------------------------------ TMA producer (both CTAs)
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int L = cluster; L < n_tiles && ok; L += n_clusters) {
        const PairTile t = decode_pair_tile<P>(a, gs, off, pts, L, rank);
        const int arow = t.m0 + t.share * static_cast<int>(rank);
        // B rows: gate/up, full tile: the leader the 128 gate rows, the peer the
        // matching up rows; tail tile: each CTA 64 gate rows and the matching 64
        // up rows (so that a TMEM lane holds both halves of its outputs). Down:
        // each CTA one 128-row half of the output columns.
        int brow, brow2 = 0;
        if constexpr (P::EP == Epi::SwigluFwd) {
          if (t.tail) {
            brow = t.e * a.b_rows_per_expert + t.n0 + 64 * static_cast<int>(rank);
            brow2 = brow + a.f_half;
          } else {
            brow = t.e * a.b_rows_per_expert + t.n0 + (leader ? 0 : a.f_half);
          }
        } else {
          brow = t.e * a.b_rows_per_expert + t.n0 + 128 * static_cast<int>(rank);
        }
        for (int kb = 0; kb < a.K_total / P::BK; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u)) {
            report(a.status, DEV_WAIT_TIMEOUT_PRODUCER);
            ok = false;
            break;
          }
          unsigned char* sa = stage_base + static_cast<size_t>(stage) * P::STAGE_BYTES;
          if (leader)
            mbar_arrive_expect_tx(&full[stage], t.tail ? 2 * (P::A_TAIL_BYTES + P::B_BYTES) : 2 * P::STAGE_BYTES);
          tma_load_2d_pair(t.tail ? &tmA64 : &tmA, &full[stage], sa, kb * P::BK, arow);
          if (P::EP == Epi::SwigluFwd && t.tail) {
            tma_load_2d_pair(&tmB64, &full[stage], sa + P::A_BYTES, kb * P::BK, brow);
            tma_load_2d_pair(&tmB64, &full[stage], sa + P::A_BYTES + 64 * 128, kb * P::BK, brow2);
          } else {
            tma_load_2d_pair(&tmB, &full[stage], sa + P::A_BYTES, kb * P::BK, brow);
          }
          if (++stage == P::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer (leader only)
    if (leader && lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      const int nk = a.K_total / P::BK;
      for (int L = cluster; L < n_tiles && ok; L += n_clusters) {
        const uint32_t idesc = decode_pair_tile<P>(a, gs, off, pts, L, rank).tail ? P::IDESC_TAIL : P::IDESC;
        if (!mbar_wait(&acc_empty[acc], acc_phase ^ 1u)) {
          report(a.status, DEV_WAIT_TIMEOUT_MMA);
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * P::BN);
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(&full[stage], phase)) {
            report(a.status, DEV_WAIT_TIMEOUT_MMA);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(stage_base + static_cast<size_t>(stage) * P::STAGE_BYTES);
          const uint32_t sb = sa + P::A_BYTES;
#pragma unroll
          for (int kk = 0; kk < P::KSTEPS; ++kk)
            umma_bf16_pair(d_tmem, smem_desc_sw128(sa + kk * 32, 16, 1024), smem_desc_sw128(sb + kk * 32, 16, 1024),
                           idesc, (kb > 0 || kk > 0) ? 1u : 0u);
          umma_commit_pair(&empty[stage], 0x3);  // frees the slot in both CTAs
          if (++stage == P::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit_pair(&acc_full[acc], 0x3);
        if (++acc == P::ACC_BUFS) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
      umma_commit_pair(drain, 0x1);
      if (!mbar_wait(drain, 0)) report(a.status, DEV_WAIT_TIMEOUT_DRAIN);
      // both epilogues have released every accumulator they were handed, so no
      // remote arrival reaches this CTA after it exits
      for (int b = 0; b < P::ACC_BUFS; ++b) {
        // buffer b was handed out `uses` times; wait for the completion of its last phase
        const int tiles = (n_tiles > cluster) ? (n_tiles - 1 - cluster) / n_clusters + 1 : 0;
        const int uses = (tiles > b) ? (tiles - 1 - b) / P::ACC_BUFS + 1 : 0;
        if (uses > 0 && !mbar_wait(&acc_empty[b], static_cast<uint32_t>((uses - 1) & 1)))
          report(a.status, DEV_WAIT_TIMEOUT_DRAIN);
      }
    }
  } else {
    // ------------------------------------------------ epilogue (both CTAs)
    const int q = warp & 3;
    const int csel = (warp - 2) >> 2;  // which half of the warp's output columns
    const uint32_t acc_empty_leader0 = mapa_shared(smem_u32(&acc_empty[0]), 0);
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int L = cluster; L < n_tiles; L += n_clusters) {
      const PairTile t = decode_pair_tile<P>(a, gs, off, pts, L, rank);
      if (!__all_sync(0xffffffffu, mbar_wait(&acc_full[acc], acc_phase))) {  // warp-uniform
        report(a.status, DEV_WAIT_TIMEOUT_EPILOGUE);
        break;
      }
      tc_fence_after();
      {
        // this warp's 32 rows of the CTA's share, and the accumulator columns
        // its lane quadrant holds (a tail tile's quadrants 2 and 3 hold the
        // second half of the columns for the same rows as quadrants 0 and 1)
        const int rq = t.tail ? (q & 1) : q;
        const int half = t.tail ? (q >> 1) : 0;
        const bool row_ok = rq * 32 + lane < t.valid;
        const int64_t wrow0 = static_cast<int64_t>(t.m0) + t.share * static_cast<int>(rank) + rq * 32;
        unsigned char* stg = stg_base + (warp - 2) * P::STG_WARP_BYTES;
        const uint32_t tq = tmem_base + static_cast<uint32_t>(acc * P::BN) + (static_cast<uint32_t>(q * 32) << 16);
        if constexpr (P::EP == Epi::Store) {
          // output columns: full tile 128 per warp; tail tile 64 of its quadrant's half
          const int wc = t.tail ? 64 : 128;
          OutT* obase = static_cast<OutT*>(a.out) + wrow0 * a.ld_out + t.n0 + half * 128 + csel * wc;
          const uint32_t tbase = tq + static_cast<uint32_t>(csel * wc);
#pragma unroll 1
          for (int c = 0; c < wc; c += 32) {
            uint32_t r[32];
            tmem_ld32(tbase + c, r);
            tmem_ld_wait();
            float v[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = row_ok ? __uint_as_float(r[i]) : 0.f;
            warp_store_chunk<OutT, P::STG_PITCH>(stg, v, obase + c, a.ld_out, lane);
          }
        } else {
          // h columns: full tile 64 per warp (gate at accumulator column j, up at
          // 128 + j); tail tile 32 of its quadrant's 64 (gate at j, up at 64 + j)
          const int wc = t.tail ? 32 : 64;
          const int up_off = t.tail ? 64 : P::BN / 2;
          const int64_t ocol = t.n0 + half * 64 + csel * wc;
          HT* obase = static_cast<HT*>(a.out) + wrow0 * a.ld_out + ocol;
          OutT* pbase = (a.out2 != nullptr) ? static_cast<OutT*>(a.out2) + wrow0 * a.ld_out2 + ocol : nullptr;
          const uint32_t tbase = tq + static_cast<uint32_t>(csel * wc);
#pragma unroll 1
          for (int c = 0; c < wc; c += 32) {
            uint32_t rg[32], ru[32];
            tmem_ld32(tbase + c, rg);
            tmem_ld32(tbase + up_off + c, ru);
            tmem_ld_wait();
            float hv[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const float g = row_ok ? __uint_as_float(rg[i]) : 0.f;
              const float u = row_ok ? __uint_as_float(ru[i]) : 0.f;
              hv[i] = silu_fast(g) * u;
            }
            warp_store_chunk<HT, P::STG_PITCH>(stg, hv, obase + c, a.ld_out, lane);
            if (pbase != nullptr) {  // the pre-activations, kept for the backward
              float g[32], u[32];
#pragma unroll
              for (int i = 0; i < 32; ++i) {
                g[i] = row_ok ? __uint_as_float(rg[i]) : 0.f;
                u[i] = row_ok ? __uint_as_float(ru[i]) : 0.f;
              }
              warp_store_chunk<OutT, P::STG_PITCH>(stg, g, pbase + c, a.ld_out2, lane);
              warp_store_chunk<OutT, P::STG_PITCH>(stg, u, pbase + a.f_half + c, a.ld_out2, lane);
            }
          }
        }
      }
      // the warp's TMEM reads are complete (wait::ld) and fenced; one arrive per
      // warp releases the accumulator to the leader's MMA issuer (nothing in
      // this kernel reads the stored rows, so no global ordering is needed)
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(acc_empty_leader0 + static_cast<uint32_t>(acc * sizeof(uint64_t)));
      if (++acc == P::ACC_BUFS) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
  }

  __syncwarp();  // single-lane roles rejoin their warp before the block barrier
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, P::TMEM_COLS);
  }
}

// -------------------------------------------------------------- host side

}  // namespace

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

namespace {

template <class C>
cudaError_t launch(const CUtensorMap& ta, const CUtensorMap& ta32, const CUtensorMap& tb, const Args& a,
                   int max_tiles, cudaStream_t st) {
  static std::atomic<size_t> smem_set[kMaxDevices];
  cudaError_t e = raise_smem_limit(reinterpret_cast<const void*>(grouped_gemm_kernel<C>), C::SMEM_BYTES, smem_set);
  if (e != cudaSuccess) return e;
  int grid = device_sm_count();
  if (max_tiles < grid) grid = max_tiles;
  if (grid <= 0) return cudaSuccess;
  return launch_dependent(grouped_gemm_kernel<C>, dim3(grid), dim3(C::THREADS), C::SMEM_BYTES, st, nullptr, 0, ta,
                          ta32, tb, a);
}

template <class P>
cudaError_t launch_pair(const CUtensorMap& ta, const CUtensorMap& ta64, const CUtensorMap& tb,
                        const CUtensorMap& tb64, const Args& a, int max_pair_tiles, cudaStream_t st) {
  static std::atomic<size_t> smem_set[kMaxDevices];
  cudaError_t e = raise_smem_limit(reinterpret_cast<const void*>(pair_gemm_kernel<P>), P::SMEM_BYTES, smem_set);
  if (e != cudaSuccess) return e;
  int clusters = device_sm_count() / 2;
  if (max_pair_tiles < clusters) clusters = max_pair_tiles;
  if (clusters <= 0) return cudaSuccess;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  return launch_dependent(pair_gemm_kernel<P>, dim3(static_cast<unsigned>(2 * clusters)), dim3(P::THREADS),
                          P::SMEM_BYTES, st, attr, 1, ta, ta64, tb, tb64, a);
}

// Pair tiles of 256 rows are used when the groups are large: a group of R rows
// costs ceil(R / 256) pair tiles, so groups of a few hundred rows would waste
// much of the MMA work; from 384 routed rows per expert on average they pay.
bool use_pairs(const Shape& s) { return !s.fp32 && s.T * s.k >= 384 * static_cast<int64_t>(s.E); }

Args base_args(const Shape& s, const int32_t* gs, const int32_t* off, int32_t* status) {
  Args a{};
  a.group_start = gs;
  a.offsets = off;
  a.E = s.E;
  a.status = status;
  return a;
}

int ch_elems(bool fp32) { return fp32 ? 32 : 64; }

// Instantiates the kernel for the dtype, tile N and tile M (h 128-row halves).
template <bool A_MN, bool B_MN, Group G, Epi EP, bool O32 = false>
cudaError_t run_variant(bool fp32, int bn, int h, const CUtensorMap& ta, const CUtensorMap& ta32,
                        const CUtensorMap& tb, const Args& a, int max_tiles, cudaStream_t st) {
  if (fp32) {
    if (bn == 256) return launch<Cfg<true, A_MN, B_MN, G, EP, 256, 1>>(ta, ta32, tb, a, max_tiles, st);
    return launch<Cfg<true, A_MN, B_MN, G, EP, 128, 1>>(ta, ta32, tb, a, max_tiles, st);
  }
  (void)h;
  if (bn == 256) return launch<Cfg<false, A_MN, B_MN, G, EP, 256, 1, O32>>(ta, ta32, tb, a, max_tiles, st);
  return launch<Cfg<false, A_MN, B_MN, G, EP, 128, 1, O32>>(ta, ta32, tb, a, max_tiles, st);
}

// Tile M. 256-row tiles (H = 2) halve the operand bytes per MMA cycle, but two
// 128 x 256 fp32 accumulators fill TMEM, so the epilogue of a tile cannot
// overlap the next tile's MMAs, and 16 epilogue warps cap the registers at 96;
// on B200 the gate/up GEMM at T = 4096 took 333 us with them against 235 us
// with 128-row tiles and double-buffered accumulators, so 128-row tiles are used.
int pick_h(const Shape&) { return 1; }

}  // namespace

// Tile N for a forward GEMM whose accumulator covers `n` columns per expert.
static int pick_bn(int n) { return (n % 256 == 0) ? 256 : 128; }

// Few routed rows (decode): at most min(T*k, E) expert groups of one or two
// 128-row tiles. When 256-column tiles would leave SMs idle, 128-column tiles
// double the number of CTAs streaming the experts' weights.
static bool few_tiles(const Shape& s, int n_cols) {
  const int64_t groups = (s.T * s.k < s.E) ? s.T * s.k : s.E;
  const int64_t m_tiles = groups + (s.T * s.k) / 128;
  return m_tiles * (n_cols / 256) < device_sm_count();
}

cudaError_t launch_gate_up(const Shape& s, const void* x_perm, const int32_t* group_start,
                           const int32_t* offsets, const void* w_gate_up, void* h, void* preact, int32_t* status,
                           cudaStream_t st) {
  if (use_pairs(s)) {
    CUtensorMap ta, ta64, tb, tb64;
    if (!make_map(&ta, x_perm, false, s.P, s.d, 64, 128)) return cudaErrorInvalidValue;
    if (!make_map(&ta64, x_perm, false, s.P, s.d, 64, 64)) return cudaErrorInvalidValue;
    if (!make_map(&tb, w_gate_up, false, static_cast<uint64_t>(s.E) * 2 * s.f, s.d, 64, 128))
      return cudaErrorInvalidValue;
    if (!make_map(&tb64, w_gate_up, false, static_cast<uint64_t>(s.E) * 2 * s.f, s.d, 64, 64))
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
    const int max_pairs = static_cast<int>((s.P / 256 + s.E) * (s.f / 128));
    if (preact != nullptr) return launch_pair<PairCfg<Epi::SwigluFwd, true>>(ta, ta64, tb, tb64, a, max_pairs, st);
    return launch_pair<PairCfg<Epi::SwigluFwd>>(ta, ta64, tb, tb64, a, max_pairs, st);
  }
  // accumulator: BN/2 gate columns and BN/2 up columns of the same outputs
  const int bn = few_tiles(s, 2 * s.f) ? 128 : 256;
  const int kcols = ch_elems(s.fp32);
  CUtensorMap ta, ta32, tb;
  if (!make_map(&ta, x_perm, s.fp32, s.P, s.d, kcols, 128)) return cudaErrorInvalidValue;
  if (!make_map(&ta32, x_perm, s.fp32, s.P, s.d, kcols, 32)) return cudaErrorInvalidValue;
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
  if (preact != nullptr)  // pre-activations kept in fp32 for the backward
    return run_variant<false, false, Group::M, Epi::SwigluFwd, true>(s.fp32, bn, pick_h(s), ta, ta32, tb, a, max_tiles,
                                                                     st);
  return run_variant<false, false, Group::M, Epi::SwigluFwd>(s.fp32, bn, pick_h(s), ta, ta32, tb, a, max_tiles, st);
}

cudaError_t launch_down(const Shape& s, const void* h, const int32_t* group_start, const int32_t* offsets,
                        const void* w_down, void* o_perm, bool out32, int32_t* status, cudaStream_t st) {
  if (use_pairs(s) && s.d % 256 == 0) {
    CUtensorMap ta, ta64, tb;
    if (!make_map(&ta, h, false, s.P, s.f, 64, 128)) return cudaErrorInvalidValue;
    if (!make_map(&ta64, h, false, s.P, s.f, 64, 64)) return cudaErrorInvalidValue;
    if (!make_map(&tb, w_down, false, static_cast<uint64_t>(s.E) * s.d, s.f, 64, 128)) return cudaErrorInvalidValue;
    Args a = base_args(s, group_start, offsets, status);
    a.N_total = s.d;
    a.K_total = s.f;
    a.b_rows_per_expert = s.d;
    a.out = o_perm;
    a.ld_out = s.d;
    const int max_pairs = static_cast<int>((s.P / 256 + s.E) * (s.d / 256));
    if (out32) return launch_pair<PairCfg<Epi::Store, true>>(ta, ta64, tb, tb, a, max_pairs, st);
    return launch_pair<PairCfg<Epi::Store>>(ta, ta64, tb, tb, a, max_pairs, st);
  }
  const int bn = few_tiles(s, s.d) ? 128 : pick_bn(s.d);
  const int kcols = ch_elems(s.fp32);
  CUtensorMap ta, ta32, tb;
  if (!make_map(&ta, h, s.fp32, s.P, s.f, kcols, 128)) return cudaErrorInvalidValue;
  if (!make_map(&ta32, h, s.fp32, s.P, s.f, kcols, 32)) return cudaErrorInvalidValue;
  if (!make_map(&tb, w_down, s.fp32, static_cast<uint64_t>(s.E) * s.d, s.f, kcols, bn))
    return cudaErrorInvalidValue;
  Args a = base_args(s, group_start, offsets, status);
  a.N_total = s.d;
  a.K_total = s.f;
  a.b_rows_per_expert = s.d;
  a.out = o_perm;
  a.ld_out = s.d;
  const int max_tiles = static_cast<int>((s.P / 128) * (s.d / bn));
  if (out32)
    return run_variant<false, false, Group::M, Epi::Store, true>(s.fp32, bn, pick_h(s), ta, ta32, tb, a, max_tiles, st);
  return run_variant<false, false, Group::M, Epi::Store>(s.fp32, bn, pick_h(s), ta, ta32, tb, a, max_tiles, st);
}

// dG = dO W_down (K = d, B read MN-major from W_down [E*d, f]); epilogue forms
// dA = dG * b * silu'(a), dB = dG * silu(a) from the saved pre-activations.
cudaError_t launch_down_backward_data(const Shape& s, const void* dout, const int32_t* group_start,
                                      const int32_t* offsets, const void* w_down, const void* preact, void* dab,
                                      int32_t* status, cudaStream_t st) {
  const int bn = pick_bn(s.f);
  const int kc = ch_elems(s.fp32);
  const int bk = s.fp32 ? 32 : 64;
  CUtensorMap ta, ta32, tb;
  if (!make_map(&ta, dout, s.fp32, s.P, s.d, kc, 128)) return cudaErrorInvalidValue;
  if (!make_map(&ta32, dout, s.fp32, s.P, s.d, kc, 32)) return cudaErrorInvalidValue;
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
  return run_variant<false, true, Group::M, Epi::SwigluBwd>(s.fp32, bn, pick_h(s), ta, ta32, tb, a, max_tiles, st);
}

// dX_perm = [dA|dB] W_gate_up (K = 2f, B read MN-major from W_gate_up [E*2f, d]).
cudaError_t launch_gate_up_backward_data(const Shape& s, const void* dab, const int32_t* group_start,
                                         const int32_t* offsets, const void* w_gate_up, void* dx_perm,
                                         int32_t* status, cudaStream_t st) {
  const int bn = pick_bn(s.d);
  const int kc = ch_elems(s.fp32);
  const int bk = s.fp32 ? 32 : 64;
  CUtensorMap ta, ta32, tb;
  if (!make_map(&ta, dab, s.fp32, s.P, 2 * s.f, kc, 128)) return cudaErrorInvalidValue;
  if (!make_map(&ta32, dab, s.fp32, s.P, 2 * s.f, kc, 32)) return cudaErrorInvalidValue;
  if (!make_map(&tb, w_gate_up, s.fp32, static_cast<uint64_t>(s.E) * 2 * s.f, s.d, kc, bk))
    return cudaErrorInvalidValue;
  Args a = base_args(s, group_start, offsets, status);
  a.N_total = s.d;
  a.K_total = 2 * s.f;
  a.b_rows_per_expert = 2 * s.f;
  a.out = dx_perm;
  a.ld_out = s.d;
  const int max_tiles = static_cast<int>((s.P / 128) * (s.d / bn));
  return run_variant<false, true, Group::M, Epi::Store>(s.fp32, bn, pick_h(s), ta, ta32, tb, a, max_tiles, st);
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
  const CUtensorMap& ta32 = ta;  // MN-major A: whole halves only
  if (!make_map(&tb, B, s.fp32, s.P, N_total, kc, bk)) return cudaErrorInvalidValue;
  Args a = base_args(s, gs, off, status);
  a.M_total = M_total;
  a.N_total = N_total;
  a.out = out;
  a.ld_out = N_total;
  a.out_expert_stride = static_cast<int64_t>(M_total) * N_total;
  const int h = pick_h(s);
  const int max_tiles = s.E * (M_total / (128 * h)) * (N_total / bn);
  if (s.grad32 && !s.fp32)
    return run_variant<true, true, Group::K, Epi::Store, true>(s.fp32, bn, h, ta, ta32, tb, a, max_tiles, st);
  return run_variant<true, true, Group::K, Epi::Store>(s.fp32, bn, h, ta, ta32, tb, a, max_tiles, st);
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
