// sgemm.cu -- the two GEMMs of the router backward on the tensor cores, with
// FP32-level accuracy from exact bf16 splits of their FP32 operands.
//
// Passage: dots.llm1 Technical Report, §Architecture "Mixture of Experts layer"
// (the gate is computed in FP32); the gradients are those of logit = X Wg^T:
//   GDX  dX[t, c] += sum_e dlogit[t, e] Wg[e, c]      (M = tokens, N = d, K = E)
//   GDW  dWg[e, c]  = sum_t dlogit[t, e] X[t, c]      (M = E,      N = d, K = T)
// dlogit (FP32) and Wg (FP32) are each split exactly into three bf16 planes,
// v = hi + mid + lo; X is bf16 already.  A product of two bf16 values is exact in
// FP32, so each GEMM is a sum of plane products:
//   GDX  the six pairs (hi,hi) (hi,mid) (mid,hi) (hi,lo) (lo,hi) (mid,mid); the
//        three dropped pairs are below 2^-24 of the result's terms
//   GDW  the three planes of dlogit against X
// Both are written as ONE GEMM over a stacked K: K block kb names a plane pair
// and a 64-wide slice of the real K, and every K block is a plain bf16 MMA
// into the same FP32 accumulator.  GDW splits the stacked K across CTAs (the
// real K = T is long and its output small); the partial sums go to the
// workspace and a second kernel adds them in a fixed order.
//
// One CTA per SM, persistent over work items (128 x 256 output tiles, and for
// GDW also K splits):
//   warp 0        TMA producer, 4-stage ring of 48 KB (A 16 KB + B 32 KB)
//   warp 1        tensor-memory owner; lane 0 issues tcgen05.mma (M = 128,
//                 N = 256, K = 16) into one of two 256-column accumulators
//   warps 2..9    epilogue, two per tensor-memory lane quarter (column halves):
//                 GDX adds the tile into dX (bf16 read-modify-write), GDW stores
//                 the FP32 partial
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "moe_internal.cuh"
#include "sm100.cuh"

namespace moe {
namespace {

constexpr int SG_BM = 128;
constexpr int SG_BN = 256;
constexpr int SG_BK = 64;
constexpr int SG_STAGES = 4;
constexpr int SG_A_BYTES = SG_BM * SG_BK * 2;  // 16 KB
constexpr int SG_B_BYTES = SG_BN * SG_BK * 2;  // 32 KB
constexpr int SG_STAGE_BYTES = SG_A_BYTES + SG_B_BYTES;
constexpr int SG_EPI_WARPS = 8;
constexpr int SG_THREADS = 64 + 32 * SG_EPI_WARPS;
constexpr uint32_t SG_TMEM_COLS = 512;  // two 256-column FP32 accumulators

enum { SG_GDX = 0, SG_GDW = 1 };

// GDX plane pairs (dlogit plane, Wg plane) of the stacked K.
__constant__ int kPairA[6] = {0, 0, 1, 0, 2, 1};
__constant__ int kPairB[6] = {0, 1, 0, 2, 0, 1};

struct SgArgs {
  int* status;
  int64_t T;
  int t_pad, d, e_pad;
  int n_tiles, items;
  int kb_total;      // stacked K blocks of one output tile
  int kb_per_split;  // GDW: K blocks per split
  int splits;        // GDW
  int kbE;           // GDX: 64-wide K blocks per plane pair (ceil(e_pad / 64))
  int kb_plane;      // GDW: K blocks per dlogit plane (t_pad / 64)
  void* out;         // GDX: dX bf16 [T, d]; GDW: partial f32 [splits][e_pad][d]
  uint32_t idesc;
  uint64_t budget_ns;
};

struct SgCtl {
  uint64_t full[SG_STAGES];
  uint64_t empty[SG_STAGES];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};

struct Item {
  int m0, n0, kb0, kb1, split;
};

// GDX: tiles in m-major order, n inside (the pairs of CTAs running together share
// the A rows of 128 tokens).  GDW: (tile, split) with the splits of a tile adjacent.
template <int MODE>
__device__ __forceinline__ Item decode_item(int it, const SgArgs& a) {
  Item r;
  if constexpr (MODE == SG_GDX) {
    const int mt = it / a.n_tiles, nt = it - mt * a.n_tiles;
    r.m0 = mt * SG_BM;
    r.n0 = nt * SG_BN;
    r.kb0 = 0;
    r.kb1 = a.kb_total;
    r.split = 0;
  } else {
    const int tile = it / a.splits, sp = it - tile * a.splits;
    const int mt = tile / a.n_tiles, nt = tile - mt * a.n_tiles;
    r.m0 = mt * SG_BM;
    r.n0 = nt * SG_BN;
    r.split = sp;
    r.kb0 = sp * a.kb_per_split;
    r.kb1 = min(a.kb_total, r.kb0 + a.kb_per_split);
  }
  return r;
}

__device__ __forceinline__ uint32_t pack2_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

template <int MODE>
__global__ void __launch_bounds__(SG_THREADS, 1)
    sgemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                 const SgArgs a) {
  constexpr bool A_MN = (MODE == SG_GDW);
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  SgCtl* ctl = reinterpret_cast<SgCtl*>(smem + SG_STAGES * SG_STAGE_BYTES);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile int* abort_flag = &ctl->abort_flag;

  if (threadIdx.x == 0) {
    for (int s = 0; s < SG_STAGES; ++s) {
      mbar_init(&ctl->full[s], 1);
      mbar_init(&ctl->empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&ctl->tfull[b], 1);
      mbar_init(&ctl->tempty[b], SG_EPI_WARPS);
    }
    mbar_init(&ctl->drain, 1);
    ctl->abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(&ctl->tmem_base, SG_TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = ctl->tmem_base;
  const uint64_t drain_budget = a.budget_ns > 2000000000ull ? a.budget_ns : 2000000000ull;

  if (warp == 0) {
    // ------------------------------------------------------------ producer --
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0, issued = 0, lastpar = 0;
      bool ok = true;
      for (int it = blockIdx.x; ok && it < a.items; it += gridDim.x) {
        const Item w = decode_item<MODE>(it, a);
        for (int kb = w.kb0; kb < w.kb1; ++kb) {
          if (!mbar_wait(&ctl->empty[stage], phase ^ 1, abort_flag, a.status,
                         MOE_ERR_DEVICE_TIMEOUT, a.budget_ns)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&ctl->full[stage], SG_STAGE_BYTES);
          uint8_t* a_dst = smem + stage * SG_STAGE_BYTES;
          uint8_t* b_dst = a_dst + SG_A_BYTES;
          if constexpr (MODE == SG_GDX) {
            // A: 128 token rows of dlogit plane pa, K columns e0..e0+63 (K-major);
            // B: rows e0..e0+63 of Wg plane pb, 256 columns of d (N-major)
            const int p = kb / a.kbE, e0 = (kb - p * a.kbE) * SG_BK;
            tma_load_2d(a_dst, &tmA, &ctl->full[stage], e0, kPairA[p] * a.t_pad + w.m0);
#pragma unroll
            for (int c = 0; c < 4; ++c)
              tma_load_2d(b_dst + c * 8192, &tmB, &ctl->full[stage], w.n0 + c * 64,
                          kPairB[p] * a.e_pad + e0);
          } else {
            // A: token rows t0..t0+63 of dlogit plane pl, 128 expert columns (M-major);
            // B: the same token rows of X, 256 columns of d (N-major)
            const int pl = kb / a.kb_plane, t0 = (kb - pl * a.kb_plane) * SG_BK;
#pragma unroll
            for (int c = 0; c < 2; ++c)
              tma_load_2d(a_dst + c * 8192, &tmA, &ctl->full[stage], w.m0 + c * 64,
                          pl * a.t_pad + t0);
#pragma unroll
            for (int c = 0; c < 4; ++c)
              tma_load_2d(b_dst + c * 8192, &tmB, &ctl->full[stage], w.n0 + c * 64, t0);
          }
          issued |= 1u << stage;
          lastpar = (lastpar & ~(1u << stage)) | (phase << stage);
          if (++stage == SG_STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      // after an abort, stages may hold copies nobody consumed: let them land
      if (*abort_flag)
        for (int s = 0; s < SG_STAGES; ++s)
          if (issued & (1u << s)) {
            volatile int never = 0;
            mbar_wait(&ctl->full[s], (lastpar >> s) & 1u, &never, a.status,
                      MOE_ERR_DEVICE_TIMEOUT, drain_budget);
          }
    }
  } else if (warp == 1) {
    // --------------------------------------------------------- MMA issuer --
    if (lane == 0) {
      int stage = 0, n = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int it = blockIdx.x; ok && it < a.items; it += gridDim.x, ++n) {
        const Item w = decode_item<MODE>(it, a);
        const int acc = n & 1;
        const uint32_t use = (uint32_t)(n >> 1);
        if (!mbar_wait(&ctl->tempty[acc], (use & 1u) ^ 1u, abort_flag, a.status,
                       MOE_ERR_DEVICE_TIMEOUT, a.budget_ns))
          break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * SG_BN);
        for (int kb = w.kb0; kb < w.kb1; ++kb) {
          if (!mbar_wait(&ctl->full[stage], phase, abort_flag, a.status, MOE_ERR_DEVICE_TIMEOUT,
                         a.budget_ns)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_base = smem_u32(smem + stage * SG_STAGE_BYTES);
          const uint32_t b_base = a_base + SG_A_BYTES;
#pragma unroll
          for (int kk = 0; kk < SG_BK / 16; ++kk) {
            const uint64_t ad = A_MN ? smem_desc_sw128(a_base + kk * 2048, 8192, 1024)
                                     : smem_desc_sw128(a_base + kk * 32, 16, 1024);
            const uint64_t bd = smem_desc_sw128(b_base + kk * 2048, 8192, 1024);
            umma_f16(d_tmem, ad, bd, a.idesc, (kb > w.kb0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(&ctl->empty[stage]);
          if (++stage == SG_STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        umma_commit(&ctl->tfull[acc]);
      }
      // every MMA issued has completed before tensor memory is freed
      umma_commit(&ctl->drain);
      volatile int never = 0;
      mbar_wait(&ctl->drain, 0, &never, a.status, MOE_ERR_DEVICE_TIMEOUT, drain_budget);
    }
  } else {
    // ------------------------------------------------------------ epilogue --
    const int q = warp & 3;         // tensor-memory lane quarter
    const int h = (warp - 2) >> 2;  // column half
    const int row = q * 32 + lane;
    int n = 0;
    for (int it = blockIdx.x; it < a.items; it += gridDim.x, ++n) {
      const Item w = decode_item<MODE>(it, a);
      const int acc = n & 1;
      const uint32_t use = (uint32_t)(n >> 1);
      if (!mbar_wait(&ctl->tfull[acc], use & 1u, abort_flag, a.status, MOE_ERR_DEVICE_TIMEOUT,
                     a.budget_ns))
        break;
      __syncwarp();  // tcgen05.ld is warp-collective
      tc_fence_after();
      const uint32_t taddr = tmem_base + (uint32_t)(acc * SG_BN) + ((uint32_t)(q * 32) << 16);
#pragma unroll 1
      for (int cc = 0; cc < 4; ++cc) {
        const int col = h * 128 + cc * 32;
        uint32_t r[32];
        tmem_ld32_sync(taddr + (uint32_t)col, r);
        const int c = w.n0 + col;  // d % 64 == 0: a 32-column chunk is all in or all out
        if (c >= a.d) continue;
        if constexpr (MODE == SG_GDX) {
          const int64_t t = (int64_t)w.m0 + row;
          if (t < a.T) {
            uint4* p = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(a.out) +
                                                t * a.d + c);
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              uint4 o = p[v];
              uint32_t u[4] = {o.x, o.y, o.z, o.w};
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                const float lo = __uint_as_float(u[j] << 16) + __uint_as_float(r[8 * v + 2 * j]);
                const float hi =
                    __uint_as_float(u[j] & 0xFFFF0000u) + __uint_as_float(r[8 * v + 2 * j + 1]);
                u[j] = pack2_bf16(lo, hi);
              }
              p[v] = make_uint4(u[0], u[1], u[2], u[3]);
            }
          }
        } else {
          const int e = w.m0 + row;
          if (e < a.e_pad) {
            float4* p = reinterpret_cast<float4*>(reinterpret_cast<float*>(a.out) +
                                                  ((int64_t)w.split * a.e_pad + e) * a.d + c);
#pragma unroll
            for (int v = 0; v < 8; ++v)
              p[v] = make_float4(__uint_as_float(r[4 * v]), __uint_as_float(r[4 * v + 1]),
                                 __uint_as_float(r[4 * v + 2]), __uint_as_float(r[4 * v + 3]));
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl->tempty[acc]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, SG_TMEM_COLS);
  }
}

}  // namespace

namespace {

template <int MODE>
int launch_sg(const CUtensorMap& ma, const CUtensorMap& mb, const SgArgs& a, cudaStream_t st) {
  constexpr size_t kSmem = 1024 + SG_STAGES * SG_STAGE_BYTES + sizeof(SgCtl);
  static_assert(kSmem <= 232448, "shared memory per CTA exceeds 227 KB");
  static int num_sms = 0;
  if (num_sms == 0) {
    if (!cuda_ok(cudaFuncSetAttribute(sgemm_kernel<MODE>,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmem)))
      return MOE_ERR_CUDA;
    int dev = 0, n = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    num_sms = n > 0 ? n : 148;
  }
  const int grid = a.items < num_sms ? a.items : num_sms;
  sgemm_kernel<MODE><<<grid, SG_THREADS, kSmem, st>>>(ma, mb, a);
  return cuda_ok(cudaGetLastError()) ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace

int launch_gate_dx(const moe_dims& dm, const void* dl_planes, const void* wg_planes, void* dx,
                   int* status, void* stream) {
  if (dm.T == 0) return MOE_OK;
  const WsLayout L = ws_layout(dm);
  SgArgs a{};
  a.status = status;
  a.T = dm.T;
  a.t_pad = L.t_pad;
  a.d = dm.d;
  a.e_pad = L.e_pad;
  a.n_tiles = (dm.d + SG_BN - 1) / SG_BN;
  a.items = (L.t_pad / SG_BM) * a.n_tiles;
  a.kbE = (L.e_pad + SG_BK - 1) / SG_BK;
  a.kb_total = 6 * a.kbE;
  a.out = dx;
  a.idesc = idesc_bf16_f32(SG_BM, SG_BN, false, true);
  a.budget_ns = wait_budget_ns();
  CUtensorMap ma{}, mb{};
  if (!make_map_bf16(&ma, dl_planes, (int64_t)3 * L.t_pad, L.e_pad, SG_BM) ||
      !make_map_bf16(&mb, wg_planes, (int64_t)3 * L.e_pad, dm.d, 64))
    return MOE_ERR_CUDA;
  return launch_sg<SG_GDX>(ma, mb, a, reinterpret_cast<cudaStream_t>(stream));
}

int launch_gate_dw(const moe_dims& dm, const void* dl_planes, const void* x, float* partial,
                   int* status, void* stream) {
  if (dm.T == 0) return MOE_OK;
  const WsLayout L = ws_layout(dm);
  SgArgs a{};
  a.status = status;
  a.T = dm.T;
  a.t_pad = L.t_pad;
  a.d = dm.d;
  a.e_pad = L.e_pad;
  a.n_tiles = (dm.d + SG_BN - 1) / SG_BN;
  a.kb_plane = L.t_pad / SG_BK;
  a.kb_total = 3 * a.kb_plane;
  a.splits = L.gdw_splits;
  a.kb_per_split = (a.kb_total + a.splits - 1) / a.splits;
  a.items = ((L.e_pad + SG_BM - 1) / SG_BM) * a.n_tiles * a.splits;
  a.out = partial;
  a.idesc = idesc_bf16_f32(SG_BM, SG_BN, true, true);
  a.budget_ns = wait_budget_ns();
  CUtensorMap ma{}, mb{};
  if (!make_map_bf16(&ma, dl_planes, (int64_t)3 * L.t_pad, L.e_pad, 64) ||
      !make_map_bf16(&mb, x, dm.T, dm.d, 64))
    return MOE_ERR_CUDA;
  return launch_sg<SG_GDW>(ma, mb, a, reinterpret_cast<cudaStream_t>(stream));
}

}  // namespace moe
