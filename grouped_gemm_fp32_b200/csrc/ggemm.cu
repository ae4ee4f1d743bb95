// ggemm.cu -- persistent grouped GEMM on the 5th-generation tensor cores
// (tcgen05.mma, accumulators in tensor memory, operands staged by TMA).
//
// Passage: dots.llm1 Technical Report, §3.2 "Efficient implementation of
// Grouped GEMM".  Every expert's token segment is padded to a fixed block, so
// a 128-row tile never straddles two experts and scheduling reduces to that of
// a plain GEMM: tiles are (group, m-tile, n-tile) triples enumerated from a
// per-group prefix of m-tile counts that is built on the device (no host
// round trip).  The pages' version targets sm_90 warpgroup MMA; this one is
// written for sm_100a: one CTA per SM walks tiles persistently,
//   warp 0        TMA producer (4-stage shared-memory ring, 48 KB a stage)
//   warp 1        tensor-memory owner and single-thread tcgen05.mma issuer
//   warps 2..5    epilogue: tcgen05.ld of the FP32 accumulator, fused
//                 SwiGLU / SwiGLU-backward / bf16 or f32 store
// with two 128x256 FP32 accumulators in tensor memory so the epilogue of one
// tile overlaps the MMAs of the next.
//
// Six GEMMs of the expert FFN share this kernel (A is M x K, B is N x K):
//   FWD1  A = x rows (K-major)     B = W1 gate|up rows (K-major)  -> SwiGLU -> H (+ A1)
//   FWD2  A = H rows (K-major)     B = W2 rows (K-major)          -> Y
//   DX2   A = dY rows (K-major)    B = W2 as [d, I] (N-major)     -> SwiGLU bwd -> dA
//   DX1   A = dA rows (K-major)    B = W1 as [2I, d] (N-major)    -> dX rows
//   DW2   A = dY^T (M-major)       B = H^T (N-major), K = group rows -> dW2 f32
//   DW1   A = dA^T (M-major)       B = x^T (N-major), K = group rows -> dW1 f32
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdio>
#include <mutex>

#include "moe_internal.cuh"
#include "sm100.cuh"

namespace moe {

namespace {

constexpr int BM = 128;           // UMMA M (rows of A per tile)
constexpr int BK = 64;            // K per stage: one 128-byte swizzle row of bf16
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;    // 16 KB
constexpr int B_BYTES = 256 * BK * 2;   // 32 KB (N up to 256)
constexpr int NUM_THREADS = 192;
constexpr uint32_t TMEM_COLS = 512;     // two 256-column FP32 accumulators
constexpr int MAX_GROUPS = 264;

struct GemmArgs {
  int* status;
  const GroupRec* groups;
  const int* mtile_prefix;
  const int* dw_order;
  int G, E;
  int K;             // reduction length (FWD/DX)
  int n_out;         // valid output columns
  int m_out;         // DW: valid output rows
  int NT, MT;        // n-tiles per group; DW: m-tiles per group
  int hn;            // FWD1: H columns per tile (64 or 128)
  int I;             // FWD1 / DX2: intermediate size
  int b_group_rows;  // rows one group occupies in B's 2-D view
  void* out;
  void* out2;
  const void* aux;
  int64_t ld_out, ld_out2, ld_aux;
  int accumulate;
  uint32_t idesc;
  uint64_t budget_ns;
};

struct SmemCtl {
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
  int total_tiles;
};

constexpr size_t kSmemBytes = 1024 /* alignment slack */ + STAGES * (A_BYTES + B_BYTES) +
                              sizeof(SmemCtl) + sizeof(GroupRec) * MAX_GROUPS +
                              sizeof(int) * (MAX_GROUPS + 1) + sizeof(int) * MAX_GROUPS + 64;

struct TileInfo {
  int g, m0, n0, nkb;
};

template <int MODE>
__device__ __forceinline__ TileInfo decode_tile(int tile, const GemmArgs& a, const GroupRec* sg,
                                                const int* spre, const int* sord) {
  TileInfo t;
  if constexpr (MODE == MODE_DW2 || MODE == MODE_DW1) {
    const int per = a.MT * a.NT;
    const int gi = tile / per, local = tile - gi * per;
    t.g = sord[gi];
    const int nt = local / a.MT, mt = local - nt * a.MT;
    t.m0 = mt * BM;
    t.n0 = nt * 256;
    t.nkb = (sg[t.g].rows_pad + BK - 1) / BK;  // the tail block reads zeros past the end
  } else {
    // largest g with spre[g] * NT <= tile  (spre is non-decreasing)
    int lo = 0, hi = a.G - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (spre[mid] * a.NT <= tile) lo = mid; else hi = mid - 1;
    }
    t.g = lo;
    const int mt_g = spre[lo + 1] - spre[lo];
    const int local = tile - spre[lo] * a.NT;
    const int nt = local / mt_g, mt = local - nt * mt_g;
    t.m0 = mt * BM;
    t.n0 = nt * (MODE == MODE_FWD1 ? a.hn : 256);
    t.nkb = a.K / BK;
  }
  return t;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ void store_bf16x32(__nv_bfloat16* dst, const float* v) {
  uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint4 w;
    w.x = pack_bf16(v[8 * q + 0], v[8 * q + 1]);
    w.y = pack_bf16(v[8 * q + 2], v[8 * q + 3]);
    w.z = pack_bf16(v[8 * q + 4], v[8 * q + 5]);
    w.w = pack_bf16(v[8 * q + 6], v[8 * q + 7]);
    d4[q] = w;
  }
}

__device__ __forceinline__ void load_bf16x32(const __nv_bfloat16* src, float* v) {
  const uint4* s4 = reinterpret_cast<const uint4*>(src);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint4 w = s4[q];
    const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      v[8 * q + 2 * p] = __uint_as_float(u[p] << 16);
      v[8 * q + 2 * p + 1] = __uint_as_float(u[p] & 0xFFFF0000u);
    }
  }
}

template <int MODE>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    ggemm_kernel(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmA1,
                 const __grid_constant__ CUtensorMap tmB0, const __grid_constant__ CUtensorMap tmB1,
                 const GemmArgs args) {
  constexpr bool A_MN = (MODE == MODE_DW2 || MODE == MODE_DW1);
  constexpr bool B_MN = (MODE != MODE_FWD1 && MODE != MODE_FWD2);
  constexpr bool IS_DW = A_MN;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * A_BYTES;
  SmemCtl* ctl = reinterpret_cast<SmemCtl*>(sB + STAGES * B_BYTES);
  GroupRec* sg = reinterpret_cast<GroupRec*>(ctl + 1);
  int* spre = reinterpret_cast<int*>(sg + MAX_GROUPS);
  int* sord = spre + (MAX_GROUPS + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  volatile int* abort_flag = &ctl->abort_flag;

  for (int i = threadIdx.x; i < args.G; i += NUM_THREADS) {
    sg[i] = args.groups[i];
    spre[i] = args.mtile_prefix[i];
    sord[i] = args.dw_order[i];
  }
  if (threadIdx.x == 0) {
    spre[args.G] = args.mtile_prefix[args.G];
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&ctl->full[s], 1);
      mbar_init(&ctl->empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&ctl->tfull[a], 1);
      mbar_init(&ctl->tempty[a], 4);
    }
    mbar_init(&ctl->drain, 1);
    ctl->abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmA0);
    tma_prefetch_desc(&tmA1);
    tma_prefetch_desc(&tmB0);
    tma_prefetch_desc(&tmB1);
  }
  if (warp == 1) {
    tmem_alloc(&ctl->tmem_base, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = ctl->tmem_base;
  const int total_tiles = IS_DW ? args.G * args.MT * args.NT : spre[args.G] * args.NT;

  if (warp == 0) {
    // ------------------------------------------------------------ producer --
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0, issued = 0, lastpar = 0;
      const uint32_t a_bytes = A_BYTES;
      const uint32_t b_bytes = (MODE == MODE_FWD1) ? (uint32_t)(2 * args.hn * BK * 2) : B_BYTES;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < total_tiles; tile += gridDim.x) {
        const TileInfo t = decode_tile<MODE>(tile, args, sg, spre, sord);
        const GroupRec gr = sg[t.g];
        const bool shared = t.g >= args.E;
        for (int kb = 0; kb < t.nkb; ++kb) {
          if (!mbar_wait(&ctl->empty[stage], phase ^ 1, abort_flag, args.status,
                         MOE_ERR_DEVICE_TIMEOUT, args.budget_ns)) {
            ok = false;
            break;
          }
          uint64_t* fb = &ctl->full[stage];
          mbar_arrive_expect_tx(fb, a_bytes + b_bytes);
          uint8_t* a_dst = sA + stage * A_BYTES;
          uint8_t* b_dst = sB + stage * B_BYTES;
          const int k0 = kb * BK;
          if constexpr (MODE == MODE_FWD1) {
            tma_load_2d(a_dst, shared ? &tmA1 : &tmA0, fb, k0, (shared ? 0 : gr.a_row) + t.m0);
            const int brow = t.g * args.b_group_rows + t.n0;
            tma_load_2d(b_dst, &tmB0, fb, k0, brow);
            tma_load_2d(b_dst + args.hn * 128, &tmB0, fb, k0, brow + args.I);
          } else if constexpr (MODE == MODE_FWD2) {
            tma_load_2d(a_dst, &tmA0, fb, k0, gr.out_row + t.m0);
            tma_load_2d(b_dst, &tmB0, fb, k0, t.g * args.b_group_rows + t.n0);
          } else if constexpr (MODE == MODE_DX2 || MODE == MODE_DX1) {
            if constexpr (MODE == MODE_DX2)
              tma_load_2d(a_dst, shared ? &tmA1 : &tmA0, fb, k0, (shared ? 0 : gr.a_row) + t.m0);
            else
              tma_load_2d(a_dst, &tmA0, fb, k0, gr.out_row + t.m0);
            const int brow = t.g * args.b_group_rows + k0;
#pragma unroll
            for (int c = 0; c < 4; ++c) tma_load_2d(b_dst + c * 8192, &tmB0, fb, t.n0 + c * 64, brow);
          } else {  // DW2 / DW1: K runs over the group's rows
            const CUtensorMap* ma;
            const CUtensorMap* mb;
            int arow, brow;
            if constexpr (MODE == MODE_DW2) {
              ma = shared ? &tmA1 : &tmA0;
              arow = shared ? 0 : gr.a_row;
              mb = &tmB0;
              brow = gr.out_row;
            } else {
              ma = &tmA0;
              arow = gr.out_row;
              mb = shared ? &tmB1 : &tmB0;
              brow = shared ? 0 : gr.a_row;
            }
#pragma unroll
            for (int c = 0; c < 2; ++c) tma_load_2d(a_dst + c * 8192, ma, fb, t.m0 + c * 64, arow + k0);
#pragma unroll
            for (int c = 0; c < 4; ++c) tma_load_2d(b_dst + c * 8192, mb, fb, t.n0 + c * 64, brow + k0);
          }
          issued |= 1u << stage;
          lastpar = (lastpar & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      // Every copy this thread started must land before the CTA may exit.
      for (int s = 0; s < STAGES; ++s)
        if (issued & (1u << s)) {
          volatile int never = 0;
          mbar_wait(&ctl->full[s], (lastpar >> s) & 1u, &never, args.status,
                    MOE_ERR_DEVICE_TIMEOUT, args.budget_ns);
        }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer --
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < total_tiles; tile += gridDim.x, ++it) {
        const TileInfo t = decode_tile<MODE>(tile, args, sg, spre, sord);
        const int acc = it & 1;
        const uint32_t use = (uint32_t)(it >> 1);
        if (!mbar_wait(&ctl->tempty[acc], (use & 1u) ^ 1u, abort_flag, args.status,
                       MOE_ERR_DEVICE_TIMEOUT, args.budget_ns))
          break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * 256);
        for (int kb = 0; kb < t.nkb; ++kb) {
          if (!mbar_wait(&ctl->full[stage], phase, abort_flag, args.status,
                         MOE_ERR_DEVICE_TIMEOUT, args.budget_ns)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_base = smem_u32(sA + stage * A_BYTES);
          const uint32_t b_base = smem_u32(sB + stage * B_BYTES);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint64_t ad = A_MN ? smem_desc_sw128(a_base + kk * 2048, 8192, 1024)
                                     : smem_desc_sw128(a_base + kk * 32, 16, 1024);
            const uint64_t bd = B_MN ? smem_desc_sw128(b_base + kk * 2048, 8192, 1024)
                                     : smem_desc_sw128(b_base + kk * 32, 16, 1024);
            umma_f16(d_tmem, ad, bd, args.idesc, (kb | kk) != 0 ? 1u : 0u);
          }
          umma_commit(&ctl->empty[stage]);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        umma_commit(&ctl->tfull[acc]);
      }
      // Drain: all MMAs issued by this thread complete before tensor memory is freed.
      umma_commit(&ctl->drain);
      volatile int never = 0;
      mbar_wait(&ctl->drain, 0, &never, args.status, MOE_ERR_DEVICE_TIMEOUT, args.budget_ns);
    }
  } else {
    // ------------------------------------------------------------ epilogue --
    const int q = warp & 3;  // this warp may read TMEM lanes [32q, 32q + 32)
    const int r_in_tile = q * 32 + lane;
    int it = 0;
    for (int tile = blockIdx.x; tile < total_tiles; tile += gridDim.x, ++it) {
      const TileInfo t = decode_tile<MODE>(tile, args, sg, spre, sord);
      const int acc = it & 1;
      const uint32_t use = (uint32_t)(it >> 1);
      if (!mbar_wait(&ctl->tfull[acc], use & 1u, abort_flag, args.status, MOE_ERR_DEVICE_TIMEOUT,
                     args.budget_ns))
        break;
      tc_fence_after();
      const uint32_t taddr = tmem_base + (uint32_t)(acc * 256) + ((uint32_t)(q * 32) << 16);
      const GroupRec gr = sg[t.g];
      uint32_t r[32];
      float v[32];
      if constexpr (MODE == MODE_FWD1) {
        const int rloc = t.m0 + r_in_tile;
        const bool rv = rloc < gr.rows_pad;
        const int64_t orow = (int64_t)gr.out_row + rloc;
        __nv_bfloat16* H = reinterpret_cast<__nv_bfloat16*>(args.out) + orow * args.ld_out + t.n0;
        __nv_bfloat16* A1 = reinterpret_cast<__nv_bfloat16*>(args.out2);
        for (int c0 = 0; c0 < args.hn; c0 += 32) {
          uint32_t u[32];
          tmem_ld32_sync(taddr + c0, r);
          tmem_ld32_sync(taddr + args.hn + c0, u);
          if (rv) {
            float hv[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const float g = __uint_as_float(r[i]), up = __uint_as_float(u[i]);
              hv[i] = g / (1.0f + expf(-g)) * up;
            }
            store_bf16x32(H + c0, hv);
            if (A1 != nullptr) {
              __nv_bfloat16* a1r = A1 + orow * args.ld_out2 + t.n0 + c0;
#pragma unroll
              for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
              store_bf16x32(a1r, v);
#pragma unroll
              for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(u[i]);
              store_bf16x32(a1r + args.I, v);
            }
          }
        }
      } else if constexpr (MODE == MODE_FWD2 || MODE == MODE_DX1) {
        const int rloc = t.m0 + r_in_tile;
        const bool rv = rloc < gr.rows_pad;
        const int64_t orow = (int64_t)gr.out_row + rloc;
        __nv_bfloat16* O = reinterpret_cast<__nv_bfloat16*>(args.out) + orow * args.ld_out + t.n0;
        for (int c0 = 0; c0 < 256 && t.n0 + c0 < args.n_out; c0 += 32) {
          tmem_ld32_sync(taddr + c0, r);
          if (rv) {
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
            store_bf16x32(O + c0, v);
          }
        }
      } else if constexpr (MODE == MODE_DX2) {
        const int rloc = t.m0 + r_in_tile;
        const bool rv = rloc < gr.rows_pad;
        const int64_t orow = (int64_t)gr.out_row + rloc;
        const __nv_bfloat16* A1 =
            reinterpret_cast<const __nv_bfloat16*>(args.aux) + orow * args.ld_aux;
        __nv_bfloat16* dA = reinterpret_cast<__nv_bfloat16*>(args.out) + orow * args.ld_out;
        for (int c0 = 0; c0 < 256 && t.n0 + c0 < args.I; c0 += 32) {
          tmem_ld32_sync(taddr + c0, r);
          if (rv) {
            const int col = t.n0 + c0;
            float gv[32], uv[32], dg[32], du[32];
            load_bf16x32(A1 + col, gv);
            load_bf16x32(A1 + args.I + col, uv);
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const float dh = __uint_as_float(r[i]);
              const float g = gv[i];
              const float s = 1.0f / (1.0f + expf(-g));
              dg[i] = dh * uv[i] * s * (1.0f + g * (1.0f - s));
              du[i] = dh * g * s;
            }
            store_bf16x32(dA + col, dg);
            store_bf16x32(dA + args.I + col, du);
          }
        }
      } else {  // DW2 / DW1: f32 output [G, m_out, n_out]
        const int m = t.m0 + r_in_tile;
        const bool rv = m < args.m_out;
        float* O = reinterpret_cast<float*>(args.out) +
                   ((int64_t)t.g * args.m_out + m) * (int64_t)args.n_out + t.n0;
        for (int c0 = 0; c0 < 256 && t.n0 + c0 < args.n_out; c0 += 32) {
          if (t.nkb > 0) {
            tmem_ld32_sync(taddr + c0, r);
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = 0.0f;
          }
          if (rv) {
            float4* o4 = reinterpret_cast<float4*>(O + c0);
#pragma unroll
            for (int q4 = 0; q4 < 8; ++q4) {
              float4 w = make_float4(v[4 * q4], v[4 * q4 + 1], v[4 * q4 + 2], v[4 * q4 + 3]);
              if (args.accumulate) {
                const float4 o = o4[q4];
                w.x += o.x; w.y += o.y; w.z += o.z; w.w += o.w;
              }
              o4[q4] = w;
            }
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
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

// ------------------------------------------------------------------ host side --
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// bf16 matrix [rows, cols] (row-major, cols contiguous), box {64, box_rows}, 128B swizzle.
bool make_map(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, int box_rows) {
  EncodeTiledFn enc = get_encode();
  if (!enc || base == nullptr) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)(cols * 2)};
  cuuint32_t box[2] = {64u, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1u, 1u};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int MODE>
int launch_mode(const CUtensorMap& a0, const CUtensorMap& a1, const CUtensorMap& b0,
                const CUtensorMap& b1, const GemmArgs& args, cudaStream_t st) {
  static int num_sms = 0;
  static bool attr_set = false;
  if (!attr_set) {
    if (cudaFuncSetAttribute(ggemm_kernel<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kSmemBytes) != cudaSuccess)
      return MOE_ERR_CUDA;
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&num_sms, cudaDevAttrMultiProcessorCount, dev);
    attr_set = true;
  }
  ggemm_kernel<MODE><<<num_sms, NUM_THREADS, kSmemBytes, st>>>(a0, a1, b0, b1, args);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

uint64_t wait_budget_ns() {
  static uint64_t v = [] {
    const char* s = getenv("MOE_WAIT_BUDGET_NS");
    return s ? strtoull(s, nullptr, 10) : 4000000000ull;
  }();
  return v;
}

}  // namespace

int launch_grouped_gemm(GemmMode mode, const moe_dims& dm, const void* ws,
                        const GemmOperands& ops, void* stream) {
  const int G = dm.E + dm.S;
  if (G > MAX_GROUPS) return MOE_ERR_UNSUPPORTED_SHAPE;
  const WsLayout L = ws_layout(dm);
  const int64_t Rr = rows_routed(dm), Rt = rows_total(dm);
  const int64_t T = dm.T;
  const int d = dm.d, I = dm.I;
  const uint8_t* wsb = reinterpret_cast<const uint8_t*>(ws);

  GemmArgs a{};
  a.status = reinterpret_cast<int*>(const_cast<void*>(ws));
  a.groups = reinterpret_cast<const GroupRec*>(wsb + L.groups);
  a.mtile_prefix = reinterpret_cast<const int*>(wsb + L.mtile_prefix);
  a.dw_order = reinterpret_cast<const int*>(wsb + L.dw_order);
  a.G = G;
  a.E = dm.E;
  a.I = I;
  a.out = ops.out;
  a.out2 = ops.out2;
  a.aux = ops.aux;
  a.accumulate = ops.accumulate;
  a.budget_ns = wait_budget_ns();

  CUtensorMap m0{}, m1{}, n0{}, n1{};
  bool ok = true;
  // a dummy map stands in for unused slots (never read by the kernel)
  auto same = [](CUtensorMap& dst, const CUtensorMap& src) { dst = src; };
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);

  switch (mode) {
    case MODE_FWD1: {
      const int hn = (I % 128 == 0) ? 128 : 64;
      a.hn = hn;
      a.K = d;
      a.NT = I / hn;
      a.n_out = I;
      a.b_group_rows = 2 * I;
      a.ld_out = I;
      a.ld_out2 = 2 * I;
      a.idesc = idesc_bf16_f32(BM, 2 * hn, false, false);
      ok &= make_map(&m0, ops.a0, Rr, d, BM);
      if (dm.S > 0) ok &= make_map(&m1, ops.a1, T, d, BM); else same(m1, m0);
      ok &= make_map(&n0, ops.b0, (int64_t)G * 2 * I, d, hn);
      same(n1, n0);
      if (!ok) return MOE_ERR_CUDA;
      return launch_mode<MODE_FWD1>(m0, m1, n0, n1, a, st);
    }
    case MODE_FWD2: {
      a.K = I;
      a.NT = (d + 255) / 256;
      a.n_out = d;
      a.b_group_rows = d;
      a.ld_out = d;
      a.idesc = idesc_bf16_f32(BM, 256, false, false);
      ok &= make_map(&m0, ops.a0, Rt, I, BM);
      same(m1, m0);
      ok &= make_map(&n0, ops.b0, (int64_t)G * d, I, 256);
      same(n1, n0);
      if (!ok) return MOE_ERR_CUDA;
      return launch_mode<MODE_FWD2>(m0, m1, n0, n1, a, st);
    }
    case MODE_DX2: {
      a.K = d;
      a.NT = (I + 255) / 256;
      a.n_out = I;
      a.b_group_rows = d;
      a.ld_out = 2 * I;
      a.ld_aux = 2 * I;
      a.idesc = idesc_bf16_f32(BM, 256, false, true);
      ok &= make_map(&m0, ops.a0, Rr, d, BM);
      if (dm.S > 0) ok &= make_map(&m1, ops.a1, T, d, BM); else same(m1, m0);
      ok &= make_map(&n0, ops.b0, (int64_t)G * d, I, 64);
      same(n1, n0);
      if (!ok) return MOE_ERR_CUDA;
      return launch_mode<MODE_DX2>(m0, m1, n0, n1, a, st);
    }
    case MODE_DX1: {
      a.K = 2 * I;
      a.NT = (d + 255) / 256;
      a.n_out = d;
      a.b_group_rows = 2 * I;
      a.ld_out = d;
      a.idesc = idesc_bf16_f32(BM, 256, false, true);
      ok &= make_map(&m0, ops.a0, Rt, 2 * I, BM);
      same(m1, m0);
      ok &= make_map(&n0, ops.b0, (int64_t)G * 2 * I, d, 64);
      same(n1, n0);
      if (!ok) return MOE_ERR_CUDA;
      return launch_mode<MODE_DX1>(m0, m1, n0, n1, a, st);
    }
    case MODE_DW2: {  // dW2_g [d, I] = dY_g^T H_g
      a.m_out = d;
      a.n_out = I;
      a.MT = (d + BM - 1) / BM;
      a.NT = (I + 255) / 256;
      a.idesc = idesc_bf16_f32(BM, 256, true, true);
      ok &= make_map(&m0, ops.a0, Rr, d, 64);
      if (dm.S > 0) ok &= make_map(&m1, ops.a1, T, d, 64); else same(m1, m0);
      ok &= make_map(&n0, ops.b0, Rt, I, 64);
      same(n1, n0);
      if (!ok) return MOE_ERR_CUDA;
      return launch_mode<MODE_DW2>(m0, m1, n0, n1, a, st);
    }
    case MODE_DW1: {  // dW1_g [2I, d] = dA_g^T X_g
      a.m_out = 2 * I;
      a.n_out = d;
      a.MT = (2 * I) / BM;
      a.NT = (d + 255) / 256;
      a.idesc = idesc_bf16_f32(BM, 256, true, true);
      ok &= make_map(&m0, ops.a0, Rt, 2 * I, 64);
      same(m1, m0);
      ok &= make_map(&n0, ops.b0, Rr, d, 64);
      if (dm.S > 0) ok &= make_map(&n1, ops.b1, T, d, 64); else same(n1, n0);
      if (!ok) return MOE_ERR_CUDA;
      return launch_mode<MODE_DW1>(m0, m1, n0, n1, a, st);
    }
  }
  return MOE_ERR_INVALID_ARG;
}

}  // namespace moe
