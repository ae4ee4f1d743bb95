// combine.cu -- weighted un-permute / combine of the expert outputs, and its
// backward.
//
// Passage: dots.llm1 Technical Report, §Architecture "Mixture of Experts layer":
// a token's output sums its top-6 routed experts (weighted) and the 2 shared
// experts that every token uses.
//
// HBM-bound; one warp per token, 16-byte vector accesses along the hidden
// dimension, FP32 accumulation.  The backward keeps the token's upstream row in
// registers for its k picks when d is 2048 or 4096.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "ep_internal.cuh"
#include "moe_internal.cuh"

namespace moe {
namespace {

__device__ __forceinline__ void acc8(float* a, uint4 v, float w) {
  const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    a[2 * p] = fmaf(w, __uint_as_float(u[p] << 16), a[2 * p]);
    a[2 * p + 1] = fmaf(w, __uint_as_float(u[p] & 0xFFFF0000u), a[2 * p + 1]);
  }
}

__device__ __forceinline__ uint4 pack8(const float* a) {
  uint4 r;
  uint32_t* u = reinterpret_cast<uint32_t*>(&r);
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    __nv_bfloat162 b = __floats2bfloat162_rn(a[2 * p], a[2 * p + 1]);
    u[p] = *reinterpret_cast<uint32_t*>(&b);
  }
  return r;
}

// Eight accumulated columns to the output: bf16 (one 16-byte vector) or, F32,
// the FP32 sums themselves (two).  Both take the same sums in the same order.
template <bool F32>
__device__ __forceinline__ void store8(void* out, int64_t i, const float* a) {
  if constexpr (F32) {
    float4* o = reinterpret_cast<float4*>(out) + 2 * i;
    o[0] = make_float4(a[0], a[1], a[2], a[3]);
    o[1] = make_float4(a[4], a[5], a[6], a[7]);
  } else {
    reinterpret_cast<uint4*>(out)[i] = pack8(a);
  }
}

// out[t] = sum_j w[t, j] y[row_of[t, j]] + sum_s ys[s T + t]  (ys = y + Rr rows when the
// shared experts' rows follow the routed ones in one buffer)
template <int KMAX, bool F32>
__global__ void combine_kernel(const uint4* __restrict__ y, const uint4* __restrict__ ys,
                               const int32_t* __restrict__ row_of, const float* __restrict__ w,
                               int64_t T, int row_vec, int k, int S, int64_t Rr,
                               void* __restrict__ out) {
  const int64_t t = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (t >= T) return;
  const uint4* src[KMAX];
  float wt[KMAX];
#pragma unroll
  for (int j = 0; j < KMAX; ++j) {
    if (j < k) {
      const int32_t r = row_of[t * k + j];
      const bool ok = r >= 0 && r < Rr;  // -1 (a pick without a row) or stale: skipped
      src[j] = y + (ok ? (int64_t)r * row_vec : 0);
      wt[j] = ok ? (w ? w[t * k + j] : 1.0f) : 0.0f;
    } else if (j < k + S) {
      src[j] = ys + ((int64_t)(j - k) * T + t) * row_vec;
      wt[j] = 1.0f;
    }
  }
  for (int c = lane; c < row_vec; c += 32) {
    float a[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    uint4 v[KMAX];
#pragma unroll
    for (int j = 0; j < KMAX; ++j)
      if (j < k + S) v[j] = src[j][c];
#pragma unroll
    for (int j = 0; j < KMAX; ++j)
      if (j < k + S) acc8(a, v[j], wt[j]);
    store8<F32>(out, t * row_vec + c, a);
  }
}

// Generic fallback (any k + S): rows gathered on the fly.
template <bool F32>
__global__ void combine_kernel_any(const uint4* __restrict__ y, const uint4* __restrict__ ys,
                                   const int32_t* __restrict__ row_of, const float* __restrict__ w,
                                   int64_t T, int row_vec, int k, int S, int64_t Rr,
                                   void* __restrict__ out) {
  const int64_t t = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (t >= T) return;
  for (int c = lane; c < row_vec; c += 32) {
    float a[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    for (int j = 0; j < k + S; ++j) {
      if (j < k) {
        const int64_t r = row_of[t * k + j];
        if (r < 0 || r >= Rr) continue;  // a pick without a row
        acc8(a, y[r * row_vec + c], w ? w[t * k + j] : 1.0f);
      } else {
        acc8(a, ys[((int64_t)(j - k) * T + t) * row_vec + c], 1.0f);
      }
    }
    store8<F32>(out, t * row_vec + c, a);
  }
}

// The pads of a local dY: with `pads` set, the launch's last E * kPadSplit CTAs
// zero the segments' pad rows (the dW GEMMs read them as K rows) while the others
// scatter.  Not used under expert parallelism, where the owners zero theirs.
struct DyPads {
  const GroupRec* groups;  // null: no pad CTAs
  int E;
  int* status;
};

// dy[row_of[t, j]] = w[t, j] dout[t] (bf16);  dw[t, j] = <dout[t], y[row_of[t, j]]>
__global__ void combine_bwd_kernel(const uint4* __restrict__ dout, const uint4* __restrict__ y,
                                   const int32_t* __restrict__ row_of, const float* __restrict__ w,
                                   int64_t T, int row_vec, int k, int64_t Rr,
                                   uint4* __restrict__ dy,
                                   float* __restrict__ dw, EpDy ep, DyPads pads) {
  if (pads.groups != nullptr) {
    const unsigned tok_blocks = gridDim.x - (unsigned)pads.E * kPadSplit;
    if (blockIdx.x >= tok_blocks) {
      const int pb = (int)(blockIdx.x - tok_blocks);
      zero_group_pad_rows(pads.groups, pb / kPadSplit, pb % kPadSplit, row_vec, dy, Rr,
                          pads.status);
      return;
    }
  }
  const int64_t t = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  for (int j = 0; t < T && j < k; ++j) {
    const int64_t r = row_of[t * k + j];
    const float wj = w[t * k + j];
    if (r < 0 || r >= Rr) {  // a pick without a row: nothing to scatter, no gradient
      if (lane == 0) dw[t * k + j] = 0.0f;
      continue;
    }
    uint4* drow = ep_dy_row(ep, dy, t, k, j, r, row_vec);
    float dot = 0.0f;
    for (int c = lane; c < row_vec; c += 32) {
      const uint4 g = dout[t * row_vec + c];
      const uint4 yv = y[r * row_vec + c];
      float a[8] = {0, 0, 0, 0, 0, 0, 0, 0};
      acc8(a, g, wj);
      if (drow) drow[c] = pack8(a);
      const uint32_t gu[4] = {g.x, g.y, g.z, g.w}, yu[4] = {yv.x, yv.y, yv.z, yv.w};
#pragma unroll
      for (int p = 0; p < 4; ++p) {
        dot = fmaf(__uint_as_float(gu[p] << 16), __uint_as_float(yu[p] << 16), dot);
        dot = fmaf(__uint_as_float(gu[p] & 0xFFFF0000u), __uint_as_float(yu[p] & 0xFFFF0000u), dot);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
    if (lane == 0) dw[t * k + j] = dot;
  }
  if (ep.W) ep_signal_last_cta(ep.done, ep.peer_ws, ep.W, EP_CTR_DY);
}

// Same, with the token's dOut row held in registers for all k picks: lane l owns
// vectors l, l + 32, ... of the row (VPL = row_vec / 32 of them), and each pick's
// Y row is loaded whole before it is used, so VPL loads are in flight per lane.
template <int VPL>
__global__ void combine_bwd_reg_kernel(const uint4* __restrict__ dout, const uint4* __restrict__ y,
                                       const int32_t* __restrict__ row_of,
                                       const float* __restrict__ w, int64_t T, int k, int64_t Rr,
                                       uint4* __restrict__ dy, float* __restrict__ dw, EpDy ep,
                                       DyPads pads) {
  constexpr int row_vec = 32 * VPL;
  if (pads.groups != nullptr) {
    const unsigned tok_blocks = gridDim.x - (unsigned)pads.E * kPadSplit;
    if (blockIdx.x >= tok_blocks) {
      const int pb = (int)(blockIdx.x - tok_blocks);
      zero_group_pad_rows(pads.groups, pb / kPadSplit, pb % kPadSplit, row_vec, dy, Rr,
                          pads.status);
      return;
    }
  }
  const int64_t t = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  uint4 g[VPL];
  if (t < T) {
#pragma unroll
    for (int i = 0; i < VPL; ++i) g[i] = dout[t * row_vec + lane + 32 * i];
  }
  for (int j = 0; t < T && j < k; ++j) {
    const int64_t r = row_of[t * k + j];
    const float wj = w[t * k + j];
    if (r < 0 || r >= Rr) {  // a pick without a row: nothing to scatter, no gradient
      if (lane == 0) dw[t * k + j] = 0.0f;
      continue;
    }
    uint4* drow = ep_dy_row(ep, dy, t, k, j, r, row_vec);
    uint4 yv[VPL];
#pragma unroll
    for (int i = 0; i < VPL; ++i) yv[i] = y[r * row_vec + lane + 32 * i];
    float dot = 0.0f;
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      float a[8] = {0, 0, 0, 0, 0, 0, 0, 0};
      acc8(a, g[i], wj);
      if (drow) drow[lane + 32 * i] = pack8(a);
      const uint32_t gu[4] = {g[i].x, g[i].y, g[i].z, g[i].w};
      const uint32_t yu[4] = {yv[i].x, yv[i].y, yv[i].z, yv[i].w};
#pragma unroll
      for (int p = 0; p < 4; ++p) {
        dot = fmaf(__uint_as_float(gu[p] << 16), __uint_as_float(yu[p] << 16), dot);
        dot = fmaf(__uint_as_float(gu[p] & 0xFFFF0000u), __uint_as_float(yu[p] & 0xFFFF0000u),
                   dot);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
    if (lane == 0) dw[t * k + j] = dot;
  }
  if (ep.W) ep_signal_last_cta(ep.done, ep.peer_ws, ep.W, EP_CTR_DY);
}

}  // namespace

int launch_combine(const moe_dims& dm, const void* y, const void* y_shared,
                   const int32_t* row_of, const float* w, void* out, bool f32_out, void* stream) {
  if (dm.T == 0) return MOE_OK;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int warps = 8;
  const unsigned blocks = (unsigned)((dm.T + warps - 1) / warps);
  const int row_vec = dm.d / 8;
  const int64_t Rr = rows_routed(dm);
  const uint4* yv = reinterpret_cast<const uint4*>(y);
  // the shared experts' rows: their own buffer, or the rows after the routed ones
  const uint4* ys = y_shared ? reinterpret_cast<const uint4*>(y_shared) : yv + Rr * row_vec;
  if (dm.k + dm.S <= 8) {
    if (f32_out)
      combine_kernel<8, true><<<blocks, warps * 32, 0, st>>>(yv, ys, row_of, w, dm.T, row_vec,
                                                            dm.k, dm.S, Rr, out);
    else
      combine_kernel<8, false><<<blocks, warps * 32, 0, st>>>(yv, ys, row_of, w, dm.T, row_vec,
                                                             dm.k, dm.S, Rr, out);
  } else {
    if (f32_out)
      combine_kernel_any<true><<<blocks, warps * 32, 0, st>>>(yv, ys, row_of, w, dm.T, row_vec,
                                                             dm.k, dm.S, Rr, out);
    else
      combine_kernel_any<false><<<blocks, warps * 32, 0, st>>>(yv, ys, row_of, w, dm.T, row_vec,
                                                              dm.k, dm.S, Rr, out);
  }
  return cuda_ok(cudaGetLastError()) ? MOE_OK : MOE_ERR_CUDA;
}

static int combine_bwd_kernels(const moe_dims& dm, const void* dout, const void* y,
                               const int32_t* row_of, const float* w, void* dy, float* dw,
                               const EpDy& ep, const DyPads& pads, cudaStream_t st) {
  const int warps = 8;
  const unsigned pad_blocks = pads.groups != nullptr ? (unsigned)dm.E * kPadSplit : 0u;
  // one CTA at least: under expert parallelism the last CTA signals the owners
  const unsigned blocks = (unsigned)(dm.T > 0 ? (dm.T + warps - 1) / warps : 1) + pad_blocks;
  const int64_t Rr = rows_routed(dm);
  const uint4* dv = reinterpret_cast<const uint4*>(dout);
  const uint4* yv = reinterpret_cast<const uint4*>(y);
  uint4* dyv = reinterpret_cast<uint4*>(dy);
  const int row_vec = dm.d / 8;
  // the register-resident form uses ~170 registers a thread: 4-warp CTAs, three per SM
  const unsigned blocks4 = (unsigned)(dm.T > 0 ? (dm.T + 3) / 4 : 1) + pad_blocks;
  if (row_vec == 512)
    combine_bwd_reg_kernel<16><<<blocks4, 128, 0, st>>>(dv, yv, row_of, w, dm.T, dm.k, Rr, dyv,
                                                        dw, ep, pads);
  else if (row_vec == 256)
    combine_bwd_reg_kernel<8><<<blocks4, 128, 0, st>>>(dv, yv, row_of, w, dm.T, dm.k, Rr, dyv,
                                                       dw, ep, pads);
  else
    combine_bwd_kernel<<<blocks, warps * 32, 0, st>>>(dv, yv, row_of, w, dm.T, row_vec, dm.k, Rr,
                                                      dyv, dw, ep, pads);
  return cuda_ok(cudaGetLastError()) ? MOE_OK : MOE_ERR_CUDA;
}

int launch_combine_bwd(const moe_dims& dm, const void* ws, const void* dout, const void* y,
                       const int32_t* row_of, const float* w, void* dy, float* dw, void* stream) {
  if (dm.T == 0) return MOE_OK;  // no routed rows, so no pad rows either
  EpDy none{};
  DyPads pads{};
  const uint8_t* wsb = reinterpret_cast<const uint8_t*>(ws);
  pads.groups = reinterpret_cast<const GroupRec*>(wsb + ws_layout(dm).groups);
  pads.E = dm.E;
  pads.status = reinterpret_cast<int*>(const_cast<void*>(ws));
  return combine_bwd_kernels(dm, dout, y, row_of, w, dy, dw, none, pads,
                             reinterpret_cast<cudaStream_t>(stream));
}

// Under expert parallelism: dY rows go to their owners' receive buffers (whose
// pad rows the owners zero), and the last CTA signals every owner.
int launch_combine_bwd_ep(const moe_dims& dm, const moe_ep_peers& pe, const void* dout,
                          const void* y, const int32_t* row_of, const float* w,
                          const int32_t* idx, const int32_t* offsets, float* dw, void* stream) {
  const EpLayout L = ep_layout(dm.E, pe.world);
  uint8_t* epb = reinterpret_cast<uint8_t*>(pe.ep_ws[pe.rank]);
  EpDy ep{};
  ep.rows = ep_ptrs(pe.rows, pe.world);
  ep.peer_ws = ep_ptrs(pe.ep_ws, pe.world);
  ep.send_dst = reinterpret_cast<const int32_t*>(epb + L.send_dst);
  ep.over = reinterpret_cast<const int32_t*>(epb + L.over);
  ep.idx = idx;
  ep.offsets = offsets;
  ep.done = reinterpret_cast<int*>(epb) + EP_DONE_DY;
  ep.El = dm.E / pe.world;
  ep.W = pe.world;
  return combine_bwd_kernels(dm, dout, y, row_of, w, nullptr, dw, ep, DyPads{},
                             reinterpret_cast<cudaStream_t>(stream));
}

}  // namespace moe
