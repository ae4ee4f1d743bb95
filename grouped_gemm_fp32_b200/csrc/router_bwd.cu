// router_bwd.cu -- backward of the router and the aux-loss-free bias step.
//
// Passage: dots.llm1 Technical Report, §Architecture "Mixture of Experts layer"
// (FP32 gate; the combine weights are the affinities of the chosen experts) and
// "Load balancing" (a per-expert bias, used only to choose the top-k, adjusted
// during training to keep the loads balanced).
//
// The combine weights w_j = p_j / Z over the chosen set C (Z = sum_{j in C} p_j)
// depend on the logits through the renormalisation and the softmax; the
// selection itself (made on p + bias) carries no gradient.  Given dL/dw:
//   dp_j     = (dw_j - sum_i dw_i w_i) / Z              for j in C, 0 elsewhere
//   dlogit_e = p_e (dp_e - sum_j p_j dp_j)
//   dX      += dlogit Wg          dWg = dlogit^T X      (sgemm.cu)
// dlogits_kernel: one warp per token, FP32; it also writes dlogit as three
// exact bf16 planes (hi, mid, lo) for the tensor-core GEMMs, rows T..t_pad-1
// and columns E..e_pad-1 zero.  reduce_dwg_kernel adds the GEMM's split-K
// partial sums in split order (deterministic).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "moe_internal.cuh"

namespace moe {
namespace {

constexpr int DL_WARPS = 8;

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// v = hi + mid + lo exactly (to below 2^-24 |v|), each a bf16 value
__device__ __forceinline__ void split3(float v, __nv_bfloat16& hi, __nv_bfloat16& mid,
                                       __nv_bfloat16& lo) {
  hi = __float2bfloat16_rn(v);
  const float r1 = v - __bfloat162float(hi);  // exact
  mid = __float2bfloat16_rn(r1);
  const float r2 = r1 - __bfloat162float(mid);  // exact
  lo = __float2bfloat16_rn(r2);
}

__global__ void __launch_bounds__(DL_WARPS * 32)
    dlogits_kernel(const float* __restrict__ probs, const int32_t* __restrict__ idx,
                   const float* __restrict__ w, const float* __restrict__ dw, int64_t T,
                   int t_pad, int E, int e_pad, int k, float* __restrict__ dlogits,
                   __nv_bfloat16* __restrict__ planes) {
  __shared__ float dp_s[DL_WARPS][256];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float* dp = dp_s[warp];
  const int64_t plane = (int64_t)t_pad * e_pad;
  for (int64_t t = (int64_t)blockIdx.x * DL_WARPS + warp; t < t_pad;
       t += (int64_t)gridDim.x * DL_WARPS) {
    __nv_bfloat16* row = planes + t * e_pad;
    if (t >= T) {  // pad rows of the planes: zero
      const __nv_bfloat16 z = __float2bfloat16_rn(0.0f);
      for (int e = lane; e < e_pad; e += 32) {
        row[e] = z;
        row[plane + e] = z;
        row[2 * plane + e] = z;
      }
      continue;
    }
    for (int e = lane; e < e_pad; e += 32) dp[e] = 0.0f;
    __syncwarp();
    float zc = 0.0f, dot = 0.0f;
    for (int j = lane; j < k; j += 32) {
      const int e = idx[t * k + j];
      if (e >= 0 && e < E) zc += probs[t * E + e];
      dot += dw[t * k + j] * w[t * k + j];
    }
    zc = warp_sum(zc);
    dot = warp_sum(dot);
    const float rz = 1.0f / zc;
    float c = 0.0f;
    for (int j = lane; j < k; j += 32) {
      const int e = idx[t * k + j];
      if (e >= 0 && e < E) {
        const float dpj = (dw[t * k + j] - dot) * rz;
        dp[e] = dpj;
        c += probs[t * E + e] * dpj;
      }
    }
    c = warp_sum(c);
    __syncwarp();
    for (int e = lane; e < e_pad; e += 32) {
      float v = 0.0f;
      if (e < E) {
        v = probs[t * E + e] * (dp[e] - c);
        if (dlogits) dlogits[t * E + e] = v;
      }
      __nv_bfloat16 hi, mid, lo;
      split3(v, hi, mid, lo);
      row[e] = hi;
      row[plane + e] = mid;
      row[2 * plane + e] = lo;
    }
    __syncwarp();
  }
}

// dwg[e, c] (+)= sum_s partial[s][e][c], s ascending; four columns per thread.
__global__ void reduce_dwg_kernel(const float4* __restrict__ partial, int splits, int e_pad,
                                  int E, int d, int accumulate, float4* __restrict__ dwg) {
  const int64_t n4 = (int64_t)E * d / 4;
  const int64_t split4 = (int64_t)e_pad * d / 4;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4;
       i += (int64_t)gridDim.x * blockDim.x) {
    float4 s = accumulate ? dwg[i] : make_float4(0.f, 0.f, 0.f, 0.f);
    for (int p = 0; p < splits; ++p) {
      const float4 v = partial[p * split4 + i];  // row e of split p: same index as in dwg
      s.x += v.x;
      s.y += v.y;
      s.z += v.z;
      s.w += v.w;
    }
    dwg[i] = s;
  }
}

// bias_out[e] = bias_in[e] + gamma * sign(T k - E load_e)  (sign(mean - load_e))
__global__ void bias_update_kernel(const int32_t* __restrict__ counts, int E, int64_t Tk,
                                   float gamma, const float* bias_in, float* bias_out) {
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= E) return;
  const int64_t diff = Tk - (int64_t)counts[e] * E;
  const float s = diff > 0 ? gamma : diff < 0 ? -gamma : 0.0f;
  bias_out[e] = bias_in[e] + s;
}

}  // namespace

int launch_router_bwd(const moe_dims& dm, const void* x, const float* wg, const float* probs,
                      const int32_t* idx, const float* w, const float* dw, float* dlogits,
                      void* dx, float* dwg, int accumulate, void* ws, void* stream) {
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const WsLayout L = ws_layout(dm);
  uint8_t* wsb = reinterpret_cast<uint8_t*>(ws);
  int* status = reinterpret_cast<int*>(ws);
  if (dm.T == 0) {  // no tokens: dX untouched, dWg = 0 (or unchanged)
    if (!accumulate &&
        !cuda_ok(cudaMemsetAsync(dwg, 0, sizeof(float) * (size_t)dm.E * dm.d, st)))
      return MOE_ERR_CUDA;
    return MOE_OK;
  }
  void* wg_planes = wsb + L.gate_split;
  __nv_bfloat16* dl_planes = reinterpret_cast<__nv_bfloat16*>(wsb + L.dl_planes);
  float* partial = reinterpret_cast<float*>(wsb + L.gdw_part);
  int rc = launch_split_wg(dm, wg, wg_planes, stream);
  if (rc != MOE_OK) return rc;
  {
    int64_t blocks = (L.t_pad + DL_WARPS - 1) / DL_WARPS;
    if (blocks > 8192) blocks = 8192;
    dlogits_kernel<<<(unsigned)blocks, DL_WARPS * 32, 0, st>>>(
        probs, idx, w, dw, dm.T, L.t_pad, dm.E, L.e_pad, dm.k, dlogits, dl_planes);
    if (!cuda_ok(cudaGetLastError())) return MOE_ERR_CUDA;
  }
  rc = launch_gate_dx(dm, dl_planes, wg_planes, dx, status, stream);
  if (rc != MOE_OK) return rc;
  rc = launch_gate_dw(dm, dl_planes, x, partial, status, stream);
  if (rc != MOE_OK) return rc;
  {
    const int64_t n4 = (int64_t)dm.E * dm.d / 4;
    int64_t blocks = (n4 + 255) / 256;
    if (blocks > 4096) blocks = 4096;
    reduce_dwg_kernel<<<(unsigned)blocks, 256, 0, st>>>(
        reinterpret_cast<const float4*>(partial), L.gdw_splits, L.e_pad, dm.E, dm.d, accumulate,
        reinterpret_cast<float4*>(dwg));
  }
  return cuda_ok(cudaGetLastError()) ? MOE_OK : MOE_ERR_CUDA;
}

int launch_bias_update(const moe_dims& dm, const int32_t* counts, float gamma,
                       const float* bias_in, float* bias_out, void* stream) {
  bias_update_kernel<<<(dm.E + 255) / 256, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      counts, dm.E, dm.T * dm.k, gamma, bias_in, bias_out);
  return cuda_ok(cudaGetLastError()) ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace moe
