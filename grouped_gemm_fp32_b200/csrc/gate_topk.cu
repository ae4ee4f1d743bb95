// gate_topk.cu -- FP32 gate and aux-loss-free top-k routing.
//
// Passage: dots.llm1 Technical Report, §Architecture "Mixture of Experts layer"
// (the gating layer is computed in FP32 rather than BF16, for stable and
// accurate expert selection; each token picks its top-6 of 128 routed experts)
// and "Load balancing" (a per-expert bias is added to the affinity scores only
// to decide the top-k routing).
//
// One CTA owns TM tokens and all E experts.  The logits tile [TM, E] is an
// FP32 SIMT GEMM (no tensor cores: the gate is the one FP32 contraction of the
// layer): X and Wg are staged through shared memory in K chunks of 32, each
// thread accumulates 4 tokens x 8 experts in registers, so every Wg value
// loaded from L2 is reused TM times.  TM is chosen so the grid is about one
// CTA per SM.  The finished logits go to shared memory and each warp then
// routes one token at a time: softmax (max-subtracted, expf), s = p + bias,
// k rounds of a warp-shuffle arg-max (equal s -> lower index), and the
// renormalised weights.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "moe_internal.cuh"

namespace moe {
namespace {

constexpr int KC = 32;  // K chunk

__global__ void gate_topk_kernel(const __nv_bfloat16* __restrict__ x, const float* __restrict__ wg,
                                 const float* __restrict__ bias, int64_t T, int d, int E, int k,
                                 int TM, int32_t* __restrict__ topk_idx,
                                 float* __restrict__ topk_w, float* __restrict__ probs) {
  extern __shared__ float sm[];
  const int NE = E / 8;                 // expert groups (8 experts each)
  const int tid = threadIdx.x;
  const int eg = tid % NE, tg = tid / NE;  // this thread: experts 8eg.., tokens 4tg..
  const bool active = tg < TM / 4;         // the block is padded to whole warps
  const int64_t t0 = (int64_t)blockIdx.x * TM;
  const int nthreads = blockDim.x;

  float* Xs = sm;             // [KC][TM]  transposed token chunk
  float* Ws = sm + KC * TM;   // [KC][E]   transposed gate chunk

  float acc[4][8];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.0f;

  for (int k0 = 0; k0 < d; k0 += KC) {
    // stage X[t0 .. t0+TM, k0 .. k0+KC) (bf16 -> f32, exact) and Wg[:, k0 .. k0+KC)
    for (int i = tid; i < TM * (KC / 8); i += nthreads) {
      const int r = i / (KC / 8), c8 = (i % (KC / 8)) * 8;
      const int64_t t = t0 + r;
      uint4 v = make_uint4(0, 0, 0, 0);
      if (t < T) v = *reinterpret_cast<const uint4*>(x + t * d + k0 + c8);
      const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int p = 0; p < 4; ++p) {
        Xs[(c8 + 2 * p) * TM + r] = __uint_as_float(u[p] << 16);
        Xs[(c8 + 2 * p + 1) * TM + r] = __uint_as_float(u[p] & 0xFFFF0000u);
      }
    }
    for (int i = tid; i < E * (KC / 4); i += nthreads) {
      const int e = i / (KC / 4), c4 = (i % (KC / 4)) * 4;
      const float4 v = *reinterpret_cast<const float4*>(wg + (int64_t)e * d + k0 + c4);
      Ws[(c4 + 0) * E + e] = v.x;
      Ws[(c4 + 1) * E + e] = v.y;
      Ws[(c4 + 2) * E + e] = v.z;
      Ws[(c4 + 3) * E + e] = v.w;
    }
    __syncthreads();
    if (active) {
#pragma unroll 8
      for (int kk = 0; kk < KC; ++kk) {
        const float4 xa = *reinterpret_cast<const float4*>(Xs + kk * TM + tg * 4);
        const float4 w0 = *reinterpret_cast<const float4*>(Ws + kk * E + eg * 8);
        const float4 w1 = *reinterpret_cast<const float4*>(Ws + kk * E + eg * 8 + 4);
        const float xv[4] = {xa.x, xa.y, xa.z, xa.w};
        const float wv[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(xv[i], wv[j], acc[i][j]);
      }
    }
    __syncthreads();
  }

  // logits tile -> shared memory [TM][E]
  float* L = sm;
  if (active) {
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 8; ++j) L[(tg * 4 + i) * E + eg * 8 + j] = acc[i][j];
  }
  __syncthreads();

  // routing: one warp per token
  const int warp = tid >> 5, lane = tid & 31, nwarps = nthreads >> 5;
  const int per = (E + 31) / 32;  // experts per lane (<= 8)
  for (int r = warp; r < TM; r += nwarps) {
    const int64_t t = t0 + r;
    if (t >= T) break;
    float p[8], s[8];
    float m = -INFINITY;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int e = lane + 32 * q;
      p[q] = (q < per && e < E) ? L[r * E + e] : -INFINITY;
      m = fmaxf(m, p[q]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    float z = 0.0f;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int e = lane + 32 * q;
      p[q] = (q < per && e < E) ? expf(p[q] - m) : 0.0f;
      z += p[q];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
    const float inv = 1.0f / z;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int e = lane + 32 * q;
      const bool valid = q < per && e < E;
      p[q] = valid ? p[q] * inv : 0.0f;
      s[q] = valid ? p[q] + (bias ? bias[e] : 0.0f) : -INFINITY;
      if (valid && probs) probs[t * E + e] = p[q];
    }
    float psel = 0.0f;
    for (int j = 0; j < k; ++j) {
      // lane-local best: larger s, then lower index (q ascending = index ascending)
      float bs = -INFINITY, bp = 0.0f;
      int be = 0x7fffffff;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        if (s[q] > bs) { bs = s[q]; be = lane + 32 * q; bp = p[q]; }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float os = __shfl_xor_sync(0xffffffffu, bs, o);
        const int oe = __shfl_xor_sync(0xffffffffu, be, o);
        const float op = __shfl_xor_sync(0xffffffffu, bp, o);
        if (os > bs || (os == bs && oe < be)) { bs = os; be = oe; bp = op; }
      }
#pragma unroll
      for (int q = 0; q < 8; ++q)
        if (lane + 32 * q == be) s[q] = -INFINITY;  // remove the winner
      psel += bp;
      if (lane == 0) {
        topk_idx[t * k + j] = be;
        topk_w[t * k + j] = bp;
      }
    }
    __syncwarp();
    const float rn = 1.0f / psel;
    for (int j = lane; j < k; j += 32) topk_w[t * k + j] *= rn;
    __syncwarp();
  }
}

}  // namespace

int launch_gate_topk(const moe_dims& dm, const void* x, const float* wg, const float* bias,
                     int32_t* idx, float* w, float* probs, void* stream) {
  static int num_sms = 0;
  if (num_sms == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&num_sms, cudaDevAttrMultiProcessorCount, dev);
    if (num_sms <= 0) num_sms = 148;
  }
  const int64_t T = dm.T;
  if (T == 0) return MOE_OK;
  // about one CTA per SM: TM tokens per CTA, a multiple of 4 in [4, 128]
  int64_t per = (T + num_sms - 1) / num_sms;
  int TM = (int)((per + 3) / 4 * 4);
  if (TM < 4) TM = 4;
  if (TM > 128) TM = 128;
  const int NE = dm.E / 8;
  while (TM > 4 && (TM / 4) * NE > 1024) TM -= 4;
  const int threads = ((TM / 4) * NE + 31) / 32 * 32;
  const size_t stage_bytes = sizeof(float) * KC * (TM + dm.E);
  const size_t logit_bytes = sizeof(float) * (size_t)TM * dm.E;
  const size_t smem = stage_bytes > logit_bytes ? stage_bytes : logit_bytes;
  if (smem > 48 * 1024) {
    if (cudaFuncSetAttribute(gate_topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem) != cudaSuccess)
      return MOE_ERR_CUDA;
  }
  const int64_t blocks = (T + TM - 1) / TM;
  gate_topk_kernel<<<(unsigned)blocks, threads, smem, reinterpret_cast<cudaStream_t>(stream)>>>(
      reinterpret_cast<const __nv_bfloat16*>(x), wg, bias, T, dm.d, dm.E, dm.k, TM, idx, w,
      probs);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace moe
