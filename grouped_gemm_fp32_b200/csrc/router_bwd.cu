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
// With the sequence-wise balance loss (same section, "Load balancing": the
// pages name it; the report they cite for their method defines it) its
// gradient dL/dp of every token, g[s, e] = alpha f_s,e / (n_seq L_s), joins dp
// before the softmax backward (seqbal_*_kernel compute g and the loss).
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

// seq_grad (nullable) [n_seq, E]: the balance loss's dL/dp of every token of a
// sequence of seq_len tokens, added to dp before the softmax backward.
__global__ void __launch_bounds__(DL_WARPS * 32)
    dlogits_kernel(const float* __restrict__ probs, const int32_t* __restrict__ idx,
                   const float* __restrict__ w, const float* __restrict__ dw,
                   const float* __restrict__ seq_grad, int64_t seq_len, int64_t T, int t_pad,
                   int E, int e_pad, int k, float* __restrict__ dlogits,
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
    if (seq_grad != nullptr) {  // dp += g over all experts; c += sum_e p_e g_e
      const float* g = seq_grad + (t / seq_len) * E;
      float cb = 0.0f;
      for (int e = lane; e < E; e += 32) {
        const float ge = g[e];
        dp[e] += ge;
        cb += probs[t * E + e] * ge;
      }
      c += warp_sum(cb);
      __syncwarp();
    }
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

// Sequence-wise balance loss, step 1: per chunk of <= kSeqChunk tokens inside
// one sequence, the column sums of the affinities and the pick counts of every
// expert.  Chunk c of sequence s covers tokens s L + c kSeqChunk onwards; cps
// chunks per full sequence.  Thread (r, e), r < R = blockDim / E, sums the
// chunk's tokens r, r + R, ... of column e; the R sums are then added in r order
// (fixed order: the same bits every run).
__global__ void __launch_bounds__(256)
    seqbal_partial_kernel(const float* __restrict__ probs, const int32_t* __restrict__ idx,
                          int64_t T, int E, int k, int64_t L, int cps,
                          float* __restrict__ psum, int32_t* __restrict__ pcnt) {
  __shared__ int hist[256];
  __shared__ float part[256];
  const int chunk = blockIdx.x;
  const int64_t s = chunk / cps;
  const int64_t c = chunk - s * cps;
  const int64_t t0 = s * L + c * kSeqChunk;
  const int64_t t1 = min(min(t0 + kSeqChunk, (s + 1) * L), T);
  const int tid = threadIdx.x;
  const int R = blockDim.x / E;
  const int r = tid / E, e = tid - r * E;
  if (tid < E) hist[tid] = 0;
  __syncthreads();
  for (int64_t i = t0 * k + tid; i < t1 * k; i += blockDim.x) {
    const int v = idx[i];
    if (v >= 0 && v < E) atomicAdd(&hist[v], 1);  // integer: the same counts in any order
  }
  float acc = 0.0f;
  if (r < R) {
#pragma unroll 8
    for (int64_t t = t0 + r; t < t1; t += R) acc += probs[t * E + e];
  }
  part[tid] = acc;
  __syncthreads();
  if (tid < E) {
    float sum = part[tid];
    for (int q = 1; q < R; ++q) sum += part[q * E + tid];
    psum[(int64_t)chunk * E + tid] = sum;
    pcnt[(int64_t)chunk * E + tid] = hist[tid];
  }
}

// Step 2 (one CTA of 1024 threads): per sequence s with L_s tokens and expert e
//   f = E cnt / (k L_s),  P = sum / L_s,  g[s, e] = alpha f / (n_seq L_s)
// and loss = alpha / n_seq * sum_s sum_e f P.  Thread (q, e), q < Q = 1024 / E,
// adds chunks q, q + Q, ... of the sequence; the Q sums, the experts and the
// sequences are then added in a fixed order.
__global__ void __launch_bounds__(1024)
    seqbal_finish_kernel(const float* __restrict__ psum, const int32_t* __restrict__ pcnt,
                         int64_t T, int E, int k, int64_t L, int64_t nseq, int cps, float alpha,
                         float* __restrict__ loss, float* __restrict__ seq_grad) {
  __shared__ float ps[1024];
  __shared__ int pc[1024];
  __shared__ float red[256];
  const int tid = threadIdx.x;
  const int Q = blockDim.x / E;
  const int q = tid / E, e = tid - q * E;
  float acc = 0.0f;  // thread e < E: its expert's f P over the sequences so far
  for (int64_t s = 0; s < nseq; ++s) {
    const int64_t Ls = min(L, T - s * L);
    const int nc = (int)((Ls + kSeqChunk - 1) / kSeqChunk);
    float P = 0.0f;
    int cnt = 0;
    if (q < Q) {
#pragma unroll 8
      for (int c = q; c < nc; c += Q) {
        const int64_t i = (s * cps + c) * E + e;
        P += psum[i];
        cnt += pcnt[i];
      }
    }
    ps[tid] = P;
    pc[tid] = cnt;
    __syncthreads();
    if (tid < E) {
      float Ps = ps[tid];
      int64_t cs = pc[tid];
      for (int j = 1; j < Q; ++j) {
        Ps += ps[j * E + tid];
        cs += pc[j * E + tid];
      }
      const float f = (float)E * (float)cs / ((float)k * (float)Ls);
      acc += f * (Ps / (float)Ls);
      seq_grad[s * E + tid] = alpha * f / ((float)nseq * (float)Ls);
    }
    __syncthreads();
  }
  if (tid < 256) red[tid] = tid < E ? acc : 0.0f;
  __syncthreads();
  for (int o = 128; o > 0; o >>= 1) {
    if (tid < o) red[tid] += red[tid + o];
    __syncthreads();
  }
  if (tid == 0) *loss = alpha * red[0] / (float)nseq;
}

}  // namespace

int launch_seq_balance(const moe_dims& dm, int64_t seq_len, float alpha, const int32_t* idx,
                       const float* probs, float* loss, float* seq_grad, void* ws,
                       void* stream) {
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (dm.T == 0) return cuda_ok(cudaMemsetAsync(loss, 0, sizeof(float), st)) ? MOE_OK : MOE_ERR_CUDA;
  const WsLayout L = ws_layout(dm);
  const int64_t nseq = (dm.T + seq_len - 1) / seq_len;
  const int64_t cps = (seq_len + kSeqChunk - 1) / kSeqChunk;
  const int64_t last = dm.T - (nseq - 1) * seq_len;
  const int64_t chunks = (nseq - 1) * cps + (last + kSeqChunk - 1) / kSeqChunk;
  if (chunks > L.sb_chunks || cps > (1 << 30)) return MOE_ERR_UNSUPPORTED_SHAPE;
  uint8_t* wsb = reinterpret_cast<uint8_t*>(ws);
  float* psum = reinterpret_cast<float*>(wsb + L.seqbal);
  int32_t* pcnt = reinterpret_cast<int32_t*>(psum + (size_t)L.sb_chunks * dm.E);
  seqbal_partial_kernel<<<(unsigned)chunks, 256, 0, st>>>(probs, idx, dm.T, dm.E, dm.k, seq_len,
                                                          (int)cps, psum, pcnt);
  seqbal_finish_kernel<<<1, 1024, 0, st>>>(psum, pcnt, dm.T, dm.E, dm.k, seq_len, nseq,
                                           (int)cps, alpha, loss, seq_grad);
  return cuda_ok(cudaGetLastError()) ? MOE_OK : MOE_ERR_CUDA;
}

int launch_router_bwd(const moe_dims& dm, const void* x, const float* wg, const float* probs,
                      const int32_t* idx, const float* w, const float* dw,
                      const float* seq_grad, int64_t seq_len, float* dlogits, void* dx,
                      float* dwg, int accumulate, void* ws, void* stream) {
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
        probs, idx, w, dw, seq_grad, seq_len, dm.T, L.t_pad, dm.E, L.e_pad, dm.k, dlogits,
        dl_planes);
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
