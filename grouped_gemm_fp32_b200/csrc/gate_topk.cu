// gate_topk.cu -- FP32 gate and aux-loss-free top-k routing.
//
// Passage: dots.llm1 Technical Report, §Architecture "Mixture of Experts layer"
// (the gating layer is computed in FP32 rather than BF16, for stable and
// accurate expert selection; each token picks its top-6 of 128 routed experts)
// and "Load balancing" (a per-expert bias is added to the affinity scores only
// to decide the top-k routing).
//
// One CTA owns a tile of tokens and all E experts.  The logits tile [TM, E] is an
// FP32 SIMT GEMM (no tensor cores: the gate is the one FP32 contraction of the
// layer): X and Wg are staged through shared memory in K chunks of 32, each
// thread accumulates 4 tokens x 8 experts in registers, so every Wg value
// loaded from L2 is reused TM times.  TM is chosen so the grid is about one
// CTA per SM; the next K chunk is prefetched into registers while the current
// one is multiplied (one barrier per chunk).  The finished logits go to shared
// memory and each warp then
// routes one token at a time: softmax (max-subtracted, expf), s = p + bias,
// k rounds of a warp-shuffle arg-max (equal s -> lower index), and the
// renormalised weights.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "moe_internal.cuh"

namespace moe {
namespace {

constexpr int KC = 32;    // K chunk
constexpr int MAXV = 4;   // 16-byte prefetch registers per thread and operand

constexpr int MAX_THREADS = 512;

// Routing of the TM tokens whose logits sit in shared memory L[TM][E]: one warp
// per token.
__device__ __forceinline__ void route_tile(const float* L, int64_t t0, int TM, int64_t T, int E,
                                           int k, const float* __restrict__ bias,
                                           int32_t* __restrict__ topk_idx,
                                           float* __restrict__ topk_w, float* __restrict__ probs) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarps = blockDim.x >> 5;
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

// Generic path (any E % 8 == 0): 4 tokens x 8 experts per thread.
__global__ void __launch_bounds__(MAX_THREADS)
    gate_topk_kernel(const __nv_bfloat16* __restrict__ x, const float* __restrict__ wg,
                                 const float* __restrict__ bias, int64_t T, int d, int E, int k,
                                 int TM, int32_t* __restrict__ topk_idx,
                                 float* __restrict__ topk_w, float* __restrict__ probs) {
  extern __shared__ float sm[];
  const int NE = E / 8;                    // expert groups (8 experts each)
  const int tid = threadIdx.x;
  const int eg = tid % NE, tg = tid / NE;  // this thread: experts 8eg.., tokens 4tg..
  const bool active = tg < TM / 4;         // the block is padded to whole warps
  const int64_t t0 = (int64_t)blockIdx.x * TM;
  const int nthreads = blockDim.x;
  const int buf_floats = KC * (TM + E);    // one stage: Xs [KC][TM] then Ws [KC][E]

  float acc[4][8];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.0f;

  // Prefetch of one K chunk into registers.  X: 16-byte piece (row r, cols c8..c8+7)
  // for i = r + TM * (c8 / 8); W: (expert e, cols c4..c4+3) for i = e + E * (c4 / 4).
  // Consecutive threads take consecutive rows / experts, so the transposed
  // shared-memory stores below hit consecutive banks.
  uint4 xr[MAXV];
  float4 wr[MAXV];
  auto load_chunk = [&](int k0) {
#pragma unroll
    for (int u = 0; u < MAXV; ++u) {
      const int i = tid + u * nthreads;
      if (i < TM * (KC / 8)) {
        const int r = i % TM, c8 = (i / TM) * 8;
        const int64_t t = t0 + r;
        xr[u] = t < T ? *reinterpret_cast<const uint4*>(x + t * d + k0 + c8) : make_uint4(0, 0, 0, 0);
      }
      if (i < E * (KC / 4)) {
        const int e = i % E, c4 = (i / E) * 4;
        wr[u] = *reinterpret_cast<const float4*>(wg + (int64_t)e * d + k0 + c4);
      }
    }
  };
  auto store_chunk = [&](float* buf) {
    float* Xs = buf;
    float* Ws = buf + KC * TM;
#pragma unroll
    for (int u = 0; u < MAXV; ++u) {
      const int i = tid + u * nthreads;
      if (i < TM * (KC / 8)) {
        const int r = i % TM, c8 = (i / TM) * 8;
        const uint32_t w4[4] = {xr[u].x, xr[u].y, xr[u].z, xr[u].w};
#pragma unroll
        for (int p = 0; p < 4; ++p) {
          Xs[(c8 + 2 * p) * TM + r] = __uint_as_float(w4[p] << 16);
          Xs[(c8 + 2 * p + 1) * TM + r] = __uint_as_float(w4[p] & 0xFFFF0000u);
        }
      }
      if (i < E * (KC / 4)) {
        const int e = i % E, c4 = (i / E) * 4;
        Ws[(c4 + 0) * E + e] = wr[u].x;
        Ws[(c4 + 1) * E + e] = wr[u].y;
        Ws[(c4 + 2) * E + e] = wr[u].z;
        Ws[(c4 + 3) * E + e] = wr[u].w;
      }
    }
  };

  const int nchunks = d / KC;
  load_chunk(0);
  store_chunk(sm);
  __syncthreads();
  for (int c = 0; c < nchunks; ++c) {
    if (c + 1 < nchunks) load_chunk((c + 1) * KC);  // in flight while this chunk computes
    const float* Xs = sm + (c & 1) * buf_floats;
    const float* Ws = Xs + KC * TM;
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
    if (c + 1 < nchunks) store_chunk(sm + ((c + 1) & 1) * buf_floats);
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

  route_tile(L, t0, TM, T, E, k, bias, topk_idx, topk_w, probs);
}


// Fast path (E % 32 == 0): 8 * TI tokens per CTA (32 or 64), TI tokens x 4
// experts per thread, E * 2 threads (8 warps for E = 128).
//  * Wg chunks [E][32] are copied into shared memory unchanged with cp.async
//    (whole 128-byte rows: coalesced, no register staging), three chunks in
//    flight; X chunks are widened to f32 through registers one chunk ahead.
//  * Thread (tg, eg) owns tokens tg + 8i and experts eg + (E/4) j and reads
//    4 consecutive K values of each as one float4.  Rows are padded to 36
//    floats, so the 8 expert rows / 4 token rows a warp reads at once fall in
//    distinct banks: every read is a conflict-free broadcast, 8 reads per 64
//    FFMAs.  Small CTAs let several share an SM to hide latency.
constexpr int RS = KC + 4;  // padded row stride (floats)
constexpr int WSTAGES = 3;

__device__ __forceinline__ void cp_async16(float* dst, const float* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(
                   static_cast<uint32_t>(__cvta_generic_to_shared(dst))),
               "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// TI = token rows per thread (4 or 8): the CTA covers TM = 8 * TI tokens.
template <int TI>
__global__ void __launch_bounds__(512)
    gate_topk_kernel_t32(const __nv_bfloat16* __restrict__ x, const float* __restrict__ wg,
                         const float* __restrict__ bias, int64_t T, int d, int E, int k,
                         int32_t* __restrict__ topk_idx, float* __restrict__ topk_w,
                         float* __restrict__ probs) {
  constexpr int TM32 = 8 * TI;             // tokens of this CTA
  extern __shared__ float sm[];
  float* Ws = sm;                          // [WSTAGES][E][RS]
  float* Xs = sm + WSTAGES * E * RS;       // [2][TM32][RS]
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int EQ = E / 4;                          // expert groups
  const int WE = E / 32;                         // warps across the experts
  const int eg = (warp % WE) * 8 + (lane & 7);   // experts eg + EQ * j
  const int tg = (warp / WE) * 4 + (lane >> 3);  // tokens tg + 8 * i  (tg < 8)
  const int64_t t0 = (int64_t)blockIdx.x * TM32;
  const int nthreads = blockDim.x;  // 2E

  float acc[TI][4];
#pragma unroll
  for (int i = 0; i < TI; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.0f;

  auto issue_w = [&](int c) {  // Wg[:, 32c .. 32c+32) -> stage c % 3, 8 pieces of 16 B a row
    float* dst = Ws + (c % WSTAGES) * E * RS;
    for (int i = tid; i < E * 8; i += nthreads) {
      const int e = i >> 3, q = i & 7;
      cp_async16(dst + e * RS + q * 4, wg + (int64_t)e * d + c * KC + q * 4);
    }
  };
  // X pieces of 8 bf16: TM32 * 4 of them, at most 2 per thread (2E >= 64 threads... E >= 32)
  constexpr int XP = (TM32 * (KC / 8) + 63) / 64;
  uint4 xr[XP];
  auto load_x = [&](int c) {
#pragma unroll
    for (int u = 0; u < XP; ++u) {
      const int i = tid + u * nthreads;
      if (i < TM32 * (KC / 8)) {
        const int xrow = i % TM32, xc8 = (i / TM32) * 8;
        const int64_t t = t0 + xrow;
        xr[u] = t < T ? *reinterpret_cast<const uint4*>(x + t * d + c * KC + xc8)
                      : make_uint4(0, 0, 0, 0);
      }
    }
  };
  auto store_x = [&](int c) {
#pragma unroll
    for (int u = 0; u < XP; ++u) {
      const int i = tid + u * nthreads;
      if (i < TM32 * (KC / 8)) {
        const int xrow = i % TM32, xc8 = (i / TM32) * 8;
        float* dst = Xs + (c & 1) * TM32 * RS + xrow * RS + xc8;
        const uint32_t w4[4] = {xr[u].x, xr[u].y, xr[u].z, xr[u].w};
        *reinterpret_cast<float4*>(dst) =
            make_float4(__uint_as_float(w4[0] << 16), __uint_as_float(w4[0] & 0xFFFF0000u),
                        __uint_as_float(w4[1] << 16), __uint_as_float(w4[1] & 0xFFFF0000u));
        *reinterpret_cast<float4*>(dst + 4) =
            make_float4(__uint_as_float(w4[2] << 16), __uint_as_float(w4[2] & 0xFFFF0000u),
                        __uint_as_float(w4[3] << 16), __uint_as_float(w4[3] & 0xFFFF0000u));
      }
    }
  };

  const int n = d / KC;
  issue_w(0);
  cp_async_commit();
  if (n > 1) issue_w(1);
  cp_async_commit();
  load_x(0);
  store_x(0);
  if (n > 1) load_x(1);
  for (int c = 0; c < n; ++c) {
    cp_async_wait<1>();  // this thread's copies of chunk c have landed
    __syncthreads();     // everyone's have; chunk c - 1 is no longer being read
    if (c + 2 < n) issue_w(c + 2);
    cp_async_commit();   // (possibly empty: keeps the group count uniform)
    if (c + 1 < n) store_x(c + 1);
    if (c + 2 < n) load_x(c + 2);
    const float* W = Ws + (c % WSTAGES) * E * RS;
    const float* X = Xs + (c & 1) * TM32 * RS;
#pragma unroll 2
    for (int kk = 0; kk < KC; kk += 4) {
      float4 xv[TI], wv[4];
#pragma unroll
      for (int i = 0; i < TI; ++i) xv[i] = *reinterpret_cast<const float4*>(X + (tg + 8 * i) * RS + kk);
#pragma unroll
      for (int j = 0; j < 4; ++j) wv[j] = *reinterpret_cast<const float4*>(W + (eg + EQ * j) * RS + kk);
#pragma unroll
      for (int i = 0; i < TI; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          acc[i][j] = fmaf(xv[i].x, wv[j].x, acc[i][j]);
          acc[i][j] = fmaf(xv[i].y, wv[j].y, acc[i][j]);
          acc[i][j] = fmaf(xv[i].z, wv[j].z, acc[i][j]);
          acc[i][j] = fmaf(xv[i].w, wv[j].w, acc[i][j]);
        }
    }
  }
  __syncthreads();

  float* L = sm;  // logits tile [TM32][E] (reuses the Wg stages)
#pragma unroll
  for (int i = 0; i < TI; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) L[(tg + 8 * i) * E + eg + EQ * j] = acc[i][j];
  __syncthreads();
  route_tile(L, t0, TM32, T, E, k, bias, topk_idx, topk_w, probs);
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
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (dm.E % 32 == 0 && dm.E <= 256) {
    // 64 tokens per CTA (half the Wg staging per token) while that still gives
    // every SM at least ~1.5 CTAs; 32 otherwise.
    const bool wide = T >= (int64_t)64 * num_sms * 3 / 2;
    const int TMv = wide ? 64 : 32;
    const int threads = 2 * dm.E;
    size_t smem = sizeof(float) * RS * (WSTAGES * dm.E + 2 * TMv);
    if (smem < sizeof(float) * (size_t)TMv * dm.E) smem = sizeof(float) * (size_t)TMv * dm.E;
    const int64_t blocks = (T + TMv - 1) / TMv;
    const __nv_bfloat16* xb = reinterpret_cast<const __nv_bfloat16*>(x);
    if (wide) {
      if (smem > 48 * 1024 &&
          !cuda_ok(cudaFuncSetAttribute(gate_topk_kernel_t32<8>,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)))
        return MOE_ERR_CUDA;
      gate_topk_kernel_t32<8><<<(unsigned)blocks, threads, smem, st>>>(xb, wg, bias, T, dm.d, dm.E,
                                                                      dm.k, idx, w, probs);
    } else {
      if (smem > 48 * 1024 &&
          !cuda_ok(cudaFuncSetAttribute(gate_topk_kernel_t32<4>,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)))
        return MOE_ERR_CUDA;
      gate_topk_kernel_t32<4><<<(unsigned)blocks, threads, smem, st>>>(xb, wg, bias, T, dm.d, dm.E,
                                                                      dm.k, idx, w, probs);
    }
    return cuda_ok(cudaGetLastError()) ? MOE_OK : MOE_ERR_CUDA;
  }
  // about one CTA per SM: TM tokens per CTA, a multiple of 4 in [4, 128]
  int64_t per = (T + num_sms - 1) / num_sms;
  int TM = (int)((per + 3) / 4 * 4);
  if (TM < 4) TM = 4;
  if (TM > 128) TM = 128;
  const int NE = dm.E / 8;
  while (TM > 4 && (TM / 4) * NE > MAX_THREADS) TM -= 4;
  auto r32 = [](int v) { return (v + 31) / 32 * 32; };
  int threads = r32((TM / 4) * NE);
  // every thread's share of a chunk must fit its MAXV prefetch registers
  while (threads < MAX_THREADS &&
         (TM * (KC / 8) > MAXV * threads || dm.E * (KC / 4) > MAXV * threads))
    threads += 32;
  if (TM * (KC / 8) > MAXV * threads || dm.E * (KC / 4) > MAXV * threads)
    return MOE_ERR_UNSUPPORTED_SHAPE;
  const size_t stage_bytes = 2 * sizeof(float) * KC * (TM + dm.E);
  const size_t logit_bytes = sizeof(float) * (size_t)TM * dm.E;
  const size_t smem = stage_bytes > logit_bytes ? stage_bytes : logit_bytes;
  if (smem > 48 * 1024 &&
      !cuda_ok(cudaFuncSetAttribute(gate_topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    (int)smem)))
    return MOE_ERR_CUDA;
  const int64_t blocks = (T + TM - 1) / TM;
  gate_topk_kernel<<<(unsigned)blocks, threads, smem, st>>>(
      reinterpret_cast<const __nv_bfloat16*>(x), wg, bias, T, dm.d, dm.E, dm.k, TM, idx, w,
      probs);
  return cuda_ok(cudaGetLastError()) ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace moe
