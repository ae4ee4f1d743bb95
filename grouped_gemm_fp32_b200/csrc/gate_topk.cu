// gate_topk.cu -- FP32 gate and aux-loss-free top-k routing.
//
// Passage: dots.llm1 Technical Report, §Architecture "Mixture of Experts layer"
// (the gating layer is computed in FP32 rather than BF16, for stable and
// accurate expert selection; each token picks its top-6 of 128 routed experts)
// and "Load balancing" (a per-expert bias is added to the affinity scores only
// to decide the top-k routing).
//
// The logits X Wg^T are a dense [T, d] x [d, E] contraction, so they run on the
// tensor cores, without giving up FP32 accuracy:
//   * X is bf16, an exact tcgen05 kind::f16 operand;
//   * every FP32 gate weight is split into three bf16 terms, w = hi + mid + lo
//     with hi = bf16(w), mid = bf16(w - hi), lo = bf16(w - hi - mid).  Both
//     differences are exact in FP32, and what the three terms miss is below
//     2^-24 |w|, under FP32's own rounding of w;
//   * a product of two bf16 values is exact in FP32;
//   * the tensor cores' FP32 accumulation is not round-to-nearest: measured on
//     the layer workload, one accumulator over all of d = 4096 drifts ~10x
//     further from the exact logits than an FP32 FMA loop.  So each 64-wide K
//     block accumulates from zero in tensor memory (12 MMAs over small partial
//     sums; with E_pad <= 128 the hi products in one set of columns and the mid
//     and lo products in another), and the block results are added in FP32
//     registers with round-to-nearest; the truncations of different blocks then
//     have random signs and the logits match an FP32 FMA loop's accuracy.
//
// split_wg_kernel writes the three planes [3][E_pad][d] (bf16, rows E..E_pad-1
// zero) into the layer workspace.  gate_tc_kernel, one CTA per 128 tokens:
//   warp 0, lane 0   TMA producer: per 64-wide K block the 128 x 64 tile of X
//                    and the three E_pad x 64 tiles of the planes, 128-byte swizzle
//   warp 1           tensor-memory owner; lane 0 issues, per K block, 12 MMAs
//                    (four 16-wide K steps x hi, mid, lo; M = 128, N = E_pad) into
//                    one of two E_pad-column accumulators, alternating.  With
//                    E_pad <= 128 the hi and mid tiles, consecutive in shared memory,
//                    form one N = 2 E_pad operand: 8 MMAs, x.hi in the accumulator's
//                    first E_pad columns and x.mid + x.lo in the next E_pad, which the
//                    summing warps add (a third fewer MMAs, and X read twice instead
//                    of three times per K step)
//   warps 2..9       summing warps (two per tensor-memory lane quarter, one column
//                    half each): add each finished block accumulator into FP32
//                    registers, then write the logits to shared memory
//   all warps        routing, eight lanes per token (four tokens per warp at a
//                    time): softmax (max-subtracted, expf), s = p + bias, k rounds of
//                    a shuffle arg-max within the token's lanes (equal s -> lower
//                    index), the renormalised weights
// With fewer 128-token tiles than half the SMs (T <= 9472 on 148 SMs) each tile
// runs on a cluster pair instead: CTA 0 takes the first half of the K blocks,
// CTA 1 the second, and after an exchange of partial logits through distributed
// shared memory each CTA routes 64 of the tokens.  The kernel is bound by the
// latency of its K-block chain, so halving the chain halves its time; the two
// halves are added once, low + high, the same FP32 sum in both CTAs.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "moe_internal.cuh"
#include "sm100.cuh"

namespace moe {
namespace {

constexpr int GT_BM = 128;                    // tokens per CTA (UMMA M)
constexpr int GT_BK = 64;                     // K per stage: one 128-byte swizzle row
constexpr int GT_SUM_WARPS = 8;                // two per tensor-memory lane quarter
constexpr int GT_THREADS = 64 + 32 * GT_SUM_WARPS;
constexpr int GT_MAX_STAGES = 6;
constexpr int GT_A_BYTES = GT_BM * GT_BK * 2;  // 16 KB
constexpr int GT_MAX_SMEM = 232448;            // 227 KB

struct GateArgs {
  int* status;
  const float* bias;
  int32_t* topk_idx;
  float* topk_w;
  float* probs;
  int64_t T;
  int d, E, e_pad, k, stages;
  uint32_t stage_bytes, tmem_cols, idesc, idesc2;
  uint64_t budget_ns;
};

struct GateCtl {
  uint64_t full[GT_MAX_STAGES];
  uint64_t empty[GT_MAX_STAGES];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};

// Routing of the TM tokens whose logits sit in shared memory, row r at L + r * LS:
// eight lanes per token, four tokens per warp at a time (lane l of a token's group
// holds experts l, l + 8, ..., EPL of them).  Softmax with the max subtracted, s = p
// + bias, then k rounds of an arg-max over the group (equal s -> lower index; a NaN
// score ranks as -inf), the chosen affinities renormalised.  A group reduction is
// three shuffle steps, and a warp has 3-4 rounds of four tokens in a 128-token tile
// instead of 13 tokens one after another.
template <int EPL>
__device__ __forceinline__ void route_tile(const float* L, int LS, int64_t t0, int TM, int64_t T,
                                           int E, int k, const float* __restrict__ bias,
                                           int32_t* __restrict__ topk_idx,
                                           float* __restrict__ topk_w, float* __restrict__ probs) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarps = blockDim.x >> 5;
  const int gl = lane & 7;  // this lane's place in its token's group
  for (int rb = 4 * warp; rb < TM; rb += 4 * nwarps) {
    const int r = rb + (lane >> 3);
    const int64_t t = t0 + r;
    const bool active = r < TM && t < T;  // idle groups still join the shuffles
    float p[EPL], s[EPL];
    float m = -INFINITY;
#pragma unroll
    for (int q = 0; q < EPL; ++q) {
      const int e = gl + 8 * q;
      p[q] = (active && e < E) ? L[r * LS + e] : -INFINITY;
      m = fmaxf(m, p[q]);
    }
#pragma unroll
    for (int o = 4; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    float z = 0.0f;
#pragma unroll
    for (int q = 0; q < EPL; ++q) {
      const int e = gl + 8 * q;
      p[q] = (active && e < E) ? expf(p[q] - m) : 0.0f;
      z += p[q];
    }
#pragma unroll
    for (int o = 4; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
    const float inv = 1.0f / z;
    uint32_t alive = 0;  // experts this lane may still pick (a bit per q)
#pragma unroll
    for (int q = 0; q < EPL; ++q) {
      const int e = gl + 8 * q;
      const bool valid = active && e < E;
      p[q] = valid ? p[q] * inv : 0.0f;
      s[q] = valid ? p[q] + (bias ? bias[e] : 0.0f) : -INFINITY;
      if (s[q] != s[q]) s[q] = -INFINITY;  // a NaN score ranks last (ties by index)
      if (valid && probs) probs[t * E + e] = p[q];
      if (valid) alive |= 1u << q;
    }
    float psel = 0.0f;
    for (int j = 0; j < k; ++j) {
      // lane-local best: larger s, then lower index (q ascending = index ascending).  The
      // first live expert is taken before any comparison, so even non-finite inputs
      // yield k distinct, valid experts.
      float bs = -INFINITY, bp = 0.0f;
      int be = 0x7fffffff;
#pragma unroll
      for (int q = 0; q < EPL; ++q) {
        if (((alive >> q) & 1u) && (be == 0x7fffffff || s[q] > bs)) {
          bs = s[q];
          be = gl + 8 * q;
          bp = p[q];
        }
      }
#pragma unroll
      for (int o = 4; o > 0; o >>= 1) {
        const float os = __shfl_xor_sync(0xffffffffu, bs, o);
        const int oe = __shfl_xor_sync(0xffffffffu, be, o);
        const float op = __shfl_xor_sync(0xffffffffu, bp, o);
        if (oe != 0x7fffffff && (be == 0x7fffffff || os > bs || (os == bs && oe < be))) {
          bs = os;
          be = oe;
          bp = op;
        }
      }
#pragma unroll
      for (int q = 0; q < EPL; ++q)
        if (gl + 8 * q == be) alive &= ~(1u << q);  // remove the winner
      psel += bp;
      if (gl == 0 && active) {
        topk_idx[t * k + j] = be;
        topk_w[t * k + j] = bp;
      }
    }
    __syncwarp();
    const float rn = 1.0f / psel;
    if (active)
      for (int j = gl; j < k; j += 8) topk_w[t * k + j] *= rn;
    __syncwarp();
  }
}

// wg [E, d] f32 -> planes [3][e_pad][d] bf16: hi, mid, lo with hi + mid + lo = w
// to below 2^-24 |w| (rows E..e_pad-1 are zero).  Four columns per thread.
__global__ void split_wg_kernel(const float* __restrict__ wg, int E, int e_pad, int d,
                                __nv_bfloat16* __restrict__ planes) {
  const int64_t n4 = (int64_t)e_pad * d / 4;
  const int64_t plane = (int64_t)e_pad * d;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t e = i * 4 / d;
    float4 w = make_float4(0.f, 0.f, 0.f, 0.f);
    if (e < E) w = reinterpret_cast<const float4*>(wg)[i];
    const float v[4] = {w.x, w.y, w.z, w.w};
    uint32_t hi[2], mid[2], lo[2];
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      __nv_bfloat16 h[2], m[2], l[2];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const float f = v[2 * c + u];
        h[u] = __float2bfloat16_rn(f);
        const float r1 = f - __bfloat162float(h[u]);  // exact
        m[u] = __float2bfloat16_rn(r1);
        const float r2 = r1 - __bfloat162float(m[u]);  // exact
        l[u] = __float2bfloat16_rn(r2);
      }
      __nv_bfloat162 ph = __halves2bfloat162(h[0], h[1]);
      __nv_bfloat162 pm = __halves2bfloat162(m[0], m[1]);
      __nv_bfloat162 pl = __halves2bfloat162(l[0], l[1]);
      hi[c] = *reinterpret_cast<uint32_t*>(&ph);
      mid[c] = *reinterpret_cast<uint32_t*>(&pm);
      lo[c] = *reinterpret_cast<uint32_t*>(&pl);
    }
    *reinterpret_cast<uint2*>(planes + i * 4) = make_uint2(hi[0], hi[1]);
    *reinterpret_cast<uint2*>(planes + plane + i * 4) = make_uint2(mid[0], mid[1]);
    *reinterpret_cast<uint2*>(planes + 2 * plane + i * 4) = make_uint2(lo[0], lo[1]);
  }
}

// SPLIT: two CTAs of a cluster share one 128-token tile, CTA 0 taking the first
// half of the K blocks and CTA 1 the second; each then adds the two partial
// logits (low half + high half, the same FP32 sum in both) for 64 of the tokens
// and routes them.  Used when one CTA per tile would leave most SMs idle.
// PAIRED (E_pad <= 128): the hi and mid planes go through one N = 2 E_pad MMA, and each
// summing thread keeps two 32-column groups of its row (four otherwise).
template <bool SPLIT, bool PAIRED>
__global__ void __launch_bounds__(GT_THREADS, 1)
    gate_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                   const GateArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  GateCtl* ctl = reinterpret_cast<GateCtl*>(smem + (size_t)a.stages * a.stage_bytes);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t crank = SPLIT ? cluster_ctarank() : 0u;
  const int64_t m0 = (int64_t)(SPLIT ? (blockIdx.x >> 1) : blockIdx.x) * GT_BM;
  const int nkb_all = a.d / GT_BK;
  const int kb0 = (SPLIT && crank) ? nkb_all / 2 : 0;  // this CTA's K blocks [kb0, kb0 + nkb)
  const int nkb = SPLIT ? (crank ? nkb_all - nkb_all / 2 : nkb_all / 2) : nkb_all;
  const uint32_t plane_bytes = (uint32_t)a.e_pad * GT_BK * 2;
  const int acc_cols = PAIRED ? 2 * a.e_pad : a.e_pad;  // columns of one block accumulator
  constexpr int NI = PAIRED ? 2 : 4;                     // column groups a summing thread keeps
  volatile int* abort_flag = &ctl->abort_flag;

  if (threadIdx.x == 0) {
    for (int s = 0; s < a.stages; ++s) {
      mbar_init(&ctl->full[s], 1);
      mbar_init(&ctl->empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&ctl->tfull[b], 1);
      mbar_init(&ctl->tempty[b], GT_SUM_WARPS);
    }
    mbar_init(&ctl->drain, 1);
    ctl->abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmX);
    tma_prefetch_desc(&tmW);
  }
  if (warp == 1) {
    tmem_alloc(&ctl->tmem_base, a.tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = ctl->tmem_base;
  // waits for work already started (copies in flight, MMAs issued) get a long
  // budget of their own, so the CTA never frees tensor memory or exits under them
  const uint64_t drain_budget = a.budget_ns > 2000000000ull ? a.budget_ns : 2000000000ull;

  // Logits of this thread's row, in registers: 32-column groups g = 2 i + h of the
  // accumulator (h = this warp's column half), summed over the K blocks.
  float sum[NI][32];
  const int ngroups = a.e_pad / 32;
  const int q = warp & 3;             // tensor-memory lane quarter of a summing warp
  const int h = (warp - 2) >> 2;      // its column half
  const int row = q * 32 + lane;

  if (warp == 0) {
    // ------------------------------------------------------------ producer --
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0, issued = 0, lastpar = 0;
      for (int kb = 0; kb < nkb; ++kb) {
        if (!mbar_wait(&ctl->empty[stage], phase ^ 1, abort_flag, a.status,
                       MOE_ERR_DEVICE_TIMEOUT, a.budget_ns))
          break;
        mbar_arrive_expect_tx(&ctl->full[stage], GT_A_BYTES + 3 * plane_bytes);
        uint8_t* st = smem + (size_t)stage * a.stage_bytes;
        const int k0 = (kb0 + kb) * GT_BK;
        tma_load_2d(st, &tmX, &ctl->full[stage], k0, (int32_t)m0);  // rows past T read as zero
#pragma unroll
        for (int j = 0; j < 3; ++j)
          tma_load_2d(st + GT_A_BYTES + j * plane_bytes, &tmW, &ctl->full[stage], k0,
                      j * a.e_pad);
        issued |= 1u << stage;
        lastpar = (lastpar & ~(1u << stage)) | (phase << stage);
        if (++stage == a.stages) {
          stage = 0;
          phase ^= 1;
        }
      }
      // after an abort, stages may hold copies nobody consumed: let them land
      if (*abort_flag)
        for (int s = 0; s < a.stages; ++s)
          if (issued & (1u << s)) {
            volatile int never = 0;
            mbar_wait(&ctl->full[s], (lastpar >> s) & 1u, &never, a.status,
                      MOE_ERR_DEVICE_TIMEOUT, drain_budget);
          }
    }
  } else if (warp == 1) {
    // --------------------------------------------------------- MMA issuer --
    // K block kb accumulates, from zero, into accumulator kb % 2; the summing
    // warps add it to their FP32 registers and hand it back.
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      for (int kb = 0; kb < nkb; ++kb) {
        const int acc = kb & 1;
        const uint32_t use = (uint32_t)(kb >> 1);
        if (!mbar_wait(&ctl->tempty[acc], (use & 1u) ^ 1u, abort_flag, a.status,
                       MOE_ERR_DEVICE_TIMEOUT, a.budget_ns))
          break;
        if (!mbar_wait(&ctl->full[stage], phase, abort_flag, a.status, MOE_ERR_DEVICE_TIMEOUT,
                       a.budget_ns))
          break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * acc_cols);
        const uint32_t a_base = smem_u32(smem + (size_t)stage * a.stage_bytes);
        const uint32_t b_base = a_base + GT_A_BYTES;
#pragma unroll
        for (int kk = 0; kk < GT_BK / 16; ++kk) {
          const uint64_t ad = smem_desc_sw128(a_base + kk * 32, 16, 1024);
          if constexpr (PAIRED) {
            // the hi and mid planes are consecutive E_pad-row tiles: one N = 2 E_pad MMA
            // puts x.hi in columns [0, E_pad) and x.mid in [E_pad, 2 E_pad); x.lo is added
            // to the mid columns
            const uint64_t b01 = smem_desc_sw128(b_base + kk * 32, 16, 1024);
            const uint64_t b2 = smem_desc_sw128(b_base + 2 * plane_bytes + kk * 32, 16, 1024);
            umma_f16(d_tmem, ad, b01, a.idesc2, kk != 0 ? 1u : 0u);
            umma_f16(d_tmem + (uint32_t)a.e_pad, ad, b2, a.idesc, 1u);
          } else {
#pragma unroll
            for (int j = 0; j < 3; ++j) {
              const uint64_t bd = smem_desc_sw128(b_base + j * plane_bytes + kk * 32, 16, 1024);
              umma_f16(d_tmem, ad, bd, a.idesc, (kk | j) != 0 ? 1u : 0u);
            }
          }
        }
        umma_commit(&ctl->empty[stage]);
        umma_commit(&ctl->tfull[acc]);
        if (++stage == a.stages) {
          stage = 0;
          phase ^= 1;
        }
      }
      // every MMA issued has completed before tensor memory is freed
      umma_commit(&ctl->drain);
      volatile int never = 0;
      mbar_wait(&ctl->drain, 0, &never, a.status, MOE_ERR_DEVICE_TIMEOUT, drain_budget);
    }
  } else {
    // ----------------------------------------------------- summing warps --
#pragma unroll
    for (int i = 0; i < NI; ++i)
#pragma unroll
      for (int j = 0; j < 32; ++j) sum[i][j] = 0.0f;
    for (int kb = 0; kb < nkb; ++kb) {
      const int acc = kb & 1;
      const uint32_t use = (uint32_t)(kb >> 1);
      if (!mbar_wait(&ctl->tfull[acc], use & 1u, abort_flag, a.status, MOE_ERR_DEVICE_TIMEOUT,
                     a.budget_ns))
        break;
      __syncwarp();  // tcgen05.ld is warp-collective
      tc_fence_after();
      const uint32_t taddr = tmem_base + (uint32_t)(acc * acc_cols) + ((uint32_t)(q * 32) << 16);
#pragma unroll
      for (int i = 0; i < NI; ++i) {
        const int g = 2 * i + h;
        if (g < ngroups) {
          uint32_t r[32];
          tmem_ld32_sync(taddr + (uint32_t)(g * 32), r);
#pragma unroll
          for (int j = 0; j < 32; ++j) sum[i][j] += __uint_as_float(r[j]);
          if constexpr (PAIRED) {  // the block's mid + lo sums of the same experts
            tmem_ld32_sync(taddr + (uint32_t)(a.e_pad + g * 32), r);
#pragma unroll
            for (int j = 0; j < 32; ++j) sum[i][j] += __uint_as_float(r[j]);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl->tempty[acc]);
    }
  }
  __syncwarp();

  tc_fence_before();
  __syncthreads();  // every role is done: the stages are free, the abort flag is final
  const bool aborted = *abort_flag != 0;
  // Logits to shared memory, row stride E + 1 (odd): thread `lane` writing row
  // lane, column c hits bank (lane + c) % 32, so these stores are conflict-free.
  float* L = reinterpret_cast<float*>(smem);
  const int LS = a.E + 1;
  if (warp >= 2 && !aborted) {
#pragma unroll
    for (int i = 0; i < NI; ++i) {
      const int g = 2 * i + h;
      if (g < ngroups)
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (g * 32 + j < a.E) L[row * LS + g * 32 + j] = sum[i][j];
    }
  }
  __syncthreads();
  int r0 = 0, rows = GT_BM;
  if constexpr (SPLIT) {
    cluster_sync();  // both CTAs' partial logits are in shared memory
    r0 = (int)crank * (GT_BM / 2);
    rows = GT_BM / 2;
    if (!aborted) {
      const uint32_t peer = map_to_rank(L, crank ^ 1u);
      for (int i = threadIdx.x; i < rows * a.E; i += blockDim.x) {
        const int off = (r0 + i / a.E) * LS + i % a.E;
        L[off] = L[off] + ld_shared_cluster_f32(peer + (uint32_t)off * 4u);
      }
    }
    __syncthreads();
  }
  if (!aborted) {
    if (a.E <= 128)
      route_tile<16>(L + r0 * LS, LS, m0 + r0, rows, a.T, a.E, a.k, a.bias, a.topk_idx,
                     a.topk_w, a.probs);
    else
      route_tile<32>(L + r0 * LS, LS, m0 + r0, rows, a.T, a.E, a.k, a.bias, a.topk_idx,
                     a.topk_w, a.probs);
  }
  if constexpr (SPLIT) cluster_sync();  // the peer has read this CTA's partials
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, a.tmem_cols);
  }
}

}  // namespace

int launch_split_wg(const moe_dims& dm, const float* wg, void* planes, void* stream) {
  const int e_pad = (dm.E + 31) / 32 * 32;
  const int64_t n4 = (int64_t)e_pad * dm.d / 4;
  const int threads = 256;
  int64_t blocks = (n4 + threads - 1) / threads;
  if (blocks > 4096) blocks = 4096;
  split_wg_kernel<<<(unsigned)blocks, threads, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      wg, dm.E, e_pad, dm.d, reinterpret_cast<__nv_bfloat16*>(planes));
  return cuda_ok(cudaGetLastError()) ? MOE_OK : MOE_ERR_CUDA;
}

int launch_gate_topk(const moe_dims& dm, const void* x, const float* wg, const float* bias,
                     int32_t* idx, float* w, float* probs, void* ws, void* stream) {
  const int64_t T = dm.T;
  if (T == 0) return MOE_OK;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const WsLayout L = ws_layout(dm);
  uint8_t* wsb = reinterpret_cast<uint8_t*>(ws);
  __nv_bfloat16* planes = reinterpret_cast<__nv_bfloat16*>(wsb + L.gate_split);
  const int e_pad = L.e_pad;

  {
    const int rc = launch_split_wg(dm, wg, planes, stream);
    if (rc != MOE_OK) return rc;
  }

  GateArgs a{};
  a.status = reinterpret_cast<int*>(ws);
  a.bias = bias;
  a.topk_idx = idx;
  a.topk_w = w;
  a.probs = probs;
  a.T = T;
  a.d = dm.d;
  a.E = dm.E;
  a.e_pad = e_pad;
  a.k = dm.k;
  a.stage_bytes = (uint32_t)(GT_A_BYTES + 3 * e_pad * GT_BK * 2);  // a multiple of 1024
  const size_t fixed = 1024 /* alignment slack */ + sizeof(GateCtl);
  int stages = (int)((GT_MAX_SMEM - fixed) / a.stage_bytes);
  if (stages > GT_MAX_STAGES) stages = GT_MAX_STAGES;
  if (stages < 2) return MOE_ERR_UNSUPPORTED_SHAPE;
  a.stages = stages;
  // the logits tile [128][E + 1] f32 reuses the stage buffers
  if ((size_t)GT_BM * (dm.E + 1) * sizeof(float) > (size_t)stages * a.stage_bytes)
    return MOE_ERR_UNSUPPORTED_SHAPE;
  const bool paired = e_pad <= 128;
  uint32_t cols = 32;  // two accumulators of e_pad (paired: 2 e_pad) columns
  while (cols < (uint32_t)((paired ? 4 : 2) * e_pad)) cols <<= 1;
  a.tmem_cols = cols;
  a.idesc = idesc_bf16_f32(GT_BM, e_pad, false, false);
  a.idesc2 = idesc_bf16_f32(GT_BM, 2 * e_pad, false, false);
  a.budget_ns = wait_budget_ns();

  CUtensorMap mx{}, mw{};
  if (!make_map_bf16(&mx, x, T, dm.d, GT_BM) ||
      !make_map_bf16(&mw, planes, (int64_t)3 * e_pad, dm.d, e_pad))
    return MOE_ERR_CUDA;
  const size_t smem = fixed + (size_t)stages * a.stage_bytes;
  static bool attr_set = false;
  static int num_sms = 0;
  if (!attr_set) {
    if (!cuda_ok(cudaFuncSetAttribute(gate_tc_kernel<false, false>,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize, GT_MAX_SMEM)) ||
        !cuda_ok(cudaFuncSetAttribute(gate_tc_kernel<true, false>,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize, GT_MAX_SMEM)) ||
        !cuda_ok(cudaFuncSetAttribute(gate_tc_kernel<false, true>,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize, GT_MAX_SMEM)) ||
        !cuda_ok(cudaFuncSetAttribute(gate_tc_kernel<true, true>,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize, GT_MAX_SMEM)))
      return MOE_ERR_CUDA;
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&num_sms, cudaDevAttrMultiProcessorCount, dev);
    attr_set = true;
  }
  const int64_t tiles = (T + GT_BM - 1) / GT_BM;
  if (2 * tiles <= num_sms && a.d / GT_BK >= 2) {
    // fewer tiles than half the SMs: a CTA pair per tile, each on half of K
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(2 * tiles));
    cfg.blockDim = dim3(GT_THREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (!cuda_ok(cudaLaunchKernelEx(&cfg, paired ? gate_tc_kernel<true, true>
                                                 : gate_tc_kernel<true, false>,
                                    mx, mw, a)))
      return MOE_ERR_CUDA;
  } else if (paired) {
    gate_tc_kernel<false, true><<<(unsigned)tiles, GT_THREADS, smem, st>>>(mx, mw, a);
  } else {
    gate_tc_kernel<false, false><<<(unsigned)tiles, GT_THREADS, smem, st>>>(mx, mw, a);
  }
  return cuda_ok(cudaGetLastError()) ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace moe
