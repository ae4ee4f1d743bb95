// permute.cu -- histogram / prefix-scan permutation into padded per-expert
// segments, and the device-built group table of the grouped GEMM.
//
// Passage: dots.llm1 Technical Report, §3.2 "Efficient implementation of
// Grouped GEMM" (each expert's token segment M_i is aligned to a fixed block,
// so a tile belongs to one expert) and §Architecture "Load balancing" (no
// token is dropped, so segments have no capacity limit).
//
// Deterministic and stable (tokens ascend inside a segment) without any
// dependence on atomic ordering:
//   1. hist:     each chunk of 1024 (t, j) assignments counts its experts.
//   2. groups:   one CTA turns the chunk counts into per-chunk bases (exclusive
//                scan over chunks per expert), pads each c_e to P, scans the
//                experts, and writes the group table, the tile prefix and the
//                heavy-first group order used by the weight-gradient GEMMs.
//   3. scatter:  each chunk ranks its assignments in order (warp match + per-
//                warp counts) and writes sorted_ids and row_of.
//   4. copy:     one warp per token reads x[t] once and writes its k rows.
//   5. pad rows of x_perm are zeroed.
// Steps 4 and 5 are skipped when no x_perm is asked for: the grouped GEMMs can
// gather the x rows themselves through sorted_ids.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "moe_internal.cuh"

namespace moe {
namespace {

constexpr int kScatterThreads = 256;

__global__ void hist_kernel(const int32_t* __restrict__ idx, int64_t n, int E,
                            int32_t* __restrict__ chunk_hist, int* header) {
  __shared__ int cnt[256];
  for (int e = threadIdx.x; e < E; e += blockDim.x) cnt[e] = 0;
  __syncthreads();
  const int64_t base = (int64_t)blockIdx.x * kChunk;
  for (int i = threadIdx.x; i < kChunk; i += blockDim.x) {
    const int64_t f = base + i;
    if (f < n) {
      const int e = idx[f];
      if (e >= 0 && e < E) {
        atomicAdd(&cnt[e], 1);
      } else {
        atomicCAS(header, 0, MOE_ERR_BAD_ROUTING);
        header[4] = 1;
      }
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) chunk_hist[(int64_t)blockIdx.x * E + e] = cnt[e];
}

// One CTA of 256 threads (E <= 256, G <= 264).  hist holds per-chunk counts
// [nchunks, E]; they are replaced by per-chunk exclusive bases.
__global__ void groups_kernel(int32_t* __restrict__ hist, int nchunks, int E, int S, int64_t T,
                              int P, int64_t Rr, int32_t* __restrict__ counts_out,
                              int32_t* __restrict__ offsets, GroupRec* __restrict__ groups,
                              int32_t* __restrict__ mtile_prefix, int32_t* __restrict__ order,
                              int* ws_header) {
  __shared__ int32_t s_pad[264];
  __shared__ int32_t s_scan[265];
  __shared__ int32_t s_mt[265];
  __shared__ int bad;
  const int G = E + S;
  const int tid = threadIdx.x;
  // hist_kernel raised header[4] if it saw an expert id outside [0, E)
  if (tid == 0) bad = ws_header[4] != 0;
  __syncthreads();
  int c = 0;
  if (tid < E) {
    // exclusive scan of this expert's chunk counts, 16 independent loads at a time
    int ch = 0;
    for (; ch + 16 <= nchunks; ch += 16) {
      int v[16];
#pragma unroll
      for (int u = 0; u < 16; ++u) v[u] = hist[(int64_t)(ch + u) * E + tid];
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        hist[(int64_t)(ch + u) * E + tid] = c;
        c += v[u];
      }
    }
    for (; ch < nchunks; ++ch) {
      const int v = hist[(int64_t)ch * E + tid];
      hist[(int64_t)ch * E + tid] = c;
      c += v;
    }
    if (c < 0) atomicExch(&bad, 1);
    if (counts_out) counts_out[tid] = c;
    s_pad[tid] = c > 0 ? (c + P - 1) / P * P : 0;
  }
  __syncthreads();
  if (tid == 0) {
    int64_t acc = 0;
    for (int e = 0; e < E; ++e) {
      s_scan[e] = (int32_t)acc;
      acc += s_pad[e];
    }
    if (acc > Rr) bad = 1;
    s_scan[E] = (int32_t)(acc > Rr ? Rr : acc);
    if (bad) atomicCAS(ws_header, 0, MOE_ERR_BAD_ROUTING);
  }
  __syncthreads();
  for (int e = tid; e <= E; e += blockDim.x) offsets[e] = s_scan[e];
  for (int g = tid; g < G; g += blockDim.x) {
    GroupRec r;
    if (g < E) {
      r.a_row = s_scan[g];
      r.out_row = s_scan[g];
      r.rows = bad ? 0 : c;
      r.rows_pad = bad ? 0 : s_pad[g];
    } else {
      r.a_row = 0;
      r.out_row = (int32_t)(Rr + (int64_t)(g - E) * T);
      r.rows = (int32_t)T;
      r.rows_pad = (int32_t)T;
    }
    groups[g] = r;  // (routed g < E <= 256 is handled by thread g, which holds c_g)
    s_mt[g] = (r.rows_pad + 255) / 256;  // 256-row tiles of the paired-CTA GEMM
    s_pad[g] = r.rows_pad;
  }
  __syncthreads();
  if (tid == 0) {
    int acc = 0;
    for (int g = 0; g < G; ++g) {
      mtile_prefix[g] = acc;
      acc += s_mt[g];
    }
    mtile_prefix[G] = acc;
    ws_header[1] = s_scan[E];
    ws_header[2] = acc;
    ws_header[3] = bad ? 0 : 1;  // routing valid: the scatter and copy may run
  }
  // heavy-first order: rank = #groups with more padded rows, ties by index
  for (int g = tid; g < G; g += blockDim.x) {
    const int mine = s_pad[g];
    int rank = 0;
    for (int h = 0; h < G; ++h) {
      const int o = s_pad[h];
      rank += (o > mine) || (o == mine && h < g);
    }
    order[rank] = g;
  }
}

// Chunk-ordered ranking: assignment f of chunk c goes to
//   offsets[e] + base[c][e] + (# earlier assignments of e inside the chunk).
__global__ void __launch_bounds__(kScatterThreads)
    scatter_kernel(const int32_t* __restrict__ idx, int64_t n, int k, int E,
                   const int32_t* __restrict__ chunk_base, const int32_t* __restrict__ offsets,
                   int32_t* __restrict__ sorted_ids, int32_t* __restrict__ row_of,
                   const int* header) {
  __shared__ int32_t running[256];
  __shared__ int32_t wcnt[kScatterThreads / 32][256];
  if (header[3] != 1) {
    // the group table flagged the routing as invalid: no pick gets a row, and
    // row_of says so (-1), so no later call follows a stale index
    const int64_t base = (int64_t)blockIdx.x * kChunk;
    for (int i = threadIdx.x; i < kChunk; i += kScatterThreads)
      if (base + i < n) row_of[base + i] = -1;
    return;
  }
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  for (int e = tid; e < E; e += kScatterThreads) running[e] = 0;
  for (int i = tid; i < (kScatterThreads / 32) * 256; i += kScatterThreads) (&wcnt[0][0])[i] = 0;
  __syncthreads();
  const int64_t base = (int64_t)blockIdx.x * kChunk;
  const unsigned lt = (1u << lane) - 1u;
  for (int round = 0; round < kChunk / kScatterThreads; ++round) {
    const int64_t f = base + round * kScatterThreads + tid;
    int e = f < n ? idx[f] : -1;
    const bool valid = e >= 0 && e < E;
    if (!valid) e = -1 - lane;  // unique per lane, never a real expert
    const unsigned same = __match_any_sync(0xffffffffu, e);
    const int rank_w = __popc(same & lt);
    const bool leader = (same & lt) == 0;
    if (valid && leader) wcnt[warp][e] = __popc(same);
    __syncthreads();
    if (valid) {
      int before = 0;
      for (int w = 0; w < warp; ++w) before += wcnt[w][e];
      const int32_t pos = offsets[e] + chunk_base[(int64_t)blockIdx.x * E + e] + running[e] +
                          before + rank_w;
      sorted_ids[pos] = (int32_t)(f / k);
      row_of[f] = pos;
    }
    __syncthreads();
    for (int ee = tid; ee < E; ee += kScatterThreads) {
      int add = 0;
      for (int w = 0; w < kScatterThreads / 32; ++w) {
        add += wcnt[w][ee];
        wcnt[w][ee] = 0;
      }
      running[ee] += add;
    }
    __syncthreads();
  }
}

// One warp per token: x[t] is read once and written to its k routed rows.  The
// last E * kPadSplit CTAs zero the segments' pad rows meanwhile (no launch of
// their own).
__global__ void copy_rows_kernel(const uint4* __restrict__ x, int64_t T, int row_vec, int k,
                                 const int32_t* __restrict__ row_of, uint4* __restrict__ x_perm,
                                 int* header, const GroupRec* __restrict__ groups, int E,
                                 int64_t Rr) {
  if (header[3] != 1) return;
  const unsigned tok_blocks = gridDim.x - (unsigned)E * kPadSplit;
  if (blockIdx.x >= tok_blocks) {
    const int pb = (int)(blockIdx.x - tok_blocks);
    zero_group_pad_rows(groups, pb / kPadSplit, pb % kPadSplit, row_vec, x_perm, Rr, header);
    return;
  }
  const int64_t t = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (t >= T) return;
  int32_t rows[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) rows[j] = j < k ? row_of[t * k + j] : 0;
  const uint4* src = x + t * row_vec;
  for (int c = lane; c < row_vec; c += 128) {
    uint4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u)
      if (c + 32 * u < row_vec) v[u] = src[c + 32 * u];
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      if (j < k) {
        uint4* dst = x_perm + (int64_t)rows[j] * row_vec;
#pragma unroll
        for (int u = 0; u < 4; ++u)
          if (c + 32 * u < row_vec) dst[c + 32 * u] = v[u];
      }
    }
  }
}

// Generic version for k > 16 (rows read from row_of on the fly).
__global__ void copy_rows_kernel_bigk(const uint4* __restrict__ x, int64_t T, int row_vec, int k,
                                      const int32_t* __restrict__ row_of,
                                      uint4* __restrict__ x_perm, int* header,
                                      const GroupRec* __restrict__ groups, int E, int64_t Rr) {
  if (header[3] != 1) return;
  const unsigned tok_blocks = gridDim.x - (unsigned)E * kPadSplit;
  if (blockIdx.x >= tok_blocks) {
    const int pb = (int)(blockIdx.x - tok_blocks);
    zero_group_pad_rows(groups, pb / kPadSplit, pb % kPadSplit, row_vec, x_perm, Rr, header);
    return;
  }
  const int64_t t = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (t >= T) return;
  const uint4* src = x + t * row_vec;
  for (int c = lane; c < row_vec; c += 32) {
    const uint4 v = src[c];
    for (int j = 0; j < k; ++j) x_perm[(int64_t)row_of[t * k + j] * row_vec + c] = v;
  }
}

}  // namespace

static int launch_groups(const moe_dims& dm, int32_t* hist, int nchunks, int32_t* counts,
                         int32_t* offsets, void* ws, cudaStream_t st) {
  const WsLayout L = ws_layout(dm);
  uint8_t* wsb = reinterpret_cast<uint8_t*>(ws);
  groups_kernel<<<1, 256, 0, st>>>(hist, nchunks, dm.E, dm.S, dm.T, dm.P, rows_routed(dm), counts,
                                   offsets, reinterpret_cast<GroupRec*>(wsb + L.groups),
                                   reinterpret_cast<int32_t*>(wsb + L.mtile_prefix),
                                   reinterpret_cast<int32_t*>(wsb + L.dw_order),
                                   reinterpret_cast<int*>(wsb));
  return cuda_ok(cudaGetLastError()) ? MOE_OK : MOE_ERR_CUDA;
}

int launch_permute(const moe_dims& dm, const int32_t* idx, const void* x, int32_t* counts,
                   int32_t* offsets, int32_t* sorted_ids, int32_t* row_of, void* x_perm, void* ws,
                   void* stream) {
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const WsLayout L = ws_layout(dm);
  uint8_t* wsb = reinterpret_cast<uint8_t*>(ws);
  int* status = reinterpret_cast<int*>(wsb);
  int32_t* hist = reinterpret_cast<int32_t*>(wsb + L.chunk_hist);
  const int64_t n = dm.T * dm.k;
  const int64_t Rr = rows_routed(dm);

  if (!cuda_ok(cudaMemsetAsync(sorted_ids, 0xFF, sizeof(int32_t) * Rr, st)) ||
      !cuda_ok(cudaMemsetAsync(wsb + 3 * sizeof(int), 0, kHeaderClearBytes, st)))
    return MOE_ERR_CUDA;
  if (n > 0) {
    hist_kernel<<<L.nchunks, 256, 0, st>>>(idx, n, dm.E, hist, status);
  } else if (!cuda_ok(cudaMemsetAsync(hist, 0, sizeof(int32_t) * dm.E, st))) {
    return MOE_ERR_CUDA;
  }
  int rc = launch_groups(dm, hist, L.nchunks, counts, offsets, ws, st);
  if (rc != MOE_OK) return rc;
  if (n == 0) return MOE_OK;
  scatter_kernel<<<L.nchunks, kScatterThreads, 0, st>>>(idx, n, dm.k, dm.E, hist, offsets,
                                                        sorted_ids, row_of, status);
  if (x_perm == nullptr)  // routing tables only: the GEMMs gather x rows themselves
    return cuda_ok(cudaGetLastError()) ? MOE_OK : MOE_ERR_CUDA;
  const int row_vec = dm.d / 8;
  const int warps = 8;
  // one warp per token, then E * kPadSplit CTAs for the pad rows
  const unsigned blocks = (unsigned)((dm.T + warps - 1) / warps + (int64_t)dm.E * kPadSplit);
  const GroupRec* groups = reinterpret_cast<const GroupRec*>(wsb + L.groups);
  if (dm.k <= 16)
    copy_rows_kernel<<<blocks, warps * 32, 0, st>>>(reinterpret_cast<const uint4*>(x), dm.T,
                                                    row_vec, dm.k, row_of,
                                                    reinterpret_cast<uint4*>(x_perm), status,
                                                    groups, dm.E, Rr);
  else
    copy_rows_kernel_bigk<<<blocks, warps * 32, 0, st>>>(reinterpret_cast<const uint4*>(x), dm.T,
                                                         row_vec, dm.k, row_of,
                                                         reinterpret_cast<uint4*>(x_perm), status,
                                                         groups, dm.E, Rr);
  return cuda_ok(cudaGetLastError()) ? MOE_OK : MOE_ERR_CUDA;
}

int launch_set_groups(const moe_dims& dm, const int32_t* counts, int32_t* offsets, void* ws,
                      void* stream) {
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const WsLayout L = ws_layout(dm);
  uint8_t* wsb = reinterpret_cast<uint8_t*>(ws);
  int32_t* hist = reinterpret_cast<int32_t*>(wsb + L.chunk_hist);
  if (!cuda_ok(cudaMemcpyAsync(hist, counts, sizeof(int32_t) * dm.E, cudaMemcpyDeviceToDevice,
                               st)) ||
      !cuda_ok(cudaMemsetAsync(wsb + 3 * sizeof(int), 0, kHeaderClearBytes, st)))
    return MOE_ERR_CUDA;
  return launch_groups(dm, hist, 1, nullptr, offsets, ws, st);
}

// Zero the pad rows of a routed-space bf16 matrix with `cols` columns.

}  // namespace moe
