// moe_internal.cuh -- workspace layout and records shared by the kernels of
// libmoe.so (host and device).
#pragma once
#include <cstddef>
#include <cstdint>

#include <cuda.h>
#include <cuda_runtime.h>

#include "moe.h"  // include/ is on the include path

// MOE_DEBUG=1 (libmoe_debug.so): kernels that take the group table, the tile
// prefix or row indices from memory a caller could have overwritten validate
// them against the tensor extents before using them; a bad entry records
// MOE_ERR_BAD_ROUTING in the status word and its work is skipped.  Nothing traps.
#ifndef MOE_DEBUG
#define MOE_DEBUG 0
#endif

namespace moe {

// Records the error of a failing CUDA call for moe_last_cuda_error(); true on success.
bool cuda_ok(cudaError_t e);

// Argument and shape checks every entry point runs first (moe_api.cu): dims_ok
// is false for a null or non-positive shape; check_shape returns
// MOE_ERR_INVALID_ARG / MOE_ERR_UNSUPPORTED_SHAPE / MOE_OK for the shapes the
// kernels support (include/moe.h), need_bwd adding the backward's P % 64 == 0.
bool dims_ok(const moe_dims* dm);
int check_shape(const moe_dims* dm, bool need_bwd);

// One group of the grouped GEMM: a routed expert (g < E) or a shared expert.
//   a_row    first row of the group in its A source (x_perm for routed groups,
//            x for shared groups, i.e. 0)
//   out_row  first row of the group in the grouped row space [0, Rt)
//   rows     real rows (tokens) of the group
//   rows_pad rows rounded up to the pad block (shared groups: T)
struct GroupRec {
  int32_t a_row, out_row, rows, rows_pad;
};

constexpr int kPadSplit = 8;  // CTAs per routed group zeroing its pad rows

#ifdef __CUDACC__
// Zero the pad rows [out_row + rows, out_row + rows_pad) of routed group e of a
// bf16 matrix [Rr, row_vec * 8]; this CTA is part `part` of kPadSplit CTAs on the
// group.  The debug build reports a record outside the routed rows instead of
// following it.
__device__ __forceinline__ void zero_group_pad_rows(const GroupRec* __restrict__ groups, int e,
                                                    int part, int row_vec, uint4* __restrict__ m,
                                                    int64_t Rr, int* status) {
  const GroupRec g = groups[e];
  const int64_t r0 = (int64_t)g.out_row + g.rows, r1 = (int64_t)g.out_row + g.rows_pad;
  if (MOE_DEBUG && (g.out_row < 0 || g.rows < 0 || r0 > r1 || r1 > Rr)) {
    if (threadIdx.x == 0) atomicCAS(status, 0, MOE_ERR_BAD_ROUTING);
    return;
  }
  const int64_t n = (r1 - r0) * row_vec;
  const uint4 z = make_uint4(0, 0, 0, 0);
  for (int64_t i = (int64_t)part * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)kPadSplit * blockDim.x)
    m[r0 * row_vec + i] = z;
}
#endif

constexpr int kChunk = 1024;      // routed assignments per histogram chunk
constexpr int kHeaderWords = 16;  // [0] status, [1] padded routed total, [2] tiles total,
                                  // [3] routing valid, [4] bad expert id seen,
                                  // [5 + mode] tile counter of each grouped-GEMM mode
constexpr int kTileCtrWord = 5;
// what each routing call clears: header words 3 (routing valid) to 10 (the last
// tile counter); a counter left past 0 by a launch that was cut short starts the
// next step at 0 again
constexpr size_t kHeaderClearBytes = (kTileCtrWord + 6 - 3) * sizeof(int32_t);

// Layer workspace: the routing tables first (`bytes` of them), then the
// gate's split weights, then the router backward's scratch.
struct WsLayout {
  size_t groups;        // GroupRec[G]
  size_t mtile_prefix;  // int32[G + 1]  prefix of ceil(rows_pad / 256) (pair tiles)
  size_t dw_order;      // int32[G]      groups by padded rows, largest first
  size_t chunk_hist;    // int32[nchunks * E]
  size_t bytes;         // end of the routing tables
  size_t gate_split;    // bf16[3][e_pad][d]  the gate weights as hi, mid, lo planes
  size_t dl_planes;     // bf16[3][t_pad][e_pad]  dL/dlogit as hi, mid, lo planes
  size_t gdw_part;      // f32[gdw_splits][e_pad][d]  split-K partial sums of dWg
  size_t seqbal;        // sequence-wise balance loss: f32[sb_chunks][E] affinity sums,
                        // then int32[sb_chunks][E] pick counts
  size_t total;         // whole workspace
  int nchunks;
  int e_pad;            // E rounded up to a multiple of 32
  int t_pad;            // T rounded up to a multiple of 128
  int gdw_splits;       // K splits of the dWg GEMM
  int sb_chunks;        // token chunks (of <= kSeqChunk, inside one sequence) the
                        // balance loss can need: sequences of >= kSeqMin tokens
};

constexpr int kSeqChunk = 64;  // tokens per chunk of the balance loss's column sums
constexpr int kSeqMin = 128;   // shortest sequence the balance loss accepts

// K splits of the dWg GEMM: as many work items as fit one wave on a B200's 148
// SMs, at most 16 splits, and no split left empty.
inline int gdw_splits_of(int e_pad, int d, int t_pad) {
  const int tiles = ((e_pad + 127) / 128) * ((d + 255) / 256);
  const int kb = 3 * (t_pad / 64);
  if (kb == 0) return 1;
  int s = 148 / tiles;
  if (s < 1) s = 1;
  if (s > 16) s = 16;
  if (s > kb) s = kb;
  const int per = (kb + s - 1) / s;
  return (kb + per - 1) / per;
}

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

inline WsLayout ws_layout(const moe_dims& dm) {
  WsLayout L;
  const int G = dm.E + dm.S;
  const int64_t assignments = dm.T * dm.k;
  L.nchunks = (int)((assignments + kChunk - 1) / kChunk);
  if (L.nchunks < 1) L.nchunks = 1;
  size_t off = kHeaderWords * sizeof(int32_t);
  L.groups = off = align_up(off, 16);
  off += sizeof(GroupRec) * G;
  L.mtile_prefix = off = align_up(off, 16);
  off += sizeof(int32_t) * (G + 1);
  L.dw_order = off = align_up(off, 16);
  off += sizeof(int32_t) * G;
  L.chunk_hist = off = align_up(off, 16);
  off += sizeof(int32_t) * (size_t)L.nchunks * dm.E;
  L.bytes = align_up(off, 256);
  L.e_pad = (dm.E + 31) / 32 * 32;
  L.t_pad = (int)((dm.T + 127) / 128 * 128);
  L.gdw_splits = gdw_splits_of(L.e_pad, dm.d, L.t_pad);
  L.gate_split = align_up(L.bytes, 1024);
  L.dl_planes = align_up(L.gate_split + (size_t)3 * L.e_pad * dm.d * 2, 1024);
  L.gdw_part = align_up(L.dl_planes + (size_t)3 * L.t_pad * L.e_pad * 2, 1024);
  // chunks of sequences of L >= kSeqMin >= kSeqChunk tokens:
  // sum_s ceil(L_s / kSeqChunk) <= T / kSeqChunk + n_seq <= 2 ceil(T / kSeqChunk)
  L.sb_chunks = (int)(2 * ((dm.T + kSeqChunk - 1) / kSeqChunk)) + 1;
  L.seqbal = align_up(L.gdw_part + (size_t)L.gdw_splits * L.e_pad * dm.d * 4, 256);
  L.total = align_up(L.seqbal + (size_t)L.sb_chunks * dm.E * 8, 256);
  return L;
}

inline int64_t rows_routed(const moe_dims& dm) {
  return dm.rows_cap > 0 ? dm.rows_cap : dm.T * dm.k + (int64_t)dm.E * (dm.P - 1);
}
inline int64_t rows_total(const moe_dims& dm) { return rows_routed(dm) + (int64_t)dm.S * dm.T; }

// Launch helpers implemented in the .cu files (all return a moe_status).
int launch_gate_topk(const moe_dims& dm, const void* x, const float* wg, const float* bias,
                     int32_t* idx, float* w, float* probs, void* ws, void* stream);
int launch_permute(const moe_dims& dm, const int32_t* idx, const void* x, int32_t* counts,
                   int32_t* offsets, int32_t* sorted_ids, int32_t* row_of, void* x_perm, void* ws,
                   void* stream);
int launch_set_groups(const moe_dims& dm, const int32_t* counts, int32_t* offsets, void* ws,
                      void* stream);
int launch_split_wg(const moe_dims& dm, const float* wg, void* planes, void* stream);
int launch_router_bwd(const moe_dims& dm, const void* x, const float* wg, const float* probs,
                      const int32_t* idx, const float* w, const float* dw,
                      const float* seq_grad, int64_t seq_len, float* dlogits, void* dx,
                      float* dwg, int accumulate, void* ws, void* stream);
int launch_bias_update(const moe_dims& dm, const int32_t* counts, float gamma,
                       const float* bias_in, float* bias_out, void* stream);
int launch_seq_balance(const moe_dims& dm, int64_t seq_len, float alpha, const int32_t* idx,
                       const float* probs, float* loss, float* seq_grad, void* ws, void* stream);
// Router-backward GEMMs (sgemm.cu); planes and partial sums live in the workspace.
int launch_gate_dx(const moe_dims& dm, const void* dl_planes, const void* wg_planes, void* dx,
                   int* status, void* stream);
int launch_gate_dw(const moe_dims& dm, const void* dl_planes, const void* x, float* partial,
                   int* status, void* stream);
int launch_combine(const moe_dims& dm, const void* y, const void* y_shared,
                   const int32_t* row_of, const float* w, void* out, bool f32_out, void* stream);
int launch_combine_bwd(const moe_dims& dm, const void* ws, const void* dout, const void* y,
                       const int32_t* row_of, const float* w, void* dy, float* dw, void* stream);

enum GemmMode { MODE_FWD1 = 0, MODE_FWD2, MODE_DX2, MODE_DX1, MODE_DW2, MODE_DW1 };

// Operand set of one grouped GEMM call (device pointers).
struct GemmOperands {
  const void* a0;  // A source (routed rows / grouped row space)
  const void* a1;  // A source for shared groups (FWD1: x, DX2 / DW2: upstream grad)
  const void* b0;  // B source (weights, or rhs rows for DW)
  const void* b1;  // B source for shared groups (DW1: x)
  void* out;
  void* out2;       // FWD1: saved pre-activations (nullable)
  const void* aux;  // DX2: saved pre-activations
  int accumulate;
  // FWD1 / DW1: when set, the routed groups' x rows are gathered from a1 (x)
  // through these token ids (sorted_ids [Rr]) instead of read from a permuted copy
  const int32_t* gather_ids;
  // expert parallelism (null: none): this rank's routed groups are its local
  // experts; FWD1 / DX2 wait for the other ranks' rows, FWD2 / DX1 write the
  // routed output rows into their sources' buffers (ep->rows) and signal them
  const moe_ep_peers* ep;
  int shared_first;  // the shared groups' tiles first (they need no exchange)
};

// Tensor map of a row-major bf16 matrix [rows, cols] (cols contiguous): box of
// 64 columns (128 bytes) x box_rows rows, 128-byte swizzle, zero fill past the edges.
bool make_map_bf16(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, int box_rows);

// Wall-time budget of one bounded wait inside a kernel (MOE_WAIT_BUDGET_NS, default 4 s).
uint64_t wait_budget_ns();

int launch_grouped_gemm(GemmMode mode, const moe_dims& dm, const void* ws,
                        const GemmOperands& ops, void* stream);

// Expert parallelism (ep.cu); each returns a moe_status.
bool ep_peers_ok(const moe_ep_peers* p, bool need_rows);
int launch_ep_plan(const moe_dims& dm, const moe_ep_peers& pe, const int32_t* counts_all,
                   int32_t* counts_loc, int64_t cap, void* stream);
int launch_ep_dispatch(const moe_dims& dm, const moe_ep_peers& pe, const int32_t* sorted_ids,
                       const int32_t* offsets, const void* x, void* stream);
int launch_ep_zero_pads(const moe_dims& dm, const moe_ep_peers& pe, void* buf, void* stream);
int launch_ep_wait(const moe_ep_peers& pe, int ctr, void* stream);
int launch_combine_bwd_ep(const moe_dims& dm, const moe_ep_peers& pe, const void* dout,
                          const void* y, const int32_t* row_of, const float* w,
                          const int32_t* idx, const int32_t* offsets, float* dw, void* stream);

}  // namespace moe
