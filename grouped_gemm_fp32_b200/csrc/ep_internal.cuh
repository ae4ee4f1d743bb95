// ep_internal.cuh -- expert parallelism on the device: the EP workspace layout,
// the peer tables the kernels take by value, and the arrival-counter protocol.
//
// Passage: dots.llm1 Technical Report, §3.1 "Interleaved-1F1B based
// communication/computation overlap" (the all-to-all dispatch and combine of
// expert parallelism overlapped with computation) and §3.2 (expert-aligned
// segments).
//
// Every transfer is a kernel that writes rows straight into other ranks' buffers
// through peer pointers and ends with the last CTA of the launch adding 1 to a
// counter in every receiving rank's EP workspace (release at system scope).  A
// receiver waits, bounded, until its counter reaches world x epoch (its own step
// count), so no segment size ever goes to the host.
#pragma once
#include <cstdint>

#include "moe_internal.cuh"

namespace moe {

constexpr int kEpMaxWorld = MOE_EP_MAX_WORLD;

// Counters and flags of the EP workspace (int32 words).
enum EpWord {
  EP_STATUS = 0,     // device status word (moe_get_device_status reads it)
  EP_EPOCH = 1,      // steps planned so far on this rank
  EP_CTR_ROWS = 2,   // (unused: forward rows arrive per expert, in `arrive` below)
  EP_CTR_Y = 3,      // expert outputs returned (one per owner and step)
  EP_CTR_DY = 4,     // backward rows arrived (one per source and step)
  EP_CTR_DX = 5,     // data gradients returned (one per owner and step)
  EP_DONE_ROWS = 6,  // (unused)
  EP_DONE_Y = 7,
  EP_DONE_DY = 8,
  EP_DONE_DX = 9,
  EP_HEADER = 16
};

// Plan arrays after the header (rank r, W ranks, E_l local experts, E = W E_l):
//   send_dst [E]        first row of this rank's segment of expert g in its owner's
//                       receive buffer
//   recv_row [W][E_l]   (owner view) first local row of source s's segment of local
//                       expert e: sum_{e' < e} sum_s pad(c[s][r E_l + e'])
//                                 + sum_{s' < s} pad(c[s'][r E_l + e])
//   recv_cnt [W][E_l]   its padded rows pad(c[s][r E_l + e])
//   recv_real[W][E_l]   its real rows c[s][r E_l + e]
//   src_off  [W][E_l]   the same segment's first row in source s's permuted rows
//   over     [W]        1 when owner o would receive more rows than its buffers hold
//   arrive   [E_l]      (owner) forward segments of local expert e arrived: one per
//                       source and step, never reset
//   own_cnt  [E]        (source) this rank's rows of expert g, c[r][g]
//   done     [E]        (source) dispatch work items of expert g finished this step
//                       (zeroed by the plan)
//   chunk_pre[E + 1]    (source) prefix of the dispatch work items per expert, in the
//                       order q = e W + o (each owner's local expert 0 first, then 1, ...)
struct EpLayout {
  size_t send_dst, recv_row, recv_cnt, recv_real, src_off, over, arrive, own_cnt, done,
      chunk_pre, bytes;
};

constexpr int kEpDispatchRows = 16;  // rows of one segment a dispatch work item copies

inline EpLayout ep_layout(int E, int world) {
  EpLayout L;
  const int El = E / world;
  size_t off = EP_HEADER * sizeof(int32_t);
  L.send_dst = off;
  off += sizeof(int32_t) * E;
  L.recv_row = off;
  off += sizeof(int32_t) * world * El;
  L.recv_cnt = off;
  off += sizeof(int32_t) * world * El;
  L.recv_real = off;
  off += sizeof(int32_t) * world * El;
  L.src_off = off;
  off += sizeof(int32_t) * world * El;
  L.over = off;
  off += sizeof(int32_t) * world;
  L.arrive = off;
  off += sizeof(int32_t) * El;
  L.own_cnt = off;
  off += sizeof(int32_t) * E;
  L.done = off;
  off += sizeof(int32_t) * E;
  L.chunk_pre = off;
  off += sizeof(int32_t) * (E + 1);
  L.bytes = align_up(off, 256);
  return L;
}

// Every rank's address of something (its EP workspace counters, or its rows),
// as mapped in this process; taken by value by the kernels.
struct EpPtrs {
  uint64_t p[kEpMaxWorld];
};

EpPtrs ep_ptrs(void* const* v, int world);

// The last CTA of a launch (counted on `done`, a monotonic counter of this
// rank's workspace: every launch of one kernel has the same grid) adds 1 to word
// `ctr` of every rank's EP workspace.  Called by all threads of every CTA after
// the CTA's writes; the CTA's writes are released at system scope first.
__device__ __forceinline__ void ep_signal_last_cta(int* done, const EpPtrs& ws, int world,
                                                   int ctr) {
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence_system();
    const unsigned total = gridDim.x * gridDim.y * gridDim.z;
    const unsigned old = atomicAdd(reinterpret_cast<unsigned*>(done), 1u);
    if (old % total == total - 1) {
      __threadfence_system();
      for (int o = 0; o < world; ++o)
        atomicAdd_system(reinterpret_cast<int*>(ws.p[o]) + ctr, 1);
    }
  }
}

__device__ __forceinline__ int ld_acquire_sys(const int* p) {
  int v;
  asm volatile("ld.acquire.sys.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Bounded wait until word `ctr` of this rank's EP workspace reaches world x
// epoch; false (and `code` in *status, first error wins) when `budget_ns` ran out.
__device__ __forceinline__ bool ep_wait_counter(const int* ep_ws, int ctr, int world, int* status,
                                                int code, uint64_t budget_ns) {
  const int target = world * ld_acquire_sys(ep_ws + EP_EPOCH);
  if (ld_acquire_sys(ep_ws + ctr) - target >= 0) return true;
  uint64_t t0;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t0));
  for (;;) {
    if (ld_acquire_sys(ep_ws + ctr) - target >= 0) return true;
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    if (t - t0 > budget_ns) {
      atomicCAS(status, 0, code);
      return false;
    }
  }
}

// What the grouped GEMM needs to run as the owner's side of the exchange: wait
// for the rows (FWD1 / DX2), or write the routed groups' output rows straight
// into their sources' buffers and signal them (FWD2 / DX1).
struct EpGemm {
  const int* ep_ws;      // this rank's EP workspace (null: no exchange)
  int wait_ctr;          // word of the counter to wait on (EP_CTR_DY), or 0: no wait
  int per_group;         // 1: wait on word wait_ctr + g (the group's own arrival counter)
  int world, El;
  int ret_ctr;           // EP_CTR_Y / EP_CTR_DX, or 0: outputs stay local
  int done_word;         // EP_DONE_Y / EP_DONE_DX
  EpPtrs peer_ws;        // every rank's EP workspace
  const int32_t* recv_row;
  const int32_t* src_off;
};

// Expert parallelism in the combine backward: where each pick's dY row goes (its
// owner's receive buffer, at the row the plan gives its segment), and whom to
// signal once all are written.  W = 0: no exchange, dY stays in the local buffer.
struct EpDy {
  EpPtrs rows;              // every owner's receive buffer for dY
  EpPtrs peer_ws;           // every rank's EP workspace
  const int32_t* send_dst;  // [E] this rank's segment starts in the owners' buffers
  const int32_t* over;      // [W] owners whose buffers are too small
  const int32_t* idx;       // [T, k] the picks' experts
  const int32_t* offsets;   // [E + 1] this rank's segment starts in its permuted rows
  int* done;                // this rank's launch counter of the kernel
  int El, W;
};

__device__ __forceinline__ uint4* ep_dy_row(const EpDy& ep, uint4* dy, int64_t t, int k, int j,
                                            int64_t r, int row_vec) {
  if (ep.W == 0) return dy + r * row_vec;
  const int g = ep.idx[t * k + j];
  if (g < 0 || g >= ep.W * ep.El || ep.over[g / ep.El]) return nullptr;
  return reinterpret_cast<uint4*>(ep.rows.p[g / ep.El]) +
         ((int64_t)ep.send_dst[g] + r - ep.offsets[g]) * row_vec;
}

}  // namespace moe
