// ep.cu -- expert parallelism on the device: the step's exchange plan built from
// the ranks' per-expert counts, the dispatch of x rows straight into the
// owners' receive buffers (segment by segment, each expert's arrival signalled on
// its own), the owners' pad rows, and the bounded wait on an arrival counter.
//
// Passage: dots.llm1 Technical Report, §3.1 "Interleaved-1F1B based
// communication/computation overlap" (all-to-all dispatch and combine of expert
// parallelism, overlapped with computation) and §3.2 (each expert's segment
// padded to a fixed block, so a received segment is a run of whole blocks).
//
// Rank r owns routed experts r E_l .. (r+1) E_l - 1.  An owner lays its received
// rows out expert-major: for each of its experts, the P-padded segments of ranks
// 0 .. W-1.  Every rank computes the whole plan from the count table of all
// ranks (an all-gather of E int32 per rank), so sender and receiver agree on
// every offset without talking.
#include <cuda_runtime.h>

#include "ep_internal.cuh"

namespace moe {
namespace {

__global__ void __launch_bounds__(256)
    ep_plan_kernel(const int32_t* __restrict__ counts_all, int rank, int W, int El, int P,
                   int64_t cap, int* __restrict__ ws, int32_t* __restrict__ counts_loc,
                   EpLayout L) {
  const int E = W * El;
  __shared__ int32_t s_pad[kEpMaxWorld][256];
  __shared__ int32_t s_base[kEpMaxWorld][257];  // owner o: rows before its local expert e
  __shared__ int32_t s_pre[kEpMaxWorld][257];   // source s: permuted rows before expert g
  __shared__ int s_bad;
  const int tid = threadIdx.x;
  if (tid == 0) s_bad = 0;
  __syncthreads();
  for (int i = tid; i < W * E; i += blockDim.x) {
    const int s = i / E, g = i - s * E;
    const int c = counts_all[i];
    if (c < 0) atomicExch(&s_bad, 1);
    s_pad[s][g] = c > 0 ? (c + P - 1) / P * P : 0;
  }
  __syncthreads();
  if (tid < W) {  // thread o: owner o's expert-major layout; thread s: source s's segments
    int64_t acc = 0;
    for (int e = 0; e < El; ++e) {
      s_base[tid][e] = (int32_t)acc;
      for (int s = 0; s < W; ++s) acc += s_pad[s][tid * El + e];
    }
    s_base[tid][El] = (int32_t)(acc > cap ? cap : acc);
    reinterpret_cast<int32_t*>(reinterpret_cast<uint8_t*>(ws) + L.over)[tid] = acc > cap;
    int64_t pre = 0;
    for (int g = 0; g < E; ++g) {
      s_pre[tid][g] = (int32_t)pre;
      pre += s_pad[tid][g];
    }
    if (acc > cap) atomicExch(&s_bad, 1);
  }
  __syncthreads();
  uint8_t* wsb = reinterpret_cast<uint8_t*>(ws);
  int32_t* send_dst = reinterpret_cast<int32_t*>(wsb + L.send_dst);
  int32_t* recv_row = reinterpret_cast<int32_t*>(wsb + L.recv_row);
  int32_t* recv_cnt = reinterpret_cast<int32_t*>(wsb + L.recv_cnt);
  int32_t* recv_real = reinterpret_cast<int32_t*>(wsb + L.recv_real);
  int32_t* src_off = reinterpret_cast<int32_t*>(wsb + L.src_off);
  for (int g = tid; g < E; g += blockDim.x) {  // this rank as a source
    const int o = g / El, e = g - o * El;
    int32_t row = s_base[o][e];
    for (int s = 0; s < rank; ++s) row += s_pad[s][g];
    send_dst[g] = row;
  }
  for (int i = tid; i < W * El; i += blockDim.x) {  // this rank as an owner
    const int s = i / El, e = i - s * El, g = rank * El + e;
    int32_t row = s_base[rank][e];
    for (int s2 = 0; s2 < s; ++s2) row += s_pad[s2][g];
    recv_row[i] = row;
    recv_cnt[i] = s_pad[s][g];
    recv_real[i] = counts_all[s * E + g];
    src_off[i] = s_pre[s][g];
  }
  for (int e = tid; e < El; e += blockDim.x) {
    int32_t n = 0;
    for (int s = 0; s < W; ++s) n += s_pad[s][rank * El + e];
    counts_loc[e] = n;
  }
  // this rank as a source: its rows per expert, and its dispatch work items of
  // kEpDispatchRows rows (one at least per expert, so that every owner hears about
  // every expert every step), counted in the order q = e W + o
  int32_t* own_cnt = reinterpret_cast<int32_t*>(wsb + L.own_cnt);
  int32_t* done = reinterpret_cast<int32_t*>(wsb + L.done);
  int32_t* chunk_pre = reinterpret_cast<int32_t*>(wsb + L.chunk_pre);
  for (int g = tid; g < E; g += blockDim.x) {
    own_cnt[g] = counts_all[rank * E + g];
    done[g] = 0;
  }
  if (tid == 0) {
    int32_t acc = 0;
    for (int q = 0; q < E; ++q) {
      chunk_pre[q] = acc;
      const int g = (q % W) * El + q / W;
      const int c = counts_all[rank * E + g];
      acc += c > 0 ? (c + kEpDispatchRows - 1) / kEpDispatchRows : 1;
    }
    chunk_pre[E] = acc;
  }
  __syncthreads();
  if (tid == 0) {
    if (s_bad) atomicCAS(ws + EP_STATUS, 0, MOE_ERR_BAD_ROUTING);
    ws[EP_EPOCH] += 1;  // read by this rank's later kernels only (stream order)
  }
}

// Dispatch, segment by segment: work item i of expert g copies rows
// [16 i, 16 i + 16) of this rank's segment of g (the tokens sorted_ids lists, in
// order) into the owner's receive buffer at the row the plan gives, through the
// owner's peer pointer, two rows a warp.  Items run in the order q = e W + o, so
// every owner receives its local experts' segments in expert order.  The CTA that
// finishes an expert's last item raises that expert's arrival counter at its owner,
// so the owner's grouped GEMM can start on the expert before later ones arrive.
__global__ void __launch_bounds__(256)
    ep_dispatch_kernel(const uint4* __restrict__ x, int64_t T, int row_vec,
                       const int32_t* __restrict__ sorted_ids,
                       const int32_t* __restrict__ offsets, int* ws, EpLayout L, EpPtrs rows,
                       EpPtrs peer_ws, int W, int El) {
  const int E = W * El;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint8_t* wsb = reinterpret_cast<const uint8_t*>(ws);
  const int32_t* send_dst = reinterpret_cast<const int32_t*>(wsb + L.send_dst);
  const int32_t* over = reinterpret_cast<const int32_t*>(wsb + L.over);
  const int32_t* own_cnt = reinterpret_cast<const int32_t*>(wsb + L.own_cnt);
  const int32_t* chunk_pre = reinterpret_cast<const int32_t*>(wsb + L.chunk_pre);
  int32_t* done = reinterpret_cast<int32_t*>(reinterpret_cast<uint8_t*>(ws) + L.done);
  const int arrive_word = (int)(L.arrive / sizeof(int32_t));
  const int total = chunk_pre[E];
  for (int item = blockIdx.x; item < total; item += gridDim.x) {
    int lo = 0, hi = E - 1;  // largest q with chunk_pre[q] <= item
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (chunk_pre[mid] <= item) lo = mid; else hi = mid - 1;
    }
    const int q = lo, e = q / W, o = q - e * W, g = o * El + e;
    const int c = own_cnt[g];
    // an owner whose buffers are too small (the plan reported it) gets no rows
    if (!over[o]) {
      for (int rr = warp; rr < kEpDispatchRows; rr += blockDim.x >> 5) {
        const int row = (item - chunk_pre[q]) * kEpDispatchRows + rr;
        if (row >= c) break;
        const int tok = sorted_ids[offsets[g] + row];
        if (tok < 0 || tok >= T) continue;  // a routing the permutation refused
        const uint4* src = x + (int64_t)tok * row_vec;
        uint4* dst =
            reinterpret_cast<uint4*>(rows.p[o]) + ((int64_t)send_dst[g] + row) * row_vec;
        for (int cc = lane; cc < row_vec; cc += 32) dst[cc] = src[cc];
      }
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      __threadfence_system();  // this CTA's rows before its count
      const int nch = chunk_pre[q + 1] - chunk_pre[q];
      if (atomicAdd(done + g, 1) + 1 == nch) {
        __threadfence_system();  // every item of the segment counted: release them all
        atomicAdd_system(reinterpret_cast<int*>(peer_ws.p[o]) + arrive_word + e, 1);
      }
    }
    __syncthreads();
  }
}

// Owner: zero the pad rows of every received segment of a [cap, row_vec * 8]
// bf16 buffer.  grid = (W E_l, split).
__global__ void ep_zero_pads_kernel(const int* ws, EpLayout L, uint4* __restrict__ m,
                                    int row_vec, int rank) {
  const uint8_t* wsb = reinterpret_cast<const uint8_t*>(ws);
  const int i = blockIdx.x;
  // an owner over its capacity has no valid layout (reported by the plan): write nothing
  if (reinterpret_cast<const int32_t*>(wsb + L.over)[rank]) return;
  const int64_t row = reinterpret_cast<const int32_t*>(wsb + L.recv_row)[i];
  const int64_t real = reinterpret_cast<const int32_t*>(wsb + L.recv_real)[i];
  const int64_t cnt = reinterpret_cast<const int32_t*>(wsb + L.recv_cnt)[i];
  const int64_t n = (cnt - real) * row_vec;
  const uint4 z = make_uint4(0, 0, 0, 0);
  for (int64_t q = (int64_t)blockIdx.y * blockDim.x + threadIdx.x; q < n;
       q += (int64_t)gridDim.y * blockDim.x)
    m[(row + real) * row_vec + q] = z;
}

__global__ void ep_wait_kernel(int* ws, int ctr, int W, uint64_t budget_ns) {
  if (threadIdx.x == 0) ep_wait_counter(ws, ctr, W, ws + EP_STATUS, MOE_ERR_DEVICE_TIMEOUT,
                                        budget_ns);
}

}  // namespace

bool ep_peers_ok(const moe_ep_peers* p, bool need_rows) {
  if (!p || p->world < 1 || p->world > kEpMaxWorld || p->rank < 0 || p->rank >= p->world)
    return false;
  for (int o = 0; o < p->world; ++o) {
    if (!p->ep_ws[o]) return false;
    if (need_rows && !p->rows[o]) return false;
  }
  return p->ep_ws[p->rank] != nullptr;
}

EpPtrs ep_ptrs(void* const* v, int world) {
  EpPtrs e{};
  for (int o = 0; o < world; ++o) e.p[o] = reinterpret_cast<uint64_t>(v[o]);
  return e;
}

int launch_ep_plan(const moe_dims& dm, const moe_ep_peers& pe, const int32_t* counts_all,
                   int32_t* counts_loc, int64_t cap, void* stream) {
  const EpLayout L = ep_layout(dm.E, pe.world);
  ep_plan_kernel<<<1, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      counts_all, pe.rank, pe.world, dm.E / pe.world, dm.P, cap,
      reinterpret_cast<int*>(pe.ep_ws[pe.rank]), counts_loc, L);
  return cuda_ok(cudaGetLastError()) ? MOE_OK : MOE_ERR_CUDA;
}

int launch_ep_dispatch(const moe_dims& dm, const moe_ep_peers& pe, const int32_t* sorted_ids,
                       const int32_t* offsets, const void* x, void* stream) {
  const EpLayout L = ep_layout(dm.E, pe.world);
  static int num_sms = 0;
  if (num_sms == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    if (cudaDeviceGetAttribute(&num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        num_sms <= 0)
      num_sms = 148;
  }
  // persistent CTAs over the step's work items (their number lives on the device)
  ep_dispatch_kernel<<<(unsigned)(4 * num_sms), 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      reinterpret_cast<const uint4*>(x), dm.T, dm.d / 8, sorted_ids, offsets,
      reinterpret_cast<int*>(pe.ep_ws[pe.rank]), L, ep_ptrs(pe.rows, pe.world),
      ep_ptrs(pe.ep_ws, pe.world), pe.world, dm.E / pe.world);
  return cuda_ok(cudaGetLastError()) ? MOE_OK : MOE_ERR_CUDA;
}

int launch_ep_zero_pads(const moe_dims& dm, const moe_ep_peers& pe, void* buf, void* stream) {
  const EpLayout L = ep_layout(dm.E, pe.world);
  const int segs = pe.world * (dm.E / pe.world);
  ep_zero_pads_kernel<<<dim3(segs, 4), 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      reinterpret_cast<const int*>(pe.ep_ws[pe.rank]), L, reinterpret_cast<uint4*>(buf),
      dm.d / 8, pe.rank);
  return cuda_ok(cudaGetLastError()) ? MOE_OK : MOE_ERR_CUDA;
}

int launch_ep_wait(const moe_ep_peers& pe, int ctr, void* stream) {
  ep_wait_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      reinterpret_cast<int*>(pe.ep_ws[pe.rank]), ctr, pe.world, wait_budget_ns());
  return cuda_ok(cudaGetLastError()) ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace moe
