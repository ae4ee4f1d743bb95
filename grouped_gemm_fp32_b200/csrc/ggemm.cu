// ggemm.cu -- persistent grouped GEMM on the 5th-generation tensor cores
// (tcgen05.mma, accumulators in tensor memory, operands staged by TMA).
//
// Passage: dots.llm1 Technical Report, §3.2 "Efficient implementation of
// Grouped GEMM".  Every expert's token segment is padded to a fixed block, so
// a 128-row tile never straddles two experts and scheduling reduces to that of
// a plain GEMM: tiles are (group, 256-row tile, n-tile) triples enumerated from
// a per-group prefix of 256-row tile counts that is built on the device (no host
// round trip).  The pages' version targets sm_90 warpgroup MMA; this one is
// written for sm_100a.  CTAs run in pairs (a 2-CTA cluster, one CTA per SM) and
// work through 256 x 256 tiles persistently, each pair drawing its next tile from
// a counter in the workspace, with the paired tcgen05.mma (cta_group::2):
// each CTA stages its own 128 rows of A and half of B (N/2 columns), so one
// SM's shared memory feeds half the B traffic of a 1-CTA 128 x 256 tile.
//   warp 0        TMA producer of this CTA's rows of A (6-stage ring, 32 KB a stage
//                 with B); in the leader CTA also the tile hand-out and the arming of
//                 each stage; completions are counted on the leader CTA's barriers
//   warp 1        tensor-memory owner; in the leader CTA the single-thread
//                 tcgen05.mma issuer for the pair
//   warps 2..9    epilogue of this CTA's 128 accumulator rows (two warps per
//                 32-lane quarter, each on half the columns): tcgen05.ld, fused
//                 SwiGLU / SwiGLU-backward, bf16 or f32 stores
//   warp 10       TMA producer of this CTA's half of B
// with two 256-column FP32 accumulators in tensor memory per CTA so the
// epilogue of one tile overlaps the MMAs of the next.  Segments are padded to
// 128-row blocks, so a group's last m-tile may hold only 128 rows: it runs as a
// half tile (the paired MMA with M = 128, 64 rows per CTA), whose accumulator
// puts the first N/2 columns of the CTA's rows in lanes 0-63 and the last N/2
// in lanes 64-127 of tensor-memory columns [0, N/2).
//
// Six GEMMs of the expert FFN share this kernel (A is M x K, B is N x K):
//   FWD1  A = x rows (K-major)     B = W1 gate|up rows (K-major)  -> SwiGLU -> H (+ A1)
//   FWD2  A = H rows (K-major)     B = W2 rows (K-major)          -> Y
//   DX2   A = dY rows (K-major)    B = W2 as [d, I] (N-major)     -> SwiGLU bwd -> dA
//   DX1   A = dA rows (K-major)    B = W1 as [2I, d] (N-major)    -> dX rows
//   DW2   A = dY^T (M-major)       B = H^T (N-major), K = group rows -> dW2 f32
//   DW1   A = dA^T (M-major)       B = x^T (N-major), K = group rows -> dW1 f32
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdio>
#include <cstring>
#include <mutex>
#include <type_traits>

#include "ep_internal.cuh"
#include "moe_internal.cuh"
#include "sm100.cuh"

namespace moe {

namespace {

constexpr int BM = 128;           // rows of A per CTA (the pair's UMMA M is 256)
constexpr int PM = 2 * BM;        // rows of a pair tile
constexpr int BK = 64;            // K per stage: one 128-byte swizzle row of bf16
constexpr int MAX_STAGES = 6;
constexpr int A_BYTES = BM * BK * 2;    // 16 KB: this CTA's 128 rows of A
constexpr int B_BYTES = 128 * BK * 2;   // 16 KB: this CTA's half of B (N/2 <= 128)
constexpr int EPI_WARPS = 8;            // two per tensor-memory lane quarter
constexpr int SLOT_BYTES = 32 * 128;    // an epilogue warp's staging slot: 32 rows x 128 B
constexpr int B_WARP = 2 + EPI_WARPS;        // the producer of B (after the epilogue warps)
constexpr int NUM_THREADS = 96 + 32 * EPI_WARPS;
constexpr uint32_t TMEM_COLS = 512;     // two 256-column FP32 accumulators
constexpr int MAX_GROUPS = 264;  // E <= 256 routed + S <= 8 shared
constexpr int M_BAND = 8;        // m-tiles per band of the FWD / DX tile order
// Tile indices reach the roles of a pair through a ring of SCHED_SLOTS entries in
// each CTA's shared memory.  Each entry is read once by the MMA thread, by the
// peer CTA's A producer, by both CTAs' B producers and by every epilogue warp of
// both CTAs.
constexpr int SCHED_SLOTS = 8;
constexpr int SCHED_READERS = 4 + 2 * EPI_WARPS;

struct GemmArgs {
  int* status;
  const GroupRec* groups;
  const int* mtile_prefix;
  const int* dw_order;
  int G, E;
  int K;             // reduction length (FWD/DX)
  int n_out;         // valid output columns
  int m_out;         // DW: valid output rows
  int NT, MT;        // n-tiles per group; DW: 256-row m-tiles per group
  int hn;            // FWD1: H columns per tile (64 or 128)
  int I;             // FWD1 / DX2: intermediate size
  int b_group_rows;  // rows one group occupies in B's 2-D view
  void* out;
  void* out2;
  const void* aux;
  int64_t ld_out, ld_out2, ld_aux;
  int accumulate;
  uint32_t idesc;
  uint32_t idesc_narrow;  // N = 128 (modes whose B is N-major)
  uint32_t idesc_h;         // half tiles: the pair's M = 128 (64 rows per CTA)
  uint32_t idesc_h_narrow;  // half tile with N = 128
  int half_ok;              // FWD / DX modes: a group's last 128 rows run as a half tile
  int staged;             // epilogue writes through shared memory + TMA stores
  int mn3;                // DX / DW: an N- or M-major operand's two 64-column chunks of a
                          // stage come in one 3-D copy (bit 0: A, bit 1: B)
  uint64_t budget_ns;
  const int32_t* gather_ids;  // FWD1 / DW1: token of each routed row, or null
  int gather_T;               // rows of the gathered tensor x
  int shared_first;           // FWD / DX: the shared groups' tiles come first
  int* tile_ctr;              // this mode's tile counter in the workspace header (0 between
                              // launches; the launch's last ticket puts it back to 0)
  EpGemm ep;                  // expert parallelism: rows to wait for, outputs to return
  // extents for the checks of the debug build: rows of the grouped row space (Rt), of
  // the routed A / B sources (Rr) and of x (T)
  int64_t rows_total, rows_routed, rows_x;
};

// Tensor maps of every source rank's rows (expert parallelism: FWD2 / DX1 write
// a routed group's output rows straight into the buffers of the ranks the rows
// came from).
struct EpMaps {
  CUtensorMap m[kEpMaxWorld];
};

// full[] and tempty[] are used in the leader CTA only (both CTAs' producers and
// epilogues signal the leader's); empty[] and tfull[] exist in both CTAs and
// receive the leader's multicast commits.  The tile ring: the leader's producer
// writes sched[] in both CTAs and arrives on both CTAs' sfull[]; every reader
// arrives on the leader's sempty[].
struct SmemCtl {
  uint64_t full[MAX_STAGES];
  uint64_t empty[MAX_STAGES];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t drain;
  uint64_t sfull[SCHED_SLOTS];
  uint64_t sempty[SCHED_SLOTS];
  int sched[SCHED_SLOTS];
  uint32_t tmem_base;
  int abort_flag;
};

template <int MODE>
__host__ __device__ constexpr int stages_of() {
  return MAX_STAGES;
}

template <int MODE>
constexpr size_t smem_bytes() {
  return 1024 /* alignment slack */ + stages_of<MODE>() * (A_BYTES + B_BYTES) +
         EPI_WARPS * SLOT_BYTES + sizeof(SmemCtl) + 64;
}

struct TileInfo {
  int g, m0, n0, nkb;
  int nw;    // N of this tile's MMA: 256, or 128 for a last tile with <= 128 columns left
  int half;  // 1: at most 128 rows of the group are left, the pair runs M = 128
             // (64 rows per CTA) instead of computing 128 rows past the group's end
};

__device__ __forceinline__ GroupRec load_group(const GemmArgs& a, int g) {
  const int4 v = __ldg(reinterpret_cast<const int4*>(a.groups) + g);
  return GroupRec{v.x, v.y, v.z, v.w};
}

// Gathered x rows.  Every row a gather copies must lie inside x, so rows that
// hold no token -- pad rows (id -1), rows past the group's padded end, and ids
// outside [0, T) -- read the group's first token instead.  Their products are
// never used: pad rows' forward results are not read, and their upstream
// gradients are zero in the backward, so they add nothing to dW.
__device__ __forceinline__ int gather_first(const GemmArgs& a, const GroupRec& gr) {
  const int id = __ldg(a.gather_ids + gr.a_row);
  return (id >= 0 && id < a.gather_T) ? id : 0;
}

// Tokens of the group's rows local .. local + 3.
__device__ __forceinline__ int4 gather_rows4(const GemmArgs& a, const GroupRec& gr, int local,
                                             int first) {
  int v[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int r = local + j;
    const int id = r < gr.rows_pad ? __ldg(a.gather_ids + gr.a_row + r) : -1;
    v[j] = (id >= 0 && id < a.gather_T) ? id : first;
  }
  return make_int4(v[0], v[1], v[2], v[3]);
}

template <int MODE>
__device__ __forceinline__ TileInfo decode_tile(int tile, const GemmArgs& a) {
  TileInfo t;
  if constexpr (MODE == MODE_DW2 || MODE == MODE_DW1) {
    const int per = a.MT * a.NT;
    const int gi = tile / per, local = tile - gi * per;
    t.g = __ldg(a.dw_order + gi);
    const int nt = local / a.MT, mt = local - nt * a.MT;
    t.m0 = mt * PM;
    t.n0 = nt * 256;
    if (MOE_DEBUG && (t.g < 0 || t.g >= a.G)) {
      t.nkb = 0;
      t.nw = 256;
      t.half = 0;
      return t;
    }
    t.nkb = (load_group(a, t.g).rows_pad + BK - 1) / BK;  // the tail block reads zeros past the end
    t.nw = (a.n_out - t.n0 > 128) ? 256 : 128;
    t.half = 0;
  } else {
    const int* pre = a.mtile_prefix;
    if (a.shared_first) {  // rotate: the shared groups' tiles (they need no exchange) first
      const int tot = __ldg(pre + a.G) * a.NT, sh = __ldg(pre + a.E) * a.NT;
      tile += sh;
      if (tile >= tot) tile -= tot;
    }
    // largest g with prefix[g] * NT <= tile  (the prefix is non-decreasing)
    int lo = 0, hi = a.G - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (__ldg(pre + mid) * a.NT <= tile) lo = mid; else hi = mid - 1;
    }
    t.g = lo;
    const int p0 = __ldg(pre + lo);
    const int mt_g = __ldg(pre + lo + 1) - p0;
    const int local = tile - p0 * a.NT;
    // n-tile-major inside bands of up to M_BAND m-tiles: the pairs running at one
    // time share a B slice, and a band's A rows stay in L2 across all n-tiles
    // (a shared group's 64 m-tiles would otherwise stream all of A once per n-tile)
    const int b = local / (M_BAND * a.NT);
    const int r = local - b * M_BAND * a.NT;
    const int bm = min(M_BAND, mt_g - b * M_BAND);
    const int nt = r / bm, mt = b * M_BAND + (r - nt * bm);
    t.m0 = mt * PM;
    t.n0 = nt * (MODE == MODE_FWD1 ? a.hn : 256);
    t.nkb = a.K / BK;
    t.nw = (MODE == MODE_DX2 || MODE == MODE_DX1) && (a.n_out - t.n0 <= 128) ? 128 : 256;
    t.half = a.half_ok && load_group(a, lo).rows_pad - t.m0 <= BM;
  }
  return t;
}

// Debug build: the tile's group id and its record must describe rows inside the
// tensors the kernel reads and writes; otherwise MOE_ERR_BAD_ROUTING is recorded
// and every role skips the tile (all roles decide alike, from the same record).
template <int MODE>
__device__ __forceinline__ bool tile_ok(const GemmArgs& a, const TileInfo& t) {
  if constexpr (!MOE_DEBUG) {
    return true;
  } else {
    bool ok = t.g >= 0 && t.g < a.G;
    if (ok) {
      const GroupRec gr = load_group(a, t.g);
      const bool shared = t.g >= a.E;
      ok = gr.rows_pad >= 0 && gr.out_row >= 0 && gr.a_row >= 0 &&
           (int64_t)gr.out_row + gr.rows_pad <= a.rows_total &&
           (int64_t)gr.a_row + gr.rows_pad <= (shared ? a.rows_x : a.rows_routed);
      if (MODE == MODE_DW2 || MODE == MODE_DW1) ok = ok && t.m0 < a.m_out && t.n0 < a.n_out;
      else ok = ok && t.n0 < a.n_out && t.m0 < gr.rows_pad;
    }
    if (!ok) atomicCAS(a.status, 0, MOE_ERR_BAD_ROUTING);
    return ok;
  }
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ void store_bf16x32(__nv_bfloat16* dst, const float* v) {
  uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint4 w;
    w.x = pack_bf16(v[8 * q + 0], v[8 * q + 1]);
    w.y = pack_bf16(v[8 * q + 2], v[8 * q + 3]);
    w.z = pack_bf16(v[8 * q + 4], v[8 * q + 5]);
    w.w = pack_bf16(v[8 * q + 6], v[8 * q + 7]);
    d4[q] = w;
  }
}

// Eight 16-byte pieces of bf16: v[8 q .. 8 q + 7] -> piece q.
__device__ __forceinline__ uint4 pack_bf16x8(const float* v) {
  uint4 w;
  w.x = pack_bf16(v[0], v[1]);
  w.y = pack_bf16(v[2], v[3]);
  w.z = pack_bf16(v[4], v[5]);
  w.w = pack_bf16(v[6], v[7]);
  return w;
}

// Staged stores.  An epilogue warp owns a 4 KB shared-memory slot for 32 rows x
// 128 bytes in the 128-byte swizzled layout (16-byte piece j of row r sits at
// j ^ (r % 8), so a warp's 16-byte writes cover all banks).  Thread `lane` writes
// row `lane`; lane 0 then issues one TMA store -- or f32 add-reduction -- of the
// 32-row box.  The slot is rewritten only after the previous store has read it.
__device__ __forceinline__ void slot_acquire(int lane) {
  if (lane == 0) bulk_wait_read<0>();
  __syncwarp();
}

__device__ __forceinline__ void slot_put(uint8_t* slot, int lane, int j, uint4 v) {
  *reinterpret_cast<uint4*>(slot + lane * 128 + ((j ^ (lane & 7)) << 4)) = v;
}

template <bool REDUCE>
__device__ __forceinline__ void slot_issue(uint8_t* slot, const CUtensorMap* map, int x, int y,
                                           int lane) {
  fence_proxy_async_smem();  // the generic-proxy writes become visible to the TMA unit
  __syncwarp();
  if (lane == 0) {
    if (REDUCE)
      tma_reduce_add_2d(map, slot, x, y);
    else
      tma_store_2d(map, slot, x, y);
    bulk_commit();
  }
}

template <bool REDUCE>
__device__ __forceinline__ void staged_store(uint8_t* slot, const uint4 (&v)[8],
                                             const CUtensorMap* map, int x, int y, int lane) {
  slot_acquire(lane);
#pragma unroll
  for (int j = 0; j < 8; ++j) slot_put(slot, lane, j, v[j]);
  slot_issue<REDUCE>(slot, map, x, y, lane);
}

// bf16 of 32 accumulator words, as four 16-byte pieces
__device__ __forceinline__ void pack_acc_bf16(const uint32_t (&r)[32], uint4 (&p)[4]) {
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    p[j].x = pack_bf16(__uint_as_float(r[8 * j + 0]), __uint_as_float(r[8 * j + 1]));
    p[j].y = pack_bf16(__uint_as_float(r[8 * j + 2]), __uint_as_float(r[8 * j + 3]));
    p[j].z = pack_bf16(__uint_as_float(r[8 * j + 4]), __uint_as_float(r[8 * j + 5]));
    p[j].w = pack_bf16(__uint_as_float(r[8 * j + 6]), __uint_as_float(r[8 * j + 7]));
  }
}

template <int MODE>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(NUM_THREADS, 1)
    ggemm_kernel(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmA1,
                 const __grid_constant__ CUtensorMap tmB0, const __grid_constant__ CUtensorMap tmB1,
                 const __grid_constant__ CUtensorMap tmC /* DW1: shared groups' x as 3-D chunks */,
                 const __grid_constant__ CUtensorMap tmO0 /* output (FWD1: H) */,
                 const __grid_constant__ CUtensorMap tmO1 /* FWD1: saved A1 */,
                 const __grid_constant__ CUtensorMap tmA0h /* half tiles: 64-row A boxes
                                                              (DW: A as 3-D chunks) */,
                 const __grid_constant__ CUtensorMap tmA1h,
                 const __grid_constant__ CUtensorMap tmBh /* FWD1 half tiles: 64-row B boxes
                                                             (DX / DW: B as 3-D chunks) */,
                 const __grid_constant__ EpMaps epm, const GemmArgs args) {
  constexpr bool A_MN = (MODE == MODE_DW2 || MODE == MODE_DW1);
  constexpr bool B_MN = (MODE != MODE_FWD1 && MODE != MODE_FWD2);
  constexpr bool IS_DW = A_MN;
  constexpr int STAGES = stages_of<MODE>();

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * A_BYTES;
  uint8_t* sSlots = sB + STAGES * B_BYTES;  // epilogue staging, one slot per epilogue warp
  SmemCtl* ctl = reinterpret_cast<SmemCtl*>(sSlots + EPI_WARPS * SLOT_BYTES);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();  // 0 = leader of the pair
  const bool leader = rank == 0;
  const int npairs = gridDim.x >> 1;
  volatile int* abort_flag = &ctl->abort_flag;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&ctl->full[s], 1);
      mbar_init(&ctl->empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&ctl->tfull[a], 1);
      mbar_init(&ctl->tempty[a], 2 * EPI_WARPS);  // every epilogue warp of both CTAs
    }
    mbar_init(&ctl->drain, 1);
    for (int s = 0; s < SCHED_SLOTS; ++s) {
      mbar_init(&ctl->sfull[s], 1);
      mbar_init(&ctl->sempty[s], SCHED_READERS);
      ctl->sched[s] = -1;
    }
    ctl->abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmA0);
    tma_prefetch_desc(&tmA1);
    tma_prefetch_desc(&tmB0);
    tma_prefetch_desc(&tmB1);
    if (args.staged) {
      tma_prefetch_desc(&tmO0);
      if (MODE == MODE_FWD1 && args.out2 != nullptr) tma_prefetch_desc(&tmO1);
    }
  }
  if (warp == 1) {
    tmem_alloc_pair(&ctl->tmem_base, TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // both CTAs' barriers exist before either signals the other
  tc_fence_after();
  const uint32_t tmem_base = ctl->tmem_base;
  // Waits that only make sure work already started has finished (copies in
  // flight, MMAs issued) get a long budget of their own, so a short wait budget
  // can never let this CTA free tensor memory or exit under them.
  const uint64_t drain_budget = args.budget_ns > 2000000000ull ? args.budget_ns : 2000000000ull;
  // A role that gives up tells the peer CTA too, so both stop issuing work.
  const uint32_t peer_abort = map_to_rank(&ctl->abort_flag, rank ^ 1u);
  auto abort_pair = [&]() {
    *abort_flag = 1;
    st_shared_cluster_u32(peer_abort, 1u);
  };
  const int total_tiles =
      IS_DW ? args.G * args.MT * args.NT : __ldg(args.mtile_prefix + args.G) * args.NT;

  // Tiles are handed out at run time: the leader's producer draws each next tile
  // from the launch's counter (a ticket) and publishes it in the ring; -1 ends the
  // pair's work.  All pairs therefore work on one window of consecutive tiles, in
  // the order decode_tile gives, however long their tiles take, so the operands of
  // the tiles in flight are shared in L2.  Every pair draws exactly one ticket at
  // or past total_tiles, so the pair that draws total_tiles + npairs - 1 is the
  // last to draw and puts the counter back to 0 for the next launch.
  // No ring operation is a release fence at cluster scope (a hand-off built on
  // release-arrives measured 8-20% slower in every mode, as if each fence waited for
  // the thread's copies or MMAs in flight): the peer's entry is written by st.async,
  // whose bytes complete the peer's sfull phase, and a reader hands an entry back
  // with an arrive predicated on the value it read.
  auto ring_put = [&](int seq, int tile) -> bool {
    const int s = seq % SCHED_SLOTS;
    const uint32_t par = (uint32_t)(seq / SCHED_SLOTS) & 1u;
    if (!mbar_wait(&ctl->sempty[s], par ^ 1u, abort_flag, args.status, MOE_ERR_DEVICE_TIMEOUT,
                   args.budget_ns))
      return false;
    ctl->sched[s] = tile;
    mbar_arrive(&ctl->sfull[s]);
    const uint32_t peer_full = map_to_rank(&ctl->sfull[s], 1);
    mbar_arrive_expect_tx_remote(peer_full, 4u);
    st_async_u32(map_to_rank(&ctl->sched[s], 1), (uint32_t)tile, peer_full);
    return true;
  };
  auto ring_get = [&](int seq, int& tile) -> bool {
    const int s = seq % SCHED_SLOTS;
    const uint32_t par = (uint32_t)(seq / SCHED_SLOTS) & 1u;
    if (!mbar_wait(&ctl->sfull[s], par, abort_flag, args.status, MOE_ERR_DEVICE_TIMEOUT,
                   args.budget_ns))
      return false;
    tile = *reinterpret_cast<volatile int*>(&ctl->sched[s]);
    mbar_arrive_remote_after(map_to_rank(&ctl->sempty[s], 0), tile);
    return true;
  };
  auto ticket_done = [&](int ticket) {
    if (ticket == total_tiles + npairs - 1) atomicExch(args.tile_ctr, 0);
  };

  if (warp == 0 || warp == B_WARP) {
    // ----------------------------------------------------------- producers --
    // Two producer warps per CTA, each waiting for free stages on its own: warp 0
    // copies this CTA's A and hands out the tiles (the leader's warp 0 draws them and
    // arms the leader's full barrier with both operands' bytes of both CTAs; the
    // other operand's copies may land before it arms, the barrier's transaction count
    // allows that), warp B_WARP copies this CTA's half of B.  Lane 0 issues the
    // copies; with gathered x rows (FWD1's routed A, DW1's routed B) all 32 lanes of
    // that operand's warp issue four-row gathers.
    constexpr bool GATHER_A = MODE == MODE_FWD1;
    constexpr bool GATHER_B = MODE == MODE_DW1;
    // one loop, compiled per operand (PART 0: A and the tiles, 1: B) and per width
    // (WIDE: all lanes, gathers; otherwise lane 0 alone)
    auto produce = [&](auto wide_tag, auto part_tag) {
      constexpr bool WIDE = decltype(wide_tag)::value;
      constexpr int PART = decltype(part_tag)::value;
      const bool writer = PART == 0 && leader;  // draws and publishes the tiles
      int stage = 0;
      uint32_t phase = 0, issued = 0, lastpar = 0;
      bool ok = true;
      bool rows_in = PART == 1 || args.ep.wait_ctr == 0;  // other ranks' A rows have arrived
      int waited_g = -1;  // per-group waits: the last group whose rows this CTA waited for
      // The writer feeds the ring one tile ahead: it draws the next tile's ticket when
      // a tile starts and publishes it a few K blocks in (the draw has returned by
      // then), so no other producer waits for a tile at a tile boundary.
      int seq = 0;        // ring position of the current tile
      int cur = -1;       // writer: the tile at ring position seq (-1: no more)
      int nxt = -1;       // writer: the next tile's ticket, drawn but not yet published
      bool last = false;  // writer: this pair has drawn its ticket past the last tile
      auto publish = [&](int pos, int tk) -> bool {
        cur = tk;
        if (tk >= total_tiles) {
          ticket_done(tk);
          last = true;
          cur = -1;
        }
        return ring_put(pos, cur);
      };
      if (writer && lane == 0 && !publish(0, atomicAdd(args.tile_ctr, 1))) abort_pair();
      while (ok) {
        int tile = -1, got = 1;
        if (lane == 0) {
          if (writer) {
            tile = cur;
            if (tile >= 0) nxt = atomicAdd(args.tile_ctr, 1);
          } else {
            got = ring_get(seq, tile);
          }
        }
        if constexpr (WIDE) {
          got = __shfl_sync(0xffffffffu, got, 0);
          tile = __shfl_sync(0xffffffffu, tile, 0);
        }
        if (!got) {
          if (lane == 0) abort_pair();
          break;
        }
        if (tile < 0) break;
        bool pub_done = !writer;
        auto pub = [&]() {  // writer: the next tile goes to ring position seq + 1
          if (!pub_done) {
            pub_done = true;
            if (lane == 0) {
              const int tk = nxt;
              nxt = -1;
              if (!publish(seq + 1, tk)) abort_pair();
            }
          }
        };
        const TileInfo t = decode_tile<MODE>(tile, args);
        if (!tile_ok<MODE>(args, t)) {
          pub();
          ++seq;
          continue;
        }
        const GroupRec gr = load_group(args, t.g);
        const int roff = (int)rank * (t.half ? BM / 2 : BM);  // this CTA's rows of A
        const bool shared = t.g >= args.E;
        if (!shared && !rows_in && t.g != waited_g) {
          // expert parallelism: every source's rows of this group (per-group counters),
          // or of all groups, must have landed before the tile's A copies (bounded wait)
          int got = 1;
          if (lane == 0) {
            got = ep_wait_counter(args.ep.ep_ws, args.ep.wait_ctr + (args.ep.per_group ? t.g : 0),
                                  args.ep.world, args.status, MOE_ERR_DEVICE_TIMEOUT,
                                  args.budget_ns);
            // the rows were written through the generic proxy; the copies read them
            // through the async proxy
            asm volatile("fence.proxy.async.global;" ::: "memory");
          }
          if constexpr (WIDE) got = __shfl_sync(0xffffffffu, got, 0);
          if (!got) {
            if (lane == 0) abort_pair();
            break;
          }
          if (args.ep.per_group) waited_g = t.g; else rows_in = true;
        }
        const bool gat = WIDE && !shared;
        // this CTA's half of B: N/2 columns from n0 + rank * N/2, in 64-column chunks
        const int bchunks = t.nw / 128;
        [[maybe_unused]] const int boff = (int)rank * (t.nw / 2);
        const uint32_t b_bytes = (MODE == MODE_FWD1) ? (uint32_t)(args.hn * BK * 2)
                                 : B_MN ? (uint32_t)(bchunks * 8192) : (uint32_t)B_BYTES;
        const uint32_t a_bytes = t.half ? A_BYTES / 2 : A_BYTES;
        const uint32_t pair_bytes = 2 * (a_bytes + b_bytes);  // both CTAs' copies
        int first = 0;
        int4 rows4 = make_int4(0, 0, 0, 0);  // the four x rows this lane gathers
        if (gat) {
          first = gather_first(args, gr);
          // FWD1: rows 4 lane .. 4 lane + 3 of this CTA's 128, fixed over the K loop;
          // DW1: rows 4 (lane % 16) .. of the first K block (then one block ahead)
          rows4 = gather_rows4(args, gr, MODE == MODE_FWD1 ? t.m0 + roff + 4 * lane
                                                           : 4 * (lane & 15), first);
        }
        for (int kb = 0; kb < t.nkb; ++kb) {
          int got = 1;
          if (lane == 0)
            got = mbar_wait(&ctl->empty[stage], phase ^ 1, abort_flag, args.status,
                            MOE_ERR_DEVICE_TIMEOUT, args.budget_ns);
          if constexpr (WIDE) got = __shfl_sync(0xffffffffu, got, 0);
          if (!got) {
            if (lane == 0) abort_pair();
            ok = false;
            break;
          }
          if (writer && lane == 0) mbar_arrive_expect_tx(&ctl->full[stage], pair_bytes);
          const uint32_t fb = map_to_rank(&ctl->full[stage], 0);
          [[maybe_unused]] uint8_t* a_dst = sA + stage * A_BYTES;
          [[maybe_unused]] uint8_t* b_dst = sB + stage * B_BYTES;
          const int k0 = kb * BK;
          if constexpr (PART == 0) {
            // ---- A: this CTA's rows of the tile (DW: its 128 columns of A^T)
            if constexpr (MODE == MODE_FWD1) {
              if (gat && (!t.half || lane < 16))
                tma_gather4_pair(a_dst + lane * 512, &tmA0, fb, k0, rows4.x, rows4.y, rows4.z,
                                 rows4.w);
              if (lane == 0 && !gat)
                tma_load_2d_pair(a_dst,
                                 t.half ? (shared ? &tmA1h : &tmA0h) : (shared ? &tmA1 : &tmA0),
                                 fb, k0, (shared ? 0 : gr.a_row) + t.m0 + roff);
            } else if constexpr (MODE == MODE_FWD2 || MODE == MODE_DX1) {
              tma_load_2d_pair(a_dst, t.half ? &tmA0h : &tmA0, fb, k0, gr.out_row + t.m0 + roff);
            } else if constexpr (MODE == MODE_DX2) {
              tma_load_2d_pair(a_dst,
                               t.half ? (shared ? &tmA1h : &tmA0h) : (shared ? &tmA1 : &tmA0),
                               fb, k0, (shared ? 0 : gr.a_row) + t.m0 + roff);
            } else {  // DW2 / DW1: K runs over the group's rows
              const int arow = (MODE == MODE_DW2) ? (shared ? 0 : gr.a_row) : gr.out_row;
              if (args.mn3 & 1) {
                const CUtensorMap* ma3 = (MODE == MODE_DW2 && shared) ? &tmA1h : &tmA0h;
                tma_load_3d_pair(a_dst, ma3, fb, 0, arow + k0, (t.m0 + roff) >> 6);
              } else {
                const CUtensorMap* ma = (MODE == MODE_DW2 && shared) ? &tmA1 : &tmA0;
#pragma unroll
                for (int c = 0; c < 2; ++c)
                  tma_load_2d_pair(a_dst + c * 8192, ma, fb, t.m0 + roff + c * 64, arow + k0);
              }
            }
          } else {
            // ---- B: this CTA's half of the tile's columns
            if constexpr (MODE == MODE_FWD1) {
              // the leader stages the gate rows, the peer the up rows -- in a half tile
              // each CTA stages 64 gate rows and the matching 64 up rows, so a row's
              // gate and up sums land in the same tensor-memory lane
              const int brow = t.g * args.b_group_rows + t.n0;
              if (t.half) {
                tma_load_2d_pair(b_dst, &tmBh, fb, k0, brow + (int)rank * 64);
                tma_load_2d_pair(b_dst + 8192, &tmBh, fb, k0, brow + args.I + (int)rank * 64);
              } else {
                tma_load_2d_pair(b_dst, &tmB0, fb, k0, brow + (leader ? 0 : args.I));
              }
            } else if constexpr (MODE == MODE_FWD2) {
              tma_load_2d_pair(b_dst, &tmB0, fb, k0,
                               t.g * args.b_group_rows + t.n0 + (int)rank * 128);
            } else if constexpr (MODE == MODE_DX2 || MODE == MODE_DX1) {
              const int brow = t.g * args.b_group_rows + k0;
              if (bchunks == 2 && (args.mn3 & 2))
                tma_load_3d_pair(b_dst, &tmBh, fb, 0, brow, (t.n0 + boff) >> 6);
              else
                for (int c = 0; c < bchunks; ++c)
                  tma_load_2d_pair(b_dst + c * 8192, &tmB0, fb, t.n0 + boff + c * 64, brow);
            } else {  // DW2 / DW1
              const CUtensorMap* mb;
              const CUtensorMap* mb3;  // the same tensor as 3-D chunks
              int brow;
              if constexpr (MODE == MODE_DW2) {
                mb = &tmB0;
                mb3 = &tmBh;
                brow = gr.out_row;
              } else {
                mb = shared ? &tmB1 : &tmB0;
                mb3 = shared ? &tmC : &tmBh;
                brow = shared ? 0 : gr.a_row;
              }
              if (lane == 0 && !gat) {
                if (bchunks == 2 && (args.mn3 & 2))
                  tma_load_3d_pair(b_dst, mb3, fb, 0, brow + k0, (t.n0 + boff) >> 6);
                else
                  for (int c = 0; c < bchunks; ++c)
                    tma_load_2d_pair(b_dst + c * 8192, mb, fb, t.n0 + boff + c * 64, brow + k0);
              }
              if constexpr (MODE == MODE_DW1) {
                if (gat) {
                  // lanes 0..15: 64-column chunk 0, lanes 16..31: chunk 1; lane i % 16
                  // brings K rows 4 i .. 4 i + 3 of this block
                  const int c = lane >> 4;
                  if (c < bchunks)
                    tma_gather4_pair(b_dst + c * 8192 + (lane & 15) * 512, mb, fb,
                                     t.n0 + boff + c * 64, rows4.x, rows4.y, rows4.z, rows4.w);
                  if (kb + 1 < t.nkb)
                    rows4 = gather_rows4(args, gr, k0 + BK + 4 * (lane & 15), first);
                }
              }
            }
          }
          issued |= 1u << stage;
          lastpar = (lastpar & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
          if (kb == min(t.nkb - 1, 3)) pub();
        }
        pub();  // a tile without K blocks (a DW group with no rows), or an early stop
        ++seq;
      }
      // A pair that stopped early still draws up to its ticket past the last tile,
      // so the launch's last ticket is drawn and the counter goes back to 0.
      if (writer && lane == 0 && !last) {
        int tk = nxt >= 0 ? nxt : atomicAdd(args.tile_ctr, 1);
        while (tk < total_tiles) tk = atomicAdd(args.tile_ctr, 1);
        ticket_done(tk);
      }
      // The leader's full barriers count both operands' copies of both CTAs: once the
      // phases it armed have completed, every copy of those stages has landed.
      if (writer && lane == 0)
        for (int s = 0; s < STAGES; ++s)
          if (issued & (1u << s)) {
            volatile int never = 0;
            mbar_wait(&ctl->full[s], (lastpar >> s) & 1u, &never, args.status,
                      MOE_ERR_DEVICE_TIMEOUT, drain_budget);
          }
    };
    using A_PART = std::integral_constant<int, 0>;
    using B_PART = std::integral_constant<int, 1>;
    if (warp == 0) {
      if (GATHER_A && args.gather_ids != nullptr) {
        if constexpr (GATHER_A) produce(std::true_type{}, A_PART{});
      } else if (lane == 0) {
        produce(std::false_type{}, A_PART{});
      }
    } else {
      if (GATHER_B && args.gather_ids != nullptr) {
        if constexpr (GATHER_B) produce(std::true_type{}, B_PART{});
      } else if (lane == 0) {
        produce(std::false_type{}, B_PART{});
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------- MMA issuer (leader) --
    if (leader && lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;  // tiles processed (the debug build skips invalid ones)
      bool ok = true;
      for (int seq = 0; ok; ++seq) {
        int tile = -1;
        if (!ring_get(seq, tile)) {
          abort_pair();
          break;
        }
        if (tile < 0) break;
        const TileInfo t = decode_tile<MODE>(tile, args);
        if (!tile_ok<MODE>(args, t)) continue;
        const int acc = it & 1;
        const uint32_t use = (uint32_t)(it >> 1);
        if (!mbar_wait(&ctl->tempty[acc], (use & 1u) ^ 1u, abort_flag, args.status,
                       MOE_ERR_DEVICE_TIMEOUT, args.budget_ns)) {
          abort_pair();
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * 256);
        const uint32_t idesc = t.half ? (t.nw == 256 ? args.idesc_h : args.idesc_h_narrow)
                                      : (t.nw == 256 ? args.idesc : args.idesc_narrow);
        for (int kb = 0; kb < t.nkb; ++kb) {
          if (!mbar_wait(&ctl->full[stage], phase, abort_flag, args.status,
                         MOE_ERR_DEVICE_TIMEOUT, args.budget_ns)) {
            abort_pair();
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_base = smem_u32(sA + stage * A_BYTES);
          const uint32_t b_base = smem_u32(sB + stage * B_BYTES);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint64_t ad = A_MN ? smem_desc_sw128(a_base + kk * 2048, 8192, 1024)
                                     : smem_desc_sw128(a_base + kk * 32, 16, 1024);
            const uint64_t bd = B_MN ? smem_desc_sw128(b_base + kk * 2048, 8192, 1024)
                                     : smem_desc_sw128(b_base + kk * 32, 16, 1024);
            umma_f16_pair(d_tmem, ad, bd, idesc, (kb | kk) != 0 ? 1u : 0u);
          }
          umma_commit_pair(&ctl->empty[stage], 0x3);  // frees this stage in both CTAs
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        umma_commit_pair(&ctl->tfull[acc], 0x3);  // both CTAs' epilogues may read
        ++it;
      }
      // Drain: every MMA issued completes before tensor memory is freed.
      umma_commit_pair(&ctl->drain, 0x1);
      volatile int never = 0;
      mbar_wait(&ctl->drain, 0, &never, args.status, MOE_ERR_DEVICE_TIMEOUT, drain_budget);
    }
  } else {
    // ------------------------------------------------------------ epilogue --
    // Warps 2..9: warp w reads tensor-memory lanes [32q, 32q + 32), q = w % 4,
    // and the half h of the accumulator's columns.  A full tile gives this CTA the
    // tile's rows rank * 128 + [0, 128), quarter q holding rows 32q..; a half tile
    // (M = 128) gives it rows rank * 64 + [0, 64) with quarters q and q + 2 on the
    // same 32 rows (q % 2): q < 2 the first N/2 columns, q >= 2 the last N/2, both
    // in tensor-memory columns [0, N/2).
    const int q = warp & 3;
    const int h = (warp - 2) >> 2;
    const uint32_t tempty_leader[2] = {map_to_rank(&ctl->tempty[0], 0),
                                       map_to_rank(&ctl->tempty[1], 0)};
    // hand the accumulator back to the leader's MMA thread once this warp's last
    // columns are in registers
    auto release = [&](int acc) {
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(tempty_leader[acc]);
    };
    int it = 0;  // tiles processed
    for (int seq = 0;; ++seq, ++it) {
      int tile = -1, got = 1;
      if (lane == 0) got = ring_get(seq, tile);
      got = __shfl_sync(0xffffffffu, got, 0);
      tile = __shfl_sync(0xffffffffu, tile, 0);
      if (!got) {
        abort_pair();
        break;
      }
      if (tile < 0) break;
      const TileInfo t = decode_tile<MODE>(tile, args);
      if (!tile_ok<MODE>(args, t)) {
        --it;
        continue;
      }
      const int acc = it & 1;
      const uint32_t use = (uint32_t)(it >> 1);
      if (!mbar_wait(&ctl->tfull[acc], use & 1u, abort_flag, args.status, MOE_ERR_DEVICE_TIMEOUT,
                     args.budget_ns)) {
        abort_pair();
        break;
      }
      tc_fence_after();
      const uint32_t taddr = tmem_base + (uint32_t)(acc * 256) + ((uint32_t)(q * 32) << 16);
      const GroupRec gr = load_group(args, t.g);
      uint32_t r[32];
      float v[32];
      uint8_t* slot = sSlots + (warp - 2) * SLOT_BYTES;
      // this warp's 32 rows within its group: all real (staged TMA stores), none,
      // or cut by the group's end (direct stores of the real rows)
      const int qr = t.half ? (q & 1) : q;
      const int r_in_tile = (int)rank * (t.half ? BM / 2 : BM) + qr * 32 + lane;  // row in the tile
      const int rb = t.m0 + (int)rank * (t.half ? BM / 2 : BM) + qr * 32;
      if constexpr (MODE == MODE_FWD1) {
        const int rloc = t.m0 + r_in_tile;
        const bool rv = rloc < gr.rows_pad;
        const bool whole = rb + 32 <= gr.rows_pad;
        const int64_t orow = (int64_t)gr.out_row + rloc;
        // this warp's H columns [cb, ce), counted from H column n0 + hc0; a column's gate
        // sum sits at tensor-memory column c, its up sum at c + uofs (a half tile: one
        // warp per quarter takes all 64 of the quarter's H columns)
        const int hc0 = t.half ? 64 * (q >> 1) : 0;
        const int uofs = t.half ? 64 : args.hn;
        const int cb = t.half ? 0 : h * (args.hn >> 1);
        const int ce = t.half ? (h == 0 ? 64 : 0) : cb + (args.hn >> 1);
        __nv_bfloat16* H =
            reinterpret_cast<__nv_bfloat16*>(args.out) + orow * args.ld_out + t.n0 + hc0;
        __nv_bfloat16* A1 = reinterpret_cast<__nv_bfloat16*>(args.out2);
        if (args.staged && whole && cb < ce) {
          // hn == 128: 64 H columns per warp, one 128-byte row each of H, then of the
          // saved gate and up pre-activations (read from tensor memory again)
          const int y = gr.out_row + rb;
          slot_acquire(lane);
#pragma unroll
          for (int s2 = 0; s2 < 2; ++s2) {
            uint32_t u[32];
            tmem_ld32_sync(taddr + cb + 32 * s2, r);
            tmem_ld32_sync(taddr + uofs + cb + 32 * s2, u);
            if (s2 == 1 && A1 == nullptr) release(acc);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              float hv[8];
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                const float g = __uint_as_float(r[8 * j + i]), up = __uint_as_float(u[8 * j + i]);
                hv[i] = g / (1.0f + expf(-g)) * up;
              }
              slot_put(slot, lane, 4 * s2 + j, pack_bf16x8(hv));
            }
          }
          slot_issue<false>(slot, &tmO0, t.n0 + hc0 + cb, y, lane);
          if (A1 != nullptr) {
#pragma unroll
            for (int part = 0; part < 2; ++part) {  // gate columns, then up columns
              slot_acquire(lane);
#pragma unroll
              for (int s2 = 0; s2 < 2; ++s2) {
                uint4 pk[4];
                tmem_ld32_sync(taddr + part * uofs + cb + 32 * s2, r);
                if (part == 1 && s2 == 1) release(acc);
                pack_acc_bf16(r, pk);
#pragma unroll
                for (int j = 0; j < 4; ++j) slot_put(slot, lane, 4 * s2 + j, pk[j]);
              }
              slot_issue<false>(slot, &tmO1, part * args.I + t.n0 + hc0 + cb, y, lane);
            }
          }
        } else {
          for (int c0 = cb; c0 < ce; c0 += 32) {
            uint32_t u[32];
            tmem_ld32_sync(taddr + c0, r);
            tmem_ld32_sync(taddr + uofs + c0, u);
            if (c0 + 32 >= ce) release(acc);
            if (rv) {
              float hv[32];
#pragma unroll
              for (int i = 0; i < 32; ++i) {
                const float g = __uint_as_float(r[i]), up = __uint_as_float(u[i]);
                hv[i] = g / (1.0f + expf(-g)) * up;
              }
              store_bf16x32(H + c0, hv);
              if (A1 != nullptr) {
                __nv_bfloat16* a1r = A1 + orow * args.ld_out2 + t.n0 + hc0 + c0;
#pragma unroll
                for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
                store_bf16x32(a1r, v);
#pragma unroll
                for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(u[i]);
                store_bf16x32(a1r + args.I, v);
              }
            }
          }
          if (cb >= ce) release(acc);
        }
      } else if constexpr (MODE == MODE_FWD2 || MODE == MODE_DX1) {
        const int rloc = t.m0 + r_in_tile;
        const bool rv = rloc < gr.rows_pad;
        const bool whole = rb + 32 <= gr.rows_pad;
        const int64_t orow = (int64_t)gr.out_row + rloc;
        // logical column of this quarter's tensor-memory column 0, and this warp's
        // tensor-memory columns [cb, ce) (multiples of 64)
        const int coff = t.half ? (t.nw >> 1) * (q >> 1) : 0;
        const int cb = t.half ? h * 64 : h * 128;
        const int ce = t.half ? min(min(cb + 64, t.nw >> 1), args.n_out - t.n0 - coff)
                              : min(cb + 128, args.n_out - t.n0);
        __nv_bfloat16* O =
            reinterpret_cast<__nv_bfloat16*>(args.out) + orow * args.ld_out + t.n0 + coff;
        for (int c0 = cb; c0 < ce; c0 += 64) {
          uint32_t u[32];
          tmem_ld32_sync(taddr + c0, r);
          tmem_ld32_sync(taddr + c0 + 32, u);
          if (c0 + 64 >= ce) release(acc);
          if (args.staged && whole) {
            uint4 pk[8];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
#pragma unroll
              for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[8 * j + i]);
              pk[j] = pack_bf16x8(v);
#pragma unroll
              for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(u[8 * j + i]);
              pk[4 + j] = pack_bf16x8(v);
            }
            const CUtensorMap* om = &tmO0;
            int orow_y = gr.out_row + rb;
            if (args.ep.ret_ctr != 0 && t.g < args.E) {
              // this 32-row block lies inside one source's segment (segments are
              // padded to a multiple of 32 rows): its rows go back to that rank
              const int El = args.ep.El;
              int src = 0;
              while (src + 1 < args.ep.world && orow_y >= __ldg(args.ep.recv_row + (src + 1) * El + t.g))
                ++src;
              orow_y = __ldg(args.ep.src_off + src * El + t.g) +
                       (orow_y - __ldg(args.ep.recv_row + src * El + t.g));
              om = &epm.m[src];
            }
            staged_store<false>(slot, pk, om, t.n0 + coff + c0, orow_y, lane);
          } else if (rv) {
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
            store_bf16x32(O + c0, v);
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(u[i]);
            store_bf16x32(O + c0 + 32, v);
          }
        }
        if (cb >= ce) release(acc);
      } else if constexpr (MODE == MODE_DX2) {
        const int rloc = t.m0 + r_in_tile;
        const bool rv = rloc < gr.rows_pad;
        const bool whole = rb + 32 <= gr.rows_pad;
        const int64_t orow = (int64_t)gr.out_row + rloc;
        const __nv_bfloat16* A1 =
            reinterpret_cast<const __nv_bfloat16*>(args.aux) + orow * args.ld_aux;
        __nv_bfloat16* dA = reinterpret_cast<__nv_bfloat16*>(args.out) + orow * args.ld_out;
        const int coff = t.half ? (t.nw >> 1) * (q >> 1) : 0;  // as in FWD2 / DX1
        const int cb = t.half ? h * 64 : h * 128;
        const int ce = t.half ? min(min(cb + 64, t.nw >> 1), args.I - t.n0 - coff)
                              : min(cb + 128, args.I - t.n0);
        const bool staged = args.staged && whole;
        for (int c0 = cb; c0 < ce; c0 += 64) {
          const int col = t.n0 + coff + c0;
          uint4 upk[8];  // staged: the du pieces wait here while dg goes out through the slot
          if (staged) slot_acquire(lane);
#pragma unroll
          for (int s2 = 0; s2 < 2; ++s2) {
            const int cc = col + 32 * s2;
            uint4 gq[4], uq[4];  // saved G and U of these 32 columns, bf16
            if (rv) {  // issue the saved-activation loads before waiting on tensor memory
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                gq[j] = reinterpret_cast<const uint4*>(A1 + cc)[j];
                uq[j] = reinterpret_cast<const uint4*>(A1 + args.I + cc)[j];
              }
            }
            tmem_ld32_sync(taddr + c0 + 32 * s2, r);
            if (s2 == 1 && c0 + 64 >= ce) release(acc);
            if (rv) {
#pragma unroll
              for (int j = 0; j < 4; ++j) {  // 8 columns at a time
                float dg[8], du[8];
                const uint32_t gw[4] = {gq[j].x, gq[j].y, gq[j].z, gq[j].w};
                const uint32_t uw[4] = {uq[j].x, uq[j].y, uq[j].z, uq[j].w};
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                  const float dh = __uint_as_float(r[8 * j + i]);
                  const float g = __uint_as_float(i & 1 ? gw[i >> 1] & 0xFFFF0000u : gw[i >> 1] << 16);
                  const float up =
                      __uint_as_float(i & 1 ? uw[i >> 1] & 0xFFFF0000u : uw[i >> 1] << 16);
                  const float sg = 1.0f / (1.0f + expf(-g));
                  dg[i] = dh * up * sg * (1.0f + g * (1.0f - sg));
                  du[i] = dh * g * sg;
                }
                const uint4 pg = pack_bf16x8(dg), pu = pack_bf16x8(du);
                if (staged) {
                  slot_put(slot, lane, 4 * s2 + j, pg);
                  upk[4 * s2 + j] = pu;
                } else {
                  reinterpret_cast<uint4*>(dA + cc)[j] = pg;
                  reinterpret_cast<uint4*>(dA + args.I + cc)[j] = pu;
                }
              }
            }
          }
          if (staged) {
            slot_issue<false>(slot, &tmO0, col, gr.out_row + rb, lane);
            staged_store<false>(slot, upk, &tmO0, args.I + col, gr.out_row + rb, lane);
          }
        }
        if (cb >= ce) release(acc);
      } else {  // DW2 / DW1: f32 output [G, m_out, n_out], 32 columns (128 B) a store
        const bool wvalid = rb < args.m_out;  // m_out % 32 == 0: all rows or none
        const bool write = wvalid && !((t.nkb == 0) && args.accumulate);
        const int cb = h * 128, ce = min(cb + 128, args.n_out - t.n0);
        const int y = t.g * args.m_out + rb;
        for (int c0 = cb; c0 < ce; c0 += 32) {
          if (t.nkb > 0) {
            tmem_ld32_sync(taddr + c0, r);
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) r[i] = 0u;
          }
          if (c0 + 32 >= ce) release(acc);
          if (write) {
            uint4 pk[8];
#pragma unroll
            for (int j = 0; j < 8; ++j)
              pk[j] = make_uint4(r[4 * j], r[4 * j + 1], r[4 * j + 2], r[4 * j + 3]);
            if (args.accumulate)
              staged_store<true>(slot, pk, &tmO0, t.n0 + c0, y, lane);
            else
              staged_store<false>(slot, pk, &tmO0, t.n0 + c0, y, lane);
          }
        }
        if (cb >= ce) release(acc);
      }
    }
    // every staged store has finished (written to global memory) before the CTA can exit
    if (lane == 0) {
      bulk_wait_all();
      if (args.ep.ret_ctr != 0) asm volatile("fence.proxy.async.global;" ::: "memory");
    }
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  // After an abort, copies the peer started for this pair may still be landing
  // (their completions are counted on the leader's barriers, which the
  // aborting roles stopped waiting on): give them time before either CTA leaves.
  if (*abort_flag && threadIdx.x == 0) spin_ns(100000);
  __syncthreads();
  cluster_sync();  // neither CTA leaves while the other may still signal it or use the pair's memory
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc_pair(tmem_base, TMEM_COLS);
  }
  // expert parallelism: once every CTA's output rows are in their sources'
  // buffers, the last CTA tells each source rank
  if (args.ep.ret_ctr != 0)
    ep_signal_last_cta(const_cast<int*>(args.ep.ep_ws) + args.ep.done_word, args.ep.peer_ws,
                       args.ep.world, args.ep.ret_ctr);
}

template <int MODE>
int launch_mode(const CUtensorMap& a0, const CUtensorMap& a1, const CUtensorMap& b0,
                const CUtensorMap& b1, const CUtensorMap& c, const CUtensorMap& o0,
                const CUtensorMap& o1, const CUtensorMap& a0h, const CUtensorMap& a1h,
                const CUtensorMap& bh, const EpMaps& epm, const GemmArgs& args, cudaStream_t st) {
  static int num_sms = 0;
  static bool attr_set = false;
  constexpr size_t kSmem = smem_bytes<MODE>();
  static_assert(kSmem <= 232448, "shared memory per CTA exceeds 227 KB");
  if (!attr_set) {
    if (!cuda_ok(cudaFuncSetAttribute(ggemm_kernel<MODE>,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmem)))
      return MOE_ERR_CUDA;
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&num_sms, cudaDevAttrMultiProcessorCount, dev);
    num_sms &= ~1;  // whole CTA pairs, one CTA per SM
    // A pair needs two co-scheduled SMs: launch only as many pairs as can be
    // resident at once (one persistent pair per two SMs; tiles are drawn at run time).
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)num_sms);
    cfg.blockDim = dim3(NUM_THREADS);
    cfg.dynamicSmemBytes = kSmem;
    int clusters = 0;
    if (cudaOccupancyMaxActiveClusters(&clusters, ggemm_kernel<MODE>, &cfg) == cudaSuccess &&
        clusters > 0 && 2 * clusters < num_sms)
      num_sms = 2 * clusters;
    cudaGetLastError();  // a failed query only leaves the default grid
    attr_set = true;
  }
  ggemm_kernel<MODE><<<num_sms, NUM_THREADS, kSmem, st>>>(a0, a1, b0, b1, c, o0, o1, a0h, a1h,
                                                          bh, epm, args);
  return cuda_ok(cudaGetLastError()) ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace

// ------------------------------------------------------------------ host side --
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn get_encode() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// Row-major matrix [rows, cols] (cols contiguous) of bf16 (esz 2) or f32 (esz 4);
// box = 128 bytes of a row x box_rows rows, 128-byte swizzle.
static bool make_map_2d(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, int esz,
                        int box_rows) {
  EncodeTiledFn enc = get_encode();
  if (!enc || base == nullptr) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)(cols * esz)};
  cuuint32_t box[2] = {(cuuint32_t)(128 / esz), (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1u, 1u};
  CUresult r = enc(m, esz == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                   2, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool make_map_bf16(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, int box_rows) {
  return make_map_2d(m, base, rows, cols, 2, box_rows);
}

// A row-major bf16 matrix [rows, cols] seen as 64-column chunks [cols / 64][rows][64]
// (the chunk index outermost, 128 bytes apart): one box = 64 rows of two adjacent
// chunks, landing in shared memory as chunk 0's 64 x 128-byte rows, then chunk 1's
// -- the layout of two 64-row 2-D boxes 8 KB apart.  False when cols is not a
// multiple of 64 or the driver does not take the map; the caller then keeps the
// 2-D boxes.
static bool make_map_mn3(CUtensorMap* m, const void* base, int64_t rows, int64_t cols) {
  EncodeTiledFn enc = get_encode();
  if (!enc || base == nullptr || rows <= 0 || cols % 64 != 0 || cols < 128) return false;
  cuuint64_t dims[3] = {64u, (cuuint64_t)rows, (cuuint64_t)(cols / 64)};
  cuuint64_t strides[2] = {(cuuint64_t)(cols * 2), 128u};
  cuuint32_t box[3] = {64u, 64u, 2u};
  cuuint32_t estr[3] = {1u, 1u, 1u};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

uint64_t wait_budget_ns() {
  static uint64_t v = [] {
    const char* s = getenv("MOE_WAIT_BUDGET_NS");
    return s ? strtoull(s, nullptr, 10) : 4000000000ull;
  }();
  return v;
}


int launch_grouped_gemm(GemmMode mode, const moe_dims& dm, const void* ws,
                        const GemmOperands& ops, void* stream) {
  const int G = dm.E + dm.S;
  if (G > MAX_GROUPS) return MOE_ERR_UNSUPPORTED_SHAPE;
  const WsLayout L = ws_layout(dm);
  const int64_t Rr = rows_routed(dm), Rt = rows_total(dm);
  const int64_t T = dm.T;
  const int d = dm.d, I = dm.I;
  const uint8_t* wsb = reinterpret_cast<const uint8_t*>(ws);

  GemmArgs a{};
  a.status = reinterpret_cast<int*>(const_cast<void*>(ws));
  a.groups = reinterpret_cast<const GroupRec*>(wsb + L.groups);
  a.mtile_prefix = reinterpret_cast<const int*>(wsb + L.mtile_prefix);
  a.dw_order = reinterpret_cast<const int*>(wsb + L.dw_order);
  a.tile_ctr = reinterpret_cast<int*>(const_cast<void*>(ws)) + kTileCtrWord + (int)mode;
  a.G = G;
  a.E = dm.E;
  a.I = I;
  a.out = ops.out;
  a.out2 = ops.out2;
  a.aux = ops.aux;
  a.accumulate = ops.accumulate;
  a.budget_ns = wait_budget_ns();
  a.shared_first = ops.shared_first;
  a.rows_total = Rt;
  a.rows_routed = Rr;
  a.rows_x = T;

  // expert parallelism: rows to wait for (FWD1 / DX2), outputs to return (FWD2 / DX1)
  EpMaps epm;
  memset(&epm, 0, sizeof(epm));
  if (ops.ep != nullptr) {
    const moe_ep_peers& pe = *ops.ep;
    const EpLayout EL = ep_layout(dm.E * pe.world, pe.world);
    const uint8_t* epb = reinterpret_cast<const uint8_t*>(pe.ep_ws[pe.rank]);
    a.ep.ep_ws = reinterpret_cast<const int*>(epb);
    a.ep.world = pe.world;
    a.ep.El = dm.E;
    a.ep.peer_ws = ep_ptrs(pe.ep_ws, pe.world);
    a.ep.recv_row = reinterpret_cast<const int32_t*>(epb + EL.recv_row);
    a.ep.src_off = reinterpret_cast<const int32_t*>(epb + EL.src_off);
    if (mode == MODE_FWD1) {  // each local expert's rows arrive on their own
      a.ep.wait_ctr = (int)(EL.arrive / sizeof(int32_t));
      a.ep.per_group = 1;
    } else if (mode == MODE_DX2) {
      a.ep.wait_ctr = EP_CTR_DY;
    } else if (mode == MODE_FWD2 || mode == MODE_DX1) {
      a.ep.ret_ctr = mode == MODE_FWD2 ? EP_CTR_Y : EP_CTR_DX;
      a.ep.done_word = mode == MODE_FWD2 ? EP_DONE_Y : EP_DONE_DX;
      for (int o = 0; o < pe.world; ++o)
        if (!make_map_2d(&epm.m[o], pe.rows[o], pe.rows_cap, dm.d, 2, 32)) return MOE_ERR_CUDA;
    }
  }

  CUtensorMap m0{}, m1{}, n0{}, n1{}, o0{}, o1{};
  CUtensorMap mh0{}, mh1{}, nh{};  // half tiles: 64-row boxes of A (and of B in FWD1);
                                   // DX / DW: 3-D chunk maps of A (mh) and B (nh)
  CUtensorMap cw{};                // DW1: 3-D chunk map of the shared groups' x
  bool ok = true;
  // a dummy map stands in for unused slots (never read by the kernel)
  auto same = [](CUtensorMap& dst, const CUtensorMap& src) { dst = src; };
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);

  switch (mode) {
    case MODE_FWD1: {
      const int hn = (I % 128 == 0) ? 128 : 64;
      a.hn = hn;
      a.K = d;
      a.NT = I / hn;
      a.n_out = I;
      a.b_group_rows = 2 * I;
      a.ld_out = I;
      a.ld_out2 = 2 * I;
      a.idesc = idesc_bf16_f32(PM, 2 * hn, false, false);
      ok &= make_map_bf16(&n0, ops.b0, (int64_t)G * 2 * I, d, hn);
      same(n1, n0);
      if (ops.gather_ids != nullptr) {
        // routed A rows gathered from x, one-row boxes (four rows a copy)
        a.gather_ids = ops.gather_ids;
        a.gather_T = (int)T;
        if (T > 0) ok &= make_map_bf16(&m0, ops.a1, T, d, 1); else same(m0, n0);
      } else {
        ok &= make_map_bf16(&m0, ops.a0, Rr, d, BM);
      }
      if (dm.S > 0 && T > 0) ok &= make_map_bf16(&m1, ops.a1, T, d, BM); else same(m1, m0);
      // a group's last <= 128 rows run as a half tile (M = 128), whose B rows are
      // staged as 64 gate + 64 up rows per CTA: needs hn == 128
      a.half_ok = hn == 128;
      a.idesc_h = idesc_bf16_f32(BM, 2 * hn, false, false);
      if (ops.gather_ids == nullptr) ok &= make_map_bf16(&mh0, ops.a0, Rr, d, BM / 2);
      else same(mh0, m0);
      if (dm.S > 0 && T > 0) ok &= make_map_bf16(&mh1, ops.a1, T, d, BM / 2); else same(mh1, mh0);
      ok &= make_map_bf16(&nh, ops.b0, (int64_t)G * 2 * I, d, BM / 2);
      if (!ok) return MOE_ERR_CUDA;
      // staged stores need 64 H columns per epilogue warp
      a.staged = hn == 128;
      ok &= make_map_2d(&o0, ops.out, Rt, I, 2, 32);
      if (ops.out2 != nullptr) ok &= make_map_2d(&o1, ops.out2, Rt, 2 * I, 2, 32); else same(o1, o0);
      if (!ok) return MOE_ERR_CUDA;
      return launch_mode<MODE_FWD1>(m0, m1, n0, n1, n0, o0, o1, mh0, mh1, nh, epm, a, st);
    }
    case MODE_FWD2: {
      a.K = I;
      a.NT = (d + 255) / 256;
      a.n_out = d;
      a.b_group_rows = d;
      a.ld_out = d;
      a.idesc = idesc_bf16_f32(PM, 256, false, false);
      ok &= make_map_bf16(&m0, ops.a0, Rt, I, BM);
      same(m1, m0);
      ok &= make_map_bf16(&n0, ops.b0, (int64_t)G * d, I, 128);
      same(n1, n0);
      a.half_ok = 1;
      a.idesc_h = idesc_bf16_f32(BM, 256, false, false);
      ok &= make_map_bf16(&mh0, ops.a0, Rt, I, BM / 2);
      same(mh1, mh0);
      same(nh, n0);
      if (!ok) return MOE_ERR_CUDA;
      a.staged = 1;
      if (!make_map_2d(&o0, ops.out, Rt, d, 2, 32)) return MOE_ERR_CUDA;
      return launch_mode<MODE_FWD2>(m0, m1, n0, n1, n0, o0, o0, mh0, mh1, nh, epm, a, st);
    }
    case MODE_DX2: {
      a.K = d;
      a.NT = (I + 255) / 256;
      a.n_out = I;
      a.b_group_rows = d;
      a.ld_out = 2 * I;
      a.ld_aux = 2 * I;
      a.idesc = idesc_bf16_f32(PM, 256, false, true);
      a.idesc_narrow = idesc_bf16_f32(PM, 128, false, true);
      ok &= make_map_bf16(&m0, ops.a0, Rr, d, BM);
      if (dm.S > 0 && T > 0) ok &= make_map_bf16(&m1, ops.a1, T, d, BM); else same(m1, m0);
      ok &= make_map_bf16(&n0, ops.b0, (int64_t)G * d, I, 64);
      same(n1, n0);
      a.half_ok = 1;
      a.idesc_h = idesc_bf16_f32(BM, 256, false, true);
      a.idesc_h_narrow = idesc_bf16_f32(BM, 128, false, true);
      ok &= make_map_bf16(&mh0, ops.a0, Rr, d, BM / 2);
      if (dm.S > 0 && T > 0) ok &= make_map_bf16(&mh1, ops.a1, T, d, BM / 2); else same(mh1, mh0);
      if (make_map_mn3(&nh, ops.b0, (int64_t)G * d, I)) a.mn3 = 2; else same(nh, n0);
      if (!ok) return MOE_ERR_CUDA;
      a.staged = 1;
      if (!make_map_2d(&o0, ops.out, Rt, 2 * I, 2, 32)) return MOE_ERR_CUDA;
      return launch_mode<MODE_DX2>(m0, m1, n0, n1, n0, o0, o0, mh0, mh1, nh, epm, a, st);
    }
    case MODE_DX1: {
      a.K = 2 * I;
      a.NT = (d + 255) / 256;
      a.n_out = d;
      a.b_group_rows = 2 * I;
      a.ld_out = d;
      a.idesc = idesc_bf16_f32(PM, 256, false, true);
      a.idesc_narrow = idesc_bf16_f32(PM, 128, false, true);
      ok &= make_map_bf16(&m0, ops.a0, Rt, 2 * I, BM);
      same(m1, m0);
      ok &= make_map_bf16(&n0, ops.b0, (int64_t)G * 2 * I, d, 64);
      same(n1, n0);
      a.half_ok = 1;
      a.idesc_h = idesc_bf16_f32(BM, 256, false, true);
      a.idesc_h_narrow = idesc_bf16_f32(BM, 128, false, true);
      ok &= make_map_bf16(&mh0, ops.a0, Rt, 2 * I, BM / 2);
      same(mh1, mh0);
      if (make_map_mn3(&nh, ops.b0, (int64_t)G * 2 * I, d)) a.mn3 = 2; else same(nh, n0);
      if (!ok) return MOE_ERR_CUDA;
      a.staged = 1;
      if (!make_map_2d(&o0, ops.out, Rt, d, 2, 32)) return MOE_ERR_CUDA;
      return launch_mode<MODE_DX1>(m0, m1, n0, n1, n0, o0, o0, mh0, mh1, nh, epm, a, st);
    }
    case MODE_DW2: {  // dW2_g [d, I] = dY_g^T H_g
      a.m_out = d;
      a.n_out = I;
      a.MT = (d + PM - 1) / PM;
      a.NT = (I + 255) / 256;
      a.idesc = idesc_bf16_f32(PM, 256, true, true);
      a.idesc_narrow = idesc_bf16_f32(PM, 128, true, true);
      ok &= make_map_bf16(&m0, ops.a0, Rr, d, 64);
      if (dm.S > 0 && T > 0) ok &= make_map_bf16(&m1, ops.a1, T, d, 64); else same(m1, m0);
      ok &= make_map_bf16(&n0, ops.b0, Rt, I, 64);
      same(n1, n0);
      if (!ok) return MOE_ERR_CUDA;
      if (make_map_mn3(&mh0, ops.a0, Rr, d) &&
          (dm.S > 0 && T > 0 ? make_map_mn3(&mh1, ops.a1, T, d) : (same(mh1, mh0), true)))
        a.mn3 |= 1;
      else
        same(mh0, m0), same(mh1, m0);
      if (make_map_mn3(&nh, ops.b0, Rt, I)) a.mn3 |= 2; else same(nh, n0);
      a.staged = 1;
      if (!make_map_2d(&o0, ops.out, (int64_t)G * d, I, 4, 32)) return MOE_ERR_CUDA;
      return launch_mode<MODE_DW2>(m0, m1, n0, n1, n0, o0, o0, mh0, mh1, nh, epm, a, st);
    }
    case MODE_DW1: {  // dW1_g [2I, d] = dA_g^T X_g
      a.m_out = 2 * I;
      a.n_out = d;
      a.MT = (2 * I + PM - 1) / PM;
      a.NT = (d + 255) / 256;
      a.idesc = idesc_bf16_f32(PM, 256, true, true);
      a.idesc_narrow = idesc_bf16_f32(PM, 128, true, true);
      ok &= make_map_bf16(&m0, ops.a0, Rt, 2 * I, 64);
      same(m1, m0);
      if (ops.gather_ids != nullptr) {
        // routed x rows (the reduction's K rows) gathered, four a copy
        a.gather_ids = ops.gather_ids;
        a.gather_T = (int)T;
        if (T > 0) ok &= make_map_bf16(&n0, ops.b1, T, d, 1); else same(n0, m0);
      } else {
        ok &= make_map_bf16(&n0, ops.b0, Rr, d, 64);
      }
      if (dm.S > 0 && T > 0) ok &= make_map_bf16(&n1, ops.b1, T, d, 64); else same(n1, n0);
      if (!ok) return MOE_ERR_CUDA;
      if (make_map_mn3(&mh0, ops.a0, Rt, 2 * I)) a.mn3 |= 1; else same(mh0, m0);
      same(mh1, mh0);
      {
        // B: the routed rows (unless gathered) and the shared groups' x rows
        const bool rb = ops.gather_ids != nullptr || make_map_mn3(&nh, ops.b0, Rr, d);
        const bool sb = !(dm.S > 0 && T > 0) || make_map_mn3(&cw, ops.b1, T, d);
        if (ops.gather_ids != nullptr) same(nh, n0);
        if (!(dm.S > 0 && T > 0)) same(cw, n0);
        if (rb && sb) a.mn3 |= 2; else same(nh, n0), same(cw, n0);
      }
      a.staged = 1;
      if (!make_map_2d(&o0, ops.out, (int64_t)G * 2 * I, d, 4, 32)) return MOE_ERR_CUDA;
      return launch_mode<MODE_DW1>(m0, m1, n0, n1, cw, o0, o0, mh0, mh1, nh, epm, a, st);
    }
  }
  return MOE_ERR_INVALID_ARG;
}

}  // namespace moe
