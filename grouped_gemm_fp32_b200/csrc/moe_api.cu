// moe_api.cu -- the extern "C" entry points of libmoe.so: argument and shape
// validation, then the launches.  No allocation, no host synchronisation
// (except moe_get_device_status), nothing but plain pointers and sizes.
#include <cuda_runtime.h>

#include "ep_internal.cuh"
#include "moe_internal.cuh"

using namespace moe;

namespace moe {

namespace {
thread_local cudaError_t g_last_error = cudaSuccess;
}

bool cuda_ok(cudaError_t e) {
  if (e == cudaSuccess) return true;
  g_last_error = e;
  return false;
}

}  // namespace moe

namespace moe {

bool dims_ok(const moe_dims* dm) {
  if (!dm) return false;
  if (dm->T < 0 || dm->d <= 0 || dm->E <= 0 || dm->k <= 0 || dm->S < 0 || dm->I <= 0 ||
      dm->P <= 0)
    return false;
  return true;
}

// Shapes the kernels support (see include/moe.h).
int check_shape(const moe_dims* dm, bool need_bwd) {
  if (!dims_ok(dm)) return MOE_ERR_INVALID_ARG;
  if (dm->d % 64 || dm->I % 64) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (dm->E > 256 || dm->k > dm->E || dm->S > 8) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (dm->P % 8 || dm->P < 8) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (need_bwd && dm->P % 64) return MOE_ERR_UNSUPPORTED_SHAPE;
  // rows and (t, j) indices are int32 on the device
  if (rows_total(*dm) >= (int64_t(1) << 31) || dm->T * dm->k >= (int64_t(1) << 31))
    return MOE_ERR_UNSUPPORTED_SHAPE;
  if (rows_routed(*dm) < 0) return MOE_ERR_INVALID_ARG;
  return MOE_OK;
}

}  // namespace moe

namespace {

bool ws_ok(const moe_dims* dm, const void* ws, size_t bytes) {
  return ws != nullptr && bytes >= ws_layout(*dm).bytes;
}

}  // namespace

extern "C" {

int64_t moe_rows_routed(const moe_dims* dims) { return dims_ok(dims) ? rows_routed(*dims) : -1; }
int64_t moe_rows_total(const moe_dims* dims) { return dims_ok(dims) ? rows_total(*dims) : -1; }

size_t moe_workspace_size(const moe_dims* dims) {
  return dims_ok(dims) ? ws_layout(*dims).total : 0;
}

int moe_gate_topk(const moe_dims* dims, const void* x, const float* wg, const float* bias,
                  int32_t* topk_idx, float* topk_w, float* probs, void* ws, size_t ws_bytes,
                  void* stream) {
  int rc = check_shape(dims, false);
  if (rc) return rc;
  if (dims->E % 8) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (!ws || ws_bytes < ws_layout(*dims).total) return MOE_ERR_INVALID_ARG;
  if (dims->T > 0 && (!x || !wg || !topk_idx || !topk_w)) return MOE_ERR_INVALID_ARG;
  return launch_gate_topk(*dims, x, wg, bias, topk_idx, topk_w, probs, ws, stream);
}

int moe_router_bwd(const moe_dims* dims, const void* x, const float* wg, const float* probs,
                   const int32_t* topk_idx, const float* topk_w, const float* dw, float* dlogits,
                   void* dx, float* dwg, int accumulate, void* ws, size_t ws_bytes,
                   void* stream) {
  int rc = check_shape(dims, false);
  if (rc) return rc;
  if (dims->E % 8) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (!ws || ws_bytes < ws_layout(*dims).total || !wg || !dwg) return MOE_ERR_INVALID_ARG;
  if (dims->T > 0 && (!x || !probs || !topk_idx || !topk_w || !dw || !dx))
    return MOE_ERR_INVALID_ARG;
  return launch_router_bwd(*dims, x, wg, probs, topk_idx, topk_w, dw, nullptr, 1, dlogits, dx,
                           dwg, accumulate ? 1 : 0, ws, stream);
}

int moe_router_bwd_seqbal(const moe_dims* dims, const void* x, const float* wg,
                          const float* probs, const int32_t* topk_idx, const float* topk_w,
                          const float* dw, const float* seq_grad, int64_t seq_len,
                          float* dlogits, void* dx, float* dwg, int accumulate, void* ws,
                          size_t ws_bytes, void* stream) {
  int rc = check_shape(dims, false);
  if (rc) return rc;
  if (dims->E % 8) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (!ws || ws_bytes < ws_layout(*dims).total || !wg || !dwg) return MOE_ERR_INVALID_ARG;
  if (dims->T > 0 && (!x || !probs || !topk_idx || !topk_w || !dw || !dx || !seq_grad ||
                      seq_len < kSeqMin))
    return MOE_ERR_INVALID_ARG;
  return launch_router_bwd(*dims, x, wg, probs, topk_idx, topk_w, dw, seq_grad, seq_len,
                           dlogits, dx, dwg, accumulate ? 1 : 0, ws, stream);
}

int moe_seq_balance_loss(const moe_dims* dims, int64_t seq_len, float alpha,
                         const int32_t* topk_idx, const float* probs, float* loss,
                         float* seq_grad, void* ws, size_t ws_bytes, void* stream) {
  int rc = check_shape(dims, false);
  if (rc) return rc;
  if (seq_len < kSeqMin) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (!ws || ws_bytes < ws_layout(*dims).total || !loss) return MOE_ERR_INVALID_ARG;
  if (dims->T > 0 && (!topk_idx || !probs || !seq_grad)) return MOE_ERR_INVALID_ARG;
  return launch_seq_balance(*dims, seq_len, alpha, topk_idx, probs, loss, seq_grad, ws, stream);
}

int moe_bias_update(const moe_dims* dims, const int32_t* counts, float gamma,
                    const float* bias_in, float* bias_out, void* stream) {
  if (!dims_ok(dims)) return MOE_ERR_INVALID_ARG;
  if (!counts || !bias_in || !bias_out) return MOE_ERR_INVALID_ARG;
  return launch_bias_update(*dims, counts, gamma, bias_in, bias_out, stream);
}

int moe_permute_align(const moe_dims* dims, const int32_t* topk_idx, const void* x,
                      int32_t* counts, int32_t* offsets, int32_t* sorted_ids, int32_t* row_of,
                      void* x_perm, void* ws, size_t ws_bytes, void* stream) {
  int rc = check_shape(dims, false);
  if (rc) return rc;
  if (!counts || !offsets || !sorted_ids || !ws_ok(dims, ws, ws_bytes)) return MOE_ERR_INVALID_ARG;
  if (dims->T > 0 && (!topk_idx || !row_of || (x_perm && !x))) return MOE_ERR_INVALID_ARG;
  return launch_permute(*dims, topk_idx, x, counts, offsets, sorted_ids, row_of, x_perm, ws,
                        stream);
}

int grouped_gemm_set_groups(const moe_dims* dims, const int32_t* counts, int32_t* offsets,
                            void* ws, size_t ws_bytes, void* stream) {
  int rc = check_shape(dims, false);
  if (rc) return rc;
  if (!counts || !offsets || !ws_ok(dims, ws, ws_bytes)) return MOE_ERR_INVALID_ARG;
  return launch_set_groups(*dims, counts, offsets, ws, stream);
}

// FWD1 then FWD2; routed A rows from x_perm, or gathered from x by sorted_ids.
static int gemm_fwd(const moe_dims* dims, const void* ws, const void* x_perm,
                    const int32_t* sorted_ids, const void* x, const void* w1, const void* w2,
                    void* h, void* a1, void* y, void* stream) {
  GemmOperands o{};
  o.a0 = x_perm;
  o.a1 = x;
  o.b0 = w1;
  o.out = h;
  o.out2 = a1;
  o.gather_ids = sorted_ids;
  int rc = launch_grouped_gemm(MODE_FWD1, *dims, ws, o, stream);
  if (rc) return rc;
  GemmOperands o2{};
  o2.a0 = h;
  o2.b0 = w2;
  o2.out = y;
  return launch_grouped_gemm(MODE_FWD2, *dims, ws, o2, stream);
}

int grouped_gemm_fwd(const moe_dims* dims, const void* ws, const void* x_perm, const void* x,
                     const void* w1, const void* w2, void* h, void* a1, void* y, void* stream) {
  int rc = check_shape(dims, false);
  if (rc) return rc;
  if (!ws || !x_perm || !w1 || !w2 || !h || !y || (dims->S > 0 && dims->T > 0 && !x)) return MOE_ERR_INVALID_ARG;
  return gemm_fwd(dims, ws, x_perm, nullptr, x, w1, w2, h, a1, y, stream);
}

int grouped_gemm_fwd_gather(const moe_dims* dims, const void* ws, const int32_t* sorted_ids,
                            const void* x, const void* w1, const void* w2, void* h, void* a1,
                            void* y, void* stream) {
  int rc = check_shape(dims, false);
  if (rc) return rc;
  if (!ws || !sorted_ids || !w1 || !w2 || !h || !y || (dims->T > 0 && !x)) return MOE_ERR_INVALID_ARG;
  return gemm_fwd(dims, ws, nullptr, sorted_ids, x, w1, w2, h, a1, y, stream);
}

int grouped_gemm_bwd_dx(const moe_dims* dims, const void* ws, int which, const void* dy_routed,
                        const void* dy_shared, const void* w, const void* a1, void* out,
                        void* stream) {
  int rc = check_shape(dims, true);
  if (rc) return rc;
  if (!ws || !dy_routed || !w || !out) return MOE_ERR_INVALID_ARG;
  GemmOperands o{};
  o.a0 = dy_routed;
  o.b0 = w;
  o.out = out;
  if (which == MOE_GEMM2) {
    if (!a1 || (dims->S > 0 && dims->T > 0 && !dy_shared)) return MOE_ERR_INVALID_ARG;
    o.a1 = dy_shared;
    o.aux = a1;
    return launch_grouped_gemm(MODE_DX2, *dims, ws, o, stream);
  }
  if (which == MOE_GEMM1) return launch_grouped_gemm(MODE_DX1, *dims, ws, o, stream);
  return MOE_ERR_INVALID_ARG;
}

int grouped_gemm_bwd_dw(const moe_dims* dims, const void* ws, int which, const void* lhs_routed,
                        const void* lhs_shared, const void* rhs_routed, const void* rhs_shared,
                        float* dw, int accumulate, void* stream) {
  int rc = check_shape(dims, true);
  if (rc) return rc;
  if (!ws || !lhs_routed || !rhs_routed || !dw || (accumulate != 0 && accumulate != 1))
    return MOE_ERR_INVALID_ARG;
  GemmOperands o{};
  o.a0 = lhs_routed;
  o.b0 = rhs_routed;
  o.out = dw;
  o.accumulate = accumulate;
  if (which == MOE_GEMM2) {
    if (dims->S > 0 && dims->T > 0 && !lhs_shared) return MOE_ERR_INVALID_ARG;
    o.a1 = lhs_shared;
    return launch_grouped_gemm(MODE_DW2, *dims, ws, o, stream);
  }
  if (which == MOE_GEMM1) {
    if (dims->S > 0 && dims->T > 0 && !rhs_shared) return MOE_ERR_INVALID_ARG;
    o.b1 = rhs_shared;
    return launch_grouped_gemm(MODE_DW1, *dims, ws, o, stream);
  }
  return MOE_ERR_INVALID_ARG;
}

int grouped_gemm_bwd_dw1_gather(const moe_dims* dims, const void* ws, const int32_t* sorted_ids,
                                const void* da, const void* x, float* dw1, int accumulate,
                                void* stream) {
  int rc = check_shape(dims, true);
  if (rc) return rc;
  if (!ws || !sorted_ids || !da || !dw1 || (dims->T > 0 && !x) ||
      (accumulate != 0 && accumulate != 1))
    return MOE_ERR_INVALID_ARG;
  GemmOperands o{};
  o.a0 = da;
  o.b1 = x;
  o.out = dw1;
  o.accumulate = accumulate;
  o.gather_ids = sorted_ids;
  return launch_grouped_gemm(MODE_DW1, *dims, ws, o, stream);
}

int moe_combine(const moe_dims* dims, const void* y, const int32_t* row_of, const float* topk_w,
                void* out, void* stream) {
  int rc = check_shape(dims, false);
  if (rc) return rc;
  if (dims->T > 0 && (!y || !row_of || !out)) return MOE_ERR_INVALID_ARG;
  return launch_combine(*dims, y, nullptr, row_of, topk_w, out, false, stream);
}

int moe_combine_split(const moe_dims* dims, const void* y_routed, const void* y_shared,
                      const int32_t* row_of, const float* topk_w, void* out, void* stream) {
  int rc = check_shape(dims, false);
  if (rc) return rc;
  if (dims->T > 0 && (!y_routed || !row_of || !out || (dims->S > 0 && !y_shared)))
    return MOE_ERR_INVALID_ARG;
  return launch_combine(*dims, y_routed, dims->S > 0 ? y_shared : y_routed, row_of, topk_w, out,
                        false, stream);
}

int moe_combine_f32(const moe_dims* dims, const void* y, const int32_t* row_of,
                    const float* topk_w, float* out, void* stream) {
  int rc = check_shape(dims, false);
  if (rc) return rc;
  if (dims->T > 0 && (!y || !row_of || !out)) return MOE_ERR_INVALID_ARG;
  return launch_combine(*dims, y, nullptr, row_of, topk_w, out, true, stream);
}

int moe_combine_bwd(const moe_dims* dims, const void* ws, const void* dout, const void* y,
                    const int32_t* row_of, const float* topk_w, void* dy_routed, float* dw,
                    void* stream) {
  int rc = check_shape(dims, false);
  if (rc) return rc;
  if (!ws || !dy_routed) return MOE_ERR_INVALID_ARG;
  if (dims->T > 0 && (!dout || !y || !row_of || !topk_w || !dw)) return MOE_ERR_INVALID_ARG;
  return launch_combine_bwd(*dims, ws, dout, y, row_of, topk_w, dy_routed, dw, stream);
}

// ------------------------------------------------------ expert parallelism --
static int check_ep(const moe_dims* dims, const moe_ep_peers* peers, bool need_rows) {
  int rc = check_shape(dims, false);
  if (rc) return rc;
  if (!ep_peers_ok(peers, need_rows)) return MOE_ERR_INVALID_ARG;
  if (dims->E % peers->world || dims->P % 32 || dims->k > 32) return MOE_ERR_UNSUPPORTED_SHAPE;
  return MOE_OK;
}

size_t moe_ep_workspace_size(const moe_dims* dims, int32_t world) {
  if (!dims_ok(dims) || world < 1 || world > MOE_EP_MAX_WORLD || dims->E % world) return 0;
  return ep_layout(dims->E, world).bytes;
}

int moe_ep_plan(const moe_dims* dims, const moe_ep_peers* peers, const int32_t* counts_all,
                int32_t* counts_loc, int64_t recv_cap, void* stream) {
  int rc = check_ep(dims, peers, false);
  if (rc) return rc;
  if (!counts_all || !counts_loc || recv_cap < 0) return MOE_ERR_INVALID_ARG;
  return launch_ep_plan(*dims, *peers, counts_all, counts_loc, recv_cap, stream);
}

int moe_ep_dispatch(const moe_dims* dims, const moe_ep_peers* peers, const int32_t* sorted_ids,
                    const int32_t* offsets, const void* x, void* stream) {
  int rc = check_ep(dims, peers, true);
  if (rc) return rc;
  if (!offsets || !sorted_ids || (dims->T > 0 && !x)) return MOE_ERR_INVALID_ARG;
  return launch_ep_dispatch(*dims, *peers, sorted_ids, offsets, x, stream);
}

int moe_ep_zero_pads(const moe_dims* dims, const moe_ep_peers* peers, void* recv, void* stream) {
  int rc = check_ep(dims, peers, false);
  if (rc) return rc;
  if (!recv) return MOE_ERR_INVALID_ARG;
  return launch_ep_zero_pads(*dims, *peers, recv, stream);
}

int moe_ep_wait(const moe_ep_peers* peers, int which, void* stream) {
  if (!ep_peers_ok(peers, false)) return MOE_ERR_INVALID_ARG;
  if (which != MOE_EP_WAIT_Y && which != MOE_EP_WAIT_DX) return MOE_ERR_INVALID_ARG;
  return launch_ep_wait(*peers, which, stream);
}

int moe_ep_combine_bwd(const moe_dims* dims, const moe_ep_peers* peers, const void* dout,
                       const void* y, const int32_t* row_of, const float* topk_w,
                       const int32_t* topk_idx, const int32_t* offsets, float* dw, void* stream) {
  int rc = check_ep(dims, peers, true);
  if (rc) return rc;
  if (!offsets || (dims->T > 0 && (!dout || !y || !row_of || !topk_w || !topk_idx || !dw)))
    return MOE_ERR_INVALID_ARG;
  return launch_combine_bwd_ep(*dims, *peers, dout, y, row_of, topk_w, topk_idx, offsets, dw,
                               stream);
}

// The local dims of an owner: E_l routed groups; its peers' ep workspaces were sized
// for E = E_l W.
static int check_ep_local(const moe_dims* dims, const moe_ep_peers* peers, bool need_rows) {
  int rc = check_shape(dims, true);
  if (rc) return rc;
  if (!ep_peers_ok(peers, need_rows)) return MOE_ERR_INVALID_ARG;
  if (dims->P % 32 || (int64_t)dims->E * peers->world > 256) return MOE_ERR_UNSUPPORTED_SHAPE;
  return MOE_OK;
}

int grouped_gemm_fwd_ep(const moe_dims* dims, const void* ws, const moe_ep_peers* peers,
                        const void* x_recv, const void* x, const void* w1, const void* w2,
                        void* h, void* a1, void* y, void* stream) {
  int rc = check_ep_local(dims, peers, true);
  if (rc) return rc;
  if (!ws || !x_recv || !w1 || !w2 || !h || !y || (dims->S > 0 && dims->T > 0 && !x))
    return MOE_ERR_INVALID_ARG;
  GemmOperands o{};
  o.a0 = x_recv;
  o.a1 = x;
  o.b0 = w1;
  o.out = h;
  o.out2 = a1;
  o.ep = peers;
  o.shared_first = 1;
  rc = launch_grouped_gemm(MODE_FWD1, *dims, ws, o, stream);
  if (rc) return rc;
  GemmOperands o2{};
  o2.a0 = h;
  o2.b0 = w2;
  o2.out = y;
  o2.ep = peers;
  return launch_grouped_gemm(MODE_FWD2, *dims, ws, o2, stream);
}

int grouped_gemm_bwd_dx_ep(const moe_dims* dims, const void* ws, const moe_ep_peers* peers,
                           int which, const void* dy_recv, const void* dy_shared, const void* w,
                           const void* a1, void* out, void* stream) {
  int rc = check_ep_local(dims, peers, which == MOE_GEMM1);
  if (rc) return rc;
  if (!ws || !dy_recv || !w || !out) return MOE_ERR_INVALID_ARG;
  GemmOperands o{};
  o.a0 = dy_recv;
  o.b0 = w;
  o.out = out;
  o.ep = peers;
  if (which == MOE_GEMM2) {
    if (!a1 || (dims->S > 0 && dims->T > 0 && !dy_shared)) return MOE_ERR_INVALID_ARG;
    o.a1 = dy_shared;
    o.aux = a1;
    o.shared_first = 1;
    return launch_grouped_gemm(MODE_DX2, *dims, ws, o, stream);
  }
  if (which == MOE_GEMM1) return launch_grouped_gemm(MODE_DX1, *dims, ws, o, stream);
  return MOE_ERR_INVALID_ARG;
}

int moe_get_device_status(void* ws, int32_t* status_out, void* stream) {
  if (!ws || !status_out) return MOE_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int32_t v = 0;
  if (!cuda_ok(cudaMemcpyAsync(&v, ws, sizeof(int32_t), cudaMemcpyDeviceToHost, st)) ||
      !cuda_ok(cudaStreamSynchronize(st)))
    return MOE_ERR_CUDA;
  if (!cuda_ok(cudaMemsetAsync(ws, 0, sizeof(int32_t), st)) || !cuda_ok(cudaStreamSynchronize(st)))
    return MOE_ERR_CUDA;
  *status_out = v;
  return MOE_OK;
}

const char* moe_last_cuda_error(void) {
  return g_last_error == cudaSuccess ? "no error" : cudaGetErrorString(g_last_error);
}

const char* moe_status_string(int status) {
  switch (status) {
    case MOE_OK: return "MOE_OK";
    case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG";
    case MOE_ERR_UNSUPPORTED_SHAPE: return "MOE_ERR_UNSUPPORTED_SHAPE";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA";
    case MOE_ERR_DEVICE_TIMEOUT: return "MOE_ERR_DEVICE_TIMEOUT";
    case MOE_ERR_BAD_ROUTING: return "MOE_ERR_BAD_ROUTING";
    default: return "MOE_ERR_UNKNOWN";
  }
}

}  // extern "C"
