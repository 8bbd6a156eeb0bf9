// libflashcart: C ABI of the VJP-of-VJP of the edge convolution (FlashCart
// App. C Eq. C2, Algorithm 3); the kernels are in fc_edge_conv_vvjp.cuh.
#include "fc_edge_conv_vvjp.cuh"

namespace fc {
int launch_vvjp_rank1(const VvjpArgs& a, cudaStream_t s);
int launch_vvjp_rank2(const VvjpArgs& a, cudaStream_t s);
int launch_vvjp_rank3(const VvjpArgs& a, cudaStream_t s);
int launch_vvjp_rank4(const VvjpArgs& a, cudaStream_t s);
int launch_vvjp_rank5_part0(const VvjpArgs& a, cudaStream_t s);
int launch_vvjp_rank5_part1(const VvjpArgs& a, cudaStream_t s);
int launch_vvjp_rank5_part2(const VvjpArgs& a, cudaStream_t s);
int launch_vvjp_rank5_part3(const VvjpArgs& a, cudaStream_t s);

// rank 5: one launch per path group, in four ranges
static int launch_vvjp_rank5(const VvjpArgs& a, cudaStream_t s) {
  int st;
  if ((st = launch_vvjp_rank5_part0(a, s)) != FC_OK || (st = launch_vvjp_rank5_part1(a, s)) != FC_OK ||
      (st = launch_vvjp_rank5_part2(a, s)) != FC_OK)
    return st;
  return launch_vvjp_rank5_part3(a, s);
}
}  // namespace fc

using namespace fc;

extern "C" int fc_edge_conv_vjp_vjp(const fc_conv_desc* d, int n_nodes, int n_edges,
                                    const int32_t* rowptr, const int32_t* edge_index,
                                    const float* edge_vec, const float* x, const float* w,
                                    const float* g, const float* v_x, const float* v_w,
                                    const float* v_r, float* g_hat, float* x_hat, float* w_hat,
                                    float* r_hat, fc_stream_t stream) {
  int st = check_conv_desc(d);
  if (st != FC_OK) return st;
  if (d->envelope) return FC_ERR_ARG;
  if (n_nodes < 0 || n_edges < 0) return FC_ERR_ARG;
  if (n_nodes == 0) return n_edges == 0 ? FC_OK : FC_ERR_ARG;
  if (!rowptr || !x || !g) return FC_ERR_ARG;
  if (n_edges > 0 && (!edge_index || !edge_vec || !w)) return FC_ERR_ARG;
  if (!aligned16(x) || !aligned16(g) || (w && !aligned16(w)) || (v_x && !aligned16(v_x)) ||
      (v_w && !aligned16(v_w)) || (v_r && !aligned4(v_r)) || (g_hat && !aligned16(g_hat)) ||
      (x_hat && !aligned16(x_hat)) || (w_hat && !aligned16(w_hat)) || (r_hat && !aligned4(r_hat)) ||
      !aligned4(rowptr) || (edge_index && !aligned4(edge_index)) ||
      (edge_vec && !aligned4(edge_vec)))
    return FC_ERR_ALIGN;
  const int L = d->lmax_in;
  const int C = d->channels;
  VvjpArgs a;
  a.rowptr = rowptr;
  a.send = edge_index ? edge_index + n_edges : nullptr;
  a.vec = edge_vec;
  a.x = x;
  a.w = w;
  a.g = g;
  a.vx = v_x;
  a.vw = v_w;
  a.vr = v_r;
  a.ghat = g_hat;
  a.xhat = x_hat;
  a.what = w_hat;
  a.rhat = r_hat;
  a.n_nodes = n_nodes;
  a.n_send = n_nodes;
  a.n_edges = n_edges;
  a.C = C;
  a.ntiles = (C + 127) / 128;
  a.xrow = (L + 1) * (L + 1);
  a.zrow = out_row(L, d->sum_paths);
  a.P = num_paths(L);
  a.sum_paths = d->sum_paths;
  if ((long long)n_nodes * a.ntiles > 0x7fffffffLL) return FC_ERR_ARG;
  cudaStream_t s = (cudaStream_t)stream;
  if (g_hat && cudaMemsetAsync(g_hat, 0, sizeof(float) * (size_t)n_nodes * a.zrow * C, s) != cudaSuccess)
    return FC_ERR_CUDA;
  if (x_hat && cudaMemsetAsync(x_hat, 0, sizeof(float) * (size_t)n_nodes * a.xrow * C, s) != cudaSuccess)
    return FC_ERR_CUDA;
  if (r_hat && n_edges > 0 &&
      cudaMemsetAsync(r_hat, 0, sizeof(float) * 3 * (size_t)n_edges, s) != cudaSuccess)
    return FC_ERR_CUDA;
  if (w_hat && n_edges > 0 && !v_x && !v_r &&
      cudaMemsetAsync(w_hat, 0, sizeof(float) * (size_t)n_edges * a.P * C, s) != cudaSuccess)
    return FC_ERR_CUDA;
  if (n_edges == 0) return FC_OK;
  if (!g_hat && !x_hat && !w_hat && !r_hat) return FC_OK;
  switch (L) {
    case 1: return launch_vvjp_rank1(a, s);
    case 2: return launch_vvjp_rank2(a, s);
    case 3: return launch_vvjp_rank3(a, s);
    case 4: return launch_vvjp_rank4(a, s);
    case 5: return launch_vvjp_rank5(a, s);
    default: return FC_ERR_UNSUPPORTED_RANK;
  }
}
