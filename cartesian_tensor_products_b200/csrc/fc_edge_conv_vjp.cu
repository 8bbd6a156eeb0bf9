// libflashcart: receiver-sorted edge convolution, vector-Jacobian product (FlashCart
// App. C Eq. (C1), Algorithm 2): C ABI entry point and the rank 1-4
// instantiations; the kernel templates and their design notes are in
// fc_edge_conv_vjp.cuh, rank 5 is instantiated in fc_edge_conv_vjp_L5.cu.
#include "fc_edge_conv_vjp.cuh"
#include "generated/fc_vjp_L1.cuh"
#include "generated/fc_vjp_L2.cuh"
#include "generated/fc_vjp_L3.cuh"
#include "generated/fc_vjp_L4.cuh"

namespace fc {
int launch_vjp_rank5(const VjpArgs& a, cudaStream_t s);
}  // namespace fc

using namespace fc;

extern "C" int fc_edge_conv_vjp_rect(const fc_conv_desc* d, int n_nodes, int n_send, int n_edges,
                                     const int32_t* rowptr, const int32_t* edge_index,
                                     const float* edge_vec, const float* x, const float* w,
                                     const float* g, float* x_bar, float* w_bar, float* r_bar,
                                     fc_stream_t stream) {
  int st = check_conv_desc(d);
  if (st != FC_OK) return st;
  if (n_nodes < 0 || n_send < 0 || n_edges < 0) return FC_ERR_ARG;
  if (n_nodes == 0) return n_edges == 0 ? FC_OK : FC_ERR_ARG;
  if (!rowptr || !x || !g) return FC_ERR_ARG;
  if (n_edges > 0 && (!edge_index || !edge_vec || !w)) return FC_ERR_ARG;
  if (!aligned16(x) || !aligned16(g) || (w && !aligned16(w)) || (x_bar && !aligned16(x_bar)) ||
      (w_bar && !aligned16(w_bar)) || (r_bar && !aligned4(r_bar)) || !aligned4(rowptr) ||
      (edge_index && !aligned4(edge_index)) || (edge_vec && !aligned4(edge_vec)))
    return FC_ERR_ALIGN;
  const int L = d->lmax_in;
  const int C = d->channels;
  VjpArgs a;
  a.rowptr = rowptr;
  a.send = edge_index ? edge_index + n_edges : nullptr;
  a.vec = edge_vec;
  a.x = x;
  a.w = w;
  a.g = g;
  a.xbar = x_bar;
  a.wbar = w_bar;
  a.rbar = r_bar;
  a.n_nodes = n_nodes;
  a.n_send = n_send;
  a.n_edges = n_edges;
  a.C = C;
  a.ntiles = (C + 127) / 128;
  a.xrow = (L + 1) * (L + 1);
  a.zrow = out_row(L, d->sum_paths);
  a.P = num_paths(L);
  a.sum_paths = d->sum_paths;
  a.envelope = d->envelope;
  a.r_cut = d->r_cut;
  a.edge_scale = d->edge_scale;
  if ((long long)n_nodes * a.ntiles > 0x7fffffffLL) return FC_ERR_ARG;
  cudaStream_t s = (cudaStream_t)stream;
  if (x_bar && cudaMemsetAsync(x_bar, 0, sizeof(float) * (size_t)n_send * a.xrow * C, s) != cudaSuccess)
    return FC_ERR_CUDA;
  if (r_bar && n_edges > 0 &&
      cudaMemsetAsync(r_bar, 0, sizeof(float) * 3 * (size_t)n_edges, s) != cudaSuccess)
    return FC_ERR_CUDA;
  if (n_edges == 0) return FC_OK;
  if (!x_bar && !w_bar && !r_bar) return FC_OK;
  switch (L) {
    case 1: return launch_vjp<1>(a, s);
    case 2: return launch_vjp<2>(a, s);
    case 3: return launch_vjp<3>(a, s);
    case 4: return launch_vjp<4>(a, s);
    case 5: return launch_vjp_rank5(a, s);
    default: return FC_ERR_UNSUPPORTED_RANK;
  }
}

extern "C" int fc_edge_conv_vjp(const fc_conv_desc* d, int n_nodes, int n_edges,
                                const int32_t* rowptr, const int32_t* edge_index,
                                const float* edge_vec, const float* x, const float* w,
                                const float* g, float* x_bar, float* w_bar, float* r_bar,
                                fc_stream_t stream) {
  return fc_edge_conv_vjp_rect(d, n_nodes, n_nodes, n_edges, rowptr, edge_index, edge_vec, x, w, g,
                               x_bar, w_bar, r_bar, stream);
}
