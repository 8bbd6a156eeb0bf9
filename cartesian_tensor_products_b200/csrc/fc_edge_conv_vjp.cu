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
  cudaStream_t s = (cudaStream_t)stream;
  VjpArgs a;
  bool launch = false;
  int st = vjp_setup(d, n_nodes, n_send, n_edges, rowptr, edge_index, edge_vec, x, w, g, x_bar,
                     w_bar, r_bar, 0, s, a, &launch);
  if (st != FC_OK || !launch) return st;
  switch (d->lmax_in) {
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
