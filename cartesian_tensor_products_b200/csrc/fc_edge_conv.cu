// libflashcart: receiver-sorted edge convolution, forward (FlashCart
// Sec. 4 Eq. (1), Algorithm 1): C ABI entry point and the rank 1-4
// instantiations; the kernel templates and their design notes are in
// fc_edge_conv.cuh, rank 5 is instantiated in fc_edge_conv_L5.cu.
#include "fc_edge_conv.cuh"
#include "generated/fc_fwd_L1.cuh"
#include "generated/fc_fwd_L2.cuh"
#include "generated/fc_fwd_L3.cuh"
#include "generated/fc_fwd_L4.cuh"

namespace fc {
int launch_fwd_rank5(const ConvArgs& a, cudaStream_t s);
}  // namespace fc

using namespace fc;

extern "C" int fc_edge_conv_rect(const fc_conv_desc* d, int n_nodes, int n_send, int n_edges,
                                 const int32_t* rowptr, const int32_t* edge_index,
                                 const float* edge_vec, const float* x, const float* w, float* z,
                                 fc_stream_t stream) {
  cudaStream_t s = (cudaStream_t)stream;
  ConvArgs a;
  bool launch = false;
  int st = conv_setup(d, n_nodes, n_send, n_edges, rowptr, edge_index, edge_vec, x, w, z, 0, s, a,
                      &launch);
  if (st != FC_OK || !launch) return st;
  switch (d->lmax_in) {
    case 1: return launch_fwd<1>(a, s);
    case 2: return launch_fwd<2>(a, s);
    case 3: return launch_fwd<3>(a, s);
    case 4: return launch_fwd<4>(a, s);
    case 5: return launch_fwd_rank5(a, s);
    default: return FC_ERR_UNSUPPORTED_RANK;
  }
}

extern "C" int fc_edge_conv(const fc_conv_desc* d, int n_nodes, int n_edges,
                            const int32_t* rowptr, const int32_t* edge_index,
                            const float* edge_vec, const float* x, const float* w, float* z,
                            fc_stream_t stream) {
  return fc_edge_conv_rect(d, n_nodes, n_nodes, n_edges, rowptr, edge_index, edge_vec, x, w, z,
                           stream);
}

extern "C" size_t fc_edge_conv_workspace_size(const fc_conv_desc* d, int n_nodes, int n_edges) {
  (void)d;
  (void)n_nodes;
  (void)n_edges;
  return 0;   // the receiver sums stay on chip; no call of the convolution family needs scratch
}
