// libflashcart: vector-Jacobian product of the odd-J (Levi-Civita) path
// convolution (fc_edge_conv_odd).  FlashCart (arXiv 2610.06409) App. C
// Eq. (C1) summed as in Algorithm 2, with the odd-path coefficients (App. B,
// paragraph after Eq. (B1)); the kernel is the one of fc_edge_conv_vjp,
// instantiated with the odd-path tables under rank key L + kOddKey.
#include "fc_edge_conv_vjp.cuh"
#include "generated/fc_vjp_odd_L1.cuh"
#include "generated/fc_vjp_odd_L2.cuh"
#include "generated/fc_vjp_odd_L3.cuh"
#include "generated/fc_vjp_odd_L4.cuh"

using namespace fc;

extern "C" int fc_edge_conv_odd_vjp(const fc_conv_desc* d, int n_nodes, int n_edges,
                                    const int32_t* rowptr, const int32_t* edge_index,
                                    const float* edge_vec, const float* x, const float* w,
                                    const float* g, float* x_bar, float* w_bar, float* r_bar,
                                    fc_stream_t stream) {
  cudaStream_t s = (cudaStream_t)stream;
  VjpArgs a;
  bool launch = false;
  int st = vjp_setup(d, n_nodes, n_nodes, n_edges, rowptr, edge_index, edge_vec, x, w, g, x_bar,
                     w_bar, r_bar, 1, s, a, &launch);
  if (st != FC_OK || !launch) return st;
  switch (d->lmax_in) {
    case 1: return launch_vjp<1 + kOddKey>(a, s);
    case 2: return launch_vjp<2 + kOddKey>(a, s);
    case 3: return launch_vjp<3 + kOddKey>(a, s);
    case 4: return launch_vjp<4 + kOddKey>(a, s);
    default: return FC_ERR_UNSUPPORTED_RANK;
  }
}
