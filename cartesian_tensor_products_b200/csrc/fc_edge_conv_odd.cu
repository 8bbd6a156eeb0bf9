// libflashcart: edge convolution over the odd-J (Levi-Civita) paths,
// forward.  FlashCart (arXiv 2610.06409) App. B, paragraph after Eq. (B1),
// and Sec. 7: the products of opposite parity, one index of each input
// contracted through the Levi-Civita symbol, the output a pseudo-tensor.
// Same receiver-sorted kernel as fc_edge_conv (Sec. 4 Eq. (1), Algorithm
// 1), instantiated with the odd-path tables under rank key L + kOddKey.
#include "fc_edge_conv.cuh"
#include "generated/fc_fwd_odd_L1.cuh"
#include "generated/fc_fwd_odd_L2.cuh"
#include "generated/fc_fwd_odd_L3.cuh"
#include "generated/fc_fwd_odd_L4.cuh"

using namespace fc;

extern "C" int fc_edge_conv_odd(const fc_conv_desc* d, int n_nodes, int n_edges,
                                const int32_t* rowptr, const int32_t* edge_index,
                                const float* edge_vec, const float* x, const float* w, float* z,
                                fc_stream_t stream) {
  cudaStream_t s = (cudaStream_t)stream;
  ConvArgs a;
  bool launch = false;
  int st = conv_setup(d, n_nodes, n_nodes, n_edges, rowptr, edge_index, edge_vec, x, w, z, 1, s, a,
                      &launch);
  if (st != FC_OK || !launch) return st;
  switch (d->lmax_in) {
    case 1: return launch_fwd<1 + kOddKey>(a, s);
    case 2: return launch_fwd<2 + kOddKey>(a, s);
    case 3: return launch_fwd<3 + kOddKey>(a, s);
    case 4: return launch_fwd<4 + kOddKey>(a, s);
    default: return FC_ERR_UNSUPPORTED_RANK;
  }
}

extern "C" int fc_conv_odd_num_paths(const fc_conv_desc* d) {
  if (check_conv_desc(d) != FC_OK || d->lmax_in > 4) return -1;
  return num_odd_paths(d->lmax_in);
}

extern "C" int fc_conv_odd_out_row(const fc_conv_desc* d) {
  if (check_conv_desc(d) != FC_OK || d->lmax_in > 4) return -1;
  return odd_out_row(d->lmax_out, d->sum_paths);
}

extern "C" int fc_conv_odd_path(const fc_conv_desc* d, int p, int* l1, int* l2, int* l3) {
  if (check_conv_desc(d) != FC_OK || d->lmax_in > 4 || !l1 || !l2 || !l3) return FC_ERR_ARG;
  const int L = d->lmax_in;
  int n = 0;
  for (int c = 0; c <= L; ++c)
    for (int a = 0; a <= L; ++a)
      for (int b = 0; b <= L; ++b)
        if (odd_admissible(a, b, c)) {
          if (n == p) {
            *l1 = a;
            *l2 = b;
            *l3 = c;
            return FC_OK;
          }
          ++n;
        }
  return FC_ERR_ARG;
}
