// libflashcart: receiver-sorted edge-convolution VJP, rank 5 instantiation
// (generic channel count, no envelope).
#include "fc_edge_conv_vjp.cuh"
#include "generated/fc_vjp_L5.cuh"

namespace fc {
int launch_vjp_rank5(const VjpArgs& a, cudaStream_t s) {
  if (a.envelope) return FC_ERR_ARG;   // rank 5: no envelope variant is built
  return launch_vjp_cc<5, 0>(a, s);
}
}  // namespace fc
