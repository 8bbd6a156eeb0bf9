// libflashcart: receiver-sorted edge convolution, rank 5 instantiation
// (generic channel count, no envelope).
#include "fc_edge_conv.cuh"
#include "generated/fc_fwd_L5.cuh"

namespace fc {
int launch_fwd_rank5(const ConvArgs& a, cudaStream_t s) {
  if (a.envelope) return FC_ERR_ARG;   // rank 5: no envelope variant is built
  return launch_fwd_cc<5, 0, false>(a, s);
}
}  // namespace fc
