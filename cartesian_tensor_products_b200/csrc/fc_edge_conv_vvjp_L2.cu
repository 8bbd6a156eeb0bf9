// libflashcart: VJP-of-VJP of the edge convolution, rank 2 instantiation.
#include "fc_edge_conv_vvjp.cuh"
#include "generated/fc_vvjp_L2.cuh"

namespace fc {
int launch_vvjp_rank2(const VvjpArgs& a, cudaStream_t s) {
  return a.C == 64 ? launch_vvjp_cc<2, 64>(a, s) : launch_vvjp_cc<2, 0>(a, s);
}
}  // namespace fc
