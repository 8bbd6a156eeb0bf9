// libflashcart: VJP-of-VJP of the edge convolution, rank 4 instantiation.
#include "fc_edge_conv_vvjp.cuh"
#include "generated/fc_vvjp_L4.cuh"

namespace fc {
int launch_vvjp_rank4(const VvjpArgs& a, cudaStream_t s) {
  return a.C == 64 ? launch_vvjp_cc<4, 64>(a, s) : launch_vvjp_cc<4, 0>(a, s);
}
}  // namespace fc
