// libflashcart: VJP-of-VJP of the edge convolution, rank 3 instantiation.
#include "fc_edge_conv_vvjp.cuh"
#include "generated/fc_vvjp_L3.cuh"

namespace fc {
int launch_vvjp_rank3(const VvjpArgs& a, cudaStream_t s) {
  if (a.C == 128) return launch_vvjp_cc<3, 128>(a, s);
  return a.C == 64 ? launch_vvjp_cc<3, 64>(a, s) : launch_vvjp_cc<3, 0>(a, s);
}
}  // namespace fc
