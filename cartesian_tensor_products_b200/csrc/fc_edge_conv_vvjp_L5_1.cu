// libflashcart: VJP-of-VJP of the edge convolution, rank 5, split launches
// of path groups [13, 26) (one translation unit per range so that they
// compile in parallel).
#include "fc_edge_conv_vvjp.cuh"
#include "generated/fc_vvjp_L5.cuh"

namespace fc {
int launch_vvjp_rank5_part1(const VvjpArgs& a, cudaStream_t s) {
  return a.C == 128 ? launch_vvjp_groups<5, 128, 13, 26>(a, s) : launch_vvjp_groups<5, 0, 13, 26>(a, s);
}
}  // namespace fc
