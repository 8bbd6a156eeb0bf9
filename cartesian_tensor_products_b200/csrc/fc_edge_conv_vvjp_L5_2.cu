// libflashcart: VJP-of-VJP of the edge convolution, rank 5, split launches
// of path groups [26, 39) (one translation unit per range so that they
// compile in parallel).
#include "fc_edge_conv_vvjp.cuh"
#include "generated/fc_vvjp_L5.cuh"

namespace fc {
int launch_vvjp_rank5_part2(const VvjpArgs& a, cudaStream_t s) {
  return a.C == 128 ? launch_vvjp_groups<5, 128, 26, 39>(a, s) : launch_vvjp_groups<5, 0, 26, 39>(a, s);
}
}  // namespace fc
