// libflashcart: receiver-sorted edge convolution, vector-Jacobian product.
//
// FlashCart (arXiv 2610.06409) App. C Eq. (C1) per edge, path and channel
// (f bilinear, c = w f):
//   x_bar_b1 = w sum_a g_a dF_a/dx_b1 = w (M^T g)_b1      -> sender v_e
//   w_bar    = <g, f(x, y)> = <M^T g, x>                   -> stored per edge
//   y_bar_b2 = w sum_a g_a dF_a/dy_b2                      -> edge e
// summed as in Algorithm 2 (receiver-sorted, the receiver's g loaded once),
// and carried through the direction tensors to the edge vector (App. C,
// last paragraph of "Symbolic derivatives"):
//   r_bar = (I - u u^T)/|r| (dT/du)^T y_bar,   u = r/|r|.
//
// B200 design.  Output paths are cut offline into G groups of whole paths
// (h = M^T g needs every row of a path).  A CTA is (group, 4 consecutive
// receiver tiles): its 4 warps run the same code, one receiver each, and
// hold the receiver's g rows of the group's paths in registers for all its
// edges; blocks are ordered group-major so an SMSP mostly runs one
// instruction stream.  Sender
// rows and edge weights are streamed through a per-warp cp.async ring as
// in the forward kernel; M and dT/du are formed lane-per-edge into a
// warp-private window.  Per edge a lane computes, for its 4 channels,
// h = M^T g, w_bar = <h, x> (one coalesced 16-byte store per path), the
// sender contribution w h (summed over the warp's paths, then one vector
// atomic add per x_bar row, as Algorithm 2 adds sender gradients
// atomically), and y_bar through d_(a,b1) = <g_a, w x_b1>; y_bar is folded
// into u_bar = (dT/du)^T y_bar, reduced over the warp with shuffles and
// added atomically (3 floats per warp and edge) into r_bar.
#include "fc_edge_conv_vjp.cuh"
#include "generated/fc_vjp_L1.cuh"
#include "generated/fc_vjp_L2.cuh"
#include "generated/fc_vjp_L3.cuh"
#include "generated/fc_vjp_L4.cuh"

namespace fc {
int launch_vjp_rank5(const VjpArgs& a, cudaStream_t s);
}  // namespace fc

using namespace fc;

extern "C" int fc_edge_conv_vjp(const fc_conv_desc* d, int n_nodes, int n_edges,
                                const int32_t* rowptr, const int32_t* edge_index,
                                const float* edge_vec, const float* x, const float* w,
                                const float* g, float* x_bar, float* w_bar, float* r_bar,
                                fc_stream_t stream) {
  int st = check_conv_desc(d);
  if (st != FC_OK) return st;
  if (n_nodes < 0 || n_edges < 0) return FC_ERR_ARG;
  if (n_nodes == 0) return n_edges == 0 ? FC_OK : FC_ERR_ARG;
  if (!rowptr || !x || !g) return FC_ERR_ARG;
  if (n_edges > 0 && (!edge_index || !edge_vec || !w)) return FC_ERR_ARG;
  if (!aligned16(x) || !aligned16(g) || (w && !aligned16(w)) || (x_bar && !aligned16(x_bar)) ||
      (w_bar && !aligned16(w_bar)) || (r_bar && !aligned4(r_bar)) || !aligned4(rowptr) ||
      (edge_index && !aligned4(edge_index)) || (edge_vec && !aligned4(edge_vec)))
    return FC_ERR_ALIGN;
  const int L = d->lmax_in;
  const int C = d->channels;
  VjpArgs a;
  a.rowptr = rowptr;
  a.send = edge_index ? edge_index + n_edges : nullptr;
  a.vec = edge_vec;
  a.x = x;
  a.w = w;
  a.g = g;
  a.xbar = x_bar;
  a.wbar = w_bar;
  a.rbar = r_bar;
  a.n_nodes = n_nodes;
  a.n_edges = n_edges;
  a.C = C;
  a.ntiles = (C + 127) / 128;
  a.xrow = (L + 1) * (L + 1);
  a.zrow = out_row(L, d->sum_paths);
  a.P = num_paths(L);
  a.sum_paths = d->sum_paths;
  a.envelope = d->envelope;
  a.r_cut = d->r_cut;
  a.edge_scale = d->edge_scale;
  if ((long long)n_nodes * a.ntiles > 0x7fffffffLL) return FC_ERR_ARG;
  cudaStream_t s = (cudaStream_t)stream;
  if (x_bar && cudaMemsetAsync(x_bar, 0, sizeof(float) * (size_t)n_nodes * a.xrow * C, s) != cudaSuccess)
    return FC_ERR_CUDA;
  if (r_bar && n_edges > 0 &&
      cudaMemsetAsync(r_bar, 0, sizeof(float) * 3 * (size_t)n_edges, s) != cudaSuccess)
    return FC_ERR_CUDA;
  if (n_edges == 0) return FC_OK;
  if (!x_bar && !w_bar && !r_bar) return FC_OK;
  switch (L) {
    case 1: return launch_vjp<1>(a, s);
    case 2: return launch_vjp<2>(a, s);
    case 3: return launch_vjp<3>(a, s);
    case 4: return launch_vjp<4>(a, s);
    case 5: return launch_vjp_rank5(a, s);
    default: return FC_ERR_UNSUPPORTED_RANK;
  }
}
