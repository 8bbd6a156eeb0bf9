/*
 * flashcart.h -- C ABI of libflashcart: irreducible-Cartesian tensor
 * products for equivariant interatomic potentials on NVIDIA B200 (sm_100a).
 *
 * The operations are those of "FlashCart: Fast Cartesian Tensor Products
 * for Equivariant Interatomic Potentials" (arXiv 2610.06409):
 *   - fc_edge_conv          receiver-sorted edge convolution, Sec. 4 Eq. (1)
 *                           and Algorithm 1 (App. D "Receiver-sorted forward")
 *   - fc_edge_conv_vjp      its vector-Jacobian product, App. C Eq. (C1)
 *                           summed as in Algorithm 2, extended through the
 *                           direction tensors to the edge vectors (App. C,
 *                           last paragraph of "Symbolic derivatives")
 *   - fc_product_ladder     node-local correlation ladder, Sec. 5 Eq. (2)
 *                           with path-reduced products (App. E)
 *   - fc_product_ladder_vjp its vector-Jacobian product
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Tensors.  A rank-l feature is a symmetric trace-free (STF) Cartesian
 * tensor stored by its 2l+1 independent components (Sec. 3): those with at
 * most one z index, ordered p_z = 0 with p_x descending, then p_z = 1 with
 * p_x descending (l=1: x,y,z; l=2: xx,xy,yy,xz,yz; l=3: xxx,xxy,xyy,yyy,
 * xxz,xyz,yyz).
 * Paths.  Admissible (l1, l2) -> l3 with |l1-l2| <= l3 <= l1+l2 and
 * l1+l2+l3 even (Sec. 2), ordered by l3, then l1, then l2; eta is the
 * position of a path among those with the same l3.  Path normalisation
 * C_{l1 l2 l3} of Eq. (B1) is chosen so that T_l1(r) (x) T_l2(r) -> T_l3(r).
 * Layout (App. D "Data layout").  Row per node or edge, rank blocks in
 * increasing l; inside block l the component c, then the path eta, then the
 * channel k is fastest: offset off(l) + (c P_l + eta) C + k with
 * off(l) = sum_{l'<l} (2l'+1) P_l' C.  Node features have P_l = 1, so x is
 * [N][(L+1)^2 C].  Weights are [E][P][C] (channel fastest).
 * Edges.  edge_index is int32 [2][E]: row 0 receivers u_e, row 1 senders
 * v_e, sorted by receiver (non-decreasing).  edge_vec is float [E][3] and
 * points from the receiver to the sender, r_e = pos[v_e] - pos[u_e] (+ any
 * periodic shift) (Sec. 2).  rowptr [N+1]: incoming edges of u are
 * [rowptr[u], rowptr[u+1]) (Sec. 4, App. D).
 * Memory.  Every pointer argument of a compute call is DEVICE memory owned
 * by the caller, 16-byte aligned, and stays valid until the stream has
 * executed the call.  The library allocates no device memory; scratch comes
 * from a caller-provided workspace whose size a *_workspace_size call gives.
 * Streams.  Compute calls are asynchronous on `stream` (NULL = the legacy
 * default stream).  Host-side argument checks happen before anything is
 * enqueued; a failing call enqueues nothing and returns an error status.
 * Outputs are overwritten, never accumulated into.
 * Precision.  FP32 inputs and outputs, FP32 arithmetic with fused
 * multiply-adds.  Results that combine per-sender or per-edge gradient
 * contributions are not bitwise reproducible run to run.
 */
#ifndef FLASHCART_H
#define FLASHCART_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t. */
typedef struct CUstream_st *fc_stream_t;

typedef enum {
  FC_OK = 0,
  FC_ERR_ARG = 1,              /* NULL pointer, negative size, bad descriptor */
  FC_ERR_CSR = 2,              /* receivers unsorted or out of range, senders out of range */
  FC_ERR_DEGENERATE_EDGE = 3,  /* an edge vector of zero (or non-finite) length */
  FC_ERR_UNSUPPORTED_RANK = 4, /* a rank combination this build has no kernel for */
  FC_ERR_ALIGN = 5,            /* pointer not 16-byte aligned or channels not a multiple of 4 */
  FC_ERR_CUDA = 6,             /* a CUDA runtime call failed (launch, copy) */
  FC_ERR_WORKSPACE = 7         /* workspace NULL or smaller than required */
} fc_status;

/* Human-readable text of a status code; never NULL. */
const char *fc_status_string(int status);

/* Library version as 10000*major + 100*minor + patch. */
int fc_version(void);

/* Edge-convolution descriptor.  This build supports
 * lmax_in == lmax_edge == lmax_out in {1, 2, 3, 4, 5}, channels >= 4 and
 * a multiple of 4 (rank 5: without the envelope; its VJP-of-VJP runs one
 * kernel launch per path group).  sum_paths = 0 keeps the P_l paths of each output rank
 * separate (z row = sum_l (2l+1) P_l C); sum_paths = 1 sums them (z row =
 * (lmax_out+1)^2 C, the node-feature layout).
 * envelope = 1 multiplies the direction tensors of edge e by
 *   s_e = edge_scale * (cos(pi |r_e| / r_cut) + 1) / 2   (|r_e| < r_cut, else 0),
 * a radial envelope that takes each edge's contribution smoothly to zero
 * at the cutoff (Sec. 2, paragraph on equivariant convolution); by
 * bilinearity this equals scaling all weights of edge e by s_e, and
 * edge_scale can carry a 1/sqrt(mean neighbours) factor (App. E Eq. E1).
 * The VJP's r_bar then includes the derivative of s_e.
 * envelope = 0 (r_cut and edge_scale ignored) means s_e = 1. */
typedef struct {
  int lmax_in;      /* rank of node features x (l1)           */
  int lmax_edge;    /* rank of direction tensors T_l2(r-hat) */
  int lmax_out;     /* rank of outputs (l3)                   */
  int channels;     /* C                                      */
  int sum_paths;    /* 0 or 1                                 */
  int envelope;     /* 0 or 1                                 */
  float r_cut;      /* cutoff radius (envelope = 1), > 0      */
  float edge_scale; /* global factor of s_e (envelope = 1)    */
} fc_conv_desc;

/* Number of paths P of the descriptor, or -1 if it is not supported. */
int fc_conv_num_paths(const fc_conv_desc *desc);

/* Output components per channel of one z row (z row = this x C), or -1. */
int fc_conv_out_row(const fc_conv_desc *desc);

/* Path p of the descriptor: writes l1, l2, l3.  Returns FC_OK or FC_ERR_ARG. */
int fc_conv_path(const fc_conv_desc *desc, int p, int *l1, int *l2, int *l3);

/* Scratch bytes the convolution calls need: always 0.  Every receiver's sums
 * are accumulated on chip and stored once (Algorithm 1), so fc_edge_conv,
 * fc_edge_conv_vjp and fc_edge_conv_vjp_vjp take no workspace argument; the
 * query exists for callers written against a workspace-size convention.
 * The descriptor and sizes are not inspected. */
size_t fc_edge_conv_workspace_size(const fc_conv_desc *desc, int n_nodes, int n_edges);

/* Build the receiver row pointer of a receiver-sorted edge list and
 * validate the graph (App. D "Receiver-sorted forward").
 *   edge_index [2][n_edges] int32 (device), edge_vec [n_edges][3] float
 *   (device, may be NULL to skip the length check), rowptr [n_nodes+1]
 *   int32 (device, written), flag: one int32 of device scratch.
 * Rejects receivers out of [0, n_nodes) or not sorted (FC_ERR_CSR),
 * senders out of range (FC_ERR_CSR), and edge vectors of zero or
 * non-finite length (FC_ERR_DEGENERATE_EDGE).  Synchronises `stream` to
 * read the verdict; rowptr is only meaningful when FC_OK is returned.
 * n_edges = 0 is valid (rowptr all zero). */
int fc_build_rowptr(int n_nodes, int n_edges, const int32_t *edge_index,
                    const float *edge_vec, int32_t *rowptr, int32_t *flag,
                    fc_stream_t stream);

/* fc_build_rowptr for a receiver range (see fc_edge_conv_rect): receivers
 * in [0, n_nodes), senders in [0, n_send). */
int fc_build_rowptr_rect(int n_nodes, int n_send, int n_edges, const int32_t *edge_index,
                         const float *edge_vec, int32_t *rowptr, int32_t *flag,
                         fc_stream_t stream);

/* Receiver-sorted edge convolution, Sec. 4 Eq. (1):
 *   z[u, eta, k] = sum_{e: u_e = u} w[e, eta, k] f_eta(x[v_e, :, k], T(r-hat_e))
 * with f_eta the Cartesian product of path eta (App. B Eq. (B1)) and
 * T(r-hat) = (T_0, ..., T_lmax_edge) the direction tensors of App. B.
 * Each receiver's sum is accumulated on chip and stored once (Algorithm 1:
 * no atomics, no per-edge message tensor), except with sum_paths = 1, where
 * path partial sums from different warps are added atomically into z after
 * the call zeroes it.
 *   rowptr [n_nodes+1] from fc_build_rowptr; edge_index, edge_vec as above;
 *   x [n_nodes][(lmax_in+1)^2 C]; w [n_edges][P][C];
 *   z [n_nodes][fc_conv_out_row() C] (written; receivers without edges get 0).
 * The graph must have passed fc_build_rowptr: the kernel does not fault on
 * a bad graph (rowptr is clamped to [0, n_edges], out-of-range senders
 * contribute nothing) but its output is then meaningless.
 * Returns FC_OK, FC_ERR_ARG, FC_ERR_UNSUPPORTED_RANK, FC_ERR_ALIGN or
 * FC_ERR_CUDA. */
int fc_edge_conv(const fc_conv_desc *desc, int n_nodes, int n_edges,
                 const int32_t *rowptr, const int32_t *edge_index,
                 const float *edge_vec, const float *x, const float *w,
                 float *z, fc_stream_t stream);

/* fc_edge_conv with separate receiver and sender counts, for a graph cut
 * into contiguous receiver ranges (one per GPU): the n_nodes receivers of
 * this range (rowptr [n_nodes+1], z [n_nodes][...], receivers numbered
 * from 0) take their edges from any of the n_send senders of the whole
 * graph (x [n_send][(lmax_in+1)^2 C], senders < n_send).  Everything else
 * as fc_edge_conv, which is this call with n_send = n_nodes.  The
 * convolution is a sum over each receiver's own edges (Sec. 4 Eq. (1)), so
 * the ranges' outputs are disjoint rows of the whole graph's z. */
int fc_edge_conv_rect(const fc_conv_desc *desc, int n_nodes, int n_send, int n_edges,
                      const int32_t *rowptr, const int32_t *edge_index,
                      const float *edge_vec, const float *x, const float *w,
                      float *z, fc_stream_t stream);

/* Vector-Jacobian product of fc_edge_conv, App. C Eq. (C1) summed over the
 * receiver-sorted edges as in Algorithm 2, with the direction-tensor
 * gradient carried to the edge vectors (App. C "Symbolic derivatives"):
 *   x_bar[v, :, k]  = sum_{e: v_e = v} sum_eta w[e,eta,k] (M_eta,e^T g[u_e,eta,k])
 *   w_bar[e, eta, k] = <g[u_e, eta, k], f_eta(x[v_e, :, k], T(r-hat_e))>
 *   r_bar[e]        = (d T(r_e/|r_e|) / d r_e)^T y_bar[e],
 *   y_bar[e]        = sum_{eta,k} w[e,eta,k] d<g, f_eta(x, y)>/dy at y = T(r-hat_e)
 * where M_eta,e[a][b] = d f_eta,a / d x_b and the gradients are taken with
 * respect to the independent components as free variables (App. C).
 *   g has the layout of z (fc_conv_out_row() x C per node);
 *   x_bar [n_nodes][(lmax_in+1)^2 C], w_bar [n_edges][P][C], r_bar
 *   [n_edges][3]: each may be NULL to skip it.  x_bar and r_bar are zeroed
 *   on the stream and then accumulated with atomic additions (their bits
 *   can differ run to run); w_bar is written once per entry.
 * Same graph requirements and error returns as fc_edge_conv. */
int fc_edge_conv_vjp(const fc_conv_desc *desc, int n_nodes, int n_edges,
                     const int32_t *rowptr, const int32_t *edge_index,
                     const float *edge_vec, const float *x, const float *w,
                     const float *g, float *x_bar, float *w_bar, float *r_bar,
                     fc_stream_t stream);

/* fc_edge_conv_vjp with separate receiver and sender counts (see
 * fc_edge_conv_rect): g [n_nodes][...] for this range's receivers, x and
 * x_bar [n_send][...] over all senders of the graph.  x_bar is then this
 * range's partial sum of the sender gradients; the ranges' partials add up
 * to the whole graph's x_bar (a reduce-scatter to the sender owners when
 * the graph is spread over GPUs).  w_bar and r_bar are per edge, local to
 * the range. */
int fc_edge_conv_vjp_rect(const fc_conv_desc *desc, int n_nodes, int n_send, int n_edges,
                          const int32_t *rowptr, const int32_t *edge_index,
                          const float *edge_vec, const float *x, const float *w,
                          const float *g, float *x_bar, float *w_bar, float *r_bar,
                          fc_stream_t stream);

/* Edge convolution over the odd-J (Levi-Civita) paths: App. B, paragraph
 * after Eq. (B1), and Sec. 7 ("Limitations") -- the same construction as
 * Eq. (B1) with one index of each input contracted through the Levi-Civita
 * symbol, so that parity is tracked explicitly.  An odd path (l1, l2) -> l3
 * has l1, l2 >= 1, |l1 - l2| <= l3 <= l1 + l2 - 1 and l1 + l2 + l3 odd;
 * with n = (l1 + l2 - l3 - 1) / 2,
 *   f(x, y) = STF part of  eps_{pqc} x_{i.. p k1..kn} y_{k1..kn q j..}
 * (n index pairs contracted, the free indices i.., j.., c symmetrised, the
 * traces removed, no further factor: (1,1) -> 1 is the cross product x x y).
 * The outputs are pseudo-tensors: under an improper rotation they pick up
 * det(R) = -1 in addition to the rotation of a true tensor.
 *   z[u, eta, k] = sum_{e: u_e = u} w[e, eta, k] f_eta(x[v_e, :, k], T(r-hat_e))
 * over the odd paths, ordered by l3, then l1, then l2 (fc_conv_odd_path);
 * output layout as for fc_edge_conv with the odd path counts P_l
 * (fc_conv_odd_out_row components per channel; no odd path ends in rank 0,
 * so the rank-0 block is empty, or zero with sum_paths = 1);
 * w [n_edges][fc_conv_odd_num_paths()][C].  Ranks 1..4, otherwise the
 * descriptor rules, graph requirements and error returns of fc_edge_conv. */
int fc_conv_odd_num_paths(const fc_conv_desc *desc);
int fc_conv_odd_out_row(const fc_conv_desc *desc);
int fc_conv_odd_path(const fc_conv_desc *desc, int p, int *l1, int *l2, int *l3);
int fc_edge_conv_odd(const fc_conv_desc *desc, int n_nodes, int n_edges,
                     const int32_t *rowptr, const int32_t *edge_index,
                     const float *edge_vec, const float *x, const float *w,
                     float *z, fc_stream_t stream);

/* VJP of fc_edge_conv_odd (App. C Eq. (C1) with the odd-path coefficients,
 * summed as in Algorithm 2): x_bar, w_bar, r_bar exactly as documented for
 * fc_edge_conv_vjp, g in the layout of fc_edge_conv_odd's output. */
int fc_edge_conv_odd_vjp(const fc_conv_desc *desc, int n_nodes, int n_edges,
                         const int32_t *rowptr, const int32_t *edge_index,
                         const float *edge_vec, const float *x, const float *w,
                         const float *g, float *x_bar, float *w_bar, float *r_bar,
                         fc_stream_t stream);

/* VJP-of-VJP of fc_edge_conv (the derivative of fc_edge_conv_vjp), App. C
 * Eq. (C2) summed over the receiver-sorted edges as in Algorithm 3, with the
 * direction tensors differentiated twice (App. C, paragraph after Eq. C2).
 * Given the incoming gradient g of fc_edge_conv and cotangents v_x, v_w,
 * v_r of the VJP outputs x_bar, w_bar, r_bar, it returns the gradients of
 *   <v_x, x_bar> + <v_w, w_bar> + <v_r, r_bar>
 * with respect to g, x, w and the edge vectors:
 *   g_hat[u,eta,k] = sum_{e: u_e = u} w (f(v_x, y) + f(x, v_y)) + v_w f(x, y)
 *   x_hat[v, :, k] = sum_{e: v_e = v} sum_eta VJP1_eta(g, w v_y + v_w y)
 *   w_hat[e,eta,k] = <g, f(v_x, y) + f(x, v_y)>
 *   r_hat[e]       = (dy/dr)^T y_hat + (d^2 <y_bar, y> / dr dr) v_r,
 *   y_hat[e]       = sum_{eta,k} VJP2_eta(g, w v_x + v_w x),
 *   y_bar[e]       = sum_{eta,k} w VJP2_eta(g, x)   (the first VJP's y gradient)
 * with y = T(r-hat_e), v_y = (dy/dr) v_r[e] and every f, x, v_x, g at the
 * edge's sender, receiver and channel.
 *   x, w, g as for fc_edge_conv_vjp; v_x like x, v_w like w, v_r
 *   [n_edges][3]: each may be NULL for a zero cotangent.
 *   g_hat (layout of z), x_hat (layout of x), w_hat (layout of w), r_hat
 *   [n_edges][3]: each may be NULL to skip it.  g_hat, x_hat and r_hat are
 *   zeroed on the stream and accumulated with atomic additions; w_hat is
 *   written once per entry.
 * The radial envelope is not supported here: FC_ERR_ARG if desc->envelope.
 * Same graph requirements and other error returns as fc_edge_conv. */
int fc_edge_conv_vjp_vjp(const fc_conv_desc *desc, int n_nodes, int n_edges,
                         const int32_t *rowptr, const int32_t *edge_index,
                         const float *edge_vec, const float *x, const float *w,
                         const float *g, const float *v_x, const float *v_w,
                         const float *v_r, float *g_hat, float *x_hat,
                         float *w_hat, float *r_hat, fc_stream_t stream);

/* Scalar readout of a node-layout array z [n_nodes][(lmax+1)^2 C]:
 *   energy[0] = sum_{n,k} z[n, rank 0, k]   (device float, overwritten)
 *   gz[n, rank 0, k] = 1, every other entry 0  (device, may be NULL)
 * i.e. E as the sum of the rank-0 outputs and dE/dz.  The sum uses atomic
 * additions (not bitwise reproducible). */
int fc_scalar_readout(int n_nodes, int lmax, int channels, const float *z,
                      float *energy, float *gz, fc_stream_t stream);

/* Forces from edge-vector gradients, for r_e = pos[v_e] - pos[u_e]
 * (+ a fixed periodic shift):
 *   forces[i] = -(sum_{e: v_e = i} r_bar[e] - sum_{e: u_e = i} r_bar[e])
 * = -dE/dpos_i.  forces [n_nodes][3] (device, overwritten; atomic sums). */
int fc_edge_forces(int n_nodes, int n_edges, const int32_t *edge_index,
                   const float *r_bar, float *forces, fc_stream_t stream);

/* Product-ladder descriptor: ranks 0..lmax for every state (lmax in
 * {1,2,3,4}), channels a multiple of 4, order >= 1 (order-1 products). */
typedef struct {
  int lmax;
  int channels;
  int order;
} fc_ladder_desc;

/* Number of paths P of the ladder products (all l1, l2, l3 <= lmax), or -1. */
int fc_ladder_num_paths(const fc_ladder_desc *desc);

/* Node-local correlation ladder, Sec. 5 Eq. (2) with path-reduced products
 * (App. E) and a per-rank channel mix after every product:
 *   B_v[n,l3,c,k]   = sum_{p = (l1,l2)->l3} path_w[v-1][p][k]
 *                       f_p(A_v[n,l1,:,k], A_1[n,l2,:,k])_c
 *   A_{v+1}[n,l,c,k] = sum_k' mix_w[v-1][l][k][k'] B_v[n,l,c,k']
 *   z = A_1 + A_2 + ... + A_order          (v = 1 .. order-1)
 * Products couple equal channels only (channel-diagonal, Sec. 5).
 *   A1 [n_nodes][(lmax+1)^2 C] (node layout), path_w [order-1][P][C],
 *   mix_w [order-1][lmax+1][C][C] (row = output channel),
 *   states [order-1][n_nodes][(lmax+1)^2 C] receives A_2 .. A_order,
 *   z [n_nodes][(lmax+1)^2 C].
 * At C = 128 and 256 the per-rank mix runs on the tcgen05 tensor cores
 * (FP32 accuracy through a three-term TF32 split) and z is summed in one
 * pass at the end; other widths use FP32 SIMT kernels.
 * workspace: fc_product_ladder_workspace_size() bytes of device scratch,
 * 16-byte aligned, ws_bytes = its real size; FC_ERR_WORKSPACE if NULL or
 * smaller.  At C = 128 and 256 that is the product as FP32 128-node tiles
 * per rank and component (about one product state, node count rounded up to
 * 128) plus one step's TF32 hi / lo matrices; otherwise one product state.
 * order = 1 copies A1 to z and needs no workspace. */
size_t fc_product_ladder_workspace_size(const fc_ladder_desc *desc, int n_nodes);
int fc_product_ladder(const fc_ladder_desc *desc, int n_nodes, const float *A1,
                      const float *path_w, const float *mix_w, float *states,
                      float *z, void *workspace, size_t ws_bytes,
                      fc_stream_t stream);

/* VJP of fc_product_ladder by reverse accumulation through its steps:
 * given gz (gradient of z, node layout) and the states of the forward call,
 * writes A1_bar (node layout), path_w_bar [order-1][P][C] and mix_w_bar
 * [order-1][lmax+1][C][C].  The weight gradients sum over all nodes with
 * atomic additions (not bitwise reproducible).  At C = 128 the mix
 * B_bar = A_bar M and the weight gradient run on the tensor cores, at
 * C = 256 the mix only.  workspace: fc_product_ladder_vjp_workspace_size()
 * bytes (four product states, plus at C = 128 and 256 the gradient as
 * TF32-split or FP32 128-row tiles and one step's split matrices); ws_bytes
 * = its real size, FC_ERR_WORKSPACE if smaller. */
size_t fc_product_ladder_vjp_workspace_size(const fc_ladder_desc *desc, int n_nodes);
int fc_product_ladder_vjp(const fc_ladder_desc *desc, int n_nodes,
                          const float *A1, const float *path_w,
                          const float *mix_w, const float *states,
                          const float *gz, float *A1_bar, float *path_w_bar,
                          float *mix_w_bar, void *workspace, size_t ws_bytes,
                          fc_stream_t stream);

/* fc_product_ladder without a workspace argument and without allocating.
 * No counterpart in the paper: it exists for callers that cannot allocate
 * device memory -- code that runs inside another framework's memory pool
 * (the pool already holds nearly all of HBM, so a raw cudaMalloc would
 * fail or fragment it) and latency-critical loops (cudaMalloc may
 * synchronise the device).  The caller still passes inputs and outputs
 * exactly as for fc_product_ladder; its scratch is a fixed 16 MiB array
 * inside the library, held by every GPU that loads the library until the
 * process exits.
 *   Limit: fc_product_ladder_workspace_size(desc, n_nodes) <= 16 MiB (at
 *   rank 3, C = 128: up to 1,920 nodes), else FC_ERR_WORKSPACE and nothing
 *   is enqueued.
 *   The first call on a device looks up the array's device address (a
 *   runtime query, no allocation); make that first call before any stream
 *   capture on that device.
 *   Every call shares the one array, which keeps the last call's contents
 *   (nothing in it needs to start at zero): calls that overlap on the GPU,
 *   on different streams or in different host threads, race and must be
 *   serialised by the caller.
 * Returns the statuses of fc_product_ladder, or FC_ERR_CUDA if the
 * address look-up fails. */
int fc_product_ladder_noalloc(const fc_ladder_desc *desc, int n_nodes,
                              const float *A1, const float *path_w,
                              const float *mix_w, float *states, float *z,
                              fc_stream_t stream);

/* The full correlation ladder, forward: Sec. 5 Eq. (2) with every coupling
 * path kept and a learned map that mixes paths and channels per output rank:
 *   phi_1[l,c,:] = W1_l A[l,c,:]                              (C x C per rank)
 *   B_q[eta,c,k] = f_eta(phi_{q-1}[l1,:,k], A[l2,:,k])_c      (q = 2 .. order)
 *   phi_q[l,c,j] = sum_{eta -> l} sum_k Wq_l[j][eta_l C + k] B_q[eta,c,k]
 *   z = phi_1 + ... + phi_order
 * with eta_l the path's position among the paths into rank l (paths ordered
 * by l3, then l1, then l2).  Ranks 1..4, channels a multiple of 4.
 *   A [n_nodes][(lmax+1)^2 C]; W1 [lmax+1][C][C] (row = output channel);
 *   Wq [order-1][C P C]: per step the rank blocks [C][P_l C] one after the
 *   other (rank l at C C sum_{l'<l} P_l'); states [order][n_nodes][(lmax+1)^2 C]
 *   receives phi_1 .. phi_order; z [n_nodes][(lmax+1)^2 C].
 * C = 128 runs the maps on the tensor cores (three-term TF32 split, FP32
 * accuracy); the workspace then holds one path-separated product as FP32
 * tiles (about n_nodes x fc_conv_out_row x C floats, node count rounded up
 * to 128) and the maps of one step as hi / lo TF32 tiles (2 C P C floats),
 * order 1 included.  Other widths use
 * FP32 SIMT maps: one path-separated product (n_nodes x fc_conv_out_row x C
 * floats), none for order 1.
 * workspace: fc_full_ladder_workspace_size() bytes, 16-byte aligned (0 means
 * none is needed).  Returns the statuses of fc_product_ladder; a wait of the
 * tensor-core kernel that gives up sets the fc_device_error word. */
size_t fc_full_ladder_workspace_size(const fc_ladder_desc *desc, int n_nodes);
int fc_full_ladder(const fc_ladder_desc *desc, int n_nodes, const float *A,
                   const float *W1, const float *Wq, float *states, float *z,
                   void *workspace, size_t ws_bytes, fc_stream_t stream);

/* VJP of fc_full_ladder by reverse accumulation through its steps (Sec. 5
 * Eq. (2); each bilinear product differentiated as in App. C Eq. (C1)):
 * given gz (gradient of z) and the states phi_1 .. phi_order of the forward
 * call, writes the gradients of <gz, z>
 *   A_bar [n_nodes][(lmax+1)^2 C], W1_bar like W1 ([lmax+1][C][C]),
 *   Wq_bar like Wq ([order-1][C P C]; unused for order 1).
 * Going down from q = order, the running gradient pbar of phi_q (gz plus
 * what step q+1 sends back) gives Wq_bar_l += pbar^T B_q and
 * Bbar_q = pbar Wq_l per rank, and the product VJP of B_q = f(phi_{q-1}, A)
 * sends Bbar_q to phi_{q-1} and A; the first map gives W1_bar_l += pbar^T A
 * and A_bar += pbar W1_l.  B_q is recomputed from the saved phi_{q-1}.
 * Outputs are overwritten; the weight gradients sum over all nodes with
 * atomic additions (not bitwise reproducible).  FP32 throughout.
 * workspace: fc_full_ladder_vjp_workspace_size() bytes (two node-layout
 * gradients plus one step's path-separated product and its gradient,
 * n_nodes x fc_conv_out_row x C floats each), 16-byte aligned; ws_bytes its
 * real size, FC_ERR_WORKSPACE if smaller.  Returns the statuses of
 * fc_full_ladder. */
size_t fc_full_ladder_vjp_workspace_size(const fc_ladder_desc *desc, int n_nodes);
int fc_full_ladder_vjp(const fc_ladder_desc *desc, int n_nodes, const float *A,
                       const float *W1, const float *Wq, const float *states,
                       const float *gz, float *A_bar, float *W1_bar, float *Wq_bar,
                       void *workspace, size_t ws_bytes, fc_stream_t stream);

/* Sticky device-side error word of the kernels that wait on barriers (the
 * tensor-core mixes and maps of the ladders): each wait gives up after a
 * bounded time (fc_set_wait_timeout), skips the rest of its CTA's work --
 * after letting the copies and MMAs it already started finish -- and sets
 * the word instead of hanging; that call's outputs are then meaningless.
 * Synchronises `stream`, writes the word to *flag (0 = no wait gave up
 * since the last call) and clears it.  FC_ERR_ARG if flag is NULL. */
int fc_device_error(int *flag, fc_stream_t stream);

/* Bound, in nanoseconds of the GPU's global timer, of every barrier wait in
 * the tensor-core kernels on the current device (ns = 0 restores the
 * default of 500 ms; a healthy wait lasts microseconds).  A synchronous
 * copy to the device: it applies to kernels launched after it returns, so
 * call it while none of this library's kernels runs on the device.  A
 * very small bound makes the waits give up (fc_device_error then reports
 * 1), which is how the give-up path can be exercised.  Returns FC_OK or
 * FC_ERR_CUDA. */
int fc_set_wait_timeout(uint64_t ns);

#ifdef __cplusplus
}
#endif
#endif /* FLASHCART_H */
