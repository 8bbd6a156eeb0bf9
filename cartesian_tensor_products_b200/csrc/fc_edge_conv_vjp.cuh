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
// added atomically (3 floats per warp and edge) into r_bar.  At C = 64 a
// warp runs two receivers, one per half-warp (vjp_warp_half).
#pragma once
#include "fc_common.cuh"
#include "fc_device.cuh"

namespace fc {

struct VjpArgs {
  const int32_t* rowptr;
  const int32_t* send;
  const float* vec;
  const float* x;
  const float* w;
  const float* g;
  float* xbar;
  float* wbar;
  float* rbar;
  int n_nodes, n_edges, C, ntiles, xrow, zrow, P, sum_paths;
  int n_send;   // rows of x (senders index x); n_nodes = receivers = rows of rowptr - 1 and z
  int envelope;
  float r_cut, edge_scale;
};

struct VEdgeWin {
  int v;
  float rx, ry, rz;
};

__device__ __forceinline__ VEdgeWin vload_win(const VjpArgs& a, int e, int e1) {
  VEdgeWin wv;
  if (e < e1) {
    wv.v = __ldg(a.send + e);
    wv.rx = __ldg(a.vec + 3 * e);
    wv.ry = __ldg(a.vec + 3 * e + 1);
    wv.rz = __ldg(a.vec + 3 * e + 2);
  } else {
    wv.v = -1;
    wv.rx = 1.0f;
    wv.ry = 0.0f;
    wv.rz = 0.0f;
  }
  return wv;
}

template <class Grp>
__device__ __forceinline__ void vissue_edge(const VjpArgs& a, int C, float* st, int q, int v,
                                            int k0, bool act) {
  const bool vok = act && v >= 0 && v < a.n_send;
  const int kk = act ? k0 : 0;
  const float* xv = a.x + (size_t)(vok ? v : 0) * a.xrow * C + kk;
  const float* we = a.w + (size_t)q * a.P * C + kk;
  Grp::issue(st, xv, we, C, vok, act);
}

template <class Grp, int S, int MW, int CC>
__device__ __forceinline__ void vjp_warp(const VjpArgs& a, float* smem, int lane, int unit) {
  constexpr int STAGE = Grp::NROW * 128;
  constexpr int NYB = Grp::NYD > 0 ? Grp::NYD : 1;
  const int C = CC > 0 ? CC : a.C;
  const int u = CC == 128 ? unit : unit / a.ntiles;
  const int tile = unit - u * (CC == 128 ? 1 : a.ntiles);
  const int k0 = tile * 128 + lane * 4;
  const bool act = k0 < C;
  int e0 = __ldg(a.rowptr + u), e1 = __ldg(a.rowptr + u + 1);
  e0 = e0 < 0 ? 0 : (e0 > a.n_edges ? a.n_edges : e0);
  e1 = e1 < e0 ? e0 : (e1 > a.n_edges ? a.n_edges : e1);
  if (e0 == e1) return;
  float* st = smem + Grp::RING_OFF + lane * 4;
  float* mwin = smem + Grp::MWIN_OFF;
  const bool wstore = act && a.wbar != nullptr;
  float* wbase = a.wbar != nullptr ? a.wbar : a.xbar;   // any valid pointer when unused

  float4 gr[Grp::NA];
  if (act) {
    Grp::load_g(a.g + (size_t)u * a.zrow * C + k0, C, a.sum_paths, gr);
  } else {
#pragma unroll
    for (int i = 0; i < Grp::NA; ++i) gr[i] = zero4();
  }
  float4 xb[Grp::NX];
#pragma unroll
  for (int i = 0; i < Grp::NX; ++i) xb[i] = zero4();
  float yb[NYB];
#pragma unroll
  for (int i = 0; i < NYB; ++i) yb[i] = 0.0f;

  VEdgeWin cur = vload_win(a, e0 + lane, e1);
  VEdgeWin nxt = vload_win(a, e0 + 32 + lane, e1);
#pragma unroll
  for (int s = 0; s < S; ++s) {
    const int q = e0 + s;
    const int v = __shfl_sync(0xffffffffu, cur.v, s);
    if (q < e1) vissue_edge<Grp>(a, C, st + s * STAGE, q, v, k0, act);
    cp_async_commit();
  }

  for (int q = e0; q < e1; ++q) {
    const int p = q - e0;
    if (p > 0 && (p & 31) == 0) {
      cur = nxt;
      nxt = vload_win(a, q + 32 + lane, e1);
    }
    if ((p % MW) == 0) {
      const int src = (p & 31) + (lane % MW);
      const float rx = __shfl_sync(0xffffffffu, cur.rx, src);
      const float ry = __shfl_sync(0xffffffffu, cur.ry, src);
      const float rz = __shfl_sync(0xffffffffu, cur.rz, src);
      __syncwarp();
      if (lane < MW && q + lane < e1) {
        const float r = sqrtf(rx * rx + ry * ry + rz * rz);
        const float inv = 1.0f / r;
        float es, esp;
        edge_envelope(a.envelope, r, a.r_cut, a.edge_scale, es, esp);
        Grp::make_row(rx * inv, ry * inv, rz * inv, es, esp, mwin + lane * Grp::MSTRIDE);
      }
      __syncwarp();
    }
    const int slot = p % S;
    cp_async_wait<S - 1>();
    const float* m = mwin + (p % MW) * Grp::MSTRIDE;
    Grp::edge(gr, st + slot * STAGE, m, xb, yb,
              wbase + (wstore ? (size_t)q * a.P * C + k0 : 0), C, wstore);
    // sender gradient
    const int v = __shfl_sync(0xffffffffu, cur.v, p & 31);
    if (a.xbar != nullptr && act && v >= 0 && v < a.n_send) {
      Grp::flush_xbar(a.xbar + (size_t)v * a.xrow * C + k0, C, xb);
    } else {
#pragma unroll
      for (int i = 0; i < Grp::NX; ++i) xb[i] = zero4();
    }
    // edge-vector gradient
    if constexpr (Grp::NYD > 0) {
      if (a.rbar != nullptr) {
        float ux, uy, uz, rho;
        Grp::ubar(yb, m, ux, uy, uz, rho);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          ux += __shfl_xor_sync(0xffffffffu, ux, o);
          uy += __shfl_xor_sync(0xffffffffu, uy, o);
          uz += __shfl_xor_sync(0xffffffffu, uz, o);
          rho += __shfl_xor_sync(0xffffffffu, rho, o);
        }
        const float rx = __shfl_sync(0xffffffffu, cur.rx, p & 31);
        const float ry = __shfl_sync(0xffffffffu, cur.ry, p & 31);
        const float rz = __shfl_sync(0xffffffffu, cur.rz, p & 31);
        if (lane == 0) {
          const float inv = 1.0f / sqrtf(rx * rx + ry * ry + rz * rz);
          const float nx = rx * inv, ny = ry * inv, nz = rz * inv;
          const float dotu = ux * nx + uy * ny + uz * nz;
          // direction part (I - u u^T)/|r| u_bar plus the radial part of the
          // envelope, s'(|r|) (y_bar . y) r-hat
          atomicAdd(a.rbar + 3 * (size_t)q + 0, (ux - nx * dotu) * inv + rho * nx);
          atomicAdd(a.rbar + 3 * (size_t)q + 1, (uy - ny * dotu) * inv + rho * ny);
          atomicAdd(a.rbar + 3 * (size_t)q + 2, (uz - nz * dotu) * inv + rho * nz);
        }
      }
#pragma unroll
      for (int i = 0; i < NYB; ++i) yb[i] = 0.0f;
    }
    const int pn = p + S;
    if (q + S < e1) {
      int vn;
      if ((pn >> 5) == (p >> 5))
        vn = __shfl_sync(0xffffffffu, cur.v, pn & 31);
      else
        vn = __shfl_sync(0xffffffffu, nxt.v, pn & 31);
      vissue_edge<Grp>(a, C, st + slot * STAGE, q + S, vn, k0, act);
    }
    cp_async_commit();
  }
  cp_async_wait<0>();
}

// C = 64: two receivers per warp, half-warp h (lanes 16 h .. 16 h + 15, 4
// channels each) runs receiver 2 unit + h.  As in the forward's pairing,
// each half keeps its own 16-edge register window and 8 edges of the M
// window, and the halves walk their edges in step; the per-edge reduction of
// the edge-vector gradient runs over the 16 lanes of a half, whose first
// lane adds it into r_bar.
template <class Grp, int S, int MW>
__device__ __forceinline__ void vjp_warp_half(const VjpArgs& a, float* smem, int lane, int unit) {
  constexpr int STAGE = Grp::NROW * 128;
  constexpr int NYB = Grp::NYD > 0 ? Grp::NYD : 1;
  constexpr int C = 64;
  constexpr int HW = MW / 2;
  static_assert(S <= 16 && HW >= 1, "ring depth within a 16-edge window");
  const int h = lane >> 4, hl = lane & 15, hbase = lane & 16;
  const int u = 2 * unit + h;
  const bool has = u < a.n_nodes;
  const int k0 = hl * 4;
  int e0 = has ? __ldg(a.rowptr + u) : 0, e1 = has ? __ldg(a.rowptr + u + 1) : 0;
  e0 = e0 < 0 ? 0 : (e0 > a.n_edges ? a.n_edges : e0);
  e1 = e1 < e0 ? e0 : (e1 > a.n_edges ? a.n_edges : e1);
  const int len = e1 - e0;
  int lmax = len;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) lmax = max(lmax, __shfl_xor_sync(0xffffffffu, lmax, o));
  if (lmax == 0) return;
  float* st = smem + Grp::RING_OFF + lane * 4;
  float* mwin = smem + Grp::MWIN_OFF + h * HW * Grp::MSTRIDE;
  const bool wstore = a.wbar != nullptr;
  float* wbase = a.wbar != nullptr ? a.wbar : a.xbar;   // any valid pointer when unused

  float4 gr[Grp::NA];
  if (has) {
    Grp::load_g(a.g + (size_t)u * a.zrow * C + k0, C, a.sum_paths, gr);
  } else {
#pragma unroll
    for (int i = 0; i < Grp::NA; ++i) gr[i] = zero4();
  }
  float4 xb[Grp::NX];
#pragma unroll
  for (int i = 0; i < Grp::NX; ++i) xb[i] = zero4();
  float yb[NYB];
#pragma unroll
  for (int i = 0; i < NYB; ++i) yb[i] = 0.0f;

  VEdgeWin cur = vload_win(a, e0 + hl, e1);
  VEdgeWin nxt = vload_win(a, e0 + 16 + hl, e1);
#pragma unroll
  for (int s = 0; s < S; ++s) {
    const int v = __shfl_sync(0xffffffffu, cur.v, hbase + s);
    if (s < len) vissue_edge<Grp>(a, C, st + s * STAGE, e0 + s, v, k0, true);
    cp_async_commit();
  }

  for (int p = 0; p < lmax; ++p) {
    const bool on = p < len;
    const int q = e0 + p;
    if (p > 0 && (p & 15) == 0) {
      cur = nxt;
      nxt = vload_win(a, q + 16 + hl, e1);
    }
    if ((p % HW) == 0) {
      const int src = hbase + (p & 15) + (hl % HW);
      const float rx = __shfl_sync(0xffffffffu, cur.rx, src);
      const float ry = __shfl_sync(0xffffffffu, cur.ry, src);
      const float rz = __shfl_sync(0xffffffffu, cur.rz, src);
      __syncwarp();
      if (hl < HW && p + hl < len) {
        const float r = sqrtf(rx * rx + ry * ry + rz * rz);
        const float inv = 1.0f / r;
        float es, esp;
        edge_envelope(a.envelope, r, a.r_cut, a.edge_scale, es, esp);
        Grp::make_row(rx * inv, ry * inv, rz * inv, es, esp, mwin + hl * Grp::MSTRIDE);
      }
      __syncwarp();
    }
    const int slot = p % S;
    cp_async_wait<S - 1>();
    const float* m = mwin + (p % HW) * Grp::MSTRIDE;
    if (on)
      Grp::edge(gr, st + slot * STAGE, m, xb, yb, wbase + (wstore ? (size_t)q * a.P * C + k0 : 0), C,
                wstore);
    // sender gradient
    const int v = __shfl_sync(0xffffffffu, cur.v, hbase + (p & 15));
    if (on && a.xbar != nullptr && v >= 0 && v < a.n_send) {
      Grp::flush_xbar(a.xbar + (size_t)v * a.xrow * C + k0, C, xb);
    } else {
#pragma unroll
      for (int i = 0; i < Grp::NX; ++i) xb[i] = zero4();
    }
    // edge-vector gradient
    if constexpr (Grp::NYD > 0) {
      if (a.rbar != nullptr) {
        float ux = 0.0f, uy = 0.0f, uz = 0.0f, rho = 0.0f;
        if (on) Grp::ubar(yb, m, ux, uy, uz, rho);
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) {
          ux += __shfl_xor_sync(0xffffffffu, ux, o);
          uy += __shfl_xor_sync(0xffffffffu, uy, o);
          uz += __shfl_xor_sync(0xffffffffu, uz, o);
          rho += __shfl_xor_sync(0xffffffffu, rho, o);
        }
        const float rx = __shfl_sync(0xffffffffu, cur.rx, hbase + (p & 15));
        const float ry = __shfl_sync(0xffffffffu, cur.ry, hbase + (p & 15));
        const float rz = __shfl_sync(0xffffffffu, cur.rz, hbase + (p & 15));
        if (hl == 0 && on) {
          const float inv = 1.0f / sqrtf(rx * rx + ry * ry + rz * rz);
          const float nx = rx * inv, ny = ry * inv, nz = rz * inv;
          const float dotu = ux * nx + uy * ny + uz * nz;
          atomicAdd(a.rbar + 3 * (size_t)q + 0, (ux - nx * dotu) * inv + rho * nx);
          atomicAdd(a.rbar + 3 * (size_t)q + 1, (uy - ny * dotu) * inv + rho * ny);
          atomicAdd(a.rbar + 3 * (size_t)q + 2, (uz - nz * dotu) * inv + rho * nz);
        }
      }
#pragma unroll
      for (int i = 0; i < NYB; ++i) yb[i] = 0.0f;
    }
    const int pn = p + S;
    int vn;
    if ((pn >> 4) == (p >> 4))
      vn = __shfl_sync(0xffffffffu, cur.v, hbase + (pn & 15));
    else
      vn = __shfl_sync(0xffffffffu, nxt.v, hbase + (pn & 15));
    if (pn < len) vissue_edge<Grp>(a, C, st + slot * STAGE, e0 + pn, vn, k0, true);
    cp_async_commit();
  }
  cp_async_wait<0>();
}

template <int L, int CC, int g>
__device__ __forceinline__ void dispatch_vjp(int grp, const VjpArgs& a, float* smem, int lane,
                                             int unit) {
  if constexpr (g < VjpMeta<L>::G) {
    using Grp = VjpGroup<L, VjpMeta<L>::G, g>;
    if (grp == g) {
      if constexpr (CC == 64)
        vjp_warp_half<Grp, VjpMeta<L>::S, VjpMeta<L>::MWIN>(a, smem, lane, unit);
      else
        vjp_warp<Grp, VjpMeta<L>::S, VjpMeta<L>::MWIN, CC>(a, smem, lane, unit);
      return;
    }
    dispatch_vjp<L, CC, g + 1>(grp, a, smem, lane, unit);
  }
}

// CTA = (path group, WARPS consecutive receiver units): every warp of a CTA
// runs the same code, and blocks are ordered group-major, so an SMSP mostly
// executes one instruction stream.
template <int L, int CC>
__global__ void __launch_bounds__(VjpMeta<L>::WARPS * 32, VjpMeta<L>::MINB) edge_conv_vjp_kernel(const VjpArgs a) {
  extern __shared__ __align__(16) float smem[];
  constexpr int WARPS = VjpMeta<L>::WARPS;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int units = CC == 64 ? (a.n_nodes + 1) / 2 : a.n_nodes * a.ntiles;   // CC = 64: receiver pairs
  const int nb = (units + WARPS - 1) / WARPS;
  const int grp = blockIdx.x / nb;
  const int unit = (blockIdx.x - grp * nb) * WARPS + warp;
  if (unit >= units) return;
  dispatch_vjp<L, CC, 0>(grp, a, smem + warp * VjpMeta<L>::WARP_FLOATS, lane, unit);
}

template <int L, int CC>
static int launch_vjp_cc(const VjpArgs& a, cudaStream_t s) {
  static_assert(sizeof(float) * VjpMeta<L>::SMEM_FLOATS <= 227 * 1024,
                "VJP kernel shared memory exceeds the 227 KB per-CTA limit of sm_100");
  const size_t smem = sizeof(float) * (size_t)VjpMeta<L>::SMEM_FLOATS;
  static DeviceFlags configured;
  if (set_smem_once(configured, edge_conv_vjp_kernel<L, CC>, smem) != FC_OK) return FC_ERR_CUDA;
  const long long units = CC == 64 ? ((long long)a.n_nodes + 1) / 2 : (long long)a.n_nodes * a.ntiles;
  constexpr int WARPS = VjpMeta<L>::WARPS;
  const long long blocks = (units + WARPS - 1) / WARPS * VjpMeta<L>::G;
  if (blocks > 0x7fffffffLL) return FC_ERR_ARG;
  edge_conv_vjp_kernel<L, CC><<<(unsigned)blocks, WARPS * 32, smem, s>>>(a);
  return cudaGetLastError() == cudaSuccess ? FC_OK : FC_ERR_CUDA;
}

// Host checks and kernel arguments shared by the VJP entry points
// (natural-parity paths, odd = 0, or odd-J paths, odd = 1).  Zeroes x_bar
// and r_bar on the stream (they are accumulated atomically); *launch is
// false when there is nothing to launch.
inline int vjp_setup(const fc_conv_desc* d, int n_nodes, int n_send, int n_edges,
                     const int32_t* rowptr, const int32_t* edge_index, const float* edge_vec,
                     const float* x, const float* w, const float* g, float* x_bar, float* w_bar,
                     float* r_bar, int odd, cudaStream_t s, VjpArgs& a, bool* launch) {
  *launch = false;
  int st = check_conv_desc(d);
  if (st != FC_OK) return st;
  if (odd && d->lmax_in > 4) return FC_ERR_UNSUPPORTED_RANK;
  if (n_nodes < 0 || n_send < 0 || n_edges < 0) return FC_ERR_ARG;
  if (n_nodes == 0) return n_edges == 0 ? FC_OK : FC_ERR_ARG;
  if (!rowptr || !x || !g) return FC_ERR_ARG;
  if (n_edges > 0 && (!edge_index || !edge_vec || !w)) return FC_ERR_ARG;
  if (!aligned16(x) || !aligned16(g) || (w && !aligned16(w)) || (x_bar && !aligned16(x_bar)) ||
      (w_bar && !aligned16(w_bar)) || (r_bar && !aligned4(r_bar)) || !aligned4(rowptr) ||
      (edge_index && !aligned4(edge_index)) || (edge_vec && !aligned4(edge_vec)))
    return FC_ERR_ALIGN;
  const int L = d->lmax_in;
  const int C = d->channels;
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
  a.n_send = n_send;
  a.n_edges = n_edges;
  a.C = C;
  a.ntiles = (C + 127) / 128;
  a.xrow = (L + 1) * (L + 1);
  a.zrow = odd ? odd_out_row(L, d->sum_paths) : out_row(L, d->sum_paths);
  a.P = odd ? num_odd_paths(L) : num_paths(L);
  a.sum_paths = d->sum_paths;
  a.envelope = d->envelope;
  a.r_cut = d->r_cut;
  a.edge_scale = d->edge_scale;
  if ((long long)n_nodes * a.ntiles > 0x7fffffffLL) return FC_ERR_ARG;
  if (x_bar && cudaMemsetAsync(x_bar, 0, sizeof(float) * (size_t)n_send * a.xrow * C, s) != cudaSuccess)
    return FC_ERR_CUDA;
  if (r_bar && n_edges > 0 &&
      cudaMemsetAsync(r_bar, 0, sizeof(float) * 3 * (size_t)n_edges, s) != cudaSuccess)
    return FC_ERR_CUDA;
  if (n_edges == 0) return FC_OK;
  if (!x_bar && !w_bar && !r_bar) return FC_OK;
  *launch = true;
  return FC_OK;
}

template <int L>
static int launch_vjp(const VjpArgs& a, cudaStream_t s) {
  if (a.C == 128) return launch_vjp_cc<L, 128>(a, s);
  return a.C == 64 ? launch_vjp_cc<L, 64>(a, s) : launch_vjp_cc<L, 0>(a, s);
}

}  // namespace fc
