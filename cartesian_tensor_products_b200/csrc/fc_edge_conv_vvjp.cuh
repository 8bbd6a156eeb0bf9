// libflashcart: receiver-sorted VJP-of-VJP of the edge convolution (kernel
// templates; instantiated per rank in fc_edge_conv_vvjp_L*.cu).
//
// FlashCart (arXiv 2610.06409) App. C Eq. (C2), summed as in Algorithm 3:
// given the incoming gradient g of the convolution and cotangents vx, vw, vr
// of its VJP outputs x_bar, w_bar, r_bar, the gradients of
// <vx, x_bar> + <vw, w_bar> + <vr, r_bar> are, per edge, path and channel
// (y = T(r-hat), vy = (d y / d r) vr, f bilinear):
//   g_hat += w [f(vx, y) + f(x, vy)] + vw f(x, y)   summed over the receiver's edges
//   x_hat += VJP1(g, w vy + vw y)                   atomically per sender row
//   w_hat  = <g, f(vx, y) + f(x, vy)>               stored per edge
//   y_hat += VJP2(g, w vx + vw x)
// and through the direction tensors (App. C, paragraph after Eq. C2)
//   r_hat  = (d y / d r)^T y_hat + (d^2 <y_bar, y> / dr dr) vr,
// y_bar = sum w VJP2(g, x) being the edge's first-order direction gradient.
//
// B200 design: the VJP kernel's structure.  Whole-path warp groups; a CTA is
// (group, 4 consecutive receivers), one receiver per warp, blocks ordered
// group-major (one instruction stream per SMSP).  The receiver's g rows and
// its g_hat accumulators stay in registers for all its edges (g_hat is added
// once per receiver at the end: with summed paths several groups share a
// slot).  Sender rows x and vx and the edge's w and vw are streamed through
// a per-warp cp.async ring; the per-edge matrices M(y) and M(vy), d y/du,
// d^2 y/du du and the edge's u, (I - u u^T) vr/|r|, 1/|r|, u.vr are formed
// lane-per-edge into a warp-private window.  Per edge a lane folds its
// channels' y_hat and y_bar into 12 numbers in u-space (D^T y_hat,
// G = D^T y_bar, H_u = sum y_bar d^2y/du du), the warp reduces them and lane
// 0 adds (I - u u^T) D^T y_hat / |r| plus the Hessian-vector product
//   [-(w (u.G) + u (w.G)) + (I - u u^T) H_u w] / |r| - (I - u u^T) G (u.vr) / |r|^2,
// w = (I - u u^T) vr / |r|, atomically into r_hat.  At C = 64 (ranks 1-4)
// a warp runs two receivers, one per half-warp (vvjp_warp_half).
#pragma once
#include "fc_common.cuh"
#include "fc_device.cuh"

namespace fc {

struct VvjpArgs {
  const int32_t* rowptr;
  const int32_t* send;
  const float* vec;
  const float* x;
  const float* w;
  const float* g;
  const float* vx;   // may be null (zero)
  const float* vw;   // may be null (zero)
  const float* vr;   // may be null (zero)
  float* ghat;
  float* xhat;
  float* what;
  float* rhat;
  int n_nodes, n_edges, C, ntiles, xrow, zrow, P, sum_paths;
  int n_send;   // rows of x (senders index x); n_nodes = receivers = rows of rowptr - 1 and z
};

struct VvEdgeWin {
  int v;
  float rx, ry, rz, vrx, vry, vrz;
};

__device__ __forceinline__ VvEdgeWin vvload_win(const VvjpArgs& a, int e, int e1) {
  VvEdgeWin wv;
  if (e < e1) {
    wv.v = __ldg(a.send + e);
    wv.rx = __ldg(a.vec + 3 * e);
    wv.ry = __ldg(a.vec + 3 * e + 1);
    wv.rz = __ldg(a.vec + 3 * e + 2);
    if (a.vr != nullptr) {
      wv.vrx = __ldg(a.vr + 3 * e);
      wv.vry = __ldg(a.vr + 3 * e + 1);
      wv.vrz = __ldg(a.vr + 3 * e + 2);
    } else {
      wv.vrx = wv.vry = wv.vrz = 0.0f;
    }
  } else {
    wv.v = -1;
    wv.rx = 1.0f;
    wv.ry = wv.rz = 0.0f;
    wv.vrx = wv.vry = wv.vrz = 0.0f;
  }
  return wv;
}

template <class Grp>
__device__ __forceinline__ void vvissue_edge(const VvjpArgs& a, int C, float* st, int q, int v,
                                             int k0, bool act) {
  const bool vok = act && v >= 0 && v < a.n_send;
  const int kk = act ? k0 : 0;
  const size_t xo = (size_t)(vok ? v : 0) * a.xrow * C + kk;
  const size_t wo = (size_t)q * a.P * C + kk;
  Grp::issue(st, a.x + xo, (a.vx ? a.vx : a.x) + xo, a.w + wo, (a.vw ? a.vw : a.w) + wo, C, vok,
             vok && a.vx != nullptr, act, act && a.vw != nullptr);
}

// Lane 0 of a reduced group: (I - u u^T) D^T y_hat / |r| plus the
// Hessian-vector product, added into r_hat of edge q.
template <class Grp>
__device__ __forceinline__ void vvjp_rhat_add(const VvjpArgs& a, const float* m, const float (&red)[12],
                                              int q) {
  const float* sc = m + Grp::SBASE;
  const float ux = sc[0], uy = sc[1], uz = sc[2];
  const float wx = sc[3], wy = sc[4], wz = sc[5];
  const float inv = sc[6], uv = sc[7];
  const float ua = ux * red[0] + uy * red[1] + uz * red[2];
  float ox = (red[0] - ux * ua) * inv, oy = (red[1] - uy * ua) * inv, oz = (red[2] - uz * ua) * inv;
  const float Gx = red[3], Gy = red[4], Gz = red[5];
  const float uG = ux * Gx + uy * Gy + uz * Gz, wG = wx * Gx + wy * Gy + wz * Gz;
  const float Hwx = red[6] * wx + red[7] * wy + red[8] * wz;
  const float Hwy = red[7] * wx + red[9] * wy + red[10] * wz;
  const float Hwz = red[8] * wx + red[10] * wy + red[11] * wz;
  const float uHw = ux * Hwx + uy * Hwy + uz * Hwz;
  const float c2 = uv * inv * inv;
  ox += (-(wx * uG + ux * wG) + Hwx - ux * uHw) * inv - (Gx - ux * uG) * c2;
  oy += (-(wy * uG + uy * wG) + Hwy - uy * uHw) * inv - (Gy - uy * uG) * c2;
  oz += (-(wz * uG + uz * wG) + Hwz - uz * uHw) * inv - (Gz - uz * uG) * c2;
  atomicAdd(a.rhat + 3 * (size_t)q + 0, ox);
  atomicAdd(a.rhat + 3 * (size_t)q + 1, oy);
  atomicAdd(a.rhat + 3 * (size_t)q + 2, oz);
}

template <class Grp, int S, int MW, int CC>
__device__ __forceinline__ void vvjp_warp(const VvjpArgs& a, float* smem, int lane, int unit) {
  constexpr int STAGE = Grp::NROW * 128;
  constexpr int NDB = Grp::ND > 0 ? Grp::ND : 1;
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
  const bool wstore = act && a.what != nullptr;
  float* wbase = a.what != nullptr ? a.what : a.ghat;   // any valid pointer when unused

  float4 gr[Grp::NA], gh[Grp::NA];
  if (act) {
    Grp::load_g(a.g + (size_t)u * a.zrow * C + k0, C, a.sum_paths, gr);
  } else {
#pragma unroll
    for (int i = 0; i < Grp::NA; ++i) gr[i] = zero4();
  }
#pragma unroll
  for (int i = 0; i < Grp::NA; ++i) gh[i] = zero4();
  float4 xh[Grp::NX];
#pragma unroll
  for (int i = 0; i < Grp::NX; ++i) xh[i] = zero4();
  float yh[NDB], yb[NDB];
#pragma unroll
  for (int i = 0; i < NDB; ++i) yh[i] = yb[i] = 0.0f;

  VvEdgeWin cur = vvload_win(a, e0 + lane, e1);
  VvEdgeWin nxt = vvload_win(a, e0 + 32 + lane, e1);
#pragma unroll
  for (int s = 0; s < S; ++s) {
    const int q = e0 + s;
    const int v = __shfl_sync(0xffffffffu, cur.v, s);
    if (q < e1) vvissue_edge<Grp>(a, C, st + s * STAGE, q, v, k0, act);
    cp_async_commit();
  }

  for (int q = e0; q < e1; ++q) {
    const int p = q - e0;
    if (p > 0 && (p & 31) == 0) {
      cur = nxt;
      nxt = vvload_win(a, q + 32 + lane, e1);
    }
    if ((p % MW) == 0) {
      const int src = (p & 31) + (lane % MW);
      const float rx = __shfl_sync(0xffffffffu, cur.rx, src);
      const float ry = __shfl_sync(0xffffffffu, cur.ry, src);
      const float rz = __shfl_sync(0xffffffffu, cur.rz, src);
      const float vrx = __shfl_sync(0xffffffffu, cur.vrx, src);
      const float vry = __shfl_sync(0xffffffffu, cur.vry, src);
      const float vrz = __shfl_sync(0xffffffffu, cur.vrz, src);
      __syncwarp();
      if (lane < MW && q + lane < e1) {
        const float inv = 1.0f / sqrtf(rx * rx + ry * ry + rz * rz);
        Grp::make_row(rx * inv, ry * inv, rz * inv, inv, vrx, vry, vrz, mwin + lane * Grp::MSTRIDE);
      }
      __syncwarp();
    }
    const int slot = p % S;
    cp_async_wait<S - 1>();
    const float* m = mwin + (p % MW) * Grp::MSTRIDE;
    Grp::edge(gr, gh, st + slot * STAGE, m, xh, yh, yb,
              wbase + (wstore ? (size_t)q * a.P * C + k0 : 0), C, wstore);
    // sender gradient
    const int v = __shfl_sync(0xffffffffu, cur.v, p & 31);
    if (a.xhat != nullptr && act && v >= 0 && v < a.n_send) {
      Grp::flush_xhat(a.xhat + (size_t)v * a.xrow * C + k0, C, xh);
    } else {
#pragma unroll
      for (int i = 0; i < Grp::NX; ++i) xh[i] = zero4();
    }
    // edge-vector gradient
    if constexpr (Grp::ND > 0) {
      if (a.rhat != nullptr) {
        float red[12];
        Grp::fold(yh, yb, m, red);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
#pragma unroll
          for (int i = 0; i < 12; ++i) red[i] += __shfl_xor_sync(0xffffffffu, red[i], o);
        if (lane == 0) vvjp_rhat_add<Grp>(a, m, red, q);
      }
#pragma unroll
      for (int i = 0; i < NDB; ++i) yh[i] = yb[i] = 0.0f;
    }
    const int pn = p + S;
    if (q + S < e1) {
      int vn;
      if ((pn >> 5) == (p >> 5))
        vn = __shfl_sync(0xffffffffu, cur.v, pn & 31);
      else
        vn = __shfl_sync(0xffffffffu, nxt.v, pn & 31);
      vvissue_edge<Grp>(a, C, st + slot * STAGE, q + S, vn, k0, act);
    }
    cp_async_commit();
  }
  cp_async_wait<0>();
  if (a.ghat != nullptr && act) Grp::store_ghat(a.ghat + (size_t)u * a.zrow * C + k0, C, a.sum_paths, gh);
}

// C = 64: two receivers per warp, half-warp h (lanes 16 h .. 16 h + 15, 4
// channels each) runs receiver 2 unit + h, as in the forward's and the VJP's
// pairing: per half a 16-edge register window, 8 edges of the M window, and
// the reduction of the 12 u-space numbers over the half's 16 lanes.
template <class Grp, int S, int MW>
__device__ __forceinline__ void vvjp_warp_half(const VvjpArgs& a, float* smem, int lane, int unit) {
  constexpr int STAGE = Grp::NROW * 128;
  constexpr int NDB = Grp::ND > 0 ? Grp::ND : 1;
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
  const bool wstore = a.what != nullptr;
  float* wbase = a.what != nullptr ? a.what : a.ghat;   // any valid pointer when unused

  float4 gr[Grp::NA], gh[Grp::NA];
  if (has) {
    Grp::load_g(a.g + (size_t)u * a.zrow * C + k0, C, a.sum_paths, gr);
  } else {
#pragma unroll
    for (int i = 0; i < Grp::NA; ++i) gr[i] = zero4();
  }
#pragma unroll
  for (int i = 0; i < Grp::NA; ++i) gh[i] = zero4();
  float4 xh[Grp::NX];
#pragma unroll
  for (int i = 0; i < Grp::NX; ++i) xh[i] = zero4();
  float yh[NDB], yb[NDB];
#pragma unroll
  for (int i = 0; i < NDB; ++i) yh[i] = yb[i] = 0.0f;

  VvEdgeWin cur = vvload_win(a, e0 + hl, e1);
  VvEdgeWin nxt = vvload_win(a, e0 + 16 + hl, e1);
#pragma unroll
  for (int s = 0; s < S; ++s) {
    const int v = __shfl_sync(0xffffffffu, cur.v, hbase + s);
    if (s < len) vvissue_edge<Grp>(a, C, st + s * STAGE, e0 + s, v, k0, true);
    cp_async_commit();
  }

  for (int p = 0; p < lmax; ++p) {
    const bool on = p < len;
    const int q = e0 + p;
    if (p > 0 && (p & 15) == 0) {
      cur = nxt;
      nxt = vvload_win(a, q + 16 + hl, e1);
    }
    if ((p % HW) == 0) {
      const int src = hbase + (p & 15) + (hl % HW);
      const float rx = __shfl_sync(0xffffffffu, cur.rx, src);
      const float ry = __shfl_sync(0xffffffffu, cur.ry, src);
      const float rz = __shfl_sync(0xffffffffu, cur.rz, src);
      const float vrx = __shfl_sync(0xffffffffu, cur.vrx, src);
      const float vry = __shfl_sync(0xffffffffu, cur.vry, src);
      const float vrz = __shfl_sync(0xffffffffu, cur.vrz, src);
      __syncwarp();
      if (hl < HW && p + hl < len) {
        const float inv = 1.0f / sqrtf(rx * rx + ry * ry + rz * rz);
        Grp::make_row(rx * inv, ry * inv, rz * inv, inv, vrx, vry, vrz, mwin + hl * Grp::MSTRIDE);
      }
      __syncwarp();
    }
    const int slot = p % S;
    cp_async_wait<S - 1>();
    const float* m = mwin + (p % HW) * Grp::MSTRIDE;
    if (on)
      Grp::edge(gr, gh, st + slot * STAGE, m, xh, yh, yb,
                wbase + (wstore ? (size_t)q * a.P * C + k0 : 0), C, wstore);
    // sender gradient
    const int v = __shfl_sync(0xffffffffu, cur.v, hbase + (p & 15));
    if (on && a.xhat != nullptr && v >= 0 && v < a.n_send) {
      Grp::flush_xhat(a.xhat + (size_t)v * a.xrow * C + k0, C, xh);
    } else {
#pragma unroll
      for (int i = 0; i < Grp::NX; ++i) xh[i] = zero4();
    }
    // edge-vector gradient
    if constexpr (Grp::ND > 0) {
      if (a.rhat != nullptr) {
        float red[12];
        if (on) {
          Grp::fold(yh, yb, m, red);
        } else {
#pragma unroll
          for (int i = 0; i < 12; ++i) red[i] = 0.0f;
        }
#pragma unroll
        for (int o = 8; o > 0; o >>= 1)
#pragma unroll
          for (int i = 0; i < 12; ++i) red[i] += __shfl_xor_sync(0xffffffffu, red[i], o);
        if (hl == 0 && on) vvjp_rhat_add<Grp>(a, m, red, q);
      }
#pragma unroll
      for (int i = 0; i < NDB; ++i) yh[i] = yb[i] = 0.0f;
    }
    const int pn = p + S;
    int vn;
    if ((pn >> 4) == (p >> 4))
      vn = __shfl_sync(0xffffffffu, cur.v, hbase + (pn & 15));
    else
      vn = __shfl_sync(0xffffffffu, nxt.v, hbase + (pn & 15));
    if (pn < len) vvissue_edge<Grp>(a, C, st + slot * STAGE, e0 + pn, vn, k0, true);
    cp_async_commit();
  }
  cp_async_wait<0>();
  if (a.ghat != nullptr && has) Grp::store_ghat(a.ghat + (size_t)u * a.zrow * C + k0, C, a.sum_paths, gh);
}

template <int L, int CC, int g>
__device__ __forceinline__ void dispatch_vvjp(int grp, const VvjpArgs& a, float* smem, int lane,
                                              int unit) {
  if constexpr (g < VvjpMeta<L>::G) {
    using Grp = VvjpGroup<L, VvjpMeta<L>::G, g>;
    if (grp == g) {
      if constexpr (CC == 64)
        vvjp_warp_half<Grp, VvjpMeta<L>::S, VvjpMeta<L>::MWIN>(a, smem, lane, unit);
      else
        vvjp_warp<Grp, VvjpMeta<L>::S, VvjpMeta<L>::MWIN, CC>(a, smem, lane, unit);
      return;
    }
    dispatch_vvjp<L, CC, g + 1>(grp, a, smem, lane, unit);
  }
}

template <int L, int CC>
__global__ void __launch_bounds__(VvjpMeta<L>::WARPS * 32, 1) edge_conv_vvjp_kernel(const VvjpArgs a) {
  extern __shared__ __align__(16) float smem[];
  constexpr int WARPS = VvjpMeta<L>::WARPS;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int units = CC == 64 ? (a.n_nodes + 1) / 2 : a.n_nodes * a.ntiles;   // CC = 64: receiver pairs
  const int nb = (units + WARPS - 1) / WARPS;
  const int grp = blockIdx.x / nb;
  const int unit = (blockIdx.x - grp * nb) * WARPS + warp;
  if (unit >= units) return;
  dispatch_vvjp<L, CC, 0>(grp, a, smem + warp * VvjpMeta<L>::WARP_FLOATS, lane, unit);
}

// Split launches (ranks above 4, VvjpMeta<L>::SPLIT): path group g is a
// kernel of its own, so its registers are allocated for that group alone
// instead of for the largest group of one fused kernel; the launches of all
// groups run back to back on the stream and add into the same outputs.
template <int L, int CC, int g>
__global__ void __launch_bounds__(VvjpMeta<L>::WARPS * 32, 1) edge_conv_vvjp_group_kernel(const VvjpArgs a) {
  extern __shared__ __align__(16) float smem[];
  using Grp = VvjpGroup<L, VvjpMeta<L>::G, g>;
  constexpr int WARPS = VvjpMeta<L>::WARPS;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int unit = blockIdx.x * WARPS + warp;
  if (unit >= a.n_nodes * a.ntiles) return;
  vvjp_warp<Grp, VvjpMeta<L>::S, VvjpMeta<L>::MWIN, CC>(a, smem + warp * VvjpMeta<L>::WARP_FLOATS, lane,
                                                          unit);
}

// launches of groups [g, G1)
template <int L, int CC, int g, int G1>
int launch_vvjp_groups(const VvjpArgs& a, cudaStream_t s) {
  if constexpr (g < G1 && g < VvjpMeta<L>::G) {
    static_assert(sizeof(float) * VvjpMeta<L>::SMEM_FLOATS <= 227 * 1024,
                  "VJP-of-VJP kernel shared memory exceeds the 227 KB per-CTA limit of sm_100");
    const size_t smem = sizeof(float) * (size_t)VvjpMeta<L>::SMEM_FLOATS;
    static DeviceFlags configured;
    if (set_smem_once(configured, edge_conv_vvjp_group_kernel<L, CC, g>, smem) != FC_OK)
      return FC_ERR_CUDA;
    constexpr int WARPS = VvjpMeta<L>::WARPS;
    const long long blocks = ((long long)a.n_nodes * a.ntiles + WARPS - 1) / WARPS;
    if (blocks > 0x7fffffffLL) return FC_ERR_ARG;
    edge_conv_vvjp_group_kernel<L, CC, g><<<(unsigned)blocks, WARPS * 32, smem, s>>>(a);
    if (cudaGetLastError() != cudaSuccess) return FC_ERR_CUDA;
    return launch_vvjp_groups<L, CC, g + 1, G1>(a, s);
  }
  return FC_OK;
}

template <int L, int CC>
int launch_vvjp_cc(const VvjpArgs& a, cudaStream_t s) {
  static_assert(sizeof(float) * VvjpMeta<L>::SMEM_FLOATS <= 227 * 1024,
                "VJP-of-VJP kernel shared memory exceeds the 227 KB per-CTA limit of sm_100");
  const size_t smem = sizeof(float) * (size_t)VvjpMeta<L>::SMEM_FLOATS;
  static DeviceFlags configured;
  if (set_smem_once(configured, edge_conv_vvjp_kernel<L, CC>, smem) != FC_OK) return FC_ERR_CUDA;
  const long long units = CC == 64 ? ((long long)a.n_nodes + 1) / 2 : (long long)a.n_nodes * a.ntiles;
  constexpr int WARPS = VvjpMeta<L>::WARPS;
  const long long blocks = (units + WARPS - 1) / WARPS * VvjpMeta<L>::G;
  if (blocks > 0x7fffffffLL) return FC_ERR_ARG;
  edge_conv_vvjp_kernel<L, CC><<<(unsigned)blocks, WARPS * 32, smem, s>>>(a);
  return cudaGetLastError() == cudaSuccess ? FC_OK : FC_ERR_CUDA;
}

}  // namespace fc
