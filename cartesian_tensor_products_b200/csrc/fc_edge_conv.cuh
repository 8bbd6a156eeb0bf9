// libflashcart: receiver-sorted edge convolution, forward.
//
// FlashCart (arXiv 2610.06409) Sec. 4 Eq. (1) and Algorithm 1:
//   z_{u eta k} = sum_{e: u_e = u} w_{e eta k} f_eta(x_{v_e k}, y_e),
//   y_e = T(r-hat_e) shared by all channels.
// Every receiver's sums are accumulated on chip and stored once.
//
// B200 design.  One CTA per (receiver, 128-channel tile); its G warps each
// own a fixed group of output rows (path, component), cut offline so that
// the warps do near-equal work.  A lane owns 4 consecutive channels, so
// every global access is a coalesced 16-byte vector.  Per incoming edge a
// warp needs the sender's x rows its rows touch and the edge's weight rows
// of its paths: each lane streams its own 16-byte slices of those rows into
// a 3-deep shared-memory ring with cp.async, three edges ahead of use, and
// reads back only what it copied (no barrier on the data path).  Every 16
// edges the warp forms, lane-per-edge, the entries
// M[a][b] = sum_b2 K[a][b][b2] y_b2 (y = T(r-hat)) of its rows into a
// warp-private shared-memory window; the per-edge loop then reads them as
// broadcasts and applies them to the lane's 4 channels with packed FP32x2
// FMAs.  Sender indices and edge vectors come from a 32-edge register
// window (one per lane) read with warp shuffles.  With 4 groups every SMSP
// runs one instruction stream (warp g of each resident CTA).  At C = 64 a
// warp runs two receivers, one per half-warp (fwd_warp_half).
#pragma once
#include "fc_common.cuh"
#include "fc_device.cuh"

namespace fc {

struct ConvArgs {
  const int32_t* rowptr;
  const int32_t* send;
  const float* vec;
  const float* x;
  const float* w;
  float* z;
  int n_nodes, n_edges, C, ntiles, xrow, zrow, P, sum_paths;
  int n_send;   // rows of x (senders index x); n_nodes = receivers = rows of rowptr - 1 and z
  int envelope;
  float r_cut, edge_scale;
};

// sender and edge vector of edge `e` for this lane's window slot
struct EdgeWin {
  int v;
  float rx, ry, rz;
};

__device__ __forceinline__ EdgeWin load_win(const ConvArgs& a, int e, int e1) {
  EdgeWin wv;
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
__device__ __forceinline__ void issue_edge(const ConvArgs& a, int C, float* st, int q, int v,
                                           int k0, bool act) {
  const bool vok = act && v >= 0 && v < a.n_send;
  const int kk = act ? k0 : 0;
  const float* xv = a.x + (size_t)(vok ? v : 0) * a.xrow * C + kk;
  const float* we = a.w + (size_t)q * a.P * C + kk;
  Grp::issue(st, xv, we, C, vok, act);
}

// CC > 0: the channel count is the compile-time constant CC (every row
// offset becomes an immediate); CC == 0: runtime a.C.
template <class Grp, int S, int MW, int CC, bool ENV>
__device__ __forceinline__ void fwd_warp(const ConvArgs& a, float* smem, int lane, int unit) {
  constexpr int STAGE = Grp::NROW * 128;  // floats per stage (all lanes)
  const int C = CC > 0 ? CC : a.C;
  const int u = CC == 128 ? unit : unit / a.ntiles;
  const int tile = unit - u * (CC == 128 ? 1 : a.ntiles);
  const int k0 = tile * 128 + lane * 4;
  const bool act = k0 < C;
  int e0 = __ldg(a.rowptr + u), e1 = __ldg(a.rowptr + u + 1);
  e0 = e0 < 0 ? 0 : (e0 > a.n_edges ? a.n_edges : e0);
  e1 = e1 < e0 ? e0 : (e1 > a.n_edges ? a.n_edges : e1);
  float* st = smem + Grp::RING_OFF + lane * 4;
  float* mwin = smem + Grp::MWIN_OFF;

  float4 acc[Grp::NA];
#pragma unroll
  for (int i = 0; i < Grp::NA; ++i) acc[i] = zero4();

  EdgeWin cur = load_win(a, e0 + lane, e1);
  EdgeWin nxt = load_win(a, e0 + 32 + lane, e1);

  // prefill S edges
#pragma unroll
  for (int s = 0; s < S; ++s) {
    const int q = e0 + s;
    const int v = __shfl_sync(0xffffffffu, cur.v, s);
    if (q < e1) issue_edge<Grp>(a, C, st + s * STAGE, q, v, k0, act);
    cp_async_commit();
  }

  for (int q = e0; q < e1; ++q) {
    const int p = q - e0;
    if (p > 0 && (p & 31) == 0) {
      cur = nxt;
      nxt = load_win(a, q + 32 + lane, e1);
    }
    if ((p % MW) == 0) {
      // M entries of the next MW edges, lane-per-edge, into the warp's window
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
        Grp::template make_m<ENV>(rx * inv, ry * inv, rz * inv, es, mwin + lane * Grp::MSTRIDE);
      }
      __syncwarp();
    }
    const int slot = p % S;
    cp_async_wait<S - 1>();
    Grp::template accum<ENV>(acc, st + slot * STAGE, mwin + (p % MW) * Grp::MSTRIDE);
    // refill this slot with edge q + S
    const int pn = p + S;
    if (q + S < e1) {
      int v;
      if ((pn >> 5) == (p >> 5))
        v = __shfl_sync(0xffffffffu, cur.v, pn & 31);
      else
        v = __shfl_sync(0xffffffffu, nxt.v, pn & 31);
      issue_edge<Grp>(a, C, st + slot * STAGE, q + S, v, k0, act);
    }
    cp_async_commit();
  }
  cp_async_wait<0>();
  if (act) Grp::store(a.z + (size_t)u * a.zrow * C + k0, C, a.sum_paths, acc);
}

// C = 64: a warp covers two receivers, half-warp h (lanes 16 h .. 16 h + 15,
// 4 channels each) runs receiver 2 unit + h, so no lane idles.  Each half
// keeps its own 16-edge register window of senders and edge vectors, and the
// M window holds 8 edges per half (the same shared memory as the full warp's
// 16); both halves walk their edges in step, a half whose receiver has fewer
// edges (or none) sitting out the remaining iterations.
template <class Grp, int S, int MW, bool ENV>
__device__ __forceinline__ void fwd_warp_half(const ConvArgs& a, float* smem, int lane, int unit) {
  constexpr int STAGE = Grp::NROW * 128;
  constexpr int C = 64;
  constexpr int HW = MW / 2;   // edges per half in one M window
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
  float* st = smem + Grp::RING_OFF + lane * 4;
  float* mwin = smem + Grp::MWIN_OFF + h * HW * Grp::MSTRIDE;

  float4 acc[Grp::NA];
#pragma unroll
  for (int i = 0; i < Grp::NA; ++i) acc[i] = zero4();

  // lane (h, i) holds edge e0 + 16 j + i of its half's receiver
  EdgeWin cur = load_win(a, e0 + hl, e1);
  EdgeWin nxt = load_win(a, e0 + 16 + hl, e1);

#pragma unroll
  for (int s = 0; s < S; ++s) {
    const int v = __shfl_sync(0xffffffffu, cur.v, hbase + s);
    if (s < len) issue_edge<Grp>(a, C, st + s * STAGE, e0 + s, v, k0, true);
    cp_async_commit();
  }

  for (int p = 0; p < lmax; ++p) {
    if (p > 0 && (p & 15) == 0) {
      cur = nxt;
      nxt = load_win(a, e0 + p + 16 + hl, e1);
    }
    if ((p % HW) == 0) {
      // M entries of the next HW edges of each half, lanes (h, 0 .. HW-1)
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
        Grp::template make_m<ENV>(rx * inv, ry * inv, rz * inv, es, mwin + hl * Grp::MSTRIDE);
      }
      __syncwarp();
    }
    const int slot = p % S;
    cp_async_wait<S - 1>();
    if (p < len) Grp::template accum<ENV>(acc, st + slot * STAGE, mwin + (p % HW) * Grp::MSTRIDE);
    const int pn = p + S;
    int v;
    if ((pn >> 4) == (p >> 4))
      v = __shfl_sync(0xffffffffu, cur.v, hbase + (pn & 15));
    else
      v = __shfl_sync(0xffffffffu, nxt.v, hbase + (pn & 15));
    if (pn < len) issue_edge<Grp>(a, C, st + slot * STAGE, e0 + pn, v, k0, true);
    cp_async_commit();
  }
  cp_async_wait<0>();
  if (has) Grp::store(a.z + (size_t)u * a.zrow * C + k0, C, a.sum_paths, acc);
}

template <int L, int CC, bool ENV, int g>
__device__ __forceinline__ void dispatch_fwd(int grp, const ConvArgs& a, float* smem, int lane,
                                             int unit) {
  if constexpr (g < FwdMeta<L>::G) {
    using Grp = FwdGroup<L, FwdMeta<L>::G, g>;
    if (grp == g) {
      if constexpr (CC == 64)
        fwd_warp_half<Grp, FwdMeta<L>::S, FwdMeta<L>::MWIN, ENV>(a, smem, lane, unit);
      else
        fwd_warp<Grp, FwdMeta<L>::S, FwdMeta<L>::MWIN, CC, ENV>(a, smem, lane, unit);
      return;
    }
    dispatch_fwd<L, CC, ENV, g + 1>(grp, a, smem, lane, unit);
  }
}

// Up to 4 groups: a CTA is the G groups of one receiver tile (warp g runs
// group g, one warp per SMSP).  More groups: a CTA is one group for WARPS
// consecutive receiver tiles, blocks ordered group-major, so an SMSP still
// mostly runs one instruction stream.
template <int L, int CC, bool ENV>
__global__ void __launch_bounds__(FwdMeta<L>::WARPS * 32, 2) edge_conv_fwd_kernel(const ConvArgs a) {
  extern __shared__ __align__(16) float smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if constexpr (!FwdMeta<L>::GROUP_MAJOR) {
    dispatch_fwd<L, CC, ENV, 0>(warp, a, smem, lane, blockIdx.x);
  } else {
    constexpr int WARPS = FwdMeta<L>::WARPS;
    const int units = CC == 64 ? (a.n_nodes + 1) / 2 : a.n_nodes * a.ntiles;
    const int nb = (units + WARPS - 1) / WARPS;
    const int grp = blockIdx.x / nb;
    const int unit = (blockIdx.x - grp * nb) * WARPS + warp;
    if (unit >= units) return;
    dispatch_fwd<L, CC, ENV, 0>(grp, a, smem + warp * FwdMeta<L>::WARP_FLOATS, lane, unit);
  }
}

template <int L, int CC, bool ENV>
static int launch_fwd_cc(const ConvArgs& a, cudaStream_t s) {
  static_assert(sizeof(float) * FwdMeta<L>::SMEM_FLOATS <= 227 * 1024,
                "forward kernel shared memory exceeds the 227 KB per-CTA limit of sm_100");
  const size_t smem = sizeof(float) * (size_t)FwdMeta<L>::SMEM_FLOATS;
  static DeviceFlags configured;
  if (set_smem_once(configured, edge_conv_fwd_kernel<L, CC, ENV>, smem) != FC_OK) return FC_ERR_CUDA;
  // CC = 64: a unit is a pair of receivers (one per half-warp)
  const long long units = CC == 64 ? ((long long)a.n_nodes + 1) / 2 : (long long)a.n_nodes * a.ntiles;
  constexpr int WARPS = FwdMeta<L>::WARPS;
  const long long blocks =
      FwdMeta<L>::GROUP_MAJOR ? (units + WARPS - 1) / WARPS * FwdMeta<L>::G : units;
  if (blocks > 0x7fffffffLL) return FC_ERR_ARG;
  edge_conv_fwd_kernel<L, CC, ENV><<<(unsigned)blocks, WARPS * 32, smem, s>>>(a);
  return cudaGetLastError() == cudaSuccess ? FC_OK : FC_ERR_CUDA;
}

// Host checks and kernel arguments shared by the forward entry points
// (natural-parity paths, odd = 0, or odd-J paths, odd = 1).  Returns FC_OK
// with *launch = false when there is nothing to launch; with sum_paths the
// output is zeroed on the stream (the kernels then add path sums into it).
inline int conv_setup(const fc_conv_desc* d, int n_nodes, int n_send, int n_edges,
                      const int32_t* rowptr, const int32_t* edge_index, const float* edge_vec,
                      const float* x, const float* w, float* z, int odd, cudaStream_t s,
                      ConvArgs& a, bool* launch) {
  *launch = false;
  int st = check_conv_desc(d);
  if (st != FC_OK) return st;
  if (odd && d->lmax_in > 4) return FC_ERR_UNSUPPORTED_RANK;
  if (n_nodes < 0 || n_send < 0 || n_edges < 0) return FC_ERR_ARG;
  if (n_nodes == 0) return n_edges == 0 ? FC_OK : FC_ERR_ARG;
  if (!rowptr || !x || !z) return FC_ERR_ARG;
  if (n_edges > 0 && (!edge_index || !edge_vec || !w)) return FC_ERR_ARG;
  if (!aligned16(x) || !aligned16(z) || (w && !aligned16(w)) || !aligned4(rowptr) ||
      (edge_index && !aligned4(edge_index)) || (edge_vec && !aligned4(edge_vec)))
    return FC_ERR_ALIGN;
  const int L = d->lmax_in;
  const int C = d->channels;
  a.rowptr = rowptr;
  a.send = edge_index ? edge_index + n_edges : nullptr;
  a.vec = edge_vec;
  a.x = x;
  a.w = w;
  a.z = z;
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
  if (d->sum_paths) {
    if (cudaMemsetAsync(z, 0, sizeof(float) * (size_t)n_nodes * a.zrow * C, s) != cudaSuccess)
      return FC_ERR_CUDA;
  }
  *launch = true;
  return FC_OK;
}

template <int L>
static int launch_fwd(const ConvArgs& a, cudaStream_t s) {
  if (a.envelope) {
    if (a.C == 128) return launch_fwd_cc<L, 128, true>(a, s);
    return a.C == 64 ? launch_fwd_cc<L, 64, true>(a, s) : launch_fwd_cc<L, 0, true>(a, s);
  }
  if (a.C == 128) return launch_fwd_cc<L, 128, false>(a, s);
  return a.C == 64 ? launch_fwd_cc<L, 64, false>(a, s) : launch_fwd_cc<L, 0, false>(a, s);
}

}  // namespace fc
