// libflashcart: per-rank channel mix of the correlation ladder on the
// tcgen05 tensor cores, FP32-accurate through a three-term TF32 split.
//
// FlashCart (arXiv 2610.06409) Sec. 5 Eq. (2): after each product, every
// rank-l component row of a node is mapped by the same C x C matrix M_l.  Over
// all rows of rank l this is one dense contraction [N(2l+1) x C] x [C x C], the
// one step of the ladder that is a GEMM.  With x = x_hi + x_lo and
// m = m_hi + m_lo split into TF32 values, x m = x_hi m_hi + x_lo m_hi + x_hi m_lo
// up to a relative 2^-21, so three TF32 MMAs per K step keep the 1e-5
// forward tolerance of FP32 arithmetic while running on the tensor pipe.
//
// Operands arrive pre-split in the "tiled" layout the MMA reads (written by
// the product kernel, or by ladder_split_rows_kernel / ladder_split_mix_kernel
// below): rows of rank l form 128-row tiles (tile_start[l] .. tile_start[l+1]),
// each tile a 64 KB hi block and a 64 KB lo block of 128 rows x 128 channels
// in the core-matrix layout of fc_tc.cuh, so K chunk c (32 channels) is the
// contiguous 16 KB at c * 16 KB of either block; rows past the last row of a
// rank are zeros.  The matrix of rank l is a 64 KB hi and a 64 KB lo block.
//
// The mix kernel moves no data through the SM's load path.  One persistent
// CTA per SM walks a contiguous range of tiles with warp-specialised roles:
//  * warp 0, one thread: bulk copies (TMA engine) of each chunk (hi and lo,
//    32 KB) into one of three shared-memory stages, and of the 128 KB matrix
//    whenever the rank changes, each completing on an mbarrier;
//  * warp 1, one thread: the 12 MMAs of a chunk (128 x 128 x 8 each, the
//    matrix as operand A, the rows as operand B) into a TMEM accumulator
//    D[channel][row], two tiles deep (256 columns); commits free the stage
//    and publish the tile;
//  * warps 4-7: drain D from TMEM (lane = output channel, so every store of a
//    warp is one 128-byte row segment) into the new state while the next
//    tile's MMAs run.  (Staging the drain in shared memory and writing each
//    node's run of rows with bulk stores from one thread measured slower.)
//
// C = 128 only (the tile is the whole channel range); other widths use the
// FP32 SIMT kernels.
//
// This file holds three tensor-core kernels:
//  * ladder_mix_tc_kernel: the mix above.  It is the VJP's B_bar = A_bar M.
//  * path_mix_tc_kernel (further down): the per-rank maps with any K = 32 k_l
//    over FP32 component-major tiles, split in shared memory.  It serves the
//    full ladder's (P_l C -> C) maps and the ladder's forward mix (k_l = 4).
//  * rows_wgrad_tc_kernel (last): weight gradients sum_rows a^T b straight
//    from FP32 rows, transposed and split in shared memory.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <cstring>

#include "fc_common.cuh"
#include "fc_device.cuh"
#include "fc_tc.cuh"

namespace fc {

namespace {

constexpr int kTcC = 128;              // channels = K of every MMA = its M (output channels)
constexpr int kTcRows = 128;           // rows per tile = N of every MMA
constexpr int kTcChunk = 32;           // channels per K chunk
constexpr int kTcChunks = kTcC / kTcChunk;
constexpr int kTcStages = 3;           // shared-memory stages of the row operand
constexpr int kTcThreads = 256;        // warp 0 copies, warp 1 issues, warps 4..7 drain
constexpr int kTcBlockFloats = kTcRows * kTcChunk;   // 4096: one hi or lo chunk block
constexpr int kTcChunkFloats = 2 * kTcBlockFloats;   // hi + lo of one chunk
constexpr int kTcWFloats = kTcC * kTcC;              // 16384: one hi or lo block (tile or matrix)
constexpr int kTcTileFloats = 2 * kTcWFloats;        // hi + lo of a tile
// Bounds of the mbarrier waits (global-timer nanoseconds).  A wait that runs
// out skips the rest of the CTA's work and sets g_tc_error instead of
// hanging; g_tc_wait_ns is the bound of every ordinary wait (settable per
// device through fc_set_wait_timeout), kTcDrainNs the fixed, longer bound of
// the waits on work already in flight (bulk copies, MMAs) that a CTA must
// see finish before it releases TMEM and exits.
constexpr uint64_t kTcDrainNs = 2000000000ull;
constexpr unsigned long long kTcDefaultWaitNs = 500000000ull;
constexpr int kTcBars = 2 * kTcStages + 6;   // stage_full[3], stage_free[3], w_full, acc_full[2], acc_free[2], drain
constexpr size_t kTcSmemBytes =
    sizeof(float) * (2 * kTcWFloats + kTcStages * kTcChunkFloats) + 8 * kTcBars + 8;
static_assert(kTcSmemBytes <= 232448, "shared memory per CTA");

__device__ int g_tc_error = 0;
__device__ unsigned long long g_tc_wait_ns = kTcDefaultWaitNs;

// Launch geometry in registers (scalar fields only, so the argument block is
// never copied to local memory).
struct Geom {
  int N, NY, L;
  int t1, t2, t3, t4, t5, t6, t7;   // tile_start[1..7] (tile_start[0] = 0)
};

__host__ __device__ __forceinline__ int tile_rank(const Geom& g, int t) {
  return (g.L >= 1 && t >= g.t1) + (g.L >= 2 && t >= g.t2) + (g.L >= 3 && t >= g.t3) +
         (g.L >= 4 && t >= g.t4) + (g.L >= 5 && t >= g.t5) + (g.L >= 6 && t >= g.t6);
}

__host__ __device__ __forceinline__ int tile_first(const Geom& g, int l) {
  return l == 0 ? 0 : l == 1 ? g.t1 : l == 2 ? g.t2 : l == 3 ? g.t3 : l == 4 ? g.t4
       : l == 5 ? g.t5 : g.t6;
}

__host__ __device__ __forceinline__ int tile_count(const Geom& g) {
  return g.L == 0 ? g.t1 : g.L == 1 ? g.t2 : g.L == 2 ? g.t3 : g.L == 3 ? g.t4
       : g.L == 4 ? g.t5 : g.L == 5 ? g.t6 : g.t7;
}

Geom make_geom(int L, int N) {
  Geom g{};
  g.N = N;
  g.NY = (L + 1) * (L + 1);
  g.L = L;
  int ts[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  int T = 0;
  for (int l = 0; l <= 7; ++l) {
    ts[l] = T;
    if (l <= L) T += (N * (2 * l + 1) + kTcRows - 1) / kTcRows;
  }
  g.t1 = ts[1]; g.t2 = ts[2]; g.t3 = ts[3]; g.t4 = ts[4]; g.t5 = ts[5]; g.t6 = ts[6]; g.t7 = ts[7];
  return g;
}

__device__ __forceinline__ size_t tc_rank_row(int i, int l, int NY) {
  const int w = 2 * l + 1;
  const int n = i / w;
  return ((size_t)n * NY + l * l + (i - n * w)) * kTcC;
}

__device__ __forceinline__ void split4(const float4 v, uint4& h, uint4& w) {
  tc::split_tf32(v.x, h.x, w.x);
  tc::split_tf32(v.y, h.y, w.y);
  tc::split_tf32(v.z, h.z, w.z);
  tc::split_tf32(v.w, h.w, w.w);
}

// ---------------------------------------------------------------------------
// natural layout [N][NY][128] -> tiled split layout (one CTA per tile chunk)
// ---------------------------------------------------------------------------
// Thread p moves 4 float4 of chunk c of tile t: (row r, K group q) with
// r = 16 (p/32) + 8 (it/2) + p%8, q = (p%32)/8 + 4 (it%2): a warp reads 8 rows
// x 64 contiguous bytes and eight consecutive threads fill one 128-byte core
// matrix.  Rows past the rank's last row are written as zeros.
__global__ void __launch_bounds__(256) ladder_split_rows_kernel(Geom g, const float* __restrict__ in,
                                                                float* __restrict__ xs) {
  const int t = blockIdx.x, c = blockIdx.y;
  const int p = threadIdx.x, lane = p & 31;
  const int l = tile_rank(g, t);
  const int R = g.N * (2 * l + 1);
  const int row0 = (t - tile_first(g, l)) * kTcRows;
  float* hi = xs + (size_t)t * kTcTileFloats + c * kTcBlockFloats;
  float* lo = hi + kTcWFloats;
#pragma unroll
  for (int it = 0; it < 4; ++it) {
    const int r = 16 * (p >> 5) + 8 * (it >> 1) + (lane & 7);
    const int q = (lane >> 3) + 4 * (it & 1);
    const int i = row0 + r;
    float4 v = zero4();
    if (i < R) v = __ldg(reinterpret_cast<const float4*>(in + tc_rank_row(i, l, g.NY) + c * kTcChunk) + q);
    uint4 h, w;
    split4(v, h, w);
    const int off = tc::core_offset(r, 4 * q, kTcRows);
    *reinterpret_cast<uint4*>(hi + off) = h;
    *reinterpret_cast<uint4*>(lo + off) = w;
  }
}

// Mixing matrices [L+1][128][128] -> [L+1][hi, lo][16384] in the core layout
// of operand A (row = output channel j, K = input channel t): forward
// A(j, t) = M[j][t], VJP A(j, t) = M[t][j].
template <int MODE>
__global__ void __launch_bounds__(256) ladder_split_mix_kernel(const float* __restrict__ M,
                                                               float* __restrict__ ws) {
  const int l = blockIdx.y;
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;   // 0 .. 4095
  const int j = idx & (kTcC - 1), q = idx >> 7;            // output channel, K group
  const float* Ml = M + (size_t)l * kTcC * kTcC;
  float4 v;
  if (MODE == 0) {
    v = __ldg(reinterpret_cast<const float4*>(Ml + (size_t)j * kTcC) + q);
  } else {
    v.x = __ldg(Ml + (size_t)(4 * q + 0) * kTcC + j);
    v.y = __ldg(Ml + (size_t)(4 * q + 1) * kTcC + j);
    v.z = __ldg(Ml + (size_t)(4 * q + 2) * kTcC + j);
    v.w = __ldg(Ml + (size_t)(4 * q + 3) * kTcC + j);
  }
  uint4 h, w;
  split4(v, h, w);
  float* hi = ws + (size_t)l * 2 * kTcWFloats;
  const int off = tc::core_offset(j, 4 * q, kTcC);
  *reinterpret_cast<uint4*>(hi + off) = h;
  *reinterpret_cast<uint4*>(hi + kTcWFloats + off) = w;
}

// ---------------------------------------------------------------------------
// the mix: out[row][j] = sum_t A(j, t) x[row][t] over the tiles of every rank
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kTcThreads, 1) ladder_mix_tc_kernel(Geom geo,
                                                                      const float* __restrict__ xs,
                                                                      const float* __restrict__ ws,
                                                                      float* __restrict__ out) {
  extern __shared__ __align__(1024) unsigned char smem[];
  float* w_s = reinterpret_cast<float*>(smem);                // hi, lo: 2 x 16384
  float* x_s = w_s + 2 * kTcWFloats;                          // stages of (hi, lo): 3 x 8192
  uint64_t* stage_full = reinterpret_cast<uint64_t*>(x_s + kTcStages * kTcChunkFloats);
  uint64_t* stage_free = stage_full + kTcStages;
  uint64_t* w_full = stage_free + kTcStages;
  uint64_t* acc_full = w_full + 1;
  uint64_t* acc_free = acc_full + 2;
  uint64_t* drain = acc_free + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int T = tile_count(geo);
  const int t_begin = (int)((long long)blockIdx.x * T / gridDim.x);
  const int t_end = (int)((long long)(blockIdx.x + 1) * T / gridDim.x);

  if (warp == 0) tc::tmem_alloc(tmem_slot, 2 * kTcRows);
  if (tid == 0) {
    for (int s = 0; s < kTcStages; ++s) {
      tc::bar_init(&stage_full[s], 1);
      tc::bar_init(&stage_free[s], 1);
    }
    tc::bar_init(w_full, 1);
    tc::bar_init(&acc_full[0], 1);
    tc::bar_init(&acc_full[1], 1);
    tc::bar_init(&acc_free[0], 128);
    tc::bar_init(&acc_free[1], 128);
    tc::bar_init(drain, 1);
    tc::fence_bar_init();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  const uint64_t lim = g_tc_wait_ns;
  bool fail = false;

  if (warp == 0) {
    // ---------------- bulk-copy producer ----------------
    if (lane == 0) {
      int cur_l = -1, w_loads = 0, g = 0;
      for (int t = t_begin; t < t_end && !fail; ++t) {
        const int ti = t - t_begin;
        const int l = tile_rank(geo, t);
        if (l != cur_l) {
          if (ti > 0) {   // the MMAs of the previous tile have read the old matrix
            const int gl = g - 1;
            if (!tc::bar_wait(&stage_free[gl % kTcStages], (gl / kTcStages) & 1, lim)) {
              fail = true;
              break;
            }
          }
          tc::bar_arrive_expect_tx(w_full, 2 * kTcWFloats * sizeof(float));
          tc::bulk_load(w_s, ws + (size_t)l * 2 * kTcWFloats, 2 * kTcWFloats * sizeof(float), w_full);
          ++w_loads;
          cur_l = l;
        }
        for (int c = 0; c < kTcChunks; ++c, ++g) {
          const int s = g % kTcStages;
          if (g >= kTcStages &&
              !tc::bar_wait(&stage_free[s], ((g - kTcStages) / kTcStages) & 1, lim)) {
            fail = true;
            break;
          }
          const float* src = xs + (size_t)t * kTcTileFloats + c * kTcBlockFloats;
          tc::bar_arrive_expect_tx(&stage_full[s], kTcChunkFloats * sizeof(float));
          tc::bulk_load(x_s + s * kTcChunkFloats, src, kTcBlockFloats * sizeof(float), &stage_full[s]);
          tc::bulk_load(x_s + s * kTcChunkFloats + kTcBlockFloats, src + kTcWFloats,
                        kTcBlockFloats * sizeof(float), &stage_full[s]);
        }
      }
      if (fail) {
        // let the copies already issued land before the CTA can exit
        for (int k = 1; k <= kTcStages && g - k >= 0; ++k)
          tc::bar_wait(&stage_full[(g - k) % kTcStages], ((g - k) / kTcStages) & 1, kTcDrainNs);
        if (w_loads > 0) tc::bar_wait(w_full, (w_loads - 1) & 1, kTcDrainNs);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      constexpr uint32_t idesc = tc::idesc_tf32(kTcC, kTcRows);
      constexpr uint32_t kLbo = kTcRows * 16, kSbo = 128;   // both operands are 128-row blocks
      const uint32_t wh = tc::smem_addr(w_s), wl = tc::smem_addr(w_s + kTcWFloats);
      int cur_l = -1, w_loads = 0, g = 0;
      for (int t = t_begin; t < t_end && !fail; ++t) {
        const int ti = t - t_begin;
        const int l = tile_rank(geo, t);
        const uint32_t d_tmem = tmem + (uint32_t)(ti & 1) * kTcRows;
        if (l != cur_l) {
          if (!tc::bar_wait(w_full, w_loads & 1, lim)) {
            fail = true;
            break;
          }
          ++w_loads;
          cur_l = l;
        }
        // the epilogue has drained this accumulator (tile ti - 2)
        if (ti >= 2 && !tc::bar_wait(&acc_free[ti & 1], ((ti - 2) >> 1) & 1, lim)) {
          fail = true;
          break;
        }
        tc::fence_after_sync();
        for (int c = 0; c < kTcChunks; ++c, ++g) {
          const int s = g % kTcStages;
          if (!tc::bar_wait(&stage_full[s], (g / kTcStages) & 1, lim)) {
            fail = true;
            break;
          }
          tc::fence_after_sync();
          const uint32_t xh = tc::smem_addr(x_s + s * kTcChunkFloats);
          const uint32_t xl = xh + kTcBlockFloats * sizeof(float);
#pragma unroll
          for (int j = 0; j < kTcChunk / 8; ++j) {
            const uint32_t kx = 2 * j * kLbo;                          // K group 2j of the chunk
            const uint32_t kw = (c * (kTcChunk / 4) + 2 * j) * kLbo;   // same K group of A
            const uint64_t dwh = tc::smem_desc(wh + kw, kLbo, kSbo);
            const uint64_t dwl = tc::smem_desc(wl + kw, kLbo, kSbo);
            const uint64_t dxh = tc::smem_desc(xh + kx, kLbo, kSbo);
            const uint64_t dxl = tc::smem_desc(xl + kx, kLbo, kSbo);
            tc::mma_tf32(d_tmem, dwh, dxh, idesc, (c | j) != 0);
            tc::mma_tf32(d_tmem, dwh, dxl, idesc, 1u);
            tc::mma_tf32(d_tmem, dwl, dxh, idesc, 1u);
          }
          tc::commit(&stage_free[s]);
          if (c == kTcChunks - 1) tc::commit(&acc_full[ti & 1]);
        }
      }
      // every MMA issued above has finished (also after a wait gave up)
      // before the CTA releases TMEM and its shared memory
      tc::commit(drain);
      if (!tc::bar_wait(drain, 0, kTcDrainNs)) fail = true;
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ---------------- epilogue: TMEM -> new state ----------------
    const int ew = warp - 4;                         // TMEM lane quarter
    const int j = 32 * ew + lane;                    // output channel
    for (int t = t_begin; t < t_end; ++t) {
      const int ti = t - t_begin;
      const int l = tile_rank(geo, t);
      const int w = 2 * l + 1;
      const int R = geo.N * w;
      const int row0 = (t - tile_first(geo, l)) * kTcRows;
      const uint32_t d_tmem = tmem + (uint32_t)(ti & 1) * kTcRows + ((uint32_t)(32 * ew) << 16);
      if (!tc::bar_wait(&acc_full[ti & 1], (ti >> 1) & 1, lim)) {
        fail = true;
        break;
      }
      tc::fence_after_sync();
#pragma unroll
      for (int q = 0; q < kTcRows / 32; ++q) {
        float v[32];
        tc::tmem_ld32(d_tmem + 32 * q, v);
        const int i0 = row0 + 32 * q;
        int n = i0 / w, cc = i0 - (i0 / w) * w;
#pragma unroll
        for (int r = 0; r < 32; ++r) {
          if (i0 + r < R) out[((size_t)n * geo.NY + l * l + cc) * kTcC + j] = v[r];
          if (++cc == w) { cc = 0; ++n; }
        }
      }
      tc::fence_before_sync();
      tc::bar_arrive(&acc_free[ti & 1]);
    }
  }
  if (fail) atomicExch(&g_tc_error, 1);
  // every MMA completed before its tile was drained; release TMEM
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, 2 * kTcRows);
  }
}

// ---------------------------------------------------------------------------
// path + channel map of the full ladder: out[row][j] = sum_k W_l[j][k] x[row][k]
// ---------------------------------------------------------------------------
// A row of rank l has K = 32 k_l inputs (P_l paths x 128 channels), more than
// one stage holds, so each stage carries a K chunk of both operands: the
// tile's 128 rows x 32 inputs in FP32 and the map's 128 outputs x 32 inputs
// as TF32 hi and lo (48 KB), three stages deep.  The row operand crosses HBM
// once in FP32 (half the bytes of a pre-split operand): two converter warps
// split each chunk into hi / lo blocks in shared memory (two buffers) for the
// MMAs, with a proxy fence before they publish it.  The map chunks are
// re-read from L2 by every tile of the rank (a map is at most 1.3 MB split).  CTAs take
// contiguous tile ranges of equal K-chunk count (tiles of different ranks
// differ in length).  Roles as in the mix above, with one change for
// accuracy: the tensor core's FP32 accumulation loses a little at every
// MMA, and over K = P_l 128 inputs (up to 336 MMAs) that loss builds up past
// the forward tolerance.  So each path (4 chunks, the K of the plain mix)
// goes to its own TMEM accumulator, two alternating, and the epilogue adds
// the partial sums in FP32 registers (round-to-nearest) before it writes
// the tile out.  The epilogue only stores (a read-modify-write of a running
// sum here serialised on load latency and starved the tensor pipe).
constexpr int kPmGroup = 4;   // chunks per accumulator: one path of 128 inputs

constexpr int kPmStageFloats = 3 * kTcBlockFloats;   // x (FP32), W hi, W lo
constexpr int kPmCvtFloats = 2 * kTcBlockFloats;     // x hi, x lo
constexpr int kPmCvtThreads = 128;                   // warps 2, 3, 8 and 9
constexpr int kPmThreads = 320;   // w0 copies, w1 issues, w2-3 and w8-9 convert, w4-7 drain
constexpr uint32_t kPmTmemCols = 512;                 // 2 accumulators + the running sum of a tile
constexpr uint32_t kPmSumCol = 2 * kTcRows;
constexpr size_t kPmSmemBytes =
    sizeof(float) * (kTcStages * kPmStageFloats + 2 * kPmCvtFloats) + 8 * 16 + 8;
static_assert(kPmSmemBytes <= 232448, "shared memory per CTA");

// Units of work: (map e, tile t) pairs, rank by rank, the maps of a rank one
// after the other (a map is loaded once per run of the rank's tiles); a unit
// of rank l is k_l K chunks.
__host__ __device__ __forceinline__ int pg_units(const PathGeom& g, int l) {
  return (pg_ts(g, l + 1) - pg_ts(g, l)) * pg_pe(g, l);
}

__device__ __forceinline__ long long pg_chunks_before(const PathGeom& g, int l) {
  long long c = 0;
#pragma unroll
  for (int r = 0; r < 5; ++r)
    if (r < l) c += (long long)pg_units(g, r) * pg_kc(g, r);
  return c;
}

// first unit that starts at or after K chunk P of the whole run
__device__ __forceinline__ int pg_unit_at(const PathGeom& g, long long P) {
  long long cum = 0;
  int us = 0;
  for (int l = 0; l <= g.L; ++l) {
    const int nu = pg_units(g, l), kc = pg_kc(g, l);
    const long long cl = (long long)nu * kc;
    if (P < cum + cl) return us + (int)((P - cum + kc - 1) / kc);
    cum += cl;
    us += nu;
  }
  return us;
}

// unit u -> rank l, tile t, map e
__device__ __forceinline__ void pg_unit(const PathGeom& g, int u, int& l, int& t, int& e) {
  int us = 0;
  l = 0;
  while (l < g.L && u >= us + pg_units(g, l)) {
    us += pg_units(g, l);
    ++l;
  }
  const int nt = pg_ts(g, l + 1) - pg_ts(g, l);
  const int v = u - us;
  e = v / nt;
  t = pg_ts(g, l) + (v - e * nt);
}

// natural [N][NY][128] -> component-major FP32 operand tiles with k_l = 4
// (one CTA per tile chunk; thread mapping as in ladder_split_rows_kernel).
__global__ void __launch_bounds__(256) path_split_rows_kernel(PathGeom g, const float* __restrict__ in,
                                                              float* __restrict__ xs) {
  const int t = blockIdx.x, c = blockIdx.y;
  const int p = threadIdx.x, lane = p & 31;
  const int l = pg_rank(g, t);
  const int kc = pg_kc(g, l);   // rows of 32 kc channels (128 or 256)
  if (c >= kc) return;
  const int tr = t - pg_ts(g, l);
  const int comp = tr / g.nb, n0 = (tr - comp * g.nb) * kTcRows;
  float* dst = xs + pg_xbase(g, l) + (size_t)tr * kc * kTcBlockFloats + c * kTcBlockFloats;
#pragma unroll
  for (int it = 0; it < 4; ++it) {
    const int r = 16 * (p >> 5) + 8 * (it >> 1) + (lane & 7);
    const int q = (lane >> 3) + 4 * (it & 1);
    const int n = n0 + r;
    float4 v = zero4();
    if (n < g.N)
      v = __ldg(reinterpret_cast<const float4*>(in + ((size_t)n * g.NY + l * l + comp) * (kTcChunk * kc) +
                                                c * kTcChunk) + q);
    *reinterpret_cast<float4*>(dst + tc::core_offset(r, 4 * q, kTcRows)) = v;
  }
}

// Map e of rank l is rows 128 e .. 128 e + 127 of the rank's [128 e_l][K]
// matrix (e_l = 1: the whole [128][K] map).
__global__ void __launch_bounds__(256) path_split_map_kernel(PathGeom g, const float* __restrict__ W,
                                                             float* __restrict__ ws) {
  const int l = blockIdx.y, c = blockIdx.x, e = blockIdx.z;
  if (l > g.L) return;
  const int kc = pg_kc(g, l);
  if (c >= kc || e >= pg_pe(g, l)) return;
  const int K = 32 * kc;
  long long woff = 0;
  for (int r = 0; r < l; ++r) woff += 4096LL * pg_kc(g, r) * pg_pe(g, r);
  const float* Wl = W + woff + (long long)e * kTcC * K;
  float* hi = ws + pg_wbase(g, l) + (long long)e * 2 * kc * kTcBlockFloats + (size_t)c * kTcBlockFloats;
#pragma unroll
  for (int it = 0; it < 4; ++it) {
    const int idx = it * 256 + threadIdx.x;   // 0 .. 1023
    const int j = idx >> 3, q = idx & 7;      // output channel, group of 4 inputs
    const float4 v = __ldg(reinterpret_cast<const float4*>(Wl + (size_t)j * K + 32 * c) + q);
    uint4 h, w;
    split4(v, h, w);
    const int off = tc::core_offset(j, 4 * q, kTcC);
    *reinterpret_cast<uint4*>(hi + off) = h;
    *reinterpret_cast<uint4*>(hi + (size_t)kc * kTcBlockFloats + off) = w;
  }
}

// Map e of rank l: A(j', t) = Wq_l[t][e 128 + j'], the transposed block e of
// Wq_l = [32 k_l][128 e_l] at Wq + 4096 sum_{l'<l} k_l' e_l' (the full
// ladder: k_l = 4, e_l = P_l; the ladder VJP at 256 channels: k_l = 8, e_l = 2,
// Wq_l = M_l), split to hi / lo blocks at ws + pg_wbase(l) + e 2 k_l 4096.
// One CTA per (K chunk, map, rank).
__global__ void __launch_bounds__(256) path_split_map_t_kernel(PathGeom g, const float* __restrict__ Wq,
                                                               float* __restrict__ ws) {
  const int c = blockIdx.x, e = blockIdx.y, l = blockIdx.z;
  if (l > g.L || e >= pg_pe(g, l)) return;
  const int kc = pg_kc(g, l);
  if (c >= kc) return;
  long long qoff = 0;   // Wq_r is [32 k_r][128 e_r]
  for (int r = 0; r < l; ++r) qoff += 4096LL * pg_kc(g, r) * pg_pe(g, r);
  const int row = kTcC * pg_pe(g, l);   // floats per row of Wq_l
  const float* Wl = Wq + qoff;
  float* hi = ws + pg_wbase(g, l) + (long long)e * 2 * kc * kTcBlockFloats + (size_t)c * kTcBlockFloats;
#pragma unroll
  for (int it = 0; it < 4; ++it) {
    const int idx = it * 256 + threadIdx.x;   // 0 .. 1023
    const int j = idx & (kTcC - 1), q = idx >> 7;   // output column j', group of 4 inputs
    const int t = 32 * c + 4 * q;
    float4 v;
    v.x = __ldg(Wl + (size_t)(t + 0) * row + e * kTcC + j);
    v.y = __ldg(Wl + (size_t)(t + 1) * row + e * kTcC + j);
    v.z = __ldg(Wl + (size_t)(t + 2) * row + e * kTcC + j);
    v.w = __ldg(Wl + (size_t)(t + 3) * row + e * kTcC + j);
    uint4 h, w;
    split4(v, h, w);
    const int off = tc::core_offset(j, 4 * q, kTcC);
    *reinterpret_cast<uint4*>(hi + off) = h;
    *reinterpret_cast<uint4*>(hi + (size_t)kc * kTcBlockFloats + off) = w;
  }
}

__global__ void __launch_bounds__(kPmThreads, 1) path_mix_tc_kernel(PathGeom geo,
                                                                    const float* __restrict__ xs,
                                                                    const float* __restrict__ ws,
                                                                    float* __restrict__ out) {
  extern __shared__ __align__(1024) unsigned char smem[];
  float* st = reinterpret_cast<float*>(smem);
  float* cv = st + kTcStages * kPmStageFloats;   // converted x: 2 buffers of (hi, lo)
  uint64_t* stage_full = reinterpret_cast<uint64_t*>(cv + 2 * kPmCvtFloats);
  uint64_t* stage_free = stage_full + kTcStages;
  uint64_t* cvt_full = stage_free + kTcStages;
  uint64_t* cvt_free = cvt_full + 2;
  uint64_t* acc_full = cvt_free + 2;
  uint64_t* acc_free = acc_full + 2;
  uint64_t* drain = acc_free + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const long long total = pg_chunks_before(geo, geo.L + 1);
  const int u_begin = pg_unit_at(geo, (long long)blockIdx.x * total / gridDim.x);
  const int u_end = pg_unit_at(geo, (long long)(blockIdx.x + 1) * total / gridDim.x);

  if (warp == 0) tc::tmem_alloc(tmem_slot, kPmTmemCols);
  if (tid == 0) {
    for (int s = 0; s < kTcStages; ++s) {
      tc::bar_init(&stage_full[s], 1);
      tc::bar_init(&stage_free[s], kPmCvtThreads / 32 + 1);   // converter warps + the MMA commit
    }
    for (int b = 0; b < 2; ++b) {
      tc::bar_init(&cvt_full[b], kPmCvtThreads / 32);
      tc::bar_init(&cvt_free[b], 1);
      tc::bar_init(&acc_full[b], 1);
      tc::bar_init(&acc_free[b], 128);
    }
    tc::bar_init(drain, 1);
    tc::fence_bar_init();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  const uint64_t lim = g_tc_wait_ns;
  bool fail = false;

  if (warp == 0) {
    // ---------------- bulk-copy producer ----------------
    if (lane == 0) {
      int g = 0;
      for (int u = u_begin; u < u_end && !fail; ++u) {
        int l, t, e;
        pg_unit(geo, u, l, t, e);
        const int kc = pg_kc(geo, l);
        const float* xt = xs + pg_xbase(geo, l) + (long long)(t - pg_ts(geo, l)) * kc * kTcBlockFloats;
        const float* wt = ws + pg_wbase(geo, l) + (long long)e * 2 * kc * kTcBlockFloats;
        const size_t lo = (size_t)kc * kTcBlockFloats;
        for (int c = 0; c < kc; ++c, ++g) {
          const int s = g % kTcStages;
          if (g >= kTcStages &&
              !tc::bar_wait(&stage_free[s], ((g - kTcStages) / kTcStages) & 1, lim)) {
            fail = true;
            break;
          }
          float* dst = st + s * kPmStageFloats;
          const size_t co = (size_t)c * kTcBlockFloats;
          constexpr uint32_t kB = kTcBlockFloats * sizeof(float);
          tc::bar_arrive_expect_tx(&stage_full[s], kPmStageFloats * sizeof(float));
          tc::bulk_load(dst, xt + co, kB, &stage_full[s]);
          tc::bulk_load(dst + kTcBlockFloats, wt + co, kB, &stage_full[s]);
          tc::bulk_load(dst + 2 * kTcBlockFloats, wt + lo + co, kB, &stage_full[s]);
        }
      }
      if (fail)   // let the copies already issued land
        for (int k = 1; k <= kTcStages && g - k >= 0; ++k)
          tc::bar_wait(&stage_full[(g - k) % kTcStages], ((g - k) / kTcStages) & 1, kTcDrainNs);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      constexpr uint32_t idesc = tc::idesc_tf32(kTcC, kTcRows);
      constexpr uint32_t kLbo = kTcRows * 16, kSbo = 128;
      int g = 0, h = 0;   // chunks and accumulator groups issued
      for (int u = u_begin; u < u_end && !fail; ++u) {
        int l, t, e;
        pg_unit(geo, u, l, t, e);
        const int kc = pg_kc(geo, l);
        for (int c = 0; c < kc; ++c, ++g) {
          const uint32_t d_tmem = tmem + (uint32_t)(h & 1) * kTcRows;
          if (c % kPmGroup == 0) {   // the epilogue has added group h - 2
            if (h >= 2 && !tc::bar_wait(&acc_free[h & 1], ((h - 2) >> 1) & 1, lim)) {
              fail = true;
              break;
            }
            tc::fence_after_sync();
          }
          const int s = g % kTcStages, b = g & 1;
          if (!tc::bar_wait(&stage_full[s], (g / kTcStages) & 1, lim) ||
              !tc::bar_wait(&cvt_full[b], (g >> 1) & 1, lim)) {
            fail = true;
            break;
          }
          tc::fence_after_sync();
          const uint32_t wh = tc::smem_addr(st + s * kPmStageFloats) + kTcBlockFloats * sizeof(float);
          const uint32_t wl = wh + kTcBlockFloats * sizeof(float);
          const uint32_t xh = tc::smem_addr(cv + b * kPmCvtFloats);
          const uint32_t xl = xh + kTcBlockFloats * sizeof(float);
#pragma unroll
          for (int j = 0; j < kTcChunk / 8; ++j) {
            const uint32_t kx = 2 * j * kLbo;
            const uint64_t dwh = tc::smem_desc(wh + kx, kLbo, kSbo);
            const uint64_t dwl = tc::smem_desc(wl + kx, kLbo, kSbo);
            const uint64_t dxh = tc::smem_desc(xh + kx, kLbo, kSbo);
            const uint64_t dxl = tc::smem_desc(xl + kx, kLbo, kSbo);
            tc::mma_tf32(d_tmem, dwh, dxh, idesc, ((c % kPmGroup) | j) != 0);
            tc::mma_tf32(d_tmem, dwh, dxl, idesc, 1u);
            tc::mma_tf32(d_tmem, dwl, dxh, idesc, 1u);
          }
          tc::commit(&stage_free[s]);
          tc::commit(&cvt_free[b]);
          if (c % kPmGroup == kPmGroup - 1 || c == kc - 1) tc::commit(&acc_full[(h++) & 1]);
        }
      }
      // every MMA issued above has finished (also after a wait gave up)
      // before the CTA releases TMEM and its shared memory
      tc::commit(drain);
      if (!tc::bar_wait(drain, 0, kTcDrainNs)) fail = true;
    }
    __syncwarp();
  } else if (warp < 4 || warp >= 8) {
    // ---------------- converter: FP32 chunk -> TF32 hi / lo blocks ----------------
    const int ct = warp < 4 ? tid - 64 : tid - 192;   // 0 .. 127
    int g = 0;
    for (int u = u_begin; u < u_end && !fail; ++u) {
      int l, t, e;
      pg_unit(geo, u, l, t, e);
      const int kc = pg_kc(geo, l);
      for (int c = 0; c < kc; ++c, ++g) {
        const int s = g % kTcStages, b = g & 1;
        if (!tc::bar_wait(&stage_full[s], (g / kTcStages) & 1, lim) ||
            (g >= 2 && !tc::bar_wait(&cvt_free[b], ((g - 2) >> 1) & 1, lim))) {
          fail = true;
          break;
        }
        const uint32_t src = tc::smem_addr(st + s * kPmStageFloats) + 16 * ct;
        const uint32_t hi = tc::smem_addr(cv + b * kPmCvtFloats) + 16 * ct;
        constexpr uint32_t kLo = kTcBlockFloats * sizeof(float), kStep = 16 * kPmCvtThreads;
        constexpr int kIters = kTcBlockFloats / 4 / kPmCvtThreads;   // 8
        float4 v[kIters];
#pragma unroll
        for (int i = 0; i < kIters; ++i)
          asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                       : "=f"(v[i].x), "=f"(v[i].y), "=f"(v[i].z), "=f"(v[i].w)
                       : "r"(src + i * kStep));
#pragma unroll
        for (int i = 0; i < kIters; ++i) {
          uint4 h, w;
          split4(v[i], h, w);
          asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(hi + i * kStep), "r"(h.x),
                       "r"(h.y), "r"(h.z), "r"(h.w) : "memory");
          asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(hi + kLo + i * kStep), "r"(w.x),
                       "r"(w.y), "r"(w.z), "r"(w.w) : "memory");
        }
        tc::fence_proxy_async();   // the generic-proxy writes, visible to the MMAs
        __syncwarp();              // one arrival per warp
        if (lane == 0) {
          tc::bar_arrive(&cvt_full[b]);
          tc::bar_arrive(&stage_free[s]);
        }
      }
    }
  } else {
    // ---------------- epilogue: sum the groups of a tile, write out ----------------
    // Group sums stay in TMEM (columns kPmSumCol..): the first group of a
    // multi-group tile is copied there, later ones added; the last group is
    // added on the way out.  A one-group tile is stored straight from its
    // accumulator.  (128 running sums in registers capped the block at two
    // converter warps.)
    const int ew = warp - 4;
    const int j = 32 * ew + lane;
    const uint32_t lane_off = (uint32_t)(32 * ew) << 16;
    int h = 0;
    for (int u = u_begin; u < u_end && !fail; ++u) {
      int l, t, e;
      pg_unit(geo, u, l, t, e);
      const int kc = pg_kc(geo, l);
      const int tr = t - pg_ts(geo, l);
      const int cmc = tr / geo.nb;                     // the tile's component
      const int cmn = (tr - cmc * geo.nb) * kTcRows;   // and its first node
      const int ng = (kc + kPmGroup - 1) / kPmGroup;
      float* o = out + ((size_t)cmn * geo.orow + pg_ooff(geo, l) + (size_t)cmc * pg_pe(geo, l) + e) * kTcC + j;
      const size_t step = (size_t)geo.orow * kTcC;
      const int nr = min(kTcRows, geo.N - cmn);
      for (int gi = 0; gi < ng; ++gi, ++h) {
        if (!tc::bar_wait(&acc_full[h & 1], (h >> 1) & 1, lim)) {
          fail = true;
          break;
        }
        tc::fence_after_sync();
        const uint32_t d_tmem = tmem + (uint32_t)(h & 1) * kTcRows + lane_off;
        const uint32_t s_tmem = tmem + kPmSumCol + lane_off;
        const bool last = gi == ng - 1;
#pragma unroll 1
        for (int q = 0; q < kTcRows / 32; ++q) {
          float v[32];
          tc::tmem_ld32(d_tmem + 32 * q, v);
          if (gi > 0) {
            float sv[32];
            tc::tmem_ld32(s_tmem + 32 * q, sv);
#pragma unroll
            for (int r = 0; r < 32; ++r) v[r] += sv[r];
          }
          if (last) {
            float* oq = o + (size_t)(32 * q) * step;
#pragma unroll
            for (int r = 0; r < 32; ++r) {
              if (32 * q + r < nr) *oq = v[r];
              oq += step;
            }
          } else {
            uint32_t w[32];
#pragma unroll
            for (int r = 0; r < 32; ++r) w[r] = __float_as_uint(v[r]);
            tc::tmem_st32(s_tmem + 32 * q, w);
          }
        }
        if (!last) tc::tmem_wait_st();
        tc::fence_before_sync();
        tc::bar_arrive(&acc_free[h & 1]);
      }
    }
  }
  if (fail) atomicExch(&g_tc_error, 1);
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, kPmTmemCols);
  }
}

// ---------------------------------------------------------------------------
// weight gradient from FP32 rows: Wb_l[j][e 128 + k] += sum_i a[i][j] b_e[i][k]
// ---------------------------------------------------------------------------
// The contraction runs over the rows i of rank l (node n, component c): K is
// the row index, so both operands enter the MMA transposed.  Nothing is
// pre-split in global memory.  A K chunk is wg_nodes(l) = 32 / (2l+1) whole
// nodes of rank l (32, 30, 30, 28, 27 rows for l = 0..4): one thread loads it
// for both operands with two tiled TMA copies (operand a as a 3-D tensor:
// channel, component, node; operand b as a 4-D tensor: channel, map e,
// component, node; nodes past N are filled with zeros) into one of four FP32
// stages.  Eight converter warps read a stage (one channel of all 32 rows per
// thread, conflict-free), release it, and split the values into TF32 hi / lo:
// operand a goes to tensor memory as the MMA's A operand (row j of A in TMEM
// lane j, the K rows along columns: one 32-column store per thread), operand
// b to K-major core-matrix blocks in shared memory.  One thread issues the 12
// MMAs of a chunk (M = N = 128: D[j][k], three TF32 products per K step, A
// from TMEM), three converted buffers deep, and four warps add each finished
// accumulator into Wb with vector atomics.
//
// Measured on the way here (4096 nodes, rank 3, 2048 row chunks of 32):
//  * a row per copy (cp.async from one warp, or one bulk copy per lane) took
//    2300 and 4000 cycles per chunk to issue;
//  * with both MMA operands in shared memory only two FP32 stages and two
//    converted buffers (64 KB each) fit, about one chunk was in flight per SM,
//    and a chunk cost about one loaded memory latency (2400 cycles);
//  * A in TMEM halves the converted buffers and the MMA's shared-memory reads.
// The CTAs share the chunk list evenly; a segment (one accumulator chain) is
// a run of at most kRwSeg chunks of one (rank, map), which bounds the chain
// at 12 kRwSeg MMAs for FP32-level accuracy.  Two accumulators alternate in
// TMEM so that a drain overlaps the next segment's MMAs.
constexpr int kRwSeg = 32;                            // chunks per accumulator chain
constexpr int kRwThreads = 448;                       // w0 loads, w1 issues, w2-9 convert, w10-13 drain
constexpr int kRwCvtWarps = 8;
constexpr int kRwStages = 4;                          // FP32 stages
constexpr int kRwBufs = 3;                            // converted buffers (B in smem, A in TMEM)
constexpr int kRwRowFloats = kTcChunk * kTcC;         // 4096: 32 rows x 128 channels
constexpr int kRwStageFloats = 2 * kRwRowFloats;      // both operands, FP32
constexpr int kRwCvtFloats = 2 * kTcBlockFloats;      // operand b, hi and lo
constexpr uint32_t kRwTmemCols = 512;                 // 2 accumulators + kRwBufs x (A hi, A lo)
constexpr uint32_t kRwACol = 2 * kTcC;                // first A column
constexpr size_t kRwSmemBytes =
    sizeof(float) * (kRwStages * kRwStageFloats + kRwBufs * kRwCvtFloats) + 8 * 24 + 8;
static_assert(kRwSmemBytes <= 232448, "shared memory per CTA");
static_assert(kRwACol + kRwBufs * 2 * kTcChunk <= kRwTmemCols, "tensor memory columns");

// Tensor maps of the two operands, one per rank (unused ranks zero).
struct WgMaps {
  CUtensorMap a[5];   // 3-D: 128 channels, 2l+1 components (row stride), N nodes (stride sa rows)
  CUtensorMap b[5];   // 4-D: 128 channels, pe_l maps, 2l+1 components, N nodes (stride sb rows)
};

// nodes per K chunk of rank l, and the chunk list: rank by rank, the maps of
// a rank one after the other, a map's chunks in node order
__host__ __device__ __forceinline__ int wg_nodes(int l) { return kTcChunk / (2 * l + 1); }
__host__ __device__ __forceinline__ int wg_chunks(const WgGeom& g, int l) {
  return (g.N + wg_nodes(l) - 1) / wg_nodes(l);
}
__device__ __forceinline__ void wg_chunk(const WgGeom& g, int ch, int& l, int& e, int& q) {
  l = 0;
  int c0 = 0;
  while (l < g.L && ch >= c0 + wg_pe(g, l) * wg_chunks(g, l)) {
    c0 += wg_pe(g, l) * wg_chunks(g, l);
    ++l;
  }
  const int nc = wg_chunks(g, l);
  e = (ch - c0) / nc;
  q = ch - c0 - e * nc;
}

__global__ void __launch_bounds__(kRwThreads, 1) rows_wgrad_tc_kernel(WgGeom geo,
                                                                      const __grid_constant__ WgMaps maps,
                                                                      float* __restrict__ Wb) {
  extern __shared__ __align__(1024) unsigned char smem[];
  float* st = reinterpret_cast<float*>(smem);       // stages: a rows, b rows (FP32)
  float* cv = st + kRwStages * kRwStageFloats;      // converted b: hi, lo
  uint64_t* stage_full = reinterpret_cast<uint64_t*>(cv + kRwBufs * kRwCvtFloats);
  uint64_t* stage_free = stage_full + kRwStages;
  uint64_t* cvt_full = stage_free + kRwStages;
  uint64_t* cvt_free = cvt_full + kRwBufs;
  uint64_t* acc_full = cvt_free + kRwBufs;
  uint64_t* acc_free = acc_full + 2;
  uint64_t* drain = acc_free + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  int total = 0;
  for (int l = 0; l <= geo.L; ++l) total += wg_pe(geo, l) * wg_chunks(geo, l);
  const int c_begin = (int)((long long)blockIdx.x * total / gridDim.x);
  const int c_end = (int)((long long)(blockIdx.x + 1) * total / gridDim.x);

  if (warp == 0) tc::tmem_alloc(tmem_slot, kRwTmemCols);
  if (tid == 0) {
    for (int i = 0; i < kRwStages; ++i) {
      tc::bar_init(&stage_full[i], 1);
      tc::bar_init(&stage_free[i], kRwCvtWarps);
    }
    for (int i = 0; i < kRwBufs; ++i) {
      tc::bar_init(&cvt_full[i], kRwCvtWarps);
      tc::bar_init(&cvt_free[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      tc::bar_init(&acc_full[i], 1);
      tc::bar_init(&acc_free[i], 128);
    }
    tc::bar_init(drain, 1);
    tc::fence_bar_init();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  const uint64_t lim = g_tc_wait_ns;
  bool fail = false;

  if (warp == 0) {
    // ---------------- producer: two tiled TMA loads per chunk ----------------
    int g = 0;
    if (lane == 0) {
      for (int ch = c_begin; ch < c_end && !fail; ++ch, ++g) {
        int l, e, q;
        wg_chunk(geo, ch, l, e, q);
        const int s = g % kRwStages;
        if (g >= kRwStages && !tc::bar_wait(&stage_free[s], ((g / kRwStages) - 1) & 1, lim)) {
          fail = true;
          break;
        }
        const int nn = wg_nodes(l), rows = nn * (2 * l + 1);
        float* dst = st + s * kRwStageFloats;
        tc::bar_arrive_expect_tx(&stage_full[s], (uint32_t)(2 * rows * kTcC * sizeof(float)));
        tc::tma_load_3d(dst, &maps.a[l], 0, 0, q * nn, &stage_full[s]);
        tc::tma_load_4d(dst + kRwRowFloats, &maps.b[l], 0, e, 0, q * nn, &stage_full[s]);
      }
    }
    if (fail && lane == 0)   // let the copies already issued land
      for (int k = 1; k <= kRwStages && g - k >= 0; ++k)
        tc::bar_wait(&stage_full[(g - k) % kRwStages], ((g - k) / kRwStages) & 1, kTcDrainNs);
    __syncwarp();
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      constexpr uint32_t idesc = tc::idesc_tf32(kTcC, kTcC);
      constexpr uint32_t kLbo = kTcC * 16, kSbo = 128;   // K group (4 rows), 8-channel group
      int g = 0, h = -1, run = 0, pl = -1, pe = -1;
      for (int ch = c_begin; ch < c_end && !fail; ++ch, ++g) {
        int l, e, q;
        wg_chunk(geo, ch, l, e, q);
        const bool fresh = (l != pl || e != pe || run == kRwSeg);
        if (fresh) {
          if (h >= 0) tc::commit(&acc_full[h & 1]);   // the previous segment is complete
          ++h;
          run = 0;
          pl = l;
          pe = e;
          if (h >= 2 && !tc::bar_wait(&acc_free[h & 1], ((h - 2) >> 1) & 1, lim)) {
            fail = true;
            break;
          }
          tc::fence_after_sync();
        }
        const int bb = g % kRwBufs;
        if (!tc::bar_wait(&cvt_full[bb], (g / kRwBufs) & 1, lim)) {
          fail = true;
          break;
        }
        tc::fence_after_sync();
        const uint32_t d_tmem = tmem + (uint32_t)(h & 1) * kTcC;
        const uint32_t a_hi = tmem + kRwACol + (uint32_t)bb * 2 * kTcChunk;
        const uint32_t bh = tc::smem_addr(cv + bb * kRwCvtFloats);
        const uint32_t bl = bh + kTcBlockFloats * sizeof(float);
#pragma unroll
        for (int j = 0; j < kTcChunk / 8; ++j) {
          const uint32_t kx = 2 * j * kLbo;
          const uint64_t dbh = tc::smem_desc(bh + kx, kLbo, kSbo);
          const uint64_t dbl = tc::smem_desc(bl + kx, kLbo, kSbo);
          tc::mma_tf32_ts(d_tmem, a_hi + 8 * j, dbh, idesc, (run | j) != 0);
          tc::mma_tf32_ts(d_tmem, a_hi + kTcChunk + 8 * j, dbh, idesc, 1u);
          tc::mma_tf32_ts(d_tmem, a_hi + 8 * j, dbl, idesc, 1u);
        }
        tc::commit(&cvt_free[bb]);
        ++run;
      }
      if (!fail && h >= 0) tc::commit(&acc_full[h & 1]);   // the last segment
      // every MMA issued above has finished (also after a wait gave up)
      // before the CTA releases TMEM and its shared memory
      tc::commit(drain);
      if (!tc::bar_wait(drain, 0, kTcDrainNs)) fail = true;
    }
    __syncwarp();
  } else if (warp < 10) {
    // ---------------- converters: FP32 rows -> TF32 hi / lo ----------------
    // Warps 4-7 take operand a: lane i of warp w converts channel
    // 32 (w % 4) + i (its TMEM lane) and writes its 32 rows to 32 columns.
    // Warps 2, 3, 8, 9 take operand b: thread t converts channel t and
    // writes 4 rows per 16-byte store into the K-major blocks (a warp fills
    // 512 contiguous bytes).
    const bool op_a = warp >= 4 && warp < 8;
    const int quarter = warp & 3;
    const int chn = op_a ? 32 * quarter + lane : 32 * (warp < 4 ? warp - 2 : warp - 6) + lane;
    const uint32_t src0 = tc::smem_addr(st) + 4u * (uint32_t)((op_a ? 0 : kRwRowFloats) + chn);
    const uint32_t dstb = tc::smem_addr(cv) + 4u * (uint32_t)tc::core_offset(chn, 0, kTcC);
    const uint32_t dsta = tmem + ((uint32_t)(32 * quarter) << 16) + kRwACol;
    int g = 0;
    for (int ch = c_begin; ch < c_end && !fail; ++ch, ++g) {
      int l, e, q;
      wg_chunk(geo, ch, l, e, q);
      const int kv = wg_nodes(l) * (2 * l + 1);   // stage rows the loads wrote
      const int s = g % kRwStages, bb = g % kRwBufs;
      if (!tc::bar_wait(&stage_full[s], (g / kRwStages) & 1, lim)) {
        fail = true;
        break;
      }
      const uint32_t src = src0 + 4u * s * kRwStageFloats;
      float v[kTcChunk];
#pragma unroll
      for (int r = 0; r < kTcChunk; ++r)
        asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v[r]) : "r"(src + 4u * r * kTcC) : "memory");
#pragma unroll
      for (int r = 0; r < kTcChunk; ++r)
        if (r >= kv) v[r] = 0.0f;
      __syncwarp();   // the stage's values are in registers: release it
      if (lane == 0) tc::bar_arrive(&stage_free[s]);
      if (g >= kRwBufs && !tc::bar_wait(&cvt_free[bb], ((g / kRwBufs) - 1) & 1, lim)) {
        fail = true;
        break;
      }
      if (op_a) {
        tc::fence_after_sync();
        uint32_t hi[kTcChunk], lo[kTcChunk];
#pragma unroll
        for (int r = 0; r < kTcChunk; ++r) tc::split_tf32(v[r], hi[r], lo[r]);
        const uint32_t ta = dsta + (uint32_t)bb * 2 * kTcChunk;
        tc::tmem_st32(ta, hi);
        tc::tmem_st32(ta + kTcChunk, lo);
        tc::tmem_wait_st();
        tc::fence_before_sync();
      } else {
        const uint32_t d = dstb + 4u * bb * kRwCvtFloats;
#pragma unroll
        for (int m = 0; m < kTcChunk / 4; ++m) {
          uint4 hv, lv;
          split4(make_float4(v[4 * m], v[4 * m + 1], v[4 * m + 2], v[4 * m + 3]), hv, lv);
          const uint32_t o = d + 4u * (m * (kTcC / 8) * 32);   // K group m
          asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(o), "r"(hv.x), "r"(hv.y), "r"(hv.z),
                       "r"(hv.w) : "memory");
          asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(o + 4u * kTcBlockFloats), "r"(lv.x),
                       "r"(lv.y), "r"(lv.z), "r"(lv.w) : "memory");
        }
        tc::fence_proxy_async();   // the generic-proxy writes, visible to the MMAs
      }
      __syncwarp();
      if (lane == 0) tc::bar_arrive(&cvt_full[bb]);
    }
  } else {
    // ---------------- drain: D[j][k] -> Wb_l[j][e 128 + k] ----------------
    const int ew = warp & 3;        // the TMEM lane quarter this warp may read
    const int j = 32 * ew + lane;   // output row
    int h = -1, run = 0, pl = -1, pe = -1;
    for (int ch = c_begin; ch <= c_end && !fail; ++ch) {
      int l = -1, e = -1, q = 0;
      if (ch < c_end) wg_chunk(geo, ch, l, e, q);
      const bool fresh = ch == c_end || l != pl || e != pe || run == kRwSeg;
      if (fresh && h >= 0) {   // segment h (rank pl, map pe) is complete: add it
        if (!tc::bar_wait(&acc_full[h & 1], (h >> 1) & 1, lim)) {
          fail = true;
          break;
        }
        tc::fence_after_sync();
        float* Wr = Wb + wg_wo(geo, pl) + (size_t)j * (wg_pe(geo, pl) * kTcC) + pe * kTcC;
#pragma unroll 1
        for (int c = 0; c < kTcC / 32; ++c) {
          float v[32];
          tc::tmem_ld32(tmem + (uint32_t)(h & 1) * kTcC + ((uint32_t)(32 * ew) << 16) + 32 * c, v);
#pragma unroll
          for (int u = 0; u < 8; ++u)
            red_add4(Wr + 32 * c + 4 * u, make_float4(v[4 * u], v[4 * u + 1], v[4 * u + 2], v[4 * u + 3]));
        }
        tc::fence_before_sync();
        tc::bar_arrive(&acc_free[h & 1]);
      }
      if (ch == c_end) break;
      if (fresh) {
        ++h;
        run = 0;
        pl = l;
        pe = e;
      }
      ++run;
    }
  }
  if (fail) atomicExch(&g_tc_error, 1);
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, kRwTmemCols);
  }
}

DeviceFlags g_rw_smem_set;
DeviceFlags g_tc_smem_set;
DeviceFlags g_pm_smem_set;

}  // namespace

bool mix_tc_supported(int L, int C) { return C == kTcC && L >= 0 && L <= 6; }

MixTiles mix_tc_tiles(int L, int N) {
  const Geom g = make_geom(L, N);
  MixTiles m{};
  m.ts[0] = 0;
  m.ts[1] = g.t1; m.ts[2] = g.t2; m.ts[3] = g.t3; m.ts[4] = g.t4;
  m.ts[5] = g.t5; m.ts[6] = g.t6; m.ts[7] = g.t7;
  m.total = tile_count(g);
  return m;
}

size_t mix_tc_operand_floats(int L, int N) {
  return (size_t)mix_tc_tiles(L, N).total * kTcTileFloats;
}

size_t mix_tc_matrix_floats(int L) { return (size_t)(L + 1) * 2 * kTcWFloats; }

int launch_mix_tc_split_rows(int L, int N, const float* in, float* xs, cudaStream_t s) {
  const Geom g = make_geom(L, N);
  const int T = tile_count(g);
  if (T == 0) return FC_OK;
  ladder_split_rows_kernel<<<dim3(T, kTcChunks), 256, 0, s>>>(g, in, xs);
  return cudaGetLastError() == cudaSuccess ? FC_OK : FC_ERR_CUDA;
}

int launch_mix_tc_split_matrix(int mode, int L, const float* M, float* ws, cudaStream_t s) {
  const dim3 grid(kTcWFloats / 4 / 256, L + 1);
  if (mode == 0)
    ladder_split_mix_kernel<0><<<grid, 256, 0, s>>>(M, ws);
  else
    ladder_split_mix_kernel<1><<<grid, 256, 0, s>>>(M, ws);
  return cudaGetLastError() == cudaSuccess ? FC_OK : FC_ERR_CUDA;
}

int launch_mix_tc(int L, int N, const float* xs, const float* ws, float* out, cudaStream_t s) {
  if (!mix_tc_supported(L, kTcC)) return FC_ERR_UNSUPPORTED_RANK;
  if (set_smem_once(g_tc_smem_set, ladder_mix_tc_kernel, kTcSmemBytes) != FC_OK) return FC_ERR_CUDA;
  const Geom g = make_geom(L, N);
  const int T = tile_count(g);
  if (T == 0) return FC_OK;
  const int sms = device_sm_count();
  const int grid = T < sms ? T : sms;
  ladder_mix_tc_kernel<<<grid, kTcThreads, kTcSmemBytes, s>>>(g, xs, ws, out);
  return cudaGetLastError() == cudaSuccess ? FC_OK : FC_ERR_CUDA;
}

PathGeom path_geom(int L, int N, const int* kc) {
  PathGeom g{};
  g.N = N;
  g.NY = (L + 1) * (L + 1);
  g.L = L;
  g.nb = (N + kTcRows - 1) / kTcRows;
  int ts[6] = {0, 0, 0, 0, 0, 0}, k[5] = {0, 0, 0, 0, 0};
  int T = 0;
  for (int l = 0; l <= 5; ++l) {
    ts[l] = T;
    if (l <= L && l < 5) {
      T += (2 * l + 1) * g.nb;
      k[l] = kc[l];
    }
  }
  g.t1 = ts[1]; g.t2 = ts[2]; g.t3 = ts[3]; g.t4 = ts[4]; g.t5 = ts[5];
  g.k0 = k[0]; g.k1 = k[1]; g.k2 = k[2]; g.k3 = k[3]; g.k4 = k[4];
  g.e0 = g.e1 = g.e2 = g.e3 = g.e4 = 1;
  g.orow = g.NY;
  return g;
}

PathGeom path_geom_maps(int L, int N, const int* kc, const int* pe) {
  PathGeom g = path_geom(L, N, kc);
  int e[5] = {0, 0, 0, 0, 0};
  for (int l = 0; l <= L && l < 5; ++l) e[l] = pe[l];
  g.e0 = e[0]; g.e1 = e[1]; g.e2 = e[2]; g.e3 = e[3]; g.e4 = e[4];
  g.orow = 0;
  for (int l = 0; l <= L && l < 5; ++l) g.orow += (2 * l + 1) * e[l];
  return g;
}

int launch_path_split_rows(const PathGeom& g, const float* in, float* xs, cudaStream_t s) {
  for (int l = 0; l <= g.L; ++l)
    if (pg_kc(g, l) != pg_kc(g, 0) || (pg_kc(g, l) != 4 && pg_kc(g, l) != 8)) return FC_ERR_ARG;
  const int T = pg_ts(g, g.L + 1);
  if (T == 0) return FC_OK;
  path_split_rows_kernel<<<dim3(T, pg_kc(g, 0)), 256, 0, s>>>(g, in, xs);
  return cudaGetLastError() == cudaSuccess ? FC_OK : FC_ERR_CUDA;
}

int launch_path_split_map(const PathGeom& g, const float* W, float* ws, cudaStream_t s) {
  int kmax = 0, emax = 0;
  for (int l = 0; l <= g.L; ++l) {
    kmax = pg_kc(g, l) > kmax ? pg_kc(g, l) : kmax;
    emax = pg_pe(g, l) > emax ? pg_pe(g, l) : emax;
  }
  if (kmax == 0 || emax == 0) return FC_OK;
  path_split_map_kernel<<<dim3(kmax, g.L + 1, emax), 256, 0, s>>>(g, W, ws);
  return cudaGetLastError() == cudaSuccess ? FC_OK : FC_ERR_CUDA;
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (CUDA
// 12.0 ABI), looked up once.
static PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static std::atomic<void*> fn{nullptr};
  void* f = fn.load(std::memory_order_acquire);
  if (!f) {
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &f, 12000, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess || !f)
      return nullptr;
    fn.store(f, std::memory_order_release);
  }
  return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
}

// FP32 row tensor with `rank` dimensions: 128 channels (contiguous), then
// dims[1..] with byte strides strides[0..]; box 128 x box[1..].
static bool encode_rows(PFN_cuTensorMapEncodeTiled_v12000 enc, CUtensorMap* m, const float* base, int rank,
                        const cuuint64_t* dims, const cuuint64_t* strides, const cuuint32_t* box) {
  const cuuint32_t es[4] = {1, 1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, (cuuint32_t)rank, const_cast<float*>(base), dims, strides, box,
             es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int launch_rows_wgrad_tc(const WgGeom& g, const float* a, const float* b, float* Wb, cudaStream_t s) {
  if (g.L < 0 || g.L > 4 || g.N < 0) return FC_ERR_UNSUPPORTED_RANK;
  long long total = 0;
  for (int l = 0; l <= g.L; ++l) total += (long long)wg_pe(g, l) * wg_chunks(g, l);
  if (total == 0) return FC_OK;
  if (set_smem_once(g_rw_smem_set, rows_wgrad_tc_kernel, kRwSmemBytes) != FC_OK) return FC_ERR_CUDA;
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (!enc) return FC_ERR_CUDA;
  WgMaps maps;
  memset(&maps, 0, sizeof(maps));
  const cuuint64_t row = kTcC * sizeof(float);   // bytes per row
  for (int l = 0; l <= g.L; ++l) {
    const int pe = wg_pe(g, l), w = 2 * l + 1;
    if (pe == 0) continue;
    const cuuint64_t da[3] = {(cuuint64_t)kTcC, (cuuint64_t)w, (cuuint64_t)g.N};
    const cuuint64_t sa[2] = {row, (cuuint64_t)g.sa * row};
    const cuuint32_t ba[3] = {(cuuint32_t)kTcC, (cuuint32_t)w, (cuuint32_t)wg_nodes(l)};
    const cuuint64_t db[4] = {(cuuint64_t)kTcC, (cuuint64_t)pe, (cuuint64_t)w, (cuuint64_t)g.N};
    const cuuint64_t sb[3] = {row, (cuuint64_t)pe * row, (cuuint64_t)g.sb * row};
    const cuuint32_t bb[4] = {(cuuint32_t)kTcC, 1u, (cuuint32_t)w, (cuuint32_t)wg_nodes(l)};
    if (!encode_rows(enc, &maps.a[l], a + (size_t)l * l * kTcC, 3, da, sa, ba) ||
        !encode_rows(enc, &maps.b[l], b + (size_t)wg_ob(g, l) * kTcC, 4, db, sb, bb))
      return FC_ERR_CUDA;
  }
  const int sms = device_sm_count();
  const int grid = total < sms ? (int)total : sms;
  rows_wgrad_tc_kernel<<<grid, kRwThreads, kRwSmemBytes, s>>>(g, maps, Wb);
  return cudaGetLastError() == cudaSuccess ? FC_OK : FC_ERR_CUDA;
}

int launch_path_split_map_t(const PathGeom& g, const float* Wq, float* ws, cudaStream_t s) {
  int emax = 0, kmax = 0;
  for (int l = 0; l <= g.L; ++l) {
    if (pg_kc(g, l) != 4 && pg_kc(g, l) != 8) return FC_ERR_ARG;
    emax = pg_pe(g, l) > emax ? pg_pe(g, l) : emax;
    kmax = pg_kc(g, l) > kmax ? pg_kc(g, l) : kmax;
  }
  if (emax == 0) return FC_OK;
  path_split_map_t_kernel<<<dim3(kmax, emax, g.L + 1), 256, 0, s>>>(g, Wq, ws);
  return cudaGetLastError() == cudaSuccess ? FC_OK : FC_ERR_CUDA;
}

int launch_path_mix_tc(const PathGeom& g, const float* xs, const float* ws, float* out, cudaStream_t s) {
  if (g.L < 0 || g.L > 4) return FC_ERR_UNSUPPORTED_RANK;
  if (set_smem_once(g_pm_smem_set, path_mix_tc_kernel, kPmSmemBytes) != FC_OK) return FC_ERR_CUDA;
  int T = 0;   // units of work
  for (int l = 0; l <= g.L; ++l) T += pg_units(g, l);
  if (T == 0) return FC_OK;
  const int sms = device_sm_count();
  const int grid = T < sms ? T : sms;
  path_mix_tc_kernel<<<grid, kPmThreads, kPmSmemBytes, s>>>(g, xs, ws, out);
  return cudaGetLastError() == cudaSuccess ? FC_OK : FC_ERR_CUDA;
}

}  // namespace fc

extern "C" int fc_device_error(int* flag, fc_stream_t stream) {
  if (!flag) return FC_ERR_ARG;
  cudaStream_t s = (cudaStream_t)stream;
  int h = 0;
  if (cudaMemcpyFromSymbolAsync(&h, fc::g_tc_error, sizeof(int), 0, cudaMemcpyDeviceToHost, s) !=
          cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return FC_ERR_CUDA;
  *flag = h;
  if (h) {
    const int zero = 0;
    if (cudaMemcpyToSymbolAsync(fc::g_tc_error, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, s) !=
            cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
      return FC_ERR_CUDA;
  }
  return FC_OK;
}

extern "C" int fc_set_wait_timeout(uint64_t ns) {
  const unsigned long long v = ns ? (unsigned long long)ns : fc::kTcDefaultWaitNs;
  if (cudaMemcpyToSymbol(fc::g_tc_wait_ns, &v, sizeof(v)) != cudaSuccess) return FC_ERR_CUDA;
  return FC_OK;
}
