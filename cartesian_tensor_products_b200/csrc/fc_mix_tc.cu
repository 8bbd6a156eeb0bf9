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
// One persistent CTA per SM walks a contiguous range of 128-row tiles (tiles
// never straddle two ranks), warp-specialised:
//  * warps 0-7 (producers) hold the next tile's rows in registers (64 KB per
//    SM in flight, coalesced 64-byte row segments), split them into TF32 hi
//    and lo and write them in the core-matrix layout into one of three
//    shared-memory stages, one K chunk (32 channels) at a time.  The rank's
//    matrix, split likewise, stays in shared memory (128 KB) until the rank
//    changes.  Thread 0 issues the 12 MMAs of a chunk (128 x 128 x 8 each,
//    the matrix as operand A, the rows as operand B) and commits them to the
//    stage's mbarrier, which frees the stage;
//  * warps 8-11 (epilogue) drain the accumulator D[channel][row] from TMEM,
//    two tiles deep (256 columns), so the stores of one tile overlap the
//    MMAs of the next: lane = output channel, so every store of a warp is
//    one 128-byte row segment, and the epilogue issues no loads at all.
// C = 128 only (the tile is the whole channel range); other widths use the
// FP32 SIMT kernels.
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
constexpr int kTcProducers = 256;      // warps 0..7 load, split and issue
constexpr int kTcThreads = 384;        // + warps 8..11 drain the accumulator
constexpr int kTcStageFloats = kTcRows * kTcChunk;   // 4096 (one of hi / lo)
constexpr int kTcWFloats = kTcC * kTcC;              // 16384 (one of hi / lo)
constexpr uint32_t kTcWaitPolls = 1u << 22;
constexpr int kTcBars = kTcStages + 4;               // stage_free[3], acc_full[2], acc_free[2]
constexpr size_t kTcSmemBytes =
    sizeof(float) * (2 * kTcWFloats + 2 * kTcStages * kTcStageFloats) + 8 * kTcBars + 8;
static_assert(kTcSmemBytes <= 232448, "shared memory per CTA");

struct MixTcArgs {
  int N, NY, L;
  const float* in;          // [N][NY][C]
  const float* M;           // [L+1][C][C] of this ladder step
  float* out;               // [N][NY][C]
  int tile_start[8];        // first tile of rank l; tile_start[L+1] = total
};

__device__ int g_tc_error = 0;

__device__ __forceinline__ size_t tc_rank_row(int i, int l, int NY) {
  const int w = 2 * l + 1;
  const int n = i / w;
  return ((size_t)n * NY + l * l + (i - n * w)) * kTcC;
}

__device__ __forceinline__ int tile_rank(const MixTcArgs& a, int t) {
  int l = 0;
  while (l < a.L && t >= a.tile_start[l + 1]) ++l;
  return l;
}

// Producer thread p's share of K chunk c of tile t: 4 float4 at (row r, K group q)
// with r = 16 (p/32) + 8 (it/2) + p%8, q = (p%32)/8 + 4 (it%2).  One warp
// instruction reads 8 rows x 64 contiguous bytes; zeros past the last row.
__device__ __forceinline__ void load_chunk(const MixTcArgs& a, int t, int t_end, int c,
                                           float4 (&v)[4]) {
  if (t >= t_end) return;
  const int p = threadIdx.x, lane = p & 31;
  const int l = tile_rank(a, t);
  const int R = a.N * (2 * l + 1);
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int i = (t - a.tile_start[l]) * kTcRows + 16 * (p >> 5) + 8 * h + (lane & 7);
    if (i < R) {
      const float4* src = reinterpret_cast<const float4*>(a.in + tc_rank_row(i, l, a.NY) + c * kTcChunk);
      v[2 * h] = __ldg(src + (lane >> 3));
      v[2 * h + 1] = __ldg(src + (lane >> 3) + 4);
    } else {
      v[2 * h] = zero4();
      v[2 * h + 1] = zero4();
    }
  }
}

// The same elements into one stage, split into TF32 hi and lo, core-matrix
// layout (eight consecutive threads fill one 128-byte core matrix).
__device__ __forceinline__ void store_chunk(const float4 (&v)[4], float* hi, float* lo) {
  const int p = threadIdx.x, lane = p & 31;
#pragma unroll
  for (int it = 0; it < 4; ++it) {
    const int r = 16 * (p >> 5) + 8 * (it >> 1) + (lane & 7);
    const int q = (lane >> 3) + 4 * (it & 1);
    uint4 h, w;
    tc::split_tf32(v[it].x, h.x, w.x);
    tc::split_tf32(v[it].y, h.y, w.y);
    tc::split_tf32(v[it].z, h.z, w.z);
    tc::split_tf32(v[it].w, h.w, w.w);
    const int off = tc::core_offset(r, 4 * q, kTcRows);
    *reinterpret_cast<uint4*>(hi + off) = h;
    *reinterpret_cast<uint4*>(lo + off) = w;
  }
}

// A operand (row = output channel j, K = input channel t): forward M[j][t],
// VJP M[t][j]; split into hi and lo by the 256 producer threads.
template <int MODE>
__device__ __forceinline__ void load_weights(const float* Ml, float* hi, float* lo) {
  const int p = threadIdx.x;
  const int j = p & (kTcC - 1);
#pragma unroll 4
  for (int it = 0; it < kTcWFloats / 4 / kTcProducers; ++it) {
    const int q = 2 * it + (p >> 7);
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
    tc::split_tf32(v.x, h.x, w.x);
    tc::split_tf32(v.y, h.y, w.y);
    tc::split_tf32(v.z, h.z, w.z);
    tc::split_tf32(v.w, h.w, w.w);
    const int off = tc::core_offset(j, 4 * q, kTcC);
    *reinterpret_cast<uint4*>(hi + off) = h;
    *reinterpret_cast<uint4*>(lo + off) = w;
  }
}

// MODE 0: out[r][j] = sum_t in[r][t] M_l[j][t].
// MODE 1: out[r][j] = sum_t in[r][t] M_l[t][j].
// The accumulator of a tile is D[j][r] (TMEM lane = output channel, column =
// tile row), two tiles deep (256 columns).
template <int MODE>
__global__ void __launch_bounds__(kTcThreads, 1) ladder_mix_tc_kernel(const MixTcArgs a) {
  extern __shared__ __align__(1024) unsigned char smem[];
  float* w_hi = reinterpret_cast<float*>(smem);
  float* w_lo = w_hi + kTcWFloats;
  float* x_hi = w_lo + kTcWFloats;                       // kTcStages stages
  float* x_lo = x_hi + kTcStages * kTcStageFloats;       // kTcStages stages
  uint64_t* stage_free = reinterpret_cast<uint64_t*>(x_lo + kTcStages * kTcStageFloats);
  uint64_t* acc_full = stage_free + kTcStages;
  uint64_t* acc_free = acc_full + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_free + 2);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int T = a.tile_start[a.L + 1];
  const int t_begin = (int)((long long)blockIdx.x * T / gridDim.x);
  const int t_end = (int)((long long)(blockIdx.x + 1) * T / gridDim.x);

  if (warp == 0) tc::tmem_alloc(tmem_slot, 2 * kTcRows);
  if (tid == 0) {
    for (int s = 0; s < kTcStages; ++s) tc::bar_init(&stage_free[s], 1);
    tc::bar_init(&acc_full[0], 1);
    tc::bar_init(&acc_full[1], 1);
    tc::bar_init(&acc_free[0], kTcThreads - kTcProducers);
    tc::bar_init(&acc_free[1], kTcThreads - kTcProducers);
    tc::fence_bar_init();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  bool fail = false;

  if (tid < kTcProducers) {
    // ---------------- producers (and the MMA issuer, thread 0) ----------------
    constexpr uint32_t idesc = tc::idesc_tf32(kTcC, kTcRows);
    constexpr uint32_t kLbo = kTcRows * 16, kSbo = 128;   // both operands are 128-row tiles
    float4 buf[kTcChunks][4];
#pragma unroll
    for (int c = 0; c < kTcChunks; ++c) load_chunk(a, t_begin, t_end, c, buf[c]);
    int cur_l = -1;
    for (int t = t_begin; t < t_end && !fail; ++t) {
      const int ti = t - t_begin;
      const int l = tile_rank(a, t);
      const uint32_t d_tmem = tmem + (uint32_t)(ti & 1) * kTcRows;
      if (l != cur_l) {
        if (ti > 0) {   // every MMA of the previous tile has read the old matrix
          const int gl = kTcChunks * ti - 1;
          if (!tc::bar_wait(&stage_free[gl % kTcStages], (gl / kTcStages) & 1, kTcWaitPolls))
            fail = true;
          if (tc::named_bar_or(1, kTcProducers, fail)) {
            fail = true;
            break;
          }
        }
        load_weights<MODE>(a.M + (size_t)l * kTcC * kTcC, w_hi, w_lo);
        cur_l = l;
      }
#pragma unroll
      for (int c = 0; c < kTcChunks; ++c) {
        const int g = kTcChunks * ti + c;
        const int s = g % kTcStages;
        bool bad = false;
        if (g >= kTcStages &&
            !tc::bar_wait(&stage_free[s], ((g - kTcStages) / kTcStages) & 1, kTcWaitPolls))
          bad = true;
        store_chunk(buf[c], x_hi + s * kTcStageFloats, x_lo + s * kTcStageFloats);
        load_chunk(a, t + 1, t_end, c, buf[c]);
        tc::fence_proxy_async();
        if (tc::named_bar_or(1, kTcProducers, bad || fail)) {
          fail = true;
          break;
        }
        if (tid == 0) {
          // the epilogue has drained this accumulator buffer (tile ti - 2)
          if (c == 0 && ti >= 2 &&
              !tc::bar_wait(&acc_free[ti & 1], ((ti - 2) >> 1) & 1, kTcWaitPolls)) {
            fail = true;
          } else {
            tc::fence_after_sync();
            const uint32_t xh = tc::smem_addr(x_hi + s * kTcStageFloats);
            const uint32_t xl = tc::smem_addr(x_lo + s * kTcStageFloats);
            const uint32_t wh = tc::smem_addr(w_hi), wl = tc::smem_addr(w_lo);
#pragma unroll
            for (int j = 0; j < kTcChunk / 8; ++j) {
              const uint32_t kx = 2 * j * kLbo;                          // K group 2j of the stage
              const uint32_t kw = (c * (kTcChunk / 4) + 2 * j) * kLbo;   // same K group of M
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
      }
    }
  } else {
    // ---------------- epilogue: TMEM -> new state (and z) ----------------
    const int ew = warp - kTcProducers / 32;        // 0..3 = TMEM lane quarter
    const int j = 32 * ew + lane;                    // output channel
    for (int t = t_begin; t < t_end; ++t) {
      const int ti = t - t_begin;
      const int l = tile_rank(a, t);
      const int w = 2 * l + 1;
      const int R = a.N * w;
      const int row0 = (t - a.tile_start[l]) * kTcRows;
      const uint32_t d_tmem = tmem + (uint32_t)(ti & 1) * kTcRows + ((uint32_t)(32 * ew) << 16);
      if (!tc::bar_wait(&acc_full[ti & 1], (ti >> 1) & 1, kTcWaitPolls)) {
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
          if (i0 + r < R) a.out[((size_t)n * a.NY + l * l + cc) * kTcC + j] = v[r];
          if (++cc == w) { cc = 0; ++n; }
        }
      }
      tc::fence_before_sync();
      tc::bar_arrive(&acc_free[ti & 1]);
    }
  }
  if (fail) atomicExch(&g_tc_error, 1);
  // every MMA completed before its tile's accumulator was read; release TMEM
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, 2 * kTcRows);
  }
}

int g_tc_smem_set[64] = {0};
int g_sm_count[64] = {0};

template <int MODE>
int launch_mix_tc_mode(int L, int N, const float* in, const float* M, float* out,
                       cudaStream_t s) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return FC_ERR_CUDA;
  if (!(g_tc_smem_set[dev] & (1 << MODE))) {
    if (cudaFuncSetAttribute(ladder_mix_tc_kernel<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kTcSmemBytes) != cudaSuccess)
      return FC_ERR_CUDA;
    g_tc_smem_set[dev] |= 1 << MODE;
  }
  if (g_sm_count[dev] == 0 &&
      cudaDeviceGetAttribute(&g_sm_count[dev], cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return FC_ERR_CUDA;
  MixTcArgs a{};
  a.N = N;
  a.NY = (L + 1) * (L + 1);
  a.L = L;
  a.in = in;
  a.M = M;
  a.out = out;
  int T = 0;
  for (int l = 0; l <= L; ++l) {
    a.tile_start[l] = T;
    T += (N * (2 * l + 1) + kTcRows - 1) / kTcRows;
  }
  a.tile_start[L + 1] = T;
  if (T == 0) return FC_OK;
  const int grid = T < g_sm_count[dev] ? T : g_sm_count[dev];
  ladder_mix_tc_kernel<MODE><<<grid, kTcThreads, kTcSmemBytes, s>>>(a);
  return cudaGetLastError() == cudaSuccess ? FC_OK : FC_ERR_CUDA;
}

}  // namespace

bool mix_tc_supported(int L, int C) { return C == kTcC && L >= 0 && L <= 6; }

int launch_mix_tc(int mode, int L, int N, const float* in, const float* M, float* out,
                  cudaStream_t s) {
  if (!mix_tc_supported(L, kTcC)) return FC_ERR_UNSUPPORTED_RANK;
  return mode == 0 ? launch_mix_tc_mode<0>(L, N, in, M, out, s)
                   : launch_mix_tc_mode<1>(L, N, in, M, out, s);
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
