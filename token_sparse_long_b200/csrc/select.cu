// Threshold / top-k block selection and stream compaction.
// Jenga notes §4.2 (layer-specific threshold, Algorithm 1) / Jenga summary §4.2.3:
// a token block is kept when its score clears the layer threshold; Algorithm 1
// initialises the threshold to the layer's average block score.
//
// Small nb (<= 8192, the per-layer case: nb = S / blk): one CTA per sequence,
// scores staged in shared memory, warp-ballot + prefix-sum compaction.
// Large nb: multi-CTA mark / emit (scores read once; the mean for MEAN_GE takes one more
// read before it).
#include <cmath>

#include "common.cuh"

namespace jenga {

constexpr int SEL_SMALL_MAX = 8192;
constexpr int SEL_THREADS = 1024;
constexpr int SEL_TILE = 4096;  // scores per CTA in the large-nb path
constexpr int SEL_PER = SEL_TILE / 256;  // 16 consecutive scores per thread

__device__ __forceinline__ float clean_score(float v) { return isnan(v) ? -INFINITY : v; }

// Deterministic float64 sum of n values held in shared memory by one warp:
// lane l sums a contiguous chunk in index order, then a fixed butterfly.
__device__ double warp_sum_f64(const float* s, int n, int lane) {
  int chunk = (n + 31) / 32;
  int lo = lane * chunk, hi = min(n, lo + chunk);
  double acc = 0.0;
  for (int i = lo; i < hi; ++i) acc += (double)s[i];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  return acc;
}

// mode: 0 mean_ge, 1/3 top-k (k given), 2 abs_ge
__global__ void __launch_bounds__(SEL_THREADS) select_small_kernel(const float* __restrict__ scores, int nb,
                                                                   int mode, float thr, int k,
                                                                   int32_t* __restrict__ idx,
                                                                   int32_t* __restrict__ n_kept,
                                                                   uint8_t* __restrict__ mask) {
  extern __shared__ float s_sc[];  // nb floats
  __shared__ double s_mean;
  __shared__ int s_warp[SEL_THREADS / 32];
  __shared__ int s_base;
  __shared__ int s_chunk;
  const int b = blockIdx.x;
  const float* sc = scores + (int64_t)b * nb;
  for (int i = threadIdx.x; i < nb; i += blockDim.x) s_sc[i] = clean_score(sc[i]);
  __syncthreads();
  if (mode == 0) {
    if (threadIdx.x < 32) {
      double t = warp_sum_f64(s_sc, nb, threadIdx.x);
      if (threadIdx.x == 0) s_mean = t / (double)nb;
    }
    __syncthreads();
  }
  const double mean = (mode == 0) ? s_mean : 0.0;
  if (threadIdx.x == 0) s_base = 0;
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int c0 = 0; c0 < nb; c0 += SEL_THREADS) {
    int n = c0 + threadIdx.x;
    bool keep = false;
    if (n < nb) {
      float v = s_sc[n];
      if (mode == 0) {
        keep = (double)v >= mean;
      } else if (mode == 2) {
        keep = v >= thr;
      } else {
        int rank = 0;
        for (int m = 0; m < nb; ++m) {
          float u = s_sc[m];
          rank += (u > v) || (u == v && m < n);
        }
        keep = rank < k;
      }
      if (mask) mask[(int64_t)b * nb + n] = keep ? 1 : 0;
    }
    unsigned bal = __ballot_sync(0xffffffffu, keep);
    if (lane == 0) s_warp[warp] = __popc(bal);
    __syncthreads();
    if (warp == 0) {  // exclusive scan over the 32 warp counts
      int v = s_warp[lane];
      int incl = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        int t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
      }
      s_warp[lane] = incl - v;
      if (lane == 31) s_chunk = incl;
    }
    __syncthreads();
    int pos = s_base + s_warp[warp] + __popc(bal & ((1u << lane) - 1));
    if (keep) idx[(int64_t)b * nb + pos] = n;
    __syncthreads();
    if (threadIdx.x == 0) s_base += s_chunk;
    __syncthreads();
  }
  const int total = s_base;
  for (int i = total + threadIdx.x; i < nb; i += blockDim.x) idx[(int64_t)b * nb + i] = -1;
  if (threadIdx.x == 0) n_kept[b] = total;
}

// SEL_PER consecutive scores of one thread (-inf past nb): 16-byte loads when aligned
__device__ __forceinline__ void sel_load16(const float* sc, int nb, int lo, float* v) {
  if (lo + SEL_PER <= nb && (((uintptr_t)(sc + lo)) & 15) == 0) {
#pragma unroll
    for (int q = 0; q < SEL_PER / 4; ++q) {
      const float4 f = __ldg(reinterpret_cast<const float4*>(sc + lo) + q);
      v[4 * q] = f.x;
      v[4 * q + 1] = f.y;
      v[4 * q + 2] = f.z;
      v[4 * q + 3] = f.w;
    }
  } else {
#pragma unroll
    for (int e = 0; e < SEL_PER; ++e) v[e] = (lo + e < nb) ? sc[lo + e] : -INFINITY;
  }
}

// ---- large nb: pass A (optional) fp64 partial sums per tile
__global__ void __launch_bounds__(256) sel_partial_sum_kernel(const float* __restrict__ scores, int nb,
                                                              double* __restrict__ part, int ntiles) {
  const int b = blockIdx.y, t = blockIdx.x;
  const float* sc = scores + (int64_t)b * nb;
  __shared__ double s_w[8];
  int lo = t * SEL_TILE, hi = min(nb, lo + SEL_TILE);
  // each thread sums a contiguous run of 16 in index order, then a fixed tree
  double acc = 0.0;
  const int r0 = lo + threadIdx.x * (SEL_TILE / 256);
  float v[SEL_TILE / 256];
  sel_load16(sc, nb, r0, v);
#pragma unroll
  for (int e = 0; e < SEL_TILE / 256; ++e)
    if (r0 + e < hi) acc += (double)clean_score(v[e]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if ((threadIdx.x & 31) == 0) s_w[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    double s = 0.0;
    for (int w = 0; w < 8; ++w) s += s_w[w];
    part[(int64_t)b * ntiles + t] = s;
  }
}

// pass A2: the mean from the tile partials, fixed order (one CTA per sequence)
__global__ void __launch_bounds__(1024) sel_mean_kernel(const double* __restrict__ part, int ntiles, int nb,
                                                        double* __restrict__ mean) {
  const int b = blockIdx.x;
  __shared__ double s_w[32];
  int chunk = (ntiles + 1023) / 1024;
  int lo = threadIdx.x * chunk, hi = min(ntiles, lo + chunk);
  double acc = 0.0;
  for (int i = lo; i < hi; ++i) acc += part[(int64_t)b * ntiles + i];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if ((threadIdx.x & 31) == 0) s_w[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    double t = 0.0;
    for (int w = 0; w < 32; ++w) t += s_w[w];
    mean[b] = t / (double)nb;
  }
}

// ---- large nb: mark, then emit.  Mark reads the scores once and writes the mask bytes, a
// packed keep bitmask and each tile's keep count (also added into its superblock's sum, a
// superblock being ~sqrt(ntiles) tiles); emit finds its tile's offset from the superblock
// sums before it and its superblock's earlier counts, reads only the bitmask (1 bit per
// score) and writes the kept indices plus the -1 fill of its own position range.  Traffic
// is 4 + 1 + 1/8 + 1/8 + 4 bytes per score against the 4 + 1 + 4 the output needs; no CTA
// waits for another.  A tile is SEL_TILE scores, SEL_PER consecutive per thread.
__global__ void __launch_bounds__(256) sel_mark_kernel(const float* __restrict__ scores, int nb, int mode,
                                                       float thr, const double* __restrict__ means, int ntiles,
                                                       int sb_tiles, int nsb, int* __restrict__ counts,
                                                       int* __restrict__ sb_sum, uint32_t* __restrict__ bits,
                                                       uint8_t* __restrict__ mask) {
  const int b = blockIdx.y, t = blockIdx.x;
  const float* sc = scores + (int64_t)b * nb;
  const double mean = (mode == 0) ? means[b] : 0.0;
  const int lo = t * SEL_TILE + threadIdx.x * SEL_PER;
  float v[SEL_PER];
  sel_load16(sc, nb, lo, v);
  uint32_t keep = 0;
#pragma unroll
  for (int e = 0; e < SEL_PER; ++e) {
    const float x = clean_score(v[e]);
    const bool k = (lo + e < nb) && ((mode == 0) ? ((double)x >= mean) : (x >= thr));
    keep |= (uint32_t)k << e;
  }
  bits[((int64_t)b * ntiles + t) * 256 + threadIdx.x] = keep;
  if (mask) {
    uint8_t* mrow = mask + (int64_t)b * nb;
    if (lo + SEL_PER <= nb && ((((uintptr_t)mrow) + lo) & 15) == 0) {
#pragma unroll
      for (int h = 0; h < SEL_PER / 16; ++h) {
        uint32_t w4[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint32_t w = 0;
#pragma unroll
          for (int e = 0; e < 4; ++e) w |= ((keep >> (16 * h + 4 * q + e)) & 1u) << (8 * e);
          w4[q] = w;
        }
        *reinterpret_cast<uint4*>(mrow + lo + 16 * h) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
      }
    } else {
      for (int e = 0; e < SEL_PER; ++e)
        if (lo + e < nb) mrow[lo + e] = (uint8_t)((keep >> e) & 1u);
    }
  }
  int c = __popc(keep);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
  __shared__ int s_w[8];
  if ((threadIdx.x & 31) == 0) s_w[threadIdx.x >> 5] = c;
  __syncthreads();
  if (threadIdx.x == 0) {
    int tot = 0;
#pragma unroll
    for (int w = 0; w < 8; ++w) tot += s_w[w];
    counts[(int64_t)b * ntiles + t] = tot;
    atomicAdd(&sb_sum[(int64_t)b * nsb + t / sb_tiles], tot);
  }
}

// 288 threads: warps 0..7 rank and stage the tile's kept scores while warp 8 sums the
// superblock and tile counts before it (the tile's output offset) and all of them (n_kept)
__global__ void __launch_bounds__(288) sel_emit_kernel(int nb, int ntiles, int sb_tiles, int nsb,
                                                       const uint32_t* __restrict__ bits,
                                                       const int* __restrict__ counts, const int* __restrict__ sb_sum,
                                                       int32_t* __restrict__ n_kept, int32_t* __restrict__ idx) {
  const int b = blockIdx.y, t = blockIdx.x;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  __shared__ int s_w[8];
  __shared__ int s_base, s_nk;
  __shared__ int s_out[SEL_TILE];
  uint32_t keep = 0;
  int cnt = 0, incl = 0;
  if (warp == 8) {
    // all counts are final here: the mark kernel completed
    const int sb = t / sb_tiles;
    const int* sbb = sb_sum + (int64_t)b * nsb;
    int before = 0, all = 0;
    for (int i = lane; i < nsb; i += 32) {
      const int x = sbb[i];
      all += x;
      before += (i < sb) ? x : 0;
    }
    for (int i = sb * sb_tiles + lane; i < t; i += 32) before += counts[(int64_t)b * ntiles + i];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      before += __shfl_xor_sync(0xffffffffu, before, o);
      all += __shfl_xor_sync(0xffffffffu, all, o);
    }
    if (lane == 0) {
      s_base = before;
      s_nk = all;
      if (t == 0) n_kept[b] = all;
    }
  } else {
    keep = bits[((int64_t)b * ntiles + t) * 256 + threadIdx.x];  // SEL_PER consecutive scores
    cnt = __popc(keep);
    incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == 31) s_w[warp] = incl;
  }
  __syncthreads();
  int wbase = 0, agg = 0;
#pragma unroll
  for (int w = 0; w < 8; ++w) {
    wbase += (w < warp) ? s_w[w] : 0;
    agg += s_w[w];
  }
  if (warp < 8) {
    const int lo = t * SEL_TILE + threadIdx.x * SEL_PER;
    int r = wbase + incl - cnt;
#pragma unroll
    for (int e = 0; e < SEL_PER; ++e)
      if ((keep >> e) & 1u) s_out[r++] = lo + e;
  }
  __syncthreads();
  if (warp == 8) return;
  int32_t* orow = idx + (int64_t)b * nb;
  const int base = s_base;
  // kept indices to [base, base + agg): scalar up to a 16-byte boundary, then int4
  const int head = min(agg, (int)((4 - (((uintptr_t)(orow + base) >> 2) & 3)) & 3));
  if (threadIdx.x < head) orow[base + threadIdx.x] = s_out[threadIdx.x];
  const int nvec = (agg - head) >> 2;
  int4* ov = reinterpret_cast<int4*>(orow + base + head);
  for (int i = threadIdx.x; i < nvec; i += 256) {
    const int j = head + 4 * i;
    ov[i] = make_int4(s_out[j], s_out[j + 1], s_out[j + 2], s_out[j + 3]);
  }
  for (int i = head + 4 * nvec + threadIdx.x; i < agg; i += 256) orow[base + i] = s_out[i];
  // -1 on this tile's position range past n_kept (every position is written exactly once)
  const int nk = s_nk;
  const int p0 = max(t * SEL_TILE, nk), p1 = min(nb, (t + 1) * SEL_TILE);
  if (p0 < p1) {
    const int fh = min(p1 - p0, (int)((4 - (((uintptr_t)(orow + p0) >> 2) & 3)) & 3));
    if (threadIdx.x < fh) orow[p0 + threadIdx.x] = -1;
    const int fv = (p1 - p0 - fh) >> 2;
    int4* fvp = reinterpret_cast<int4*>(orow + p0 + fh);
    for (int i = threadIdx.x; i < fv; i += 256) fvp[i] = make_int4(-1, -1, -1, -1);
    for (int p = p0 + fh + 4 * fv + threadIdx.x; p < p1; p += 256) orow[p] = -1;
  }
}

static int topk_count(float p, int nb) {
  double k = std::ceil((double)p * nb - 1e-6);
  if (k < 0) k = 0;
  if (k > nb) k = nb;
  return (int)k;
}

}  // namespace jenga

using namespace jenga;

static int sel_sb_tiles(int ntiles) {
  int sbt = 64;
  while ((long long)sbt * sbt < ntiles) sbt *= 2;
  return sbt;
}

extern "C" size_t jenga_select_workspace_bytes(int B, int nb) {
  if (B < 1 || nb <= SEL_SMALL_MAX) return 0;
  const int ntiles = (nb + SEL_TILE - 1) / SEL_TILE;
  const int nsb = (ntiles + sel_sb_tiles(ntiles) - 1) / sel_sb_tiles(ntiles);
  // tile partial sums (mean), keep bitmask, tile counts, superblock sums, means
  return (size_t)B * ntiles * (sizeof(double) + 256 * sizeof(uint32_t) + sizeof(int)) + (size_t)B * nsb * sizeof(int) +
         (size_t)B * sizeof(double) + 256;
}

extern "C" jenga_status jenga_select(const float* scores, int B, int nb, jenga_select_mode mode, float param,
                                     int32_t* idx, int32_t* n_kept, uint8_t* mask, void* ws, size_t ws_bytes,
                                     jenga_stream_t stream) {
  JENGA_CHECK_ARG(scores && idx && n_kept, "jenga_select: null pointer");
  JENGA_CHECK_ARG(B >= 1 && nb >= 1, "jenga_select: bad sizes B=%d nb=%d", B, nb);
  JENGA_CHECK_ARG(mode >= JENGA_SELECT_MEAN_GE && mode <= JENGA_SELECT_TOPK, "jenga_select: bad mode %d", (int)mode);
  cudaStream_t st = (cudaStream_t)stream;
  int k = 0;
  int kmode = 0;
  if (mode == JENGA_SELECT_MEAN_GE) kmode = 0;
  if (mode == JENGA_SELECT_ABS_GE) kmode = 2;
  if (mode == JENGA_SELECT_TOPK_FRAC) { kmode = 1; k = topk_count(param, nb); }
  if (mode == JENGA_SELECT_TOPK) {
    kmode = 1;
    JENGA_CHECK_ARG(param >= 0 && param <= (float)nb && param == std::floor(param), "jenga_select: k=%g", param);
    k = (int)param;
  }
  if (nb <= SEL_SMALL_MAX) {
    size_t smem = (size_t)nb * sizeof(float);
    if (smem > 48 * 1024)
      JENGA_CUDA_TRY(cudaFuncSetAttribute(select_small_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          (int)smem));
    {
    const int _ps = ::jenga::prof_begin("select_small", st);
    select_small_kernel<<<B, SEL_THREADS, smem, st>>>(scores, nb, kmode, param, k, idx, n_kept, mask);
    ::jenga::prof_end(_ps, st);
    }
    JENGA_LAUNCH_CHECK();
    return JENGA_OK;
  }
  if (kmode == 1) return fail(JENGA_EUNSUPPORTED, "jenga_select: top-k supports nb <= %d", SEL_SMALL_MAX);
  const size_t need = jenga_select_workspace_bytes(B, nb);
  if (!ws || ws_bytes < need) return fail(JENGA_EWORKSPACE, "jenga_select: workspace %zu < %zu", ws_bytes, need);
  const int ntiles = (nb + SEL_TILE - 1) / SEL_TILE;
  JENGA_CHECK_ARG(ntiles <= (1 << 20), "jenga_select: nb too large");
  char* w = (char*)(((uintptr_t)ws + 15) & ~(uintptr_t)15);
  const int sb_tiles = sel_sb_tiles(ntiles);
  const int nsb = (ntiles + sb_tiles - 1) / sb_tiles;
  double* part = (double*)w;
  uint32_t* bits = (uint32_t*)(part + (size_t)B * ntiles);
  int* counts = (int*)(bits + (size_t)B * ntiles * 256);
  int* sb_sum = counts + (size_t)B * ntiles;
  double* means = (double*)(((uintptr_t)(sb_sum + (size_t)B * nsb) + 7) & ~(uintptr_t)7);
  dim3 g(ntiles, B);
  if (kmode == 0) {
    {
    const int _ps = ::jenga::prof_begin("sel_partial_sum", st);
    sel_partial_sum_kernel<<<g, 256, 0, st>>>(scores, nb, part, ntiles);
    ::jenga::prof_end(_ps, st);
    }
    JENGA_LAUNCH_CHECK();
    {
    const int _ps = ::jenga::prof_begin("sel_mean", st);
    sel_mean_kernel<<<B, 1024, 0, st>>>(part, ntiles, nb, means);
    ::jenga::prof_end(_ps, st);
    }
    JENGA_LAUNCH_CHECK();
  }
  JENGA_CUDA_TRY(cudaMemsetAsync(sb_sum, 0, (size_t)B * nsb * sizeof(int), st));
  {
  const int _ps = ::jenga::prof_begin("sel_mark", st);
  sel_mark_kernel<<<g, 256, 0, st>>>(scores, nb, kmode, param, means, ntiles, sb_tiles, nsb, counts, sb_sum, bits,
                                     mask);
  ::jenga::prof_end(_ps, st);
  }
  JENGA_LAUNCH_CHECK();
  {
  const int _ps = ::jenga::prof_begin("sel_emit", st);
  sel_emit_kernel<<<g, 288, 0, st>>>(nb, ntiles, sb_tiles, nsb, bits, counts, sb_sum, n_kept, idx);
  ::jenga::prof_end(_ps, st);
  }
  JENGA_LAUNCH_CHECK();
  return JENGA_OK;
}
