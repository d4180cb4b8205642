// Threshold / top-k block selection and stream compaction.
// Jenga notes §4.2 (layer-specific threshold, Algorithm 1) / Jenga summary §4.2.3:
// a token block is kept when its score clears the layer threshold; Algorithm 1
// initialises the threshold to the layer's average block score.
//
// Small nb (<= 8192, the per-layer case: nb = S / blk): one CTA per sequence,
// scores staged in shared memory, warp-ballot + prefix-sum compaction.
// Large nb: multi-CTA two-pass compaction (per-tile counts, one scan, then write).
#include <cmath>

#include "common.cuh"

namespace jenga {

constexpr int SEL_SMALL_MAX = 8192;
constexpr int SEL_THREADS = 1024;
constexpr int SEL_TILE = 4096;  // scores per CTA in the large-nb path

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

// ---- large nb: pass A (optional) fp64 partial sums per tile
__global__ void __launch_bounds__(256) sel_partial_sum_kernel(const float* __restrict__ scores, int nb,
                                                              double* __restrict__ part, int ntiles) {
  const int b = blockIdx.y, t = blockIdx.x;
  const float* sc = scores + (int64_t)b * nb;
  __shared__ double s_w[8];
  int lo = t * SEL_TILE, hi = min(nb, lo + SEL_TILE);
  // each thread sums a contiguous run of 16 in index order, then a fixed tree
  double acc = 0.0;
  int r0 = lo + threadIdx.x * (SEL_TILE / 256);
  for (int i = r0; i < min(hi, r0 + SEL_TILE / 256); ++i) acc += (double)clean_score(sc[i]);
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

// pass B: per-tile keep counts (needs the mean for mode 0)
__global__ void __launch_bounds__(256) sel_count_kernel(const float* __restrict__ scores, int nb, int mode,
                                                        float thr, const double* __restrict__ means, int ntiles,
                                                        int* __restrict__ counts) {
  const int b = blockIdx.y, t = blockIdx.x;
  const float* sc = scores + (int64_t)b * nb;
  const double mean = (mode == 0) ? means[b] : 0.0;
  int lo = t * SEL_TILE, hi = min(nb, lo + SEL_TILE);
  int c = 0;
  for (int i = lo + threadIdx.x; i < hi; i += 256) {
    float v = clean_score(sc[i]);
    c += (mode == 0) ? ((double)v >= mean) : (v >= thr);
  }
  __shared__ int s_c[256];
  s_c[threadIdx.x] = c;
  __syncthreads();
  for (int o = 128; o > 0; o >>= 1) {
    if (threadIdx.x < o) s_c[threadIdx.x] += s_c[threadIdx.x + o];
    __syncthreads();
  }
  if (threadIdx.x == 0) counts[(int64_t)b * ntiles + t] = s_c[0];
}

// pass C: exclusive scan of tile counts (one CTA per sequence)
__global__ void __launch_bounds__(1024) sel_scan_kernel(const int* __restrict__ counts, int ntiles,
                                                        int* __restrict__ offsets, int32_t* __restrict__ n_kept) {
  const int b = blockIdx.x;
  __shared__ int s_carry;
  __shared__ int s_w[32];
  if (threadIdx.x == 0) s_carry = 0;
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int c0 = 0; c0 < ntiles; c0 += 1024) {
    int i = c0 + threadIdx.x;
    int v = i < ntiles ? counts[(int64_t)b * ntiles + i] : 0;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int t = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += t;
    }
    if (lane == 31) s_w[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      int wv = s_w[lane];
      int wi = wv;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        int t = __shfl_up_sync(0xffffffffu, wi, o);
        if (lane >= o) wi += t;
      }
      s_w[lane] = wi - wv;
    }
    __syncthreads();
    int excl = s_carry + s_w[warp] + incl - v;
    if (i < ntiles) offsets[(int64_t)b * ntiles + i] = excl;
    __syncthreads();
    if (threadIdx.x == 1023) s_carry = excl + v;
    __syncthreads();
  }
  if (threadIdx.x == 0) n_kept[b] = s_carry;
}

// pass D: write indices and mask of each tile at its offset; fill -1 past the total
__global__ void __launch_bounds__(256) sel_write_kernel(const float* __restrict__ scores, int nb, int mode,
                                                        float thr, const double* __restrict__ means, int ntiles,
                                                        const int* __restrict__ offsets,
                                                        const int32_t* __restrict__ n_kept,
                                                        int32_t* __restrict__ idx, uint8_t* __restrict__ mask) {
  const int b = blockIdx.y, t = blockIdx.x;
  const float* sc = scores + (int64_t)b * nb;
  const double mean = (mode == 0) ? means[b] : 0.0;
  __shared__ int s_w[8];
  __shared__ int s_carry;
  if (threadIdx.x == 0) s_carry = offsets[(int64_t)b * ntiles + t];
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int lo = t * SEL_TILE, hi = min(nb, lo + SEL_TILE);
  for (int c0 = lo; c0 < hi; c0 += 256) {
    int i = c0 + threadIdx.x;
    bool keep = false;
    if (i < hi) {
      float v = clean_score(sc[i]);
      keep = (mode == 0) ? ((double)v >= mean) : (v >= thr);
      if (mask) mask[(int64_t)b * nb + i] = keep;
    }
    unsigned bal = __ballot_sync(0xffffffffu, keep);
    if (lane == 0) s_w[warp] = __popc(bal);
    __syncthreads();
    int before = 0, total = 0;
    for (int w = 0; w < 8; ++w) {
      before += (w < warp) ? s_w[w] : 0;
      total += s_w[w];
    }
    if (keep) idx[(int64_t)b * nb + s_carry + before + __popc(bal & ((1u << lane) - 1))] = i;
    __syncthreads();
    if (threadIdx.x == 0) s_carry += total;
    __syncthreads();
  }
  // fill: tile t covers positions [lo, hi) of the padding region
  const int nk = n_kept[b];
  for (int i = max(lo, nk) + threadIdx.x; i < hi; i += 256) idx[(int64_t)b * nb + i] = -1;
}

static int topk_count(float p, int nb) {
  double k = std::ceil((double)p * nb - 1e-6);
  if (k < 0) k = 0;
  if (k > nb) k = nb;
  return (int)k;
}

}  // namespace jenga

using namespace jenga;

extern "C" size_t jenga_select_workspace_bytes(int B, int nb) {
  if (B < 1 || nb <= SEL_SMALL_MAX) return 0;
  int ntiles = (nb + SEL_TILE - 1) / SEL_TILE;
  return (size_t)B * ntiles * (sizeof(double) + 2 * sizeof(int)) + (size_t)B * sizeof(double) + 256;
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
  double* part = (double*)w;
  int* counts = (int*)(part + (size_t)B * ntiles);
  int* offsets = counts + (size_t)B * ntiles;
  double* means = (double*)(((uintptr_t)(offsets + (size_t)B * ntiles) + 7) & ~(uintptr_t)7);
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
  {
  const int _ps = ::jenga::prof_begin("sel_count", st);
  sel_count_kernel<<<g, 256, 0, st>>>(scores, nb, kmode, param, means, ntiles, counts);
  ::jenga::prof_end(_ps, st);
  }
  JENGA_LAUNCH_CHECK();
  {
  const int _ps = ::jenga::prof_begin("sel_scan", st);
  sel_scan_kernel<<<B, 1024, 0, st>>>(counts, ntiles, offsets, n_kept);
  ::jenga::prof_end(_ps, st);
  }
  JENGA_LAUNCH_CHECK();
  {
  const int _ps = ::jenga::prof_begin("sel_write", st);
  sel_write_kernel<<<g, 256, 0, st>>>(scores, nb, kmode, param, means, ntiles, offsets, n_kept, idx, mask);
  ::jenga::prof_end(_ps, st);
  }
  JENGA_LAUNCH_CHECK();
  return JENGA_OK;
}
