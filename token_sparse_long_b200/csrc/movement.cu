// Permutation-free token movement: gather of retained rows, in-place residual
// scatter-add, row scaling.  Jenga notes §4.4 / Jenga summary §4.4.1 (Fig. 9):
// retained rows are read straight from the original input and results are added
// back in place, so the sequence is never permuted in global memory.
//
// All three are HBM-bound row moves: 128-bit loads/stores, several independent
// vectors in flight per thread, grid sized to a multiple of the SM count.
#include <cooperative_groups.h>

#include "common.cuh"

namespace jenga {

// Unsigned division by a runtime constant d >= 1 as a multiply-high and a shift (the
// round-up method of Granlund and Montgomery, "Division by invariant integers using
// multiplication", 1994): with s = ceil(log2 d) and m = floor(2^32 (2^s - d) / d) + 1,
// n / d = (umulhi(n, m) + n) >> s for every n < 2^31.
struct FastDiv {
  uint32_t d, mul, shift;
};

static FastDiv make_fastdiv(uint32_t d) {
  uint32_t s = 0;
  while ((1ull << s) < d) ++s;
  const uint64_t m = ((1ull << 32) * ((1ull << s) - d)) / d + 1;
  return FastDiv{d, (uint32_t)m, s};
}

__device__ __forceinline__ uint32_t fast_div(uint32_t n, const FastDiv& f) {
  return (__umulhi(n, f.mul) + n) >> f.shift;
}

// Work decomposition shared by gather and scatter-add: item w is chunk j = w % cpb of
// kept block i = w / cpb, a chunk being MV_CHUNK consecutive vectors (16 bytes each) of the
// block's blk x vpr vectors; vector e of block i is row e / vpr, column e % vpr.  Compact
// row i * blk + t maps to sequence row idx[i] * blk + t.  Divisions are by invariant
// constants (FastDiv) on 32-bit values: the item count and blk * vpr stay below 2^31.
constexpr int MV_UNROLL = 8;
constexpr int MV_CHUNK = 256 * MV_UNROLL;

__global__ void __launch_bounds__(256) gather_rows_kernel(const uint4* __restrict__ x, int64_t ldx_v,
                                                          int64_t bsx_v, uint4* __restrict__ out, int64_t ldo_v,
                                                          int64_t bso_v, FastDiv vpr, FastDiv cpb, int blk, int nb,
                                                          const int32_t* __restrict__ idx,
                                                          const int32_t* __restrict__ n_kept, int n_cap) {
  const int b = blockIdx.y;
  const int nk = n_kept[b];
  if (nk < 0 || (int64_t)nk * blk > n_cap || nk > nb) {
    if (threadIdx.x == 0 && blockIdx.x == 0) record_device_error(JENGA_EINTERNAL, SITE_NKEPT_RANGE, nk);
    return;
  }
  const int32_t* ib = idx + (int64_t)b * nb;
  const uint32_t per_blk = (uint32_t)blk * vpr.d;
  const uint32_t items = (uint32_t)nk * cpb.d;
  for (uint32_t w = blockIdx.x; w < items; w += gridDim.x) {
    const uint32_t bi = fast_div(w, cpb), j = w - bi * cpb.d;
    const int src_blk = __ldg(ib + bi);
    if (src_blk < 0 || src_blk >= nb) {
      if (threadIdx.x == 0) record_device_error(JENGA_EINTERNAL, SITE_INDEX_RANGE, (unsigned)src_blk);
      continue;
    }
    const uint4* src = x + b * bsx_v + (int64_t)src_blk * blk * ldx_v;
    uint4* dst = out + b * bso_v + (int64_t)bi * blk * ldo_v;
    uint4 v[MV_UNROLL];
    int64_t so[MV_UNROLL], dof[MV_UNROLL];
#pragma unroll
    for (int u = 0; u < MV_UNROLL; ++u) {
      const uint32_t e = j * MV_CHUNK + u * 256 + threadIdx.x;
      so[u] = -1;
      if (e < per_blk) {
        const uint32_t t = fast_div(e, vpr), c = e - t * vpr.d;
        so[u] = (int64_t)t * ldx_v + c;
        dof[u] = (int64_t)t * ldo_v + c;
        v[u] = __ldcs(src + so[u]);
      }
    }
#pragma unroll
    for (int u = 0; u < MV_UNROLL; ++u)
      if (so[u] >= 0) dst[dof[u]] = v[u];
  }
}

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ float2 unpack_bf16x2(uint32_t u) {
  __nv_bfloat162 h = *reinterpret_cast<__nv_bfloat162*>(&u);
  return __bfloat1622float2(h);
}

// x = round(x + alpha * y): one fp32 FMA, then (bf16) one more rounding.
template <bool BF16>
__device__ __forceinline__ uint4 axpy_vec(uint4 xv, uint4 yv, float alpha) {
  uint4 o;
  if (BF16) {
    uint32_t* xs = reinterpret_cast<uint32_t*>(&xv);
    uint32_t* ys = reinterpret_cast<uint32_t*>(&yv);
    uint32_t* os = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float2 a = unpack_bf16x2(xs[i]), b = unpack_bf16x2(ys[i]);
      os[i] = pack_bf16x2(fmaf(alpha, b.x, a.x), fmaf(alpha, b.y, a.y));
    }
  } else {
    o.x = __float_as_uint(fmaf(alpha, __uint_as_float(yv.x), __uint_as_float(xv.x)));
    o.y = __float_as_uint(fmaf(alpha, __uint_as_float(yv.y), __uint_as_float(xv.y)));
    o.z = __float_as_uint(fmaf(alpha, __uint_as_float(yv.z), __uint_as_float(xv.z)));
    o.w = __float_as_uint(fmaf(alpha, __uint_as_float(yv.w), __uint_as_float(xv.w)));
  }
  return o;
}

// x[seq row] = x + alpha * y[compact row] in place, same decomposition as the gather
template <bool BF16>
__global__ void __launch_bounds__(256) scatter_add_kernel(uint4* __restrict__ x, int64_t ldx_v, int64_t bsx_v,
                                                          const uint4* __restrict__ y, int64_t ldy_v,
                                                          int64_t bsy_v, FastDiv vpr, FastDiv cpb, int blk, int nb,
                                                          const int32_t* __restrict__ idx,
                                                          const int32_t* __restrict__ n_kept, int n_cap,
                                                          float alpha) {
  const int b = blockIdx.y;
  const int nk = n_kept[b];
  if (nk < 0 || (int64_t)nk * blk > n_cap || nk > nb) {
    if (threadIdx.x == 0 && blockIdx.x == 0) record_device_error(JENGA_EINTERNAL, SITE_NKEPT_RANGE, nk);
    return;
  }
  const int32_t* ib = idx + (int64_t)b * nb;
  const uint32_t per_blk = (uint32_t)blk * vpr.d;
  const uint32_t items = (uint32_t)nk * cpb.d;
  for (uint32_t w = blockIdx.x; w < items; w += gridDim.x) {
    const uint32_t bi = fast_div(w, cpb), j = w - bi * cpb.d;
    const int dst_blk = __ldg(ib + bi);
    if (dst_blk < 0 || dst_blk >= nb) {
      if (threadIdx.x == 0) record_device_error(JENGA_EINTERNAL, SITE_INDEX_RANGE, (unsigned)dst_blk);
      continue;
    }
    uint4* xb = x + b * bsx_v + (int64_t)dst_blk * blk * ldx_v;
    const uint4* yb = y + b * bsy_v + (int64_t)bi * blk * ldy_v;
    uint4 xv[MV_UNROLL], yv[MV_UNROLL];
    int64_t xo[MV_UNROLL];
#pragma unroll
    for (int u = 0; u < MV_UNROLL; ++u) {
      const uint32_t e = j * MV_CHUNK + u * 256 + threadIdx.x;
      xo[u] = -1;
      if (e < per_blk) {
        const uint32_t t = fast_div(e, vpr), c = e - t * vpr.d;
        xo[u] = (int64_t)t * ldx_v + c;
        yv[u] = __ldcs(yb + (int64_t)t * ldy_v + c);
        xv[u] = xb[xo[u]];
      }
    }
#pragma unroll
    for (int u = 0; u < MV_UNROLL; ++u)
      if (xo[u] >= 0) xb[xo[u]] = axpy_vec<BF16>(xv[u], yv[u], alpha);
  }
}

template <bool BF16>
__global__ void scale_rows_kernel(uint4* __restrict__ x, int64_t ldx_v, int64_t bsx_v, int vpr, int S,
                                  const int32_t* __restrict__ rows, int n_rows, float f) {
  const int b = blockIdx.y;
  const int64_t total = (int64_t)n_rows * vpr;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total;
       e += (int64_t)gridDim.x * blockDim.x) {
    int i = (int)(e / vpr);
    int c = (int)(e - (int64_t)i * vpr);
    int r = rows[(int64_t)b * n_rows + i];
    if (r < 0 || r >= S) {
      record_device_error(JENGA_EINTERNAL, SITE_INDEX_RANGE, (unsigned)r);
      continue;
    }
    uint4* p = x + b * bsx_v + (int64_t)r * ldx_v + c;
    uint4 v = *p;
    uint4 z = make_uint4(0, 0, 0, 0);
    *p = axpy_vec<BF16>(z, v, f);
  }
}

// MLP-block elimination criterion (Jenga summary §4.2.4): block i's score is the sum of
// |a| over its blk rows and the F intermediate neurons, a = SiLU(gate) * up the MLP's
// intermediate activation (bf16, compact retained rows).  A cluster of MLP_SPLIT CTAs per
// block (CTA p takes rows p, p + MLP_SPLIT, ...; 16-byte loads, 4 in flight per thread,
// fp32 sums); the cluster's partial sums meet in the first CTA's shared memory and are
// added in rank order, so the result does not depend on scheduling.  Blocks at or past
// the device count n_kept score -inf.
constexpr int MLP_SPLIT = 4;
__global__ void __cluster_dims__(1, MLP_SPLIT, 1) __launch_bounds__(256)
    mlp_block_scores_kernel(const bf16* __restrict__ a, int64_t lda, int F, int blk,
                            const int32_t* __restrict__ n_kept, int n_cap, float* __restrict__ scores) {
  namespace cg = cooperative_groups;
  const int i = blockIdx.x, part = blockIdx.y;
  int nk = n_kept ? *n_kept : n_cap;
  nk = nk < 0 ? 0 : (nk > n_cap ? n_cap : nk);
  if (i >= nk) {  // uniform over the cluster (same block)
    if (part == 0 && threadIdx.x == 0) scores[i] = -INFINITY;
    return;
  }
  __shared__ float s_w[8];
  __shared__ float s_part;
  float acc = 0.f;
  const int vpr = F / 8;                                    // 16-byte vectors per row
  const int nrow = (blk - part + MLP_SPLIT - 1) / MLP_SPLIT;  // this CTA's rows of the block
  const int total = nrow * vpr;
  const bf16* ab = a + ((int64_t)i * blk + part) * lda;
  for (int e0 = threadIdx.x; e0 < total; e0 += 4 * 256) {
    uint4 u[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int e = e0 + q * 256;
      const int r = e / vpr, c = e - r * vpr;
      u[q] = (e < total) ? __ldcs(reinterpret_cast<const uint4*>(ab + (int64_t)r * MLP_SPLIT * lda) + c)
                         : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&u[q]);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float2 f = __bfloat1622float2(p[k]);
        acc += fabsf(f.x) + fabsf(f.y);
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if ((threadIdx.x & 31) == 0) s_w[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    float t = 0.f;
    for (int w = 0; w < 8; ++w) t += s_w[w];
    s_part = t;
  }
  cg::cluster_group cluster = cg::this_cluster();
  cluster.sync();  // every CTA's partial is in its shared memory
  if (part == 0 && threadIdx.x == 0) {
    float t = 0.f;
    for (int r = 0; r < MLP_SPLIT; ++r) t += *cluster.map_shared_rank(&s_part, r);
    scores[i] = t;
  }
  cluster.sync();  // the partials are read before any CTA of the cluster exits
}

// out[i] = outer[pos[i]] for i < *n_pos, -1 after (pos indexes the outer list)
__global__ void compose_indices_kernel(const int32_t* __restrict__ outer, int n_outer_cap,
                                       const int32_t* __restrict__ pos, const int32_t* __restrict__ n_pos, int n_cap,
                                       int32_t* __restrict__ out) {
  const int np = *n_pos;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n_cap; i += gridDim.x * blockDim.x) {
    int v = -1;
    if (i < np) {
      const int p = pos[i];
      if (p < 0 || p >= n_outer_cap) {
        record_device_error(JENGA_EINTERNAL, SITE_INDEX_RANGE, (unsigned)p);
      } else {
        v = outer[p];
      }
    }
    out[i] = v;
  }
}

static int grid_for(int64_t vectors, int unroll) {
  int64_t want = (vectors + 256LL * unroll - 1) / (256LL * unroll);
  int cap = sm_count() * 8;  // 8 resident 256-thread CTAs per SM
  if (want < 1) want = 1;
  return (int)(want < cap ? want : cap);
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

}  // namespace jenga

using namespace jenga;

extern "C" jenga_status jenga_gather(const void* x, int64_t ldx, int B, int S, int h, int blk, const int32_t* idx,
                                     const int32_t* n_kept, jenga_dtype dt, void* out, int64_t ldo, int n_cap,
                                     jenga_stream_t stream) {
  JENGA_CHECK_ARG(x && idx && n_kept && (out || n_cap == 0), "jenga_gather: null pointer");
  JENGA_CHECK_ARG(B >= 1 && S >= 1 && h >= 1 && blk >= 1 && S % blk == 0 && n_cap >= 0,
                  "jenga_gather: bad sizes B=%d S=%d h=%d blk=%d", B, S, h, blk);
  JENGA_CHECK_ARG(dt == JENGA_F32 || dt == JENGA_BF16, "jenga_gather: dtype");
  const int es = dt == JENGA_F32 ? 4 : 2;
  JENGA_CHECK_ARG(ldx >= h && ldo >= h, "jenga_gather: row pitch smaller than h");
  JENGA_CHECK_ARG((h * es) % 16 == 0 && (ldx * es) % 16 == 0 && (ldo * es) % 16 == 0 && aligned16(x) &&
                      (n_cap == 0 || aligned16(out)),
                  "jenga_gather: rows must be 16-byte aligned multiples of 16 bytes");
  if (n_cap == 0) return JENGA_OK;
  const int vpr = h * es / 16;
  const int64_t ldx_v = ldx * es / 16, ldo_v = ldo * es / 16;
  JENGA_CHECK_ARG((int64_t)blk * vpr < (1ll << 30) && (int64_t)n_cap * vpr < (1ll << 40),
                  "jenga_gather: rows too long");
  const int cpb = (int)(((int64_t)blk * vpr + MV_CHUNK - 1) / MV_CHUNK);
  JENGA_CHECK_ARG((int64_t)(S / blk) * cpb < (1ll << 31), "jenga_gather: too many blocks");
  dim3 grid(grid_for((int64_t)n_cap * vpr, MV_UNROLL), B);
  {
  const int _ps = ::jenga::prof_begin("gather_rows", (cudaStream_t)stream);
  gather_rows_kernel<<<grid, 256, 0, (cudaStream_t)stream>>>(
      (const uint4*)x, ldx_v, (int64_t)S * ldx_v, (uint4*)out, ldo_v, (int64_t)n_cap * ldo_v, make_fastdiv(vpr),
      make_fastdiv(cpb), blk, S / blk, idx, n_kept, n_cap);
  ::jenga::prof_end(_ps, (cudaStream_t)stream);
  }
  JENGA_LAUNCH_CHECK();
  return JENGA_OK;
}

extern "C" jenga_status jenga_scatter_add(void* x, int64_t ldx, const void* y, int64_t ldy, int B, int S, int h,
                                          int blk, const int32_t* idx, const int32_t* n_kept, float alpha,
                                          jenga_dtype dt, int n_cap, jenga_stream_t stream) {
  JENGA_CHECK_ARG(x && idx && n_kept && (y || n_cap == 0), "jenga_scatter_add: null pointer");
  JENGA_CHECK_ARG(B >= 1 && S >= 1 && h >= 1 && blk >= 1 && S % blk == 0 && n_cap >= 0,
                  "jenga_scatter_add: bad sizes B=%d S=%d h=%d blk=%d", B, S, h, blk);
  JENGA_CHECK_ARG(dt == JENGA_F32 || dt == JENGA_BF16, "jenga_scatter_add: dtype");
  const int es = dt == JENGA_F32 ? 4 : 2;
  JENGA_CHECK_ARG(ldx >= h && ldy >= h, "jenga_scatter_add: row pitch smaller than h");
  JENGA_CHECK_ARG((h * es) % 16 == 0 && (ldx * es) % 16 == 0 && (ldy * es) % 16 == 0 && aligned16(x) &&
                      (n_cap == 0 || aligned16(y)),
                  "jenga_scatter_add: rows must be 16-byte aligned multiples of 16 bytes");
  if (n_cap == 0) return JENGA_OK;
  const int vpr = h * es / 16;
  const int64_t ldx_v = ldx * es / 16, ldy_v = ldy * es / 16;
  JENGA_CHECK_ARG((int64_t)blk * vpr < (1ll << 30), "jenga_scatter_add: rows too long");
  const int cpb = (int)(((int64_t)blk * vpr + MV_CHUNK - 1) / MV_CHUNK);
  JENGA_CHECK_ARG((int64_t)(S / blk) * cpb < (1ll << 31), "jenga_scatter_add: too many blocks");
  const FastDiv vd = make_fastdiv(vpr), cd = make_fastdiv(cpb);
  dim3 grid(grid_for((int64_t)n_cap * vpr, MV_UNROLL), B);
  if (dt == JENGA_BF16)
    {
    const int _ps = ::jenga::prof_begin("scatter_add", (cudaStream_t)stream);
    scatter_add_kernel<true><<<grid, 256, 0, (cudaStream_t)stream>>>(
        (uint4*)x, ldx_v, (int64_t)S * ldx_v, (const uint4*)y, ldy_v, (int64_t)n_cap * ldy_v, vd, cd, blk, S / blk,
        idx, n_kept, n_cap, alpha);
    ::jenga::prof_end(_ps, (cudaStream_t)stream);
    }
  else
    {
    const int _ps = ::jenga::prof_begin("scatter_add", (cudaStream_t)stream);
    scatter_add_kernel<false><<<grid, 256, 0, (cudaStream_t)stream>>>(
        (uint4*)x, ldx_v, (int64_t)S * ldx_v, (const uint4*)y, ldy_v, (int64_t)n_cap * ldy_v, vd, cd, blk, S / blk,
        idx, n_kept, n_cap, alpha);
    ::jenga::prof_end(_ps, (cudaStream_t)stream);
    }
  JENGA_LAUNCH_CHECK();
  return JENGA_OK;
}

extern "C" jenga_status jenga_scale_rows(void* x, int64_t ldx, int B, int S, int h, const int32_t* rows,
                                         int n_rows, float factor, jenga_dtype dt, jenga_stream_t stream) {
  JENGA_CHECK_ARG(x && (rows || n_rows == 0), "jenga_scale_rows: null pointer");
  JENGA_CHECK_ARG(B >= 1 && S >= 1 && h >= 1 && n_rows >= 0 && ldx >= h, "jenga_scale_rows: bad sizes");
  const int es = dt == JENGA_F32 ? 4 : 2;
  JENGA_CHECK_ARG((h * es) % 16 == 0 && (ldx * es) % 16 == 0 && aligned16(x),
                  "jenga_scale_rows: rows must be 16-byte aligned multiples of 16 bytes");
  if (n_rows == 0) return JENGA_OK;
  const int vpr = h * es / 16;
  const int64_t ldx_v = ldx * es / 16;
  dim3 grid(grid_for((int64_t)n_rows * vpr, 1), B);
  if (dt == JENGA_BF16)
    {
    const int _ps = ::jenga::prof_begin("scale_rows", (cudaStream_t)stream);
    scale_rows_kernel<true><<<grid, 256, 0, (cudaStream_t)stream>>>((uint4*)x, ldx_v, (int64_t)S * ldx_v, vpr, S,
                                                                     rows, n_rows, factor);
    ::jenga::prof_end(_ps, (cudaStream_t)stream);
    }
  else
    {
    const int _ps = ::jenga::prof_begin("scale_rows", (cudaStream_t)stream);
    scale_rows_kernel<false><<<grid, 256, 0, (cudaStream_t)stream>>>((uint4*)x, ldx_v, (int64_t)S * ldx_v, vpr,
                                                                      S, rows, n_rows, factor);
    ::jenga::prof_end(_ps, (cudaStream_t)stream);
    }
  JENGA_LAUNCH_CHECK();
  return JENGA_OK;
}

extern "C" jenga_status jenga_mlp_block_scores(const void* a, int64_t lda, int F, int blk, const int32_t* n_kept,
                                               int n_cap, float* scores, jenga_stream_t stream) {
  JENGA_CHECK_ARG(a && scores, "jenga_mlp_block_scores: null pointer");
  JENGA_CHECK_ARG(F >= 8 && F % 8 == 0 && lda >= F && lda % 8 == 0 && blk >= 1 && n_cap >= 0 &&
                      (int64_t)blk * (F / 8) < (1ll << 30) &&
                      ((uintptr_t)a & 15) == 0,
                  "jenga_mlp_block_scores: F and lda multiples of 8, 16-byte aligned rows");
  if (n_cap == 0) return JENGA_OK;
  cudaStream_t st = (cudaStream_t)stream;
  {
    const int _ps = ::jenga::prof_begin("mlp_block_scores", st);
    mlp_block_scores_kernel<<<dim3(n_cap, MLP_SPLIT), 256, 0, st>>>((const bf16*)a, lda, F, blk, n_kept, n_cap,
                                                                    scores);
    ::jenga::prof_end(_ps, st);
  }
  JENGA_LAUNCH_CHECK();
  return JENGA_OK;
}

extern "C" jenga_status jenga_compose_block_indices(const int32_t* outer, int n_outer_cap, const int32_t* pos,
                                                    const int32_t* n_pos, int n_cap, int32_t* out,
                                                    jenga_stream_t stream) {
  JENGA_CHECK_ARG(outer && pos && n_pos && out && n_outer_cap >= 0 && n_cap >= 0,
                  "jenga_compose_block_indices: bad arguments");
  if (n_cap == 0) return JENGA_OK;
  cudaStream_t st = (cudaStream_t)stream;
  compose_indices_kernel<<<(n_cap + 255) / 256 < 1024 ? (n_cap + 255) / 256 : 1024, 256, 0, st>>>(
      outer, n_outer_cap, pos, n_pos, n_cap, out);
  JENGA_LAUNCH_CHECK();
  return JENGA_OK;
}
