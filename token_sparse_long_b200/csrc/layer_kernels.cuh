// Row kernels of the retained-token layer: RMSNorm (with the permutation-free
// gather of the retained rows), RMSNorm backward (with the in-place scatter of dX),
// segment gather, RoPE backward + dQKV packing, LoRA gradient reductions, and the
// weight re-layout used by jenga_layer_pack.
#pragma once

#include "common.cuh"

namespace jenga {

constexpr int ROW_THREADS = 256;
// The one-CTA-per-row kernels take the 8-element chunks per thread as a template argument
// MAXC (2 for hidden <= 4096, 4 for hidden <= 8192), so a row's registers do not cap the
// resident CTAs.

__device__ __forceinline__ float block_sum_256(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float t = 0.f;
#pragma unroll
  for (int w = 0; w < ROW_THREADS / 32; ++w) t += red[w];
  return t;
}

__device__ __forceinline__ float block_max_256(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float t = 0.f;
#pragma unroll
  for (int w = 0; w < ROW_THREADS / 32; ++w) t = fmaxf(t, red[w]);
  return t;
}

// Row scale of an fp16 GEMM operand: sc = 2^(13 - e) for amax in [2^e, 2^(e+1)), so the
// row's largest magnitude lands in [2^13, 2^14) (fp16 keeps 11 significant bits up to
// 65504); r = 1 / sc.  Both are powers of two built from their exponent bits, so the
// scaling and its undoing in the GEMM epilogue are exact.
__device__ __forceinline__ void pow2_row_scale(float amax, float& sc, float& r) {
  int e = (int)((__float_as_uint(amax) >> 23) & 255u) - 127;
  e = e < -113 ? -113 : (e > 127 ? 127 : e);
  sc = __uint_as_float((uint32_t)(127 + 13 - e) << 23);
  r = __uint_as_float((uint32_t)(127 - 13 + e) << 23);
}

__device__ __forceinline__ void unpack8(const uint4& u, float* f) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 t = __bfloat1622float2(h[i]);
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}
__device__ __forceinline__ uint4 pack8(const float* f) {
  uint4 u;
  uint32_t* w = reinterpret_cast<uint32_t*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    __nv_bfloat162 h = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
    w[i] = *reinterpret_cast<uint32_t*>(&h);
  }
  return u;
}

__device__ __forceinline__ int valid_rows(const int32_t* n_valid, int mult, int row_offset, int cap) {
  if (!n_valid) return cap;
  int v = (*n_valid) * mult - row_offset;
  return v < 0 ? 0 : (v < cap ? v : cap);
}

__device__ __forceinline__ int64_t seq_row(const int32_t* idx, int blk, int c) {
  if (!idx) return c;
  const int b = c / blk;
  return (int64_t)__ldg(idx + b) * blk + (c - b * blk);
}

// xn[m] = bf16(x[row(m)] * rstd * gain); rstd[m]; optionally xr[m] = x[row(m)] (gathered copy).
// One CTA per compact row m in [0, rows); row(m) = seq_row(idx, blk, row_offset + m).
template <int MAXC>
__global__ void __launch_bounds__(ROW_THREADS) rmsnorm_rows_kernel(
    const bf16* __restrict__ x, int64_t ldx, const int32_t* __restrict__ idx, int blk, int row_offset,
    const int32_t* __restrict__ n_valid, int valid_mult, int h, float eps, const bf16* __restrict__ gain,
    bf16* __restrict__ xr, int64_t ldr, bf16* __restrict__ xn, int64_t ldn, float* __restrict__ rstd_out,
    int64_t x_rows) {
  __shared__ float red[ROW_THREADS / 32];
  const int m = blockIdx.x;
  if (m >= valid_rows(n_valid, valid_mult, row_offset, gridDim.x)) return;
  // with a kept-block list, x is the full sequence; without one, x is already compact
  const int64_t row = idx ? seq_row(idx, blk, row_offset + m) : m;
  if (row < 0 || row >= x_rows) {
    if (threadIdx.x == 0) record_device_error(JENGA_EINTERNAL, SITE_INDEX_RANGE, (unsigned)row);
    return;
  }
  const uint4* src = reinterpret_cast<const uint4*>(x + row * ldx);
  const int nch = h >> 3;
  float v[MAXC][8];
  uint4 raw[MAXC];
  float ss = 0.f;
#pragma unroll
  for (int i = 0; i < MAXC; ++i) {
    const int c = threadIdx.x + i * ROW_THREADS;
    if (c < nch) {
      raw[i] = src[c];
      unpack8(raw[i], v[i]);
#pragma unroll
      for (int e = 0; e < 8; ++e) ss = fmaf(v[i][e], v[i][e], ss);
    }
  }
  ss = block_sum_256(ss, red);
  const float r = rsqrtf(ss / (float)h + eps);
  if (threadIdx.x == 0 && rstd_out) rstd_out[m] = r;
  const uint4* gp = reinterpret_cast<const uint4*>(gain);
#pragma unroll
  for (int i = 0; i < MAXC; ++i) {
    const int c = threadIdx.x + i * ROW_THREADS;
    if (c < nch) {
      if (xr) reinterpret_cast<uint4*>(xr + (int64_t)m * ldr)[c] = raw[i];
      float gv[8], o[8];
      unpack8(gp[c], gv);
#pragma unroll
      for (int e = 0; e < 8; ++e) o[e] = v[i][e] * r * gv[e];
      reinterpret_cast<uint4*>(xn + (int64_t)m * ldn)[c] = pack8(o);
    }
  }
}

// RMSNorm backward fused with the residual:
//   out[m] = base[m] + r g dy - x r^3 / h * sum(dy g x)
// base: fp32 (base_f) or bf16 (base_b); outputs: fp32 out_f, the fp16 GEMM operand out_h
// (row m scaled by the power of two of pow2_row_scale, its inverse in out_rs[m]), and/or
// the bf16 scatter into dst[row(m)] (in place, pitch ldd).
template <int MAXC>
__global__ void __launch_bounds__(ROW_THREADS) rmsnorm_bwd_rows_kernel(
    const float* __restrict__ dy, int64_t lddy, const bf16* __restrict__ x, int64_t ldx,
    const float* __restrict__ rstd, const bf16* __restrict__ gain, const float* __restrict__ base_f,
    const bf16* __restrict__ base_b, int64_t ldb, float* __restrict__ out_f, __half* __restrict__ out_h,
    float* __restrict__ out_rs, int64_t ldo, bf16* __restrict__ dst, int64_t ldd, const int32_t* __restrict__ idx, int blk, int row_offset,
    const int32_t* __restrict__ n_valid, int valid_mult, int h, int64_t dst_rows,
    const uint8_t* __restrict__ keep_mask = nullptr, int mask_blk = 1) {
  __shared__ float red[ROW_THREADS / 32];
  const int m = blockIdx.x;
  if (m >= valid_rows(n_valid, valid_mult, row_offset, gridDim.x)) return;
  const int nch = h >> 3;
  // a row of a masked block (keep_mask entry 0) has no sub-block gradient: out = base
  const bool live = !keep_mask || __ldg(keep_mask + (row_offset + m) / mask_blk);
  const float r = live ? rstd[m] : 0.f;
  float dyg[MAXC][8], xv[MAXC][8], bv[MAXC][8];
  float dot = 0.f;
#pragma unroll
  for (int i = 0; i < MAXC; ++i) {
    const int c = threadIdx.x + i * ROW_THREADS;
    if (c < nch) {
      // the residual base is loaded here too, so its latency overlaps the row reduction
      if (base_f) {
        const float4* bp = reinterpret_cast<const float4*>(base_f + (int64_t)m * ldb) + 2 * c;
        const float4 a = bp[0], b = bp[1];
        bv[i][0] = a.x; bv[i][1] = a.y; bv[i][2] = a.z; bv[i][3] = a.w;
        bv[i][4] = b.x; bv[i][5] = b.y; bv[i][6] = b.z; bv[i][7] = b.w;
      } else {
        unpack8(reinterpret_cast<const uint4*>(base_b + (int64_t)m * ldb)[c], bv[i]);
      }
      if (live) {
        const float4* dp = reinterpret_cast<const float4*>(dy + (int64_t)m * lddy) + 2 * c;
        float4 a = dp[0], b = dp[1];
        float gv[8];
        unpack8(reinterpret_cast<const uint4*>(gain)[c], gv);
        unpack8(reinterpret_cast<const uint4*>(x + (int64_t)m * ldx)[c], xv[i]);
        const float d[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          dyg[i][e] = d[e] * gv[e];
          dot = fmaf(dyg[i][e], xv[i][e], dot);
        }
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          dyg[i][e] = 0.f;
          xv[i][e] = 0.f;
        }
      }
    }
  }
  dot = block_sum_256(dot, red);
  const float k = r * r * r * dot / (float)h;
  const int64_t drow = dst ? seq_row(idx, blk, row_offset + m) : 0;
  if (dst && (drow < 0 || drow >= dst_rows)) {
    if (threadIdx.x == 0) record_device_error(JENGA_EINTERNAL, SITE_INDEX_RANGE, (unsigned)drow);
    return;
  }
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < MAXC; ++i) {
    const int c = threadIdx.x + i * ROW_THREADS;
    if (c < nch) {
      float* o = bv[i];  // the output overwrites the residual base in registers
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        o[e] = bv[i][e] + r * dyg[i][e] - xv[i][e] * k;
        amax = fmaxf(amax, fabsf(o[e]));
      }
      if (out_f) {
        float4* op = reinterpret_cast<float4*>(out_f + (int64_t)m * ldo) + 2 * c;
        op[0] = make_float4(o[0], o[1], o[2], o[3]);
        op[1] = make_float4(o[4], o[5], o[6], o[7]);
      }
      if (dst) reinterpret_cast<uint4*>(dst + drow * ldd)[c] = pack8(o);
    }
  }
  if (out_h) {  // block-uniform branch: the reduction's barriers are reached by every thread
    amax = block_max_256(amax, red);
    float sc, rs;
    pow2_row_scale(amax, sc, rs);
    if (threadIdx.x == 0) out_rs[m] = rs;
#pragma unroll
    for (int i = 0; i < MAXC; ++i) {
      const int c = threadIdx.x + i * ROW_THREADS;
      if (c < nch) {
        uint4 u;
        uint32_t* w = reinterpret_cast<uint32_t*>(&u);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const __half2 hv = __floats2half2_rn(bv[i][2 * e] * sc, bv[i][2 * e + 1] * sc);
          w[e] = *reinterpret_cast<const uint32_t*>(&hv);
        }
        reinterpret_cast<uint4*>(out_h + (int64_t)m * ldo)[c] = u;
      }
    }
  }
}

// out[m] = src[row(row_offset + m)] for m in [0, rows) (bf16 rows, 16-byte vectors)
__global__ void gather_seg_kernel(const bf16* __restrict__ src, int64_t lds, bf16* __restrict__ out, int64_t ldo,
                                  const int32_t* __restrict__ idx, int blk, int row_offset,
                                  const int32_t* __restrict__ n_valid, int valid_mult, int rows, int h,
                                  int64_t src_rows) {
  const int vpr = h >> 3;
  const int nv = valid_rows(n_valid, valid_mult, row_offset, rows);
  const int64_t total = (int64_t)nv * vpr;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total; e += (int64_t)gridDim.x * blockDim.x) {
    const int m = (int)(e / vpr), c = (int)(e - (int64_t)m * vpr);
    const int64_t r = seq_row(idx, blk, row_offset + m);
    if (r < 0 || r >= src_rows) {
      record_device_error(JENGA_EINTERNAL, SITE_INDEX_RANGE, (unsigned)r);
      continue;
    }
    reinterpret_cast<uint4*>(out + (int64_t)m * ldo)[c] = reinterpret_cast<const uint4*>(src + r * lds)[c];
  }
}

// Backward of RoPE on dq / dk (the transpose rotation) and the pack of dQ | dK | dV of the
// segment's rows [s0, s0 + nv) into one fp16 GEMM operand, each row scaled by the power of
// two of pow2_row_scale (its inverse in rs[m]).  One CTA per row: thread e of the row's
// H x 32 (head, frequency pair) items takes pair (2 ip, 2 ip + 1) of head hh, reading its
// (cos, sin) pairs from the segment's RoPE table (tab[m][j], rope_table_kernel at offset
// s0); the rotated values wait in registers for the row's largest magnitude.
// RB items per thread (a template argument: 4 for H <= 32, 8 for H <= 64)
template <int RB>
__global__ void __launch_bounds__(ROW_THREADS) rope_bwd_pack_kernel(
    const float* __restrict__ dq, int64_t ld_dq, const float* __restrict__ dk, const float* __restrict__ dv,
    int64_t ld_acc, int s0, __half* __restrict__ dqkv, float* __restrict__ rs, int64_t ld_out,
    const float2* __restrict__ tab, const int32_t* __restrict__ n_valid, int valid_mult, int rows, int H) {
  __shared__ float red[ROW_THREADS / 32];
  const int m = blockIdx.x;
  if (m >= valid_rows(n_valid, valid_mult, s0, rows)) return;
  const int HD = H * 128, items = H * 32;
  float val[RB][12];
  float amax = 0.f;
#pragma unroll
  for (int k = 0; k < RB; ++k) {
    const int e = threadIdx.x + k * ROW_THREADS;
    if (e < items) {
      const int ip = e & 31, hh = e >> 5;
      const float4 t = __ldg(reinterpret_cast<const float4*>(tab + (int64_t)m * 64) + ip);  // (cos, sin) x 2
      const int c1 = hh * 128 + 2 * ip, c2 = c1 + 64;
      const float2 a1 = *reinterpret_cast<const float2*>(dq + (int64_t)m * ld_dq + c1);
      const float2 a2 = *reinterpret_cast<const float2*>(dq + (int64_t)m * ld_dq + c2);
      const float2 b1 = *reinterpret_cast<const float2*>(dk + (int64_t)(s0 + m) * ld_acc + c1);
      const float2 b2 = *reinterpret_cast<const float2*>(dk + (int64_t)(s0 + m) * ld_acc + c2);
      const float2 v1 = *reinterpret_cast<const float2*>(dv + (int64_t)(s0 + m) * ld_acc + c1);
      const float2 v2 = *reinterpret_cast<const float2*>(dv + (int64_t)(s0 + m) * ld_acc + c2);
      // per frequency: (x1, x2) -> (x1 cos + x2 sin, x2 cos - x1 sin)
      val[k][0] = a1.x * t.x + a2.x * t.y;
      val[k][1] = a1.y * t.z + a2.y * t.w;
      val[k][2] = a2.x * t.x - a1.x * t.y;
      val[k][3] = a2.y * t.z - a1.y * t.w;
      val[k][4] = b1.x * t.x + b2.x * t.y;
      val[k][5] = b1.y * t.z + b2.y * t.w;
      val[k][6] = b2.x * t.x - b1.x * t.y;
      val[k][7] = b2.y * t.z - b1.y * t.w;
      val[k][8] = v1.x;
      val[k][9] = v1.y;
      val[k][10] = v2.x;
      val[k][11] = v2.y;
#pragma unroll
      for (int j = 0; j < 12; ++j) amax = fmaxf(amax, fabsf(val[k][j]));
    }
  }
  amax = block_max_256(amax, red);
  float sc, r;
  pow2_row_scale(amax, sc, r);
  if (threadIdx.x == 0) rs[m] = r;
  __half* o = dqkv + (int64_t)m * ld_out;
#pragma unroll
  for (int k = 0; k < RB; ++k) {
    const int e = threadIdx.x + k * ROW_THREADS;
    if (e < items) {
      const int ip = e & 31, hh = e >> 5;
      const int c1 = hh * 128 + 2 * ip, c2 = c1 + 64;
      const int col[6] = {c1, c2, HD + c1, HD + c2, 2 * HD + c1, 2 * HD + c2};
#pragma unroll
      for (int j = 0; j < 6; ++j)
        *reinterpret_cast<__half2*>(o + col[j]) = __floats2half2_rn(val[k][2 * j] * sc, val[k][2 * j + 1] * sc);
    }
  }
}

// Split-K partials of  P[chunk][c][r] = sum_{m in chunk} X[m, c] * xs[m] * Y[m, r]   (r < 16)
// X bf16 or fp16 [rows, ldx] (columns [0, C)), xs an optional per-row factor, Y fp32
// [rows, ldy] (columns [0, 16)).
constexpr int LG_CHUNK = 512;   // rows per partial sum
constexpr int LG_COLS = 512;    // columns per block (2 per thread)

// One LoRA gradient product: out[c * so_c + r * so_r] += scale * sum_m X[m, c] Y[m, r]
// (r < 16).  The four of a layer segment (dB_q, dB_v from dQ / dV and t; dA_q, dA_v from
// xn and dt) run in one launch, blockIdx.z = job.
struct LoraGradJob {
  const void* X;   // bf16, or fp16 when x_f16
  int64_t ldx;
  const float* Y;  // 16 consecutive fp32 per row, row pitch ldy
  int C;
  float scale;
  float* out;
  int64_t so_c, so_r;
  const float* xs;  // per-row factor of X (the inverse of its fp16 row scale), or null
  int x_f16;
};
struct LoraGradJobs {
  LoraGradJob j[4];
};

// part[job][chunk][c][16]: each thread owns 2 columns x 16 ranks of one 512-row chunk; the
// chunk's Y rows are staged in shared memory (broadcast reads), X arrives as bf16 pairs
// and the products accumulate as packed f32x2 FMAs.
__global__ void __launch_bounds__(256) lora_grad_partial_kernel(LoraGradJobs jobs, int64_t ldy, int rows,
                                                                const int32_t* __restrict__ n_valid, int valid_mult,
                                                                int row_offset, int cmax, float* __restrict__ part) {
  __shared__ __align__(16) float sY[LG_CHUNK * 16];
  const LoraGradJob jb = jobs.j[blockIdx.z];
  const int nv = valid_rows(n_valid, valid_mult, row_offset, rows);
  const int m0 = blockIdx.y * LG_CHUNK, m1 = min(nv, m0 + LG_CHUNK);
  const int c = blockIdx.x * LG_COLS + threadIdx.x * 2;
  if (blockIdx.x * LG_COLS >= jb.C) return;  // uniform per block
  for (int e = threadIdx.x; e < LG_CHUNK * 4; e += 256) {
    const int rr = e >> 2, q = e & 3;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (m0 + rr < m1) {
      v = *reinterpret_cast<const float4*>(jb.Y + (int64_t)(m0 + rr) * ldy + 4 * q);
      if (jb.xs) {  // X's row factor rides on Y
        const float f = __ldg(jb.xs + m0 + rr);
        v.x *= f;
        v.y *= f;
        v.z *= f;
        v.w *= f;
      }
    }
    reinterpret_cast<float4*>(sY)[e] = v;
  }
  __syncthreads();
  uint64_t acc[16];  // acc[r] = (column c, column c + 1) pair of rank r
#pragma unroll
  for (int r = 0; r < 16; ++r) acc[r] = 0ull;
  if (c < jb.C) {
    const uint16_t* xp = reinterpret_cast<const uint16_t*>(jb.X) + (int64_t)m0 * jb.ldx + c;
    const bool xh = jb.x_f16;
    auto rank_update = [&](uint32_t xw, int mr) {  // row mr (chunk-relative) of X and Y
      const float2 x = xh ? __half22float2(*reinterpret_cast<const __half2*>(&xw))
                          : __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&xw));
      const uint64_t x2 = f2pack(x.x, x.y);
      const float4* yr = reinterpret_cast<const float4*>(sY + mr * 16);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float4 y = yr[q];
        acc[4 * q] = ffma2(x2, f2pack(y.x, y.x), acc[4 * q]);
        acc[4 * q + 1] = ffma2(x2, f2pack(y.y, y.y), acc[4 * q + 1]);
        acc[4 * q + 2] = ffma2(x2, f2pack(y.z, y.z), acc[4 * q + 2]);
        acc[4 * q + 3] = ffma2(x2, f2pack(y.w, y.w), acc[4 * q + 3]);
      }
    };
    int m = m0;
    // eight rows' X pairs in flight per step (the loop is load-latency bound otherwise)
    for (; m + 8 <= m1; m += 8, xp += 8 * jb.ldx) {
      uint32_t xw[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) xw[u] = *reinterpret_cast<const uint32_t*>(xp + u * jb.ldx);
#pragma unroll
      for (int u = 0; u < 8; ++u) rank_update(xw[u], m - m0 + u);
    }
    for (; m < m1; ++m, xp += jb.ldx) rank_update(*reinterpret_cast<const uint32_t*>(xp), m - m0);
    float lo[16], hi[16];
#pragma unroll
    for (int r = 0; r < 16; ++r) f2unpack(acc[r], lo[r], hi[r]);
    float* p = part + (((int64_t)blockIdx.z * gridDim.y + blockIdx.y) * cmax + c) * 16;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      reinterpret_cast<float4*>(p)[q] = make_float4(lo[4 * q], lo[4 * q + 1], lo[4 * q + 2], lo[4 * q + 3]);
      reinterpret_cast<float4*>(p + 16)[q] = make_float4(hi[4 * q], hi[4 * q + 1], hi[4 * q + 2], hi[4 * q + 3]);
    }
  }
}

// The LoRA term of the dX product from the split dt product (ksplit partial sums of
// acc = dQKV' [Bq; Bv]^T over ranges of the reduction, dQKV' the row-scaled fp16 operand):
//   dt[m, j] = ls r_m sum_ks part[ks][m][j]          (fp32, for the LoRA gradients)
//   aux[m, j], aux[m, 32 + j] = fp16 hi, lo of ls sum_ks part[ks][m][j] / c
// (the K-padded fp16 operand of the dX product; c = *cdiv, r_m = rs[m]).  The partial sums
// are added in range order.
__global__ void lora_t_reduce_kernel(const float* __restrict__ part, int ksplit, int rows,
                                     const int32_t* __restrict__ n_valid, int valid_mult, int row_offset, float ls,
                                     const float* __restrict__ rs, const float* __restrict__ cdiv,
                                     float* __restrict__ dt, int64_t ld_dt, __half* __restrict__ aux, int64_t ld_aux) {
  const int nv = valid_rows(n_valid, valid_mult, row_offset, rows);
  const float ic = 1.f / __ldg(cdiv);  // a power of two: exact
  for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < nv * 32; e += gridDim.x * blockDim.x) {
    const int m = e >> 5, j = e & 31;
    float a = 0.f;
    for (int ks = 0; ks < ksplit; ++ks) a += part[((int64_t)ks * rows + m) * 32 + j];
    dt[(int64_t)m * ld_dt + j] = a * ls * __ldg(rs + m);
    const float w = a * ls * ic;
    const __half hi = __float2half_rn(w);
    aux[(int64_t)m * ld_aux + j] = hi;
    aux[(int64_t)m * ld_aux + 32 + j] = __float2half_rn(w - __half2float(hi));
  }
}

// out[c * so_c + r * so_r] += scale * sum_chunk part[job][chunk][c][r]   (fixed chunk order)
__global__ void lora_grad_reduce_kernel(LoraGradJobs jobs, const float* __restrict__ part, int chunks, int cmax) {
  const LoraGradJob jb = jobs.j[blockIdx.y];
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= jb.C * 16) return;
  const int c = e >> 4, r = e & 15;
  float s = 0.f;
  for (int k = 0; k < chunks; ++k) s += part[(((int64_t)blockIdx.y * chunks + k) * cmax + c) * 16 + r];
  jb.out[c * jb.so_c + r * jb.so_r] += jb.scale * s;
}

// RoPE table: tab[m][j] = (cos, sin)(position(m) * inv_freq[j]) for the rows m of a QKV GEMM
// (position through the kept-block list when idx is given), the angle reduced to [-pi, pi] in
// float64 before a float sincos.  Rows past the device-side valid count get position 0.
__global__ void rope_table_kernel(float2* __restrict__ tab, int rows, const int32_t* __restrict__ idx, int blk,
                                  const int32_t* __restrict__ n_valid, int valid_mult, int row_offset,
                                  const double* __restrict__ inv_freq) {
  const int nv = valid_rows(n_valid, valid_mult, row_offset, rows);
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < (int64_t)rows * 64;
       e += (int64_t)gridDim.x * blockDim.x) {
    const int m = (int)(e >> 6), j = (int)(e & 63);
    const int64_t pos = (m < nv) ? (idx ? seq_row(idx, blk, row_offset + m) : row_offset + m) : 0;
    const double ang = (double)pos * inv_freq[j];
    const double red = ang - 6.283185307179586 * rint(ang * 0.15915494309189535);
    float sn, cs;
    sincosf((float)red, &sn, &cs);
    tab[e] = make_float2(cs, sn);
  }
}

// dst[m, 0:cols] = src[row(m), 0:cols] for the compact rows m below the device-side valid
// count (row(m) through the kept-block list), 16-byte vectors; cols % 8 == 0.
__global__ void gather_rows_bf16_kernel(const bf16* __restrict__ src, int64_t lds, bf16* __restrict__ dst,
                                        int64_t ldd, int cols, const int32_t* __restrict__ idx, int blk,
                                        const int32_t* __restrict__ n_valid, int valid_mult, int rows) {
  const int nv = valid_rows(n_valid, valid_mult, 0, rows);
  const int vpr = cols / 8;
  const int64_t total = (int64_t)nv * vpr;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total; e += (int64_t)gridDim.x * blockDim.x) {
    const int m = (int)(e / vpr), c = (int)(e - (int64_t)m * vpr);
    const int64_t r = seq_row(idx, blk, m);
    reinterpret_cast<uint4*>(dst + (int64_t)m * ldd)[c] = __ldg(reinterpret_cast<const uint4*>(src + r * lds) + c);
  }
}

// ---- weight re-layout (pack)
// dst[(dr0 + c) * ldd + dc0 + r] = src[(sr0 + r) * lds + sc0 + c] for r < R, c < C   (transpose)
__global__ void transpose_bf16_kernel(const bf16* __restrict__ src, int64_t lds, bf16* __restrict__ dst,
                                      int64_t ldd, int R, int C) {
  __shared__ bf16 tile[32][33];
  const int r0 = blockIdx.y * 32, c0 = blockIdx.x * 32;
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int r = r0 + i, c = c0 + threadIdx.x;
    if (r < R && c < C) tile[i][threadIdx.x] = src[(int64_t)r * lds + c];
  }
  __syncthreads();
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int c = c0 + i, r = r0 + threadIdx.x;
    if (r < R && c < C) dst[(int64_t)c * ldd + r] = tile[threadIdx.x][i];
  }
}

// dst[r * ldd + c] = src[r * lds + c]
__global__ void copy_bf16_kernel(const bf16* __restrict__ src, int64_t lds, bf16* __restrict__ dst, int64_t ldd,
                                 int R, int C) {
  const int64_t total = (int64_t)R * C;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total; e += (int64_t)gridDim.x * blockDim.x) {
    const int r = (int)(e / C), c = (int)(e - (int64_t)r * C);
    dst[(int64_t)r * ldd + c] = src[(int64_t)r * lds + c];
  }
}

// wgu row r: group g = r / 128; rows 0..63 of a group are gate rows 64g.., 64..127 up rows 64g..
__global__ void interleave_gate_up_kernel(const bf16* __restrict__ wg, const bf16* __restrict__ wu,
                                          bf16* __restrict__ wgu, int F, int h) {
  const int64_t total = (int64_t)2 * F * h;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total; e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = e / h, c = e - r * h;
    const int g = (int)(r >> 7), j = (int)(r & 127);
    const bf16* src = (j < 64) ? wg + ((int64_t)g * 64 + j) * h : wu + ((int64_t)g * 64 + j - 64) * h;
    wgu[e] = src[c];
  }
}

// Rows [valid, cap) of a bf16 [cap, cols] buffer set to zero (valid read on the device).
__global__ void zero_tail_rows_kernel(bf16* __restrict__ x, int64_t ld, int cols, const int32_t* __restrict__ n_valid,
                                      int valid_mult, int cap) {
  int v = n_valid ? (*n_valid) * valid_mult : cap;
  v = v < 0 ? 0 : (v < cap ? v : cap);
  const int vpr = cols >> 3;
  const int64_t total = (int64_t)(cap - v) * vpr;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total; e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = v + e / vpr;
    const int c = (int)(e % vpr);
    reinterpret_cast<uint4*>(x + r * ld)[c] = make_uint4(0, 0, 0, 0);
  }
}

// In-place bf16 -> fp16 re-encoding of a backward weight operand, times an optional
// power-of-two factor *mul (exact for magnitudes in [2^-14, 65504] after the factor, which
// frozen weights are well inside; smaller ones keep fp16's subnormal spacing 2^-24).  A
// finite value that would overflow fp16 records JENGA_EINVAL at SITE_PACK_RANGE.
__global__ void bf16_to_f16_inplace_kernel(uint16_t* __restrict__ x, int64_t n, const float* __restrict__ mul) {
  const float f0 = mul ? *mul : 1.f;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += (int64_t)gridDim.x * blockDim.x) {
    const float f = __uint_as_float((uint32_t)x[e] << 16) * f0;
    const __half hv = __float2half_rn(f);
    if (fabsf(f) < INFINITY && __hisinf(hv)) record_device_error(JENGA_EINVAL, SITE_PACK_RANGE, (unsigned)e);
    x[e] = *reinterpret_cast<const uint16_t*>(&hv);
  }
}

// c[0] = the power of two >= 2 max(lscale, 1) max_j sum_k |b[j, k]| over the rows of the LoRA
// up-projection operand b [rows, cols] (bf16), at least 1.  It divides the fp16 LoRA operand
// s_m dt_m of the dX product (and multiplies the matching [Aq; Av] columns): a dQKV row
// scaled below 2^14 gives |s_m dt_m| <= lscale 2^14 max_j sum_k |b[j, k]|, so the stored
// s_m dt_m / c stays below 2^13 for a backward LoRA scale up to max(lscale, 1).
// One CTA of 32 warps, warp j < rows sums row j.
__global__ void lora_l1_divisor_kernel(const bf16* __restrict__ b, int rows, int cols, float lscale,
                                       float* __restrict__ c) {
  __shared__ float rmax[32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float s = 0.f;
  if (warp < rows)
    for (int k = lane; k < cols; k += 32) s += fabsf(__bfloat162float(b[(int64_t)warp * cols + k]));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if (lane == 0) rmax[warp] = s;
  __syncthreads();
  if (threadIdx.x == 0) {
    float mx = 0.f;
    for (int w = 0; w < 32; ++w) mx = fmaxf(mx, rmax[w]);
    const float need = 2.f * fmaxf(lscale, 1.f) * mx;
    float v = 1.f;
    while (v < need && v < 0x1p100f) v *= 2.f;
    c[0] = v;
  }
}

__global__ void zero_bf16_kernel(bf16* __restrict__ dst, int64_t n) {
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += (int64_t)gridDim.x * blockDim.x)
    dst[e] = __float2bfloat16_rn(0.f);
}

// ---------------------------------------------------------------- fp16 operands of the
// attention backward (attn_bwd_tc.cuh): fp16 copies of q | k | v, a power-of-two scale for
// the segment's dO, and a dS scale that cannot overflow.
// gscal (fp32 words): [0] max over rows and heads of |v_row,head|_2 (float bits, atomicMax),
// [1] the same for the segment's dO, [2] s_dO, [3] s_dS.

// out = fp16(in) for rows x cols (bf16 -> fp16, 8 values per thread and step); with
// vnorm_col0 >= 0 the per-head row norms of columns [vnorm_col0, cols) (the v section) are
// max-reduced into gscal[0].
__global__ void qkv_to_f16_kernel(const bf16* __restrict__ in, int64_t ldi, __half* __restrict__ out, int64_t ldo,
                                  int rows, int cols, int vnorm_col0, unsigned int* __restrict__ gmax) {
  // rows x (cols / 8) < 2^31 (checked by the caller): 32-bit index arithmetic
  const unsigned vpr = (unsigned)cols / 8u;
  const unsigned total = (unsigned)rows * vpr;
  for (unsigned e = blockIdx.x * blockDim.x + threadIdx.x; e < total; e += gridDim.x * blockDim.x) {
    const unsigned r = e / vpr, c = (e - r * vpr) * 8u;
    float f[8];
    unpack8(*reinterpret_cast<const uint4*>(in + (int64_t)r * ldi + c), f);
    uint4 o;
    uint32_t* ow = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      __half2 h = __floats2half2_rn(f[2 * i], f[2 * i + 1]);
      ow[i] = *reinterpret_cast<uint32_t*>(&h);
    }
    *reinterpret_cast<uint4*>(out + (int64_t)r * ldo + c) = o;
  }
  if (vnorm_col0 < 0) return;
  // per (row, v head): one warp sums the squares of the head's 128 values; the maxima are
  // reduced over the warp's rows, then over the block, then one atomicMax per block
  const int H = (cols - vnorm_col0) / 128;
  const int lane = threadIdx.x & 31;
  const unsigned nw = (unsigned)rows * (unsigned)H;
  float best = 0.f;
  for (unsigned w = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; w < nw; w += (gridDim.x * blockDim.x) >> 5) {
    const unsigned r = w / (unsigned)H, hh = w - r * (unsigned)H;
    const uint2 u = *reinterpret_cast<const uint2*>(in + (int64_t)r * ldi + vnorm_col0 + hh * 128 + lane * 4);
    const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&u);
    const float2 a = __bfloat1622float2(p2[0]), b = __bfloat1622float2(p2[1]);
    float ss = a.x * a.x + a.y * a.y + b.x * b.x + b.y * b.y;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    best = fmaxf(best, ss);
  }
  __shared__ float wmax[32];
  if (lane == 0) wmax[threadIdx.x >> 5] = best;
  __syncthreads();
  if (threadIdx.x == 0) {
    float m = 0.f;
    for (int i = 0; i < (int)(blockDim.x >> 5); ++i) m = fmaxf(m, wmax[i]);
    if (m > 0.f) atomicMax(gmax, __float_as_uint(sqrtf(m)));  // non-negative: bit order = value order
  }
}

// gscal[1] = max over the segment's valid rows and heads of |dO_row,head|_2 (dO fp32 [T, ld]).
__global__ void do_norm_max_kernel(const float* __restrict__ dO, int64_t ld, int T, int H, int s0,
                                   const int32_t* __restrict__ n_valid, int valid_mult,
                                   unsigned int* __restrict__ gscal_bits) {
  const int nv = valid_rows(n_valid, valid_mult, s0, T);
  const int lane = threadIdx.x & 31;
  const unsigned nw = (unsigned)nv * (unsigned)H;
  float best = 0.f;
  for (unsigned w = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; w < nw; w += (gridDim.x * blockDim.x) >> 5) {
    const unsigned r = w / (unsigned)H, hh = w - r * (unsigned)H;
    const float4 v = *reinterpret_cast<const float4*>(dO + (int64_t)r * ld + hh * 128 + lane * 4);
    float ss = v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    best = fmaxf(best, ss);
  }
  // one atomicMax per block (the warps' maxima reduced in shared memory first)
  __shared__ float wmax[32];
  if (lane == 0) wmax[threadIdx.x >> 5] = best;
  __syncthreads();
  if (threadIdx.x == 0) {
    float m = 0.f;
    for (int i = 0; i < (int)(blockDim.x >> 5); ++i) m = fmaxf(m, wmax[i]);
    if (m > 0.f) atomicMax(gscal_bits + 1, __float_as_uint(sqrtf(m)));
  }
}

__device__ __forceinline__ float pow2_floor(float x) {  // largest power of two <= x (x > 0, finite)
  return exp2f(floorf(log2f(x)));
}

// dO16 = fp16(dO s_dO) with s_dO the power of two that brings the largest per-head row norm
// into (2^13, 2^14]; delta[h, r] = -sum_d dO16[r, h, d] o[r, h, d] (the scaled Delta, negated;
// o = the bf16 o plus its stored rounding residual o_lo when given); s_dS = the largest power of
// two <= 1 / Vmax (so |dS s_dS| <= |dO16_i| |v_j - o_i| s_dS <= 2^14 2 Vmax s_dS <= 2^15 < 65504).
// Rows past the valid count get zeros.  gscal[2] = s_dO, gscal[3] = s_dS.
__global__ void do_to_f16_delta_kernel(const float* __restrict__ dO, int64_t ld, const bf16* __restrict__ o,
                                       const bf16* __restrict__ o_lo, int64_t ldo, __half* __restrict__ dO16,
                                       int64_t ld16,
                                       float* __restrict__ delta, int64_t delta_ld, int T, int H, int s0,
                                       const int32_t* __restrict__ n_valid, int valid_mult,
                                       float* __restrict__ gscal) {
  const int nv = valid_rows(n_valid, valid_mult, s0, T);
  const float dmax = __uint_as_float(reinterpret_cast<const unsigned int*>(gscal)[1]);
  const float vmax = __uint_as_float(reinterpret_cast<const unsigned int*>(gscal)[0]);
  // dO's largest per-head row norm (and so every element) scaled to at most 2^14: fp16's range
  // above 1 holds the rows with large gradients, and ordinary rows stay far from the subnormal
  // range (a scale to norm <= 1 put their elements near 2^-14 when a few rows dominated)
  const float s_dO = (dmax > 0.f && dmax < INFINITY) ? exp2f(14.f - ceilf(log2f(dmax))) : 1.f;
  // |dS| <= |dP - Delta| = |dO16_i . (v_j - o_i)| <= 2^14 * 2 Vmax, so 2^15 / (2^15 Vmax) keeps
  // |dS s_dS| <= 2^15 < 65504
  const float s_dS = (vmax > 0.f && vmax < INFINITY) ? fminf(pow2_floor(1.f / vmax), 0x1p60f) : 1.f;
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    gscal[2] = s_dO;
    gscal[3] = s_dS;
  }
  const int lane = threadIdx.x & 31;
  for (int64_t w = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; w < (int64_t)T * H;
       w += ((int64_t)gridDim.x * blockDim.x) >> 5) {
    const int r = (int)(w / H), hh = (int)(w - (int64_t)r * H);
    const int c = hh * 128 + lane * 4;
    float d = 0.f;
    uint2 packed = make_uint2(0u, 0u);
    if (r < nv) {
      const float4 v = *reinterpret_cast<const float4*>(dO + (int64_t)r * ld + c);
      const __half2 h01 = __floats2half2_rn(v.x * s_dO, v.y * s_dO), h23 = __floats2half2_rn(v.z * s_dO, v.w * s_dO);
      packed = make_uint2(*reinterpret_cast<const uint32_t*>(&h01), *reinterpret_cast<const uint32_t*>(&h23));
      const uint2 ob = *reinterpret_cast<const uint2*>(o + (int64_t)(s0 + r) * ldo + c);
      const __nv_bfloat162* op = reinterpret_cast<const __nv_bfloat162*>(&ob);
      float2 o01 = __bfloat1622float2(op[0]), o23 = __bfloat1622float2(op[1]);
      if (o_lo) {  // o = hi + lo (the forward's rounding residual)
        const uint2 lb = *reinterpret_cast<const uint2*>(o_lo + (int64_t)(s0 + r) * ldo + c);
        const __nv_bfloat162* lp = reinterpret_cast<const __nv_bfloat162*>(&lb);
        const float2 l01 = __bfloat1622float2(lp[0]), l23 = __bfloat1622float2(lp[1]);
        o01.x += l01.x; o01.y += l01.y; o23.x += l23.x; o23.y += l23.y;
      }
      const float2 f01 = __half22float2(h01), f23 = __half22float2(h23);
      d = f01.x * o01.x + f01.y * o01.y + f23.x * o23.x + f23.y * o23.y;
    }
    *reinterpret_cast<uint2*>(dO16 + (int64_t)r * ld16 + c) = packed;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) d += __shfl_xor_sync(0xffffffffu, d, off);
    if (lane == 0) delta[(int64_t)hh * delta_ld + r] = -d;
  }
}

__global__ void inv_freq_kernel(double* __restrict__ out, int D, double log2_theta) {
  const int i = threadIdx.x;
  if (i < D / 2) out[i] = exp2(-(double)(2 * i) / (double)D * log2_theta);
}

}  // namespace jenga
