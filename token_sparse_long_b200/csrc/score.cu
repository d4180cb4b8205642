// Block informativeness scoring (Jenga summary §4.2.1 Eq. (1), §4.2.3; Jenga notes §4.2).
//
// score[b, n] = sum_h sum_{j in block n} sum_{i >= j} P^h_ij,  P^h_i. = softmax_j(q_i.k_j / sqrt(D))
//
// Two passes, memory linear in S (the notes' FlashAttention-integrated scoring, §4.3):
//   pass 1: per (head, query) the row log-sum-exp of the causal logits;
//   pass 2: per (head, key) the column mass sum_i exp(s_ij - LSE_i);
//   reduce: per block, sum over its keys and over heads in a fixed order (deterministic).
// fp32 inputs: exact fp32 SIMT dot products.  bf16 inputs (head_dim 128): tensor-core
// tiles of 64 queries x 64 keys.
#include "attn_frag.cuh"
#include "score_tc.cuh"
#include "score_mass_tc.cuh"

namespace jenga {

constexpr float SC_LOG2E = 1.4426950408889634f;
constexpr float SC_LN2 = 0.6931471805599453f;

// ------------------------------------------------------------------ fp32 SIMT path
__global__ void __launch_bounds__(256) score_lse_f32_kernel(const float* __restrict__ q, int64_t ldq,
                                                            const float* __restrict__ k, int64_t ldk, int S, int H,
                                                            int D, int causal, float scale,
                                                            float* __restrict__ lse) {
  __shared__ float sq[8][128];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int i = blockIdx.x * 8 + warp, h = blockIdx.y, b = blockIdx.z;
  if (i >= S) return;
  const float* qi = q + ((int64_t)b * S + i) * ldq + h * D;
  for (int d = lane; d < D; d += 32) sq[warp][d] = qi[d];
  __syncwarp();
  const float* kb = k + (int64_t)b * S * ldk + h * D;
  const int jend = causal ? i + 1 : S;
  float m = -INFINITY, l = 0.f;
  for (int j = lane; j < jend; j += 32) {
    const float4* kr = reinterpret_cast<const float4*>(kb + (int64_t)j * ldk);
    float dot = 0.f;
    for (int d4 = 0; d4 < D / 4; ++d4) {
      float4 kv = kr[d4];
      dot = fmaf(sq[warp][4 * d4], kv.x, dot);
      dot = fmaf(sq[warp][4 * d4 + 1], kv.y, dot);
      dot = fmaf(sq[warp][4 * d4 + 2], kv.z, dot);
      dot = fmaf(sq[warp][4 * d4 + 3], kv.w, dot);
    }
    const float s = dot * scale;
    if (s > m) {
      l = l * expf(m - s) + 1.f;
      m = s;
    } else {
      l += expf(s - m);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float m2 = __shfl_xor_sync(0xffffffffu, m, o);
    const float l2 = __shfl_xor_sync(0xffffffffu, l, o);
    const float mn = fmaxf(m, m2);
    l = (mn == -INFINITY) ? 0.f : l * expf(m - mn) + l2 * expf(m2 - mn);
    m = mn;
  }
  if (lane == 0) lse[((int64_t)b * H + h) * S + i] = m + logf(l);
}

__global__ void __launch_bounds__(256) score_mass_f32_kernel(const float* __restrict__ q, int64_t ldq,
                                                             const float* __restrict__ k, int64_t ldk, int S, int H,
                                                             int D, int causal, float scale,
                                                             const float* __restrict__ lse,
                                                             float* __restrict__ mass) {
  __shared__ float sk[8][128];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int j = blockIdx.x * 8 + warp, h = blockIdx.y, b = blockIdx.z;
  if (j >= S) return;
  const float* kj = k + ((int64_t)b * S + j) * ldk + h * D;
  for (int d = lane; d < D; d += 32) sk[warp][d] = kj[d];
  __syncwarp();
  const float* qb = q + (int64_t)b * S * ldq + h * D;
  const float* lb = lse + ((int64_t)b * H + h) * S;
  float acc = 0.f;
  for (int i = (causal ? j : 0) + lane; i < S; i += 32) {
    const float4* qr = reinterpret_cast<const float4*>(qb + (int64_t)i * ldq);
    float dot = 0.f;
    for (int d4 = 0; d4 < D / 4; ++d4) {
      float4 qv = qr[d4];
      dot = fmaf(qv.x, sk[warp][4 * d4], dot);
      dot = fmaf(qv.y, sk[warp][4 * d4 + 1], dot);
      dot = fmaf(qv.z, sk[warp][4 * d4 + 2], dot);
      dot = fmaf(qv.w, sk[warp][4 * d4 + 3], dot);
    }
    acc += expf(dot * scale - lb[i]);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (lane == 0) mass[((int64_t)b * H + h) * S + j] = acc;
}

// ------------------------------------------------------------------ bf16 tensor-core path
// pass 1: 64 query rows per CTA (4 warps x 16), key tiles streamed, online max / sum.
__global__ void __launch_bounds__(128) score_lse_bf16_kernel(const bf16* __restrict__ q, int64_t ldq,
                                                             const bf16* __restrict__ k, int64_t ldk, int S, int H,
                                                             int causal, float scale_log2,
                                                             float* __restrict__ lse) {
  extern __shared__ __align__(128) uint8_t sm[];
  const int h = blockIdx.y, b = blockIdx.z;
  const int qt = gridDim.x - 1 - blockIdx.x;
  const int q0 = qt * AT_ROWS;
  const bf16* qh = q + (int64_t)b * S * ldq + h * AT_D;
  const bf16* kh = k + (int64_t)b * S * ldk + h * AT_D;
  uint8_t* sQ = sm;
  uint8_t* sK[2] = {sm + AT_TILE_BYTES, sm + 2 * AT_TILE_BYTES};
  load_tile_async(sQ, qh, ldq, q0, S);
  load_tile_async(sK[0], kh, ldk, 0, S);
  cp_async_commit();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const int row0 = q0 + warp * 16 + g, row1 = row0 + 8;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  uint32_t qa[8][4];
  const int nkt = causal ? qt + 1 : S / AT_ROWS;
  for (int kt = 0; kt < nkt; ++kt) {
    if (kt + 1 < nkt) {
      load_tile_async(sK[(kt + 1) & 1], kh, ldk, (kt + 1) * AT_ROWS, S);
      cp_async_commit();
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    if (kt == 0) {
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) ld_a(sQ, warp * 16, ks * 16, qa[ks]);
    }
    float s[8][4];
    mm_regs_x_rowsT(qa, sK[kt & 1], s);
    const bool diag = causal && (kt == qt);
    float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int col = kt * AT_ROWS + j * 8 + 2 * t + e;
        s[j][e] = (!diag || col <= row0) ? s[j][e] * scale_log2 : -INFINITY;
        s[j][2 + e] = (!diag || col <= row1) ? s[j][2 + e] * scale_log2 : -INFINITY;
        mx0 = fmaxf(mx0, s[j][e]);
        mx1 = fmaxf(mx1, s[j][2 + e]);
      }
    }
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
    const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
    l0 *= exp2f(m0 - mn0);
    l1 *= exp2f(m1 - mn1);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      l0 += exp2f(s[j][0] - mn0) + exp2f(s[j][1] - mn0);
      l1 += exp2f(s[j][2] - mn1) + exp2f(s[j][3] - mn1);
    }
    m0 = mn0;
    m1 = mn1;
    __syncthreads();
  }
  l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
  if (t == 0) {
    float* lb = lse + ((int64_t)b * H + h) * S;
    lb[row0] = (m0 + log2f(l0)) * SC_LN2;
    lb[row1] = (m1 + log2f(l1)) * SC_LN2;
  }
}

// pass 2: 64 keys per CTA (K fragments in registers), query tiles streamed;
// each key accumulates exp(s_ij - LSE_i) over the queries i it is visible to.
__global__ void __launch_bounds__(128) score_mass_bf16_kernel(const bf16* __restrict__ q, int64_t ldq,
                                                              const bf16* __restrict__ k, int64_t ldk, int S, int H,
                                                              int causal, float scale_log2,
                                                              const float* __restrict__ lse,
                                                              float* __restrict__ mass) {
  extern __shared__ __align__(128) uint8_t sm[];
  __shared__ float sL[2][AT_ROWS];
  const int h = blockIdx.y, b = blockIdx.z;
  const int kt = blockIdx.x;  // early key tiles see the most queries: launched first
  const int k0 = kt * AT_ROWS;
  const bf16* qh = q + (int64_t)b * S * ldq + h * AT_D;
  const bf16* kh = k + (int64_t)b * S * ldk + h * AT_D;
  const float* lb = lse + ((int64_t)b * H + h) * S;
  uint8_t* sK = sm;
  uint8_t* sQ[2] = {sm + AT_TILE_BYTES, sm + 2 * AT_TILE_BYTES};
  const int qt_begin = causal ? kt : 0;
  const int qt_end = S / AT_ROWS;
  load_tile_async(sK, kh, ldk, k0, S);
  load_tile_async(sQ[0], qh, ldq, qt_begin * AT_ROWS, S);
  if (threadIdx.x < AT_ROWS) sL[0][threadIdx.x] = lb[qt_begin * AT_ROWS + threadIdx.x] * SC_LOG2E;
  cp_async_commit();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const int krow0 = k0 + warp * 16 + g, krow1 = krow0 + 8;
  float acc0 = 0.f, acc1 = 0.f;
  uint32_t ka[8][4];
  for (int qt = qt_begin; qt < qt_end; ++qt) {
    const int buf = (qt - qt_begin) & 1;
    if (qt + 1 < qt_end) {
      load_tile_async(sQ[buf ^ 1], qh, ldq, (qt + 1) * AT_ROWS, S);
      if (threadIdx.x < AT_ROWS) sL[buf ^ 1][threadIdx.x] = lb[(qt + 1) * AT_ROWS + threadIdx.x] * SC_LOG2E;
      cp_async_commit();
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    if (qt == qt_begin) {
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) ld_a(sK, warp * 16, ks * 16, ka[ks]);
    }
    float s[8][4];
    mm_regs_x_rowsT(ka, sQ[buf], s);
    const bool diag = causal && (qt == kt);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int cl = j * 8 + 2 * t + e;
        const int col = qt * AT_ROWS + cl;
        const float L = sL[buf][cl];
        acc0 += (!diag || col >= krow0) ? exp2f(s[j][e] * scale_log2 - L) : 0.f;
        acc1 += (!diag || col >= krow1) ? exp2f(s[j][2 + e] * scale_log2 - L) : 0.f;
      }
    }
    __syncthreads();
  }
  acc0 += __shfl_xor_sync(0xffffffffu, acc0, 1);
  acc0 += __shfl_xor_sync(0xffffffffu, acc0, 2);
  acc1 += __shfl_xor_sync(0xffffffffu, acc1, 1);
  acc1 += __shfl_xor_sync(0xffffffffu, acc1, 2);
  if (t == 0) {
    float* mb = mass + ((int64_t)b * H + h) * S;
    mb[krow0] = acc0;
    mb[krow1] = acc1;
  }
}

// ------------------------------------------------------------------ block reduce (both paths)
// scores[b, n] = sum over the block's keys of (sum_h mass[b, h, key]) ; fixed order.
__global__ void __launch_bounds__(1024) score_reduce_kernel(const float* __restrict__ mass, int S, int H, int blk,
                                                            float* __restrict__ scores) {
  __shared__ float red[1024];
  const int nb = S / blk, n = blockIdx.x, b = blockIdx.y;
  float acc = 0.f;
  for (int i = threadIdx.x; i < blk; i += 1024) {
    float s = 0.f;
    for (int h = 0; h < H; ++h) s += mass[((int64_t)b * H + h) * S + (int64_t)n * blk + i];
    acc += s;
  }
  red[threadIdx.x] = acc;
  __syncthreads();
  for (int o = 512; o > 0; o >>= 1) {
    if (threadIdx.x < o) red[threadIdx.x] += red[threadIdx.x + o];
    __syncthreads();
  }
  if (threadIdx.x == 0) scores[(int64_t)b * nb + n] = red[0];
}

// ------------------------------------------------------------------ paper block-max (Eq. 2)
// score[b, n] = sum_m max_{(i,j) in block (m,n), j <= i} sum_h max(q_i.k_j / sqrt(D), 0) / H
// fp32 SIMT, one CTA per (query block m, key block n); intended for the small
// diagnostic workloads (cost S^2 * H * D).
__global__ void __launch_bounds__(256) score_blockmax_f32_kernel(const void* __restrict__ qv, int64_t ldq,
                                                                 const void* __restrict__ kv, int64_t ldk, int S,
                                                                 int H, int D, int blk, int causal, int is_bf16,
                                                                 float scale, float* __restrict__ part) {
  const int m = blockIdx.x, n = blockIdx.y, b = blockIdx.z;
  const int nb = S / blk;
  __shared__ float red[256];
  float best = -1.f;  // every aggregated value is >= 0; -1 marks "no causal entry"
  if (!causal || n <= m) {
    for (int e = threadIdx.x; e < blk * blk; e += 256) {
      const int i = m * blk + e / blk, j = n * blk + e % blk;
      if (causal && j > i) continue;
      float tot = 0.f;
      for (int hh = 0; hh < H; ++hh) {
        float dot = 0.f;
        for (int d = 0; d < D; ++d) {
          float a, c;
          if (is_bf16) {
            a = __bfloat162float(((const bf16*)qv)[((int64_t)b * S + i) * ldq + hh * D + d]);
            c = __bfloat162float(((const bf16*)kv)[((int64_t)b * S + j) * ldk + hh * D + d]);
          } else {
            a = ((const float*)qv)[((int64_t)b * S + i) * ldq + hh * D + d];
            c = ((const float*)kv)[((int64_t)b * S + j) * ldk + hh * D + d];
          }
          dot = fmaf(a, c, dot);
        }
        dot *= scale;
        if (dot > 0.f) tot += dot;
      }
      best = fmaxf(best, tot / (float)H);
    }
  }
  red[threadIdx.x] = best;
  __syncthreads();
  for (int o = 128; o > 0; o >>= 1) {
    if (threadIdx.x < o) red[threadIdx.x] = fmaxf(red[threadIdx.x], red[threadIdx.x + o]);
    __syncthreads();
  }
  if (threadIdx.x == 0) part[((int64_t)b * nb + n) * nb + m] = red[0];
}

__global__ void score_blockmax_sum_kernel(const float* __restrict__ part, int nb, float* __restrict__ scores) {
  const int n = blockIdx.x * blockDim.x + threadIdx.x, b = blockIdx.y;
  if (n >= nb) return;
  float s = 0.f;
  for (int m = 0; m < nb; ++m) {
    const float v = part[((int64_t)b * nb + n) * nb + m];
    if (v >= 0.f) s += v;
  }
  scores[(int64_t)b * nb + n] = s;
}

}  // namespace jenga

using namespace jenga;

extern "C" size_t jenga_score_workspace_bytes(int B, int S, int H, int D, int blk) {
  (void)D;
  if (B < 1 || S < 1 || H < 1 || blk < 1) return 0;
  const size_t nb = (size_t)S / blk;
  size_t a = 2 * (size_t)B * H * S * sizeof(float);  // LSE + column mass
  size_t c = (size_t)B * nb * nb * sizeof(float);    // block-max partials
  return (a > c ? a : c) + 256;
}

extern "C" jenga_status jenga_score_blocks(const void* q, int64_t ldq, const void* k, int64_t ldk, int B, int S,
                                           int H, int D, int blk, int causal, jenga_dtype dt, jenga_score_mode mode,
                                           float* scores, void* ws, size_t ws_bytes, jenga_stream_t stream) {
  JENGA_CHECK_ARG(q && k && scores, "jenga_score_blocks: null pointer");
  JENGA_CHECK_ARG(B >= 1 && S >= 1 && H >= 1 && D >= 4 && blk >= 1 && S % blk == 0,
                  "jenga_score_blocks: bad sizes B=%d S=%d H=%d D=%d blk=%d", B, S, H, D, blk);
  JENGA_CHECK_ARG(ldq >= (int64_t)H * D && ldk >= (int64_t)H * D, "jenga_score_blocks: row pitch < H*D");
  JENGA_CHECK_ARG(dt == JENGA_F32 || dt == JENGA_BF16, "jenga_score_blocks: dtype");
  JENGA_CHECK_ARG(mode == JENGA_SCORE_SOFTMAX_MASS || mode == JENGA_SCORE_PAPER_BLOCKMAX,
                  "jenga_score_blocks: mode");
  const size_t need = jenga_score_workspace_bytes(B, S, H, D, blk);
  if (!ws || ws_bytes < need) return fail(JENGA_EWORKSPACE, "jenga_score_blocks: workspace %zu < %zu", ws_bytes, need);
  cudaStream_t st = (cudaStream_t)stream;
  float* wsf = (float*)(((uintptr_t)ws + 255) & ~(uintptr_t)255);
  const float scale = 1.f / sqrtf((float)D);
  const int nb = S / blk;
  if (mode == JENGA_SCORE_PAPER_BLOCKMAX) {
    {
    const int _ps = ::jenga::prof_begin("score_blockmax_f32", st);
    score_blockmax_f32_kernel<<<dim3(nb, nb, B), 256, 0, st>>>(q, ldq, k, ldk, S, H, D, blk, causal ? 1 : 0,
                                                              dt == JENGA_BF16 ? 1 : 0, scale, wsf);
    ::jenga::prof_end(_ps, st);
    }
    JENGA_LAUNCH_CHECK();
    {
    const int _ps = ::jenga::prof_begin("score_blockmax_sum", st);
    score_blockmax_sum_kernel<<<dim3((nb + 127) / 128, B), 128, 0, st>>>(wsf, nb, scores);
    ::jenga::prof_end(_ps, st);
    }
    JENGA_LAUNCH_CHECK();
    return JENGA_OK;
  }
  float* lse = wsf;
  float* mass = wsf + (size_t)B * H * S;
  if (dt == JENGA_F32) {
    JENGA_CHECK_ARG(D % 4 == 0 && D <= 128 && ldq % 4 == 0 && ldk % 4 == 0 &&
                        ((uintptr_t)q & 15) == 0 && ((uintptr_t)k & 15) == 0,
                    "jenga_score_blocks: fp32 path needs D % 4 == 0, D <= 128 and 16-byte aligned rows");
    dim3 g((S + 7) / 8, H, B);
    {
    const int _ps = ::jenga::prof_begin("score_lse_f32", st);
    score_lse_f32_kernel<<<g, 256, 0, st>>>((const float*)q, ldq, (const float*)k, ldk, S, H, D, causal, scale, lse);
    ::jenga::prof_end(_ps, st);
    }
    JENGA_LAUNCH_CHECK();
    {
    const int _ps = ::jenga::prof_begin("score_mass_f32", st);
    score_mass_f32_kernel<<<g, 256, 0, st>>>((const float*)q, ldq, (const float*)k, ldk, S, H, D, causal, scale, lse,
                                             mass);
    ::jenga::prof_end(_ps, st);
    }
    JENGA_LAUNCH_CHECK();
  } else {
    if (D != AT_D || S % AT_ROWS || ldq % 8 || ldk % 8 || ((uintptr_t)q & 15) || ((uintptr_t)k & 15))
      return fail(JENGA_EUNSUPPORTED, "jenga_score_blocks: bf16 path needs D == 128, S % 64 == 0, aligned rows");
    const float sl2 = SC_LOG2E * scale;
    if (S % SCT_ROWS == 0) {
      // tcgen05 path: 128-token tiles, TMA-fed, accumulators in tensor memory
      CUtensorMap tq, tk;
      jenga_status s1 = make_tmap_bf16(&tq, q, (uint64_t)B * S, (uint64_t)H * D, ldq, SCT_ROWS);
      if (s1 != JENGA_OK) return s1;
      s1 = make_tmap_bf16(&tk, k, (uint64_t)B * S, (uint64_t)H * D, ldk, SCT_ROWS);
      if (s1 != JENGA_OK) return s1;
      JENGA_CUDA_TRY(cudaFuncSetAttribute(score_lse_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SCT_SMEM));
      JENGA_CUDA_TRY(cudaFuncSetAttribute(score_mass_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMT_SMEM));
      dim3 gt(S / SCT_ROWS, H, B);
      {
        const int _ps = ::jenga::prof_begin("score_lse_tc", st);
        score_lse_tc_kernel<<<gt, SCT_THREADS, SCT_SMEM, st>>>(tq, tk, S, H, causal ? 1 : 0, sl2, lse);
        ::jenga::prof_end(_ps, st);
      }
      JENGA_LAUNCH_CHECK();
      {
        const int _ps = ::jenga::prof_begin("score_mass_tc", st);
        score_mass_tc_kernel<<<gt, SMT_THREADS, SMT_SMEM, st>>>(tq, tk, S, H, causal ? 1 : 0, sl2, lse, mass);
        ::jenga::prof_end(_ps, st);
      }
      JENGA_LAUNCH_CHECK();
      {
        const int _ps = ::jenga::prof_begin("score_reduce", st);
        score_reduce_kernel<<<dim3(nb, B), 1024, 0, st>>>(mass, S, H, blk, scores);
        ::jenga::prof_end(_ps, st);
      }
      JENGA_LAUNCH_CHECK();
      return JENGA_OK;
    }
    dim3 g(S / AT_ROWS, H, B);
    JENGA_CUDA_TRY(
        cudaFuncSetAttribute(score_lse_bf16_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 3 * AT_TILE_BYTES));
    JENGA_CUDA_TRY(
        cudaFuncSetAttribute(score_mass_bf16_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 3 * AT_TILE_BYTES));
    {
    const int _ps = ::jenga::prof_begin("score_lse_bf16", st);
    score_lse_bf16_kernel<<<g, 128, 3 * AT_TILE_BYTES, st>>>((const bf16*)q, ldq, (const bf16*)k, ldk, S, H,
                                                              causal ? 1 : 0, sl2, lse);
    ::jenga::prof_end(_ps, st);
    }
    JENGA_LAUNCH_CHECK();
    {
    const int _ps = ::jenga::prof_begin("score_mass_bf16", st);
    score_mass_bf16_kernel<<<g, 128, 3 * AT_TILE_BYTES, st>>>((const bf16*)q, ldq, (const bf16*)k, ldk, S, H,
                                                               causal ? 1 : 0, sl2, lse, mass);
    ::jenga::prof_end(_ps, st);
    }
    JENGA_LAUNCH_CHECK();
  }
  {
  const int _ps = ::jenga::prof_begin("score_reduce", st);
  score_reduce_kernel<<<dim3(nb, B), 1024, 0, st>>>(mass, S, H, blk, scores);
  ::jenga::prof_end(_ps, st);
  }
  JENGA_LAUNCH_CHECK();
  return JENGA_OK;
}
