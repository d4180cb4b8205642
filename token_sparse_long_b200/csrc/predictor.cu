// Block-score predictor (Jenga notes §4.3 / Jenga summary §4.3.1, Fig. 8): a light
// MLP that maps a representative embedding of each token block (the mean of the
// block's raw layer-input rows) to an informativeness score,
//     s_n = W2 . GELU(W1 xbar_n + b1) + b2,   GELU exact (erf) form.
// Pass 1 (HBM-bound, reads X once): block means in fp32, one CTA per (block,
// 512-column slice).  Pass 2: the 2-layer MLP per block (W1 is L2-resident).
// The pages' own Q/K predictor pair (Eq. (3)) shares pass 1 and follows below.
#include "common.cuh"

namespace jenga {

constexpr int PRED_COLS = 512;  // columns per pass-1 CTA

// xbar[b, n, c] for c in the CTA's slice: 256 threads = 4 row groups x 64 uint4 columns
__global__ void __launch_bounds__(256) pred_block_mean_kernel(const bf16* __restrict__ x, int S, int h, int blk,
                                                              float* __restrict__ xbar) {
  const int n = blockIdx.x, cs = blockIdx.y, b = blockIdx.z;
  const int nb = S / blk;
  const int vc = threadIdx.x & 63, rg = threadIdx.x >> 6;
  const int c0 = cs * PRED_COLS + vc * 8;
  __shared__ float part[4][PRED_COLS];
  float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  if (c0 < h) {
    const bf16* base = x + ((int64_t)b * S + (int64_t)n * blk) * h + c0;
    for (int r = rg; r < blk; r += 4) {
      uint4 u = __ldcs(reinterpret_cast<const uint4*>(base + (int64_t)r * h));
      const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        float2 f = __bfloat1622float2(p[i]);
        acc[2 * i] += f.x;
        acc[2 * i + 1] += f.y;
      }
    }
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) part[rg][vc * 8 + i] = acc[i];
  __syncthreads();
  for (int i = threadIdx.x; i < PRED_COLS; i += 256) {
    const int c = cs * PRED_COLS + i;
    if (c < h) {
      const float s = ((part[0][i] + part[1][i]) + part[2][i]) + part[3][i];
      xbar[((int64_t)b * nb + n) * h + c] = s / (float)blk;
    }
  }
}

// One CTA per block: hidden unit j = W1[j] . xbar + b1[j] (warp per unit, lanes over h),
// then s = sum_j W2[j] GELU(hidden_j) + b2 in a fixed order.
__global__ void __launch_bounds__(256) pred_mlp_kernel(const float* __restrict__ xbar, int nb, int h,
                                                       const bf16* __restrict__ w1, const float* __restrict__ b1,
                                                       const bf16* __restrict__ w2, const float* __restrict__ b2, int m,
                                                       float* __restrict__ scores) {
  extern __shared__ float s_x[];  // h floats
  __shared__ float s_hid[256];
  const int n = blockIdx.x, b = blockIdx.y;
  const float* xb = xbar + ((int64_t)b * nb + n) * h;
  for (int i = threadIdx.x; i < h; i += 256) s_x[i] = xb[i];
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int j = warp; j < m; j += 8) {
    const bf16* wr = w1 + (int64_t)j * h;
    float acc = 0.f;
    for (int c = lane * 8; c < h; c += 256) {
      uint4 u = *reinterpret_cast<const uint4*>(wr + c);
      const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        float2 f = __bfloat1622float2(p[i]);
        acc = fmaf(f.x, s_x[c + 2 * i], acc);
        acc = fmaf(f.y, s_x[c + 2 * i + 1], acc);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) {
      const float z = acc + b1[j];
      const float gz = 0.5f * z * (1.f + erff(z * 0.70710678118654752f));
      s_hid[j] = gz * __bfloat162float(w2[j]);
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    float s = 0.f;
    for (int j = 0; j < m; ++j) s += s_hid[j];
    scores[(int64_t)b * nb + n] = s + b2[0];
  }
}

// ------------------------------------------------------------------ Q/K predictor pair
// Jenga summary §4.3.1 Eq. (3), Fig. 8: per layer a query-side and a key-side predictor,
// each three bias-free low-rank matrices with ReLU between them, applied to the block
// means; the score block (m, n) is the dot product of query block m's and key block n's
// outputs, and key block n's score is the sum of its column (causal: m >= n).
// Side pass: one CTA per (block, side), a warp per output unit of each matrix.
__global__ void __launch_bounds__(256) pred_pair_side_kernel(const float* __restrict__ xbar, int B, int nb, int h,
                                                             const bf16* __restrict__ qw1, const bf16* __restrict__ qw2,
                                                             const bf16* __restrict__ qw3, const bf16* __restrict__ kw1,
                                                             const bf16* __restrict__ kw2, const bf16* __restrict__ kw3,
                                                             int r1, int r2, int d, float* __restrict__ out) {
  extern __shared__ float s_x[];  // [h] block mean, then [r1] and [r2] activations
  float* s_a1 = s_x + h;
  float* s_a2 = s_a1 + r1;
  const int n = blockIdx.x, side = blockIdx.y, b = blockIdx.z;
  const bf16* w1 = side ? kw1 : qw1;
  const bf16* w2 = side ? kw2 : qw2;
  const bf16* w3 = side ? kw3 : qw3;
  const float* xb = xbar + ((int64_t)b * nb + n) * h;
  for (int i = threadIdx.x; i < h; i += 256) s_x[i] = xb[i];
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int j = warp; j < r1; j += 8) {  // a1 = ReLU(W1 xbar): lanes over h, 8 columns per load
    const bf16* wr = w1 + (int64_t)j * h;
    float acc = 0.f;
    for (int c = lane * 8; c < h; c += 256) {
      const uint4 u = *reinterpret_cast<const uint4*>(wr + c);
      const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 f = __bfloat1622float2(p[i]);
        acc = fmaf(f.x, s_x[c + 2 * i], acc);
        acc = fmaf(f.y, s_x[c + 2 * i + 1], acc);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) s_a1[j] = fmaxf(acc, 0.f);
  }
  __syncthreads();
  for (int j = warp; j < r2; j += 8) {  // a2 = ReLU(W2 a1)
    float acc = 0.f;
    for (int c = lane; c < r1; c += 32) acc = fmaf(__bfloat162float(w2[(int64_t)j * r1 + c]), s_a1[c], acc);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) s_a2[j] = fmaxf(acc, 0.f);
  }
  __syncthreads();
  for (int j = warp; j < d; j += 8) {  // out = W3 a2
    float acc = 0.f;
    for (int c = lane; c < r2; c += 32) acc = fmaf(__bfloat162float(w3[(int64_t)j * r2 + c]), s_a2[c], acc);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) out[(((int64_t)side * B + b) * nb + n) * d + j] = acc;
  }
}

// Column sums of the score-block matrix: key block n = blockIdx.x, query blocks m (>= n
// when causal) over the threads, fixed-order reduction.
__global__ void __launch_bounds__(256) pred_pair_scores_kernel(const float* __restrict__ qk, int B, int nb, int d,
                                                               int causal, float* __restrict__ scores) {
  const int n = blockIdx.x, b = blockIdx.y;
  const float* qh = qk + (int64_t)b * nb * d;
  const float* kh = qk + ((int64_t)B + b) * nb * d + (int64_t)n * d;
  __shared__ float s_k[64];
  __shared__ float s_w[8];
  for (int i = threadIdx.x; i < d; i += 256) s_k[i] = kh[i];
  __syncthreads();
  float part = 0.f;
  for (int m = (causal ? n : 0) + threadIdx.x; m < nb; m += 256) {
    float dot = 0.f;
    for (int i = 0; i < d; ++i) dot = fmaf(qh[(int64_t)m * d + i], s_k[i], dot);
    part += dot;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
  if ((threadIdx.x & 31) == 0) s_w[threadIdx.x >> 5] = part;
  __syncthreads();
  if (threadIdx.x == 0) {
    float t = 0.f;
    for (int w = 0; w < 8; ++w) t += s_w[w];
    scores[(int64_t)b * nb + n] = t;
  }
}

}  // namespace jenga

using namespace jenga;

extern "C" size_t jenga_predict_workspace_bytes(int B, int S, int h, int blk) {
  if (B < 1 || S < 1 || h < 1 || blk < 1) return 0;
  return (size_t)B * (S / blk) * h * sizeof(float) + 256;
}

extern "C" jenga_status jenga_predict_blocks(const void* x, int B, int S, int h, int blk, const void* w1,
                                             const float* b1, const void* w2, const float* b2, int m, float* scores,
                                             void* ws, size_t ws_bytes, jenga_stream_t stream) {
  JENGA_CHECK_ARG(x && w1 && b1 && w2 && b2 && scores, "jenga_predict_blocks: null pointer");
  JENGA_CHECK_ARG(B >= 1 && S >= 1 && blk >= 1 && S % blk == 0 && h % 8 == 0 && h <= 12288,
                  "jenga_predict_blocks: bad sizes (h %% 8 == 0, h <= 12288, S %% blk == 0)");
  JENGA_CHECK_ARG(m >= 1 && m <= 256, "jenga_predict_blocks: hidden width must be in [1, 256]");
  JENGA_CHECK_ARG(((uintptr_t)x & 15) == 0 && ((uintptr_t)w1 & 15) == 0, "jenga_predict_blocks: 16-byte alignment");
  const size_t need = jenga_predict_workspace_bytes(B, S, h, blk);
  if (!ws || ws_bytes < need) return fail(JENGA_EWORKSPACE, "jenga_predict_blocks: workspace %zu < %zu", ws_bytes, need);
  cudaStream_t st = (cudaStream_t)stream;
  float* xbar = (float*)(((uintptr_t)ws + 255) & ~(uintptr_t)255);
  const int nb = S / blk;
  {
  const int _ps = ::jenga::prof_begin("pred_block_mean", st);
  pred_block_mean_kernel<<<dim3(nb, (h + PRED_COLS - 1) / PRED_COLS, B), 256, 0, st>>>((const bf16*)x, S, h, blk, xbar);
  ::jenga::prof_end(_ps, st);
  }
  JENGA_LAUNCH_CHECK();
  const size_t smem = (size_t)h * sizeof(float);
  if (smem > 48 * 1024)
    JENGA_CUDA_TRY(cudaFuncSetAttribute(pred_mlp_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
  {
  const int _ps = ::jenga::prof_begin("pred_mlp", st);
  pred_mlp_kernel<<<dim3(nb, B), 256, smem, st>>>(xbar, nb, h, (const bf16*)w1, b1, (const bf16*)w2, b2, m, scores);
  ::jenga::prof_end(_ps, st);
  }
  JENGA_LAUNCH_CHECK();
  return JENGA_OK;
}

extern "C" size_t jenga_predict_qk_workspace_bytes(int B, int S, int h, int blk, int d) {
  if (B < 1 || S < 1 || h < 1 || blk < 1 || d < 1) return 0;
  return (size_t)B * (S / blk) * h * sizeof(float) + 256 + (size_t)2 * B * (S / blk) * d * sizeof(float) + 256;
}

extern "C" jenga_status jenga_predict_blocks_qk(const void* x, int B, int S, int h, int blk, const void* q_w1,
                                                const void* q_w2, const void* q_w3, const void* k_w1,
                                                const void* k_w2, const void* k_w3, int r1, int r2, int d, int causal,
                                                float* scores, void* ws, size_t ws_bytes, jenga_stream_t stream) {
  JENGA_CHECK_ARG(x && q_w1 && q_w2 && q_w3 && k_w1 && k_w2 && k_w3 && scores, "jenga_predict_blocks_qk: null pointer");
  JENGA_CHECK_ARG(B >= 1 && S >= 1 && blk >= 1 && S % blk == 0 && h % 8 == 0 && h <= 12288,
                  "jenga_predict_blocks_qk: bad sizes (h %% 8 == 0, h <= 12288, S %% blk == 0)");
  JENGA_CHECK_ARG(r1 >= 1 && r1 <= 1024 && r2 >= 1 && r2 <= 1024 && d >= 1 && d <= 64,
                  "jenga_predict_blocks_qk: ranks r1, r2 in [1, 1024], output width d in [1, 64]");
  JENGA_CHECK_ARG((((uintptr_t)x | (uintptr_t)q_w1 | (uintptr_t)k_w1) & 15) == 0,
                  "jenga_predict_blocks_qk: 16-byte alignment");
  const size_t need = jenga_predict_qk_workspace_bytes(B, S, h, blk, d);
  if (!ws || ws_bytes < need)
    return fail(JENGA_EWORKSPACE, "jenga_predict_blocks_qk: workspace %zu < %zu", ws_bytes, need);
  cudaStream_t st = (cudaStream_t)stream;
  const int nb = S / blk;
  float* xbar = (float*)(((uintptr_t)ws + 255) & ~(uintptr_t)255);
  float* qk = (float*)((((uintptr_t)(xbar + (size_t)B * nb * h)) + 255) & ~(uintptr_t)255);
  {
    const int _ps = ::jenga::prof_begin("pred_block_mean", st);
    pred_block_mean_kernel<<<dim3(nb, (h + PRED_COLS - 1) / PRED_COLS, B), 256, 0, st>>>((const bf16*)x, S, h, blk,
                                                                                         xbar);
    ::jenga::prof_end(_ps, st);
  }
  JENGA_LAUNCH_CHECK();
  const size_t smem = (size_t)(h + r1 + r2) * sizeof(float);
  if (smem > 48 * 1024)
    JENGA_CUDA_TRY(
        cudaFuncSetAttribute(pred_pair_side_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
  {
    const int _ps = ::jenga::prof_begin("pred_pair_side", st);
    pred_pair_side_kernel<<<dim3(nb, 2, B), 256, smem, st>>>(xbar, B, nb, h, (const bf16*)q_w1, (const bf16*)q_w2,
                                                             (const bf16*)q_w3, (const bf16*)k_w1, (const bf16*)k_w2,
                                                             (const bf16*)k_w3, r1, r2, d, qk);
    ::jenga::prof_end(_ps, st);
  }
  JENGA_LAUNCH_CHECK();
  {
    const int _ps = ::jenga::prof_begin("pred_pair_scores", st);
    pred_pair_scores_kernel<<<dim3(nb, B), 256, 0, st>>>(qk, B, nb, d, causal ? 1 : 0, scores);
    ::jenga::prof_end(_ps, st);
  }
  JENGA_LAUNCH_CHECK();
  return JENGA_OK;
}
