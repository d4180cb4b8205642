// Block informativeness scoring (Jenga summary §4.2.1 Eq. (1), §4.2.3; Jenga notes §4.2).
//
// score[b, n] = sum_h sum_{j in block n} sum_{i >= j} P^h_ij,  P^h_i. = softmax_j(q_i.k_j / sqrt(D))
//
// Memory linear in S (the notes' FlashAttention-integrated scoring, §4.3).
// bf16 inputs (head_dim 128): one tcgen05 pass (score_fused_tc.cuh) that keeps, per query
// row, the log-sum-exp of every key chunk next to the row's running sum, and turns them into
// chunk masses once the row's log-sum-exp is final; a deterministic reduction over heads and
// query tiles gives the block scores.
// fp32 inputs: exact fp32 SIMT dot products in two passes (per (head, query) the row
// log-sum-exp; per (head, key) the column mass sum_i exp(s_ij - LSE_i)), then the same kind
// of fixed-order reduction.
#include "score_fused_tc.cuh"
#include "score_blockmax_tc.cuh"

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

// ------------------------------------------------------------------ block reduce (fp32 path)
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

// bf16 path: chunk width (keys) of the single-pass kernel for a block size (0: unsupported)
static int score_chunk(int blk) { return blk % 64 == 0 ? 64 : (blk % 32 == 0 ? 32 : 0); }

struct ScoreWs {  // byte offsets of the bf16 path's workspace regions
  size_t lse, part, counter, scratch, total;
  int grid;
};

static size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// bf16 block-max path: sub-tile group size for a block size (0: unsupported)
static int blockmax_group(int blk) { return (blk == 32 || blk == 64) ? blk : (blk % 128 == 0 ? 128 : 0); }

static ScoreWs score_ws_layout(int B, int S, int H, int blk) {
  ScoreWs w{};
  const int ch = score_chunk(blk);
  if (!ch) return w;
  const int nt = (S + SF_ROWS - 1) / SF_ROWS;
  const long n_items = (long)nt * H * B;
  w.grid = (int)(n_items < SF_GRID_CAP ? n_items : SF_GRID_CAP);
  w.lse = 0;
  w.part = align256((size_t)B * H * S * sizeof(float));
  w.counter = w.part + align256((size_t)B * H * nt * nt * (SF_ROWS / ch) * sizeof(float));
  w.scratch = w.counter + 256;
  w.total = w.scratch + (size_t)w.grid * sf_scratch_floats_per_cta(nt, ch) * sizeof(float);
  return w;
}

extern "C" size_t jenga_score_workspace_bytes(int B, int S, int H, int D, int blk) {
  (void)D;
  if (B < 1 || S < 1 || H < 1 || blk < 1) return 0;
  const size_t nb = (size_t)S / blk;
  size_t a = 2 * (size_t)B * H * S * sizeof(float);  // fp32 path: row LSE + column mass
  const int bg = blockmax_group(blk);
  const size_t ng = bg ? (size_t)S / bg : 0;
  size_t c = (size_t)B * (ng > nb ? ng * ng : nb * nb) * sizeof(float);  // block-max partials
  size_t d = score_ws_layout(B, S, H, blk).total;    // bf16 single pass
  size_t m = a > c ? a : c;
  return (m > d ? m : d) + 256;
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
    if (dt == JENGA_BF16) {
      const int g = blockmax_group(blk);
      if (D != 128 || !g || ldq % 8 || ldk % 8 || ((uintptr_t)q & 15) || ((uintptr_t)k & 15))
        return fail(JENGA_EUNSUPPORTED,
                    "jenga_score_blocks: bf16 block-max path needs D == 128, blk 32, 64 or a multiple of 128 and "
                    "16-byte aligned rows");
      CUtensorMap tq, tk;
      jenga_status s1 = make_tmap_bf16(&tq, q, (uint64_t)B * S, (uint64_t)H * D, ldq, 128);
      if (s1 != JENGA_OK) return s1;
      s1 = make_tmap_bf16(&tk, k, (uint64_t)B * S, (uint64_t)H * D, ldk, 128);
      if (s1 != JENGA_OK) return s1;
      const int nt = (S + 127) / 128;
      const int pairs = causal ? nt * (nt + 1) / 2 : nt * nt;
      JENGA_CUDA_TRY(
          cudaFuncSetAttribute(score_blockmax_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, BM_SMEM));
      {
        const int _ps = ::jenga::prof_begin("score_blockmax_tc", st);
        score_blockmax_tc_kernel<<<dim3(pairs, B), BM_THREADS, BM_SMEM, st>>>(
            tq, tk, S, H, g, causal ? 1 : 0, scale / (float)H, wsf);
        ::jenga::prof_end(_ps, st);
      }
      JENGA_LAUNCH_CHECK();
      {
        const int _ps = ::jenga::prof_begin("score_blockmax_colsum", st);
        score_blockmax_colsum_kernel<<<dim3((nb + 127) / 128, B), 128, 0, st>>>(wsf, nb, blk / g, causal ? 1 : 0,
                                                                                 scores);
        ::jenga::prof_end(_ps, st);
      }
      JENGA_LAUNCH_CHECK();
      return JENGA_OK;
    }
    {
    const int _ps = ::jenga::prof_begin("score_blockmax_f32", st);
    score_blockmax_f32_kernel<<<dim3(nb, nb, B), 256, 0, st>>>(q, ldq, k, ldk, S, H, D, blk, causal ? 1 : 0,
                                                              0, scale, wsf);
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
    const int ch = score_chunk(blk);
    if (D != 128 || !ch || ldq % 8 || ldk % 8 || ((uintptr_t)q & 15) || ((uintptr_t)k & 15))
      return fail(JENGA_EUNSUPPORTED,
                  "jenga_score_blocks: bf16 path needs D == 128, blk a multiple of 32 and 16-byte aligned rows");
    const ScoreWs w = score_ws_layout(B, S, H, blk);
    char* base = (char*)wsf;
    float* neg_lse = (float*)(base + w.lse);
    float* part = (float*)(base + w.part);
    float* scratch = (float*)(base + w.scratch);
    unsigned int* counter = (unsigned int*)(base + w.counter);
    JENGA_CUDA_TRY(cudaMemsetAsync(counter, 0, sizeof(unsigned int), st));
    CUtensorMap tq, tk;
    jenga_status s1 = make_tmap_bf16(&tq, q, (uint64_t)B * S, (uint64_t)H * D, ldq, SF_ROWS);
    if (s1 != JENGA_OK) return s1;
    s1 = make_tmap_bf16(&tk, k, (uint64_t)B * S, (uint64_t)H * D, ldk, SF_ROWS);
    if (s1 != JENGA_OK) return s1;
    int grid = sm_count();
    if (grid > w.grid) grid = w.grid;
    const float sl2 = SC_LOG2E * scale;
    {
      const int _ps = ::jenga::prof_begin("score_fused_tc", st);
      if (ch == 64) {
        JENGA_CUDA_TRY(
            cudaFuncSetAttribute(score_fused_tc_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, SF_SMEM));
        score_fused_tc_kernel<64><<<grid, SF_THREADS, SF_SMEM, st>>>(tq, tk, S, H, B, causal ? 1 : 0, sl2, neg_lse,
                                                                     part, scratch, counter);
      } else {
        JENGA_CUDA_TRY(
            cudaFuncSetAttribute(score_fused_tc_kernel<32>, cudaFuncAttributeMaxDynamicSharedMemorySize, SF_SMEM));
        score_fused_tc_kernel<32><<<grid, SF_THREADS, SF_SMEM, st>>>(tq, tk, S, H, B, causal ? 1 : 0, sl2, neg_lse,
                                                                     part, scratch, counter);
      }
      ::jenga::prof_end(_ps, st);
    }
    JENGA_LAUNCH_CHECK();
    {
      const int _ps = ::jenga::prof_begin("score_chunk_reduce", st);
      score_chunk_reduce_kernel<<<dim3(nb, B), 256, 0, st>>>(part, S, H, blk, ch, causal ? 1 : 0, scores);
      ::jenga::prof_end(_ps, st);
    }
    JENGA_LAUNCH_CHECK();
    return JENGA_OK;
  }
  {
  const int _ps = ::jenga::prof_begin("score_reduce", st);
  score_reduce_kernel<<<dim3(nb, B), 1024, 0, st>>>(mass, S, H, blk, scores);
  ::jenga::prof_end(_ps, st);
  }
  JENGA_LAUNCH_CHECK();
  return JENGA_OK;
}
