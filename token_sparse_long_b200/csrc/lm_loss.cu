// Segmented causal-LM loss over the vocabulary (Jenga summary §4.4.2, segment-based peak
// cutting, Fig. 10): the vocabulary-wide logits of a long sequence are the transient
// activation that sets the memory peak, so the tokens are processed in segments of
// `segment_tokens` rows and each segment's logits are dropped once its hidden-state
// gradient is formed.  Per segment [s0, s0 + T):
//   logits  = hidden[s0:s0+T] W^T                       gemm_tc, fp32 out   [T, V]
//   per row: lse = logsumexp(logits), loss_t = lse - logits[label]  (valid labels only),
//            dlogits = (softmax - onehot(label)) / n_valid as bf16            [T, V]
//   dhidden[s0:s0+T] = dlogits W                        gemm_tc, bf16 out   [T, h]
// n_valid (labels in [0, V)) is counted before the first segment; the loss is the
// fixed-order sum of the per-row losses / n_valid.  Every row depends only on itself,
// so any segmentation gives the same bits.  Peak workspace: T x V x 6 bytes plus the
// transposed W (h x V bf16).
namespace jenga {

// n_valid[0] = number of labels in [0, V) (one CTA)
__global__ void __launch_bounds__(1024) lm_count_valid_kernel(const int32_t* __restrict__ labels, int S, int V,
                                                              int32_t* __restrict__ n_valid) {
  __shared__ int s_w[32];
  int c = 0;
  for (int t = threadIdx.x; t < S; t += 1024) {
    const int l = labels[t];
    c += (l >= 0 && l < V) ? 1 : 0;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
  if ((threadIdx.x & 31) == 0) s_w[threadIdx.x >> 5] = c;
  __syncthreads();
  if (threadIdx.x == 0) {
    int tot = 0;
    for (int w = 0; w < 32; ++w) tot += s_w[w];
    *n_valid = tot;
  }
}

// One CTA per row of the segment: online max / sum over the vocabulary (8 columns per
// thread-step, 16-byte loads when V % 8 == 0), then the row's loss and its bf16
// softmax-minus-onehot row scaled by 1 / n_valid (zeros for an ignored label).
__global__ void __launch_bounds__(256) lm_ce_rows_kernel(const float* __restrict__ logits, int V,
                                                         const int32_t* __restrict__ labels,
                                                         const int32_t* __restrict__ n_valid,
                                                         float* __restrict__ row_loss, bf16* __restrict__ dlogits) {
  const int t = blockIdx.x;
  const float* z = logits + (int64_t)t * V;
  bf16* d = dlogits + (int64_t)t * V;
  const int label = labels[t];
  const bool valid = label >= 0 && label < V;
  const bool vec = (V % 8) == 0;
  float m = -INFINITY, s = 0.f;
  auto acc = [&](float x) {
    if (x > m) {
      s = s * __expf(m - x) + 1.f;
      m = x;
    } else {
      s += __expf(x - m);
    }
  };
  if (vec) {
    for (int c = threadIdx.x * 8; c < V; c += 256 * 8) {
      const float4 a = *reinterpret_cast<const float4*>(z + c), b = *reinterpret_cast<const float4*>(z + c + 4);
      acc(a.x); acc(a.y); acc(a.z); acc(a.w); acc(b.x); acc(b.y); acc(b.z); acc(b.w);
    }
  } else {
    for (int c = threadIdx.x; c < V; c += 256) acc(z[c]);
  }
  // combine (m, s) across the CTA
  __shared__ float s_m[8], s_s[8];
  __shared__ float s_lse;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float mo = __shfl_xor_sync(0xffffffffu, m, o), so = __shfl_xor_sync(0xffffffffu, s, o);
    const float mn = fmaxf(m, mo);
    s = (mn == -INFINITY) ? 0.f : s * __expf(m - mn) + so * __expf(mo - mn);
    m = mn;
  }
  if ((threadIdx.x & 31) == 0) {
    s_m[threadIdx.x >> 5] = m;
    s_s[threadIdx.x >> 5] = s;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    float mm = -INFINITY;
    for (int w = 0; w < 8; ++w) mm = fmaxf(mm, s_m[w]);
    float ss = 0.f;
    for (int w = 0; w < 8; ++w) ss += (s_m[w] == -INFINITY) ? 0.f : s_s[w] * __expf(s_m[w] - mm);
    const float lse = mm + __logf(ss);
    s_lse = lse;
    row_loss[t] = valid ? lse - z[label] : 0.f;
  }
  __syncthreads();
  const float lse = s_lse;
  const int n = *n_valid;
  const float inv = (valid && n > 0) ? 1.f / (float)n : 0.f;
  if (vec) {
    for (int c = threadIdx.x * 8; c < V; c += 256 * 8) {
      const float4 a = *reinterpret_cast<const float4*>(z + c), b = *reinterpret_cast<const float4*>(z + c + 4);
      const float x[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
      uint32_t w[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float p0 = (__expf(x[2 * i] - lse) - (c + 2 * i == label ? 1.f : 0.f)) * inv;
        const float p1 = (__expf(x[2 * i + 1] - lse) - (c + 2 * i + 1 == label ? 1.f : 0.f)) * inv;
        __nv_bfloat162 hb = __floats2bfloat162_rn(p0, p1);
        w[i] = *reinterpret_cast<uint32_t*>(&hb);
      }
      *reinterpret_cast<uint4*>(d + c) = make_uint4(w[0], w[1], w[2], w[3]);
    }
  } else {
    for (int c = threadIdx.x; c < V; c += 256)
      d[c] = __float2bfloat16_rn((__expf(z[c] - lse) - (c == label ? 1.f : 0.f)) * inv);
  }
}

// loss = (sum_t row_loss[t], fixed order, fp64) / n_valid (one CTA)
__global__ void __launch_bounds__(1024) lm_loss_reduce_kernel(const float* __restrict__ row_loss, int S,
                                                              const int32_t* __restrict__ n_valid,
                                                              float* __restrict__ loss) {
  __shared__ double s_w[32];
  const int run = (S + 1023) / 1024;
  const int lo = threadIdx.x * run, hi = min(S, lo + run);
  double a = 0.0;
  for (int t = lo; t < hi; ++t) a += (double)row_loss[t];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
  if ((threadIdx.x & 31) == 0) s_w[threadIdx.x >> 5] = a;
  __syncthreads();
  if (threadIdx.x == 0) {
    double tot = 0.0;
    for (int w = 0; w < 32; ++w) tot += s_w[w];
    const int n = *n_valid;
    *loss = n > 0 ? (float)(tot / (double)n) : 0.f;
  }
}

}  // namespace jenga

using namespace jenga;

static size_t lm_carve(void* base, int S, int h, int V, int T, bf16** wT, float** logits, bf16** dlogits,
                       float** row_loss, int32_t** n_valid) {
  Carve c(base);
  bf16* a = c.take<bf16>((size_t)h * V);
  float* b = c.take<float>((size_t)T * V);
  bf16* d = c.take<bf16>((size_t)T * V);
  float* r = c.take<float>((size_t)S);
  int32_t* n = c.take<int32_t>(4);
  if (wT) {
    *wT = a;
    *logits = b;
    *dlogits = d;
    *row_loss = r;
    *n_valid = n;
  }
  return c.used();
}

extern "C" size_t jenga_lm_loss_workspace_bytes(int S, int h, int V, int segment_tokens) {
  if (S < 1 || h < 1 || V < 1 || segment_tokens < 1) return 0;
  const int T = segment_tokens < S ? segment_tokens : S;
  return lm_carve(nullptr, S, h, V, T, nullptr, nullptr, nullptr, nullptr, nullptr);
}

extern "C" jenga_status jenga_lm_loss_segmented(const void* hidden, const void* w, const int32_t* labels, int S,
                                                int h, int V, int segment_tokens, float* loss, void* dhidden,
                                                void* ws, size_t ws_bytes, jenga_stream_t stream) {
  JENGA_CHECK_ARG(hidden && w && labels && loss && dhidden, "jenga_lm_loss_segmented: null pointer");
  JENGA_CHECK_ARG(S >= 1 && segment_tokens >= 1, "jenga_lm_loss_segmented: bad sizes S=%d segment=%d", S,
                  segment_tokens);
  JENGA_CHECK_ARG(h >= 64 && h % 64 == 0 && V >= 64 && V % 64 == 0,
                  "jenga_lm_loss_segmented: h and V must be positive multiples of 64 (h=%d V=%d)", h, V);
  JENGA_CHECK_ARG((((uintptr_t)hidden | (uintptr_t)w | (uintptr_t)dhidden) & 15) == 0,
                  "jenga_lm_loss_segmented: 16-byte aligned operands");
  const int T = segment_tokens < S ? segment_tokens : S;
  const size_t need = jenga_lm_loss_workspace_bytes(S, h, V, segment_tokens);
  if (!ws || ws_bytes < need)
    return fail(JENGA_EWORKSPACE, "jenga_lm_loss_segmented: workspace %zu < %zu", ws_bytes, need);
  cudaStream_t st = (cudaStream_t)stream;
  bf16 *wT, *dlog;
  float *logits, *row_loss;
  int32_t* n_valid;
  lm_carve(ws, S, h, V, T, &wT, &logits, &dlog, &row_loss, &n_valid);
  {
    const int _ps = ::jenga::prof_begin("lm_count_valid", st);
    lm_count_valid_kernel<<<1, 1024, 0, st>>>(labels, S, V, n_valid);
    ::jenga::prof_end(_ps, st);
  }
  JENGA_LAUNCH_CHECK();
  JENGA_TRY(transpose((const bf16*)w, h, wT, V, V, h, st));  // [V, h] -> [h, V]
  const bf16* hid = (const bf16*)hidden;
  bf16* dh = (bf16*)dhidden;
  for (int s0 = 0; s0 < S; s0 += T) {
    const int Ts = (S - s0) < T ? (S - s0) : T;
    {
      EpiParams e = epi_base(nullptr, 1, nullptr, 0);
      e.out = logits;
      e.ldo = V;
      JENGA_TRY((launch_gemm<256, EPI_STORE_F32>({hid + (size_t)s0 * h, Ts, h}, {w, V, h}, h, nullptr, nullptr, 0, Ts,
                                                 V, e, st, "gemm_lm_logits")));
    }
    {
      const int _ps = ::jenga::prof_begin("lm_ce_rows", st);
      lm_ce_rows_kernel<<<Ts, 256, 0, st>>>(logits, V, labels + s0, n_valid, row_loss + s0, dlog);
      ::jenga::prof_end(_ps, st);
    }
    JENGA_LAUNCH_CHECK();
    {
      EpiParams e = epi_base(nullptr, 1, nullptr, 0);
      e.out = dh + (size_t)s0 * h;
      e.ldo = h;
      JENGA_TRY((launch_gemm<256, EPI_STORE_BF16>({dlog, Ts, V}, {wT, h, V}, V, nullptr, nullptr, 0, Ts, h, e, st,
                                                  "gemm_lm_dhidden")));
    }
  }
  {
    const int _ps = ::jenga::prof_begin("lm_loss_reduce", st);
    lm_loss_reduce_kernel<<<1, 1024, 0, st>>>(row_loss, S, n_valid, loss);
    ::jenga::prof_end(_ps, st);
  }
  JENGA_LAUNCH_CHECK();
  return JENGA_OK;
}
