// Causal softmax attention over the retained tokens: forward, and backward split
// into a dQ pass and a dK/dV pass (no atomics; deterministic).
//
// Retained tokens are compact rows 0..n-1 in ascending original order, so causal
// attention among them is the lower triangle in compact index (eliminated tokens are
// neither queries nor keys).  head_dim 128; q/k/v rows have pitch ld elements and the
// head h occupies columns [h*128, h*128+128).
//
// Backward (segment-wise, Jenga summary §4.4.2): the dQ pass covers the query rows
// of one segment; the dK/dV pass adds that segment's query contribution into fp32
// accumulators for keys [0, segment end).  Processing segments last-first completes
// a segment's key gradients exactly when its own queries have been processed.
#include "attn_frag.cuh"
#include "attn_tc.cuh"
#include "attn_bwd_tc.cuh"

namespace jenga {

constexpr float LOG2E = 1.4426950408889634f;

__device__ __forceinline__ int attn_rows(const int32_t* n_valid, int mult, int cap) {
  int n = n_valid ? (*n_valid) * mult : cap;
  return n < cap ? n : cap;
}

// ------------------------------------------------------------------ backward helpers
// delta[h, r] = -sum_d dO[r, h, d] * O[r, h, d] for rows r in [0, T) (negated: the
// backward adds it to dP)
__global__ void attn_delta_kernel(const bf16* __restrict__ dO, int64_t ld_do, const bf16* __restrict__ o,
                                  int64_t ldo, float* __restrict__ delta, int64_t delta_ld, int T, int H) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (warp >= T * H) return;
  const int r = warp / H, h = warp - r * H;
  const uint2 a = *reinterpret_cast<const uint2*>(dO + (int64_t)r * ld_do + h * AT_D + lane * 4);
  const uint2 b = *reinterpret_cast<const uint2*>(o + (int64_t)r * ldo + h * AT_D + lane * 4);
  const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&a);
  const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&b);
  float2 x0 = __bfloat1622float2(a2[0]), x1 = __bfloat1622float2(a2[1]);
  float2 y0 = __bfloat1622float2(b2[0]), y1 = __bfloat1622float2(b2[1]);
  float s = x0.x * y0.x + x0.y * y0.y + x1.x * y1.x + x1.y * y1.y;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
  if (lane == 0) delta[(int64_t)h * delta_ld + r] = -s;
}

// dQ for the query rows [s0, s0 + gridDim.x*64) (segment), keys [0, q tile end).
// dq_out rows are segment-local: dq_out[(r - s0) * ld_dq + h*128 + d] (fp32, scaled by 1/sqrt(D)).
__global__ void __launch_bounds__(128) attn_bwd_dq_kernel(
    const bf16* __restrict__ q, const bf16* __restrict__ k, const bf16* __restrict__ v, int64_t ld,
    const bf16* __restrict__ dO, int64_t ld_do, const float* __restrict__ lse, int64_t lse_ld,
    const float* __restrict__ delta, int64_t delta_ld, float* __restrict__ dq_out, int64_t ld_dq, int s0,
    const int32_t* __restrict__ n_valid, int valid_mult, int n_cap, float scale_log2, float scale) {
  extern __shared__ __align__(128) uint8_t sm[];
  const int h = blockIdx.y;
  const int n = attn_rows(n_valid, valid_mult, n_cap);
  const int qt = s0 / AT_ROWS + (gridDim.x - 1 - blockIdx.x);
  const int q0 = qt * AT_ROWS;
  if (q0 >= n) return;
  const bf16* qh = q + h * AT_D;
  const bf16* kh = k + h * AT_D;
  const bf16* vh = v + h * AT_D;
  uint8_t* sQ = sm;
  uint8_t* sO = sm + AT_TILE_BYTES;  // dO tile (segment-local rows)
  uint8_t* sK[2] = {sm + 2 * AT_TILE_BYTES, sm + 4 * AT_TILE_BYTES};
  uint8_t* sV[2] = {sm + 3 * AT_TILE_BYTES, sm + 5 * AT_TILE_BYTES};
  load_tile_async(sQ, qh, ld, q0, n);
  load_tile_async(sO, dO + h * AT_D, ld_do, q0 - s0, n - s0);
  load_tile_async(sK[0], kh, ld, 0, n);
  load_tile_async(sV[0], vh, ld, 0, n);
  cp_async_commit();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const int row0 = q0 + warp * 16 + g, row1 = row0 + 8;
  // both stored negated (log2 units for the log-sum-exp)
  const float L0 = -lse[(int64_t)h * lse_ld + row0], L1 = -lse[(int64_t)h * lse_ld + row1];
  const float D0 = -delta[(int64_t)h * delta_ld + row0 - s0], D1 = -delta[(int64_t)h * delta_ld + row1 - s0];
  float dq[16][4];
#pragma unroll
  for (int i = 0; i < 16; ++i) dq[i][0] = dq[i][1] = dq[i][2] = dq[i][3] = 0.f;
  uint32_t qa[8][4], oa[8][4];
  const int nkt = qt + 1;
  for (int kt = 0; kt < nkt; ++kt) {
    if (kt + 1 < nkt) {
      load_tile_async(sK[(kt + 1) & 1], kh, ld, (kt + 1) * AT_ROWS, n);
      load_tile_async(sV[(kt + 1) & 1], vh, ld, (kt + 1) * AT_ROWS, n);
      cp_async_commit();
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    if (kt == 0) {
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        ld_a(sQ, warp * 16, ks * 16, qa[ks]);
        ld_a(sO, warp * 16, ks * 16, oa[ks]);
      }
    }
    float p[8][4], dp[8][4];
    mm_regs_x_rowsT(qa, sK[kt & 1], p);
    mm_regs_x_rowsT(oa, sV[kt & 1], dp);
    const bool diag = (kt == qt);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int col = kt * AT_ROWS + j * 8 + 2 * t + e;
        const float p0 = (!diag || col <= row0) ? exp2f(p[j][e] * scale_log2 - L0) : 0.f;
        const float p1 = (!diag || col <= row1) ? exp2f(p[j][2 + e] * scale_log2 - L1) : 0.f;
        p[j][e] = p0 * (dp[j][e] - D0);
        p[j][2 + e] = p1 * (dp[j][2 + e] - D1);
      }
    }
    mm_p_x_cols(p, sK[kt & 1], dq);
    __syncthreads();
  }
  float* d0 = dq_out + (int64_t)(row0 - s0) * ld_dq + h * AT_D;
  float* d1 = dq_out + (int64_t)(row1 - s0) * ld_dq + h * AT_D;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    *reinterpret_cast<float2*>(d0 + i * 8 + 2 * t) = make_float2(dq[i][0] * scale, dq[i][1] * scale);
    *reinterpret_cast<float2*>(d1 + i * 8 + 2 * t) = make_float2(dq[i][2] * scale, dq[i][3] * scale);
  }
}

// dK, dV contributions of the query rows [s0, s1) to keys [0, s1), added into fp32
// accumulators dk_acc / dv_acc [n_cap, H*128] (pitch ld_acc).  One CTA per key tile.
__global__ void __launch_bounds__(128) attn_bwd_dkdv_kernel(
    const bf16* __restrict__ q, const bf16* __restrict__ k, const bf16* __restrict__ v, int64_t ld,
    const bf16* __restrict__ dO, int64_t ld_do, const float* __restrict__ lse, int64_t lse_ld,
    const float* __restrict__ delta, int64_t delta_ld, float* __restrict__ dk_acc, float* __restrict__ dv_acc,
    int64_t ld_acc, int s0, int s1, const int32_t* __restrict__ n_valid, int valid_mult, int n_cap,
    float scale_log2, float scale) {
  extern __shared__ __align__(128) uint8_t sm[];
  __shared__ float sL[2][AT_ROWS], sD[2][AT_ROWS];
  const int h = blockIdx.y;
  const int n = attn_rows(n_valid, valid_mult, n_cap);
  const int kt = blockIdx.x;
  const int k0 = kt * AT_ROWS;
  const int send = min(s1, n);
  if (k0 >= send || s0 >= send) return;
  const int qt_begin = max(kt, s0 / AT_ROWS);
  const int qt_end = (send + AT_ROWS - 1) / AT_ROWS;
  if (qt_begin >= qt_end) return;
  const bf16* qh = q + h * AT_D;
  uint8_t* sK = sm;
  uint8_t* sV = sm + AT_TILE_BYTES;
  uint8_t* sQ[2] = {sm + 2 * AT_TILE_BYTES, sm + 4 * AT_TILE_BYTES};
  uint8_t* sO[2] = {sm + 3 * AT_TILE_BYTES, sm + 5 * AT_TILE_BYTES};
  load_tile_async(sK, k + h * AT_D, ld, k0, n);
  load_tile_async(sV, v + h * AT_D, ld, k0, n);
  auto load_q = [&](int qt, int buf) {
    load_tile_async(sQ[buf], qh, ld, qt * AT_ROWS, n);
    load_tile_async(sO[buf], dO + h * AT_D, ld_do, qt * AT_ROWS - s0, n - s0);
    if (threadIdx.x < AT_ROWS) {
      const int r = qt * AT_ROWS + threadIdx.x;
      sL[buf][threadIdx.x] = (r < n) ? -lse[(int64_t)h * lse_ld + r] : 0.f;  // stored negated, log2 units
      sD[buf][threadIdx.x] = (r < n) ? -delta[(int64_t)h * delta_ld + r - s0] : 0.f;
    }
  };
  load_q(qt_begin, 0);
  cp_async_commit();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const int krow0 = k0 + warp * 16 + g, krow1 = krow0 + 8;
  float dk[16][4], dv[16][4];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    dk[i][0] = dk[i][1] = dk[i][2] = dk[i][3] = 0.f;
    dv[i][0] = dv[i][1] = dv[i][2] = dv[i][3] = 0.f;
  }
  for (int qt = qt_begin; qt < qt_end; ++qt) {
    const int buf = (qt - qt_begin) & 1;
    if (qt + 1 < qt_end) {
      load_q(qt + 1, buf ^ 1);
      cp_async_commit();
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    float p[8][4], dp[8][4];
    mm_rows_x_rowsT(sK, warp * 16, sQ[buf], p);
    const bool diag = (qt == kt);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int cl = j * 8 + 2 * t + e;
        const int col = qt * AT_ROWS + cl;
        const float L = sL[buf][cl];
        p[j][e] = (!diag || col >= krow0) ? exp2f(p[j][e] * scale_log2 - L) : 0.f;
        p[j][2 + e] = (!diag || col >= krow1) ? exp2f(p[j][2 + e] * scale_log2 - L) : 0.f;
      }
    }
    mm_p_x_cols(p, sO[buf], dv);
    mm_rows_x_rowsT(sV, warp * 16, sO[buf], dp);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const float Dv = sD[buf][j * 8 + 2 * t + e];
        p[j][e] *= (dp[j][e] - Dv);
        p[j][2 + e] *= (dp[j][2 + e] - Dv);
      }
    }
    mm_p_x_cols(p, sQ[buf], dk);
    __syncthreads();
  }
  float* a0 = dk_acc + (int64_t)krow0 * ld_acc + h * AT_D;
  float* a1 = dk_acc + (int64_t)krow1 * ld_acc + h * AT_D;
  float* b0 = dv_acc + (int64_t)krow0 * ld_acc + h * AT_D;
  float* b1 = dv_acc + (int64_t)krow1 * ld_acc + h * AT_D;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const int c = i * 8 + 2 * t;
    float2 x;
    x = *reinterpret_cast<float2*>(a0 + c);
    *reinterpret_cast<float2*>(a0 + c) = make_float2(x.x + dk[i][0] * scale, x.y + dk[i][1] * scale);
    x = *reinterpret_cast<float2*>(a1 + c);
    *reinterpret_cast<float2*>(a1 + c) = make_float2(x.x + dk[i][2] * scale, x.y + dk[i][3] * scale);
    x = *reinterpret_cast<float2*>(b0 + c);
    *reinterpret_cast<float2*>(b0 + c) = make_float2(x.x + dv[i][0], x.y + dv[i][1]);
    x = *reinterpret_cast<float2*>(b1 + c);
    *reinterpret_cast<float2*>(b1 + c) = make_float2(x.x + dv[i][2], x.y + dv[i][3]);
  }
}

// ------------------------------------------------------------------ host launchers
constexpr int ATTN_BWD_SMEM = 6 * AT_TILE_BYTES;

jenga_status attn_forward(const bf16* q, const bf16* k, const bf16* v, int64_t ld, bf16* o, int64_t ldo, float* lse,
                          int64_t lse_ld, int H, const int32_t* n_valid, int valid_mult, int n_cap, cudaStream_t st) {
  if (n_cap <= 0) return JENGA_OK;
  if (n_cap % AT_ROWS) return fail(JENGA_EINVAL, "attention: rows must be a multiple of 64");
  const float scale_log2 = LOG2E / sqrtf((float)AT_D);
  {
    // TMA-fed 128-row tiles (rows of q/k/v past the valid count must be finite: the layer
    // zeroes them before this call)
    CUtensorMap tq, tk, tv;
    jenga_status s1;
    if ((s1 = make_tmap_bf16(&tq, q, n_cap, (uint64_t)H * AT_D, ld, ATC_ROWS)) != JENGA_OK) return s1;
    if ((s1 = make_tmap_bf16(&tk, k, n_cap, (uint64_t)H * AT_D, ld, ATC_ROWS)) != JENGA_OK) return s1;
    if ((s1 = make_tmap_bf16(&tv, v, n_cap, (uint64_t)H * AT_D, ld, ATC_ROWS)) != JENGA_OK) return s1;
    JENGA_CUDA_TRY(cudaFuncSetAttribute(attn_fwd_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, ATC_SMEM));
    const int _ps = ::jenga::prof_begin("attn_fwd_tc", st);
    attn_fwd_tc_kernel<<<dim3((n_cap + ATC_ROWS - 1) / ATC_ROWS, H), ATC_THREADS, ATC_SMEM, st>>>(
        tq, tk, tv, o, ldo, lse, lse_ld, n_valid, valid_mult, n_cap, scale_log2);
    ::jenga::prof_end(_ps, st);
    JENGA_LAUNCH_CHECK();
    return JENGA_OK;
  }
}

jenga_status attn_backward_segment(const bf16* q, const bf16* k, const bf16* v, int64_t ld, const bf16* o,
                                   int64_t ldo, const float* lse, int64_t lse_ld, const bf16* dO, int64_t ld_do,
                                   float* delta, int64_t delta_ld, float* dq, int64_t ld_dq, float* dk_acc,
                                   float* dv_acc, int64_t ld_acc, int H, int s0, int s1, const int32_t* n_valid,
                                   int valid_mult, int n_cap, cudaStream_t st) {
  if (s1 <= s0) return JENGA_OK;
  if (s0 % AT_ROWS || s1 % AT_ROWS) return fail(JENGA_EINVAL, "attention bwd: segment bounds must be multiples of 64");
  const int T = s1 - s0;
  const float scale = 1.f / sqrtf((float)AT_D);
  const float scale_log2 = LOG2E * scale;
  {
    const int warps = T * H;
    {
    const int _ps = ::jenga::prof_begin("attn_delta", st);
    attn_delta_kernel<<<(warps + 7) / 8, 256, 0, st>>>(dO, ld_do, o + (int64_t)s0 * ldo, ldo, delta, delta_ld, T, H);
    ::jenga::prof_end(_ps, st);
    }
    JENGA_LAUNCH_CHECK();
  }
  const bool bulk_ok = lse_ld % 4 == 0 && delta_ld % 4 == 0 && ((uintptr_t)lse & 15) == 0 &&
                       ((uintptr_t)delta & 15) == 0;
  if (s0 % 128 == 0 && bulk_ok) {
    // tcgen05 path (segment starts are multiples of 128 tokens; L and Delta rows are
    // bulk-copied, so their pitches and bases must be 16-byte multiples)
    CUtensorMap tk128, tv128, tq64, tdo64, tq128, tdo128, tk64, tv64;
    jenga_status e;
    const uint64_t HDc = (uint64_t)H * AT_D;
    if ((e = make_tmap_bf16(&tk128, k, n_cap, HDc, ld, 128)) != JENGA_OK) return e;
    if ((e = make_tmap_bf16(&tv128, v, n_cap, HDc, ld, 128)) != JENGA_OK) return e;
    if ((e = make_tmap_bf16(&tq64, q, n_cap, HDc, ld, 64)) != JENGA_OK) return e;
    if ((e = make_tmap_bf16(&tdo64, dO, T, HDc, ld_do, 64)) != JENGA_OK) return e;
    if ((e = make_tmap_bf16(&tq128, q, n_cap, HDc, ld, 128)) != JENGA_OK) return e;
    if ((e = make_tmap_bf16(&tdo128, dO, T, HDc, ld_do, 128)) != JENGA_OK) return e;
    if ((e = make_tmap_bf16(&tk64, k, n_cap, HDc, ld, 64)) != JENGA_OK) return e;
    if ((e = make_tmap_bf16(&tv64, v, n_cap, HDc, ld, 64)) != JENGA_OK) return e;
    CUtensorMap tdq;  // fp32 dQ rows of the segment [T, H * 128]
    if ((e = make_tmap_f32(&tdq, dq, T, HDc, ld_dq, 128)) != JENGA_OK) return e;
    CUtensorMap tdk, tdv;  // fp32 accumulators [n_cap, H * 128], 128-row x 32-column boxes
    if ((e = make_tmap_f32(&tdk, dk_acc, n_cap, HDc, ld_acc, 128)) != JENGA_OK) return e;
    if ((e = make_tmap_f32(&tdv, dv_acc, n_cap, HDc, ld_acc, 128)) != JENGA_OK) return e;
    JENGA_CUDA_TRY(cudaFuncSetAttribute(attn_bwd_dq_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, DQ_SMEM));
    JENGA_CUDA_TRY(
        cudaFuncSetAttribute(attn_bwd_dkdv_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, DKV_SMEM));
    {
      const int _ps = ::jenga::prof_begin("attn_bwd_dq_tc", st);
      attn_bwd_dq_tc_kernel<<<dim3((T + 127) / 128, H), ABT_THREADS, DQ_SMEM, st>>>(
          tq128, tdo128, tk64, tv64, lse, lse_ld, delta, delta_ld, tdq, s0, n_valid, valid_mult, n_cap, scale_log2,
          scale);
      ::jenga::prof_end(_ps, st);
    }
    JENGA_LAUNCH_CHECK();
    {
      const int _ps = ::jenga::prof_begin("attn_bwd_dkdv_tc", st);
      attn_bwd_dkdv_tc_kernel<<<dim3((s1 + 127) / 128, H), DKV_THREADS, DKV_SMEM, st>>>(
          tk128, tv128, tq64, tdo64, lse, lse_ld, delta, delta_ld, tdk, tdv, s0, s1, n_valid, valid_mult, n_cap,
          scale_log2, scale);
      ::jenga::prof_end(_ps, st);
    }
    JENGA_LAUNCH_CHECK();
    return JENGA_OK;
  }
  JENGA_CUDA_TRY(cudaFuncSetAttribute(attn_bwd_dq_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, ATTN_BWD_SMEM));
  JENGA_CUDA_TRY(
      cudaFuncSetAttribute(attn_bwd_dkdv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, ATTN_BWD_SMEM));
  {
  const int _ps = ::jenga::prof_begin("attn_bwd_dq", st);
  attn_bwd_dq_kernel<<<dim3(T / AT_ROWS, H), 128, ATTN_BWD_SMEM, st>>>(q, k, v, ld, dO, ld_do, lse, lse_ld, delta,
                                                                      delta_ld, dq, ld_dq, s0, n_valid, valid_mult,
                                                                      n_cap, scale_log2, scale);
  ::jenga::prof_end(_ps, st);
  }
  JENGA_LAUNCH_CHECK();
  {
  const int _ps = ::jenga::prof_begin("attn_bwd_dkdv", st);
  attn_bwd_dkdv_kernel<<<dim3(s1 / AT_ROWS, H), 128, ATTN_BWD_SMEM, st>>>(
      q, k, v, ld, dO, ld_do, lse, lse_ld, delta, delta_ld, dk_acc, dv_acc, ld_acc, s0, s1, n_valid, valid_mult,
      n_cap, scale_log2, scale);
  ::jenga::prof_end(_ps, st);
  }
  JENGA_LAUNCH_CHECK();
  return JENGA_OK;
}

}  // namespace jenga
