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
// accumulators for keys [0, segment end).  The backward runs on fp16 operands (see
// attn_bwd_tc.cuh); the layer prepares the fp16 copies, dO's scale and Delta.  Processing segments last-first completes
// a segment's key gradients exactly when its own queries have been processed.
#include "attn_tc.cuh"
#include "attn_bwd_tc.cuh"

namespace jenga {

constexpr float LOG2E = 1.4426950408889634f;
constexpr int AT_D = 128;     // head dim
constexpr int AT_ROWS = 64;   // row granularity of the retained-row count

__device__ __forceinline__ int attn_rows(const int32_t* n_valid, int mult, int cap) {
  int n = n_valid ? (*n_valid) * mult : cap;
  return n < cap ? n : cap;
}

// ------------------------------------------------------------------ host launchers
// v16: an fp16 copy of v (row pitch ld_v16), the B operand of the PV product (fp16 P).
// o_lo (nullable): bf16 rounding residual of o (same layout), so that hi + lo carries ~16 bits.
jenga_status attn_forward(const bf16* q, const bf16* k, const void* v16, int64_t ld, int64_t ld_v16, bf16* o,
                          int64_t ldo, float* lse, int64_t lse_ld, int H, const int32_t* n_valid, int valid_mult,
                          int n_cap, cudaStream_t st, bf16* o_lo) {
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
    if ((s1 = make_tmap_f16(&tv, v16, n_cap, (uint64_t)H * AT_D, ld_v16, ATC_ROWS)) != JENGA_OK) return s1;
    JENGA_CUDA_TRY(cudaFuncSetAttribute(attn_fwd_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, ATC_SMEM));
    const int _ps = ::jenga::prof_begin("attn_fwd_tc", st);
    attn_fwd_tc_kernel<<<dim3((n_cap + ATC_ROWS - 1) / ATC_ROWS, H), ATC_THREADS, ATC_SMEM, st>>>(
        tq, tk, tv, o, ldo, lse, lse_ld, n_valid, valid_mult, n_cap, scale_log2, o_lo);
    ::jenga::prof_end(_ps, st);
    JENGA_LAUNCH_CHECK();
    return JENGA_OK;
  }
}

// Backward of one query segment [s0, s1) on fp16 operands (attn_bwd_tc.cuh): q16 / k16 / v16
// are fp16 copies of the forward's q / k / v (row pitch ld), dO16 the segment's dO scaled by
// gscal[2] (fp16, rows segment-local), delta the segment's -Delta_i = -dO16_i . o_i (fp32,
// [H, delta_ld]), gscal[3] the dS scale.
jenga_status attn_backward_segment(const void* q16, const void* k16, const void* v16, int64_t ld, const float* lse,
                                   int64_t lse_ld, const void* dO16, int64_t ld_do, const float* delta,
                                   int64_t delta_ld, float* dq, int64_t ld_dq, float* dk_acc, float* dv_acc,
                                   int64_t ld_acc, int H, int s0, int s1, const int32_t* n_valid, int valid_mult,
                                   int n_cap, const float* gscal, cudaStream_t st) {
  if (s1 <= s0) return JENGA_OK;
  if (s0 % AT_ROWS || s1 % AT_ROWS) return fail(JENGA_EINVAL, "attention bwd: segment bounds must be multiples of 64");
  const int T = s1 - s0;
  const float scale = 1.f / sqrtf((float)AT_D);
  const float scale_log2 = LOG2E * scale;
  const bool bulk_ok = lse_ld % 4 == 0 && delta_ld % 4 == 0 && ((uintptr_t)lse & 15) == 0 &&
                       ((uintptr_t)delta & 15) == 0;
  if (s0 % 128 != 0 || !bulk_ok)
    return fail(JENGA_EINTERNAL, "attention bwd: segment start %d not a multiple of 128 or misaligned L / Delta rows",
                s0);
  {
    // tcgen05 path (segment starts are multiples of 128 tokens; L and Delta rows are
    // bulk-copied, so their pitches and bases must be 16-byte multiples)
    CUtensorMap tk128, tv128, tq64, tdo64, tq128, tdo128, tk64, tv64;
    jenga_status e;
    const uint64_t HDc = (uint64_t)H * AT_D;
    if ((e = make_tmap_f16(&tk128, k16, n_cap, HDc, ld, 128)) != JENGA_OK) return e;
    if ((e = make_tmap_f16(&tv128, v16, n_cap, HDc, ld, 128)) != JENGA_OK) return e;
    if ((e = make_tmap_f16(&tq64, q16, n_cap, HDc, ld, 64)) != JENGA_OK) return e;
    if ((e = make_tmap_f16(&tdo64, dO16, T, HDc, ld_do, 64)) != JENGA_OK) return e;
    if ((e = make_tmap_f16(&tq128, q16, n_cap, HDc, ld, 128)) != JENGA_OK) return e;
    if ((e = make_tmap_f16(&tdo128, dO16, T, HDc, ld_do, 128)) != JENGA_OK) return e;
    if ((e = make_tmap_f16(&tk64, k16, n_cap, HDc, ld, 64)) != JENGA_OK) return e;
    if ((e = make_tmap_f16(&tv64, v16, n_cap, HDc, ld, 64)) != JENGA_OK) return e;
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
          scale, gscal);
      ::jenga::prof_end(_ps, st);
    }
    JENGA_LAUNCH_CHECK();
    {
      const int _ps = ::jenga::prof_begin("attn_bwd_dkdv_tc", st);
      attn_bwd_dkdv_tc_kernel<<<dim3((s1 + 127) / 128, H), DKV_THREADS, DKV_SMEM, st>>>(
          tk128, tv128, tq64, tdo64, lse, lse_ld, delta, delta_ld, tdk, tdv, s0, s1, n_valid, valid_mult, n_cap,
          scale_log2, scale, gscal);
      ::jenga::prof_end(_ps, st);
    }
    JENGA_LAUNCH_CHECK();
    return JENGA_OK;
  }
}

}  // namespace jenga
