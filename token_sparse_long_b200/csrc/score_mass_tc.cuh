// tcgen05 block-scoring pass 2 (head_dim 128, 128-token tiles): per key j,
//
//   mass_j = sum_{i >= j} 2^(log2(e) q_i . k_j / sqrt(D) - L_i)
//
// with -L_i, the negated row log-sum-exp in log2 units, from pass 1 (score_tc.cuh).
// One CTA per (128-key tile, head, sequence), 608 threads:
//   warp 0       TMA: the CTA's key tile (two 64-column swizzled boxes), then the query
//                tiles through a 4-stage shared-memory ring
//   warps 1, 2   TMEM allocation (warp 1); one lane of each issues tcgen05.mma (M 128,
//                N 128, K 16) x 8 per query tile, warp 1 for even and warp 2 for odd tiles,
//                into one of three 128-column TMEM accumulators; A = the key tile, read
//                from tensor memory (quad 0 of the epilogue copies it there once), B = the
//                query tile from shared memory
//   warps 3..18  four quads; in each quad one TMEM lane (= one key) per thread, quad c
//                taking query columns 32c .. 32c + 31: tcgen05.ld, release the accumulator,
//                then exponentials and sums in registers (packed f32x2 arithmetic; a few
//                column pairs on the FMA pipe, exp2_fma); the four partial sums of each key
//                are added in shared memory at the end
// Why this shape and not pass 1's N 256: each thread needs the 32 values -L_i of its
// columns in registers next to the 32 logits, and with 64 columns per thread they do not
// fit beside the accumulator values; 32 columns per thread with three accumulators, so
// the MMAs can run ahead of the slowest epilogue warp, measured fastest.  Causal diagonal
// tiles are masked in a separate branch.  All waits are bounded.
#pragma once

#include "score_tc.cuh"

namespace jenga {

constexpr int SMT_STAGES = 4;
constexpr int SMT_EPI_WARPS = 16;
constexpr int SMT_EPI_WARP0 = 3;  // warps 0 TMA, 1 and 2 MMA issue, 3 .. 18 epilogue
constexpr int SMT_THREADS = 32 * SMT_EPI_WARP0 + 32 * SMT_EPI_WARPS;
constexpr int SMT_SBUF = 3;        // TMEM accumulators (128 columns each)
constexpr int SMT_TA_COL = 384;    // tensor-memory columns of the key tile (A operand): 384 .. 447
constexpr int SMT_XCH_BYTES = 4 * 128 * 4;
constexpr int SMT_SMEM = (1 + SMT_STAGES) * SCT_TILE_BYTES + 256 + SMT_XCH_BYTES + 1024;
#ifndef SMT_EMU_PAIRS
#define SMT_EMU_PAIRS 0x5252u  // column pairs p (of 16) with bit p set use exp2_fma: 6 of 16
#endif

__global__ void __launch_bounds__(SMT_THREADS, 1)
    score_mass_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK, int S,
                         int H, int causal, float scale_log2, const float* __restrict__ neg_lse,
                         float* __restrict__ out) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* fix = smem;
  uint8_t* ring = smem + SCT_TILE_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + (1 + SMT_STAGES) * SCT_TILE_BYTES);
  uint64_t* full = bars;                       // [STAGES]
  uint64_t* empty = full + SMT_STAGES;         // [STAGES]
  uint64_t* s_full = empty + SMT_STAGES;       // [SBUF]
  uint64_t* s_empty = s_full + SMT_SBUF;       // [SBUF]
  uint64_t* fix_full = s_empty + SMT_SBUF;
  uint64_t* a_ready = fix_full + 1;            // the key tile is in tensor memory
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(a_ready + 1);
  float* xch = reinterpret_cast<float*>(smem + (1 + SMT_STAGES) * SCT_TILE_BYTES + 256);  // [4][128]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ntile = S / SCT_ROWS;
  const int h = blockIdx.y, b = blockIdx.z;
  const int t = blockIdx.x;  // key tile; tile 0 sees the most queries, so it starts first
  const int j0 = causal ? t : 0;
  const int nj = ntile - j0;
  const int col0 = h * 128;
  const int rowbase = b * S;

  if (threadIdx.x == 0) {
    for (int s = 0; s < SMT_STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int s = 0; s < SMT_SBUF; ++s) {
      mbar_init(&s_full[s], 1);
      mbar_init(&s_empty[s], SMT_EPI_WARPS);
    }
    mbar_init(fix_full, 1);
    mbar_init(a_ready, 4);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmQ);
    mbar_arrive_expect_tx(fix_full, SCT_TILE_BYTES);
    tma_load_2d(fix, &tmK, fix_full, col0, rowbase + t * SCT_ROWS);
    tma_load_2d(fix + SCT_BOX_BYTES, &tmK, fix_full, col0 + 64, rowbase + t * SCT_ROWS);
    for (int i = 0; i < nj; ++i) {
      const int s = i % SMT_STAGES;
      if (i >= SMT_STAGES && !mbar_wait(&empty[s], ((i / SMT_STAGES) - 1) & 1, SITE_SCORE_TC)) break;
      uint8_t* dst = ring + s * SCT_TILE_BYTES;
      const int row = rowbase + (j0 + i) * SCT_ROWS;
      mbar_arrive_expect_tx(&full[s], SCT_TILE_BYTES);
      tma_load_2d(dst, &tmQ, &full[s], col0, row);
      tma_load_2d(dst + SCT_BOX_BYTES, &tmQ, &full[s], col0 + 64, row);
    }
  } else if ((warp == 1 || warp == 2) && lane == 0) {
    // tile i goes to warp 1 + (i & 1), which also owns ring stage i % 4 (tiles i and i + 4
    // share a stage and a parity); accumulator i % 3 is shared, but tile i + 3 waits for
    // the epilogue to have read tile i, so its phases stay in tile order
    constexpr uint32_t idesc = umma_idesc_bf16(128, 128);
    bool ok = mbar_wait(a_ready, 0, SITE_SCORE_TC);
    for (int i = warp - 1; ok && i < nj; i += 2) {
      const int s = i % SMT_STAGES, buf = i % SMT_SBUF;
      if (!mbar_wait(&full[s], (i / SMT_STAGES) & 1, SITE_SCORE_TC)) break;
      if (i >= SMT_SBUF && !mbar_wait(&s_empty[buf], ((i / SMT_SBUF) - 1) & 1, SITE_SCORE_TC)) break;
      tc_fence_after();
      const uint32_t sb = smem_u32(ring + s * SCT_TILE_BYTES);
#pragma unroll
      for (int kc = 0; kc < 2; ++kc)
#pragma unroll
        for (int k = 0; k < 4; ++k)
          umma_bf16_ts(tmem + buf * 128, tmem + SMT_TA_COL + kc * 32 + k * 8,
                       umma_desc_k_sw128(sb + kc * SCT_BOX_BYTES + k * 32), idesc, (kc | k) ? 1u : 0u);
      umma_commit(&empty[s]);
      umma_commit(&s_full[buf]);
    }
  } else if (warp >= SMT_EPI_WARP0) {
    // quad c = (warp - 3) / 4 takes query columns 32c .. 32c + 31; warp w reads TMEM lanes
    // 32 * (w % 4) ..
    const int quarter = warp & 3;
    const int quad = (warp - SMT_EPI_WARP0) >> 2;
    const int r = quarter * 32 + lane;
    const int cbase = quad * 32;
    const uint32_t tl = tmem + ((uint32_t)(quarter * 32) << 16) + cbase;
    float acc = 0.f;
    bool ok = true;
    if (quad == 0) {
      // the key tile (A operand of every MMA) goes from shared to tensor memory once
      if (__all_sync(0xffffffffu, mbar_wait(fix_full, 0, SITE_SCORE_TC))) {
        tile_row_to_tmem(fix, r, tmem + ((uint32_t)(quarter * 32) << 16) + SMT_TA_COL);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(a_ready);
      } else {
        ok = false;
      }
    }
    const float* lb = neg_lse + ((int64_t)b * H + h) * S + cbase;
    const uint64_t sl2x2 = f2pack(scale_log2, scale_log2);
    for (int i = 0; ok && i < nj; ++i) {
      const int buf = i % SMT_SBUF, j = j0 + i;
      float4 L4[8];  // -L of this quad's 32 queries, loaded before the wait
#pragma unroll
      for (int c4 = 0; c4 < 8; ++c4) L4[c4] = __ldg(reinterpret_cast<const float4*>(lb + (int64_t)j * SCT_ROWS) + c4);
      // warp vote: the tcgen05.ld below is collective, so all lanes leave together
      if (!__all_sync(0xffffffffu, mbar_wait(&s_full[buf], (i / SMT_SBUF) & 1, SITE_SCORE_TC))) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t v[32];
      tmem_ld32_nowait(tl + buf * 128, v);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_empty[buf]);
      if (!(causal && j == t)) {
        uint64_t acc2[4] = {0ull, 0ull, 0ull, 0ull};  // (0.f, 0.f) pairs
#pragma unroll
        for (int c4 = 0; c4 < 8; ++c4) {
          const uint64_t x01 = ffma2(f2pack(__uint_as_float(v[4 * c4]), __uint_as_float(v[4 * c4 + 1])), sl2x2,
                                     f2pack(L4[c4].x, L4[c4].y));
          const uint64_t x23 = ffma2(f2pack(__uint_as_float(v[4 * c4 + 2]), __uint_as_float(v[4 * c4 + 3])), sl2x2,
                                     f2pack(L4[c4].z, L4[c4].w));
          const int p0 = 2 * c4, p1 = 2 * c4 + 1;
          acc2[p0 & 3] = fadd2(acc2[p0 & 3], ((SMT_EMU_PAIRS >> p0) & 1u) ? exp2_fma_x2<-1>(x01) : exp2_mufu_x2(x01));
          acc2[p1 & 3] = fadd2(acc2[p1 & 3], ((SMT_EMU_PAIRS >> p1) & 1u) ? exp2_fma_x2<-1>(x23) : exp2_mufu_x2(x23));
        }
        acc += f2sum4(acc2);
      } else {  // diagonal tile: query column c sees key r iff cbase + c >= r
        float sm[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int c4 = 0; c4 < 8; ++c4) {
          const float Ls[4] = {L4[c4].x, L4[c4].y, L4[c4].z, L4[c4].w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int c = 4 * c4 + e;
            const float p = fast_exp2(fmaf(__uint_as_float(v[c]), scale_log2, Ls[e]));
            sm[e] += (cbase + c < r) ? 0.f : p;
          }
        }
        acc += (sm[0] + sm[1]) + (sm[2] + sm[3]);
      }
    }
    // add the four partial sums of each key in a fixed order (quad 0, 1, 2, 3)
    xch[quad * 128 + r] = acc;
    asm volatile("bar.sync 1, %0;" ::"n"(32 * SMT_EPI_WARPS) : "memory");
    if (quad == 0 && ok)
      out[((int64_t)b * H + h) * S + t * SCT_ROWS + r] = ((xch[r] + xch[128 + r]) + xch[256 + r]) + xch[384 + r];
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace jenga
