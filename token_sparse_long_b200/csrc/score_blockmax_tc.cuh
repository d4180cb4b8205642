// tcgen05 paper-form block score (Jenga summary §4.2.2 Eq. (2), aggregated per §4.2.3), bf16,
// head_dim 128:
//
//   A_ij = sum_h max(q^h_i . k^h_j / sqrt(D), 0) / N_head             (score matrix)
//   I(B^S_mn) = max over the causal entries (j <= i) of A_ij, i in query block m, j in key block n
//   score[n] = sum over the query blocks m >= n of I(B^S_mn)
//
// One CTA per (128-query tile, 128-key tile at or before it, sequence), 608 threads:
//   warp 0       TMA: per head the query tile's and the key tile's 128 x 128 slices through a
//                3-stage ring
//   warps 1, 2   TMEM allocation (warp 1); one lane of each issues S^h = Q^h K^h^T (M 128,
//                N 128, K 16 x 8) into one of two 128-column accumulators, warp 1 for even and
//                warp 2 for odd heads
//   warps 3..18  four quads, one TMEM lane (= one query row) per thread, quad c taking key
//                columns 32c .. 32c + 31: tcgen05.ld, release, add max(s, 0) into 32 running
//                sums in registers; after the last head, the maxima over each (query block,
//                key block) sub-tile are reduced across threads and written
// The logits' positive parts are summed unscaled and multiplied by 1/(sqrt(D) N_head) at the
// end (a positive factor commutes with max(., 0) and max).  Every wait is bounded.
#pragma once

#include "common.cuh"

namespace jenga {

constexpr int BM_STAGES = 3;
constexpr int BM_BOX_BYTES = 128 * 64 * 2;
constexpr int BM_TILE_BYTES = 2 * BM_BOX_BYTES;     // 128 x 128 bf16
constexpr int BM_STAGE_BYTES = 2 * BM_TILE_BYTES;   // Q^h tile + K^h tile
constexpr int BM_EPI_WARPS = 16;
constexpr int BM_EPI_WARP0 = 3;
constexpr int BM_THREADS = 32 * (BM_EPI_WARP0 + BM_EPI_WARPS);
constexpr int BM_BAR_OFF = BM_STAGES * BM_STAGE_BYTES;
constexpr int BM_RED_OFF = BM_BAR_OFF + 256;        // [16 warps][4 row groups of 32]: warp maxima
constexpr int BM_SMEM = BM_RED_OFF + 16 * 4 * 4 + 1024;

// part[b, ng, mg] = max over the causal entries of the (query group mg, key group ng) sub-tile
// of this tile pair, for groups of g = 32, 64 or 128 tokens (-1 where the sub-tile has no
// causal entry); a block of blk tokens is blk / g groups (blk 32 or 64: g = blk; blk a multiple
// of 128: g = 128).
__global__ void __launch_bounds__(BM_THREADS, 1)
    score_blockmax_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK, int S,
                             int H, int g, int causal, float out_scale, float* __restrict__ part) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + BM_BAR_OFF);
  uint64_t* full = bars;                // [STAGES]
  uint64_t* empty = full + BM_STAGES;   // [STAGES]
  uint64_t* s_full = empty + BM_STAGES; // [2]
  uint64_t* s_empty = s_full + 2;       // [2]
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(s_empty + 2);
  float* red = reinterpret_cast<float*>(smem + BM_RED_OFF);  // [16 epilogue warps][4]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nt = (S + 127) / 128;
  // tile pair: blockIdx.x enumerates (query tile it, key tile jt) with jt <= it when causal
  int it, jt;
  if (causal) {
    const int p = blockIdx.x;  // p = it (it + 1) / 2 + jt
    it = (int)((sqrtf(8.f * (float)p + 1.f) - 1.f) * 0.5f);
    while ((it + 1) * (it + 2) / 2 <= p) ++it;
    while (it * (it + 1) / 2 > p) --it;
    jt = p - it * (it + 1) / 2;
  } else {
    it = blockIdx.x / nt;
    jt = blockIdx.x % nt;
  }
  const int b = blockIdx.y;
  const int rowq = b * S + it * 128, rowk = b * S + jt * 128;

  if (threadIdx.x == 0) {
    for (int s = 0; s < BM_STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&s_full[s], 1);
      mbar_init(&s_empty[s], BM_EPI_WARPS);
    }
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmK);
    for (int h = 0; h < H; ++h) {
      const int s = h % BM_STAGES;
      if (h >= BM_STAGES && !mbar_wait(&empty[s], (uint32_t)(((h / BM_STAGES) - 1) & 1), SITE_SCORE_TC)) break;
      uint8_t* dst = smem + s * BM_STAGE_BYTES;
      mbar_arrive_expect_tx(&full[s], BM_STAGE_BYTES);
#pragma unroll
      for (int kc = 0; kc < 2; ++kc) {
        tma_load_2d(dst + kc * BM_BOX_BYTES, &tmQ, &full[s], h * 128 + 64 * kc, rowq);
        tma_load_2d(dst + BM_TILE_BYTES + kc * BM_BOX_BYTES, &tmK, &full[s], h * 128 + 64 * kc, rowk);
      }
    }
  } else if ((warp == 1 || warp == 2) && lane == 0) {
    constexpr uint32_t idesc = umma_idesc_bf16(128, 128);
    for (int h = warp - 1; h < H; h += 2) {
      const int s = h % BM_STAGES, buf = h & 1;
      if (!mbar_wait(&full[s], (uint32_t)((h / BM_STAGES) & 1), SITE_SCORE_TC)) break;
      if (h >= 2 && !mbar_wait(&s_empty[buf], (uint32_t)(((h >> 1) - 1) & 1), SITE_SCORE_TC)) break;
      tc_fence_after();
      const uint32_t qa = smem_u32(smem + s * BM_STAGE_BYTES);
      const uint32_t ka = qa + BM_TILE_BYTES;
#pragma unroll
      for (int kc = 0; kc < 2; ++kc)
#pragma unroll
        for (int k = 0; k < 4; ++k)
          umma_bf16(tmem + buf * 128, umma_desc_k_sw128(qa + kc * BM_BOX_BYTES + k * 32),
                    umma_desc_k_sw128(ka + kc * BM_BOX_BYTES + k * 32), idesc, (kc | k) ? 1u : 0u);
      umma_commit(&empty[s]);
      umma_commit(&s_full[buf]);
    }
  } else if (warp >= BM_EPI_WARP0) {
    const int quarter = warp & 3;
    const int quad = (warp - BM_EPI_WARP0) >> 2;
    const int ew = warp - BM_EPI_WARP0;
    const int r = quarter * 32 + lane;
    const uint32_t tl = tmem + ((uint32_t)(quarter * 32) << 16) + quad * 32;
    float acc[32];
#pragma unroll
    for (int c = 0; c < 32; ++c) acc[c] = 0.f;
    bool ok = true;
    for (int h = 0; h < H; ++h) {
      const int buf = h & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(&s_full[buf], (uint32_t)((h >> 1) & 1), SITE_SCORE_TC))) {
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
#pragma unroll
      for (int c = 0; c < 32; ++c) acc[c] += fmaxf(__uint_as_float(v[c]), 0.f);
    }
    // this thread's maximum over its visible columns (-1: none visible)
    const int i = it * 128 + r;
    float mx = -1.f;
#pragma unroll
    for (int c = 0; c < 32; ++c) {
      const int j = jt * 128 + quad * 32 + c;
      const bool vis = i < S && j < S && (!causal || j <= i);
      mx = vis ? fmaxf(mx, acc[c] * out_scale) : mx;
    }
    // query blocks of 32 rows are warps; max over the warp's lanes, then over the warps and
    // quads that make up each (query block, key block) sub-tile
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if (lane == 0) red[quad * 4 + quarter] = mx;
    asm volatile("bar.sync 1, %0;" ::"n"(32 * BM_EPI_WARPS) : "memory");
    const int per = g / 32;   // 32-row / 32-column groups per sub-tile side (1, 2 or 4)
    const int nbt = 4 / per;  // sub-tiles per tile side
    if (ew == 0 && lane < nbt * nbt && ok) {
      const int qm = lane / nbt, kn = lane % nbt;  // sub-tile (query group, key group)
      float best = -1.f;
      for (int a = 0; a < per; ++a)
        for (int c = 0; c < per; ++c) best = fmaxf(best, red[(kn * per + c) * 4 + (qm * per + a)]);
      const int mg = (it * 128) / g + qm, ng = (jt * 128) / g + kn;
      const int ngr = S / g;
      if (mg < ngr && ng < ngr) part[((int64_t)b * ngr + ng) * ngr + mg] = best;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

// scores[b, n] = sum over the query blocks m with a causal entry in column n (m >= n, or all m
// when not causal) of the max over the block's (query group, key group) sub-tiles that hold
// causal entries (mg >= ng) of part[b, ng, mg]; f = blk / g groups per block; fixed order.
__global__ void score_blockmax_colsum_kernel(const float* __restrict__ part, int nb, int f, int causal,
                                             float* __restrict__ scores) {
  const int n = blockIdx.x * blockDim.x + threadIdx.x, b = blockIdx.y;
  if (n >= nb) return;
  const int ngr = nb * f;
  float s = 0.f;
  for (int m = causal ? n : 0; m < nb; ++m) {
    float best = -1.f;
    for (int a = 0; a < f; ++a)
      for (int c = 0; c < f; ++c) {
        const int mg = m * f + a, ng = n * f + c;
        if (!causal || mg >= ng) best = fmaxf(best, part[((int64_t)b * ngr + ng) * ngr + mg]);
      }
    s += best;
  }
  scores[(int64_t)b * nb + n] = s;
}

}  // namespace jenga
