// tcgen05 block-scoring passes (head_dim 128, 128-token tiles).
//
//   pass 1 (ROWS = queries): L_i = log2 sum_{j <= i} 2^(log2(e) q_i . k_j / sqrt(D))
//   pass 2 (ROWS = keys):    mass_j = sum_{i >= j} 2^(log2(e) q_i . k_j / sqrt(D) - L_i)
//
// One CTA per (128-row tile, head, sequence), 576 threads:
//   warp 0       TMA: the CTA's fixed 128 x 128 tile (two 64-column swizzled boxes), then
//                the streamed tiles through a 4-stage shared-memory ring
//   warp 1       TMEM allocation; one lane issues tcgen05.mma (M 128, N 128, K 16) x 8 per
//                streamed tile into one of two 128-column TMEM accumulators
//   warps 2..17  four quads; in each quad one TMEM lane (= one row of the tile) per thread,
//                quad c taking columns 32c .. 32c + 31: tcgen05.ld, release the accumulator,
//                then exponentials and sums in registers, which overlaps the next tile's
//                MMA; the four quarter rows are merged in shared memory at the end
// The exponentials, one per causal (query, key) pair and pass, bound the kernel: the
// multi-function unit returns 16 per clock per SM against 8192 tensor flops, so a 128 x 128
// tile costs 1024 clocks of exponentials for 512 of MMA.  SCT_EMU_MASK routes some columns
// of each thread through exp2_fma (FMA / integer pipes) instead.
// Pass 1 keeps a per-row reference m (log2 units) and sums 2^(x - m) without a per-element
// max; a tile is redone with its exact max only when its sum leaves [0, 2^60) (a new
// maximum more than ~60 above m, or the first tile).  Causal diagonal tiles are masked in
// a separate branch.  All waits are bounded.
#pragma once

#include "common.cuh"

namespace jenga {

constexpr int SCT_ROWS = 128;
constexpr int SCT_STAGES = 4;
constexpr int SCT_BOX_BYTES = 128 * 64 * 2;          // one 128 x 64 bf16 box
constexpr int SCT_TILE_BYTES = 2 * SCT_BOX_BYTES;     // 128 x 128 tile
constexpr int SCT_EPI_WARPS = 16;
constexpr int SCT_THREADS = 64 + 32 * SCT_EPI_WARPS;
constexpr int SCT_XCH_BYTES = 2 * 4 * 128 * 4;        // per quad: m (or mass) and l of 128 rows
constexpr int SCT_SMEM = (1 + SCT_STAGES) * SCT_TILE_BYTES + 256 + SCT_XCH_BYTES + 1024;
#ifndef SCT_EMU_MASK
#define SCT_EMU_MASK 0x88888888u  // columns c (of 32) with bit c set use exp2_fma: 8 of 32
#endif

template <bool EMU>
__device__ __forceinline__ float sct_exp2(float x) {
  if constexpr (EMU) return exp2_fma<64>(x);
  else return fast_exp2(x);
}

template <int MODE>  // 0: row LSE (rows = queries), 1: column mass (rows = keys)
__global__ void __launch_bounds__(SCT_THREADS, 1)
    score_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK, int S,
                    int H, int causal, float scale_log2, const float* __restrict__ lse_in,
                    float* __restrict__ out) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* fix = smem;
  uint8_t* ring = smem + SCT_TILE_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + (1 + SCT_STAGES) * SCT_TILE_BYTES);
  uint64_t* full = bars;                       // [STAGES]
  uint64_t* empty = full + SCT_STAGES;         // [STAGES]
  uint64_t* s_full = empty + SCT_STAGES;       // [2]
  uint64_t* s_empty = s_full + 2;              // [2]
  uint64_t* fix_full = s_empty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(fix_full + 1);
  float* xch = reinterpret_cast<float*>(smem + (1 + SCT_STAGES) * SCT_TILE_BYTES + 256);  // [2][4][128]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ntile = S / SCT_ROWS;
  const int h = blockIdx.y, b = blockIdx.z;
  // pass 1: longest query tiles first; pass 2: key tile 0 sees the most queries
  const int t = (MODE == 0) ? (ntile - 1 - (int)blockIdx.x) : (int)blockIdx.x;
  const int j0 = (MODE == 0) ? 0 : (causal ? t : 0);
  const int j1 = (MODE == 0) ? (causal ? t + 1 : ntile) : ntile;
  const int nj = j1 - j0;
  const int col0 = h * 128;
  const int rowbase = b * S;
  const CUtensorMap* tm_fix = (MODE == 0) ? &tmQ : &tmK;
  const CUtensorMap* tm_str = (MODE == 0) ? &tmK : &tmQ;

  if (threadIdx.x == 0) {
    for (int s = 0; s < SCT_STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&s_full[s], 1);
      mbar_init(&s_empty[s], SCT_EPI_WARPS);
    }
    mbar_init(fix_full, 1);
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
    prefetch_tmap(tm_fix);
    prefetch_tmap(tm_str);
    mbar_arrive_expect_tx(fix_full, SCT_TILE_BYTES);
    tma_load_2d(fix, tm_fix, fix_full, col0, rowbase + t * SCT_ROWS);
    tma_load_2d(fix + SCT_BOX_BYTES, tm_fix, fix_full, col0 + 64, rowbase + t * SCT_ROWS);
    for (int i = 0; i < nj; ++i) {
      const int s = i % SCT_STAGES;
      if (i >= SCT_STAGES && !mbar_wait(&empty[s], ((i / SCT_STAGES) - 1) & 1, SITE_SCORE_TC)) break;
      uint8_t* dst = ring + s * SCT_TILE_BYTES;
      const int row = rowbase + (j0 + i) * SCT_ROWS;
      mbar_arrive_expect_tx(&full[s], SCT_TILE_BYTES);
      tma_load_2d(dst, tm_str, &full[s], col0, row);
      tma_load_2d(dst + SCT_BOX_BYTES, tm_str, &full[s], col0 + 64, row);
    }
  } else if (warp == 1 && lane == 0) {
    constexpr uint32_t idesc = umma_idesc_bf16(128, 128);
    bool ok = mbar_wait(fix_full, 0, SITE_SCORE_TC);
    const uint32_t fa = smem_u32(fix);
    for (int i = 0; ok && i < nj; ++i) {
      const int s = i % SCT_STAGES, buf = i & 1;
      if (!mbar_wait(&full[s], (i / SCT_STAGES) & 1, SITE_SCORE_TC)) break;
      if (i >= 2 && !mbar_wait(&s_empty[buf], ((i >> 1) - 1) & 1, SITE_SCORE_TC)) break;
      tc_fence_after();
      const uint32_t sb = smem_u32(ring + s * SCT_TILE_BYTES);
#pragma unroll
      for (int kc = 0; kc < 2; ++kc)
#pragma unroll
        for (int k = 0; k < 4; ++k)
          umma_bf16(tmem + buf * 128, umma_desc_k_sw128(fa + kc * SCT_BOX_BYTES + k * 32),
                    umma_desc_k_sw128(sb + kc * SCT_BOX_BYTES + k * 32), idesc, (kc | k) ? 1u : 0u);
      umma_commit(&empty[s]);
      umma_commit(&s_full[buf]);
    }
  } else if (warp >= 2) {
    // quad c = (warp - 2) / 4 takes columns 32c .. 32c + 31 of every row; warp w reads
    // TMEM lanes 32 * (w % 4) ..
    const int quarter = warp & 3;
    const int quad = (warp - 2) >> 2;
    const int r = quarter * 32 + lane;
    const int cbase = quad * 32;
    const uint32_t tl = tmem + ((uint32_t)(quarter * 32) << 16) + cbase;
    float m = -INFINITY, l = 0.f, acc = 0.f;
    bool ok = true;
    const float* lb = (MODE == 1) ? lse_in + ((int64_t)b * H + h) * S + cbase : nullptr;
    for (int i = 0; i < nj; ++i) {
      const int buf = i & 1, j = j0 + i;
      float4 L4[8];
      if (MODE == 1) {
#pragma unroll
        for (int c4 = 0; c4 < 8; ++c4) L4[c4] = __ldg(reinterpret_cast<const float4*>(lb + (int64_t)j * SCT_ROWS) + c4);
      }
      // warp vote: the tcgen05.ld below is collective, so all lanes leave together
      if (!__all_sync(0xffffffffu, mbar_wait(&s_full[buf], (i >> 1) & 1, SITE_SCORE_TC))) {
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
      const bool diag = causal && (j == t);
      if (MODE == 0) {
        if (!diag && m != -INFINITY) {
          float sm[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            const float x = fmaf(__uint_as_float(v[c]), scale_log2, -m);
            sm[c & 3] += ((SCT_EMU_MASK >> c) & 1u) ? sct_exp2<true>(x) : sct_exp2<false>(x);
          }
          const float sum = (sm[0] + sm[1]) + (sm[2] + sm[3]);
          if (sum < 0x1p60f) {  // false for inf / NaN too: then the exact path below
            l += sum;
            continue;
          }
        }
        float mx = -INFINITY;
        if (diag) {
#pragma unroll
          for (int c = 0; c < 32; ++c)
            if (cbase + c <= r) mx = fmaxf(mx, __uint_as_float(v[c]));
        } else {
#pragma unroll
          for (int c = 0; c < 32; ++c) mx = fmaxf(mx, __uint_as_float(v[c]));
        }
        const float mn = fmaxf(m, mx * scale_log2);
        if (mn != -INFINITY) {  // a quarter row of the diagonal tile can be fully masked
          float sm[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            const float p = fast_exp2(fmaf(__uint_as_float(v[c]), scale_log2, -mn));
            sm[c & 3] += (!diag || cbase + c <= r) ? p : 0.f;
          }
          const float sum = (sm[0] + sm[1]) + (sm[2] + sm[3]);
          l = l * fast_exp2(m - mn) + sum;
          m = mn;
        }
      } else {
        float sm[4] = {0.f, 0.f, 0.f, 0.f};
        if (!diag) {
#pragma unroll
          for (int c4 = 0; c4 < 8; ++c4) {
            const float Ls[4] = {L4[c4].x, L4[c4].y, L4[c4].z, L4[c4].w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int c = 4 * c4 + e;
              const float x = fmaf(__uint_as_float(v[c]), scale_log2, -Ls[e]);
              sm[e] += ((SCT_EMU_MASK >> c) & 1u) ? sct_exp2<true>(x) : sct_exp2<false>(x);
            }
          }
        } else {
#pragma unroll
          for (int c4 = 0; c4 < 8; ++c4) {
            const float Ls[4] = {L4[c4].x, L4[c4].y, L4[c4].z, L4[c4].w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int c = 4 * c4 + e;
              const float p = fast_exp2(fmaf(__uint_as_float(v[c]), scale_log2, -Ls[e]));
              sm[e] += (cbase + c < r) ? 0.f : p;  // key r is seen by queries >= r only
            }
          }
        }
        acc += (sm[0] + sm[1]) + (sm[2] + sm[3]);
      }
    }
    // merge the four quarter rows in a fixed order (quad 0, 1, 2, 3)
    xch[quad * 128 + r] = (MODE == 0) ? m : acc;
    xch[512 + quad * 128 + r] = l;
    asm volatile("bar.sync 1, %0;" ::"n"(32 * SCT_EPI_WARPS) : "memory");
    if (quad == 0 && ok) {
      float res;
      if (MODE == 0) {
        float mm = xch[r];
#pragma unroll
        for (int c = 1; c < 4; ++c) mm = fmaxf(mm, xch[c * 128 + r]);
        float ll = 0.f;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const float mc = xch[c * 128 + r];
          if (mc != -INFINITY) ll += xch[512 + c * 128 + r] * fast_exp2(mc - mm);
        }
        res = mm + __log2f(ll);  // log-sum-exp in log2 units (pass 2 consumes it directly)
      } else {
        res = ((xch[r] + xch[128 + r]) + xch[256 + r]) + xch[384 + r];
      }
      out[((int64_t)b * H + h) * S + t * SCT_ROWS + r] = res;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

}  // namespace jenga
