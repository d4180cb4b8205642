// tcgen05 block-scoring pass 1 (head_dim 128, 128-token tiles): per query i,
//
//   L_i = log2 sum_{j <= i} 2^(log2(e) q_i . k_j / sqrt(D)),  stored as -L_i
//
// (pass 2, the column mass, is score_mass_tc.cuh).
// One CTA per (128-query tile, head, sequence), 608 threads:
//   warp 0       TMA: the CTA's query tile (two 64-column swizzled boxes), then the key
//                tiles two at a time (256 rows) through a 3-stage shared-memory ring
//   warps 1, 2   TMEM allocation (warp 1); one lane of each issues tcgen05.mma (M 128, N 256,
//                K 16) x 8 per streamed pair, warp 1 for even and warp 2 for odd pairs, into
//                one of two 256-column TMEM accumulators (A = query tile, B = the key pair)
//   warps 3..18  four quads; in each quad one TMEM lane (= one query) per thread, quad c
//                taking accumulator columns 64c .. 64c + 63 (quads 0, 1 the first key tile,
//                2, 3 the second): tcgen05.ld, release the accumulator, then exponentials
//                and sums in registers, which overlaps the next pair's MMAs; the four
//                partial rows are merged in shared memory at the end
// Measured on B200: a warp issues its next tcgen05.mma only ~100 clocks after the last, so
// M 128 x N 128 products from one issuer reach ~60% of the tensor peak and N 256 ~92%; and
// every handshake (barrier round trip, TMEM load, fences) costs an epilogue warp a few
// hundred clocks, so each warp takes 64 columns per handshake.  The exponentials, one per
// causal (query, key) pair, then bound the kernel: the multi-function unit returns 16 per
// clock per SM against 8192 tensor flops, so a 128 x 128 tile costs 1024 clocks of
// exponentials for 512 of MMA.  SCT_EMU_PAIRS routes some column pairs of each thread
// through exp2_fma (FMA / integer pipes) instead, and the arithmetic around the
// exponentials runs as packed f32x2 pairs to keep the issue slots free.
// Each row keeps a reference m (log2 units) and sums 2^(x - m) without a per-element max;
// a tile is redone with its exact max only when its sum leaves [0, 2^60) (a new maximum
// more than ~60 above m, or the first tile).  Causal diagonal tiles are masked in a
// separate branch.  All waits are bounded.
#pragma once

#include "common.cuh"

namespace jenga {

constexpr int SCT_ROWS = 128;
constexpr int SCT_STAGES = 3;                         // ring stages of 256 streamed rows
constexpr int SCT_BOX_BYTES = 128 * 64 * 2;           // one 128 x 64 bf16 box
constexpr int SCT_TILE_BYTES = 2 * SCT_BOX_BYTES;     // 128 x 128 fixed tile
constexpr int SCT_PAIR_BYTES = 4 * SCT_BOX_BYTES;     // 256 x 128 streamed pair: [k half][256 rows x 64]
constexpr int SCT_EPI_WARPS = 16;
constexpr int SCT_EPI_WARP0 = 3;  // warps 0 TMA, 1 and 2 MMA issue, 3 .. 18 epilogue
constexpr int SCT_THREADS = 32 * SCT_EPI_WARP0 + 32 * SCT_EPI_WARPS;
constexpr int SCT_RING_OFF = SCT_TILE_BYTES;
constexpr int SCT_BAR_OFF = SCT_RING_OFF + SCT_STAGES * SCT_PAIR_BYTES;
constexpr int SCT_SMEM = SCT_BAR_OFF + 256 + 1024;    // + barriers, align
// the row exchange at the end (2 x 4 x 128 fp32) reuses the fixed tile's shared memory
#ifndef SCT_EMU_PAIRS
#define SCT_EMU_PAIRS 0x0202u  // column pairs p (of 16) with bit p set use exp2_fma: 2 of 16
#endif

// 2^x for one column pair: the FMA-pipe cubic for the pairs SCT_EMU_PAIRS selects, the
// multi-function unit for the rest (HI: upper clamp of the cubic's input, < 0 for none)
template <int HI>
__device__ __forceinline__ uint64_t sct_exp2_pair(uint64_t x2, int pair) {
  return ((SCT_EMU_PAIRS >> pair) & 1u) ? exp2_fma_x2<HI>(x2) : exp2_mufu_x2(x2);
}

__device__ __forceinline__ float f2sum4(const uint64_t* a) {
  float s[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) f2unpack(a[i], s[2 * i], s[2 * i + 1]);
  return ((s[0] + s[1]) + (s[2] + s[3])) + ((s[4] + s[5]) + (s[6] + s[7]));
}

// Pass-1 update of a row's (m, l) with 32 raw logits v (columns cb .. cb + 31 of the tile;
// diag: the causal diagonal tile, where column c is a key visible to row r iff c <= r).
__device__ __forceinline__ void sct_lse_update(const uint32_t* v, int cb, int r, bool diag, float scale_log2,
                                               float& m, float& l) {
  if (!diag && m != -INFINITY) {
    const uint64_t sl2x2 = f2pack(scale_log2, scale_log2), nm2 = f2pack(-m, -m);
    uint64_t acc2[4] = {0ull, 0ull, 0ull, 0ull};  // (0.f, 0.f) pairs
#pragma unroll
    for (int pr = 0; pr < 16; ++pr) {
      const uint64_t x2 = ffma2(f2pack(__uint_as_float(v[2 * pr]), __uint_as_float(v[2 * pr + 1])), sl2x2, nm2);
      acc2[pr & 3] = fadd2(acc2[pr & 3], sct_exp2_pair<64>(x2, pr));
    }
    const float sum = f2sum4(acc2);
    if (sum < 0x1p60f) {  // false for inf / NaN too: then the exact path below
      l += sum;
      return;
    }
  }
  float mx = -INFINITY;
  if (diag) {
#pragma unroll
    for (int c = 0; c < 32; ++c)
      if (cb + c <= r) mx = fmaxf(mx, __uint_as_float(v[c]));
  } else {
#pragma unroll
    for (int c = 0; c < 32; ++c) mx = fmaxf(mx, __uint_as_float(v[c]));
  }
  const float mn = fmaxf(m, mx * scale_log2);
  if (mn != -INFINITY) {  // a part of a row of the diagonal tile can be fully masked
    float sm[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int c = 0; c < 32; ++c) {
      const float p = fast_exp2(fmaf(__uint_as_float(v[c]), scale_log2, -mn));
      sm[c & 3] += (!diag || cb + c <= r) ? p : 0.f;
    }
    l = l * fast_exp2(m - mn) + ((sm[0] + sm[1]) + (sm[2] + sm[3]));
    m = mn;
  }
}

__global__ void __launch_bounds__(SCT_THREADS, 1)
    score_lse_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK, int S,
                        int H, int causal, float scale_log2, float* __restrict__ out) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* fix = smem;
  uint8_t* ring = smem + SCT_RING_OFF;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + SCT_BAR_OFF);
  uint64_t* full = bars;                       // [STAGES]
  uint64_t* empty = full + SCT_STAGES;         // [STAGES]
  uint64_t* s_full = empty + SCT_STAGES;       // [2]
  uint64_t* s_empty = s_full + 2;              // [2]
  uint64_t* fix_full = s_empty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(fix_full + 1);
  float* xch = reinterpret_cast<float*>(fix);  // [2][4][128], once every MMA is done

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ntile = S / SCT_ROWS;
  const int h = blockIdx.y, b = blockIdx.z;
  const int t = ntile - 1 - (int)blockIdx.x;  // query tile; longest first
  const int j0 = 0, j1 = causal ? t + 1 : ntile;
  const int np = (j1 - j0 + 1) >> 1;  // key-tile pairs (the last may hold one tile)
  const int col0 = h * 128;
  const int rowbase = b * S;
  const CUtensorMap* tm_fix = &tmQ;
  const CUtensorMap* tm_str = &tmK;

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
    tmem_alloc(tmem_holder, 512);
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
    for (int p = 0; p < np; ++p) {
      const int s = p % SCT_STAGES;
      if (p >= SCT_STAGES && !mbar_wait(&empty[s], ((p / SCT_STAGES) - 1) & 1, SITE_SCORE_TC)) break;
      uint8_t* dst = ring + s * SCT_PAIR_BYTES;
      // rows of a pair's second tile past the range are loaded too (zeros past the tensor,
      // else rows nobody reads): the epilogue skips them
      const int row = rowbase + (j0 + 2 * p) * SCT_ROWS;
      mbar_arrive_expect_tx(&full[s], SCT_PAIR_BYTES);
#pragma unroll
      for (int kc = 0; kc < 2; ++kc)
#pragma unroll
        for (int hh = 0; hh < 2; ++hh)
          tma_load_2d(dst + kc * 2 * SCT_BOX_BYTES + hh * SCT_BOX_BYTES, tm_str, &full[s], col0 + 64 * kc,
                      row + SCT_ROWS * hh);
    }
  } else if ((warp == 1 || warp == 2) && lane == 0) {
    // pair p goes to warp 1 + (p & 1), which owns accumulator p & 1 (pairs p and p + 2);
    // ring stage p % 3 alternates between the issuers, and pair p + 3 only finds its
    // stage full after the MMAs of pair p released it, so its phases stay in order
    constexpr uint32_t idesc = umma_idesc_bf16(128, 256);
    bool ok = mbar_wait(fix_full, 0, SITE_SCORE_TC);
    const uint32_t fa = smem_u32(fix);
    for (int p = warp - 1; ok && p < np; p += 2) {
      const int s = p % SCT_STAGES, buf = p & 1;
      if (!mbar_wait(&full[s], (p / SCT_STAGES) & 1, SITE_SCORE_TC)) break;
      if (p >= 2 && !mbar_wait(&s_empty[buf], ((p >> 1) - 1) & 1, SITE_SCORE_TC)) break;
      tc_fence_after();
      const uint32_t sb = smem_u32(ring + s * SCT_PAIR_BYTES);
#pragma unroll
      for (int kc = 0; kc < 2; ++kc)
#pragma unroll
        for (int k = 0; k < 4; ++k)
          umma_bf16(tmem + buf * 256, umma_desc_k_sw128(fa + kc * SCT_BOX_BYTES + k * 32),
                    umma_desc_k_sw128(sb + kc * 2 * SCT_BOX_BYTES + k * 32), idesc, (kc | k) ? 1u : 0u);
      umma_commit(&empty[s]);
      umma_commit(&s_full[buf]);
    }
  } else if (warp >= SCT_EPI_WARP0) {
    // quad c = (warp - 3) / 4 takes accumulator columns 64c .. 64c + 63: tile (c >> 1) of
    // the pair, its columns 64 (c & 1) ..; warp w reads TMEM lanes 32 * (w % 4) ..
    const int quarter = warp & 3;
    const int quad = (warp - SCT_EPI_WARP0) >> 2;
    const int r = quarter * 32 + lane;
    const int hp = quad >> 1, wc = (quad & 1) * 64;
    const uint32_t tl = tmem + ((uint32_t)(quarter * 32) << 16) + quad * 64;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int p = 0; p < np; ++p) {
      const int buf = p & 1, j = j0 + 2 * p + hp;
      const bool live = j < j1;  // warp-uniform
      // warp vote: the tcgen05.ld below is collective, so all lanes leave together
      if (!__all_sync(0xffffffffu, mbar_wait(&s_full[buf], (p >> 1) & 1, SITE_SCORE_TC))) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t v[64];
      if (live) {
        tmem_ld32_nowait(tl + buf * 256, v);
        tmem_ld32_nowait(tl + buf * 256 + 32, v + 32);
        tmem_wait_ld();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_empty[buf]);
      if (!live) continue;
      const bool diag = causal && (j == t);
      sct_lse_update(v, wc, r, diag, scale_log2, m, l);
      sct_lse_update(v + 32, wc + 32, r, diag, scale_log2, m, l);
    }
    // merge the four partial rows in a fixed order (quad 0, 1, 2, 3); every MMA (which
    // reads the fixed tile whose memory the exchange reuses) is done once all warps passed
    // their last wait above
    asm volatile("bar.sync 1, %0;" ::"n"(32 * SCT_EPI_WARPS) : "memory");
    xch[quad * 128 + r] = m;
    xch[512 + quad * 128 + r] = l;
    asm volatile("bar.sync 1, %0;" ::"n"(32 * SCT_EPI_WARPS) : "memory");
    if (quad == 0 && ok) {
      float mm = xch[r];
#pragma unroll
      for (int c = 1; c < 4; ++c) mm = fmaxf(mm, xch[c * 128 + r]);
      float ll = 0.f;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const float mc = xch[c * 128 + r];
        if (mc != -INFINITY) ll += xch[512 + c * 128 + r] * fast_exp2(mc - mm);
      }
      // negated log-sum-exp in log2 units (pass 2's FMA addend)
      out[((int64_t)b * H + h) * S + t * SCT_ROWS + r] = -(mm + __log2f(ll));
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace jenga
