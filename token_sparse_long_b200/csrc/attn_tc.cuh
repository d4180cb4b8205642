// tcgen05 causal attention forward over the retained tokens (head_dim 128).
//
// One CTA per (128-query tile, head), 352 threads:
//   warp 0      TMA: the Q tile once, then K_j and V_j through two 3-stage rings (K_j is
//               free once S_j is computed, V_j only after the PV product, so separate rings
//               let each load start as early as it can)
//   warp 1      TMEM allocation (S0 | S1 | O | P0 | P1); one lane issues
//                 S_j = Q K_j^T            (A = Q smem K-major, B = K_j smem K-major) into S[j % 2]
//   warp 2      one lane issues O += P_j V_j (A = P_j from tensor memory, B = V smem MN-major)
//   warps 3..10 softmax, one TMEM lane (= one query row) per thread and one half of the
//               key columns per warp (warps w and w + 4 share rows and exchange their
//               half-row maxima): load S_j, mask (causal diagonal, keys past n; only on
//               those tiles), online max with lazy rescaling (O and l are rescaled in TMEM
//               only when the running max grows by more than 2^8), P = 2^(s log2e /
//               sqrt(D) - m) x 2^6 as fp16 pairs into tensor memory P[j % 2] (P <= 2^8 under
//               the lazy rescale, so the scaled value stays below 2^14; one exponential in
//               four on the FMA pipe, exp2_fma), row sums in fp32; V is an fp16 copy of v
//               (fp16 has 3 more mantissa bits than bf16 for P and v, which the PV product
//               needs at long sequence lengths)
// The softmax of tile j overlaps the PV product of tile j-1 and the QK^T product of
// tile j+1; with P double-buffered it waits only for the PV product of tile j-2.  Output o = O / l (bf16) and the negated row log-sum-exp in log2 units (the
// backward adds it to the scaled logits directly).
#pragma once

#include "common.cuh"

namespace jenga {

constexpr int ATC_ROWS = 128;
constexpr int ATC_K_STAGES = 3;
constexpr int ATC_V_STAGES = 3;
constexpr int ATC_BOX = 128 * 64 * 2;     // 16 KB: 128 rows x 64 bf16
constexpr int ATC_TILE = 2 * ATC_BOX;      // 32 KB: 128 x 128
constexpr int ATC_Q_OFF = 0;
constexpr int ATC_K_OFF = ATC_TILE;                             // K stage s at + s * TILE
constexpr int ATC_V_OFF = ATC_K_OFF + ATC_K_STAGES * ATC_TILE;  // V stage s at + s * TILE
constexpr int ATC_XM_OFF = ATC_V_OFF + ATC_V_STAGES * ATC_TILE;  // [2 halves][128 rows] fp32 exchange
constexpr int ATC_BAR_OFF = ATC_XM_OFF + 2 * 128 * 4;
constexpr int ATC_SMEM = ATC_BAR_OFF + 256 + 1024;
static_assert(ATC_SMEM <= 232448, "shared memory per CTA");
constexpr int ATC_THREADS = 352;

__global__ void __launch_bounds__(ATC_THREADS, 1)
    attn_fwd_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, bf16* __restrict__ o, int64_t ldo,
                       float* __restrict__ lse, int64_t lse_ld, const int32_t* __restrict__ n_valid, int valid_mult,
                       int n_cap, float scale_log2, bf16* __restrict__ o_lo) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + ATC_BAR_OFF);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;                        // [K_STAGES]
  uint64_t* k_empty = k_full + ATC_K_STAGES;          // [K_STAGES]
  uint64_t* v_full = k_empty + ATC_K_STAGES;          // [V_STAGES]
  uint64_t* v_empty = v_full + ATC_V_STAGES;          // [V_STAGES]
  uint64_t* s_full = v_empty + ATC_V_STAGES;          // [2]
  uint64_t* s_free = s_full + 2;                      // [2]
  uint64_t* p_full = s_free + 2;                      // [2] P_j written (8 softmax warps)
  uint64_t* p_free = p_full + 2;                      // [2] PV product of P_j complete
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(p_free + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.y;
  int n = n_valid ? (*n_valid) * valid_mult : n_cap;
  n = n < n_cap ? n : n_cap;
  const int qt = gridDim.x - 1 - blockIdx.x;  // longest query tiles first
  const int q0 = qt * ATC_ROWS;
  if (q0 >= n) return;
  const int nj = qt + 1;
  const int col = h * 128;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < ATC_K_STAGES; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
    }
    for (int s = 0; s < ATC_V_STAGES; ++s) {
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&s_full[s], 1);
      mbar_init(&s_free[s], 8);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&p_full[s], 8);
      mbar_init(&p_free[s], 1);
    }
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
  const uint32_t tO = tmem + 256, tP = tmem + 384;  // P[b] at tP + 64 b (bf16 pairs)

  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
    mbar_arrive_expect_tx(q_full, ATC_TILE);
    tma_load_2d(smem + ATC_Q_OFF, &tmQ, q_full, col, q0);
    tma_load_2d(smem + ATC_Q_OFF + ATC_BOX, &tmQ, q_full, col + 64, q0);
    // in order K_0 V_0 K_1 V_1 ...: K_j waits for S_{j-3}, V_j for the PV product of tile
    // j-3, both issued before anything that needs K_j or V_j
    for (int j = 0; j < nj; ++j) {
      const int sk = j % ATC_K_STAGES, sv = j % ATC_V_STAGES;
      if (j >= ATC_K_STAGES && !mbar_wait_at(&k_empty[sk], ((j / ATC_K_STAGES) - 1) & 1, 101, (qt << 16) | j)) break;
      uint8_t* kd = smem + ATC_K_OFF + sk * ATC_TILE;
      mbar_arrive_expect_tx(&k_full[sk], ATC_TILE);
      tma_load_2d(kd, &tmK, &k_full[sk], col, j * ATC_ROWS);
      tma_load_2d(kd + ATC_BOX, &tmK, &k_full[sk], col + 64, j * ATC_ROWS);
      if (j >= ATC_V_STAGES && !mbar_wait_at(&v_empty[sv], ((j / ATC_V_STAGES) - 1) & 1, 110, (qt << 16) | j)) break;
      uint8_t* vd = smem + ATC_V_OFF + sv * ATC_TILE;
      mbar_arrive_expect_tx(&v_full[sv], ATC_TILE);
      tma_load_2d(vd, &tmV, &v_full[sv], col, j * ATC_ROWS);
      tma_load_2d(vd + ATC_BOX, &tmV, &v_full[sv], col + 64, j * ATC_ROWS);
    }
  } else if (warp == 1 && lane == 0) {
    // S_j = Q K_j^T (warp 2 issues the PV products: a warp can issue a tcgen05.mma only
    // every ~100 clocks, so one issuer would cap these M 128 x N 128 products near 60%)
    constexpr uint32_t idesc_s = umma_idesc_bf16(128, 128);
    const uint32_t qa = smem_u32(smem + ATC_Q_OFF);
    bool ok = mbar_wait_at(q_full, 0, 102, qt << 16);
    for (int j = 0; ok && j < nj; ++j) {
      const int s = j % ATC_K_STAGES, sb = j & 1;
      if (!mbar_wait_at(&k_full[s], (j / ATC_K_STAGES) & 1, 104, (qt << 16) | j)) break;
      if (j >= 2 && !mbar_wait_at(&s_free[sb], ((j >> 1) - 1) & 1, 105, (qt << 16) | j)) break;
      tc_fence_after();
      const uint32_t ka = smem_u32(smem + ATC_K_OFF + s * ATC_TILE);
#pragma unroll
      for (int kc = 0; kc < 2; ++kc)
#pragma unroll
        for (int k = 0; k < 4; ++k)
          umma_bf16(tmem + sb * 128, umma_desc_k_sw128(qa + kc * ATC_BOX + k * 32),
                    umma_desc_k_sw128(ka + kc * ATC_BOX + k * 32), idesc_s, (kc | k) ? 1u : 0u);
      umma_commit(&k_empty[s]);
      umma_commit(&s_full[sb]);
    }
  } else if (warp == 2 && lane == 0) {
    // O += P_j V_j once the softmax has written P_j
    constexpr uint32_t idesc_o = umma_idesc_bf16_bmn(128, 128) & ~((7u << 7) | (7u << 10));  // fp16 P, V
    for (int j = 0; j < nj; ++j) {
      const int sv = j % ATC_V_STAGES, b = j & 1;
      if (!mbar_wait_at(&p_full[b], (j >> 1) & 1, 103, (qt << 16) | j)) break;
      if (!mbar_wait_at(&v_full[sv], (j / ATC_V_STAGES) & 1, 111, (qt << 16) | j)) break;
      tc_fence_after();
      const uint32_t va = smem_u32(smem + ATC_V_OFF + sv * ATC_TILE);
#pragma unroll
      for (int ks = 0; ks < 8; ++ks)  // K = 128 keys in steps of 16 (8 TMEM columns of P)
        umma_bf16_ts(tO, tP + b * 64 + ks * 8, umma_desc_mn_sw128(va + ks * 2048, ATC_BOX), idesc_o,
                     (j > 0 || ks > 0) ? 1u : 0u);
      umma_commit(&v_empty[sv]);
      umma_commit(&p_free[b]);
    }
  } else if (warp >= 3) {
    // eight softmax warps: warp w reads TMEM lanes 32 * (w % 4) (its 32 query rows) and
    // half hf = (w - 3) / 4 of every tile's 128 key columns; the two warps of a pair
    // (w, w + 4) exchange their half-row maxima through shared memory each tile
    const int quarter = warp & 3;
    const int hf = (warp - 3) >> 2;
    const int r = quarter * 32 + lane;
    const int qrow = q0 + r;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    float* xm = reinterpret_cast<float*>(smem + ATC_XM_OFF);  // [2 halves][128 rows]
    const int pair_bar = 1 + quarter;
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < nj; ++j) {
      const int sb = j & 1;
      // both warps of a pair must reach every named barrier, so a failed wait (here, or
      // one recorded in the previous tile) ends the loop for the pair at this point only
      ok = pair_all(ok && __all_sync(0xffffffffu, mbar_wait_at(&s_full[sb], (j >> 1) & 1, 106, (qt << 16) | j)),
                    pair_bar);
      if (!ok) break;
      tc_fence_after();
      uint32_t v[64];
      tmem_ld32_nowait(tmem + lane_off + sb * 128 + hf * 64, v);
      tmem_ld32_nowait(tmem + lane_off + sb * 128 + hf * 64 + 32, v + 32);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_free[sb]);
      const int key0 = j * ATC_ROWS;
      const bool full = (j < qt) && (key0 + ATC_ROWS <= n);  // CTA-uniform
      float mx = -INFINITY;
      if (full) {
#pragma unroll
        for (int c = 0; c < 64; ++c) mx = fmaxf(mx, __uint_as_float(v[c]));
      } else {
        const int lim = min(n - key0, (j == qt) ? r + 1 : ATC_ROWS) - hf * 64;  // valid keys: c < lim
#pragma unroll
        for (int c = 0; c < 64; ++c) {
          const float x = (c < lim) ? __uint_as_float(v[c]) : -INFINITY;
          v[c] = __float_as_uint(x);
          mx = fmaxf(mx, x);
        }
      }
      xm[hf * 128 + r] = mx;
      asm volatile("bar.sync %0, 64;" ::"r"(pair_bar) : "memory");
      const float mxs = fmaxf(mx, xm[(1 - hf) * 128 + r]) * scale_log2;
      bool waited = false;
      // tcgen05.ld / tcgen05.st are warp-collective: the rescale decision must be the
      // same for all 32 rows of the warp (rows that need no rescale use factor 1); both
      // warps of the pair see the same maxima, so they decide alike
      const bool rescale = (j > 0) && __any_sync(0xffffffffu, mxs > m_used + 8.f);
      if (j == 0) {
        m_used = mxs;
      } else if (rescale) {
        // rescale this half's 64 output columns: the PV product of tile j-1 must have landed
        // (a failed wait skips the TMEM access and ends the pair's loop at the next tile)
        waited = true;
        if (__all_sync(0xffffffffu, mbar_wait_at(&p_free[(j - 1) & 1], ((j - 1) >> 1) & 1, 107, (qt << 16) | j))) {
          tc_fence_after();
          const float m_new = fmaxf(m_used, mxs);
          const float f = fast_exp2(m_used - m_new);
          l *= f;
#pragma unroll 1
          for (int cc = 0; cc < 2; ++cc) {
            uint32_t ob[32];
            tmem_ld32_nowait(tO + lane_off + hf * 64 + cc * 32, ob);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) ob[i] = __float_as_uint(__uint_as_float(ob[i]) * f);
            tmem_st32(tO + lane_off + hf * 64 + cc * 32, ob);
          }
          tmem_wait_st();
          m_used = m_new;
        } else {
          ok = false;
        }
      }
      float ps[4] = {0.f, 0.f, 0.f, 0.f};
      uint32_t pk[32];
      if (full) {
#pragma unroll
        for (int c = 0; c < 64; c += 2) {
          const float x0 = fmaf(__uint_as_float(v[c]), scale_log2, -m_used);
          const float x1 = fmaf(__uint_as_float(v[c + 1]), scale_log2, -m_used);
          const float a = fast_exp2(x0);
          const float b2 = ((c & 3) == 2) ? exp2_fma<64>(x1) : fast_exp2(x1);  // 1 in 4 on the FMA pipe
          const __half2 hp = __floats2half2_rn(a * 64.f, b2 * 64.f);
          pk[c >> 1] = *reinterpret_cast<const uint32_t*>(&hp);
          ps[(c >> 1) & 3] += a + b2;
        }
      } else {  // masked entries are -inf: ex2 gives exactly 0 (exp2_fma would floor at 2^-125)
#pragma unroll
        for (int c = 0; c < 64; c += 2) {
          const float a = fast_exp2(fmaf(__uint_as_float(v[c]), scale_log2, -m_used));
          const float b2 = fast_exp2(fmaf(__uint_as_float(v[c + 1]), scale_log2, -m_used));
          const __half2 hp = __floats2half2_rn(a * 64.f, b2 * 64.f);
          pk[c >> 1] = *reinterpret_cast<const uint32_t*>(&hp);
          ps[(c >> 1) & 3] += a + b2;
        }
      }
      l += (ps[0] + ps[1]) + (ps[2] + ps[3]);
      // P buffer j % 2 is free once the PV product of tile j-2 completed (implied by the
      // wait for tile j-1 a rescale made); a failed wait skips the TMEM store and ends the
      // pair's loop at the next tile
      const int pb = j & 1;
      if (j >= 2 && !waited &&
          !__all_sync(0xffffffffu, mbar_wait_at(&p_free[pb], ((j >> 1) - 1) & 1, 108, (qt << 16) | j)))
        ok = false;
      if (ok) {
        tmem_st32(tP + lane_off + pb * 64 + hf * 32, pk);  // keys 64 hf .. 64 hf + 63 as fp16 pairs
        tmem_wait_st();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[pb]);
    }
    const bool fin =
        pair_all(ok && mbar_wait_at(&p_free[(nj - 1) & 1], ((nj - 1) >> 1) & 1, 109, (qt << 16) | nj), pair_bar);
    // merge the two halves' row sums (same maxima history, so they add directly)
    asm volatile("bar.sync %0, 64;" ::"r"(pair_bar) : "memory");
    xm[hf * 128 + r] = l;
    asm volatile("bar.sync %0, 64;" ::"r"(pair_bar) : "memory");
    const float l_row = l + xm[(1 - hf) * 128 + r];
    if (__all_sync(0xffffffffu, fin)) {  // warp-uniform: the loads below are collective
      tc_fence_after();
      const float inv = 1.f / (64.f * l_row);  // P entered the PV product scaled by 2^6
      const bool row_ok = qrow < n;
#pragma unroll 1
      for (int cc = 0; cc < 2; ++cc) {
        const int c0 = hf * 64 + cc * 32;
        uint32_t ob[32];
        tmem_ld32_nowait(tO + lane_off + c0, ob);
        tmem_wait_ld();
        if (row_ok) {
          uint4* dst = reinterpret_cast<uint4*>(o + (int64_t)qrow * ldo + col + c0);
          uint4* dlo = o_lo ? reinterpret_cast<uint4*>(o_lo + (int64_t)qrow * ldo + col + c0) : nullptr;
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            uint32_t w[4], wl[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const float x0 = __uint_as_float(ob[q4 * 8 + 2 * i]) * inv;
              const float x1 = __uint_as_float(ob[q4 * 8 + 2 * i + 1]) * inv;
              w[i] = pack_bf2(x0, x1);
              // the rounding residual (o = hi + lo to ~16 bits) for the backward's Delta = dO . o,
              // which cancels strongly on rows that attend to few keys
              const __nv_bfloat162 hb = *reinterpret_cast<const __nv_bfloat162*>(&w[i]);
              const float2 hf2 = __bfloat1622float2(hb);
              wl[i] = pack_bf2(x0 - hf2.x, x1 - hf2.y);
            }
            dst[q4] = make_uint4(w[0], w[1], w[2], w[3]);
            if (dlo) dlo[q4] = make_uint4(wl[0], wl[1], wl[2], wl[3]);
          }
        }
      }
      // negated row log-sum-exp in log2 units: the backward's exponent addend
      if (row_ok && hf == 0) lse[(int64_t)h * lse_ld + qrow] = -(m_used + __log2f(l_row));
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
