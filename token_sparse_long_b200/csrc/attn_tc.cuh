// tcgen05 causal attention forward over the retained tokens (head_dim 128).
//
// One CTA per (128-query tile, head), 192 threads:
//   warp 0      TMA: the Q tile once, then (K_j, V_j) pairs through a 2-stage ring
//   warp 1      TMEM allocation (S0 | S1 | O, 384 of 512 columns); one lane issues
//                 S_j = Q K_j^T            (A = Q smem K-major, B = K_j smem K-major) into S[j % 2]
//                 O  += P_{j-1} V_{j-1}    (A = P smem K-major, B = V smem MN-major) into O
//   warps 2..5  softmax, one TMEM lane (= one query row) per thread: load S_j, mask
//               (causal diagonal, keys past n), online max with lazy rescaling (O and l
//               are rescaled in TMEM only when the running max grows by more than 2^8),
//               P = 2^(s log2e / sqrt(D) - m) as bf16 into a 128-byte-swizzled smem tile
// The softmax of tile j overlaps the PV product of tile j-1 and the QK^T product of
// tile j+1.  Output o = O / l (bf16) and the row log-sum-exp (natural log).
#pragma once

#include "common.cuh"

namespace jenga {

constexpr int ATC_ROWS = 128;
constexpr int ATC_KV_STAGES = 2;
constexpr int ATC_BOX = 128 * 64 * 2;     // 16 KB: 128 rows x 64 bf16
constexpr int ATC_TILE = 2 * ATC_BOX;      // 32 KB: 128 x 128
constexpr int ATC_Q_OFF = 0;
constexpr int ATC_KV_OFF = ATC_TILE;                                  // stage s: K at +2s*TILE, V at +(2s+1)*TILE
constexpr int ATC_P_OFF = ATC_KV_OFF + 2 * ATC_KV_STAGES * ATC_TILE;
constexpr int ATC_BAR_OFF = ATC_P_OFF + ATC_TILE;
constexpr int ATC_SMEM = ATC_BAR_OFF + 256 + 1024;
constexpr int ATC_THREADS = 192;

__global__ void __launch_bounds__(ATC_THREADS, 1)
    attn_fwd_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, bf16* __restrict__ o, int64_t ldo,
                       float* __restrict__ lse, int64_t lse_ld, const int32_t* __restrict__ n_valid, int valid_mult,
                       int n_cap, float scale_log2) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + ATC_BAR_OFF);
  uint64_t* q_full = bars;
  uint64_t* kv_full = bars + 1;                       // [2]
  uint64_t* kv_empty = kv_full + ATC_KV_STAGES;       // [2]
  uint64_t* s_full = kv_empty + ATC_KV_STAGES;        // [2]
  uint64_t* s_free = s_full + 2;                      // [2]
  uint64_t* p_full = s_free + 2;
  uint64_t* pv_done = p_full + 1;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(pv_done + 1);

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
    for (int s = 0; s < ATC_KV_STAGES; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&s_full[s], 1);
      mbar_init(&s_free[s], 4);
    }
    mbar_init(p_full, 4);
    mbar_init(pv_done, 1);
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
  const uint32_t tO = tmem + 256;

  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
    mbar_arrive_expect_tx(q_full, ATC_TILE);
    tma_load_2d(smem + ATC_Q_OFF, &tmQ, q_full, col, q0);
    tma_load_2d(smem + ATC_Q_OFF + ATC_BOX, &tmQ, q_full, col + 64, q0);
    for (int j = 0; j < nj; ++j) {
      const int s = j % ATC_KV_STAGES;
      if (j >= ATC_KV_STAGES && !mbar_wait_at(&kv_empty[s], ((j / ATC_KV_STAGES) - 1) & 1, 101, (qt << 16) | j)) break;
      uint8_t* kd = smem + ATC_KV_OFF + 2 * s * ATC_TILE;
      uint8_t* vd = kd + ATC_TILE;
      mbar_arrive_expect_tx(&kv_full[s], 2 * ATC_TILE);
      tma_load_2d(kd, &tmK, &kv_full[s], col, j * ATC_ROWS);
      tma_load_2d(kd + ATC_BOX, &tmK, &kv_full[s], col + 64, j * ATC_ROWS);
      tma_load_2d(vd, &tmV, &kv_full[s], col, j * ATC_ROWS);
      tma_load_2d(vd + ATC_BOX, &tmV, &kv_full[s], col + 64, j * ATC_ROWS);
    }
  } else if (warp == 1 && lane == 0) {
    constexpr uint32_t idesc_s = umma_idesc_bf16(128, 128);
    constexpr uint32_t idesc_o = umma_idesc_bf16_bmn(128, 128);
    const uint32_t qa = smem_u32(smem + ATC_Q_OFF);
    const uint32_t pa = smem_u32(smem + ATC_P_OFF);
    bool ok = mbar_wait_at(q_full, 0, 102, qt << 16);
    auto issue_pv = [&](int jj) -> bool {
      if (!mbar_wait_at(p_full, jj & 1, 103, (qt << 16) | jj)) return false;
      tc_fence_after();
      const uint32_t va = smem_u32(smem + ATC_KV_OFF + (2 * (jj % ATC_KV_STAGES) + 1) * ATC_TILE);
#pragma unroll
      for (int ks = 0; ks < 8; ++ks)
        umma_bf16(tO, umma_desc_k_sw128(pa + (ks >> 2) * ATC_BOX + (ks & 3) * 32),
                  umma_desc_mn_sw128(va + ks * 2048, ATC_BOX), idesc_o, (jj > 0 || ks > 0) ? 1u : 0u);
      umma_commit(&kv_empty[jj % ATC_KV_STAGES]);
      umma_commit(pv_done);
      return true;
    };
    for (int j = 0; ok && j < nj; ++j) {
      const int s = j % ATC_KV_STAGES, sb = j & 1;
      if (!mbar_wait_at(&kv_full[s], (j / ATC_KV_STAGES) & 1, 104, (qt << 16) | j)) {
        ok = false;
        break;
      }
      if (j >= 2 && !mbar_wait_at(&s_free[sb], ((j >> 1) - 1) & 1, 105, (qt << 16) | j)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t ka = smem_u32(smem + ATC_KV_OFF + 2 * s * ATC_TILE);
#pragma unroll
      for (int kc = 0; kc < 2; ++kc)
#pragma unroll
        for (int k = 0; k < 4; ++k)
          umma_bf16(tmem + sb * 128, umma_desc_k_sw128(qa + kc * ATC_BOX + k * 32),
                    umma_desc_k_sw128(ka + kc * ATC_BOX + k * 32), idesc_s, (kc | k) ? 1u : 0u);
      umma_commit(&s_full[sb]);
      if (j >= 1 && !issue_pv(j - 1)) {
        ok = false;
        break;
      }
    }
    if (ok) issue_pv(nj - 1);
  } else if (warp >= 2) {
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const int qrow = q0 + r;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    uint8_t* P = smem + ATC_P_OFF;
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < nj; ++j) {
      const int sb = j & 1;
      if (!__all_sync(0xffffffffu, mbar_wait_at(&s_full[sb], (j >> 1) & 1, 106, (qt << 16) | j))) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t v[128];
      tmem_ld32_nowait(tmem + lane_off + sb * 128 + 0, v);
      tmem_ld32_nowait(tmem + lane_off + sb * 128 + 32, v + 32);
      tmem_ld32_nowait(tmem + lane_off + sb * 128 + 64, v + 64);
      tmem_ld32_nowait(tmem + lane_off + sb * 128 + 96, v + 96);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_free[sb]);
      const int key0 = j * ATC_ROWS;
      const int lim = min(n - key0, (j == qt) ? r + 1 : ATC_ROWS);  // valid keys: c < lim
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < 128; ++c) {
        const float x = (c < lim) ? __uint_as_float(v[c]) : -INFINITY;
        v[c] = __float_as_uint(x);
        mx = fmaxf(mx, x);
      }
      const float mxs = mx * scale_log2;
      bool waited = false;
      // tcgen05.ld / tcgen05.st are warp-collective: the rescale decision must be the
      // same for all 32 rows of the warp (rows that need no rescale use factor 1)
      const bool rescale = (j > 0) && __any_sync(0xffffffffu, mxs > m_used + 8.f);
      if (j == 0) {
        m_used = mxs;
      } else if (rescale) {
        // rescale the running output: the PV product of tile j-1 must have landed first
        const bool w_ok = mbar_wait_at(pv_done, (j - 1) & 1, 107, (qt << 16) | j);
        if (!__all_sync(0xffffffffu, w_ok)) {
          ok = false;
          break;
        }
        waited = true;
        tc_fence_after();
        const float m_new = fmaxf(m_used, mxs);
        const float f = fast_exp2(m_used - m_new);
        l *= f;
#pragma unroll 1
        for (int cc = 0; cc < 4; ++cc) {
          uint32_t ob[32];
          tmem_ld32_nowait(tO + lane_off + cc * 32, ob);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) ob[i] = __float_as_uint(__uint_as_float(ob[i]) * f);
          tmem_st32(tO + lane_off + cc * 32, ob);
        }
        tmem_wait_st();
        m_used = m_new;
      }
      float ps[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      uint32_t pk[64];
#pragma unroll
      for (int c = 0; c < 128; c += 2) {
        const float a = fast_exp2(fmaf(__uint_as_float(v[c]), scale_log2, -m_used));
        const float b2 = fast_exp2(fmaf(__uint_as_float(v[c + 1]), scale_log2, -m_used));
        __nv_bfloat162 pb = __floats2bfloat162_rn(a, b2);
        pk[c >> 1] = *reinterpret_cast<uint32_t*>(&pb);
        const float2 back = __bfloat1622float2(pb);  // sum what the PV product will use
        ps[(c >> 1) & 7] += back.x + back.y;
      }
      l += ((ps[0] + ps[1]) + (ps[2] + ps[3])) + ((ps[4] + ps[5]) + (ps[6] + ps[7]));
      // P smem tile is free once the PV product of tile j-1 completed
      if (j >= 1 && !waited) {
        const bool w_ok = mbar_wait_at(pv_done, (j - 1) & 1, 108, (qt << 16) | j);
        if (!__all_sync(0xffffffffu, w_ok)) {
          ok = false;
          break;
        }
      }
#pragma unroll
      for (int cc = 0; cc < 16; ++cc) {
        const int box = cc >> 3, ch = cc & 7;
        uint4 w = make_uint4(pk[cc * 4], pk[cc * 4 + 1], pk[cc * 4 + 2], pk[cc * 4 + 3]);
        *reinterpret_cast<uint4*>(P + box * ATC_BOX + r * 128 + ((ch ^ (r & 7)) << 4)) = w;
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full);
    }
    const bool fin = ok && mbar_wait_at(pv_done, (nj - 1) & 1, 109, (qt << 16) | nj);
    if (__all_sync(0xffffffffu, fin)) {  // warp-uniform: the loads below are collective
      tc_fence_after();
      const float inv = 1.f / l;
      const bool row_ok = qrow < n;
#pragma unroll 1
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t ob[32];
        tmem_ld32_nowait(tO + lane_off + cc * 32, ob);
        tmem_wait_ld();
        if (row_ok) {
          uint4* dst = reinterpret_cast<uint4*>(o + (int64_t)qrow * ldo + col + cc * 32);
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            uint32_t w[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              __nv_bfloat162 pb = __floats2bfloat162_rn(__uint_as_float(ob[q4 * 8 + 2 * i]) * inv,
                                                        __uint_as_float(ob[q4 * 8 + 2 * i + 1]) * inv);
              w[i] = *reinterpret_cast<uint32_t*>(&pb);
            }
            dst[q4] = make_uint4(w[0], w[1], w[2], w[3]);
          }
        }
      }
      if (row_ok) lse[(int64_t)h * lse_ld + qrow] = (m_used + __log2f(l)) * 0.6931471805599453f;
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
