// tcgen05 causal attention backward over the retained tokens (head_dim 128), one query
// segment [s0, s1) at a time (the segment-wise gradient schedule of the layer backward).
//
//   dK/dV pass  one CTA per (128-key tile, head).  K and V resident in smem; the segment's
//               64-query tiles of Q and dO stream through a 3-stage TMA ring.  Per tile:
//                 S^T  = K Q^T        dP^T = V dO^T           (TMEM, double-buffered)
//                 P^T  = 2^(S^T log2e/sqrt(D) - L_q),  dS^T = P^T (dP^T - Delta_q)   (epilogue;
//                 L_q, the forward's row log-sum-exp in log2 units, and Delta_q ride in the
//                 Q / dO stage as two 256-byte bulk copies; both are stored negated, so the
//                 epilogue's packed f32x2 arithmetic adds them)
//                 dV  += P^T dO       dK  += dS^T Q           (A: smem K-major, B: MN-major)
//               and at the end dV, dK (x 1/sqrt(D)) are added into fp32 accumulators by TMA
//               reduce-adds staged in the ring.
//   dQ pass     one CTA per (128-query tile of the segment, head).  Q and dO resident in
//               tensor memory; the 64-key tiles of K and V stream through a 5-stage ring.
//               S = Q K^T, dP = dO V^T (double-buffered), dS = P (dP - Delta), dQ += dS K;
//               dQ (x 1/sqrt(D)) stored fp32.
// A ring stage is read by the score products and the gradient product of its tile, which
// runs an epilogue later, so the rings hold 4 (Q/dO) and 5 (K/V) tiles.
// Warp roles (a warp can issue a tcgen05.mma only every ~100 clocks, so one issuer would
// cap these M 128 x N 64 / N 128 products well below the tensor peak, and an issuer that
// also waits on the epilogue stalls the products queued behind that wait):
//   dK/dV pass  0 TMA; 1 S^T, 2 dP^T, 3 dV, 4 dK issue (1 also allocates TMEM); 5..20
//               epilogue in four quads, quad c taking columns 16c .. 16c + 15 of a tile (two
//               epilogue warps per SMSP left the exponentials latency-bound)
//   dQ pass     0 TMA; 1-2 S, 3-4 dP (even / odd tiles), 5 dQ issue (1 also allocates TMEM);
//               6..21 epilogue in four quads, quad c taking key columns 16c .. 16c + 15
// Each quad covers all 128 TMEM lanes, one row per thread.  P / dS tiles are double-buffered in shared memory so the epilogue of
// tile i overlaps the gradient products of tile i-1 and the score products of tile i+1.
// Causal masking, keys / queries past the valid count, and the segment bounds are applied
// in the epilogue.  Every wait is bounded; waits that guard collective TMEM loads are voted.
// Operands are fp16 (3 more mantissa bits than bf16): fp16 copies of q, k, v, the segment's dO
// scaled by a power of two s_dO (max per-head row norm in (2^13, 2^14]), P scaled by 2^8 (P <= 1)
// and dS scaled by s_dS = 2^floor(log2(1 / Vmax)) with Vmax the largest per-head row norm of v,
// so |dS s_dS| <= |P (dP - Delta)| s_dS <= |dO_i| |v_j - o_i| s_dS <= 2^15 can never overflow
// (gscal[2] = s_dO, gscal[3] = s_dS, set on the device before the launch).  The fp32 results
// are divided by the scales again before they leave the kernels.
#pragma once

#include "common.cuh"

namespace jenga {

constexpr int ABT_BOX128 = 128 * 64 * 2;   // 16 KB box: 128 rows x 64 bf16
constexpr int ABT_BOX64 = 64 * 64 * 2;     // 8 KB box: 64 rows x 64 bf16
constexpr int DQ_EPI_WARP0 = 6;   // dQ pass: warps 0 TMA, 1-2 S, 3-4 dP, 5 dQ issue, 6 .. 21 epilogue
constexpr int DQ_EPI_WARPS = 16;
constexpr int ABT_THREADS = 32 * (DQ_EPI_WARP0 + DQ_EPI_WARPS);
constexpr int DKV_EPI_WARPS = 16;
constexpr int DKV_EPI_WARP0 = 5;  // dK/dV pass: warps 0 TMA, 1 .. 4 MMA issue, 5 .. 20 epilogue
constexpr int DKV_THREADS = 32 * (DKV_EPI_WARP0 + DKV_EPI_WARPS);

// smem layout of the dK/dV pass.  K and V are staged through the P^T / dS^T buffers and
// copied into tensor memory (the A operands of S^T and dP^T) before the first tile.
constexpr int DKV_PT_OFF = 0;                              // [2] x 128 x 64 bf16 (first: K)
constexpr int DKV_DST_OFF = DKV_PT_OFF + 2 * ABT_BOX128;   // [2] x 128 x 64 bf16 (first: V)
constexpr int DKV_RING_OFF = DKV_DST_OFF + 2 * ABT_BOX128;  // stage s: Q (2 x 8 KB), dO (2 x 8 KB)
constexpr int DKV_STAGE = 4 * ABT_BOX64;
constexpr int DKV_STAGES = 4;  // a stage lives from its load to the gradient products of its tile
constexpr int DKV_LD_OFF = DKV_RING_OFF + DKV_STAGES * DKV_STAGE;  // stage s: L (64 fp32), Delta (64 fp32)
constexpr int DKV_LD_BYTES = 512;
constexpr int DKV_F32_BOX = 128 * 32 * 4;  // 16 KB: one quad's dV or dK columns, staged in the ring
static_assert(8 * DKV_F32_BOX <= DKV_STAGES * DKV_STAGE, "final dV/dK staging fits in the ring");
constexpr int DKV_BAR_OFF = DKV_LD_OFF + DKV_STAGES * DKV_LD_BYTES;
constexpr int DKV_SMEM = DKV_BAR_OFF + 256 + 1024;

// smem layout of the dQ pass.  Q and dO are staged and copied into tensor memory (the A
// operands of S and dP) before the first tile; the Q staging then holds the dS buffers.
constexpr int DQ_Q_OFF = 0;
constexpr int DQ_DO_OFF = 2 * ABT_BOX128;
constexpr int DQ_DS_OFF = DQ_Q_OFF;                        // [2] x 128 x 64 bf16, after the copy
constexpr int DQ_RING_OFF = 4 * ABT_BOX128;                // stage s: K (2 x 8 KB), V (2 x 8 KB)
constexpr int DQ_STAGE = 4 * ABT_BOX64;
constexpr int DQ_STAGES = 5;  // a stage lives from S(j) to the dQ product of tile j
constexpr int DQ_BAR_OFF = DQ_RING_OFF + DQ_STAGES * DQ_STAGE;
constexpr int DQ_SMEM = DQ_BAR_OFF + 256 + 1024;
static_assert(DQ_SMEM <= 232448 && DKV_SMEM <= 232448, "shared memory per CTA");

// Write 32 bf16 values (packed pairs pk[0..15]) as columns [32 * half, 32 * half + 32) of
// row r of a 128 x 64 K-major tile with the 128-byte swizzle (row = 8 chunks of 16 bytes).
__device__ __forceinline__ void st_row32_sw128(uint8_t* tile, int r, int half, const uint32_t* pk);

// Write 16 bf16 values (packed pairs pk[0..7]) as columns [16 * quad, 16 * quad + 16) of row r
// of a 128 x 64 K-major tile with the 128-byte swizzle.
__device__ __forceinline__ void st_row16_sw128(uint8_t* tile, int r, int quad, const uint32_t* pk) {
#pragma unroll
  for (int c = 0; c < 2; ++c) {
    const int ch = quad * 2 + c;
    *reinterpret_cast<uint4*>(tile + r * 128 + ((ch ^ (r & 7)) << 4)) =
        make_uint4(pk[c * 4], pk[c * 4 + 1], pk[c * 4 + 2], pk[c * 4 + 3]);
  }
}

// fp16 forms of the instruction descriptors (operand format fields 0 = fp16)
__host__ __device__ constexpr uint32_t idesc_f16(uint32_t bf16_desc) { return bf16_desc & ~((7u << 7) | (7u << 10)); }

// two floats -> packed fp16 pair (round to nearest even), a in the low half
__device__ __forceinline__ uint32_t pack_h2(float a, float b) {
  __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ void st_row32_sw128(uint8_t* tile, int r, int half, const uint32_t* pk) {
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const int ch = half * 4 + c;
    *reinterpret_cast<uint4*>(tile + r * 128 + ((ch ^ (r & 7)) << 4)) =
        make_uint4(pk[c * 4], pk[c * 4 + 1], pk[c * 4 + 2], pk[c * 4 + 3]);
  }
}

// ------------------------------------------------------------------ dK / dV
__global__ void __launch_bounds__(DKV_THREADS, 1)
    attn_bwd_dkdv_tc_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                            const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmDO,
                            const float* __restrict__ lse, int64_t lse_ld, const float* __restrict__ delta,
                            int64_t delta_ld, const __grid_constant__ CUtensorMap tmDK,
                            const __grid_constant__ CUtensorMap tmDV, int s0, int s1,
                            const int32_t* __restrict__ n_valid, int valid_mult, int n_cap, float scale_log2,
                            float scale, const float* __restrict__ gscal) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + DKV_BAR_OFF);
  uint64_t* kv_full = bars;
  uint64_t* q_full = bars + 1;                // [DKV_STAGES]
  uint64_t* q_empty = q_full + DKV_STAGES;    // [DKV_STAGES]
  uint64_t* s_full = q_empty + DKV_STAGES;    // S^T / dP^T of the current tile written
  uint64_t* s_free = s_full + 1;              // ... and read by the epilogue
  uint64_t* pd_full = s_free + 1;   // [2]
  uint64_t* pd_free = pd_full + 2;  // [2]
  uint64_t* done = pd_free + 2;
  uint64_t* kv_tmem = done + 1;     // K and V are in tensor memory
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(kv_tmem + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.y;
  int n = n_valid ? (*n_valid) * valid_mult : n_cap;
  n = n < n_cap ? n : n_cap;
  const int send = min(s1, n);
  const int k0 = blockIdx.x * 128;
  if (k0 >= send || s0 >= send) return;
  const int qa0 = max(k0, s0) >> 6;  // first 64-query tile
  const int qa1 = (send + 63) >> 6;  // one past the last
  const int nq = qa1 - qa0;
  if (nq <= 0) return;
  const int col = h * 128;

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    for (int s = 0; s < DKV_STAGES; ++s) {
      mbar_init(&q_full[s], 1);
      mbar_init(&q_empty[s], 4);  // all four products read the stage
    }
    mbar_init(s_full, 2);
    mbar_init(s_free, DKV_EPI_WARPS);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&pd_full[s], DKV_EPI_WARPS);
      mbar_init(&pd_free[s], 2);
    }
    mbar_init(done, 2);
    mbar_init(kv_tmem, 8);
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
  // TMEM columns: dV 0..127, dK 128..255, K 256..319, V 320..383 (bf16 pairs, A operands),
  // S^T 384..447, dP^T 448..511
  const uint32_t tdV = tmem, tdK = tmem + 128, tK = tmem + 256, tV = tmem + 320, tS = tmem + 384, tP = tmem + 448;

  if (warp == 0 && lane == 0) {
    mbar_arrive_expect_tx(kv_full, 4 * ABT_BOX128);
    tma_load_2d(smem + DKV_PT_OFF, &tmK, kv_full, col, k0);
    tma_load_2d(smem + DKV_PT_OFF + ABT_BOX128, &tmK, kv_full, col + 64, k0);
    tma_load_2d(smem + DKV_DST_OFF, &tmV, kv_full, col, k0);
    tma_load_2d(smem + DKV_DST_OFF + ABT_BOX128, &tmV, kv_full, col + 64, k0);
    for (int i = 0; i < nq; ++i) {
      const int s = i % DKV_STAGES;
      if (i >= DKV_STAGES && !mbar_wait_at(&q_empty[s], ((i / DKV_STAGES) - 1) & 1, 121, i)) break;
      uint8_t* st = smem + DKV_RING_OFF + s * DKV_STAGE;
      const int qrow = (qa0 + i) * 64;
      uint8_t* ldst = smem + DKV_LD_OFF + s * DKV_LD_BYTES;
      mbar_arrive_expect_tx(&q_full[s], DKV_STAGE + DKV_LD_BYTES);
      tma_load_2d(st, &tmQ, &q_full[s], col, qrow);
      tma_load_2d(st + ABT_BOX64, &tmQ, &q_full[s], col + 64, qrow);
      tma_load_2d(st + 2 * ABT_BOX64, &tmDO, &q_full[s], col, qrow - s0);
      tma_load_2d(st + 3 * ABT_BOX64, &tmDO, &q_full[s], col + 64, qrow - s0);
      // the tile's 64 query log-sum-exps (log2 units) and Delta values
      bulk_load_1d(ldst, lse + (int64_t)h * lse_ld + qrow, 256, &q_full[s]);
      bulk_load_1d(ldst + 256, delta + (int64_t)h * delta_ld + (qrow - s0), 256, &q_full[s]);
    }
  } else if ((warp == 1 || warp == 2) && lane == 0) {
    // score products, one issuing warp each (a warp can issue a tcgen05.mma only every ~100
    // clocks): warp 1 S^T = K Q^T, warp 2 dP^T = V dO^T, A (K, V) from tensor memory and B
    // (Q, dO) from the ring, independent of the gradient products.  One accumulator each:
    // tile i + 1's product starts as soon as the epilogue has read tile i's.
    const bool s_chain = (warp == 1);
    constexpr uint32_t idesc_s = idesc_f16(umma_idesc_bf16(128, 64));
    const uint32_t ta = s_chain ? tK : tV;
    const uint32_t acc_s = s_chain ? tS : tP;
    const int b_s_off = s_chain ? 0 : 2 * ABT_BOX64;  // Q or dO
    bool ok = mbar_wait_at(kv_tmem, 0, 122, 0);
    for (int i = 0; ok && i < nq; ++i) {
      const int rs = i % DKV_STAGES;
      if (!mbar_wait_at(&q_full[rs], (i / DKV_STAGES) & 1, 124, i)) break;
      if (i >= 1 && !mbar_wait_at(s_free, (i - 1) & 1, 125, i)) break;
      tc_fence_after();
      const uint32_t st = smem_u32(smem + DKV_RING_OFF + rs * DKV_STAGE + b_s_off);
#pragma unroll
      for (int kc = 0; kc < 2; ++kc)
#pragma unroll
        for (int k = 0; k < 4; ++k)
          umma_bf16_ts(acc_s, ta + kc * 32 + k * 8, umma_desc_k_sw128(st + kc * ABT_BOX64 + k * 32), idesc_s,
                       (kc | k) ? 1u : 0u);
      umma_commit(s_full);
      umma_commit(&q_empty[rs]);
    }
  } else if ((warp == 3 || warp == 4) && lane == 0) {
    // gradient products: warp 3 dV += P^T dO, warp 4 dK += dS^T Q, each as soon as the
    // epilogue has written tile i's P^T / dS^T
    const bool p_chain = (warp == 3);
    constexpr uint32_t idesc_g = idesc_f16(umma_idesc_bf16_bmn(128, 128));
    const uint32_t acc_g = p_chain ? tdV : tdK;
    const int gbuf_off = p_chain ? DKV_PT_OFF : DKV_DST_OFF;  // P^T or dS^T tiles
    const int b_g_off = p_chain ? 2 * ABT_BOX64 : 0;          // dO or Q
    bool ok = true;
    for (int i = 0; i < nq; ++i) {
      const int b = i & 1, rs = i % DKV_STAGES;
      if (!mbar_wait_at(&pd_full[b], (i >> 1) & 1, 123, i)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t bs = smem_u32(smem + DKV_RING_OFF + rs * DKV_STAGE + b_g_off);
      const uint32_t ga = smem_u32(smem + gbuf_off + b * ABT_BOX128);
#pragma unroll
      for (int ks = 0; ks < 4; ++ks)  // K = 64 queries in steps of 16
        umma_bf16(acc_g, umma_desc_k_sw128(ga + ks * 32), umma_desc_mn_sw128(bs + ks * 2048, ABT_BOX64), idesc_g,
                  (i > 0 || ks > 0) ? 1u : 0u);
      umma_commit(&pd_free[b]);
      umma_commit(&q_empty[rs]);
    }
    if (ok) umma_commit(done);
  } else if (warp >= DKV_EPI_WARP0) {
    // 16 epilogue warps in four quads: quad c takes query columns 16c .. 16c + 15 of every
    // 64-query tile (four warps per SMSP hide the exponential and conversion latencies)
    const int quarter = warp & 3;
    const int quad = (warp - DKV_EPI_WARP0) >> 2;
    const int r = quarter * 32 + lane;
    const int key = k0 + r;
    const uint32_t lo = (uint32_t)(quarter * 32) << 16;
    bool ok = true;
    if (quad < 2) {
      // quad 0 copies K, quad 1 V from their staging tiles into tensor memory
      if (__all_sync(0xffffffffu, mbar_wait_at(kv_full, 0, 130, 0))) {
        tile_row_to_tmem(smem + (quad == 0 ? DKV_PT_OFF : DKV_DST_OFF), r, (quad == 0 ? tK : tV) + lo);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(kv_tmem);
      } else {
        ok = false;
      }
    }
    // the staging tiles become the P^T / dS^T buffers only after every copy is done
    asm volatile("bar.sync 1, %0;" ::"n"(32 * DKV_EPI_WARPS) : "memory");
    const uint64_t sl2x2 = f2pack(scale_log2, scale_log2);
    const float s_dO = __ldg(gscal + 2), s_dS = __ldg(gscal + 3);
    const uint64_t pscale2 = f2pack(256.f, 256.f), dscale2 = f2pack(s_dS, s_dS);
    for (int i = 0; ok && i < nq; ++i) {
      const int s = i & 1, rs = i % DKV_STAGES;
      const int qbase = (qa0 + i) * 64 + quad * 16;
      // S^T(i) done implies the stage landed; the second wait makes the bulk-copied L and
      // Delta visible to these threads (the stage cannot be refilled before pd_full(i))
      if (!__all_sync(0xffffffffu, mbar_wait_at(s_full, i & 1, 126, i) &&
                                       mbar_wait_at(&q_full[rs], (i / DKV_STAGES) & 1, 129, i))) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t sv[16], dp[16];
      tmem_ld16_nowait(tS + lo + quad * 16, sv);
      tmem_ld16_nowait(tP + lo + quad * 16, dp);
      const float4* L4 = reinterpret_cast<const float4*>(smem + DKV_LD_OFF + rs * DKV_LD_BYTES) + quad * 4;
      const float4* D4 = L4 + 16;
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(s_free);
      uint32_t pk[8], dk[8];
      if (qbase >= key && qbase + 16 <= send) {  // every (query, key) pair of this row is live
        // packed pairs: x = s log2(e)/sqrt(D) - L, p = 2^x, dS = p (dP - Delta)
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) {
          const float4 Lq = L4[c4], Dq = D4[c4];  // -L, -Delta
          const uint64_t p01 = exp2_mufu_x2(
              ffma2(f2pack(__uint_as_float(sv[4 * c4]), __uint_as_float(sv[4 * c4 + 1])), sl2x2, f2pack(Lq.x, Lq.y)));
          const uint64_t p23 = exp2_mufu_x2(ffma2(f2pack(__uint_as_float(sv[4 * c4 + 2]), __uint_as_float(sv[4 * c4 + 3])),
                                                  sl2x2, f2pack(Lq.z, Lq.w)));
          const uint64_t d01 =
              fmul2(p01, fadd2(f2pack(__uint_as_float(dp[4 * c4]), __uint_as_float(dp[4 * c4 + 1])), f2pack(Dq.x, Dq.y)));
          const uint64_t d23 = fmul2(
              p23, fadd2(f2pack(__uint_as_float(dp[4 * c4 + 2]), __uint_as_float(dp[4 * c4 + 3])), f2pack(Dq.z, Dq.w)));
          float a, bb;
          f2unpack(fmul2(p01, pscale2), a, bb);
          pk[2 * c4] = pack_h2(a, bb);
          f2unpack(fmul2(p23, pscale2), a, bb);
          pk[2 * c4 + 1] = pack_h2(a, bb);
          f2unpack(fmul2(d01, dscale2), a, bb);
          dk[2 * c4] = pack_h2(a, bb);
          f2unpack(fmul2(d23, dscale2), a, bb);
          dk[2 * c4 + 1] = pack_h2(a, bb);
        }
      } else {  // causal diagonal or the segment's ragged end
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) {
          const float4 Lq = L4[c4], Dq = D4[c4];
          const float Ls[4] = {Lq.x, Lq.y, Lq.z, Lq.w};
          const float Ds[4] = {Dq.x, Dq.y, Dq.z, Dq.w};
          float p[4], d[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int c = 4 * c4 + e, q = qbase + c;
            const bool valid = (q >= key) && (q < send);
            const float pe = valid ? fast_exp2(fmaf(__uint_as_float(sv[c]), scale_log2, Ls[e])) : 0.f;
            p[e] = pe;
            d[e] = valid ? pe * (__uint_as_float(dp[c]) + Ds[e]) : 0.f;  // L, Delta past n are unset
          }
          pk[2 * c4] = pack_h2(p[0] * 256.f, p[1] * 256.f);
          pk[2 * c4 + 1] = pack_h2(p[2] * 256.f, p[3] * 256.f);
          dk[2 * c4] = pack_h2(d[0] * s_dS, d[1] * s_dS);
          dk[2 * c4 + 1] = pack_h2(d[2] * s_dS, d[3] * s_dS);
        }
      }
      // buffer s was last read by the gradient products of tile i-2
      if (i >= 2 && !__all_sync(0xffffffffu, mbar_wait_at(&pd_free[s], ((i >> 1) - 1) & 1, 127, i))) {
        ok = false;
        break;
      }
      st_row16_sw128(smem + DKV_PT_OFF + s * ABT_BOX128, r, quad, pk);
      st_row16_sw128(smem + DKV_DST_OFF + s * ABT_BOX128, r, quad, dk);
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&pd_full[s]);
    }
    // dV and dK (x 1/sqrt(D)) are added into the fp32 accumulators by TMA reduce-adds
    // (the L2 does the additions, so no read-modify-write round trips from this SM): each
    // quad stages its 32 columns of both in the ring, free once every product is done.
    // Keys past n carry exact zeros (no valid query reaches them); rows past n_cap are
    // clipped by the tensor maps.
    const bool fin = __all_sync(0xffffffffu, ok && mbar_wait_at(done, 0, 128, nq));
    uint8_t* bv = smem + DKV_RING_OFF + quad * 2 * DKV_F32_BOX;  // [128 rows][32 fp32], 128-byte swizzle
    uint8_t* bk = bv + DKV_F32_BOX;
    if (fin) {
      tc_fence_after();
      const int c0 = quad * 32;  // this quad's 32 of the 128 head dimensions
#pragma unroll 1
      for (int t = 0; t < 2; ++t) {  // dV, then dK
        uint32_t a[32];
        tmem_ld32_nowait((t ? tdK : tdV) + lo + c0, a);
        tmem_wait_ld();
        const float f = t ? scale / (s_dS * s_dO) : 1.f / (256.f * s_dO);
        uint8_t* dst = t ? bk : bv;
#pragma unroll
        for (int c = 0; c < 8; ++c)
          *reinterpret_cast<float4*>(dst + r * 128 + ((c ^ (r & 7)) << 4)) =
              make_float4(__uint_as_float(a[4 * c]) * f, __uint_as_float(a[4 * c + 1]) * f,
                          __uint_as_float(a[4 * c + 2]) * f, __uint_as_float(a[4 * c + 3]) * f);
      }
      fence_proxy_async_smem();
    }
    // every epilogue warp staged its rows (or none did: the vote is CTA-wide)
    const bool all_fin = bar_and(fin, 1, 32 * DKV_EPI_WARPS);
    if (all_fin && (warp - DKV_EPI_WARP0) % 4 == 0 && lane == 0) {
      tma_reduce_add_2d(&tmDV, bv, col + quad * 32, k0);
      tma_reduce_add_2d(&tmDK, bk, col + quad * 32, k0);
      bulk_commit_group();
      bulk_wait_group_read0();  // shared memory must outlive the reads
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------------ dQ
__global__ void __launch_bounds__(ABT_THREADS, 1)
    attn_bwd_dq_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmDO,
                          const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                          const float* __restrict__ lse, int64_t lse_ld, const float* __restrict__ delta,
                          int64_t delta_ld, const __grid_constant__ CUtensorMap tmDQ, int s0,
                          const int32_t* __restrict__ n_valid, int valid_mult, int n_cap, float scale_log2,
                          float scale, const float* __restrict__ gscal) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + DQ_BAR_OFF);
  uint64_t* qd_full = bars;
  uint64_t* kv_full = bars + 1;               // [DQ_STAGES]
  uint64_t* kv_empty = kv_full + DQ_STAGES;   // [DQ_STAGES]: S, dP and dQ products read a stage
  uint64_t* s_full = kv_empty + DQ_STAGES;    // [2]
  uint64_t* s_free = s_full + 2;     // [2]
  uint64_t* ds_full = s_free + 2;    // [2]
  uint64_t* ds_free = ds_full + 2;   // [2]
  uint64_t* done = ds_free + 2;
  uint64_t* qd_tmem = done + 1;      // Q and dO are in tensor memory
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(qd_tmem + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.y;
  int n = n_valid ? (*n_valid) * valid_mult : n_cap;
  n = n < n_cap ? n : n_cap;
  const int qt = s0 / 128 + (gridDim.x - 1 - blockIdx.x);  // longest first
  const int q0 = qt * 128;
  if (q0 >= n) return;
  const int kend = min(q0 + 128, n);
  const int nk = (kend + 63) >> 6;
  const int col = h * 128;

  if (threadIdx.x == 0) {
    mbar_init(qd_full, 1);
    for (int s = 0; s < DQ_STAGES; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 3);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&s_full[s], 2);
      mbar_init(&s_free[s], DQ_EPI_WARPS);
      mbar_init(&ds_full[s], DQ_EPI_WARPS);
      mbar_init(&ds_free[s], 1);
    }
    mbar_init(done, 1);
    mbar_init(qd_tmem, 8);
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
  // TMEM columns: S[2] 0, 64; dP[2] 128, 192; dQ 256..383; Q 384..447, dO 448..511 (bf16
  // pairs, A operands)
  const uint32_t tdQ = tmem + 256, tQ = tmem + 384, tDO = tmem + 448;

  if (warp == 0 && lane == 0) {
    mbar_arrive_expect_tx(qd_full, 4 * ABT_BOX128);
    tma_load_2d(smem + DQ_Q_OFF, &tmQ, qd_full, col, q0);
    tma_load_2d(smem + DQ_Q_OFF + ABT_BOX128, &tmQ, qd_full, col + 64, q0);
    tma_load_2d(smem + DQ_DO_OFF, &tmDO, qd_full, col, q0 - s0);
    tma_load_2d(smem + DQ_DO_OFF + ABT_BOX128, &tmDO, qd_full, col + 64, q0 - s0);
    for (int j = 0; j < nk; ++j) {
      const int s = j % DQ_STAGES;
      if (j >= DQ_STAGES && !mbar_wait_at(&kv_empty[s], ((j / DQ_STAGES) - 1) & 1, 131, j)) break;
      uint8_t* st = smem + DQ_RING_OFF + s * DQ_STAGE;
      mbar_arrive_expect_tx(&kv_full[s], DQ_STAGE);
      tma_load_2d(st, &tmK, &kv_full[s], col, j * 64);
      tma_load_2d(st + ABT_BOX64, &tmK, &kv_full[s], col + 64, j * 64);
      tma_load_2d(st + 2 * ABT_BOX64, &tmV, &kv_full[s], col, j * 64);
      tma_load_2d(st + 3 * ABT_BOX64, &tmV, &kv_full[s], col + 64, j * 64);
    }
  } else if (warp >= 1 && warp <= 4 && lane == 0) {
    // score products: warps 1 and 2 S = Q K^T, warps 3 and 4 dP = dO V^T, each warp the
    // tiles of one parity (its accumulator buffer), so the two buffers fill concurrently;
    // A (Q, dO) from tensor memory, B (K, V) from the ring
    const bool s_chain = (warp <= 2);
    const int par = (warp - 1) & 1;
    constexpr uint32_t idesc_s = idesc_f16(umma_idesc_bf16(128, 64));
    const uint32_t ta = s_chain ? tQ : tDO;
    const uint32_t acc0 = tmem + (s_chain ? 0 : 128);
    const int b_off = s_chain ? 0 : 2 * ABT_BOX64;  // K or V
    bool ok = mbar_wait_at(qd_tmem, 0, 132, 0);
    for (int j = par; ok && j < nk; j += 2) {
      const int s = j & 1, rs = j % DQ_STAGES;
      if (!mbar_wait_at(&kv_full[rs], (j / DQ_STAGES) & 1, 134, j)) break;
      if (j >= 2 && !mbar_wait_at(&s_free[s], ((j >> 1) - 1) & 1, 135, j)) break;
      tc_fence_after();
      const uint32_t st = smem_u32(smem + DQ_RING_OFF + rs * DQ_STAGE + b_off);
#pragma unroll
      for (int kc = 0; kc < 2; ++kc)
#pragma unroll
        for (int k = 0; k < 4; ++k)
          umma_bf16_ts(acc0 + s * 64, ta + kc * 32 + k * 8, umma_desc_k_sw128(st + kc * ABT_BOX64 + k * 32), idesc_s,
                       (kc | k) ? 1u : 0u);
      umma_commit(&s_full[s]);
      umma_commit(&kv_empty[rs]);
    }
  } else if (warp == 5 && lane == 0) {
    // dQ += dS K as soon as the epilogue has written tile j's dS (A: smem K-major, B: the
    // ring's K tile MN-major)
    constexpr uint32_t idesc_g = idesc_f16(umma_idesc_bf16_bmn(128, 128));
    bool ok = true;
    for (int j = 0; j < nk; ++j) {
      const int b = j & 1, rs = j % DQ_STAGES;
      if (!mbar_wait_at(&ds_full[b], (j >> 1) & 1, 133, j)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t ks_ = smem_u32(smem + DQ_RING_OFF + rs * DQ_STAGE);
      const uint32_t dsa = smem_u32(smem + DQ_DS_OFF + b * ABT_BOX128);
#pragma unroll
      for (int ks = 0; ks < 4; ++ks)
        umma_bf16(tdQ, umma_desc_k_sw128(dsa + ks * 32), umma_desc_mn_sw128(ks_ + ks * 2048, ABT_BOX64), idesc_g,
                  (j > 0 || ks > 0) ? 1u : 0u);
      umma_commit(&ds_free[b]);
      umma_commit(&kv_empty[rs]);
    }
    if (ok) umma_commit(done);
  } else if (warp >= DQ_EPI_WARP0) {
    // 16 epilogue warps in four quads: quad c takes key columns 16c .. 16c + 15 of every
    // 64-key tile, one query row per thread
    const int quarter = warp & 3;
    const int quad = (warp - DQ_EPI_WARP0) >> 2;
    const int r = quarter * 32 + lane;
    const int q = q0 + r;
    const uint32_t lo = (uint32_t)(quarter * 32) << 16;
    const bool qvalid = q < n;
    static_assert(4 * DKV_F32_BOX <= DQ_STAGES * DQ_STAGE, "final dQ staging fits in the ring");
    const float L = qvalid ? lse[(int64_t)h * lse_ld + q] : 0.f;  // -L, log2 units
    const float Dq = qvalid ? delta[(int64_t)h * delta_ld + q - s0] : 0.f;  // -Delta
    const uint64_t sl2x2 = f2pack(scale_log2, scale_log2), nL2 = f2pack(L, L), nD2 = f2pack(Dq, Dq);
    const float s_dO = __ldg(gscal + 2), s_dS = __ldg(gscal + 3);
    const uint64_t dscale2 = f2pack(s_dS, s_dS);
    bool ok = true;
    if (quad < 2) {
      // quad 0 copies Q, quad 1 dO from their staging tiles into tensor memory
      if (__all_sync(0xffffffffu, mbar_wait_at(qd_full, 0, 139, 0))) {
        tile_row_to_tmem(smem + (quad == 0 ? DQ_Q_OFF : DQ_DO_OFF), r, (quad == 0 ? tQ : tDO) + lo);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(qd_tmem);
      } else {
        ok = false;
      }
    }
    // the Q staging tiles become the dS buffers only after every copy is done
    asm volatile("bar.sync 1, %0;" ::"n"(32 * DQ_EPI_WARPS) : "memory");
    for (int j = 0; ok && j < nk; ++j) {
      const int s = j & 1;
      if (!__all_sync(0xffffffffu, mbar_wait_at(&s_full[s], (j >> 1) & 1, 136, j))) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t sv[16], dp[16];
      tmem_ld16_nowait(tmem + lo + s * 64 + quad * 16, sv);
      tmem_ld16_nowait(tmem + lo + 128 + s * 64 + quad * 16, dp);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_free[s]);
      const int lim = qvalid ? min(q + 1, n) - j * 64 - quad * 16 : 0;  // valid keys of this quad: c < lim
      uint32_t dk[8];
      if (lim >= 16) {  // every key of this quad is live for this row
#pragma unroll
        for (int c = 0; c < 16; c += 2) {
          const uint64_t p2 =
              exp2_mufu_x2(ffma2(f2pack(__uint_as_float(sv[c]), __uint_as_float(sv[c + 1])), sl2x2, nL2));
          const uint64_t d2 = fmul2(p2, fadd2(f2pack(__uint_as_float(dp[c]), __uint_as_float(dp[c + 1])), nD2));
          float a, bb;
          f2unpack(fmul2(d2, dscale2), a, bb);
          dk[c >> 1] = pack_h2(a, bb);
        }
      } else {
#pragma unroll
        for (int c = 0; c < 16; c += 2) {
          float d2[2];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const bool valid = c + e < lim;
            const float pe = valid ? fast_exp2(fmaf(__uint_as_float(sv[c + e]), scale_log2, L)) : 0.f;
            d2[e] = valid ? pe * (__uint_as_float(dp[c + e]) + Dq) : 0.f;
          }
          dk[c >> 1] = pack_h2(d2[0] * s_dS, d2[1] * s_dS);
        }
      }
      if (j >= 2 && !__all_sync(0xffffffffu, mbar_wait_at(&ds_free[s], ((j >> 1) - 1) & 1, 137, j))) {
        ok = false;
        break;
      }
      st_row16_sw128(smem + DQ_DS_OFF + s * ABT_BOX128, r, quad, dk);
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ds_full[s]);
    }
    // dQ (x 1/sqrt(D)) leaves through TMA stores: each quad stages its 32 columns in the
    // ring (free once every product is done); rows past the segment are clipped by the
    // tensor map, and rows of queries past n hold exact zeros
    const bool fin = __all_sync(0xffffffffu, ok && mbar_wait_at(done, 0, 138, nk));
    uint8_t* box = smem + DQ_RING_OFF + quad * DKV_F32_BOX;  // [128 rows][32 fp32], 128-byte swizzle
    if (fin) {
      tc_fence_after();
      uint32_t a[32];
      tmem_ld32_nowait(tdQ + lo + quad * 32, a);
      tmem_wait_ld();
      const float f = scale / (s_dS * s_dO);
#pragma unroll
      for (int c = 0; c < 8; ++c)
        *reinterpret_cast<float4*>(box + r * 128 + ((c ^ (r & 7)) << 4)) =
            make_float4(__uint_as_float(a[4 * c]) * f, __uint_as_float(a[4 * c + 1]) * f,
                        __uint_as_float(a[4 * c + 2]) * f, __uint_as_float(a[4 * c + 3]) * f);
      fence_proxy_async_smem();
    }
    const bool all_fin = bar_and(fin, 1, 32 * DQ_EPI_WARPS);
    if (all_fin && (warp - DQ_EPI_WARP0) % 4 == 0 && lane == 0) {
      tma_store_2d(&tmDQ, box, col + quad * 32, q0 - s0);
      bulk_commit_group();
      bulk_wait_group_read0();  // shared memory must outlive the reads
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
