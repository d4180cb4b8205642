// tcgen05 GEMM for the retained-token layer projections (sm_100a).
//
//   C[M, N] = A1 B1^T (+ A2 B2^T (+ A3 B3^T))     bf16 (or fp16) in, fp32 accumulate
//
// All operands are K-major (row-major [rows, K]).  The optional second and third
// operand pairs extend the reduction: they fold the LoRA up-projection into the QKV
// projection and the LoRA down-projection's input gradient into the dX GEMM.  A
// gradient operand enters as fp16 rows scaled by powers of two into fp16's range; the
// epilogue multiplies each output row by the inverse scale (EpiParams::row_scale).
//
// Structure: persistent, one CTA per SM walking the 128 x BN output tiles in a fixed
// stride (tile = blockIdx.x, + gridDim.x, ...; N tiles fastest), 192 threads:
//   warp 0      TMA producer: 128 x 64 A box + BN x 64 B box per stage into a
//               STAGES-deep shared-memory ring (128-byte swizzle) that runs on across
//               tiles, mbarrier tx counts
//   warp 1      allocates 2 x BN TMEM columns (two accumulators); one lane issues
//               tcgen05.mma (M=128, N=BN, K=16) x 4 per stage into the accumulator of the
//               tile's parity and tcgen05.commit to release the stage
//   warps 2..5  epilogue: tcgen05.ld 32 columns at a time of their TMEM lane quarter
//               (row = 32 * (warp % 4) + lane), release the accumulator after its last
//               load, fused epilogue, global stores -- overlapping the next tile's MMAs
// With one tile per CTA the tensor core idled through every tile's prologue (barrier
// set-up, TMEM allocation, first TMA round trip) and epilogue stores; K = 4096 projections
// ran at about half the rate of the long-K ones.
// Every wait is bounded (see mbar_wait); rows past the device-side valid count are
// neither loaded usefully nor stored.
#pragma once

#include "common.cuh"

namespace jenga {

constexpr int GEMM_BM = 128;
constexpr int GEMM_BK = 64;
constexpr int GEMM_THREADS = 192;

enum GemmEpi : int {
  EPI_STORE_BF16 = 0,   // out[m, n] = bf16(acc * alpha)
  EPI_STORE_F32 = 1,    // out[m, n] = acc * alpha (fp32)
  EPI_SCATTER_ADD = 2,  // x[row(m), n] = bf16(x + acc); aux[m, n] = same value (optional)
  EPI_SWIGLU = 3,       // 64-col groups (gate, up) -> out[m, n/2 + j] = bf16(silu(g) * u);
                        // with aux: (g, u) also stored fp16 in the interleaved layout
  EPI_QKV_ROPE = 4,     // q/k/v sections of width hd; RoPE(pos(m)) on q and k -> bf16
  EPI_SWIGLU_BWD = 5,   // acc = dA; aux = (g, u) interleaved fp32 (fp16 with aux_f16) -> out = (dg, du)
                        // interleaved fp16
  EPI_LORA_T = 6,       // out fp32 [m, 0:N] = beta * acc ; aux bf16 [m, 0:64] = (hi, lo) of alpha * acc:
                        // cols 0..N-1 bf16(alpha acc), cols 32..32+N-1 bf16(alpha acc - hi), else 0
};

struct EpiParams {
  void* out = nullptr;
  int64_t ldo = 0;
  void* aux = nullptr;
  int64_t ld_aux = 0;
  bf16* x = nullptr;  // scatter target [x_rows, ldx]
  int64_t ldx = 0;
  int64_t x_rows = 0;
  const int32_t* idx = nullptr;  // kept block list (row map); null = identity rows
  int blk = 1;
  int row_offset = 0;            // compact row of local row 0 (segment start)
  const int32_t* n_valid = nullptr;  // device: valid rows = (*n_valid) * valid_mult - row_offset
  int valid_mult = 1;
  int m_host = 0;                // host bound on rows (M of the launch)
  float alpha = 1.f;
  float beta = 1.f;              // LORA_T: scale of the fp32 copy
  int hd = 0;                    // QKV: H * D (section width)
  int col0 = 0;                  // QKV: column of this GEMM's first output in the q | k | v layout
  const float2* rope_tab = nullptr;  // QKV: (cos, sin) of position(m) x frequency j, [M rows][64]
  bool tma_out = false;          // set by the launcher: the output tensor map is valid
  // optional keep mask per block of mask_blk compact rows (indexed by (row_offset + m) /
  // mask_blk): 128-row tiles with no kept row are skipped by every role (no loads, no MMAs,
  // no stores), and the scatter-add epilogue leaves the rows of masked blocks untouched
  const uint8_t* blk_mask = nullptr;
  int mask_blk = 1;
  // STORE_F32: optional per-row factor of the accumulator (local row m), the inverse
  // power-of-two scale of an fp16 A operand whose rows were scaled into fp16's range
  const float* row_scale = nullptr;
  // SWIGLU_BWD: the saved (g, u) are fp16 (else fp32)
  bool aux_f16 = false;
  // STORE_F32 only: split the reduction into ksplit consecutive ranges of k-blocks, one per
  // CTA tile; range ks writes its partial product to rows [ks * M, ks * M + M) of out
  int ksplit = 1;
};

// Does the 128-row tile at local row m0 hold a row of a kept block (always, without a mask)?
__device__ __forceinline__ bool gemm_tile_live(const EpiParams& p, int m0, int valid) {
  if (!p.blk_mask) return true;
  const int r0 = p.row_offset + m0;
  const int r1 = p.row_offset + min(m0 + 128, valid);
  for (int b = r0 / p.mask_blk; b * p.mask_blk < r1; ++b)
    if (__ldg(p.blk_mask + b)) return true;
  return false;
}

__device__ __forceinline__ int epi_valid_rows(const EpiParams& p) {
  int v = p.m_host;
  if (p.n_valid) {
    int nv = (*p.n_valid) * p.valid_mult - p.row_offset;
    v = min(v, max(nv, 0));
  }
  return v;
}

// sequence row of compact row c (through the kept-block list)
__device__ __forceinline__ int64_t map_row(const EpiParams& p, int c) {
  if (!p.idx) return c;
  int b = c / p.blk;
  return (int64_t)__ldg(p.idx + b) * p.blk + (c - b * p.blk);
}

__device__ __forceinline__ void store_bf16x32(bf16* dst, const float* v) {
  uint4* d = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint4 w;
    uint32_t* ws = reinterpret_cast<uint32_t*>(&w);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      __nv_bfloat162 h = __floats2bfloat162_rn(v[q * 8 + 2 * i], v[q * 8 + 2 * i + 1]);
      ws[i] = *reinterpret_cast<uint32_t*>(&h);
    }
    d[q] = w;
  }
}

__device__ __forceinline__ void store_f16x32(__half* dst, const float* v) {
  uint4* d = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint4 w;
    uint32_t* ws = reinterpret_cast<uint32_t*>(&w);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      __half2 h = __floats2half2_rn(v[q * 8 + 2 * i], v[q * 8 + 2 * i + 1]);
      ws[i] = *reinterpret_cast<uint32_t*>(&h);
    }
    d[q] = w;
  }
}

// 32 floats -> 16 packed pairs (bf16, or fp16 with F16), round to nearest even
template <bool F16>
__device__ __forceinline__ void pack32(const float* v, uint32_t* w) {
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    if (F16) {
      __half2 h = __floats2half2_rn(v[2 * i], v[2 * i + 1]);
      w[i] = *reinterpret_cast<uint32_t*>(&h);
    } else {
      __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
      w[i] = *reinterpret_cast<uint32_t*>(&h);
    }
  }
}

// 16 packed words (32 two-byte values) as the 16-byte chunks ch0 .. ch0 + 3 of row `row` of
// a 32 x 64 staging tile (128-byte rows, 128-byte swizzle)
__device__ __forceinline__ void stage_row32(uint8_t* tile, int row, int ch0, const uint32_t* w) {
#pragma unroll
  for (int q = 0; q < 4; ++q)
    *reinterpret_cast<uint4*>(tile + row * 128 + (((ch0 + q) ^ (row & 7)) << 4)) =
        make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
}

__device__ __forceinline__ void load_bf16x32(const bf16* src, float* v) {
  const uint4* s = reinterpret_cast<const uint4*>(src);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint4 w = s[q];
    const uint32_t* ws = reinterpret_cast<const uint32_t*>(&w);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      __nv_bfloat162 h = *reinterpret_cast<const __nv_bfloat162*>(&ws[i]);
      float2 f = __bfloat1622float2(h);
      v[q * 8 + 2 * i] = f.x;
      v[q * 8 + 2 * i + 1] = f.y;
    }
  }
}

__device__ __forceinline__ float silu_f(float z) { return z / (1.f + __expf(-z)); }

template <int BN>
struct GemmSmem {
  // (the static_assert below keeps TOTAL within the 227 KB a CTA may use)
  static constexpr int STAGES = BN >= 256 ? 4 : (BN >= 128 ? 6 : 8);
  static constexpr int A_BYTES = GEMM_BM * GEMM_BK * 2;
  static constexpr int B_BYTES = BN * GEMM_BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  // fp32 output staging: per epilogue warp two 32-row x 32-column tiles (4 KB each) for
  // TMA stores
  static constexpr int STG_OFF = STAGES * STAGE_BYTES;
  static constexpr int STG_BYTES = 4 * 2 * 4096;
  static constexpr int BAR_OFF = STG_OFF + STG_BYTES;
  static constexpr int TOTAL = BAR_OFF + 256 + 1024;  // barriers + 1 KB alignment slack
  static_assert(TOTAL <= 232448, "shared memory per CTA");
};

template <int BN, int EPI>
__global__ void __launch_bounds__(GEMM_THREADS, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA1, const __grid_constant__ CUtensorMap tmB1,
                   const __grid_constant__ CUtensorMap tmA2, const __grid_constant__ CUtensorMap tmB2,
                   const __grid_constant__ CUtensorMap tmA3, const __grid_constant__ CUtensorMap tmB3,
                   const __grid_constant__ CUtensorMap tmOut, int nkb1, int nkb2, int nkb3, int N, uint32_t idesc,
                   EpiParams ep) {
  using L = GemmSmem<BN>;
  constexpr int STAGES = L::STAGES;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::BAR_OFF);
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;  // [2]
  uint64_t* acc_empty = acc_full + 2;   // [2]
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(acc_empty + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int valid = epi_valid_rows(ep);
  const int ntn = (N + BN - 1) / BN;
  const int ntm = (min(valid, ep.m_host) + GEMM_BM - 1) / GEMM_BM;  // tiles past the valid rows are skipped
  const int nbase = ntn * ntm;  // output tiles; each runs as ksplit work tiles
  const int ntiles = nbase * ep.ksplit;
  if ((int)blockIdx.x >= ntiles) return;  // uniform per CTA
  const int nkb = nkb1 + nkb2 + nkb3;
  // k-block range of work tile `tile` (the whole reduction without a split)
  auto kb_range = [&](int tile, int& lo, int& hi) {
    const int ks = tile / nbase;
    lo = (int)((int64_t)nkb * ks / ep.ksplit);
    hi = (int)((int64_t)nkb * (ks + 1) / ep.ksplit);
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 4);
    }
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, 2 * (BN < 32 ? 32 : BN));
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp == 0 && lane == 0) {
    // ---------------- TMA producer
    prefetch_tmap(&tmA1);
    prefetch_tmap(&tmB1);
    int g = 0;  // k-blocks issued by this CTA so far (ring position)
    bool ok = true;
    for (int tile = blockIdx.x; ok && tile < ntiles; tile += gridDim.x) {
    const int bt = tile % nbase;
    const int n0 = (bt % ntn) * BN, m0 = (bt / ntn) * GEMM_BM;
    if (!gemm_tile_live(ep, m0, valid)) continue;
    int kb_lo, kb_hi;
    kb_range(tile, kb_lo, kb_hi);
    for (int kb = kb_lo; kb < kb_hi; ++kb, ++g) {
      const int s = g % STAGES;
      if (g >= STAGES && !mbar_wait(&empty[s], ((g / STAGES) - 1) & 1, SITE_GEMM_PRODUCER)) {
        ok = false;
        break;
      }
      uint8_t* sa = smem + s * L::STAGE_BYTES;
      uint8_t* sb = sa + L::A_BYTES;
      mbar_arrive_expect_tx(&full[s], L::STAGE_BYTES);
      if (kb < nkb1) {
        tma_load_2d(sa, &tmA1, &full[s], kb * GEMM_BK, m0);
        tma_load_2d(sb, &tmB1, &full[s], kb * GEMM_BK, n0);
      } else if (kb < nkb1 + nkb2) {
        tma_load_2d(sa, &tmA2, &full[s], (kb - nkb1) * GEMM_BK, m0);
        tma_load_2d(sb, &tmB2, &full[s], (kb - nkb1) * GEMM_BK, n0);
      } else {
        tma_load_2d(sa, &tmA3, &full[s], (kb - nkb1 - nkb2) * GEMM_BK, m0);
        tma_load_2d(sb, &tmB3, &full[s], (kb - nkb1 - nkb2) * GEMM_BK, n0);
      }
    }
    }
  } else if (warp == 1 && lane == 0) {
    // ---------------- MMA issuer
    // idesc: kind::f16 instruction descriptor (bf16 or fp16 operands, fp32 accumulate)
    bool ok = true;
    int g = 0, it = 0;
    for (int tile = blockIdx.x; ok && tile < ntiles; tile += gridDim.x) {
      if (!gemm_tile_live(ep, ((tile % nbase) / ntn) * GEMM_BM, valid)) continue;
      int kb_lo, kb_hi;
      kb_range(tile, kb_lo, kb_hi);
      const int buf = it & 1;
      // the epilogue must have read this accumulator's previous tile (two tiles ago)
      if (it >= 2 && !mbar_wait(&acc_empty[buf], ((it >> 1) - 1) & 1, SITE_GEMM_MMA)) break;
      tc_fence_after();
      const uint32_t acc = tmem + buf * (BN < 32 ? 32 : BN);
      for (int kb = kb_lo; kb < kb_hi; ++kb, ++g) {
        const int s = g % STAGES;
        if (!mbar_wait(&full[s], (g / STAGES) & 1, SITE_GEMM_MMA)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t sa = smem_u32(smem + s * L::STAGE_BYTES);
        const uint32_t sb = sa + L::A_BYTES;
#pragma unroll
        for (int k = 0; k < GEMM_BK / 16; ++k) {
          umma_bf16(acc, umma_desc_k_sw128(sa + k * 32), umma_desc_k_sw128(sb + k * 32), idesc,
                    (kb > kb_lo || k > 0) ? 1u : 0u);
        }
        umma_commit(&empty[s]);
      }
      if (ok) umma_commit(&acc_full[buf]);
      ++it;  // live tiles only: the accumulator parity follows the tiles actually computed
    }
  } else if (warp >= 2) {
    // ---------------- epilogue
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    uint8_t* stg = smem + L::STG_OFF + quarter * 2 * 4096;  // this warp's two staging tiles
    int nst = 0;  // TMA stores issued by this warp (lane 0)
    // Output tiles of 32 rows leave through TMA stores when all 32 rows of the warp are
    // valid.  tile_wait(k): before staging into the next k tiles (k = 1: tile nst & 1;
    // k = 2: both), wait until the stores that last read them are done.
    auto tile_wait = [&](int k) {
      if (lane == 0 && nst >= 3 - k) {
        if (k == 1)
          bulk_wait_group_read<1>();
        else
          bulk_wait_group_read<0>();
      }
      __syncwarp();
    };
    auto tile_store = [&](uint8_t* tile, int x, int y) {  // after the warp staged `tile`
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        tma_store_2d(&tmOut, tile, x, y);
        bulk_commit_group();
      }
      ++nst;
    };
    int it = 0;
    for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
    const int bt = tile % nbase;
    const int n0 = (bt % ntn) * BN, m0 = (bt / ntn) * GEMM_BM;
    if (!gemm_tile_live(ep, m0, valid)) continue;
    // split reduction: range ks stores its partial in the ks-th block of M output rows
    const int orow0 = EPI == EPI_STORE_F32 ? (tile / nbase) * ep.m_host : 0;
    const int buf = it & 1;
    const int m = m0 + r;
    // warp vote: the tcgen05.ld calls below are collective, so all lanes take one path
    const bool ok = __all_sync(0xffffffffu, mbar_wait(&acc_full[buf], (it >> 1) & 1, SITE_GEMM_EPILOGUE));
    tc_fence_after();
    if (!ok) break;
    {
      const uint32_t tbase = tmem + ((uint32_t)(quarter * 32) << 16) + buf * (BN < 32 ? 32 : BN);
      const bool row_ok = m < valid;
      const float rfac = EPI == EPI_STORE_F32 && ep.row_scale && row_ok ? __ldg(ep.row_scale + m) : 1.f;
      float v[32];
      if (EPI == EPI_STORE_BF16 || EPI == EPI_STORE_F32 || EPI == EPI_SCATTER_ADD) {
        const float oscale = EPI == EPI_STORE_F32 ? ep.alpha * rfac : ep.alpha;
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
          tmem_ld32(tbase + c * 32, v);
          const int n = n0 + c * 32;
          if (EPI == EPI_STORE_F32 && ep.tma_out && n < N && m0 + quarter * 32 + 32 <= valid) {
            // the warp's 32 rows are all valid: stage them (128-byte swizzle) and write the
            // 32 x 32 tile with one TMA store (full-line writes instead of 32 rows of 16-byte
            // pieces per instruction); a staging tile is reused once its store has read it
            uint8_t* sb = stg + (nst & 1) * 4096;
            if (lane == 0 && nst >= 2) bulk_wait_group_read<1>();
            __syncwarp();
#pragma unroll
            for (int q = 0; q < 8; ++q)
              *reinterpret_cast<float4*>(sb + lane * 128 + ((q ^ (lane & 7)) << 4)) =
                  make_float4(v[4 * q] * oscale, v[4 * q + 1] * oscale, v[4 * q + 2] * oscale,
                              v[4 * q + 3] * oscale);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              tma_store_2d(&tmOut, sb, n, orow0 + m0 + quarter * 32);
              bulk_commit_group();
            }
            ++nst;
            continue;
          }
          if (EPI == EPI_STORE_BF16 && ep.tma_out && n < N && m0 + quarter * 32 + 32 <= valid) {
            // two 32-column chunks per 64-column bf16 tile
            uint8_t* tb = stg + (nst & 1) * 4096;
            if ((c & 1) == 0) tile_wait(1);
            uint32_t w[16];
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] *= ep.alpha;
            pack32<false>(v, w);
            stage_row32(tb, lane, (c & 1) * 4, w);
            if ((c & 1) || c + 1 == BN / 32 || n + 32 >= N) tile_store(tb, n0 + (c >> 1) * 64, m0 + quarter * 32);
            continue;
          }
          if (!row_ok || n >= N) continue;
          if (EPI == EPI_STORE_BF16) {
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] *= ep.alpha;
            store_bf16x32(reinterpret_cast<bf16*>(ep.out) + (int64_t)m * ep.ldo + n, v);
          } else if (EPI == EPI_STORE_F32) {
            float4* d = reinterpret_cast<float4*>(reinterpret_cast<float*>(ep.out) + (int64_t)(orow0 + m) * ep.ldo + n);
#pragma unroll
            for (int q = 0; q < 8; ++q)
              d[q] = make_float4(v[4 * q] * oscale, v[4 * q + 1] * oscale, v[4 * q + 2] * oscale,
                                 v[4 * q + 3] * oscale);
          } else {  // scatter-add into the residual rows
            if (ep.blk_mask && !__ldg(ep.blk_mask + (m + ep.row_offset) / ep.mask_blk)) continue;
            const int64_t row = map_row(ep, m + ep.row_offset);
            if (row < 0 || row >= ep.x_rows) {
              record_device_error(JENGA_EINTERNAL, SITE_INDEX_RANGE, (unsigned)row);
              continue;
            }
            bf16* xp = ep.x + row * ep.ldx + n;
            float xv[32];
            load_bf16x32(xp, xv);
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = xv[i] + v[i];
            store_bf16x32(xp, v);
            if (ep.aux) store_bf16x32(reinterpret_cast<bf16*>(ep.aux) + (int64_t)m * ep.ld_aux + n, v);
          }
        }
      } else if (EPI == EPI_SWIGLU) {
#pragma unroll 1
        for (int g = 0; g < BN / 128; ++g) {
#pragma unroll 1
          for (int hh = 0; hh < 2; ++hh) {
            float u[32];
            tmem_ld32(tbase + g * 128 + hh * 32, v);
            tmem_ld32(tbase + g * 128 + 64 + hh * 32, u);
            const int n = n0 + g * 128;
            if (n >= N) continue;
            const bool tma = ep.tma_out && m0 + quarter * 32 + 32 <= valid;
            if (!tma && !row_ok) continue;
            if (ep.aux) {  // the pre-activations, saved for the backward
              __half* ga = reinterpret_cast<__half*>(ep.aux) + (int64_t)m * ep.ld_aux + n + hh * 32;
              store_f16x32(ga, v);
              store_f16x32(ga + 64, u);
            }
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = silu_f(v[i]) * u[i];
            if (tma) {  // the group's 64 outputs form one bf16 tile
              uint8_t* tb = stg + (nst & 1) * 4096;
              if (hh == 0) tile_wait(1);
              uint32_t w[16];
              pack32<false>(v, w);
              stage_row32(tb, lane, hh * 4, w);
              if (hh == 1) tile_store(tb, n >> 1, m0 + quarter * 32);
              continue;
            }
            store_bf16x32(reinterpret_cast<bf16*>(ep.out) + (int64_t)m * ep.ldo + (n >> 1) + hh * 32, v);
          }
        }
      } else if (EPI == EPI_SWIGLU_BWD) {
        // acc column j (of ffn) -> group j/64, gate at 128*group + j%64, up at +64
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
          tmem_ld32(tbase + c * 32, v);
          const int j = n0 + c * 32;
          if (j >= N) continue;
          const bool tma = ep.tma_out && m0 + quarter * 32 + 32 <= valid;
          if (!tma && !row_ok) continue;
          const int64_t col = (int64_t)(j >> 6) * 128 + (j & 63);
          float gv[32], uv[32], dg[32];
          if (ep.aux_f16) {
            const __half* gu = reinterpret_cast<const __half*>(ep.aux) + (int64_t)m * ep.ld_aux + col;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const uint4 a = reinterpret_cast<const uint4*>(gu)[q];
              const uint4 b = reinterpret_cast<const uint4*>(gu + 64)[q];
              const __half2* ah = reinterpret_cast<const __half2*>(&a);
              const __half2* bh = reinterpret_cast<const __half2*>(&b);
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const float2 fa = __half22float2(ah[e]), fb = __half22float2(bh[e]);
                gv[8 * q + 2 * e] = fa.x;
                gv[8 * q + 2 * e + 1] = fa.y;
                uv[8 * q + 2 * e] = fb.x;
                uv[8 * q + 2 * e + 1] = fb.y;
              }
            }
          } else {
            const float* gu = reinterpret_cast<const float*>(ep.aux) + (int64_t)m * ep.ld_aux + col;
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              const float4 a = reinterpret_cast<const float4*>(gu)[q];
              const float4 b = reinterpret_cast<const float4*>(gu + 64)[q];
              gv[4 * q] = a.x; gv[4 * q + 1] = a.y; gv[4 * q + 2] = a.z; gv[4 * q + 3] = a.w;
              uv[4 * q] = b.x; uv[4 * q + 1] = b.y; uv[4 * q + 2] = b.z; uv[4 * q + 3] = b.w;
            }
          }
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float sg = 1.f / (1.f + __expf(-gv[i]));
            const float da = v[i];
            dg[i] = da * uv[i] * sg * (1.f + gv[i] * (1.f - sg));
            v[i] = da * gv[i] * sg;  // du = dA * silu(g)
          }
          if (tma) {  // a 64-column group of dA gives one fp16 tile of dg and one of du
            if ((j & 63) == 0) tile_wait(2);
            uint32_t w[16];
            pack32<true>(dg, w);
            stage_row32(stg, lane, (j & 32) >> 3, w);
            pack32<true>(v, w);
            stage_row32(stg + 4096, lane, (j & 32) >> 3, w);
            if ((j & 63) == 32 || j + 32 >= N) {
              const int x = (j >> 6) * 128;
              tile_store(stg, x, m0 + quarter * 32);
              tile_store(stg + 4096, x + 64, m0 + quarter * 32);
            }
            continue;
          }
          __half* o = reinterpret_cast<__half*>(ep.out) + (int64_t)m * ep.ldo + col;
          store_f16x32(o, dg);
          store_f16x32(o + 64, v);
        }
      } else if (EPI == EPI_LORA_T) {
        // N <= 32 (t_q, t_v): fp32 copy + the scaled value as a bf16 hi + lo pair (columns
        // 0..31 and 32..63 of the K-padded operand of the next product)
        tmem_ld32(tbase, v);
        if (row_ok) {
          float* o = reinterpret_cast<float*>(ep.out) + (int64_t)m * ep.ldo;
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (i < N) o[i] = v[i] * ep.beta;
          float w[32], lo[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            w[i] = i < N ? v[i] * ep.alpha : 0.f;
            lo[i] = w[i] - __bfloat162float(__float2bfloat16_rn(w[i]));
          }
          bf16* a = reinterpret_cast<bf16*>(ep.aux) + (int64_t)m * ep.ld_aux;
          store_bf16x32(a, w);
          store_bf16x32(a + 32, lo);
        }
      } else if (EPI == EPI_QKV_ROPE) {
        // tile = BN/128 heads; section = (n / hd): 0 q, 1 k, 2 v; RoPE on q and k with this
        // row's (cos, sin) from the table (rope_table_kernel: same angles, computed once)
        const float4* tab = reinterpret_cast<const float4*>(ep.rope_tab + (int64_t)(row_ok ? m : 0) * 64);
#pragma unroll 1
        for (int g = 0; g < BN / 128; ++g) {
          const int nh = n0 + g * 128;
          const bool rope = ep.col0 + nh < 2 * ep.hd;
#pragma unroll 1
          for (int hh = 0; hh < 2; ++hh) {
            float u[32];
            tmem_ld32(tbase + g * 128 + hh * 32, v);
            tmem_ld32(tbase + g * 128 + 64 + hh * 32, u);
            if (nh >= N) continue;
            const bool tma = ep.tma_out && m0 + quarter * 32 + 32 <= valid;
            if (!tma && !row_ok) continue;
            if (rope) {
#pragma unroll
              for (int i2 = 0; i2 < 16; ++i2) {
                const float4 t = __ldg(tab + hh * 16 + i2);  // (cos, sin) of frequencies 2 i2, 2 i2 + 1
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                  const int i = 2 * i2 + e;
                  const float cs = e ? t.z : t.x, sn = e ? t.w : t.y;
                  const float a = v[i], b = u[i];
                  v[i] = a * cs - b * sn;
                  u[i] = b * cs + a * sn;
                }
              }
            }
            if (tma) {  // the head's 128 outputs form two bf16 tiles (v: columns 0-63, u: 64-127)
              if (hh == 0) tile_wait(2);
              uint32_t w[16];
              pack32<false>(v, w);
              stage_row32(stg, lane, hh * 4, w);
              pack32<false>(u, w);
              stage_row32(stg + 4096, lane, hh * 4, w);
              if (hh == 1) {
                tile_store(stg, nh, m0 + quarter * 32);
                tile_store(stg + 4096, nh + 64, m0 + quarter * 32);
              }
              continue;
            }
            bf16* o = reinterpret_cast<bf16*>(ep.out) + (int64_t)m * ep.ldo + nh;
            store_bf16x32(o + hh * 32, v);
            store_bf16x32(o + 64 + hh * 32, u);
          }
        }
      }
    }
    // every TMEM load of this accumulator is done: the MMAs of tile it + 2 may overwrite it
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&acc_empty[buf]);
    ++it;
    }
    if (lane == 0 && nst > 0) bulk_wait_group_read<0>();  // staging outlives the stores' reads
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 2 * (BN < 32 ? 32 : BN));
  }
}

// ------------------------------------------------------------------ host launcher
struct GemmOperand {
  const void* ptr;
  int64_t rows;  // tensor-map extent (rows may extend past the valid rows)
  int64_t ld;    // row pitch in elements
};

template <int BN, int EPI>
jenga_status launch_gemm(const GemmOperand& A1, const GemmOperand& B1, int K1, const GemmOperand* A2,
                         const GemmOperand* B2, int K2, int M, int N, const EpiParams& ep, cudaStream_t st,
                         const char* name = "gemm", const GemmOperand* A3 = nullptr,
                         const GemmOperand* B3 = nullptr, int K3 = 0, bool f16_inputs = false) {
  using L = GemmSmem<BN>;
  if (M <= 0 || N <= 0) return JENGA_OK;
  if (K1 % GEMM_BK || K2 % GEMM_BK || K1 <= 0) return fail(JENGA_EINVAL, "gemm: K must be a multiple of 64");
  CUtensorMap ta1, tb1, ta2, tb2;
  jenga_status s;
  if ((s = make_tmap_bf16(&ta1, A1.ptr, A1.rows, K1, A1.ld, GEMM_BM)) != JENGA_OK) return s;
  if ((s = make_tmap_bf16(&tb1, B1.ptr, B1.rows, K1, B1.ld, BN)) != JENGA_OK) return s;
  if (K2 > 0) {
    if ((s = make_tmap_bf16(&ta2, A2->ptr, A2->rows, K2, A2->ld, GEMM_BM)) != JENGA_OK) return s;
    if ((s = make_tmap_bf16(&tb2, B2->ptr, B2->rows, K2, B2->ld, BN)) != JENGA_OK) return s;
  } else {
    ta2 = ta1;
    tb2 = tb1;
  }
  CUtensorMap ta3 = ta1, tb3 = tb1;
  if (K3 % GEMM_BK) return fail(JENGA_EINVAL, "gemm: K must be a multiple of 64");
  if (K3 > 0) {
    if ((s = make_tmap_bf16(&ta3, A3->ptr, A3->rows, K3, A3->ld, GEMM_BM)) != JENGA_OK) return s;
    if ((s = make_tmap_bf16(&tb3, B3->ptr, B3->rows, K3, B3->ld, BN)) != JENGA_OK) return s;
  }
  // output tensor map of the TMA-store epilogues (fp32 32 x 32 boxes, bf16 / fp16 32 x 64);
  // an output the map cannot describe (alignment) keeps the per-thread stores
  CUtensorMap tout = ta1;
  EpiParams p = ep;
  p.m_host = M;
  if (ep.ksplit < 1 || (ep.ksplit > 1 && EPI != EPI_STORE_F32))
    return fail(JENGA_EINVAL, "gemm: a split reduction needs the fp32 store epilogue");
  if (ep.ksplit > (K1 + K2 + K3) / GEMM_BK) p.ksplit = (K1 + K2 + K3) / GEMM_BK;  // >= 1 k-block per range
  {
    jenga_status ts = JENGA_EUNSUPPORTED;
    const bool al = ((reinterpret_cast<uintptr_t>(ep.out) & 15) == 0);
    if (al && EPI == EPI_STORE_F32 && ep.ldo % 4 == 0)
      ts = make_tmap_f32(&tout, ep.out, (uint64_t)M * p.ksplit, (uint64_t)N, (uint64_t)ep.ldo, 32);
    else if (al && (EPI == EPI_STORE_BF16 || EPI == EPI_QKV_ROPE) && ep.ldo % 8 == 0)
      ts = make_tmap_bf16(&tout, ep.out, (uint64_t)M, (uint64_t)N, (uint64_t)ep.ldo, 32);
    else if (al && EPI == EPI_SWIGLU && ep.ldo % 8 == 0)
      ts = make_tmap_bf16(&tout, ep.out, (uint64_t)M, (uint64_t)N / 2, (uint64_t)ep.ldo, 32);
    else if (al && EPI == EPI_SWIGLU_BWD && ep.ldo % 8 == 0)
      ts = make_tmap_f16(&tout, ep.out, (uint64_t)M, 2 * (uint64_t)N, (uint64_t)ep.ldo, 32);
    if (ts == JENGA_OK) p.tma_out = true;
    else tout = ta1;
  }
  JENGA_CUDA_TRY(
      cudaFuncSetAttribute(gemm_tc_kernel<BN, EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize, L::TOTAL));
  // persistent: one CTA per SM (or per tile when there are fewer tiles)
  const int ntiles = ((N + BN - 1) / BN) * ((M + GEMM_BM - 1) / GEMM_BM) * p.ksplit;
  dim3 grid(ntiles < sm_count() ? ntiles : sm_count());
  // operand format fields (bits 7-9: A, 10-12: B) are 1 for bf16 and 0 for fp16
  const uint32_t idesc = f16_inputs ? (umma_idesc_bf16(GEMM_BM, BN) & ~((7u << 7) | (7u << 10)))
                                    : umma_idesc_bf16(GEMM_BM, BN);
  const int ps = prof_begin(name, st);
  gemm_tc_kernel<BN, EPI><<<grid, GEMM_THREADS, L::TOTAL, st>>>(ta1, tb1, ta2, tb2, ta3, tb3, tout, K1 / GEMM_BK,
                                                                 K2 / GEMM_BK, K3 / GEMM_BK, N, idesc, p);
  prof_end(ps, st);
  JENGA_LAUNCH_CHECK();
  return JENGA_OK;
}

}  // namespace jenga
