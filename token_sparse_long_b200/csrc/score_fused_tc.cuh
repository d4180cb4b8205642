// Single-pass tcgen05 block scoring (bf16, head_dim 128): the softmax column mass of every
// key chunk from ONE pass over the causal logits.
//
// For query row i (one head) with log-sum-exp L_i = log2 sum_{j<=i} 2^(x_ij) (x_ij the
// logit in log2 units, log2(e) q_i . k_j / sqrt(D)), the softmax mass that key chunk c
// receives from row i is
//
//   sum_{j in c} 2^(x_ij - L_i) = 2^(lse_ic - L_i),   lse_ic = log2 sum_{j in c, j<=i} 2^(x_ij).
//
// While the row's exponentials are summed for L_i, each chunk's partial sum is kept as lse_ic
// in a per-CTA scratch area; when the query tile's last key tile is done, L_i is final and the
// chunk masses of the tile are sum_i 2^(lse_ic - L_i): one exponential per (row, chunk)
// instead of a second pass that recomputes every logit and exponential (the notes' scoring
// integrated with the attention computation, memory linear in S: Jenga notes §4.3).
//
// Persistent grid (at most one CTA per SM, a fixed scratch slot per CTA); work items are
// (128-query tile, head, sequence), head-major with the longest query tiles of each head first,
// taken from a global counter as CTAs become free.  Per CTA,
// 608 threads:
//   warp 0       TMA: the item's first key-tile pairs, then (once the previous item's MMAs are
//                done) its query tile, then the remaining key pairs through a 3-stage ring
//   warps 1, 2   TMEM allocation (warp 1); one lane of each issues tcgen05.mma (M 128, N 256,
//                K 16) x 8 per key pair into one of two 256-column TMEM accumulators,
//                warp 1 for even and warp 2 for odd pairs (global pair count)
//   warps 3..18  four quads, one TMEM lane (= one query row) per thread, quad c taking
//                accumulator columns 64c .. 64c + 63: tcgen05.ld, release, then exponentials
//                (a few column pairs on the FMA pipe, exp2_fma) and the chunk partial sums;
//                at the end of an item the four quads' (m, l) of each row are merged, and the
//                16 warps reduce the scratch to per-(head, query tile, chunk) masses
// Each row sums 2^(x - m) against a reference m and redoes a 64-column chunk with its exact
// max only when the sum leaves [0, 2^60) (a new maximum far above m, or the row's first
// chunk).  Causal diagonal tiles and partial last tiles are masked.  All waits are bounded;
// the epilogue warps leave the item loop together (predicate-reduced named barrier).
#pragma once

#include "common.cuh"

namespace jenga {

constexpr int SF_ROWS = 128;
constexpr int SF_STAGES = 3;                        // ring stages of 256 streamed key rows
constexpr int SF_BOX_BYTES = 128 * 64 * 2;          // one 128 x 64 bf16 box
constexpr int SF_TILE_BYTES = 2 * SF_BOX_BYTES;     // 128 x 128 query tile
constexpr int SF_PAIR_BYTES = 4 * SF_BOX_BYTES;     // 256 x 128 key pair: [k half][256 rows x 64]
constexpr int SF_EPI_WARPS = 16;
constexpr int SF_EPI_WARP0 = 3;
constexpr int SF_THREADS = 32 * SF_EPI_WARP0 + 32 * SF_EPI_WARPS;
constexpr int SF_RING_OFF = SF_TILE_BYTES;
constexpr int SF_BAR_OFF = SF_RING_OFF + SF_STAGES * SF_PAIR_BYTES;
constexpr int SF_L_OFF = SF_BAR_OFF + 256;          // final row log-sum-exp of the item [128]
constexpr int SF_SMEM = SF_L_OFF + 512 + 1024;      // + alignment slack
constexpr int SF_GRID_CAP = 160;                    // scratch slots (>= SMs of the part)
#ifndef SF_EMU_PAIRS
#define SF_EMU_PAIRS 0x0202u  // column pairs p (of 16) with bit p set use exp2_fma: 2 of 16
#endif

// scratch floats per CTA: chunk log-sum-exps [chunks][128] + (m, l) of 4 quads [8][128]
__host__ __device__ inline size_t sf_scratch_floats_per_cta(int nt, int ch) {
  return (size_t)128 * ((size_t)nt * (128 / ch) + 8);
}

__device__ __forceinline__ uint64_t sf_exp2_pair(uint64_t x2, int pair) {
  return ((SF_EMU_PAIRS >> (pair & 15)) & 1u) ? exp2_fma_x2<64>(x2) : exp2_mufu_x2(x2);
}

__device__ __forceinline__ float sf_lg2(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// One thread's 64 logits v (accumulator columns of one key tile, starting at tile column cb)
// for row r: update the row's (m, l) and return the chunk log-sum-exps (log2 units) of the
// NH = 64 / CH chunks in lp[].  limit: columns c with cb + c < limit are visible (the causal
// diagonal: limit = r + 1; a partial last key tile: the keys left in the sequence; else 128).
template <int CH>
__device__ __forceinline__ void sf_update(const uint32_t* v, int cb, int limit, float sl2, float& m, float& l,
                                          float* lp) {
  constexpr int NH = 64 / CH;
  const bool masked = cb + 64 > limit;
  if (!masked && m != -INFINITY) {
    const uint64_t sl2x2 = f2pack(sl2, sl2), nm2 = f2pack(-m, -m);
    float part[NH];
#pragma unroll
    for (int hh = 0; hh < NH; ++hh) {
      uint64_t acc2[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
      for (int pr = 0; pr < CH / 2; ++pr) {
        const int c = hh * CH + 2 * pr;
        const uint64_t x2 = ffma2(f2pack(__uint_as_float(v[c]), __uint_as_float(v[c + 1])), sl2x2, nm2);
        acc2[pr & 3] = fadd2(acc2[pr & 3], sf_exp2_pair(x2, c >> 1));
      }
      float s[8];
#pragma unroll
      for (int i = 0; i < 4; ++i) f2unpack(acc2[i], s[2 * i], s[2 * i + 1]);
      part[hh] = ((s[0] + s[1]) + (s[2] + s[3])) + ((s[4] + s[5]) + (s[6] + s[7]));
    }
    float tot = part[0];
#pragma unroll
    for (int hh = 1; hh < NH; ++hh) tot += part[hh];
    if (tot < 0x1p60f) {  // false for inf / NaN too: then the exact path below
      l += tot;
#pragma unroll
      for (int hh = 0; hh < NH; ++hh) lp[hh] = m + sf_lg2(part[hh]);
      return;
    }
  }
  float mx = -INFINITY;
#pragma unroll
  for (int c = 0; c < 64; ++c)
    if (cb + c < limit) mx = fmaxf(mx, __uint_as_float(v[c]));
  const float mn = fmaxf(m, mx * sl2);
  if (mn == -INFINITY) {  // nothing visible yet in this row
#pragma unroll
    for (int hh = 0; hh < NH; ++hh) lp[hh] = -INFINITY;
    return;
  }
  float part[NH];
#pragma unroll
  for (int hh = 0; hh < NH; ++hh) {
    float sm[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int e = 0; e < CH; ++e) {
      const int c = hh * CH + e;
      const float p = fast_exp2(fmaf(__uint_as_float(v[c]), sl2, -mn));
      sm[e & 3] += (cb + c < limit) ? p : 0.f;
    }
    part[hh] = (sm[0] + sm[1]) + (sm[2] + sm[3]);
  }
  float tot = part[0];
#pragma unroll
  for (int hh = 1; hh < NH; ++hh) tot += part[hh];
  l = l * fast_exp2(m - mn) + tot;
  m = mn;
#pragma unroll
  for (int hh = 0; hh < NH; ++hh) lp[hh] = mn + sf_lg2(part[hh]);
}

template <int CH>
__global__ void __launch_bounds__(SF_THREADS, 1)
    score_fused_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK, int S,
                          int H, int B, int causal, float sl2, float* __restrict__ neg_lse,
                          float* __restrict__ part, float* __restrict__ scratch,
                          unsigned int* __restrict__ work_counter) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* fix = smem;
  uint8_t* ring = smem + SF_RING_OFF;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + SF_BAR_OFF);
  uint64_t* full = bars;                 // [STAGES]
  uint64_t* empty = full + SF_STAGES;    // [STAGES]
  uint64_t* s_full = empty + SF_STAGES;  // [2]
  uint64_t* s_empty = s_full + 2;        // [2]
  uint64_t* fix_full = s_empty + 2;
  uint64_t* fix_empty = fix_full + 1;
  uint64_t* item_full = fix_empty + 1;   // [4] work-item queue: slot written
  uint64_t* item_empty = item_full + 4;  // [4] ... and read by every consumer
  int* item_q = reinterpret_cast<int*>(item_empty + 4);  // [4]
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(item_q + 4);
  float* Lsm = reinterpret_cast<float*>(smem + SF_L_OFF);

  constexpr int CPT = SF_ROWS / CH;  // chunks per key tile
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nt = (S + SF_ROWS - 1) / SF_ROWS;
  const int nch_row = nt * CPT;  // chunk columns of part per (head, query tile)
  const int HB = H * B;
  const int n_items = nt * HB;
  float* my_lp = scratch + (size_t)blockIdx.x * sf_scratch_floats_per_cta(nt, CH);
  float* my_ml = my_lp + (size_t)nt * CPT * 128;  // [8][128]: m then l of quads 0..3

  if (threadIdx.x == 0) {
    for (int s = 0; s < SF_STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&s_full[s], 1);
      mbar_init(&s_empty[s], SF_EPI_WARPS);
    }
    mbar_init(fix_full, 1);
    mbar_init(fix_empty, 2);
    for (int s = 0; s < 4; ++s) {
      mbar_init(&item_full[s], 1);
      mbar_init(&item_empty[s], 2 + SF_EPI_WARPS);  // the two issuing threads and the epilogue warps
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

  // Work items are taken from a global counter (dynamic balance: a CTA that finishes early
  // takes the next item); the producer thread fetches item r and publishes it in queue slot
  // r % 4 for the issuing and epilogue warps.  Item numbers >= n_items end every role's loop.
  auto take_item = [&](int r, int& u) -> bool {  // the consumers' read of slot r % 4
    if (!mbar_wait(&item_full[r & 3], (uint32_t)((r >> 2) & 1), SITE_SCORE_TC)) return false;
    u = item_q[r & 3];
    return true;
  };
  // items in (sequence, head)-major order, query tiles longest first within each head: the
  // ~148 items in flight at a time belong to one or two heads, so their key tiles stay in L2
  // (an order that interleaved heads had every head's keys in flight and read them from DRAM
  // again for each query tile)
  auto decode = [&](int u, int& t, int& h, int& b) {
    const int hb = u / nt;
    t = nt - 1 - u % nt;
    h = hb % H;
    b = hb / H;
  };

  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmK);
    bool ok = true;
    long P = 0;  // key pairs streamed so far
    for (int r = 0; ok; ++r) {
      if (r >= 4 && !mbar_wait(&item_empty[r & 3], (uint32_t)(((r >> 2) - 1) & 1), SITE_SCORE_TC)) break;
      const int u = (int)atomicAdd(work_counter, 1u);
      item_q[r & 3] = u;
      mbar_arrive(&item_full[r & 3]);
      if (u >= n_items) break;
      int t, h, b;
      decode(u, t, h, b);
      const int j_end = causal ? t + 1 : nt;
      const int np = (j_end + 1) >> 1;
      const int col0 = h * 128, rowbase = b * S;
      auto load_pair = [&](int p) -> bool {
        const long gp = P + p;
        const int s = (int)(gp % SF_STAGES);
        if (gp >= SF_STAGES && !mbar_wait(&empty[s], (uint32_t)(((gp / SF_STAGES) - 1) & 1), SITE_SCORE_TC))
          return false;
        uint8_t* dst = ring + s * SF_PAIR_BYTES;
        const int row = rowbase + 2 * p * SF_ROWS;
        mbar_arrive_expect_tx(&full[s], SF_PAIR_BYTES);
#pragma unroll
        for (int kc = 0; kc < 2; ++kc)
#pragma unroll
          for (int hh = 0; hh < 2; ++hh)
            tma_load_2d(dst + kc * 2 * SF_BOX_BYTES + hh * SF_BOX_BYTES, &tmK, &full[s], col0 + 64 * kc,
                        row + SF_ROWS * hh);
        return true;
      };
      // the first key pairs do not depend on the query tile: stream them while the previous
      // item's MMAs still read the query buffer
      const int early = np < 2 ? np : 2;
      for (int p = 0; ok && p < early; ++p) ok = load_pair(p);
      if (!ok) break;
      if (r > 0 && !mbar_wait(fix_empty, (uint32_t)((r - 1) & 1), SITE_SCORE_TC)) break;
      mbar_arrive_expect_tx(fix_full, SF_TILE_BYTES);
      tma_load_2d(fix, &tmQ, fix_full, col0, rowbase + t * SF_ROWS);
      tma_load_2d(fix + SF_BOX_BYTES, &tmQ, fix_full, col0 + 64, rowbase + t * SF_ROWS);
      for (int p = early; ok && p < np; ++p) ok = load_pair(p);
      P += np;
    }
  } else if ((warp == 1 || warp == 2) && lane == 0) {
    constexpr uint32_t idesc = umma_idesc_bf16(128, 256);
    const uint32_t fa = smem_u32(fix);
    bool ok = true;
    long P = 0;
    for (int r = 0; ok; ++r) {
      int u;
      if (!take_item(r, u)) break;
      mbar_arrive(&item_empty[r & 3]);
      if (u >= n_items) break;
      int t, h, b;
      decode(u, t, h, b);
      const int j_end = causal ? t + 1 : nt;
      const int np = (j_end + 1) >> 1;
      if (!mbar_wait(fix_full, (uint32_t)(r & 1), SITE_SCORE_TC)) break;
      for (int p = 0; p < np; ++p) {
        const long gp = P + p;
        if ((int)(gp & 1) != warp - 1) continue;
        const int s = (int)(gp % SF_STAGES), buf = (int)(gp & 1);
        if (!mbar_wait(&full[s], (uint32_t)((gp / SF_STAGES) & 1), SITE_SCORE_TC)) {
          ok = false;
          break;
        }
        if (gp >= 2 && !mbar_wait(&s_empty[buf], (uint32_t)(((gp >> 1) - 1) & 1), SITE_SCORE_TC)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t sb = smem_u32(ring + s * SF_PAIR_BYTES);
#pragma unroll
        for (int kc = 0; kc < 2; ++kc)
#pragma unroll
          for (int k = 0; k < 4; ++k)
            umma_bf16(tmem + buf * 256, umma_desc_k_sw128(fa + kc * SF_BOX_BYTES + k * 32),
                      umma_desc_k_sw128(sb + kc * 2 * SF_BOX_BYTES + k * 32), idesc, (kc | k) ? 1u : 0u);
        umma_commit(&empty[s]);
        umma_commit(&s_full[buf]);
      }
      // the query tile may be replaced once this warp's MMAs of the item are done
      umma_commit(fix_empty);
      P += np;
    }
  } else if (warp >= SF_EPI_WARP0) {
    const int quarter = warp & 3;
    const int quad = (warp - SF_EPI_WARP0) >> 2;
    const int ew = warp - SF_EPI_WARP0;  // 0 .. 15
    const int r = quarter * 32 + lane;
    const int hp = quad >> 1, wc = (quad & 1) * 64;
    const uint32_t tl = tmem + ((uint32_t)(quarter * 32) << 16) + quad * 64;
    bool ok = true;
    long P = 0;
    for (int it = 0;; ++it) {
      int u = 0;
      const bool got = __all_sync(0xffffffffu, take_item(it, u));
      __syncwarp();
      if (got && lane == 0) mbar_arrive(&item_empty[it & 3]);
      // all epilogue warps leave together (they meet at named barriers inside the item)
      if (!bar_and(got && ok, 1, 32 * SF_EPI_WARPS)) break;
      if (u >= n_items) break;
      int t, h, b;
      decode(u, t, h, b);
      const int j_end = causal ? t + 1 : nt;
      const int np = (j_end + 1) >> 1;
      float m = -INFINITY, l = 0.f;
      for (int p = 0; ok && p < np; ++p) {
        const long gp = P + p;
        const int buf = (int)(gp & 1), j = 2 * p + hp;
        const bool live = j < j_end;  // warp-uniform
        if (!__all_sync(0xffffffffu, mbar_wait(&s_full[buf], (uint32_t)((gp >> 1) & 1), SITE_SCORE_TC))) {
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
        // visible key columns of this tile for row r
        int limit = SF_ROWS;
        if (causal && j == t) limit = r + 1;
        if (!causal && (j + 1) * SF_ROWS > S) limit = S - j * SF_ROWS;
        float lp[64 / CH];
        sf_update<CH>(v, wc, limit, sl2, m, l, lp);
        const int c0 = (j * SF_ROWS + wc) / CH;
#pragma unroll
        for (int hh = 0; hh < 64 / CH; ++hh) my_lp[(size_t)(c0 + hh) * 128 + r] = lp[hh];
      }
      P += np;
      // merge the four quads' (m, l) of each row; all epilogue warps leave together if any
      // wait gave up
      my_ml[quad * 128 + r] = m;
      my_ml[(4 + quad) * 128 + r] = l;
      if (!bar_and(ok, 1, 32 * SF_EPI_WARPS)) break;
      if (quad == 0) {
        float mm = my_ml[r];
#pragma unroll
        for (int c = 1; c < 4; ++c) mm = fmaxf(mm, my_ml[c * 128 + r]);
        float ll = 0.f;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const float mc = my_ml[c * 128 + r];
          if (mc != -INFINITY) ll += my_ml[(4 + c) * 128 + r] * fast_exp2(mc - mm);
        }
        const float L = mm + sf_lg2(ll);
        Lsm[r] = L;
        const int row = t * SF_ROWS + r;
        if (row < S) neg_lse[((int64_t)b * H + h) * S + row] = -L;
      }
      asm volatile("bar.sync 1, %0;" ::"n"(32 * SF_EPI_WARPS) : "memory");
      // chunk masses of this query tile: sum over its valid rows of 2^(lse_ic - L_i)
      const int nchunk = j_end * CPT;
      const int rows_valid = S - t * SF_ROWS;  // >= 1
      const float4 L4 = reinterpret_cast<const float4*>(Lsm)[lane];
      float* out = part + (((int64_t)b * H + h) * nt + t) * nch_row;
      // four chunks per warp and step: their loads are in flight together
      for (int c0 = ew; c0 < nchunk; c0 += 4 * SF_EPI_WARPS) {
        float4 a[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int c = c0 + u * SF_EPI_WARPS;
          a[u] = c < nchunk ? *reinterpret_cast<const float4*>(my_lp + (size_t)c * 128 + 4 * lane)
                            : make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int c = c0 + u * SF_EPI_WARPS;
          float s = 0.f;
          s += (4 * lane + 0 < rows_valid) ? fast_exp2(a[u].x - L4.x) : 0.f;
          s += (4 * lane + 1 < rows_valid) ? fast_exp2(a[u].y - L4.y) : 0.f;
          s += (4 * lane + 2 < rows_valid) ? fast_exp2(a[u].z - L4.z) : 0.f;
          s += (4 * lane + 3 < rows_valid) ? fast_exp2(a[u].w - L4.w) : 0.f;
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
          if (lane == 0 && c < nchunk) out[c] = s;
        }
      }
      // the next item overwrites the scratch and Lsm only after every warp read them
      asm volatile("bar.sync 1, %0;" ::"n"(32 * SF_EPI_WARPS) : "memory");
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// scores[b, n] = sum over heads h and query tiles t of part[b, h, t, c] over the chunks c of
// block n (chunk tile c * CH / 128 <= t when causal: earlier query tiles see none of its
// keys).  One CTA per (block, sequence); fixed summation order (deterministic).
__global__ void __launch_bounds__(256) score_chunk_reduce_kernel(const float* __restrict__ part, int S, int H,
                                                                 int blk, int ch, int causal,
                                                                 float* __restrict__ scores) {
  const int n = blockIdx.x, b = blockIdx.y;
  const int nb = S / blk;
  const int nt = (S + SF_ROWS - 1) / SF_ROWS;
  const int nch_row = nt * (SF_ROWS / ch);
  const int c0 = n * blk / ch, c1 = (n + 1) * blk / ch;
  const int t_first = causal ? (c0 * ch) / SF_ROWS : 0;
  const int nterm = H * (nt - t_first);
  __shared__ float red[256];
  float acc = 0.f;
  for (int e = threadIdx.x; e < nterm; e += 256) {
    const int h = e / (nt - t_first), t = t_first + e % (nt - t_first);
    const float* pr = part + (((int64_t)b * H + h) * nt + t) * nch_row;
    float s = 0.f;
    for (int c = c0; c < c1; ++c)
      if (!causal || (c * ch) / SF_ROWS <= t) s += pr[c];
    acc += s;
  }
  red[threadIdx.x] = acc;
  __syncthreads();
  for (int o = 128; o > 0; o >>= 1) {
    if (threadIdx.x < o) red[threadIdx.x] += red[threadIdx.x + o];
    __syncthreads();
  }
  if (threadIdx.x == 0 && n < nb) scores[(int64_t)b * nb + n] = red[0];
}

}  // namespace jenga
