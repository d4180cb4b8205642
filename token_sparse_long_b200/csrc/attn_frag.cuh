// Warp-level bf16 tensor-core fragments for the flash-style attention and
// scoring kernels (head_dim 128, 64-row tiles, 4 warps x 16 rows).
//
// Shared-memory tiles are [64 rows][128 bf16] with 16-byte chunks XOR-swizzled by
// (row % 8) so that ldmatrix phases hit 32 distinct banks.
#pragma once

#include "common.cuh"

namespace jenga {

constexpr int AT_D = 128;     // head dim
constexpr int AT_ROWS = 64;   // rows per tile
constexpr int AT_TILE_BYTES = AT_ROWS * AT_D * 2;

__device__ __forceinline__ uint32_t swz(int row, int chunk) {  // byte offset inside a tile
  return (uint32_t)(row * 256 + ((chunk ^ (row & 7)) << 4));
}

// cp.async one 64 x 128 bf16 tile (rows r0.., pitch ld elements) into swizzled smem.
// Rows >= rmax are zero-filled.  128 threads, 8 chunks each.
__device__ __forceinline__ void load_tile_async(uint8_t* s, const bf16* g, int64_t ld, int r0, int rmax) {
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    int e = threadIdx.x + i * 128;  // 0..1023
    int row = e >> 4, ch = e & 15;
    uint32_t dst = smem_u32(s + swz(row, ch));
    const bf16* src = g + (int64_t)(r0 + row) * ld + ch * 8;
    int bytes = (r0 + row < rmax) ? 16 : 0;
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(bytes) : "memory");
  }
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void mma_bf16(float* c, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack2(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

// A fragment (16 x 16) of rows [r0, r0+16), cols [k0, k0+16) of a swizzled tile.
__device__ __forceinline__ void ld_a(const uint8_t* tile, int r0, int k0, uint32_t* a) {
  const int l = threadIdx.x & 31;
  const int row = r0 + (l & 7) + ((l >> 3) & 1) * 8;
  const int ch = (k0 >> 3) + (l >> 4);
  ldsm_x4(smem_u32(tile + swz(row, ch)), a[0], a[1], a[2], a[3]);
}

// B fragments for two n8 tiles, where B[k][n] = T[n][k] (T rows = n, e.g. K for S = Q K^T):
// n rows [n0, n0+16), k cols [k0, k0+16).  b[0..1] -> tile n0, b[2..3] -> tile n0+8.
__device__ __forceinline__ void ld_b_rows(const uint8_t* tile, int n0, int k0, uint32_t* b) {
  const int l = threadIdx.x & 31;
  const int row = n0 + (l & 7) + (l >> 4) * 8;
  const int ch = (k0 >> 3) + ((l >> 3) & 1);
  ldsm_x4(smem_u32(tile + swz(row, ch)), b[0], b[1], b[2], b[3]);
}

// B fragments for two n8 tiles, where B[k][n] = T[k][n] (T rows = k, e.g. V for O = P V):
// k rows [k0, k0+16), n cols [n0, n0+16).
__device__ __forceinline__ void ld_b_cols(const uint8_t* tile, int k0, int n0, uint32_t* b) {
  const int l = threadIdx.x & 31;
  const int row = k0 + (l & 7) + ((l >> 3) & 1) * 8;
  const int ch = (n0 >> 3) + (l >> 4);
  ldsm_x4_t(smem_u32(tile + swz(row, ch)), b[0], b[1], b[2], b[3]);
}

// C (16 x 64 fp32: 8 n8 tiles) = A_tile rows [r0, r0+16) x B^T where B rows come from tileB
// (S = Q K^T pattern).  Clears c first.
__device__ __forceinline__ void mm_rows_x_rowsT(const uint8_t* tA, int r0, const uint8_t* tB, float (*c)[4]) {
#pragma unroll
  for (int j = 0; j < 8; ++j) c[j][0] = c[j][1] = c[j][2] = c[j][3] = 0.f;
#pragma unroll
  for (int ks = 0; ks < AT_D / 16; ++ks) {
    uint32_t a[4];
    ld_a(tA, r0, ks * 16, a);
#pragma unroll
    for (int np = 0; np < 4; ++np) {
      uint32_t b[4];
      ld_b_rows(tB, np * 16, ks * 16, b);
      mma_bf16(c[2 * np], a, b[0], b[1]);
      mma_bf16(c[2 * np + 1], a, b[2], b[3]);
    }
  }
}

// Same with the A operand held in registers (a[8][4]: 8 k-steps of 16 over head_dim).
__device__ __forceinline__ void mm_regs_x_rowsT(const uint32_t (*a)[4], const uint8_t* tB, float (*c)[4]) {
#pragma unroll
  for (int j = 0; j < 8; ++j) c[j][0] = c[j][1] = c[j][2] = c[j][3] = 0.f;
#pragma unroll
  for (int ks = 0; ks < AT_D / 16; ++ks) {
#pragma unroll
    for (int np = 0; np < 4; ++np) {
      uint32_t b[4];
      ld_b_rows(tB, np * 16, ks * 16, b);
      mma_bf16(c[2 * np], a[ks], b[0], b[1]);
      mma_bf16(c[2 * np + 1], a[ks], b[2], b[3]);
    }
  }
}

// acc (16 x 128 fp32: 16 n8 tiles) += P (16 x 64, as C fragments p[8][4]) x T (64 x 128 tile, rows = k)
__device__ __forceinline__ void mm_p_x_cols(const float (*p)[4], const uint8_t* tB, float (*acc)[4]) {
#pragma unroll
  for (int kk = 0; kk < 4; ++kk) {
    uint32_t a[4];
    a[0] = pack2(p[2 * kk][0], p[2 * kk][1]);
    a[1] = pack2(p[2 * kk][2], p[2 * kk][3]);
    a[2] = pack2(p[2 * kk + 1][0], p[2 * kk + 1][1]);
    a[3] = pack2(p[2 * kk + 1][2], p[2 * kk + 1][3]);
#pragma unroll
    for (int dp = 0; dp < 8; ++dp) {
      uint32_t b[4];
      ld_b_cols(tB, kk * 16, dp * 16, b);
      mma_bf16(acc[2 * dp], a, b[0], b[1]);
      mma_bf16(acc[2 * dp + 1], a, b[2], b[3]);
    }
  }
}

}  // namespace jenga
