// Retained-token Llama decoder layer: weight packing, all-S q/k projection for
// scoring, forward, segment-wise backward (Jenga summary §4.1, §4.4.1, §4.4.2).
#include "gemm_tc.cuh"
#include "layer_kernels.cuh"

namespace jenga {

jenga_status attn_forward(const bf16* q, const bf16* k, const void* v16, int64_t ld, int64_t ld_v16, bf16* o,
                          int64_t ldo, float* lse, int64_t lse_ld, int H, const int32_t* n_valid, int valid_mult,
                          int n_cap, cudaStream_t st, bf16* o_lo);
jenga_status attn_backward_segment(const void* q16, const void* k16, const void* v16, int64_t ld, const float* lse,
                                   int64_t lse_ld, const void* dO16, int64_t ld_do, const float* delta,
                                   int64_t delta_ld, float* dq, int64_t ld_dq, float* dk_acc, float* dv_acc,
                                   int64_t ld_acc, int H, int s0, int s1, const int32_t* n_valid, int valid_mult,
                                   int n_cap, const float* gscal, cudaStream_t st);

constexpr int LORA_R = 16;
constexpr int LORA_PAD = 64;  // padded K of the LoRA operand pairs

// A bump allocator over a caller buffer (256-byte aligned sub-buffers).
struct Carve {
  uintptr_t base, cur, end;
  explicit Carve(void* p, size_t bytes = ~size_t(0) >> 1)
      : base((uintptr_t)p), cur((uintptr_t)p), end(bytes == (~size_t(0) >> 1) ? ~uintptr_t(0) : (uintptr_t)p + bytes) {}
  template <class T>
  T* take(size_t count) {
    cur = (cur + 255) & ~uintptr_t(255);
    T* r = (T*)cur;
    cur += count * sizeof(T);
    return r;
  }
  size_t used() const { return (size_t)(cur - base) + 256; }
  bool ok() const { return cur <= end; }
};

struct Dims {
  int h, H, D, HD, F;
};

static jenga_status check_weights(const jenga_layer_weights* w, const jenga_lora* lora, Dims* d) {
  JENGA_CHECK_ARG(w && lora, "layer: null weights");
  JENGA_CHECK_ARG(w->head_dim == 128, "layer: head_dim must be 128 (got %d)", w->head_dim);
  JENGA_CHECK_ARG(w->hidden > 0 && w->hidden % 256 == 0 && w->hidden <= 8192, "layer: hidden must be a multiple of 256, <= 8192");
  JENGA_CHECK_ARG(w->heads > 0 && w->heads <= 64, "layer: heads must be in [1, 64] (got %d)", w->heads);
  JENGA_CHECK_ARG(w->ffn > 0 && w->ffn % 256 == 0, "layer: ffn must be a multiple of 256");
  JENGA_CHECK_ARG(lora->rank == LORA_R, "layer: LoRA rank must be 16");
  JENGA_CHECK_ARG(w->wq && w->wk && w->wv && w->wo && w->wg && w->wu && w->wd && w->attn_norm && w->mlp_norm,
                  "layer: null weight pointer");
  JENGA_CHECK_ARG(lora->aq && lora->bq && lora->av && lora->bv, "layer: null LoRA pointer");
  d->h = w->hidden;
  d->H = w->heads;
  d->D = w->head_dim;
  d->HD = w->heads * w->head_dim;
  d->F = w->ffn;
  JENGA_CHECK_ARG(d->HD % 256 == 0, "layer: heads * head_dim must be a multiple of 256");
  return JENGA_OK;
}

// The backward operands woT, wqkvT, bcat and aqvT (and wguT) are stored fp16: the products
// that read them take fp16 A operands (row-scaled gradients), and one tcgen05 product has
// one operand type.  aqvT carries the factor lora_c (lora_l1_divisor_kernel).
struct Packed {
  bf16 *wqkv, *lorab, *aqv, *wgu, *woT, *wdT, *wguT, *wqkvT, *bcat, *aqvT;
  double* inv_freq;
  float* lora_c;
};

static size_t carve_packed(Carve& c, const Dims& d, Packed* p) {
  p->wqkv = c.take<bf16>((size_t)3 * d.HD * d.h);
  p->lorab = c.take<bf16>((size_t)3 * d.HD * LORA_PAD);
  p->aqv = c.take<bf16>((size_t)2 * LORA_R * d.h);
  p->wgu = c.take<bf16>((size_t)2 * d.F * d.h);
  p->woT = c.take<bf16>((size_t)d.HD * d.h);
  p->wdT = c.take<bf16>((size_t)d.F * d.h);
  p->wguT = c.take<bf16>((size_t)d.h * 2 * d.F);
  p->wqkvT = c.take<bf16>((size_t)d.h * 3 * d.HD);
  p->bcat = c.take<bf16>((size_t)2 * LORA_R * 3 * d.HD);
  p->aqvT = c.take<bf16>((size_t)d.h * LORA_PAD);
  p->inv_freq = c.take<double>(64);
  p->lora_c = c.take<float>(4);
  return c.used();
}

struct Saved {
  bf16 *xr, *qkv, *o, *hres;
  float *t, *lse, *rstd1, *rstd2;
  uint8_t* mlp_mask;  // [n_kept_max]: 1 = the MLP sub-block runs on this retained block
  bf16* olo;          // [nc, HD] bf16 rounding residual of o (the backward's Delta uses hi + lo)
  __half* gu;         // [nc, 2F] fp16 MLP pre-activations (g, u) in the interleaved gate/up layout
};

static size_t carve_saved(Carve& c, const Dims& d, int nc, Saved* s) {
  s->xr = c.take<bf16>((size_t)nc * d.h);
  s->qkv = c.take<bf16>((size_t)nc * 3 * d.HD);
  s->o = c.take<bf16>((size_t)nc * d.HD);
  s->hres = c.take<bf16>((size_t)nc * d.h);
  s->t = c.take<float>((size_t)nc * 2 * LORA_R);
  s->lse = c.take<float>((size_t)d.H * nc);
  s->rstd1 = c.take<float>(nc);
  s->rstd2 = c.take<float>(nc);
  s->mlp_mask = c.take<uint8_t>(nc > 0 ? (size_t)nc : 1);  // >= n_kept_max entries (one per retained block)
  s->olo = c.take<bf16>((size_t)nc * d.HD);
  s->gu = c.take<__half>((size_t)nc * 2 * d.F);
  return c.used();
}

struct FwdWs {
  bf16 *xn, *tb, *a;
  float2* rope;  // [nc][64] (cos, sin) of the retained rows' positions
  float* mlp_scores;  // MLP-block criterion per retained block
  int32_t *mlp_pos, *n_mlp;
  __half* v16;        // [nc, HD] fp16 copy of v (the PV product's operand)
};
static size_t carve_fwd_ws(Carve& c, const Dims& d, int nc, FwdWs* w) {
  w->xn = c.take<bf16>((size_t)nc * d.h);
  w->tb = c.take<bf16>((size_t)nc * LORA_PAD);
  w->a = c.take<bf16>((size_t)nc * d.F);
  w->rope = c.take<float2>((size_t)nc * 64);
  const size_t nbk = nc > 0 ? (size_t)nc : 1;  // >= n_kept_max
  w->mlp_scores = c.take<float>(nbk);
  w->mlp_pos = c.take<int32_t>(nbk);
  w->n_mlp = c.take<int32_t>(1);
  w->v16 = c.take<__half>((size_t)nc * d.HD);
  return c.used();
}

// The dt product (M = segment rows, N = 32, K = 3 H D) has one output tile per 128 rows: its
// reduction is split into up to DT_SPLIT_MAX ranges so that about one work tile per SM runs.
constexpr int DT_SPLIT_MAX = 8;
static int dt_split(int T, int K) {
  const int ntm = (T + 127) / 128;
  int ks = sm_count() / (ntm > 0 ? ntm : 1);
  ks = ks < 1 ? 1 : (ks > DT_SPLIT_MAX ? DT_SPLIT_MAX : ks);
  return ks < K / 64 ? ks : K / 64;
}

struct BwdWs {
  float *dk_acc, *dv_acc;
  bf16 *xn, *g, *dgu, *dO;
  __half *dh16, *dqkv16, *dtb;  // fp16 A operands: dh and dQKV row-scaled, the LoRA term / lora_c
  float *rs_dh, *rs_qkv;        // their per-row inverse scales
  float* dtpart;                // [DT_SPLIT_MAX][T][32] partial sums of the split dt product
  float *dhn, *dh, *delta, *dq, *dt, *part;
  float2* rope;  // [T][64] (cos, sin) of the segment rows' positions
  __half* qkv16;   // [nc, 3 HD] fp16 copy of the saved q | k | v (attention backward operands)
  float* dOf;      // [T, HD] fp32 dO of the segment (scaled to fp16 into dO)
  float* gscal;    // [4] norms and scales of the fp16 attention backward
};
static size_t carve_bwd_ws(Carve& c, const Dims& d, int nc, int T, BwdWs* w) {
  w->dk_acc = c.take<float>((size_t)nc * d.HD);
  w->dv_acc = c.take<float>((size_t)nc * d.HD);
  w->qkv16 = c.take<__half>((size_t)nc * 3 * d.HD);
  w->dOf = c.take<float>((size_t)T * d.HD);
  w->gscal = c.take<float>(4);
  w->xn = c.take<bf16>((size_t)T * d.h);
  w->g = c.take<bf16>((size_t)T * d.h);
  w->dgu = c.take<bf16>((size_t)T * 2 * d.F);
  w->dh16 = c.take<__half>((size_t)T * d.h);
  w->dO = c.take<bf16>((size_t)T * d.HD);
  w->dqkv16 = c.take<__half>((size_t)T * 3 * d.HD);
  w->dtb = c.take<__half>((size_t)T * LORA_PAD);
  w->rs_dh = c.take<float>(T);
  w->rs_qkv = c.take<float>(T);
  w->dtpart = c.take<float>((size_t)DT_SPLIT_MAX * T * 2 * LORA_R);
  w->dhn = c.take<float>((size_t)T * d.h);
  w->dh = c.take<float>((size_t)T * d.h);
  w->delta = c.take<float>((size_t)d.H * T);
  w->dq = c.take<float>((size_t)T * d.HD);
  w->dt = c.take<float>((size_t)T * 2 * LORA_R);
  w->rope = c.take<float2>((size_t)T * 64);
  const int chunks = (T + LG_CHUNK - 1) / LG_CHUNK;
  const int cmax = d.HD > d.h ? d.HD : d.h;
  w->part = c.take<float>((size_t)4 * chunks * cmax * 16);
  return c.used();
}

static int grid_cap(int64_t work, int per_block) {
  int64_t g = (work + per_block - 1) / per_block;
  int cap = sm_count() * 16;
  if (g < 1) g = 1;
  return (int)(g < cap ? g : cap);
}

static jenga_status transpose(const bf16* src, int64_t lds, bf16* dst, int64_t ldd, int R, int C, cudaStream_t st) {
  dim3 g((C + 31) / 32, (R + 31) / 32);
  {
  const int _ps = ::jenga::prof_begin("transpose_bf16", st);
  transpose_bf16_kernel<<<g, dim3(32, 8), 0, st>>>(src, lds, dst, ldd, R, C);
  ::jenga::prof_end(_ps, st);
  }
  JENGA_LAUNCH_CHECK();
  return JENGA_OK;
}
static jenga_status copy2d(const bf16* src, int64_t lds, bf16* dst, int64_t ldd, int R, int C, cudaStream_t st) {
  {
  const int _ps = ::jenga::prof_begin("copy_bf16", st);
  copy_bf16_kernel<<<grid_cap((int64_t)R * C, 256), 256, 0, st>>>(src, lds, dst, ldd, R, C);
  ::jenga::prof_end(_ps, st);
  }
  JENGA_LAUNCH_CHECK();
  return JENGA_OK;
}
static jenga_status zero(bf16* dst, int64_t n, cudaStream_t st) {
  {
  const int _ps = ::jenga::prof_begin("zero_bf16", st);
  zero_bf16_kernel<<<grid_cap(n, 256), 256, 0, st>>>(dst, n);
  ::jenga::prof_end(_ps, st);
  }
  JENGA_LAUNCH_CHECK();
  return JENGA_OK;
}

#define JENGA_TRY(expr)                   \
  do {                                    \
    jenga_status _s = (expr);             \
    if (_s != JENGA_OK) return _s;        \
  } while (0)

static EpiParams epi_base(const int32_t* idx, int blk, const int32_t* n_kept, int row_offset) {
  EpiParams e;
  e.idx = idx;
  e.blk = blk;
  e.n_valid = n_kept;
  e.valid_mult = blk;
  e.row_offset = row_offset;
  return e;
}

static jenga_status rmsnorm(const bf16* x, int64_t ldx, const int32_t* idx, int blk, int row_offset,
                            const int32_t* n_valid, int mult, int rows, int h, float eps, const bf16* gain, bf16* xr,
                            bf16* xn, float* rstd, cudaStream_t st, int64_t x_rows = 0) {
  if (rows <= 0) return JENGA_OK;
  {
  const int _ps = ::jenga::prof_begin("rmsnorm_rows", st);
  if (h <= 16 * ROW_THREADS)
    rmsnorm_rows_kernel<2><<<rows, ROW_THREADS, 0, st>>>(x, ldx, idx, blk, row_offset, n_valid, mult, h, eps, gain,
                                                         xr, h, xn, h, rstd, x_rows ? x_rows : rows);
  else
    rmsnorm_rows_kernel<4><<<rows, ROW_THREADS, 0, st>>>(x, ldx, idx, blk, row_offset, n_valid, mult, h, eps, gain,
                                                         xr, h, xn, h, rstd, x_rows ? x_rows : rows);
  ::jenga::prof_end(_ps, st);
  }
  JENGA_LAUNCH_CHECK();
  return JENGA_OK;
}

}  // namespace jenga

using namespace jenga;

// ==================================================================== pack
extern "C" size_t jenga_layer_pack_bytes(const jenga_layer_weights* w, const jenga_lora* lora) {
  Dims d;
  if (check_weights(w, lora, &d) != JENGA_OK) return 0;
  Carve c(nullptr);
  Packed p;
  return carve_packed(c, d, &p);
}

extern "C" jenga_status jenga_layer_pack(const jenga_layer_weights* w, const jenga_lora* lora, void* packed,
                                         size_t packed_bytes, jenga_stream_t stream) {
  Dims d;
  JENGA_TRY(check_weights(w, lora, &d));
  const size_t need = jenga_layer_pack_bytes(w, lora);
  if (!packed || packed_bytes < need) return fail(JENGA_EWORKSPACE, "jenga_layer_pack: %zu < %zu bytes", packed_bytes, need);
  cudaStream_t st = (cudaStream_t)stream;
  Carve c(packed, packed_bytes);
  Packed p;
  carve_packed(c, d, &p);
  const int h = d.h, HD = d.HD, F = d.F;
  const bf16* wq = (const bf16*)w->wq;
  const bf16* wk = (const bf16*)w->wk;
  const bf16* wv = (const bf16*)w->wv;
  const bf16* wg = (const bf16*)w->wg;
  const bf16* wu = (const bf16*)w->wu;
  // fused QKV [3HD, h]
  JENGA_TRY(copy2d(wq, h, p.wqkv, h, HD, h, st));
  JENGA_TRY(copy2d(wk, h, p.wqkv + (size_t)HD * h, h, HD, h, st));
  JENGA_TRY(copy2d(wv, h, p.wqkv + (size_t)2 * HD * h, h, HD, h, st));
  // LoRA up-projection as a K=64 operand: rows of q -> cols 0..15 = Bq, rows of v -> cols 16..31 = Bv
  // The A operand of that phase is [s t (bf16), s t - bf16(s t) (bf16)] (EPI_LORA_T), so the
  // B columns repeat: q rows cols 0..15 and 32..47 = Bq, v rows cols 16..31 and 48..63 = Bv;
  // the LoRA term then carries the rounding residual of s t (about 16 mantissa bits).
  JENGA_TRY(zero(p.lorab, (int64_t)3 * HD * LORA_PAD, st));
  for (int half = 0; half < 2; ++half) {
    JENGA_TRY(copy2d((const bf16*)lora->bq, LORA_R, p.lorab + half * 2 * LORA_R, LORA_PAD, HD, LORA_R, st));
    JENGA_TRY(copy2d((const bf16*)lora->bv, LORA_R, p.lorab + (size_t)2 * HD * LORA_PAD + LORA_R + half * 2 * LORA_R,
                     LORA_PAD, HD, LORA_R, st));
  }
  // LoRA down-projection [Aq; Av] (32 x h)
  JENGA_TRY(copy2d((const bf16*)lora->aq, h, p.aqv, h, LORA_R, h, st));
  JENGA_TRY(copy2d((const bf16*)lora->av, h, p.aqv + (size_t)LORA_R * h, h, LORA_R, h, st));
  // gate/up interleaved in groups of 64 rows: [g 0..63, u 0..63, g 64..127, u 64..127, ...]
  {
    const int _ps = ::jenga::prof_begin("interleave_gate_up", st);
    interleave_gate_up_kernel<<<grid_cap((int64_t)2 * F * h, 256), 256, 0, st>>>(wg, wu, p.wgu, F, h);
    ::jenga::prof_end(_ps, st);
  }
  JENGA_LAUNCH_CHECK();
  // transposes for the backward
  JENGA_TRY(transpose((const bf16*)w->wo, HD, p.woT, h, h, HD, st));          // Wo [h, HD] -> [HD, h]
  JENGA_TRY(transpose((const bf16*)w->wd, F, p.wdT, h, h, F, st));            // Wd [h, F]  -> [F, h]
  JENGA_TRY(transpose(p.wgu, h, p.wguT, 2 * F, 2 * F, h, st));                // [2F, h]    -> [h, 2F]
  JENGA_TRY(transpose(p.wqkv, h, p.wqkvT, 3 * HD, 3 * HD, h, st));            // [3HD, h]   -> [h, 3HD]
  // dt = dqkv * bcat^T : rows 0..15 = [Bq^T | 0 | 0], rows 16..31 = [0 | 0 | Bv^T]
  JENGA_TRY(zero(p.bcat, (int64_t)2 * LORA_R * 3 * HD, st));
  JENGA_TRY(transpose((const bf16*)lora->bq, LORA_R, p.bcat, 3 * HD, HD, LORA_R, st));
  JENGA_TRY(transpose((const bf16*)lora->bv, LORA_R, p.bcat + (size_t)LORA_R * 3 * HD + 2 * HD, 3 * HD, HD, LORA_R, st));
  // [Aq; Av]^T padded to 64 columns: [h, 64]
  // (columns 32..63 repeat 0..31: the A operand carries dt's hi and lo halves, EPI_LORA_T)
  JENGA_TRY(transpose(p.aqv, h, p.aqvT, LORA_PAD, 2 * LORA_R, h, st));
  JENGA_TRY(transpose(p.aqv, h, p.aqvT + 2 * LORA_R, LORA_PAD, 2 * LORA_R, h, st));
  {  // the divisor of the fp16 LoRA operand of the dX product (from bcat while it is bf16)
    const int _ps = ::jenga::prof_begin("lora_l1_divisor", st);
    lora_l1_divisor_kernel<<<1, 1024, 0, st>>>(p.bcat, 2 * LORA_R, 3 * HD, lora->scale, p.lora_c);
    ::jenga::prof_end(_ps, st);
  }
  JENGA_LAUNCH_CHECK();
  // the backward products run on fp16 operands: re-encode their weight operands in place
  {
    struct {
      bf16* w;
      int64_t n;
      const float* mul;
    } conv[5] = {{p.wguT, (int64_t)h * 2 * F, nullptr},
                 {p.woT, (int64_t)HD * h, nullptr},
                 {p.wqkvT, (int64_t)h * 3 * HD, nullptr},
                 {p.bcat, (int64_t)2 * LORA_R * 3 * HD, nullptr},
                 {p.aqvT, (int64_t)h * LORA_PAD, p.lora_c}};
    for (int i = 0; i < 5; ++i) {
      const int _ps = ::jenga::prof_begin("bf16_to_f16_inplace", st);
      bf16_to_f16_inplace_kernel<<<grid_cap(conv[i].n, 256), 256, 0, st>>>((uint16_t*)conv[i].w, conv[i].n,
                                                                          conv[i].mul);
      ::jenga::prof_end(_ps, st);
      JENGA_LAUNCH_CHECK();
    }
  }
  {
  const int _ps = ::jenga::prof_begin("inv_freq", st);
  inv_freq_kernel<<<1, 64, 0, st>>>(p.inv_freq, d.D, log2((double)w->rope_theta));
  ::jenga::prof_end(_ps, st);
  }
  JENGA_LAUNCH_CHECK();
  return JENGA_OK;
}

// ==================================================================== score q/k (a1)
extern "C" size_t jenga_layer_score_qk_workspace_bytes(const jenga_layer_weights* w, int B, int S) {
  if (!w || B < 1 || S < 1) return 0;
  Carve c(nullptr);
  c.take<bf16>((size_t)S * w->hidden);
  c.take<float>((size_t)S * 2 * LORA_R);
  c.take<bf16>((size_t)S * LORA_PAD);
  c.take<float2>((size_t)S * 64);
  return c.used();
}

extern "C" jenga_status jenga_layer_score_qk(const jenga_layer_weights* w, const jenga_lora* lora, const void* packed,
                                             const void* x, int B, int S, void* qk, void* ws, size_t ws_bytes,
                                             jenga_stream_t stream) {
  Dims d;
  JENGA_TRY(check_weights(w, lora, &d));
  JENGA_CHECK_ARG(packed && x && qk, "jenga_layer_score_qk: null pointer");
  JENGA_CHECK_ARG(B == 1, "jenga_layer_score_qk: batch 1 only");
  JENGA_CHECK_ARG(S >= 1, "jenga_layer_score_qk: S");
  const size_t need = jenga_layer_score_qk_workspace_bytes(w, B, S);
  if (!ws || ws_bytes < need) return fail(JENGA_EWORKSPACE, "jenga_layer_score_qk: workspace %zu < %zu", ws_bytes, need);
  cudaStream_t st = (cudaStream_t)stream;
  Carve pc((void*)packed);
  Packed p;
  carve_packed(pc, d, &p);
  Carve c(ws, ws_bytes);
  bf16* xn = c.take<bf16>((size_t)S * d.h);
  float* t = c.take<float>((size_t)S * 2 * LORA_R);
  bf16* tb = c.take<bf16>((size_t)S * LORA_PAD);
  float2* rope = c.take<float2>((size_t)S * 64);
  {
    const int _ps = ::jenga::prof_begin("rope_table", st);
    rope_table_kernel<<<grid_cap((int64_t)S * 64, 256), 256, 0, st>>>(rope, S, nullptr, 1, nullptr, 1, 0, p.inv_freq);
    ::jenga::prof_end(_ps, st);
  }
  JENGA_LAUNCH_CHECK();
  JENGA_TRY(rmsnorm((const bf16*)x, d.h, nullptr, 1, 0, nullptr, 1, S, d.h, w->rms_eps, (const bf16*)w->attn_norm,
                    nullptr, xn, nullptr, st));
  EpiParams e;
  e.out = t;
  e.ldo = 2 * LORA_R;
  e.aux = tb;
  e.ld_aux = LORA_PAD;
  e.alpha = lora->scale;
  e.beta = 1.f;
  JENGA_TRY((launch_gemm<32, EPI_LORA_T>({xn, S, d.h}, {p.aqv, 2 * LORA_R, d.h}, d.h, nullptr, nullptr, 0, S,
                                         2 * LORA_R, e, st, "gemm_lora_t_all")));
  EpiParams q;
  q.out = qk;
  q.ldo = 2 * d.HD;
  q.hd = d.HD;
  q.rope_tab = rope;
  GemmOperand a2{tb, S, LORA_PAD}, b2{p.lorab, 2 * d.HD, LORA_PAD};
  JENGA_TRY((launch_gemm<256, EPI_QKV_ROPE>({xn, S, d.h}, {p.wqkv, 2 * d.HD, d.h}, d.h, &a2, &b2, LORA_PAD, S,
                                            2 * d.HD, q, st, "gemm_qk_rope_all")));
  return JENGA_OK;
}

// ==================================================================== forward
extern "C" size_t jenga_layer_saved_bytes(const jenga_layer_weights* w, int B, int blk, int n_kept_max) {
  if (!w || B < 1 || blk < 1 || n_kept_max < 0) return 0;
  Dims d{w->hidden, w->heads, w->head_dim, w->heads * w->head_dim, w->ffn};
  Carve c(nullptr);
  Saved s;
  return carve_saved(c, d, n_kept_max * blk, &s);
}

extern "C" size_t jenga_layer_fwd_workspace_bytes(const jenga_layer_weights* w, int B, int blk, int n_kept_max) {
  if (!w || B < 1 || blk < 1 || n_kept_max < 0) return 0;
  Dims d{w->hidden, w->heads, w->head_dim, w->heads * w->head_dim, w->ffn};
  Carve c(nullptr);
  FwdWs f;
  return carve_fwd_ws(c, d, n_kept_max * blk, &f);
}

// mlp_mode < 0: the MLP sub-block runs on every retained block.  Otherwise the MLP-block
// criterion (jenga_mlp_block_scores over a = SiLU(g) * u of the retained blocks) is selected
// with jenga_select(mlp_mode, mlp_param) over the n_kept_max retained positions, and the MLP
// sub-block (down projection and its residual add here; its backward later) runs only on
// the kept positions (Jenga summary §4.2.4).
static jenga_status layer_fwd(const jenga_layer_weights* w, const jenga_lora* lora, const void* packed, void* x,
                              int B, int S, int blk, const int32_t* idx, const int32_t* n_kept, int n_kept_max,
                              void* saved, size_t saved_bytes, void* ws, size_t ws_bytes, const void* qk_all,
                              int64_t ld_qk, jenga_stream_t stream, int mlp_mode = -1, float mlp_param = 0.f,
                              int32_t* mlp_pos_out = nullptr, int32_t* n_mlp_out = nullptr,
                              float* mlp_scores_out = nullptr) {
  Dims d;
  JENGA_TRY(check_weights(w, lora, &d));
  JENGA_CHECK_ARG(packed && x && idx && n_kept, "jenga_sparse_layer_fwd: null pointer");
  JENGA_CHECK_ARG(B == 1, "jenga_sparse_layer_fwd: batch 1 only");
  JENGA_CHECK_ARG(blk >= 64 && blk % 64 == 0 && S % blk == 0, "jenga_sparse_layer_fwd: blk must be a multiple of 64 dividing S");
  JENGA_CHECK_ARG(n_kept_max >= 0 && n_kept_max <= S / blk, "jenga_sparse_layer_fwd: n_kept_max");
  const size_t need_s = jenga_layer_saved_bytes(w, B, blk, n_kept_max);
  const size_t need_w = jenga_layer_fwd_workspace_bytes(w, B, blk, n_kept_max);
  if (!saved || saved_bytes < need_s) return fail(JENGA_EWORKSPACE, "jenga_sparse_layer_fwd: saved %zu < %zu", saved_bytes, need_s);
  if (!ws || ws_bytes < need_w) return fail(JENGA_EWORKSPACE, "jenga_sparse_layer_fwd: workspace %zu < %zu", ws_bytes, need_w);
  const int nc = n_kept_max * blk;
  if (nc == 0) return JENGA_OK;
  cudaStream_t st = (cudaStream_t)stream;
  Carve pc((void*)packed);
  Packed p;
  carve_packed(pc, d, &p);
  Carve sc(saved, saved_bytes);
  Saved s;
  carve_saved(sc, d, nc, &s);
  Carve wc(ws, ws_bytes);
  FwdWs f;
  carve_fwd_ws(wc, d, nc, &f);
  bf16* X = (bf16*)x;
  const int h = d.h, HD = d.HD, F = d.F;

  // 1. permutation-free gather of the retained rows + RMSNorm
  JENGA_TRY(rmsnorm(X, h, idx, blk, 0, n_kept, blk, nc, h, w->rms_eps, (const bf16*)w->attn_norm, s.xr, f.xn, s.rstd1, st,
                    S));
  // 2. LoRA down-projection t = xn [Aq; Av]^T (fp32 saved) and s * t (bf16, K-padded)
  {
    EpiParams e = epi_base(idx, blk, n_kept, 0);
    e.out = s.t;
    e.ldo = 2 * LORA_R;
    e.aux = f.tb;
    e.ld_aux = LORA_PAD;
    e.alpha = lora->scale;
    e.beta = 1.f;
    JENGA_TRY((launch_gemm<32, EPI_LORA_T>({f.xn, nc, h}, {p.aqv, 2 * LORA_R, h}, h, nullptr, nullptr, 0, nc,
                                           2 * LORA_R, e, st, "gemm_lora_t")));
  }
  // 3. QKV (+ LoRA up-projection as a second K phase) with RoPE at original positions.
  //    With the scoring's q | k of all rows (same x, same kernels, so the same bits), the
  //    retained rows' q and k are copied from it and only v (+ LoRA-v) is projected.
  if (qk_all) {
    {
      const int _ps = ::jenga::prof_begin("gather_qk_rows", st);
      gather_rows_bf16_kernel<<<grid_cap((int64_t)nc * (2 * HD / 8), 256), 256, 0, st>>>(
          (const bf16*)qk_all, ld_qk, s.qkv, 3 * HD, 2 * HD, idx, blk, n_kept, blk, nc);
      ::jenga::prof_end(_ps, st);
    }
    JENGA_LAUNCH_CHECK();
    EpiParams e = epi_base(idx, blk, n_kept, 0);
    e.out = s.qkv + 2 * HD;
    e.ldo = 3 * HD;
    e.hd = HD;
    e.col0 = 2 * HD;  // the v section: no RoPE
    GemmOperand a2{f.tb, nc, LORA_PAD}, b2{p.lorab + (size_t)2 * HD * LORA_PAD, HD, LORA_PAD};
    JENGA_TRY((launch_gemm<256, EPI_QKV_ROPE>({f.xn, nc, h}, {p.wqkv + (size_t)2 * HD * h, HD, h}, h, &a2, &b2,
                                              LORA_PAD, nc, HD, e, st, "gemm_v")));
  } else {
    EpiParams e = epi_base(idx, blk, n_kept, 0);
    e.out = s.qkv;
    e.ldo = 3 * HD;
    e.hd = HD;
    e.rope_tab = f.rope;
    {
      const int _ps = ::jenga::prof_begin("rope_table", st);
      rope_table_kernel<<<grid_cap((int64_t)nc * 64, 256), 256, 0, st>>>(f.rope, nc, idx, blk, n_kept, blk, 0,
                                                                        p.inv_freq);
      ::jenga::prof_end(_ps, st);
    }
    JENGA_LAUNCH_CHECK();
    GemmOperand a2{f.tb, nc, LORA_PAD}, b2{p.lorab, 3 * HD, LORA_PAD};
    JENGA_TRY((launch_gemm<256, EPI_QKV_ROPE>({f.xn, nc, h}, {p.wqkv, 3 * HD, h}, h, &a2, &b2, LORA_PAD, nc, 3 * HD,
                                              e, st, "gemm_qkv_rope")));
  }
  // 4. causal attention among retained tokens (q/k/v rows past the device count are
  //    zeroed first: the tensor-core tiles read them and multiply them by zero weights)
  {
    const int _ps = ::jenga::prof_begin("zero_tail_rows", st);
    zero_tail_rows_kernel<<<sm_count(), 256, 0, st>>>(s.qkv, 3 * HD, 3 * HD, n_kept, blk, nc);
    ::jenga::prof_end(_ps, st);
  }
  JENGA_LAUNCH_CHECK();
  {
    const int _ps = ::jenga::prof_begin("v_to_f16", st);
    qkv_to_f16_kernel<<<grid_cap((int64_t)nc * (HD / 8), 256), 256, 0, st>>>(s.qkv + 2 * HD, 3 * HD, f.v16, HD, nc, HD,
                                                                              -1, nullptr);
    ::jenga::prof_end(_ps, st);
  }
  JENGA_LAUNCH_CHECK();
  JENGA_TRY(attn_forward(s.qkv, s.qkv + HD, f.v16, 3 * HD, HD, s.o, HD, s.lse, nc, d.H, n_kept, blk, nc, st, s.olo));
  // 5. o_proj with the in-place residual add into X (and a compact copy of h)
  {
    EpiParams e = epi_base(idx, blk, n_kept, 0);
    e.x = X;
    e.ldx = h;
    e.x_rows = S;
    e.aux = s.hres;
    e.ld_aux = h;
    JENGA_TRY((launch_gemm<256, EPI_SCATTER_ADD>({s.o, nc, HD}, {w->wo, h, HD}, HD, nullptr, nullptr, 0, nc, h, e, st, "gemm_o_scatter")));
  }
  // 6. RMSNorm before the MLP
  JENGA_TRY(rmsnorm(s.hres, h, nullptr, 1, 0, n_kept, blk, nc, h, w->rms_eps, (const bf16*)w->mlp_norm, nullptr, f.xn,
                    s.rstd2, st));
  // 7. gate/up with SiLU(g) * u
  {
    EpiParams e = epi_base(idx, blk, n_kept, 0);
    e.out = f.a;
    e.ldo = F;
    e.aux = s.gu;  // (g, u) saved for the backward's SwiGLU derivative
    e.ld_aux = 2 * F;
    JENGA_TRY((launch_gemm<256, EPI_SWIGLU>({f.xn, nc, h}, {p.wgu, 2 * F, h}, h, nullptr, nullptr, 0, nc, 2 * F, e, st, "gemm_gateup_swiglu")));
  }
  // 8. the blocks the MLP sub-block runs on: all retained blocks, or the ones the MLP-block
  //    criterion keeps (a mask over retained positions, saved for the backward)
  if (mlp_mode < 0) {
    JENGA_CUDA_TRY(cudaMemsetAsync(s.mlp_mask, 1, (size_t)n_kept_max, st));
  } else {
    float* msc = mlp_scores_out ? mlp_scores_out : f.mlp_scores;
    JENGA_TRY(jenga_mlp_block_scores(f.a, F, F, blk, n_kept, n_kept_max, msc, stream));
    JENGA_TRY(jenga_select(msc, 1, n_kept_max, (jenga_select_mode)mlp_mode, mlp_param,
                           mlp_pos_out ? mlp_pos_out : f.mlp_pos, n_mlp_out ? n_mlp_out : f.n_mlp, s.mlp_mask,
                           nullptr, 0, stream));
  }
  // 9. down_proj with the in-place residual add into X (kept MLP blocks only)
  {
    EpiParams e = epi_base(idx, blk, n_kept, 0);
    e.x = X;
    e.ldx = h;
    e.x_rows = S;
    e.blk_mask = s.mlp_mask;
    e.mask_blk = blk;
    JENGA_TRY((launch_gemm<256, EPI_SCATTER_ADD>({f.a, nc, F}, {w->wd, h, F}, F, nullptr, nullptr, 0, nc, h, e, st, "gemm_down_scatter")));
  }
  return JENGA_OK;
}

extern "C" jenga_status jenga_sparse_layer_fwd(const jenga_layer_weights* w, const jenga_lora* lora,
                                               const void* packed, void* x, int B, int S, int blk, const int32_t* idx,
                                               const int32_t* n_kept, int n_kept_max, void* saved, size_t saved_bytes,
                                               void* ws, size_t ws_bytes, jenga_stream_t stream) {
  return layer_fwd(w, lora, packed, x, B, S, blk, idx, n_kept, n_kept_max, saved, saved_bytes, ws, ws_bytes, nullptr,
                   0, stream);
}

extern "C" jenga_status jenga_sparse_layer_fwd_qk(const jenga_layer_weights* w, const jenga_lora* lora,
                                                  const void* packed, void* x, int B, int S, int blk,
                                                  const int32_t* idx, const int32_t* n_kept, int n_kept_max,
                                                  const void* qk_all, int64_t ld_qk, void* saved, size_t saved_bytes,
                                                  void* ws, size_t ws_bytes, jenga_stream_t stream) {
  Dims d;
  JENGA_TRY(check_weights(w, lora, &d));
  JENGA_CHECK_ARG(qk_all && ld_qk >= 2 * (int64_t)d.HD && ld_qk % 8 == 0 && ((uintptr_t)qk_all & 15) == 0,
                  "jenga_sparse_layer_fwd_qk: qk_all must be [S, >= 2 H D] bf16, 16-byte aligned rows");
  return layer_fwd(w, lora, packed, x, B, S, blk, idx, n_kept, n_kept_max, saved, saved_bytes, ws, ws_bytes, qk_all,
                   ld_qk, stream);
}

extern "C" jenga_status jenga_sparse_layer_fwd_mlp(const jenga_layer_weights* w, const jenga_lora* lora,
                                                   const void* packed, void* x, int B, int S, int blk,
                                                   const int32_t* idx, const int32_t* n_kept, int n_kept_max,
                                                   const void* qk_all, int64_t ld_qk, jenga_select_mode mlp_mode,
                                                   float mlp_param, float* mlp_scores, int32_t* mlp_pos,
                                                   int32_t* n_mlp, void* saved, size_t saved_bytes, void* ws,
                                                   size_t ws_bytes, jenga_stream_t stream) {
  Dims d;
  JENGA_TRY(check_weights(w, lora, &d));
  JENGA_CHECK_ARG(mlp_mode == JENGA_SELECT_TOPK_FRAC || mlp_mode == JENGA_SELECT_TOPK || mlp_mode == JENGA_SELECT_ABS_GE,
                  "jenga_sparse_layer_fwd_mlp: MLP selection mode must be TOPK_FRAC, TOPK or ABS_GE");
  JENGA_CHECK_ARG(n_kept_max <= 8192, "jenga_sparse_layer_fwd_mlp: n_kept_max <= 8192");
  if (qk_all)
    JENGA_CHECK_ARG(ld_qk >= 2 * (int64_t)d.HD && ld_qk % 8 == 0 && ((uintptr_t)qk_all & 15) == 0,
                    "jenga_sparse_layer_fwd_mlp: qk_all must be [S, >= 2 H D] bf16, 16-byte aligned rows");
  return layer_fwd(w, lora, packed, x, B, S, blk, idx, n_kept, n_kept_max, saved, saved_bytes, ws, ws_bytes, qk_all,
                   ld_qk, stream, (int)mlp_mode, mlp_param, mlp_pos, n_mlp, mlp_scores);
}

// ==================================================================== backward
extern "C" size_t jenga_layer_bwd_workspace_bytes(const jenga_layer_weights* w, int B, int blk, int n_kept_max,
                                                  int segment_tokens) {
  if (!w || B < 1 || blk < 1 || n_kept_max < 0 || segment_tokens < 1) return 0;
  Dims d{w->hidden, w->heads, w->head_dim, w->heads * w->head_dim, w->ffn};
  const int nc = n_kept_max * blk;
  const int T = segment_tokens < nc ? segment_tokens : (nc > 0 ? nc : 1);
  Carve c(nullptr);
  BwdWs b;
  return carve_bwd_ws(c, d, nc, T, &b);
}

extern "C" jenga_status jenga_sparse_layer_bwd(const jenga_layer_weights* w, const jenga_lora* lora,
                                               const void* packed, void* dx, int B, int S, int blk, const int32_t* idx,
                                               const int32_t* n_kept, int n_kept_max, const void* saved,
                                               size_t saved_bytes, jenga_lora_grads* grads, int segment_tokens,
                                               void* ws, size_t ws_bytes, jenga_stream_t stream) {
  Dims d;
  JENGA_TRY(check_weights(w, lora, &d));
  JENGA_CHECK_ARG(packed && dx && idx && n_kept && saved && grads, "jenga_sparse_layer_bwd: null pointer");
  JENGA_CHECK_ARG(grads->daq && grads->dbq && grads->dav && grads->dbv, "jenga_sparse_layer_bwd: null gradient");
  JENGA_CHECK_ARG(B == 1, "jenga_sparse_layer_bwd: batch 1 only");
  JENGA_CHECK_ARG(blk >= 64 && blk % 64 == 0 && S % blk == 0, "jenga_sparse_layer_bwd: blk");
  JENGA_CHECK_ARG(n_kept_max >= 0 && n_kept_max <= S / blk, "jenga_sparse_layer_bwd: n_kept_max");
  JENGA_CHECK_ARG(segment_tokens >= 128 && segment_tokens % 128 == 0 && segment_tokens % blk == 0,
                  "jenga_sparse_layer_bwd: segment_tokens must be a multiple of 128 and of blk");
  const size_t need_s = jenga_layer_saved_bytes(w, B, blk, n_kept_max);
  const size_t need_w = jenga_layer_bwd_workspace_bytes(w, B, blk, n_kept_max, segment_tokens);
  if (saved_bytes < need_s) return fail(JENGA_EWORKSPACE, "jenga_sparse_layer_bwd: saved %zu < %zu", saved_bytes, need_s);
  if (!ws || ws_bytes < need_w) return fail(JENGA_EWORKSPACE, "jenga_sparse_layer_bwd: workspace %zu < %zu", ws_bytes, need_w);
  const int nc = n_kept_max * blk;
  if (nc == 0) return JENGA_OK;
  cudaStream_t st = (cudaStream_t)stream;
  const int h = d.h, HD = d.HD, F = d.F, H = d.H;
  const float ls = lora->scale;
  Carve pc((void*)packed);
  Packed p;
  carve_packed(pc, d, &p);
  Carve sc((void*)saved, saved_bytes);
  Saved s;
  carve_saved(sc, d, nc, &s);
  const int Tmax = segment_tokens < nc ? segment_tokens : nc;
  Carve wc(ws, ws_bytes);
  BwdWs b;
  carve_bwd_ws(wc, d, nc, Tmax, &b);
  bf16* dX = (bf16*)dx;

  JENGA_CUDA_TRY(cudaMemsetAsync(b.dk_acc, 0, (size_t)nc * HD * sizeof(float), st));
  JENGA_CUDA_TRY(cudaMemsetAsync(b.dv_acc, 0, (size_t)nc * HD * sizeof(float), st));
  // fp16 operands of the attention backward: q | k | v copies and the largest per-head v norm
  if ((int64_t)nc * (3 * HD / 8) >= (int64_t)1 << 31)
    return fail(JENGA_EUNSUPPORTED, "jenga_sparse_layer_bwd: retained rows x 3 H D too large");
  JENGA_CUDA_TRY(cudaMemsetAsync(b.gscal, 0, 4 * sizeof(float), st));
  {
    const int _ps = ::jenga::prof_begin("qkv_to_f16", st);
    qkv_to_f16_kernel<<<grid_cap((int64_t)nc * (3 * HD / 8), 256), 256, 0, st>>>(
        s.qkv, 3 * HD, b.qkv16, 3 * HD, nc, 3 * HD, 2 * HD, reinterpret_cast<unsigned int*>(b.gscal));
    ::jenga::prof_end(_ps, st);
  }
  JENGA_LAUNCH_CHECK();
  const int nseg = (nc + segment_tokens - 1) / segment_tokens;
  for (int sg = nseg - 1; sg >= 0; --sg) {
    const int s0 = sg * segment_tokens;
    const int s1 = (s0 + segment_tokens < nc) ? s0 + segment_tokens : nc;
    const int T = s1 - s0;
    // --- MLP block (the forward saved the pre-activations (g, u) in fp16)
    // upstream gradient rows of this segment
    {
    const int _ps = ::jenga::prof_begin("gather_seg", st);
    gather_seg_kernel<<<grid_cap((int64_t)T * (h / 8), 256), 256, 0, st>>>(dX, h, b.g, h, idx, blk, s0, n_kept, blk, T, h,
                                                                         S);
    ::jenga::prof_end(_ps, st);
    }
    JENGA_LAUNCH_CHECK();
    // dA = G Wd ; (dg, du) from SiLU(g) * u; the MLP GEMMs skip the 128-row tiles whose
    // blocks the MLP sub-block did not run on
    {
      EpiParams e = epi_base(idx, blk, n_kept, s0);
      e.out = b.dgu;
      e.ldo = 2 * F;
      e.aux = s.gu + (size_t)s0 * 2 * F;
      e.ld_aux = 2 * F;
      e.aux_f16 = true;
      e.blk_mask = s.mlp_mask;
      e.mask_blk = blk;
      JENGA_TRY((launch_gemm<256, EPI_SWIGLU_BWD>({b.g, T, h}, {p.wdT, F, h}, h, nullptr, nullptr, 0, T, F, e, st, "gemm_da_swiglu_bwd")));
    }
    // dhn = [dg, du] [Wg; Wu]
    {
      EpiParams e = epi_base(idx, blk, n_kept, s0);
      e.out = b.dhn;
      e.ldo = h;
      e.blk_mask = s.mlp_mask;
      e.mask_blk = blk;
      JENGA_TRY((launch_gemm<256, EPI_STORE_F32>({b.dgu, T, 2 * F}, {p.wguT, h, 2 * F}, 2 * F, nullptr, nullptr, 0, T,
                                                 h, e, st, "gemm_dhn", nullptr, nullptr, 0, /*f16_inputs=*/true)));
    }
    // dh = G + RMSNorm_bwd(dhn)
    {
    const int _ps = ::jenga::prof_begin("rmsnorm_bwd_rows", st);
    (h <= 16 * ROW_THREADS ? rmsnorm_bwd_rows_kernel<2> : rmsnorm_bwd_rows_kernel<4>)<<<T, ROW_THREADS, 0, st>>>(
        b.dhn, h, s.hres + (size_t)s0 * h, h, s.rstd2 + s0,
                                                        (const bf16*)w->mlp_norm, nullptr, b.g, h, b.dh, b.dh16,
                                                        b.rs_dh, h, nullptr, 0, idx, blk, s0, n_kept, blk, h, S,
                                                        s.mlp_mask, blk);
    ::jenga::prof_end(_ps, st);
    }
    JENGA_LAUNCH_CHECK();
    // --- attention block: dO = dh Wo (fp32), then its fp16 form with a power-of-two scale and
    //     the scaled Delta
    {
      EpiParams e = epi_base(idx, blk, n_kept, s0);
      e.out = b.dOf;
      e.ldo = HD;
      // dh enters as fp16 rows scaled into [2^13, 2^14); the epilogue undoes the row scale
      e.row_scale = b.rs_dh;
      JENGA_TRY((launch_gemm<256, EPI_STORE_F32>({b.dh16, T, h}, {p.woT, HD, h}, h, nullptr, nullptr, 0, T, HD, e,
                                                 st, "gemm_do", nullptr, nullptr, 0, /*f16_inputs=*/true)));
    }
    JENGA_CUDA_TRY(cudaMemsetAsync(b.gscal + 1, 0, sizeof(float), st));
    {
      const int _ps = ::jenga::prof_begin("do_norm_max", st);
      do_norm_max_kernel<<<grid_cap((int64_t)T * H * 32, 256), 256, 0, st>>>(
          b.dOf, HD, T, H, s0, n_kept, blk, reinterpret_cast<unsigned int*>(b.gscal));
      ::jenga::prof_end(_ps, st);
    }
    JENGA_LAUNCH_CHECK();
    {
      const int _ps = ::jenga::prof_begin("do_to_f16_delta", st);
      do_to_f16_delta_kernel<<<grid_cap((int64_t)T * H * 32, 256), 256, 0, st>>>(
          b.dOf, HD, s.o, s.olo, HD, reinterpret_cast<__half*>(b.dO), HD, b.delta, T, T, H, s0, n_kept, blk, b.gscal);
      ::jenga::prof_end(_ps, st);
    }
    JENGA_LAUNCH_CHECK();
    JENGA_TRY(attn_backward_segment(b.qkv16, b.qkv16 + HD, b.qkv16 + 2 * HD, 3 * HD, s.lse, nc, b.dO, HD, b.delta, T,
                                    b.dq, HD, b.dk_acc, b.dv_acc, HD, H, s0, s1, n_kept, blk, nc, b.gscal, st));
    // keys of this segment are complete: RoPE^T and pack dQKV (bf16)
    {
    const int _ps = ::jenga::prof_begin("rope_table", st);
    rope_table_kernel<<<grid_cap((int64_t)T * 64, 256), 256, 0, st>>>(b.rope, T, idx, blk, n_kept, blk, s0,
                                                                       p.inv_freq);
    ::jenga::prof_end(_ps, st);
    }
    JENGA_LAUNCH_CHECK();
    {
    const int _ps = ::jenga::prof_begin("rope_bwd_pack", st);
    (H <= ROW_THREADS / 8 ? rope_bwd_pack_kernel<4> : rope_bwd_pack_kernel<8>)<<<T, ROW_THREADS, 0, st>>>(
        b.dq, HD, b.dk_acc, b.dv_acc, HD, s0, b.dqkv16, b.rs_qkv, 3 * HD, b.rope, n_kept, blk, T, H);
    ::jenga::prof_end(_ps, st);
    }
    JENGA_LAUNCH_CHECK();
    // dt = s [dq Bq, dv Bv]: fp32 (the row scale undone) for the LoRA gradients, and the
    // still row-scaled value / lora_c as the fp16 K-padded LoRA operand of the dX product;
    // the product's reduction is split over ranges (partial sums, then lora_t_reduce)
    {
      const int ks = dt_split(T, 3 * HD);
      EpiParams e = epi_base(idx, blk, n_kept, s0);
      e.out = b.dtpart;
      e.ldo = 2 * LORA_R;
      e.ksplit = ks;
      JENGA_TRY((launch_gemm<32, EPI_STORE_F32>({b.dqkv16, T, 3 * HD}, {p.bcat, 2 * LORA_R, 3 * HD}, 3 * HD, nullptr,
                                                nullptr, 0, T, 2 * LORA_R, e, st, "gemm_dt", nullptr, nullptr, 0,
                                                /*f16_inputs=*/true)));
      const int _ps = ::jenga::prof_begin("lora_t_reduce", st);
      lora_t_reduce_kernel<<<grid_cap((int64_t)T * 32, 256), 256, 0, st>>>(
          b.dtpart, ks, T, n_kept, blk, s0, ls, b.rs_qkv, p.lora_c, b.dt, 2 * LORA_R, b.dtb, LORA_PAD);
      ::jenga::prof_end(_ps, st);
      JENGA_LAUNCH_CHECK();
    }
    // xn of the segment (recomputed from the saved gathered input)
    JENGA_TRY(rmsnorm(s.xr + (size_t)s0 * h, h, nullptr, 1, s0, n_kept, blk, T, h, w->rms_eps,
                      (const bf16*)w->attn_norm, nullptr, b.xn, nullptr, st));
    // LoRA gradients (deterministic split over rows), all four products in one launch
    {
      const int chunks = (T + LG_CHUNK - 1) / LG_CHUNK;
      const int cmax = HD > h ? HD : h;
      LoraGradJobs jobs;
      jobs.j[0] = {b.dqkv16, 3 * HD, s.t + (size_t)s0 * 2 * LORA_R, HD, ls, grads->dbq, LORA_R, 1, b.rs_qkv, 1};
      jobs.j[1] = {b.dqkv16 + 2 * HD, 3 * HD, s.t + (size_t)s0 * 2 * LORA_R + LORA_R, HD, ls, grads->dbv, LORA_R, 1,
                   b.rs_qkv, 1};
      jobs.j[2] = {b.xn, h, b.dt, h, 1.f, grads->daq, 1, h, nullptr, 0};
      jobs.j[3] = {b.xn, h, b.dt + LORA_R, h, 1.f, grads->dav, 1, h, nullptr, 0};
      {
        const int _ps = ::jenga::prof_begin("lora_grad_partial", st);
        lora_grad_partial_kernel<<<dim3((cmax + LG_COLS - 1) / LG_COLS, chunks, 4), 256, 0, st>>>(
            jobs, 2 * LORA_R, T, n_kept, blk, s0, cmax, b.part);
        ::jenga::prof_end(_ps, st);
      }
      JENGA_LAUNCH_CHECK();
      {
        const int _ps = ::jenga::prof_begin("lora_grad_reduce", st);
        lora_grad_reduce_kernel<<<dim3((cmax * 16 + 255) / 256, 4), 256, 0, st>>>(jobs, b.part, chunks, cmax);
        ::jenga::prof_end(_ps, st);
      }
      JENGA_LAUNCH_CHECK();
    }
    // dxn = dQKV [Wq; Wk; Wv] + dt [Aq; Av]
    {
      EpiParams e = epi_base(idx, blk, n_kept, s0);
      e.out = b.dhn;
      e.ldo = h;
      // dQKV enters as fp16 rows scaled into [2^13, 2^14); the second K phase adds the LoRA
      // term (s_m dt / lora_c) (lora_c [Aq; Av]); the epilogue undoes the row scale
      e.row_scale = b.rs_qkv;
      GemmOperand a2{b.dtb, T, LORA_PAD}, b2{p.aqvT, h, LORA_PAD};
      JENGA_TRY((launch_gemm<256, EPI_STORE_F32>({b.dqkv16, T, 3 * HD}, {p.wqkvT, h, 3 * HD}, 3 * HD, &a2, &b2,
                                                 LORA_PAD, T, h, e, st, "gemm_dxn", nullptr, nullptr, 0,
                                                 /*f16_inputs=*/true)));
    }
    // dX[rows] = dh + RMSNorm_bwd(dxn)  (written in place into the gradient buffer)
    {
    const int _ps = ::jenga::prof_begin("rmsnorm_bwd_rows", st);
    (h <= 16 * ROW_THREADS ? rmsnorm_bwd_rows_kernel<2> : rmsnorm_bwd_rows_kernel<4>)<<<T, ROW_THREADS, 0, st>>>(
        b.dhn, h, s.xr + (size_t)s0 * h, h, s.rstd1 + s0, (const bf16*)w->attn_norm, b.dh, nullptr, h, nullptr,
        nullptr, nullptr, h, dX, h, idx, blk, s0, n_kept, blk, h, S, nullptr, 1);
    ::jenga::prof_end(_ps, st);
    }
    JENGA_LAUNCH_CHECK();
  }
  return JENGA_OK;
}

// ==================================================================== test hook
// C[M, N] = A[M, K] B[N, K]^T (bf16 in, fp32 accumulate), stored bf16 or fp32.
extern "C" jenga_status jenga_test_gemm(const void* A, int64_t lda, const void* B, int64_t ldb, int M, int N, int K,
                                        void* C, int64_t ldc, int out_f32, int bn, jenga_stream_t stream) {
  JENGA_CHECK_ARG(A && B && C && M > 0 && N > 0 && K > 0 && K % 64 == 0, "jenga_test_gemm: bad args");
  EpiParams e;
  e.out = C;
  e.ldo = ldc;
  cudaStream_t st = (cudaStream_t)stream;
  if (bn == 256) {
    if (out_f32) return launch_gemm<256, EPI_STORE_F32>({A, M, lda}, {B, N, ldb}, K, nullptr, nullptr, 0, M, N, e, st);
    return launch_gemm<256, EPI_STORE_BF16>({A, M, lda}, {B, N, ldb}, K, nullptr, nullptr, 0, M, N, e, st);
  }
  if (bn == 32) return launch_gemm<32, EPI_STORE_F32>({A, M, lda}, {B, N, ldb}, K, nullptr, nullptr, 0, M, N, e, st);
  return fail(JENGA_EINVAL, "jenga_test_gemm: bn must be 256 or 32");
}

// 2^x through exp2_fma (FMA-pipe exponential) and through the multi-function unit, for
// accuracy tests of the former.
__global__ void test_exp2_kernel(const float* __restrict__ x, float* __restrict__ y_fma, float* __restrict__ y_mufu,
                                 int n) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
    y_fma[i] = exp2_fma<64>(x[i]);
    y_mufu[i] = fast_exp2(x[i]);
  }
}

extern "C" jenga_status jenga_test_exp2(const float* x, float* y_fma, float* y_mufu, int n, jenga_stream_t stream) {
  JENGA_CHECK_ARG(x && y_fma && y_mufu && n >= 0, "jenga_test_exp2: bad args");
  if (n == 0) return JENGA_OK;
  test_exp2_kernel<<<(n + 255) / 256 < 1024 ? (n + 255) / 256 : 1024, 256, 0, (cudaStream_t)stream>>>(x, y_fma,
                                                                                                     y_mufu, n);
  JENGA_LAUNCH_CHECK();
  return JENGA_OK;
}
