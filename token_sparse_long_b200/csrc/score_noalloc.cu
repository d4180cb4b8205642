// Block scoring without a caller workspace.
//
// jenga_score_blocks needs scratch (per-row log-sum-exp and per-key column mass) that
// the caller normally passes in.  Some callers cannot provide it: hosts that own all
// device memory and forbid allocations outside their own pool but offer no hook to hand
// us a buffer, and latency-critical callers for which a cudaMalloc / cudaFree (which
// can synchronise the whole device) is not acceptable.  For them this entry point runs
// the same kernels on a fixed scratch array that lives in the library image itself.
//
// The array is a file-scope __device__ object: every GPU that loads the library holds
// it (16 MiB) until the process exits.  Its device address is looked up once per device
// with cudaGetSymbolAddress while that device is current (the first call on the device
// does this, and the first call in a new context after a device reset does it again).  All calls share the array; each call overwrites every element it later
// reads, so no clearing is needed, but two calls whose kernels overlap on the GPU (e.g.
// on different streams) race on it.
#include <mutex>

#include "common.cuh"

namespace jenga {

constexpr size_t NOALLOC_SCRATCH_BYTES = (size_t)16 << 20;

static __device__ __align__(256) unsigned char g_score_scratch[NOALLOC_SCRATCH_BYTES];

static std::mutex s_noalloc_mu;
static void* s_noalloc_ptr[128];
static void* s_noalloc_ctx[128];  // the CUDA context the cached address belongs to

typedef int (*CtxGetCurrentFn)(void**);

static void* current_context() {
  static CtxGetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    cudaDriverEntryPointQueryResult q;
    void* p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(p);
  });
  void* ctx = nullptr;
  if (fn) fn(&ctx);
  return ctx;
}

// Device address of the scratch array in the current context.  Looked up with
// cudaGetSymbolAddress the first time a device is used and again whenever the current
// context differs from the one the cached address was taken in (a new primary context
// after cudaDeviceReset loads the module again, possibly at another address).
static jenga_status noalloc_scratch(void** out) {
  int dev = -1;
  JENGA_CUDA_TRY(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 128) return fail(JENGA_EUNSUPPORTED, "jenga_score_blocks_noalloc: device ordinal %d", dev);
  std::lock_guard<std::mutex> lock(s_noalloc_mu);
  void* ctx = current_context();
  if (!s_noalloc_ptr[dev] || !ctx || ctx != s_noalloc_ctx[dev]) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_score_scratch);
    if (e != cudaSuccess || !p)
      return fail(JENGA_ECUDA, "jenga_score_blocks_noalloc: cudaGetSymbolAddress failed: %s", cudaGetErrorString(e));
    s_noalloc_ptr[dev] = p;
    s_noalloc_ctx[dev] = current_context();  // bound by the lookup if it was not yet
  }
  *out = s_noalloc_ptr[dev];
  return JENGA_OK;
}

}  // namespace jenga

using namespace jenga;

extern "C" size_t jenga_score_blocks_noalloc_max_bytes(void) { return NOALLOC_SCRATCH_BYTES; }

extern "C" jenga_status jenga_score_blocks_noalloc(const void* q, int64_t ldq, const void* k, int64_t ldk, int B,
                                                   int S, int H, int D, int blk, int causal, jenga_dtype dt,
                                                   jenga_score_mode mode, float* scores, jenga_stream_t stream) {
  JENGA_CHECK_ARG(B >= 1 && S >= 1 && H >= 1 && blk >= 1, "jenga_score_blocks_noalloc: bad sizes");
  const size_t need = jenga_score_workspace_bytes(B, S, H, D, blk);
  if (need > NOALLOC_SCRATCH_BYTES)
    return fail(JENGA_EWORKSPACE,
                "jenga_score_blocks_noalloc: these sizes need %zu bytes of scratch "
                "(jenga_score_workspace_bytes), above the library's fixed %zu-byte array; use "
                "jenga_score_blocks with a workspace",
                need, NOALLOC_SCRATCH_BYTES);
  void* scratch = nullptr;
  jenga_status s = noalloc_scratch(&scratch);
  if (s != JENGA_OK) return s;
  return jenga_score_blocks(q, ldq, k, ldk, B, S, H, D, blk, causal, dt, mode, scores, scratch,
                            NOALLOC_SCRATCH_BYTES, stream);
}
