// Decode attention for callers that cannot allocate device memory.
//
// starkv_decode_attention needs a caller-provided workspace for its per-tile partial
// records.  Some callers have no way to provide one: a plugin loaded into a host process
// whose memory pool has already reserved the GPU's memory, a C caller with no allocator of its
// own, or code running where a cudaMalloc is not acceptable because it may synchronise the
// device.  This entry point keeps the partial records in a fixed-size array that lives in
// the library's own device image instead.
#include <mutex>
#include <string>

#include "internal.cuh"

namespace {

// Room for the partial records of one call: batch * n_q_heads * ceil(max_pages / 2) *
// 4 * ceil((2 + max value rank) / 4) floats.  Every GPU that loads the library holds it until
// the process exits.
constexpr size_t kScratchBytes = size_t(16) << 20;  // 16 MiB

static __device__ __align__(256) unsigned char g_decode_scratch[kScratchBytes];

// Device address of g_decode_scratch.  The address belongs to the CUDA context that loaded
// the library's module, so it is cached per context, keyed on the context's unique ID (a
// context that is destroyed and created again, e.g. after cudaDeviceReset, gets a new ID, and
// a caller's own non-primary context gets its own entry).  Host code may not pass the symbol
// itself to a kernel: on the host it is only a stand-in.
using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

struct ScratchEntry {
  unsigned long long ctx_id;
  void* ptr;
};

std::mutex g_mu;
ScratchEntry g_scratch[64] = {};
int g_scratch_n = 0, g_scratch_next = 0;

starkv_status driver_fns(CtxGetCurrentFn& get_current, CtxGetIdFn& get_id) {
  static std::once_flag once;
  static CtxGetCurrentFn s_current = nullptr;
  static CtxGetIdFn s_id = nullptr;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      s_current = reinterpret_cast<CtxGetCurrentFn>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      s_id = reinterpret_cast<CtxGetIdFn>(p);
  });
  if (!s_current || !s_id) {
    starkv::set_error_message("cuCtxGetCurrent / cuCtxGetId not available from the driver");
    return STARKV_ERR_CUDA;
  }
  get_current = s_current;
  get_id = s_id;
  return STARKV_OK;
}

starkv_status symbol_address(void** p) {
  *p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(p, g_decode_scratch);
  if (e != cudaSuccess || *p == nullptr) {
    starkv::set_error_message(std::string("cudaGetSymbolAddress(decode scratch): ") +
                              cudaGetErrorString(e));
    return STARKV_ERR_CUDA;
  }
  return STARKV_OK;
}

starkv_status scratch_address(void** out) {
  CtxGetCurrentFn get_current;
  CtxGetIdFn get_id;
  starkv_status st = driver_fns(get_current, get_id);
  if (st != STARKV_OK) return st;
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS) {
    starkv::set_error_message("cuCtxGetCurrent failed");
    return STARKV_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lock(g_mu);
  void* p = nullptr;
  if (ctx == nullptr) {
    // no context yet on this thread: the lookup itself makes the device's primary context
    // current (the runtime's rule), then its ID keys the entry
    st = symbol_address(&p);
    if (st != STARKV_OK) return st;
    if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) {
      starkv::set_error_message("no current CUDA context after the symbol lookup");
      return STARKV_ERR_CUDA;
    }
  }
  unsigned long long id = 0;
  if (get_id(ctx, &id) != CUDA_SUCCESS) {
    starkv::set_error_message("cuCtxGetId failed");
    return STARKV_ERR_CUDA;
  }
  for (int i = 0; i < g_scratch_n; ++i) {
    if (g_scratch[i].ctx_id == id) {
      *out = g_scratch[i].ptr;
      return STARKV_OK;
    }
  }
  if (p == nullptr) {
    st = symbol_address(&p);
    if (st != STARKV_OK) return st;
  }
  // a small ring of contexts: an entry of a context that no longer exists is only ever
  // overwritten, never used (context IDs are not reused within a process)
  ScratchEntry& slot = g_scratch[g_scratch_next];
  slot.ctx_id = id;
  slot.ptr = p;
  g_scratch_next = (g_scratch_next + 1) % 64;
  if (g_scratch_n < 64) ++g_scratch_n;
  *out = p;
  return STARKV_OK;
}

}  // namespace

extern "C" starkv_status starkv_decode_attention_noalloc(
    const starkv_layout* lay, const void* q, const void* cache, int64_t num_pages,
    const int32_t* block_table, int32_t max_pages, const int32_t* seq_lens, int32_t batch,
    const void* Bk_t, const float* Bv, const void* rope_table, size_t rope_table_bytes, float* out,
    const starkv_decode_opts* opts, int32_t* dev_status, starkv_stream_t stream) {
  starkv_sizes sz;
  starkv_status st = starkv_alloc(lay, 0, batch < 0 ? 0 : batch, max_pages, 0, &sz);
  if (st != STARKV_OK) return st;
  if (sz.decode_workspace_bytes > kScratchBytes) {
    starkv::set_error_message(
        "starkv_decode_attention_noalloc: the partial records of this call need " +
        std::to_string(sz.decode_workspace_bytes) + " bytes, above the built-in " +
        std::to_string(kScratchBytes) +
        "-byte scratch; use starkv_decode_attention with a caller workspace");
    return STARKV_ERR_WORKSPACE;
  }
  void* ws = nullptr;
  st = scratch_address(&ws);
  if (st != STARKV_OK) return st;
  return starkv_decode_attention(lay, q, cache, num_pages, block_table, max_pages, seq_lens, batch,
                                 Bk_t, Bv, rope_table, rope_table_bytes, out, ws, kScratchBytes,
                                 opts, dev_status, stream);
}
