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

// Device address of g_decode_scratch, looked up once per device (with that device current).
// Host code may not pass the symbol itself to a kernel: on the host it is only a stand-in.
std::mutex g_mu;
void* g_scratch_ptr[64] = {};

starkv_status scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    starkv::set_error_message(std::string("cudaGetDevice: ") + cudaGetErrorString(e));
    return STARKV_ERR_CUDA;
  }
  if (dev < 0 || dev >= 64) {
    starkv::set_error_message("device index above 63");
    return STARKV_ERR_UNSUPPORTED;
  }
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e != cudaSuccess || p == nullptr) {
      starkv::set_error_message(std::string("cudaGetSymbolAddress(decode scratch): ") +
                                cudaGetErrorString(e));
      return STARKV_ERR_CUDA;
    }
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
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
  if (lay->cfg.fmt == STARKV_FMT_HAD43) {  // refused before the scratch lookup touches a device
    starkv::set_error_message("decode of the had43 format is not implemented yet");
    return STARKV_ERR_UNSUPPORTED;
  }
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
