// The C ABI: argument validation, cache layout, launch planning, TMA tensor maps.
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>

#include "internal.cuh"

using namespace starkv;

namespace {

thread_local std::string g_last_error;

starkv_status fail(starkv_status s, const std::string& msg) {
  g_last_error = msg;
  return s;
}
starkv_status cuda_fail(cudaError_t e, const char* where) {
  return fail(STARKV_ERR_CUDA, std::string(where) + ": " + cudaGetErrorString(e));
}

int64_t align16(int64_t x) { return (x + 15) / 16 * 16; }
int ceil_div(int a, int b) { return (a + b - 1) / b; }

// ---------------------------------------------------------------- device properties
struct DevInfo {
  bool ok = false;
  int sms = 0;
  int major = 0, minor = 0;
  size_t smem_optin = 0;
};

starkv_status current_device(DevInfo& info) {
  static std::mutex mu;
  static DevInfo cache[64];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= 64) return fail(STARKV_ERR_UNSUPPORTED, "device index above 63");
  std::lock_guard<std::mutex> lock(mu);
  if (!cache[dev].ok) {
    cudaDeviceProp prop;
    e = cudaGetDeviceProperties(&prop, dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDeviceProperties");
    cache[dev].sms = prop.multiProcessorCount;
    cache[dev].major = prop.major;
    cache[dev].minor = prop.minor;
    cache[dev].smem_optin = prop.sharedMemPerBlockOptin;
    cache[dev].ok = true;
  }
  info = cache[dev];
  if (info.major != 10)
    return fail(STARKV_ERR_UNSUPPORTED, "this library is built for sm_100a (B200); device is sm_" +
                                            std::to_string(info.major * 10 + info.minor));
  return STARKV_OK;
}

// ---------------------------------------------------------------- tensor maps
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

starkv_status get_encoder(EncodeTiledFn& fn) {
  static std::once_flag once;
  static EncodeTiledFn cached = nullptr;
  static cudaError_t err = cudaSuccess;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    err = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q);
    if (err == cudaSuccess && q == cudaDriverEntryPointSuccess) cached = reinterpret_cast<EncodeTiledFn>(p);
  });
  if (!cached) return fail(STARKV_ERR_CUDA, "cuTensorMapEncodeTiled not available");
  fn = cached;
  return STARKV_OK;
}

starkv_status encode(CUtensorMap* map, CUtensorMapDataType dt, int rank, const void* base,
                     const cuuint64_t* dims, const cuuint64_t* strides, const cuuint32_t* box) {
  EncodeTiledFn fn;
  starkv_status st = get_encoder(fn);
  if (st != STARKV_OK) return st;
  cuuint32_t es[3] = {1, 1, 1};
  CUresult r = fn(map, dt, rank, const_cast<void*>(base), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return fail(STARKV_ERR_CUDA, "cuTensorMapEncodeTiled failed (" + std::to_string(int(r)) + ")");
  return STARKV_OK;
}

int elem_size(int fmt) { return fmt == STARKV_FMT_F32 ? 4 : 2; }

LatDesc lat_desc(const starkv_segment& s) {
  LatDesc d{};
  d.rank = s.rank;
  d.col = s.col;
  d.n8 = s.n8;
  d.nb4 = s.nb4;
  d.g8 = s.g8;
  d.ng = s.g8 + s.g4;
  d.pitch = s.pitch;
  if (s.off_plain >= 0) {
    d.off0 = static_cast<int>(s.off_plain);
    d.off1 = d.off2 = 0;
  } else {
    d.off0 = static_cast<int>(s.off_i8);
    d.off1 = static_cast<int>(s.off_i4);
    d.off2 = static_cast<int>(s.off_sc);
  }
  return d;
}

starkv_status check_layout(const starkv_layout* lay) {
  if (!lay) return fail(STARKV_ERR_INVALID_ARG, "layout is NULL");
  starkv_layout chk;
  const bool hybrid = lay->assignment == STARKV_ASSIGN_HYBRID;
  if (!hybrid && lay->assignment != STARKV_ASSIGN_JOINT_KEYS)
    return fail(STARKV_ERR_INVALID_ARG, "layout has an unknown assignment");
  const starkv_status st =
      hybrid ? starkv_hybrid_layout_init(&lay->hybrid, &chk) : starkv_layout_init(&lay->cfg, &chk);
  if (st != STARKV_OK) return st;
  if (std::memcmp(&chk, lay, sizeof(chk)) != 0)
    return fail(STARKV_ERR_INVALID_ARG, "layout was not produced by its layout_init for its config");
  return STARKV_OK;
}

// The joint-key decode calls (latent 0 the key latent, latent 1+g the value latent of KV
// head g) take every format (f32, bf16, int8/int4, had43) but only that assignment.
starkv_status check_decode_format(const starkv_layout* lay) {
  if (lay->assignment != STARKV_ASSIGN_JOINT_KEYS)
    return fail(STARKV_ERR_UNSUPPORTED,
                "a hybrid layout (keys head-wise, values joint) decodes with starkv_hybrid_decode");
  return STARKV_OK;
}

// Formats stored as codes with fp16 group scales, decoded by the dequantisers.
bool quantised(int fmt) { return fmt == STARKV_FMT_MIXED || fmt == STARKV_FMT_HAD43; }

// Split-K plan of the projection: about one CTA per SM of a B200 (148), every split non-empty.
constexpr int kProjCtaTarget = 148;
void proj_plan(const starkv_layout* lay, int n_tok, int& kb_total, int& kb_per_split, int& nsplit) {
  const int ke = 128 / elem_size(lay->cfg.fmt);
  kb_total = ceil_div(lay->cfg.d_model, ke);
  const int tiles = ceil_div(n_tok, 128) * ceil_div(lay->proj_cols, 256);
  int want = kProjCtaTarget / (tiles > 0 ? tiles : 1);
  if (want < 1) want = 1;
  if (want > kb_total) want = kb_total;
  kb_per_split = ceil_div(kb_total, want);
  nsplit = ceil_div(kb_total, kb_per_split);
}

size_t proj_workspace(const starkv_layout* lay, int n_tok) {
  int kt, kps, ns;
  proj_plan(lay, n_tok, kt, kps, ns);
  return static_cast<size_t>(ns) * n_tok * lay->proj_cols * sizeof(float);
}

int rope_tiles_for(int max_pages) { return ceil_div(max_pages * kPage, kTile); }
size_t rope_bytes(const starkv_layout* lay, int max_pages) {
  return static_cast<size_t>(kTile + rope_tiles_for(max_pages)) * (lay->cfg.head_dim / 2) * sizeof(float2);
}
int record_floats(const starkv_layout* lay) { return (2 + lay->value_rank_max + 3) / 4 * 4; }
int tiles_for(int max_pages) { return ceil_div(max_pages * kPage, kTile); }

// Hybrid decode: page ranges per sequence, so that batch x ranges is about kHybUnitsTarget.
void hybrid_splits(int batch, int max_pages, int& nsplit, int& pps) {
  int want = (kHybUnitsTarget + std::max(batch, 1) - 1) / std::max(batch, 1);
  want = std::max(1, std::min(want, max_pages));
  pps = ceil_div(max_pages, want);
  nsplit = ceil_div(max_pages, pps);
}
int hybrid_rec(const starkv_layout* lay) { return (2 + lay->value_rank_total + 3) / 4 * 4; }

// Bytes of the decode partial records of `batch` sequences: batch * n_q_heads * tiles * rec
// floats (hybrid: batch * n_q_heads * page ranges * rec), multiplied in 64 bits with an
// overflow check at every step.  Also refuses a batch * n_q_heads above the combine kernel's
// grid limit (one CTA per sequence and head).
starkv_status decode_ws_bytes(const starkv_layout* lay, int32_t batch, int32_t max_pages,
                              size_t* out) {
  const bool hybrid = lay->assignment == STARKV_ASSIGN_HYBRID;
  int nsplit = 0, pps = 0;
  if (hybrid) hybrid_splits(batch, max_pages, nsplit, pps);
  const uint64_t factors[4] = {static_cast<uint64_t>(lay->cfg.n_q_heads),
                               static_cast<uint64_t>(hybrid ? nsplit : tiles_for(max_pages)),
                               static_cast<uint64_t>(hybrid ? hybrid_rec(lay) : record_floats(lay)),
                               sizeof(float)};
  if (static_cast<uint64_t>(batch) * factors[0] > 0x7FFFFFFFull)
    return fail(STARKV_ERR_INVALID_ARG, "batch * n_q_heads above 2^31 - 1");
  uint64_t n = static_cast<uint64_t>(batch);
  for (uint64_t f : factors) {
    if (f != 0 && n > SIZE_MAX / f)
      return fail(STARKV_ERR_INVALID_ARG, "decode workspace size does not fit in size_t");
    n *= f;
  }
  *out = static_cast<size_t>(n);
  return STARKV_OK;
}

// Places latents of ``ranks`` (page order) into L.seg, sets their projection columns, the page
// size and the stored bytes per token.  Each block starts on a 16-byte boundary.
starkv_status place_latents(starkv_layout& L, int fmt, const int* ranks, int n) {
  int64_t off = 0, token_bytes = 0;
  int col = 0;
  auto place = [&](int64_t nbytes) {
    const int64_t o = off;
    off = align16(off + nbytes);
    return o;
  };
  for (int li = 0; li < n; ++li) {
    const int r = ranks[li];
    starkv_segment& s = L.seg[li];
    s.rank = r;
    s.col = col;
    col += r;
    s.off_plain = s.off_i8 = s.off_i4 = s.off_sc = -1;
    if (fmt == STARKV_FMT_MIXED) {
      s.n8 = (r + 3) / 4;
      s.n4 = r - s.n8;
      s.g8 = (s.n8 + STARKV_GROUP - 1) / STARKV_GROUP;
      s.g4 = (s.n4 + STARKV_GROUP - 1) / STARKV_GROUP;
      s.nb4 = (s.n4 + 1) / 2;
      s.off_i8 = place(static_cast<int64_t>(kPage) * s.n8);
      s.off_i4 = place(static_cast<int64_t>(kPage) * s.nb4);
      s.off_sc = place(static_cast<int64_t>(kPage) * 2 * (s.g8 + s.g4));
      token_bytes += s.n8 + s.nb4 + 2 * (s.g8 + s.g4);
    } else if (fmt == STARKV_FMT_HAD43) {
      s.n8 = (r + 4) / 5;  // the outlier block: a fifth of the channels, rounded up
      s.n4 = r - s.n8;
      s.g8 = (s.n8 + STARKV_GROUP - 1) / STARKV_GROUP;
      s.g4 = (s.n4 + STARKV_GROUP - 1) / STARKV_GROUP;
      s.pitch = (s.n8 + 1) / 2;
      s.nb4 = 3 * ((s.n4 + 7) / 8);
      s.off_i8 = place(static_cast<int64_t>(kPage) * s.pitch);
      s.off_i4 = place(static_cast<int64_t>(kPage) * s.nb4);
      s.off_sc = place(static_cast<int64_t>(kPage) * 2 * (s.g8 + s.g4));
      token_bytes += s.pitch + s.nb4 + 2 * (s.g8 + s.g4);
    } else {
      const int es = elem_size(fmt);
      s.pitch = r * es;
      s.off_plain = place(static_cast<int64_t>(kPage) * r * es);
      token_bytes += static_cast<int64_t>(r) * es;
    }
  }
  L.n_latents = n;
  L.proj_cols = col;
  L.page_bytes = off;
  L.token_bytes = token_bytes;
  if (L.page_bytes >= (int64_t(1) << 31)) return fail(STARKV_ERR_UNSUPPORTED, "page larger than 2 GiB");
  return STARKV_OK;
}

void fill_store(StoreParams& sp, const starkv_layout* lay) {
  sp.fmt = lay->cfg.fmt;
  sp.n_lat = lay->n_latents;
  sp.proj_cols = lay->proj_cols;
  int chunks = 0;
  for (int i = 0; i < lay->n_latents; ++i) {
    sp.lat[i] = lat_desc(lay->seg[i]);
    sp.chunk_start[i] = static_cast<short>(chunks);
    const starkv_segment& g = lay->seg[i];
    const bool grouped = lay->cfg.fmt == STARKV_FMT_MIXED || lay->cfg.fmt == STARKV_FMT_HAD43;
    chunks += grouped ? g.g8 + g.g4 : (g.rank + 31) / 32;
  }
  sp.chunk_start[lay->n_latents] = static_cast<short>(chunks);
  sp.chunks_per_token = chunks;
}

}  // namespace

namespace starkv {
void set_error_message(const std::string& msg) { g_last_error = msg; }
}  // namespace starkv

extern "C" {

const char* starkv_last_error(void) { return g_last_error.c_str(); }

int32_t starkv_version(void) { return 100; }

starkv_status starkv_layout_init(const starkv_config* cfg, starkv_layout* out) {
  if (!cfg || !out) return fail(STARKV_ERR_INVALID_ARG, "cfg/out is NULL");
  const starkv_config& c = *cfg;
  if (c.n_kv_heads < 1 || c.n_kv_heads > STARKV_MAX_KV_HEADS)
    return fail(STARKV_ERR_INVALID_ARG, "n_kv_heads must be in [1, 64]");
  if (c.n_q_heads < c.n_kv_heads || c.n_q_heads % c.n_kv_heads != 0)
    return fail(STARKV_ERR_INVALID_ARG, "n_q_heads must be a positive multiple of n_kv_heads");
  const int G = c.n_q_heads / c.n_kv_heads;
  if (G != 1 && G != 2 && G != 4 && G != 8)
    return fail(STARKV_ERR_UNSUPPORTED, "query heads per KV head must be 1, 2, 4 or 8");
  if (c.head_dim != 64 && c.head_dim != 128)
    return fail(STARKV_ERR_UNSUPPORTED, "head_dim must be 64 or 128");
  if (c.d_model < 16 || c.d_model % 16 != 0)
    return fail(STARKV_ERR_INVALID_ARG, "d_model must be a positive multiple of 16");
  if (c.key_rank < 16 || c.key_rank % 16 != 0 || c.key_rank > 2048)
    return fail(STARKV_ERR_INVALID_ARG, "key_rank must be a multiple of 16 in [16, 2048]");
  if (c.fmt != STARKV_FMT_F32 && c.fmt != STARKV_FMT_BF16 && c.fmt != STARKV_FMT_MIXED &&
      c.fmt != STARKV_FMT_HAD43)
    return fail(STARKV_ERR_INVALID_ARG, "unknown latent format");
  if (c.page_tokens != kPage) return fail(STARKV_ERR_UNSUPPORTED, "page_tokens must be 64");
  if (!(c.rope_theta > 1.0) || !std::isfinite(c.rope_theta))
    return fail(STARKV_ERR_INVALID_ARG, "rope_theta must be finite and > 1");
  for (int g = 0; g < c.n_kv_heads; ++g)
    if (c.value_rank[g] < 1 || c.value_rank[g] > c.head_dim)
      return fail(STARKV_ERR_INVALID_ARG, "value_rank[g] must be in [1, head_dim]");

  starkv_layout L;
  std::memset(&L, 0, sizeof(L));
  L.cfg = c;
  for (int g = c.n_kv_heads; g < STARKV_MAX_KV_HEADS; ++g) L.cfg.value_rank[g] = 0;
  L.assignment = STARKV_ASSIGN_JOINT_KEYS;
  int ranks[1 + STARKV_MAX_KV_HEADS];
  int rv_total = 0, rv_max = 0;
  ranks[0] = c.key_rank;
  for (int g = 0; g < c.n_kv_heads; ++g) {
    ranks[1 + g] = c.value_rank[g];
    rv_total += c.value_rank[g];
    rv_max = std::max(rv_max, c.value_rank[g]);
  }
  const starkv_status st = place_latents(L, c.fmt, ranks, 1 + c.n_kv_heads);
  if (st != STARKV_OK) return st;
  L.value_rank_total = rv_total;
  L.value_rank_max = rv_max;
  *out = L;
  return STARKV_OK;
}

starkv_status starkv_hybrid_layout_init(const starkv_hybrid_config* cfg, starkv_layout* out) {
  if (!cfg || !out) return fail(STARKV_ERR_INVALID_ARG, "cfg/out is NULL");
  const starkv_hybrid_config& c = *cfg;
  if (c.n_kv_heads < 1 || c.n_kv_heads > STARKV_MAX_KV_HEADS)
    return fail(STARKV_ERR_INVALID_ARG, "n_kv_heads must be in [1, 64]");
  if (c.n_q_heads < c.n_kv_heads || c.n_q_heads % c.n_kv_heads != 0)
    return fail(STARKV_ERR_INVALID_ARG, "n_q_heads must be a positive multiple of n_kv_heads");
  const int G = c.n_q_heads / c.n_kv_heads;
  if (G != 1 && G != 2 && G != 4 && G != 8)
    return fail(STARKV_ERR_UNSUPPORTED, "query heads per KV head must be 1, 2, 4 or 8");
  if (c.head_dim != 64 && c.head_dim != 128)
    return fail(STARKV_ERR_UNSUPPORTED, "head_dim must be 64 or 128");
  if (c.d_model < 16 || c.d_model % 16 != 0)
    return fail(STARKV_ERR_INVALID_ARG, "d_model must be a positive multiple of 16");
  for (int g = 0; g < c.n_kv_heads; ++g)
    if (c.key_rank[g] < 16 || c.key_rank[g] % 16 != 0 || c.key_rank[g] > c.head_dim)
      return fail(STARKV_ERR_INVALID_ARG, "key_rank[g] must be a multiple of 16 in [16, head_dim]");
  if (c.value_rank < 16 || c.value_rank % 16 != 0 ||
      c.value_rank > std::min(2048, c.n_kv_heads * c.head_dim))
    return fail(STARKV_ERR_INVALID_ARG,
                "value_rank must be a multiple of 16 in [16, min(2048, n_kv_heads * head_dim)]");
  if (c.fmt != STARKV_FMT_F32 && c.fmt != STARKV_FMT_BF16 && c.fmt != STARKV_FMT_MIXED &&
      c.fmt != STARKV_FMT_HAD43)
    return fail(STARKV_ERR_INVALID_ARG, "unknown latent format");
  if (c.page_tokens != kPage) return fail(STARKV_ERR_UNSUPPORTED, "page_tokens must be 64");
  if (!(c.rope_theta > 1.0) || !std::isfinite(c.rope_theta))
    return fail(STARKV_ERR_INVALID_ARG, "rope_theta must be finite and > 1");

  starkv_layout L;
  std::memset(&L, 0, sizeof(L));
  // the shared fields; the joint-key ranks stay 0
  L.cfg.n_q_heads = c.n_q_heads;
  L.cfg.n_kv_heads = c.n_kv_heads;
  L.cfg.head_dim = c.head_dim;
  L.cfg.d_model = c.d_model;
  L.cfg.fmt = c.fmt;
  L.cfg.page_tokens = c.page_tokens;
  L.cfg.rope_theta = c.rope_theta;
  L.assignment = STARKV_ASSIGN_HYBRID;
  // the config itself, copied field by field (no padding bytes of the caller's struct)
  L.hybrid.n_q_heads = c.n_q_heads;
  L.hybrid.n_kv_heads = c.n_kv_heads;
  L.hybrid.head_dim = c.head_dim;
  L.hybrid.d_model = c.d_model;
  for (int g = 0; g < c.n_kv_heads; ++g) L.hybrid.key_rank[g] = c.key_rank[g];
  L.hybrid.value_rank = c.value_rank;
  L.hybrid.fmt = c.fmt;
  L.hybrid.page_tokens = c.page_tokens;
  L.hybrid.rope_theta = c.rope_theta;
  int ranks[1 + STARKV_MAX_KV_HEADS];
  for (int g = 0; g < c.n_kv_heads; ++g) ranks[g] = c.key_rank[g];
  ranks[c.n_kv_heads] = c.value_rank;
  const starkv_status st = place_latents(L, c.fmt, ranks, 1 + c.n_kv_heads);
  if (st != STARKV_OK) return st;
  L.value_rank_total = c.value_rank;
  L.value_rank_max = c.value_rank;
  *out = L;
  return STARKV_OK;
}

starkv_status starkv_alloc(const starkv_layout* lay, int64_t num_pages, int32_t batch,
                           int32_t max_pages, int32_t max_append_tokens, starkv_sizes* out) {
  starkv_status st = check_layout(lay);
  if (st != STARKV_OK) return st;
  if (!out) return fail(STARKV_ERR_INVALID_ARG, "out is NULL");
  if (num_pages < 0 || batch < 0 || max_pages < 1 || max_append_tokens < 0)
    return fail(STARKV_ERR_INVALID_ARG, "negative size or max_pages < 1");
  if (max_pages > (1 << 24)) return fail(STARKV_ERR_INVALID_ARG, "max_pages too large");
  if (static_cast<uint64_t>(num_pages) > SIZE_MAX / static_cast<uint64_t>(lay->page_bytes))
    return fail(STARKV_ERR_INVALID_ARG, "num_pages * page_bytes does not fit in size_t");
  out->cache_bytes = static_cast<size_t>(num_pages) * lay->page_bytes;
  out->rope_table_bytes = rope_bytes(lay, max_pages);
  st = decode_ws_bytes(lay, batch, max_pages, &out->decode_workspace_bytes);
  if (st != STARKV_OK) return st;
  size_t ws = 0;
  for (int m = 1; m <= ceil_div(max_append_tokens, 128); ++m) {
    const int n = std::min(max_append_tokens, 128 * m);
    const size_t w = proj_workspace(lay, n);
    if (w > ws) ws = w;
  }
  out->append_workspace_bytes = ws;
  return STARKV_OK;
}

starkv_status starkv_rope_init(const starkv_layout* lay, int32_t max_pages, void* table,
                               size_t table_bytes, starkv_stream_t stream) {
  starkv_status st = check_layout(lay);
  if (st != STARKV_OK) return st;
  if (!table) return fail(STARKV_ERR_INVALID_ARG, "table is NULL");
  if (max_pages < 1) return fail(STARKV_ERR_INVALID_ARG, "max_pages < 1");
  if (table_bytes < rope_bytes(lay, max_pages)) return fail(STARKV_ERR_WORKSPACE, "rope table too small");
  DevInfo info;
  st = current_device(info);
  if (st != STARKV_OK) return st;
  cudaError_t e = launch_rope_init(reinterpret_cast<float2*>(table), lay->cfg.head_dim / 2, kTile,
                                   rope_tiles_for(max_pages), lay->cfg.rope_theta,
                                   lay->cfg.head_dim, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "rope init launch");
  return STARKV_OK;
}

static starkv_status store_common(const starkv_layout* lay, int32_t n_tok, const int32_t* tok_seq,
                                  const int32_t* tok_pos, const int32_t* block_table,
                                  int32_t max_pages, int32_t batch, void* cache, int64_t num_pages,
                                  int32_t* dev_status, StoreParams& sp) {
  starkv_status st = check_layout(lay);
  if (st != STARKV_OK) return st;
  if (n_tok < 0 || max_pages < 1 || batch < 1 || num_pages < 1)
    return fail(STARKV_ERR_INVALID_ARG, "n_tok < 0, or batch/max_pages/num_pages < 1");
  if (n_tok > 0 && (!tok_seq || !tok_pos || !block_table || !cache || !dev_status))
    return fail(STARKV_ERR_INVALID_ARG, "NULL pointer argument");
  std::memset(&sp, 0, sizeof(sp));
  fill_store(sp, lay);
  // the store and read-back kernels number their warps (token x chunk, token x latent) in
  // 32-bit integers
  const int64_t warps = static_cast<int64_t>(n_tok) * std::max(sp.chunks_per_token, lay->n_latents);
  if (warps > (int64_t(1) << 31) - 256)
    return fail(STARKV_ERR_INVALID_ARG, "n_tok too large for one call; split the tokens");
  sp.cache = reinterpret_cast<uint8_t*>(cache);
  sp.num_pages = num_pages;
  sp.page_bytes = lay->page_bytes;
  sp.block_table = block_table;
  sp.max_pages = max_pages;
  sp.batch = batch;
  sp.tok_seq = tok_seq;
  sp.tok_pos = tok_pos;
  sp.n_tok = n_tok;
  sp.status = dev_status;
  return STARKV_OK;
}

starkv_status starkv_quant_pack(const starkv_layout* lay, const float* latents, int32_t n_tok,
                                const int32_t* tok_seq, const int32_t* tok_pos,
                                const int32_t* block_table, int32_t max_pages, int32_t batch,
                                void* cache, int64_t num_pages, int32_t* dev_status,
                                starkv_stream_t stream) {
  StoreParams sp;
  starkv_status st = store_common(lay, n_tok, tok_seq, tok_pos, block_table, max_pages, batch,
                                  cache, num_pages, dev_status, sp);
  if (st != STARKV_OK) return st;
  if (n_tok == 0) return STARKV_OK;
  if (!latents) return fail(STARKV_ERR_INVALID_ARG, "latents is NULL");
  DevInfo info;
  st = current_device(info);
  if (st != STARKV_OK) return st;
  sp.src = latents;
  sp.nsplit = 1;
  sp.split_stride = 0;
  cudaError_t e = launch_store(sp, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "store launch");
  return STARKV_OK;
}

starkv_status starkv_dequant(const starkv_layout* lay, const void* cache, int64_t num_pages,
                             const int32_t* tok_seq, const int32_t* tok_pos, int32_t n_tok,
                             const int32_t* block_table, int32_t max_pages, int32_t batch,
                             float* latents_out, int32_t* dev_status, starkv_stream_t stream) {
  StoreParams sp;
  starkv_status st = store_common(lay, n_tok, tok_seq, tok_pos, block_table, max_pages, batch,
                                  const_cast<void*>(cache), num_pages, dev_status, sp);
  if (st != STARKV_OK) return st;
  if (n_tok == 0) return STARKV_OK;
  if (!latents_out) return fail(STARKV_ERR_INVALID_ARG, "latents_out is NULL");
  DevInfo info;
  st = current_device(info);
  if (st != STARKV_OK) return st;
  sp.latents_out = latents_out;
  cudaError_t e = launch_dequant(sp, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "dequant launch");
  return STARKV_OK;
}

starkv_status starkv_append(const starkv_layout* lay, const void* x, int32_t n_tok, const void* A_t,
                            const int32_t* tok_seq, const int32_t* tok_pos,
                            const int32_t* block_table, int32_t max_pages, int32_t batch,
                            void* cache, int64_t num_pages, float* latents_out, void* workspace,
                            size_t workspace_bytes, int32_t* dev_status, starkv_stream_t stream) {
  StoreParams sp;
  starkv_status st = store_common(lay, n_tok, tok_seq, tok_pos, block_table, max_pages, batch,
                                  cache, num_pages, dev_status, sp);
  if (st != STARKV_OK) return st;
  if (n_tok == 0) return STARKV_OK;
  if (!x || !A_t || !workspace) return fail(STARKV_ERR_INVALID_ARG, "x/A_t/workspace is NULL");
  if (workspace_bytes < proj_workspace(lay, n_tok))
    return fail(STARKV_ERR_WORKSPACE, "append workspace too small for n_tok");
  if ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(A_t) |
       reinterpret_cast<uintptr_t>(workspace)) & 15)
    return fail(STARKV_ERR_INVALID_ARG, "x, A_t and workspace must be 16-byte aligned");
  DevInfo info;
  st = current_device(info);
  if (st != STARKV_OK) return st;
  const int fmt = lay->cfg.fmt;
  const int es = elem_size(fmt);
  // A decode step (at most 32 tokens, bf16 operands): one launch that projects on the tensor
  // cores and stores, with the k-split partials added in a cluster's shared memory.  The
  // k-slice is the smallest of d_model / {8, 4, 2, 1} that is a multiple of 64 columns and
  // keeps at least 256 (d_model itself when none does).
  if (fmt != STARKV_FMT_F32 && n_tok <= kGemvMaxTokens) {
    const int dm = lay->cfg.d_model;
    int ks = 8;
    while (ks > 1 && (dm % (64 * ks) != 0 || dm / ks < 256)) ks /= 2;
    if (append_gemv_smem(dm / ks, n_tok) <= info.smem_optin) {
      GemvParams gp;
      std::memset(&gp, 0, sizeof(gp));
      gp.sp = sp;
      gp.sp.latents_out = latents_out;
      gp.x = reinterpret_cast<const __nv_bfloat16*>(x);
      gp.A_t = reinterpret_cast<const __nv_bfloat16*>(A_t);
      gp.d_model = dm;
      gp.ks = ks;
      gp.kslice = dm / ks;
      gp.timeout_ns = 4000000000ull;
      cudaError_t e = launch_append_gemv(gp, reinterpret_cast<cudaStream_t>(stream));
      if (e != cudaSuccess) return cuda_fail(e, "decode-step append launch");
      return STARKV_OK;
    }
  }
  ProjParams pp;
  std::memset(&pp, 0, sizeof(pp));
  proj_plan(lay, n_tok, pp.kb_total, pp.kb_per_split, pp.nsplit);
  pp.part = reinterpret_cast<float*>(workspace);
  pp.n_tok = n_tok;
  pp.proj_cols = lay->proj_cols;
  pp.d_model = lay->cfg.d_model;
  pp.stages = fmt == STARKV_FMT_F32 ? 2 : 4;  // fp32: hi/lo copies double each stage
  pp.idesc = idesc_make(fmt == STARKV_FMT_F32 ? 2u : 1u, 128, 256);
  pp.status = dev_status;
  pp.timeout_ns = 4000000000ull;
  CUtensorMap tmX, tmA;
  const CUtensorMapDataType dt =
      fmt == STARKV_FMT_F32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const cuuint32_t ke = 128 / es;
  {
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(lay->cfg.d_model), static_cast<cuuint64_t>(n_tok)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(lay->cfg.d_model) * es};
    cuuint32_t box[2] = {ke, 128};
    st = encode(&tmX, dt, 2, x, dims, strides, box);
    if (st != STARKV_OK) return st;
  }
  {
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(lay->cfg.d_model), static_cast<cuuint64_t>(lay->proj_cols)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(lay->cfg.d_model) * es};
    cuuint32_t box[2] = {ke, 256};
    st = encode(&tmA, dt, 2, A_t, dims, strides, box);
    if (st != STARKV_OK) return st;
  }
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = launch_project(fmt, pp, tmX, tmA, s);
  if (e != cudaSuccess) return cuda_fail(e, "projection launch");
  sp.src = pp.part;
  sp.nsplit = pp.nsplit;
  sp.split_stride = static_cast<long long>(n_tok) * lay->proj_cols;
  sp.latents_out = latents_out;
  e = launch_store(sp, s);
  if (e != cudaSuccess) return cuda_fail(e, "store launch");
  return STARKV_OK;
}

// Launch shape of the split kernel for a layout, batch and block-table width on a device with
// `sms` SMs and `smem_optin` bytes of opt-in shared memory per block: CTA pairing, chunking,
// work units, the int8/int4 key-operand mode and the shared-memory plan.  Host only, pure:
// fills the shape fields of `p` (it zeroes `p` first) and the grid.
static starkv_status plan_shape(const starkv_layout* lay, int32_t batch, int32_t max_pages,
                                const starkv_decode_opts* opts, int sms, size_t smem_optin,
                                DecodeParams& p, int& grid) {
  const starkv_config& c = lay->cfg;
  std::memset(&p, 0, sizeof(p));
  const int fmt = c.fmt, es = elem_size(fmt), d = c.head_dim;
  const int tiles_max = tiles_for(max_pages);
  p.max_pages = max_pages;
  p.batch = batch;
  p.rope_tiles = rope_tiles_for(max_pages);
  p.tiles_max = tiles_max;
  p.rec = record_floats(lay);
  const int timeout_ms = (opts && opts->timeout_ms > 0) ? opts->timeout_ms : 4000;
  p.timeout_ns = static_cast<unsigned long long>(timeout_ms) * 1000000ull;
  p.H = c.n_q_heads;
  p.Hkv = c.n_kv_heads;
  p.G = c.n_q_heads / c.n_kv_heads;
  p.d = d;
  p.rk = c.key_rank;
  p.key_rank_cols = c.key_rank;
  const int ncols = c.n_kv_heads * d;
  // fp32 latents keep hi/lo copies of both operands in shared memory: 128-column chunks
  p.NC = ncols >= 256 ? (fmt == STARKV_FMT_F32 ? 128 : 256) : ncols;
  p.n_chunks = ceil_div(ncols, p.NC);
  if (p.n_chunks > kMaxChunks) return fail(STARKV_ERR_UNSUPPORTED, "more K column chunks than supported");
  p.kb_count = ceil_div(c.key_rank * es, kKBytes);
  // CTA pairs (one cluster per 256-token tile) for 16-bit operands and 256-column chunks
  const int want_cg = opts ? opts->cta_group : 0;
  if (want_cg < 0 || want_cg > 2) return fail(STARKV_ERR_INVALID_ARG, "cta_group must be 0, 1 or 2");
  const bool pair_ok = fmt != STARKV_FMT_F32 && p.NC == 256 && sms >= 2;
  if (want_cg == 2 && !pair_ok)
    return fail(STARKV_ERR_UNSUPPORTED, "CTA pairs need bf16 or int8/int4 latents and 256-column chunks");
  // the streamed int8/int4 operand (key rank > 256, dequantised per ring stage) ran slower on
  // pairs than on single CTAs (10.1 vs 12.0 ms at batch 16, context 16384, rank 1024): the
  // default keeps single-CTA tiles there
  const bool pair_default = pair_ok && !(quantised(fmt) && p.kb_count > 4);
  p.cta_group = want_cg == 2 ? 2 : (want_cg == 1 ? 1 : (pair_default ? 2 : 1));
  const int CG = p.cta_group;
  int grid_cap = sms;
  if (opts && opts->max_ctas > 0 && opts->max_ctas < grid_cap) grid_cap = opts->max_ctas;
  grid_cap = std::max(CG, grid_cap / CG * CG);
  const long long group_tiles = ceil_div(tiles_max, CG);
  int n_ranges = 1;
  if (opts && opts->n_ranges > 0) {
    n_ranges = std::min(opts->n_ranges, p.n_chunks);
  } else {
    while (n_ranges < p.n_chunks && batch * group_tiles * n_ranges < 4LL * (grid_cap / CG))
      n_ranges *= 2;
    n_ranges = std::min(n_ranges, p.n_chunks);
  }
  p.cpr = ceil_div(p.n_chunks, n_ranges);
  p.n_ranges = ceil_div(p.n_chunks, p.cpr);
  const long long units = group_tiles * batch * p.n_ranges;
  if (units > (1LL << 30)) return fail(STARKV_ERR_INVALID_ARG, "too many work units");
  p.total_units = static_cast<int>(units);
  p.idesc = idesc_make(fmt == STARKV_FMT_F32 ? 2u : (fmt == STARKV_FMT_BF16 ? 1u : 0u),
                       static_cast<uint32_t>(128 * CG), static_cast<uint32_t>(p.NC));
  p.qscale = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(d)));
  p.key = lat_desc(lay->seg[0]);
  int vmax = 0;
  const int heads_per_chunk = p.NC / d;
  for (int ch = 0; ch < p.n_chunks; ++ch) {
    const int g0 = ch * heads_per_chunk;
    const int g1 = std::min(c.n_kv_heads, g0 + heads_per_chunk);
    const starkv_segment& first = lay->seg[1 + g0];
    const starkv_segment& last = lay->seg[g1];
    int64_t start, end;
    if (quantised(fmt)) {
      start = first.off_i8;
      end = last.off_sc + static_cast<int64_t>(kPage) * 2 * (last.g8 + last.g4);
    } else {
      start = first.off_plain;
      end = last.off_plain + static_cast<int64_t>(kPage) * last.pitch;
    }
    end = align16(end);
    p.vchunk_off[ch] = static_cast<int>(start);
    p.vchunk_bytes[ch] = static_cast<int>(end - start);
    if (end - start > vmax) vmax = static_cast<int>(end - start);
  }
  for (int g = 0; g < c.n_kv_heads; ++g) p.vh[g] = lat_desc(lay->seg[1 + g]);

  // int8/int4 keys: of rank <= 256, the dequantised tile stays resident for all its chunks
  // (mode 1, codes double-buffered); above that, the tile's codes are staged in shared memory
  // once and the operand is streamed through the ring (mode 2, one code buffer) when they
  // fit, else the dequantisers read the codes from global memory (mode 0)
  int modes[2] = {0, 0};
  int n_modes = 1;
  if (quantised(fmt)) {
    if (p.kb_count <= 4) {
      modes[0] = 1;
    } else {
      modes[0] = 2;
      modes[1] = 0;
      n_modes = 2;
    }
  }
  int key_region = 0;
  {
    const starkv_segment& k = lay->seg[0];
    if (quantised(fmt))
      key_region = static_cast<int>(k.off_sc + int64_t(kPage) * 2 * (k.g8 + k.g4) - k.off_i8);
  }
  // shared-memory plan: ring stages of (A k-block, B k-block), value buffers, small arrays
  p.vslot = (vmax + 127) / 128 * 128;
  const size_t bstage = static_cast<size_t>(p.NC / CG) * kKBytes;
  const size_t limit = std::min<size_t>(decode_smem_limit(), smem_optin);
  bool planned = false;
  const int plans[][2] = {{6, 2}, {6, 1}, {5, 2}, {5, 1}, {4, 2}, {4, 1}, {3, 2}, {3, 1}, {2, 1}};
  for (int mi = 0; mi < n_modes && !planned; ++mi)
  for (const auto& pl : plans) {
    const int mode = modes[mi];
    const bool ares = mode == 1;
    const int ncb = mode == 1 ? 2 : (mode == 2 ? 1 : 0);  // code buffers
    size_t off = 0;
    const int S = pl[0], NVB = pl[1];
    const size_t split = fmt == STARKV_FMT_F32 ? 2 : 1;  // hi/lo copies for 3xTF32
    off += (ares ? p.kb_count : S) * split * static_cast<size_t>(kAStage);
    const size_t off_b = off;
    off += S * split * bstage;
    const size_t off_codes = off;
    off += static_cast<size_t>(ncb) * 2 * static_cast<size_t>(key_region);
    const size_t off_v = off;
    off += static_cast<size_t>(NVB) * 2 * p.vslot;
    const size_t QPC = static_cast<size_t>(256 / d) * p.G;  // query heads of a full chunk
    const size_t off_q = off;
    off += QPC * d * 4;
    const size_t off_p = off;
    off += QPC * kTile * 4;
    const size_t off_part = off;
    off += 2 * QPC * kTile * 4;
    const size_t off_red = off;
    off += 2 * 2 * QPC * 4 * 4;
    off = (off + 15) / 16 * 16;
    const size_t off_ang = off;
    off += 2 * static_cast<size_t>(d / 2) * 4;
    const size_t off_pv = off;
    off += 2 * static_cast<size_t>(p.G) * kTile * 4;
    off = (off + 7) / 8 * 8;
    const size_t off_bar = off;
    off += (3 * S + 4 + 2 * NVB + 1 + 12) * 8 + 16;
    // alignment slack of the dynamic base; at least 120 KB so that one CTA occupies an SM
    // (each CTA allocates all 512 TMEM columns)
    const size_t total = std::max<size_t>(off + 1024, 120 * 1024);
    if (total <= limit) {
      p.a_resident = mode;
      p.key_region = mode ? key_region : 0;
      p.stages = S;
      p.nvb = NVB;
      p.off_b = static_cast<uint32_t>(off_b);
      p.off_codes = static_cast<uint32_t>(off_codes);
      p.off_v = static_cast<uint32_t>(off_v);
      p.off_q = static_cast<uint32_t>(off_q);
      p.off_p = static_cast<uint32_t>(off_p);
      p.off_part = static_cast<uint32_t>(off_part);
      p.off_red = static_cast<uint32_t>(off_red);
      p.off_ang = static_cast<uint32_t>(off_ang);
      p.off_pv = static_cast<uint32_t>(off_pv);
      p.off_bar = static_cast<uint32_t>(off_bar);
      p.smem_bytes = static_cast<uint32_t>(total);
      planned = true;
      break;
    }
  }
  if (!planned) return fail(STARKV_ERR_UNSUPPORTED, "value latents of one chunk do not fit in shared memory");

  grid = static_cast<int>(std::min<long long>(units * CG, grid_cap));
  return STARKV_OK;
}

static starkv_status plan_decode(const starkv_layout* lay, const void* q, const void* cache,
                                 int64_t num_pages, const int32_t* block_table, int32_t max_pages,
                                 const int32_t* seq_lens, int32_t batch, const void* Bk_t,
                                 const float* Bv, const void* rope_table, size_t rope_table_bytes,
                                 float* out, void* workspace, size_t workspace_bytes,
                                 const starkv_decode_opts* opts, int32_t* dev_status, bool split,
                                 bool combine, DecodeParams& p, CUtensorMap& tmA, CUtensorMap& tmB,
                                 int& grid) {
  starkv_status st = check_layout(lay);
  if (st != STARKV_OK) return st;
  st = check_decode_format(lay);
  if (st != STARKV_OK) return st;
  if (batch < 0 || max_pages < 1 || (split && num_pages < 1))
    return fail(STARKV_ERR_INVALID_ARG, "batch < 0, or max_pages/num_pages < 1");
  if (batch == 0) return STARKV_OK;
  if (!seq_lens || !workspace) return fail(STARKV_ERR_INVALID_ARG, "NULL pointer argument");
  if (split && (!q || !cache || !block_table || !Bk_t || !rope_table || !dev_status))
    return fail(STARKV_ERR_INVALID_ARG, "NULL pointer argument");
  if (combine && (!Bv || !out)) return fail(STARKV_ERR_INVALID_ARG, "NULL pointer argument");
  if (split && ((reinterpret_cast<uintptr_t>(cache) | reinterpret_cast<uintptr_t>(Bk_t) |
                 reinterpret_cast<uintptr_t>(rope_table)) & 15))
    return fail(STARKV_ERR_INVALID_ARG, "cache, Bk_t and rope_table must be 16-byte aligned");
  if (reinterpret_cast<uintptr_t>(workspace) & 15)
    return fail(STARKV_ERR_INVALID_ARG, "workspace must be 16-byte aligned");
  if (max_pages > (1 << 24)) return fail(STARKV_ERR_INVALID_ARG, "max_pages too large");
  if (split && rope_table_bytes < rope_bytes(lay, max_pages))
    return fail(STARKV_ERR_WORKSPACE, "rope table smaller than needed for max_pages");
  const starkv_config& c = lay->cfg;
  size_t ws_need = 0;
  st = decode_ws_bytes(lay, batch, max_pages, &ws_need);
  if (st != STARKV_OK) return st;
  if (workspace_bytes < ws_need) return fail(STARKV_ERR_WORKSPACE, "decode workspace too small");
  DevInfo info;
  st = current_device(info);
  if (st != STARKV_OK) return st;
  st = plan_shape(lay, batch, max_pages, opts, info.sms, info.smem_optin, p, grid);
  if (st != STARKV_OK) return st;
  const int fmt = c.fmt, es = elem_size(fmt), CG = p.cta_group;
  const int ncols = c.n_kv_heads * c.head_dim;
  p.cache = reinterpret_cast<const uint8_t*>(cache);
  p.num_pages = num_pages;
  p.page_bytes = lay->page_bytes;
  p.block_table = block_table;
  p.seq_lens = seq_lens;
  p.q = q;
  p.Bv = Bv;
  p.rope = reinterpret_cast<const float2*>(rope_table);
  p.ws = reinterpret_cast<float*>(workspace);
  p.out = out;
  p.status = dev_status;
  std::memset(&tmA, 0, sizeof(tmA));
  std::memset(&tmB, 0, sizeof(tmB));
  if (!split) return STARKV_OK;
  const cuuint32_t ke = static_cast<cuuint32_t>(kKBytes / es);
  if (!quantised(fmt)) {
    const CUtensorMapDataType dt =
        fmt == STARKV_FMT_F32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(c.key_rank), static_cast<cuuint64_t>(kPage),
                          static_cast<cuuint64_t>(num_pages)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(c.key_rank) * es,
                             static_cast<cuuint64_t>(lay->page_bytes)};
    cuuint32_t box[3] = {ke, static_cast<cuuint32_t>(kPage), 1};
    st = encode(&tmA, dt, 3, reinterpret_cast<const uint8_t*>(cache) + lay->seg[0].off_plain, dims,
                strides, box);
    if (st != STARKV_OK) return st;
  }
  {
    const CUtensorMapDataType dt = fmt == STARKV_FMT_F32    ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                                   : fmt == STARKV_FMT_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                                            : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(c.key_rank), static_cast<cuuint64_t>(ncols)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(c.key_rank) * es};
    cuuint32_t box[2] = {ke, static_cast<cuuint32_t>(p.NC / CG)};
    st = encode(&tmB, dt, 2, Bk_t, dims, strides, box);
    if (st != STARKV_OK) return st;
  }
  return STARKV_OK;
}

starkv_status starkv_decode_plan_query(const starkv_layout* lay, int32_t batch, int32_t max_pages,
                                       const starkv_decode_opts* opts, int32_t num_sms,
                                       int64_t smem_per_block, starkv_decode_plan* out) {
  starkv_status st = check_layout(lay);
  if (st != STARKV_OK) return st;
  st = check_decode_format(lay);
  if (st != STARKV_OK) return st;
  if (!out) return fail(STARKV_ERR_INVALID_ARG, "out is NULL");
  if (batch < 1 || max_pages < 1 || max_pages > (1 << 24) || num_sms < 1 || smem_per_block < 0)
    return fail(STARKV_ERR_INVALID_ARG, "batch, max_pages and num_sms must be >= 1");
  DecodeParams p;
  int grid = 0;
  st = plan_shape(lay, batch, max_pages, opts, num_sms, static_cast<size_t>(smem_per_block), p, grid);
  if (st != STARKV_OK) return st;
  std::memset(out, 0, sizeof(*out));
  out->cta_group = p.cta_group;
  out->key_mode = p.a_resident;
  out->chunk_cols = p.NC;
  out->n_chunks = p.n_chunks;
  out->n_ranges = p.n_ranges;
  out->stages = p.stages;
  out->value_buffers = p.nvb;
  out->smem_bytes = static_cast<int32_t>(p.smem_bytes);
  out->grid = grid;
  out->work_units = p.total_units;
  return STARKV_OK;
}

starkv_status starkv_decode_partials(const starkv_layout* lay, const void* q, const void* cache,
                                     int64_t num_pages, const int32_t* block_table,
                                     int32_t max_pages, const int32_t* seq_lens, int32_t batch,
                                     const void* Bk_t, const void* rope_table,
                                     size_t rope_table_bytes, void* workspace,
                                     size_t workspace_bytes, const starkv_decode_opts* opts,
                                     int32_t* dev_status, starkv_stream_t stream) {
  DecodeParams p;
  CUtensorMap tmA, tmB;
  int grid = 0;
  starkv_status st = plan_decode(lay, q, cache, num_pages, block_table, max_pages, seq_lens, batch,
                                 Bk_t, nullptr, rope_table, rope_table_bytes, nullptr, workspace,
                                 workspace_bytes, opts, dev_status, true, false, p, tmA, tmB, grid);
  if (st != STARKV_OK || batch == 0) return st;
  cudaError_t e = launch_decode(lay->cfg.fmt, lay->cfg.head_dim, p.G, p, tmA, tmB, grid,
                                reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "decode split launch");
  return STARKV_OK;
}

starkv_status starkv_decode_combine(const starkv_layout* lay, const int32_t* seq_lens,
                                    int32_t batch, int32_t max_pages, const float* Bv,
                                    const void* workspace, size_t workspace_bytes, float* out,
                                    starkv_stream_t stream) {
  DecodeParams p;
  CUtensorMap tmA, tmB;
  int grid = 0;
  starkv_status st = plan_decode(lay, nullptr, nullptr, 0, nullptr, max_pages, seq_lens, batch,
                                 nullptr, Bv, nullptr, 0, out, const_cast<void*>(workspace),
                                 workspace_bytes, nullptr, nullptr, false, true, p, tmA, tmB, grid);
  if (st != STARKV_OK || batch == 0) return st;
  cudaError_t e = launch_combine(p, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "decode combine launch");
  return STARKV_OK;
}

starkv_status starkv_decode_attention(const starkv_layout* lay, const void* q, const void* cache,
                                      int64_t num_pages, const int32_t* block_table,
                                      int32_t max_pages, const int32_t* seq_lens, int32_t batch,
                                      const void* Bk_t, const float* Bv, const void* rope_table,
                                      size_t rope_table_bytes, float* out, void* workspace,
                                      size_t workspace_bytes, const starkv_decode_opts* opts,
                                      int32_t* dev_status, starkv_stream_t stream) {
  DecodeParams p;
  CUtensorMap tmA, tmB;
  int grid = 0;
  starkv_status st = plan_decode(lay, q, cache, num_pages, block_table, max_pages, seq_lens, batch,
                                 Bk_t, Bv, rope_table, rope_table_bytes, out, workspace,
                                 workspace_bytes, opts, dev_status, true, true, p, tmA, tmB, grid);
  if (st != STARKV_OK || batch == 0) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = launch_decode(lay->cfg.fmt, lay->cfg.head_dim, p.G, p, tmA, tmB, grid, s);
  if (e != cudaSuccess) return cuda_fail(e, "decode split launch");
  e = launch_combine(p, s);
  if (e != cudaSuccess) return cuda_fail(e, "decode combine launch");
  return STARKV_OK;
}

// ---------------------------------------------------------------- weight absorption
static void fill_absorb(const starkv_layout* lay, int32_t d_out, int32_t batch, AbsorbParams& a) {
  std::memset(&a, 0, sizeof(a));
  const starkv_config& c = lay->cfg;
  a.H = c.n_q_heads;
  a.G = c.n_q_heads / c.n_kv_heads;
  a.d = c.head_dim;
  a.d_out = d_out;
  a.key_rank_cols = c.key_rank;
  int rv = 0;
  for (int g = 0; g < c.n_kv_heads; ++g) {
    a.vh[g] = lat_desc(lay->seg[1 + g]);
    rv += lay->seg[1 + g].rank;
  }
  a.m_rows = a.G * rv;
  // splits of M's rows (32 rows at least): with the column tiles and the 8-sequence groups,
  // enough CTAs for the HBM stream of M
  a.ksplit = std::max(1, std::min(32, a.m_rows / 32));
  a.krows = ceil_div(a.m_rows, a.ksplit);
  a.ksplit = ceil_div(a.m_rows, a.krows);
}

starkv_status starkv_absorbed_sizes(const starkv_layout* lay, int32_t batch, int32_t d_out,
                                    int64_t* m_rows, size_t* scratch_bytes) {
  starkv_status st = check_layout(lay);
  if (st != STARKV_OK) return st;
  st = check_decode_format(lay);
  if (st != STARKV_OK) return st;
  if (batch < 0 || d_out < 1 || d_out > (1 << 20))
    return fail(STARKV_ERR_INVALID_ARG, "batch < 0 or d_out outside [1, 2^20]");
  if (!m_rows || !scratch_bytes) return fail(STARKV_ERR_INVALID_ARG, "NULL output pointer");
  AbsorbParams a;
  fill_absorb(lay, d_out, batch, a);
  *m_rows = a.m_rows;
  const size_t rows_a = static_cast<size_t>(batch) * a.m_rows;
  *scratch_bytes = (rows_a + 63) / 64 * 64 * sizeof(float) +
                   static_cast<size_t>(a.ksplit) * batch * d_out * sizeof(float);
  return STARKV_OK;
}

starkv_status starkv_absorb_output_weights(const starkv_layout* lay, const float* Bv,
                                           const float* Wo, int32_t d_out, float* M,
                                           starkv_stream_t stream) {
  starkv_status st = check_layout(lay);
  if (st != STARKV_OK) return st;
  st = check_decode_format(lay);
  if (st != STARKV_OK) return st;
  if (d_out < 1 || d_out > (1 << 20)) return fail(STARKV_ERR_INVALID_ARG, "d_out outside [1, 2^20]");
  if (!Bv || !Wo || !M) return fail(STARKV_ERR_INVALID_ARG, "NULL pointer argument");
  DevInfo info;
  st = current_device(info);
  if (st != STARKV_OK) return st;
  AbsorbParams a;
  fill_absorb(lay, d_out, 1, a);
  a.Bv = Bv;
  a.Wo = Wo;
  a.M = M;
  cudaError_t e = launch_absorb_weights(a, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "weight absorption launch");
  return STARKV_OK;
}

starkv_status starkv_decode_combine_absorbed(const starkv_layout* lay, const int32_t* seq_lens,
                                             int32_t batch, int32_t max_pages, const float* M,
                                             int32_t d_out, const void* workspace,
                                             size_t workspace_bytes, void* scratch,
                                             size_t scratch_bytes, float* out,
                                             starkv_stream_t stream) {
  int64_t m_rows = 0;
  size_t need = 0;
  starkv_status st = starkv_absorbed_sizes(lay, batch, d_out, &m_rows, &need);
  if (st != STARKV_OK) return st;
  if (batch == 0) return STARKV_OK;
  if (!M || !scratch || !out) return fail(STARKV_ERR_INVALID_ARG, "NULL pointer argument");
  if (scratch_bytes < need) return fail(STARKV_ERR_WORKSPACE, "absorbed-output scratch too small");
  if (reinterpret_cast<uintptr_t>(scratch) & 15)
    return fail(STARKV_ERR_INVALID_ARG, "scratch must be 16-byte aligned");
  DecodeParams p;
  CUtensorMap tmA, tmB;
  int grid = 0;
  // the merge of the partial records: the combine without its up-projection (M stands in
  // for B_v in the argument checks and is not read by it)
  st = plan_decode(lay, nullptr, nullptr, 0, nullptr, max_pages, seq_lens, batch, nullptr, M,
                   nullptr, 0, out, const_cast<void*>(workspace), workspace_bytes, nullptr,
                   nullptr, false, true, p, tmA, tmB, grid);
  if (st != STARKV_OK) return st;
  float* A = reinterpret_cast<float*>(scratch);
  p.a_out = A;
  p.a_stride = static_cast<int>(m_rows);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = launch_combine(p, s);
  if (e != cudaSuccess) return cuda_fail(e, "decode merge launch");
  AbsorbParams a;
  fill_absorb(lay, d_out, batch, a);
  a.M = const_cast<float*>(M);  // read only by the product kernels
  a.A = A;
  a.part = A + (static_cast<size_t>(batch) * m_rows + 63) / 64 * 64;
  a.y = out;
  a.batch = batch;
  e = launch_absorbed_output(a, s);
  if (e != cudaSuccess) return cuda_fail(e, "absorbed output launch");
  return STARKV_OK;
}

starkv_status starkv_hybrid_decode(const starkv_layout* lay, const void* q, const void* cache,
                                   int64_t num_pages, const int32_t* block_table, int32_t max_pages,
                                   const int32_t* seq_lens, int32_t batch, const void* Bk_t,
                                   const float* Bv, const void* rope_table, size_t rope_table_bytes,
                                   float* out, void* workspace, size_t workspace_bytes,
                                   int32_t* dev_status, starkv_stream_t stream) {
  starkv_status st = check_layout(lay);
  if (st != STARKV_OK) return st;
  if (lay->assignment != STARKV_ASSIGN_HYBRID)
    return fail(STARKV_ERR_INVALID_ARG, "starkv_hybrid_decode takes a layout of starkv_hybrid_layout_init");
  const starkv_config& c = lay->cfg;
  if (c.fmt != STARKV_FMT_MIXED)
    return fail(STARKV_ERR_UNSUPPORTED, "the hybrid decode kernel takes the int8/int4 format");
  if (c.n_kv_heads > kHybMaxKv) return fail(STARKV_ERR_UNSUPPORTED, "hybrid decode: n_kv_heads > 16");
  const int H = c.n_q_heads, rv = lay->value_rank_total;
  const int hp = (H + 15) / 16 * 16, rvp = (rv + 63) / 64 * 64;
  if (hp / 16 > 4 || (hp / 16) * (rvp / 64) > 8)
    return fail(STARKV_ERR_UNSUPPORTED, "hybrid decode: ceil(H/16) * ceil(r_v/64) above 8, or H > 64");
  if (lay->page_bytes >= (int64_t(1) << 20))
    return fail(STARKV_ERR_UNSUPPORTED, "hybrid decode: a page of 1 MiB or more");
  if (batch < 0 || max_pages < 1 || num_pages < 1)
    return fail(STARKV_ERR_INVALID_ARG, "batch < 0, or max_pages/num_pages < 1");
  if (max_pages > (1 << 24)) return fail(STARKV_ERR_INVALID_ARG, "max_pages too large");
  if (batch == 0) return STARKV_OK;
  if (!q || !cache || !block_table || !seq_lens || !Bk_t || !Bv || !rope_table || !out ||
      !workspace || !dev_status)
    return fail(STARKV_ERR_INVALID_ARG, "NULL pointer argument");
  if ((reinterpret_cast<uintptr_t>(cache) | reinterpret_cast<uintptr_t>(Bk_t) |
       reinterpret_cast<uintptr_t>(workspace)) & 15)
    return fail(STARKV_ERR_INVALID_ARG, "cache, Bk_t and workspace must be 16-byte aligned");
  if (rope_table_bytes < rope_bytes(lay, max_pages))
    return fail(STARKV_ERR_WORKSPACE, "rope table smaller than needed for max_pages");
  size_t ws_need = 0;
  st = decode_ws_bytes(lay, batch, max_pages, &ws_need);
  if (st != STARKV_OK) return st;
  if (workspace_bytes < ws_need) return fail(STARKV_ERR_WORKSPACE, "decode workspace too small");
  DevInfo info;
  st = current_device(info);
  if (st != STARKV_OK) return st;
  HybridParams p;
  std::memset(&p, 0, sizeof(p));
  p.q = reinterpret_cast<const __nv_bfloat16*>(q);
  p.cache = reinterpret_cast<const uint8_t*>(cache);
  p.num_pages = num_pages;
  p.page_bytes = static_cast<int>(lay->page_bytes);
  p.block_table = block_table;
  p.max_pages = max_pages;
  p.seq_lens = seq_lens;
  p.batch = batch;
  p.Bk_t = reinterpret_cast<const __half*>(Bk_t);
  p.Bv = Bv;
  p.rope = reinterpret_cast<const float2*>(rope_table);
  p.out = out;
  p.ws = reinterpret_cast<float*>(workspace);
  p.status = dev_status;
  p.H = H;
  p.Hkv = c.n_kv_heads;
  p.G = H / c.n_kv_heads;
  p.d = c.head_dim;
  p.rv = rv;
  p.rvp = rvp;
  p.rec = hybrid_rec(lay);
  hybrid_splits(batch, max_pages, p.nsplit, p.pps);
  p.units = batch * p.nsplit;
  p.hp = hp;
  p.mt_pv = hp / 16;
  p.qscale = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(c.head_dim)));
  p.timeout_ns = 4000000000ull;
  int64_t elem = 0;
  for (int g = 0; g < c.n_kv_heads; ++g) {
    p.key[g] = lat_desc(lay->seg[g]);
    p.bk_elem[g] = static_cast<int>(elem);
    elem += static_cast<int64_t>(c.head_dim) * lay->seg[g].rank;
  }
  p.val = lat_desc(lay->seg[c.n_kv_heads]);
  {
    int nq = rvp / 4;
    for (int g = 0; g < c.n_kv_heads; ++g) nq += lay->seg[g].rank / 4;
    p.nquad = (nq + 31) / 32 * 32;  // whole rounds of eight quads for each of four threads
  }
  if (!hybrid_plan(p, info.smem_optin))
    return fail(STARKV_ERR_UNSUPPORTED, "hybrid decode: the shared-memory plan exceeds the device's limit");
  const int grid = std::min(p.units, info.sms);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = launch_hybrid_split(p, grid, s);
  if (e != cudaSuccess) return cuda_fail(e, "hybrid split launch");
  e = launch_hybrid_combine(p, s);
  if (e != cudaSuccess) return cuda_fail(e, "hybrid combine launch");
  return STARKV_OK;
}

starkv_status starkv_diag_bounded_wait(int32_t timeout_ms, int32_t* dev_status,
                                      starkv_stream_t stream) {
  if (timeout_ms < 1 || timeout_ms > 10000)
    return fail(STARKV_ERR_INVALID_ARG, "timeout_ms must be in [1, 10000]");
  if (!dev_status) return fail(STARKV_ERR_INVALID_ARG, "dev_status is NULL");
  DevInfo info;
  starkv_status st = current_device(info);
  if (st != STARKV_OK) return st;
  cudaError_t e = launch_bounded_wait(dev_status, static_cast<unsigned long long>(timeout_ms) * 1000000ull,
                                      reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "bounded-wait diagnostic launch");
  return STARKV_OK;
}

}  // extern "C"
