// Device-side parameter blocks and launch entry points shared by the kernels and the C ABI.
#pragma once
#include <string>
#include <utility>

#include "ptx.cuh"

namespace starkv {

constexpr int kTile = STARKV_TILE_TOKENS;  // tokens per decode tile
constexpr int kPage = 64;                  // tokens per page
constexpr int kKBytes = 128;               // bytes of K per operand row per k-block
constexpr int kAStage = kTile * kKBytes;   // 16 KB: one k-block of a 128-row tile
constexpr int kMaxChunks = 32;             // ceil(64 heads * 128 / 256)

// One latent's description for device code (offsets inside a page; page_bytes < 2^31).
struct LatDesc {
  int rank;  // channels
  int col;   // first column in the concatenated projection
  int n8, nb4, g8, ng;  // mixed split; ng = g8 + g4
  int off0;  // plain block (f32/bf16) or int8 block (mixed)
  int off1;  // packed int4 block (mixed)
  int off2;  // fp16 scale block (mixed)
  int pitch; // plain: bytes per token
};

// Latent store / read-back (quant_pack, append epilogue, dequant).
struct StoreParams {
  const float* src;        // [nsplit][n_tok][proj_cols] fp32 (summed in split order)
  long long split_stride;  // floats between splits
  int nsplit;
  float* latents_out;      // optional [n_tok][proj_cols]
  uint8_t* cache;
  long long num_pages, page_bytes;
  const int* block_table;
  int max_pages, batch;
  const int* tok_seq;
  const int* tok_pos;
  int n_tok;
  int fmt, n_lat, proj_cols;
  int* status;
  int chunks_per_token;  // sum over latents of their 32-channel chunks (one warp each)
  LatDesc lat[1 + STARKV_MAX_KV_HEADS];
  short chunk_start[2 + STARKV_MAX_KV_HEADS];  // first chunk index of each latent
};

struct DecodeParams {
  const uint8_t* cache;
  long long num_pages, page_bytes;
  const int* block_table;
  int max_pages;
  const int* seq_lens;
  int batch;
  const void* q;      // [batch][H][d] bf16 or f32
  const float* Bv;    // [R_v][d]
  const float2* rope; // fine [128][d/2] then base [rope_tiles][d/2]
  int rope_tiles;
  float* ws;          // partial records
  int tiles_max, rec; // tiles per sequence slot, floats per record
  float* out;         // [batch][H][d]
  float* a_out;       // when set, the combine writes the normalised latent outputs a_h here
  int a_stride;       // floats per sequence row of a_out (rows of all query heads)
  int* status;
  unsigned long long timeout_ns;
  int H, Hkv, G, d, rk, key_rank_cols;
  int NC, n_chunks, n_ranges, cpr, kb_count, total_units;
  int cta_group;  // 1: one CTA per 128-token tile; 2: a CTA pair per 256-token tile
  int a_resident;  // int8/int4 keys: 1 = operand resident per tile, 2 = codes staged per tile, 0 = neither
  int key_region;  // bytes of the key blocks of one page (int8 | int4 | scales)
  uint32_t idesc;
  float qscale;  // log2(e) / sqrt(d)
  // dynamic shared-memory plan (offsets from the 1024-aligned base)
  int stages, nvb, vslot;
  uint32_t off_b, off_codes, off_v, off_q, off_p, off_part, off_red, off_ang, off_pv, off_bar, smem_bytes;
  LatDesc key;
  int vchunk_off[kMaxChunks];
  int vchunk_bytes[kMaxChunks];
  LatDesc vh[STARKV_MAX_KV_HEADS];
};

// Sets the message starkv_last_error() returns on this thread (defined with the C ABI).
void set_error_message(const std::string& msg);

// Launchers (defined in the .cu files; return cudaError_t of the launch).
// Launch with programmatic stream serialization: the kernel may be scheduled while the one
// before it on the stream finishes; it calls pdl_wait() before touching global memory.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t s, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

cudaError_t launch_store(const StoreParams& p, cudaStream_t s);

// Fused latent write of a decode step (at most 32 tokens, bf16 operands): projection on the
// tensor cores and the store in one launch, one cluster of ks CTAs (k-slices) per 32-channel
// chunk.
struct GemvParams {
  StoreParams sp;              // the store (latents, chunks, tokens, pages, status)
  const __nv_bfloat16* x;      // [n_tok][d_model]
  const __nv_bfloat16* A_t;    // [proj_cols][d_model]
  int d_model, kslice, ks;     // d_model = ks * kslice, kslice a multiple of 16
  int row_bytes;               // set by the launcher
  unsigned long long timeout_ns;
};
constexpr int kGemvMaxTokens = 32;
size_t append_gemv_smem(int kslice, int n_tok);
cudaError_t launch_append_gemv(const GemvParams& p, cudaStream_t s);

// Decode with the hybrid assignment (keys head-wise, values joint).
constexpr int kHybMaxKv = 16;       // KV heads the hybrid decode kernel takes
constexpr int kHybUnitsTarget = 1184;  // (sequence, page range) units aimed at: 8 per SM of 148
struct HybridParams {
  const __nv_bfloat16* q;   // [batch][H][d]
  const uint8_t* cache;
  long long num_pages;
  int page_bytes;
  const int* block_table;   // [batch][max_pages]
  int max_pages;
  const int* seq_lens;
  int batch;
  const __half* Bk_t;       // KV head g: [d][r_k,g] at element bk_elem[g]
  const float* Bv;          // [r_v][H_kv d]
  const float2* rope;       // fine [128][d/2] then base [rope_tiles][d/2]
  float* out;               // [batch][H][d]
  float* ws;                // records [batch][nsplit][H][rec]: m (log2 units), l, a[r_v]
  int* status;
  int H, Hkv, G, d;
  int rv, rvp, rec;         // joint value rank, padded to a multiple of 64, floats per record
  int nsplit, pps, units;   // page ranges per sequence, pages per range, batch * nsplit
  int hp, mt_pv;            // H padded to 16, its 16-row tiles
  int nquad;                // entries of the quad table: the latents' 4-channel groups, padded
  float qscale;             // log2(e) / sqrt(d)
  unsigned long long timeout_ns;
  LatDesc key[kHybMaxKv];
  LatDesc val;
  int bk_elem[kHybMaxKv];
  // shared-memory plan (byte offsets), set by hybrid_plan
  int s_bk[kHybMaxKv], s_ck[kHybMaxKv];
  int s_cv, s_qhi, s_qlo, s_s, s_p, s_stat, s_qtab, s_page, s_bar, smem_bytes;
};
// Fills the shared-memory plan of ``p`` (H, Hkv, d, ranks, rvp, page_bytes set); false when
// it exceeds ``smem_limit``.
bool hybrid_plan(HybridParams& p, size_t smem_limit);
cudaError_t launch_hybrid_split(const HybridParams& p, int grid, cudaStream_t s);
cudaError_t launch_hybrid_combine(const HybridParams& p, cudaStream_t s);

// Weight absorption (attention output projection folded into the value up-projection).
struct AbsorbParams {
  const float* Bv;  // [R_v][d]
  const float* Wo;  // [H * d][d_out]
  float* M;         // [m_rows][d_out]: rows of query head h at row_start(h)
  const float* A;   // [batch][m_rows] latent outputs a_h (normalised)
  float* part;      // [ksplit][batch][d_out]
  float* y;         // [batch][d_out]
  int H, G, d, d_out, m_rows, batch, ksplit, krows, key_rank_cols;
  LatDesc vh[STARKV_MAX_KV_HEADS];
};
cudaError_t launch_absorb_weights(const AbsorbParams& p, cudaStream_t s);
cudaError_t launch_absorbed_output(const AbsorbParams& p, cudaStream_t s);
cudaError_t launch_dequant(const StoreParams& p, cudaStream_t s);
cudaError_t launch_rope_init(float2* table, int half_dim, int rows_fine, int tiles, double theta,
                             int head_dim, cudaStream_t s);
cudaError_t launch_decode(int fmt, int head_dim, int G, const DecodeParams& p,
                          const CUtensorMap& tmA, const CUtensorMap& tmB, int grid,
                          cudaStream_t s);
cudaError_t launch_combine(const DecodeParams& p, cudaStream_t s);
cudaError_t launch_bounded_wait(int* status, unsigned long long timeout_ns, cudaStream_t s);
size_t decode_smem_limit();

struct ProjParams {
  float* part;       // [nsplit][n_tok][proj_cols]
  int n_tok, proj_cols, d_model;
  int kb_total, kb_per_split, nsplit;
  int stages;
  uint32_t idesc;
  int* status;
  unsigned long long timeout_ns;
};
cudaError_t launch_project(int fmt, const ProjParams& p, const CUtensorMap& tmX,
                           const CUtensorMap& tmA, cudaStream_t s);

}  // namespace starkv
