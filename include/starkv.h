/*
 * starkv.h -- C ABI of a B200 (sm_100a) library for STAR-KV-style low-rank, quantised
 * KV-cache decode.
 *
 * What the library computes (citations are page title + section):
 *   Latent write ("append"), after "STAR-KV: Low-Rank KV Cache Compression via Soft
 *   Thresholding for Adaptive Rank Control" (abstract: low-rank projection of the KV cache)
 *   and its technical summary, Methodology §2 "Hybrid Decomposition Strategy":
 *       c_k = x A_k            one joint (JD) key latent per token, rank r_k
 *       c_v,g = x A_v,g        one head-wise (HD) value latent per KV head g, rank r_g
 *   then storage of the latents in a paged cache, either as fp32, bf16, or quantised with
 *   the int8/int4 mixed format (same summary, Methodology §3 "Low-Rank-Aware
 *   Mixed-Precision Quantization": leading singular-value channels are the outliers and
 *   get more bits).  The concrete format -- first ceil(r/4) channels int8, the rest int4,
 *   one fp16 scale per token per group of 32 channels, two int4 per byte -- is this
 *   library's reading of the stated workload; the pages print no bit layout.
 *   Decode attention straight from the cache (summary, "Problem Statement": the
 *   reconstruction overhead at inference; Methodology §2: JD costs h x more to reconstruct):
 *       K = C_k B_k, RoPE(K) per KV head, softmax(q' K'^T / sqrt(d)) per query head,
 *       a_h = p C_v,g(h), o_h = a_h B_v,g(h).
 *   Optionally with the value up-projection folded into the output projection
 *   (Methodology §2): y = sum_h a_h (B_v,g(h) W_o,h).
 *   And with the pages' own assignment (Methodology §2, "Hybrid Decomposition Strategy"):
 *   keys head-wise (c_k,g = x A_k,g per KV head), values joint (one c_v = x A_v), decoded by
 *   starkv_hybrid_decode.
 *
 * Conventions shared by every entry point:
 *   - The caller owns all memory.  The library never allocates device memory, never
 *     synchronises and never frees.  Pointers marked "device" must be device pointers of
 *     the current device; pointers marked "host" are read before the call returns.
 *   - Every call is asynchronous on ``stream`` (a cudaStream_t; NULL = legacy default).
 *     The kernels of append, decode and combine are launched with programmatic stream
 *     serialisation: each may start its setup while the kernel before it on the stream
 *     finishes, and waits for that kernel to complete before it touches global memory.
 *   - The return value reports argument validation and launch errors only.  Errors found
 *     on the device are OR-ed into ``*dev_status`` (device int32, zeroed by the caller),
 *     as STARKV_DEV_* bits, read by the caller after a synchronisation.
 *   - No C++ exception crosses this interface.  On a non-OK return, starkv_last_error()
 *     gives a one-line message (thread-local, valid until the next call on that thread).
 */
#ifndef STARKV_H
#define STARKV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* starkv_stream_t; /* identical to cudaStream_t */

#if defined(__GNUC__)
#define STARKV_API __attribute__((visibility("default")))
#else
#define STARKV_API
#endif

#define STARKV_MAX_KV_HEADS 64
#define STARKV_GROUP 32        /* channels per fp16 scale in the mixed format */
#define STARKV_TILE_TOKENS 128 /* tokens per decode tile (two 64-token pages) */

typedef enum {
  STARKV_OK = 0,
  STARKV_ERR_INVALID_ARG = 1, /* null pointer, bad size, inconsistent shapes */
  STARKV_ERR_UNSUPPORTED = 2, /* valid but not implemented (e.g. head_dim 96) */
  STARKV_ERR_CUDA = 3,        /* a CUDA runtime/driver call failed (message has details) */
  STARKV_ERR_WORKSPACE = 4    /* workspace or table smaller than the size starkv_alloc gave */
} starkv_status;

/* Bits OR-ed into *dev_status by the kernels. */
#define STARKV_DEV_BOUNDS 1  /* a block-table entry outside [0, num_pages), or a position
                                outside the block table; the access is skipped */
#define STARKV_DEV_TIMEOUT 2 /* a bounded wait inside a kernel expired; the kernel released
                                its resources and returned early; outputs are undefined */

typedef enum {
  STARKV_FMT_F32 = 0,  /* latents stored as fp32; tf32 tensor cores for K = C_k B_k  */
  STARKV_FMT_BF16 = 1, /* latents stored as bf16 (RNE); bf16 tensor cores             */
  STARKV_FMT_MIXED = 2, /* int8/int4 codes + fp16 group scales; fp16 tensor cores      */
  STARKV_FMT_HAD43 = 3  /* STAR-KV technical summary, Methodology §3: latents of factors
                           rotated by a block-wise Hadamard transform, the leading
                           ceil(r/5) channels as 4-bit codes, the rest as 3-bit codes, fp16
                           group scales; fp16 tensor cores.  The caller folds the rotation
                           into the factors (A T, T^T B); append takes bf16 operands */
} starkv_fmt;

/* Model/cache description (host struct, POD). */
typedef struct {
  int32_t n_q_heads;  /* H; a multiple of n_kv_heads                                    */
  int32_t n_kv_heads; /* H_kv, 1..STARKV_MAX_KV_HEADS                                   */
  int32_t head_dim;   /* d: 64 or 128                                                  */
  int32_t d_model;    /* hidden size of x (append); a multiple of 64                    */
  int32_t key_rank;   /* r_k of the joint key latent; a multiple of 16, <= 2048          */
  int32_t value_rank[STARKV_MAX_KV_HEADS]; /* r_g of each KV head, 1..head_dim          */
  int32_t fmt;         /* starkv_fmt                                                    */
  int32_t page_tokens; /* tokens per cache page; must be 64                             */
  double rope_theta;   /* RoPE base                                                     */
} starkv_config;

/* Which latents a layout holds (starkv_layout.assignment). */
#define STARKV_ASSIGN_JOINT_KEYS 0 /* starkv_layout_init: latent 0 the joint key latent, latent
                                      1+g the value latent of KV head g                    */
#define STARKV_ASSIGN_HYBRID 1     /* starkv_hybrid_layout_init: latent g the key latent of KV
                                      head g, latent n_kv_heads the joint value latent     */

/* The pages' own assignment (STAR-KV technical summary, Methodology §2, "Hybrid
 * Decomposition Strategy"): keys decomposed head-wise (KV head g has its own latent of rank
 * r_k,g and factor B_k,g, r_k,g x d), values jointly (one latent of rank r_v for all KV heads
 * and one factor B_v, r_v x (n_kv_heads d)).  Host struct, POD. */
typedef struct {
  int32_t n_q_heads;  /* H; a multiple of n_kv_heads, at most 8 per KV head               */
  int32_t n_kv_heads; /* H_kv, 1..STARKV_MAX_KV_HEADS                                       */
  int32_t head_dim;   /* d: 64 or 128                                                      */
  int32_t d_model;    /* hidden size of x (append); a multiple of 64                        */
  int32_t key_rank[STARKV_MAX_KV_HEADS]; /* r_k,g: a multiple of 16 in [16, head_dim]       */
  int32_t value_rank; /* r_v: a multiple of 16 in [16, min(2048, n_kv_heads head_dim)]      */
  int32_t fmt;        /* starkv_fmt (every format has a layout; decode takes mixed)         */
  int32_t page_tokens; /* must be 64                                                        */
  double rope_theta;   /* RoPE base                                                         */
} starkv_hybrid_config;

/* One latent's place in a page.  In a joint-key layout latent 0 is the key latent, latent
 * 1+g the value latent of KV head g; in a hybrid layout latent g is the key latent of KV
 * head g and latent n_kv_heads the joint value latent.  Each block is token-major ([token][...]) and starts on a 16-byte
 * boundary; absent blocks have offset -1.  The quantised formats have two channel blocks,
 * the leading (more precise) one and the rest; in had43 the fields named for int8/int4 hold
 * them as follows:
 *   n8, g8   4-bit channels [0, n8), n8 = ceil(r/5), and their scale groups ceil(n8/32)
 *   n4, g4   3-bit channels [n8, r) and their scale groups ceil(n4/32)
 *   pitch    bytes per token of the packed 4-bit codes, ceil(n8/2), at off_i8; channel 2i
 *            in the low nibble of byte i, 2i+1 in the high nibble
 *   nb4      bytes per token of the packed 3-bit codes, 3*ceil(n4/8), at off_i4; each 3
 *            bytes hold 8 codes c_0..c_7 as the little-endian 24-bit word sum_i (c_i & 7) 8^i
 *   off_sc   fp16 scales [page_tokens][g8+g4], 4-bit groups first */
typedef struct {
  int32_t rank;  /* channels r                                                          */
  int32_t col;   /* first column of this latent in the concatenated projection
                    [c_k | c_v,0 | c_v,1 | ...] (and row in the stacked B_v for values);
                    hybrid: [c_k,0 | ... | c_k,H_kv-1 | c_v]                             */
  int32_t n8;    /* mixed: int8 channels [0, n8), n8 = ceil(r/4)                         */
  int32_t n4;    /* mixed: int4 channels [n8, r)                                         */
  int32_t g8;    /* mixed: scale groups of the int8 part, ceil(n8/32)                    */
  int32_t g4;    /* mixed: scale groups of the int4 part, ceil(n4/32)                    */
  int32_t nb4;   /* mixed: bytes of packed int4 codes per token, ceil(n4/2)              */
  int32_t pitch; /* f32/bf16: bytes per token of the plain block                         */
  int64_t off_plain; /* f32/bf16: values [page_tokens][r]                                */
  int64_t off_i8;    /* mixed: int8 codes [page_tokens][n8]                              */
  int64_t off_i4;    /* mixed: packed int4 codes [page_tokens][nb4]; channel n8+2i in the
                        low nibble of byte i, n8+2i+1 in the high nibble                 */
  int64_t off_sc;    /* mixed: fp16 scales [page_tokens][g8+g4], int8 groups first       */
} starkv_segment;

typedef struct {
  starkv_config cfg;        /* hybrid: the shared fields of the hybrid config; key_rank and
                               value_rank[] are 0                                      */
  int32_t n_latents;        /* 1 + n_kv_heads                                          */
  int32_t proj_cols;        /* key_rank + value_rank_total (hybrid: sum r_k,g + r_v)    */
  int32_t value_rank_total; /* R_v = sum of value_rank (hybrid: r_v)                   */
  int32_t value_rank_max;
  int64_t page_bytes;       /* bytes of one page (a multiple of 16)                     */
  int64_t token_bytes;      /* stored bytes per token over all latents, no padding      */
  starkv_segment seg[1 + STARKV_MAX_KV_HEADS];
  int32_t assignment;       /* STARKV_ASSIGN_JOINT_KEYS or STARKV_ASSIGN_HYBRID          */
  int32_t reserved;         /* 0                                                        */
  starkv_hybrid_config hybrid; /* the config of a hybrid layout; all zero otherwise     */
} starkv_layout;

/* Buffer sizes for starkv_alloc. */
typedef struct {
  size_t cache_bytes;            /* num_pages * page_bytes                               */
  size_t rope_table_bytes;       /* table for positions < max_pages * page_tokens        */
  size_t decode_workspace_bytes; /* split partials for `batch` sequences                 */
  size_t append_workspace_bytes; /* projection partials for up to max_append_tokens rows */
} starkv_sizes;

/* Optional launch settings of starkv_decode_attention (NULL = defaults). */
typedef struct {
  int32_t max_ctas;   /* persistent CTAs; 0 = one per SM                                  */
  int32_t n_ranges;   /* split of the KV heads of one 128-token tile into this many work
                         units; 0 = chosen from the grid size                             */
  int32_t timeout_ms; /* bound of every in-kernel wait; 0 = 4000 ms                       */
  int32_t cta_group;  /* 0 = auto (pairs for bf16 latents and for int8/int4 keys of rank
                         <= 256, single CTAs otherwise); 1 = one CTA per 128-token tile;
                         2 = a pair of CTAs (one cluster) per 256-token tile sharing each
                         B_k k-block (bf16 and int8/int4 latents, 256-column chunks)       */
} starkv_decode_opts;

/* Fill ``out`` from ``cfg``: per-latent mixed split, block offsets, page size.
 * Host only, pure.  INVALID_ARG / UNSUPPORTED for configurations outside the limits above. */
STARKV_API starkv_status starkv_layout_init(const starkv_config* cfg, starkv_layout* out);

/* The layout of the hybrid assignment (keys head-wise, values joint; STAR-KV technical
 * summary, Methodology §2).  Latents in page order: the key latents of KV heads 0..H_kv-1,
 * then the joint value latent; each placed exactly as starkv_layout_init places a latent of
 * the same rank and format.  Host only, pure; INVALID_ARG / UNSUPPORTED outside the limits
 * of starkv_hybrid_config.  starkv_alloc, starkv_rope_init, starkv_quant_pack, starkv_append
 * and starkv_dequant take the result (the latents are generic there); the joint-key decode
 * calls refuse it with UNSUPPORTED, starkv_hybrid_decode takes only it. */
STARKV_API starkv_status starkv_hybrid_layout_init(const starkv_hybrid_config* cfg,
                                                   starkv_layout* out);

/* Sizes of the caller-allocated buffers (nothing is allocated).  ``max_pages`` is the
 * row length of the block table; positions run below max_pages * page_tokens.
 * ``max_append_tokens`` bounds n_tok of starkv_append. */
STARKV_API starkv_status starkv_alloc(const starkv_layout* lay, int64_t num_pages, int32_t batch,
                           int32_t max_pages, int32_t max_append_tokens, starkv_sizes* out);

/* Write the RoPE table into ``table`` (device, rope_table_bytes from starkv_alloc for the
 * same max_pages): cos/sin of t*theta^(-2j/d) computed in fp64 on the device and stored as
 * fp32, for t on a 128-token grid and for offsets 0..127 within a tile. */
STARKV_API starkv_status starkv_rope_init(const starkv_layout* lay, int32_t max_pages, void* table,
                               size_t table_bytes, starkv_stream_t stream);

/* Store fp32 latents in the cache (steps a2-a3 of the write path without the projection):
 *   latents     device fp32 [n_tok][proj_cols], rows [c_k | c_v,0 | ...]
 *   tok_seq/pos device int32 [n_tok]: sequence index (< batch) and 0-based position
 *   block_table device int32 [batch][max_pages]; token (b, p) goes to page
 *               block_table[b][p / 64], slot p % 64
 *   cache       device, num_pages * page_bytes bytes
 * f32 stores the values, bf16 rounds to nearest even, mixed and had43 quantise per group
 * (see starkv_segment) -- bit-exact with the reference definition.  Tokens with a bad page or
 * position are skipped and flagged STARKV_DEV_BOUNDS.  Tokens written by one call must be
 * distinct. */
STARKV_API starkv_status starkv_quant_pack(const starkv_layout* lay, const float* latents, int32_t n_tok,
                                const int32_t* tok_seq, const int32_t* tok_pos,
                                const int32_t* block_table, int32_t max_pages, int32_t batch,
                                void* cache, int64_t num_pages, int32_t* dev_status,
                                starkv_stream_t stream);

/* Latent write of new tokens: c = x [A_k | A_v,0 | ...] on tcgen05 tensor cores with fp32
 * accumulation, then the store of starkv_quant_pack.
 *   x           device [n_tok][d_model], bf16 (fmt bf16/mixed) or fp32 (fmt f32, tf32 MMA)
 *   A_t         device [proj_cols][d_model], same dtype as x: row c is column c of the
 *               concatenated down-projection (K-major for the tensor cores)
 *   latents_out device fp32 [n_tok][proj_cols] or NULL: receives c before storage
 *   workspace   device, >= append_workspace_bytes for n_tok (split-K partials)
 * Other arguments as starkv_quant_pack. */
STARKV_API starkv_status starkv_append(const starkv_layout* lay, const void* x, int32_t n_tok,
                            const void* A_t, const int32_t* tok_seq, const int32_t* tok_pos,
                            const int32_t* block_table, int32_t max_pages, int32_t batch,
                            void* cache, int64_t num_pages, float* latents_out, void* workspace,
                            size_t workspace_bytes, int32_t* dev_status, starkv_stream_t stream);

/* Read stored latents back as fp32 (dequantised for mixed: scale * code, exact):
 *   latents_out device fp32 [n_tok][proj_cols].  For tests and inspection. */
STARKV_API starkv_status starkv_dequant(const starkv_layout* lay, const void* cache, int64_t num_pages,
                             const int32_t* tok_seq, const int32_t* tok_pos, int32_t n_tok,
                             const int32_t* block_table, int32_t max_pages, int32_t batch,
                             float* latents_out, int32_t* dev_status, starkv_stream_t stream);

/* Single-token decode attention read from the latent cache.
 *   q          device [batch][H][d] query of the token at position seq_len-1, before RoPE;
 *              bf16 (fmt bf16/mixed) or fp32 (fmt f32)
 *   seq_lens   device int32 [batch]; 0 gives a zero output row
 *   Bk_t       device [H_kv*d][key_rank], row n = column n of B_k: fp32 (f32), bf16 (bf16),
 *              fp16 (mixed, had43) -- the tensor-core operand type of the format
 *   Bv         device fp32 [value_rank_total][d]: B_v,g stacked in head order (rows
 *              seg[1+g].col - key_rank ...)
 *   rope_table device, from starkv_rope_init with max_pages >= this call's max_pages
 *   out        device fp32 [batch][H][d]
 *   workspace  device, >= decode_workspace_bytes of starkv_alloc for this batch/max_pages
 * Two launches: a persistent split kernel (tcgen05 K reconstruction into TMEM, RoPE,
 * online softmax, latent P.C_v, one partial per 128-token tile and query head) and a
 * combine kernel (log-sum-exp merge of the partials, then o = a B_v).
 * STARKV_ERR_UNSUPPORTED, with nothing launched, when the split kernel's shared-memory plan
 * does not fit the device (fp32 latents with 8 query heads per KV head, for one);
 * starkv_decode_plan_query answers that on the host beforehand. */
STARKV_API starkv_status starkv_decode_attention(const starkv_layout* lay, const void* q, const void* cache,
                                      int64_t num_pages, const int32_t* block_table,
                                      int32_t max_pages, const int32_t* seq_lens, int32_t batch,
                                      const void* Bk_t, const float* Bv, const void* rope_table,
                                      size_t rope_table_bytes, float* out, void* workspace,
                                      size_t workspace_bytes, const starkv_decode_opts* opts,
                                      int32_t* dev_status, starkv_stream_t stream);

/* Launch shape that starkv_decode_attention / starkv_decode_partials choose for a layout,
 * batch and block-table width on a device with ``num_sms`` SMs and ``smem_per_block`` bytes
 * of opt-in shared memory per block (148 and 232448 on a B200).  Host only, pure: the decode
 * calls make the same choice with the current device's figures.  (The pages describe no such
 * interface; it exposes this library's launch planning.)  INVALID_ARG for a bad layout or
 * sizes; UNSUPPORTED for a configuration the decode calls would refuse. */
typedef struct {
  int32_t cta_group;     /* 1: one CTA per 128-token tile; 2: a CTA pair per 256-token tile  */
  int32_t key_mode;      /* int8/int4 keys: 1 = dequantised operand resident per tile, 2 =
                            codes staged per tile and the operand streamed through the ring,
                            0 = codes read from global memory; 0 for f32/bf16 (TMA ring)      */
  int32_t chunk_cols;    /* columns of K (KV heads x d) reconstructed per MMA chunk          */
  int32_t n_chunks;      /* chunks per tile                                                  */
  int32_t n_ranges;      /* work units a tile's chunks are split into                        */
  int32_t stages;        /* operand ring stages                                              */
  int32_t value_buffers; /* value-latent buffers (double-buffered page pairs)                */
  int32_t smem_bytes;    /* dynamic shared memory per CTA                                    */
  int32_t grid;          /* CTAs launched (pairs are further capped at those co-resident)    */
  int32_t work_units;    /* (tile group, sequence, range) units of the persistent loop        */
} starkv_decode_plan;

STARKV_API starkv_status starkv_decode_plan_query(const starkv_layout* lay, int32_t batch,
                                                  int32_t max_pages, const starkv_decode_opts* opts,
                                                  int32_t num_sms, int64_t smem_per_block,
                                                  starkv_decode_plan* out);

/* The split step of starkv_decode_attention alone: one partial record per (sequence b,
 * query head h, 128-token tile t) in ``workspace``, at float offset
 *   ((b * H + h) * T + t) * R,   T = ceil(max_pages * 64 / 128),  R = 4 * ceil((2 + value_rank_max) / 4)
 * holding [m, l, a_0 .. a_{r_g - 1}]: m the tile's largest score in log2 units (q'.k' *
 * log2(e)/sqrt(d)), l = sum_t 2^(s_t - m), a = sum_t 2^(s_t - m) c_v,g,t.  Tiles at or past
 * seq_len are not written.  Arguments as starkv_decode_attention. */
STARKV_API starkv_status starkv_decode_partials(const starkv_layout* lay, const void* q,
                                                const void* cache, int64_t num_pages,
                                                const int32_t* block_table, int32_t max_pages,
                                                const int32_t* seq_lens, int32_t batch,
                                                const void* Bk_t, const void* rope_table,
                                                size_t rope_table_bytes, void* workspace,
                                                size_t workspace_bytes,
                                                const starkv_decode_opts* opts, int32_t* dev_status,
                                                starkv_stream_t stream);

/* The combine step alone: for every (b, h), merge the partial records of tiles
 * 0 .. ceil(seq_len/128)-1 (log-sum-exp), normalise, and write out[b][h] = a B_v,g(h).
 * seq_len 0 writes zeros.  Arguments as starkv_decode_attention. */
STARKV_API starkv_status starkv_decode_combine(const starkv_layout* lay, const int32_t* seq_lens,
                                               int32_t batch, int32_t max_pages, const float* Bv,
                                               const void* workspace, size_t workspace_bytes,
                                               float* out, starkv_stream_t stream);

/* Weight absorption (STAR-KV technical summary, Methodology §2: the values' up-projection is
 * folded into the attention output projection, so values are never reconstructed).  With one
 * value latent per KV head, query head h gets M_h = B_v,g(h) W_o,h, where W_o,h is the rows
 * [h*d, (h+1)*d) of the output projection W_o (n_q_heads*d x d_out), and the attention block's
 * output for the decoded token of sequence b is y_b = sum_h a_b,h M_h, a_b,h the normalised
 * latent-space output of head h.
 *
 * starkv_absorbed_sizes: rows of M (sum over query heads of r_g(h)) and the bytes of scratch
 * that starkv_decode_combine_absorbed needs for ``batch`` sequences.  Host only. */
STARKV_API starkv_status starkv_absorbed_sizes(const starkv_layout* lay, int32_t batch,
                                               int32_t d_out, int64_t* m_rows,
                                               size_t* scratch_bytes);

/* Build M once (setup, fp32):
 *   Bv  device fp32 [value_rank_total][d], as for starkv_decode_attention
 *   Wo  device fp32 [n_q_heads*d][d_out], row-major (o_concat . Wo)
 *   M   device fp32 [m_rows][d_out]: the r_g rows of query head h start at
 *       G * (sum of r_g' over KV heads g' < g) + (h mod G) * r_g. */
STARKV_API starkv_status starkv_absorb_output_weights(const starkv_layout* lay, const float* Bv,
                                                      const float* Wo, int32_t d_out, float* M,
                                                      starkv_stream_t stream);

/* The combine step with absorbed weights: merge the partial records of every (b, h) as
 * starkv_decode_combine does, keep a_b,h, then out[b][:] = sum_h a_b,h M_h.
 *   M        from starkv_absorb_output_weights for the same d_out
 *   scratch  device, >= scratch_bytes of starkv_absorbed_sizes, 16-byte aligned
 *   out      device fp32 [batch][d_out]; seq_len 0 gives a zero row
 * Other arguments as starkv_decode_combine. */
STARKV_API starkv_status starkv_decode_combine_absorbed(
    const starkv_layout* lay, const int32_t* seq_lens, int32_t batch, int32_t max_pages,
    const float* M, int32_t d_out, const void* workspace, size_t workspace_bytes, void* scratch,
    size_t scratch_bytes, float* out, starkv_stream_t stream);

/* starkv_decode_attention without a workspace argument, for callers that cannot allocate
 * device memory: a plugin inside a host process whose memory pool has already reserved the
 * GPU's memory, a C caller with no device allocator, or a loop where a cudaMalloc is not
 * acceptable because it may synchronise the device.  (The pages describe no such interface;
 * it has no counterpart there.)
 *   - The partial records live in a 16 MiB array inside the library's device image; every
 *     GPU that loads the library holds it until the process exits.  Calls whose records need
 *     more (batch * n_q_heads * ceil(max_pages / 2) * 4 * ceil((2 + value_rank_max) / 4)
 *     floats) return STARKV_ERR_WORKSPACE with a message; nothing is launched.
 *   - The first call in a CUDA context (the device's primary context, or a context the
 *     caller made current) looks up the array's device address in that context and keeps
 *     it, keyed on the context's unique ID; a context created again after cudaDeviceReset
 *     gets a fresh lookup.  Make that first call before any stream capture.
 *   - All calls share the array and it keeps the last call's contents.  Nothing in it needs
 *     to start at zero: each call writes every record it reads.  Calls whose kernels overlap
 *     on the GPU (two streams, two threads, two graphs) race on it.  A CUDA graph that
 *     captured this call holds the array's address, so every such graph shares the one
 *     array too: replays of two of them must be ordered on the GPU, and the device status
 *     word does not show a race.
 *   - Allocates nothing (no cudaMalloc / cudaFree).  Other arguments, results and errors as
 *     starkv_decode_attention. */
STARKV_API starkv_status starkv_decode_attention_noalloc(
    const starkv_layout* lay, const void* q, const void* cache, int64_t num_pages,
    const int32_t* block_table, int32_t max_pages, const int32_t* seq_lens, int32_t batch,
    const void* Bk_t, const float* Bv, const void* rope_table, size_t rope_table_bytes, float* out,
    const starkv_decode_opts* opts, int32_t* dev_status, starkv_stream_t stream);

/* Single-token decode attention with the hybrid assignment (STAR-KV technical summary,
 * Methodology §2: keys head-wise, values joint).  For query head h of KV head g = h / G:
 *   K_g = C_k,g B_k,g, RoPE on K_g and on q_h (position seq_len-1), p = softmax(q' K'^T / sqrt(d)),
 *   a_h = p C_v (the joint value latent space, r_v wide), o_h = a_h B_v[:, g d : (g+1) d].
 *   lay        a layout from starkv_hybrid_layout_init, fmt mixed (int8/int4); other formats
 *              UNSUPPORTED
 *   q          device bf16 [batch][H][d], before RoPE
 *   Bk_t       device fp16: for each KV head g in order, the block [d][r_k,g] whose row n is
 *              column n of B_k,g; block g starts at element d * (r_k,0 + ... + r_k,g-1)
 *   Bv         device fp32 [r_v][H_kv d] (B_v itself)
 *   rope_table device, from starkv_rope_init with max_pages >= this call's max_pages
 *   out        device fp32 [batch][H][d]; a sequence of length 0 gives zeros
 *   workspace  device, >= decode_workspace_bytes of starkv_alloc for this batch/max_pages
 *              (per (sequence, page range, query head): m, l and the r_v-wide a)
 * Two launches: a split kernel (one CTA per SM, looping over (sequence, page range) units;
 * per 64-token page: a bulk copy of the page, int8/int4 codes to fp16, K_g on the tensor
 * cores (mma.sync, fp32 accumulation), RoPE, scores on the tensor cores from the rotated keys
 * split into two fp16 parts, online softmax, P C_v on the tensor cores) and a combine
 * (log-sum-exp merge of the page ranges, then o_h = a_h B_v,g).  Limits of the kernel
 * (UNSUPPORTED, nothing launched): n_kv_heads <= 16, H <= 64, ceil(H/16) ceil(r_v/64) <= 8,
 * a page below 1 MiB, and the shared-memory plan (all B_k,g resident) within the device's
 * per-block limit.  Errors in *dev_status as for starkv_decode_attention. */
STARKV_API starkv_status starkv_hybrid_decode(const starkv_layout* lay, const void* q,
                                              const void* cache, int64_t num_pages,
                                              const int32_t* block_table, int32_t max_pages,
                                              const int32_t* seq_lens, int32_t batch,
                                              const void* Bk_t, const float* Bv,
                                              const void* rope_table, size_t rope_table_bytes,
                                              float* out, void* workspace, size_t workspace_bytes,
                                              int32_t* dev_status, starkv_stream_t stream);

/* Failure-detection check of the in-kernel bounded waits: one CTA holds TMEM and waits on a
 * barrier that nothing completes.  After ``timeout_ms`` (1..10000) the wait gives up, the CTA
 * sets STARKV_DEV_TIMEOUT in *dev_status, releases TMEM and returns; the context stays usable.
 * Device code of every kernel here waits through the same helper. */
STARKV_API starkv_status starkv_diag_bounded_wait(int32_t timeout_ms, int32_t* dev_status,
                                                  starkv_stream_t stream);

/* One-line description of the last non-OK return on this thread. */
STARKV_API const char* starkv_last_error(void);

/* ABI version: 100 * major + minor. */
STARKV_API int32_t starkv_version(void);

#ifdef __cplusplus
}
#endif
#endif /* STARKV_H */
