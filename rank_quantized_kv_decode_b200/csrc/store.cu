// Latent storage: fp32 / bf16 / int8+int4 quantisation and packing into cache pages, the
// read-back (dequantisation) of stored latents, and the RoPE table.
//
// Quantiser (per token, per latent, per group of 32 channels; groups restart where the
// int4 part starts): s16 = fp16_rne(fp32(amax) / qmax) saturated to 65504,
// code = clamp(rint_half_even(fp32(c) / fp32(s16)), -qmax, qmax), s16 == 0 gives code 0.
// The leading ceil(r/4) channels (singular-value order: the outlier channels of STAR-KV
// technical summary, Methodology §3 "Low-Rank-Aware Mixed-Precision Quantization") are int8,
// the rest int4, two per byte with the even channel in the low nibble.
//
// The pages' own format (had43; same page, Methodology §3 "Low-Rank-Aware Mixed-Precision
// Quantization"): latents of factors already rotated by the block-wise Hadamard transform;
// the leading ceil(r/5) channels are 4-bit codes (qmax 7, two per byte as above), the rest
// 3-bit codes (qmax 3), eight per 3 bytes as the little-endian 24-bit word
// sum_i (code_i & 7) 8^i; same scale rule, groups of 32 restarting at the 3-bit block.
#include "internal.cuh"

namespace starkv {

namespace {

__device__ __forceinline__ float warp_max_abs(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// fp16 scale of a group (saturating) and the code of value c.
__device__ __forceinline__ __half group_scale(float amax, float qmax) {
  __half h = __float2half_rn(__fdiv_rn(amax, qmax));
  if (__hisinf(h)) h = __ushort_as_half(static_cast<unsigned short>(0x7BFF));
  return h;
}
__device__ __forceinline__ int quant_code(float c, float s, int qmax) {
  if (s == 0.f) return 0;
  const int q = __float2int_rn(__fdiv_rn(c, s));
  return max(-qmax, min(qmax, q));
}

struct TokenSlot {
  uint8_t* page;  // nullptr if the token's page or position is invalid
  int slot;
};

__device__ __forceinline__ TokenSlot locate(const StoreParams& p, int n, int li, int lane) {
  const int b = p.tok_seq[n], pos = p.tok_pos[n];
  TokenSlot t{nullptr, 0};
  if (b < 0 || b >= p.batch || pos < 0 || pos >= p.max_pages * kPage) {
    if (lane == 0 && li == 0 && p.status) atomicOr(p.status, STARKV_DEV_BOUNDS);
    return t;
  }
  const int pg = p.block_table[(long long)b * p.max_pages + pos / kPage];
  if (pg < 0 || pg >= p.num_pages) {
    if (lane == 0 && li == 0 && p.status) atomicOr(p.status, STARKV_DEV_BOUNDS);
    return t;
  }
  t.page = p.cache + (long long)pg * p.page_bytes;
  t.slot = pos % kPage;
  return t;
}

// Sum of the split-K partials of one value, in split order (deterministic).  Up to 16 loads
// are issued before the first add, so a decode step's partials arrive in one round trip.
__device__ __forceinline__ float split_sum(const float* src, long long stride, int nsplit) {
  float v = 0.f;
  for (int s0 = 0; s0 < nsplit; s0 += 16) {
    float t[16];
#pragma unroll
    for (int k = 0; k < 16; ++k) t[k] = s0 + k < nsplit ? __ldcg(src + (s0 + k) * stride) : 0.f;
#pragma unroll
    for (int k = 0; k < 16; ++k)
      if (s0 + k < nsplit) v = (s0 + k == 0) ? t[k] : v + t[k];
  }
  return v;
}

// One warp per (token, latent, 32-channel chunk): lane = channel.  In the int8/int4 format a
// chunk is one quantisation group (the int8 groups, then the int4 groups of the latent).
__global__ void __launch_bounds__(128) store_kernel(const __grid_constant__ StoreParams p) {
  pdl_wait();
  pdl_launch_dependents();
  const int gw = blockIdx.x * 4 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (gw >= p.n_tok * p.chunks_per_token) return;  // whole warp
  const int n = gw / p.chunks_per_token;
  const int ck = gw % p.chunks_per_token;
  int li = 0;
  while (p.chunk_start[li + 1] <= ck) ++li;
  const int cl = ck - p.chunk_start[li];  // chunk within the latent
  const LatDesc& d = p.lat[li];
  const float* src = p.src + (long long)n * p.proj_cols + d.col;
  float* lout = p.latents_out ? p.latents_out + (long long)n * p.proj_cols + d.col : nullptr;
  // this lane's channel of the chunk; the partial sums are loaded before the page lookup so
  // that both round trips overlap
  const bool plain = p.fmt == STARKV_FMT_F32 || p.fmt == STARKV_FMT_BF16;
  const bool is8 = !plain && cl < d.g8;
  const int n4 = d.rank - d.n8;
  const int j = (plain || is8) ? 0 : (cl - d.g8) * 32 + lane;  // int4 channel index
  const int i = (plain || is8) ? cl * 32 + lane : d.n8 + j;    // channel in the latent
  const bool in = plain ? i < d.rank : (is8 ? i < d.n8 : j < n4);
  const float c = in ? split_sum(src + i, p.split_stride, p.nsplit) : 0.f;
  if (lout && in) lout[i] = c;
  const TokenSlot ts = locate(p, n, (li == 0 && cl == 0) ? 0 : 1, lane);

  if (plain) {
    if (!in || !ts.page) return;
    uint8_t* dst = ts.page + d.off0 + ts.slot * d.pitch;
    if (p.fmt == STARKV_FMT_F32)
      reinterpret_cast<float*>(dst)[i] = c;
    else
      reinterpret_cast<__nv_bfloat16*>(dst)[i] = __float2bfloat16_rn(c);
    return;
  }
  __half* sc = ts.page ? reinterpret_cast<__half*>(ts.page + d.off2) + ts.slot * d.ng : nullptr;
  if (p.fmt == STARKV_FMT_HAD43) {
    const float amax = warp_max_abs(in ? fabsf(c) : 0.f);
    if (is8) {
      // 4-bit group cl: channels [32 cl, min(32 cl + 32, n8)), d.pitch packed bytes per token
      const __half h = group_scale(amax, 7.f);
      const int nib = quant_code(c, __half2float(h), 7) & 15;
      const int hi = __shfl_down_sync(0xffffffffu, nib, 1);
      if (ts.page && in && (i & 1) == 0) {
        const int byte = nib | ((i + 1 < d.n8 ? hi : 0) << 4);
        (ts.page + d.off0)[ts.slot * d.pitch + (i >> 1)] = static_cast<uint8_t>(byte);
      }
      if (ts.page && lane == 0) sc[cl] = h;
    } else {
      // 3-bit group gi: channels n8 + [32 gi, min(32 gi + 32, n4)); lanes 8k..8k+7 form word
      // k of the group (lanes past n4 hold c = 0, code 0: the padding of the last word)
      const int gi = cl - d.g8;
      const __half h = group_scale(amax, 3.f);
      const int code = quant_code(c, __half2float(h), 3) & 7;
      uint32_t w = static_cast<uint32_t>(code) << (3 * (lane & 7));
      w |= __shfl_xor_sync(0xffffffffu, w, 1);
      w |= __shfl_xor_sync(0xffffffffu, w, 2);
      w |= __shfl_xor_sync(0xffffffffu, w, 4);
      if (ts.page && in && (lane & 7) == 0) {
        uint8_t* dst = ts.page + d.off1 + ts.slot * d.nb4 + 3 * (j >> 3);
        dst[0] = static_cast<uint8_t>(w);
        dst[1] = static_cast<uint8_t>(w >> 8);
        dst[2] = static_cast<uint8_t>(w >> 16);
      }
      if (ts.page && lane == 0) sc[d.g8 + gi] = h;
    }
    return;
  }
  if (is8) {
    // int8 group cl: channels [32 cl, min(32 cl + 32, n8))
    const float amax = warp_max_abs(in ? fabsf(c) : 0.f);
    const __half h = group_scale(amax, 127.f);
    const int q = quant_code(c, __half2float(h), 127);
    if (ts.page && in) reinterpret_cast<int8_t*>(ts.page + d.off0)[ts.slot * d.n8 + i] = static_cast<int8_t>(q);
    if (ts.page && lane == 0) sc[cl] = h;
  } else {
    // int4 group gi: channels n8 + [32 gi, min(32 gi + 32, n4))
    const int gi = cl - d.g8;
    const float amax = warp_max_abs(in ? fabsf(c) : 0.f);
    const __half h = group_scale(amax, 7.f);
    const int q = quant_code(c, __half2float(h), 7);
    const int nib = q & 15;
    const int hi = __shfl_down_sync(0xffffffffu, nib, 1);
    if (ts.page && in && (j & 1) == 0) {
      const int byte = nib | ((j + 1 < n4 ? hi : 0) << 4);
      (ts.page + d.off1)[ts.slot * d.nb4 + (j >> 1)] = static_cast<uint8_t>(byte);
    }
    if (ts.page && lane == 0) sc[d.g8 + gi] = h;
  }
}

// One warp per (token, latent): stored value -> fp32 (scale * code for the mixed format).
__global__ void __launch_bounds__(128) dequant_kernel(const __grid_constant__ StoreParams p) {
  const int gw = blockIdx.x * 4 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (gw >= p.n_tok * p.n_lat) return;
  const int n = gw / p.n_lat, li = gw % p.n_lat;
  const LatDesc& d = p.lat[li];
  const TokenSlot ts = locate(p, n, li, lane);
  float* out = p.latents_out + (long long)n * p.proj_cols + d.col;
  for (int i = lane; i < d.rank; i += 32) {
    float v = 0.f;
    if (ts.page) {
      const uint8_t* pg = ts.page;
      if (p.fmt == STARKV_FMT_F32) {
        v = reinterpret_cast<const float*>(pg + d.off0 + ts.slot * d.pitch)[i];
      } else if (p.fmt == STARKV_FMT_BF16) {
        v = __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(pg + d.off0 + ts.slot * d.pitch)[i]);
      } else if (p.fmt == STARKV_FMT_HAD43) {
        const __half* sc = reinterpret_cast<const __half*>(pg + d.off2) + ts.slot * d.ng;
        if (i < d.n8) {
          const uint8_t byte = (pg + d.off0)[ts.slot * d.pitch + (i >> 1)];
          const int nib = (i & 1) ? (byte >> 4) : (byte & 15);
          v = __half2float(sc[i >> 5]) * static_cast<float>((nib ^ 8) - 8);
        } else {
          const int j = i - d.n8;
          const uint8_t* w = pg + d.off1 + ts.slot * d.nb4 + 3 * (j >> 3);
          const uint32_t word = w[0] | (static_cast<uint32_t>(w[1]) << 8) | (static_cast<uint32_t>(w[2]) << 16);
          const int code = (word >> (3 * (j & 7))) & 7;
          v = __half2float(sc[d.g8 + (j >> 5)]) * static_cast<float>((code ^ 4) - 4);
        }
      } else {
        const __half* sc = reinterpret_cast<const __half*>(pg + d.off2) + ts.slot * d.ng;
        if (i < d.n8) {
          const int8_t q = reinterpret_cast<const int8_t*>(pg + d.off0)[ts.slot * d.n8 + i];
          v = __half2float(sc[i >> 5]) * static_cast<float>(q);
        } else {
          const int j = i - d.n8;
          const uint8_t byte = (pg + d.off1)[ts.slot * d.nb4 + (j >> 1)];
          const int nib = (j & 1) ? (byte >> 4) : (byte & 15);
          v = __half2float(sc[d.g8 + (j >> 5)]) * static_cast<float>((nib ^ 8) - 8);
        }
      }
    }
    out[i] = v;
  }
}

// cos/sin of t * theta^(-2j/d) in fp64, stored as fp32: rows 0..127 are t = row (offset
// inside a 128-token tile), rows 128.. are t = 128 * (row - 128) (tile starts).
__global__ void rope_init_kernel(float2* table, int half_dim, int rows, double theta,
                                 int head_dim) {
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= rows * half_dim) return;
  const int row = idx / half_dim, j = idx % half_dim;
  const double t = row < kTile ? static_cast<double>(row) : static_cast<double>(kTile) * (row - kTile);
  const double inv = pow(theta, -2.0 * static_cast<double>(j) / static_cast<double>(head_dim));
  double s, c;
  sincos(t * inv, &s, &c);
  table[idx] = make_float2(static_cast<float>(c), static_cast<float>(s));
}

}  // namespace

cudaError_t launch_store(const StoreParams& p, cudaStream_t s) {
  const long long warps = (long long)p.n_tok * p.chunks_per_token;
  if (warps == 0) return cudaSuccess;
  return launch_pdl(store_kernel, dim3(static_cast<unsigned>((warps + 3) / 4)), dim3(128), 0, s, p);
}

cudaError_t launch_dequant(const StoreParams& p, cudaStream_t s) {
  const long long warps = (long long)p.n_tok * p.n_lat;
  if (warps == 0) return cudaSuccess;
  dequant_kernel<<<static_cast<unsigned>((warps + 3) / 4), 128, 0, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_rope_init(float2* table, int half_dim, int rows_fine, int tiles, double theta,
                             int head_dim, cudaStream_t s) {
  const int rows = rows_fine + tiles;
  const int total = rows * half_dim;
  rope_init_kernel<<<(total + 255) / 256, 256, 0, s>>>(table, half_dim, rows, theta, head_dim);
  return cudaGetLastError();
}

}  // namespace starkv
