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
#include "store_dev.cuh"

namespace starkv {

namespace {

using namespace store_dev;

// Sum of the split-K partials of one value, in split order (deterministic).  Up to 16 loads
// are issued before the first add, so a decode step's partials arrive in one round trip.
__device__ __forceinline__ float split_sum(const float* src, long long stride, int nsplit) {
  if (nsplit == 1) return __ldcg(src);  // one split (a prefill-sized append): a single load
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

// One warp per (token, latent, 32-channel chunk): lane = channel; token n = blockIdx.x, chunk
// = 4 blockIdx.y + warp.  In the int8/int4 format a chunk is one quantisation group (the int8
// groups, then the int4 groups of the latent).  FMT is the storage format.
template <int FMT>
__global__ void __launch_bounds__(128) store_kernel(const __grid_constant__ StoreParams p) {
  pdl_wait();
  pdl_launch_dependents();
  const int ck = blockIdx.y * 4 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (ck >= p.chunks_per_token) return;  // whole warp
  const int n = blockIdx.x;
  const ChunkLane q = chunk_lane<FMT>(p, ck, lane);
  const float* src = p.src + (long long)n * p.proj_cols + p.lat[q.li].col;
  const float c = q.in ? split_sum(src + q.i, p.split_stride, p.nsplit) : 0.f;
  // the page lookup flags a bad page or position once per token: in the chunk of latent 0,
  // channel 0
  const TokenSlot ts = locate(p, n, (q.li == 0 && q.cl == 0) ? 0 : 1, lane);
  store_value_at<FMT>(p, q, n, lane, c, ts);
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
  if (p.n_tok == 0 || p.chunks_per_token == 0) return cudaSuccess;
  const dim3 grid(static_cast<unsigned>(p.n_tok), static_cast<unsigned>((p.chunks_per_token + 3) / 4));
  switch (p.fmt) {
    case STARKV_FMT_F32: return launch_pdl(store_kernel<STARKV_FMT_F32>, grid, dim3(128), 0, s, p);
    case STARKV_FMT_BF16: return launch_pdl(store_kernel<STARKV_FMT_BF16>, grid, dim3(128), 0, s, p);
    case STARKV_FMT_MIXED: return launch_pdl(store_kernel<STARKV_FMT_MIXED>, grid, dim3(128), 0, s, p);
    case STARKV_FMT_HAD43: return launch_pdl(store_kernel<STARKV_FMT_HAD43>, grid, dim3(128), 0, s, p);
    default: return cudaErrorInvalidValue;
  }
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
