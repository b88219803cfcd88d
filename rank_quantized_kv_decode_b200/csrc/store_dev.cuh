// Device side of the latent store, shared by the store kernel (fp32 latents from split-K
// partials) and the fused decode-step append (fp32 latents from its own projection): the
// quantisation, packing and scatter of one 32-channel chunk of one token, lane = channel.
// Both callers give it the same fp32 value, so both write the same bytes.
//
// Quantiser (per token, per latent, per group of 32 channels; groups restart where the
// int4 part starts): s16 = fp16_rne(fp32(amax) / qmax) saturated to 65504,
// code = clamp(rint_half_even(fp32(c) / fp32(s16)), -qmax, qmax), s16 == 0 gives code 0.
#pragma once
#include "internal.cuh"

namespace starkv {
namespace store_dev {

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

// The channel of a lane in chunk ``ck`` of a token (chunks: per latent, its 32-channel groups;
// in the quantised formats the groups of the leading block, then those of the rest).
struct ChunkLane {
  int li, cl;     // latent, chunk within the latent
  bool plain, is8, in;
  int n4, j, i;   // channels of the second block; channel index there; channel in the latent
};

// FMT: the storage format when the caller knows it at compile time, -1 to read p.fmt.
template <int FMT = -1>
__device__ __forceinline__ ChunkLane chunk_lane(const StoreParams& p, int ck, int lane) {
  const int fmt = FMT >= 0 ? FMT : p.fmt;
  ChunkLane c{};
  int li = 0;
  while (p.chunk_start[li + 1] <= ck) ++li;
  c.li = li;
  c.cl = ck - p.chunk_start[li];
  const LatDesc& d = p.lat[li];
  c.plain = fmt == STARKV_FMT_F32 || fmt == STARKV_FMT_BF16;
  c.is8 = !c.plain && c.cl < d.g8;
  c.n4 = d.rank - d.n8;
  c.j = (c.plain || c.is8) ? 0 : (c.cl - d.g8) * 32 + lane;
  c.i = (c.plain || c.is8) ? c.cl * 32 + lane : d.n8 + c.j;
  c.in = c.plain ? c.i < d.rank : (c.is8 ? c.i < d.n8 : c.j < c.n4);
  return c;
}

// Store the value ``c`` of this lane's channel for token ``n`` at its page and slot ``ts``
// (from locate; the whole warp calls it; lanes outside the chunk pass c = 0).  Writes
// latents_out too when the caller asked for it.
template <int FMT = -1>
__device__ __forceinline__ void store_value_at(const StoreParams& p, const ChunkLane& q, int n,
                                               int lane, float c, const TokenSlot& ts) {
  const int fmt = FMT >= 0 ? FMT : p.fmt;
  const LatDesc& d = p.lat[q.li];
  const int cl = q.cl, j = q.j, i = q.i, n4 = q.n4;
  const bool plain = q.plain, is8 = q.is8, in = q.in;
  float* lout = p.latents_out ? p.latents_out + (long long)n * p.proj_cols + d.col : nullptr;
  if (lout && in) lout[i] = c;

  if (plain) {
    if (!in || !ts.page) return;
    uint8_t* dst = ts.page + d.off0 + ts.slot * d.pitch;
    if (fmt == STARKV_FMT_F32)
      reinterpret_cast<float*>(dst)[i] = c;
    else
      reinterpret_cast<__nv_bfloat16*>(dst)[i] = __float2bfloat16_rn(c);
    return;
  }
  __half* sc = ts.page ? reinterpret_cast<__half*>(ts.page + d.off2) + ts.slot * d.ng : nullptr;
  if (fmt == STARKV_FMT_HAD43) {
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

}  // namespace store_dev
}  // namespace starkv
