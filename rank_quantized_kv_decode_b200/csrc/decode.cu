// Decode attention read straight from the latent cache (sm_100a).
//
// Split kernel (persistent, warp-specialised, one CTA per SM, or a CTA pair per cluster with
// cta_group::2).  A work unit is one 128-token tile (two 64-token pages) of one sequence --
// 256 tokens for a pair, each CTA owning 128 -- and a range of 256-column chunks of the
// reconstructed keys (2 KV heads of d=128, or 4 of d=64):
//   warp 0      TMA producer: latent k-blocks of the two pages (f32/bf16) and B_k^T k-blocks
//   warp 1      tcgen05 issuer: K_chunk = C_k(128 x r_k) * B_k(r_k x 256) into TMEM (fp32),
//               double-buffered accumulators (2 x 256 columns); M = 256 across a pair
//   warp 2      bulk-copy producer of the value latents of the chunk's heads (both pages)
//   warp 3      int8/int4 keys: bulk-copy stager of the tile's key codes
//   warps 4-11  two epilogue warpgroups, thread = token row (TMEM lane): warpgroup w rotates
//               and dots half of the RoPE pairs of every head of the chunk; then, for the
//               heads it owns, the tile-local softmax (max, sum) and the latent P.C_v, one
//               partial record per query head
//   warps 12-15 int8/int4 keys: dequantisers (codes * fp16 scale -> fp16 operand tile in the
//               128-byte-swizzled layout the tensor core reads), once per tile into resident
//               slots (rank <= 256) or per ring stage; fp32 latents: tf32 hi/lo splitters
// The pages' point that joint key latents cost h x more to reconstruct (STAR-KV technical
// summary, Methodology §2 "Hybrid Decomposition Strategy") is why the reconstruction runs
// on the tensor cores: it is a dense (tokens x r_k) x (r_k x H_kv*d) contraction.
//
// Combine kernel: log-sum-exp merge of the per-tile partials of each (sequence, query head),
// then the up-projection o_h = a_h B_v,g -- or, for the absorbed output, the normalised a_h
// alone.
#include "internal.cuh"

namespace starkv {

namespace {

constexpr int FMT_F32 = STARKV_FMT_F32;
constexpr int FMT_BF16 = STARKV_FMT_BF16;
constexpr int FMT_MIXED = STARKV_FMT_MIXED;
// the pages' own 4-bit/3-bit block-Hadamard format: decoded by the int8/int4 machinery (staged
// codes, fp16 operand) with its own code layout
constexpr int FMT_HAD43 = STARKV_FMT_HAD43;

struct Unit {
  int b, tile, c0, c1, L, nvalid;
  int page0, page1;  // physical pages of the tile's two halves, -1 if absent or invalid
  __device__ __forceinline__ int page(int half) const { return half ? page1 : page0; }
};

// Same answer in every role: the pipelines of all warps walk the same unit sequence.  With a
// CTA pair (CG = 2) a unit covers a 256-token tile; CTA ``crank`` owns its 128-token half.
// A unit exists when its first token is inside the sequence; the half may still be empty
// (nvalid = 0, no pages).
template <int CG>
__device__ __forceinline__ bool get_unit(const DecodeParams& p, int u, Unit& U, bool flag,
                                         int crank) {
  const int rg = u % p.n_ranges;
  const int rest = u / p.n_ranges;
  U.b = rest % p.batch;
  const int group_tile = rest / p.batch;
  U.tile = group_tile * CG + crank;
  int L = p.seq_lens[U.b];
  const int cap = p.max_pages * kPage;
  if (L > cap || L < 0) {
    if (flag && p.status) atomicOr(p.status, STARKV_DEV_BOUNDS);
    L = L < 0 ? 0 : cap;
  }
  U.L = L;
  if (group_tile * CG * kTile >= L) return false;
  U.c0 = rg * p.cpr;
  U.c1 = min(U.c0 + p.cpr, p.n_chunks);
  if (U.c0 >= U.c1) return false;
  U.nvalid = max(0, min(kTile, L - U.tile * kTile));
  int pgs[2];
#pragma unroll
  for (int pp = 0; pp < 2; ++pp) {
    int pg = -1;
    if (pp * kPage < U.nvalid) {
      pg = p.block_table[(long long)U.b * p.max_pages + U.tile * 2 + pp];
      if (pg < 0 || pg >= p.num_pages) {
        if (flag && p.status) atomicOr(p.status, STARKV_DEV_BOUNDS);
        pg = -1;
      }
    }
    pgs[pp] = pg;
  }
  U.page0 = pgs[0];
  U.page1 = pgs[1];
  return true;
}

__device__ __forceinline__ bool wait_drain(uint32_t bar, uint32_t parity, uint64_t timeout_ns) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > timeout_ns) return false;
  }
  return true;
}

template <int FMT>
struct Fmt {
  static constexpr bool kQuant = FMT == FMT_MIXED || FMT == FMT_HAD43;  // codes + fp16 scales
  static constexpr bool kTmaA = !kQuant;
  // fp32 operands: 3xTF32 (hi*hi + hi*lo + lo*hi), the hi/lo split done in shared memory
  static constexpr bool kSplit = FMT == FMT_F32;
  static constexpr int kKind = FMT == FMT_F32 ? 1 : 0;
  static constexpr int kElem = FMT == FMT_F32 ? 4 : 2;
  static constexpr int kKElems = kKBytes / kElem;  // elements per k-block
  static constexpr int kWarps = (kTmaA && !kSplit) ? 12 : 16;
  static constexpr int kFullCount = kSplit ? 4 : (kTmaA ? 1 : 5);
};

// One value-latent channel of one KV head in a staged page slot, with everything that does
// not depend on the token hoisted: byte offset and token stride of its code (or value), and
// for int8/int4 its scale's offset/stride, the nibble shift and whether it is an int8 channel.
struct VChan {
  int off, stride;
  int soff, sstride;
  int lsh, rsh;  // signed code = (w << lsh) >> rsh: int8 (24, 24), low / high nibble (28 / 24, 28),
                 // 3-bit field at bit b of a little-endian byte pair (29 - b, 29)
  int two;       // had43 3-bit channel: the code's bits may reach into the next byte
};

template <int FMT>
__device__ __forceinline__ VChan vchan(const LatDesc& vd, int vbase, int i) {
  VChan v{};
  if constexpr (FMT == FMT_F32) {
    v.off = vd.off0 - vbase + 4 * i;
    v.stride = 4 * vd.rank;
  } else if constexpr (FMT == FMT_BF16) {
    v.off = vd.off0 - vbase + 2 * i;
    v.stride = 2 * vd.rank;
  } else if constexpr (FMT == FMT_HAD43) {
    // 4-bit channels [0, n8) two per byte (pitch bytes per token); 3-bit channels eight per
    // 3-byte word, code j at bits [3 (j mod 8), +3) of word j / 8 (nb4 bytes per token)
    const bool hi = i < vd.n8;
    const int j = i - vd.n8;
    const int bit = 3 * (j & 7);
    v.off = hi ? vd.off0 - vbase + (i >> 1) : vd.off1 - vbase + 3 * (j >> 3) + (bit >> 3);
    v.stride = hi ? vd.pitch : vd.nb4;
    v.lsh = hi ? ((i & 1) ? 24 : 28) : 29 - (bit & 7);
    v.rsh = hi ? 28 : 29;
    v.two = hi ? 0 : ((bit & 7) > 5);
    v.soff = vd.off2 - vbase + 2 * (hi ? (i >> 5) : vd.g8 + (j >> 5));
    v.sstride = 2 * vd.ng;
  } else {
    const bool is8 = i < vd.n8;
    const int j = i - vd.n8;
    v.off = is8 ? vd.off0 - vbase + i : vd.off1 - vbase + (j >> 1);
    v.stride = is8 ? vd.n8 : vd.nb4;
    v.lsh = is8 ? 24 : ((j & 1) ? 24 : 28);
    v.rsh = is8 ? 24 : 28;
    v.soff = vd.off2 - vbase + 2 * (is8 ? (i >> 5) : vd.g8 + (j >> 5));
    v.sstride = 2 * vd.ng;
  }
  return v;
}

template <int FMT>
__device__ __forceinline__ float vchan_load(const uint8_t* slot, const VChan& v, int row) {
  if constexpr (FMT == FMT_F32) {
    return *reinterpret_cast<const float*>(slot + v.off + row * v.stride);
  } else if constexpr (FMT == FMT_BF16) {
    return __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(slot + v.off + row * v.stride));
  } else {
    unsigned b = slot[v.off + row * v.stride];
    if constexpr (FMT == FMT_HAD43) {
      if (v.two) b |= static_cast<unsigned>(slot[v.off + 1 + row * v.stride]) << 8;
    }
    const int q = static_cast<int>(b << v.lsh) >> v.rsh;
    const float s = __half2float(*reinterpret_cast<const __half*>(slot + v.soff + row * v.sstride));
    // q as a float without the conversion unit: 1.5 * 2^23 + q has an ulp of 1, so its bits
    // are those of 1.5 * 2^23 plus q, and one subtraction leaves q exactly
    return s * (__int_as_float(0x4B400000 + q) - 12582912.0f);
  }
}

// The G probabilities of one token for one GQA group (contiguous in the token-major layout).
template <int G>
__device__ __forceinline__ void load_p(const float* ptr, float (&out)[G]) {
  if constexpr (G % 4 == 0) {
#pragma unroll
    for (int k = 0; k < G; k += 4) {
      const float4 v = *reinterpret_cast<const float4*>(ptr + k);
      out[k] = v.x;
      out[k + 1] = v.y;
      out[k + 2] = v.z;
      out[k + 3] = v.w;
    }
  } else if constexpr (G == 2) {
    const float2 v = *reinterpret_cast<const float2*>(ptr);
    out[0] = v.x;
    out[1] = v.y;
  } else {
#pragma unroll
    for (int k = 0; k < G; ++k) out[k] = ptr[k];
  }
}

// Key-latent channel k of token row ``prow`` as the exact fp32 product scale * code.  ``base``
// is the page (or a copy of its key blocks with the offsets rebased).
template <bool H43>
__device__ __forceinline__ float key_code_value(const uint8_t* base, const LatDesc& kd, int prow,
                                                int k) {
  const __half* sc = reinterpret_cast<const __half*>(base + kd.off2) + prow * kd.ng;
  if constexpr (H43) {
    if (k < kd.n8) {  // 4-bit: two codes per byte
      const uint8_t byte = (base + kd.off0)[prow * kd.pitch + (k >> 1)];
      const int nib = (k & 1) ? (byte >> 4) : (byte & 15);
      return __half2float(sc[k >> 5]) * static_cast<float>((nib ^ 8) - 8);
    }
    // 3-bit: code j at bits [3 (j mod 8), +3) of the 3-byte word j / 8
    const int j = k - kd.n8;
    const int bit = 3 * (j & 7);
    const uint8_t* w = base + kd.off1 + prow * kd.nb4 + 3 * (j >> 3) + (bit >> 3);
    const unsigned pair = w[0] | (static_cast<unsigned>(w[1]) << 8);
    const int f = static_cast<int>((pair >> (bit & 7)) & 7u);
    return __half2float(sc[kd.g8 + (j >> 5)]) * static_cast<float>((f ^ 4) - 4);
  }
  if (k < kd.n8) {
    const int8_t q = reinterpret_cast<const int8_t*>(base + kd.off0)[prow * kd.n8 + k];
    return __half2float(sc[k >> 5]) * static_cast<float>(q);
  }
  const int j = k - kd.n8;
  const uint8_t byte = (base + kd.off1)[prow * kd.nb4 + (j >> 1)];
  const int nib = (j & 1) ? (byte >> 4) : (byte & 15);
  return __half2float(sc[kd.g8 + (j >> 5)]) * static_cast<float>((nib ^ 8) - 8);
}

__device__ __forceinline__ uint32_t pack_h2(float a, float b) {
  __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ __half2 bits_h2(uint32_t u) {
  __half2 h;
  memcpy(&h, &u, 4);
  return h;
}
__device__ __forceinline__ uint32_t h2_bits(__half2 h) {
  uint32_t u;
  memcpy(&u, &h, 4);
  return u;
}

// Channels [k0, k0+8) of token row ``prow`` of a page whose key blocks are at ``base`` + the
// offsets of ``kd`` (the page itself in global memory, or a copy of its key region in shared
// memory with the offsets rebased), one channel at a time: the ragged edges of the int8 and
// int4 parts.
template <bool H43>
__device__ __forceinline__ uint4 dequant8_at(const uint8_t* base, const LatDesc& kd, int prow, int k0) {
  float v[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const int k = k0 + e;
    v[e] = k < kd.rank ? key_code_value<H43>(base, kd, prow, k) : 0.f;
  }
  return make_uint4(pack_h2(v[0], v[1]), pack_h2(v[2], v[3]), pack_h2(v[4], v[5]),
                    pack_h2(v[6], v[7]));
}

// Channels [k0, k0+8) of the 8 tile rows r = row0 + 16 it (it < 8), as fp16 into the
// 128-byte-swizzled operand stage at shared address ``dst`` (row0 < 16, so rows it < 4 lie on
// the tile's first page).  ``key_base(it, r)`` gives the key blocks of row r's page: a 32-bit shared address (``kNoRow`` for a row past the sequence or
// on a missing page) when SMEM, else a global pointer (nullptr for such a row); those rows are
// stored as zeros.  All code loads are issued before the first store: the stores go to shared
// memory, so the compiler could not move a later row's load above an earlier row's store.
constexpr uint32_t kNoRow = 0xFFFFFFFFu;

// The 32-bit word of the codes at byte address ``a`` (any alignment), from the two aligned words
// that cover it; the bytes past the codes lie inside the page's blocks (the next block or the
// scales follow every code block).
template <bool SMEM>
__device__ __forceinline__ uint32_t word_at(uint32_t a_smem, const uint8_t* a_glob) {
  if constexpr (SMEM) {
    const uint32_t al = a_smem & ~3u;
    return __funnelshift_r(ld_shared_u32(al), ld_shared_u32(al + 4), (a_smem & 3u) * 8u);
  } else {
    const uintptr_t ga = reinterpret_cast<uintptr_t>(a_glob);
    const uint32_t* al = reinterpret_cast<const uint32_t*>(ga & ~static_cast<uintptr_t>(3));
    return __funnelshift_r(al[0], al[1], static_cast<uint32_t>(ga & 3u) * 8u);
  }
}

// had43 key channels [k0, k0+8) of 8 tile rows, as dequant_rows8 (below) does for int8/int4:
// inside the 4-bit block, nibbles as int4 codes (bias 8); inside the 3-bit block, the 8 codes
// of the group from a 48-bit window (their first code need not start a 3-byte word), each pair
// as exact fp16 under the exponent bits of 1024 with bias 4, times its group's fp16 scale
// (a group of 8 may straddle two 32-channel scale groups).  Returns false when the group
// straddles the 4-bit/3-bit boundary or the end of the latent (the caller's per-channel path).
template <bool SMEM, class BaseFn>
__device__ __forceinline__ bool dequant_rows8_h43(uint32_t dst, const LatDesc& kd, int k0, int ch,
                                                  int row0, BaseFn key_base, uint32_t safe) {
  const bool b4 = k0 + 8 <= kd.n8;
  const bool b3 = k0 >= kd.n8 && k0 + 8 <= kd.rank;
  if (!b4 && !b3) return false;
  const int j0 = k0 - kd.n8;
  const int sg0 = b4 ? (k0 >> 5) : kd.g8 + (j0 >> 5);  // scale group of the first code
  const int split = b4 ? 8 : min(8, 32 - (j0 & 31));      // codes before the next group
#pragma unroll 2
  for (int it = 0; it < 8; ++it) {
    const int r = row0 + 16 * it;
    const int prow = r & 63;
    const auto b = key_base(it, r);
    bool ok;
    uint32_t w0 = 0, w1 = 0;
    unsigned short s0 = 0, s1 = 0;
    if constexpr (SMEM) {
      ok = b != kNoRow;
      const uint32_t bs = ok ? b : safe;
      const uint32_t sa = bs + kd.off2 + 2 * (prow * kd.ng + sg0);
      s0 = ld_shared_u16(sa);
      s1 = split < 8 ? ld_shared_u16(sa + 2) : s0;
      if (b4) {
        w0 = word_at<true>(bs + kd.off0 + prow * kd.pitch + (k0 >> 1), nullptr);
      } else {
        const uint32_t a = bs + kd.off1 + prow * kd.nb4 + 3 * (j0 >> 3);
        w0 = word_at<true>(a, nullptr);
        w1 = word_at<true>(a + 4, nullptr);
      }
    } else {
      ok = b != nullptr;
      if (ok) {
        const unsigned short* sa = reinterpret_cast<const unsigned short*>(b + kd.off2) + prow * kd.ng + sg0;
        s0 = sa[0];
        s1 = split < 8 ? sa[1] : s0;
        if (b4) {
          w0 = word_at<false>(0, b + kd.off0 + prow * kd.pitch + (k0 >> 1));
        } else {
          const uint8_t* a = b + kd.off1 + prow * kd.nb4 + 3 * (j0 >> 3);
          w0 = word_at<false>(0, a);
          w1 = word_at<false>(0, a + 4);
        }
      }
    }
    if (!ok) { s0 = 0; s1 = 0; }
    uint4 z;
    if (b4) {
      // nibbles of the 4 bytes at k0/2: (n xor 8) = code + 8 under 0x64 -> 1032 + code
      const uint32_t raw = w0, hi = raw >> 4;
      const __half2 off = __half2half2(__ushort_as_half(0x6408));
      const __half2 s2 = __half2half2(__ushort_as_half(s0));
      z.x = h2_bits(__hmul2(__hsub2(bits_h2((__byte_perm(raw, hi, 0x0400) & 0x000F000Fu) ^ 0x64086408u), off), s2));
      z.y = h2_bits(__hmul2(__hsub2(bits_h2((__byte_perm(raw, hi, 0x0501) & 0x000F000Fu) ^ 0x64086408u), off), s2));
      z.z = h2_bits(__hmul2(__hsub2(bits_h2((__byte_perm(raw, hi, 0x0602) & 0x000F000Fu) ^ 0x64086408u), off), s2));
      z.w = h2_bits(__hmul2(__hsub2(bits_h2((__byte_perm(raw, hi, 0x0703) & 0x000F000Fu) ^ 0x64086408u), off), s2));
    } else {
      // the group's 24 bits: codes j0 .. j0+7 start at bit 3 (j0 mod 8) of the word pair
      const uint64_t win = (static_cast<uint64_t>(w1) << 32) | w0;
      const uint32_t c24 = static_cast<uint32_t>(win >> (3 * (j0 & 7)));
      const __half2 off = __half2half2(__ushort_as_half(0x6404));  // 1028
      uint32_t zz[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint32_t lo = (c24 >> (6 * q)) & 7u, hi = (c24 >> (6 * q + 3)) & 7u;
        const __half2 s2 = __halves2half2(__ushort_as_half(2 * q < split ? s0 : s1),
                                          __ushort_as_half(2 * q + 1 < split ? s0 : s1));
        zz[q] = h2_bits(__hmul2(__hsub2(bits_h2((lo | (hi << 16)) ^ 0x64046404u), off), s2));
      }
      z = make_uint4(zz[0], zz[1], zz[2], zz[3]);
    }
    st_shared_v4(dst + sw128_offset(r, ch), z);
  }
  return true;
}

template <bool SMEM, bool H43, class BaseFn>
__device__ __forceinline__ void dequant_rows8(uint32_t dst, const LatDesc& kd, int k0, int ch,
                                              int row0, BaseFn key_base, uint32_t safe = 0) {
  if constexpr (H43) {
    if (dequant_rows8_h43<SMEM>(dst, kd, k0, ch, row0, key_base, safe)) return;
  }
  const bool i8 = !H43 && k0 + 8 <= kd.n8 && (kd.n8 & 7) == 0;
  const bool i4 = !H43 && !i8 && k0 >= kd.n8 && ((k0 - kd.n8) & 7) == 0 && k0 + 8 <= kd.rank &&
                  (kd.nb4 & 3) == 0;
  if (i8 || i4) {
    const int j0 = k0 - kd.n8;
    const int coff = i8 ? kd.off0 + k0 : kd.off1 + (j0 >> 1);
    const int cpitch = i8 ? kd.n8 : kd.nb4;
    const int soff = kd.off2 + 2 * (i8 ? (k0 >> 5) : kd.g8 + (j0 >> 5));
    uint32_t cx[8], cy[8];
    unsigned short sb[8];
#pragma unroll
    for (int it = 0; it < 8; ++it) {
      const int r = row0 + 16 * it;
      const int prow = r & 63;
      const auto b = key_base(it, r);
      cx[it] = 0u;
      cy[it] = 0u;
      sb[it] = 0;
      if constexpr (SMEM) {
        // branch-free (a missing row reads the readable address ``safe`` and gets scale 0):
        // loads under a branch per row were not batched and cost 2.3x here
        const bool ok = b != kNoRow;
        const uint32_t bs = ok ? b : safe;
        const uint32_t a = bs + coff + prow * cpitch;
        if (i8) {
          const uint2 raw = ld_shared_v2(a);
          cx[it] = raw.x;
          cy[it] = raw.y;
        } else {
          cx[it] = ld_shared_u32(a);
        }
        const unsigned short sv = ld_shared_u16(bs + soff + prow * 2 * kd.ng);
        sb[it] = ok ? sv : static_cast<unsigned short>(0);
      } else {
        if (b) {
          if (i8) {
            const uint2 raw = *reinterpret_cast<const uint2*>(b + coff + prow * cpitch);
            cx[it] = raw.x;
            cy[it] = raw.y;
          } else {
            cx[it] = *reinterpret_cast<const uint32_t*>(b + coff + prow * cpitch);
          }
          sb[it] = *reinterpret_cast<const unsigned short*>(b + soff + prow * 2 * kd.ng);
        }
      }
    }
    // In fp16 pairs: a code c becomes the fp16 value 1024 + (c + bias) by placing c + bias in
    // the mantissa under the exponent bits 0x64 (bias 128 for int8, 8 for int4), one
    // subtraction recovers c exactly, and one multiplication by the fp16 scale rounds s*c once
    // -- the value of rounding the exact fp32 product s*c to fp16.
#pragma unroll
    for (int it = 0; it < 8; ++it) {
      const __half2 s2 = __half2half2(__ushort_as_half(sb[it]));
      uint4 z;
      if (i8) {
        const uint32_t bx = cx[it] ^ 0x80808080u, by = cy[it] ^ 0x80808080u;
        const __half2 off = __half2half2(__ushort_as_half(0x6480));  // 1152
        z.x = h2_bits(__hmul2(__hsub2(bits_h2(__byte_perm(bx, 0x64646464u, 0x4140)), off), s2));
        z.y = h2_bits(__hmul2(__hsub2(bits_h2(__byte_perm(bx, 0x64646464u, 0x4342)), off), s2));
        z.z = h2_bits(__hmul2(__hsub2(bits_h2(__byte_perm(by, 0x64646464u, 0x4140)), off), s2));
        z.w = h2_bits(__hmul2(__hsub2(bits_h2(__byte_perm(by, 0x64646464u, 0x4342)), off), s2));
      } else {
        const uint32_t raw = cx[it], hi = raw >> 4;
        const __half2 off = __half2half2(__ushort_as_half(0x6408));  // 1032
        z.x = h2_bits(__hmul2(__hsub2(bits_h2((__byte_perm(raw, hi, 0x0400) & 0x000F000Fu) ^ 0x64086408u), off), s2));
        z.y = h2_bits(__hmul2(__hsub2(bits_h2((__byte_perm(raw, hi, 0x0501) & 0x000F000Fu) ^ 0x64086408u), off), s2));
        z.z = h2_bits(__hmul2(__hsub2(bits_h2((__byte_perm(raw, hi, 0x0602) & 0x000F000Fu) ^ 0x64086408u), off), s2));
        z.w = h2_bits(__hmul2(__hsub2(bits_h2((__byte_perm(raw, hi, 0x0703) & 0x000F000Fu) ^ 0x64086408u), off), s2));
      }
      st_shared_v4(dst + sw128_offset(row0 + 16 * it, ch), z);
    }
  } else {
    // ragged edges of the int8 / int4 parts, one channel at a time (generic accesses)
#pragma unroll 2
    for (int it = 0; it < 8; ++it) {
      const int r = row0 + 16 * it;
      const auto b = key_base(it, r);
      uint4 z = make_uint4(0, 0, 0, 0);
      if constexpr (SMEM) {
        if (b != kNoRow) z = dequant8_at<H43>(smem_generic(b), kd, r & 63, k0);
      } else {
        if (b) z = dequant8_at<H43>(b, kd, r & 63, k0);
      }
      st_shared_v4(dst + sw128_offset(r, ch), z);
    }
  }
}

template <int FMT>
__device__ __forceinline__ float qload(const void* q, long long idx) {
  if constexpr (FMT == FMT_F32) return reinterpret_cast<const float*>(q)[idx];
  else return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(q)[idx]);
}

}  // namespace

template <int FMT, int HD, int G, int CG, int RES>
__global__ void __launch_bounds__(Fmt<FMT>::kWarps * 32, 1)
    decode_split_kernel(const __grid_constant__ DecodeParams p,
                        const __grid_constant__ CUtensorMap tmA,
                        const __grid_constant__ CUtensorMap tmB) {
  using F = Fmt<FMT>;
  constexpr int HALF = HD / 2;

  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned base (SW128 tiles), by pointer arithmetic on the shared array so that the
  // compiler keeps the address space and emits shared-memory instructions for every access
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  static_assert(CG == 1 || !Fmt<FMT>::kSplit, "fp32 latents use single-CTA tiles");
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int S = p.stages, NVB = p.nvb;
  // CTA pair: this CTA's rank, and the pair's unit stream
  const int crank = CG == 2 ? static_cast<int>(cluster_ctarank()) : 0;
  const bool leader = crank == 0;
  const int unit0 = blockIdx.x / CG, unit_step = gridDim.x / CG;
  // this CTA's B rows per k-block: the whole chunk, or its half of it in a pair
  const uint32_t bstage = static_cast<uint32_t>(p.NC / CG) * kKBytes;
  // stage strides: the split format keeps hi and lo copies of both operands
  const uint32_t astride = F::kSplit ? 2 * kAStage : kAStage;
  const uint32_t bstride = F::kSplit ? 2 * bstage : bstage;

  uint8_t* sA = smem;
  uint8_t* sB = smem + p.off_b;
  uint8_t* sV = smem + p.off_v;
  // epilogue scratch; QPC = query heads of a 256-column chunk
  float* sQ = reinterpret_cast<float*>(smem + p.off_q);        // [QPC][HD] rotated queries
  float* sP = reinterpret_cast<float*>(smem + p.off_p);        // [QPC][128] probabilities
  float* sPart = reinterpret_cast<float*>(smem + p.off_part);  // [2][QPC][128] partial scores
  float* sRed = reinterpret_cast<float*>(smem + p.off_red);    // [2][2][QPC][4] reductions
  float* sAng = reinterpret_cast<float*>(smem + p.off_ang);    // [2][HALF] theta_j, phi_j
  float* sPV = reinterpret_cast<float*>(smem + p.off_pv);      // [2][G][128] P.C_v partials
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + p.off_bar);
  const int B_FULL = 0, B_EMPTY = S, B_RAW = 2 * S, B_ACCF = 3 * S, B_ACCE = 3 * S + 2,
            B_VF = 3 * S + 4, B_VE = 3 * S + 4 + NVB, B_TD = 3 * S + 4 + 2 * NVB;
  // resident operand (int8/int4 keys of rank <= 256): dequantised once per tile into kb_count
  // slots, each used by every chunk of the unit; the tile's codes are staged by bulk copy
  const int B_AF = B_TD + 1, B_AE = B_AF + 4, B_CF = B_AE + 4, B_CE = B_CF + 2;
  // int8/int4 keys: RES 1 = operand dequantised once per tile and kept resident (rank <= 256);
  // RES 2 = the tile's codes staged in shared memory, operand streamed per ring stage; RES 0 =
  // operand streamed from the codes in global memory
  constexpr bool ares = RES == 1;
  constexpr bool staged = RES != 0;
  constexpr int NCB = RES == 1 ? 2 : 1;  // code buffers
  uint8_t* sCodes = smem + p.off_codes;  // [NCB buffers][2 pages][key_region]
  // misc: [0] TMEM base, [1] abort flag, [2..3] per-warpgroup stop snapshots
  uint32_t* misc = reinterpret_cast<uint32_t*>(bars + B_CE + 2);
  auto bar = [&](int i) { return smem_u32(bars + i); };

  if (threadIdx.x == 0) {
    // a pair's full barriers (in the leader) count both CTAs' producers and dequantisers;
    // its accumulator-empty barriers count the epilogue warps of both CTAs
    for (int s = 0; s < S; ++s) {
      // the resident operand is not part of a ring stage: only the producers arrive
      const int full = ares ? CG : (CG == 1 ? F::kFullCount : (F::kTmaA ? 2 : 10));
      mbar_init(bar(B_FULL + s), full);
      mbar_init(bar(B_EMPTY + s), 1);
      mbar_init(bar(B_RAW + s), 1);
    }
    for (int k = 0; k < 4; ++k) {
      mbar_init(bar(B_AF + k), 4 * CG);
      mbar_init(bar(B_AE + k), 1);
    }
    for (int k = 0; k < 2; ++k) {
      mbar_init(bar(B_CF + k), 1);
      mbar_init(bar(B_CE + k), 4);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(bar(B_ACCF + a), 1);
      mbar_init(bar(B_ACCE + a), 8 * CG);
    }
    for (int v = 0; v < NVB; ++v) {
      mbar_init(bar(B_VF + v), 1);
      mbar_init(bar(B_VE + v), 8);
    }
    mbar_init(bar(B_TD), 1);
    misc[1] = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmB);
    if constexpr (F::kTmaA) prefetch_tmap(&tmA);
  }
  if (warp == 1) {
    if constexpr (CG == 2) {
      tmem_alloc_pair(smem_u32(misc), 512);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(smem_u32(misc), 512);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  if constexpr (CG == 2)
    cluster_sync_all();  // both CTAs' barriers exist before any cross-CTA arrive or copy
  else
    __syncthreads();
  tc_fence_after();
  pdl_wait();
  pdl_launch_dependents();
  const uint32_t tmem = misc[0];
  // the pair's MMA-side barriers live in the leader CTA
  auto leader_bar = [&](int i) { return CG == 2 ? mapa_shared(bar(i), 0) : bar(i); };
  WaitCtl wc{reinterpret_cast<volatile int*>(misc + 1), p.status, p.timeout_ns};

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0, issued = 0, last_phase = 0;
      bool ok = true;
      for (int u = unit0; ok && u < p.total_units; u += unit_step) {
        Unit U;
        if (!get_unit<CG>(p, u, U, true, crank)) continue;
        for (int c = U.c0; ok && c < U.c1; ++c) {
          for (int kb = 0; kb < p.kb_count; ++kb) {
            if (!wait_bounded(bar(B_EMPTY + stage), phase ^ 1u, wc)) { ok = false; break; }
            uint32_t bytes = bstage;
            if constexpr (F::kTmaA)
              bytes += (U.page0 >= 0 ? 8192u : 0u) + (U.page1 >= 0 ? 8192u : 0u);
            const uint32_t da = smem_u32(sA + stage * astride);
            const uint32_t db = smem_u32(sB + stage * bstride);
            const int brow = c * p.NC + crank * (p.NC / CG);
            if constexpr (CG == 2) {
              // both CTAs' bytes complete the leader's full barrier
              const uint32_t fb = leader_bar(B_FULL + stage);
              if (leader)
                mbar_arrive_expect_tx(bar(B_FULL + stage), bytes);
              else
                mbar_arrive_expect_tx_cluster(fb, bytes);
              if constexpr (F::kTmaA) {
                if (U.page0 >= 0) tma_load_3d_pair(da, &tmA, fb, kb * F::kKElems, 0, U.page0);
                if (U.page1 >= 0) tma_load_3d_pair(da + 8192, &tmA, fb, kb * F::kKElems, 0, U.page1);
              }
              tma_load_2d_pair(db, &tmB, fb, kb * F::kKElems, brow);
            } else {
              // the split format lands raw fp32 tiles that the converters turn into hi/lo
              const uint32_t fb = bar((F::kSplit ? B_RAW : B_FULL) + stage);
              mbar_arrive_expect_tx(fb, bytes);
              if constexpr (F::kTmaA) {
                if (U.page0 >= 0) tma_load_3d(da, &tmA, fb, kb * F::kKElems, 0, U.page0);
                if (U.page1 >= 0) tma_load_3d(da + 8192, &tmA, fb, kb * F::kKElems, 0, U.page1);
              }
              tma_load_2d(db, &tmB, fb, kb * F::kKElems, brow);
            }
            issued |= 1u << stage;
            last_phase = (last_phase & ~(1u << stage)) | (phase << stage);
            if (++stage == S) { stage = 0; phase ^= 1u; }
          }
        }
      }
      // every copy this thread started has landed before the CTA may exit: the leader's
      // full barriers see both CTAs' bytes; after an abort the other CTA of a pair, which
      // cannot wait on them, gives its copies a fixed grace period instead
      if (CG == 1 || leader) {
        for (int s = 0; s < S; ++s)
          if (issued & (1u << s))
            wait_drain(bar((F::kSplit ? B_RAW : B_FULL) + s), (last_phase >> s) & 1u, p.timeout_ns);
      } else if (!ok) {
        const uint64_t t0 = globaltimer_ns();
        while (globaltimer_ns() - t0 < 200000ull) {
        }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0 && leader) {
      int stage = 0, ab = 0;
      uint32_t phase = 0, aph = 0, uc = 0;
      bool ok = true;
      for (int u = unit0; ok && u < p.total_units; u += unit_step) {
        Unit U;
        if (!get_unit<CG>(p, u, U, false, crank)) continue;
        ++uc;
        for (int c = U.c0; ok && c < U.c1; ++c) {
          if (!wait_bounded(bar(B_ACCE + ab), aph ^ 1u, wc)) { ok = false; break; }
          tc_fence_after();
          const uint32_t d_tmem = tmem + static_cast<uint32_t>(ab * 256);
          for (int kb = 0; kb < p.kb_count; ++kb) {
            if (ares && c == U.c0 &&
                !wait_bounded(bar(B_AF + kb), (uc - 1) & 1u, wc)) { ok = false; break; }
            if (!wait_bounded(bar(B_FULL + stage), phase, wc)) { ok = false; break; }
            tc_fence_after();
            const uint64_t da = desc_sw128(smem_u32(sA + (ares ? kb : stage) * astride));
            const uint64_t db = desc_sw128(smem_u32(sB + stage * bstride));
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              if constexpr (CG == 2) {
                umma_f16_pair(d_tmem, da + 2 * k, db + 2 * k, p.idesc, (kb | k) != 0);
              } else {
                umma<F::kKind>(d_tmem, da + 2 * k, db + 2 * k, p.idesc, (kb | k) != 0);
                if constexpr (F::kSplit) {
                  const uint64_t dal = desc_sw128(smem_u32(sA + stage * astride + kAStage));
                  const uint64_t dbl = desc_sw128(smem_u32(sB + stage * bstride + bstage));
                  umma<F::kKind>(d_tmem, da + 2 * k, dbl + 2 * k, p.idesc, 1u);
                  umma<F::kKind>(d_tmem, dal + 2 * k, db + 2 * k, p.idesc, 1u);
                }
              }
            }
            // the stage is free in both CTAs once these MMAs have read it; a resident slot
            // once the unit's last chunk has
            if constexpr (CG == 2) {
              umma_commit_pair(bar(B_EMPTY + stage), 3);
              if (ares && c + 1 == U.c1) umma_commit_pair(bar(B_AE + kb), 3);
            } else {
              umma_commit(bar(B_EMPTY + stage));
              if (ares && c + 1 == U.c1) umma_commit(bar(B_AE + kb));
            }
            if (++stage == S) { stage = 0; phase ^= 1u; }
          }
          if (!ok) break;
          if constexpr (CG == 2)
            umma_commit_pair(bar(B_ACCF + ab), 3);
          else
            umma_commit(bar(B_ACCF + ab));
          ab ^= 1;
          if (ab == 0) aph ^= 1u;
        }
      }
      if constexpr (CG == 2)
        umma_commit_pair(bar(B_TD), 1);
      else
        umma_commit(bar(B_TD));
      wait_drain(bar(B_TD), 0, p.timeout_ns);
    }
    __syncwarp();
  } else if (warp == 2) {
    // ---------------------------------------------------------------- value-latent producer
    if (lane == 0) {
      int vs = 0;
      uint32_t vph = 0, issued = 0, last_phase = 0;
      bool ok = true;
      for (int u = unit0; ok && u < p.total_units; u += unit_step) {
        Unit U;
        if (!get_unit<CG>(p, u, U, false, crank)) continue;
        for (int c = U.c0; c < U.c1; ++c) {
          if (!wait_bounded(bar(B_VE + vs), vph ^ 1u, wc)) { ok = false; break; }
          const uint32_t nbytes = static_cast<uint32_t>(p.vchunk_bytes[c]);
          const uint32_t fb = bar(B_VF + vs);
          mbar_arrive_expect_tx(fb, nbytes * ((U.page0 >= 0) + (U.page1 >= 0)));
          for (int pp = 0; pp < 2; ++pp) {
            const int pg = U.page(pp);
            if (pg < 0) continue;
            const uint8_t* src = p.cache + (long long)pg * p.page_bytes + p.vchunk_off[c];
            bulk_g2s(smem_u32(sV + (vs * 2 + pp) * p.vslot), src, nbytes, fb);
          }
          issued |= 1u << vs;
          last_phase = (last_phase & ~(1u << vs)) | (vph << vs);
          if (++vs == NVB) { vs = 0; vph ^= 1u; }
        }
      }
      for (int v = 0; v < NVB; ++v)
        if (issued & (1u << v)) wait_drain(bar(B_VF + v), (last_phase >> v) & 1u, p.timeout_ns);
    }
  } else if (warp == 3) {
    // ---------------------------------------------------------------- key-code stager
    if (staged && lane == 0) {
      const uint32_t kreg = static_cast<uint32_t>(p.key_region);
      int cb = 0;
      uint32_t cph = 0, issued = 0, last_phase = 0;
      for (int u = unit0; u < p.total_units; u += unit_step) {
        Unit U;
        if (!get_unit<CG>(p, u, U, false, crank)) continue;
        if (!wait_bounded(bar(B_CE + cb), cph ^ 1u, wc)) break;
        const uint32_t fb = bar(B_CF + cb);
        mbar_arrive_expect_tx(fb, kreg * ((U.page0 >= 0) + (U.page1 >= 0)));
        for (int pp = 0; pp < 2; ++pp) {
          const int pg = U.page(pp);
          if (pg < 0) continue;
          bulk_g2s(smem_u32(sCodes + (cb * 2 + pp) * kreg),
                   p.cache + (long long)pg * p.page_bytes + p.key.off0, kreg, fb);
        }
        issued |= 1u << cb;
        last_phase = (last_phase & ~(1u << cb)) | (cph << cb);
        if (++cb == NCB) { cb = 0; cph ^= 1u; }
      }
      for (int k = 0; k < 2; ++k)
        if (issued & (1u << k)) wait_drain(bar(B_CF + k), (last_phase >> k) & 1u, p.timeout_ns);
    }
  } else if (warp >= 4 && warp < 12) {
    // ---------------------------------------------------------------- epilogue warpgroups
    // Thread = token row (its TMEM lane).  Scores: warpgroup w rotates and dots the RoPE
    // pairs [w*JW, (w+1)*JW) of every KV head of the chunk, so each angle's sine and cosine is
    // computed once per row; the two partial scores meet in shared memory.  Softmax and the
    // latent P.C_v: warpgroup w owns half of the chunk's KV heads.
    constexpr int HPC = 256 / HD;  // KV heads in a full 256-column chunk
    constexpr int QPC = HPC * G;   // their query heads
    constexpr int JW = HALF / 2;   // RoPE pairs per warpgroup
    constexpr int JG = 8;          // pairs per step (one 8-column TMEM load per half)
    constexpr int NSTEP = (JW / JG) * HPC;
    const int wg = (warp - 4) >> 2;
    const int quad = warp & 3;          // TMEM lane quadrant of this warp
    const int row = quad * 32 + lane;   // token row in the tile == thread index in the WG
    const int et = wg * 128 + row;      // thread index over both warpgroups
    const int hpc = p.NC / HD;          // KV heads per chunk in this launch (NC may be 128)
    const int own_n = (hpc + 1) / 2;    // head slots whose softmax this warpgroup does
    const int own0 = wg * own_n;
    const float2* fine = p.rope;
    const float2* basetab = p.rope + kTile * HALF;
    // RoPE angles: theta_j (fixed) and the tile-start angle phi_j, both recovered from the
    // fp64-built table; a row's angle phi_j + r*theta_j stays below pi + 128, where the SFU
    // sine/cosine error is ~1e-5 rad -- no per-element table reads
    float* theta_s = sAng;
    float* phi_s = sAng + HALF;
    float* red = sRed + wg * 2 * QPC * 4;
    float* pv = sPV + wg * G * kTile;
    int* s_stop = reinterpret_cast<int*>(misc + 2);
    for (int j = et; j < HALF; j += 256) {
      const float2 f1 = fine[HALF + j];  // row 1: angle theta_j
      theta_s[j] = atan2f(f1.y, f1.x);
    }
    const float rowf = static_cast<float>(row);
    int ab = 0, vs = 0;
    uint32_t aph = 0, vph = 0;
    // Control flow of the epilogue only changes on a snapshot every thread reads after a
    // barrier of both warpgroups, so no thread leaves while others wait at a barrier.
    bool stop = false;
    for (int u = unit0; !stop && u < p.total_units; u += unit_step) {
      Unit U;
      if (!get_unit<CG>(p, u, U, false, crank)) continue;
      const int T = U.L - 1;  // position of the decode query
      const bool rv = row < U.nvalid && U.page(row >> 6) >= 0;
      const bool has_rows = U.nvalid > 0;  // a pair's second half may lie past the end
      // queries of a chunk are loaded one chunk ahead (QI values per thread at most)
      constexpr int QI = (QPC * HALF + 255) / 256;
      float qx0[QI], qx1[QI];
      auto load_q = [&](int cc) {
#pragma unroll
        for (int k = 0; k < QI; ++k) {
          const int idx = et + 256 * k;
          const int hq = idx / HALF, j = idx % HALF;
          const int g = cc * hpc + hq / G;
          qx0[k] = qx1[k] = 0.f;
          if (idx < hpc * G * HALF && g < p.Hkv) {
            const long long qb = ((long long)U.b * p.H + g * G + hq % G) * HD;
            qx0[k] = qload<FMT>(p.q, qb + j);
            qx1[k] = qload<FMT>(p.q, qb + j + HALF);
          }
        }
      };
      load_q(U.c0);
      // rotation of the query at position T: the same for every head and chunk (a thread's
      // pair index et % HALF does not depend on k, 256 being a multiple of HALF)
      float qcs, qsn;
      {
        const int j = et % HALF;
        const float2 bs = basetab[(T >> 7) * HALF + j], f = fine[(T & 127) * HALF + j];
        qcs = (bs.x * f.x - bs.y * f.y) * p.qscale;
        qsn = (bs.y * f.x + bs.x * f.y) * p.qscale;
      }
      for (int c = U.c0; c < U.c1; ++c) {
        const int g0 = c * hpc;  // first KV head of the chunk
        // (1) rotated, scaled queries of every head of the chunk; the tile's start angles
#pragma unroll
        for (int k = 0; k < QI; ++k) {
          const int idx = et + 256 * k;
          const int hq = idx / HALF, j = idx % HALF;
          if (idx < hpc * G * HALF) {
            sQ[hq * HD + j] = qx0[k] * qcs - qx1[k] * qsn;
            sQ[hq * HD + j + HALF] = qx1[k] * qcs + qx0[k] * qsn;
          }
        }
        if (c == U.c0) {
          for (int j = et; j < HALF; j += 256) {
            const float2 bs = basetab[min(U.tile, p.rope_tiles - 1) * HALF + j];
            phi_s[j] = atan2f(bs.y, bs.x);
          }
        }
        named_bar(1, 256);
        if (c + 1 < U.c1) load_q(c + 1);  // in flight while the accumulator is computed
        // (2) accumulator of this chunk (on a timeout the data is garbage and the snapshot
        // below ends the loop)
        wait_bounded(bar(B_ACCF + ab), aph, wc);
        tc_fence_after();
        // (3) partial scores over this warpgroup's pairs, every head; TMEM loads pipelined
        float sc[QPC];
#pragma unroll
        for (int i = 0; i < QPC; ++i) sc[i] = 0.f;
        {
          const uint32_t tbase = tmem + static_cast<uint32_t>(ab * 256) +
                                 (static_cast<uint32_t>(quad * 32) << 16);
          const int jw0 = wg * JW;
          uint32_t kb[2][16];
          float cs[JG], sn[JG];
          tmem_ld8x2(tbase + jw0, tbase + jw0 + HALF, kb[0]);
#pragma unroll
          for (int st = 0; st < NSTEP; ++st) {
            const int jg = st / HPC, sl = st % HPC;
            const int j0 = jw0 + jg * JG;
            tmem_wait_regs16(kb[st & 1]);
            if (st + 1 < NSTEP) {
              const int jn = jw0 + ((st + 1) / HPC) * JG, sn1 = (st + 1) % HPC;
              tmem_ld8x2(tbase + sn1 * HD + jn, tbase + sn1 * HD + jn + HALF, kb[(st + 1) & 1]);
            }
            if (sl == 0) {
#pragma unroll
              for (int e = 0; e < JG; e += 4) {
                const float4 th = *reinterpret_cast<const float4*>(theta_s + j0 + e);
                const float4 ph = *reinterpret_cast<const float4*>(phi_s + j0 + e);
                __sincosf(fmaf(rowf, th.x, ph.x), &sn[e + 0], &cs[e + 0]);
                __sincosf(fmaf(rowf, th.y, ph.y), &sn[e + 1], &cs[e + 1]);
                __sincosf(fmaf(rowf, th.z, ph.z), &sn[e + 2], &cs[e + 2]);
                __sincosf(fmaf(rowf, th.w, ph.w), &sn[e + 3], &cs[e + 3]);
              }
            }
            if (sl < hpc) {
              // rotated key pairs, two RoPE pairs per packed register pair:
              // k0 = a cos - b sin, k1 = b cos + a sin
              float2 k0[JG / 2], k1[JG / 2];
#pragma unroll
              for (int e = 0; e < JG; e += 2) {
                const float2 a = make_float2(__uint_as_float(kb[st & 1][e]),
                                             __uint_as_float(kb[st & 1][e + 1]));
                const float2 b = make_float2(__uint_as_float(kb[st & 1][JG + e]),
                                             __uint_as_float(kb[st & 1][JG + e + 1]));
                const float2 c2 = make_float2(cs[e], cs[e + 1]);
                const float2 s2 = make_float2(sn[e], sn[e + 1]);
                const float2 ns2 = make_float2(-sn[e], -sn[e + 1]);
                k0[e / 2] = __ffma2_rn(b, ns2, __fmul2_rn(a, c2));
                k1[e / 2] = __ffma2_rn(a, s2, __fmul2_rn(b, c2));
              }
#pragma unroll
              for (int gq = 0; gq < G; ++gq) {
                const float* qq = sQ + (sl * G + gq) * HD + j0;
                float2 t0 = make_float2(0.f, 0.f), t1 = make_float2(0.f, 0.f);
#pragma unroll
                for (int e = 0; e < JG; e += 4) {
                  const float4 qa = *reinterpret_cast<const float4*>(qq + e);
                  const float4 qb = *reinterpret_cast<const float4*>(qq + HALF + e);
                  t0 = __ffma2_rn(k0[e / 2], make_float2(qa.x, qa.y), t0);
                  t1 = __ffma2_rn(k1[e / 2], make_float2(qb.x, qb.y), t1);
                  t0 = __ffma2_rn(k0[e / 2 + 1], make_float2(qa.z, qa.w), t0);
                  t1 = __ffma2_rn(k1[e / 2 + 1], make_float2(qb.z, qb.w), t1);
                }
                const float2 t = __fadd2_rn(t0, t1);
                sc[sl * G + gq] += t.x + t.y;
              }
            }
          }
        }
        // (4) release the accumulator (the loads have completed at their wait::ld)
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if (CG == 2 && !leader)
            mbar_arrive_remote(leader_bar(B_ACCE + ab));
          else
            mbar_arrive(bar(B_ACCE + ab));
        }
        ab ^= 1;
        if (ab == 0) aph ^= 1u;
        // (5) exchange the partial scores; abort snapshot for both warpgroups
#pragma unroll
        for (int i = 0; i < QPC; ++i) sPart[(wg * QPC + i) * kTile + row] = sc[i];
        if (et == 0) s_stop[0] = *wc.abort_flag;
        named_bar(1, 256);
        if (s_stop[0]) { stop = true; break; }
        // (6) softmax of the owned heads (log2 domain: scores carry log2(e)/sqrt(d));
        // probabilities stored token-major, [row][QPC], so one vector load serves a GQA group
        constexpr int OQ = ((HPC + 1) / 2) * G;  // owned query heads (upper bound)
        float scr[OQ], rx[OQ];
#pragma unroll
        for (int oq = 0; oq < OQ; ++oq) {
          const int hq = own0 * G + oq;
          const bool ok_h = oq < own_n * G && own0 + oq / G < hpc;
          scr[oq] = (rv && ok_h) ? sPart[hq * kTile + row] + sPart[(QPC + hq) * kTile + row]
                                 : -INFINITY;
          rx[oq] = scr[oq];
        }
        // warp maxima of all owned heads, the shuffles of different heads interleaved
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
#pragma unroll
          for (int oq = 0; oq < OQ; ++oq) rx[oq] = fmaxf(rx[oq], __shfl_xor_sync(0xffffffffu, rx[oq], o));
        }
        if (lane == 0) {
#pragma unroll
          for (int oq = 0; oq < OQ; ++oq) red[oq * 4 + quad] = rx[oq];
        }
        named_bar(2 + wg, 128);
#pragma unroll
        for (int oq = 0; oq < OQ; ++oq) {
          const float mxv = fmaxf(fmaxf(red[oq * 4 + 0], red[oq * 4 + 1]),
                                  fmaxf(red[oq * 4 + 2], red[oq * 4 + 3]));
          const float pe = rv && scr[oq] > -INFINITY ? exp2f(scr[oq] - mxv) : 0.f;
          // slots beyond this launch's heads per chunk belong to the other warpgroup
          if (oq < own_n * G && own0 + oq / G < hpc) sP[row * QPC + own0 * G + oq] = pe;
          rx[oq] = pe;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
#pragma unroll
          for (int oq = 0; oq < OQ; ++oq) rx[oq] += __shfl_xor_sync(0xffffffffu, rx[oq], o);
        }
        if (lane == 0) {
#pragma unroll
          for (int oq = 0; oq < OQ; ++oq) red[OQ * 4 + oq * 4 + quad] = rx[oq];
        }
        named_bar(2 + wg, 128);
        // (7) value latents of this chunk, then the latent P.C_v of the owned heads: thread
        // row = (token group tg, channel ch) with TG = 128 / r groups of consecutive tokens;
        // the TG partials of a channel meet in shared memory
        wait_bounded(bar(B_VF + vs), vph, wc);
        const uint8_t* vslot0 = sV + (vs * 2) * p.vslot;
        const int vbase = p.vchunk_off[c];
#pragma unroll
        for (int os = 0; os < (HPC + 1) / 2; ++os) {
          const int sl = own0 + os;
          const int g = g0 + sl;
          const bool live = os < own_n && sl < hpc && g < p.Hkv && has_rows;  // WG-uniform
          if (!live) continue;
          const LatDesc& vd = p.vh[g];
          const int r = max(vd.rank, 1);
          const int TG = kTile / min(r, kTile);
          const int ch = row % r, tg = row / r;
          const bool act = tg < TG && ch < vd.rank;
          const VChan vc = vchan<FMT>(vd, vbase, ch);
          constexpr int G2 = (G + 1) / 2;
          float2 a2[G2];
#pragma unroll
          for (int k = 0; k < G2; ++k) a2[k] = make_float2(0.f, 0.f);
          if (act) {
            const int tlo = (tg * kTile) / TG, thi = ((tg + 1) * kTile) / TG;
#pragma unroll
            for (int pp = 0; pp < 2; ++pp) {
              if (U.page(pp) < 0) continue;
              const uint8_t* slot = vslot0 + pp * p.vslot;
              const int t0 = max(tlo, pp * kPage);
              const int t1 = min(min(thi, pp * kPage + kPage), U.nvalid);
#pragma unroll 4
              for (int t = t0; t < t1; ++t) {
                const float cv = vchan_load<FMT>(slot, vc, t - pp * kPage);
                const float* pt = sP + t * QPC + sl * G;
                if constexpr (G == 1) {
                  a2[0].x = fmaf(pt[0], cv, a2[0].x);
                } else {
                  const float2 cv2 = make_float2(cv, cv);
                  float pr[G];
                  load_p<G>(pt, pr);
#pragma unroll
                  for (int k = 0; k < G2; ++k)
                    a2[k] = __ffma2_rn(make_float2(pr[2 * k], pr[2 * k + 1]), cv2, a2[k]);
                }
              }
            }
          }
#pragma unroll
          for (int gq = 0; gq < G; ++gq)
            pv[gq * kTile + row] = (gq & 1) ? a2[gq >> 1].y : a2[gq >> 1].x;
          named_bar(2 + wg, 128);
          // each (head, channel) output sums its TG partials, one output per thread
          for (int o = row; o < vd.rank * G; o += kTile) {
            const int gq = o / vd.rank, oc = o - gq * vd.rank;
            const float* src = pv + gq * kTile + oc;
            float s0 = 0.f, s1 = 0.f;
            int k = 0;
            for (; k + 2 <= TG; k += 2) {
              s0 += src[k * r];
              s1 += src[(k + 1) * r];
            }
            if (k < TG) s0 += src[k * r];
            const int h = g * G + gq;
            float* rec = p.ws + (((long long)U.b * p.H + h) * p.tiles_max + U.tile) * p.rec;
            rec[2 + oc] = s0 + s1;
          }
          if (row == 0) {
#pragma unroll
            for (int gq = 0; gq < G; ++gq) {
              const int oq = os * G + gq;
              const int h = g * G + gq;
              float* rec = p.ws + (((long long)U.b * p.H + h) * p.tiles_max + U.tile) * p.rec;
              rec[0] = fmaxf(fmaxf(red[oq * 4 + 0], red[oq * 4 + 1]), fmaxf(red[oq * 4 + 2], red[oq * 4 + 3]));
              rec[1] = red[OQ * 4 + oq * 4 + 0] + red[OQ * 4 + oq * 4 + 1] +
                       red[OQ * 4 + oq * 4 + 2] + red[OQ * 4 + oq * 4 + 3];
            }
          }
          // pv is reused by the next owned head; after the last one, the barriers of the next
          // chunk order these reads before the next writes
          if (os + 1 < (HPC + 1) / 2) named_bar(2 + wg, 128);
        }
        // (8) release the value buffer
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(B_VE + vs));
        if (++vs == NVB) { vs = 0; vph ^= 1u; }
      }
    }
  } else if (warp >= 12) {
    if constexpr (F::kSplit) {
      // ---------------------------------------------------------------- tf32 hi/lo splitters
      const int tid = (warp - 12) * 32 + lane;
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int u = unit0; ok && u < p.total_units; u += unit_step) {
        Unit U;
        if (!get_unit<CG>(p, u, U, false, crank)) continue;
        for (int c = U.c0; ok && c < U.c1; ++c) {
          for (int kb = 0; kb < p.kb_count; ++kb) {
            if (!__all_sync(0xffffffffu, wait_bounded(bar(B_RAW + stage), phase, wc))) {
              ok = false;
              break;
            }
            uint8_t* a = sA + stage * astride;
            uint8_t* b = sB + stage * bstride;
            split_tf32(reinterpret_cast<float4*>(a), reinterpret_cast<float4*>(a + kAStage),
                       kAStage / 16, tid, 128);
            split_tf32(reinterpret_cast<float4*>(b), reinterpret_cast<float4*>(b + bstage),
                       static_cast<int>(bstage / 16), tid, 128);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(B_FULL + stage));
            if (++stage == S) { stage = 0; phase ^= 1u; }
          }
        }
      }
    }
    // ---------------------------------------------------------------- dequantisers (int8/int4)
    if constexpr (ares) {
      // once per tile, from the staged codes, into the resident slots
      const int tid = (warp - 12) * 32 + lane;
      const int ch = tid & 7;
      LatDesc kd = p.key;  // offsets rebased onto the staged key region
      kd.off1 -= kd.off0;
      kd.off2 -= kd.off0;
      kd.off0 = 0;
      const int kreg = p.key_region;
      int cb = 0;
      uint32_t cph = 0, uc = 0;
      bool ok = true;
      for (int u = unit0; ok && u < p.total_units; u += unit_step) {
        Unit U;
        if (!get_unit<CG>(p, u, U, false, crank)) continue;
        if (!__all_sync(0xffffffffu, wait_bounded(bar(B_CF + cb), cph, wc))) break;
        for (int kb = 0; kb < p.kb_count; ++kb) {
          if (!__all_sync(0xffffffffu, wait_bounded(bar(B_AE + kb), (uc & 1u) ^ 1u, wc))) {
            ok = false;
            break;
          }
          const uint32_t codes = smem_u32(sCodes) + static_cast<uint32_t>(cb * 2 * kreg);
          const uint32_t pb0 = U.page0 >= 0 ? codes : kNoRow;
          const uint32_t pb1 = U.page1 >= 0 ? codes + static_cast<uint32_t>(kreg) : kNoRow;
          dequant_rows8<true, FMT == FMT_HAD43>(smem_u32(sA + kb * kAStage), kd, kb * 64 + ch * 8, ch, tid >> 3,
                              [&](int it, int r) -> uint32_t {
                                return r < U.nvalid ? (it < 4 ? pb0 : pb1) : kNoRow;
                              }, codes);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            if constexpr (CG == 2)
              mbar_arrive_cluster(leader_bar(B_AF + kb));
            else
              mbar_arrive(bar(B_AF + kb));
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(B_CE + cb));
        ++uc;
        if (++cb == 2) { cb = 0; cph ^= 1u; }
      }
    } else if constexpr (!F::kTmaA) {
      // streamed operand, one ring stage per (chunk, k-block): from the tile's codes staged in
      // shared memory (RES 2) or from the pages in global memory (RES 0)
      const int tid = (warp - 12) * 32 + lane;
      const int ch = tid & 7;
      LatDesc kd = p.key;  // offsets rebased onto the staged key region
      kd.off1 -= kd.off0;
      kd.off2 -= kd.off0;
      kd.off0 = 0;
      const int kreg = p.key_region;
      int stage = 0;
      uint32_t phase = 0, cph = 0;
      bool ok = true;
      for (int u = unit0; ok && u < p.total_units; u += unit_step) {
        Unit U;
        if (!get_unit<CG>(p, u, U, false, crank)) continue;
        if constexpr (staged) {
          if (!__all_sync(0xffffffffu, wait_bounded(bar(B_CF), cph, wc))) break;
        }
        for (int c = U.c0; ok && c < U.c1; ++c) {
          for (int kb = 0; kb < p.kb_count; ++kb) {
            // warp-uniform decision (the __syncwarp below needs every lane)
            if (!__all_sync(0xffffffffu, wait_bounded(bar(B_EMPTY + stage), phase ^ 1u, wc))) {
              ok = false;
              break;
            }
            const uint32_t dst = smem_u32(sA + stage * kAStage);
            if constexpr (staged) {
              const uint32_t codes = smem_u32(sCodes);
              const uint32_t pb0 = U.page0 >= 0 ? codes : kNoRow;
              const uint32_t pb1 = U.page1 >= 0 ? codes + static_cast<uint32_t>(kreg) : kNoRow;
              dequant_rows8<true, FMT == FMT_HAD43>(dst, kd, kb * 64 + ch * 8, ch, tid >> 3,
                                  [&](int it, int r) -> uint32_t {
                                    return r < U.nvalid ? (it < 4 ? pb0 : pb1) : kNoRow;
                                  }, codes);
            } else {
              const uint8_t* gb0 = U.page0 >= 0 ? p.cache + (long long)U.page0 * p.page_bytes : nullptr;
              const uint8_t* gb1 = U.page1 >= 0 ? p.cache + (long long)U.page1 * p.page_bytes : nullptr;
              dequant_rows8<false, FMT == FMT_HAD43>(dst, p.key, kb * 64 + ch * 8, ch, tid >> 3,
                                   [&](int it, int r) -> const uint8_t* {
                                     return r < U.nvalid ? (it < 4 ? gb0 : gb1) : nullptr;
                                   });
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              if constexpr (CG == 2)
                mbar_arrive_cluster(leader_bar(B_FULL + stage));
              else
                mbar_arrive(bar(B_FULL + stage));
            }
            if (++stage == S) { stage = 0; phase ^= 1u; }
          }
        }
        if constexpr (staged) {
          // the staged codes may be overwritten once every chunk of the unit has used them
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(B_CE));
          cph ^= 1u;
        }
      }
    }
  }

  tc_fence_before();
  if constexpr (CG == 2) {
    // neither CTA leaves while the pair's MMAs may still read its shared memory or TMEM
    cluster_sync_all();
    tc_fence_after();
    if (warp == 1) tmem_dealloc_pair(tmem, 512);
  } else {
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, 512);
  }
}

// --------------------------------------------------------------------------- combine
// One CTA per (sequence, query head): merge the tile partials (m in log2 units, l, a[r]),
// normalise, then o = a B_v,g.
__global__ void __launch_bounds__(128) decode_combine_kernel(const __grid_constant__ DecodeParams p) {
  pdl_wait();
  pdl_launch_dependents();
  const int bh = blockIdx.x;
  const int b = bh / p.H, h = bh % p.H, g = h / p.G;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  __shared__ float s_m[4];
  __shared__ float s_acc[4][129];
  __shared__ float s_a[128];
  const LatDesc& vd = p.vh[g];
  const int r = vd.rank;
  float* outp = p.out + ((long long)b * p.H + h) * p.d;
  int L = p.seq_lens[b];
  L = max(0, min(L, p.max_pages * kPage));
  // merge mode: the normalised a_h goes to its rows in a_out (query heads of KV head g
  // are consecutive blocks of r_g rows after the rows of the heads of KV heads < g)
  float* a_row = p.a_out ? p.a_out + (long long)b * p.a_stride + p.G * (vd.col - p.key_rank_cols) +
                               (h % p.G) * r
                         : nullptr;
  if (L == 0) {
    if (a_row) {
      for (int i = tid; i < r; i += 128) a_row[i] = 0.f;
    } else {
      for (int c = tid; c < p.d; c += 128) outp[c] = 0.f;
    }
    return;
  }
  const int T = (L + kTile - 1) / kTile;
  const float* recs = p.ws + ((long long)b * p.H + h) * p.tiles_max * p.rec;
  float m = -INFINITY;
  for (int t = tid; t < T; t += 128) {
    const float* rc = recs + (long long)t * p.rec;
    if (rc[1] > 0.f) m = fmaxf(m, rc[0]);
  }
  m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 16));
  m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 8));
  m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 4));
  m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
  m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
  if (lane == 0) s_m[warp] = m;
  __syncthreads();
  const float M = fmaxf(fmaxf(s_m[0], s_m[1]), fmaxf(s_m[2], s_m[3]));
  // each warp takes every 4th tile, eight tiles per batch with all their loads issued first;
  // lanes cover the latent channels
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  float lsum = 0.f;
  for (int tb = warp; tb < T; tb += 32) {
    float mm[8], ll[8], vv[8][4];
#pragma unroll
    for (int jj = 0; jj < 8; ++jj) {
      const int t = tb + 4 * jj;
      const bool ok = t < T;
      const float* rc = recs + (long long)(ok ? t : tb) * p.rec;
      mm[jj] = ok ? rc[0] : 0.f;
      ll[jj] = ok ? rc[1] : 0.f;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int i = lane + 32 * k;
        vv[jj][k] = (ok && i < r) ? rc[2 + i] : 0.f;
      }
    }
#pragma unroll
    for (int jj = 0; jj < 8; ++jj) {
      // a tile without weight (none, or a garbage record) contributes nothing
      const float w = ll[jj] > 0.f ? exp2f(mm[jj] - M) : 0.f;
      if (w > 0.f) {
        lsum += ll[jj] * w;
#pragma unroll
        for (int k = 0; k < 4; ++k) acc[k] = fmaf(vv[jj][k], w, acc[k]);
      }
    }
  }
#pragma unroll
  for (int k = 0; k < 4; ++k) s_acc[warp][lane + 32 * k] = acc[k];
  if (lane == 0) s_acc[warp][128] = lsum;
  __syncthreads();
  const float l = s_acc[0][128] + s_acc[1][128] + s_acc[2][128] + s_acc[3][128];
  const float inv = l > 0.f ? 1.f / l : 0.f;
  s_a[tid] = tid < r ? (s_acc[0][tid] + s_acc[1][tid] + s_acc[2][tid] + s_acc[3][tid]) * inv : 0.f;
  if (a_row) {
    if (tid < r) a_row[tid] = s_a[tid];
    return;
  }
  __syncthreads();
  // o_c = sum_i a_i B_v[i][c], 32 rows of B_v in flight at a time (a_i = 0 for i >= r)
  const float* Bv = p.Bv + (long long)(vd.col - p.key_rank_cols) * p.d;
  for (int c = tid; c < p.d; c += 128) {
    float o0 = 0.f, o1 = 0.f;
    for (int i0 = 0; i0 < r; i0 += 32) {
      float bv[32];
#pragma unroll
      for (int k = 0; k < 32; ++k) bv[k] = i0 + k < r ? __ldg(Bv + (long long)(i0 + k) * p.d + c) : 0.f;
#pragma unroll
      for (int k = 0; k < 32; k += 2) {
        o0 = fmaf(s_a[i0 + k], bv[k], o0);
        o1 = fmaf(s_a[i0 + k + 1], bv[k + 1], o1);
      }
    }
    outp[c] = o0 + o1;
  }
}

// --------------------------------------------------------------------------- launchers
template <int FMT, int HD, int G, int CG, int RES>
static cudaError_t launch_one(const DecodeParams& p, const CUtensorMap& tmA,
                              const CUtensorMap& tmB, int grid, cudaStream_t s) {
  auto kern = decode_split_kernel<FMT, HD, G, CG, RES>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(p.smem_bytes));
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(Fmt<FMT>::kWarps * 32, 1, 1);
  cfg.dynamicSmemBytes = p.smem_bytes;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = CG;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  if (CG > 1) {
    // a persistent grid must be co-resident: not every SM can host half of a CTA pair
    // (pairs stay inside a GPC), so cap the grid at the pairs that fit at once
    int clusters = 0;
    e = cudaOccupancyMaxActiveClusters(&clusters, kern, &cfg);
    if (e != cudaSuccess) return e;
    if (clusters >= 1 && grid > clusters * CG) cfg.gridDim = dim3(clusters * CG, 1, 1);
  }
  return cudaLaunchKernelEx(&cfg, kern, p, tmA, tmB);
}

template <int FMT, int HD, int CG, int RES>
static cudaError_t launch_g(int G, const DecodeParams& p, const CUtensorMap& tmA,
                            const CUtensorMap& tmB, int grid, cudaStream_t s) {
  switch (G) {
    case 1: return launch_one<FMT, HD, 1, CG, RES>(p, tmA, tmB, grid, s);
    case 2: return launch_one<FMT, HD, 2, CG, RES>(p, tmA, tmB, grid, s);
    case 4: return launch_one<FMT, HD, 4, CG, RES>(p, tmA, tmB, grid, s);
    case 8: return launch_one<FMT, HD, 8, CG, RES>(p, tmA, tmB, grid, s);
    default: return cudaErrorInvalidValue;
  }
}

template <int FMT, int CG, int RES = 0>
static cudaError_t launch_hd(int hd, int G, const DecodeParams& p, const CUtensorMap& tmA,
                             const CUtensorMap& tmB, int grid, cudaStream_t s) {
  if (hd == 64) return launch_g<FMT, 64, CG, RES>(G, p, tmA, tmB, grid, s);
  if (hd == 128) return launch_g<FMT, 128, CG, RES>(G, p, tmA, tmB, grid, s);
  return cudaErrorInvalidValue;
}

cudaError_t launch_decode(int fmt, int head_dim, int G, const DecodeParams& p,
                          const CUtensorMap& tmA, const CUtensorMap& tmB, int grid,
                          cudaStream_t s) {
  const int res = (fmt == STARKV_FMT_MIXED || fmt == STARKV_FMT_HAD43) ? p.a_resident : 0;
  if (p.cta_group == 2) {
    switch (fmt) {
      case STARKV_FMT_BF16: return launch_hd<FMT_BF16, 2>(head_dim, G, p, tmA, tmB, grid, s);
      case STARKV_FMT_MIXED:
        return res == 1   ? launch_hd<FMT_MIXED, 2, 1>(head_dim, G, p, tmA, tmB, grid, s)
               : res == 2 ? launch_hd<FMT_MIXED, 2, 2>(head_dim, G, p, tmA, tmB, grid, s)
                          : launch_hd<FMT_MIXED, 2, 0>(head_dim, G, p, tmA, tmB, grid, s);
      case STARKV_FMT_HAD43:
        return res == 1   ? launch_hd<FMT_HAD43, 2, 1>(head_dim, G, p, tmA, tmB, grid, s)
               : res == 2 ? launch_hd<FMT_HAD43, 2, 2>(head_dim, G, p, tmA, tmB, grid, s)
                          : launch_hd<FMT_HAD43, 2, 0>(head_dim, G, p, tmA, tmB, grid, s);
      default: return cudaErrorInvalidValue;
    }
  }
  switch (fmt) {
    case STARKV_FMT_F32: return launch_hd<FMT_F32, 1>(head_dim, G, p, tmA, tmB, grid, s);
    case STARKV_FMT_BF16: return launch_hd<FMT_BF16, 1>(head_dim, G, p, tmA, tmB, grid, s);
    case STARKV_FMT_MIXED:
      return res == 1   ? launch_hd<FMT_MIXED, 1, 1>(head_dim, G, p, tmA, tmB, grid, s)
             : res == 2 ? launch_hd<FMT_MIXED, 1, 2>(head_dim, G, p, tmA, tmB, grid, s)
                        : launch_hd<FMT_MIXED, 1, 0>(head_dim, G, p, tmA, tmB, grid, s);
    case STARKV_FMT_HAD43:
      return res == 1   ? launch_hd<FMT_HAD43, 1, 1>(head_dim, G, p, tmA, tmB, grid, s)
             : res == 2 ? launch_hd<FMT_HAD43, 1, 2>(head_dim, G, p, tmA, tmB, grid, s)
                        : launch_hd<FMT_HAD43, 1, 0>(head_dim, G, p, tmA, tmB, grid, s);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_combine(const DecodeParams& p, cudaStream_t s) {
  return launch_pdl(decode_combine_kernel, dim3(p.batch * p.H), dim3(128), 0, s, p);
}

size_t decode_smem_limit() { return 232448; }

}  // namespace starkv
