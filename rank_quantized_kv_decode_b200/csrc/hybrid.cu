// Decode attention with the hybrid assignment of the STAR-KV technical summary (Methodology
// §2, "Hybrid Decomposition Strategy"): keys decomposed head-wise, values jointly.
//
// For query head h of KV head g:  K_g = C_k,g B_k,g (r_k,g x d per head, not r_k x H_kv d as
// with a joint key latent, so reconstruction costs H_kv times less), RoPE, scores, softmax,
// a_h = p C_v in the one joint value space (r_v wide), o_h = a_h B_v[:, g d : (g+1) d].
//
// Split kernel: one CTA per SM, looping over (sequence, page range) units.  Per 64-token page:
//   1. the page arrives by one bulk copy (all latents of its 64 tokens; the next page's copy
//      is issued as soon as this one has been decoded, so it overlaps the arithmetic);
//   2. int8/int4 codes become fp16 values (code x fp16 scale, rounded once) in shared memory:
//      per-head key operands [token][r_k,g] and the value operand [token][r_v];
//   3. warp w takes tokens [16 (w mod 4), +16) and every other KV head: K_g on the tensor cores
//      (mma.sync m16n8k16, fp16 operands, fp32 accumulation; B_k,g resident in shared
//      memory), RoPE on the accumulators in registers, then the scores on the tensor cores:
//      the accumulator fragments of two n-tiles are exactly the A fragment of one k-step, so
//      the rotated keys never leave the registers; each key and query value is split into
//      two fp16 parts (hi + lo) and three products keep the scores at fp32 accuracy;
//   4. online softmax per query head over the page (log2 domain), P as fp16;
//   5. a += P C_v on the tensor cores (the accumulators stay in registers across the range,
//      rescaled by exp2(m_old - m_new) per head).
// Each unit leaves one record per query head: m, l and a.  The combine kernel merges the
// records of a sequence (log-sum-exp) and applies B_v,g.
#include <cmath>

#include "internal.cuh"

namespace starkv {

namespace {

constexpr int kThreads = 256;
constexpr int kPvMax = 8;  // (head tile, channel tile) accumulators per warp

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x2_trans(uint32_t addr, uint32_t& r0, uint32_t& r1) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0,%1}, [%2];"
               : "=r"(r0), "=r"(r1)
               : "r"(addr));
}
// D (16x8 fp32) += A (16x16 fp16, row-major) * B (16x8 fp16, column-major).
__device__ __forceinline__ void mma_f16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                        uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t h2_bits(__half2 h) { return *reinterpret_cast<uint32_t*>(&h); }
__device__ __forceinline__ __half2 bits_h2(uint32_t u) { return *reinterpret_cast<__half2*>(&u); }

// (x0, x1) as fp16 pairs hi and lo with hi + lo = (x0, x1) to about 2^-22 relative.
__device__ __forceinline__ void split_h2(float x0, float x1, uint32_t& hi, uint32_t& lo) {
  const __half2 h = __floats2half2_rn(x0, x1);
  const float2 f = __half22float2(h);
  hi = h2_bits(h);
  lo = h2_bits(__floats2half2_rn(x0 - f.x, x1 - f.y));
}

// The page's latents as a list of quads (four channels [c, c + 4) of one latent; c is a
// multiple of 4, so a quad lies in one block and one scale group), one 16-byte entry each,
// built once per CTA:
//   x  source byte offset in the page for token 0 | kind << 28 (0 int8, 1 int4, 2 zeros)
//   y  source bytes per token | scale bytes per token << 16
//   z  scale byte offset in the page for token 0
//   w  destination byte offset in shared memory for token 0 | (row pitch / 16) << 20
constexpr int kQuadInt8 = 0, kQuadInt4 = 1, kQuadZero = 2;

__device__ __forceinline__ int4 quad_entry(const LatDesc& d, int c, int dst, int pitch) {
  int4 e;
  const int ng2 = 2 * d.ng;
  if (c >= d.rank) {
    e.x = kQuadZero << 28;
    e.y = 0;
    e.z = 0;
  } else if (c < d.n8) {
    e.x = (d.off0 + c) | (kQuadInt8 << 28);
    e.y = d.n8 | (ng2 << 16);
    e.z = d.off2 + 2 * (c >> 5);
  } else {
    const int c4 = c - d.n8;
    e.x = (d.off1 + (c4 >> 1)) | (kQuadInt4 << 28);
    e.y = d.nb4 | (ng2 << 16);
    e.z = d.off2 + 2 * (d.g8 + (c4 >> 5));
  }
  e.w = (dst + 2 * c) | ((pitch >> 4) << 20);
  return e;
}

// A quad's codes (an int8 word or an int4 half-word) as fp16 values code x scale, each
// rounded once.  Codes go to fp16 exactly through the exponent bias: a biased code u under
// the fp16 pattern 0x64uu is 1024 + u.
__device__ __forceinline__ uint2 dequant_codes(uint32_t w, int kind, __half s) {
  uint32_t lo, hi;
  __half2 bias;
  if (kind == kQuadInt8) {
    w ^= 0x80808080u;
    lo = __byte_perm(w, 0x64646464u, 0x5150);
    hi = __byte_perm(w, 0x64646464u, 0x5352);
    bias = bits_h2(0x64806480u);  // 1024 + 128
  } else {
    w ^= 0x8888u;
    lo = (w & 0xFu) | ((w & 0xF0u) << 12) | 0x64006400u;
    hi = ((w >> 8) & 0xFu) | ((w & 0xF000u) << 4) | 0x64006400u;
    bias = bits_h2(0x64086408u);  // 1024 + 8
  }
  const __half2 s2 = __half2half2(s);
  uint2 r;
  r.x = h2_bits(__hmul2(__hsub2(bits_h2(lo), bias), s2));
  r.y = h2_bits(__hmul2(__hsub2(bits_h2(hi), bias), s2));
  return r;
}

template <int HD, int MT>
__global__ void __launch_bounds__(kThreads, 1) hybrid_split_kernel(const __grid_constant__ HybridParams p) {
  extern __shared__ __align__(16) uint8_t smem[];
  constexpr int NT = HD / 8;    // n-tiles of one reconstructed head
  constexpr int HALF = HD / 2;  // RoPE pairs (j, j + d/2)
  constexpr int JN = HD / 16;   // n-tiles of the first half
  constexpr int QP = HD + 8;    // query row pitch (halves)
  constexpr int PP = 64 + 8;    // P row pitch (halves)
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gid = lane >> 2, tig = lane & 3;
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar = sbase + p.s_bar;
  float* sM = reinterpret_cast<float*>(smem + p.s_stat);
  float* sL = sM + p.hp;
  float* sAl = sL + p.hp;
  int* flags = reinterpret_cast<int*>(sAl + p.hp);  // [0] page copied, [1] page state
  float* sS = reinterpret_cast<float*>(smem + p.s_s);
  const int spitch = p.H + 4;
  __half* sQhi = reinterpret_cast<__half*>(smem + p.s_qhi);
  __half* sQlo = reinterpret_cast<__half*>(smem + p.s_qlo);
  __half* sP = reinterpret_cast<__half*>(smem + p.s_p);
  __half* sCv = reinterpret_cast<__half*>(smem + p.s_cv);
  const int cvp = p.rvp + 8;
  const uint8_t* page = smem + p.s_page;
  const float2* fine = p.rope;
  const float2* basetab = p.rope + kTile * HALF;

  // ---- once per CTA: the barrier, the resident key factors, the zero rows
  if (tid == 0) {
    mbar_init(bar, 1);
    fence_mbar_init();
  }
  for (int g = 0; g < p.Hkv; ++g) {
    const int r = p.key[g].rank, c8 = r >> 3;
    const uint4* src = reinterpret_cast<const uint4*>(p.Bk_t + p.bk_elem[g]);
    uint8_t* dst = smem + p.s_bk[g];
    for (int i = tid; i < HD * c8; i += kThreads) {
      const int n = i / c8, c = i - n * c8;
      *reinterpret_cast<uint4*>(dst + (n * (r + 8) + c * 8) * 2) = src[i];
    }
  }
  for (int i = tid; i < QP; i += kThreads) {
    sQhi[p.H * QP + i] = __float2half_rn(0.f);
    sQlo[p.H * QP + i] = __float2half_rn(0.f);
  }
  for (int i = p.H * PP + tid; i < p.hp * PP; i += kThreads) sP[i] = __float2half_rn(0.f);
  for (int h = tid; h < p.hp; h += kThreads) sAl[h] = 0.f;
  // the quad table: the key latents' quads in head order, then the value latent's (padded to
  // rvp channels with zero quads), then zero quads up to a multiple of 32
  int4* qtab = reinterpret_cast<int4*>(smem + p.s_qtab);
  for (int qq = tid; qq < p.nquad; qq += kThreads) {
    int rest = qq, g = 0;
    while (g < p.Hkv && rest >= (p.key[g].rank >> 2)) {
      rest -= p.key[g].rank >> 2;
      ++g;
    }
    int4 e;
    if (g < p.Hkv) {
      e = quad_entry(p.key[g], 4 * rest, p.s_ck[g], 2 * (p.key[g].rank + 8));
    } else if (4 * rest < p.rvp) {
      e = quad_entry(p.val, 4 * rest, p.s_cv, 2 * cvp);
    } else {
      // padding: every token writes its zeros to one spare slot after the table (pitch 0)
      e = make_int4(kQuadZero << 28, 0, 0, p.s_qtab + 16 * p.nquad);
    }
    qtab[qq] = e;
  }
  __syncthreads();

  uint32_t phase = 0;  // parity of the page barrier's next completion
  bool stop = false;
  for (int u = blockIdx.x; u < p.units && !stop; u += gridDim.x) {
    const int b = u / p.nsplit, sp = u - b * p.nsplit;
    const int L = max(0, min(p.seq_lens[b], p.max_pages * kPage));
    const int pg0 = sp * p.pps, pg1 = min((L + kPage - 1) / kPage, pg0 + p.pps);
    float* rec0 = p.ws + static_cast<long long>(u) * p.H * p.rec;
    if (pg0 >= pg1) {  // an empty range: a record of no weight
      for (int h = tid; h < p.H; h += kThreads) {
        rec0[static_cast<long long>(h) * p.rec] = -INFINITY;
        rec0[static_cast<long long>(h) * p.rec + 1] = 0.f;
      }
      continue;
    }
    const int* trow = p.block_table + static_cast<long long>(b) * p.max_pages;
    auto issue_page = [&](int pg) {  // thread 0
      const int pid = trow[pg];
      const bool ok = pid >= 0 && pid < p.num_pages;
      flags[0] = ok ? 1 : 0;
      if (ok) {
        fence_proxy_async_smem();
        mbar_arrive_expect_tx(bar, static_cast<uint32_t>(p.page_bytes));
        bulk_g2s(sbase + p.s_page, p.cache + static_cast<long long>(pid) * p.page_bytes,
                 static_cast<uint32_t>(p.page_bytes), bar);
      } else if (p.status) {
        atomicOr(p.status, STARKV_DEV_BOUNDS);
      }
    };
    if (tid == 0) issue_page(pg0);
    // the rotated, scaled queries of the sequence (position L - 1), split into hi + lo
    {
      const int T = L - 1;
      for (int idx = tid; idx < p.H * HALF; idx += kThreads) {
        const int h = idx / HALF, j = idx - h * HALF;
        const float2 bs = basetab[(T >> 7) * HALF + j], f = fine[(T & 127) * HALF + j];
        const float cs = bs.x * f.x - bs.y * f.y, sn = bs.y * f.x + bs.x * f.y;
        const long long qb = (static_cast<long long>(b) * p.H + h) * HD;
        const float x1 = __bfloat162float(p.q[qb + j]), x2 = __bfloat162float(p.q[qb + j + HALF]);
        const float r1 = (x1 * cs - x2 * sn) * p.qscale, r2 = (x2 * cs + x1 * sn) * p.qscale;
        const __half h1 = __float2half_rn(r1), h2 = __float2half_rn(r2);
        sQhi[h * QP + j] = h1;
        sQhi[h * QP + j + HALF] = h2;
        sQlo[h * QP + j] = __float2half_rn(r1 - __half2float(h1));
        sQlo[h * QP + j + HALF] = __float2half_rn(r2 - __half2float(h2));
      }
      for (int h = tid; h < p.H; h += kThreads) {
        sM[h] = -INFINITY;
        sL[h] = 0.f;
      }
    }
    // value accumulators: n-tile ni of this warp (channels 8 (warp + 8 ni) ..) and head tile
    // mt in acc[ni * MT + mt]
    constexpr int NI = kPvMax / MT;
    float acc[NI * MT][4];
#pragma unroll
    for (int i = 0; i < NI * MT; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
    const int ntw = p.rvp >> 6;  // value n-tiles of this warp (<= NI)

    for (int pg = pg0; pg < pg1; ++pg) {
      // (1) the page: thread 0 waits (bounded) and publishes what it found
      if (tid == 0) {
        int st = 0;  // 0: no data (bad page entry), 1: data, 2: timed out
        if (flags[0]) {
          const uint64_t t0 = globaltimer_ns();
          st = 1;
          while (!mbar_try_wait(bar, phase)) {
            if (globaltimer_ns() - t0 > p.timeout_ns) {
              st = 2;
              if (p.status) atomicOr(p.status, STARKV_DEV_TIMEOUT);
              break;
            }
          }
          if (st == 1) phase ^= 1u;
        }
        flags[1] = st;
      }
      __syncthreads();
      const int pst = flags[1];
      if (pst == 2) {
        stop = true;
        break;
      }
      const bool valid = pst == 1;
      // (2) codes -> fp16 operands; thread (token tid / 4) takes every fourth quad of it.
      // Slots past the sequence's end hold whatever the page held (scales included), so
      // they become zeros: their weight is 0 and 0 x garbage could be NaN.
      {
        const int tk = tid >> 2, sub = tid & 3;
        const bool tv = valid && pg * kPage + tk < L;
        const int4* tab = reinterpret_cast<const int4*>(smem + p.s_qtab);
        for (int j0 = sub; j0 < p.nquad; j0 += 32) {  // eight quads in flight per thread
          int4 e[8];
          uint32_t w[8];
          __half sc[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) e[u] = tab[j0 + 4 * u];
          // branch-free, so the eight quads' loads overlap: every quad reads two half-words
          // at its offset (a zero quad reads the page's first bytes: its entry holds offset 0
          // and stride 0) and its scale, and both conversions are selected by kind
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const uint8_t* src = page + (e[u].x & 0xFFFFF) + tk * (e[u].y & 0xFFFF);
            const uint32_t lo = *reinterpret_cast<const unsigned short*>(src);
            const uint32_t hi = *reinterpret_cast<const unsigned short*>(src + 2);
            w[u] = (e[u].x >> 28) == kQuadInt8 ? (lo | (hi << 16)) : lo;
            sc[u] = *reinterpret_cast<const __half*>(page + e[u].z + tk * (e[u].y >> 16));
          }
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const int kind = e[u].x >> 28;
            const uint2 v8 = dequant_codes(w[u], kQuadInt8, sc[u]);
            const uint2 v4 = dequant_codes(w[u], kQuadInt4, sc[u]);
            uint2 v = kind == kQuadInt8 ? v8 : v4;
            if (!tv || kind == kQuadZero) v = make_uint2(0u, 0u);
            *reinterpret_cast<uint2*>(smem + (e[u].w & 0xFFFFF) + tk * ((e[u].w >> 20) << 4)) = v;
          }
        }
      }
      __syncthreads();
      // (3) the next page's copy: this one has been read
      if (tid == 0 && pg + 1 < pg1) issue_page(pg + 1);
      // (4) keys, RoPE, scores
      {
        const int mt = warp & 3;
        const int tok_a = 16 * mt + gid, tok_b = tok_a + 8;
        const int pos_a = pg * kPage + tok_a, pos_b = pos_a + 8;
        const bool in_a = valid && pos_a < L, in_b = valid && pos_b < L;
        // RoPE factors of this thread's rows and columns j = 8 nt + 2 tig + e
        float rc[JN][2][2], rs[JN][2][2];
        {
          const int tb = pos_a >> 7;  // the page lies inside one 128-token table tile
#pragma unroll
          for (int nt = 0; nt < JN; ++nt)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const int j = 8 * nt + 2 * tig + e;
              const float2 bs = basetab[tb * HALF + j];
              const float2 fa = fine[(pos_a & 127) * HALF + j], fb = fine[(pos_b & 127) * HALF + j];
              rc[nt][0][e] = bs.x * fa.x - bs.y * fa.y;
              rs[nt][0][e] = bs.y * fa.x + bs.x * fa.y;
              rc[nt][1][e] = bs.x * fb.x - bs.y * fb.y;
              rs[nt][1][e] = bs.y * fb.x + bs.x * fb.y;
            }
        }
        for (int g = warp >> 2; g < p.Hkv; g += 2) {
          const int r = p.key[g].rank;
          float k[NT][4];
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) k[nt][0] = k[nt][1] = k[nt][2] = k[nt][3] = 0.f;
          const uint32_t aRow =
              sbase + p.s_ck[g] + ((16 * mt + (lane & 7) + ((lane >> 3) & 1) * 8) * (r + 8) + (lane >> 4) * 8) * 2;
          const uint32_t bRow =
              sbase + p.s_bk[g] + (((lane & 7) + (lane >> 4) * 8) * (r + 8) + ((lane >> 3) & 1) * 8) * 2;
          for (int k0 = 0; k0 < r; k0 += 16) {
            uint32_t a0, a1, a2, a3;
            ldsm_x4(aRow + k0 * 2, a0, a1, a2, a3);
#pragma unroll
            for (int np = 0; np < NT / 2; ++np) {
              uint32_t b0, b1, b2, b3;
              ldsm_x4(bRow + (np * 16 * (r + 8) + k0) * 2, b0, b1, b2, b3);
              mma_f16(k[2 * np], a0, a1, a2, a3, b0, b1);
              mma_f16(k[2 * np + 1], a0, a1, a2, a3, b2, b3);
            }
          }
          // RoPE: column j pairs with j + d/2, which is n-tile nt + JN of the same thread
#pragma unroll
          for (int nt = 0; nt < JN; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float c = rc[nt][e >> 1][e & 1], s = rs[nt][e >> 1][e & 1];
              const float x1 = k[nt][e], x2 = k[nt + JN][e];
              k[nt][e] = x1 * c - x2 * s;
              k[nt + JN][e] = x2 * c + x1 * s;
            }
          // scores of the KV head's query heads (n = gid < G; rows past G read zeros)
          const int hq = gid < p.G ? g * p.G + gid : p.H;
          const uint32_t qh = smem_u32(sQhi + hq * QP) + 4 * tig;
          const uint32_t ql = smem_u32(sQlo + hq * QP) + 4 * tig;
          // six independent accumulators (the three products x the parity of the k-step), so
          // consecutive MMAs do not wait on one another; added in a fixed order at the end
          float sp[6][4];
#pragma unroll
          for (int i = 0; i < 6; ++i) sp[i][0] = sp[i][1] = sp[i][2] = sp[i][3] = 0.f;
#pragma unroll
          for (int kk = 0; kk < HD / 16; ++kk) {
            uint32_t ah[4], al[4];
            split_h2(k[2 * kk][0], k[2 * kk][1], ah[0], al[0]);
            split_h2(k[2 * kk][2], k[2 * kk][3], ah[1], al[1]);
            split_h2(k[2 * kk + 1][0], k[2 * kk + 1][1], ah[2], al[2]);
            split_h2(k[2 * kk + 1][2], k[2 * kk + 1][3], ah[3], al[3]);
            const uint32_t bh0 = ld_shared_u32(qh + kk * 32), bh1 = ld_shared_u32(qh + kk * 32 + 16);
            const uint32_t bl0 = ld_shared_u32(ql + kk * 32), bl1 = ld_shared_u32(ql + kk * 32 + 16);
            const int o = 3 * (kk & 1);
            mma_f16(sp[o], ah[0], ah[1], ah[2], ah[3], bh0, bh1);
            mma_f16(sp[o + 1], al[0], al[1], al[2], al[3], bh0, bh1);
            mma_f16(sp[o + 2], ah[0], ah[1], ah[2], ah[3], bl0, bl1);
          }
          float sc[4];
#pragma unroll
          for (int e = 0; e < 4; ++e)
            sc[e] = ((sp[0][e] + sp[3][e]) + (sp[1][e] + sp[4][e])) + (sp[2][e] + sp[5][e]);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int hh = 2 * tig + (e & 1);
            if (hh < p.G) {
              const bool in = e < 2 ? in_a : in_b;
              sS[(e < 2 ? tok_a : tok_b) * spitch + g * p.G + hh] = in ? sc[e] : -INFINITY;
            }
          }
        }
      }
      __syncthreads();
      // (5) online softmax per query head: 8 threads per head, 8 tokens each
      for (int h0 = 0; h0 < p.H; h0 += kThreads / 8) {
        const int h = h0 + (tid >> 3), part = tid & 7;
        const bool own = h < p.H;
        float s8[8], mx = -INFINITY;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          s8[i] = own ? sS[(part + 8 * i) * spitch + h] : -INFINITY;
          mx = fmaxf(mx, s8[i]);
        }
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
        const float mo = own ? sM[h] : -INFINITY;
        const float mn = fmaxf(mo, mx);
        const bool live = mn != -INFINITY;
        float lsum = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const __half ph = __float2half_rn(live ? exp2f(s8[i] - mn) : 0.f);
          lsum += __half2float(ph);  // the same rounded weight the product uses
          if (own) sP[h * PP + part + 8 * i] = ph;
        }
        lsum += __shfl_xor_sync(0xffffffffu, lsum, 1);
        lsum += __shfl_xor_sync(0xffffffffu, lsum, 2);
        lsum += __shfl_xor_sync(0xffffffffu, lsum, 4);
        if (own && part == 0) {
          const float alpha = live ? exp2f(mo - mn) : 1.f;
          sL[h] = sL[h] * alpha + lsum;
          sM[h] = mn;
          sAl[h] = alpha;
        }
      }
      __syncthreads();
      // (6) a += P C_v: warp w holds value n-tiles w + 8 i, every 16-head tile
      {
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
          const float al0 = sAl[16 * mt + gid], al1 = sAl[16 * mt + gid + 8];
#pragma unroll
          for (int ni = 0; ni < NI; ++ni) {
            acc[ni * MT + mt][0] *= al0;
            acc[ni * MT + mt][1] *= al0;
            acc[ni * MT + mt][2] *= al1;
            acc[ni * MT + mt][3] *= al1;
          }
        }
        const uint32_t pRow = smem_u32(sP) + (((lane & 7) + ((lane >> 3) & 1) * 8) * PP + (lane >> 4) * 8) * 2;
        const uint32_t vRow = smem_u32(sCv) + (((lane & 7) + ((lane >> 3) & 1) * 8) * cvp + 8 * warp) * 2;
#pragma unroll
        for (int ks = 0; ks < kPage / 16; ++ks) {
          uint32_t a[MT][4];
#pragma unroll
          for (int mt = 0; mt < MT; ++mt)
            ldsm_x4(pRow + (16 * mt * PP + 16 * ks) * 2, a[mt][0], a[mt][1], a[mt][2], a[mt][3]);
#pragma unroll
          for (int ni = 0; ni < NI; ++ni) {
            if (ni < ntw) {
              uint32_t b0, b1;
              ldsm_x2_trans(vRow + (16 * ks * cvp + 64 * ni) * 2, b0, b1);
#pragma unroll
              for (int mt = 0; mt < MT; ++mt)
                mma_f16(acc[ni * MT + mt], a[mt][0], a[mt][1], a[mt][2], a[mt][3], b0, b1);
            }
          }
        }
      }
    }
    if (stop) break;
    // the unit's records: m, l, then a from the accumulator fragments
    for (int h = tid; h < p.H; h += kThreads) {
      rec0[static_cast<long long>(h) * p.rec] = sM[h];
      rec0[static_cast<long long>(h) * p.rec + 1] = sL[h];
    }
#pragma unroll
    for (int i = 0; i < NI * MT; ++i) {
      if (i / MT < ntw) {
        const int mt = i % MT, nc = warp + 8 * (i / MT);
        const int ch = 8 * nc + 2 * tig, ha = 16 * mt + gid, hb = ha + 8;
        if (ha < p.H) {
          float* ra = rec0 + static_cast<long long>(ha) * p.rec + 2;
          if (ch < p.rv) ra[ch] = acc[i][0];
          if (ch + 1 < p.rv) ra[ch + 1] = acc[i][1];
        }
        if (hb < p.H) {
          float* rb = rec0 + static_cast<long long>(hb) * p.rec + 2;
          if (ch < p.rv) rb[ch] = acc[i][2];
          if (ch + 1 < p.rv) rb[ch + 1] = acc[i][3];
        }
      }
    }
    __syncthreads();  // the statistics and query buffers are rewritten by the next unit
  }
  if (stop && tid == 0) {
    // a copy may still be in flight into this CTA's shared memory: the same bound again
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(bar, phase) && globaltimer_ns() - t0 < p.timeout_ns) {
    }
  }
}

// One CTA per (sequence, query head): merge the page-range records (log-sum-exp), normalise,
// then o_h = a_h B_v[:, g d : (g+1) d].
__global__ void __launch_bounds__(128) hybrid_combine_kernel(const __grid_constant__ HybridParams p) {
  __shared__ float s_a[2048];
  const int b = blockIdx.x / p.H, h = blockIdx.x % p.H, g = h / p.G;
  const int tid = threadIdx.x;
  float* outp = p.out + (static_cast<long long>(b) * p.H + h) * p.d;
  const int L = max(0, min(p.seq_lens[b], p.max_pages * kPage));
  if (L == 0) {
    for (int c = tid; c < p.d; c += 128) outp[c] = 0.f;
    return;
  }
  const long long stride = static_cast<long long>(p.H) * p.rec;  // between page ranges
  const float* r0 = p.ws + (static_cast<long long>(b) * p.nsplit * p.H + h) * p.rec;
  // each range's weight exp2(m_s - M) once (0 for a range without weight), in shared memory
  // after the r_v slots of s_a when the ranges fit, else recomputed per channel
  float* s_w = s_a + p.rv;
  const bool wfit = p.rv + p.nsplit <= 2048;
  float M = -INFINITY;
  for (int s = 0; s < p.nsplit; ++s) {
    const float* rc = r0 + s * stride;
    if (rc[1] > 0.f) M = fmaxf(M, rc[0]);
  }
  float l = 0.f;
  for (int s = 0; s < p.nsplit; ++s) {
    const float* rc = r0 + s * stride;
    if (rc[1] > 0.f) l += rc[1] * exp2f(rc[0] - M);
  }
  if (wfit) {
    for (int s = tid; s < p.nsplit; s += 128) {
      const float* rc = r0 + s * stride;
      s_w[s] = rc[1] > 0.f ? exp2f(rc[0] - M) : 0.f;
    }
    __syncthreads();
  }
  const float inv = l > 0.f ? 1.f / l : 0.f;
  for (int i = tid; i < p.rv; i += 128) {
    float a = 0.f;
    for (int s = 0; s < p.nsplit; ++s) {
      const float* rc = r0 + s * stride;
      const float w = wfit ? s_w[s] : (rc[1] > 0.f ? exp2f(rc[0] - M) : 0.f);
      if (w > 0.f) a = fmaf(rc[2 + i], w, a);
    }
    s_a[i] = a * inv;
  }
  __syncthreads();
  const int ldv = p.Hkv * p.d;
  for (int c = tid; c < p.d; c += 128) {
    const float* bv = p.Bv + g * p.d + c;
    float o0 = 0.f, o1 = 0.f;
    int i = 0;
    for (; i + 1 < p.rv; i += 2) {
      o0 = fmaf(s_a[i], bv[static_cast<long long>(i) * ldv], o0);
      o1 = fmaf(s_a[i + 1], bv[static_cast<long long>(i + 1) * ldv], o1);
    }
    if (i < p.rv) o0 = fmaf(s_a[i], bv[static_cast<long long>(i) * ldv], o0);
    outp[c] = o0 + o1;
  }
}

int align16i(int x) { return (x + 15) & ~15; }

}  // namespace

bool hybrid_plan(HybridParams& p, size_t smem_limit) {
  long long off = 0;
  auto take = [&](long long bytes) {
    const int o = static_cast<int>(off);
    off = align16i(static_cast<int>(off + bytes));
    return o;
  };
  for (int g = 0; g < p.Hkv; ++g) p.s_bk[g] = take(2LL * p.d * (p.key[g].rank + 8));
  for (int g = 0; g < p.Hkv; ++g) p.s_ck[g] = take(2LL * kPage * (p.key[g].rank + 8));
  p.s_cv = take(2LL * kPage * (p.rvp + 8));
  p.s_qhi = take(2LL * (p.H + 1) * (p.d + 8));
  p.s_qlo = take(2LL * (p.H + 1) * (p.d + 8));
  p.s_s = take(4LL * kPage * (p.H + 4));
  p.s_p = take(2LL * p.hp * (kPage + 8));
  p.s_stat = take(4LL * 3 * p.hp + 16);
  p.s_qtab = take(16LL * p.nquad + 16);  // the table, then the padding quads' spare slot
  p.s_page = take(p.page_bytes);
  p.s_bar = take(8);
  p.smem_bytes = static_cast<int>(off);
  return off <= static_cast<long long>(smem_limit);
}

cudaError_t launch_hybrid_split(const HybridParams& p, int grid, cudaStream_t s) {
  if (p.units == 0) return cudaSuccess;
  void (*kern)(HybridParams) = nullptr;
  switch (p.d * 8 + p.mt_pv) {
    case 128 * 8 + 1: kern = hybrid_split_kernel<128, 1>; break;
    case 128 * 8 + 2: kern = hybrid_split_kernel<128, 2>; break;
    case 128 * 8 + 3: kern = hybrid_split_kernel<128, 3>; break;
    case 128 * 8 + 4: kern = hybrid_split_kernel<128, 4>; break;
    case 64 * 8 + 1: kern = hybrid_split_kernel<64, 1>; break;
    case 64 * 8 + 2: kern = hybrid_split_kernel<64, 2>; break;
    case 64 * 8 + 3: kern = hybrid_split_kernel<64, 3>; break;
    case 64 * 8 + 4: kern = hybrid_split_kernel<64, 4>; break;
    default: return cudaErrorInvalidValue;
  }
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, p.smem_bytes);
  if (e != cudaSuccess) return e;
  kern<<<grid, kThreads, p.smem_bytes, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_hybrid_combine(const HybridParams& p, cudaStream_t s) {
  if (p.batch == 0) return cudaSuccess;
  hybrid_combine_kernel<<<p.batch * p.H, 128, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace starkv
