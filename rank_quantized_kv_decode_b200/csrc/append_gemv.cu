// Latent write of a decode step in one launch: for a few new tokens (at most 32, one per
// sequence of the batch), c = x [A_k | A_v,0 | ...] on the tensor cores, then the store of
// starkv_quant_pack (quantise, pack, scatter into the pages) in the same kernel.
//
// The step reads all of A once (d_model x proj_cols bf16: 4 MB for the GQA layer, 16.8 MB for
// the MHA layer) and little else, so its bound is HBM bandwidth.  One CTA takes one
// 32-channel chunk of the latents (in the quantised formats: one quantisation group) and one
// k-slice of d_model; the KS CTAs of a chunk form a cluster.  Each CTA stages its A rows and
// the tokens' x rows with bulk copies (one per row, all in flight at once), multiplies them
// with mma.sync m16n8k16 (bf16 operands, fp32 accumulation; the tokens are the M dimension, at
// most two 16-row tiles; each warp a quarter of the k-slice), and keeps its partial sums in
// shared memory.  The cluster's CTAs then share the chunk's tokens: each adds the KS partials
// of its tokens in k-slice order through distributed shared memory and stores them exactly as
// the store kernel does (same device code), so no partial goes through HBM and one launch
// does the whole step.  (mma.sync, not tcgen05: with at most 32 tokens the product is a
// GEMV whose cost is reading A, and a 128-row tcgen05 tile would be three-quarters padding.)  (STAR-KV technical summary, Methodology §3 and the abstract: the latents of
// a new token are x times the down-projection, quantised as they are written.)
#include <algorithm>

#include "store_dev.cuh"

namespace starkv {

namespace {

using namespace store_dev;

constexpr int kRowPad = 16;  // bytes added to each staged row: spreads the fragment loads over banks

__device__ __forceinline__ void cluster_arrive_release() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait_acquire() {
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ __forceinline__ float ld_dsmem_f32(uint32_t cluster_addr) {
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(cluster_addr) : "memory");
  return v;
}

// D (16x8 fp32) += A (16x16 bf16, row-major) * B (16x8 bf16, column-major).
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                               uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__global__ void __launch_bounds__(128) append_gemv_kernel(const __grid_constant__ GemvParams g) {
  extern __shared__ __align__(16) uint8_t smem[];
  const StoreParams& p = g.sp;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rank = static_cast<int>(cluster_ctarank());  // this CTA's k-slice
  const int ck = blockIdx.x / g.ks;                       // the chunk
  const int n_tok = p.n_tok;
  const int xrows = n_tok <= 16 ? 16 : 32;
  const int rb = g.row_bytes;
  uint8_t* sA = smem;                                       // [32 channels][rb]
  uint8_t* sX = smem + 32 * rb;                             // [xrows tokens][rb]
  // [32 tokens][32 channels], after the staged rows (at least 16 KB, see append_gemv_smem)
  float* sPart = reinterpret_cast<float*>(smem + max((32 + xrows) * rb, 4 * 32 * 32 * 4));
  uint64_t* bar = reinterpret_cast<uint64_t*>(sPart + 32 * 32);
  TokenSlot* sTok = reinterpret_cast<TokenSlot*>(bar + 1);  // [32 / ks]: pages of this CTA's tokens

  // the chunk's channels: latent li, channels [ch0, ch0 + nch), rows col + ch0 .. of A_t
  const ChunkLane q0 = chunk_lane(p, ck, 0);
  const LatDesc& d = p.lat[q0.li];
  const int ch0 = q0.i;
  const int nch = q0.plain ? min(32, d.rank - ch0) : (q0.is8 ? min(32, d.n8 - ch0) : min(32, q0.n4 - q0.j));
  const int kbytes = g.kslice * 2;

  if (threadIdx.x == 0) {
    mbar_init(smem_u32(bar), 1);
    fence_mbar_init();
  }
  // rows no copy fills read as zeros (channels past the chunk, tokens past the step); only
  // those rows are visited
  {
    const int nc16 = kbytes / 16;
    const int za = 32 - nch, zx = xrows - n_tok;
    for (int idx = threadIdx.x; idx < (za + zx) * nc16; idx += blockDim.x) {
      const int zr = idx / nc16, c16 = idx - zr * nc16;
      const int r = zr < za ? nch + zr : 32 + n_tok + (zr - za);
      *reinterpret_cast<uint4*>(smem + r * rb + c16 * 16) = make_uint4(0, 0, 0, 0);
    }
  }
  __syncthreads();
  pdl_wait();
  pdl_launch_dependents();
  {
    // the copies of the chunk's A rows and the tokens' x rows, one per thread (the barrier's
    // transaction count is set before any copy can complete on it)
    const uint32_t fb = smem_u32(bar);
    if (threadIdx.x == 0) mbar_arrive_expect_tx(fb, static_cast<uint32_t>((nch + n_tok) * kbytes));
    __syncthreads();
    const long long kofs = static_cast<long long>(rank) * g.kslice;
    const int r = threadIdx.x;
    if (r < nch)
      bulk_g2s(smem_u32(sA + r * rb), g.A_t + (static_cast<long long>(d.col + ch0 + r) * g.d_model + kofs),
               static_cast<uint32_t>(kbytes), fb);
    else if (r < nch + n_tok)
      bulk_g2s(smem_u32(sX + (r - nch) * rb), g.x + (static_cast<long long>(r - nch) * g.d_model + kofs),
               static_cast<uint32_t>(kbytes), fb);
  }
  // the cluster's CTAs share the chunk's tokens for the store: CTA r takes tokens r, r + ks,
  // ...; their pages are looked up now, one thread per token, while the copies fly
  const int mine = n_tok > rank ? (n_tok - rank + g.ks - 1) / g.ks : 0;
  if (threadIdx.x < mine)
    sTok[threadIdx.x] = locate(p, rank + g.ks * threadIdx.x, (q0.li == 0 && q0.cl == 0) ? 0 : 1, 0);
  // bounded wait for the copies (a timeout is reported; the cluster still meets below)
  bool ok = true;
  {
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(smem_u32(bar), 0)) {
      if (globaltimer_ns() - t0 > g.timeout_ns) {
        ok = false;
        if (lane == 0 && p.status) atomicOr(p.status, STARKV_DEV_TIMEOUT);
        break;
      }
    }
  }
  // warp w: the quarter [w kq, (w + 1) kq) of the slice's k-range, all 32 channels (four
  // n-tiles) and every token tile (m-tiles of 16): up to eight independent accumulators, so
  // consecutive MMAs do not wait on one another
  const int gid = lane >> 2, tig = lane & 3;
  const int kq = kbytes / 4;  // bytes; a multiple of 32 (the slice is a multiple of 64 columns)
  float acc[2][4][4];
#pragma unroll
  for (int mt = 0; mt < 2; ++mt)
#pragma unroll
    for (int nt = 0; nt < 4; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[mt][nt][e] = 0.f;
  if (ok) {
    const uint32_t aB = smem_u32(sA + gid * rb) + 4 * tig + warp * kq;
    const uint32_t aX = smem_u32(sX + gid * rb) + 4 * tig + warp * kq;
    for (int k0 = 0; k0 < kq; k0 += 32) {
      uint32_t b[4][2];
#pragma unroll
      for (int nt = 0; nt < 4; ++nt) {
        b[nt][0] = ld_shared_u32(aB + nt * 8 * rb + k0);
        b[nt][1] = ld_shared_u32(aB + nt * 8 * rb + k0 + 16);
      }
#pragma unroll
      for (int mt = 0; mt < 2; ++mt) {
        if (mt == 1 && xrows != 32) break;
        const uint32_t o = aX + mt * 16 * rb + k0;
        const uint32_t a0 = ld_shared_u32(o), a1 = ld_shared_u32(o + 8 * rb);
        const uint32_t a2 = ld_shared_u32(o + 16), a3 = ld_shared_u32(o + 8 * rb + 16);
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) mma_bf16_16816(acc[mt][nt], a0, a1, a2, a3, b[nt][0], b[nt][1]);
      }
    }
  }
  // the warps' quarter sums go over the staged rows, which no thread reads any more (the
  // region is at least 16 KB); this CTA's partial sums sPart[token][channel] are the quarters
  // added in order
  __syncthreads();
  float* sRed = reinterpret_cast<float*>(smem);  // [4 warps][32 tokens][32 channels]
#pragma unroll
  for (int mt = 0; mt < 2; ++mt)
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
      float* r = sRed + warp * 1024 + (16 * mt + gid) * 32 + 8 * nt + 2 * tig;
      r[0] = acc[mt][nt][0];
      r[1] = acc[mt][nt][1];
      r[8 * 32] = acc[mt][nt][2];
      r[8 * 32 + 1] = acc[mt][nt][3];
    }
  __syncthreads();
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int e = threadIdx.x + 128 * i;
    sPart[e] = ((sRed[e] + sRed[1024 + e]) + sRed[2048 + e]) + sRed[3072 + e];
  }
  // every CTA's partials (and this CTA's token pages) are visible to every CTA of the cluster
  cluster_sync_all();
  {
    // the latents of this chunk, partials added in k-slice order (deterministic), then the
    // store of starkv_quant_pack; warp w of a CTA takes every fourth of its tokens.  Every
    // partial of a value is requested before the first is added, so no remote load waits
    // for another.
    const ChunkLane q = chunk_lane(p, ck, lane);
    const uint32_t base = smem_u32(sPart);
    float* sVal = sRed;  // [32 / ks tokens][32 channels]: the sums, kept until the stores
    for (int k = warp; k < mine; k += 4) {
      const int n = rank + g.ks * k;
      float v[8];
#pragma unroll
      for (int r = 0; r < 8; ++r)
        v[r] = r < g.ks ? ld_dsmem_f32(mapa_shared(base + 4u * (n * 32 + lane), static_cast<uint32_t>(r))) : 0.f;
      float c = v[0];
#pragma unroll
      for (int r = 1; r < 8; ++r)
        if (r < g.ks) c += v[r];
      sVal[k * 32 + lane] = c;
    }
    // this CTA has read every partial it needs; the stores overlap the other CTAs' reads
    cluster_arrive_release();
    for (int k = warp; k < mine; k += 4)
      store_value_at(p, q, rank + g.ks * k, lane, q.in ? sVal[k * 32 + lane] : 0.f, sTok[k]);
  }
  cluster_wait_acquire();  // the partials stay in place until every CTA has read them
  if (!ok && threadIdx.x == 0) {
    // copies still in flight target this CTA's shared memory: give them the same bound again
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(smem_u32(bar), 0) && globaltimer_ns() - t0 < g.timeout_ns) {
    }
  }
}

}  // namespace

size_t append_gemv_smem(int kslice, int n_tok) {
  const int rb = kslice * 2 + kRowPad;
  const int xrows = n_tok <= 16 ? 16 : 32;
  // the staged rows, reused for the warps' quarter sums (4 x 32 x 32 fp32) after the MMAs
  const size_t staged = std::max<size_t>(static_cast<size_t>(32 + xrows) * rb, 4 * 32 * 32 * sizeof(float));
  return staged + 32 * 32 * sizeof(float) + 16 + 32 * 16;
}

cudaError_t launch_append_gemv(const GemvParams& gp, cudaStream_t s) {
  if (gp.sp.n_tok == 0) return cudaSuccess;
  GemvParams g = gp;
  g.row_bytes = g.kslice * 2 + kRowPad;
  const size_t smem = append_gemv_smem(g.kslice, g.sp.n_tok);
  cudaError_t e = cudaFuncSetAttribute(append_gemv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(g.sp.chunks_per_token * g.ks), 1, 1);
  cfg.blockDim = dim3(128, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(g.ks);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, append_gemv_kernel, g);
}

}  // namespace starkv
