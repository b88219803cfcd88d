// Latent projection of new tokens, c = x [A_k | A_v,0 | ...], on tcgen05 tensor cores.
//
// One CTA per (128-row tile of x, 256-column tile of the projection, K split).  TMA brings
// 128-byte-swizzled k-blocks of x and of A^T (K-major) into a shared-memory ring; one thread
// issues tcgen05.mma into a 128 x 256 fp32 TMEM accumulator; four epilogue warps read it back
// (thread = row) and store the fp32 partial sums.  The split-K partials are added in a fixed
// order by the store kernel, which then quantises and packs (deterministic results).
#include "internal.cuh"

namespace starkv {

namespace {

template <int FMT>
struct ProjFmt {
  // fp32 operands run as 3xTF32: hi/lo copies of both tiles, split in shared memory by
  // four extra warps
  static constexpr bool kSplit = FMT == STARKV_FMT_F32;
  static constexpr int kThreads = kSplit ? 320 : 192;
};

template <int FMT>
__global__ void __launch_bounds__(ProjFmt<FMT>::kThreads, 1)
    project_kernel(const __grid_constant__ ProjParams p, const __grid_constant__ CUtensorMap tmX,
                   const __grid_constant__ CUtensorMap tmA) {
  constexpr bool kSplit = ProjFmt<FMT>::kSplit;
  constexpr int kKind = FMT == STARKV_FMT_F32 ? 1 : 0;
  constexpr int kKElems = FMT == STARKV_FMT_F32 ? 32 : 64;
  constexpr uint32_t kBStage = 256 * kKBytes;
  constexpr uint32_t kAStride = kSplit ? 2 * kAStage : kAStage;
  constexpr uint32_t kBStride = kSplit ? 2 * kBStage : kBStage;
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned base (SW128 tiles), by pointer arithmetic on the shared array so that the
  // compiler keeps the address space and emits shared-memory instructions for every access
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const int S = p.stages;
  uint8_t* sA = smem;
  uint8_t* sB = smem + S * kAStride;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sB + S * kBStride);
  uint32_t* misc = reinterpret_cast<uint32_t*>(bars + 3 * S + 2);
  auto bar = [&](int i) { return smem_u32(bars + i); };
  const int B_FULL = 0, B_EMPTY = S, B_RAW = 2 * S, B_ACC = 3 * S, B_TD = 3 * S + 1;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * 128, n0 = blockIdx.y * 256;
  const int kb0 = blockIdx.z * p.kb_per_split;
  const int kb1 = min(p.kb_total, kb0 + p.kb_per_split);

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(bar(B_FULL + s), kSplit ? 4 : 1);
      mbar_init(bar(B_EMPTY + s), 1);
      mbar_init(bar(B_RAW + s), 1);
    }
    mbar_init(bar(B_ACC), 1);
    mbar_init(bar(B_TD), 1);
    misc[1] = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(misc), 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  pdl_wait();
  pdl_launch_dependents();
  const uint32_t tmem = misc[0];
  WaitCtl wc{reinterpret_cast<volatile int*>(misc + 1), p.status, p.timeout_ns};

  if (warp == 0) {
    if (lane == 0) {
      prefetch_tmap(&tmX);
      prefetch_tmap(&tmA);
      int stage = 0;
      uint32_t phase = 0, issued = 0, last_phase = 0;
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!wait_bounded(bar(B_EMPTY + stage), phase ^ 1u, wc)) break;
        const uint32_t fb = bar((kSplit ? B_RAW : B_FULL) + stage);
        mbar_arrive_expect_tx(fb, kAStage + kBStage);
        tma_load_2d(smem_u32(sA + stage * kAStride), &tmX, fb, kb * kKElems, m0);
        tma_load_2d(smem_u32(sB + stage * kBStride), &tmA, fb, kb * kKElems, n0);
        issued |= 1u << stage;
        last_phase = (last_phase & ~(1u << stage)) | (phase << stage);
        if (++stage == S) { stage = 0; phase ^= 1u; }
      }
      for (int s = 0; s < S; ++s) {
        if (!(issued & (1u << s))) continue;
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait(bar((kSplit ? B_RAW : B_FULL) + s), (last_phase >> s) & 1u))
          if (globaltimer_ns() - t0 > p.timeout_ns) break;
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = p.idesc;
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!wait_bounded(bar(B_FULL + stage), phase, wc)) { ok = false; break; }
        tc_fence_after();
        const uint64_t da = desc_sw128(smem_u32(sA + stage * kAStride));
        const uint64_t db = desc_sw128(smem_u32(sB + stage * kBStride));
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          umma<kKind>(tmem, da + 2 * k, db + 2 * k, idesc, (kb > kb0 || k > 0));
          if constexpr (kSplit) {
            const uint64_t dal = desc_sw128(smem_u32(sA + stage * kAStride + kAStage));
            const uint64_t dbl = desc_sw128(smem_u32(sB + stage * kBStride + kBStage));
            umma<kKind>(tmem, da + 2 * k, dbl + 2 * k, idesc, 1u);
            umma<kKind>(tmem, dal + 2 * k, db + 2 * k, idesc, 1u);
          }
        }
        umma_commit(bar(B_EMPTY + stage));
        if (++stage == S) { stage = 0; phase ^= 1u; }
      }
      if (ok) umma_commit(bar(B_ACC));
      umma_commit(bar(B_TD));
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(bar(B_TD), 0))
        if (globaltimer_ns() - t0 > p.timeout_ns) break;
    }
    __syncwarp();
  } else if (warp >= 6) {
    if constexpr (kSplit) {
      // tf32 hi/lo splitters (warps 6..9)
      const int tid = (warp - 6) * 32 + lane;
      int stage = 0;
      uint32_t phase = 0;
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!__all_sync(0xffffffffu, wait_bounded(bar(B_RAW + stage), phase, wc))) break;
        uint8_t* a = sA + stage * kAStride;
        uint8_t* b = sB + stage * kBStride;
        split_tf32(reinterpret_cast<float4*>(a), reinterpret_cast<float4*>(a + kAStage),
                   kAStage / 16, tid, 128);
        split_tf32(reinterpret_cast<float4*>(b), reinterpret_cast<float4*>(b + kBStage),
                   kBStage / 16, tid, 128);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(B_FULL + stage));
        if (++stage == S) { stage = 0; phase ^= 1u; }
      }
    }
  } else {
    // epilogue: warps 2..5 cover TMEM lane quadrants 2, 3, 0, 1
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    const bool ready = __all_sync(0xffffffffu, wait_bounded(bar(B_ACC), 0, wc));
    tc_fence_after();
    const int m = m0 + row;
    float* dst = p.part + ((long long)blockIdx.z * p.n_tok + m) * p.proj_cols;
    if (ready) {
#pragma unroll 1
      for (int cc = 0; cc < 8; ++cc) {
        float v[32];
        tmem_ld32_wait(tmem + cc * 32 + (static_cast<uint32_t>(quad * 32) << 16), v);
        if (m < p.n_tok) {
          const int nb = n0 + cc * 32;
          if (nb + 32 <= p.proj_cols && (p.proj_cols & 3) == 0) {
#pragma unroll
            for (int j = 0; j < 32; j += 4)
              *reinterpret_cast<float4*>(dst + nb + j) = make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]);
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (nb + j < p.proj_cols) dst[nb + j] = v[j];
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 256);
}

}  // namespace

cudaError_t launch_project(int fmt, const ProjParams& p, const CUtensorMap& tmX,
                           const CUtensorMap& tmA, cudaStream_t s) {
  const int m_tiles = (p.n_tok + 127) / 128;
  const int n_tiles = (p.proj_cols + 255) / 256;
  dim3 grid(m_tiles, n_tiles, p.nsplit);
  const size_t split = fmt == STARKV_FMT_F32 ? 2 : 1;
  const size_t smem = 1024 + static_cast<size_t>(p.stages) * split * (kAStage + 256 * kKBytes) +
                      (3 * p.stages + 2) * 8 + 16;
  cudaError_t e;
  if (fmt == STARKV_FMT_F32) {
    e = cudaFuncSetAttribute(project_kernel<STARKV_FMT_F32>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    e = launch_pdl(project_kernel<STARKV_FMT_F32>, grid, dim3(ProjFmt<STARKV_FMT_F32>::kThreads),
                   smem, s, p, tmX, tmA);
  } else {
    e = cudaFuncSetAttribute(project_kernel<STARKV_FMT_BF16>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    e = launch_pdl(project_kernel<STARKV_FMT_BF16>, grid, dim3(192), smem, s, p, tmX, tmA);
  }
  return e;
}

}  // namespace starkv
