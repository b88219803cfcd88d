// Weight absorption of the value up-projection into the attention output projection
// (STAR-KV technical summary, Methodology §2: values are never reconstructed; their
// up-projection is folded into W_o).  With per-head value latents, query head h gets
// M_h = B_v,g(h) W_o,h (r_g x d_out, W_o,h the rows [h d, (h+1) d) of W_o), and the attention
// block's output for the decoded token of sequence b is y_b = sum_h a_b,h M_h: one
// (batch x m_rows) x (m_rows x d_out) product, m_rows = G * R_v, instead of H small
// up-projections followed by the output projection.
#include "internal.cuh"

namespace starkv {

namespace {

constexpr int kCols = 128;  // output columns per CTA (one per thread)

// first row of query head h in M / in a row of A
__device__ __forceinline__ int head_row(const AbsorbParams& p, int h) {
  const LatDesc& vd = p.vh[h / p.G];
  return p.G * (vd.col - p.key_rank_cols) + (h % p.G) * vd.rank;
}

// M_h[i][c] = sum_j B_v,g[i][j] Wo[h d + j][c]; CTA (column tile, head), thread = column.
// A one-off setup product: plain fp32 FMAs.
__global__ void __launch_bounds__(kCols) absorb_weights_kernel(const __grid_constant__ AbsorbParams p) {
  const int h = blockIdx.y;
  const int c = blockIdx.x * kCols + threadIdx.x;
  const LatDesc& vd = p.vh[h / p.G];
  const int r = vd.rank;
  const float* bv = p.Bv + (long long)(vd.col - p.key_rank_cols) * p.d;
  const float* wo = p.Wo + (long long)h * p.d * p.d_out;
  float* m = p.M + (long long)head_row(p, h) * p.d_out;
  if (c >= p.d_out) return;
  for (int i = 0; i < r; ++i) {
    float acc = 0.f;
    for (int j = 0; j < p.d; ++j) acc = fmaf(bv[(long long)i * p.d + j], wo[(long long)j * p.d_out + c], acc);
    m[(long long)i * p.d_out + c] = acc;
  }
}

// part[s][b][c] = sum over rows k of split s of A[b][k] M[k][c].  CTA (column tile, split),
// thread = column; A's rows of the split for 8 sequences at a time in shared memory.
__global__ void __launch_bounds__(kCols) absorbed_gemv_kernel(const __grid_constant__ AbsorbParams p) {
  __shared__ float sa[8][256];
  const int c = blockIdx.x * kCols + threadIdx.x;
  const int k0 = blockIdx.y * p.krows, k1 = min(p.m_rows, k0 + p.krows);
  {
    const int b0 = blockIdx.z * 8;  // 8 sequences per CTA; M is re-read from L2 by the others
    const int nb = min(8, p.batch - b0);
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int kk = k0; kk < k1; kk += 256) {
      const int kn = min(256, k1 - kk);
      __syncthreads();
      for (int i = threadIdx.x; i < 8 * 256; i += kCols) {
        const int bb = i >> 8, k = i & 255;
        sa[bb][k] = (bb < nb && k < kn) ? p.A[(long long)(b0 + bb) * p.m_rows + kk + k] : 0.f;
      }
      __syncthreads();
      if (c < p.d_out) {
        const float* mk = p.M + (long long)kk * p.d_out + c;
        int k = 0;
        for (; k + 4 <= kn; k += 4) {
          const float m0 = __ldg(mk + (long long)k * p.d_out), m1 = __ldg(mk + (long long)(k + 1) * p.d_out);
          const float m2 = __ldg(mk + (long long)(k + 2) * p.d_out), m3 = __ldg(mk + (long long)(k + 3) * p.d_out);
#pragma unroll
          for (int bb = 0; bb < 8; ++bb) {
            acc[bb] = fmaf(sa[bb][k], m0, acc[bb]);
            acc[bb] = fmaf(sa[bb][k + 1], m1, acc[bb]);
            acc[bb] = fmaf(sa[bb][k + 2], m2, acc[bb]);
            acc[bb] = fmaf(sa[bb][k + 3], m3, acc[bb]);
          }
        }
        for (; k < kn; ++k) {
          const float m0 = __ldg(mk + (long long)k * p.d_out);
#pragma unroll
          for (int bb = 0; bb < 8; ++bb) acc[bb] = fmaf(sa[bb][k], m0, acc[bb]);
        }
      }
    }
    if (c < p.d_out) {
      for (int bb = 0; bb < nb; ++bb)
        p.part[((long long)blockIdx.y * p.batch + b0 + bb) * p.d_out + c] = acc[bb];
    }
  }
}

// The same product with four consecutive columns per thread (16-byte loads of M; d_out a
// multiple of 4): CTA (512-column tile, split), four rows of M in flight per thread.
__global__ void __launch_bounds__(kCols) absorbed_gemv4_kernel(const __grid_constant__ AbsorbParams p) {
  __shared__ float sa[8][128];
  const int c = (blockIdx.x * kCols + threadIdx.x) * 4;
  const int k0 = blockIdx.y * p.krows, k1 = min(p.m_rows, k0 + p.krows);
  const bool col_ok = c < p.d_out;
  {
    const int b0 = blockIdx.z * 8;  // 8 sequences per CTA; M is re-read from L2 by the others
    const int nb = min(8, p.batch - b0);
    float4 acc[8];
#pragma unroll
    for (int bb = 0; bb < 8; ++bb) acc[bb] = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int kk = k0; kk < k1; kk += 128) {
      const int kn = min(128, k1 - kk);
      __syncthreads();
      for (int i = threadIdx.x; i < 8 * 128; i += kCols) {
        const int bb = i >> 7, k = i & 127;
        sa[bb][k] = (bb < nb && k < kn) ? p.A[(long long)(b0 + bb) * p.m_rows + kk + k] : 0.f;
      }
      __syncthreads();
      if (col_ok) {
        const float* mk = p.M + (long long)kk * p.d_out + c;
        int k = 0;
        for (; k + 4 <= kn; k += 4) {
          float4 m[4];
#pragma unroll
          for (int u = 0; u < 4; ++u)
            m[u] = __ldg(reinterpret_cast<const float4*>(mk + (long long)(k + u) * p.d_out));
#pragma unroll
          for (int u = 0; u < 4; ++u) {
#pragma unroll
            for (int bb = 0; bb < 8; ++bb) {
              const float a = sa[bb][k + u];
              acc[bb].x = fmaf(a, m[u].x, acc[bb].x);
              acc[bb].y = fmaf(a, m[u].y, acc[bb].y);
              acc[bb].z = fmaf(a, m[u].z, acc[bb].z);
              acc[bb].w = fmaf(a, m[u].w, acc[bb].w);
            }
          }
        }
        for (; k < kn; ++k) {
          const float4 m0 = __ldg(reinterpret_cast<const float4*>(mk + (long long)k * p.d_out));
#pragma unroll
          for (int bb = 0; bb < 8; ++bb) {
            const float a = sa[bb][k];
            acc[bb].x = fmaf(a, m0.x, acc[bb].x);
            acc[bb].y = fmaf(a, m0.y, acc[bb].y);
            acc[bb].z = fmaf(a, m0.z, acc[bb].z);
            acc[bb].w = fmaf(a, m0.w, acc[bb].w);
          }
        }
      }
    }
    if (col_ok) {
      for (int bb = 0; bb < nb; ++bb)
        *reinterpret_cast<float4*>(p.part + ((long long)blockIdx.y * p.batch + b0 + bb) * p.d_out + c) = acc[bb];
    }
  }
}

// y[b][c] = sum_s part[s][b][c], in split order
__global__ void absorbed_reduce_kernel(const __grid_constant__ AbsorbParams p) {
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long n = (long long)p.batch * p.d_out;
  if (i >= n) return;
  float v = 0.f;
  for (int s = 0; s < p.ksplit; ++s) v += p.part[(long long)s * n + i];
  p.y[i] = v;
}

}  // namespace

cudaError_t launch_absorb_weights(const AbsorbParams& p, cudaStream_t s) {
  const dim3 grid((p.d_out + kCols - 1) / kCols, p.H);
  absorb_weights_kernel<<<grid, kCols, 0, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_absorbed_output(const AbsorbParams& p, cudaStream_t s) {
  if (p.batch == 0) return cudaSuccess;
  if (p.d_out % 4 == 0) {
    const dim3 grid((p.d_out / 4 + kCols - 1) / kCols, p.ksplit, (p.batch + 7) / 8);
    absorbed_gemv4_kernel<<<grid, kCols, 0, s>>>(p);
  } else {
    const dim3 grid((p.d_out + kCols - 1) / kCols, p.ksplit, (p.batch + 7) / 8);
    absorbed_gemv_kernel<<<grid, kCols, 0, s>>>(p);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const long long n = (long long)p.batch * p.d_out;
  absorbed_reduce_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace starkv
