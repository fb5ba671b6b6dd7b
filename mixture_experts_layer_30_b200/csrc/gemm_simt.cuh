// Grouped expert GEMMs on CUDA cores (fp32 path; also the small-shape bf16 path).
//
// For each FFN expert e with routed rows [offsets[e], offsets[e+1]) (row r of
// A is A[r], or A[a_rows[r]] when the rows are gathered from the token matrix):
//   gated (first half of the SwiGLU expert):
//       C[r, n] = SiLU(sum_k A[r,k] B0[e][n,k]) * (sum_k A[r,k] B1[e][n,k])
//   plain (second half):
//       C[r, n] = sum_k A[r,k] B0[e][n,k]
// fp32 FFMA accumulation (no TF32: its 10-bit mantissa is too coarse for an
// fp32 tolerance of 1e-4).  Persistent CTAs walk a (row chunk, column tile)
// list built from offsets[] in shared memory, so no host sync is needed to
// learn the routed row count.
#pragma once

#include "common.cuh"

namespace moe {

constexpr int kSgBM = 64, kSgBN = 64, kSgBK = 16;

template <typename TIn, bool kGated>
__global__ void __launch_bounds__(256)
grouped_gemm_simt_kernel(const TIn* __restrict__ A, const TIn* __restrict__ B0,
                         const TIn* __restrict__ B1, const int32_t* __restrict__ offsets,
                         int N, int max_rows, int n_out, int k_dim, TIn* __restrict__ C,
                         uint32_t* status, const int32_t* __restrict__ a_rows, int a_src_rows) {
  pdl_trigger();
  pdl_wait();
  __shared__ int prefix[kMaxExperts + 1];
  __shared__ int scan_tmp[33];
  __shared__ float As[kSgBK][kSgBM + 4];
  __shared__ float Bs[kGated ? 2 : 1][kSgBK][kSgBN + 4];
  build_chunk_prefix(offsets, N, max_rows, kSgBM, prefix, scan_tmp, status);
  const int ncol = (n_out + kSgBN - 1) / kSgBN;
  const int total = prefix[N] * ncol;
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
    const int chunk = tile / ncol, col = tile - chunk * ncol;
    const int e = find_expert(prefix, N, chunk);
    const int r0 = offsets[e] + (chunk - prefix[e]) * kSgBM;
    const int r1 = min(r0 + kSgBM, (int)offsets[e + 1]);
    const int n0 = col * kSgBN;
    const TIn* b0 = B0 + (size_t)e * n_out * k_dim;
    const TIn* b1 = kGated ? B1 + (size_t)e * n_out * k_dim : nullptr;
    float acc0[4][4] = {}, acc1[4][4] = {};
    for (int k0 = 0; k0 < k_dim; k0 += kSgBK) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        int idx = tid + i * 256;
        int r = idx >> 4, c = idx & 15;
        int gk = k0 + c;
        int gr = r0 + r, gn = n0 + r;
        float av = 0.f;
        if (gr < r1 && gk < k_dim) {
          // A row: routed row gr itself, or the token it came from (a_rows != NULL)
          int src = a_rows ? a_rows[gr] : gr;
          if (a_rows && (src < 0 || src >= a_src_rows)) src = -1;
          if (src >= 0) av = Cvt<TIn>::to_f(A[(size_t)src * k_dim + gk]);
        }
        As[c][r] = av;
        bool okb = gn < n_out && gk < k_dim;
        Bs[0][c][r] = okb ? Cvt<TIn>::to_f(b0[(size_t)gn * k_dim + gk]) : 0.f;
        if (kGated) Bs[kGated ? 1 : 0][c][r] = okb ? Cvt<TIn>::to_f(b1[(size_t)gn * k_dim + gk]) : 0.f;
      }
      __syncthreads();
#pragma unroll
      for (int kk = 0; kk < kSgBK; ++kk) {
        float a[4], b[4], g[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          a[i] = As[kk][ty * 4 + i];
          b[i] = Bs[0][kk][tx * 4 + i];
          if (kGated) g[i] = Bs[kGated ? 1 : 0][kk][tx * 4 + i];
        }
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            acc0[i][j] = fmaf(a[i], b[j], acc0[i][j]);
            if (kGated) acc1[i][j] = fmaf(a[i], g[j], acc1[i][j]);
          }
      }
      __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      int gr = r0 + ty * 4 + i;
      if (gr >= r1) continue;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        int gn = n0 + tx * 4 + j;
        if (gn >= n_out) continue;
        float v = kGated ? silu(acc0[i][j]) * acc1[i][j] : acc0[i][j];
        C[(size_t)gr * n_out + gn] = Cvt<TIn>::from_f(v);
      }
    }
  }
}

}  // namespace moe
