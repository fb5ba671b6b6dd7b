// Contractions of the backward pass on CUDA cores (fp32 path, and the bf16
// path for shapes the tensor-core kernels do not take).  One strided kernel
// covers every product of the backward pass of Eq. (1):
//
//   row-segment form (token-row gradients; the routed rows of expert e, or the
//   T rows of one matrix, are the output rows):
//       C[r, n] = sum_k A[r*a_sm + k*a_sk] * B_e(k, n)
//       B_e(k, n) = B0[e*b_seg + k*b_sk + n*b_sn]                for k <  k_split
//                 = B1[e*b_seg + (k - k_split)*b_sk + n*b_sn]     for k >= k_split
//     (k_split joins dx = da W1 + du W3 into one reduction over 2I)
//   K-segment form (weight gradients; the reduction runs over the rows of
//   segment e):
//       C[e*c_seg + m*c_sm + n] = sum_{r in segment e} A[r*a_sk + m*a_sm] * B0[r*b_sk + n*b_sn]
//
// Epilogues: plain store, or the SwiGLU backward of the expert FFN:
//   dh = the product;  with a = au[r, n], u = au[r, N + n], s = sigma(a):
//   C[r, n] = da = dh u s (1 + a (1 - s)),   C[r, N + n] = du = dh a s.
// fp32 FFMA accumulation in k order per output, so results are deterministic.
#pragma once

#include "common.cuh"

namespace moe {

struct SimtBwdArgs {
  const void* A;
  long long a_sm, a_sk;
  const void* B0;
  const void* B1;
  int k_split;
  long long b_sk, b_sn, b_seg;
  void* C;
  long long c_sm, c_seg;
  const int32_t* offsets;  // segment offsets [nseg + 1], or NULL for one segment
  int nseg;
  int single_rows;         // rows of the single segment when offsets == NULL
  int max_rows;            // bound for offsets
  int M;                   // K-segment form: output rows per segment
  int N;                   // output columns
  int Kd;                  // row-segment form: reduction length
  const void* au;          // SwiGLU backward: [rows, 2N] pre-activations a | u
  uint32_t* status;
};

constexpr int kSbBM = 64, kSbBN = 64, kSbBK = 16;

template <typename T, bool kKSeg, bool kSwiglu>
__global__ void __launch_bounds__(256) gemm_simt_bwd_kernel(const SimtBwdArgs p) {
  pdl_trigger();
  pdl_wait();
  __shared__ int prefix[kMaxExperts + 1];
  __shared__ int scan_tmp[33];
  __shared__ float As[kSbBK][kSbBM + 4];
  __shared__ float Bs[kSbBK][kSbBN + 4];
  const T* A = static_cast<const T*>(p.A);
  const T* B0 = static_cast<const T*>(p.B0);
  const T* B1 = static_cast<const T*>(p.B1);
  T* C = static_cast<T*>(p.C);
  const int nseg = p.offsets ? p.nseg : 1;
  const int ncol = (p.N + kSbBN - 1) / kSbBN;
  int total;
  if (!kKSeg) {
    if (p.offsets) {
      build_chunk_prefix(p.offsets, nseg, p.max_rows, kSbBM, prefix, scan_tmp, p.status);
    } else {
      if (threadIdx.x == 0) {
        prefix[0] = 0;
        prefix[1] = (p.single_rows + kSbBM - 1) / kSbBM;
      }
      __syncthreads();
    }
    total = prefix[nseg] * ncol;
  } else {
    total = nseg * ((p.M + kSbBM - 1) / kSbBM) * ncol;
  }
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
    int e, m0, n0, klen, lo = 0, mlim;
    if (!kKSeg) {
      const int chunk = tile / ncol;
      n0 = (tile - chunk * ncol) * kSbBN;
      e = p.offsets ? find_expert(prefix, nseg, chunk) : 0;
      const int s0 = p.offsets ? p.offsets[e] : 0;
      const int s1 = p.offsets ? p.offsets[e + 1] : p.single_rows;
      m0 = s0 + (chunk - prefix[e]) * kSbBM;
      mlim = min(m0 + kSbBM, s1);
      klen = p.Kd;
    } else {
      const int mblk = (p.M + kSbBM - 1) / kSbBM;
      e = tile / (mblk * ncol);
      const int rem = tile - e * mblk * ncol;
      m0 = (rem / ncol) * kSbBM;
      n0 = (rem % ncol) * kSbBN;
      mlim = min(m0 + kSbBM, p.M);
      if (p.offsets) {
        lo = p.offsets[e];
        int hi = p.offsets[e + 1];
        if (lo < 0 || hi < lo || hi > p.max_rows) {
          set_status(p.status, MOE_DEV_BAD_OFFSETS);
          lo = hi = 0;
        }
        klen = hi - lo;
      } else {
        klen = p.single_rows;
      }
    }
    float acc[4][4] = {};
    for (int k0 = 0; k0 < klen; k0 += kSbBK) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int idx = tid + i * 256;
        const int r = idx >> 4, c = idx & 15;  // r: row/col inside the tile, c: k offset
        const int gk = k0 + c;
        const int gm = m0 + r, gn = n0 + r;
        float av = 0.f, bv = 0.f;
        if (gk < klen && gm < mlim) {
          if (!kKSeg) av = Cvt<T>::to_f(A[(size_t)gm * p.a_sm + (size_t)gk * p.a_sk]);
          else av = Cvt<T>::to_f(A[(size_t)(lo + gk) * p.a_sk + (size_t)gm * p.a_sm]);
        }
        if (gk < klen && gn < p.N) {
          if (!kKSeg) {
            const bool second = p.k_split > 0 && gk >= p.k_split;
            const T* b = second ? B1 : B0;
            const int kk = second ? gk - p.k_split : gk;
            bv = Cvt<T>::to_f(b[(size_t)e * p.b_seg + (size_t)kk * p.b_sk + (size_t)gn * p.b_sn]);
          } else {
            bv = Cvt<T>::to_f(B0[(size_t)(lo + gk) * p.b_sk + (size_t)gn * p.b_sn]);
          }
        }
        As[c][r] = av;
        Bs[c][r] = bv;
      }
      __syncthreads();
#pragma unroll
      for (int kk = 0; kk < kSbBK; ++kk) {
        float a[4], b[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          a[i] = As[kk][ty * 4 + i];
          b[i] = Bs[kk][tx * 4 + i];
        }
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
      }
      __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int gm = m0 + ty * 4 + i;
      if (gm >= mlim) continue;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int gn = n0 + tx * 4 + j;
        if (gn >= p.N) continue;
        if (kSwiglu) {
          const T* au = static_cast<const T*>(p.au) + (size_t)gm * 2 * p.N;
          const float a = Cvt<T>::to_f(au[gn]);
          const float u = Cvt<T>::to_f(au[p.N + gn]);
          const float s = 1.0f / (1.0f + expf(-a));
          const float dh = acc[i][j];
          T* c = C + (size_t)gm * 2 * p.N;
          c[gn] = Cvt<T>::from_f(dh * u * s * (1.0f + a * (1.0f - s)));
          c[p.N + gn] = Cvt<T>::from_f(dh * a * s);
        } else if (!kKSeg) {
          C[(size_t)gm * p.c_sm + gn] = Cvt<T>::from_f(acc[i][j]);
        } else {
          C[(size_t)e * p.c_seg + (size_t)gm * p.c_sm + gn] = Cvt<T>::from_f(acc[i][j]);
        }
      }
    }
  }
}

}  // namespace moe
