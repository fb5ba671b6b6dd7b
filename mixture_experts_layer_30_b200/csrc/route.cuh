// Router and biased top-K selection: LongCat-Flash Technical Report, §2.1, Eq. (1).
#pragma once

#include "common.cuh"

namespace moe {

// --- router GEMM on CUDA cores ----------------------------------------------
// logits[t, e] = sum_j x[t, j] * w[e, j] (+ offset[t, e]), fp32 accumulation.
// 64x64 output tile per CTA, 256 threads, 4x4 outputs per thread.
constexpr int kRgBM = 64, kRgBN = 64, kRgBK = 16;

template <typename TIn>
__global__ void __launch_bounds__(256)
router_gemm_simt_kernel(const TIn* __restrict__ x, const TIn* __restrict__ w,
                        const float* __restrict__ offset, float* __restrict__ logits, int T,
                        int E, int d) {
  pdl_trigger();
  pdl_wait();
  __shared__ float As[kRgBK][kRgBM + 4];
  __shared__ float Bs[kRgBK][kRgBN + 4];
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const int m0 = blockIdx.y * kRgBM, n0 = blockIdx.x * kRgBN;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < d; k0 += kRgBK) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      int idx = tid + i * 256;       // 0..1023 over a 64 x 16 tile
      int r = idx >> 4, c = idx & 15;
      int gk = k0 + c;
      int gm = m0 + r, gn = n0 + r;
      As[c][r] = (gm < T && gk < d) ? Cvt<TIn>::to_f(x[(size_t)gm * d + gk]) : 0.f;
      Bs[c][r] = (gn < E && gk < d) ? Cvt<TIn>::to_f(w[(size_t)gn * d + gk]) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < kRgBK; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) { a[i] = As[kk][ty * 4 + i]; b[i] = Bs[kk][tx * 4 + i]; }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    int gm = m0 + ty * 4 + i;
    if (gm >= T) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      int gn = n0 + tx * 4 + j;
      if (gn >= E) continue;
      float v = acc[i][j];
      if (offset) v += offset[(size_t)gm * E + gn];
      logits[(size_t)gm * E + gn] = v;
    }
  }
}

// --- softmax + biased top-K + per-CTA histogram -----------------------------
// One warp per token.  Lane l holds experts e = l + 32*j, j < VPL.
// Selection key: (R_e + b_e) descending, then e ascending (lower index wins ties).

// Order-preserving map of a float to an unsigned key (larger float -> larger
// key); -0 is folded into +0 first.  Keys are > 0 for every float, so 0 means
// "no candidate".
MOE_DEV uint32_t ordered_key(float x) {
  const uint32_t u = __float_as_uint(x + 0.0f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Insert (v, j) into a lane's descending top-3 list; equal values keep the
// earlier (lower) j first.
struct Top3 {
  float v[3];
  float p[3];
  int j[3];
  MOE_DEV void clear() {
#pragma unroll
    for (int i = 0; i < 3; ++i) { v[i] = -INFINITY; p[i] = 0.f; j[i] = -1; }
  }
  MOE_DEV void insert(float vv, float pp, int jj) {
    if (j[2] >= 0 && !(vv > v[2])) return;
    if (j[1] < 0 || vv > v[1]) {
      v[2] = v[1]; p[2] = p[1]; j[2] = j[1];
      if (j[0] < 0 || vv > v[0]) {
        v[1] = v[0]; p[1] = p[0]; j[1] = j[0];
        v[0] = vv; p[0] = pp; j[0] = jj;
      } else {
        v[1] = vv; p[1] = pp; j[1] = jj;
      }
    } else {
      v[2] = vv; p[2] = pp; j[2] = jj;
    }
  }
  MOE_DEV void pop() {
    v[0] = v[1]; p[0] = p[1]; j[0] = j[1];
    v[1] = v[2]; p[1] = p[2]; j[1] = j[2];
    v[2] = -INFINITY; p[2] = 0.f; j[2] = -1;
  }
};

// kPsum: also accumulate the column sums of R (per-lane registers over the
// warp's tokens).  The biased scores are recomputed from R and the bias when a
// lane's top-3 list is rebuilt instead of being kept in registers, so up to 24
// scores per lane fit 64 registers and two CTAs share an SM (the LongCat shape,
// 8192 tokens, then runs as one wave).
template <int VPL, bool kPsum>
__global__ void __launch_bounds__(kRouteThreads, (kPsum || VPL > 24) ? 1 : 2)
softmax_topk_kernel(const float* __restrict__ logits, int nsplit, long long split_stride,
                    const float* __restrict__ bias, int T, int E, int N, int K,
                    int32_t* __restrict__ topk_idx,
                    float* __restrict__ topk_gate, uint8_t* __restrict__ n_ffn,
                    float* __restrict__ probs_out, int32_t* __restrict__ partial_hist,
                    float* __restrict__ partial_psum, unsigned int* ticket,
                    int32_t* __restrict__ counts_out, float* __restrict__ psum_out) {
  pdl_trigger();
  pdl_wait();
  __shared__ int hist[kMaxExperts];
  __shared__ float psum_acc[kMaxExperts];
  float ps[kPsum ? VPL : 1];  // this lane's running sums of R over the warp's tokens
#pragma unroll
  for (int j = 0; j < (kPsum ? VPL : 1); ++j) ps[j] = 0.f;
  for (int e = threadIdx.x; e < E; e += blockDim.x) hist[e] = 0;
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  const int t_begin = blockIdx.x * kRouteTokensPerCta;
  const int t_end = min(T, t_begin + kRouteTokensPerCta);
  for (int t = t_begin + warp; t < t_end; t += nwarps) {
    const float* lrow = logits + (size_t)t * E;
    float p[VPL];
    float m = -INFINITY;
#pragma unroll
    for (int j = 0; j < VPL; ++j) {
      int e = lane + 32 * j;
      if (e < E) {
        // split-K partial logits, summed in split order
        float v = lrow[e];
        for (int sp = 1; sp < nsplit; ++sp) v += lrow[sp * split_stride + e];
        p[j] = v;
      } else {
        p[j] = -INFINITY;
      }
      m = fmaxf(m, p[j]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    float sum = 0.f;
#pragma unroll
    for (int j = 0; j < VPL; ++j) {
      int e = lane + 32 * j;
      p[j] = e < E ? __expf(p[j] - m) : 0.f;
      sum += p[j];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    const float inv = 1.0f / sum;
    Top3 top;
    top.clear();
#pragma unroll
    for (int j = 0; j < VPL; ++j) {
      int e = lane + 32 * j;
      p[j] *= inv;                             // R_e
      if constexpr (kPsum) ps[j] += p[j];
      if (e < E) {
        if (probs_out) probs_out[(size_t)t * E + e] = p[j];
        top.insert(p[j] + __ldg(bias + e), p[j], j);  // biased score, selection only
      }
    }
    uint32_t taken = 0;
    int nf = 0;
    for (int k = 0; k < K; ++k) {
      // warp arg-max: largest score, then the smallest expert index among equals
      const uint32_t key = top.j[0] >= 0 ? ordered_key(top.v[0]) : 0u;
      const uint32_t mkey = __reduce_max_sync(0xffffffffu, key);
      const uint32_t cand =
          (key == mkey && top.j[0] >= 0) ? (uint32_t)(lane + 32 * top.j[0]) : 0xffffffffu;
      const int be = (int)__reduce_min_sync(0xffffffffu, cand);
      const int owner = be & 31;
      const float gate = __shfl_sync(0xffffffffu, top.p[0], owner);
      if (lane == owner) {
        taken |= 1u << top.j[0];
        top.pop();
        if (top.j[0] < 0) {
          // this lane's three best are used up: rebuild from what is left
#pragma unroll
          for (int j = 0; j < VPL; ++j)
            if (!(taken >> j & 1u) && lane + 32 * j < E)
              top.insert(p[j] + __ldg(bias + lane + 32 * j), p[j], j);
        }
      }
      if (lane == 0) {
        topk_idx[(size_t)t * K + k] = be;
        topk_gate[(size_t)t * K + k] = gate;
        atomicAdd(&hist[be], 1);
      }
      nf += be < N;
    }
    if (lane == 0) n_ffn[t] = (uint8_t)nf;
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x)
    partial_hist[(size_t)blockIdx.x * E + e] = hist[e];
  if (kPsum && partial_psum) {
    // column sums of R over the CTA's tokens, warps added in a fixed order
    for (int e = threadIdx.x; e < E; e += blockDim.x) psum_acc[e] = 0.f;
    __syncthreads();
    for (int w = 0; w < nwarps; ++w) {
      if (warp == w) {
#pragma unroll
        for (int j = 0; j < VPL; ++j) {
          const int e = lane + 32 * j;
          if (e < E) psum_acc[e] += ps[kPsum ? j : 0];
        }
      }
      __syncthreads();
    }
    for (int e = threadIdx.x; e < E; e += blockDim.x)
      partial_psum[(size_t)blockIdx.x * E + e] = psum_acc[e];
  }
  if (ticket) {
    // Small grids: the CTA that finishes last reduces the per-CTA partials
    // (the reduce kernels' per-expert order, so the sums are the same bits),
    // which saves their launch.  The ticket wraps back to 0 after the last CTA.
    __shared__ unsigned int s_last;
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) s_last = atomicInc(ticket, gridDim.x - 1) == gridDim.x - 1;
    __syncthreads();
    if (s_last) {
      __threadfence();
      const int nparts = gridDim.x;
      for (int e = warp; e < E; e += nwarps) {
        int c = 0;
        float q = 0.f;
        for (int p = lane; p < nparts; p += 32) {
          c += __ldcg(partial_hist + (size_t)p * E + e);
          if (psum_out) q += __ldcg(partial_psum + (size_t)p * E + e);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          c += __shfl_xor_sync(0xffffffffu, c, o);
          q += __shfl_xor_sync(0xffffffffu, q, o);
        }
        if (lane == 0) {
          counts_out[e] = c;
          if (psum_out) psum_out[e] = q;
        }
      }
    }
  }
}

// prob_sum[e] = sum over route CTAs of their column sums of R (lane-strided
// partial sums, then a fixed shuffle tree: the same order on every run).
__global__ void __launch_bounds__(256)
reduce_psum_kernel(const float* __restrict__ partial, int nparts, int E,
                   float* __restrict__ prob_sum) {
  pdl_trigger();
  pdl_wait();
  const int e = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (e >= E) return;
  float c = 0.f;
  for (int p = lane; p < nparts; p += 32) c += partial[(size_t)p * E + e];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
  if (lane == 0) prob_sum[e] = c;
}

// Device-level load-balance statistics with the zero-expert group, Eq. (3)-(5):
//   f_j = D/(K_e T) * sum_{i in group j} counts[i]      (j < D, groups of G = N/D)
//   f_D = 1/((K - K_e) T) * sum_{i >= N} counts[i]     (zero-computation experts)
//   P_j = (1/T) * sum_{i in group j} prob_sum[i],  L = alpha * sum_j f_j P_j
// One warp per group; integer selection counts, fp64 arithmetic, fp32 outputs.
__global__ void __launch_bounds__(1024)
lb_stats_kernel(int N, int Z, int D, const int32_t* __restrict__ counts,
                const float* __restrict__ prob_sum, long long T, int K, float K_e, float alpha,
                float* __restrict__ f_out, float* __restrict__ p_out, float* __restrict__ loss) {
  pdl_trigger();
  pdl_wait();
  __shared__ double f_sh[kMaxExperts + 1], p_sh[kMaxExperts + 1];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  const int G = N / D;
  for (int j = warp; j <= D; j += nwarps) {
    const int lo = j < D ? j * G : N, hi = j < D ? lo + G : N + Z;
    long long sel = 0;
    double pr = 0.0;
    for (int i = lo + lane; i < hi; i += 32) {
      sel += counts[i];
      pr += (double)prob_sum[i];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      sel += __shfl_xor_sync(0xffffffffu, sel, o);
      pr += __shfl_xor_sync(0xffffffffu, pr, o);
    }
    const double denom = j < D ? __dmul_rn((double)K_e, (double)T) / (double)D
                               : __dmul_rn((double)K - (double)K_e, (double)T);
    const double f = __ddiv_rn((double)sel, denom);
    const double P = __ddiv_rn(pr, (double)T);
    if (lane == 0) {
      f_out[j] = (float)f;
      p_out[j] = (float)P;
      f_sh[j] = f;
      p_sh[j] = P;
    }
  }
  __syncthreads();
  if (threadIdx.x == 0 && loss) {
    double acc = 0.0;
    for (int j = 0; j <= D; ++j) acc += f_sh[j] * p_sh[j];
    *loss = (float)((double)alpha * acc);
  }
}

// counts[e] = sum over route CTAs of their partial histograms.  One warp per
// expert; integer sums, so the result does not depend on the order.
__global__ void __launch_bounds__(256)
reduce_hist_kernel(const int32_t* __restrict__ partial, int nparts, int E,
                   int32_t* __restrict__ counts) {
  pdl_trigger();
  pdl_wait();
  const int e = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (e >= E) return;
  int c = 0;
  for (int p = lane; p < nparts; p += 32) c += partial[(size_t)p * E + e];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
  if (lane == 0) counts[e] = c;
}

}  // namespace moe
