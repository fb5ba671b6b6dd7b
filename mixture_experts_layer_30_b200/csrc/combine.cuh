// Weighted sum of Eq. (1) (LongCat-Flash Technical Report, §2.1) with the
// zero-computation experts folded into the epilogue: an identity expert adds
// g * x_t, so the Z identity slots of a token cost one FMA per element on the
// x row that is read anyway -- no FFN work and no extra rows.
//
// And the bias control of §2.1.1, Eq. (2).
#pragma once

#include "common.cuh"

namespace moe {

// One CTA per token; each thread owns 16-byte vectors of the d-vector.
// out = gamma * ( sum_{k: idx<N, in k order} g_k y[slot_k]  +  (sum_{k: idx>=N} g_k) x )
template <typename T>
__global__ void __launch_bounds__(256)
combine_kernel(const T* __restrict__ x, const T* __restrict__ y_perm,
               const int32_t* __restrict__ topk_idx, const float* __restrict__ topk_gate,
               const int32_t* __restrict__ slot_pos, int K, int N, int E, int d, int max_rows,
               float gamma, T* __restrict__ out, uint32_t* status) {
  pdl_trigger();
  pdl_wait();
  constexpr int VN = Vec16<T>::kN;
  __shared__ int s_row[kMaxExperts];
  __shared__ float s_g[kMaxExperts];
  __shared__ int s_nffn;
  __shared__ float s_zero;
  const int t = blockIdx.x;
  if (threadIdx.x < 32) {
    // Warp 0 reads the K slots 32 at a time, compacts the FFN slots in k order
    // and sums the zero-expert gates in k order (adding 0 for other slots
    // leaves the sum unchanged, so the order of the additions is exactly k).
    const int lane = threadIdx.x;
    const uint32_t lt = (1u << lane) - 1u;
    int n = 0;
    float zs = 0.f;
    for (int kb = 0; kb < K; kb += 32) {
      const int k = kb + lane;
      int e = -1, r = -1;
      float g = 0.f;
      if (k < K) {
        e = topk_idx[(size_t)t * K + k];
        g = topk_gate[(size_t)t * K + k];
        if (e >= 0 && e < N) r = slot_pos[(size_t)t * K + k];
      }
      if (k < K && (e < 0 || e >= E)) set_status(status, MOE_DEV_BAD_EXPERT_INDEX);
      const bool is_ffn = k < K && e >= 0 && e < N;
      const bool row_ok = r >= 0 && r < max_rows;
      if (is_ffn && !row_ok) set_status(status, MOE_DEV_BAD_OFFSETS);
      const uint32_t take = __ballot_sync(0xffffffffu, is_ffn && row_ok);
      if (is_ffn && row_ok) {
        const int pos = n + __popc(take & lt);
        s_row[pos] = r;
        s_g[pos] = g;
      }
      n += __popc(take);
      const float gz = (k < K && e >= N && e < E) ? g : 0.f;
#pragma unroll
      for (int j = 0; j < 32; ++j) zs += __shfl_sync(0xffffffffu, gz, j);
    }
    if (lane == 0) {
      s_nffn = n;
      s_zero = zs;
    }
  }
  __syncthreads();
  const int nffn = s_nffn;
  const float zs = s_zero;
  const int nvec = d / VN;
  const uint4* xv = reinterpret_cast<const uint4*>(x + (size_t)t * d);
  uint4* ov = reinterpret_cast<uint4*>(out + (size_t)t * d);
  for (int v = threadIdx.x; v < nvec; v += blockDim.x) {
    float acc[VN];
#pragma unroll
    for (int i = 0; i < VN; ++i) acc[i] = 0.f;
    for (int j = 0; j < nffn; ++j) {
      uint4 raw = __ldg(reinterpret_cast<const uint4*>(y_perm + (size_t)s_row[j] * d) + v);
      float f[VN];
      unpack16(raw, f, T());
      const float g = s_g[j];
#pragma unroll
      for (int i = 0; i < VN; ++i) acc[i] = fmaf(g, f[i], acc[i]);
    }
    float f[VN];
    unpack16(__ldg(xv + v), f, T());
#pragma unroll
    for (int i = 0; i < VN; ++i) acc[i] = gamma * fmaf(zs, f[i], acc[i]);
    ov[v] = pack16(acc, T());
  }
}

// Eq. (2): b_i += mu (K_e/K * 1/N - T_i/(K T_all)) for i < N; zero experts frozen.
// fp64 with explicit round-to-nearest operations (no contraction), one rounding to fp32.
__global__ void bias_update_kernel(int N, const int32_t* __restrict__ counts, long long T_all,
                                   int K, float K_e, float mu, float* __restrict__ bias) {
  pdl_trigger();
  pdl_wait();
  const double target = __ddiv_rn((double)K_e, __dmul_rn((double)K, (double)N));
  const double denom = __dmul_rn((double)K, (double)T_all);
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < N; i += gridDim.x * blockDim.x) {
    const double share = __ddiv_rn((double)counts[i], denom);
    const double delta = __dmul_rn((double)mu, __dsub_rn(target, share));
    bias[i] = __double2float_rn(__dadd_rn((double)bias[i], delta));
  }
}

}  // namespace moe
