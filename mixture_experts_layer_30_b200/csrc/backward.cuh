// Backward pass of the MoE layer with zero-computation experts
// (LongCat-Flash Technical Report, §2.1, Eq. (1); §2.3.2, Eq. (8) gamma):
// the memory-bound steps.  The expert and router contractions are in
// gemm_tc.cuh / gemm_wgrad.cuh (bf16) and gemm_simt_bwd.cuh (fp32).
//
//   combine_backward_kernel  dy = gamma g dout (FFN slots); dgate = gamma <dout, y | x>
//   dlogits_kernel           dlogits = R (dR - <R, dR>)    (softmax vector-Jacobian product)
//   permute_backward_kernel  dx = sum_k dx_row + gamma (sum of zero gates) dout (+ router term)
//
// Every reduction runs in a fixed order (per-thread sequential, then a fixed
// shuffle tree, then warps in index order), so two runs are bit-identical.
#pragma once

#include "common.cuh"

namespace moe {

constexpr int kCbBatch = 8;  // dot products reduced together by the combine backward

// Warp-level sum of v by a fixed xor-shuffle tree (every lane gets the total).
MOE_DEV float warp_sum_fixed(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// One CTA per token; each thread owns 16-byte vectors of the d-vector.
// Sources of the dot products: the FFN slots of the token (row of y_perm), in
// k order, then -- when the token has a zero-expert slot -- x_t once (every
// zero slot gets the same gamma <dout_t, x_t>).
template <typename T>
__global__ void __launch_bounds__(256)
combine_backward_kernel(const T* __restrict__ x, const T* __restrict__ y_perm,
                        const int32_t* __restrict__ topk_idx,
                        const float* __restrict__ topk_gate, const int32_t* __restrict__ slot_pos,
                        const T* __restrict__ dout, int K, int N, int E, int d, int max_rows,
                        float gamma, T* __restrict__ dy_perm, float* __restrict__ dgate,
                        uint32_t* status) {
  pdl_trigger();
  pdl_wait();
  constexpr int VN = Vec16<T>::kN;
  __shared__ int s_row[kMaxExperts + 1];  // -1: the x_t source
  __shared__ int s_k[kMaxExperts + 1];
  __shared__ float s_g[kMaxExperts + 1];
  __shared__ int s_n;
  __shared__ float s_part[8][kCbBatch];
  __shared__ float s_dot[kCbBatch];
  const int t = blockIdx.x;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nwarps = blockDim.x >> 5;
  if (threadIdx.x < 32) {
    const uint32_t lt = (1u << lane) - 1u;
    int n = 0;
    bool any_zero = false;
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
        s_k[pos] = k;
        s_g[pos] = g;
      }
      n += __popc(take);
      any_zero |= __any_sync(0xffffffffu, k < K && e >= N && e < E) != 0;
    }
    if (lane == 0) {
      if (any_zero) {
        s_row[n] = -1;
        s_k[n] = -1;
        s_g[n] = 0.f;
        ++n;
      }
      s_n = n;
    }
  }
  __syncthreads();
  const int nsrc = s_n;
  const int nvec = d / VN;
  const uint4* dv = reinterpret_cast<const uint4*>(dout + (size_t)t * d);
  for (int b0 = 0; b0 < nsrc; b0 += kCbBatch) {
    const int nb = min(kCbBatch, nsrc - b0);
    float part[kCbBatch];
#pragma unroll
    for (int j = 0; j < kCbBatch; ++j) part[j] = 0.f;
    for (int v = threadIdx.x; v < nvec; v += blockDim.x) {
      float g[VN];
      unpack16(__ldg(dv + v), g, T());
#pragma unroll
      for (int j = 0; j < kCbBatch; ++j) {
        if (j < nb) {
          const int r = s_row[b0 + j];
          const T* src = r >= 0 ? y_perm + (size_t)r * d : x + (size_t)t * d;
          float f[VN];
          unpack16(__ldg(reinterpret_cast<const uint4*>(src) + v), f, T());
          float acc = part[j];
#pragma unroll
          for (int i = 0; i < VN; ++i) acc = fmaf(g[i], f[i], acc);
          part[j] = acc;
          if (r >= 0) {
            const float s = gamma * s_g[b0 + j];
            float o[VN];
#pragma unroll
            for (int i = 0; i < VN; ++i) o[i] = s * g[i];
            reinterpret_cast<uint4*>(dy_perm + (size_t)r * d)[v] = pack16(o, T());
          }
        }
      }
    }
#pragma unroll
    for (int j = 0; j < kCbBatch; ++j) {
      const float w = warp_sum_fixed(part[j]);
      if (lane == 0) s_part[warp][j] = w;
    }
    __syncthreads();
    if (threadIdx.x < nb) {
      float s = 0.f;
      for (int w = 0; w < nwarps; ++w) s += s_part[w][threadIdx.x];
      s_dot[threadIdx.x] = gamma * s;
    }
    __syncthreads();
    // dgate of the FFN slots of this batch; the x_t source serves every zero slot
    if (threadIdx.x < nb) {
      const int j = b0 + threadIdx.x;
      if (s_row[j] >= 0) dgate[(size_t)t * K + s_k[j]] = s_dot[threadIdx.x];
    }
    if (b0 + nb == nsrc && s_row[nsrc - 1] < 0) {
      const float zdot = s_dot[nb - 1];
      for (int k = threadIdx.x; k < K; k += blockDim.x) {
        const int e = topk_idx[(size_t)t * K + k];
        if (e >= N && e < E) dgate[(size_t)t * K + k] = zdot;
      }
    }
    __syncthreads();
  }
}

// dlogits[t, i] = R[t, i] * (dR[t, i] - s_t),  s_t = sum_i R[t, i] dR[t, i],
// dR[t, idx_k] = dgate[t, k], plus -- with the load-balance loss of Eq. (3)-(5)
// -- c_i = lb_scale * lb_f[group(i)] on every expert (group(i) = i / G for
// i < N, D for the zero experts).  s_t sums the selected slots (k order per
// lane, then the fixed shuffle tree) and then adds sum_i R c (lane-strided,
// fixed tree).  One warp per token; dR is scattered into a per-warp shared row.
// Written as TOut (bf16 operand of the tensor-core router GEMMs, or fp32).
template <typename TOut>
__global__ void __launch_bounds__(256)
dlogits_kernel(const float* __restrict__ probs, const int32_t* __restrict__ topk_idx,
               const float* __restrict__ dgate, int T, int E, int K, const float* __restrict__ lb_f,
               int N, int G, int D, float lb_scale, TOut* __restrict__ dlogits, uint32_t* status) {
  pdl_trigger();
  pdl_wait();
  __shared__ float s_dR[8][kMaxExperts];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int t = blockIdx.x * 8 + warp;
  if (t >= T) return;
  float* dR = s_dR[warp];
  const float* p = probs + (size_t)t * E;
  for (int i = lane; i < E; i += 32) dR[i] = 0.f;
  __syncwarp();
  float s = 0.f;
  for (int k = lane; k < K; k += 32) {
    const int e = topk_idx[(size_t)t * K + k];
    const float g = dgate[(size_t)t * K + k];
    if (e >= 0 && e < E) {
      dR[e] = g;
      s = fmaf(p[e], g, s);
    } else {
      set_status(status, MOE_DEV_BAD_EXPERT_INDEX);
    }
  }
  s = warp_sum_fixed(s);
  if (lb_f) {
    __syncwarp();  // the scattered dR entries of other lanes are visible
    float s2 = 0.f;
    for (int i = lane; i < E; i += 32) {
      const float c = lb_scale * __ldg(lb_f + (i < N ? i / G : D));
      dR[i] += c;  // each lane owns entries i = lane + 32 m
      s2 = fmaf(p[i], c, s2);
    }
    s += warp_sum_fixed(s2);
  }
  __syncwarp();
  for (int i = lane; i < E; i += 32)
    dlogits[(size_t)t * E + i] = Cvt<TOut>::from_f(p[i] * (dR[i] - s));
}

// dx[t] = sum_{k: idx<N, in k order} dx_perm[slot_pos[t,k]]
//         + gamma * (sum_{k: idx>=N} g_k) * dout[t]  (+ dx_router[t])
// One CTA per token, 16-byte vectors, fp32 accumulation, one rounding.
template <typename T>
__global__ void __launch_bounds__(256)
permute_backward_kernel(const T* __restrict__ dout, const int32_t* __restrict__ topk_idx,
                        const float* __restrict__ topk_gate, const int32_t* __restrict__ slot_pos,
                        const T* __restrict__ dx_perm, const float* __restrict__ dx_router,
                        int K, int N, int E, int d, int max_rows, float gamma,
                        T* __restrict__ dx) {
  pdl_trigger();
  pdl_wait();
  constexpr int VN = Vec16<T>::kN;
  __shared__ int s_row[kMaxExperts];
  __shared__ int s_n;
  __shared__ float s_zero;
  const int t = blockIdx.x;
  if (threadIdx.x < 32) {
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
      const bool ok = k < K && e >= 0 && e < N && r >= 0 && r < max_rows;
      const uint32_t take = __ballot_sync(0xffffffffu, ok);
      if (ok) s_row[n + __popc(take & lt)] = r;
      n += __popc(take);
      const float gz = (k < K && e >= N && e < E) ? g : 0.f;
#pragma unroll
      for (int j = 0; j < 32; ++j) zs += __shfl_sync(0xffffffffu, gz, j);
    }
    if (lane == 0) {
      s_n = n;
      s_zero = zs;
    }
  }
  __syncthreads();
  const int n = s_n;
  const float zg = gamma * s_zero;
  const int nvec = d / VN;
  for (int v = threadIdx.x; v < nvec; v += blockDim.x) {
    float acc[VN];
#pragma unroll
    for (int i = 0; i < VN; ++i) acc[i] = 0.f;
    for (int j = 0; j < n; ++j) {
      float f[VN];
      unpack16(__ldg(reinterpret_cast<const uint4*>(dx_perm + (size_t)s_row[j] * d) + v), f, T());
#pragma unroll
      for (int i = 0; i < VN; ++i) acc[i] += f[i];
    }
    float g[VN];
    unpack16(__ldg(reinterpret_cast<const uint4*>(dout + (size_t)t * d) + v), g, T());
#pragma unroll
    for (int i = 0; i < VN; ++i) acc[i] = fmaf(zg, g[i], acc[i]);
    if (dx_router) {
      const float4* rr = reinterpret_cast<const float4*>(dx_router + (size_t)t * d + v * VN);
#pragma unroll
      for (int q = 0; q < VN / 4; ++q) {
        const float4 w = __ldg(rr + q);
        acc[4 * q] += w.x;
        acc[4 * q + 1] += w.y;
        acc[4 * q + 2] += w.z;
        acc[4 * q + 3] += w.w;
      }
    }
    reinterpret_cast<uint4*>(dx + (size_t)t * d)[v] = pack16(acc, T());
  }
}

}  // namespace moe
