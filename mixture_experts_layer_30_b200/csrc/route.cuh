// Router and biased top-K selection: LongCat-Flash Technical Report, §2.1, Eq. (1).
//
// Two routes to the same result:
//   * small batches (decode, the fp32 layers): route_small_kernel, one launch.
//     A cluster of CTAs computes a block of tokens' logits with fp32 FMAs, each
//     CTA over its own slice of the hidden dimension; CTA 0 of each token group
//     adds the slices in rank order through distributed shared memory, then runs
//     the softmax and the selection.  When one cluster holds every token group,
//     group 0's leader adds the groups' histograms over distributed shared
//     memory; otherwise the last cluster to finish reduces the per-cluster
//     histograms from global memory into the counts.
//   * large batches: the tensor-core router GEMM writes fp32 logits (and zeroes
//     the counts), then topk_kernel selects, one warp per token, and adds its
//     CTA's histogram to the counts with integer atomics (order-independent, so
//     the counts are exact and reproducible).
// Both use route_token: softmax over all N+Z experts in fp32, then the K
// largest R + b (ties to the lower index): the scores at or above the K-th
// largest lane maximum are sorted across the warp (K rounds of a warp arg-max
// when they do not fit one per lane).
#pragma once

#include <cooperative_groups.h>

#include "common.cuh"

namespace moe {

// --- router GEMM on CUDA cores ----------------------------------------------
// logits[t, e] = sum_j x[t, j] * w[e, j] (+ offset[t, e]), fp32 accumulation.
// 64x64 output tile per CTA, 256 threads, 4x4 outputs per thread.  CTA (0, 0)
// also zeroes `zero_counts` [zero_n] for the selection kernel that follows.
constexpr int kRgBM = 64, kRgBN = 64, kRgBK = 16;

template <typename TIn>
__global__ void __launch_bounds__(256)
router_gemm_simt_kernel(const TIn* __restrict__ x, const TIn* __restrict__ w,
                        const float* __restrict__ offset, float* __restrict__ logits, int T,
                        int E, int d, int32_t* __restrict__ zero_counts, int zero_n) {
  pdl_trigger();
  pdl_wait();
  __shared__ float As[kRgBK][kRgBM + 4];
  __shared__ float Bs[kRgBK][kRgBN + 4];
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  if (zero_counts && blockIdx.x == 0 && blockIdx.y == 0)
    for (int i = tid; i < zero_n; i += blockDim.x) zero_counts[i] = 0;
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

// --- selection of one token in one warp --------------------------------------

// Order-preserving map of a float to an unsigned key (larger float -> larger
// key); -0 is folded into +0 first.  Keys are > 0 for every float, so 0 means
// "no candidate".
MOE_DEV uint32_t ordered_key(float x) {
  const uint32_t u = __float_as_uint(x + 0.0f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Which experts a lane holds.  Strided: lane l holds e = l + 32 j.  Vec4 (row
// loads of 16 bytes): lane l holds e = 128 (j/4) + 4 l + j%4.  In both, a
// lane's experts increase with j.
template <bool kVec4> struct Lanes {
  static MOE_DEV int expert(int lane, int j) {
    return kVec4 ? 128 * (j >> 2) + 4 * lane + (j & 3) : lane + 32 * j;
  }
  static MOE_DEV int owner(int e) { return kVec4 ? (e >> 2) & 31 : e & 31; }
};

// A lane's two best candidates (biased score s, probability p, slot j; j = -1
// when empty).  Values are offered in ascending j and only a strictly larger
// score moves ahead, so equal scores keep the lower expert first.
struct Best2 {
  float s0, s1, p0, p1;
  int j0, j1;
  MOE_DEV void clear() {
    s0 = s1 = -INFINITY;
    p0 = p1 = 0.f;
    j0 = j1 = -1;
  }
  MOE_DEV void offer(float s, float p, int j) {
    if (j0 < 0 || s > s0) {
      s1 = s0; p1 = p0; j1 = j0;
      s0 = s; p0 = p; j0 = j;
    } else if (j1 < 0 || s > s1) {
      s1 = s; p1 = p; j1 = j;
    }
  }
  MOE_DEV void pop() {
    s0 = s1; p0 = p1; j0 = j1;
    s1 = -INFINITY; p1 = 0.f; j1 = -1;
  }
};

MOE_DEV float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
// Butterfly sum: every lane ends with the same bits (each step adds the same
// two numbers on both partners).
MOE_DEV float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Sorts one value per lane across the warp, descending (bitonic network, 15
// compare-exchange steps).  Equal values never swap.
MOE_DEV float warp_sort_desc(float v, int lane) {
#pragma unroll
  for (int k = 2; k <= 32; k <<= 1)
#pragma unroll
    for (int j = k >> 1; j > 0; j >>= 1) {
      const float o = __shfl_xor_sync(0xffffffffu, v, j);
      const bool keep_max = ((lane & k) == 0) == ((lane & j) == 0);
      if (keep_max ? (o > v) : (o < v)) v = o;
    }
  return v;
}
// The same network on (key, payload) pairs; keys are distinct except 0 (empty).
MOE_DEV void warp_sort_desc(unsigned long long& key, float& pay, int lane) {
#pragma unroll
  for (int k = 2; k <= 32; k <<= 1)
#pragma unroll
    for (int j = k >> 1; j > 0; j >>= 1) {
      const unsigned long long ok = __shfl_xor_sync(0xffffffffu, key, j);
      const float op = __shfl_xor_sync(0xffffffffu, pay, j);
      const bool keep_max = ((lane & k) == 0) == ((lane & j) == 0);
      if (keep_max ? (ok > key) : (ok < key)) {
        key = ok;
        pay = op;
      }
    }
}

// Softmax and biased top-K of token t.  v: this lane's logits (any value for
// experts >= E) -> its probabilities R (0 for experts >= E).  b: its biases.
// Writes topk_idx/topk_gate[t, 0..K), n_ffn[t] and adds the K choices to the
// shared histogram `hist`.  cand_key / cand_p: this warp's 32-entry scratch in
// shared memory.
//
// Selection.  Every one of the K best scores is at least tau, the K-th largest
// of the 32 lane maxima (those K lanes hold K scores >= tau).  So the scores
// >= tau are the candidates; when there are at most 32 of them (always, in
// practice, for K <= 32) they are gathered one per lane and sorted by (score
// descending, expert ascending), and lane k takes the k-th.  Otherwise K rounds
// of a warp arg-max over each lane's two best candidates select them.
template <int VPL, bool kVec4>
MOE_DEV void route_token(float (&v)[VPL], const float (&b)[VPL], int lane, int E, int N, int K,
                         int t, int32_t* __restrict__ topk_idx, float* __restrict__ topk_gate,
                         uint8_t* __restrict__ n_ffn, int* hist,
                         unsigned long long* cand_key, float* cand_p) {
  using L = Lanes<kVec4>;
  float m = -INFINITY;
#pragma unroll
  for (int j = 0; j < VPL; ++j)
    if (L::expert(lane, j) < E) m = fmaxf(m, v[j]);
  m = warp_max(m);
  float sum = 0.f;
#pragma unroll
  for (int j = 0; j < VPL; ++j) {
    v[j] = L::expert(lane, j) < E ? __expf(v[j] - m) : 0.f;
    sum += v[j];
  }
  sum = warp_sum(sum);
  const float inv = 1.0f / sum;
  float lmax = -INFINITY;
#pragma unroll
  for (int j = 0; j < VPL; ++j) {
    v[j] *= inv;  // R_e
    if (L::expert(lane, j) < E) lmax = fmaxf(lmax, v[j] + b[j]);  // biased score: selection only
  }
  if (K <= 32) {
    const float tau = __shfl_sync(0xffffffffu, warp_sort_desc(lmax, lane), K - 1);
    int cnt = 0;
#pragma unroll
    for (int j = 0; j < VPL; ++j) cnt += (L::expert(lane, j) < E && v[j] + b[j] >= tau);
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += n;
    }
    const int total = __shfl_sync(0xffffffffu, incl, 31);
    if (total <= 32) {
      int pos = incl - cnt;
#pragma unroll
      for (int j = 0; j < VPL; ++j) {
        const int e = L::expert(lane, j);
        const float sc = v[j] + b[j];
        if (e < E && sc >= tau) {
          cand_key[pos] = ((unsigned long long)ordered_key(sc) << 32) | (0xffffffffu - (uint32_t)e);
          cand_p[pos] = v[j];
          ++pos;
        }
      }
      __syncwarp();
      unsigned long long key = lane < total ? cand_key[lane] : 0ull;
      float gate = lane < total ? cand_p[lane] : 0.f;
      __syncwarp();
      warp_sort_desc(key, gate, lane);
      const int e = (int)(0xffffffffu - (uint32_t)key);
      if (lane < K) {
        topk_idx[(size_t)t * K + lane] = e;
        topk_gate[(size_t)t * K + lane] = gate;
        atomicAdd(&hist[e], 1);
      }
      const uint32_t ffn = __ballot_sync(0xffffffffu, lane < K && e < N);
      if (lane == 0) n_ffn[t] = (uint8_t)__popc(ffn);
      return;
    }
  }
  // ---- K rounds of a warp arg-max (K > 32, or more than 32 candidates) ----
  Best2 best;
  best.clear();
#pragma unroll
  for (int j = 0; j < VPL; ++j)
    if (L::expert(lane, j) < E) best.offer(v[j] + b[j], v[j], j);
  uint32_t taken = 0;
  int nf = 0, my_idx = -1;
  float my_gate = 0.f;
  for (int k = 0; k < K; ++k) {
    // warp arg-max: the largest score, then the smallest expert among equals
    const uint32_t key = best.j0 >= 0 ? ordered_key(best.s0) : 0u;
    const uint32_t mkey = __reduce_max_sync(0xffffffffu, key);
    const uint32_t cand =
        (best.j0 >= 0 && key == mkey) ? (uint32_t)L::expert(lane, best.j0) : 0xffffffffu;
    const int be = (int)__reduce_min_sync(0xffffffffu, cand);
    const int owner = L::owner(be);
    const float gate = __shfl_sync(0xffffffffu, best.p0, owner);
    if (lane == owner && best.j0 >= 0) {
      taken |= 1u << best.j0;
      best.pop();
      if (best.j0 < 0) {
        // both candidates of this lane are used: rebuild from what is left
#pragma unroll
        for (int j = 0; j < VPL; ++j)
          if (!((taken >> j) & 1u) && L::expert(lane, j) < E) best.offer(v[j] + b[j], v[j], j);
      }
    }
    if (K <= 32) {
      if (lane == k) {
        my_idx = be;
        my_gate = gate;
      }
    } else if (lane == 0) {
      topk_idx[(size_t)t * K + k] = be;
      topk_gate[(size_t)t * K + k] = gate;
      if ((unsigned)be < (unsigned)E) atomicAdd(&hist[be], 1);
    }
    nf += be < N;
  }
  if (K <= 32 && lane < K) {
    topk_idx[(size_t)t * K + lane] = my_idx;
    topk_gate[(size_t)t * K + lane] = my_gate;
    if ((unsigned)my_idx < (unsigned)E) atomicAdd(&hist[my_idx], 1);
  }
  if (lane == 0) n_ffn[t] = (uint8_t)nf;
}

// --- large batches: selection from the router GEMM's logits -------------------
// One warp per token, tokens strided over a grid of at most kTopkMaxCtas CTAs.
// logits: nsplit fp32 slabs [T, E] (split-K partials, added in split order).
// counts must be zero on entry (the router GEMM clears them).
constexpr int kTopkWarps = 8;
constexpr int kTopkMaxCtas = 1024;

template <int VPL, bool kVec4>
MOE_DEV void load_logits(const float* __restrict__ row, int lane, int E, float (&v)[VPL]) {
  if constexpr (kVec4) {
#pragma unroll
    for (int q = 0; q < VPL / 4; ++q) {
      const int e = 128 * q + 4 * lane;
      float4 f = make_float4(0.f, 0.f, 0.f, 0.f);
      if (e < E) f = __ldcs(reinterpret_cast<const float4*>(row + e));
      v[4 * q] = f.x; v[4 * q + 1] = f.y; v[4 * q + 2] = f.z; v[4 * q + 3] = f.w;
    }
  } else {
#pragma unroll
    for (int j = 0; j < VPL; ++j) {
      const int e = lane + 32 * j;
      v[j] = e < E ? __ldcs(row + e) : 0.f;
    }
  }
}

template <int VPL, bool kVec4, bool kPsum>
__global__ void __launch_bounds__(kTopkWarps * 32, VPL <= 12 ? 3 : VPL <= 24 ? 2 : 1)
topk_kernel(const float* __restrict__ logits, int nsplit, long long split_stride,
            const float* __restrict__ bias, int T, int E, int N, int K,
            int32_t* __restrict__ topk_idx, float* __restrict__ topk_gate,
            uint8_t* __restrict__ n_ffn, float* __restrict__ probs_out,
            int32_t* __restrict__ counts, float* __restrict__ partial_psum) {
  pdl_trigger();
  using L = Lanes<kVec4>;
  __shared__ int hist[kMaxExperts];
  __shared__ __align__(16) float bias_sh[kMaxExperts];
  __shared__ float psum_acc[kPsum ? kMaxExperts : 1];
  __shared__ unsigned long long cand_key[kTopkWarps][32];
  __shared__ float cand_p[kTopkWarps][32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int e = threadIdx.x; e < E; e += blockDim.x) hist[e] = 0;
  pdl_wait();
  for (int e = threadIdx.x; e < E; e += blockDim.x) bias_sh[e] = bias[e];
  float ps[kPsum ? VPL : 1];
#pragma unroll
  for (int j = 0; j < (kPsum ? VPL : 1); ++j) ps[j] = 0.f;
  __syncthreads();
  for (int t = blockIdx.x * kTopkWarps + warp; t < T; t += gridDim.x * kTopkWarps) {
    const float* row = logits + (size_t)t * E;
    float v[VPL];
    load_logits<VPL, kVec4>(row, lane, E, v);
    // split-K partials: loads of several slabs in flight, added in split order
    constexpr int kU = VPL <= 4 ? 8 : VPL <= 8 ? 2 : 1;
    for (int s0 = 1; s0 < nsplit; s0 += kU) {
      float pv[kU][VPL];
#pragma unroll
      for (int u = 0; u < kU; ++u)
        if (s0 + u < nsplit) load_logits<VPL, kVec4>(row + (s0 + u) * split_stride, lane, E, pv[u]);
#pragma unroll
      for (int u = 0; u < kU; ++u)
        if (s0 + u < nsplit) {
#pragma unroll
          for (int j = 0; j < VPL; ++j) v[j] += pv[u][j];
        }
    }
    float b[VPL];
#pragma unroll
    for (int j = 0; j < VPL; ++j) {
      const int e = L::expert(lane, j);
      b[j] = e < E ? bias_sh[e] : 0.f;
    }
    route_token<VPL, kVec4>(v, b, lane, E, N, K, t, topk_idx, topk_gate, n_ffn, hist,
                            cand_key[warp], cand_p[warp]);
    if (probs_out) {
#pragma unroll
      for (int j = 0; j < VPL; ++j) {
        const int e = L::expert(lane, j);
        if (e < E) probs_out[(size_t)t * E + e] = v[j];
      }
    }
    if constexpr (kPsum) {
#pragma unroll
      for (int j = 0; j < VPL; ++j) ps[j] += v[j];
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    const int c = hist[e];
    if (c) atomicAdd(counts + e, c);
  }
  if constexpr (kPsum) {
    // column sums of R over the CTA's tokens, warps added in a fixed order
    for (int e = threadIdx.x; e < E; e += blockDim.x) psum_acc[e] = 0.f;
    __syncthreads();
    for (int w = 0; w < kTopkWarps; ++w) {
      if (warp == w) {
#pragma unroll
        for (int j = 0; j < VPL; ++j) {
          const int e = L::expert(lane, j);
          if (e < E) psum_acc[e] += ps[j];
        }
      }
      __syncthreads();
    }
    for (int e = threadIdx.x; e < E; e += blockDim.x)
      partial_psum[(size_t)blockIdx.x * E + e] = psum_acc[e];
  }
}

// --- small batches: router + selection in one launch ---------------------------
// Grid (CL, ceil(T / kSmallTokens)): grid row g is the token group of tokens
// g*8 .. g*8+7; CTA (r, g) owns the hidden slice [r*slice, (r+1)*slice), slice =
// 32 lanes x 16-byte vectors x KIT.  Warp w computes experts w, w+8, ...: lane l
// accumulates its vectors of the slice for the 8 tokens with fp32 FMAs, then a
// fixed shuffle tree sums the 32 lanes.  The group's leader, CTA (0, g), adds the
// CL slices in rank order (+ the logit offset) and routes token g*8 + w in warp w.
// Clusters are (CL, G): G = 1 (one group per cluster, a ticket finds the last
// group) or G = every group of the batch (no ticket: group 0's leader adds the
// leaders' histograms and column sums in group order over distributed shared
// memory).  Both orders of the column sums are the same: tokens of a group in
// order, then groups in order.
constexpr int kSmallTokens = 8;
constexpr int kSmallThreads = 256;
constexpr int kSmallMaxCluster = 8;       // CTAs of one token group
constexpr int kSmallMaxWholeCluster = 16;  // CTAs of a cluster holding every group

// One cluster barrier phase in two halves: arrive (releasing this thread's
// earlier memory operations, loads of distributed shared memory included) and
// wait (acquiring every other thread's).  All threads of the cluster take the
// same phases.
MOE_DEV void cluster_arrive() { asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory"); }
MOE_DEV void cluster_wait() { asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory"); }

// Sums acc[0..8) over the warp's 32 lanes; lane l returns the total of token
// ((l >> 4) & 1) * 4 + ((l >> 3) & 1) * 2 + ((l >> 2) & 1) (lanes that differ
// only in bits 0-1 hold the same total).
MOE_DEV float transpose_sum8(const float (&acc)[8], int lane) {
  const bool h16 = lane & 16, h8 = lane & 8, h4 = lane & 4;
  float r4[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const float send = h16 ? acc[q] : acc[q + 4];
    const float keep = h16 ? acc[q + 4] : acc[q];
    r4[q] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
  }
  float r2[2];
#pragma unroll
  for (int q = 0; q < 2; ++q) {
    const float send = h8 ? r4[q] : r4[q + 2];
    const float keep = h8 ? r4[q + 2] : r4[q];
    r2[q] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
  }
  float r1 = (h4 ? r2[1] : r2[0]) + __shfl_xor_sync(0xffffffffu, h4 ? r2[0] : r2[1], 4);
  r1 += __shfl_xor_sync(0xffffffffu, r1, 2);
  r1 += __shfl_xor_sync(0xffffffffu, r1, 1);
  return r1;
}

// Dispatch layout of a whole batch of T <= kSmallThreads tokens, built by the
// one CTA that finishes the route (the layout moe_permute builds, without the
// copy of the token rows): experts 0..N-1 in order, tokens ascending inside an
// expert.  Thread t takes token t.  Bit l of bits[w][e] is set when token
// 32w + l chose FFN expert e (a token chooses an expert at most once); expert
// e's rows start at offsets[e], the rows of earlier experts, and token t's row
// is that start plus the bits of earlier tokens.  scratch: 17*N ints of shared
// memory; scan_tmp: 33 ints.
MOE_DEV void small_layout(const int32_t* __restrict__ topk_idx, int T, int K, int N,
                          int* scratch, int* scan_tmp, int32_t* __restrict__ offsets,
                          int32_t* __restrict__ row_token, int32_t* __restrict__ slot_pos) {
  uint32_t* bits = reinterpret_cast<uint32_t*>(scratch);  // [8][N]
  int* wbase = scratch + 8 * N;                            // [8][N]
  int* tot = scratch + 16 * N;                             // [N]
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int t = threadIdx.x;
  for (int i = threadIdx.x; i < 8 * N; i += blockDim.x) bits[i] = 0;
  __syncthreads();
  if (t < T)
    for (int k = 0; k < K; ++k) {
      const int e = __ldcg(topk_idx + (size_t)t * K + k);
      if (e < N) atomicOr(&bits[warp * N + e], 1u << lane);
    }
  __syncthreads();
  // exclusive scan over experts: each thread owns a run of consecutive experts
  const int per = (N + blockDim.x - 1) / blockDim.x;
  const int lo = min(N, (int)threadIdx.x * per), hi = min(N, lo + per);
  int local = 0;
  for (int e = lo; e < hi; ++e) {
    int c = 0;
#pragma unroll
    for (int w = 0; w < 8; ++w) c += __popc(bits[w * N + e]);
    tot[e] = c;
    local += c;
  }
  int run = block_exclusive_scan(local, scan_tmp, &scan_tmp[32]);
  for (int e = lo; e < hi; ++e) {
    offsets[e] = run;
    int b = run;
#pragma unroll
    for (int w = 0; w < 8; ++w) {
      wbase[w * N + e] = b;
      b += __popc(bits[w * N + e]);
    }
    run += tot[e];
  }
  if (threadIdx.x == 0) offsets[N] = scan_tmp[32];
  __syncthreads();
  if (t < T) {
    const uint32_t lt = (1u << lane) - 1u;
    for (int k = 0; k < K; ++k) {
      const int e = __ldcg(topk_idx + (size_t)t * K + k);
      int row = -1;
      if (e < N) {
        row = wbase[warp * N + e] + __popc(bits[warp * N + e] & lt);
        row_token[row] = t;
      }
      slot_pos[(size_t)t * K + k] = row;
    }
  }
}
// Largest N whose layout tables fit the kernel's slice array (8 x kMaxExperts floats).
constexpr int kSmallLayoutMaxN = 8 * kMaxExperts / 17;

template <typename TIn, int KIT, int VPL>
__global__ void __launch_bounds__(kSmallThreads)
route_small_kernel(const TIn* __restrict__ x, const TIn* __restrict__ w,
                   const float* __restrict__ offset, const float* __restrict__ bias, int T, int d,
                   int E, int N, int K, int32_t* __restrict__ topk_idx,
                   float* __restrict__ topk_gate, uint8_t* __restrict__ n_ffn,
                   float* __restrict__ probs_out, int32_t* __restrict__ part_hist,
                   float* __restrict__ part_psum, unsigned int* ticket,
                   int32_t* __restrict__ counts, float* __restrict__ prob_sum,
                   int32_t* __restrict__ offsets, int32_t* __restrict__ row_token,
                   int32_t* __restrict__ slot_pos) {
  pdl_trigger();
  namespace cg = cooperative_groups;
  constexpr int VEC = 16 / sizeof(TIn);
  __shared__ float part[kSmallTokens][kMaxExperts];
  __shared__ int hist[kMaxExperts];
  __shared__ float bias_sh[kMaxExperts];
  __shared__ float colsum[kMaxExperts];
  __shared__ unsigned long long cand_key[kSmallThreads / 32][32];
  __shared__ float cand_p[kSmallThreads / 32][32];
  __shared__ unsigned int s_last;
  __shared__ int scan_tmp[33];
  cg::cluster_group cluster = cg::this_cluster();
  const dim3 cdim = cluster.dim_blocks();
  const int CL = (int)cdim.x, G = (int)cdim.y;
  const int rank = (int)cluster.block_index().x;       // slice
  const int grp = (int)cluster.block_index().y;        // token group inside the cluster
  const bool whole = (int)gridDim.y == G;              // one cluster holds every group
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int t0 = blockIdx.y * kSmallTokens;
  const int k0 = rank * (32 * VEC * KIT);
  for (int e = threadIdx.x; e < E; e += blockDim.x) hist[e] = 0;
  pdl_wait();
  // CTA 0 needs the bias only after the slices are in; its load is in flight
  // with the first weight loads rather than on the path after them
  if (rank == 0)
    for (int e = threadIdx.x; e < E; e += blockDim.x) bias_sh[e] = bias[e];

  // ---- partial logits of the 8 tokens over this CTA's slice ----
  float xr[KIT][kSmallTokens][VEC];
#pragma unroll
  for (int i = 0; i < KIT; ++i) {
    const int kk = k0 + (i * 32 + lane) * VEC;
#pragma unroll
    for (int tt = 0; tt < kSmallTokens; ++tt) {
      if (t0 + tt < T && kk < d) {
        const uint4 u = __ldg(reinterpret_cast<const uint4*>(x + (size_t)(t0 + tt) * d + kk));
        unpack16(u, xr[i][tt], TIn());
      } else {
#pragma unroll
        for (int c = 0; c < VEC; ++c) xr[i][tt][c] = 0.f;
      }
    }
  }
  // this warp's experts warp, warp + 8, ... in groups of kG; the weight vectors
  // of the next group are loaded while the current group is computed
  constexpr int kWarps = kSmallThreads / 32, kG = 4;
  const int mine = warp < E ? (E - warp + kWarps - 1) / kWarps : 0;
  auto load_group = [&](int g, uint4 (&raw)[kG][KIT]) {
#pragma unroll
    for (int u = 0; u < kG; ++u) {
      const int e = warp + (g + u) * kWarps;
#pragma unroll
      for (int i = 0; i < KIT; ++i) {
        const int kk = k0 + (i * 32 + lane) * VEC;
        raw[u][i] = (g + u < mine && kk < d)
                        ? __ldg(reinterpret_cast<const uint4*>(w + (size_t)e * d + kk))
                        : make_uint4(0u, 0u, 0u, 0u);
      }
    }
  };
  uint4 cur[kG][KIT];
  load_group(0, cur);
  for (int g = 0; g < mine; g += kG) {
    uint4 nxt[kG][KIT];
    load_group(g + kG, nxt);
#pragma unroll
    for (int u = 0; u < kG; ++u) {
      float acc[kSmallTokens];
#pragma unroll
      for (int tt = 0; tt < kSmallTokens; ++tt) acc[tt] = 0.f;
#pragma unroll
      for (int i = 0; i < KIT; ++i) {
        float wf[VEC];
        unpack16(cur[u][i], wf, TIn());
#pragma unroll
        for (int c = 0; c < VEC; ++c)
#pragma unroll
          for (int tt = 0; tt < kSmallTokens; ++tt) acc[tt] = fmaf(wf[c], xr[i][tt][c], acc[tt]);
      }
      const float s = transpose_sum8(acc, lane);
      const int e = warp + (g + u) * kWarps;
      if ((lane & 3) == 0 && g + u < mine)
        part[((lane >> 4) & 1) * 4 + ((lane >> 3) & 1) * 2 + ((lane >> 2) & 1)][e] = s;
    }
#pragma unroll
    for (int u = 0; u < kG; ++u)
#pragma unroll
      for (int i = 0; i < KIT; ++i) cur[u][i] = nxt[u][i];
  }
  cluster.sync();  // phase 1: every CTA's slice is written and visible to the cluster

  if (rank == 0) {
    // ---- the group's leader: add the slices, then route token t0 + warp ----
    const int t = t0 + warp;
    const int base = grp * CL;  // cluster rank of this group's slice 0
    float b[VPL], v[VPL];
#pragma unroll
    for (int j = 0; j < VPL; ++j) {
      const int e = lane + 32 * j;
      b[j] = e < E ? bias_sh[e] : 0.f;
      float s = 0.f;
      if (e < E && t < T) {
        // every slice's load in flight, then the adds in rank order
        float pr[kSmallMaxCluster];
#pragma unroll
        for (int r = 0; r < kSmallMaxCluster; ++r)
          pr[r] = r < CL ? cluster.map_shared_rank(&part[warp][e], base + r)[0] : 0.f;
#pragma unroll
        for (int r = 0; r < kSmallMaxCluster; ++r)
          if (r < CL) s += pr[r];
        if (offset) s += offset[(size_t)t * E + e];
      }
      v[j] = s;
    }
    // phase 2, first half: the slices are read, so the other CTAs of the group may
    // exit; this CTA waits on the phase only after its selection
    cluster_arrive();
    if (t < T) {
      route_token<VPL, false>(v, b, lane, E, N, K, t, topk_idx, topk_gate, n_ffn, hist,
                              cand_key[warp], cand_p[warp]);
#pragma unroll
      for (int j = 0; j < VPL; ++j) {
        const int e = lane + 32 * j;
        if (e < E) {
          if (probs_out) probs_out[(size_t)t * E + e] = v[j];
          part[warp][e] = v[j];
        }
      }
    } else {
#pragma unroll
      for (int j = 0; j < VPL; ++j)
        if (lane + 32 * j < E) part[warp][lane + 32 * j] = 0.f;
    }
    __syncthreads();
    // this group's column sums of R (tokens in order)
    if (prob_sum)
      for (int e = threadIdx.x; e < E; e += blockDim.x) {
        float q = 0.f;
#pragma unroll
        for (int tt = 0; tt < kSmallTokens; ++tt) q += part[tt][e];
        colsum[e] = q;
      }
    cluster_wait();  // phase 2, second half
    if (whole) {
      if (G > 1) {
        cluster.sync();  // phase 3: every leader's histogram and column sums are in
        if (grp == 0)
          for (int e = threadIdx.x; e < E; e += blockDim.x) {
            int cnt = 0;
            float q = 0.f;
            for (int j = 0; j < G; ++j) {
              cnt += cluster.map_shared_rank(&hist[e], j * CL)[0];
              if (prob_sum) q += cluster.map_shared_rank(&colsum[e], j * CL)[0];
            }
            counts[e] = cnt;
            if (prob_sum) prob_sum[e] = q;
          }
        cluster.sync();  // phase 4: group 0 has read the other leaders' arrays
      } else {
        __syncthreads();
        for (int e = threadIdx.x; e < E; e += blockDim.x) {
          counts[e] = hist[e];
          if (prob_sum) prob_sum[e] = colsum[e];
        }
      }
      // every leader's topk_idx is visible here (cluster barrier, or this CTA's own)
      if (offsets && grp == 0)
        small_layout(topk_idx, T, K, N, reinterpret_cast<int*>(&part[0][0]), scan_tmp, offsets,
                     row_token, slot_pos);
      return;
    }
    // one group per cluster: write this group's rows; the group that finishes
    // last adds every group's rows, groups in order
    const int c = blockIdx.y;
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
      part_hist[(size_t)c * E + e] = hist[e];
      if (part_psum) part_psum[(size_t)c * E + e] = colsum[e];
    }
    // the CTA's writes are ordered before the ticket by the barrier and the
    // releasing fence of the thread that takes it
    __syncthreads();
    if (threadIdx.x == 0) {
      __threadfence();
      s_last = atomicInc(ticket, gridDim.y - 1) == gridDim.y - 1;
      if (s_last) __threadfence();
    }
    __syncthreads();
    if (s_last) {
      // one thread per expert, groups added in order; the loads of 8 groups are
      // in flight at once
      const int nparts = gridDim.y;
      for (int e = threadIdx.x; e < E; e += kSmallThreads) {
        int cnt = 0;
        float q = 0.f;
        for (int p0 = 0; p0 < nparts; p0 += 8) {
          int hv[8];
          float qv[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const bool in = p0 + u < nparts;
            hv[u] = in ? __ldcg(part_hist + (size_t)(p0 + u) * E + e) : 0;
            qv[u] = (in && part_psum) ? __ldcg(part_psum + (size_t)(p0 + u) * E + e) : 0.f;
          }
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            cnt += hv[u];
            if (p0 + u < nparts) q += qv[u];
          }
        }
        counts[e] = cnt;
        if (prob_sum) prob_sum[e] = q;
      }
      // every group's topk_idx was released before its ticket
      if (offsets)
        small_layout(topk_idx, T, K, N, reinterpret_cast<int*>(&part[0][0]), scan_tmp, offsets,
                     row_token, slot_pos);
    }
  } else {
    cluster.sync();  // phase 2: the leader has read this CTA's slice
    if (whole && G > 1) {
      cluster.sync();  // phase 3
      cluster.sync();  // phase 4
    }
  }
}

// prob_sum[e] = sum over selection CTAs of their column sums of R (lane-strided
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

}  // namespace moe
