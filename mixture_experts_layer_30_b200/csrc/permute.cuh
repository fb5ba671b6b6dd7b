// Dispatch of routed slots to the N FFN experts (zero-computation experts get
// no rows): LongCat-Flash Technical Report, §2.1 -- an identity expert needs
// neither compute nor a copy of its token.
//
// Row layout: experts 0..N-1 in order, tokens ascending inside an expert.
// Built without global atomics and without inter-CTA waits:
//   1. chunk_hist_kernel  per 256-token chunk c: H[c][e] = #tokens of c routed to e
//   2. scan_kernel        one CTA: offsets = exclusive scan of sum_c H[c][e];
//                         base[c][e] = offsets[e] + sum_{c' < c} H[c'][e]
//   3. rank_kernel        per chunk: row of (t, k) = base[c][e] + #earlier tokens of
//                         the chunk routed to e (warp bitmaps + popcount)
//   4. gather_kernel      one warp per token: x row copied to each of its rows.
// A batch of one chunk (decode) runs 1-4 as one kernel (perm_gather_small_kernel),
// or 1-3 as perm_small_kernel when no copy is asked for.
#pragma once

#include "common.cuh"

namespace moe {

__global__ void __launch_bounds__(256)
chunk_hist_kernel(const int32_t* __restrict__ topk_idx, int T, int K, int N, int E,
                  int32_t* __restrict__ chunk_hist, uint32_t* status) {
  pdl_trigger();
  pdl_wait();
  extern __shared__ int sh_hist[];  // [N]
  for (int e = threadIdx.x; e < N; e += blockDim.x) sh_hist[e] = 0;
  __syncthreads();
  const int t = blockIdx.x * kPermChunk + threadIdx.x;
  if (t < T) {
    for (int k = 0; k < K; ++k) {
      int e = topk_idx[(size_t)t * K + k];
      if (e < 0 || e >= E) { set_status(status, MOE_DEV_BAD_EXPERT_INDEX); continue; }
      if (e < N) atomicAdd(&sh_hist[e], 1);
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < N; e += blockDim.x)
    chunk_hist[(size_t)blockIdx.x * N + e] = sh_hist[e];
}

// One CTA of 1024 threads.
__global__ void __launch_bounds__(1024)
perm_scan_kernel(const int32_t* __restrict__ chunk_hist, int nchunks, int N,
                 const int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
                 int32_t* __restrict__ chunk_base, uint32_t* status) {
  pdl_trigger();
  pdl_wait();
  __shared__ int scan_tmp[33];
  __shared__ int tot_sh[kMaxExperts];
  // per-expert totals (thread per expert, chunks in order)
  for (int e = threadIdx.x; e < N; e += blockDim.x) {
    int s = 0;
    for (int c = 0; c < nchunks; ++c) s += chunk_hist[(size_t)c * N + e];
    tot_sh[e] = s;
    if (counts && counts[e] != s) set_status(status, MOE_DEV_COUNT_MISMATCH);
  }
  __syncthreads();
  // exclusive scan over experts: each thread owns a run of consecutive experts
  const int per = (N + blockDim.x - 1) / blockDim.x;
  const int lo = min(N, (int)threadIdx.x * per), hi = min(N, lo + per);
  int local = 0;
  for (int e = lo; e < hi; ++e) local += tot_sh[e];
  int run = block_exclusive_scan(local, scan_tmp, &scan_tmp[32]);
  for (int e = lo; e < hi; ++e) {
    offsets[e] = run;
    int b = run;
    for (int c = 0; c < nchunks; ++c) {
      chunk_base[(size_t)c * N + e] = b;
      b += chunk_hist[(size_t)c * N + e];
    }
    run += tot_sh[e];
  }
  if (threadIdx.x == 0) offsets[N] = scan_tmp[32];
}

// One CTA per 256-token chunk, one thread per token, 8 warps.
// Shared: bits[8][N] (which lanes of warp w route to e), wbase[8][N].
__global__ void __launch_bounds__(256)
perm_rank_kernel(const int32_t* __restrict__ topk_idx, int T, int K, int N, int E,
                 const int32_t* __restrict__ chunk_base, int32_t* __restrict__ row_token,
                 int32_t* __restrict__ slot_pos) {
  pdl_trigger();
  pdl_wait();
  extern __shared__ uint32_t sh_rank[];
  uint32_t* bits = sh_rank;                                   // [8][N]
  int* wbase = reinterpret_cast<int*>(sh_rank + 8 * N);       // [8][N]
  for (int i = threadIdx.x; i < 8 * N; i += blockDim.x) bits[i] = 0;
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int c = blockIdx.x;
  const int t = c * kPermChunk + threadIdx.x;
  if (t < T) {
    for (int k = 0; k < K; ++k) {
      int e = topk_idx[(size_t)t * K + k];
      if (e >= 0 && e < N) atomicOr(&bits[warp * N + e], 1u << lane);
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < N; e += blockDim.x) {
    int b = chunk_base[(size_t)c * N + e];
#pragma unroll
    for (int w = 0; w < 8; ++w) {
      wbase[w * N + e] = b;
      b += __popc(bits[w * N + e]);
    }
  }
  __syncthreads();
  if (t < T) {
    const uint32_t lt = (1u << lane) - 1u;
    for (int k = 0; k < K; ++k) {
      int e = topk_idx[(size_t)t * K + k];
      int row = -1;
      if (e >= 0 && e < N) {
        row = wbase[warp * N + e] + __popc(bits[warp * N + e] & lt);
        row_token[row] = t;
      }
      slot_pos[(size_t)t * K + k] = row;
    }
  }
}

// The layout of a batch of one chunk (T <= 256, decode): histogram, scan and
// rank of the three kernels above in one CTA, one thread per token.
// Shared: bits[8][N], wbase[8][N], tot[N] (68*N bytes).
__global__ void __launch_bounds__(256)
perm_small_kernel(const int32_t* __restrict__ topk_idx, int T, int K, int N, int E,
                  const int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
                  int32_t* __restrict__ row_token, int32_t* __restrict__ slot_pos,
                  uint32_t* status) {
  pdl_trigger();
  pdl_wait();
  extern __shared__ uint32_t sh_small[];
  __shared__ int scan_tmp[33];
  uint32_t* bits = sh_small;                                  // [8][N]
  int* wbase = reinterpret_cast<int*>(sh_small + 8 * N);      // [8][N]
  int* tot = reinterpret_cast<int*>(sh_small + 16 * N);       // [N]
  for (int i = threadIdx.x; i < 8 * N; i += blockDim.x) bits[i] = 0;
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int t = threadIdx.x;
  if (t < T) {
    for (int k = 0; k < K; ++k) {
      const int e = topk_idx[(size_t)t * K + k];
      if (e < 0 || e >= E) { set_status(status, MOE_DEV_BAD_EXPERT_INDEX); continue; }
      if (e < N) atomicOr(&bits[warp * N + e], 1u << lane);
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < N; e += blockDim.x) {
    int c = 0;
#pragma unroll
    for (int w = 0; w < 8; ++w) c += __popc(bits[w * N + e]);
    tot[e] = c;
    if (counts && counts[e] != c) set_status(status, MOE_DEV_COUNT_MISMATCH);
  }
  __syncthreads();
  // exclusive scan over experts: each thread owns a run of consecutive experts
  const int per = (N + blockDim.x - 1) / blockDim.x;
  const int lo = min(N, (int)threadIdx.x * per), hi = min(N, lo + per);
  int local = 0;
  for (int e = lo; e < hi; ++e) local += tot[e];
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
      const int e = topk_idx[(size_t)t * K + k];
      int row = -1;
      if (e >= 0 && e < N) {
        row = wbase[warp * N + e] + __popc(bits[warp * N + e] & lt);
        row_token[row] = t;
      }
      slot_pos[(size_t)t * K + k] = row;
    }
  }
}

// A batch of one chunk (T <= 256) together with its copy, in one launch: every
// CTA builds the whole layout of the batch in shared memory (T*K slots, a few
// microseconds), CTA 0 writes the layout outputs, and CTA c copies the x rows
// of tokens 8c .. 8c+7 (one warp each) to all of their rows; the first 4 KB of
// each row is loaded before the layout is built.  No CTA waits for another.
// Shared: bits[8][N], wbase[8][N], tot[N], rows[T*K].
template <typename T>
__global__ void __launch_bounds__(256)
perm_gather_small_kernel(const T* __restrict__ x, const int32_t* __restrict__ topk_idx,
                         int ntok, int K, int N, int E, int d,
                         const int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
                         int32_t* __restrict__ row_token, int32_t* __restrict__ slot_pos,
                         T* __restrict__ x_perm, uint32_t* status) {
  pdl_trigger();
  pdl_wait();
  extern __shared__ uint32_t sh_pg[];
  __shared__ int scan_tmp[33];
  uint32_t* bits = sh_pg;                                // [8][N]
  int* wbase = reinterpret_cast<int*>(sh_pg + 8 * N);    // [8][N]
  int* tot = reinterpret_cast<int*>(sh_pg + 16 * N);     // [N]
  int* rows = reinterpret_cast<int*>(sh_pg + 17 * N);    // [T*K]
  const bool writer = blockIdx.x == 0;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  // the first piece of this warp's x row is loaded now, its latency hidden by
  // the layout below
  const int t = blockIdx.x * 8 + warp;  // token this warp copies
  const int nvec = d * (int)sizeof(T) / 16;
  const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)t * d);
  uint4 first[8];
  if (t < ntok) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int v = i * 32 + lane;
      if (v < nvec) first[i] = __ldg(src + v);
    }
  }
  for (int i = threadIdx.x; i < 8 * N; i += blockDim.x) bits[i] = 0;
  __syncthreads();
  const int tt = threadIdx.x;  // token of this thread in the layout
  if (tt < ntok) {
    for (int k = 0; k < K; ++k) {
      const int e = topk_idx[(size_t)tt * K + k];
      if (e < 0 || e >= E) {
        if (writer) set_status(status, MOE_DEV_BAD_EXPERT_INDEX);
        continue;
      }
      if (e < N) atomicOr(&bits[warp * N + e], 1u << lane);
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < N; e += blockDim.x) {
    int c = 0;
#pragma unroll
    for (int w = 0; w < 8; ++w) c += __popc(bits[w * N + e]);
    tot[e] = c;
    if (writer && counts && counts[e] != c) set_status(status, MOE_DEV_COUNT_MISMATCH);
  }
  __syncthreads();
  const int per = (N + blockDim.x - 1) / blockDim.x;
  const int lo = min(N, (int)threadIdx.x * per), hi = min(N, lo + per);
  int local = 0;
  for (int e = lo; e < hi; ++e) local += tot[e];
  int run = block_exclusive_scan(local, scan_tmp, &scan_tmp[32]);
  for (int e = lo; e < hi; ++e) {
    if (writer) offsets[e] = run;
    int b = run;
#pragma unroll
    for (int w = 0; w < 8; ++w) {
      wbase[w * N + e] = b;
      b += __popc(bits[w * N + e]);
    }
    run += tot[e];
  }
  if (writer && threadIdx.x == 0) offsets[N] = scan_tmp[32];
  __syncthreads();
  if (tt < ntok) {
    const uint32_t lt = (1u << lane) - 1u;
    for (int k = 0; k < K; ++k) {
      const int e = topk_idx[(size_t)tt * K + k];
      int row = -1;
      if (e >= 0 && e < N) {
        row = wbase[warp * N + e] + __popc(bits[warp * N + e] & lt);
        if (writer) row_token[row] = tt;
      }
      rows[tt * K + k] = row;
      if (writer) slot_pos[(size_t)tt * K + k] = row;
    }
  }
  __syncthreads();
  // copy: warp w of CTA c takes token 8c + w
  if (t >= ntok) return;
  for (int kb = 0; kb < K; kb += 32) {
    const int my_row = kb + lane < K ? rows[t * K + kb + lane] : -1;
    const uint32_t has_rows = __ballot_sync(0xffffffffu, my_row >= 0);
    for (int v0 = 0; v0 < nvec && has_rows; v0 += 32 * 8) {
      uint4 piece[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int v = v0 + i * 32 + lane;
        if (v < nvec) piece[i] = v0 == 0 ? first[i] : __ldg(src + v);
      }
      uint32_t has = has_rows;
      while (has) {
        const int j = __ffs(has) - 1;
        has &= has - 1;
        const int row = __shfl_sync(0xffffffffu, my_row, j);
        uint4* dst = reinterpret_cast<uint4*>(x_perm + (size_t)row * d);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int v = v0 + i * 32 + lane;
          if (v < nvec) dst[v] = piece[i];
        }
      }
    }
  }
}

// One warp per token: the x row is read once from HBM, in pieces of 8 x 16 B
// per lane held in registers, and each piece is stored to every row of the token.
template <typename T>
__global__ void __launch_bounds__(256)
gather_kernel(const T* __restrict__ x, const int32_t* __restrict__ slot_pos, int ntok, int K,
              int d, T* __restrict__ x_perm) {
  pdl_trigger();
  pdl_wait();
  constexpr int kPiece = 8;
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t >= ntok) return;
  const int nvec = d * (int)sizeof(T) / 16;
  const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)t * d);
  for (int kb = 0; kb < K; kb += 32) {
    // rows of slots kb..kb+31 of this token (lane j holds slot kb+j's row)
    const int my_row = kb + lane < K ? slot_pos[(size_t)t * K + kb + lane] : -1;
    const uint32_t rows = __ballot_sync(0xffffffffu, my_row >= 0);
    if (!rows) continue;
    for (int v0 = 0; v0 < nvec; v0 += 32 * kPiece) {
      uint4 piece[kPiece];
#pragma unroll
      for (int i = 0; i < kPiece; ++i) {
        const int v = v0 + i * 32 + lane;
        if (v < nvec) piece[i] = __ldg(src + v);
      }
      uint32_t has = rows;
      while (has) {
        const int j = __ffs(has) - 1;
        has &= has - 1;
        const int row = __shfl_sync(0xffffffffu, my_row, j);
        uint4* dst = reinterpret_cast<uint4*>(x_perm + (size_t)row * d);
#pragma unroll
        for (int i = 0; i < kPiece; ++i) {
          const int v = v0 + i * 32 + lane;
          if (v < nvec) dst[v] = piece[i];
        }
      }
    }
  }
}

}  // namespace moe
