// Shared device helpers of the MoE layer kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "moe.h"

#define MOE_DEV __device__ __forceinline__

#include <atomic>

namespace moe {

// Process-wide count of kernel launches issued by this library.
inline std::atomic<unsigned long long>& launch_counter() {
  static std::atomic<unsigned long long> n{0};
  return n;
}
inline void note_launch() { launch_counter().fetch_add(1, std::memory_order_relaxed); }

// Process-wide settings of the GEMMs' bounded pipeline waits, read at every
// launch (moe_debug_set_pipeline): the time limit of one wait (0: the default
// of 4 s) and, for tests of the timeout path, a producer that issues nothing.
struct PipelineDebug {
  std::atomic<unsigned long long> wait_ns{0};
  std::atomic<int> stall_fill{0};
};
inline PipelineDebug& pipeline_debug() {
  static PipelineDebug d;
  return d;
}
constexpr unsigned long long kDefaultWaitNs = 4000000000ull;  // 4 s
inline unsigned long long pipeline_wait_ns() {
  const unsigned long long v = pipeline_debug().wait_ns.load(std::memory_order_relaxed);
  return v ? v : kDefaultWaitNs;
}

constexpr int kMaxExperts = 1024;   // E = N + Z upper bound (one warp holds <= 32 per lane)
constexpr int kPermChunk = 256;     // tokens per dispatch chunk (one thread per token)
constexpr int kRouteTokensPerCta = 32;  // 16 warps x 2 tokens: enough warps to hide latency
constexpr int kRouteThreads = 512;

// --- programmatic dependent launch ------------------------------------------
// Every kernel of this library is launched with programmatic stream
// serialisation (launch_pdl).  A kernel first lets the next kernel on the
// stream be scheduled (pdl_trigger: once all of this grid's CTAs have started)
// and then waits for the previous grid to complete and publish its memory
// (pdl_wait) before its first global-memory read or write; only work on
// registers, shared memory, barriers and TMEM may come before the wait.  The
// next kernel's launch and prologue thus overlap this kernel's tail.  Both are
// no-ops for a kernel launched without the attribute.
MOE_DEV void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
MOE_DEV void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t st, Args... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

MOE_DEV void set_status(uint32_t* st, uint32_t bit) {
  if (st) atomicOr(st, bit);
}

// --- element conversion ----------------------------------------------------
template <typename T> struct Cvt;
template <> struct Cvt<float> {
  static MOE_DEV float to_f(float v) { return v; }
  static MOE_DEV float from_f(float v) { return v; }
};
template <> struct Cvt<__nv_bfloat16> {
  static MOE_DEV float to_f(__nv_bfloat16 v) { return __bfloat162float(v); }
  static MOE_DEV __nv_bfloat16 from_f(float v) { return __float2bfloat16_rn(v); }
};

// 16-byte vector of the storage type: 4 fp32 or 8 bf16.
template <typename T> struct Vec16 {
  static constexpr int kN = 16 / sizeof(T);
};

MOE_DEV void unpack16(const uint4& v, float* f, float) {
  f[0] = __uint_as_float(v.x); f[1] = __uint_as_float(v.y);
  f[2] = __uint_as_float(v.z); f[3] = __uint_as_float(v.w);
}
MOE_DEV void unpack16(const uint4& v, float* f, __nv_bfloat16) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}
MOE_DEV uint4 pack16(const float* f, float) {
  return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]),
                    __float_as_uint(f[3]));
}
MOE_DEV uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);  // .x = lo (low half), .y = hi
  return *reinterpret_cast<uint32_t*>(&p);
}
MOE_DEV uint4 pack16(const float* f, __nv_bfloat16) {
  return make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]), pack_bf16x2(f[4], f[5]),
                    pack_bf16x2(f[6], f[7]));
}

// SiLU(a) = a * sigmoid(a) = a / (1 + e^-a); for a -> -inf, e^-a = inf gives -0.
MOE_DEV float silu(float a) { return a / (1.0f + expf(-a)); }

// --- block-wide exclusive scan (int) ----------------------------------------
// `warp_tot` is shared scratch of >= 32 ints.  Every thread of the block calls.
MOE_DEV int block_exclusive_scan(int v, int* warp_tot, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nwarps = (blockDim.x + 31) >> 5;
  int inc = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int n = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += n;
  }
  if (lane == 31) warp_tot[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    int w = lane < nwarps ? warp_tot[lane] : 0;
    int wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int n = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += n;
    }
    if (lane < nwarps) warp_tot[lane] = wi - w;  // exclusive prefix of warp totals
    if (lane == 31 && total) *total = wi;
  }
  __syncthreads();
  int r = warp_tot[warp] + inc - v;
  __syncthreads();
  return r;
}

// --- routed-row chunking shared by the grouped GEMMs ------------------------
// prefix[e] = number of row chunks of `rows_per_chunk` in experts 0..e-1,
// e in [0, N].  Segment sizes come from offsets[]; a non-monotone or
// out-of-range offsets array sets MOE_DEV_BAD_OFFSETS and counts as empty.
// Every thread of the block must call; ends with __syncthreads().
MOE_DEV void build_chunk_prefix(const int32_t* __restrict__ offsets, int N, int max_rows,
                                int rows_per_chunk, int* prefix, int* scan_tmp,
                                uint32_t* status) {
  const int per = (N + blockDim.x - 1) / blockDim.x;
  const int lo = min(N, (int)threadIdx.x * per), hi = min(N, lo + per);
  int local = 0;
  for (int e = lo; e < hi; ++e) {
    int a = offsets[e], b = offsets[e + 1];
    int m = b - a;
    if (m < 0 || a < 0 || b > max_rows) { set_status(status, MOE_DEV_BAD_OFFSETS); m = 0; }
    local += (m + rows_per_chunk - 1) / rows_per_chunk;
  }
  int run = block_exclusive_scan(local, scan_tmp, &scan_tmp[32]);
  for (int e = lo; e < hi; ++e) {
    prefix[e] = run;
    int a = offsets[e], b = offsets[e + 1];
    int m = b - a;
    if (m < 0 || a < 0 || b > max_rows) m = 0;
    run += (m + rows_per_chunk - 1) / rows_per_chunk;
  }
  if (threadIdx.x == 0) prefix[N] = scan_tmp[32];
  __syncthreads();
}

// Largest e in [0, N) with prefix[e] <= c (prefix non-decreasing, prefix[N] > c).
MOE_DEV int find_expert(const int* prefix, int N, int c) {
  int lo = 0, hi = N;  // invariant: prefix[lo] <= c < prefix[hi]
  while (hi - lo > 1) {
    int mid = (lo + hi) >> 1;
    if (prefix[mid] <= c) lo = mid; else hi = mid;
  }
  return lo;
}

// One CTA per 128 x 64 bf16 tile (16 KiB): copies tile (m, rb, cb) of the
// row-major matrices [rows, cols] to position (m*rows/128 + rb)*cols/64 + cb
// of the tiled order, row-major inside the tile.  16-byte vectors.
__global__ void __launch_bounds__(256)
pack_tiles_kernel(const uint4* __restrict__ src, int rows, int cols, uint4* __restrict__ dst) {
  pdl_trigger();
  pdl_wait();
  const long long tile = blockIdx.x;
  const int cb_n = cols / 64, rb_n = rows / 128;
  const int cb = (int)(tile % cb_n);
  const long long mr = tile / cb_n;  // m * rb_n + rb
  const int rb = (int)(mr % rb_n);
  const long long m = mr / rb_n;
  const size_t vec_per_row = (size_t)cols / 8;  // 8 bf16 per 16-byte vector
  const uint4* s = src + ((size_t)m * rows + (size_t)rb * 128) * vec_per_row + (size_t)cb * 8;
  uint4* d = dst + (size_t)tile * 1024;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int v = threadIdx.x + i * 256;  // 0..1023: row v/8, vector v%8 of the tile
    d[v] = s[(size_t)(v >> 3) * vec_per_row + (v & 7)];
  }
}

}  // namespace moe
