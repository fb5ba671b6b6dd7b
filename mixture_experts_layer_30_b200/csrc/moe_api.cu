// C ABI of the MoE layer with zero-computation experts (declared in moe.h):
// argument validation, workspace layout and kernel launches.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <vector>

#include <nvtx3/nvToolsExt.h>

#include "moe.h"
#include "common.cuh"
#include "route.cuh"
#include "permute.cuh"
#include "gemm_simt.cuh"
#include "gemm_tc.cuh"
#include "gemm_fp8.cuh"
#include "quant.cuh"
#include "combine.cuh"
#include "backward.cuh"
#include "gemm_simt_bwd.cuh"
#include "gemm_wgrad.cuh"

namespace {

thread_local char g_err[512] = "";

// NVTX range over one C-ABI call (the enqueue on the host; profilers place the
// call's kernels under it).  Header-only NVTX: a no-op unless a tool is attached.
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

moe_status fail(moe_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return st;
}

moe_status check_launch(const char* what) {
  moe::note_launch();
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(MOE_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
  return MOE_OK;
}

#define MOE_TRY(expr)                 \
  do {                                \
    moe_status _s = (expr);           \
    if (_s != MOE_OK) return _s;      \
  } while (0)

size_t align256(size_t v) { return (v + 255) & ~(size_t)255; }

struct WsLayout {
  size_t status, logits, route_hist, route_psum, perm_hist, perm_base, h, total;
};

int elem_bytes(const moe_shape& s) { return s.dtype == MOE_BF16 ? 2 : 4; }
int perm_chunks(const moe_shape& s) { return (s.T + moe::kPermChunk - 1) / moe::kPermChunk; }

moe_status validate_shape(const moe_shape* sp) {
  if (!sp) return fail(MOE_ERR_INVALID_ARG, "shape is NULL");
  const moe_shape& s = *sp;
  if (s.dtype != MOE_F32 && s.dtype != MOE_BF16)
    return fail(MOE_ERR_INVALID_ARG, "dtype %d is neither MOE_F32 nor MOE_BF16", s.dtype);
  if (s.T < 0 || s.d < 1 || s.N < 1 || s.Z < 0 || s.I < 1)
    return fail(MOE_ERR_INVALID_ARG, "bad shape T=%d d=%d N=%d Z=%d I=%d", s.T, s.d, s.N, s.Z,
                s.I);
  const int E = s.N + s.Z;
  if (E > moe::kMaxExperts)
    return fail(MOE_ERR_UNSUPPORTED, "N+Z=%d exceeds %d experts", E, moe::kMaxExperts);
  if (s.K < 1 || s.K > E) return fail(MOE_ERR_INVALID_ARG, "K=%d outside [1, N+Z=%d]", s.K, E);
  if ((long long)s.T * s.K > 0x7fffffffLL)
    return fail(MOE_ERR_UNSUPPORTED, "T*K=%lld routed rows exceed int32", (long long)s.T * s.K);
  const int vec = 16 / elem_bytes(s);
  if (s.d % vec)
    return fail(MOE_ERR_UNSUPPORTED, "d=%d must be a multiple of %d for 16-byte rows", s.d, vec);
  if (s.weight_layout != MOE_WEIGHTS_ROW_MAJOR && s.weight_layout != MOE_WEIGHTS_TILED)
    return fail(MOE_ERR_INVALID_ARG, "weight_layout %d is not a moe_weight_layout",
                s.weight_layout);
  if (s.weight_layout == MOE_WEIGHTS_TILED &&
      (s.dtype != MOE_BF16 || s.d % 128 || s.I % 128))
    return fail(MOE_ERR_UNSUPPORTED,
                "MOE_WEIGHTS_TILED needs bf16 and d, I multiples of 128 (d=%d, I=%d)", s.d, s.I);
  return MOE_OK;
}

// Router of small batches (route_small_kernel): clusters of CL CTAs split the
// hidden dimension, KIT 16-byte vectors per lane and CTA; VPL experts per lane
// in the selection.  Used for every fp32 shape it fits and for bf16 shapes
// whose router GEMM is at most kSmallRouteMaxFlops (decode batches), where one
// launch of CUDA-core FMAs beats a tensor-core GEMM plus a selection kernel.
constexpr double kSmallRouteMaxFlops = 4e8;
struct SmallRoute {
  bool ok;
  int CL, KIT, VPL;
  int G;  // token groups per cluster: 1, or every group when they fit one cluster
};
SmallRoute small_route_of(const moe_shape& s) {
  SmallRoute r{false, 0, 0, 0, 1};
  const int E = s.N + s.Z;
  const int per_cta = 32 * (16 / elem_bytes(s));  // hidden elements per CTA and KIT
  if ((s.T + moe::kSmallTokens - 1) / moe::kSmallTokens > 65535) return r;
  int kit = 1, cl = (s.d + per_cta - 1) / per_cta;
  if (cl > moe::kSmallMaxCluster) {
    kit = 2;
    cl = (s.d + 2 * per_cta - 1) / (2 * per_cta);
  }
  if (cl > moe::kSmallMaxCluster) return r;
  const bool tc = s.dtype == MOE_BF16 && moe::tc::router_supported(s);
  if (tc && 2.0 * s.T * E * s.d > kSmallRouteMaxFlops) return r;
  int vpl = 1;
  while (32 * vpl < E) vpl *= 2;
  r.ok = true;
  r.CL = cl;
  r.KIT = kit;
  r.VPL = vpl;
  const int groups = (s.T + moe::kSmallTokens - 1) / moe::kSmallTokens;
  if (groups * cl <= moe::kSmallMaxWholeCluster) r.G = groups;
  return r;
}
int small_clusters(const moe_shape& s) {
  return (s.T + moe::kSmallTokens - 1) / moe::kSmallTokens;
}

// Selection grid of the large-batch path (topk_kernel).
int topk_ctas(const moe_shape& s, int sms) {
  long long g = (s.T + moe::kTopkWarps - 1) / moe::kTopkWarps;
  const long long cap = std::min<long long>(moe::kTopkMaxCtas, 4LL * sms);
  return (int)std::max<long long>(1, std::min(g, cap));
}
int topk_ctas_bound(const moe_shape& s) {  // for sizing the workspace
  long long g = (s.T + moe::kTopkWarps - 1) / moe::kTopkWarps;
  return (int)std::max<long long>(1, std::min<long long>(g, moe::kTopkMaxCtas));
}

// K splits of the router GEMM: the tensor-core router splits K for small
// batches; the CUDA-core router does not split.
int router_nsplit(const moe_shape& s) {
  return (s.dtype == MOE_BF16 && moe::tc::router_supported(s)) ? moe::tc::router_splits(s) : 1;
}

WsLayout layout_of(const moe_shape& s) {
  WsLayout L{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off = align256(off + bytes);
    return o;
  };
  const size_t E = (size_t)s.N + s.Z;
  L.status = take(256);
  const bool small = small_route_of(s).ok;
  // fp32 logits, one [T, E] slab per K split of the tensor-core router GEMM
  L.logits = take(small ? 0 : (size_t)router_nsplit(s) * s.T * E * 4);
  // small batches: histogram and column sums of R per cluster; large batches:
  // column sums of R per selection CTA
  L.route_hist = take(small ? (size_t)small_clusters(s) * E * 4 : 0);
  L.route_psum = take((size_t)(small ? small_clusters(s) : topk_ctas_bound(s)) * E * 4);
  L.perm_hist = take((size_t)perm_chunks(s) * s.N * 4);
  L.perm_base = take((size_t)perm_chunks(s) * s.N * 4);
  L.h = take((size_t)s.T * s.K * s.I * elem_bytes(s));
  L.total = off;
  return L;
}

moe_status check_ws(const moe_shape& s, void* ws, size_t ws_bytes, WsLayout* L) {
  *L = layout_of(s);
  if (!ws) return fail(MOE_ERR_INVALID_ARG, "workspace is NULL");
  if (reinterpret_cast<uintptr_t>(ws) % 256)
    return fail(MOE_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  if (ws_bytes < L->total)
    return fail(MOE_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", ws_bytes, L->total);
  return MOE_OK;
}

moe_status need(const void* p, const char* name, size_t align = 1) {
  if (!p) return fail(MOE_ERR_INVALID_ARG, "%s is NULL", name);
  if (reinterpret_cast<uintptr_t>(p) % align)
    return fail(MOE_ERR_INVALID_ARG, "%s must be %zu-byte aligned", name, align);
  return MOE_OK;
}

template <typename T> T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<char*>(ws) + off);
}

int sm_count() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

// --- launches ---------------------------------------------------------------

cudaLaunchConfig_t cluster_config(dim3 grid, dim3 block, dim3 cluster, cudaStream_t st,
                                  cudaLaunchAttribute (&attr)[2]) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = cluster.x;
  attr[1].val.clusterDim.y = cluster.y;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cfg;
}

template <typename... KArgs, typename... Args>
cudaError_t launch_cluster_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, dim3 cluster,
                               cudaStream_t st, Args... args) {
  cudaLaunchAttribute attr[2];
  cudaLaunchConfig_t cfg = cluster_config(grid, block, cluster, st, attr);
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// Whether clusters of `size` CTAs of this kernel can be resident: sizes above
// the portable 8 need the kernel's opt-in and a device that schedules them.
// Asked once per kernel and size (no stream work, so it is safe during capture).
struct ClusterFit {
  const void* fn;
  unsigned size;
  bool ok;
};
std::mutex g_cluster_mu;
std::vector<ClusterFit> g_cluster_fit;

template <typename... KArgs>
bool cluster_size_ok(void (*kernel)(KArgs...), dim3 cluster) {
  const unsigned size = cluster.x * cluster.y;
  if (size <= 8) return true;
  if (size > (unsigned)moe::kSmallMaxWholeCluster) return false;
  const void* fn = reinterpret_cast<const void*>(kernel);
  std::lock_guard<std::mutex> lock(g_cluster_mu);
  for (const ClusterFit& f : g_cluster_fit)
    if (f.fn == fn && f.size == size) return f.ok;
  bool ok = cudaFuncSetAttribute(kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) ==
            cudaSuccess;
  if (ok) {
    int n = 0;
    cudaLaunchAttribute attr[2];
    cudaLaunchConfig_t cfg =
        cluster_config(dim3(cluster.x, cluster.y), dim3(moe::kSmallThreads), cluster, 0, attr);
    ok = cudaOccupancyMaxActiveClusters(&n, kernel, &cfg) == cudaSuccess && n > 0;
  }
  if (!ok) cudaGetLastError();  // a refused query leaves no error behind for the launch check
  g_cluster_fit.push_back({fn, size, ok});
  return ok;
}

// The dispatch layout that the small-batch route can build in its last CTA.
struct Layout {
  int32_t* offsets;  // NULL: no layout
  int32_t* row_token;
  int32_t* slot_pos;
};

template <typename T, int KIT, int VPL>
void launch_small(const moe_shape& s, const SmallRoute& r, cudaStream_t st, const void* x,
                  const void* w, const float* off, const float* bias, int32_t* idx, float* gate,
                  uint8_t* nffn, float* probs, int32_t* hist, float* psum, unsigned int* ticket,
                  int32_t* counts, float* prob_sum, const Layout& lay) {
  const int E = s.N + s.Z;
  auto* kernel = moe::route_small_kernel<T, KIT, VPL>;
  dim3 cluster((unsigned)r.CL, (unsigned)r.G);
  // one cluster per token group when every group does not fit one resident cluster
  if (!cluster_size_ok(kernel, cluster)) cluster.y = 1;
  launch_cluster_pdl(kernel, dim3((unsigned)r.CL, (unsigned)small_clusters(s)),
                     dim3(moe::kSmallThreads), cluster, st, static_cast<const T*>(x),
                     static_cast<const T*>(w), off, bias, s.T, s.d, E, s.N, s.K, idx, gate, nffn,
                     probs, hist, psum, ticket, counts, prob_sum, lay.offsets, lay.row_token,
                     lay.slot_pos);
}

template <typename T, int KIT>
void launch_small_vpl(const moe_shape& s, const SmallRoute& r, cudaStream_t st, const void* x,
                      const void* w, const float* off, const float* bias, int32_t* idx,
                      float* gate, uint8_t* nffn, float* probs, int32_t* hist, float* psum,
                      unsigned int* ticket, int32_t* counts, float* prob_sum, const Layout& lay) {
#define MOE_SMALL(V) launch_small<T, KIT, V>(s, r, st, x, w, off, bias, idx, gate, nffn, \
                                             probs, hist, psum, ticket, counts, prob_sum, lay)
  switch (r.VPL) {
    case 1: MOE_SMALL(1); break;
    case 2: MOE_SMALL(2); break;
    case 4: MOE_SMALL(4); break;
    case 8: MOE_SMALL(8); break;
    case 16: MOE_SMALL(16); break;
    default: MOE_SMALL(32); break;
  }
#undef MOE_SMALL
}

template <int VPL, bool kVec4>
void launch_topk(int grid, cudaStream_t st, const float* logits, int nsplit, const float* bias,
                 int T, int E, int N, int K, int32_t* idx, float* gate, uint8_t* nffn,
                 float* probs, int32_t* counts, float* psum) {
  if (psum)
    moe::launch_pdl(moe::topk_kernel<VPL, kVec4, true>, dim3(grid), dim3(moe::kTopkWarps * 32),
                    0, st, logits, nsplit, (long long)T * E, bias, T, E, N, K, idx, gate, nffn,
                    probs, counts, psum);
  else
    moe::launch_pdl(moe::topk_kernel<VPL, kVec4, false>, dim3(grid), dim3(moe::kTopkWarps * 32),
                    0, st, logits, nsplit, (long long)T * E, bias, T, E, N, K, idx, gate, nffn,
                    probs, counts, psum);
}

// Whether the small-batch route can also build the dispatch layout (one CTA,
// one thread per token, the layout tables in its shared memory).
bool route_builds_layout(const moe_shape& s) {
  return s.T > 0 && s.T <= moe::kSmallThreads && s.N <= moe::kSmallLayoutMaxN &&
         small_route_of(s).ok;
}

// lay.offsets != NULL only when route_builds_layout(s).
template <typename T>
moe_status route_impl(const moe_shape& s, const void* x, const void* w, const float* bias,
                      const float* off, int32_t* idx, float* gate, int32_t* counts,
                      uint8_t* nffn, float* probs, float* prob_sum, void* ws, const WsLayout& L,
                      cudaStream_t st, const Layout& lay = Layout{nullptr, nullptr, nullptr}) {
  const int E = s.N + s.Z;
  if (s.T == 0) {
    cudaError_t e = cudaMemsetAsync(counts, 0, (size_t)E * 4, st);
    if (e == cudaSuccess && prob_sum) e = cudaMemsetAsync(prob_sum, 0, (size_t)E * 4, st);
    if (e != cudaSuccess) return fail(MOE_ERR_CUDA, "memset: %s", cudaGetErrorString(e));
    return MOE_OK;
  }
  const SmallRoute sr = small_route_of(s);
  if (sr.ok) {
    // router, selection and counts in one launch
    int32_t* hist = at<int32_t>(ws, L.route_hist);
    float* psum = prob_sum ? at<float>(ws, L.route_psum) : nullptr;
    unsigned int* ticket = at<unsigned int>(ws, L.status + 4);
    if (sr.KIT == 1)
      launch_small_vpl<T, 1>(s, sr, st, x, w, off, bias, idx, gate, nffn, probs, hist, psum,
                             ticket, counts, prob_sum, lay);
    else
      launch_small_vpl<T, 2>(s, sr, st, x, w, off, bias, idx, gate, nffn, probs, hist, psum,
                             ticket, counts, prob_sum, lay);
    return check_launch("router + selection (small batch)");
  }
  float* logits = at<float>(ws, L.logits);
  float* psum = prob_sum ? at<float>(ws, L.route_psum) : nullptr;
  int nsplit = 1;
  if (s.dtype == MOE_BF16 && moe::tc::router_supported(s) &&
      reinterpret_cast<uintptr_t>(off) % 16 == 0) {
    nsplit = moe::tc::router_splits(s);
    MOE_TRY(moe::tc::launch_router_gemm(s, x, w, off, logits, counts, sm_count(), st, g_err,
                                        sizeof(g_err)));
  } else {
    dim3 g((E + moe::kRgBN - 1) / moe::kRgBN, (s.T + moe::kRgBM - 1) / moe::kRgBM);
    moe::launch_pdl(moe::router_gemm_simt_kernel<T>, dim3(g), dim3(256), 0, st,
        static_cast<const T*>(x), static_cast<const T*>(w), off, logits, s.T, E, s.d, counts, E);
    MOE_TRY(check_launch("router gemm"));
  }
  const int grid = topk_ctas(s, sm_count());
  if (E % 4 == 0) {
    const int q = (E + 127) / 128;  // float4 columns per lane
#define MOE_TOPK(V) launch_topk<V, true>(grid, st, logits, nsplit, bias, s.T, E, s.N, s.K, idx, \
                                         gate, nffn, probs, counts, psum)
    if (q <= 1) MOE_TOPK(4);
    else if (q <= 2) MOE_TOPK(8);
    else if (q <= 3) MOE_TOPK(12);
    else if (q <= 4) MOE_TOPK(16);
    else if (q <= 6) MOE_TOPK(24);
    else MOE_TOPK(32);
#undef MOE_TOPK
  } else {
    const int vpl = (E + 31) / 32;
#define MOE_TOPK(V) launch_topk<V, false>(grid, st, logits, nsplit, bias, s.T, E, s.N, s.K, idx, \
                                          gate, nffn, probs, counts, psum)
    if (vpl <= 1) MOE_TOPK(1);
    else if (vpl <= 2) MOE_TOPK(2);
    else if (vpl <= 4) MOE_TOPK(4);
    else if (vpl <= 8) MOE_TOPK(8);
    else if (vpl <= 16) MOE_TOPK(16);
    else MOE_TOPK(32);
#undef MOE_TOPK
  }
  MOE_TRY(check_launch("softmax/top-K"));
  if (prob_sum) {
    moe::launch_pdl(moe::reduce_psum_kernel, dim3((E + 7) / 8), dim3(256), 0, st, psum, grid, E,
                    prob_sum);
    MOE_TRY(check_launch("probability column sums"));
  }
  return MOE_OK;
}

bool g_rank_attr_set[64] = {};

template <typename T>
moe_status permute_impl(const moe_shape& s, const void* x, const int32_t* idx,
                        const int32_t* counts, int32_t* offsets, int32_t* row_token,
                        int32_t* slot_pos, void* x_perm, void* ws, const WsLayout& L,
                        cudaStream_t st) {
  const int E = s.N + s.Z, nch = perm_chunks(s);
  uint32_t* status = at<uint32_t>(ws, L.status);
  int32_t* chist = at<int32_t>(ws, L.perm_hist);
  int32_t* cbase = at<int32_t>(ws, L.perm_base);
  const size_t small_smem = (size_t)17 * s.N * sizeof(uint32_t);
  const size_t fused_smem = small_smem + (size_t)s.T * s.K * sizeof(int32_t);
  if (nch == 1 && x_perm && fused_smem <= 48 * 1024) {
    // one chunk with its copy: layout and gather in one launch
    moe::launch_pdl(moe::perm_gather_small_kernel<T>, dim3((s.T + 7) / 8), dim3(256), fused_smem,
                    st, static_cast<const T*>(x), idx, s.T, s.K, s.N, E, s.d, counts, offsets,
                    row_token, slot_pos, static_cast<T*>(x_perm), status);
    return check_launch("dispatch layout + gather (small batch)");
  }
  if (nch == 1 && small_smem <= 48 * 1024) {
    // one chunk (decode): histogram, scan and rank in one CTA
    moe::launch_pdl(moe::perm_small_kernel, dim3(1), dim3(256), small_smem, st, idx, s.T, s.K, s.N, E, counts, offsets,
                                                         row_token, slot_pos, status);
    MOE_TRY(check_launch("dispatch layout"));
    if (x_perm) {
      moe::launch_pdl(moe::gather_kernel<T>, dim3((s.T + 7) / 8), dim3(256), 0, st,
          static_cast<const T*>(x), slot_pos, s.T, s.K, s.d, static_cast<T*>(x_perm));
      MOE_TRY(check_launch("dispatch gather"));
    }
    return MOE_OK;
  }
  if (nch > 0) {
    moe::launch_pdl(moe::chunk_hist_kernel, dim3(nch), dim3(256), s.N * sizeof(int), st, idx, s.T, s.K, s.N, E, chist,
                                                                 status);
    MOE_TRY(check_launch("dispatch histogram"));
  }
  moe::launch_pdl(moe::perm_scan_kernel, dim3(1), dim3(1024), 0, st, chist, nch, s.N, counts, offsets, cbase, status);
  MOE_TRY(check_launch("dispatch scan"));
  if (nch > 0) {
    const size_t smem = (size_t)16 * s.N * sizeof(uint32_t);
    int dev = 0;
    cudaGetDevice(&dev);
    if (smem > 48 * 1024 && dev < 64 && !g_rank_attr_set[dev]) {
      cudaFuncSetAttribute(moe::perm_rank_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem);
      g_rank_attr_set[dev] = true;
    }
    moe::launch_pdl(moe::perm_rank_kernel, dim3(nch), dim3(256), smem, st, idx, s.T, s.K, s.N, E, cbase, row_token,
                                                   slot_pos);
    MOE_TRY(check_launch("dispatch rank"));
    if (x_perm) {
      moe::launch_pdl(moe::gather_kernel<T>, dim3((s.T + 7) / 8), dim3(256), 0, st,
          static_cast<const T*>(x), slot_pos, s.T, s.K, s.d, static_cast<T*>(x_perm));
      MOE_TRY(check_launch("dispatch gather"));
    }
  }
  return MOE_OK;
}

template <typename T, bool kGated>
moe_status grouped_simt(const moe_shape& s, const void* A, const void* B0, const void* B1,
                        const int32_t* offsets, int n_out, int k_dim, void* C,
                        uint32_t* status, cudaStream_t st, const int32_t* a_rows = nullptr) {
  const long long max_rows = (long long)s.T * s.K;
  const long long ncol = (n_out + moe::kSgBN - 1) / moe::kSgBN;
  const long long max_chunks = s.N + (max_rows + moe::kSgBM - 1) / moe::kSgBM;
  long long grid = max_chunks * ncol;
  const long long cap = (long long)sm_count() * 8;
  if (grid > cap) grid = cap;
  if (grid < 1) grid = 1;
  moe::launch_pdl(moe::grouped_gemm_simt_kernel<T, kGated>, dim3((int)grid), dim3(256), 0, st,
      static_cast<const T*>(A), static_cast<const T*>(B0), static_cast<const T*>(B1), offsets,
      s.N, (int)max_rows, n_out, k_dim, static_cast<T*>(C), status, a_rows, s.T);
  return check_launch(kGated ? "gate/up grouped gemm" : "down grouped gemm");
}

moe_status gate_up_impl(const moe_shape& s, const void* x_perm, const void* w1, const void* w3,
                        const int32_t* offsets, void* h, uint32_t* status, cudaStream_t st) {
  if (s.T == 0) return MOE_OK;
  if (s.dtype == MOE_BF16) {
    if (moe::tc::ffn_supported(s))
      return moe::tc::launch_gate_up(s, x_perm, w1, w3, offsets, h, status, sm_count(), st,
                                     g_err, sizeof(g_err));
    return grouped_simt<__nv_bfloat16, true>(s, x_perm, w1, w3, offsets, s.I, s.d, h, status, st);
  }
  return grouped_simt<float, true>(s, x_perm, w1, w3, offsets, s.I, s.d, h, status, st);
}

moe_status gate_up_gather_impl(const moe_shape& s, const void* x, const int32_t* row_token,
                               const void* w1, const void* w3, const int32_t* offsets, void* h,
                               uint32_t* status, cudaStream_t st) {
  if (s.T == 0) return MOE_OK;
  if (s.dtype == MOE_BF16) {
    if (moe::tc::ffn_supported(s))
      return moe::tc::launch_gate_up_gather(s, x, row_token, w1, w3, offsets, h, status,
                                            sm_count(), st, g_err, sizeof(g_err));
    return grouped_simt<__nv_bfloat16, true>(s, x, w1, w3, offsets, s.I, s.d, h, status, st,
                                             row_token);
  }
  return grouped_simt<float, true>(s, x, w1, w3, offsets, s.I, s.d, h, status, st, row_token);
}

// --- backward ---------------------------------------------------------------

struct BwdLayout {
  size_t status, dlogits, dau, total;
};

BwdLayout bwd_layout_of(const moe_shape& s) {
  BwdLayout L{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off = align256(off + bytes);
    return o;
  };
  L.status = take(256);
  L.dlogits = take((size_t)s.T * (s.N + s.Z) * elem_bytes(s));
  L.dau = take((size_t)s.T * s.K * 2 * s.I * elem_bytes(s));
  L.total = off;
  return L;
}

moe_status check_bwd_ws(const moe_shape& s, void* ws, size_t ws_bytes, BwdLayout* L) {
  *L = bwd_layout_of(s);
  if (!ws) return fail(MOE_ERR_INVALID_ARG, "backward workspace is NULL");
  if (reinterpret_cast<uintptr_t>(ws) % 256)
    return fail(MOE_ERR_INVALID_ARG, "backward workspace must be 256-byte aligned");
  if (ws_bytes < L->total)
    return fail(MOE_ERR_WORKSPACE, "backward workspace has %zu bytes, needs %zu", ws_bytes,
                L->total);
  return MOE_OK;
}

// The backward pass runs on the tensor cores for bf16 (d, I multiples of 128,
// E multiple of 8) and on CUDA cores for fp32.
moe_status check_bwd_shape(const moe_shape& s) {
  if (s.dtype == MOE_BF16 &&
      !(moe::tc::bwd_supported(s) && moe::tc::router_supported(s)))
    return fail(MOE_ERR_UNSUPPORTED,
                "bf16 backward needs d %% 128 == 0, I %% 128 == 0 and (N+Z) %% 8 == 0 "
                "(d=%d, I=%d, N+Z=%d)",
                s.d, s.I, s.N + s.Z);
  return MOE_OK;
}

template <bool kKSeg, bool kSwiglu>
moe_status simt_bwd(const moe::SimtBwdArgs& a, long long tiles, cudaStream_t st,
                    const char* what) {
  long long grid = tiles;
  const long long cap = (long long)sm_count() * 8;
  if (grid > cap) grid = cap;
  if (grid < 1) grid = 1;
  moe::launch_pdl(moe::gemm_simt_bwd_kernel<float, kKSeg, kSwiglu>, dim3((int)grid), dim3(256), 0, st, a);
  return check_launch(what);
}

long long simt_row_tiles(const moe_shape& s, int n_out) {
  const long long rows = (long long)s.T * s.K;
  return (s.N + (rows + moe::kSbBM - 1) / moe::kSbBM) * ((n_out + moe::kSbBN - 1) / moe::kSbBN);
}
long long simt_kseg_tiles(int nseg, int m, int n) {
  return (long long)nseg * ((m + moe::kSbBM - 1) / moe::kSbBM) * ((n + moe::kSbBN - 1) / moe::kSbBN);
}

moe_status down_impl(const moe_shape& s, const void* h, const void* w2, const int32_t* offsets,
                     void* y_perm, uint32_t* status, cudaStream_t st) {
  if (s.T == 0) return MOE_OK;
  if (s.dtype == MOE_BF16) {
    if (moe::tc::ffn_supported(s))
      return moe::tc::launch_down(s, h, w2, offsets, y_perm, status, sm_count(), st, g_err,
                                  sizeof(g_err));
    return grouped_simt<__nv_bfloat16, false>(s, h, w2, nullptr, offsets, s.d, s.I, y_perm,
                                              status, st);
  }
  return grouped_simt<float, false>(s, h, w2, nullptr, offsets, s.d, s.I, y_perm, status, st);
}

}  // namespace

// ---------------------------------------------------------------------------
// Dispatch without a caller-provided workspace (moe_permute_noalloc).
//
// Some callers cannot give this library any device memory beyond the tensors
// of the call itself: operator plug-ins of frameworks whose interface passes
// only input and output buffers, and runtimes that plan every device
// allocation at start-up and refuse allocations afterwards.  For them the
// dispatch step keeps its scratch (two [chunks x N] int32 tables and a status
// word) in one fixed array in device memory that the library owns.
// ---------------------------------------------------------------------------
namespace {

constexpr size_t kNoAllocScratchBytes = 4u << 20;  // 4 MiB, held on every device until exit
__device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_noalloc_mu;
void* g_noalloc_dev_ptr[64] = {};  // device address of the array, per device

// Device address of the scratch array on the current device.  In host code
// the array's name is only a host-side stand-in, so the address is looked up
// once per device and cached.
moe_status noalloc_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(MOE_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= 64) return fail(MOE_ERR_UNSUPPORTED, "device ordinal %d >= 64", dev);
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_dev_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || !p)
      return fail(MOE_ERR_CUDA, "cudaGetSymbolAddress of the dispatch scratch: %s",
                  cudaGetErrorString(e));
    g_noalloc_dev_ptr[dev] = p;
  }
  *out = g_noalloc_dev_ptr[dev];
  return MOE_OK;
}

}  // namespace

template <typename T>
moe_status route_dispatch_impl(const moe_shape& s, const void* x, const void* w,
                               const float* bias, const float* off, int32_t* idx, float* gate,
                               int32_t* counts, uint8_t* nffn, float* probs, float* prob_sum,
                               int32_t* offsets, int32_t* row_token, int32_t* slot_pos, void* ws,
                               const WsLayout& L, cudaStream_t st) {
  if (route_builds_layout(s))
    return route_impl<T>(s, x, w, bias, off, idx, gate, counts, nffn, probs, prob_sum, ws, L, st,
                         Layout{offsets, row_token, slot_pos});
  MOE_TRY(route_impl<T>(s, x, w, bias, off, idx, gate, counts, nffn, probs, prob_sum, ws, L, st));
  return permute_impl<T>(s, x, idx, counts, offsets, row_token, slot_pos, nullptr, ws, L, st);
}

extern "C" {

size_t moe_workspace_bytes(const moe_shape* shape) {
  if (validate_shape(shape) != MOE_OK) return 0;
  return layout_of(*shape).total;
}

moe_status moe_pack_weights(int32_t n_mats, int32_t rows, int32_t cols, int32_t dtype,
                            const void* src, void* dst, void* stream) {
  g_err[0] = 0;
  NvtxRange nvtx_range_("moe_pack_weights");
  if (dtype != MOE_BF16) return fail(MOE_ERR_UNSUPPORTED, "moe_pack_weights packs bf16 only");
  if (n_mats < 0 || rows < 0 || cols < 0 || rows % 128 || cols % 64)
    return fail(MOE_ERR_INVALID_ARG,
                "moe_pack_weights: rows=%d must be a multiple of 128, cols=%d of 64", rows, cols);
  const long long tiles = (long long)n_mats * (rows / 128) * (cols / 64);
  if (tiles == 0) return MOE_OK;
  MOE_TRY(need(src, "src", 16));
  MOE_TRY(need(dst, "dst", 16));
  const size_t bytes = (size_t)tiles * 128 * 64 * 2;
  const char* a = static_cast<const char*>(src);
  const char* b = static_cast<const char*>(dst);
  if (a < b + bytes && b < a + bytes)
    return fail(MOE_ERR_INVALID_ARG, "moe_pack_weights: src and dst overlap");
  if (tiles > 0x7fffffffLL) return fail(MOE_ERR_UNSUPPORTED, "moe_pack_weights: too many tiles");
  moe::launch_pdl(moe::pack_tiles_kernel, dim3((unsigned)tiles), dim3(256), 0, static_cast<cudaStream_t>(stream),
      static_cast<const uint4*>(src), rows, cols, static_cast<uint4*>(dst));
  return check_launch("weight pack");
}

moe_status moe_quantize_weights_mxfp8(int32_t n_mats, int32_t rows, int32_t cols,
                                      const void* src, void* dst_q, void* dst_sf, void* stream) {
  g_err[0] = 0;
  NvtxRange nvtx_range_("moe_quantize_weights_mxfp8");
  if (n_mats < 0 || rows < 0 || cols < 0 || rows % 128 || cols % 128)
    return fail(MOE_ERR_INVALID_ARG,
                "moe_quantize_weights_mxfp8: rows=%d and cols=%d must be multiples of 128", rows,
                cols);
  const long long tiles = (long long)n_mats * (rows / 128) * (cols / 128);
  if (tiles == 0) return MOE_OK;
  if (tiles > 0x7fffffffLL) return fail(MOE_ERR_UNSUPPORTED, "too many weight tiles");
  MOE_TRY(need(src, "src", 16));
  MOE_TRY(need(dst_q, "dst_q", 16));
  MOE_TRY(need(dst_sf, "dst_sf", 16));
  moe::launch_pdl(moe::quantize_weights_mxfp8_kernel, dim3((unsigned)tiles), dim3(256), 0, static_cast<cudaStream_t>(stream),
      static_cast<const __nv_bfloat16*>(src), rows, cols, static_cast<uint8_t*>(dst_q),
      static_cast<uint8_t*>(dst_sf));
  return check_launch("mxfp8 weight quantisation");
}

moe_status moe_workspace_init(void* ws, size_t ws_bytes, void* stream) {
  g_err[0] = 0;
  NvtxRange nvtx_range_("moe_workspace_init");
  if (!ws || ws_bytes < 256) return fail(MOE_ERR_INVALID_ARG, "workspace NULL or < 256 bytes");
  cudaError_t e = cudaMemsetAsync(ws, 0, 256, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(MOE_ERR_CUDA, "memset: %s", cudaGetErrorString(e));
  return MOE_OK;
}

moe_status moe_route(const moe_shape* shape, const void* x, const void* w_router,
                     const float* bias, const float* logit_offset, int32_t* topk_idx,
                     float* topk_gate, int32_t* counts, uint8_t* n_ffn, float* probs_out,
                     float* prob_sum, void* ws, size_t ws_bytes, void* stream) {
  g_err[0] = 0;
  NvtxRange nvtx_range_("moe_route");
  MOE_TRY(validate_shape(shape));
  const moe_shape& s = *shape;
  WsLayout L;
  MOE_TRY(check_ws(s, ws, ws_bytes, &L));
  MOE_TRY(need(counts, "counts", 4));
  MOE_TRY(need(bias, "bias", 4));
  MOE_TRY(need(w_router, "w_router", 16));
  if (s.T > 0) {
    MOE_TRY(need(x, "x", 16));
    MOE_TRY(need(topk_idx, "topk_idx", 4));
    MOE_TRY(need(topk_gate, "topk_gate", 4));
    MOE_TRY(need(n_ffn, "n_ffn"));
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (s.dtype == MOE_BF16)
    return route_impl<__nv_bfloat16>(s, x, w_router, bias, logit_offset, topk_idx, topk_gate,
                                     counts, n_ffn, probs_out, prob_sum, ws, L, st);
  return route_impl<float>(s, x, w_router, bias, logit_offset, topk_idx, topk_gate, counts,
                           n_ffn, probs_out, prob_sum, ws, L, st);
}

moe_status moe_permute(const moe_shape* shape, const void* x, const int32_t* topk_idx,
                       const int32_t* counts, int32_t* offsets, int32_t* row_token,
                       int32_t* slot_pos, void* x_perm, void* ws, size_t ws_bytes,
                       void* stream) {
  g_err[0] = 0;
  NvtxRange nvtx_range_("moe_permute");
  MOE_TRY(validate_shape(shape));
  const moe_shape& s = *shape;
  WsLayout L;
  MOE_TRY(check_ws(s, ws, ws_bytes, &L));
  MOE_TRY(need(offsets, "offsets", 4));
  if (s.T > 0) {
    MOE_TRY(need(topk_idx, "topk_idx", 4));
    MOE_TRY(need(row_token, "row_token", 4));
    MOE_TRY(need(slot_pos, "slot_pos", 4));
    if (x_perm) {
      MOE_TRY(need(x, "x", 16));
      MOE_TRY(need(x_perm, "x_perm", 16));
    }
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (s.dtype == MOE_BF16)
    return permute_impl<__nv_bfloat16>(s, x, topk_idx, counts, offsets, row_token, slot_pos,
                                       x_perm, ws, L, st);
  return permute_impl<float>(s, x, topk_idx, counts, offsets, row_token, slot_pos, x_perm, ws,
                             L, st);
}

moe_status moe_route_dispatch(const moe_shape* shape, const void* x, const void* w_router,
                              const float* bias, const float* logit_offset, int32_t* topk_idx,
                              float* topk_gate, int32_t* counts, uint8_t* n_ffn,
                              float* probs_out, float* prob_sum, int32_t* offsets,
                              int32_t* row_token, int32_t* slot_pos, void* ws, size_t ws_bytes,
                              void* stream) {
  g_err[0] = 0;
  NvtxRange nvtx_range_("moe_route_dispatch");
  MOE_TRY(validate_shape(shape));
  const moe_shape& s = *shape;
  WsLayout L;
  MOE_TRY(check_ws(s, ws, ws_bytes, &L));
  MOE_TRY(need(counts, "counts", 4));
  MOE_TRY(need(bias, "bias", 4));
  MOE_TRY(need(w_router, "w_router", 16));
  MOE_TRY(need(offsets, "offsets", 4));
  if (s.T > 0) {
    MOE_TRY(need(x, "x", 16));
    MOE_TRY(need(topk_idx, "topk_idx", 4));
    MOE_TRY(need(topk_gate, "topk_gate", 4));
    MOE_TRY(need(n_ffn, "n_ffn"));
    MOE_TRY(need(row_token, "row_token", 4));
    MOE_TRY(need(slot_pos, "slot_pos", 4));
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (s.dtype == MOE_BF16)
    return route_dispatch_impl<__nv_bfloat16>(s, x, w_router, bias, logit_offset, topk_idx,
                                              topk_gate, counts, n_ffn, probs_out, prob_sum,
                                              offsets, row_token, slot_pos, ws, L, st);
  return route_dispatch_impl<float>(s, x, w_router, bias, logit_offset, topk_idx, topk_gate,
                                    counts, n_ffn, probs_out, prob_sum, offsets, row_token,
                                    slot_pos, ws, L, st);
}

moe_status moe_permute_noalloc(const moe_shape* shape, const void* x, const int32_t* topk_idx,
                               const int32_t* counts, int32_t* offsets, int32_t* row_token,
                               int32_t* slot_pos, void* x_perm, void* stream) {
  g_err[0] = 0;
  NvtxRange nvtx_range_("moe_permute_noalloc");
  MOE_TRY(validate_shape(shape));
  const moe_shape& s = *shape;
  MOE_TRY(need(offsets, "offsets", 4));
  if (s.T > 0) {
    MOE_TRY(need(x, "x", 16));
    MOE_TRY(need(topk_idx, "topk_idx", 4));
    MOE_TRY(need(row_token, "row_token", 4));
    MOE_TRY(need(slot_pos, "slot_pos", 4));
    MOE_TRY(need(x_perm, "x_perm", 16));
  }
  const size_t table = align256((size_t)perm_chunks(s) * s.N * sizeof(int32_t));
  const size_t bytes = 256 + 2 * table;
  if (bytes > kNoAllocScratchBytes)
    return fail(MOE_ERR_UNSUPPORTED,
                "moe_permute_noalloc: T=%d, N=%d needs %zu bytes of dispatch scratch but the "
                "built-in array holds %zu (256 + 2*round_up(ceil(T/256)*N*4, 256) must fit); "
                "use moe_permute with a workspace",
                s.T, s.N, bytes, kNoAllocScratchBytes);
  void* scratch = nullptr;
  MOE_TRY(noalloc_scratch(&scratch));
  WsLayout L{};
  L.status = 0;
  L.perm_hist = 256;
  L.perm_base = 256 + table;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (s.dtype == MOE_BF16)
    return permute_impl<__nv_bfloat16>(s, x, topk_idx, counts, offsets, row_token, slot_pos,
                                       x_perm, scratch, L, st);
  return permute_impl<float>(s, x, topk_idx, counts, offsets, row_token, slot_pos, x_perm,
                             scratch, L, st);
}

static moe_status check_mxfp8_shape(const moe_shape* shape) {
  MOE_TRY(validate_shape(shape));
  if (!moe::f8::supported(*shape))
    return fail(MOE_ERR_UNSUPPORTED,
                "the MXFP8 path needs bf16, d %% 256 == 0 and I %% 128 == 0 (d=%d, I=%d)",
                shape->d, shape->I);
  return MOE_OK;
}

moe_status moe_permute_mxfp8(const moe_shape* shape, const void* x, const int32_t* topk_idx,
                             const int32_t* counts, int32_t* offsets, int32_t* row_token,
                             int32_t* slot_pos, void* x_perm_q, void* x_perm_sf, void* ws,
                             size_t ws_bytes, void* stream) {
  g_err[0] = 0;
  NvtxRange nvtx_range_("moe_permute_mxfp8");
  MOE_TRY(check_mxfp8_shape(shape));
  const moe_shape& s = *shape;
  WsLayout L;
  MOE_TRY(check_ws(s, ws, ws_bytes, &L));
  MOE_TRY(need(offsets, "offsets", 4));
  if (s.T > 0) {
    MOE_TRY(need(x, "x", 16));
    MOE_TRY(need(topk_idx, "topk_idx", 4));
    MOE_TRY(need(row_token, "row_token", 4));
    MOE_TRY(need(slot_pos, "slot_pos", 4));
    MOE_TRY(need(x_perm_q, "x_perm_q", 16));
    MOE_TRY(need(x_perm_sf, "x_perm_sf", 16));
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  MOE_TRY(permute_impl<__nv_bfloat16>(s, x, topk_idx, counts, offsets, row_token, slot_pos,
                                      nullptr, ws, L, st));
  if (s.T > 0) {
    moe::launch_pdl(moe::gather_quant_kernel, dim3((s.T + 7) / 8), dim3(256), 0, st,
        static_cast<const __nv_bfloat16*>(x), slot_pos, s.T, s.K, s.d,
        static_cast<uint8_t*>(x_perm_q), static_cast<uint8_t*>(x_perm_sf));
    MOE_TRY(check_launch("quantising dispatch copy"));
  }
  return MOE_OK;
}

moe_status moe_expert_gate_up_mxfp8(const moe_shape* shape, const void* x_perm_q,
                                    const void* x_perm_sf, const void* w1_q, const void* w1_sf,
                                    const void* w3_q, const void* w3_sf, const int32_t* offsets,
                                    void* h_q, void* h_sf, void* ws, size_t ws_bytes,
                                    void* stream) {
  g_err[0] = 0;
  NvtxRange nvtx_range_("moe_expert_gate_up_mxfp8");
  MOE_TRY(check_mxfp8_shape(shape));
  const moe_shape& s = *shape;
  WsLayout L;
  MOE_TRY(check_ws(s, ws, ws_bytes, &L));
  MOE_TRY(need(x_perm_q, "x_perm_q", 16));
  MOE_TRY(need(x_perm_sf, "x_perm_sf", 16));
  MOE_TRY(need(w1_q, "w1_q", 16));
  MOE_TRY(need(w1_sf, "w1_sf", 16));
  MOE_TRY(need(w3_q, "w3_q", 16));
  MOE_TRY(need(w3_sf, "w3_sf", 16));
  MOE_TRY(need(offsets, "offsets", 4));
  MOE_TRY(need(h_q, "h_q", 16));
  MOE_TRY(need(h_sf, "h_sf", 4));
  if (s.T == 0) return MOE_OK;
  return moe::f8::launch_gate_up(s, x_perm_q, x_perm_sf, w1_q, w1_sf, w3_q, w3_sf, offsets, h_q,
                                 h_sf, at<uint32_t>(ws, L.status), sm_count(),
                                 static_cast<cudaStream_t>(stream), g_err, sizeof(g_err));
}

moe_status moe_expert_down_mxfp8(const moe_shape* shape, const void* h_q, const void* h_sf,
                                 const void* w2_q, const void* w2_sf, const int32_t* offsets,
                                 void* y_perm, void* ws, size_t ws_bytes, void* stream) {
  g_err[0] = 0;
  NvtxRange nvtx_range_("moe_expert_down_mxfp8");
  MOE_TRY(check_mxfp8_shape(shape));
  const moe_shape& s = *shape;
  WsLayout L;
  MOE_TRY(check_ws(s, ws, ws_bytes, &L));
  MOE_TRY(need(h_q, "h_q", 16));
  MOE_TRY(need(h_sf, "h_sf", 16));
  MOE_TRY(need(w2_q, "w2_q", 16));
  MOE_TRY(need(w2_sf, "w2_sf", 16));
  MOE_TRY(need(offsets, "offsets", 4));
  MOE_TRY(need(y_perm, "y_perm", 16));
  if (s.T == 0) return MOE_OK;
  return moe::f8::launch_down(s, h_q, h_sf, w2_q, w2_sf, offsets, y_perm,
                              at<uint32_t>(ws, L.status), sm_count(),
                              static_cast<cudaStream_t>(stream), g_err, sizeof(g_err));
}

moe_status moe_expert_gate_up(const moe_shape* shape, const void* x_perm, const void* w1,
                              const void* w3, const int32_t* offsets, void* h, void* ws,
                              size_t ws_bytes, void* stream) {
  g_err[0] = 0;
  NvtxRange nvtx_range_("moe_expert_gate_up");
  MOE_TRY(validate_shape(shape));
  const moe_shape& s = *shape;
  WsLayout L;
  MOE_TRY(check_ws(s, ws, ws_bytes, &L));
  MOE_TRY(need(x_perm, "x_perm", 16));
  MOE_TRY(need(w1, "w1", 16));
  MOE_TRY(need(w3, "w3", 16));
  MOE_TRY(need(offsets, "offsets", 4));
  MOE_TRY(need(h, "h", 16));
  return gate_up_impl(s, x_perm, w1, w3, offsets, h, at<uint32_t>(ws, L.status),
                      static_cast<cudaStream_t>(stream));
}

moe_status moe_expert_gate_up_gather(const moe_shape* shape, const void* x,
                                     const int32_t* row_token, const void* w1, const void* w3,
                                     const int32_t* offsets, void* h, void* ws, size_t ws_bytes,
                                     void* stream) {
  g_err[0] = 0;
  NvtxRange nvtx_range_("moe_expert_gate_up_gather");
  MOE_TRY(validate_shape(shape));
  const moe_shape& s = *shape;
  WsLayout L;
  MOE_TRY(check_ws(s, ws, ws_bytes, &L));
  if (s.T > 0) {  // an empty batch reads no token row and writes no h row
    MOE_TRY(need(x, "x", 16));
    MOE_TRY(need(row_token, "row_token", 4));
    MOE_TRY(need(h, "h", 16));
  }
  MOE_TRY(need(w1, "w1", 16));
  MOE_TRY(need(w3, "w3", 16));
  MOE_TRY(need(offsets, "offsets", 4));
  return gate_up_gather_impl(s, x, row_token, w1, w3, offsets, h, at<uint32_t>(ws, L.status),
                             static_cast<cudaStream_t>(stream));
}

moe_status moe_expert_down(const moe_shape* shape, const void* h, const void* w2,
                           const int32_t* offsets, void* y_perm, void* ws, size_t ws_bytes,
                           void* stream) {
  g_err[0] = 0;
  NvtxRange nvtx_range_("moe_expert_down");
  MOE_TRY(validate_shape(shape));
  const moe_shape& s = *shape;
  WsLayout L;
  MOE_TRY(check_ws(s, ws, ws_bytes, &L));
  MOE_TRY(need(h, "h", 16));
  MOE_TRY(need(w2, "w2", 16));
  MOE_TRY(need(offsets, "offsets", 4));
  MOE_TRY(need(y_perm, "y_perm", 16));
  return down_impl(s, h, w2, offsets, y_perm, at<uint32_t>(ws, L.status),
                   static_cast<cudaStream_t>(stream));
}

moe_status moe_expert_ffn(const moe_shape* shape, const void* x_perm, const void* w1,
                          const void* w3, const void* w2, const int32_t* offsets,
                          void* y_perm, void* ws, size_t ws_bytes, void* stream) {
  g_err[0] = 0;
  NvtxRange nvtx_range_("moe_expert_ffn");
  MOE_TRY(validate_shape(shape));
  const moe_shape& s = *shape;
  WsLayout L;
  MOE_TRY(check_ws(s, ws, ws_bytes, &L));
  MOE_TRY(need(x_perm, "x_perm", 16));
  MOE_TRY(need(w1, "w1", 16));
  MOE_TRY(need(w3, "w3", 16));
  MOE_TRY(need(w2, "w2", 16));
  MOE_TRY(need(offsets, "offsets", 4));
  MOE_TRY(need(y_perm, "y_perm", 16));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  void* h = at<char>(ws, L.h);
  uint32_t* status = at<uint32_t>(ws, L.status);
  MOE_TRY(gate_up_impl(s, x_perm, w1, w3, offsets, h, status, st));
  return down_impl(s, h, w2, offsets, y_perm, status, st);
}

moe_status moe_combine(const moe_shape* shape, const void* x, const void* y_perm,
                       const int32_t* topk_idx, const float* topk_gate,
                       const int32_t* slot_pos, float gamma, void* out, void* stream) {
  g_err[0] = 0;
  NvtxRange nvtx_range_("moe_combine");
  MOE_TRY(validate_shape(shape));
  const moe_shape& s = *shape;
  if (s.T == 0) return MOE_OK;
  MOE_TRY(need(x, "x", 16));
  MOE_TRY(need(y_perm, "y_perm", 16));
  MOE_TRY(need(topk_idx, "topk_idx", 4));
  MOE_TRY(need(topk_gate, "topk_gate", 4));
  MOE_TRY(need(slot_pos, "slot_pos", 4));
  MOE_TRY(need(out, "out", 16));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int E = s.N + s.Z;
  const int nvec = s.d * elem_bytes(s) / 16;
  int threads = ((nvec + 31) / 32) * 32;
  if (threads > 256) threads = 256;
  const int max_rows = s.T * s.K;
  if (s.dtype == MOE_BF16)
    moe::launch_pdl(moe::combine_kernel<__nv_bfloat16>, dim3(s.T), dim3(threads), 0, st,
        static_cast<const __nv_bfloat16*>(x), static_cast<const __nv_bfloat16*>(y_perm),
        topk_idx, topk_gate, slot_pos, s.K, s.N, E, s.d, max_rows, gamma,
        static_cast<__nv_bfloat16*>(out), nullptr);
  else
    moe::launch_pdl(moe::combine_kernel<float>, dim3(s.T), dim3(threads), 0, st,
        static_cast<const float*>(x), static_cast<const float*>(y_perm), topk_idx, topk_gate,
        slot_pos, s.K, s.N, E, s.d, max_rows, gamma, static_cast<float*>(out), nullptr);
  return check_launch("combine");
}

moe_status moe_bias_update(int32_t N, int32_t Z, const int32_t* counts, int64_t T_all,
                           int32_t K, float K_e, float mu, float* bias, void* stream) {
  g_err[0] = 0;
  NvtxRange nvtx_range_("moe_bias_update");
  if (N < 1 || Z < 0 || N + Z > moe::kMaxExperts)
    return fail(MOE_ERR_INVALID_ARG, "bad expert counts N=%d Z=%d", N, Z);
  if (K < 1 || K > N + Z) return fail(MOE_ERR_INVALID_ARG, "K=%d outside [1, N+Z]", K);
  if (T_all < 1) return fail(MOE_ERR_INVALID_ARG, "T_all=%lld must be >= 1", (long long)T_all);
  MOE_TRY(need(counts, "counts", 4));
  MOE_TRY(need(bias, "bias", 4));
  moe::launch_pdl(moe::bias_update_kernel, dim3((N + 255) / 256), dim3(256), 0, static_cast<cudaStream_t>(stream),
      N, counts, (long long)T_all, K, K_e, mu, bias);
  return check_launch("bias update");
}

moe_status moe_lb_stats(int32_t N, int32_t Z, int32_t D, const int32_t* counts,
                        const float* prob_sum, int64_t T, int32_t K, float K_e, float alpha,
                        float* f, float* P, float* loss, void* stream) {
  g_err[0] = 0;
  NvtxRange nvtx_range_("moe_lb_stats");
  if (N < 1 || Z < 1 || N + Z > moe::kMaxExperts)
    return fail(MOE_ERR_INVALID_ARG, "moe_lb_stats: needs N >= 1 and Z >= 1 (N=%d Z=%d)", N, Z);
  if (D < 1 || N % D) return fail(MOE_ERR_INVALID_ARG, "moe_lb_stats: D=%d must divide N=%d", D, N);
  if (K < 1 || K > N + Z) return fail(MOE_ERR_INVALID_ARG, "moe_lb_stats: K=%d", K);
  if (!(K_e > 0.f) || !(K_e < (float)K))
    return fail(MOE_ERR_INVALID_ARG, "moe_lb_stats: K_e=%g must lie in (0, K)", (double)K_e);
  if (T < 1) return fail(MOE_ERR_INVALID_ARG, "moe_lb_stats: T=%lld", (long long)T);
  MOE_TRY(need(counts, "counts", 4));
  MOE_TRY(need(prob_sum, "prob_sum", 4));
  MOE_TRY(need(f, "f", 4));
  MOE_TRY(need(P, "P", 4));
  moe::launch_pdl(moe::lb_stats_kernel, dim3(1), dim3(1024), 0, static_cast<cudaStream_t>(stream),
      N, Z, D, counts, prob_sum, (long long)T, K, K_e, alpha, f, P, loss);
  return check_launch("load-balance statistics");
}

// --- backward pass ----------------------------------------------------------

size_t moe_backward_workspace_bytes(const moe_shape* shape) {
  if (validate_shape(shape) != MOE_OK) return 0;
  return bwd_layout_of(*shape).total;
}

moe_status moe_expert_gate_up_save(const moe_shape* shape, const void* x_perm, const void* w1,
                                   const void* w3, const int32_t* offsets, void* h, void* au,
                                   void* ws, size_t ws_bytes, void* stream) {
  g_err[0] = 0;
  NvtxRange nvtx_range_("moe_expert_gate_up_save");
  MOE_TRY(validate_shape(shape));
  const moe_shape& s = *shape;
  WsLayout L;
  MOE_TRY(check_ws(s, ws, ws_bytes, &L));
  MOE_TRY(need(x_perm, "x_perm", 16));
  MOE_TRY(need(w1, "w1", 16));
  MOE_TRY(need(w3, "w3", 16));
  MOE_TRY(need(offsets, "offsets", 4));
  MOE_TRY(need(h, "h", 16));
  MOE_TRY(need(au, "au", 16));
  if (s.T == 0) return MOE_OK;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint32_t* status = at<uint32_t>(ws, L.status);
  if (s.dtype == MOE_BF16 && moe::tc::ffn_supported(s))
    return moe::tc::launch_gate_up_save(s, x_perm, w1, w3, offsets, h, au, status, sm_count(),
                                        st, g_err, sizeof(g_err));
  if (s.dtype == MOE_BF16)
    return fail(MOE_ERR_UNSUPPORTED, "bf16 moe_expert_gate_up_save needs d, I multiples of 64");
  // fp32: h by the gated kernel, a and u by two plain products into au
  MOE_TRY(gate_up_impl(s, x_perm, w1, w3, offsets, h, status, st));
  moe::SimtBwdArgs a{};
  a.A = x_perm;
  a.a_sm = s.d;
  a.a_sk = 1;
  a.b_sk = 1;
  a.b_sn = s.d;
  a.b_seg = (long long)s.I * s.d;
  a.c_sm = 2LL * s.I;
  a.offsets = offsets;
  a.nseg = s.N;
  a.max_rows = s.T * s.K;
  a.N = s.I;
  a.Kd = s.d;
  a.status = status;
  a.B0 = w1;
  a.C = au;
  MOE_TRY((simt_bwd<false, false>(a, simt_row_tiles(s, s.I), st, "pre-activation a")));
  a.B0 = w3;
  a.C = static_cast<float*>(au) + s.I;
  return simt_bwd<false, false>(a, simt_row_tiles(s, s.I), st, "pre-activation u");
}

moe_status moe_combine_backward(const moe_shape* shape, const void* x, const void* y_perm,
                                const int32_t* topk_idx, const float* topk_gate,
                                const int32_t* slot_pos, const void* dout, float gamma,
                                void* dy_perm, float* dgate, void* stream) {
  g_err[0] = 0;
  NvtxRange nvtx_range_("moe_combine_backward");
  MOE_TRY(validate_shape(shape));
  const moe_shape& s = *shape;
  if (s.T == 0) return MOE_OK;
  MOE_TRY(need(x, "x", 16));
  MOE_TRY(need(y_perm, "y_perm", 16));
  MOE_TRY(need(topk_idx, "topk_idx", 4));
  MOE_TRY(need(topk_gate, "topk_gate", 4));
  MOE_TRY(need(slot_pos, "slot_pos", 4));
  MOE_TRY(need(dout, "dout", 16));
  MOE_TRY(need(dy_perm, "dy_perm", 16));
  MOE_TRY(need(dgate, "dgate", 4));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int E = s.N + s.Z;
  const int nvec = s.d * elem_bytes(s) / 16;
  int threads = ((nvec + 31) / 32) * 32;
  if (threads > 256) threads = 256;
  const int max_rows = s.T * s.K;
  if (s.dtype == MOE_BF16)
    moe::launch_pdl(moe::combine_backward_kernel<__nv_bfloat16>, dim3(s.T), dim3(threads), 0, st,
        static_cast<const __nv_bfloat16*>(x), static_cast<const __nv_bfloat16*>(y_perm),
        topk_idx, topk_gate, slot_pos, static_cast<const __nv_bfloat16*>(dout), s.K, s.N, E,
        s.d, max_rows, gamma, static_cast<__nv_bfloat16*>(dy_perm), dgate, nullptr);
  else
    moe::launch_pdl(moe::combine_backward_kernel<float>, dim3(s.T), dim3(threads), 0, st,
        static_cast<const float*>(x), static_cast<const float*>(y_perm), topk_idx, topk_gate,
        slot_pos, static_cast<const float*>(dout), s.K, s.N, E, s.d, max_rows, gamma,
        static_cast<float*>(dy_perm), dgate, nullptr);
  return check_launch("combine backward");
}

moe_status moe_route_backward(const moe_shape* shape, const void* x, const void* w_router,
                              const float* probs, const int32_t* topk_idx, const float* dgate,
                              const float* lb_f, int32_t lb_groups, float lb_alpha,
                              int64_t lb_tokens, void* dw_router, float* dx_router, void* ws,
                              size_t ws_bytes, void* stream) {
  g_err[0] = 0;
  NvtxRange nvtx_range_("moe_route_backward");
  MOE_TRY(validate_shape(shape));
  const moe_shape& s = *shape;
  MOE_TRY(check_bwd_shape(s));
  BwdLayout L;
  MOE_TRY(check_bwd_ws(s, ws, ws_bytes, &L));
  MOE_TRY(need(w_router, "w_router", 16));
  MOE_TRY(need(dw_router, "dw_router", 16));
  const int E = s.N + s.Z;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (s.T == 0) {
    // no tokens: the router weight gradient is zero
    cudaError_t e = cudaMemsetAsync(dw_router, 0, (size_t)E * s.d * elem_bytes(s), st);
    if (e != cudaSuccess) return fail(MOE_ERR_CUDA, "memset: %s", cudaGetErrorString(e));
    return MOE_OK;
  }
  MOE_TRY(need(x, "x", 16));
  MOE_TRY(need(probs, "probs", 4));
  MOE_TRY(need(topk_idx, "topk_idx", 4));
  MOE_TRY(need(dgate, "dgate", 4));
  MOE_TRY(need(dx_router, "dx_router", 16));
  int lb_G = 1;
  float lb_scale = 0.f;
  if (lb_f) {
    MOE_TRY(need(lb_f, "lb_f", 4));
    if (lb_groups < 1 || s.N % lb_groups)
      return fail(MOE_ERR_INVALID_ARG, "lb_groups=%d must divide N=%d", lb_groups, s.N);
    if (lb_tokens < 1) return fail(MOE_ERR_INVALID_ARG, "lb_tokens=%lld", (long long)lb_tokens);
    lb_G = s.N / lb_groups;
    lb_scale = (float)((double)lb_alpha / (double)lb_tokens);
  }
  uint32_t* status = at<uint32_t>(ws, L.status);
  void* dlogits = at<char>(ws, L.dlogits);
  const int sms = sm_count();
  if (s.dtype == MOE_BF16) {
    moe::launch_pdl(moe::dlogits_kernel<__nv_bfloat16>, dim3((s.T + 7) / 8), dim3(256), 0, st,
        probs, topk_idx, dgate, s.T, E, s.K, lb_f, s.N, lb_G, lb_groups, lb_scale,
      static_cast<__nv_bfloat16*>(dlogits), status);
    MOE_TRY(check_launch("router logit gradient"));
    MOE_TRY(moe::tc::launch_router_wgrad(s, dlogits, x, dw_router, status, sms, st, g_err,
                                         sizeof(g_err)));
    return moe::tc::launch_router_dx(s, dlogits, w_router, dx_router, status, sms, st, g_err,
                                     sizeof(g_err));
  }
  moe::launch_pdl(moe::dlogits_kernel<float>, dim3((s.T + 7) / 8), dim3(256), 0, st,
      probs, topk_idx, dgate, s.T, E, s.K, lb_f, s.N, lb_G, lb_groups, lb_scale,
      static_cast<float*>(dlogits), status);
  MOE_TRY(check_launch("router logit gradient"));
  moe::SimtBwdArgs a{};
  // dW_r[i, j] = sum_t dlogits[t, i] x[t, j]
  a.A = dlogits;
  a.a_sm = 1;
  a.a_sk = E;
  a.B0 = x;
  a.b_sk = s.d;
  a.b_sn = 1;
  a.C = dw_router;
  a.c_sm = s.d;
  a.single_rows = s.T;
  a.max_rows = s.T;
  a.M = E;
  a.N = s.d;
  a.status = status;
  MOE_TRY((simt_bwd<true, false>(a, simt_kseg_tiles(1, E, s.d), st, "router weight gradient")));
  // dx_router[t, j] = sum_i dlogits[t, i] W_r[i, j]
  moe::SimtBwdArgs b{};
  b.A = dlogits;
  b.a_sm = E;
  b.a_sk = 1;
  b.B0 = w_router;
  b.b_sk = s.d;
  b.b_sn = 1;
  b.C = dx_router;
  b.c_sm = s.d;
  b.single_rows = s.T;
  b.max_rows = s.T;
  b.N = s.d;
  b.Kd = E;
  b.status = status;
  const long long tiles = (long long)((s.T + moe::kSbBM - 1) / moe::kSbBM) *
                          ((s.d + moe::kSbBN - 1) / moe::kSbBN);
  return simt_bwd<false, false>(b, tiles, st, "router input gradient");
}

moe_status moe_expert_ffn_backward(const moe_shape* shape, const void* x_perm, const void* w1,
                                   const void* w3, const void* w2, const int32_t* offsets,
                                   const void* h, const void* au, const void* dy_perm,
                                   void* dx_perm, void* dw1, void* dw3, void* dw2, void* ws,
                                   size_t ws_bytes, void* stream) {
  g_err[0] = 0;
  NvtxRange nvtx_range_("moe_expert_ffn_backward");
  MOE_TRY(validate_shape(shape));
  const moe_shape& s = *shape;
  MOE_TRY(check_bwd_shape(s));
  BwdLayout L;
  MOE_TRY(check_bwd_ws(s, ws, ws_bytes, &L));
  MOE_TRY(need(x_perm, "x_perm", 16));
  MOE_TRY(need(w1, "w1", 16));
  MOE_TRY(need(w3, "w3", 16));
  MOE_TRY(need(w2, "w2", 16));
  MOE_TRY(need(offsets, "offsets", 4));
  MOE_TRY(need(h, "h", 16));
  MOE_TRY(need(au, "au", 16));
  MOE_TRY(need(dy_perm, "dy_perm", 16));
  MOE_TRY(need(dx_perm, "dx_perm", 16));
  MOE_TRY(need(dw1, "dw1", 16));
  MOE_TRY(need(dw3, "dw3", 16));
  MOE_TRY(need(dw2, "dw2", 16));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint32_t* status = at<uint32_t>(ws, L.status);
  void* dau = at<char>(ws, L.dau);
  const int sms = sm_count();
  const int rows = s.T * s.K;
  if (s.T == 0) {
    // no tokens: every weight gradient is zero
    const size_t bytes = (size_t)s.N * s.I * s.d * elem_bytes(s);
    for (void* p : {dw1, dw3, dw2}) {
      cudaError_t e = cudaMemsetAsync(p, 0, bytes, st);
      if (e != cudaSuccess) return fail(MOE_ERR_CUDA, "memset: %s", cudaGetErrorString(e));
    }
    return MOE_OK;
  }
  if (s.dtype == MOE_BF16) {
    // data gradients (weights read, dau and dx_perm written), then weight
    // gradients (dW written).  Running the write-bound weight-gradient GEMMs
    // beside the read-bound data-gradient GEMMs on split SM partitions measured
    // no faster than this order.
    MOE_TRY(moe::tc::launch_dgrad_h(s, dy_perm, w2, offsets, au, dau, status, sms, st, g_err,
                                    sizeof(g_err)));
    MOE_TRY(moe::tc::launch_dgrad_x(s, dau, w1, w3, offsets, dx_perm, status, sms, st, g_err,
                                    sizeof(g_err)));
    MOE_TRY(moe::tc::launch_wgrad_w2(s, h, dy_perm, offsets, dw2, status, sms, st, g_err,
                                     sizeof(g_err)));
    return moe::tc::launch_wgrad_w13(s, x_perm, dau, offsets, dw1, dw3, status, sms, st,
                                      g_err, sizeof(g_err));
  }
  moe::SimtBwdArgs a{};
  a.offsets = offsets;
  a.nseg = s.N;
  a.max_rows = rows;
  a.status = status;
  {
    // dh = dy W2_e, then the SwiGLU backward into dau
    a.A = dy_perm;
    a.a_sm = s.d;
    a.a_sk = 1;
    a.B0 = w2;
    a.b_seg = (long long)s.d * s.I;
    a.b_sk = s.I;
    a.b_sn = 1;
    a.C = dau;
    a.N = s.I;
    a.Kd = s.d;
    a.au = au;
    MOE_TRY((simt_bwd<false, true>(a, simt_row_tiles(s, s.I), st, "expert dh")));
    // dx_perm = da W1_e + du W3_e (one reduction over 2I)
    moe::SimtBwdArgs b = a;
    b.A = dau;
    b.a_sm = 2LL * s.I;
    b.a_sk = 1;
    b.B0 = w1;
    b.B1 = w3;
    b.k_split = s.I;
    b.b_seg = (long long)s.I * s.d;
    b.b_sk = s.d;
    b.b_sn = 1;
    b.C = dx_perm;
    b.c_sm = s.d;
    b.N = s.d;
    b.Kd = 2 * s.I;
    b.au = nullptr;
    MOE_TRY((simt_bwd<false, false>(b, simt_row_tiles(s, s.d), st, "expert dx")));
  }
  // weight gradients: reductions over each expert's rows
  moe::SimtBwdArgs w{};
  w.offsets = offsets;
  w.nseg = s.N;
  w.max_rows = rows;
  w.status = status;
  w.A = dau;  // dW1[e][i, j] = sum_r da[r, i] x_perm[r, j]
  w.a_sm = 1;
  w.a_sk = 2LL * s.I;
  w.B0 = x_perm;
  w.b_sk = s.d;
  w.b_sn = 1;
  w.C = dw1;
  w.c_seg = (long long)s.I * s.d;
  w.c_sm = s.d;
  w.M = s.I;
  w.N = s.d;
  MOE_TRY((simt_bwd<true, false>(w, simt_kseg_tiles(s.N, s.I, s.d), st, "dW1")));
  w.A = static_cast<const float*>(dau) + s.I;  // du
  w.C = dw3;
  MOE_TRY((simt_bwd<true, false>(w, simt_kseg_tiles(s.N, s.I, s.d), st, "dW3")));
  w.A = dy_perm;  // dW2[e][j, i] = sum_r dy[r, j] h[r, i]
  w.a_sm = 1;
  w.a_sk = s.d;
  w.B0 = h;
  w.b_sk = s.I;
  w.b_sn = 1;
  w.C = dw2;
  w.c_seg = (long long)s.d * s.I;
  w.c_sm = s.I;
  w.M = s.d;
  w.N = s.I;
  return simt_bwd<true, false>(w, simt_kseg_tiles(s.N, s.d, s.I), st, "dW2");
}

moe_status moe_permute_backward(const moe_shape* shape, const void* dout,
                                const int32_t* topk_idx, const float* topk_gate,
                                const int32_t* slot_pos, const void* dx_perm,
                                const float* dx_router, float gamma, void* dx, void* stream) {
  g_err[0] = 0;
  NvtxRange nvtx_range_("moe_permute_backward");
  MOE_TRY(validate_shape(shape));
  const moe_shape& s = *shape;
  if (s.T == 0) return MOE_OK;
  MOE_TRY(need(dout, "dout", 16));
  MOE_TRY(need(topk_idx, "topk_idx", 4));
  MOE_TRY(need(topk_gate, "topk_gate", 4));
  MOE_TRY(need(slot_pos, "slot_pos", 4));
  MOE_TRY(need(dx_perm, "dx_perm", 16));
  MOE_TRY(need(dx, "dx", 16));
  if (dx_router) MOE_TRY(need(dx_router, "dx_router", 16));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int E = s.N + s.Z;
  const int nvec = s.d * elem_bytes(s) / 16;
  int threads = ((nvec + 31) / 32) * 32;
  if (threads > 256) threads = 256;
  const int max_rows = s.T * s.K;
  if (s.dtype == MOE_BF16)
    moe::launch_pdl(moe::permute_backward_kernel<__nv_bfloat16>, dim3(s.T), dim3(threads), 0, st,
        static_cast<const __nv_bfloat16*>(dout), topk_idx, topk_gate, slot_pos,
        static_cast<const __nv_bfloat16*>(dx_perm), dx_router, s.K, s.N, E, s.d, max_rows, gamma,
        static_cast<__nv_bfloat16*>(dx));
  else
    moe::launch_pdl(moe::permute_backward_kernel<float>, dim3(s.T), dim3(threads), 0, st,
        static_cast<const float*>(dout), topk_idx, topk_gate, slot_pos,
        static_cast<const float*>(dx_perm), dx_router, s.K, s.N, E, s.d, max_rows, gamma,
        static_cast<float*>(dx));
  return check_launch("permute backward");
}

moe_status moe_get_device_status(void* ws, void* stream, uint32_t* status_out) {
  g_err[0] = 0;
  NvtxRange nvtx_range_("moe_get_device_status");
  if (!ws) return fail(MOE_ERR_INVALID_ARG, "workspace is NULL");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint32_t v = 0;
  cudaError_t e = cudaStreamSynchronize(st);
  if (e == cudaSuccess) e = cudaMemcpy(&v, ws, sizeof(v), cudaMemcpyDeviceToHost);
  if (e == cudaSuccess) e = cudaMemsetAsync(ws, 0, sizeof(v), st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return fail(MOE_ERR_CUDA, "status read: %s", cudaGetErrorString(e));
  if (status_out) *status_out = v;
  if (v) return fail(MOE_ERR_DEVICE_STATUS, "device status 0x%x", v);
  return MOE_OK;
}

const char* moe_last_error(void) { return g_err; }

uint64_t moe_kernel_launches(void) { return moe::launch_counter().load(); }

moe_status moe_debug_set_pipeline(uint64_t wait_limit_ns, int32_t stall_first_fill) {
  g_err[0] = 0;
  if (wait_limit_ns > 60000000000ull)
    return fail(MOE_ERR_INVALID_ARG, "wait limit %llu ns is above one minute",
                (unsigned long long)wait_limit_ns);
  moe::pipeline_debug().wait_ns.store(wait_limit_ns, std::memory_order_relaxed);
  moe::pipeline_debug().stall_fill.store(stall_first_fill ? 1 : 0, std::memory_order_relaxed);
  return MOE_OK;
}

}  // extern "C"
