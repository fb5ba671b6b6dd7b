// Tensor-core GEMMs of the bf16 path on sm_100a: tcgen05.mma with fp32
// accumulators in TMEM, operands staged in shared memory by TMA.
//
// Orientation ("swap AB"): the weight rows are the UMMA M operand (128
// output features per MMA) and the routed token rows are the N operand
// (16..256 rows, rounded up to 16).  Expert segments are ragged (about 128
// rows per expert at the LongCat shape), so putting tokens on N wastes at most
// 15 padded rows per segment instead of up to 127 with tokens on M, and every
// weight tile is streamed from HBM exactly once per (expert, 256-row chunk).
//
// One persistent CTA per SM, 6 warps:
//   warp 0      TMA producer (one lane): A0, A1 weight tiles + B token tile per stage
//   warp 1      MMA issuer (one lane); also allocates/frees the 512 TMEM columns
//   warps 2..5  epilogue: TMEM -> registers -> (SwiGLU | copy) -> shared -> global
// Pipeline: kStages shared-memory stages guarded by full/empty mbarriers, one or
// two TMEM accumulator pairs guarded by tmem_full/tmem_empty.  Every wait is bounded
// in time; on expiry the CTA raises MOE_DEV_PIPELINE_TIMEOUT, drains what it
// issued and returns.
//
// Tile = (row chunk of <= 256 token rows of one expert, feature block):
//   gated mode  (first half of the SwiGLU expert): D0 = W1 rows f0..f0+127,
//               D1 = W3 rows f0..f0+127, out h = SiLU(D0) * D1 (bf16)
//   plain modes (second half, router): D0 = rows f0..f0+127, D1 = rows
//               f0+128..f0+255 of one weight matrix; out bf16 or fp32 (+offset)
//   gated-save  (training forward): h as the gated mode, plus a = D0, u = D1
//   SwiGLU backward: D0 | D1 = dh; epilogue da = dh u SiLU'(a), du = dh SiLU(a)
// MN-major A (template flag, the backward's data gradients and the router's
// input gradient): the weights are read in their stored order with the output
// features as their columns -- 64 x 64 TMA boxes and the transpose bit of the
// instruction descriptor instead of a transposed copy -- and the reduction may
// switch from tmA0 to tmA1 part-way (dx = da W1 + du W3 in one accumulator).
// Split-K (the router at small batches): K-block ranges on separate CTAs write
// fp32 partial sums that the consumer adds in a fixed order.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstdio>

#include "common.cuh"

namespace moe {
namespace tc {

constexpr int kBK = 64;                          // K elements per stage = one 128-byte row
constexpr int kFeat = 128;                       // UMMA M
constexpr int kBoxRows = 32;                     // rows per token TMA box
constexpr int kABytes = kFeat * kBK * 2;         // 16 KiB
constexpr int kBoxBytes = kBoxRows * kBK * 2;    // 4 KiB
constexpr int kThreads = 192;
constexpr int kEpiWarps = 4;
constexpr int kStagingPitch = 36;                // fp32 staging row: 32 words + pad
constexpr int kStagingPitch16 = 40;              // bf16 staging row: 32 halves + pad (80 B)
constexpr int kStagingBytesF32 = kEpiWarps * 32 * kStagingPitch * 4;
constexpr int kStagingBytesBf16 = kEpiWarps * 32 * kStagingPitch16 * 2;
constexpr int kStagingBytesF32Half = kEpiWarps * 16 * kStagingPitch * 4;  // 16 token rows
constexpr int kCtrlBytes = 256;                  // barriers + tmem slot + abort flag
constexpr unsigned long long kWaitTimeoutNs = kDefaultWaitNs;  // when a launch sets none
constexpr unsigned long long kDrainTimeoutNs = 200000000ull;  // 0.2 s

// Tile geometry: up to kNMax token rows per tile (UMMA N), kStages shared-memory
// stages.  The D0/D1 accumulator pair takes 2*kNMax TMEM columns; when two
// pairs fit in the 512 columns the accumulators are double-buffered, so the
// epilogue of one tile overlaps the MMAs of the next.
template <int NMAX, int STAGES, int PREFIX_INTS = kMaxExperts + 1 + 33,
          bool DIRECT_F32 = false>
struct TileCfg {
  static constexpr int kNMax = NMAX;
  static constexpr int kStages = STAGES;
  // chunk prefix of the expert segments (+ scan scratch); a single-segment
  // GEMM (the router) needs two entries
  static constexpr int kPrefixInts = PREFIX_INTS;
  // fp32 epilogue (router mode) without a staging area: lane = feature, each
  // store one 128-byte row piece (faster for the one-tile-per-CTA router, slower
  // for the split-K router, whose epilogue is most of each CTA's time)
  static constexpr bool kDirectF32 = DIRECT_F32;
  static constexpr int kAccBufs = (4 * NMAX <= 512) ? 2 : 1;
  static constexpr int kTmemCols = 512;
  static constexpr int kBBytes = NMAX * kBK * 2;
  static constexpr int kStageBytes = 2 * kABytes + kBBytes;
  static constexpr int kNumBars = 2 * STAGES + 2 * kAccBufs + 1;  // full, empty, acc full/empty, drain
  // shared memory for an epilogue whose staging area takes `staging` bytes
  __host__ __device__ static constexpr int smem_bytes(int staging) {
    return 1024 + STAGES * kStageBytes + staging + kCtrlBytes + PREFIX_INTS * 4;
  }
  static_assert(NMAX % kBoxRows == 0 && NMAX <= 256, "token tile");
  static_assert(8 * kNumBars + 12 <= kCtrlBytes, "control block");
};
using CfgWide = TileCfg<256, 3>;    // segments up to 256 rows in one tile, 3 stages
using CfgN160 = TileCfg<160, 4>;    // segments up to 160 rows, 4 stages (more bytes in flight)
using CfgDouble = TileCfg<128, 4>;  // <= 128 rows, double-buffered accumulators
// decode batches (a few rows per expert): 64-row token tiles leave room for a
// fifth stage, 160 KB of weight tiles in flight per SM against 128 KB
using CfgN64 = TileCfg<64, 5>;
// router: 192 token rows (one wave at T = 8192, E = 768), one segment, four stages
// (the fp32 epilogue needs no staging area)
#ifndef MOE_ROUTER_STAGES
#define MOE_ROUTER_STAGES 4
#endif
using CfgR192 = TileCfg<192, MOE_ROUTER_STAGES, 16, true>;
static_assert(CfgWide::smem_bytes(kStagingBytesF32) <= 232448, "router tile");
static_assert(CfgR192::smem_bytes(0) <= 232448, "router tile");
static_assert(CfgN160::smem_bytes(kStagingBytesF32Half) <= 232448, "SwiGLU backward tile");

// Epilogue modes.
//   kGated      h = SiLU(D0) * D1 (bf16)                      forward gate/up
//   kPlainBf16  D0 | D1 as features f0.. / f0+128.. (bf16)    forward down, backward dx
//   kPlainF32   the same in fp32 (+ optional addend)          router logits, router dx
//   kSwigluBwd  D = dh; with a, u read from `au`:             backward of SiLU(a) * u
//               da = dh u s (1 + a (1 - s)), du = dh a s, s = sigmoid(a)
//   kGatedSave  kGated that also writes a = D0 and u = D1 to `aux_out`
enum Mode { kGated = 0, kPlainBf16 = 1, kPlainF32 = 2, kSwigluBwd = 3, kGatedSave = 4 };

template <int kMode, class Cfg> __host__ __device__ constexpr int staging_bytes() {
  return kMode == kPlainF32 ? (Cfg::kDirectF32 ? 0 : kStagingBytesF32)
                            : kMode == kSwigluBwd ? kStagingBytesF32Half : kStagingBytesBf16;
}

struct Args {
  const int32_t* seg_offsets;  // [nseg+1] routed-row offsets, or NULL for one segment
  int nseg;                    // experts (or 1)
  int single_rows;             // rows of the single segment when seg_offsets == NULL
  int max_rows;                // rows of the token matrix (bound for offsets)
  int n_out;                   // output features (row stride of `out`)
  int k_dim;                   // reduction length (multiple of 64)
  int a_seg_rows;              // weight rows per expert in the 2-D weight view
  int a1_row_off;              // D1 weight rows = D0 rows + this (plain modes)
  int feat_per_tile;           // 128 (gated) or 256 (plain)
  void* out;
  const float* add;            // fp32 addend [rows, n_out] (router logit offset) or NULL
  uint32_t* status;
  const int32_t* gather_rows;  // token of each routed row: B rows are copied from x through
                               // this map by the producer lanes (cp.async, 16 bytes each);
                               // NULL: B rows are rows of tmB itself (TMA boxes)
  int gather_src_rows;         // rows of x (bound for the gathered tokens)
  const void* gather_src;      // x [gather_src_rows, k_dim] bf16 when gathering
  int a_tiled;                 // weights in MOE_WEIGHTS_TILED order: the A tile of weight rows
                               // r..r+127 (r % 128 == 0), columns kb*64.. is row (r/128*nk+kb)*128
                               // of a [tiles*128, 64] view
  // MN-major A (the kernel's kAMN form: the output features are the weight's
  // columns, the reduction runs over its rows).  K block kb reads weight rows
  // seg*a_seg_rows + kb*64 .. +63 of tmA0, or of tmA1 from K block a_k_split on
  // (rows counted from that block); D0 = columns f0..f0+127, D1 = columns
  // f0+a1_row_off..+127.  0: no split.
  int a_k_split;
  const void* au;              // kSwigluBwd: pre-activations [rows, 2*n_out] (a | u)
  void* aux_out;               // kGatedSave: a | u output [rows, 2*n_out]
  // Split-K (kPlainF32, one segment): K blocks are cut into k_splits ranges;
  // split s writes its fp32 partial sums at out + s*split_stride (the addend
  // goes to split 0 only).  0 or 1: no split.
  int k_splits;
  long long split_stride;
  int single_half;             // plain modes: tiles of 128 features, D1 neither loaded nor computed
  int32_t* zero_i32;           // cleared by CTA 0 after the grid dependency (router: the counts
  int zero_n;                  // the selection kernel then accumulates), or NULL
  int prefetch_b;              // TMA producer: prefetch the token boxes of K block kb + this into
                               // L2 while issuing kb (0: off)
  int spec_prefetch_kb;        // before the grid dependency: L2 prefetch of the first this-many K
                               // blocks of the weight tile the CTA most likely takes (0: off)
  unsigned long long wait_ns;  // time limit of one pipeline wait (set at launch)
  int stall_fill;              // test of the timeout path: the producer issues nothing, so the
                               // MMA issuer's first wait runs out
};

// TMA coordinates (column, row) of the weight tile whose first row is `row`
// (a multiple of 128 when tiled) for K block kb.
MOE_DEV int2 a_coord(const Args& a, int row, int kb, int nk) {
  return a.a_tiled ? make_int2(0, ((row >> 7) * nk + kb) << 7) : make_int2(kb * kBK, row);
}
// MN-major form: the 64 x 64 box of weight rows krow..krow+63 (krow % 64 == 0)
// and columns col..col+63.  In the tiled order the box lies inside tile
// (krow/128, col/64) of a matrix with n_out columns.
MOE_DEV int2 a_mn_coord(const Args& a, int krow, int col) {
  return a.a_tiled
             ? make_int2(0, (((krow >> 7) * (a.n_out >> 6) + (col >> 6)) << 7) + (krow & 127))
             : make_int2(col, krow);
}

// --- PTX wrappers --------------------------------------------------------------
MOE_DEV uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
MOE_DEV uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
MOE_DEV void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
MOE_DEV void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}
MOE_DEV void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
MOE_DEV bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait: false when the abort flag is raised or the time limit passes
// (then the flag is raised and the status word records the timeout).
MOE_DEV bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                       uint32_t* status, unsigned long long limit_ns = kWaitTimeoutNs,
                       bool honour_abort = true) {
  if (limit_ns == 0) limit_ns = kWaitTimeoutNs;
  uint64_t t0 = 0;
  for (uint32_t it = 0;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 31) == 31) {
      if (honour_abort && *abort_flag) return false;
      const uint64_t now = globaltimer();
      if (t0 == 0) {
        t0 = now;
      } else if (now - t0 > limit_ns) {
        *abort_flag = 1;
        set_status(status, MOE_DEV_PIPELINE_TIMEOUT);
        return false;
      }
    }
  }
}
MOE_DEV void tma_load_2d(uint32_t dst, const CUtensorMap* map, int c0, int c1, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(bar)
      : "memory");
}
// Same copy with an L2 eviction-priority hint (a createpolicy value).
MOE_DEV void tma_load_2d_hint(uint32_t dst, const CUtensorMap* map, int c0, int c1, uint32_t bar,
                              uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(bar), "l"(policy)
      : "memory");
}
// Weights are read once per step: evict them first.  Token tiles are re-read by
// every feature block of their expert: keep them.
MOE_DEV uint64_t l2_policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}
MOE_DEV uint64_t l2_policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}
// SiLU for the bf16 epilogue: a / (1 + e^-a) with the fast exponential and
// division intrinsics (relative error ~1e-6, far below the bf16 rounding of h).
MOE_DEV float silu_fast(float a) { return __fdividef(a, 1.0f + __expf(-a)); }
// 16-byte asynchronous copy global -> shared through L2 with an eviction hint,
// and the arrival on an mbarrier once all of this thread's copies have landed.
MOE_DEV void cp_async_16_hint(uint32_t dst, const void* src, uint64_t policy) {
  asm volatile("cp.async.cg.shared.global.L2::cache_hint [%0], [%1], 16, %2;" ::"r"(dst),
               "l"(src), "l"(policy)
               : "memory");
}
MOE_DEV void cp_async_arrive_noinc(uint32_t bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
}
// Bulk prefetch of `bytes` (a multiple of 16, 16-byte aligned) into L2.
MOE_DEV void l2_prefetch_bulk(const void* p, int bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}
// L2 prefetch of one box of a tensor map (no shared memory, no barrier).
MOE_DEV void tma_prefetch_l2(const CUtensorMap* map, int c0, int c1) {
  asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(c0), "r"(c1)
               : "memory");
}
MOE_DEV void tma_prefetch_desc(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}
MOE_DEV void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
MOE_DEV void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Shared-memory matrix descriptor, K-major operand in the 128-byte swizzle
// layout: rows of 128 bytes, 8-row (1024-byte) swizzle atoms stacked densely.
//   bits  0-13 start address >> 4     bits 16-29 leading byte offset >> 4 (unused: 1)
//   bits 32-45 stride byte offset >> 4 (1024 B between 8-row groups)
//   bits 46-47 version (1 on sm_100)  bits 61-63 layout (2 = 128-byte swizzle)
MOE_DEV uint64_t smem_desc_sw128(uint32_t addr) {
  uint64_t d = 0;
  d |= (uint64_t)((addr >> 4) & 0x3fff);
  d |= (uint64_t)1 << 16;
  d |= (uint64_t)(1024 >> 4) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}
// MN-major operand in the 128-byte swizzle layout, as TMA writes 64 x 64 boxes
// (64 K rows of 128 bytes = 64 MN elements): 8 K rows form a 1024-byte
// swizzle atom, consecutive atoms along K are 1024 bytes apart (stride byte
// offset) and the next 64 MN elements start 8192 bytes further on (leading
// byte offset, the second box).  One K = 16 step advances 2048 bytes.
constexpr int kMnBoxBytes = 8192;
MOE_DEV uint64_t smem_desc_mn_sw128(uint32_t addr) {
  uint64_t d = 0;
  d |= (uint64_t)((addr >> 4) & 0x3fff);
  d |= (uint64_t)(kMnBoxBytes >> 4) << 16;
  d |= (uint64_t)(1024 >> 4) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}
// Instruction descriptor of kind::f16: fp32 D, bf16 A and B.
//   bits 4-5 D format (1 = f32), 7-9 A format (1 = bf16), 10-12 B format,
//   15/16 A/B major (0 = K, 1 = MN), 17-22 N >> 3, 24-28 M >> 4.
MOE_DEV uint32_t idesc_bf16(int m, int n, bool a_mn = false, bool b_mn = false) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn ? 1u : 0u) << 15) |
         ((b_mn ? 1u : 0u) << 16) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(m >> 4) << 24);
}
MOE_DEV void umma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
MOE_DEV void umma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   bar)
               : "memory");
}
// 32 lanes x 32 consecutive 32-bit TMEM columns: thread i gets row (lane base + i).
MOE_DEV void tmem_ld_32x32b_x32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
MOE_DEV void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// --- tile decoding ---------------------------------------------------------------
struct Tile {
  int seg, r0, n, f0;
};

template <int kNMax>
MOE_DEV Tile decode_tile(int tile, int n_fblk, const Args& a, const int* prefix) {
  Tile t;
  const int chunk = tile / n_fblk;
  const int fb = tile - chunk * n_fblk;
  int lo, hi, c0;
  if (a.seg_offsets) {
    t.seg = find_expert(prefix, a.nseg, chunk);
    lo = a.seg_offsets[t.seg];
    hi = a.seg_offsets[t.seg + 1];
    c0 = prefix[t.seg];
  } else {
    t.seg = 0;
    lo = 0;
    hi = a.single_rows;
    c0 = 0;
  }
  t.r0 = lo + (chunk - c0) * kNMax;
  t.n = min(kNMax, hi - t.r0);
  t.f0 = fb * a.feat_per_tile;
  return t;
}

// --- epilogue helpers --------------------------------------------------------------
MOE_DEV float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
MOE_DEV float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }
MOE_DEV float sigmoid_fast(float a) { return __fdividef(1.0f, 1.0f + __expf(-a)); }

// 32 tokens x this warp's 32 features, bf16 pairs packed along tokens
// (pk[j/2] = tokens j, j+1 of this lane's feature): transposed through the
// warp's staging rows and stored as 16-byte row pieces of out[row0 + j, fbase..].
MOE_DEV void stage_store_bf16x32(const uint32_t (&pk)[16], uint16_t* s16, int lane,
                                 __nv_bfloat16* out, size_t ld, int row0, int nrows, int fbase,
                                 int fmax) {
#pragma unroll
  for (int j = 0; j < 32; j += 2) {
    s16[j * kStagingPitch16 + lane] = (uint16_t)(pk[j >> 1] & 0xffffu);
    s16[(j + 1) * kStagingPitch16 + lane] = (uint16_t)(pk[j >> 1] >> 16);
  }
  __syncwarp();
#pragma unroll
  for (int it = 0; it < 4; ++it) {
    const int vec = it * 32 + lane;
    const int j = vec >> 2, c = vec & 3;
    const int f = fbase + c * 8;
    if (j < nrows && f < fmax)
      *reinterpret_cast<uint4*>(out + (size_t)(row0 + j) * ld + f) =
          *reinterpret_cast<const uint4*>(&s16[j * kStagingPitch16 + c * 8]);
  }
  __syncwarp();
}

// --- the kernel ------------------------------------------------------------------
template <int kMode, class Cfg, bool kAMN = false>
__global__ void __launch_bounds__(kThreads, 1)
gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmA1,
               const __grid_constant__ CUtensorMap tmB, const Args args) {
  pdl_trigger();
  constexpr int kNMax = Cfg::kNMax, kStages = Cfg::kStages, kAccBufs = Cfg::kAccBufs;
  constexpr int kStageBytes = Cfg::kStageBytes, kNumBars = Cfg::kNumBars;
  constexpr int kTmemCols = Cfg::kTmemCols;
  constexpr int kStagingBytes = staging_bytes<kMode, Cfg>();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* stages = smem;
  uint32_t* staging = reinterpret_cast<uint32_t*>(smem + kStages * kStageBytes);
  uint8_t* ctrl = smem + kStages * kStageBytes + kStagingBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(ctrl);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(ctrl + 8 * kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(ctrl + 8 * kNumBars + 4);
  volatile int* consumed_sh = reinterpret_cast<volatile int*>(ctrl + 8 * kNumBars + 8);
  int* prefix = reinterpret_cast<int*>(ctrl + kCtrlBytes);
  int* scan_tmp = prefix + kMaxExperts + 1;  // used only with seg_offsets (full prefix)

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t full0 = smem_u32(&bars[0]);
  const uint32_t empty0 = smem_u32(&bars[kStages]);
  const uint32_t tmem_full0 = smem_u32(&bars[2 * kStages]);             // + 8 * buffer
  const uint32_t tmem_empty0 = smem_u32(&bars[2 * kStages + kAccBufs]);  // + 8 * buffer
  const uint32_t drain_bar = smem_u32(&bars[2 * kStages + 2 * kAccBufs]);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      // gathered B rows: the producer's expect_tx plus one cp.async arrival per lane
      mbar_init(full0 + 8 * s, args.gather_rows ? 1 + 32 : 1);
      mbar_init(empty0 + 8 * s, 1);
    }
    for (int b = 0; b < kAccBufs; ++b) {
      mbar_init(tmem_full0 + 8 * b, 1);
      mbar_init(tmem_empty0 + 8 * b, kEpiWarps * 32);
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    *consumed_sh = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    tma_prefetch_desc(&tmA0);
    tma_prefetch_desc(&tmA1);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  if (args.spec_prefetch_kb > 0 && warp == 0 && args.seg_offsets) {
    // While the preceding kernel (the route) runs, HBM is idle: bring into L2
    // the first K blocks of the weight tile this CTA takes when every expert
    // has rows and fits one token tile (tile b = expert b / n_fblk, feature
    // block b % n_fblk; at decode nearly every expert is touched).  A prefetch
    // is only a hint: a wrong guess costs bandwidth, and L2 stays coherent with
    // whatever the preceding kernels write, so no result can change.
    const int nfb = (args.n_out + args.feat_per_tile - 1) / args.feat_per_tile;
    const int seg = blockIdx.x / nfb;
    if (seg < args.nseg) {
      const int a_row0 = seg * args.a_seg_rows + (blockIdx.x - seg * nfb) * args.feat_per_tile;
      const int a_row1 = a_row0 + args.a1_row_off;
      const int nk = args.k_dim / kBK;
      const int nkb = min(args.spec_prefetch_kb, nk);
      for (int kb = lane; kb < nkb; kb += 32) {
        const int2 c0 = a_coord(args, a_row0, kb, nk);
        tma_prefetch_l2(&tmA0, c0.x, c0.y);
        if (!args.single_half) {
          const int2 c1 = a_coord(args, a_row1, kb, nk);
          tma_prefetch_l2(&tmA1, c1.x, c1.y);
        }
      }
    }
  }
  pdl_wait();  // the prologue above reads no memory a preceding kernel writes
  if (args.zero_i32 && blockIdx.x == 0)
    for (int i = threadIdx.x; i < args.zero_n; i += blockDim.x) args.zero_i32[i] = 0;
  if (args.seg_offsets) {
    build_chunk_prefix(args.seg_offsets, args.nseg, args.max_rows, kNMax, prefix, scan_tmp,
                       args.status);
  } else if (threadIdx.x == 0) {
    prefix[0] = 0;
    prefix[1] = (args.single_rows + kNMax - 1) / kNMax;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int nseg = args.seg_offsets ? args.nseg : 1;
  const int n_fblk = (args.n_out + args.feat_per_tile - 1) / args.feat_per_tile;
  const int ksplit = args.k_splits > 1 ? args.k_splits : 1;
  const int base_tiles = prefix[nseg] * n_fblk;
  const int total = base_tiles * ksplit;
  const int nk = args.k_dim / kBK;
  // tile -> (row chunk, feature block) and its K-block range [kb0, kb1)
  auto tile_of = [&](int tile, int& sp, int& kb0, int& kb1) {
    sp = tile / base_tiles;
    kb0 = sp * nk / ksplit;
    kb1 = (sp + 1) * nk / ksplit;
    return decode_tile<kNMax>(tile - sp * base_tiles, n_fblk, args, prefix);
  };
  int issued = 0;  // producer: stages issued
  const int produce = args.stall_fill ? 0 : total;  // tiles the producer fills

  if (warp == 0 && args.gather_rows) {
    // ---------------- producer, B rows gathered from x with cp.async ----------------
    // Lane 0 waits for the stage and loads the two weight tiles by TMA; every
    // lane then copies the K slice of its token rows (rows lane, lane + 32, ...)
    // into the 128-byte-swizzled B tile, 16 bytes per copy, and arrives on the
    // stage barrier once its copies have landed.
    uint32_t stage = 0, phase = 0;
    bool ok = true;
    const uint64_t pol_w = l2_policy_evict_first();
    const uint64_t pol_x = l2_policy_evict_last();
    constexpr int kRowsPerLane = kNMax / 32;
    const __nv_bfloat16* xsrc = static_cast<const __nv_bfloat16*>(args.gather_src);
    for (int tile = blockIdx.x; tile < produce && ok; tile += gridDim.x) {
      int sp, kb0, kb1;
      const Tile t = tile_of(tile, sp, kb0, kb1);
      const int a_row0 = t.seg * args.a_seg_rows + t.f0;
      const int a_row1 = a_row0 + args.a1_row_off;
      const __nv_bfloat16* src[kRowsPerLane];
#pragma unroll
      for (int i = 0; i < kRowsPerLane; ++i) {
        const int row = lane + 32 * i;
        int v = 0;
        if (row < t.n) {
          v = args.gather_rows[t.r0 + row];
          if (v < 0 || v >= args.gather_src_rows) {
            set_status(args.status, MOE_DEV_BAD_OFFSETS);
            v = 0;
          }
        }
        src[i] = xsrc + (size_t)v * args.k_dim;
      }
      for (int kb = kb0; kb < kb1; ++kb) {
        int go = 1;
        if (lane == 0) go = mbar_wait(empty0 + 8 * stage, phase ^ 1, abort_flag, args.status, args.wait_ns);
        go = __shfl_sync(0xffffffffu, go, 0);
        if (!go) {
          ok = false;
          break;
        }
        const uint32_t fb = full0 + 8 * stage;
        const uint32_t sa0 = smem_u32(stages + stage * kStageBytes);
        if (lane == 0) {
          mbar_arrive_expect_tx(fb, 2 * kABytes);
          const int2 c0 = a_coord(args, a_row0, kb, nk), c1 = a_coord(args, a_row1, kb, nk);
          tma_load_2d_hint(sa0, &tmA0, c0.x, c0.y, fb, pol_w);
          tma_load_2d_hint(sa0 + kABytes, &tmA1, c1.x, c1.y, fb, pol_w);
          ++issued;
        }
        const uint32_t sb = sa0 + 2 * kABytes;
#pragma unroll
        for (int i = 0; i < kRowsPerLane; ++i) {
          const int row = lane + 32 * i;
          if (row < t.n) {
            const __nv_bfloat16* g = src[i] + kb * kBK;
#pragma unroll
            for (int c = 0; c < 8; ++c)  // 16-byte chunk c of the row, swizzled position
              cp_async_16_hint(sb + row * 128 + ((c ^ (row & 7)) << 4), g + c * 8, pol_x);
          }
        }
        cp_async_arrive_noinc(fb);
        if (++stage == kStages) { stage = 0; phase ^= 1; }
      }
    }
    __syncwarp();
  } else if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer ----------------
      uint32_t stage = 0, phase = 0;
      bool ok = true;
      const uint64_t pol_w = l2_policy_evict_first();
      const uint64_t pol_x = l2_policy_evict_last();
      for (int tile = blockIdx.x; tile < produce && ok; tile += gridDim.x) {
        int sp, kb0, kb1;
        const Tile t = tile_of(tile, sp, kb0, kb1);
        const int nbox = (t.n + kBoxRows - 1) / kBoxRows;
        if constexpr (kMode == kSwigluBwd) {
          // the epilogue of this tile reads a and u of its rows and 256 features:
          // bring them into L2 while the main loop streams the weights
          const int nf = min(2 * kFeat, args.n_out - t.f0) * 2;  // bytes per row and half
          const char* au = static_cast<const char*>(args.au);
          for (int j = 0; j < t.n; ++j) {
            const char* row = au + ((size_t)(t.r0 + j) * 2 * args.n_out + t.f0) * 2;
            l2_prefetch_bulk(row, nf);
            l2_prefetch_bulk(row + (size_t)args.n_out * 2, nf);
          }
        }
        const uint32_t tx = (args.single_half ? 1 : 2) * kABytes + nbox * kBoxBytes;
        const int a_row0 = t.seg * args.a_seg_rows + t.f0;
        const int a_row1 = a_row0 + args.a1_row_off;
        const int pf = args.prefetch_b;
        for (int kb = kb0; kb < kb1 && kb < kb0 + pf; ++kb)
          for (int b = 0; b < nbox; ++b) tma_prefetch_l2(&tmB, kb * kBK, t.r0 + b * kBoxRows);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (pf > 0 && kb + pf < kb1)
            for (int b = 0; b < nbox; ++b)
              tma_prefetch_l2(&tmB, (kb + pf) * kBK, t.r0 + b * kBoxRows);
          if (!mbar_wait(empty0 + 8 * stage, phase ^ 1, abort_flag, args.status, args.wait_ns)) {
            ok = false;
            break;
          }
          const uint32_t fb = full0 + 8 * stage;
          const uint32_t sa0 = smem_u32(stages + stage * kStageBytes);
          mbar_arrive_expect_tx(fb, tx);
          if constexpr (kAMN) {
            // four 64 x 64 boxes: D0 columns f0, f0+64; D1 columns f0+a1_row_off, +64
            const bool second = args.a_k_split > 0 && kb >= args.a_k_split;
            const CUtensorMap* am = second ? &tmA1 : &tmA0;
            const int krow = t.seg * args.a_seg_rows + (second ? kb - args.a_k_split : kb) * kBK;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const int2 c0 = a_mn_coord(args, krow, t.f0 + 64 * h);
              const int2 c1 = a_mn_coord(args, krow, t.f0 + args.a1_row_off + 64 * h);
              tma_load_2d_hint(sa0 + h * kMnBoxBytes, am, c0.x, c0.y, fb, pol_w);
              tma_load_2d_hint(sa0 + kABytes + h * kMnBoxBytes, am, c1.x, c1.y, fb, pol_w);
            }
          } else {
            const int2 c0 = a_coord(args, a_row0, kb, nk), c1 = a_coord(args, a_row1, kb, nk);
            tma_load_2d_hint(sa0, &tmA0, c0.x, c0.y, fb, pol_w);
            if (!args.single_half) tma_load_2d_hint(sa0 + kABytes, &tmA1, c1.x, c1.y, fb, pol_w);
          }
          for (int b = 0; b < nbox; ++b)
            tma_load_2d_hint(sa0 + 2 * kABytes + b * kBoxBytes, &tmB, kb * kBK,
                             t.r0 + b * kBoxRows, fb, pol_x);
          ++issued;
          if (++stage == kStages) { stage = 0; phase ^= 1; }
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer ----------------
      uint32_t stage = 0, phase = 0;
      bool ok = true;
      int consumed = 0, local = 0;
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x, ++local) {
        int sp, kb0, kb1;
        const Tile t = tile_of(tile, sp, kb0, kb1);
        int n16 = ((t.n + 15) >> 4) << 4;
        if (n16 < 16) n16 = 16;
        const uint32_t idesc = idesc_bf16(kFeat, n16, kAMN);
        const int buf = local % kAccBufs;
        const uint32_t acc_parity = (uint32_t)((local / kAccBufs) & 1);
        const uint32_t d0 = tmem_base + buf * 2 * kNMax;
        if (!mbar_wait(tmem_empty0 + 8 * buf, acc_parity ^ 1, abort_flag, args.status, args.wait_ns)) break;
        tc_fence_after();
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(full0 + 8 * stage, phase, abort_flag, args.status, args.wait_ns)) {
            ok = false;
            break;
          }
          tc_fence_after();
          // gathered B rows arrive through the generic proxy (cp.async)
          if (args.gather_rows) asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
          const uint32_t sa0 = smem_u32(stages + stage * kStageBytes);
          const uint64_t da0 = kAMN ? smem_desc_mn_sw128(sa0) : smem_desc_sw128(sa0);
          const uint64_t da1 = kAMN ? smem_desc_mn_sw128(sa0 + kABytes) : smem_desc_sw128(sa0 + kABytes);
          const uint64_t db = smem_desc_sw128(sa0 + 2 * kABytes);
          // K = 16 step: 32 bytes inside the swizzled K-major row (encoded +2), or
          // 16 K rows = 2048 bytes of the MN-major tile (encoded +128)
          constexpr uint64_t kAStep = kAMN ? 128 : 2;
#pragma unroll
          for (int k = 0; k < kBK / 16; ++k) {
            const uint32_t acc = ((kb - kb0) | k) != 0;
            umma_bf16(d0, da0 + kAStep * k, db + 2 * k, idesc, acc);
            if (!args.single_half) umma_bf16(d0 + kNMax, da1 + kAStep * k, db + 2 * k, idesc, acc);
          }
          umma_commit(empty0 + 8 * stage);
          ++consumed;
          *consumed_sh = consumed;
          if (++stage == kStages) { stage = 0; phase ^= 1; }
        }
        if (ok) umma_commit(tmem_full0 + 8 * buf);
      }
      // every MMA issued so far completes before TMEM is released
      umma_commit(drain_bar);
      mbar_wait(drain_bar, 0, abort_flag, args.status, kDrainTimeoutNs, false);
    }
    __syncwarp();
  } else {
    // ---------------- epilogue (warps 2..5) ----------------
    const int q = warp & 3;                      // TMEM lane quarter this warp may access
    uint32_t* stg = staging + (warp - 2) * (kStagingBytes / kEpiWarps / 4);
    const uint32_t lane_base = (uint32_t)(32 * q) << 16;
    int local = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x, ++local) {
      int sp, kb0, kb1;
      const Tile t = tile_of(tile, sp, kb0, kb1);
      const int buf = local % kAccBufs;
      const uint32_t acc_parity = (uint32_t)((local / kAccBufs) & 1);
      const uint32_t dbase = tmem_base + lane_base + buf * 2 * kNMax;
      if (!mbar_wait(tmem_full0 + 8 * buf, acc_parity, abort_flag, args.status, args.wait_ns)) break;
      tc_fence_after();
      if constexpr (kMode == kSwigluBwd) {
        // D0 | D1 = dh of features f0.. / f0+128..; a, u from au; da | du to out.
        // dh is transposed through shared memory in fp32, 16 token rows per
        // round; the a, u loads of round r+1 are issued before round r is
        // computed (the producer prefetched the tile's a, u rows into L2).
        const __nv_bfloat16* au = static_cast<const __nv_bfloat16*>(args.au);
        __nv_bfloat16* dau = static_cast<__nv_bfloat16*>(args.out);
        const size_t ld = 2 * (size_t)args.n_out;
        const int nr16 = (t.n + 15) >> 4;  // rounds per accumulator half
        const int nrounds = 2 * nr16;
        auto load_round = [&](int r, uint2 (&ar)[4], uint2 (&ur)[4]) {
          const int hf = r >= nr16 ? 1 : 0;
          const int jr = (r - hf * nr16) << 4;
#pragma unroll
          for (int it = 0; it < 4; ++it) {
            const int vec = it * 32 + lane;
            const int j = vec >> 3, c = vec & 7;
            const int f = t.f0 + hf * kFeat + 32 * q + c * 4;
            ar[it] = ur[it] = make_uint2(0, 0);
            if (jr + j < t.n && f < args.n_out) {
              const size_t row = (size_t)(t.r0 + jr + j);
              ar[it] = __ldg(reinterpret_cast<const uint2*>(au + row * ld + f));
              ur[it] = __ldg(reinterpret_cast<const uint2*>(au + row * ld + args.n_out + f));
            }
          }
        };
        uint2 ca[4], cu[4], na[4], nu[4];
        uint32_t v0[32];
        if (nrounds > 0) load_round(0, ca, cu);
        for (int r = 0; r < nrounds; ++r) {
          const int hf = r >= nr16 ? 1 : 0;
          const int jr = (r - hf * nr16) << 4;
          if ((jr & 31) == 0) {
            tmem_ld_32x32b_x32(dbase + hf * kNMax + jr, v0);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 16; ++j) stg[j * kStagingPitch + lane] = v0[j];
          } else {
#pragma unroll
            for (int j = 0; j < 16; ++j) stg[j * kStagingPitch + lane] = v0[16 + j];
          }
          __syncwarp();
          if (r + 1 < nrounds) load_round(r + 1, na, nu);
          float g[4][4];
#pragma unroll
          for (int it = 0; it < 4; ++it) {
            const int vec = it * 32 + lane;
            const int j = vec >> 3, c = vec & 7;
            const float4 dh = *reinterpret_cast<const float4*>(&stg[j * kStagingPitch + c * 4]);
            g[it][0] = dh.x; g[it][1] = dh.y; g[it][2] = dh.z; g[it][3] = dh.w;
          }
          __syncwarp();
#pragma unroll
          for (int it = 0; it < 4; ++it) {
            const int vec = it * 32 + lane;
            const int j = vec >> 3, c = vec & 7;
            const int f = t.f0 + hf * kFeat + 32 * q + c * 4;
            if (jr + j < t.n && f < args.n_out) {
              const size_t row = (size_t)(t.r0 + jr + j);
              const float a[4] = {bf16_lo(ca[it].x), bf16_hi(ca[it].x), bf16_lo(ca[it].y),
                                  bf16_hi(ca[it].y)};
              const float u[4] = {bf16_lo(cu[it].x), bf16_hi(cu[it].x), bf16_lo(cu[it].y),
                                  bf16_hi(cu[it].y)};
              float da[4], du[4];
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const float sg = sigmoid_fast(a[i]);
                da[i] = g[it][i] * u[i] * sg * (1.0f + a[i] * (1.0f - sg));
                du[i] = g[it][i] * a[i] * sg;
              }
              *reinterpret_cast<uint2*>(dau + row * ld + f) =
                  make_uint2(pack_bf16x2(da[0], da[1]), pack_bf16x2(da[2], da[3]));
              *reinterpret_cast<uint2*>(dau + row * ld + args.n_out + f) =
                  make_uint2(pack_bf16x2(du[0], du[1]), pack_bf16x2(du[2], du[3]));
            }
          }
#pragma unroll
          for (int it = 0; it < 4; ++it) {
            ca[it] = na[it];
            cu[it] = nu[it];
          }
        }
      } else if constexpr (kMode == kGatedSave) {
        // h = SiLU(a) * u as in kGated, plus a and u themselves (bf16)
        const int fbase = t.f0 + 32 * q;
        uint16_t* s16 = reinterpret_cast<uint16_t*>(stg);
        __nv_bfloat16* hout = static_cast<__nv_bfloat16*>(args.out);
        __nv_bfloat16* aux = static_cast<__nv_bfloat16*>(args.aux_out);
        const size_t lda = 2 * (size_t)args.n_out;
        for (int j0 = 0; j0 < t.n; j0 += 32) {
          uint32_t v0[32], v1[32];
          tmem_ld_32x32b_x32(dbase + j0, v0);
          tmem_ld_32x32b_x32(dbase + kNMax + j0, v1);
          tmem_wait_ld();
          uint32_t hp[16], ap[16], up[16];
#pragma unroll
          for (int j = 0; j < 32; j += 2) {
            const float a0 = __uint_as_float(v0[j]), a1 = __uint_as_float(v0[j + 1]);
            const float u0 = __uint_as_float(v1[j]), u1 = __uint_as_float(v1[j + 1]);
            hp[j >> 1] = pack_bf16x2(silu_fast(a0) * u0, silu_fast(a1) * u1);
            ap[j >> 1] = pack_bf16x2(a0, a1);
            up[j >> 1] = pack_bf16x2(u0, u1);
          }
          const int row0 = t.r0 + j0, nrows = t.n - j0;
          stage_store_bf16x32(hp, s16, lane, hout, args.n_out, row0, nrows, fbase, args.n_out);
          stage_store_bf16x32(ap, s16, lane, aux, lda, row0, nrows, fbase, args.n_out);
          stage_store_bf16x32(up, s16, lane, aux + args.n_out, lda, row0, nrows, fbase,
                              args.n_out);
        }
      } else {
      const int nhalves = (kMode == kGated || args.single_half) ? 1 : 2;
      for (int hf = 0; hf < nhalves; ++hf) {
        const int fbase = t.f0 + hf * kFeat + 32 * q;   // first feature of this warp
        for (int j0 = 0; j0 < t.n; j0 += 32) {
          uint32_t v0[32];
          tmem_ld_32x32b_x32(dbase + hf * kNMax + j0, v0);
          if (kMode == kGated) {
            uint32_t v1[32];
            tmem_ld_32x32b_x32(dbase + kNMax + j0, v1);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 32; j += 2) {
              float a0 = silu_fast(__uint_as_float(v0[j])) * __uint_as_float(v1[j]);
              float a1 = silu_fast(__uint_as_float(v0[j + 1])) * __uint_as_float(v1[j + 1]);
              v0[j] = pack_bf16x2(a0, a1);
            }
          } else {
            tmem_wait_ld();
            if (kMode == kPlainBf16) {
#pragma unroll
              for (int j = 0; j < 32; j += 2)
                v0[j] = pack_bf16x2(__uint_as_float(v0[j]), __uint_as_float(v0[j + 1]));
            }
          }
          if constexpr (kMode == kPlainF32 && Cfg::kDirectF32) {
            // fp32 rows need no transpose: lane = feature, register j = token, so
            // each store writes 32 consecutive floats (128 bytes) of one row
            const int f = fbase + lane;
            if (f < args.n_out) {
              float* o = static_cast<float*>(args.out) + sp * args.split_stride + f;
              const bool add = args.add && sp == 0;
#pragma unroll
              for (int j = 0; j < 32; ++j) {
                if (j0 + j < t.n) {
                  const size_t row = (size_t)(t.r0 + j0 + j) * args.n_out;
                  float v = __uint_as_float(v0[j]);
                  if (add) v += args.add[row + f];
                  o[row] = v;
                }
              }
            }
            continue;
          }
          // transpose through shared memory: stg[token j][feature lane]
          if (kMode == kPlainF32) {
#pragma unroll
            for (int j = 0; j < 32; ++j) stg[j * kStagingPitch + lane] = v0[j];
          } else {
            uint16_t* s16 = reinterpret_cast<uint16_t*>(stg);
#pragma unroll
            for (int j = 0; j < 32; j += 2) {
              s16[j * kStagingPitch16 + lane] = (uint16_t)(v0[j] & 0xffffu);
              s16[(j + 1) * kStagingPitch16 + lane] = (uint16_t)(v0[j] >> 16);
            }
          }
          __syncwarp();
          // each token row of this warp: 32 features = 64 B (bf16) or 128 B (fp32)
          constexpr int kVecPerRow = (kMode == kPlainF32) ? 8 : 4;
#pragma unroll
          for (int it = 0; it < kVecPerRow; ++it) {
            const int vec = it * 32 + lane;
            const int j = vec / kVecPerRow, c = vec % kVecPerRow;
            const int row = t.r0 + j0 + j;
            const int f = fbase + c * (kMode == kPlainF32 ? 4 : 8);
            if (j0 + j < t.n && f < args.n_out) {
              if (kMode == kPlainF32) {
                uint4 w = *reinterpret_cast<const uint4*>(&stg[j * kStagingPitch + c * 4]);
                float* o = static_cast<float*>(args.out) + sp * args.split_stride +
                           (size_t)row * args.n_out + f;
                if (args.add && sp == 0) {
                  const float4 ad =
                      *reinterpret_cast<const float4*>(args.add + (size_t)row * args.n_out + f);
                  w.x = __float_as_uint(__uint_as_float(w.x) + ad.x);
                  w.y = __float_as_uint(__uint_as_float(w.y) + ad.y);
                  w.z = __float_as_uint(__uint_as_float(w.z) + ad.z);
                  w.w = __float_as_uint(__uint_as_float(w.w) + ad.w);
                }
                *reinterpret_cast<uint4*>(o) = w;
              } else {
                const uint16_t* s16 = reinterpret_cast<const uint16_t*>(stg);
                const uint4 w = *reinterpret_cast<const uint4*>(&s16[j * kStagingPitch16 + c * 8]);
                __nv_bfloat16* o =
                    static_cast<__nv_bfloat16*>(args.out) + (size_t)row * args.n_out + f;
                *reinterpret_cast<uint4*>(o) = w;
              }
            }
          }
          __syncwarp();
        }
      }
      }
      tc_fence_before();
      mbar_arrive(tmem_empty0 + 8 * buf);
    }
  }

  __syncthreads();
  if (threadIdx.x == 0 && *abort_flag) {
    // drain copies still in flight into shared memory (bounded)
    const int consumed = *consumed_sh;
    for (int i = consumed; i < issued; ++i)
      mbar_wait(full0 + 8 * (i % kStages), (uint32_t)((i / kStages) & 1), abort_flag,
                args.status, kDrainTimeoutNs, false);
  }
  __syncwarp();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "r"(kTmemCols)
                 : "memory");
  }
}

// --- host side -------------------------------------------------------------------
inline bool router_supported(const moe_shape& s) {
  const int E = s.N + s.Z;
  return s.dtype == MOE_BF16 && s.d % kBK == 0 && E % 8 == 0;
}
inline bool ffn_supported(const moe_shape& s) {
  return s.dtype == MOE_BF16 && s.d % kBK == 0 && s.I % kBK == 0;
}

inline PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// 2-D bf16 row-major [rows, cols] view, box = box_rows x 64 columns, 128-byte swizzle.
inline bool make_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols,
                     uint32_t box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {(cuuint32_t)kBK, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int kMode, class Cfg, bool kAMN = false>
static inline moe_status launch(const CUtensorMap& a0, const CUtensorMap& a1, const CUtensorMap& b,
                         const Args& args, long long max_tiles, int sms, cudaStream_t st,
                         char* err, size_t errn) {
  static bool attr_set[64] = {};  // per device; internal linkage (one per loaded library)
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(gemm_tc_kernel<kMode, Cfg, kAMN>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         Cfg::smem_bytes(staging_bytes<kMode, Cfg>()));
    if (e != cudaSuccess) {
      snprintf(err, errn, "tcgen05 gemm smem attribute: %s", cudaGetErrorString(e));
      return MOE_ERR_CUDA;
    }
    attr_set[dev] = true;
  }
  static_assert(Cfg::smem_bytes(staging_bytes<kMode, Cfg>()) <= 232448, "shared memory");
  if (args.seg_offsets && Cfg::kPrefixInts < kMaxExperts + 1 + 33) {
    snprintf(err, errn, "tcgen05 gemm: tile config without a segment table given segments");
    return MOE_ERR_INVALID_ARG;
  }
  long long grid = max_tiles < sms ? max_tiles : sms;
  if (grid < 1) grid = 1;
  Args la = args;
  la.wait_ns = pipeline_wait_ns();
  la.stall_fill = pipeline_debug().stall_fill.load(std::memory_order_relaxed);
  launch_pdl(gemm_tc_kernel<kMode, Cfg, kAMN>, dim3((unsigned)grid), dim3(kThreads),
             (size_t)Cfg::smem_bytes(staging_bytes<kMode, Cfg>()), st, a0, a1, b, la);
  note_launch();
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    snprintf(err, errn, "tcgen05 gemm launch: %s", cudaGetErrorString(e));
    return MOE_ERR_CUDA;
  }
  return MOE_OK;
}

// Map of n_mats weight matrices [rows, cols]: row-major, or the tiled order
// seen as [n_mats*rows*cols/64, 64] (each 128 x 64 tile = 128 consecutive rows).
inline bool make_weight_map(CUtensorMap* m, const void* base, uint64_t n_mats, uint64_t rows,
                            uint64_t cols, bool tiled) {
  if (tiled) return make_map(m, base, n_mats * rows * cols / kBK, kBK, kFeat);
  return make_map(m, base, n_mats * rows, cols, kFeat);
}

inline moe_status map_error(char* err, size_t errn, const char* what) {
  snprintf(err, errn, "cuTensorMapEncodeTiled failed for %s", what);
  return MOE_ERR_CUDA;
}

// Upper bound of (row chunk, feature block) tiles for routed rows.
inline long long routed_tiles(const moe_shape& s, int n_out, int feat, int nmax) {
  const long long rows = (long long)s.T * s.K;
  const long long chunks = s.N + (rows + nmax - 1) / nmax;
  return chunks * ((n_out + feat - 1) / feat);
}

// Expert GEMM geometry.  A segment longer than the tile is split into chunks
// and each chunk streams the expert's weights again, so the tile must hold
// nearly every segment.  With uniform routing the rows per FFN expert have
// mean T*K/(N+Z); up to a mean of 128 (LongCat: exactly 128, spread ~11)
// the 160-row tile with four stages keeps more weight bytes in flight;
// longer segments use the 256-row tile with three stages.
constexpr int kDoubleBufferMaxMeanRows = 0;  // mean rows at or below which CfgDouble is used
constexpr int kN160MaxMeanRows = 128;
// mean rows per expert at or below which CfgN64 is used (decode: at 24 the
// largest expert rarely passes 64 rows; a longer segment takes several tiles)
constexpr int kN64MaxMeanRows = 24;
inline bool use_double(const moe_shape& s) {
  return (long long)s.T * s.K <= (long long)kDoubleBufferMaxMeanRows * (s.N + s.Z);
}
// L2 budget of the speculative weight prefetch of all CTAs together: K blocks
// per CTA so that sms tiles' A0 + A1 boxes take at most this many bytes.
#ifndef MOE_SPEC_PREFETCH_MB
#define MOE_SPEC_PREFETCH_MB 96
#endif
#ifndef MOE_SPEC_DOWN
#define MOE_SPEC_DOWN 1
#endif
// 96 MB of the 126 MB L2; measured at decode T = 64 / 256 against 32 and 64 MB,
// and against no prefetch for the down GEMM
constexpr long long kSpecPrefetchBytes = (long long)MOE_SPEC_PREFETCH_MB << 20;
// The guess needs nearly every expert touched: at least this many routed slots
// per expert on average (below it, untouched experts shift the tile order).
constexpr int kSpecMinMeanRows = 2;
inline int spec_prefetch_kb(const moe_shape& s, int sms, int k_dim) {
  if ((long long)s.T * s.K < (long long)kSpecMinMeanRows * (s.N + s.Z)) return 0;
  const long long per_kb = (long long)sms * 2 * kABytes;
  return (int)std::min<long long>(k_dim / kBK, kSpecPrefetchBytes / per_kb);
}
inline bool use_n64(const moe_shape& s) {
  return (long long)s.T * s.K <= (long long)kN64MaxMeanRows * (s.N + s.Z);
}
inline bool use_n160(const moe_shape& s) {
  return (long long)s.T * s.K <= (long long)kN160MaxMeanRows * (s.N + s.Z);
}

inline moe_status launch_gate_up(const moe_shape& s, const void* x_perm, const void* w1,
                                 const void* w3, const int32_t* offsets, void* h,
                                 uint32_t* status, int sms, cudaStream_t st, char* err,
                                 size_t errn) {
  CUtensorMap a0, a1, b;
  const uint64_t rows = (uint64_t)s.T * s.K;
  const bool tiled = s.weight_layout == MOE_WEIGHTS_TILED;
  if (!make_weight_map(&a0, w1, s.N, s.I, s.d, tiled)) return map_error(err, errn, "w1");
  if (!make_weight_map(&a1, w3, s.N, s.I, s.d, tiled)) return map_error(err, errn, "w3");
  if (!make_map(&b, x_perm, rows, s.d, kBoxRows)) return map_error(err, errn, "x_perm");
  Args a{};
  a.seg_offsets = offsets;
  a.nseg = s.N;
  a.max_rows = (int)rows;
  a.n_out = s.I;
  a.k_dim = s.d;
  a.a_seg_rows = s.I;
  a.a1_row_off = 0;
  a.feat_per_tile = kFeat;
  a.out = h;
  a.status = status;
  a.a_tiled = tiled;
  if (use_double(s))
    return launch<kGated, CfgDouble>(a0, a1, b, a, routed_tiles(s, s.I, kFeat, CfgDouble::kNMax),
                                     sms, st, err, errn);
  if (use_n64(s)) {
    a.spec_prefetch_kb = spec_prefetch_kb(s, sms, s.d);
    return launch<kGated, CfgN64>(a0, a1, b, a, routed_tiles(s, s.I, kFeat, CfgN64::kNMax),
                                  sms, st, err, errn);
  }
  if (use_n160(s))
    return launch<kGated, CfgN160>(a0, a1, b, a, routed_tiles(s, s.I, kFeat, CfgN160::kNMax),
                                   sms, st, err, errn);
  return launch<kGated, CfgWide>(a0, a1, b, a, routed_tiles(s, s.I, kFeat, CfgWide::kNMax), sms,
                                 st, err, errn);
}

// Gate/up GEMM reading its token rows straight from x through row_token
// (cp.async row copies by the producer lanes), so the dispatch needs no
// x_perm copy.
inline moe_status launch_gate_up_gather(const moe_shape& s, const void* x,
                                        const int32_t* row_token, const void* w1,
                                        const void* w3, const int32_t* offsets, void* h,
                                        uint32_t* status, int sms, cudaStream_t st, char* err,
                                        size_t errn) {
  CUtensorMap a0, a1, b;
  const uint64_t rows = (uint64_t)s.T * s.K;
  const bool tiled = s.weight_layout == MOE_WEIGHTS_TILED;
  if (!make_weight_map(&a0, w1, s.N, s.I, s.d, tiled)) return map_error(err, errn, "w1");
  if (!make_weight_map(&a1, w3, s.N, s.I, s.d, tiled)) return map_error(err, errn, "w3");
  if (!make_map(&b, x, (uint64_t)s.T, s.d, kBoxRows)) return map_error(err, errn, "x");
  Args a{};
  a.seg_offsets = offsets;
  a.nseg = s.N;
  a.max_rows = (int)rows;
  a.n_out = s.I;
  a.k_dim = s.d;
  a.a_seg_rows = s.I;
  a.a1_row_off = 0;
  a.feat_per_tile = kFeat;
  a.out = h;
  a.status = status;
  a.gather_rows = row_token;
  a.gather_src_rows = s.T;
  a.gather_src = x;
  a.a_tiled = tiled;
  if (use_double(s))
    return launch<kGated, CfgDouble>(a0, a1, b, a, routed_tiles(s, s.I, kFeat, CfgDouble::kNMax),
                                     sms, st, err, errn);
  if (use_n64(s)) {
    a.spec_prefetch_kb = spec_prefetch_kb(s, sms, s.d);
    return launch<kGated, CfgN64>(a0, a1, b, a, routed_tiles(s, s.I, kFeat, CfgN64::kNMax),
                                  sms, st, err, errn);
  }
  if (use_n160(s))
    return launch<kGated, CfgN160>(a0, a1, b, a, routed_tiles(s, s.I, kFeat, CfgN160::kNMax),
                                   sms, st, err, errn);
  return launch<kGated, CfgWide>(a0, a1, b, a, routed_tiles(s, s.I, kFeat, CfgWide::kNMax), sms,
                                 st, err, errn);
}

inline moe_status launch_down(const moe_shape& s, const void* h, const void* w2,
                              const int32_t* offsets, void* y_perm, uint32_t* status, int sms,
                              cudaStream_t st, char* err, size_t errn) {
  CUtensorMap a, b;
  const uint64_t rows = (uint64_t)s.T * s.K;
  const bool tiled = s.weight_layout == MOE_WEIGHTS_TILED;
  if (!make_weight_map(&a, w2, s.N, s.d, s.I, tiled)) return map_error(err, errn, "w2");
  if (!make_map(&b, h, rows, s.I, kBoxRows)) return map_error(err, errn, "h");
  Args g{};
  g.seg_offsets = offsets;
  g.nseg = s.N;
  g.max_rows = (int)rows;
  g.n_out = s.d;
  g.k_dim = s.I;
  g.a_seg_rows = s.d;
  g.a1_row_off = kFeat;
  g.feat_per_tile = 2 * kFeat;
  g.out = y_perm;
  g.status = status;
  g.a_tiled = tiled;
  if (use_double(s))
    return launch<kPlainBf16, CfgDouble>(a, a, b, g,
                                         routed_tiles(s, s.d, 2 * kFeat, CfgDouble::kNMax), sms,
                                         st, err, errn);
  if (use_n64(s)) {
    g.spec_prefetch_kb = MOE_SPEC_DOWN ? spec_prefetch_kb(s, sms, s.I) : 0;
    return launch<kPlainBf16, CfgN64>(a, a, b, g, routed_tiles(s, s.d, 2 * kFeat, CfgN64::kNMax),
                                      sms, st, err, errn);
  }
  if (use_n160(s))
    return launch<kPlainBf16, CfgN160>(a, a, b, g,
                                       routed_tiles(s, s.d, 2 * kFeat, CfgN160::kNMax), sms, st,
                                       err, errn);
  return launch<kPlainBf16, CfgWide>(a, a, b, g, routed_tiles(s, s.d, 2 * kFeat, CfgWide::kNMax),
                                     sms, st, err, errn);
}

// K splits of the router GEMM for a shape.  A small batch has few
// (256-token, 256-expert) tiles, so each would walk all d/64 K blocks on one SM;
// splitting K spreads it over ~128 CTAs, and the top-K kernel sums the fp32
// partial logits in split order.  The count depends on the shape only (it sizes
// the workspace): 1 at the LongCat prefill shape.
inline int router_splits(const moe_shape& s) {
  const int E = s.N + s.Z;
  const long long tiles = (long long)((s.T + 255) / 256) * ((E + 255) / 256);
  long long sp = tiles > 0 ? 128 / tiles : 1;
  const int nk = s.d / kBK;
  if (sp > 32) sp = 32;
  if (sp > nk) sp = nk;
  if (sp < 1) sp = 1;
  return (int)sp;
}

inline moe_status launch_router_gemm(const moe_shape& s, const void* x, const void* w,
                                     const float* offset, float* logits, int32_t* counts,
                                     int sms, cudaStream_t st, char* err, size_t errn) {
  CUtensorMap a, b;
  const int E = s.N + s.Z;
  if (!make_map(&a, w, (uint64_t)E, s.d, kFeat)) return map_error(err, errn, "w_router");
  if (!make_map(&b, x, (uint64_t)s.T, s.d, kBoxRows)) return map_error(err, errn, "x");
  Args g{};
  g.seg_offsets = nullptr;
  g.nseg = 1;
  g.single_rows = s.T;
  g.max_rows = s.T;
  g.n_out = E;
  g.k_dim = s.d;
  g.a_seg_rows = 0;
  g.a1_row_off = kFeat;
  g.feat_per_tile = 2 * kFeat;
  g.out = logits;
  g.add = offset;
  g.status = nullptr;
  g.zero_i32 = counts;  // the selection kernel adds its histograms into them
  g.zero_n = E;
  g.prefetch_b = 0;
  if (E <= kFeat) {
    // at most 128 experts: one accumulator, the second weight half neither loaded nor computed
    g.feat_per_tile = kFeat;
    g.single_half = 1;
  }
  const long long fblk = (E + g.feat_per_tile - 1) / g.feat_per_tile;
  const int splits = router_splits(s);
  if (splits > 1) {
    g.k_splits = splits;
    g.split_stride = (long long)s.T * E;
    return launch<kPlainF32, CfgWide>(a, a, b, g, (long long)((s.T + 255) / 256) * fblk * splits,
                                      sms, st, err, errn);
  }
  // The router is one dense GEMM: pick the token tile so that all tiles run
  // in one wave when 256-row tiles would leave SMs idle.
  const long long tiles256 = (long long)((s.T + 255) / 256) * fblk;
  const long long tiles192 = (long long)((s.T + 191) / 192) * fblk;
  if (tiles256 < sms && tiles192 <= sms)
    return launch<kPlainF32, CfgR192>(a, a, b, g, tiles192, sms, st, err, errn);
  return launch<kPlainF32, CfgWide>(a, a, b, g, tiles256, sms, st, err, errn);
}

// Forward gate/up for training: h as launch_gate_up, and a | u to au [rows, 2I].
inline moe_status launch_gate_up_save(const moe_shape& s, const void* x_perm, const void* w1,
                                      const void* w3, const int32_t* offsets, void* h, void* au,
                                      uint32_t* status, int sms, cudaStream_t st, char* err,
                                      size_t errn) {
  CUtensorMap a0, a1, b;
  const uint64_t rows = (uint64_t)s.T * s.K;
  const bool tiled = s.weight_layout == MOE_WEIGHTS_TILED;
  if (!make_weight_map(&a0, w1, s.N, s.I, s.d, tiled)) return map_error(err, errn, "w1");
  if (!make_weight_map(&a1, w3, s.N, s.I, s.d, tiled)) return map_error(err, errn, "w3");
  if (!make_map(&b, x_perm, rows, s.d, kBoxRows)) return map_error(err, errn, "x_perm");
  Args a{};
  a.seg_offsets = offsets;
  a.nseg = s.N;
  a.max_rows = (int)rows;
  a.n_out = s.I;
  a.k_dim = s.d;
  a.a_seg_rows = s.I;
  a.feat_per_tile = kFeat;
  a.out = h;
  a.aux_out = au;
  a.status = status;
  a.a_tiled = tiled;
  if (use_n160(s))
    return launch<kGatedSave, CfgN160>(a0, a1, b, a, routed_tiles(s, s.I, kFeat, CfgN160::kNMax),
                                       sms, st, err, errn);
  return launch<kGatedSave, CfgWide>(a0, a1, b, a, routed_tiles(s, s.I, kFeat, CfgWide::kNMax),
                                     sms, st, err, errn);
}

// MN-major view of n_mats weight matrices [rows, cols] for 64 x 64 boxes:
// row-major [n_mats*rows, cols], or the tiled order seen as [n_mats*rows*cols/64, 64].
inline bool make_weight_map_mn(CUtensorMap* m, const void* base, uint64_t n_mats, uint64_t rows,
                               uint64_t cols, bool tiled) {
  if (tiled) return make_map(m, base, n_mats * rows * cols / kBK, kBK, 64);
  return make_map(m, base, n_mats * rows, cols, 64);
}

// Backward through the down projection and the SwiGLU:
//   dh = dy_perm W2_e (reduction over d; W2_e [d, I] read MN-major), then
//   da = dh u SiLU'(a), du = dh SiLU(a) written to dau [rows, 2I].
inline moe_status launch_dgrad_h(const moe_shape& s, const void* dy, const void* w2,
                                 const int32_t* offsets, const void* au, void* dau,
                                 uint32_t* status, int sms, cudaStream_t st, char* err,
                                 size_t errn) {
  CUtensorMap a, b;
  const uint64_t rows = (uint64_t)s.T * s.K;
  const bool tiled = s.weight_layout == MOE_WEIGHTS_TILED;
  if (!make_weight_map_mn(&a, w2, s.N, s.d, s.I, tiled)) return map_error(err, errn, "w2");
  if (!make_map(&b, dy, rows, s.d, kBoxRows)) return map_error(err, errn, "dy_perm");
  Args g{};
  g.seg_offsets = offsets;
  g.nseg = s.N;
  g.max_rows = (int)rows;
  g.n_out = s.I;
  g.k_dim = s.d;
  g.a_seg_rows = s.d;
  g.a1_row_off = kFeat;
  g.feat_per_tile = 2 * kFeat;
  g.out = dau;
  g.au = au;
  g.status = status;
  g.a_tiled = tiled;
  if (use_n160(s))
    return launch<kSwigluBwd, CfgN160, true>(a, a, b, g,
                                             routed_tiles(s, s.I, 2 * kFeat, CfgN160::kNMax),
                                             sms, st, err, errn);
  return launch<kSwigluBwd, CfgWide, true>(a, a, b, g,
                                           routed_tiles(s, s.I, 2 * kFeat, CfgWide::kNMax), sms,
                                           st, err, errn);
}

// dx_perm = da W1_e + du W3_e: one reduction over 2I (K blocks of W1, then of
// W3), W1_e / W3_e [I, d] read MN-major, dau [rows, 2I] the token operand.
inline moe_status launch_dgrad_x(const moe_shape& s, const void* dau, const void* w1,
                                 const void* w3, const int32_t* offsets, void* dx_perm,
                                 uint32_t* status, int sms, cudaStream_t st, char* err,
                                 size_t errn) {
  CUtensorMap a0, a1, b;
  const uint64_t rows = (uint64_t)s.T * s.K;
  const bool tiled = s.weight_layout == MOE_WEIGHTS_TILED;
  if (!make_weight_map_mn(&a0, w1, s.N, s.I, s.d, tiled)) return map_error(err, errn, "w1");
  if (!make_weight_map_mn(&a1, w3, s.N, s.I, s.d, tiled)) return map_error(err, errn, "w3");
  if (!make_map(&b, dau, rows, 2 * (uint64_t)s.I, kBoxRows)) return map_error(err, errn, "dau");
  Args g{};
  g.seg_offsets = offsets;
  g.nseg = s.N;
  g.max_rows = (int)rows;
  g.n_out = s.d;
  g.k_dim = 2 * s.I;
  g.a_seg_rows = s.I;
  g.a_k_split = s.I / kBK;
  g.a1_row_off = kFeat;
  g.feat_per_tile = 2 * kFeat;
  g.out = dx_perm;
  g.status = status;
  g.a_tiled = tiled;
  if (use_n160(s))
    return launch<kPlainBf16, CfgN160, true>(a0, a1, b, g,
                                             routed_tiles(s, s.d, 2 * kFeat, CfgN160::kNMax),
                                             sms, st, err, errn);
  return launch<kPlainBf16, CfgWide, true>(a0, a1, b, g,
                                           routed_tiles(s, s.d, 2 * kFeat, CfgWide::kNMax), sms,
                                           st, err, errn);
}

// dx_router = dlogits W_r [T, d] fp32: reduction over the E experts (W_r [E, d]
// read MN-major, the K tail past E zero-filled by TMA).
inline moe_status launch_router_dx(const moe_shape& s, const void* dlogits, const void* w,
                                   float* dx_router, uint32_t* status, int sms, cudaStream_t st,
                                   char* err, size_t errn) {
  CUtensorMap a, b;
  const int E = s.N + s.Z;
  if (!make_map(&a, w, (uint64_t)E, s.d, 64)) return map_error(err, errn, "w_router");
  if (!make_map(&b, dlogits, (uint64_t)s.T, E, kBoxRows)) return map_error(err, errn, "dlogits");
  Args g{};
  g.seg_offsets = nullptr;
  g.nseg = 1;
  g.single_rows = s.T;
  g.max_rows = s.T;
  g.n_out = s.d;
  g.k_dim = (E + kBK - 1) / kBK * kBK;
  g.a_seg_rows = 0;
  g.a1_row_off = kFeat;
  g.feat_per_tile = 2 * kFeat;
  g.out = dx_router;
  g.status = status;
  const long long tiles = (long long)((s.T + 255) / 256) * ((s.d + 2 * kFeat - 1) / (2 * kFeat));
  return launch<kPlainF32, CfgWide, true>(a, a, b, g, tiles, sms, st, err, errn);
}

// Tensor-core backward needs whole 128-feature tiles on both expert axes.
inline bool bwd_supported(const moe_shape& s) {
  return s.dtype == MOE_BF16 && s.d % 128 == 0 && s.I % 128 == 0;
}

}  // namespace tc
}  // namespace moe
