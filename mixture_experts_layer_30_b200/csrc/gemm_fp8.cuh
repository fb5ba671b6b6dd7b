// MXFP8 expert GEMMs on sm_100a: tcgen05.mma kind::mxf8f6f4 with hardware
// block scaling (one UE8M0 scale per 32 K values of every row of A and B).
//
// Same structure as the bf16 kernel (gemm_tc.cuh): swap-AB, weight rows on
// UMMA M = 128, routed token rows on N (rounded up to 32 here, <= 160), one
// persistent CTA per SM, warp 0 producer, warp 1 MMA issuer, warps 2-5
// epilogue, 4 shared-memory stages of 128 K values (128-byte swizzled rows).
// Per stage the scales travel beside the operands:
//   SFA0, SFA1 -- the two weight tiles' 512-byte scale atoms (bulk copies);
//   SFB        -- the token rows' scales, gathered 4 bytes per row by the
//                 producer lanes (cp.async) into the same 32-lane x 16-byte
//                 image;
// and the MMA warp moves each image into tensor memory with
// tcgen05.cp.32x128b.warpx4 (row m -> lane m % 32 of every sub-partition,
// column m / 32, byte = K step) before issuing the stage's MMAs.
#pragma once

#include "gemm_tc.cuh"
#include "quant.cuh"

namespace moe {
namespace f8 {

using namespace moe::tc;

constexpr int kNMax = 160;                       // token rows per tile
constexpr int kStages = 4;
constexpr int kBKf = 128;                        // K values (bytes) per stage row
constexpr int kBBytes = kNMax * kBKf;            // 20 KiB
constexpr int kSfBytes = 2048;                   // SFA0 | SFA1 | SFB (two 512-byte images)
constexpr int kStageBytes = 2 * kABytes + kBBytes + kSfBytes;
constexpr int kAccCols = 2 * kNMax;              // D0, D1
constexpr int kSfCols = 16;                      // per stage: SFA0 4, SFA1 4, SFB 8
constexpr int kNumBars = 2 * kStages + 3;
constexpr int kPitchH = 32;                      // fp8 h staging row: 32 bytes
constexpr int kPitchY = 32;                      // bf16 y staging row: 32 halves (64 B, 16-B aligned)
template <bool kGatedOut> __host__ __device__ constexpr int staging() {
  // bf16 y is staged 16 tokens at a time to keep four stages in shared memory
  return kGatedOut ? kEpiWarps * 32 * kPitchH : kEpiWarps * 16 * kPitchY * 2;
}
template <bool kGatedOut> __host__ __device__ constexpr int smem_bytes() {
  return 1024 + kStages * kStageBytes + staging<kGatedOut>() + kCtrlBytes +
         (kMaxExperts + 1 + 33) * 4;
}
static_assert(kStageBytes % 1024 == 0, "stage alignment");
static_assert(smem_bytes<false>() <= 232448 && smem_bytes<true>() <= 232448, "shared memory");
static_assert(kAccCols + kStages * kSfCols <= 512, "tensor memory");

struct ArgsF8 {
  const int32_t* seg_offsets;  // [nseg+1] routed-row offsets
  int nseg;
  int max_rows;
  int n_out;                   // output features
  int k_dim;                   // reduction length (multiple of 128)
  int a_seg_rows;              // weight rows per expert
  int a1_row_off;              // 0 (gated: second weight matrix) or 128 (next row block)
  int feat_per_tile;           // 128 (gated) or 256 (plain)
  const uint8_t* sfa0;         // scale atoms of the first / second weight map
  const uint8_t* sfa1;
  const uint8_t* sfb;          // token-row scales, [rows, k_dim / 32] bytes
  void* out;                   // gated: h E4M3 [rows, n_out]; plain: y bf16 [rows, n_out]
  uint8_t* out_sf;             // gated: h scales [rows, n_out / 32]
  uint32_t* status;
  unsigned long long wait_ns;  // time limit of one pipeline wait (set at launch)
};

// --- PTX wrappers ----------------------------------------------------------
// Instruction descriptor, kind::mxf8f6f4 with block scaling: E4M3 A and B,
// K-major, UE8M0 scales; sf_id picks the scale byte (K step) in each column.
//   bits 4-5 B scale id, 7-9 A format (0 = E4M3), 10-12 B format, 17-22 N >> 3,
//   23 scale format (1 = UE8M0), 24-28 M >> 4, 29-30 A scale id, 31 K = 32.
MOE_DEV uint32_t idesc_mxf8(int m, int n, uint32_t sf_id) {
  return (sf_id << 4) | ((uint32_t)(n >> 3) << 17) | (1u << 23) | ((uint32_t)(m >> 4) << 24) |
         (sf_id << 29);
}
MOE_DEV void umma_mxf8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                       uint32_t accumulate, uint32_t sfa_tmem, uint32_t sfb_tmem) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
      ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem),
      "r"(sfb_tmem)
      : "memory");
}
// 32 rows x 16 bytes of shared memory -> lanes 0-31 (and copies in lanes
// 32-63, 64-95, 96-127) x 4 columns of tensor memory.
MOE_DEV void tmem_cp_32x128b_warpx4(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc)
               : "memory");
}
// Descriptor of a dense, unswizzled 32-row x 16-byte image: core matrices of
// 8 rows x 16 bytes, 128 bytes apart.
MOE_DEV uint64_t smem_desc_plain(uint32_t addr) {
  uint64_t d = 0;
  d |= (uint64_t)((addr >> 4) & 0x3fff);
  d |= (uint64_t)1 << 16;            // leading byte offset (one core matrix wide: unused)
  d |= (uint64_t)(128 >> 4) << 32;   // stride byte offset: next 8 rows
  d |= (uint64_t)1 << 46;            // version
  return d;                           // layout type 0: no swizzle
}
MOE_DEV void bulk_load_hint(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar,
                            uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1], %2, [%3], %4;" ::"r"(dst),
      "l"(src), "r"(bytes), "r"(bar), "l"(policy)
      : "memory");
}
MOE_DEV void cp_async_4(uint32_t dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}

// --- the kernel --------------------------------------------------------------
template <bool kGatedOut>
__global__ void __launch_bounds__(kThreads, 1)
gemm_mxf8_kernel(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmA1,
                 const __grid_constant__ CUtensorMap tmB, const ArgsF8 args) {
  pdl_trigger();
  constexpr int kStagingBytes = staging<kGatedOut>();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* stages = smem;
  uint8_t* staging_base = smem + kStages * kStageBytes;
  uint8_t* ctrl = staging_base + kStagingBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(ctrl);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(ctrl + 8 * kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(ctrl + 8 * kNumBars + 4);
  volatile int* consumed_sh = reinterpret_cast<volatile int*>(ctrl + 8 * kNumBars + 8);
  int* prefix = reinterpret_cast<int*>(ctrl + kCtrlBytes);
  int* scan_tmp = prefix + kMaxExperts + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t full0 = smem_u32(&bars[0]);
  const uint32_t empty0 = smem_u32(&bars[kStages]);
  const uint32_t tmem_full = smem_u32(&bars[2 * kStages]);
  const uint32_t tmem_empty = smem_u32(&bars[2 * kStages + 1]);
  const uint32_t drain_bar = smem_u32(&bars[2 * kStages + 2]);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(full0 + 8 * s, 1 + 32);  // producer's expect_tx + one cp.async arrive per lane
      mbar_init(empty0 + 8 * s, 1);
    }
    mbar_init(tmem_full, 1);
    mbar_init(tmem_empty, kEpiWarps * 32);
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
                 "r"(512)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  pdl_wait();  // the prologue above touches no global memory
  build_chunk_prefix(args.seg_offsets, args.nseg, args.max_rows, kNMax, prefix, scan_tmp,
                     args.status);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int n_fblk = (args.n_out + args.feat_per_tile - 1) / args.feat_per_tile;
  const int total = prefix[args.nseg] * n_fblk;
  const int nk = args.k_dim / kBKf;
  const int sfb_row = args.k_dim / 32;  // scale bytes per token row
  Args targs{};                          // only the fields decode_tile reads
  targs.seg_offsets = args.seg_offsets;
  targs.nseg = args.nseg;
  targs.feat_per_tile = args.feat_per_tile;
  int issued = 0;

  if (warp == 0) {
    // ---------------- producer: TMA operands + scale images ----------------
    uint32_t stage = 0, phase = 0;
    bool ok = true;
    const uint64_t pol_w = l2_policy_evict_first();
    const uint64_t pol_x = l2_policy_evict_last();
    for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
      const Tile t = decode_tile<kNMax>(tile, n_fblk, targs, prefix);
      const int nbox = (t.n + kBoxRows - 1) / kBoxRows;
      const uint32_t tx = 2 * kABytes + nbox * kBoxBytes + 1024;
      const int a_row0 = t.seg * args.a_seg_rows + t.f0;
      const int a_row1 = a_row0 + args.a1_row_off;
      // this lane's token rows (one per 32-row group; clamped into the segment)
      const uint8_t* sfb_src[kNMax / 32];
#pragma unroll
      for (int c = 0; c < kNMax / 32; ++c)
        sfb_src[c] = args.sfb + (size_t)(t.r0 + min(32 * c + lane, t.n - 1)) * sfb_row;
      const uint8_t* sfb_rot[4];  // row group (i + lane/8) % 4 of copy i
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int c = (i + (lane >> 3)) & 3;
        sfb_rot[i] = args.sfb + (size_t)(t.r0 + min(32 * c + lane, t.n - 1)) * sfb_row;
      }
      for (int kb = 0; kb < nk; ++kb) {
        int go = 1;
        if (lane == 0) go = mbar_wait(empty0 + 8 * stage, phase ^ 1, abort_flag, args.status, args.wait_ns);
        go = __shfl_sync(0xffffffffu, go, 0);
        if (!go) {
          ok = false;
          break;
        }
        const uint32_t fb = full0 + 8 * stage;
        const uint32_t sa0 = smem_u32(stages + stage * kStageBytes);
        const uint32_t sf = sa0 + 2 * kABytes + kBBytes;
        if (lane == 0) {
          const int i0 = (a_row0 >> 7) * nk + kb, i1 = (a_row1 >> 7) * nk + kb;
          mbar_arrive_expect_tx(fb, tx);
          tma_load_2d_hint(sa0, &tmA0, 0, i0 << 7, fb, pol_w);
          tma_load_2d_hint(sa0 + kABytes, &tmA1, 0, i1 << 7, fb, pol_w);
          for (int b = 0; b < nbox; ++b)
            tma_load_2d_hint(sa0 + 2 * kABytes + b * kBoxBytes, &tmB, kb * kBKf,
                             t.r0 + b * kBoxRows, fb, pol_x);
          bulk_load_hint(sf, args.sfa0 + (size_t)i0 * 512, 512, fb, pol_w);
          bulk_load_hint(sf + 512, args.sfa1 + (size_t)i1 * 512, 512, fb, pol_w);
          ++issued;
        }
        // token scales: 4 bytes (the stage's four K steps) per row.  Row groups
        // 0-3 rotate with the lane so the 32 writes of one copy hit 32 banks.
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int c = (i + (lane >> 3)) & 3;
          cp_async_4(sf + 1024 + lane * 16 + c * 4, sfb_rot[i] + 4 * kb);
        }
#pragma unroll
        for (int c = 4; c < kNMax / 32; ++c)
          cp_async_4(sf + 1024 + (c >> 2) * 512 + lane * 16 + (c & 3) * 4, sfb_src[c] + 4 * kb);
        cp_async_arrive_noinc(fb);
        if (++stage == kStages) { stage = 0; phase ^= 1; }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer ----------------
      uint32_t stage = 0, phase = 0, acc_phase = 0;
      bool ok = true;
      int consumed = 0;
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
        const Tile t = decode_tile<kNMax>(tile, n_fblk, targs, prefix);
        const int n32 = ((t.n + 31) >> 5) << 5;
        if (!mbar_wait(tmem_empty, acc_phase ^ 1, abort_flag, args.status, args.wait_ns)) break;
        acc_phase ^= 1;
        tc_fence_after();
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(full0 + 8 * stage, phase, abort_flag, args.status, args.wait_ns)) {
            ok = false;
            break;
          }
          tc_fence_after();
          // the token scales arrived through the generic proxy (cp.async)
          asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
          const uint32_t sa0 = smem_u32(stages + stage * kStageBytes);
          const uint32_t sf = sa0 + 2 * kABytes + kBBytes;
          const uint32_t tsf = tmem_base + kAccCols + stage * kSfCols;
          tmem_cp_32x128b_warpx4(tsf + 0, smem_desc_plain(sf));          // SFA0
          tmem_cp_32x128b_warpx4(tsf + 4, smem_desc_plain(sf + 512));    // SFA1
          tmem_cp_32x128b_warpx4(tsf + 8, smem_desc_plain(sf + 1024));   // SFB rows 0-127
          tmem_cp_32x128b_warpx4(tsf + 12, smem_desc_plain(sf + 1536));  // SFB rows 128-255
          const uint64_t da0 = smem_desc_sw128(sa0);
          const uint64_t da1 = smem_desc_sw128(sa0 + kABytes);
          const uint64_t db = smem_desc_sw128(sa0 + 2 * kABytes);
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            // K step k: 32 E4M3 values = 32 bytes along the swizzled row; scale byte k
            const uint32_t acc = (kb | k) != 0;
            const uint32_t id = idesc_mxf8(kFeat, n32, (uint32_t)k);
            const uint32_t kb30 = (uint32_t)k << 30;
            umma_mxf8(tmem_base, da0 + 2 * k, db + 2 * k, id, acc, (tsf + 0) | kb30,
                      (tsf + 8) | kb30);
            umma_mxf8(tmem_base + kNMax, da1 + 2 * k, db + 2 * k, id, acc, (tsf + 4) | kb30,
                      (tsf + 8) | kb30);
          }
          umma_commit(empty0 + 8 * stage);
          ++consumed;
          *consumed_sh = consumed;
          if (++stage == kStages) { stage = 0; phase ^= 1; }
        }
        if (ok) umma_commit(tmem_full);
      }
      umma_commit(drain_bar);
      mbar_wait(drain_bar, 0, abort_flag, args.status, kDrainTimeoutNs, false);
    }
    __syncwarp();
  } else {
    // ---------------- epilogue (warps 2..5) ----------------
    const int q = warp & 3;
    uint32_t acc_phase = 0;
    const uint32_t lane_base = (uint32_t)(32 * q) << 16;
    uint8_t* stg = staging_base + (warp - 2) * (kStagingBytes / kEpiWarps);
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
      const Tile t = decode_tile<kNMax>(tile, n_fblk, targs, prefix);
      if (!mbar_wait(tmem_full, acc_phase, abort_flag, args.status, args.wait_ns)) break;
      acc_phase ^= 1;
      tc_fence_after();
      constexpr int nhalves = kGatedOut ? 1 : 2;
      for (int hf = 0; hf < nhalves; ++hf) {
        const int fbase = t.f0 + hf * kFeat + 32 * q;  // first feature of this warp
        for (int j0 = 0; j0 < t.n; j0 += 32) {
          uint32_t v0[32];
          tmem_ld_32x32b_x32(tmem_base + lane_base + hf * kNMax + j0, v0);
          if constexpr (kGatedOut) {
            uint32_t v1[32];
            tmem_ld_32x32b_x32(tmem_base + lane_base + kNMax + j0, v1);
            tmem_wait_ld();
            // h = SiLU(gate) * up for this lane's feature, tokens j0..j0+31, then
            // MXFP8: the warp's 32 features of one token are one scale block
            float hv[32], am[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              hv[j] = silu_fast(__uint_as_float(v0[j])) * __uint_as_float(v1[j]);
              am[j] = fabsf(hv[j]);
            }
            // per-token amax over the 32 lanes by a butterfly transpose-reduce:
            // each round a lane keeps half of its tokens and merges the partner's
            // half; afterwards am[0] of lane j is the amax of token j
#pragma unroll
            for (int off = 16; off >= 1; off >>= 1) {
              const bool upper = (lane & off) != 0;
#pragma unroll
              for (int i = 0; i < off; ++i) {
                const float send = upper ? am[i] : am[i + off];
                const float keep = upper ? am[i + off] : am[i];
                am[i] = fmaxf(keep, __shfl_xor_sync(0xffffffffu, send, off));
              }
            }
            const int my_s = mx_scale_exp(am[0]);           // scale of token j0 + lane
            const float my_inv = mx_inv_scale(my_s);
#pragma unroll
            for (int j = 0; j < 32; ++j)
              stg[j * kPitchH + lane] =
                  mx_quant_inv(hv[j], __shfl_sync(0xffffffffu, my_inv, j));
            __syncwarp();
            // 32 tokens x 32 bytes: two 16-byte stores per lane
#pragma unroll
            for (int it = 0; it < 2; ++it) {
              const int vec = it * 32 + lane;
              const int j = vec >> 1, c = vec & 1;
              if (j0 + j < t.n && fbase < args.n_out) {
                const uint4 w = *reinterpret_cast<const uint4*>(stg + j * kPitchH + c * 16);
                *reinterpret_cast<uint4*>(static_cast<uint8_t*>(args.out) +
                                          (size_t)(t.r0 + j0 + j) * args.n_out + fbase +
                                          c * 16) = w;
              }
            }
            if (j0 + lane < t.n && fbase < args.n_out)
              args.out_sf[(size_t)(t.r0 + j0 + lane) * (args.n_out / 32) + fbase / 32] =
                  mx_scale_byte(my_s);
            __syncwarp();
          } else {
            tmem_wait_ld();
            uint16_t* s16 = reinterpret_cast<uint16_t*>(stg);
#pragma unroll
            for (int half = 0; half < 2; ++half) {
#pragma unroll
              for (int j = 0; j < 16; j += 2) {
                const uint32_t p = pack_bf16x2(__uint_as_float(v0[16 * half + j]),
                                               __uint_as_float(v0[16 * half + j + 1]));
                s16[j * kPitchY + lane] = (uint16_t)(p & 0xffffu);
                s16[(j + 1) * kPitchY + lane] = (uint16_t)(p >> 16);
              }
              __syncwarp();
              // 16 tokens x 32 features (64 B): two 16-byte stores per lane
#pragma unroll
              for (int it = 0; it < 2; ++it) {
                const int vec = it * 32 + lane;
                const int j = vec >> 2, c = vec & 3;
                const int tok = j0 + 16 * half + j;
                const int f = fbase + c * 8;
                if (tok < t.n && f < args.n_out) {
                  const uint4 w = *reinterpret_cast<const uint4*>(&s16[j * kPitchY + c * 8]);
                  *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(args.out) +
                                            (size_t)(t.r0 + tok) * args.n_out + f) = w;
                }
              }
              __syncwarp();
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(tmem_empty);
    }
  }

  __syncthreads();
  if (threadIdx.x == 0 && *abort_flag) {
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
                 "r"(512)
                 : "memory");
  }
}

// --- host side -------------------------------------------------------------------
// d % 256: the down GEMM's 256-feature tiles read two whole 128-row scale
// atoms per step (bulk copies have no out-of-bounds fill).
inline bool supported(const moe_shape& s) {
  return s.dtype == MOE_BF16 && s.d % 256 == 0 && s.I % 128 == 0;
}

// 2-D byte map [rows, cols], box 128 bytes x box_rows, 128-byte swizzle.
inline bool make_map_u8(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols,
                        uint32_t box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols};
  cuuint32_t box[2] = {(cuuint32_t)kBKf, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <bool kGatedOut>
static inline moe_status launch_f8(const CUtensorMap& a0, const CUtensorMap& a1, const CUtensorMap& b,
                            const ArgsF8& args, long long max_tiles, int sms, cudaStream_t st,
                            char* err, size_t errn) {
  static bool attr_set[64] = {};  // per device; internal linkage (one per loaded library)
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(gemm_mxf8_kernel<kGatedOut>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         smem_bytes<kGatedOut>());
    if (e != cudaSuccess) {
      snprintf(err, errn, "mxfp8 gemm smem attribute: %s", cudaGetErrorString(e));
      return MOE_ERR_CUDA;
    }
    attr_set[dev] = true;
  }
  long long grid = max_tiles < sms ? max_tiles : sms;
  if (grid < 1) grid = 1;
  ArgsF8 la = args;
  la.wait_ns = pipeline_wait_ns();
  launch_pdl(gemm_mxf8_kernel<kGatedOut>, dim3((unsigned)grid), dim3(kThreads),
             (size_t)smem_bytes<kGatedOut>(), st, a0, a1, b, la);
  note_launch();
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    snprintf(err, errn, "mxfp8 gemm launch: %s", cudaGetErrorString(e));
    return MOE_ERR_CUDA;
  }
  return MOE_OK;
}

// h = SiLU(x W1^T) * (x W3^T) from MXFP8 x_perm and weights; h written as MXFP8.
inline moe_status launch_gate_up(const moe_shape& s, const void* xq, const void* xsf,
                                 const void* w1q, const void* w1sf, const void* w3q,
                                 const void* w3sf, const int32_t* offsets, void* hq, void* hsf,
                                 uint32_t* status, int sms, cudaStream_t st, char* err,
                                 size_t errn) {
  CUtensorMap a0, a1, b;
  const uint64_t rows = (uint64_t)s.T * s.K;
  const uint64_t wrows = (uint64_t)s.N * s.I * s.d / kBKf;  // tiled: 128-byte rows
  if (!make_map_u8(&a0, w1q, wrows, kBKf, kFeat)) return map_error(err, errn, "w1 (fp8)");
  if (!make_map_u8(&a1, w3q, wrows, kBKf, kFeat)) return map_error(err, errn, "w3 (fp8)");
  if (!make_map_u8(&b, xq, rows, s.d, kBoxRows)) return map_error(err, errn, "x_perm (fp8)");
  ArgsF8 a{};
  a.seg_offsets = offsets;
  a.nseg = s.N;
  a.max_rows = (int)rows;
  a.n_out = s.I;
  a.k_dim = s.d;
  a.a_seg_rows = s.I;
  a.a1_row_off = 0;
  a.feat_per_tile = kFeat;
  a.sfa0 = static_cast<const uint8_t*>(w1sf);
  a.sfa1 = static_cast<const uint8_t*>(w3sf);
  a.sfb = static_cast<const uint8_t*>(xsf);
  a.out = hq;
  a.out_sf = static_cast<uint8_t*>(hsf);
  a.status = status;
  const long long tiles = (s.N + (long long)(rows + kNMax - 1) / kNMax) * (s.I / kFeat);
  return launch_f8<true>(a0, a1, b, a, tiles, sms, st, err, errn);
}

// y = h W2^T from MXFP8 h and W2; y written as bf16.
inline moe_status launch_down(const moe_shape& s, const void* hq, const void* hsf,
                              const void* w2q, const void* w2sf, const int32_t* offsets,
                              void* y, uint32_t* status, int sms, cudaStream_t st, char* err,
                              size_t errn) {
  CUtensorMap a, b;
  const uint64_t rows = (uint64_t)s.T * s.K;
  const uint64_t wrows = (uint64_t)s.N * s.d * s.I / kBKf;
  if (!make_map_u8(&a, w2q, wrows, kBKf, kFeat)) return map_error(err, errn, "w2 (fp8)");
  if (!make_map_u8(&b, hq, rows, s.I, kBoxRows)) return map_error(err, errn, "h (fp8)");
  ArgsF8 g{};
  g.seg_offsets = offsets;
  g.nseg = s.N;
  g.max_rows = (int)rows;
  g.n_out = s.d;
  g.k_dim = s.I;
  g.a_seg_rows = s.d;
  g.a1_row_off = kFeat;
  g.feat_per_tile = 2 * kFeat;
  g.sfa0 = static_cast<const uint8_t*>(w2sf);
  g.sfa1 = static_cast<const uint8_t*>(w2sf);
  g.sfb = static_cast<const uint8_t*>(hsf);
  g.out = y;
  g.status = status;
  const long long tiles =
      (s.N + (long long)(rows + kNMax - 1) / kNMax) * ((s.d + 2 * kFeat - 1) / (2 * kFeat));
  return launch_f8<false>(a, a, b, g, tiles, sms, st, err, errn);
}

}  // namespace f8
}  // namespace moe
