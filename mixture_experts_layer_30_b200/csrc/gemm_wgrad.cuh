// Weight gradients of the backward pass on the tensor cores (sm_100a):
//   dW1_e = da_e^T x_e,  dW3_e = du_e^T x_e,  dW2_e = dy_e^T h_e   (per FFN expert)
//   dW_r  = dlogits^T x                                            (router, one segment)
// Both operands are token-row matrices read "MN-major": the reduction runs
// over the routed rows of the expert (a ragged K of ~T*K_e/N rows), and the
// output features are their columns.
//
// Tile = (segment e, m-block, n-block of 128 output columns).  Two fp32
// accumulators of 128 x 128 per tile (D0, D1):
//   two-output form  (m_step 128)  D0 -> out0 rows m0.., D1 -> out1 rows m0..
//                                  (dW1 and dW3 share the x tile: A1 = du)
//   one-output form  (m_step 256)  D0 -> rows m0.., D1 -> rows m0+128..
// Two accumulator pairs fill the 512 TMEM columns, so the epilogue of one
// tile overlaps the MMAs of the next.
//
// One persistent CTA per SM, 10 warps:
//   warp 0      TMA producer (one lane)
//   warp 1      MMA warp: zeroes the K rows past the segment end (generic
//               stores + proxy fence) and issues the MMAs (in the A-stationary
//               kernel one lane does both, with no warp-wide broadcast per
//               stage: the tensor pipe's short queue must be refilled as soon
//               as a stage lands)
//   warps 2..9  epilogue, two warps per TMEM lane quarter (warps 2..5: D0,
//               6..9: D1): all 128 columns of its 32 rows loaded behind one
//               wait -> bf16 -> swizzled staging box -> TMA store (32 rows x
//               64 columns per store, kWgStgBoxes staging boxes per warp)
// A tile writes 64 KiB of bf16 and performs only 2*R_e*256*128 FLOPs (R_e ~
// 128 routed rows): a stream of gradient writes paced by the MMA issue and
// the epilogue.
// Waits are bounded as in gemm_tc.cuh; on expiry the status word records
// MOE_DEV_PIPELINE_TIMEOUT and the CTA drains and returns.
#pragma once

#include "gemm_tc.cuh"

namespace moe {
namespace tc {

constexpr int kWgStages = 3;
constexpr int kWgThreads = 320;
constexpr int kWgEpiWarps = 8;
constexpr int kWgN = 128;                         // output columns per tile (UMMA N)
constexpr int kWgStageBytes = 6 * kMnBoxBytes;    // A0, A1, B: two 64 x 64 boxes each
constexpr int kWgStoreBox = 32 * 128;             // 32 rows x 64 bf16 output columns
constexpr int kWgStgBoxes = 1;                    // staging boxes per epilogue warp
constexpr int kWgStagingBytes = kWgEpiWarps * kWgStgBoxes * kWgStoreBox;
constexpr int kWgNumBars = 2 * kWgStages + 2 * 2 + 1;
constexpr int kWgSmemBytes = 1024 + kWgStages * kWgStageBytes + kWgStagingBytes + kCtrlBytes;
static_assert(kWgSmemBytes <= 232448, "wgrad shared memory");
static_assert(8 * kWgNumBars + 12 <= kCtrlBytes, "wgrad control block");

struct WgArgs {
  const int32_t* seg_offsets;  // [nseg + 1] row offsets, or NULL for one segment
  int nseg;
  int single_rows;             // rows of the single segment when seg_offsets == NULL
  int max_rows;                // rows of the operand matrices (bound for offsets)
  int m_out, n_out;            // each output matrix is [m_out, n_out]; segment e's at rows e*m_out
  int m_step;                  // 128: two outputs; 256: D1 = rows m0 + 128
  int a1_col_off;              // column of the A1 boxes relative to A0's
  int out1_row_off;            // row offset of D1's output (0 or 128)
  uint32_t* status;
  unsigned long long wait_ns;  // time limit of one pipeline wait (set at launch)
};

struct WgTile {
  int seg, m0, n0, lo, rows;
};

MOE_DEV WgTile wg_decode(int tile, const WgArgs& a, int mblk, int nblk) {
  WgTile t;
  const int per = mblk * nblk;
  t.seg = tile / per;
  const int rem = tile - t.seg * per;
  t.m0 = (rem / nblk) * a.m_step;
  t.n0 = (rem % nblk) * kWgN;
  if (a.seg_offsets) {
    int lo = a.seg_offsets[t.seg], hi = a.seg_offsets[t.seg + 1];
    if (lo < 0 || hi < lo || hi > a.max_rows) {
      set_status(a.status, MOE_DEV_BAD_OFFSETS);
      lo = hi = 0;
    }
    t.lo = lo;
    t.rows = hi - lo;
  } else {
    t.lo = 0;
    t.rows = a.single_rows;
  }
  return t;
}

MOE_DEV void tma_store_2d(const CUtensorMap* map, uint32_t src, int c0, int c1) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(c0), "r"(c1), "r"(src)
               : "memory");
}
// The same store with an L2 eviction-priority hint (a createpolicy value).
MOE_DEV void tma_store_2d_hint(const CUtensorMap* map, uint32_t src, int c0, int c1,
                               uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.global.shared::cta.bulk_group.L2::cache_hint [%0, {%1, %2}], [%3], "
      "%4;" ::"l"(reinterpret_cast<uint64_t>(map)),
      "r"(c0), "r"(c1), "r"(src), "l"(policy)
      : "memory");
}
MOE_DEV void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
template <int N>
MOE_DEV void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
MOE_DEV void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// One accumulator half of a finished tile: the warp's 32 output rows x 128
// columns.  TMEM (address `ta`: lane quarter, buffer and half applied) is read
// with four loads behind one wait and released on `tmem_empty` before the
// stores; each 64-column piece goes bf16 -> swizzled staging box -> TMA store.
// has_data false: the segment had no rows and the gradient is zero.
MOE_DEV void wg_store_half(const CUtensorMap* om, uint32_t ta, bool has_data, bool row_ok,
                           int out_row, int n0, int n_out, uint32_t stg0, int lane, int& nstore,
                           uint32_t tmem_empty, uint64_t store_policy = 0) {
  if (!row_ok) {
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(tmem_empty);
    return;
  }
  uint32_t v[4][32];
  if (has_data) {
#pragma unroll
    for (int c = 0; c < 4; ++c) tmem_ld_32x32b_x32(ta + 32 * c, v[c]);
    tmem_wait_ld();
  } else {
#pragma unroll
    for (int c = 0; c < 4; ++c)
#pragma unroll
      for (int i = 0; i < 32; ++i) v[c][i] = 0u;
  }
  tc_fence_before();
  __syncwarp();
  if (lane == 0) mbar_arrive(tmem_empty);  // TMEM is free once the warp's loads landed
#pragma unroll
  for (int c = 0; c < kWgN / 64; ++c) {
    const int col = n0 + 64 * c;
    if (col >= n_out) continue;
    // this lane's output row: 64 columns -> 32 bf16 pairs -> 8 16-byte pieces,
    // written to the 128-byte-swizzled staging box (piece p at p ^ (row & 7))
    const uint32_t sb = stg0 + (nstore % kWgStgBoxes) * kWgStoreBox;
    if (lane == 0) bulk_wait_read<kWgStgBoxes - 1>();
    __syncwarp();
#pragma unroll
    for (int p = 0; p < 8; ++p) {
      const uint32_t* w = &v[2 * c + (p >> 2)][8 * (p & 3)];
      const uint32_t w0 = pack_bf16x2(__uint_as_float(w[0]), __uint_as_float(w[1]));
      const uint32_t w1 = pack_bf16x2(__uint_as_float(w[2]), __uint_as_float(w[3]));
      const uint32_t w2 = pack_bf16x2(__uint_as_float(w[4]), __uint_as_float(w[5]));
      const uint32_t w3 = pack_bf16x2(__uint_as_float(w[6]), __uint_as_float(w[7]));
      const uint32_t addr = sb + lane * 128 + ((p ^ (lane & 7)) << 4);
      asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(w0), "r"(w1),
                   "r"(w2), "r"(w3)
                   : "memory");
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    __syncwarp();
    if (lane == 0) {
      if (store_policy) tma_store_2d_hint(om, sb, col, out_row, store_policy);
      else tma_store_2d(om, sb, col, out_row);
      bulk_commit();
    }
    ++nstore;
  }
}

// Zero K rows nv .. 16*ceil(nv/16)-1 of `nbox` consecutive 64 x 64 boxes at
// shared address `base` (whole 128-byte rows, so the swizzle does not matter),
// then make the stores visible to the tensor cores.  The whole warp calls.
MOE_DEV void wg_zero_tail(uint32_t base, int nbox, int nv, int lane) {
  const int zrows = ((nv + 15) & ~15) - nv;
  if (zrows <= 0) return;
  const int per_box = zrows * 8;  // 16-byte pieces per box
  for (int i = lane; i < nbox * per_box; i += 32) {
    const int box = i / per_box, piece = i - box * per_box;
    const uint32_t addr = base + box * kMnBoxBytes + nv * 128 + piece * 16;
    asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(addr), "r"(0u) : "memory");
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  __syncwarp();
}

// The same clearing done by one thread (the A-stationary MMA issuer).
MOE_DEV void wg_zero_tail_one(uint32_t base, int nbox, int nv) {
  const int zrows = ((nv + 15) & ~15) - nv;
  if (zrows <= 0) return;
  for (int box = 0; box < nbox; ++box)
    for (int piece = 0; piece < zrows * 8; ++piece) {
      const uint32_t addr = base + box * kMnBoxBytes + nv * 128 + piece * 16;
      asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(addr), "r"(0u) : "memory");
    }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__global__ void __launch_bounds__(kWgThreads, 1)
gemm_wgrad_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                  const __grid_constant__ CUtensorMap tmO0,
                  const __grid_constant__ CUtensorMap tmO1, const WgArgs args) {
  pdl_trigger();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* stages = smem;
  uint8_t* staging = smem + kWgStages * kWgStageBytes;
  uint8_t* ctrl = staging + kWgStagingBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(ctrl);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(ctrl + 8 * kWgNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(ctrl + 8 * kWgNumBars + 4);
  volatile int* consumed_sh = reinterpret_cast<volatile int*>(ctrl + 8 * kWgNumBars + 8);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t full0 = smem_u32(&bars[0]);
  const uint32_t empty0 = smem_u32(&bars[kWgStages]);
  const uint32_t tmem_full0 = smem_u32(&bars[2 * kWgStages]);
  const uint32_t tmem_empty0 = smem_u32(&bars[2 * kWgStages + 2]);
  const uint32_t drain_bar = smem_u32(&bars[2 * kWgStages + 4]);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kWgStages; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tmem_full0 + 8 * b, 1);
      mbar_init(tmem_empty0 + 8 * b, kWgEpiWarps);  // one arrival per warp
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    *consumed_sh = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    tma_prefetch_desc(&tmO0);
    tma_prefetch_desc(&tmO1);
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(512)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait();  // the prologue above touches no global memory

  const int nseg = args.seg_offsets ? args.nseg : 1;
  const int mblk = (args.m_out + args.m_step - 1) / args.m_step;
  const int nblk = (args.n_out + kWgN - 1) / kWgN;
  const int total = nseg * mblk * nblk;
  int issued = 0;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer ----------------
      uint32_t stage = 0, phase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
        const WgTile t = wg_decode(tile, args, mblk, nblk);
        const int nk = (t.rows + kBK - 1) / kBK;
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(empty0 + 8 * stage, phase ^ 1, abort_flag, args.status, args.wait_ns)) {
            ok = false;
            break;
          }
          const uint32_t fb = full0 + 8 * stage;
          const uint32_t sa = smem_u32(stages + stage * kWgStageBytes);
          const int row = t.lo + kb * kBK;
          mbar_arrive_expect_tx(fb, kWgStageBytes);
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            tma_load_2d(sa + h * kMnBoxBytes, &tmA, t.m0 + 64 * h, row, fb);
            tma_load_2d(sa + 2 * kMnBoxBytes + h * kMnBoxBytes, &tmA,
                        t.m0 + args.a1_col_off + 64 * h, row, fb);
            tma_load_2d(sa + 4 * kMnBoxBytes + h * kMnBoxBytes, &tmB, t.n0 + 64 * h, row, fb);
          }
          ++issued;
          if (++stage == kWgStages) { stage = 0; phase ^= 1; }
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------- MMA warp ----------------
    uint32_t stage = 0, phase = 0;
    bool ok = true;
    int consumed = 0, local = 0;
    const uint32_t idesc = idesc_bf16(kFeat, kWgN, true, true);
    for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x, ++local) {
      const WgTile t = wg_decode(tile, args, mblk, nblk);
      const int nk = (t.rows + kBK - 1) / kBK;
      const int buf = local & 1;
      const uint32_t acc_parity = (uint32_t)((local >> 1) & 1);
      const uint32_t d0 = tmem_base + buf * 2 * kWgN;
      int go = 1;
      if (lane == 0) go = mbar_wait(tmem_empty0 + 8 * buf, acc_parity ^ 1, abort_flag, args.status, args.wait_ns);
      if (!__shfl_sync(0xffffffffu, go, 0)) break;
      tc_fence_after();
      for (int kb = 0; kb < nk; ++kb) {
        go = 1;
        if (lane == 0) go = mbar_wait(full0 + 8 * stage, phase, abort_flag, args.status, args.wait_ns);
        if (!__shfl_sync(0xffffffffu, go, 0)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t sa = smem_u32(stages + stage * kWgStageBytes);
        const int nv = min(kBK, t.rows - kb * kBK);  // live K rows of this block
        const int ksteps = (nv + 15) >> 4;
        wg_zero_tail(sa, 6, nv, lane);
        if (lane == 0) {
          const uint64_t da0 = smem_desc_mn_sw128(sa);
          const uint64_t da1 = smem_desc_mn_sw128(sa + 2 * kMnBoxBytes);
          const uint64_t db = smem_desc_mn_sw128(sa + 4 * kMnBoxBytes);
          for (int k = 0; k < ksteps; ++k) {
            const uint32_t acc = (kb | k) != 0;
            umma_bf16(d0, da0 + 128 * k, db + 128 * k, idesc, acc);
            umma_bf16(d0 + kWgN, da1 + 128 * k, db + 128 * k, idesc, acc);
          }
          umma_commit(empty0 + 8 * stage);
          ++consumed;
          *consumed_sh = consumed;
        }
        __syncwarp();
        if (++stage == kWgStages) { stage = 0; phase ^= 1; }
      }
      if (ok && lane == 0) umma_commit(tmem_full0 + 8 * buf);
      __syncwarp();
    }
    if (lane == 0) {
      umma_commit(drain_bar);
      mbar_wait(drain_bar, 0, abort_flag, args.status, kDrainTimeoutNs, false);
    }
    __syncwarp();
  } else {
    // ---------------- epilogue (warps 2..9) ----------------
    const int q = warp & 3;         // TMEM lane quarter = output rows 32q..32q+31 of a half
    const int hf = (warp - 2) >> 2; // accumulator D0 or D1
    const uint32_t stg0 = smem_u32(staging + (warp - 2) * kWgStgBoxes * kWgStoreBox);
    const uint32_t lane_base = (uint32_t)(32 * q) << 16;
    const CUtensorMap* om = hf ? &tmO1 : &tmO0;
    int local = 0, nstore = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x, ++local) {
      const WgTile t = wg_decode(tile, args, mblk, nblk);
      const int buf = local & 1;
      const uint32_t acc_parity = (uint32_t)((local >> 1) & 1);
      if (!mbar_wait(tmem_full0 + 8 * buf, acc_parity, abort_flag, args.status, args.wait_ns)) break;
      tc_fence_after();
      const int r = (hf ? t.m0 + args.out1_row_off : t.m0) + 32 * q;  // first output row
      wg_store_half(om, tmem_base + lane_base + buf * 2 * kWgN + hf * kWgN, t.rows > 0,
                    r < args.m_out, t.seg * args.m_out + r, t.n0, args.n_out, stg0, lane, nstore,
                    tmem_empty0 + 8 * buf);
    }
    if (lane == 0) bulk_wait_all();
    __syncwarp();
  }

  __syncthreads();
  if (threadIdx.x == 0 && *abort_flag) {
    const int consumed = *consumed_sh;
    for (int i = consumed; i < issued; ++i)
      mbar_wait(full0 + 8 * (i % kWgStages), (uint32_t)((i / kWgStages) & 1), abort_flag,
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

// --- expert weight gradients with the A operand resident -------------------------
// Work unit = (expert e, m-block): the A rows of the segment (da | du, or dy:
// 256 columns x R_e rows) are loaded once into up to kAsSlots resident blocks
// and every n-block of the unit streams only its B block (x_perm or h, 128
// columns x R_e rows), so the token rows cross L2 ~3x less often than with a
// (A, B) pair per tile.  A unit whose segment is longer than the resident
// blocks hold streams A with B, block by block, through the same slots.
constexpr int kAsSlots = 3;                       // resident A blocks: segments up to 192 rows
constexpr int kAsSlotBytes = 4 * kMnBoxBytes;     // A0 and A1, two 64 x 64 boxes each
constexpr int kAsBStages = 6;
constexpr int kAsBBytes = 2 * kMnBoxBytes;        // B: two 64 x 64 boxes
constexpr int kAsNumBars = 2 * kAsSlots + 2 * kAsBStages + 2 * 2 + 1;
constexpr int kAsSmemBytes = 1024 + kAsSlots * kAsSlotBytes + kAsBStages * kAsBBytes +
                             kWgStagingBytes + kCtrlBytes;
static_assert(kAsSmemBytes <= 232448, "A-stationary wgrad shared memory");
static_assert(8 * kAsNumBars + 16 <= kCtrlBytes, "A-stationary wgrad control block");

struct AsUnit {
  int seg, m0, lo, rows, nk;
  bool stat;
};

MOE_DEV AsUnit as_decode(int unit, const WgArgs& a, int mblk) {
  AsUnit u;
  u.seg = unit / mblk;
  u.m0 = (unit - u.seg * mblk) * a.m_step;
  int lo = a.seg_offsets[u.seg], hi = a.seg_offsets[u.seg + 1];
  if (lo < 0 || hi < lo || hi > a.max_rows) {
    set_status(a.status, MOE_DEV_BAD_OFFSETS);
    lo = hi = 0;
  }
  u.lo = lo;
  u.rows = hi - lo;
  u.nk = (u.rows + kBK - 1) / kBK;
  u.stat = u.nk <= kAsSlots;
  return u;
}

__global__ void __launch_bounds__(kWgThreads, 1)
gemm_wgrad_as_kernel(const __grid_constant__ CUtensorMap tmA,
                     const __grid_constant__ CUtensorMap tmB,
                     const __grid_constant__ CUtensorMap tmO0,
                     const __grid_constant__ CUtensorMap tmO1, const WgArgs args) {
  pdl_trigger();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* aslots = smem;
  uint8_t* bstages = aslots + kAsSlots * kAsSlotBytes;
  uint8_t* staging = bstages + kAsBStages * kAsBBytes;
  uint8_t* ctrl = staging + kWgStagingBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(ctrl);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(ctrl + 8 * kAsNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(ctrl + 8 * kAsNumBars + 4);
  volatile int* a_seen_sh = reinterpret_cast<volatile int*>(ctrl + 8 * kAsNumBars + 8);
  volatile int* b_seen_sh = reinterpret_cast<volatile int*>(ctrl + 8 * kAsNumBars + 12);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t a_full0 = smem_u32(&bars[0]);
  const uint32_t a_empty0 = smem_u32(&bars[kAsSlots]);
  const uint32_t b_full0 = smem_u32(&bars[2 * kAsSlots]);
  const uint32_t b_empty0 = smem_u32(&bars[2 * kAsSlots + kAsBStages]);
  const uint32_t tmem_full0 = smem_u32(&bars[2 * kAsSlots + 2 * kAsBStages]);
  const uint32_t tmem_empty0 = smem_u32(&bars[2 * kAsSlots + 2 * kAsBStages + 2]);
  const uint32_t drain_bar = smem_u32(&bars[2 * kAsSlots + 2 * kAsBStages + 4]);

  if (threadIdx.x == 0) {
    for (int i = 0; i < kAsSlots; ++i) {
      mbar_init(a_full0 + 8 * i, 1);
      mbar_init(a_empty0 + 8 * i, 1);
    }
    for (int i = 0; i < kAsBStages; ++i) {
      mbar_init(b_full0 + 8 * i, 1);
      mbar_init(b_empty0 + 8 * i, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tmem_full0 + 8 * b, 1);
      mbar_init(tmem_empty0 + 8 * b, kWgEpiWarps);  // one arrival per warp
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    *a_seen_sh = 0;
    *b_seen_sh = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    tma_prefetch_desc(&tmO0);
    tma_prefetch_desc(&tmO1);
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(512)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait();  // the prologue above touches no global memory

  const int mblk = (args.m_out + args.m_step - 1) / args.m_step;
  const int nblk = (args.n_out + kWgN - 1) / kWgN;
  const int units = args.nseg * mblk;
  int a_issued = 0, b_issued = 0;  // producer: A and B fills

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer ----------------
      bool ok = true;
      // the B block of an expert is read by all of its m-block units: keep it in L2
      const uint64_t pol_a = l2_policy_evict_first();
      const uint64_t pol_b = l2_policy_evict_last();
      auto fill_a = [&](const AsUnit& u, int kb) -> bool {
        const int slot = a_issued % kAsSlots;
        const uint32_t par = (uint32_t)((a_issued / kAsSlots) & 1);
        if (!mbar_wait(a_empty0 + 8 * slot, par ^ 1, abort_flag, args.status, args.wait_ns)) return false;
        const uint32_t fb = a_full0 + 8 * slot;
        const uint32_t sa = smem_u32(aslots + slot * kAsSlotBytes);
        const int row = u.lo + kb * kBK;
        mbar_arrive_expect_tx(fb, kAsSlotBytes);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          tma_load_2d_hint(sa + h * kMnBoxBytes, &tmA, u.m0 + 64 * h, row, fb, pol_a);
          tma_load_2d_hint(sa + 2 * kMnBoxBytes + h * kMnBoxBytes, &tmA,
                           u.m0 + args.a1_col_off + 64 * h, row, fb, pol_a);
        }
        ++a_issued;
        return true;
      };
      auto fill_b = [&](const AsUnit& u, int nb, int kb) -> bool {
        const int st = b_issued % kAsBStages;
        const uint32_t par = (uint32_t)((b_issued / kAsBStages) & 1);
        if (!mbar_wait(b_empty0 + 8 * st, par ^ 1, abort_flag, args.status, args.wait_ns)) return false;
        const uint32_t fb = b_full0 + 8 * st;
        const uint32_t sb = smem_u32(bstages + st * kAsBBytes);
        const int row = u.lo + kb * kBK;
        mbar_arrive_expect_tx(fb, kAsBBytes);
        tma_load_2d_hint(sb, &tmB, nb * kWgN, row, fb, pol_b);
        tma_load_2d_hint(sb + kMnBoxBytes, &tmB, nb * kWgN + 64, row, fb, pol_b);
        ++b_issued;
        return true;
      };
      for (int unit = blockIdx.x; unit < units && ok; unit += gridDim.x) {
        const AsUnit u = as_decode(unit, args, mblk);
        if (u.stat) {
          for (int kb = 0; kb < u.nk && ok; ++kb) ok = fill_a(u, kb);
          for (int nb = 0; nb < nblk && ok; ++nb)
            for (int kb = 0; kb < u.nk && ok; ++kb) ok = fill_b(u, nb, kb);
        } else {
          for (int nb = 0; nb < nblk && ok; ++nb)
            for (int kb = 0; kb < u.nk && ok; ++kb) ok = fill_a(u, kb) && fill_b(u, nb, kb);
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------- MMA issuer (lane 0 alone) ----------------
    // One thread waits, clears tails and issues: no warp-wide broadcast between
    // a stage's arrival and its MMAs, so the tensor pipe's short queue is
    // refilled as soon as the data is there.
    if (lane == 0) {
      bool ok = true;
      int a_seen = 0, b_seen = 0, local = 0;
      const uint32_t idesc = idesc_bf16(kFeat, kWgN, true, true);
      int data_end = args.seg_offsets[args.nseg];  // rows written by the forward pass
      if (data_end < 0 || data_end > args.max_rows) data_end = 0;  // (offsets checked per unit)
      for (int unit = blockIdx.x; unit < units && ok; unit += gridDim.x) {
        const AsUnit u = as_decode(unit, args, mblk);
        const int a0 = a_seen;  // first A fill of this unit
        if (u.stat) {
          for (int kb = 0; kb < u.nk && ok; ++kb) {
            const int i = a0 + kb;
            ok = mbar_wait(a_full0 + 8 * (i % kAsSlots), (uint32_t)((i / kAsSlots) & 1), abort_flag,
                           args.status, args.wait_ns);
          }
          if (!ok) break;
          a_seen = a0 + u.nk;
          *a_seen_sh = a_seen;
          tc_fence_after();
          // resident A: K rows past the segment end cleared once per unit
          for (int kb = 0; kb < u.nk; ++kb)
            wg_zero_tail_one(smem_u32(aslots + ((a0 + kb) % kAsSlots) * kAsSlotBytes), 4,
                             min(kBK, u.rows - kb * kBK));
        }
        for (int nb = 0; nb < nblk && ok; ++nb, ++local) {
          const int buf = local & 1;
          if (!mbar_wait(tmem_empty0 + 8 * buf, (uint32_t)(((local >> 1) & 1) ^ 1), abort_flag,
                         args.status, args.wait_ns)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t d0 = tmem_base + buf * 2 * kWgN;
          for (int kb = 0; kb < u.nk; ++kb) {
            const int nv = min(kBK, u.rows - kb * kBK);
            int ai;
            if (u.stat) {
              ai = a0 + kb;
            } else {
              ai = a_seen;
              if (!mbar_wait(a_full0 + 8 * (ai % kAsSlots), (uint32_t)((ai / kAsSlots) & 1),
                             abort_flag, args.status, args.wait_ns)) {
                ok = false;
                break;
              }
              ++a_seen;
              tc_fence_after();
              wg_zero_tail_one(smem_u32(aslots + (ai % kAsSlots) * kAsSlotBytes), 4, nv);
            }
            const int bs = b_seen % kAsBStages;
            if (!mbar_wait(b_full0 + 8 * bs, (uint32_t)((b_seen / kAsBStages) & 1), abort_flag,
                           args.status, args.wait_ns)) {
              ok = false;
              break;
            }
            ++b_seen;
            *a_seen_sh = a_seen;
            *b_seen_sh = b_seen;
            tc_fence_after();
            const uint32_t sa = smem_u32(aslots + (ai % kAsSlots) * kAsSlotBytes);
            const uint32_t sb = smem_u32(bstages + bs * kAsBBytes);
            // A holds the gradient rows and is zeroed past every segment end, so
            // the next expert's gradient rows never enter.  B holds forward
            // activations (x_perm or h): past a segment end they are the next
            // expert's rows, finite whenever the forward pass was, and meet those
            // zero rows.  Only B rows past the last segment (never written,
            // possibly not finite) are cleared.
            if (u.lo + kb * kBK + ((nv + 15) & ~15) > data_end) wg_zero_tail_one(sb, 2, nv);
            const int ksteps = (nv + 15) >> 4;
            const uint64_t da0 = smem_desc_mn_sw128(sa);
            const uint64_t da1 = smem_desc_mn_sw128(sa + 2 * kMnBoxBytes);
            const uint64_t db = smem_desc_mn_sw128(sb);
            for (int k = 0; k < ksteps; ++k) {
              const uint32_t acc = (kb | k) != 0;
              umma_bf16(d0, da0 + 128 * k, db + 128 * k, idesc, acc);
              umma_bf16(d0 + kWgN, da1 + 128 * k, db + 128 * k, idesc, acc);
            }
            umma_commit(b_empty0 + 8 * bs);
            if (!u.stat) umma_commit(a_empty0 + 8 * (ai % kAsSlots));
          }
          if (ok) umma_commit(tmem_full0 + 8 * buf);
        }
        // resident A blocks are released once the unit's last MMAs complete
        if (ok && u.stat)
          for (int kb = 0; kb < u.nk; ++kb) umma_commit(a_empty0 + 8 * ((a0 + kb) % kAsSlots));
      }
      umma_commit(drain_bar);
      mbar_wait(drain_bar, 0, abort_flag, args.status, kDrainTimeoutNs, false);
    }
    __syncwarp();
  } else {
    // ---------------- epilogue (warps 2..9) ----------------
    const int q = warp & 3;
    const int hf = (warp - 2) >> 2;
    const uint32_t stg0 = smem_u32(staging + (warp - 2) * kWgStgBoxes * kWgStoreBox);
    const uint32_t lane_base = (uint32_t)(32 * q) << 16;
    const CUtensorMap* om = hf ? &tmO1 : &tmO0;
    const uint64_t pol_out = l2_policy_evict_first();  // written once, never read back here
    int local = 0, nstore = 0;
    bool ok = true;
    for (int unit = blockIdx.x; unit < units && ok; unit += gridDim.x) {
      const AsUnit u = as_decode(unit, args, mblk);
      const int r = (hf ? u.m0 + args.out1_row_off : u.m0) + 32 * q;  // first output row
      for (int nb = 0; nb < nblk; ++nb, ++local) {
        const int buf = local & 1;
        if (!mbar_wait(tmem_full0 + 8 * buf, (uint32_t)((local >> 1) & 1), abort_flag,
                       args.status, args.wait_ns)) {
          ok = false;
          break;
        }
        tc_fence_after();
        wg_store_half(om, tmem_base + lane_base + buf * 2 * kWgN + hf * kWgN, u.rows > 0,
                      r < args.m_out, u.seg * args.m_out + r, nb * kWgN, args.n_out, stg0, lane,
                      nstore, tmem_empty0 + 8 * buf, pol_out);
      }
    }
    if (lane == 0) bulk_wait_all();
    __syncwarp();
  }

  __syncthreads();
  if (threadIdx.x == 0 && *abort_flag) {
    // drain the copies still in flight into shared memory (bounded)
    for (int i = *a_seen_sh; i < a_issued; ++i)
      mbar_wait(a_full0 + 8 * (i % kAsSlots), (uint32_t)((i / kAsSlots) & 1), abort_flag,
                args.status, kDrainTimeoutNs, false);
    for (int i = *b_seen_sh; i < b_issued; ++i)
      mbar_wait(b_full0 + 8 * (i % kAsBStages), (uint32_t)((i / kAsBStages) & 1), abort_flag,
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

// Output view [rows, cols] bf16 for TMA stores: 32-row x 64-column boxes, 128-byte swizzle.
inline bool make_store_map(CUtensorMap* m, void* base, uint64_t rows, uint64_t cols) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {64, 32};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

static inline moe_status launch_wgrad(const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& o0,
                               const CUtensorMap& o1, const WgArgs& args, int sms,
                               cudaStream_t st, char* err, size_t errn) {
  static bool attr_set[64] = {};  // per device; internal linkage (one per loaded library)
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(gemm_wgrad_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, kWgSmemBytes);
    if (e != cudaSuccess) {
      snprintf(err, errn, "wgrad smem attribute: %s", cudaGetErrorString(e));
      return MOE_ERR_CUDA;
    }
    attr_set[dev] = true;
  }
  const long long nseg = args.seg_offsets ? args.nseg : 1;
  const long long tiles = nseg * ((args.m_out + args.m_step - 1) / args.m_step) *
                          ((args.n_out + kWgN - 1) / kWgN);
  long long grid = tiles < sms ? tiles : sms;
  if (grid < 1) grid = 1;
  WgArgs la = args;
  la.wait_ns = pipeline_wait_ns();
  launch_pdl(gemm_wgrad_kernel, dim3((unsigned)grid), dim3(kWgThreads), (size_t)kWgSmemBytes, st,
             a, b, o0, o1, la);
  note_launch();
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    snprintf(err, errn, "wgrad launch: %s", cudaGetErrorString(e));
    return MOE_ERR_CUDA;
  }
  return MOE_OK;
}

static inline moe_status launch_wgrad_as(const CUtensorMap& a, const CUtensorMap& b,
                                  const CUtensorMap& o0, const CUtensorMap& o1,
                                  const WgArgs& args, int sms, cudaStream_t st, char* err,
                                  size_t errn) {
  static bool attr_set[64] = {};  // per device; internal linkage (one per loaded library)
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(gemm_wgrad_as_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, kAsSmemBytes);
    if (e != cudaSuccess) {
      snprintf(err, errn, "wgrad smem attribute: %s", cudaGetErrorString(e));
      return MOE_ERR_CUDA;
    }
    attr_set[dev] = true;
  }
  const long long units = (long long)args.nseg * ((args.m_out + args.m_step - 1) / args.m_step);
  long long grid = units < sms ? units : sms;
  if (grid < 1) grid = 1;
  WgArgs la = args;
  la.wait_ns = pipeline_wait_ns();
  launch_pdl(gemm_wgrad_as_kernel, dim3((unsigned)grid), dim3(kWgThreads), (size_t)kAsSmemBytes,
             st, a, b, o0, o1, la);
  note_launch();
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    snprintf(err, errn, "wgrad launch: %s", cudaGetErrorString(e));
    return MOE_ERR_CUDA;
  }
  return MOE_OK;
}

// dW1[e] = da_e^T x_perm_e and dW3[e] = du_e^T x_perm_e (dau = da | du [rows, 2I]).
inline moe_status launch_wgrad_w13(const moe_shape& s, const void* x_perm, const void* dau,
                                   const int32_t* offsets, void* dw1, void* dw3,
                                   uint32_t* status, int sms, cudaStream_t st, char* err,
                                   size_t errn) {
  const uint64_t rows = (uint64_t)s.T * s.K;
  CUtensorMap a, b, o0, o1;
  if (!make_map(&a, dau, rows, 2 * (uint64_t)s.I, 64)) return map_error(err, errn, "dau");
  if (!make_map(&b, x_perm, rows, s.d, 64)) return map_error(err, errn, "x_perm");
  if (!make_store_map(&o0, dw1, (uint64_t)s.N * s.I, s.d)) return map_error(err, errn, "dw1");
  if (!make_store_map(&o1, dw3, (uint64_t)s.N * s.I, s.d)) return map_error(err, errn, "dw3");
  WgArgs g{};
  g.seg_offsets = offsets;
  g.nseg = s.N;
  g.max_rows = (int)rows;
  g.m_out = s.I;
  g.n_out = s.d;
  g.m_step = 128;
  g.a1_col_off = s.I;
  g.out1_row_off = 0;
  g.status = status;
  return launch_wgrad_as(a, b, o0, o1, g, sms, st, err, errn);
}

// dW2[e] = dy_e^T h_e.
inline moe_status launch_wgrad_w2(const moe_shape& s, const void* h, const void* dy,
                                  const int32_t* offsets, void* dw2, uint32_t* status, int sms,
                                  cudaStream_t st, char* err, size_t errn) {
  const uint64_t rows = (uint64_t)s.T * s.K;
  CUtensorMap a, b, o0;
  if (!make_map(&a, dy, rows, s.d, 64)) return map_error(err, errn, "dy_perm");
  if (!make_map(&b, h, rows, s.I, 64)) return map_error(err, errn, "h");
  if (!make_store_map(&o0, dw2, (uint64_t)s.N * s.d, s.I)) return map_error(err, errn, "dw2");
  WgArgs g{};
  g.seg_offsets = offsets;
  g.nseg = s.N;
  g.max_rows = (int)rows;
  g.m_out = s.d;
  g.n_out = s.I;
  g.m_step = 256;
  g.a1_col_off = 128;
  g.out1_row_off = 128;
  g.status = status;
  return launch_wgrad_as(a, b, o0, o0, g, sms, st, err, errn);
}

// dW_r = dlogits^T x over all T tokens (one segment).
inline moe_status launch_router_wgrad(const moe_shape& s, const void* dlogits, const void* x,
                                      void* dw_router, uint32_t* status, int sms,
                                      cudaStream_t st, char* err, size_t errn) {
  const int E = s.N + s.Z;
  CUtensorMap a, b, o;
  if (!make_map(&a, dlogits, (uint64_t)s.T, E, 64)) return map_error(err, errn, "dlogits");
  if (!make_map(&b, x, (uint64_t)s.T, s.d, 64)) return map_error(err, errn, "x");
  if (!make_store_map(&o, dw_router, (uint64_t)E, s.d)) return map_error(err, errn, "dw_router");
  WgArgs g{};
  g.seg_offsets = nullptr;
  g.nseg = 1;
  g.single_rows = s.T;
  g.max_rows = s.T;
  g.m_out = E;
  g.n_out = s.d;
  g.m_step = 256;
  g.a1_col_off = 128;
  g.out1_row_off = 128;
  g.status = status;
  return launch_wgrad(a, b, o, o, g, sms, st, err, errn);
}

}  // namespace tc
}  // namespace moe
