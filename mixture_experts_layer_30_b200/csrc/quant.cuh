// MXFP8 quantisation for the FP8 expert path: E4M3 elements with one
// power-of-two scale 2^s per 32 consecutive values of a row (along the GEMM
// reduction axis).  s is the smallest integer with amax <= 448 * 2^s, so no
// element saturates; the scale is stored as the biased exponent byte s + 127
// (the UE8M0 encoding the block-scaled tensor-core instructions read).
// The LongCat series notes describe FP8 blockwise-quantised experts for
// inference; this is that scheme in the block shape sm_100 consumes.
#pragma once

#include <cuda_fp8.h>

#include "common.cuh"

namespace moe {

// Smallest s with amax <= 448 * 2^s, for finite amax >= 0 (0 when amax == 0).
// amax = M * 2^e with M in [1, 2): amax * 2^-(e-8) = 256 M <= 448 iff M <= 1.75.
MOE_DEV int mx_scale_exp(float amax) {
  const uint32_t b = __float_as_uint(amax) & 0x7fffffffu;
  if (b == 0) return 0;
  uint32_t ef = b >> 23, frac = b & 0x7fffffu;
  int e;
  if (ef) {
    e = (int)ef - 127;
  } else {  // subnormal: normalise the fraction
    const int p = 31 - __clz(frac);
    e = p - 149;
    frac = (frac << (23 - p)) & 0x7fffffu;
  }
  return frac <= 0x600000u ? e - 8 : e - 7;
}

MOE_DEV uint8_t mx_scale_byte(int s) { return (uint8_t)min(254, max(0, s + 127)); }

// 2^-s as a float: exact for -126 <= -s <= 127 (built from the exponent bits),
// ldexpf outside that range.
MOE_DEV float mx_inv_scale(int s) {
  const int e = 127 - s;
  return (e >= 1 && e <= 254) ? __uint_as_float((uint32_t)e << 23) : ldexpf(1.0f, -s);
}

// E4M3 code of v * 2^-s, round to nearest even (|v| <= 448 * 2^s never saturates).
// Multiplying by a power of two is exact, so this is the rounding of v / 2^s.
MOE_DEV uint8_t mx_quant_inv(float v, float inv) {
  return (uint8_t)__nv_cvt_float_to_fp8(v * inv, __NV_SATFINITE, __NV_E4M3);
}
MOE_DEV uint8_t mx_quant(float v, int s) {
  return (uint8_t)__nv_cvt_float_to_fp8(ldexpf(v, -s), __NV_SATFINITE, __NV_E4M3);
}

// Quantise 32 values (one block) held as 4 x 16 bytes of bf16; returns the
// scale exponent and writes 32 E4M3 codes into q (2 x 16 bytes).
MOE_DEV int mx_quant_block_bf16(const uint4 (&in)[4], uint4 (&q)[2]) {
  float f[32];
#pragma unroll
  for (int i = 0; i < 4; ++i) unpack16(in[i], f + 8 * i, __nv_bfloat16());
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(f[i]));
  const int s = mx_scale_exp(amax);
  const float inv = mx_inv_scale(s);
  uint32_t w[8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
    w[i] = (uint32_t)mx_quant_inv(f[4 * i], inv) | ((uint32_t)mx_quant_inv(f[4 * i + 1], inv) << 8) |
           ((uint32_t)mx_quant_inv(f[4 * i + 2], inv) << 16) |
           ((uint32_t)mx_quant_inv(f[4 * i + 3], inv) << 24);
  q[0] = make_uint4(w[0], w[1], w[2], w[3]);
  q[1] = make_uint4(w[4], w[5], w[6], w[7]);
  return s;
}

// Weights: n matrices [rows, cols] bf16 (row-major) -> 128 x 128 E4M3 tiles,
// each 16 KiB row-major, at tile index (m * rows/128 + rb) * cols/128 + cb, and
// one 512-byte scale atom per tile: byte 16*(r % 32) + 4*(r / 32) + b holds
// the scale of tile row r, 32-column block b (the replicated-lane order the
// tensor memory scale copy expects).  One CTA per tile.
__global__ void __launch_bounds__(256)
quantize_weights_mxfp8_kernel(const __nv_bfloat16* __restrict__ src, int rows, int cols,
                              uint8_t* __restrict__ dst_q, uint8_t* __restrict__ dst_sf) {
  pdl_trigger();
  pdl_wait();
  const long long tile = blockIdx.x;
  const int cb_n = cols / 128, rb_n = rows / 128;
  const int cb = (int)(tile % cb_n);
  const long long mr = tile / cb_n;
  const int rb = (int)(mr % rb_n);
  const long long m = mr / rb_n;
  for (int pair = threadIdx.x; pair < 512; pair += blockDim.x) {
    const int r = pair >> 2, blk = pair & 3;
    const uint4* s = reinterpret_cast<const uint4*>(
        src + ((size_t)m * rows + (size_t)rb * 128 + r) * cols + (size_t)cb * 128 + blk * 32);
    uint4 in[4], q[2];
#pragma unroll
    for (int i = 0; i < 4; ++i) in[i] = s[i];
    const int sx = mx_quant_block_bf16(in, q);
    uint4* d = reinterpret_cast<uint4*>(dst_q + (size_t)tile * 16384 + r * 128 + blk * 32);
    d[0] = q[0];
    d[1] = q[1];
    dst_sf[(size_t)tile * 512 + 16 * (r & 31) + 4 * (r >> 5) + blk] = mx_scale_byte(sx);
  }
}

// Dispatch copy with quantisation: one warp per token; lane handles 32-value
// blocks b = lane, lane + 32, ...; every row of the token receives the E4M3
// codes of x[t] (row-major [rows, d] bytes) and the block scales (row-major
// [rows, d/32] bytes).
__global__ void __launch_bounds__(256)
gather_quant_kernel(const __nv_bfloat16* __restrict__ x, const int32_t* __restrict__ slot_pos,
                    int ntok, int K, int d, uint8_t* __restrict__ xq, uint8_t* __restrict__ xsf) {
  pdl_trigger();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t >= ntok) return;
  const int nblk = d / 32;
  for (int kb = 0; kb < K; kb += 32) {
    const int my_row = kb + lane < K ? slot_pos[(size_t)t * K + kb + lane] : -1;
    const uint32_t rows = __ballot_sync(0xffffffffu, my_row >= 0);
    if (!rows) continue;
    for (int b0 = 0; b0 < nblk; b0 += 32) {  // warp-uniform trip count
      const int b = b0 + lane;
      const bool active = b < nblk;
      uint4 q[2] = {};
      uint8_t sb = 0;
      if (active) {
        const uint4* s = reinterpret_cast<const uint4*>(x + (size_t)t * d + b * 32);
        uint4 in[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) in[i] = __ldg(s + i);
        sb = mx_scale_byte(mx_quant_block_bf16(in, q));
      }
      uint32_t has = rows;
      while (has) {
        const int j = __ffs(has) - 1;
        has &= has - 1;
        const int row = __shfl_sync(0xffffffffu, my_row, j);
        if (active) {
          uint4* dq = reinterpret_cast<uint4*>(xq + (size_t)row * d + b * 32);
          dq[0] = q[0];
          dq[1] = q[1];
          xsf[(size_t)row * nblk + b] = sb;
        }
      }
    }
  }
}

}  // namespace moe
