// quant_int8.cuh -- symmetric 8-bit quantisation of Q (per token) and K (per 128-token block)
// for the INT8 QK^T variant of the attention kernel.
//
// The one-pass backend of "TARA: Native Temporal Alignment for MiniMax H3 References"
// (section "Three backends") runs the rule on dense INT8 attention; the page leaves the scaling
// open.  Here: amax = max |x| over the group, inv = 127 / amax, code = rint(x * inv) (float32
// product, ties to even), scale = amax / 127, all float32 with IEEE division; a group with
// amax <= 1e-30 gets codes 0 and scale 0.  The dequantised operand is code * scale.
//
// Both kernels are HBM-bound: each reads its 16-bit operand once and writes half as many bytes
// of codes plus the scales.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

namespace tara {

constexpr float kQ8Max = 127.0f;
constexpr float kQ8AmaxFloor = 1e-30f;
constexpr int kQ8Block = 128;        // K tokens per scale (one key tile)
constexpr int kQ8Threads = 256;

template <bool kBF16>
__device__ __forceinline__ float widen16(uint16_t bits) {
  if (kBF16) return __uint_as_float((uint32_t)bits << 16);
  return __half2float(__ushort_as_half(bits));
}

__device__ __forceinline__ uint32_t q8_code(float x, float inv, bool live) {
  const int c = live ? (int)rintf(__fmul_rn(x, inv)) : 0;
  return (uint32_t)(c & 0xFF);
}

// Q: rows of D (64 or 128) values, 16 bytes (8 values) per lane, so D/8 lanes per row and
// 32/(D/8) rows per warp-wide load; each warp walks kQRowsUnroll such row groups at once, so
// that many 16-byte loads are in flight per lane.  The row amax is a max over the row's lanes
// (shuffles within the lane group).  rows = B*H*N.
constexpr int kQRowsUnroll = 4;

template <bool kBF16, int D>
__global__ void __launch_bounds__(kQ8Threads)
quant_q_kernel(const uint16_t* __restrict__ x, long long rows, int8_t* __restrict__ codes,
               float* __restrict__ scales) {
  constexpr int kLanesPerRow = D / 8;
  constexpr int kRowsPerLoad = 32 / kLanesPerRow;
  constexpr int kRowsPerWarp = kRowsPerLoad * kQRowsUnroll;
  const int lane = threadIdx.x & 31;
  const int sub = lane % kLanesPerRow;          // this lane's 8 values within the row
  const int grp = lane / kLanesPerRow;          // which row of a load group
  const long long warp_row0 =
      ((long long)blockIdx.x * (kQ8Threads / 32) + (threadIdx.x >> 5)) * kRowsPerWarp;
  uint4 raw[kQRowsUnroll];
#pragma unroll
  for (int u = 0; u < kQRowsUnroll; ++u) {
    const long long row = warp_row0 + u * kRowsPerLoad + grp;
    raw[u] = row < rows ? *reinterpret_cast<const uint4*>(x + row * D + sub * 8)
                        : make_uint4(0u, 0u, 0u, 0u);
  }
#pragma unroll
  for (int u = 0; u < kQRowsUnroll; ++u) {
    const long long row = warp_row0 + u * kRowsPerLoad + grp;
    const uint32_t w[4] = {raw[u].x, raw[u].y, raw[u].z, raw[u].w};
    float v[8];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      v[2 * k] = widen16<kBF16>((uint16_t)(w[k] & 0xFFFFu));
      v[2 * k + 1] = widen16<kBF16>((uint16_t)(w[k] >> 16));
    }
    // |x| as bits: non-negative floats order like unsigned integers
    uint32_t am = 0;
#pragma unroll
    for (int k = 0; k < 8; ++k) am = max(am, __float_as_uint(v[k]) & 0x7FFFFFFFu);
#pragma unroll
    for (int o = kLanesPerRow / 2; o > 0; o >>= 1) am = max(am, __shfl_xor_sync(0xffffffffu, am, o));
    const float amax = __uint_as_float(am);
    const bool live = amax > kQ8AmaxFloor;
    const float inv = live ? __fdiv_rn(kQ8Max, amax) : 0.0f;
    uint32_t lo = 0, hi = 0;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      lo |= q8_code(v[k], inv, live) << (8 * k);
      hi |= q8_code(v[4 + k], inv, live) << (8 * k);
    }
    if (row < rows) {
      *reinterpret_cast<uint2*>(codes + row * D + sub * 8) = make_uint2(lo, hi);
      if (sub == 0) scales[row] = live ? __fdiv_rn(amax, kQ8Max) : 0.0f;
    }
  }
}

// K: one CTA per (branch x head, 128-token block).  The block is contiguous in [N][D] memory;
// thread t owns 16-byte chunks t, t + 256, ... (8 values each) and keeps them in registers
// between the block-wide amax and the coding pass.
template <bool kBF16, int D>
__global__ void __launch_bounds__(kQ8Threads)
quant_k_kernel(const uint16_t* __restrict__ x, int N, int nblocks, int8_t* __restrict__ codes,
               float* __restrict__ scales) {
  constexpr int kMaxChunks = kQ8Block * D / 8 / kQ8Threads;   // 8 (D=128) or 4 (D=64)
  const int blk = blockIdx.x, bh = blockIdx.y;
  const int r0 = blk * kQ8Block;
  const int nrows = min(kQ8Block, N - r0);
  const int nchunks = nrows * D / 8;
  const long long base = ((long long)bh * N + r0) * D;
  const uint4* src = reinterpret_cast<const uint4*>(x + base);

  uint4 raw[kMaxChunks];
  uint32_t am = 0;
#pragma unroll
  for (int i = 0; i < kMaxChunks; ++i) {
    const int c = threadIdx.x + i * kQ8Threads;
    raw[i] = c < nchunks ? src[c] : make_uint4(0u, 0u, 0u, 0u);
    const uint32_t w[4] = {raw[i].x, raw[i].y, raw[i].z, raw[i].w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      am = max(am, __float_as_uint(widen16<kBF16>((uint16_t)(w[k] & 0xFFFFu))) & 0x7FFFFFFFu);
      am = max(am, __float_as_uint(widen16<kBF16>((uint16_t)(w[k] >> 16))) & 0x7FFFFFFFu);
    }
  }
  am = __reduce_max_sync(0xffffffffu, am);
  __shared__ uint32_t warp_am[kQ8Threads / 32];
  if ((threadIdx.x & 31) == 0) warp_am[threadIdx.x >> 5] = am;
  __syncthreads();
  am = 0;
#pragma unroll
  for (int w = 0; w < kQ8Threads / 32; ++w) am = max(am, warp_am[w]);
  const float amax = __uint_as_float(am);
  const bool live = amax > kQ8AmaxFloor;
  const float inv = live ? __fdiv_rn(kQ8Max, amax) : 0.0f;

  uint2* dst = reinterpret_cast<uint2*>(codes + base);
#pragma unroll
  for (int i = 0; i < kMaxChunks; ++i) {
    const int c = threadIdx.x + i * kQ8Threads;
    if (c >= nchunks) break;
    const uint32_t w[4] = {raw[i].x, raw[i].y, raw[i].z, raw[i].w};
    uint32_t out[2] = {0u, 0u};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const uint32_t lo = q8_code(widen16<kBF16>((uint16_t)(w[k] & 0xFFFFu)), inv, live);
      const uint32_t hi = q8_code(widen16<kBF16>((uint16_t)(w[k] >> 16)), inv, live);
      out[k >> 1] |= (lo | (hi << 8)) << (16 * (k & 1));
    }
    dst[c] = make_uint2(out[0], out[1]);
  }
  if (threadIdx.x == 0) scales[(long long)bh * nblocks + blk] = live ? __fdiv_rn(amax, kQ8Max) : 0.0f;
}

}  // namespace tara
