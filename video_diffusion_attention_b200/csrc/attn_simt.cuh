// attn_simt.cuh -- the exact CUDA-core path: the biased attention forward in fp32 FFMA.
//
// Used for fp32 inputs, where tensor-core tf32 rounding would not meet a 1e-5 bound.  One warp
// owns one query row; the CTA's four warps share 32-key chunks of K and V staged in shared
// memory.  Lane j scores key j of the chunk; the chunk max and sum are combined across the
// warp with shuffles (online softmax), and lane c accumulates output dims c, c+32, ...
#pragma once

#include "tara_common.cuh"

namespace tara {

constexpr int kSimtRows = 4;     // query rows (warps) per CTA
constexpr int kSimtChunk = 32;   // keys per shared-memory chunk
constexpr int kSimtMaxD = 256;

__global__ void __launch_bounds__(kSimtRows * 32)
attn_simt_kernel(const float* __restrict__ Q, const float* __restrict__ K,
                 const float* __restrict__ V, float* __restrict__ O, float* __restrict__ LSE,
                 const uint8_t* __restrict__ seg, const float* __restrict__ time_s,
                 const uint8_t* __restrict__ pic, const float* __restrict__ mw,
                 long long batch_stride, int H, int N, int D, BiasParams bp, ExtraMasks xm,
                 int* status) {
  extern __shared__ float smem[];
  const int ld = D + 1;                           // padded row: conflict-free column reads
  float* sK = smem;                               // [chunk][ld]
  float* sV = sK + kSimtChunk * ld;               // [chunk][ld]
  float* sQ = sV + kSimtChunk * ld;               // [rows][D]

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int h = blockIdx.y, b = blockIdx.z;
  const long long head = ((long long)b * H + h) * (long long)N * D;
  const long long mb = (long long)b * batch_stride;
  const int row = blockIdx.x * kSimtRows + warp;
  const bool row_ok = row < N;

  // this row's query vector and metadata
  for (int c = lane; c < D; c += 32) sQ[warp * D + c] = row_ok ? Q[head + (long long)row * D + c] : 0.0f;
  const bool tgt = row_ok && seg[mb + row] == kSegTarget;
  const float t_q = row_ok ? time_s[mb + row] : 0.0f;
  const float m_q = row_ok ? mw[mb + row] : 0.0f;
  // debug build: a target row's time and mask weight are finite numbers
  if (lane == 0) TARA_DCHECK_RECORD(!tgt || (isfinite(t_q) && isfinite(m_q)), status);

  const float ninf = __int_as_float(0xff800000);
  float m_run = ninf, l_run = 0.0f;
  float acc[kSimtMaxD / 32];
#pragma unroll
  for (int i = 0; i < kSimtMaxD / 32; ++i) acc[i] = 0.0f;

  for (int k0 = 0; k0 < N; k0 += kSimtChunk) {
    __syncthreads();
    const int nk = min(kSimtChunk, N - k0);
    for (int e = threadIdx.x; e < kSimtChunk * D; e += blockDim.x) {
      int r = e / D, c = e - r * D;
      float kv = 0.0f, vv = 0.0f;
      if (r < nk) {
        kv = K[head + (long long)(k0 + r) * D + c];
        vv = V[head + (long long)(k0 + r) * D + c];
      }
      sK[r * ld + c] = kv;
      sV[r * ld + c] = vv;
    }
    __syncthreads();
    if (!row_ok) continue;

    // lane scores key k0 + lane
    float x = ninf;
    if (lane < nk) {
      float dot = 0.0f;
      for (int c = 0; c < D; ++c) dot = fmaf(sQ[warp * D + c], sK[lane * ld + c], dot);
      float bias = 0.0f;
      if (tgt) {
        const int j = k0 + lane;
        const int sj = seg[mb + j];
        if (sj == kSegGuide) {
          bias = -penalty_f32(fabsf(t_q - time_s[mb + j]), bp);
        } else if (sj == kSegPicture) {
          const int pj = pic[mb + j];
          bias = m_q * (pj < 16 ? bp.lng[pj] : 0.0f);
          for (int k = 0; k < bp.n_extra; ++k)
            bias += xm.m[k * xm.stride + mb + row] * (pj < 16 ? bp.lng_x[k][pj] : 0.0f);
        }
      }
      x = fmaf(dot, bp.scale_log2, bias * kLog2e);   // log2 units
    }
    // online softmax across the warp
    float cmax = x;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) cmax = fmaxf(cmax, __shfl_xor_sync(0xffffffffu, cmax, o));
    const float m_new = fmaxf(m_run, cmax);
    const float alpha = exp2f(m_run - m_new);     // 0 on the first chunk
    const float p = exp2f(x - m_new);
    float psum = p;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) psum += __shfl_xor_sync(0xffffffffu, psum, o);
    l_run = l_run * alpha + psum;
    m_run = m_new;
#pragma unroll
    for (int i = 0; i < kSimtMaxD / 32; ++i) acc[i] *= alpha;
    for (int j = 0; j < nk; ++j) {
      const float pj = __shfl_sync(0xffffffffu, p, j);
#pragma unroll
      for (int i = 0; i < kSimtMaxD / 32; ++i) {
        const int c = lane + 32 * i;
        if (c < D) acc[i] = fmaf(pj, sV[j * ld + c], acc[i]);
      }
    }
  }
  if (!row_ok) return;
  const float inv_l = 1.0f / l_run;
#pragma unroll
  for (int i = 0; i < kSimtMaxD / 32; ++i) {
    const int c = lane + 32 * i;
    if (c < D) O[head + (long long)row * D + c] = acc[i] * inv_l;
  }
  if (lane == 0) LSE[((long long)b * H + h) * N + row] = (m_run + log2f(l_run)) * kLn2;
}

}  // namespace tara
