// target_mask.cuh -- target-mask preparation on the device: a soft pixel mask (one frame, or
// one per frame of the prepared shot) becomes one weight per target token, the value the
// attention kernels read as m ("BFS H3 Reference Attention Binding (Experimental)": masks are
// area-downsampled to the target's patch resolution and averaged across the latent temporal
// spans).
//
// One CTA per (patch row y, latent frame f).  Its threads own pixel columns (thread t: columns
// t, t + 256, ...), so every load of a pixel row is coalesced and each thread has many
// independent loads in flight: per column they sum the pixels of the cell row's pixel rows
// (weighted by each row's overlap with the cell row) over the latent frame's pixel frames.
// The column sums are then added into the cells they overlap (shared-memory accumulators)
// and normalised.  Overlaps are integers in units of 1/Hq pixel (rows) and 1/Wq pixel
// (columns), so the area weights are exact.  HBM-bound: each pixel is read once (twice for a
// pixel row straddling two cell rows).
#pragma once

#include <cstdint>

namespace tara {

constexpr int kMaskThreads = 256;
constexpr int kMaskColsPerPass = 8;   // columns per thread per pass (register sums)

__global__ void __launch_bounds__(kMaskThreads)
target_mask_kernel(const float* __restrict__ mask, int F_in, int Hp, int Wp, int L, int tau,
                   int F_lat, int Hq, int Wq, float* __restrict__ out) {
  extern __shared__ float cell_acc[];   // [Wq]
  const int y = blockIdx.x;
  const int f = blockIdx.y;             // latent frame (0 when one static mask)
  const int tid = threadIdx.x;

  for (int x = tid; x < Wq; x += kMaskThreads) cell_acc[x] = 0.0f;
  __syncthreads();

  // pixel rows overlapping cell row y: [y*Hp, (y+1)*Hp) in units of 1/Hq pixel
  const long long ylo = (long long)y * Hp, yhi = (long long)(y + 1) * Hp;
  const int r0 = (int)(ylo / Hq);
  const int r1 = (int)((yhi + Hq - 1) / Hq);          // exclusive
  int t0 = 0, t1 = 1;
  if (F_in > 1) {
    t0 = f * tau;
    t1 = min(t0 + tau, L);
  }

  // columns are handled in groups of 4 (one 16-byte load per pixel row) when every row starts
  // on a 16-byte boundary, else one at a time
  const bool vec4 = (Wp % 4 == 0) && ((reinterpret_cast<uintptr_t>(mask) & 15u) == 0);
  // a pass covers 2048 columns: 8 register sums per thread (2 x 4 columns, or 8 x 1)
  constexpr int kSlots = kMaskColsPerPass;
  for (int base = 0; base < Wp; base += kMaskThreads * kSlots) {
    float colsum[kSlots];
#pragma unroll
    for (int k = 0; k < kSlots; ++k) colsum[k] = 0.0f;
    for (int t = t0; t < t1; ++t) {
#pragma unroll 2
      for (int r = r0; r < r1; ++r) {
        const long long rlo = (long long)r * Hq;
        const float wy = (float)(min(yhi, rlo + Hq) - max(ylo, rlo));
        const float* row = mask + ((long long)t * Hp + r) * Wp;
        if (vec4) {
#pragma unroll
          for (int k = 0; k < 2; ++k) {
            const int c = base + (k * kMaskThreads + tid) * 4;
            if (c < Wp) {
              const float4 v = __ldg(reinterpret_cast<const float4*>(row + c));
              colsum[4 * k + 0] = fmaf(wy, v.x, colsum[4 * k + 0]);
              colsum[4 * k + 1] = fmaf(wy, v.y, colsum[4 * k + 1]);
              colsum[4 * k + 2] = fmaf(wy, v.z, colsum[4 * k + 2]);
              colsum[4 * k + 3] = fmaf(wy, v.w, colsum[4 * k + 3]);
            }
          }
        } else {
#pragma unroll
          for (int k = 0; k < kSlots; ++k) {
            const int c = base + k * kMaskThreads + tid;
            if (c < Wp) colsum[k] = fmaf(wy, __ldg(row + c), colsum[k]);
          }
        }
      }
    }
    // add each column sum into the cells the column overlaps, weighted by the overlap
#pragma unroll
    for (int k = 0; k < kSlots; ++k) {
      const int c = vec4 ? base + ((k >> 2) * kMaskThreads + tid) * 4 + (k & 3)
                         : base + k * kMaskThreads + tid;
      if (c >= Wp) continue;
      const long long clo = (long long)c * Wq, chi = clo + Wq;
      for (int x = (int)(clo / Wp); x < Wq && (long long)x * Wp < chi; ++x) {
        const long long xlo = (long long)x * Wp;
        const float wx = (float)(min(xlo + Wp, chi) - max(xlo, clo));
        atomicAdd(&cell_acc[x], wx * colsum[k]);
      }
    }
  }
  __syncthreads();

  const float norm = 1.0f / ((float)Hp * (float)Wp * (float)(t1 - t0));
  for (int x = tid; x < Wq; x += kMaskThreads) {
    const float v = cell_acc[x] * norm;
    if (F_in > 1) {
      out[((long long)f * Hq + y) * Wq + x] = v;
    } else {
      for (int ff = 0; ff < F_lat; ++ff) out[((long long)ff * Hq + y) * Wq + x] = v;
    }
  }
}

// Adds the weighted column sums of pixel columns c..c+3 into the cells they overlap.
__device__ __forceinline__ void add_column_group(float* cell_acc, float4 cs, int c, int Wp,
                                                 int Wq) {
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const float vk = k == 0 ? cs.x : k == 1 ? cs.y : k == 2 ? cs.z : cs.w;
    const long long clo = (long long)(c + k) * Wq, chi = clo + Wq;
    for (int x = (int)(clo / Wp); x < Wq && (long long)x * Wp < chi; ++x) {
      const long long xlo = (long long)x * Wp;
      const float wx = (float)(min(xlo + Wp, chi) - max(xlo, clo));
      atomicAdd(&cell_acc[x], wx * vk);
    }
  }
}

// Narrow rows (Wp <= 1024, every pixel row 16-byte aligned): 128 threads, thread t owns the
// 16-byte column groups t and t + 128 (one load each per pixel row), so a CTA needs few
// registers and the whole grid of a shot is resident at once.  The (pixel frame, pixel row)
// pairs of the cell row are walked with an incremented index pair (no division in the loop),
// four at a time, so eight loads are in flight per thread.
constexpr int kMaskNarrowThreads = 128;

__global__ void __launch_bounds__(kMaskNarrowThreads)
target_mask_narrow_kernel(const float* __restrict__ mask, int F_in, int Hp, int Wp, int L,
                          int tau, int F_lat, int Hq, int Wq, float* __restrict__ out) {
  extern __shared__ float cell_acc[];   // [Wq]
  const int y = blockIdx.x;
  const int f = blockIdx.y;
  const int tid = threadIdx.x;
  for (int x = tid; x < Wq; x += kMaskNarrowThreads) cell_acc[x] = 0.0f;
  __syncthreads();

  const long long ylo = (long long)y * Hp, yhi = (long long)(y + 1) * Hp;
  const int r0 = (int)(ylo / Hq);
  const int r1 = (int)((yhi + Hq - 1) / Hq);
  int t0 = 0, t1 = 1;
  if (F_in > 1) {
    t0 = f * tau;
    t1 = min(t0 + tau, L);
  }
  const int npairs = (t1 - t0) * (r1 - r0);
  const int c0 = tid * 4, c1 = (tid + kMaskNarrowThreads) * 4;
  const bool has1 = c1 < Wp;
  float4 a0 = make_float4(0.0f, 0.0f, 0.0f, 0.0f), a1 = a0;
  if (c0 < Wp) {
    int t = t0, r = r0;
#pragma unroll 4
    for (int i = 0; i < npairs; ++i) {
      const long long rlo = (long long)r * Hq;
      const float wy = (float)(min(yhi, rlo + Hq) - max(ylo, rlo));
      const float* row = mask + ((long long)t * Hp + r) * Wp;
      const float4 v = __ldg(reinterpret_cast<const float4*>(row + c0));
      a0.x = fmaf(wy, v.x, a0.x);
      a0.y = fmaf(wy, v.y, a0.y);
      a0.z = fmaf(wy, v.z, a0.z);
      a0.w = fmaf(wy, v.w, a0.w);
      if (has1) {
        const float4 u = __ldg(reinterpret_cast<const float4*>(row + c1));
        a1.x = fmaf(wy, u.x, a1.x);
        a1.y = fmaf(wy, u.y, a1.y);
        a1.z = fmaf(wy, u.z, a1.z);
        a1.w = fmaf(wy, u.w, a1.w);
      }
      if (++r == r1) {
        r = r0;
        ++t;
      }
    }
    add_column_group(cell_acc, a0, c0, Wp, Wq);
    if (has1) add_column_group(cell_acc, a1, c1, Wp, Wq);
  }
  __syncthreads();

  const float norm = 1.0f / ((float)Hp * (float)Wp * (float)(t1 - t0));
  for (int x = tid; x < Wq; x += kMaskNarrowThreads) {
    const float v = cell_acc[x] * norm;
    if (F_in > 1) {
      out[((long long)f * Hq + y) * Wq + x] = v;
    } else {
      for (int ff = 0; ff < F_lat; ++ff) out[((long long)ff * Hq + y) * Wq + x] = v;
    }
  }
}

}  // namespace tara
