// tile_summary.cuh -- per-tile summaries and per-key bias records of the packed sequence.
//
// One CTA of 128 threads per (metadata set, 128-token tile).  Thread t reads token
// tile*128 + t once and the CTA reduces role bits, Picture bits and the min/max times of the
// TARGET and GUIDE tokens with warp shuffles, then combines the four warps in shared memory.
// The attention kernels classify every (query tile, key tile) pair from two of these records
// instead of evaluating the bias on every edge.
//
// Layout (nsets = gridDim.y metadata sets): recs[set * ntiles + tile] and
// keyinfo[set * ntiles * 128 + tok] in ascending tile order, the key records past the
// sequence's end zero; then the same records with the tile order reversed, at
// recs[(nsets + set) * ntiles + ntiles - 1 - tile] and
// keyinfo[(nsets + set) * ntiles * 128 + (ntiles - 1 - tile) * 128 + t], for work that walks
// the keys from the last tile to the first.
#pragma once

#include "tara_common.cuh"

namespace tara {

__global__ void __launch_bounds__(128)
tile_summary_kernel(const uint8_t* __restrict__ seg, const float* __restrict__ time_s,
                    const uint8_t* __restrict__ pic, int N, long long batch_stride, int ntiles,
                    BiasParams bp, TileRec* __restrict__ recs, float4* __restrict__ keyinfo,
                    int* status) {
  const int tile = blockIdx.x;
  const int set = blockIdx.y;
  const int t = threadIdx.x;
  const int lane = t & 31, warp = t >> 5;
  const long long base = (long long)set * batch_stride;
  const int tok = tile * kTile + t;
  const bool valid = tok < N;

  uint32_t s = 0, pc = 0;
  float tm = 0.0f;
  if (valid) {
    s = seg[base + tok];
    tm = time_s[base + tok];
    pc = pic[base + tok];
    // debug build: the clock of every target and guide token is a finite number
    TARA_DCHECK_RECORD(!(s == kSegTarget || s == kSegGuide) || isfinite(tm), status);
  }
  const float inf = __int_as_float(0x7f800000);
  float tq_lo = (valid && s == kSegTarget) ? tm : inf;
  float tq_hi = (valid && s == kSegTarget) ? tm : -inf;
  float tk_lo = (valid && s == kSegGuide) ? tm : inf;
  float tk_hi = (valid && s == kSegGuide) ? tm : -inf;
  uint32_t segbit = valid ? (1u << (s <= 5u ? s : 31u)) : 0u;   // unknown roles: bit 31
  uint32_t picbit = (valid && s == kSegPicture && pc < 32) ? (1u << pc) : 0u;
  // all-same-picture test: every valid token PICTURE with the same index
  uint32_t pic_or_any = (valid && s == kSegPicture) ? pc : 0xFFu;

  // per-key record (the key side of the bias); zero for positions past the end
  const int nsets = (int)gridDim.y;
  const long long kstride = (long long)ntiles * kTile;
  {
    float4 rec = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    if (valid && s == kSegGuide) {
      rec.x = tm;
      rec.z = 1.0f;
    } else if (valid && s == kSegPicture && pc < 16 && ((bp.lng_nz >> pc) & 1u)) {
      rec.y = bp.lng[pc];
      rec.w = (float)pc;
    }
    keyinfo[(long long)set * kstride + tok] = rec;
    keyinfo[(long long)(nsets + set) * kstride + (long long)(ntiles - 1 - tile) * kTile + t] = rec;
  }

#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    tq_lo = fminf(tq_lo, __shfl_xor_sync(0xffffffffu, tq_lo, o));
    tq_hi = fmaxf(tq_hi, __shfl_xor_sync(0xffffffffu, tq_hi, o));
    tk_lo = fminf(tk_lo, __shfl_xor_sync(0xffffffffu, tk_lo, o));
    tk_hi = fmaxf(tk_hi, __shfl_xor_sync(0xffffffffu, tk_hi, o));
  }
  segbit = __reduce_or_sync(0xffffffffu, segbit);
  picbit = __reduce_or_sync(0xffffffffu, picbit);
  const uint32_t pmin = __reduce_min_sync(0xffffffffu, valid ? pic_or_any : 0xFFFFFFFFu);
  const uint32_t pmax = __reduce_max_sync(0xffffffffu, valid ? pic_or_any : 0u);
  const uint32_t nval = __popc(__ballot_sync(0xffffffffu, valid));

  __shared__ float sh_f[4][4];
  __shared__ uint32_t sh_u[4][5];
  if (lane == 0) {
    sh_f[warp][0] = tq_lo;
    sh_f[warp][1] = tq_hi;
    sh_f[warp][2] = tk_lo;
    sh_f[warp][3] = tk_hi;
    sh_u[warp][0] = segbit;
    sh_u[warp][1] = picbit;
    sh_u[warp][2] = nval ? pmin : 0xFFFFFFFFu;   // warps without valid tokens are neutral
    sh_u[warp][3] = nval ? pmax : 0u;
    sh_u[warp][4] = nval;
  }
  __syncthreads();
  if (t == 0) {
    TileRec r;
    r.tq_min = fminf(fminf(sh_f[0][0], sh_f[1][0]), fminf(sh_f[2][0], sh_f[3][0]));
    r.tq_max = fmaxf(fmaxf(sh_f[0][1], sh_f[1][1]), fmaxf(sh_f[2][1], sh_f[3][1]));
    r.tk_min = fminf(fminf(sh_f[0][2], sh_f[1][2]), fminf(sh_f[2][2], sh_f[3][2]));
    r.tk_max = fmaxf(fmaxf(sh_f[0][3], sh_f[1][3]), fmaxf(sh_f[2][3], sh_f[3][3]));
    r.segmask = sh_u[0][0] | sh_u[1][0] | sh_u[2][0] | sh_u[3][0];
    r.picmask = sh_u[0][1] | sh_u[1][1] | sh_u[2][1] | sh_u[3][1];
    uint32_t lo = min(min(sh_u[0][2], sh_u[1][2]), min(sh_u[2][2], sh_u[3][2]));
    uint32_t hi = max(max(sh_u[0][3], sh_u[1][3]), max(sh_u[2][3], sh_u[3][3]));
    r.nvalid = sh_u[0][4] + sh_u[1][4] + sh_u[2][4] + sh_u[3][4];
    r.single_pic = (r.segmask == (1u << kSegPicture) && lo == hi && lo >= 1 && lo <= 9) ? lo : 0u;
    recs[(long long)set * ntiles + tile] = r;
    recs[(long long)(nsets + set) * ntiles + (ntiles - 1 - tile)] = r;
  }
}

}  // namespace tara
