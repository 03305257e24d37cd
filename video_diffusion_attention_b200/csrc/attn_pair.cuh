// attn_pair.cuh -- the tensor-core path on SM pairs: 2-SM tcgen05 MMA, S double-buffered.
//
// A cluster of two CTAs (an SM pair) owns 256 query rows of one (branch, head): 128 per CTA.
// The even CTA issues every MMA with cta_group::2, M = 256: each CTA supplies its 128 rows of
// Q (and of P), and half of each B operand -- K rows [64r, 64r+64) of a key tile for S = Q K^T,
// and V columns [64r, 64r+64) of a value tile for O += P V (r = the CTA's rank in the pair).
// S, P and O of a CTA's rows live in its own tensor memory: S in two 128-column buffers
// (tile j in buffer j&1), O in columns 256..383.  Because S is double-buffered, the MMA for
// S_{j+1} runs while the softmax warps work on S_j; only the PV product waits for P_j.
//
// Warp roles in each CTA (384 threads):
//   warps 0-3  softmax, key columns 0..63 of every tile (thread = row = TMEM lane)
//   warps 4-7  softmax, key columns 64..127 (same rows as warps 0-3)
//   warp  8    TMA producer: this CTA's halves of Q, K_j, V_j (completion counted on the
//              even CTA's barriers)
//   warp  9    MMA issuer in the even CTA; tensor-memory allocation in both
//   warps 10-11 idle
// The two softmax warpgroups exchange their row maxima (and, at the end, row sums) through
// shared memory; both then hold the same running max, so their rescaling decisions agree.
// P_j is written over columns 0..63 of its S buffer (warpgroup w: columns 32w..32w+31) after
// both groups have loaded their S columns.
//
// Bias: same exact tile classes as the single-SM kernel (tara_common.cuh), per-edge tiles
// staged in shared memory and evaluated branch-free.  Every wait is bounded.
#pragma once

#include "attn_tc.cuh"
#include "sm100_ptx.cuh"
#include "tara_common.cuh"

namespace tara {

struct PairShape {
  static constexpr int D = 128;
  static constexpr int kQBytes = kTile * D * 2;       // 32 KB: two 16 KB panels (128 rows x 128 B)
  static constexpr int kHalfBytes = 16384;            // K half: 64 keys x 128 d (two 8 KB panels)
                                                      // V half: 128 keys x 64 d (one panel)
  static constexpr int kStages = 8;                   // ring slots (K_j and V_j alternate)
  static constexpr int kKeyBufBytes = 2 * kTile * 16; // [parity][key] float4
  static constexpr int kRowWBytes = kTile * 17 * 4;   // [row] extra-binding weights
  static constexpr int kXchgBytes = 2 * 2 * kTile * 4 + 2 * kTile * 4;  // max [par][wg][row], sum
  static constexpr int kBarCount = 1 + 2 * kStages + 2 + 2 + 1 + 1 + 1 + 4 + 1;
  static constexpr int kSmemBytes = 1024 + kQBytes + kStages * kHalfBytes + kKeyBufBytes +
                                    kRowWBytes + kXchgBytes + kBarCount * 8 + 16;
  static constexpr uint32_t kColO = 256;
};

// Max of 64 row values as 8 chains and a tree.
__device__ __forceinline__ float row_max64(const uint32_t (&s)[64]) {
  float a[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) a[i] = __uint_as_float(s[i]);
#pragma unroll
  for (int c = 8; c < 64; ++c) a[c & 7] = fmaxf(a[c & 7], __uint_as_float(s[c]));
  return fmaxf(fmaxf(fmaxf(a[0], a[1]), fmaxf(a[2], a[3])), fmaxf(fmaxf(a[4], a[5]), fmaxf(a[6], a[7])));
}

template <bool kBF16>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(384, 1)
attn_pair_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                 const __grid_constant__ CUtensorMap tmV, const TcArgs args) {
  using S = PairShape;
  constexpr int NS = S::kStages;
  constexpr int HB = S::kHalfBytes;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sKV = smem + S::kQBytes;
  float4* kbuf = reinterpret_cast<float4*>(sKV + NS * HB);
  float* rowx = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(kbuf) + S::kKeyBufBytes);
  float* xmax = rowx + kTile * 17;
  float* xsum = xmax + 2 * 2 * kTile;
  uint64_t* bars = reinterpret_cast<uint64_t*>(xsum + 2 * kTile);
  uint64_t* q_full = bars;
  uint64_t* kv_full = bars + 1;
  uint64_t* kv_empty = kv_full + NS;
  uint64_t* s_full = kv_empty + NS;     // [2] per S buffer
  uint64_t* p_full = s_full + 2;        // [2] per S buffer, 16 arrivals (8 warps x 2 CTAs)
  uint64_t* pv_done = p_full + 2;
  uint64_t* drain = pv_done + 1;
  uint64_t* exit_bar = drain + 1;
  uint64_t* xbar = exit_bar + 1;        // [4] per row quarter: warps q and q+4
  uint64_t* stage_bar = xbar + 4;       // the 8 softmax warps
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(stage_bar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int N = args.N;
  const int bh = blockIdx.z * args.H + blockIdx.y;
  const int qtile = blockIdx.x;
  const int nk = (N + kTile - 1) / kTile;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&p_full[b], 16);
    }
    mbar_init(pv_done, 1);
    mbar_init(drain, 1);
    mbar_init(exit_bar, 1);
    for (int q = 0; q < 4; ++q) mbar_init(&xbar[q], 2);
    mbar_init(stage_bar, 8);
    *abort_flag = 0;
    fence_mbar_init();
  }
  cluster_sync_all();
  // one decision for both CTAs: skip all work if an earlier CTA of this launch gave up
  if (threadIdx.x == 0 && leader) {
    const int st = *reinterpret_cast<volatile int*>(args.status) != 0 ? 1 : 0;
    const uint32_t peer_flag = mapa_shared(smem_u32((const void*)abort_flag), 1);
    *abort_flag = st;
    asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(peer_flag), "r"(st) : "memory");
  }
  cluster_sync_all();
  if (*abort_flag) return;

  if (warp == 9) {
    tmem_alloc_pair(tmem_slot, 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp >= 8) {
    if (warp == 8 && lane == 0) {
      // ------------------------------ TMA producer (both CTAs) -------------------------
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      const uint32_t q_full_l = mapa_shared(smem_u32(q_full), 0);
      if (leader) mbar_arrive_expect_tx(q_full, 2 * S::kQBytes);
      for (int p = 0; p < 2; ++p)
        tma_load_3d_pair(sQ + p * (kTile * 128), &tmQ, q_full_l, p * 64, qtile * kTile, bh);
      int issued = 0;
      for (int i = 0; i < 2 * nk; ++i) {
        const int slot = i % NS;
        const uint32_t ph = (uint32_t)(i / NS) & 1u;
        if (!mbar_wait_cluster(&kv_empty[slot], ph ^ 1u, abort_flag, kWaitLimitNs)) break;
        if (leader) mbar_arrive_expect_tx(&kv_full[slot], 2 * HB);
        const uint32_t full_l = mapa_shared(smem_u32(&kv_full[slot]), 0);
        uint8_t* dst = sKV + slot * HB;
        const int j = i >> 1;
        if ((i & 1) == 0) {
          // K_j rows [64r, 64r+64): two 64-row x 128-byte panels
          for (int p = 0; p < 2; ++p)
            tma_load_3d_pair(dst + p * (64 * 128), &tmK, full_l, p * 64, j * kTile + (int)rank * 64, bh);
        } else {
          // V_j columns [64r, 64r+64): one 128-row x 128-byte panel
          tma_load_3d_pair(dst, &tmV, full_l, (int)rank * 64, j * kTile, bh);
        }
        issued = i + 1;
      }
      if (*abort_flag && issued > 0) {
        // copies already issued land within microseconds; give them 1 ms before this CTA's
        // shared memory can be released (their completion is counted in the even CTA)
        for (int k = 0; k < 1000; ++k) __nanosleep(1000);
      }
    } else if (warp == 9 && lane == 0 && leader) {
      // ------------------------------ MMA issuer (even CTA) ----------------------------
      constexpr uint32_t idesc_qk = make_idesc_f16(256, 128, kBF16, false);
      constexpr uint32_t idesc_pv = make_idesc_f16(256, 128, kBF16, true);
      const uint64_t qd0 = make_sdesc_sw128(smem_u32(sQ), 16, 1024);
      const uint64_t kd0 = make_sdesc_sw128(smem_u32(sKV), 16, 1024);
      const uint64_t vd0 = make_sdesc_sw128(smem_u32(sKV), 16384, 1024);
      bool ok = mbar_wait_cluster(q_full, 0, abort_flag, kWaitLimitNs);
      tc_fence_after();
      for (int j = 0; ok && j <= nk; ++j) {
        if (j < nk) {
          // S_j into buffer j&1 (its previous P was read by PV_{j-2}, issued earlier)
          const int i = 2 * j, slot = i % NS;
          if (!(ok = mbar_wait_cluster(&kv_full[slot], (uint32_t)(i / NS) & 1u, abort_flag, kWaitLimitNs))) break;
          tc_fence_after();
          const uint32_t d_s = tmem + (uint32_t)((j & 1) * 128);
          const uint64_t kd = kd0 + (uint64_t)((slot * HB) >> 4);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint64_t qoff = (uint64_t)((((kk >> 2) * (kTile * 128)) + (kk & 3) * 32) >> 4);
            const uint64_t koff = (uint64_t)((((kk >> 2) * (64 * 128)) + (kk & 3) * 32) >> 4);
            umma_ss_pair(d_s, qd0 + qoff, kd + koff, idesc_qk, kk > 0 ? 1u : 0u);
          }
          umma_commit_pair(&s_full[j & 1]);
          umma_commit_pair(&kv_empty[slot]);
        }
        if (j >= 1) {
          // O += P_{j-1} V_{j-1}
          const int jj = j - 1;
          const int i = 2 * jj + 1, slot = i % NS;
          if (!(ok = mbar_wait_cluster(&kv_full[slot], (uint32_t)(i / NS) & 1u, abort_flag, kWaitLimitNs))) break;
          if (!(ok = mbar_wait_cluster(&p_full[jj & 1], (uint32_t)(jj >> 1) & 1u, abort_flag, kWaitLimitNs))) break;
          tc_fence_after();
          const uint32_t a_p = tmem + (uint32_t)((jj & 1) * 128);
          const uint64_t vd = vd0 + (uint64_t)((slot * HB) >> 4);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            umma_ts_pair(tmem + S::kColO, a_p + kk * 8, vd + (uint64_t)((kk * 2048) >> 4), idesc_pv,
                         (jj > 0 || kk > 0) ? 1u : 0u);
          umma_commit_pair(pv_done);
          umma_commit_pair(&kv_empty[slot]);
        }
      }
      umma_commit_pair(drain);
      volatile int no_abort = 0;
      mbar_wait_cluster(drain, 0, &no_abort, kDrainLimitNs);
    }
  } else {
    // ------------------------------ softmax warps ------------------------------------
    const int wg = warp >> 2;           // 0: key columns 0..63, 1: columns 64..127
    const int wq = warp & 3;            // TMEM lane quarter
    const int r = wq * 32 + lane;       // row within the tile
    const int row = qtile * kTile + r;
    const bool row_ok = (qtile < args.ntiles) && (row < N);
    const BiasParams& bp = args.bp;
    const int mset = args.per_branch_meta ? blockIdx.z : 0;
    const long long mtok = (long long)mset * args.meta_stride;
    const TileRec* recs = args.recs + (long long)mset * args.ntiles;
    const float4* kinfo = args.keyinfo + (long long)mset * N;
    const uint32_t p_full_l[2] = {mapa_shared(smem_u32(&p_full[0]), 0),
                                  mapa_shared(smem_u32(&p_full[1]), 0)};

    bool is_tgt = false;
    float t_q = 0.0f, m_q = 0.0f;
    if (row_ok) {
      is_tgt = args.seg[mtok + row] == kSegTarget;
      t_q = args.time_s[mtok + row];
      m_q = args.m[mtok + row];
    }
    // weights of the extra bindings for this row, one per Picture index (0 for index 0)
    float* wx = rowx + r * 17;
    if (bp.n_extra > 0) {
      for (int pidx = 0; pidx < 16; ++pidx) {
        float acc = 0.0f;
        if (is_tgt)
          for (int k = 0; k < bp.n_extra; ++k)
            acc += args.xm.m[k * args.xm.stride + mtok + row] * bp.lng_x[k][pidx];
        wx[pidx] = acc;
      }
    }
    TileRec qr;
    if (qtile < args.ntiles) {
      qr = recs[qtile];
    } else {
      qr.segmask = 0;
      qr.picmask = 0;
      qr.nvalid = 0;
      qr.single_pic = 0;
      qr.tq_min = qr.tk_min = 0.0f;
      qr.tq_max = qr.tk_max = 0.0f;
    }
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    const uint32_t tO = tmem + lane_off + S::kColO + wg * 64;
    const float ninf = __int_as_float(0xff800000);
    float m_run = ninf, l_run = 0.0f;
    bool ok = true;
    const int col0 = wg * 64;            // first key column of this group

    uint32_t stage_phase = 0, x_phase = 0;
    TileRec kr_next = recs[0];
    for (int j = 0; j < nk; ++j) {
      const TileRec kr = kr_next;
      if (j + 1 < nk) kr_next = recs[j + 1];
      float cval;
      const int cls = classify_pair(qr, kr, bp, &cval);
      float rowb2 = 0.0f;
      if (is_tgt) {
        if (cls == kClsConstCap) rowb2 = cval * kLog2e;
        else if (cls == kClsRowGuide) rowb2 = -penalty_f32(fabsf(t_q - kr.tk_min), bp) * kLog2e;
        else if (cls == kClsConstPic)
          rowb2 = (bp.n_extra > 0 ? m_q * cval + wx[kr.single_pic & 15] : m_q * cval) * kLog2e;
      }
      float4* kb = kbuf + (j & 1) * kTile;
      if (cls == kClsFull) {
        // both groups stage the 128 key records, double-buffered by tile parity
        const int tid = wg * 128 + r;
        if (tid < kTile) {
          const int key = j * kTile + tid;
          kb[tid] = key < N ? kinfo[key] : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
        }
        if (!(ok = warp_rendezvous(stage_bar, stage_phase, abort_flag, kWaitLimitNs))) break;
      }
      const int b = j & 1;
      if (!(ok = __all_sync(0xffffffffu, mbar_wait_cluster(&s_full[b], (uint32_t)(j >> 1) & 1u,
                                                           abort_flag, kWaitLimitNs)))) break;
      tc_fence_after();
      const uint32_t tS = tmem + lane_off + (uint32_t)(b * 128);
      uint32_t s[64];
      tmem_ld32(tS + col0, *reinterpret_cast<uint32_t(*)[32]>(&s[0]));
      tmem_ld32(tS + col0 + 32, *reinterpret_cast<uint32_t(*)[32]>(&s[32]));
      tmem_ld_wait();
      reg_fence<64>(s);
      const int nv = (int)kr.nvalid - col0;   // valid columns of this group (may be <= 0)
      if (nv < 64) {
#pragma unroll
        for (int c = 0; c < 64; ++c)
          if (c >= nv) s[c] = 0xff800000u;
      }
      float scl, off_base;
      if (cls == kClsFull) {
        const float w = bp.window, inv_f = bp.inv_falloff, st = bp.strength, cap = bp.cap;
        const float sl = bp.scale_log2;
#pragma unroll
        for (int c = 0; c < 64; ++c) {
          const float4 kv = kb[col0 + c];
          const float x = fmaxf(fabsf(t_q - kv.x) - w, 0.0f) * inv_f;
          const float pen = fminf(st * (x * x), cap);
          float bb = fmaf(-kv.z, pen, m_q * kv.y);
          if (bp.n_extra > 0) bb += wx[(int)kv.w];
          bb = is_tgt ? bb : 0.0f;
          s[c] = __float_as_uint(fmaf(__uint_as_float(s[c]), sl, bb * kLog2e));
        }
        scl = 1.0f;
        off_base = 0.0f;
      } else {
        scl = bp.scale_log2;
        off_base = rowb2;
      }
      // row max over both groups' columns; the barrier also guarantees that both groups have
      // read their S columns before either writes P over the buffer
      const float mloc = fmaf(row_max64(s), scl, off_base);
      float* xm = xmax + (j & 1) * (2 * kTile);
      xm[wg * kTile + r] = mloc;
      if (!(ok = warp_rendezvous(&xbar[wq], x_phase, abort_flag, kWaitLimitNs))) break;
      const float mx = fmaxf(mloc, xm[(1 - wg) * kTile + r]);
      const float m_new = fmaxf(m_run, mx);
      const bool need = (m_new - m_run) > 8.0f;        // true on the first tile
      const bool warp_need = __any_sync(0xffffffffu, need);
      const float m_use = need ? m_new : m_run;
      const float alpha = ex2_approx(m_run - m_use);
      l_run *= alpha;
      const float off = off_base - m_use;
      float lsum[4] = {0.0f, 0.0f, 0.0f, 0.0f};
      uint32_t pk[32];
#pragma unroll
      for (int c = 0; c < 64; c += 2) {
        const float p0 = ex2_approx(fmaf(__uint_as_float(s[c]), scl, off));
        const float p1 = ex2_approx(fmaf(__uint_as_float(s[c + 1]), scl, off));
        lsum[(c >> 1) & 3] += p0 + p1;
        pk[c >> 1] = pack_p<kBF16>(p0, p1);
      }
      l_run += (lsum[0] + lsum[1]) + (lsum[2] + lsum[3]);
      tmem_st32(tS + wg * 32, pk);
      if (j > 0 && warp_need) {
        // rescale this group's half of the O rows once the previous PV has landed
        if (!(ok = __all_sync(0xffffffffu, mbar_wait_cluster(pv_done, (uint32_t)(j - 1) & 1u,
                                                             abort_flag, kWaitLimitNs)))) break;
        tc_fence_after();
#pragma unroll 1
        for (int cc = 0; cc < 2; ++cc) {
          uint32_t o[32];
          tmem_ld32(tO + cc * 32, o);
          tmem_ld_wait();
          reg_fence<32>(o);
#pragma unroll
          for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
          tmem_st32(tO + cc * 32, o);
        }
      }
      m_run = m_use;
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(p_full_l[b]);
    }

    // ------------------------------ epilogue ---------------------------------------
    // PV_{nk-2} is issued after S_{nk-1}, so it may still be pending here: wait for its phase
    // first (a parity wait on phase nk-1 alone would pass while the barrier is at nk-2)
    if (ok && nk >= 2)
      ok = __all_sync(0xffffffffu, mbar_wait_cluster(pv_done, (uint32_t)(nk - 2) & 1u, abort_flag,
                                                     kWaitLimitNs));
    if (ok && __all_sync(0xffffffffu, mbar_wait_cluster(pv_done, (uint32_t)(nk - 1) & 1u,
                                                        abort_flag, kWaitLimitNs))) {
      tc_fence_after();
      xsum[wg * kTile + r] = l_run;
      // the partner warp may have given up; then this warp skips the store as well
      if (warp_rendezvous(&xbar[wq], x_phase, abort_flag, kWaitLimitNs)) {
      const float l_tot = l_run + xsum[(1 - wg) * kTile + r];
      const float inv_l = 1.0f / l_tot;
      uint16_t* orow = reinterpret_cast<uint16_t*>(args.O) + ((long long)bh * N + row) * PairShape::D + wg * 64;
#pragma unroll 1
      for (int cc = 0; cc < 2; ++cc) {
        uint32_t o[32];
        tmem_ld32(tO + cc * 32, o);
        tmem_ld_wait();
        reg_fence<32>(o);
        if (row_ok) {
          uint32_t w[16];
#pragma unroll
          for (int c = 0; c < 16; ++c)
            w[c] = pack_p<kBF16>(__uint_as_float(o[2 * c]) * inv_l, __uint_as_float(o[2 * c + 1]) * inv_l);
          uint4* dst = reinterpret_cast<uint4*>(orow + cc * 32);
#pragma unroll
          for (int v = 0; v < 4; ++v) dst[v] = make_uint4(w[4 * v], w[4 * v + 1], w[4 * v + 2], w[4 * v + 3]);
        }
      }
      if (row_ok && wg == 0) args.LSE[(long long)bh * N + row] = (m_run + log2f(l_tot)) * kLn2;
      }
    }
    tc_fence_before();
  }

  __syncthreads();
  // neither CTA of the pair leaves (and frees its shared and tensor memory) before the other
  // is done with the pair's barriers; bounded
  if (threadIdx.x == 0) {
    mbar_arrive_remote(mapa_shared(smem_u32(exit_bar), rank ^ 1u));
    volatile int no_abort = 0;
    mbar_wait_cluster(exit_bar, 0, &no_abort, kWaitLimitNs);
    if (*abort_flag) atomicExch(args.status, 1);
  }
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, 512);
  }
}

}  // namespace tara
