// attn_pair.cuh -- the 16-bit, head-dim-128 tensor-core path on SM pairs, with P in shared
// memory so that the next QK^T of a query tile does not wait for the previous PV.
//
// The kernel is persistent: one cluster of two CTAs (an SM pair) per two SMs, each walking work
// items c, c + G, c + 2G, ... (G clusters) in head-major order.  An item is four 128-row query
// tiles of one (branch, head): CTA r of the pair holds tiles 4q + 2t + r for t = 0, 1.  All
// clusters start their n-th item at about the same time and stream the same head's K and V in
// near lockstep, so a head's keys and values are read from DRAM about once per round of items
// and then served from L2 to every cluster (a grid of one CTA pair per item let later waves
// re-read them).  Consecutive rounds walk the key tiles in opposite directions: a round starts
// on the tiles the round before read last, which L2 still holds, instead of on the tiles it
// read first, which a head's 55 MB of K and V (at 107k tokens) has pushed out by then.
//
// The even CTA issues every MMA with cta_group::2, M = 256: MMA "t" covers tile t of both
// CTAs.  Each CTA supplies its own 128 rows of the A operand (Q for S = Q K^T, P for
// O += P V) and half of every B operand: keys [64r, 64r + 64) of a key tile for QK^T and
// head-dim columns [64r, 64r + 64) of a value tile for PV, so each SM loads and stores half
// of K and V.
//
// Tensor memory of each CTA (512 columns): S_0 | S_1 | O_0 | O_1, fp32.  P_t (16-bit) is written
// by the softmax threads to shared memory in the K-major 128-byte-swizzled layout the MMA reads
// as its A operand.  Because P does not live over S, the MMA of S_t for key tile j+1 is issued
// as soon as the softmax of tile t has loaded S_t(j) into registers: the softmax of tile j+1
// finds its scores ready, and the tensor pipe and the exponentials of both tiles overlap.
//
// Warp roles in each CTA (384 threads):
//   warps 0-3  softmax for query tile 0   (thread = one query row = one TMEM lane)
//   warps 4-7  softmax for query tile 1
//   warp  8    TMA producer: this CTA's Q tiles, then its halves of K_j and V_j into a ring of
//              shared-memory slots; completion is counted on the even CTA's barriers
//   warp  9    tensor-memory allocation (both CTAs); in the even CTA, one thread issues the
//              QK^T stream: S_t(j+1) once S_t(j) is consumed and K_{j+1} has landed
//   warp 10    in the even CTA, one thread issues the PV stream: PV_t(j) once P_t(j) is
//              written and V_j has landed (two issuers: a single thread issuing both streams
//              in turn left the tensor pipe idle between MMA groups)
//   warp 11    one thread classifies the (query tile, key tile) pairs ahead of the softmax
//              (tara_common.cuh: zero, constant, per-row or per-edge bias) into a ring of
//              shared-memory entries, so the softmax warps read one entry per key tile
//              instead of loading two tile summaries and classifying them
//
// Per key tile and query tile the softmax: reads the tile pair's class, waits for S, loads the
// whole row (one 128-column tcgen05.ld), tells the issuer that S may be overwritten, applies
// the class's bias, takes the row max, computes all 128 exponentials into packed 16-bit
// registers, then waits for the previous PV of its tile (the P buffer's last reader; usually
// long done by then), stores P, rescales the O row if the running max grew by more than 2^8,
// and signals P ready.  Every wait is bounded; a CTA that gives up sets an abort flag, the pair
// drains what it issued, and the device status word records the failure.
#pragma once

#include "attn_tc.cuh"
#include "sm100_ptx.cuh"
#include "tara_common.cuh"

namespace tara {

struct PairShape {
  static constexpr int D = 128;
  static constexpr int kQTileBytes = kTile * D * 2;       // 32 KB: 2 panels of 128 rows x 128 B
  static constexpr int kPanelBytes = kTile * 128;         // 16 KB
  static constexpr int kHalfBytes = 16384;                // K half: 64 keys x 128 d (2 x 8 KB)
                                                          // V half: 128 keys x 64 d (1 panel)
  static constexpr int kStages = 4;                       // ring slots (K_j, V_j alternate)
  static constexpr int kPTileBytes = kTile * kTile * 2;   // 32 KB: P of one query tile
  static constexpr int kKeyBufBytes = 2 * 2 * kTile * 16; // [query tile][parity][key] float4
  static constexpr int kRowWBytes = 2 * kTile * 17 * 4;   // [tile][row] extra-binding weights
  static constexpr int kClsRing = 8;                      // classification ring slots
  static constexpr int kClsBytes = kClsRing * 2 * 8;      // [slot][query tile] uint2
  static constexpr int kBarCount = 2 + 2 * kStages + 2 * 4 + 2 + 1 + 2 + 8 + 2 * kClsRing;
  static constexpr int kSmemBytes = 1024 /*alignment slack*/ + 2 * kQTileBytes +
                                    kStages * kHalfBytes + 2 * kPTileBytes + kKeyBufBytes +
                                    kRowWBytes + kClsBytes + kBarCount * 8 + 16;
  static_assert(kSmemBytes <= 232448, "dynamic shared memory above the 227 KB per-CTA limit");
  static constexpr uint32_t kColO = 256;                  // O_t at kColO + 128 t
};

// Query tiles per cluster (two per CTA).
constexpr int kPairTiles = 4;

template <bool kBF16>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kTcThreads, 1)
attn_pair_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                 const __grid_constant__ CUtensorMap tmV, const TcArgs args) {
  using S = PairShape;
  constexpr int NS = S::kStages;
  constexpr int HB = S::kHalfBytes;
  constexpr int D = S::D;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;                                   // 2 tiles
  uint8_t* sKV = sQ + 2 * S::kQTileBytes;               // NS half-tile slots
  uint8_t* sP = sKV + NS * HB;                          // 2 tiles
  float4* kbuf = reinterpret_cast<float4*>(sP + 2 * S::kPTileBytes);
  float* rowx = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(kbuf) + S::kKeyBufBytes);
  uint2* cls_ring = reinterpret_cast<uint2*>(reinterpret_cast<uint8_t*>(rowx) + S::kRowWBytes);
  uint64_t* bars = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(cls_ring) + S::kClsBytes);
  uint64_t* q_full = bars;              // even CTA: Q of both CTAs landed
  uint64_t* q_empty = q_full + 1;       // both CTAs (2-SM commit): the last QK^T of an item read Q
  uint64_t* kv_full = q_empty + 1;      // even CTA: both halves of slot s landed
  uint64_t* kv_empty = kv_full + NS;    // both CTAs (2-SM commit): slot s may be refilled
  uint64_t* s_full = kv_empty + NS;     // both CTAs (2-SM commit): S_t holds the next key tile
  uint64_t* s_free = s_full + 2;        // even CTA: 8 softmax warps have loaded S_t
  uint64_t* p_full = s_free + 2;        // even CTA: 8 softmax warps have stored P_t
  uint64_t* pv_done = p_full + 2;       // both CTAs (2-SM commit): PV_t completed
  uint64_t* drain = pv_done + 2;        // [2] even CTA: every MMA of an issuer has completed
  uint64_t* exit_bar = drain + 2;       // the peer is done with this CTA's memory
  uint64_t* stage_bar = exit_bar + 1;   // [2] per query tile: the 4 warps of its group
  uint64_t* exp_tok = stage_bar + 2;    // [lane quarter][tile]: that warp may run its exponentials
  uint64_t* cls_full = exp_tok + 8;     // [slot] the classifier wrote both tiles' entries
  uint64_t* cls_empty = cls_full + S::kClsRing;   // [slot] the 8 softmax warps have read them
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(cls_empty + S::kClsRing);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int N = args.N;
  const int nk = (N + kTile - 1) / kTile;
  // work items: (branch, head) planes x groups of four query tiles, head-major
  const int groups = (args.ntiles + kPairTiles - 1) / kPairTiles;
  const int n_items = args.B * args.H * groups;
  const int n_clusters = (int)(gridDim.x >> 1);
  const int first_item = (int)(blockIdx.x >> 1);
  // Every role walks the same items in the same order.  Barrier phases run on across items:
  // the g-th key tile this cluster processes (g = item ordinal * nk + j) completes phase g of
  // the per-tile barriers, and ring slot s holds K or V half-tile number 2g or 2g + 1.  Step j
  // of an item processes key tile j, or nk - 1 - j on items that walk the keys descending (the
  // order changes the softmax's result by rounding only).
  auto descending = [&](int item) -> bool {
    return (((uint32_t)(args.item_base + item)) / (uint32_t)args.order_span) & 1u;
  };

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&s_full[t], 1);
      mbar_init(&s_free[t], 8);    // 4 softmax warps of tile t in each CTA
      mbar_init(&p_full[t], 8);
      mbar_init(&pv_done[t], 1);
      mbar_init(&stage_bar[t], 4);
    }
    for (int q = 0; q < 4; ++q) {
      mbar_init(&exp_tok[2 * q], 1);
      mbar_init(&exp_tok[2 * q + 1], 1);
      mbar_arrive(&exp_tok[2 * q]);   // tile 0 goes first
    }
    for (int c = 0; c < S::kClsRing; ++c) {
      mbar_init(&cls_full[c], 1);
      mbar_init(&cls_empty[c], 8);
    }
    mbar_init(&drain[0], 1);
    mbar_init(&drain[1], 1);
    mbar_init(exit_bar, 1);
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
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;\n" ::"n"(kTcControlRegs) : "memory");
    if (warp == 8 && lane == 0) {
      // ------------------------------ TMA producer (both CTAs) -------------------------
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      const uint32_t q_full_l = mapa_shared(smem_u32(q_full), 0);
      // every cluster streams the same head's K and V at about the same time: keep them in L2;
      // Q is read once per item
      const uint64_t keep = l2_policy_evict_last(), once = l2_policy_evict_first();
      bool ok = true;
      int i = 0;   // half-tiles issued (K_j, V_j alternate)
      int issued = 0;
      for (int item = first_item, k = 0; ok && item < n_items; item += n_clusters, ++k) {
        const int bh = item / groups;
        const int qt_base = (item - bh * groups) * kPairTiles + (int)rank;
        const bool desc = descending(item);
        // Q of the previous item is read by its last QK^T
        if (k > 0 && !(ok = mbar_wait(q_empty, (uint32_t)(k - 1) & 1u, abort_flag, kWaitLimitNs))) break;
        if (leader) mbar_arrive_expect_tx(q_full, 2 * 2 * S::kQTileBytes);
        for (int t = 0; t < 2; ++t)
          for (int p = 0; p < 2; ++p)
            tma_load_3d_pair_hint(sQ + t * S::kQTileBytes + p * S::kPanelBytes, &tmQ, q_full_l,
                                  p * 64, (qt_base + 2 * t) * kTile, bh, once);
        for (int h2 = 0; h2 < 2 * nk; ++h2, ++i) {
          const int slot = i % NS;
          const uint32_t ph = (uint32_t)(i / NS) & 1u;
          if (!(ok = mbar_wait(&kv_empty[slot], ph ^ 1u, abort_flag, kWaitLimitNs))) break;
          if (leader) mbar_arrive_expect_tx(&kv_full[slot], 2 * HB);
          const uint32_t full_l = mapa_shared(smem_u32(&kv_full[slot]), 0);
          uint8_t* dst = sKV + slot * HB;
          const int j = desc ? nk - 1 - (h2 >> 1) : h2 >> 1;
          if ((h2 & 1) == 0) {
            // K_j rows [64r, 64r + 64): two 64-row x 128-byte panels (head-dim halves)
            for (int p = 0; p < 2; ++p)
              tma_load_3d_pair_hint(dst + p * (64 * 128), &tmK, full_l, p * 64,
                                    j * kTile + (int)rank * 64, bh, keep);
          } else {
            // V_j head-dim columns [64r, 64r + 64): one 128-row x 128-byte panel
            tma_load_3d_pair_hint(dst, &tmV, full_l, (int)rank * 64, j * kTile, bh, keep);
          }
          issued = i + 1;
        }
      }
      if (*abort_flag && issued > 0) {
        // copies already issued land within microseconds; their completion is counted in the
        // even CTA, so give them 1 ms before this CTA's shared memory can be released
        for (int w = 0; w < 1000; ++w) __nanosleep(1000);
      }
    } else if ((warp == 9 || warp == 10) && lane == 0 && leader) {
      // ------------------------------ MMA issuers (even CTA) ---------------------------
      // Two threads, one per stream, each issuing in order as its operands become ready:
      // warp 9 the QK^T stream QK_0(0), QK_1(0), QK_0(1), ... and warp 10 the PV stream
      // PV_0(0), PV_1(0), ...  The streams write different tensor-memory columns (S, O) and
      // read different operands, and each thread's commits track only its own MMAs.
      const bool qk_role = warp == 9;
      bool ok = true;
      if (qk_role) {
        constexpr uint32_t idesc_qk = make_idesc_f16(256, 128, kBF16, false);
        // base descriptors; a byte offset moves the start-address field by offset >> 4
        // (shared addresses stay below 2^18, so the 14-bit field never carries)
        const uint64_t qd0 = make_sdesc_sw128(smem_u32(sQ), 16, 1024);
        const uint64_t kd0 = make_sdesc_sw128(smem_u32(sKV), 16, 1024);
        int g = 0;   // key tiles processed so far, over all items
        for (int item = first_item, k = 0; ok && item < n_items; item += n_clusters, ++k) {
          if (!(ok = mbar_wait(q_full, (uint32_t)k & 1u, abort_flag, kWaitLimitNs))) break;
          for (int n = 0; ok && n < 2 * nk; ++n) {
            const int t = n & 1, gj = g + (n >> 1);
            const int ki = 2 * gj, kslot = ki % NS;
            // K is waited for once, for t = 0; its slot is released only after QK_1
            if (t == 0 && !(ok = mbar_wait(&kv_full[kslot], (uint32_t)(ki / NS) & 1u, abort_flag,
                                           kWaitLimitNs)))
              break;
            // S_t is free once both CTAs' softmax warps have loaded the previous key tile
            if (gj > 0 && !(ok = mbar_wait(&s_free[t], (uint32_t)(gj - 1) & 1u, abort_flag,
                                           kWaitLimitNs)))
              break;
            tc_fence_after();
            const uint32_t d_s = tmem + (uint32_t)(t * 128);
            const uint64_t qd = qd0 + (uint64_t)((t * S::kQTileBytes) >> 4);
            const uint64_t kd = kd0 + (uint64_t)((kslot * HB) >> 4);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint64_t qoff = (uint64_t)((((kk >> 2) * S::kPanelBytes) + (kk & 3) * 32) >> 4);
              const uint64_t koff = (uint64_t)((((kk >> 2) * (64 * 128)) + (kk & 3) * 32) >> 4);
              umma_ss_pair(d_s, qd + qoff, kd + koff, idesc_qk, kk > 0 ? 1u : 0u);
            }
            umma_commit_pair(&s_full[t]);
            if (t == 1) umma_commit_pair(&kv_empty[kslot]);
          }
          // the item's Q may be replaced once its last QK^T has read it
          if (ok) umma_commit_pair(q_empty);
          g += nk;
        }
      } else {
        constexpr uint32_t idesc_pv = make_idesc_f16(256, 128, kBF16, true);
        const uint64_t vd0 = make_sdesc_sw128(smem_u32(sKV), S::kPanelBytes, 1024);
        const uint64_t pd0 = make_sdesc_sw128(smem_u32(sP), 16, 1024);
        int g = 0;
        for (int item = first_item; ok && item < n_items; item += n_clusters) {
          for (int n = 0; ok && n < 2 * nk; ++n) {
            const int t = n & 1, j = n >> 1, gj = g + j;
            const int vi = 2 * gj + 1, vslot = vi % NS;
            if (t == 0 && !(ok = mbar_wait(&kv_full[vslot], (uint32_t)(vi / NS) & 1u, abort_flag,
                                           kWaitLimitNs)))
              break;
            // P_t is in shared memory in both CTAs (and O_t rescaled where needed)
            if (!(ok = mbar_wait(&p_full[t], (uint32_t)gj & 1u, abort_flag, kWaitLimitNs))) break;
            tc_fence_after();
            const uint32_t d_o = tmem + S::kColO + (uint32_t)(t * 128);
            const uint64_t pd = pd0 + (uint64_t)((t * S::kPTileBytes) >> 4);
            const uint64_t vd = vd0 + (uint64_t)((vslot * HB) >> 4);
#pragma unroll
            for (int kk = 0; kk < kTile / 16; ++kk) {
              const uint64_t poff = (uint64_t)((((kk >> 2) * S::kPanelBytes) + (kk & 3) * 32) >> 4);
              // the first PV of an item starts O afresh
              umma_ss_pair(d_o, pd + poff, vd + (uint64_t)((kk * 2048) >> 4), idesc_pv,
                           (j > 0 || kk > 0) ? 1u : 0u);
            }
            umma_commit_pair(&pv_done[t]);
            if (t == 1) umma_commit_pair(&kv_empty[vslot]);
          }
          g += nk;
        }
      }
      // every MMA this thread issued completes before either CTA releases its memory
      uint64_t* my_drain = &drain[qk_role ? 0 : 1];
      umma_commit_pair(my_drain);
      volatile int no_abort = 0;
      mbar_wait(my_drain, 0, &no_abort, kDrainLimitNs);
    } else if (warp == 11 && lane == 0) {
      // ------------------------------ tile-pair classifier (both CTAs) -----------------
      // Runs up to kClsRing key tiles ahead of the softmax warps: for step g of the walk it
      // classifies (query tile t of this CTA, the step's key tile) for t = 0, 1 and writes
      // {class | Picture index << 8 | valid keys << 16, parameter} to ring slot g % kClsRing,
      // the parameter being the constant bias (natural units) of the constant classes and
      // the guide frame's time of a single-frame guide tile.
      const BiasParams& bp = args.bp;
      bool ok = true;
      int g = 0;
      for (int item = first_item; ok && item < n_items; item += n_clusters, g += nk) {
        const int bh = item / groups;
        const int mset = args.per_branch_meta ? bh / args.H : 0;
        const TileRec* qrecs = args.recs + (long long)mset * args.ntiles;
        const TileRec* krecs =
            (descending(item) ? args.recs_desc : args.recs) + (long long)mset * args.ntiles;
        TileRec qr[2];
        for (int t = 0; t < 2; ++t) {
          const int qtile = (item - bh * groups) * kPairTiles + (int)rank + 2 * t;
          if (qtile < args.ntiles) {
            qr[t] = qrecs[qtile];
          } else {
            qr[t].segmask = 0;   // no rows: classified as unbiased
            qr[t].picmask = 0;
            qr[t].nvalid = 0;
            qr[t].single_pic = 0;
            qr[t].tq_min = qr[t].tk_min = 0.0f;
            qr[t].tq_max = qr[t].tk_max = 0.0f;
          }
        }
        TileRec kr_next = krecs[0];
        for (int j = 0; j < nk; ++j) {
          const int gj = g + j;
          const int slot = gj & (S::kClsRing - 1);
          const TileRec kr = kr_next;
          if (j + 1 < nk) kr_next = krecs[j + 1];
          if (!(ok = mbar_wait(&cls_empty[slot], ((uint32_t)(gj / S::kClsRing) & 1u) ^ 1u,
                               abort_flag, kWaitLimitNs)))
            break;
          for (int t = 0; t < 2; ++t) {
            float cval;
            const int cls = classify_pair(qr[t], kr, bp, &cval);
            const float par = cls == kClsRowGuide ? kr.tk_min : cval;
            cls_ring[slot * 2 + t] =
                make_uint2((uint32_t)cls | ((kr.single_pic & 15u) << 8) | (kr.nvalid << 16),
                           __float_as_uint(par));
          }
          mbar_arrive(&cls_full[slot]);
        }
      }
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;\n" ::"n"(kTcSoftmaxRegs) : "memory");
    // ------------------------------ softmax warps (both CTAs) --------------------------
    const int t = warp >> 2;            // query tile of this warpgroup
    const int wq = warp & 3;            // TMEM lane quarter
    const int r = wq * 32 + lane;       // row within the tile
    const BiasParams& bp = args.bp;
    const uint32_t s_free_l = mapa_shared(smem_u32(&s_free[t]), 0);
    const uint32_t p_full_l = mapa_shared(smem_u32(&p_full[t]), 0);
    // this thread's row of P: 16-byte chunk c of panel p at p*16 KB + r*128 + ((c ^ (r%8))*16),
    // the 128-byte swizzle of a K-major operand (an 8-row atom of 1 KB per 8 rows)
    const uint32_t p_row = smem_u32(sP + t * S::kPTileBytes) + (uint32_t)(r * 128);
    const uint32_t p_sw = (uint32_t)(r & 7);
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    const uint32_t tS = tmem + lane_off + (uint32_t)(t * 128);
    const uint32_t tO = tmem + lane_off + S::kColO + (uint32_t)(t * 128);
    const float ninf = __int_as_float(0xff800000);
    // weights of the extra bindings for this row, one per Picture index (0 for index 0)
    float* wx = rowx + (t * kTile + r) * 17;
    bool ok = true;
    uint32_t stage_phase = 0;
    int g = 0;   // key tiles processed so far, over all items

    for (int item = first_item; ok && item < n_items; item += n_clusters, g += nk) {
      const int bh = item / groups;
      const int qtile = (item - bh * groups) * kPairTiles + (int)rank + 2 * t;
      const int row = qtile * kTile + r;
      const bool row_ok = (qtile < args.ntiles) && (row < N);
      const int mset = args.per_branch_meta ? bh / args.H : 0;
      const long long mtok = (long long)mset * args.meta_stride;
      // the key records in the order this item walks the keys: step j reads records
      // [128 j, 128 j + 128) of the ascending or the descending copy
      const float4* kinfo = (descending(item) ? args.keyinfo_desc : args.keyinfo) +
                            (long long)mset * args.ntiles * kTile;

      bool is_tgt = false;
      float t_q = 0.0f, m_q = 0.0f;
      if (row_ok) {
        is_tgt = args.seg[mtok + row] == kSegTarget;
        t_q = args.time_s[mtok + row];
        m_q = args.m[mtok + row];
      }
      // debug build: the plane exists, a target row's time and mask weight are finite, and
      // this row's part of P stays inside its tile's buffer
      TARA_DCHECK_RECORD(bh < args.B * args.H, args.status);
      TARA_DCHECK_RECORD(!is_tgt || (isfinite(t_q) && isfinite(m_q)), args.status);
      TARA_DCHECK_RECORD(p_row + S::kPanelBytes + 128 <= smem_u32(sP) + (uint32_t)(t + 1) * S::kPTileBytes,
                  args.status);
      if (bp.n_extra > 0) {
        for (int pidx = 0; pidx < 16; ++pidx) {
          float acc = 0.0f;
          if (is_tgt)
            for (int kx = 0; kx < bp.n_extra; ++kx)
              acc += args.xm.m[kx * args.xm.stride + mtok + row] * bp.lng_x[kx][pidx];
          wx[pidx] = acc;
        }
      }
      float m_run = ninf, l_run = 0.0f;

      for (int j = 0; j < nk; ++j) {
        const int gj = g + j;
        const float sl = bp.scale_log2;
        // this tile pair's class from the classifier warp (normally written long before)
        const int cs = gj & (S::kClsRing - 1);
        if (!(ok = warp_wait(&cls_full[cs], (uint32_t)(gj / S::kClsRing) & 1u, abort_flag,
                             kWaitLimitNs)))
          break;
        const uint2 ce = cls_ring[cs * 2 + t];
        __syncwarp();
        if (lane == 0) mbar_arrive(&cls_empty[cs]);
        const int cls = (int)(ce.x & 0xffu);
        const float cpar = __uint_as_float(ce.y);
        float rowb2 = 0.0f;
        if (is_tgt) {
          if (cls == kClsConstCap) rowb2 = cpar * kLog2e;
          else if (cls == kClsRowGuide) rowb2 = -penalty_f32(fabsf(t_q - cpar), bp) * kLog2e;
          else if (cls == kClsConstPic)
            rowb2 = (bp.n_extra > 0 ? m_q * cpar + wx[(ce.x >> 8) & 15u] : m_q * cpar) * kLog2e;
        }
        float4* kb = kbuf + (t * 2 + (gj & 1)) * kTile;
        if (cls == kClsFull) {
          // stage the tile's key records in shared memory (one coalesced load per thread);
          // two buffers, so a warp one iteration ahead never overwrites records another warp
          // of the group still reads
          kb[r] = kinfo[j * kTile + r];   // zero records past the sequence's end
          if (!(ok = warp_rendezvous(&stage_bar[t], stage_phase, abort_flag, kWaitLimitNs))) break;
        }
        if (!(ok = warp_wait(&s_full[t], (uint32_t)gj & 1u, abort_flag, kWaitLimitNs))) break;
        tc_fence_after();
        uint32_t s[128];
        tmem_ld128(tS, s);
        tmem_ld_wait();
        reg_fence<128>(s);
        // S_t may now be overwritten by the next key tile's QK^T
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(s_free_l);

        const int nv = (int)(ce.x >> 16);
        if (nv < kTile) {
#pragma unroll
          for (int c = 0; c < 128; ++c)
            if (c >= nv) s[c] = 0xff800000u;
        }
        float mx, scl, off_base;
        if (cls == kClsFull) {
          if (bp.n_extra == 0) add_edge_bias<false>(s, kb, t_q, m_q, is_tgt, sl, wx, bp);
          else add_edge_bias<true>(s, kb, t_q, m_q, is_tgt, sl, wx, bp);
          mx = row_max128(s);
          scl = 1.0f;
          off_base = 0.0f;
        } else {
          mx = fmaf(row_max128(s), sl, rowb2);
          scl = sl;
          off_base = rowb2;
        }
        const float m_new = fmaxf(m_run, mx);
        const bool need = (m_new - m_run) > 8.0f;        // true on the first tile (m_run = -inf)
        const bool warp_need = __any_sync(0xffffffffu, need);
        const float m_use = need ? m_new : m_run;
        const float alpha = ex2_approx(m_run - m_use);   // 1 when not raised, 0 on the first tile
        l_run *= alpha;
        const float off = off_base - m_use;
        // The two warps of a lane quarter (one per query tile) share an SM sub-partition and
        // its exponential unit, which both tiles together keep busy for as long as the tensor
        // pipe needs per key tile.  Their exponential phases take turns (tile 0 of one key
        // tile, tile 1 of it, tile 0 of the next, ...), so that one warp's loads, max and
        // stores overlap the other's exponentials instead of both contending for the unit.
        if (!(ok = warp_wait(&exp_tok[2 * wq + t], (uint32_t)gj & 1u, abort_flag, kWaitLimitNs))) break;
        // all 128 exponentials first, into 64 packed 16-bit pairs (each score register dies as
        // its pair is formed); columns in pairs: one packed FMA forms both exponents, one
        // packed add accumulates both probabilities (two accumulators break the dependency
        // chain)
        const uint64_t scl2 = f32x2_pack(scl, scl), off2 = f32x2_pack(off, off);
        uint64_t lsum2[2] = {0ull, 0ull};
        uint32_t pk[64];
#pragma unroll
        for (int c = 0; c < 128; c += 2) {
          float x0, x1;
          f32x2_unpack(f32x2_fma(f32x2_pack_bits(s[c], s[c + 1]), scl2, off2), x0, x1);
          const float p0 = ex2_approx(x0);
          const float p1 = ex2_approx(x1);
          lsum2[(c >> 1) & 1] = f32x2_add(lsum2[(c >> 1) & 1], f32x2_pack(p0, p1));
          pk[c >> 1] = pack_p<kBF16>(p0, p1);
        }
        {
          float a0, a1;
          f32x2_unpack(f32x2_add(lsum2[0], lsum2[1]), a0, a1);
          l_run += a0 + a1;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&exp_tok[2 * wq + (t ^ 1)]);
        // the P buffer's previous reader (and the last writer of O_t) is the previous PV_t
        if (gj > 0) {
          if (!(ok = warp_wait(&pv_done[t], (uint32_t)(gj - 1) & 1u, abort_flag, kWaitLimitNs))) break;
          tc_fence_after();
        }
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          const uint32_t addr = p_row + (uint32_t)((c >> 3) * S::kPanelBytes) +
                                ((((uint32_t)c & 7u) ^ p_sw) << 4);
          st_shared_v4(addr, pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
        }
        if (j > 0 && warp_need) {
          // rescale this warp's O rows; the previous PV_t has landed and the next waits for P
#pragma unroll 1
          for (int cc = 0; cc < D / 32; ++cc) {
            uint32_t o[32];
            tmem_ld32(tO + cc * 32, o);
            tmem_ld_wait();
            reg_fence<32>(o);
#pragma unroll
            for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
            tmem_st32(tO + cc * 32, o);
          }
          tmem_st_wait();
        }
        m_run = m_use;
        // P (generic-proxy stores) must be visible to the tensor core (async proxy)
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(p_full_l);
      }

      // ------------------------------ epilogue of the item ---------------------------
      // The next item's first PV_t overwrites O_t; it waits for this warp's P of that item,
      // which comes after these reads in program order.
      if (ok && (ok = warp_wait(&pv_done[t], (uint32_t)(g + nk - 1) & 1u, abort_flag, kWaitLimitNs))) {
        tc_fence_after();
        const float inv_l = 1.0f / l_run;
        uint16_t* orow = reinterpret_cast<uint16_t*>(args.O) + ((long long)bh * N + row) * D;
        const bool out_ok =
            row_ok && TARA_DCHECK((long long)bh * N + row < (long long)args.B * args.H * N, args.status);
#pragma unroll 1
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t o[32];
          tmem_ld32(tO + cc * 32, o);
          tmem_ld_wait();
          reg_fence<32>(o);
          if (out_ok) {
            uint32_t w[16];
#pragma unroll
            for (int c = 0; c < 16; ++c)
              w[c] = pack_p<kBF16>(__uint_as_float(o[2 * c]) * inv_l,
                                   __uint_as_float(o[2 * c + 1]) * inv_l);
            uint4* dst = reinterpret_cast<uint4*>(orow + cc * 32);
#pragma unroll
            for (int v = 0; v < 4; ++v)
              st_global_v4_stream(dst + v, make_uint4(w[4 * v], w[4 * v + 1], w[4 * v + 2], w[4 * v + 3]));
          }
        }
        if (out_ok) args.LSE[(long long)bh * N + row] = (m_run + log2f(l_run)) * kLn2;
        tc_fence_before();
      }
    }
    tc_fence_before();
  }

  __syncthreads();
  // neither CTA of the pair leaves (and frees its shared and tensor memory) before the other
  // is done with the pair's barriers and operands; bounded
  if (threadIdx.x == 0) {
    mbar_arrive_cluster(mapa_shared(smem_u32(exit_bar), rank ^ 1u));
    volatile int no_abort = 0;
    mbar_wait(exit_bar, 0, &no_abort, kWaitLimitNs);
    if (*abort_flag) atomicExch(args.status, 1);
  }
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, 512);
  }
}

}  // namespace tara
