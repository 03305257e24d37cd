// attn_tc.cuh -- the tensor-core path: one-pass TARA-biased attention forward on sm_100a.
//
// One CTA owns two 128-row query tiles of one (branch, head) and streams every 128-key tile
// of K and V once.  Warp roles (384 threads):
//   warps 0-3  softmax for query tile 0   (thread = one query row = one TMEM lane)
//   warps 4-7  softmax for query tile 1
//   warp  8    TMA producer: Q once, then K_j, V_j into a ring of shared-memory slots
//   warp  9    MMA issuer (one thread): S_t = Q_t K_j^T and O_t += P_t V_j with tcgen05.mma;
//              also owns the tensor-memory allocation
//   warps 10-11 idle (complete the third warpgroup for the register split)
// Tensor memory (512 columns): S_0 | S_1 | O_0 | O_1, fp32.  P_t (16-bit) is written by the
// softmax threads into columns 64..127 of S_t and read from there as the A operand of the PV
// MMA, so P never goes through shared memory.
//
// The bias never exists as an N x N tensor.  For each (query tile, key tile) pair the softmax
// warps classify the pair from the two tile summaries: no bias, a constant -cap on every
// target row, a constant m_row*ln(gain) on every target row, one penalty per target row (a key
// tile inside one guide frame), or per-edge evaluation from the per-key records.  Constant and
// per-row biases fold into the per-row exponent offset, so they cost no per-element work.
// Logits are kept in log2 units: x = s*scale*log2(e) + bias*log2(e).
//
// Online softmax: a thread holds its whole row of S (32x32b TMEM loads give one row per
// thread), so the row max and sum need no cross-thread reduction; exponents and sums run on
// column pairs with packed f32x2 arithmetic.  The running max is only raised when it grows by
// more than 2^8 in weight (P stays below 256), and only then is the O row in TMEM rescaled,
// after the previous PV MMA has completed.
//
// kQ8 (the INT8 QK^T variant): Q and K arrive as 8-bit codes with per-row and per-key-tile
// scales, QK^T runs as tcgen05.mma.kind::i8 into s32 S, and the scales join the softmax scale
// in the per-tile row multiplier.
#pragma once

#include "sm100_ptx.cuh"
#include "tara_common.cuh"

namespace tara {

constexpr int kTcThreads = 384;
// setmaxnreg split: the launch gives every thread kTcLaunchRegs; the two softmax warpgroups
// raise theirs to kTcSoftmaxRegs, the control warpgroup lowers its own to kTcControlRegs.  The
// sum must equal the launch pool, or the raise would wait for registers that never come; the
// host refuses to launch when ptxas gave the kernel a different register count.
constexpr int kTcLaunchRegs = 168;
constexpr int kTcSoftmaxRegs = 176;
constexpr int kTcControlRegs = 152;
static_assert(2 * 128 * kTcSoftmaxRegs + 128 * kTcControlRegs == kTcThreads * kTcLaunchRegs,
              "register split must use the launch pool exactly");

constexpr uint64_t kWaitLimitNs = 2000000000ull;   // 2 s per wait; a normal wait is microseconds
constexpr uint64_t kDrainLimitNs = 200000000ull;   // 0.2 s to let in-flight copies/MMAs land

template <int D, bool kQ8 = false>
struct TcShape {
  static constexpr int kTileBytes = kTile * D * 2;          // one 128 x D 16-bit tile
  // Q and K tiles: 16-bit, or 8-bit codes (one 128-byte swizzle panel per row at D = 128)
  static constexpr int kQKTileBytes = kQ8 ? kTile * D : kTileBytes;
  static constexpr int kPanels = D / 64;                    // 128-byte swizzle panels per row
  static constexpr int kPanelBytes = kTile * 128;           // 128 rows x 128 bytes
  static constexpr int kStages = (D == 128) ? 4 : 8;        // K/V ring slots
  static constexpr int kKeyBufBytes = 2 * 2 * kTile * 16;  // [query tile][parity][key] float4
  static constexpr int kRowWBytes = 2 * kTile * 17 * 4;     // [tile][row] extra-binding weights
  static constexpr int kBarCount = 1 + 2 * kStages + 2 + 2 + 2 + 1 + 2;
  static constexpr int kSmemBytes = 1024 /*alignment slack*/ + 2 * kQKTileBytes +
                                    kStages * kTileBytes + kKeyBufBytes + kRowWBytes +
                                    kBarCount * 8 + 16;
  static_assert(kSmemBytes <= 232448, "dynamic shared memory above the 227 KB per-CTA limit");
  static constexpr uint32_t kColS = 0;        // S_t at kColS + 128 t
  static constexpr uint32_t kColO = 256;      // O_t at kColO + D t
  static constexpr uint32_t kColP = 64;       // P_t at S_t + kColP
};

struct TcArgs {
  void* O;
  float* LSE;
  const uint8_t* seg;
  const float* time_s;
  const float* m;
  // Records written by the tile-summary kernel, per metadata set: ntiles tile records and
  // ntiles * 128 key records (zero past the sequence's end), in ascending tile order; the
  // *_desc copies hold the same records with the tile order reversed (tile ntiles - 1 first)
  const TileRec* recs;
  const float4* keyinfo;
  const TileRec* recs_desc;
  const float4* keyinfo_desc;
  long long meta_stride;   // tokens between metadata sets (0: one set for all branches)
  int N, H, ntiles;
  int B;                   // branches (the persistent kernel walks all B x H planes)
  int per_branch_meta;     // 1 when every branch has its own metadata set
  int* status;
  BiasParams bp;
  ExtraMasks xm;           // masks of chained bindings beyond the first (bp.n_extra of them)
  const float* q_scale;    // INT8 QK^T: per-token Q scales [B*H][N]
  const float* k_scale;    // INT8 QK^T: per-key-tile K scales [B*H][ntiles]
  // SM-pair kernel: work item i of this call is item item_base + i of the larger call its
  // planes were cut from (item_base 0 for an uncut call); it walks the keys ascending when
  // ((item_base + i) / order_span) is even, descending when it is odd
  long long plane_base;    // host side: index of this call's plane 0 in the larger call
  int item_base;
  int order_span;
};

// A wait every lane of the warp leaves together (the tcgen05 loads and stores that follow are
// warp-collective).
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort,
                                          uint64_t limit_ns) {
  const bool ok = mbar_wait(bar, parity, abort, limit_ns);
  return __all_sync(0xffffffffu, ok);
}

// Max of the 128 values of a row: eight independent chains of three-input max, then a tree.
__device__ __forceinline__ float row_max128(const uint32_t (&s)[128]) {
  float a[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) a[i] = __uint_as_float(s[i]);
#pragma unroll
  for (int c = 8; c < 120; c += 16) {
#pragma unroll
    for (int i = 0; i < 8; ++i)
      a[i] = fmax3(a[i], __uint_as_float(s[c + i]), __uint_as_float(s[c + 8 + i]));
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) a[i] = fmaxf(a[i], __uint_as_float(s[120 + i]));
  return fmaxf(fmax3(a[0], a[1], a[2]), fmax3(a[3], a[4], fmax3(a[5], a[6], a[7])));
}

// Bounded rendezvous of the warps counted by `bar` (lane 0 of each warp arrives; every lane
// waits).  Shared-memory writes made before it by any lane are visible to all lanes of the
// participating warps after it.  `phase` is the caller's phase bit for this barrier.
__device__ __forceinline__ bool warp_rendezvous(uint64_t* bar, uint32_t& phase,
                                                volatile int* abort, uint64_t limit_ns) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(bar);
  const bool ok = warp_wait(bar, phase, abort, limit_ns);
  phase ^= 1u;
  return ok;
}

// Max of 128 signed 32-bit values (the 8-bit path's integer scores): eight independent
// chains of three-input integer max, then a tree (64 operations instead of 127).
__device__ __forceinline__ int row_max128_s32(const uint32_t (&s)[128]) {
  int a[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) a[i] = (int)s[i];
#pragma unroll
  for (int c = 8; c < 120; c += 16) {
#pragma unroll
    for (int i = 0; i < 8; ++i) a[i] = __vimax3_s32(a[i], (int)s[c + i], (int)s[c + 8 + i]);
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) a[i] = max(a[i], (int)s[120 + i]);
  return __vimax3_s32(__vimax3_s32(a[0], a[1], a[2]), __vimax3_s32(a[3], a[4], a[5]),
                      max(a[6], a[7]));
}

// Scores of one row of a per-edge (kClsFull) tile, in place: s[c] <- s[c]*sl + bias*log2(e),
// with the bias of the edge (row, key c) from the staged key records kb (tara_common.cuh) and,
// with chained bindings (kExtra), the row's weight wx[Picture index].  The bias is computed
// for every row and zeroed by a select on non-target rows: a per-element branch on the row
// role costs ~10x here.
template <bool kExtra>
__device__ __forceinline__ void add_edge_bias(uint32_t (&s)[128], const float4* kb, float t_q,
                                              float m_q, bool is_tgt, float sl, const float* wx,
                                              const BiasParams& bp) {
  const float w = bp.window, inv_f = bp.inv_falloff, st = bp.strength, cap = bp.cap;
#pragma unroll
  for (int c = 0; c < 128; ++c) {
    const float4 kv = kb[c];
    const float x = fmaxf(fabsf(t_q - kv.x) - w, 0.0f) * inv_f;
    const float pen = fminf(st * (x * x), cap);
    float b = fmaf(-kv.z, pen, m_q * kv.y);
    if (kExtra) b += wx[(int)kv.w];
    b = is_tgt ? b : 0.0f;
    s[c] = __float_as_uint(fmaf(__uint_as_float(s[c]), sl, b * kLog2e));
  }
}

template <bool kBF16>
__device__ __forceinline__ uint32_t pack_p(float lo, float hi) {
  return kBF16 ? pack_bf16x2(lo, hi) : pack_f16x2(lo, hi);
}

// kQ8: Q and K arrive as 8-bit codes (tmQ, tmK map the code arrays), QK^T runs as
// tcgen05.mma.kind::i8 into an s32 S, and the softmax scales row i of key tile j by
// q_scale[i] * k_scale[j]; P and V stay 16-bit.
template <bool kBF16, int D, bool kQ8 = false>
__global__ void __launch_bounds__(kTcThreads, 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, const TcArgs args) {
  static_assert(!kQ8 || D == 128, "8-bit Q/K tiles use one 128-byte panel per row");
  using S = TcShape<D, kQ8>;
  constexpr int TB = S::kTileBytes;
  constexpr int QKB = S::kQKTileBytes;
  constexpr int NS = S::kStages;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;                       // 2 tiles
  uint8_t* sKV = smem + 2 * QKB;            // NS slots
  float4* kbuf = reinterpret_cast<float4*>(sKV + NS * TB);    // per-key records of full tiles
  float* rowx = reinterpret_cast<float*>(sKV + NS * TB + S::kKeyBufBytes);   // [tile][row][17]
  uint64_t* bars = reinterpret_cast<uint64_t*>(sKV + NS * TB + S::kKeyBufBytes + S::kRowWBytes);
  uint64_t* q_full = bars;
  uint64_t* kv_full = bars + 1;
  uint64_t* kv_empty = kv_full + NS;
  uint64_t* s_full = kv_empty + NS;
  uint64_t* p_full = s_full + 2;
  uint64_t* pv_done = p_full + 2;
  uint64_t* drain = pv_done + 2;
  uint64_t* stage_bar = drain + 1;      // [2] per query tile: the 4 warps of its group
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(stage_bar + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int N = args.N;
  const int bh = blockIdx.z * args.H + blockIdx.y;
  const int qt0 = blockIdx.x * 2;
  const int nk = (N + kTile - 1) / kTile;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&s_full[t], 1);
      mbar_init(&p_full[t], 4);   // one arrival per softmax warp
      mbar_init(&pv_done[t], 1);
    }
    mbar_init(drain, 1);
    mbar_init(&stage_bar[0], 4);
    mbar_init(&stage_bar[1], 4);
    // a CTA that starts after another one gave up does no work at all
    *abort_flag = (*reinterpret_cast<volatile int*>(args.status) != 0) ? 1 : 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (*abort_flag) return;
  if (warp == 9) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp >= 8) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;\n" ::"n"(kTcControlRegs) : "memory");
    if (warp == 8 && lane == 0) {
      // ------------------------------ TMA producer ------------------------------
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      mbar_arrive_expect_tx(q_full, 2 * QKB);
      for (int t = 0; t < 2; ++t) {
        if (kQ8) {
          tma_load_3d(sQ + t * QKB, &tmQ, q_full, 0, (qt0 + t) * kTile, bh);
        } else {
          for (int p = 0; p < S::kPanels; ++p)
            tma_load_3d(sQ + t * TB + p * S::kPanelBytes, &tmQ, q_full, p * 64, (qt0 + t) * kTile, bh);
        }
      }
      int issued = 0;
      for (int i = 0; i < 2 * nk; ++i) {
        const int slot = i % NS;
        const uint32_t ph = (uint32_t)(i / NS) & 1u;
        if (!mbar_wait(&kv_empty[slot], ph ^ 1u, abort_flag, kWaitLimitNs)) break;
        if (kQ8 && !(i & 1)) {
          mbar_arrive_expect_tx(&kv_full[slot], QKB);
          tma_load_3d(sKV + slot * TB, &tmK, &kv_full[slot], 0, (i >> 1) * kTile, bh);
        } else {
          mbar_arrive_expect_tx(&kv_full[slot], TB);
          const CUtensorMap* map = (i & 1) ? &tmV : &tmK;
          for (int p = 0; p < S::kPanels; ++p)
            tma_load_3d(sKV + slot * TB + p * S::kPanelBytes, map, &kv_full[slot], p * 64,
                        (i >> 1) * kTile, bh);
        }
        issued = i + 1;
      }
      if (*abort_flag) {
        // let the copies already issued land before the CTA's shared memory is released
        volatile int no_abort = 0;
        mbar_wait(q_full, 0, &no_abort, kDrainLimitNs);
        for (int i = issued - NS < 0 ? 0 : issued - NS; i < issued; ++i)
          mbar_wait(&kv_full[i % NS], (uint32_t)(i / NS) & 1u, &no_abort, kDrainLimitNs);
      }
    } else if (warp == 9 && lane == 0) {
      // ------------------------------ MMA issuer --------------------------------
      constexpr uint32_t idesc_qk = kQ8 ? make_idesc_s8(128, 128) : make_idesc_f16(128, 128, kBF16, false);
      constexpr uint32_t idesc_pv = make_idesc_f16(128, D, kBF16, true);
      const uint32_t sQa = smem_u32(sQ), sKVa = smem_u32(sKV);
      // base descriptors; a byte offset moves the start-address field by offset >> 4 (shared
      // addresses stay below 2^18, so the 14-bit field never carries)
      const uint64_t qd0 = make_sdesc_sw128(sQa, 16, 1024);
      const uint64_t kd0 = make_sdesc_sw128(sKVa, 16, 1024);
      const uint64_t vd0 = make_sdesc_sw128(sKVa, S::kPanelBytes, 1024);
      bool ok = mbar_wait(q_full, 0, abort_flag, kWaitLimitNs);
      tc_fence_after();
      for (int j = 0; ok && j <= nk; ++j) {
        const int ki = 2 * j, kslot = ki % NS;
        if (j < nk) {
          if (!(ok = mbar_wait(&kv_full[kslot], (uint32_t)(ki / NS) & 1u, abort_flag, kWaitLimitNs))) break;
          tc_fence_after();
        }
        for (int t = 0; t < 2 && ok; ++t) {
          if (j > 0) {
            const int vi = 2 * (j - 1) + 1, vslot = vi % NS;
            if (t == 0) {
              if (!(ok = mbar_wait(&kv_full[vslot], (uint32_t)(vi / NS) & 1u, abort_flag, kWaitLimitNs))) break;
            }
            if (!(ok = mbar_wait(&p_full[t], (uint32_t)(j - 1) & 1u, abort_flag, kWaitLimitNs))) break;
            tc_fence_after();
            const uint32_t d_o = tmem + S::kColO + t * D;
            const uint32_t a_p = tmem + S::kColS + t * 128 + S::kColP;
            const uint64_t vd = vd0 + (uint64_t)((vslot * TB) >> 4);
#pragma unroll
            for (int kk = 0; kk < kTile / 16; ++kk)
              umma_ts(d_o, a_p + kk * 8, vd + (uint64_t)((kk * 2048) >> 4), idesc_pv,
                      (j > 1 || kk > 0) ? 1u : 0u);
          }
          if (j < nk) {
            const uint32_t d_s = tmem + S::kColS + t * 128;
            const uint64_t qd = qd0 + (uint64_t)((t * QKB) >> 4);
            const uint64_t kd = kd0 + (uint64_t)((kslot * TB) >> 4);
            if (kQ8) {
              // 32 one-byte codes per instruction: K-steps of 32 bytes along the single panel
#pragma unroll
              for (int kk = 0; kk < D / 32; ++kk)
                umma_ss_i8(d_s, qd + (uint64_t)((kk * 32) >> 4), kd + (uint64_t)((kk * 32) >> 4),
                           idesc_qk, kk > 0 ? 1u : 0u);
            } else {
#pragma unroll
              for (int kk = 0; kk < D / 16; ++kk) {
                const uint64_t off = (uint64_t)((((kk >> 2) * S::kPanelBytes) + (kk & 3) * 32) >> 4);
                umma_ss(d_s, qd + off, kd + off, idesc_qk, kk > 0 ? 1u : 0u);
              }
            }
            umma_commit(&s_full[t]);
          }
          // PV's completion and the V slot's release are committed after the next QK^T is
          // issued: a commit costs the issuing thread ~55 cycles, and here it is off the
          // P -> PV -> QK^T -> S path (the only waiters on pv_done waited for that QK^T
          // already, through s_full, or are the epilogue, where no QK^T follows)
          if (j > 0) {
            umma_commit(&pv_done[t]);
            if (t == 1) umma_commit(&kv_empty[(2 * (j - 1) + 1) % NS]);
          }
          if (j < nk && t == 1) umma_commit(&kv_empty[kslot]);
        }
      }
      // every MMA issued above completes before tensor memory is released
      umma_commit(drain);
      volatile int no_abort = 0;
      mbar_wait(drain, 0, &no_abort, kDrainLimitNs);
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;\n" ::"n"(kTcSoftmaxRegs) : "memory");
    // ------------------------------ softmax warps -------------------------------
    const int t = warp >> 2;            // query tile of this warpgroup
    const int wq = warp & 3;            // TMEM lane quarter
    const int r = wq * 32 + lane;       // row within the tile
    const int qtile = qt0 + t;
    const int row = qtile * kTile + r;
    const bool row_ok = (qtile < args.ntiles) && (row < N);
    const BiasParams& bp = args.bp;
    const int mset = args.per_branch_meta ? blockIdx.z : 0;
    const long long mtok = (long long)mset * args.meta_stride;
    const TileRec* recs = args.recs + (long long)mset * args.ntiles;
    const float4* kinfo = args.keyinfo + (long long)mset * args.ntiles * kTile;

    bool is_tgt = false;
    float t_q = 0.0f, m_q = 0.0f;
    if (row_ok) {
      is_tgt = args.seg[mtok + row] == kSegTarget;
      t_q = args.time_s[mtok + row];
      m_q = args.m[mtok + row];
    }
    // debug build: the plane exists and a target row's time and mask weight are finite
    TARA_DCHECK_RECORD(bh < args.B * args.H, args.status);
    TARA_DCHECK_RECORD(!is_tgt || (isfinite(t_q) && isfinite(m_q)), args.status);
    // logit scale in log2 units; with 8-bit Q/K it also carries the row's and the key tile's
    // dequantisation scales
    const float row_sl = kQ8 ? bp.scale_log2 * (row_ok ? args.q_scale[(long long)bh * N + row] : 0.0f)
                             : bp.scale_log2;
    const float* kscale = kQ8 ? args.k_scale + (long long)bh * args.ntiles : nullptr;
    float ks_next = kQ8 ? kscale[0] : 1.0f;
    // weights of the extra bindings for this row, one per Picture index (0 for index 0)
    float* wx = rowx + (t * kTile + r) * 17;
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
    const uint32_t tS = tmem + lane_off + S::kColS + t * 128;
    const uint32_t tP = tS + S::kColP;
    const uint32_t tO = tmem + lane_off + S::kColO + t * D;
    const float ninf = __int_as_float(0xff800000);
    float m_run = ninf, l_run = 0.0f;
    bool ok = true;

    uint32_t stage_phase = 0;
    TileRec kr_next = recs[0];
    for (int j = 0; j < nk; ++j) {
      const TileRec kr = kr_next;
      if (j + 1 < nk) kr_next = recs[j + 1];   // in flight while this tile is processed
      float sl = row_sl;
      if (kQ8) {
        // a zero scale (an all-zero Q row or K tile, whose codes are all 0) is raised to the
        // smallest normal float: valid logits stay exactly 0 and the -inf of masked columns
        // stays -inf instead of becoming 0 * -inf
        sl = fmaxf(row_sl * ks_next, 1.17549435e-38f);
        if (j + 1 < nk) ks_next = kscale[j + 1];
      }
      float cval;
      const int cls = classify_pair(qr, kr, bp, &cval);
      float rowb2 = 0.0f;
      if (is_tgt) {
        if (cls == kClsConstCap) rowb2 = cval * kLog2e;
        else if (cls == kClsRowGuide) rowb2 = -penalty_f32(fabsf(t_q - kr.tk_min), bp) * kLog2e;
        else if (cls == kClsConstPic)
          rowb2 = (bp.n_extra > 0 ? m_q * cval + wx[kr.single_pic & 15] : m_q * cval) * kLog2e;
      }
      float4* kb = kbuf + (t * 2 + (j & 1)) * kTile;
      if (cls == kClsFull) {
        // stage the tile's key records in shared memory (one coalesced load per thread, in
        // flight while S is computed); two buffers, so a warp one iteration ahead never
        // overwrites records another warp of the group still reads
        const int key = j * kTile + r;
        kb[r] = key < N ? kinfo[key] : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
        if (!(ok = warp_rendezvous(&stage_bar[t], stage_phase, abort_flag, kWaitLimitNs))) break;
      }
      if (!(ok = warp_wait(&s_full[t], (uint32_t)j & 1u, abort_flag, kWaitLimitNs))) break;
      tc_fence_after();
      uint32_t s[128];
      tmem_ld128(tS, s);
      tmem_ld_wait();
      reg_fence<128>(s);
      const int nv = (int)kr.nvalid;
      // 8-bit path: S holds s32 dot products of the codes, |S| <= 127 * 127 * 128 < 2^22.  On
      // full-width tiles without per-edge bias they stay integers: the row max is an integer
      // max, and the exponent loop converts them inside its FMA (the integer add places S in
      // the mantissa of 1.5 * 2^23, whose offset is folded into the FMA's addend).  Other
      // tiles are converted exactly up front.
      const bool s_int = kQ8 && nv == kTile && cls != kClsFull;
      if (kQ8 && !s_int) {
#pragma unroll
        for (int c = 0; c < 128; ++c) s[c] = __float_as_uint(i32_to_f32_small(s[c]));
      }
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
        mx = fmaf(s_int ? (float)row_max128_s32(s) : row_max128(s), sl, rowb2);
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
      // columns in pairs: one packed FMA forms both exponents, one packed add accumulates
      // both probabilities (two accumulators break the dependency chain)
      // integer S: x = (S + 1.5 * 2^23) * scl + (off - 1.5 * 2^23 * scl), the addend in one rounding
      const uint32_t s_add = s_int ? 0x4B400000u : 0u;
      const float off_x = s_int ? fmaf(-12582912.0f, scl, off) : off;
      const uint64_t scl2 = f32x2_pack(scl, scl), off2 = f32x2_pack(off_x, off_x);
      uint64_t lsum2[2] = {0ull, 0ull};
#pragma unroll
      for (int qtr = 0; qtr < 4; ++qtr) {
        // 32 columns at a time: their P (16 packed words) is stored while the next quarter
        // runs (a small P buffer leaves registers for more exponentials in flight)
        uint32_t pk[16];
#pragma unroll
        for (int c2 = 0; c2 < 32; c2 += 2) {
          const int c = qtr * 32 + c2;
          float x0, x1;
          f32x2_unpack(f32x2_fma(f32x2_pack_bits(s[c] + s_add, s[c + 1] + s_add), scl2, off2), x0, x1);
          const float p0 = ex2_approx(x0);
          const float p1 = ex2_approx(x1);
          lsum2[(c >> 1) & 1] = f32x2_add(lsum2[(c >> 1) & 1], f32x2_pack(p0, p1));
          pk[c2 >> 1] = pack_p<kBF16>(p0, p1);
        }
        tmem_st16(tP + qtr * 16, pk);
      }
      {
        float a0, a1;
        f32x2_unpack(f32x2_add(lsum2[0], lsum2[1]), a0, a1);
        l_run += a0 + a1;
      }
      if (j > 0 && warp_need) {
        // rescale this warp's O rows once the previous PV has landed
        if (!(ok = warp_wait(&pv_done[t], (uint32_t)(j - 1) & 1u, abort_flag, kWaitLimitNs))) break;
        tc_fence_after();
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
      }
      m_run = m_use;
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[t]);
    }

    // ------------------------------ epilogue ---------------------------------------
    if (ok && warp_wait(&pv_done[t], (uint32_t)(nk - 1) & 1u, abort_flag, kWaitLimitNs)) {
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
          for (int v = 0; v < 4; ++v) dst[v] = make_uint4(w[4 * v], w[4 * v + 1], w[4 * v + 2], w[4 * v + 3]);
        }
      }
      if (out_ok) args.LSE[(long long)bh * N + row] = (m_run + log2f(l_run)) * kLn2;
    }
    tc_fence_before();
  }

  __syncthreads();
  if (threadIdx.x == 0 && *abort_flag) atomicExch(args.status, 1);
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace tara
