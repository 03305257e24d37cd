// tara_common.cuh -- data shared by the kernels: rule parameters as the device sees them,
// per-tile summaries, per-key bias records, and the fp32 bias evaluation every kernel uses.
#pragma once

#include <cstdint>

namespace tara {

constexpr int kSegText = 0, kSegPicture = 1, kSegTarget = 2, kSegGuide = 3;
constexpr float kLog2e = 1.4426950408889634f;   // log2(e)
constexpr float kLn2 = 0.6931471805599453f;     // ln(2)
constexpr int kTile = 128;                       // tokens per tile (rows and keys)

// Device-side checks of the debug build (compiled with -DTARA_DEBUG=1): a failed check sets
// bit 1 of the device status word (tara_device_status then reports TARA_ERR_DEBUG_CHECK);
// nothing traps.  TARA_DCHECK is an expression that guards an access (the access is skipped
// when the check fails), TARA_DCHECK_RECORD a statement that only records.  The release
// build evaluates neither condition.
#if defined(TARA_DEBUG) && TARA_DEBUG
#define TARA_DCHECK(cond, status) ((cond) ? true : (atomicOr((status), 2), false))
#define TARA_DCHECK_RECORD(cond, status) \
  do {                                   \
    if (!(cond)) atomicOr((status), 2);  \
  } while (0)
#else
#define TARA_DCHECK(cond, status) true
#define TARA_DCHECK_RECORD(cond, status) ((void)0)
#endif

// The rule's parameters prepared on the host (double precision, then rounded once).
struct BiasParams {
  float window;        // free window (s)
  float inv_falloff;   // 1 / falloff
  float strength;
  float cap;
  float scale;         // softmax scale (natural units)
  float scale_log2;    // softmax scale * log2(e)
  float lng[16];       // ln(gain of Picture p), p = 0..15; 0 for p outside 1..9
  uint32_t lng_nz;     // bit p set when lng[p] != 0 for any binding
  int32_t n_extra;     // chained bindings beyond the first (0..3)
  uint32_t pad[2];
  float lng_x[3][16];  // ln(gain) of each extra binding
};

// Extra-binding masks as the kernels see them (token arrays like m, one per binding).
struct ExtraMasks {
  const float* m;      // binding k, set b, token i at m[k * stride + b * batch_stride + i]
  long long stride;
};

// Summary of one 128-token tile of the packed sequence (written by the tile-summary kernel).
struct __align__(16) TileRec {
  uint32_t segmask;    // bit s set when a valid token of role s is in the tile
  uint32_t picmask;    // bit p set when a PICTURE token with index p is in the tile
  float tq_min, tq_max;   // min / max time over TARGET tokens (+inf / -inf when none)
  float tk_min, tk_max;   // min / max time over GUIDE tokens  (+inf / -inf when none)
  uint32_t nvalid;     // tokens of the tile inside the sequence
  uint32_t single_pic; // p when every valid token is PICTURE with the same index p, else 0
};

// Per-key bias record (float4): x = time of a GUIDE key (else 0), y = ln(gain) of the first
// binding for a PICTURE key with a non-neutral gain in any binding (else 0), z = 1 for a GUIDE
// key (else 0), w = its Picture index (else 0).  The bias of the edge (TARGET row with time t
// and mask m, key) is then -z*penalty(|t - x|) + m*y (+ the row's extra-binding weight of
// Picture w), with no branch on the key's role.

// Tile-pair classes (per 128-row query tile x 128-key tile).
constexpr int kClsZero = 0;      // no edge of the pair is biased
constexpr int kClsConstCap = 1;  // every target-row x key edge carries exactly -cap
constexpr int kClsConstPic = 2;  // every target-row x key edge carries m_row * ln(gain_p)
constexpr int kClsFull = 3;      // evaluate the bias edge by edge
constexpr int kClsRowGuide = 4;  // every valid key is GUIDE at one time: -penalty per target row

// The temporal penalty in fp32: min(strength * (max(dt - window, 0) / falloff)^2, cap)
// ("TARA: Native Temporal Alignment for MiniMax H3 References", "The temporal rule").
// Every operation is monotone non-decreasing in dt, which the tile classifier relies on.
__host__ __device__ __forceinline__ float penalty_f32(float dt, const BiasParams& p) {
  float x = fmaxf(dt - p.window, 0.0f) * p.inv_falloff;
  float y = p.strength * (x * x);
  return fminf(y, p.cap);
}

// Class of the (query tile, key tile) pair from the two summaries.  Exact: a class other than
// kClsFull is returned only when the per-edge fp32 evaluation gives that value on every edge.
// *cval receives the constant bias (natural units) for the constant classes.
__device__ __forceinline__ int classify_pair(const TileRec& q, const TileRec& k,
                                             const BiasParams& p, float* cval) {
  *cval = 0.0f;
  if (!(q.segmask & (1u << kSegTarget))) return kClsZero;
  bool has_g = (k.segmask & (1u << kSegGuide)) != 0;
  bool has_p = (k.segmask & (1u << kSegPicture)) != 0 && (k.picmask & p.lng_nz) != 0;
  if (has_g) {
    float dt_max = fmaxf(q.tq_max - k.tk_min, k.tk_max - q.tq_min);
    if (penalty_f32(dt_max, p) == 0.0f) has_g = false;
  }
  if (!has_g && !has_p) return kClsZero;
  if (has_g && !has_p) {
    if (k.segmask == (1u << kSegGuide)) {
      float dt_min = fmaxf(0.0f, fmaxf(k.tk_min - q.tq_max, q.tq_min - k.tk_max));
      if (penalty_f32(dt_min, p) == p.cap) {
        *cval = -p.cap;
        return kClsConstCap;
      }
      // a key tile inside one guide frame: the bias depends on the query row only
      if (k.tk_min == k.tk_max) return kClsRowGuide;
    }
    return kClsFull;
  }
  if (has_p && !has_g && k.segmask == (1u << kSegPicture) && k.single_pic != 0) {
    *cval = p.lng[k.single_pic & 15];
    return kClsConstPic;
  }
  return kClsFull;
}

}  // namespace tara
